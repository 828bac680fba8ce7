// TQ4 split-K decode attention for one query token per request (sm_100a).
//
// Same computation as the general split-K kernel (rotated-domain attention over
// packed pages; [KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into 24 GiB
// of Laptop Memory", section "KVExec"; [V2] wpnews.pro "JustFit: Run Qwen 27B
// Fast ...", mechanism table row KVExec), organised so that warps never wait on
// each other inside the main loop:
//
//   * a CTA (8 warps) owns one (request, KV head, split); warp w takes the
//     32-position tiles w, w+8, w+16, ... of the split's full rounds of 256
//     positions; a last round of at most 128 positions is dealt out as 16-position
//     half tiles (one per warp), so every warp of a split of 256 r + 128 positions
//     does the same work;
//   * lane 0 of each warp streams its tiles with TMA (2D tensor loads of the
//     K and V word rows with the 128-byte swizzle, bulk copies of the two norm
//     rows) into a private two-stage ring, completion on an mbarrier;
//   * K phase: S = C_k (q'_hi + q'_lo) on mma.m16n8k16 for two m-tiles
//     (M = 16 positions, N = 6 query heads padded to 8, K = 256 dims);
//   * in-warp online softmax with lazy rescaling (the reference max is raised
//     only when a row max grows by more than 2^8); P' = p * n_v split into f16
//     hi + lo and moved into B-operand layout with movmatrix;
//   * V phase: O'^T += C_v^T P'^T over all 256 dims (M = dims, K = positions);
//   * at the end the 8 warp states (m, l, o') are merged through shared memory
//     and written as one split-K partial for the combine pass.
//   * 2- and 3-bit pools (kBits): the same kernel; lane 0 copies a tile's word rows
//     (64 or 96 B per position) and norms with plain bulk copies, and each lane
//     widens the plane words it loads into the nibble words of the four-bit layout,
//     so the table lookups, MMAs and softmax below are shared; the table holds the
//     b-bit codebook (codes never exceed 2^b - 1); the fused append encodes with
//     the b-bit quantiser and packing;
//   * fused append: in the CTA that owns a request's last position, warps 6 and 7
//     encode the new K and V vectors of this KV head (the append kernel's
//     arithmetic), store them in the pool and fence them for the tensor-copy
//     proxy; the warp whose tile holds that position issues that tile's TMA only
//     after both have arrived on an mbarrier (normally long before it gets there).
#pragma once
#include <cuda.h>
#include <type_traits>
#include "tq4_decode.cuh"
#include "tq4_encode.cuh"

namespace tq4 {

constexpr int kQ1Warps = 8;
constexpr int kQ1Threads = 32 * kQ1Warps;
constexpr int kQ1Tile = 32;                    // positions per warp iteration (two mma m-tiles)
constexpr int kQ1Stages = 2;                   // TMA ring depth per warp
constexpr int kQ1KV = kQ1Tile * 128;           // 4,096 B: one K (or V) tile, 128-B swizzled rows
constexpr int kQ1Buf = 2 * kQ1KV;              // K then V
constexpr int kQ1Bufs = kQ1Warps * kQ1Stages;  // 16 tile buffers
// Shared-window layout (absolute 32-bit shared addresses). The centroid table
// sits at 0x10000 so that one byte permute builds a lookup address
// (0x10000 | byte << 8 | lane * 4). Row `byte` (256 B) holds 32 copies of the
// byte's c16 pair, then 32 copies of its r16 pair: each lane reads its own copy,
// so a warp's 4-byte loads of either half hit 32 different banks, and a lookup
// that needs only the c16 pair costs one wavefront. Below the table: control
// words, q', mbarriers, norm rows and the first tile buffers; above it: the other
// tile buffers.
constexpr uint32_t kQ1Lut = 0x10000;
constexpr uint32_t kQ1Hi = 0x20000;
constexpr uint32_t kQ1QvOff = 128;
constexpr uint32_t kQ1BarOff = kQ1QvOff + 2 * 8 * kQvStride * 2;      // 8,576
constexpr uint32_t kQ1NrmOff = kQ1BarOff + 128;                        // 16 x 128 B of norm rows
constexpr uint32_t kQ1CtlBytes = kQ1NrmOff + kQ1Bufs * 128;           // 10,752
constexpr int kQ1LowBufs = 6;
constexpr uint32_t kQ1DynBytes = kQ1Hi + (kQ1Bufs - kQ1LowBufs) * kQ1Buf;   // 212,992
// merge area, per warp: 8 rows of o' with each 32-dim block padded to 36 floats and
// rows 292 floats apart (conflict-free float4 stores of the mma fragments and reads
// of row slices), then m[8], l[8]
constexpr int kQ1MrgBlk = 36, kQ1MrgRow = 8 * kQ1MrgBlk + 4, kQ1MrgWarp = 8 * kQ1MrgRow + 16;
constexpr int kQ1MergeBytes = kQ1Warps * kQ1MrgWarp * 4;
static_assert(kQ1MergeBytes <= (kQ1Bufs - kQ1LowBufs) * kQ1Buf, "merge area fits above the table");
static_assert(kQ1DynBytes <= 227 * 1024, "fits the per-CTA shared memory");
constexpr float kQ1PScale = 1.0f / 256.0f;   // P' = p * n_v / 256 (undone when the partial is written)
constexpr float kQ1Lazy = 8.0f;              // rescale only when a row max grows by > 2^8 (log2 units)
constexpr uint32_t kQ1DrainPolls = TQ4_DEFAULT_WAIT_POLLS;  // drain of a copy still in flight at exit

constexpr size_t decode_q1_smem_bytes() { return kQ1DynBytes; }

// MMA row m (0..15) of an m-tile holds tile-local position sigma(m & 7) + (m & 8):
// with the 128-B swizzle (16-B chunk index XOR row & 7) this makes the K-phase
// and V-phase shared loads conflict-free.
__host__ __device__ constexpr int q1_sigma(int m) {
  return ((0x37156240u >> (4 * (m & 7))) & 7) + (m & 8);
}
// The b-bit pools' rows are 64 or 96 B (no swizzle): with sigma = [0,1,2,3,5,4,7,6]
// the 8-byte plane-0 loads of both phases are conflict-free for 96-B rows (each
// half warp meets four rows whose bank offsets 24 r mod 32 differ) and 2-way for
// 64-B rows (two offsets only).
template <int kBits>
__host__ __device__ constexpr int q1_sigma_b(int m) {
  return kBits == 4 ? q1_sigma(m) : ((0x67453210u >> (4 * (m & 7))) & 7) + (m & 8);
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint16_t ld_shared_u16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.b16 %0, [%1];\n" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void st_shared_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a), "r"(v) : "memory");
}
// byte K of w -> the hi (c16) and lo (r16) f16x2 centroid pairs from the table at
// kQ1Lut (lanebase = kQ1Lut | 4 * lane: one byte permute forms the address)
template <int K>
__device__ __forceinline__ uint32_t lut_addr(uint32_t w, uint32_t lanebase) {
  constexpr uint32_t sel = (7u << 12) | (6u << 8) | (uint32_t(K) << 4) | 4u;
  return __byte_perm(w, lanebase, sel);
}
template <int K>
__device__ __forceinline__ void lut64k(uint32_t w, uint32_t lanebase, uint32_t& hi, uint32_t& lo) {
  const uint32_t a = lut_addr<K>(w, lanebase);
  hi = ld_shared_u32(a);
  lo = ld_shared_u32(a + 128);
}
template <int K>
__device__ __forceinline__ uint32_t lut64k_hi(uint32_t w, uint32_t lanebase) {
  return ld_shared_u32(lut_addr<K>(w, lanebase));
}
// byte K of four words -> four A-fragment registers (hi), and their lo pairs when kLo
template <int K, bool kLo>
__device__ __forceinline__ void lut4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t lanebase,
                                     uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3, uint32_t& r0,
                                     uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  if constexpr (kLo) {
    lut64k<K>(w0, lanebase, a0, r0);
    lut64k<K>(w1, lanebase, a1, r1);
    lut64k<K>(w2, lanebase, a2, r2);
    lut64k<K>(w3, lanebase, a3, r3);
  } else {
    a0 = lut64k_hi<K>(w0, lanebase);
    a1 = lut64k_hi<K>(w1, lanebase);
    a2 = lut64k_hi<K>(w2, lanebase);
    a3 = lut64k_hi<K>(w3, lanebase);
  }
}

// ---- mbarrier and bulk-copy primitives (one CTA = its own cluster; no multicast)
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ void mbar_arrive_q1(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// The pool seen by the tensor map: rows of 128 B (32 u32), 2,080 rows per page:
// K words (4 heads x 256 slots), V words, then 32 rows of norms.
constexpr int kRowsPerPage = int(kPageBytes / 128);   // 2,080

// Nibble words 4i .. 4i + 3 (dims 32i .. 32i + 31) of one position of a b-bit pool,
// from its staged row at `row`: plane-0 words 2i, 2i + 1 widened to the low two
// bits of each nibble and, with 3 bits, byte m of plane-1 word 16 + i as bit 2 of
// nibble word 4i + m.
template <int kBits>
__device__ __forceinline__ uint4 widen_words32(uint32_t row, int i) {
  uint32_t a, b;
  ld_shared_v2(row + 8 * i, a, b);
  uint4 r = make_uint4(widen2(a), widen2_hi(a), widen2(b), widen2_hi(b));
  if constexpr (kBits == 3) {
    const uint32_t hb = ld_shared_u32(row + 64 + 4 * i);
    r.x |= widen1_bit2<0>(hb);
    r.y |= widen1_bit2<1>(hb);
    r.z |= widen1_bit2<2>(hb);
    r.w |= widen1_bit2<3>(hb);
  }
  return r;
}

// kExact: fp32 outputs, C_lo P' on every tile (see kVloNorm). kBits: 4 (TQ4 pool,
// tiles by tensor copies through tmap), or 2 / 3 (b-bit pools, tmap unused).
template <bool kExact, int kBits = 4>
__global__ void __launch_bounds__(kQ1Threads, 1)
    decode_q1_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap) {
  static_assert(kBits == 4 || kBits == 2 || kBits == 3, "bit width");
  constexpr uint32_t kRB = uint32_t(tqb_row_bytes<kBits>());   // bytes of a staged word row: 32 b
  static_assert(kQ1Tile * kRB <= uint32_t(kQ1KV), "a tile's word rows fit their half of the buffer");
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const uint32_t low0 = (base + kQ1CtlBytes + 1023) & ~1023u;
  if (low0 + kQ1LowBufs * kQ1Buf > kQ1Lut) {   // the layout needs the dynamic window to start low
    if (tid == 0) record_error(p.status, TQ4_ERR_CUDA);
    return;
  }
  int* s_item = reinterpret_cast<int*>(smem);
  __half* qv_hi = reinterpret_cast<__half*>(smem + kQ1QvOff);
  __half* qv_lo = qv_hi + 8 * kQvStride;
  auto buf_addr = [&](int b) { return b < kQ1LowBufs ? low0 + b * kQ1Buf : kQ1Hi + (b - kQ1LowBufs) * kQ1Buf; };
  const uint32_t lanebase = kQ1Lut | (uint32_t(lane) * 4u);

  // prologue that reads none of the call's inputs (overlaps the previous kernel)
  const uint32_t bar_new = base + 8;   // the fused append's new position is in the pool (count 2)
  if (tid < kQ1Bufs) mbar_init(base + kQ1BarOff + tid * 8, 1);
  if (tid == kQ1Bufs) mbar_init(bar_new, 2);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  // table rows: 32 copies of the c16 pair, then 32 copies of the r16 pair (16-B stores of 4 copies)
  for (int e = tid; e < 256 * 16; e += kQ1Threads) {
    uint2 v;
    if constexpr (kBits == 4) v = lut_row(e >> 4);
    else v = lut_row_bits<kBits>(e >> 4);
    const uint32_t x = (e & 8) ? v.y : v.x;
    asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};\n" ::"r"(kQ1Lut + (e >> 4) * 256 + (e & 15) * 16), "r"(x)
                 : "memory");
  }
  __syncthreads();   // barriers initialised before any warp arms one
  pdl_wait();
  pdl_launch_dependents();
  // (request, split) of this CTA: with one request it is (0, blockIdx.x); otherwise
  // warp 0 scans the lengths
  int r = 0, split = int(blockIdx.x);
  if (p.n_req > 1) {
    if (w == 0) {
      int req = 0, sp = 0, total = 0;
      const bool ok = find_item(p, blockIdx.x, req, sp, total);
      if (lane == 0) {
        s_item[0] = ok ? req : -1;
        s_item[1] = sp;
        if (blockIdx.x == 0 && h == 0 && total > p.items_ub) record_error(p.status, TQ4_ERR_SEQ);
      }
      if (blockIdx.x == 0 && h == 0) {   // a length the page table cannot hold: no output for that request
        bool bad = false;
        for (int rr = lane; rr < p.n_req; rr += 32) bad |= !seq_ok(__ldg(p.seq_lens + rr), p.n_q, p.max_pages);
        if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(p.status, TQ4_ERR_SEQ);
      }
    }
    __syncthreads();
    r = s_item[0];
    split = s_item[1];
    if (r < 0 || int(blockIdx.x) >= p.items_ub) return;
  }
  const int32_t* table = p.page_tables + int64_t(r) * p.max_pages;
  const int pos_b = split * p.split_len;
  // independent loads go out together: the length, this warp's first page id
  // (speculative, inside the table: its first tile starts at 32 w, or at 16 w when
  // the split is a single half round) and this warp's query row
  const int seq_len = __ldg(p.seq_lens + r);
  const int c_full = pos_b + w * kQ1Tile, c_half = pos_b + w * (kQ1Tile / 2);
  const int32_t page_full = (c_full >> 8) < p.max_pages ? __ldg(table + (c_full >> 8)) : -1;
  const int32_t page_half = (c_half >> 8) < p.max_pages ? __ldg(table + (c_half >> 8)) : -1;
  uint4 qraw = make_uint4(0, 0, 0, 0);
  if (w < kGroup)
    qraw = __ldg(reinterpret_cast<const uint4*>(p.q + (int64_t(r) * kHq + h * kGroup + w) * kD + lane * 8));
  if (p.n_req == 1) {
    const bool len_ok = seq_ok(seq_len, p.n_q, p.max_pages);
    const int S = len_ok ? (seq_len + p.split_len - 1) / p.split_len : 0;
    if (tid == 0 && blockIdx.x == 0 && h == 0 && (!len_ok || S > p.items_ub)) record_error(p.status, TQ4_ERR_SEQ);
    if (split >= S || split >= p.items_ub) return;   // the same decision in every thread of the CTA
  }
  const int pos_e = min(pos_b + p.split_len, seq_len);
  // Tiles: full rounds of 8 x 32 positions (warp w takes the w-th tile of each), then
  // the remainder: at most 128 positions as eight 16-position half tiles, else as
  // eight 32-position tiles (masked past pos_e).
  const int n_pos = pos_e - pos_b;
  const int rounds = n_pos >> 8, rem = n_pos & 255;
  const bool half_round = rem > 0 && rem <= 128;
  const int chunk = half_round ? kQ1Tile / 2 : kQ1Tile;
  const int my_tiles = rounds + ((rem > 0 && chunk * w < rem) ? 1 : 0);
  const int32_t page_first = (rounds == 0 && half_round) ? page_half : page_full;
  // fused append: this CTA holds the request's last position (seq_len - 1)
  const bool append_here = p.pool_w != nullptr && pos_e == seq_len && pos_b < pos_e;
  // warp 6: K, warp 7: V of KV head h. The input row is loaded early (fused_load);
  // the encode, the store and the release to the tile's TMA follow (fused_encode).
  float x_new[8];
  auto fused_load = [&]() {
    const int kv = w - (kQ1Warps - 2);
    const void* src = kv ? p.v_new : p.k_new;
    if (p.new_dtype == TQ4_DTYPE_F32)
      load8<float>(static_cast<const float*>(src) + (int64_t(r) * kHkv + h) * kD + lane * 8, x_new);
    else
      load8<uint16_t>(static_cast<const uint16_t*>(src) + (int64_t(r) * kHkv + h) * kD + lane * 8, x_new);
  };
  auto fused_encode = [&]() {
    const int kv = w - (kQ1Warps - 2);
    float nrm;
    if constexpr (kBits == 4) {
      const uint32_t word = encode_vector_warp(x_new, p.signs, nrm);
      store_packed_warp(p.pool_w, p.num_pages, table, seq_len - 1, h, kv, word, nrm, p.status);
    } else {
      uint32_t w0, w1;
      encode_bits_warp<kBits>(x_new, p.signs, w0, w1, nrm);
      store_bits_warp<kBits>(p.pool_w, p.num_pages, table, seq_len - 1, h, kv, w0, w1, nrm, p.status);
    }
    asm volatile("fence.proxy.async.global;\n" ::: "memory");   // generic stores -> the tile copies below
    __syncwarp();
    if (lane == 0) mbar_arrive_q1(bar_new);
  };
  const int p_last = n_pos - 1;   // split-relative position of the last one
  const int last_w = p_last < rounds * 256 ? (p_last >> 5) & (kQ1Warps - 1) : (p_last - rounds * 256) / chunk;
  const int last_k = p_last < rounds * 256 ? (p_last >> 8) : rounds;
  const bool encoder = append_here && w >= kQ1Warps - 2;
  // When the tile with the new position is its owner's first tile, its TMA is issued
  // before the block-wide barrier below, so the encode must precede that barrier;
  // otherwise it follows it and delays no warp.
  const bool encode_first = encoder && last_k == 0;

  // ---- lane 0 of each warp streams the warp's tiles: tile k -> buffer w*2 + k%2
  auto tile_pos = [&](int k) {
    return pos_b + (k < rounds ? (w + k * kQ1Warps) * kQ1Tile : rounds * 256 + chunk * w);
  };
  auto tile_half = [&](int k) { return half_round && k == rounds; };
  // page id of tile k of this warp, loaded one iteration before its copy is issued
  // (a tile never straddles a page); -1 past the table
  auto tile_page = [&](int k) -> int32_t {
    const int c = tile_pos(k);
    return (k < my_tiles && (c >> 8) < p.max_pages) ? __ldg(table + (c >> 8)) : -1;
  };
  // (test hook: the first tile's copy is withheld, so the wait on it runs out)
  auto issue_tile = [&](int k, int32_t page) {
    if (lane == 0 && k < my_tiles && !(p.test_withhold && k == 0)) {
      const int c = tile_pos(k);
      const int b = w * kQ1Stages + (k % kQ1Stages);
      const uint32_t bar = base + kQ1BarOff + b * 8;
      if (append_here && w == last_w && k == last_k) {   // the tile with the appended position
        uint32_t spins = 0;
        while (!mbar_try_wait(bar_new, 0) && ++spins < p.spin_limit) {
        }
        if (spins >= p.spin_limit) record_error(p.status, TQ4_ERR_TIMEOUT);
      }
      if (page < 0 || page >= p.num_pages) {
        record_error(p.status, TQ4_ERR_PAGE_RANGE);
        page = 0;   // still complete the barrier (reading page 0); the call's output is then
                    // undefined and the status word reports the page
      }
      const int slot0 = h * kPage + (c & (kPage - 1));
      const uint32_t kdst = buf_addr(b), ndst = base + kQ1NrmOff + b * 128;
      const uint32_t nbytes = tile_half(k) ? kQ1Tile : 2 * kQ1Tile;
      if constexpr (kBits == 4) {
        const int row = page * kRowsPerPage + slot0;
        const uint8_t* pg = p.pool + int64_t(page) * kPageBytes;
        // A half tile still takes 32-row word boxes (the extra rows stay inside the
        // page: at most row 2,063 of its 2,080) but only its own 16 norms, since the
        // V norms end the page.
        mbar_expect_tx(bar, 2 * kQ1KV + 2 * nbytes);
        tma_load_2d(kdst, &tmap, 0, row, bar);                       // K words of 32 positions
        tma_load_2d(kdst + kQ1KV, &tmap, 0, row + 4 * kPage, bar);   // V words
        bulk_load(ndst, pg + kKNorms + slot0 * 2, nbytes, bar);
        bulk_load(ndst + 64, pg + kVNorms + slot0 * 2, nbytes, bar);
      } else {
        // b-bit pool: a tile's rows are contiguous (slot0 is a multiple of 16, so
        // every source is 16-byte aligned); a half tile copies its 16 rows only
        const uint8_t* pg = p.pool + int64_t(page) * tqb_page_bytes<kBits>();
        const uint32_t wbytes = (tile_half(k) ? kQ1Tile / 2 : kQ1Tile) * kRB;
        mbar_expect_tx(bar, 2 * wbytes + 2 * nbytes);
        bulk_load(kdst, pg + int64_t(slot0) * kRB, wbytes, bar);
        bulk_load(kdst + kQ1KV, pg + tqb_v_words<kBits>() + int64_t(slot0) * kRB, wbytes, bar);
        bulk_load(ndst, pg + tqb_k_norms<kBits>() + slot0 * 2, nbytes, bar);
        bulk_load(ndst + 64, pg + tqb_v_norms<kBits>() + slot0 * 2, nbytes, bar);
      }
    }
  };
  if (encoder) fused_load();
  if (encode_first) fused_encode();
  issue_tile(0, page_first);
  int32_t page_next = tile_page(1);

  // ---- q' = R q * scale for the 6 query heads of this KV head, split hi + lo, virtual order
  {
    const int row = w;
    float v[8];
    if (row < 6) {
      const uint32_t ww[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(ww[i] << 16) * sign_of(p.signs, lane * 8 + 2 * i);
        v[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u) * sign_of(p.signs, lane * 8 + 2 * i + 1);
      }
      warp_fwht256(v);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= p.scale * 0.0625f;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    const int tt = (lane & 15) >> 2, wsel = (lane & 3) + 4 * (lane >> 4);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int kk = 2 * wsel + (i >> 2);
      const int col = kk * 16 + ((i >> 1) & 1) * 8 + 2 * tt;
      const __half2 hi = __floats2half2_rn(v[i], v[i + 1]);
      const float2 hfl = __half22float2(hi);
      *reinterpret_cast<__half2*>(qv_hi + row * kQvStride + col) = hi;
      *reinterpret_cast<__half2*>(qv_lo + row * kQvStride + col) = __floats2half2_rn(v[i] - hfl.x, v[i + 1] - hfl.y);
    }
  }
  __syncthreads();
  if (encoder && !encode_first) fused_encode();   // after the block-wide barrier: no warp waits for it

  // q'_hi B fragments stay in registers; the q'_lo fragments are read from shared
  // memory two k-steps at a time inside the K phase (registers are the limit)
  uint32_t qh[16][2];
  const int qfrag_off = (lane & 7) * kQvStride + ((lane >> 4) & 1) * 16 + ((lane >> 3) & 1) * 8;
  const uint32_t ql_addr = smem_u32(qv_lo + qfrag_off);
#pragma unroll
  for (int kk = 0; kk < 16; kk += 2)
    ldmatrix_x4(qh[kk][0], qh[kk][1], qh[kk + 1][0], qh[kk + 1][1], smem_u32(qv_hi + qfrag_off + kk * 16));

  const bool row_ok0 = 2 * t < 6, row_ok1 = 2 * t + 1 < 6;   // query heads 2t, 2t+1
  float m_ref[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int mt = 0; mt < 16; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;

  // positions of this lane: K phase rows g, g+8 -> sigma; V phase k-indices 2t, 2t+1 (+8)
  const int pk = q1_sigma_b<kBits>(g);               // and pk + 8 (same swizzle phase)
  const int pv0 = q1_sigma_b<kBits>(2 * t), pv1 = q1_sigma_b<kBits>(2 * t + 1);
  const uint32_t k_off0 = pk * 128 + ((t ^ (pk & 7)) << 4);          // words 4t..4t+3
  const uint32_t k_off1 = pk * 128 + (((4 + t) ^ (pk & 7)) << 4);    // words 16+4t..16+4t+3
  const uint32_t v_off0 = pv0 * 128 + ((g ^ (pv0 & 7)) << 4);        // words 4g..4g+3 of position pv0
  const uint32_t v_off1 = pv1 * 128 + ((g ^ (pv1 & 7)) << 4);
  bool timed_out = false;
  int k_stop = my_tiles;   // first tile not consumed (a timeout stops the walk early)

  for (int k = 0; k < my_tiles; ++k) {
    issue_tile(k + 1, page_next);
    page_next = tile_page(k + 2);   // used by the next iteration's copy
    const int b = w * kQ1Stages + (k % kQ1Stages);
    const uint32_t bar = base + kQ1BarOff + b * 8;
    {
      uint32_t spins = 0;
      while (!mbar_try_wait(bar, (k / kQ1Stages) & 1)) {
        if (++spins > p.spin_limit) { timed_out = true; break; }
      }
      if (__any_sync(0xffffffffu, timed_out)) {
        if (lane == 0) record_error(p.status, TQ4_ERR_TIMEOUT);
        k_stop = k;
        break;
      }
    }
    const uint32_t kst = buf_addr(b), vst = kst + kQ1KV;
    const uint32_t nb = base + kQ1NrmOff + b * 128;
    const int c = tile_pos(k);
    const bool two = !tile_half(k);   // warp-uniform: m-tile 1 exists (a half tile has m-tile 0 only)

    // ------------------------------------------------------------ K phase, two m-tiles
    uint4 ka[2], kb4[2], kc[2], kd[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j == 1 && !two) {
        ka[1] = kb4[1] = kc[1] = kd[1] = make_uint4(0, 0, 0, 0);
        break;
      }
      if constexpr (kBits == 4) {
        const uint32_t mrow = kst + j * 16 * 128;
        ka[j] = ld_shared_v4(mrow + k_off0);
        kb4[j] = ld_shared_v4(mrow + k_off1);
        kc[j] = ld_shared_v4(mrow + 8 * 128 + k_off0);
        kd[j] = ld_shared_v4(mrow + 8 * 128 + k_off1);
      } else {   // the same nibble words, widened from positions pk, pk + 8
        const uint32_t r0 = kst + (16 * j + pk) * kRB, r8 = r0 + 8 * kRB;
        ka[j] = widen_words32<kBits>(r0, t);
        kb4[j] = widen_words32<kBits>(r0, 4 + t);
        kc[j] = widen_words32<kBits>(r8, t);
        kd[j] = widen_words32<kBits>(r8, 4 + t);
      }
    }
    // S = (C_hi + C_lo)(q'_hi + q'_lo) less C_lo q'_lo: sc = C_hi q'_hi, sd = C_hi q'_lo,
    // se = C_lo q'_hi (three accumulators: three independent chains of 16 MMAs)
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float sd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float se[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    uint32_t ql4[4];
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      if ((kk & 1) == 0) ldmatrix_x4(ql4[0], ql4[1], ql4[2], ql4[3], ql_addr + kk * 32);
      const uint32_t ql0 = ql4[2 * (kk & 1)], ql1 = ql4[2 * (kk & 1) + 1];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (j == 1 && !two) break;
        const uint32_t wg = pick(ka[j], kb4[j], kk >> 1);
        const uint32_t wg8 = pick(kc[j], kd[j], kk >> 1);
        uint32_t a0, a1, a2, a3, r0, r1, r2, r3;
        if (kk & 1) {
          lut64k<2>(wg, lanebase, a0, r0); lut64k<2>(wg8, lanebase, a1, r1);
          lut64k<3>(wg, lanebase, a2, r2); lut64k<3>(wg8, lanebase, a3, r3);
        } else {
          lut64k<0>(wg, lanebase, a0, r0); lut64k<0>(wg8, lanebase, a1, r1);
          lut64k<1>(wg, lanebase, a2, r2); lut64k<1>(wg8, lanebase, a3, r3);
        }
        mma_16816(sc[j], a0, a1, a2, a3, qh[kk][0], qh[kk][1]);
        mma_16816(sd[j], a0, a1, a2, a3, ql0, ql1);
        mma_16816(se[j], r0, r1, r2, r3, qh[kk][0], qh[kk][1]);
      }
    }

    // ------------------------------------------------------------ online softmax over 32 positions
    float s[2][4], kn[2][2], vn[2][2];
    bool vbig = false;   // a visible position of this lane has a V norm above kVloNorm
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = 16 * j + pk + 8 * e;
        kn[j][e] = __half2float(__ushort_as_half(ld_shared_u16(nb + 2 * pos)));
        vn[j][e] = __half2float(__ushort_as_half(ld_shared_u16(nb + 64 + 2 * pos))) * kQ1PScale;
        const bool ok = (j == 0 || two) && c + pos < pos_e;
        vbig |= ok && vn[j][e] > kVloNorm * kQ1PScale;
        s[j][2 * e] = (ok && row_ok0) ? (sc[j][2 * e] + (sd[j][2 * e] + se[j][2 * e])) * kn[j][e] * kLog2e : -INFINITY;
        s[j][2 * e + 1] = (ok && row_ok1) ? (sc[j][2 * e + 1] + (sd[j][2 * e + 1] + se[j][2 * e + 1])) * kn[j][e] * kLog2e : -INFINITY;
      }
    // Lazy reference: a row's reference is raised only when the row max exceeds it by
    // more than 2^8. Each lane first tests its own scores; the row maxima (shuffles)
    // are formed only in the rare tiles where some lane needs a raise.
    float lmax[2];
    bool need = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {   // e: row 2t+e
      lmax[e] = fmaxf(fmaxf(s[0][e], s[0][e + 2]), fmaxf(s[1][e], s[1][e + 2]));
      need |= lmax[e] > m_ref[e] + kQ1Lazy;
    }
    if (__any_sync(0xffffffffu, need)) {
      float alpha[2] = {1.f, 1.f};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = lmax[e];
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        if (v > m_ref[e] + kQ1Lazy) {           // weights would exceed 2^8
          alpha[e] = fast_exp2(m_ref[e] - v);   // 0 on the first raise (m_ref = -inf)
          m_ref[e] = v;
        }
      }
      l_part[0] *= alpha[0];
      l_part[1] *= alpha[1];
#pragma unroll
      for (int mt = 0; mt < 16; ++mt) {
        o[mt][0] *= alpha[0];
        o[mt][1] *= alpha[1];
        o[mt][2] *= alpha[0];
        o[mt][3] *= alpha[1];
      }
    }
    const float mu0 = m_ref[0] == -INFINITY ? 0.f : m_ref[0];
    const float mu1 = m_ref[1] == -INFINITY ? 0.f : m_ref[1];
    uint32_t bh[2][2], bl[2][2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float pw[4];
      pw[0] = fast_exp2(s[j][0] - mu0);
      pw[1] = fast_exp2(s[j][1] - mu1);
      pw[2] = fast_exp2(s[j][2] - mu0);
      pw[3] = fast_exp2(s[j][3] - mu1);
      l_part[0] += pw[0] + pw[2];
      l_part[1] += pw[1] + pw[3];
      // P' = p * n_v / 256 (zero where masked, so stale norms never enter), f16 hi + lo,
      // transposed into B fragments (k index = mma row = position sigma(row))
      const float w0 = s[j][0] == -INFINITY ? 0.f : pw[0] * vn[j][0];
      const float w1 = s[j][1] == -INFINITY ? 0.f : pw[1] * vn[j][0];
      const float w2 = s[j][2] == -INFINITY ? 0.f : pw[2] * vn[j][1];
      const float w3 = s[j][3] == -INFINITY ? 0.f : pw[3] * vn[j][1];
      const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(w0 - f01.x, w1 - f01.y);
      const __half2 l23 = __floats2half2_rn(w2 - f23.x, w3 - f23.y);
      bh[j][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
      bh[j][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
      bl[j][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&l01));
      bl[j][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&l23));
    }

    // ------------------------------------------------------------ V phase (all 256 dims), two k-steps
    // O'^T += (C_hi + C_lo)^T (P'_hi + P'_lo) less C_lo P'_lo; with bf16 outputs
    // without C_lo on tiles whose V norms are all small (kVloNorm), where only the
    // c16 halves of the table are read
    auto v_phase = [&](auto lo_tag) {
    constexpr bool kLo = decltype(lo_tag)::value;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j == 1 && !two) break;   // a half tile's positions 16-31 carry P' = 0
      uint4 x0, x1, y0, y1;
      if constexpr (kBits == 4) {
        const uint32_t vrow = vst + j * 16 * 128;
        x0 = ld_shared_v4(vrow + v_off0);              // position sigma(2t)
        x1 = ld_shared_v4(vrow + v_off1);              // position sigma(2t+1)
        y0 = ld_shared_v4(vrow + 8 * 128 + v_off0);    // +8
        y1 = ld_shared_v4(vrow + 8 * 128 + v_off1);
      } else {   // nibble words 4g .. 4g + 3 of the same positions
        const uint32_t vrow = vst + 16 * j * kRB;
        x0 = widen_words32<kBits>(vrow + pv0 * kRB, g);
        x1 = widen_words32<kBits>(vrow + pv1 * kRB, g);
        y0 = widen_words32<kBits>(vrow + (pv0 + 8) * kRB, g);
        y1 = widen_words32<kBits>(vrow + (pv1 + 8) * kRB, g);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t lo01, hi01, lo89, hi89;
        interleave_nibbles(pick(x0, x0, q), pick(x1, x1, q), lo01, hi01);
        interleave_nibbles(pick(y0, y0, q), pick(y1, y1, q), lo89, hi89);
#pragma unroll
        for (int kb_ = 0; kb_ < 4; ++kb_) {
          uint32_t a0, a1, a2, a3, r0 = 0, r1 = 0, r2 = 0, r3 = 0;
          switch (kb_) {
            case 0: lut4<0, kLo>(lo01, hi01, lo89, hi89, lanebase, a0, a1, a2, a3, r0, r1, r2, r3); break;
            case 1: lut4<1, kLo>(lo01, hi01, lo89, hi89, lanebase, a0, a1, a2, a3, r0, r1, r2, r3); break;
            case 2: lut4<2, kLo>(lo01, hi01, lo89, hi89, lanebase, a0, a1, a2, a3, r0, r1, r2, r3); break;
            default: lut4<3, kLo>(lo01, hi01, lo89, hi89, lanebase, a0, a1, a2, a3, r0, r1, r2, r3); break;
          }
          mma_16816(o[4 * q + kb_], a0, a1, a2, a3, bh[j][0], bh[j][1]);
          mma_16816(o[4 * q + kb_], a0, a1, a2, a3, bl[j][0], bl[j][1]);
          if constexpr (kLo) mma_16816(o[4 * q + kb_], r0, r1, r2, r3, bh[j][0], bh[j][1]);
        }
      }
    }
    };
    if (kExact || __any_sync(0xffffffffu, vbig)) v_phase(std::true_type{});
    else v_phase(std::false_type{});
    __syncwarp();   // all lanes are done with this buffer before lane 0 refills it
  }

  // drain: a warp that stopped early at tile k_stop may still have the copies of
  // tiles k_stop and k_stop + 1 in flight (tile k + 1 is issued before tile k is
  // waited for); wait for them before the buffers are reused or the CTA exits
  for (int k = k_stop; k < min(k_stop + kQ1Stages, my_tiles); ++k) {
    if (p.test_withhold && k == 0) continue;   // never issued
    const int b = w * kQ1Stages + (k % kQ1Stages);
    uint32_t spins = 0;
    while (!mbar_try_wait(base + kQ1BarOff + b * 8, (k / kQ1Stages) & 1) && ++spins < kQ1DrainPolls) {
    }
  }

  // ---------------------------------------------------------------- merge the 8 warp states
  // (m in natural-log units, so the combine pass sees the same units from every kernel)
  __syncthreads();
  float* mrg = reinterpret_cast<float*>(smem + (kQ1Hi - base));   // per warp: o'[8 rows][256], m[8], l[8]
  float* mine = mrg + w * kQ1MrgWarp;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float lv = l_part[e];
    lv += __shfl_xor_sync(0xffffffffu, lv, 4);
    lv += __shfl_xor_sync(0xffffffffu, lv, 8);
    lv += __shfl_xor_sync(0xffffffffu, lv, 16);
    const int row = 2 * t + e;
    if (g == 0) {
      mine[8 * kQ1MrgRow + row] = m_ref[e] == -INFINITY ? -INFINITY : m_ref[e] / kLog2e;
      mine[8 * kQ1MrgRow + 8 + row] = lv;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {   // dims 32g + 8q + 0..7 of row 2t+e
      float* d = mine + row * kQ1MrgRow + g * kQ1MrgBlk + 8 * q;
      reinterpret_cast<float4*>(d)[0] =
          make_float4(o[4 * q][e], o[4 * q][e + 2], o[4 * q + 1][e], o[4 * q + 1][e + 2]);
      reinterpret_cast<float4*>(d)[1] =
          make_float4(o[4 * q + 2][e], o[4 * q + 2][e + 2], o[4 * q + 3][e], o[4 * q + 3][e + 2]);
    }
  }
  __syncthreads();
  {
    const int row = tid >> 5, d0 = (tid & 31) * 8;   // 8 rows x 32 lanes x 8 dims
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kQ1Warps; ++ww) M = fmaxf(M, mrg[ww * kQ1MrgWarp + 8 * kQ1MrgRow + row]);
    float L = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kQ1Warps; ++ww) {
        const float* src = mrg + ww * kQ1MrgWarp;
        const float a = fast_exp2((src[8 * kQ1MrgRow + row] - M) * kLog2e);
        L = fmaf(a, src[8 * kQ1MrgRow + 8 + row], L);
        const float* sl = src + row * kQ1MrgRow + (d0 >> 5) * kQ1MrgBlk + (d0 & 31);
        const float4 u0 = reinterpret_cast<const float4*>(sl)[0];
        const float4 u1 = reinterpret_cast<const float4*>(sl)[1];
        acc[0] = fmaf(a, u0.x, acc[0]); acc[1] = fmaf(a, u0.y, acc[1]);
        acc[2] = fmaf(a, u0.z, acc[2]); acc[3] = fmaf(a, u0.w, acc[3]);
        acc[4] = fmaf(a, u1.x, acc[4]); acc[5] = fmaf(a, u1.y, acc[5]);
        acc[6] = fmaf(a, u1.z, acc[6]); acc[7] = fmaf(a, u1.w, acc[7]);
      }
    }
    const int64_t rec = (int64_t(blockIdx.x) * kHkv + h) * p.rows_pad;
    float* dst = p.ws_o + (rec + row) * kD + d0;
    constexpr float kUndo = 1.0f / kQ1PScale;   // exact power of two
    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0] * kUndo, acc[1] * kUndo, acc[2] * kUndo, acc[3] * kUndo);
    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4] * kUndo, acc[5] * kUndo, acc[6] * kUndo, acc[7] * kUndo);
    if ((tid & 31) == 0) p.ws_ml[rec + row] = make_float2(M, L);
  }
}

}  // namespace tq4
