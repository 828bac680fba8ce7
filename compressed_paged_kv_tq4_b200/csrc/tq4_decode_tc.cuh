// TQ4 decode attention for 2 to 4 query tokens per request on the 5th-generation
// tensor cores (tcgen05 + TMEM), one CTA per split-K item and KV head, sm_100a.
//
// What it computes is the split-K decode of tq4_decode.cuh ([KVEXEC]
// simpleprog.com "Fitting a 27B-Parameter LLM into 24 GiB of Laptop Memory",
// section "KVExec": page-native decode straight on the compressed data; [V2]
// wpnews.pro "JustFit: Run Qwen 27B Fast ...", mechanism table row KVExec:
// rotated-domain attention), over the same items, into the same partial
// records, merged by the same combine pass. Only the arithmetic's layout differs.
//
// Layout. A tile is 128 positions of one page. The positions are the MMA's
// M = 128 rows and the request's query rows its N columns:
//   S^T  = C16 . [q'hi ; q'lo]^T + R16 . [q'hi ; q'lo]^T     (A: the tile's keys
//          as centroid hi (C16) and lo (R16) halves in TMEM, K = 256 dims)
//   O'^T += C16^T . [P'hi ; P'lo] (+ R16^T . [P'hi ; P'lo])  (A: the tile's values
//          in shared memory, M = 128 dims per half, K = positions)
// N = 2 x 8 NT columns: the hi parts of the query rows (zero-padded to whole
// n-tiles of 8), then their lo parts; a score, or an output row, is the sum of
// its hi and lo columns. The value side takes the R16 pass on chunks whose
// largest V norm exceeds kVloNorm and always for fp32 outputs, as the other
// decode kernels do; the key side always takes it.
//
// Roles (416 threads, one CTA per SM):
//   warps 0-3   softmax: thread i of warp w owns tile position 32w + i (its
//               TMEM lane). They first write q' = R q * scale, split into f16
//               hi + lo, as the shared B panel of the score MMAs. Per tile: the
//               thread reads its score row from TMEM, applies the K norm and
//               the causal limits, and takes an online softmax against a
//               per-row reference shared by all 128 threads and raised lazily:
//               only when some score exceeds it by more than 2^8, decided by one
//               barrier reduction, are the row maxima exchanged through shared
//               memory (and O rescaled in TMEM). P' = p n_v / 16 goes to a shared
//               panel as f16 hi + lo, one 128-byte row per position.
//   warps 4-7   keys: thread i of warp 4 + q owns position 32q + i and expands its
//               packed words, 64 dims at a time, through a per-lane table of
//               {hi pair, lo pair} slots into a TMEM slot (C16 in 32 columns, R16
//               in the next 32), for the tensor core to read as A.
//   warps 8-11  values: chunks of 128 dims x 64 positions; lane i of warp 8 + q
//               expands positions i and i + 32, dims 32q .. 32q + 31, into
//               swizzled shared panels (MN-major A), C16 and, where the chunk
//               needs it, R16.
//   warp 12     one thread issues every tcgen05.mma, in the order QK(j), PV(j-1),
//               and commits their completions to the producers' barriers.
// TMEM (512 columns): K ring [0, 256) (four 64-dim slots), S [256, 384) (two
// buffers), O [384, 512) (dims 0-127 and 128-255).
// Every wait is bounded by spin_limit polls; on a timeout the CTA records
// TQ4_ERR_TIMEOUT, raises its abort flag, every role leaves its loop (the
// softmax warps together, through their barrier reductions), the issuer drains
// the MMAs it issued and TMEM is freed.
#pragma once
#include "tq4_decode.cuh"
#include "tq4_prefill_tc.cuh"   // tcgen05 descriptors, fences, TMEM loads and stores, mbarrier waits

namespace tq4 {

constexpr int kDtTile = 128;                       // positions per tile (the MMA's M)
constexpr int kDtSoftWarps = 4;
constexpr int kDtKWarp0 = 4, kDtVWarp0 = 8, kDtMmaWarp = 12;
constexpr int kDtThreads = 32 * (kDtMmaWarp + 1);  // 416
constexpr int kDtKSlots = 4;                       // TMEM key ring: one 64-dim chunk per slot
constexpr int kDtVSlots = 4;                       // shared value ring: 128 dims x 64 positions per slot
constexpr uint32_t kDtVPanel = 64 * 128;           // 8 KiB: 64 positions x 64 dims f16
constexpr uint32_t kDtVPart = 2 * kDtVPanel;       // 16 KiB: the slot's 128 dims, C16 (or R16)
constexpr uint32_t kDtVSlot = 2 * kDtVPart;        // 32 KiB
constexpr uint32_t kDtQOff = kDtVSlots * kDtVSlot;
constexpr uint32_t kDtQPanelMax = 48 * 128;        // N rows x 128 B per 64-dim panel (N <= 48)
constexpr uint32_t kDtPOff = kDtQOff + 4 * kDtQPanelMax;
constexpr uint32_t kDtPBuf = kDtTile * 128;        // 16 KiB: one 128-byte row per position
constexpr uint32_t kDtLutOff = kDtPOff + 2 * kDtPBuf;
constexpr uint32_t kDtLutBytes = 256 * 16 * 8;     // 256 byte values x 16 copies x 8 B
constexpr int kDtRedRows = 24;                     // query rows of the widest request (4 tokens x 6 heads)
constexpr uint32_t kDtRedOff = kDtLutOff + kDtLutBytes;   // f32 [3][4 warps][24 rows]
constexpr uint32_t kDtFlagOff = kDtRedOff + 3 * 4 * kDtRedRows * 4;
constexpr uint32_t kDtBarOff = kDtFlagOff + 64;
constexpr uint32_t kDtMiscOff = kDtBarOff + 256;   // u32 [0] TMEM base, [1] abort
constexpr uint32_t kDtSmem = kDtMiscOff + 64 + 1024;   // + alignment slack
static_assert(kDtSmem <= 227u * 1024u, "shared memory");
static_assert(kDtQOff % 1024 == 0 && kDtPOff % 1024 == 0 && kDtPBuf % 1024 == 0 && kDtVPanel % 1024 == 0,
              "swizzled panels start on 1 KiB");

constexpr uint32_t kDtTmK = 0, kDtTmS = 256, kDtTmO = 384;   // TMEM columns
// barriers (8 B each at kDtBarOff)
constexpr int kDbKFull = 0, kDbKEmpty = 4, kDbVFull = 8, kDbVEmpty = 12, kDbSFull = 16, kDbPFull = 18,
              kDbPvDone = 20, kDbQReady = 22, kDbDrain = 23, kDbCount = 24;
static_assert(kDbKEmpty - kDbKFull == kDtKSlots && kDbVEmpty - kDbVFull == kDtVSlots, "barrier map");
static_assert(kDbCount * 8 <= 256, "barrier area");

// single-CTA MMA, A from TMEM
__device__ __forceinline__ void tc1_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// single-CTA MMA, A from shared memory
__device__ __forceinline__ void tc1_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// completion of this thread's earlier MMAs -> one arrival on the barrier
__device__ __forceinline__ void tc1_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
// OR of v over the `count` threads of named barrier `id` (a barrier of its own)
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_named_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}
// maximum over the warp of a float (order-preserving integer image, one redux)
__device__ __forceinline__ float warp_max_f32(float v) {
  int k = __float_as_int(v);
  k = k >= 0 ? k : (k ^ 0x7FFFFFFF);
  k = __reduce_max_sync(0xffffffffu, k);
  return __int_as_float(k >= 0 ? k : (k ^ 0x7FFFFFFF));
}
// 48 consecutive TMEM columns of this thread's lane -> registers (loads and wait in one statement)
__device__ __forceinline__ void tm_ld48(uint32_t taddr, uint32_t (&r)[48]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%48];\n"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47}, [%49];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47])
      : "r"(taddr), "r"(taddr + 32u)
      : "memory");
}
template <int NQ>
__device__ __forceinline__ void tm_ld_row(uint32_t taddr, uint32_t (&r)[NQ]) {
  static_assert(NQ == 32 || NQ == 48, "row width");
  if constexpr (NQ == 32) tm_ld32(taddr, r);
  else tm_ld48(taddr, r);
}
template <int NQ>
__device__ __forceinline__ void tm_st_row(uint32_t taddr, const uint32_t (&r)[NQ]) {
  static_assert(NQ == 32 || NQ == 48, "row width");
  if constexpr (NQ == 32) {
    tm_st32(taddr, r);
  } else {
    uint32_t a[32], b[16];
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = r[i];
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = r[32 + i];
    tm_st32(taddr, a);
    tm_st16(taddr + 32u, b);
  }
}

template <int NT, bool kExact>   // NT: n-tiles of 8 query rows (2: two tokens, 3: three or four)
__global__ void __launch_bounds__(kDtThreads, 1) decode_tc_kernel(const DecodeParams p) {
  constexpr int NRp = 8 * NT;    // one request's query rows, padded
  constexpr int NQ = 2 * NRp;    // MMA N: hi columns, then lo columns
  constexpr uint32_t kQPanel = uint32_t(NQ) * 128;
  static_assert(NRp <= kDtRedRows && NQ * 128 <= kDtQPanelMax && NQ * 2 <= 128, "row capacity");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int s_item[kItWords];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int h = blockIdx.y;
  const int x = int(blockIdx.x);
  pdl_wait();   // every read of the call's inputs comes after the previous kernel
  pdl_launch_dependents();
  if (w == 0) describe_private_item(p, x, h, s_item);
  if (tid == 0) check_item_records(p, s_item);
  __syncthreads();
  if (s_item[kItNMem] == 0 || x >= p.items_ub) return;

  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t sbase = (raw_s + 1023) & ~1023u;   // the swizzled panels need 1 KiB alignment
  uint8_t* smem = smem_raw + (sbase - raw_s);
  auto bar = [sbase](int i) -> uint32_t { return sbase + kDtBarOff + 8u * uint32_t(i); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kDtMiscOff);
  volatile uint32_t* vflag = reinterpret_cast<volatile uint32_t*>(smem + kDtFlagOff);
  float* red = reinterpret_cast<float*>(smem + kDtRedOff);

  const int pos_b = s_item[kItPosB], pos_e = s_item[kItPosE];
  // items start on a tile boundary, so that a tile lies in one page (the host's split
  // lengths are whole tiles); anything else is reported and contributes nothing
  const bool aligned_item = (pos_b % kDtTile) == 0;
  if (!aligned_item && tid == 0) record_error(p.status, TQ4_ERR_SEQ);
  const int n_tiles = (aligned_item && pos_e > pos_b) ? (pos_e - pos_b + kDtTile - 1) / kDtTile : 0;
  const int rq = s_item[kItReq];
  const int32_t* const table = p.page_tables + int64_t(rq) * p.max_pages;
  const int NR = 6 * p.n_q;   // the request's query rows (token-major, then head)
  const uint8_t* const pool = p.pool;
  const int32_t num_pages = p.num_pages;

  if (tid == 0) {
    for (int i = 0; i < kDtKSlots; ++i) {
      mbar_init(bar(kDbKFull + i), 4);
      mbar_init(bar(kDbKEmpty + i), 1);
    }
    for (int i = 0; i < kDtVSlots; ++i) {
      mbar_init(bar(kDbVFull + i), 4);
      mbar_init(bar(kDbVEmpty + i), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kDbSFull + b), 1);
      mbar_init(bar(kDbPFull + b), kDtSoftWarps);
      mbar_init(bar(kDbPvDone + b), 1);
    }
    mbar_init(bar(kDbQReady), kDtSoftWarps);
    mbar_init(bar(kDbDrain), 1);
    misc[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (w == 0) {   // all 512 columns; shared memory admits one CTA per SM
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(sbase + kDtMiscOff)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // per-lane centroid table: row b (a byte = two indices, 128 B) holds, in each of
  // 16 copies, the 8-byte slot {c16 pair, r16 pair}; lanes l and l + 16 share copy
  // l & 15, so each half warp's 64-bit loads hit 32 different banks
  for (int e = tid; e < 256 * 16; e += kDtThreads)
    reinterpret_cast<uint2*>(smem + kDtLutOff)[e] = lut_row(e >> 4);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  int* const status = p.status;
  const uint32_t spin_limit = p.spin_limit;
  auto bounded_wait = [misc, status, spin_limit](uint32_t b, uint32_t parity) -> bool {
    uint32_t spins = 0;
    while (!mbar_try_wait_cluster(b, parity)) {
      if (misc[1]) return false;
      if (++spins > spin_limit) {
        misc[1] = 1;
        record_error(status, TQ4_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  };
  auto warp_arrive = [lane](uint32_t b) {
    __syncwarp();
    if (lane == 0) mbar_arrive_local(b);
  };
  auto page_of = [table, pos_b, n_tiles](int i) -> int32_t {
    return i < n_tiles ? __ldg(table + ((pos_b + i * kDtTile) >> 8)) : -1;
  };

  if (w < kDtSoftWarps) {
    // =========================================================== softmax / records
    const int pl = 32 * w + lane;
    const uint32_t lane_t = tmem + (uint32_t(32 * w) << 16);
    {   // q' rows -> the B panel of the score MMAs (K-major, 128-byte swizzle):
        // hi in rows [0, NRp), lo in rows [NRp, 2 NRp); dims 64 k .. 64 k + 63 in panel k
      uint8_t* qp = smem + kDtQOff + (lane >> 3) * kQPanel;
      for (int row = w; row < NRp; row += kDtSoftWarps) {
        float v[8];
        if (row < NR) {
          const int tok = row / 6, j = row % 6;
          const uint16_t* src = p.q + ((int64_t(rq) * p.n_q + tok) * kHq + h * kGroup + j) * kD + lane * 8;
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
          const uint32_t ww[4] = {raw.x, raw.y, raw.z, raw.w};
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
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hi[i] = pack_half2(v[2 * i], v[2 * i + 1]);
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hi[i]));
          lo[i] = pack_half2(v[2 * i] - f.x, v[2 * i + 1] - f.y);
        }
        const int chs = ((lane & 7) ^ (row & 7)) << 4;   // rows row and NRp + row share row & 7
        *reinterpret_cast<uint4*>(qp + row * 128 + chs) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(qp + (NRp + row) * 128 + chs) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy stores -> tensor-core reads
      warp_arrive(bar(kDbQReady));
    }

    float m_ref[NRp], l_th[NRp];   // per-row reference (log2 units, equal in all 128 threads), this thread's sum
#pragma unroll
    for (int n = 0; n < NRp; ++n) {
      m_ref[n] = -INFINITY;
      l_th[n] = 0.f;
    }
    const int s_len = __ldg(p.seq_lens + rq);
    int lim_tok[4];   // token t of the request sees positions [0, s_len - n_q + t]
#pragma unroll
    for (int t = 0; t < 4; ++t) lim_tok[t] = s_len - p.n_q + t + 1;
    // the K and V norms of this thread's position of tile i (0 past the item's end)
    auto norms_of = [&](int i, float& kn, float& vn) {
      kn = vn = 0.f;
      const int32_t page = page_of(i);
      const int pos = pos_b + i * kDtTile + pl;
      if (i < n_tiles && pos < pos_e && page >= 0 && page < num_pages) {
        const uint8_t* pg = pool + int64_t(page) * kPageBytes;
        const int slot = h * kPage + (pos & (kPage - 1));
        kn = ldg_half(pg + kKNorms + slot * 2);
        vn = ldg_half(pg + kVNorms + slot * 2);
      }
    };
    // norms of tiles i + 1 and i + 2 in flight; loaded after a tile's proxy fence, which
    // would otherwise wait for them
    float kn_n1, vn_n1, kn_n2, vn_n2;
    norms_of(0, kn_n1, vn_n1);
    norms_of(1, kn_n2, vn_n2);
    bool fail = false;
    for (int i = 0; i < n_tiles; ++i) {
      const int b = i & 1;
      const float kn = kn_n1 * kLog2e, vn = vn_n1 * kPfPScale;
      kn_n1 = kn_n2;
      vn_n1 = vn_n2;
      const bool ok = bounded_wait(bar(kDbSFull + b), (i >> 1) & 1);
      if (bar_any(1, 32 * kDtSoftWarps, !ok)) {
        fail = true;
        break;
      }
      tc_fence_after();
      uint32_t sr[NQ];
      tm_ld_row<NQ>(lane_t + kDtTmS + 64 * b, sr);
      const int pos = pos_b + i * kDtTile + pl;
      float s[NRp];
      bool need = false;
#pragma unroll
      for (int n = 0; n < NRp; ++n) {
        const bool vis = n < NR && pos < pos_e && pos < lim_tok[n / 6];
        s[n] = vis ? (__uint_as_float(sr[n]) + __uint_as_float(sr[NRp + n])) * kn : -INFINITY;
        need = need || s[n] > m_ref[n] + kPfLazy;
      }
      // raise the references only when some score of the tile exceeds its row's by > 2^8
      need = bar_any(1, 32 * kDtSoftWarps, need);
      float* rb = red + b * (4 * kDtRedRows);   // this tile's exchange area; row n's factor lands in rb[n]
      if (need) {
#pragma unroll
        for (int n = 0; n < NRp; ++n) {
          const float wm = warp_max_f32(s[n]);
          if (lane == 0) rb[w * kDtRedRows + n] = wm;
        }
        bar_named_sync(1, 32 * kDtSoftWarps);
        float mt[NRp];
#pragma unroll
        for (int n = 0; n < NRp; ++n)
          mt[n] = fmaxf(fmaxf(rb[n], rb[kDtRedRows + n]), fmaxf(rb[2 * kDtRedRows + n], rb[3 * kDtRedRows + n]));
        bar_named_sync(1, 32 * kDtSoftWarps);   // every thread has read the maxima
#pragma unroll
        for (int n = 0; n < NRp; ++n) {
          float alpha = 1.f;
          if (mt[n] > m_ref[n] + kPfLazy) {
            alpha = fast_exp2(m_ref[n] - mt[n]);
            m_ref[n] = mt[n];
            l_th[n] *= alpha;
          }
          if (w == 0 && lane == 0) rb[n] = alpha;   // the same in every thread; read for the O rescale
        }
      }
      // P' = p n_v / 16 of this position: hi in elements [0, NRp), lo in [NRp, 2 NRp) of its
      // 128-byte row (MN-major B panel: 16-byte chunk c at c ^ (position & 7))
      uint32_t phi[NRp / 2], plo[NRp / 2];
#pragma unroll
      for (int k = 0; k < NRp / 2; ++k) {
        const float mu0 = m_ref[2 * k] == -INFINITY ? 0.f : m_ref[2 * k];
        const float mu1 = m_ref[2 * k + 1] == -INFINITY ? 0.f : m_ref[2 * k + 1];
        const float p0 = fast_exp2(s[2 * k] - mu0), p1 = fast_exp2(s[2 * k + 1] - mu1);   // 0 where masked
        l_th[2 * k] += p0;
        l_th[2 * k + 1] += p1;
        const float w0 = p0 * vn, w1 = p1 * vn;
        phi[k] = pack_half2(w0, w1);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&phi[k]));
        plo[k] = pack_half2(w0 - f.x, w1 - f.y);
      }
      uint8_t* prow = smem + kDtPOff + b * kDtPBuf + pl * 128;
#pragma unroll
      for (int c = 0; c < NRp / 8; ++c) {
        *reinterpret_cast<uint4*>(prow + ((c ^ (pl & 7)) << 4)) =
            make_uint4(phi[4 * c], phi[4 * c + 1], phi[4 * c + 2], phi[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + (((NRp / 8 + c) ^ (pl & 7)) << 4)) =
            make_uint4(plo[4 * c], plo[4 * c + 1], plo[4 * c + 2], plo[4 * c + 3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      norms_of(i + 2, kn_n2, vn_n2);
      // PV(i - 1) has completed before O is rescaled (waited at every tile, so each
      // buffer's barrier never runs more than one phase ahead of this wait)
      if (i > 0) {
        const bool ok2 = bounded_wait(bar(kDbPvDone + ((i - 1) & 1)), ((i - 1) >> 1) & 1);
        if (bar_any(1, 32 * kDtSoftWarps, !ok2)) {
          fail = true;
          break;
        }
        tc_fence_after();
        if (need) {
#pragma unroll 1
          for (int dh = 0; dh < 2; ++dh) {
            uint32_t ov[NQ];
            tm_ld_row<NQ>(lane_t + kDtTmO + 64 * dh, ov);
#pragma unroll
            for (int n = 0; n < NRp; ++n) {
              const float alpha = rb[n];   // written before the barrier reduction above
              ov[n] = __float_as_uint(__uint_as_float(ov[n]) * alpha);
              ov[NRp + n] = __float_as_uint(__uint_as_float(ov[NRp + n]) * alpha);
            }
            tm_st_row<NQ>(lane_t + kDtTmO + 64 * dh, ov);
          }
          tm_wait_st();
        }
      }
      tc_fence_before();
      warp_arrive(bar(kDbPFull + b));
    }
    // ---- the last PV, then the item's partial records
    bool ok_end = !fail;
    if (ok_end && n_tiles > 0) {
      const bool okw = bounded_wait(bar(kDbPvDone + ((n_tiles - 1) & 1)), ((n_tiles - 1) >> 1) & 1);
      ok_end = !bar_any(1, 32 * kDtSoftWarps, !okw);
    }
    tc_fence_after();
    float* lr = red + 2 * (4 * kDtRedRows);
#pragma unroll
    for (int n = 0; n < NRp; ++n) {
      float v = l_th[n];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) lr[w * kDtRedRows + n] = v;
    }
    bar_named_sync(1, 32 * kDtSoftWarps);
    const bool have_o = ok_end && n_tiles > 0;
    const int64_t rec0 = (int64_t(s_item[kItRec]) * kHkv + h) * p.rows_pad;
#pragma unroll 1
    for (int dh = 0; dh < 2; ++dh) {
      uint32_t ov[NQ];
      if (have_o) {
        tm_ld_row<NQ>(lane_t + kDtTmO + 64 * dh, ov);
      } else {
#pragma unroll
        for (int n = 0; n < NQ; ++n) ov[n] = 0u;
      }
#pragma unroll
      for (int n = 0; n < NRp; ++n)
        if (n < NR)
          p.ws_o[(rec0 + n) * kD + 128 * dh + pl] =
              (__uint_as_float(ov[n]) + __uint_as_float(ov[NRp + n])) * (1.0f / kPfPScale);
    }
    if (w == 0) {
#pragma unroll
      for (int n = 0; n < NRp; ++n)
        if (lane == n && n < NR) {
          const float l = (lr[n] + lr[kDtRedRows + n]) + (lr[2 * kDtRedRows + n] + lr[3 * kDtRedRows + n]);
          p.ws_ml[rec0 + n] = have_o ? make_float2(m_ref[n] * (1.0f / kLog2e), l) : make_float2(-INFINITY, 0.f);
        }
    }
  } else if (w < kDtVWarp0) {
    // =========================================================== keys -> TMEM
    const int q4 = w - kDtKWarp0;
    const int pl = 32 * q4 + lane;
    const uint32_t lane_t = tmem + (uint32_t(32 * q4) << 16);
    const uint32_t lut_s = sbase + kDtLutOff;
    const uint32_t lane16 = uint32_t(lane & 15) * 16u;   // (byte << 8 | 16 copy) >> 1 = byte * 128 + 8 copy
    // raw[2 dc], raw[2 dc + 1]: words 8 dc .. 8 dc + 7 of this thread's position of the
    // tile about to be expanded; refilled with the next tile's right after use
    uint4 raw[8];
    auto fetch = [&](int i, int dc, int32_t page) {
      raw[2 * dc] = raw[2 * dc + 1] = make_uint4(0, 0, 0, 0);
      if (i >= n_tiles) return;
      if (page >= 0 && page < num_pages) {
        const uint8_t* src = pool + int64_t(page) * kPageBytes + kKWords +
                             (int64_t(h) * kPage + ((pos_b + i * kDtTile + pl) & (kPage - 1))) * 128 + dc * 32;
        raw[2 * dc] = ldg128(src);
        raw[2 * dc + 1] = ldg128(src + 16);
      } else if (dc == 0 && lane == 0) {
        record_error(status, TQ4_ERR_PAGE_RANGE);   // words stay 0 and the K norm 0: no contribution
      }
    };
    {
      const int32_t pg0 = page_of(0);
#pragma unroll
      for (int dc = 0; dc < 4; ++dc) fetch(0, dc, pg0);
    }
    int32_t pg_next = page_of(1);
    for (int i = 0; i < n_tiles; ++i) {
      bool ok = true;
#pragma unroll
      for (int dc = 0; dc < 4; ++dc) {
        if (i > 0 && !__all_sync(0xffffffffu, bounded_wait(bar(kDbKEmpty + dc), (i - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // words 4 hh .. 4 hh + 3 (dims 32 hh ..) -> columns 16 hh .. 16 hh + 15
          const uint4 u = raw[2 * dc + hh];
          const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
          uint32_t c[16], r[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // word k: dims 8k .. 8k + 7 -> columns 4k .. 4k + 3
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5504u) >> 1), c[4 * k], r[4 * k]);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5514u) >> 1), c[4 * k + 1], r[4 * k + 1]);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5524u) >> 1), c[4 * k + 2], r[4 * k + 2]);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5534u) >> 1), c[4 * k + 3], r[4 * k + 3]);
          }
          tm_st16(lane_t + kDtTmK + 64 * dc + 16 * hh, c);
          tm_st16(lane_t + kDtTmK + 64 * dc + 32 + 16 * hh, r);
        }
        tm_wait_st();
        tc_fence_before();
        // (test hook: the first chunk's signal is withheld, so the issuer's wait for it runs out)
        if (!(p.test_withhold && i == 0 && dc == 0)) warp_arrive(bar(kDbKFull + dc));
        fetch(i + 1, dc, pg_next);   // the next tile's words, once this chunk is signalled
      }
      if (!ok) break;
      pg_next = page_of(i + 2);
    }
  } else if (w < kDtMmaWarp) {
    // =========================================================== values -> shared panels
    const int q4 = w - kDtVWarp0;
    const uint32_t lut_s = sbase + kDtLutOff;
    const uint32_t lane16 = uint32_t(lane & 15) * 16u;
    // chunk vc of a tile: dims 128 (vc >> 1) .. + 127, positions 64 (vc & 1) .. + 63. This
    // thread takes chunk positions lane and lane + 32, dims 32 q4 .. 32 q4 + 31 of the
    // half (words 16 (vc >> 1) + 4 q4 .. + 3): raw[2 vc + e] for position lane + 32 e.
    // vnr[e]: V norm of tile position lane + 32 e (0 past the item's end).
    uint4 raw[8];
    float vnr[4];
    auto fetch = [&](int i, int vc, int32_t page) {
      raw[2 * vc] = raw[2 * vc + 1] = make_uint4(0, 0, 0, 0);
      if (vc >= 2) vnr[2 * (vc & 1)] = vnr[2 * (vc & 1) + 1] = 0.f;
      if (i >= n_tiles || page < 0 || page >= num_pages) return;
      const uint8_t* pg = pool + int64_t(page) * kPageBytes;
      const int t0 = pos_b + i * kDtTile;
      const int64_t slot0 = int64_t(h) * kPage + (t0 & (kPage - 1));
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tp = 64 * (vc & 1) + lane + 32 * e;
        raw[2 * vc + e] = ldg128(pg + kVWords + (slot0 + tp) * 128 + (16 * (vc >> 1) + 4 * q4) * 4);
        if (vc >= 2) vnr[2 * (vc & 1) + e] = t0 + tp < pos_e ? ldg_half(pg + kVNorms + (slot0 + tp) * 2) : 0.f;
      }
    };
    {
      const int32_t pg0 = page_of(0);
#pragma unroll
      for (int vc = 0; vc < 4; ++vc) fetch(0, vc, pg0);
    }
    int32_t pg_next = page_of(1);
    for (int i = 0; i < n_tiles; ++i) {
      bool ok = true;
#pragma unroll
      for (int vc = 0; vc < 4; ++vc) {
        const int sq = 4 * i + vc, slot = sq % kDtVSlots, f = sq / kDtVSlots;
        if (f > 0 && !__all_sync(0xffffffffu, bounded_wait(bar(kDbVEmpty + slot), (f - 1) & 1))) {
          ok = false;
          break;
        }
        const int ph = vc & 1;
        // every warp sees all 64 positions' norms, so all four take the same decision
        const bool vlo = kExact || __any_sync(0xffffffffu, vnr[2 * ph] > kVloNorm || vnr[2 * ph + 1] > kVloNorm);
        const uint32_t vs = sbase + uint32_t(slot) * kDtVSlot + uint32_t(q4 >> 1) * kDtVPanel;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int prow = lane + 32 * e;   // chunk-local position
          const uint32_t ww[4] = {raw[2 * vc + e].x, raw[2 * vc + e].y, raw[2 * vc + e].z, raw[2 * vc + e].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // word k: dims 32 q4 + 8k .. + 7 = 16-byte chunk 4 (q4 & 1) + k of the panel row
            uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5504u) >> 1), h0, l0);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5514u) >> 1), h1, l1);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5524u) >> 1), h2, l2);
            ld_shared_v2(lut_s + (__byte_perm(ww[k], lane16, 0x5534u) >> 1), h3, l3);
            const uint32_t off = uint32_t(prow) * 128u + uint32_t(((4 * (q4 & 1) + k) ^ (prow & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + off), "r"(h0), "r"(h1), "r"(h2),
                         "r"(h3)
                         : "memory");
            if (vlo)
              asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + kDtVPart + off), "r"(l0), "r"(l1),
                           "r"(l2), "r"(l3)
                           : "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy writes -> tensor-core reads
        if (q4 == 0 && lane == 0) vflag[slot] = vlo ? 1u : 0u;
        warp_arrive(bar(kDbVFull + slot));
        // the next tile's words go out only now: the proxy fence waits for this
        // thread's outstanding loads as well
        fetch(i + 1, vc, pg_next);
      }
      if (!ok) break;
      pg_next = page_of(i + 2);
    }
  } else {
    // =========================================================== MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc_idesc(kDtTile, NQ, 0);                // A (TMEM) and B K-major
      constexpr uint32_t idesc_pv = tc_idesc(kDtTile, NQ, 1) | (1u << 15);   // A and B MN-major
      bool ok = bounded_wait(bar(kDbQReady), 0);   // q' panel stored
      tc_fence_after();
      for (int i = 0; ok && i <= n_tiles; ++i) {
        if (i < n_tiles) {   // S[i & 1] = (C16 + R16)(K) . [q'hi ; q'lo]^T, 64 dims per slot
          const int b = i & 1;
          const uint32_t s_t = tmem + kDtTmS + 64 * b;
#pragma unroll 1
          for (int dc = 0; dc < 4 && ok; ++dc) {
            if (!bounded_wait(bar(kDbKFull + dc), i & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t q0 = tc_sdesc(sbase + kDtQOff + dc * kQPanel, 16, 1024);
            const uint32_t ka = tmem + kDtTmK + 64 * dc;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc1_mma_ts(s_t, ka + 8 * ks, q0 + uint64_t((ks * 32) >> 4), idesc_qk, (dc | ks) ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc1_mma_ts(s_t, ka + 32 + 8 * ks, q0 + uint64_t((ks * 32) >> 4), idesc_qk, 1u);
            tc1_commit(bar(kDbKEmpty + dc));   // the slot is free once these have run
          }
          if (!ok) break;
          tc1_commit(bar(kDbSFull + b));
        }
        if (i >= 1) {        // O += V^T . P'^T for tile i - 1, in chunks of 128 dims x 64 positions
          const int jb = i - 1, bp = jb & 1;
          if (!bounded_wait(bar(kDbPFull + bp), (jb >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t pb = sbase + kDtPOff + bp * kDtPBuf;
#pragma unroll 1
          for (int vc = 0; vc < 4; ++vc) {
            const int sq = 4 * jb + vc, slot = sq % kDtVSlots, f = sq / kDtVSlots;
            const int dh = vc >> 1, ph = vc & 1;
            if (!bounded_wait(bar(kDbVFull + slot), f & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const bool vlo = kExact || vflag[slot] != 0;
            const uint32_t vb = sbase + uint32_t(slot) * kDtVSlot;
            const uint64_t vhi = tc_sdesc(vb, kDtVPanel, 1024), vlo_d = tc_sdesc(vb + kDtVPart, kDtVPanel, 1024);
            const uint64_t pd = tc_sdesc(pb + uint32_t(ph) * 64u * 128u, kDtPBuf, 1024);
            const uint32_t o_t = tmem + kDtTmO + 64 * dh;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // 16 positions per step
              const uint64_t o = uint64_t((ks * 16 * 128) >> 4);
              tc1_mma_ss(o_t, vhi + o, pd + o, idesc_pv, (jb > 0 || ph > 0 || ks > 0) ? 1u : 0u);
              if (vlo) tc1_mma_ss(o_t, vlo_d + o, pd + o, idesc_pv, 1u);
            }
            tc1_commit(bar(kDbVEmpty + slot));
          }
          if (!ok) break;
          tc1_commit(bar(kDbPvDone + bp));   // P buffer bp is free and O holds tile jb
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      tc1_commit(bar(kDbDrain));
      for (uint32_t spins = 0; !mbar_try_wait_cluster(bar(kDbDrain), 0) && spins < TQ4_DEFAULT_WAIT_POLLS;
           ++spins) {
      }
    }
  }

  // =========================================================== free TMEM
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
}

}  // namespace tq4
