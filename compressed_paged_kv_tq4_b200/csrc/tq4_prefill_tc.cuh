// TQ4 prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
// What it computes ([KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into
// 24 GiB of Laptop Memory", section "KVExec": multi-query prefill reconstructs
// the packed history and feeds scaled dot-product attention): chunk token i
// attends causally to the TQ4 prefix [0, prefix_len) and to chunk tokens 0..i,
// whose K/V are used at full precision. Everything is in the rotated domain
// ([V2] wpnews.pro "JustFit: Run Qwen 27B Fast ...", mechanism table row
// KVExec): q' = R q * scale; prefix keys/values are their centroid values (the
// K norm scales score columns, the V norm is folded into P); chunk keys/values
// are R k, R v; each output row gets R^T once at the end.
//
// One CTA = 128 query rows (row = token * 6 + head within the KV head's group)
// of one KV head, walking KV tiles of 64 positions.
//   warps 0-3   softmax: thread i of warp w owns row 32w + i = TMEM lane. Puts
//               its q' hi row into TMEM and its q' lo row into shared memory. Reads
//               its score row from TMEM, applies K norms, the causal mask and an
//               online softmax with a lazily raised reference; writes
//               P = p * n_v / 256 back into TMEM as an f16 hi + lo pair (the two
//               halves keep P V at fp32-level precision); final epilogue.
//   warps 4-11  dequant, two groups of four warps; group g fills the shared
//               stage g for tiles j = g, g+2, ... : packed words are prefetched
//               into registers one tile ahead, expanded through a per-lane
//               centroid table (32 KiB: row = one byte of indices, one 4-byte slot
//               per lane) into f16 panels [4 dim blocks][64 positions][128 B]
//               with the 128-byte swizzle; the chunk's own K/V are copied.
//   warp 12     one thread issues tcgen05.mma: S = Q'hi K^T (+ Q'lo K^T where the
//               tile needs it; A = Q'hi in TMEM, A = Q'lo in shared memory; B = K
//               panels, K-major) and
//               O += P V (A = P in TMEM, B = V panels, MN-major), in the order
//               QK(j), PV(j-1), so the tensor pipe holds the next score tile while
//               the softmax runs.
// TMEM (512 columns): Q'hi [0,128), S/P buffers [128,192) and [192,256), O [256,512).
// The q' hi + lo pair keeps the scores at fp32-level precision: with a single f16
// q', the score error grows with the key norm, and keys with 8x norms move
// softmax weights by about 1%.
// Every wait is bounded; on a timeout the CTA records TQ4_ERR_TIMEOUT, skips the
// remaining work, drains its issued MMAs, frees its TMEM and returns.
#pragma once
#include "tq4_device.cuh"
#include "tq4_prefill.cuh"

namespace tq4 {

constexpr int kTcRows = 128;
constexpr int kTcTile = 64;                              // KV positions per tile
constexpr int kTcSoftWarps = 4, kTcDeqWarps = 8;
constexpr int kTcMmaWarp = kTcSoftWarps + kTcDeqWarps;   // 12
constexpr int kTcThreads = 32 * (kTcMmaWarp + 1);        // 416
constexpr int kTcGroupThreads = 128;                     // one dequant group
constexpr int kTcUnits = 8;                              // 16-B word groups per dequant thread per tile
constexpr int kTcPanel = kTcTile * 128;                  // 8 KiB: 64 positions x 64 dims f16
constexpr int kTcKV = 4 * kTcPanel;                      // 32 KiB: one K or V tile
constexpr int kTcStage = 2 * kTcKV;                      // K then V
constexpr int kTcQloPanel = kTcRows * 128;              // 16 KiB: 128 rows x 64 dims f16
constexpr int kTcLutBytes = 256 * 128;                   // 256 byte values x 32 lanes x 4 B
// dynamic shared memory (offsets from the 1 KiB-aligned base)
constexpr uint32_t kTcStageOff = 0;                      // 2 stages x 64 KiB
constexpr uint32_t kTcQloOff = 2 * kTcStage;             // q' lo panels [4][128 rows][128 B], 64 KiB
constexpr uint32_t kTcLutOff = kTcQloOff + 4 * kTcQloPanel;   // 32 KiB per-lane centroid table
constexpr uint32_t kTcNormOff = kTcLutOff + kTcLutBytes; // [2 stages][K 64, V 64] fp32
constexpr uint32_t kTcBarOff = kTcNormOff + 2 * 2 * kTcTile * 4;
constexpr uint32_t kTcMiscOff = kTcBarOff + 128;   // u32 [0] TMEM base, [1] abort; f32 [8 + 4 stage + warp] K norm max
constexpr uint32_t kTcSmem = kTcMiscOff + 128 + 1024;    // + alignment slack
constexpr int kTcOsStride = kD + 4;                      // epilogue rows (fp32), reuse the stages + q' lo
static_assert(uint32_t(kTcRows * kTcOsStride * 4) <= kTcLutOff, "epilogue rows overlap the table");
static_assert(kTcSmem <= 227u * 1024u, "shared memory");
static_assert(kTcQloOff % 1024 == 0 && kTcStage % 1024 == 0, "swizzled panels start on 1 KiB");
static_assert(kTcDeqWarps * 32 == 2 * kTcGroupThreads, "two dequant groups");
static_assert(kTcGroupThreads * kTcUnits == 2 * kTcTile * 8, "units cover K and V of one tile");
constexpr uint32_t kTcSpin = 1u << 24;
constexpr float kTcPScale = 1.0f / 256.0f;   // P carries 1/256, undone in the epilogue
constexpr float kTcLazy = 8.0f;              // raise the row reference only when the max grows by > 2^8
// The q' lo correction (Q'lo K^T) runs for a tile when it holds chunk positions or
// a prefix key whose norm exceeds kQloNorm (see its definition).

// TMEM columns
constexpr uint32_t kTmQ = 0, kTmS0 = 128, kTmO = 256;

// ---- descriptors (layouts of the PTX ISA's tcgen05 matrix descriptors)
// instruction descriptor, kind::f16: D f32 (bit 4), A = B = f16 (formats 0),
// A K-major, B K-major (0) or MN-major (1) at bit 16, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int b_mn_major) {
  return (1u << 4) | (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// shared-memory descriptor: start, leading / stride byte offsets (>> 4), version 1
// at bit 46, 128-byte swizzle (layout type 2) at bits 61-63.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t start, uint32_t lbo, uint32_t sbo) {
  return uint64_t((start >> 4) & 0x3FFF) | (uint64_t((lbo >> 4) & 0x3FFF) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFF) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool tc_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// 32 consecutive TMEM columns of this thread's lane -> 32 registers (load and wait
// in one statement, so no use of the registers can be scheduled before the wait)
__device__ __forceinline__ void tm_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tm_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tm_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tm_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t sbase = (raw_s + 1023) & ~1023u;   // the swizzled panels need 1 KiB alignment
  uint8_t* smem = smem_raw + (sbase - raw_s);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * kTcRows;
  const int m_total = 6 * p.n_tok;
  const int last_row = min(row0 + kTcRows, m_total) - 1;
  const int kv_end = p.prefix_len + last_row / 6 + 1;
  const int n_tiles = (kv_end + kTcTile - 1) / kTcTile;

  // K and V halves of a stage have their own barriers: a K slot is free again as
  // soon as its QK has run, a V slot once its PV has run. Both norms of a tile are
  // written with its V half (the softmax of the tile two back may still read them
  // while the K half is refilled).
  const uint32_t bar_k_full = sbase + kTcBarOff;    // [2] count 128 (one dequant group)
  const uint32_t bar_v_full = bar_k_full + 16;      // [2] count 128; also covers both norms
  const uint32_t bar_k_empty = bar_k_full + 32;     // [2] count 1 (commit after QK)
  const uint32_t bar_v_empty = bar_k_full + 48;     // [2] count 1 (commit after PV)
  const uint32_t bar_s_full = bar_k_full + 64;      // [2] count 1 (commit after QK)
  const uint32_t bar_p_full = bar_k_full + 80;      // [2] count 128 (softmax threads)
  const uint32_t bar_o_ready = bar_k_full + 96;     // count 1 (commit after PV)
  const uint32_t bar_drain = bar_k_full + 104;      // count 1 (final commit)
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kTcMiscOff);   // [0] TMEM base, [1] abort
  float* norms = reinterpret_cast<float*>(smem + kTcNormOff);

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_k_full + 8 * b, kTcGroupThreads);
      mbar_init(bar_v_full + 8 * b, kTcGroupThreads);
      mbar_init(bar_k_empty + 8 * b, 1);
      mbar_init(bar_v_empty + 8 * b, 1);
      mbar_init(bar_s_full + 8 * b, 1);
      mbar_init(bar_p_full + 8 * b, 32 * kTcSoftWarps);
    }
    mbar_init(bar_o_ready, 1);
    mbar_init(bar_drain, 1);
    misc[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (w == 0) {   // 512 TMEM columns; shared memory admits one CTA per SM, so no CTA of this kernel competes
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(sbase + kTcMiscOff)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // per-lane centroid table: row b (a byte = two indices, 128 B) holds f16x2
  // {c[b & 15], c[b >> 4]} in each lane's 4-byte slot, so a warp's lookups never
  // share a bank
  for (int e = tid; e < 256 * 32; e += kTcThreads) {
    const int b = e >> 5, l = e & 31;
    reinterpret_cast<uint32_t*>(smem + kTcLutOff)[b * 32 + l] =
        uint32_t(g_codebook.c16[b & 15]) | (uint32_t(g_codebook.c16[b >> 4]) << 16);
  }
  pdl_wait();   // q', the chunk rows and the pool may come from the previous kernels
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  int* const status = p.status;
  auto bounded_wait = [misc, status](uint32_t bar, uint32_t parity) -> bool {
    uint32_t spins = 0;
    while (!tc_try_wait(bar, parity)) {
      if (misc[1]) return false;
      if (++spins > kTcSpin) {
        misc[1] = 1;
        record_error(status, TQ4_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  };
  // the softmax warps use TMEM loads/stores that all 32 lanes must execute
  // together, so every wait and every decision before one is taken warp-wide
  auto warp_wait = [&bounded_wait](uint32_t bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, bounded_wait(bar, parity));
  };

  if (w < kTcSoftWarps) {
    // =========================================================== softmax / epilogue
    const int r_local = 32 * w + lane;
    const int row = row0 + r_local;
    const bool row_ok = row < m_total;
    const int tok = row_ok ? row / 6 : 0;
    const int lim = row_ok ? p.prefix_len + tok + 1 : 0;   // positions [0, lim) are visible
    const uint32_t lane_addr = tmem + (uint32_t(32 * w) << 16);
    {   // q' row -> TMEM columns [0,128) as f16 pairs (A operand of S = Q' K^T)
      const uint4* src =
          reinterpret_cast<const uint4*>(p.qr + (int64_t(tok) * kHq + h * kGroup + (row_ok ? row % 6 : 0)) * kD);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 u = row_ok ? __ldg(src + c * 8 + i) : make_uint4(0, 0, 0, 0);
          v[4 * i] = u.x;
          v[4 * i + 1] = u.y;
          v[4 * i + 2] = u.z;
          v[4 * i + 3] = u.w;
        }
        tm_st32(lane_addr + kTmQ + 32 * c, v);
      }
      tm_wait_st();
      // q' lo row -> shared panels (K-major, 128-byte swizzle): dims 64 k .. 64 k + 63 in panel k
      const uint4* src_lo =
          reinterpret_cast<const uint4*>(p.qlo + (int64_t(tok) * kHq + h * kGroup + (row_ok ? row % 6 : 0)) * kD);
      uint8_t* qlo_row = smem + kTcQloOff + r_local * 128;
#pragma unroll 8
      for (int g = 0; g < 32; ++g) {   // g = 16-byte chunk (8 dims)
        const uint4 u = row_ok ? __ldg(src_lo + g) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qlo_row + (g >> 3) * kTcQloPanel + (((g & 7) ^ (r_local & 7)) << 4)) = u;
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy stores -> tensor-core reads
    }
    tc_fence_before();
    mbar_arrive(bar_p_full + 8);   // extra phase of p_full[1]: q' hi is in TMEM, q' lo in shared memory

    float m_ref = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      if (!warp_wait(bar_s_full + 8 * b, (j >> 1) & 1)) break;
      if (!warp_wait(bar_v_full + 8 * b, (j >> 1) & 1)) break;   // V half and both norms of this tile
      tc_fence_after();
      const float4* kn4 = reinterpret_cast<const float4*>(norms + b * 2 * kTcTile);   // K norm * log2(e)
      const float4* vn4 = kn4 + kTcTile / 4;                                          // V norm / 256
      const int pos0 = j * kTcTile;
      uint32_t sr[2][32];
      tm_ld32(lane_addr + kTmS0 + 64 * b, sr[0]);
      tm_ld32(lane_addr + kTmS0 + 64 * b + 32, sr[1]);
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // scores in log2 units
      if (__all_sync(0xffffffffu, pos0 + kTcTile <= lim)) {           // the whole tile is visible
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          const float4 k = kn4[g];
          const float kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s = __uint_as_float(sr[g >> 3][(4 * g + e) & 31]) * kk[e];
            sr[g >> 3][(4 * g + e) & 31] = __float_as_uint(s);
            mx4[e] = fmaxf(mx4[e], s);
          }
        }
      } else {                                                        // causal edge or past the end
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          const float4 k = kn4[g];
          const float kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s = (pos0 + 4 * g + e < lim) ? __uint_as_float(sr[g >> 3][(4 * g + e) & 31]) * kk[e]
                                                     : -INFINITY;
            sr[g >> 3][(4 * g + e) & 31] = __float_as_uint(s);
            mx4[e] = fmaxf(mx4[e], s);
          }
        }
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const bool raise = mx > m_ref + kTcLazy;   // raise the reference: rescale l and the O row accumulated so far
      float alpha = 1.f;
      if (raise) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        l_sum *= alpha;
      }
      if (j > 0 && __any_sync(0xffffffffu, raise)) {   // warp-wide; lanes that keep their reference use alpha = 1
        if (!warp_wait(bar_o_ready, (j - 1) & 1)) break;   // PV(j-1) has completed
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t ov[32];
          tm_ld32(lane_addr + kTmO + 32 * c, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tm_st32(lane_addr + kTmO + 32 * c, ov);
        }
        tm_wait_st();
      }
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const float4 v = vn4[g];
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pr = fast_exp2(__uint_as_float(sr[g >> 3][(4 * g + e) & 31]) - mu);   // +0 when masked
          l4[e] += pr;
          sr[g >> 3][(4 * g + e) & 31] = __float_as_uint(pr * vv[e]);
        }
      }
      l_sum += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // P hi (columns 0-31: positions 2k, 2k+1 in column k) and P lo = P - f16(P)
      // (columns 32-63), written over the scores in halves of 32 positions
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = pack_half2(__uint_as_float(sr[c][2 * k]), __uint_as_float(sr[c][2 * k + 1]));
        tm_st16(lane_addr + kTmS0 + 64 * b + 16 * c, pk);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&pk[k]));
          pk[k] = pack_half2(__uint_as_float(sr[c][2 * k]) - hi.x, __uint_as_float(sr[c][2 * k + 1]) - hi.y);
        }
        tm_st16(lane_addr + kTmS0 + 64 * b + 32 + 16 * c, pk);
      }
      tm_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full + 8 * b);
    }
    // ---- O / l -> shared memory rows (reusing the stages): wait for the last PV
    const bool ok = __all_sync(0xffffffffu, misc[1] == 0) && warp_wait(bar_o_ready, (n_tiles - 1) & 1);
    tc_fence_after();
    float* os = reinterpret_cast<float*>(smem + kTcStageOff) + r_local * kTcOsStride;
    const float inv = (ok && l_sum > 0.f) ? (0.0625f / kTcPScale) / l_sum : 0.f;   // 1/256 of P and 1/16 of R^T
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t ov[32];
      tm_ld32(lane_addr + kTmO + 32 * c, ov);
      if (!ok) {
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(os + 32 * c + i) =
            make_float4(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv,
                        __uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
    }
  } else if (w < kTcMmaWarp) {
    // =========================================================== dequant groups
    const int grp_id = (w - kTcSoftWarps) >> 2;                 // stage b == grp_id, tiles j = grp_id, +2, ...
    const int gt = tid - 32 * kTcSoftWarps - kTcGroupThreads * grp_id;   // 0..127
    // unit u of this thread: 16 bytes (4 words = 32 dims) of one position's K or V.
    // A quarter warp covers 4 positions x 2 adjacent word groups, so its 16-B
    // shared stores land in 8 distinct bank groups under the swizzle.
    const int grp = (lane & 1) | (((lane >> 3) & 3) << 1);     // word group 0..7 -> dims 32 grp ..
    const int pl_lo = (lane >> 1) & 3;
    const char* lut = reinterpret_cast<const char*>(smem + kTcLutOff);
    const uint32_t lane8 = uint32_t(lane) * 8u;   // (byte << 8 | 8 lane) >> 1 = byte * 128 + 4 lane
    const int prefix_end = min(p.prefix_len, kv_end);
    uint8_t* st = smem + kTcStageOff + grp_id * kTcStage;
    float* nb = norms + grp_id * 2 * kTcTile;

    // raw[u] holds unit u's packed words for the tile about to be expanded (units
    // 0-3: K, 4-7: V); each register is refilled with the group's next tile (j + 2)
    // right after use, so the loads fly while the stage is waited for. A tile lies
    // in one page; its page id is loaded two tiles ahead of use.
    uint4 raw[kTcUnits];
    float rawn[kTcUnits];
    const uint8_t* const pool = p.pool;
    const int32_t* const page_table = p.page_table;
    const int32_t num_pages = p.num_pages;
    auto page_of = [=](int j) -> int32_t {
      return (j < n_tiles && j * kTcTile < prefix_end) ? __ldg(page_table + ((j * kTcTile) >> 8)) : 0;
    };
    auto fetch = [&raw, &rawn, gt, pl_lo, prefix_end, pool, num_pages, h, grp, status](int j, int u, int32_t page) {
      const int q = (gt >> 5) + 4 * u;   // 0..31: bit 4 = V, bits 0-3 = position group
      const int kv = q >> 4, pos = j * kTcTile + 4 * (q & 15) + pl_lo;
      raw[u] = make_uint4(0, 0, 0, 0);
      rawn[u] = 0.f;
      if (pos < prefix_end) {
        if (page >= 0 && page < num_pages) {
          const uint8_t* pg = pool + int64_t(page) * kPageBytes;
          const int slot = h * kPage + (pos & (kPage - 1));
          raw[u] = ldg128(pg + (kv ? kVWords : kKWords) + int64_t(slot) * 128 + grp * 16);
          if (grp == 0) rawn[u] = ldg_half(pg + (kv ? kVNorms : kKNorms) + slot * 2);
        } else if (grp == 0) {
          record_error(status, TQ4_ERR_PAGE_RANGE);   // words stay 0 and the norm 0: no contribution
        }
      }
    };
    // expand unit u of tile j into the stage: centroid values for a prefix position,
    // an asynchronous copy of the prologue's f16 row for a chunk position, zeros past
    // the CTA's last visible position. Returns the unit's norm (1 for chunk rows: the
    // rotated row carries its own length; 0 past the end).
    auto expand = [&](int j, int u) -> float {
      const int q = (gt >> 5) + 4 * u;
      const int kv = q >> 4, pl = 4 * (q & 15) + pl_lo, pos = j * kTcTile + pl;
      // dims 32 grp .. +31 = panel grp / 2, 16-B chunks 4 (grp & 1) .. +3 of row pl, 128-byte swizzle
      uint8_t* prow = st + kv * kTcKV + (grp >> 1) * kTcPanel + pl * 128;
      const int sw = pl & 7, c0 = (grp & 1) * 4;
      if (pos < prefix_end) {
        const uint32_t ww[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // word c = dims 8c .. 8c + 7 of the span
          const uint32_t a = *reinterpret_cast<const uint32_t*>(lut + (__byte_perm(ww[c], lane8, 0x5504u) >> 1));
          const uint32_t b = *reinterpret_cast<const uint32_t*>(lut + (__byte_perm(ww[c], lane8, 0x5514u) >> 1));
          const uint32_t d = *reinterpret_cast<const uint32_t*>(lut + (__byte_perm(ww[c], lane8, 0x5524u) >> 1));
          const uint32_t e = *reinterpret_cast<const uint32_t*>(lut + (__byte_perm(ww[c], lane8, 0x5534u) >> 1));
          *reinterpret_cast<uint4*>(prow + (((c0 + c) ^ sw) << 4)) = make_uint4(a, b, d, e);
        }
        return rawn[u];
      }
      if (pos < kv_end) {
        const __half* src = (kv ? p.vr : p.kr) + (int64_t(pos - p.prefix_len) * kHkv + h) * kD + 32 * grp;
#pragma unroll
        for (int c = 0; c < 4; ++c) cp_async16(smem_u32(prow + (((c0 + c) ^ sw) << 4)), src + 8 * c);
        return 1.f;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(prow + (((c0 + c) ^ sw) << 4)) = make_uint4(0, 0, 0, 0);
      return 0.f;
    };
    int32_t pg_next = 0;   // page of tile j + 2
    if (grp_id < n_tiles) {
      const int32_t pg0 = page_of(grp_id);
      pg_next = page_of(grp_id + 2);
#pragma unroll
      for (int u = 0; u < kTcUnits; ++u) fetch(grp_id, u, pg0);
    }
    volatile float* kmax = reinterpret_cast<volatile float*>(misc) + 8 + 4 * grp_id;
    for (int j = grp_id; j < n_tiles; j += 2) {
      const int32_t pg_far = page_of(j + 4);
      const bool more = j + 2 < n_tiles;
      const bool chunk_rows = (j + 1) * kTcTile > prefix_end;   // this tile reaches the chunk (or past it)
      float kn[4];
      // ---- K half: free once QK(j - 2) has run
      if (j >= 2 && !bounded_wait(bar_k_empty + 8 * grp_id, ((j >> 1) - 1) & 1)) break;
      float big = chunk_rows ? INFINITY : 0.f;   // largest K norm; chunk rows always take the q' lo pass
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        kn[u] = expand(j, u);
        big = fmaxf(big, kn[u]);
      }
      cp_async_commit();
      cp_async_wait<0>();
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) big = fmaxf(big, __shfl_xor_sync(0xffffffffu, big, o));
      if (lane == 0) kmax[(w - kTcSoftWarps) & 3] = big;   // read by the MMA thread after k_full
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy writes -> tensor-core reads
      mbar_arrive(bar_k_full + 8 * grp_id);
      // the next tile's loads go out only now: the wait and the proxy fence above
      // would otherwise wait for them as well
      if (more) {
#pragma unroll
        for (int u = 0; u < 4; ++u) fetch(j + 2, u, pg_next);
      }
      // ---- V half and both norms: free once PV(j - 2) has run
      if (j >= 2 && !bounded_wait(bar_v_empty + 8 * grp_id, ((j >> 1) - 1) & 1)) break;
#pragma unroll
      for (int u = 4; u < 8; ++u) {
        const float vn = expand(j, u);
        if (grp == 0) {
          const int pl = 4 * (((gt >> 5) + 4 * u) & 15) + pl_lo;
          nb[pl] = kn[u - 4] * kLog2e;
          nb[kTcTile + pl] = vn * kTcPScale;
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      mbar_arrive(bar_v_full + 8 * grp_id);
      if (more) {
#pragma unroll
        for (int u = 4; u < 8; ++u) fetch(j + 2, u, pg_next);
      }
      pg_next = pg_far;
    }
  } else {
    // =========================================================== MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc_idesc(kTcRows, kTcTile, 0);
      constexpr uint32_t idesc_pv = tc_idesc(kTcRows, kD, 1);
      bool ok = bounded_wait(bar_p_full + 8, 0);   // Q' stored
      tc_fence_after();
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {   // S[j & 1] = Q'hi K_j^T + Q'lo K_j^T  (K = 256 dims in 16 steps each)
          const int b = j & 1;
          if (!bounded_wait(bar_k_full + 8 * b, (j >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t kbase = sbase + kTcStageOff + b * kTcStage;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint64_t bd = tc_sdesc(kbase + (kk >> 2) * kTcPanel + (kk & 3) * 32, 16, 1024);
            tc_mma(tmem + kTmS0 + 64 * b, tmem + kTmQ + 8 * kk, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          const volatile float* km = reinterpret_cast<const volatile float*>(misc) + 8 + 4 * b;
          if (fmaxf(fmaxf(km[0], km[1]), fmaxf(km[2], km[3])) > kQloNorm) {
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
              const uint64_t ad = tc_sdesc(sbase + kTcQloOff + (kk >> 2) * kTcQloPanel + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = tc_sdesc(kbase + (kk >> 2) * kTcPanel + (kk & 3) * 32, 16, 1024);
              tc_mma_ss(tmem + kTmS0 + 64 * b, ad, bd, idesc_qk, 1u);
            }
          }
          tc_commit(bar_s_full + 8 * b);
          tc_commit(bar_k_empty + 8 * b);
        }
        if (j >= 1) {   // O += P_hi V + P_lo V for tile j - 1 (K = 64 positions in 4 steps)
          const int jb = j - 1, b = jb & 1;
          // p_full[1] completed one extra phase for Q': its tile phases are shifted by one
          const uint32_t par = b ? (((jb >> 1) + 1) & 1) : ((jb >> 1) & 1);
          if (!bounded_wait(bar_p_full + 8 * b, par)) break;
          if (!bounded_wait(bar_v_full + 8 * b, (jb >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t vbase = sbase + kTcStageOff + b * kTcStage + kTcKV;
#pragma unroll
          for (int ks = 0; ks < kTcTile / 16; ++ks) {
            const uint64_t bd = tc_sdesc(vbase + ks * 16 * 128, kTcPanel, 1024);
            tc_mma(tmem + kTmO, tmem + kTmS0 + 64 * b + 8 * ks, bd, idesc_pv, (jb > 0 || ks > 0) ? 1u : 0u);
            tc_mma(tmem + kTmO, tmem + kTmS0 + 64 * b + 32 + 8 * ks, bd, idesc_pv, 1u);
          }
          tc_commit(bar_v_empty + 8 * b);
          tc_commit(bar_o_ready);
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      tc_commit(bar_drain);
      for (uint32_t spins = 0; !tc_try_wait(bar_drain, 0) && spins < kTcSpin; ++spins) {
      }
    }
    __syncwarp();
  }

  // =========================================================== R^T per row, bf16 out; free TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
  const float* os = reinterpret_cast<const float*>(smem + kTcStageOff);
  uint32_t sgn = 0;   // sign bits of coordinates 8 lane .. 8 lane + 7 (constant indices keep p in registers)
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t wk = p.signs.bits[k];
    asm("" : "+r"(wk));   // keep the selection as selects (no indexed copy of the parameters)
    sgn = ((lane >> 2) == k) ? wk : sgn;
  }
  sgn = (sgn >> (8 * (lane & 3))) & 0xFFu;
  for (int rl = w; rl < kTcRows; rl += kTcThreads / 32) {
    const int row = row0 + rl;
    if (row >= m_total) break;
    float v[8];
    const float4 a = *reinterpret_cast<const float4*>(os + rl * kTcOsStride + lane * 8);
    const float4 c = *reinterpret_cast<const float4*>(os + rl * kTcOsStride + lane * 8 + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
    warp_fwht256(v);
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(__float_as_uint(v[2 * i]) ^ (((sgn >> (2 * i)) & 1u) << 31)),
                                                __uint_as_float(__float_as_uint(v[2 * i + 1]) ^ (((sgn >> (2 * i + 1)) & 1u) << 31)));
      pk[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    const int tok = row / 6, jh = row % 6;
    *reinterpret_cast<uint4*>(p.out + (int64_t(tok) * kHq + h * kGroup + jh) * kD + lane * 8) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

inline cudaError_t prefill_tc_set_attrs() {
  return cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kTcSmem));
}

// rotate prologue, then the tcgen05 attention kernel
inline cudaError_t launch_prefill_tc(const uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                                     int32_t prefix_len, const uint16_t* q, const uint16_t* kc,
                                     const uint16_t* vc, int32_t n_tok, float scale, uint16_t* out,
                                     void* workspace, const Signs& signs, int* status, cudaStream_t stream) {
  __half* qr = static_cast<__half*>(workspace);
  __half* qlo = qr + size_t(n_tok) * kHq * kD;
  __half* kr = qlo + size_t(n_tok) * kHq * kD;
  __half* vr = kr + size_t(n_tok) * kHkv * kD;
  const int64_t vecs = int64_t(n_tok) * (kHq + 2 * kHkv);
  cudaError_t e = launch_pdl(prefill_rotate_kernel, dim3(unsigned((vecs + 7) / 8)), dim3(256), 0, stream, q, kc, vc,
                             n_tok, scale, qr, qlo, kr, vr, signs);
  if (e != cudaSuccess) return e;
  PrefillParams p{};
  p.pool = pool;
  p.num_pages = num_pages;
  p.page_table = page_table;
  p.prefix_len = prefix_len;
  p.n_tok = n_tok;
  p.qr = qr;
  p.qlo = qlo;
  p.kr = kr;
  p.vr = vr;
  p.out = out;
  p.signs = signs;
  p.status = status;
  const dim3 grid(unsigned((6 * n_tok + kTcRows - 1) / kTcRows), kHkv);
  return launch_pdl(prefill_tc_kernel, grid, dim3(kTcThreads), size_t(kTcSmem), stream, p);
}

}  // namespace tq4
