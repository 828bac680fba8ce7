// TQ4 prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM),
// one CTA pair per 256 query rows (cta_group::2), sm_100a.
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
// Precision. Every tensor-core operand is an f16 hi + lo pair: q' = q'hi + q'lo,
// a centroid c = c16 + r16 (c16 = f16(c), r16 = f16(c - c16)), chunk rows
// likewise, P = Phi + Plo. The scores take the three terms that matter
// (q'hi Khi + q'lo Khi + q'hi Klo); O takes Phi Vhi + Plo Vhi, plus Phi Vlo on
// tiles whose largest V norm exceeds kVloNorm and on every tile when the output is
// fp32 (the fp32 check holds the result to ~1e-5 relative).
//
// Work split. A cluster of two CTAs (ranks 0 and 1) owns 256 query rows
// (row = token * 6 + head within the KV head's group; rank r holds rows
// 128 r .. 128 r + 127, one per TMEM lane) of one KV head and walks KV tiles of
// 64 positions. The pair's MMAs have M = 256: A (q' or P) is split by rows, B by
// its N columns and each CTA keeps its 128 rows of D. So each CTA expands only
// half of every tile: K for positions 32 r .. 32 r + 31 (all 256 dims) and V for
// dims 128 r .. 128 r + 127 (all 64 positions).
//   warps 0-3   softmax: thread i of warp w owns row 32w + i = TMEM lane. Puts
//               its q' hi row into TMEM and its q' lo row into shared memory.
//               Reads its score row from TMEM, applies K norms, the causal mask
//               and an online softmax with a lazily raised reference; writes
//               P = p * n_v / 16 over S (f16 hi and lo).
//   warps 4-11  dequant, two groups of four; group g fills stage g for tiles
//               g, g+2, ...: packed words are prefetched into registers two
//               tiles ahead and expanded through a per-lane table of 8-byte
//               {hi pair, lo pair} slots into swizzled f16 panels (K hi, K lo,
//               V hi, V lo); chunk rows are copied from the prologue's output.
//   warp 12     rank 0 only: one thread issues every tcgen05.mma of the pair, in
//               the order QK(j), PV(j-1), and commits to both CTAs' barriers.
// TMEM (512 columns per CTA): q'hi [0,128), S/P buffers [128,192) and
// [192,256), O [256,512).
// Producers signal the issuer through barriers in rank 0's shared memory (lane 0
// of each producer warp arrives after the warp's writes, from either CTA); the
// issuer's commits arrive on both CTAs' barriers. Every wait is bounded by
// spin_limit polls; on a timeout the CTA records TQ4_ERR_TIMEOUT, raises the
// abort flag of both CTAs, skips the remaining work, drains its issued MMAs and
// frees its TMEM after a cluster barrier.
#pragma once
#include "tq4_device.cuh"
#include "tq4_prefill.cuh"

namespace tq4 {

constexpr int kPfRows = 128;                       // query rows per CTA; a pair covers 256
constexpr int kPfTile = 64;                        // KV positions per tile
constexpr int kPfKPos = kPfTile / 2;               // K positions each CTA expands per tile
constexpr int kPfSoftWarps = 4, kPfDeqWarps = 8;
constexpr int kPfMmaWarp = kPfSoftWarps + kPfDeqWarps;   // 12
constexpr int kPfThreads = 32 * (kPfMmaWarp + 1);        // 416
constexpr int kPfGroupThreads = 128;                     // one dequant group
constexpr uint32_t kPfKPanel = kPfKPos * 128;            // 4 KiB: 32 positions x 64 dims f16
constexpr uint32_t kPfKPart = 4 * kPfKPanel;             // 16 KiB: K hi (or lo), 4 dim blocks
constexpr uint32_t kPfVPanel = kPfTile * 128;            // 8 KiB: 64 positions x 64 dims f16
constexpr uint32_t kPfVPart = 2 * kPfVPanel;             // 16 KiB: V hi (or lo), this CTA's 2 dim blocks
constexpr uint32_t kPfKHi = 0, kPfKLo = kPfKPart, kPfVHi = 2 * kPfKPart, kPfVLo = 2 * kPfKPart + kPfVPart;
constexpr uint32_t kPfStage = 2 * kPfKPart + 2 * kPfVPart;   // 64 KiB
constexpr uint32_t kPfQloPanel = kPfRows * 128;             // 16 KiB: 128 rows x 64 dims f16
constexpr uint32_t kPfQloOff = 2 * kPfStage;                 // two stages first
constexpr uint32_t kPfLutOff = kPfQloOff + 4 * kPfQloPanel;
constexpr uint32_t kPfLutBytes = 256 * 16 * 8;              // 256 byte values x 16 copies x 8 B
constexpr uint32_t kPfNormOff = kPfLutOff + kPfLutBytes;     // [2 stages][K 64, V 64] f32
constexpr uint32_t kPfBarOff = kPfNormOff + 2 * 2 * kPfTile * 4;
constexpr uint32_t kPfMiscOff = kPfBarOff + 256;   // u32 [0] TMEM base, [1] abort; f32 [8 + 2 stage + k] V norm max
constexpr uint32_t kPfSmem = kPfMiscOff + 128 + 1024;    // + alignment slack
constexpr int kPfOsStride = kD + 4;                      // epilogue rows (fp32) reuse the stages + q' lo
static_assert(uint32_t(kPfRows * kPfOsStride * 4) <= kPfLutOff, "epilogue rows overlap the table");
static_assert(kPfSmem <= 227u * 1024u, "shared memory");
static_assert(kPfQloOff % 1024 == 0 && kPfStage % 1024 == 0 && kPfKPart % 1024 == 0 && kPfKPanel % 1024 == 0,
              "swizzled panels start on 1 KiB");
// P = p * n_v * kPfPScale, undone in the epilogue. p <= 2^8 (the lazy reference) and
// n_v stays below ~300 even for 8x outliers, so P < 4,800 fits f16; a larger scale
// keeps the small weights of dense rows (n_v = 1: chunk rows, reconstructed prefix
// rows) out of f16's subnormal range.
constexpr float kPfPScale = 1.0f / 16.0f;
constexpr float kPfLazy = 8.0f;              // raise the row reference only when the max grows by > 2^8

// TMEM columns
constexpr uint32_t kTmQ = 0, kTmS0 = 128, kTmO = 256;

// barriers (8 B each at kPfBarOff): in rank 0, counted from both CTAs
constexpr int kBQReady = 0, kBKFull = 1, kBVFull = 3, kBPFull = 5;
// in each CTA: committed by the issuer to both CTAs, or local. S_FULL(b) completes when
// QK of a stage-b tile is done (its scores are in TMEM, its K half is free); V_EMPTY(b)
// when PV of a stage-b tile is done (its V half is free, O holds it).
constexpr int kBSFull = 7, kBVEmpty = 9, kBDrain = 11, kBNFull = 12;
constexpr int kBarriers = 14;
static_assert(kBarriers * 8 <= 256, "barrier area");

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

// pair MMA, A from TMEM (each CTA's rows at the same address)
__device__ __forceinline__ void tc2_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// pair MMA, A from shared memory (each CTA's rows at the same offset)
__device__ __forceinline__ void tc2_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// completion of this thread's earlier MMAs -> one arrival on the barrier at this
// offset in both CTAs of the pair
__device__ __forceinline__ void tc2_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::"r"(
          bar),
      "h"(uint16_t(3))
      : "memory");
}
// ... on this CTA's barrier only
__device__ __forceinline__ void tc2_commit_own(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// the shared::cluster address of offset `addr` (a shared::cta address) in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// arrive (release, cluster scope) on a barrier given by its shared::cluster address
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// acquire at cluster scope: arrivals may come from the peer CTA
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// one non-blocking look at the phase (acquire, cluster scope)
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\nbarrier.cluster.wait.acquire;\n" ::: "memory");
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1) prefill_tc_kernel(const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t sbase = (raw_s + 1023) & ~1023u;   // the swizzled panels need 1 KiB alignment
  uint8_t* smem = smem_raw + (sbase - raw_s);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int h = blockIdx.y;
  // pair unit u = row block rb, KV segment seg: segment seg of n_seg covers tiles
  // [t0, t0 + n_tiles) of the row block's range (one segment: the whole range)
  const int unit = int(blockIdx.x >> 1), rb = unit / p.n_seg, seg = unit % p.n_seg;
  const int pair_row0 = rb * (2 * kPfRows);
  const int row0 = pair_row0 + int(rank) * kPfRows;
  const int m_total = 6 * p.n_tok;
  const int last_row = min(pair_row0 + 2 * kPfRows, m_total) - 1;   // the pair's last row
  const int kv_end = p.prefix_len + last_row / 6 + 1;
  const int n_all = (kv_end + kPfTile - 1) / kPfTile;
  const int t0 = int(int64_t(seg) * n_all / p.n_seg);
  const int n_tiles = int(int64_t(seg + 1) * n_all / p.n_seg) - t0;   // local tile j is tile t0 + j
  const bool exact = p.out_dtype == TQ4_DTYPE_F32;

  auto bar = [sbase](int i) -> uint32_t { return sbase + kPfBarOff + 8u * uint32_t(i); };
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kPfMiscOff);   // [0] TMEM base, [1] abort
  float* norms = reinterpret_cast<float*>(smem + kPfNormOff);
  const uint32_t lead_bar0 = map_to_rank(bar(0), 0);   // rank 0's barrier area, seen from this CTA

  if (tid == 0) {
    mbar_init(bar(kBQReady), 2 * kPfSoftWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kBKFull + b), 2 * (kPfGroupThreads / 32));
      mbar_init(bar(kBVFull + b), 2 * (kPfGroupThreads / 32));
      mbar_init(bar(kBPFull + b), 2 * kPfSoftWarps);
      mbar_init(bar(kBSFull + b), 1);
      mbar_init(bar(kBVEmpty + b), 1);
      mbar_init(bar(kBNFull + b), kPfGroupThreads / 32);
    }
    mbar_init(bar(kBDrain), 1);
    misc[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (w == 0) {   // 512 TMEM columns in both CTAs; shared memory admits one CTA per SM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(sbase + kPfMiscOff)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  // per-lane centroid table: row b (a byte = two indices, 128 B) holds, in each of
  // 16 copies, the 8-byte slot {c16 pair, r16 pair}; lanes l and l + 16 share copy
  // l & 15, so each half warp's 64-bit loads hit 32 different banks
  for (int e = tid; e < 256 * 16; e += kPfThreads)
    reinterpret_cast<uint2*>(smem + kPfLutOff)[e] = lut_row(e >> 4);
  pdl_wait();   // q', the chunk rows and the pool may come from the previous kernels
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = misc[0];

  int* const status = p.status;
  const uint32_t spin_limit = p.spin_limit;
  const uint32_t peer_abort = map_to_rank(sbase + kPfMiscOff + 4, peer);
  auto abort_both = [misc, status, peer_abort]() {
    misc[1] = 1;
    st_cluster_u32(peer_abort, 1u);
    record_error(status, TQ4_ERR_TIMEOUT);
  };
  auto bounded_wait = [misc, spin_limit, &abort_both](uint32_t b, uint32_t parity) -> bool {
    uint32_t spins = 0;
    while (!mbar_try_wait_cluster(b, parity)) {
      if (misc[1]) return false;
      if (++spins > spin_limit) {
        abort_both();
        return false;
      }
    }
    return true;
  };
  // the softmax warps use TMEM loads/stores that all 32 lanes must execute
  // together, so every wait and every decision before one is taken warp-wide
  auto warp_wait = [&bounded_wait](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, bounded_wait(b, parity));
  };
  // lane 0 signals a producer barrier in rank 0 after the whole warp's writes
  auto warp_arrive_lead = [lead_bar0, lane](int i) {
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(lead_bar0 + 8u * uint32_t(i));
  };

  if (w < kPfSoftWarps) {
    // =========================================================== softmax / epilogue
    const int r_local = 32 * w + lane;
    const int row = row0 + r_local;
    const bool row_ok = row < m_total;
    const int tok = row_ok ? row / 6 : 0;
    const int lim = row_ok ? p.prefix_len + tok + 1 : 0;   // positions [0, lim) are visible
    const uint32_t lane_addr = tmem + (uint32_t(32 * w) << 16);
    {   // q' row -> TMEM columns [0,128) as f16 pairs (A operand of S = Q' K^T)
      const int64_t qrow = (int64_t(tok) * kHq + h * kGroup + (row_ok ? row % 6 : 0)) * kD;
      const uint4* src = reinterpret_cast<const uint4*>(p.qr + qrow);
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
      const uint4* src_lo = reinterpret_cast<const uint4*>(p.qlo + qrow);
      uint8_t* qlo_row = smem + kPfQloOff + r_local * 128;
#pragma unroll 8
      for (int g = 0; g < 32; ++g) {   // g = 16-byte chunk (8 dims)
        const uint4 u = row_ok ? __ldg(src_lo + g) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qlo_row + (g >> 3) * kPfQloPanel + (((g & 7) ^ (r_local & 7)) << 4)) = u;
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy stores -> tensor-core reads
    }
    tc_fence_before();
    warp_arrive_lead(kBQReady);

    float m_ref = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      if (!warp_wait(bar(kBSFull + b), (j >> 1) & 1)) break;
      if (!warp_wait(bar(kBNFull + b), (j >> 1) & 1)) break;   // both norm rows of this tile
      tc_fence_after();
      const float4* kn4 = reinterpret_cast<const float4*>(norms + b * 2 * kPfTile);   // K norm * log2(e)
      const float4* vn4 = kn4 + kPfTile / 4;                                          // V norm / 256
      const int pos0 = (t0 + j) * kPfTile;
      uint32_t sr[2][32];
      tm_ld32(lane_addr + kTmS0 + 64 * b, sr[0]);
      tm_ld32(lane_addr + kTmS0 + 64 * b + 32, sr[1]);
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // scores in log2 units
      if (__all_sync(0xffffffffu, pos0 + kPfTile <= lim)) {           // the whole tile is visible
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
      const bool raise = mx > m_ref + kPfLazy;   // raise the reference: rescale l and the O row accumulated so far
      float alpha = 1.f;
      if (raise) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        l_sum *= alpha;
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
      // PV(j - 1) has completed (V_EMPTY of its stage). Waited for at every tile, not
      // only when O is rescaled: each stage's barrier is then waited for every other
      // tile and never trails this warp by more than one phase, so its parity names
      // one phase only (the final wait below relies on the same).
      if (j > 0) {
        if (!warp_wait(bar(kBVEmpty + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, raise)) {   // lanes that keep their reference use alpha = 1
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
      }
      tc_fence_before();
      // (test hook: tile min(1, n_tiles - 1)'s P signal is withheld, so the issuer's
      // wait for it runs out after some MMAs of the pair have been issued)
      if (!(p.test_withhold && j == min(1, n_tiles - 1))) warp_arrive_lead(kBPFull + b);
    }
    // ---- O / l -> shared memory rows (reusing the stages): wait for the last PV
    const bool ok = __all_sync(0xffffffffu, misc[1] == 0) && warp_wait(bar(kBVEmpty + ((n_tiles - 1) & 1)), ((n_tiles - 1) >> 1) & 1);
    tc_fence_after();
    float* os = reinterpret_cast<float*>(smem) + r_local * kPfOsStride;
    // one segment: o' / l with the scale of P and 1/16 of R^T; several: the raw partial,
    // with (m, l) beside it for the combine pass
    const bool split = p.n_seg > 1;
    const float inv = split ? (ok ? 1.f : 0.f) : (ok && l_sum > 0.f) ? (0.0625f / kPfPScale) / l_sum : 0.f;
    if (split && row_ok)
      p.ws_pml[(int64_t(unit) * kHkv + h) * (2 * kPfRows) + int(rank) * kPfRows + r_local] =
          make_float2(ok ? m_ref : -INFINITY, ok ? l_sum : 0.f);
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
  } else if (w < kPfMmaWarp) {
    // =========================================================== dequant groups
    const int grp_id = (w - kPfSoftWarps) >> 2;                           // stage b == grp_id
    const int gt = tid - 32 * kPfSoftWarps - kPfGroupThreads * grp_id;   // 0..127
    const int wq = gt >> 5;                                               // warp within the group
    // K units: 16 bytes (4 words = 32 dims) of one of this CTA's 32 positions. A
    // quarter warp covers 4 positions x 2 adjacent word groups, so its 16-B stores
    // land in 8 distinct bank groups under the swizzle.
    const int kgrp = (lane & 1) | (((lane >> 3) & 3) << 1);   // word group 0..7 -> dims 32 kgrp ..
    const int kpl_lo = (lane >> 1) & 3;
    // V units: 16 bytes of this CTA's 128 dims (word groups 4 rank .. 4 rank + 3) of one
    // of the tile's 64 positions; again 4 positions x 2 word groups per quarter warp
    const int vgrp = (lane & 1) | (((lane >> 4) & 1) << 1);   // local word group 0..3
    const int vpl_lo = ((lane >> 1) & 3) | (((lane >> 3) & 1) << 2);
    const uint32_t lut_s = sbase + kPfLutOff;
    const uint32_t lane16 = uint32_t(lane & 15) * 16u;   // (byte << 8 | 16 copy) >> 1 = byte * 128 + 8 copy
    const int prefix_end = min(p.prefix_len, kv_end);
    const bool dense = p.pkr != nullptr;   // the prefix comes as reconstructed rows, not packed words
    const uint32_t st_s = sbase + grp_id * kPfStage;
    float* nb = norms + grp_id * 2 * kPfTile;
    const uint8_t* const pool = p.pool;
    const int32_t* const page_table = p.page_table;
    const int32_t num_pages = p.num_pages;

    // tile-local position and source word group of unit u (0, 1: K; 2, 3: V)
    auto unit_pos = [=](int u) -> int {
      return u < 2 ? int(rank) * kPfKPos + 4 * (wq + 4 * u) + kpl_lo : 8 * (wq + 4 * (u - 2)) + vpl_lo;
    };
    auto unit_grp = [=](int u) -> int { return u < 2 ? kgrp : 4 * int(rank) + vgrp; };
    // raw[u]: unit u's packed words for the tile about to be expanded; rawn: the norm
    // this thread loads for the tile (K norm of position gt for gt < 64, V norm of
    // position gt - 64 otherwise). Refilled with the group's next tile (j + 2) right
    // after use, so the loads fly while the stage is waited for. A tile lies in one
    // page; its page id is loaded two tiles ahead of use.
    uint4 raw[4];
    float rawn = 0.f;
    auto page_of = [=](int j) -> int32_t {
      return (j < n_tiles && (t0 + j) * kPfTile < prefix_end) ? __ldg(page_table + (((t0 + j) * kPfTile) >> 8)) : 0;
    };
    auto fetch = [&raw, t0, prefix_end, dense, pool, num_pages, h, status, &unit_pos, &unit_grp](int j, int u,
                                                                                             int32_t page) {
      const int pos = (t0 + j) * kPfTile + unit_pos(u);
      raw[u] = make_uint4(0, 0, 0, 0);
      if (pos < prefix_end && !dense) {
        if (page >= 0 && page < num_pages) {
          const uint8_t* pg = pool + int64_t(page) * kPageBytes;
          const int slot = h * kPage + (pos & (kPage - 1));
          raw[u] = ldg128(pg + (u < 2 ? kKWords : kVWords) + int64_t(slot) * 128 + unit_grp(u) * 16);
        } else {
          record_error(status, TQ4_ERR_PAGE_RANGE);   // words stay 0 and the norm 0: no contribution
        }
      }
    };
    auto fetch_norm = [&rawn, t0, gt, prefix_end, pool, num_pages, h](int j, int32_t page) {
      const int pos = (t0 + j) * kPfTile + (gt & 63);
      rawn = 0.f;
      if (pos < prefix_end && page >= 0 && page < num_pages)
        rawn = ldg_half(pool + int64_t(page) * kPageBytes + (gt < 64 ? kKNorms : kVNorms) +
                        (h * kPage + (pos & (kPage - 1))) * 2);
    };
    // expand unit u of tile j into the stage: hi and lo centroid values for a prefix
    // position, asynchronous copies of the prologue's hi and lo rows for a chunk
    // position, zeros past the pair's last visible position
    auto expand = [&](int j, int u) {
      const int pl = unit_pos(u), pos = (t0 + j) * kPfTile + pl;
      const int g = u < 2 ? kgrp : vgrp;   // word group within the panels of this CTA
      const int sw = pl & 7, c0 = (g & 1) * 4;
      const int prow = (u < 2 ? pl - int(rank) * kPfKPos : pl) * 128;
      const uint32_t hi_s = st_s + (u < 2 ? kPfKHi + (g >> 1) * kPfKPanel : kPfVHi + (g >> 1) * kPfVPanel) + prow;
      const uint32_t lo_s = hi_s + (u < 2 ? kPfKLo - kPfKHi : kPfVLo - kPfVHi);
      if (pos < prefix_end && !dense) {
        const uint32_t ww[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // word c = dims 8c .. 8c + 7 of the span
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          ld_shared_v2(lut_s + (__byte_perm(ww[c], lane16, 0x5504u) >> 1), h0, l0);
          ld_shared_v2(lut_s + (__byte_perm(ww[c], lane16, 0x5514u) >> 1), h1, l1);
          ld_shared_v2(lut_s + (__byte_perm(ww[c], lane16, 0x5524u) >> 1), h2, l2);
          ld_shared_v2(lut_s + (__byte_perm(ww[c], lane16, 0x5534u) >> 1), h3, l3);
          const uint32_t off = uint32_t(((c0 + c) ^ sw) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(hi_s + off), "r"(h0), "r"(h1), "r"(h2),
                       "r"(h3)
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(lo_s + off), "r"(l0), "r"(l1), "r"(l2),
                       "r"(l3)
                       : "memory");
        }
        return;
      }
      if (pos < kv_end) {   // a chunk row, or a reconstructed prefix row
        const bool pre = pos < p.prefix_len;
        const int64_t row = (int64_t(pre ? pos : pos - p.prefix_len) * kHkv + h) * kD + 32 * unit_grp(u);
        const __half* src_hi = (u < 2 ? (pre ? p.pkr : p.kr) : (pre ? p.pvr : p.vr)) + row;
        const __half* src_lo = (u < 2 ? (pre ? p.pkrlo : p.krlo) : (pre ? p.pvrlo : p.vrlo)) + row;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t off = uint32_t(((c0 + c) ^ sw) << 4);
          cp_async16(hi_s + off, src_hi + 8 * c);
          cp_async16(lo_s + off, src_lo + 8 * c);
        }
        return;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = uint32_t(((c0 + c) ^ sw) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};\n" ::"r"(hi_s + off), "r"(0u) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};\n" ::"r"(lo_s + off), "r"(0u) : "memory");
      }
    };
    int32_t pg_next = 0;   // page of tile j + 2
    if (grp_id < n_tiles) {
      const int32_t pg0 = page_of(grp_id);
      pg_next = page_of(grp_id + 2);
#pragma unroll
      for (int u = 0; u < 4; ++u) fetch(grp_id, u, pg0);
      fetch_norm(grp_id, pg0);
    }
    volatile float* vmax_slot = reinterpret_cast<volatile float*>(misc) + 8 + 2 * grp_id;
    for (int j = grp_id; j < n_tiles; j += 2) {
      const int32_t pg_far = page_of(j + 4);
      const bool more = j + 2 < n_tiles;
      // ---- K half: free once QK(j - 2) has run
      if (j >= 2 && !bounded_wait(bar(kBSFull + grp_id), ((j >> 1) - 1) & 1)) break;   // QK(j - 2) done
      expand(j, 0);
      expand(j, 1);
      cp_async_commit();
      cp_async_wait<0>();
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic-proxy writes -> tensor-core reads
      warp_arrive_lead(kBKFull + grp_id);
      // the next tile's loads go out only now: the wait and the proxy fence above
      // would otherwise wait for them as well
      if (more) {
        fetch(j + 2, 0, pg_next);
        fetch(j + 2, 1, pg_next);
      }
      // ---- V half and both norm rows: free once PV(j - 2) has run
      if (j >= 2 && !bounded_wait(bar(kBVEmpty + grp_id), ((j >> 1) - 1) & 1)) break;
      expand(j, 2);
      expand(j, 3);
      {
        const int pl = gt & 63;
        const int pos = (t0 + j) * kPfTile + pl;
        const bool chunk = pos >= prefix_end && pos < kv_end;
        const bool row = chunk || (dense && pos < prefix_end);
        const float n = row ? 1.f : rawn;   // dense rows (chunk or reconstructed) carry their own length
        if (gt < 64) {
          nb[pl] = n * kLog2e;
        } else {
          nb[kPfTile + pl] = n * kPfPScale;
          float m = chunk ? 16.f : rawn;   // the V norm (a rotated N(0,1) chunk row has length ~16)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) vmax_slot[wq - 2] = m;   // read by the issuer after v_full
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive_local(bar(kBNFull + grp_id));
      warp_arrive_lead(kBVFull + grp_id);
      if (more) {
        fetch(j + 2, 2, pg_next);
        fetch(j + 2, 3, pg_next);
        fetch_norm(j + 2, pg_next);
      }
      pg_next = pg_far;
    }
  } else if (rank == 0) {
    // =========================================================== MMA issuer (one thread of rank 0)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc_idesc(2 * kPfRows, kPfTile, 0);
      constexpr uint32_t idesc_pv = tc_idesc(2 * kPfRows, kD, 1);
      bool ok = bounded_wait(bar(kBQReady), 0);   // q' of both CTAs stored
      tc_fence_after();
      // Waits on barriers that have long completed still cost hundreds of cycles, and
      // between two MMA bursts they would leave the tensor pipe idle. The issue of an
      // MMA blocks while the tensor core's queue is full, so the next burst's barriers
      // are looked at (non-blocking) between the MMAs of the current one; the blocking,
      // bounded wait runs only for a barrier not yet seen complete.
      bool k_seen = false;    // K_FULL of the next QK seen complete during the last PV burst
      for (int j = 0; ok && j <= n_tiles; ++j) {
        bool pv_seen = false;   // P_FULL and V_FULL of tile j - 1 seen complete during the QK burst
        const int jb = j - 1, bp = jb & 1;
        const uint32_t pv_par = uint32_t(jb >> 1) & 1u;
        auto look_pv = [&]() {
          if (j >= 1 && !pv_seen)
            pv_seen = mbar_test_wait_cluster(bar(kBPFull + bp), pv_par) && mbar_test_wait_cluster(bar(kBVFull + bp), pv_par);
        };
        if (j < n_tiles) {   // S[j & 1] = Q'hi Khi^T + Q'lo Khi^T + Q'hi Klo^T  (K = 256 dims in 16 steps each)
          const int b = j & 1;
          if (!k_seen && !bounded_wait(bar(kBKFull + b), (j >> 1) & 1)) break;
          k_seen = false;
          tc_fence_after();
          const uint32_t kb = sbase + b * kPfStage;
          const uint32_t s_t = tmem + kTmS0 + 64 * b;
          // descriptors of the panels' first rows; a k-step adds its byte offset >> 4 to the
          // start-address field (no carry: shared addresses stay below 2^18)
          const uint64_t khi0 = tc_sdesc(kb + kPfKHi, 16, 1024), klo0 = tc_sdesc(kb + kPfKLo, 16, 1024);
          const uint64_t qlo0 = tc_sdesc(sbase + kPfQloOff, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint64_t o = uint64_t(((kk >> 2) * kPfKPanel + (kk & 3) * 32) >> 4);
            tc2_mma_ts(s_t, tmem + kTmQ + 8 * kk, khi0 + o, idesc_qk, kk > 0 ? 1u : 0u);
          }
          look_pv();
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint64_t o = uint64_t(((kk >> 2) * kPfKPanel + (kk & 3) * 32) >> 4);
            const uint64_t oq = uint64_t(((kk >> 2) * kPfQloPanel + (kk & 3) * 32) >> 4);
            tc2_mma_ss(s_t, qlo0 + oq, khi0 + o, idesc_qk, 1u);
          }
          look_pv();
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint64_t o = uint64_t(((kk >> 2) * kPfKPanel + (kk & 3) * 32) >> 4);
            tc2_mma_ts(s_t, tmem + kTmQ + 8 * kk, klo0 + o, idesc_qk, 1u);
          }
          look_pv();
          // S_FULL also tells the dequant group that the K half of stage b is free again
          tc2_commit_both(bar(kBSFull + b));
        }
        if (j >= 1) {   // O += P_hi V_hi (+ P_lo V_hi, + P_hi V_lo) for tile j - 1 (K = 64 positions in 4 steps)
          if (!pv_seen) {
            if (!bounded_wait(bar(kBPFull + bp), pv_par)) break;
            if (!bounded_wait(bar(kBVFull + bp), pv_par)) break;
          }
          tc_fence_after();
          const volatile float* vm = reinterpret_cast<const volatile float*>(misc) + 8 + 2 * bp;
          // reconstructed prefix rows carry each value's own f16 rounding (not one fixed
          // residual per centroid), so that path takes the V lo product on every tile
          const bool vlo = exact || p.pkr != nullptr || fmaxf(vm[0], vm[1]) > kVloNorm;
          const uint32_t vb = sbase + bp * kPfStage;
          const uint32_t p_t = tmem + kTmS0 + 64 * bp;
          const uint64_t vhi0 = tc_sdesc(vb + kPfVHi, kPfVPanel, 1024), vlo0 = tc_sdesc(vb + kPfVLo, kPfVPanel, 1024);
          const int jn = j + 1;   // the next QK's tile
#pragma unroll
          for (int ks = 0; ks < kPfTile / 16; ++ks) {
            const uint64_t o = uint64_t((ks * 16 * 128) >> 4);
            tc2_mma_ts(tmem + kTmO, p_t + 8 * ks, vhi0 + o, idesc_pv, (jb > 0 || ks > 0) ? 1u : 0u);
            tc2_mma_ts(tmem + kTmO, p_t + 32 + 8 * ks, vhi0 + o, idesc_pv, 1u);
            if (vlo) tc2_mma_ts(tmem + kTmO, p_t + 8 * ks, vlo0 + o, idesc_pv, 1u);
            if (ks == 1 && jn < n_tiles) k_seen = mbar_test_wait_cluster(bar(kBKFull + (jn & 1)), uint32_t(jn >> 1) & 1u);
          }
          // V_EMPTY: the V half of stage bp is free, and (to the softmax) PV(j - 1) has completed
          tc2_commit_both(bar(kBVEmpty + bp));
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      tc2_commit_own(bar(kBDrain));
      for (uint32_t spins = 0; !mbar_try_wait_cluster(bar(kBDrain), 0) && spins < TQ4_DEFAULT_WAIT_POLLS; ++spins) {
      }
    }
    __syncwarp();
  }

  // =========================================================== R^T per row, out; free TMEM
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no MMA of the pair and no remote access is outstanding past this point
  tc_fence_after();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
  const float* os = reinterpret_cast<const float*>(smem);
  uint32_t sgn = 0;   // sign bits of coordinates 8 lane .. 8 lane + 7 (constant indices keep p in registers)
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t wk = p.signs.bits[k];
    asm("" : "+r"(wk));   // keep the selection as selects (no indexed copy of the parameters)
    sgn = ((lane >> 2) == k) ? wk : sgn;
  }
  sgn = (sgn >> (8 * (lane & 3))) & 0xFFu;
  for (int rl = w; rl < kPfRows; rl += kPfThreads / 32) {
    const int row = row0 + rl;
    if (row >= m_total) break;
    float v[8];
    const float4 a = *reinterpret_cast<const float4*>(os + rl * kPfOsStride + lane * 8);
    const float4 c = *reinterpret_cast<const float4*>(os + rl * kPfOsStride + lane * 8 + 4);
    if (p.n_seg > 1) {   // the segment's partial row; the combine pass merges, rotates and stores
      float* dst = p.ws_po + ((int64_t(unit) * kHkv + h) * (2 * kPfRows) + int(rank) * kPfRows + rl) * kD + lane * 8;
      reinterpret_cast<float4*>(dst)[0] = a;
      reinterpret_cast<float4*>(dst)[1] = c;
      continue;
    }
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
    warp_fwht256(v);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((sgn >> i) & 1u) << 31));
    const int tok = row / 6, jh = row % 6;
    const int64_t off = (int64_t(tok) * kHq + h * kGroup + jh) * kD + lane * 8;
    if (exact) {
      float* dst = static_cast<float*>(p.out) + off;
      reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        pk[i] = *reinterpret_cast<uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

// Merge of a row's KV segments (several segments per row block): one warp per
// (row, KV head): m = max m_s, o' = sum 2^(m_s - m) o'_s, l = sum 2^(m_s - m) l_s
// (m in log2 units), then o = R^T (o' / l) with the scale of P, as the attention
// kernel's own epilogue does with one segment.
__global__ void __launch_bounds__(256) prefill_combine_kernel(const PrefillParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int m_total = 6 * p.n_tok;
  pdl_wait();
  pdl_launch_dependents();
  if (wid >= int64_t(m_total) * kHkv) return;
  const int h = int(wid % kHkv), row = int(wid / kHkv);
  const int rb = row / (2 * kPfRows), rr = row % (2 * kPfRows);
  float M = -INFINITY;
  for (int s = 0; s < p.n_seg; ++s)
    M = fmaxf(M, p.ws_pml[(int64_t(rb * p.n_seg + s) * kHkv + h) * (2 * kPfRows) + rr].x);
  float L = 0.f, o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.n_seg; ++s) {
      const int64_t rec = (int64_t(rb * p.n_seg + s) * kHkv + h) * (2 * kPfRows) + rr;
      const float2 ml = p.ws_pml[rec];
      const float wgt = fast_exp2(ml.x - M);   // 0 for a segment that saw nothing of this row
      L = fmaf(wgt, ml.y, L);
      const float4* src = reinterpret_cast<const float4*>(p.ws_po + rec * kD + lane * 8);
      const float4 a = src[0], c = src[1];
      o[0] = fmaf(wgt, a.x, o[0]); o[1] = fmaf(wgt, a.y, o[1]); o[2] = fmaf(wgt, a.z, o[2]);
      o[3] = fmaf(wgt, a.w, o[3]); o[4] = fmaf(wgt, c.x, o[4]); o[5] = fmaf(wgt, c.y, o[5]);
      o[6] = fmaf(wgt, c.z, o[6]); o[7] = fmaf(wgt, c.w, o[7]);
    }
  }
  warp_fwht256(o);
  const float inv = (L > 0.f) ? (0.0625f / kPfPScale) / L : 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] *= inv * sign_of(p.signs, lane * 8 + i);
  const int tok = row / 6, jh = row % 6;
  const int64_t off = (int64_t(tok) * kHq + h * kGroup + jh) * kD + lane * 8;
  if (p.out_dtype == TQ4_DTYPE_F32) {
    float* dst = static_cast<float*>(p.out) + off;
    reinterpret_cast<float4*>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
  } else {
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      pk[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// KV segments per row block: the fewest that fill the SMs' pair slots (one pair per
// two SMs) to within a few percent over the waves the units take; several only when
// every segment keeps at least 8 prefix tiles.
inline int prefill_segments(int n_tok, int prefix_len, int num_sms) {
  const int64_t pairs = int64_t((6 * n_tok + 2 * kPfRows - 1) / (2 * kPfRows)) * kHkv;
  const int64_t slots = std::max(num_sms / 2, 1);
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= kPfMaxSegments; ++s) {
    if (s > 1 && prefix_len < s * 8 * kPfTile) break;
    const int64_t units = pairs * s;
    const double eff = double(units) / double(((units + slots - 1) / slots) * slots) - 0.02 * (s - 1);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

inline cudaError_t prefill_tc_set_attrs() {
  return cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPfSmem));
}

// rotate prologue (and, with reconstruct, the prefix's dense rows), then the
// tcgen05 attention kernel (clusters of two CTAs). bits: 4 (TQ4 pool), or 2 / 3,
// whose pools are always rebuilt as dense rows first and are read by that rebuild
// only (the attention kernel gets no packed pool).
inline cudaError_t launch_prefill_tc(const uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                                     int32_t prefix_len, const uint16_t* q, const uint16_t* kc,
                                     const uint16_t* vc, int32_t n_tok, float scale, void* out, int out_dtype,
                                     void* workspace, const Signs& signs, int* status, uint32_t spin_limit,
                                     int test_withhold, cudaStream_t stream, int num_sms, bool reconstruct = false,
                                     int bits = 4) {
  __half* qr = static_cast<__half*>(workspace);
  __half* qlo = qr + size_t(n_tok) * kHq * kD;
  __half* kr = qlo + size_t(n_tok) * kHq * kD;
  __half* krlo = kr + size_t(n_tok) * kHkv * kD;
  __half* vr = krlo + size_t(n_tok) * kHkv * kD;
  __half* vrlo = vr + size_t(n_tok) * kHkv * kD;
  const int64_t vecs = int64_t(n_tok) * (kHq + 2 * kHkv);
  cudaError_t e = launch_pdl(prefill_rotate_kernel, dim3(unsigned((vecs + 7) / 8)), dim3(256), 0, stream, q, kc, vc,
                             n_tok, scale, qr, qlo, kr, krlo, vr, vrlo, signs);
  if (e != cudaSuccess) return e;
  PrefillParams p{};
  // segment partials after the chunk's rows, then (with reconstruct) the prefix rows
  const int64_t pairs = (6 * n_tok + 2 * kPfRows - 1) / (2 * kPfRows);
  p.n_seg = prefill_segments(n_tok, prefix_len, num_sms);
  p.ws_po = reinterpret_cast<float*>(vrlo + size_t(n_tok) * kHkv * kD);
  p.ws_pml = reinterpret_cast<float2*>(p.ws_po + size_t(pairs) * kPfMaxSegments * kHkv * (2 * kPfRows) * kD);
  if ((reconstruct || bits != 4) && prefix_len > 0) {   // rows after the partials: [prefix_len][4][256] each
    __half* rows = reinterpret_cast<__half*>(p.ws_pml + size_t(pairs) * kPfMaxSegments * kHkv * (2 * kPfRows));
    const size_t n = size_t(prefix_len) * kHkv * kD;
    p.pkr = rows;
    p.pkrlo = rows + n;
    p.pvr = rows + 2 * n;
    p.pvrlo = rows + 3 * n;
    const int64_t rvecs = int64_t(prefix_len) * kHkv * 2;
    const dim3 rgrid(unsigned((rvecs + 7) / 8));
    if (bits == 2)
      e = launch_pdl(prefill_reconstruct_rows_bits_kernel<2>, rgrid, dim3(256), 0, stream, pool, num_pages,
                     page_table, prefix_len, rows, rows + n, rows + 2 * n, rows + 3 * n, status);
    else if (bits == 3)
      e = launch_pdl(prefill_reconstruct_rows_bits_kernel<3>, rgrid, dim3(256), 0, stream, pool, num_pages,
                     page_table, prefix_len, rows, rows + n, rows + 2 * n, rows + 3 * n, status);
    else
      e = launch_pdl(prefill_reconstruct_rows_kernel, rgrid, dim3(256), 0, stream, pool, num_pages, page_table,
                     prefix_len, rows, rows + n, rows + 2 * n, rows + 3 * n, status);
    if (e != cudaSuccess) return e;
  }
  p.pool = bits == 4 ? pool : nullptr;   // a b-bit pool has been read by the rebuild above
  p.num_pages = bits == 4 ? num_pages : 0;
  p.page_table = page_table;
  p.prefix_len = prefix_len;
  p.n_tok = n_tok;
  p.qr = qr;
  p.qlo = qlo;
  p.kr = kr;
  p.krlo = krlo;
  p.vr = vr;
  p.vrlo = vrlo;
  p.out = out;
  p.out_dtype = out_dtype;
  p.signs = signs;
  p.status = status;
  p.spin_limit = spin_limit;
  p.test_withhold = test_withhold;
  e = launch_pdl(prefill_tc_kernel, dim3(unsigned(2 * pairs * p.n_seg), kHkv), dim3(kPfThreads), size_t(kPfSmem),
                 stream, p);
  if (e != cudaSuccess || p.n_seg == 1) return e;
  const int64_t warps = int64_t(6) * n_tok * kHkv;
  return launch_pdl(prefill_combine_kernel, dim3(unsigned((warps + 7) / 8)), dim3(256), 0, stream, p);
}

}  // namespace tq4
