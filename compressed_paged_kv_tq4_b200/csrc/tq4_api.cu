// C ABI of the TQ4 paged-KV attention library: context, argument checks,
// planning and launches. Every kernel of the library is compiled in this one
// translation unit (the kernel headers are included below).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tq4.h"
#include "tq4_device.cuh"
#include "tq4_encode.cuh"
#include "tq4_decode.cuh"
#include "tq4_decode_q1.cuh"
#include "tq4_prefill.cuh"
#include "tq4_prefill_tc.cuh"
#include "tq4_decode_tc.cuh"

struct tq4_ctx {
  int device;
  int num_sms;
  tq4::Signs signs;
  double centroids[16];
  double boundaries[15];
  int* d_status;
  uint32_t wait_polls;   // bounded device waits give up after this many polls
  int withhold;          // test hook: kernels withhold one producer signal (see tq4_ctx_set_wait_limit)
  void* noalloc_scratch; // device address of the library's fixed split-K array on this device
  int decode_path;       // TQ4_DECODE_PATH_*: which kernel decodes 2-4 query tokens
  double centroids_b[2][8];   // the 2- and 3-bit variants' fp64 codebooks (4 and 8 levels)
  double boundaries_b[2][7];
};

namespace {

// ---------------------------------------------------------------------------
// 16-level Lloyd-Max quantiser for N(0, sigma^2) in fp64: alternate the two
// optimality conditions (boundaries at centroid midpoints; centroids at the
// Gaussian conditional mean of their cell) until nothing moves. The Gaussian
// density is log-concave, so the fixed point is unique and the starting
// spread does not matter.
// ---------------------------------------------------------------------------
double std_normal_pdf(double z) { return std::isinf(z) ? 0.0 : std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI); }

void lloyd_max_levels(int levels, double sigma, double* c, double* b) {
  for (int j = 0; j < levels; ++j) c[j] = sigma * (-2.5 + 5.0 * j / double(levels - 1));
  for (int it = 0; it < 200000; ++it) {
    for (int j = 0; j + 1 < levels; ++j) b[j] = 0.5 * (c[j] + c[j + 1]);
    double moved = 0.0;
    double cn[16];
    for (int j = 0; j < levels; ++j) {
      const double lo = j == 0 ? -INFINITY : b[j - 1] / sigma;
      const double hi = j == levels - 1 ? INFINITY : b[j] / sigma;
      // P(lo < Z < hi) = (erfc(lo/sqrt2) - erfc(hi/sqrt2)) / 2
      const double mass = 0.5 * (std::erfc(lo / M_SQRT2) - std::erfc(hi / M_SQRT2));
      cn[j] = sigma * (std_normal_pdf(lo) - std_normal_pdf(hi)) / mass;
      moved = std::fmax(moved, std::fabs(cn[j] - c[j]));
    }
    std::memcpy(c, cn, sizeof(double) * levels);
    if (moved < 1e-19) break;
  }
  for (int j = 0; j + 1 < levels; ++j) b[j] = 0.5 * (c[j] + c[j + 1]);
}
void lloyd_max_16(double sigma, double c[16], double b[15]) { lloyd_max_levels(16, sigma, c, b); }

uint16_t half_bits(double x) {
  const __half h = __double2half(x);
  uint16_t u;
  std::memcpy(&u, &h, 2);
  return u;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? TQ4_OK : TQ4_ERR_CUDA; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_device(const tq4_ctx* ctx) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ4_ERR_CUDA;
  return dev == ctx->device ? TQ4_OK : TQ4_ERR_ARG;
}

template <int NT, int NTG, bool kI8>
cudaError_t set_decode_attrs() {
  cudaError_t e = cudaFuncSetAttribute(tq4::decode_splitk_kernel<NT, NTG, kI8, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(tq4::decode_smem_bytes<NT, NTG, kI8>()));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tq4::decode_splitk_kernel<NT, NTG, kI8, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(tq4::decode_smem_bytes<NT, NTG, kI8>()));
  return e;
}

template <int NT>
cudaError_t set_decode_tc_attrs() {
  cudaError_t e = cudaFuncSetAttribute(tq4::decode_tc_kernel<NT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(tq4::kDtSmem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tq4::decode_tc_kernel<NT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(tq4::kDtSmem));
  return e;
}
// the tensor-memory decode of 2-4 query tokens (n-tiles 2 or 3)
cudaError_t launch_decode_tc(int nt, dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  const bool exact = p.out_dtype == TQ4_DTYPE_F32;
  const dim3 block(tq4::kDtThreads);
  const size_t smem = tq4::kDtSmem;
  if (nt == 2)
    return exact ? tq4::launch_pdl(tq4::decode_tc_kernel<2, true>, grid, block, smem, st, p)
                 : tq4::launch_pdl(tq4::decode_tc_kernel<2, false>, grid, block, smem, st, p);
  return exact ? tq4::launch_pdl(tq4::decode_tc_kernel<3, true>, grid, block, smem, st, p)
               : tq4::launch_pdl(tq4::decode_tc_kernel<3, false>, grid, block, smem, st, p);
}

// shared memory of a b-bit split-K launch: the wider of its two item bodies
template <int NT, int NTG, int kBits>
constexpr size_t bits_smem_bytes() {
  return std::max(tq4::decode_item_smem_bytes<NT, false, kBits>(), tq4::decode_item_smem_bytes<NTG, false, kBits>());
}
template <int kBits>
cudaError_t set_decode_bits_attrs() {
  cudaError_t e = cudaSuccess;
  auto set = [&e](auto kernel, size_t bytes) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  };
  constexpr int G = tq4::kShareNT;
  set(tq4::decode_bits_kernel<2, 2, false, kBits>, bits_smem_bytes<2, 2, kBits>());
  set(tq4::decode_bits_kernel<2, 2, true, kBits>, bits_smem_bytes<2, 2, kBits>());
  set(tq4::decode_bits_kernel<3, 3, false, kBits>, bits_smem_bytes<3, 3, kBits>());
  set(tq4::decode_bits_kernel<3, 3, true, kBits>, bits_smem_bytes<3, 3, kBits>());
  set(tq4::decode_bits_kernel<1, G, false, kBits>, bits_smem_bytes<1, G, kBits>());
  set(tq4::decode_bits_kernel<1, G, true, kBits>, bits_smem_bytes<1, G, kBits>());
  set(tq4::decode_bits_kernel<2, G, false, kBits>, bits_smem_bytes<2, G, kBits>());
  set(tq4::decode_bits_kernel<2, G, true, kBits>, bits_smem_bytes<2, G, kBits>());
  set(tq4::decode_bits_kernel<3, G, false, kBits>, bits_smem_bytes<3, G, kBits>());
  set(tq4::decode_bits_kernel<3, G, true, kBits>, bits_smem_bytes<3, G, kBits>());
  return e;
}
template <int NT, int NTG, int kBits>
cudaError_t launch_bits_nt(dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  const size_t smem = bits_smem_bytes<NT, NTG, kBits>();
  if (p.out_dtype == TQ4_DTYPE_F32)
    return tq4::launch_pdl(tq4::decode_bits_kernel<NT, NTG, true, kBits>, grid, dim3(tq4::kDecThreads), smem, st, p);
  return tq4::launch_pdl(tq4::decode_bits_kernel<NT, NTG, false, kBits>, grid, dim3(tq4::kDecThreads), smem, st, p);
}
// One query token over a b-bit pool: the one-token kernel (tiles by bulk copies,
// so the tensor map argument is unused).
template <int kBits>
cudaError_t launch_q1_bits(bool exact, dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  const CUtensorMap unused{};
  if (exact)
    return tq4::launch_pdl(tq4::decode_q1_kernel<true, kBits>, grid, dim3(tq4::kQ1Threads),
                           tq4::decode_q1_smem_bytes(), st, p, unused);
  return tq4::launch_pdl(tq4::decode_q1_kernel<false, kBits>, grid, dim3(tq4::kQ1Threads),
                         tq4::decode_q1_smem_bytes(), st, p, unused);
}

// a 2- or 3-bit pool's split-K decode: two to four query tokens, or any count with
// shared-prefix group items (kShareNT n-tiles)
template <int kBits>
cudaError_t launch_decode_bits_b(int nt, bool groups, dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  constexpr int G = tq4::kShareNT;
  if (groups) {
    switch (nt) {
      case 1: return launch_bits_nt<1, G, kBits>(grid, st, p);
      case 2: return launch_bits_nt<2, G, kBits>(grid, st, p);
      default: return launch_bits_nt<3, G, kBits>(grid, st, p);
    }
  }
  return nt == 2 ? launch_bits_nt<2, 2, kBits>(grid, st, p) : launch_bits_nt<3, 3, kBits>(grid, st, p);
}
cudaError_t launch_decode_bits(int bits, int nt, bool groups, dim3 grid, cudaStream_t st,
                               const tq4::DecodeParams& p) {
  return bits == 2 ? launch_decode_bits_b<2>(nt, groups, grid, st, p) : launch_decode_bits_b<3>(nt, groups, grid, st, p);
}

// one split-K decode launch with the output precision chosen at run time
template <int NT, int NTG, bool kI8>
cudaError_t launch_splitk(dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  if (p.out_dtype == TQ4_DTYPE_F32)
    return tq4::launch_pdl(tq4::decode_splitk_kernel<NT, NTG, kI8, true>, grid, dim3(tq4::kDecThreads),
                           tq4::decode_smem_bytes<NT, NTG, kI8>(), st, p);
  return tq4::launch_pdl(tq4::decode_splitk_kernel<NT, NTG, kI8, false>, grid, dim3(tq4::kDecThreads),
                         tq4::decode_smem_bytes<NT, NTG, kI8>(), st, p);
}
// with shared-prefix groups: their items use kShareNT n-tiles
template <bool kI8>
cudaError_t launch_splitk_nt(int nt, bool groups, dim3 grid, cudaStream_t st, const tq4::DecodeParams& p) {
  constexpr int G = tq4::kShareNT;
  if (groups && !kI8) {
    switch (nt) {
      case 1: return launch_splitk<1, G, false>(grid, st, p);
      case 2: return launch_splitk<2, G, false>(grid, st, p);
      default: return launch_splitk<3, G, false>(grid, st, p);
    }
  }
  switch (nt) {
    case 1: return launch_splitk<1, 1, kI8>(grid, st, p);
    case 2: return launch_splitk<2, 2, kI8>(grid, st, p);
    default: return launch_splitk<3, 3, kI8>(grid, st, p);
  }
}

struct DecodePlan {
  int split_len;
  int items_ub;
  int records_ub;
  int rows_pad;
  size_t ws_o_bytes;
  size_t ws_ml_bytes;
  size_t total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// cuTensorMapEncodeTiled, fetched from the driver through the runtime once.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map over one layer's pool seen as rows of 128 B (32 u32), 2,080 rows
// per page; boxes of 32 rows; 128-byte swizzle in shared memory.
int pool_tensor_map(const void* pool, int32_t num_pages, CUtensorMap* map) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return TQ4_ERR_CUDA;
  const cuuint64_t dims[2] = {32, cuuint64_t(num_pages) * (TQ4_PAGE_BYTES / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t elem[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(pool), dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TQ4_OK : TQ4_ERR_CUDA;
}

// Shared-prefix groups from the caller's per-request description (host arrays):
// requests with the same leader (leader[r] == r for a leader) share their first
// pages[r] pages. Groups of more members than one group item's rows allow are cut
// into several groups over the same pages; past kMaxShareGroups, requests read
// their shared pages on their own. Returns TQ4_ERR_ARG for an inconsistent
// description.
int build_share(int32_t n_req, int32_t n_q, int32_t max_pages, const int32_t* leader, const int32_t* pages,
                tq4::SharePlan& sp, int64_t& grouped_pos, int64_t& group_pos) {
  std::memset(&sp, 0, sizeof(sp));
  grouped_pos = group_pos = 0;
  if (!leader || !pages) return TQ4_OK;
  for (int r = 0; r < n_req; ++r) {
    const int l = leader[r];
    if (l < 0 || l >= n_req || leader[l] != l || pages[r] < 0 || pages[r] > max_pages || pages[r] != pages[l])
      return TQ4_ERR_ARG;
  }
  const int cap = std::min(tq4::kMaxShareMembers, (8 * tq4::kShareNT) / (tq4::kGroup * n_q));
  for (int l = 0; l < n_req; ++l) {
    if (leader[l] != l || pages[l] == 0) continue;
    int k = 0;
    for (int r = l; r < n_req; ++r) {
      if (leader[r] != l) continue;
      if (k == 0) {
        if (sp.n_groups == tq4::kMaxShareGroups) break;
        sp.pos[sp.n_groups] = pages[l] * tq4::kPage;
        sp.n_mem[sp.n_groups] = 0;
      }
      sp.mem[sp.n_groups][k++] = r;
      sp.n_mem[sp.n_groups] = k;
      if (k == cap) {   // close this group
        ++sp.n_groups;
        k = 0;
      }
    }
    if (k > 0) ++sp.n_groups;
  }
  // a group of one member dedups nothing: drop it
  int out = 0;
  for (int g = 0; g < sp.n_groups; ++g) {
    if (sp.n_mem[g] < 2) continue;
    if (out != g) {
      sp.pos[out] = sp.pos[g];
      sp.n_mem[out] = sp.n_mem[g];
      std::memcpy(sp.mem[out], sp.mem[g], sizeof(sp.mem[g]));
    }
    grouped_pos += int64_t(sp.pos[out]) * sp.n_mem[out];
    group_pos += sp.pos[out];
    ++out;
  }
  sp.n_groups = out;
  return TQ4_OK;
}

// Split lengths: one wave of CTAs (one per SM, 4 KV heads each) even in the worst
// case, where every request's (and group's) last split is a sliver: a request of
// length s has ceil(s / L) <= s / L + 1 items. With one request the count is exact.
// A group item scores up to kShareNT n-tiles of rows against each position, so it
// gets proportionally fewer positions (cost per position taken as 2 + n-tiles: the
// centroid expansion plus the MMAs of each n-tile).
DecodePlan plan_decode(const tq4_ctx* ctx, int32_t n_req, int32_t n_q, int64_t total_seq_len,
                       tq4::SharePlan* share = nullptr, int64_t grouped_pos = 0, int64_t group_pos = 0) {
  DecodePlan pl{};
  const int64_t slots = std::max<int64_t>(ctx->num_sms / tq4::kHkv, 1);   // items per KV head in one wave
  const int64_t own = std::max<int64_t>(total_seq_len - grouped_pos, 0);   // positions outside the groups
  const int n_groups = share ? share->n_groups : 0;
  const int nt = tq4::decode_nt(n_q);
  const double wg = n_groups ? double(2 + tq4::kShareNT) / double(2 + nt) : 1.0;   // group / own cost per position
  const double work = double(own) + double(group_pos) * wg;
  const int64_t spare = slots - (n_req == 1 && !n_groups ? 0 : n_req + n_groups);
  const int64_t div = spare > 0 ? spare : slots;              // too many requests for one wave: as many as fit
  auto round_chunk = [](int64_t L) {
    L = ((L + tq4::kChunk - 1) / tq4::kChunk) * tq4::kChunk;
    return std::min<int64_t>(std::max<int64_t>(L, tq4::kChunk), int64_t(1) << 30);
  };
  const int64_t L = round_chunk(int64_t(std::ceil(work / double(div))));
  pl.split_len = int(L);
  int64_t g_items = 0, g_records = 0;
  if (share) {
    // group split: L / wg positions, down to a whole number of chunks
    const int64_t Lg = std::max<int64_t>(int64_t(double(L) / wg) / tq4::kChunk * tq4::kChunk, tq4::kChunk);
    share->split_len = int32_t(Lg);
    share->item0[0] = 0;
    for (int g = 0; g < share->n_groups; ++g) {
      const int64_t n = (share->pos[g] + Lg - 1) / Lg;
      share->item0[g + 1] = int32_t(share->item0[g] + n);
      g_records += n * share->n_mem[g];
    }
    share->n_gitems = share->item0[share->n_groups];
    g_items = share->n_gitems;
  }
  const int64_t own_items = (n_req == 1 && !n_groups) ? (own + L - 1) / L : own / L + n_req;
  pl.items_ub = int(g_items + own_items);
  pl.records_ub = int(g_records + own_items);
  pl.rows_pad = 8 * tq4::decode_nt(n_q);
  const size_t recs = size_t(pl.records_ub) * tq4::kHkv * pl.rows_pad;
  pl.ws_o_bytes = align256(recs * tq4::kD * sizeof(float));
  pl.ws_ml_bytes = align256(recs * sizeof(float2));
  pl.total = pl.ws_o_bytes + pl.ws_ml_bytes;
  return pl;
}

}  // namespace

// ---------------------------------------------------------------------------
// Decode attention without any allocation by the caller or the library.
//
// Some callers cannot allocate device memory: plugin code running inside a host
// program that owns the whole device-memory budget (a raw cudaMalloc would
// bypass its accounting), and serving processes that reserve all device memory
// up front and run under a hard memory guard. For them the split-K partial
// results live in this fixed array instead of a caller-provided workspace.
// The array is part of the library image: every GPU that loads the library
// holds TQ4_NOALLOC_SCRATCH_BYTES of it until the process exits. In host code
// its name is only a host-side stand-in, so tq4_ctx_create asks the runtime for
// the array's device address on the context's device (with that device current)
// and keeps it in the context.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ4_NOALLOC_SCRATCH_BYTES];

extern "C" {

int tq4_ctx_create(const int8_t* signs, tq4_ctx** out) {
  if (!signs || !out) return TQ4_ERR_ARG;
  *out = nullptr;
  tq4::Signs sb{};
  for (int i = 0; i < 256; ++i) {
    if (signs[i] != 1 && signs[i] != -1) return TQ4_ERR_ARG;
    if (signs[i] < 0) sb.bits[i >> 5] |= 1u << (i & 31);
  }
  tq4_ctx* ctx = new (std::nothrow) tq4_ctx();
  if (!ctx) return TQ4_ERR_ARG;
  ctx->signs = sb;
  ctx->wait_polls = TQ4_DEFAULT_WAIT_POLLS;
  ctx->decode_path = TQ4_DECODE_PATH_WARP_MMA;
  // the fp64 Lloyd-Max solution is the codebook: encode compares against its
  // midpoints (rounded to fp32), reconstruction reads the centroids rounded to
  // fp32, and the attention kernels read each centroid as an f16 hi + lo pair
  tq4::Codebook cb{};
  lloyd_max_16(1.0 / 16.0, ctx->centroids, ctx->boundaries);
  for (int j = 0; j < 16; ++j) {
    cb.c[j] = float(ctx->centroids[j]);
    cb.c16[j] = half_bits(ctx->centroids[j]);
    __half hh;
    std::memcpy(&hh, &cb.c16[j], 2);
    cb.r16[j] = half_bits(ctx->centroids[j] - double(__half2float(hh)));
  }
  for (int j = 0; j < 15; ++j) cb.b[j] = float(ctx->boundaries[j]);
  tq4::CodebookB cbb[2]{};   // the 2- and 3-bit variants, stored the same way
  for (int v = 0; v < 2; ++v) {
    const int levels = 4 << v;
    lloyd_max_levels(levels, 1.0 / 16.0, ctx->centroids_b[v], ctx->boundaries_b[v]);
    for (int j = 0; j < levels; ++j) {
      cbb[v].c[j] = float(ctx->centroids_b[v][j]);
      cbb[v].c16[j] = half_bits(ctx->centroids_b[v][j]);
      __half hh;
      std::memcpy(&hh, &cbb[v].c16[j], 2);
      cbb[v].r16[j] = half_bits(ctx->centroids_b[v][j] - double(__half2float(hh)));
    }
    for (int j = 0; j + 1 < levels; ++j) cbb[v].b[j] = float(ctx->boundaries_b[v][j]);
  }
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(tq4::g_codebook, &cb, sizeof(cb));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(tq4::g_codebook_b, cbb, sizeof(cbb));
  if (e == cudaSuccess) e = set_decode_bits_attrs<2>();
  if (e == cudaSuccess) e = set_decode_bits_attrs<3>();
  for (const void* fn : {reinterpret_cast<const void*>(tq4::decode_q1_kernel<false, 4>),
                         reinterpret_cast<const void*>(tq4::decode_q1_kernel<true, 4>),
                         reinterpret_cast<const void*>(tq4::decode_q1_kernel<false, 2>),
                         reinterpret_cast<const void*>(tq4::decode_q1_kernel<true, 2>),
                         reinterpret_cast<const void*>(tq4::decode_q1_kernel<false, 3>),
                         reinterpret_cast<const void*>(tq4::decode_q1_kernel<true, 3>)})
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tq4::decode_q1_smem_bytes()));
  if (e == cudaSuccess) e = set_decode_attrs<1, 1, false>();
  if (e == cudaSuccess) e = set_decode_attrs<2, 2, false>();
  if (e == cudaSuccess) e = set_decode_attrs<3, 3, false>();
  if (e == cudaSuccess) e = set_decode_attrs<1, tq4::kShareNT, false>();
  if (e == cudaSuccess) e = set_decode_attrs<2, tq4::kShareNT, false>();
  if (e == cudaSuccess) e = set_decode_attrs<3, tq4::kShareNT, false>();
  if (e == cudaSuccess) e = set_decode_attrs<1, 1, true>();
  if (e == cudaSuccess) e = set_decode_attrs<2, 2, true>();
  if (e == cudaSuccess) e = set_decode_attrs<3, 3, true>();
  if (e == cudaSuccess) e = tq4::prefill_tc_set_attrs();
  if (e == cudaSuccess) e = set_decode_tc_attrs<2>();
  if (e == cudaSuccess) e = set_decode_tc_attrs<3>();
  if (e == cudaSuccess) e = cudaGetSymbolAddress(&ctx->noalloc_scratch, g_noalloc_scratch);
  if (e == cudaSuccess && !ctx->noalloc_scratch) e = cudaErrorInvalidSymbol;
  if (e == cudaSuccess) e = cudaMalloc(&ctx->d_status, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(ctx->d_status, 0, sizeof(int));
  if (e != cudaSuccess) {
    if (ctx->d_status) cudaFree(ctx->d_status);
    delete ctx;
    return TQ4_ERR_CUDA;
  }
  *out = ctx;
  return TQ4_OK;
}

int tq4_ctx_destroy(tq4_ctx* ctx) {
  if (!ctx) return TQ4_OK;
  cudaDeviceSynchronize();
  const cudaError_t e = cudaFree(ctx->d_status);
  delete ctx;
  return cuda_status(e);
}

int tq4_ctx_set_wait_limit(tq4_ctx* ctx, uint32_t polls, int withhold_signal) {
  if (!ctx) return TQ4_ERR_ARG;
  ctx->wait_polls = polls ? polls : TQ4_DEFAULT_WAIT_POLLS;
  ctx->withhold = withhold_signal ? 1 : 0;
  return TQ4_OK;
}

int tq4_ctx_set_decode_path(tq4_ctx* ctx, int path) {
  if (!ctx || (path != TQ4_DECODE_PATH_TENSOR_MEMORY && path != TQ4_DECODE_PATH_WARP_MMA)) return TQ4_ERR_ARG;
  ctx->decode_path = path;
  return TQ4_OK;
}

int tq4_codebook(const tq4_ctx* ctx, double* centroids, double* boundaries) {
  if (!ctx || !centroids || !boundaries) return TQ4_ERR_ARG;
  std::memcpy(centroids, ctx->centroids, sizeof(ctx->centroids));
  std::memcpy(boundaries, ctx->boundaries, sizeof(ctx->boundaries));
  return TQ4_OK;
}

int tq4_encode_append(tq4_ctx* ctx, void* pool, int32_t num_pages, const int32_t* page_table,
                      int32_t table_len, int32_t start_pos, int32_t n_tok, const void* k_new,
                      const void* v_new, int dtype, void* stream) {
  if (!ctx || n_tok < 0 || start_pos < 0) return TQ4_ERR_ARG;
  if (n_tok == 0) return TQ4_OK;
  if (!pool || !page_table || !k_new || !v_new || num_pages <= 0 || table_len <= 0) return TQ4_ERR_ARG;
  if (dtype != TQ4_DTYPE_F32 && dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  if ((int64_t(start_pos) + n_tok + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16)) return TQ4_ERR_ARG;
  if (int rc = check_device(ctx)) return rc;
  return cuda_status(tq4::launch_encode_append(static_cast<uint8_t*>(pool), num_pages, page_table,
                                               start_pos, n_tok, k_new, v_new, dtype, ctx->signs,
                                               ctx->d_status, static_cast<cudaStream_t>(stream)));
}

int tq4_reconstruct(tq4_ctx* ctx, const void* pool, int32_t num_pages, const int32_t* page_table,
                    int32_t table_len, int32_t start, int32_t n, float* k_out, float* v_out,
                    void* stream) {
  if (!ctx || n < 0 || start < 0) return TQ4_ERR_ARG;
  if (n == 0) return TQ4_OK;
  if (!pool || !page_table || !k_out || !v_out || num_pages <= 0 || table_len <= 0) return TQ4_ERR_ARG;
  if ((int64_t(start) + n + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(k_out, 16) || !aligned(v_out, 16)) return TQ4_ERR_ARG;
  if (int rc = check_device(ctx)) return rc;
  return cuda_status(tq4::launch_reconstruct(static_cast<const uint8_t*>(pool), num_pages, page_table,
                                             start, n, k_out, v_out, ctx->signs, ctx->d_status,
                                             static_cast<cudaStream_t>(stream)));
}

int tq4_tqb_reconstruct(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages, const int32_t* page_table,
                        int32_t table_len, int32_t start, int32_t n, float* k_out, float* v_out, void* stream) {
  if (bits != 2 && bits != 3) return ctx ? TQ4_ERR_UNSUPPORTED : TQ4_ERR_ARG;
  if (!ctx || n < 0 || start < 0) return TQ4_ERR_ARG;
  if (n == 0) return TQ4_OK;
  if (!pool || !page_table || !k_out || !v_out || num_pages <= 0 || table_len <= 0) return TQ4_ERR_ARG;
  if ((int64_t(start) + n + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(k_out, 16) || !aligned(v_out, 16)) return TQ4_ERR_ARG;
  if (int rc = check_device(ctx)) return rc;
  return cuda_status(tq4::launch_reconstruct(static_cast<const uint8_t*>(pool), num_pages, page_table, start, n,
                                             k_out, v_out, ctx->signs, ctx->d_status,
                                             static_cast<cudaStream_t>(stream), bits));
}

size_t tq4_decode_workspace_bytes(const tq4_ctx* ctx, int32_t n_req, int32_t n_q, int64_t total_seq_len) {
  if (!ctx || n_req <= 0 || n_q < 1 || n_q > TQ4_MAX_QUERY_TOKENS || total_seq_len <= 0) return 0;
  return plan_decode(ctx, n_req, n_q, total_seq_len).total;
}

size_t tq4_decode_shared_workspace_bytes(const tq4_ctx* ctx, int32_t n_req, int32_t n_q, int64_t total_seq_len,
                                         int32_t max_pages, const int32_t* prefix_leader,
                                         const int32_t* prefix_pages) {
  if (!ctx || n_req <= 0 || n_q < 1 || n_q > TQ4_MAX_QUERY_TOKENS || total_seq_len <= 0 || max_pages <= 0) return 0;
  tq4::SharePlan sp;
  int64_t grouped_pos = 0, group_pos = 0;
  if (build_share(n_req, n_q, max_pages, prefix_leader, prefix_pages, sp, grouped_pos, group_pos) != TQ4_OK) return 0;
  return plan_decode(ctx, n_req, n_q, total_seq_len, &sp, grouped_pos, group_pos).total;
}

}  // extern "C"

namespace {

struct AppendArgs {   // the fused append of tq4_decode_append_attention
  void* pool;
  const void* k_new;
  const void* v_new;
  int dtype;
};

int decode_impl(tq4_ctx* ctx, const void* pool, int32_t num_pages, const uint16_t* q, const int32_t* page_tables,
                int32_t max_pages, const int32_t* seq_lens, int32_t n_req, int32_t n_q, int64_t total_seq_len,
                float scale, void* out, int out_dtype, void* workspace, size_t workspace_bytes, void* stream,
                const AppendArgs* app, bool int8 = false, const int32_t* prefix_leader = nullptr,
                const int32_t* prefix_pages = nullptr, int bits = 4) {
  if (!ctx || n_req < 0) return TQ4_ERR_ARG;
  if (n_q < 1 || n_q > TQ4_MAX_QUERY_TOKENS) return TQ4_ERR_UNSUPPORTED;
  if (n_req == 0) return TQ4_OK;
  if (!pool || !q || !page_tables || !seq_lens || !out || num_pages <= 0 || max_pages <= 0)
    return TQ4_ERR_ARG;
  if (out_dtype != TQ4_DTYPE_F32 && out_dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  if (!std::isfinite(scale)) return TQ4_ERR_ARG;
  if (total_seq_len < int64_t(n_req) * n_q || total_seq_len > int64_t(n_req) * max_pages * tq4::kPage)
    return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(q, 16) || !aligned(out, 16)) return TQ4_ERR_ARG;
  if (app) {
    if (!app->k_new || !app->v_new || !aligned(app->k_new, 16) || !aligned(app->v_new, 16)) return TQ4_ERR_ARG;
    if (app->dtype != TQ4_DTYPE_F32 && app->dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  }
  tq4::DecodeParams p{};
  int64_t grouped_pos = 0, group_pos = 0;
  if (int rc = build_share(n_req, n_q, max_pages, prefix_leader, prefix_pages, p.share, grouped_pos, group_pos))
    return rc;
  const bool groups = p.share.n_groups > 0;
  const DecodePlan pl = plan_decode(ctx, n_req, n_q, total_seq_len, &p.share, grouped_pos, group_pos);
  if (!workspace || workspace_bytes < pl.total || !aligned(workspace, 256)) return TQ4_ERR_WORKSPACE;
  if (int rc = check_device(ctx)) return rc;

  p.pool = static_cast<const uint8_t*>(pool);
  p.num_pages = num_pages;
  p.q = q;
  p.page_tables = page_tables;
  p.max_pages = max_pages;
  p.seq_lens = seq_lens;
  p.n_req = n_req;
  p.n_q = n_q;
  p.scale = scale;
  p.split_len = pl.split_len;
  p.items_ub = pl.items_ub;
  p.records_ub = pl.records_ub;
  p.rows_pad = pl.rows_pad;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + pl.ws_o_bytes);
  p.out = out;
  p.out_dtype = out_dtype;
  p.signs = ctx->signs;
  p.status = ctx->d_status;
  p.spin_limit = ctx->wait_polls;
  p.test_withhold = ctx->withhold;
  p.rotate = int8 ? 0 : 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (app && n_q == 1 && !groups) {   // appended inside the decode kernel
    p.pool_w = static_cast<uint8_t*>(app->pool);
    p.k_new = app->k_new;
    p.v_new = app->v_new;
    p.new_dtype = app->dtype;
  } else if (app) {        // a tail-encode kernel ahead of the decode
    e = tq4::launch_encode_tail(static_cast<uint8_t*>(app->pool), num_pages, page_tables, max_pages, seq_lens,
                                n_req, n_q, app->k_new, app->v_new, app->dtype, ctx->signs, ctx->d_status, st, bits);
    if (e != cudaSuccess) return TQ4_ERR_CUDA;
  }
  const dim3 grid(unsigned(pl.items_ub), tq4::kHkv);
  if (bits != 4) {
    const bool exact = out_dtype == TQ4_DTYPE_F32;
    if (tq4::decode_nt(n_q) == 1 && !groups)
      e = bits == 2 ? launch_q1_bits<2>(exact, grid, st, p) : launch_q1_bits<3>(exact, grid, st, p);
    else
      e = launch_decode_bits(bits, tq4::decode_nt(n_q), groups, grid, st, p);
  } else if (int8) {
    e = launch_splitk_nt<true>(tq4::decode_nt(n_q), false, grid, st, p);
  } else if (groups) {     // group items and the requests' own items in one launch
    e = launch_splitk_nt<false>(tq4::decode_nt(n_q), true, grid, st, p);
  } else {
    switch (tq4::decode_nt(n_q)) {
      case 1: {
        CUtensorMap map;
        if (int rc = pool_tensor_map(pool, num_pages, &map)) return rc;
        if (out_dtype == TQ4_DTYPE_F32)
          e = tq4::launch_pdl(tq4::decode_q1_kernel<true>, grid, dim3(tq4::kQ1Threads), tq4::decode_q1_smem_bytes(),
                              st, p, map);
        else
          e = tq4::launch_pdl(tq4::decode_q1_kernel<false>, grid, dim3(tq4::kQ1Threads),
                              tq4::decode_q1_smem_bytes(), st, p, map);
        break;
      }
      default:
        e = ctx->decode_path == TQ4_DECODE_PATH_TENSOR_MEMORY ? launch_decode_tc(tq4::decode_nt(n_q), grid, st, p)
                                                             : launch_splitk_nt<false>(tq4::decode_nt(n_q), false, grid, st, p);
        break;
    }
  }
  if (e != cudaSuccess) return TQ4_ERR_CUDA;
  const int rows = n_req * n_q * tq4::kHq;
  return cuda_status(tq4::launch_pdl(tq4::decode_combine_kernel, dim3(rows), dim3(32 * tq4::kCombWarps), 0, st, p));
}

}  // namespace

extern "C" {

int tq4_decode_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages, const uint16_t* q,
                         const int32_t* page_tables, int32_t max_pages, const int32_t* seq_lens,
                         int32_t n_req, int32_t n_q, int64_t total_seq_len, float scale, void* out,
                         int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, nullptr);
}

int tq4_decode_append_attention(tq4_ctx* ctx, void* pool, int32_t num_pages, const void* k_new, const void* v_new,
                                int new_dtype, const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                const int32_t* seq_lens, int32_t n_req, int32_t n_q, int64_t total_seq_len,
                                float scale, void* out, int out_dtype, void* workspace, size_t workspace_bytes,
                                void* stream) {
  const AppendArgs app{pool, k_new, v_new, new_dtype};
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, &app);
}

int tq4_decode_attention_shared(tq4_ctx* ctx, void* pool, int32_t num_pages, const void* k_new, const void* v_new,
                                int new_dtype, const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                const int32_t* seq_lens, int32_t n_req, int32_t n_q, int64_t total_seq_len,
                                const int32_t* prefix_leader, const int32_t* prefix_pages, float scale, void* out,
                                int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!prefix_leader || !prefix_pages || (k_new == nullptr) != (v_new == nullptr)) return TQ4_ERR_ARG;
  const AppendArgs app{pool, k_new, v_new, new_dtype};
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, k_new ? &app : nullptr, false, prefix_leader,
                     prefix_pages);
}

int tq4_tqb_decode_attention_shared(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages, const void* k_new,
                                    const void* v_new, int new_dtype, const uint16_t* q, const int32_t* page_tables,
                                    int32_t max_pages, const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                    int64_t total_seq_len, const int32_t* prefix_leader, const int32_t* prefix_pages,
                                    float scale, void* out, int out_dtype, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (bits != 2 && bits != 3) return ctx ? TQ4_ERR_UNSUPPORTED : TQ4_ERR_ARG;
  if (!prefix_leader || !prefix_pages || (k_new == nullptr) != (v_new == nullptr)) return TQ4_ERR_ARG;
  const AppendArgs app{pool, k_new, v_new, new_dtype};
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, k_new ? &app : nullptr, false, prefix_leader,
                     prefix_pages, bits);
}

int tq4_int8_encode_append(tq4_ctx* ctx, void* pool, int32_t num_pages, const int32_t* page_table,
                           int32_t table_len, int32_t start_pos, int32_t n_tok, const void* k_new,
                           const void* v_new, int dtype, void* stream) {
  if (!ctx || n_tok < 0 || start_pos < 0) return TQ4_ERR_ARG;
  if (n_tok == 0) return TQ4_OK;
  if (!pool || !page_table || !k_new || !v_new || num_pages <= 0 || table_len <= 0) return TQ4_ERR_ARG;
  if (dtype != TQ4_DTYPE_F32 && dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  if ((int64_t(start_pos) + n_tok + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16)) return TQ4_ERR_ARG;
  if (int rc = check_device(ctx)) return rc;
  return cuda_status(tq4::launch_int8_encode_append(static_cast<uint8_t*>(pool), num_pages, page_table, start_pos,
                                                    n_tok, k_new, v_new, dtype, ctx->d_status,
                                                    static_cast<cudaStream_t>(stream)));
}

int tq4_int8_decode_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages, const uint16_t* q,
                              const int32_t* page_tables, int32_t max_pages, const int32_t* seq_lens,
                              int32_t n_req, int32_t n_q, int64_t total_seq_len, float scale, void* out,
                              int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, nullptr, true);
}

int tq4_tqb_codebook(const tq4_ctx* ctx, int bits, double* centroids, double* boundaries) {
  if (!ctx || !centroids || !boundaries || (bits != 2 && bits != 3)) return TQ4_ERR_ARG;
  const int v = bits - 2, levels = 4 << v;
  std::memcpy(centroids, ctx->centroids_b[v], sizeof(double) * levels);
  std::memcpy(boundaries, ctx->boundaries_b[v], sizeof(double) * (levels - 1));
  return TQ4_OK;
}

int tq4_tqb_encode_append(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages, const int32_t* page_table,
                          int32_t table_len, int32_t start_pos, int32_t n_tok, const void* k_new, const void* v_new,
                          int dtype, void* stream) {
  if (!ctx || n_tok < 0 || start_pos < 0) return TQ4_ERR_ARG;
  if (bits != 2 && bits != 3) return TQ4_ERR_UNSUPPORTED;
  if (n_tok == 0) return TQ4_OK;
  if (!pool || !page_table || !k_new || !v_new || num_pages <= 0 || table_len <= 0) return TQ4_ERR_ARG;
  if (dtype != TQ4_DTYPE_F32 && dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  if ((int64_t(start_pos) + n_tok + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!aligned(pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16)) return TQ4_ERR_ARG;
  if (int rc = check_device(ctx)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* pl = static_cast<uint8_t*>(pool);
  return cuda_status(bits == 2 ? tq4::launch_encode_bits<2>(pl, num_pages, page_table, start_pos, n_tok, k_new, v_new,
                                                            dtype, ctx->signs, ctx->d_status, st)
                               : tq4::launch_encode_bits<3>(pl, num_pages, page_table, start_pos, n_tok, k_new, v_new,
                                                            dtype, ctx->signs, ctx->d_status, st));
}

int tq4_tqb_decode_attention(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages, const uint16_t* q,
                             const int32_t* page_tables, int32_t max_pages, const int32_t* seq_lens, int32_t n_req,
                             int32_t n_q, int64_t total_seq_len, float scale, void* out, int out_dtype,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (bits != 2 && bits != 3) return ctx ? TQ4_ERR_UNSUPPORTED : TQ4_ERR_ARG;
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, nullptr, false, nullptr, nullptr, bits);
}

int tq4_tqb_decode_append_attention(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages, const void* k_new,
                                    const void* v_new, int new_dtype, const uint16_t* q, const int32_t* page_tables,
                                    int32_t max_pages, const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                    int64_t total_seq_len, float scale, void* out, int out_dtype, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (bits != 2 && bits != 3) return ctx ? TQ4_ERR_UNSUPPORTED : TQ4_ERR_ARG;
  const AppendArgs app{pool, k_new, v_new, new_dtype};
  return decode_impl(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len, scale,
                     out, out_dtype, workspace, workspace_bytes, stream, &app, false, nullptr, nullptr, bits);
}

size_t tq4_prefill_workspace_bytes(int32_t n_tok) {
  if (n_tok <= 0) return 0;
  return tq4::prefill_workspace_bytes(n_tok);
}

}  // extern "C"

namespace {

int prefill_impl(tq4_ctx* ctx, const void* pool, int32_t num_pages, const int32_t* page_table, int32_t table_len,
                 int32_t prefix_len, const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk,
                 int32_t n_tok, float scale, void* out, int out_dtype, void* workspace, size_t workspace_bytes,
                 void* stream, bool reconstruct, int bits = 4) {
  if (!ctx || n_tok < 0 || prefix_len < 0) return TQ4_ERR_ARG;
  if (n_tok == 0) return TQ4_OK;
  if (!q || !k_chunk || !v_chunk || !out) return TQ4_ERR_ARG;
  if (out_dtype != TQ4_DTYPE_F32 && out_dtype != TQ4_DTYPE_BF16) return TQ4_ERR_ARG;
  if (prefix_len > 0 && (!pool || !page_table || num_pages <= 0 || table_len <= 0)) return TQ4_ERR_ARG;
  if (prefix_len > 0 && (int64_t(prefix_len) + tq4::kPage - 1) / tq4::kPage > table_len) return TQ4_ERR_ARG;
  if (!std::isfinite(scale)) return TQ4_ERR_ARG;
  if ((pool && !aligned(pool, 16)) || !aligned(q, 16) || !aligned(k_chunk, 16) || !aligned(v_chunk, 16) ||
      !aligned(out, 16))
    return TQ4_ERR_ARG;
  const bool rows = reconstruct || bits != 4;   // the prefix rebuilt as dense rows first
  const size_t need = tq4::prefill_workspace_bytes(n_tok) + (rows ? tq4::prefill_prefix_rows_bytes(prefix_len) : 0);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return TQ4_ERR_WORKSPACE;
  if (int rc = check_device(ctx)) return rc;
  return cuda_status(tq4::launch_prefill_tc(static_cast<const uint8_t*>(pool), num_pages, page_table,
                                            prefix_len, q, k_chunk, v_chunk, n_tok, scale, out, out_dtype,
                                            workspace, ctx->signs, ctx->d_status, ctx->wait_polls,
                                            ctx->withhold, static_cast<cudaStream_t>(stream), ctx->num_sms,
                                            reconstruct, bits));
}

}  // namespace

extern "C" {

int tq4_prefill_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages, const int32_t* page_table,
                          int32_t table_len, int32_t prefix_len, const uint16_t* q,
                          const uint16_t* k_chunk, const uint16_t* v_chunk, int32_t n_tok, float scale,
                          void* out, int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_impl(ctx, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk, v_chunk, n_tok, scale, out,
                      out_dtype, workspace, workspace_bytes, stream, false);
}

size_t tq4_prefill_reconstructed_workspace_bytes(int32_t prefix_len, int32_t n_tok) {
  if (n_tok <= 0 || prefix_len < 0) return 0;
  return tq4::prefill_workspace_bytes(n_tok) + tq4::prefill_prefix_rows_bytes(prefix_len);
}

int tq4_prefill_attention_reconstructed(tq4_ctx* ctx, const void* pool, int32_t num_pages, const int32_t* page_table,
                                        int32_t table_len, int32_t prefix_len, const uint16_t* q,
                                        const uint16_t* k_chunk, const uint16_t* v_chunk, int32_t n_tok, float scale,
                                        void* out, int out_dtype, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  return prefill_impl(ctx, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk, v_chunk, n_tok, scale, out,
                      out_dtype, workspace, workspace_bytes, stream, true);
}

int tq4_tqb_prefill_attention(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages, const int32_t* page_table,
                              int32_t table_len, int32_t prefix_len, const uint16_t* q, const uint16_t* k_chunk,
                              const uint16_t* v_chunk, int32_t n_tok, float scale, void* out, int out_dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (bits != 2 && bits != 3) return ctx ? TQ4_ERR_UNSUPPORTED : TQ4_ERR_ARG;
  return prefill_impl(ctx, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk, v_chunk, n_tok, scale, out,
                      out_dtype, workspace, workspace_bytes, stream, true, bits);
}

int tq4_get_status(tq4_ctx* ctx, void* stream) {
  if (!ctx) return TQ4_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TQ4_ERR_CUDA;
  if (cudaMemcpy(&h, ctx->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ4_ERR_CUDA;
  if (cudaMemset(ctx->d_status, 0, sizeof(int)) != cudaSuccess) return TQ4_ERR_CUDA;
  return h;
}

const char* tq4_status_string(int status) {
  switch (status) {
    case TQ4_OK: return "ok";
    case TQ4_ERR_ARG: return "invalid argument";
    case TQ4_ERR_UNSUPPORTED: return "unsupported shape";
    case TQ4_ERR_PAGE_RANGE: return "page id out of range";
    case TQ4_ERR_CUDA: return "CUDA runtime error";
    case TQ4_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case TQ4_ERR_SEQ: return "sequence length inconsistent with page table or plan";
    case TQ4_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case TQ4_ERR_NO_PAGES: return "not enough page-pool capacity";
    default: return "unknown status";
  }
}

int tq4_decode_attention_noalloc(tq4_ctx* ctx, const void* pool, int32_t num_pages, const uint16_t* q,
                                 const int32_t* page_tables, int32_t max_pages, const int32_t* seq_lens,
                                 int32_t n_req, int32_t n_q, int64_t total_seq_len, float scale, void* out,
                                 int out_dtype, void* stream) {
  if (!ctx) return TQ4_ERR_ARG;
  if (n_q < 1 || n_q > TQ4_MAX_QUERY_TOKENS) return TQ4_ERR_UNSUPPORTED;
  if (n_req == 0) return TQ4_OK;
  if (n_req < 0 || total_seq_len <= 0) return TQ4_ERR_ARG;
  if (tq4_decode_workspace_bytes(ctx, n_req, n_q, total_seq_len) > TQ4_NOALLOC_SCRATCH_BYTES)
    return TQ4_ERR_WORKSPACE;
  return tq4_decode_attention(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q,
                              total_seq_len, scale, out, out_dtype, ctx->noalloc_scratch, TQ4_NOALLOC_SCRATCH_BYTES,
                              stream);
}

}  // extern "C"
