// TQ4 prefill: parameters and the rotate prologue of the attention kernel.
//
// What the prologue computes ([V2] wpnews.pro "JustFit: Run Qwen 27B Fast ...",
// mechanism table row KVExec: attention in the rotated domain): q' = R q * scale
// for every chunk query vector and R k, R v for the chunk's own keys and values,
// each split into an f16 hi part and an f16 lo part (x = hi + lo to about 2^-22
// relative), so that the tensor-core products keep fp32-level precision.
// R = H diag(s) / 16; one warp rotates one 256-vector.
#pragma once
#include "tq4_device.cuh"

namespace tq4 {

struct PrefillParams {
  const uint8_t* pool;
  int32_t num_pages;
  const int32_t* page_table;
  int32_t prefix_len;
  int32_t n_tok;
  const __half* qr;     // [n_tok][24][256] rotated, scaled queries: hi part
  const __half* qlo;    // [n_tok][24][256] lo part (q' - hi)
  const __half* kr;     // [n_tok][4][256] rotated chunk keys: hi part
  const __half* krlo;   //                                     lo part
  const __half* vr;     // [n_tok][4][256] rotated chunk values: hi part
  const __half* vrlo;   //                                       lo part
  void* out;            // [n_tok][24][256], bf16 or fp32 (out_dtype)
  int out_dtype;
  Signs signs;
  int* status;
  uint32_t spin_limit;  // polls before a bounded wait gives up (TQ4_ERR_TIMEOUT)
  int test_withhold;    // test hook: withhold the softmax's P signal of one tile (the issuer's wait runs out)
  // direct inverse reconstruction: the prefix rebuilt as dense rows [prefix_len][4][256]
  // (n c[idx] in the rotated domain, hi and lo) read like the chunk's rows; nullptr:
  // the prefix is expanded from the packed pages inside the kernel
  const __half* pkr;
  const __half* pkrlo;
  const __half* pvr;
  const __half* pvrlo;
  // KV segments per row block (1: none); with several, each segment's pair writes its
  // partial rows ws_po [unit][4][256][256] and (m, l) ws_pml [unit][4][256], merged by
  // the combine pass (unit = row block * n_seg + segment)
  int n_seg;
  float* ws_po;
  float2* ws_pml;
};

constexpr int kPfMaxSegments = 3;

// q' hi, q' lo, R k hi, R k lo, R v hi, R v lo, then room for the segment partials
inline size_t prefill_workspace_bytes(int32_t n_tok) {
  const size_t pairs = (size_t(6) * n_tok + 255) / 256;
  return size_t(n_tok) * (2 * kHq + 4 * kHkv) * kD * sizeof(__half) +
         pairs * kPfMaxSegments * kHkv * 256 * (kD * sizeof(float) + sizeof(float2));
}
// the reconstructed prefix's K hi, K lo, V hi, V lo rows
inline size_t prefill_prefix_rows_bytes(int32_t prefix_len) {
  return size_t(prefix_len) * 4 * kHkv * kD * sizeof(__half);
}

// Direct inverse reconstruction of the prefix ([KVEXEC] simpleprog.com "Fitting a
// 27B-Parameter LLM into 24 GiB of Laptop Memory", section "KVExec": multi-query
// prefill reconstructs the history directly, with the packed path as the
// alternative): every prefix vector becomes a dense row n * c[idx] in the rotated
// domain, split f16 hi + lo. One warp per (position, KV head, K/V); lane l unpacks
// word l (coordinates 8 l .. 8 l + 7). A page id out of range records
// TQ4_ERR_PAGE_RANGE and leaves a zero row.
__global__ void __launch_bounds__(256) prefill_reconstruct_rows_kernel(
    const uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table, int32_t prefix_len,
    __half* __restrict__ kr, __half* __restrict__ krlo, __half* __restrict__ vr, __half* __restrict__ vrlo,
    int* status) {
  __shared__ float cb[16];   // the centroids (a per-lane index into constant memory would serialise)
  if (threadIdx.x < 16) cb[threadIdx.x] = g_codebook.c[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);   // (pos, h, kv)
  pdl_wait();   // the pool may be written by the previous kernel
  pdl_launch_dependents();
  if (vec >= int64_t(prefix_len) * kHkv * 2) return;
  const int kv = int(vec & 1), h = int((vec >> 1) % kHkv);
  const int64_t pos = (vec >> 1) / kHkv;
  const int32_t page = __ldg(page_table + (pos >> 8));
  float v[8];
  if (page >= 0 && page < num_pages) {
    const uint8_t* pg = pool + int64_t(page) * kPageBytes;
    const int slot = h * kPage + int(pos & (kPage - 1));
    const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(pg + (kv ? kVWords : kKWords) + int64_t(slot) * 128) + lane);
    const float n = ldg_half(pg + (kv ? kVNorms : kKNorms) + slot * 2);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = n * cb[(word >> (4 * i)) & 15u];
  } else {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = pack_half2(v[2 * i], v[2 * i + 1]);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi[i]));
    lo[i] = pack_half2(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
  }
  const int64_t row = (pos * kHkv + h) * kD + lane * 8;
  *reinterpret_cast<uint4*>((kv ? vr : kr) + row) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4*>((kv ? vrlo : krlo) + row) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// The same rebuild for a 2- or 3-bit pool (bit-plane words, the 2^b-level codebook
// of g_codebook_b): lane l's eight indices are the two-bit fields of plane-0 word
// l / 2 (its half l & 1) and, with 3 bits, the bits of byte l & 3 of plane-1 word
// 16 + l / 4 as their bit 2.
template <int kBits>
__global__ void __launch_bounds__(256) prefill_reconstruct_rows_bits_kernel(
    const uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table, int32_t prefix_len,
    __half* __restrict__ kr, __half* __restrict__ krlo, __half* __restrict__ vr, __half* __restrict__ vrlo,
    int* status) {
  __shared__ float cb[1 << kBits];
  if (threadIdx.x < (1 << kBits)) cb[threadIdx.x] = g_codebook_b[kBits - 2].c[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);   // (pos, h, kv)
  pdl_wait();   // the pool may be written by the previous kernel
  pdl_launch_dependents();
  if (vec >= int64_t(prefix_len) * kHkv * 2) return;
  const int kv = int(vec & 1), h = int((vec >> 1) % kHkv);
  const int64_t pos = (vec >> 1) / kHkv;
  const int32_t page = __ldg(page_table + (pos >> 8));
  float v[8];
  if (page >= 0 && page < num_pages) {
    const uint8_t* pg = pool + int64_t(page) * tqb_page_bytes<kBits>();
    const int slot = h * kPage + int(pos & (kPage - 1));
    const uint32_t* words = reinterpret_cast<const uint32_t*>(pg + (kv ? tqb_v_words<kBits>() : 0) +
                                                              int64_t(slot) * tqb_row_bytes<kBits>());
    const uint32_t lo = __ldg(words + (lane >> 1)) >> (16 * (lane & 1));
    uint32_t hb = 0;
    if constexpr (kBits == 3) hb = __ldg(words + 16 + (lane >> 2)) >> (8 * (lane & 3));
    const float n = ldg_half(pg + (kv ? tqb_v_norms<kBits>() : tqb_k_norms<kBits>()) + slot * 2);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = n * cb[((lo >> (2 * i)) & 3u) | (((hb >> i) & 1u) << 2)];
  } else {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  uint32_t hi[4], lo16[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = pack_half2(v[2 * i], v[2 * i + 1]);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi[i]));
    lo16[i] = pack_half2(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
  }
  const int64_t row = (pos * kHkv + h) * kD + lane * 8;
  *reinterpret_cast<uint4*>((kv ? vr : kr) + row) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4*>((kv ? vrlo : krlo) + row) = make_uint4(lo16[0], lo16[1], lo16[2], lo16[3]);
}

// one warp per vector: rotate queries (with scale) and the chunk's K/V; f16 hi + lo
__global__ void __launch_bounds__(256) prefill_rotate_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
    int32_t n_tok, float scale, __half* __restrict__ qr, __half* __restrict__ qlo, __half* __restrict__ kr,
    __half* __restrict__ krlo, __half* __restrict__ vr, __half* __restrict__ vrlo, Signs signs) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nq = int64_t(n_tok) * kHq, nk = int64_t(n_tok) * kHkv;
  pdl_wait();   // inputs may come from the previous kernel
  pdl_launch_dependents();
  if (vec >= nq + 2 * nk) return;
  const uint16_t* src;
  __half* dst;
  __half* dst_lo;
  float mul;
  if (vec < nq) {
    src = q + vec * kD;
    dst = qr + vec * kD;
    dst_lo = qlo + vec * kD;
    mul = scale * 0.0625f;
  } else if (vec < nq + nk) {
    src = kc + (vec - nq) * kD;
    dst = kr + (vec - nq) * kD;
    dst_lo = krlo + (vec - nq) * kD;
    mul = 0.0625f;
  } else {
    src = vc + (vec - nq - nk) * kD;
    dst = vr + (vec - nq - nk) * kD;
    dst_lo = vrlo + (vec - nq - nk) * kD;
    mul = 0.0625f;
  }
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + lane * 8));
  const uint32_t ww[4] = {raw.x, raw.y, raw.z, raw.w};
  float v[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(ww[i] << 16) * sign_of(signs, lane * 8 + 2 * i);
    v[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u) * sign_of(signs, lane * 8 + 2 * i + 1);
  }
  warp_fwht256(v);
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = v[2 * i] * mul, b = v[2 * i + 1] * mul;
    hi[i] = pack_half2(a, b);
    const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hi[i]));
    lo[i] = pack_half2(a - h.x, b - h.y);
  }
  *reinterpret_cast<uint4*>(dst + lane * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4*>(dst_lo + lane * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

}  // namespace tq4
