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
};

// q' hi, q' lo, R k hi, R k lo, R v hi, R v lo
inline size_t prefill_workspace_bytes(int32_t n_tok) {
  return size_t(n_tok) * (2 * kHq + 4 * kHkv) * kD * sizeof(__half);
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
