// TQ4 encode + append, and explicit reconstruction (sm_100a).
//
// Encode ([KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into 24 GiB of
// Laptop Memory", section "KVExec": four-bit TurboQuant encoding, 32 U32 words
// with eight indices each + one FP16 norm): per head vector x,
//   n = ||x||_2, u = x / n, y = R u with R = H diag(s) / 16,
//   idx_i = number of decision boundaries below y_i (nearest centroid, ties low),
//   word w = sum_i idx_{8w+i} << 4i, norm stored as fp16(n).
// Reconstruction (same section: centroid lookup, inverse Hadamard rotation,
// norm restore): x_hat = fp16(n) * diag(s) H c[idx] / 16.
//
// One warp per vector; lane l owns coordinates 8l..8l+7, i.e. exactly word l.
#pragma once
#include "tq4_device.cuh"

namespace tq4 {

template <typename T>
__device__ __forceinline__ void load8(const T* src, float v[8]);

template <>
__device__ __forceinline__ void load8<float>(const float* src, float v[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* src, float v[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Quantise one head vector held by a warp (lane l: coordinates 8l..8l+7 in x).
// Returns lane l's packed word (word l of the vector); n receives ||x||_2.
__device__ __forceinline__ uint32_t encode_vector_warp(const float x[8], const Signs& signs, float& n) {
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  n = sqrtf(ss);
  uint32_t word = 0;
  if (n > 0.f) {
    const uint32_t sb = lane_sign_bits(signs);
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = apply_sign(x[i] / n, sb, i);
    warp_fwht256(y);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float yi = y[i] * 0.0625f;  // 1/16, exact
      uint32_t idx = 0;
#pragma unroll
      for (int j = 0; j < 15; ++j) idx += (yi > g_codebook.b[j]) ? 1u : 0u;
      word |= idx << (4 * i);
    }
  }
  return word;
}

// Store a packed vector (word of this lane, fp16 norm by lane 0) at position pos of
// a request (page table `table`), head `head`, K (kv = 0) or V. A page id outside
// [0, num_pages) records TQ4_ERR_PAGE_RANGE and writes nothing; returns false then.
__device__ __forceinline__ bool store_packed_warp(uint8_t* pool, int32_t num_pages, const int32_t* table, int32_t pos,
                                                  int head, int kv, uint32_t word, float n, int* status) {
  const int lane = threadIdx.x & 31;
  const int32_t page = __ldg(table + (pos >> 8));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
    return false;
  }
  const int slot = pos & (kPage - 1);
  uint8_t* base = pool + int64_t(page) * kPageBytes;
  uint32_t* words = reinterpret_cast<uint32_t*>(base + (kv ? kVWords : kKWords)) + (head * kPage + slot) * kWords;
  words[lane] = word;
  if (lane == 0) {
    __half* norms = reinterpret_cast<__half*>(base + (kv ? kVNorms : kKNorms));
    norms[head * kPage + slot] = __float2half_rn(n);
  }
  return true;
}

// grid: ceil(n_tok * 8 / warps_per_block); warp -> (token, kv, head)
template <typename T>
__global__ void __launch_bounds__(256) encode_append_kernel(
    uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table,
    int32_t start_pos, int32_t n_tok, const T* __restrict__ k_new, const T* __restrict__ v_new,
    Signs signs, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();   // inputs and the pool may come from the previous kernel
  pdl_launch_dependents();
  if (vec >= int64_t(n_tok) * 2 * kHkv) return;
  const int tok = int(vec / (2 * kHkv));
  const int kv = int(vec / kHkv) & 1;       // 0 = K, 1 = V
  const int head = int(vec % kHkv);
  float x[8];
  load8<T>((kv ? v_new : k_new) + (int64_t(tok) * kHkv + head) * kD + lane * 8, x);
  float n;
  const uint32_t word = encode_vector_warp(x, signs, n);
  store_packed_warp(pool, num_pages, page_table, start_pos + tok, head, kv, word, n, status);
}

// grid: ceil(n * 8 / warps_per_block); writes fp32 [n][4][256] for K and V.
// kBits: 4 (TQ4 pool), or 2 / 3 (bit-plane pool: lane l's indices are the two-bit
// fields of plane-0 word l / 2, half l & 1, and with 3 bits byte l & 3 of plane-1
// word 16 + l / 4 as their bit 2; the 2^b-level codebook).
template <int kBits>
__global__ void __launch_bounds__(256) reconstruct_kernel(
    const uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table,
    int32_t start, int32_t n, float* __restrict__ k_out, float* __restrict__ v_out, Signs signs,
    int* status) {
  __shared__ float cb[1 << kBits];
  if (threadIdx.x < (1 << kBits)) {
    if constexpr (kBits == 4) cb[threadIdx.x] = g_codebook.c[threadIdx.x];
    else cb[threadIdx.x] = g_codebook_b[kBits - 2].c[threadIdx.x];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (vec >= int64_t(n) * 2 * kHkv) return;
  const int tok = int(vec / (2 * kHkv));
  const int kv = int(vec / kHkv) & 1;
  const int head = int(vec % kHkv);
  float* dst = (kv ? v_out : k_out) + (int64_t(tok) * kHkv + head) * kD + lane * 8;

  const int32_t p = start + tok;
  const int32_t page = __ldg(page_table + (p >> 8));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = 0.f;
    return;
  }
  const int slot = p & (kPage - 1);
  float v[8], nrm;
  if constexpr (kBits == 4) {
    const uint8_t* base = pool + int64_t(page) * kPageBytes;
    const uint32_t word = ldg32(base + (kv ? kVWords : kKWords) + ((head * kPage + slot) * kWords + lane) * 4);
    nrm = ldg_half(base + (kv ? kVNorms : kKNorms) + (head * kPage + slot) * 2);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = cb[(word >> (4 * i)) & 15u];
  } else {
    const uint8_t* base = pool + int64_t(page) * tqb_page_bytes<kBits>();
    const uint8_t* row = base + (kv ? tqb_v_words<kBits>() : 0) + int64_t(head * kPage + slot) * tqb_row_bytes<kBits>();
    const uint32_t lo = ldg32(row + (lane >> 1) * 4) >> (16 * (lane & 1));
    const uint32_t hb = kBits == 3 ? ldg32(row + (16 + (lane >> 2)) * 4) >> (8 * (lane & 3)) : 0u;
    nrm = ldg_half(base + (kv ? tqb_v_norms<kBits>() : tqb_k_norms<kBits>()) + (head * kPage + slot) * 2);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = cb[((lo >> (2 * i)) & 3u) | (((hb >> i) & 1u) << 2)];
  }
  warp_fwht256(v);
  float o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = nrm * (v[i] * 0.0625f * sign_of(signs, lane * 8 + i));
  reinterpret_cast<float4*>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// Uniform INT8 comparison arm: per head vector, scale s = max |x_i| / 127 and codes
// round-half-even(x_i / s), in double precision (the divisions and the rounding are
// those of an fp64 reference, so the codes come out bit-identical); the scale is
// stored as fp16. Page layout: K codes [4][256][256] int8, V codes, K scales
// [4][256] fp16, V scales. One warp per vector; lane l owns dims 8l .. 8l + 7.
template <typename T>
__global__ void __launch_bounds__(256) int8_encode_kernel(
    uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table, int32_t start_pos,
    int32_t n_tok, const T* __restrict__ k_new, const T* __restrict__ v_new, int* status) {
  constexpr int64_t kPB = TQ4_INT8_PAGE_BYTES;
  constexpr int64_t kVC = int64_t(kHkv) * kPage * kD, kKS = 2 * kVC, kVS = kKS + int64_t(kHkv) * kPage * 2;
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (vec >= int64_t(n_tok) * 2 * kHkv) return;
  const int tok = int(vec / (2 * kHkv));
  const int kv = int(vec / kHkv) & 1;
  const int head = int(vec % kHkv);
  float x[8];
  load8<T>((kv ? v_new : k_new) + (int64_t(tok) * kHkv + head) * kD + lane * 8, x);
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(x[i]));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
  const double sc = double(am) / 127.0;
  uint32_t w[2] = {0u, 0u};
  if (am > 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = __double2int_rn(double(x[i]) / sc);
      w[i >> 2] |= (uint32_t(q) & 0xFFu) << (8 * (i & 3));
    }
  }
  const int32_t pos = start_pos + tok;
  const int32_t page = __ldg(page_table + (pos >> 8));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
    return;
  }
  const int slot = head * kPage + (pos & (kPage - 1));
  uint8_t* base = pool + int64_t(page) * kPB;
  *reinterpret_cast<uint2*>(base + (kv ? kVC : 0) + int64_t(slot) * kD + lane * 8) = make_uint2(w[0], w[1]);
  if (lane == 0) reinterpret_cast<__half*>(base + (kv ? kVS : kKS))[slot] = __double2half(sc);
}

// The 2- and 3-bit variants: the four-bit encode with a 2^kBits-level codebook
// (g_codebook_b) and the bit-plane packing of tqb_row_bytes: lane l's indices of
// coordinates 8l .. 8l + 7 give the 16 low bits (plane 0) of word l / 2 and the 8
// bits at 8 (l & 3) of plane-1 word 16 + l / 4. One warp per vector: w0 receives
// plane-0 word l / 2 (meaningful in even lanes), w1 plane-1 word 16 + l / 4
// (meaningful in lanes 4w), n the norm.
template <int kBits>
__device__ __forceinline__ void encode_bits_warp(const float x[8], const Signs& signs, uint32_t& w0, uint32_t& w1,
                                                 float& n) {
  const int lane = threadIdx.x & 31;
  const CodebookB& cb = g_codebook_b[kBits - 2];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  n = sqrtf(ss);
  uint32_t lo16 = 0, hi8 = 0;
  if (n > 0.f) {
    const uint32_t sb = lane_sign_bits(signs);
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = apply_sign(x[i] / n, sb, i);
    warp_fwht256(y);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float yi = y[i] * 0.0625f;
      uint32_t idx = 0;
#pragma unroll
      for (int j = 0; j < (1 << kBits) - 1; ++j) idx += (yi > cb.b[j]) ? 1u : 0u;
      lo16 |= (idx & 3u) << (2 * i);
      hi8 |= ((idx >> 2) & 1u) << i;
    }
  }
  // plane 0: word w = lanes 2w (low half) and 2w + 1; plane 1: word w = lanes 4w .. 4w + 3
  w0 = lo16 | (__shfl_down_sync(0xffffffffu, lo16, 1) << 16);
  w1 = hi8 << (8 * (lane & 3));
  w1 |= __shfl_xor_sync(0xffffffffu, w1, 1);
  w1 |= __shfl_xor_sync(0xffffffffu, w1, 2);
}

// Store a b-bit vector at position pos of a request (page table `table`), head
// `head`, K (kv = 0) or V. A page id outside [0, num_pages) records
// TQ4_ERR_PAGE_RANGE and writes nothing; returns false then.
template <int kBits>
__device__ __forceinline__ bool store_bits_warp(uint8_t* pool, int32_t num_pages, const int32_t* table, int32_t pos,
                                                int head, int kv, uint32_t w0, uint32_t w1, float n, int* status) {
  const int lane = threadIdx.x & 31;
  const int32_t page = __ldg(table + (pos >> 8));
  if (page < 0 || page >= num_pages) {
    if (lane == 0) record_error(status, TQ4_ERR_PAGE_RANGE);
    return false;
  }
  const int slot = head * kPage + (pos & (kPage - 1));
  uint8_t* base = pool + int64_t(page) * tqb_page_bytes<kBits>();
  uint32_t* words = reinterpret_cast<uint32_t*>(base + (kv ? tqb_v_words<kBits>() : 0) +
                                                int64_t(slot) * tqb_row_bytes<kBits>());
  if ((lane & 1) == 0) words[lane >> 1] = w0;
  if (kBits == 3 && (lane & 3) == 0) words[16 + (lane >> 2)] = w1;
  if (lane == 0)
    reinterpret_cast<__half*>(base + (kv ? tqb_v_norms<kBits>() : tqb_k_norms<kBits>()))[slot] = __float2half_rn(n);
  return true;
}

// One warp per new b-bit vector: grid ceil(n_tok * 8 / warps_per_block)
template <typename T, int kBits>
__global__ void __launch_bounds__(256) encode_bits_kernel(
    uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_table, int32_t start_pos,
    int32_t n_tok, const T* __restrict__ k_new, const T* __restrict__ v_new, Signs signs, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (vec >= int64_t(n_tok) * 2 * kHkv) return;
  const int tok = int(vec / (2 * kHkv));
  const int kv = int(vec / kHkv) & 1;
  const int head = int(vec % kHkv);
  float x[8];
  load8<T>((kv ? v_new : k_new) + (int64_t(tok) * kHkv + head) * kD + lane * 8, x);
  uint32_t w0, w1;
  float n;
  encode_bits_warp<kBits>(x, signs, w0, w1, n);
  store_bits_warp<kBits>(pool, num_pages, page_table, start_pos + tok, head, kv, w0, w1, n, status);
}

// The last n_q positions of every request, with positions taken from the device
// lengths: new token t of request r goes to position seq_lens[r] - n_q + t.
// grid: ceil(n_req * n_q * 8 / warps_per_block); inputs [n_req][n_q][4][256].
// kBits: 4 (TQ4 pool) or 2 / 3 (b-bit pools).
template <typename T, int kBits>
__global__ void __launch_bounds__(256) encode_tail_kernel(
    uint8_t* __restrict__ pool, int32_t num_pages, const int32_t* __restrict__ page_tables, int32_t max_pages,
    const int32_t* __restrict__ seq_lens, int32_t n_req, int32_t n_q, const T* __restrict__ k_new,
    const T* __restrict__ v_new, Signs signs, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (vec >= int64_t(n_req) * n_q * 2 * kHkv) return;
  const int64_t tok = vec / (2 * kHkv);       // request-major token index
  const int r = int(tok / n_q), t = int(tok % n_q);
  const int kv = int(vec / kHkv) & 1;
  const int head = int(vec % kHkv);
  const int32_t len = __ldg(seq_lens + r);
  if (len < n_q || len > max_pages * kPage) {   // the decode kernels record TQ4_ERR_SEQ for it
    return;
  }
  float x[8];
  load8<T>((kv ? v_new : k_new) + (tok * kHkv + head) * kD + lane * 8, x);
  float n;
  const int32_t* table = page_tables + int64_t(r) * max_pages;
  if constexpr (kBits == 4) {
    const uint32_t word = encode_vector_warp(x, signs, n);
    store_packed_warp(pool, num_pages, table, len - n_q + t, head, kv, word, n, status);
  } else {
    uint32_t w0, w1;
    encode_bits_warp<kBits>(x, signs, w0, w1, n);
    store_bits_warp<kBits>(pool, num_pages, table, len - n_q + t, head, kv, w0, w1, n, status);
  }
}

// ---------------------------------------------------------------- launchers
template <int kBits>
cudaError_t launch_encode_bits(uint8_t* pool, int32_t num_pages, const int32_t* page_table, int32_t start_pos,
                               int32_t n_tok, const void* k_new, const void* v_new, int dtype, const Signs& signs,
                               int* status, cudaStream_t stream) {
  const int threads = 256, wpb = threads / 32;
  const unsigned blocks = unsigned((int64_t(n_tok) * 2 * kHkv + wpb - 1) / wpb);
  if (dtype == TQ4_DTYPE_F32)
    return launch_pdl(encode_bits_kernel<float, kBits>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                      page_table, start_pos, n_tok, static_cast<const float*>(k_new),
                      static_cast<const float*>(v_new), signs, status);
  return launch_pdl(encode_bits_kernel<uint16_t, kBits>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                    page_table, start_pos, n_tok, static_cast<const uint16_t*>(k_new),
                    static_cast<const uint16_t*>(v_new), signs, status);
}

cudaError_t launch_int8_encode_append(uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                                      int32_t start_pos, int32_t n_tok, const void* k_new, const void* v_new,
                                      int dtype, int* status, cudaStream_t stream) {
  const int threads = 256, wpb = threads / 32;
  const unsigned blocks = unsigned((int64_t(n_tok) * 2 * kHkv + wpb - 1) / wpb);
  if (dtype == TQ4_DTYPE_F32)
    return launch_pdl(int8_encode_kernel<float>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                      page_table, start_pos, n_tok, static_cast<const float*>(k_new),
                      static_cast<const float*>(v_new), status);
  return launch_pdl(int8_encode_kernel<uint16_t>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                    page_table, start_pos, n_tok, static_cast<const uint16_t*>(k_new),
                    static_cast<const uint16_t*>(v_new), status);
}

cudaError_t launch_encode_append(uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                                 int32_t start_pos, int32_t n_tok, const void* k_new,
                                 const void* v_new, int dtype, const Signs& signs, int* status,
                                 cudaStream_t stream) {
  const int threads = 256, wpb = threads / 32;
  const int64_t vecs = int64_t(n_tok) * 2 * kHkv;
  const unsigned blocks = unsigned((vecs + wpb - 1) / wpb);
  if (dtype == TQ4_DTYPE_F32)
    return launch_pdl(encode_append_kernel<float>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                      page_table, start_pos, n_tok, static_cast<const float*>(k_new),
                      static_cast<const float*>(v_new), signs, status);
  return launch_pdl(encode_append_kernel<uint16_t>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                    page_table, start_pos, n_tok, static_cast<const uint16_t*>(k_new),
                    static_cast<const uint16_t*>(v_new), signs, status);
}

template <int kBits>
cudaError_t launch_encode_tail_b(uint8_t* pool, int32_t num_pages, const int32_t* page_tables, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t n_req, int32_t n_q, const void* k_new,
                                 const void* v_new, int dtype, const Signs& signs, int* status, cudaStream_t stream) {
  const int threads = 256, wpb = threads / 32;
  const int64_t vecs = int64_t(n_req) * n_q * 2 * kHkv;
  const unsigned blocks = unsigned((vecs + wpb - 1) / wpb);
  if (dtype == TQ4_DTYPE_F32)
    return launch_pdl(encode_tail_kernel<float, kBits>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                      page_tables, max_pages, seq_lens, n_req, n_q, static_cast<const float*>(k_new),
                      static_cast<const float*>(v_new), signs, status);
  return launch_pdl(encode_tail_kernel<uint16_t, kBits>, dim3(blocks), dim3(threads), 0, stream, pool, num_pages,
                    page_tables, max_pages, seq_lens, n_req, n_q, static_cast<const uint16_t*>(k_new),
                    static_cast<const uint16_t*>(v_new), signs, status);
}
// bits: 4 (TQ4 pool), 2 or 3
inline cudaError_t launch_encode_tail(uint8_t* pool, int32_t num_pages, const int32_t* page_tables,
                                      int32_t max_pages, const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                      const void* k_new, const void* v_new, int dtype, const Signs& signs,
                                      int* status, cudaStream_t stream, int bits = 4) {
  switch (bits) {
    case 2: return launch_encode_tail_b<2>(pool, num_pages, page_tables, max_pages, seq_lens, n_req, n_q, k_new,
                                           v_new, dtype, signs, status, stream);
    case 3: return launch_encode_tail_b<3>(pool, num_pages, page_tables, max_pages, seq_lens, n_req, n_q, k_new,
                                           v_new, dtype, signs, status, stream);
    default: return launch_encode_tail_b<4>(pool, num_pages, page_tables, max_pages, seq_lens, n_req, n_q, k_new,
                                            v_new, dtype, signs, status, stream);
  }
}

// bits: 4 (TQ4 pool), 2 or 3
cudaError_t launch_reconstruct(const uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                               int32_t start, int32_t n, float* k_out, float* v_out,
                               const Signs& signs, int* status, cudaStream_t stream, int bits = 4) {
  const int threads = 256, wpb = threads / 32;
  const int64_t vecs = int64_t(n) * 2 * kHkv;
  const unsigned blocks = unsigned((vecs + wpb - 1) / wpb);
  auto kernel = bits == 2 ? reconstruct_kernel<2> : bits == 3 ? reconstruct_kernel<3> : reconstruct_kernel<4>;
  return launch_pdl(kernel, dim3(blocks), dim3(threads), 0, stream, pool, num_pages, page_table, start, n, k_out,
                    v_out, signs, status);
}

}  // namespace tq4
