// TQ4 prefill attention (sm_100a), tiled flash attention on tensor cores.
//
// What it computes ([KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into
// 24 GiB of Laptop Memory", section "KVExec": multi-query prefill reconstructs
// the packed history and consumes it with scaled dot-product attention):
// chunk token i attends causally to the TQ4 prefix [0, prefix_len) and to
// chunk tokens 0..i, whose K/V are used at full (bf16) precision.
//
// Everything runs in the rotated domain ([V2] wpnews.pro "JustFit: Run Qwen
// 27B Fast ...", mechanism table row KVExec): a prologue rotates the queries
// (q' = R q * scale) and the chunk's own K/V (R k, R v) once; prefix tiles are
// expanded from their centroid indices straight into shared memory (no norm,
// no inverse rotation: the K norm scales the score columns, the V norm is
// folded into P); the epilogue applies R^T to each output row once.
//
// Tiles: a CTA owns 64 query rows (row = token * 6 + head within the KV
// head's group of 6) of one KV head and walks KV tiles of 64 positions.
#pragma once
#include "tq4_device.cuh"

namespace tq4 {

constexpr int kPfRows = 64;               // query rows per CTA
constexpr int kPfTile = 64;               // KV positions per tile
constexpr int kPfThreads = 128;
constexpr int kPfStride = kD + 8;         // halves per smem row
constexpr size_t kPfSmem = size_t(3) * kPfRows * kPfStride * 2 + 2 * kPfTile * 4 + 256 * 4;

struct PrefillParams {
  const uint8_t* pool;
  int32_t num_pages;
  const int32_t* page_table;
  int32_t prefix_len;
  int32_t n_tok;
  const __half* qr;   // [n_tok][24][256] rotated, scaled queries
  const __half* kr;   // [n_tok][4][256] rotated chunk keys
  const __half* vr;   // [n_tok][4][256] rotated chunk values
  uint16_t* out;      // bf16 [n_tok][24][256]
  Signs signs;
  int* status;
};

inline size_t prefill_workspace_bytes(int32_t n_tok) {
  return size_t(n_tok) * (kHq + 2 * kHkv) * kD * sizeof(__half);
}

// one warp per vector: rotate queries (with scale) and the chunk's K/V into f16
__global__ void __launch_bounds__(256) prefill_rotate_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
    int32_t n_tok, float scale, __half* __restrict__ qr, __half* __restrict__ kr, __half* __restrict__ vr,
    Signs signs) {
  const int lane = threadIdx.x & 31;
  const int64_t vec = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nq = int64_t(n_tok) * kHq, nk = int64_t(n_tok) * kHkv;
  if (vec >= nq + 2 * nk) return;
  const uint16_t* src;
  __half* dst;
  float mul;
  if (vec < nq) {
    src = q + vec * kD;
    dst = qr + vec * kD;
    mul = scale * 0.0625f;
  } else if (vec < nq + nk) {
    src = kc + (vec - nq) * kD;
    dst = kr + (vec - nq) * kD;
    mul = 0.0625f;
  } else {
    src = vc + (vec - nq - nk) * kD;
    dst = vr + (vec - nq - nk) * kD;
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
  uint4 o;
  o.x = pack_half2(v[0] * mul, v[1] * mul);
  o.y = pack_half2(v[2] * mul, v[3] * mul);
  o.z = pack_half2(v[4] * mul, v[5] * mul);
  o.w = pack_half2(v[6] * mul, v[7] * mul);
  *reinterpret_cast<uint4*>(dst + lane * 8) = o;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_attn_kernel(const PrefillParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __half* qs = reinterpret_cast<__half*>(smem);
  __half* ks = qs + kPfRows * kPfStride;
  __half* vs = ks + kPfTile * kPfStride;
  float* nks = reinterpret_cast<float*>(vs + kPfTile * kPfStride);
  float* nvs = nks + kPfTile;
  uint32_t* lut = reinterpret_cast<uint32_t*>(nvs + kPfTile);

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * kPfRows;
  const int m_total = 6 * p.n_tok;

  for (int b = tid; b < 256; b += kPfThreads)
    lut[b] = uint32_t(g_codebook.c16[b & 15]) | (uint32_t(g_codebook.c16[b >> 4]) << 16);
  // query rows -> smem (zeros past the end)
  for (int e = tid; e < kPfRows * 32; e += kPfThreads) {
    const int r = e >> 5, seg = e & 31;
    const int row = row0 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < m_total) {
      const int tok = row / 6, j = row % 6;
      v = __ldg(reinterpret_cast<const uint4*>(p.qr + (int64_t(tok) * kHq + h * kGroup + j) * kD) + seg);
    }
    *reinterpret_cast<uint4*>(qs + r * kPfStride + seg * 8) = v;
  }

  const int last_row = min(row0 + kPfRows, m_total) - 1;
  const int kv_end = p.prefix_len + last_row / 6 + 1;
  int lim[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int row = row0 + 16 * w + g + 8 * e;
    lim[e] = row < m_total ? p.prefix_len + row / 6 + 1 : 0;
  }

  float o[32][4];
#pragma unroll
  for (int nd = 0; nd < 32; ++nd)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[nd][i] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int tile = 0; tile < kv_end; tile += kPfTile) {
    __syncthreads();
    // ---- expand the KV tile into smem (rotated-domain f16; norms separately)
    for (int e = tid; e < 2 * kPfTile * 32; e += kPfThreads) {
      const int kv = e / (kPfTile * 32);
      const int pl = (e >> 5) % kPfTile, wd = e & 31;
      const int pos = tile + pl;
      uint4 v = make_uint4(0, 0, 0, 0);
      float nrm = 0.f;
      if (pos < kv_end) {
        if (pos < p.prefix_len) {
          int32_t page = __ldg(p.page_table + (pos >> 8));
          if (page < 0 || page >= p.num_pages) {
            record_error(p.status, TQ4_ERR_PAGE_RANGE);
          } else {
            const uint8_t* pg = p.pool + int64_t(page) * kPageBytes;
            const int slot = (h * kPage) + (pos & (kPage - 1));
            const uint32_t word = ldg32(pg + (kv ? kVWords : kKWords) + (int64_t(slot) * kWords + wd) * 4);
            v.x = lut[word & 0xFF];
            v.y = lut[(word >> 8) & 0xFF];
            v.z = lut[(word >> 16) & 0xFF];
            v.w = lut[word >> 24];
            if (wd == 0) nrm = ldg_half(pg + (kv ? kVNorms : kKNorms) + slot * 2);
          }
        } else {
          const __half* src = (kv ? p.vr : p.kr) + (int64_t(pos - p.prefix_len) * kHkv + h) * kD;
          v = __ldg(reinterpret_cast<const uint4*>(src) + wd);
          nrm = 1.f;
        }
      }
      *reinterpret_cast<uint4*>((kv ? vs : ks) + pl * kPfStride + wd * 8) = v;
      if (wd == 0) (kv ? nvs : nks)[pl] = nrm;
    }
    __syncthreads();

    // ---- S = Q' K'^T for the warp's 16 rows x 64 positions
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a0, a1, a2, a3, smem_u32(qs + (16 * w + (lane & 15)) * kPfStride + kk * 16 + (lane >> 4) * 8));
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b0, b1, b2, b3,
                    smem_u32(ks + (8 * nt + (lane & 7) + 8 * (lane >> 4)) * kPfStride + kk * 16 +
                             ((lane >> 3) & 1) * 8));
        mma_16816(s[nt], a0, a1, a2, a3, b0, b1);
        mma_16816(s[nt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // ---- scale by K norms, mask, online softmax (rows g and g+8)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pl = 8 * nt + 2 * t + (i & 1);
        const bool ok = tile + pl < lim[i >> 1];
        s[nt][i] = ok ? s[nt][i] * nks[pl] : -INFINITY;
        mx[i >> 1] = fmaxf(mx[i >> 1], s[nt][i]);
      }
    float alpha[2], mu[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
      const float m_new = fmaxf(m_run[e], mx[e]);
      mu[e] = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[e] = exp2f((m_run[e] - mu[e]) * 1.4426950408889634f);
      m_run[e] = m_new;
      l_run[e] *= alpha[e];
    }
    // P' = p * n_v as an f16 hi + lo pair (two mma per step keep PV at fp32 precision)
    uint32_t pa[8][2], pb[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        pr[i] = exp2f((s[nt][i] - mu[i >> 1]) * 1.4426950408889634f);
        l_run[i >> 1] += pr[i];
      }
      const int pl = 8 * nt + 2 * t;
      const float v0 = nvs[pl], v1 = nvs[pl + 1];
      const float w0 = s[nt][0] == -INFINITY ? 0.f : pr[0] * v0, w1 = s[nt][1] == -INFINITY ? 0.f : pr[1] * v1;
      const float w2 = s[nt][2] == -INFINITY ? 0.f : pr[2] * v0, w3 = s[nt][3] == -INFINITY ? 0.f : pr[3] * v1;
      const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      pa[nt][0] = *reinterpret_cast<const uint32_t*>(&h01);
      pa[nt][1] = *reinterpret_cast<const uint32_t*>(&h23);
      pb[nt][0] = pack_half2(w0 - f01.x, w1 - f01.y);
      pb[nt][1] = pack_half2(w2 - f23.x, w3 - f23.y);
    }
#pragma unroll
    for (int nd = 0; nd < 32; ++nd) {
      o[nd][0] *= alpha[0];
      o[nd][1] *= alpha[0];
      o[nd][2] *= alpha[1];
      o[nd][3] *= alpha[1];
    }
    // ---- O' += P' V'
#pragma unroll
    for (int ks_ = 0; ks_ < 4; ++ks_) {
      const uint32_t a0 = pa[2 * ks_][0], a1 = pa[2 * ks_][1], a2 = pa[2 * ks_ + 1][0], a3 = pa[2 * ks_ + 1][1];
      const uint32_t c0 = pb[2 * ks_][0], c1 = pb[2 * ks_][1], c2 = pb[2 * ks_ + 1][0], c3 = pb[2 * ks_ + 1][1];
#pragma unroll
      for (int nd = 0; nd < 32; nd += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3,
                          smem_u32(vs + (16 * ks_ + (lane & 7) + 8 * ((lane >> 3) & 1)) * kPfStride +
                                   8 * (nd + (lane >> 4))));
        mma_16816(o[nd], a0, a1, a2, a3, b0, b1);
        mma_16816(o[nd + 1], a0, a1, a2, a3, b2, b3);
        mma_16816(o[nd], c0, c1, c2, c3, b0, b1);
        mma_16816(o[nd + 1], c0, c1, c2, c3, b2, b3);
      }
    }
  }

  // ---- epilogue: o' / l -> smem (fp32), then R^T per row and bf16 out
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], 1);
    l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], 2);
  }
  __syncthreads();
  float* os = reinterpret_cast<float*>(ks);  // [64][kD + 4] fp32 fits in the K and V tiles
  constexpr int kOs = kD + 4;
  const float inv0 = l_run[0] > 0.f ? 0.0625f / l_run[0] : 0.f;
  const float inv1 = l_run[1] > 0.f ? 0.0625f / l_run[1] : 0.f;
#pragma unroll
  for (int nd = 0; nd < 32; ++nd) {
    const int col = 8 * nd + 2 * t;
    os[(16 * w + g) * kOs + col] = o[nd][0] * inv0;
    os[(16 * w + g) * kOs + col + 1] = o[nd][1] * inv0;
    os[(16 * w + g + 8) * kOs + col] = o[nd][2] * inv1;
    os[(16 * w + g + 8) * kOs + col + 1] = o[nd][3] * inv1;
  }
  __syncthreads();
  for (int r = w; r < kPfRows; r += kPfThreads / 32) {
    const int row = row0 + r;
    if (row >= m_total) break;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = os[r * kOs + lane * 8 + i];
    warp_fwht256(v);
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i] * sign_of(p.signs, lane * 8 + 2 * i),
                                                v[2 * i + 1] * sign_of(p.signs, lane * 8 + 2 * i + 1));
      pk[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    const int tok = row / 6, j = row % 6;
    *reinterpret_cast<uint4*>(p.out + (int64_t(tok) * kHq + h * kGroup + j) * kD + lane * 8) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

inline cudaError_t prefill_set_attrs() {
  return cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPfSmem));
}

inline cudaError_t launch_prefill(const uint8_t* pool, int32_t num_pages, const int32_t* page_table,
                                  int32_t prefix_len, const uint16_t* q, const uint16_t* kc,
                                  const uint16_t* vc, int32_t n_tok, float scale, uint16_t* out,
                                  void* workspace, const Signs& signs, int* status, int num_sms,
                                  cudaStream_t stream) {
  (void)num_sms;
  __half* qr = static_cast<__half*>(workspace);
  __half* kr = qr + size_t(n_tok) * kHq * kD;
  __half* vr = kr + size_t(n_tok) * kHkv * kD;
  const int64_t vecs = int64_t(n_tok) * (kHq + 2 * kHkv);
  prefill_rotate_kernel<<<unsigned((vecs + 7) / 8), 256, 0, stream>>>(q, kc, vc, n_tok, scale, qr, kr, vr,
                                                                        signs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  PrefillParams p{};
  p.pool = pool;
  p.num_pages = num_pages;
  p.page_table = page_table;
  p.prefix_len = prefix_len;
  p.n_tok = n_tok;
  p.qr = qr;
  p.kr = kr;
  p.vr = vr;
  p.out = out;
  p.signs = signs;
  p.status = status;
  const dim3 grid(unsigned((6 * n_tok + kPfRows - 1) / kPfRows), kHkv);
  prefill_attn_kernel<<<grid, kPfThreads, kPfSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace tq4
