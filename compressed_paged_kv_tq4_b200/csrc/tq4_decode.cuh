// TQ4 split-K decode attention + combine (sm_100a).
//
// What it computes ([KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into
// 24 GiB of Laptop Memory", section "KVExec": page-native decode straight on
// the compressed data; [V2] wpnews.pro "JustFit: Run Qwen 27B Fast ...",
// mechanism table row KVExec: rotated-domain attention):
//
//   o = softmax_j(scale * q . x_hat_j) over positions j, with
//   x_hat_j = n_j R^T c[idx_j]. Because R is orthogonal,
//   q . x_hat_j = n_j (R q) . c[idx_j]   and   sum_j p_j v_hat_j = R^T sum_j p_j n_j c[idx_j],
// so each CTA rotates its queries once (q' = R q * scale), scores packed keys
// directly against centroid values, accumulates o' = sum p n c in the rotated
// domain and the combine pass applies R^T once per output row.
//
// Work split: grid (items, 4 KV heads); an item is (request, split) where a
// split is split_len consecutive positions (split_len % 64 == 0). A CTA of 4
// warps walks its split in chunks of 64 positions:
//   K phase  warp w takes positions 16w..16w+15 of the chunk: S = C_k . Q'^T
//            on mma.m16n8k16 (M = positions, N = 6 query heads x n_q tokens,
//            K = dims), nibble pairs decoded through a per-lane smem table.
//   softmax  chunk max exchanged through smem; p = exp(s - m), P' = p * n_v
//            written transposed (f16) to smem.
//   V phase  warp w takes dims 64w..64w+63 of all 64 positions:
//            O'^T += C_v^T . P'^T (M = dims, N = query rows, K = positions).
// Per-split partial results (m, l, o') go to the workspace; the combine pass
// merges them (log-sum-exp), rotates back and writes bf16/fp32.
#pragma once
#include "tq4_device.cuh"

namespace tq4 {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kChunk = 16 * kDecWarps;       // positions per chunk
constexpr int kQvStride = kD + 8;            // halves per Q' row in smem (bank-conflict pad)
constexpr int kPsStride = kChunk + 8;        // halves per P' row in smem
constexpr int kRowsMax = 24;                 // 6 query heads x 4 tokens
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
  const uint8_t* pool;
  int32_t num_pages;
  const uint16_t* q;
  const int32_t* page_tables;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t n_req;
  int32_t n_q;
  float scale;
  int32_t split_len;
  int32_t items_ub;
  int32_t rows_pad;    // 8 * NT
  float* ws_o;         // [items_ub][4][rows_pad][256]
  float2* ws_ml;       // [items_ub][4][rows_pad] (m, l)
  void* out;
  int out_dtype;
  Signs signs;
  int* status;
};

__host__ __device__ constexpr int decode_nt(int n_q) { return (6 * n_q + 7) / 8; }

template <int NT>
constexpr size_t decode_smem_bytes() {
  return size_t(kLutBytes) + size_t(8 * NT) * kQvStride * 2 + size_t(8 * NT) * kPsStride * 2 +
         size_t(kDecWarps) * 8 * NT * 4;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

__device__ __forceinline__ bool seq_ok(int s, int n_q, int max_pages) {
  return s >= n_q && s <= max_pages * kPage;
}

// Warp-collective: find (request, split) of item x. Returns false if x is not
// an item. *total receives the number of items (sum of splits).
__device__ __forceinline__ bool find_item(const DecodeParams& p, int x, int& req, int& split,
                                          int& total) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  bool found = false;
  for (int r0 = 0; r0 < p.n_req; r0 += 32) {
    const int r = r0 + lane;
    int S = 0;
    if (r < p.n_req) {
      const int s = __ldg(p.seq_lens + r);
      S = seq_ok(s, p.n_q, p.max_pages) ? (s + p.split_len - 1) / p.split_len : 0;
    }
    const int incl = warp_incl_scan(S);
    const int excl = incl - S;
    const bool hit = S > 0 && x >= base + excl && x < base + incl;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m && !found) {
      const int src = __ffs(m) - 1;
      req = r0 + src;
      split = x - base - __shfl_sync(0xffffffffu, excl, src);
      found = true;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  total = base;
  return found;
}

// Registers holding one chunk's packed data for one thread.
struct ChunkRegs {
  uint4 ka0, ka1, kb0, kb1;   // K words: positions g and g+8 of the warp's 16
  uint32_t vw[16];            // V word (8w+g) of positions 16ks + {2t, 2t+1, 2t+8, 2t+9}
  float kn[2], vn[2];         // K and V norms of positions g and g+8
};

__device__ __forceinline__ uint32_t pick(const uint4& a, const uint4& b, int i) {
  switch (i) {
    case 0: return a.x; case 1: return a.y; case 2: return a.z; case 3: return a.w;
    case 4: return b.x; case 5: return b.y; case 6: return b.z; default: return b.w;
  }
}

template <int NT>
__global__ void __launch_bounds__(kDecThreads, 2) decode_splitk_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const char* lut = reinterpret_cast<const char*>(smem);
  __half* qv = reinterpret_cast<__half*>(smem + kLutBytes);
  __half* ps = qv + 8 * NT * kQvStride;
  float* red = reinterpret_cast<float*>(ps + 8 * NT * kPsStride);   // [warps][8*NT]
  __shared__ int s_item[3];

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const uint32_t lane4 = uint32_t(lane) * 4u;

  if (w == 0) {
    int req = 0, split = 0, total = 0;
    const bool ok = find_item(p, blockIdx.x, req, split, total);
    if (lane == 0) {
      s_item[0] = ok ? req : -1;
      s_item[1] = split;
      if (blockIdx.x == 0 && h == 0 && total > p.items_ub) record_error(p.status, TQ4_ERR_SEQ);
    }
  }
  __syncthreads();
  const int r = s_item[0];
  if (r < 0 || int(blockIdx.x) >= p.items_ub) return;
  const int split = s_item[1];
  const int seq_len = __ldg(p.seq_lens + r);
  const int pos_b = split * p.split_len;
  const int pos_e = min(pos_b + p.split_len, seq_len);
  const int NR = 6 * p.n_q;

  // ---- rotate the queries of this (request, KV head): q' = R q * scale, f16, virtual order
  for (int row = w; row < 8 * NT; row += kDecWarps) {
    float v[8];
    if (row < NR) {
      const int tok = row / 6, j = row % 6;
      const uint16_t* src = p.q + ((int64_t(r) * p.n_q + tok) * kHq + h * kGroup + j) * kD + lane * 8;
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
    // lane owns real dims 8*lane + i (word lane). Word lane is loaded by K-phase thread
    // t = (lane & 15) >> 2 as its word index ws = (lane & 3) + 4*(lane >> 4); k-step
    // kk = 2*ws + (i >> 2), mma column 2t + (i & 1) + 8*((i >> 1) & 1).
    const int tt = (lane & 15) >> 2, wsel = (lane & 3) + 4 * (lane >> 4);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int kk = 2 * wsel + (i >> 2);
      const int col = kk * 16 + ((i >> 1) & 1) * 8 + 2 * tt;
      *reinterpret_cast<uint32_t*>(qv + row * kQvStride + col) = pack_half2(v[i], v[i + 1]);
    }
  }
  lut_fill(reinterpret_cast<uint32_t*>(smem), tid, kDecThreads);
  __syncthreads();

  // ---- B fragments of Q' for the K phase (registers when they fit)
  constexpr bool kQReg = (NT == 1);
  uint32_t qb[kQReg ? 16 : 1][2];
  if constexpr (kQReg) {
#pragma unroll
    for (int kk = 0; kk < 16; kk += 2) {
      const int m = lane >> 3;
      const uint32_t addr = smem_u32(qv + (lane & 7) * kQvStride + (kk + (m >> 1)) * 16 + (m & 1) * 8);
      ldmatrix_x4(qb[kk][0], qb[kk][1], qb[kk + 1][0], qb[kk + 1][1], addr);
    }
  }

  // per-row visibility limits for the rows this thread scores (rows nt*8 + 2t + e)
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = nt * 8 + 2 * t + e;
      lim[nt][e] = row < NR ? seq_len - p.n_q + row / 6 + 1 : 0;
    }

  float m_run[NT][2], l_part[NT][2];
  float o[NT][4][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_part[nt][0] = l_part[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[nt][mt][i] = 0.f;
  }

  const int32_t* table = p.page_tables + int64_t(r) * p.max_pages;
  const int64_t head_slot0 = int64_t(h) * kPage;

  auto load_chunk = [&](int c, ChunkRegs& cr) {
    int32_t page = __ldg(table + (c >> 8));
    const bool page_ok = page >= 0 && page < p.num_pages;
    if (!page_ok) {
      if (tid == 0) record_error(p.status, TQ4_ERR_PAGE_RANGE);
      page = 0;
    }
    const uint8_t* pg = p.pool + int64_t(page) * kPageBytes;
    const int slot0 = c & (kPage - 1);
    const int pk = c + 16 * w + g;  // K-phase positions pk, pk + 8
    const bool v0 = page_ok && pk < pos_e, v8 = page_ok && pk + 8 < pos_e;
    const uint8_t* kb = pg + kKWords + (head_slot0 + slot0 + 16 * w + g) * 128;
    const uint4 z = make_uint4(0, 0, 0, 0);
    cr.ka0 = v0 ? ldg128(kb + 16 * t) : z;
    cr.ka1 = v0 ? ldg128(kb + 64 + 16 * t) : z;
    cr.kb0 = v8 ? ldg128(kb + 8 * 128 + 16 * t) : z;
    cr.kb1 = v8 ? ldg128(kb + 8 * 128 + 64 + 16 * t) : z;
    const uint8_t* kn = pg + kKNorms + (head_slot0 + slot0 + 16 * w + g) * 2;
    const uint8_t* vn = pg + kVNorms + (head_slot0 + slot0 + 16 * w + g) * 2;
    cr.kn[0] = v0 ? ldg_half(kn) : 0.f;
    cr.kn[1] = v8 ? ldg_half(kn + 16) : 0.f;
    cr.vn[0] = v0 ? ldg_half(vn) : 0.f;
    cr.vn[1] = v8 ? ldg_half(vn + 16) : 0.f;
    const uint8_t* vb = pg + kVWords + (head_slot0 + slot0) * 128 + (8 * w + g) * 4;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pl = 16 * ks + 2 * t + (j & 1) + 8 * (j >> 1);
        cr.vw[ks * 4 + j] = (page_ok && c + pl < pos_e) ? ldg32(vb + pl * 128) : 0u;
      }
  };

  ChunkRegs nxt;
  if (pos_b < pos_e) load_chunk(pos_b, nxt);

  for (int c = pos_b; c < pos_e; c += kChunk) {
    const ChunkRegs cur = nxt;
    if (c + kChunk < pos_e) load_chunk(c + kChunk, nxt);

    // ------------------------------------------------------------ K phase: S = C_k Q'^T
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const uint32_t wg = pick(cur.ka0, cur.ka1, kk >> 1);
      const uint32_t wg8 = pick(cur.kb0, cur.kb1, kk >> 1);
      uint32_t a0, a1, a2, a3;
      if (kk & 1) {
        a0 = lut_decode<2>(lut, wg, lane4);
        a1 = lut_decode<2>(lut, wg8, lane4);
        a2 = lut_decode<3>(lut, wg, lane4);
        a3 = lut_decode<3>(lut, wg8, lane4);
      } else {
        a0 = lut_decode<0>(lut, wg, lane4);
        a1 = lut_decode<0>(lut, wg8, lane4);
        a2 = lut_decode<1>(lut, wg, lane4);
        a3 = lut_decode<1>(lut, wg8, lane4);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t b0, b1;
        if constexpr (kQReg) {
          b0 = qb[kk][0];
          b1 = qb[kk][1];
        } else {
          const int m = (lane >> 3) & 1;
          ldmatrix_x2(b0, b1, smem_u32(qv + (nt * 8 + (lane & 7)) * kQvStride + kk * 16 + m * 8));
        }
        mma_16816(s[nt], a0, a1, a2, a3, b0, b1);
      }
    }

    // ------------------------------------------------------------ online softmax
    const int pk = c + 16 * w + g;
    float mx[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pos = pk + 8 * (i >> 1);
        const bool ok = pos < pos_e && pos < lim[nt][i & 1];
        s[nt][i] = ok ? s[nt][i] * cur.kn[i >> 1] : -INFINITY;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = fmaxf(s[nt][e], s[nt][e + 2]);
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        mx[nt][e] = v;
      }
      if (g == 0) {
        red[w * 8 * NT + nt * 8 + 2 * t] = mx[nt][0];
        red[w * 8 * NT + nt * 8 + 2 * t + 1] = mx[nt][1];
      }
    }
    __syncthreads();
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mc = red[nt * 8 + 2 * t + e];
#pragma unroll
        for (int ww = 1; ww < kDecWarps; ++ww) mc = fmaxf(mc, red[ww * 8 * NT + nt * 8 + 2 * t + e]);
        const float m_new = fmaxf(m_run[nt][e], mc);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][e] = exp2f((m_run[nt][e] - m_use) * kLog2e);
        m_run[nt][e] = m_new;
        mx[nt][e] = m_use;
      }
      float pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pr[i] = exp2f((s[nt][i] - mx[nt][i & 1]) * kLog2e);
      l_part[nt][0] = l_part[nt][0] * alpha[nt][0] + pr[0] + pr[2];
      l_part[nt][1] = l_part[nt][1] * alpha[nt][1] + pr[1] + pr[3];
      const uint32_t p0 = pack_half2(pr[0] * cur.vn[0], pr[1] * cur.vn[0]);
      const uint32_t p1 = pack_half2(pr[2] * cur.vn[1], pr[3] * cur.vn[1]);
      const int j = lane & 7, mat = (lane >> 3) & 1;
      stmatrix_x2_trans(smem_u32(ps + (nt * 8 + j) * kPsStride + 16 * w + 8 * mat), p0, p1);
    }
    __syncthreads();

    // ------------------------------------------------------------ V phase: O'^T += C_v^T P'^T
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        o[nt][mt][0] *= alpha[nt][0];
        o[nt][mt][1] *= alpha[nt][1];
        o[nt][mt][2] *= alpha[nt][0];
        o[nt][mt][3] *= alpha[nt][1];
      }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t lo01, hi01, lo89, hi89;
      interleave_nibbles(cur.vw[ks * 4 + 0], cur.vw[ks * 4 + 1], lo01, hi01);
      interleave_nibbles(cur.vw[ks * 4 + 2], cur.vw[ks * 4 + 3], lo89, hi89);
      uint32_t b[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = (lane >> 3) & 1;
        ldmatrix_x2(b[nt][0], b[nt][1], smem_u32(ps + (nt * 8 + (lane & 7)) * kPsStride + 16 * ks + 8 * m));
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t a0, a1, a2, a3;
        switch (mt) {
          case 0:
            a0 = lut_decode<0>(lut, lo01, lane4); a1 = lut_decode<0>(lut, hi01, lane4);
            a2 = lut_decode<0>(lut, lo89, lane4); a3 = lut_decode<0>(lut, hi89, lane4);
            break;
          case 1:
            a0 = lut_decode<1>(lut, lo01, lane4); a1 = lut_decode<1>(lut, hi01, lane4);
            a2 = lut_decode<1>(lut, lo89, lane4); a3 = lut_decode<1>(lut, hi89, lane4);
            break;
          case 2:
            a0 = lut_decode<2>(lut, lo01, lane4); a1 = lut_decode<2>(lut, hi01, lane4);
            a2 = lut_decode<2>(lut, lo89, lane4); a3 = lut_decode<2>(lut, hi89, lane4);
            break;
          default:
            a0 = lut_decode<3>(lut, lo01, lane4); a1 = lut_decode<3>(lut, hi01, lane4);
            a2 = lut_decode<3>(lut, lo89, lane4); a3 = lut_decode<3>(lut, hi89, lane4);
            break;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(o[nt][mt], a0, a1, a2, a3, b[nt][0], b[nt][1]);
      }
    }
  }

  // ---------------------------------------------------------------- partial results
  // l: sum over the lanes sharing t (positions g) and over the 4 warps' K phases
  __syncthreads();
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = l_part[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      if (g == 0) red[w * 8 * NT + nt * 8 + 2 * t + e] = v;
    }
  __syncthreads();
  const int64_t rec = (int64_t(blockIdx.x) * kHkv + h) * p.rows_pad;
  if (tid < 8 * NT) {
    float l = 0.f;
#pragma unroll
    for (int ww = 0; ww < kDecWarps; ++ww) l += red[ww * 8 * NT + tid];
    // m of row tid: held by the lanes with t = (tid % 8) / 2 of n-tile tid / 8 (any warp)
    red[tid] = l;  // only this thread reads/writes slot tid after the barrier above
  }
  // each thread with g == 0 knows m for its rows; publish through ws directly
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = nt * 8 + 2 * t + e;
      float* dst = p.ws_o + (rec + row) * kD + 64 * w + 8 * g;
      reinterpret_cast<float4*>(dst)[0] =
          make_float4(o[nt][0][e], o[nt][0][e + 2], o[nt][1][e], o[nt][1][e + 2]);
      reinterpret_cast<float4*>(dst)[1] =
          make_float4(o[nt][2][e], o[nt][2][e + 2], o[nt][3][e], o[nt][3][e + 2]);
    }
  __syncthreads();
  if (w == 0 && g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = nt * 8 + 2 * t + e;
        p.ws_ml[rec + row] = make_float2(m_run[nt][e], red[row]);
      }
  }
}

// One warp per output row (request, token, query head).
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const int lane = threadIdx.x & 31;
  const int row_id = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row_id >= p.n_req * p.n_q * kHq) return;
  const int qh = row_id % kHq;
  const int tok = (row_id / kHq) % p.n_q;
  const int r = row_id / (kHq * p.n_q);
  const int h = qh / kGroup;
  const int row = tok * kGroup + qh % kGroup;

  // first item of request r and its number of splits
  int first = 0;
  for (int r0 = 0; r0 < r; r0 += 32) {
    const int rr = r0 + lane;
    int S = 0;
    if (rr < r) {
      const int s = __ldg(p.seq_lens + rr);
      S = seq_ok(s, p.n_q, p.max_pages) ? (s + p.split_len - 1) / p.split_len : 0;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    first += S;
  }
  const int s_len = __ldg(p.seq_lens + r);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float l = 0.f;
  const bool ok = seq_ok(s_len, p.n_q, p.max_pages);
  const int n_split = ok ? (s_len + p.split_len - 1) / p.split_len : 0;
  if (!ok && lane == 0) record_error(p.status, TQ4_ERR_SEQ);
  if (first + n_split > p.items_ub) {
    if (lane == 0) record_error(p.status, TQ4_ERR_SEQ);
  } else if (n_split > 0) {
    float m = -INFINITY;
    for (int x = first; x < first + n_split; ++x)
      m = fmaxf(m, p.ws_ml[(int64_t(x) * kHkv + h) * p.rows_pad + row].x);
    for (int x = first; x < first + n_split; ++x) {
      const int64_t rec = (int64_t(x) * kHkv + h) * p.rows_pad + row;
      const float2 ml = p.ws_ml[rec];
      if (ml.x == -INFINITY) continue;
      const float wgt = exp2f((ml.x - m) * kLog2e);
      l = fmaf(wgt, ml.y, l);
      const float4* src = reinterpret_cast<const float4*>(p.ws_o + rec * kD + lane * 8);
      const float4 u0 = src[0], u1 = src[1];
      acc[0] = fmaf(wgt, u0.x, acc[0]); acc[1] = fmaf(wgt, u0.y, acc[1]);
      acc[2] = fmaf(wgt, u0.z, acc[2]); acc[3] = fmaf(wgt, u0.w, acc[3]);
      acc[4] = fmaf(wgt, u1.x, acc[4]); acc[5] = fmaf(wgt, u1.y, acc[5]);
      acc[6] = fmaf(wgt, u1.z, acc[6]); acc[7] = fmaf(wgt, u1.w, acc[7]);
    }
  }
  // o = R^T (o' / l) = diag(s) H (o' / l) / 16
  warp_fwht256(acc);
  const float inv = (l > 0.f) ? 0.0625f / l : 0.f;
  float res[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) res[i] = acc[i] * inv * sign_of(p.signs, lane * 8 + i);
  const int64_t off = ((int64_t(r) * p.n_q + tok) * kHq + qh) * kD + lane * 8;
  if (p.out_dtype == TQ4_DTYPE_F32) {
    float* dst = static_cast<float*>(p.out) + off;
    reinterpret_cast<float4*>(dst)[0] = make_float4(res[0], res[1], res[2], res[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(res[4], res[5], res[6], res[7]);
  } else {
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(res[2 * i], res[2 * i + 1]);
      pk[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

}  // namespace tq4
