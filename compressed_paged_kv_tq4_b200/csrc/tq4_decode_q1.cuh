// TQ4 split-K decode attention for one query token per request (sm_100a).
//
// Same computation as the general split-K kernel (rotated-domain attention over
// packed pages; [KVEXEC] simpleprog.com "Fitting a 27B-Parameter LLM into 24 GiB
// of Laptop Memory", section "KVExec"; [V2] wpnews.pro "JustFit: Run Qwen 27B
// Fast ...", mechanism table row KVExec), organised so that warps never wait on
// each other inside the main loop:
//
//   * a CTA (8 warps) owns one (request, KV head, split); warp w takes the
//     16-position tiles w, w+8, w+16, ... of the split;
//   * each warp stages its own tiles through a private cp.async ring
//     (K words, V words, norms: 4,160 bytes per tile);
//   * K phase: S = C_k (q'_hi + q'_lo) on mma.m16n8k16 (M = 16 positions,
//     N = 6 query heads padded to 8, K = 256 dims);
//   * in-warp online softmax; P' = p * n_v split into f16 hi + lo and moved
//     into B-operand layout with movmatrix (no shared memory);
//   * V phase: O'^T += C_v^T P'^T over all 256 dims (M = dims, K = positions);
//   * at the end the 8 warp states (m, l, o') are merged through shared memory
//     and written as one split-K partial for the combine pass.
#pragma once
#include "tq4_decode.cuh"

namespace tq4 {

constexpr int kQ1Warps = 8;
constexpr int kQ1Threads = 32 * kQ1Warps;
constexpr int kQ1Stages = 4;
constexpr int kQ1TileBytes = 16 * 128 * 2 + 16 * 2 * 2;    // K words, V words, K norms, V norms
constexpr int kQ1WarpRing = kQ1Stages * kQ1TileBytes;        // 16,640 B
// Shared-window layout (absolute 32-bit shared addresses): the centroid table
// sits at 0x10000 so that one byte permute builds a lookup address
// (0x10000 | byte << 8 | lane * 4). Below it: control words, q' and the rings
// of warps 0..2; above it: the rings of warps 3..7 (also the merge area).
constexpr uint32_t kQ1Lut = 0x10000;
constexpr uint32_t kQ1Hi = 0x20000;
constexpr int kQ1LowWarps = 3;
constexpr uint32_t kQ1LowBytes = 128 + 2 * 8 * kQvStride * 2 + kQ1LowWarps * kQ1WarpRing;   // 58,496
constexpr uint32_t kQ1DynBytes = kQ1Hi + (kQ1Warps - kQ1LowWarps) * kQ1WarpRing;            // 214,272
constexpr int kQ1MergeBytes = kQ1Warps * (8 * kD + 16) * 4;
static_assert(kQ1MergeBytes <= (kQ1Warps - kQ1LowWarps) * kQ1WarpRing, "merge area fits above the table");
constexpr float kQ1PScale = 1.0f / 256.0f;   // P' = p * n_v / 256 (undone in the combine)
constexpr float kQ1Lazy = 8.0f;              // rescale only when a row max grows by > 2^8 (log2 units)

constexpr size_t decode_q1_smem_bytes() { return kQ1DynBytes; }

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
// byte K of w -> f16x2 centroid pair from the table at kQ1Lut
template <int K>
__device__ __forceinline__ uint32_t lut64k(uint32_t w, uint32_t lanebase) {
  constexpr uint32_t sel = (7u << 12) | (6u << 8) | (uint32_t(K) << 4) | 4u;
  return ld_shared_u32(__byte_perm(w, lanebase, sel));
}

__global__ void __launch_bounds__(kQ1Threads, 1) decode_q1_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  if (base + kQ1LowBytes > kQ1Lut) {   // the layout needs the dynamic window to start low
    if (tid == 0) record_error(p.status, TQ4_ERR_CUDA);
    return;
  }
  int* s_item = reinterpret_cast<int*>(smem);
  __half* qv_hi = reinterpret_cast<__half*>(smem + 128);
  __half* qv_lo = qv_hi + 8 * kQvStride;
  const uint32_t ring = w < kQ1LowWarps ? base + 128 + 2 * 8 * kQvStride * 2 + w * kQ1WarpRing
                                        : kQ1Hi + (w - kQ1LowWarps) * kQ1WarpRing;
  const uint32_t lanebase = kQ1Lut | (uint32_t(lane) * 4u);

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
  const int n_tiles = (pos_e - pos_b + 15) >> 4;
  const int my_tiles = n_tiles > w ? (n_tiles - w + kQ1Warps - 1) / kQ1Warps : 0;
  const int32_t* table = p.page_tables + int64_t(r) * p.max_pages;
  const uint8_t* pool = p.pool;
  const int num_pages = p.num_pages;
  const int64_t head_off = int64_t(h) * kPage * 128;        // head's first word row inside a region

  // per-lane copy plan: 8 word segments (K then V) and, for lanes 0..3, one norm segment
  int src_off[8];
  uint32_t dst_off[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    const int kv = e >> 7, pl = (e >> 3) & 15, sg = e & 7;
    src_off[j] = int(kv ? kVWords : kKWords) + pl * 128 + sg * 16;
    dst_off[j] = uint32_t(kv * 2048 + pl * 128 + ((sg ^ seg_swz(pl)) << 4));
  }
  const int nrm_src = int((lane >> 1) ? kVNorms : kKNorms) + (lane & 1) * 16;
  const uint32_t nrm_dst = 4096 + (lane >> 1) * 32 + (lane & 1) * 16;

  auto tile_pos = [&](int k) { return pos_b + ((w + k * kQ1Warps) << 4); };
  int page_next = my_tiles > 0 ? __ldg(table + (tile_pos(0) >> 8)) : 0;
  auto issue_tile = [&](int k) {
    if (k < my_tiles) {
      const int c = tile_pos(k);
      const int page = page_next;
      if (k + 1 < my_tiles) page_next = __ldg(table + (tile_pos(k + 1) >> 8));
      if (page < 0 || page >= num_pages) {
        if (lane == 0) record_error(p.status, TQ4_ERR_PAGE_RANGE);
      } else {
        const int nvalid = min(16, pos_e - c);
        const uint8_t* tb = pool + int64_t(page) * kPageBytes + head_off + (c & (kPage - 1)) * 128;
        const uint32_t st = ring + (k % kQ1Stages) * kQ1TileBytes;
        if (nvalid == 16) {
#pragma unroll
          for (int j = 0; j < 8; ++j) cp_async16(st + dst_off[j], tb + src_off[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (((lane + 32 * j) >> 3 & 15) < nvalid) cp_async16(st + dst_off[j], tb + src_off[j]);
        }
        // norms: K and V, 16 halves each (2 x 2 segments); slot offset = word offset / 64
        if (lane < 4 && (lane & 1) * 8 < nvalid)
          cp_async16(st + nrm_dst, pool + int64_t(page) * kPageBytes + nrm_src +
                                       (head_off + (c & (kPage - 1)) * 128) / 64);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < kQ1Stages - 1; ++k) issue_tile(k);

  // ---- q' = R q * scale for the 6 query heads of this KV head, split hi + lo, virtual order
  {
    const int row = w;
    float v[8];
    if (row < 6) {
      const uint16_t* src = p.q + (int64_t(r) * kHq + h * kGroup + row) * kD + lane * 8;
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
    const int tt = (lane & 15) >> 2, wsel = (lane & 3) + 4 * (lane >> 4);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int kk = 2 * wsel + (i >> 2);
      const int col = kk * 16 + ((i >> 1) & 1) * 8 + 2 * tt;
      const __half2 hi = __floats2half2_rn(v[i], v[i + 1]);
      const float2 hf = __half22float2(hi);
      *reinterpret_cast<__half2*>(qv_hi + row * kQvStride + col) = hi;
      *reinterpret_cast<__half2*>(qv_lo + row * kQvStride + col) = __floats2half2_rn(v[i] - hf.x, v[i + 1] - hf.y);
    }
  }
  for (int e = tid; e < 256 * 32; e += kQ1Threads) {
    const int b = e >> 5, l = e & 31;
    st_shared_u32(kQ1Lut + b * 256 + l * 4,
                  uint32_t(g_codebook.c16[b & 15]) | (uint32_t(g_codebook.c16[b >> 4]) << 16));
  }
  __syncthreads();

  uint32_t qh[16][2], ql[16][2];
#pragma unroll
  for (int kk = 0; kk < 16; kk += 2) {
    const int m = lane >> 3;
    const int off = (lane & 7) * kQvStride + (kk + (m >> 1)) * 16 + (m & 1) * 8;
    ldmatrix_x4(qh[kk][0], qh[kk][1], qh[kk + 1][0], qh[kk + 1][1], smem_u32(qv_hi + off));
    ldmatrix_x4(ql[kk][0], ql[kk][1], ql[kk + 1][0], ql[kk + 1][1], smem_u32(qv_lo + off));
  }

  // rows 2t, 2t+1 (query heads); only 6 are real
  const bool row_ok0 = 2 * t < 6, row_ok1 = 2 * t + 1 < 6;
  // m_ref: the reference the exponentials use (raised lazily); m_run: true running max
  float m_ref[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int mt = 0; mt < 16; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;

  const uint32_t k_off0 = g * 128 + ((t ^ seg_swz(g)) << 4);
  const uint32_t k_off1 = g * 128 + (((4 + t) ^ seg_swz(g)) << 4);
  const uint32_t v_off0 = 2048 + (2 * t) * 128 + ((g ^ seg_swz(2 * t)) << 4);      // words 4g..4g+3, pos 2t
  const uint32_t v_off1 = 2048 + (2 * t + 1) * 128 + ((g ^ seg_swz(2 * t + 1)) << 4);  // pos 2t+1
  for (int k = 0; k < my_tiles; ++k) {
    issue_tile(k + kQ1Stages - 1);
    cp_async_wait<kQ1Stages - 1>();
    __syncwarp();
    const uint32_t st = ring + (k % kQ1Stages) * kQ1TileBytes;
    const int c = tile_pos(k);

    // ------------------------------------------------------------ K phase
    const uint4 ka0 = ld_shared_v4(st + k_off0);
    const uint4 ka1 = ld_shared_v4(st + k_off1);
    const uint4 kb0 = ld_shared_v4(st + k_off0 + 8 * 128);
    const uint4 kb1 = ld_shared_v4(st + k_off1 + 8 * 128);
    float sh[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float sl[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const uint32_t wg = pick(ka0, ka1, kk >> 1);
      const uint32_t wg8 = pick(kb0, kb1, kk >> 1);
      uint32_t a0, a1, a2, a3;
      if (kk & 1) {
        a0 = lut64k<2>(wg, lanebase); a1 = lut64k<2>(wg8, lanebase);
        a2 = lut64k<3>(wg, lanebase); a3 = lut64k<3>(wg8, lanebase);
      } else {
        a0 = lut64k<0>(wg, lanebase); a1 = lut64k<0>(wg8, lanebase);
        a2 = lut64k<1>(wg, lanebase); a3 = lut64k<1>(wg8, lanebase);
      }
      mma_16816(sh[kk & 1], a0, a1, a2, a3, qh[kk][0], qh[kk][1]);
      mma_16816(sl[kk & 1], a0, a1, a2, a3, ql[kk][0], ql[kk][1]);
    }

    // ------------------------------------------------------------ in-warp online softmax
    const float kn0 = __half2float(__ushort_as_half(ld_shared_u16(st + 4096 + 2 * g)));
    const float kn8 = __half2float(__ushort_as_half(ld_shared_u16(st + 4096 + 2 * g + 16)));
    const float vn0 = __half2float(__ushort_as_half(ld_shared_u16(st + 4128 + 2 * g))) * kQ1PScale;
    const float vn8 = __half2float(__ushort_as_half(ld_shared_u16(st + 4128 + 2 * g + 16))) * kQ1PScale;
    const bool p0 = c + g < pos_e, p8 = c + g + 8 < pos_e;
    float s[4];
    s[0] = (p0 && row_ok0) ? ((sh[0][0] + sh[1][0]) + (sl[0][0] + sl[1][0])) * kn0 : -INFINITY;
    s[1] = (p0 && row_ok1) ? ((sh[0][1] + sh[1][1]) + (sl[0][1] + sl[1][1])) * kn0 : -INFINITY;
    s[2] = (p8 && row_ok0) ? ((sh[0][2] + sh[1][2]) + (sl[0][2] + sl[1][2])) * kn8 : -INFINITY;
    s[3] = (p8 && row_ok1) ? ((sh[0][3] + sh[1][3]) + (sl[0][3] + sl[1][3])) * kn8 : -INFINITY;
    // scores in log2 units from here on
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j] *= kLog2e;
    bool raise = false;
    float alpha[2] = {1.f, 1.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = fmaxf(s[e], s[e + 2]);
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      if (v > m_ref[e] + kQ1Lazy) {       // raise the reference: weights would exceed 2^8
        alpha[e] = fast_exp2(m_ref[e] - v);   // 0 on the first raise (m_ref = -inf)
        m_ref[e] = v;
        raise = true;
      }
    }
    const float mu0 = m_ref[0] == -INFINITY ? 0.f : m_ref[0];
    const float mu1 = m_ref[1] == -INFINITY ? 0.f : m_ref[1];
    float pr[4];
    pr[0] = fast_exp2(s[0] - mu0);
    pr[1] = fast_exp2(s[1] - mu1);
    pr[2] = fast_exp2(s[2] - mu0);
    pr[3] = fast_exp2(s[3] - mu1);
    if (__any_sync(0xffffffffu, raise)) {
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
    l_part[0] += pr[0] + pr[2];
    l_part[1] += pr[1] + pr[3];
    // P' = p * n_v / 256 (exp2(-inf) = 0 where masked; stale norms are multiplied by 0
    // only if finite, so select), f16 hi + lo, transposed into B fragments
    const float w0 = s[0] == -INFINITY ? 0.f : pr[0] * vn0;
    const float w1 = s[1] == -INFINITY ? 0.f : pr[1] * vn0;
    const float w2 = s[2] == -INFINITY ? 0.f : pr[2] * vn8;
    const float w3 = s[3] == -INFINITY ? 0.f : pr[3] * vn8;
    const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    const __half2 l01 = __floats2half2_rn(w0 - f01.x, w1 - f01.y);
    const __half2 l23 = __floats2half2_rn(w2 - f23.x, w3 - f23.y);
    const uint32_t bh0 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
    const uint32_t bh1 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
    const uint32_t bl0 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&l01));
    const uint32_t bl1 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&l23));

    // ------------------------------------------------------------ V phase (all 256 dims)
    const uint4 x0 = ld_shared_v4(st + v_off0);             // words 4g..4g+3 of position 2t
    const uint4 x1 = ld_shared_v4(st + v_off1);             // position 2t+1
    const uint4 y0 = ld_shared_v4(st + v_off0 + 8 * 128);   // position 2t+8 (same swizzle)
    const uint4 y1 = ld_shared_v4(st + v_off1 + 8 * 128);   // position 2t+9
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t lo01, hi01, lo89, hi89;
      interleave_nibbles(pick(x0, x0, q), pick(x1, x1, q), lo01, hi01);
      interleave_nibbles(pick(y0, y0, q), pick(y1, y1, q), lo89, hi89);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        uint32_t a0, a1, a2, a3;
        switch (kb) {
          case 0:
            a0 = lut64k<0>(lo01, lanebase); a1 = lut64k<0>(hi01, lanebase);
            a2 = lut64k<0>(lo89, lanebase); a3 = lut64k<0>(hi89, lanebase);
            break;
          case 1:
            a0 = lut64k<1>(lo01, lanebase); a1 = lut64k<1>(hi01, lanebase);
            a2 = lut64k<1>(lo89, lanebase); a3 = lut64k<1>(hi89, lanebase);
            break;
          case 2:
            a0 = lut64k<2>(lo01, lanebase); a1 = lut64k<2>(hi01, lanebase);
            a2 = lut64k<2>(lo89, lanebase); a3 = lut64k<2>(hi89, lanebase);
            break;
          default:
            a0 = lut64k<3>(lo01, lanebase); a1 = lut64k<3>(hi01, lanebase);
            a2 = lut64k<3>(lo89, lanebase); a3 = lut64k<3>(hi89, lanebase);
            break;
        }
        mma_16816(o[4 * q + kb], a0, a1, a2, a3, bh0, bh1);
        mma_16816(o[4 * q + kb], a0, a1, a2, a3, bl0, bl1);
      }
    }
    __syncwarp();   // all lanes are done with this slot before it is refilled
  }
  cp_async_wait<0>();

  // ---------------------------------------------------------------- merge the 8 warp states
  // (m in natural-log units, so the combine pass sees the same units from every kernel)
  __syncthreads();
  float* mrg = reinterpret_cast<float*>(smem + (kQ1Hi - base));   // per warp: o'[8 rows][256], m[8], l[8]
  float* mine = mrg + w * (8 * kD + 16);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float lv = l_part[e];
    lv += __shfl_xor_sync(0xffffffffu, lv, 4);
    lv += __shfl_xor_sync(0xffffffffu, lv, 8);
    lv += __shfl_xor_sync(0xffffffffu, lv, 16);
    const int row = 2 * t + e;
    if (g == 0) {
      mine[8 * kD + row] = m_ref[e] == -INFINITY ? -INFINITY : m_ref[e] / kLog2e;
      mine[8 * kD + 8 + row] = lv;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {   // dims 32g + 8q + 0..7 of row 2t+e
      float* d = mine + row * kD + 32 * g + 8 * q;
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
    for (int ww = 0; ww < kQ1Warps; ++ww) M = fmaxf(M, mrg[ww * (8 * kD + 16) + 8 * kD + row]);
    float L = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kQ1Warps; ++ww) {
        const float* src = mrg + ww * (8 * kD + 16);
        const float a = fast_exp2((src[8 * kD + row] - M) * kLog2e);
        L = fmaf(a, src[8 * kD + 8 + row], L);
        const float4 u0 = reinterpret_cast<const float4*>(src + row * kD + d0)[0];
        const float4 u1 = reinterpret_cast<const float4*>(src + row * kD + d0)[1];
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
