// Device-side building blocks shared by the TQ4 kernels (sm_100a).
//
// Format ([KVEXEC]: simpleprog.com "Fitting a 27B-Parameter LLM into 24 GiB of
// Laptop Memory", section "KVExec: Fused Reconstruction with Layer-Scoped
// Lifetime"): a 256-dim head vector is 32 u32 words of eight 4-bit centroid
// indices plus one fp16 norm; pages hold 256 positions of one layer.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/tq4.h"

namespace tq4 {

constexpr int kD = 256;          // head dim
constexpr int kPage = 256;       // positions per page
constexpr int kHkv = 4;          // KV heads
constexpr int kHq = 24;          // query heads
constexpr int kGroup = 6;        // query heads per KV head
constexpr int kWords = 32;       // u32 words per vector

// byte offsets inside one page (one layer)
constexpr int64_t kPageBytes = TQ4_PAGE_BYTES;
constexpr int64_t kKWords = 0;
constexpr int64_t kVWords = int64_t(kHkv) * kPage * kWords * 4;   // 131072
constexpr int64_t kKNorms = 2 * kVWords;                           // 262144
constexpr int64_t kVNorms = kKNorms + int64_t(kHkv) * kPage * 2;   // 264192

// Codebook in constant memory, written by the host from its fp64 Lloyd-Max
// solution (the same for every context; the signs are per context).
// The attention kernels feed the centroids to f16 tensor-core products as a
// hi + lo pair: c16 = f16(c), r16 = f16(c - c16), so c16 + r16 carries c to
// about 2^-21 relative while each half is an exact f16 operand.
struct Codebook {
  float c[16];        // centroids rounded to fp32 (reconstruction)
  float b[15];        // decision boundaries: fp64 midpoints of adjacent centroids, rounded to fp32 (encode)
  uint16_t c16[16];   // f16 bits of the centroids (round to nearest even)
  uint16_t r16[16];   // f16 bits of the rounding residuals c - c16
};
__constant__ Codebook g_codebook;  // one translation unit (tq4_api.cu) includes every kernel header

// Codebooks of the 2- and 3-bit variants (entry 0: 4 levels, entry 1: 8 levels),
// written by the host from its fp64 Lloyd-Max solutions like the 16-level one.
struct CodebookB {
  float c[8];         // centroids rounded to fp32
  float b[7];         // decision boundaries (fp64 midpoints, rounded to fp32)
  uint16_t c16[8];    // f16 bits of the centroids
  uint16_t r16[8];    // f16 bits of the rounding residuals
};
__constant__ CodebookB g_codebook_b[2];

// 256 sign bits: bit i set <=> s_i = -1. Passed by value to kernels.
struct Signs {
  uint32_t bits[8];
};

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// --------------------------------------------------------------------------
// Unnormalised Walsh-Hadamard transform of a 256-vector held by one warp,
// lane l owning coordinates 8l..8l+7 in v[0..7] (Sylvester / natural order).
// Butterflies over index bits 0..2 are in registers, bits 3..7 cross lanes.
// --------------------------------------------------------------------------
__device__ __forceinline__ void warp_fwht256(float v[8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & h) == 0) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

// The 8 sign bits of coordinates 8*lane .. 8*lane + 7 (bit i = coordinate 8*lane + i).
// Word lane / 4 is picked with constant indices behind an empty asm, so a Signs
// held in kernel parameters is not copied to local memory for an indexed read.
__device__ __forceinline__ uint32_t lane_sign_bits(const Signs& s) {
  const int lane = threadIdx.x & 31;
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t wk = s.bits[k];
    asm("" : "+r"(wk));
    w = ((lane >> 2) == k) ? wk : w;
  }
  return (w >> (8 * (lane & 3))) & 0xFFu;
}
// flip the sign of x when bit i of sb is set
__device__ __forceinline__ float apply_sign(float x, uint32_t sb, int i) {
  return __uint_as_float(__float_as_uint(x) ^ (((sb >> i) & 1u) << 31));
}

// sign of coordinate 8*lane + i as a float multiplier
__device__ __forceinline__ float sign_of(const Signs& s, int coord) {
  return ((s.bits[coord >> 5] >> (coord & 31)) & 1u) ? -1.0f : 1.0f;
}

// --------------------------------------------------------------------------
// Nibble-pair decode through a per-lane table in shared memory.
// Row b (one byte = two 4-bit indices) is 256 bytes; lane l reads its own
// 8-byte slot at b*256 + 8*l, so a warp's 64-bit loads are two conflict-free
// wavefronts. A slot holds f16x2 {c16[b & 15], c16[b >> 4]} followed by
// f16x2 {r16[b & 15], r16[b >> 4]} (the hi and lo halves of the centroids).
// --------------------------------------------------------------------------
constexpr int kLutBytes = 256 * 256;

// shared-memory load through a 32-bit shared-window address
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void ld_shared_v2(uint32_t addr, uint32_t& x, uint32_t& y) {
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];\n" : "=r"(x), "=r"(y) : "r"(addr));
}

// byte k (0..3) of w -> hi and lo f16x2 of its two nibbles (low nibble in the low half).
// lut_s is the table's 32-bit shared address; the byte lands in bits 8..15 of
// the offset and the lane's slot (8 * lane) in bits 0..7.
template <int K>
__device__ __forceinline__ void lut_decode(uint32_t lut_s, uint32_t w, uint32_t lane8, uint32_t& hi,
                                           uint32_t& lo) {
  constexpr uint32_t sel = (5u << 12) | (5u << 8) | (uint32_t(K) << 4) | 4u;
  ld_shared_v2(lut_s + __byte_perm(w, lane8, sel), hi, lo);
}

// One table row b as the 8-byte slot every lane stores: {c pair, r pair}.
__device__ __forceinline__ uint2 lut_row(int b) {
  return make_uint2(uint32_t(g_codebook.c16[b & 15]) | (uint32_t(g_codebook.c16[b >> 4]) << 16),
                    uint32_t(g_codebook.r16[b & 15]) | (uint32_t(g_codebook.r16[b >> 4]) << 16));
}

// The same slot for a 2- or 3-bit pool whose codes have been widened to nibbles
// (an index never exceeds 2^kBits - 1).
template <int kBits>
__device__ __forceinline__ uint2 lut_row_bits(int b) {
  const CodebookB& cb = g_codebook_b[kBits - 2];
  constexpr int m = (1 << kBits) - 1;
  return make_uint2(uint32_t(cb.c16[b & m]) | (uint32_t(cb.c16[(b >> 4) & m]) << 16),
                    uint32_t(cb.r16[b & m]) | (uint32_t(cb.r16[(b >> 4) & m]) << 16));
}

// Page layout of the 2- and 3-bit variants: per 256-dim vector 8 kBits u32 words
// (plane 0: the low two bits of every index, coordinate 16w + i in bits 2i..2i+1 of
// word w; plane 1, 3 bits only: bit 2, coordinate 32w + i in bit i of word 16 + w)
// plus one fp16 norm; per page K words [4][256][8 kBits], V words, K norms [4][256],
// V norms.
template <int kBits>
constexpr int tqb_row_bytes() { return 32 * kBits; }
template <int kBits>
constexpr int64_t tqb_page_bytes() { return int64_t(2) * kHkv * kPage * (tqb_row_bytes<kBits>() + 2); }
template <int kBits>
constexpr int64_t tqb_v_words() { return int64_t(kHkv) * kPage * tqb_row_bytes<kBits>(); }
template <int kBits>
constexpr int64_t tqb_k_norms() { return 2 * tqb_v_words<kBits>(); }
template <int kBits>
constexpr int64_t tqb_v_norms() { return tqb_k_norms<kBits>() + int64_t(kHkv) * kPage * 2; }
static_assert(tqb_page_bytes<2>() == TQ4_TQB2_PAGE_BYTES && tqb_page_bytes<3>() == TQ4_TQB3_PAGE_BYTES,
              "page sizes of the header");

// Widen 8 two-bit fields (bits 2i..2i+1 of x) to the low bits of 8 nibbles, and the
// 8 single bits of byte M of h (bit i) to bit 2 of 8 nibbles. A byte permute places the input
// bytes; each spreading step then ORs a shifted copy under a mask. Where a shifted
// copy cannot overlap the original, the step is a multiply (the sum equals the OR).
__device__ __forceinline__ uint32_t spread_fields2(uint32_t x) {   // bytes 0 and 2 hold 4 fields each
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  return (x | (x << 2)) & 0x33333333u;
}
__device__ __forceinline__ uint32_t widen2(uint32_t x) {      // fields of bits 0..15
  return spread_fields2(__byte_perm(x, 0u, 0x4140u));
}
__device__ __forceinline__ uint32_t widen2_hi(uint32_t x) {   // fields of bits 16..31
  return spread_fields2(__byte_perm(x, 0u, 0x4342u));
}
// byte M of h -> its bit pairs 2k, 2k + 1 at bits 8k, 8k + 1
template <int M>
__device__ __forceinline__ uint32_t spread_bits_pairs(uint32_t h) {
  uint32_t t = __byte_perm(h, 0u, 0x4440u | uint32_t(M));
  t = (t * 0x1001u) & 0x000F000Fu;   // bits 4..7 -> 16..19
  return (t * 0x41u) & 0x03030303u;  // bits 2..3 -> 8..9 (and 18..19 -> 24..25)
}
template <int M>
__device__ __forceinline__ uint32_t widen1_bit2(uint32_t h) { // byte M of h -> bit 2 of 8 nibbles
  return (spread_bits_pairs<M>(h) * 0x24u) & 0x44444444u;
}

constexpr float kLog2e = 1.4426950408889634f;

// With bf16 outputs the attention kernels skip the one product that a bf16 result
// cannot resolve: the centroid residual of the V side (C_lo P') on tiles whose V
// norms all stay at or below kVloNorm. The keys always take all three score terms
// and P' lo always enters. Norms 16 s with s in [0.5, 2] stay under ~34; the 8x
// outliers of the long-context workload start at 64. fp32 outputs run every product.
constexpr float kVloNorm = 48.0f;

// 16-byte global -> shared copies that bypass registers (generic proxy; wait before use)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Programmatic dependent launch. A kernel launched with launch_pdl may start
// while the previous kernel of its stream is still running; pdl_wait() blocks
// until that kernel has completed and its writes are visible, so every read of
// the call's inputs comes after it. pdl_launch_dependents() lets the next kernel
// of the stream be scheduled early. Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// mbarrier initialisation (shared::cta address)
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

// 2^x on the special-function unit (max relative error about 2^-22), used for
// softmax weights; -inf maps to +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Interleave the nibbles of two words: lo byte k = x_{2k} | y_{2k} << 4,
// hi byte k = x_{2k+1} | y_{2k+1} << 4 (x, y = words of two positions).
__device__ __forceinline__ void interleave_nibbles(uint32_t x, uint32_t y, uint32_t& lo, uint32_t& hi) {
  lo = (x & 0x0F0F0F0Fu) | ((y << 4) & 0xF0F0F0F0u);
  hi = ((x >> 4) & 0x0F0F0F0Fu) | (y & 0xF0F0F0F0u);
}

// --------------------------------------------------------------------------
// Warp-level tensor-core primitives (register operands).
// --------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ void stmatrix_x2_trans(uint32_t addr, uint32_t r0, uint32_t r1) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.trans.shared.b16 [%0], {%1,%2};\n" ::"r"(addr), "r"(r0),
               "r"(r1)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// read-only global loads
__device__ __forceinline__ uint4 ldg128(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ uint32_t ldg32(const void* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ float ldg_half(const void* p) {
  return __half2float(__ldg(reinterpret_cast<const __half*>(p)));
}

// Launch with programmatic stream serialisation (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace tq4
