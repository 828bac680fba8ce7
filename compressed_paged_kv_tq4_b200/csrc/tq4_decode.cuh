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
// split is split_len consecutive positions (split_len % 128 == 0). Requests that
// share their leading pages ([STATE] simpleprog.com "Fitting a 27B-Parameter LLM
// into 24 GiB of Laptop Memory", section "StateTrans": reference-counted shared
// prefixes) may be grouped: a group item covers a split of the group's shared
// positions and scores every member's query rows against it, so those pages are
// loaded and expanded once for the group (up to kShareNT n-tiles of rows); each
// member's own positions after the shared ones are ordinary items. Every item
// writes one partial record per request it serves. A CTA of 8 warps walks its
// split in chunks of 128 positions:
//   K phase  warp w takes positions 16w..16w+15 of the chunk: S = C_k . Q'^T
//            on mma.m16n8k16 (M = positions, N = 6 query heads x n_q tokens,
//            K = dims), nibble pairs decoded through a per-lane smem table.
//   softmax  chunk max exchanged through smem; p = exp(s - m), P' = p * n_v
//            written transposed to smem as an f16 hi + lo pair.
//   V phase  warp w takes dims 64w..64w+63 of all 64 positions:
//            O'^T += C_v^T . P'^T (M = dims, N = query rows, K = positions).
// Per-split partial results (m, l, o') go to the workspace; the combine pass
// merges them (log-sum-exp), rotates back and writes bf16/fp32.
#pragma once
#include <type_traits>

#include "tq4_device.cuh"

namespace tq4 {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kChunk = 16 * kDecWarps;       // positions per chunk (half a page)
constexpr int kStages = 3;                   // cp.async ring depth
constexpr int kQvStride = kD + 8;            // halves per Q' row in smem (bank-conflict pad)
constexpr int kPsStride = kChunk + 8;        // halves per P' row in smem
constexpr int kStageBytes = 2 * kChunk * 128 + 2 * kChunk * 2;   // K words, V words, K norms, V norms

// Uniform INT8 comparison arm: a page holds 256 positions of one layer as
// K codes [4 heads][256 slots][256 int8], V codes, K scales [4][256] fp16, V scales.
constexpr int64_t kI8PageBytes = TQ4_INT8_PAGE_BYTES;   // 528,384
constexpr int64_t kI8KCodes = 0;
constexpr int64_t kI8VCodes = int64_t(kHkv) * kPage * kD;          // 262,144
constexpr int64_t kI8KScales = 2 * kI8VCodes;                       // 524,288
constexpr int64_t kI8VScales = kI8KScales + int64_t(kHkv) * kPage * 2;   // 526,336
constexpr int kI8Stages = 2;
constexpr int kI8StageBytes = 2 * kChunk * 256 + 2 * kChunk * 2;   // K codes, V codes, K scales, V scales

// Shared-prefix groups (the one-launch dedup of shared pages). Items
// [0, n_gitems) are group items, item0[g] .. item0[g + 1] - 1 those of group g,
// each over share.split_len shared positions (shorter than a private item's:
// it scores more query rows); the rest are the requests' private items. A
// request's records are consecutive: first ceil(pos / share.split_len) for the
// shared positions of its group (if any), then one per split of its own positions.
constexpr int kMaxShareGroups = 32;
constexpr int kMaxShareMembers = 8;
constexpr int kShareNT = 6;   // a group item's n-tiles: up to 48 query rows
struct SharePlan {
  int32_t n_groups;
  int32_t n_gitems;
  int32_t split_len;                                   // positions per group item
  int32_t item0[kMaxShareGroups + 1];
  int32_t pos[kMaxShareGroups];                        // shared positions (whole pages)
  int32_t n_mem[kMaxShareGroups];
  int32_t mem[kMaxShareGroups][kMaxShareMembers];      // member request ids, ascending
};

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
  int32_t items_ub;    // grid size (items)
  int32_t records_ub;  // partial records the workspace holds
  int32_t rows_pad;    // 8 * NT (one request's query rows, padded)
  float* ws_o;         // [records][4][rows_pad][256]
  float2* ws_ml;       // [records][4][rows_pad] (m, l)
  void* out;
  int out_dtype;
  Signs signs;
  int* status;
  // fused append (n_q == 1): the new position of each request, [n_req][4][256] of
  // new_dtype, is encoded into pool_w at position seq_len - 1 before it is attended;
  // pool_w == nullptr means the positions are already in the pool
  uint8_t* pool_w;
  const void* k_new;
  const void* v_new;
  int new_dtype;
  uint32_t spin_limit;   // polls before a bounded wait gives up (TQ4_ERR_TIMEOUT)
  int test_withhold;     // test hook: withhold the first tile copy of each warp (its wait runs out)
  int rotate;            // 1: o = R^T o' (TQ4, rotated domain); 0: o = o' (the INT8 arm)
  SharePlan share;       // n_groups == 0: no shared-prefix groups
};

__host__ __device__ constexpr int decode_nt(int n_q) { return (6 * n_q + 7) / 8; }

// ring stages: three, two for the wide group items (shared memory)
template <int NT, bool kI8>
constexpr int decode_stages() { return kI8 ? kI8Stages : (NT >= 4 ? 2 : kStages); }
// 2- and 3-bit pools: a chunk's rows are staged as they are in the page (K and V
// packed words, then K and V norms) and widened to the four-bit stage layout in
// one work stage
template <int kBits>
constexpr size_t tqb_raw_stage_bytes() { return size_t(2) * kChunk * tqb_row_bytes<kBits>() + size_t(2) * kChunk * 2; }
template <int NT, bool kI8, int kBits>
constexpr size_t decode_ring_bytes() {
  return kBits != 4 ? size_t(decode_stages<NT, kI8>()) * tqb_raw_stage_bytes<kBits>() + kStageBytes
                    : size_t(decode_stages<NT, kI8>()) * (kI8 ? kI8StageBytes : kStageBytes);
}
template <int NT, bool kI8, int kBits = 4>
constexpr size_t decode_item_smem_bytes() {
  return (kI8 ? 0 : size_t(kLutBytes)) + decode_ring_bytes<NT, kI8, kBits>() +
         2 * size_t(8 * NT) * kQvStride * 2 + 2 * size_t(8 * NT) * kPsStride * 2 + size_t(kDecWarps) * 8 * NT * 4;
}
template <int NT, int NTG, bool kI8>
constexpr size_t decode_smem_bytes() {
  return decode_item_smem_bytes<NT, kI8>() > decode_item_smem_bytes<NTG, kI8>() ? decode_item_smem_bytes<NT, kI8>()
                                                                                : decode_item_smem_bytes<NTG, kI8>();
}
static_assert(decode_item_smem_bytes<kShareNT, false>() <= 227u * 1024u, "group items fit shared memory");
static_assert(decode_item_smem_bytes<3, false, 3>() <= 227u * 1024u, "3-bit items fit shared memory");
static_assert(decode_item_smem_bytes<kShareNT, false, 3>() <= 227u * 1024u, "3-bit group items fit shared memory");

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

// Shared positions of request r (those of its group; 0 if it is in none).
__device__ __forceinline__ int shared_pos(const DecodeParams& p, int r) {
  for (int g = 0; g < p.share.n_groups; ++g)
    for (int k = 0; k < p.share.n_mem[g]; ++k)
      if (p.share.mem[g][k] == r) return p.share.pos[g];
  return 0;
}
// Records of request r: its group's shared splits, then its own splits (none if
// its length is inconsistent, which the kernels report).
__device__ __forceinline__ void request_records(const DecodeParams& p, int r, int s_len, int& n_shared,
                                                int& n_own) {
  const int P = shared_pos(p, r);
  n_shared = P > 0 ? (P + p.share.split_len - 1) / p.share.split_len : 0;
  n_own = seq_ok(s_len, p.n_q, p.max_pages) ? (max(s_len - P, 0) + p.split_len - 1) / p.split_len : 0;
}

// Warp-collective: find (request, split) of private item x (counted after the
// group items). Returns false if x is not an item. *total receives the number of
// private items.
__device__ __forceinline__ bool find_item(const DecodeParams& p, int x, int& req, int& split,
                                          int& total) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  bool found = false;
  for (int r0 = 0; r0 < p.n_req; r0 += 32) {
    const int r = r0 + lane;
    int S = 0;
    if (r < p.n_req) {
      int nsh = 0;
      request_records(p, r, __ldg(p.seq_lens + r), nsh, S);
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

// Warp-collective: the first record of request r (the records of requests 0..r-1).
__device__ __forceinline__ int request_first_record(const DecodeParams& p, int r) {
  const int lane = threadIdx.x & 31;
  int first = 0;
  for (int r0 = 0; r0 < r; r0 += 32) {
    const int rr = r0 + lane;
    int n = 0;
    if (rr < r) {
      int nsh = 0, own = 0;
      request_records(p, rr, __ldg(p.seq_lens + rr), nsh, own);
      n = nsh + own;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    first += n;
  }
  return first;
}

__device__ __forceinline__ uint32_t pick(const uint4& a, const uint4& b, int i) {
  switch (i) {
    case 0: return a.x; case 1: return a.y; case 2: return a.z; case 3: return a.w;
    case 4: return b.x; case 5: return b.y; case 6: return b.z; default: return b.w;
  }
}

// 16-byte segment swizzle inside a staged 128-byte word row: the K phase
// (segments t and 4+t of positions g, g+8 per quarter warp) and the V phase
// (one word of positions 2t / 2t+1 per lane group) both hit 32 distinct banks.
__device__ __forceinline__ int seg_swz(int pos) { return (((pos >> 1) & 3) << 1) ^ ((pos & 1) << 2); }


// INT8 rows are 256 B (16 segments of 16 B). The swizzle makes both the K phase
// (segments 4m + t of positions g, g + 1 per quarter warp) and the V phase (8-byte
// pieces of one segment pair from positions 2t, t = 0..3, per half warp) hit
// distinct banks.
__device__ __forceinline__ int i8_swz(int pos) { return (((pos >> 1) & 3) << 1) ^ ((pos & 1) << 2); }

// int8 codes in bits 0-7 and 16-23 of t (the rest ignored) -> f16x2 holding them
// exactly: the code plus 128 (its sign bit flipped) sits in the mantissa of 1024
// (f16 0x6400), and 1152 is subtracted
__device__ __forceinline__ uint32_t i8_pair_bytes(uint32_t t) {
  uint32_t u;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;\n" : "=r"(u) : "r"(t), "r"(0x00FF00FFu), "r"(0x64806480u));   // (a & b) ^ c
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&u), __floats2half2_rn(1152.f, 1152.f));
  return *reinterpret_cast<const uint32_t*>(&h);
}
// int8 codes in bytes B0, B1 of w -> exact f16x2 (byte B0 in the low half)
template <int B0, int B1>
__device__ __forceinline__ uint32_t i8_pair(uint32_t w) {
  return i8_pair_bytes(__byte_perm(w, 0u, uint32_t(B0) | (4u << 4) | (uint32_t(B1) << 8) | (4u << 12)));
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// An item's description in shared memory (written by warp 0 of the CTA)
constexpr int kItPosB = 0, kItPosE = 1, kItTable = 2, kItNMem = 3, kItReq = 4,
              kItRec = kItReq + kMaxShareMembers, kItWords = kItRec + kMaxShareMembers;

// One item: positions [pos_b, pos_e) of the pages in request item[kItTable]'s
// table, scored against the query rows of item[kItNMem] requests (request
// item[kItReq + k], partial record item[kItRec + k]); NT n-tiles hold their
// n_mem * 6 * n_q rows (member-major, then token, then head).
// kExact: fp32 outputs, C_lo P' on every chunk (see kVloNorm). kBits: 4 (TQ4), or 2
// or 3 for the narrower variants, whose codes are widened to nibbles per chunk.
template <int NT, bool kI8, bool kExact, int kBits = 4>
__device__ __forceinline__ void decode_item(const DecodeParams& p, uint8_t* smem, const int* item) {
  static_assert(kBits == 4 || (!kI8 && (kBits == 2 || kBits == 3)), "bit width");
  constexpr bool kTQB = kBits != 4;
  constexpr int kRB = kI8 ? 256 : 128;                 // bytes of one staged K or V row
  constexpr int kNS = decode_stages<NT, kI8>();        // ring stages; chunks prefetched kNS - 1 ahead
  constexpr int kSB = kTQB ? int(tqb_raw_stage_bytes<kBits>()) : (kI8 ? kI8StageBytes : kStageBytes);
  const uint32_t lut = smem_u32(smem);                 // the centroid table (TQ4 only)
  uint8_t* ring = smem + (kI8 ? 0 : kLutBytes);
  uint8_t* work = ring + kNS * kSB;                    // the widened chunk (2- and 3-bit pools)
  __half* qv_hi = reinterpret_cast<__half*>(smem + (kI8 ? 0 : kLutBytes) + decode_ring_bytes<NT, kI8, kBits>());
  __half* qv_lo = qv_hi + 8 * NT * kQvStride;
  __half* ps_hi = qv_lo + 8 * NT * kQvStride;
  __half* ps_lo = ps_hi + 8 * NT * kPsStride;   // P' = hi + lo, both f16
  float* red = reinterpret_cast<float*>(ps_lo + 8 * NT * kPsStride);   // [warps][8*NT]

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const uint32_t lane8 = uint32_t(lane) * 8u;

  const int pos_b = item[kItPosB], pos_e = item[kItPosE];
  const int n_chunks = (pos_e - pos_b + kChunk - 1) / kChunk;
  const int NR = 6 * p.n_q;                 // query rows of one request
  const int NRT = item[kItNMem] * NR;       // query rows of the item
  const int32_t* table = p.page_tables + int64_t(item[kItTable]) * p.max_pages;
  const int64_t head_slot0 = int64_t(h) * kPage;

  // ---- staging: chunk i -> ring stage i % kStages (all threads issue 16-byte copies)
  auto issue_chunk = [&](int i) {
    if (i < n_chunks) {
      const int c = pos_b + i * kChunk;
      const int32_t page = __ldg(table + (c >> 8));
      if (page < 0 || page >= p.num_pages) {
        if (tid == 0) record_error(p.status, TQ4_ERR_PAGE_RANGE);
      } else if constexpr (kTQB) {
        constexpr int kRBb = tqb_row_bytes<kBits>(), kSegB = kRBb / 16;
        const uint8_t* pg = p.pool + int64_t(page) * tqb_page_bytes<kBits>();
        const int64_t slot0 = head_slot0 + (c & (kPage - 1));
        uint8_t* st = ring + (i % kNS) * kSB;
        const int nvalid = min(kChunk, pos_e - c);
        for (int e = tid; e < 2 * kChunk * kSegB; e += kDecThreads) {
          const int kv = e / (kChunk * kSegB), pl = (e / kSegB) % kChunk, sg = e % kSegB;
          if (pl < nvalid)
            cp_async16(smem_u32(st + (kv * kChunk + pl) * kRBb + sg * 16),
                       pg + (kv ? tqb_v_words<kBits>() : 0) + (slot0 + pl) * kRBb + sg * 16);
        }
        if (tid < 2 * (kChunk / 8)) {
          const int kv = tid / (kChunk / 8), sg = tid % (kChunk / 8);
          if (sg * 8 < nvalid)
            cp_async16(smem_u32(st + 2 * kChunk * kRBb + kv * kChunk * 2 + sg * 16),
                       pg + (kv ? tqb_v_norms<kBits>() : tqb_k_norms<kBits>()) + (slot0 + sg * 8) * 2);
        }
      } else {
        constexpr int64_t kPB = kI8 ? kI8PageBytes : kPageBytes;
        constexpr int64_t kKR = kI8 ? kI8KCodes : kKWords, kVR = kI8 ? kI8VCodes : kVWords;
        constexpr int64_t kKN = kI8 ? kI8KScales : kKNorms, kVN = kI8 ? kI8VScales : kVNorms;
        constexpr int kSeg = kRB / 16;   // 16-byte segments per row
        const uint8_t* pg = p.pool + int64_t(page) * kPB;
        const int64_t slot0 = head_slot0 + (c & (kPage - 1));
        uint8_t* st = ring + (i % kNS) * kSB;
        const int nvalid = min(kChunk, pos_e - c);
        // K and V rows: 2 x kChunk positions x kSeg segments
        for (int e = tid; e < 2 * kChunk * kSeg; e += kDecThreads) {
          const int kv = e / (kChunk * kSeg), pl = (e / kSeg) % kChunk, sg = e % kSeg;
          if (pl < nvalid) {
            const uint8_t* src = pg + (kv ? kVR : kKR) + (slot0 + pl) * kRB + sg * 16;
            const int sw = kI8 ? i8_swz(pl) : seg_swz(pl);
            cp_async16(smem_u32(st + kv * kChunk * kRB + pl * kRB + ((sg ^ sw) << 4)), src);
          }
        }
        // norms (scales): 2 x kChunk halves = 2 x (kChunk / 8) segments
        if (tid < 2 * (kChunk / 8)) {
          const int kv = tid / (kChunk / 8), sg = tid % (kChunk / 8);
          if (sg * 8 < nvalid) {
            const uint8_t* src = pg + (kv ? kVN : kKN) + (slot0 + sg * 8) * 2;
            cp_async16(smem_u32(st + 2 * kChunk * kRB + kv * kChunk * 2 + sg * 16), src);
          }
        }
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kNS - 1; ++i) issue_chunk(i);

  // ---- the queries of this (request, KV head): q' = R q * scale (TQ4) or q * scale
  // (INT8), split hi + lo f16, stored in the K phase's virtual dim order
  for (int row = w; row < 8 * NT; row += kDecWarps) {
    float v[8];
    if (row < NRT) {
      const int rq = item[kItReq + row / NR], tok = (row % NR) / 6, j = row % 6;
      const uint16_t* src = p.q + ((int64_t(rq) * p.n_q + tok) * kHq + h * kGroup + j) * kD + lane * 8;
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
      const uint32_t ww[4] = {raw.x, raw.y, raw.z, raw.w};
      if constexpr (kI8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = __uint_as_float(ww[i] << 16) * p.scale;
          v[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u) * p.scale;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = __uint_as_float(ww[i] << 16) * sign_of(p.signs, lane * 8 + 2 * i);
          v[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u) * sign_of(p.signs, lane * 8 + 2 * i + 1);
        }
        warp_fwht256(v);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= p.scale * 0.0625f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    // lane owns real dims 8*lane + i (word lane). Word lane is read in the K phase by
    // thread t = (lane & 15) >> 2 as its word index ws = (lane & 3) + 4*(lane >> 4);
    // k-step kk = 2*ws + (i >> 2), mma column 2t + (i & 1) + 8*((i >> 1) & 1).
    // INT8: dim d = 8 lane + i is read in the K phase by thread t = (d >> 4) & 3 from
    // its 16-byte segment 4m + t (m = d >> 6) as byte (d & 3) of word j = (d >> 2) & 3:
    // k-step kk = 4m + j, mma column 2t + (d & 1) + 8 ((d >> 1) & 1).
    const int tt = (lane & 15) >> 2, wsel = (lane & 3) + 4 * (lane >> 4);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int kk = kI8 ? 4 * (lane >> 3) + ((2 * lane + (i >> 2)) & 3) : 2 * wsel + (i >> 2);
      const int col = kI8 ? kk * 16 + 2 * ((lane >> 1) & 3) + 8 * ((i >> 1) & 1)
                          : kk * 16 + ((i >> 1) & 1) * 8 + 2 * tt;
      const __half2 hi = __floats2half2_rn(v[i], v[i + 1]);
      const float2 hf = __half22float2(hi);
      *reinterpret_cast<__half2*>(qv_hi + row * kQvStride + col) = hi;
      *reinterpret_cast<__half2*>(qv_lo + row * kQvStride + col) = __floats2half2_rn(v[i] - hf.x, v[i + 1] - hf.y);
    }
  }
  // centroid table: row b holds each lane's 8-byte slot {c16 pair, r16 pair} at +8*lane
  if constexpr (!kI8)
    for (int e = tid; e < 256 * 32; e += kDecThreads)
      reinterpret_cast<uint2*>(smem)[e] = kTQB ? lut_row_bits<kBits>(e >> 5) : lut_row(e >> 5);
  __syncthreads();

  // ---- B fragments of Q' (hi, lo) for the K phase, in registers when they fit
  constexpr bool kQReg = (NT == 1);
  uint32_t qh[kQReg ? 16 : 1][2], ql[kQReg ? 16 : 1][2];
  if constexpr (kQReg) {
#pragma unroll
    for (int kk = 0; kk < 16; kk += 2) {
      const int m = lane >> 3;
      const int off = (lane & 7) * kQvStride + (kk + (m >> 1)) * 16 + (m & 1) * 8;
      ldmatrix_x4(qh[kk][0], qh[kk][1], qh[kk + 1][0], qh[kk + 1][1], smem_u32(qv_hi + off));
      ldmatrix_x4(ql[kk][0], ql[kk][1], ql[kk + 1][0], ql[kk + 1][1], smem_u32(qv_lo + off));
    }
  }

  // per-row visibility limits for the rows this thread scores (rows nt*8 + 2t + e):
  // token tok of request rq sees positions [0, seq_len(rq) - n_q + tok]
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = nt * 8 + 2 * t + e;
      lim[nt][e] = row < NRT ? __ldg(p.seq_lens + item[kItReq + row / NR]) - p.n_q + (row % NR) / 6 + 1 : 0;
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
  const int dg = w & 3, ph = w >> 2;   // V phase: 64-dim group, 64-position half

  for (int i = 0; i < n_chunks; ++i) {
    cp_async_wait<kNS - 2>();
    __syncthreads();            // chunk i visible to all; everyone is done with chunk i-1
    issue_chunk(i + kNS - 1);
    const int c = pos_b + i * kChunk;
    const uint8_t* st = ring + (i % kNS) * kSB;
    if constexpr (kTQB) {
      // widen the staged chunk into the four-bit layout: thread -> (K or V, position,
      // 16-byte segment of four nibble words = dims 32 sg .. 32 sg + 31)
      constexpr int kRBb = tqb_row_bytes<kBits>();
      for (int e = tid; e < 2 * kChunk * 8; e += kDecThreads) {
        const int kv = e / (kChunk * 8), pl = (e >> 3) % kChunk, sg = e & 7;
        const uint8_t* r = st + (kv * kChunk + pl) * kRBb;
        const uint2 lo = lds64(r + sg * 8);                    // plane 0: words 2 sg, 2 sg + 1
        const uint32_t hb = kBits == 3 ? lds32(r + 64 + sg * 4) : 0u;   // plane 1: word sg
        uint4 o;
        o.x = widen2(lo.x) | widen1_bit2<0>(hb);
        o.y = widen2_hi(lo.x) | widen1_bit2<1>(hb);
        o.z = widen2(lo.y) | widen1_bit2<2>(hb);
        o.w = widen2_hi(lo.y) | widen1_bit2<3>(hb);
        *reinterpret_cast<uint4*>(work + (kv * kChunk + pl) * 128 + ((sg ^ seg_swz(pl)) << 4)) = o;
      }
      if (tid < 2 * kChunk * 2 / 16)   // the norms, unchanged
        reinterpret_cast<uint4*>(work + 2 * kChunk * 128)[tid] =
            reinterpret_cast<const uint4*>(st + 2 * kChunk * kRBb)[tid];
      __syncthreads();
      st = work;
    }
    const uint8_t* kst = st;
    const uint8_t* vst = st + kChunk * kRB;
    const __half* knr = reinterpret_cast<const __half*>(st + 2 * kChunk * kRB);
    const __half* vnr = knr + kChunk;

    // ---------------------------------------------------------- K phase: S = C_k Q'^T (fp32-grade)
    const int pg0 = 16 * w + g;   // chunk-local positions pg0, pg0 + 8
    // scores = (C_hi + C_lo)(q'_hi + q'_lo) to fp32 precision: C_hi q'_hi + [C_hi q'_lo + C_lo q'_hi]
    // (the two small terms share one accumulator; C_lo q'_lo is below fp32 resolution);
    // INT8 codes are exact f16 values, so there C_lo = 0. Even/odd k-steps use
    // separate accumulators to halve the dependent mma chains.
    constexpr int kAcc = NT >= 4 ? 1 : 2;   // wide items have NT independent chains already
    float shh[kAcc][NT][4], sx[kAcc][NT][4];
#pragma unroll
    for (int a = 0; a < kAcc; ++a)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) shh[a][nt][j] = sx[a][nt][j] = 0.f;
    // B fragments of q' hi / lo for k-step kk and n-tile nt
    auto qfrag = [&](int kk, int nt, uint32_t& bh0, uint32_t& bh1, uint32_t& bl0, uint32_t& bl1) {
      if constexpr (kQReg) {
        bh0 = qh[kk][0]; bh1 = qh[kk][1]; bl0 = ql[kk][0]; bl1 = ql[kk][1];
      } else {
        const int m = (lane >> 3) & 1;
        const int off = (nt * 8 + (lane & 7)) * kQvStride + kk * 16 + m * 8;
        ldmatrix_x2(bh0, bh1, smem_u32(qv_hi + off));
        ldmatrix_x2(bl0, bl1, smem_u32(qv_lo + off));
      }
    };
    if constexpr (kI8) {
      const int sz = i8_swz(pg0);   // same for pg0 + 8
#pragma unroll
      for (int m = 0; m < 4; ++m) {   // k-steps 4m .. 4m + 3: one 16-byte segment per position
        const uint4 ka = lds128(kst + pg0 * 256 + (((4 * m + t) ^ sz) << 4));
        const uint4 kb = lds128(kst + (pg0 + 8) * 256 + (((4 * m + t) ^ sz) << 4));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kk = 4 * m + j;
          const uint32_t wa = pick(ka, ka, j), wb = pick(kb, kb, j);
          const uint32_t a0 = i8_pair<0, 1>(wa), a1 = i8_pair<0, 1>(wb);
          const uint32_t a2 = i8_pair<2, 3>(wa), a3 = i8_pair<2, 3>(wb);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            uint32_t bh0, bh1, bl0, bl1;
            qfrag(kk, nt, bh0, bh1, bl0, bl1);
            mma_16816(shh[kk % kAcc][nt], a0, a1, a2, a3, bh0, bh1);
            mma_16816(sx[kk % kAcc][nt], a0, a1, a2, a3, bl0, bl1);
          }
        }
      }
    } else {
    const int sz = seg_swz(pg0);  // same for pg0 + 8
    const uint4 ka0 = lds128(kst + pg0 * 128 + ((t ^ sz) << 4));
    const uint4 ka1 = lds128(kst + pg0 * 128 + (((4 + t) ^ sz) << 4));
    const uint4 kb0 = lds128(kst + (pg0 + 8) * 128 + ((t ^ sz) << 4));
    const uint4 kb1 = lds128(kst + (pg0 + 8) * 128 + (((4 + t) ^ sz) << 4));
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const uint32_t wg = pick(ka0, ka1, kk >> 1);
      const uint32_t wg8 = pick(kb0, kb1, kk >> 1);
      uint32_t a0, a1, a2, a3, r0, r1, r2, r3;
      if (kk & 1) {
        lut_decode<2>(lut, wg, lane8, a0, r0);
        lut_decode<2>(lut, wg8, lane8, a1, r1);
        lut_decode<3>(lut, wg, lane8, a2, r2);
        lut_decode<3>(lut, wg8, lane8, a3, r3);
      } else {
        lut_decode<0>(lut, wg, lane8, a0, r0);
        lut_decode<0>(lut, wg8, lane8, a1, r1);
        lut_decode<1>(lut, wg, lane8, a2, r2);
        lut_decode<1>(lut, wg8, lane8, a3, r3);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t bh0, bh1, bl0, bl1;
        qfrag(kk, nt, bh0, bh1, bl0, bl1);
        mma_16816(shh[kk % kAcc][nt], a0, a1, a2, a3, bh0, bh1);
        mma_16816(sx[kk % kAcc][nt], a0, a1, a2, a3, bl0, bl1);
        mma_16816(sx[kk % kAcc][nt], r0, r1, r2, r3, bh0, bh1);
      }
    }
    }

    // ---------------------------------------------------------- online softmax over the chunk
    const float kn0 = __half2float(knr[pg0]), kn8 = __half2float(knr[pg0 + 8]);
    const float vn0 = __half2float(vnr[pg0]), vn8 = __half2float(vnr[pg0 + 8]);
    const int pos0 = c + pg0;
    const bool vbig = (pos0 < pos_e && vn0 > kVloNorm) || (pos0 + 8 < pos_e && vn8 > kVloNorm);
    float s[NT][4], mx[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pos = pos0 + 8 * (j >> 1);
        const bool ok = pos < pos_e && pos < lim[nt][j & 1];
        const float acc = kAcc == 2 ? (shh[0][nt][j] + shh[kAcc - 1][nt][j]) + (sx[0][nt][j] + sx[kAcc - 1][nt][j])
                                    : shh[0][nt][j] + sx[0][nt][j];
        s[nt][j] = ok ? acc * ((j >> 1) ? kn8 : kn0) : -INFINITY;
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
        alpha[nt][e] = fast_exp2((m_run[nt][e] - m_use) * kLog2e);
        m_run[nt][e] = m_new;
        mx[nt][e] = m_use;
      }
      float pr[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) pr[j] = fast_exp2((s[nt][j] - mx[nt][j & 1]) * kLog2e);
      l_part[nt][0] = l_part[nt][0] * alpha[nt][0] + pr[0] + pr[2];
      l_part[nt][1] = l_part[nt][1] * alpha[nt][1] + pr[1] + pr[3];
      // P' = p * n_v (zero where masked, so stale norms never enter)
      const float w0 = s[nt][0] == -INFINITY ? 0.f : pr[0] * vn0;
      const float w1 = s[nt][1] == -INFINITY ? 0.f : pr[1] * vn0;
      const float w2 = s[nt][2] == -INFINITY ? 0.f : pr[2] * vn8;
      const float w3 = s[nt][3] == -INFINITY ? 0.f : pr[3] * vn8;
      const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
      const int jr = lane & 7, mat = (lane >> 3) & 1;
      const int poff = (nt * 8 + jr) * kPsStride + 16 * w + 8 * mat;
      stmatrix_x2_trans(smem_u32(ps_hi + poff), *reinterpret_cast<const uint32_t*>(&h01),
                        *reinterpret_cast<const uint32_t*>(&h23));
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(w0 - f01.x, w1 - f01.y);
      const __half2 l23 = __floats2half2_rn(w2 - f23.x, w3 - f23.y);
      stmatrix_x2_trans(smem_u32(ps_lo + poff), *reinterpret_cast<const uint32_t*>(&l01),
                        *reinterpret_cast<const uint32_t*>(&l23));
    }
    // P' is complete; the chunk takes the C_lo P' products when one of its visible
    // V norms is large (or the output is fp32)
    const bool vlo = __syncthreads_or(vbig) != 0 || kExact;

    // ---------------------------------------------------------- V phase: O'^T += C_v^T P'^T
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        o[nt][mt][0] *= alpha[nt][0];
        o[nt][mt][1] *= alpha[nt][1];
        o[nt][mt][2] *= alpha[nt][0];
        o[nt][mt][3] *= alpha[nt][1];
      }
    if constexpr (kI8) {
      // lane (g, t): 8 codes (dims 64 dg + 8 g .. + 7) of positions 2t, 2t+1, 2t+8, 2t+9
      // of each k-step; m-tile mt's rows g, g + 8 are dims 64 dg + 8 g + 2 mt, + 1
      const int seg = 4 * dg + (g >> 1), off8 = (g & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int pb = 64 * ph + 16 * ks + 2 * t;
        const uint2 x0 = lds64(vst + pb * 256 + ((seg ^ i8_swz(pb)) << 4) + off8);
        const uint2 x1 = lds64(vst + (pb + 1) * 256 + ((seg ^ i8_swz(pb + 1)) << 4) + off8);
        const uint2 y0 = lds64(vst + (pb + 8) * 256 + ((seg ^ i8_swz(pb + 8)) << 4) + off8);
        const uint2 y1 = lds64(vst + (pb + 9) * 256 + ((seg ^ i8_swz(pb + 9)) << 4) + off8);
        uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int m = (lane >> 3) & 1;
          const int off = (nt * 8 + (lane & 7)) * kPsStride + 64 * ph + 16 * ks + 8 * m;
          ldmatrix_x2(bh[nt][0], bh[nt][1], smem_u32(ps_hi + off));
          ldmatrix_x2(bl[nt][0], bl[nt][1], smem_u32(ps_lo + off));
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const uint32_t xa = mt < 2 ? x0.x : x0.y, xb = mt < 2 ? x1.x : x1.y;
          const uint32_t ya = mt < 2 ? y0.x : y0.y, yb = mt < 2 ? y1.x : y1.y;
          constexpr uint32_t kS0 = 0x0400u, kS1 = 0x0501u, kS2 = 0x0602u, kS3 = 0x0703u;   // byte b of a, byte b of b
          const uint32_t s0 = (mt & 1) ? kS2 : kS0, s1 = (mt & 1) ? kS3 : kS1;
          const uint32_t a0 = i8_pair_bytes(__byte_perm(xa, xb, s0)), a1 = i8_pair_bytes(__byte_perm(xa, xb, s1));
          const uint32_t a2 = i8_pair_bytes(__byte_perm(ya, yb, s0)), a3 = i8_pair_bytes(__byte_perm(ya, yb, s1));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816(o[nt][mt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
            mma_16816(o[nt][mt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
          }
        }
      }
      continue;
    }
    (void)vlo;
    const int wd = 8 * dg + g;                       // the word (8 dims) this lane decodes
    const int wseg = wd >> 2, wofs = (wd & 3) * 4;   // its 16-byte segment and offset
    auto v_phase = [&](auto lo_tag) {
    constexpr bool kLo = decltype(lo_tag)::value;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int pb = 64 * ph + 16 * ks + 2 * t;
      const uint32_t x0 = lds32(vst + pb * 128 + ((wseg ^ seg_swz(pb)) << 4) + wofs);
      const uint32_t x1 = lds32(vst + (pb + 1) * 128 + ((wseg ^ seg_swz(pb + 1)) << 4) + wofs);
      const uint32_t y0 = lds32(vst + (pb + 8) * 128 + ((wseg ^ seg_swz(pb + 8)) << 4) + wofs);
      const uint32_t y1 = lds32(vst + (pb + 9) * 128 + ((wseg ^ seg_swz(pb + 9)) << 4) + wofs);
      uint32_t lo01, hi01, lo89, hi89;
      interleave_nibbles(x0, x1, lo01, hi01);
      interleave_nibbles(y0, y1, lo89, hi89);
      uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = (lane >> 3) & 1;
        const int off = (nt * 8 + (lane & 7)) * kPsStride + 64 * ph + 16 * ks + 8 * m;
        ldmatrix_x2(bh[nt][0], bh[nt][1], smem_u32(ps_hi + off));
        ldmatrix_x2(bl[nt][0], bl[nt][1], smem_u32(ps_lo + off));
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t a0, a1, a2, a3, r0, r1, r2, r3;
        switch (mt) {
          case 0:
            lut_decode<0>(lut, lo01, lane8, a0, r0); lut_decode<0>(lut, hi01, lane8, a1, r1);
            lut_decode<0>(lut, lo89, lane8, a2, r2); lut_decode<0>(lut, hi89, lane8, a3, r3);
            break;
          case 1:
            lut_decode<1>(lut, lo01, lane8, a0, r0); lut_decode<1>(lut, hi01, lane8, a1, r1);
            lut_decode<1>(lut, lo89, lane8, a2, r2); lut_decode<1>(lut, hi89, lane8, a3, r3);
            break;
          case 2:
            lut_decode<2>(lut, lo01, lane8, a0, r0); lut_decode<2>(lut, hi01, lane8, a1, r1);
            lut_decode<2>(lut, lo89, lane8, a2, r2); lut_decode<2>(lut, hi89, lane8, a3, r3);
            break;
          default:
            lut_decode<3>(lut, lo01, lane8, a0, r0); lut_decode<3>(lut, hi01, lane8, a1, r1);
            lut_decode<3>(lut, lo89, lane8, a2, r2); lut_decode<3>(lut, hi89, lane8, a3, r3);
            break;
        }
        // O'^T += (C_hi + C_lo)^T (P'_hi + P'_lo), less the C_lo P'_lo term (and, with bf16
        // outputs, less C_lo where the chunk's V norms are all small)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816(o[nt][mt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
          mma_16816(o[nt][mt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
          if constexpr (kLo) mma_16816(o[nt][mt], r0, r1, r2, r3, bh[nt][0], bh[nt][1]);
        }
      }
    }
    };
    if (vlo) v_phase(std::true_type{});
    else v_phase(std::false_type{});
  }
  cp_async_wait<0>();

  // ---------------------------------------------------------------- partial results
  // l: over the lanes sharing t and over the 8 warps' K phases; o': over the two position halves
  __syncthreads();
  float* ohalf = reinterpret_cast<float*>(ring);   // [4 dim groups][8*NT rows][64 dims] from warps 4..7
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = l_part[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      if (g == 0) red[w * 8 * NT + nt * 8 + 2 * t + e] = v;
      if (ph == 1) {
        const int row = nt * 8 + 2 * t + e;
        float* d = ohalf + (dg * 8 * NT + row) * 64 + 8 * g;
        reinterpret_cast<float4*>(d)[0] = make_float4(o[nt][0][e], o[nt][0][e + 2], o[nt][1][e], o[nt][1][e + 2]);
        reinterpret_cast<float4*>(d)[1] = make_float4(o[nt][2][e], o[nt][2][e + 2], o[nt][3][e], o[nt][3][e + 2]);
      }
    }
  __syncthreads();
  // row -> its request's record: (record * 4 + h) * rows_pad + row within the request
  auto rec_row = [&](int row) {
    return (int64_t(item[kItRec + row / NR]) * kHkv + h) * p.rows_pad + row % NR;
  };
  if (ph == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = nt * 8 + 2 * t + e;
        if (row >= NRT) continue;
        const float* sidx = ohalf + (dg * 8 * NT + row) * 64 + 8 * g;
        const float4 u0 = reinterpret_cast<const float4*>(sidx)[0];
        const float4 u1 = reinterpret_cast<const float4*>(sidx)[1];
        float* dst = p.ws_o + rec_row(row) * kD + 64 * dg + 8 * g;
        reinterpret_cast<float4*>(dst)[0] = make_float4(o[nt][0][e] + u0.x, o[nt][0][e + 2] + u0.y,
                                                        o[nt][1][e] + u0.z, o[nt][1][e + 2] + u0.w);
        reinterpret_cast<float4*>(dst)[1] = make_float4(o[nt][2][e] + u1.x, o[nt][2][e + 2] + u1.y,
                                                        o[nt][3][e] + u1.z, o[nt][3][e + 2] + u1.w);
      }
  }
  if (w == 0 && g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = nt * 8 + 2 * t + e;
        if (row >= NRT) continue;
        float l = 0.f;
#pragma unroll
        for (int ww = 0; ww < kDecWarps; ++ww) l += red[ww * 8 * NT + row];
        p.ws_ml[rec_row(row)] = make_float2(m_run[nt][e], l);
      }
  }
}

// Warp-collective (one warp; lane 0 writes): the description of private item x
// of the grid (items [0, share.n_gitems) are group items) in s_item, with
// kItNMem = 0 when x is no item. Records TQ4_ERR_SEQ when the device lengths make
// more items than the grid holds.
__device__ __forceinline__ void describe_private_item(const DecodeParams& p, int x, int h, int* s_item) {
  const int lane = threadIdx.x & 31;
  int req = 0, sp = 0, total = 0;
  const bool ok = find_item(p, x - p.share.n_gitems, req, sp, total);
  int first = 0, P = 0, nsh = 0, own = 0;
  if (ok) {
    first = request_first_record(p, req);
    P = shared_pos(p, req);
    request_records(p, req, __ldg(p.seq_lens + req), nsh, own);
  }
  if (lane == 0) {
    s_item[kItNMem] = ok ? 1 : 0;
    s_item[kItReq] = req;
    s_item[kItRec] = first + nsh + sp;
    s_item[kItTable] = req;
    s_item[kItPosB] = P + sp * p.split_len;
    s_item[kItPosE] = min(P + (sp + 1) * p.split_len, ok ? __ldg(p.seq_lens + req) : 0);
    if (x == p.share.n_gitems && h == 0 && p.share.n_gitems + total > p.items_ub)
      record_error(p.status, TQ4_ERR_SEQ);
  }
}
// (one thread) every record the item writes must lie inside the workspace; an
// item that would write outside it records TQ4_ERR_SEQ and is dropped
__device__ __forceinline__ void check_item_records(const DecodeParams& p, int* s_item) {
  bool in = true;
  for (int k = 0; k < s_item[kItNMem]; ++k) in = in && s_item[kItRec + k] < p.records_ub;
  if (!in) {
    record_error(p.status, TQ4_ERR_SEQ);
    s_item[kItNMem] = 0;
  }
}

// Warp-collective: group item x (x < share.n_gitems): group gi, split sp of its
// shared positions, one record per member.
__device__ __forceinline__ void describe_group_item(const DecodeParams& p, int x, int* s_item) {
  const int lane = threadIdx.x & 31;
  int gi = 0;
  while (gi + 1 < p.share.n_groups && x >= p.share.item0[gi + 1]) ++gi;
  const int sp = x - p.share.item0[gi];
  const int nm = p.share.n_mem[gi];
  const int gl = p.share.split_len;
  for (int k = 0; k < nm; ++k) {
    const int rq = p.share.mem[gi][k];
    const int first = request_first_record(p, rq);
    if (lane == 0) {
      s_item[kItReq + k] = rq;
      s_item[kItRec + k] = first + sp;
    }
  }
  if (lane == 0) {
    s_item[kItPosB] = sp * gl;
    s_item[kItPosE] = min((sp + 1) * gl, p.share.pos[gi]);
    s_item[kItTable] = p.share.mem[gi][0];
    s_item[kItNMem] = nm;
  }
}

// Split-K decode: grid (items, 4 KV heads). Items [0, share.n_gitems) are group
// items (NTG n-tiles), the rest the requests' own items (NT n-tiles).
template <int NT, int NTG, bool kI8, bool kExact>
__global__ void __launch_bounds__(kDecThreads, 1) decode_splitk_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_item[kItWords];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int h = blockIdx.y;
  pdl_wait();   // every read of the call's inputs comes after the previous kernel
  pdl_launch_dependents();
  const int x = int(blockIdx.x);
  const bool group = x < p.share.n_gitems;
  if (w == 0) {
    if (group) describe_group_item(p, x, s_item);
    else describe_private_item(p, x, h, s_item);   // request req, split sp of its own positions
  }
  if (w == 0 && lane == 0) check_item_records(p, s_item);
  __syncthreads();
  if (s_item[kItNMem] == 0 || x >= p.items_ub) return;
  if constexpr (NTG != NT) {
    if (group) {
      decode_item<NTG, kI8, kExact>(p, smem, s_item);
      return;
    }
  }
  decode_item<NT, kI8, kExact>(p, smem, s_item);
}

// Split-K decode over a 2- or 3-bit pool: grid (items, 4 KV heads). Without
// shared-prefix groups it serves two to four query tokens (one token takes the
// one-token kernel); with groups, items [0, share.n_gitems) are group items (NTG
// n-tiles) and the rest the requests' own items (NT n-tiles), as in the four-bit
// split-K kernel.
template <int NT, int NTG, bool kExact, int kBits>
__global__ void __launch_bounds__(kDecThreads, 1) decode_bits_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_item[kItWords];
  const int w = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int x = int(blockIdx.x);
  pdl_wait();
  pdl_launch_dependents();
  const bool group = x < p.share.n_gitems;
  if (w == 0) {
    if (group) describe_group_item(p, x, s_item);
    else describe_private_item(p, x, h, s_item);
  }
  if (threadIdx.x == 0) check_item_records(p, s_item);
  __syncthreads();
  if (s_item[kItNMem] == 0 || x >= p.items_ub) return;
  if constexpr (NTG != NT) {
    if (group) {
      decode_item<NTG, false, kExact, kBits>(p, smem, s_item);
      return;
    }
  }
  decode_item<NT, false, kExact, kBits>(p, smem, s_item);
}

// One CTA of 8 warps per output row (request, token, query head). Warp w
// merges items first + w, first + w + 8, ... kCombBatch (8) at a time (all loads of a
// group are issued before any is used, so the L2 round trips overlap), then
// the 8 warp results are merged through shared memory, rotated back by R^T
// and written out.
constexpr int kCombWarps = 8;
constexpr int kCombBatch = 8;   // splits each warp loads before using any (one L2 round for up to 64 splits)

__global__ void __launch_bounds__(32 * kCombWarps) decode_combine_kernel(const DecodeParams p) {
  __shared__ float s_m[kCombWarps], s_l[kCombWarps];
  __shared__ float4 s_acc[kCombWarps][32][2];
  __shared__ int s_first;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row_id = blockIdx.x;
  pdl_wait();   // the split partials come from the previous kernel
  pdl_launch_dependents();
  const int qh = row_id % kHq;
  const int tok = (row_id / kHq) % p.n_q;
  const int r = row_id / (kHq * p.n_q);
  const int h = qh / kGroup;
  const int row = tok * kGroup + qh % kGroup;

  const int s_len = __ldg(p.seq_lens + r);   // issued before the scan below needs anything
  int first = 0;   // a single request's records start at 0
  if (p.n_req > 1) {
    if (w == 0) {
      const int f = request_first_record(p, r);
      if (lane == 0) s_first = f;
    }
    __syncthreads();
    first = s_first;
  }
  const bool ok = seq_ok(s_len, p.n_q, p.max_pages);
  int nsh = 0, own = 0;
  request_records(p, r, s_len, nsh, own);
  int n_split = ok ? nsh + own : 0;   // the request's records: shared splits, then its own
  if (first + n_split > p.records_ub) n_split = 0;
  if (threadIdx.x == 0 && (!ok || n_split == 0)) record_error(p.status, TQ4_ERR_SEQ);

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int x0 = first + w; x0 < first + n_split; x0 += kCombBatch * kCombWarps) {
    float2 ml[kCombBatch];
    float4 u[kCombBatch][2];
#pragma unroll
    for (int j = 0; j < kCombBatch; ++j) {
      const int x = x0 + j * kCombWarps;
      if (x < first + n_split) {
        const int64_t rec = (int64_t(x) * kHkv + h) * p.rows_pad + row;
        ml[j] = p.ws_ml[rec];
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + rec * kD + lane * 8);
        u[j][0] = src[0];
        u[j][1] = src[1];
      } else {
        ml[j] = make_float2(-INFINITY, 0.f);
        u[j][0] = u[j][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mn = m;
#pragma unroll
    for (int j = 0; j < kCombBatch; ++j) mn = fmaxf(mn, ml[j].x);
    if (mn == -INFINITY) continue;
    const float a = fast_exp2((m - mn) * kLog2e);
    l *= a;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= a;
#pragma unroll
    for (int j = 0; j < kCombBatch; ++j) {
      const float wj = fast_exp2((ml[j].x - mn) * kLog2e);   // 0 for empty slots (m = -inf)
      l = fmaf(wj, ml[j].y, l);
      acc[0] = fmaf(wj, u[j][0].x, acc[0]); acc[1] = fmaf(wj, u[j][0].y, acc[1]);
      acc[2] = fmaf(wj, u[j][0].z, acc[2]); acc[3] = fmaf(wj, u[j][0].w, acc[3]);
      acc[4] = fmaf(wj, u[j][1].x, acc[4]); acc[5] = fmaf(wj, u[j][1].y, acc[5]);
      acc[6] = fmaf(wj, u[j][1].z, acc[6]); acc[7] = fmaf(wj, u[j][1].w, acc[7]);
    }
    m = mn;
  }
  if (lane == 0) {
    s_m[w] = m;
    s_l[w] = l;
  }
  s_acc[w][lane][0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  s_acc[w][lane][1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  __syncthreads();
  if (w != 0) return;
  float M = -INFINITY;
#pragma unroll
  for (int ww = 0; ww < kCombWarps; ++ww) M = fmaxf(M, s_m[ww]);
  float L = 0.f, o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int ww = 0; ww < kCombWarps; ++ww) {
      const float a = fast_exp2((s_m[ww] - M) * kLog2e);
      L = fmaf(a, s_l[ww], L);
      const float4 v0 = s_acc[ww][lane][0], v1 = s_acc[ww][lane][1];
      o[0] = fmaf(a, v0.x, o[0]); o[1] = fmaf(a, v0.y, o[1]); o[2] = fmaf(a, v0.z, o[2]);
      o[3] = fmaf(a, v0.w, o[3]); o[4] = fmaf(a, v1.x, o[4]); o[5] = fmaf(a, v1.y, o[5]);
      o[6] = fmaf(a, v1.z, o[6]); o[7] = fmaf(a, v1.w, o[7]);
    }
  }
  float res[8];
  if (p.rotate) {   // o = R^T (o' / l) = diag(s) H (o' / l) / 16
    warp_fwht256(o);
    const float inv = (L > 0.f) ? 0.0625f / L : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) res[i] = o[i] * inv * sign_of(p.signs, lane * 8 + i);
  } else {          // the INT8 arm attends in the original domain: o = o' / l
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) res[i] = o[i] * inv;
  }
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
