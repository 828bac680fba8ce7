/*
 * tq4.h -- C ABI of the TQ4 paged-KV attention library (libtq4.so, CUDA sm_100a).
 *
 * The operation comes from the JustFit pages:
 *   [KVEXEC] simpleprog.com, "Fitting a 27B-Parameter LLM into 24 GiB of Laptop
 *            Memory", section "KVExec: Fused Reconstruction with Layer-Scoped
 *            Lifetime": each 256-dim K or V head vector is stored as 32 U32 words
 *            (eight 4-bit centroid indices per word) plus one FP16 norm;
 *            reconstruction reads the packed page IDs, looks up centroids, applies
 *            the inverse Hadamard rotation, restores the norm and feeds scaled
 *            dot-product attention; single-query decode runs page-native on the
 *            compressed data, multi-query prefill reconstructs then attends;
 *            256-dim heads, 256-token pages.
 *   [BUDGET] same page, section "The Memory Budget Equation": 16 attention
 *            layers x 4 KV heads x 256 dims; 1,040 B per layer-position.
 *   [V2]     wpnews.pro, "JustFit: Run Qwen 27B Fast with its full 256K context
 *            on a 24 GB Mac", mechanism table, row KVExec: rotated-domain attention.
 *
 * Conventions fixed by this library where the pages are silent:
 *   codebook   16-level Lloyd-Max quantiser for N(0, 1/256), solved by the
 *              library in fp64 at context creation; index j -> centroid c_j,
 *              ascending; nearest centroid, ties to the lower index. Encode
 *              compares against the fp64 midpoints rounded to fp32;
 *              reconstruction reads the centroids rounded to fp32; the attention
 *              kernels feed each centroid to f16 tensor-core products as the
 *              pair c16 = f16(c_j), r16 = f16(c_j - c16), which carries c_j to
 *              about 2^-21 relative.
 *   rotation   R = H diag(s) / 16, H the Sylvester Hadamard matrix, s the
 *              caller's +-1 sign diagonal. Encode quantises y = R x / ||x||;
 *              reconstruction is x_hat = fp16(||x||) * R^T c[idx].
 *   packing    coordinate 8w+i is bits 4i..4i+3 of word w (little-endian u32).
 *   norm       ||x||_2 rounded to fp16 (nearest even); zero vectors store 0.
 *   GQA        24 query heads, query head h reads KV head h / 6.
 *   page       one layer's pool is num_pages pages of TQ4_PAGE_BYTES bytes:
 *                [0, 131072)       K words  [4 heads][256 slots][32 u32]
 *                [131072, 262144)  V words  [4 heads][256 slots][32 u32]
 *                [262144, 264192)  K norms  [4 heads][256 slots] fp16
 *                [264192, 266240)  V norms  [4 heads][256 slots] fp16
 *              Position p of a request lives in page page_table[p / 256],
 *              slot p % 256. Page tables are int32 physical page ids; the
 *              host page pool of tq4_pages.h can supply them.
 *
 * Memory: the caller owns every buffer. Pointers documented as "device" must be
 * device memory (or managed memory) of the current device; "host" pointers are
 * read before the call returns. The library allocates device memory only in
 * tq4_ctx_create (a 4-byte status word) and frees it in tq4_ctx_destroy.
 *
 * Errors: every call returns TQ4_OK (0) or a negative TQ4_ERR_* code.
 * Argument errors are detected on the host and returned synchronously, before
 * anything is launched. Kernels run asynchronously on the given stream
 * (a cudaStream_t passed as void*, NULL = legacy default stream). Problems that
 * only the device can see (a page id outside [0, num_pages), a sequence length
 * inconsistent with the table or the host-side bounds) make the kernel skip the
 * affected work and record the first error code in the context's status word;
 * tq4_get_status() reads and clears it. No kernel traps, and no kernel waits on
 * another block.
 *
 * Dtypes: bf16 tensors are passed as raw uint16_t bit patterns.
 */
#ifndef TQ4_H
#define TQ4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ4_OK                 0
#define TQ4_ERR_ARG           -1  /* bad pointer, size, count or dtype             */
#define TQ4_ERR_UNSUPPORTED   -2  /* shape the library is not specialised for     */
#define TQ4_ERR_PAGE_RANGE    -3  /* page id outside [0, num_pages) (device check) */
#define TQ4_ERR_CUDA          -4  /* a CUDA runtime call failed                    */
#define TQ4_ERR_WORKSPACE     -5  /* workspace missing or smaller than required    */
#define TQ4_ERR_SEQ           -6  /* device-side sequence length check failed      */
#define TQ4_ERR_TIMEOUT       -7  /* a bounded device-side wait gave up            */
#define TQ4_ERR_NO_PAGES      -8  /* page pool: not enough capacity (tq4_pages.h)  */

#define TQ4_HEAD_DIM        256
#define TQ4_PAGE_POSITIONS  256
#define TQ4_KV_HEADS        4
#define TQ4_Q_HEADS         24
#define TQ4_WORDS           32
#define TQ4_VECTOR_BYTES    130
#define TQ4_POSITION_BYTES  1040          /* one layer-position: 4 heads x (K+V) x 130 B */
#define TQ4_PAGE_BYTES      266240        /* 256 layer-positions                         */
#define TQ4_MAX_QUERY_TOKENS 4
#define TQ4_INT8_POSITION_BYTES 2064      /* INT8 arm: 4 heads x (K+V) x (256 + 2) B    */
#define TQ4_INT8_PAGE_BYTES     528384    /* INT8 arm: 256 layer-positions             */
#define TQ4_TQB2_PAGE_BYTES     135168    /* 2-bit variant: 256 x 528 B                */
#define TQ4_TQB3_PAGE_BYTES     200704    /* 3-bit variant: 256 x 784 B                */

#define TQ4_DTYPE_F32   0
#define TQ4_DTYPE_BF16  1

typedef struct tq4_ctx tq4_ctx;

/* Create a context on the current CUDA device.
 * signs: host, int8[256], each +1 or -1 (the rotation's sign diagonal).
 * The context holds the signs, the codebook and a device status word.
 * Returns TQ4_ERR_ARG for a NULL pointer or a sign that is not +-1. */
int tq4_ctx_create(const int8_t* signs, tq4_ctx** out);

/* Destroy a context; synchronises the device first. NULL is accepted. */
int tq4_ctx_destroy(tq4_ctx* ctx);

/* Copy the context's codebook: centroids[16] and decision boundaries[15]
 * (midpoints of adjacent centroids), both host double arrays. */
int tq4_codebook(const tq4_ctx* ctx, double* centroids, double* boundaries);

/* Encode n_tok new positions of one layer and write them into the pool
 * (step "rotate + quantize + pack new K/V into pages"; [KVEXEC], [BUDGET]).
 *   pool        device, num_pages * TQ4_PAGE_BYTES bytes, written in place.
 *   page_table  device int32[table_len], this request's physical page ids.
 *   start_pos   position of the first new token; positions
 *               [start_pos, start_pos + n_tok) must satisfy
 *               (start_pos + n_tok + 255) / 256 <= table_len.
 *   k_new,v_new device [n_tok][4][256] of dtype (TQ4_DTYPE_F32 or TQ4_DTYPE_BF16).
 * n_tok == 0 is a no-op. Positions whose page id is out of range are skipped
 * and TQ4_ERR_PAGE_RANGE is recorded in the status word. */
int tq4_encode_append(tq4_ctx* ctx, void* pool, int32_t num_pages,
                      const int32_t* page_table, int32_t table_len,
                      int32_t start_pos, int32_t n_tok,
                      const void* k_new, const void* v_new, int dtype, void* stream);

/* Reconstruct positions [start, start + n) of one request as explicit fp32 K/V
 * (centroid lookup, inverse rotation, norm restore; [KVEXEC]). Test/export path,
 * not used by attention.
 *   k_out, v_out device float[n][4][256]. */
int tq4_reconstruct(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                    const int32_t* page_table, int32_t table_len,
                    int32_t start, int32_t n, float* k_out, float* v_out, void* stream);

/* Bytes of device workspace tq4_decode_attention needs for this problem
 * (split-K partial results). total_seq_len = sum of seq_lens over requests. */
size_t tq4_decode_workspace_bytes(const tq4_ctx* ctx, int32_t n_req, int32_t n_q,
                                  int64_t total_seq_len);

/* Decode attention: n_q (1..4) query tokens per request against the request's
 * paged TQ4 history, fused with reconstruction, split-K with a combine pass
 * ([KVEXEC] single-query page-native decode and packed verifier; [V2]
 * rotated-domain attention). No full-precision K/V is written to memory.
 *   pool         device, one layer, num_pages * TQ4_PAGE_BYTES bytes.
 *   q            device bf16 [n_req][n_q][24][256].
 *   page_tables  device int32 [n_req][max_pages].
 *   seq_lens     device int32 [n_req]; positions per request INCLUDING the n_q
 *                new ones, which must already be appended. Query token t of a
 *                request sees positions [0, seq_len - n_q + t] (causal among the
 *                n_q tokens).
 *   total_seq_len host; sum of seq_lens (used to plan the split; the kernel
 *                checks it and records TQ4_ERR_SEQ if the device values exceed it).
 *   scale        softmax scale (e.g. 1/16 for dim 256).
 *   out          device [n_req][n_q][24][256], out_dtype TQ4_DTYPE_BF16 or _F32.
 *   workspace    device, at least tq4_decode_workspace_bytes(...) bytes, 256-B aligned.
 * Softmax and all accumulation are fp32. */
int tq4_decode_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                         const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                         const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                         int64_t total_seq_len, float scale,
                         void* out, int out_dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Decode step with its append ([KVEXEC]: the step's new K/V are encoded into the
 * request's TQ4 pages, then attention runs over the paged history including them):
 * the same result as tq4_encode_append of each request's n_q new positions
 * followed by tq4_decode_attention, in one call.
 *   pool        device, written: the new positions are stored in it.
 *   k_new,v_new device [n_req][n_q][4][256] of new_dtype (TQ4_DTYPE_F32 or
 *               TQ4_DTYPE_BF16). Token t of request r is stored at position
 *               seq_lens[r] - n_q + t of that request (seq_lens count the new
 *               positions, as in tq4_decode_attention).
 *   all other arguments, the workspace, outputs and errors: as tq4_decode_attention.
 * With n_q == 1 the encode runs inside the decode kernel: the CTA that holds a
 * request's last position encodes it (per KV head) and stores it before it loads
 * that tile, so no separate append launch is made. With n_q > 1 a tail-encode
 * kernel runs ahead of the decode. A new position whose page id is out of range
 * records TQ4_ERR_PAGE_RANGE and is not written. */
int tq4_decode_append_attention(tq4_ctx* ctx, void* pool, int32_t num_pages,
                                const void* k_new, const void* v_new, int new_dtype,
                                const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                int64_t total_seq_len, float scale,
                                void* out, int out_dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Decode over requests that share leading pages, reading the shared pages once
 * ([STATE] simpleprog.com, "Fitting a 27B-Parameter LLM into 24 GiB of Laptop
 * Memory", section "StateTrans", and [REUSE] section "Prefix Reuse": a restored
 * prefix is referenced by every request that reuses it, so several requests'
 * tables hold the same page ids). Same computation and arguments as
 * tq4_decode_attention (tq4_decode_append_attention when k_new, v_new are given;
 * both NULL: no append), plus:
 *   prefix_leader host int32[n_req]: the request whose table this request's first
 *                 pages share (the same page ids); a leader names itself.
 *   prefix_pages  host int32[n_req]: the number of shared leading pages; equal for
 *                 every request of a group (leader included), at most max_pages.
 * Requests with the same leader form a group; its shared positions are loaded
 * and expanded once per KV head and scored against all members' query rows in
 * one pass (at most 48 rows, i.e. 8 one-token, 4 two-token or 2 three/four-token
 * members per group; larger groups are cut into several; past 32 groups the
 * rest read their shared pages on their own). Shared pages must hold history:
 * every member's seq_len - n_q must be at least prefix_pages * 256 (positions a
 * query may not see are still masked). Results equal tq4_decode_attention's up
 * to fp32 summation order. A leader out of range, a leader that is not its own
 * leader, or unequal page counts within a group: TQ4_ERR_ARG. The append (n_q
 * tokens per request) runs as a tail-encode kernel ahead of the decode.
 *   workspace    device, at least tq4_decode_shared_workspace_bytes(...) bytes. */
size_t tq4_decode_shared_workspace_bytes(const tq4_ctx* ctx, int32_t n_req, int32_t n_q,
                                         int64_t total_seq_len, int32_t max_pages,
                                         const int32_t* prefix_leader, const int32_t* prefix_pages);
int tq4_decode_attention_shared(tq4_ctx* ctx, void* pool, int32_t num_pages,
                                const void* k_new, const void* v_new, int new_dtype,
                                const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                int64_t total_seq_len, const int32_t* prefix_leader,
                                const int32_t* prefix_pages, float scale,
                                void* out, int out_dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Prefill attention: a causal chunk of n_tok query tokens against the request's
 * TQ4 prefix [0, prefix_len) plus the chunk itself, whose K/V are given at full
 * precision ([KVEXEC] multi-query prefill). The chunk is not appended; call
 * tq4_encode_append afterwards.
 *   q                 device bf16 [n_tok][24][256].
 *   k_chunk, v_chunk  device bf16 [n_tok][4][256].
 *   page_table        device int32[table_len] covering the prefix.
 *   out               device [n_tok][24][256], out_dtype TQ4_DTYPE_BF16 or _F32.
 *                     The fp32 output also runs the products that only an fp32
 *                     result can resolve (about 1.5x the tensor work).
 *   workspace         device scratch of tq4_prefill_workspace_bytes(n_tok) bytes,
 *                     256-B aligned.
 * Softmax and all accumulation are fp32. */
size_t tq4_prefill_workspace_bytes(int32_t n_tok);
int tq4_prefill_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                          const int32_t* page_table, int32_t table_len, int32_t prefix_len,
                          const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk,
                          int32_t n_tok, float scale, void* out, int out_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/* The same prefill by direct inverse reconstruction ([KVEXEC]: multi-query
 * prefill reconstructs the history directly, with the packed path as the
 * alternative): a prologue kernel rebuilds every prefix K/V vector as a dense
 * rotated-domain row n * c[idx] (f16 hi + lo) in the workspace, and the attention
 * kernel then reads prefix positions as rows, like the chunk's own, instead of
 * expanding packed words. Same arguments, results (up to fp32 rounding order) and
 * errors as tq4_prefill_attention; the prefix rows cost
 * prefix_len * 8 KiB of workspace and their write and re-reads in HBM.
 *   workspace device scratch of tq4_prefill_reconstructed_workspace_bytes(
 *             prefix_len, n_tok) bytes, 256-B aligned. */
size_t tq4_prefill_reconstructed_workspace_bytes(int32_t prefix_len, int32_t n_tok);
int tq4_prefill_attention_reconstructed(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                                        const int32_t* page_table, int32_t table_len,
                                        int32_t prefix_len, const uint16_t* q,
                                        const uint16_t* k_chunk, const uint16_t* v_chunk,
                                        int32_t n_tok, float scale, void* out, int out_dtype,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Bounded device-side waits (a tile's copy, a tensor-core step, the fused
 * append) give up after a number of polls, record TQ4_ERR_TIMEOUT in the status
 * word and let the kernel finish without the rest of its work: it drains the
 * copies and tensor-core operations it has issued, frees its tensor memory and
 * returns, and the context stays usable. This call exists to test that path.
 *   polls            polls before a wait gives up, for later calls on the
 *                    context; 0 restores the default TQ4_DEFAULT_WAIT_POLLS.
 *                    The drains before exit always use the default.
 *   withhold_signal  nonzero: later calls withhold one producer signal so that
 *                    a wait is sure to run out (the one-token decode kernel
 *                    does not issue the copy of each warp's first tile; the
 *                    tensor-memory decode of 2-4 tokens does not signal the
 *                    tensor-core issuer that the first key chunk is ready; the
 *                    prefill kernel does not signal it that P of tile
 *                    min(1, tiles - 1) is ready); their results are
 *                    then undefined and the status is TQ4_ERR_TIMEOUT. 0 (the
 *                    default) restores normal operation.
 * Returns TQ4_ERR_ARG for a NULL context. */
#define TQ4_DEFAULT_WAIT_POLLS (1u << 24)
int tq4_ctx_set_wait_limit(tq4_ctx* ctx, uint32_t polls, int withhold_signal);

/* Which kernel decodes requests of 2 to 4 query tokens (the tq4_decode_attention
 * family, without shared-prefix groups; the arithmetic is the same, see
 * tq4_decode_attention):
 *   TQ4_DECODE_PATH_TENSOR_MEMORY  tcgen05 MMAs with tensor-memory
 *        accumulators: tile positions are the MMA's rows, the keys are expanded
 *        into tensor memory and the values into shared memory;
 *   TQ4_DECODE_PATH_WARP_MMA       (default) the warp-level mma.sync kernel that
 *        also serves one-token groups, shared-prefix groups and the INT8 arm.
 * The two give the same results up to fp32 summation order. The choice holds
 * for later calls on the context.
 * Returns TQ4_ERR_ARG for a NULL context or an unknown path. */
#define TQ4_DECODE_PATH_TENSOR_MEMORY 0
#define TQ4_DECODE_PATH_WARP_MMA      1
int tq4_ctx_set_decode_path(tq4_ctx* ctx, int path);

/* Decode attention for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for the library's users.
 * Some callers cannot allocate: plugin code inside a host program that owns the
 * whole device-memory budget (a raw cudaMalloc would bypass its accounting),
 * and serving processes that reserve all device memory up front and run under
 * a hard memory guard. This call takes the same arguments as
 * tq4_decode_attention minus the workspace, and keeps the split-K partial
 * results in a fixed array of TQ4_NOALLOC_SCRATCH_BYTES (8 MiB) that is part of
 * the library: every GPU that loads the library holds it until the process
 * exits. It allocates nothing and calls no allocating routine.
 *   - tq4_ctx_create looks up the array's device address on the context's
 *     device (the runtime call cudaGetSymbolAddress, with that device current)
 *     and keeps it in the context, so this call does no set-up of its own. A
 *     device reset (cudaDeviceReset, or any teardown of the device's primary
 *     context) invalidates every context made before it, this address included:
 *     create a new context afterwards.
 *   - Every call on a device shares the one array, so calls whose kernels may
 *     overlap on the GPU (different streams, no ordering between them) race
 *     and give wrong results; order them, e.g. issue them on one stream.
 *   - Nothing in the array needs to start at zero: each call writes every
 *     partial result it later reads.
 *   - A problem whose tq4_decode_workspace_bytes() exceeds
 *     TQ4_NOALLOC_SCRATCH_BYTES is rejected with TQ4_ERR_WORKSPACE before
 *     anything is launched. The workspace grows with the number of split-K
 *     items (about one per SM / 4 KV heads for the whole batch, plus one per
 *     request) times 8 (one query token) or 24 (two to four) query rows: on a
 *     148-SM B200 the array holds 254 items with one query token (about 217
 *     requests with long histories) and 84 items with four (about 47). */
#define TQ4_NOALLOC_SCRATCH_BYTES (8u << 20)
int tq4_decode_attention_noalloc(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                                 const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                 int64_t total_seq_len, float scale,
                                 void* out, int out_dtype, void* stream);

/* The uniform INT8 comparison arm ([REASONING] simpleprog.com, "Fitting a
 * 27B-Parameter LLM into 24 GiB of Laptop Memory", section "Reasoning at 200K":
 * "a uniform INT8 comparison" arm runs next to TQ4; the page defines it no
 * further). This library's reading: each 256-dim K or V head vector is stored as
 * 256 int8 codes q_i = round-half-to-even(x_i / s), s = max_i |x_i| / 127, plus s
 * as fp16 (the codes use the unrounded s; a zero vector stores s = 0); no rotation
 * and no codebook; reconstruction is x_hat = fp16(s) * q. A pool of the INT8 arm is
 * num_pages pages of TQ4_INT8_PAGE_BYTES bytes:
 *   [0, 262144)       K codes  [4 heads][256 slots][256 int8]
 *   [262144, 524288)  V codes  [4 heads][256 slots][256 int8]
 *   [524288, 526336)  K scales [4 heads][256 slots] fp16
 *   [526336, 528384)  V scales [4 heads][256 slots] fp16
 * Page tables, lengths, queries, outputs, workspaces (tq4_decode_workspace_bytes)
 * and errors are as for the TQ4 calls of the same shape. */
int tq4_int8_encode_append(tq4_ctx* ctx, void* pool, int32_t num_pages,
                           const int32_t* page_table, int32_t table_len,
                           int32_t start_pos, int32_t n_tok,
                           const void* k_new, const void* v_new, int dtype, void* stream);
int tq4_int8_decode_attention(tq4_ctx* ctx, const void* pool, int32_t num_pages,
                              const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                              const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                              int64_t total_seq_len, float scale,
                              void* out, int out_dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The 2- and 3-bit variants of the format. The pages describe the four-bit
 * encoding only ([KVEXEC] simpleprog.com, "Fitting a 27B-Parameter LLM into
 * 24 GiB of Laptop Memory", section "KVExec"); this library's reading keeps every
 * step of it (norm, rotation R = H diag(s) / 16, nearest-centroid quantiser with
 * ties low, fp16 norm, rotated-domain attention) with b = bits per coordinate and
 * a 2^b-level Lloyd-Max codebook for N(0, 1/256) computed in fp64 by the library.
 * Per 256-dim vector: 8 b u32 words and one fp16 norm. Plane 0, words 0..15: the
 * low two bits of every index, coordinate 16w + i in bits 2i..2i+1 of word w;
 * plane 1 (b = 3 only), words 16..23: bit 2, coordinate 32w + i in bit i of word
 * 16 + w. A pool is num_pages pages of TQ4_TQB2_PAGE_BYTES (b = 2) or
 * TQ4_TQB3_PAGE_BYTES (b = 3) bytes:
 *   [0, 4*256*32b)          K words [4 heads][256 slots][8b u32]
 *   [.., 2*4*256*32b)       V words (same shape)
 *   then K norms [4][256] fp16, then V norms [4][256] fp16.
 * Page tables, lengths, queries, outputs, workspaces (tq4_decode_workspace_bytes)
 * and errors are as for the four-bit calls of the same shape; bits other than 2
 * and 3 return TQ4_ERR_UNSUPPORTED. tq4_tqb_decode_append_attention is the fused
 * step of tq4_decode_append_attention for a b-bit pool: the n_q new tokens' K and
 * V are encoded into the last n_q positions of every request (one query token:
 * inside the decode kernel; more: a tail-encode kernel ahead of it), then
 * decoded as tq4_tqb_decode_attention does. k_new, v_new, new_dtype and the
 * pool's ownership are as for tq4_decode_append_attention.
 * tq4_tqb_prefill_attention is tq4_prefill_attention_reconstructed over a b-bit
 * pool: the prefix is rebuilt as dense rows n * c[idx] (the 2^b-level codebook)
 * in the workspace, then the same causal attention of the chunk runs over them;
 * workspace size tq4_prefill_reconstructed_workspace_bytes(prefix_len, n_tok).
 * tq4_tqb_reconstruct is tq4_reconstruct for a b-bit pool (explicit fp32 K/V).
 * tq4_tqb_decode_attention_shared is tq4_decode_attention_shared for a b-bit pool
 * (the same group description, workspace and append arguments).
 * tq4_tqb_codebook copies the fp64 centroids (2^b) and boundaries (2^b - 1). */
int tq4_tqb_codebook(const tq4_ctx* ctx, int bits, double* centroids, double* boundaries);
int tq4_tqb_encode_append(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages,
                          const int32_t* page_table, int32_t table_len,
                          int32_t start_pos, int32_t n_tok,
                          const void* k_new, const void* v_new, int dtype, void* stream);
int tq4_tqb_decode_attention(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages,
                             const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                             const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                             int64_t total_seq_len, float scale,
                             void* out, int out_dtype,
                             void* workspace, size_t workspace_bytes, void* stream);
int tq4_tqb_decode_attention_shared(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages,
                                    const void* k_new, const void* v_new, int new_dtype,
                                    const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                    const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                    int64_t total_seq_len, const int32_t* prefix_leader,
                                    const int32_t* prefix_pages, float scale,
                                    void* out, int out_dtype,
                                    void* workspace, size_t workspace_bytes, void* stream);
int tq4_tqb_reconstruct(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages,
                        const int32_t* page_table, int32_t table_len,
                        int32_t start, int32_t n, float* k_out, float* v_out, void* stream);
int tq4_tqb_prefill_attention(tq4_ctx* ctx, int bits, const void* pool, int32_t num_pages,
                              const int32_t* page_table, int32_t table_len,
                              int32_t prefix_len, const uint16_t* q,
                              const uint16_t* k_chunk, const uint16_t* v_chunk,
                              int32_t n_tok, float scale, void* out, int out_dtype,
                              void* workspace, size_t workspace_bytes, void* stream);
int tq4_tqb_decode_append_attention(tq4_ctx* ctx, int bits, void* pool, int32_t num_pages,
                                    const void* k_new, const void* v_new, int new_dtype,
                                    const uint16_t* q, const int32_t* page_tables, int32_t max_pages,
                                    const int32_t* seq_lens, int32_t n_req, int32_t n_q,
                                    int64_t total_seq_len, float scale,
                                    void* out, int out_dtype,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise the stream, return the first device-side error recorded since
 * the last call (TQ4_OK if none) and clear it. */
int tq4_get_status(tq4_ctx* ctx, void* stream);

/* Static description of a status code. */
const char* tq4_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* TQ4_H */
