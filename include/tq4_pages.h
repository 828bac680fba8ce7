/*
 * tq4_pages.h - host page pool for the paged TQ4 KV cache: which physical
 * 256-position page each request's logical page maps to (the page tables that
 * tq4_decode_attention, tq4_decode_append_attention and tq4_prefill_attention
 * read), with reference-counted shared prefixes, admission by reserved page
 * equivalents and release at step boundaries.
 *
 * Sources (cited by page title and section):
 *   [KVEXEC] simpleprog.com, "Fitting a 27B-Parameter LLM into 24 GiB of Laptop
 *            Memory", section "StateTrans": admission reserves
 *            ceil((prompt + min(output budget, 8192)) / 256) physical-page
 *            equivalents; shared prefixes are reference counted; on completion
 *            or cancellation the page references are decremented after the
 *            current step, and a page id returns to the free list only when its
 *            count reaches zero after that boundary.
 *   [KVEXEC] same page, section "Prefix Reuse": a request whose prefix is cached
 *            restores those positions and prefills only the remainder.
 *
 * Model (readings where the page is silent):
 *   - Pages are ids 0 .. num_pages-1. The free list is first-in first-out; it
 *     starts in ascending id order, and the pages freed at one boundary join
 *     its tail in ascending id order.
 *   - A request holds a page table (logical page i -> page id) and a length in
 *     positions. Growing it to a length L maps ceil(L / 256) pages.
 *   - Admission reserves R = ceil((prompt_len + min(out_budget, 8192)) / 256)
 *     page equivalents, less the full pages it shares with a restored prefix
 *     (those need no new page). Pages the request takes for itself draw on its
 *     reservation first; beyond it (output past the guaranteed part) a page is
 *     taken only from capacity nobody has reserved. "Available" capacity is the
 *     free pages minus every live request's unused reservation, and a request
 *     is admitted only if its reservation fits in it. Which blocked request to
 *     admit or bypass is the caller's policy.
 *   - Prefix restore maps the source request's first floor(L / 256) pages by
 *     reference (count + 1). A partial last page (L % 256 > 0) cannot be shared,
 *     because the source may still write its later slots: the new request gets a
 *     fresh page, and the call reports (copy_src, copy_dst) for the caller to
 *     copy the page bytes (TQ4_PAGE_BYTES, one cudaMemcpyAsync) before the new
 *     request's first attention call.
 *   - tq4_pages_finish marks a request as leaving. Its unused reservation is
 *     released at once (those page equivalents were never mapped), but its pages
 *     keep their references until tq4_pages_step_boundary, which the caller
 *     makes once the step's kernels have completed (they may still read the
 *     pages). At the boundary every page of every leaving request loses one
 *     reference, the pages that reach zero join the free list, and the leaving
 *     requests are forgotten.
 *
 * Ownership and threads: the pool is host memory owned by the handle; calls on
 * one handle are serialised by an internal lock. No call touches the GPU.
 * Errors: TQ4_OK (0) or a negative TQ4_ERR_* code from tq4.h; a failed call
 * changes nothing. TQ4_ERR_NO_PAGES means the capacity is not there now.
 */
#ifndef TQ4_PAGES_H
#define TQ4_PAGES_H

#include <stdint.h>

#include "tq4.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq4_pages tq4_pages;

/* A pool of num_pages pages (num_pages >= 1), all free. */
int tq4_pages_create(int32_t num_pages, tq4_pages** out);
/* Frees the handle (NULL is accepted). */
int tq4_pages_destroy(tq4_pages* pp);

/* Page equivalents admission reserves: ceil((prompt_len + min(out_budget, 8192)) / 256).
 * Returns -1 if either length is negative or prompt_len exceeds 2^53. */
int64_t tq4_pages_reservation(int64_t prompt_len, int64_t out_budget);

/* Admits a request (length 0, or prefix_len after a restore) and returns its id
 * in *req_out (ids count up from 0 and are not reused).
 * src_req < 0: no restore (prefix_len must be 0). Otherwise the first prefix_len
 * positions of live request src_req (1 <= prefix_len <= its length) are restored:
 * full pages are shared, a partial last page is copied. *copy_src and *copy_dst
 * (both may be NULL when src_req < 0) receive the page copy to perform, or -1.
 * prompt_len counts the restored positions too (prefix_len <= prompt_len).
 * TQ4_ERR_NO_PAGES if the reservation does not fit the available capacity;
 * TQ4_ERR_ARG once 2^31 - 1 ids have been handed out. */
int tq4_pages_admit(tq4_pages* pp, int64_t prompt_len, int64_t out_budget, int32_t src_req, int64_t prefix_len,
                    int32_t* req_out, int32_t* copy_src, int32_t* copy_dst);

/* Grows live request req to new_len positions (never shrinks: new_len below its
 * length is TQ4_ERR_ARG), mapping ceil(new_len / 256) pages. All or nothing:
 * TQ4_ERR_NO_PAGES if the pages beyond its reservation are not available. */
int tq4_pages_grow(tq4_pages* pp, int32_t req, int64_t new_len);

/* Marks live request req as leaving (completion and cancellation alike); its
 * references are dropped at the next step boundary. */
int tq4_pages_finish(tq4_pages* pp, int32_t req);

/* The step boundary: applies every pending release. Returns the number of pages
 * that joined the free list (>= 0), or a negative error. */
int tq4_pages_step_boundary(tq4_pages* pp);

/* Page table row of request req (live or leaving): writes its page ids to
 * table[0 .. n), n = its page count, and -1 to table[n .. max_pages). *n_pages
 * and *len (either may be NULL) receive n and its length in positions.
 * TQ4_ERR_ARG if n > max_pages or req is unknown. */
int tq4_pages_table(const tq4_pages* pp, int32_t req, int32_t* table, int32_t max_pages, int32_t* n_pages,
                    int64_t* len);

/* Counts: free pages; capacity available to new reservations or surplus growth
 * (free pages minus unused reservations of live requests); references held on
 * one page. Negative TQ4_ERR_ARG for a NULL handle or a page id out of range. */
int32_t tq4_pages_free_count(const tq4_pages* pp);
int32_t tq4_pages_available(const tq4_pages* pp);
int32_t tq4_pages_refcount(const tq4_pages* pp, int32_t page);

/* The free list in order (head first): writes min(count, cap) ids to out and
 * returns count. */
int32_t tq4_pages_free_list(const tq4_pages* pp, int32_t* out, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* TQ4_PAGES_H */
