// Host page pool for the paged TQ4 KV cache (include/tq4_pages.h).
//
// [KVEXEC] simpleprog.com, "Fitting a 27B-Parameter LLM into 24 GiB of Laptop
// Memory": section "StateTrans" (admission reservation, reference-counted shared
// prefixes, release after the step boundary, free list) and section "Prefix
// Reuse" (restore a cached prefix, prefill the remainder). The header states the
// model and the readings taken where the page is silent.
//
// Plain host C++: a FIFO free list, one reference count per page, and per
// request its page table, length, reservation and the pages it took itself.
// Every call validates first and then mutates, so a failed call changes nothing.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <deque>
#include <map>
#include <mutex>
#include <new>
#include <vector>

#include "tq4.h"
#include "tq4_pages.h"

namespace {

constexpr int64_t kPage = TQ4_PAGE_POSITIONS;
constexpr int64_t kGuaranteedOutput = 8192;   // output positions admission always reserves for

struct Request {
  std::vector<int32_t> pages;   // logical page i -> page id
  int64_t len = 0;              // positions
  int64_t reserve = 0;          // page equivalents reserved at admission (shared pages excluded)
  int64_t own = 0;              // pages this request took itself (fresh and copied)
  bool leaving = false;
  int64_t unused_reserve() const { return leaving ? 0 : std::max<int64_t>(reserve - own, 0); }
};

int64_t pages_for(int64_t len) { return (len + kPage - 1) / kPage; }

}  // namespace

struct tq4_pages {
  int32_t num_pages = 0;
  std::vector<int32_t> refs;
  std::deque<int32_t> free_list;
  std::map<int32_t, Request> reqs;   // ordered: deterministic iteration at the boundary
  int32_t next_id = 0;
  mutable std::mutex mu;

  int64_t reserved_unused() const {
    int64_t s = 0;
    for (const auto& kv : reqs) s += kv.second.unused_reserve();
    return s;
  }
  int64_t available() const { return int64_t(free_list.size()) - reserved_unused(); }
  Request* live(int32_t id) {
    auto it = reqs.find(id);
    return (it == reqs.end() || it->second.leaving) ? nullptr : &it->second;
  }
  int32_t take() {   // caller has checked that the free list is long enough
    const int32_t id = free_list.front();
    free_list.pop_front();
    refs[size_t(id)] = 1;
    return id;
  }
  // Pages of a request of `own` own pages and reservation `reserve` that must come
  // from unreserved capacity when it takes `extra` more pages.
  static int64_t beyond_reserve(int64_t reserve, int64_t own, int64_t extra) {
    const int64_t inside = std::max<int64_t>(std::min<int64_t>(reserve - own, extra), 0);
    return extra - inside;
  }
};

extern "C" {

int tq4_pages_create(int32_t num_pages, tq4_pages** out) {
  if (!out || num_pages < 1) return TQ4_ERR_ARG;
  *out = nullptr;
  tq4_pages* pp = new (std::nothrow) tq4_pages();
  if (!pp) return TQ4_ERR_ARG;
  pp->num_pages = num_pages;
  pp->refs.assign(size_t(num_pages), 0);
  for (int32_t i = 0; i < num_pages; ++i) pp->free_list.push_back(i);
  *out = pp;
  return TQ4_OK;
}

int tq4_pages_destroy(tq4_pages* pp) {
  delete pp;
  return TQ4_OK;
}

int64_t tq4_pages_reservation(int64_t prompt_len, int64_t out_budget) {
  if (prompt_len < 0 || out_budget < 0 || prompt_len > (int64_t(1) << 53)) return -1;
  return pages_for(prompt_len + std::min(out_budget, kGuaranteedOutput));
}

int tq4_pages_admit(tq4_pages* pp, int64_t prompt_len, int64_t out_budget, int32_t src_req, int64_t prefix_len,
                    int32_t* req_out, int32_t* copy_src, int32_t* copy_dst) {
  if (!pp || !req_out || prompt_len < 0 || out_budget < 0 || prefix_len < 0) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  const Request* src = nullptr;
  if (src_req >= 0) {
    src = pp->live(src_req);
    if (!src || prefix_len < 1 || prefix_len > src->len || prefix_len > prompt_len) return TQ4_ERR_ARG;
  } else if (prefix_len != 0) {
    return TQ4_ERR_ARG;
  }
  const int64_t shared = src ? prefix_len / kPage : 0;       // full pages mapped by reference
  const int64_t copied = (src && prefix_len % kPage) ? 1 : 0;
  const int64_t full = tq4_pages_reservation(prompt_len, out_budget);
  if (full < 0) return TQ4_ERR_ARG;
  const int64_t reserve = std::max<int64_t>(full - shared, 0);
  // the reservation must fit what nobody else holds; the copied page comes out of it
  // (or, if the reservation is zero, out of unreserved capacity)
  const int64_t need = std::max<int64_t>(reserve, copied);
  if (need > pp->available()) return TQ4_ERR_NO_PAGES;
  if (pp->next_id == INT32_MAX) return TQ4_ERR_ARG;   // request ids are never reused

  Request r;
  r.reserve = reserve;
  if (src) {
    for (int64_t i = 0; i < shared; ++i) {
      const int32_t id = src->pages[size_t(i)];
      pp->refs[size_t(id)] += 1;
      r.pages.push_back(id);
    }
    r.len = prefix_len;
  }
  int32_t cs = -1, cd = -1;
  if (copied) {
    cs = src->pages[size_t(shared)];
    cd = pp->take();
    r.pages.push_back(cd);
    r.own = 1;
  }
  const int32_t id = pp->next_id++;
  pp->reqs.emplace(id, std::move(r));
  *req_out = id;
  if (copy_src) *copy_src = cs;
  if (copy_dst) *copy_dst = cd;
  return TQ4_OK;
}

int tq4_pages_grow(tq4_pages* pp, int32_t req, int64_t new_len) {
  if (!pp) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  Request* r = pp->live(req);
  if (!r || new_len < r->len) return TQ4_ERR_ARG;
  const int64_t extra = pages_for(new_len) - int64_t(r->pages.size());
  if (extra > 0) {
    // pages inside the reservation are already set aside (counted out of "available");
    // the rest must be unreserved capacity
    const int64_t outside = tq4_pages::beyond_reserve(r->reserve, r->own, extra);
    if (outside > pp->available()) return TQ4_ERR_NO_PAGES;
    for (int64_t i = 0; i < extra; ++i) r->pages.push_back(pp->take());
    r->own += extra;
  }
  r->len = new_len;
  return TQ4_OK;
}

int tq4_pages_finish(tq4_pages* pp, int32_t req) {
  if (!pp) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  Request* r = pp->live(req);
  if (!r) return TQ4_ERR_ARG;
  r->leaving = true;
  return TQ4_OK;
}

int tq4_pages_step_boundary(tq4_pages* pp) {
  if (!pp) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  std::vector<int32_t> freed;
  for (auto it = pp->reqs.begin(); it != pp->reqs.end();) {
    if (!it->second.leaving) {
      ++it;
      continue;
    }
    for (int32_t id : it->second.pages)
      if (--pp->refs[size_t(id)] == 0) freed.push_back(id);
    it = pp->reqs.erase(it);
  }
  std::sort(freed.begin(), freed.end());
  for (int32_t id : freed) pp->free_list.push_back(id);
  return int(freed.size());
}

int tq4_pages_table(const tq4_pages* pp, int32_t req, int32_t* table, int32_t max_pages, int32_t* n_pages,
                    int64_t* len) {
  if (!pp || max_pages < 0 || (max_pages > 0 && !table)) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  auto it = pp->reqs.find(req);
  if (it == pp->reqs.end()) return TQ4_ERR_ARG;
  const Request& r = it->second;
  if (int64_t(r.pages.size()) > max_pages) return TQ4_ERR_ARG;
  for (int32_t i = 0; i < max_pages; ++i) table[i] = i < int32_t(r.pages.size()) ? r.pages[size_t(i)] : -1;
  if (n_pages) *n_pages = int32_t(r.pages.size());
  if (len) *len = r.len;
  return TQ4_OK;
}

int32_t tq4_pages_free_count(const tq4_pages* pp) {
  if (!pp) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  return int32_t(pp->free_list.size());
}

int32_t tq4_pages_available(const tq4_pages* pp) {
  if (!pp) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  return int32_t(pp->available());
}

int32_t tq4_pages_refcount(const tq4_pages* pp, int32_t page) {
  if (!pp || page < 0 || page >= pp->num_pages) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  return pp->refs[size_t(page)];
}

int32_t tq4_pages_free_list(const tq4_pages* pp, int32_t* out, int32_t cap) {
  if (!pp || cap < 0 || (cap > 0 && !out)) return TQ4_ERR_ARG;
  std::lock_guard<std::mutex> lock(pp->mu);
  int32_t i = 0;
  for (int32_t id : pp->free_list) {
    if (i < cap) out[i] = id;
    ++i;
  }
  return i;
}

}  // extern "C"
