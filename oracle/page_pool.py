"""Oracle model of the host page pool (plain Python lists and dicts).

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports this module;
only ``tests/`` call it. It shares no code with the library's page pool
(``csrc/tq4_pages.cpp``); the tests drive both with the same operation
sequences and compare every observable result.

Where each rule comes from (simpleprog.com, "Fitting a 27B-Parameter LLM into
24 GiB of Laptop Memory"):

[STATE]   section "StateTrans: Request Transitions at Safe Boundaries":
          admission reserves physical-page equivalents equal to the ceiling of
          (prompt length + min(output budget, 8,192)) / 256; shared prefixes are
          reference counted; on completion or cancellation the step finishes
          first and the page references are decremented after it; a page id goes
          back to the free list only when its count reaches zero after that
          boundary.
[REUSE]   section "Prefix Reuse: Making Long Context Practical": a request with a
          cached prefix restores it and prefills only the remainder.

Readings where the page is silent (the same ones the library's header states):
 * the free list is first-in first-out, starts as 0..N-1, and the pages freed at
   one boundary join its tail in ascending id order;
 * a request of length L maps ceil(L / 256) pages;
 * admission reserves R - (pages shared by a restored prefix); a request's own
   pages draw on its reservation first; capacity "available" to others is the
   free pages minus the unused reservations of live requests; a reservation or a
   growth beyond one must fit in it, else the call fails and changes nothing;
 * a restored prefix shares its full pages; a partial last page is copied into a
   fresh page of the new request (the source may still write its later slots);
 * finishing releases the unused reservation at once and the page references at
   the next step boundary.

Status values mirror the library's: 0 ok, -1 bad argument, -8 no capacity.
"""
from __future__ import annotations

OK, ERR_ARG, ERR_NO_PAGES = 0, -1, -8
PAGE = 256
GUARANTEED_OUTPUT = 8192


def reservation(prompt_len: int, out_budget: int) -> int:
    """[STATE]: ceil((prompt + min(output budget, 8192)) / 256) page equivalents."""
    if prompt_len < 0 or out_budget < 0 or prompt_len > 2 ** 53:
        return -1
    total = prompt_len + min(out_budget, GUARANTEED_OUTPUT)
    return -(-total // PAGE)


class PagePoolModel:
    def __init__(self, num_pages: int):
        assert num_pages >= 1
        self.num_pages = num_pages
        self.refs = [0] * num_pages
        self.free = list(range(num_pages))
        self.reqs = {}          # id -> dict(pages, len, reserve, own, leaving)
        self.next_id = 0

    # ------------------------------------------------------------ queries
    def unused_reserve(self, r) -> int:
        if r["leaving"]:
            return 0
        return max(r["reserve"] - r["own"], 0)

    def available(self) -> int:
        return len(self.free) - sum(self.unused_reserve(r) for r in self.reqs.values())

    def free_count(self) -> int:
        return len(self.free)

    def refcount(self, page: int) -> int:
        return self.refs[page] if 0 <= page < self.num_pages else ERR_ARG

    def free_list(self):
        return list(self.free)

    def table(self, req: int, max_pages: int):
        r = self.reqs.get(req)
        if r is None or len(r["pages"]) > max_pages:
            return ERR_ARG, None, None
        return OK, r["pages"] + [-1] * (max_pages - len(r["pages"])), r["len"]

    def _live(self, req):
        r = self.reqs.get(req)
        return None if (r is None or r["leaving"]) else r

    def _take(self) -> int:
        page = self.free.pop(0)
        self.refs[page] = 1
        return page

    # ------------------------------------------------------------ transitions
    def admit(self, prompt_len, out_budget, src_req=-1, prefix_len=0):
        """Returns (status, request id, copy_src, copy_dst)."""
        if prompt_len < 0 or out_budget < 0 or prefix_len < 0:
            return ERR_ARG, -1, -1, -1
        src = None
        if src_req >= 0:
            src = self._live(src_req)
            if src is None or prefix_len < 1 or prefix_len > src["len"] or prefix_len > prompt_len:
                return ERR_ARG, -1, -1, -1
        elif prefix_len != 0:
            return ERR_ARG, -1, -1, -1
        full = reservation(prompt_len, out_budget)
        if full < 0:
            return ERR_ARG, -1, -1, -1
        shared = prefix_len // PAGE if src is not None else 0
        copied = 1 if (src is not None and prefix_len % PAGE) else 0
        reserve = max(full - shared, 0)
        if max(reserve, copied) > self.available():
            return ERR_NO_PAGES, -1, -1, -1
        pages = []
        for i in range(shared):                      # [STATE]: shared prefix pages, counted
            self.refs[src["pages"][i]] += 1
            pages.append(src["pages"][i])
        cs = cd = -1
        own = 0
        if copied:                                    # partial last page: a private copy
            cs = src["pages"][shared]
            cd = self._take()
            pages.append(cd)
            own = 1
        rid = self.next_id
        self.next_id += 1
        self.reqs[rid] = {"pages": pages, "len": prefix_len if src is not None else 0,
                          "reserve": reserve, "own": own, "leaving": False}
        return OK, rid, cs, cd

    def grow(self, req, new_len):
        r = self._live(req)
        if r is None or new_len < r["len"]:
            return ERR_ARG
        extra = -(-new_len // PAGE) - len(r["pages"])
        if extra > 0:
            inside = max(min(r["reserve"] - r["own"], extra), 0)
            if extra - inside > self.available():
                return ERR_NO_PAGES
            for _ in range(extra):
                r["pages"].append(self._take())
            r["own"] += extra
        r["len"] = new_len
        return OK

    def finish(self, req):
        r = self._live(req)
        if r is None:
            return ERR_ARG
        r["leaving"] = True
        return OK

    def step_boundary(self):
        """[STATE]: after the step, drop the leaving requests' references; pages at
        zero go back to the free list."""
        freed = []
        for rid in sorted(self.reqs):
            r = self.reqs[rid]
            if not r["leaving"]:
                continue
            for page in r["pages"]:
                self.refs[page] -= 1
                if self.refs[page] == 0:
                    freed.append(page)
            del self.reqs[rid]
        for page in sorted(freed):
            self.free.append(page)
        return len(freed)
