"""Test-only model of the page allocator (predicts physical page ids).

The pages fix the two-stream policy but not which physical page a frame
gets.  The reading used: patch pages 0..patch_pages-1
and special pages patch_pages..max_pages-1 sit in two FIFO free lists handed
out from the front; evicted window pages go to the back; a rolled-back frame
returns its pages to the front.  This model restates that policy in plain
Python so that the library's tables can be checked bit for bit.

Without cross-frame special retention each frame's special tokens sit after
its patch tokens in the frame's own page (page_size + num_special tokens), so
no special pages are used, eviction drops a frame's specials with its patches,
and every visible page is full.
"""
from collections import deque


class StreamModel:
    def __init__(self):
        self.scale, self.window, self.special = [], deque(), []
        self.special_tokens = 0
        self.frame_count = 0
        self.defer = False
        self.prov = None          # (was_scale, n_new_special)


class AllocModel:
    def __init__(self, max_pages, P, ns, S, W, num_streams=1, patch_pages=0,
                 cross_frame_special=True):
        self.max_pages, self.P, self.ns, self.S, self.W = max_pages, P, ns, S, W
        self.cross = cross_frame_special
        self.patch_pages = patch_pages or num_streams * (S + W + 1)
        self.patch_free = deque(range(self.patch_pages))
        self.special_free = deque(range(self.patch_pages, max_pages))
        self.st = [StreamModel() for _ in range(num_streams)]

    def append(self, s):
        st = self.st[s]
        assert st.prov is None and len(st.window) <= self.W
        n0 = st.special_tokens
        last_pg = (n0 + self.ns - 1) // self.P if self.ns else -1
        n_new = max(0, last_pg + 1 - len(st.special)) if self.cross else 0
        if not self.patch_free or len(self.special_free) < n_new:
            raise MemoryError
        page = self.patch_free.popleft()
        for _ in range(n_new):
            st.special.append(self.special_free.popleft())
        was_scale = len(st.scale) < self.S
        (st.scale if was_scale else st.window).append(page)
        st.special_tokens += self.ns
        st.frame_count += 1
        st.prov = (was_scale, n_new) if st.defer else None
        return page

    def evict(self, s):
        st = self.st[s]
        if st.prov is not None:
            return
        while len(st.window) > self.W:
            self.patch_free.append(st.window.popleft())
            if not self.cross:
                st.special_tokens -= self.ns

    def accept(self, s):
        st = self.st[s]
        assert st.prov is not None
        st.prov = None
        self.evict(s)

    def rollback(self, s):
        st = self.st[s]
        was_scale, n_new = st.prov
        for _ in range(n_new):
            self.special_free.appendleft(st.special.pop())
        page = st.scale.pop() if was_scale else st.window.pop()
        self.patch_free.appendleft(page)
        st.special_tokens -= self.ns
        st.frame_count -= 1
        st.prov = None

    def table(self):
        indptr, indices, lpl = [0], [], []
        for st in self.st:
            indices += st.scale + list(st.window) + st.special
            indptr.append(len(indices))
            if st.special:
                lpl.append((st.special_tokens - 1) % self.P + 1)
            elif st.scale or st.window:
                lpl.append(self.P if self.cross else self.P + self.ns)
            else:
                lpl.append(0)
        return indptr, indices, lpl

    def stats(self, s):
        st = self.st[s]
        return {"frame_count": st.frame_count, "scale_pages": len(st.scale),
                "live_pages": len(st.window), "free_pages": len(self.patch_free),
                "special_tokens": st.special_tokens}
