"""Python binding of the C ABI: argument marshalling only.

``PagedKVCache`` owns one ``svt_cache`` handle and the caller-side pool
tensor; every method forwards to the call of the same name in
include/svt.h with torch tensors turned into device pointers and the
current CUDA stream.  All computation happens in libsvt.so's kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib as L

_DTYPE_CODES = {"bf16": L.SVT_BF16, "fp16": L.SVT_FP16, "fp32": L.SVT_FP32}


class SvtError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{L.STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def _check(rc: int) -> None:
    if rc != 0:
        raise SvtError(rc, L.load().svt_last_error().decode())


def _torch():
    import torch
    return torch


def _stream_handle(stream=None) -> ctypes.c_void_p:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class PagedKVCache:
    """Handle on one paged KV cache (``svt_create_cache``)."""

    def __init__(self, max_pages: int, page_size: int, H: int, D: int, sliding_window: int,
                 scale_frames: int, *, num_blocks: int = 1, num_special: int = 6,
                 num_streams: int = 1, dtype: str = "bf16", patch_pages: int = 0,
                 max_qo_len: int = 0, max_splits: int = 16, rope_grid: int = 0,
                 rope_theta: float = 100.0, host_only: bool = False,
                 cross_frame_special: bool = True, device=None):
        self._lib = L.load()
        self._h = ctypes.c_void_p(0)
        self.max_pages, self.page_size, self.H, self.D = max_pages, page_size, H, D
        self.sliding_window, self.scale_frames = sliding_window, scale_frames
        self.num_blocks, self.num_special, self.num_streams = num_blocks, num_special, num_streams
        self.dtype = dtype
        self.host_only = host_only
        self.cross_frame_special = cross_frame_special
        # tokens per pool page: a frame's specials share its page without retention
        self.page_tokens = page_size + (0 if cross_frame_special else num_special)
        opts = L.CacheOpts()
        self._lib.svt_default_opts(ctypes.byref(opts))
        opts.num_blocks, opts.num_special, opts.num_streams = num_blocks, num_special, num_streams
        opts.dtype = _DTYPE_CODES[dtype]
        opts.patch_pages, opts.max_qo_len, opts.max_splits = patch_pages, max_qo_len, max_splits
        opts.rope_grid, opts.rope_theta, opts.host_only = rope_grid, rope_theta, int(host_only)
        opts.no_cross_frame_special = int(not cross_frame_special)
        self.pool = None
        if not host_only:
            torch = _torch()
            nbytes = self._lib.svt_pool_bytes(max_pages, page_size, H, D, ctypes.byref(opts))
            if nbytes == 0:
                raise SvtError(L.SVT_EINVAL, "bad pool shape")
            tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[dtype]
            self.pool = torch.zeros(
                (num_blocks, max_pages, 2, self.page_tokens, H, D), dtype=tdt,
                device=device if device is not None else "cuda")
            opts.pool = self.pool.data_ptr()
        _check(self._lib.svt_create_cache(max_pages, page_size, H, D, sliding_window,
                                          scale_frames, ctypes.byref(opts), ctypes.byref(self._h)))
        self.patch_pages = patch_pages or num_streams * (scale_frames + sliding_window + 1)

    # ----------------------------------------------------------- lifetime
    def close(self) -> None:
        if self._h:
            self._lib.svt_destroy_cache(self._h)
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ------------------------------------------------------ bookkeeping
    def reset(self) -> None:
        _check(self._lib.svt_reset(self._h))

    def set_free_lists(self, patch_ids, special_ids) -> None:
        a = np.ascontiguousarray(patch_ids, dtype=np.int32)
        b = np.ascontiguousarray(special_ids, dtype=np.int32)
        _check(self._lib.svt_set_free_lists(
            self._h, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(a),
            b.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(b)))

    def append_frame(self, block: int, k=None, v=None, stream: int = 0, cuda_stream=None) -> None:
        cs = ctypes.c_void_p(0) if self.host_only else _stream_handle(cuda_stream)
        _check(self._lib.svt_append_frame(self._h, block, stream, _ptr(k), _ptr(v), cs))

    def evict_frames(self, stream: int = 0) -> None:
        _check(self._lib.svt_evict_frames(self._h, stream))

    def set_defer_eviction(self, on: bool, stream: int = 0) -> None:
        _check(self._lib.svt_set_defer_eviction(self._h, stream, int(on)))

    def execute_deferred_eviction(self, stream: int = 0) -> None:
        _check(self._lib.svt_execute_deferred_eviction(self._h, stream))

    def rollback_last_frame(self, stream: int = 0) -> None:
        _check(self._lib.svt_rollback_last_frame(self._h, stream))

    def get_cache_stats(self, stream: int = 0) -> dict:
        st = L.Stats()
        _check(self._lib.svt_get_cache_stats(self._h, stream, ctypes.byref(st)))
        return {k: int(getattr(st, k)) for k, _ in L.Stats._fields_}

    # ----------------------------------------------------- page tables
    def _table_buffers(self):
        cap = self.num_streams * (self.scale_frames + self.sliding_window + 1) + self.max_pages
        ip = np.zeros(self.num_streams + 1, np.int32)
        ix = np.zeros(cap, np.int32)
        lp = np.zeros(self.num_streams, np.int32)
        n = ctypes.c_int(0)
        p32 = ctypes.POINTER(ctypes.c_int32)
        return ip, ix, lp, n, cap, [a.ctypes.data_as(p32) for a in (ip, ix, lp)]

    def build_visible_page_table(self, cuda_stream=None) -> None:
        cs = ctypes.c_void_p(0) if self.host_only else _stream_handle(cuda_stream)
        _check(self._lib.svt_build_visible_page_table(self._h, cs))

    def get_page_table(self):
        """Host view: (indptr, indices, last_page_len) numpy int32 arrays."""
        ip, ix, lp, n, cap, ptrs = self._table_buffers()
        _check(self._lib.svt_get_page_table(self._h, *ptrs, cap, ctypes.byref(n)))
        return ip, ix[:n.value].copy(), lp

    def read_device_page_table(self, cuda_stream=None):
        """Device table as written by the builder kernel (synchronises)."""
        ip, ix, lp, n, cap, ptrs = self._table_buffers()
        _check(self._lib.svt_read_device_page_table(self._h, *ptrs, cap, ctypes.byref(n),
                                                    _stream_handle(cuda_stream)))
        return ip, ix[:n.value].copy(), lp

    # ------------------------------------------------------- plan / run
    def plan(self, qo_len_per_stream, extra_len=None, cuda_stream=None) -> None:
        """``svt_plan``, or ``svt_plan_extra`` when ``extra_len`` (rows of a dense
        K/V segment per stream, attended without being stored) is given."""
        q = np.ascontiguousarray(qo_len_per_stream, dtype=np.int32)
        if len(q) != self.num_streams:
            raise ValueError("one qo_len per stream")
        cs = ctypes.c_void_p(0) if self.host_only else _stream_handle(cuda_stream)
        p32 = ctypes.POINTER(ctypes.c_int32)
        if extra_len is None:
            _check(self._lib.svt_plan(self._h, q.ctypes.data_as(p32), cs))
        else:
            x = np.ascontiguousarray(extra_len, dtype=np.int32)
            if len(x) != self.num_streams:
                raise ValueError("one extra_len per stream")
            _check(self._lib.svt_plan_extra(self._h, q.ctypes.data_as(p32), x.ctypes.data_as(p32),
                                            cs))

    def plan_info(self) -> dict:
        pi = L.PlanInfo()
        _check(self._lib.svt_get_plan_info(self._h, ctypes.byref(pi)))
        n = self.num_streams
        return {"num_items": pi.num_items, "splits": list(pi.splits[:n]),
                "kv_tiles": list(pi.kv_tiles[:n]), "kv_tokens": list(pi.kv_tokens[:n]),
                "qo_len": list(pi.qo_len[:n])}

    def run(self, block: int, q, out=None, lse=None, force_fp32: bool = False, cuda_stream=None,
            k_extra=None, v_extra=None):
        """Paged attention of ``block``; returns ``out`` ([rows, H, D]).  With
        ``k_extra``/``v_extra`` (``svt_run_extra``) the planned dense segments are
        attended after the pages."""
        torch = _torch()
        if out is None:
            fp32 = force_fp32 or self.dtype == "fp32"
            out = torch.empty(q.shape, dtype=torch.float32 if fp32 else q.dtype, device=q.device)
        if k_extra is None and v_extra is None:
            _check(self._lib.svt_run(self._h, block, _ptr(q), _ptr(out), _ptr(lse),
                                     int(force_fp32), _stream_handle(cuda_stream)))
        else:
            _check(self._lib.svt_run_extra(self._h, block, _ptr(q), _ptr(k_extra), _ptr(v_extra),
                                           _ptr(out), _ptr(lse), int(force_fp32),
                                           _stream_handle(cuda_stream)))
        return out

    def frame_step(self, ks, vs, qs, outs, stream: int = 0, use_graph: bool = True,
                   cuda_stream=None):
        """``svt_frame_step``: append the frame of every block, evict, build, plan
        and run every block in one call (one CUDA graph launch with
        ``use_graph``).  ``ks, vs, qs, outs``: one device tensor per block."""
        L_ = self.num_blocks
        if not (len(ks) == len(vs) == len(qs) == len(outs) == L_):
            raise ValueError("one k, v, q and out per block")
        arr = ctypes.c_void_p * L_
        ptrs = [arr(*[_ptr(t).value for t in xs]) for xs in (ks, vs, qs, outs)]
        _check(self._lib.svt_frame_step(self._h, stream, *ptrs, int(use_graph),
                                        _stream_handle(cuda_stream)))
        return outs

    def graph_counts(self):
        """(graphs built, graph replays) of ``frame_step``."""
        b, r = ctypes.c_int(0), ctypes.c_int(0)
        _check(self._lib.svt_get_graph_counts(self._h, ctypes.byref(b), ctypes.byref(r)))
        return b.value, r.value

    def device_error(self, cuda_stream=None) -> None:
        _check(self._lib.svt_device_error(self._h, _stream_handle(cuda_stream)))


def attention_noalloc(q, out, pool_block, indices, indptr, last_page_len, qo_len, max_pages,
                      page_size, lse=None, num_splits=0, cuda_stream=None) -> None:
    """``svt_attention_noalloc``: paged attention without any device allocation.

    q, out, lse, pool_block (one block's pool region) and indices are device
    tensors; indptr, last_page_len and qo_len are host sequences.
    """
    lib = L.load()
    H, D = q.shape[1], q.shape[2]
    dtype = {"torch.bfloat16": L.SVT_BF16, "torch.float16": L.SVT_FP16}[str(q.dtype)]
    p32 = ctypes.POINTER(ctypes.c_int32)
    ip = np.ascontiguousarray(indptr, dtype=np.int32)
    lp = np.ascontiguousarray(last_page_len, dtype=np.int32)
    ql = np.ascontiguousarray(qo_len, dtype=np.int32)
    if indices.dtype != _torch().int32:
        raise ValueError("indices must be int32")
    _check(lib.svt_attention_noalloc(
        _ptr(q), _ptr(out), _ptr(lse), _ptr(pool_block), _ptr(indices), ip.ctypes.data_as(p32),
        lp.ctypes.data_as(p32), ql.ctypes.data_as(p32), len(ql), max_pages, page_size, H, D,
        dtype, num_splits, _stream_handle(cuda_stream)))


def noalloc_device_error(cuda_stream=None) -> None:
    """``svt_noalloc_device_error``: synchronises, reads and clears the device
    error word of ``attention_noalloc``; raises SvtError(SVT_EDEVICE) if set."""
    _check(L.load().svt_noalloc_device_error(_stream_handle(cuda_stream)))


def selftest_wait_limit(limit_us: int, cuda_stream=None) -> None:
    """``svt_selftest_wait_limit``: raises SvtError(SVT_EDEVICE) when the bounded
    wait gave up at its limit, which is the expected outcome."""
    _check(L.load().svt_selftest_wait_limit(int(limit_us), _stream_handle(cuda_stream)))
