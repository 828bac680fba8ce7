"""Thin Python binding of libtq4.so (ctypes). Argument marshalling only.

Every function here forwards to the C ABI declared in include/tq4.h under the
same name; torch is used only to own device memory and to name the stream.
There is no fallback: if the shared library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq4.so")

TQ4_OK = 0
TQ4_ERR_ARG = -1
TQ4_ERR_UNSUPPORTED = -2
TQ4_ERR_PAGE_RANGE = -3
TQ4_ERR_CUDA = -4
TQ4_ERR_WORKSPACE = -5
TQ4_ERR_SEQ = -6
TQ4_ERR_TIMEOUT = -7
TQ4_ERR_NO_PAGES = -8

HEAD_DIM = 256
PAGE_POSITIONS = 256
KV_HEADS = 4
Q_HEADS = 24
PAGE_BYTES = 266240
POSITION_BYTES = 1040
INT8_PAGE_BYTES = 528384
TQB_PAGE_BYTES = {2: 135168, 3: 200704}   # the 2- and 3-bit variants
INT8_POSITION_BYTES = 2064

DTYPE_F32 = 0
DTYPE_BF16 = 1

DECODE_PATH_TENSOR_MEMORY = 0   # tcgen05 kernel for 2-4 query tokens
DECODE_PATH_WARP_MMA = 1        # warp-level mma.sync kernel (default)

EXPORTS = (
    "tq4_ctx_create", "tq4_ctx_destroy", "tq4_codebook", "tq4_encode_append", "tq4_reconstruct",
    "tq4_decode_workspace_bytes", "tq4_decode_attention", "tq4_prefill_workspace_bytes",
    "tq4_prefill_attention", "tq4_get_status", "tq4_status_string", "tq4_decode_attention_noalloc",
    "tq4_decode_append_attention", "tq4_ctx_set_wait_limit", "tq4_int8_encode_append", "tq4_int8_decode_attention",
    "tq4_decode_shared_workspace_bytes", "tq4_decode_attention_shared",
    "tq4_prefill_reconstructed_workspace_bytes", "tq4_prefill_attention_reconstructed",
    "tq4_ctx_set_decode_path", "tq4_tqb_codebook", "tq4_tqb_encode_append", "tq4_tqb_decode_attention",
    "tq4_tqb_decode_append_attention", "tq4_tqb_prefill_attention", "tq4_tqb_reconstruct",
    "tq4_tqb_decode_attention_shared",
    # host page pool (include/tq4_pages.h)
    "tq4_pages_create", "tq4_pages_destroy", "tq4_pages_reservation", "tq4_pages_admit", "tq4_pages_grow",
    "tq4_pages_finish", "tq4_pages_step_boundary", "tq4_pages_table", "tq4_pages_free_count",
    "tq4_pages_available", "tq4_pages_refcount", "tq4_pages_free_list",
)
NOALLOC_SCRATCH_BYTES = 8 << 20
DEFAULT_WAIT_POLLS = 1 << 24


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m compressed_paged_kv_tq4_b200.build`")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_f = ctypes.c_float

_sig = {
    "tq4_ctx_create": ([_p, ctypes.POINTER(_p)], ctypes.c_int),
    "tq4_ctx_destroy": ([_p], ctypes.c_int),
    "tq4_codebook": ([_p, _p, _p], ctypes.c_int),
    "tq4_encode_append": ([_p, _p, _i32, _p, _i32, _i32, _i32, _p, _p, ctypes.c_int, _p], ctypes.c_int),
    "tq4_reconstruct": ([_p, _p, _i32, _p, _i32, _i32, _i32, _p, _p, _p], ctypes.c_int),
    "tq4_decode_workspace_bytes": ([_p, _i32, _i32, _i64], _sz),
    "tq4_decode_attention": ([_p, _p, _i32, _p, _p, _i32, _p, _i32, _i32, _i64, _f, _p, ctypes.c_int,
                              _p, _sz, _p], ctypes.c_int),
    "tq4_prefill_workspace_bytes": ([_i32], _sz),
    "tq4_prefill_attention": ([_p, _p, _i32, _p, _i32, _i32, _p, _p, _p, _i32, _f, _p, ctypes.c_int, _p, _sz,
                               _p], ctypes.c_int),
    "tq4_ctx_set_wait_limit": ([_p, ctypes.c_uint32, ctypes.c_int], ctypes.c_int),
    "tq4_ctx_set_decode_path": ([_p, ctypes.c_int], ctypes.c_int),
    "tq4_tqb_codebook": ([_p, ctypes.c_int, _p, _p], ctypes.c_int),
    "tq4_tqb_encode_append": ([_p, ctypes.c_int, _p, _i32, _p, _i32, _i32, _i32, _p, _p, ctypes.c_int, _p],
                              ctypes.c_int),
    "tq4_tqb_decode_attention": ([_p, ctypes.c_int, _p, _i32, _p, _p, _i32, _p, _i32, _i32, _i64, _f, _p,
                                  ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_tqb_decode_attention_shared": ([_p, ctypes.c_int, _p, _i32, _p, _p, ctypes.c_int, _p, _p, _i32, _p, _i32,
                                         _i32, _i64, _p, _p, _f, _p, ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_tqb_reconstruct": ([_p, ctypes.c_int, _p, _i32, _p, _i32, _i32, _i32, _p, _p, _p], ctypes.c_int),
    "tq4_tqb_prefill_attention": ([_p, ctypes.c_int, _p, _i32, _p, _i32, _i32, _p, _p, _p, _i32, _f, _p,
                                   ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_tqb_decode_append_attention": ([_p, ctypes.c_int, _p, _i32, _p, _p, ctypes.c_int, _p, _p, _i32, _p, _i32,
                                         _i32, _i64, _f, _p, ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_int8_encode_append": ([_p, _p, _i32, _p, _i32, _i32, _i32, _p, _p, ctypes.c_int, _p], ctypes.c_int),
    "tq4_int8_decode_attention": ([_p, _p, _i32, _p, _p, _i32, _p, _i32, _i32, _i64, _f, _p, ctypes.c_int,
                                   _p, _sz, _p], ctypes.c_int),
    "tq4_get_status": ([_p, _p], ctypes.c_int),
    "tq4_decode_attention_noalloc": ([_p, _p, _i32, _p, _p, _i32, _p, _i32, _i32, _i64, _f, _p, ctypes.c_int, _p],
                                     ctypes.c_int),
    "tq4_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "tq4_decode_append_attention": ([_p, _p, _i32, _p, _p, ctypes.c_int, _p, _p, _i32, _p, _i32, _i32, _i64, _f,
                                     _p, ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_decode_shared_workspace_bytes": ([_p, _i32, _i32, _i64, _i32, _p, _p], _sz),
    "tq4_decode_attention_shared": ([_p, _p, _i32, _p, _p, ctypes.c_int, _p, _p, _i32, _p, _i32, _i32, _i64, _p, _p,
                                     _f, _p, ctypes.c_int, _p, _sz, _p], ctypes.c_int),
    "tq4_prefill_reconstructed_workspace_bytes": ([_i32, _i32], _sz),
    "tq4_prefill_attention_reconstructed": ([_p, _p, _i32, _p, _i32, _i32, _p, _p, _p, _i32, _f, _p, ctypes.c_int,
                                             _p, _sz, _p], ctypes.c_int),
    "tq4_pages_create": ([_i32, ctypes.POINTER(_p)], ctypes.c_int),
    "tq4_pages_destroy": ([_p], ctypes.c_int),
    "tq4_pages_reservation": ([_i64, _i64], _i64),
    "tq4_pages_admit": ([_p, _i64, _i64, _i32, _i64, ctypes.POINTER(_i32), ctypes.POINTER(_i32),
                         ctypes.POINTER(_i32)], ctypes.c_int),
    "tq4_pages_grow": ([_p, _i32, _i64], ctypes.c_int),
    "tq4_pages_finish": ([_p, _i32], ctypes.c_int),
    "tq4_pages_step_boundary": ([_p], ctypes.c_int),
    "tq4_pages_table": ([_p, _i32, _p, _i32, ctypes.POINTER(_i32), ctypes.POINTER(_i64)], ctypes.c_int),
    "tq4_pages_free_count": ([_p], _i32),
    "tq4_pages_available": ([_p], _i32),
    "tq4_pages_refcount": ([_p, _i32], _i32),
    "tq4_pages_free_list": ([_p, _p, _i32], _i32),
}
for _name, (_args, _res) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class TQ4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {tq4_status_string(code)} ({code})")
        self.code = code


def _check(code: int, what: str) -> int:
    if code != TQ4_OK:
        raise TQ4Error(code, what)
    return code


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------- raw ABI, same names
def tq4_status_string(code: int) -> str:
    return _lib.tq4_status_string(code).decode()


def tq4_ctx_create(signs) -> int:
    """signs: 256 values of +-1 (any int sequence / numpy array). Returns the context handle."""
    buf = (ctypes.c_int8 * 256)(*[int(s) for s in signs])
    out = _p()
    _check(_lib.tq4_ctx_create(ctypes.cast(buf, _p), ctypes.byref(out)), "tq4_ctx_create")
    return out.value


def tq4_ctx_destroy(ctx: int) -> None:
    _check(_lib.tq4_ctx_destroy(ctx), "tq4_ctx_destroy")


def tq4_codebook(ctx: int):
    c = (ctypes.c_double * 16)()
    b = (ctypes.c_double * 15)()
    _check(_lib.tq4_codebook(ctx, ctypes.cast(c, _p), ctypes.cast(b, _p)), "tq4_codebook")
    return list(c), list(b)


def tq4_encode_append(ctx, pool, num_pages, page_table, table_len, start_pos, n_tok, k_new, v_new,
                      dtype, stream=None) -> int:
    return _lib.tq4_encode_append(ctx, _ptr(pool), num_pages, _ptr(page_table), table_len, start_pos,
                                  n_tok, _ptr(k_new), _ptr(v_new), dtype, _stream(stream))


def tq4_reconstruct(ctx, pool, num_pages, page_table, table_len, start, n, k_out, v_out,
                    stream=None) -> int:
    return _lib.tq4_reconstruct(ctx, _ptr(pool), num_pages, _ptr(page_table), table_len, start, n,
                                _ptr(k_out), _ptr(v_out), _stream(stream))


def tq4_decode_workspace_bytes(ctx, n_req, n_q, total_seq_len) -> int:
    return _lib.tq4_decode_workspace_bytes(ctx, n_req, n_q, total_seq_len)


def tq4_decode_attention(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q,
                         total_seq_len, scale, out, out_dtype, workspace, workspace_bytes,
                         stream=None) -> int:
    return _lib.tq4_decode_attention(ctx, _ptr(pool), num_pages, _ptr(q), _ptr(page_tables), max_pages,
                                     _ptr(seq_lens), n_req, n_q, total_seq_len, scale, _ptr(out),
                                     out_dtype, _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_decode_append_attention(ctx, pool, num_pages, k_new, v_new, new_dtype, q, page_tables, max_pages,
                                seq_lens, n_req, n_q, total_seq_len, scale, out, out_dtype, workspace,
                                workspace_bytes, stream=None) -> int:
    return _lib.tq4_decode_append_attention(ctx, _ptr(pool), num_pages, _ptr(k_new), _ptr(v_new), new_dtype,
                                            _ptr(q), _ptr(page_tables), max_pages, _ptr(seq_lens), n_req, n_q,
                                            total_seq_len, scale, _ptr(out), out_dtype, _ptr(workspace),
                                            workspace_bytes, _stream(stream))


def _host_i32(a):
    """A host int32 array for the C ABI (kept alive by the caller)."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def tq4_decode_shared_workspace_bytes(ctx, n_req, n_q, total_seq_len, max_pages, prefix_leader, prefix_pages) -> int:
    ld, pg = _host_i32(prefix_leader), _host_i32(prefix_pages)
    return _lib.tq4_decode_shared_workspace_bytes(ctx, n_req, n_q, total_seq_len, max_pages, ld.ctypes.data,
                                                  pg.ctypes.data)


def tq4_decode_attention_shared(ctx, pool, num_pages, k_new, v_new, new_dtype, q, page_tables, max_pages, seq_lens,
                                n_req, n_q, total_seq_len, prefix_leader, prefix_pages, scale, out, out_dtype,
                                workspace, workspace_bytes, stream=None) -> int:
    ld, pg = _host_i32(prefix_leader), _host_i32(prefix_pages)
    return _lib.tq4_decode_attention_shared(ctx, _ptr(pool), num_pages, _ptr(k_new), _ptr(v_new), new_dtype,
                                            _ptr(q), _ptr(page_tables), max_pages, _ptr(seq_lens), n_req, n_q,
                                            total_seq_len, ld.ctypes.data, pg.ctypes.data, scale, _ptr(out),
                                            out_dtype, _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_prefill_workspace_bytes(n_tok) -> int:
    return _lib.tq4_prefill_workspace_bytes(n_tok)


def tq4_prefill_attention(ctx, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk, v_chunk,
                          n_tok, scale, out, out_dtype, workspace, workspace_bytes, stream=None) -> int:
    return _lib.tq4_prefill_attention(ctx, _ptr(pool), num_pages, _ptr(page_table), table_len, prefix_len,
                                      _ptr(q), _ptr(k_chunk), _ptr(v_chunk), n_tok, scale, _ptr(out), out_dtype,
                                      _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_prefill_reconstructed_workspace_bytes(prefix_len, n_tok) -> int:
    return _lib.tq4_prefill_reconstructed_workspace_bytes(prefix_len, n_tok)


def tq4_prefill_attention_reconstructed(ctx, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk,
                                        v_chunk, n_tok, scale, out, out_dtype, workspace, workspace_bytes,
                                        stream=None) -> int:
    return _lib.tq4_prefill_attention_reconstructed(ctx, _ptr(pool), num_pages, _ptr(page_table), table_len,
                                                    prefix_len, _ptr(q), _ptr(k_chunk), _ptr(v_chunk), n_tok, scale,
                                                    _ptr(out), out_dtype, _ptr(workspace), workspace_bytes,
                                                    _stream(stream))


def tq4_int8_encode_append(ctx, pool, num_pages, page_table, table_len, start_pos, n_tok, k_new, v_new,
                           dtype, stream=None) -> int:
    return _lib.tq4_int8_encode_append(ctx, _ptr(pool), num_pages, _ptr(page_table), table_len, start_pos,
                                       n_tok, _ptr(k_new), _ptr(v_new), dtype, _stream(stream))


def tq4_int8_decode_attention(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q,
                              total_seq_len, scale, out, out_dtype, workspace, workspace_bytes,
                              stream=None) -> int:
    return _lib.tq4_int8_decode_attention(ctx, _ptr(pool), num_pages, _ptr(q), _ptr(page_tables), max_pages,
                                          _ptr(seq_lens), n_req, n_q, total_seq_len, scale, _ptr(out),
                                          out_dtype, _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_tqb_codebook(ctx: int, bits: int):
    c = (ctypes.c_double * 8)()
    b = (ctypes.c_double * 7)()
    _check(_lib.tq4_tqb_codebook(ctx, bits, ctypes.cast(c, _p), ctypes.cast(b, _p)), "tq4_tqb_codebook")
    levels = 1 << bits
    return list(c)[:levels], list(b)[:levels - 1]


def tq4_tqb_encode_append(ctx, bits, pool, num_pages, page_table, table_len, start_pos, n_tok, k_new, v_new,
                          dtype, stream=None) -> int:
    return _lib.tq4_tqb_encode_append(ctx, bits, _ptr(pool), num_pages, _ptr(page_table), table_len, start_pos,
                                      n_tok, _ptr(k_new), _ptr(v_new), dtype, _stream(stream))


def tq4_tqb_decode_attention(ctx, bits, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q,
                             total_seq_len, scale, out, out_dtype, workspace, workspace_bytes, stream=None) -> int:
    return _lib.tq4_tqb_decode_attention(ctx, bits, _ptr(pool), num_pages, _ptr(q), _ptr(page_tables), max_pages,
                                         _ptr(seq_lens), n_req, n_q, total_seq_len, scale, _ptr(out), out_dtype,
                                         _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_tqb_decode_append_attention(ctx, bits, pool, num_pages, k_new, v_new, new_dtype, q, page_tables, max_pages,
                                    seq_lens, n_req, n_q, total_seq_len, scale, out, out_dtype, workspace,
                                    workspace_bytes, stream=None) -> int:
    return _lib.tq4_tqb_decode_append_attention(ctx, bits, _ptr(pool), num_pages, _ptr(k_new), _ptr(v_new),
                                                new_dtype, _ptr(q), _ptr(page_tables), max_pages, _ptr(seq_lens),
                                                n_req, n_q, total_seq_len, scale, _ptr(out), out_dtype,
                                                _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_tqb_decode_attention_shared(ctx, bits, pool, num_pages, k_new, v_new, new_dtype, q, page_tables, max_pages,
                                    seq_lens, n_req, n_q, total_seq_len, prefix_leader, prefix_pages, scale, out,
                                    out_dtype, workspace, workspace_bytes, stream=None) -> int:
    ld, pg = _host_i32(prefix_leader), _host_i32(prefix_pages)
    return _lib.tq4_tqb_decode_attention_shared(ctx, bits, _ptr(pool), num_pages, _ptr(k_new), _ptr(v_new),
                                                new_dtype, _ptr(q), _ptr(page_tables), max_pages, _ptr(seq_lens),
                                                n_req, n_q, total_seq_len, ld.ctypes.data, pg.ctypes.data, scale,
                                                _ptr(out), out_dtype, _ptr(workspace), workspace_bytes,
                                                _stream(stream))


def tq4_tqb_reconstruct(ctx, bits, pool, num_pages, page_table, table_len, start, n, k_out, v_out, stream=None) -> int:
    return _lib.tq4_tqb_reconstruct(ctx, bits, _ptr(pool), num_pages, _ptr(page_table), table_len, start, n,
                                    _ptr(k_out), _ptr(v_out), _stream(stream))


def tq4_tqb_prefill_attention(ctx, bits, pool, num_pages, page_table, table_len, prefix_len, q, k_chunk, v_chunk,
                              n_tok, scale, out, out_dtype, workspace, workspace_bytes, stream=None) -> int:
    return _lib.tq4_tqb_prefill_attention(ctx, bits, _ptr(pool), num_pages, _ptr(page_table), table_len, prefix_len,
                                          _ptr(q), _ptr(k_chunk), _ptr(v_chunk), n_tok, scale, _ptr(out), out_dtype,
                                          _ptr(workspace), workspace_bytes, _stream(stream))


def tq4_ctx_set_wait_limit(ctx, polls, withhold_signal=0) -> int:
    return _lib.tq4_ctx_set_wait_limit(ctx, polls, withhold_signal)


def tq4_ctx_set_decode_path(ctx, path) -> int:
    return _lib.tq4_ctx_set_decode_path(ctx, path)


def tq4_decode_attention_noalloc(ctx, pool, num_pages, q, page_tables, max_pages, seq_lens, n_req, n_q,
                                 total_seq_len, scale, out, out_dtype, stream=None) -> int:
    """Decode attention whose split-K scratch is the library's fixed device array
    (for callers that cannot allocate device memory; see include/tq4.h)."""
    return _lib.tq4_decode_attention_noalloc(ctx, _ptr(pool), num_pages, _ptr(q), _ptr(page_tables), max_pages,
                                             _ptr(seq_lens), n_req, n_q, total_seq_len, scale, _ptr(out),
                                             out_dtype, _stream(stream))


def tq4_get_status(ctx, stream=None) -> int:
    return _lib.tq4_get_status(ctx, _stream(stream))


# ---------------------------------------------------------------- host page pool (include/tq4_pages.h)
def tq4_pages_create(num_pages: int) -> int:
    out = _p()
    _check(_lib.tq4_pages_create(num_pages, ctypes.byref(out)), "tq4_pages_create")
    return out.value


def tq4_pages_destroy(pp: int) -> None:
    _check(_lib.tq4_pages_destroy(pp), "tq4_pages_destroy")


def tq4_pages_reservation(prompt_len: int, out_budget: int) -> int:
    return _lib.tq4_pages_reservation(prompt_len, out_budget)


def tq4_pages_admit(pp, prompt_len, out_budget, src_req=-1, prefix_len=0):
    """Returns (status, request id, copy_src, copy_dst); the id is -1 unless status is TQ4_OK."""
    req, cs, cd = _i32(-1), _i32(-1), _i32(-1)
    rc = _lib.tq4_pages_admit(pp, prompt_len, out_budget, src_req, prefix_len, ctypes.byref(req),
                              ctypes.byref(cs), ctypes.byref(cd))
    return rc, (req.value if rc == TQ4_OK else -1), cs.value, cd.value


def tq4_pages_grow(pp, req, new_len) -> int:
    return _lib.tq4_pages_grow(pp, req, new_len)


def tq4_pages_finish(pp, req) -> int:
    return _lib.tq4_pages_finish(pp, req)


def tq4_pages_step_boundary(pp) -> int:
    return _lib.tq4_pages_step_boundary(pp)


def tq4_pages_table(pp, req, max_pages):
    """Returns (status, page-table row as a list of max_pages ids padded with -1, length)."""
    row = (_i32 * max(max_pages, 1))()
    n, ln = _i32(0), _i64(0)
    rc = _lib.tq4_pages_table(pp, req, ctypes.cast(row, _p), max_pages, ctypes.byref(n), ctypes.byref(ln))
    return rc, list(row)[:max_pages], ln.value


def tq4_pages_free_count(pp) -> int:
    return _lib.tq4_pages_free_count(pp)


def tq4_pages_available(pp) -> int:
    return _lib.tq4_pages_available(pp)


def tq4_pages_refcount(pp, page) -> int:
    return _lib.tq4_pages_refcount(pp, page)


def tq4_pages_free_list(pp):
    n = _lib.tq4_pages_free_list(pp, None, 0)
    buf = (_i32 * max(n, 1))()
    _lib.tq4_pages_free_list(pp, ctypes.cast(buf, _p), n)
    return list(buf)[:n]


class PagePool:
    """Owns a tq4_pages handle (host page pool; no GPU involved)."""

    def __init__(self, num_pages: int):
        self.num_pages = num_pages
        self.handle = tq4_pages_create(num_pages)

    def __del__(self, _destroy=_lib.tq4_pages_destroy):   # bound early: safe at interpreter exit
        if getattr(self, "handle", None):
            _destroy(self.handle)
            self.handle = None

    def admit(self, prompt_len, out_budget, src_req=-1, prefix_len=0):
        return tq4_pages_admit(self.handle, prompt_len, out_budget, src_req, prefix_len)

    def grow(self, req, new_len):
        return tq4_pages_grow(self.handle, req, new_len)

    def finish(self, req):
        return tq4_pages_finish(self.handle, req)

    def step_boundary(self):
        return tq4_pages_step_boundary(self.handle)

    def table(self, req, max_pages):
        return tq4_pages_table(self.handle, req, max_pages)

    def free_count(self):
        return tq4_pages_free_count(self.handle)

    def available(self):
        return tq4_pages_available(self.handle)

    def refcount(self, page):
        return tq4_pages_refcount(self.handle, page)

    def free_list(self):
        return tq4_pages_free_list(self.handle)


# ---------------------------------------------------------------- tensor-level helpers
def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("TQ4 kernels take CUDA tensors")


class Context:
    """Owns a tq4_ctx for the current device."""

    def __init__(self, signs):
        self.handle = tq4_ctx_create(signs)

    def close(self):
        if self.handle:
            tq4_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def codebook(self):
        return tq4_codebook(self.handle)

    def status(self, stream=None) -> int:
        return tq4_get_status(self.handle, stream)

    def set_wait_limit(self, polls: int, withhold_signal: bool = False) -> None:
        """Polls a bounded device wait makes before it gives up (0 = the default);
        withhold_signal makes later calls withhold one producer signal (testing)."""
        _check(tq4_ctx_set_wait_limit(self.handle, polls, int(withhold_signal)), "tq4_ctx_set_wait_limit")

    def set_decode_path(self, path: int) -> None:
        """Kernel for 2-4 query tokens: DECODE_PATH_TENSOR_MEMORY or DECODE_PATH_WARP_MMA (default)."""
        _check(tq4_ctx_set_decode_path(self.handle, path), "tq4_ctx_set_decode_path")

    # -- pool helpers
    @staticmethod
    def new_pool(num_pages: int, device="cuda") -> torch.Tensor:
        return torch.zeros(num_pages * PAGE_BYTES, dtype=torch.uint8, device=device)

    def encode_append(self, pool, page_table, start_pos, k_new, v_new, stream=None):
        _need_cuda(pool, page_table, k_new, v_new)
        dtype = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
        if dtype is None or v_new.dtype != k_new.dtype:
            raise ValueError("k_new/v_new must both be float32 or bfloat16")
        n_tok = k_new.shape[0]
        _check(tq4_encode_append(self.handle, pool, pool.numel() // PAGE_BYTES, page_table,
                                 page_table.numel(), start_pos, n_tok, k_new, v_new, dtype, stream),
               "tq4_encode_append")

    def reconstruct(self, pool, page_table, start, n, stream=None):
        _need_cuda(pool, page_table)
        k = torch.empty((n, KV_HEADS, HEAD_DIM), dtype=torch.float32, device=pool.device)
        v = torch.empty_like(k)
        _check(tq4_reconstruct(self.handle, pool, pool.numel() // PAGE_BYTES, page_table, page_table.numel(),
                               start, n, k, v, stream), "tq4_reconstruct")
        return k, v

    def decode_workspace(self, n_req, n_q, total_seq_len, device="cuda") -> torch.Tensor:
        nbytes = tq4_decode_workspace_bytes(self.handle, n_req, n_q, total_seq_len)
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)

    def decode_attention(self, pool, q, page_tables, seq_lens, total_seq_len, scale, out=None,
                         out_dtype=torch.bfloat16, workspace=None, stream=None):
        """q: bf16 [n_req, n_q, 24, 256]; page_tables int32 [n_req, max_pages]; seq_lens int32 [n_req]."""
        _need_cuda(pool, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            workspace = self.decode_workspace(n_req, n_q, total_seq_len, q.device)
        _check(tq4_decode_attention(self.handle, pool, pool.numel() // PAGE_BYTES, q, page_tables,
                                    page_tables.shape[1], seq_lens, n_req, n_q, total_seq_len, scale, out,
                                    od, workspace, workspace.numel(), stream), "tq4_decode_attention")
        return out

    def decode_append_attention(self, pool, k_new, v_new, q, page_tables, seq_lens, total_seq_len, scale,
                                out=None, out_dtype=torch.bfloat16, workspace=None, stream=None):
        """Append k_new/v_new [n_req, n_q, 4, 256] (float32 or bfloat16) at the last n_q
        positions of each request, then decode as decode_attention."""
        _need_cuda(pool, k_new, v_new, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        nd = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
        if nd is None or v_new.dtype != k_new.dtype:
            raise ValueError("k_new/v_new must both be float32 or bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        if tuple(k_new.shape) != (n_req, n_q, KV_HEADS, HEAD_DIM) or k_new.shape != v_new.shape:
            raise ValueError("k_new/v_new must be [n_req, n_q, 4, 256]")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            workspace = self.decode_workspace(n_req, n_q, total_seq_len, q.device)
        _check(tq4_decode_append_attention(self.handle, pool, pool.numel() // PAGE_BYTES, k_new, v_new, nd, q,
                                           page_tables, page_tables.shape[1], seq_lens, n_req, n_q,
                                           total_seq_len, scale, out, od, workspace, workspace.numel(), stream),
               "tq4_decode_append_attention")
        return out

    def decode_attention_shared(self, pool, q, page_tables, seq_lens, total_seq_len, scale, prefix_leader,
                                prefix_pages, k_new=None, v_new=None, out=None, out_dtype=torch.bfloat16,
                                workspace=None, stream=None):
        """decode_attention (with the append of k_new/v_new when given) for requests that
        share leading pages: prefix_leader / prefix_pages are host int sequences [n_req]."""
        _need_cuda(pool, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        nd = DTYPE_F32
        if k_new is not None:
            _need_cuda(k_new, v_new)
            nd = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
            if nd is None or v_new.dtype != k_new.dtype or tuple(k_new.shape) != (n_req, n_q, KV_HEADS, HEAD_DIM):
                raise ValueError("k_new/v_new must be float32 or bfloat16 [n_req, n_q, 4, 256]")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        max_pages = page_tables.shape[1]
        if workspace is None:
            nbytes = tq4_decode_shared_workspace_bytes(self.handle, n_req, n_q, total_seq_len, max_pages,
                                                       prefix_leader, prefix_pages)
            if nbytes == 0:
                raise TQ4Error(TQ4_ERR_ARG, "tq4_decode_shared_workspace_bytes")
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        _check(tq4_decode_attention_shared(self.handle, pool, pool.numel() // PAGE_BYTES, k_new, v_new, nd, q,
                                           page_tables, max_pages, seq_lens, n_req, n_q, total_seq_len,
                                           prefix_leader, prefix_pages, scale, out, od, workspace,
                                           workspace.numel(), stream), "tq4_decode_attention_shared")
        return out

    def tqb_decode_attention_shared(self, bits, pool, q, page_tables, seq_lens, total_seq_len, scale, prefix_leader,
                                    prefix_pages, k_new=None, v_new=None, out=None, out_dtype=torch.bfloat16,
                                    workspace=None, stream=None):
        """decode_attention_shared over a 2- or 3-bit pool."""
        _need_cuda(pool, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        nd = DTYPE_F32
        if k_new is not None:
            _need_cuda(k_new, v_new)
            nd = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
            if nd is None or v_new.dtype != k_new.dtype or tuple(k_new.shape) != (n_req, n_q, KV_HEADS, HEAD_DIM):
                raise ValueError("k_new/v_new must be float32 or bfloat16 [n_req, n_q, 4, 256]")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        max_pages = page_tables.shape[1]
        if workspace is None:
            nbytes = tq4_decode_shared_workspace_bytes(self.handle, n_req, n_q, total_seq_len, max_pages,
                                                       prefix_leader, prefix_pages)
            if nbytes == 0:
                raise TQ4Error(TQ4_ERR_ARG, "tq4_decode_shared_workspace_bytes")
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        _check(tq4_tqb_decode_attention_shared(self.handle, bits, pool, pool.numel() // TQB_PAGE_BYTES[bits], k_new,
                                               v_new, nd, q, page_tables, max_pages, seq_lens, n_req, n_q,
                                               total_seq_len, prefix_leader, prefix_pages, scale, out, od,
                                               workspace, workspace.numel(), stream),
               "tq4_tqb_decode_attention_shared")
        return out

    # -- the uniform INT8 comparison arm
    @staticmethod
    def new_int8_pool(num_pages: int, device="cuda") -> torch.Tensor:
        return torch.zeros(num_pages * INT8_PAGE_BYTES, dtype=torch.uint8, device=device)

    def int8_encode_append(self, pool, page_table, start_pos, k_new, v_new, stream=None):
        _need_cuda(pool, page_table, k_new, v_new)
        dtype = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
        if dtype is None or v_new.dtype != k_new.dtype:
            raise ValueError("k_new/v_new must both be float32 or bfloat16")
        _check(tq4_int8_encode_append(self.handle, pool, pool.numel() // INT8_PAGE_BYTES, page_table,
                                      page_table.numel(), start_pos, k_new.shape[0], k_new, v_new, dtype, stream),
               "tq4_int8_encode_append")

    def int8_decode_attention(self, pool, q, page_tables, seq_lens, total_seq_len, scale, out=None,
                              out_dtype=torch.bfloat16, workspace=None, stream=None):
        _need_cuda(pool, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            workspace = self.decode_workspace(n_req, n_q, total_seq_len, q.device)
        _check(tq4_int8_decode_attention(self.handle, pool, pool.numel() // INT8_PAGE_BYTES, q, page_tables,
                                         page_tables.shape[1], seq_lens, n_req, n_q, total_seq_len, scale, out,
                                         od, workspace, workspace.numel(), stream), "tq4_int8_decode_attention")
        return out

    # -- the 2- and 3-bit variants
    @staticmethod
    def new_tqb_pool(bits: int, num_pages: int, device="cuda") -> torch.Tensor:
        return torch.zeros(num_pages * TQB_PAGE_BYTES[bits], dtype=torch.uint8, device=device)

    def tqb_codebook(self, bits: int):
        return tq4_tqb_codebook(self.handle, bits)

    def tqb_encode_append(self, bits, pool, page_table, start_pos, k_new, v_new, stream=None):
        _need_cuda(pool, page_table, k_new, v_new)
        dtype = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
        if dtype is None or v_new.dtype != k_new.dtype:
            raise ValueError("k_new/v_new must both be float32 or bfloat16")
        _check(tq4_tqb_encode_append(self.handle, bits, pool, pool.numel() // TQB_PAGE_BYTES[bits], page_table,
                                     page_table.numel(), start_pos, k_new.shape[0], k_new, v_new, dtype, stream),
               "tq4_tqb_encode_append")

    def tqb_decode_attention(self, bits, pool, q, page_tables, seq_lens, total_seq_len, scale, out=None,
                             out_dtype=torch.bfloat16, workspace=None, stream=None):
        _need_cuda(pool, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            workspace = self.decode_workspace(n_req, n_q, total_seq_len, q.device)
        _check(tq4_tqb_decode_attention(self.handle, bits, pool, pool.numel() // TQB_PAGE_BYTES[bits], q,
                                        page_tables, page_tables.shape[1], seq_lens, n_req, n_q, total_seq_len,
                                        scale, out, od, workspace, workspace.numel(), stream),
               "tq4_tqb_decode_attention")
        return out

    def tqb_decode_append_attention(self, bits, pool, k_new, v_new, q, page_tables, seq_lens, total_seq_len, scale,
                                    out=None, out_dtype=torch.bfloat16, workspace=None, stream=None):
        """decode_append_attention for a b-bit pool: k_new/v_new [n_req, n_q, 4, 256]
        (float32 or bfloat16) encoded at the last n_q positions, then the decode."""
        _need_cuda(pool, k_new, v_new, q, page_tables, seq_lens)
        if q.dtype != torch.bfloat16:
            raise ValueError("q must be bfloat16")
        nd = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(k_new.dtype)
        if nd is None or v_new.dtype != k_new.dtype:
            raise ValueError("k_new/v_new must both be float32 or bfloat16")
        n_req, n_q = q.shape[0], q.shape[1]
        if tuple(k_new.shape) != (n_req, n_q, KV_HEADS, HEAD_DIM) or k_new.shape != v_new.shape:
            raise ValueError("k_new/v_new must be [n_req, n_q, 4, 256]")
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            workspace = self.decode_workspace(n_req, n_q, total_seq_len, q.device)
        _check(tq4_tqb_decode_append_attention(self.handle, bits, pool, pool.numel() // TQB_PAGE_BYTES[bits], k_new,
                                               v_new, nd, q, page_tables, page_tables.shape[1], seq_lens, n_req,
                                               n_q, total_seq_len, scale, out, od, workspace, workspace.numel(),
                                               stream),
               "tq4_tqb_decode_append_attention")
        return out

    def prefill_attention(self, pool, page_table, prefix_len, q, k_chunk, v_chunk, scale, out=None,
                          out_dtype=torch.bfloat16, workspace=None, stream=None, reconstruct=False):
        """q: bf16 [n_tok, 24, 256]; k_chunk/v_chunk bf16 [n_tok, 4, 256]; out bf16 or float32.
        reconstruct=True: the direct-inverse-reconstruction variant (the prefix rebuilt as
        dense rows first)."""
        _need_cuda(q, k_chunk, v_chunk)
        n_tok = q.shape[0]
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            nbytes = (tq4_prefill_reconstructed_workspace_bytes(prefix_len, n_tok) if reconstruct
                      else tq4_prefill_workspace_bytes(n_tok))
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
        num_pages = pool.numel() // PAGE_BYTES if pool is not None else 0
        tlen = page_table.numel() if page_table is not None else 0
        fn = tq4_prefill_attention_reconstructed if reconstruct else tq4_prefill_attention
        _check(fn(self.handle, pool, num_pages, page_table, tlen, prefix_len, q, k_chunk, v_chunk, n_tok, scale, out,
                  od, workspace, workspace.numel(), stream), fn.__name__)
        return out

    def tqb_reconstruct(self, bits, pool, page_table, start, n, stream=None):
        _need_cuda(pool, page_table)
        k = torch.empty((n, KV_HEADS, HEAD_DIM), dtype=torch.float32, device=pool.device)
        v = torch.empty_like(k)
        _check(tq4_tqb_reconstruct(self.handle, bits, pool, pool.numel() // TQB_PAGE_BYTES[bits], page_table,
                                   page_table.numel(), start, n, k, v, stream), "tq4_tqb_reconstruct")
        return k, v

    def tqb_prefill_attention(self, bits, pool, page_table, prefix_len, q, k_chunk, v_chunk, scale, out=None,
                              out_dtype=torch.bfloat16, workspace=None, stream=None):
        """prefill_attention over a 2- or 3-bit pool (the prefix rebuilt as dense rows first)."""
        _need_cuda(q, k_chunk, v_chunk)
        n_tok = q.shape[0]
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        od = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
        if workspace is None:
            nbytes = tq4_prefill_reconstructed_workspace_bytes(prefix_len, n_tok)
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
        num_pages = pool.numel() // TQB_PAGE_BYTES[bits] if pool is not None else 0
        tlen = page_table.numel() if page_table is not None else 0
        _check(tq4_tqb_prefill_attention(self.handle, bits, pool, num_pages, page_table, tlen, prefix_len, q, k_chunk,
                                         v_chunk, n_tok, scale, out, od, workspace, workspace.numel(), stream),
               "tq4_tqb_prefill_attention")
        return out
