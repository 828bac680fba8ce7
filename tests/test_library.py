"""The C ABI without a GPU: libtq4.so loads, exports every function the headers in
include/ declare, the Python binding names exactly those, and the host-only parts
(status strings, workspace sizes, argument checks that return before any CUDA
call) behave as the header states."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq4.h")
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))

tq4 = pytest.importorskip("compressed_paged_kv_tq4_b200.tq4")


def header_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", " ", open(h).read(), flags=re.S)   # drop comments
        names |= set(re.findall(r"\b(tq4_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def header_defines():
    return dict((m.group(1), int(m.group(2))) for m in
                re.finditer(r"#define\s+(TQ4_[A-Z0-9_]+)\s+\(?(-?\d+)", open(HEADER).read()))


def test_header_declares_the_calls():
    assert [os.path.basename(h) for h in HEADERS] == ["tq4.h", "tq4_pages.h"]
    names = header_functions()
    for required in ("tq4_encode_append", "tq4_decode_attention", "tq4_prefill_attention",
                     "tq4_decode_append_attention", "tq4_reconstruct", "tq4_get_status"):
        assert required in names


def test_library_exports_every_header_function():
    lib = ctypes.CDLL(tq4.LIB_PATH)
    missing = [n for n in header_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_header():
    assert sorted(tq4.EXPORTS) == header_functions()
    for n in header_functions():
        assert callable(getattr(tq4, n)), n


def test_constants_match_header():
    d = header_defines()
    assert d["TQ4_PAGE_BYTES"] == tq4.PAGE_BYTES == 266240
    assert d["TQ4_POSITION_BYTES"] == tq4.POSITION_BYTES == 1040
    assert d["TQ4_DTYPE_F32"] == tq4.DTYPE_F32 and d["TQ4_DTYPE_BF16"] == tq4.DTYPE_BF16
    for name in ("TQ4_OK", "TQ4_ERR_ARG", "TQ4_ERR_PAGE_RANGE", "TQ4_ERR_WORKSPACE", "TQ4_ERR_SEQ",
                 "TQ4_ERR_TIMEOUT", "TQ4_ERR_NO_PAGES"):
        assert getattr(tq4, name) == d[name]


def test_status_strings():
    d = header_defines()
    seen = set()
    for name, code in d.items():
        if name == "TQ4_OK" or name.startswith("TQ4_ERR_"):
            s = tq4.tq4_status_string(code)
            assert isinstance(s, str) and s and s != "unknown status", name
            seen.add(s)
    assert len(seen) == sum(1 for n in d if n == "TQ4_OK" or n.startswith("TQ4_ERR_"))
    assert tq4.tq4_status_string(12345) == "unknown status"


def test_workspace_sizes_are_host_arithmetic():
    assert tq4.tq4_prefill_workspace_bytes(0) == 0
    # q' hi + lo ([n][24][256] f16 each) and the rotated chunk K, V as hi + lo ([n][4][256] f16 each)
    # rotated q' and chunk rows (hi + lo f16), then room for up to 3 KV segments of
    # partial rows per 256-row block and KV head: 256 x (256 fp32 + (m, l))
    assert tq4.tq4_prefill_workspace_bytes(2048) == 2048 * (2 * 24 + 4 * 4) * 256 * 2 + 48 * 3 * 4 * 256 * (1024 + 8)
    assert (tq4.tq4_prefill_reconstructed_workspace_bytes(32768, 2048)
            == tq4.tq4_prefill_workspace_bytes(2048) + 32768 * 4 * 4 * 256 * 2)
    assert tq4.tq4_decode_workspace_bytes(None, 1, 1, 32768) == 0   # no context: no plan


def test_argument_errors_return_before_any_launch():
    """Calls made straight on the library (NULL stream): each returns TQ4_ERR_ARG from its host checks."""
    lib, E = tq4._lib, tq4.TQ4_ERR_ARG
    assert lib.tq4_ctx_destroy(None) == tq4.TQ4_OK          # NULL is accepted
    assert lib.tq4_encode_append(None, None, 0, None, 0, 0, 1, None, None, 0, None) == E
    assert lib.tq4_decode_attention(None, None, 0, None, None, 0, None, 1, 1, 1, 0.0625, None, 1, None, 0,
                                    None) == E
    assert lib.tq4_decode_append_attention(None, None, 0, None, None, 0, None, None, 0, None, 1, 1, 1, 0.0625,
                                           None, 1, None, 0, None) == E
    assert lib.tq4_prefill_attention(None, None, 0, None, 0, 0, None, None, None, 1, 0.0625, None, 1, None, 0,
                                     None) == E
    assert lib.tq4_ctx_set_wait_limit(None, 4, 0) == E
    assert lib.tq4_ctx_set_decode_path(None, 0) == E
    assert lib.tq4_tqb_codebook(None, 2, None, None) == E
    assert lib.tq4_tqb_encode_append(None, 2, None, 0, None, 0, 0, 1, None, None, 1, None) == E
    assert lib.tq4_tqb_decode_attention(None, 3, None, 0, None, None, 0, None, 1, 1, 1, 0.0625, None, 1, None, 0,
                                        None) == E
    assert lib.tq4_tqb_reconstruct(None, 3, None, 0, None, 0, 0, 1, None, None, None) == E
    assert lib.tq4_tqb_decode_attention_shared(None, 2, None, 0, None, None, 1, None, None, 0, None, 1, 1, 1, None,
                                               None, 0.0625, None, 1, None, 0, None) == E
    assert lib.tq4_tqb_prefill_attention(None, 2, None, 0, None, 0, 0, None, None, None, 1, 0.0625, None, 1, None, 0,
                                         None) == E
    assert lib.tq4_tqb_decode_append_attention(None, 2, None, 0, None, None, 1, None, None, 0, None, 1, 1, 1, 0.0625,
                                               None, 1, None, 0, None) == E
    assert lib.tq4_reconstruct(None, None, 0, None, 0, 0, 1, None, None, None) == E
    assert lib.tq4_get_status(None, None) == E
