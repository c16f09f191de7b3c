"""The C ABI without a GPU: libpagedkv.so builds, loads, exports every
function include/pagedkv.h declares, and rejects bad arguments before any CUDA
call (so none of these tests launches anything)."""
import ctypes
import os
import re

import pytest

from paged_kv_decode_31_b200 import binding
from paged_kv_decode_31_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def header_macros():
    return dict((k, int(v)) for k, v in re.findall(r"#define\s+(PKV_\w+)\s+(-?\d+)", open(HEADER).read()))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"pkv_kv_append", "pkv_paged_decode_attn", "pkv_paged_prefill_attn",
            "pkv_workspace_size", "pkv_strerror"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in pagedkv.h but not exported"


def test_constants_agree_with_header(lib):
    m = header_macros()
    assert lib.pkv_split_tokens() == m["PKV_SPLIT_TOKENS"] == binding.SPLIT_TOKENS
    assert m["PKV_TILE_TOKENS"] == binding.TILE_TOKENS
    assert m["PKV_DEVERR_BAD_BLOCK"] == binding.DEVERR_BAD_BLOCK
    assert m["PKV_DEVERR_TABLE_WIDTH"] == binding.DEVERR_TABLE_WIDTH
    assert m["PKV_DEVERR_TIMEOUT"] == binding.DEVERR_TIMEOUT
    assert m["PKV_DEVERR_QUERY_LEN"] == binding.DEVERR_QUERY_LEN
    assert m["PKV_DEVERR_SEQ_LEN"] == binding.DEVERR_SEQ_LEN


def test_strerror_covers_every_status(lib):
    m = header_macros()
    for key in ("PKV_OK", "PKV_ERR_ARG", "PKV_ERR_WORKSPACE", "PKV_ERR_CUDA", "PKV_ERR_LAYOUT"):
        s = binding.strerror(m[key])
        assert s and s != "unknown pagedkv status"
    assert binding.strerror(12345) == "unknown pagedkv status"


def test_workspace_size_formula(lib):
    # fp32 acc[D] per (row, split), padded to 256 B, then (m, l) per (row, split)
    rows, S, D = 4 * 1 * 32, 131072 // 4096, 128
    acc = rows * S * D * 4
    acc = (acc + 255) // 256 * 256
    assert binding.workspace_size(4, 1, 32, 128, 131072) == acc + rows * S * 2 * 4
    assert binding.workspace_size(1, 1, 1, 64, 0) == 256 + 8
    assert binding.workspace_size(0, 1, 1, 64, 10) == 0


def _attn_args(**over):
    """Arguments of pkv_paged_decode_attn with plausible (never dereferenced)
    pointers; `over` replaces fields by name."""
    st = (ctypes.c_int64 * 3)(2048, 2048, 128)
    kst = (ctypes.c_int64 * 3)(16 * 8 * 128, 8 * 128, 128)
    ost = (ctypes.c_int64 * 3)(4096, 4096, 128)
    a = dict(q=0x10000, q_st=st, k=0x20000, k_st=kst, v=0x30000, v_st=kst, num_blocks=64,
             table=0x40000, bt_stride=16, max_blocks=16, seqlens=0x50000, max_seqlen_k=256,
             batch=2, sq=1, Hq=32, Hkv=8, D=128, bs=16, scale=0.088, causal=0,
             out=0x60000, o_st=ost, lse=0x70000, ws=0x80000, ws_bytes=1 << 30, err=None,
             stream=None)
    a.update(over)
    return list(a.values())


@pytest.mark.parametrize("over", [
    dict(D=96), dict(Hq=30), dict(bs=24), dict(bs=8), dict(bs=512), dict(batch=0),
    dict(sq=0), dict(num_blocks=0), dict(max_blocks=0), dict(bt_stride=4),
    dict(q=0x10008), dict(k=0x20002), dict(scale=0.0), dict(scale=float("nan")),
    dict(q=None), dict(max_seqlen_k=-1),
    dict(k_st=(ctypes.c_int64 * 3)(16 * 8 * 128, 8 * 128, 100)),
])
def test_invalid_arguments_rejected_before_any_launch(lib, over):
    rc = lib.pkv_paged_decode_attn(*_attn_args(**over))
    assert rc == header_macros()["PKV_ERR_ARG"]
    rc = lib.pkv_paged_prefill_attn(*_attn_args(**over))
    assert rc == header_macros()["PKV_ERR_ARG"]


def test_small_workspace_rejected_before_any_launch(lib):
    rc = lib.pkv_paged_decode_attn(*_attn_args(ws_bytes=100))
    assert rc == header_macros()["PKV_ERR_WORKSPACE"]
    rc = lib.pkv_paged_decode_attn(*_attn_args(ws=None))
    assert rc == header_macros()["PKV_ERR_WORKSPACE"]


def test_kv_append_rejects_bad_arguments(lib):
    st = (ctypes.c_int64 * 3)(1024, 1024, 128)
    kst = (ctypes.c_int64 * 3)(16 * 8 * 128, 8 * 128, 128)
    good = [0x10000, st, 0x20000, st, 0x30000, kst, 0x40000, kst, 64, 0x50000, 16, 16,
            0x60000, 2, 1, 8, 128, 16, None, None]
    for idx, bad in ((16, 96), (17, 20), (13, 0), (14, -1), (8, 0), (0, 0x10004)):
        args = list(good)
        args[idx] = bad
        assert lib.pkv_kv_append(*args) == header_macros()["PKV_ERR_ARG"], (idx, bad)
    args = list(good)
    args[14] = 0                                     # n_new = 0: nothing to do
    assert lib.pkv_kv_append(*args) == 0


def test_product_path_has_no_cpu_fallback():
    """The binding loads only the CUDA library; it never imports the oracle."""
    import paged_kv_decode_31_b200 as pkg
    pkg_dir = os.path.dirname(pkg.__file__)
    for fn in os.listdir(pkg_dir):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg_dir, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn


def test_packed_cp_and_backward_sizes(lib):
    m = header_macros()
    assert m["PKV_DEVERR_QUERY_LEN"] == binding.DEVERR_QUERY_LEN
    # packed queries: the dense formula with one sequence of total_q tokens
    assert binding.varlen_workspace_size(3632, 32, 128, 16384) == \
        binding.workspace_size(1, 3632, 32, 128, 16384)
    assert binding.varlen_workspace_size(0, 32, 128, 100) == 0
    # one CP rank's partial block: the dense formula over its local splits
    assert binding.partials_size(4, 1, 32, 128, 8) == binding.workspace_size(4, 1, 32, 128, 8 * 4096)
    assert binding.partials_size(4, 1, 32, 128, 0) == 0
    # backward: two fp32 per row, each array padded to 256 bytes
    lib.pkv_bwd_workspace_size.argtypes = [ctypes.c_int] * 3
    lib.pkv_bwd_workspace_size.restype = ctypes.c_size_t
    rows = 8 * 2048 * 16
    assert lib.pkv_bwd_workspace_size(8, 2048, 16) == 2 * ((rows * 4 + 255) // 256 * 256)
    assert lib.pkv_bwd_workspace_size(0, 1, 1) == 0


def test_packed_entry_points_reject_bad_arguments(lib):
    E = header_macros()
    st2 = (ctypes.c_int64 * 2)(4096, 128)
    kst = (ctypes.c_int64 * 3)(16 * 8 * 128, 8 * 128, 128)

    def varlen(**over):
        a = dict(q=0x10000, q_st=st2, cu=0x90000, total_q=100, max_q=40, k=0x20000, k_st=kst,
                 v=0x30000, v_st=kst, num_blocks=64, table=0x40000, bt_stride=16,
                 max_blocks=16, seqlens=0x50000, max_seqlen_k=256, batch=2, Hq=32, Hkv=8,
                 D=128, bs=16, scale=0.088, causal=1, out=0x60000, o_st=st2, lse=0x70000,
                 fo=None, fo_st=None, fl=None, ws=0x80000, ws_bytes=1 << 30, err=None,
                 stream=None)
        a.update(over)
        return lib.pkv_paged_varlen_attn(*a.values())

    for over in (dict(total_q=0), dict(max_q=0), dict(cu=None), dict(q_st=None), dict(D=96),
                 dict(Hq=30), dict(fo=0xA0000)):  # final_out without final_lse / strides
        assert varlen(**over) == E["PKV_ERR_ARG"], over
    assert varlen(ws_bytes=64) == E["PKV_ERR_WORKSPACE"]

    st = (ctypes.c_int64 * 3)(2048, 2048, 128)
    fn = lib.pkv_paged_attn_partials
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                   ctypes.c_int64, ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 6 + \
                  [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                   ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int

    def partials(begin=0, n_local=2, pbytes=1 << 30, D=128):
        return fn(0x10000, st, 0x20000, kst, 0x30000, kst, 64, 0x40000, 16, 16, 0x50000,
                  2, 1, 32, 8, D, 16, 0.088, 0, begin, n_local, 0x80000, pbytes, None, None)

    assert partials(n_local=0) == E["PKV_ERR_ARG"]
    assert partials(begin=-1) == E["PKV_ERR_ARG"]
    assert partials(D=96) == E["PKV_ERR_ARG"]
    assert partials(pbytes=64) == E["PKV_ERR_WORKSPACE"]

    mg = lib.pkv_merge_partials
    mg.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_size_t,
                   ctypes.c_void_p] + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4
    mg.restype = ctypes.c_int
    need = binding.partials_size(2, 1, 32, 128, 2)
    assert mg(None, 2, 2, need, 0x50000, 2, 1, 32, 128, 0, 0x60000, st, 0x70000, None) == E["PKV_ERR_ARG"]
    assert mg(0x80000, 0, 2, need, 0x50000, 2, 1, 32, 128, 0, 0x60000, st, 0x70000, None) == E["PKV_ERR_ARG"]
    assert mg(0x80000, 2, 2, need - 16, 0x50000, 2, 1, 32, 128, 0, 0x60000, st, 0x70000,
              None) == E["PKV_ERR_WORKSPACE"]


def test_backward_and_packed_append_reject_bad_arguments(lib):
    E = header_macros()
    st = (ctypes.c_int64 * 3)(2048, 2048, 128)
    kst = (ctypes.c_int64 * 3)(16 * 8 * 128, 8 * 128, 128)
    bw = lib.pkv_paged_prefill_attn_bwd
    bw.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                   ctypes.c_int64, ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 7 + \
                  [ctypes.c_float, ctypes.c_int] + [ctypes.c_void_p] * 12 + \
                  [ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    bw.restype = ctypes.c_int

    def bwd(D=128, Hq=32, dout=0xB0000, ws_bytes=1 << 30):
        return bw(0x10000, st, 0x20000, kst, 0x30000, kst, 64, 0x40000, 16, 16, 0x50000, 256,
                  2, 16, Hq, 8, D, 16, 0.088, 1, 0x60000, st, 0x70000, dout, st, 0xC0000, st,
                  0xD0000, kst, 0xE0000, kst, 0x80000, ws_bytes, None, None)

    assert bwd(D=96) == E["PKV_ERR_ARG"]
    assert bwd(Hq=30) == E["PKV_ERR_ARG"]
    assert bwd(dout=None) == E["PKV_ERR_ARG"]
    assert bwd(ws_bytes=16) == E["PKV_ERR_WORKSPACE"]

    ap = lib.pkv_kv_append_varlen
    ap.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] + [ctypes.c_void_p] * 4 + \
                  [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                   ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    ap.restype = ctypes.c_int
    st2 = (ctypes.c_int64 * 2)(1024, 128)

    def app(cu=0x90000, total=10, D=128):
        return ap(0x10000, st2, 0x20000, st2, cu, total, 0x30000, kst, 0x40000, kst, 64,
                  0x50000, 16, 16, 0x60000, 2, 8, D, 16, None, None)

    assert app(cu=None) == E["PKV_ERR_ARG"]
    assert app(D=96) == E["PKV_ERR_ARG"]
    assert app(total=-1) == E["PKV_ERR_ARG"]
    assert app(total=0) == 0   # nothing to append: no launch


def test_debug_wait_limit_above_the_default_is_rejected_before_any_cuda_call(lib):
    # the debug entry point may only lower the 2 s limit of every pipeline wait
    fn = lib.pkv_debug_paged_decode_attn
    fn.argtypes = binding._ATTN_ARGS + [ctypes.c_uint64]
    fn.restype = ctypes.c_int
    assert fn(*_attn_args(), 2_000_000_001) == header_macros()["PKV_ERR_ARG"]
    # and it checks every other argument like pkv_paged_decode_attn
    assert fn(*_attn_args(D=96), 0) == header_macros()["PKV_ERR_ARG"]
    assert fn(*_attn_args(ws_bytes=100), 0) == header_macros()["PKV_ERR_WORKSPACE"]


def test_debug_final_out_checks_its_arguments_before_any_cuda_call(lib):
    fn = lib.pkv_debug_final_out
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    E = header_macros()
    assert fn(None, None, None, -1, None) == E["PKV_ERR_ARG"]
    assert fn(None, None, None, 4, None) == E["PKV_ERR_ARG"]
    assert fn(None, None, None, 0, None) == 0  # nothing to do: no launch
