"""The C-ABI library builds for sm_100a, loads, exports every function that
include/twilight.h declares, and rejects bad arguments on the host before
touching the GPU (these calls run without a GPU)."""
import ctypes

import pytest

from adaptive_top_sparse_quest_b200 import _capi, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _capi.load()


def test_exports_every_declared_function(lib):
    names = _capi.header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(_capi._SIGS) <= set(names)


def test_status_strings(lib):
    for s in range(6):
        assert lib.tw_status_string(s).decode().startswith("TW_")
    assert lib.tw_version() >= 100


def _kv(**kw):
    s = _capi.TwKv()
    s.k = 4096
    s.v = 8192
    s.batch = 1
    s.num_kv_heads = 2
    s.max_seq_len = 64
    s.page_size = 16
    s.head_dim = 128
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def test_workspace_size_checks(lib):
    n = ctypes.c_size_t(0)
    assert lib.tw_workspace_size(1, 4, 2, 1024, 512, ctypes.byref(n)) == _capi.TW_OK
    assert n.value > 0 and n.value % 256 == 0
    assert lib.tw_workspace_size(1, 3, 2, 1024, 512, ctypes.byref(n)) == _capi.TW_ERR_INVALID_ARG
    assert lib.tw_workspace_size(1, 6, 2, 1024, 512, ctypes.byref(n)) == _capi.TW_ERR_UNSUPPORTED
    assert lib.tw_workspace_size(1, 4, 2, 1024, 0, ctypes.byref(n)) == _capi.TW_ERR_INVALID_ARG
    assert lib.tw_workspace_size(1, 4, 2, 1024, 512, None) == _capi.TW_ERR_INVALID_ARG


def test_kv_descriptor_checks(lib):
    out = 1 << 20
    assert lib.tw_quantize_keys(None, out, out, out, None) == _capi.TW_ERR_INVALID_ARG
    assert lib.tw_quantize_keys(ctypes.byref(_kv(head_dim=64)), out, out, out, None) == \
        _capi.TW_ERR_UNSUPPORTED
    assert lib.tw_quantize_keys(ctypes.byref(_kv(page_size=32)), out, out, out, None) == \
        _capi.TW_ERR_UNSUPPORTED
    assert lib.tw_quantize_keys(ctypes.byref(_kv(k=4100)), out, out, out, None) == \
        _capi.TW_ERR_INVALID_ARG                      # misaligned K
    assert lib.tw_quantize_keys(ctypes.byref(_kv()), None, out, out, None) == \
        _capi.TW_ERR_INVALID_ARG
    # paged: max_seq_len must equal max_pages_per_seq * 16
    bad = _kv(page_table=1 << 16, max_pages_per_seq=3, num_pool_pages=8, max_seq_len=64)
    assert lib.tw_page_meta(ctypes.byref(bad), out, None) == _capi.TW_ERR_INVALID_ARG
    # empty batch: nothing to launch, success without a device
    assert lib.tw_quantize_keys(ctypes.byref(_kv(batch=0)), out, out, out, None) == _capi.TW_OK
    # key-cache width: 0 (read as 4), 4 or 2; anything else is unsupported
    for bits in (0, 2, 4):
        assert lib.tw_quantize_keys(ctypes.byref(_kv(batch=0, key_bits=bits)), out, out, out,
                                    None) == _capi.TW_OK
    for bits in (1, 3, 8, -4):
        assert lib.tw_quantize_keys(ctypes.byref(_kv(batch=0, key_bits=bits)), out, out, out,
                                    None) == _capi.TW_ERR_UNSUPPORTED
        assert lib.tw_append_keys(ctypes.byref(_kv(batch=0, key_bits=bits)), out, out, out, out,
                                  None) == _capi.TW_ERR_UNSUPPORTED


def test_host_staged_step_argument_checks(lib):
    # null host buffers or a null step: rejected before any device work
    assert lib.tw_decode_step_host(None, 1 << 20, 1 << 20, None) == _capi.TW_ERR_INVALID_ARG
    st = _capi.TwStep()
    assert lib.tw_decode_step_host(ctypes.byref(st), None, 1 << 20, None) == \
        _capi.TW_ERR_INVALID_ARG
    assert lib.tw_decode_step_host(ctypes.byref(st), 1 << 20, None, None) == \
        _capi.TW_ERR_INVALID_ARG


def test_struct_layout_matches_header():
    """The ctypes mirror of tw_kv ends with key_bits, after head_dim."""
    names = [f[0] for f in _capi.TwKv._fields_]
    assert names[-2:] == ["head_dim", "key_bits"]
    text = open(_capi.HEADER).read()
    body = text[text.index("typedef struct tw_kv {"):text.index("} tw_kv;")]
    import re
    fields = re.findall(r"\b([a-z_]+);", re.sub(r"/\*.*?\*/", "", body, flags=re.S))
    assert fields == names


def test_topp_and_select_argument_checks(lib):
    kv = _kv()
    p = 1 << 20
    args = lambda **o: dict(dict(q=p, Hq=4, codes=p, scales=p, zeros=p, cand=None, stride=0,
                                 ncand=None, pp=0.85, gm=1, idx=p, cap=64, count=p), **o)

    def topp(a):
        return lib.tw_topp_prune(a["q"], a["Hq"], ctypes.byref(kv), a["codes"], a["scales"],
                                 a["zeros"], a["cand"], a["stride"], a["ncand"], a["pp"], a["gm"],
                                 a["idx"], a["cap"], a["count"], None, 0, None)
    assert topp(args(pp=0.0)) == _capi.TW_ERR_INVALID_ARG
    assert topp(args(pp=1.5)) == _capi.TW_ERR_INVALID_ARG
    assert topp(args(pp=float("nan"))) == _capi.TW_ERR_INVALID_ARG
    assert topp(args(gm=2)) == _capi.TW_ERR_INVALID_ARG
    assert topp(args(cap=63)) == _capi.TW_ERR_CAPACITY        # 64 candidates, capacity 63
    assert topp(args(Hq=3)) == _capi.TW_ERR_INVALID_ARG
    assert topp(args(Hq=32)) == _capi.TW_ERR_UNSUPPORTED      # G = 16
    # with candidate pages the bound is min(stride, pages) * 16
    assert topp(args(cand=p, ncand=p, stride=2, cap=31)) == _capi.TW_ERR_CAPACITY
    # workspace missing
    assert topp(args()) == _capi.TW_ERR_INVALID_ARG
    sel = lambda budget, stride: lib.tw_select_pages(p, 4, ctypes.byref(kv), p, budget, p, stride,
                                                     p, None, 0, None)
    assert sel(15, 4) == _capi.TW_ERR_INVALID_ARG              # budget below one page
    assert sel(64, 3) == _capi.TW_ERR_CAPACITY                 # 4 pages do not fit stride 3
    assert sel(64, 4) == _capi.TW_ERR_INVALID_ARG              # no workspace


def test_candidates_limit(lib):
    kv = _kv(max_seq_len=131072 + 16)
    p = 1 << 20
    r = lib.tw_topp_prune(p, 2, ctypes.byref(kv), p, p, p, None, 0, None, 0.9, 1, p,
                          131072 + 16, p, None, 0, None)
    assert r == _capi.TW_ERR_UNSUPPORTED


def test_product_package_does_not_import_oracle():
    import os
    import re
    pkg = os.path.dirname(_capi.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), f


def test_bounded_wait_selftest_argument_checks(lib):
    assert lib.tw_selftest_bounded_wait(None, None) == _capi.TW_ERR_INVALID_ARG
    assert lib.tw_selftest_bounded_wait(ctypes.c_void_p(2), None) == _capi.TW_ERR_INVALID_ARG
