"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

from hybrid_prefill_decode_pod_b200 import build as B
from hybrid_prefill_decode_pod_b200 import pod_attn as pa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "pod_attn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return pa.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"POD_API\s+[\w\s\*]*?\b(pod_attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("pod_attn_create", "pod_attn_hybrid", "pod_attn_prefill_only",
                 "pod_attn_decode_only", "pod_attn_destroy"):
        assert name in syms
    assert set(syms) == set(pa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(pa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), name


def test_library_is_built_for_sm100a():
    out = open(pa.LIB_PATH, "rb").read()
    assert b"sm_100a" in out or b"compute_100a" in out


def _cfg(**kw):
    base = dict(num_qo_heads=32, num_kv_heads=8, head_dim=128, kv_layout=0, page_size=0,
                max_prefill_reqs=1, max_prefill_tokens=512, max_decode_reqs=64,
                max_kv_tokens=8192, device=0, flags=0)
    base.update(kw)
    return pa.Config(*[base[k] for k, _ in pa.Config._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(num_kv_heads=3), pa.POD_EINVAL),            # H % Hk != 0
    (dict(num_qo_heads=0), pa.POD_EINVAL),
    (dict(head_dim=96), pa.POD_EUNSUPPORTED),
    (dict(head_dim=256), pa.POD_EUNSUPPORTED),
    (dict(num_qo_heads=32, num_kv_heads=2), pa.POD_EUNSUPPORTED),   # G = 16
    (dict(kv_layout=1, page_size=32), pa.POD_EUNSUPPORTED),
    (dict(kv_layout=7), pa.POD_EINVAL),
    (dict(max_prefill_reqs=17), pa.POD_ECAPACITY),
    (dict(max_kv_tokens=0), pa.POD_EINVAL),
    (dict(max_decode_reqs=-1), pa.POD_EINVAL),
])
def test_create_rejects_bad_config_on_host(lib, kw, code):
    h = ctypes.c_void_p()
    assert lib.pod_attn_create(ctypes.byref(h), ctypes.byref(_cfg(**kw))) == code
    assert not h.value


def test_null_arguments(lib):
    h = ctypes.c_void_p()
    assert lib.pod_attn_create(None, ctypes.byref(_cfg())) == pa.POD_EINVAL
    assert lib.pod_attn_create(ctypes.byref(h), None) == pa.POD_EINVAL
    assert lib.pod_attn_hybrid(None, None, None, 0, None) == pa.POD_EINVAL
    assert lib.pod_attn_prefill_only(None, None, None) == pa.POD_EINVAL
    assert lib.pod_attn_decode_only(None, None, None) == pa.POD_EINVAL
    assert lib.pod_attn_status(None, None) == pa.POD_EINVAL
    assert lib.pod_attn_destroy(None) == pa.POD_OK
    assert lib.pod_attn_strerror(pa.POD_ETIMEOUT) == b"device wait timed out"


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        pa._lib_backup = pa._lib
        try:
            pa._lib = None
            pa.load_library(str(tmp_path / "nope.so"))
        finally:
            pa._lib = pa._lib_backup


def test_static_decode_refuses_oversize_batches_on_host(lib):
    """pod_attn_decode_static checks its fixed array's limits before any CUDA
    call: more (request, KV head) pairs than its unit table holds, too many
    requests, too many KV heads."""
    ctx = (ctypes.c_int * 600)(*([100] * 600))
    a = pa.DecodeArgs()
    a.ctx_lens = ctypes.cast(ctx, ctypes.POINTER(ctypes.c_int))
    a.num_reqs = 300            # 300 x 16 KV heads = 4800 > 4096 units
    assert lib.pod_attn_decode_static(16, 16, 64, 0, ctypes.byref(a), None) == pa.POD_ECAPACITY
    a.num_reqs = 513            # more requests than the request table holds
    assert lib.pod_attn_decode_static(8, 2, 128, 0, ctypes.byref(a), None) == pa.POD_ECAPACITY
    a.num_reqs = 4              # 32 KV heads > 16
    assert lib.pod_attn_decode_static(32, 32, 128, 0, ctypes.byref(a), None) == pa.POD_ECAPACITY
    a.num_reqs = -1
    assert lib.pod_attn_decode_static(8, 2, 128, 0, ctypes.byref(a), None) == pa.POD_EINVAL
    assert lib.pod_attn_decode_static(8, 2, 96, 0, ctypes.byref(a), None) == pa.POD_EUNSUPPORTED
    assert lib.pod_attn_decode_static(8, 2, 128, 0, None, None) == pa.POD_EINVAL
