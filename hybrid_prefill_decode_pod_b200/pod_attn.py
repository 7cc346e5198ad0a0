"""ctypes binding over libpod_attn.so (argument marshalling only).

Every step of the attention runs in the library's CUDA kernels; this module
turns torch tensors into the device pointers, host length arrays and stream
handle the C ABI (``include/pod_attn.h``) takes, and raises on a non-zero
status. PyTorch is used only to own device memory and streams.

There is no fallback: if ``libpod_attn.so`` is missing or fails to load,
importing :class:`PodAttention` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpod_attn.so")

POD_OK = 0
POD_EINVAL = -1
POD_EUNSUPPORTED = -2
POD_ENOMEM = -3
POD_ECUDA = -4
POD_ETIMEOUT = -5
POD_ECAPACITY = -6

POD_KV_CONTIGUOUS = 0
POD_KV_PAGED = 1

MODE_FUSED = 0
MODE_SERIAL = 1
MODE_TWO_STREAM = 2
MODES = {"fused": MODE_FUSED, "serial": MODE_SERIAL, "two_stream": MODE_TWO_STREAM}

FLAG_STATS = 0x1
FLAG_TEST_FORCE_TIMEOUT = 0x2

# Every symbol include/pod_attn.h declares.
EXPORTED = ("pod_attn_create", "pod_attn_hybrid", "pod_attn_prefill_only",
            "pod_attn_decode_only", "pod_attn_status", "pod_attn_last_plan",
            "pod_attn_get_stats", "pod_attn_destroy", "pod_attn_decode_static",
            "pod_attn_strerror")


class PodError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (what, strerror(code), code))


class Config(ctypes.Structure):
    _fields_ = [("num_qo_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("kv_layout", ctypes.c_int),
                ("page_size", ctypes.c_int), ("max_prefill_reqs", ctypes.c_int),
                ("max_prefill_tokens", ctypes.c_int), ("max_decode_reqs", ctypes.c_int),
                ("max_kv_tokens", ctypes.c_longlong), ("device", ctypes.c_int),
                ("flags", ctypes.c_uint)]


class PrefillArgs(ctypes.Structure):
    _fields_ = [("num_reqs", ctypes.c_int), ("chunk_lens", ctypes.POINTER(ctypes.c_int)),
                ("prior_lens", ctypes.POINTER(ctypes.c_int)), ("q", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("k_ptrs", ctypes.POINTER(ctypes.c_void_p)),
                ("v_ptrs", ctypes.POINTER(ctypes.c_void_p)), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("block_table_stride", ctypes.c_int), ("pool_blocks", ctypes.c_longlong)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("num_reqs", ctypes.c_int), ("ctx_lens", ctypes.POINTER(ctypes.c_int)),
                ("q", ctypes.c_void_p), ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("k_ptrs", ctypes.POINTER(ctypes.c_void_p)),
                ("v_ptrs", ctypes.POINTER(ctypes.c_void_p)), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("block_table_stride", ctypes.c_int), ("pool_blocks", ctypes.c_longlong)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int), ("slots_per_sm", ctypes.c_int),
                ("prefill_units", ctypes.c_int), ("prefill_split", ctypes.c_int),
                ("decode_units", ctypes.c_int), ("decode_split_len", ctypes.c_int),
                ("ratio_num", ctypes.c_int), ("ratio_den", ctypes.c_int),
                ("plan_bytes", ctypes.c_longlong), ("prefill_sm_cap", ctypes.c_int),
                ("pair_clusters", ctypes.c_int)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class Stats(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int), ("prefill_claims", ctypes.c_longlong),
                ("decode_claims", ctypes.c_longlong), ("sms_with_both", ctypes.c_int)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpod_attn.so (raises if it is missing: no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libpod_attn.so is not built (%s); run "
                           "`python -m hybrid_prefill_decode_pod_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.pod_attn_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(Config)]
    lib.pod_attn_hybrid.argtypes = [vp, ctypes.POINTER(PrefillArgs), ctypes.POINTER(DecodeArgs), i, vp]
    lib.pod_attn_prefill_only.argtypes = [vp, ctypes.POINTER(PrefillArgs), vp]
    lib.pod_attn_decode_only.argtypes = [vp, ctypes.POINTER(DecodeArgs), vp]
    lib.pod_attn_status.argtypes = [vp, vp]
    lib.pod_attn_last_plan.argtypes = [vp, ctypes.POINTER(PlanInfo)]
    lib.pod_attn_get_stats.argtypes = [vp, vp, ctypes.POINTER(Stats)]
    lib.pod_attn_destroy.argtypes = [vp]
    lib.pod_attn_decode_static.argtypes = [i, i, i, i, ctypes.POINTER(DecodeArgs), vp]
    lib.pod_attn_strerror.argtypes = [i]
    lib.pod_attn_strerror.restype = ctypes.c_char_p
    for name in EXPORTED:
        if name != "pod_attn_strerror":
            getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def strerror(code: int) -> str:
    try:
        return load_library().pod_attn_strerror(int(code)).decode()
    except Exception:  # pragma: no cover
        return "status %d" % code


def _int_array(xs: Sequence[int]):
    arr = (ctypes.c_int * max(1, len(xs)))(*[int(x) for x in xs])
    return arr


def _ptr_array(ts):
    return (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])


def _dptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class PodAttention:
    """One library context (``pod_attn_create`` ... ``pod_attn_destroy``)."""

    def __init__(self, num_qo_heads: int, num_kv_heads: int, head_dim: int, *,
                 paged: bool = False, max_prefill_reqs: int = 16,
                 max_prefill_tokens: int = 8192, max_decode_reqs: int = 1024,
                 max_kv_tokens: int = 1 << 20, device: int = 0, flags: int = 0):
        self._lib = load_library()
        self.cfg = Config(num_qo_heads, num_kv_heads, head_dim,
                          POD_KV_PAGED if paged else POD_KV_CONTIGUOUS, 16 if paged else 0,
                          max_prefill_reqs, max_prefill_tokens, max_decode_reqs,
                          max_kv_tokens, device, flags)
        h = ctypes.c_void_p()
        rc = self._lib.pod_attn_create(ctypes.byref(h), ctypes.byref(self.cfg))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_create")
        self._h = h
        self.paged = paged
        self._keep = []

    # -- argument structs (the keep-alive list holds the ctypes arrays)
    def prefill_args(self, chunk_lens, prior_lens, q, o, lse, k=None, v=None, k_pool=None,
                     v_pool=None, block_table=None) -> PrefillArgs:
        n = len(chunk_lens)
        cl, pl = _int_array(chunk_lens), _int_array(prior_lens)
        keep = [cl, pl]
        a = PrefillArgs()
        a.num_reqs = n
        a.chunk_lens = ctypes.cast(cl, ctypes.POINTER(ctypes.c_int))
        a.prior_lens = ctypes.cast(pl, ctypes.POINTER(ctypes.c_int))
        a.q, a.o, a.lse = _dptr(q), _dptr(o), _dptr(lse)
        if self.paged:
            a.k_pool, a.v_pool = _dptr(k_pool), _dptr(v_pool)
            a.block_table = _dptr(block_table)
            a.block_table_stride = int(block_table.shape[1]) if block_table is not None else 0
            a.pool_blocks = int(k_pool.shape[0]) if k_pool is not None else 0
        else:
            kp, vp = _ptr_array(k or []), _ptr_array(v or [])
            for t in list(k or []) + list(v or []):
                _dptr(t)
            keep += [kp, vp]
            a.k_ptrs = ctypes.cast(kp, ctypes.POINTER(ctypes.c_void_p))
            a.v_ptrs = ctypes.cast(vp, ctypes.POINTER(ctypes.c_void_p))
        a._keep = keep
        return a

    def decode_args(self, ctx_lens, q, o, lse, k=None, v=None, k_pool=None, v_pool=None,
                    block_table=None) -> DecodeArgs:
        n = len(ctx_lens)
        cl = _int_array(ctx_lens)
        keep = [cl]
        a = DecodeArgs()
        a.num_reqs = n
        a.ctx_lens = ctypes.cast(cl, ctypes.POINTER(ctypes.c_int))
        a.q, a.o, a.lse = _dptr(q), _dptr(o), _dptr(lse)
        if self.paged:
            a.k_pool, a.v_pool = _dptr(k_pool), _dptr(v_pool)
            a.block_table = _dptr(block_table)
            a.block_table_stride = int(block_table.shape[1]) if block_table is not None else 0
            a.pool_blocks = int(k_pool.shape[0]) if k_pool is not None else 0
        else:
            kp, vp = _ptr_array(k or []), _ptr_array(v or [])
            for t in list(k or []) + list(v or []):
                _dptr(t)
            keep += [kp, vp]
            a.k_ptrs = ctypes.cast(kp, ctypes.POINTER(ctypes.c_void_p))
            a.v_ptrs = ctypes.cast(vp, ctypes.POINTER(ctypes.c_void_p))
        a._keep = keep
        return a

    # -- calls
    def hybrid(self, prefill: Optional[PrefillArgs], decode: Optional[DecodeArgs],
               mode: int = MODE_FUSED, stream=None) -> None:
        rc = self._lib.pod_attn_hybrid(self._h, ctypes.byref(prefill) if prefill else None,
                                       ctypes.byref(decode) if decode else None, int(mode),
                                       ctypes.c_void_p(_stream_handle(stream)))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_hybrid")

    def prefill_only(self, prefill: PrefillArgs, stream=None) -> None:
        rc = self._lib.pod_attn_prefill_only(self._h, ctypes.byref(prefill),
                                             ctypes.c_void_p(_stream_handle(stream)))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_prefill_only")

    def decode_only(self, decode: DecodeArgs, stream=None) -> None:
        rc = self._lib.pod_attn_decode_only(self._h, ctypes.byref(decode),
                                            ctypes.c_void_p(_stream_handle(stream)))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_decode_only")

    def status(self, stream=None) -> int:
        return int(self._lib.pod_attn_status(self._h, ctypes.c_void_p(_stream_handle(stream))))

    def last_plan(self) -> dict:
        info = PlanInfo()
        rc = self._lib.pod_attn_last_plan(self._h, ctypes.byref(info))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_last_plan")
        return info.as_dict()

    def stats(self, stream=None) -> dict:
        st = Stats()
        rc = self._lib.pod_attn_get_stats(self._h, ctypes.c_void_p(_stream_handle(stream)),
                                          ctypes.byref(st))
        if rc != POD_OK:
            raise PodError(rc, "pod_attn_get_stats")
        return st.as_dict()

    def close(self) -> int:
        if getattr(self, "_h", None):
            rc = int(self._lib.pod_attn_destroy(self._h))
            self._h = None
            return rc
        return POD_OK

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def decode_static(num_qo_heads: int, num_kv_heads: int, head_dim: int, decode: DecodeArgs,
                  paged: bool = False, stream=None) -> None:
    """``pod_attn_decode_static``: decode attention that allocates no device
    memory (for callers whose device memory is all owned by someone else).
    Runs on the current CUDA device; calls must not overlap on the GPU."""
    lib = load_library()
    rc = lib.pod_attn_decode_static(int(num_qo_heads), int(num_kv_heads), int(head_dim),
                                    POD_KV_PAGED if paged else POD_KV_CONTIGUOUS,
                                    ctypes.byref(decode), ctypes.c_void_p(_stream_handle(stream)))
    if rc != POD_OK:
        raise PodError(rc, "pod_attn_decode_static")


class DeviceBatch:
    """A hybrid batch resident on the GPU plus its output buffers."""

    def __init__(self, batch, device="cuda", paged: Optional[bool] = None):
        cfg = batch.cfg
        self.batch = batch
        self.paged = cfg.paged if paged is None else paged
        H, d = cfg.num_qo_heads, cfg.head_dim
        dev = torch.device(device)
        self.q_p = batch.q_prefill.to(dev)
        self.q_d = batch.q_decode.to(dev)
        if self.paged:
            self.k_pool = batch.k_pool.to(dev)
            self.v_pool = batch.v_pool.to(dev)
            self.bt_p = batch.block_table_prefill.to(dev)
            self.bt_d = batch.block_table_decode.to(dev)
            self.k_p = self.v_p = self.k_d = self.v_d = None
        else:
            self.k_p = [k.to(dev) for k in batch.k_prefill]
            self.v_p = [v.to(dev) for v in batch.v_prefill]
            self.k_d = [k.to(dev) for k in batch.k_decode]
            self.v_d = [v.to(dev) for v in batch.v_decode]
            self.k_pool = self.v_pool = self.bt_p = self.bt_d = None
        tp, nd = batch.total_prefill_tokens, batch.num_decodes
        self.o_p = torch.empty(tp, H, d, dtype=torch.bfloat16, device=dev)
        self.lse_p = torch.empty(tp, H, dtype=torch.float32, device=dev)
        self.o_d = torch.empty(nd, H, d, dtype=torch.bfloat16, device=dev)
        self.lse_d = torch.empty(nd, H, dtype=torch.float32, device=dev)

    def args(self, pod: PodAttention):
        b = self.batch
        pa = pod.prefill_args(b.chunks, b.priors, self.q_p, self.o_p, self.lse_p, k=self.k_p,
                              v=self.v_p, k_pool=self.k_pool, v_pool=self.v_pool,
                              block_table=self.bt_p) if b.chunks else None
        da = pod.decode_args(b.ctx, self.q_d, self.o_d, self.lse_d, k=self.k_d, v=self.v_d,
                             k_pool=self.k_pool, v_pool=self.v_pool,
                             block_table=self.bt_d) if b.ctx else None
        return pa, da

    def fill_outputs(self, value=float("nan")):
        for t in (self.o_p, self.o_d):
            t.fill_(value)
        for t in (self.lse_p, self.lse_d):
            t.fill_(value)


def context_for(batch, paged: Optional[bool] = None, flags: int = 0, device: int = 0,
                max_kv_tokens: Optional[int] = None) -> PodAttention:
    """A context sized for ``batch`` (a workloads.HybridBatch)."""
    cfg = batch.cfg
    longest = max([p + c for p, c in zip(batch.priors, batch.chunks)] + list(batch.ctx) + [1])
    return PodAttention(cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim,
                        paged=cfg.paged if paged is None else paged,
                        max_prefill_reqs=max(1, len(batch.chunks)),
                        max_prefill_tokens=max(1, batch.total_prefill_tokens),
                        max_decode_reqs=max(1, batch.num_decodes),
                        max_kv_tokens=max_kv_tokens or longest, device=device, flags=flags)
