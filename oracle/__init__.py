"""fp64 CPU oracle for hybrid prefill + decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` leg are the only callers.
The product library never imports, links or runs anything here, and this
package imports nothing from the product (inputs arrive as plain CPU tensors
from the shared seeded generator).

What it computes is the plain definition of the operation POD-Attention
fuses ("POD-Attention: Unlocking Full Prefill-Decode Overlap", §2.1: a hybrid
batch holds prefill chunks and decodes; the Silicon & Systems digest,
"Virtual CTAs and SM-aware balance": fusion leaves the attention values
unchanged). For every query row and query head h:

* KV head ``g = h // (H / Hk)``;
* visible keys: prefill token t (0-based in its chunk) of a request with
  ``prior`` cached tokens sees keys ``0 .. prior + t`` (its own chunk's K/V are
  already in the cache at prior .. prior + chunk - 1); decode request r sees
  keys ``0 .. ctx_r - 1``;
* ``O = softmax(q K^T / sqrt(d)) V`` and ``LSE = ln sum_j exp(q.k_j / sqrt(d))``.

The arithmetic lives in ``pod_oracle.c`` (fp64, two passes per row). This
module only lists the (row, head, key range) items and marshals pointers.
``merge_partials`` states the split-merge identity used to pin the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pod_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``pod_oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp,
                               _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get_lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.pod_oracle_items.restype = ctypes.c_int
            lib.pod_oracle_items.argtypes = [
                ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            lib.pod_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_get_lib().pod_oracle_max_threads())


def _u16(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16)


def attention_items(q: torch.Tensor, caches_k: Sequence[torch.Tensor],
                    caches_v: Sequence[torch.Tensor], rows: np.ndarray, heads: np.ndarray,
                    cache_idx: np.ndarray, kbeg: np.ndarray, kend: np.ndarray,
                    group: int, n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """O (fp64 [n, d]) and LSE (fp64 [n]) for explicit items.

    Item i: query ``q[rows[i], heads[i], :]`` against keys ``[kbeg[i], kend[i])``
    of cache ``cache_idx[i]`` (bf16 ``[len, Hk, d]``), KV head ``heads[i] // group``.
    """
    lib = _get_lib()
    qq = _u16(q)
    n_rows, H, d = qq.shape
    ks = [_u16(k) for k in caches_k]
    vs = [_u16(v) for v in caches_v]
    Hk = ks[0].shape[1] if ks else max(1, H // group)
    n = int(len(rows))
    rows = np.asarray(rows, dtype=np.int64)
    heads = np.asarray(heads, dtype=np.int64)
    assert (rows >= 0).all() and (rows < n_rows).all() and (heads >= 0).all() and (heads < H).all()
    q_base = qq.data_ptr()
    q_ptrs = (q_base + ((rows * H + heads) * d) * 2).astype(np.uint64)
    k_ptrs = np.array([k.data_ptr() for k in ks] or [0], dtype=np.uint64)
    v_ptrs = np.array([v.data_ptr() for v in vs] or [0], dtype=np.uint64)
    cache_idx = np.ascontiguousarray(cache_idx, dtype=np.int32)
    kb = np.ascontiguousarray(kbeg, dtype=np.int64)
    ke = np.ascontiguousarray(kend, dtype=np.int64)
    for i in range(len(ks)):
        sel = cache_idx == i
        if sel.any():
            assert ke[sel].max() <= ks[i].shape[0] and kb[sel].min() >= 0
    hkv = np.ascontiguousarray(heads // group, dtype=np.int32)
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    if n:
        rc = lib.pod_oracle_items(
            n, Hk, d, q_ptrs.ctypes.data, cache_idx.ctypes.data, kb.ctypes.data,
            ke.ctypes.data, hkv.ctypes.data, k_ptrs.ctypes.data, v_ptrs.ctypes.data,
            o.ctypes.data, lse.ctypes.data, int(n_threads))
        if rc != 0:
            raise MemoryError("oracle scratch allocation failed")
    return o, lse


def prefill_items(priors: Sequence[int], chunks: Sequence[int], H: int,
                  sample: Optional[np.ndarray] = None):
    """Items for prefill rows: causal, bottom-right aligned.

    Returns (rows, heads, cache_idx, kbeg, kend). ``sample`` optionally lists
    flat (row * H + head) indices to keep.
    """
    rows, reqs, kend = [], [], []
    off = 0
    for p, (prior, c) in enumerate(zip(priors, chunks)):
        t = np.arange(c, dtype=np.int64)
        rows.append(off + t)
        reqs.append(np.full(c, p, dtype=np.int64))
        kend.append(prior + t + 1)   # keys 0 .. prior + t
        off += c
    rows = np.concatenate(rows) if rows else np.zeros(0, np.int64)
    reqs = np.concatenate(reqs) if reqs else np.zeros(0, np.int64)
    kend = np.concatenate(kend) if kend else np.zeros(0, np.int64)
    flat = np.arange(len(rows) * H, dtype=np.int64) if sample is None else np.asarray(sample)
    r = flat // H
    h = flat % H
    return rows[r], h, reqs[r], np.zeros(len(flat), np.int64), kend[r]


def decode_items(ctx: Sequence[int], H: int, sample: Optional[np.ndarray] = None):
    """Items for decode rows: request r sees keys 0 .. ctx[r] - 1, no mask."""
    n = len(ctx)
    flat = np.arange(n * H, dtype=np.int64) if sample is None else np.asarray(sample)
    r = flat // H
    h = flat % H
    ctx = np.asarray(ctx, dtype=np.int64)
    return r, h, r, np.zeros(len(flat), np.int64), ctx[r] if n else np.zeros(0, np.int64)


def hybrid(batch, prefill_sample: Optional[np.ndarray] = None,
           decode_sample: Optional[np.ndarray] = None, n_threads: int = 0) -> Dict[str, np.ndarray]:
    """Reference outputs of a whole hybrid batch (or of sampled (row, head) pairs).

    Without samples: ``prefill_o`` [sum chunk, H, d], ``prefill_lse``
    [sum chunk, H], ``decode_o`` [n_dec, H, d], ``decode_lse`` [n_dec, H]. With a
    sample (flat row * H + head indices) the arrays are [n_sample, d] / [n_sample].
    """
    cfg = batch.cfg
    H, Hk, d = cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim
    G = H // Hk
    out = {}
    r, h, c, kb, ke = prefill_items(batch.priors, batch.chunks, H, prefill_sample)
    o, lse = attention_items(batch.q_prefill, batch.k_prefill, batch.v_prefill, r, h, c, kb, ke,
                             G, n_threads)
    if prefill_sample is None:
        o = o.reshape(batch.total_prefill_tokens, H, d)
        lse = lse.reshape(batch.total_prefill_tokens, H)
    out["prefill_o"], out["prefill_lse"] = o, lse
    r, h, c, kb, ke = decode_items(batch.ctx, H, decode_sample)
    o, lse = attention_items(batch.q_decode, batch.k_decode, batch.v_decode, r, h, c, kb, ke,
                             G, n_threads)
    if decode_sample is None:
        o = o.reshape(batch.num_decodes, H, d)
        lse = lse.reshape(batch.num_decodes, H)
    out["decode_o"], out["decode_lse"] = o, lse
    return out


def merge_partials(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]):
    """Combine attention over disjoint key ranges into attention over their union.

    With ``M = max_s lse_s`` and ``w_s = exp(lse_s - M)``:
    ``O = sum_s w_s O_s / sum_s w_s`` and ``LSE = M + ln sum_s w_s``. This is the
    log-sum-exp merge of split-KV partial results (POD-Attention's partial
    results meet where split tiles end: Silicon & Systems digest, "Virtual
    CTAs and SM-aware balance"). Parts with ``lse = -inf`` carry zero weight.
    """
    lse = np.stack([np.asarray(x, np.float64) for x in lse_parts])    # [S, ...]
    o = np.stack([np.asarray(x, np.float64) for x in o_parts])        # [S, ..., d]
    M = lse.max(axis=0)
    w = np.exp(lse - M)
    W = w.sum(axis=0)
    merged = (w[..., None] * o).sum(axis=0) / W[..., None]
    return merged, M + np.log(W)
