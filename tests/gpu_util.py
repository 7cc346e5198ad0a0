"""Helpers for the GPU parity tests: run a batch through the C ABI and compare
with the fp64 oracle at the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from hybrid_prefill_decode_pod_b200 import pod_attn as pa

# Tolerances for bf16 outputs against the fp64 oracle on identical inputs.
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def run(batch, mode="fused", paged=None, pod=None, flags=0, fill=float("nan")):
    """One call through the library; returns (outputs dict of CPU tensors, pod)."""
    own = pod is None
    if own:
        pod = pa.context_for(batch, paged=paged, flags=flags)
    db = pa.DeviceBatch(batch, paged=pod.paged)
    db.fill_outputs(fill)
    prefill, decode = db.args(pod)
    if mode == "prefill_only":
        pod.prefill_only(prefill)
    elif mode == "decode_only":
        pod.decode_only(decode)
    else:
        pod.hybrid(prefill, decode, pa.MODES[mode])
    st = pod.status()
    assert st == pa.POD_OK, st
    out = {"prefill_o": db.o_p.cpu(), "prefill_lse": db.lse_p.cpu(),
           "decode_o": db.o_d.cpu(), "decode_lse": db.lse_d.cpu()}
    plan = pod.last_plan()
    if own:
        assert pod.close() == pa.POD_OK
    return out, plan


def compare(ref, out, keys=("prefill", "decode"), sample=None):
    """Element-wise comparison at the stated tolerances. With `sample`
    ({"prefill": idx, "decode": idx} of flat row*H+head), compares sampled rows."""
    report = {}
    for k in keys:
        o_ref = np.asarray(ref[k + "_o"])
        l_ref = np.asarray(ref[k + "_lse"])
        o = out[k + "_o"].float().numpy().astype(np.float64)
        l = out[k + "_lse"].numpy().astype(np.float64)
        if sample is not None and sample.get(k) is not None:
            d = o.shape[-1]
            o = o.reshape(-1, d)[sample[k]]
            l = l.reshape(-1)[sample[k]]
        if o_ref.size == 0:
            continue
        assert np.isfinite(o).all(), "%s: non-finite outputs" % k
        err = np.abs(o - o_ref)
        rel = np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30)
        lerr = np.abs(l - l_ref).max()
        report[k] = (float(err.max()), float(rel), float(lerr))
        assert err.max() <= O_MAX_ABS, "%s O max-abs %.3g" % (k, err.max())
        assert rel <= O_REL_L2, "%s O rel-L2 %.3g" % (k, rel)
        assert lerr <= LSE_MAX_ABS, "%s LSE max-abs %.3g" % (k, lerr)
    return report


def sample_indices(n_rows, H, count, seed):
    """Sampled flat (row * H + head) indices: first/last rows, plus random ones."""
    g = np.random.default_rng(seed)
    total = n_rows * H
    if total == 0:
        return np.zeros(0, np.int64)
    edge = [0, H - 1, total - H, total - 1]
    rnd = g.integers(0, total, size=count)
    return np.unique(np.clip(np.concatenate([edge, rnd]), 0, total - 1)).astype(np.int64)


def bitwise_equal(a, b):
    for k in a:
        if not torch.equal(a[k].view(torch.int16) if a[k].dtype == torch.bfloat16 else
                           a[k].view(torch.int32),
                           b[k].view(torch.int16) if b[k].dtype == torch.bfloat16 else
                           b[k].view(torch.int32)):
            return False
    return True
