"""pod_attn_decode_static: decode attention that allocates no device memory.

It exists for callers whose device memory is all owned by someone else (an
engine that reserves HBM for its KV cache up front, a plugin handed its
buffers by a host framework) and so cannot cudaMalloc when they call
attention. Its output must agree with the context-based pod_attn_decode_only
at the parity tolerances, on two calls in a row (the second call reuses the
library's scratch array the first one left behind).

This file is collected last so that a run that stops at its first failure has
already run every other test; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

from hybrid_prefill_decode_pod_b200 import pod_attn as pa
from hybrid_prefill_decode_pod_b200 import workloads as W

from gpu_util import LSE_MAX_ABS, O_MAX_ABS, O_REL_L2

pytestmark = pytest.mark.gpu


def _close(o, lse, o_ref, lse_ref):
    o, o_ref = o.float().cpu().double(), o_ref.float().cpu().double()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert (o - o_ref).abs().max().item() <= O_MAX_ABS
    assert (torch.linalg.norm(o - o_ref) / torch.linalg.norm(o_ref)).item() <= O_REL_L2
    assert (lse.cpu().double() - lse_ref.cpu().double()).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.parametrize("paged", [False, True])
def test_static_decode_matches_decode_only_twice(paged):
    # splits and single-split requests, G = 4, contexts with ragged tails
    b = W.make_custom(32, 8, 128, [], [4096, 1, 700, 5000, 9000, 513, 2048, 77], seed=61,
                      paged=paged)
    pod = pa.context_for(b, paged=paged)
    db = pa.DeviceBatch(b, paged=paged)
    _, dec = db.args(pod)
    pod.decode_only(dec)
    assert pod.status() == pa.POD_OK
    ref_o, ref_lse = db.o_d.clone(), db.lse_d.clone()
    cfg = b.cfg
    for _ in range(2):
        db.o_d.fill_(float("nan"))
        db.lse_d.fill_(float("nan"))
        pa.decode_static(cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim, dec, paged=paged)
        torch.cuda.synchronize()
        _close(db.o_d, db.lse_d, ref_o, ref_lse)
    assert pod.close() == pa.POD_OK


def test_static_decode_rejects_sizes_beyond_its_array():
    b = W.make_custom(8, 2, 64, [], [3] * 4, seed=3)
    db = pa.DeviceBatch(b, paged=False)
    pod = pa.context_for(b)
    _, dec = db.args(pod)
    dec.num_reqs = 513  # above POD_STATIC_MAX_DECODE_REQS, refused before use
    with pytest.raises(pa.PodError) as e:
        pa.decode_static(8, 2, 64, dec)
    assert e.value.code == pa.POD_ECAPACITY
    pod.close()
