"""pod_attn_decode_static: decode attention that allocates no device memory.

It exists for callers whose device memory is all owned by someone else (an
engine that reserves HBM for its KV cache up front, a plugin handed its
buffers by a host framework) and so cannot cudaMalloc when they call
attention. Each case checks its output against the fp64 oracle at the parity
tolerances and against the context-based pod_attn_decode_only, on two calls in
a row (the second call reuses the library's scratch array the first one left
behind), and a batch of another shape runs right after a large one.

This file is collected last so that a run that stops at its first failure has
already run every other test; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_prefill_decode_pod_b200 import pod_attn as pa
from hybrid_prefill_decode_pod_b200 import workloads as W

from gpu_util import compare

pytestmark = pytest.mark.gpu


def _static_twice(b, paged):
    """Two pod_attn_decode_static calls on `b`; each compared with the oracle
    and with pod_attn_decode_only on the same inputs."""
    cfg = b.cfg
    ref = oracle.hybrid(b)
    pod = pa.context_for(b, paged=paged)
    db = pa.DeviceBatch(b, paged=paged)
    _, dec = db.args(pod)
    pod.decode_only(dec)
    assert pod.status() == pa.POD_OK
    ctx_o, ctx_lse = db.o_d.clone(), db.lse_d.clone()
    for _ in range(2):
        db.o_d.fill_(float("nan"))
        db.lse_d.fill_(float("nan"))
        pa.decode_static(cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim, dec, paged=paged)
        torch.cuda.synchronize()
        out = {"decode_o": db.o_d.cpu(), "decode_lse": db.lse_d.cpu()}
        compare(ref, out, keys=("decode",))
        ctx = {"decode_o": ctx_o.cpu(), "decode_lse": ctx_lse.cpu()}
        compare({"decode_o": ctx["decode_o"].double().numpy(),
                 "decode_lse": ctx["decode_lse"].double().numpy()}, out, keys=("decode",))
    assert pod.close() == pa.POD_OK


@pytest.mark.parametrize("paged", [False, True])
def test_static_decode_g4_d128_matches_oracle_twice(paged):
    # split and single-split requests, G = 4, contexts with ragged tails
    b = W.make_custom(32, 8, 128, [], [4096, 1, 700, 5000, 9000, 513, 2048, 77], seed=61,
                      paged=paged)
    _static_twice(b, paged)


def test_static_decode_g8_d64_matches_oracle_twice():
    b = W.make_custom(64, 8, 64, [], [3000, 17, 1024, 6001, 2], seed=67)
    _static_twice(b, False)


def test_static_decode_split_growth_then_smaller_batch():
    # 190 short + 10 long requests with 16 KV heads: at 512 keys per split the
    # units exceed the array's 4096, so the split length grows (to 4096 keys);
    # the long requests still split 5 ways. A smaller batch of another shape
    # then reuses the array the large one left behind.
    ctx = [600] * 190 + [20000] * 10
    big = W.make_custom(16, 16, 64, [], ctx, seed=71)
    _static_twice(big, False)
    small = W.make_custom(16, 4, 128, [], [900, 5, 3333], seed=73)
    _static_twice(small, False)


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
