"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerances (bf16 outputs vs fp64): O max-abs <= 1e-2 and relative L2 <= 5e-3;
LSE max-abs <= 1e-3. Every output element is compared, on scaled-down shapes
that span several tiles with ragged tails and on the five full-size
configurations in the launch configuration the benchmark times.
"""
import contextlib
import os

import numpy as np
import pytest
import torch

import oracle
from hybrid_prefill_decode_pod_b200 import workloads as W
from hybrid_prefill_decode_pod_b200 import pod_attn as pa

from gpu_util import bitwise_equal, compare, run

pytestmark = pytest.mark.gpu


def test_tiny_config_all_modes_match_oracle():
    b = W.make_batch(W.CONFIGS["tiny"])
    ref = oracle.hybrid(b)
    outs = {}
    for mode in ("fused", "serial", "two_stream"):
        outs[mode], _ = run(b, mode)
        compare(ref, outs[mode])
    assert bitwise_equal(outs["fused"], outs["serial"])
    assert bitwise_equal(outs["fused"], outs["two_stream"])


SHAPES = [
    # (H, Hk, d, prefill[(prior, chunk)], decode ctx) -- several tiles, ragged tails
    (8, 2, 128, [(300, 200)], [1, 17, 64, 65, 1000, 3000]),
    (16, 2, 128, [(0, 130), (77, 257)], [5, 4096, 513]),          # G = 8, prior 0, 2 chunks
    (4, 4, 128, [(1000, 64)], [2048, 31]),                        # G = 1
    (8, 4, 64, [(129, 129)], [128, 129, 700]),                    # d = 64, G = 2
    (32, 8, 128, [(4096, 512)], [4096] * 4),                      # llama-3-8B rows
    # G odd: a prefill unit pairs two token tiles of one head (the first tile's
    # rows meet fully masked KV tiles of the pair's range), with KV splits
    (6, 2, 128, [(900, 300)], [50, 700]),                         # G = 3, 3 tiles
    (3, 1, 64, [(1100, 260), (0, 1)], [33]),                      # G = 3, d = 64, 1-token chunk
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode", ["fused", "serial"])
def test_scaled_shapes_match_oracle(shape, mode):
    H, Hk, d, pre, ctx = shape
    b = W.make_custom(H, Hk, d, pre, ctx, seed=5)
    ref = oracle.hybrid(b)
    out, plan = run(b, mode)
    compare(ref, out)


@pytest.mark.parametrize("d", [128, 64])
def test_paged_matches_contiguous_bitwise_and_oracle(d):
    # d = 64 decode stages hold two 16-key blocks, so a stage spans two pages
    b = W.make_custom(8, 2, d, [(333, 190), (0, 40)], [1, 16, 17, 33, 999, 2500], seed=9,
                      paged=True)
    ref = oracle.hybrid(b)
    paged, _ = run(b, "fused", paged=True)
    contig, _ = run(b, "fused", paged=False)
    compare(ref, paged)
    assert bitwise_equal(paged, contig)


@pytest.mark.parametrize("tile", ["pair", "1sm"])
def test_run_to_run_bitwise_and_modes_bitwise(tile):
    b = W.make_custom(8, 2, 128, [(2000, 300)], [100, 5000, 7000, 64], seed=13)
    with plan_env(POD_ATTN_PREFILL_TILE=tile):
        a1, p1 = run(b, "fused")
        a2, _ = run(b, "fused")
    assert bitwise_equal(a1, a2)
    assert (p1["pair_clusters"] > 0) == (tile == "pair")
    # FUSED may plan the prefill split differently from the separate-launch
    # modes (it leaves it unsplit when decode is the longer phase); on the
    # same plan all three modes give identical bits
    for split in ("1", "3"):
        with plan_env(POD_ATTN_PREFILL_SPLIT=split, POD_ATTN_PREFILL_TILE=tile):
            f, pf = run(b, "fused")
            s1, ps = run(b, "serial")
            t1, _ = run(b, "two_stream")
        assert pf["prefill_split"] == ps["prefill_split"] == int(split)
        assert bitwise_equal(f, s1)
        assert bitwise_equal(f, t1)


PAIR_SHAPES = [
    # the one-SM prefill tile against the CTA-pair tile, both against the oracle
    (8, 2, 128, [(300, 200)], [1, 17, 1000]),
    (6, 2, 128, [(900, 300)], [50, 700]),                         # G = 3: token-tile pairs
    (4, 4, 128, [(1000, 64)], [2048]),                            # G = 1, missing 2nd tile
    (16, 2, 128, [(0, 130), (77, 257)], [5, 4096]),               # G = 8, two requests
]


@pytest.mark.parametrize("shape", PAIR_SHAPES)
def test_pair_and_one_sm_prefill_tiles_match_oracle(shape):
    H, Hk, d, pre, ctx = shape
    b = W.make_custom(H, Hk, d, pre, ctx, seed=7)
    ref = oracle.hybrid(b)
    for tile in ("pair", "1sm"):
        for split in ("0", "3"):
            with plan_env(POD_ATTN_PREFILL_TILE=tile, POD_ATTN_PREFILL_SPLIT=split):
                out, plan = run(b, "fused")
            assert (plan["pair_clusters"] > 0) == (tile == "pair")
            compare(ref, out)


POLICIES = ["front", "prefill_first", "even", "proportional", "balanced", "decode_first"]


@pytest.mark.parametrize("tile", ["1sm", "pair"])
def test_every_role_policy_matches_oracle_and_agrees_bitwise(tile):
    """The role policy decides which SM runs which unit and when, never what a
    unit computes: every policy gives the same bits on the same plan, and
    they match the oracle."""
    b = W.make_custom(8, 2, 128, [(1500, 400), (0, 130)], [64, 700, 3000, 9000, 17], seed=23)
    ref = oracle.hybrid(b)
    first = None
    for policy in POLICIES:
        with plan_env(POD_ATTN_PREFILL_TILE=tile, POD_ATTN_POLICY=policy):
            out, plan = run(b, "fused")
        assert (plan["pair_clusters"] > 0) == (tile == "pair")
        compare(ref, out)
        if first is None:
            first = (out, plan)
        else:
            assert plan["prefill_split"] == first[1]["prefill_split"]
            assert plan["decode_split_len"] == first[1]["decode_split_len"]
            assert bitwise_equal(first[0], out), policy


def test_prefill_only_and_decode_only_match_hybrid():
    b = W.make_custom(8, 2, 128, [(700, 300)], [3000, 20], seed=17)
    h, _ = run(b, "fused")
    p, _ = run(b, "prefill_only")
    d, _ = run(b, "decode_only")
    assert torch.equal(h["prefill_o"].view(torch.int16), p["prefill_o"].view(torch.int16))
    assert torch.equal(h["decode_o"].view(torch.int16), d["decode_o"].view(torch.int16))
    assert torch.equal(h["decode_lse"], d["decode_lse"])


def test_invariants_on_gpu():
    """Constant V returns V; K == 0 gives ln(#keys); one key returns its V."""
    b = W.make_custom(8, 2, 128, [(0, 150)], [1, 200, 3000], seed=21)
    for v in b.v_prefill + b.v_decode:
        v[:, 0] = 0.5
        v[:, 1] = -2.0
    for k in b.k_prefill + b.k_decode:
        k.zero_()
    out, _ = run(b, "fused")
    c = torch.tensor([0.5] * 4 + [-2.0] * 4)
    # P is rounded to bf16 for the tensor cores, the normaliser is not: within
    # one bf16 ulp of |c| (the rows-sum-to-one invariant on the GPU).
    tol = c.abs()[None, :, None] * 2.0 ** -7
    assert ((out["decode_o"].float() - c[None, :, None]).abs() <= tol).all()
    assert ((out["prefill_o"].float() - c[None, :, None]).abs() <= tol).all()
    for r, L in enumerate(b.ctx):
        assert np.abs(out["decode_lse"][r].numpy() - np.log(L)).max() < 1e-5
    t = np.arange(150)
    # every score is 0, so every weight is exactly 1 and the row sum is the
    # exact key count: the LSE differs from ln(count) only by the rounding of
    # the final log
    assert np.abs(out["prefill_lse"].numpy() - np.log(t + 1)[:, None]).max() < 1e-5
    # single key: decode L = 1 returns V0 bitwise
    b2 = W.make_custom(8, 2, 128, [], [1, 1], seed=23)
    out2, _ = run(b2, "fused")
    for r in range(2):
        for h in range(8):
            assert torch.equal(out2["decode_o"][r, h], b2.v_decode[r][0, h // 4])


def test_causal_mask_on_gpu():
    """Changing K/V at position P leaves rows with prior + t < P bitwise unchanged."""
    prior, c = 200, 300
    b = W.make_custom(8, 2, 128, [(prior, c)], [], seed=29)
    a, _ = run(b, "fused")
    P = prior + 123
    b.k_prefill[0][P] = 3.0
    b.v_prefill[0][P] = -3.0
    a2, _ = run(b, "fused")
    assert torch.equal(a["prefill_o"][:123].view(torch.int16), a2["prefill_o"][:123].view(torch.int16))
    assert not torch.equal(a["prefill_o"][123:].view(torch.int16), a2["prefill_o"][123:].view(torch.int16))


def test_decode_permutation_permutes_outputs():
    b = W.make_custom(8, 2, 128, [], [5, 8000, 333, 1], seed=31)
    a, _ = run(b, "fused")
    perm = [2, 0, 3, 1]
    b2 = W.make_custom(8, 2, 128, [], [b.ctx[i] for i in perm], seed=31)
    b2.q_decode = b.q_decode[perm].clone()
    b2.k_decode = [b.k_decode[i] for i in perm]
    b2.v_decode = [b.v_decode[i] for i in perm]
    a2, _ = run(b2, "fused")
    assert torch.equal(a2["decode_o"].view(torch.int16), a["decode_o"][perm].view(torch.int16))


def test_empty_sides():
    b = W.make_custom(8, 2, 128, [(10, 0)], [50], seed=37)      # chunk 0 is a no-op
    ref = oracle.hybrid(b)
    out, _ = run(b, "fused")
    compare(ref, out, keys=("decode",))
    b2 = W.make_custom(8, 2, 128, [(10, 70)], [], seed=37)      # no decodes
    out2, _ = run(b2, "fused")
    compare(oracle.hybrid(b2), out2, keys=("prefill",))


def test_timeout_path_reports_status_and_keeps_results():
    b = W.make_custom(8, 2, 128, [(64, 64)], [100], seed=41)
    pod = pa.context_for(b, flags=pa.FLAG_TEST_FORCE_TIMEOUT)
    db = pa.DeviceBatch(b)
    pre, dec = db.args(pod)
    pod.hybrid(pre, dec, pa.MODE_FUSED)
    assert pod.status() == pa.POD_ETIMEOUT
    assert pod.status() == pa.POD_OK       # cleared by the read
    out = {"prefill_o": db.o_p.cpu(), "prefill_lse": db.lse_p.cpu(),
           "decode_o": db.o_d.cpu(), "decode_lse": db.lse_d.cpu()}
    compare(oracle.hybrid(b), out)
    assert pod.close() == pa.POD_OK


@contextlib.contextmanager
def plan_env(**kv):
    """Planner levers for the contexts created inside (read at creation)."""
    old = {k: os.environ.get(k) for k in kv}
    os.environ.update(kv)
    try:
        yield
    finally:
        for k, v in old.items():
            if v is None:
                del os.environ[k]
            else:
                os.environ[k] = v


def _stats_for(b, policy=None):
    with plan_env(**({"POD_ATTN_POLICY": policy} if policy else {})):
        pod = pa.context_for(b, flags=pa.FLAG_STATS)
    db = pa.DeviceBatch(b)
    pre, dec = db.args(pod)
    pod.hybrid(pre, dec, pa.MODE_FUSED)
    st, plan = pod.stats(), pod.last_plan()
    assert pod.close() == pa.POD_OK
    return st, plan


def test_stats_show_both_roles_per_sm():
    b = W.make_batch(W.CONFIGS["llama3_8b"])
    # balanced: a decode-heavy batch gives prefill to a subset of the SMs
    # first; every prefill unit is claimed once and some SMs run both roles
    st, plan = _stats_for(b, "balanced")
    assert st["prefill_claims"] == plan["prefill_units"]
    assert 1 <= plan["prefill_sm_cap"] < plan["num_sms"]
    assert st["sms_with_both"] >= 1
    # front (the default): every SM's first claim takes prefill, so every SM
    # that got a prefill unit also runs decode turns after it
    st, plan = _stats_for(b)
    assert st["prefill_claims"] == plan["prefill_units"]
    assert st["sms_with_both"] >= min(plan["prefill_units"], plan["num_sms"]) // 2


_FULL_REF = {}


def _full_ref(name):
    """Batch and full fp64 oracle outputs of a full-size configuration (cached
    per test session: the oracle is the expensive side)."""
    if name not in _FULL_REF:
        _FULL_REF.clear()  # keep one configuration's tensors alive at a time
        b = W.make_batch(W.get_config(name))
        _FULL_REF[name] = (b, oracle.hybrid(b))
    return _FULL_REF[name]


FULL_SIZE = [("llama3_8b", "fused"), ("decode_heavy", "fused"),
             ("long_context", "fused"), ("long_context", "serial"), ("long_context", "two_stream"),
             ("paged", "fused"), ("paged", "serial"), ("paged", "two_stream"),
             # shape variants: multi-head, group of 8, head_dim 64, 16 small chunks
             ("llama2_7b_mha", "fused"), ("yi6b_g8", "fused"), ("d64_mix", "fused"),
             ("many_chunks", "fused"), ("many_chunks", "serial"),
             # a late chunk of the chunked 16K prompt (prior 15872 + 512, 64 decodes)
             ("chunked16k_31", "fused"),
             # the CTA-pair prefill tile (POD_ATTN_PREFILL_TILE=pair)
             ("long_context", "fused+pair"), ("paged", "fused+pair")]


@pytest.mark.slow
@pytest.mark.parametrize("name,mode", FULL_SIZE)
def test_full_size_configs_every_element(name, mode):
    """Full-size configuration in the launch configuration the benchmark times,
    every output element against the fp64 oracle. SERIAL and TWO_STREAM take
    their own prefill plans (they may split the KV range where FUSED does not)."""
    b, ref = _full_ref(name)
    mode, _, tile = mode.partition("+")
    with plan_env(POD_ATTN_PREFILL_TILE=tile or "1sm"):
        out, plan = run(b, mode)
    assert (plan["pair_clusters"] > 0) == (tile == "pair")
    compare(ref, out)
