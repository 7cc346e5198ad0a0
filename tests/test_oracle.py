"""Pins for the fp64 CPU oracle (no GPU).

The pages print no worked numeric example, so the oracle is pinned by what the
mathematics of ``softmax(q K^T / sqrt(d)) V`` and its log-sum-exp fix: closed
forms (tests/golden/closed_forms.json), invariants (rows sum to one, constant
V, single key, causal masking, split/merge, GQA head map, request
permutation) and brute force against an independent library routine
(``torch.nn.functional.scaled_dot_product_attention`` in float64 with an
explicit mask) on tiny shapes. Each pin targets a plausible slip in the
oracle: a wrong scale, a dropped max-subtraction, an off-by-one in the causal
bound, a top-left instead of bottom-right mask, a wrong GQA map, a transposed
operand.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from hybrid_prefill_decode_pod_b200 import workloads as W

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


def _bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _sdpa_reference(batch):
    """Independent formulation: explicit [rows x keys] boolean mask + float64 SDPA."""
    cfg = batch.cfg
    H, Hk, d = cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim
    out_p, out_d = [], []
    off = 0
    for p, (prior, c) in enumerate(zip(batch.priors, batch.chunks)):
        q = batch.q_prefill[off:off + c].double().permute(1, 0, 2)      # [H, c, d]
        k = batch.k_prefill[p].double().permute(1, 0, 2)                # [Hk, L, d]
        v = batch.v_prefill[p].double().permute(1, 0, 2)
        L = prior + c
        rows = torch.arange(c)[:, None]
        keys = torch.arange(L)[None, :]
        mask = keys <= prior + rows                                     # bottom-right causal
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask,
                                           enable_gqa=True)[0]
        out_p.append(o.permute(1, 0, 2))
        off += c
    for r, L in enumerate(batch.ctx):
        q = batch.q_decode[r:r + 1].double().permute(1, 0, 2)           # [H, 1, d]
        k = batch.k_decode[r].double().permute(1, 0, 2)
        v = batch.v_decode[r].double().permute(1, 0, 2)
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], enable_gqa=True)[0]
        out_d.append(o.permute(1, 0, 2))
    return (torch.cat(out_p) if out_p else None), (torch.cat(out_d) if out_d else None)


@pytest.mark.parametrize("shape", [
    # (H, Hk, d, prefill[(prior, chunk)], decode ctx)
    (4, 2, 64, [(64, 32)], [40, 77, 128, 200]),         # the tiny config's shape
    (8, 1, 64, [(0, 17), (5, 9)], [1, 3, 256]),          # G = 8, prior 0, several chunks
    (8, 2, 32, [(100, 31)], [256, 2]),                   # G = 4
    (4, 4, 16, [(3, 40)], [7]),                          # G = 1 (MHA)
    (2, 1, 128, [(0, 1)], [1, 9]),                       # one-row chunk, single key decode
])
def test_oracle_matches_sdpa_float64(shape):
    """I9: oracle == explicit-mask float64 SDPA (library routine) to 1e-12."""
    H, Hk, d, pre, ctx = shape
    b = W.make_custom(H, Hk, d, pre, ctx, seed=3)
    ref = oracle.hybrid(b)
    sp, sd = _sdpa_reference(b)
    np.testing.assert_allclose(ref["prefill_o"], sp.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref["decode_o"], sd.numpy(), rtol=0, atol=1e-12)


def test_oracle_lse_matches_logsumexp():
    """LSE == torch.logsumexp over explicitly built float64 scores (library routine)."""
    b = W.make_custom(4, 2, 64, [(10, 6)], [33], seed=5)
    ref = oracle.hybrid(b)
    G = 2
    # decode row 0, every head
    for h in range(4):
        q = b.q_decode[0, h].double()
        k = b.k_decode[0][:, h // G].double()
        s = (k @ q) / math.sqrt(64)
        assert abs(torch.logsumexp(s, 0).item() - ref["decode_lse"][0, h]) < 1e-12
    # prefill token t sees prior + t + 1 keys
    for t in range(6):
        for h in range(4):
            q = b.q_prefill[t, h].double()
            k = b.k_prefill[0][: 10 + t + 1, h // G].double()
            s = (k @ q) / math.sqrt(64)
            assert abs(torch.logsumexp(s, 0).item() - ref["prefill_lse"][t, h]) < 1e-12


def test_golden_two_keys_sigmoid():
    g = GOLDEN["two_keys_sigmoid"]
    d = g["d"]
    q = torch.zeros(1, 1, d); q[0, 0, 0] = 1.0
    k = torch.zeros(2, 1, d); k[1, 0, 0] = 16.0
    v = torch.zeros(2, 1, d); v[0, 0, 0] = 1.0; v[1, 0, 1] = 1.0
    o, lse = oracle.attention_items(_bf(q), [_bf(k)], [_bf(v)], np.array([0]), np.array([0]),
                                    np.array([0]), np.array([0]), np.array([2]), group=1)
    assert abs(o[0, 0] - g["o0"]) < 1e-15
    assert abs(o[0, 1] - g["o1"]) < 1e-15
    assert np.all(o[0, 2:] == 0)
    assert abs(lse[0] - g["lse"]) < 1e-14


def test_golden_zero_keys_mean_and_log_count():
    """I8: K == 0 gives O = mean(V over visible keys) and LSE = ln |J|."""
    g = GOLDEN["zero_keys_decode_200"]
    b = W.make_custom(4, 2, 64, [(64, 32)], [40, 77, 128, g["n_keys"]], seed=0)
    for k in b.k_prefill + b.k_decode:
        k.zero_()
    ref = oracle.hybrid(b)
    assert abs(ref["decode_lse"][3, 0] - g["lse"]) < 1e-13
    for r, L in enumerate(b.ctx):
        for h in range(4):
            mean = b.v_decode[r][:, h // 2].double().mean(0).numpy()
            np.testing.assert_allclose(ref["decode_o"][r, h], mean, rtol=0, atol=1e-13)
            assert abs(ref["decode_lse"][r, h] - math.log(L)) < 1e-13
    for t in range(32):
        n = 64 + t + 1
        mean = b.v_prefill[0][:n, 1].double().mean(0).numpy()
        np.testing.assert_allclose(ref["prefill_o"][t, 3], mean, rtol=0, atol=1e-13)
        assert abs(ref["prefill_lse"][t, 3] - math.log(n)) < 1e-13


def test_golden_equal_scores_pins_scale():
    g = GOLDEN["equal_scores_scale"]
    d, n = g["d"], g["n_keys"]
    q = torch.zeros(1, 1, d); q[0, 0, 0] = 1.0
    k = torch.zeros(n, 1, d); k[:, 0, 0] = 16.0
    v = torch.randn(n, 1, d, generator=torch.Generator().manual_seed(1))
    o, lse = oracle.attention_items(_bf(q), [_bf(k)], [_bf(v)], np.array([0]), np.array([0]),
                                    np.array([0]), np.array([0]), np.array([n]), group=1)
    assert abs(lse[0] - g["lse"]) < 1e-13
    np.testing.assert_allclose(o[0], _bf(v)[:, 0].double().mean(0).numpy(), atol=1e-13, rtol=0)


def test_rows_sum_to_one_constant_v():
    """I2/I3: V constant per KV head returns that constant for every row."""
    b = W.make_custom(8, 2, 64, [(20, 50)], [5, 300], seed=7)
    consts = [0.5, -1.25]
    for v in b.v_prefill + b.v_decode:
        for gk in range(2):
            v[:, gk] = consts[gk]
    ref = oracle.hybrid(b)
    for h in range(8):
        c = consts[h // 4]
        assert np.abs(ref["prefill_o"][:, h] - c).max() < 1e-12
        assert np.abs(ref["decode_o"][:, h] - c).max() < 1e-12


def test_single_key_returns_its_value():
    """I4: one visible key gives O = V0 exactly and LSE = q.k0 / sqrt(d)."""
    b = W.make_custom(4, 2, 64, [(0, 3)], [1, 1], seed=11)
    ref = oracle.hybrid(b)
    for r in range(2):
        for h in range(4):
            np.testing.assert_array_equal(ref["decode_o"][r, h],
                                          b.v_decode[r][0, h // 2].double().numpy())
            s = float(b.q_decode[r, h].double() @ b.k_decode[r][0, h // 2].double()) / 8.0
            assert abs(ref["decode_lse"][r, h] - s) < 1e-13
    # prefill row 0 with prior 0 sees only key 0
    for h in range(4):
        np.testing.assert_array_equal(ref["prefill_o"][0, h],
                                      b.v_prefill[0][0, h // 2].double().numpy())


def test_causal_mask_future_keys_do_not_matter():
    """I5: changing K/V at absolute position P changes no row with prior + t < P."""
    prior, c = 30, 40
    b = W.make_custom(4, 2, 64, [(prior, c)], [], seed=13)
    ref0 = oracle.hybrid(b)
    P = prior + 17
    b.k_prefill[0][P] = 7.0
    b.v_prefill[0][P] = -3.0
    ref1 = oracle.hybrid(b)
    t_unchanged = P - prior          # rows t < 17 do not see P
    np.testing.assert_array_equal(ref0["prefill_o"][:t_unchanged], ref1["prefill_o"][:t_unchanged])
    np.testing.assert_array_equal(ref0["prefill_lse"][:t_unchanged], ref1["prefill_lse"][:t_unchanged])
    # and row t = 17 (which sees exactly up to P) does change
    assert np.abs(ref0["prefill_o"][t_unchanged] - ref1["prefill_o"][t_unchanged]).max() > 1e-3


def test_prefill_items_bottom_right_alignment():
    r, h, c, kb, ke = oracle.prefill_items([2, 0], [3, 2], H=1)
    assert list(r) == [0, 1, 2, 3, 4]
    assert list(c) == [0, 0, 0, 1, 1]
    assert list(ke) == [3, 4, 5, 1, 2]
    assert list(kb) == [0] * 5


@pytest.mark.parametrize("split_points", [[1], [64], [100, 101], [13, 128, 250], [299]])
def test_split_merge_equals_unsplit(split_points):
    """I6: attention over [0,a) and [a,L) merged by the LSE rule == attention over [0,L)."""
    L, H, Hk, d = 300, 4, 2, 64
    b = W.make_custom(H, Hk, d, [], [L], seed=17)
    full = oracle.hybrid(b)
    bounds = [0] + list(split_points) + [L]
    o_parts, l_parts = [], []
    for a, e in zip(bounds[:-1], bounds[1:]):
        o, lse = oracle.attention_items(b.q_decode, b.k_decode, b.v_decode,
                                        np.zeros(H, np.int64), np.arange(H), np.zeros(H, np.int64),
                                        np.full(H, a), np.full(H, e), group=H // Hk)
        o_parts.append(o)
        l_parts.append(lse)
    mo, ml = oracle.merge_partials(o_parts, l_parts)
    np.testing.assert_allclose(mo, full["decode_o"][0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ml, full["decode_lse"][0], rtol=0, atol=1e-12)


def test_merge_with_empty_part():
    o1 = np.ones((2, 4)); l1 = np.array([0.3, -1.0])
    o2 = np.zeros((2, 4)); l2 = np.array([-np.inf, -np.inf])
    mo, ml = oracle.merge_partials([o1, o2], [l1, l2])
    np.testing.assert_array_equal(mo, o1)
    np.testing.assert_array_equal(ml, l1)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_gqa_equals_mha_with_repeated_kv(G):
    """I10: GQA with group G == MHA after repeat-interleaving each KV head G times."""
    Hk, d = 2, 32
    H = Hk * G
    b = W.make_custom(H, Hk, d, [(9, 12)], [50, 3], seed=19)
    ref = oracle.hybrid(b)
    m = W.make_custom(H, H, d, [(9, 12)], [50, 3], seed=19)
    m.q_prefill = b.q_prefill.clone(); m.q_decode = b.q_decode.clone()
    m.k_prefill = [k.repeat_interleave(G, dim=1) for k in b.k_prefill]
    m.v_prefill = [v.repeat_interleave(G, dim=1) for v in b.v_prefill]
    m.k_decode = [k.repeat_interleave(G, dim=1) for k in b.k_decode]
    m.v_decode = [v.repeat_interleave(G, dim=1) for v in b.v_decode]
    ref_m = oracle.hybrid(m)
    for key in ref:
        np.testing.assert_array_equal(ref[key], ref_m[key])


def test_decode_permutation_permutes_outputs():
    """I11: requests are independent, so permuting decodes permutes outputs."""
    b = W.make_custom(4, 2, 64, [], [5, 80, 33, 1], seed=23)
    ref = oracle.hybrid(b)
    perm = [2, 0, 3, 1]
    b2 = W.make_custom(4, 2, 64, [], [b.ctx[i] for i in perm], seed=23)
    b2.q_decode = b.q_decode[perm].clone()
    b2.k_decode = [b.k_decode[i] for i in perm]
    b2.v_decode = [b.v_decode[i] for i in perm]
    ref2 = oracle.hybrid(b2)
    np.testing.assert_array_equal(ref2["decode_o"], ref["decode_o"][perm])
    np.testing.assert_array_equal(ref2["decode_lse"], ref["decode_lse"][perm])


def test_sampled_items_match_full():
    b = W.make_custom(4, 2, 64, [(64, 32)], [40, 77], seed=0)
    full = oracle.hybrid(b)
    ps = np.array([0, 5, 127])
    ds = np.array([1, 7])
    samp = oracle.hybrid(b, prefill_sample=ps, decode_sample=ds)
    np.testing.assert_array_equal(samp["prefill_o"], full["prefill_o"].reshape(-1, 64)[ps])
    np.testing.assert_array_equal(samp["decode_lse"], full["decode_lse"].reshape(-1)[ds])


def test_tiny_config_oracle_is_fast_and_finite():
    b = W.make_batch(W.CONFIGS["tiny"])
    ref = oracle.hybrid(b)
    assert ref["prefill_o"].shape == (32, 4, 64)
    assert ref["decode_o"].shape == (4, 4, 64)
    for v in ref.values():
        assert np.isfinite(v).all()
