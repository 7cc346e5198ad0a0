"""Host-side checks of the seeded input generator (no GPU, no attention math)."""
import math

import torch

from hybrid_prefill_decode_pod_b200 import workloads as W


def test_tiny_config_shapes_and_determinism():
    a = W.make_batch(W.CONFIGS["tiny"])
    b = W.make_batch(W.CONFIGS["tiny"])
    assert a.q_prefill.shape == (32, 4, 64) and a.q_prefill.dtype == torch.bfloat16
    assert [k.shape[0] for k in a.k_prefill] == [96]
    assert a.ctx == [40, 77, 128, 200]
    assert torch.equal(a.q_prefill, b.q_prefill)
    assert torch.equal(a.v_decode[3], b.v_decode[3])


def test_ranged_contexts_inclusive_and_seeded():
    cfg = W.HybridConfig("t", 4, 2, 16, prefill=((1, 1),), decode_range=(3, 5, 400))
    b = W.make_batch(cfg)
    assert min(b.ctx) == 3 and max(b.ctx) == 5
    assert W.make_batch(cfg).ctx == b.ctx


def test_paged_pool_holds_the_same_values():
    b = W.make_custom(4, 2, 16, [(20, 13), (0, 5)], [1, 16, 17, 40], seed=3, paged=True)
    page = W.PAGE_SIZE
    lens = b.kv_lens_prefill + b.ctx
    ks = b.k_prefill + b.k_decode
    vs = b.v_prefill + b.v_decode
    tables = list(b.block_table_prefill) + list(b.block_table_decode)
    used = []
    for L, k, v, tab in zip(lens, ks, vs, tables):
        for j in range(L):
            blk = int(tab[j // page])
            used.append(blk)
            assert torch.equal(b.k_pool[blk, j % page], k[j])
            assert torch.equal(b.v_pool[blk, j % page], v[j])
    total = sum(math.ceil(L / page) for L in lens)
    assert b.k_pool.shape[0] == total
    assert sorted(set(used)) == list(range(total))


def test_paged_and_contiguous_variants_share_values():
    cfg = W.CONFIGS["tiny"]
    a = W.make_batch(cfg)
    b = W.make_batch(cfg, with_pool=True)
    assert torch.equal(a.k_decode[2], b.k_decode[2])
    assert b.k_pool is not None and a.k_pool is None


def test_algorithmic_work_counts():
    # one prefill request prior 0 chunk 2 (keys 1 and 2) and one decode of 3 keys, H = Hk = d = 1
    f_p, f_d, b_p, b_d = W.algorithmic_work(1, 1, 1, [0], [2], [3])
    assert f_p == 4 * (1 + 2)
    assert f_d == 4 * 3
    assert b_p == 2 * 2 * 2 + 2 * 2 * 2 + 2 * 4
    assert b_d == 3 * 2 * 2 + 2 * 2 + 4


def test_chunked_16k_sweep_points():
    """Chunk i of a 16K prompt: prior 512 i, a 512-token chunk, 64 decodes at the
    context the prompt has reached."""
    for i in (0, 5, 31):
        c = W.get_config("chunked16k_%d" % i)
        assert (c.num_qo_heads, c.num_kv_heads, c.head_dim) == (32, 8, 128)
        assert c.prefill == ((512 * i, 512),)
        assert c.decode_ctx == (512 * (i + 1),) * 64
        assert "chunked16k_%d" % i in W.CONFIG_DESCRIPTIONS
    assert sum(k.startswith("chunked16k_") for k in W.PROBE_CONFIGS) == 32
