"""The host planner of libpod_attn, run without a GPU.

`planner_harness.cpp` compiles the library's API translation unit with a
stand-in tensor-map encoder and prints the plan of one call as JSON. These
tests check the plan's invariants on explicit and random batches: every query
tile is covered once per KV split, units are ordered longest first, split
partials fit the context's buffers, decode units cover every request, the
split and policy rules hold, and oversize calls are refused.
"""
import json
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
QT = 128   # query rows per tile
KVT = 128  # keys per KV tile
POD_ECAPACITY = -6


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    gxx = shutil.which("g++")
    if not gxx or not os.path.exists(os.path.join(CUDA, "include", "cuda.h")):
        pytest.skip("g++ or the CUDA headers are missing")
    out = str(tmp_path_factory.mktemp("planner") / "planner_harness")
    subprocess.check_call([
        gxx, "-std=c++17", "-O1", "-w", "-I", os.path.join(ROOT, "include"),
        "-I", os.path.join(ROOT, "hybrid_prefill_decode_pod_b200", "csrc"),
        "-I", os.path.join(CUDA, "include"), "-o", out,
        os.path.join(ROOT, "tests", "planner_harness.cpp"),
        "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")])
    return out


def plan(harness, H, Hk, pre, dec, D=128, sms=148, decode_grid=296, policy=4, fused=True,
         pre_split=0, dec_split=0, paged=False, max_prefill_tokens=None, max_decode_reqs=None,
         max_kv=None):
    longest = max([p + c for p, c in pre] + list(dec) + [1])
    args = [harness, H, Hk, D, sms, decode_grid, policy, int(fused), pre_split, dec_split,
            int(paged), ",".join("%d:%d" % pc for pc in pre), ",".join(map(str, dec)),
            max_prefill_tokens or max(1, sum(c for _, c in pre)),
            max_decode_reqs or max(1, len(dec)), max_kv or longest]
    out = subprocess.run([str(a) for a in args], capture_output=True, text=True, check=True)
    return json.loads(out.stdout)


def covered_tiles(p, H, Hk):
    """(req, head, qtile, split) for every query tile the prefill units compute."""
    pair_heads = (H // Hk) % 2 == 0
    seen = []
    for req, head, qt, split in p["punits"]:
        n_qt = p["preq"][req]["n_qtiles"]
        if pair_heads:
            seen += [(req, head, qt, split), (req, head + 1, qt, split)]
        else:
            seen.append((req, head, qt, split))
            if qt + 1 < n_qt:
                seen.append((req, head, qt + 1, split))
    return seen


def unit_key(p, H, Hk, u):
    """KV tiles per split of a unit (the planner's longest-first key)."""
    req, head, qt, split = u
    r = p["preq"][req]
    last = qt if (H // Hk) % 2 == 0 else min(qt + 1, r["n_qtiles"] - 1)
    kv_hi = r["prior"] + min(r["chunk"], (last + 1) * QT)
    return (kv_hi + KVT - 1) // KVT // r["n_split"]


CASES = [
    (32, 8, [(4096, 512)], [4096] * 8),          # G = 4: head pairs
    (6, 2, [(900, 300)], [50, 700]),             # G = 3: token-tile pairs, 3 tiles
    (4, 4, [(1000, 64)], [2048, 31]),            # G = 1: a single tile (pair partner missing)
    (16, 2, [(0, 130), (77, 257)], [5, 4096]),   # G = 8, two requests, prior 0
    (8, 2, [(2000, 300), (0, 0), (5, 1)], []),   # prefill only, an empty chunk, one token
]


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("case", CASES)
def test_every_query_tile_once_per_split(harness, case, fused):
    H, Hk, pre, dec = case
    p = plan(harness, H, Hk, pre, dec, fused=fused)
    assert p["status"] == 0
    seen = covered_tiles(p, H, Hk)
    assert len(seen) == len(set(seen))
    want = set()
    for req, (prior, chunk) in enumerate(pre):
        r = p["preq"][req]
        assert r["n_qtiles"] == (chunk + QT - 1) // QT and r["kv_len"] == prior + chunk
        for h in range(H):
            for qt in range(r["n_qtiles"]):
                for s in range(r["n_split"]):
                    want.add((req, h, qt, s))
    assert set(seen) == want


@pytest.mark.parametrize("case", CASES)
def test_units_longest_first(harness, case):
    H, Hk, pre, dec = case
    p = plan(harness, H, Hk, pre, dec, fused=False)
    keys = [unit_key(p, H, Hk, u) for u in p["punits"]]
    assert keys == sorted(keys, reverse=True)


def test_fused_call_with_decodes_leaves_prefill_unsplit(harness):
    pre, dec = [(4096, 512)], [4096] * 64
    fused = plan(harness, 32, 8, pre, dec, fused=True)
    serial = plan(harness, 32, 8, pre, dec, fused=False)
    alone = plan(harness, 32, 8, pre, [], fused=True)
    assert fused["preq"][0]["n_split"] == 1 and len(fused["punits"]) == 64
    # without decodes in the launch the makespan model splits the 64 units
    assert serial["preq"][0]["n_split"] == alone["preq"][0]["n_split"] == 2
    assert len(serial["punits"]) == 128


def test_forced_split_respects_two_waves(harness):
    p = plan(harness, 8, 2, [(2000, 300)], [64], pre_split=3)
    assert p["preq"][0]["n_split"] == 3
    # 64 x 16 units would exceed 2 x 148 slots: the count is lowered until it fits
    p = plan(harness, 32, 8, [(8192, 512)], [64], pre_split=16)
    n = len(p["punits"])
    assert p["preq"][0]["n_split"] == 4 and n == 64 * 4 and n <= 2 * p["slots"]


def test_random_batches_fit_the_buffers(harness):
    rng = random.Random(7)
    for _ in range(40):
        Hk = rng.choice([1, 2, 4, 8])
        H = Hk * rng.choice([1, 2, 3, 4, 8])
        pre = [(rng.randrange(0, 20000), rng.randrange(0, 1500)) for _ in range(rng.randrange(0, 5))]
        dec = [rng.randrange(1, 30000) for _ in range(rng.randrange(0, 40))]
        fused = rng.random() < 0.5
        p = plan(harness, H, Hk, pre, dec, D=rng.choice([64, 128]), fused=fused,
                 sms=rng.choice([148, 132, 8]), paged=rng.random() < 0.3)
        assert p["status"] == 0
        c = p["caps"]
        assert len(p["punits"]) <= c["punits"]
        seen = covered_tiles(p, H, Hk)
        assert len(seen) == len(set(seen))
        for r in p["preq"]:
            if r["n_split"] > 1:  # split partials: one slot per (tile, head, split)
                assert r["slot0"] + r["n_qtiles"] * H * r["n_split"] <= c["pslots"]
                assert r["group0"] + r["n_qtiles"] * H <= c["pgroups"]
        # decode units: n_split x Hk consecutive units per request, all keys covered
        sl = p["dec_split_len"]
        if dec:
            assert sl % 16 == 0 and sl >= 256
        n_du = 0
        for i, r in enumerate(p["dreq"]):
            assert r["len"] == dec[i] and r["n_split"] == (dec[i] + sl - 1) // sl
            assert r["unit0"] == n_du
            assert p["dunit"][n_du:n_du + r["n_split"] * Hk] == [i] * (r["n_split"] * Hk)
            n_du += r["n_split"] * Hk
        assert len(p["dunit"]) == n_du <= c["dunits"]


def test_role_policies(harness):
    pre, dec = [(4096, 512)], [4096] * 64
    front = plan(harness, 32, 8, pre, dec, policy=4)
    assert front["flags"] & 0x200 and front["p_cap"] == front["slots"]
    assert front["rho"] == [1, 2]
    balanced = plan(harness, 32, 8, pre, dec, policy=5)
    assert balanced["flags"] & 0x400 and 1 <= balanced["p_cap"] < balanced["slots"]
    # proportional: the prefill share of claims follows the two queue lengths
    prop = plan(harness, 32, 8, pre, dec, policy=0)
    num, den = prop["rho"]
    assert num == len(prop["punits"]) and 0 < num < den


def test_tensor_maps_per_request(harness):
    p = plan(harness, 8, 2, [(100, 50), (0, 0), (7, 300)], [10])
    assert p["maps"] == 1 + 2 * 2  # Q, then K and V of each non-empty chunk
    p = plan(harness, 8, 2, [(100, 50), (7, 300)], [10], paged=True)
    assert p["maps"] == 3          # Q and the K / V pools


def test_oversize_calls_are_refused(harness):
    p = plan(harness, 8, 2, [(0, 64)], [10] * 5, max_decode_reqs=4)
    assert p["status"] == POD_ECAPACITY
    p = plan(harness, 8, 2, [(0, 300)], [10], max_prefill_tokens=200)
    assert p["status"] == POD_ECAPACITY
    p = plan(harness, 8, 2, [(1000, 64)], [10], max_kv=1000)
    assert p["status"] == POD_ECAPACITY
