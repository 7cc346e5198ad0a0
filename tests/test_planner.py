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
         max_kv=None, clusters=0):
    """Plan one call; clusters > 0 plans for the CTA-pair prefill kernel."""
    longest = max([p + c for p, c in pre] + list(dec) + [1])
    args = [harness, H, Hk, D, sms, decode_grid, policy, int(fused), pre_split, dec_split,
            int(paged), ",".join("%d:%d" % pc for pc in pre), ",".join(map(str, dec)),
            max_prefill_tokens or max(1, sum(c for _, c in pre)),
            max_decode_reqs or max(1, len(dec)), max_kv or longest, clusters]
    out = subprocess.run([str(a) for a in args], capture_output=True, text=True, check=True)
    return json.loads(out.stdout)


def tiles_of_unit(p, H, Hk, u):
    """(req, head, qtile) of the query tiles a unit computes."""
    req, head, qt = u[0], u[1], u[2]
    if (H // Hk) % 2 == 0:
        return [(req, head, qt), (req, head + 1, qt)]
    out = [(req, head, qt)]
    if qt + 1 < p["preq"][req]["n_qtiles"]:
        out.append((req, head, qt + 1))
    return out


def covered_tiles(p, H, Hk):
    """(req, head, qtile, split, n_split) for every query tile the units compute."""
    seen = []
    for u in p["punits"]:
        for t in tiles_of_unit(p, H, Hk, u):
            seen.append(t + (u[3], u[4]))
    return seen


def unit_kv_tiles(p, H, Hk, u):
    """KV tiles of a unit's whole (unsplit) key range."""
    req, qt = u[0], u[2]
    r = p["preq"][req]
    last = qt if (H // Hk) % 2 == 0 else min(qt + 1, r["n_qtiles"] - 1)
    kv_hi = r["prior"] + min(r["chunk"], (last + 1) * QT)
    return (kv_hi + KVT - 1) // KVT


def check_packing(p):
    """The call copies its plan packed: every table inside the copied bytes,
    the counters zeroed."""
    assert p["tables_inside_copy"] and p["counters_zeroed"]


def check_units(p, H, Hk, pre):
    """Every query tile of every request once per split of its unit, the
    splits of a unit partition its KV range, split units own distinct merge
    groups and partial slots inside the buffers, and the queue is ordered by
    split length, longest first."""
    seen = covered_tiles(p, H, Hk)
    assert len(seen) == len(set(seen))
    by_tile = {}
    for req, h, qt, s, n in seen:
        by_tile.setdefault((req, h, qt), []).append((s, n))
    want = set()
    for req, (prior, chunk) in enumerate(pre):
        r = p["preq"][req]
        assert r["n_qtiles"] == (chunk + QT - 1) // QT and r["kv_len"] == prior + chunk
        for h in range(H):
            for qt in range(r["n_qtiles"]):
                want.add((req, h, qt))
    assert set(by_tile) == want
    for splits in by_tile.values():
        n = splits[0][1]
        assert sorted(splits) == [(s, n) for s in range(n)]
    check_packing(p)
    c = p["caps"]
    groups, slots = set(), set()
    works = []
    for u in p["punits"]:
        req, head, qt, split, n, g0, s0, work = u
        total = unit_kv_tiles(p, H, Hk, u)
        assert work == (total * (split + 1)) // n - (total * split) // n
        if n > 1:
            assert work >= 4                      # a split keeps >= 4 KV tiles
            assert 0 <= g0 and g0 + 2 <= c["pgroups"] and 0 <= s0 and s0 + 2 * n <= c["pslots"]
            groups.add((g0, req, head, qt))
            for i in range(2):
                slots.add((s0 + i * n + split, req, head, qt))
        works.append(work)
    assert works == sorted(works, reverse=True)
    # distinct units own distinct groups and slots
    assert len({g for g, *_ in groups}) == len(groups)
    assert len({s for s, *_ in slots}) == len(slots)


CASES = [
    (32, 8, [(4096, 512)], [4096] * 8),          # G = 4: head pairs
    (6, 2, [(900, 300)], [50, 700]),             # G = 3: token-tile pairs, 3 tiles
    (4, 4, [(1000, 64)], [2048, 31]),            # G = 1: a single tile (pair partner missing)
    (16, 2, [(0, 130), (77, 257)], [5, 4096]),   # G = 8, two requests, prior 0
    (8, 2, [(2000, 300), (0, 0), (5, 1)], []),   # prefill only, an empty chunk, one token
]


@pytest.mark.parametrize("clusters", [0, 74])
@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("case", CASES)
def test_every_query_tile_once_per_split(harness, case, fused, clusters):
    H, Hk, pre, dec = case
    p = plan(harness, H, Hk, pre, dec, fused=fused, clusters=clusters)
    assert p["status"] == 0
    check_units(p, H, Hk, pre)


def test_fused_call_with_decodes_leaves_prefill_unsplit(harness):
    pre, dec = [(4096, 512)], [4096] * 64
    fused = plan(harness, 32, 8, pre, dec, fused=True)
    serial = plan(harness, 32, 8, pre, dec, fused=False)
    alone = plan(harness, 32, 8, pre, [], fused=True)
    # decode is the longer phase: the decode units fill the idle SMs
    assert fused["preq"][0]["n_split"] == 1 and len(fused["punits"]) == 64
    # without decodes in the launch the makespan model splits the 64 units
    assert serial["preq"][0]["n_split"] == alone["preq"][0]["n_split"] == 2
    assert len(serial["punits"]) == 128


def lpt_makespan(works, slots, overhead=2):
    """Finish time of a longest-first assignment of parts to slots."""
    import heapq
    q = [0] * slots
    for w in sorted(works, reverse=True):
        t = heapq.heappop(q) + w + overhead
        heapq.heappush(q, t)
    return max(q)


def test_pair_kernel_splits_the_tail_wave(harness):
    """Long-context prefill (64/8 heads, 1024 rows after 16384) on 74 CTA
    pairs: 256 pair units are 3.46 waves; splitting the units of the partial
    last wave in two shortens the finish time below that of no split and of
    any uniform split."""
    pre, dec = [(16384, 1024)], [20000 + 900 * i for i in range(16)]
    for fused in (False, True):
        p = plan(harness, 64, 8, pre, [], fused=fused, clusters=74)
        check_units(p, 64, 8, pre)
        splits = [u[4] for u in p["punits"]]
        n_split_units = len({(u[0], u[1], u[2]) for u in p["punits"] if u[4] > 1})
        assert n_split_units == 256 % 74 and set(splits) == {1, 2}
        works = [u[7] for u in p["punits"]]
        unsplit = [unit_kv_tiles(p, 64, 8, u) for u in p["punits"] if u[3] == 0]
        assert len(unsplit) == 256
        assert lpt_makespan(works, 74) < 0.97 * lpt_makespan(unsplit, 74)
        for s in (2, 3, 4):
            uniform = [(w * (k + 1)) // s - (w * k) // s for w in unsplit for k in range(s)]
            assert lpt_makespan(works, 74) <= lpt_makespan(uniform, 74)


def test_fused_call_with_decodes_keeps_the_last_wave_whole(harness):
    """One-SM tile, long-context batch: 256 units are 1.73 waves of 148 SMs.
    A launch of the prefill alone splits the last wave's 108 units in four
    (each SM then ends after 1.75 units of work, not 2); a fused launch that
    carries the decodes keeps them whole, so the SMs the last wave leaves
    free stream decode."""
    pre, dec = [(16384, 1024)], [20000 + 900 * i for i in range(16)]
    alone = plan(harness, 64, 8, pre, [], fused=False, clusters=0)
    check_units(alone, 64, 8, pre)
    parts = {}
    for u in alone["punits"]:
        parts.setdefault((u[0], u[1], u[2]), u[4])
    assert sorted(parts.values()).count(4) == 256 - 148
    assert sorted(parts.values()).count(1) == 148
    fused = plan(harness, 64, 8, pre, dec, fused=True, clusters=0)
    check_units(fused, 64, 8, pre)
    assert {u[4] for u in fused["punits"]} == {1} and len(fused["punits"]) == 256


def test_pair_kernel_maps_k_in_halves(harness):
    # contiguous: Q (128 rows), then per request K in 64-key halves, V in 128-key tiles
    p = plan(harness, 8, 2, [(100, 50), (7, 300)], [10], clusters=74)
    assert p["boxes"] == [128, 64, 128, 64, 128]
    p = plan(harness, 8, 2, [(100, 50), (7, 300)], [10], clusters=0)
    assert p["boxes"] == [128, 128, 128, 128, 128]
    # paged: one 16-key page per box for K and V
    p = plan(harness, 8, 2, [(100, 50), (7, 300)], [10], paged=True, clusters=74)
    assert p["boxes"] == [128, 16, 16]


def test_forced_split_respects_two_waves(harness):
    p = plan(harness, 8, 2, [(2000, 300)], [64], pre_split=3)
    assert {u[4] for u in p["punits"]} == {3}
    # 64 x 16 units would exceed 2 x 148 slots: the count is lowered until it fits
    p = plan(harness, 32, 8, [(8192, 512)], [64], pre_split=16)
    n = len(p["punits"])
    assert {u[4] for u in p["punits"]} == {4} and n == 64 * 4 and n <= 2 * p["slots"]


def test_plan_copy_is_packed(harness):
    # the long-context batch: 256 pair units, 16 decodes; the copy holds the
    # tables it uses, not the context's capacity
    pre, dec = [(16384, 1024)], [20000 + 900 * i for i in range(16)]
    p = plan(harness, 64, 8, pre, dec, clusters=74)
    check_packing(p)
    n_pu, n_du = len(p["punits"]), len(p["dunit"])
    assert p["plan_bytes"] <= 4096 + 64 * 8 + 32 * (1 + n_pu + len(dec)) + 4 * n_du + 6 * 64


def test_random_batches_fit_the_buffers(harness):
    rng = random.Random(7)
    for _ in range(40):
        Hk = rng.choice([1, 2, 4, 8])
        H = Hk * rng.choice([1, 2, 3, 4, 8])
        pre = [(rng.randrange(0, 20000), rng.randrange(0, 1500)) for _ in range(rng.randrange(0, 5))]
        dec = [rng.randrange(1, 30000) for _ in range(rng.randrange(0, 40))]
        fused = rng.random() < 0.5
        sms = rng.choice([148, 132, 8])
        D = rng.choice([64, 128])
        clusters = rng.choice([0, sms // 2]) if D == 128 else 0
        p = plan(harness, H, Hk, pre, dec, D=D, fused=fused, sms=sms,
                 paged=rng.random() < 0.3, clusters=clusters)
        assert p["status"] == 0
        c = p["caps"]
        assert len(p["punits"]) <= c["punits"]
        check_units(p, H, Hk, pre)
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
