"""The work schedules of the tensor-core GEMM kernels, on CPU: the library
lists the exact units its kernels run (tpmlp_schedule_units evaluates the
same functions the kernels call), and these tests check that every schedule
covers each output tile's K range exactly once, in pieces numbered in
ascending k, and that split tiles use distinct, in-bounds partial slots and
counters. Whole tiles; one unit per shard group; the stream-K tail."""
import random
from collections import defaultdict

import pytest

from tensor_transformer_mlp_block_b200 import binding

pytestmark = []


def _check(units, m_blocks, n_blocks, k_blocks, workers, sched, groups=1):
    tiles = m_blocks * n_blocks
    by_tile = defaultdict(list)
    for u in units:
        assert 0 <= u["worker"] < workers
        assert 0 <= u["mb"] < m_blocks and 0 <= u["nb"] < n_blocks
        assert 0 <= u["kb0"] < u["kb1"] <= k_blocks, u  # never empty
        by_tile[(u["mb"], u["nb"])].append(u)
    assert len(by_tile) == tiles  # every tile has work
    keys, slots = {}, set()
    for tile, us in by_tile.items():
        us.sort(key=lambda u: u["kb0"])
        # the K range exactly once, in consecutive pieces
        assert us[0]["kb0"] == 0 and us[-1]["kb1"] == k_blocks, (tile, us)
        for a, b in zip(us, us[1:]):
            assert a["kb1"] == b["kb0"], (tile, us)
        n = len(us)
        assert all(u["pieces"] == n for u in us), (tile, us)
        assert [u["piece"] for u in us] == list(range(n)), (tile, us)
        if n == 1:
            assert us[0]["key"] == -1 and us[0]["slot"] == -1
            continue
        # one counter index per split tile, distinct between tiles
        ks = {u["key"] for u in us}
        assert len(ks) == 1, (tile, us)
        k = ks.pop()
        assert k not in keys.values(), (tile, k)
        keys[tile] = k
        for u in us:
            assert u["slot"] not in slots, (tile, u)  # no two pieces share a partial tile
            slots.add(u["slot"])
    if sched == binding.SCHED_STREAMK:
        assert all(0 <= k < workers for k in keys.values())
        assert all(0 <= s < 2 * workers for s in slots)
        # each worker's k-blocks: whole-tile waves plus one segment
        work = defaultdict(int)
        for u in units:
            work[u["worker"]] += u["kb1"] - u["kb0"]
        assert max(work.values()) - min(work.values()) <= 1
        assert sum(work.values()) == tiles * k_blocks
    elif sched == binding.SCHED_GROUPS:
        assert len(keys) == tiles and all(0 <= k < tiles for k in keys.values())
        assert all(0 <= s < tiles * groups for s in slots)
        assert all(len(us) == groups for us in by_tile.values())
    else:
        assert not keys
    # each worker runs its units in its own order without gaps
    per = defaultdict(list)
    for u in units:
        per[u["worker"]].append(u["local"])
    for w, ls in per.items():
        assert ls == list(range(len(ls))), w


@pytest.mark.parametrize("m,n,k,P", [
    (8, 48, 768, 74),    # 175B-class row-parallel products (pair tiles, K = F)
    (8, 192, 192, 74),   # 175B-class F1 / B2
    (32, 16, 256, 74),   # 7B-class row-parallel products
    (12, 3, 64, 74),     # GPT-2-small weight gradients: fewer tiles than pairs
    (1, 1, 500, 74),     # one tile over every pair
    (75, 1, 400, 74),    # one tile past a full wave
    (5, 7, 33, 148),     # single-CTA geometry
])
def test_streamk_tail_covers_every_tile_once(m, n, k, P):
    units = binding.schedule_units(binding.SCHED_STREAMK, m, n, k, P)
    assert units is not None
    _check(units, m, n, k, P, binding.SCHED_STREAMK)
    # the tail is one segment per worker after floor(tiles / P) whole waves
    whole = (m * n) // P * P
    assert sum(1 for u in units if u["pieces"] == 1) >= whole


@pytest.mark.parametrize("m,n,k,P,S", [(8, 48, 768, 74, 8), (2, 2, 16, 74, 4), (3, 5, 12, 148, 3)])
def test_shard_groups_cover_every_tile_once(m, n, k, P, S):
    units = binding.schedule_units(binding.SCHED_GROUPS, m, n, k, P, groups=S)
    _check(units, m, n, k, P, binding.SCHED_GROUPS, S)


@pytest.mark.parametrize("m,n,k,P", [(32, 64, 64, 74), (1, 1, 1, 74), (3, 3, 5, 148)])
def test_whole_tiles(m, n, k, P):
    units = binding.schedule_units(binding.SCHED_TILES, m, n, k, P)
    _check(units, m, n, k, P, binding.SCHED_TILES)
    assert len(units) == m * n


def test_seeded_random_grids():
    rng = random.Random(7)
    checked = 0
    for _ in range(300):
        m, n = rng.randint(1, 40), rng.randint(1, 40)
        k = rng.randint(1, 400)
        P = rng.choice([1, 2, 7, 74, 148])
        units = binding.schedule_units(binding.SCHED_STREAMK, m, n, k, P)
        if units is None:
            # only where the kernels would not take the tail either
            tiles = m * n
            assert tiles % P == 0 or (tiles % P) * k < 4 * P
            continue
        _check(units, m, n, k, P, binding.SCHED_STREAMK)
        checked += 1
        S = rng.choice([2, 3, 4, 8])
        if k % S == 0:
            _check(binding.schedule_units(binding.SCHED_GROUPS, m, n, k, P, groups=S), m, n, k, P,
                   binding.SCHED_GROUPS, S)
    assert checked > 100


def test_invalid_schedules_are_refused():
    assert binding.schedule_units(binding.SCHED_STREAMK, 74, 1, 64, 74) is None  # no tail
    assert binding.schedule_units(binding.SCHED_STREAMK, 1, 1, 3, 74) is None    # too little work
    assert binding.schedule_units(binding.SCHED_GROUPS, 2, 2, 10, 74, groups=3) is None
    assert binding.schedule_units(7, 2, 2, 10, 74) is None
