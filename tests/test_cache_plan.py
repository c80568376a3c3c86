"""moe_cache_plan, the host-side admission/eviction plan of the expert cache,
through the C ABI (no GPU: the call touches host memory only).

The plan is a reading (the pages say only that the most used experts stay in
VRAM and that the cache follows use), so it is pinned to the properties its
declaration states: free slots go to the strongest non-resident experts; with
hysteresis 1 and no move limit the residents afterwards are exactly the top
n_slots of (residents + non-residents with score > 0) when scores are
distinct (brute force over small random cases); every eviction passes the
hysteresis test and the first refused candidate fails it; a move limit keeps
a prefix of the unlimited plan; staying residents keep their slots; ties
resolve by id; bad arguments are refused."""
import numpy as np
import pytest

from bit_expert_ffn_route_b200 import build, moe


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.lib()


def _check_table(table, new_table, moves, slots):
    for slot, evict, admit in moves:
        assert new_table[admit] == slot
        assert table[admit] == -1
        if evict >= 0:
            assert table[evict] == slot and new_table[evict] == -1
        else:
            assert slot not in set(table[table >= 0].tolist())
    moved = {int(m[2]) for m in moves} | {int(m[1]) for m in moves if m[1] >= 0}
    for e in range(len(table)):
        if e not in moved:
            assert new_table[e] == table[e]
    used = new_table[new_table >= 0]
    assert len(set(used.tolist())) == len(used)
    assert set(used.tolist()) <= set(int(s) for s in slots)


def test_free_slots_go_to_the_strongest_candidates():
    score = np.array([0.0, 5.0, 1.0, 7.0, 5.0, 0.5], np.float32)
    table = np.full(6, -1, np.int32)
    table[2] = 40
    slots = np.array([40, 41, 42], np.int32)
    moves, new = moe.moe_cache_plan(score, table, slots)
    # candidates by score desc, id asc: 3 (7), 1 (5), 4 (5), 5 (0.5); expert 0 (score 0) never
    assert moves.tolist() == [[41, -1, 3], [42, -1, 1], [40, 2, 4]]
    _check_table(table, new, moves, slots)
    assert new[0] == -1 and new[5] == -1


@pytest.mark.parametrize("seed", range(40))
def test_top_n_of_eligible_with_distinct_scores(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(4, 24))
    n_slots = int(rng.integers(1, E))
    score = rng.permutation(E).astype(np.float32) * 0.25          # distinct, one of them 0
    slots = rng.permutation(1000)[:n_slots].astype(np.int32)
    table = np.full(E, -1, np.int32)
    n_res = int(rng.integers(0, n_slots + 1))
    for e, s in zip(rng.permutation(E)[:n_res], rng.permutation(slots)[:n_res]):
        table[e] = s
    moves, new = moe.moe_cache_plan(score, table, slots)
    _check_table(table, new, moves, slots)
    eligible = [e for e in range(E) if table[e] >= 0 or score[e] > 0]
    want = set(sorted(eligible, key=lambda e: -score[e])[:n_slots])
    assert set(np.nonzero(new >= 0)[0].tolist()) == want


def test_hysteresis_and_move_limit():
    rng = np.random.default_rng(7)
    E, n_slots, h = 64, 16, 1.5
    score = rng.random(E).astype(np.float32)
    slots = np.arange(100, 100 + n_slots, dtype=np.int32)
    table = np.full(E, -1, np.int32)
    table[:n_slots] = slots                                        # experts 0..15 resident
    moves, new = moe.moe_cache_plan(score, table, slots, hysteresis=h)
    _check_table(table, new, moves, slots)
    for slot, evict, admit in moves:
        assert evict >= 0 and score[admit] > h * score[evict]
    # the strongest candidate left fails against the weakest resident left
    res = [e for e in range(E) if new[e] >= 0 and table[e] >= 0]
    cand = [e for e in range(E) if new[e] < 0 and score[e] > 0]
    if cand and res:
        best = max(cand, key=lambda e: (score[e], -e))
        weak = min(res, key=lambda e: (score[e], -e))
        assert not score[best] > h * score[weak]
    for m in range(len(moves) + 1):
        part, _ = moe.moe_cache_plan(score, table, slots, hysteresis=h, max_moves=m)
        assert part.tolist() == moves[:m].tolist()


def test_equal_scores_resolve_by_id():
    score = np.array([1.0, 1.0, 1.0, 2.0, 2.0, 2.0], np.float32)
    table = np.array([10, 11, 12, -1, -1, -1], np.int32)
    slots = np.array([10, 11, 12], np.int32)
    moves, new = moe.moe_cache_plan(score, table, slots)
    # candidates 3, 4, 5 (ids ascending) replace residents weakest-first: highest id first
    assert moves.tolist() == [[12, 2, 3], [11, 1, 4], [10, 0, 5]]
    # equal scores never displace an incumbent
    moves, new = moe.moe_cache_plan(np.ones(6, np.float32), table, slots)
    assert len(moves) == 0 and np.array_equal(new, table)


@pytest.mark.parametrize("case", ["nan", "negative", "dup_slots", "foreign_slot", "shared_slot", "hysteresis"])
def test_bad_arguments_are_refused(case):
    score = np.ones(4, np.float32)
    table = np.array([5, -1, -1, -1], np.int32)
    slots = np.array([5, 6], np.int32)
    h = 1.0
    if case == "nan":
        score[1] = np.nan
    elif case == "negative":
        score[2] = -1.0
    elif case == "dup_slots":
        slots = np.array([5, 5], np.int32)
    elif case == "foreign_slot":
        table[1] = 9
    elif case == "shared_slot":
        table[1] = 5
    else:
        h = 0.5
    with pytest.raises(moe.MoeError):
        moe.moe_cache_plan(score, table, slots, hysteresis=h)
