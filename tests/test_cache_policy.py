"""CPU tests of the expert cache's placement policy (the host code that
decides which routed experts occupy the HBM slots of a cached layer):
least-recently-used eviction among experts that are neither pinned nor needed
by the current batch, pinned experts never evicted, best-effort prefetch
("Colibri: 2400 lines of pure C ...", section 二: per-layer LRU cache with a
learned hot set; the router one layer ahead).

A small driver compiled with g++ runs the policy; the expected placements of
a hand-worked scenario are written out below, and random streams are checked
against invariants and against a direct model of the rule.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("policy") / "cache_policy")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-o", exe, os.path.join(HERE, "native", "cache_policy_driver.cpp")])
    return exe


def run(driver, lines):
    out = subprocess.run([driver], input="\n".join(lines) + "\n", capture_output=True, text=True, check=True).stdout
    return out.split("\n")


def parse(out):
    """Replies in order: ('ok', [(e, s)...]) / ('full',) / ('ok',) / ('refused',) / ('slots', [...]) / ('stats', ...)."""
    res, i = [], 0
    while i < len(out):
        w = out[i].split()
        i += 1
        if not w:
            continue
        if w[0] == "ok" and len(w) == 2:
            n = int(w[1])
            res.append(("ok", [tuple(map(int, out[i + j].split())) for j in range(n)]))
            i += n
        elif w[0] == "slots":
            res.append(("slots", list(map(int, w[1:]))))
        elif w[0] == "uses":
            res.append(("uses", list(map(int, w[1:]))))
        elif w[0] in ("full", "ok", "refused"):
            res.append((w[0],))
        else:
            res.append(("stats", int(w[0]), int(w[1])))
    return res


def test_hand_worked_lru_scenario(driver):
    """E = 6 experts, R = 3 slots; experts 0, 1, 2 start in slots 0, 1, 2.
    [0]      hit                      (use order: 0)
    [3]      miss, evicts 1 (slot 1: never used; slot 2 also never used,
             the tie goes to the lower slot)
    [4, 0]   4 misses: candidates 2 (unused) and 3 (used at batch 2) -> 2 (slot 2)
    [5]      miss: LRU among 0 (batch 3), 3 (batch 2), 4 (batch 3) -> 3 (slot 1)
    pin [0] with reserve 2 -> ok (1 <= 3 - 2); [1, 2] miss twice: 0 is pinned,
             so they take slot 2 (4: batch 3) and slot 1 (5: batch 4)
    """
    out = parse(run(driver, ["init 6 3", "admit 1 0", "admit 1 3", "admit 2 4 0", "admit 1 5", "table",
                             "pin 2 1 0", "admit 2 1 2", "table", "stats"]))
    assert out[0] == ("ok", [])
    assert out[1] == ("ok", [(3, 1)])
    assert out[2] == ("ok", [(4, 2)])
    assert out[3] == ("ok", [(5, 1)])
    assert out[4] == ("slots", [0, -1, -1, -1, 2, 1])
    assert out[5] == ("ok",)
    assert out[6] == ("ok", [(1, 2), (2, 1)])
    assert out[7] == ("slots", [0, 2, 1, -1, -1, -1])
    assert out[8] == ("stats", 2, 5)
    assert out[9] == ("uses", [2, 1, 1, 1, 1, 1])


def test_a_batch_larger_than_the_free_slots_is_refused_unchanged(driver):
    out = parse(run(driver, ["init 5 2", "pin 0 1 0", "admit 2 3 4", "table", "admit 1 4", "table"]))
    assert out[0] == ("ok",)
    assert out[1] == ("full",)           # only slot 1 may be evicted, two experts are missing
    assert out[2] == ("slots", [0, 1, -1, -1, -1])
    assert out[3] == ("ok", [(4, 1)])
    assert out[4] == ("slots", [0, -1, -1, -1, 1])


def test_pin_limit(driver):
    out = parse(run(driver, ["init 8 4", "pin 2 3 0 1 2", "pin 2 2 0 1", "pin 2 1 8", "pin 2 2 5 5"]))
    assert out == [("refused",), ("ok",), ("refused",), ("ok",)]   # duplicates count once


def test_prefetch_is_best_effort_and_counts_nothing(driver):
    out = parse(run(driver, ["init 6 3", "pin 1 2 0 1", "prefetch 3 3 4 5", "table", "stats"]))
    assert out[1] == ("ok", [(3, 2)])       # one unpinned slot: 3 takes it, 4 and 5 do not fit
    assert out[2] == ("slots", [0, 1, -1, 2, -1, -1])
    assert out[3] == ("stats", 0, 0)


def lru_model(E, R, batches, pinned=()):
    """Slots with the batch index of their last use (0 at the start); a miss
    takes the slot of the expert used least recently, ties to the lower slot,
    among experts neither pinned nor in the batch."""
    slot_expert = list(range(min(E, R)))
    last = [0] * R
    hits = misses = 0
    for j, b in enumerate(batches, start=1):
        need = list(dict.fromkeys(b))
        given = []
        for e in need:
            if e in slot_expert:
                hits += 1
                continue
            misses += 1
            cands = [s for s in range(R) if s not in given and slot_expert[s] not in pinned
                     and slot_expert[s] not in need]
            s = min(cands, key=lambda s: (last[s], s))
            given.append(s)
            slot_expert[s] = e
        for e in need:
            last[slot_expert.index(e)] = j
    return set(slot_expert), hits, misses


@pytest.mark.parametrize("seed", range(4))
def test_random_zipf_stream_matches_lru_model_and_invariants(driver, seed):
    rng = np.random.default_rng(seed)
    E, R, K = 40, 12, 4
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    batches = [list(rng.choice(E, size=K, replace=False, p=p)) for _ in range(300)]
    lines = [f"init {E} {R}"]
    for b in batches:
        lines += [f"admit {len(b)} " + " ".join(map(str, b)), "table"]
    lines.append("stats")
    out = parse(run(driver, lines))
    for j, b in enumerate(batches):
        copies, table = out[2 * j][1], out[2 * j + 1][1]
        resident = [e for e in range(E) if table[e] >= 0]
        assert len(resident) == R and len(set(table[e] for e in resident)) == R
        assert all(table[e] >= 0 for e in b)
        assert all(table[e] == s for e, s in copies)
    model_set, hits, misses = lru_model(E, R, batches)
    assert out[-2] == ("stats", hits, misses)
    final = out[-3][1]
    assert {e for e in range(E) if final[e] >= 0} == model_set
