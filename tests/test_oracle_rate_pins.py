"""Pins of the per-sketch rate oracle (format 1 with 2, 4 or 8 hash slots per
class) and of the space-allocation procedure ("UltraSketchLLM" explainer,
Resumen Tecnico, Metodologia §2: units of higher importance E[a^2] receive
larger sketch spaces).  Expected values come from the format-1 oracle (the
4-slot case is format 1), the independent brute force, closed forms and the
properties the allocation must have (budget, monotonicity, maximality, a
brute-force optimum on tiny cases)."""
import itertools

import numpy as np
import pytest

import gen
import oracle
from tests import brute_force


def test_four_slots_is_format_one():
    W = gen.weights_student_t(128, 1024, 3, 4.0, 0.02, 0.01, 20.0, "bf16")
    imp = gen.importance_lognormal(1024, 3)
    a = oracle.build_sketch_rate(W, imp, 5, 4)
    b = oracle.build_sketch(W, imp, 5)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def _brute_rate(W, imp, seed, slots):
    """Member lists with this file's own bucket function (8-bit codes)."""
    Wf = brute_force.to_f32(np.ascontiguousarray(W))
    M, K = Wf.shape
    impv = np.ones(K, np.float32) if imp is None else np.asarray(imp, np.float32)
    nb = M * K * slots // 64
    members = [[] for _ in range(nb)]
    for i in range(M):
        for j in range(K):
            rb, r = divmod(i, 64)
            tc, c = divmod(j, 256)
            z = brute_force.splitmix64_output(seed, rb * (K // 256) + tc + 1)
            A, C = (z & 0xFFFFFFFF) | 1, z >> 32
            o = c // 8
            h = (A * (32 * r + o) + C) & 0xFFFFFFFF
            b = (((slots * h) >> 32) * 32 + (o + r) % 32) * 8 + c % 8
            members[rb * slots * K + 256 * slots * tc + b].append(i * K + j)
    flat = Wf.reshape(-1)
    value = np.zeros(nb, np.float32)
    for b, mem in enumerate(members):
        if mem:
            q = sorted((-float(np.float32(abs(flat[m])) * impv[m % K]), m) for m in mem)[0][1]
            value[b] = flat[q]
    codes = np.zeros(nb, np.int8)
    scales = np.zeros(M // 64, np.uint16)
    per = slots * K
    for rb in range(M // 64):
        v = value[rb * per:(rb + 1) * per]
        s16 = np.float16(np.float32(np.max(np.abs(v))) / np.float32(127.0))
        scales[rb] = s16.view(np.uint16)
        s = np.float32(s16)
        if s != 0:
            codes[rb * per:(rb + 1) * per] = np.clip(np.rint(v / s), -127, 127).astype(np.int8)
    return codes, scales


@pytest.mark.parametrize("slots", [2, 8])
@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
@pytest.mark.parametrize("with_imp", [False, True])
def test_rate_build_matches_brute_force(slots, wdtype, with_imp):
    M, K, seed = 128, 512, 11 + slots
    W = gen.weights_student_t(M, K, seed, 4.0, 0.02, 0.01, 20.0, wdtype)
    imp = gen.importance_lognormal(K, seed) if with_imp else None
    o = oracle.build_sketch_rate(W, imp, seed, slots)
    assert o["status"] == oracle.OK
    codes, scales = _brute_rate(W, imp, seed, slots)
    assert np.array_equal(o["scales"], scales) and np.array_equal(o["codes"], codes)


@pytest.mark.parametrize("slots", [2, 4, 8])
def test_storage_and_members_per_bucket(slots):
    M, K = 64, 512
    o = oracle.build_sketch_rate(gen.weights_normal(M, K, 1, 0.02, "bf16"), None, 1, slots)
    assert o["codes"].nbytes * 8 == M * K * slots // 8  # slots/8 bit per weight
    cnt = np.zeros(M * K * slots // 64, np.int64)
    for i in range(M):
        for j in range(K):
            cnt[oracle.rate_bucket(K, 1, slots, i, j)] += 1
    assert cnt.mean() == 64 / slots
    # each (class, sub) owns one octet column per row: 64 members over `slots` slots
    t = cnt[:256 * slots].reshape(slots, 32, 8)
    assert np.all(t.sum(axis=0) == 64)


@pytest.mark.parametrize("slots", [2, 8])
def test_rate_gemv_matches_numpy(slots):
    M, K, seed = 128, 768, 4
    W = gen.weights_normal(M, K, seed, 0.02, "bf16")
    o = oracle.build_sketch_rate(W, None, seed, slots)
    x = gen.activations(3, K, seed, "bf16")
    s = np.repeat(o["scales"].view(np.float16).astype(np.float64), 64)
    Wh = np.zeros((M, K))
    for i in range(M):
        for j in range(K):
            Wh[i, j] = float(o["codes"][oracle.rate_bucket(K, seed, slots, i, j)]) * s[i]
    ref = gen.bf16_bits_to_f32(x).astype(np.float64) @ Wh.T
    y = oracle.gemv_rate_f64(o["codes"], o["scales"], M, K, x, seed, slots)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


# ---------------------------------------------------------------- allocation

def test_plan_uniform_importance_fills_budget_evenly():
    w = [4096 * 4096] * 7
    assert oracle.plan_slots(w, [1.0] * 7, 0.5) == [4] * 7
    assert oracle.plan_slots(w, [1.0] * 7, 0.25) == [2] * 7
    assert oracle.plan_slots(w, [1.0] * 7, 1.0) == [8] * 7


def test_plan_respects_budget_and_is_monotone_and_maximal():
    g = np.random.default_rng(5)
    for trial in range(50):
        n = int(g.integers(1, 40))
        w = [int(v) * 4096 for v in g.integers(1, 12, size=n)]
        imp = list(g.lognormal(0, 1.5, size=n))
        budget = float(g.uniform(0.25, 1.0))
        s = oracle.plan_slots(w, imp, budget)
        bits = sum(oracle.SLOT_BITS[si] * wi for si, wi in zip(s, w))
        assert bits <= budget * sum(w) + 1e-9
        for i in range(n):
            for j in range(n):
                if w[i] == w[j] and imp[i] > imp[j]:
                    assert s[i] >= s[j]
        # maximal: no single upgrade of a unit still fits
        for i in range(n):
            if s[i] < 8:
                extra = (oracle.SLOT_BITS[2 * s[i]] - oracle.SLOT_BITS[s[i]]) * w[i]
                assert bits + extra > budget * sum(w) + 1e-9


def test_plan_closed_forms():
    # two equal-size units: the importance order decides who gets the larger
    # space; a 4 -> 8 step costs twice a 2 -> 4 step
    assert oracle.plan_slots([1, 1], [10.0, 1.0], 0.75) == [8, 4]
    assert oracle.plan_slots([1, 1], [3.0, 1.0], 0.75) == [8, 4]
    assert oracle.plan_slots([1, 1], [3.0, 1.0], 0.5) == [4, 4]
    assert oracle.plan_slots([1, 1], [1.0, 3.0], 0.375) == [2, 4]
    # 8x the importance: its 4 -> 8 step (gain per bit 8 / 4 = 2) comes before
    # the others' 2 -> 4 steps (gain per bit 1); the budget then covers one more
    assert oracle.plan_slots([1, 1, 1, 1], [8.0, 1.0, 1.0, 1.0], 0.5) == [8, 4, 2, 2]
    # a large important unit and small unimportant ones under a tight budget
    assert oracle.plan_slots([4, 1, 1], [1.0, 0.5, 0.5], 0.5) == [4, 4, 4]
    assert oracle.plan_slots([4, 1, 1], [1.0, 0.5, 0.5], 0.45) == [4, 2, 2]


def test_plan_never_beats_the_exhaustive_optimum_and_reaches_it_without_a_tight_step():
    # the greedy never does better than the best of all 3^n assignments within
    # the budget (a pin on its budget accounting), and equals it when the budget
    # leaves no room for a 4 -> 8 step (all units at 2 or 4)
    g = np.random.default_rng(7)
    for trial in range(40):
        n = int(g.integers(1, 6))
        w = [int(v) for v in g.integers(1, 4, size=n)]
        imp = list(g.lognormal(0, 1, size=n))
        budget = float(g.uniform(0.25, 0.5))
        s = oracle.plan_slots(w, imp, budget)
        obj = sum(i * wi / si for i, wi, si in zip(imp, w, s))
        feas = [c for c in itertools.product((2, 4, 8), repeat=n)
                if sum(oracle.SLOT_BITS[x] * wi for x, wi in zip(c, w)) <= budget * sum(w) + 1e-12]
        best = min(sum(i * wi / si for i, wi, si in zip(imp, w, c)) for c in feas)
        assert obj >= best - 1e-12
        if all(x <= 4 for x in s) and all(w[0] == wi for wi in w):
            assert obj <= best + 1e-12 or any(c for c in feas if max(c) == 8)
