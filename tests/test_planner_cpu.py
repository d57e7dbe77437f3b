"""The weight-page bitwidth planner (host code in the library) against the
plain oracle restatement, and the oracle against a hand-worked example,
exhaustive search and invariants (PagedWeight: Efficient MoE LLM Serving with
Dynamic Quality-Aware Weight Quantization, 'What carries the argument' and
Figure 4)."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import planner as op

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = json.load(open(os.path.join(ROOT, "tests", "golden", "planner_example.json")))


def _blocks(golden_blocks, committed=None):
    out = []
    for i, b in enumerate(golden_blocks):
        d = dict(b)
        d["sensitivity"] = {int(k): float(np.float32(v)) for k, v in b["sensitivity"].items()}
        for k in (3, 4):
            d["sensitivity"].setdefault(k, 0.0)
        d["routing_mult"] = float(np.float32(b["routing_mult"]))
        d["prompt_factor"] = float(np.float32(b["prompt_factor"]))
        if committed is not None:
            d["committed_bits"] = committed[i]
            d["floor_bits"] = min(d["floor_bits"], committed[i])
        out.append(d)
    return out


@pytest.fixture(scope="module")
def bq():
    from bit_quantized_moe_top_b200 import build
    build.build()
    import bit_quantized_moe_top_b200 as m
    return m


EPS = float(np.float32(GOLDEN["eps"]))


@pytest.mark.parametrize("case", GOLDEN["reduce"], ids=lambda c: str(c["bytes_target"]))
def test_oracle_reduce_golden(case):
    met, bits, rel = op.plan_reduce(_blocks(GOLDEN["blocks"]), case["bytes_target"], EPS)
    assert (met, bits, rel) == (case["met"], case["new_bits"], case["bytes_released"])


def test_oracle_restore_golden():
    r = GOLDEN["restore"]
    bits, used = op.plan_restore(_blocks(GOLDEN["blocks"], r["committed_bits"]), r["max_bits"], r["bytes_budget"], EPS)
    assert (bits, used) == (r["new_bits"], r["bytes_used"])


def _random_blocks(rng, n, equal_bytes=False, convex=False):
    blocks = []
    for _ in range(n):
        q = int(rng.integers(2, 5))
        g3, g4 = (float(np.float32(x)) for x in rng.uniform(0, 2, 2))
        if convex:  # dropping the 4th plane hurts no more than dropping the 3rd
            g3, g4 = max(g3, g4), min(g3, g4)
        blocks.append({"committed_bits": q, "floor_bits": int(rng.integers(2, q + 1)),
                       "max_steps": int(rng.integers(0, 3)),
                       "plane_bytes": 64 if equal_bytes else int(rng.integers(1, 5)) * 32,
                       "sensitivity": {3: g3, 4: g4},
                       "routing_mult": float(np.float32(rng.choice([0.5, 1.0, 2.0]))),
                       "prompt_factor": float(np.float32(rng.uniform(0.5, 1.5)))})
    return blocks


def test_oracle_greedy_is_optimal_when_convex():
    """Equal plane sizes and per-block damages that grow with depth: taking the
    m cheapest actions one at a time is the minimum-damage way to drop m
    planes, which exhaustive search over all bit assignments confirms."""
    rng = np.random.default_rng(3)
    for _ in range(40):
        blocks = _random_blocks(rng, 4, equal_bytes=True, convex=True)
        eps = 0.05
        for m in range(1, 6):
            met, bits, rel = op.plan_reduce(blocks, m * 64, eps)
            lows = [max(b["floor_bits"], b["committed_bits"] - b["max_steps"]) for b in blocks]
            ranges = [range(lo, b["committed_bits"] + 1) for lo, b in zip(lows, blocks)]
            best = None
            for cand in itertools.product(*ranges):
                drop = sum(b["committed_bits"] - c for b, c in zip(blocks, cand))
                if drop != m:
                    continue
                dmg = sum(op.damage(b, x, eps) for b, c in zip(blocks, cand)
                          for x in range(c + 1, b["committed_bits"] + 1))
                best = dmg if best is None else min(best, dmg)
            if best is None:
                assert not met
                continue
            got = sum(op.damage(b, x, eps) for b, c in zip(blocks, bits) for x in range(c + 1, b["committed_bits"] + 1))
            assert met and rel == m * 64
            assert got == pytest.approx(best, rel=1e-12, abs=1e-15)


def test_oracle_invariants():
    rng = np.random.default_rng(4)
    for _ in range(60):
        blocks = _random_blocks(rng, 6)
        prev = None
        for target in range(0, 1200, 96):
            met, bits, rel = op.plan_reduce(blocks, target, 0.01)
            for b, x in zip(blocks, bits):
                assert max(b["floor_bits"], b["committed_bits"] - b["max_steps"]) <= x <= b["committed_bits"]
            assert rel == sum((b["committed_bits"] - x) * b["plane_bytes"] for b, x in zip(blocks, bits))
            assert met == (rel >= target)
            if prev is not None:  # a larger target extends the smaller target's plan
                assert all(x <= y for x, y in zip(bits, prev))
            prev = bits


@pytest.mark.parametrize("case", GOLDEN["reduce"], ids=lambda c: str(c["bytes_target"]))
def test_library_reduce_golden(bq, case):
    st, bits, rel = bq.moe_plan_reduce(_blocks(GOLDEN["blocks"]), case["bytes_target"], EPS)
    assert (st == 0, bits, rel) == (case["met"], case["new_bits"], case["bytes_released"])


def test_library_restore_golden(bq):
    r = GOLDEN["restore"]
    bits, used = bq.moe_plan_restore(_blocks(GOLDEN["blocks"], r["committed_bits"]), r["max_bits"], r["bytes_budget"],
                                     EPS)
    assert (bits, used) == (r["new_bits"], r["bytes_used"])


def test_library_matches_oracle_random(bq):
    rng = np.random.default_rng(5)
    for trial in range(200):
        blocks = _random_blocks(rng, int(rng.integers(1, 9)))
        eps = float(np.float32(rng.choice([0.0, 0.01, 0.5])))
        target = int(rng.integers(0, 1500))
        met, bits, rel = op.plan_reduce(blocks, target, eps)
        st, lbits, lrel = bq.moe_plan_reduce(blocks, target, eps)
        assert (st == 0, lbits, lrel) == (met, bits, rel), trial
        max_bits = [int(rng.integers(b["committed_bits"], 5)) for b in blocks]
        budget = int(rng.integers(0, 1000))
        assert bq.moe_plan_restore(blocks, max_bits, budget, eps) == op.plan_restore(blocks, max_bits, budget, eps)


def test_library_rejects_bad_plans(bq):
    good = _blocks(GOLDEN["blocks"])
    for field, value in [("committed_bits", 5), ("floor_bits", 1), ("plane_bytes", 0), ("max_steps", -1),
                         ("routing_mult", -1.0)]:
        bad = [dict(b) for b in good]
        bad[1][field] = value
        with pytest.raises(bq.MoEError) as ei:
            bq.moe_plan_reduce(bad, 100, EPS)
        assert ei.value.status == 1
    with pytest.raises(bq.MoEError):
        bq.moe_plan_reduce(good, -1, EPS)
    with pytest.raises(bq.MoEError):
        bq.moe_plan_restore(good, [3, 4, 3, 4], 100, EPS)  # A's max below its committed bits
