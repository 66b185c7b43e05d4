"""Pins of the split-KV scheduler specification (oracle side).

The pages give only the call shape of the metadata pass (OpenSourceWeek Day 1 - FlashMLA,
section V.2); the plan is this library's own specification, so these tests pin it by
hand-worked cases and by the invariants any correct split plan must satisfy.
"""

import json
import os
import random

import pytest

from oracle import metadata as M

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_cases():
    spec = json.load(open(os.path.join(GOLDEN, "metadata_cases.json")))
    for case in spec["cases"]:
        tiles, splits = M.schedule(case["seqlens"], case["num_parts"], case["rows_per_kv_head"])
        assert tiles == case["tiles"], case["work"]
        assert splits == case["num_splits"], case["work"]


def check_plan(lens, num_parts, tiles, splits, R=16):
    """Coverage: every page of every sequence exactly once, in order; split counts agree;
    no part does more than payload + OVH units of work; ordinals count earlier parts
    touching a sequence."""
    OVH = M.overhead_pages(R)
    payload = M.payload_of(lens, num_parts, R) + OVH
    assert len(tiles) == num_parts and len(splits) == len(lens) + 1 and splits[0] == 0
    segs = M.segments(tiles, lens)
    cursor = {}
    touched = [0] * len(lens)
    seen_ord = [0] * len(lens)
    for part in segs:
        cost = 0
        for (b, t0, t1, ordv) in part:
            assert t0 % M.PAGE == 0
            assert cursor.get(b, 0) == t0, "pieces must continue where the last one ended"
            assert t1 > t0 or (lens[b] == 0 and t0 == t1 == 0)
            assert t1 <= lens[b]
            assert ordv == seen_ord[b]
            seen_ord[b] += 1
            touched[b] += 1
            cursor[b] = t1
            cost += -(-(t1 - t0) // M.PAGE) + OVH
        assert cost <= payload
    for b, L in enumerate(lens):
        assert cursor.get(b, None) == L, f"sequence {b} not fully covered"
        assert splits[b + 1] - splits[b] == touched[b]
    # sequences are visited in order across parts
    order = [b for part in segs for (b, *_rest) in part]
    assert order == sorted(order)


@pytest.mark.parametrize("seed", range(40))
def test_random_plans_cover_everything(seed):
    rng = random.Random(seed)
    B = rng.randint(1, 40)
    lens = [rng.choice([0, 1, 63, 64, 65, rng.randint(1, 5000), rng.randint(1, 70000)]) for _ in range(B)]
    num_parts = rng.randint(1, 160)
    R = rng.choice([1, 16, 33, 64, 128, 256, 1000])
    tiles, splits = M.schedule(lens, num_parts, R)
    check_plan(lens, num_parts, tiles, splits, R)


def test_workload_plans():
    from paged_mla_decode_11_b200 import workloads as W
    for w in W.WORKLOADS.values():
        lens = W._draw_seqlens(w, __import__("torch").Generator().manual_seed(0)).tolist()
        parts = M.num_parts_for(148, w.rows_per_kv_head, w.h_kv)
        tiles, splits = M.schedule(lens, parts, w.rows_per_kv_head)
        check_plan(lens, parts, tiles, splits, w.rows_per_kv_head)


def test_num_parts_formula():
    assert M.num_parts_for(148, 16, 1) == 148
    assert M.num_parts_for(148, 64, 1) == 148
    assert M.num_parts_for(148, 128, 1) == 74
    assert M.num_parts_for(148, 256, 1) == 37
    assert M.num_parts_for(148, 128, 2) == 37
    assert M.num_parts_for(4, 4096, 1) == 1


def test_overhead_pages():
    assert [M.overhead_pages(r) for r in (1, 16, 32, 33, 64, 128, 256)] == [1, 1, 1, 2, 2, 4, 8]
