"""Pins of the oracle's dispatch layout: the page's example routings (counts by
hand), brute force over every tiny routing with a counting definition that
does not sort, and invariants on seeded workloads."""
import itertools

import numpy as np
import pytest

import oracle
import workloads
from golden_io import read


def _check_invariants(idx, counts, send, assist, num_experts, n_ids, a_cap, mask=None):
    bs, k = idx.shape
    r = int(send[-1])
    assert send[0] == 0 and np.all(np.diff(send) == counts) and counts.sum() == r
    assert r <= a_cap
    slot_of = assist[a_cap:]
    pair_of = assist[:a_cap]
    assert np.all(pair_of[r:] == -1)
    # slot list and pair list are inverse bijections on [0, R)
    assert np.array_equal(np.sort(pair_of[:r]), np.sort(np.nonzero(slot_of >= 0)[0]))
    assert np.all(slot_of[pair_of[:r]] == np.arange(r))
    # every slot sits inside its expert's segment, tokens ascend in a segment
    for e in range(num_experts):
        seg = pair_of[send[e]:send[e + 1]]
        assert np.all(idx.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg // k) > 0)


@pytest.mark.parametrize("name", ["layout_single_op_example.txt",
                                  "layout_graph_mode_example.txt"])
def test_page_examples(name):
    g = read(name)
    idx = np.array(g["topk_idx"], np.int32)
    e = g["num_experts"]
    n = e + g["zero_expert_num"] + g["copy_expert_num"] + g["const_expert_num"]
    bs, k = idx.shape
    a_cap = bs * k
    counts, send, assist, st = oracle.dispatch_layout(idx, e, n, a_cap)
    assert st == 0
    assert counts.tolist() == g["expert_token_nums"]
    assert int(send[-1]) == g["routed_total"]
    head = g["assist_head"]
    assert assist[:len(head)].tolist() == head
    specials = {(t, kk) for (t, kk, _) in g["special_pairs"]}
    for t in range(bs):
        for kk in range(k):
            has_slot = assist[a_cap + t * k + kk] >= 0
            assert has_slot == ((t, kk) not in specials)
    _check_invariants(idx, counts, send, assist, e, n, a_cap)


def _brute(idx, e_routed, n_ids, a_cap, mask):
    """slot(t,k) = start of expert e + number of earlier tokens routed to e,
    where start of e = number of routed pairs with a smaller expert id."""
    bs, k = idx.shape
    status = 0
    routed = np.zeros((bs, k), bool)
    for t in range(bs):
        for kk in range(k):
            v = idx[t, kk]
            if v < 0 or v >= n_ids:
                status |= 1
                continue
            if v in idx[t, :kk]:
                status |= 2
                continue
            act = True if mask is None else (mask[t] if mask.ndim == 1 else mask[t, kk])
            routed[t, kk] = bool(act) and v < e_routed
    counts = np.array([int(np.sum(routed & (idx == e))) for e in range(e_routed)], np.int32)
    slots = np.full(bs * k, -1, np.int64)
    for t in range(bs):
        for kk in range(k):
            if routed[t, kk]:
                e = idx[t, kk]
                start = int(np.sum(routed & (idx < e)))
                earlier = int(np.sum(routed[:t] & (idx[:t] == e)))
                slots[t * k + kk] = start + earlier
    return counts, slots, status


def test_brute_force_all_tiny_routings():
    cases = 0
    for e_routed, specials, k, bs in [(3, 1, 2, 3), (4, 0, 2, 3), (2, 2, 1, 3), (4, 0, 3, 2)]:
        n = e_routed + specials
        rows = list(itertools.permutations(range(n), k))
        for routing in itertools.product(rows, repeat=bs):
            idx = np.array(routing, np.int32).reshape(bs, k)
            a_cap = bs * k
            counts, send, assist, st = oracle.dispatch_layout(idx, e_routed, n, a_cap)
            bc, bslots, bst = _brute(idx, e_routed, n, a_cap, None)
            assert st == bst == 0
            assert np.array_equal(counts, bc)
            assert np.array_equal(assist[a_cap:], bslots)
            cases += 1
    assert cases > 3000


def test_brute_force_masks_and_invalid_ids():
    rng = np.random.default_rng(3)
    vals = [-1, 0, 1, 2, 3, 4]  # 4 is out of range for n_ids = 4
    for row0 in itertools.product(vals, repeat=2):
        for row1 in itertools.product(vals, repeat=2):
            idx = np.array([row0, row1], np.int32)
            for mask in (None, rng.integers(0, 2, 2).astype(np.uint8),
                         rng.integers(0, 2, (2, 2)).astype(np.uint8)):
                counts, send, assist, st = oracle.dispatch_layout(idx, 3, 4, 4, mask)
                bc, bslots, bst = _brute(idx, 3, 4, 4, mask)
                assert st == bst
                assert np.array_equal(counts, bc)
                assert np.array_equal(assist[4:], bslots)


@pytest.mark.parametrize("wl", workloads.WORKLOADS, ids=lambda w: w.name)
def test_invariants_on_workloads(wl):
    small = wl.scaled(bs=min(wl.bs, 512), h=64)
    inp = workloads.generate(small)
    counts, send, assist, st = oracle.dispatch_layout(
        inp["topk_idx"], small.num_experts, small.n_ids, small.a_capacity, inp["mask"])
    assert st == 0
    _check_invariants(inp["topk_idx"], counts, send, assist, small.num_experts, small.n_ids,
                      small.a_capacity, inp["mask"])
    if small.n_ids == small.num_experts and inp["mask"] is None:
        assert int(send[-1]) == small.bs * small.k  # every pair routed, distinct per row
