"""The persistent grid's work partition (tfa_plan_pieces), checked on the CPU
against the per-tile key ranges of tfa_plan_qtile: every key-tile step of
every query tile is done exactly once, split tiles have exactly one
finalizer whose merge list names exactly the CTAs holding the rest, those
pieces never wait (they are the first piece of their CTA), and the split
schedule gives every CTA the same amount of work to within one step.  With
head pairs (split bit 2, for an even number of query heads per KV group) an
item is one query tile of two heads, both tiles with that tile's key range."""
from collections import defaultdict

import pytest

from sliding_window_gqa_tfa_b200 import binding as tb
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS

CASES = [(w.B, w.Hq, w.L, w.S, w.causal, w.window) for w in WORKLOADS.values() if w.L >= 9] + [
    (1, 1, 256, 1 << 20, True, 0),      # one item far longer than a CTA's share
    (2, 3, 300, 301, True, 0),
    (1, 4, 130, 700, True, 129),
    (3, 2, 9, 9, True, 0),
    (1, 2, 1000, 5000, False, 0),
]


def _tile_range(L, S, causal, window, qp, t, hp=0):
    qt = qp if hp else 2 * qp + t
    if qt * 128 >= L:
        return None
    rc, lo, hi, _ = tb.tfa_plan_qtile(L, S, causal, window, 0, qt)
    assert rc == 0
    return lo, hi


@pytest.mark.parametrize("hp", [0, 1], ids=["tile_pairs", "head_pairs"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("grid", [148, 37, 1])
def test_split_schedule_partitions_every_tile_exactly(case, grid, hp):
    B, Hq, L, S, causal, window = case
    if hp and Hq % 2:
        pytest.skip("head pairs need an even head count")
    split = 1 | (2 if hp else 0)
    rc, W, _ = tb.tfa_plan_pieces(B, Hq, L, S, causal, window, 1, split, 0, max_pieces=1 << 16)
    assert rc == 0
    grid = min(grid, W)
    per_cta, cover = [], defaultdict(list)
    first_piece = {}
    for c in range(grid):
        rc, W2, pieces = tb.tfa_plan_pieces(B, Hq, L, S, causal, window, grid, split, c,
                                            max_pieces=1 << 16)
        assert rc == 0 and W2 == W
        per_cta.append(sum(p[5] - p[4] + 1 for p in pieces))
        for k, p in enumerate(pieces):
            cover[p[0]].append((c, k, p))
            if k == 0:
                first_piece[c] = p
    assert sum(per_cta) == W
    assert max(per_cta) - min(per_cta) <= 1
    n_qp = (L + 127) // 128 if hp else (L + 255) // 256
    assert len(cover) == B * (Hq // 2 if hp else Hq) * n_qp
    for item, lst in cover.items():
        qp = lst[0][2][1]
        for t in range(2):
            rng = _tile_range(L, S, causal, window, qp, t, hp)
            active = [(c, k, p) for c, k, p in lst if p[6 + t] & 1]
            if rng is None:
                assert not active
                continue
            lo, hi = rng
            steps = sorted(j for _, _, p in active
                           for j in range(max(p[4], lo), min(p[5], hi) + 1))
            assert steps == list(range(lo, hi + 1)), (item, t)
            fins = [(c, k, p) for c, k, p in active if p[6 + t] & 2]
            assert len(fins) == 1
            c_f, _, p_f = fins[0]
            assert p_f[4] <= lo
            others = sorted(c for c, _, p in active if c != c_f)
            if not others:
                assert p_f[6 + t] & 4 and p_f[8 + t] == -1
            else:
                assert not p_f[6 + t] & 4
                assert others == list(range(c_f + 1, p_f[8 + t] + 1))
                for c in others:  # contributors: their CTA's first piece, not a finalizer
                    assert first_piece[c][0] == item
                    assert not first_piece[c][6 + t] & 2


@pytest.mark.parametrize("hp", [0, 1], ids=["tile_pairs", "head_pairs"])
@pytest.mark.parametrize("case", CASES[:6], ids=lambda c: "x".join(map(str, c)))
def test_whole_item_schedule_deals_each_item_once(case, hp):
    B, Hq, L, S, causal, window = case
    if hp and Hq % 2:
        pytest.skip("head pairs need an even head count")
    n_items = B * (Hq // 2 * ((L + 127) // 128) if hp else Hq * ((L + 255) // 256))
    grid = min(148, n_items)
    seen = []
    for c in range(grid):
        rc, _, pieces = tb.tfa_plan_pieces(B, Hq, L, S, causal, window, grid, 2 if hp else 0, c)
        assert rc == 0
        for p in pieces:
            assert p[6] & 4 and (p[7] & 4 or not p[7] & 1)
        seen += [p[0] for p in pieces]
        # snake order: c, 2G-1-c, 2G+c, 4G-1-c, ... (each round reverses the last)
        want, item, stride = [], c, 2 * grid - 1 - 2 * c
        while item < n_items:
            want.append(item)
            item, stride = item + stride, 2 * grid - stride
        assert [p[0] for p in pieces] == want
    assert sorted(seen) == list(range(n_items))


def test_plan_pieces_rejects_bad_grid():
    assert tb.tfa_plan_pieces(1, 8, 33, 47, 1, 0, 0, 1, 0)[0] == tb.TFA_ERR_SHAPE
    assert tb.tfa_plan_pieces(1, 8, 33, 47, 1, 0, 4, 1, 4)[0] == tb.TFA_ERR_SHAPE
    assert tb.tfa_plan_pieces(1, 7, 300, 300, 1, 0, 4, 3, 0)[0] == tb.TFA_ERR_SHAPE  # odd head count
