"""CPU checks of the split-KV work plan, through la_pbd_plan (the same plan code the attention
kernels run on the device, evaluated on the host).

The plan must cover the visible keys [0, P_b + W) of every (sequence, KV head) exactly once,
in whole key tiles (only a sequence's last tile may be short, and no tile is shared by two
CTAs), give every CTA at most its share of plan units (its tiles, plus the fixed segment cost
of every segment after its first, which starts a sequence inside the CTA's run), mark a
segment as whole exactly when it is the only segment of its sequence, and hand partial
segments distinct workspace slots below num_ctas + B * Hkv (the slot count the workspace is
sized for)."""
import random

import torch

import pytest

import block_masked_window_b200 as bmw


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_masked_window_b200 import build
    build.build()
    bmw.load()


def check_plan(seq_lens, W, S, Hkv, num_ctas, unit, Hq=None, seg=0):
    Hq = Hq or 8 * Hkv
    cfg = bmw.Config.make(len(seq_lens), Hq, Hkv, S)
    segs = bmw.la_pbd_plan(cfg, W, seq_lens, num_ctas, unit, seg)
    B = len(seq_lens)
    valid = [0 <= P and P + W <= S for P in seq_lens]
    n_of = [P + W if ok else 0 for P, ok in zip(seq_lens, valid)]
    units = sum(Hkv * (-(-n // unit) + seg) for n in n_of if n > 0)
    C = max(1, -(-units // num_ctas))

    covered = {}
    per_cta_units = {}
    slots = set()
    last_cta = -1
    for cta, b, h, j0, j1, slot in segs:
        assert 0 <= cta < num_ctas
        assert cta >= last_cta, "segments must come in CTA order"
        last_cta = cta
        assert 0 <= b < B and 0 <= h < Hkv
        assert valid[b], "an invalid sequence received work"
        n = n_of[b]
        assert 0 <= j0 < j1 <= n
        assert j0 % unit == 0, "segments start on a tile boundary"
        assert j1 % unit == 0 or j1 == n, "segments end on a tile boundary or at the end"
        covered.setdefault((b, h), []).append((j0, j1, cta, slot))
        # a segment after the CTA's first starts its sequence inside the run: its fixed cost
        # units are in the run too
        fixed = seg if cta in per_cta_units else 0
        if fixed:
            assert j0 == 0, "only a CTA's first segment may continue a sequence"
        per_cta_units[cta] = per_cta_units.get(cta, 0) + fixed + -(-(j1 - j0) // unit)
        if slot != -1:
            assert slot not in slots, "partial slots must be distinct"
            assert 0 <= slot < num_ctas + B * Hkv
            slots.add(slot)

    for cta, u in per_cta_units.items():
        assert u <= C, f"CTA {cta} got {u} units, share is {C}"
    for b in range(B):
        for h in range(Hkv):
            parts = sorted(covered.get((b, h), []))
            if not valid[b]:
                assert not parts
                continue
            pos = 0
            for j0, j1, _, _ in parts:
                assert j0 == pos, f"gap or overlap in ({b}, {h}) at key {pos}"
                pos = j1
            assert pos == n_of[b], f"({b}, {h}) covered up to {pos} of {n_of[b]}"
            ctas = [c for _, _, c, _ in parts]
            assert ctas == list(range(ctas[0], ctas[0] + len(ctas))), "consecutive CTAs"
            whole = [s == -1 for _, _, _, s in parts]
            assert whole == ([True] if len(parts) == 1 else [False] * len(parts))
    return segs


@pytest.mark.parametrize("seg", [0, 2, 5])
@pytest.mark.parametrize("unit", [128, 32])
@pytest.mark.parametrize("num_ctas", [1, 7, 17, 148, 592])
def test_plan_single_image_and_long(unit, num_ctas, seg):
    check_plan([1024], 6, 1088, 2, num_ctas, unit, seg=seg)
    check_plan([32768] * 8, 6, 32832, 2, num_ctas, unit, seg=seg)


@pytest.mark.parametrize("seed", range(6))
def test_plan_ragged(seed):
    rng = random.Random(seed)
    B = rng.choice([1, 3, 64, 300])
    S = 4160
    W = rng.choice([1, 6, 16])
    lens = [rng.randint(0, S - W) for _ in range(B)]
    for num_ctas in (1, 13, 148, 592):
        for unit in (128, 32):
            for seg in (0, 1, 2, 3):
                check_plan(lens, W, S, 2, num_ctas, unit, seg=seg)


def test_plan_params():
    assert bmw.la_pbd_plan_params(bmw.LA_ALGO_TCGEN05) == (128, 3)
    assert bmw.la_pbd_plan_params(bmw.LA_ALGO_SIMT) == (32, 0)
    with pytest.raises(bmw.LaError):
        bmw.la_pbd_plan_params(bmw.LA_ALGO_AUTO)


def cta_costs(segs, seg):
    """Cost of each CTA in tile times: its tiles plus `seg` for each of its segments."""
    cost = {}
    for cta, b, h, j0, j1, slot in segs:
        cost[cta] = cost.get(cta, 0) + seg + -(-(j1 - j0) // 128)
    return cost


def test_plan_fixed_cost_balances_ragged_batch():
    """The 64-sequence ragged batch (prefixes U{512..4096} + U{1..5}, window 6): with the
    fixed segment cost in the plan, the costliest CTA (tiles + 2 per segment) is cheaper than
    with a plan of tiles only, where CTAs that cross several sequence starts finish last."""
    gen = torch.Generator().manual_seed(3)
    base = torch.randint(512, 4096 + 1, (64,), generator=gen, dtype=torch.int64)
    acc = torch.randint(1, 5 + 1, (64,), generator=gen, dtype=torch.int64)
    lens = (base + acc).tolist()
    unit, seg = bmw.la_pbd_plan_params(bmw.LA_ALGO_TCGEN05)
    flat = check_plan(lens, 6, 4160, 2, 148, unit, seg=0)
    fixed = check_plan(lens, 6, 4160, 2, 148, unit, seg=seg)
    worst_flat = max(cta_costs(flat, seg).values())
    worst_fixed = max(cta_costs(fixed, seg).values())
    assert worst_fixed < worst_flat, (worst_fixed, worst_flat)


def test_plan_edge_cases():
    # empty prefixes, exact tile multiples, invalid lengths, one head
    for seg in (0, 2):
        check_plan([0, 0, 0], 6, 64, 2, 5, 128, seg=seg)
        check_plan([122, 250, 506], 6, 512, 2, 3, 128, seg=seg)    # P + W = 128, 256, 512
        check_plan([-1, 100, 60, 59], 6, 66, 2, 4, 32, seg=seg)    # P = -1, 100 invalid
        check_plan([5, 7], 1, 8, 1, 2, 128, Hq=16, seg=seg)
    segs = check_plan([1024], 6, 1088, 2, 18, 128)
    # single-image decode at one tile per CTA: 9 tiles per KV head, every CTA one segment
    assert len(segs) == 18 and len({s[0] for s in segs}) == 18
    # with the fixed cost, 22 units at one per CTA: each KV head's two fixed-cost units
    # fall in CTAs of their own, which get no segment; the 18 tiles still go one per CTA
    segs = check_plan([1024], 6, 1088, 2, 22, 128, seg=2)
    assert sorted(s[0] for s in segs) == list(range(2, 11)) + list(range(13, 22))


def test_plan_rejects_bad_arguments():
    cfg = bmw.Config.make(2, 16, 2, 128)
    for num_ctas, unit, seg in ((0, 128, 0), (4, 0, 0), (4, 128, -1)):
        with pytest.raises(bmw.LaError):
            bmw.la_pbd_plan(cfg, 6, [1, 2], num_ctas, unit, seg)
    with pytest.raises(bmw.LaError):
        bmw.la_pbd_plan(bmw.Config.make(2, 16, 3, 128), 6, [1, 2], 4, 128)


def test_plan_spreads_units_over_every_cta():
    """With at least as many units as CTAs, every CTA gets floor(T/G) or ceil(T/G) of them, so
    on the ragged batch all 148 CTAs get work (a uniform chunk of ceil(T/G) left the last
    CTAs idle); with fewer units than CTAs the units go one per CTA from CTA 0, so the pieces
    of a sequence stay in consecutive CTAs."""
    gen = torch.Generator().manual_seed(3)
    base = torch.randint(512, 4096 + 1, (64,), generator=gen, dtype=torch.int64)
    acc = torch.randint(1, 5 + 1, (64,), generator=gen, dtype=torch.int64)
    lens = (base + acc).tolist()
    unit, seg = bmw.la_pbd_plan_params(bmw.LA_ALGO_TCGEN05)
    segs = check_plan(lens, 6, 4160, 2, 148, unit, seg=seg)
    assert {s[0] for s in segs} == set(range(148))
    T = sum(2 * (-(-(P + 6) // unit) + seg) for P in lens)
    units = {}
    for cta, b, h, j0, j1, slot in segs:
        units[cta] = units.get(cta, 0) + -(-(j1 - j0) // unit)
    # tiles alone never exceed the share; the fixed costs fill the rest of it
    assert max(units.values()) <= -(-T // 148)
    segs = check_plan([1024], 6, 1088, 2, 148, unit)     # 18 tiles on 148 CTAs
    assert sorted(s[0] for s in segs) == list(range(18))
