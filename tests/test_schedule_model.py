"""A model of the forward kernel's persistent schedule, checked over many shapes and SM counts
(CPU).

The kernel's work-item decoding (each CTA walks items it = 0, 1, ... of a static schedule) and
the host's plan for a split last wave are restated here in Python, step for step.  The GPU parity
tests check the code itself, on the B200's 148 SMs; this model checks the schedule's design for
any SM count: every unit (256 query rows of one head) is computed exactly once; in a split last
wave the two KV ranges of a unit partition its KV blocks and own distinct workspace slots; a
causal step pairs a head's heaviest remaining pair with its lightest, so that steps cost the
same.
"""
import itertools

import pytest

BLOCK = 128


def plan(units, steps, num_blocks, sms, causal, allow_split=True):
    """The host's schedule: grid size, whole units per CTA, split tail units, parts."""
    grid = min(steps, sms)
    if causal or not allow_split or units <= 0:
        return dict(grid=grid, whole=0, tail=0, parts=1)
    tail, whole = units % sms, units // sms
    if tail == 0 or 2 * tail > sms or num_blocks < 4:
        return dict(grid=grid, whole=0, tail=0, parts=1)
    return dict(grid=sms if whole > 0 else tail * 2, whole=whole, tail=tail, parts=2)


def make_unit(N, num_blocks, causal, head, pair):
    q0 = pair * 2 * BLOCK
    if causal:
        n0, n1 = min(num_blocks, 2 * pair + 1), min(num_blocks, 2 * pair + 2)
    else:
        n0 = n1 = num_blocks
    valid1 = q0 + BLOCK < N
    return dict(head=head, pair=pair, jb=0, n0=n0, n1=n1, valid1=valid1, nmax=n1 if valid1 else n0,
                part=0, parts=1, tail=0)


def item_at(P, cta, it):
    """0: no more items; (1, unit): an item; (2, None): an empty slot."""
    pairs, nb, N = P["pairs"], P["num_blocks"], P["N"]
    if P["causal"]:
        step = cta + (it >> 1) * P["grid"]
        if step >= P["num_steps"]:
            return 0, None
        sph = (pairs + 1) // 2
        head, s = divmod(step, sph)
        part = it & 1
        pair = pairs - 1 - s if part == 0 else s
        if part == 1 and pair == pairs - 1 - s:
            return 2, None
        return 1, make_unit(N, nb, True, head, pair)
    if P["parts"] <= 1 or it < P["whole"]:
        u = cta + it * P["grid"]
        if u >= P["units"]:
            return 0, None
        return 1, make_unit(N, nb, False, u // pairs, u % pairs)
    if it > P["whole"]:
        return 0, None
    q = cta
    if q >= P["tail"] * P["parts"]:
        return 0, None
    u = P["whole"] * P["grid"] + q // P["parts"]
    w = make_unit(N, nb, False, u // pairs, u % pairs)
    w.update(parts=P["parts"], part=q % P["parts"], tail=q // P["parts"])
    w["jb"] = w["part"] * nb // P["parts"]
    w["n0"] = w["n1"] = w["nmax"] = (w["part"] + 1) * nb // P["parts"]
    return 1, w


def walk(B, Hq, N, causal, sms, allow_split=True):
    pairs = -(-N // (2 * BLOCK))
    nb = -(-N // BLOCK)
    units = B * Hq * pairs
    steps = B * Hq * ((pairs + 1) // 2) if causal else units
    P = dict(pairs=pairs, num_blocks=nb, N=N, causal=causal, units=units, num_steps=steps)
    P.update(plan(units, steps, nb, sms, causal, allow_split))
    items = []
    for cta in range(P["grid"]):
        it = 0
        while True:
            got, w = item_at(P, cta, it)
            if got == 0:
                break
            if got == 1:
                items.append((cta, w))
            it += 1
            assert it < 10 * (units + 2), "runaway item walk"
    return P, items


SMS = [1, 2, 3, 7, 16, 64, 132, 148, 160]
SHAPES = [(B, Hq, N) for B, Hq, N in itertools.product((1, 2, 3), (1, 2, 5, 16),
                                                        (1, 100, 256, 257, 511, 512, 1000, 2048, 4097))]


@pytest.mark.parametrize("sms", SMS)
@pytest.mark.parametrize("causal", [False, True])
def test_every_unit_computed_once(sms, causal):
    for B, Hq, N in SHAPES:
        P, items = walk(B, Hq, N, causal, sms)
        heads, pairs, nb = B * Hq, P["pairs"], P["num_blocks"]
        cover = {}
        for cta, w in items:
            assert 0 <= w["head"] < heads and 0 <= w["pair"] < pairs
            assert 0 <= w["jb"] < w["nmax"] <= nb
            if causal:  # tile t of pair j sees KV blocks up to and including its diagonal block
                assert w["n0"] == min(nb, 2 * w["pair"] + 1) and w["n1"] == min(nb, 2 * w["pair"] + 2)
            cover.setdefault((w["head"], w["pair"]), []).append((w["jb"], w["nmax"], w["part"], w["tail"]))
        assert sorted(cover) == [(h, p) for h in range(heads) for p in range(pairs)], (B, Hq, N, sms)
        tails = set()
        for key, ranges in cover.items():
            if len(ranges) == 1:
                jb, end, part, _ = ranges[0]
                assert (jb, part) == (0, 0) and end == (nb if not causal else end)
            else:
                # a split tail unit: two ranges that partition [0, num_blocks), two blocks or more each
                assert not causal and len(ranges) == 2
                (a0, a1, p0, t0), (b0, b1, p1, t1) = sorted(ranges, key=lambda r: r[2])
                assert (p0, p1) == (0, 1) and a0 == 0 and a1 == b0 and b1 == nb
                assert a1 - a0 >= 2 and b1 - b0 >= 2
                assert t0 == t1 and 0 <= t0 < P["tail"] and t0 not in tails
                tails.add(t0)
        assert len(tails) == P["tail"]


@pytest.mark.parametrize("sms", [7, 148])
def test_split_tail_only_when_the_last_wave_is_at_most_half_full(sms):
    for B, Hq, N in SHAPES:
        P, items = walk(B, Hq, N, False, sms)
        units = P["units"]
        if P["parts"] == 2:
            assert 0 < units % sms <= sms // 2 and P["num_blocks"] >= 4
            # each CTA runs at most one split range, after its whole units
            per_cta = {}
            for cta, w in items:
                per_cta.setdefault(cta, []).append(w["parts"])
            for seq in per_cta.values():
                assert seq.count(2) <= 1 and (2 not in seq or seq[-1] == 2)
        else:
            assert all(w["parts"] == 1 for _, w in items)


@pytest.mark.parametrize("N", [2048, 4096, 8192, 1000])
def test_causal_steps_pair_heavy_with_light(N):
    """Each causal step holds pair P-1-s and pair s of one head: their KV-block work sums to
    the same total for every full step (the middle step of an odd pair count holds one pair)."""
    B, Hq, sms = 2, 3, 148
    P, items = walk(B, Hq, N, True, sms)
    pairs = P["pairs"]
    work = {}
    for cta, w in items:
        s = min(w["pair"], pairs - 1 - w["pair"])
        work.setdefault((w["head"], s), []).append(w["n0"] + (w["n1"] if w["valid1"] else 0))
    totals = {k: sum(v) for k, v in work.items() if len(v) == 2}
    if N % 512 == 0:  # no ragged tail: every step is a full pair of pairs
        assert len(set(totals.values())) == 1
    assert all(len(v) in (1, 2) for v in work.values())


def walk_head_pairs(B, Hq, Hkv, N, sms):
    """Causal GQA with an even group: a unit is query tile `tile` of heads 2hp and 2hp + 1 (one KV
    head), both tiles seeing KV blocks 0..tile; steps pair a head pair's heaviest and lightest tiles."""
    assert (Hq // Hkv) % 2 == 0
    T = -(-N // BLOCK)
    steps = B * (Hq // 2) * ((T + 1) // 2)
    grid = min(steps, sms)
    sph = (T + 1) // 2
    g = Hq // Hkv
    items = []
    for cta in range(grid):
        it = 0
        while True:
            step = cta + (it >> 1) * grid
            if step >= steps:
                break
            slot, s = divmod(step, sph)
            part = it & 1
            tile = T - 1 - s if part == 0 else s
            if not (part == 1 and tile == T - 1 - s):
                b, hp = divmod(slot, Hq // 2)
                h0 = b * Hq + 2 * hp
                items.append(dict(cta=cta, step=step, heads=(h0, h0 + 1), kv=b * Hkv + (2 * hp) // g,
                                  rows=tile * BLOCK, n=min(T, tile + 1)))
            it += 1
    return T, items


@pytest.mark.parametrize("sms", [1, 7, 148])
@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 2, 1, 1), (1, 4, 2, 300), (2, 8, 2, 1000), (8, 32, 8, 8192),
                                        (1, 4, 1, 4097), (3, 6, 3, 256)])
def test_head_pair_units_cover_every_tile_once(B, Hq, Hkv, N, sms):
    T, items = walk_head_pairs(B, Hq, Hkv, N, sms)
    seen = {}
    for w in items:
        h0, h1 = w["heads"]
        assert h1 == h0 + 1 and h0 // Hq == h1 // Hq           # same batch row
        g = Hq // Hkv
        assert (h0 % Hq) // g == (h1 % Hq) // g                # same KV head
        assert w["kv"] == (h0 // Hq) * Hkv + (h0 % Hq) // g
        assert 0 <= w["rows"] < N and w["n"] == w["rows"] // BLOCK + 1
        for h in (h0, h1):
            seen[(h, w["rows"] // BLOCK)] = seen.get((h, w["rows"] // BLOCK), 0) + 1
    assert seen == {(h, t): 1 for h in range(B * Hq) for t in range(T)}


def test_head_pair_steps_balance_work():
    T, items = walk_head_pairs(2, 8, 2, 8192, 148)
    work = {}
    for w in items:
        work.setdefault(w["step"], []).append(w["n"])
    full = [sum(v) for v in work.values() if len(v) == 2]
    assert set(full) == {T + 1}
