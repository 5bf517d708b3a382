"""A model of the wide-head forward kernel's synchronisation (D = 192, 256), run on the CPU.

`attn_fwd_wide_sm100` coordinates, in each CTA, a TMA producer warp, an MMA-issuing warp, the
tensor pipe (which runs MMAs and commits in issue order) and one softmax warpgroup over one
128-row query tile at a time, with two score buffers in tensor memory (P written over the
scores) and one O accumulator.  CTAs walk work items with a stride of the grid: an item is one
query tile or, causal, a head's heaviest and lightest remaining tiles.  Across the tiles of a
CTA the block counter g (which score buffer, which barrier phase) runs on, the producer loads
the next tile's Q once the current tile's last S has read the buffer (q_empty), the MMA warp
computes the next tile's first scores while the softmax finishes the current tile, the first
P V of a tile waits until the softmax has read the previous tile's O (o_free, a guard the
softmax's own order already implies, see below), and the lazy O
rescale at a block waits for the previous block's P V (pv_done, phases counted over all tiles).

Each agent's program is restated step for step as a Python generator, the mbarrier waits are
evaluated with the hardware's parity rule, and a scheduler runs all agents of all CTAs of a
small grid in many random interleavings (TMA loads land in any order).  Each run checks that
every agent finishes, that no wait is issued two phases behind its barrier, that every read
finds the data it expects (Q, K and V tiles, S and P of the right tile and block, O of the
right tile), that no buffer is reloaded or overwritten while a reader is pending, that a
rescale never races a P V, and that each (head, query tile) is written once from all of its KV
blocks.  Planted mistakes in the restated protocol fail it.
"""
import random

import pytest

BLOCK = 128


class Deadlock(Exception):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, f"{self.name}: too many arrivals"
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


def wide_tile(nb, causal, pair, k, which):
    """The kernel's item decoder: (head, query tile) of tile `which` of item k, or None."""
    if not pair:
        if which:
            return None
        head, kk = divmod(k, nb)
        return head, (nb - 1 - kk if causal else kk)
    sph = (nb + 1) // 2
    head, s = divmod(k, sph)
    heavy = nb - 1 - s
    if which == 0:
        return head, heavy
    return (head, s) if s < heavy else None


def schedule(BH, N, causal, sms, persistent=True):
    """Host plan (pairing, items, grid) and each CTA's list of (head, tile, KV blocks)."""
    nb = -(-N // BLOCK)
    pairs = BH * ((nb + 1) // 2)
    pair = causal and pairs >= sms
    items = pairs if pair else BH * nb
    grid = min(items, sms) if persistent else items
    ctas = []
    for c in range(grid):
        tiles = []
        for k in range(c, items, grid):
            for which in (0, 1):
                t = wide_tile(nb, causal, pair, k, which)
                if t is not None:
                    tiles.append((t[0], t[1], t[1] + 1 if causal else nb))
        ctas.append(tiles)
    return dict(nb=nb, causal=causal, pair=pair, items=items, grid=grid), ctas


def run_grid(ctas, stages, rng, mutation=None):
    outputs = {}
    agents, pending, done, sims = {}, {}, set(), []

    def make_cta(ci, tiles):
        bars = {name: Barrier(name, count) for name, count in (
            ("q_full", 1), ("q_empty", 1), ("pv_done", 1), ("o_full", 1), ("o_free", BLOCK), ("drain", 1))}
        for b in range(2):
            bars[f"s_full{b}"] = Barrier(f"s_full{b}", 1)
            bars[f"p_full{b}"] = Barrier(f"p_full{b}", BLOCK)
        for s in range(stages):
            bars[f"kv_full{s}"] = Barrier(f"kv_full{s}", 1)
            bars[f"kv_empty{s}"] = Barrier(f"kv_empty{s}", 1)
        st = {
            "stage": [None] * stages, "stage_busy": [0] * stages, "q": None, "q_busy": 0,
            "s": [None, None],       # ("S" | "P", tile index, block) in score buffer b
            "p_read": [True, True],  # the P in buffer b has been read by its P V
            "o": None,               # [tile index, blocks accumulated, epilogue read]
            "pv_last": -1,           # global block index of the last completed P V
        }
        tensor_q, tma_q = [], []

        def W(name, parity, k):
            assert (k >= 0 and parity == (k & 1)) or (k == -1 and parity == 1), (ci, name, parity, k)
            yield ("wait", ci, name, k)

        def producer():
            stage, phase, uses = 0, 0, [0] * stages
            for ti, (head, qt, n) in enumerate(tiles):
                if ti > 0 and mutation != "producer_ignores_q_empty":
                    yield from W("q_empty", (ti - 1) & 1, ti - 1)
                assert st["q_busy"] == 0, "Q reloaded while an S still reads it"
                tma_q.append(("q", ti))
                order = []
                for i in range(2 * n):
                    if i < 2:
                        order.append(("K", 0 if i == 0 else (1 if n > 1 else 0)) if (i == 0 or n > 1) else ("V", 0))
                    else:
                        q2, second = (i - 2) >> 1, (i - 2) & 1
                        if not second:
                            order.append(("V", q2))
                        else:
                            order.append(("K", q2 + 2) if q2 + 2 < n else ("V", q2 + 1))
                for kind, j in order:
                    yield from W(f"kv_empty{stage}", phase ^ 1, uses[stage] - 1)
                    assert st["stage_busy"][stage] == 0, "ring stage reloaded while an MMA still reads it"
                    uses[stage] += 1
                    tma_q.append(("kv", stage, (kind, ti, j)))
                    stage += 1
                    if stage == stages:
                        stage, phase = 0, phase ^ 1

        def mma():
            stage, phase, uses = 0, 0, [0] * stages
            g = 0

            def take():
                nonlocal stage, phase
                s = stage
                yield from W(f"kv_full{s}", phase, uses[s])
                uses[s] += 1
                stage += 1
                if stage == stages:
                    stage, phase = 0, phase ^ 1
                return s

            def issue_s(b, ti, j, s):
                assert st["stage"][s] == ("K", ti, j), f"S({ti},{j}) reads {st['stage'][s]}"
                assert st["q"] == ti, f"S({ti},{j}) reads Q of tile {st['q']}"
                st["stage_busy"][s] += 1
                st["q_busy"] += 1
                tensor_q.append(("S", b, ti, j, s))

            def commit(name):
                tensor_q.append(("commit", name))

            for ti, (head, qt, n) in enumerate(tiles):
                yield from W("q_full", ti & 1, ti)
                s = yield from take()
                issue_s(g & 1, ti, 0, s)
                commit(f"s_full{g & 1}")
                commit(f"kv_empty{s}")
                if n == 1 and mutation != "q_empty_dropped":
                    commit("q_empty")
                if n > 1:
                    s = yield from take()
                    issue_s((g + 1) & 1, ti, 1, s)
                    commit(f"s_full{(g + 1) & 1}")
                    commit(f"kv_empty{s}")
                    if n == 2 and mutation != "q_empty_dropped":
                        commit("q_empty")
                for j in range(n):
                    gj = g + j
                    b = gj & 1
                    yield from W(f"p_full{b}", (gj >> 1) & 1, gj >> 1)
                    if j == 0 and ti > 0 and mutation != "o_free_not_awaited":
                        yield from W("o_free", (ti - 1) & 1, ti - 1)
                    v = yield from take()
                    assert st["stage"][v] == ("V", ti, j), f"PV({ti},{j}) reads {st['stage'][v]}"
                    assert st["s"][b] == ("P", ti, j), f"PV({ti},{j}) reads {st['s'][b]}"
                    st["stage_busy"][v] += 1
                    tensor_q.append(("PV", b, ti, j, v, j > 0, gj))
                    if mutation != "pv_done_dropped":
                        commit("pv_done")
                    commit(f"kv_empty{v}")
                    if j + 2 < n:
                        s = yield from take()
                        issue_s(b, ti, j + 2, s)
                        commit(f"s_full{b}")
                        commit(f"kv_empty{s}")
                        if j + 3 == n and mutation != "q_empty_dropped":
                            commit("q_empty")
                commit("o_full")
                g += n if mutation != "block_counter_restarts" else 0
            commit("drain")
            yield from W("drain", 0, 0)

        def softmax():
            g = 0
            for ti, (head, qt, n) in enumerate(tiles):
                for j in range(n):
                    gj = g + j
                    b = gj & 1
                    yield from W(f"s_full{b}", (gj >> 1) & 1, gj >> 1)
                    assert st["s"][b] == ("S", ti, j), f"softmax reads {st['s'][b]} for {(ti, j)}"
                    if j > 0 and rng.random() < 0.5:
                        # the lazy rescale of O: wait for the previous block's P V
                        if mutation != "rescale_without_wait":
                            par = (gj - 1) & 1 if mutation != "pv_done_parity" else gj & 1
                            yield from W("pv_done", par, gj - 1 if mutation != "pv_done_parity" else gj)
                        assert st["pv_last"] == gj - 1, "O rescaled while a P V still runs"
                    st["s"][b] = ("P", ti, j)
                    st["p_read"][b] = False
                    bars[f"p_full{b}"].arrive(BLOCK)
                yield from W("o_full", ti & 1, ti)
                o = st["o"]
                assert o is not None and o[0] == ti and o[1] == set(range(n)) and not o[2], \
                    f"epilogue of tile {ti} reads O {o}"
                o[2] = True
                bars["o_free"].arrive(BLOCK)
                tile = (head, qt)
                assert tile not in outputs, f"output tile {tile} written twice"
                outputs[tile] = set(o[1])
                g += n

        def complete_tensor():
            op = tensor_q.pop(0)
            if op[0] == "S":
                _, b, ti, j, s = op
                assert st["p_read"][b], "S overwrote a P that its P V had not read"
                st["s"][b] = ("S", ti, j)
                st["stage_busy"][s] -= 1
                st["q_busy"] -= 1
            elif op[0] == "PV":
                _, b, ti, j, v, acc, gj = op
                assert st["s"][b] == ("P", ti, j)
                st["p_read"][b] = True
                if not acc:
                    prev = st["o"]
                    assert prev is None or prev[2], "O overwritten before the previous epilogue read it"
                    st["o"] = [ti, set(), False]
                assert st["o"][0] == ti
                st["o"][1].add(j)
                st["pv_last"] = gj
                st["stage_busy"][v] -= 1
            else:
                bars[op[1]].arrive()

        def land_tma():
            op = tma_q.pop(rng.randrange(len(tma_q)))
            if op[0] == "q":
                st["q"] = op[1]
                bars["q_full"].arrive()
            else:
                st["stage"][op[1]] = op[2]
                bars[f"kv_full{op[1]}"].arrive()

        return dict(bars=bars, tensor_q=tensor_q, tma_q=tma_q,
                    progs={"producer": producer(), "mma": mma(), "softmax": softmax()},
                    complete_tensor=complete_tensor, land_tma=land_tma)

    for ci, tiles in enumerate(ctas):
        sims.append(make_cta(ci, tiles))
        for name, gen in sims[-1]["progs"].items():
            agents[(ci, name)] = gen
            pending[(ci, name)] = None

    def ready(a):
        ev = pending[a]
        if ev is None:
            return True
        return sims[ev[1]]["bars"][ev[2]].phase > ev[3]

    for _ in range(10 ** 7):
        if len(done) == len(agents):
            break
        for a, ev in pending.items():
            if ev is not None:
                assert sims[ev[1]]["bars"][ev[2]].phase <= ev[3] + 1, f"{a} waits two phases behind on {ev[2]}"
        options = [a for a in agents if a not in done and ready(a)]
        options += [("tensor", ci) for ci, s in enumerate(sims) if s["tensor_q"]]
        options += [("tma", ci) for ci, s in enumerate(sims) if s["tma_q"]]
        if not options:
            raise Deadlock(f"all agents blocked: { {a: e for a, e in pending.items() if a not in done} }")
        a = rng.choice(options)
        if a[0] == "tensor":
            sims[a[1]]["complete_tensor"]()
            continue
        if a[0] == "tma":
            sims[a[1]]["land_tma"]()
            continue
        try:
            pending[a] = next(agents[a])
        except StopIteration:
            pending[a] = None
            done.add(a)
    else:
        raise AssertionError("runaway simulation")
    for s in sims:
        assert not s["tensor_q"] and not s["tma_q"]
    return outputs


def check_outputs(P, BH, outputs):
    nb = P["nb"]
    expected = {(h, t) for h in range(BH) for t in range(nb)}
    assert set(outputs) == expected
    for (h, t), blocks in outputs.items():
        assert blocks == (set(range(t + 1)) if P["causal"] else set(range(nb))), ((h, t), sorted(blocks))


CASES = [
    # (heads B*Hq, N, causal, SMs): causal tile pairs (odd and even tile counts), single causal
    # tiles (fewer pairs than SMs), non-causal persistent CTAs, and one tile per CTA
    (2, 1000, True, 2), (3, 640, True, 2), (4, 384, True, 3), (1, 1, True, 2), (2, 1, False, 3),
    (2, 700, False, 3), (5, 256, False, 2), (1, 600, True, 8), (2, 500, False, 100),
]


@pytest.mark.parametrize("stages", [2, 3, 4])
@pytest.mark.parametrize("case", CASES)
def test_wide_protocol_runs_without_deadlock_or_race(case, stages):
    BH, N, causal, sms = case
    P, ctas = schedule(BH, N, causal, sms)
    for seed in range(8):
        outputs = run_grid(ctas, stages, random.Random(6151 * seed + N + stages))
        check_outputs(P, BH, outputs)


def test_cases_cover_every_item_kind():
    kinds = set()
    for BH, N, causal, sms in CASES:
        P, ctas = schedule(BH, N, causal, sms)
        if P["pair"]:
            kinds.add("pair")
            nb = P["nb"]
            if nb % 2 == 1:
                kinds.add("lone_middle")
        elif causal:
            kinds.add("single_causal")
        if any(len(t) > 1 for t in ctas):
            kinds.add("many_tiles_per_cta")
        if all(len(t) == 1 for t in ctas):
            kinds.add("one_tile_per_cta")
    assert kinds == {"pair", "lone_middle", "single_causal", "many_tiles_per_cta", "one_tile_per_cta"}


def test_o_free_is_implied_by_the_softmax_order():
    """The MMA warp's wait for o_free before a tile's first P V is a guard that the protocol
    already implies: that P V needs P of the tile's first block, which the one softmax warpgroup
    writes only after it has read the previous tile's O.  Without the wait every run stays
    correct."""
    for BH, N, causal, sms in CASES:
        P, ctas = schedule(BH, N, causal, sms)
        for seed in range(4):
            check_outputs(P, BH, run_grid(ctas, 2, random.Random(seed), mutation="o_free_not_awaited"))


@pytest.mark.parametrize("mutation", [
    "producer_ignores_q_empty", "q_empty_dropped", "pv_done_dropped",
    "rescale_without_wait", "pv_done_parity", "block_counter_restarts"])
def test_planted_protocol_mistakes_are_caught(mutation):
    """Each planted mistake makes some interleaving deadlock or read the wrong data."""
    for BH, N, causal, sms in CASES:
        P, ctas = schedule(BH, N, causal, sms)
        for seed in range(10):
            try:
                outputs = run_grid(ctas, 2, random.Random(seed), mutation=mutation)
                check_outputs(P, BH, outputs)
            except (AssertionError, Deadlock):
                return
    raise AssertionError(f"mutation {mutation} went unnoticed")
