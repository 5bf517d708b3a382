"""A model of the backward kernels' synchronisation (`attn_bwd_sm100`, both passes), on the CPU.

Each CTA runs a TMA producer warp, an MMA-issuing warp, the tensor pipe (MMAs and commits in
issue order) and the softmax warps (two warpgroups, modelled as one agent that arrives with all
256 threads at once).  A unit keeps its row tiles R0, R1 in shared memory and streams column
tiles C0, C1 through rings of their own; per column tile the MMAs are S = R0 C0^T, dP = R1 C1^T
into one dP buffer (or, D <= 64, two alternating ones), then acc_ds += dS C0 and (dK/dV pass)
acc_p += P C1 with dS and P written over the dP columns they came from.  Persistent CTAs walk
the units (a causal item pairs a head's heaviest and lightest blocks): the row tiles are
reloaded once the unit's last S and dP have read them (r_empty), the next unit's first S and dP
run while the softmax stores the previous unit's gradients, and the first accumulating MMAs of
a unit wait until those are read (acc_free, a guard the softmax's own order already implies);
per-tile barrier phases count the tiles of all units.

The programs are restated step for step as Python generators, the mbarrier waits follow the
hardware's parity rule, and a scheduler runs all agents of a small grid in many random
interleavings (TMA loads land in any order).  Each run checks that every agent finishes, that no
wait is issued two phases behind its barrier, that every read finds the data it expects (row
and column tiles, S, dP, dS and P of the right unit and tile), that nothing is reloaded or
overwritten while a reader is pending, and that every unit's gradients are stored once, from
all of its column tiles.  Planted mistakes in the restated protocol fail it, among them the
earlier single dS-ready and P-ready barriers of the two-buffer form: there the softmax can
finish tile t+1 before the MMA warp waits for tile t, and the barrier completes twice.
"""
import random

import pytest

from test_wide_protocol_model import Barrier, Deadlock


def units_of(heads, nb, causal, kv, sms):
    """The kernel's item decoder over one pass: each CTA's list of units (head, block, tiles)."""
    pairs = heads * ((nb + 1) // 2)
    pair = causal and pairs >= sms
    items = pairs if pair else heads * nb
    grid = min(items, sms)

    def unit(item, which):
        if pair:
            sph = (nb + 1) // 2
            head, s = divmod(item, sph)
            if which == 1 and s >= nb - 1 - s:
                return None
            k = nb - 1 - s if which else s
        else:
            if which:
                return None
            head, k = divmod(item, nb)
        if kv:
            rb = k
            n = (nb - rb) if causal else nb     # column tiles (one query head per KV head here)
        else:
            rb = nb - 1 - k
            n = (rb + 1) if causal else nb
        return head, rb, n

    ctas = []
    for c in range(grid):
        us = []
        for item in range(c, items, grid):
            for which in (0, 1):
                u = unit(item, which)
                if u is not None:
                    us.append(u)
        ctas.append(us)
    return pair, ctas


def run_grid(ctas, kv, dual, S0, S1, rng, mutation=None):
    outputs = {}
    agents, pending, done, sims = {}, {}, set(), []
    ndp = 2 if dual else 1

    def dp_col(t):
        return t & 1 if dual else 0

    def dp_par(t):
        return (t >> 1) & 1 if dual else t & 1

    def ready_bar(name, t):
        # dS / P of tile t ready: one barrier per dP buffer (a single one in the planted mistake)
        return f"{name}{dp_col(t)}" if mutation != "shared_ready_barriers" else f"{name}0"

    def ready_wait(t):
        if mutation == "shared_ready_barriers":
            return t & 1, t
        return dp_par(t), t // ndp

    def make_cta(ci, units):
        bars = {name: Barrier(name, count) for name, count in (
            ("r_full", 1), ("r_empty", 1), ("s_full", 1), ("s_free", 256), ("p_ready0", 256),
            ("ds_ready0", 256), ("p_ready1", 256), ("ds_ready1", 256), ("acc_full", 1),
            ("acc_free", 256), ("drain", 1))}
        bars["dp_full0"] = Barrier("dp_full0", 1)
        bars["dp_full1"] = Barrier("dp_full1", 1)
        for s in range(S0):
            bars[f"c0_full{s}"] = Barrier(f"c0_full{s}", 1)
            bars[f"c0_empty{s}"] = Barrier(f"c0_empty{s}", 1)
        for s in range(S1):
            bars[f"c1_full{s}"] = Barrier(f"c1_full{s}", 1)
            bars[f"c1_empty{s}"] = Barrier(f"c1_empty{s}", 1)
        st = {
            "r": None, "r_busy": 0,
            "c0": [None] * S0, "c0_busy": [0] * S0, "vec_busy": [0] * S0,
            "c1": [None] * S1, "c1_busy": [0] * S1,
            "s": None, "s_read": True,
            "dp": [None] * ndp,          # [kind, unit, tile, ds_pending, p_pending]
            "acc": None,                 # [unit, tiles accumulated (acc_ds), tiles (acc_p), read]
        }
        tensor_q, tma_q = [], []

        def W(name, parity, k):
            assert (k >= 0 and parity == (k & 1)) or (k == -1 and parity == 1), (ci, name, parity, k)
            yield ("wait", ci, name, k)

        class Ring:
            def __init__(self, n):
                self.n, self.stage, self.phase = n, 0, 0

            def copy(self):
                r = Ring(self.n)
                r.stage, r.phase = self.stage, self.phase
                return r

            def advance(self):
                self.stage += 1
                if self.stage == self.n:
                    self.stage, self.phase = 0, self.phase ^ 1

        def producer():
            r0, r1 = Ring(S0), Ring(S1)
            u0 = [0] * S0
            u1 = [0] * S1
            for ui, (head, rb, n) in enumerate(units):
                if ui > 0 and mutation != "producer_ignores_r_empty":
                    yield from W("r_empty", (ui - 1) & 1, ui - 1)
                assert st["r_busy"] == 0, "row tiles reloaded while an MMA still reads them"
                tma_q.append(("r", ui))
                for it in range(n):
                    yield from W(f"c0_empty{r0.stage}", r0.phase ^ 1, u0[r0.stage] - 1)
                    assert st["c0_busy"][r0.stage] == 0 and st["vec_busy"][r0.stage] == 0, \
                        "C0 stage reloaded while it is still read"
                    u0[r0.stage] += 1
                    tma_q.append(("c0", r0.stage, (ui, it)))
                    r0.advance()
                    yield from W(f"c1_empty{r1.stage}", r1.phase ^ 1, u1[r1.stage] - 1)
                    assert st["c1_busy"][r1.stage] == 0, "C1 stage reloaded while an MMA still reads it"
                    u1[r1.stage] += 1
                    tma_q.append(("c1", r1.stage, (ui, it)))
                    r1.advance()

        def mma():
            r0, r1 = Ring(S0), Ring(S1)
            T = 0
            u0, u1 = [0] * S0, [0] * S1   # waits on each stage so far: the next wait's phase index

            def wait_c0(ring):
                k = u0[ring.stage]
                u0[ring.stage] += 1
                yield from W(f"c0_full{ring.stage}", ring.phase, k)

            def wait_c1(ring):
                k = u1[ring.stage]
                u1[ring.stage] += 1
                yield from W(f"c1_full{ring.stage}", ring.phase, k)

            def commit(name):
                tensor_q.append(("commit", name))

            def issue_s(ui, it, ring):
                assert st["c0"][ring.stage] == (ui, it), f"S({ui},{it}) reads C0 {st['c0'][ring.stage]}"
                assert st["r"] == ui, "S reads another unit's row tiles"
                st["c0_busy"][ring.stage] += 1
                st["r_busy"] += 1
                tensor_q.append(("S", ui, it, ring.stage))

            def issue_dp(ui, it, t, ring):
                assert st["c1"][ring.stage] == (ui, it), f"dP({ui},{it}) reads C1 {st['c1'][ring.stage]}"
                assert st["r"] == ui, "dP reads another unit's row tiles"
                st["c1_busy"][ring.stage] += 1
                st["r_busy"] += 1
                tensor_q.append(("dP", ui, it, t, ring.stage))

            for ui, (head, rb, n) in enumerate(units):
                yield from W("r_full", ui & 1, ui)
                # first tile's S and dP
                yield from wait_c0(r0)
                issue_s(ui, 0, r0)
                commit("s_full")
                yield from wait_c1(r1)
                issue_dp(ui, 0, T, r1)
                commit(f"dp_full{dp_col(T)}")
                if not kv:
                    commit(f"c1_empty{r1.stage}")
                if n == 1 and mutation != "r_empty_dropped":
                    commit("r_empty")
                for it in range(n):
                    t = T + it
                    par = t & 1
                    n0, n1 = r0.copy(), r1.copy()
                    n0.advance()
                    n1.advance()
                    has_next = it + 1 < n
                    yield from W("s_free", par, t)
                    if has_next:
                        yield from wait_c0(n0)
                        issue_s(ui, it + 1, n0)
                        commit("s_full")
                        if dual:
                            yield from wait_c1(n1)
                            issue_dp(ui, it + 1, t + 1, n1)
                            commit(f"dp_full{dp_col(t + 1)}")
                            if not kv:
                                commit(f"c1_empty{n1.stage}")
                            if it + 2 == n and mutation != "r_empty_dropped":
                                commit("r_empty")
                    if it == 0 and ui > 0 and mutation != "acc_free_not_awaited":
                        yield from W("acc_free", (ui - 1) & 1, ui - 1)
                    yield from W(ready_bar("ds_ready", t), *ready_wait(t))
                    assert st["c0"][r0.stage] == (ui, it)
                    st["c0_busy"][r0.stage] += 1
                    tensor_q.append(("acc_ds", ui, it, t, r0.stage))
                    commit(f"c0_empty{r0.stage}")
                    if kv:
                        yield from W(ready_bar("p_ready", t), *ready_wait(t))
                        assert st["c1"][r1.stage] == (ui, it)
                        st["c1_busy"][r1.stage] += 1
                        tensor_q.append(("acc_p", ui, it, t, r1.stage))
                        commit(f"c1_empty{r1.stage}")
                    if not dual and has_next:
                        yield from wait_c1(n1)
                        issue_dp(ui, it + 1, t + 1, n1)
                        commit("dp_full0")
                        if not kv:
                            commit(f"c1_empty{n1.stage}")
                        if it + 2 == n and mutation != "r_empty_dropped":
                            commit("r_empty")
                    r0, r1 = n0, n1
                commit("acc_full")
                T += n if mutation != "tile_counter_restarts" else 0
            commit("drain")
            yield from W("drain", 0, 0)

        def softmax():
            T = 0
            ring = Ring(S0)
            v_uses = [0] * S0
            for ui, (head, rb, n) in enumerate(units):
                for it0 in range(n):
                    t = T + it0
                    par = t & 1
                    yield from W("s_full", par, t)
                    if kv:
                        yield from W(f"c0_full{ring.stage}", ring.phase, v_uses[ring.stage])
                        assert st["c0"][ring.stage] == (ui, it0), "per-query vectors of another tile"
                        st["vec_busy"][ring.stage] += 1
                    v_uses[ring.stage] += 1
                    assert st["s"] == ("S", ui, it0), f"softmax reads S {st['s']} for {(ui, it0)}"
                    st["s_read"] = True
                    bars["s_free"].arrive(256)
                    yield from W(f"dp_full{dp_col(t)}", dp_par(t), t // ndp)
                    buf = st["dp"][dp_col(t)]
                    assert buf is not None and buf[:3] == ["dP", ui, it0], f"softmax reads dP {buf} for {(ui, it0)}"
                    buf[0], buf[3], buf[4] = "dSP", True, kv
                    if kv:
                        st["vec_busy"][ring.stage] -= 1
                    bars[ready_bar("ds_ready", t)].arrive(256)
                    if kv:
                        bars[ready_bar("p_ready", t)].arrive(256)
                    ring.advance()
                yield from W("acc_full", ui & 1, ui)
                acc = st["acc"]
                assert acc is not None and acc[0] == ui and acc[1] == set(range(n)) and not acc[3], \
                    f"epilogue of unit {ui} reads {acc}"
                if kv:
                    assert acc[2] == set(range(n))
                acc[3] = True
                bars["acc_free"].arrive(256)
                key = (head, rb)
                assert key not in outputs, f"unit {key} stored twice"
                outputs[key] = n
                T += n

        def complete_tensor():
            op = tensor_q.pop(0)
            kind = op[0]
            if kind == "S":
                _, ui, it, s = op
                assert st["s_read"], "S overwrote scores the softmax had not loaded"
                st["s"], st["s_read"] = ("S", ui, it), False
                st["c0_busy"][s] -= 1
                st["r_busy"] -= 1
            elif kind == "dP":
                _, ui, it, t, s = op
                prev = st["dp"][dp_col(t)]
                assert prev is None or (prev[0] == "dSP" and not prev[3] and not prev[4]), \
                    f"dP overwrote {prev} before its readers"
                st["dp"][dp_col(t)] = ["dP", ui, it, False, False]
                st["c1_busy"][s] -= 1
                st["r_busy"] -= 1
            elif kind == "acc_ds":
                _, ui, it, t, s = op
                buf = st["dp"][dp_col(t)]
                assert buf[:3] == ["dSP", ui, it] and buf[3], f"acc_ds reads {buf}"
                buf[3] = False
                if it == 0:
                    prev = st["acc"]
                    assert prev is None or prev[3], "accumulators overwritten before the epilogue read them"
                    st["acc"] = [ui, set(), set(), False]
                assert st["acc"][0] == ui
                st["acc"][1].add(it)
                st["c0_busy"][s] -= 1
            elif kind == "acc_p":
                _, ui, it, t, s = op
                buf = st["dp"][dp_col(t)]
                assert buf[:3] == ["dSP", ui, it] and buf[4], f"acc_p reads {buf}"
                buf[4] = False
                assert st["acc"][0] == ui
                st["acc"][2].add(it)
                st["c1_busy"][s] -= 1
            else:
                bars[op[1]].arrive()

        def land_tma():
            op = tma_q.pop(rng.randrange(len(tma_q)))
            if op[0] == "r":
                st["r"] = op[1]
                bars["r_full"].arrive()
            elif op[0] == "c0":
                st["c0"][op[1]] = op[2]
                bars[f"c0_full{op[1]}"].arrive()
            else:
                st["c1"][op[1]] = op[2]
                bars[f"c1_full{op[1]}"].arrive()

        return dict(bars=bars, tensor_q=tensor_q, tma_q=tma_q,
                    progs={"producer": producer(), "mma": mma(), "softmax": softmax()},
                    complete_tensor=complete_tensor, land_tma=land_tma)

    for ci, units in enumerate(ctas):
        sims.append(make_cta(ci, units))
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


def check_outputs(ctas, outputs):
    expected = {}
    for units in ctas:
        for head, rb, n in units:
            expected[(head, rb)] = n
    assert outputs == expected


CASES = [
    # (heads of the pass, tiles per head, causal, SMs): paired causal units (odd and even block
    # counts), unpaired causal units (fewer pairs than SMs), non-causal with many units per CTA
    (2, 5, True, 2), (3, 4, True, 3), (1, 3, True, 4), (2, 3, False, 2), (1, 1, True, 2), (3, 2, False, 5),
]


@pytest.mark.parametrize("kv", [True, False], ids=["dKdV", "dQ"])
@pytest.mark.parametrize("dual,S0,S1", [(False, 2, 2), (False, 3, 2), (True, 4, 4), (True, 2, 2)])
@pytest.mark.parametrize("case", CASES)
def test_bwd_protocol_runs_without_deadlock_or_race(case, kv, dual, S0, S1):
    heads, nb, causal, sms = case
    _, ctas = units_of(heads, nb, causal, kv, sms)
    for seed in range(6):
        outputs = run_grid(ctas, kv, dual, S0, S1, random.Random(7411 * seed + nb + S0))
        check_outputs(ctas, outputs)


def test_cases_cover_paired_unpaired_and_multi_unit_ctas():
    kinds = set()
    for heads, nb, causal, sms in CASES:
        pair, ctas = units_of(heads, nb, causal, True, sms)
        kinds.add("pair" if pair else ("single_causal" if causal else "noncausal"))
        if pair and nb % 2 == 1:
            kinds.add("lone_middle")
        if any(len(u) > 1 for u in ctas):
            kinds.add("many_units_per_cta")
    assert kinds >= {"pair", "lone_middle", "single_causal", "noncausal", "many_units_per_cta"}


def test_acc_free_is_implied_by_the_softmax_order():
    """The MMA warp's wait for acc_free before a unit's first accumulating MMAs is a guard the
    protocol already implies: those MMAs need the unit's first dS, which the softmax warps write
    only after they have read the previous unit's accumulators.  Without the wait every run stays
    correct."""
    for kv in (True, False):
        for dual, S0, S1 in ((False, 2, 2), (True, 2, 2)):
            for heads, nb, causal, sms in CASES:
                _, ctas = units_of(heads, nb, causal, kv, sms)
                for seed in range(3):
                    check_outputs(ctas, run_grid(ctas, kv, dual, S0, S1, random.Random(seed), "acc_free_not_awaited"))


@pytest.mark.parametrize("mutation", [
    "producer_ignores_r_empty", "r_empty_dropped", "tile_counter_restarts", "shared_ready_barriers"])
def test_planted_protocol_mistakes_are_caught(mutation):
    """Each planted mistake makes some interleaving deadlock or read the wrong data."""
    for kv in (True, False):
        for dual, S0, S1 in ((False, 2, 2), (True, 2, 2)):
            for heads, nb, causal, sms in CASES:
                _, ctas = units_of(heads, nb, causal, kv, sms)
                for seed in range(8):
                    try:
                        check_outputs(ctas, run_grid(ctas, kv, dual, S0, S1, random.Random(seed), mutation))
                    except (AssertionError, Deadlock):
                        return
    raise AssertionError(f"mutation {mutation} went unnoticed")
