"""A model of the column-split forward kernel's schedule and synchronisation, run on the CPU.

The kernel (one 128-row Q tile per work unit, two score buffers, the score columns of each block
split between two softmax warpgroups) coordinates six agents through mbarriers: the TMA producer,
the MMA issuer, the tensor pipe (which runs MMAs and their commits in issue order), the two
softmax warpgroups, and the store warp (which writes each unit's O, staged in the unit's Q
buffer, with TMA stores and then gives the buffer back to the producer).  Here each agent's program is restated step for step as a Python generator,
the mbarrier waits are evaluated with the hardware's parity rule (a wait on parity P passes when
the barrier's current phase has the other parity), and a scheduler runs the agents in many
different interleavings.  Each run checks that

  * every agent finishes (no deadlock);
  * no wait is ever issued two phases behind its barrier (the parity rule would then stall);
  * every read finds the data it expects: the score buffer holds S of the right block, the P
    halves of the right block are present when P V is issued, a ring stage holds the K or V tile
    the MMA expects, the Q buffer holds the unit's Q, O is overwritten only after the previous
    unit's epilogue has read it, the O rescale waits for the last P V of the block before, O is
    staged in a Q buffer only after every S of that unit has read it, and the producer reloads a
    Q buffer only after the stores of the O staged in it have read it;
  * the units of all CTAs cover every (head, query tile) exactly once, each with its KV blocks.
"""
import random

import pytest

BLOCK = 128


def units_of_cta(P, cta):
    """The work items of one CTA, as the kernel's item decoder lists them (None: empty slot)."""
    T = P["T"]
    out = []
    it = 0
    while True:
        if P["causal"]:
            step = cta + (it >> 1) * P["grid"]
            if step >= P["steps"]:
                break
            sph = (T + 1) // 2
            head, s = divmod(step, sph)
            heavy = T - 1 - s
            if (it & 1) and s == heavy:
                out.append(None)
            else:
                tile = s if (it & 1) else heavy
                out.append((head, tile, tile + 1))
        else:
            u = cta + it * P["grid"]
            if u >= P["units"]:
                break
            head, tile = divmod(u, T)
            out.append((head, tile, T))
        it += 1
    return out


def blocks_of(units):
    """The CTA's sequence of (unit ordinal, unit, block j) in MMA order."""
    seq = []
    u = 0
    for w in units:
        if w is None:
            continue
        for j in range(w[2]):
            seq.append((u, w, j))
        u += 1
    return seq


class Deadlock(Exception):
    pass


class Barrier:
    """An mbarrier: `count` arrivals complete the current phase; `phase` counts completed phases."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, f"{self.name}: too many arrivals"
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


def run_cta(P, units, S_stages, rng, rescale_every_block=True):
    """Run one CTA's agents to completion in one random interleaving, checking as it goes."""
    seq = blocks_of(units)
    G = len(seq)
    bars = {}
    for i in range(2):
        for name in (f"q_full{i}", f"q_empty{i}", f"s_full{i}", f"p_full{i}0", f"p_full{i}1"):
            bars[name] = Barrier(name, 1)
        bars[f"o_staged{i}"] = Barrier(f"o_staged{i}", 2)
    for i in range(S_stages):
        bars[f"kv_full{i}"] = Barrier(f"kv_full{i}", 1)
        bars[f"kv_empty{i}"] = Barrier(f"kv_empty{i}", 1)
    for name, count in (("pv_done", 1), ("o_full", 1), ("o_free", 2), ("drain", 1)):
        bars[name] = Barrier(name, count)

    state = {
        "smem_stage": [None] * S_stages,     # tile held by each ring stage
        "stage_busy": [0] * S_stages,        # issued MMAs that read the stage and have not completed
        "q_buf": [None, None],
        "q_busy": [0, 0],
        "q_staged": [None, None],            # unit whose O is staged in each Q buffer (until stored)
        "q_store_reading": [False, False],
        "s_buf": [None, None],               # which block's S each score buffer holds
        "p_buf": [[None, None], [None, None]],
        "o_unit": None,                      # (unit, "acc" | "done") accumulated in O
        "o_read_by": set(),                  # warpgroups whose epilogue read O for that unit
        "pv_completed": -1,                  # last block whose P V (both halves) completed
    }
    tensor_q = []                            # issued, not yet completed tcgen05 operations (FIFO)
    tma_q = []                               # issued, not yet landed TMA loads (any order)

    def W(name, parity, k):
        """A bounded wait of the kernel: `parity` as the kernel computes it, `k` the phase the
        model expects it to wait for (-1: the completed phase before the first)."""
        assert (k >= 0 and parity == (k & 1)) or (k == -1 and parity == 1), (name, parity, k)
        yield ("wait", name, k)

    # ------------------------------------------------------------ producer
    def producer():
        ring = {"stage": 0, "phase": 0, "uses": [0] * S_stages}
        q_par = 3
        q_uses = [0, 0]

        def load_kv(kind, u, w, j):
            st = ring["stage"]
            yield from W(f"kv_empty{st}", ring["phase"] ^ 1, ring["uses"][st] - 1)
            assert state["stage_busy"][st] == 0, "ring stage reloaded while an MMA still reads it"
            ring["uses"][st] += 1
            tma_q.append(("kv", st, (kind, u, j, w)))
            ring["stage"] += 1
            if ring["stage"] == S_stages:
                ring["stage"], ring["phase"] = 0, ring["phase"] ^ 1

        def load_k(pos):
            nonlocal q_par
            u, w, j = seq[pos]
            if j == 0:
                qb = u & 1
                yield from W(f"q_empty{qb}", (q_par >> qb) & 1, q_uses[qb] - 1)
                q_par ^= 1 << qb
                q_uses[qb] += 1
                assert state["q_busy"][qb] == 0, "Q buffer reloaded while an S MMA still reads it"
                assert state["q_staged"][qb] is None and not state["q_store_reading"][qb], \
                    "Q buffer reloaded while its staged O is still being stored"
                tma_q.append(("q", qb, u))
            yield from load_kv("K", u, w, j)

        sc = 0
        for _ in range(2):
            if sc < G:
                yield from load_k(sc)
                sc += 1
        for pc in range(G):
            u, w, j = seq[pc]
            yield from load_kv("V", u, w, j)
            if sc < G:
                yield from load_k(sc)
                sc += 1

    # ------------------------------------------------------------ MMA issuer
    def mma():
        ring = {"stage": 0, "phase": 0, "uses": [0] * S_stages}
        q_par, of_par = 0, 1
        q_uses = [0, 0]

        def next_stage():
            st = ring["stage"]
            yield from W(f"kv_full{st}", ring["phase"], ring["uses"][st])
            ring["uses"][st] += 1
            ring["stage"] += 1
            if ring["stage"] == S_stages:
                ring["stage"], ring["phase"] = 0, ring["phase"] ^ 1
            return st

        def issue_s(gs):
            nonlocal q_par
            u, w, j = seq[gs]
            qb = u & 1
            if j == 0:
                yield from W(f"q_full{qb}", (q_par >> qb) & 1, q_uses[qb])
                q_par ^= 1 << qb
                q_uses[qb] += 1
            st = yield from next_stage()
            assert state["smem_stage"][st] == ("K", u, j, w), f"S({gs}) reads {state['smem_stage'][st]}"
            assert state["q_buf"][qb] == u, "S reads the wrong Q"
            state["stage_busy"][st] += 1
            state["q_busy"][qb] += 1
            tensor_q.append(("S", gs, gs & 1, st, qb))
            tensor_q.append(("commit", f"s_full{gs & 1}"))
            tensor_q.append(("commit", f"kv_empty{st}"))

        gs = 0
        for _ in range(2):
            if gs < G:
                yield from issue_s(gs)
                gs += 1
        for gp in range(G):
            u, w, j = seq[gp]
            b, ph = gp & 1, (gp >> 1) & 1
            yield from W(f"p_full{b}0", ph, gp >> 1)
            if j == 0:
                yield from W("o_free", of_par, u - 1)
                of_par ^= 1
            vst = yield from next_stage()
            assert state["smem_stage"][vst] == ("V", u, j, w), f"PV({gp}) reads {state['smem_stage'][vst]}"
            assert state["p_buf"][b][0] == gp, "P_0 missing"
            state["stage_busy"][vst] += 1
            tensor_q.append(("PV", gp, b, 0, vst, u, j))
            yield from W(f"p_full{b}1", ph, gp >> 1)
            assert state["p_buf"][b][1] == gp, "P_1 missing"
            tensor_q.append(("PV", gp, b, 1, vst, u, j))
            tensor_q.append(("commit", "pv_done"))
            tensor_q.append(("commit", f"kv_empty{vst}"))
            if j == w[2] - 1:
                tensor_q.append(("commit", "o_full"))
            if gs < G:
                yield from issue_s(gs)
                gs += 1
        tensor_q.append(("commit", "drain"))
        yield from W("drain", 0, 0)

    # ------------------------------------------------------------ softmax warpgroups
    def softmax(h):
        g, o_par, u = 0, 0, 0
        for w in units:
            if w is None:
                continue
            for j in range(w[2]):
                b = g & 1
                yield from W(f"s_full{b}", (g >> 1) & 1, g >> 1)
                assert state["s_buf"][b] == g, f"softmax {h} reads S of block {state['s_buf'][b]} for {g}"
                assert state["pv_completed"] >= g - 2   # S(g) complete implies P V of block g-2 complete
                if j > 0 and rescale_every_block:
                    yield from W("pv_done", (g - 1) & 1, g - 1)
                    assert state["pv_completed"] >= g - 1, "O rescaled while the last P V still runs"
                state["p_buf"][b][h] = g
                bars[f"p_full{b}{h}"].arrive()
                g += 1
            yield from W("o_full", o_par, u)
            o_par ^= 1
            yield ("agree", u)   # the end-of-unit barrier of both warpgroups
            assert state["o_unit"] == (u, "done"), "epilogue before the unit's last P V completed"
            state["o_read_by"].add(h)
            bars["o_free"].arrive()
            qb = u & 1
            assert state["q_busy"][qb] == 0 and state["q_buf"][qb] == u, "O staged over a Q still read by S"
            assert state["q_staged"][qb] in (None, u) and not state["q_store_reading"][qb]
            state["q_staged"][qb] = u
            bars[f"o_staged{qb}"].arrive()
            u += 1

    # ------------------------------------------------------------ store warp
    def store():
        st_par = 0
        u = 0
        for w in units:
            if w is None:
                continue
            qb = u & 1
            yield from W(f"o_staged{qb}", (st_par >> qb) & 1, u >> 1)
            st_par ^= 1 << qb
            assert state["q_staged"][qb] == u
            state["q_store_reading"][qb] = True
            yield ("store_read",)          # the TMA engine reads the staged rows (any time later)
            state["q_store_reading"][qb] = False
            state["q_staged"][qb] = None
            bars[f"q_empty{qb}"].arrive()
            u += 1

    # ------------------------------------------------------------ tensor pipe and TMA engine
    def complete_tensor_op():
        op = tensor_q.pop(0)
        if op[0] == "S":
            _, gs, buf, st, qb = op
            assert state["pv_completed"] >= gs - 2   # in-order pipe: the P V reading this buffer is done
            state["s_buf"][buf] = gs
            state["p_buf"][buf] = [None, None]
            state["stage_busy"][st] -= 1
            state["q_busy"][qb] -= 1
        elif op[0] == "PV":
            _, gp, buf, h, vst, u, j = op
            if j == 0 and h == 0:
                prev = state["o_unit"]
                assert prev is None or (prev[0] == u - 1 and state["o_read_by"] == {0, 1}), \
                    "O overwritten before the previous unit's epilogue read it"
                state["o_unit"] = (u, "acc")
                state["o_read_by"] = set()
            if h == 1:
                state["stage_busy"][vst] -= 1
                state["pv_completed"] = gp
                if j == seq[gp][1][2] - 1:
                    state["o_unit"] = (u, "done")
        else:
            bars[op[1]].arrive()

    def land_tma():
        op = tma_q.pop(rng.randrange(len(tma_q)))
        if op[0] == "q":
            state["q_buf"][op[1]] = op[2]
            bars[f"q_full{op[1]}"].arrive()
        else:
            state["smem_stage"][op[1]] = op[2]
            bars[f"kv_full{op[1]}"].arrive()

    agents = {"producer": producer(), "mma": mma(), "sm0": softmax(0), "sm1": softmax(1), "store": store()}
    pending = {a: None for a in agents}   # the event an agent is blocked on (None: runnable)
    done = set()
    for _ in range(10 ** 6):
        if len(done) == len(agents):
            break
        # a wait two phases behind its barrier would stall on the hardware
        for a, ev in pending.items():
            if ev is not None and ev[0] == "wait":
                assert bars[ev[1]].phase <= ev[2] + 1, f"{a} waits on {ev[1]} phase {ev[2]}: two phases behind"

        def ready(a):
            ev = pending[a]
            if ev is None:
                return True
            if ev[0] == "wait":
                return bars[ev[1]].phase > ev[2]
            if ev[0] == "store_read":
                return True
            other = "sm1" if a == "sm0" else "sm0"
            return pending[other] == ev

        options = [a for a in agents if a not in done and ready(a)]
        if tensor_q:
            options.append("tensor")
        if tma_q:
            options.append("tma")
        if not options:
            raise Deadlock(f"all agents blocked: {pending}")
        a = rng.choice(options)
        if a == "tensor":
            complete_tensor_op()
            continue
        if a == "tma":
            land_tma()
            continue
        if pending[a] is not None and pending[a][0] == "agree":
            pending["sm0"] = pending["sm1"] = None
        try:
            pending[a] = next(agents[a])
        except StopIteration:
            pending[a] = None
            done.add(a)
    else:
        raise AssertionError("runaway simulation")
    assert not tensor_q and not tma_q
    assert state["o_unit"] is None or state["o_read_by"] == {0, 1}
    return state


def schedule(B, Hq, N, causal, sms):
    T = -(-N // BLOCK)
    units = B * Hq * T
    steps = B * Hq * ((T + 1) // 2) if causal else units
    return dict(T=T, units=units, steps=steps, grid=min(steps, sms), causal=causal, B=B, Hq=Hq, N=N)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sms", [1, 3, 7, 148])
def test_units_cover_every_tile_once(causal, sms):
    for B, Hq, N in [(1, 1, 1), (1, 2, 127), (2, 3, 257), (1, 5, 1000), (3, 2, 2048), (1, 1, 4097)]:
        P = schedule(B, Hq, N, causal, sms)
        seen = {}
        for cta in range(P["grid"]):
            for w in units_of_cta(P, cta):
                if w is None:
                    continue
                head, tile, n = w
                assert 0 <= head < B * Hq and 0 <= tile < P["T"] and tile * BLOCK < N
                assert n == (tile + 1 if causal else P["T"]) and 1 <= n <= P["T"]
                seen[(head, tile)] = seen.get((head, tile), 0) + 1
        assert seen == {(h, t): 1 for h in range(B * Hq) for t in range(P["T"])}


@pytest.mark.parametrize("N", [1024, 1000, 8192])
def test_causal_steps_balance_work(N):
    P = schedule(2, 3, N, True, 148)
    T = P["T"]
    for cta in range(P["grid"]):
        us = units_of_cta(P, cta)
        for k in range(0, len(us), 2):
            pair = [w for w in us[k:k + 2] if w is not None]
            work = sum(w[2] for w in pair)
            assert work == T + 1 or (len(pair) == 1 and pair[0][2] == (T + 1) // 2)


@pytest.mark.parametrize("stages", [4, 8])
@pytest.mark.parametrize("case", [
    (1, 1, 128, False), (1, 1, 1, True), (1, 2, 300, True), (1, 3, 1000, False), (2, 2, 700, True),
    (1, 1, 2048, True), (1, 4, 513, False),
])
def test_protocol_runs_without_deadlock_or_race(case, stages):
    B, Hq, N, causal = case
    P = schedule(B, Hq, N, causal, 3)
    for cta in range(P["grid"]):
        units = units_of_cta(P, cta)
        for seed in range(6):
            run_cta(P, units, stages, random.Random(1000 * cta + seed))
