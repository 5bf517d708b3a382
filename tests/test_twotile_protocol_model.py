"""A model of the two-tile forward kernel's synchronisation, run on the CPU.

`attn_fwd_sm100` (the kernel behind every bf16 and E4M3 forward at D <= 128 outside the
column-split case) coordinates, in each CTA, the TMA producer warp, the MMA-issuing warp, the
tensor pipe (which runs MMAs and commits in issue order), two softmax warpgroups (one per 128-row
query tile; P is written over the tile's scores in tensor memory) and, for bf16 D = 128, a store
warp that writes each tile's O from a shared-memory staging buffer with TMA stores.  For
non-causal bf16 D <= 64 the kernel takes a second form (`sep` below): P has tensor-memory columns
of its own beside O, and each tile has its own MMA warp, which issues the tile's next S once the
softmax has read the current one (S-free and P-free barriers; each K/V stage is released by both
MMA warps, used or not).  Split units
of a non-causal last wave add a protocol between two CTAs: the KV range that finishes first
publishes its unnormalised rows and (m, l) in the workspace and raises a ready flag; the other
waits for the flag and merges.

Each agent's program is restated here step for step as a Python generator over the work items the
kernel's item decoder lists (`test_schedule_model.item_at`, and its head-pair form), the mbarrier
waits are evaluated with the hardware's parity rule, and a scheduler runs all agents of all CTAs
of a small grid in many random interleavings (TMA loads land in any order).  Each run checks that

  * every agent finishes (no deadlock) and no wait is issued two phases behind its barrier;
  * every read finds the data it expects: S of the right (item, tile, block) when the softmax
    reads it and P of that block when P V reads it; the ring stage holds the K or V tile the MMA
    expects; the Q buffer holds the item's Q tile; a stage or Q buffer is reloaded only after the
    MMAs reading it completed; O accumulates from its first block only after the previous
    epilogue read it, and the epilogue reads it only after the tile's last P V; the O rescale
    never races a P V; the staging buffer is rewritten only after the stores read it;
  * each (head, query tile) output is written exactly once, from all of its KV blocks (a split
    unit's two ranges merged).
Planted mistakes in the restated protocol (a commit dropped or moved, a wrong parity) fail it.
"""
import random

import pytest

from test_schedule_model import item_at as decode_item
from test_schedule_model import plan

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


def schedule(B, Hq, Hkv, N, causal, sms, allow_split=True):
    """Host plan and per-CTA item lists: each item is None (empty slot) or a dict with jb, n0, n1
    (0 when tile 1 has no rows), nmax, parts, part, tail and the output tiles it owns."""
    T = -(-N // BLOCK)
    pairs = -(-N // (2 * BLOCK))
    head_pairs = causal and (Hq // Hkv) % 2 == 0
    if head_pairs:
        units = B * (Hq // 2) * T
        steps = B * (Hq // 2) * ((T + 1) // 2)
    else:
        units = B * Hq * pairs
        steps = B * Hq * ((pairs + 1) // 2) if causal else units
    P = dict(pairs=T if head_pairs else pairs, num_blocks=T, N=N, causal=causal, units=units,
             num_steps=steps)
    P.update(plan(units, steps, T, sms, causal, allow_split))
    ctas = []
    for cta in range(P["grid"]):
        items, it = [], 0
        while True:
            got, w = decode_item(P, cta, it)
            if got == 0:
                break
            it += 1
            if got == 2:
                items.append(None)
                continue
            if head_pairs:
                # the decoder's "head" is the head pair's slot and its "pair" the query tile
                slot, tile = w["head"], w["pair"]
                b, hp = divmod(slot, Hq // 2)
                h0 = b * Hq + 2 * hp
                n = min(T, tile + 1)
                item = dict(jb=0, n0=n, n1=n, nmax=n, parts=1, part=0, tail=0,
                            tiles=[(h0, tile), (h0 + 1, tile)])
            else:
                rows1 = w["pair"] * 2 * BLOCK + BLOCK
                item = dict(jb=w["jb"], n0=w["n0"], n1=w["n1"] if w["valid1"] else 0, nmax=w["nmax"],
                            parts=w["parts"], part=w["part"], tail=w["tail"],
                            tiles=[(w["head"], 2 * w["pair"]), (w["head"], 2 * w["pair"] + 1) if rows1 < N else None])
            items.append(item)
        ctas.append(items)
    return P, ctas


def blocks_needed(P, tile):
    """KV blocks a query tile's output depends on."""
    return set(range(min(P["num_blocks"], tile[1] + 1))) if P["causal"] else set(range(P["num_blocks"]))


def run_grid(P, ctas, S_stages, staged, rng, mutation=None, sep=False):
    """All agents of all CTAs in one random interleaving; returns the outputs written.  sep: the
    D <= 64 form (P in columns of its own, one MMA warp per tile)."""
    outputs = {}                     # (head, tile) -> set of KV blocks folded into the written rows
    ws = {}                          # (tail, t) -> {"count", "ready", "rows"}
    agents, pending, done = {}, {}, set()
    sims = []

    def make_cta(ci, items):
        bars = {}
        for t in range(2):
            for name, count in (("q_full", 1), ("q_empty", 1), ("s_full", 1), ("p_full", BLOCK),
                                ("o_full", 1), ("o_free", BLOCK)):
                bars[f"{name}{t}"] = Barrier(f"{name}{t}", count)
        for s in range(S_stages):
            bars[f"kv_full{s}"] = Barrier(f"kv_full{s}", 1)
            bars[f"kv_empty{s}"] = Barrier(f"kv_empty{s}", 2 if sep else 1)
        for name, count in (("drain", 2 if sep else 1), ("o_staged", BLOCK), ("stage_free", 1)):
            bars[name] = Barrier(name, count)
        for t in range(2):
            bars[f"s_free{t}"] = Barrier(f"s_free{t}", BLOCK)
            bars[f"p_free{t}"] = Barrier(f"p_free{t}", 1)
        st = {
            "stage": [None] * S_stages, "stage_busy": [0] * S_stages,
            "q": [None, None], "q_busy": [0, 0],
            "s": [None, None],       # ("S" | "P", item index, block) held in tile t's score columns
            "p_read": [True, True],  # the P in the score columns has been read by its P V
            "p": [None, None],       # sep: ("P", item index, block) in tile t's own P columns
            "s_read": [True, True],  # sep: the softmax has read the S in tile t's score columns
            "o": [None, None],       # [item index, blocks accumulated, epilogue read]
            "pv_last": [(-1, -1), (-1, -1)],   # (item, block) of tile t's last completed P V
            "staging": None, "store_reading": False,
        }
        tensor_q, tma_q = [], []
        seq = [(i, w) for i, w in enumerate(items) if w is not None]

        def W(name, parity, k):
            assert (k >= 0 and parity == (k & 1)) or (k == -1 and parity == 1), (ci, name, parity, k)
            yield ("wait", ci, name, k)

        def producer():
            stage, phase, uses = 0, 0, [0] * S_stages
            q_uses = [0, 0]

            def load_kv(kind, i, j):
                nonlocal stage, phase
                yield from W(f"kv_empty{stage}", phase ^ 1, uses[stage] - 1)
                assert st["stage_busy"][stage] == 0, "ring stage reloaded while an MMA still reads it"
                uses[stage] += 1
                tma_q.append(("kv", stage, (kind, i, j)))
                stage += 1
                if stage == S_stages:
                    stage, phase = 0, phase ^ 1

            def load_q(t, i):
                yield from W(f"q_empty{t}", (q_uses[t] - 1) & 1 if q_uses[t] else 1, q_uses[t] - 1)
                assert st["q_busy"][t] == 0, "Q buffer reloaded while an S MMA still reads it"
                q_uses[t] += 1
                tma_q.append(("q", t, i))

            for i, w in seq:
                yield from load_q(0, i)
                yield from load_kv("K", i, w["jb"])
                if w["n1"] > 0:
                    yield from load_q(1, i)
                yield from load_kv("V", i, w["jb"])
                for j in range(w["jb"] + 1, w["nmax"]):
                    yield from load_kv("K", i, j)
                    yield from load_kv("V", i, j)

        def mma():
            stage, phase, uses = 0, 0, [0] * S_stages
            q_par, pf_par, of_par = [0, 0], [0, 0], [1, 1]
            q_uses, pf_uses, of_uses = [0, 0], [0, 0], [0, 0]

            def take_stage():
                nonlocal stage, phase
                s = stage
                yield from W(f"kv_full{s}", phase, uses[s])
                uses[s] += 1
                stage += 1
                if stage == S_stages:
                    stage, phase = 0, phase ^ 1
                return s

            def issue_s(t, i, j, s):
                assert st["stage"][s] == ("K", i, j), f"S({t},{i},{j}) reads {st['stage'][s]}"
                assert st["q"][t] == i, "S reads the wrong Q tile"
                st["stage_busy"][s] += 1
                st["q_busy"][t] += 1
                tensor_q.append(("S", t, i, j, s))

            def commit(name):
                tensor_q.append(("commit", name))

            for i, w in seq:
                jb, n = w["jb"], (w["n0"], w["n1"])
                yield from W("q_full0", q_par[0], q_uses[0])
                q_par[0] ^= 1
                q_uses[0] += 1
                k0 = yield from take_stage()
                issue_s(0, i, jb, k0)
                commit("s_full0")
                if n[0] == jb + 1:
                    commit("q_empty0")
                if n[1] > 0:
                    yield from W("q_full1", q_par[1], q_uses[1])
                    q_par[1] ^= 1
                    q_uses[1] += 1
                    issue_s(1, i, jb, k0)
                    commit("s_full1")
                    if n[1] == jb + 1:
                        commit("q_empty1")
                if mutation != "kv_empty_before_s1":
                    commit(f"kv_empty{k0}")
                for j in range(jb, w["nmax"]):
                    v = yield from take_stage()
                    has_next = j + 1 < w["nmax"]
                    kn = stage
                    if has_next:
                        yield from W(f"kv_full{kn}", phase, uses[kn])
                    for t in range(2):
                        if j >= n[t]:
                            continue
                        yield from W(f"p_full{t}", pf_par[t], pf_uses[t])
                        pf_par[t] ^= 1
                        pf_uses[t] += 1
                        if j == jb:
                            of = of_par[t] if mutation != "o_free_parity" else of_par[t] ^ 1
                            yield from W(f"o_free{t}", of, of_uses[t] - 1)
                            of_par[t] ^= 1
                            of_uses[t] += 1
                        assert st["stage"][v] == ("V", i, j), f"PV({t},{i},{j}) reads {st['stage'][v]}"
                        assert st["s"][t] == ("P", i, j), f"PV({t},{i},{j}) reads {st['s'][t]}"
                        st["stage_busy"][v] += 1
                        tensor_q.append(("PV", t, i, j, v, j > jb))
                        if j == n[t] - 1:
                            commit(f"o_full{t}")
                        if j + 1 < n[t]:
                            issue_s(t, i, j + 1, kn)
                            commit(f"s_full{t}")
                            if j + 2 == n[t] and mutation != "q_empty_dropped":
                                commit(f"q_empty{t}")
                    commit(f"kv_empty{v}")
                    if has_next:
                        if mutation != "kv_empty_next_dropped":
                            commit(f"kv_empty{kn}")
                        uses[kn] += 1
                        stage += 1
                        if stage == S_stages:
                            stage, phase = 0, phase ^ 1
                if mutation == "kv_empty_before_s1":
                    commit(f"kv_empty{k0}")
            commit("drain")
            yield from W("drain", 0, 0)

        def mma_sep(t):
            """The D <= 64 form: one MMA warp per tile; a tile's next S follows the softmax's read of
            the current one; every ring stage is released by both warps (used or not)."""
            stage, phase, uses = 0, 0, [0] * S_stages
            cnt = {"q": 0, "p": 0, "s": 0, "o": 0}
            issued = False

            def take():
                nonlocal stage, phase
                s_ = stage
                yield from W(f"kv_full{s_}", phase, uses[s_])
                uses[s_] += 1
                stage += 1
                if stage == S_stages:
                    stage, phase = 0, phase ^ 1
                return s_

            def issue_s(i, j, s_):
                nonlocal issued
                if issued and mutation != "sep_s_without_free":
                    yield from W(f"s_free{t}", cnt["s"] & 1, cnt["s"])
                    cnt["s"] += 1
                issued = True
                assert st["stage"][s_] == ("K", i, j), f"S({t},{i},{j}) reads {st['stage'][s_]}"
                assert st["q"][t] == i, "S reads the wrong Q tile"
                st["stage_busy"][s_] += 1
                st["q_busy"][t] += 1
                tensor_q.append(("S", t, i, j, s_))
                tensor_q.append(("commit", f"s_full{t}"))

            for i, w in seq:
                jb = w["jb"]
                n = w["n0"] if t == 0 else w["n1"]
                j_end = jb
                if n > jb:
                    yield from W(f"q_full{t}", cnt["q"] & 1, cnt["q"])
                    cnt["q"] += 1
                    ks = yield from take()
                    yield from issue_s(i, jb, ks)
                    if n == jb + 1:
                        tensor_q.append(("commit", f"q_empty{t}"))
                    tensor_q.append(("commit", f"kv_empty{ks}"))
                    for j in range(jb, n):
                        vs, vuse = stage, uses[stage]
                        stage += 1
                        if stage == S_stages:
                            stage, phase = 0, phase ^ 1
                        if j + 1 < n:
                            ks = yield from take()
                            yield from issue_s(i, j + 1, ks)
                            if j + 2 == n:
                                tensor_q.append(("commit", f"q_empty{t}"))
                            tensor_q.append(("commit", f"kv_empty{ks}"))
                        yield from W(f"p_full{t}", cnt["p"] & 1, cnt["p"])
                        cnt["p"] += 1
                        if j == jb:
                            yield from W(f"o_free{t}", (cnt["o"] - 1) & 1 if cnt["o"] else 1, cnt["o"] - 1)
                            cnt["o"] += 1
                        yield from W(f"kv_full{vs}", vuse & 1, vuse)
                        uses[vs] = vuse + 1
                        assert st["stage"][vs] == ("V", i, j), f"PV({t},{i},{j}) reads {st['stage'][vs]}"
                        assert st["p"][t] == ("P", i, j), f"PV({t},{i},{j}) reads P {st['p'][t]}"
                        st["stage_busy"][vs] += 1
                        tensor_q.append(("PV", t, i, j, vs, j > jb))
                        if mutation != "sep_p_free_dropped":
                            tensor_q.append(("commit", f"p_free{t}"))
                        if j == n - 1:
                            tensor_q.append(("commit", f"o_full{t}"))
                        tensor_q.append(("commit", f"kv_empty{vs}"))
                    j_end = n
                for j in range(j_end, w["nmax"]):
                    for _ in range(2):
                        if mutation == "sep_skip_without_wait":
                            s_ = stage
                            uses[s_] += 1
                            stage += 1
                            if stage == S_stages:
                                stage, phase = 0, phase ^ 1
                        else:
                            s_ = yield from take()
                        bars[f"kv_empty{s_}"].arrive()
            tensor_q.append(("commit", "drain"))
            yield from W("drain", 0, 0)

        def softmax(t):
            s_uses, o_uses, stage_uses, p_uses = 0, 0, 0, 0
            for i, w in seq:
                my_use = stage_uses + t
                if w["parts"] == 1:
                    stage_uses += 2 if w["n1"] > 0 else 1
                n = w["n0"] if t == 0 else w["n1"]
                if n == 0:
                    continue
                for j in range(w["jb"], n):
                    yield from W(f"s_full{t}", s_uses & 1, s_uses)
                    s_uses += 1
                    assert st["s"][t] == ("S", i, j), f"softmax {t} reads {st['s'][t]} for {(i, j)}"
                    if sep:
                        st["s_read"][t] = True
                        bars[f"s_free{t}"].arrive(BLOCK)
                        if p_uses > 0:
                            yield from W(f"p_free{t}", (p_uses - 1) & 1, p_uses - 1)
                        assert st["p_read"][t], "P rewritten before its P V read it"
                        p_uses += 1
                    if j > w["jb"]:
                        # the lazy O rescale: the P V of every earlier block has completed
                        assert st["pv_last"][t] == (i, j - 1), "O rescaled while a P V still runs"
                    if sep:
                        st["p"][t] = ("P", i, j)
                    else:
                        st["s"][t] = ("P", i, j)
                    st["p_read"][t] = False
                    bars[f"p_full{t}"].arrive(BLOCK)
                yield from W(f"o_full{t}", o_uses & 1, o_uses)
                o_uses += 1
                o = st["o"][t]
                assert o is not None and o[0] == i and o[1] == set(range(w["jb"], n)) and not o[2], \
                    f"epilogue of tile {t} item {i} reads O {o}"
                o[2] = True
                tile = w["tiles"][t]
                if w["parts"] == 1 and staged:
                    bars[f"o_free{t}"].arrive(BLOCK)
                    if my_use > 0 and mutation != "stage_without_free":
                        yield from W("stage_free", (my_use - 1) & 1, my_use - 1)
                    assert not st["store_reading"] and st["staging"] is None, "staging rewritten under a store"
                    st["staging"] = (i, t, tile, frozenset(o[1]))
                    bars["o_staged"].arrive(BLOCK)
                elif w["parts"] == 1:
                    write_output(tile, o[1])
                    bars[f"o_free{t}"].arrive(BLOCK)
                else:
                    slot = ws.setdefault((w["tail"], t), {"count": 0, "ready": False, "rows": None})
                    order = slot["count"]
                    slot["count"] += 1
                    if order == 0:
                        if mutation == "flag_before_rows":
                            slot["ready"] = True
                            yield ("step",)
                        slot["rows"] = (tile, frozenset(o[1]))
                        bars[f"o_free{t}"].arrive(BLOCK)
                        slot["ready"] = True
                    else:
                        yield ("flag", (w["tail"], t))
                        assert slot["rows"] is not None, "merged before the other range published"
                        other_tile, other_blocks = slot["rows"]
                        assert other_tile == tile, "merged with another tile's rows"
                        write_output(tile, set(o[1]) | set(other_blocks))
                        bars[f"o_free{t}"].arrive(BLOCK)

        def store():
            uses = 0
            for i, w in seq:
                if w["parts"] > 1:
                    continue
                for t in range(2):
                    if t == 1 and w["n1"] == 0:
                        continue
                    yield from W("o_staged", uses & 1, uses)
                    assert st["staging"] is not None and st["staging"][:2] == (i, t), \
                        f"store of ({i},{t}) finds {st['staging']}"
                    _, _, tile, blocks = st["staging"]
                    st["store_reading"] = True
                    yield ("store_read",)
                    write_output(tile, set(blocks))
                    st["store_reading"] = False
                    st["staging"] = None
                    if mutation != "stage_free_dropped" or uses != 0:
                        bars["stage_free"].arrive()
                    uses += 1

        def complete_tensor():
            op = tensor_q.pop(0)
            if op[0] == "S":
                _, t, i, j, s = op
                if sep:
                    assert st["s_read"][t], "S overwrote scores the softmax had not read"
                    st["s_read"][t] = False
                else:
                    assert st["p_read"][t], "S overwrote a P that its P V had not read"
                st["s"][t] = ("S", i, j)
                st["stage_busy"][s] -= 1
                st["q_busy"][t] -= 1
            elif op[0] == "PV":
                _, t, i, j, v, acc = op
                assert (st["p"] if sep else st["s"])[t] == ("P", i, j)
                st["p_read"][t] = True
                if not acc:
                    prev = st["o"][t]
                    assert prev is None or prev[2], "O overwritten before the previous epilogue read it"
                    st["o"][t] = [i, set(), False]
                assert st["o"][t][0] == i
                st["o"][t][1].add(j)
                st["pv_last"][t] = (i, j)
                st["stage_busy"][v] -= 1
            else:
                bars[op[1]].arrive()

        def land_tma():
            op = tma_q.pop(rng.randrange(len(tma_q)))
            if op[0] == "q":
                st["q"][op[1]] = op[2]
                bars[f"q_full{op[1]}"].arrive()
            else:
                st["stage"][op[1]] = op[2]
                bars[f"kv_full{op[1]}"].arrive()

        progs = {"producer": producer(), "sm0": softmax(0), "sm1": softmax(1)}
        if sep:
            progs["mma0"], progs["mma1"] = mma_sep(0), mma_sep(1)
        else:
            progs["mma"] = mma()
        if staged:
            progs["store"] = store()
        return dict(bars=bars, state=st, tensor_q=tensor_q, tma_q=tma_q, progs=progs,
                    complete_tensor=complete_tensor, land_tma=land_tma)

    def write_output(tile, blocks):
        assert tile is not None
        assert tile not in outputs, f"output tile {tile} written twice"
        outputs[tile] = set(blocks)

    for ci, items in enumerate(ctas):
        sims.append(make_cta(ci, items))
        for name, g in sims[-1]["progs"].items():
            agents[(ci, name)] = g
            pending[(ci, name)] = None

    def ready(a):
        ev = pending[a]
        if ev is None or ev[0] in ("store_read", "step"):
            return True
        if ev[0] == "wait":
            return sims[ev[1]]["bars"][ev[2]].phase > ev[3]
        if ev[0] == "flag":
            return ws[ev[1]]["ready"]
        raise AssertionError(ev)

    for _ in range(10 ** 7):
        if len(done) == len(agents):
            break
        for a, ev in pending.items():
            if ev is not None and ev[0] == "wait":
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


def check_outputs(P, ctas, outputs):
    expected = set()
    for items in ctas:
        for w in items:
            if w is not None:
                expected.update(t for t in w["tiles"] if t is not None)
    assert set(outputs) == expected
    for tile, blocks in outputs.items():
        assert blocks == blocks_needed(P, tile), (tile, sorted(blocks))


CASES = [
    # (B, Hq, Hkv, N, causal, SMs)
    (1, 1, 1, 128, False, 2), (1, 1, 1, 1, True, 2), (1, 2, 2, 300, True, 3), (1, 3, 3, 1000, False, 3),
    (2, 2, 1, 700, True, 3), (1, 4, 2, 513, True, 3),          # head pairs (even group)
    (1, 4, 4, 1024, True, 4), (1, 2, 1, 1000, True, 2),         # head pairs, odd tile count
    (1, 3, 3, 1024, False, 5),                                  # 12 units on 5 SMs: two split units
    (1, 1, 1, 768, False, 7),                                   # 3 units on 7 SMs: every unit split
    (2, 1, 1, 1100, False, 3), (1, 2, 2, 1100, False, 4),       # split tails, one with a lone tile
]


@pytest.mark.parametrize("staged", [True, False])
@pytest.mark.parametrize("stages", [4, 8])
@pytest.mark.parametrize("case", CASES)
def test_protocol_runs_without_deadlock_or_race(case, stages, staged):
    B, Hq, Hkv, N, causal, sms = case
    P, ctas = schedule(B, Hq, Hkv, N, causal, sms)
    for seed in range(8):
        outputs = run_grid(P, ctas, stages, staged, random.Random(7919 * seed + N))
        check_outputs(P, ctas, outputs)


@pytest.mark.parametrize("stages", [4, 8])
@pytest.mark.parametrize("case", CASES)
def test_separate_p_protocol_runs_without_deadlock_or_race(case, stages):
    """The separate-P form (non-causal D <= 64 runs it with an 8-stage ring; 4 stages as a
    harder case, and the causal and head-pair items as well)."""
    B, Hq, Hkv, N, causal, sms = case
    P, ctas = schedule(B, Hq, Hkv, N, causal, sms)
    for seed in range(8):
        outputs = run_grid(P, ctas, stages, False, random.Random(104729 * seed + N), sep=True)
        check_outputs(P, ctas, outputs)


def test_cases_cover_split_tails_head_pairs_and_empty_slots():
    kinds = set()
    for B, Hq, Hkv, N, causal, sms in CASES:
        P, ctas = schedule(B, Hq, Hkv, N, causal, sms)
        for items in ctas:
            for w in items:
                if w is None:
                    kinds.add("empty")
                elif w["parts"] > 1:
                    kinds.add("split")
                elif causal and (Hq // Hkv) % 2 == 0:
                    kinds.add("head_pair")
                elif w["n1"] == 0:
                    kinds.add("lone_tile")
    assert kinds == {"empty", "split", "head_pair", "lone_tile"}


@pytest.mark.parametrize("mutation,sep", [
    ("kv_empty_before_s1", False), ("o_free_parity", False), ("q_empty_dropped", False),
    ("kv_empty_next_dropped", False), ("stage_free_dropped", False), ("stage_without_free", False),
    ("flag_before_rows", False), ("sep_s_without_free", True), ("sep_p_free_dropped", True),
    ("sep_skip_without_wait", True)])
def test_planted_protocol_mistakes_are_caught(mutation, sep):
    """Each planted mistake makes some interleaving deadlock or read the wrong data."""
    caught = False
    for case in CASES:
        B, Hq, Hkv, N, causal, sms = case
        P, ctas = schedule(B, Hq, Hkv, N, causal, sms)
        for seed in range(8):
            try:
                outputs = run_grid(P, ctas, 4, not sep, random.Random(seed), mutation=mutation, sep=sep)
                check_outputs(P, ctas, outputs)
            except (AssertionError, Deadlock):
                caught = True
                break
        if caught:
            break
    assert caught, f"mutation {mutation} went unnoticed"
