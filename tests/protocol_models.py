"""Random-interleaving models of the mbarrier protocols of the tensor-core
kernels (host only; no GPU code runs).

Every role of a kernel is a Python generator that yields the waits and
arrivals it performs; the scheduler runs any runnable role (or completes any
outstanding asynchronous operation) at random.  A run fails on

* a deadlock (nothing runnable, roles unfinished);
* a parity alias: mbarrier waits test the parity of a phase, so a waiter for
  phase k must proceed while the barrier has completed exactly k + 1 phases;
  a barrier two phases ahead would make the wait hang on the hardware;
* a broken hand-off: a buffer overwritten while a reader still needs it, or
  read before its producer wrote it.

Models:

* ``unit_ring`` -- attn_fwd_tc.cu: the producer warp draws unit ids from a
  counter shared by all CTAs and hands each to three consumer roles through a
  ring of R slots (full / empty barriers); -1 ends every role.
* ``dkdv_pair`` -- attn_bwd_tc.cu, dkdv_tc_kernel: producer (the unit's fixed
  K / V pair, one stage per step with its record), the S^T and dP^T issuers,
  the dV and dK issuers (tcgen05 commits arrive once the issuing thread's
  earlier MMAs are done, so each issuer is an in-order engine), the
  elementwise group and its epilogue, TMA copies landing at any time.

* ``score_gemm`` -- score_tc.cu (and qkv_tc.cu, with four stages): operand
  stage ring, two TMEM accumulators handed between the issuer and the
  epilogue.
* ``staging_ring`` -- qkv_tc.cu's epilogue: four warps stage each 64-column
  chunk in one of two shared-memory tiles, meet at one named barrier per
  chunk, then read the whole tile (row stores and block sums).
* ``fwd_pipeline`` -- attn_fwd_tc.cu after the unit ring: Q / K producer, V
  producer, the MMA issuer, the softmax group with its O rescale and
  epilogue.  Units without tiles do not signal O (mutation
  "o_final_for_empty_units" restores the earlier protocol, in which two such
  units in a row could leave o_final two phases past its waiter).

``mutation`` plants one mistake in the protocol (not in a kernel); the tests
require each to be caught.
"""
from __future__ import annotations

import random


class ProtocolError(Exception):
    pass


class _Bar:
    def __init__(self, count: int):
        self.count, self.arrived, self.done = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.done += 1


def _run(roles: dict, bars: dict, engines: dict, execute, rnd: random.Random):
    """Interleave `roles` (generators of ("wait", bar, phase) / ("arrive", bar))
    and the asynchronous `engines` (queues of operations run by `execute`)."""
    pending = {r: None for r in roles}
    done = set()
    while True:
        runnable = []
        for r, gen in roles.items():
            if r in done:
                continue
            if pending[r] is None:
                try:
                    pending[r] = next(gen)
                except StopIteration:
                    done.add(r)
                    continue
            op = pending[r]
            if op[0] == "arrive":
                runnable.append(("role", r))
            else:
                bar = bars[op[1]]
                if bar.done > op[2] + 1:
                    raise ProtocolError(f"parity alias: {r} waits {op[1]} phase {op[2]}, done {bar.done}")
                if bar.done > op[2]:
                    runnable.append(("role", r))
        runnable += [("engine", e) for e, q in engines.items() if q]
        if not runnable:
            if len(done) == len(roles):
                return
            raise ProtocolError(f"deadlock: {[pending[r] for r in roles if r not in done]}")
        kind, x = rnd.choice(runnable)
        if kind == "engine":
            execute(x, engines[x].pop(0))
        else:
            op = pending[x]
            pending[x] = None
            if op[0] == "arrive":
                bars[op[1]].arrive()


def unit_ring(n_units: int, n_cta: int, seed: int, R: int = 4, mutation: str | None = None) -> None:
    rnd = random.Random(seed)
    counter = [0]
    roles, bars, logs = {}, {}, []
    consumers = ("v_producer", "mma", "softmax")
    for c in range(n_cta):
        for s in range(R):
            bars[(c, "full", s)] = _Bar(1)
            bars[(c, "empty", s)] = _Bar(len(consumers) - (1 if mutation == "empty_count" else 0))
        slots = [None] * R
        log = {r: [] for r in ("producer",) + consumers}
        logs.append(log)

        def producer(c=c, slots=slots, log=log):
            k = 0
            while True:
                s = k % R
                if k >= R and mutation != "no_empty_wait":
                    yield ("wait", (c, "empty", s), k // R - 1)
                u = counter[0]
                counter[0] += 1
                slots[s] = u if u < n_units else -1
                log["producer"].append(slots[s])
                yield ("arrive", (c, "full", s))
                if u >= n_units:
                    return
                k += 1

        def consumer(name, c=c, slots=slots, log=log):
            k = 0
            while True:
                s = k % R
                yield ("wait", (c, "full", s), k // R)
                u = slots[s]
                log[name].append(u)
                yield ("arrive", (c, "empty", s))
                if u < 0:
                    return
                k += 1

        roles[(c, "producer")] = producer()
        for name in consumers:
            roles[(c, name)] = consumer(name)
    _run(roles, bars, {}, None, rnd)
    drawn = []
    for log in logs:
        for name in consumers:
            if log[name] != log["producer"]:
                raise ProtocolError(f"{name} saw {log[name]}, producer handed {log['producer']}")
        drawn += [u for u in log["producer"] if u >= 0]
    if sorted(drawn) != list(range(n_units)):
        raise ProtocolError("units lost or drawn twice")


def dkdv_pair(units: list, seed: int, KS: int = 4, mutation: str | None = None) -> None:
    """units: the number of steps of each unit this CTA runs (0 = no query
    block kept either key block)."""
    rnd = random.Random(seed)
    bars = {"fixed_full": _Bar(1), "fixed_empty": _Bar(2), "acc_full": _Bar(2), "acc_empty": _Bar(1),
            "drain": _Bar(4)}
    for s in range(KS):
        bars[f"in_full{s}"] = _Bar(1)
        bars[f"in_empty{s}"] = _Bar(2)
    for b in range(2):
        bars[f"s_full{b}"] = _Bar(2)
        bars[f"pd_full{b}"] = _Bar(1)
        bars[f"pd_empty{b}"] = _Bar(1 if mutation == "pd_empty_count" else 2)
    st = {"stage": [None] * KS, "stage_readers": [set() for _ in range(KS)], "record": [None] * KS,
          "buf": [dict(S=None, dP=None, P=None, readers=set()) for _ in range(2)],
          "kv": None, "kv_readers": set(), "acc": {"dV": None, "dK": None}, "epilogue_done": -1}
    engines = {e: [] for e in ("S", "dP", "dV", "dK", "tma")}

    def producer():
        g = fixed = 0
        for u, n in enumerate(units):
            if n == 0:
                continue
            if fixed > 0:
                yield ("wait", "fixed_empty", fixed - 1)
            engines["tma"].append(("kv", u))
            fixed += 1
            for t in range(n):
                s, use = g % KS, g // KS
                if use > 0:
                    yield ("wait", f"in_empty{s}", use - 1)
                if st["stage_readers"][s]:
                    raise ProtocolError(f"record of step {g} written while {st['stage_readers'][s]} read stage {s}")
                st["record"][s] = (u, t, n, g)
                engines["tma"].append(("stage", g, s))
                g += 1

    def s_issuer(name):
        g = fixed = 0
        for u, n in enumerate(units):
            if n == 0:
                continue
            yield ("wait", "fixed_full", fixed)
            fixed += 1
            steps, t = -1, 0
            while steps < 0 or t < steps:
                s, b = g % KS, g & 1
                yield ("wait", f"in_full{s}", g // KS)
                rec = st["record"][s]
                if rec[3] != g:
                    raise ProtocolError(f"{name} read the record of step {rec[3]} at step {g}")
                steps = rec[2] if steps < 0 else steps
                if g >= 2 and mutation != "no_buffer_wait":
                    yield ("wait", f"pd_empty{b}", (g >> 1) - 1)
                st["stage_readers"][s].add((name, g))
                st["kv_readers"].add((name, u))
                engines[name].append(("mma", g, s, b, u))
                engines[name].append(("commit", f"s_full{b}"))
                t += 1
                g += 1
            engines[name].append(("commit", "fixed_empty"))
        engines[name].append(("commit", "drain"))

    def acc_issuer(name):
        g = 0
        for u, n in enumerate(units):
            if u > 0 and mutation != "no_acc_wait":
                yield ("wait", "acc_empty", u - 1)
            steps, t = (0 if n == 0 else -1), 0
            while steps < 0 or t < steps:
                s, b = g % KS, g & 1
                yield ("wait", f"pd_full{b}", g >> 1)
                rec = st["record"][s]
                if rec[3] != g:
                    raise ProtocolError(f"{name} read the record of step {rec[3]} at step {g}")
                steps = rec[2] if steps < 0 else steps
                st["stage_readers"][s].add((name, g))
                st["buf"][b]["readers"].add((name, g))
                engines[name].append(("mma", g, s, b, u, t))
                engines[name].append(("commit", f"pd_empty{b}"))
                if mutation != "no_stage_release":
                    engines[name].append(("commit", f"in_empty{s}"))
                t += 1
                g += 1
            engines[name].append(("commit", "acc_full"))
        engines[name].append(("commit", "drain"))

    def elementwise():
        g = 0
        for u, n in enumerate(units):
            steps, t = (0 if n == 0 else -1), 0
            while steps < 0 or t < steps:
                s, b = g % KS, g & 1
                yield ("wait", f"s_full{b}", g >> 1)
                yield ("wait", f"in_full{s}", g // KS)
                rec = st["record"][s]
                if rec[3] != g:
                    raise ProtocolError(f"elementwise read the record of step {rec[3]} at step {g}")
                steps = rec[2] if steps < 0 else steps
                buf = st["buf"][b]
                if buf["S"] != g or buf["dP"] != g:
                    raise ProtocolError(f"elementwise read S {buf['S']} / dP {buf['dP']} at step {g}")
                if st["stage"][s] != g:
                    raise ProtocolError(f"elementwise read stats of step {st['stage'][s]} at step {g}")
                buf["P"] = g
                yield ("arrive", f"pd_full{b}")
                t += 1
                g += 1
            yield ("wait", "acc_full", u)
            want = (u, steps - 1) if steps > 0 else None
            if steps > 0 and (st["acc"]["dV"] != want or st["acc"]["dK"] != want):
                raise ProtocolError(f"epilogue of unit {u} read accumulators {st['acc']}")
            st["epilogue_done"] = u
            yield ("arrive", "acc_empty")

    def execute(e, op):
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        if e == "tma":
            if op[0] == "kv":
                live = [x for x in st["kv_readers"] if x[1] != op[1]]
                if live:
                    raise ProtocolError(f"K / V pair overwritten while {live} read it")
                st["kv"] = op[1]
                bars["fixed_full"].arrive()
            else:
                _, g, s = op
                live = [x for x in st["stage_readers"][s] if x[1] != g]
                if live:
                    raise ProtocolError(f"stage {s} overwritten for step {g} while {live} read it")
                st["stage"][s] = g
                bars[f"in_full{s}"].arrive()
            return
        if e in ("S", "dP"):
            _, g, s, b, u = op
            buf = st["buf"][b]
            if st["stage"][s] != g or st["kv"] != u:
                raise ProtocolError(f"{e} of step {g} read stage {st['stage'][s]} / K-V {st['kv']}")
            if g >= 2 and (any(x[1] == g - 2 for x in buf["readers"]) or buf["P"] != g - 2):
                raise ProtocolError(f"{e} of step {g} overwrote buffer {b} before step {g - 2} was done with it")
            buf[e] = g
            st["stage_readers"][s].discard((e, g))
            st["kv_readers"].discard((e, u))
            return
        _, g, s, b, u, t = op
        buf = st["buf"][b]
        if buf["P"] != g or st["stage"][s] != g:
            raise ProtocolError(f"{e} of step {g} read P of {buf['P']} / stage {st['stage'][s]}")
        if t == 0 and st["epilogue_done"] < u - 1:
            raise ProtocolError(f"{e} overwrote the accumulator before the epilogue of unit {u - 1}")
        st["acc"][e] = (u, t)
        buf["readers"].discard((e, g))
        st["stage_readers"][s].discard((e, g))

    roles = {"producer": producer(), "S": s_issuer("S"), "dP": s_issuer("dP"), "dV": acc_issuer("dV"),
             "dK": acc_issuer("dK"), "elementwise": elementwise()}
    _run(roles, bars, engines, execute, rnd)
    if bars["drain"].done != 1:
        raise ProtocolError("teardown barrier did not complete")


def fwd_pipeline(units: list, seed: int, KS: int = 3, VS: int = 2, mutation: str | None = None) -> None:
    """attn_fwd_tc.cu, one CTA after the unit ring: the Q / K producer, the V
    producer, the single MMA issuer (S of tile g into TMEM buffer g & 1, then
    P V of tile g - 1; its MMAs and commits complete in issue order), the
    softmax group (P over S, a rescale of O that waits for P V of tile g - 1,
    the epilogue) and TMA copies landing at any time.  units: tiles per unit."""
    rnd = random.Random(seed)
    bars = {"q_full": _Bar(1), "q_empty": _Bar(1), "o_done": _Bar(1), "o_final": _Bar(1)}
    for s in range(KS):
        bars[f"k_full{s}"] = _Bar(1)
        bars[f"k_empty{s}"] = _Bar(1)
    for s in range(VS):
        bars[f"v_full{s}"] = _Bar(1)
        bars[f"v_empty{s}"] = _Bar(1)
    for b in range(2):
        bars[f"s_full{b}"] = _Bar(1)
        bars[f"p_full{b}"] = _Bar(1)
    st = {"q": None, "q_readers": set(), "k": [None] * KS, "k_readers": [set() for _ in range(KS)],
          "v": [None] * VS, "v_readers": [set() for _ in range(VS)],
          "buf": [dict(S=None, P=None) for _ in range(2)], "pv_done": -1, "o_unit": None,
          "epilogue_done": -1}
    first = []  # global index of each unit's first tile
    g = 0
    for n in units:
        first.append(g)
        g += n
    engines = {"mma": [], "tma": []}

    def qk_producer():
        g = q_it = 0
        for u, n in enumerate(units):
            if q_it > 0 and mutation != "no_q_wait":
                yield ("wait", "q_empty", q_it - 1)
            engines["tma"].append(("q", u))
            q_it += 1
            for _ in range(n):
                s, use = g % KS, g // KS
                if use > 0:
                    yield ("wait", f"k_empty{s}", use - 1)
                engines["tma"].append(("k", g, s))
                g += 1

    def v_producer():
        g = 0
        for n in units:
            for _ in range(n):
                s, use = g % VS, g // VS
                if use > 0 and mutation != "no_v_wait":
                    yield ("wait", f"v_empty{s}", use - 1)
                engines["tma"].append(("v", g, s))
                g += 1

    def mma():
        g = 0
        for u, n in enumerate(units):
            yield ("wait", "q_full", u)
            for t in range(n):
                s = g % KS
                if mutation != "no_k_wait":
                    yield ("wait", f"k_full{s}", g // KS)
                st["q_readers"].add(("S", g))
                st["k_readers"][s].add(g)
                engines["mma"].append(("S", g, u))
                engines["mma"].append(("commit", f"k_empty{s}"))
                engines["mma"].append(("commit", f"s_full{g & 1}"))
                if t >= 1:
                    yield from _pv(g - 1, u)
                g += 1
            if n >= 1:
                yield from _pv(g - 1, u)
                engines["mma"].append(("commit", "o_final"))  # only units with tiles signal O
            elif mutation == "o_final_for_empty_units":
                engines["mma"].append(("commit", "o_final"))
            engines["mma"].append(("commit", "q_empty"))

    def _pv(h, u):
        yield ("wait", f"p_full{h & 1}", h >> 1)
        yield ("wait", f"v_full{h % VS}", h // VS)
        st["v_readers"][h % VS].add(h)
        engines["mma"].append(("PV", h, u))
        engines["mma"].append(("commit", f"v_empty{h % VS}"))
        engines["mma"].append(("commit", "o_done"))

    def softmax():
        g = finals = 0  # finals: o_final phases waited for (units with tiles)
        for u, n in enumerate(units):
            for t in range(n):
                b = g & 1
                yield ("wait", f"s_full{b}", g >> 1)
                if st["buf"][b]["S"] != g:
                    raise ProtocolError(f"softmax read S of tile {st['buf'][b]['S']} at tile {g}")
                if t >= 1 and rnd.random() < 0.3:  # the running max grew: rescale O
                    lag = 2 if mutation == "rescale_lag" else 1
                    yield ("wait", "o_done", g - lag)
                    if st["pv_done"] != g - 1:
                        raise ProtocolError(f"O rescaled at tile {g} with P V done up to {st['pv_done']}")
                st["buf"][b]["P"] = g
                yield ("arrive", f"p_full{b}")
                g += 1
            if n > 0 or mutation == "o_final_for_empty_units":
                yield ("wait", "o_final", finals)
                finals += 1
            if n > 0 and st["pv_done"] != first[u] + n - 1:
                raise ProtocolError(f"epilogue of unit {u} read O with P V done up to {st['pv_done']}")
            st["epilogue_done"] = u

    def execute(e, op):
        if op[0] == "commit":
            bars[op[1]].arrive()
            return
        if op[0] == "q":
            if st["q_readers"]:
                raise ProtocolError(f"Q of unit {op[1]} landed while {st['q_readers']} read the previous one")
            st["q"] = op[1]
            bars["q_full"].arrive()
        elif op[0] == "k":
            _, g, s = op
            if st["k_readers"][s]:
                raise ProtocolError(f"K slot {s} refilled for tile {g} while tiles {st['k_readers'][s]} read it")
            st["k"][s] = g
            bars[f"k_full{s}"].arrive()
        elif op[0] == "v":
            _, g, s = op
            if st["v_readers"][s]:
                raise ProtocolError(f"V slot {s} refilled for tile {g} while tiles {st['v_readers'][s]} read it")
            st["v"][s] = g
            bars[f"v_full{s}"].arrive()
        elif op[0] == "S":
            _, g, u = op
            buf = st["buf"][g & 1]
            if st["q"] != u or st["k"][g % KS] != g:
                raise ProtocolError(f"S of tile {g} read Q of unit {st['q']} / K of tile {st['k'][g % KS]}")
            if g >= 2 and (buf["P"] != g - 2 or st["pv_done"] < g - 2):
                raise ProtocolError(f"S of tile {g} overwrote buffer {g & 1} before P V of tile {g - 2}")
            buf["S"] = g
            st["q_readers"].discard(("S", g))
            st["k_readers"][g % KS].discard(g)
        else:
            _, h, u = op
            if st["buf"][h & 1]["P"] != h or st["v"][h % VS] != h:
                raise ProtocolError(f"P V of tile {h} read P of {st['buf'][h & 1]['P']} / V of {st['v'][h % VS]}")
            if h == first[u] and st["epilogue_done"] < u - 1:
                raise ProtocolError(f"P V of tile {h} overwrote O before the epilogue of unit {u - 1}")
            st["pv_done"] = h
            st["v_readers"][h % VS].discard(h)

    roles = {"qk_producer": qk_producer(), "v_producer": v_producer(), "mma": mma(), "softmax": softmax()}
    _run(roles, bars, engines, execute, rnd)


def score_gemm(n_tiles: int, seed: int, S: int = 2, n_sub: int = 4, mutation: str | None = None) -> None:
    """score_tc.cu: the producer streams n_sub operand sub-chunks per tile
    through S stages (full / empty), the issuer accumulates each tile into one
    of two TMEM accumulators (acc_full after its last sub-chunk; before reusing
    an accumulator it waits acc_empty of the tile two back), and the epilogue
    drains them in tile order and releases each one once read.  Mutations:
    "no_stage_wait" (the producer refills a stage without waiting empty),
    "no_acc_wait" (the issuer reuses an accumulator without waiting acc_empty),
    "early_release" (the epilogue releases an accumulator before reading it)."""
    rnd = random.Random(seed)
    bars = {}
    for s in range(S):
        bars[f"full{s}"] = _Bar(1)
        bars[f"empty{s}"] = _Bar(1)
    for b in range(2):
        bars[f"acc_full{b}"] = _Bar(1)
        bars[f"acc_empty{b}"] = _Bar(1)
    bars["tick"] = _Bar(1)
    st = {"stage": [None] * S, "acc": [None, None], "chunks": [0, 0], "reading": [False, False], "drained": []}
    engines = {"tma": [], "mma": []}

    def producer():
        g = 0
        for t in range(n_tiles):
            for s in range(n_sub):
                k, use = g % S, g // S
                if use > 0 and mutation != "no_stage_wait":
                    yield ("wait", f"empty{k}", use - 1)
                engines["tma"].append(("load", k, (t, s)))
                g += 1

    def issuer():
        g = 0
        for lt in range(n_tiles):
            ab = lt & 1
            if lt >= 2 and mutation != "no_acc_wait":
                yield ("wait", f"acc_empty{ab}", (lt >> 1) - 1)
            for s in range(n_sub):
                k = g % S
                yield ("wait", f"full{k}", g // S)
                engines["mma"].append(("mma", k, (lt, s), ab))
                engines["mma"].append(("commit", f"empty{k}"))
                g += 1
            engines["mma"].append(("commit", f"acc_full{ab}"))

    def epilogue():
        for lt in range(n_tiles):
            ab = lt & 1
            yield ("wait", f"acc_full{ab}", lt >> 1)
            if mutation == "early_release":
                yield ("arrive", f"acc_empty{ab}")
            if st["acc"][ab] != lt or st["chunks"][ab] != n_sub:
                raise ProtocolError(f"epilogue of tile {lt} found {st['acc'][ab]} with {st['chunks'][ab]} chunks")
            st["reading"][ab] = True
            yield ("arrive", "tick")                  # the TMEM loads take a while
            if st["acc"][ab] != lt or st["chunks"][ab] != n_sub:
                raise ProtocolError(f"accumulator {ab} overwritten while tile {lt} was read")
            st["reading"][ab] = False
            st["drained"].append(lt)
            if mutation != "early_release":
                yield ("arrive", f"acc_empty{ab}")

    def execute(e, op):
        if op[0] == "load":
            st["stage"][op[1]] = op[2]
            bars[f"full{op[1]}"].arrive()
        elif op[0] == "mma":
            _, k, want, ab = op
            if st["stage"][k] != want:
                raise ProtocolError(f"MMA of {want} read stage {k} holding {st['stage'][k]}")
            lt, s = want
            if s == 0:
                if st["reading"][ab]:
                    raise ProtocolError(f"tile {lt} started accumulator {ab} during the previous tile's read")
                st["acc"][ab], st["chunks"][ab] = lt, 1
            else:
                if st["acc"][ab] != lt or st["chunks"][ab] != s:
                    raise ProtocolError(f"tile {lt} sub-chunk {s} found accumulator {ab} = {st['acc'][ab]}")
                st["chunks"][ab] += 1
        else:
            bars[op[1]].arrive()

    _run({"producer": producer(), "issuer": issuer(), "epilogue": epilogue()}, bars, engines, execute, rnd)
    if st["drained"] != list(range(n_tiles)):
        raise ProtocolError(f"tiles drained {st['drained']}")


def staging_ring(n_chunks: int, seed: int, n_warps: int = 4, mutation: str | None = None) -> None:
    """qkv_tc.cu's epilogue: for chunk c every warp writes its rows into
    staging tile c % 2, arrives at the named barrier (one phase per chunk) and
    waits for it, then reads rows of every warp.  A warp writes tile c % 2
    again only at chunk c + 2, after the barrier of chunk c + 1, which no warp
    reaches before it has finished reading chunk c.  Mutation "one_tile" stages
    every chunk in the same tile."""
    rnd = random.Random(seed)
    bars = {"named": _Bar(n_warps)}
    st = {"tile": [dict(), dict()], "readers": [set(), set()]}

    def warp(w):
        for c in range(n_chunks):
            b = 0 if mutation == "one_tile" else c & 1
            if st["readers"][b] - {w}:
                raise ProtocolError(f"warp {w} writes tile {b} for chunk {c} while {st['readers'][b]} read it")
            st["tile"][b][w] = c
            yield ("arrive", "named")
            yield ("wait", "named", c)
            st["readers"][b].add(w)
            for v in range(n_warps):
                if st["tile"][b].get(v) != c:
                    raise ProtocolError(f"warp {w} reads chunk {c} and finds warp {v}'s rows of {st['tile'][b].get(v)}")
                yield ("arrive", f"tick{w}")          # the reads take a while
            st["readers"][b].discard(w)

    for w in range(n_warps):
        bars[f"tick{w}"] = _Bar(1)
    _run({f"warp{w}": warp(w) for w in range(n_warps)}, bars, {}, lambda e, op: None, rnd)
