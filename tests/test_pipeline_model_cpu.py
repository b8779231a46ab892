"""A randomised model of the forward kernel's synchronisation protocol where
one MMA-issuing thread serves each Q tile (attn_fwd_kernel.cuh:
mma_role_tile, producer_role, softmax_role; d = 64 and block-sparse units).

The model runs the roles as coroutines under a random scheduler: the Q/K
and V loaders, the two issuing threads, the two softmax groups, an in-order
tensor pipe that executes MMAs and commits some time after they are issued,
and a copy engine that lands TMA copies in any order.  Barriers are mbarriers
with an arrival count and a phase counter.  It checks, on every interleaving
it draws:

  * every parity wait is for the barrier's current phase or the one before
    (the only phases a parity bit can tell apart), and its parity answer
    equals the true one;
  * every arrival lands in the phase it is meant for;
  * every MMA reads the Q, K, V, S and P it expects, O is rescaled only
    after every earlier P.V, and the epilogue reads the complete O;
  * nothing deadlocks.

Units are lists of K/V tiles, each marked with the Q tiles that compute it
(dense pairs, causal pairs, single tiles, block-sparse unions).  The second
test plants the mistakes the protocol guards against and checks that the
model catches each.
"""
import random

import pytest


class Deadlock(Exception):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, phase=None):
        if phase is not None:
            assert phase == self.done, (self.name, "arrival for phase", phase, "in", self.done)
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1

    def passed(self, phase):
        """Parity probe for `phase` (absolute); checks it is exact."""
        if phase < 0:
            return True
        assert self.done <= phase + 1, (self.name, "two phases ahead", self.done, phase)
        by_parity = (self.done & 1) != (phase & 1)
        assert by_parity == (self.done > phase), (self.name, "parity alias", self.done, phase)
        return by_parity


def simulate(units, split, sparse, seed, k_stages=2, v_stages=2, plant=None):
    """Run one random interleaving; raises on a violated check or a
    deadlock.  units: lists of use bits per K/V tile (bit t: Q tile t
    computes it).  split: P in its own TMEM columns (d = 64)."""
    rnd = random.Random(seed)
    bars = {}

    def mk(name, count=1):
        bars[name] = Barrier(name, count)

    for t in range(2):
        for nm in ("Q_FULL", "Q_EMPTY", "S_FULL", "P_HALF", "P_FULL", "S_FREE",
                   "O_FULL", "O_EMPTY"):
            mk((nm, t))
    for s in range(k_stages):
        mk(("K_FULL", s))
        mk(("K_EMPTY", s), 2)
    for s in range(v_stages):
        mk(("V_FULL", s))
        mk(("V_EMPTY", s), 2)
    mk("DRAIN", 2)
    smem_q, smem_k, smem_v = [None, None], [None] * k_stages, [None] * v_stages
    tmem_s, tmem_p, tmem_o = [None, None], [None, None], [None, None]
    k_pos, v_pos = [-1] * k_stages, [-1] * v_stages
    pipe, copies, finished = [], [], set()

    def counts(u):
        return (sum(1 for b in u if b & 1), sum(1 for b in u if b & 2), len(u))

    def wait(name, phase):
        while not bars[name].passed(phase):
            yield

    def loader(qk):
        q_occ, k_n, v_n = [0, 0], 0, 0
        for ui, u in enumerate(units):
            n0, n1, nu = counts(u)
            if qk:
                for t, n in enumerate((n0, n1)):
                    if n == 0:
                        continue
                    yield from wait(("Q_EMPTY", t), q_occ[t] - 1)
                    q_occ[t] += 1
                    copies.append((("Q_FULL", t), smem_q, t, ("Q", ui, t)))
            for j in range(nu):
                one_user = u[j] != 3
                if qk:
                    st = k_n % k_stages
                    yield from wait(("K_EMPTY", st), k_n // k_stages - 1)
                    if plant != "no_slot_index":
                        k_pos[st] = k_n
                    if one_user and plant != "no_loader_arrival":
                        bars[("K_EMPTY", st)].arrive(k_n // k_stages)
                    yield
                    copies.append((("K_FULL", st), smem_k, st, ("K", ui, j)))
                    k_n += 1
                else:
                    st = v_n % v_stages
                    yield from wait(("V_EMPTY", st), v_n // v_stages - 1)
                    if plant != "no_slot_index":
                        v_pos[st] = v_n
                    if one_user:
                        bars[("V_EMPTY", st)].arrive(v_n // v_stages)
                    yield
                    copies.append((("V_FULL", st), smem_v, st, ("V", ui, j)))
                    v_n += 1
                yield

    def slot_claimed(pos, idx):
        if plant == "no_slot_index":
            return
        while pos[idx % len(pos)] != idx:
            assert pos[idx % len(pos)] < idx
            yield

    def issuer(t):
        q_occ = p_cnt = o_occ = s_done = 0
        ring = 0
        for ui, u in enumerate(units):
            n = counts(u)[t]
            nu = len(u)
            if n == 0:
                ring += nu
                continue
            mine = [i for i in range(nu) if (u[i] >> t) & 1]

            def issue_s(at, j):
                nonlocal s_done
                if split and s_done > 0:
                    yield from wait(("S_FREE", t), s_done - 1)
                ka = ring + at
                yield from slot_claimed(k_pos, ka)
                yield from wait(("K_FULL", ka % k_stages), ka // k_stages)
                pipe.append(("S", ui, t, at, ka % k_stages))
                pipe.append(("commit", ("S_FULL", t), None))
                if j + 1 == n:
                    pipe.append(("commit", ("Q_EMPTY", t), None))
                pipe.append(("commit", ("K_EMPTY", ka % k_stages), ka // k_stages))
                s_done += 1

            yield from wait(("Q_FULL", t), q_occ)
            q_occ += 1
            yield from issue_s(mine[0], 0)
            for j in range(n):
                at = mine[j]
                early = False
                if split and j + 1 < n:
                    early = True
                    if sparse and plant != "sparse_waits_for_k":
                        # ahead of the P.V only if that K tile has landed
                        yield from wait(("S_FREE", t), s_done - 1)
                        ka = ring + mine[j + 1]
                        early = (k_pos[ka % k_stages] == ka and
                                 bars[("K_FULL", ka % k_stages)].passed(ka // k_stages))
                    if early:
                        yield from issue_s(mine[j + 1], j + 1)
                yield from wait(("P_HALF", t), p_cnt)
                va = ring + at
                yield from slot_claimed(v_pos, va)
                yield from wait(("V_FULL", va % v_stages), va // v_stages)
                if j == 0 and o_occ > 0:
                    yield from wait(("O_EMPTY", t), o_occ - 1)
                pipe.append(("PV", ui, t, j, at, 0, va % v_stages))
                yield
                yield from wait(("P_FULL", t), p_cnt)
                pipe.append(("PV", ui, t, j, at, 1, va % v_stages))
                p_cnt += 1
                pipe.append(("commit", ("O_FULL", t), None))
                pipe.append(("commit", ("V_EMPTY", va % v_stages), va // v_stages))
                if not early and j + 1 < n:
                    yield from issue_s(mine[j + 1], j + 1)
                yield
            ring += nu
            o_occ += 1
        pipe.append(("commit", "DRAIN", None))
        yield from wait("DRAIN", 0)

    def softmax(t):
        s_cnt = o_cnt = 0
        for ui, u in enumerate(units):
            n = counts(u)[t]
            if n == 0:
                continue
            mine = [i for i in range(len(u)) if (u[i] >> t) & 1]
            for j in range(n):
                yield from wait(("S_FULL", t), s_cnt)
                s_cnt += 1
                assert tmem_s[t] == ("S", ui, t, mine[j]), ("stale S", tmem_s[t], ui, t, j)
                yield
                if split:
                    bars[("S_FREE", t)].arrive()
                    yield
                    if j > 0 and plant != "no_pv_wait":
                        yield from wait(("O_FULL", t), o_cnt)
                        o_cnt += 1
                if j > 0 and (not split or plant != "no_pv_wait"):
                    assert tmem_o[t] == (ui, t, mine[:j]), ("rescale too early", tmem_o[t])
                half = ("Pa", ui, t, mine[j])
                if split:
                    tmem_p[t] = half
                else:
                    tmem_s[t] = half
                yield
                bars[("P_HALF", t)].arrive()
                yield
                full = ("P", ui, t, mine[j])
                if split:
                    tmem_p[t] = full
                else:
                    tmem_s[t] = full
                bars[("P_FULL", t)].arrive()
                yield
            last = o_cnt if split else o_cnt + n - 1
            if split and plant == "no_pv_wait":
                last = o_cnt + n - 1
            yield from wait(("O_FULL", t), last)
            o_cnt = last + 1
            assert tmem_o[t] == (ui, t, mine), ("incomplete O", tmem_o[t], ui, t)
            finished.add((ui, t))
            tmem_o[t] = ("read",)
            bars[("O_EMPTY", t)].arrive()
            yield

    def tensor_pipe():
        while True:
            if pipe:
                op = pipe.pop(0)
                if op[0] == "commit":
                    bars[op[1]].arrive(op[2])
                elif op[0] == "S":
                    _, ui, t, at, st = op
                    assert smem_q[t] == ("Q", ui, t), ("S reads stale Q", smem_q[t], op)
                    assert smem_k[st] == ("K", ui, at), ("S reads wrong K", smem_k[st], op)
                    tmem_s[t] = ("S", ui, t, at)
                else:
                    _, ui, t, j, at, h, st = op
                    assert smem_v[st] == ("V", ui, at), ("P.V reads wrong V", smem_v[st], op)
                    src = tmem_p[t] if split else tmem_s[t]
                    ok = (("Pa", ui, t, at), ("P", ui, t, at)) if h == 0 else (("P", ui, t, at),)
                    assert src in ok, ("P.V reads wrong P", src, op)
                    if j == 0 and h == 0:
                        assert tmem_o[t] in (None, ("read",)), ("O overwritten", tmem_o[t])
                        tmem_o[t] = (ui, t, [])
                    if h == 1:
                        tmem_o[t][2].append(at)
            yield

    def copy_engine():
        while True:
            if copies:
                name, mem, idx, data = copies.pop(rnd.randrange(len(copies)))
                mem[idx] = data
                bars[name].arrive()
            yield

    roles = {"qk": loader(True), "v": loader(False), "mma0": issuer(0), "mma1": issuer(1),
             "sm0": softmax(0), "sm1": softmax(1)}
    engines = [tensor_pipe(), copy_engine()]
    steps = 0
    while roles:
        steps += 1
        if steps > 400_000:
            raise Deadlock(sorted(roles))
        r = rnd.random()
        if r < 0.25:
            next(engines[0])
        elif r < 0.4:
            next(engines[1])
        else:
            k = rnd.choice(sorted(roles))
            try:
                next(roles[k])
            except StopIteration:
                del roles[k]
    want = {(ui, t) for ui, u in enumerate(units) for t in range(2) if counts(u)[t]}
    assert finished == want


def _units(rnd, sparse):
    units = []
    for _ in range(rnd.randint(1, 5)):
        kind = rnd.random()
        if kind < 0.25:
            units.append([3] * rnd.randint(1, 8))                     # dense pair
        elif kind < 0.5:
            units.append([3] * rnd.randint(1, 7) + [2])               # causal pair
        elif kind < 0.6:
            units.append([1] * rnd.randint(1, 8))                     # single tile
        elif sparse:
            units.append([rnd.choice([1, 2, 3]) for _ in range(rnd.randint(1, 10))])
        else:
            units.append([3] * rnd.randint(1, 8))
    return units


CONFIGS = [(split, sparse, ks, vs) for split in (False, True) for sparse in (False, True)
           for ks, vs in ((2, 2), (4, 4), (2, 3))]


@pytest.mark.parametrize("split,sparse,k_stages,v_stages", CONFIGS)
def test_protocol_holds_on_random_interleavings(split, sparse, k_stages, v_stages):
    for seed in range(25):
        rnd = random.Random(1000 * k_stages + 10 * v_stages + seed)
        simulate(_units(rnd, sparse), split, sparse, seed, k_stages, v_stages)


@pytest.mark.parametrize("plant,split,sparse", [
    ("no_slot_index", False, True),        # parity probe on a slot not yet claimed
    ("no_loader_arrival", False, True),    # a slot one tile skips is never released
    ("sparse_waits_for_k", True, True),    # next S waits for its K ahead of the P.V
    ("no_pv_wait", True, False),           # P overwritten / O rescaled too early
])
def test_model_catches_planted_mistakes(plant, split, sparse):
    caught = 0
    for seed in range(80):
        rnd = random.Random(7 + seed)
        units = _units(rnd, sparse)
        if sparse:
            # one tile with long runs of K tiles only the other one computes
            units.append([3] + [1] * rnd.randint(3, 7) + [3, 2, 3, 3])
        try:
            simulate(units, split, sparse, seed, 2, 2, plant=plant)
        except (AssertionError, Deadlock):
            caught += 1
    assert caught > 0, plant
