"""Host-side model check of the kernels' barrier protocols: the forward and
backward tile kernels (fwd_sm100.cuh, bwd_sm100.cuh), the persistent backward
(bwd_persist_sm100.cuh) and the persistent forward (fwd_persist_sm100.cuh).

Each role of a block (the TMA producers, the MMA issuer, the sigma
warpgroups) is written as the sequence of barrier waits, arrivals, tensor-core
MMAs, commits, TMA loads and TMEM reads and writes that the kernels run.  MMAs and commits complete in issue order at arbitrary
later times (one tensor pipe per block), and TMA loads land at arbitrary later
times.  Many random interleavings, with per-run random speeds per role, are
explored, and each is checked for:

* parity aliasing: an mbarrier parity wait cannot tell phase k from phase
  k + 2, so a wait that starts when its barrier has already completed two
  phases past the one it wants blocks for good (the kernel would end in its
  bounded-wait timeout);
* miscounted phases: every arrival lands in the phase its sender means (a
  fast warpgroup's arrival for tile i + 1 must never complete tile i's phase);
* data flow: every read of a TMEM buffer, ring slot or accumulator, by an MMA
  when it runs or by a warpgroup when it loads, finds the tile it expects;
* progress: every role finishes (no deadlock).

The kernels' protocols pass at several ring depths, tile counts, item mixes
and warpgroup counts.  Planted mistakes must be caught: the two-buffer dK/dV
form with one readiness barrier each for P^T and dS^T (the warpgroups can
finish tile i + 1 before the MMA thread has waited for tile i), an S MMA
issued without waiting for the warpgroups to have read the previous S, a P^T
readiness arrival sent before P^T is written, a resident slot of the
persistent backward reloaded too early, and the persistent forward's first
build, with one scores-ready barrier per TMEM buffer shared by both query
tiles.
"""
import random
import re

import pytest


class ProtocolError(Exception):
    pass


class Barrier:
    def __init__(self, count):
        self.count, self.arrived, self.done = count, 0, 0   # done: completed phases

    def arrive(self, who, name, phase):
        if phase is not None and phase != self.done:
            raise ProtocolError(f"{who} arrives on {name} for phase {phase}, "
                                f"but phase {self.done} is open")
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived, self.done = 0, self.done + 1


class Model:
    """Roles are generators of ops:
    ('wait', bar, phase)                  parity wait for `phase` of `bar`
    ('arrive', bar, phase)                plain arrival on the open `phase`
    ('mma', reads, writes)                queued on the pipe; reads/writes are
                                          lists of (buffer, tile)
    ('commit', bar, phase)                queued; arrives once earlier MMAs ran
    ('tma', bar, phase, buffer, tile)     lands later, then arrives
    ('use', buffer, tile)                 warpgroup reads a buffer now
    ('write', buffer, tile)               warpgroup writes a buffer now"""

    def __init__(self, barriers, roles, seed):
        self.bars = {k: Barrier(c) for k, c in barriers.items()}
        self.roles = roles
        self.rng = random.Random(seed)
        self.speed = {name: self.rng.choice((0.05, 0.3, 1.0, 3.0)) for name in roles}
        self.speed["pipe"] = self.rng.choice((0.1, 1.0, 3.0))
        self.speed["tma"] = self.rng.choice((0.1, 1.0, 3.0))
        self.buf = {}
        self.pipe = []
        self.tma = []

    def _check(self, who, buffer, tile):
        got = self.buf.get(buffer)
        if got != tile:
            raise ProtocolError(f"{who} reads {buffer} expecting {tile}, finds {got}")

    def run(self, max_steps=500000):
        gens = dict(self.roles)
        cur = {name: next(g, None) for name, g in gens.items()}
        for _ in range(max_steps):
            ready = []
            for name, op in cur.items():
                if op is None:
                    continue
                if op[0] == "wait":
                    bar = self.bars[op[1]]
                    if bar.done >= op[2] + 2:
                        raise ProtocolError(f"{name} waits for phase {op[2]} of {op[1]}, "
                                            f"which has completed {bar.done} phases")
                    if bar.done == op[2] + 1:
                        ready.append(name)
                else:
                    ready.append(name)
            if self.pipe:
                ready.append("pipe")
            if self.tma:
                ready.append("tma")
            if not ready:
                if all(op is None for op in cur.values()):
                    return
                raise ProtocolError("deadlock: " + "; ".join(
                    f"{n} at {op}" for n, op in cur.items() if op is not None))
            ev = self.rng.choices(ready, weights=[self.speed[e] for e in ready])[0]
            if ev == "pipe":
                item = self.pipe.pop(0)
                if item[0] == "mma":
                    for b, t in item[1]:
                        self._check("an MMA", b, t)
                    for b, t in item[2]:
                        self.buf[b] = t
                else:
                    self.bars[item[1]].arrive("a commit", item[1], item[2])
                continue
            if ev == "tma":
                _, bar, phase, b, t = self.tma.pop(self.rng.randrange(len(self.tma)))
                self.buf[b] = t
                self.bars[bar].arrive("a TMA load", bar, phase)
                continue
            op = cur[ev]
            kind = op[0]
            if kind == "arrive":
                self.bars[op[1]].arrive(ev, op[1], op[2])
            elif kind in ("mma", "commit"):
                self.pipe.append(op)
            elif kind == "tma":
                self.tma.append(op)
            elif kind == "use":
                self._check(ev, op[1], op[2])
            elif kind == "write":
                self.buf[op[1]] = op[2]
            cur[ev] = next(gens[ev], None)
        raise ProtocolError("step limit")


def _ring_producer(n, S, full, empty, ring, tile, resident=()):
    """ring_load over tiles 0..n-1 into S slots, then ring_drain; `resident`
    lists (buffer, tile) loads issued first on the res_full barrier."""
    def g():
        for b, t in resident:
            yield ("tma", "res_full", 0, b, t)
        for j in range(n):
            if j >= S:
                yield ("wait", f"{empty}{j % S}", j // S - 1)
            yield ("tma", f"{full}{j % S}", j // S, f"{ring}{j % S}", f"{tile}{j}")
        if resident:
            yield ("wait", "res_full", 0)
        for j in range(max(n - S, 0), n):
            yield ("wait", f"{full}{j % S}", j // S)
    return g()


def _ring_barriers(SX, SY):
    bars = {"res_full": 2, "s_full": 1, "drain": 1}
    for s in range(SX):
        bars[f"x_full{s}"] = 1
        bars[f"x_empty{s}"] = 1
    for s in range(SY):
        bars[f"y_full{s}"] = 1
        bars[f"y_empty{s}"] = 1
    return bars


# ---------------------------------------------------------------- dK/dV kernel
#
# One block owns a 128-key tile; Q_i and dO_i stream through rings X and Y.
# Per query tile i: S^T_i = K Q_i^T and dP^T_i = V dO_i^T into TMEM; each
# warpgroup w turns its columns of dP^T into P^T (first half, packed bf16)
# and dS^T (second half); dV += P^T dO_i, dK += dS^T Q_i.

def dkdv_roles(n, SX, SY, NG, mistake=None):
    two_dp = mistake == "dp2_single_ready"
    W = range(NG)

    def dpa(i, w):
        return f"dPa{i & 1 if two_dp else 0}.{w}"

    def dpb(i, w):
        return f"dPb{i & 1 if two_dp else 0}.{w}"

    def dp_bar(i):
        return (f"dp_full{i & 1}", i >> 1) if two_dp else ("dp_full0", i)

    def s_mma(i):
        return ("mma", [("K", "K"), (f"X{i % SX}", f"Q{i}")], [(f"S.{w}", f"S{i}") for w in W])

    def dp_mma(i):
        return ("mma", [("V", "V"), (f"Y{i % SY}", f"dO{i}")],
                [(dpa(i, w), f"dP{i}") for w in W] + [(dpb(i, w), f"dP{i}") for w in W])

    def mma():
        yield ("wait", "res_full", 0)
        yield ("wait", "x_full0", 0)
        yield ("wait", "y_full0", 0)
        yield s_mma(0)
        yield ("commit", "s_full", 0)
        yield dp_mma(0)
        yield ("commit", *dp_bar(0))
        for i in range(n):
            more = i + 1 < n
            if more:
                yield ("wait", f"x_full{(i + 1) % SX}", (i + 1) // SX)
                if mistake != "no_s_free_wait":
                    yield ("wait", "s_free", i)
                yield s_mma(i + 1)
                yield ("commit", "s_full", i + 1)
                if two_dp:
                    yield ("wait", f"y_full{(i + 1) % SY}", (i + 1) // SY)
                    yield dp_mma(i + 1)
                    yield ("commit", *dp_bar(i + 1))
            yield ("wait", "p_ready", i)
            yield ("mma", [(dpa(i, w), f"P{i}") for w in W] + [(f"Y{i % SY}", f"dO{i}")] +
                   ([("dV", f"dV{i - 1}")] if i else []), [("dV", f"dV{i}")])
            yield ("commit", f"y_empty{i % SY}", i // SY)
            yield ("wait", "ds_ready", i)
            yield ("mma", [(dpb(i, w), f"dS{i}") for w in W] + [(f"X{i % SX}", f"Q{i}")] +
                   ([("dK", f"dK{i - 1}")] if i else []), [("dK", f"dK{i}")])
            yield ("commit", f"x_empty{i % SX}", i // SX)
            if more and not two_dp:
                yield ("wait", f"y_full{(i + 1) % SY}", (i + 1) // SY)
                yield dp_mma(i + 1)
                yield ("commit", *dp_bar(i + 1))
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(w):
        for i in range(n):
            yield ("wait", "s_full", i)
            yield ("use", f"S.{w}", f"S{i}")
            yield ("arrive", "s_free", i)
            yield ("wait", *dp_bar(i))
            yield ("use", dpa(i, w), f"dP{i}")
            if mistake == "p_ready_before_write":
                yield ("arrive", "p_ready", i)
                yield ("write", dpa(i, w), f"P{i}")
            else:
                yield ("write", dpa(i, w), f"P{i}")
                yield ("arrive", "p_ready", i)
            yield ("use", dpb(i, w), f"dP{i}")
            yield ("write", dpb(i, w), f"dS{i}")
            yield ("arrive", "ds_ready", i)
        yield ("wait", "drain", 0)
        acc = "dV" if w < max(NG // 2, 1) else "dK"
        yield ("use", acc, f"{acc}{n - 1}")

    bars = _ring_barriers(SX, SY)
    bars.update({"dp_full0": 1, "dp_full1": 1, "s_free": NG, "p_ready": NG, "ds_ready": NG})
    roles = {"loadQ": _ring_producer(n, SX, "x_full", "x_empty", "X", "Q", (("K", "K"), ("V", "V"))),
             "loadDO": _ring_producer(n, SY, "y_full", "y_empty", "Y", "dO"),
             "mma": mma()}
    roles.update({f"sigma{w}": sigma(w) for w in W})
    return bars, roles


# ---------------------------------------------------------------- dQ kernel
#
# One block owns a 128-query tile; K_j and V_j stream through rings X and Y.
# Per key tile j: S_j = Q K_j^T into one TMEM buffer, dP_j = dO V_j^T into
# buffer j % 2; each warpgroup writes dS_j (packed bf16) over its dP_j
# columns; dQ += dS_j K_j.

def dq_roles(n, SX, SY, NG, mistake=None):
    W = range(NG)

    def s_mma(j):
        return ("mma", [("Q", "Q"), (f"X{j % SX}", f"K{j}")], [(f"S.{w}", f"S{j}") for w in W])

    def dp_mma(j):
        return ("mma", [("dO", "dO"), (f"Y{j % SY}", f"V{j}")], [(f"dP{j & 1}.{w}", f"dP{j}") for w in W])

    def mma():
        yield ("wait", "res_full", 0)
        yield ("wait", "x_full0", 0)
        yield ("wait", "y_full0", 0)
        yield s_mma(0)
        yield ("commit", "s_full", 0)
        yield dp_mma(0)
        yield ("commit", "dp_full0", 0)
        yield ("commit", "y_empty0", 0)
        for j in range(n):
            if j + 1 < n:
                yield ("wait", f"x_full{(j + 1) % SX}", (j + 1) // SX)
                if mistake != "no_s_free_wait":
                    yield ("wait", "s_free", j)
                yield s_mma(j + 1)
                yield ("commit", "s_full", j + 1)
                yield ("wait", f"y_full{(j + 1) % SY}", (j + 1) // SY)
                yield dp_mma(j + 1)
                yield ("commit", f"dp_full{(j + 1) & 1}", (j + 1) >> 1)
                yield ("commit", f"y_empty{(j + 1) % SY}", (j + 1) // SY)
            yield ("wait", f"ds_ready{j & 1}", j >> 1)
            yield ("mma", [(f"dP{j & 1}.{w}", f"dS{j}") for w in W] + [(f"X{j % SX}", f"K{j}")] +
                   ([("dQ", f"dQ{j - 1}")] if j else []), [("dQ", f"dQ{j}")])
            yield ("commit", f"x_empty{j % SX}", j // SX)
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(w):
        for j in range(n):
            yield ("wait", "s_full", j)
            yield ("use", f"S.{w}", f"S{j}")
            yield ("arrive", "s_free", j)
            yield ("wait", f"dp_full{j & 1}", j >> 1)
            yield ("use", f"dP{j & 1}.{w}", f"dP{j}")
            yield ("write", f"dP{j & 1}.{w}", f"dS{j}")
            yield ("arrive", f"ds_ready{j & 1}", j >> 1)
        yield ("wait", "drain", 0)
        yield ("use", "dQ", f"dQ{n - 1}")

    bars = _ring_barriers(SX, SY)
    bars.update({"dp_full0": 1, "dp_full1": 1, "s_free": NG, "ds_ready0": NG, "ds_ready1": NG})
    roles = {"loadK": _ring_producer(n, SX, "x_full", "x_empty", "X", "K", (("Q", "Q"), ("dO", "dO"))),
             "loadV": _ring_producer(n, SY, "y_full", "y_empty", "Y", "V"),
             "mma": mma()}
    roles.update({f"sigma{w}": sigma(w) for w in W})
    return bars, roles


# ring depths (X, Y) and sigma warpgroups of the two head dimensions
SHAPES = [pytest.param(3, 2, 2, id="D128"), pytest.param(4, 4, 4, id="D64")]
TILES = [1, 2, 3, 5, 8]
SEEDS = 150


def _explore(make, seeds=SEEDS):
    for seed in range(seeds):
        bars, roles = make()
        Model(bars, roles, seed).run()


def _errors(make, seeds=1500):
    """The distinct errors that `seeds` runs of a (mistaken) protocol raise."""
    found = []
    for seed in range(seeds):
        bars, roles = make()
        try:
            Model(bars, roles, seed).run()
        except ProtocolError as e:
            found.append(str(e))
    return found


@pytest.mark.parametrize("n", TILES)
@pytest.mark.parametrize("SX,SY,NG", SHAPES)
def test_dkdv_protocol(n, SX, SY, NG):
    _explore(lambda: dkdv_roles(n, SX, SY, NG))


@pytest.mark.parametrize("n", TILES)
@pytest.mark.parametrize("SX,SY,NG", SHAPES)
def test_dq_protocol(n, SX, SY, NG):
    _explore(lambda: dq_roles(n, SX, SY, NG))


@pytest.mark.parametrize("NG", [1, 2])
def test_two_dp_buffers_with_one_readiness_barrier_are_caught(NG):
    errs = _errors(lambda: dkdv_roles(5, 4, 4, NG, mistake="dp2_single_ready"))
    # the MMA thread finds p_ready two phases ahead of the one it waits for
    assert any(re.search(r"mma waits for phase \d+ of p_ready, which has completed", e) for e in errs)


@pytest.mark.parametrize("roles", [dkdv_roles, dq_roles])
def test_s_overwritten_before_read_is_caught(roles):
    errs = _errors(lambda: roles(4, 3, 2, 2, mistake="no_s_free_wait"))
    assert any(re.search(r"sigma\d reads S\.\d expecting S\d, finds S\d", e) for e in errs)


def test_early_p_ready_arrival_is_caught():
    errs = _errors(lambda: dkdv_roles(3, 3, 2, 2, mistake="p_ready_before_write"))
    assert any(re.search(r"an MMA reads dPa0\.\d expecting P\d, finds dP\d", e) for e in errs)


# ---------------------------------------------------------------- persistent forms
#
# One block per SM walks a list of items (tiles with work); an item of n units
# is one tile's loop above.  The units of all the block's items form one
# stream: ring slots and hand-off phases run on across items, the resident
# tiles (dQ: Q, dO; dK/dV: K, V) of consecutive items alternate between NR
# shared-memory slots (res_full / res_empty), and the MMA thread commits
# acc_full after an item's last unit, after which the warpgroups read the
# item's accumulators.  The next item's first accumulating MMA overwrites
# them only after every warpgroup's next readiness arrival, which comes after
# those reads.

def _units(items):
    return [(k, j) for k, n in enumerate(items) for j in range(n)]


def _persistent_producer(items, S, full, empty, ring, tile, NR=None, mistake=None):
    def g():
        q = 0
        for k, n in enumerate(items):
            if NR is not None:
                rs = k % NR
                if k >= NR and mistake != "no_res_empty_wait":
                    yield ("wait", f"res_empty{rs}", k // NR - 1)
                yield ("tma", f"res_full{rs}", k // NR, f"Res{rs}", f"R{k}")
            for j in range(n):
                if q >= S:
                    yield ("wait", f"{empty}{q % S}", q // S - 1)
                yield ("tma", f"{full}{q % S}", q // S, f"{ring}{q % S}", f"{tile}{k}.{j}")
                q += 1
        if NR is not None:
            for k in range(max(len(items) - NR, 0), len(items)):
                yield ("wait", f"res_full{k % NR}", k // NR)
        for qq in range(max(q - S, 0), q):
            yield ("wait", f"{full}{qq % S}", qq // S)
    return g()


def _persistent_barriers(SX, SY, NR):
    bars = _ring_barriers(SX, SY)
    del bars["res_full"]
    bars["acc_full"] = 1
    for r in range(NR):
        bars[f"res_full{r}"] = 1
        bars[f"res_empty{r}"] = 1
    return bars


def dq_persistent_roles(items, SX, SY, NG, NR=2, mistake=None):
    W = range(NG)
    units = _units(items)
    U = len(units)

    def s_mma(u):
        k, j = units[u]
        return ("mma", [(f"Res{k % NR}", f"R{k}"), (f"X{u % SX}", f"K{k}.{j}")],
                [(f"S.{w}", f"S{u}") for w in W])

    def dp_mma(u):
        k, j = units[u]
        return ("mma", [(f"Res{k % NR}", f"R{k}"), (f"Y{u % SY}", f"V{k}.{j}")],
                [(f"dP{u & 1}.{w}", f"dP{u}") for w in W])

    def mma():
        yield ("wait", "res_full0", 0)
        yield ("wait", "x_full0", 0)
        yield ("wait", "y_full0", 0)
        yield s_mma(0)
        yield ("commit", "s_full", 0)
        yield dp_mma(0)
        yield ("commit", "dp_full0", 0)
        yield ("commit", "y_empty0", 0)
        for u in range(U):
            k, j = units[u]
            if u + 1 < U:
                k2, j2 = units[u + 1]
                if j2 == 0:
                    yield ("wait", f"res_full{k2 % NR}", k2 // NR)
                yield ("wait", f"x_full{(u + 1) % SX}", (u + 1) // SX)
                yield ("wait", "s_free", u)
                yield s_mma(u + 1)
                yield ("commit", "s_full", u + 1)
                yield ("wait", f"y_full{(u + 1) % SY}", (u + 1) // SY)
                yield dp_mma(u + 1)
                yield ("commit", f"dp_full{(u + 1) & 1}", (u + 1) >> 1)
                yield ("commit", f"y_empty{(u + 1) % SY}", (u + 1) // SY)
            yield ("wait", f"ds_ready{u & 1}", u >> 1)
            yield ("mma", [(f"dP{u & 1}.{w}", f"dS{u}") for w in W] + [(f"X{u % SX}", f"K{k}.{j}")] +
                   ([("dQ", f"dQ{k}.{j - 1}")] if j else []), [("dQ", f"dQ{k}.{j}")])
            yield ("commit", f"x_empty{u % SX}", u // SX)
            if j == items[k] - 1:
                yield ("commit", f"res_empty{k % NR}", k // NR)
                yield ("commit", "acc_full", k)
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(w):
        for u in range(U):
            k, j = units[u]
            yield ("wait", "s_full", u)
            yield ("use", f"S.{w}", f"S{u}")
            yield ("arrive", "s_free", u)
            yield ("wait", f"dp_full{u & 1}", u >> 1)
            yield ("use", f"dP{u & 1}.{w}", f"dP{u}")
            yield ("write", f"dP{u & 1}.{w}", f"dS{u}")
            yield ("arrive", f"ds_ready{u & 1}", u >> 1)
            if j == items[k] - 1:
                yield ("wait", "acc_full", k)
                yield ("use", "dQ", f"dQ{k}.{j}")

    bars = _persistent_barriers(SX, SY, NR)
    bars.update({"dp_full0": 1, "dp_full1": 1, "s_free": NG, "ds_ready0": NG, "ds_ready1": NG})
    roles = {"loadK": _persistent_producer(items, SX, "x_full", "x_empty", "X", "K", NR, mistake),
             "loadV": _persistent_producer(items, SY, "y_full", "y_empty", "Y", "V"),
             "mma": mma()}
    roles.update({f"sigma{w}": sigma(w) for w in W})
    return bars, roles


def dkdv_persistent_roles(items, SX, SY, NG, NR=2, mistake=None):
    W = range(NG)
    units = _units(items)
    U = len(units)

    def s_mma(u):
        k, i = units[u]
        return ("mma", [(f"Res{k % NR}", f"R{k}"), (f"X{u % SX}", f"Q{k}.{i}")],
                [(f"S.{w}", f"S{u}") for w in W])

    def dp_mma(u):
        k, i = units[u]
        return ("mma", [(f"Res{k % NR}", f"R{k}"), (f"Y{u % SY}", f"dO{k}.{i}")],
                [(f"dPa.{w}", f"dP{u}") for w in W] + [(f"dPb.{w}", f"dP{u}") for w in W])

    def mma():
        yield ("wait", "res_full0", 0)
        yield ("wait", "x_full0", 0)
        yield ("wait", "y_full0", 0)
        yield s_mma(0)
        yield ("commit", "s_full", 0)
        yield dp_mma(0)
        yield ("commit", "dp_full", 0)
        for u in range(U):
            k, i = units[u]
            more = u + 1 < U
            if more:
                k2, i2 = units[u + 1]
                if i2 == 0:
                    yield ("wait", f"res_full{k2 % NR}", k2 // NR)
                yield ("wait", f"x_full{(u + 1) % SX}", (u + 1) // SX)
                yield ("wait", "s_free", u)
                yield s_mma(u + 1)
                yield ("commit", "s_full", u + 1)
            yield ("wait", "p_ready", u)
            yield ("mma", [(f"dPa.{w}", f"P{u}") for w in W] + [(f"Y{u % SY}", f"dO{k}.{i}")] +
                   ([("dV", f"dV{k}.{i - 1}")] if i else []), [("dV", f"dV{k}.{i}")])
            yield ("commit", f"y_empty{u % SY}", u // SY)
            yield ("wait", "ds_ready", u)
            yield ("mma", [(f"dPb.{w}", f"dS{u}") for w in W] + [(f"X{u % SX}", f"Q{k}.{i}")] +
                   ([("dK", f"dK{k}.{i - 1}")] if i else []), [("dK", f"dK{k}.{i}")])
            yield ("commit", f"x_empty{u % SX}", u // SX)
            if i == items[k] - 1:
                yield ("commit", f"res_empty{k % NR}", k // NR)
                yield ("commit", "acc_full", k)
            if more:
                yield ("wait", f"y_full{(u + 1) % SY}", (u + 1) // SY)
                yield dp_mma(u + 1)
                yield ("commit", "dp_full", u + 1)
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(w):
        acc = "dV" if w < max(NG // 2, 1) else "dK"
        for u in range(U):
            k, i = units[u]
            yield ("wait", "s_full", u)
            yield ("use", f"S.{w}", f"S{u}")
            yield ("arrive", "s_free", u)
            yield ("wait", "dp_full", u)
            yield ("use", f"dPa.{w}", f"dP{u}")
            yield ("write", f"dPa.{w}", f"P{u}")
            yield ("arrive", "p_ready", u)
            yield ("use", f"dPb.{w}", f"dP{u}")
            yield ("write", f"dPb.{w}", f"dS{u}")
            yield ("arrive", "ds_ready", u)
            if i == items[k] - 1:
                yield ("wait", "acc_full", k)
                yield ("use", acc, f"{acc}{k}.{i}")

    bars = _persistent_barriers(SX, SY, NR)
    bars.update({"dp_full": 1, "s_free": NG, "p_ready": NG, "ds_ready": NG})
    roles = {"loadQ": _persistent_producer(items, SX, "x_full", "x_empty", "X", "Q", NR, mistake),
             "loadDO": _persistent_producer(items, SY, "y_full", "y_empty", "Y", "dO"),
             "mma": mma()}
    roles.update({f"sigma{w}": sigma(w) for w in W})
    return bars, roles


ITEM_LISTS = [[1], [3], [1, 1, 1], [3, 1, 2], [1, 4, 1, 1, 2], [5, 5], [2, 1, 1, 1, 1, 3]]


@pytest.mark.parametrize("items", ITEM_LISTS, ids=lambda it: "-".join(map(str, it)))
@pytest.mark.parametrize("SX,SY,NG", SHAPES)
def test_dq_persistent_protocol(items, SX, SY, NG):
    _explore(lambda: dq_persistent_roles(items, SX, SY, NG), 100)


@pytest.mark.parametrize("items", ITEM_LISTS, ids=lambda it: "-".join(map(str, it)))
@pytest.mark.parametrize("SX,SY,NG", SHAPES)
def test_dkdv_persistent_protocol(items, SX, SY, NG):
    _explore(lambda: dkdv_persistent_roles(items, SX, SY, NG), 100)


@pytest.mark.parametrize("roles", [dq_persistent_roles, dkdv_persistent_roles])
def test_resident_slot_reused_too_early_is_caught(roles):
    errs = _errors(lambda: roles([1, 1, 1, 2], 4, 4, 4, mistake="no_res_empty_wait"), 800)
    assert any(re.search(r"reads Res\d expecting R\d, finds R\d", e) for e in errs)


# ---------------------------------------------------------------- persistent forward
#
# fwd_persist_sm100.cuh: items of one or two 128-row query tiles; units
# u = (item, key tile j, query tile t), t fastest.  Unit u's scores go to TMEM
# buffer u % NB; each warpgroup (t, c) evaluates half c of its tile's scores
# and writes P over them; O_t += P V_j reads P from the buffer, and the MMA
# thread issues the scores of unit u + NB right after it (same buffer).  Each
# buffer has one scores-ready barrier per query tile; p_full[buffer] collects
# the two warpgroups of the unit's tile; o_full[t] completes once per item that
# has tile t, after which tile t's warpgroups read O_t.

def fwd_persistent_roles(items, NB=3, NQ=2, KS=4, VS=4, mistake=None):
    """items: (ntiles, nkv) per item of one block."""
    units = [(n, j, t) for n, (nt, nkv) in enumerate(items) for j in range(nkv) for t in range(nt)]
    U = len(units)
    one_sfull = mistake == "one_scores_barrier_per_buffer"

    def s_bar(u):
        n, j, t = units[u]
        return f"s_full{u % NB}" if one_sfull else f"s_full{u % NB}.{t}"

    def loadQK():
        jk = 0
        for n, (nt, nkv) in enumerate(items):
            qs = n % NQ
            if n >= NQ:
                yield ("wait", f"q_empty{qs}", n // NQ - 1)
            # the item's one or two query tiles land on one barrier: one load here
            yield ("tma", f"q_full{qs}", n // NQ, f"Q{qs}", f"Q{n}")
            for j in range(nkv):
                ks = jk % KS
                if jk >= KS:
                    yield ("wait", f"k_empty{ks}", jk // KS - 1)
                yield ("tma", f"k_full{ks}", jk // KS, f"K{ks}", f"K{n}.{j}")
                jk += 1
        for i in range(max(len(items) - NQ, 0), len(items)):
            yield ("wait", f"q_full{i % NQ}", i // NQ)
        for i in range(max(jk - KS, 0), jk):
            yield ("wait", f"k_full{i % KS}", i // KS)

    def loadV():
        jv = 0
        for n, (nt, nkv) in enumerate(items):
            for j in range(nkv):
                vs = jv % VS
                if jv >= VS:
                    yield ("wait", f"v_empty{vs}", jv // VS - 1)
                yield ("tma", f"v_full{vs}", jv // VS, f"V{vs}", f"V{n}.{j}")
                jv += 1
        for i in range(max(jv - VS, 0), jv):
            yield ("wait", f"v_full{i % VS}", i // VS)

    # ring indices of each unit: item n's query slot, key / value index of (n, j)
    kv_index = {}
    for n, (nt, nkv) in enumerate(items):
        for j in range(nkv):
            kv_index[(n, j)] = len(kv_index)
    uses = {}   # scores-barrier completions so far, per barrier

    def issue_s(u):
        n, j, t = units[u]
        nt, nkv = items[n]
        q = kv_index[(n, j)]
        if j == 0 and t == 0:
            yield ("wait", f"q_full{n % NQ}", n // NQ)
        if t == 0:
            yield ("wait", f"k_full{q % KS}", q // KS)
        b = u % NB
        yield ("mma", [(f"Q{n % NQ}", f"Q{n}"), (f"K{q % KS}", f"K{n}.{j}")],
               [(f"S{b}.0", f"S{u}"), (f"S{b}.1", f"S{u}")])
        bar = s_bar(u)
        yield ("commit", bar, uses.get(bar, 0))
        uses[bar] = uses.get(bar, 0) + 1
        if t == nt - 1:
            yield ("commit", f"k_empty{q % KS}", q // KS)
            if j == nkv - 1:
                yield ("commit", f"q_empty{n % NQ}", n // NQ)

    def mma():
        for u in range(min(NB, U)):
            yield from issue_s(u)
        seen_o = [0, 0]
        for u in range(U):
            n, j, t = units[u]
            nt, nkv = items[n]
            q = kv_index[(n, j)]
            if t == 0:
                yield ("wait", f"v_full{q % VS}", q // VS)
            yield ("wait", f"p_full{u % NB}", u // NB)
            b = u % NB
            yield ("mma", [(f"S{b}.0", f"P{u}"), (f"S{b}.1", f"P{u}"), (f"V{q % VS}", f"V{n}.{j}")] +
                   ([(f"O{t}", f"O{n}.{j - 1}")] if j else []), [(f"O{t}", f"O{n}.{j}")])
            if t == nt - 1:
                yield ("commit", f"v_empty{q % VS}", q // VS)
            if j == nkv - 1:
                yield ("commit", f"o_full{t}", seen_o[t])
                seen_o[t] += 1
            if u + NB < U:
                yield from issue_s(u + NB)
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(t, c):
        used = {}
        no = 0
        for u in range(U):
            n, j, tt = units[u]
            if tt != t:
                continue
            bar = s_bar(u)
            if one_sfull:
                # the first build: each tile counted its own uses of the buffer
                key = f"{u % NB}"
            else:
                key = bar
            ph = used.get(key, 0)
            used[key] = ph + 1
            yield ("wait", bar, ph)
            b = u % NB
            yield ("use", f"S{b}.{c}", f"S{u}")
            yield ("write", f"S{b}.{c}", f"P{u}")
            yield ("arrive", f"p_full{b}", u // NB)
            nt, nkv = items[n]
            if j == nkv - 1:
                yield ("wait", f"o_full{t}", no)
                no += 1
                yield ("use", f"O{t}", f"O{n}.{j}")

    bars = {"drain": 1, "o_full0": 1, "o_full1": 1}
    for s in range(NQ):
        bars[f"q_full{s}"] = 1
        bars[f"q_empty{s}"] = 1
    for s in range(KS):
        bars[f"k_full{s}"] = 1
        bars[f"k_empty{s}"] = 1
    for s in range(VS):
        bars[f"v_full{s}"] = 1
        bars[f"v_empty{s}"] = 1
    for b in range(NB):
        bars[f"p_full{b}"] = 2          # the two warpgroups of the unit's tile
        if one_sfull:
            bars[f"s_full{b}"] = 1
        else:
            bars[f"s_full{b}.0"] = 1
            bars[f"s_full{b}.1"] = 1
    roles = {"loadQK": loadQK(), "loadV": loadV(), "mma": mma()}
    roles.update({f"sigma{t}{c}": sigma(t, c) for t in range(2) for c in range(2)})
    return bars, roles


FWD_ITEMS = [[(2, 3)], [(1, 2)], [(2, 1), (1, 1), (2, 2)], [(1, 3), (2, 2), (1, 1), (1, 2)],
             [(2, 4), (2, 1), (1, 3)], [(1, 1)] * 5]


@pytest.mark.parametrize("items", FWD_ITEMS, ids=lambda it: "-".join(f"{a}x{b}" for a, b in it))
@pytest.mark.parametrize("NB", [2, 3])
def test_fwd_persistent_protocol(items, NB):
    _explore(lambda: fwd_persistent_roles(items, NB=NB), 150)


def test_fwd_one_scores_barrier_per_buffer_is_caught():
    """The persistent forward's first build kept one scores-ready barrier per
    TMEM buffer: with one- and two-tile items mixed, a tile that sits out some
    units waits on a phase the other tile has already moved past."""
    errs = _errors(lambda: fwd_persistent_roles([(2, 2), (1, 2), (2, 1), (1, 1)],
                                                mistake="one_scores_barrier_per_buffer"), 800)
    assert any(re.search(r"sigma\d\d waits for phase \d+ of s_full\d, which has completed|"
                         r"reads S\d\.\d expecting S\d+, finds|deadlock", e) for e in errs)


# ---------------------------------------------------------------- tile forward (D = 128)
#
# fwd_sm100.cuh: one block per pair of query tiles.  S_t (scores of tile t)
# lives in its own TMEM buffer; per key tile j the MMA thread issues
# O_t += P_t V_j as tile t's warpgroups publish P_t (p_full[t]) and then S_t
# of key tile j + 1 into the same buffer (MMAs run in issue order).

def fwd_tiles_roles(ntiles, nkv, KS=2, VS=3, mistake=None):
    def loadQK():
        yield ("tma", "q_full", 0, "Q", "Q")
        for j in range(nkv):
            if j >= KS:
                yield ("wait", f"k_empty{j % KS}", j // KS - 1)
            yield ("tma", f"k_full{j % KS}", j // KS, f"K{j % KS}", f"K{j}")
        yield ("wait", "q_full", 0)
        for j in range(max(nkv - KS, 0), nkv):
            yield ("wait", f"k_full{j % KS}", j // KS)

    def loadV():
        for j in range(nkv):
            if j >= VS:
                yield ("wait", f"v_empty{j % VS}", j // VS - 1)
            yield ("tma", f"v_full{j % VS}", j // VS, f"V{j % VS}", f"V{j}")
        for j in range(max(nkv - VS, 0), nkv):
            yield ("wait", f"v_full{j % VS}", j // VS)

    def issue_s(t, j):
        yield ("mma", [("Q", "Q"), (f"K{j % KS}", f"K{j}")], [(f"S{t}.0", f"S{t}:{j}"), (f"S{t}.1", f"S{t}:{j}")])
        yield ("commit", f"s_full{t}", j)

    def mma():
        yield ("wait", "q_full", 0)
        yield ("wait", "k_full0", 0)
        for t in range(ntiles):
            yield from issue_s(t, 0)
        yield ("commit", "k_empty0", 0)
        for j in range(nkv):
            more = j + 1 < nkv
            yield ("wait", f"v_full{j % VS}", j // VS)
            for t in range(ntiles):
                if mistake != "no_p_wait":
                    yield ("wait", f"p_full{t}", j)
                yield ("mma", [(f"S{t}.0", f"P{t}:{j}"), (f"S{t}.1", f"P{t}:{j}"), (f"V{j % VS}", f"V{j}")] +
                       ([(f"O{t}", f"O{t}:{j - 1}")] if j else []), [(f"O{t}", f"O{t}:{j}")])
                if t == ntiles - 1:
                    yield ("commit", f"v_empty{j % VS}", j // VS)
                if more:
                    if t == 0:
                        yield ("wait", f"k_full{(j + 1) % KS}", (j + 1) // KS)
                    yield from issue_s(t, j + 1)
                    if t == ntiles - 1:
                        yield ("commit", f"k_empty{(j + 1) % KS}", (j + 1) // KS)
        yield ("commit", "drain", 0)
        yield ("wait", "drain", 0)

    def sigma(t, c):
        if t >= ntiles:
            return
        for j in range(nkv):
            yield ("wait", f"s_full{t}", j)
            yield ("use", f"S{t}.{c}", f"S{t}:{j}")
            yield ("write", f"S{t}.{c}", f"P{t}:{j}")
            yield ("arrive", f"p_full{t}", j)
        yield ("wait", "drain", 0)
        yield ("use", f"O{t}", f"O{t}:{nkv - 1}")

    bars = {"q_full": 1, "drain": 1, "s_full0": 1, "s_full1": 1, "p_full0": 2, "p_full1": 2}
    for s in range(KS):
        bars[f"k_full{s}"] = 1
        bars[f"k_empty{s}"] = 1
    for s in range(VS):
        bars[f"v_full{s}"] = 1
        bars[f"v_empty{s}"] = 1
    roles = {"loadQK": loadQK(), "loadV": loadV(), "mma": mma()}
    roles.update({f"sigma{t}{c}": sigma(t, c) for t in range(2) for c in range(2)})
    return bars, roles


@pytest.mark.parametrize("ntiles", [1, 2])
@pytest.mark.parametrize("nkv", [1, 2, 3, 6])
def test_fwd_tiles_protocol(ntiles, nkv):
    _explore(lambda: fwd_tiles_roles(ntiles, nkv), 150)


def test_fwd_tiles_missing_p_wait_is_caught():
    errs = _errors(lambda: fwd_tiles_roles(2, 3, mistake="no_p_wait"), 800)
    assert any(re.search(r"an MMA reads S\d\.\d expecting P\d:\d, finds S\d:\d", e) for e in errs)
