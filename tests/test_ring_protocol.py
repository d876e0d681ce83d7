"""A model of the fused GEMM's barrier protocol, checked under random schedules (CPU only).

The kernel hands stages between its warp roles through rings of shared-memory or tensor-memory slots guarded by
mbarriers, and every waiter derives the phase parity it waits for from its own running count of the ring's uses.
That is sound only under the ring-depth relations the kernel asserts at compile time (Q ring >= A ring + groups,
groups <= A ring).  This test models the protocol -- barrier phases and parity waits exactly as the hardware
defines them, every warp role (the four warps of a dequantizer group run independently), and the asynchronous
landing of copies and completion of MMAs at random times -- and runs it under random schedules:

  * with the depths the kernel uses -- read from the kernel's own configuration for every dequantizing
    instantiation (tests/ring_depths.cu, built for the host) -- every consumer must read the stage it expects,
    the MMAs' operands must stay intact until their completion is signalled, and the schedule must never
    deadlock;
  * with a planted violation (more dequantizer groups than A slots, a configuration that once hung its waits
    on the GPU) some schedule must break one of those properties.
"""

import os
import random
import shutil
import subprocess
from dataclasses import dataclass, field

import pytest


class Barrier:
    """An mbarrier: a phase completes when all expected arrivals (and transaction bytes) have come in."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0  # number of completed phases

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier expects in one phase"
        self._maybe_complete()

    def expect_tx(self, nbytes):
        self.tx += nbytes

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def try_wait(self, parity):
        # true once the phase with this parity has completed: the current phase's parity differs
        return (self.completed & 1) != parity


@dataclass
class Cfg:
    QS: int
    AS: int
    BS: int
    G: int
    units: list  # (n_extra, n_main) per unit of this CTA
    acc_bufs: int = 2


@dataclass
class World:
    cfg: Cfg
    rng: random.Random
    q_full: list = field(default_factory=list)
    q_empty: list = field(default_factory=list)
    a_full: list = field(default_factory=list)
    a_empty: list = field(default_factory=list)
    b_full: list = field(default_factory=list)
    b_empty: list = field(default_factory=list)
    t_full: list = field(default_factory=list)
    t_empty: list = field(default_factory=list)
    q_slot: list = field(default_factory=list)   # stage tag held by each slot
    a_slot: list = field(default_factory=list)   # per slot: tag written by each of the 4 warp quarters
    b_slot: list = field(default_factory=list)
    events: list = field(default_factory=list)   # pending asynchronous completions: (callable)
    errors: list = field(default_factory=list)


def make_world(cfg, seed):
    w = World(cfg, random.Random(seed))
    w.q_full = [Barrier(1) for _ in range(cfg.QS)]
    w.q_empty = [Barrier(4) for _ in range(cfg.QS)]  # the consuming group's warps (each lane's arrival folded in)
    w.a_full = [Barrier(4) for _ in range(cfg.AS)]
    w.a_empty = [Barrier(1) for _ in range(cfg.AS)]
    w.b_full = [Barrier(1) for _ in range(cfg.BS)]
    w.b_empty = [Barrier(1) for _ in range(cfg.BS)]
    w.t_full = [Barrier(1) for _ in range(cfg.acc_bufs)]
    w.t_empty = [Barrier(4) for _ in range(cfg.acc_bufs)]
    w.q_slot = [None] * cfg.QS
    w.a_slot = [[None] * 4 for _ in range(cfg.AS)]
    w.b_slot = [None] * cfg.BS
    return w


def stages(cfg):
    """(global stage g, main index q or None, unit index, index within the unit) in issue order: a unit's main
    stages, then its extra (LoRA) stages, as the kernel issues them."""
    out, g, q = [], 0, 0
    for ui, (ne, nm) in enumerate(cfg.units):
        for it in range(ne + nm):
            main = it < nm
            out.append((g, q if main else None, ui, it))
            g += 1
            if main:
                q += 1
    return out


def wait(bar, parity):
    """Coroutine step: block until the parity wait succeeds."""
    while not bar.try_wait(parity):
        yield


def q_producer(w):
    c = w.cfg
    for g, q, _, _ in stages(c):
        if q is None:
            continue
        s = q % c.QS
        yield from wait(w.q_empty[s], ((q // c.QS) & 1) ^ 1)
        w.q_full[s].expect_tx(1)       # arrive.expect_tx: the bytes are expected first, then the arrival
        w.q_full[s].arrive()

        def land(s=s, q=q):
            w.q_slot[s] = q
            w.q_full[s].complete_tx(1)
        w.events.append(land)


def b_producer(w):
    c = w.cfg
    for g, _, _, _ in stages(c):
        s = g % c.BS
        yield from wait(w.b_empty[s], ((g // c.BS) & 1) ^ 1)
        w.b_full[s].expect_tx(1)
        w.b_full[s].arrive()

        def land(s=s, g=g):
            w.b_slot[s] = g
            w.b_full[s].complete_tx(1)
        w.events.append(land)


def dequant_warp(w, grp, quarter):
    c = w.cfg
    for g, q, _, _ in stages(c):
        if g % c.G != grp:
            continue
        if q is not None:
            qs = q % c.QS
            yield from wait(w.q_full[qs], (q // c.QS) & 1)
            if w.q_slot[qs] != q:
                w.errors.append(f"dequantizer read Q slot {qs} holding stage {w.q_slot[qs]}, expected {q}")
            w.q_empty[qs].arrive()
        s = g % c.AS
        yield from wait(w.a_empty[s], ((g // c.AS) & 1) ^ 1)
        w.a_slot[s][quarter] = g
        w.a_full[s].arrive()
        yield


def mma(w):
    c = w.cfg
    g = 0
    for lu, (ne, nm) in enumerate(c.units):
        acc = lu % c.acc_bufs
        yield from wait(w.t_empty[acc], ((lu // c.acc_bufs) & 1) ^ 1)
        for _ in range(ne + nm):
            a, b = g % c.AS, g % c.BS
            yield from wait(w.a_full[a], (g // c.AS) & 1)
            yield from wait(w.b_full[b], (g // c.BS) & 1)

            def check(where, a=a, b=b, g=g):
                if any(t != g for t in w.a_slot[a]) or w.b_slot[b] != g:
                    w.errors.append(f"MMA {where} of stage {g}: A slot {w.a_slot[a]}, B slot {w.b_slot[b]}")
            check("issue")

            def complete(a=a, b=b, check=check):
                check("completion")  # operands must still be intact when the MMAs finish reading them
                w.a_empty[a].arrive()
                w.b_empty[b].arrive()
            w.events.append(complete)
            g += 1
            yield

        def unit_done(acc=acc):
            w.t_full[acc].arrive()
        w.events.append(unit_done)


def epilogue_warp(w):
    c = w.cfg
    for lu in range(len(c.units)):
        acc = lu % c.acc_bufs
        yield from wait(w.t_full[acc], (lu // c.acc_bufs) & 1)
        yield
        w.t_empty[acc].arrive()


def run(cfg, seed, max_steps=200000):
    w = make_world(cfg, seed)
    roles = [q_producer(w), b_producer(w), mma(w)]
    roles += [dequant_warp(w, grp, qd) for grp in range(cfg.G) for qd in range(4)]
    roles += [epilogue_warp(w) for _ in range(4)]
    live = list(roles)
    # MMA completions are in issue order; copies may land in any order
    for _ in range(max_steps):
        if w.errors:
            return w.errors
        if not live and not w.events:
            return []
        choices = len(live) + (1 if w.events else 0)
        k = w.rng.randrange(choices)
        if k == len(live):
            # deliver the oldest pending MMA completion, or a random pending copy landing
            i = w.rng.randrange(len(w.events))
            if w.events[i].__name__ in ("complete", "unit_done"):
                # MMA completions (and the commits that signal them) come in issue order
                i = next(j for j, e in enumerate(w.events) if e.__name__ in ("complete", "unit_done"))
            w.events.pop(i)()
            continue
        role = live[k]
        try:
            next(role)
        except StopIteration:
            live.remove(role)
    # a schedule that cannot finish within the bound is a deadlock
    return w.errors or ["deadlock: no progress within the step bound"]


UNITS = [(1, 16), (0, 16), (1, 9), (0, 5), (1, 1), (0, 12)]


@pytest.mark.parametrize("QS,AS,BS,G", [
    (14, 8, 4, 4),   # forward at BN = 256
    (16, 8, 8, 4),   # token-light forward, one-block stages
    (7, 3, 8, 3),    # token-light forward, four-block stages
    (10, 3, 3, 3),   # dX at BN = 256
])
def test_kernel_depths_are_safe_under_random_schedules(QS, AS, BS, G):
    assert QS >= AS + G and G <= AS  # the kernel's compile-time relations
    cfg = Cfg(QS, AS, BS, G, UNITS)
    for seed in range(60):
        errs = run(cfg, seed)
        assert not errs, (seed, errs[:3])


@pytest.mark.parametrize("QS,AS,G", [(14, 4, 5),   # more groups than A slots (an earlier build's configuration)
                                     (7, 4, 4),    # Q ring one short of A ring + groups
                                     (11, 8, 4),
                                     (5, 3, 3)])
def test_violated_relations_are_caught(QS, AS, G):
    """Each relation is needed, and the Q-ring bound is tight: one slot fewer fails some schedule."""
    cfg = Cfg(QS=QS, AS=AS, BS=max(AS, 4), G=G, units=UNITS)
    assert sum(1 for seed in range(150) if run(cfg, seed)) > 0


@pytest.mark.parametrize("QS,AS,G", [(8, 4, 4), (12, 8, 4), (6, 3, 3)])
def test_relations_at_their_boundary_hold(QS, AS, G):
    cfg = Cfg(QS=QS, AS=AS, BS=max(AS, 4), G=G, units=UNITS)
    for seed in range(100):
        errs = run(cfg, seed)
        assert not errs, (seed, errs[:3])


def kernel_depths(tmpdir):
    """(BN, AM, KB, QS, AS, BS, G, acc_bufs) of every dequantizing instantiation, from the kernel's own
    configuration (tests/ring_depths.cu, built for the host with nvcc)."""
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = os.path.join(tmpdir, "ring_depths")
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "ring_depths.cu")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "--expt-relaxed-constexpr",
                    "-o", exe, src], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return [tuple(int(v) for v in line.split()) for line in out.strip().splitlines()]


def test_every_instantiation_is_safe_under_random_schedules(tmp_path):
    """The model with the depths each dequantizing kernel instantiation actually uses (not a copy of them)."""
    rows = kernel_depths(str(tmp_path))
    assert len(rows) == 20
    for BN, AM, KB, QS, AS, BS, G, acc in sorted({r for r in rows}):
        assert QS >= AS + G and G <= AS, (BN, AM, KB)
        cfg = Cfg(QS, AS, BS, G, UNITS, acc_bufs=acc)
        for seed in range(12):
            errs = run(cfg, 1000 + seed)
            assert not errs, ((BN, AM, KB), seed, errs[:3])
