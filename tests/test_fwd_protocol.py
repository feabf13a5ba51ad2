"""A model of the prefill kernel's hand-off protocol at d = 128 (csrc/attn_fwd.cu: two query tiles per
CTA, P written over S, a 4-stage K/V ring, units handed out through a 4-slot ring), one persistent CTA
walking a list of units, run under random timings on the CPU (tests/protocol_sim.py).

The roles follow the kernel's order of waits, arrivals, commits and accesses: the producer (unit
claims, the Q tiles of a unit, K_j and V_j through the ring), the MMA issuer (QK(0,0) QK(1,0) |
PV(0,j) QK(0,j+1) PV(1,j) QK(1,j+1) | ..., a causal unit's first tile ending a K/V tile early with its
O released right after its last PV), and one softmax warpgroup per query tile (S read out, O rescaled
in tensor memory on some tiles, P written over S, O read out after the unit's last product of that
tile). Units mix causal shapes (the first tile one K/V tile short), non-causal ones, first tiles
without keys and units without any key. The checks are those of the simulator: versions read as
expected, no write under a read, no parity aliasing, no role left waiting.
"""
import random

import pytest

from protocol_sim import Hazard, Sim

STAGES, SCHED = 4, 4
ROLES = {"producer", "mma", "softmax0", "softmax1"}


def forward_cta(sim, units, early_q_release=False, no_final_wait=False, phase_for_keyless_tile=False,
                sep_p=False, no_p_free_wait=False):
    """units: (n, n0) per unit: K/V tiles of the unit and of its first query tile. sep_p: the d <= 64
    variant, P in tensor-memory buffers of its own, the next S computed while the softmax works on
    the current one (s_free: S read out; p_free: the PV reading the P buffer is done).

    The other arguments plant mistakes (for the tests that show the model catches them): Q released
    after the unit's first QK instead of its last; the second tile's O read out without waiting for
    the unit's last product; an o_final phase committed (and waited for) also for a first tile
    without keys, whose warpgroup then takes no part in the unit; and (sep_p) P written into its
    buffer without waiting for the previous PV that reads it."""
    sim.bar("q_full")
    sim.bar("q_empty")
    for s in range(STAGES):
        sim.bar(f"kv_full{s}")
        sim.bar(f"kv_empty{s}")
    for i in range(2):
        sim.bar(f"s_full{i}")
        sim.bar(f"p_full{i}")
        sim.bar(f"o_final{i}")
        sim.bar(f"s_free{i}")
        sim.bar(f"p_free{i}")
    for i in range(SCHED):
        sim.bar(f"sched_full{i}")
        sim.bar(f"sched_empty{i}", 3)  # the MMA issuer and the two softmax warpgroups
    end = len(units)

    def unit(k):
        return units[k] if k < end else None

    def producer():
        qc, pos = 0, 0
        for k in range(end + 1):
            slot = k % SCHED
            yield ("wait", f"sched_empty{slot}", k // SCHED - 1)
            yield ("access", [], [(f"sched{slot}", f"unit {k}")], 0.3)
            yield ("arrive", f"sched_full{slot}")
            u = unit(k)
            if u is None:
                break
            n, _ = u
            if n == 0:
                continue
            if qc > 0:
                yield ("wait", "q_empty", qc - 1)
            yield ("async", [], [("Q", f"Q {k}")], 4.0, lambda: sim.arrive("q_full"))
            qc += 1
            for j in range(n):
                for kv in ("K", "V"):
                    s = pos % STAGES
                    yield ("wait", f"kv_empty{s}", pos // STAGES - 1)
                    yield ("async", [], [(f"KV{s}", f"{kv}{j} u{k}")], 3.0, (lambda s=s: sim.arrive(f"kv_full{s}")))
                    pos += 1

    def consume_slot(k):
        slot = k % SCHED
        yield ("wait", f"sched_full{slot}", k // SCHED)
        yield ("access", [(f"sched{slot}", f"unit {k}")], [], 0.2)
        yield ("arrive", f"sched_empty{slot}")

    def mma():
        if sep_p:
            yield from mma_sep_p()
            return
        qc, pos, pc = 0, 0, [0, 0]
        for k in range(end + 1):
            yield from consume_slot(k)
            u = unit(k)
            if u is None:
                break
            n, n0 = u
            if n == 0:
                continue
            yield ("wait", "q_full", qc)
            qc += 1
            base = pos
            nt = (n0, n)
            s0 = base % STAGES
            yield ("wait", f"kv_full{s0}", base // STAGES)
            for qt in range(2):
                if nt[qt] == 0:
                    continue
                yield ("mma", [("Q", f"Q {k}"), (f"KV{s0}", f"K0 u{k}")], [(f"S{qt}", f"S {qt} 0 u{k}")])
                yield ("commit", f"s_full{qt}")
                if (qt == 1 and n == 1) or (early_q_release and qt == 1):
                    yield ("commit", "q_empty")
            yield ("commit", f"kv_empty{s0}")
            for j in range(n):
                pv, pk = base + 2 * j + 1, base + 2 * j + 2
                nxt = j + 1 < n
                yield ("wait", f"kv_full{pv % STAGES}", pv // STAGES)
                if nxt:
                    yield ("wait", f"kv_full{pk % STAGES}", pk // STAGES)
                for qt in range(2):
                    if j >= nt[qt]:
                        continue
                    yield ("wait", f"p_full{qt}", pc[qt])
                    pc[qt] += 1
                    acc = [(f"O{qt}", f"O {qt} u{k}")] if j > 0 else []
                    yield ("mma", [(f"S{qt}", f"P {qt} {j} u{k}"), (f"KV{pv % STAGES}", f"V{j} u{k}")] + acc,
                           [(f"O{qt}", f"O {qt} u{k}")])
                    if qt == 0 and j == n0 - 1 and n0 < n:
                        yield ("commit", "o_final0")
                    if j + 1 < nt[qt]:
                        yield ("mma", [("Q", f"Q {k}"), (f"KV{pk % STAGES}", f"K{j + 1} u{k}")],
                               [(f"S{qt}", f"S {qt} {j + 1} u{k}")])
                        yield ("commit", f"s_full{qt}")
                        if qt == 1 and j + 2 == n and not early_q_release:
                            yield ("commit", "q_empty")
                yield ("commit", f"kv_empty{pv % STAGES}")
                if nxt:
                    yield ("commit", f"kv_empty{pk % STAGES}")
            pos = base + 2 * n
            if n0 == n or (phase_for_keyless_tile and n0 == 0):
                yield ("commit", "o_final0")
            yield ("commit", "o_final1")

    def mma_sep_p():
        qc, pos, pc, qk_cnt = 0, 0, [0, 0], [0, 0]
        for k in range(end + 1):
            yield from consume_slot(k)
            u = unit(k)
            if u is None:
                break
            n, n0 = u
            if n == 0:
                continue
            yield ("wait", "q_full", qc)
            qc += 1
            base = pos
            nt = (n0, n)

            def qk_into(qt, jj, stage_pos):
                if qk_cnt[qt] > 0:
                    yield ("wait", f"s_free{qt}", qk_cnt[qt] - 1)   # S read out by the softmax
                yield ("mma", [("Q", f"Q {k}"), (f"KV{stage_pos % STAGES}", f"K{jj} u{k}")],
                       [(f"S{qt}", f"S {qt} {jj} u{k}")])
                yield ("commit", f"s_full{qt}")
                if qt == 1 and jj == n - 1:
                    yield ("commit", "q_empty")
                qk_cnt[qt] += 1

            yield ("wait", f"kv_full{base % STAGES}", base // STAGES)
            for qt in range(2):
                if nt[qt] > 0:
                    yield from qk_into(qt, 0, base)
            yield ("commit", f"kv_empty{base % STAGES}")
            for j in range(n):
                pv, pk = base + 2 * j + 1, base + 2 * j + 2
                nxt = j + 1 < n
                yield ("wait", f"kv_full{pv % STAGES}", pv // STAGES)
                if nxt:
                    yield ("wait", f"kv_full{pk % STAGES}", pk // STAGES)
                for qt in range(2):
                    if j + 1 < nt[qt]:
                        yield from qk_into(qt, j + 1, pk)
                for qt in range(2):
                    if j >= nt[qt]:
                        continue
                    yield ("wait", f"p_full{qt}", pc[qt])
                    pc[qt] += 1
                    acc = [(f"O{qt}", f"O {qt} u{k}")] if j > 0 else []
                    yield ("mma", [(f"P{qt}", f"P {qt} {j} u{k}"), (f"KV{pv % STAGES}", f"V{j} u{k}")] + acc,
                           [(f"O{qt}", f"O {qt} u{k}")])
                    yield ("commit", f"p_free{qt}")
                    if qt == 0 and j == n0 - 1 and n0 < n:
                        yield ("commit", "o_final0")
                yield ("commit", f"kv_empty{pv % STAGES}")
                if nxt:
                    yield ("commit", f"kv_empty{pk % STAGES}")
            pos = base + 2 * n
            if n0 == n or (phase_for_keyless_tile and n0 == 0):
                yield ("commit", "o_final0")
            yield ("commit", "o_final1")

    def softmax(qt):
        rng = random.Random(sim.rng.random())
        sc, uc, pt = 0, 0, 0
        for k in range(end + 1):
            yield from consume_slot(k)
            u = unit(k)
            if u is None:
                break
            n, n0 = u
            my = n0 if qt == 0 else n
            for j in range(my):
                yield ("wait", f"s_full{qt}", sc)
                sc += 1
                yield ("access", [(f"S{qt}", f"S {qt} {j} u{k}")], [], 1.0)
                if sep_p:
                    yield ("arrive", f"s_free{qt}")                           # the next QK may overwrite S
                yield ("delay", 1.0)                                          # max
                if j > 0 and rng.random() < 0.3:                              # O rescale in place
                    if sep_p and pt > 0:
                        yield ("wait", f"p_free{qt}", pt - 1)                 # the previous PV has landed
                    yield ("access", [(f"O{qt}", f"O {qt} u{k}")], [], 0.5)
                    yield ("access", [], [(f"O{qt}", f"O {qt} u{k}")], 0.5)
                yield ("delay", 4.0)                                          # exponentials
                if sep_p:
                    if pt > 0 and not no_p_free_wait:
                        yield ("wait", f"p_free{qt}", pt - 1)                 # the P buffer is free again
                    yield ("access", [], [(f"P{qt}", f"P {qt} {j} u{k}")], 1.0)
                else:
                    yield ("access", [], [(f"S{qt}", f"P {qt} {j} u{k}")], 1.0)  # P over S
                yield ("arrive", f"p_full{qt}")
                pt += 1
            if n == 0 or (my == 0 and not phase_for_keyless_tile):
                continue                                                      # no key: zeros, no wait
            if not (no_final_wait and qt == 1):
                yield ("wait", f"o_final{qt}", uc)
            uc += 1
            if my > 0:
                yield ("access", [(f"O{qt}", f"O {qt} u{k}")], [], 2.0)      # epilogue read-out

    for name, gen in (("producer", producer()), ("mma", mma()), ("softmax0", softmax(0)), ("softmax1", softmax(1))):
        sim.run(name, gen)


def random_units(rng, count):
    units = []
    for _ in range(count):
        kind = rng.random()
        n = rng.randint(1, 5)
        if kind < 0.45:
            units.append((n, n - 1))          # causal: the first tile one K/V tile short
        elif kind < 0.8:
            units.append((n, n))              # non-causal (or causal off the diagonal)
        elif kind < 0.92:
            units.append((n, 0))              # first tile without keys
        else:
            units.append((0, 0))              # no key at all
    return units


@pytest.mark.parametrize("n_units", [1, 3, 9])
def test_forward_protocol_has_no_hazard_and_finishes(n_units):
    for seed in range(80):
        rng = random.Random(7000 + 100 * n_units + seed)
        units = random_units(rng, n_units)
        sim = Sim(seed)
        forward_cta(sim, units)
        sim.go()
        assert sim.finished == ROLES, f"units {units}, seed {seed}: left waiting {sorted(ROLES - sim.finished)}"
        assert sim.pipe_done == sim.pipe_issued


def _caught(seeds, **planted):
    caught = 0
    for seed in range(seeds):
        units = random_units(random.Random(seed), 5)
        sim = Sim(seed)
        forward_cta(sim, units, **planted)
        try:
            sim.go()
        except Hazard:
            caught += 1
            continue
        if sim.finished != ROLES:
            caught += 1
    return caught


def test_the_model_catches_an_early_q_release():
    """Planted mistake (in the model): Q released after the unit's first QK, so the next unit's Q
    load can overwrite it while later QKs still read it."""
    assert _caught(60, early_q_release=True) > 0


def test_the_model_catches_a_phase_for_a_keyless_first_tile():
    """The scheme the kernel used before the model flagged it: an o_final phase for a first tile
    without keys too. Two such units in a row can complete both phases before that tile's warpgroup
    waits for the first, and a parity wait then aliases."""
    caught = 0
    for seed in range(300):
        rng = random.Random(seed)
        units = [(rng.randint(1, 2), 0) for _ in range(6)] + random_units(rng, 3)
        sim = Sim(seed)
        forward_cta(sim, units, phase_for_keyless_tile=True)
        try:
            sim.go()
        except Hazard:
            caught += 1
            continue
        if sim.finished != ROLES:
            caught += 1
    assert caught > 0


def test_the_model_catches_a_read_out_before_the_last_product():
    """Planted mistake (in the model): the second tile's O read out without waiting for o_final."""
    assert _caught(60, no_final_wait=True) > 0


@pytest.mark.parametrize("n_units", [1, 3, 9])
def test_forward_protocol_with_separate_p_buffers(n_units):
    for seed in range(80):
        rng = random.Random(9000 + 100 * n_units + seed)
        units = random_units(rng, n_units)
        sim = Sim(seed)
        forward_cta(sim, units, sep_p=True)
        sim.go()
        assert sim.finished == ROLES, f"units {units}, seed {seed}: left waiting {sorted(ROLES - sim.finished)}"
        assert sim.pipe_done == sim.pipe_issued


def test_the_model_catches_a_p_buffer_written_under_its_pv():
    """Planted mistake (in the model, d <= 64 variant): P written into its buffer without waiting for
    the previous PV, which may still be reading it."""
    assert _caught(60, sep_p=True, no_p_free_wait=True) > 0


PAIR_STAGES = 5
PAIR_ROLES = {"producer0", "producer1", "mma", "softmax0", "softmax1"}


def pair_cta(sim, units, rescale_without_o_done=False):
    """The d = 256 variant on a CTA pair: one query tile of 128 rows per CTA (a 256-row unit), S
    alternating between two slots (QK_0, QK_1, PV_0, QK_2, PV_1, ...), 2-SM products issued by the
    leader that read and write both CTAs' halves, each CTA's producer loading its own halves with
    the completion counted on the leader's barriers, commits reaching both CTAs. units: K/V tiles
    per unit (the pair's units are a fixed list). rescale_without_o_done plants a mistake: O
    rescaled without waiting for the previous PV."""
    sim.bar("q_full", 2)
    sim.bar("q_empty")
    for st in range(PAIR_STAGES):
        sim.bar(f"kv_full{st}", 2)
        sim.bar(f"kv_empty{st}")
    for i in range(2):
        sim.bar(f"s_full{i}")
        sim.bar(f"p_full{i}", 2)  # one arrival per CTA's softmax warpgroup
    sim.bar("o_done")
    sim.bar("o_final0")

    def producer(r):
        qc, pos = 0, 0
        for k, n in enumerate(units):
            if n == 0:
                continue
            if qc > 0:
                yield ("wait", "q_empty", qc - 1)
            yield ("async", [], [(f"Q_{r}", f"Q {k}")], 4.0, lambda: sim.arrive("q_full"))
            qc += 1
            for j in range(n):
                for kv in ("K", "V"):
                    st = pos % PAIR_STAGES
                    yield ("wait", f"kv_empty{st}", pos // PAIR_STAGES - 1)
                    yield ("async", [], [(f"KV{st}_{r}", f"{kv}{j} u{k}")], 3.0,
                           (lambda st=st: sim.arrive(f"kv_full{st}")))
                    pos += 1

    def both(name, tag):
        return [(f"{name}_0", tag), (f"{name}_1", tag)]

    def mma():
        qc, pos, t_run = 0, 0, 0
        for k, n in enumerate(units):
            if n == 0:
                continue
            yield ("wait", "q_full", qc)
            qc += 1
            base, t0 = pos, t_run
            for j in range(min(2, n)):
                kp = base + 2 * j
                yield ("wait", f"kv_full{kp % PAIR_STAGES}", kp // PAIR_STAGES)
                slot = (t0 + j) & 1
                yield ("mma", both("Q", f"Q {k}") + both(f"KV{kp % PAIR_STAGES}", f"K{j} u{k}"),
                       both(f"S{slot}", f"S {j} u{k}"))
                yield ("commit", f"s_full{slot}")
                if j == n - 1:
                    yield ("commit", "q_empty")
                yield ("commit", f"kv_empty{kp % PAIR_STAGES}")
            for j in range(n):
                t = t0 + j
                slot = t & 1
                vp = base + 2 * j + 1
                yield ("wait", f"kv_full{vp % PAIR_STAGES}", vp // PAIR_STAGES)
                yield ("wait", f"p_full{slot}", t >> 1)
                acc = both("O", f"O u{k}") if j > 0 else []
                yield ("mma", both(f"S{slot}", f"P {j} u{k}") + both(f"KV{vp % PAIR_STAGES}", f"V{j} u{k}") + acc,
                       both("O", f"O u{k}"))
                yield ("commit", "o_done")
                yield ("commit", f"kv_empty{vp % PAIR_STAGES}")
                if j + 2 < n:
                    kp = base + 2 * (j + 2)
                    yield ("wait", f"kv_full{kp % PAIR_STAGES}", kp // PAIR_STAGES)
                    yield ("mma", both("Q", f"Q {k}") + both(f"KV{kp % PAIR_STAGES}", f"K{j + 2} u{k}"),
                           both(f"S{slot}", f"S {j + 2} u{k}"))
                    yield ("commit", f"s_full{slot}")
                    if j + 3 == n:
                        yield ("commit", "q_empty")
                    yield ("commit", f"kv_empty{kp % PAIR_STAGES}")
            t_run = t0 + n
            pos = base + 2 * n
            yield ("commit", "o_final0")

    def softmax(r):
        rng = random.Random(sim.rng.random())
        t_run, uc = 0, 0
        for k, n in enumerate(units):
            for j in range(n):
                slot = t_run & 1
                yield ("wait", f"s_full{slot}", t_run >> 1)
                t_run += 1
                yield ("access", [(f"S{slot}_{r}", f"S {j} u{k}")], [], 1.0)
                yield ("delay", 1.0)
                if j > 0 and rng.random() < 0.3:
                    if not rescale_without_o_done:
                        yield ("wait", "o_done", t_run - 2)                   # the previous PV has landed
                    yield ("access", [(f"O_{r}", f"O u{k}")], [], 0.5)
                    yield ("access", [], [(f"O_{r}", f"O u{k}")], 0.5)
                yield ("delay", 4.0)
                yield ("access", [], [(f"S{slot}_{r}", f"P {j} u{k}")], 1.0)  # P over S
                yield ("arrive", f"p_full{slot}")
            if n == 0:
                continue
            yield ("wait", "o_final0", uc)
            uc += 1
            yield ("access", [(f"O_{r}", f"O u{k}")], [], 2.0)

    for name, gen in (("producer0", producer(0)), ("producer1", producer(1)), ("mma", mma()),
                      ("softmax0", softmax(0)), ("softmax1", softmax(1))):
        sim.run(name, gen)


@pytest.mark.parametrize("n_units", [1, 2, 5])
def test_pair_protocol_has_no_hazard_and_finishes(n_units):
    for seed in range(80):
        rng = random.Random(11000 + 100 * n_units + seed)
        units = [rng.choice((0, 1, 2, 3, 5, 8)) for _ in range(n_units)]
        sim = Sim(seed)
        pair_cta(sim, units)
        sim.go()
        assert sim.finished == PAIR_ROLES, f"units {units}, seed {seed}: left waiting {sorted(PAIR_ROLES - sim.finished)}"
        assert sim.pipe_done == sim.pipe_issued


def test_the_model_catches_a_pair_rescale_without_o_done():
    caught = 0
    for seed in range(60):
        sim = Sim(seed)
        pair_cta(sim, [4, 6, 3], rescale_without_o_done=True)
        try:
            sim.go()
        except Hazard:
            caught += 1
            continue
        if sim.finished != PAIR_ROLES:
            caught += 1
    assert caught > 0
