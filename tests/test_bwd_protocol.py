"""A model of the backward kernel's hand-off protocol (csrc/attn_bwd.cu, one CTA), run under random
timings on the CPU.

The roles are coroutines: the TMA producer, the MMA issuer (its products run in issue order on an
asynchronous tensor pipe, and a commit arrives once every product issued before it is done), the
elementwise warps, the dQ warps and the end-of-unit dK/dV store. Every tensor-memory column range
and shared-memory buffer holds a tagged version ("S 3" = S^T of step 3). The checks:

- every wait on an mbarrier targets one phase and sees it complete without the barrier having moved
  two phases past it (a parity wait cannot tell those apart);
- every read finds the version it expects, and nothing is written while it is being read;
- all roles finish (no wait is left without its arrival).

The model follows the kernel's order of waits, arrivals, commits and accesses step by step; its
durations are random and roles are now and then held up for long stretches, so each seed is another
interleaving. Two tests plant mistakes in the model (not in the kernel) to show the checks bite: dQ's
columns released before they are read, and one barrier instead of two alternating slots for dK's
completion (caught as parity aliasing in some interleavings).
"""
import pytest

from protocol_sim import Hazard, Sim


BARRIERS = ("kv_full", "q_full0", "q_full1", "q_empty0", "q_empty1", "st_full", "s_full", "pt_full", "p_full",
            "dq_full", "dq_free", "dk_done0", "dk_done1", "dkv_full", "epi_full", "epi_free")
ROLES = {"producer", "mma", "elementwise", "store", "dq"}


def backward_cta(sim, n_steps, early_release=False, single_dk=False):
    """Starts the roles of one backward CTA over n_steps steps (one key block). Each barrier takes one
    arrival per phase here (the kernel's counts are per warp; a role stands for its warps).

    early_release and single_dk plant mistakes (for the tests that show the model can catch them):
    the dQ warps release dQ's columns before reading them out, or dK's completion is tracked in one
    barrier for every step instead of two slots used on alternate steps."""
    for name in BARRIERS:
        sim.bar(name)
    if single_dk:
        sim.bars["dk_done1"] = sim.bars["dk_done0"]

    def producer():
        yield ("async", [], [("K", "K"), ("V", "V")], 6.0, lambda: sim.arrive("kv_full"))
        for t in range(n_steps):
            st = t & 1
            if t >= 2:
                yield ("wait", f"q_empty{st}", (t - 2) >> 1)
            yield ("async", [], [(f"Q{st}", f"Q {t}"), (f"dO{st}", f"dO {t}"), (f"LD{st}", f"LD {t}")], 6.0,
                   (lambda s=st: sim.arrive(f"q_full{s}")))

    def mma():
        yield ("wait", "kv_full", 0)
        for t in range(n_steps):
            st = t & 1
            yield ("wait", f"q_full{st}", t >> 1)
            if t > 0:
                yield ("wait", "dq_free", t - 1)                 # dQ of the last step read out
            yield ("mma", [("K", "K"), (f"Q{st}", f"Q {t}")], [("S", f"S {t}")])
            yield ("commit", "st_full")
            yield ("mma", [("V", "V"), (f"dO{st}", f"dO {t}")], [("DP", f"DP {t}")])
            yield ("commit", "s_full")
            yield ("wait", "pt_full", t)
            acc = [("DV", "DV")] if t > 0 else []
            yield ("mma", [("S", f"P {t}"), (f"dO{st}", f"dO {t}")] + acc, [("DV", "DV")])
            yield ("wait", "p_full", t)
            yield ("mma", [("dS", f"dS {t}"), ("K", "K")], [("S", f"dQ {t}")])
            yield ("commit", "dq_full")
            acc = [("DK", "DK")] if t > 0 else []
            yield ("mma", [("DP", f"dS^T {t}"), (f"Q{st}", f"Q {t}")] + acc, [("DK", "DK")])
            yield ("commit", f"dk_done{t & 1}")
            if t == n_steps - 1:
                yield ("commit", "dkv_full")

    def elementwise():
        for t in range(n_steps):
            st = t & 1
            yield ("wait", "st_full", t)
            yield ("access", [(f"LD{st}", f"LD {t}")], [], 1.0)
            yield ("access", [("S", f"S {t}")], [], 2.0)         # S^T read out
            yield ("delay", 6.0)                                 # exponentials
            yield ("access", [], [("S", f"P {t}")], 1.0)         # P^T over S^T
            yield ("arrive", "pt_full")
            yield ("wait", "s_full", t)
            yield ("access", [("DP", f"DP {t}"), (f"LD{st}", f"LD {t}")], [], 2.0)
            yield ("access", [], [("DP", f"dS^T {t}"), ("dS", f"dS {t}")], 2.0)
            yield ("arrive", "p_full")
        if n_steps == 0:
            return
        # end of the key block: dK and dV through the dS tile and TMA stores
        yield ("wait", "dkv_full", 0)
        for which, name in enumerate(("DK", "DV")):
            yield ("access", [(name, name)], [("dS", f"epi {name}")], 2.0)
            yield ("arrive", "epi_full")
            yield ("wait", "epi_free", which)

    def epilogue_store():
        if n_steps == 0:
            return
        for which, name in enumerate(("DK", "DV")):
            yield ("wait", "epi_full", which)
            done = []                                            # the store's read completion
            yield ("async", [("dS", f"epi {name}")], [], 3.0, lambda: done.append(1))
            while not done:
                yield ("delay", 0.5)
            yield ("arrive", "epi_free")

    def dq_warps():
        for t in range(n_steps):
            st = t & 1
            yield ("wait", "dq_full", t)
            if early_release:
                yield ("arrive", "dq_free")
                yield ("delay", 8.0)
            yield ("access", [("S", f"dQ {t}")], [(f"dO{st}", f"dQ hi {t}")], 2.0)  # columns 64..127
            reads = []
            yield ("async", [(f"dO{st}", f"dQ hi {t}")], [], 3.0, lambda: reads.append(1))
            yield ("access", [("S", f"dQ {t}")], [], 1.0)                            # columns 0..63
            if not early_release:
                yield ("arrive", "dq_free")
            if single_dk:
                yield ("wait", "dk_done0", t)
            else:
                yield ("wait", f"dk_done{t & 1}", t >> 1)
            yield ("access", [], [(f"Q{st}", f"dQ lo {t}")], 1.0)
            yield ("async", [(f"Q{st}", f"dQ lo {t}")], [], 3.0, lambda: reads.append(1))
            while len(reads) < 2:                                # both reduce-adds have read their boxes
                yield ("delay", 0.5)
            yield ("arrive", f"q_empty{st}")

    for name, gen in (("producer", producer()), ("mma", mma()), ("elementwise", elementwise()),
                      ("store", epilogue_store()), ("dq", dq_warps())):
        sim.run(name, gen)


@pytest.mark.parametrize("n_steps", [1, 2, 3, 7, 16])
def test_backward_protocol_has_no_hazard_and_finishes(n_steps):
    for seed in range(60):
        sim = Sim(1000 * n_steps + seed)
        backward_cta(sim, n_steps)
        sim.go()
        assert sim.finished == ROLES, f"seed {seed}: roles left waiting: {sorted(ROLES - sim.finished)}"
        assert sim.pipe_done == sim.pipe_issued == 5 * n_steps


def _caught(n_steps, seeds, **planted):
    caught = 0
    for seed in range(seeds):
        sim = Sim(seed)
        backward_cta(sim, n_steps, **planted)
        try:
            sim.go()
        except Hazard:
            caught += 1
            continue
        if sim.finished != ROLES:
            caught += 1
    return caught


def test_the_model_catches_a_release_before_the_read():
    """Planted mistake (in the model): dQ's columns released before they are read out; the next
    step's S^T may then overwrite dQ first."""
    assert _caught(4, 40, early_release=True) > 0


def test_the_model_catches_a_single_dk_barrier():
    """Planted mistake (in the model): one dk_done barrier for every step. With the columns released
    before that wait, the next step's dK can complete too before the dQ warps look, and a parity
    wait cannot tell the two phases apart."""
    assert _caught(8, 300, single_dk=True) > 0
