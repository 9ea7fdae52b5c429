"""A model of the attention kernel's mbarrier protocol, checked for deadlock.

Three actors run their steps in program order, and a step may run only once
the barrier phases it waits on have completed:
  producer  K(n) into K slot n % 2 once S(n-2) = Q K^T has read that slot;
            V(n) into V slot n % 2 once PV(n-2) has read that slot;
  MMA       S(0), S(1); then per stage n: PV(n) once P(n) is written and
            V(n) has landed, then S(n+2) into S buffer n % 2 once K(n+2) has
            landed (the buffer holds P(n), which PV(n), issued just before,
            reads first: tcgen05 MMAs from one thread run in issue order);
  softmax   per stage n: read S(n) once it is computed, then publish P(n)
            once PV(n-1) has completed (the O rescale and the in-order parity
            of the O-ready barrier need it).

The kernel's waits are bounded, so a deadlock would not hang the GPU but would
abort every CTA.  The model checks that no tile length (number of stages)
deadlocks, and, as a control, that it does catch a protocol that deadlocks: a
variant with a single V slot whose MMA issues S(n+2) before PV(n), fed by a
producer that loads K(n) and V(n) in turn.
"""

import pytest


def _run(prog, ready):
    done, pcs = set(), [0] * len(prog)
    while any(pc < len(p) for pc, p in zip(pcs, prog)):
        moved = False
        for i, p in enumerate(prog):
            while pcs[i] < len(p) and ready(p[pcs[i]], done):
                done.add(p[pcs[i]])
                pcs[i] += 1
                moved = True
        if not moved:
            return [p[pc] if pc < len(p) else None for pc, p in zip(pcs, prog)]
    return None


def kernel_protocol(T, ring=2):
    prod = [e for n in range(T) for e in (("K", n), ("V", n))]
    mma = [("S", n) for n in range(min(2, T))]
    for n in range(T):
        mma.append(("PV", n))
        if n + 2 < T:
            mma.append(("S", n + 2))
    soft = [e for n in range(T) for e in (("read", n), ("P", n))]

    def ready(ev, done):
        kind, n = ev
        if kind == "K":
            return n < ring or ("S", n - ring) in done
        if kind == "V":
            return n < ring or ("PV", n - ring) in done
        if kind == "S":
            return ("K", n) in done and (n < 2 or ("PV", n - 2) in done)
        if kind == "PV":
            return ("P", n) in done and ("V", n) in done
        if kind == "read":
            return ("S", n) in done
        if kind == "P":
            return n == 0 or ("PV", n - 1) in done
        raise AssertionError(kind)

    return _run([prod, mma, soft], ready)


def single_v_early_s_protocol(T):
    """The control: one V slot, S(n+2) issued before PV(n), K and V loaded in turn."""
    prod = [e for n in range(T) for e in (("K", n), ("V", n))]
    mma = [("S", n) for n in range(min(2, T))]
    for n in range(T):
        if n + 2 < T:
            mma.append(("S", n + 2))
        mma.append(("PV", n))
    soft = [e for n in range(T) for e in (("read", n), ("P", n))]

    def ready(ev, done):
        kind, n = ev
        if kind == "K":
            return n < 2 or ("S", n - 2) in done
        if kind == "V":
            return n < 1 or ("PV", n - 1) in done
        if kind == "S":
            return ("K", n) in done and (n < 2 or ("read", n - 2) in done)
        if kind == "PV":
            return ("P", n) in done and ("V", n) in done
        if kind == "read":
            return ("S", n) in done
        if kind == "P":
            return n == 0 or ("PV", n - 1) in done
        raise AssertionError(kind)

    return _run([prod, mma, soft], ready)


@pytest.mark.parametrize("ring", [2, 3])
def test_kernel_protocol_never_deadlocks(ring):
    for T in range(0, 65):
        assert kernel_protocol(T, ring) is None, (T, kernel_protocol(T, ring))


def test_model_detects_a_deadlocking_protocol():
    assert single_v_early_s_protocol(2) is None
    stuck = single_v_early_s_protocol(5)
    # producer waits for V(1)'s slot (PV(0)), the MMA for K(2), the softmax for PV(0)
    assert stuck == [("V", 1), ("S", 2), ("P", 1)]
