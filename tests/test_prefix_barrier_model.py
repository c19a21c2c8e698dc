"""The barrier protocol of the tensor-core shared-prefix kernel
(paged_kv_cache_410_b200/csrc/pa_prefix_umma.cuh), model-checked on the CPU.

A model of the kernel's three roles for one row tile: the TMA producer
(K and V stages, NSTAGE deep), the MMA thread (issues S(i) = Q K_i^T into S
buffer i & 1, and P.V(it), as asynchronous operations that may complete in
ANY order), and the softmax warps (one thread stands for them: a barrier's
arrival count is reached by all of them together). Barriers are counters of
completed phases, and a wait sees only the parity of the phase it names, as
mbarrier.try_wait.parity does. Every interleaving is explored; the checks:

  * no state where some role waits forever (deadlock);
  * no parity wait that fires for a phase that has not completed (a phase
    that wrapped would read as complete);
  * no S buffer, P tile, O accumulator or K/V stage written while an
    operation that reads it, or a thread reading it, is still in flight.

The protocol modelled is the kernel's: S(i) waits for K stage i and for the
softmax to have loaded S(i-2) (sfree); S(it+1) is issued before P.V(it); the
softmax loads S(it), frees its buffer, waits for P.V(it-1) (the single P tile
and O), rescales O if its reference max moved, writes P and arrives on pfull;
P.V(it) waits for pfull and V stage it. Planted mistakes check that the
model is not vacuous. (The model also shows the sfree wait to be implied by
the pfull one: S(i) is issued only after P.V(i-2), which waited for the
softmax to arrive after loading S(i-2); the kernel keeps it as a cheap
second guard.)
"""
from collections import deque

import pytest

NSTAGE = 2


class Violation(Exception):
    pass


def check(nsteps, fault=None, nstage=NSTAGE):
    """Explore every interleaving; returns the number of states, raises
    Violation (with a reason) on a hazard, a wrapped parity or a deadlock.
    `nstage`: K/V stages (the kernel's build-time stage count)."""
    NSTAGE = nstage  # noqa: N806 (shadows the module default inside the model)

    def wait(st, name, k, what):
        c = st["bar"][name]
        if (c & 1) == (k & 1):          # try_wait.parity: phase with parity k&1 not done
            return False
        if c <= k:
            raise Violation(f"{what}: wait on {name} phase {k} fired with {c} completed")
        return True

    def freeze(st):
        return (st["prod"], st["prod_v"], st["mma"], st["smx"], tuple(sorted(st["pending"])),
                tuple(sorted(st["bar"].items())), st["s_reading"], st["p_unread"])

    def cp(st, **kw):
        n = dict(st)
        n["bar"] = dict(st["bar"])
        n.update(kw)
        return n

    def successors(st):
        out = []
        i = st["prod"]                                   # ---- producer
        if i < nsteps:
            s, kind = i % NSTAGE, ("v" if st["prod_v"] else "k")
            if i < NSTAGE or (fault == "no_kfree_wait" and kind == "k") or \
                    wait(st, f"{kind}free{s}", i // NSTAGE - 1, f"load {kind}{i}"):
                for op, j in st["pending"]:
                    if j % NSTAGE == s and j != i and (op == "S") == (kind == "k"):
                        raise Violation(f"{kind} stage {s} reloaded while {op}({j}) reads it")
                n = cp(st)
                n["bar"][f"{kind}full{s}"] += 1
                n.update(prod_v=False, prod=i + 1) if kind == "v" else n.update(prod_v=True)
                out.append(n)
        for op in st["pending"]:                         # ---- MMA completions, any order
            kind, j = op
            n = cp(st, pending=tuple(x for x in st["pending"] if x != op))
            if kind == "S":
                n["bar"][f"sfull{j & 1}"] += 1
                n["bar"][f"kfree{j % NSTAGE}"] += 1
            else:
                n["bar"]["pv"] += 1
                n["bar"][f"vfree{j % NSTAGE}"] += 1
                n["p_unread"] = None
            out.append(n)
        pc, it = st["mma"]                               # ---- MMA thread

        def issue_s(j):
            if st["s_reading"] is not None and (st["s_reading"] & 1) == (j & 1):
                raise Violation(f"S({j}) written while the softmax reads S({st['s_reading']})")
            return cp(st, pending=st["pending"] + (("S", j),))

        if pc == "start":
            if wait(st, "kfull0", 0, "S(0)"):
                out.append(dict(issue_s(0), mma=("s", 0)))
        elif pc == "s":
            j = it + 1
            if j < nsteps:
                ready = wait(st, f"kfull{j % NSTAGE}", j // NSTAGE, f"S({j}) K")
                if ready and j >= 2 and fault != "no_sfree_wait":
                    ready = wait(st, f"sfree{j & 1}", (j - 2) >> 1, f"S({j}) sfree")
                if ready:
                    out.append(dict(issue_s(j), mma=("pv", it)))
            else:
                out.append(cp(st, mma=("pv", it)))
        elif pc == "pv":
            if wait(st, "pfull", it + (1 if fault == "pfull_phase" else 0), f"P.V({it}) P") and \
                    wait(st, f"vfull{it % NSTAGE}", it // NSTAGE, f"P.V({it}) V"):
                out.append(cp(st, pending=st["pending"] + (("PV", it),),
                              mma=("s", it + 1) if it + 1 < nsteps else ("end", it)))
        pc, it = st["smx"][0], st["smx"][1]              # ---- softmax
        if pc == "wait_s" and it < nsteps:
            if wait(st, f"sfull{it & 1}", it >> 1, f"softmax S({it})"):
                out.append(cp(st, s_reading=it, smx=("loaded", it)))
        elif pc == "loaded":
            n = cp(st, s_reading=None, smx=("wait_pv", it))
            n["bar"][f"sfree{it & 1}"] += 1
            out.append(n)
        elif pc == "wait_pv":
            if it == 0 or fault == "no_pv_wait" or wait(st, "pv", it - 1, f"P({it}) tile"):
                if any(op == "PV" for op, _ in st["pending"]):
                    raise Violation(f"P({it}) tile / O written while a P.V is in flight")
                out.append(cp(st, p_unread=it, smx=("arrive", it)))
        elif pc == "arrive":
            n = cp(st, smx=("wait_s", it + 1))
            n["bar"]["pfull"] += 1
            out.append(n)
        return out

    start = {"prod": 0, "prod_v": False, "mma": ("start", 0), "smx": ("wait_s", 0),
             "pending": (), "s_reading": None, "p_unread": None,
             "bar": {b: 0 for b in [f"{x}{i}" for x in ("kfull", "vfull", "kfree", "vfree")
                                    for i in range(NSTAGE)] +
                     ["sfull0", "sfull1", "sfree0", "sfree1", "pfull", "pv"]}}
    seen, q = {freeze(start)}, deque([start])
    while q:
        st = q.popleft()
        succ = successors(st)
        done = (st["smx"] == ("wait_s", nsteps) and st["mma"][0] == "end" and not st["pending"]
                and st["prod"] == nsteps)
        if not succ and not done:
            raise Violation(f"deadlock: mma={st['mma']} softmax={st['smx']} bars={st['bar']}")
        for n in succ:
            f = freeze(n)
            if f not in seen:
                seen.add(f)
                q.append(n)
    return len(seen)


@pytest.mark.parametrize("nstage", [1, 2, 3, 4])
@pytest.mark.parametrize("nsteps", [1, 2, 3, 4, 6, 8])
def test_the_kernels_protocol_has_no_hazard_wrap_or_deadlock(nsteps, nstage):
    assert check(nsteps, nstage=nstage) > 0


@pytest.mark.parametrize("fault,reason", [
    # a K stage refilled early: under its MMA, or twice before it (kfull wraps)
    ("no_kfree_wait", "reloaded while S|deadlock"),
    ("no_pv_wait", "while a P.V is in flight"),     # the P tile rewritten too early
    ("pfull_phase", "fired with"),                  # P.V waits on the wrong phase's parity
])
def test_planted_protocol_mistakes_are_caught(fault, reason):
    with pytest.raises(Violation, match=reason):
        check(5, fault)
