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
  * no S buffer, P, O accumulator or K/V stage written while an operation
    that reads it, or a thread reading it, is still in flight.

The kernel keeps P in tensor memory (mode "tmem"): the softmax writes P(it),
packed to 16 bits, over the S buffer it loaded S(it) from, and P.V(it) takes
its A operand from there. So S buffer i & 1 holds S(i), then P(i), until
P.V(i) has read it; S(i + 2) may be written into it only after that. The
protocol: S(i) waits for K stage i and, for i >= 2, for P.V(i - 2) to have
completed; S(it+1) is issued before P.V(it); the softmax loads S(it), writes
P(it) into the same buffer, waits for P.V(it-1) (O), rescales O if its
reference max moved, and arrives on pfull; P.V(it) waits for pfull and V
stage it.

Mode "smem" is the earlier form of the kernel, kept as a second model: one P
tile in shared memory, S(i) waiting on an sfree barrier the softmax arrives
on once it has loaded S(i - 2). Planted mistakes check that neither model
is vacuous.
"""
from collections import deque

import pytest

NSTAGE = 2


class Violation(Exception):
    pass


def check(nsteps, fault=None, nstage=NSTAGE, mode="tmem"):
    """Explore every interleaving; returns the number of states, raises
    Violation (with a reason) on a hazard, a wrapped parity or a deadlock.
    `nstage`: K/V stages (the kernel's build-time stage count)."""
    NSTAGE = nstage  # noqa: N806 (shadows the module default inside the model)
    tmem = mode == "tmem"

    def wait(st, name, k, what):
        c = st["bar"][name]
        if (c & 1) == (k & 1):          # try_wait.parity: phase with parity k&1 not done
            return False
        if c <= k:
            raise Violation(f"{what}: wait on {name} phase {k} fired with {c} completed")
        return True

    def freeze(st):
        return (st["prod"], st["prod_v"], st["mma"], st["smx"], tuple(sorted(st["pending"])),
                tuple(sorted(st["bar"].items())), st["s_reading"], st["p_unread"], st["p_buf"])

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
                if tmem:                                 # P(j) consumed from buffer j & 1
                    pb = list(st["p_buf"])
                    if pb[j & 1] == j:
                        pb[j & 1] = None
                    n["p_buf"] = tuple(pb)
            out.append(n)
        pc, it = st["mma"]                               # ---- MMA thread

        def issue_s(j):
            b = j & 1
            if st["s_reading"] is not None and (st["s_reading"] & 1) == b:
                raise Violation(f"S({j}) written while the softmax reads S({st['s_reading']})")
            if tmem:
                for op, k in st["pending"]:
                    if op == "PV" and (k & 1) == b:
                        raise Violation(f"S({j}) written while P.V({k}) reads P({k})")
                if st["p_buf"][b] is not None:
                    raise Violation(f"S({j}) written over P({st['p_buf'][b]}) before its P.V")
            return cp(st, pending=st["pending"] + (("S", j),))

        def s_ready(j):
            """S(j)'s waits besides its K stage."""
            if j < 2:
                return True
            if tmem:
                return fault == "no_pv_before_s" or wait(st, "pv", j - 2, f"S({j}) after P.V")
            return fault == "no_sfree_wait" or wait(st, f"sfree{j & 1}", (j - 2) >> 1,
                                                    f"S({j}) sfree")

        if pc == "start":
            if wait(st, "kfull0", 0, "S(0)"):
                out.append(dict(issue_s(0), mma=("s", 0)))
        elif pc == "s":
            j = it + 1
            if j < nsteps:
                if wait(st, f"kfull{j % NSTAGE}", j // NSTAGE, f"S({j}) K") and s_ready(j):
                    out.append(dict(issue_s(j), mma=("pv", it)))
            else:
                out.append(cp(st, mma=("pv", it)))
        elif pc == "pv":
            if wait(st, "pfull", it + (1 if fault == "pfull_phase" else 0), f"P.V({it}) P") and \
                    wait(st, f"vfull{it % NSTAGE}", it // NSTAGE, f"P.V({it}) V"):
                if tmem and st["p_buf"][it & 1] != it:
                    raise Violation(f"P.V({it}) issued before P({it}) was written")
                out.append(cp(st, pending=st["pending"] + (("PV", it),),
                              mma=("s", it + 1) if it + 1 < nsteps else ("end", it)))
        pc, it = st["smx"][0], st["smx"][1]              # ---- softmax
        if pc == "wait_s" and it < nsteps:
            if wait(st, f"sfull{it & 1}", it >> 1, f"softmax S({it})"):
                out.append(cp(st, s_reading=it, smx=("loaded", it)))
        elif pc == "loaded":
            if tmem:
                # P(it) goes over S(it)'s buffer (the wrong one when planted)
                b = (it + 1) & 1 if fault == "p_other_buffer" else it & 1
                for op, k in st["pending"]:
                    if (k & 1) == b and op in ("S", "PV"):
                        raise Violation(f"P({it}) written while {op}({k}) uses its buffer")
                pb = list(st["p_buf"])
                if pb[b] is not None:
                    raise Violation(f"P({it}) written over P({pb[b]}) before its P.V")
                pb[b] = it
                out.append(cp(st, s_reading=None, p_buf=tuple(pb), smx=("wait_pv", it)))
            else:
                n = cp(st, s_reading=None, smx=("wait_pv", it))
                n["bar"][f"sfree{it & 1}"] += 1
                out.append(n)
        elif pc == "wait_pv":
            if it == 0 or fault == "no_pv_wait" or wait(st, "pv", it - 1, f"O before P.V({it})"):
                if any(op == "PV" for op, _ in st["pending"]):
                    raise Violation(f"P({it}) tile / O written while a P.V is in flight")
                out.append(cp(st, p_unread=None if tmem else it, smx=("arrive", it)))
        elif pc == "arrive":
            n = cp(st, smx=("wait_s", it + 1))
            n["bar"]["pfull"] += 1
            out.append(n)
        return out

    bars = [f"{x}{i}" for x in ("kfull", "vfull", "kfree", "vfree") for i in range(NSTAGE)]
    bars += ["sfull0", "sfull1", "pfull", "pv"] + ([] if tmem else ["sfree0", "sfree1"])
    start = {"prod": 0, "prod_v": False, "mma": ("start", 0), "smx": ("wait_s", 0),
             "pending": (), "s_reading": None, "p_unread": None, "p_buf": (None, None),
             "bar": {b: 0 for b in bars}}
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


@pytest.mark.parametrize("mode", ["tmem", "smem"])
@pytest.mark.parametrize("nstage", [1, 2, 3, 4])
@pytest.mark.parametrize("nsteps", [1, 2, 3, 4, 6, 8])
def test_the_kernels_protocol_has_no_hazard_wrap_or_deadlock(nsteps, nstage, mode):
    assert check(nsteps, nstage=nstage, mode=mode) > 0


@pytest.mark.parametrize("mode,fault,reason", [
    # a K stage refilled early: under its MMA, or twice before it (kfull wraps)
    ("tmem", "no_kfree_wait", "reloaded while S|deadlock"),
    ("smem", "no_kfree_wait", "reloaded while S|deadlock"),
    ("tmem", "no_pv_wait", "while a P.V is in flight"),   # O rescaled under P.V(it-1)
    ("smem", "no_pv_wait", "while a P.V is in flight"),   # the P tile rewritten too early
    ("tmem", "pfull_phase", "fired with"),                # P.V waits on the wrong phase's parity
    ("smem", "pfull_phase", "fired with"),
    # S(i) written over P(i-2) while P.V(i-2) may still read it
    ("tmem", "no_pv_before_s", r"while P\.V\(\d+\) reads P|over P\(\d+\) before its P\.V"),
    # P written into the other S buffer, which S(it+1) fills
    ("tmem", "p_other_buffer", r"P\(\d+\) written|issued before P"),
])
def test_planted_protocol_mistakes_are_caught(mode, fault, reason):
    with pytest.raises(Violation, match=reason):
        check(5, fault, mode=mode)
