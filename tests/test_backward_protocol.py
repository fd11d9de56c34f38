"""Randomised model of the two tcgen05 backward kernels' synchronisation (CPU only).

The dq and dk/dv kernels (block_sparse_taylor_b200/csrc/backward_tc.cuh) coordinate a TMA
producer, a single-thread MMA issuer and the softmax warps through mbarriers.  This model follows
each role's sequence of waits, arrivals, TMA loads, MMAs and commits, and runs them against one
another in random interleavings, with TMA loads and MMAs completing asynchronously (MMAs in issue
order, as the tensor pipe runs them).  It checks that:
- no role can deadlock;
- a parity wait never sees its barrier two phases ahead (an aliased phase);
- no TMA load lands in shared memory that an issued MMA has yet to read, or that the softmax is
  writing;
- no MMA writes TMEM columns that the softmax is reading;
- no MMA reads TMEM columns or shared memory that the softmax is writing.

It covers the three stage layouts of the dk/dv kernel, (Q, dO) stages = (2, 1), (1, 1) and
(2, 2), and the dq kernel's three K and two V stages.  Four planted mistakes must be caught,
so the checks are known to bite.
"""
import random

import pytest


class ProtocolError(Exception):
    pass


class Bar:
    """An mbarrier: `count` arrivals plus the expected transaction bytes complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.arr, self.tx, self.phase = name, count, 0, 0, 0

    def _check(self):
        if self.arr == self.count and self.tx == 0:
            self.phase += 1
            self.arr = 0

    def arrive(self, n=1):
        self.arr += n
        if self.arr > self.count:
            raise ProtocolError(f"over-arrival on {self.name}")
        self._check()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arr += 1
        self._check()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        if self.tx < 0:
            raise ProtocolError(f"transaction underflow on {self.name}")
        self._check()


def overlap(a, b):
    return a[0] < b[1] and b[0] < a[1]


def run_roles(roles, bars, rng):
    """Interleave the role generators at random.  Requests:
    ("wait", bar, phase)                      parity wait for that phase to complete
    ("tma", bar, bytes, smem range)           async load completing on bar
    ("mma", smem reads, TMEM reads, TMEM writes, smem reads the softmax may write)
    ("commit", bar)                           arrives once every earlier MMA has run
    ("tread"/"tdone", range)                  softmax reads (or writes) TMEM columns
    ("swrite"/"sdone", range)                 softmax writes shared memory
    ("arrive", bar, n)
    """
    tma_q, pipe, pend_reads = [], [], []
    t_held, s_held = [], []
    pending = {n: None for n in roles}
    done = set()

    def step_role(name):
        gen = roles[name]
        while True:
            req = pending[name]
            if req is None:
                try:
                    req = next(gen)
                except StopIteration:
                    done.add(name)
                    return True
                pending[name] = req
            kind = req[0]
            if kind == "wait":
                b = bars[req[1]]
                if b.phase > req[2] + 1:
                    raise ProtocolError(f"{name}: parity alias on {req[1]} (phase {req[2]}, at {b.phase})")
                if b.phase <= req[2]:
                    return False
            elif kind == "tma":
                _, bar, nbytes, rg = req
                if any(overlap(rr, rg) for rr in pend_reads):
                    raise ProtocolError(f"TMA into {rg} while an MMA has yet to read it")
                if any(overlap(hr, rg) for hr in s_held):
                    raise ProtocolError(f"TMA into {rg} while the softmax writes it")
                bars[bar].expect_tx(nbytes)
                tma_q.append((bar, nbytes, rg))
            elif kind == "mma":
                pend_reads.extend(req[1])
                pipe.append(req)
            elif kind == "commit":
                pipe.append(req)
            elif kind == "tread":
                t_held.append(req[1])
            elif kind == "tdone":
                t_held.remove(req[1])
            elif kind == "swrite":
                if any(overlap(rr, req[1]) for rr in pend_reads):
                    raise ProtocolError(f"softmax writes {req[1]} while an MMA has yet to read it")
                if any(overlap(rg, req[1]) for (_, _, rg) in tma_q):
                    raise ProtocolError(f"softmax writes {req[1]} while a TMA lands there")
                s_held.append(req[1])
            elif kind == "sdone":
                s_held.remove(req[1])
            elif kind == "arrive":
                bars[req[1]].arrive(req[2])
            pending[name] = None
            if rng.random() < 0.3:
                return True

    for _ in range(10 ** 6):
        if len(done) == len(roles):
            return
        choices = [n for n in roles if n not in done] + (["tma"] if tma_q else []) + (["pipe"] if pipe else [])
        rng.shuffle(choices)
        progressed = False
        for c in choices:
            if c == "tma":
                bar, nbytes, _ = tma_q.pop(rng.randrange(len(tma_q)))
                bars[bar].complete_tx(nbytes)
                progressed = True
                break
            if c == "pipe":
                op = pipe.pop(0)
                if op[0] == "mma":
                    _, sreads, treads, twrites, sm_reads = op
                    for w in twrites:
                        if any(overlap(w, h) for h in t_held):
                            raise ProtocolError(f"MMA writes TMEM {w} while the softmax uses it")
                    for r in treads:
                        if any(overlap(r, h) for h in t_held):
                            raise ProtocolError(f"MMA reads TMEM {r} while the softmax writes it")
                    for r in sm_reads:
                        if any(overlap(r, h) for h in s_held):
                            raise ProtocolError(f"MMA reads smem {r} while the softmax writes it")
                    for r in sreads:
                        pend_reads.remove(r)
                else:
                    bars[op[1]].arrive(1)
                progressed = True
                break
            before = pending[c]
            if step_role(c) or pending[c] is not before:
                progressed = True
                break
        if not progressed:
            raise ProtocolError(f"deadlock: {[(n, pending[n]) for n in roles if n not in done]}")
    raise ProtocolError("no end after 10^6 steps")


T = 32768  # one 128 x 128 bf16 tile in shared memory


def dkdv_model(nqt, nsq, nso, seed, mistake=None):
    """bwd_dkdv_tc_kernel: TMEM S | G | dV | dK; shared K, V, Q[nsq], dO[nso], P, dS."""
    rng = random.Random(seed)
    K_, V_ = (0, T), (T, 2 * T)
    q0 = 2 * T
    o0 = q0 + nsq * T
    Qr = lambda s: (q0 + s * T, q0 + (s + 1) * T)  # noqa: E731
    Or = lambda s: (o0 + s * T, o0 + (s + 1) * T)  # noqa: E731
    Pr = (o0 + nso * T, o0 + nso * T + T)
    DSr = (Pr[1], Pr[1] + T)
    Sc, Gc, DVc, DKc = (0, 128), (128, 256), (256, 384), (384, 512)
    early_s, early_g = nsq >= 2, nso >= 2
    bars = {"KVFULL": Bar("KVFULL", 1)}
    for s in range(nsq):
        bars[f"QFULL{s}"], bars[f"QEMPTY{s}"] = Bar(f"QFULL{s}", 1), Bar(f"QEMPTY{s}", 1)
    for s in range(nso):
        bars[f"DOFULL{s}"], bars[f"DOEMPTY{s}"] = Bar(f"DOFULL{s}", 1), Bar(f"DOEMPTY{s}", 1)
    for n in ("SFULL", "GFULL", "PFREE", "DSFREE", "DKVFULL", "DONE"):
        bars[n] = Bar(n, 1)
    for n in ("SFREE", "GFREE", "PREADY", "DSREADY"):
        bars[n] = Bar(n, 256)

    def producer():
        yield ("tma", "KVFULL", 2 * T, (0, 2 * T))

        def load_q(i):
            s, u = i % nsq, i // nsq
            if u > 0:
                yield ("wait", f"QEMPTY{s}", u - 1)
            yield ("tma", f"QFULL{s}", T, Qr(s))

        def load_do(i):
            s, u = i % nso, i // nso
            if u > 0:
                yield ("wait", f"DOEMPTY{s}", u - 1)
            yield ("tma", f"DOFULL{s}", T, Or(s))

        q_first = early_s if mistake != "dO first with two Q stages" else False
        for i in range(nqt):
            if q_first:
                yield from load_q(i)
                yield from load_do(i)
            else:
                yield from load_do(i)
                yield from load_q(i)

    def issuer():
        def put_s(i):
            if i > 0 and mistake != "S without SFREE":
                yield ("wait", "SFREE", i - 1)
            s, u = i % nsq, i // nsq
            yield ("wait", f"QFULL{s}", u)
            yield ("mma", [Qr(s), K_], [], [Sc], [])
            yield ("commit", "SFULL")

        def put_g(i):
            if i > 0:
                yield ("wait", "GFREE", i - 1)
            s, u = i % nso, i // nso
            yield ("wait", f"DOFULL{s}", u)
            yield ("mma", [Or(s), V_], [], [Gc], [])
            yield ("commit", "GFULL")

        yield ("wait", "KVFULL", 0)
        yield from put_s(0)
        yield from put_g(0)
        for i in range(nqt):
            sq, so, more = i % nsq, i % nso, i + 1 < nqt
            if early_s and more:
                yield from put_s(i + 1)
            yield ("wait", "PREADY", i)
            yield ("mma", [Pr, Or(so)], [], [DVc], [Pr])
            yield ("commit", f"DOEMPTY{so}")
            yield ("commit", "PFREE")
            if early_g and more:
                yield from put_g(i + 1)
            yield ("wait", "DSREADY", i)
            if mistake == "Q released before dK":
                yield ("commit", f"QEMPTY{sq}")
                yield ("mma", [DSr, Qr(sq)], [], [DKc], [DSr])
            else:
                yield ("mma", [DSr, Qr(sq)], [], [DKc], [DSr])
                yield ("commit", f"QEMPTY{sq}")
            yield ("commit", "DSFREE")
            if not early_s and more:
                yield from put_s(i + 1)
            if not early_g and more:
                yield from put_g(i + 1)
        yield ("commit", "DKVFULL")
        yield ("commit", "DONE")
        yield ("wait", "DONE", 0)

    def softmax():
        for i in range(nqt):
            yield ("wait", "SFULL", i)
            yield ("tread", Sc)
            yield ("tdone", Sc)
            yield ("arrive", "SFREE", 256)
            if i > 0 and mistake != "P written without PFREE":
                yield ("wait", "PFREE", i - 1)
            yield ("swrite", Pr)
            yield ("sdone", Pr)
            yield ("arrive", "PREADY", 256)
            yield ("wait", "GFULL", i)
            yield ("tread", Gc)
            yield ("tdone", Gc)
            yield ("arrive", "GFREE", 256)
            if i > 0:
                yield ("wait", "DSFREE", i - 1)
            yield ("swrite", DSr)
            yield ("sdone", DSr)
            yield ("arrive", "DSREADY", 256)
        yield ("wait", "DKVFULL", 0)
        yield ("tread", DKc)
        yield ("tread", DVc)
        yield ("tdone", DKc)
        yield ("tdone", DVc)

    run_roles({"producer": producer(), "issuer": issuer(), "softmax": softmax()}, bars, rng)


def dq_model(nt, seed):
    """bwd_dq_tc_kernel: TMEM S0 | S1 | G | dQ; shared Q, dO, K[3], V[2].  The softmax writes dS
    (bf16) over the S buffer it read, and dQ reads it from there."""
    rng = random.Random(seed)
    nsk, nsv = 3, 2
    Kr = lambda s: (2 * T + s * T, 2 * T + (s + 1) * T)  # noqa: E731
    Vr = lambda s: (5 * T + s * T, 5 * T + (s + 1) * T)  # noqa: E731
    Sc = lambda b: (b * 128, b * 128 + 128)  # noqa: E731
    Gc, DQc = (256, 384), (384, 512)
    bars = {n: Bar(n, 1) for n in ("QFULL", "GFULL", "DQFULL", "DONE")}
    bars["GFREE"] = Bar("GFREE", 256)
    for s in range(nsk):
        bars[f"KFULL{s}"], bars[f"KEMPTY{s}"] = Bar(f"KFULL{s}", 1), Bar(f"KEMPTY{s}", 1)
    for s in range(nsv):
        bars[f"VFULL{s}"], bars[f"VEMPTY{s}"] = Bar(f"VFULL{s}", 1), Bar(f"VEMPTY{s}", 1)
    for b in range(2):
        bars[f"SFULL{b}"], bars[f"DSREADY{b}"] = Bar(f"SFULL{b}", 1), Bar(f"DSREADY{b}", 256)

    def producer():
        yield ("tma", "QFULL", 2 * T, (0, 2 * T))
        for j in range(nt):
            sk, uk, sv, uv = j % nsk, j // nsk, j % nsv, j // nsv
            if uk > 0:
                yield ("wait", f"KEMPTY{sk}", uk - 1)
            yield ("tma", f"KFULL{sk}", T, Kr(sk))
            if uv > 0:
                yield ("wait", f"VEMPTY{sv}", uv - 1)
            yield ("tma", f"VFULL{sv}", T, Vr(sv))

    def issuer():
        yield ("wait", "QFULL", 0)
        yield ("wait", "KFULL0", 0)
        yield ("mma", [(0, T), Kr(0)], [], [Sc(0)], [])
        yield ("commit", "SFULL0")
        yield ("wait", "VFULL0", 0)
        yield ("mma", [(T, 2 * T), Vr(0)], [], [Gc], [])
        yield ("commit", "GFULL")
        yield ("commit", "VEMPTY0")
        if nt > 1:
            yield ("wait", "KFULL1", 0)
            yield ("mma", [(0, T), Kr(1)], [], [Sc(1)], [])
            yield ("commit", "SFULL1")
        for j in range(nt):
            b = j & 1
            yield ("wait", "GFREE", j)
            if j + 1 < nt:
                sv, uv = (j + 1) % nsv, (j + 1) // nsv
                yield ("wait", f"VFULL{sv}", uv)
                yield ("mma", [(T, 2 * T), Vr(sv)], [], [Gc], [])
                yield ("commit", "GFULL")
                yield ("commit", f"VEMPTY{sv}")
            yield ("wait", f"DSREADY{b}", j >> 1)
            yield ("mma", [Kr(j % nsk)], [Sc(b)], [DQc], [])
            yield ("commit", f"KEMPTY{j % nsk}")
            if j + 2 < nt:
                sk, uk = (j + 2) % nsk, (j + 2) // nsk
                yield ("wait", f"KFULL{sk}", uk)
                yield ("mma", [(0, T), Kr(sk)], [], [Sc(b)], [])
                yield ("commit", f"SFULL{b}")
        yield ("commit", "DQFULL")
        yield ("commit", "DONE")
        yield ("wait", "DONE", 0)

    def softmax():
        for j in range(nt):
            b = j & 1
            yield ("wait", f"SFULL{b}", j >> 1)
            yield ("wait", "GFULL", j)
            yield ("tread", Sc(b))
            yield ("tread", Gc)
            yield ("tdone", Gc)
            yield ("arrive", "GFREE", 256)
            yield ("tdone", Sc(b))  # dS written over the S buffer, then handed to dQ
            yield ("arrive", f"DSREADY{b}", 256)
        yield ("wait", "DQFULL", 0)
        yield ("tread", DQc)
        yield ("tdone", DQc)

    run_roles({"producer": producer(), "issuer": issuer(), "softmax": softmax()}, bars, rng)


TILES = [1, 2, 3, 4, 7, 12]


@pytest.mark.parametrize("stages", [(2, 1), (1, 1), (2, 2)], ids=["q2_do1", "q1_do1", "q2_do2"])
def test_dkdv_protocol_runs_clean_under_random_timing(stages):
    for nqt in TILES:
        for seed in range(25):
            dkdv_model(nqt, *stages, seed)


def test_dq_protocol_runs_clean_under_random_timing():
    for nt in TILES:
        for seed in range(25):
            dq_model(nt, seed)


@pytest.mark.parametrize("mistake,stages", [
    ("P written without PFREE", (2, 1)),
    ("S without SFREE", (2, 1)),
    ("dO first with two Q stages", (2, 1)),
    ("Q released before dK", (1, 1)),
])
def test_the_model_catches_planted_mistakes(mistake, stages):
    with pytest.raises(ProtocolError):
        for seed in range(40):
            dkdv_model(6, *stages, seed, mistake=mistake)
