"""The mbarrier protocol of the prefill state chain (csrc/k_prefill_chain.cuh),
checked as a model under random interleavings on the CPU.

Each role of the kernel is written out as the sequence of waits and
completions it performs, in the kernel's order:
  chain warps  per chunk c: wait P4(c-1) [and P5a(c-1)], wait the image; E4;
               (first thread) wait P2a(c), issue P3, wait P3(c), [wait
               P5b(c-1)]; E5; (first thread) wait K(c), issue P4; at the end
               wait P4(last)
  out warps    per chunk c (outputs only): wait P5b(c); read O -> arrive X2FREE
  load thread  prologue loads; P2a(0); per chunk c: the next V load once
               P2a(c) is done (V(c+2), or V(c+1) with the conv folded in, whose
               halo is the previous tile); wait P3(c): [P5a(c) after
               X2FREE(c-2)], P2a(c+1) after its image and V; wait P4(c):
               [P5b(c)], K and image
               loads once chunk c no longer reads their buffers
Loads and MMA commit groups complete after random delays (each issuer's
groups in order). A waiter of phase n is released when the barrier has
completed n + 1 phases; seeing n + 2 would make its parity wait ambiguous.
The model checks: no deadlock, no waiter two phases behind, every issued
operation completes, and (folded conv) no V load overwrites a tile while a
later P2a still needs it as its halo.
"""
import random

import pytest


def run(nch, nkbuf, write_o, conv, seed, mutant=None, patience=None):
    """One random interleaving; raises AssertionError on a protocol fault.
    mutant (for the tests of the model itself): "plain_v" keeps the two-ahead
    V schedule of plain V with the conv folded in; "one_p2" shares a single
    P2a barrier between the two V buffers; "e4_early" lets E4 start without
    waiting for the previous chunk's P5a; "skip_p2a1" leaves out P2a of
    chunk 1 (the test build's hook), with `patience` the number of rounds a
    wait may block before it gives up and raises the abort flag (after which
    every blocked wait gives up). Returns whether the abort flag was raised."""
    plain_v = not conv or mutant == "plain_v"
    p2 = (lambda c: ("P2", 0)) if mutant == "one_p2" else (lambda c: ("P2", c & 1))
    p2n = (lambda c: c) if mutant == "one_p2" else (lambda c: c >> 1)
    rng = random.Random(seed)
    comp = {}
    C = lambda b: comp.get(b, 0)
    pending, mq = [], {"M": [], "L": [], "O": []}
    last_v = {0: None, 1: None}          # buffer -> chunk of the last V load issued into it
    nv = [0]

    def load(bar):
        if bar[0] == "V":
            last_v[bar[1]] = nv[0]
            nv[0] += 1
        pending.append([rng.randint(1, 8), bar])

    def mma(who, bar):
        mq[who].append([rng.randint(1, 4), bar])

    def chain():
        for c in range(nch):
            if c >= 1:
                yield ("SD", (c - 1) & 1), (c - 1) >> 1
                if write_o and mutant != "e4_early":
                    yield ("PA", (c - 1) & 1), (c - 1) >> 1
            yield ("IMG", c & 1), c >> 1
            if write_o and c >= 1:   # E4 overwrites the S copy that P5a(c-1) reads
                assert C(("PA", (c - 1) & 1)) > (c - 1) >> 1, f"S copy of chunk {c - 1} overwritten"
            yield p2(c), p2n(c)
            mma("M", ("P3",))
            yield ("P3",), c
            if write_o and c >= 1:
                yield ("OD", (c - 1) & 1), (c - 1) >> 1
                # E5 overwrites the Wt^T copy that P5b(c-1) reads
                assert C(("OD", (c - 1) & 1)) > (c - 1) >> 1, f"Wt copy of chunk {c - 1} overwritten"
            yield ("K", c % nkbuf), c // nkbuf
            mma("M", ("SD", c & 1))
        if nch:
            yield ("SD", (nch - 1) & 1), (nch - 1) >> 1

    def out():
        for c in range(nch if write_o else 0):
            yield ("OD", c & 1), c >> 1
            comp[("X2F", c & 1)] = C(("X2F", c & 1)) + 1

    def loader():
        if nch == 0:
            return
        load(("IMG", 0)); load(("V", 0)); load(("K", 0))
        if conv:
            load(("H0",))
        if nch > 1:
            load(("IMG", 1))
            if plain_v:
                load(("V", 1))
        if nkbuf == 2 and nch > 1:
            load(("K", 1))
        yield ("IMG", 0), 0
        yield ("V", 0), 0
        if conv:
            yield ("H0",), 0
        mma("L", p2(0))
        for c in range(nch):
            ahead = 2 if plain_v else 1
            if c + ahead < nch:
                yield p2(c), p2n(c)
                load(("V", (c + ahead) & 1))
            yield ("P3",), c
            if write_o:
                if c >= 2:
                    yield ("X2F", c & 1), (c - 2) >> 1
                mma("L", ("PA", c & 1))
            if c + 1 < nch:
                yield ("IMG", (c + 1) & 1), (c + 1) >> 1
                yield ("V", (c + 1) & 1), (c + 1) >> 1
                if conv:   # the halo of P2a(c+1) is V(c): still the last load into its buffer
                    assert last_v[c & 1] == c, f"halo of chunk {c + 1} overwritten"
                if not (mutant == "skip_p2a1" and c == 0):
                    mma("L", p2(c + 1))
            yield ("SD", c & 1), c >> 1
            if write_o:
                mma("L", ("OD", c & 1))
            if c + nkbuf < nch or c + 2 < nch:
                if write_o:
                    yield ("OD", c & 1), c >> 1
                if c + nkbuf < nch:
                    load(("K", (c + nkbuf) % nkbuf))
                if c + 2 < nch:
                    load(("IMG", (c + 2) & 1))

    roles = {"chain": chain(), "out": out(), "load": loader()}
    cur = dict.fromkeys(roles)
    slow = {k: rng.choice([0.0, 0.5, 0.9, 0.97]) for k in roles}
    done = set()
    blocked = dict.fromkeys(roles, 0)
    abort = False
    for _ in range(200000):
        if len(done) == len(roles) and not pending and not any(mq.values()):
            break
        moved = False
        for k in rng.sample(list(roles), len(roles)):
            if k in done:
                continue
            if rng.random() < slow[k]:
                moved = True
                continue
            if cur[k] is None:
                try:
                    cur[k] = next(roles[k])
                except StopIteration:
                    done.add(k)
                moved = True
                continue
            bar, n = cur[k]
            assert C(bar) < n + 2, f"{k} waits phase {n} of {bar} after {C(bar)} completions"
            if C(bar) == n + 1:
                cur[k] = None
                blocked[k] = 0
                moved = True
            elif patience is not None:
                blocked[k] += 1                        # time passes for a bounded wait
                moved = True
                if abort or blocked[k] > patience:     # the bounded wait gives up; the role winds down
                    abort = True
                    roles[k].close()
                    done.add(k)
                    moved = True
        for p in pending:
            p[0] -= 1
        for p in [p for p in pending if p[0] <= 0]:
            comp[p[1]] = C(p[1]) + 1
            pending.remove(p)
            moved = True
        for who in ("M", "L", "O"):
            q = mq[who]
            if q and rng.random() < 0.7:
                q[0][0] -= 1
                if q[0][0] <= 0:
                    b = q.pop(0)[1]
                    comp[b] = C(b) + 1
                    moved = True
        assert moved or pending or any(mq.values()), f"deadlock: {cur}"
    else:
        raise AssertionError("no progress within the step budget")
    assert not pending and not any(mq.values()), "operations left in flight"
    return abort


@pytest.mark.parametrize("conv", [False, True])
@pytest.mark.parametrize("write_o", [False, True])
@pytest.mark.parametrize("nkbuf", [1, 2])
def test_chain_protocol_has_no_deadlock_and_no_two_phase_lag(conv, write_o, nkbuf):
    for nch in range(0, 10):
        for seed in range(40):
            run(nch, nkbuf, write_o, conv, seed)


def test_the_model_catches_a_halo_overwrite():
    # with the folded conv, the plain two-ahead V schedule would overwrite the tile that the
    # next P2a still reads as its halo: the model must see it
    with pytest.raises(AssertionError, match="halo"):
        for seed in range(200):
            run(6, 2, False, True, seed, mutant="plain_v")


def test_the_model_catches_an_early_overwrite():
    # E4 of chunk c+1 rewrites the bf16 S copy: starting it before P5a(c) has read the copy
    # (dropping that wait) must be caught
    with pytest.raises(AssertionError, match="overwritten"):
        for seed in range(300):
            run(8, 2, True, False, seed, mutant="e4_early")


@pytest.mark.parametrize("conv", [False, True])
@pytest.mark.parametrize("nkbuf", [1, 2])
def test_a_missing_product_ends_in_a_wind_down(conv, nkbuf):
    # the GPU test build's hook leaves out P2a of chunk 1: with bounded waits the chain's
    # wait runs out, the abort reaches every role, and every issued copy and product still
    # completes (what the roles' drains wait for before TMEM is freed)
    for nch in (2, 3, 5):
        for seed in range(40):
            assert run(nch, nkbuf, True, conv, seed, mutant="skip_p2a1", patience=60)
    # with nothing left out, the same bounded waits never give up
    for seed in range(40):
        assert not run(5, nkbuf, True, conv, seed, patience=100000)
