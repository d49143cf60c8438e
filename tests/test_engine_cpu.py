"""Host logic of the serving loop (linear_attention_lm_gen_b200.engine): pool
entries, chunked-prefill pieces and the calls it makes, checked on the CPU
with recording stand-ins for the two library calls (no kernel runs here)."""
import pytest
import torch

from linear_attention_lm_gen_b200 import engine as eng

H, DK, DV, D = 2, 16, 32, 64


class Calls:
    def __init__(self):
        self.prefill, self.decode = [], []

    def fake_prefill(self, x, W1, W2, q, k, v, g, beta, hist_in, hist_out, S0, o, S_out, workspace):
        T = x.shape[1]
        assert S0 is S_out or S0.data_ptr() == S_out.data_ptr()          # the state advances in place
        assert hist_out.data_ptr() != hist_in.data_ptr()                  # new history into a separate buffer
        self.prefill.append((T, S0.data_ptr(), hist_in.data_ptr()))
        hist_out.copy_(hist_in + 1)                                       # marks: one per piece
        S_out.add_(T)
        return torch.full((1, T, H, DV), float(len(self.prefill))), S_out

    def fake_decode(self, x, W1, W2, q, k, v, g, beta, hist_pool, S_pool, slots):
        self.decode.append(slots.tolist())
        for b, s in enumerate(slots.tolist()):
            S_pool[s] += 1000
        return torch.zeros((x.shape[0], H, DV))


@pytest.fixture
def engine(monkeypatch):
    c = Calls()
    monkeypatch.setattr(eng, "jet_jetblock_prefill", c.fake_prefill)
    monkeypatch.setattr(eng, "jet_jetblock_decode_slots", c.fake_decode)
    monkeypatch.setattr(eng, "jet_jetblock_prefill_workspace_size", lambda *a, **k: 64)
    e = eng.JetEngine(torch.zeros(D, 32), torch.zeros(32, 4 * H), H, DK, DV, max_seqs=3, chunk_tokens=128)
    return e, c


def prompt(T):
    return (torch.zeros(T, D), torch.zeros(T, H, DK), torch.zeros(T, H, DK), torch.zeros(T, H, DV),
            torch.zeros(T, H), torch.zeros(T, H))


def test_pool_entries_are_handed_out_and_reused(engine):
    e, _ = engine
    assert [e.admit(s) for s in ("a", "b", "c")] == [0, 1, 2]
    with pytest.raises(RuntimeError):
        e.admit("d")
    with pytest.raises(KeyError):
        e.admit("a")
    e.S[1].fill_(5.0)
    e.hist[1].fill_(3.0)
    e.release("b")
    assert e.free_slots == 1
    assert e.admit("d") == 1
    assert float(e.S[1].abs().sum()) == 0.0 and float(e.hist[1].abs().sum()) == 0.0   # a fresh sequence


def test_prefill_runs_in_pieces_that_continue_the_state(engine):
    e, c = engine
    e.admit("a")
    s = e.admit("b")
    assert e.pieces(333) == [(0, 128), (128, 256), (256, 333)]
    o = e.prefill("b", *prompt(333))
    assert [t for t, _, _ in c.prefill] == [128, 128, 77]
    assert all(p == e.S[s].data_ptr() for _, p, _ in c.prefill)          # every piece on the same entry
    assert all(h == e.hist[s].data_ptr() for _, _, h in c.prefill)
    assert o.shape == (333, H, DV)
    assert torch.equal(o[:128], torch.full((128, H, DV), 1.0)) and torch.equal(o[256:], torch.full((77, H, DV), 3.0))
    assert float(e.S[s].flatten()[0]) == 333.0                             # each piece continued the last
    assert float(e.hist[s].flatten()[0]) == 3.0                            # history carried piece to piece
    assert float(e.S[0].abs().sum()) == 0.0                                # other entries untouched
    assert e.pos["b"] == 333


def test_decode_batches_by_pool_entry(engine):
    e, c = engine
    for s in ("a", "b", "c"):
        e.admit(s)
    e.release("a")
    e.admit("d")                                                           # takes entry 0 again
    e.decode(["c", "d", "b"], torch.zeros(3, D), torch.zeros(3, H, DK), torch.zeros(3, H, DK),
             torch.zeros(3, H, DV), torch.zeros(3, H), torch.zeros(3, H))
    assert c.decode == [[2, 0, 1]]
    assert e.pos == {"b": 1, "c": 1, "d": 1}
    with pytest.raises(ValueError):
        e.decode(["b", "b"], torch.zeros(2, D), torch.zeros(2, H, DK), torch.zeros(2, H, DK), torch.zeros(2, H, DV),
                 torch.zeros(2, H), torch.zeros(2, H))


# ---------------------------------------------------------------- batched chunked prefill, numerically
# The library call is stood in for by the float64 oracle of the whole mixer
# (with initial state and history), so the test checks that the engine's
# rounds, groups, gathers and scatters continue every sequence correctly.
def oracle_prefill(orc, calls):
    def run(x, W1, W2, q, k, v, g, beta, hist_in, hist_out, S0, o, S_out, workspace):
        n = lambda t: t.double().numpy()
        r = orc.jetblock_prefill(n(x), n(W1), n(W2), n(q), n(k), n(v), n(g), n(beta), n(S0), n(hist_in))
        calls.append(tuple(x.shape[:2]))
        S_out.copy_(torch.from_numpy(r["S"]))
        hist_out.copy_(torch.from_numpy(r["hist"]))
        return torch.from_numpy(r["o"]), S_out
    return run


def test_prefill_many_batches_equal_pieces_and_continues_every_sequence(monkeypatch):
    import numpy as np
    import synth
    from oracle import get as get_oracle
    orc = get_oracle()
    calls = []
    monkeypatch.setattr(eng, "jet_jetblock_prefill", oracle_prefill(orc, calls))
    monkeypatch.setattr(eng, "jet_jetblock_prefill_workspace_size", lambda *a, **k: 64)
    shp = synth.JetShape("t", B=1, T=1, H=H, dk=DK, dv=DV, D=D, dtype="f32")
    lens = {"a": 300, "b": 300, "c": 77}
    inp = {n: synth.prefill_inputs(shp, seed=30 + i, T=T) for i, (n, T) in enumerate(lens.items())}
    W1 = torch.from_numpy(inp["a"]["W1"]).double()
    W2 = torch.from_numpy(inp["a"]["W2"]).double()
    e = eng.JetEngine(W1, W2, H, DK, DV, max_seqs=4, chunk_tokens=128)
    for n in ("c", "a", "b"):
        e.admit(n)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a[0])).double()
    outs = e.prefill_many({n: tuple(t(inp[n][k]) for k in ("x", "q", "k", "v", "g", "beta")) for n in lens})
    # rounds: (a, b) full + (c) tail; (a, b) full; (a, b) tails of 44
    assert calls == [(2, 128), (1, 77), (2, 128), (2, 44)]
    for n, T in lens.items():
        d = {k: inp[n][k].astype(np.float64) for k in ("x", "q", "k", "v", "g", "beta")}
        r = orc.jetblock_prefill(d["x"], inp["a"]["W1"].astype(np.float64), inp["a"]["W2"].astype(np.float64),
                                 d["q"], d["k"], d["v"], d["g"], d["beta"])
        np.testing.assert_allclose(outs[n].numpy(), r["o"][0], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(e.S[e.slot[n]].double().numpy(), r["S"][0], rtol=1e-5, atol=1e-5)
        np.testing.assert_array_equal(e.hist[e.slot[n]].numpy(), r["hist"][0])
        assert e.pos[n] == T


def oracle_decode(orc):
    def run(x, W1, W2, q, k, v, g, beta, hist_pool, S_pool, slots):
        n = lambda t: t.double().numpy()
        idx = slots.long()
        r = orc.jetblock_decode(n(x)[None], n(W1), n(W2), n(q)[None], n(k)[None], n(v)[None], n(g)[None],
                                n(beta)[None], n(S_pool[idx]), n(hist_pool[idx]))
        S_pool[idx] = torch.from_numpy(r["S"]).to(S_pool.dtype)
        hist_pool[idx] = torch.from_numpy(r["hist"]).to(hist_pool.dtype)
        return torch.from_numpy(r["o"][0])
    return run


def test_serving_steps_spend_the_prefill_budget_and_decode_finished_prompts(monkeypatch):
    import numpy as np
    import synth
    from oracle import get as get_oracle
    orc = get_oracle()
    calls = []
    monkeypatch.setattr(eng, "jet_jetblock_prefill", oracle_prefill(orc, calls))
    monkeypatch.setattr(eng, "jet_jetblock_decode_slots", oracle_decode(orc))
    monkeypatch.setattr(eng, "jet_jetblock_prefill_workspace_size", lambda *a, **k: 64)
    shp = synth.JetShape("t", B=1, T=1, H=H, dk=DK, dv=DV, D=D, dtype="f32")
    lens, dec = {"a": 250, "b": 60}, 3
    inp = {n: synth.prefill_inputs(shp, seed=50 + i, T=T + dec) for i, (n, T) in enumerate(lens.items())}
    W1 = torch.from_numpy(inp["a"]["W1"]).double()
    W2 = torch.from_numpy(inp["a"]["W2"]).double()
    e = eng.JetEngine(W1, W2, H, DK, DV, max_seqs=2, chunk_tokens=100)
    t = lambda n, a, b: tuple(torch.from_numpy(np.ascontiguousarray(inp[n][k][0, a:b])).double()
                              for k in ("x", "q", "k", "v", "g", "beta"))
    for n, T in lens.items():
        e.submit(n, t(n, 0, T))
    outs = {n: [] for n in lens}
    tok = lambda n, i: tuple(a[0] for a in t(n, i, i + 1))
    with pytest.raises(ValueError):
        e.step({"b": tok("b", 60)})                        # b has not finished its prompt: nothing runs
    assert calls == [] and e.pos == {"a": 0, "b": 0} and float(e.S.abs().sum()) == 0.0
    plan = [None, None, None, {"a": 250}, {"a": 251, "b": 60}, {"a": 252, "b": 61}, {"b": 62}]
    for want in plan:
        r = e.step({n: tok(n, i) for n, i in want.items()} if want else None)
        for n, o in r.items():
            outs[n].append(o if o.dim() == 3 else o[None])
    # prefill budget: a 100 | a 100 | a 50 + b 50 | b 10 (then decode a) | decode | decode | decode b
    assert calls == [(1, 100), (1, 100), (2, 50), (1, 10)]
    assert e.prefilling == []
    for n, T in lens.items():
        d = {k: inp[n][k].astype(np.float64) for k in ("x", "q", "k", "v", "g", "beta")}
        r = orc.jetblock_prefill(d["x"], inp["a"]["W1"].astype(np.float64), inp["a"]["W2"].astype(np.float64),
                                 d["q"], d["k"], d["v"], d["g"], d["beta"])
        np.testing.assert_allclose(torch.cat(outs[n]).numpy(), r["o"][0], rtol=1e-5, atol=1e-5)
        assert e.pos[n] == T + dec


def test_step_checks_every_input_before_any_work(engine):
    e, c = engine
    e.submit("a", prompt(40))
    one = tuple(a[0] for a in prompt(1))
    S_before = e.S.clone()
    with pytest.raises(KeyError):                 # a decode token for a sequence never admitted
        e.step({"ghost": one})
    assert c.prefill == [] and c.decode == [] and e.prefilling == ["a"] and e.pos["a"] == 0
    assert torch.equal(e.S, S_before)
    e.step()                                       # the prompt (40 <= 128 tokens) finishes
    e.release("a")
    with pytest.raises(KeyError):                 # ... or one already released
        e.step({"a": one})
    with pytest.raises(KeyError):
        e.decode(["a"], *[a[None] for a in one])
    assert c.decode == []


def test_submit_rejects_empty_and_ragged_prompts(engine):
    e, _ = engine
    with pytest.raises(ValueError):
        e.submit("empty", prompt(0))
    ragged = prompt(5)[:5] + (torch.zeros(4, H),)
    with pytest.raises(ValueError):
        e.submit("ragged", ragged)
    assert e.free_slots == 3 and e.prefilling == []


def test_prefill_many_packs_every_piece_of_a_round_into_one_call(monkeypatch):
    # bf16 tensor-core shapes: each round is one variable-length call over all live sequences
    calls = []

    def fake_varlen(x, W1, W2, q, k, v, g, beta, cu, hist_in, hist_out, S0, o, S_out):
        calls.append(list(cu))
        assert S0.data_ptr() == S_out.data_ptr()
        hist_out.copy_(hist_in + 1)
        for i in range(len(cu) - 1):
            S_out[i] += cu[i + 1] - cu[i]
        return torch.full((cu[-1], 2, 128), float(len(calls))), S_out
    monkeypatch.setattr(eng, "jet_jetblock_prefill_varlen", fake_varlen)
    bf = torch.bfloat16
    e = eng.JetEngine(torch.zeros(64, 32, dtype=bf), torch.zeros(32, 8, dtype=bf), 2, 64, 128, max_seqs=4,
                      chunk_tokens=100)
    assert e.varlen
    lens = {"a": 250, "b": 60, "c": 100}
    for sq in lens:
        e.admit(sq)
    p = lambda T: (torch.zeros(T, 64), torch.zeros(T, 2, 64), torch.zeros(T, 2, 64), torch.zeros(T, 2, 128),
                   torch.zeros(T, 2), torch.zeros(T, 2))
    out = e.prefill_many({sq: p(T) for sq, T in lens.items()})
    # round 0: a 100, b 60, c 100; round 1: a 100; round 2: a 50
    assert calls == [[0, 100, 160, 260], [0, 100], [0, 50]]
    assert {sq: o.shape[0] for sq, o in out.items()} == lens
    assert e.pos == lens
    for sq, T in lens.items():
        assert float(e.S[e.slot[sq]].flatten()[0]) == T            # every piece advanced its own state
        rounds = (T + 99) // 100
        assert float(e.hist[e.slot[sq]].flatten()[0]) == rounds    # and its own history, once per round
