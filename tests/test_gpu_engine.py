"""GPU: decode over a state cache (jet_jetblock_decode_slots) and the
chunked-prefill serving loop (engine.JetEngine), against the batched calls
and the float64 oracle."""
import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, dev, gpu_inputs, host64, to_oracle
from oracle import get as get_oracle

pytestmark = pytest.mark.gpu

jet = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global jet
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from linear_attention_lm_gen_b200 import build
    build.build()
    import linear_attention_lm_gen_b200 as m
    m.load_library()
    jet = m
    yield
    assert m.jet_device_error() == 0


@pytest.mark.parametrize("dtype,H,dk,dv", [("bf16", 12, 96, 256), ("f32", 2, 16, 32), ("bf16", 3, 128, 64)])
def test_decode_slots_equals_the_batched_calls(dtype, H, dk, dv):
    # pool of 7 entries, 4 sequences on entries 5, 0, 3, 6: the same kernels with an index, so bit-exact
    N, slots = 7, [5, 0, 3, 6]
    s = synth.JetShape("t", B=len(slots), T=1, H=H, dk=dk, dv=dv, D=64, dtype=dtype)
    inp = synth.decode_inputs(s, seed=13, steps=3)
    d = gpu_inputs(inp)
    g = torch.Generator(device="cpu").manual_seed(3)
    S_pool = (torch.randn((N, H, dv, dk), generator=g) * 0.02).cuda()
    hist_pool = torch.randn((N, 3, H, dv), generator=g).to(d["v"].dtype).cuda()
    S_ref, hist_ref = S_pool.clone(), hist_pool.clone()
    idx = torch.tensor(slots, dtype=torch.int32, device="cuda")
    for t in range(3):
        o = jet.jet_jetblock_decode_slots(d["x"][t], d["W1"], d["W2"], d["q"][t], d["k"][t], d["v"][t], d["g"][t],
                                          d["beta"][t], hist_pool, S_pool, idx)
        # reference: gather the entries, the two batched calls, scatter back
        il = idx.long()
        Sb, hb = S_ref[il].contiguous(), hist_ref[il].contiguous()
        hn = torch.empty_like(hb)
        vc, _ = jet.jet_dyn_conv_v(d["x"][t][:, None], d["W1"], d["W2"], d["v"][t][:, None], hb, None, hn)
        o_ref = jet.jet_gdn_decode_step(d["q"][t], d["k"][t], vc[:, 0], d["g"][t], d["beta"][t], Sb)
        S_ref[il], hist_ref[il] = Sb, hn
        assert torch.equal(o, o_ref)
        assert torch.equal(S_pool, S_ref)          # entries not in the batch untouched as well
        assert torch.equal(hist_pool, hist_ref)
    assert jet.jet_device_error() == 0


def test_decode_slots_out_of_range_entry_is_reported_and_skipped():
    # the kernels check every index before they use it: a bad one sets the error word and is skipped
    N, H, dk, dv = 4, 2, 16, 32
    s = synth.JetShape("t", B=2, T=1, H=H, dk=dk, dv=dv, D=64, dtype="bf16")
    inp = synth.decode_inputs(s, seed=14, steps=1)
    d = gpu_inputs(inp)
    S_pool = torch.full((N, H, dv, dk), 0.5, device="cuda")
    hist_pool = torch.ones((N, 3, H, dv), device="cuda", dtype=torch.bfloat16)
    before_S, before_h = S_pool.clone(), hist_pool.clone()
    o = torch.full((2, H, dv), float("nan"), device="cuda", dtype=torch.bfloat16)
    idx = torch.tensor([1, N], dtype=torch.int32, device="cuda")      # entry N does not exist
    jet.jet_jetblock_decode_slots(d["x"][0], d["W1"], d["W2"], d["q"][0], d["k"][0], d["v"][0], d["g"][0],
                                  d["beta"][0], hist_pool, S_pool, idx, o)
    assert jet.jet_device_error() == 6                                # JET_ERR_DEVICE, and cleared
    assert not torch.equal(S_pool[1], before_S[1])                    # the valid sequence ran
    for e in (0, 2, 3):
        assert torch.equal(S_pool[e], before_S[e]) and torch.equal(hist_pool[e], before_h[e])
    assert torch.isnan(o[1].float()).all()                            # nothing written for the bad one
    assert jet.jet_device_error() == 0


@pytest.mark.parametrize("dtype,H,dk,dv,D,chunk", [("bf16", 12, 96, 256, 1536, 128), ("f32", 2, 16, 32, 64, 64)])
def test_engine_chunked_prefill_then_decode_matches_the_oracle(dtype, H, dk, dv, D, chunk):
    from linear_attention_lm_gen_b200.engine import JetEngine
    orc = get_oracle()
    lens, steps = {"a": 150, "b": 70, "c": 333}, 4
    shp = synth.JetShape("t", B=1, T=1, H=H, dk=dk, dv=dv, D=D, dtype=dtype)
    seqs = {n: synth.prefill_inputs(shp, seed=20 + i, T=T + steps) for i, (n, T) in enumerate(lens.items())}
    W = gpu_inputs(seqs["a"])                          # every sequence shares the weights of seed 20
    for n in seqs:
        seqs[n]["W1"], seqs[n]["W2"] = seqs["a"]["W1"], seqs["a"]["W2"]
    e = JetEngine(W["W1"], W["W2"], H, dk, dv, max_seqs=5, chunk_tokens=chunk)
    e.admit("x")                                       # occupy an entry, then free it: the pool is not in order
    for n in lens:
        e.admit(n)
    e.release("x")
    outs = {}
    for n, T in lens.items():                          # chunked prefill of each prompt
        d = gpu_inputs(seqs[n])
        outs[n] = [e.prefill(n, *(d[k_][0, :T] for k_ in ("x", "q", "k", "v", "g", "beta")))]
    order = ["c", "a", "b"]
    for t in range(steps):                             # batched decode, all three sequences
        toks = {n: gpu_inputs(seqs[n]) for n in order}
        pick = lambda k_: torch.stack([toks[n][k_][0, lens[n] + t] for n in order])
        o = e.decode(order, pick("x"), pick("q"), pick("k"), pick("v"), pick("g"), pick("beta"))
        for i, n in enumerate(order):
            outs[n].append(o[i:i + 1])
    for n, T in lens.items():
        ref = to_oracle(seqs[n])
        r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"])
        assert_close(host64(torch.cat(outs[n])), r["o"][0], dtype, f"{n} o")
        assert_close(host64(e.S[e.slot[n]]), r["S"][0], dtype, f"{n} S")
        np.testing.assert_array_equal(host64(e.hist[e.slot[n]]), r["hist"][0])
        assert e.pos[n] == T + steps


def test_engine_batched_prefill_matches_the_oracle():
    # prompts of 300, 300 and 77 tokens in 128-token pieces: equal pieces share one batched call
    from linear_attention_lm_gen_b200.engine import JetEngine
    orc = get_oracle()
    H, dk, dv, D = 12, 96, 256, 1536
    lens = {"a": 300, "b": 300, "c": 77}
    shp = synth.JetShape("t", B=1, T=1, H=H, dk=dk, dv=dv, D=D, dtype="bf16")
    seqs = {n: synth.prefill_inputs(shp, seed=40 + i, T=T) for i, (n, T) in enumerate(lens.items())}
    for n in seqs:
        seqs[n]["W1"], seqs[n]["W2"] = seqs["a"]["W1"], seqs["a"]["W2"]
    W = gpu_inputs(seqs["a"])
    e = JetEngine(W["W1"], W["W2"], H, dk, dv, max_seqs=4, chunk_tokens=128)
    for n in ("b", "c", "a"):
        e.admit(n)
    prompts = {}
    for n in lens:
        d = gpu_inputs(seqs[n])
        prompts[n] = tuple(d[k_][0] for k_ in ("x", "q", "k", "v", "g", "beta"))
    outs = e.prefill_many(prompts)
    for n in lens:
        ref = to_oracle(seqs[n])
        r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"])
        assert_close(host64(outs[n]), r["o"][0], "bf16", f"{n} o")
        assert_close(host64(e.S[e.slot[n]]), r["S"][0], "bf16", f"{n} S")
        np.testing.assert_array_equal(host64(e.hist[e.slot[n]]), r["hist"][0])
