"""The exchange of the sequence-parallel prefill (linear_attention_lm_gen_b200.seqpar),
run as gloo ranks on the CPU with the float64 oracle standing in for the
library's three calls:
  range pass  the oracle's whole mixer over the range from its start state
              (rank 0: the sequence's; the others: zero) with the previous
              range's last three V tokens as the conv history; the transition
              A is the oracle's state after the range started from the
              identity with zero values (the product of the transitions);
  compose     S*_1 = E_0, S*_{r+1} = S*_r A_r + E_r in float64;
  correct     adds the outputs that the start state alone produces (the oracle
              with zero values from S*), by joint linearity in (state, values).
Every rank's outputs, and the final state and history, must equal the oracle
run over the whole sequence. What is under test is the exchange: the halo,
who takes which start state, the gathers, the final state."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_ops(orc):
    import torch

    f = lambda t: None if t is None else t.numpy()

    class Ops:
        @staticmethod
        def range_pass(x, W1, W2, q, k, v, g, beta, hist_in, S0, first):
            r = orc.jetblock_prefill(f(x), f(W1), f(W2), f(q), f(k), f(v), f(g), f(beta), f(S0), f(hist_in))
            o, E = torch.from_numpy(r["o"]), torch.from_numpy(r["S"])
            if first:
                return o, E, None, None
            B, T, H, dk = q.shape
            eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
            _, A = orc.gdn_sequential(f(q), f(k), np.zeros((B, T, H, dk)), f(g), f(beta), eye)
            return o, E, torch.from_numpy(A), (f(q), f(k), f(g), f(beta))

        @staticmethod
        def compose(E_all, A_all):
            R = E_all.shape[0]
            S = [None, E_all[0]]
            for r in range(1, R):
                S.append(S[r] @ A_all[r] + E_all[r])
            return torch.stack([torch.zeros_like(E_all[0])] + S[1:R]), S[R]

        @staticmethod
        def correct(ctx, S_start, o):
            q, k, g, beta = ctx
            B, T, H, _ = q.shape
            add, _ = orc.gdn_sequential(q, k, np.zeros((B, T, H, S_start.shape[2])), g, beta, S_start.numpy())
            return o + torch.from_numpy(add)
    return Ops


def _rank_main(rank, world, port, bounds, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import synth
    from oracle import get as get_oracle
    from linear_attention_lm_gen_b200 import seqpar

    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    s = synth.JetShape("sp", B=2, T=bounds[-1], H=2, dk=8, dv=6, D=16, dtype="f32")
    inp = synth.prefill_inputs(s, seed=71, s0_std=0.3, gate_scale=0.05)
    hist = synth.jetblock._draw(np.random.default_rng(3), (2, 3, 2, 6), "f32")
    a, b = bounds[rank], bounds[rank + 1]
    t = lambda key: torch.from_numpy(np.ascontiguousarray(inp[key][:, a:b], dtype=np.float64))
    w = lambda key: torch.from_numpy(inp[key].astype(np.float64))
    o, S, h = seqpar.sequence_parallel_prefill(t("x"), w("W1"), w("W2"), t("q"), t("k"), t("v"), t("g"), t("beta"),
                                               S0=w("S0"), hist_in=torch.from_numpy(hist.astype(np.float64)),
                                               ops=oracle_ops(get_oracle()))
    dist.barrier()
    dist.destroy_process_group()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), o=o.numpy(), S=S.numpy(), h=h.numpy())


@pytest.mark.parametrize("bounds", [[0, 70, 150], [0, 40, 41 + 60, 140]])
def test_ranges_exchange_and_compose_to_the_whole_sequence(tmp_path, bounds):
    import synth
    from oracle import get as get_oracle
    world = len(bounds) - 1
    mp.start_processes(_rank_main, args=(world, _free_port(), bounds, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    s = synth.JetShape("sp", B=2, T=bounds[-1], H=2, dk=8, dv=6, D=16, dtype="f32")
    inp = synth.prefill_inputs(s, seed=71, s0_std=0.3, gate_scale=0.05)
    hist = synth.jetblock._draw(np.random.default_rng(3), (2, 3, 2, 6), "f32").astype(np.float64)
    d = {k: v.astype(np.float64) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ref = get_oracle().jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"],
                                        d["S0"], hist)
    for r in range(world):
        res = np.load(tmp_path / f"rank{r}.npz")
        np.testing.assert_allclose(res["o"], ref["o"][:, bounds[r]:bounds[r + 1]], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(res["S"], ref["S"], rtol=1e-9, atol=1e-11)      # every rank holds it
        np.testing.assert_array_equal(res["h"], ref["hist"])


def test_a_range_shorter_than_the_conv_reach_is_refused():
    import torch
    from linear_attention_lm_gen_b200 import seqpar
    z = torch.zeros
    with pytest.raises(ValueError):
        seqpar.sequence_parallel_prefill(z(1, 2, 8), z(8, 32), z(32, 4), z(1, 2, 1, 8), z(1, 2, 1, 8),
                                         z(1, 2, 1, 4), z(1, 2, 1), z(1, 2, 1), ops=None)
