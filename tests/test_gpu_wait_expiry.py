"""A bounded in-kernel wait that runs out, on the GPU, without faulting it.

Every mbarrier wait of the library is bounded in time (1 s in the library):
a waiter that gives up sets the device error word and raises its CTA's
abort flag, the other roles stop waiting, every role lets the copies and
tensor-core products it issued complete, and TMEM is freed; the host then
reads JET_ERR_TIMEOUT from jet_device_error and the context stays usable.

This test builds the library once more with two test-only definitions: a
2 ms wait limit, and a hook through which the load thread of the prefill
chain leaves out one product (P2a of chunk 1), so that the chain's wait for
it can never complete. It checks that the call returns, that the error word
says JET_ERR_TIMEOUT, and that the next call (hook off) and a call of the
library itself are correct. The hook exists only in that test build.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, gpu_inputs, host64, to_oracle
from oracle import get as get_oracle

pytestmark = pytest.mark.gpu

OK, TIMEOUT = 0, 5


@pytest.fixture(scope="module")
def libs(tmp_path_factory):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from linear_attention_lm_gen_b200 import build
    import linear_attention_lm_gen_b200 as jet
    build.build()
    jet.load_library()
    path = str(tmp_path_factory.mktemp("waittest") / "libjet_waittest.so")
    build.build(force=True, extra=["-DJET_TEST_WAIT_EXPIRY", "-DJET_WAIT_LIMIT_NS=2000000ull"], out=path)
    L = jet.declare(ctypes.CDLL(path))
    L.jet_test_skip_p2a.argtypes = [ctypes.c_int]
    L.jet_test_skip_p2a.restype = ctypes.c_int
    return jet, L


def call(L, d, o, S_out, ws, stream):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return L.jet_gdn_prefill(p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]), p(d["beta"]), None, p(o), p(S_out),
                             p(ws), ws.numel(), B, T, H, dk, dv, 64, 1, ctypes.c_void_p(stream))


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable(libs):
    jet, L = libs
    # two chunks of one (sequence, head): the tensor-core prefill in a single pass
    s = synth.JetShape("expiry", B=1, T=128, H=1, dk=64, dv=128, D=64)
    inp = synth.prefill_inputs(s, seed=61)
    d = gpu_inputs(inp)
    ws = torch.empty(jet.jet_gdn_prefill_workspace_size(1, s.T, 1, s.dk, s.dv), dtype=torch.uint8, device="cuda")
    o = torch.full_like(d["v"], float("nan"))
    S_out = torch.full((1, 1, s.dv, s.dk), float("nan"), device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    assert L.jet_test_skip_p2a(1) == 0
    assert call(L, d, o, S_out, ws, stream) == OK          # the launches themselves succeed
    t0 = time.time()
    assert L.jet_device_error(ctypes.c_void_p(stream)) == TIMEOUT
    assert time.time() - t0 < 10.0                          # a few 2 ms waits, not a hang
    assert L.jet_device_error(ctypes.c_void_p(stream)) == OK   # read and cleared
    # the same build with the hook off, then the library itself: both correct
    ref = to_oracle(inp)
    ro, rS = get_oracle().gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"])
    assert L.jet_test_skip_p2a(0) == 0
    o.fill_(float("nan"))
    assert call(L, d, o, S_out, ws, stream) == OK
    assert L.jet_device_error(ctypes.c_void_p(stream)) == OK
    assert_close(host64(o), ro, "bf16", "o after the timeout")
    assert_close(host64(S_out), rS, "bf16", "S after the timeout")
    o2, S2 = jet.jet_gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"])
    assert jet.jet_device_error() == OK
    assert_close(host64(o2), ro, "bf16", "o of the library")
    assert_close(host64(S2), rS, "bf16", "S of the library")
