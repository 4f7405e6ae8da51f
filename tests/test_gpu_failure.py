"""Failure detection on the GPU without a fault: a bounded wait whose
condition never comes true gives up, records UW_ERR_TIMEOUT and returns; the
context stays usable (a GEMM right after is correct)."""
import time

import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import device_matrix, empty_bf16, gemm_ref, to_dev, to_host_u16, within_tol

pytestmark = pytest.mark.gpu


def test_bounded_waits_time_out_and_the_context_stays_usable():
    import torch
    ws = uw.Workspace(4096)
    t0 = time.time()
    uw.selftest_bounded_wait(ws, 20000)  # 20 ms per wait
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert ws.status() == uw.UW_ERR_TIMEOUT
    words = ws.t[64:76].cpu().numpy().view(np.uint32)
    assert list(words) == [0, 0, 0]  # both waits gave up; the counter stayed 0
    assert 0.03 < elapsed < 5.0      # two 20 ms limits, not a hang
    assert ws.status() == uw.UW_OK   # reading the status cleared it

    w = synth.weight_matrix(256, 512, 0.02, 5e-4, 200.0, 0)
    x = synth.activations(4, 512, 1)
    dm = device_matrix(w)
    ws2 = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 4))
    y = empty_bf16(4, 256)
    uw.gemm(dm, uw.PIPE_DIRECT, to_dev(x), y, ws2)
    ws2.check("gemm after the timeout self-test")
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x))
    assert ok, (err, rms)


def test_selftest_argument_errors():
    ws = uw.Workspace(4096)
    for bad in (0, 1000001):
        assert uw.lib().uw_selftest_bounded_wait(ws.ptr, ws.nbytes, bad, None) == uw.UW_ERR_INVALID_ARG
    assert uw.lib().uw_selftest_bounded_wait(ws.ptr, 128, 1000, None) == uw.UW_ERR_INVALID_ARG


def test_failed_call_leaves_a_workspace_the_next_call_can_use():
    """A call that gives up part way may leave split-K tile counters raised.
    Reading its status re-zeroes the workspace, so the next split-K GEMM on
    it is correct.  (The failure is made on the host: raised counters and a
    status word written into the workspace.)"""
    w = synth.weight_matrix(1024, 4096, 0.02, 1e-4, 100.0, 60)
    x_host = synth.activations(8, 4096, 61)
    dm = device_matrix(w)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8))
    ws.t[256:256 + 64] = 7                      # stale tile counters
    ws.t[0:4] = torch_u8([uw.UW_ERR_TIMEOUT, 0, 0, 0])
    assert ws.status() == uw.UW_ERR_TIMEOUT
    assert int(ws.t[256:256 + 64].sum()) == 0
    y = empty_bf16(8, 1024)
    uw.gemm_direct_palette(dm, to_dev(x_host), y, ws)
    ws.check("after recovery")
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x_host))
    assert ok, (err, rms)


def torch_u8(vals):
    import torch
    return torch.tensor(vals, dtype=torch.uint8, device="cuda")
