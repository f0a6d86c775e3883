"""Runtime behaviour on the GPU: the failure path of the bounded waits, and
capture of fd_decode into a CUDA graph."""
import time

import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import OnDevice, assert_close, dev_bf16, host_bf16, reference, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_the_context_survives(cuda_device):
    assert fd.fd_check_device_error() == fd.FD_OK
    t0 = time.time()
    assert fd.fd_selftest_device_timeout(50_000) == fd.FD_OK  # 50 ms wait on nothing
    assert fd.fd_check_device_error() == fd.FD_ERR_DEVICE_TIMEOUT
    assert time.time() - t0 < 10.0
    assert fd.fd_check_device_error() == fd.FD_OK  # the word was cleared
    # the context still decodes correctly
    w = wl.make_problem(2, 16, 2, 128, 700, seed=31, seqlens=[700, 129])
    got, gl, _ = run_gpu(OnDevice(w), 3)
    ref, rl = reference(w)
    assert_close(got, gl, ref, rl, "after timeout")


def test_selftest_rejects_out_of_range_limits(cuda_device):
    assert fd.fd_selftest_device_timeout(0) == fd.FD_ERR_INVALID_ARGUMENT
    assert fd.fd_selftest_device_timeout(10_000_000) == fd.FD_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("S", [1, 5, 24])
def test_cuda_graph_capture_and_replay(cuda_device, S):
    import torch
    w = wl.make_problem(2, 16, 2, 128, 3000, seed=32, seqlens=[3000, 1111])
    d = OnDevice(w)
    prob = d.problem()
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, S)
    ws = torch.empty(max(nbytes, 4) // 4, dtype=torch.float32, device="cuda")

    def call():
        st = fd.fd_decode(prob, d.q, d.k, d.v, d.seqlens, None, w.scale, S, out, lse, ws, nbytes)
        assert st == fd.FD_OK

    call()  # eager call first: the library's one-time set-up happens outside the capture
    torch.cuda.synchronize()
    eager_out, eager_lse = out.clone(), lse.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager_out) and torch.equal(lse, eager_lse)
    # new query values in the same buffer: a replay recomputes
    w2 = wl.make_problem(2, 16, 2, 128, 3000, seed=33, seqlens=[3000, 1111])
    d.q.copy_(dev_bf16(w2.q))
    g.replay()
    torch.cuda.synchronize()
    w.q = w2.q
    ref, rl = reference(w)
    assert_close(host_bf16(out), lse.cpu().numpy().astype(np.float64), ref, rl, "graph replay")
    assert fd.fd_check_device_error() == fd.FD_OK
