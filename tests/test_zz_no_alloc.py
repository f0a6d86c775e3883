"""fd_decode_static_workspace: decode attention for callers that cannot
allocate device memory.

Some callers cannot call cudaMalloc. Examples: a plain C host that links only
this library and has no device allocator of its own; code inside a framework
whose memory pool owns all device memory; a decode loop that must not block or
fail on an allocation mid-step. This entry point takes the same inputs and
outputs as fd_decode. Its scratch is the library's static device array
(FD_STATIC_WORKSPACE_BYTES), so the caller allocates nothing. The test calls
it twice in a row through the C ABI. Each result must equal fd_decode's with a
caller-allocated workspace bit for bit (same split count, same kernels, no
atomics in the data path), and must match the fp64 oracle within the
tolerances of the other parity tests. This file sorts last so that a run
stopping at the first failure has already run every other test. It must also
pass on its own, in a fresh process.
"""
import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import OnDevice, assert_close, host_bf16, reference

pytestmark = pytest.mark.gpu


def cases():
    return {
        # CodeLlama-34B-shaped decode at 16K tokens, planner split count (> 1)
        "gqa8-L16K": (wl.config(2, L=16384), None),
        # ragged batch with NaN padding and an empty sequence
        "varlen": (wl.make_problem(4, 32, 8, 128, 4000, seed=77, seqlens=[4000, 1, 2500, 0],
                                   nan_pad=True), 7),
        # paged cache, 16-token pages
        "paged": (wl.make_problem(3, 32, 8, 128, 2048, seed=78, seqlens=[2048, 1000, 17],
                                  block_size=16), 5),
    }


@pytest.mark.parametrize("name", ["gqa8-L16K", "varlen", "paged"])
def test_static_workspace_matches_fd_decode(cuda_device, name):
    import torch
    w, S = cases()[name]
    d = OnDevice(w)
    S = S or d.plan()
    assert fd.fd_workspace_bytes(w.B, w.Hq, w.D, S) <= fd.FD_STATIC_WORKSPACE_BYTES
    ref_out, ref_lse, _ = d.run(S)  # fd_decode with a torch-allocated workspace
    torch.cuda.synchronize()
    oracle_out, oracle_lse = reference(w)
    for i in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = fd.fd_decode_static_workspace(d.problem(), d.q, d.k, d.v, d.seqlens, d.table,
                                           w.scale, S, out, lse, None)
        assert st == fd.FD_OK, fd.fd_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), f"call {i}: out differs from fd_decode's"
        assert torch.equal(lse, ref_lse), f"call {i}: lse differs from fd_decode's"
        assert_close(host_bf16(out), lse.cpu().numpy().astype(np.float64), oracle_out,
                     oracle_lse, f"{name}, call {i}")
    assert fd.fd_check_device_error() == fd.FD_OK


def test_static_workspace_rejects_requests_above_its_size(cuda_device):
    import torch
    B, Hq, Hkv, D, L, S = 64, 64, 8, 128, 4096, 64
    need = fd.fd_workspace_bytes(B, Hq, D, S)
    assert need > fd.FD_STATIC_WORKSPACE_BYTES
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Hkv, L, D), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    prob = fd.make_problem(B, Hq, Hkv, D, L)
    st = fd.fd_decode_static_workspace(prob, q, k, v, None, None, 0.125, S, out, None, None)
    assert st == fd.FD_ERR_WORKSPACE
    # the same problem with one split needs no workspace at all
    st = fd.fd_decode_static_workspace(prob, q, k, v, None, None, 0.125, 1, out, None, None)
    assert st == fd.FD_OK
    torch.cuda.synchronize()
    assert fd.fd_check_device_error() == fd.FD_OK
