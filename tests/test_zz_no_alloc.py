"""The no-allocation entry point (more_route_unfused_static) against the scratch-taking one.

more_route_unfused_static is for callers that may not allocate device memory (an
external allocator or memory budget that forbids raw allocations, or a latency-critical
path where an allocation is not acceptable): it runs the materialise-then-top-k kernels
on a fixed scratch array inside the library.  Two calls in a row, on different inputs,
must match more_route_unfused within the parity tolerances.  tests/conftest.py runs
this file after every other GPU test file.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def call_static(lib, X, R1, R2, k, outs):
    N, h = X.shape
    r, M = R2.shape
    P = ctypes.c_void_p
    return lib.more_route_unfused_static(P(X.data_ptr()), P(R1.data_ptr()), P(R2.data_ptr()), N, h, r, M, k,
                                         P(outs[0].data_ptr()), P(outs[1].data_ptr()), P(outs[2].data_ptr()),
                                         P(outs[3].data_ptr()), P(torch.cuda.current_stream().cuda_stream))


def new_outputs(N, k, M):
    return (torch.empty((N, k), dtype=torch.int32, device="cuda"),
            torch.empty((N, k), dtype=torch.float32, device="cuda"),
            torch.full((M,), 12345, dtype=torch.int32, device="cuda"),
            torch.empty((N, k), dtype=torch.float32, device="cuda"))


def test_static_scratch_matches_caller_scratch_twice():
    import mixture_experts_rank_b200 as m
    lib = m._lib
    cases = [(4096, 128, 32, 192, 4, 0), (1500, 512, 64, 1024, 8, 7)]   # two calls in a row
    for (N, h, r, M, k, seed) in cases:
        X, R1, R2 = (dev_bf16(a) for a in syn.router_inputs(N, h, r, M, seed=seed))
        outs = new_outputs(N, k, M)
        assert call_static(lib, X, R1, R2, k, outs) == 0
        ref = m.route_unfused(X, R1, R2, k)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        got = [t.cpu().numpy() for t in outs]
        want = [t.cpu().numpy() for t in ref]
        np.testing.assert_array_equal(got[0], want[0])                 # expert indices
        np.testing.assert_allclose(got[1], want[1], rtol=0, atol=2e-3)  # gates
        np.testing.assert_array_equal(got[2], want[2])                 # counts
        rms = np.sqrt(np.mean(want[3] ** 2, axis=1, keepdims=True))
        assert np.all(np.abs(got[3] - want[3]) <= 1e-2 * rms)           # logits


def test_static_scratch_rejects_problems_beyond_its_size():
    import mixture_experts_rank_b200 as m
    lib = m._lib
    N, h, r, M, k = 16384, 64, 32, 1024, 4     # 64 MiB of logits: more than the fixed scratch
    assert m.unfused_scratch_bytes(N, r, M) > m.STATIC_SCRATCH_BYTES
    X = torch.zeros((N, h), dtype=torch.bfloat16, device="cuda")
    R1 = torch.zeros((h, r), dtype=torch.bfloat16, device="cuda")
    R2 = torch.zeros((r, M), dtype=torch.bfloat16, device="cuda")
    outs = new_outputs(N, k, M)
    assert call_static(lib, X, R1, R2, k, outs) == 2   # MORE_ERR_UNSUPPORTED
