"""The allocation-free gate (salad_gate_noalloc) against the regular gate.

Some callers cannot allocate device memory at all -- a plug-in that is handed
only its input and output buffers, or code running where an allocator call is
not permitted -- so they cannot provide the workspace salad_gate needs.  The
no-allocation variant keeps its partial sums in a fixed array inside the
library.  This test calls it through the C ABI twice in a row, on different
inputs, and checks each result against salad_gate and against the float64
oracle within the gate tests' tolerance (1e-5 absolute on s); on a 148-SM
B200 the two CUDA gates share one partition, so they must agree bit for bit.
It also checks that a batch larger than the array serves is refused before
any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def salad():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_hybrid_top_b200 as m
    return m


def _inputs(B, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, N, D, generator=g).to(torch.bfloat16).cuda()
    w = (0.02 * torch.randn(D, generator=g)).to(torch.bfloat16).cuda()
    return x, w


def _noalloc(salad, x, w, bias):
    B, N, D = x.shape
    s = torch.full((B,), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = salad.lib.salad_gate_noalloc(x.data_ptr(), w.data_ptr(), ctypes.c_float(bias), B, N, D,
                                      s.data_ptr(), stream)
    assert rc == 0, salad.status_string(rc)
    return s


def test_noalloc_gate_matches_gate_on_two_calls_in_a_row(salad):
    cases = [(2, 31200, 1536, 0.0, 11), (3, 1000, 256, 0.25, 12)]
    outs = []
    for B, N, D, bias, seed in cases:
        x, w = _inputs(B, N, D, seed)
        s_new = _noalloc(salad, x, w, bias)
        s_ref = salad.gate(x, w, bias)
        outs.append((s_new, s_ref, oracle.gate(x.cpu(), w.cpu(), bias)))
    torch.cuda.synchronize()
    salad.check_error()
    same_partition = torch.cuda.get_device_properties(0).multi_processor_count == 148
    for s_new, s_ref, s_oracle in outs:
        assert torch.isfinite(s_new).all()
        torch.testing.assert_close(s_new, s_ref, rtol=0, atol=1e-5)
        np.testing.assert_allclose(s_new.cpu().double().numpy(), s_oracle, rtol=0, atol=1e-5)
        if same_partition:
            assert torch.equal(s_new, s_ref)


def test_noalloc_gate_refuses_batches_beyond_its_array(salad):
    x, w = _inputs(1, 16, 8, 13)
    s = torch.empty(257, dtype=torch.float32, device="cuda")
    rc = salad.lib.salad_gate_noalloc(x.data_ptr(), w.data_ptr(), ctypes.c_float(0.0), 257, 16, 8,
                                      s.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == -1
