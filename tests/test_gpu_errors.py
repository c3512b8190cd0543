"""Failure surfacing on the GPU without a fault: a bounded wait that runs out
must come back as SALAD_ERR_TIMEOUT from salad_check_error, and the context
must stay usable afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def salad():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_hybrid_top_b200 as m
    return m


def test_wait_timeout_is_reported_and_cleared(salad):
    salad.check_error()                       # clean start
    assert salad.debug_wait_timeout(2_000_000) == 0   # 2 ms limit
    with pytest.raises(salad.SaladError) as e:
        salad.check_error()
    assert e.value.code == -4
    salad.check_error()                       # the word was cleared
    # The context still runs kernels.
    x = torch.ones(1, 64, 16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    s = salad.gate(x, w, 0.0)
    assert abs(float(s.item()) - 0.5) < 1e-7


def test_invalid_arguments_raise_before_launch(salad):
    q = torch.zeros(1, 1, 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(salad.SaladError) as e:
        salad.dense_attn(q, q, q)
    assert e.value.code == -2
