"""The binding checks every tensor's shape before anything reaches the device
(a wrong size would make a kernel read past a tensor).  On the CPU the checks
run on host tensors: a well-formed call stops at the device check, a
malformed one at the shape check."""
import pytest
import torch

import sparse_linear_hybrid_top_b200 as salad
from synth import WORKLOADS, generate, generate_projections
from tests.test_gpu_attention import SWA_SMALL
from tests.test_gpu_kernels import CASES


def _expect_device_error(fn):
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn()


def _expect_shape_error(fn, name):
    with pytest.raises(ValueError, match=f"{name} must"):
        fn()


def _plan(w, inp, **kw):
    extra = dict(window=w.window, space_major_heads=w.space_major_heads, F=w.F, Hh=w.Hh,
                 Wh=w.Wh) if w.mode == "swa" else {}
    return salad.ForwardPlan(inp["q"], inp["k"], inp["v"], inp["x"], inp["w_gate"],
                             kw.pop("w_lin", inp["w_lin"]), mode=w.mode, topk=w.topk,
                             bias=w.bias, eps=w.eps, **extra, **kw)


@pytest.mark.parametrize("w", CASES + [SWA_SMALL], ids=lambda w: w.name)
def test_forward_plan_shapes_accepted(w):
    inp = generate(w)
    nb = w.nb
    idx = torch.empty(w.B, w.H, nb, max(w.topk, 1), dtype=torch.int32) if w.mode == "topk" \
        else None
    s_out = torch.empty(w.B, dtype=torch.float32)
    _expect_device_error(lambda: _plan(w, inp, idx_out=idx, s_out=s_out))
    proj = generate_projections(w, d_out=256)
    _expect_device_error(lambda: _plan(w, inp, w_lin=None, w_lin_full=proj["w_lin_full"],
                                       w_out=proj["w_out"], idx_out=idx, s_out=s_out))


def test_forward_plan_shapes_rejected():
    w = WORKLOADS["tiny"]
    inp = generate(w)
    bad = dict(inp)
    bad["k"] = inp["k"][:, :, :-1]
    _expect_shape_error(lambda: _plan(w, bad), "k")
    bad = dict(inp)
    bad["w_gate"] = inp["w_gate"][:-8]
    _expect_shape_error(lambda: _plan(w, bad), "w_gate")
    _expect_shape_error(lambda: _plan(w, inp, w_lin=inp["w_lin"][:, :, :-1]), "w_lin")
    proj = generate_projections(w)
    _expect_shape_error(lambda: _plan(w, inp, w_lin_full=proj["w_lin_full"][:-64]), "w_lin_full")
    _expect_shape_error(lambda: _plan(w, inp, w_out=proj["w_out"][:-64]), "w_out")
    _expect_shape_error(lambda: _plan(w, inp, w_out=proj["w_out"],
                                      out=torch.empty(w.B, w.N, 64, dtype=torch.bfloat16)), "out")
    _expect_shape_error(lambda: _plan(w, inp, idx_out=torch.empty(w.B, w.H, w.nb, w.topk + 1,
                                                                  dtype=torch.int32)), "idx_out")
    _expect_shape_error(lambda: _plan(w, inp, s_out=torch.empty(w.B + 1)), "s_out")


def test_project_shapes():
    B, H, N, d = 2, 3, 50, 64
    a = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    w = torch.zeros(H * d, 192, dtype=torch.bfloat16)
    res = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    s = torch.zeros(B)
    _expect_device_error(lambda: salad.project(a, w, out_per_head=True, resid=res, s=s))
    _expect_device_error(lambda: salad.project(a, torch.zeros(H * d, 320, dtype=torch.bfloat16)))
    _expect_shape_error(lambda: salad.project(a, w[:-64]), "w")
    _expect_shape_error(lambda: salad.project(a, w, out_per_head=True, resid=res[:, :, :-1]),
                        "resid")
    _expect_shape_error(lambda: salad.project(a, w, out=torch.zeros(B, N, 64)), "out")
    _expect_shape_error(lambda: salad.project(a, w, s=torch.zeros(B + 1)), "s")


def test_piecewise_calls_shapes():
    w = WORKLOADS["tiny"]
    inp = generate(w)
    q, k, v, x, wg = inp["q"], inp["k"], inp["v"], inp["x"], inp["w_gate"]
    B, H, N, d = q.shape
    nb = w.nb
    # Well-formed calls stop at the device check.
    _expect_device_error(lambda: salad.gate(x, wg, 0.0))
    _expect_device_error(lambda: salad.gate_noalloc(x, wg, 0.0, s=torch.zeros(B)))
    _expect_device_error(lambda: salad.select_blocks(q, k, w.topk))
    _expect_device_error(lambda: salad.select_blocks(
        q, k, 2, idx=torch.zeros(B, H, nb, 2, dtype=torch.int32)))
    _expect_device_error(lambda: salad.linear_state(k, v))
    _expect_device_error(lambda: salad.linear_apply(q, torch.zeros(B, H, d, d), torch.zeros(B, H, d)))
    _expect_device_error(lambda: salad.permute_tokens(torch.zeros(2, N, d, dtype=torch.bfloat16),
                                                      w.F, w.Hh, w.Wh))
    idx = torch.zeros(B, H, nb, w.topk, dtype=torch.int32)
    _expect_device_error(lambda: salad.sparse_attn(q, k, v, "topk", topk=w.topk, idx=idx))
    _expect_device_error(lambda: salad.sparse_attn(q, k, v, "swa", window=8))
    _expect_device_error(lambda: salad.dense_attn(q, k, v))
    # Malformed ones stop at the shape check.
    _expect_shape_error(lambda: salad.gate(x, wg[:-8], 0.0), "w")
    _expect_shape_error(lambda: salad.gate(x, wg, 0.0, s=torch.zeros(B + 1)), "s")
    _expect_shape_error(lambda: salad.select_blocks(q, k[:, :, :-1], w.topk), "k")
    _expect_shape_error(lambda: salad.select_blocks(
        q, k, 2, idx=torch.zeros(B, H, nb, 3, dtype=torch.int32)), "idx")
    _expect_shape_error(lambda: salad.linear_state(k, v[..., :-1]), "v")
    _expect_shape_error(lambda: salad.linear_apply(q, torch.zeros(B, H, d, d - 1),
                                                   torch.zeros(B, H, d)), "Hst")
    _expect_shape_error(lambda: salad.linear_apply(q, torch.zeros(B, H, d, d),
                                                   torch.zeros(B, H + 1, d)), "Z")
    _expect_shape_error(lambda: salad.permute_tokens(
        torch.zeros(2, N, d, dtype=torch.bfloat16), w.F, w.Hh, w.Wh,
        dst=torch.zeros(2, N - 1, d, dtype=torch.bfloat16)), "dst")
    _expect_shape_error(lambda: salad.sparse_attn(q, k, v, "topk", topk=w.topk,
                                                  idx=idx[:, :, :-1]), "idx")
    _expect_shape_error(lambda: salad.sparse_attn(q, k, v[:, :1], "swa", window=8), "v")
    _expect_shape_error(lambda: salad.dense_attn(q, k, v, o=q[:, :, :-1]), "o")


@pytest.mark.gpu
def test_outputs_checked_like_inputs():
    # Device inputs with a caller-supplied output on the host, of the wrong
    # dtype or not contiguous: every call refuses before any launch (a host
    # pointer handed to a kernel would fault; a wrong dtype would be misread).
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = WORKLOADS["tiny"]
    inp = {k: (t.cuda() if isinstance(t, torch.Tensor) else t) for k, t in generate(w).items()}
    q, k, v, x, wg = inp["q"], inp["k"], inp["v"], inp["x"], inp["w_gate"]
    B, H, N, d = q.shape
    nb = w.nb
    bad_s = [torch.zeros(B), torch.zeros(B, dtype=torch.float64, device="cuda")]
    for s in bad_s:
        with pytest.raises(ValueError, match="s must|s is on"):
            salad.gate(x, wg, 0.0, s=s)
        with pytest.raises(ValueError, match="s must|s is on"):
            salad.gate_noalloc(x, wg, 0.0, s=s)
    for idx in (torch.zeros(B, H, nb, 2, dtype=torch.int32),
                torch.zeros(B, H, nb, 2, dtype=torch.int64, device="cuda")):
        with pytest.raises(ValueError, match="idx must"):
            salad.select_blocks(q, k, 2, idx=idx)
        with pytest.raises(ValueError, match="idx must"):
            salad.sparse_attn(q, k, v, "topk", topk=2, idx=idx)
    strided = torch.empty(B, H, N, 2 * d, dtype=torch.bfloat16, device="cuda")[..., ::2]
    assert strided.shape == q.shape and not strided.is_contiguous()
    for o in (torch.empty_like(q, device="cpu"), torch.empty(q.shape, device="cuda"), strided):
        with pytest.raises(ValueError, match="o must"):
            salad.dense_attn(q, k, v, o=o)
        with pytest.raises(ValueError, match="o must"):
            salad.sparse_attn(q, k, v, "swa", window=8, o=o)
        with pytest.raises(ValueError, match="o must"):
            salad.linear_apply(q, torch.zeros(B, H, d, d, device="cuda"),
                               torch.zeros(B, H, d, device="cuda"), o=o)
        with pytest.raises(ValueError, match="o must"):
            _plan(w, inp, o=o)
    with pytest.raises(ValueError, match="dst must"):
        salad.permute_tokens(q.reshape(-1, N, d), w.F, w.Hh, w.Wh,
                             dst=torch.empty(B * H, N, d, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="s_out must"):
        _plan(w, inp, s_out=torch.zeros(B))
    with pytest.raises(ValueError, match="idx_out must"):
        _plan(w, inp, idx_out=torch.zeros(B, H, nb, w.topk, dtype=torch.int64, device="cuda"))
    with pytest.raises(ValueError, match="workspace must"):
        salad.gate(x, wg, 0.0, workspace=torch.zeros(1 << 20, dtype=torch.uint8))
