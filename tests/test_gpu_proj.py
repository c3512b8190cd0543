"""GPU parity of the full-width projections (salad_project, and salad_forward
with w_lin_full / w_out) against the oracle.

The projection GEMM is compared with the oracle's combine_full (per-head
output with the gated residual) and output_projection (token-major output),
element by element, on shapes that span several 128-token tiles with a
ragged tail, every output tile width (256, 128, 64 columns) and both head
widths.  The layer is compared on the small workloads in full and on the
480p Top-K workload at seeded query blocks the oracle computes one by one.
Bar: max |err| <= 2e-2, relative L2 <= 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import WORKLOADS, generate, generate_projections
from tests._parity import assert_close, device_inputs, to64
from tests.test_gpu_attention import SWA_SMALL
from tests.test_gpu_forward import RAGGED128_B2, _plan, _selection_used
from tests.test_gpu_kernels import CASES

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def salad():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_hybrid_top_b200 as m
    return m


def _bf16(rng, shape, scale=1.0):
    return torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(
        torch.bfloat16)


# (B, H, N, d, n_out): n_out a multiple of 256 runs on CTA pairs (256-token
# tiles), the others on single CTAs with 128- or 64-column tiles; ragged and
# single-token N (a pair tile whose second CTA has no valid row).
PER_HEAD = [(1, 2, 930, 128, 256), (2, 3, 198, 64, 192), (1, 1, 1, 128, 128),
            (2, 12, 1000, 128, 1536), (1, 4, 129, 64, 256), (1, 2, 1, 128, 256),
            (2, 2, 300, 128, 256)]
TOKEN_MAJOR = [(1, 2, 930, 128, 64), (2, 3, 198, 64, 320), (1, 12, 700, 128, 1536),
               (1, 1, 1, 64, 128), (2, 5, 260, 64, 384), (1, 2, 257, 64, 512)]


@pytest.mark.parametrize("shape", PER_HEAD, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("in_place", [False, True])
def test_project_per_head_gated_residual(salad, shape, in_place):
    B, H, N, d, n_out = shape
    rng = np.random.default_rng(sum(shape) + in_place)
    a = _bf16(rng, (B, H, N, d))
    w = _bf16(rng, (H * d, n_out), 0.02)
    resid = _bf16(rng, (B, H, N, d))
    s = torch.from_numpy(rng.uniform(0.1, 0.9, B).astype(np.float32))
    ad, wd, rd, sd = a.cuda(), w.cuda(), resid.cuda(), s.cuda()
    if in_place:
        out = rd.clone()
        got = salad.project(ad, wd, out_per_head=True, resid=out, s=sd, out=out)
        assert got.data_ptr() == out.data_ptr()
    else:
        got = salad.project(ad, wd, out_per_head=True, resid=rd, s=sd)
    torch.cuda.synchronize()
    salad.check_error()
    want = np.stack([oracle.combine_full(resid[b], a[b], w, float(s[b])) for b in range(B)])
    assert_close(got, want, f"project per-head {shape}")


@pytest.mark.parametrize("shape", TOKEN_MAJOR, ids=lambda s: "x".join(map(str, s)))
def test_project_token_major(salad, shape):
    B, H, N, d, n_out = shape
    rng = np.random.default_rng(100 + sum(shape))
    a = _bf16(rng, (B, H, N, d))
    w = _bf16(rng, (H * d, n_out), 0.02)
    got = salad.project(a.cuda(), w.cuda())
    torch.cuda.synchronize()
    salad.check_error()
    assert got.shape == (B, N, n_out)
    want = np.stack([oracle.output_projection(a[b], w) for b in range(B)])
    assert_close(got, want, f"project token-major {shape}")


def test_project_leaves_dropped_samples_unwritten(salad):
    B, H, N, d = 3, 2, 300, 64
    rng = np.random.default_rng(7)
    a = _bf16(rng, (B, H, N, d)).cuda()
    w = _bf16(rng, (H * d, H * d), 0.02).cuda()
    resid = _bf16(rng, (B, H, N, d)).cuda()
    s = torch.tensor([0.2, 0.8, 0.45], dtype=torch.float32, device="cuda")
    sentinel = torch.full_like(resid, 7.0)
    out = sentinel.clone()
    salad.project(a, w, out_per_head=True, resid=resid, s=s, drop_threshold=0.5, out=out)
    ref = salad.project(a, w, out_per_head=True, resid=resid, s=s)
    torch.cuda.synchronize()
    salad.check_error()
    assert torch.equal(out[0], sentinel[0]) and torch.equal(out[2], sentinel[2])
    assert torch.equal(out[1], ref[1])
    # NaN or 0 never drops.
    for thr in (float("nan"), 0.0):
        o2 = sentinel.clone()
        salad.project(a, w, out_per_head=True, resid=resid, s=s, drop_threshold=thr, out=o2)
        assert torch.equal(o2, ref)


def test_project_is_deterministic(salad):
    rng = np.random.default_rng(11)
    a = _bf16(rng, (1, 12, 2000, 128)).cuda()
    w = _bf16(rng, (1536, 1536), 0.02).cuda()
    x = salad.project(a, w)
    y = salad.project(a, w)
    assert torch.equal(x, y)


# ------------------------------------------------------------ the layer ---
def _full_plan(salad, w, dev, proj, **kw):
    return _plan(salad, w, dev, w_lin_full=proj["w_lin_full"], w_out=proj["w_out"], **kw)


def _oracle_kw(w, inp, plan):
    kw = dict(mode=w.mode, block=w.block, topk=w.topk, window=w.window,
              space_major_heads=w.space_major_heads, F=w.F, Hh=w.Hh, Wh=w.Wh, eps=w.eps)
    if w.mode == "topk":
        kw["idx_override"] = _selection_used(w, inp, plan.idx_out)
    return kw


@pytest.mark.parametrize("w", CASES + [SWA_SMALL], ids=lambda w: w.name)
def test_forward_full_width(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    proj_cpu = generate_projections(w, d_out=128 if w.d == 64 else None)
    proj = device_inputs(proj_cpu)
    plan = _full_plan(salad, w, dev, proj)
    o = plan.run()
    torch.cuda.synchronize()
    salad.check_error()
    ref = oracle.forward(inp, w_lin_full=proj_cpu["w_lin_full"], w_out=proj_cpu["w_out"],
                         **_oracle_kw(w, inp, plan))
    assert_close(o, ref["o"], f"forward full-width {w.name}")
    assert_close(plan.out, ref["out"], f"forward output projection {w.name}")


@pytest.mark.parametrize("w", CASES + [SWA_SMALL], ids=lambda w: w.name)
def test_forward_full_width_rope3d(salad, w):
    # The rotary encoding turns phi(q) in the linear-apply kernel that feeds
    # the full-width projection (numerator only, as in the per-head path).
    inp = generate(w)
    dev = device_inputs(inp)
    proj_cpu = generate_projections(w)
    proj = device_inputs(proj_cpu)
    grid = {} if w.mode == "swa" else dict(F=w.F, Hh=w.Hh, Wh=w.Wh)
    plan = _full_plan(salad, w, dev, proj, rope3d=True, **grid)
    o = plan.run()
    torch.cuda.synchronize()
    salad.check_error()
    ref = oracle.forward(inp, w_lin_full=proj_cpu["w_lin_full"], w_out=proj_cpu["w_out"],
                         rope3d=True, **_oracle_kw(w, inp, plan))
    assert_close(o, ref["o"], f"forward full-width with rope3d {w.name}")
    assert_close(plan.out, ref["out"], f"output projection with rope3d {w.name}")


def test_forward_full_width_branch_dropping(salad):
    w = RAGGED128_B2
    inp = generate(w)
    inp["x"][1] = (inp["x"][1].float() + 0.5).to(torch.bfloat16)
    dev = device_inputs(inp)
    proj_cpu = generate_projections(w)
    proj = device_inputs(proj_cpu)
    full = _full_plan(salad, w, dev, proj)
    full.run()
    torch.cuda.synchronize()
    s = full.s_out.cpu()
    lo, hi = (0, 1) if s[0] < s[1] else (1, 0)
    # Above both gate values: the sparse branch alone, bit for bit.
    every = _full_plan(salad, w, dev, proj, drop_threshold=1.0)
    o_all = every.run().clone()
    o_sparse = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "topk", topk=w.topk,
                                 idx=every.idx_out)
    torch.cuda.synchronize()
    salad.check_error()
    assert torch.equal(o_all, o_sparse)
    # Between the two: only the lower sample loses its linear branch.
    thr = float(s[lo] + s[hi]) / 2
    mid = _full_plan(salad, w, dev, proj, drop_threshold=thr)
    o_mid = mid.run()
    torch.cuda.synchronize()
    salad.check_error()
    ref = oracle.forward(inp, w_lin_full=proj_cpu["w_lin_full"], w_out=proj_cpu["w_out"],
                         drop_threshold=thr, **_oracle_kw(w, inp, mid))
    assert list(ref["dropped"]) == [b == lo for b in range(2)]
    assert_close(o_mid, ref["o"], "forward full-width with branch dropping")
    assert_close(mid.out, ref["out"], "output projection with branch dropping")


def test_forward_full_width_topk480_sampled(salad):
    # Full size, in the configuration the benchmark times; the oracle
    # recomputes every head of 6 seeded query blocks plus the ragged tail.
    w = WORKLOADS["topk480"]
    inp = generate(w)
    dev = device_inputs(inp)
    proj_cpu = generate_projections(w)
    proj = device_inputs(proj_cpu)
    plan = _full_plan(salad, w, dev, proj)
    o = plan.run()
    torch.cuda.synchronize()
    salad.check_error()
    idx = _selection_used(w, inp, plan.idx_out)
    s = oracle.gate(inp["x"], inp["w_gate"], inp["bias"])
    rng = np.random.default_rng(5)
    blocks = sorted(set(int(i) for i in rng.integers(0, w.nb, 6)) | {w.nb - 1})
    rows = np.concatenate([np.arange(i * w.block, min(w.N, (i + 1) * w.block)) for i in blocks])
    o_s = np.empty((w.H, len(rows), w.d))
    o_l = np.empty_like(o_s)
    for h in range(w.H):
        q, k, v = (to64(inp[n][0, h]) for n in ("q", "k", "v"))
        res = oracle.topk_attention_rows(q, k, v, idx[0, h], w.block, blocks)
        o_s[h] = np.concatenate([res[i] for i in blocks])
        Hst, Z = oracle.linear_state(k, v)
        o_l[h] = oracle.linear_apply(q[rows], Hst, Z, w.eps)
    want_o = oracle.combine_full(o_s, o_l, proj_cpu["w_lin_full"], s[0])
    want_out = oracle.output_projection(want_o, proj_cpu["w_out"])
    r = torch.from_numpy(rows)
    assert_close(o[0][:, r].cpu(), want_o, f"forward full-width topk480 ({len(blocks)} blocks)")
    assert_close(plan.out[0][r].cpu(), want_out, "output projection topk480")
