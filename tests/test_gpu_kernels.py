"""GPU parity of the building blocks against the CPU oracle (through the C ABI).

Bars: integer / index / byte work bit-exact (selection up to the near-tie
rule, permutation exact); float32 state of the linear branch within a
relative L2 of 1e-4 (float32 accumulation of up to ~1e5 exact bf16 products,
split over many partial sums: a few ulps of float32 per partial); gate
within 1e-5 absolute; bf16 outputs at max |err| <= 2e-2, rel-L2 <= 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import WORKLOADS, Workload, generate
from tests._parity import assert_close, device_inputs, err_stats, to64

pytestmark = pytest.mark.gpu

# Several tiles plus a ragged tail, at both head sizes.
RAGGED128 = Workload(name="ragged128", B=1, H=2, d=128, F=3, Hh=10, Wh=31, D=256, mode="topk",
                     topk=3, lowrank_scale=0.5, seeds=(3,))          # N = 930, nb = 15
RAGGED64 = Workload(name="ragged64", B=2, H=3, d=64, F=2, Hh=9, Wh=11, D=64, mode="topk",
                    topk=2, lowrank_scale=0.5, seeds=(4, 5))         # N = 198, nb = 4
SINGLE_ROW = Workload(name="one_token", B=1, H=1, d=128, F=1, Hh=1, Wh=1, D=8, mode="topk",
                      topk=1, seeds=(6,))                             # N = 1

CASES = [WORKLOADS["tiny"], RAGGED128, RAGGED64, SINGLE_ROW]


@pytest.fixture(scope="module")
def salad():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_hybrid_top_b200 as m
    return m


def _gen(w):
    return device_inputs(generate(w))


@pytest.mark.parametrize("w", CASES + [WORKLOADS["topk480"]], ids=lambda w: w.name)
def test_gate(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    s = salad.gate(dev["x"], dev["w_gate"], inp["bias"])
    torch.cuda.synchronize()
    want = oracle.gate(inp["x"], inp["w_gate"], inp["bias"])
    np.testing.assert_allclose(to64(s), want, rtol=0, atol=1e-5)
    salad.check_error()


def _check_selection(idx_gpu, q, k, block, topk):
    """idx rows must equal the oracle's kept sets up to the near-tie rule."""
    B, H = q.shape[:2]
    idx_gpu = idx_gpu.cpu().numpy()
    ties = 0
    for b in range(B):
        for h in range(H):
            S = oracle.block_scores(q[b, h], k[b, h], block)
            ref = oracle.select_topk(S, topk)
            for i in range(S.shape[0]):
                row = idx_gpu[b, h, i]
                assert np.all(np.diff(row) > 0), "kept list must be strictly ascending"
                if set(row.tolist()) != set(ref[i].tolist()):
                    assert oracle.near_tie_equivalent(S[i], ref[i], row), (b, h, i, row, ref[i])
                    ties += 1
    return ties


@pytest.mark.parametrize("w", CASES + [WORKLOADS["topk480"]], ids=lambda w: w.name)
def test_select_blocks(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    idx = salad.select_blocks(dev["q"], dev["k"], w.topk)
    torch.cuda.synchronize()
    _check_selection(idx, to64(inp["q"]), to64(inp["k"]), w.block, w.topk)
    salad.check_error()


# Rows longer than 2048 key blocks (128 scores per lane, 8 query blocks per
# CTA): 2091 full blocks and a ragged one of 51 rows, one head of d = 64,
# 10% kept.
LONG_ROWS = Workload(name="long_rows", B=1, H=1, d=64, F=5, Hh=105, Wh=255, D=64, mode="topk",
                     topk=210, lowrank_scale=0.5, seeds=(14,))      # N = 133875, nb = 2092


def test_select_blocks_long_rows(salad):
    w = LONG_ROWS
    assert w.nb > 2048
    inp = generate(w)
    dev = device_inputs(inp)
    idx = salad.select_blocks(dev["q"], dev["k"], w.topk)
    torch.cuda.synchronize()
    _check_selection(idx, to64(inp["q"]), to64(inp["k"]), w.block, w.topk)
    salad.check_error()


def test_select_all_blocks_and_ties(salad):
    # topk = nb keeps everything; equal scores (all-zero Q) keep the lowest
    # indices -- including the -0.0 / +0.0 mix a zero query produces.
    w = RAGGED128
    inp = generate(w)
    dev = device_inputs(inp)
    idx = salad.select_blocks(dev["q"], dev["k"], w.nb)
    assert torch.equal(idx.cpu(), torch.arange(w.nb, dtype=torch.int32).expand(1, 2, w.nb, w.nb))
    qz = torch.zeros_like(dev["q"])
    idx = salad.select_blocks(qz, dev["k"], 4)
    assert torch.equal(idx.cpu(), torch.arange(4, dtype=torch.int32).expand(1, 2, w.nb, 4))
    salad.check_error()


def _tie_case(nb, N, big_in, big_out, scale=1.0):
    """Q, K [1,1,N,128] whose block scores agree to ~1e-10 relative, beyond
    float32 resolution: every query row is all ones (times `scale`); key
    channel 0 is zero but for row 0 of block j, which carries a distinct tiny
    value t_j (exact in bf16), and every other key channel is one, so the
    float64 scores 127 + t_j / 64 (times scale^2) differ only in t_j.  The
    first `big_in` blocks get 2 on channel 1 of every row (decided in float32,
    kept) and the last `big_out` blocks 0 there (decided, dropped)."""
    d = 128
    q = torch.full((1, 1, N, d), scale, dtype=torch.float32)
    k = torch.full((1, 1, N, d), scale, dtype=torch.float32)
    k[..., 0] = 0.0
    for j in range(nb):
        t = ((j * 37) % nb + 1) * 2.0 ** -20
        k[0, 0, j * 64, 0] = scale * t
        if j < big_in:
            k[0, 0, j * 64:(j + 1) * 64, 1] = 2.0 * scale
        elif j >= nb - big_out:
            k[0, 0, j * 64:(j + 1) * 64, 1] = 0.0
    return q.to(torch.bfloat16), k.to(torch.bfloat16)


@pytest.mark.parametrize("nb,N,topk,big_in,big_out,scale", [
    (96, 96 * 64 - 17, 30, 0, 0, 1.0),     # every block a candidate: radix path over float64 keys
    (40, 40 * 64, 10, 5, 15, 1.0),          # 20 candidates, 5 to keep: buffered float64 ranking
    (24, 24 * 64, 7, 3, 3, 2.0 ** 64),      # float32 would overflow: every block goes to float64
])
def test_select_decided_in_float64(salad, nb, N, topk, big_in, big_out, scale):
    # The kept sets must equal the float64 selection exactly -- no near-tie
    # excuse, although the scores differ by far less than 1e-5 relative: the
    # float32 pass cannot order these blocks, the float64 recheck must.
    q, k = _tie_case(nb, N, big_in, big_out, scale)
    assert (N + 63) // 64 == nb
    t = ((np.arange(nb) * 37) % nb + 1)
    assert len(set(t.tolist())) == nb        # distinct perturbations
    idx = salad.select_blocks(q.cuda(), k.cuda(), topk)
    torch.cuda.synchronize()
    salad.check_error()
    S = oracle.block_scores(to64(q)[0, 0], to64(k)[0, 0], 64)
    ref = oracle.select_topk(S, topk)
    got = idx.cpu().numpy()[0, 0]
    for i in range(nb):
        assert np.array_equal(np.sort(ref[i]), got[i]), (i, sorted(ref[i].tolist()), got[i].tolist())
    # The case really is below float32 resolution: float32 scores tie.
    qm32 = oracle.block_means(to64(q)[0, 0], 64).astype(np.float32)
    km32 = oracle.block_means(to64(k)[0, 0], 64).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        S32 = qm32 @ km32.T
    assert len(np.unique(S32[0, big_in:nb - big_out])) == 1


@pytest.mark.parametrize("w", CASES + [WORKLOADS["topk480"]], ids=lambda w: w.name)
def test_linear_state(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    Hst, Z = salad.linear_state(dev["k"], dev["v"])
    torch.cuda.synchronize()
    k, v = to64(inp["k"]), to64(inp["v"])
    for b in range(w.B):
        for h in range(w.H):
            Hr, Zr = oracle.linear_state(k[b, h], v[b, h])
            _, rh = err_stats(Hst[b, h], Hr)
            _, rz = err_stats(Z[b, h], Zr)
            assert rh <= 1e-4 and rz <= 1e-4, (b, h, rh, rz)
    salad.check_error()


@pytest.mark.parametrize("w", CASES + [WORKLOADS["topk480"]], ids=lambda w: w.name)
def test_linear_apply(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    k, v, q = to64(inp["k"]), to64(inp["v"]), to64(inp["q"])
    Hs = np.zeros((w.B, w.H, w.d, w.d)); Zs = np.zeros((w.B, w.H, w.d))
    for b in range(w.B):
        for h in range(w.H):
            Hs[b, h], Zs[b, h] = oracle.linear_state(k[b, h], v[b, h])
    # The apply kernel is tested on the oracle's state (float32 copy).
    Ht = torch.from_numpy(Hs).float().cuda()
    Zt = torch.from_numpy(Zs).float().cuda()
    o = salad.linear_apply(dev["q"], Ht, Zt, w.eps)
    torch.cuda.synchronize()
    want = np.stack([np.stack([oracle.linear_apply(q[b, h], Hs[b, h], Zs[b, h], w.eps)
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(o, want, f"linear_apply {w.name}")
    salad.check_error()


def test_linear_apply_zero_query_rows(salad):
    # phi(q) = 0 -> the row is exactly 0 (0 / eps).
    w = RAGGED128
    inp = generate(w)
    dev = device_inputs(inp)
    q = -dev["q"].abs()
    Hst, Z = salad.linear_state(dev["k"], dev["v"])
    o = salad.linear_apply(q, Hst, Z, 1e-6)
    assert torch.count_nonzero(o).item() == 0
    salad.check_error()


@pytest.mark.parametrize("grid", [(3, 10, 31), (2, 9, 11), (20, 30, 52)])
@pytest.mark.parametrize("d", [64, 128])
def test_permute_tokens_exact(salad, grid, d):
    F, Hh, Wh = grid
    N = F * Hh * Wh
    g = torch.Generator().manual_seed(N + d)
    src = torch.randn(2, N, d, generator=g).to(torch.bfloat16)
    dev = src.cuda()
    out = salad.permute_tokens(dev, F, Hh, Wh)
    back = salad.permute_tokens(out, F, Hh, Wh, inverse=True)
    perm = torch.from_numpy(oracle.space_major_order(F, Hh, Wh))
    assert torch.equal(out.cpu(), src[:, perm])
    assert torch.equal(back.cpu(), src)
    salad.check_error()
