"""GPU parity of the attention kernel (sparse branch alone, dense comparator)
against the CPU oracle, through the C ABI.  Bar: max |err| <= 2e-2 and
relative L2 <= 5e-3 on the bf16 outputs."""
import numpy as np
import pytest
import torch

import oracle
from synth import WORKLOADS, Workload, generate
from tests._parity import assert_close, device_inputs, to64
from tests.test_gpu_kernels import CASES, RAGGED64, RAGGED128

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def salad():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_hybrid_top_b200 as m
    return m


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_dense_attention(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    o = salad.dense_attn(dev["q"], dev["k"], dev["v"])
    torch.cuda.synchronize()
    q, k, v = to64(inp["q"]), to64(inp["k"]), to64(inp["v"])
    want = np.stack([np.stack([oracle.dense_attention(q[b, h], k[b, h], v[b, h])
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(o, want, f"dense {w.name}")
    salad.check_error()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_topk_attention_given_selection(salad, w):
    inp = generate(w)
    dev = device_inputs(inp)
    q, k, v = to64(inp["q"]), to64(inp["k"]), to64(inp["v"])
    # Selection from the oracle; the kernel must attend exactly to it.
    idx = np.stack([np.stack([oracle.select_topk(oracle.block_scores(q[b, h], k[b, h], w.block), w.topk)
                              for h in range(w.H)]) for b in range(w.B)])
    idx_t = torch.from_numpy(idx).to(torch.int32).cuda()
    o = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "topk", topk=w.topk, idx=idx_t)
    torch.cuda.synchronize()
    want = np.stack([np.stack([oracle.topk_attention(q[b, h], k[b, h], v[b, h], idx[b, h], w.block)
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(o, want, f"topk {w.name}")
    salad.check_error()


def test_topk_random_selection_patterns(salad):
    # Arbitrary (not score-driven) kept sets: every mask combination of a
    # query-block pair, tiles only one block of a pair needs, and the ragged
    # last pair (nb = 15: its second block does not exist).
    w = RAGGED128
    inp = generate(w)
    dev = device_inputs(inp)
    q, k, v = to64(inp["q"]), to64(inp["k"]), to64(inp["v"])
    rng = np.random.default_rng(0)
    for kk in (1, 5, w.nb):
        idx = np.stack([np.stack([np.sort(rng.permutation(w.nb)[:kk]) for _ in range(w.nb)])
                        for _ in range(w.H)])[None]
        idx_t = torch.from_numpy(idx).to(torch.int32).cuda()
        o = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "topk", topk=kk, idx=idx_t)
        want = np.stack([oracle.topk_attention(q[0, h], k[0, h], v[0, h], idx[0, h], w.block)
                         for h in range(w.H)])[None]
        assert_close(o, want, f"random topk k={kk}")
    # Structured sets: each block keeps only itself, a block far away, or
    # blocks that differ between the two halves of each group of four.
    for name, rows in (("diagonal", [[i] for i in range(w.nb)]),
                       ("far", [[(i + w.nb // 2) % w.nb] for i in range(w.nb)]),
                       ("slot-disjoint", [[0, 1] if i % 4 < 2 else [w.nb - 2, w.nb - 1]
                                          for i in range(w.nb)])):
        kk = len(rows[0])
        idx = np.array([rows for _ in range(w.H)])[None]
        idx_t = torch.from_numpy(idx).to(torch.int32).cuda()
        o = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "topk", topk=kk, idx=idx_t)
        want = np.stack([oracle.topk_attention(q[0, h], k[0, h], v[0, h], idx[0, h], w.block)
                         for h in range(w.H)])[None]
        assert_close(o, want, f"{name} topk k={kk}")
    salad.check_error()


def test_topk_all_blocks_equals_dense(salad):
    w = RAGGED128
    inp = generate(w)
    dev = device_inputs(inp)
    idx = torch.arange(w.nb, dtype=torch.int32).expand(1, w.H, w.nb, w.nb).contiguous().cuda()
    o1 = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "topk", topk=w.nb, idx=idx)
    o2 = salad.dense_attn(dev["q"], dev["k"], dev["v"])
    assert torch.equal(o1, o2)
    salad.check_error()


SWA_SMALL = Workload(name="swa_small", B=1, H=4, d=128, F=4, Hh=6, Wh=13, D=64, mode="swa",
                     window=78, space_major_heads=(0, 2), lowrank_scale=0.5, seeds=(7,))  # N=312
SWA_SMALL64 = Workload(name="swa_small64", B=2, H=2, d=64, F=5, Hh=4, Wh=7, D=64, mode="swa",
                       window=40, space_major_heads=(1,), lowrank_scale=0.5, seeds=(8, 9))  # N=140


# Grids with the frame counts of the 480p and 720p latents (F = 20, 28) and
# one more (F = 36): a position's F rows straddle the 64-row blocks and the
# 128-row tiles of the regrouped order differently in each.
SWA_F20 = Workload(name="swa_f20", B=1, H=3, d=128, F=20, Hh=3, Wh=5, D=64, mode="swa",
                   window=70, space_major_heads=(0, 2), lowrank_scale=0.5, seeds=(10,))  # N=300
SWA_F28 = Workload(name="swa_f28", B=2, H=2, d=64, F=28, Hh=2, Wh=5, D=64, mode="swa",
                   window=100, space_major_heads=(0, 1), lowrank_scale=0.5, seeds=(11, 12))  # N=280
SWA_F36 = Workload(name="swa_f36", B=1, H=2, d=128, F=36, Hh=2, Wh=3, D=64, mode="swa",
                   window=50, space_major_heads=(1,), lowrank_scale=0.5, seeds=(13,))  # N=216
SWA_CASES = [SWA_SMALL, SWA_SMALL64, SWA_F20, SWA_F28, SWA_F36]


@pytest.mark.parametrize("w", SWA_CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("window", [None, 0, 1, 1000000])
def test_swa_attention(salad, w, window):
    W = w.window if window is None else window
    inp = generate(w)
    dev = device_inputs(inp)
    o = salad.sparse_attn(dev["q"], dev["k"], dev["v"], "swa", window=W,
                          space_major_heads=w.space_major_heads, F=w.F, Hh=w.Hh, Wh=w.Wh)
    torch.cuda.synchronize()
    q, k, v = to64(inp["q"]), to64(inp["k"]), to64(inp["v"])
    want = np.stack([np.stack([oracle.swa_attention(q[b, h], k[b, h], v[b, h], W,
                                                    h in w.space_major_heads, w.F, w.Hh, w.Wh)
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(o, want, f"swa {w.name} W={W}")
    if W == 0:
        # Each token attends to itself only: the output is V rounded to bf16.
        assert torch.equal(o, dev["v"])
    salad.check_error()
