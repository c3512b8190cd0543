"""Pins for the CPU oracle: brute force, closed forms, library routines and
hand-derived fixtures.  Each test is chosen so that a plausible slip in the
oracle (dropped term, wrong sign or index, transposed operand, wrong divisor,
wrong tie rule) fails it.  No test here needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synth import WORKLOADS, generate, topk_for_sparsity

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _sdpa(q, k, v, mask=None):
    """Library routine: torch scaled_dot_product_attention in float64 on CPU."""
    tq = torch.from_numpy(np.ascontiguousarray(q))[None, None]
    tk = torch.from_numpy(np.ascontiguousarray(k))[None, None]
    tv = torch.from_numpy(np.ascontiguousarray(v))[None, None]
    tm = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm)[0, 0].numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------ gate ---
def test_gate_golden():
    for case in _load("gate.json")["cases"]:
        s = oracle.gate(np.array(case["x"]), np.array(case["w"]), case["bias"])
        np.testing.assert_allclose(s, case["s"], rtol=0, atol=1e-15, err_msg=case["why"])


def test_gate_range_and_scipy():
    from scipy.special import expit
    x = _rand((3, 50, 16), 1)
    w = _rand(16, 2)
    s = oracle.gate(x, w, 0.3)
    assert np.all((s > 0) & (s < 1))
    np.testing.assert_allclose(s, expit(x.mean(axis=1) @ w + 0.3), rtol=1e-15)


# ------------------------------------------------------- block selection ---
def test_block_means_ragged_divisor():
    # N = 130 -> blocks of 64, 64, 2 rows; the last mean averages 2 rows.
    t = np.zeros((130, 3))
    t[:64, 0] = 1.0
    t[64:128, 0] = 2.0
    t[128:, 0] = [3.0, 5.0]
    t[:, 1] = np.arange(130)
    m = oracle.block_means(t, 64)
    assert m.shape == (3, 3)
    np.testing.assert_array_equal(m[:, 0], [1.0, 2.0, 4.0])
    np.testing.assert_array_equal(m[:, 1], [31.5, 95.5, 128.5])
    np.testing.assert_array_equal(m[:, 2], [0, 0, 0])


def test_block_scores_orientation_and_selection_closed_form():
    # Every query-block mean is e0; key block j rows all equal (j + 1) * e0, so
    # S[i, j] = j + 1 and the top-k are the last k blocks.  A ragged last key
    # block (2 rows) must still rank first.
    N, d, bs = 64 * 4 + 2, 4, 64
    q = np.zeros((N, d)); q[:, 0] = 1.0
    k = np.zeros((N, d))
    for j in range(5):
        k[j * bs:(j + 1) * bs, 0] = j + 1.0
    # Query rows of block 1 get a second component so S is not symmetric in
    # (i, j): only the key side carries the ranking.
    q[bs:2 * bs, 1] = 7.0
    S = oracle.block_scores(q, k, bs)
    assert S.shape == (5, 5)
    np.testing.assert_array_equal(S, np.tile(np.arange(1.0, 6.0), (5, 1)))
    idx = oracle.select_topk(S, 2)
    np.testing.assert_array_equal(idx, np.tile([3, 4], (5, 1)))


def test_select_topk_ties_lower_index_and_ascending_output():
    S = np.zeros((3, 6))
    np.testing.assert_array_equal(oracle.select_topk(S, 3), np.tile([0, 1, 2], (3, 1)))
    S = np.array([[5, 1, 5, 0, 5, 9.0]])
    # 9 (j=5) then the three 5s by index: j=0, 2 -> kept {0, 2, 5} for k=3.
    np.testing.assert_array_equal(oracle.select_topk(S, 3), [[0, 2, 5]])
    with pytest.raises(ValueError):
        oracle.select_topk(S, 7)


def test_select_topk_vs_python_sort_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(20):
        nb = int(rng.integers(2, 12))
        kk = int(rng.integers(1, nb + 1))
        S = rng.integers(-3, 4, size=(nb, nb)).astype(np.float64)  # many ties
        got = oracle.select_topk(S, kk)
        for i in range(nb):
            pairs = sorted(((float(S[i, j]), j) for j in range(nb)), key=lambda p: (-p[0], p[1]))
            want = sorted(j for _, j in pairs[:kk])
            assert list(got[i]) == want


# ---------------------------------------------------- Top-K attention ------
def _topk_mask(N, bs, idx):
    """Explicit additive mask M in {-inf, 0}^{N x N} for a block selection."""
    M = np.full((N, N), -np.inf)
    for r in range(N):
        for j in idx[r // bs]:
            M[r, j * bs:min(N, (j + 1) * bs)] = 0.0
    return M


@pytest.mark.parametrize("N,bs,kk", [(200, 64, 2), (256, 64, 1), (130, 64, 3), (97, 32, 2)])
def test_topk_attention_vs_masked_dense_sdpa(N, bs, kk):
    d = 16
    q, k, v = _rand((N, d), 10), _rand((N, d), 11), _rand((N, d), 12)
    idx = oracle.select_topk(oracle.block_scores(q, k, bs), kk)
    got = oracle.topk_attention(q, k, v, idx, bs)
    want = _sdpa(q, k, v, _topk_mask(N, bs, idx))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_topk_all_blocks_is_full_attention():
    N, d, bs = 150, 8, 32
    q, k, v = _rand((N, d), 20), _rand((N, d), 21), _rand((N, d), 22)
    nb = (N + bs - 1) // bs
    idx = oracle.select_topk(oracle.block_scores(q, k, bs), nb)
    np.testing.assert_allclose(oracle.topk_attention(q, k, v, idx, bs), _sdpa(q, k, v),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.dense_attention(q, k, v), _sdpa(q, k, v),
                               rtol=1e-12, atol=1e-12)


def test_topk_single_constant_block_gives_value_mean():
    # One kept block whose key rows are identical: all its scores are equal,
    # so every query's output is the plain mean of that block's value rows.
    N, d, bs = 128, 4, 64
    q = _rand((N, d), 30)
    k = np.zeros((N, d)); k[64:] = 2.0; k[:64] = _rand((64, d), 31)
    v = _rand((N, d), 32)
    idx = np.array([[1], [1]])
    got = oracle.topk_attention(q, k, v, idx, bs)
    np.testing.assert_allclose(got, np.tile(v[64:].mean(axis=0), (N, 1)), rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------- ST-SWA ----
def test_space_major_order_golden():
    g = _load("space_major_order.json")
    perm = oracle.space_major_order(g["F"], g["Hh"], g["Wh"])
    np.testing.assert_array_equal(perm, g["perm_r_to_t"])


def test_space_major_order_is_bijection_and_groups_frames():
    F, Hh, Wh = 3, 4, 5
    perm = oracle.space_major_order(F, Hh, Wh)
    assert sorted(perm.tolist()) == list(range(F * Hh * Wh))
    # Consecutive r within a group of F share the spatial position, frames 0..F-1.
    for r in range(F * Hh * Wh):
        t = perm[r]
        assert t // (Hh * Wh) == r % F
        assert t % (Hh * Wh) == r // F


@pytest.mark.parametrize("space_major", [False, True])
def test_swa_window_zero_returns_values(space_major):
    F, Hh, Wh, d = 3, 2, 5, 4
    N = F * Hh * Wh
    q, k, v = _rand((N, d), 40), _rand((N, d), 41), _rand((N, d), 42)
    got = oracle.swa_attention(q, k, v, 0, space_major, F, Hh, Wh)
    np.testing.assert_allclose(got, v, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("space_major", [False, True])
def test_swa_wide_window_is_full_attention(space_major):
    F, Hh, Wh, d = 2, 4, 9, 8
    N = F * Hh * Wh
    q, k, v = _rand((N, d), 50), _rand((N, d), 51), _rand((N, d), 52)
    got = oracle.swa_attention(q, k, v, N, space_major, F, Hh, Wh, chunk=16)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("W", [1, 5, 17])
def test_swa_vs_band_masked_sdpa(W):
    # Space-major head: reorder with the hand-checked permutation, apply a
    # band mask |r - c| <= W through the library attention, scatter back.
    F, Hh, Wh, d = 4, 3, 5, 8
    N = F * Hh * Wh
    q, k, v = _rand((N, d), 60 + W), _rand((N, d), 61 + W), _rand((N, d), 62 + W)
    r = np.arange(N)
    band = np.where(np.abs(r[:, None] - r[None, :]) <= W, 0.0, -np.inf)
    np.testing.assert_allclose(oracle.swa_attention(q, k, v, W, False, F, Hh, Wh, chunk=7),
                               _sdpa(q, k, v, band), rtol=1e-12, atol=1e-12)
    perm = np.array(oracle.space_major_order(F, Hh, Wh))
    o_perm = _sdpa(q[perm], k[perm], v[perm], band)
    want = np.empty_like(o_perm)
    want[perm] = o_perm
    np.testing.assert_allclose(oracle.swa_attention(q, k, v, W, True, F, Hh, Wh, chunk=9),
                               want, rtol=1e-12, atol=1e-12)


# -------------------------------------------------------- linear branch ----
def test_linear_golden():
    g = _load("linear_attention.json")
    H, Z = oracle.linear_state(np.array(g["k"]), np.array(g["v"]))
    np.testing.assert_array_equal(H, g["H"])
    np.testing.assert_array_equal(Z, g["Z"])
    q = np.array(g["q"])
    o0 = oracle.linear_apply(q[:2], H, Z, 0.0)
    np.testing.assert_allclose(o0, g["o_eps0"][:2], rtol=1e-15)
    o = oracle.linear_apply(q, H, Z, 1e-6)
    np.testing.assert_array_equal(o[2], [0.0, 0.0])
    np.testing.assert_allclose(o[:2], g["o_eps0"][:2], rtol=1e-6)


def test_linear_associativity_vs_quadratic_form():
    N, d, eps = 300, 16, 1e-6
    q, k, v = _rand((N, d), 70), _rand((N, d), 71), _rand((N, d), 72)
    H, Z = oracle.linear_state(k, v)
    got = oracle.linear_apply(q, H, Z, eps)
    A = np.maximum(q, 0) @ np.maximum(k, 0).T           # phi(Q) phi(K)^T, N x N
    want = (A @ v) / (A.sum(axis=1) + eps)[:, None]
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_linear_state_token_shuffle_invariant():
    N, d = 257, 8
    k, v = _rand((N, d), 80), _rand((N, d), 81)
    p = np.random.default_rng(82).permutation(N)
    H1, Z1 = oracle.linear_state(k, v)
    H2, Z2 = oracle.linear_state(k[p], v[p])
    np.testing.assert_allclose(H1, H2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Z1, Z2, rtol=1e-12, atol=1e-12)
    assert np.all(Z1 >= 0)


# ------------------------------------------------------- 3-D rotary code ---
def test_rope3d_angles_per_axis_closed_form():
    F, Hh, Wh, d = 3, 4, 5, 64
    N = F * Hh * Wh
    gt, gy, gx = oracle.rope3d_split(d)
    assert (gt, gy, gx) == (24, 20, 20) and oracle.rope3d_split(128) == (44, 42, 42)
    A = oracle.rope3d_angles(N, d, F, Hh, Wh, base=100.0)
    assert A.shape == (N, d // 2)
    f, y, x = 2, 3, 1
    t = (f * Hh + y) * Wh + x
    for i in range(gt // 2):
        assert math.isclose(A[t, i], f * 100.0 ** (-2 * i / gt), rel_tol=1e-13)
    for i in range(gy // 2):
        assert math.isclose(A[t, gt // 2 + i], y * 100.0 ** (-2 * i / gy), rel_tol=1e-13)
    for i in range(gx // 2):
        assert math.isclose(A[t, (gt + gy) // 2 + i], x * 100.0 ** (-2 * i / gx), rel_tol=1e-13)
    np.testing.assert_array_equal(A[0], 0.0)


def test_rope3d_rotation_is_complex_multiplication_and_relative():
    rng = np.random.default_rng(95)
    F, Hh, Wh, d = 2, 3, 4, 16
    N = F * Hh * Wh
    A = oracle.rope3d_angles(N, d, F, Hh, Wh)
    x = rng.standard_normal((N, d))
    r = oracle.rope3d_rotate(x, A)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * A)
    np.testing.assert_allclose(r[:, 0::2], z.real, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(r[:, 1::2], z.imag, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # (R_s a) . (R_t b) depends on the positions only through their difference:
    # the same vectors at two token pairs with equal (df, dy, dx) give one value.
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    tok = lambda f, yy, xx: (f * Hh + yy) * Wh + xx
    def dot(s_, t_):
        return float(oracle.rope3d_rotate(a[None], A[[s_]])[0] @ oracle.rope3d_rotate(b[None], A[[t_]])[0])
    assert math.isclose(dot(tok(0, 0, 1), tok(1, 1, 3)), dot(tok(0, 1, 0), tok(1, 2, 2)),
                        rel_tol=1e-12, abs_tol=1e-12)


def test_linear_branch_with_rope_vs_quadratic_form():
    # The rotation enters the numerator only: num_i = sum_j (R_i phi(q_i)) .
    # (R_j phi(k_j)) v_j, den_i = sum_j phi(q_i) . phi(k_j) + eps, written out
    # token pair by token pair.
    rng = np.random.default_rng(96)
    F, Hh, Wh, d = 2, 3, 5, 8
    N = F * Hh * Wh
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    A = oracle.rope3d_angles(N, d, F, Hh, Wh)
    Hst, Z = oracle.linear_state(k, v, A)
    got = oracle.linear_apply(q, Hst, Z, 1e-6, A)
    pq, pk = np.maximum(q, 0), np.maximum(k, 0)
    want = np.zeros((N, d))
    for i in range(N):
        num, den = np.zeros(d), 1e-6
        for j in range(N):
            qi = pq[i].copy(); kj = pk[j].copy()
            w_ = 0.0
            for m in range(d // 2):
                ai, aj = A[i, m], A[j, m]
                qa = (qi[2 * m] * math.cos(ai) - qi[2 * m + 1] * math.sin(ai),
                      qi[2 * m] * math.sin(ai) + qi[2 * m + 1] * math.cos(ai))
                ka = (kj[2 * m] * math.cos(aj) - kj[2 * m + 1] * math.sin(aj),
                      kj[2 * m] * math.sin(aj) + kj[2 * m + 1] * math.cos(aj))
                w_ += qa[0] * ka[0] + qa[1] * ka[1]
            num += w_ * v[j]
            den += float(qi @ kj)
        want[i] = num / den
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)
    # Z ignores the rotation; at a single token (every position 0) nothing turns.
    np.testing.assert_allclose(Z, pk.sum(axis=0), rtol=1e-13)
    H0, Z0 = oracle.linear_state(k[:1], v[:1], oracle.rope3d_angles(1, d, 1, 1, 1))
    H1, Z1 = oracle.linear_state(k[:1], v[:1])
    np.testing.assert_array_equal(H0, H1)


# ----------------------------------------------------- combine / forward ---
def _tiny_inputs(N=192, H=2, d=16, D=32, seed=90, B=1):
    rng = np.random.default_rng(seed)
    return {
        "q": rng.standard_normal((B, H, N, d)), "k": rng.standard_normal((B, H, N, d)),
        "v": rng.standard_normal((B, H, N, d)), "x": rng.standard_normal((B, N, D)),
        "w_gate": rng.normal(0, 0.5, D), "bias": 0.1,
        "w_lin": rng.normal(0, 0.2, (H, d, d)),
    }


def test_forward_gate_zero_is_sparse_branch_exactly():
    inp = _tiny_inputs()
    r = oracle.forward(inp, mode="topk", block=64, topk=2, gate_override=0.0)
    np.testing.assert_array_equal(r["o"], r["o_sparse"])
    inp["w_lin"] = np.zeros_like(inp["w_lin"])
    r = oracle.forward(inp, mode="topk", block=64, topk=2)
    np.testing.assert_array_equal(r["o"], r["o_sparse"])


def test_forward_branch_dropping_per_sample_threshold():
    # Step 8 of the method: a sample whose gate value is below the threshold
    # keeps only its sparse branch; the others are untouched.
    inp = _tiny_inputs(B=2, seed=93)
    inp["x"][1] += 0.5          # separates the two samples' gate values
    full = oracle.forward(inp, mode="topk", block=64, topk=2)
    s = full["s"]
    assert s[0] != s[1]
    lo, hi = sorted(range(2), key=lambda b: s[b])
    none = oracle.forward(inp, mode="topk", block=64, topk=2, drop_threshold=0.0)
    np.testing.assert_array_equal(none["o"], full["o"])
    assert not none["dropped"].any()
    both = oracle.forward(inp, mode="topk", block=64, topk=2, drop_threshold=1.0)
    np.testing.assert_array_equal(both["o"], full["o_sparse"])
    np.testing.assert_array_equal(both["o"],
                                  oracle.forward(inp, mode="topk", block=64, topk=2,
                                                 gate_override=0.0)["o"])
    mid = oracle.forward(inp, mode="topk", block=64, topk=2,
                         drop_threshold=float(s[lo] + s[hi]) / 2)
    assert mid["dropped"][lo] and not mid["dropped"][hi]
    np.testing.assert_array_equal(mid["o"][lo], full["o_sparse"][lo])
    np.testing.assert_array_equal(mid["o"][hi], full["o"][hi])
    # The comparison is strict: a gate value equal to the threshold is kept.
    at = oracle.forward(inp, mode="topk", block=64, topk=2, drop_threshold=float(s[lo]))
    assert not at["dropped"][lo]


def test_full_width_projection_reduces_and_orients():
    inp = _tiny_inputs(seed=97)
    H, d = 2, 16
    per_head = oracle.forward(inp, mode="topk", block=64, topk=2)
    # A block-diagonal full-width matrix is the per-head projection.
    W = np.zeros((H * d, H * d))
    for h in range(H):
        W[h * d:(h + 1) * d, h * d:(h + 1) * d] = inp["w_lin"][h]
    full = oracle.forward(inp, mode="topk", block=64, topk=2, w_lin_full=W)
    np.testing.assert_allclose(full["o"], per_head["o"], rtol=1e-12, atol=1e-13)
    # Identity: O_s + s * O_l.
    ident = oracle.forward(inp, mode="topk", block=64, topk=2, w_lin_full=np.eye(H * d))
    np.testing.assert_allclose(ident["o"], ident["o_sparse"] + ident["s"][0] * ident["o_lin"],
                               rtol=1e-12, atol=1e-13)
    # One entry W[h1*d + c1, h2*d + c2] = 1 moves column c1 of head h1's O_l
    # into column c2 of head h2, and nothing else.
    W = np.zeros((H * d, H * d)); W[0 * d + 3, 1 * d + 5] = 1.0
    one = oracle.forward(inp, mode="topk", block=64, topk=2, w_lin_full=W)
    diff = one["o"] - one["o_sparse"]
    np.testing.assert_allclose(diff[0, 1, :, 5], one["s"][0] * one["o_lin"][0, 0, :, 3], rtol=1e-12)
    diff[0, 1, :, 5] = 0.0
    np.testing.assert_array_equal(diff, 0.0)


def test_full_width_golden():
    # Hand-derived worked example (tests/golden/full_width_projection.json).
    g = json.load(open(os.path.join(GOLD, "full_width_projection.json")))
    o = oracle.combine_full(np.array(g["o_sparse"]), np.array(g["o_lin"]), np.array(g["w_full"]),
                            g["s"])
    np.testing.assert_array_equal(o, np.array(g["o"]))
    out = oracle.output_projection(o, np.array(g["w_out"]))
    np.testing.assert_array_equal(out, np.array(g["out"]))


def test_output_projection_orients():
    inp = _tiny_inputs(seed=98)
    H, d, N = 2, 16, 192
    r = oracle.forward(inp, mode="topk", block=64, topk=2, w_out=np.eye(H * d))
    np.testing.assert_array_equal(r["out"][0], r["o"][0].transpose(1, 0, 2).reshape(N, H * d))
    Wo = np.zeros((H * d, 7)); Wo[1 * d + 2, 4] = 1.0
    r = oracle.forward(inp, mode="topk", block=64, topk=2, w_out=Wo)
    np.testing.assert_array_equal(r["out"][0][:, 4], r["o"][0, 1, :, 2])
    assert not np.any(np.delete(r["out"][0], 4, axis=1))


def test_forward_linear_in_gate_and_projection():
    inp = _tiny_inputs(seed=91)
    r1 = oracle.forward(inp, mode="topk", block=64, topk=2, gate_override=0.25)
    r2 = oracle.forward(inp, mode="topk", block=64, topk=2, gate_override=0.5)
    np.testing.assert_allclose(r2["o"] - r2["o_sparse"], 2 * (r1["o"] - r1["o_sparse"]),
                               rtol=1e-12, atol=1e-13)
    # The projection right-multiplies rows: with W_lin = identity the term is O_l.
    inp["w_lin"] = np.stack([np.eye(16)] * 2)
    r = oracle.forward(inp, mode="topk", block=64, topk=2, gate_override=1.0)
    np.testing.assert_allclose(r["o"] - r["o_sparse"], r["o_lin"], rtol=1e-12, atol=1e-13)
    # A non-symmetric W_lin distinguishes O_l W from W O_l^T.
    W = np.zeros((16, 16)); W[0, 1] = 1.0
    inp["w_lin"] = np.stack([W, W])
    r = oracle.forward(inp, mode="topk", block=64, topk=2, gate_override=1.0)
    diff = r["o"] - r["o_sparse"]
    np.testing.assert_allclose(diff[..., 1], r["o_lin"][..., 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(diff[..., 0], 0.0)


def test_forward_modes_agree_at_full_coverage():
    inp = _tiny_inputs(N=130, seed=92)
    rt = oracle.forward(inp, mode="topk", block=64, topk=3)
    rd = oracle.forward(inp, mode="dense")
    rs = oracle.forward(inp, mode="swa", window=200, space_major_heads=(0,), F=2, Hh=5, Wh=13)
    np.testing.assert_allclose(rt["o"], rd["o"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(rs["o"], rd["o"], rtol=1e-12, atol=1e-12)
    for h in range(2):
        np.testing.assert_allclose(rd["o_sparse"][0, h],
                                   _sdpa(inp["q"][0, h], inp["k"][0, h], inp["v"][0, h]),
                                   rtol=1e-12, atol=1e-12)


def test_near_tie_rule():
    row = np.array([3.0, 2.0, 2.0 + 1e-9, 1.0])
    assert oracle.near_tie_equivalent(row, [0, 2], [0, 2])
    assert oracle.near_tie_equivalent(row, [0, 2], [0, 1])      # k-th vs (k+1)-th tie
    assert not oracle.near_tie_equivalent(row, [0, 2], [0, 3])  # 1.0 is far below
    row2 = np.array([3.0, 2.0, 2.5, 1.0])
    assert not oracle.near_tie_equivalent(row2, [0, 2], [0, 1])


# ------------------------------------------------------------- workloads ---
def test_workload_shapes_match_the_stated_configs():
    w = WORKLOADS["topk480"]
    assert (w.N, w.nb, w.topk) == (31200, 488, 49)
    w = WORKLOADS["topk720"]
    assert (w.N, w.nb, w.topk) == (100800, 1575, 158)
    assert WORKLOADS["tiny"].N == 1024 and WORKLOADS["tiny"].nb == 16
    assert WORKLOADS["swa480"].window == 1560 == 30 * 52
    assert [WORKLOADS[f"cfg_b2h40_s{s}"].topk for s in (80, 90, 95)] == [98, 49, 25]
    assert topk_for_sparsity(488, 0.9) == 49


def test_generator_is_seeded_and_head_subset_consistent():
    w = WORKLOADS["tiny"]
    a = generate(w)
    b = generate(w, heads=[1])
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (1, 2, 1024, 64)
    assert torch.equal(a["q"][:, 1:2], b["q"]) and torch.equal(a["v"][:, 1:2], b["v"])
    assert torch.equal(a["w_lin"][1:2], b["w_lin"])
    c = generate(w)
    assert torch.equal(a["k"], c["k"]) and torch.equal(a["x"], c["x"])


def test_tiny_workload_oracle_end_to_end_properties():
    w = WORKLOADS["tiny"]
    inp = generate(w)
    r = oracle.forward(inp, mode="topk", block=w.block, topk=w.topk)
    assert r["idx"].shape == (1, 2, 16, 2)
    assert np.all(np.diff(r["idx"], axis=-1) > 0)
    assert 0 < r["s"][0] < 1
    assert np.all(np.isfinite(r["o"]))
