"""CPU oracle for the SALAD hybrid-attention forward pass (float64, numpy).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it and shares no code with it.

Every function restates one step of the method as the SALAD pages give it, in
float64, with no blocking, fusion or reordering beyond what the step states.
Sources (page title, then section):
  * "SALAD ... (paper.rainbus.top)": 前置知识 -- Sparse Attention (mask
    M in {-inf, 0}^{N x N}), Linear Attention (H = phi(K)^T V, Z = phi(K)^T 1,
    O = phi(Q) H / (phi(Q) Z), phi = ReLU); 方法步骤详情 steps 2-6 (sparse branch
    O_s, linear branch O_l, zero-init projection O_l' = ZeroInitProj(O_l),
    sigmoid gate s, residual O~ = O_s + s * O_l'), step 8 (optional dropping
    of linear branches whose gate value is small).
  * "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)": 1.1 (ST-SWA: frame-major
    flattening, per-head regrouping by spatial position, 1-D sliding window),
    1.2 (Top-K: block partition, block mean vectors, similarity to key-block
    means, keep Top-K blocks, attend only to them), 2.3 (gate: token mean ->
    linear -> sigmoid), 3.1-3.2 (post-training branch pruning below a
    gate-value threshold).
Readings where the pages are silent (each is listed in the design notes):
  softmax scale 1/sqrt(d); query side of the selection pooled per query block;
  block means over valid rows only; no forced blocks; ties broken towards the
  lower block index; eps = 1e-6 added to the linear-attention denominator;
  gate s = sigmoid(w . mean_tokens(X) + b) with X already time-modulated;
  W_lin per head, d x d, right-multiplying row vectors; the 3-D rotary
  encoding of the linear branch (optional) rotates adjacent channel pairs of
  phi(q) and phi(k) in the numerator only, channel groups (frame, row,
  column) of d - 4*floor(d/6), 2*floor(d/6), 2*floor(d/6) channels, base
  10000; space-major order r = (y * Wh + x) * F + f; window
  |r - c| <= W clipped at the sequence ends.

Parity pins: every function here is checked by ``tests/test_oracle_pins.py``
against brute force, closed forms, library routines or hand-derived fixtures.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence

import numpy as np

__all__ = [
    "as64", "gate", "block_means", "block_scores", "select_topk",
    "topk_attention_rows", "topk_attention", "space_major_order",
    "swa_attention_rows", "swa_attention", "dense_attention",
    "rope3d_split", "rope3d_angles", "rope3d_rotate",
    "linear_state", "linear_apply", "combine", "combine_full", "output_projection",
    "forward",
    "near_tie_equivalent",
]


def as64(t) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> float64 numpy array (exact)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


# ----------------------------------------------------------------- gate ----
def gate(x: np.ndarray, w: np.ndarray, bias: float) -> np.ndarray:
    """Input-aware scalar gate, one value per batch sample.

    "SALAD ... (paper.rainbus.top)" 方法步骤详情 step 5 and
    "视频扩散模型中的稀疏注意力机制解析" 2.3: average the hidden state over tokens,
    apply a linear map, then a sigmoid.  x: [B, N, D]; w: [D]; returns s [B].
    """
    x = as64(x)
    w = as64(w)
    xbar = x.mean(axis=1)                      # token mean   [B, D]
    z = xbar @ w + float(bias)                 # linear       [B]
    return 1.0 / (1.0 + np.exp(-z))            # sigmoid      [B]


# ------------------------------------------------------ Top-K selection ----
def block_means(t: np.ndarray, block: int) -> np.ndarray:
    """Mean vector of each block of ``block`` consecutive rows (valid rows only).

    "视频扩散模型中的稀疏注意力机制解析" 1.2, step "块划分与均值计算".
    t: [N, d] -> [nb, d], nb = ceil(N / block); the last block averages the
    rows it actually holds.
    """
    t = as64(t)
    N = t.shape[0]
    nb = (N + block - 1) // block
    out = np.empty((nb, t.shape[1]), np.float64)
    for i in range(nb):
        rows = t[i * block:min(N, (i + 1) * block)]
        out[i] = rows.sum(axis=0) / rows.shape[0]
    return out


def block_scores(q: np.ndarray, k: np.ndarray, block: int) -> np.ndarray:
    """Similarity of every query-block mean with every key-block mean.

    "视频扩散模型中的稀疏注意力机制解析" 1.2, step "相似度筛选": dot products of
    block means (unscaled; the ranking does not depend on a scale).
    q, k: [N, d] -> [nb, nb] with S[i, j] = qbar_i . kbar_j.
    """
    return block_means(q, block) @ block_means(k, block).T


def select_topk(scores: np.ndarray, topk: int) -> np.ndarray:
    """For each query block, the ``topk`` key blocks of largest score.

    Order: score descending, then block index ascending (tie rule).  The kept
    indices are returned in ascending order.  scores: [nb, nb] -> [nb, topk].
    """
    nb = scores.shape[1]
    if not 1 <= topk <= nb:
        raise ValueError("topk must be in [1, nb]")
    out = np.empty((scores.shape[0], topk), np.int64)
    cols = np.arange(nb)
    for i in range(scores.shape[0]):
        # np.lexsort sorts by the last key first: (-score) then column index.
        order = np.lexsort((cols, -scores[i]))
        out[i] = np.sort(order[:topk])
    return out


def _softmax_attend(q_rows, k_cols, v_cols, extra_mask=None) -> np.ndarray:
    """softmax(q k^T / sqrt(d) + M) v for a set of rows, max-subtracted."""
    d = q_rows.shape[1]
    s = (q_rows @ k_cols.T) / math.sqrt(d)
    if extra_mask is not None:
        s = s + extra_mask
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ v_cols) / p.sum(axis=1, keepdims=True)


def topk_attention_rows(q, k, v, idx, block: int, qblocks: Iterable[int]) -> Dict[int, np.ndarray]:
    """Top-K block-sparse attention for the listed query blocks of one head.

    "视频扩散模型中的稀疏注意力机制解析" 1.2, step "局部注意力计算": each query
    token attends only to the tokens of the key blocks selected for its block.
    q, k, v: [N, d]; idx: [nb, topk].  Returns {i: [rows_i, d]}.
    """
    q, k, v = as64(q), as64(k), as64(v)
    N = q.shape[0]
    out = {}
    for i in qblocks:
        rows = slice(i * block, min(N, (i + 1) * block))
        cols = np.concatenate([np.arange(j * block, min(N, (j + 1) * block)) for j in idx[i]])
        out[i] = _softmax_attend(q[rows], k[cols], v[cols])
    return out


def topk_attention(q, k, v, idx, block: int) -> np.ndarray:
    """Top-K block-sparse attention over all query blocks of one head: [N, d]."""
    q = as64(q)
    nb = idx.shape[0]
    res = topk_attention_rows(q, k, v, idx, block, range(nb))
    return np.concatenate([res[i] for i in range(nb)], axis=0)


# -------------------------------------------------------------- ST-SWA ----
def space_major_order(F: int, Hh: int, Wh: int) -> np.ndarray:
    """Token permutation of the spatio-temporal sliding window.

    "视频扩散模型中的稀疏注意力机制解析" 1.1: the latent is flattened with time
    slowest, t = (f * Hh + y) * Wh + x; heads with temporal locality regroup the
    tokens by spatial position so that one position's frames are adjacent:
    r = (y * Wh + x) * F + f.  Returns perm with perm[r] = t.
    """
    perm = np.empty(F * Hh * Wh, np.int64)
    for f in range(F):
        for y in range(Hh):
            for x in range(Wh):
                t = (f * Hh + y) * Wh + x
                r = (y * Wh + x) * F + f
                perm[r] = t
    return perm


def swa_attention_rows(q, k, v, window: int, rows: Sequence[int]) -> np.ndarray:
    """Sliding-window attention for the listed rows of one (already ordered) head.

    Row r attends to every key c with |r - c| <= window, clipped to [0, N).
    The band is written as the page's additive mask M in {-inf, 0}.
    """
    q, k, v = as64(q), as64(k), as64(v)
    N = q.shape[0]
    rows = np.asarray(list(rows), np.int64)
    lo = max(0, int(rows.min()) - window)
    hi = min(N, int(rows.max()) + window + 1)
    cols = np.arange(lo, hi)
    mask = np.where(np.abs(rows[:, None] - cols[None, :]) <= window, 0.0, -np.inf)
    return _softmax_attend(q[rows], k[cols], v[cols], mask)


def swa_attention(q, k, v, window: int, space_major: bool, F: int, Hh: int, Wh: int,
                  chunk: int = 64) -> np.ndarray:
    """ST-SWA for one head in frame-major token order: [N, d].

    A space-major head is reordered, attended with the 1-D window, and its
    output rows are put back at their frame-major positions.
    """
    q, k, v = as64(q), as64(k), as64(v)
    N = q.shape[0]
    if space_major:
        perm = space_major_order(F, Hh, Wh)
        qo, ko, vo = q[perm], k[perm], v[perm]
    else:
        qo, ko, vo = q, k, v
    out_o = np.empty_like(qo)
    for r0 in range(0, N, chunk):
        rows = np.arange(r0, min(N, r0 + chunk))
        out_o[rows] = swa_attention_rows(qo, ko, vo, window, rows)
    if not space_major:
        return out_o
    out = np.empty_like(out_o)
    out[perm] = out_o
    return out


def dense_attention(q, k, v) -> np.ndarray:
    """Full softmax attention softmax(Q K^T / sqrt(d)) V for one head."""
    q, k, v = as64(q), as64(k), as64(v)
    out = np.empty_like(q)
    for r0 in range(0, q.shape[0], 256):
        out[r0:r0 + 256] = _softmax_attend(q[r0:r0 + 256], k, v)
    return out


# ------------------------------------------------------ linear branch -----
def rope3d_split(d: int):
    """Channel groups (frame, row, column) of the 3-D rotary encoding.

    The pages give no split (reading): 2*floor(d/6) channels each for the row
    and column positions, the remaining channels for the frame position, in
    that order: d = 128 -> (44, 42, 42).
    """
    dy = 2 * (d // 6)
    return d - 2 * dy, dy, dy


def rope3d_angles(N: int, d: int, F: int, Hh: int, Wh: int, base: float = 10000.0) -> np.ndarray:
    """Rotation angle of each channel pair of each token: [N, d // 2].

    Token t (frame-major) sits at frame f = t // (Hh*Wh), row y = (t // Wh) %
    Hh, column x = t % Wh.  Pair i of a group with g channels turns by
    position * base^(-2i/g) (the rotary encoding, applied per axis).
    """
    assert F * Hh * Wh == N
    t = np.arange(N)
    pos = (t // (Hh * Wh), (t // Wh) % Hh, t % Wh)
    cols = []
    for g, p in zip(rope3d_split(d), pos):
        theta = base ** (-2.0 * np.arange(g // 2) / g)
        cols.append(np.outer(p, theta))
    return np.concatenate(cols, axis=1)


def rope3d_rotate(x, angles) -> np.ndarray:
    """Turns each adjacent channel pair (2i, 2i+1) of each row by its angle."""
    x = as64(x)
    a, b = x[:, 0::2], x[:, 1::2]
    c, s = np.cos(angles), np.sin(angles)
    out = np.empty_like(x)
    out[:, 0::2] = a * c - b * s
    out[:, 1::2] = a * s + b * c
    return out


def linear_state(k, v, angles=None):
    """H = phi(K)^T V and Z = phi(K)^T 1 with phi = ReLU, for one head.

    "SALAD ... (paper.rainbus.top)" 前置知识 Linear Attention.  k, v: [N, d]
    -> H [d, d], Z [d].  With ``angles`` (the 3-D rotary encoding the linear
    branch integrates, 方法步骤详情 step 3), H sums the rotated features
    R_j phi(k_j) v_j^T; Z stays unrotated (reading: the rotation enters the
    numerator only, which keeps the denominator positive).
    """
    k, v = as64(k), as64(v)
    pk = np.maximum(k, 0.0)
    rk = pk if angles is None else rope3d_rotate(pk, angles)
    return rk.T @ v, pk.sum(axis=0)


def linear_apply(q, Hst, Z, eps: float, angles=None) -> np.ndarray:
    """O_l = phi(Q) H / (phi(Q) Z + eps) for one head: [N, d].  With
    ``angles`` the numerator uses the rotated R_i phi(q_i)."""
    q = as64(q)
    pq = np.maximum(q, 0.0)
    rq = pq if angles is None else rope3d_rotate(pq, angles)
    return (rq @ Hst) / ((pq @ Z) + eps)[:, None]


# ------------------------------------------------------------ combine -----
def combine(o_sparse, o_lin, w_lin_h, s: float) -> np.ndarray:
    """O = O_s + s * (O_l W_lin) for one head (steps 4 and 6 of the method)."""
    return as64(o_sparse) + float(s) * (as64(o_lin) @ as64(w_lin_h))


def combine_full(o_sparse, o_lin, w_full, s: float) -> np.ndarray:
    """O = O_s + s * (O_l W_full) with the projection over all heads.

    Reading of the zero-init projection as one full-width linear layer (its
    share of the parameters in "SALAD ... (paper.rainbus.top)" suggests a
    full-width layer; 方法步骤详情 step 4): the heads' linear outputs of a token
    are concatenated (head-major: column h*d + c), multiplied by w_full
    [H*d, H*d] as a row vector, and split back into heads.  o_sparse, o_lin:
    [H, N, d] of one sample.
    """
    o_sparse, o_lin, w_full = as64(o_sparse), as64(o_lin), as64(w_full)
    H, N, d = o_lin.shape
    cat = o_lin.transpose(1, 0, 2).reshape(N, H * d)
    mixed = (cat @ w_full).reshape(N, H, d).transpose(1, 0, 2)
    return o_sparse + float(s) * mixed


def output_projection(o, w_out) -> np.ndarray:
    """The final projection of 方法步骤详情 step 7: the heads of a token
    concatenated (column h*d + c) times w_out [H*d, D_out].  o: [H, N, d] of
    one sample -> [N, D_out]."""
    o = as64(o)
    H, N, d = o.shape
    return o.transpose(1, 0, 2).reshape(N, H * d) @ as64(w_out)


# ------------------------------------------------------------ forward -----
def forward(inp: Dict, *, mode: str, block: int = 64, topk: int = 0, window: int = 0,
            space_major_heads: Sequence[int] = (), F: int = 0, Hh: int = 0, Wh: int = 0,
            eps: float = 1e-6, gate_override: Optional[float] = None,
            idx_override: Optional[np.ndarray] = None,
            drop_threshold: float = 0.0, rope3d: bool = False,
            rope_base: float = 10000.0, w_lin_full=None,
            w_out=None) -> Dict[str, np.ndarray]:
    """The whole hybrid layer, in the step order of the method.

    inp: q, k, v [B, H, N, d]; x [B, N, D]; w_gate [D]; bias; w_lin [H, d, d].
    mode: "topk" | "swa" | "dense".  ``idx_override`` replaces the selection
    (used when another correct selection is compared at a near tie).
    ``drop_threshold``: post-training branch dropping ("SALAD ...
    (paper.rainbus.top)" 方法步骤详情 step 8; "视频扩散模型中的稀疏注意力机制解析"
    3.1-3.2): a sample whose gate value s_b is below the threshold keeps only
    its sparse branch, O = O_sparse (0 never drops, since s_b > 0).
    Returns s [B], idx [B, H, nb, topk] (topk mode), scores, o_sparse, o_lin,
    o and dropped [B].  ``rope3d``: the linear branch integrates the 3-D
    rotary encoding over the (F, Hh, Wh) grid of the tokens (see
    ``linear_state``).  ``w_lin_full`` [H*d, H*d]: the projection of the
    linear branch mixes the heads (``combine_full``) instead of the per-head
    ``w_lin``.  ``w_out`` [H*d, D_out]: also return ``out`` [B, N, D_out],
    the output projection of the combined heads (step 7).
    """
    q, k, v = as64(inp["q"]), as64(inp["k"]), as64(inp["v"])
    B, H, N, d = q.shape
    s = gate(inp["x"], inp["w_gate"], inp["bias"]) if gate_override is None \
        else np.full(B, float(gate_override))
    w_lin = as64(inp["w_lin"])
    nb = (N + block - 1) // block
    o_sparse = np.empty_like(q)
    o_lin = np.empty_like(q)
    o = np.empty_like(q)
    angles = rope3d_angles(N, d, F, Hh, Wh, rope_base) if rope3d else None
    idx = np.zeros((B, H, nb, max(topk, 1)), np.int64) if mode == "topk" else None
    scores = np.zeros((B, H, nb, nb)) if mode == "topk" else None
    for b in range(B):
        for h in range(H):
            if mode == "topk":
                scores[b, h] = block_scores(q[b, h], k[b, h], block)
                idx[b, h] = select_topk(scores[b, h], topk) if idx_override is None \
                    else idx_override[b, h]
                o_sparse[b, h] = topk_attention(q[b, h], k[b, h], v[b, h], idx[b, h], block)
            elif mode == "swa":
                o_sparse[b, h] = swa_attention(q[b, h], k[b, h], v[b, h], window,
                                               h in space_major_heads, F, Hh, Wh)
            elif mode == "dense":
                o_sparse[b, h] = dense_attention(q[b, h], k[b, h], v[b, h])
            else:
                raise ValueError(mode)
            Hst, Z = linear_state(k[b, h], v[b, h], angles)
            o_lin[b, h] = linear_apply(q[b, h], Hst, Z, eps, angles)
            if s[b] < drop_threshold:
                o[b, h] = o_sparse[b, h]
            elif w_lin_full is None:
                o[b, h] = combine(o_sparse[b, h], o_lin[b, h], w_lin[h], s[b])
        if w_lin_full is not None and not s[b] < drop_threshold:
            o[b] = combine_full(o_sparse[b], o_lin[b], w_lin_full, s[b])
    out = None
    if w_out is not None:
        out = np.stack([output_projection(o[b], w_out) for b in range(B)])
    return {"s": s, "idx": idx, "scores": scores, "o_sparse": o_sparse,
            "o_lin": o_lin, "o": o, "dropped": s < drop_threshold, "out": out}


# ------------------------------------------------- selection comparison ---
def near_tie_equivalent(scores_row: np.ndarray, idx_ref: Sequence[int], idx_other: Sequence[int],
                        rel: float = 1e-5) -> bool:
    """Whether another kept set is an acceptable answer at a near tie.

    Equal sets always pass.  Otherwise the reference's k-th and (k+1)-th
    largest scores must lie within ``rel`` (relative) of each other, and every
    block that differs between the two sets must score within that band.
    """
    a, b = set(int(x) for x in idx_ref), set(int(x) for x in idx_other)
    if a == b:
        return True
    if len(b) != len(a) or len(b) != len(list(idx_other)):
        return False
    srt = np.sort(scores_row)[::-1]
    kk = len(a)
    if kk >= len(srt):
        return False
    sk, sk1 = srt[kk - 1], srt[kk]
    scale = max(abs(sk), abs(sk1), np.finfo(np.float64).tiny)
    if abs(sk - sk1) >= rel * scale:
        return False
    band_lo, band_hi = sk1 - rel * scale, sk + rel * scale
    for j in a.symmetric_difference(b):
        if not band_lo <= scores_row[j] <= band_hi:
            return False
    return True
