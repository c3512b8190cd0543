"""Seeded synthetic inputs for the SALAD hybrid-attention forward pass.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA path read
the same bytes produced here.

Workloads follow the video-DiT shapes the SALAD pages describe (Wan2.1 latents:
about 30k tokens at 480p x 77 frames, about 100k at 720p; page "SALAD ...
(paper.rainbus.top)", section 前置知识 / 研究动机).  No dataset, prompt or trained
weight is used: every tensor is a seeded draw.

Recipe (per batch sample b, per head h):
  * Q, K, V ~ N(0, 1) per element, drawn in float32 and rounded to bfloat16
    with round-to-nearest-even.
  * For the video-shaped workloads a per-frame low-rank component is added so
    that block means are informative: a basis U in R^{r x d} with entries
    N(0, 1/r) and per-frame coefficients a_f in R^r ~ N(0, 1); every Q row and
    every K row of frame f gets ``scale * a_f @ U`` (shared by Q and K), and V
    gets its own independently drawn component of the same form.
  * Tokens are flattened frame-major: t = (f * Hh + y) * Wh + x.
  * Gate input X ~ N(0, 1) [B, N, D]; gate weight w ~ N(0, 0.02) [D]; bias 0.
  * Per-head linear-branch projection W_lin ~ N(0, 0.02) [H, d, d].
  * Full-width variants (``generate_projections``): W_lin_full ~ N(0, 0.02)
    [H*d, H*d] and the output projection W_out ~ N(0, 0.02) [H*d, D_out],
    from their own stream (seed sequence [seed_0, 0x5A1AD]).
Random streams: numpy PCG64 seeded by ``SeedSequence(seed_b).spawn(...)``, one
child stream per tensor.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "generate", "generate_device", "generate_projections",
           "topk_for_sparsity"]


def topk_for_sparsity(nb: int, sparsity: float) -> int:
    """Key blocks kept per query block for a target sparsity: ceil((1-s)*nb)."""
    return max(1, int(math.ceil(round((1.0 - sparsity) * nb, 9))))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    F: int
    Hh: int
    Wh: int
    D: int
    mode: str = "topk"            # "topk" | "swa" | "dense"
    block: int = 64
    topk: int = 0                 # key blocks per query block (topk mode)
    window: int = 0               # half-width |r - c| <= window (swa mode)
    space_major_heads: tuple = () # heads reordered space-major (swa mode)
    lowrank_rank: int = 8
    lowrank_scale: float = 0.0
    seeds: tuple = (0,)           # one seed per batch sample
    eps: float = 1e-6
    bias: float = 0.0

    @property
    def N(self) -> int:
        return self.F * self.Hh * self.Wh

    @property
    def nb(self) -> int:
        return (self.N + self.block - 1) // self.block

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> Dict:
        out = dataclasses.asdict(self)
        out["N"] = self.N
        out["nb"] = self.nb
        out["space_major_heads"] = list(self.space_major_heads)
        out["seeds"] = list(self.seeds)
        return out


def _topk480() -> Workload:
    w = Workload(name="topk480", B=1, H=12, d=128, F=20, Hh=30, Wh=52, D=1536,
                 mode="topk", lowrank_scale=0.5)
    return w.with_(topk=topk_for_sparsity(w.nb, 0.90))


def _topk720() -> Workload:
    w = Workload(name="topk720", B=1, H=40, d=128, F=28, Hh=45, Wh=80, D=5120,
                 mode="topk", lowrank_scale=0.5)
    return w.with_(topk=topk_for_sparsity(w.nb, 0.90))


def _sweep(sparsity: Optional[float]) -> Workload:
    w = Workload(name="cfg_b2h40", B=2, H=40, d=128, F=20, Hh=30, Wh=52, D=5120,
                 mode="topk", lowrank_scale=0.5, seeds=(0, 1))
    k = w.nb if sparsity is None else topk_for_sparsity(w.nb, sparsity)
    tag = "all" if sparsity is None else f"s{int(round(sparsity * 100))}"
    return w.with_(name=f"cfg_b2h40_{tag}", topk=k)


WORKLOADS: Dict[str, Workload] = {
    # 4x16x16 latent, two heads of d=64, 16 blocks, 2 kept per query block.
    "tiny": Workload(name="tiny", B=1, H=2, d=64, F=4, Hh=16, Wh=16, D=128,
                     mode="topk", topk=2, lowrank_scale=0.0),
    # 480p-like: 20x30x52 latent (N=31200, 488 blocks), 90% sparsity (k=49).
    "topk480": _topk480(),
    # Same shapes and values, spatio-temporal sliding window: heads 0..5 are
    # reordered space-major, window half-width 1560 tokens (one frame).
    "swa480": _topk480().with_(name="swa480", mode="swa", topk=0, window=1560,
                               space_major_heads=tuple(range(6))),
    # 720p-like long sequence: 28x45x80 latent (N=100800, 1575 blocks), k=158.
    "topk720": _topk720(),
    # The 720p layer with 8 of its 40 heads (the same N, k and values per head):
    # a case small enough for profiler captures of the 720p kernels.
    "topk720_h8": _topk720().with_(name="topk720_h8", H=8, D=1024),
    # Batch of two independent samples, 40 heads, sparsity sweep + all blocks.
    "cfg_b2h40_s80": _sweep(0.80),
    "cfg_b2h40_s90": _sweep(0.90),
    "cfg_b2h40_s95": _sweep(0.95),
    "cfg_b2h40_all": _sweep(None),
}


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _sample_qkv(w: Workload, seed: int, heads: List[int]):
    """Q, K, V float32 [len(heads), N, d] for one batch sample."""
    ss = np.random.SeedSequence(seed)
    ch = ss.spawn(9)
    N, d = w.N, w.d
    rq, rk, rv = (np.random.Generator(np.random.PCG64(c)) for c in ch[0:3])
    rb_qk = np.random.Generator(np.random.PCG64(ch[3]))
    rc_qk = np.random.Generator(np.random.PCG64(ch[4]))
    rb_v = np.random.Generator(np.random.PCG64(ch[5]))
    rc_v = np.random.Generator(np.random.PCG64(ch[6]))
    frame_of_token = np.arange(N) // (w.Hh * w.Wh)
    q = np.empty((len(heads), N, d), np.float32)
    k = np.empty_like(q)
    v = np.empty_like(q)
    for hi in range(w.H):
        # Every head's draws are taken, in head order, so a subset of heads
        # reproduces exactly the values of the full tensor.
        nq = rq.standard_normal((N, d), dtype=np.float32)
        nk = rk.standard_normal((N, d), dtype=np.float32)
        nv = rv.standard_normal((N, d), dtype=np.float32)
        r = w.lowrank_rank
        u_qk = rb_qk.standard_normal((r, d)) / math.sqrt(r)
        a_qk = rc_qk.standard_normal((w.F, r))
        u_v = rb_v.standard_normal((r, d)) / math.sqrt(r)
        a_v = rc_v.standard_normal((w.F, r))
        if hi not in heads:
            continue
        j = heads.index(hi)
        if w.lowrank_scale != 0.0:
            lr_qk = (w.lowrank_scale * (a_qk @ u_qk)).astype(np.float32)[frame_of_token]
            lr_v = (w.lowrank_scale * (a_v @ u_v)).astype(np.float32)[frame_of_token]
            nq += lr_qk
            nk += lr_qk
            nv += lr_v
        q[j], k[j], v[j] = nq, nk, nv
    return q, k, v, ch


def generate(w: Workload, heads: Optional[List[int]] = None) -> Dict[str, torch.Tensor]:
    """Draw all inputs of one layer as CPU tensors.

    Returns q, k, v: bf16 [B, Hsel, N, d]; x: bf16 [B, N, D]; w_gate: bf16 [D];
    w_lin: bf16 [Hsel, d, d]; bias: python float.  ``heads`` selects a subset
    of heads (values identical to the same heads of the full draw).
    """
    heads = list(range(w.H)) if heads is None else list(heads)
    B = w.B
    qs, ks, vs, xs = [], [], [], []
    params_ch = None
    for b in range(B):
        seed = w.seeds[b] if b < len(w.seeds) else w.seeds[0] + 7919 * b
        q, k, v, ch = _sample_qkv(w, seed, heads)
        qs.append(_bf16(q)); ks.append(_bf16(k)); vs.append(_bf16(v))
        del q, k, v
        rx = np.random.Generator(np.random.PCG64(ch[7]))
        xs.append(_bf16(rx.standard_normal((w.N, w.D), dtype=np.float32)))
        if b == 0:
            params_ch = ch[8]
    rp = np.random.Generator(np.random.PCG64(params_ch))
    w_gate = _bf16(rp.normal(0.0, 0.02, size=(w.D,)))
    w_lin_all = rp.normal(0.0, 0.02, size=(w.H, w.d, w.d))
    w_lin = _bf16(w_lin_all[heads])
    return {
        "q": torch.stack(qs), "k": torch.stack(ks), "v": torch.stack(vs),
        "x": torch.stack(xs), "w_gate": w_gate, "w_lin": w_lin,
        "bias": float(w.bias),
    }


def generate_device(w: Workload, device, seed: int = 0) -> Dict[str, torch.Tensor]:
    """The same recipe as ``generate`` drawn on the device with torch's
    generator: the same distributions, shapes and frame structure, not the
    same bytes.  For timing runs at sizes whose host-side draws would take
    minutes; parity checks use ``generate``."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + 12345)
    B, H, N, d, r = w.B, w.H, w.N, w.d, w.lowrank_rank
    frame = torch.arange(N, device=device) // (w.Hh * w.Wh)

    def qkv():
        out = []
        for _ in range(3):
            out.append(torch.randn(B, H, N, d, generator=g, device=device, dtype=torch.float32))
        q, k, v = out
        if w.lowrank_scale != 0.0:
            for b in range(B):
                for h in range(H):
                    u_qk = torch.randn(r, d, generator=g, device=device) / math.sqrt(r)
                    a_qk = torch.randn(w.F, r, generator=g, device=device)
                    u_v = torch.randn(r, d, generator=g, device=device) / math.sqrt(r)
                    a_v = torch.randn(w.F, r, generator=g, device=device)
                    lr_qk = (w.lowrank_scale * (a_qk @ u_qk))[frame]
                    q[b, h] += lr_qk
                    k[b, h] += lr_qk
                    v[b, h] += (w.lowrank_scale * (a_v @ u_v))[frame]
        return [t.to(torch.bfloat16) for t in (q, k, v)]

    q, k, v = qkv()
    x = torch.randn(B, N, w.D, generator=g, device=device).to(torch.bfloat16)
    w_gate = (0.02 * torch.randn(w.D, generator=g, device=device)).to(torch.bfloat16)
    w_lin = (0.02 * torch.randn(H, d, d, generator=g, device=device)).to(torch.bfloat16)
    return {"q": q, "k": k, "v": v, "x": x, "w_gate": w_gate, "w_lin": w_lin,
            "bias": float(w.bias)}


def generate_projections(w: Workload, d_out: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Full-width projection weights of one layer as CPU tensors.

    w_lin_full: bf16 [H*d, H*d]; w_out: bf16 [H*d, d_out] (d_out defaults to
    H*d, the model width of the video DiTs the workloads follow).
    """
    K = w.H * w.d
    d_out = K if d_out is None else int(d_out)
    rp = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seeds[0], 0x5A1AD])))
    w_full = _bf16(rp.normal(0.0, 0.02, size=(K, K)).astype(np.float32))
    w_out = _bf16(rp.normal(0.0, 0.02, size=(K, d_out)).astype(np.float32))
    return {"w_lin_full": w_full, "w_out": w_out}
