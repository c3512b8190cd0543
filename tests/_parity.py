"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""
import numpy as np
import torch

# Output bar of the hybrid layer and of every attention output (bf16 in,
# float32 accumulation): max |err| <= 2e-2 and relative L2 <= 5e-3.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def err_stats(got, want):
    g, w = to64(got), to64(want)
    assert g.shape == w.shape, (g.shape, w.shape)
    diff = g - w
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(w.ravel()))
    rel = float(np.linalg.norm(diff.ravel())) / max(den, 1e-300)
    return max_abs, rel


def assert_close(got, want, what, max_abs=MAX_ABS, rel_l2=REL_L2):
    g = to64(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    m, r = err_stats(got, want)
    assert m <= max_abs and r <= rel_l2, f"{what}: max_abs={m:.3e} (<= {max_abs}) rel_l2={r:.3e} (<= {rel_l2})"
    return m, r


def device_inputs(inp, device="cuda"):
    out = {}
    for k, v in inp.items():
        out[k] = v.to(device).contiguous() if isinstance(v, torch.Tensor) else v
    return out
