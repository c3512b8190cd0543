"""Python binding of libsalad (include/salad.h): argument marshalling only.

Every step of the SALAD hybrid-attention forward pass runs in the CUDA
kernels of libsalad.so.  PyTorch supplies device memory (tensors, the
workspace) and the current CUDA stream.  There is no fallback: if the library
cannot be loaded, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "SaladError", "lib", "status_string", "version",
    "gate", "gate_noalloc", "select_blocks", "linear_state", "linear_apply", "permute_tokens",
    "project",
    "sparse_attn", "dense_attn", "forward", "ForwardPlan", "forward_workspace_bytes",
    "check_error", "debug_wait_timeout",
    "MODE_TOPK", "MODE_SWA", "MODE_DENSE", "EXPORTED_SYMBOLS",
]

MODE_TOPK, MODE_SWA, MODE_DENSE = 0, 1, 2
_MODES = {"topk": MODE_TOPK, "swa": MODE_SWA, "dense": MODE_DENSE}

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsalad.so")

# Every function include/salad.h declares.
EXPORTED_SYMBOLS = (
    "salad_status_string", "salad_version",
    "salad_gate_workspace_bytes", "salad_gate",
    "salad_select_workspace_bytes", "salad_select_blocks",
    "salad_linear_state_workspace_bytes", "salad_linear_state", "salad_linear_apply",
    "salad_permute_tokens",
    "salad_sparse_attn_workspace_bytes", "salad_sparse_attn", "salad_dense_attn",
    "salad_forward_workspace_bytes", "salad_forward",
    "salad_check_error", "salad_debug_wait_timeout",
    "salad_gate_noalloc", "salad_project",
)


class SaladError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})" if what else status_string(code))


class ForwardArgs(ctypes.Structure):
    """Mirror of salad_forward_args."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("x", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("gate_bias", ctypes.c_float),
        ("w_lin", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("D", ctypes.c_int),
        ("mode", ctypes.c_int), ("block", ctypes.c_int), ("topk", ctypes.c_int),
        ("window", ctypes.c_int),
        ("space_major_heads", ctypes.c_void_p),
        ("F", ctypes.c_int), ("Hh", ctypes.c_int), ("Wh", ctypes.c_int),
        ("eps", ctypes.c_float), ("gate_override", ctypes.c_float),
        ("drop_threshold", ctypes.c_float),
        ("rope3d", ctypes.c_int), ("rope_base", ctypes.c_float),
        ("w_lin_full", ctypes.c_void_p), ("w_out", ctypes.c_void_p), ("d_out", ctypes.c_int),
        ("out", ctypes.c_void_p),
        ("s_out", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("phase_events", ctypes.c_void_p),
        ("regroup_in_load", ctypes.c_int),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsalad.so not built ({LIB_PATH}); run "
                          "`python -m sparse_linear_hybrid_top_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "salad_status_string": (ctypes.c_char_p, [i]),
        "salad_version": (i, []),
        "salad_gate_workspace_bytes": (sz, [i, i, i]),
        "salad_gate": (i, [vp, vp, f, i, i, i, vp, vp, sz, vp]),
        "salad_select_workspace_bytes": (sz, [i, i, i, i, i]),
        "salad_select_blocks": (i, [vp, vp, i, i, i, i, i, i, vp, vp, sz, vp]),
        "salad_linear_state_workspace_bytes": (sz, [i, i, i, i]),
        "salad_linear_state": (i, [vp, vp, i, i, i, i, vp, vp, vp, sz, vp]),
        "salad_linear_apply": (i, [vp, vp, vp, f, i, i, i, i, vp, vp]),
        "salad_permute_tokens": (i, [vp, vp, i, i, i, i, i, i, i, vp]),
        "salad_sparse_attn_workspace_bytes": (sz, [i, i, i, i, i, i, vp]),
        "salad_sparse_attn": (i, [vp, vp, vp, i, i, i, i, i, i, i, vp, i, vp, i, i, i, vp, vp,
                                  sz, vp]),
        "salad_dense_attn": (i, [vp, vp, vp, i, i, i, i, vp, vp]),
        "salad_project": (i, [vp, i, i, i, i, vp, i, vp, i, vp, vp, f, vp]),
        "salad_forward_workspace_bytes": (sz, [ctypes.POINTER(ForwardArgs)]),
        "salad_forward": (i, [ctypes.POINTER(ForwardArgs), vp]),
        "salad_check_error": (i, [vp]),
        "salad_debug_wait_timeout": (i, [ctypes.c_ulonglong, vp]),
        "salad_gate_noalloc": (i, [vp, vp, f, i, i, i, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


class _Lib:
    """The loaded libsalad.so, opened on first use (so that the build step can
    import this package before the library exists).  Raises ImportError on
    first use if the library is missing: there is no fallback."""

    _cdll = None

    def __getattr__(self, name):
        if _Lib._cdll is None:
            _Lib._cdll = _load()
        return getattr(_Lib._cdll, name)


lib = _Lib()


def status_string(code: int) -> str:
    return lib.salad_status_string(int(code)).decode()


def version() -> int:
    return int(lib.salad_version())


def _check(code: int, what: str):
    if code != 0:
        raise SaladError(code, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _shape(t, shape, name: str):
    """Exact shape check, before any device access (a wrong size would make a
    kernel read past the tensor)."""
    if not isinstance(t, torch.Tensor) or tuple(t.shape) != tuple(shape):
        got = tuple(t.shape) if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {got}")


def _dims(t, n: int, name: str, layout: str):
    if not isinstance(t, torch.Tensor) or t.dim() != n:
        raise ValueError(f"{name} must be a {layout} tensor")


def _dev_tensor(t: torch.Tensor, dtype, name: str):
    """A tensor the library reads or writes: on the current CUDA device (the
    library launches there), of the documented dtype, contiguous.  Checked
    for inputs and caller-supplied outputs alike, before any launch: a host
    tensor would hand the kernel a host pointer, a tensor of another device
    would be used on the wrong GPU, and a wrong dtype would be misread."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return workspace
    if workspace is not None:
        _dev_tensor(workspace, None, "workspace")
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _flags(space_major_heads, H: int):
    if space_major_heads is None:
        return None, None
    arr = (ctypes.c_uint8 * H)()
    for h in range(H):
        arr[h] = 0
    for h in space_major_heads:
        arr[int(h)] = 1
    return arr, ctypes.cast(arr, ctypes.c_void_p)


# ------------------------------------------------------------ entry points --
def gate(x: torch.Tensor, w: torch.Tensor, bias: float = 0.0, *, s=None, workspace=None,
         stream=None) -> torch.Tensor:
    """s[b] = sigmoid(w . mean_n x[b, n, :] + bias); x bf16 [B,N,D], w bf16 [D]."""
    _dims(x, 3, "x", "[B, N, D]")
    B, N, D = x.shape
    _shape(w, (D,), "w")
    if s is not None:
        _shape(s, (B,), "s")
    _dev_tensor(x, torch.bfloat16, "x"); _dev_tensor(w, torch.bfloat16, "w")
    if s is not None:
        _dev_tensor(s, torch.float32, "s")
    s = torch.empty(B, dtype=torch.float32, device=x.device) if s is None else s
    ws = _workspace(lib.salad_gate_workspace_bytes(B, N, D), x.device, workspace)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.salad_gate(_ptr(x), _ptr(w), float(bias), B, N, D, _ptr(s), _ptr(ws), nbytes,
                          _stream(stream)), "salad_gate")
    return s


def gate_noalloc(x: torch.Tensor, w: torch.Tensor, bias: float = 0.0, *, s=None,
                 stream=None) -> torch.Tensor:
    """The gate for callers that cannot allocate scratch: same result as
    gate(), partial sums kept in the library's own fixed device array
    (B <= 256; calls that overlap on the GPU race on that array)."""
    _dims(x, 3, "x", "[B, N, D]")
    B, N, D = x.shape
    _shape(w, (D,), "w")
    if s is not None:
        _shape(s, (B,), "s")
    _dev_tensor(x, torch.bfloat16, "x"); _dev_tensor(w, torch.bfloat16, "w")
    if s is not None:
        _dev_tensor(s, torch.float32, "s")
    s = torch.empty(B, dtype=torch.float32, device=x.device) if s is None else s
    _check(lib.salad_gate_noalloc(_ptr(x), _ptr(w), float(bias), B, N, D, _ptr(s),
                                  _stream(stream)), "salad_gate_noalloc")
    return s


def select_blocks(q: torch.Tensor, k: torch.Tensor, topk: int, *, block: int = 64, idx=None,
                  workspace=None, stream=None) -> torch.Tensor:
    """Top-K key blocks per query block: int32 [B, H, nb, topk], ascending."""
    _dims(q, 4, "q", "[B, H, N, d]")
    B, H, N, d = q.shape
    nb = (N + block - 1) // block
    _shape(k, q.shape, "k")
    if idx is not None:
        _shape(idx, (B, H, nb, int(topk)), "idx")
    _dev_tensor(q, torch.bfloat16, "q"); _dev_tensor(k, torch.bfloat16, "k")
    if idx is not None:
        _dev_tensor(idx, torch.int32, "idx")
    idx = torch.empty(B, H, nb, topk, dtype=torch.int32, device=q.device) if idx is None else idx
    ws = _workspace(lib.salad_select_workspace_bytes(B, H, N, d, block), q.device, workspace)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.salad_select_blocks(_ptr(q), _ptr(k), B, H, N, d, block, topk, _ptr(idx),
                                   _ptr(ws), nbytes, _stream(stream)), "salad_select_blocks")
    return idx


def linear_state(k: torch.Tensor, v: torch.Tensor, *, workspace=None, stream=None):
    """(H, Z): float32 [B,H,d,d] = relu(K)^T V and [B,H,d] = relu(K)^T 1."""
    _dims(k, 4, "k", "[B, H, N, d]")
    _shape(v, k.shape, "v")
    _dev_tensor(k, torch.bfloat16, "k"); _dev_tensor(v, torch.bfloat16, "v")
    B, H, N, d = k.shape
    Hst = torch.empty(B, H, d, d, dtype=torch.float32, device=k.device)
    Z = torch.empty(B, H, d, dtype=torch.float32, device=k.device)
    ws = _workspace(lib.salad_linear_state_workspace_bytes(B, H, N, d), k.device, workspace)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.salad_linear_state(_ptr(k), _ptr(v), B, H, N, d, _ptr(Hst), _ptr(Z), _ptr(ws),
                                  nbytes, _stream(stream)), "salad_linear_state")
    return Hst, Z


def linear_apply(q: torch.Tensor, Hst: torch.Tensor, Z: torch.Tensor, eps: float = 1e-6, *,
                 o=None, stream=None) -> torch.Tensor:
    """relu(q) H / (relu(q) . Z + eps) as bf16 [B,H,N,d]."""
    _dims(q, 4, "q", "[B, H, N, d]")
    B, H, N, d = q.shape
    _shape(Hst, (B, H, d, d), "Hst")
    _shape(Z, (B, H, d), "Z")
    if o is not None:
        _shape(o, q.shape, "o")
    _dev_tensor(q, torch.bfloat16, "q")
    _dev_tensor(Hst, torch.float32, "Hst"); _dev_tensor(Z, torch.float32, "Z")
    if o is not None:
        _dev_tensor(o, torch.bfloat16, "o")
    o = torch.empty_like(q) if o is None else o
    _check(lib.salad_linear_apply(_ptr(q), _ptr(Hst), _ptr(Z), float(eps), B, H, N, d, _ptr(o),
                                  _stream(stream)), "salad_linear_apply")
    return o


def project(a: torch.Tensor, w: torch.Tensor, *, out_per_head: bool = False, resid=None,
            s=None, drop_threshold: float = 0.0, out=None, stream=None) -> torch.Tensor:
    """resid + s_b * (cat_heads(a) @ w): a bf16 [B,H,N,d], w bf16 [H*d, n_out].

    out_per_head: out is [B,H,N,d] (n_out == H*d), else [B,N,n_out].  resid
    (same layout as out, may be ``out`` itself) and s (float32 [B]) are
    optional; samples with s_b < drop_threshold are left unwritten.
    """
    if not isinstance(a, torch.Tensor) or a.dim() != 4:
        raise ValueError("a must be a [B, H, N, d] tensor")
    B, H, N, d = a.shape
    if not isinstance(w, torch.Tensor) or w.dim() != 2:
        raise ValueError("w must be a [H*d, n_out] tensor")
    n_out = w.shape[-1]
    _shape(w, (H * d, n_out), "w")
    out_shape = (B, H, N, d) if out_per_head else (B, N, n_out)
    if out is not None:
        _shape(out, out_shape, "out")
    if resid is not None:
        _shape(resid, out_shape, "resid")
    if s is not None:
        _shape(s, (B,), "s")
    _dev_tensor(a, torch.bfloat16, "a")
    _dev_tensor(w, torch.bfloat16, "w")
    if out is None:
        out = torch.empty((B, H, N, d) if out_per_head else (B, N, n_out), dtype=torch.bfloat16,
                          device=a.device)
    _dev_tensor(out, torch.bfloat16, "out")
    if resid is not None:
        _dev_tensor(resid, torch.bfloat16, "resid")
    if s is not None:
        _dev_tensor(s, torch.float32, "s")
    _check(lib.salad_project(_ptr(a), B, H, N, d, _ptr(w), n_out, _ptr(out), int(bool(out_per_head)),
                             _ptr(resid), _ptr(s), float(drop_threshold), _stream(stream)),
           "salad_project")
    return out


def permute_tokens(src: torch.Tensor, F: int, Hh: int, Wh: int, *, inverse: bool = False,
                   dst=None, stream=None) -> torch.Tensor:
    """Frame-major <-> space-major row order of [..., N, d] slabs."""
    if not isinstance(src, torch.Tensor) or src.dim() < 2:
        raise ValueError("src must be a [..., N, d] tensor")
    if dst is not None:
        _shape(dst, src.shape, "dst")
    _dev_tensor(src, torch.bfloat16, "src")
    if dst is not None:
        _dev_tensor(dst, torch.bfloat16, "dst")
    N, d = src.shape[-2:]
    S = src.numel() // (N * d)
    dst = torch.empty_like(src) if dst is None else dst
    _check(lib.salad_permute_tokens(_ptr(src), _ptr(dst), S, N, d, F, Hh, Wh, int(bool(inverse)),
                                    _stream(stream)), "salad_permute_tokens")
    return dst


def sparse_attn(q, k, v, mode: str = "topk", *, topk: int = 0, idx=None, window: int = 0,
                space_major_heads: Optional[Sequence[int]] = None, F: int = 0, Hh: int = 0,
                Wh: int = 0, block: int = 64, o=None, workspace=None, stream=None):
    """Normalised sparse-branch attention output, bf16 [B,H,N,d]."""
    _dims(q, 4, "q", "[B, H, N, d]")
    B, H, N, d = q.shape
    _shape(k, q.shape, "k")
    _shape(v, q.shape, "v")
    if o is not None:
        _shape(o, q.shape, "o")
    if mode == "topk" and idx is not None:
        _shape(idx, (B, H, (N + block - 1) // block, int(topk)), "idx")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, torch.bfloat16, n)
    if o is not None:
        _dev_tensor(o, torch.bfloat16, "o")
    if mode == "topk" and idx is not None:
        _dev_tensor(idx, torch.int32, "idx")
    m = _MODES[mode]
    flags, fptr = _flags(space_major_heads, H)
    o = torch.empty_like(q) if o is None else o
    need = lib.salad_sparse_attn_workspace_bytes(B, H, N, d, m, int(topk), fptr)
    ws = _workspace(need, q.device, workspace)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.salad_sparse_attn(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, m, block, int(topk),
                                 _ptr(idx), int(window), fptr, F, Hh, Wh, _ptr(o), _ptr(ws),
                                 nbytes, _stream(stream)), "salad_sparse_attn")
    return o


def dense_attn(q, k, v, *, o=None, stream=None):
    """Dense flash attention softmax(Q K^T / sqrt(d)) V, bf16 [B,H,N,d]."""
    _dims(q, 4, "q", "[B, H, N, d]")
    _shape(k, q.shape, "k")
    _shape(v, q.shape, "v")
    if o is not None:
        _shape(o, q.shape, "o")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, torch.bfloat16, n)
    if o is not None:
        _dev_tensor(o, torch.bfloat16, "o")
    B, H, N, d = q.shape
    o = torch.empty_like(q) if o is None else o
    _check(lib.salad_dense_attn(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(o), _stream(stream)),
           "salad_dense_attn")
    return o


class ForwardPlan:
    """Arguments and workspace of repeated salad_forward calls on fixed buffers.

    The plan owns its workspace (a torch uint8 tensor) and the packed argument
    struct; ``run()`` enqueues the whole layer on the given stream.  The
    keyword arguments mirror ``salad_forward_args`` (include/salad.h), e.g.
    ``regroup_in_load=True`` regroups the ST-SWA heads inside the attention's
    loads instead of copying them (no copy workspace; slower on a B200).
    """

    def __init__(self, q, k, v, x, w_gate, w_lin, *, mode: str = "topk", topk: int = 0,
                 window: int = 0, space_major_heads: Optional[Sequence[int]] = None,
                 F: int = 0, Hh: int = 0, Wh: int = 0, bias: float = 0.0, eps: float = 1e-6,
                 gate_override: Optional[float] = None, drop_threshold: float = 0.0,
                 rope3d: bool = False, rope_base: float = 10000.0, o=None,
                 s_out=None, idx_out=None, block: int = 64, w_lin_full=None, w_out=None,
                 out=None, regroup_in_load: bool = False):
        # Shapes first (a wrong size would make a kernel read past a tensor).
        if not isinstance(q, torch.Tensor) or q.dim() != 4:
            raise ValueError("q must be a [B, H, N, d] tensor")
        B, H, N, d = q.shape
        _shape(k, q.shape, "k")
        _shape(v, q.shape, "v")
        if not isinstance(x, torch.Tensor) or x.dim() != 3:
            raise ValueError("x must be a [B, N, D] tensor")
        _shape(x, (B, N, x.shape[-1]), "x")
        _shape(w_gate, (x.shape[-1],), "w_gate")
        if w_lin is not None:
            _shape(w_lin, (H, d, d), "w_lin")
        if w_lin_full is not None:
            _shape(w_lin_full, (H * d, H * d), "w_lin_full")
        if w_out is not None:
            if w_out.dim() != 2:
                raise ValueError("w_out must be a [H*d, d_out] tensor")
            _shape(w_out, (H * d, w_out.shape[-1]), "w_out")
            if out is not None:
                _shape(out, (B, N, w_out.shape[-1]), "out")
        if o is not None:
            _shape(o, q.shape, "o")
        if s_out is not None:
            _shape(s_out, (B,), "s_out")
        if idx_out is not None and mode == "topk":
            _shape(idx_out, (B, H, (N + block - 1) // block, int(topk)), "idx_out")
        for n, t in (("q", q), ("k", k), ("v", v), ("x", x), ("w_gate", w_gate),
                     ("w_lin", w_lin), ("w_lin_full", w_lin_full), ("w_out", w_out)):
            if t is not None or n in ("q", "k", "v", "x", "w_gate"):
                _dev_tensor(t, torch.bfloat16, n)
        for n, t, dt in (("o", o, torch.bfloat16), ("out", out, torch.bfloat16),
                         ("s_out", s_out, torch.float32), ("idx_out", idx_out, torch.int32)):
            if t is not None:
                _dev_tensor(t, dt, n)
        self.tensors = dict(q=q, k=k, v=v, x=x, w_gate=w_gate, w_lin=w_lin,
                            w_lin_full=w_lin_full, w_out=w_out)
        # Output projection (optional): out [B,N,d_out] = cat_heads(O) w_out.
        self.out = None
        if w_out is not None:
            self.out = torch.empty((B, N, w_out.shape[-1]), dtype=torch.bfloat16,
                                   device=q.device) if out is None else out
        self.o = torch.empty_like(q) if o is None else o
        self.s_out, self.idx_out = s_out, idx_out
        self._flags, fptr = _flags(space_major_heads, H)
        a = ForwardArgs()
        a.q, a.k, a.v, a.x, a.w_gate, a.w_lin = (_ptr(t) for t in (q, k, v, x, w_gate, w_lin))
        a.gate_bias = float(bias)
        a.o = _ptr(self.o)
        a.B, a.H, a.N, a.d, a.D = B, H, N, d, x.shape[-1]
        a.mode, a.block, a.topk, a.window = _MODES[mode], block, int(topk), int(window)
        a.space_major_heads = fptr
        a.F, a.Hh, a.Wh = F, Hh, Wh
        a.regroup_in_load = 1 if regroup_in_load else 0
        a.eps = float(eps)
        a.gate_override = float("nan") if gate_override is None else float(gate_override)
        # Post-training branch dropping: sample b's linear branch is skipped
        # (on the device) when s_b < drop_threshold; 0 never drops.
        a.drop_threshold = float(drop_threshold)
        # 3-D rotary encoding of the linear branch over the F x Hh x Wh grid.
        a.rope3d = 1 if rope3d else 0
        a.rope_base = float(rope_base)
        # Full-width projection of the linear branch instead of the per-head w_lin.
        a.w_lin_full = _ptr(w_lin_full)
        a.w_out = _ptr(w_out)
        a.d_out = 0 if w_out is None else int(w_out.shape[-1])
        a.out = _ptr(self.out)
        a.s_out = _ptr(s_out)
        a.idx_out = _ptr(idx_out)
        need = lib.salad_forward_workspace_bytes(ctypes.byref(a))
        if need == 0:
            raise SaladError(-1, "salad_forward_workspace_bytes")
        self.workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        a.workspace = _ptr(self.workspace)
        a.workspace_bytes = need
        self.args = a

    def set_phase_events(self, events: Optional[Sequence[torch.cuda.Event]]) -> None:
        """Record these 5 events inside each run (start, gate, pattern, linear, attention)."""
        if events is None:
            self._events, self.args.phase_events = None, None
            return
        if len(events) != 5:
            raise ValueError("need 5 events")
        for ev in events:
            ev.record()   # creates the underlying cudaEvent_t
        self._events = (ctypes.c_void_p * 5)(*[ev.cuda_event for ev in events])
        self.args.phase_events = ctypes.cast(self._events, ctypes.c_void_p)

    def run(self, stream=None) -> torch.Tensor:
        _check(lib.salad_forward(ctypes.byref(self.args), _stream(stream)), "salad_forward")
        return self.o


def forward_workspace_bytes(plan: ForwardPlan) -> int:
    return int(lib.salad_forward_workspace_bytes(ctypes.byref(plan.args)))


def forward(q, k, v, x, w_gate, w_lin, **kw) -> torch.Tensor:
    """The whole hybrid layer (one call): O = O_sparse + s * (O_lin W_lin)."""
    stream = kw.pop("stream", None)
    return ForwardPlan(q, k, v, x, w_gate, w_lin, **kw).run(stream)


def check_error(stream=None) -> None:
    """Synchronises the stream and raises if a bounded device wait ran out."""
    _check(lib.salad_check_error(_stream(stream)), "salad_check_error")


def debug_wait_timeout(timeout_ns: int, stream=None) -> int:
    """Enqueues a wait that nothing satisfies; returns the launch status."""
    return int(lib.salad_debug_wait_timeout(int(timeout_ns), _stream(stream)))
