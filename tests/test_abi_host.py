"""Host-side checks of the C ABI: no GPU needed, no kernel launched.

Every argument check of include/salad.h runs before the first CUDA call, so
invalid calls return their status here even without a device.
"""
import ctypes
import os
import re

import pytest

import sparse_linear_hybrid_top_b200 as salad
from sparse_linear_hybrid_top_b200 import ForwardArgs, lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUP, CUDA, TIMEOUT, WS = 0, -1, -2, -3, -4, -5
A = 0x10000  # a 256-aligned fake device address (never dereferenced)


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "salad.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(salad_\w+)\s*\(", text)))


def test_header_declarations_match_binding_and_exports():
    declared = _declared_functions()
    assert declared == sorted(salad.EXPORTED_SYMBOLS)
    so = ctypes.CDLL(salad.LIB_PATH)
    for name in declared:
        assert hasattr(so, name), name


def test_library_is_built_for_sm100a_only():
    # The binding loads the in-tree library (no fallback path exists).
    assert os.path.dirname(salad.LIB_PATH) == os.path.join(ROOT, "sparse_linear_hybrid_top_b200")
    assert salad.version() == 40200


def test_status_strings():
    for code in (OK, INVALID, UNSUP, CUDA, TIMEOUT, WS):
        assert isinstance(salad.status_string(code), str) and salad.status_string(code)
    assert salad.status_string(12345) == "unknown status"


def test_gate_argument_checks():
    ws = lib.salad_gate_workspace_bytes(1, 100, 64)
    assert ws > 0
    assert lib.salad_gate(None, A, 0.0, 1, 100, 64, A, A, ws, None) == INVALID
    assert lib.salad_gate(A + 8, A, 0.0, 1, 100, 64, A, A, ws, None) == INVALID   # misaligned
    assert lib.salad_gate(A, A, 0.0, 1, 100, 60, A, A, ws, None) == INVALID       # D % 8
    assert lib.salad_gate(A, A, 0.0, 1, 100, 64, A, None, ws, None) == WS
    assert lib.salad_gate(A, A, 0.0, 1, 100, 64, A, A, ws - 1, None) == WS
    assert lib.salad_gate(A, A, 0.0, 1, 100, 64, A, A + 16, ws, None) == WS       # ws alignment


def test_select_argument_checks():
    ws = lib.salad_select_workspace_bytes(1, 2, 1000, 128, 64)
    assert ws > 0
    assert lib.salad_select_workspace_bytes(1, 2, 1000, 96, 64) == 0
    assert lib.salad_select_blocks(A, A, 1, 2, 1000, 96, 64, 2, A, A, ws, None) == UNSUP
    assert lib.salad_select_blocks(A, A, 1, 2, 1000, 128, 32, 2, A, A, ws, None) == UNSUP
    assert lib.salad_select_blocks(A, A, 1, 2, 1000, 128, 64, 0, A, A, ws, None) == INVALID
    assert lib.salad_select_blocks(A, A, 1, 2, 1000, 128, 64, 17, A, A, ws, None) == INVALID  # > nb
    assert lib.salad_select_blocks(A, A, 1, 2, 0, 128, 64, 1, A, A, ws, None) == INVALID
    assert lib.salad_select_blocks(A, A, 1, 2, 262145, 128, 64, 1, A, A, ws, None) == INVALID
    assert lib.salad_select_blocks(A, A, 1, 2, 1000, 128, 64, 2, A, A, ws // 2, None) == WS


def test_attention_argument_checks():
    assert lib.salad_dense_attn(A, A, A, 1, 2, 100, 80, A, None) == UNSUP
    assert lib.salad_dense_attn(A, None, A, 1, 2, 100, 64, A, None) == INVALID
    assert lib.salad_dense_attn(A, A, A, 1, 257, 100, 64, A, None) == INVALID     # H > 256
    assert lib.salad_sparse_attn(A, A, A, 1, 2, 100, 64, 7, 64, 1, A, 0, None, 0, 0, 0, A, None,
                                 0, None) == INVALID                             # bad mode
    assert lib.salad_sparse_attn(A, A, A, 1, 2, 100, 64, 0, 64, 1, None, 0, None, 0, 0, 0, A,
                                 None, 0, None) == INVALID                       # no idx
    flags = (ctypes.c_uint8 * 2)(1, 0)
    fp = ctypes.cast(flags, ctypes.c_void_p)
    need = lib.salad_sparse_attn_workspace_bytes(1, 2, 120, 64, 1, 0, fp)
    assert need == 3 * ((120 * 64 * 2 + 255) // 256 * 256)
    # window < 0; grid that does not multiply to N.
    assert lib.salad_sparse_attn(A, A, A, 1, 2, 120, 64, 1, 64, 0, None, -1, fp, 2, 6, 10, A, A,
                                 need, None) == INVALID
    assert lib.salad_sparse_attn(A, A, A, 1, 2, 120, 64, 1, 64, 0, None, 5, fp, 2, 6, 11, A, A,
                                 need, None) == INVALID
    assert lib.salad_sparse_attn(A, A, A, 1, 2, 120, 64, 1, 64, 0, None, 5, fp, 2, 6, 10, A, A,
                                 need - 256, None) == WS


def test_permute_argument_checks():
    assert lib.salad_permute_tokens(A, A + 64, 2, 12, 64, 2, 2, 3, 0, None) == INVALID  # overlap
    assert lib.salad_permute_tokens(A, A + (1 << 20), 2, 12, 64, 2, 2, 4, 0, None) == INVALID
    assert lib.salad_permute_tokens(A, A + (1 << 20), 2, 12, 64, 2, 2, 3, 2, None) == INVALID
    # more slabs than one grid dimension holds
    assert lib.salad_permute_tokens(A, A + (1 << 36), 65536, 12, 64, 2, 2, 3, 0, None) == INVALID


def test_project_argument_checks():
    # a [1,2,100,64] -> n_out 128 (per head) or 192 (token-major).
    P = lib.salad_project
    big = A + (1 << 24)
    assert P(A, 1, 2, 100, 64, big, 100, big * 2, 0, None, None, 0.0, None) == INVALID  # n_out % 64
    assert P(A, 1, 2, 100, 64, big, 0, big * 2, 0, None, None, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 64, big, 192, big * 2, 1, None, None, 0.0, None) == INVALID  # != H*d
    assert P(A, 1, 2, 100, 64, big, 128, big * 2, 2, None, None, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 96, big, 192, big * 2, 0, None, None, 0.0, None) == UNSUP    # d
    assert P(A + 8, 1, 2, 100, 64, big, 128, big * 2, 0, None, None, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 64, None, 128, big * 2, 0, None, None, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 64, big, 128, A + 64, 0, None, None, 0.0, None) == INVALID   # out over a
    assert P(A, 1, 2, 100, 64, big, 128, big + 64, 0, None, None, 0.0, None) == INVALID  # over w
    assert P(A, 1, 2, 100, 64, big, 128, big * 2, 0, big * 2 + 64, None, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 64, big, 128, big * 2, 0, None, big * 3 + 2, 0.0, None) == INVALID
    assert P(A, 1, 2, 100, 64, big, 128, big * 2, 0, None, None, float("inf"), None) == INVALID


def _fwd_args(**kw):
    a = ForwardArgs()
    a.q = a.k = a.v = a.x = a.w_gate = a.w_lin = a.o = A
    a.B, a.H, a.N, a.d, a.D = 1, 2, 1000, 64, 128
    a.mode, a.block, a.topk, a.window = 0, 64, 2, 0
    a.eps = 1e-6
    a.gate_override = float("nan")
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_forward_argument_checks_and_workspace_query():
    a = _fwd_args()
    need = lib.salad_forward_workspace_bytes(ctypes.byref(a))
    assert need > 0 and need % 256 == 0
    a.workspace, a.workspace_bytes = A, need - 1
    assert lib.salad_forward(ctypes.byref(a), None) == WS
    a.workspace_bytes = need
    bad = _fwd_args(topk=100, workspace=A, workspace_bytes=need)
    assert lib.salad_forward(ctypes.byref(bad), None) == INVALID
    bad = _fwd_args(d=32, workspace=A, workspace_bytes=need)
    assert lib.salad_forward(ctypes.byref(bad), None) == UNSUP
    bad = _fwd_args(eps=-1.0, workspace=A, workspace_bytes=need)
    assert lib.salad_forward(ctypes.byref(bad), None) == INVALID
    bad = _fwd_args(gate_override=float("inf"), workspace=A, workspace_bytes=need)
    assert lib.salad_forward(ctypes.byref(bad), None) == INVALID
    assert lib.salad_forward(None, None) == INVALID
    # Full-width projections: d_out a multiple of 64, out given and apart
    # from o.
    big = A + (1 << 24)
    for kw in (dict(w_out=big, d_out=100, out=big * 2), dict(w_out=big, d_out=128, out=None),
               dict(w_out=big, d_out=128, out=A + 64), dict(w_out=big + 8, d_out=128, out=big * 2),
               dict(w_lin_full=big + 8)):
        bad = _fwd_args(workspace=A, workspace_bytes=need, **kw)
        assert lib.salad_forward(ctypes.byref(bad), None) == INVALID, kw
    # The full-width path keeps O_l (bf16 [B,H,N,d]) instead of the folded images.
    full = _fwd_args(w_lin_full=big)
    assert (lib.salad_forward_workspace_bytes(ctypes.byref(full)) -
            lib.salad_forward_workspace_bytes(ctypes.byref(_fwd_args()))) == \
        2 * 1000 * 64 * 2 - 2 * 64 * 64 * 2
    # Larger problems need more workspace; SWA with regrouped heads adds copies.
    big = _fwd_args(N=31200, d=128, H=12, D=1536, topk=49)
    assert lib.salad_forward_workspace_bytes(ctypes.byref(big)) > need
    flags = (ctypes.c_uint8 * 2)(1, 1)
    swa = _fwd_args(mode=1, topk=0, window=10, N=1000, F=10, Hh=10, Wh=10,
                    space_major_heads=ctypes.cast(flags, ctypes.c_void_p).value)
    none = _fwd_args(mode=1, topk=0, window=10, N=1000)
    assert (lib.salad_forward_workspace_bytes(ctypes.byref(swa)) -
            lib.salad_forward_workspace_bytes(ctypes.byref(none))) == 3 * 2 * 1000 * 64 * 2
    # Regrouping inside the attention's loads needs no copies; it takes 0 or 1
    # and a whole position (F <= 128 rows) per 128-row tile.
    inload = _fwd_args(mode=1, topk=0, window=10, N=1000, F=10, Hh=10, Wh=10, regroup_in_load=1,
                       space_major_heads=ctypes.cast(flags, ctypes.c_void_p).value)
    assert (lib.salad_forward_workspace_bytes(ctypes.byref(inload)) ==
            lib.salad_forward_workspace_bytes(ctypes.byref(none)))
    ws = lib.salad_forward_workspace_bytes(ctypes.byref(swa))
    for kw, want in ((dict(regroup_in_load=2, F=10, Hh=10, Wh=10), INVALID),
                     (dict(regroup_in_load=1, F=250, Hh=2, Wh=2), UNSUP)):
        bad = _fwd_args(mode=1, topk=0, window=10, N=1000, workspace=A, workspace_bytes=ws,
                        space_major_heads=ctypes.cast(flags, ctypes.c_void_p).value, **kw)
        assert lib.salad_forward(ctypes.byref(bad), None) == want, kw


def test_valid_call_without_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("only meaningful on a host without a GPU")
    a = _fwd_args()
    need = lib.salad_forward_workspace_bytes(ctypes.byref(a))
    a.workspace, a.workspace_bytes = A, need
    assert lib.salad_forward(ctypes.byref(a), None) in (CUDA, UNSUP)
