"""ctypes wrapper of the CPU oracle (``oracle/moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``.  The CUDA library and its
Python binding never import or call anything here.

The oracle is a plain fp64 restatement of the MoE layer forward (router with
top-K and a softmax over the kept logits, stable permutation, expert FFNs,
gate-weighted combine or pure unpermute).  See the C file's header for the
page passages each function follows.  Arrays are numpy; torch CPU tensors are
accepted and viewed without copies.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

F32, BF16, E4M3 = 0, 1, 2
ACT = {"none": 0, "relu": 1, "swiglu": 2}
DTYPE = {"f32": F32, "bf16": BF16, "e4m3": E4M3}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC",
                               "-shared", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    """The oracle library; ORACLE_LIB may name another build of moe_oracle.c
    (the mutation tests point it at deliberately broken copies)."""
    global _lib
    if _lib is None:
        path = os.environ.get("ORACLE_LIB")
        if not path:
            build()
            path = _LIB
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i, i64, d = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.orc_router.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P]
        L.orc_topk_from_logits.argtypes = [i, i, i, P, P, P, P]
        L.orc_permute.argtypes = [i, i, i, P, P, i64, P, P, P, P, P]
        L.orc_expert_rows.argtypes = [i, P, i, i, i, P, i, i, i, P, P, P, d, d, P]
        L.orc_combine.argtypes = [i, i, i, P, P, P, P]
        L.orc_expert_rows_scaled.argtypes = [i, P, i, i, i, P, i, i, P, d, P, d, P, P]
        L.orc_forward_tokens.argtypes = [i, P, i, i, i, i, i, P, P, P, P, i, i, i, P, P, P, d, d,
                                         i, P, P, P, P]
        L.orc_dense_masked.argtypes = [i, i, i, i, P, P, i, i, i, P, P, P, d, d, P]
        L.orc_matmul.argtypes = [i, i, i, P, P, P]
        L.orc_quantize_rows_dynamic.argtypes = [i, i, P, P, P]
        L.orc_expert_rows_mx.argtypes = [i, P, i, i, P, P, i, P, P, P]
        L.orc_expert_rows_kscaled.argtypes = [i, P, i, i, i, P, P, d, i, i, P, P, P]
        L.orc_e8m0_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_to_f64.restype = d
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f64.restype = d
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_f64.restype = d
        L.orc_f64_to_e4m3.argtypes = [d]
        L.orc_f64_to_e4m3.restype = ctypes.c_uint8
        L.orc_f64_to_bf16.argtypes = [d]
        L.orc_f64_to_bf16.restype = ctypes.c_uint16
        L.orc_to_f64.argtypes = [P, i, i64, i64, P]
        L.orc_num_threads.restype = i
        _lib = L
    return _lib


def _np(a):
    """numpy view of a numpy array or torch CPU tensor (bf16 -> uint16 view)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a)
    import torch
    t = a.detach().contiguous()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.uint16) if hasattr(torch, "uint16") else t.view(torch.int16)
    return t.numpy()


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed (code {rc})")


def num_threads() -> int:
    return lib().orc_num_threads()


def to_f64(a, dtype: int) -> np.ndarray:
    """Decode an array stored in `dtype` (f32 / bf16 bits / e4m3 codes) to float64."""
    a = _np(a)
    out = np.empty(a.shape, np.float64)
    lib().orc_to_f64(_p(a), dtype, 0, a.size, _p(out))
    return out


def bf16_to_f64(b: int) -> float:
    return lib().orc_bf16_to_f64(b)


def e4m3_to_f64(c: int) -> float:
    return lib().orc_e4m3_to_f64(c)


def f64_to_e4m3(v: float) -> int:
    return lib().orc_f64_to_e4m3(v)


def f64_to_bf16(v: float) -> int:
    return lib().orc_f64_to_bf16(v)


def router(x, x_dtype: int, w_r, bias, K: int, want_logits: bool = False):
    """(ids int32 (N,K), gates f64 (N,K), margin f64 (N,), logits or None)."""
    x, w_r, bias = _np(x), _np(w_r).astype(np.float32, copy=False), _np(bias)
    N, d = x.shape
    E = w_r.shape[1]
    ids = np.empty((N, K), np.int32)
    gates = np.empty((N, K), np.float64)
    margin = np.empty(N, np.float64)
    logits = np.empty((N, E), np.float64) if want_logits else None
    _check(lib().orc_router(N, d, E, K, x_dtype, _p(x), _p(w_r), _p(bias), _p(ids), _p(gates),
                            _p(margin), _p(logits)), "router")
    return ids, gates, margin, logits


def topk_from_logits(logits, K: int):
    logits = np.ascontiguousarray(logits, np.float64)
    N, E = logits.shape
    ids = np.empty((N, K), np.int32)
    gates = np.empty((N, K), np.float64)
    margin = np.empty(N, np.float64)
    _check(lib().orc_topk_from_logits(N, E, K, _p(logits), _p(ids), _p(gates), _p(margin)), "topk")
    return ids, gates, margin


def permute(ids, E: int, x=None):
    """(counts (E,), offsets (E+1,), pos (N*K,), src (N*K,), x_perm or None)."""
    ids = _np(ids).astype(np.int32, copy=False)
    N, K = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    pos = np.empty(N * K, np.int32)
    src = np.empty(N * K, np.int32)
    xp, row_bytes, xperm = None, 0, None
    if x is not None:
        xp = _np(x)
        row_bytes = xp.strides[0] if xp.ndim > 1 else xp.itemsize
        xperm = np.empty((N * K,) + xp.shape[1:], xp.dtype)
    _check(lib().orc_permute(N, K, E, _p(ids), _p(xp), row_bytes, _p(counts), _p(offsets), _p(pos),
                             _p(src), _p(xperm)), "permute")
    return counts, offsets, pos, src, xperm


def expert_rows(row_expert, xrows, x_dtype: int, act: str, w1, w3, w2, w_dtype: int,
                x_scale: float = 1.0, w_scale: float = 1.0):
    """Each input row r through expert row_expert[r]; rows with expert < 0 are left NaN."""
    row_expert = np.ascontiguousarray(row_expert, np.int32)
    xr = _np(xrows)
    w1n, w3n, w2n = _np(w1), _np(w3), _np(w2)
    E, F, din = w1n.shape
    dout = F if ACT[act] == 0 else din
    y = np.full((len(row_expert), dout), np.nan)
    _check(lib().orc_expert_rows(len(row_expert), _p(row_expert), E, din, x_dtype, _p(xr), ACT[act],
                                 F, w_dtype, _p(w1n), _p(w3n), _p(w2n), x_scale, w_scale, _p(y)),
           "expert_rows")
    return y


def expert_rows_scaled(row_expert, xrows, x_dtype: int, w1, w_dtype: int, x_scale: float = 1.0,
                       x_row_scales=None, w_scale: float = 1.0, w_channel_scales=None):
    """Single-matrix experts with per-row x scales and per-(expert, output
    channel) weight scales (NULL -> the per-tensor scalar)."""
    row_expert = np.ascontiguousarray(row_expert, np.int32)
    xr = _np(xrows)
    w1n = _np(w1)
    E, F, din = w1n.shape
    xs = None if x_row_scales is None else np.ascontiguousarray(x_row_scales, np.float64)
    ws = None if w_channel_scales is None else np.ascontiguousarray(w_channel_scales, np.float64)
    y = np.full((len(row_expert), F), np.nan)
    _check(lib().orc_expert_rows_scaled(len(row_expert), _p(row_expert), E, din, x_dtype, _p(xr), F,
                                        w_dtype, _p(w1n), x_scale, _p(xs), w_scale, _p(ws), _p(y)),
           "expert_rows_scaled")
    return y


def combine(pos, gates, y_perm, N: int, K: int):
    pos = np.ascontiguousarray(pos, np.int32)
    y_perm = np.ascontiguousarray(y_perm, np.float64)
    dout = y_perm.shape[1]
    g = None if gates is None else np.ascontiguousarray(gates, np.float64)
    y = np.empty((N if g is not None else N * K, dout), np.float64)
    _check(lib().orc_combine(N, K, dout, _p(pos), _p(g), _p(y_perm), _p(y)), "combine")
    return y


def forward_tokens(inp, tokens, gates_mode: int = 1):
    """Whole layer for the listed tokens (route, K experts, combine), straight
    from the inputs: returns (y, ids, gates, margin)."""
    cfg = inp.cfg
    tok = np.ascontiguousarray(tokens, np.int32)
    x = _np(inp.x)
    w_r = None if inp.w_r is None else _np(inp.w_r)
    bias = None if inp.bias is None else _np(inp.bias)
    given = None if inp.ids is None else _np(inp.ids).astype(np.int32, copy=False)
    w1, w3, w2 = _np(inp.w1), _np(inp.w3), _np(inp.w2)
    dt = DTYPE[cfg.dtype]
    dout = cfg.F if cfg.act == "none" else cfg.d
    rows = len(tok) if gates_mode else len(tok) * cfg.K
    y = np.empty((rows, dout), np.float64)
    ids = np.empty((len(tok), cfg.K), np.int32)
    gates = np.empty((len(tok), cfg.K), np.float64)
    margin = np.empty(len(tok), np.float64)
    _check(lib().orc_forward_tokens(len(tok), _p(tok), cfg.N, cfg.d, cfg.E, cfg.K, dt, _p(x), _p(w_r),
                                    _p(bias), _p(given), ACT[cfg.act], cfg.F, dt, _p(w1), _p(w3),
                                    _p(w2), inp.x_scale, inp.w_scale, gates_mode, _p(y), _p(ids),
                                    _p(gates), _p(margin)), "forward_tokens")
    return y, ids, gates, margin


def dense_masked(x, x_dtype: int, G, act: str, w1, w3, w2, w_dtype: int, x_scale=1.0, w_scale=1.0):
    xn = _np(x)
    G = np.ascontiguousarray(G, np.float64)
    w1n, w3n, w2n = _np(w1), _np(w3), _np(w2)
    E, F, din = w1n.shape
    N = xn.shape[0]
    dout = F if ACT[act] == 0 else din
    y = np.empty((N, dout), np.float64)
    _check(lib().orc_dense_masked(N, din, E, x_dtype, _p(xn), _p(G), ACT[act], F, w_dtype, _p(w1n),
                                  _p(w3n), _p(w2n), x_scale, w_scale, _p(y)), "dense_masked")
    return y


def quantize_rows_dynamic(x):
    """Per-token dynamic e4m3 quantization of bf16 rows: (codes uint8 (n, d),
    scales float32 (n,)), decisions in fp32 as the layer takes them."""
    xn = _np(x)
    n, d = xn.shape
    codes = np.empty((n, d), np.uint8)
    scales = np.empty(n, np.float32)
    _check(lib().orc_quantize_rows_dynamic(n, d, _p(xn), _p(codes), _p(scales)),
           "quantize_rows_dynamic")
    return codes, scales


def e8m0_to_f64(s: int) -> float:
    return lib().orc_e8m0_to_f64(s)


def expert_rows_mx(row_expert, x, xs, w, ws):
    """Single-matrix experts with MX block scales: x (n, din) e4m3 codes, xs
    (n, din/32) E8M0, w (E, F, din) e4m3, ws (E, F, din/32) E8M0 -> y (n, F)
    in double; rows with expert < 0 are left NaN."""
    row_expert = np.ascontiguousarray(row_expert, np.int32)
    xn, xsn = _np(x), _np(xs)
    wn, wsn = _np(w), _np(ws)
    E, F, din = wn.shape
    y = np.full((len(row_expert), F), np.nan)
    _check(lib().orc_expert_rows_mx(len(row_expert), _p(row_expert), E, din, _p(xn), _p(xsn), F,
                                    _p(wn), _p(wsn), _p(y)), "expert_rows_mx")
    return y


def expert_rows_kscaled(row_expert, xrows, x_dtype: int, w1, w_dtype: int, w_group_scales,
                        x_group_scales=None, x_scale: float = 1.0):
    """Single-matrix experts with fp32 scales per 128-element group of K:
    w_group_scales (E, F, din/128), x_group_scales (n, din/128) or the scalar
    x_scale; rows with expert < 0 are left NaN."""
    row_expert = np.ascontiguousarray(row_expert, np.int32)
    xr, w1n = _np(xrows), _np(w1)
    E, F, din = w1n.shape
    ws = np.ascontiguousarray(w_group_scales, np.float64)
    xs = None if x_group_scales is None else np.ascontiguousarray(x_group_scales, np.float64)
    y = np.full((len(row_expert), F), np.nan)
    _check(lib().orc_expert_rows_kscaled(len(row_expert), _p(row_expert), E, din, x_dtype, _p(xr),
                                         _p(xs), x_scale, F, w_dtype, _p(w1n), _p(ws), _p(y)),
           "expert_rows_kscaled")
    return y


def block_to_group_scales(w_block_scales, F: int):
    """128 x 128 weight-block scales (E, ceil(F/128), G) -> per-channel group
    scales (E, F, G): channel n takes block n // 128."""
    wb = np.asarray(w_block_scales, np.float64)
    return np.ascontiguousarray(np.repeat(wb, 128, axis=1)[:, :F])


def matmul(A, B):
    A = np.ascontiguousarray(A, np.float64)
    B = np.ascontiguousarray(B, np.float64)
    C = np.empty((A.shape[0], B.shape[1]), np.float64)
    lib().orc_matmul(A.shape[0], A.shape[1], B.shape[1], _p(A), _p(B), _p(C))
    return C
