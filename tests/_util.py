"""Shared helpers of the tests: moving synthetic inputs to the GPU, building a
plan through the C ABI binding, comparing with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth

# Float tolerances against the fp64 oracle: fp32 1e-5, bf16 2e-2, fp8 6e-2.
# Each bounds both the normwise error (max|gpu - ref| / max|ref| over the
# tensor) and the worst row's error relative to that row's own max|ref|
# (floored at ROW_FLOOR of the tensor's max|ref|, so that a row of near-zero
# values is judged on absolute error): a small-valued row cannot hide behind
# large rows elsewhere.
TOL = {"f32": 1e-5, "bf16": 2e-2, "e4m3": 6e-2}
NEAR_TIE = 1e-5
ROW_FLOOR = 1e-3


def normwise_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max() if ref.size else 0.0
    if den == 0.0:
        return float(np.abs(gpu).max()) if gpu.size else 0.0
    return float(np.abs(gpu - ref).max() / den)


def row_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Worst row of |gpu - ref| / max(max|ref row|, ROW_FLOOR * max|ref|)
    (rows = the last axis; a 1-D array is one row)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if not ref.size:
        return 0.0
    g2 = gpu.reshape(-1, ref.shape[-1]) if ref.ndim > 1 else gpu.reshape(1, -1)
    r2 = ref.reshape(-1, ref.shape[-1]) if ref.ndim > 1 else ref.reshape(1, -1)
    top = np.abs(r2).max()
    if top == 0.0:
        return float(np.abs(g2).max())
    den = np.maximum(np.abs(r2).max(axis=1), ROW_FLOOR * top)
    return float((np.abs(g2 - r2).max(axis=1) / den).max())


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """The larger of the normwise and the worst-row relative error."""
    return max(normwise_err(gpu, ref), row_err(gpu, ref))


def to_gpu(inp: synth.MoEInputs) -> dict:
    dev = "cuda"
    w = {"w1": inp.w1.to(dev)}
    if inp.w3 is not None:
        w["w3"] = inp.w3.to(dev)
    if inp.w2 is not None:
        w["w2"] = inp.w2.to(dev)
    if inp.w_r is not None:
        w["w_r"] = inp.w_r.to(dev)
    if inp.bias is not None:
        w["bias"] = inp.bias.to(dev)
    w["w_scale"] = inp.w_scale
    return w


def make_plan(inp: synth.MoEInputs, weights: dict | None = None):
    import top_routing_grouped_gemv_b200 as moe
    c = inp.cfg
    weights = weights if weights is not None else to_gpu(inp)
    return moe.Plan(c.N, c.d, c.E, c.K, c.F, c.dtype, c.act, weights), weights


def f64(t: torch.Tensor) -> np.ndarray:
    """GPU/CPU tensor (fp32 / bf16) -> float64 numpy."""
    return t.detach().to("cpu").double().numpy()


def near_tie_tokens(logits: np.ndarray, K: int) -> np.ndarray:
    """Tokens whose K-th/(K+1)-th logit margin, or the gap between two of the
    K+1 largest logits, is below NEAR_TIE (the order there is decided by
    rounding, not by the method)."""
    E = logits.shape[1]
    srt = -np.sort(-logits, axis=1)[:, :min(K + 1, E)]
    if srt.shape[1] < 2:
        return np.zeros(len(logits), bool)
    gaps = srt[:, :-1] - srt[:, 1:]
    return (gaps < NEAR_TIE).any(axis=1)


def check_routing(ids_gpu: np.ndarray, gates_gpu: np.ndarray, logits: np.ndarray,
                  ids_ref: np.ndarray, gates_ref: np.ndarray):
    """Bit-exact ids on every token that is not a near tie; on near ties the
    GPU's set must still be a valid top-K of the fp64 logits (within NEAR_TIE).
    Returns (near-tie token indices, tokens whose ids differ)."""
    K = ids_ref.shape[1]
    tie = near_tie_tokens(logits, K)
    diff = np.nonzero((ids_gpu != ids_ref).any(axis=1))[0]
    bad = [t for t in diff if not tie[t]]
    assert not bad, f"routing differs on non-tie tokens {bad[:10]}"
    for t in diff:
        kth = np.sort(logits[t])[::-1][K - 1]
        assert np.all(logits[t][ids_gpu[t]] >= kth - NEAR_TIE), t
        assert len(set(ids_gpu[t].tolist())) == K
    same = np.setdiff1d(np.arange(len(ids_ref)), diff)
    if len(same):
        assert np.abs(gates_gpu[same] - gates_ref[same]).max() <= TOL["f32"]
    return np.nonzero(tie)[0], diff
