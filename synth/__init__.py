"""Seeded synthetic inputs for the one-GPU MoE layer forward.

This module is the only code that both the CUDA path's tests/bench and the
CPU oracle consume.  It draws random numbers and lays them out in the byte
formats the layer takes; it holds none of the layer's arithmetic (no logits,
no top-k, no softmax, no permutation, no matmul).

Workloads (the five shapes the layer is measured and checked on):

* ``fp32_n256_d256_e8_k2_f1024_relu``      fp32, ReLU FFN d->1024->d
* ``bf16_n4096_d2048_e8_k2_f8192_swiglu``   bf16, SwiGLU FFN, ~uniform routing
* ``bf16_n64_d4096_e64_k8_f1408_swiglu``    bf16, decode-shaped (weight streaming)
* ``bf16_n16384_d2048_e128_k8_f768_swiglu_zipf``  bf16, fine-grained experts,
  router bias 1.2*ln(1/rank) (Zipf-like skew, some experts empty)
* ``e4m3_n8192_h7168_e256_k8_n2048_gmm``    fp8 e4m3 per-tensor grouped matmul
  + token-major unpermute, plus a shared-expert matmul (8192x7168)@(7168x2048)
* ``e4m3mx_n8192_h7168_e256_k8_n2048_gmm``  the same grouped matmul with MX block
  scales (OCP MXFP8: one E8M0 scale per 32 consecutive elements along H1)
* ``e4m3blk_n8192_h7168_e256_k8_n2048_gmm``  the same grouped matmul with fp32 scales per
  128 x 128 weight block and per token and 128-element group of the activations
* ``e4m3grp_n8192_h7168_e256_k8_n2048_gmm``  the same with fp32 scales per output column and
  128-element group of K for the weights (per token and group for the activations)
* ``e4m3_n2048_h7168_e64_k8_n2048_gmm``, ``e4m3mx_n2048_h7168_e64_k8_n2048_gmm``,
  ``e4m3blk_n2048_h7168_e64_k8_n2048_gmm``, ``e4m3grp_n2048_h7168_e64_k8_n2048_gmm`` reduced copies of
  the fp8 layers for kernel profiling

Value recipe: x ~ N(0,1); router and expert weights ~ N(0, 1/fan_in)
(fan_in = d for the router and the first FFN matrices, F for the second);
for the fp8 workload x and W ~ N(0,1) quantised with one amax scale per
tensor (scale = amax/448, e4m3 round-to-nearest-even, saturating), or, for
the MX workload, per block of 32 (scale 2^(floor(log2 amax) - 8)).  Routing
for the fp8 workload is an ordered set of K distinct experts per token, drawn
uniformly (the same law as the top-K of iid N(0,1) logits).

Physical weight layout: every expert matrix is stored output-major,
``(E, d_out, d_in)`` row-major (the layout of a Linear layer's weight), i.e.
the per-expert transpose of the logical ``(e, H1, N1)`` gmmWeight shape of the
Ascend grouped-matmul page ("aclnnQuantGroupedMatMulAlltoAllv", parameter
constraints).  The router weight is ``(d, E)`` row-major fp32.

Random streams: numpy Philox bit generators seeded from
``SeedSequence([seed, stream_id])`` and spawned per 16 Mi-element chunk, so
the bytes are independent of the thread count.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

DTYPE_F32 = "f32"
DTYPE_BF16 = "bf16"
DTYPE_E4M3 = "e4m3"

ACT_NONE = "none"
ACT_RELU = "relu"
ACT_SWIGLU = "swiglu"

SEED_BASE = 0x4D6F45
_CHUNK = 1 << 24


@dataclass(frozen=True)
class MoEConfig:
    """Shape of one MoE layer workload.

    For the fp8 grouped-matmul workload ``d`` is H1 (the routed experts'
    input width), ``F`` is N1 (their output width) and ``shared`` holds
    (H2, N2) of the shared expert.
    """
    name: str
    dtype: str
    N: int
    d: int
    E: int
    K: int
    F: int
    act: str
    index: int = 0
    zipf_bias: float = 0.0          # router bias b_e = zipf_bias * ln(1/(e+1)); 0 = no bias
    shared: tuple | None = None     # (H2, N2) shared-expert matmul, fp8 workload only
    routing: str = "router"         # "router" (logits from x @ W_r) or "given" (drawn ids)
    quant: str = "tensor"           # fp8 scales: "tensor" (one per tensor), "mx" (E8M0 per 32),
                                    # "group" (fp32 per 128 of K and channel), "block" (128 x 128)

    @property
    def d_out(self) -> int:
        return self.F if self.act == ACT_NONE else self.d

    @property
    def R(self) -> int:
        return self.N * self.K

    def scaled(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


CONFIGS: dict[str, MoEConfig] = {}


def _reg(cfg: MoEConfig) -> MoEConfig:
    CONFIGS[cfg.name] = cfg
    return cfg


FP32_RELU = _reg(MoEConfig("fp32_n256_d256_e8_k2_f1024_relu", DTYPE_F32, 256, 256, 8, 2, 1024,
                           ACT_RELU, index=0))
BF16_PREFILL = _reg(MoEConfig("bf16_n4096_d2048_e8_k2_f8192_swiglu", DTYPE_BF16, 4096, 2048, 8, 2,
                              8192, ACT_SWIGLU, index=1))
BF16_DECODE = _reg(MoEConfig("bf16_n64_d4096_e64_k8_f1408_swiglu", DTYPE_BF16, 64, 4096, 64, 8,
                             1408, ACT_SWIGLU, index=2))
BF16_FINEGRAINED = _reg(MoEConfig("bf16_n16384_d2048_e128_k8_f768_swiglu_zipf", DTYPE_BF16, 16384,
                                  2048, 128, 8, 768, ACT_SWIGLU, index=3, zipf_bias=1.2))
FP8_GMM = _reg(MoEConfig("e4m3_n8192_h7168_e256_k8_n2048_gmm", DTYPE_E4M3, 8192, 7168, 256, 8, 2048,
                         ACT_NONE, index=4, shared=(7168, 2048), routing="given"))
MX_GMM = _reg(MoEConfig("e4m3mx_n8192_h7168_e256_k8_n2048_gmm", DTYPE_E4M3, 8192, 7168, 256, 8,
                        2048, ACT_NONE, index=5, routing="given", quant="mx"))
BLOCK_GMM = _reg(MoEConfig("e4m3blk_n8192_h7168_e256_k8_n2048_gmm", DTYPE_E4M3, 8192, 7168, 256, 8,
                           2048, ACT_NONE, index=8, routing="given", quant="block"))
GROUP_GMM = _reg(MoEConfig("e4m3grp_n8192_h7168_e256_k8_n2048_gmm", DTYPE_E4M3, 8192, 7168, 256, 8,
                           2048, ACT_NONE, index=10, routing="given", quant="group"))
# Reduced copies of the two fp8 layers (a quarter of the tokens, E = 64, the
# same per-expert shape and ~256 rows per expert): small enough for kernel
# captures that replay every launch many times, weights (0.94 GB) still far
# larger than L2.
FP8_GMM_PROFILE = _reg(MoEConfig("e4m3_n2048_h7168_e64_k8_n2048_gmm", DTYPE_E4M3, 2048, 7168, 64, 8,
                                 2048, ACT_NONE, index=6, shared=(7168, 2048), routing="given"))
MX_GMM_PROFILE = _reg(MoEConfig("e4m3mx_n2048_h7168_e64_k8_n2048_gmm", DTYPE_E4M3, 2048, 7168, 64,
                                8, 2048, ACT_NONE, index=7, routing="given", quant="mx"))
BLOCK_GMM_PROFILE = _reg(MoEConfig("e4m3blk_n2048_h7168_e64_k8_n2048_gmm", DTYPE_E4M3, 2048, 7168,
                                   64, 8, 2048, ACT_NONE, index=9, routing="given", quant="block"))
GROUP_GMM_PROFILE = _reg(MoEConfig("e4m3grp_n2048_h7168_e64_k8_n2048_gmm", DTYPE_E4M3, 2048, 7168,
                                   64, 8, 2048, ACT_NONE, index=11, routing="given", quant="group"))


# ----------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------

def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_f32(seed: int, stream: int, n: int, std: float = 1.0) -> np.ndarray:
    """n iid N(0, std^2) float32 values, chunked Philox streams."""
    out = np.empty(n, np.float32)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    children = np.random.SeedSequence([seed, stream]).spawn(nchunks)

    def work(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.Philox(children[i]))
        v = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[lo:hi] = v

    if nchunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def uniform_u64(seed: int, stream: int, n: int) -> np.ndarray:
    g = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, stream])))
    return g.integers(0, np.iinfo(np.uint64).max, size=n, dtype=np.uint64, endpoint=True)


# ----------------------------------------------------------------------------
# storage formats (input preparation only)
# ----------------------------------------------------------------------------

def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 -> bf16 (round to nearest even), as a torch CPU tensor."""
    return torch.from_numpy(a).to(torch.bfloat16)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Encode float values as e4m3 codes (see _e4m3_encode_block), in
    cache-sized blocks."""
    v = np.asarray(v, np.float64)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, np.uint8)
    blk = 1 << 18
    for lo in range(0, flat.size, blk):
        out[lo:lo + blk] = _e4m3_encode_block(flat[lo:lo + blk])
    return out.reshape(v.shape)


def _e4m3_encode_block(v: np.ndarray) -> np.ndarray:
    """Encode float values as OCP FP8 E4M3 ("FN": bias 7, max 448, no inf)
    bytes, round-to-nearest-even, saturating to +-448.  Input preparation for
    the pre-quantised fp8 workload (the grouped matmul consumes codes and
    scales, as the Ascend page's gmmX/gmmWeight do)."""
    v = np.asarray(v, np.float64)
    sign = (v.view(np.uint64) >> np.uint64(63)).astype(np.uint8) << np.uint8(7)
    a = np.minimum(np.abs(v), 448.0)
    bits = a.view(np.int64)
    e = (bits >> 52) - 1023                      # unbiased exponent
    m = bits & ((1 << 52) - 1)                   # 52 fraction bits
    # keep 3 fraction bits, round to nearest even; q == 8 carries into e
    q = (m + ((1 << 48) - 1) + ((m >> 49) & 1)) >> 49
    code = ((e + 7) << 3) + q
    # below the smallest normal (2^-6) the grid step is 2^-9
    code = np.where(a < 2.0 ** -6, np.rint(a * 512.0).astype(np.int64), code)
    return code.astype(np.uint8) | sign


def quantize_e4m3_per_tensor(a: np.ndarray) -> tuple[np.ndarray, float]:
    """(codes, scale) with scale = amax/448 and codes = e4m3(a / scale)."""
    amax = float(np.max(np.abs(a))) if a.size else 1.0
    scale = float(np.float32(amax / 448.0)) if amax > 0 else 1.0
    out = np.empty(a.shape, np.uint8)
    flat_in, flat_out = a.reshape(-1), out.reshape(-1)
    n = flat_in.size
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def work(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        flat_out[lo:hi] = e4m3_encode(flat_in[lo:hi].astype(np.float64) / scale)

    _run(work, nchunks)
    return out, scale


def quantize_e4m3_rows(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation of a 2-D array: scale[i] = amax(|a[i]|)/448
    (1 for an all-zero row), codes[i] = e4m3(a[i] / scale[i])."""
    amax = np.max(np.abs(a), axis=1).astype(np.float64)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    codes = e4m3_encode(a.astype(np.float64) / scale.astype(np.float64)[:, None])
    return codes, scale


def normal_e4m3(seed: int, stream: int, n: int) -> tuple[np.ndarray, float]:
    """n iid N(0,1) draws quantised per tensor to e4m3, without holding the
    float draws: pass 1 finds amax chunk by chunk, pass 2 redraws each chunk
    (same stream) and encodes it.  Same bytes as
    quantize_e4m3_per_tensor(normal_f32(seed, stream, n))."""
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    children = np.random.SeedSequence([seed, stream]).spawn(nchunks)

    def draw(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        return lo, hi, np.random.Generator(np.random.Philox(children[i])).standard_normal(
            hi - lo, dtype=np.float32)

    amax = np.zeros(nchunks)

    def pass1(i):
        amax[i] = float(np.max(np.abs(draw(i)[2])))

    _run(pass1, nchunks)
    a = float(amax.max())
    scale = float(np.float32(a / 448.0)) if a > 0 else 1.0
    out = np.empty(n, np.uint8)

    def pass2(i):
        lo, hi, v = draw(i)
        out[lo:hi] = e4m3_encode(v.astype(np.float64) / scale)

    _run(pass2, nchunks)
    return out, scale


def quantize_mx(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """OCP MXFP8 (E4M3) quantisation along the last axis (a multiple of 32):
    each block of 32 gets the E8M0 scale 2^X, X = floor(log2(amax)) - 8 (8 =
    the exponent of e4m3's largest normal, 448 = 1.75 * 2^8), clamped to
    [-127, 127]; its elements become e4m3(v / 2^X), round to nearest even,
    saturating.  An all-zero block gets X = -127 (scale code 0).  Returns
    (codes uint8, same shape; scales uint8, last axis / 32)."""
    a = np.asarray(a, np.float64)
    d = a.shape[-1]
    assert d % 32 == 0, "MX blocks are 32 elements"
    b = a.reshape(-1, d // 32, 32)
    amax = np.max(np.abs(b), axis=2)
    _, ex = np.frexp(amax)                  # amax = m * 2^ex, m in [0.5, 1): floor(log2) = ex - 1
    X = np.where(amax > 0, ex.astype(np.int64) - 1 - 8, -127)
    X = np.clip(X, -127, 127)
    codes = e4m3_encode(b / np.ldexp(1.0, X)[..., None])
    return codes.reshape(a.shape), (X + 127).astype(np.uint8).reshape(a.shape[:-1] + (d // 32,))


def quantize_groups(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """e4m3 quantisation with one fp32 scale per 128 consecutive elements of
    the last axis: scale = amax/448 (1 for an all-zero group), codes
    e4m3(v / scale) rounded to nearest even, saturating."""
    a = np.asarray(a, np.float64)
    d = a.shape[-1]
    assert d % 128 == 0, "groups are 128 elements"
    b = a.reshape(-1, d // 128, 128)
    amax = np.max(np.abs(b), axis=2)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    codes = e4m3_encode(b / scale.astype(np.float64)[..., None])
    return codes.reshape(a.shape), scale.reshape(a.shape[:-1] + (d // 128,))


def quantize_blocks(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """e4m3 quantisation of (E, F, d) weights with one fp32 scale per 128 x 128
    block (128 output channels x 128 elements of K; the last channel block may
    be ragged): scale = amax/448 (1 for an all-zero block)."""
    w = np.asarray(w, np.float64)
    E, F, d = w.shape
    assert d % 128 == 0
    fb = (F + 127) // 128
    pad = np.zeros((E, fb * 128, d))
    pad[:, :F] = w
    b = pad.reshape(E, fb, 128, d // 128, 128)
    amax = np.max(np.abs(b), axis=(2, 4))
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    codes = e4m3_encode(b / scale.astype(np.float64)[:, :, None, :, None])
    return codes.reshape(E, fb * 128, d)[:, :F], scale


def normal_mx(seed: int, stream: int, rows: int, cols: int) -> tuple[np.ndarray, np.ndarray]:
    """rows x cols iid N(0,1) draws quantised to MXFP8 (quantize_mx), chunk by
    chunk of whole rows: (codes (rows, cols) uint8, scales (rows, cols/32))."""
    rows_per = max(1, _CHUNK // cols)
    nchunks = max(1, (rows + rows_per - 1) // rows_per)
    children = np.random.SeedSequence([seed, stream]).spawn(nchunks)
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 32), np.uint8)

    def work(i):
        lo, hi = i * rows_per, min(rows, (i + 1) * rows_per)
        v = np.random.Generator(np.random.Philox(children[i])).standard_normal(
            (hi - lo) * cols, dtype=np.float32).reshape(hi - lo, cols)
        codes[lo:hi], scales[lo:hi] = quantize_mx(v)

    _run(work, nchunks)
    return codes, scales


def _run(fn, nchunks):
    if nchunks == 1:
        fn(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fn, range(nchunks)))


# ----------------------------------------------------------------------------
# the workload
# ----------------------------------------------------------------------------

@dataclass
class MoEInputs:
    """Host (CPU) tensors of one workload.

    ``x``       (N, d) in the workload dtype (f32 / bf16 / uint8 e4m3 codes)
    ``w_r``     (d, E) float32, or None when routing is given
    ``bias``    (E,) float32 or None
    ``w1``      (E, F, d)  first matrix (ReLU W1, SwiGLU gate, or the single fp8 matrix)
    ``w3``      (E, F, d)  SwiGLU up matrix, else None
    ``w2``      (E, d, F)  second matrix, None for the single-matrix workload
    ``ids``     (N, K) int32 routing given to the fp8 workload, else None
    ``x_scale``, ``w_scale``  per-tensor fp32 scales (fp8 workload), else 1.0
    ``w_sh``    (N2, H2) e4m3 shared-expert weight (output-major), ``w_sh_scale``
    """
    cfg: MoEConfig
    x: torch.Tensor
    w_r: torch.Tensor | None
    bias: torch.Tensor | None
    w1: torch.Tensor
    w3: torch.Tensor | None
    w2: torch.Tensor | None
    ids: torch.Tensor | None = None
    x_scale: float = 1.0
    w_scale: float = 1.0
    w_sh: torch.Tensor | None = None
    w_sh_scale: float = 1.0
    x_sf: torch.Tensor | None = None    # (N, d/32) uint8 E8M0, MX workload
    w_sf: torch.Tensor | None = None    # (E, F, d/32) uint8 E8M0, MX workload
    x_gs: torch.Tensor | None = None    # (N, d/128) fp32, group / block workloads
    w_gs: torch.Tensor | None = None    # (E, F, d/128) fp32 (group) or (E, F/128, d/128) (block)
    extra: dict = field(default_factory=dict)


def zipf_bias(E: int, strength: float) -> np.ndarray:
    """b_e = strength * ln(1/rank), rank = e + 1 (natural log), float32."""
    return np.array([strength * math.log(1.0 / (e + 1)) for e in range(E)], np.float32)


def given_routing(seed: int, N: int, E: int, K: int) -> np.ndarray:
    """(N, K) int32: per token an ordered set of K distinct experts, uniform.

    Partial Fisher-Yates per token driven by 64-bit uniforms (bias of the
    modulo reduction is < E/2^64, immaterial)."""
    u = uniform_u64(seed, 91, N * K).reshape(N, K)
    ids = np.empty((N, K), np.int32)
    base = np.arange(E, dtype=np.int32)
    for t in range(N):
        perm = base.copy()
        for j in range(K):
            r = j + int(u[t, j] % np.uint64(E - j))
            perm[j], perm[r] = perm[r], perm[j]
        ids[t] = perm[:K]
    return ids


def make_inputs(cfg: MoEConfig, seed: int | None = None) -> MoEInputs:
    """Draw the workload's inputs.  Deterministic in (cfg shape, seed)."""
    if seed is None:
        seed = SEED_BASE + cfg.index
    N, d, E, K, F = cfg.N, cfg.d, cfg.E, cfg.K, cfg.F
    if cfg.dtype == DTYPE_E4M3 and cfg.quant in ("group", "block"):
        xv = normal_f32(seed, 1, N * d).reshape(N, d)
        xq, xgs = quantize_groups(xv)
        wq = np.empty((E, F, d), np.uint8)
        wgs = np.empty((E, F, d // 128) if cfg.quant == "group" else (E, (F + 127) // 128, d // 128),
                       np.float32)
        def expert(e):   # expert by expert (bounded memory), experts in parallel
            wv = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, 100, e]))) \
                .standard_normal(F * d, dtype=np.float32).reshape(1, F, d)
            if cfg.quant == "group":
                c, sc = quantize_groups(wv[0])
                wq[e], wgs[e] = c, sc
            else:
                c, sc = quantize_blocks(wv)
                wq[e], wgs[e] = c[0], sc[0]

        _run(expert, E)
        return MoEInputs(cfg, torch.from_numpy(xq), None, None, torch.from_numpy(wq), None, None,
                         ids=torch.from_numpy(given_routing(seed, N, E, K)),
                         x_gs=torch.from_numpy(xgs), w_gs=torch.from_numpy(wgs))
    if cfg.dtype == DTYPE_E4M3 and cfg.quant == "mx":
        xq, xsf = normal_mx(seed, 1, N, d)
        wq, wsf = normal_mx(seed, 2, E * F, d)
        return MoEInputs(cfg, torch.from_numpy(xq), None, None,
                         torch.from_numpy(wq.reshape(E, F, d)), None, None,
                         ids=torch.from_numpy(given_routing(seed, N, E, K)),
                         x_sf=torch.from_numpy(xsf),
                         w_sf=torch.from_numpy(wsf.reshape(E, F, d // 32)))
    if cfg.dtype == DTYPE_E4M3:
        xq, xs = normal_e4m3(seed, 1, N * d)
        wq, ws = normal_e4m3(seed, 2, E * F * d)
        inp = MoEInputs(cfg, torch.from_numpy(xq.reshape(N, d)), None, None,
                        torch.from_numpy(wq.reshape(E, F, d)), None, None,
                        ids=torch.from_numpy(given_routing(seed, N, E, K)), x_scale=xs, w_scale=ws)
        if cfg.shared is not None:
            H2, N2 = cfg.shared
            assert H2 == d, "the shared expert reads the same token matrix"
            shq, shs = normal_e4m3(seed, 3, N2 * H2)
            inp.w_sh, inp.w_sh_scale = torch.from_numpy(shq.reshape(N2, H2)), shs
        return inp

    conv = (lambda a: torch.from_numpy(a)) if cfg.dtype == DTYPE_F32 else to_bf16
    x = conv(normal_f32(seed, 1, N * d).reshape(N, d))
    w_r = torch.from_numpy(normal_f32(seed, 4, d * E, 1.0 / math.sqrt(d)).reshape(d, E))
    bias = torch.from_numpy(zipf_bias(E, cfg.zipf_bias)) if cfg.zipf_bias else None
    w1 = conv(normal_f32(seed, 2, E * F * d, 1.0 / math.sqrt(d)).reshape(E, F, d))
    w3 = None
    if cfg.act == ACT_SWIGLU:
        w3 = conv(normal_f32(seed, 5, E * F * d, 1.0 / math.sqrt(d)).reshape(E, F, d))
    w2 = None
    if cfg.act != ACT_NONE:
        w2 = conv(normal_f32(seed, 6, E * d * F, 1.0 / math.sqrt(F)).reshape(E, d, F))
    return MoEInputs(cfg, x, w_r, bias, w1, w3, w2)


def small_variant(cfg: MoEConfig, **kw) -> MoEConfig:
    """A reduced copy of a workload (same dtype/act/routing law) for tests."""
    return replace(cfg, name=cfg.name + "_small", **kw)


def dtype_bytes(dtype: str) -> int:
    return {DTYPE_F32: 4, DTYPE_BF16: 2, DTYPE_E4M3: 1}[dtype]
