"""The oracle's pins must catch plausible mistakes.  Each case below plants
one mistake (a flipped comparison, a dropped term, a wrong index, a
transposed operand, an off-by-one) in a copy of oracle/moe_oracle.c,
compiles it, and runs tests/test_oracle_pins.py against it; the pin suite
must fail.  The committed oracle is never modified."""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = [
    ("tie goes to the higher expert index",
     "if (!taken[e] && (best < 0 || L[e] > L[best])) best = e;",
     "if (!taken[e] && (best < 0 || L[e] >= L[best])) best = e;"),
    ("softmax not shifted by the kept maximum but by the first expert",
     "double lmax = L[ids[0]], z = 0.0;",
     "double lmax = L[0], z = 0.0;\n        lmax = lmax + 1e-3;"),
    ("margin sign flipped",
     "*margin = L[ids[K - 1]] - L[next];",
     "*margin = L[next] - L[ids[K - 1]];"),
    ("router bias dropped",
     "for (int e = 0; e < E; ++e) L[e] += (double)bias[e];",
     "for (int e = 0; e < E; ++e) L[e] += 0.0 * (double)bias[e];"),
    ("router weight transposed",
     "const float* wrow = w_r + (int64_t)k * E;\n        for (int e = 0; e < E; ++e) L[e] += xk * (double)wrow[e];",
     "for (int e = 0; e < E; ++e) L[e] += xk * (double)w_r[((int64_t)e * d + k) % ((int64_t)d * E)];"),
    ("offsets inclusive instead of exclusive",
     "for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];",
     "for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];\n    for (int e = 0; e < E; ++e) offsets[e] += counts[e] > 0 ? 1 : 0;"),
    ("permutation not stable (slot-major order)",
     "for (int t = 0; t < N; ++t)\n        for (int j = 0; j < K; ++j) {\n            int e = ids[(int64_t)t * K + j];",
     "for (int j0 = 0; j0 < K * N; ++j0) {\n            int j = j0 / N, t = j0 % N;\n            int e = ids[(int64_t)t * K + j];"),
    ("expert weight indexed input-major (transposed operand)",
     "case ORC_BF16: {\n        const uint16_t* p = (const uint16_t*)w + base;\n        for (int k = 0; k < din; ++k) acc += a[k] * orc_bf16_to_f64(p[k]);",
     "case ORC_BF16: {\n        const uint16_t* p = (const uint16_t*)w;\n        int64_t nrow = base / din, nrows = 1 + nrow;\n        for (int k = 0; k < din; ++k) acc += a[k] * orc_bf16_to_f64(p[(k * nrows + nrow) % (base + din)]);"),
    ("SwiGLU activation applied to the up projection",
     "h[n] = silu(g) * u;",
     "h[n] = g * silu(u);"),
    ("ReLU dropped",
     "h[n] = g > 0.0 ? g : 0.0;",
     "h[n] = g;"),
    ("combine uses the gate of the next slot",
     "double g = gates[(int64_t)t * K + j];",
     "double g = gates[(int64_t)t * K + (j + 1) % K];"),
    ("fp8 scales divided instead of multiplied",
     "y[n] = dot_row(din, x, w1, w_dtype, (int64_t)e * F + n) * x_scale * w_scale;",
     "y[n] = dot_row(din, x, w1, w_dtype, (int64_t)e * F + n) / (x_scale * w_scale);"),
    ("dynamic quantization scaled to the e4m3fnuz maximum 240",
     "volatile float scale = amax > 0.0f ? amax / 448.0f : 1.0f;",
     "volatile float scale = amax > 0.0f ? amax / 240.0f : 1.0f;"),
    ("dynamic quantization multiplies by the scale",
     "volatile float q = (float)orc_bf16_to_f64(row[k]) / scale;",
     "volatile float q = (float)orc_bf16_to_f64(row[k]) * scale;"),
    ("e4m3 exponent bias 8 instead of 7",
     "v = ldexp(1.0 + m / 8.0, e - 7);",
     "v = ldexp(1.0 + m / 8.0, e - 8);"),
    ("e4m3 subnormals scaled like normals",
     "v = ldexp((double)m, -9);              /* m/8 * 2^(1-7) */",
     "v = ldexp((double)m, -10);"),
    ("MX scale taken from the next block",
     "orc_e8m0_to_f64(xs[(int64_t)r * nb + k / 32]);",
     "orc_e8m0_to_f64(xs[(int64_t)r * nb + (k / 32 + 1) % nb]);"),
    ("MX weight scales of expert 0 for every expert",
     "orc_e8m0_to_f64(ws[wrow * nb + k / 32]));",
     "orc_e8m0_to_f64(ws[(int64_t)n * nb + k / 32]));"),
    ("E8M0 bias 128 instead of 127",
     "return ldexp(1.0, (int)s - 127);",
     "return ldexp(1.0, (int)s - 128);"),
    ("group of 64 instead of 128 elements",
     "for (int k = 128 * g; k < 128 * g + 128; ++k)",
     "for (int k = 64 * g; k < 64 * g + 128; ++k)"),
    ("group scale of the activations taken from the first group",
     "double sx = xs ? xs[(int64_t)r * ng + g] : x_scale;",
     "double sx = xs ? xs[(int64_t)r * ng] : x_scale;"),
    ("group weight scales indexed group-major",
     "acc += sx * ws[wrow * ng + g] * part;",
     "acc += sx * ws[((int64_t)e * ng + g) * F + n] * part;"),
    ("source token of a permuted row off by one",
     "if (src) src[p] = t;",
     "if (src) src[p] = t + (t + 1 < N);"),
    ("pure unpermute writes slot j from the next slot's row",
     "                       y_perm + (int64_t)pos[(int64_t)t * K + j] * dout, sizeof(double) * (size_t)dout);",
     "                       y_perm + (int64_t)pos[(int64_t)t * K + (j + 1) % K] * dout, sizeof(double) * (size_t)dout);"),
    ("E8M0 code 255 decoded as a number instead of NaN",
     "    if (s == 0xFF) return NAN;\n    return ldexp(1.0, (int)s - 127);",
     "    return ldexp(1.0, (int)s - 127);"),
    ("bf16 widened from the wrong half",
     "uint32_t u = (uint32_t)b << 16;",
     "uint32_t u = ((uint32_t)b << 16) | 0x8000u;"),
]


def _run_mutant(tmp, i, old, new):
    src = open(SRC).read()
    assert old in src, f"mutant {i} no longer matches the oracle source"
    path_c = os.path.join(tmp, f"mutant_{i}.c")
    path_so = os.path.join(tmp, f"libmutant_{i}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new, 1))
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC",
                           "-shared", "-o", path_so, path_c, "-lm"])
    env = dict(os.environ, ORACLE_LIB=path_so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests",
                        "test_oracle_pins.py"), "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
            futs = [ex.submit(_run_mutant, tmp, i, old, new)
                    for i, (_, old, new) in enumerate(MUTANTS)]
            results = [f.result() for f in futs]
    survivors = [MUTANTS[i][0] for i, (rc, _) in enumerate(results) if rc == 0]
    assert not survivors, f"mistakes not caught by any pin: {survivors}"
