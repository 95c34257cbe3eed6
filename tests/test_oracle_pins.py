"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: values
worked by hand (tests/golden), closed forms, invariants, brute force on tiny
inputs, or a library routine (numpy / torch fp64) on a special case.  None of
these needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats

def test_e4m3_decode_golden(orc):
    g = _gold("e4m3_codes.json")
    for c, v in zip(g["codes"], g["values"]):
        got = orc.e4m3_to_f64(c)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (c, got, v)
    for v, c in g["rne"]:
        assert orc.f64_to_e4m3(v) == c, (v, orc.f64_to_e4m3(v), c)


def test_e4m3_all_codes_roundtrip_and_order(orc):
    vals = []
    for c in range(256):
        v = orc.e4m3_to_f64(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v)
            continue
        assert orc.f64_to_e4m3(v) == c or (v == 0.0 and c in (0, 128)), c
        if c < 128:
            vals.append(v)
    # positive codes are strictly increasing in value (monotone encoding)
    assert all(a < b for a, b in zip(vals, vals[1:]))
    assert max(vals) == 448.0


def test_e4m3_generator_encoder_agrees_with_oracle(orc):
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 1e-1, 1.0, 30.0, 300.0)])
    mids = [(orc.e4m3_to_f64(c) + orc.e4m3_to_f64(c + 1)) / 2 for c in range(0, 126)]
    v = np.concatenate([v, mids, -np.array(mids), [500.0, -1e9]])
    gen = synth.e4m3_encode(v)
    ref = np.array([orc.f64_to_e4m3(float(a)) for a in v], np.uint8)
    assert np.array_equal(gen, ref)


def test_bf16_decode_and_rne(orc):
    assert orc.bf16_to_f64(0x3F80) == 1.0
    assert orc.bf16_to_f64(0xC000) == -2.0
    assert orc.bf16_to_f64(0x0001) == 2.0 ** -133
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even (1.0)
    assert orc.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert orc.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert orc.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    # agrees with torch's float32 -> bf16 on values exact in float32
    rng = np.random.default_rng(3)
    v = rng.standard_normal(2000).astype(np.float32)
    t = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    o = np.array([orc.f64_to_bf16(float(a)) for a in v], np.uint16)
    assert np.array_equal(t, o)
    dec = orc.to_f64(torch.from_numpy(v).to(torch.bfloat16), orc.BF16)
    assert np.array_equal(dec, torch.from_numpy(v).to(torch.bfloat16).double().numpy())


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("name", ["router_top2_worked.json", "router_tie_worked.json"])
def test_router_worked_examples(orc, name):
    g = _gold(name)
    x = np.array(g["x"], np.float32)
    w = np.array(g["w_r"], np.float32)
    ids, gates, margin, _ = orc.router(x, orc.F32, w, None, g["K"])
    assert ids.tolist() == g["ids"]
    assert np.allclose(gates, g["gates"], rtol=0, atol=1e-15)
    assert np.allclose(margin, g["margin"], rtol=0, atol=0)


def test_router_logits_match_library_matmul(orc):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((40, 96)).astype(np.float32)
    w = (rng.standard_normal((96, 24)) / 10).astype(np.float32)
    b = rng.standard_normal(24).astype(np.float32)
    _, _, _, L = orc.router(x, orc.F32, w, b, 3, want_logits=True)
    ref = torch.from_numpy(x).double() @ torch.from_numpy(w).double() + torch.from_numpy(b).double()
    assert np.allclose(L, ref.numpy(), rtol=1e-13, atol=1e-13)


def _sort_topk(L, K):
    order = sorted(range(len(L)), key=lambda e: (-L[e], e))
    return order[:K], (L[order[K - 1]] - L[order[K]] if K < len(L) else math.inf)


def test_router_topk_bruteforce_with_ties(orc):
    rng = np.random.default_rng(5)
    for E in (1, 2, 3, 5, 8):
        for K in range(1, E + 1):
            # integer logits on a tiny range: many exact ties
            L = rng.integers(-2, 3, size=(64, E)).astype(np.float64)
            ids, gates, margin = orc.topk_from_logits(L, K)
            for t in range(64):
                want, m = _sort_topk(list(L[t]), K)
                assert ids[t].tolist() == want, (E, K, t, L[t])
                assert margin[t] == m
                sel = L[t][want]
                ref = torch.softmax(torch.tensor(sel, dtype=torch.float64), 0).numpy()
                assert np.allclose(gates[t], ref, rtol=0, atol=1e-15)


def test_router_full_softmax_when_k_equals_e(orc):
    rng = np.random.default_rng(9)
    L = rng.standard_normal((32, 8)) * 3
    ids, gates, margin = orc.topk_from_logits(L, 8)
    full = torch.softmax(torch.from_numpy(L), 1).numpy()
    for t in range(32):
        assert np.allclose(gates[t], full[t][ids[t]], rtol=0, atol=1e-15)
        assert set(ids[t].tolist()) == set(range(8))
    assert np.all(np.isinf(margin))


def test_router_gate_properties(orc):
    rng = np.random.default_rng(21)
    L = rng.standard_normal((200, 16)) * 4
    for K in (1, 2, 4, 8):
        ids, gates, _ = orc.topk_from_logits(L, K)
        assert np.allclose(gates.sum(1), 1.0, atol=1e-12)
        assert np.all(gates > 0) and np.all(gates <= 1)
        assert np.all(np.diff(gates, axis=1) <= 0)
        # K == 2 closed form: g0 = logistic(L0 - L1)
        if K == 2:
            d = L[np.arange(200), ids[:, 0]] - L[np.arange(200), ids[:, 1]]
            assert np.allclose(gates[:, 0], 1 / (1 + np.exp(-d)), atol=1e-14)
    # equal kept logits -> 1/K each
    ids, gates, _ = orc.topk_from_logits(np.zeros((3, 6)), 4)
    assert np.allclose(gates, 0.25, atol=0) and ids.tolist() == [[0, 1, 2, 3]] * 3


def test_router_softmax_is_stable_for_large_logits(orc):
    """The softmax subtracts the largest kept logit: logits far from zero give
    finite gates equal to the closed form (K = 2: logistic of the gap)."""
    L = np.array([[0.0, 800.0, 900.0, -50.0], [-1000.0, -999.0, -2000.0, -1500.0]])
    ids, gates, margin = orc.topk_from_logits(L, 2)
    assert ids.tolist() == [[2, 1], [1, 0]]
    assert np.isfinite(gates).all()
    assert np.allclose(gates[0], [1 / (1 + np.exp(-100.0)), 1 - 1 / (1 + np.exp(-100.0))], atol=1e-15)
    assert np.allclose(gates[1], [1 / (1 + np.exp(-1.0)), 1 / (1 + np.exp(1.0))], atol=1e-15)
    assert margin.tolist() == [800.0, 500.0]


def test_router_zipf_bias_closed_form(orc):
    """x = 0 leaves only the bias 1.2*ln(1/(e+1)): ids = 0..K-1, g_j ~ (j+1)^-1.2."""
    E, K, d = 128, 8, 16
    bias = synth.zipf_bias(E, 1.2)
    x = np.zeros((4, d), np.float32)
    w = np.ones((d, E), np.float32)
    ids, gates, margin, _ = orc.router(x, orc.F32, w, bias, K)
    assert ids.tolist() == [list(range(K))] * 4
    p = np.array([(j + 1) ** -1.2 for j in range(K)])
    assert np.allclose(gates, p / p.sum(), rtol=1e-6)  # bias is fp32: relative 1e-7 per logit
    assert np.allclose(margin, float(bias[K - 1]) - float(bias[K]), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- permute

def _brute_permute(ids, E):
    N, K = ids.shape
    flat = [(t, j, int(ids[t, j])) for t in range(N) for j in range(K)]
    counts = [sum(1 for f in flat if f[2] == e) for e in range(E)]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    pos = []
    for i, (t, j, e) in enumerate(flat):
        earlier = sum(1 for f in flat[:i] if f[2] == e)
        pos.append(offsets[e] + earlier)
    return counts, offsets, pos


@pytest.mark.parametrize("N,E,K", [(1, 1, 1), (7, 3, 2), (33, 8, 2), (50, 16, 8), (20, 5, 5)])
def test_permute_bruteforce(orc, N, E, K):
    rng = np.random.default_rng(N * 100 + E)
    ids = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
    x = rng.integers(0, 255, size=(N, 12), dtype=np.uint8)
    counts, offsets, pos, src, xp = orc.permute(ids, E, x)
    bc, bo, bp = _brute_permute(ids, E)
    assert counts.tolist() == bc and offsets.tolist() == bo and pos.tolist() == bp
    assert counts.sum() == N * K and offsets[E] == N * K
    assert np.array_equal(src[pos], np.repeat(np.arange(N), K))
    assert np.array_equal(xp[pos], np.repeat(x, K, axis=0))
    # stable: within one expert the source tokens are non-decreasing
    for e in range(E):
        seg = src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) >= 0)


def test_permute_duplicate_ids_and_empty_experts(orc):
    ids = np.array([[2, 2], [0, 2], [2, 0]], np.int32)
    counts, offsets, pos, src, _ = orc.permute(ids, 4)
    bc, bo, bp = _brute_permute(ids, 4)
    assert counts.tolist() == bc == [2, 0, 4, 0]
    assert offsets.tolist() == bo and pos.tolist() == bp
    with pytest.raises(ValueError):
        orc.permute(np.array([[0, 4]], np.int32), 4)


def test_unpermute_of_permute_is_identity(orc):
    rng = np.random.default_rng(2)
    N, E, K, D = 64, 8, 3, 10
    ids = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
    x = rng.standard_normal((N, D))
    _, _, pos, _, xp = orc.permute(ids, E, x)
    # identity experts + pure reorder: y[t*K + j] = x[t] bitwise
    y = orc.combine(pos, None, xp, N, K)
    assert np.array_equal(y, np.repeat(x, K, axis=0))
    # gate-weighted combine of identity experts: sum_j g_j x = x
    L = rng.standard_normal((N, E))
    _, gates, _ = orc.topk_from_logits(L, K)
    y = orc.combine(pos, gates, xp, N, K)
    assert np.allclose(y, x, rtol=0, atol=1e-13)


def test_pure_unpermute_returns_each_slot_its_own_expert(orc):
    """Label every permuted row with the expert whose segment (from the
    offsets) holds it: the pure reorder must put label ids[t][j] in slot
    t*K + j -- each slot gets its own expert's result, whatever the order of
    the slots (identity experts cannot tell slots of one token apart)."""
    rng = np.random.default_rng(12)
    N, E, K = 50, 9, 4
    ids = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
    _, offsets, pos, _, _ = orc.permute(ids, E)
    labels = np.repeat(np.arange(E, dtype=np.float64), np.diff(offsets))[:, None]
    y = orc.combine(pos, None, labels, N, K)
    assert np.array_equal(y[:, 0], ids.reshape(-1).astype(np.float64))


# ---------------------------------------------------------------- experts

def _scaled_identity_experts(E, D, c, dtype):
    w = np.zeros((E, D, D), np.float32)
    for e in range(E):
        w[e] = np.eye(D, dtype=np.float32) * c[e]
    return torch.from_numpy(w) if dtype == "f32" else torch.from_numpy(w).to(torch.bfloat16)


def test_k_equals_e_scalar_experts_closed_form(orc):
    """K = E and E_e(x) = c_e x: y = (sum_e softmax(L)_e c_e) x."""
    rng = np.random.default_rng(4)
    N, D, E = 24, 16, 6
    c = np.array([0.5, 1.0, 2.0, -1.0, 0.25, 3.0])
    x = rng.standard_normal((N, D)).astype(np.float32)
    w_r = rng.standard_normal((D, E)).astype(np.float32)
    w1 = _scaled_identity_experts(E, D, c, "f32")
    cfg = synth.MoEConfig("t", "f32", N, D, E, E, D, "none")
    inp = synth.MoEInputs(cfg, torch.from_numpy(x), torch.from_numpy(w_r), None, w1, None, None)
    y, ids, gates, _ = orc.forward_tokens(inp, np.arange(N))
    L = x.astype(np.float64) @ w_r.astype(np.float64)
    s = torch.softmax(torch.from_numpy(L), 1).numpy() @ c
    assert np.allclose(y, s[:, None] * x.astype(np.float64), rtol=1e-13, atol=1e-13)


def _moe_tiny(act, dtype, N=20, d=16, E=4, K=2, F=24, seed=1):
    cfg = synth.MoEConfig("tiny", dtype, N, d, E, K, F, act)
    return synth.make_inputs(cfg, seed)


@pytest.mark.parametrize("act", ["relu", "swiglu", "none"])
def test_single_expert_matches_library_matmul(orc, act):
    """E = 1: the expert FFN is a plain matmul chain; compare with torch fp64."""
    inp = _moe_tiny(act, "bf16", N=12, d=32, E=1, K=1, F=40)
    X = inp.x.double()
    W1 = inp.w1[0].double()
    y = orc.expert_rows(np.zeros(12, np.int32), inp.x, orc.BF16, act, inp.w1, inp.w3, inp.w2, orc.BF16)
    if act == "none":
        ref = X @ W1.T
    else:
        a = X @ W1.T
        if act == "relu":
            h = torch.relu(a)
        else:
            h = torch.nn.functional.silu(a) * (X @ inp.w3[0].double().T)
        ref = h @ inp.w2[0].double().T
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_fp8_grouped_matmul_exact_integers(orc):
    """Small integers are exact in e4m3 and their products sum exactly in fp64:
    gmmY = (X @ W_e) * xs * ws computed by brute-force Python integers."""
    rng = np.random.default_rng(8)
    E, F, din, R = 3, 5, 9, 7
    Xi = rng.integers(-8, 9, size=(R, din))
    Wi = rng.integers(-8, 9, size=(E, F, din))
    enc = np.vectorize(orc.f64_to_e4m3, otypes=[np.uint8])
    Xq, Wq = enc(Xi.astype(np.float64)), enc(Wi.astype(np.float64))
    rexp = rng.integers(0, E, size=R).astype(np.int32)
    xs, ws = 0.5, 0.25
    y = orc.expert_rows(rexp, Xq, orc.E4M3, "none", Wq, None, None, orc.E4M3, xs, ws)
    for r in range(R):
        for n in range(F):
            exact = sum(int(Xi[r, k]) * int(Wi[rexp[r], n, k]) for k in range(din))
            assert y[r, n] == exact * xs * ws


def test_fp8_per_channel_and_per_token_scales_exact(orc):
    """Ascend quant modes 2 (per-channel weights) and 3 (per-token x): with
    small-integer codes the product sums are exact, so y = (sum x w) * xs[r] *
    ws[e][n] is checked against Python integers times the scales."""
    rng = np.random.default_rng(13)
    E, F, din, R = 3, 6, 10, 9
    Xi = rng.integers(-8, 9, size=(R, din))
    Wi = rng.integers(-8, 9, size=(E, F, din))
    enc = np.vectorize(orc.f64_to_e4m3, otypes=[np.uint8])
    Xq, Wq = enc(Xi.astype(np.float64)), enc(Wi.astype(np.float64))
    rexp = rng.integers(0, E, size=R).astype(np.int32)
    xs = 2.0 ** rng.integers(-6, 3, size=R)
    ws = 2.0 ** rng.integers(-6, 3, size=(E, F))
    y = orc.expert_rows_scaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3, x_row_scales=xs,
                               w_channel_scales=ws)
    for r in range(R):
        for n in range(F):
            exact = sum(int(Xi[r, k]) * int(Wi[rexp[r], n, k]) for k in range(din))
            assert y[r, n] == exact * xs[r] * ws[rexp[r], n]
    # NULL arrays fall back to the per-tensor scalars of the plain function
    y0 = orc.expert_rows_scaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3, x_scale=0.5, w_scale=0.25)
    y1 = orc.expert_rows(rexp, Xq, orc.E4M3, "none", Wq, None, None, orc.E4M3, 0.5, 0.25)
    assert np.array_equal(y0, y1)


def test_e8m0_decode_definition(orc):
    """OCP MX E8M0 scale: 2^(code - 127), code 255 is NaN."""
    assert orc.e8m0_to_f64(127) == 1.0
    assert orc.e8m0_to_f64(128) == 2.0
    assert orc.e8m0_to_f64(120) == 2.0 ** -7
    assert orc.e8m0_to_f64(0) == 2.0 ** -127
    assert orc.e8m0_to_f64(254) == 2.0 ** 127
    assert math.isnan(orc.e8m0_to_f64(255))


def _mx_ones(*shape):
    return np.full(shape, 0x38, np.uint8)   # e4m3 1.0


def test_mx_block_scales_closed_form(orc):
    """Quant mode 6 (MX): with every element 1.0 and scales xs[r][b] =
    127 + r + b, ws[e][n][b] = 127 - n + 2b + e, each block of 32 adds
    32 * 2^(r + b) * 2^(2b - n + e), so y[r][n] = 32 * 2^(r - n + e) *
    (8^nb - 1) / 7 with nb = din / 32 blocks.  A block size other than 32,
    a transposed scale index or another expert's scales all change it."""
    E, F, nb, R = 3, 5, 4, 6
    din = 32 * nb
    xs = np.array([[127 + r + b for b in range(nb)] for r in range(R)], np.uint8)
    ws = np.array([[[127 - n + 2 * b + e for b in range(nb)] for n in range(F)] for e in range(E)],
                  np.uint8)
    rexp = np.array([0, 1, 2, 2, 1, 0], np.int32)
    y = orc.expert_rows_mx(rexp, _mx_ones(R, din), xs, _mx_ones(E, F, din), ws)
    for r in range(R):
        e = int(rexp[r])
        for n in range(F):
            assert y[r, n] == 32 * 2.0 ** (r - n + e) * (8 ** nb - 1) / 7


def test_mx_exact_integers_random_block_scales(orc):
    """Small integer codes and random power-of-two block scales: every product
    and partial sum is exact in fp64, so y equals the exact value
    sum_b 2^(xs + ws - 254) * sum_{k in block b} X*W from Python integers."""
    rng = np.random.default_rng(21)
    E, F, nb, R = 3, 4, 3, 7
    din = 32 * nb
    Xi = rng.integers(-8, 9, size=(R, din))
    Wi = rng.integers(-8, 9, size=(E, F, din))
    enc = np.vectorize(orc.f64_to_e4m3, otypes=[np.uint8])
    Xq, Wq = enc(Xi.astype(np.float64)), enc(Wi.astype(np.float64))
    xs = rng.integers(120, 135, size=(R, nb)).astype(np.uint8)
    ws = rng.integers(120, 135, size=(E, F, nb)).astype(np.uint8)
    rexp = rng.integers(0, E, size=R).astype(np.int32)
    rexp[2] = -1
    y = orc.expert_rows_mx(rexp, Xq, xs, Wq, ws)
    assert np.isnan(y[2]).all()
    for r in range(R):
        e = int(rexp[r])
        if e < 0:
            continue
        for n in range(F):
            exact = 0.0
            for b in range(nb):
                blk = sum(int(Xi[r, k]) * int(Wi[e, n, k]) for k in range(32 * b, 32 * b + 32))
                exact += blk * 2.0 ** (int(xs[r, b]) + int(ws[e, n, b]) - 254)
            assert y[r, n] == exact


def test_mx_unit_scales_equal_plain_fp8(orc):
    """With every block scale 1 (code 127) the MX matmul is the per-tensor fp8
    matmul with unit scales, bit for bit (same products, same order)."""
    cfg = synth.MoEConfig("mx1", "e4m3", 12, 64, 4, 2, 24, "none", routing="given", quant="mx")
    inp = synth.make_inputs(cfg, 7)
    rexp = np.arange(12, dtype=np.int32) % 4
    ones_x = np.full((12, 2), 127, np.uint8)
    ones_w = np.full((4, 24, 2), 127, np.uint8)
    y = orc.expert_rows_mx(rexp, inp.x, ones_x, inp.w1, ones_w)
    y0 = orc.expert_rows(rexp, inp.x, orc.E4M3, "none", inp.w1, None, None, orc.E4M3, 1.0, 1.0)
    assert np.array_equal(y, y0)


def test_mx_row_and_column_constant_scales_reduce_to_matmul(orc):
    """When a row's blocks share one scale 2^a[r] and an output column's blocks
    share 2^c[n], y = diag(2^a) (Xd W_e^T) diag(2^c): the library matmul (fp64)
    of the decoded codes, per expert."""
    rng = np.random.default_rng(4)
    cfg = synth.MoEConfig("mx2", "e4m3", 10, 96, 2, 1, 16, "none", routing="given", quant="mx")
    inp = synth.make_inputs(cfg, 11)
    a = rng.integers(118, 136, size=10)
    c = rng.integers(118, 136, size=(2, 16))
    xs = np.repeat(a[:, None], 3, axis=1).astype(np.uint8)
    ws = np.repeat(c[:, :, None], 3, axis=2).astype(np.uint8)
    rexp = np.array([0, 1] * 5, np.int32)
    y = orc.expert_rows_mx(rexp, inp.x, xs, inp.w1, ws)
    dec = np.array([orc.e4m3_to_f64(v) for v in range(256)])
    Xd = torch.from_numpy(dec[inp.x.numpy()])
    for e in range(2):
        rows = np.nonzero(rexp == e)[0]
        Wd = torch.from_numpy(dec[inp.w1[e].numpy()])
        ref = (Xd[rows] @ Wd.T).numpy() * 2.0 ** (a[rows, None] - 127) * 2.0 ** (c[e][None, :] - 127)
        assert np.abs(y[rows] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_mx_quantiser_blocks(orc):
    """The MX input quantiser (OCP MXFP8): a block of e4m3 values whose largest
    magnitude is in [256, 448], times 2^p, gets scale code 127 + p and its
    codes back exactly; an all-zero block gets scale code 0; every block's
    largest element lands in [256, 448] times its scale."""
    base = [448.0, 1.0, -2.0, 0.5, -300.0, 3.5, -448.0, 0.001953125] * 4
    codes_ref = [orc.f64_to_e4m3(v) for v in base]
    for p in (-9, -1, 0, 5):
        c, s = synth.quantize_mx(np.array([[v * 2.0 ** p for v in base]]))
        assert int(s[0, 0]) == 127 + p
        assert [int(v) for v in c[0]] == codes_ref
    c, s = synth.quantize_mx(np.zeros((1, 64)))
    assert not s.any() and not c.any()
    rng = np.random.default_rng(2)
    v = rng.standard_normal((8, 128)) * np.exp(rng.uniform(-5, 5, (8, 1)))
    c, s = synth.quantize_mx(v)
    dec = np.array([orc.e4m3_to_f64(int(q)) for q in c.ravel()]).reshape(c.shape)
    for r in range(8):
        for b in range(4):
            blk = np.abs(dec[r, 32 * b:32 * b + 32])
            assert 256.0 <= blk.max() <= 448.0
            scale = 2.0 ** (int(s[r, b]) - 127)
            err = np.abs(dec[r, 32 * b:32 * b + 32] * scale - v[r, 32 * b:32 * b + 32])
            # half an e4m3 step (2^-4 relative) or the saturation at 448
            big = np.abs(v[r, 32 * b:32 * b + 32]) / scale > 448.0
            assert np.all((err <= np.abs(v[r, 32 * b:32 * b + 32]) * 2.0 ** -4 + 2.0 ** -10 * scale)
                          | big)


def test_group_scales_closed_form(orc):
    """Quant modes 4/5 (fp32 scales per 128-element group of K): with every
    element 1.0, xs[r][g] = 2^(r + g) and ws[e][n][g] = 2^(2g - n + e), each
    group adds 128 * 2^(r - n + e) * 8^g: y = 128 * 2^(r - n + e) * (8^G - 1) / 7.
    A group size other than 128, a transposed index or another expert's
    scales change it."""
    E, F, G, R = 3, 5, 3, 6
    din = 128 * G
    xs = np.array([[2.0 ** (r + g) for g in range(G)] for r in range(R)])
    ws = np.array([[[2.0 ** (2 * g - n + e) for g in range(G)] for n in range(F)] for e in range(E)])
    rexp = np.array([0, 1, 2, 2, 1, 0], np.int32)
    y = orc.expert_rows_kscaled(rexp, _mx_ones(R, din), orc.E4M3, _mx_ones(E, F, din), orc.E4M3,
                                ws, x_group_scales=xs)
    for r in range(R):
        e = int(rexp[r])
        for n in range(F):
            assert y[r, n] == 128 * 2.0 ** (r - n + e) * (8 ** G - 1) / 7


def test_group_scales_exact_integers(orc):
    """Small integer codes, random power-of-two group scales: exact in fp64,
    so y equals sum_g xs * ws * (sum_{k in g} X*W) from Python integers; the
    scalar x_scale replaces missing activation scales."""
    rng = np.random.default_rng(17)
    E, F, G, R = 3, 4, 2, 7
    din = 128 * G
    Xi = rng.integers(-8, 9, size=(R, din))
    Wi = rng.integers(-8, 9, size=(E, F, din))
    enc = np.vectorize(orc.f64_to_e4m3, otypes=[np.uint8])
    Xq, Wq = enc(Xi.astype(np.float64)), enc(Wi.astype(np.float64))
    xs = 2.0 ** rng.integers(-5, 4, size=(R, G))
    ws = 2.0 ** rng.integers(-5, 4, size=(E, F, G))
    rexp = rng.integers(0, E, size=R).astype(np.int32)
    y = orc.expert_rows_kscaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3, ws, x_group_scales=xs)
    y2 = orc.expert_rows_kscaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3, ws, x_scale=0.5)
    for r in range(R):
        e = int(rexp[r])
        for n in range(F):
            parts = [sum(int(Xi[r, k]) * int(Wi[e, n, k]) for k in range(128 * g, 128 * g + 128))
                     for g in range(G)]
            assert y[r, n] == sum(p * xs[r, g] * ws[e, n, g] for g, p in enumerate(parts))
            assert y2[r, n] == sum(p * 0.5 * ws[e, n, g] for g, p in enumerate(parts))


def test_group_scales_constant_over_groups_reduce_to_channel_scales(orc):
    """Scales that do not change along K reduce modes 4/5 to per-channel
    weights times per-token activations (modes 2/3), exactly on integer data."""
    rng = np.random.default_rng(19)
    E, F, G, R = 2, 6, 3, 5
    din = 128 * G
    enc = np.vectorize(orc.f64_to_e4m3, otypes=[np.uint8])
    Xq = enc(rng.integers(-6, 7, size=(R, din)).astype(np.float64))
    Wq = enc(rng.integers(-6, 7, size=(E, F, din)).astype(np.float64))
    a = 2.0 ** rng.integers(-4, 4, size=R)
    c = 2.0 ** rng.integers(-4, 4, size=(E, F))
    rexp = np.array([0, 1, 1, 0, 1], np.int32)
    y = orc.expert_rows_kscaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3,
                                np.repeat(c[:, :, None], G, axis=2),
                                x_group_scales=np.repeat(a[:, None], G, axis=1))
    y0 = orc.expert_rows_scaled(rexp, Xq, orc.E4M3, Wq, orc.E4M3, x_row_scales=a,
                                w_channel_scales=c)
    assert np.array_equal(y, y0)


def test_block_scales_expand_to_channels(orc):
    """A 128 x 128 weight block's scale applies to its 128 output channels:
    channel n of a 300-channel expert takes block n // 128 (the last block
    ragged)."""
    E, F, G = 2, 300, 3
    wb = np.arange(E * 3 * G, dtype=np.float64).reshape(E, 3, G) + 1.0
    wg = orc.block_to_group_scales(wb, F)
    assert wg.shape == (E, F, G)
    for e in range(E):
        for n in (0, 127, 128, 255, 256, 299):
            assert np.array_equal(wg[e, n], wb[e, n // 128])


def test_group_and_block_quantisers(orc):
    """The per-group and per-block input quantisers: a group (or 128 x 128
    block) of e4m3 values whose largest magnitude is 448, times p, gets scale
    p (amax / 448) and its codes back exactly; an all-zero group gets scale
    1 and zero codes; every dequantised group lies within half an e4m3 step."""
    base = np.array([448.0, 1.0, -2.0, 0.5, -300.0, 3.5, -448.0, 0.001953125] * 16)
    codes_ref = [orc.f64_to_e4m3(v) for v in base]
    for p in (0.25, 1.0, 8.0):
        c, s = synth.quantize_groups(np.stack([base * p, np.zeros(128)]))
        assert s[0, 0] == np.float32(p) and s[1, 0] == 1.0
        assert [int(v) for v in c[0]] == codes_ref and not c[1].any()
    rng = np.random.default_rng(6)
    w = rng.standard_normal((2, 200, 256)) * np.exp(rng.uniform(-4, 4, (2, 1, 1)))
    c, s = synth.quantize_blocks(w)
    assert c.shape == w.shape and s.shape == (2, 2, 2)
    dec = np.array([orc.e4m3_to_f64(int(q)) for q in c.ravel()]).reshape(c.shape)
    for e in range(2):
        for nb in range(2):
            for g in range(2):
                blk = np.s_[e, 128 * nb:128 * nb + 128, 128 * g:128 * g + 128]
                amax = np.abs(w[blk]).max()
                assert s[e, nb, g] == np.float32(amax / 448.0)
                err = np.abs(dec[blk] * float(s[e, nb, g]) - w[blk])
                assert np.all(err <= np.abs(w[blk]) * 2.0 ** -4 * (1 + 1e-6)
                              + 2.0 ** -10 * float(s[e, nb, g]))


def test_per_row_quantiser_round_trip():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((50, 64)) * rng.uniform(0.01, 100, size=(50, 1))
    a[3] = 0.0
    codes, scale = synth.quantize_e4m3_rows(a)
    import oracle as orc
    dec = orc.to_f64(codes, orc.E4M3) * scale[:, None]
    # each row's max maps to 448 * scale; e4m3 rounding error is <= 2^-4
    # relative for normal codes, <= half the subnormal step 2^-10 absolute
    bound = 2.0 ** -4 * np.abs(a) + 2.0 ** -10 * scale[:, None].astype(np.float64)
    assert np.all(np.abs(dec - a) <= bound)
    keep = np.arange(50) != 3
    assert np.array_equal(np.abs(dec).max(1)[keep], 448.0 * scale.astype(np.float64)[keep])
    assert scale[3] == 1.0 and np.all(dec[3] == 0)


# ------------------------------------------- per-token dynamic quantization

def _bf16_rows(vals):
    t = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_dynamic_quant_exact_when_row_is_scaled_e4m3(orc):
    """A row that is e4m3 values (largest 448) times a power of two has scale
    exactly that power of two and codes exactly the original ones."""
    base = [448.0, 1.0, -2.0, 0.5, -0.0, 3.5, -448.0, 0.001953125]   # all e4m3 values
    codes_ref = [orc.f64_to_e4m3(v) for v in base]
    for p in (-7, -3, 0, 4):
        row = _bf16_rows([[v * 2.0 ** p for v in base]])
        codes, scales = orc.quantize_rows_dynamic(row)
        assert scales[0] == np.float32(2.0 ** p)
        assert [int(c) for c in codes[0]] == codes_ref


def test_dynamic_quant_bounds_and_extremes(orc):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-6, 6, (64, 1)))
    rows = _bf16_rows(x)
    xd = torch.from_numpy(rows.view(np.int16)).view(torch.bfloat16).double().numpy()
    codes, scales = orc.quantize_rows_dynamic(rows)
    for r in range(64):
        amax = np.abs(xd[r]).max()
        # scale = amax / 448 rounded once to fp32
        assert scales[r] == np.float32(np.float32(amax) / np.float32(448.0))
        deq = np.array([orc.e4m3_to_f64(int(c)) for c in codes[r]]) * float(scales[r])
        # half an e4m3 step: 2^-4 relative for normals, 2^-10 * scale below
        # 2^-6 * scale (subnormal codes); plus the fp32 quotient's rounding
        bound = np.maximum(np.abs(xd[r]) * 2.0 ** -4, 2.0 ** -10 * float(scales[r])) * (1 + 1e-6)
        assert np.all(np.abs(deq - xd[r]) <= bound)
        k = int(np.argmax(np.abs(xd[r])))
        assert codes[r, k] & 0x7F == 0x7E                     # the largest maps to 448
    # negating a row flips every sign bit (zeros keep +0 vs -0 from the input)
    c2, s2 = orc.quantize_rows_dynamic(_bf16_rows(-x))
    assert np.array_equal(s2, scales)
    nz = (codes & 0x7F) != 0
    assert np.array_equal(c2[nz] ^ 0x80, codes[nz])


def test_dynamic_quant_zero_row(orc):
    codes, scales = orc.quantize_rows_dynamic(_bf16_rows([[0.0] * 16, [1.0] + [0.0] * 15]))
    assert scales[0] == 1.0 and not codes[0].any()
    assert scales[1] == np.float32(1.0 / 448.0) and codes[1, 0] == 0x7E and not codes[1, 1:].any()


@pytest.mark.parametrize("act,dtype", [("relu", "f32"), ("swiglu", "bf16"), ("none", "e4m3")])
def test_dense_masked_reference_equals_sparse(orc, act, dtype):
    """SpMM page: the dense product over the (N,E) gate matrix equals the sparse
    top-K evaluation; also the sparse permute -> experts -> combine path."""
    if dtype == "e4m3":
        cfg = synth.MoEConfig("t8", "e4m3", 24, 32, 6, 2, 16, "none", routing="given")
        inp = synth.make_inputs(cfg, 3)
        ids = inp.ids.numpy()
        gates = np.full(ids.shape, 1.0)
        rng = np.random.default_rng(0)
        gates = rng.random(ids.shape)
    else:
        inp = _moe_tiny(act, dtype, N=30, d=24, E=6, K=3, F=20)
        ids, gates, _, _ = orc.router(inp.x, orc.DTYPE[dtype], inp.w_r, inp.bias, 3)
    cfg = inp.cfg
    dt = orc.DTYPE[dtype]
    N, K, E = cfg.N, cfg.K, cfg.E
    G = np.zeros((N, E))
    for t in range(N):
        for j in range(K):
            G[t, ids[t, j]] = gates[t, j]
    dense = orc.dense_masked(inp.x, dt, G, act, inp.w1, inp.w3, inp.w2, dt, inp.x_scale, inp.w_scale)
    counts, offsets, pos, src, xp = orc.permute(ids, E, inp.x)
    row_e = np.repeat(np.arange(E), counts).astype(np.int32)
    yp = orc.expert_rows(row_e, xp, dt, act, inp.w1, inp.w3, inp.w2, dt, inp.x_scale, inp.w_scale)
    sparse = orc.combine(pos, gates, yp, N, K)
    scale = np.abs(dense).max()
    assert np.abs(sparse - dense).max() <= 1e-12 * scale


def test_dense_masked_rank0_experts_is_spmm(orc):
    """Constant experts E_e(x) = B[e]: y = G @ B, the SpMM page's C = A @ B."""
    rng = np.random.default_rng(12)
    N, E, K, D = 40, 8, 2, 6
    L = rng.standard_normal((N, E))
    ids, gates, _ = orc.topk_from_logits(L, K)
    B = rng.standard_normal((E, D))
    counts, offsets, pos, _, _ = orc.permute(ids, E)
    yp = B[np.repeat(np.arange(E), counts)]
    y = orc.combine(pos, gates, yp, N, K)
    G = np.zeros((N, E))
    np.put_along_axis(G, ids.astype(np.int64), gates, 1)
    assert np.allclose(y, G @ B, rtol=0, atol=1e-13)
    assert np.allclose(orc.matmul(G, B), G @ B, rtol=0, atol=1e-13)
    # the binary expert-activation matrix has exactly K ones per row
    A = (G > 0).astype(np.float64)
    assert np.all(A.sum(1) == K)


def test_forward_tokens_equals_stagewise(orc):
    """Token-by-token layer == router -> permute -> experts -> combine."""
    inp = _moe_tiny("swiglu", "bf16", N=26, d=16, E=5, K=2, F=12, seed=9)
    y_tok, ids_t, g_t, m_t = orc.forward_tokens(inp, np.arange(26))
    ids, gates, margin, _ = orc.router(inp.x, orc.BF16, inp.w_r, inp.bias, 2)
    assert np.array_equal(ids, ids_t) and np.array_equal(gates, g_t) and np.array_equal(margin, m_t)
    counts, offsets, pos, src, xp = orc.permute(ids, 5, inp.x)
    yp = orc.expert_rows(np.repeat(np.arange(5), counts).astype(np.int32), xp, orc.BF16, "swiglu",
                         inp.w1, inp.w3, inp.w2, orc.BF16)
    y = orc.combine(pos, gates, yp, 26, 2)
    assert np.allclose(y, y_tok, rtol=0, atol=1e-13 * np.abs(y).max())


def test_oracle_deterministic(orc):
    inp = _moe_tiny("relu", "f32", N=40, d=16, E=4, K=2, F=8, seed=2)
    a = orc.forward_tokens(inp, np.arange(40))
    b = orc.forward_tokens(inp, np.arange(40))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_given_routing_distinct_and_uniform():
    ids = synth.given_routing(5, 4000, 16, 4)
    assert all(len(set(r)) == 4 for r in ids.tolist())
    c = np.bincount(ids.ravel(), minlength=16)
    assert c.min() > 0.8 * c.mean() and c.max() < 1.2 * c.mean()
    assert np.array_equal(ids, synth.given_routing(5, 4000, 16, 4))
