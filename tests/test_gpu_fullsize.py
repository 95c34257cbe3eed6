"""Full-size workloads on the GPU, in the launch configuration the benchmark
times (moe_forward for the routed layers; permute -> grouped matmul ->
unpermute plus the shared-expert matmul for the fp8 layer).

Routing, counts, offsets and the permutation are compared with the oracle in
full (bit-exact, near ties reported).  Float outputs are compared on sampled
rows that the oracle computes one by one: rows at expert-segment and 128-row
tile boundaries, the heaviest and lightest experts, and random rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL, check_routing, f64, make_plan, rel_err

pytestmark = pytest.mark.gpu


def setup_module(module):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def sample_rows(offsets: np.ndarray, R: int, n_random: int, seed: int) -> np.ndarray:
    """Rows of the permuted matrix worth checking: first/last row of each
    expert segment, the rows around 128-row tile edges of the largest
    segment, and random rows."""
    E = len(offsets) - 1
    counts = np.diff(offsets)
    rows = set()
    for e in range(E):
        if counts[e]:
            rows.update([offsets[e], offsets[e + 1] - 1])
    big = int(np.argmax(counts))
    for edge in range(offsets[big] + 127, offsets[big + 1], 128 * max(1, counts[big] // 1024)):
        rows.update([edge, min(edge + 1, offsets[big + 1] - 1)])
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, R, size=n_random).tolist())
    rows = np.array(sorted(r for r in rows if 0 <= r < R), np.int32)
    if len(rows) > 160:
        keep = rng.choice(len(rows), 160, replace=False)
        rows = np.sort(rows[keep])
    return rows


def run_routed_layer(cfg: synth.MoEConfig, n_tok_sample: int):
    inp = synth.make_inputs(cfg)
    plan, w = make_plan(inp)
    c = cfg
    R = c.N * c.K
    dt = oracle.DTYPE[c.dtype]
    x = inp.x.cuda()
    ws = plan.new_workspace()

    # routing, full
    ids = torch.empty(c.N, c.K, dtype=torch.int32, device="cuda")
    gates = torch.empty(c.N, c.K, dtype=torch.float32, device="cuda")
    plan.router_topk(x, ids, gates, ws)
    rid, rg, _, logits = oracle.router(inp.x, dt, inp.w_r, inp.bias, c.K, want_logits=True)
    ids_g = ids.cpu().numpy()
    ties, diff = check_routing(ids_g, gates.cpu().double().numpy(), logits, rid, rg)
    print(f"{c.name}: near-tie tokens {len(ties)}, ids differing {len(diff)}")

    # permutation of the GPU routing, full and bit-exact
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(R, c.d, dtype=x.dtype, device="cuda")
    plan.permute(x, ids, counts, offsets, pos, src, x_perm, ws)
    rc, ro, rp, rs, rx = oracle.permute(ids_g, c.E, inp.x)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(src.cpu().numpy(), rs)
    assert torch.equal(x_perm.cpu().view(torch.int16), torch.from_numpy(rx).view(torch.int16))
    print(f"{c.name}: empty experts {int((rc == 0).sum())}, largest {int(rc.max())}")

    # grouped FFN on sampled rows
    y_perm = torch.empty(R, c.d_out, dtype=x.dtype, device="cuda")
    plan.grouped_ffn(x_perm, offsets, y_perm, ws)
    assert plan.read_device_status(ws) == 0
    rows = sample_rows(ro, R, 48, 3)
    row_e = (np.searchsorted(ro, rows, side="right") - 1).astype(np.int32)
    ref = oracle.expert_rows(row_e, rx[rows], dt, c.act, inp.w1, inp.w3, inp.w2, dt)
    got = f64(y_perm[torch.from_numpy(rows).long().cuda()])
    assert rel_err(got, ref) <= TOL[c.dtype]

    # the whole layer (the benchmark's call), sampled tokens
    y = torch.empty(c.N, c.d_out, dtype=x.dtype, device="cuda")
    plan.forward(x, y, ws)
    assert plan.read_device_status(ws) == 0
    rng = np.random.default_rng(5)
    tok = np.unique(np.concatenate([[0, c.N - 1], rng.integers(0, c.N, n_tok_sample)]))
    tok = np.setdiff1d(tok, diff)
    yref, _, _, _ = oracle.forward_tokens(inp, tok)
    assert rel_err(f64(y[torch.from_numpy(tok).long().cuda()]), yref) <= TOL[c.dtype]
    # combine stage in full, fed the GPU's own y_perm
    yc = oracle.combine(rp, gates.cpu().double().numpy(), f64(y_perm), c.N, c.K)
    assert rel_err(f64(y), yc) <= 8e-3


def test_bf16_prefill_n4096_d2048_e8_k2_f8192():
    run_routed_layer(synth.BF16_PREFILL, 24)


def test_bf16_decode_n64_d4096_e64_k8_f1408():
    run_routed_layer(synth.BF16_DECODE, 24)


def test_bf16_finegrained_zipf_n16384_d2048_e128_k8_f768():
    run_routed_layer(synth.BF16_FINEGRAINED, 24)


def test_e4m3_gmm_unpermute_shared_n8192_h7168_e256_k8_n2048():
    cfg = synth.FP8_GMM
    inp = synth.make_inputs(cfg)
    plan, w = make_plan(inp)
    c = cfg
    R = c.N * c.K
    x = inp.x.cuda()
    ids_c = inp.ids.numpy()
    ws = plan.new_workspace()
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(R, c.d, dtype=torch.uint8, device="cuda")
    plan.permute(x, inp.ids.cuda(), counts, offsets, pos, src, x_perm, ws)
    rc, ro, rp, rs, rx = oracle.permute(ids_c, c.E, inp.x)
    assert np.array_equal(offsets.cpu().numpy(), ro) and np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(src.cpu().numpy(), rs)
    assert torch.equal(x_perm.cpu(), torch.from_numpy(rx))

    # grouped matmul, sampled rows
    y_perm = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn(x_perm, offsets, y_perm, ws, x_scale=inp.x_scale)
    assert plan.read_device_status(ws) == 0
    rows = sample_rows(ro, R, 48, 4)
    row_e = (np.searchsorted(ro, rows, side="right") - 1).astype(np.int32)
    ref = oracle.expert_rows(row_e, rx[rows], oracle.E4M3, "none", inp.w1, None, None, oracle.E4M3,
                             inp.x_scale, inp.w_scale)
    assert rel_err(f64(y_perm[torch.from_numpy(rows).long().cuda()]), ref) <= TOL["e4m3"]

    # unpermute of the GPU's gmmY: a pure reorder, exact, in full
    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.unpermute_combine(y_perm, pos, None, y, ws)
    yp = y_perm.cpu().view(torch.int16).numpy()
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), yp[rp])

    # the benchmark's call: permute -> grouped matmul -> unpermute
    y2 = torch.empty_like(y)
    plan.forward_routed(x, inp.ids.cuda(), None, y2, ws, x_scale=inp.x_scale)
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    tok = np.array([0, 1, 4095, c.N - 1])
    yref, _, _, _ = oracle.forward_tokens(inp, tok, gates_mode=0)
    rows_tok = (tok[:, None] * c.K + np.arange(c.K)).reshape(-1)
    assert rel_err(f64(y2[torch.from_numpy(rows_tok).long().cuda()]), yref) <= TOL["e4m3"]

    # shared expert, sampled rows
    H2, N2 = c.shared
    ysh = torch.empty(c.N, N2, dtype=torch.bfloat16, device="cuda")
    plan.shared_matmul(x, inp.w_sh.cuda(), inp.x_scale, inp.w_sh_scale, ysh)
    srows = np.array([0, 127, 128, 4000, c.N - 1])
    sref = oracle.expert_rows(np.zeros(len(srows), np.int32), inp.x.numpy()[srows], oracle.E4M3,
                              "none", inp.w_sh.reshape(1, N2, H2), None, None, oracle.E4M3,
                              inp.x_scale, inp.w_sh_scale)
    assert rel_err(f64(ysh[torch.from_numpy(srows).long().cuda()]), sref) <= TOL["e4m3"]


def test_e4m3_gmm_dynamic_per_token_quant_n8192_h7168_e256_k8_n2048():
    """The fp8 workload fed bf16 activations: per-token dynamic quantization
    fused into the permute (codes, scales and permutation bit-exact in full),
    then the grouped matmul with each row's token scale, unpermuted by its
    stores (sampled tokens against the oracle)."""
    cfg = synth.FP8_GMM
    inp = synth.make_inputs(cfg)
    plan, w = make_plan(inp)
    c = cfg
    R = c.N * c.K
    rng = np.random.default_rng(31)
    xb = torch.from_numpy(rng.standard_normal((c.N, c.d), dtype=np.float32)).to(torch.bfloat16)
    ws = plan.new_workspace()
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(R, c.d, dtype=torch.uint8, device="cuda")
    scales = torch.empty(c.N, dtype=torch.float32, device="cuda")
    plan.permute_quant(xb.cuda(), inp.ids.cuda(), counts, offsets, pos, src, x_perm, scales, ws)
    assert plan.read_device_status(ws) == 0
    codes, rscale = oracle.quantize_rows_dynamic(xb)
    rc, ro, rp, rs, rx = oracle.permute(inp.ids.numpy(), c.E, codes)
    assert np.array_equal(scales.cpu().numpy(), rscale)
    assert np.array_equal(pos.cpu().numpy(), rp) and np.array_equal(src.cpu().numpy(), rs)
    assert np.array_equal(x_perm.cpu().numpy(), rx)

    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_dynamic(xb.cuda(), inp.ids.cuda(), None, y, ws)
    assert plan.read_device_status(ws) == 0
    tok = np.array([0, 1, 4095, c.N - 1])
    ids = inp.ids.numpy()
    rows_tok = (tok[:, None] * c.K + np.arange(c.K)).reshape(-1)
    row_e = ids.reshape(-1)[rows_tok].astype(np.int32)
    ref = oracle.expert_rows_scaled(row_e, codes[np.repeat(tok, c.K)], oracle.E4M3, inp.w1,
                                    oracle.E4M3, x_scale=1.0,
                                    x_row_scales=rscale[np.repeat(tok, c.K)].astype(np.float64),
                                    w_scale=inp.w_scale)
    assert rel_err(f64(y[torch.from_numpy(rows_tok).long().cuda()]), ref) <= TOL["e4m3"]


def test_e4m3_mx_gmm_unpermute_n8192_h7168_e256_k8_n2048():
    """The grouped matmul with MX block scales (quant mode 6) at full size:
    permute and permuted scale rows bit-exact in full, the grouped matmul on
    sampled rows against the oracle, the fused call (unpermute by the GEMM's
    stores) equal to the stage composition bit for bit, sampled tokens of the
    fused result against the oracle."""
    import top_routing_grouped_gemv_b200 as moe
    c = synth.MX_GMM
    inp = synth.make_inputs(c)
    R = c.N * c.K
    w = {"w1": inp.w1.cuda(), "w_mx_scales": inp.w_sf.cuda()}
    plan = moe.Plan(c.N, c.d, c.E, c.K, c.F, "e4m3", "none", w)
    x, xsf, ids = inp.x.cuda(), inp.x_sf.cuda(), inp.ids.cuda()
    xs = inp.x_sf.numpy()
    ws = plan.new_workspace()
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, offsets = torch.empty(c.E, **i32), torch.empty(c.E + 1, **i32)
    pos, src = torch.empty(R, **i32), torch.empty(R, **i32)
    x_perm = torch.empty(R, c.d, dtype=torch.uint8, device="cuda")
    sf_perm = torch.empty(R, c.d // 32, dtype=torch.uint8, device="cuda")
    plan.permute_mx(x, xsf, ids, counts, offsets, pos, src, x_perm, sf_perm, ws)
    assert plan.read_device_status(ws) == 0
    rc, ro, rp, rs, rx = oracle.permute(inp.ids.numpy(), c.E, inp.x)
    assert np.array_equal(offsets.cpu().numpy(), ro) and np.array_equal(pos.cpu().numpy(), rp)
    assert torch.equal(x_perm.cpu(), torch.from_numpy(rx))
    assert np.array_equal(sf_perm.cpu().numpy(), xs[rs])

    y_perm = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn_mx(x_perm, sf_perm, offsets, y_perm, ws)
    assert plan.read_device_status(ws) == 0
    rows = sample_rows(ro, R, 48, 9)
    row_e = (np.searchsorted(ro, rows, side="right") - 1).astype(np.int32)
    ref = oracle.expert_rows_mx(row_e, rx[rows], xs[rs[rows]], inp.w1, inp.w_sf)
    assert rel_err(f64(y_perm[torch.from_numpy(rows).long().cuda()]), ref) <= 1e-2

    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_mx(x, xsf, ids, None, y, ws)
    assert plan.read_device_status(ws) == 0
    yp = y_perm.cpu().view(torch.int16).numpy()
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), yp[rp])
    tok = np.array([0, 1, 4095, c.N - 1])
    rows_tok = (tok[:, None] * c.K + np.arange(c.K)).reshape(-1)
    row_e = inp.ids.numpy().reshape(-1)[rows_tok].astype(np.int32)
    tr = np.repeat(tok, c.K)
    yref = oracle.expert_rows_mx(row_e, inp.x.numpy()[tr], xs[tr], inp.w1, inp.w_sf)
    assert rel_err(f64(y[torch.from_numpy(rows_tok).long().cuda()]), yref) <= 1e-2


def test_e4m3_block_scales_gmm_unpermute_n8192_h7168_e256_k8_n2048():
    """The grouped matmul with fp32 scales per 128 x 128 weight block and per
    token and 128-element group (quant mode 5) at full size: sampled rows of
    the stage call against the oracle, the fused call (unpermute by the
    GEMM's stores) equal to the stage composition bit for bit."""
    import top_routing_grouped_gemv_b200 as moe
    c = synth.BLOCK_GMM
    inp = synth.make_inputs(c)
    R = c.N * c.K
    w = {"w1": inp.w1.cuda(), "w_block_scales": inp.w_gs.cuda()}
    plan = moe.Plan(c.N, c.d, c.E, c.K, c.F, "e4m3", "none", w)
    ws = plan.new_workspace()
    xg = inp.x_gs.numpy()
    rc, ro, rp, rs, rx = oracle.permute(inp.ids.numpy(), c.E, inp.x)
    y_perm = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn_group_scales(torch.from_numpy(rx).cuda(), torch.from_numpy(ro).cuda(), y_perm,
                                  ws, x_group_scales=torch.from_numpy(xg[rs]).cuda())
    assert plan.read_device_status(ws) == 0
    rows = sample_rows(ro, R, 48, 13)
    row_e = (np.searchsorted(ro, rows, side="right") - 1).astype(np.int32)
    wfull = oracle.block_to_group_scales(inp.w_gs.numpy(), c.F)
    ref = oracle.expert_rows_kscaled(row_e, rx[rows], oracle.E4M3, inp.w1, oracle.E4M3, wfull,
                                     x_group_scales=xg[rs[rows]])
    assert rel_err(f64(y_perm[torch.from_numpy(rows).long().cuda()]), ref) <= 1e-2
    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_group_scales(inp.x.cuda(), inp.ids.cuda(), None, y, ws,
                                     x_group_scales=inp.x_gs.cuda())
    assert plan.read_device_status(ws) == 0
    yp = y_perm.cpu().view(torch.int16).numpy()
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), yp[rp])
