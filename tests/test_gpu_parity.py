"""GPU parity of every stage of the MoE layer forward against the fp64 oracle,
called through the C ABI (libmoe.so via the ctypes binding).

Bars: routing ids, counts, offsets, permutation and x_perm bit-exact (near-tie
tokens reported separately); floats within the normwise tolerance of their
dtype (fp32 1e-5, bf16 2e-2, fp8 6e-2).  Each stage is fed the same inputs as
the oracle stage it is compared with, so a routing near tie cannot hide an
FFN or combine error.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL, check_routing, f64, make_plan, rel_err

pytestmark = pytest.mark.gpu

SMALL = {
    "f32_relu_n256": synth.FP32_RELU,
    "f32_relu_ragged": synth.small_variant(synth.FP32_RELU, N=77, d=64, E=5, K=2, F=96),
    "f32_swiglu": synth.MoEConfig("f32_swiglu", "f32", 100, 128, 6, 3, 64, "swiglu"),
    "f32_none": synth.MoEConfig("f32_none", "f32", 50, 64, 4, 2, 40, "none"),
    "bf16_swiglu_ragged": synth.small_variant(synth.BF16_PREFILL, N=300, d=256, E=8, K=2, F=384),
    "bf16_swiglu_k4": synth.small_variant(synth.BF16_PREFILL, N=200, d=512, E=16, K=4, F=256),
    "bf16_decode": synth.small_variant(synth.BF16_DECODE, N=8, d=1024, E=64, K=8, F=256),
    "bf16_zipf": synth.small_variant(synth.BF16_FINEGRAINED, N=1000, d=256, E=64, K=8, F=128),
    "bf16_k1": synth.small_variant(synth.BF16_PREFILL, N=130, d=128, E=4, K=1, F=128),
    "bf16_f_not_tile": synth.small_variant(synth.BF16_PREFILL, N=160, d=192, E=3, K=2, F=200),
    # token rows not a whole number of 128-byte K blocks (partial K box)
    "bf16_d_not_kblock": synth.small_variant(synth.BF16_PREFILL, N=150, d=200, E=5, K=2, F=136),
    "e4m3_gmm": synth.small_variant(synth.FP8_GMM, N=256, d=512, E=16, K=4, F=512,
                                    shared=(512, 384)),
    "e4m3_gmm_ragged": synth.small_variant(synth.FP8_GMM, N=45, d=256, E=40, K=8, F=96,
                                           shared=(256, 136)),
    # > 32 experts with bf16 tokens: router logits on the tensor cores
    "bf16_tc_router_e64": synth.small_variant(synth.BF16_DECODE, N=200, d=512, E=64, K=8, F=128),
    "bf16_tc_router_e100_k3": synth.MoEConfig("tc_e100", "bf16", 333, 256, 100, 3, 128, "swiglu",
                                              zipf_bias=1.2),
    "bf16_tc_router_e256_k1": synth.MoEConfig("tc_e256", "bf16", 130, 128, 256, 1, 64, "swiglu"),
    # the fused router's expert splits: 33 experts (the upper half of the
    # 64-column tile holds one), 96 (48-expert halves, two MMAs of N = 192
    # and 96), 127 (one padding column); ragged token counts, K from 1 to 8
    "bf16_tc_router_e33_k2": synth.MoEConfig("tc_e33", "bf16", 300, 256, 33, 2, 64, "swiglu"),
    "bf16_tc_router_e96_k8": synth.MoEConfig("tc_e96", "bf16", 520, 384, 96, 8, 64, "swiglu",
                                             zipf_bias=1.2),
    "bf16_tc_router_e127_k1": synth.MoEConfig("tc_e127", "bf16", 777, 192, 127, 1, 64, "swiglu"),
    # few tokens with long rows: split-K router (partial logits per slice of d)
    "bf16_splitk_e8": synth.MoEConfig("sk_e8", "bf16", 40, 2048, 8, 2, 128, "swiglu"),
    "bf16_splitk_e256_k8": synth.MoEConfig("sk_e256", "bf16", 130, 1024, 256, 8, 64, "swiglu"),
    "bf16_splitk_e100_k3": synth.MoEConfig("sk_e100", "bf16", 33, 1536, 100, 3, 64, "swiglu",
                                           zipf_bias=1.2),
    "f32_splitk_e16": synth.MoEConfig("sk_f32", "f32", 50, 1024, 16, 4, 64, "relu"),
    # single-token batches (split-K router with one token; one row per expert tile)
    "bf16_n1": synth.MoEConfig("n1_bf16", "bf16", 1, 1024, 8, 2, 128, "swiglu"),
    "f32_n1": synth.MoEConfig("n1_f32", "f32", 1, 256, 4, 2, 64, "relu"),
    "e4m3_n1": synth.small_variant(synth.FP8_GMM, N=1, d=256, E=16, K=8, F=128,
                                   shared=(256, 64)),
    # the largest expert count with the largest K, on the tensor-core router
    "bf16_e256_k8": synth.MoEConfig("e256_k8", "bf16", 600, 256, 256, 8, 64, "swiglu",
                                    zipf_bias=1.2),
    # >= 512 routed rows per expert on average: 256-row tiles on CTA pairs
    "bf16_pair": synth.small_variant(synth.BF16_PREFILL, N=1024, d=256, E=4, K=2, F=384),
    "bf16_pair_ragged": synth.small_variant(synth.BF16_PREFILL, N=1300, d=320, E=4, K=2, F=200),
    "bf16_pair_zipf": synth.small_variant(synth.BF16_FINEGRAINED, N=2100, d=256, E=8, K=2, F=256),
    # >= 2048 rows per expert: the SwiGLU gate/up GEMM pairs as well
    "bf16_pair_swiglu": synth.MoEConfig("pair_sw", "bf16", 4100, 128, 2, 1, 256, "swiglu"),
    "e4m3_pair": synth.small_variant(synth.FP8_GMM, N=1100, d=256, E=4, K=2, F=392,
                                     shared=(256, 392)),
    # bf16, at most 16 experts: router on the warp-level MMA; rows not a whole
    # number of 32-element blocks, two expert tiles, a ragged 16-token group
    "bf16_mma_router_e13": synth.MoEConfig("mma_e13", "bf16", 333, 424, 13, 3, 64, "swiglu"),
    # enough 16-token groups for two per CTA (one and two expert tiles)
    "bf16_mma_router_g2_e8": synth.MoEConfig("mma_g2_e8", "bf16", 4801, 256, 8, 2, 64, "swiglu"),
    "bf16_mma_router_g2_e16": synth.MoEConfig("mma_g2_e16", "bf16", 4900, 160, 16, 4, 64,
                                              "swiglu", zipf_bias=1.2),
    # at most 16 routed rows per expert on average: the whole-layer call's
    # gate/up GEMM gathers its rows from x (tile::gather4), the permute copies
    # no rows; ragged row counts, and a skewed router that gives one expert
    # more than a full 128-row tile
    "bf16_decode_ragged": synth.MoEConfig("dec_rag", "bf16", 37, 520, 32, 4, 192, "swiglu"),
    "bf16_decode_zipf": synth.MoEConfig("dec_zipf", "bf16", 200, 256, 64, 4, 128, "swiglu",
                                        zipf_bias=1.2),
}

_cache = {}


def setup_module(module):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import top_routing_grouped_gemv_b200 as moe
    moe.build()
    moe.load()


def case(name):
    if name not in _cache:
        cfg = SMALL[name]
        inp = synth.make_inputs(cfg, seed=1234 + sum(map(ord, name)))
        plan, w = make_plan(inp)
        _cache[name] = (inp, plan, w)
    return _cache[name]


def ref_routing(inp):
    """Oracle routing: (ids, gates, logits) -- given ids for the fp8 workload."""
    if inp.ids is not None:
        ids = inp.ids.numpy()
        return ids, np.ones(ids.shape), None
    ids, gates, margin, logits = oracle.router(inp.x, oracle.DTYPE[inp.cfg.dtype], inp.w_r,
                                               inp.bias, inp.cfg.K, want_logits=True)
    return ids, gates, logits


ROUTED = [n for n in SMALL if SMALL[n].routing == "router"]


@pytest.mark.parametrize("name", ROUTED)
def test_router_parity(name):
    inp, plan, w = case(name)
    c = inp.cfg
    x = inp.x.cuda()
    ids = torch.empty(c.N, c.K, dtype=torch.int32, device="cuda")
    gates = torch.empty(c.N, c.K, dtype=torch.float32, device="cuda")
    margin = torch.empty(c.N, dtype=torch.float32, device="cuda")
    ws = plan.new_workspace()
    plan.router_topk(x, ids, gates, ws, margin)
    torch.cuda.synchronize()
    rid, rg, logits = ref_routing(inp)
    ties, diff = check_routing(ids.cpu().numpy(), gates.cpu().double().numpy(), logits, rid, rg)
    # margin: K-th minus (K+1)-th logit, fp32 logits vs fp64
    _, _, rmargin, _ = oracle.router(inp.x, oracle.DTYPE[c.dtype], inp.w_r, inp.bias, c.K)
    m = margin.cpu().double().numpy()
    if c.K == c.E:
        assert np.all(np.isinf(m))
    else:
        ok = np.setdiff1d(np.arange(c.N), diff)
        assert np.abs(m[ok] - rmargin[ok]).max() < 1e-4
    print(f"{name}: near-tie tokens {len(ties)}, differing ids {len(diff)}")


@pytest.mark.parametrize("name", list(SMALL))
def test_permute_parity(name):
    inp, plan, w = case(name)
    c = inp.cfg
    rid, _, _ = ref_routing(inp)
    ids = torch.from_numpy(np.ascontiguousarray(rid)).cuda()
    x = inp.x.cuda()
    R = c.N * c.K
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((R,) + tuple(inp.x.shape[1:]), dtype=inp.x.dtype, device="cuda")
    ws = plan.new_workspace()
    plan.permute(x, ids, counts, offsets, pos, src, x_perm, ws)
    assert plan.read_device_status(ws) == 0
    rc, ro, rp, rs, rx = oracle.permute(rid, c.E, inp.x)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(src.cpu().numpy(), rs)
    xp = x_perm.cpu()
    if xp.dtype == torch.bfloat16:
        xp = xp.view(torch.int16)
    assert np.array_equal(xp.numpy().view(np.uint8), np.ascontiguousarray(rx).view(np.uint8))


@pytest.mark.parametrize("name", list(SMALL))
def test_grouped_ffn_parity(name):
    inp, plan, w = case(name)
    c = inp.cfg
    rid, _, _ = ref_routing(inp)
    rc, ro, rp, rs, rx = oracle.permute(rid, c.E, inp.x)
    xp_cpu = torch.from_numpy(rx) if isinstance(rx, np.ndarray) else rx
    if c.dtype == "bf16":
        xp_cpu = torch.from_numpy(np.ascontiguousarray(rx)).view(torch.bfloat16)
    x_perm = xp_cpu.cuda()
    offsets = torch.from_numpy(ro).cuda()
    R = c.N * c.K
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    y_perm = torch.full((R, c.d_out), float("nan"), dtype=ydt, device="cuda")
    ws = plan.new_workspace()
    plan.grouped_ffn(x_perm, offsets, y_perm, ws, x_scale=inp.x_scale)
    assert plan.read_device_status(ws) == 0
    row_e = np.repeat(np.arange(c.E), rc).astype(np.int32)
    dt = oracle.DTYPE[c.dtype]
    ref = oracle.expert_rows(row_e, rx, dt, c.act, inp.w1, inp.w3, inp.w2, dt, inp.x_scale,
                             inp.w_scale)
    got = f64(y_perm)
    assert np.isfinite(got).all()
    err = rel_err(got, ref)
    assert err <= TOL[c.dtype], err


# Row counts per expert around the 256-row tile of the CTA-pair mode (each
# CTA of the pair holds 128 rows of a tile): last tiles holding 128, 129, 128
# (the whole expert) and 126 / 22 rows.
TAIL_COUNTS = [384, 385, 128, 1151]


@pytest.mark.parametrize("name", ["bf16_pair", "e4m3_pair"])
def test_pair_tile_tail_boundaries(name):
    inp, plan, w = case(name)
    c = inp.cfg
    R = c.N * c.K
    assert R >= 512 * c.E and c.E == len(TAIL_COUNTS)
    counts = np.array(TAIL_COUNTS, np.int64)
    counts[-1] += R - counts.sum() - 1        # one row short of R: m_total > offsets[E]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rng = np.random.default_rng(11)
    rows = rng.integers(0, c.N, R)            # any token rows as the permuted input
    xn = inp.x.numpy() if c.dtype == "e4m3" else inp.x.view(torch.int16).numpy()
    xp = np.ascontiguousarray(xn[rows])
    x_perm = torch.from_numpy(xp).cuda()
    if c.dtype == "bf16":
        x_perm = x_perm.view(torch.bfloat16)
    y_perm = torch.full((R, c.d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = plan.new_workspace()
    plan.grouped_ffn(x_perm, torch.from_numpy(offsets).cuda(), y_perm, ws, x_scale=inp.x_scale)
    assert plan.read_device_status(ws) == 0
    used = int(offsets[-1])
    row_e = np.repeat(np.arange(c.E), counts).astype(np.int32)
    dt = oracle.DTYPE[c.dtype]
    xsrc = inp.x.numpy()[rows[:used]] if c.dtype == "e4m3" else inp.x[torch.from_numpy(rows[:used])]
    ref = oracle.expert_rows(row_e, xsrc, dt, c.act, inp.w1, inp.w3, inp.w2, dt, inp.x_scale,
                             inp.w_scale)
    got = f64(y_perm)
    assert np.isnan(got[used:]).all()         # rows past offsets[E] are never stored
    for e in range(c.E):
        a, b = offsets[e], offsets[e + 1]
        assert rel_err(got[a:b], ref[a:b]) <= TOL[c.dtype], e


@pytest.mark.parametrize("name", list(SMALL))
def test_combine_parity(name):
    """Combine fed a synthetic y_perm of the layer's dtype and the oracle's
    pos/gates; compared with the oracle combine of the same values."""
    inp, plan, w = case(name)
    c = inp.cfg
    rid, rg, _ = ref_routing(inp)
    rc, ro, rp, rs, _ = oracle.permute(rid, c.E)
    R = c.N * c.K
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    yp = torch.from_numpy(synth.normal_f32(77, 9, R * c.d_out).reshape(R, c.d_out)).to(ydt)
    gated = c.act != "none"
    gates = torch.from_numpy(rg.astype(np.float32)) if gated else None
    rows = c.N if gated else R
    y = torch.empty(rows, c.d_out, dtype=ydt, device="cuda")
    ws = plan.new_workspace()
    plan.unpermute_combine(yp.cuda(), torch.from_numpy(rp).cuda(),
                           gates.cuda() if gated else None, y, ws)
    assert plan.read_device_status(ws) == 0
    ref = oracle.combine(rp, gates.double().numpy() if gated else None, yp.double().numpy(), c.N,
                         c.K)
    got = f64(y)
    if gated:
        # one fp32 accumulation in slot order, one rounding to the output dtype
        assert rel_err(got, ref) <= (1e-6 if c.dtype == "f32" else 8e-3)
    else:
        assert np.array_equal(got, ref)  # pure reorder: exact


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_end_to_end(name):
    inp, plan, w = case(name)
    c = inp.cfg
    x = inp.x.cuda()
    ws = plan.new_workspace()
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    if c.routing == "router":
        y = torch.empty(c.N, c.d_out, dtype=ydt, device="cuda")
        plan.forward(x, y, ws)
        gate_mode = 1
    else:
        y = torch.empty(c.N * c.K, c.d_out, dtype=ydt, device="cuda")
        plan.forward_routed(x, inp.ids.cuda(), None, y, ws, x_scale=inp.x_scale)
        gate_mode = 0
    assert plan.read_device_status(ws) == 0
    # router, rank (+ scan), gather, GEMM(s), combine -- the pure unpermute of
    # the routed single-matrix layer is done by its GEMM's stores
    assert plan.last_launch_count() >= (5 if c.routing == "router" else 3)
    ref, rids, _, _ = oracle.forward_tokens(inp, np.arange(c.N), gates_mode=gate_mode)
    got = f64(y)
    if c.routing == "router":
        # exclude near-tie tokens whose routing differs (their y is a different sum)
        ids = torch.empty(c.N, c.K, dtype=torch.int32, device="cuda")
        gates = torch.empty(c.N, c.K, dtype=torch.float32, device="cuda")
        plan.router_topk(x, ids, gates, ws)
        rid, rg, logits = ref_routing(inp)
        ties, diff = check_routing(ids.cpu().numpy(), gates.cpu().double().numpy(), logits, rid, rg)
        keep = np.setdiff1d(np.arange(c.N), diff)
        assert len(keep) >= 0.9 * c.N
        err = rel_err(got[keep], ref[keep])
    else:
        err = rel_err(got, ref)
    assert err <= TOL[c.dtype], err


@pytest.mark.parametrize("name", ["bf16_zipf", "f32_relu_n256", "e4m3_gmm", "bf16_pair_ragged"])
def test_forward_deterministic(name):
    inp, plan, w = case(name)
    c = inp.cfg
    x = inp.x.cuda()
    ws = plan.new_workspace()
    outs = []
    for _ in range(3):
        if c.routing == "router":
            y = torch.empty(c.N, c.d_out, dtype=torch.float32 if c.dtype == "f32" else torch.bfloat16,
                            device="cuda")
            plan.forward(x, y, ws)
        else:
            y = torch.empty(c.N * c.K, c.d_out, dtype=torch.bfloat16, device="cuda")
            plan.forward_routed(x, inp.ids.cuda(), None, y, ws, x_scale=inp.x_scale)
        torch.cuda.synchronize()
        outs.append(y.cpu().view(torch.uint8 if y.dtype == torch.float32 else torch.int16).clone())
    assert all(torch.equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("name", ["e4m3_gmm", "e4m3_gmm_ragged", "e4m3_pair"])
def test_shared_expert_matmul(name):
    inp, plan, w = case(name)
    c = inp.cfg
    H2, N2 = c.shared
    x = inp.x.cuda()
    wsh = inp.w_sh.cuda()
    y = torch.empty(c.N, N2, dtype=torch.bfloat16, device="cuda")
    plan.shared_matmul(x, wsh, inp.x_scale, inp.w_sh_scale, y)
    torch.cuda.synchronize()
    ref = oracle.expert_rows(np.zeros(c.N, np.int32), inp.x, oracle.E4M3, "none",
                             inp.w_sh.reshape(1, N2, H2), None, None, oracle.E4M3, inp.x_scale,
                             inp.w_sh_scale)
    assert rel_err(f64(y), ref) <= TOL["e4m3"]


@pytest.mark.parametrize("name", ["bf16_swiglu_ragged", "bf16_pair", "f32_relu_n256"])
def test_forward_host_matches_device(name):
    """moe_forward_host (token chunks with copies overlapping compute when the
    experts are large enough) gives the bytes of moe_forward."""
    inp, plan, w = case(name)
    c = inp.cfg
    ws = plan.new_workspace()
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    y_dev = torch.empty(c.N, c.d_out, dtype=ydt, device="cuda")
    plan.forward(inp.x.cuda(), y_dev, ws)
    x_host = inp.x.clone().pin_memory()
    y_host = torch.full((c.N, c.d_out), float("nan"), dtype=ydt).pin_memory()
    plan.forward_host(x_host, y_host, ws)
    assert plan.read_device_status(ws) == 0
    assert torch.equal(y_host.view(torch.uint8), y_dev.cpu().view(torch.uint8))


def test_forward_host_async_stream_of_batches():
    """Three batches through moe_forward_host_async (alternating staging
    slots, copies on the plan's streams) equal moe_forward of each batch."""
    inp, plan, w = case("bf16_pair")
    c = inp.cfg
    ws = plan.new_workspace()
    xs = [inp.x.clone(), (inp.x.float() * -0.5).to(torch.bfloat16), inp.x.flip(0).contiguous()]
    ref = []
    for x in xs:
        y = torch.empty(c.N, c.d, dtype=torch.bfloat16, device="cuda")
        plan.forward(x.cuda(), y, ws)
        ref.append(y.cpu())
    xh = [x.pin_memory() for x in xs]
    yh = [torch.empty(c.N, c.d, dtype=torch.bfloat16).pin_memory() for _ in xs]
    for x, y in zip(xh, yh):
        plan.forward_host_async(x, y, ws)
    plan.host_join()
    torch.cuda.synchronize()
    assert plan.read_device_status(ws) == 0
    for y, r in zip(yh, ref):
        assert torch.equal(y.view(torch.int16), r.view(torch.int16))


def test_bad_expert_ids_set_device_status():
    inp, plan, w = case("bf16_k1")
    c = inp.cfg
    ids = torch.zeros(c.N, c.K, dtype=torch.int32)
    ids[5, 0] = c.E        # out of range
    ids[7, 0] = -3
    R = c.N * c.K
    ws = plan.new_workspace()
    out = [torch.empty(c.E, dtype=torch.int32, device="cuda"),
           torch.empty(c.E + 1, dtype=torch.int32, device="cuda"),
           torch.empty(R, dtype=torch.int32, device="cuda"),
           torch.empty(R, dtype=torch.int32, device="cuda"),
           torch.empty(R, c.d, dtype=torch.bfloat16, device="cuda")]
    plan.permute(inp.x.cuda(), ids.cuda(), *out, ws)
    import top_routing_grouped_gemv_b200 as moe
    assert plan.read_device_status(ws) == 5
    assert plan.read_device_status(ws) == 0          # read clears it
    assert out[2].cpu()[5].item() == -1              # skipped, not written elsewhere
    assert int(out[1].cpu()[c.E]) == R - 2


def test_workspace_too_small_and_misaligned():
    import top_routing_grouped_gemv_b200 as moe
    inp, plan, w = case("bf16_k1")
    c = inp.cfg
    ws = plan.new_workspace()
    small = ws[: 1024]
    y = torch.empty(c.N, c.d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        plan.forward(inp.x.cuda(), y, small)
    assert e.value.code == 3
    with pytest.raises(moe.MoEError) as e:
        plan.forward(inp.x.cuda(), y, ws[16:])
    assert e.value.code == 1


TC_CASES = [n for n in SMALL if SMALL[n].dtype != "f32"]


@pytest.mark.parametrize("name", TC_CASES)
def test_fused_forward_matches_stage_composition(name):
    """The whole-layer calls keep their intermediates in the workspace (and,
    for the single-matrix layer without gates, the GEMM stores its rows
    straight to their unpermuted place); the stage calls take caller buffers.
    Same operands, same MMA order: the results agree bit for bit."""
    inp, plan, w = case(name)
    c = inp.cfg
    x = inp.x.cuda()
    ws = plan.new_workspace()
    R = c.N * c.K
    ydt = torch.bfloat16
    if c.routing == "router":
        ids = torch.empty(c.N, c.K, dtype=torch.int32, device="cuda")
        gates = torch.empty(c.N, c.K, dtype=torch.float32, device="cuda")
        plan.router_topk(x, ids, gates, ws)
        y_fused = torch.empty(c.N, c.d_out, dtype=ydt, device="cuda")
        plan.forward(x, y_fused, ws)
    else:
        ids = inp.ids.cuda()
        gates = None
        y_fused = torch.full((R, c.d_out), float("nan"), dtype=ydt, device="cuda")
        plan.forward_routed(x, ids, None, y_fused, ws, x_scale=inp.x_scale)
    assert plan.read_device_status(ws) == 0
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((R,) + tuple(x.shape[1:]), dtype=x.dtype, device="cuda")
    y_perm = torch.empty(R, c.d_out, dtype=ydt, device="cuda")
    plan.permute(x, ids, counts, offsets, pos, src, x_perm, ws)
    plan.grouped_ffn(x_perm, offsets, y_perm, ws, x_scale=inp.x_scale)
    y_stage = torch.empty_like(y_fused)
    plan.unpermute_combine(y_perm, pos, gates, y_stage, ws)
    assert plan.read_device_status(ws) == 0
    assert torch.equal(y_fused.view(torch.int16), y_stage.view(torch.int16))


@pytest.mark.parametrize("name", ["e4m3_gmm", "e4m3_pair"])
def test_fused_routed_with_gates_and_token_scales(name):
    """Single-matrix layer with gates (combine as its own pass) and
    per-token activation scales read through the source-token index."""
    inp, plan, w = case(name)
    c = inp.cfg
    ws = plan.new_workspace()
    rng = np.random.default_rng(7)
    ids = inp.ids.numpy()
    g = rng.random((c.N, c.K)).astype(np.float32)
    xs = (inp.x_scale * rng.uniform(0.5, 2.0, c.N)).astype(np.float32)
    y = torch.empty(c.N, c.d_out, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed(inp.x.cuda(), inp.ids.cuda(), torch.from_numpy(g).cuda(), y, ws,
                        x_scale=1.0, x_token_scales=torch.from_numpy(xs).cuda())
    assert plan.read_device_status(ws) == 0
    # oracle: per-row scales of the permuted rows, then the gated combine
    _, _, rp, rs, rx = oracle.permute(ids, c.E, inp.x)
    row_e = np.repeat(np.arange(c.E, dtype=np.int32), np.bincount(ids.ravel(), minlength=c.E))
    yp = oracle.expert_rows_scaled(row_e, rx, oracle.E4M3, inp.w1, oracle.E4M3, x_scale=1.0,
                                   x_row_scales=xs[rs].astype(np.float64), w_scale=inp.w_scale)
    ref = oracle.combine(rp, g.astype(np.float64), yp, c.N, c.K)
    assert rel_err(f64(y), ref) <= TOL["e4m3"]


@pytest.mark.parametrize("name", ["e4m3_gmm", "e4m3_pair"])
@pytest.mark.parametrize("gated", [False, True])
def test_forward_routed_shared_matches_separate_calls(name, gated):
    """Routed layer and shared expert on forked streams: both outputs equal
    the separate calls on one stream bit for bit."""
    inp, plan, w = case(name)
    c = inp.cfg
    H2, N2 = c.shared
    x, ids, wsh = inp.x.cuda(), inp.ids.cuda(), inp.w_sh.cuda()
    g = None
    rows = c.N * c.K
    if gated:
        g = torch.from_numpy(np.random.default_rng(4).random((c.N, c.K)).astype(np.float32)).cuda()
        rows = c.N
    ws = plan.new_workspace()
    y1 = torch.empty(rows, c.d_out, dtype=torch.bfloat16, device="cuda")
    s1 = torch.empty(c.N, N2, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed(x, ids, g, y1, ws, x_scale=inp.x_scale)
    plan.shared_matmul(x, wsh, inp.x_scale, inp.w_sh_scale, s1)
    y2 = torch.empty_like(y1)
    s2 = torch.empty_like(s1)
    plan.forward_routed_shared(x, ids, g, y2, wsh, inp.w_sh_scale, s2, ws, x_scale=inp.x_scale)
    assert plan.read_device_status(ws) == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(s1.view(torch.int16), s2.view(torch.int16))


def _dyn_input(c, seed):
    """bf16 activations for a dynamic-quantization case: rows of widely
    different magnitudes and one all-zero row."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((c.N, c.d)) * np.exp(rng.uniform(-4, 4, (c.N, 1)))
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xb[min(1, c.N - 1)] = 0
    return xb


DYN = ["e4m3_gmm", "e4m3_gmm_ragged", "e4m3_pair"]


@pytest.mark.parametrize("name", DYN)
def test_permute_quant_bit_exact(name):
    """Per-token dynamic quantization fused into the permute: codes, scales
    and the permutation bit-exact against the oracle (the codes are fp32
    decisions on both sides)."""
    inp, plan, w = case(name)
    c = inp.cfg
    xb = _dyn_input(c, 21)
    R = c.N * c.K
    counts = torch.empty(c.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(R, dtype=torch.int32, device="cuda")
    src = torch.empty(R, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(R, c.d, dtype=torch.uint8, device="cuda")
    scales = torch.empty(c.N, dtype=torch.float32, device="cuda")
    ws = plan.new_workspace()
    plan.permute_quant(xb.cuda(), inp.ids.cuda(), counts, offsets, pos, src, x_perm, scales, ws)
    assert plan.read_device_status(ws) == 0
    codes, rscale = oracle.quantize_rows_dynamic(xb)
    rc, ro, rp, rs, rx = oracle.permute(inp.ids.numpy(), c.E, codes)
    assert np.array_equal(scales.cpu().numpy(), rscale)
    assert np.array_equal(counts.cpu().numpy(), rc) and np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(pos.cpu().numpy(), rp) and np.array_equal(src.cpu().numpy(), rs)
    assert np.array_equal(x_perm.cpu().numpy(), rx)


@pytest.mark.parametrize("name", DYN)
@pytest.mark.parametrize("gated", [False, True])
def test_forward_routed_dynamic(name, gated):
    inp, plan, w = case(name)
    c = inp.cfg
    xb = _dyn_input(c, 22)
    ws = plan.new_workspace()
    ids = inp.ids.numpy()
    g = None
    if gated:
        g = np.random.default_rng(9).random((c.N, c.K)).astype(np.float32)
        y = torch.empty(c.N, c.d_out, dtype=torch.bfloat16, device="cuda")
    else:
        y = torch.full((c.N * c.K, c.d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_dynamic(xb.cuda(), inp.ids.cuda(),
                                None if g is None else torch.from_numpy(g).cuda(), y, ws)
    assert plan.read_device_status(ws) == 0
    codes, rscale = oracle.quantize_rows_dynamic(xb)
    _, _, rp, rs, rx = oracle.permute(ids, c.E, codes)
    row_e = np.repeat(np.arange(c.E, dtype=np.int32), np.bincount(ids.ravel(), minlength=c.E))
    yp = oracle.expert_rows_scaled(row_e, rx, oracle.E4M3, inp.w1, oracle.E4M3, x_scale=1.0,
                                   x_row_scales=rscale[rs].astype(np.float64),
                                   w_scale=inp.w_scale)
    ref = oracle.combine(rp, None if g is None else g.astype(np.float64), yp, c.N, c.K)
    assert rel_err(f64(y), ref) <= TOL["e4m3"]


def test_stage_profile_names():
    inp, plan, w = case("bf16_swiglu_ragged")
    c = inp.cfg
    ws = plan.new_workspace()
    y = torch.empty(c.N, c.d, dtype=torch.bfloat16, device="cuda")
    plan.profile(True)
    plan.forward(inp.x.cuda(), y, ws)
    prof = plan.profile_read()
    plan.profile(False)
    names = [n for n, _ in prof]
    assert names == ["router_mma", "permute_rank", "permute_gather", "ffn1_swiglu_tc",
                     "ffn2_tc", "combine"]
    assert all(ms >= 0 for _, ms in prof)
    assert plan.last_launch_count() == 6


def test_bounded_wait_timeout_sets_status_and_context_survives():
    """A wait on a barrier that nothing arrives at gives up after its limit,
    records MOE_ERR_DEVICE_TIMEOUT and the other waiter leaves through the
    abort flag; the context keeps working afterwards."""
    import time
    import top_routing_grouped_gemv_b200 as moe
    inp, plan, w = case("bf16_k1")
    c = inp.cfg
    ws = plan.new_workspace()
    order = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.selftest_wait_timeout(ws, 20_000, order)          # 20 ms limit
    assert plan.read_device_status(ws) == 6               # MOE_ERR_DEVICE_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 0.9                          # gave up near its own limit
    assert sorted(order.cpu().tolist()) == [0, 1]         # both waiters left
    assert plan.read_device_status(ws) == 0               # cleared by the read
    y = torch.empty(c.N, c.d, dtype=torch.bfloat16, device="cuda")
    plan.forward(inp.x.cuda(), y, ws)                     # the context still works
    assert plan.read_device_status(ws) == 0
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("N,d,E,K,F", [(300, 256, 8, 4, 384), (1100, 256, 4, 2, 392)])
def test_e4m3_per_channel_weights_per_token_activations(N, d, E, K, F):
    """Ascend quant modes 2 (weights, one scale per expert output channel) and
    3 (activations, one scale per token) on the grouped matmul, the routed
    layer (scales follow each token to its K permuted rows) and the shared
    expert; the second shape runs on CTA pairs."""
    import synth as sy
    xq, xs = sy.quantize_e4m3_rows(sy.normal_f32(31, 1, N * d).reshape(N, d))
    wq, wsc = sy.quantize_e4m3_rows(sy.normal_f32(31, 2, E * F * d).reshape(E * F, d))
    wq, wsc = wq.reshape(E, F, d), wsc.reshape(E, F)
    ids = sy.given_routing(31, N, E, K)
    import top_routing_grouped_gemv_b200 as moe
    w = {"w1": torch.from_numpy(wq).cuda(), "w_channel_scales": torch.from_numpy(wsc).cuda()}
    plan = moe.Plan(N, d, E, K, F, "e4m3", "none", w)
    ws = plan.new_workspace()
    R = N * K
    y = torch.empty(R, F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed(torch.from_numpy(xq).cuda(), torch.from_numpy(ids).cuda(), None, y, ws,
                        x_token_scales=torch.from_numpy(xs).cuda())
    assert plan.read_device_status(ws) == 0
    rows_tok = np.repeat(np.arange(N), K)
    ref = oracle.expert_rows_scaled(ids.reshape(-1), xq[rows_tok], oracle.E4M3, wq, oracle.E4M3,
                                    x_row_scales=xs[rows_tok].astype(np.float64),
                                    w_channel_scales=wsc.astype(np.float64))
    assert rel_err(f64(y), ref) <= TOL["e4m3"]
    # the grouped-matmul stage with per-row scales of the permuted rows
    rc, ro, rp, rs, rx = oracle.permute(ids, E, xq)
    yp = torch.empty(R, F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn(torch.from_numpy(rx).cuda(), torch.from_numpy(ro).cuda(), yp, ws,
                     x_row_scales=torch.from_numpy(xs[rs]).cuda())
    ref_p = oracle.expert_rows_scaled(np.repeat(np.arange(E), rc).astype(np.int32), rx, oracle.E4M3,
                                      wq, oracle.E4M3, x_row_scales=xs[rs].astype(np.float64),
                                      w_channel_scales=wsc.astype(np.float64))
    assert rel_err(f64(yp), ref_p) <= TOL["e4m3"]
    # shared expert with both finer scales
    shq, shs = sy.quantize_e4m3_rows(sy.normal_f32(31, 3, 136 * d).reshape(136, d))
    ysh = torch.empty(N, 136, dtype=torch.bfloat16, device="cuda")
    plan.shared_matmul(torch.from_numpy(xq).cuda(), torch.from_numpy(shq).cuda(), 1.0, 1.0, ysh,
                       x_token_scales=torch.from_numpy(xs).cuda(),
                       w_channel_scales=torch.from_numpy(shs).cuda())
    ref_s = oracle.expert_rows_scaled(np.zeros(N, np.int32), xq, oracle.E4M3, shq.reshape(1, 136, d),
                                      oracle.E4M3, x_row_scales=xs.astype(np.float64),
                                      w_channel_scales=shs.astype(np.float64).reshape(1, 136))
    assert rel_err(f64(ysh), ref_s) <= TOL["e4m3"]


@pytest.mark.parametrize("name", ["bf16_swiglu_ragged", "bf16_zipf", "bf16_pair", "f32_relu_ragged"])
def test_expert_parallel_stages_single_rank_equal_forward(name):
    """The expert-parallel layer's GPU stages (a routing-only plan over all
    experts, a K = 1 plan of the local experts on a variable row count) at
    world size 1 reproduce moe_forward bit for bit."""
    from top_routing_grouped_gemv_b200.ep import ExpertParallelMoE, LibraryStages
    inp, plan, w = case(name)
    c = inp.cfg
    x = inp.x.cuda()
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    y_ref = torch.empty(c.N, c.d, dtype=ydt, device="cuda")
    ws = plan.new_workspace()
    plan.forward(x, y_ref, ws)
    stages = LibraryStages(c.N, c.d, c.E, c.K, c.F, c.dtype, c.act, 1, w["w_r"], w["w1"],
                           w.get("w3"), w.get("w2"), bias=w.get("bias"))
    y = ExpertParallelMoE(stages, c.E, c.K).forward(x)
    assert stages.check() == 0
    assert torch.equal(y.view(torch.int32 if c.dtype == "f32" else torch.int16),
                       y_ref.view(torch.int32 if c.dtype == "f32" else torch.int16))


# ---------------------------------------------------------------- MX (quant mode 6)

MX = {
    # two K stages, two column tiles (the second ragged), ~75 rows per expert
    "mx_small": synth.MoEConfig("mx_small", "e4m3", 300, 256, 8, 2, 384, "none",
                                routing="given", quant="mx"),
    # K = 160: one full 128-element stage and a 32-element tail; ragged rows
    "mx_ragged": synth.MoEConfig("mx_ragged", "e4m3", 257, 160, 5, 3, 200, "none",
                                 routing="given", quant="mx"),
    # many small experts (K = 8 of 64, ~16 rows each), several row tiles
    "mx_fine": synth.MoEConfig("mx_fine", "e4m3", 128, 512, 64, 8, 256, "none",
                               routing="given", quant="mx"),
    # empty experts, single-row groups
    "mx_sparse": synth.MoEConfig("mx_sparse", "e4m3", 20, 128, 16, 1, 64, "none",
                                 routing="given", quant="mx"),
    # an expert with more than one 128-row tile (500 rows over 2 experts)
    "mx_tall": synth.MoEConfig("mx_tall", "e4m3", 500, 384, 2, 1, 512, "none",
                               routing="given", quant="mx"),
}
_mx_cache = {}


def mx_case(name, wide=True):
    """Inputs of an MX case; wide=True replaces the quantiser's scales (which
    are nearly equal for N(0,1) data) by independent random E8M0 codes in
    [117, 137] for every block of x and W, so that any misplaced scale shows."""
    key = (name, wide)
    if key not in _mx_cache:
        import top_routing_grouped_gemv_b200 as moe
        c = MX[name]
        inp = synth.make_inputs(c, 31 + sum(map(ord, name)))
        xs, ws = inp.x_sf.numpy(), inp.w_sf.numpy()
        if wide:
            rng = np.random.default_rng(sum(map(ord, name)))
            xs = rng.integers(117, 138, size=xs.shape).astype(np.uint8)
            ws = rng.integers(117, 138, size=ws.shape).astype(np.uint8)
        w = {"w1": inp.w1.cuda(), "w_mx_scales": torch.from_numpy(ws).cuda()}
        plan = moe.Plan(c.N, c.d, c.E, c.K, c.F, "e4m3", "none", w)
        _mx_cache[key] = (inp, plan, w, xs, ws)
    return _mx_cache[key]


def mx_ref(inp, xs, ws, gates):
    """Oracle: permute, MX experts on the permuted rows, unpermute/combine."""
    c = inp.cfg
    ids = inp.ids.numpy()
    _, _, rp, rs, rx = oracle.permute(ids, c.E, inp.x.numpy())
    row_e = np.repeat(np.arange(c.E, dtype=np.int32), np.bincount(ids.ravel(), minlength=c.E))
    yp = oracle.expert_rows_mx(row_e, rx, xs[rs], inp.w1, ws)
    return oracle.combine(rp, gates, yp, c.N, c.K), yp


@pytest.mark.parametrize("name", list(MX))
@pytest.mark.parametrize("gated", [False, True])
def test_forward_routed_mx(name, gated):
    inp, plan, w, xs, ws = mx_case(name)
    c = inp.cfg
    wsp = plan.new_workspace()
    g = None
    if gated:
        g = np.random.default_rng(3).random((c.N, c.K)).astype(np.float32)
        y = torch.empty(c.N, c.F, dtype=torch.bfloat16, device="cuda")
    else:
        y = torch.full((c.N * c.K, c.F), float("nan"), dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_mx(inp.x.cuda(), torch.from_numpy(xs).cuda(), inp.ids.cuda(),
                           None if g is None else torch.from_numpy(g).cuda(), y, wsp)
    assert plan.read_device_status(wsp) == 0
    ref, _ = mx_ref(inp, xs, ws, None if g is None else g.astype(np.float64))
    err = rel_err(f64(y), ref)
    assert err <= TOL["e4m3"], err
    # fp32 accumulation of exact e4m3 x E8M0 products, one bf16 rounding: far
    # inside the fp8 bar; a misplaced scale (a factor 2^1..2^20) is not
    assert err <= 1e-2, err


@pytest.mark.parametrize("name", ["mx_small", "mx_ragged", "mx_sparse"])
def test_mx_stage_calls_and_fused_path_agree(name):
    """moe_permute_mx (codes and scale rows bit-exact), moe_grouped_ffn_mx
    (against the oracle), and the fused call's unpermuted rows equal to the
    stage composition bit for bit."""
    inp, plan, w, xs, ws = mx_case(name)
    c = inp.cfg
    R = c.N * c.K
    wsp = plan.new_workspace()
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, offsets = torch.empty(c.E, **i32), torch.empty(c.E + 1, **i32)
    pos, src = torch.empty(R, **i32), torch.empty(R, **i32)
    x_perm = torch.empty(R, c.d, dtype=torch.uint8, device="cuda")
    sf_perm = torch.empty(R, c.d // 32, dtype=torch.uint8, device="cuda")
    plan.permute_mx(inp.x.cuda(), torch.from_numpy(xs).cuda(), inp.ids.cuda(), counts, offsets,
                    pos, src, x_perm, sf_perm, wsp)
    assert plan.read_device_status(wsp) == 0
    _, ro, rp, rs, rx = oracle.permute(inp.ids.numpy(), c.E, inp.x.numpy())
    assert np.array_equal(offsets.cpu().numpy(), ro) and np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(x_perm.cpu().numpy(), rx)
    assert np.array_equal(sf_perm.cpu().numpy(), xs[rs])
    y_perm = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn_mx(x_perm, sf_perm, offsets, y_perm, wsp)
    assert plan.read_device_status(wsp) == 0
    _, yp_ref = mx_ref(inp, xs, ws, None)
    assert rel_err(f64(y_perm), yp_ref) <= 1e-2
    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_mx(inp.x.cuda(), torch.from_numpy(xs).cuda(), inp.ids.cuda(), None, y, wsp)
    yp = y_perm.cpu().view(torch.int16).numpy()
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), yp[rp])


def test_mx_with_quantiser_scales():
    """The same path on the MX quantiser's own scales (OCP MXFP8 of N(0,1))."""
    inp, plan, w, xs, ws = mx_case("mx_small", wide=False)
    c = inp.cfg
    wsp = plan.new_workspace()
    y = torch.empty(c.N * c.K, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_mx(inp.x.cuda(), torch.from_numpy(xs).cuda(), inp.ids.cuda(), None, y, wsp)
    assert plan.read_device_status(wsp) == 0
    ref, _ = mx_ref(inp, xs, ws, None)
    assert rel_err(f64(y), ref) <= 1e-2


def test_mx_and_per_tensor_calls_are_not_mixed():
    import top_routing_grouped_gemv_b200 as moe
    inp, plan, w, xs, ws = mx_case("mx_sparse")
    c = inp.cfg
    wsp = plan.new_workspace()
    y = torch.empty(c.N * c.K, c.F, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        plan.forward_routed(inp.x.cuda(), inp.ids.cuda(), None, y, wsp)
    assert e.value.code == 2
    inp8, plan8, _ = case("e4m3_gmm")
    ws8 = plan8.new_workspace()
    y8 = torch.empty(inp8.cfg.N * inp8.cfg.K, inp8.cfg.F, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        plan8.forward_routed_mx(inp8.x.cuda(), torch.zeros(inp8.cfg.N, inp8.cfg.d // 32,
                                                           dtype=torch.uint8, device="cuda"),
                                inp8.ids.cuda(), None, y8, ws8)
    assert e.value.code == 2


# ------------------------------------------------- group / block scales (quant modes 4, 5)

GS = {
    # two 128-element groups, two column tiles (the second ragged)
    "gs_small": synth.MoEConfig("gs_small", "e4m3", 300, 256, 8, 2, 384, "none", routing="given"),
    # many small experts, four groups
    "gs_fine": synth.MoEConfig("gs_fine", "e4m3", 128, 512, 64, 8, 256, "none", routing="given"),
    # empty experts, one group, F below one 128-channel block
    "gs_sparse": synth.MoEConfig("gs_sparse", "e4m3", 20, 128, 16, 1, 72, "none", routing="given"),
    # an expert with several 128-row tiles, three groups
    "gs_tall": synth.MoEConfig("gs_tall", "e4m3", 500, 384, 2, 1, 512, "none", routing="given"),
}
_gs_cache = {}


def gs_case(name, quant):
    """Inputs of a group/block case with independent random fp32 scales in
    [0.25, 4) per weight group (or block) and per token and group."""
    key = (name, quant)
    if key not in _gs_cache:
        import top_routing_grouped_gemv_b200 as moe
        c = GS[name].scaled(quant=quant)
        inp = synth.make_inputs(c, 77 + sum(map(ord, name)))
        rng = np.random.default_rng(sum(map(ord, name)) + (0 if quant == "group" else 1))
        G = c.d // 128
        wshape = (c.E, c.F, G) if quant == "group" else (c.E, (c.F + 127) // 128, G)
        ws = rng.uniform(0.25, 4.0, size=wshape).astype(np.float32)
        xs = rng.uniform(0.25, 4.0, size=(c.N, G)).astype(np.float32)
        wkey = "w_group_scales" if quant == "group" else "w_block_scales"
        w = {"w1": inp.w1.cuda(), wkey: torch.from_numpy(ws).cuda()}
        plan = moe.Plan(c.N, c.d, c.E, c.K, c.F, "e4m3", "none", w)
        ws_full = ws.astype(np.float64) if quant == "group" else \
            oracle.block_to_group_scales(ws, c.F)
        _gs_cache[key] = (inp, plan, w, xs, ws_full)
    return _gs_cache[key]


def gs_ref(inp, ws_full, x_group=None, x_tok=None, x_scale=1.0, gates=None):
    c = inp.cfg
    ids = inp.ids.numpy()
    _, _, rp, rs, rx = oracle.permute(ids, c.E, inp.x.numpy())
    row_e = np.repeat(np.arange(c.E, dtype=np.int32), np.bincount(ids.ravel(), minlength=c.E))
    G = c.d // 128
    xg = None
    if x_group is not None:
        xg = x_group[rs].astype(np.float64)
    elif x_tok is not None:
        xg = np.repeat(x_tok[rs].astype(np.float64)[:, None], G, axis=1)
    yp = oracle.expert_rows_kscaled(row_e, rx, oracle.E4M3, inp.w1, oracle.E4M3, ws_full,
                                    x_group_scales=xg, x_scale=x_scale)
    return oracle.combine(rp, gates, yp, c.N, c.K), yp, rp, rs


@pytest.mark.parametrize("name", list(GS))
@pytest.mark.parametrize("quant", ["group", "block"])
@pytest.mark.parametrize("gated", [False, True])
def test_forward_routed_group_scales(name, quant, gated):
    inp, plan, w, xs, ws_full = gs_case(name, quant)
    c = inp.cfg
    wsp = plan.new_workspace()
    g = None
    if gated:
        g = np.random.default_rng(4).random((c.N, c.K)).astype(np.float32)
        y = torch.empty(c.N, c.F, dtype=torch.bfloat16, device="cuda")
    else:
        y = torch.full((c.N * c.K, c.F), float("nan"), dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_group_scales(inp.x.cuda(), inp.ids.cuda(),
                                     None if g is None else torch.from_numpy(g).cuda(), y, wsp,
                                     x_group_scales=torch.from_numpy(xs).cuda())
    assert plan.read_device_status(wsp) == 0
    ref, _, _, _ = gs_ref(inp, ws_full, x_group=xs,
                          gates=None if g is None else g.astype(np.float64))
    err = rel_err(f64(y), ref)
    assert err <= TOL["e4m3"], err
    assert err <= 1e-2, err   # fp32 stage sums and promotion, one bf16 rounding


@pytest.mark.parametrize("quant", ["group", "block"])
def test_group_scales_with_token_and_scalar_activation_scales(quant):
    inp, plan, w, xs, ws_full = gs_case("gs_small", quant)
    c = inp.cfg
    wsp = plan.new_workspace()
    tok = np.random.default_rng(8).uniform(0.5, 2.0, size=c.N).astype(np.float32)
    y = torch.empty(c.N * c.K, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_group_scales(inp.x.cuda(), inp.ids.cuda(), None, y, wsp,
                                     x_token_scales=torch.from_numpy(tok).cuda())
    assert plan.read_device_status(wsp) == 0
    ref, _, _, _ = gs_ref(inp, ws_full, x_tok=tok)
    assert rel_err(f64(y), ref) <= 1e-2
    plan.forward_routed_group_scales(inp.x.cuda(), inp.ids.cuda(), None, y, wsp, x_scale=0.375)
    ref, _, _, _ = gs_ref(inp, ws_full, x_scale=0.375)
    assert rel_err(f64(y), ref) <= 1e-2


@pytest.mark.parametrize("name", ["gs_small", "gs_sparse", "gs_tall"])
@pytest.mark.parametrize("quant", ["group", "block"])
def test_group_scales_stage_call_equals_fused(name, quant):
    """moe_grouped_ffn_group_scales on the permuted rows (scales per permuted
    row) against the oracle, and the fused call's unpermuted rows equal to it
    bit for bit."""
    inp, plan, w, xs, ws_full = gs_case(name, quant)
    c = inp.cfg
    R = c.N * c.K
    wsp = plan.new_workspace()
    ref, yp_ref, rp, rs = gs_ref(inp, ws_full, x_group=xs)
    _, ro, _, _, rx = oracle.permute(inp.ids.numpy(), c.E, inp.x.numpy())
    y_perm = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.grouped_ffn_group_scales(torch.from_numpy(rx).cuda(), torch.from_numpy(ro).cuda(), y_perm,
                                  wsp, x_group_scales=torch.from_numpy(xs[rs]).cuda())
    assert plan.read_device_status(wsp) == 0
    assert rel_err(f64(y_perm), yp_ref) <= 1e-2
    y = torch.empty(R, c.F, dtype=torch.bfloat16, device="cuda")
    plan.forward_routed_group_scales(inp.x.cuda(), inp.ids.cuda(), None, y, wsp,
                                     x_group_scales=torch.from_numpy(xs).cuda())
    yp = y_perm.cpu().view(torch.int16).numpy()
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), yp[rp])


@pytest.mark.parametrize("name", ["bf16_swiglu_ragged", "f32_relu_n256", "e4m3_gmm"])
def test_stage_calls_with_zero_rows(name):
    """n = 0 (an expert-parallel rank that receives no rows): the row-count
    stage calls succeed, give all-zero counts and offsets and write nothing."""
    inp, plan, w = case(name)
    c = inp.cfg
    ws = plan.new_workspace()
    i32 = dict(dtype=torch.int32, device="cuda")
    counts = torch.full((c.E,), -7, **i32)
    offsets = torch.full((c.E + 1,), -7, **i32)
    pos = torch.full((c.N * c.K,), -7, **i32)
    src = torch.full((c.N * c.K,), -7, **i32)
    xdt = inp.x.dtype
    x_perm = torch.zeros(c.N * c.K, c.d, dtype=xdt, device="cuda")
    plan.permute(inp.x.cuda(), torch.zeros(c.N, c.K, **i32), counts, offsets, pos, src, x_perm, ws,
                 n=0)
    assert plan.read_device_status(ws) == 0
    assert not counts.cpu().any() and not offsets.cpu().any()
    ydt = torch.float32 if c.dtype == "f32" else torch.bfloat16
    y_perm = torch.full((c.N * c.K, c.d_out), 3.0, dtype=ydt, device="cuda")
    plan.grouped_ffn(x_perm, offsets, y_perm, ws, n=0, x_scale=inp.x_scale)
    y = torch.full((c.N, c.d_out), 5.0, dtype=ydt, device="cuda")
    plan.unpermute_combine(y_perm, pos, torch.ones(c.N, c.K, device="cuda"), y, ws, n=0)
    assert plan.read_device_status(ws) == 0
    assert bool((y_perm == 3.0).all()) and bool((y == 5.0).all())


def test_plan_refuses_host_scale_tables():
    """The plan-time kernels read the MX and group scale tables: a host
    pointer is refused with MOE_ERR_INVALID_ARG before any launch."""
    import top_routing_grouped_gemv_b200 as moe
    c = MX["mx_sparse"]
    inp = synth.make_inputs(c, 1)
    with pytest.raises(moe.MoEError) as e:
        moe.Plan(c.N, c.d, c.E, c.K, c.F, "e4m3", "none",
                 {"w1": inp.w1.cuda(), "w_mx_scales": inp.w_sf})   # host tensor
    assert e.value.code == 1
    g = GS["gs_sparse"].scaled(quant="block")
    ginp = synth.make_inputs(g, 1)
    with pytest.raises(moe.MoEError) as e:
        moe.Plan(g.N, g.d, g.E, g.K, g.F, "e4m3", "none",
                 {"w1": ginp.w1.cuda(), "w_block_scales": ginp.w_gs})
    assert e.value.code == 1


def test_refresh_router_after_weights_change():
    """A bf16 plan with at most 16 experts routes from its own split copy of
    w_r, taken at plan creation: changing w_r in place leaves the routing as it
    was until moe_plan_refresh_router, after which it follows the new weights
    (checked against the oracle)."""
    cfg = synth.MoEConfig("refresh", "bf16", 600, 256, 8, 2, 64, "swiglu")
    inp = synth.make_inputs(cfg, seed=5)
    plan, w = make_plan(inp)
    x = inp.x.cuda()
    ws = plan.new_workspace()

    def route():
        ids = torch.empty(cfg.N, cfg.K, dtype=torch.int32, device="cuda")
        gates = torch.empty(cfg.N, cfg.K, dtype=torch.float32, device="cuda")
        plan.router_topk(x, ids, gates, ws)
        torch.cuda.synchronize()
        return ids.cpu().numpy(), gates.cpu().double().numpy()

    ids0, _ = route()
    new_wr = torch.flip(inp.w_r, dims=[1]).contiguous()   # the experts in reverse order
    w["w_r"].copy_(new_wr.cuda())
    ids_stale, _ = route()
    assert np.array_equal(ids_stale, ids0)
    plan.refresh_router()
    ids1, g1 = route()
    rid, rg, _, logits = oracle.router(inp.x, oracle.DTYPE["bf16"], new_wr, None, cfg.K,
                                       want_logits=True)
    check_routing(ids1, g1, logits, rid, rg)
    assert not np.array_equal(ids1, ids0)
