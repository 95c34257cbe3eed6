"""moe_permute_noalloc, the permute entry point for callers that cannot
allocate device memory (a framework that owns all device memory and passes
only inputs and outputs, or a latency-critical path that must not risk the
device synchronisation of cudaMalloc/cudaFree).  Its scratch lives in the
library's static device memory instead of a caller workspace.

Checked through the C ABI against moe_permute on two calls in a row with
different routings, so a stale scratch array from the first call would
show up in the second.  Collected last so that a run stopping at the first
failure has already run every other test.  It needs no state from other
tests (it builds and loads the library itself), so it passes both after the
rest of the suite and on its own (pytest tests/test_zz_no_alloc.py).
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _routing(seed, N, E, K):
    return torch.from_numpy(synth.given_routing(seed, N, E, K)).cuda()


def test_noalloc_permute_matches_workspace_permute_twice():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    import top_routing_grouped_gemv_b200 as moe
    moe.build()
    cfg = synth.small_variant(synth.BF16_FINEGRAINED, N=1000, d=256, E=64, K=8, F=128)
    inp = synth.make_inputs(cfg, seed=99)
    w = {"w1": inp.w1.cuda(), "w3": inp.w3.cuda(), "w2": inp.w2.cuda(), "w_r": inp.w_r.cuda()}
    plan = moe.Plan(cfg.N, cfg.d, cfg.E, cfg.K, cfg.F, cfg.dtype, cfg.act, w)
    ws = plan.new_workspace()
    x = inp.x.cuda()
    R = cfg.N * cfg.K

    def bufs():
        return [torch.empty(cfg.E, dtype=torch.int32, device="cuda"),
                torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda"),
                torch.empty(R, dtype=torch.int32, device="cuda"),
                torch.empty(R, dtype=torch.int32, device="cuda"),
                torch.empty(R, cfg.d, dtype=torch.bfloat16, device="cuda")]

    for call, seed in enumerate((1, 2)):
        ids = _routing(seed, cfg.N, cfg.E, cfg.K)
        ref = bufs()
        plan.permute(x, ids, *ref, ws)
        got = bufs()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        plan.permute_noalloc(x, ids, *got, device_status=status)
        assert plan.last_launch_count() == 2  # rank (+ scan) and gather, as moe_permute
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        for a, b in zip(got, ref):
            a, b = a.cpu(), b.cpu()
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), f"call {call}: differs from moe_permute"
    assert plan.read_device_status(ws) == 0


def test_noalloc_permute_refuses_plans_beyond_its_scratch():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    import top_routing_grouped_gemv_b200 as moe
    moe.build()
    # 256 + ceil(300000/256) * 256 experts * 4 bytes = 1.2 MB > the 1 MiB static scratch
    dummy = torch.empty(16, dtype=torch.float32, device="cuda")
    plan = moe.Plan(300000, 16, 256, 8, 16, "f32", "none", {"w1": dummy})
    with pytest.raises(moe.MoEError) as e:
        plan.permute_noalloc(dummy, dummy, dummy, dummy, dummy, dummy, dummy)
    assert e.value.code == 3  # MOE_ERR_WORKSPACE_TOO_SMALL, nothing launched
