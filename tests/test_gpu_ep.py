"""The expert-parallel layer (top_routing_grouped_gemv_b200.ep) with the
library's GPU stages on two ranks: two processes on one GPU, each holding
half of the experts, exchanging rows over gloo through host copies (no
kernel waits on another rank: the exchange is between kernel launches on
the host).  Each rank's output must equal the single-GPU moe_forward of its
tokens bit for bit (every routed row goes through the same kernels with the
same K order, whichever rank computes it), and the fp64 oracle's layer on
those tokens within the dtype's tolerance (tokens whose routing is a near
tie left out)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import synth

pytestmark = pytest.mark.gpu

CFGS = {
    "bf16_swiglu": synth.MoEConfig("ep_bf16", "bf16", 256, 256, 8, 2, 384, "swiglu"),
    "bf16_zipf_k4": synth.MoEConfig("ep_zipf", "bf16", 384, 256, 16, 4, 256, "swiglu",
                                    zipf_bias=1.2),
    "f32_relu": synth.MoEConfig("ep_f32", "f32", 192, 128, 8, 2, 256, "relu"),
    # a router bias of 50 ln(1/rank) sends every token to experts 0 and 1:
    # rank 1 (experts 2, 3) receives no rows and returns none
    "bf16_rank_empty": synth.MoEConfig("ep_empty", "bf16", 128, 256, 4, 2, 256, "swiglu",
                                       zipf_bias=50.0),
    # the fp8 grouped matmul with given routing and the pure unpermute (fp8
    # codes cross the exchange), against moe_forward_routed
    "e4m3_given": synth.MoEConfig("ep_e4m3", "e4m3", 256, 512, 8, 4, 384, "none",
                                  routing="given"),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, name, q, mode="a2a"):
    import datetime
    import torch.distributed as dist
    import top_routing_grouped_gemv_b200 as moe
    from top_routing_grouped_gemv_b200.ep import ExpertParallelMoE, LibraryStages
    import numpy as np
    import oracle
    from tests._util import NEAR_TIE, TOL, f64, rel_err, to_gpu
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        moe.load()
        c = CFGS[name]
        inp = synth.make_inputs(c, seed=5)
        w = to_gpu(inp)
        n_loc = c.N // world
        E_loc = c.E // world
        e0 = rank * E_loc
        x_all = inp.x.cuda()
        x = x_all[rank * n_loc:(rank + 1) * n_loc].contiguous()
        sl = lambda t: None if t is None else t[e0:e0 + E_loc].contiguous()
        stages = LibraryStages(n_loc, c.d, c.E, c.K, c.F, c.dtype, c.act, world, w.get("w_r"),
                               sl(w["w1"]), sl(w.get("w3")), sl(w.get("w2")), bias=w.get("bias"),
                               w_scale=inp.w_scale, x_scale=inp.x_scale)
        layer = ExpertParallelMoE(stages, c.E, c.K, host_exchange=True,
                                  overlap=mode == "overlap", capacity=mode == "capacity")
        # the whole layer on one GPU, all experts, this rank's tokens
        plan = moe.Plan(n_loc, c.d, c.E, c.K, c.F, c.dtype, c.act, w)
        ws = plan.new_workspace()
        if c.routing == "given":
            ids = inp.ids[rank * n_loc:(rank + 1) * n_loc].contiguous().cuda()
            y = layer.forward(x, ids=ids)
            torch.cuda.synchronize()
            y_ref = torch.empty_like(y)
            plan.forward_routed(x, ids, None, y_ref, ws, x_scale=inp.x_scale)
        else:
            y = layer.forward(x)
            torch.cuda.synchronize()
            y_ref = torch.empty_like(y)
            plan.forward(x, y_ref, ws)
        torch.cuda.synchronize()
        iv = torch.int32 if c.dtype == "f32" else torch.int16
        # the oracle's layer on this rank's tokens
        tok = np.arange(rank * n_loc, (rank + 1) * n_loc)
        given = c.routing == "given"
        ref, _, _, margin = oracle.forward_tokens(inp, tok, gates_mode=0 if given else 1)
        got = f64(y)
        if given:
            err = rel_err(got, ref)
        else:
            keep = margin > NEAR_TIE
            err = rel_err(got[keep], ref[keep])
        q.put((rank, stages.check(), plan.read_device_status(ws),
               bool(torch.equal(y.view(iv), y_ref.view(iv))), err, TOL[c.dtype]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


CASES = ([(n, "a2a") for n in CFGS] +
         [(n, "overlap") for n in ("bf16_zipf_k4", "bf16_rank_empty", "e4m3_given")] +
         [(n, "capacity") for n in ("bf16_swiglu", "bf16_zipf_k4", "bf16_rank_empty",
                                    "e4m3_given")])


@pytest.mark.parametrize("name,mode", CASES)
def test_expert_parallel_two_ranks_on_gpu_equal_single_gpu(name, mode):
    """mode a2a: variable-split all-to-alls; overlap: peer-to-peer blocks, own
    rows computed while the others travel; capacity: fixed-size padded blocks
    with the counts inside, no host read of the counts."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q, mode))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in res] == list(range(world))
    for rank, st_ep, st_ref, equal, err, tol in res:
        assert st_ep == 0 and st_ref == 0, (rank, st_ep, st_ref)
        assert equal, rank
        assert err <= tol, (rank, err)
