"""Expert parallelism (top_routing_grouped_gemv_b200.ep) over two and four
gloo ranks on the CPU: the dispatch / combine logic -- count exchange, split
sizes, the two all-to-alls, the regrouping by local expert and the restore --
with the oracle standing in for each rank's compute.  Every row is computed
as on one rank, so each rank's output must equal the oracle's whole layer on
that rank's tokens exactly (fp64, same per-row arithmetic)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from top_routing_grouped_gemv_b200.ep import ExpertParallelMoE


class OracleStages:
    """Each rank's compute done by the oracle (test only): routing over all
    experts, and this rank's experts for the rows it receives."""

    def __init__(self, inp, rank, world, n_loc):
        c = inp.cfg
        self.inp, self.c, self.n_loc = inp, c, n_loc
        self.dt = oracle.DTYPE[c.dtype]
        self.E_loc = c.E // world
        e0 = rank * self.E_loc
        self.w1 = inp.w1[e0:e0 + self.E_loc]
        self.w3 = None if inp.w3 is None else inp.w3[e0:e0 + self.E_loc]
        self.w2 = None if inp.w2 is None else inp.w2[e0:e0 + self.E_loc]
        self.d_out = c.d_out
        self.ydt = torch.float64

    def route(self, x):
        ids, gates, _, _ = oracle.router(x.numpy(), self.dt, self.inp.w_r, self.inp.bias, self.c.K)
        return torch.from_numpy(ids), torch.from_numpy(gates)

    def permute(self, x, ids):
        counts, offsets, pos, _, xp = oracle.permute(ids.numpy(), self.c.E, x.numpy())
        return (torch.from_numpy(counts), torch.from_numpy(offsets), torch.from_numpy(pos),
                torch.from_numpy(xp))

    def local_permute(self, n, x_recv, ids_recv):
        _, offsets, pos, _, xs = oracle.permute(ids_recv.numpy(), self.E_loc, x_recv.numpy())
        return torch.from_numpy(offsets), torch.from_numpy(pos), torch.from_numpy(xs)

    def local_ffn(self, n, x_sorted, offsets):
        row_e = np.repeat(np.arange(self.E_loc, dtype=np.int32), np.diff(offsets.numpy()))
        y = oracle.expert_rows(row_e, x_sorted.numpy(), self.dt, self.c.act, self.w1, self.w3,
                               self.w2, self.dt, self.inp.x_scale, self.inp.w_scale)
        return torch.from_numpy(y)

    def local_unpermute(self, n, y_sorted, pos):
        return torch.from_numpy(oracle.combine(pos.numpy(), None, y_sorted.numpy(), n, 1))

    def combine(self, y_perm, pos, gates):
        g = None if gates is None else gates.numpy()
        return torch.from_numpy(oracle.combine(pos.numpy(), g, y_perm.numpy(), self.n_loc,
                                               self.c.K))


CFGS = {
    # fp32 (gloo moves float32 rows), ReLU and SwiGLU, uneven routing
    "relu": synth.MoEConfig("ep_relu", "f32", 96, 64, 8, 2, 48, "relu"),
    "swiglu_zipf": synth.MoEConfig("ep_sw", "f32", 120, 32, 8, 3, 40, "swiglu", zipf_bias=1.2),
    # the fp8 single-matrix layer with given routing and the pure unpermute:
    # fp8 codes cross the exchange
    "e4m3_given": synth.MoEConfig("ep_e4m3", "e4m3", 96, 64, 8, 4, 48, "none", routing="given"),
    # a bias of 50 ln(1/rank) sends every token to experts 0 and 1: the ranks
    # holding experts 2 and 3 receive no rows
    "relu_ranks_empty": synth.MoEConfig("ep_empty", "f32", 64, 32, 4, 2, 16, "relu",
                                        zipf_bias=50.0),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, name, q, host_exchange=False, overlap=False, capacity=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CFGS[name]
        inp = synth.make_inputs(cfg, seed=99)
        n_loc = cfg.N // world
        x = inp.x[rank * n_loc:(rank + 1) * n_loc].contiguous()
        layer = ExpertParallelMoE(OracleStages(inp, rank, world, n_loc), cfg.E, cfg.K,
                                  host_exchange=host_exchange, overlap=overlap,
                                  capacity=capacity)
        tok = np.arange(rank * n_loc, (rank + 1) * n_loc)
        if cfg.routing == "given":
            y = layer.forward(x, ids=inp.ids[rank * n_loc:(rank + 1) * n_loc].contiguous()).numpy()
            ref, _, _, _ = oracle.forward_tokens(inp, tok, gates_mode=0)
        else:
            y = layer.forward(x).numpy()
            ref, _, _, _ = oracle.forward_tokens(inp, tok)
        q.put((rank, float(np.abs(y - ref).max()), float(np.abs(ref).max())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,host_exchange,overlap,capacity",
                         [(2, False, False, False), (4, False, False, False),
                          (2, True, False, False), (2, False, True, False), (4, True, True, False),
                          (2, False, False, True), (4, True, False, True)])
@pytest.mark.parametrize("name", list(CFGS))
def test_expert_parallel_matches_single_rank_oracle(name, world, host_exchange, overlap,
                                                    capacity):
    """host_exchange: the rows travel as byte views of host copies; overlap:
    peer-to-peer blocks, own rows computed while the others travel;
    capacity: fixed-size padded blocks with the counts inside, no host read
    of the counts."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker,
                         args=(r, world, port, name, q, host_exchange, overlap, capacity))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r for r, _, _ in res] == list(range(world))
    for rank, err, scale in res:
        assert scale > 0
        assert err == 0.0, (rank, err)


@pytest.mark.parametrize("capacity", [False, True])
def test_single_rank_without_process_group(capacity):
    cfg = CFGS["relu"]
    inp = synth.make_inputs(cfg, seed=3)
    layer = ExpertParallelMoE(OracleStages(inp, 0, 1, cfg.N), cfg.E, cfg.K, capacity=capacity)
    y = layer.forward(inp.x).numpy()
    ref, _, _, _ = oracle.forward_tokens(inp, np.arange(cfg.N))
    assert np.abs(y - ref).max() == 0.0


def test_capacity_exchange_reads_no_counts_on_the_host(monkeypatch):
    """The fixed-capacity exchange never moves a tensor's values to the host:
    every Tensor.cpu / .item / .tolist / bool / int / float during its
    exchange fails the test."""
    cfg = CFGS["swiglu_zipf"]
    inp = synth.make_inputs(cfg, seed=4)
    st = OracleStages(inp, 0, 1, cfg.N)
    layer = ExpertParallelMoE(st, cfg.E, cfg.K, capacity=True)
    x = inp.x
    ids, gates = st.route(x)
    counts, offsets, pos, x_perm = st.permute(x, ids)
    calls = []
    for name in ("cpu", "item", "tolist", "__bool__", "__int__", "__float__"):
        monkeypatch.setattr(torch.Tensor, name, lambda self, *a, _n=name, **k: calls.append(_n))
    monkeypatch.setattr(st, "local_ffn",
                        lambda n, xs, offs: torch.zeros(n, st.d_out, dtype=torch.float64))
    y_perm = layer._exchange_capacity(None, 1, cfg.E, x_perm, counts, offsets)
    monkeypatch.undo()
    assert calls == []
    assert tuple(y_perm.shape) == (cfg.N * cfg.K, st.d_out)
