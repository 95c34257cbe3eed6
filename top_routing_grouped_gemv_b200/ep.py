"""Expert parallelism across GPUs: the experts of one layer are split over the
ranks of a process group (rank r holds experts [r*E/G, (r+1)*E/G)), and each
rank's tokens travel to the ranks that hold their experts and back
("Advanced GPU Optimization ... Part 5", section 1.2 Expert Parallelism with
All-to-All Communication: dispatch, local expert FFNs, combine;
aclnnQuantGroupedMatMulAlltoAllv: AlltoAllv around the grouped matmul).

One step on rank r (G ranks, E experts, E_loc = E / G):
  1. route its N tokens over all E experts (router, top-K, gates);
  2. permute the routed rows by expert: rows for rank q's experts are the
     q-th contiguous block;
  3. exchange the per-expert row counts (all-to-all of G x E_loc counts), so
     that every rank knows how many rows it sends to and receives from each
     rank (the host reads them: the split sizes of the next exchange);
  4. all-to-all the rows (variable splits);
  5. regroup the received rows by local expert (a permute with K = 1; rows
     of one expert keep source-rank order), run the local experts on them,
     and restore the received order (the pure reorder);
  6. all-to-all the results back (the splits of step 4 swapped);
  7. unpermute and combine with the gates.
Every row is computed exactly as on one GPU, so the result equals the
single-GPU layer's bit for bit.

The per-step work is done by a `stages` object (the library's kernels on the
GPU: `LibraryStages`); the exchanges use torch.distributed (NCCL on GPUs).
With `host_exchange=True` the exchanged tensors travel as host copies (byte
views of the rows), for process groups whose backend moves only host memory
(gloo).  With `overlap=True` the rows travel peer to peer (isend / irecv):
the rank's rows for its own experts are computed while the others are in
flight, then every peer's rows as they arrive, each block's results sent
straight back (computing and communicating overlap; more, smaller expert
launches).  Every row is still computed as on one GPU.  Without an
initialized process group the layer runs on one rank with no exchange.

With `capacity=True` the host never reads the counts: every per-peer block
has a fixed capacity of N*K rows (all of a rank's routed rows could go to one
peer), the block's per-expert counts travel in header rows at its start, and
both exchanges are all-to-alls of equal, fixed splits.  The sender fills its
blocks, and the receiver regroups the rows by local expert and returns the
results into the same padded layout, by index arithmetic on the device
(cumulative counts, searchsorted, row gathers), so a step has no device to
host synchronisation.  The price is bytes on the wire: G * (header + N*K)
rows per rank and direction against the about N*K rows of the variable-split
exchange, i.e. about G times as many.  Every rank must hold the same number
of tokens (the capacity is the same on all ranks).
"""
from __future__ import annotations

import torch

__all__ = ["ExpertParallelMoE", "LibraryStages"]


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


class LibraryStages:
    """The step's compute on this GPU through the C-ABI library: a
    routing-only plan over all E experts for the rank's own tokens, and a
    plan of the rank's E_loc experts (K = 1) for the rows it receives.

    ``w_r`` (d, E) fp32 and optional ``bias`` route over all experts (None:
    the caller gives the routing to ExpertParallelMoE.forward);
    ``w1``/``w3``/``w2`` are this rank's experts only ((E_loc, F, d) etc.).
    e4m3 layers take the per-tensor ``w_scale`` and ``x_scale``: the rows
    cross the exchange as fp8 codes."""

    def __init__(self, N, d, E, K, F, dtype, act, world, w_r, w1, w3=None, w2=None, bias=None,
                 w_scale=1.0, x_scale=1.0):
        from . import Plan
        if E % world:
            raise ValueError(f"{E} experts do not split over {world} ranks")
        self.N, self.d, self.E, self.K, self.F = N, d, E, K, F
        self.E_loc = E // world
        self.d_out = F if act == "none" else d
        self.dtype = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[dtype]
        self.ydt = torch.float32 if dtype == "f32" else torch.bfloat16
        self.x_scale = x_scale
        route_w = {}
        if w_r is not None:
            route_w["w_r"] = w_r
        if bias is not None:
            route_w["bias"] = bias
        self.glob = Plan(N, d, E, K, F, dtype, act, route_w)
        self.n_max = N * K * world  # every row of every rank may come here
        local_w = {"w1": w1, "w_scale": w_scale}
        if w3 is not None:
            local_w["w3"] = w3
        if w2 is not None:
            local_w["w2"] = w2
        self.loc = Plan(self.n_max, d, self.E_loc, 1, F, dtype, act, local_w)
        self.ws_g = self.glob.new_workspace()
        self.ws_l = self.loc.new_workspace()
        dev = w1.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.ids = torch.empty(N, K, **i32)
        self.gates = torch.empty(N, K, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.pos = torch.empty(N * K, **i32)
        self.src = torch.empty(N * K, **i32)
        self.x_perm = torch.empty(N * K, d, dtype=self.dtype, device=dev)
        self.counts_l = torch.empty(self.E_loc, **i32)
        self.offsets_l = torch.empty(self.E_loc + 1, **i32)
        self.pos_l = torch.empty(self.n_max, **i32)
        self.src_l = torch.empty(self.n_max, **i32)
        self.x_sorted = torch.empty(self.n_max, d, dtype=self.dtype, device=dev)
        self.y_sorted = torch.empty(self.n_max, self.d_out, dtype=self.ydt, device=dev)

    def route(self, x):
        self.glob.router_topk(x, self.ids, self.gates, self.ws_g)
        return self.ids, self.gates

    def permute(self, x, ids):
        self.glob.permute(x, ids, self.counts, self.offsets, self.pos, self.src, self.x_perm,
                          self.ws_g)
        return self.counts, self.offsets, self.pos, self.x_perm

    def local_permute(self, n, x_recv, ids_recv):
        if n == 0:  # nothing received: no launches (an empty tensor may have no address)
            self.offsets_l.zero_()
            return self.offsets_l, self.pos_l[:0], self.x_sorted[:0]
        self.loc.permute(x_recv, ids_recv, self.counts_l, self.offsets_l, self.pos_l, self.src_l,
                         self.x_sorted, self.ws_l, n=n)
        return self.offsets_l, self.pos_l, self.x_sorted

    def local_ffn(self, n, x_sorted, offsets):
        if n == 0:
            return self.y_sorted[:0]
        self.loc.grouped_ffn(x_sorted, offsets, self.y_sorted, self.ws_l, n=n, x_scale=self.x_scale)
        return self.y_sorted

    def local_unpermute(self, n, y_sorted, pos):
        if n == 0:
            return torch.empty(0, self.d_out, dtype=self.ydt, device=y_sorted.device)
        y_recv = torch.empty(n, self.d_out, dtype=self.ydt, device=y_sorted.device)
        self.loc.unpermute_combine(y_sorted, pos, None, y_recv, self.ws_l, n=n)
        return y_recv

    def combine(self, y_perm, pos, gates):
        """gates None: the pure unpermute, y (N*K, d_out) token-major."""
        rows = self.N if gates is not None else self.N * self.K
        y = torch.empty(rows, self.d_out, dtype=self.ydt, device=y_perm.device)
        self.glob.unpermute_combine(y_perm, pos, gates, y, self.ws_g)
        return y

    def check(self):
        """Sticky device status of both plans' workspaces (0 = clean)."""
        return self.glob.read_device_status(self.ws_g) or self.loc.read_device_status(self.ws_l)


class ExpertParallelMoE:
    """The expert-parallel layer on this rank (see the module docstring)."""

    def __init__(self, stages, E: int, K: int, group=None, host_exchange: bool = False,
                 overlap: bool = False, capacity: bool = False):
        if overlap and capacity:
            raise ValueError("choose one exchange: overlap or capacity")
        self.stages, self.E, self.K, self.group = stages, E, K, group
        self.host_exchange = host_exchange
        self.overlap = overlap
        self.capacity = capacity

    def _all_to_all(self, dist, t, out_rows, out_splits=None, in_splits=None):
        """all_to_all_single of the rows of t (variable splits if given)."""
        shape = (out_rows,) + tuple(t.shape[1:])
        if not self.host_exchange:
            out = t.new_empty(shape)
            dist.all_to_all_single(out, t.contiguous(), out_splits, in_splits, group=self.group)
            return out
        # host copies, rows as bytes (the backend may not know the dtype)
        src_b = self._wire_host(t)
        row_bytes = src_b.shape[1]
        out_b = torch.empty((out_rows, row_bytes), dtype=torch.uint8)
        dist.all_to_all_single(out_b, src_b, out_splits, in_splits, group=self.group)
        return out_b.view(t.dtype).reshape(shape).to(t.device)

    def _world(self):
        dist = _dist()
        if dist is None:
            return None, 1, 0
        return dist, dist.get_world_size(self.group), dist.get_rank(self.group)

    def forward(self, x, ids=None, gates=None):
        """ids (N, K) int32 / gates (N, K) fp32: routing given by the caller
        (default: the stages' router); with given ids and no gates the result
        is the pure unpermute (N*K, d_out), as the single-GPU routed layer."""
        st = self.stages
        dist, G, _ = self._world()
        if self.E % G:
            raise ValueError(f"{self.E} experts do not split over {G} ranks")
        E_loc = self.E // G
        if ids is None:
            ids, gates = st.route(x)
        counts, offsets, pos, x_perm = st.permute(x, ids)
        if self.capacity:
            y_perm = self._exchange_capacity(dist, G, E_loc, x_perm, counts, offsets)
            return st.combine(y_perm, pos, gates)

        # per-expert row counts: block q of my counts goes to rank q
        send_counts = counts.to(torch.int64).reshape(G, E_loc)
        if dist is not None:
            recv_counts = self._all_to_all(dist, send_counts, G)
        else:
            recv_counts = send_counts.clone()
        send_h, recv_h = send_counts.cpu(), recv_counts.cpu()
        send_rows = send_h.sum(1).tolist()
        recv_rows = recv_h.sum(1).tolist()
        n_send, n_recv = sum(send_rows), sum(recv_rows)

        if self.overlap and dist is not None and G > 1:
            y_perm = self._exchange_overlapped(dist, G, x_perm, send_h, recv_h)
            return st.combine(y_perm, pos, gates)

        # dispatch: the rows, source-major, expert-minor within each source
        if dist is not None:
            x_recv = self._all_to_all(dist, x_perm[:n_send], n_recv, recv_rows, send_rows)
        else:
            x_recv = x_perm[:n_send]
        # regroup by local expert, run the local experts, restore the order
        eids = torch.arange(E_loc, dtype=torch.int32).repeat(G)
        ids_recv = torch.repeat_interleave(eids, recv_h.reshape(-1)).to(x_recv.device)
        ids_recv = ids_recv.reshape(-1, 1).contiguous()
        offsets_l, pos_l, x_sorted = st.local_permute(n_recv, x_recv, ids_recv)
        y_sorted = st.local_ffn(n_recv, x_sorted, offsets_l)
        y_recv = st.local_unpermute(n_recv, y_sorted, pos_l)

        # return the results: the dispatch splits swapped
        if dist is not None:
            y_perm = self._all_to_all(dist, y_recv, n_send, send_rows, recv_rows)
        else:
            y_perm = y_recv
        return st.combine(y_perm, pos, gates)

    # ---- fixed-capacity exchange: no host read of the counts ------------------

    @staticmethod
    def _bytes(t):
        """(rows, row bytes) uint8 view of a contiguous row tensor."""
        t = t.contiguous()
        row_bytes = t.element_size()
        for n in t.shape[1:]:
            row_bytes *= n
        return t.view(torch.uint8).reshape(t.shape[0], row_bytes)

    def _exchange_capacity(self, dist, G, E_loc, x_perm, counts, offsets):
        st = self.stages
        dev = x_perm.device
        i64 = dict(dtype=torch.int64, device=dev)
        NK = x_perm.shape[0]
        C = NK                                   # rows per peer block
        xb = self._bytes(x_perm)                 # (NK, rb)
        rb = xb.shape[1]
        H = -(-4 * E_loc // rb)                  # header rows holding E_loc int32 counts
        cnt = counts.to(**i64).reshape(G, E_loc)
        send_rows = cnt.sum(1)                                   # rows for rank q
        send_off = offsets.to(**i64)[torch.arange(G, device=dev) * E_loc]
        # my blocks: rows [send_off[q], send_off[q] + send_rows[q]) of x_perm
        slot = torch.arange(C, **i64)
        src = send_off[:, None] + slot[None, :]
        src = torch.where(slot[None, :] < send_rows[:, None], src, torch.zeros_like(src))
        hdr = torch.zeros(G, H * rb, dtype=torch.uint8, device=dev)
        hdr[:, :4 * E_loc] = cnt.to(torch.int32).contiguous().view(torch.uint8)
        send = torch.cat([hdr.reshape(G, H, rb), xb[src.reshape(-1)].reshape(G, C, rb)], dim=1)
        recv = self._fixed_all_to_all(dist, G, send)             # (G, H + C, rb)
        # counts of the rows from rank q for my local expert l
        rcnt = recv[:, :H].reshape(G, H * rb)[:, :4 * E_loc].contiguous().view(torch.int32)
        rcnt = rcnt.to(torch.int64)                              # (G, E_loc)
        tot = rcnt.sum(0)
        offs_l = torch.zeros(E_loc + 1, **i64)
        offs_l[1:] = torch.cumsum(tot, 0)
        sstart = torch.cumsum(rcnt, 1) - rcnt                    # start of (q, l) in block q
        dstart = offs_l[:-1][None, :] + (torch.cumsum(rcnt, 0) - rcnt)  # start of (q, l) sorted
        # sorted row j <- its (expert l, source q) segment, expert-major, source-minor
        flat_cnt = rcnt.t().reshape(-1)
        flat_end = torch.cumsum(flat_cnt, 0)
        j = torch.arange(G * C, **i64)
        k = torch.searchsorted(flat_end, j, right=True)
        kk = k.clamp(max=E_loc * G - 1)
        l, q = kk // G, kk % G
        i = j - (flat_end[kk] - flat_cnt[kk])
        rows_src = q * (H + C) + H + sstart[q, l] + i
        rows_src = torch.where(k < E_loc * G, rows_src, torch.zeros_like(rows_src))
        x_sorted = recv.reshape(-1, rb)[rows_src].contiguous().view(x_perm.dtype)
        x_sorted = x_sorted.reshape((G * C,) + tuple(x_perm.shape[1:]))
        y_sorted = st.local_ffn(G * C, x_sorted, offs_l.to(torch.int32))
        # results into the padded blocks: block q row H + sstart[q, l] + i <- y_sorted[dstart + i]
        rc_end = torch.cumsum(rcnt, 1)
        r = torch.arange(C, **i64).expand(G, C).contiguous()
        lq = torch.searchsorted(rc_end, r, right=True)
        lq_c = lq.clamp(max=E_loc - 1)
        i2 = r - (rc_end.gather(1, lq_c) - rcnt.gather(1, lq_c))
        ysrc = dstart.gather(1, lq_c) + i2
        ysrc = torch.where(lq < E_loc, ysrc, torch.zeros_like(ysrc))
        if y_sorted.shape[0] == 0:       # no rows anywhere on this rank's experts
            like = self._result_like(x_perm)
            yb = torch.zeros(G * C, self._bytes(like).shape[1], dtype=torch.uint8, device=dev)
            ydt, tail = like.dtype, tuple(like.shape[1:])
        else:
            yb = self._bytes(y_sorted)[ysrc.reshape(-1)]
            ydt, tail = y_sorted.dtype, tuple(y_sorted.shape[1:])
        ret = self._fixed_all_to_all(dist, G, yb.reshape(G, C, -1))   # my rows' results
        # back in my permuted order: row r of x_perm was row r - send_off[q] of block q
        send_end = torch.cumsum(send_rows, 0)
        rr = torch.arange(NK, **i64)
        rq = torch.searchsorted(send_end, rr, right=True).clamp(max=G - 1)
        yrow = rq * C + (rr - send_off[rq])
        yrow = torch.where(rr < send_end[-1], yrow, torch.zeros_like(yrow))
        return ret.reshape(G * C, -1)[yrow].contiguous().view(ydt).reshape((NK,) + tail)

    def _fixed_all_to_all(self, dist, G, t):
        """all_to_all_single of G equal blocks of a (G, rows, bytes) uint8 tensor."""
        if dist is None:
            return t
        flat = t.reshape(t.shape[0] * t.shape[1], t.shape[2])
        out = self._all_to_all(dist, flat, flat.shape[0])
        return out.reshape(t.shape)

    # ---- peer-to-peer exchange overlapped with the local experts -------------

    @staticmethod
    def _wire_host(t):
        """Host byte view of the rows of t (rows, row bytes); a zero-row tensor
        (whose strides may not allow a view) gives an empty byte tensor."""
        row_bytes = t.element_size()
        for n in t.shape[1:]:
            row_bytes *= n
        if t.shape[0] == 0:
            return torch.empty((0, row_bytes), dtype=torch.uint8)
        return t.contiguous().cpu().view(torch.uint8).reshape(t.shape[0], row_bytes)

    def _wire(self, t):
        """The tensor as it travels: itself, or a host byte view."""
        if not self.host_exchange:
            return t.contiguous()
        return self._wire_host(t)

    def _wire_buffer(self, rows, like):
        shape = (rows,) + tuple(like.shape[1:])
        if not self.host_exchange:
            return like.new_empty(shape)
        row_bytes = like.element_size()
        for n in like.shape[1:]:
            row_bytes *= n
        return torch.empty((rows, row_bytes), dtype=torch.uint8)

    def _unwire(self, buf, like, rows):
        if not self.host_exchange:
            return buf
        return buf.view(like.dtype).reshape((rows,) + tuple(like.shape[1:])).to(like.device)

    def _compute_block(self, rows, x_rows, counts_q):
        """This rank's experts on rows received from one source (expert-
        contiguous, counts_q rows per local expert): regroup, FFN, restore."""
        st = self.stages
        E_loc = counts_q.numel()
        ids_q = torch.repeat_interleave(torch.arange(E_loc, dtype=torch.int32), counts_q)
        ids_q = ids_q.to(x_rows.device).reshape(-1, 1).contiguous()
        offsets_l, pos_l, x_sorted = st.local_permute(rows, x_rows, ids_q)
        y_sorted = st.local_ffn(rows, x_sorted, offsets_l)
        return st.local_unpermute(rows, y_sorted, pos_l)

    def _exchange_overlapped(self, dist, G, x_perm, send_h, recv_h):
        rank = dist.get_rank(self.group)
        send_rows = send_h.sum(1).tolist()
        recv_rows = recv_h.sum(1).tolist()
        send_off = [0] * G
        for q in range(1, G):
            send_off[q] = send_off[q - 1] + send_rows[q - 1]
        peer = (lambda q: dist.get_global_rank(self.group, q)) if self.group is not None else \
            (lambda q: q)
        # post every dispatch receive and send (tag 1); empty blocks are not sent
        recv_buf, reqs, sends = {}, [], []
        for q in range(G):
            if q == rank:
                continue
            if recv_rows[q]:
                recv_buf[q] = self._wire_buffer(recv_rows[q], x_perm)
                reqs.append((q, dist.irecv(recv_buf[q], src=peer(q), group=self.group, tag=1)))
            if send_rows[q]:
                blk = self._wire(x_perm[send_off[q]:send_off[q] + send_rows[q]])
                recv_buf[("send", q)] = blk   # alive until its send completes
                sends.append(dist.isend(blk, dst=peer(q), group=self.group, tag=1))
        y_parts = {}
        # my own rows first, while the others travel
        if send_rows[rank]:
            own = x_perm[send_off[rank]:send_off[rank] + send_rows[rank]]
            y_parts[rank] = self._compute_block(send_rows[rank], own, recv_h[rank])
        # then each peer's rows as they arrive; the results go straight back (tag 2)
        back_recv, back_keep = {}, []
        y_like = None
        for q, req in reqs:
            req.wait()
            x_q = self._unwire(recv_buf[q], x_perm, recv_rows[q])
            y_q = self._compute_block(recv_rows[q], x_q, recv_h[q])
            y_like = y_q
            w = self._wire(y_q)
            back_keep.append(w)
            sends.append(dist.isend(w, dst=peer(q), group=self.group, tag=2))
        if y_like is None and rank in y_parts:
            y_like = y_parts[rank]
        # collect my rows' results from every peer
        pending = []
        for q in range(G):
            if q != rank and send_rows[q]:
                like = y_like if y_like is not None else self._result_like(x_perm)
                back_recv[q] = self._wire_buffer(send_rows[q], like)
                pending.append((q, like, dist.irecv(back_recv[q], src=peer(q), group=self.group,
                                                    tag=2)))
        for q, like, req in pending:
            req.wait()
            y_parts[q] = self._unwire(back_recv[q], like, send_rows[q])
        for w in sends:
            w.wait()
        # the results in the permuted order (rank blocks in rank order)
        blocks = [y_parts[q] for q in range(G) if send_rows[q]]
        if not blocks:
            return self._result_like(x_perm)[:0]
        return torch.cat(blocks, dim=0)

    def _result_like(self, x_perm):
        """An empty result-shaped tensor (rows, d_out) of the stages' output dtype."""
        st = self.stages
        d_out = getattr(st, "d_out", None)
        ydt = getattr(st, "ydt", None)
        if d_out is None or ydt is None:
            raise ValueError("the stages give no result shape")
        return torch.empty(1, d_out, dtype=ydt, device=x_perm.device)
