"""Expert-parallel form of the MoE layer: the routed experts split over
`ep_size` ranks, each rank's tokens sent to the experts' owners and their
outputs sent back (two all-to-alls around the expert GEMMs).

This is the deployment the pages describe for the model ("Xiaohongshu dots3
note Open Source Deep Dive", §8.2: FUSED_MC2 "dispatch -> gmm1 -> swiglu ->
gmm2 -> combine" across devices; §10.2: expert parallelism with an
all-to-all backend).  Rank d owns experts [d E/ep_size, (d+1) E/ep_size) and
holds the router and the shared expert in full.  One rank's step:

  1. route and permute its own tokens (moe_route, moe_permute), then pack the
     routed rows in expert order, which is destination order (moe_ep_pack);
  2. all-to-all of the per-destination row counts, then of the rows, their
     routing weights and their experts' local indices;
  3. the received rows form a k = 1 layer over the rank's own experts
     (moe_permute, moe_expert_ffn, moe_combine back to the receive order);
  4. the reverse all-to-all returns every row to its sender, in send order;
  5. the shared expert and the combine over the returned rows (moe_shared_expert,
     moe_combine) give the rank's output.

Host orchestration only: every step of the layer runs in the library's
kernels (`CudaSteps`); the collective is the caller's process group
(`DistExchange`: torch.distributed, NCCL over NVLink on GPUs) or, for N
virtual ranks on one GPU, device copies (`ep_forward_virtual`).

The second form moves the rows with the library's own kernels over peer
memory (`ep_forward_peer`, `ep_forward_peer_virtual`): the sender stores each
routed row straight into its owner's receive buffer, already in the owner's
expert order, and after the owners' expert GEMMs its combine kernel loads the
rows' outputs back and sums them with the shared expert; only the per-expert
counts go through a collective.  No TMA multicast is involved anywhere.
"""
from __future__ import annotations

from dataclasses import replace

import torch


def local_config(cfg, rows: int, ep_size: int):
    """The k = 1 layer a rank runs over the rows it received: its
    E / ep_size experts, no shared expert, the weights given per row."""
    return replace(cfg, T=rows, E=cfg.E // ep_size, k=1, n_shared=0, n_group=1, topk_group=1,
                   norm_topk_prob=False, routed_scaling_factor=1.0)


class CudaSteps:
    """The library's kernels for each step (argument marshalling only)."""

    def __init__(self, binding=None):
        if binding is None:
            from . import binding
        self.B = binding

    def route_and_pack(self, cfg, ep_size, x, w_router, bias):
        B = self.B
        T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.k
        dev = x.device
        ws = B.alloc_workspace(cfg, device=dev)
        logits = torch.empty((T, E), device=dev)
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), device=dev)
        B.moe_route(cfg, x, w_router, bias, logits, idx, w, ws)
        offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        rows = torch.empty((T * k,), dtype=torch.int32, device=dev)
        pos = torch.empty((T * k,), dtype=torch.int32, device=dev)
        B.moe_permute(cfg, idx, offsets, rows, pos, ws)
        st = {"ws": ws, "idx": idx, "w": w, "pos": pos,
              "x_send": torch.empty((T * k, H), dtype=torch.bfloat16, device=dev),
              "w_send": torch.empty((T * k,), device=dev),
              "e_send": torch.empty((T * k,), dtype=torch.int32, device=dev),
              "send_counts": torch.empty((ep_size,), dtype=torch.int32, device=dev)}
        B.moe_ep_pack(cfg, ep_size, x, idx, w, offsets, pos, st["x_send"], st["w_send"],
                      st["e_send"], st["send_counts"])
        return st

    def experts(self, cfg, ep_size, x_recv, w_recv, e_recv, w13_local, w2_local):
        B = self.B
        R, H = x_recv.shape[0], cfg.H
        out = torch.empty((R, H), dtype=torch.bfloat16, device=x_recv.device)
        if R == 0:
            return out
        lc = local_config(cfg, R, ep_size)
        ws = B.alloc_workspace(lc, device=x_recv.device)
        offsets = torch.empty((lc.E + 1,), dtype=torch.int32, device=x_recv.device)
        rows = torch.empty((R,), dtype=torch.int32, device=x_recv.device)
        pos = torch.empty((R,), dtype=torch.int32, device=x_recv.device)
        B.moe_permute(lc, e_recv.view(R, 1), offsets, rows, pos, ws)
        y = torch.empty((R, H), dtype=torch.float32, device=x_recv.device)  # k = 1: fp32 rows
        B.moe_expert_ffn(lc, x_recv, offsets, rows, pos, w_recv, w13_local, w2_local, None, None,
                         y, None, ws)
        B.moe_combine(lc, y, pos, None, out)  # back to the receive order, one bf16 rounding
        return out

    def shared_and_combine(self, cfg, st, x, y_ret, w13s, w2s):
        B = self.B
        ysh = None
        if cfg.n_shared > 0:
            ysh = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device=x.device)
            B.moe_shared_expert(cfg, x, w13s, w2s, ysh, st["ws"])
        out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=x.device)
        B.moe_combine(cfg, y_ret, st["pos"], ysh, out)
        return out


class DistExchange:
    """All-to-alls over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for host tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def counts(self, send_counts: torch.Tensor) -> list[int]:
        recv = torch.empty_like(send_counts)
        self.dist.all_to_all_single(recv, send_counts.contiguous(), group=self.group)
        return [int(v) for v in recv.tolist()]

    def rows(self, send: torch.Tensor, send_counts: list[int], recv_counts: list[int]):
        recv = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype,
                           device=send.device)
        self.dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=recv_counts,
                                    input_split_sizes=send_counts, group=self.group)
        return recv


def ep_forward(cfg, ep_rank: int, ep_size: int, x, w_router, bias, w13_local, w2_local, w13s,
               w2s, exchange=None, steps=None):
    """One rank's layer output [T, H] with the experts split over ep_size
    ranks; w13_local / w2_local are this rank's E / ep_size experts.  Every
    rank of the group calls it with the same cfg (its own T tokens)."""
    steps = steps or CudaSteps()
    exchange = exchange or DistExchange()
    if cfg.E % ep_size:
        raise ValueError("ep_size %d must divide E = %d" % (ep_size, cfg.E))
    st = steps.route_and_pack(cfg, ep_size, x, w_router, bias)
    send_counts = [int(v) for v in st["send_counts"].tolist()]
    recv_counts = exchange.counts(st["send_counts"])
    x_recv = exchange.rows(st["x_send"], send_counts, recv_counts)
    w_recv = exchange.rows(st["w_send"], send_counts, recv_counts)
    e_recv = exchange.rows(st["e_send"], send_counts, recv_counts)
    y_back = steps.experts(cfg, ep_size, x_recv, w_recv, e_recv, w13_local, w2_local)
    y_ret = exchange.rows(y_back, recv_counts, send_counts)
    return steps.shared_and_combine(cfg, st, x, y_ret, w13s, w2s)


def ep_forward_virtual(cfg, xs, w_router, bias, w13, w2, w13s, w2s, steps=None):
    """N = len(xs) virtual ranks on one device: rank r holds tokens xs[r] and
    experts [r E/N, (r+1) E/N) of w13 / w2; the all-to-alls are device copies.
    Returns the N ranks' outputs."""
    steps = steps or CudaSteps()
    N = len(xs)
    if cfg.E % N:
        raise ValueError("N = %d must divide E = %d" % (N, cfg.E))
    el = cfg.E // N
    sts = [steps.route_and_pack(cfg, N, x, w_router, bias) for x in xs]
    cnt = [[int(v) for v in st["send_counts"].tolist()] for st in sts]  # [src][dst]

    def chunk(t, counts, d):
        start = sum(counts[:d])
        return t[start:start + counts[d]]

    y_back = []
    for d in range(N):
        recv = {key: torch.cat([chunk(sts[s][key], cnt[s], d) for s in range(N)])
                for key in ("x_send", "w_send", "e_send")}
        y_back.append(steps.experts(cfg, N, recv["x_send"], recv["w_send"], recv["e_send"],
                                    w13[d * el:(d + 1) * el], w2[d * el:(d + 1) * el]))
    outs = []
    for s in range(N):
        parts = []
        for d in range(N):
            off = sum(cnt[s2][d] for s2 in range(s))  # rows from s in d's receive buffer
            parts.append(y_back[d][off:off + cnt[s][d]])
        y_ret = torch.cat(parts)
        outs.append(steps.shared_and_combine(cfg, sts[s], xs[s], y_ret, w13s, w2s))
    return outs


# ---------------------------------------------------------------------------
# The exchange over peer memory (moe_ep_expert_counts, moe_ep_plan,
# moe_ep_dispatch_peer, moe_ep_combine_peer): the sender's kernel stores each
# routed row into its owner's receive buffer, already in the owner's expert
# order, and its combine kernel loads the rows' outputs back from the owners'
# buffers.  Only the per-expert counts are exchanged by a collective.

def _peer_step_front(B, cfg, x, w_router, bias):
    """Route, permute and count one rank's tokens."""
    T, E, k = cfg.T, cfg.E, cfg.k
    dev = x.device
    st = {"ws": B.alloc_workspace(cfg, device=dev)}
    st["logits"] = torch.empty((T, E), device=dev)
    st["idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
    st["w"] = torch.empty((T, k), device=dev)
    B.moe_route(cfg, x, w_router, bias, st["logits"], st["idx"], st["w"], st["ws"])
    st["offsets"] = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    st["rows"] = torch.empty((T * k,), dtype=torch.int32, device=dev)
    st["pos"] = torch.empty((T * k,), dtype=torch.int32, device=dev)
    B.moe_permute(cfg, st["idx"], st["offsets"], st["rows"], st["pos"], st["ws"])
    st["counts"] = torch.empty((E,), dtype=torch.int32, device=dev)
    B.moe_ep_expert_counts(cfg, st["offsets"], st["counts"])
    return st


def _peer_plan_dispatch(B, cfg, ep_size, rank, st, x, counts_all, bufs, ptrs, cap):
    E, dev = cfg.E, x.device
    st["exp_base"] = torch.empty((E,), dtype=torch.int32, device=dev)
    st["src_base"] = torch.empty((E,), dtype=torch.int32, device=dev)
    st["recv_offsets"] = torch.empty((E // ep_size + 1,), dtype=torch.int32, device=dev)
    st["recv_ident"] = torch.empty((cap,), dtype=torch.int32, device=dev)
    B.moe_ep_plan(cfg, ep_size, rank, counts_all, st["exp_base"], st["src_base"],
                  st["recv_offsets"], st["recv_ident"], cap, st["ws"])
    B.moe_ep_dispatch_peer(cfg, ep_size, rank, x, st["idx"], st["w"], st["offsets"], st["pos"],
                           st["exp_base"], st["src_base"], ptrs["x"], ptrs["w"], cap)


def _peer_experts(B, cfg, ep_size, rank, st, rows, buf, w13_local, w2_local):
    if rows == 0:
        return
    lc = local_config(cfg, rows, ep_size)
    ws = B.alloc_workspace(lc, device=buf["x"].device)
    ident = st["recv_ident"][:rows]
    B.moe_expert_ffn(lc, buf["x"][:rows], st["recv_offsets"], ident, ident, buf["w"][:rows],
                     w13_local, w2_local, None, None, buf["y"][:rows], None, ws)


def _peer_combine(B, cfg, ep_size, rank, st, x, w13s, w2s, ptrs, cap):
    ysh = None
    if cfg.n_shared > 0:
        ysh = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device=x.device)
        B.moe_shared_expert(cfg, x, w13s, w2s, ysh, st["ws"])
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=x.device)
    B.moe_ep_combine_peer(cfg, ep_size, rank, st["idx"], st["offsets"], st["pos"], st["exp_base"],
                          st["src_base"], ptrs["y"], ysh, out, cap)
    return out, st


def _rows_of(counts_all_host, rank, el):
    return int(counts_all_host[:, rank * el:(rank + 1) * el].sum())


def ep_forward_peer_virtual(cfg, xs, w_router, bias, w13, w2, w13s, w2s, binding=None):
    """N = len(xs) virtual ranks on one device with the peer-memory exchange:
    every rank's receive buffers are ordinary device buffers, addressed by
    the other ranks' kernels through the same pointer arrays a multi-GPU run
    fills with peer-mapped addresses.  Returns the N outputs."""
    if binding is None:
        from . import binding as B
    else:
        B = binding
    N, T, k, H, E = len(xs), cfg.T, cfg.k, cfg.H, cfg.E
    el = E // N
    dev = xs[0].device
    cap = T * k * N
    bufs = [{"x": torch.empty((cap, H), dtype=torch.bfloat16, device=dev),
             "w": torch.empty((cap,), dtype=torch.float32, device=dev),
             "y": torch.empty((cap, H), dtype=torch.float32, device=dev)} for _ in range(N)]
    ptrs = {key: torch.tensor([b[key].data_ptr() for b in bufs], dtype=torch.int64, device=dev)
            for key in ("x", "w", "y")}
    sts = [_peer_step_front(B, cfg, x, w_router, bias) for x in xs]
    counts_all = torch.stack([st["counts"] for st in sts])  # the all-gather
    for r in range(N):
        _peer_plan_dispatch(B, cfg, N, r, sts[r], xs[r], counts_all, bufs, ptrs, cap)
    host = counts_all.cpu()  # (one device: stream order is the barrier)
    for d in range(N):
        _peer_experts(B, cfg, N, d, sts[d], _rows_of(host, d, el), bufs[d],
                      w13[d * el:(d + 1) * el], w2[d * el:(d + 1) * el])
    return [_peer_combine(B, cfg, N, r, sts[r], xs[r], w13s, w2s, ptrs, cap)[0]
            for r in range(N)]


class PeerBuffers:
    """One rank's receive buffers in symmetric memory (every rank of the group
    maps every other rank's buffers over NVLink) and the device arrays of the
    ranks' addresses.  recv_cap rows: T * k * ep_size covers any routing."""

    def __init__(self, cfg, ep_size, group=None, device=None):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm
        group = group if group is not None else dist.group.WORLD
        dev = device or torch.device("cuda", torch.cuda.current_device())
        self.cap = cfg.T * cfg.k * ep_size
        shapes = {"x": ((self.cap, cfg.H), torch.bfloat16), "w": ((self.cap,), torch.float32),
                  "y": ((self.cap, cfg.H), torch.float32)}
        self.local, self.ptrs, self._handles = {}, {}, []
        for key, (shape, dt) in shapes.items():
            t = symm.empty(*shape, dtype=dt, device=dev)
            h = symm.rendezvous(t, group)
            self.local[key] = t
            self._handles.append(h)
            self.ptrs[key] = torch.tensor([h.get_buffer(r, shape, dt).data_ptr()
                                           for r in range(ep_size)], dtype=torch.int64, device=dev)


def ep_forward_peer(cfg, ep_rank, ep_size, x, w_router, bias, w13_local, w2_local, w13s, w2s,
                    bufs, group=None, binding=None):
    """One rank's layer output with the peer-memory exchange across ep_size
    GPUs of a process group: the counts are all-gathered (NCCL), the rows
    move by the library's peer stores and loads, and two barriers order the
    dispatch, the expert GEMMs and the combine across ranks.  bufs: this
    rank's PeerBuffers."""
    import torch.distributed as dist
    if binding is None:
        from . import binding as B
    else:
        B = binding
    el = cfg.E // ep_size
    st = _peer_step_front(B, cfg, x, w_router, bias)
    counts_all = torch.empty((ep_size, cfg.E), dtype=torch.int32, device=x.device)
    dist.all_gather_into_tensor(counts_all, st["counts"], group=group)
    _peer_plan_dispatch(B, cfg, ep_size, ep_rank, st, x, counts_all, bufs.local, bufs.ptrs,
                        bufs.cap)
    torch.cuda.current_stream().synchronize()
    dist.barrier(group=group)          # every rank's rows have landed
    rows = _rows_of(counts_all.cpu(), ep_rank, el)
    _peer_experts(B, cfg, ep_size, ep_rank, st, rows, bufs.local, w13_local, w2_local)
    torch.cuda.current_stream().synchronize()
    dist.barrier(group=group)          # every rank's expert outputs are written
    out, _ = _peer_combine(B, cfg, ep_size, ep_rank, st, x, w13s, w2s, bufs.ptrs, bufs.cap)
    torch.cuda.current_stream().synchronize()
    dist.barrier(group=group)          # no rank reuses its buffers while others read them
    return out
