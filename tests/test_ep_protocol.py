"""The expert-parallel protocol (sigmoid_top_routing_warp_b200/ep.py) on CPU:
world size 2 over gloo, with the compute steps done by the fp64 oracle
instead of the library's kernels.  What is checked is the protocol: which
rows go to which rank, the exchanged counts, the local expert indices, the
return path in send order and the final combine.  Each rank's output must
equal the oracle's whole layer (every expert, shared included) on that
rank's own tokens, to fp64 rounding."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleSteps:
    """The steps of ep.CudaSteps computed by the oracle on the host (fp64
    rows travel as float64 tensors)."""

    def __init__(self, O):
        self.O = O

    def _cfg(self, cfg, **kw):
        d = dict(T=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.n_shared,
                 n_group=cfg.n_group, topk_group=cfg.topk_group, group_topn=cfg.group_topn,
                 norm_topk_prob=cfg.norm_topk_prob,
                 routed_scaling_factor=cfg.routed_scaling_factor)
        d.update(kw)
        return self.O.Config(**d)

    def route_and_pack(self, cfg, ep_size, x, w_router, bias):
        O = self.O
        oc = self._cfg(cfg)
        L = O.router_logits(oc, u16(x), u16(w_router)).astype(np.float32)
        idx, w, _ = O.route(oc, L, bias.numpy())
        offsets, rows, pos = O.permute(oc, idx)
        T, k, H, el = cfg.T, cfg.k, cfg.H, cfg.E // ep_size
        xf = x.float().numpy().astype(np.float64)
        x_send = np.zeros((T * k, H))
        w_send = np.zeros(T * k)
        e_send = np.zeros(T * k, np.int32)
        for s in range(T * k):
            r, e = pos[s], idx.flat[s]
            x_send[r] = xf[s // k]
            w_send[r] = w.flat[s]
            e_send[r] = e - (e // el) * el
        counts = [int(offsets[(d + 1) * el] - offsets[d * el]) for d in range(ep_size)]
        return {"idx": idx, "w": w, "pos": pos, "x_send": torch.from_numpy(x_send),
                "w_send": torch.from_numpy(w_send), "e_send": torch.from_numpy(e_send),
                "send_counts": torch.tensor(counts, dtype=torch.int64)}

    def experts(self, cfg, ep_size, x_recv, w_recv, e_recv, w13_local, w2_local):
        O = self.O
        R = x_recv.shape[0]
        if R == 0:
            return torch.zeros((0, cfg.H), dtype=torch.float64)
        xb = u16(x_recv.to(torch.float32).to(torch.bfloat16))  # exact: the rows are bf16 values
        oc = self._cfg(cfg, T=R, E=cfg.E // ep_size, k=1, n_shared=0)
        y = O.layer(oc, xb, e_recv.numpy().reshape(R, 1).astype(np.int32),
                    w_recv.numpy().reshape(R, 1).astype(np.float32), u16(w13_local),
                    u16(w2_local), None, None)
        return torch.from_numpy(y)

    def shared_and_combine(self, cfg, st, x, y_ret, w13s, w2s):
        O = self.O
        T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
        # the shared expert alone: one routed expert of weight 0 beside it
        oc = self._cfg(cfg, E=1, k=1, n_group=1, topk_group=1)
        ysh = O.layer(oc, u16(x), np.zeros((T, 1), np.int32), np.zeros((T, 1), np.float32),
                      np.zeros((1, 2 * I, H), np.uint16), np.zeros((1, H, I), np.uint16),
                      u16(w13s), u16(w2s))
        yr = y_ret.numpy()
        out = ysh.copy()
        for t in range(T):
            for j in range(k):
                out[t] += yr[st["pos"][t * k + j]]
        return out


def _rank(rank, world, port, q, skew=False):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from oracle import oracle as O
    from sigmoid_top_routing_warp_b200 import ep
    from sigmoid_top_routing_warp_b200 import workloads as W
    from sigmoid_top_routing_warp_b200.binding import MoeConfig
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.Workload("ep_tiny", T=40, H=128, E=32, k=4, I=128, n_shared=1, seed=0)
        inp = W.make_inputs(wl, device="cpu")  # the same weights on every rank
        if skew:  # every choice among rank 0's experts: rank 1 receives no rows
            bias = torch.full((wl.E,), -20.0)
            bias[: wl.E // world] = 20.0
            inp = dict(inp, bias=bias)
        g = torch.Generator().manual_seed(100 + rank)
        x = (torch.randn((wl.T, wl.H), generator=g)).to(torch.bfloat16)  # this rank's tokens
        cfg = MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=1)
        el = wl.E // world
        mine = slice(rank * el, (rank + 1) * el)
        out = ep.ep_forward(cfg, rank, world, x, inp["w_router"], inp["bias"], inp["w13"][mine],
                            inp["w2"][mine], inp["w13s"], inp["w2s"],
                            exchange=ep.DistExchange(), steps=OracleSteps(O))
        # the oracle's whole layer on this rank's tokens
        oc = O.Config(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=1)
        L = O.router_logits(oc, u16(x), u16(inp["w_router"])).astype(np.float32)
        idx, w, _ = O.route(oc, L, inp["bias"].numpy())
        ref = O.layer(oc, u16(x), idx, w, u16(inp["w13"]), u16(inp["w2"]), u16(inp["w13s"]),
                      u16(inp["w2s"]))
        err = float(np.abs(out - ref).max() / np.abs(ref).max())
        # rows really crossed: both ranks' experts served this rank's tokens
        owners = np.unique(idx // el)
        q.put((rank, err, owners.tolist()))
    finally:
        dist.destroy_process_group()


def run_two_ranks(skew):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q, skew)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    return sorted(q.get(timeout=5) for _ in range(2))


def test_expert_parallel_protocol_two_ranks_gloo():
    for rank, err, owners in run_two_ranks(skew=False):
        assert err < 1e-12, (rank, err)
        assert owners == [0, 1], (rank, owners)


def test_expert_parallel_protocol_empty_exchanges_gloo():
    """Every choice on rank 0's experts: rank 1 sends all its rows to rank 0,
    rank 0 sends none, and rank 1 runs its expert step on zero rows."""
    for rank, err, owners in run_two_ranks(skew=True):
        assert err < 1e-12, (rank, err)
        assert owners == [0], (rank, owners)
