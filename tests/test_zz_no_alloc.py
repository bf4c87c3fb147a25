"""moe_permute_noalloc: the dispatch permutation for callers that cannot
allocate device memory (a plugin handed only its input and output buffers, a
runtime whose memory planner owns all of HBM).  Its scratch is a fixed array
inside the library instead of a caller workspace.  Checked through the C ABI
against moe_permute (which takes a workspace) and against the oracle's stable
counting sort, on two calls in a row, on the single-block and the multi-block
paths, for an empty batch and for the size limit.

Kept in a file of its own that pytest collects last; it also passes alone in
a fresh process (the first call does the per-device set-up).
"""
import numpy as np
import pytest
import torch

from helpers import oracle_cfg
from oracle import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    assert torch.cuda.is_available()
    return binding


def routing(T, E, k, seed, skew=False):
    g = torch.Generator().manual_seed(seed)
    if skew:  # heavy experts, so some segments span many chunks
        p = torch.arange(1, E + 1, dtype=torch.float64) ** -1.1
        return torch.stack([torch.multinomial(p, k, replacement=False, generator=g)
                            for _ in range(T)]).int()
    return torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).int()


def permute_both(B, cfg, idx):
    dev = "cuda"
    n = max(cfg.T * cfg.k, 1)  # the entry points take non-NULL rows / pos even when T = 0
    ref = [torch.full((cfg.E + 1,), -7, dtype=torch.int32, device=dev),
           torch.full((n,), -7, dtype=torch.int32, device=dev),
           torch.full((n,), -7, dtype=torch.int32, device=dev)]
    got = [torch.full_like(t, -9) for t in ref]
    ws = B.alloc_workspace(cfg)
    B.moe_permute(cfg, idx, *ref, ws)
    B.moe_permute_noalloc(cfg, idx, *got)
    torch.cuda.synchronize()
    return ref, got


@pytest.mark.parametrize("T,E,k", [(64, 256, 8), (8192, 256, 8), (16384, 128, 6), (300, 64, 6)])
def test_noalloc_matches_workspace_permute_twice(B, T, E, k):
    cfg = B.MoeConfig(T=T, H=512, E=E, k=k, I=128)
    for call, seed in enumerate((11, 12)):  # two calls in a row, different routings
        idx = routing(T, E, k, seed + T, skew=(call == 1)).cuda()
        ref, got = permute_both(B, cfg, idx)
        for name, r, g in zip(("offsets", "rows", "pos"), ref, got):
            assert torch.equal(r, g), "call %d: %s differs" % (call, name)
        offs = got[0].cpu().numpy()
        assert offs[0] == 0 and offs[-1] == T * k and (np.diff(offs) >= 0).all()
        # the definition: a stable counting sort of the slots by expert
        for name, o, g in zip(("offsets", "rows", "pos"), O.permute(oracle_cfg(cfg), idx.cpu().numpy()),
                              got):
            assert (g.cpu().numpy() == o).all(), "call %d: %s differs from the oracle" % (call, name)


def test_noalloc_empty_batch_writes_zero_offsets(B):
    """T = 0: offsets[0..E] are all zero, as moe_permute writes them."""
    cfg = B.MoeConfig(T=0, H=512, E=64, k=6, I=128)
    idx = torch.zeros((1, cfg.k), dtype=torch.int32, device="cuda")
    ref, got = permute_both(B, cfg, idx)
    assert torch.equal(ref[0], got[0])
    assert (got[0] == 0).all()


def test_noalloc_rejects_sizes_beyond_its_scratch(B):
    # E=1024 with T*k = 2048*65 slots needs 65 chunks x 1024 experts > 65536 entries
    cfg = B.MoeConfig(T=2048 * 65 // 8, H=512, E=1024, k=8, I=128)
    idx = torch.zeros((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    out = [torch.empty((cfg.E + 1,), dtype=torch.int32, device="cuda"),
           torch.empty((cfg.T * cfg.k,), dtype=torch.int32, device="cuda"),
           torch.empty((cfg.T * cfg.k,), dtype=torch.int32, device="cuda")]
    with pytest.raises(B.MoeError) as ei:
        B.moe_permute_noalloc(cfg, idx, *out)
    assert ei.value.status == B.MOE_ERR_UNSUPPORTED
    assert "scratch" in B.get_last_error()
