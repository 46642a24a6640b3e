"""Expert-parallel layer: the dispatch plan, and the whole forward on two and three gloo CPU
ranks (experts split over the ranks, every rank with its own tokens) against the FP64 oracle's
single-process layer; on a GPU, the same layer through libmoe on a one-rank NCCL group."""
import os
import socket

import numpy as np
import pytest

import moe_inputs as mi
from mixture_experts_gemv_b200.expert_parallel import dispatch_plan, inverse_order


def test_dispatch_plan_is_a_stable_sort_by_destination():
    ids = np.array([[5, 0, 3], [1, 7, 4], [6, 2, 0]])
    order, dest, counts = dispatch_plan(ids, E=8, world=2)     # ranks own experts 0-3, 4-7
    flat = ids.reshape(-1)
    assert list(counts) == [5, 4]
    assert list(dest) == [0] * 5 + [1] * 4
    assert list(order) == [1, 2, 3, 7, 8, 0, 4, 5, 6]         # slot order kept inside a destination
    assert (flat[order[:5]] < 4).all() and (flat[order[5:]] >= 4).all()
    inv = inverse_order(order)
    assert np.array_equal(order[inv], np.arange(9)) and np.array_equal(inv[order], np.arange(9))
    with pytest.raises(ValueError):
        dispatch_plan(ids, E=8, world=3)
    with pytest.raises(ValueError):
        dispatch_plan(np.array([[8]]), E=8, world=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, E, d, f, k, T, q):
    import torch
    import torch.distributed as dist
    from ep_cpu_ops import CpuOracleOps
    from mixture_experts_gemv_b200.expert_parallel import ExpertParallelLayer
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lw = mi.make_layer(seed=70, d=d, f=f, E=E)
        x = mi.make_tokens(80 + rank, T + rank, d)          # ranks hold different numbers of tokens
        el = E // world
        sl = slice(rank * el, (rank + 1) * el)
        layer = ExpertParallelLayer(E, d, f, k, CpuOracleOps())
        out = layer.forward(torch.from_numpy(x.view(np.int16)), torch.from_numpy(lw.router_w),
                            torch.from_numpy(lw.router_scale), torch.from_numpy(lw.gate_up[sl]),
                            torch.from_numpy(lw.down[sl]), torch.from_numpy(lw.expert_scale[sl]), x.shape[0])
        ref, _, _, _ = oracle.moe_layer(x, lw.router_w, lw.router_scale, lw.gate_up, lw.down, lw.expert_scale, k)
        err = float(np.max(np.abs(out.numpy() - ref)) / np.max(np.abs(ref)))
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_forward_on_gloo_ranks_matches_the_layer(world):
    import torch.multiprocessing as tmp
    E, d, f, k, T = 12, 64, 32, 3, 5
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, E, d, f, k, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err in res:
        assert err <= 1e-12, (rank, err)


@pytest.mark.gpu
def test_expert_parallel_forward_on_one_gpu_rank():
    """One NCCL rank holding every expert: the dispatch, the experts-only path, the return and
    the combine through libmoe, against the oracle (2 tokens: 16 expert rows, the GEMV path at
    1e-3; 8 and 40 tokens: 64 and 320 rows, the grouped GEMM at 2e-2)."""
    import torch
    import torch.distributed as dist
    import oracle
    import mixture_experts_gemv_b200 as moe
    from mixture_experts_gemv_b200.expert_parallel import ExpertParallelLayer, LibmoeOps
    from gpu_util import dev, ensure_init, rel_err
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        E, d, f, k = 32, 512, 128, 4
        lw = mi.make_layer(seed=71, d=d, f=f, E=E)
        for T, tol in ((2, 1e-3), (8, 2e-2), (40, 2e-2)):
            ensure_init(T, d, f, E, k)
            moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
            x = mi.make_tokens(90 + T, T, d)
            layer = ExpertParallelLayer(E, d, f, k, LibmoeOps(torch.device("cuda", 0)))
            out = layer.forward(dev(x), dev(lw.router_w), dev(lw.router_scale), dev(lw.gate_up), dev(lw.down),
                                dev(lw.expert_scale), T)
            moe.moe_debug_check()
            ref, _, _, flags = oracle.moe_layer(x, lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                                                lw.expert_scale, k)
            ok = (flags & 1) == 0
            assert rel_err(out.cpu().numpy()[ok], ref[ok]) <= tol
    finally:
        dist.destroy_process_group()
