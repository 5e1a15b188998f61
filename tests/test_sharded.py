"""Key-sharded selection (keys split across GPUs, one all-gather, a merge).

CPU: two ``gloo`` ranks run the orchestration with the oracle standing in for
each rank's selection and a sort for the merge, which checks the key ranges,
the shifted query positions (the causal rule over absolute key positions)
and the exchange; the result must equal the oracle over all keys.
GPU: the ranges run one after another in one process through the CUDA
selection and csa_merge_topk; with integer inputs the merge must equal the
oracle over all keys bit for bit, and the relaxed mode's recall is measured.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads

WL = workloads.Workload("shard", B=2, S=96, T=700, H=8, d=32, m=4, topk=40, values="integer", seed=77)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_select(q, w, k_range, *, start, T_total, m, k_local, k_scale, causal, mode, q_offset):
    """The oracle over one key range, shifted like the CUDA path."""
    from lightning_indexer_top_02_b200 import sharded
    S = q.shape[1]
    qo = sharded.local_q_offset(S, T_total, m, start, q_offset)
    qb, wb, kb, _ = workloads.as_numpy_bits({"q": q, "w": w, "k": k_range, "k_scale": None})
    B, _, H, d = q.shape
    idx, sc, _, _ = oracle.topk(qb, wb, kb, None, B=B, S=S, T=k_range.shape[1], H=H, d=d, m=m,
                                topk=k_local, causal=causal, mode=mode, q_offset=qo)
    return (torch.from_numpy(idx.reshape(B, S, k_local)),
            torch.from_numpy(sc.reshape(B, S, k_local)))


def _cpu_merge(idx_all, sc_all, offsets, topk):
    """Top-k of the union by (score descending, index ascending)."""
    idx = np.concatenate([np.where(i.numpy() >= 0, i.numpy() + o, -1) for i, o in zip(idx_all, offsets)], -1)
    sc = np.concatenate([s.numpy() for s in sc_all], -1)
    shp = idx.shape[:-1]
    idx = idx.reshape(-1, idx.shape[-1])
    sc = sc.reshape(-1, sc.shape[-1])
    out_i = np.full((idx.shape[0], topk), -1, np.int32)
    out_s = np.full((idx.shape[0], topk), -np.inf, np.float32)
    for r in range(idx.shape[0]):
        cand = sorted((-float(s), int(i)) for i, s in zip(idx[r], sc[r]) if i >= 0)[:topk]
        out_i[r, :len(cand)] = [c[1] for c in cand]
        out_s[r, :len(cand)] = [-c[0] for c in cand]
    return out_i.reshape(shp + (topk,)), out_s.reshape(shp + (topk,))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from lightning_indexer_top_02_b200 import sharded
        inp = workloads.make_inputs(WL)
        start, end = sharded.shard_range(WL.T, world, rank)
        idx, sc = sharded.sharded_indexer_topk(
            inp["q"], inp["w"], inp["k"][:, start:end].contiguous(), start=start, T_total=WL.T,
            m=WL.m, topk=WL.topk, select_fn=_cpu_select, merge_fn=_cpu_merge)
        out[rank] = (idx, sc)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_oracle():
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    inp = workloads.make_inputs(WL)
    q, w, k, _ = workloads.as_numpy_bits(inp)
    ri, rs, _, _ = oracle.topk(q, w, k, None, B=WL.B, S=WL.S, T=WL.T, H=WL.H, d=WL.d, m=WL.m,
                               topk=WL.topk)
    for rank in range(world):
        gi, gs = out[rank]
        assert np.array_equal(gi.reshape(ri.shape), ri)
        assert np.array_equal(gs.reshape(rs.shape).view(np.uint32), rs.view(np.uint32))


def test_shard_ranges_cover_the_keys():
    from lightning_indexer_top_02_b200 import sharded
    for T, world in ((700, 2), (131072, 8), (5, 3), (1, 4)):
        ranges = [sharded.shard_range(T, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    # the shifted offset keeps the causal rule over absolute positions
    assert sharded.local_q_offset(S=64, T_total=131072, m=4, start=65536) == 131072 * 4 - 64 - 65536 * 4


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3, 4])
def test_sharded_merge_on_gpu(world):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    from lightning_indexer_top_02_b200 import sharded
    from lightning_indexer_top_02_b200.build import build
    from parity import check_exact
    build()
    L.load_library()
    wl = workloads.Workload("shg", B=3, S=64, T=9000, H=64, d=128, m=4, topk=512,
                            values="integer", seed=90 + world)
    inp = workloads.make_inputs(wl, device="cuda")
    lists_i, lists_s, offs = [], [], []
    for r in range(world):
        start, end = sharded.shard_range(wl.T, world, r)
        i, s = sharded.select_local(inp["q"], inp["w"], inp["k"][:, start:end].contiguous(),
                                    start=start, T_total=wl.T, m=wl.m, k_local=wl.topk)
        lists_i.append(i)
        lists_s.append(s)
        offs.append(start)
    gi, gs = sharded.merge_topk(lists_i, lists_s, offs, wl.topk)
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    q, w, k, _ = workloads.as_numpy_bits(inp)
    ri, rs, _, _ = oracle.topk(q, w, k, None, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                               topk=wl.topk)
    check_exact(gi.cpu().numpy().reshape(-1, wl.topk), gs.cpu().numpy().reshape(-1, wl.topk),
                ri, rs, label=f"{world} key shards")


@pytest.mark.gpu
def test_relaxed_local_k_recall():
    """Random-normal inputs over 4 key ranges: exact local k reproduces the
    unsharded selection; keeping only k/4 per range (a quarter of the
    exchange) loses the keys a range holds beyond its quarter -- the recall
    against the exact answer is measured and recorded."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    from lightning_indexer_top_02_b200 import sharded
    wl = workloads.Workload("shr", B=4, S=32, T=32768, H=64, d=128, m=4, topk=2048, seed=95)
    inp = workloads.make_inputs(wl, device="cuda")
    full, _ = L.indexer_topk(inp["q"], inp["w"], inp["k"], m=wl.m, topk=wl.topk)
    world = 4
    for k_local, bar in ((wl.topk, 1.0), (wl.topk // 4, 0.5)):
        li, ls, offs = [], [], []
        for r in range(world):
            a, b = sharded.shard_range(wl.T, world, r)
            i, s = sharded.select_local(inp["q"], inp["w"], inp["k"][:, a:b].contiguous(), start=a,
                                        T_total=wl.T, m=wl.m, k_local=k_local)
            li.append(i)
            ls.append(s)
            offs.append(a)
        gi, _ = sharded.merge_topk(li, ls, offs, wl.topk)
        torch.cuda.synchronize()
        g = gi.cpu().numpy().reshape(-1, wl.topk)
        f = full.cpu().numpy().reshape(-1, wl.topk)
        rec = np.array([len(np.intersect1d(g[r][g[r] >= 0], f[r][f[r] >= 0])) / max(1, np.sum(f[r] >= 0))
                        for r in range(g.shape[0])])
        print(f"{world} key ranges, local k {k_local}: recall mean {rec.mean():.4f} min {rec.min():.4f}")
        if k_local == wl.topk:
            assert np.array_equal(g, f), "exact local k must reproduce the unsharded selection"
        assert rec.min() >= bar
