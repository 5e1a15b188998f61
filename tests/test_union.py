"""OR-union of several layers' selections: the oracle pinned on the CPU, the
CUDA kernel against it on the GPU (bit-exact: integer work)."""
import numpy as np
import pytest
import torch

from oracle import union as U


def test_union_oracle_pins():
    # a hand-worked row: {5, 2, 9} u {9, 1} u {} = 1 2 5 9
    a = np.array([[5, 2, 9, -1]]); b = np.array([[9, 1, -1, -1]]); c = np.full((1, 4), -1)
    out, cnt = U.union_selections([a, b, c], T=10, cap=12)
    assert cnt.tolist() == [4] and out[0, :5].tolist() == [1, 2, 5, 9, -1]
    # keys outside [0, T) are padding; cap keeps the smallest keys
    out, cnt = U.union_selections([np.array([[3, 10, 11, 0]])], T=10, cap=1)
    assert cnt.tolist() == [1] and out.tolist() == [[0]]
    # invariants on random rows: every input key is in, strictly increasing, size bound
    rng = np.random.default_rng(3)
    lists = [np.where(rng.random((20, 30)) < 0.2, -1, rng.integers(0, 50, (20, 30))) for _ in range(3)]
    out, cnt = U.union_selections(lists, T=50, cap=90)
    for r in range(20):
        got = out[r, :cnt[r]]
        assert np.all(np.diff(got) > 0) and np.all(out[r, cnt[r]:] == -1)
        for x in lists:
            assert set(x[r][x[r] >= 0].tolist()) <= set(got.tolist())
        assert cnt[r] <= sum(int(np.sum(x[r] >= 0)) for x in lists)
    # the union of a list with itself is its own distinct keys
    same, n = U.union_selections([lists[0], lists[0]], T=50, cap=30)
    for r in range(20):
        assert same[r, :n[r]].tolist() == sorted(set(lists[0][r][lists[0][r] >= 0].tolist()))


@pytest.mark.gpu
def test_union_gpu_matches_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    import workloads
    from lightning_indexer_top_02_b200.build import build
    build()
    L.load_library()
    # three "layers": gated selections of three indexers over one key cache
    wl = workloads.Workload("u", B=4, S=8, T=5000, H=64, d=128, m=4, topk=512, seed=31)
    sels = []
    k = None
    for layer in range(3):
        inp = workloads.make_inputs(wl, device="cuda", seed=31 + layer)
        if k is None:
            k = inp["k"]
        idx, _ = L.indexer_topk(inp["q"], inp["w"], k, m=wl.m, topk=wl.topk, mode=L.CSA_MODE_GATE)
        sels.append(idx)
    for cap in (3 * wl.topk, 700):
        out, cnt = L.union_selections(sels, T=wl.T, cap=cap)
        torch.cuda.synchronize()
        ref, rcnt = U.union_selections([s.cpu().numpy() for s in sels], T=wl.T, cap=cap)
        assert np.array_equal(cnt.cpu().numpy(), rcnt)
        assert np.array_equal(out.cpu().numpy(), ref)
    # a large key range (bitmap of 400,000 keys) and a single list
    big = torch.randint(-1, 400000, (3, 2048), dtype=torch.int32, device="cuda")
    out, cnt = L.union_selections([big], T=400000)
    torch.cuda.synchronize()
    ref, rcnt = U.union_selections([big.cpu().numpy()], T=400000, cap=2048)
    assert np.array_equal(out.cpu().numpy(), ref) and np.array_equal(cnt.cpu().numpy(), rcnt)


@pytest.mark.gpu
def test_layer_schedules_match_sequential():
    """The MLI schedule (indexer of layer l on a second stream, read by layer
    l+1) and the IndexCache schedule give exactly the selections and outputs
    of running the same calls one after another."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    import workloads
    from lightning_indexer_top_02_b200 import schedule
    from lightning_indexer_top_02_b200.build import build
    build()
    L.load_library()
    B, S, T, topk, m = 4, 2, 3000, 256, 4
    wl = workloads.Workload("sch", B=B, S=S, T=T, H=64, d=128, m=m, topk=topk, seed=41)
    g = torch.Generator(device="cuda").manual_seed(42)
    layers = []
    for l in range(5):
        inp = workloads.make_inputs(wl, device="cuda", seed=41 + l)
        layers.append(schedule.Layer(
            iq=inp["q"], iw=inp["w"], ik=inp["k"],
            aq=torch.randn((B, S, 32, 128), generator=g, device="cuda").to(torch.bfloat16),
            kc=torch.randn((B, T, 128), generator=g, device="cuda").to(torch.bfloat16),
            scale=128 ** -0.5))
    outs, used = schedule.decode_layers(layers, m=m, topk=topk, schedule="mli")
    torch.cuda.synchronize()
    own = [L.indexer_topk(x.iq, x.iw, x.ik, m=m, topk=topk)[0] for x in layers]
    for l, x in enumerate(layers):
        want_sel = own[0] if l == 0 else own[l - 1]
        assert torch.equal(used[l], want_sel), f"layer {l}: wrong selection"
        want = L.sparse_attention(x.aq, x.kc, want_sel, scale=x.scale)
        assert torch.equal(outs[l], want), f"layer {l}: output differs"
    outs, used = schedule.decode_layers(layers, m=m, topk=topk, schedule="indexcache", refresh=2)
    torch.cuda.synchronize()
    for l in range(len(layers)):
        assert torch.equal(used[l], own[l - l % 2])
