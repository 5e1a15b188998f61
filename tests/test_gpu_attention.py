"""The sparse-attention consumer on the GPU vs its CPU oracle, through the C
ABI, on the indexer's own selections (needs a B200).

The GPU multiplies bf16 on the tensor cores with fp32 accumulation and rounds
the softmax probabilities to bf16 before P.V, so outputs are held to 1e-2 of
the largest |value| among the selected keys of the row, element by element.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import attention as attn_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    from lightning_indexer_top_02_b200.build import build
    build()
    L.load_library()
    return L


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def attn_case(L, *, B, S, T, HA, Dk, Dv, topk, m=4, seed=0, shared=False, rows=None,
              idx_override=None, scale=None):
    """Indexer selection on random inputs, then the attention over it."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    wl = workloads.Workload("att", B=B, S=S, T=T, H=16, d=64, m=m, topk=topk, seed=seed)
    inp = workloads.make_inputs(wl, device="cuda")
    if idx_override is None:
        idx, _ = L.indexer_topk(inp["q"], inp["w"], inp["k"], m=m, topk=topk)
    else:
        idx = idx_override
    qa = torch.randn((B, S, HA, Dk), generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn((B, T, Dk), generator=g, device="cuda").to(torch.bfloat16)
    vc = None if shared else torch.randn((B, T, Dv), generator=g, device="cuda").to(torch.bfloat16)
    scale = Dk ** -0.5 if scale is None else scale
    out = L.sparse_attention(qa, kc, idx, scale=scale, v=vc, dv=Dv)
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    kb = bits(kc)
    vb = kb if shared else bits(vc)
    ref = attn_oracle.sparse_attention(bits(qa), kb, vb, idx.cpu().numpy(), B=B, S=S, T=T, HA=HA,
                                       Dk=Dk, Dv=Dv, topk=topk, scale=scale,
                                       ld_v=Dk if shared else Dv, rows=rows)
    got = out.cpu().numpy().reshape(B * S, HA, Dv)
    if rows is not None:
        got = got[rows]
    idx_np = idx.cpu().numpy().reshape(B * S, topk)
    vals = (kc if shared else vc).float().cpu().numpy()
    sel_rows = np.arange(B * S) if rows is None else rows
    for n, r in enumerate(sel_rows):
        b = r // S
        sel = idx_np[r][(idx_np[r] >= 0) & (idx_np[r] < T)]
        vmax = np.abs(vals[b, sel, :Dv]).max() if len(sel) else 1.0
        err = np.abs(got[n] - ref[n]).max()
        assert err <= 1e-2 * vmax, f"row {r}: max error {err:.3g} vs values up to {vmax:.3g}"
    return got, ref


def test_attention_small(lib):
    """Causal selections of all sizes (early queries select fewer keys than
    topk, the rest a full 2048... here 256), several batches, HA=64, D=128."""
    attn_case(lib, B=2, S=300, T=500, HA=64, Dk=128, Dv=128, topk=256, seed=1)


def test_attention_dims(lib):
    for Dk, Dv, HA in ((64, 64, 128), (128, 64, 16), (192, 128, 1), (256, 256, 32),
                       (128, 192, 40), (192, 192, 100)):
        attn_case(lib, B=1, S=70, T=300, HA=HA, Dk=Dk, Dv=Dv, topk=200, seed=Dk + Dv + HA)


def test_attention_shared_latent_cache(lib):
    """Values read as the first Dv elements of each key row (ld_v = Dk)."""
    attn_case(lib, B=2, S=90, T=400, HA=128, Dk=192, Dv=128, topk=300, seed=5, shared=True)


def test_attention_full_topk_rows(lib):
    """Late queries of a long causal prefill select a full top-2048 (16 tiles
    of 128 keys): sampled rows."""
    rows = np.array([0, 5, 4000, 8191, 8100, 6000], np.int64)
    attn_case(lib, B=1, S=8192, T=8192, HA=64, Dk=128, Dv=128, topk=2048, m=1, seed=7,
              rows=rows)


def test_attention_padding_and_empty_rows(lib):
    """Rows with no selected key give zeros; padding slots (-1 or >= T) are
    ignored wherever they stand, including between keys and in whole tiles."""
    B, S, T, topk = 1, 8, 300, 390
    idx = torch.full((B, S, topk), -1, dtype=torch.int32, device="cuda")
    idx[0, 1, :1] = 17
    idx[0, 2, :129] = torch.arange(129, dtype=torch.int32, device="cuda")
    idx[0, 3, :130] = torch.arange(130, 260, dtype=torch.int32, device="cuda")
    idx[0, 5, 0:390:3] = torch.arange(0, 260, 2, dtype=torch.int32, device="cuda")  # holes
    idx[0, 5, 7] = T + 5                                                           # out of range
    idx[0, 6, 300] = 42                                    # one key in the third tile only
    idx[0, 7, 128:256] = torch.arange(128, dtype=torch.int32, device="cuda")       # empty first tile
    got, ref = attn_case(lib, B=B, S=S, T=T, HA=8, Dk=64, Dv=64, topk=topk, seed=9,
                         idx_override=idx)
    assert np.all(got[0] == 0.0) and np.all(got[4] == 0.0)
    assert np.any(got[5] != 0.0) and np.any(got[6] != 0.0)


def test_attention_large_logits_rescale(lib):
    """A large scale makes later tiles exceed the running maximum by more
    than 2^8, which rescales O in tensor memory."""
    attn_case(lib, B=1, S=64, T=2048, HA=32, Dk=128, Dv=128, topk=1024, m=1, seed=11, scale=2.0)


def test_attention_negative_scale_and_odd_heads(lib):
    """A negative scale (the softmax then favours the smallest dot products)
    and head counts that fill a TMEM lane quarter only in part, on both sides
    of 64 heads (two warps share a row's keys up to 64 heads)."""
    for HA, seed in ((48, 21), (96, 22)):
        attn_case(lib, B=1, S=150, T=700, HA=HA, Dk=128, Dv=128, topk=300, seed=seed, scale=-0.09)
