"""Pins of the sparse-attention oracle (CPU only).

The oracle writes out softmax attention over the selected keys; these tests
fix it to values the mathematics determines independently of its own code:
a single selected key returns that key's value row exactly; zero queries give
the plain mean of the selected value rows; two keys whose logits differ by a
known amount give the logistic mix of their values; the selection's slot order
and its -1 padding do not matter; every output lies in the convex hull of the
selected values; a very large scale turns softmax into the argmax; values that
are a prefix of each key row (one shared latent cache) read the right
elements.  A planted mistake in a copy of the oracle must fail one of them.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import attention as A

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def bf16_bits(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def bf16_round(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy() \
        .astype(np.float64)


def rand_case(rng, B=2, S=3, T=40, HA=4, Dk=16, Dv=8, topk=12):
    qa = bf16_round(rng.standard_normal((B, S, HA, Dk)))
    kc = bf16_round(rng.standard_normal((B, T, Dk)))
    vc = bf16_round(rng.standard_normal((B, T, Dv)))
    idx = np.stack([np.stack([rng.choice(T, topk, replace=False) for _ in range(S)])
                    for _ in range(B)]).astype(np.int32)
    return qa, kc, vc, idx


def run(orc, qa, kc, vc, idx, scale, ld_v=None, rows=None):
    B, S, HA, Dk = qa.shape
    T = kc.shape[1]
    Dv = vc.shape[-1] if ld_v is None else (vc.shape[-1] if vc is not kc else vc.shape[-1])
    return orc.sparse_attention(bf16_bits(qa), bf16_bits(kc), bf16_bits(vc), idx, B=B, S=S, T=T,
                                HA=HA, Dk=Dk, Dv=Dv, topk=idx.shape[-1], scale=scale, ld_v=ld_v,
                                rows=rows)


@pytest.fixture(scope="module")
def orc():
    return A.default()


def all_pins(orc):
    rng = np.random.default_rng(7)
    # 1. one selected key (the rest padding): the output is that key's value row
    qa, kc, vc, idx = rand_case(rng)
    one = np.full_like(idx, -1)
    one[..., 3] = idx[..., 0]
    o = run(orc, qa, kc, vc, one, 0.125).reshape(qa.shape[0], qa.shape[1], qa.shape[2], -1)
    for b in range(qa.shape[0]):
        for i in range(qa.shape[1]):
            assert np.array_equal(o[b, i], np.broadcast_to(vc[b, idx[b, i, 0]], o[b, i].shape)), \
                "one key: output != its value row"
    # 2. zero queries: every selected key weighs the same
    z = run(orc, np.zeros_like(qa), kc, vc, idx, 0.3).reshape(o.shape[0], o.shape[1], o.shape[2], -1)
    for b in range(qa.shape[0]):
        for i in range(qa.shape[1]):
            mean = vc[b, idx[b, i]].mean(axis=0)
            assert np.allclose(z[b, i], mean[None, :], rtol=0, atol=1e-12), "zero query: not the mean"
    # 3. two keys, logits scale*a*b1 and scale*a*b2 along one axis: logistic mix
    Dk, Dv, T = 8, 4, 6
    qa2 = np.zeros((1, 1, 1, Dk))
    qa2[..., 2] = 1.5
    kc2 = np.zeros((1, T, Dk))
    kc2[0, 1, 2] = 2.0
    kc2[0, 4, 2] = -0.5
    vc2 = bf16_round(np.arange(T * Dv, dtype=np.float64).reshape(1, T, Dv) / 7.0)
    idx2 = np.array([[[4, -1, 1]]], np.int32)
    scale = 0.75
    o2 = run(orc, qa2, kc2, vc2, idx2, scale)[0, 0]
    delta = scale * 1.5 * (2.0 - (-0.5))
    p1 = 1.0 / (1.0 + np.exp(-delta))
    assert np.allclose(o2, p1 * vc2[0, 1] + (1 - p1) * vc2[0, 4], rtol=0, atol=1e-12), \
        "two keys: not the logistic mix"
    # 4. slot order and padding do not matter
    qa, kc, vc, idx = rand_case(rng)
    base = run(orc, qa, kc, vc, idx, 0.2)
    perm = idx[..., ::-1].copy()
    padded = np.concatenate([np.full(idx.shape[:-1] + (3,), -1, np.int32), idx], axis=-1)
    assert np.allclose(run(orc, qa, kc, vc, perm, 0.2), base, rtol=0, atol=1e-12), "order matters"
    assert np.allclose(run(orc, qa, kc, vc, padded, 0.2), base, rtol=0, atol=1e-12), "padding read"
    # 5. convex hull of the selected values, per output element
    o5 = base.reshape(qa.shape[0], qa.shape[1], qa.shape[2], -1)
    for b in range(qa.shape[0]):
        for i in range(qa.shape[1]):
            sel = vc[b, idx[b, i]]
            assert np.all(o5[b, i] >= sel.min(axis=0) - 1e-12), "below the selected values"
            assert np.all(o5[b, i] <= sel.max(axis=0) + 1e-12), "above the selected values"
    # 6. a very large scale: the key with the largest logit takes all the weight
    o6 = run(orc, qa, kc, vc, idx, 1e4).reshape(o5.shape)
    for b in range(qa.shape[0]):
        for i in range(qa.shape[1]):
            for g in range(qa.shape[2]):
                logits = kc[b, idx[b, i]] @ qa[b, i, g]
                best = idx[b, i][np.argmax(logits)]
                assert np.allclose(o6[b, i, g], vc[b, best], rtol=0, atol=1e-9), "not the argmax"
    # 7. values as a prefix of each key row (one latent cache): the same as
    #    handing the prefix over as a separate array
    qa, kc, _, idx = rand_case(rng, Dk=24, Dv=8)
    shared = run_shared(orc, qa, kc, idx, Dv=8, scale=0.1)
    separate = run(orc, qa, kc, np.ascontiguousarray(kc[..., :8]), idx, 0.1)
    assert np.array_equal(shared, separate), "latent-cache values read wrongly"
    # 8. an empty selection gives zeros; a subset of rows equals those rows of a full run
    empty = np.full_like(idx, -1)
    assert np.all(run(orc, qa, kc, np.ascontiguousarray(kc[..., :8]), empty, 0.1) == 0.0)
    rows = np.array([4, 1], np.int64)
    sub = run(orc, qa, kc, np.ascontiguousarray(kc[..., :8]), idx, 0.1, rows=rows)
    assert np.array_equal(sub, separate[rows]), "row subset differs"


def run_shared(orc, qa, kc, idx, *, Dv, scale):
    B, S, HA, Dk = qa.shape
    T = kc.shape[1]
    kb = bf16_bits(kc)
    return orc.sparse_attention(bf16_bits(qa), kb, kb, idx, B=B, S=S, T=T, HA=HA, Dk=Dk, Dv=Dv,
                                topk=idx.shape[-1], scale=scale, ld_v=Dk)


def test_attention_oracle_pins(orc):
    all_pins(orc)


MUTANTS = {
    "no max subtraction, no normalisation": ("p_j = z[j] / denom;", "p_j = z[j];"),
    "scale ignored": ("z[j] = scale * dot;", "z[j] = dot;"),
    "value stride Dv instead of ld_v": ("const uint16_t *vr = vc + (b * T + sel[j]) * ld_v;",
                                        "const uint16_t *vr = vc + (b * T + sel[j]) * (long long)Dv;"),
    "padding read as key 0": ("if (s >= 0 && s < T)", "if (s < T) if (s < 0) s = 0; if (1)"),
    "query of head 0 for every head": ("const uint16_t *qg = qa + (row * HA + g) * Dk;",
                                       "const uint16_t *qg = qa + (row * HA) * Dk;"),
    "key of the wrong batch": ("const uint16_t *kr = kc + (b * T + sel[j]) * (long long)Dk;",
                               "const uint16_t *kr = kc + ((long long)sel[j]) * (long long)Dk;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "csa_attn_oracle.c")).read()
    if name == "no max subtraction, no normalisation":
        old, new = "double p = z[j] / denom;", "double p = z[j];"
    assert src.count(old) == 1, name
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    lib = A.build(force=True, src=str(mut), lib=str(tmp_path / "libmut.so"))
    with pytest.raises(AssertionError):
        all_pins(A.AttentionOracle(lib))
