"""Host checks of the float32 identities the indexer's kernels rely on.

The score of a (query, key) pair is sum_h w_h * ReLU(q_h . k) (DeepSeek-V3.2
lightning indexer, "DeepSeek Sparse Attention" section; the CSA indexer of the
DeepSeek-V4 pages uses the same form).  The fused kernel forms each ReLU as
x + |x| (twice the ReLU, in one packed add) and multiplies by the weight held
halved.  In IEEE float32 with round-to-nearest that product equals
max(x, 0) * w bit for bit whenever w / 2 is exact (w normal) and 2x does not
overflow; this test checks it over every class of x (both zeros, subnormals,
normals up to half the largest float) and weights of both signs.  The
selectors' order image (score -> unsigned integer of the same order) is
checked the same way.
"""
import numpy as np
import pytest


def _logits(rng, n):
    f32 = np.float32
    parts = [
        np.array([0.0, -0.0, 1.0, -1.0, np.finfo(f32).tiny, -np.finfo(f32).tiny,
                  np.finfo(f32).max / 2, -np.finfo(f32).max], dtype=f32),
        # subnormals of both signs
        (rng.integers(1, 1 << 23, n) .astype(np.uint32)
         | (rng.integers(0, 2, n).astype(np.uint32) << 31)).view(f32),
        # normals over every binade below half the largest float
        (np.ldexp(rng.uniform(1.0, 2.0, n), rng.integers(-126, 127, n))
         * rng.choice([-1.0, 1.0], n)).astype(f32),
    ]
    x = np.concatenate(parts)
    return x[np.abs(x) <= np.finfo(f32).max / 2]


@pytest.mark.parametrize("seed", [0, 1])
def test_twice_relu_times_half_weight_is_exact(seed):
    rng = np.random.default_rng(seed)
    x = _logits(rng, 200_000)
    w = (np.ldexp(rng.uniform(1.0, 2.0, x.size), rng.integers(-100, 100, x.size))
         * rng.choice([-1.0, 1.0], x.size)).astype(np.float32)
    with np.errstate(over="ignore", under="ignore"):
        twice = x + np.abs(x)                          # the packed add
        assert np.array_equal(twice.view(np.uint32),
                              (2 * np.maximum(x, np.float32(0))).view(np.uint32))
        got = twice * (w * np.float32(0.5))            # product the FMA adds
        want = np.maximum(x, np.float32(0)) * w
    # equal including signed zeros, infinities from large products and
    # results that underflow
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_negative_logits_give_positive_zero():
    x = np.array([-0.0, -1e-45, -3.0, -np.finfo(np.float32).max], dtype=np.float32)
    twice = x + np.abs(x)
    assert np.all(twice.view(np.uint32) == 0)


def test_order_image_is_monotone_and_folds_zero():
    """The selectors map a float32 score to an unsigned integer of the same
    order (negative: complement; otherwise: sign bit set) with one XOR against
    the sign-spread mask; -0.0 is added to +0.0 first, so both zeros share one
    image.  Checked on every class of float: the images sort like the scores."""
    rng = np.random.default_rng(7)
    f32 = np.finfo(np.float32)
    bits = rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = np.concatenate([x[np.isfinite(x)],
                        np.array([0.0, -0.0, f32.max, -f32.max, f32.tiny, -f32.tiny,
                                  np.inf, -np.inf], dtype=np.float32)])
    b = (x + np.float32(0.0)).view(np.uint32)
    spread = (b.view(np.int32) >> 31).view(np.uint32)
    img = b ^ (spread | np.uint32(0x80000000))
    ref = np.where(b & np.uint32(0x80000000), ~b, b | np.uint32(0x80000000))
    assert np.array_equal(img, ref)
    order = np.argsort(x, kind="stable")
    assert np.all(np.diff(img[order].astype(np.int64)) >= 0)
    assert img[x == 0.0].min() == img[x == 0.0].max()
