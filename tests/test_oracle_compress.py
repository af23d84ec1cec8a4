"""Pins of the oracle's KV compressor, indexer-K projection and bf16 encoder against what
the definitions fix independently of the oracle's own code: a library cast, closed forms,
invariances and special cases.

Pages: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary),
Methodology in Plain English (no overlapping source entries, no absolute positional
embedding, indexer K projected from the main KV entries); "DeepSeek V4.1 Flash: smaller
KV cache, same post-training", How did DeepSeek V4.1 reduce the KV cache? (C_l, Z_l)."""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _bits(x):
    """bf16 bit patterns of values that are exactly bf16 (as a float32 tensor)."""
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _val(bits):
    return O.bf16_array_to_f64(bits)


# ---- bf16 encoder ---------------------------------------------------------------------------

def test_bf16_encode_matches_torch_cast_on_float32_inputs():
    rng = np.random.default_rng(5)
    mant = rng.uniform(1.0, 2.0, 60000)
    expo = rng.integers(-140, 120, 60000)
    sign = rng.choice([-1.0, 1.0], 60000)
    v = (sign * mant * np.exp2(expo.astype(np.float64))).astype(np.float32)
    # exact float32 inputs: torch's float32 -> bf16 cast rounds once, to nearest even
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_encode_many(v.astype(np.float64))
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("v,bits", [
    (1.0 + 2.0 ** -8, 0x3F80),            # midpoint between 1 and 1 + 2^-7: even (1)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),        # midpoint between 1 + 2^-7 and 1 + 2^-6: even
    (-(1.0 + 2.0 ** -8 + 2.0 ** -30), 0xBF81),   # just above a midpoint: up
    (255.5, 0x4380),                      # rounds up across the binade to 256
    (2.0 ** -133, 0x0001),                # smallest subnormal
    (2.0 ** -134, 0x0000),                # half of it: tie to even (zero)
    (3 * 2.0 ** -134, 0x0002),            # 1.5 quanta: tie to even (2)
    (0.0, 0x0000),
    (-0.0, 0x8000),
])
def test_bf16_encode_hand_placed_cases(v, bits):
    assert O.bf16_encode(v) == bits


# ---- compressor -------------------------------------------------------------------------------

def _rand_bits(rng, shape, scale=1.0):
    return _bits(rng.standard_normal(shape) * scale)


def test_ratio_one_is_the_identity():
    rng = np.random.default_rng(1)
    c = _rand_bits(rng, (7, 512))
    z = _rand_bits(rng, (7, 512), 3.0)
    np.testing.assert_array_equal(O.compress_entries(c, z, 1), _val(c))


@pytest.mark.parametrize("r", [2, 4])
def test_equal_logits_give_the_mean(r):
    rng = np.random.default_rng(2)
    c = _rand_bits(rng, (3 * r, 512))
    z = np.repeat(_rand_bits(rng, (3, 1, 512)), r, axis=1).reshape(3 * r, 512)
    want = _val(c).reshape(3, r, 512).mean(axis=1)
    np.testing.assert_allclose(O.compress_entries(c, z, r), want, rtol=1e-14, atol=1e-300)


def test_dominant_logit_selects_its_token_per_channel():
    r = 4
    rng = np.random.default_rng(3)
    c = _rand_bits(rng, (2 * r, 512))
    z = np.zeros((2 * r, 512), np.float32)
    for j in range(2):
        for d in range(512):
            z[j * r + (d + j) % r, d] = 120.0   # exp(-120) ~ 8e-53 for the others
    out = O.compress_entries(c, _bits(z), r)
    cv = _val(c)
    for j in range(2):
        want = np.array([cv[j * r + (d + j) % r, d] for d in range(512)])
        np.testing.assert_allclose(out[j], want, rtol=1e-40, atol=0)


def test_two_tokens_hand_worked():
    # logits 0 and ln 3 would weigh 1/4 and 3/4; bf16 has no ln 3, so take logits 0 and 2:
    # weights 1/(1+e^2) and e^2/(1+e^2); latents 4 and 8 -> (4 + 8 e^2) / (1 + e^2)
    c = _bits([[4.0], [8.0]])
    z = _bits([[0.0], [2.0]])
    e2 = math.exp(2.0)
    assert O.compress_entries(c, z, 2)[0, 0] == pytest.approx((4 + 8 * e2) / (1 + e2), rel=1e-15)
    # and logits (-1, -1): the plain mean 6
    assert O.compress_entries(c, _bits([[-1.0], [-1.0]]), 2)[0, 0] == 6.0


def test_logit_shift_and_token_permutation_change_nothing():
    r = 3
    rng = np.random.default_rng(4)
    c = _rand_bits(rng, (5 * r, 512))
    zi = rng.integers(-6, 7, (5 * r, 512)).astype(np.float32)     # small integers: exact
    base = O.compress_entries(c, _bits(zi), r)
    shifted = O.compress_entries(c, _bits(zi + rng.integers(-5, 6, (1, 512))), r)
    np.testing.assert_allclose(shifted, base, rtol=1e-13)
    perm = np.concatenate([j * r + rng.permutation(r) for j in range(5)])
    permuted = O.compress_entries(c[perm], _bits(zi)[perm], r)
    np.testing.assert_allclose(permuted, base, rtol=1e-13)


def test_outputs_lie_inside_their_tokens_range():
    r = 2
    rng = np.random.default_rng(6)
    c = _rand_bits(rng, (64 * r, 512), 4.0)
    z = _rand_bits(rng, (64 * r, 512), 2.0)
    out = O.compress_entries(c, z, r)
    cv = _val(c).reshape(64, r, 512)
    assert np.all(out >= cv.min(axis=1) - 1e-12) and np.all(out <= cv.max(axis=1) + 1e-12)


# ---- projection -------------------------------------------------------------------------------

def test_projection_one_hot_and_identity():
    rng = np.random.default_rng(7)
    w = _rand_bits(rng, (128, 512))
    x = np.zeros((3, 512))
    for i, d in enumerate((0, 77, 511)):
        x[i, d] = 1.0
    out = O.project_keys(x, w)
    wv = _val(w)
    for i, d in enumerate((0, 77, 511)):
        np.testing.assert_array_equal(out[i], wv[:, d])
    eye = np.zeros((128, 512), np.float32)
    eye[np.arange(128), np.arange(128)] = 1.0
    xr = _val(_rand_bits(rng, (4, 512)))
    np.testing.assert_array_equal(O.project_keys(xr, _bits(eye)), xr[:, :128])


def test_projection_matches_a_float64_matrix_vector_product():
    rng = np.random.default_rng(8)
    w = _rand_bits(rng, (128, 512), 0.05)
    x = _val(_rand_bits(rng, (16, 512)))
    np.testing.assert_allclose(O.project_keys(x, w), x @ _val(w).T, rtol=1e-12, atol=1e-12)


def test_compress_write_composes_the_pinned_steps():
    """The whole write: bf16 latent -> the pinned FP4 quantizer and the projection, with the
    key stored by the pinned E4M3 encoder."""
    rng = np.random.default_rng(9)
    r = 2
    c = _rand_bits(rng, (6 * r, 512))
    z = _rand_bits(rng, (6 * r, 512))
    w = _rand_bits(rng, (128, 512), 0.05)
    lat, codes, scales, key, k = O.compress_write(c, z, r, w, O.E4M3)
    np.testing.assert_array_equal(lat, O.bf16_encode_many(O.compress_entries(c, z, r)))
    qc, qs = O.quantize_entries(lat)
    np.testing.assert_array_equal(codes, qc)
    np.testing.assert_array_equal(scales, qs)
    want = torch.from_numpy(k.astype(np.float32)).to(torch.float8_e4m3fn)
    # the float32 cast is exact here unless k sits within 2^-24 of an E4M3 midpoint
    assert (key == want.view(torch.uint8).numpy()).mean() > 0.999
