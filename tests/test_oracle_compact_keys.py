"""Pins of the oracle's compact 68-byte indexer keys (E2M1 codes + one fp32 scale per key).

Pages: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (AI summary), Main
Findings (890 bytes of global KV per token); "DeepSeek V4.1 Flash: smaller KV cache, same
post-training", How is DeepSeek V4.1 Flash different (Figure 1). The key format itself is a
reading: the pages give only the byte total."""
import numpy as np
import pytest
import torch

from oracle import oracle as O

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _nibbles(codes):
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def test_record_is_68_bytes_and_gives_890_per_token():
    codes, scales = O.quantize_keys_fp4(_bits(np.ones((1, 128))))
    per_entry = codes.shape[1] + scales.dtype.itemsize
    assert per_entry == 68
    assert O.bytes_per_token(indexer_entry_bytes=per_entry) == pytest.approx(890.0)


def test_power_of_two_scale_round_trips_exactly():
    rng = np.random.default_rng(1)
    for e in (-6, -2, 0, 3):
        s = 2.0 ** e
        mags = rng.choice(E2M1, (16, 128))
        mags[:, 5] = 6.0                                   # amax = 6 s, so the scale is s
        x = rng.choice([-1.0, 1.0], (16, 128)) * mags * s
        codes, scales = O.quantize_keys_fp4(_bits(x))
        assert np.all(scales == np.float32(s))
        np.testing.assert_array_equal(O.dequant_keys_fp4(codes, scales), x)


def test_largest_magnitude_takes_code_six_and_zero_key():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128))
    codes, scales = O.quantize_keys_fp4(_bits(x))
    nib = _nibbles(codes)
    xv = O.bf16_array_to_f64(_bits(x))
    arg = np.argmax(np.abs(xv), axis=1)
    assert np.all((nib[np.arange(64), arg] & 7) == 7)
    np.testing.assert_allclose(scales, np.abs(xv).max(axis=1) / 6, rtol=2 ** -23)
    codes0, scales0 = O.quantize_keys_fp4(_bits(np.zeros((2, 128))))
    assert np.all(scales0 == 0) and np.all(codes0 == 0)


def test_negation_flips_only_sign_bits():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 128))
    c1, s1 = O.quantize_keys_fp4(_bits(x))
    c2, s2 = O.quantize_keys_fp4(_bits(-x))
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(_nibbles(c1) ^ 8, _nibbles(c2))


def test_midpoints_round_to_even():
    # scale 1 (amax 6); |x| on the midpoints between E2M1 magnitudes
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0, 2, 2, 4, 4, 6, 6]                   # magnitude codes: even mantissa wins
    x = np.zeros((1, 128))
    x[0, 0] = 6.0
    x[0, 1:1 + len(mids)] = mids
    codes, scales = O.quantize_keys_fp4(_bits(x))
    assert scales[0] == 1.0
    nib = _nibbles(codes)[0]
    assert list(nib[1:1 + len(mids)] & 7) == want


def test_random_keys_match_an_independent_nearest_grid_search():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((200, 128)) * rng.lognormal(0, 2, (200, 1))
    kb = _bits(x)
    codes, scales = O.quantize_keys_fp4(kb)
    xv = O.bf16_array_to_f64(kb).astype(np.float32)
    s = (np.abs(xv).max(axis=1) / np.float32(6)).astype(np.float32)     # fp32 division
    q = (np.abs(xv) / s[:, None]).astype(np.float32).astype(np.float64)  # fp32 quotient
    d = np.abs(q[..., None] - E2M1)                                      # distance to each
    best = np.argmin(d, axis=-1)                                         # lowest code on ties
    tie = np.sort(d, axis=-1)[..., 1] == d.min(axis=-1)
    best = np.where(tie & (best % 2 == 1), best + 1, best)               # ties to even code
    want = best | (np.signbit(xv).astype(np.int64) << 3)
    np.testing.assert_array_equal(scales, s)
    np.testing.assert_array_equal(_nibbles(codes), want)


def test_scores_against_compact_keys_equal_bf16_key_scores_of_the_same_values():
    rng = np.random.default_rng(5)
    H, Di, n = 16, 128, 50
    mags = rng.choice(E2M1, (n, Di))
    mags[:, 0] = 6.0
    e = rng.integers(-4, 3, (n, 1)).astype(np.float64)
    x = rng.choice([-1.0, 1.0], (n, Di)) * mags * np.exp2(e)      # power-of-two scales
    codes, scales = O.quantize_keys_fp4(_bits(x))
    q = torch.randn((H, Di)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    w = rng.uniform(0, 1, H).astype(np.float32)
    # the same key values as bf16 keys, with an E4M3 query (the bf16 scorer takes both in
    # one dtype, so the query is widened to bf16: exact for E4M3 values)
    qb = _bits(O.e4m3_array_to_f64(q.ravel()).reshape(H, Di))
    want = O.index_scores(qb, w, _bits(x), O.BF16)
    got = O.index_scores_fp4key(q, w, codes, scales)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)
    rows = np.array([3, 0, 49], np.int32)
    np.testing.assert_allclose(O.index_scores_fp4key(q, w, codes, scales, rows), want[rows],
                               rtol=1e-14, atol=0)
