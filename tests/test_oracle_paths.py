"""Pins of the oracle's indexer score, Top-K, candidate pool, attention and byte
accounting against closed forms, invariants, brute force and library routines."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLD, "pages_numbers.json")) as f:
        return json.load(f)


def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _e4m3_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


# ---- indexer score -------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [O.BF16, O.E4M3])
def test_index_score_relu_identity_reduces_to_matmul(dtype):
    """ReLU(a) - ReLU(-a) = a, so s(q) - s(-q) = sum_h w_h q_h.k: a plain matmul."""
    rng = np.random.default_rng(1)
    H, Di, n = 5, 128, 37
    enc = _bf16_bits if dtype == O.BF16 else _e4m3_bits
    dec = O.bf16_array_to_f64 if dtype == O.BF16 else O.e4m3_array_to_f64
    q = enc(rng.standard_normal((H, Di)))
    k = enc(rng.standard_normal((n, Di)))
    qneg = enc(-dec(q))
    w = rng.random(H).astype(np.float32)
    s_pos = O.index_scores(q, w, k, dtype)
    s_neg = O.index_scores(qneg, w, k, dtype)
    dots = np.matmul(dec(k).reshape(n, Di), dec(q).reshape(H, Di).T)  # [n, H]
    lin = dots @ w.astype(np.float64)
    np.testing.assert_allclose(s_pos - s_neg, lin, rtol=0, atol=1e-9 * np.abs(dots).sum())
    absd = np.abs(dots) @ w.astype(np.float64)
    np.testing.assert_allclose(s_pos + s_neg, absd, rtol=1e-12)


def test_index_score_closed_forms():
    Di = 128
    k = _e4m3_bits(np.random.default_rng(2).standard_normal((9, Di)))
    kd = O.e4m3_array_to_f64(k).reshape(9, Di)
    # unit query on channel 7, one head, weight 1: s_j = max(0, k_j[7])
    q = np.zeros((1, Di), np.float32)
    q[0, 7] = 1.0
    s = O.index_scores(_e4m3_bits(q), np.ones(1, np.float32), k, O.E4M3)
    np.testing.assert_array_equal(s, np.maximum(kd[:, 7], 0.0))
    # zero weights give +0 scores
    q2 = _e4m3_bits(np.random.default_rng(3).standard_normal((4, Di)))
    s0 = O.index_scores(q2, np.zeros(4, np.float32), k, O.E4M3)
    assert np.all(s0 == 0.0) and not np.any(np.signbit(s0))
    # a weight of 2 on a duplicated head doubles it (linearity in w)
    s1 = O.index_scores(q2[:1], np.ones(1, np.float32), k, O.E4M3)
    s2 = O.index_scores(np.concatenate([q2[:1], q2[:1]]), np.ones(2, np.float32), k, O.E4M3)
    np.testing.assert_array_equal(s2, 2 * s1)


def test_index_score_row_subset():
    rng = np.random.default_rng(4)
    q = _e4m3_bits(rng.standard_normal((3, 128)))
    k = _e4m3_bits(rng.standard_normal((50, 128)))
    w = rng.random(3).astype(np.float32)
    full = O.index_scores(q, w, k, O.E4M3)
    rows = np.array([49, 3, 3, 0], np.int32)
    np.testing.assert_array_equal(O.index_scores(q, w, k, O.E4M3, rows=rows), full[rows])


# ---- Top-K -----------------------------------------------------------------------------

def _brute_topk(s, K, ids=None):
    ids = list(range(len(s))) if ids is None else list(ids)
    order = sorted(range(len(s)), key=lambda i: (-s[i], ids[i]))
    chosen = sorted(ids[i] for i in order[:K])
    return chosen + [-1] * (K - len(chosen))


@pytest.mark.parametrize("n,K", [(1, 4), (7, 4), (16, 16), (33, 8), (200, 64), (513, 512)])
def test_topk_equals_full_sort_with_planted_ties(n, K):
    rng = np.random.default_rng(n * 31 + K)
    s = rng.integers(0, max(2, n // 3), size=n).astype(np.float64)  # many exact ties
    got = O.topk(s, K)
    assert list(got) == _brute_topk(list(s), K)


def test_topk_with_ids_tie_breaks_on_id():
    s = np.array([5.0, 5.0, 5.0, 1.0])
    ids = np.array([90, 10, 50, 0], np.int32)
    assert list(O.topk(s, 2, ids)) == [10, 50]
    assert list(O.topk(s, 5, ids)) == [0, 10, 50, 90, -1]


# ---- candidate pool --------------------------------------------------------------------

@pytest.mark.parametrize("n,nblk", [(5, 2), (64, 3), (1000, 16), (4099, 40), (100, 500)])
def test_pool_invariants(n, nblk):
    rng = np.random.default_rng(n + nblk)
    s = rng.integers(0, 50, size=n).astype(np.float64)
    pool = O.pool(s, nblk)
    got = [int(p) for p in pool if p >= 0]
    assert got == sorted(got) and len(set(got)) == len(got)
    assert all(0 <= p < n for p in got)
    assert all(p == -1 for p in pool[len(got):])
    nb = (n + 7) // 8
    blocks = sorted({p // 8 for p in got})
    assert len(blocks) == min(nblk, nb)
    # whole blocks (their visible part) only
    for c in blocks:
        assert all(j in got for j in range(8 * c, min(8 * c + 8, n)))
    # every kept block's max >= every dropped block's max; equal maxima prefer lower block
    bmax = [max(s[8 * c:8 * c + 8]) for c in range(nb)]
    kept = set(blocks)
    for c in range(nb):
        if c in kept:
            continue
        for c2 in kept:
            assert bmax[c2] > bmax[c] or (bmax[c2] == bmax[c] and c2 < c)


def test_full_topk_inside_pool():
    """Any block holding a Top-K entry has a max >= s_K, so with >= K blocks kept the
    pool contains the Top-K (planted ties included)."""
    rng = np.random.default_rng(9)
    for trial in range(20):
        n = int(rng.integers(100, 3000))
        s = np.round(rng.standard_normal(n), 1)
        K = int(rng.integers(1, 64))
        top = set(int(i) for i in O.topk(s, K) if i >= 0)
        pool = set(int(p) for p in O.pool(s, max(K, 8)) if p >= 0)
        assert top <= pool


# ---- attention -------------------------------------------------------------------------

def test_attention_all_entries_is_dense_attention():
    rng = np.random.default_rng(11)
    H, D, n = 6, 512, 40
    q = rng.standard_normal((H, D))
    rows = rng.standard_normal((n, D)) * 0.5
    tau = 1.0 / math.sqrt(D)
    ours = O.attention(q, rows, tau)
    tq = torch.from_numpy(q)[None, :, None, :]           # [1, H, 1, D]
    tk = torch.from_numpy(rows)[None, None].expand(1, H, n, D)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tk, scale=tau)
    np.testing.assert_allclose(ours, ref[0, :, 0, :].numpy(), rtol=1e-12, atol=1e-13)


def test_attention_closed_forms():
    rng = np.random.default_rng(12)
    D = 512
    x = rng.standard_normal((1, D))
    q = rng.standard_normal((3, D))
    np.testing.assert_array_equal(O.attention(q, x, 0.1), np.repeat(x, 3, axis=0))
    rows = rng.standard_normal((17, D))
    np.testing.assert_allclose(O.attention(np.zeros((2, D)), rows, 0.3),
                               np.repeat(rows.mean(axis=0, keepdims=True), 2, axis=0),
                               rtol=1e-12, atol=1e-14)
    assert np.all(O.attention(q, np.zeros((0, D)), 0.1) == 0.0)
    perm = rng.permutation(17)
    np.testing.assert_allclose(O.attention(q, rows, 0.05), O.attention(q, rows[perm], 0.05),
                               rtol=1e-12, atol=1e-14)


def test_reuse_output_equals_full_output_given_same_indices():
    rng = np.random.default_rng(13)
    kv = _bf16_bits(rng.standard_normal((300, 512)))
    codes, scales = O.quantize_entries(kv)
    idx = O.topk(rng.standard_normal(300), 64)
    swa = _e4m3_bits(rng.standard_normal((128, 512)))
    q = _bf16_bits(rng.standard_normal((8, 512)))
    a = O.attention_decode_query(q, codes, scales, idx, swa, 1 / math.sqrt(512))
    b = O.attention_decode_query(q, codes, scales, idx.copy(), swa, 1 / math.sqrt(512))
    np.testing.assert_array_equal(a, b)


# ---- byte accounting ------------------------------------------------------------------

def test_bytes_per_token_accounting():
    g = _golden()
    D = g["latent_channels"]["value"]
    assert O.main_entry_bytes(D) == D // 2 + D // g["channels_per_scale"]["value"] == 288
    enc, dec = g["encoder_layout"], g["decoder_layout"]
    assert enc["groups"] * (enc["full_per_group"] + enc["reuse_per_group"]) == enc["csa2_layers"]
    args = dict(enc_full=enc["groups"] * enc["full_per_group"], enc_ratio=enc["ratio"],
                dec_full=dec["full_layers"], dec_ratio=dec["ratio"])
    # 890 B/token is met with a 68-byte indexer-key entry; a 128-dim FP8 key gives 1040
    assert O.bytes_per_token(D, 68.0, **args) == g["global_kv_bytes_per_token"]["value"]
    assert O.bytes_per_token(D, 128.0, **args) == 1040.0
    v4 = g["v4_flash_bytes_per_token"]["value"]
    v1 = g["v1_bytes_per_token"]["value"]
    assert round(v4 / g["global_kv_bytes_per_token"]["value"]) == 4
    assert round(v1 / g["global_kv_bytes_per_token"]["value"]) == g["v1_bytes_per_token"]["ratio_claim"]
    assert g["pool_blocks"]["value"] * g["pool_block_size"]["value"] == g["pool_positions"]["value"]


# ---- prefill visibility and the causal window ------------------------------------------

def _simulated_visible_counts(ratio, last_pos):
    """Feed tokens one by one to a compressor that emits an entry whenever `ratio` tokens
    have arrived; the count after token p is what that token can read."""
    counts, pending, emitted = [], 0, 0
    for _p in range(last_pos + 1):
        pending += 1
        if pending == ratio:
            emitted += 1
            pending = 0
        counts.append(emitted)
    return counts


@pytest.mark.parametrize("ratio", [1, 2, 3])
def test_prefill_visible_matches_token_by_token_compressor(ratio):
    counts = _simulated_visible_counts(ratio, 200)
    assert [O.prefill_visible(p, ratio) for p in range(201)] == counts
    # positions whose p + 1 is not a multiple of the ratio see the previous whole entry only
    if ratio > 1:
        assert O.prefill_visible(ratio - 2, ratio) == 0
        assert O.prefill_visible(2 * ratio - 2, ratio) == 1


def test_prefill_visible_at_workload_ends():
    # 4,096 new tokens on 131,072 cached at ratio 2: the first new token sees the 65,536
    # cached entries, the last one all 67,584
    assert O.prefill_visible(131072, 2) == 65536
    assert O.prefill_visible(131072 + 4095, 2) == 67584
    assert O.prefill_visible(0, 1) == 1 and O.prefill_visible(0, 2) == 0


@pytest.mark.parametrize("q_pos0,W,T", [(0, 4, 9), (3, 4, 6), (0, 128, 200), (127, 128, 3),
                                        (300, 128, 5), (5, 1, 4), (14, 16, 8)])
def test_prefill_window_rows_match_buffer_scan(q_pos0, W, T):
    """Scan the window buffer row by row (row i holds position q_pos0 - (W-1) + i) and keep
    the rows whose position exists and lies in the token's last W positions."""
    buf_pos = [q_pos0 - (W - 1) + i for i in range(W - 1 + T)]
    for t in range(T):
        p = q_pos0 + t
        expect = [i for i, pos in enumerate(buf_pos) if pos >= 0 and p - W < pos <= p]
        got = O.prefill_window_rows(q_pos0, W, t).tolist()
        assert got == expect, (q_pos0, W, t)
        assert len(got) == min(W, p + 1)
        assert got[-1] == t + W - 1          # the token's own row is the last one


def test_prefill_query_with_every_entry_selected_is_dense_attention():
    """K >= visible entries: the prefill query attends over all visible entries and the
    token's window rows, i.e. plain dense attention over those rows."""
    rng = np.random.default_rng(21)
    ratio, q_pos0, T, W, H, D, K = 2, 5, 4, 4, 3, 512, 16
    cap = (q_pos0 + T) // ratio
    kv = _bf16_bits(rng.standard_normal((cap, D)))
    k_I = _e4m3_bits(rng.standard_normal((cap, 128)))
    swa = _e4m3_bits(rng.standard_normal((W - 1 + T, D)))
    tau = 1 / math.sqrt(D)
    for t in range(T):
        qi = _e4m3_bits(rng.standard_normal((2, 128)))
        w = rng.random(2).astype(np.float32)
        q = _bf16_bits(rng.standard_normal((H, D)))
        idx, out = O.prefill_query(qi, w, k_I, O.E4M3, kv, q, swa, q_pos0, t, ratio, K, W, tau)
        n = sum(1 for j in range(cap) if ratio * j + ratio - 1 <= q_pos0 + t)
        assert idx.tolist() == list(range(n)) + [-1] * (K - n)
        c, s = O.quantize_entries(kv[:n])
        rows = np.concatenate([O.dequant_entries(c, s),
                               O.e4m3_array_to_f64(swa[max(t, W - 1 - q_pos0):t + W]).reshape(-1, D)])
        tq = torch.from_numpy(O.bf16_array_to_f64(q).reshape(H, D))[None, :, None, :]
        tk = torch.from_numpy(rows)[None, None].expand(1, H, rows.shape[0], D)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tk, scale=tau)
        np.testing.assert_allclose(out, ref[0, :, 0, :].numpy(), rtol=1e-12, atol=1e-13)
