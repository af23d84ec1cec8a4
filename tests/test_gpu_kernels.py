"""GPU parity of each CSA2 kernel against the CPU oracle, through the C ABI, on small
seeded inputs that still span several tiles and ragged tails."""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import (bits16, bits8, check_attention, check_topk, odt, oracle_main_rows,
                           raw_qk)

pytestmark = pytest.mark.gpu

dev = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from fp4_compressed_sparse_quantize_b200 import csa2
    csa2.lib()
    yield


def C():
    from fp4_compressed_sparse_quantize_b200 import csa2
    return csa2


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


# ---- quantize-on-write ---------------------------------------------------------------------

def _quantize_gpu(kv, cap=None, dst=None):
    B, n, D = kv.shape
    cap = cap or n
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    dst = dst if dst is not None else torch.zeros(B, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    C().quantize_kv(kv, dst, codes, scales, status=st)
    torch.cuda.synchronize()
    return codes, scales, int(st.item())


def test_quantize_random_bit_exact():
    g = _gen(1)
    x = torch.randn((3, 700, 512), generator=g) * torch.exp(torch.randn((3, 1, 512), generator=g) * 2)
    x[0, 5, :16] = 0.0
    x[0, 6, :16] = -0.0
    x[1, 7, 16:32] = 3000.0
    x[1, 8, 32:48] = -2688.0
    x[2, 9, 48:64] = 1e-30
    kv = x.to(torch.bfloat16)
    codes, scales, st = _quantize_gpu(kv.to(dev))
    assert st == 0
    rc, rs = O.quantize_entries(bits16(kv).reshape(-1, 512))
    np.testing.assert_array_equal(bits8(scales).reshape(-1, 32), rs)
    np.testing.assert_array_equal(bits8(codes).reshape(-1, 256), rc)


def test_quantize_every_scale_and_magnitude():
    """For every finite positive scale s with 6s representable, blocks whose max is 6s carry
    every bf16 magnitude up to 6s (both signs): covers every (x, s) code decision."""
    rows = []
    for sc in range(1, 127):
        s = O.e4m3_value(sc)
        top = torch.tensor([6.0 * s], dtype=torch.float32).to(torch.bfloat16)
        if float(top) != 6.0 * s:
            continue
        mags = torch.arange(0, 0x7F80, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
        mags = mags[mags.float() <= 6.0 * s]
        vals = torch.cat([mags, -mags])
        nblk = (vals.numel() + 14) // 15
        pad = torch.zeros(nblk * 15, dtype=torch.bfloat16)
        pad[: vals.numel()] = vals
        blocks = torch.cat([top.expand(nblk, 1), pad.view(nblk, 15)], dim=1)
        rows.append(blocks.reshape(-1))
    flat = torch.cat(rows)
    n = (flat.numel() + 511) // 512
    full = torch.zeros(n * 512, dtype=torch.bfloat16)
    full[: flat.numel()] = flat
    kv = full.view(1, n, 512)
    codes, scales, st = _quantize_gpu(kv.to(dev))
    rc, rs = O.quantize_entries(bits16(kv).reshape(-1, 512))
    np.testing.assert_array_equal(bits8(scales).reshape(-1, 32), rs)
    np.testing.assert_array_equal(bits8(codes).reshape(-1, 256), rc)


def test_quantize_offsets_and_bad_offset_flag():
    g = _gen(2)
    kv = torch.randn((2, 5, 512), generator=g).to(torch.bfloat16)
    dst = torch.tensor([3, 9], dtype=torch.int32, device=dev)  # second sequence overflows cap=12
    codes, scales, st = _quantize_gpu(kv.to(dev), cap=12, dst=dst)
    assert st & C().DEV_BAD_INDEX
    rc, rs = O.quantize_entries(bits16(kv[0]))
    np.testing.assert_array_equal(bits8(codes[0, 3:8]), rc)
    rc1, _ = O.quantize_entries(bits16(kv[1, :3]))
    np.testing.assert_array_equal(bits8(codes[1, 9:12]), rc1)
    assert int(codes[0, :3].sum()) == 0


# ---- indexer + Top-K (Full decode) -----------------------------------------------------------

def _keys(B, cap, dtype, g, dup=False):
    k = torch.randn((B, cap, 128), generator=g)
    if dup and cap > 40:
        k[:, 30] = k[:, 10]   # exact duplicate rows -> exact score ties
        k[:, 31] = k[:, 10]
    return k.to(dtype)


def _full_decode(q_I, w, k_I, n_vis, K, pool_blocks=0):
    B, T, H_I, _ = q_I.shape
    cap = k_I.shape[1]
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    scores = torch.zeros((B, T, cap), dtype=torch.float32, device=dev)
    pool = None
    if pool_blocks:
        pool = torch.empty((B, T, pool_blocks * 8), dtype=torch.int32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, T, H_I, cap, K, pool_blocks))
    C().index_score_topk("full", q_I.to(dev), w.to(dev), k_I.to(dev), K, idx, ws,
                         n_vis0=torch.tensor(n_vis, dtype=torch.int32, device=dev),
                         pool_out=pool, pool_blocks=pool_blocks, scores_out=scores)
    torch.cuda.synchronize()
    st = C().read_device_status(ws)
    return idx.cpu().numpy(), scores.cpu().numpy(), (pool.cpu().numpy() if pool is not None else None), st


@pytest.mark.parametrize("dtype,H_I,K", [(torch.bfloat16, 8, 64), (torch.float8_e4m3fn, 64, 512),
                                         (torch.float8_e4m3fn, 16, 32)])
@pytest.mark.parametrize("n_list", [[1, 7, 16], [511, 512, 513], [4096, 1000, 129],
                                    # long rows split over a cluster, beside short rows whose
                                    # later parts are empty
                                    [40000, 9, 70], [20000, 5, 4100]])
def test_full_decode_scores_and_topk(dtype, H_I, K, n_list):
    g = _gen(sum(n_list) + H_I)
    B = len(n_list)
    cap = max(n_list)
    k_I = _keys(B, cap, dtype, g, dup=True)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(dtype)
    w = torch.rand((B, 1, H_I), generator=g)
    idx, scores, _, st = _full_decode(q_I, w, k_I, n_list, K)
    assert st == 0
    for b, n in enumerate(n_list):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b, :n]), odt(q_I))
        # fp32 accumulation vs exact: bound by the sum of |terms|
        qd = (O.bf16_array_to_f64 if dtype == torch.bfloat16 else O.e4m3_array_to_f64)(
            raw_qk(q_I[b, 0])).reshape(H_I, 128)
        kd = (O.bf16_array_to_f64 if dtype == torch.bfloat16 else O.e4m3_array_to_f64)(
            raw_qk(k_I[b, :n])).reshape(n, 128)
        mag = np.abs(kd) @ np.abs(qd).T @ w[b, 0].numpy().astype(np.float64)
        np.testing.assert_array_less(np.abs(scores[b, 0, :n] - s), 2e-6 * mag + 1e-6)
        check_topk(idx[b, 0], s, np.arange(n), K, f"b={b} n={n}")


def test_topk_long_rows_odd_stride():
    """Rows long enough for the multi-CTA row selection, an odd row stride (rows start at
    every 4-byte alignment) and ragged lengths."""
    g = _gen(77)
    n_list = [40003, 33000, 65537]
    B, cap, H_I, K = len(n_list), max(n_list), 64, 512
    k_I = _keys(B, cap, torch.float8_e4m3fn, g)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, 1, H_I), generator=g)
    idx, scores, _, st = _full_decode(q_I, w, k_I, n_list, K)
    assert st == 0
    for b, n in enumerate(n_list):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b, :n]), O.E4M3)
        check_topk(idx[b, 0], s, np.arange(n), K, f"b={b} n={n}")


def test_topk_rows_beyond_the_bitmap_kernel():
    """Rows longer than 262,144 entries go to the chunked kernel (every CTA classifies a
    chunk, the last one of the row finishes it); at 300,001 entries its picks are emitted
    through a bitmap of positions."""
    g = _gen(78)
    n, K = 300001, 512
    k_I = _keys(1, n, torch.float8_e4m3fn, g, dup=True)
    q_I = torch.randn((1, 1, 16, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((1, 1, 16), generator=g)
    idx, scores, _, st = _full_decode(q_I, w, k_I, [n], K)
    assert st == 0
    s = O.index_scores(raw_qk(q_I[0, 0]), w[0, 0].numpy(), raw_qk(k_I[0]), O.E4M3)
    check_topk(idx[0, 0], s, np.arange(n), K, "n=300001")


def test_topk_degenerate_all_equal_scores():
    """w = 0: every score is +0, the K lowest positions must win (slow exact path)."""
    g = _gen(7)
    n = 70000
    k_I = torch.randn((1, n, 128), generator=g).to(torch.float8_e4m3fn)
    q_I = torch.randn((1, 1, 64, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.zeros((1, 1, 64))
    idx, scores, _, st = _full_decode(q_I, w, k_I, [n], 512)
    assert st == 0
    np.testing.assert_array_equal(idx[0, 0], np.arange(512))
    assert np.all(scores[0, 0] == 0.0)


def test_topk_tied_maximum_overflowing_one_cluster_part():
    """The row's best key repeated 3,000 times: exact ties at the top, so the K lowest of
    those positions win. Rows of 40,000 entries split over a 4-CTA cluster (parts of ~10,000):
    row 0 puts every copy in the first part, row 1 straddles the first two parts; either way
    one part holds more candidates than its share of the list, and the selection goes back
    to the row."""
    g = _gen(9)
    n, K = 40000, 512
    k_I = torch.randn((2, n, 128), generator=g).to(torch.float8_e4m3fn)
    q_I = torch.randn((2, 1, 64, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((2, 1, 64), generator=g)
    starts = [0, 9000]
    for b in range(2):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b]), O.E4M3)
        best = int(np.argmax(s))
        k_I[b, starts[b]:starts[b] + 3000] = k_I[b, best]
    idx, scores, _, st = _full_decode(q_I, w, k_I, [n, n], K)
    assert st == 0
    for b in range(2):
        copies = np.arange(starts[b], starts[b] + 3000)
        assert np.all(scores[b, 0, copies] == scores[b, 0, copies[0]])
        assert np.all(scores[b, 0] <= scores[b, 0, copies[0]])
        want = np.sort(np.concatenate([copies, np.nonzero(scores[b, 0] == scores[b, 0, copies[0]])[0]]))
        want = np.unique(want)[:K]
        np.testing.assert_array_equal(idx[b, 0], want)


def test_topk_many_ties_mixed():
    """Integer-valued scores with heavy ties: one-hot keys and a one-head query."""
    g = _gen(8)
    n = 9000
    ch = torch.randint(0, 8, (n,), generator=g)
    k = torch.zeros((1, n, 128))
    k[0, torch.arange(n), ch] = 1.0
    q = torch.zeros((1, 1, 16, 128))
    q[0, 0, 0, :8] = torch.arange(8, dtype=torch.float32)
    w = torch.zeros((1, 1, 16))
    w[0, 0, 0] = 1.0
    k_I, q_I = k.to(torch.float8_e4m3fn), q.to(torch.float8_e4m3fn)
    idx, scores, _, st = _full_decode(q_I, w, k_I, [n], 700)
    s = O.index_scores(raw_qk(q_I[0, 0]), w[0, 0].numpy(), raw_qk(k_I[0]), O.E4M3)
    expect = O.topk(s, 700)  # integer scores: the GPU's fp32 sums are exact
    np.testing.assert_array_equal(idx[0, 0], expect)


@pytest.mark.parametrize("H_I,K,n_list", [(128, 256, [5000, 300, 40000]), (32, 512, [9000, 513])])
def test_full_decode_other_head_counts(H_I, K, n_list):
    """FP8 scans with 32 and 128 indexer heads: 128 heads take a single 384-column
    accumulator and one epilogue group, 32 heads a query operand of 32 columns."""
    g = _gen(H_I + 5)
    B, cap = len(n_list), max(n_list)
    k_I = _keys(B, cap, torch.float8_e4m3fn, g, dup=True)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, 1, H_I), generator=g)
    idx, scores, _, st = _full_decode(q_I, w, k_I, n_list, K)
    assert st == 0
    for b, n in enumerate(n_list):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b, :n]), O.E4M3)
        qd = O.e4m3_array_to_f64(raw_qk(q_I[b, 0]).ravel()).reshape(H_I, 128)
        kd = O.e4m3_array_to_f64(raw_qk(k_I[b, :n]).ravel()).reshape(n, 128)
        mag = np.abs(kd) @ np.abs(qd).T @ w[b, 0].numpy().astype(np.float64)
        np.testing.assert_array_less(np.abs(scores[b, 0, :n] - s), 2e-6 * mag + 1e-6)
        check_topk(idx[b, 0], s, np.arange(n), K, f"H_I={H_I} b={b} n={n}")


def test_pool_and_reindex_decode():
    g = _gen(9)
    B, n, H_I, K, nblk = 2, 20000, 64, 512, 512
    k_I = _keys(B, n, torch.float8_e4m3fn, g)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, 1, H_I), generator=g)
    n_list = [n, n - 5]
    idx, scores, pool, st = _full_decode(q_I, w, k_I, n_list, K, pool_blocks=nblk)
    assert st == 0
    q2 = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w2 = torch.rand((B, 1, H_I), generator=g)
    for b in range(B):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b, :n_list[b]]), O.E4M3)
        check_topk(idx[b, 0], s, np.arange(n_list[b]), K, f"full b={b}")
        # pool: compare block selection with the near-tie rule on block maxima
        nb = (n_list[b] + 7) // 8
        bmax = np.array([s[8 * c:8 * c + 8].max() for c in range(nb)])
        got_blocks = np.unique(pool[b, 0][pool[b, 0] >= 0] // 8)
        gb = np.full(nblk, -1)
        gb[: len(got_blocks)] = got_blocks
        check_topk(gb, bmax, np.arange(nb), nblk, f"pool b={b}")
        vis = pool[b, 0][pool[b, 0] >= 0]
        assert np.all(np.diff(vis) > 0) and vis.max() < n_list[b]
        assert set(idx[b, 0].tolist()) <= set(vis.tolist())
    # Reindex with the oracle's own pool (an oracle value may feed the GPU)
    pool_o = np.stack([O.pool(O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(),
                                             raw_qk(k_I[b, :n_list[b]]), O.E4M3), nblk)
                       for b in range(B)])[:, None, :]
    idx2 = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    P = pool_o.shape[-1]
    sc2 = torch.zeros((B, 1, P), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, 1, H_I, P, K))
    C().index_score_topk("reindex", q2.to(dev), w2.to(dev), k_I.to(dev), K, idx2, ws,
                         n_vis0=torch.tensor(n_list, dtype=torch.int32, device=dev),
                         pool_in=torch.from_numpy(pool_o.astype(np.int32)).to(dev),
                         scores_out=sc2)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    idx2 = idx2.cpu().numpy()
    for b in range(B):
        ids = pool_o[b, 0][pool_o[b, 0] >= 0]
        s2 = O.index_scores(raw_qk(q2[b, 0]), w2[b, 0].numpy(), raw_qk(k_I[b]), O.E4M3, rows=ids)
        check_topk(idx2[b, 0], s2, ids, K, f"reindex b={b}")


def test_pool_and_reindex_with_bf16_keys():
    """The candidate pool and the Reindex gather with bf16 indexer keys (two 128-byte halves
    per key row): block selection, the rescored pool and its Top-K against the oracle."""
    g = _gen(79)
    B, n, H_I, K, nblk = 2, 6000, 16, 64, 128
    k_I = _keys(B, n, torch.bfloat16, g)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.bfloat16)
    w = torch.rand((B, 1, H_I), generator=g)
    n_list = [n, n - 11]
    idx, scores, pool, st = _full_decode(q_I, w, k_I, n_list, K, pool_blocks=nblk)
    assert st == 0
    for b in range(B):
        s = O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(), raw_qk(k_I[b, :n_list[b]]), O.BF16)
        check_topk(idx[b, 0], s, np.arange(n_list[b]), K, f"full b={b}")
        nb = (n_list[b] + 7) // 8
        bmax = np.array([s[8 * c:8 * c + 8].max() for c in range(nb)])
        got_blocks = np.unique(pool[b, 0][pool[b, 0] >= 0] // 8)
        gb = np.full(nblk, -1)
        gb[: len(got_blocks)] = got_blocks
        check_topk(gb, bmax, np.arange(nb), nblk, f"pool b={b}")
    q2 = torch.randn((B, 1, H_I, 128), generator=g).to(torch.bfloat16)
    w2 = torch.rand((B, 1, H_I), generator=g)
    pool_o = np.stack([O.pool(O.index_scores(raw_qk(q_I[b, 0]), w[b, 0].numpy(),
                                             raw_qk(k_I[b, :n_list[b]]), O.BF16), nblk)
                       for b in range(B)])[:, None, :]
    P = pool_o.shape[-1]
    idx2 = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    sc2 = torch.zeros((B, 1, P), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, 1, H_I, P, K))
    C().index_score_topk("reindex", q2.to(dev), w2.to(dev), k_I.to(dev), K, idx2, ws,
                         n_vis0=torch.tensor(n_list, dtype=torch.int32, device=dev),
                         pool_in=torch.from_numpy(pool_o.astype(np.int32)).to(dev),
                         scores_out=sc2)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    idx2 = idx2.cpu().numpy()
    sc2 = sc2.cpu().numpy()
    for b in range(B):
        slots = np.nonzero(pool_o[b, 0] >= 0)[0]
        ids = pool_o[b, 0][slots]
        s2 = O.index_scores(raw_qk(q2[b, 0]), w2[b, 0].numpy(), raw_qk(k_I[b]), O.BF16, rows=ids)
        qd = O.bf16_array_to_f64(raw_qk(q2[b, 0]).ravel()).reshape(H_I, 128)
        kd = O.bf16_array_to_f64(raw_qk(k_I[b]).ravel()).reshape(n, 128)[ids]
        mag = np.abs(kd) @ np.abs(qd).T @ w2[b, 0].numpy().astype(np.float64)
        np.testing.assert_array_less(np.abs(sc2[b, 0, slots] - s2), 2e-6 * mag + 1e-6)
        check_topk(idx2[b, 0], s2, ids, K, f"reindex b={b}")


# ---- attention ----------------------------------------------------------------------------

def _attn_case(B, H, K, W, n, seed, valid=None):
    g = _gen(seed)
    kv = (torch.randn((B, n, 512), generator=g) *
          torch.exp(torch.randn((B, 1, 512), generator=g))).to(torch.bfloat16)
    codes = torch.zeros((B, n, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, n, 32), dtype=torch.uint8, device=dev)
    C().quantize_kv(kv.to(dev), torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    idx = np.stack([np.sort(np.random.default_rng(seed + b).choice(n, size=min(K, n), replace=False))
                    for b in range(B)]).astype(np.int32)
    if K > n:
        idx = np.concatenate([idx, -np.ones((B, K - n), np.int32)], axis=1)
    q = torch.randn((B, H, 512), generator=g).to(torch.bfloat16)
    swa = torch.randn((B, W, 512), generator=g).to(torch.float8_e4m3fn)
    return kv, codes, scales, idx, q, swa


@pytest.mark.parametrize("B,H,K,W,n", [(1, 16, 64, 128, 4096), (3, 64, 512, 128, 3000),
                                       (2, 64, 100, 5, 300), (2, 40, 512, 0, 700),
                                       (1, 64, 0, 128, 10), (2, 8, 7, 1, 20),
                                       (24, 32, 512, 128, 2000),
                                       # more than 8 splits: partials and the merge kernel
                                       (2, 64, 2048, 128, 4000)])
def test_attention_decode(B, H, K, W, n):
    kv, codes, scales, idx, q, swa = _attn_case(B, H, K, W, n, seed=B * 100 + K + W)
    out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, n, K))
    tau = 1 / math.sqrt(512)
    C().sparse_attn_decode("full", q.to(dev), codes, scales,
                           torch.from_numpy(idx).to(dev) if K else None,
                           swa.to(dev) if W else None, out, ws, scale=tau)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    for b in range(B):
        sel = [i for i in idx[b] if i >= 0]
        rows = [oracle_main_rows(bits16(kv[b, sel]))] if sel else []
        if W:
            rows.append(O.e4m3_array_to_f64(bits8(swa[b])).reshape(W, 512))
        allrows = np.concatenate(rows) if rows else np.zeros((0, 512))
        ref = O.attention(O.bf16_array_to_f64(bits16(q[b])).reshape(H, 512), allrows, tau)
        check_attention(out[b].cpu().numpy(), ref, f"b={b}")


def test_attention_decode_with_no_rows():
    """K = 0 and W = 0: the softmax of an empty set contributes nothing. The output is zero
    (the oracle's value), and a partial result is (maximum -inf, sum 0, output 0)."""
    g = _gen(61)
    B, H = 3, 64
    q = torch.randn((B, H, 512), generator=g).to(torch.bfloat16).to(dev)
    codes = torch.zeros((B, 8, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, 8, 32), dtype=torch.uint8, device=dev)
    idx = torch.empty((B, 0), dtype=torch.int32, device=dev)
    out = torch.full((B, H, 512), 7.0, dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, 8, 0))
    C().sparse_attn_decode("full", q, codes, scales, idx, None, out, ws)
    o = torch.full((B, H, 512), 7.0, dtype=torch.float32, device=dev)
    ml = torch.full((B, 2, H), 7.0, dtype=torch.float32, device=dev)
    C().sparse_attn_decode_partial("full", q, codes, scales, idx, None, o, ml, ws)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    ref = O.attention(O.bf16_array_to_f64(bits16(q[0])).reshape(H, 512), np.zeros((0, 512)), 0.1)
    assert np.all(ref == 0.0)
    assert torch.count_nonzero(out).item() == 0
    assert torch.count_nonzero(o).item() == 0
    assert torch.all(ml[:, 0] == -float("inf")) and torch.all(ml[:, 1] == 0)


def test_attention_reuse_equals_full_and_bad_index_flag():
    B, H, K, W, n = 2, 64, 512, 128, 2000
    kv, codes, scales, idx, q, swa = _attn_case(B, H, K, W, n, seed=77)
    tI = torch.from_numpy(idx).to(dev)
    outs = []
    for mode in ("full", "reuse", "reindex"):
        out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
        ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, n, K))
        C().sparse_attn_decode(mode, q.to(dev), codes, scales, tI, swa.to(dev), out, ws)
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    bad = tI.clone()
    bad[0, 3] = n + 5          # outside the cache: skipped + flagged, no fault
    bad[1, 4] = -7
    out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, n, K))
    C().sparse_attn_decode("full", q.to(dev), codes, scales, bad, swa.to(dev), out, ws)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) & C().DEV_BAD_INDEX
    assert torch.isfinite(out).all()


def test_attention_swa_valid_prefix():
    B, H, K, W, n = 2, 16, 64, 128, 500
    kv, codes, scales, idx, q, swa = _attn_case(B, H, K, W, n, seed=5)
    valid = torch.tensor([128, 17], dtype=torch.int32, device=dev)
    out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, n, K))
    C().sparse_attn_decode("full", q.to(dev), codes, scales, torch.from_numpy(idx).to(dev),
                           swa.to(dev), out, ws, swa_valid=valid)
    torch.cuda.synchronize()
    for b in range(B):
        sel = [i for i in idx[b] if i >= 0]
        rows = np.concatenate([oracle_main_rows(bits16(kv[b, sel])),
                               O.e4m3_array_to_f64(bits8(swa[b, W - int(valid[b]):])).reshape(-1, 512)])
        ref = O.attention(O.bf16_array_to_f64(bits16(q[b])).reshape(H, 512), rows, 512 ** -0.5)
        check_attention(out[b].cpu().numpy(), ref, f"b={b}")


def test_attention_decode_one_split_dominates():
    """A window row aligned with head 5's query: the last of the four splits holds a logit
    far above every other split's, so the cluster merge weighs the others by ~2^-200."""
    B, H, K, W, n = 2, 64, 512, 128, 3000
    kv, codes, scales, idx, q, swa = _attn_case(B, H, K, W, n, seed=81)
    for b in range(B):
        swa[b, 120] = (torch.sign(q[b, 5].float()) * 8).to(torch.float8_e4m3fn)
    out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(1, B, 1, H, n, K))
    tau = 1 / math.sqrt(512)
    C().sparse_attn_decode("full", q.to(dev), codes, scales, torch.from_numpy(idx).to(dev),
                           swa.to(dev), out, ws, scale=tau)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    out = out.cpu().numpy()
    for b in range(B):
        rows = np.concatenate([oracle_main_rows(bits16(kv[b, idx[b]])),
                               O.e4m3_array_to_f64(bits8(swa[b])).reshape(W, 512)])
        ref = O.attention(O.bf16_array_to_f64(bits16(q[b])).reshape(H, 512), rows, tau)
        others = [h for h in range(H) if h != 5]
        check_attention(out[b, 5:6], ref[5:6], f"b={b} head 5")
        check_attention(out[b, others], ref[others], f"b={b} other heads")
        planted = O.e4m3_array_to_f64(bits8(swa[b, 120]))
        assert np.max(np.abs(ref[5] - planted)) <= 1e-6 * np.max(np.abs(planted))


# ---- prefill ---------------------------------------------------------------------------------

def test_prefill_indexer_and_attention_small():
    g = _gen(11)
    B, T, H_I, K, H, W, r = 2, 8, 64, 64, 64, 16, 2
    q_pos0 = [300, 5]
    cap = (max(q_pos0) + T) // r
    k_I = _keys(B, cap, torch.float8_e4m3fn, g)
    q_I = torch.randn((B, T, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, T, H_I), generator=g)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, T, H_I, cap, K))
    qp = torch.tensor(q_pos0, dtype=torch.int32, device=dev)
    C().index_score_topk("full", q_I.to(dev), w.to(dev), k_I.to(dev), K, idx, ws, q_pos0=qp, ratio=r)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    idx_np = idx.cpu().numpy()
    for b in range(B):
        for t in range(T):
            n = O.prefill_visible(q_pos0[b] + t, r)
            s = O.index_scores(raw_qk(q_I[b, t]), w[b, t].numpy(), raw_qk(k_I[b, :n]), O.E4M3)
            check_topk(idx_np[b, t], s, np.arange(n), K, f"b={b} t={t}")
    # attention with the oracle's indices
    kv = torch.randn((B, cap, 512), generator=g).to(torch.bfloat16)
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    C().quantize_kv(kv.to(dev), torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    q = torch.randn((B, T, H, 512), generator=g).to(torch.bfloat16)
    swa = torch.randn((B, W - 1 + T, 512), generator=g).to(torch.float8_e4m3fn)
    # the oracle's whole prefill query: visibility, scores, Top-K, window rows, attention
    oidx = np.zeros((B, T, K), np.int32)
    refs = {}
    for b in range(B):
        for t in range(T):
            oidx[b, t], refs[b, t] = O.prefill_query(
                raw_qk(q_I[b, t]), w[b, t].numpy(), raw_qk(k_I[b]), O.E4M3, bits16(kv[b]),
                bits16(q[b, t]), bits8(swa[b]), q_pos0[b], t, r, K, W, 512 ** -0.5)
    out = torch.empty((B, T, H, 512), dtype=torch.float32, device=dev)
    wsa = C().new_workspace(C().workspace_bytes(2, B, T, H, cap, K))
    C().sparse_attn_prefill(q.to(dev), codes, scales, torch.from_numpy(oidx).to(dev), swa.to(dev),
                            out, wsa, W, q_pos0=qp)
    torch.cuda.synchronize()
    assert C().read_device_status(wsa) == 0
    for b in range(B):
        for t in range(T):
            check_attention(out[b, t].cpu().numpy(), refs[b, t], f"b={b} t={t}")


def test_prefill_attention_padded_heads_ragged_chunks_and_rescale():
    """24 query heads (padded to the kernel's 64), 200 selected entries with 10 empty slots
    plus the 128-row window (three chunks of rows, the last one partial), and one window row
    aligned with head 0 whose logit exceeds every earlier one by far: the running maximum of
    that head rises in the last chunk and its accumulator columns are rescaled."""
    g = _gen(80)
    B, T, H, K, W, r = 1, 6, 24, 200, 128, 2
    q_pos0 = [600]
    cap = (q_pos0[0] + T) // r
    kv = torch.randn((B, cap, 512), generator=g).to(torch.bfloat16)
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    C().quantize_kv(kv.to(dev), torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    q = torch.randn((B, T, H, 512), generator=g).to(torch.bfloat16)
    q[:, :, 0] = q[:, :1, 0]                       # head 0: one vector for every token
    swa = torch.randn((B, W - 1 + T, 512), generator=g).to(torch.float8_e4m3fn)
    swa[0, 100] = (torch.sign(q[0, 0, 0].float()) * 8).to(torch.float8_e4m3fn)
    rng = np.random.default_rng(80)
    oidx = np.full((B, T, K), -1, np.int32)
    for t in range(T):
        n = O.prefill_visible(q_pos0[0] + t, r)
        oidx[0, t, :K - 10] = np.sort(rng.choice(n, K - 10, replace=False))
    out = torch.empty((B, T, H, 512), dtype=torch.float32, device=dev)
    wsa = C().new_workspace(C().workspace_bytes(2, B, T, H, cap, K))
    C().sparse_attn_prefill(q.to(dev), codes, scales, torch.from_numpy(oidx).to(dev), swa.to(dev),
                            out, wsa, W, q_pos0=torch.tensor(q_pos0, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert C().read_device_status(wsa) == 0
    out = out.cpu().numpy()
    for t in range(T):
        _, ref = O.prefill_query(None, None, None, None, bits16(kv[0]), bits16(q[0, t]),
                                 bits8(swa[0]), q_pos0[0], t, r, K, W, 512 ** -0.5,
                                 idx_override=oidx[0, t])
        # each against its own scale: head 0's output is the planted row (magnitude 8)
        check_attention(out[0, t, :1], ref[:1], f"t={t} head 0")
        check_attention(out[0, t, 1:], ref[1:], f"t={t} heads 1..")
        # head 0 is the planted window row, as the oracle says
        row = O.e4m3_array_to_f64(bits8(swa[0, 100]))
        assert np.max(np.abs(ref[0] - row)) <= 1e-6 * np.max(np.abs(row))


def test_prefill_indexer_back_to_back_calls():
    """Consecutive prefill index calls in one process, each launched while the previous
    kernel may still run: one workspace reused with a different tile prefix (other query
    positions), then a freshly zeroed one. Every call must read the prefix its own prep
    kernel wrote, not what the workspace held before."""
    g = _gen(23)
    B, T, H_I, K, r = 2, 256, 64, 256, 2
    cap = 6000
    k_I = _keys(B, cap, torch.float8_e4m3fn, g).to(dev)
    q_I = torch.randn((B, T, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, T, H_I), generator=g)
    q_Id, wd = q_I.to(dev), w.to(dev)
    wsb = C().workspace_bytes(0, B, T, H_I, cap, K)
    ws = C().new_workspace(wsb)
    pick = [0, 1, 77, T - 1]
    for q_pos0, fresh in (([4000, 900], False), ([11000, 2300], False), ([7000, 11700], True)):
        if fresh:
            ws = C().new_workspace(wsb)
        idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
        qp = torch.tensor(q_pos0, dtype=torch.int32, device=dev)
        C().index_score_topk("full", q_Id, wd, k_I, K, idx, ws, q_pos0=qp, ratio=r)
        torch.cuda.synchronize()
        assert C().read_device_status(ws) == 0, q_pos0
        idx_np = idx.cpu().numpy()
        for b in range(B):
            for t in pick:
                n = O.prefill_visible(q_pos0[b] + t, r)
                s = O.index_scores(raw_qk(q_I[b, t]), w[b, t].numpy(),
                                   raw_qk(k_I[b, :n].cpu()), O.E4M3)
                check_topk(idx_np[b, t], s, np.arange(n), K, f"q_pos0={q_pos0} b={b} t={t}")


# ---- bounded waits -------------------------------------------------------------------------

def test_bounded_wait_reports_timeout():
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    C().debug_bounded_wait(st, 20_000_000)   # 20 ms, nothing ever signals the barrier
    torch.cuda.synchronize()
    assert int(st.item()) & C().DEV_TIMEOUT
    x = torch.ones(4, device=dev)
    assert float((x * 2).sum()) == 8.0   # the context is still healthy
