"""GPU parity of the compact 68-byte indexer keys (csa2_quantize_keys_fp4 and
csa2_index_score_topk with CSA2_DTYPE_E4M3_FP4KEY) with the oracle, through the C ABI.

The quantizer's decisions are taken in fp32 on both sides (bit-exact codes and scales);
scores are compared within the fp32-accumulation bound of the existing scan tests, and the
selections with the Top-K near-tie rule."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import bits8, bits16, check_topk

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


def _keys_bf16(B, n, g):
    # per-key magnitudes over several binades exercise the fp32 scale
    return (torch.randn((B, n, 128), generator=g) *
            torch.exp(torch.randn((B, n, 1), generator=g) * 2)).to(torch.bfloat16)


def _compact(k, cap, dst):
    B = k.shape[0]
    keys = C().Fp4Keys(B, cap)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    C().quantize_keys_fp4(k.to(dev), torch.tensor(dst, dtype=torch.int32, device=dev), keys,
                          status=st)
    torch.cuda.synchronize()
    return keys, int(st.item())


def test_quantize_keys_bit_exact_and_offsets():
    g = _gen(41)
    B, n, cap = 3, 333, 400
    dst = [0, 50, 67]
    k = _keys_bf16(B, n, g)
    k[1, 3] = 0                                        # a zero key: scale 0, zero codes
    keys, st = _compact(k, cap, dst)
    assert st == 0
    codes = keys.codes.cpu().numpy()
    scales = keys.scales.cpu().numpy()
    for b in range(B):
        oc, os_ = O.quantize_keys_fp4(bits16(k[b]))
        np.testing.assert_array_equal(codes[b, dst[b]:dst[b] + n], oc, f"codes b={b}")
        np.testing.assert_array_equal(scales[b, dst[b]:dst[b] + n].view(np.uint32),
                                      os_.view(np.uint32), f"scales b={b}")
    assert codes[1, :50].sum() == 0 and scales[1, :50].sum() == 0
    assert scales[1, 53] == 0 and codes[1, 53].sum() == 0
    # an offset past the capacity: those keys are skipped and flagged
    keys2, st2 = _compact(k[:, :10], 20, [0, 15, 5])
    assert st2 & C().DEV_BAD_INDEX
    oc, _ = O.quantize_keys_fp4(bits16(k[1, :5]))
    np.testing.assert_array_equal(keys2.codes[1, 15:20].cpu().numpy(), oc)


def _decode(q_I, w, keys, n_vis, K, pool_blocks=0):
    B, T, H_I, _ = q_I.shape
    cap = keys.cap
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    scores = torch.zeros((B, T, cap), dtype=torch.float32, device=dev)
    pool = torch.empty((B, T, pool_blocks * 8), dtype=torch.int32, device=dev) if pool_blocks else None
    ws = C().new_workspace(C().workspace_bytes(0, B, T, H_I, cap, K, pool_blocks))
    C().index_score_topk("full", q_I.to(dev), w.to(dev), keys, K, idx, ws,
                         n_vis0=torch.tensor(n_vis, dtype=torch.int32, device=dev),
                         pool_out=pool, pool_blocks=pool_blocks, scores_out=scores)
    torch.cuda.synchronize()
    return (idx.cpu().numpy(), scores.cpu().numpy(),
            pool.cpu().numpy() if pool is not None else None, C().read_device_status(ws))


def _oracle_scores(q, w, codes, scales, n):
    s = O.index_scores_fp4key(q, w, codes[:n], scales[:n])
    qd = O.e4m3_array_to_f64(q.ravel()).reshape(q.shape)
    kd = O.dequant_keys_fp4(codes[:n], scales[:n])
    mag = np.abs(kd) @ np.abs(qd).T @ w.astype(np.float64)
    return s, mag


@pytest.mark.parametrize("H_I,K,n_list", [(64, 512, [4096, 1000, 129, 7]),
                                          (16, 64, [511, 512, 513]),
                                          (64, 512, [70001, 40000])])
def test_full_decode_with_compact_keys(H_I, K, n_list):
    g = _gen(sum(n_list) + H_I)
    B, cap = len(n_list), max(n_list)
    k = _keys_bf16(B, cap, g)
    keys, st = _compact(k, cap, [0] * B)
    assert st == 0
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, 1, H_I), generator=g)
    idx, scores, _, st = _decode(q_I, w, keys, n_list, K)
    assert st == 0
    codes = keys.codes.cpu().numpy()
    kscale = keys.scales.cpu().numpy()
    for b, n in enumerate(n_list):
        q = bits8(q_I[b, 0])
        s, mag = _oracle_scores(q, w[b, 0].numpy(), codes[b], kscale[b], n)
        np.testing.assert_array_less(np.abs(scores[b, 0, :n] - s), 2e-6 * mag + 1e-30)
        check_topk(idx[b, 0], s, np.arange(n), K, f"b={b} n={n}")


def test_pool_with_compact_keys():
    g = _gen(43)
    B, n, H_I, K, nblk = 2, 20000, 64, 512, 512
    k = _keys_bf16(B, n, g)
    keys, _ = _compact(k, n, [0, 0])
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, 1, H_I), generator=g)
    n_list = [n, n - 5]
    idx, scores, pool, st = _decode(q_I, w, keys, n_list, K, pool_blocks=nblk)
    assert st == 0
    codes = keys.codes.cpu().numpy()
    kscale = keys.scales.cpu().numpy()
    for b in range(B):
        s, _ = _oracle_scores(bits8(q_I[b, 0]), w[b, 0].numpy(), codes[b], kscale[b], n_list[b])
        check_topk(idx[b, 0], s, np.arange(n_list[b]), K, f"full b={b}")
        nb = (n_list[b] + 7) // 8
        bmax = np.array([s[8 * c:8 * c + 8].max() for c in range(nb)])
        got_blocks = np.unique(pool[b, 0][pool[b, 0] >= 0] // 8)
        gb = np.full(nblk, -1)
        gb[: len(got_blocks)] = got_blocks
        check_topk(gb, bmax, np.arange(nb), nblk, f"pool b={b}")


def test_prefill_with_compact_keys():
    g = _gen(44)
    B, T, H_I, K, r = 2, 8, 64, 64, 2
    q_pos0 = [300, 5]
    cap = (max(q_pos0) + T) // r
    k = _keys_bf16(B, cap, g)
    keys, _ = _compact(k, cap, [0, 0])
    q_I = torch.randn((B, T, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w = torch.rand((B, T, H_I), generator=g)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, T, H_I, cap, K))
    qp = torch.tensor(q_pos0, dtype=torch.int32, device=dev)
    C().index_score_topk("full", q_I.to(dev), w.to(dev), keys, K, idx, ws, q_pos0=qp, ratio=r)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    idx = idx.cpu().numpy()
    codes = keys.codes.cpu().numpy()
    kscale = keys.scales.cpu().numpy()
    for b in range(B):
        for t in range(T):
            n = O.prefill_visible(q_pos0[b] + t, r)
            s, _ = _oracle_scores(bits8(q_I[b, t]), w[b, t].numpy(), codes[b], kscale[b], n)
            check_topk(idx[b, t], s, np.arange(n), K, f"b={b} t={t}")


def test_reindex_with_compact_keys():
    """Reindex over compact keys: a second layer's query rescored inside the oracle's pool
    (pool rows gathered with 8-byte copies into the unpacked operand layout, each key's
    scale looked up through its pool position)."""
    g = _gen(45)
    B, n, H_I, K, nblk = 2, 20000, 64, 512, 512
    k = _keys_bf16(B, n, g)
    keys, _ = _compact(k, n, [0, 0])
    codes = keys.codes.cpu().numpy()
    kscale = keys.scales.cpu().numpy()
    q1 = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w1 = torch.rand((B, 1, H_I), generator=g)
    q2 = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn)
    w2 = torch.rand((B, 1, H_I), generator=g)
    n_list = [n, n - 13]
    pool_o = np.stack([O.pool(_oracle_scores(bits8(q1[b, 0]), w1[b, 0].numpy(), codes[b], kscale[b],
                                             n_list[b])[0], nblk) for b in range(B)])[:, None, :]
    P = pool_o.shape[-1]
    idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    sc = torch.zeros((B, 1, P), dtype=torch.float32, device=dev)
    ws = C().new_workspace(C().workspace_bytes(0, B, 1, H_I, P, K))
    C().index_score_topk("reindex", q2.to(dev), w2.to(dev), keys, K, idx, ws,
                         n_vis0=torch.tensor(n_list, dtype=torch.int32, device=dev),
                         pool_in=torch.from_numpy(pool_o.astype(np.int32)).to(dev), scores_out=sc)
    torch.cuda.synchronize()
    assert C().read_device_status(ws) == 0
    idx = idx.cpu().numpy()
    sc = sc.cpu().numpy()
    for b in range(B):
        slots = np.nonzero(pool_o[b, 0] >= 0)[0]
        ids = pool_o[b, 0][slots]
        s2 = O.index_scores_fp4key(bits8(q2[b, 0]), w2[b, 0].numpy(), codes[b], kscale[b], rows=ids)
        qd = O.e4m3_array_to_f64(bits8(q2[b, 0]).ravel()).reshape(H_I, 128)
        kd = O.dequant_keys_fp4(codes[b][ids], kscale[b][ids])
        mag = np.abs(kd) @ np.abs(qd).T @ w2[b, 0].numpy().astype(np.float64)
        np.testing.assert_array_less(np.abs(sc[b, 0, slots] - s2), 2e-6 * mag + 1e-30)
        check_topk(idx[b, 0], s2, ids, K, f"reindex b={b}")
