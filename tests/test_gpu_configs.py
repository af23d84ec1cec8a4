"""GPU parity of the whole CSA2 path at the five workloads' full sizes, in the launch
configuration bench.py times (same library calls, same shapes), against the CPU oracle on
sampled outputs the oracle computes one by one:

  decode_full_b1_ctx4k          every output
  decode_full_b32_ctx64k_r2     every query's Top-512; attention and FP4 codes on samples
  decode_full_b32_ctx64k_r2_key68  the same with compact 68-byte indexer keys
  decode_group4_b64_ctx256k     Full + 3 Reuse: 16 sampled queries, every layer
  decode_pool_reindex_b4_ctx1m  Full + pool + Reindex on every query; planted-key recall
  prefill_b2_t4k_ctx128k_r2     ~90 sampled query tokens per sequence (first, last, every
                                64th, a seeded scatter) through the oracle's prefill query

Where the step's own Top-K differs from the oracle's inside the near-tie exemption, the
step's own attention output is checked against the oracle's attention over those picks.

Inputs are drawn on the GPU by the seeded generator; the oracle reads copies of them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import bits16, bits8, check_attention, check_topk, odt, raw_qk

pytestmark = pytest.mark.gpu
dev = "cuda"
SEED = 4321


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    torch.cuda.empty_cache()


def _bench():
    import bench
    return bench


def _oracle_scores(state, li, b, rows=None):
    L = state.layers[li]
    w = state.w
    if w.key_format == "fp4":
        return O.index_scores_fp4key(bits8(L["q_I"][b, 0]), L["w"][b, 0].cpu().numpy(),
                                     state.k_I.codes[b, :w.N].cpu().numpy(),
                                     state.k_I.scales[b, :w.N].cpu().numpy(), rows=rows)
    return O.index_scores(raw_qk(L["q_I"][b, 0]), L["w"][b, 0].cpu().numpy(),
                          raw_qk(state.k_I[b, :w.N]), odt(L["q_I"]), rows=rows)


def _oracle_attention(state, li, b, idx_row):
    bench = _bench()
    w = state.w
    L = state.layers[li]
    sel = [int(i) for i in idx_row if i >= 0]
    src = bench._main_rows(w, state.seed, b, state.dev)
    kvb = bits16(src[sel]) if sel else np.zeros((0, 512), np.uint16)
    c, s = O.quantize_entries(kvb)
    rows = np.concatenate([O.dequant_entries(c, s),
                           O.e4m3_array_to_f64(bits8(L["swa"][b])).reshape(-1, 512)])
    return O.attention(O.bf16_array_to_f64(bits16(L["q"][b])).reshape(w.H, 512), rows, state.tau)


def _gpu_attention(state, li, idx_rows):
    """The same decode attention call on given indices [B, K] (oracle indices)."""
    from fp4_compressed_sparse_quantize_b200 import csa2
    w = state.w
    L = state.layers[li]
    out = torch.empty((w.B, w.H, 512), dtype=torch.float32, device=dev)
    csa2.sparse_attn_decode("full", L["q"], state.codes, state.scales,
                            torch.from_numpy(np.ascontiguousarray(idx_rows)).to(dev), L["swa"], out,
                            state.ws_attn, scale=state.tau)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _run_decode(name, sample_b):
    bench = _bench()
    from fp4_compressed_sparse_quantize_b200 import csa2, synth
    w = synth.WORKLOADS[name]
    state = bench.Decode(w, SEED, torch.device(dev))
    for _ in range(2):
        state.step()
    torch.cuda.synchronize()
    assert csa2.read_device_status(state.ws_idx) == 0
    assert csa2.read_device_status(state.ws_attn) == 0
    return state


def _check_decode(state, sample_b, check_codes_b=()):
    w = state.w
    bench = _bench()
    # FP4 cache bit-exact on sampled sequences
    for b in check_codes_b:
        src = bench._main_rows(w, state.seed, b, state.dev)
        rc, rs = O.quantize_entries(bits16(src))
        np.testing.assert_array_equal(bits8(state.codes[b]), rc)
        np.testing.assert_array_equal(bits8(state.scales[b]), rs)
    kinds = []
    oracle_idx = {}
    for li, mode in enumerate(w.layers):
        if mode == "reuse":
            # Reuse: the GPU output of this layer must equal attention over the same indices
            continue
        for b in sample_b:
            if mode == "full":
                s = _oracle_scores(state, li, b)
                ids = np.arange(w.N)
            else:
                pool_o = O.pool(_oracle_scores(state, 0, b), 2048)
                ids = pool_o[pool_o >= 0]
                s = _oracle_scores(state, li, b, rows=ids)
            kinds.append(check_topk(state.idx[li][b, 0].cpu().numpy(), s, ids, w.K,
                                    f"{w.name} layer {li} b={b}"))
            oracle_idx[(li, b)] = O.topk(s, w.K, ids if mode != "full" else None)
    # attention: the oracle's indices through the same GPU call, every sampled query/layer
    cur = None
    for li, mode in enumerate(w.layers):
        if mode != "reuse":
            cur = li
        oi = np.stack([oracle_idx.get((cur, b), np.full(w.K, -1, np.int32)) for b in range(w.B)])
        g = _gpu_attention(state, li, oi)
        e2e = state.out[li].cpu().numpy()
        for b in sample_b:
            ref = _oracle_attention(state, li, b, oi[b])
            check_attention(g[b], ref, f"{w.name} layer {li} b={b}")
            own = state.idx[cur][b, 0].cpu().numpy()
            if np.array_equal(own, oi[b]):
                np.testing.assert_array_equal(e2e[b], g[b])   # same indices -> same output
            else:
                # picks that differ inside the near-tie exemption: the step's own output
                # against the oracle's attention over those same picks
                check_attention(e2e[b], _oracle_attention(state, li, b, own),
                                f"{w.name} layer {li} b={b} (own picks)")
    return kinds


def test_decode_full_b1_ctx4k():
    state = _run_decode("decode_full_b1_ctx4k", [0])
    _check_decode(state, [0], check_codes_b=[0])


def test_decode_full_b32_ctx64k_r2():
    state = _run_decode("decode_full_b32_ctx64k_r2", None)
    kinds = _check_decode(state, list(range(32)), check_codes_b=[0, 31])
    assert kinds.count("exact") >= 24, kinds


def test_decode_full_b32_ctx64k_r2_key68():
    """The same decode step with compact 68-byte indexer keys: every query's Top-512 against
    the oracle's scores over the keys' decoded values, attention on samples; the compact key
    cache against the oracle's quantiser on two sequences."""
    from fp4_compressed_sparse_quantize_b200 import synth
    state = _run_decode("decode_full_b32_ctx64k_r2_key68", None)
    w = state.w
    kb, _ = synth.indexer_keys(w, SEED, torch.device(dev))
    for b in (0, 31):
        oc, os_ = O.quantize_keys_fp4(bits16(kb[b]))
        np.testing.assert_array_equal(state.k_I.codes[b].cpu().numpy(), oc)
        np.testing.assert_array_equal(state.k_I.scales[b].cpu().numpy().view(np.uint32),
                                      os_.view(np.uint32))
    del kb
    kinds = _check_decode(state, list(range(32)), check_codes_b=[0])
    assert kinds.count("exact") >= 24, kinds


def test_decode_group4_b64_ctx256k():
    state = _run_decode("decode_group4_b64_ctx256k", None)
    sample = sorted(set([0, 63] + np.random.default_rng(SEED).choice(64, 14, replace=False).tolist()))
    _check_decode(state, sample, check_codes_b=[0, 63])
    # the three Reuse layers attended over exactly the Full layer's indices
    for li in (1, 2, 3):
        assert state.idx[li] is not None


def test_decode_pool_reindex_b4_ctx1m():
    state = _run_decode("decode_pool_reindex_b4_ctx1m", None)
    w = state.w
    _check_decode(state, list(range(w.B)))
    pool = state.pool.cpu().numpy()
    for b in range(w.B):
        s = _oracle_scores(state, 0, b)
        nb = (w.N + 7) // 8
        bmax = s.reshape(nb, 8).max(axis=1)
        got = np.unique(pool[b, 0][pool[b, 0] >= 0] // 8)
        gb = np.full(2048, -1)
        gb[: len(got)] = got
        check_topk(gb, bmax, np.arange(nb), 2048, f"pool b={b}")
        planted = state.planted[b].numpy()
        for li in (0, 1):
            rec = len(set(planted.tolist()) & set(state.idx[li][b, 0].cpu().numpy().tolist()))
            assert rec == len(planted), f"layer {li} b={b}: planted recall {rec}/{len(planted)}"
        assert set(planted.tolist()) <= set(pool[b, 0].tolist())


def test_prefill_b2_t4k_ctx128k_r2():
    from fp4_compressed_sparse_quantize_b200 import csa2, synth
    w = synth.WORKLOADS["prefill_b2_t4k_ctx128k_r2"]
    bench = _bench()
    B, T, cap, K, H, W = w.B, w.T, w.cap, w.K, w.H, synth.WINDOW
    L = synth.layer_inputs(w, 0, SEED, dev)
    k_I, _ = synth.indexer_keys(w, SEED, dev)
    # cached entries quantised once, the new ones by the prefill step itself
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    src = torch.stack([bench._main_rows(w, SEED, b, dev) for b in range(B)])
    n_old = w.ctx // w.ratio
    csa2.quantize_kv(src[:, :n_old], torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    q_pos0 = synth.prefill_positions(w, dev)
    csa2.quantize_kv(src[:, n_old:], torch.full((B,), n_old, dtype=torch.int32, device=dev),
                     codes, scales)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    ws = csa2.new_workspace(csa2.workspace_bytes(0, B, T, w.H_I, cap, K))
    csa2.index_score_topk("full", L["q_I"], L["w"], k_I, K, idx, ws, q_pos0=q_pos0, ratio=w.ratio)
    out = torch.empty((B, T, H, 512), dtype=torch.float32, device=dev)
    wsa = csa2.new_workspace(csa2.workspace_bytes(2, B, T, H, cap, K))
    csa2.sparse_attn_prefill(L["q"], codes, scales, idx, L["swa"], out, wsa, W, q_pos0=q_pos0)
    torch.cuda.synchronize()
    assert csa2.read_device_status(ws) == 0 and csa2.read_device_status(wsa) == 0
    rc, rs = O.quantize_entries(bits16(src[1, n_old:]))
    np.testing.assert_array_equal(bits8(codes[1, n_old:]), rc)
    np.testing.assert_array_equal(bits8(scales[1, n_old:]), rs)
    # sampled tokens: first, last, every 64th, and a seeded scatter
    rng = np.random.default_rng(SEED)
    ts = sorted(set([0, 1, T - 1] + list(range(63, T, 64)) + rng.integers(0, T, 24).tolist()))
    idx_np = idx.cpu().numpy()
    oidx = idx_np.copy()
    refs = {}
    qpos = q_pos0.cpu().numpy()
    for b in range(B):
        kb = raw_qk(k_I[b])
        srcb = bits16(src[b])
        swab = bits8(L["swa"][b])
        for t in ts:
            qi = raw_qk(L["q_I"][b, t])
            wt = L["w"][b, t].cpu().numpy()
            n = O.prefill_visible(int(qpos[b]) + t, w.ratio)
            s = O.index_scores(qi, wt, kb[:n], O.E4M3)
            check_topk(idx_np[b, t], s, np.arange(n), K, f"prefill b={b} t={t}")
            oidx[b, t], refs[b, t] = O.prefill_query(qi, wt, kb, O.E4M3, srcb,
                                                     bits16(L["q"][b, t]), swab, int(qpos[b]), t,
                                                     w.ratio, K, W, 1 / math.sqrt(512))
    # attention with the oracle's indices at the sampled tokens
    out2 = torch.empty_like(out)
    csa2.sparse_attn_prefill(L["q"], codes, scales, torch.from_numpy(oidx).to(dev), L["swa"],
                             out2, wsa, W, q_pos0=q_pos0)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    got2 = out2.cpu().numpy()
    for b in range(B):
        srcb = bits16(src[b])
        kb = raw_qk(k_I[b])
        swab = bits8(L["swa"][b])
        for t in ts:
            check_attention(got2[b, t], refs[b, t], f"prefill b={b} t={t}")
            if np.array_equal(oidx[b, t], idx_np[b, t]):
                np.testing.assert_array_equal(got[b, t], got2[b, t])
            else:
                # the product's own picks (inside the near-tie exemption) through the oracle
                _, ref_own = O.prefill_query(None, None, kb, O.E4M3, srcb,
                                             bits16(L["q"][b, t]), swab, int(qpos[b]), t,
                                             w.ratio, K, W, 1 / math.sqrt(512),
                                             idx_override=idx_np[b, t])
                check_attention(got[b, t], ref_own, f"prefill own picks b={b} t={t}")
