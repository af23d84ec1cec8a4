"""Context-parallel Full-layer selection (one shard of the entries per rank).

CPU (gloo, world size 2): the decomposition itself. Each rank selects on its shard with the
oracle, the lists travel through cp.all_gather_last, and the merge by the oracle's own
(score desc, index asc) selection equals the oracle's selection over the whole context, for
the Top-K and for the block pool, with planted exact ties at both boundaries.

GPU (one device, shards run one after another): the cp_* kernels. The selection merged from
G shard scans is bit-identical to the single-scan selection (indices and pool) and passes
the oracle's Top-K and pool checks; cp.select and cp.attend run over a one-rank NCCL group.
cp.attend's own logic (local indices, the window on one rank, the exchange) also runs over
two gloo ranks on CPU with the kernels replaced by oracle stand-ins."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp4_compressed_sparse_quantize_b200 import cp
from oracle import oracle as O


def test_shards_cover_and_align():
    for n in (0, 1, 7, 8, 9, 4095, 32768, 32773, 1 << 20):
        for g in (1, 2, 3, 4, 7, 8):
            sh = cp.shards(n, g)
            assert len(sh) == g and sh[0][0] == 0 and sh[-1][1] == n
            for (a, b), (c, d) in zip(sh, sh[1:]):
                assert b == c
            sizes = [b - a for a, b in sh]
            assert all(a % 8 == 0 for a, _ in sh)
            assert max(sizes) - min(sizes) <= 8


def test_local_counts():
    n_vis = torch.tensor([0, 5, 100, 260], dtype=torch.int32)
    assert cp.local_counts(n_vis, 96, 200).tolist() == [0, 0, 4, 104]
    assert cp.local_counts(n_vis, 0, 64).tolist() == [0, 5, 64, 64]


def _scores(seed, n):
    g = torch.Generator().manual_seed(seed)
    s = torch.randn(n, generator=g, dtype=torch.float64).abs().numpy()
    s[100:104] = s[7]                    # exact ties with a low-index entry
    s[n // 2 + 3] = s[7]                 # ... and one in the second shard
    s[np.argsort(-s)[60:70]] = s[np.argsort(-s)[60]]   # a tie run across the K boundary
    return s


def _local(s, lo, hi, K, nblk):
    """One shard's selections as exchange lists (global ids, -1 padded)."""
    loc = s[lo:hi]
    ti = O.topk(loc, K)
    v = ti >= 0
    cand_s = np.where(v, loc[np.maximum(ti, 0)], 0.0)
    cand_i = np.where(v, ti + lo, -1).astype(np.int32)
    pos = O.pool(loc, nblk)
    pos = pos[pos >= 0]
    blocks = np.unique(pos // 8)
    bmax = np.array([loc[b * 8:min(b * 8 + 8, hi - lo)].max() for b in blocks])
    cb = np.zeros(nblk)
    ci = np.full(nblk, -1, np.int32)
    cb[:len(blocks)] = bmax
    ci[:len(blocks)] = blocks + lo // 8
    return cand_s, cand_i, cb, ci


def _merge(cand_s, cand_i, K):
    v = cand_i >= 0
    return O.topk(cand_s[v], K, ids=cand_i[v])


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for n, K, nblk in ((5000, 64, 32), (4093, 64, 600), (130, 64, 8)):
            s = _scores(n, n)
            lo, hi = cp.shards(n, world)[rank]
            cs, ci, cb, cblk = _local(s, lo, hi, K, nblk)
            t = [torch.from_numpy(x) for x in (cs, ci, cb, cblk)]
            g = [cp.all_gather_last(x) for x in t]
            idx = _merge(g[0].numpy(), g[1].numpy(), K)
            blocks = _merge(g[2].numpy(), g[3].numpy(), nblk)
            blocks = blocks[blocks >= 0]
            pool = np.concatenate([np.arange(b * 8, min(b * 8 + 8, n)) for b in blocks]) \
                if len(blocks) else np.zeros(0, np.int64)
            ref_pool = O.pool(s, nblk)
            res.append((np.array_equal(idx, O.topk(s, K)),
                        np.array_equal(pool, ref_pool[ref_pool >= 0])))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def _free_port():
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    p = sk.getsockname()[1]
    sk.close()
    return p


def test_two_rank_merge_equals_whole_context():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res in out:
        for k, (topk_ok, pool_ok) in enumerate(res):
            assert topk_ok, f"rank {rank} case {k}: merged Top-K differs"
            assert pool_ok, f"rank {rank} case {k}: merged pool differs"


def test_planted_decomposition_fails_without_shard_offsets():
    """The check above is sensitive: dropping the shard offset of rank 1's ids breaks it."""
    s = _scores(5000, 5000)
    (lo0, hi0), (lo1, hi1) = cp.shards(5000, 2)
    a = _local(s, lo0, hi0, 64, 32)
    b = _local(s, lo1, hi1, 64, 32)
    bad_i = np.where(b[1] >= 0, b[1] - lo1, -1).astype(np.int32)
    good = _merge(np.concatenate([a[0], b[0]]), np.concatenate([a[1], b[1]]), 64)
    bad = _merge(np.concatenate([a[0], b[0]]), np.concatenate([a[1], bad_i]), 64)
    assert np.array_equal(good, O.topk(s, 64))
    assert not np.array_equal(bad, O.topk(s, 64))


def test_cp_calls_reject_bad_arguments():
    """Argument checks that run before any launch (no GPU needed)."""
    import ctypes as C
    from fp4_compressed_sparse_quantize_b200 import csa2
    L, f = csa2.lib(), C.c_void_p(256)
    assert L.csa2_cp_merge(1, 16385, f, f, 512, f, None) == csa2.ERR_UNSUPPORTED
    assert L.csa2_cp_merge(1, 100, f, f, 101, f, None) == csa2.ERR_ARG
    assert L.csa2_cp_merge(1, 100, None, f, 10, f, None) == csa2.ERR_ARG
    assert L.csa2_cp_pool_candidates(1, f, 64, f, 64, 8, 12, f, f, None) == csa2.ERR_ARG
    assert L.csa2_cp_topk_candidates(1, f, 64, f, 8, -1, f, f, None) == csa2.ERR_ARG
    assert L.csa2_cp_topk_candidates(1, f, 1 << 30, f, 8, 1 << 30, f, f, None) == csa2.ERR_UNSUPPORTED
    assert L.csa2_cp_local_idx(10, f, 5, 4, f, None) == csa2.ERR_ARG
    assert L.csa2_attn_merge_partials(1, 65, 2, f, f, f, None) == csa2.ERR_ARG
    with pytest.raises(csa2.Csa2Error):
        cp.select(torch.zeros((1, 2, 1, 128)), None, None, None, 0, 1, None)


# ---- GPU: the cp_* kernels ---------------------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("G,n_list,K,nblk", [(2, [32768, 20001, 9], 512, 2048),
                                              (3, [40000, 32773, 4000], 512, 2048),
                                              (4, [262144, 131075], 512, 2048),
                                              (8, [262144, 100003], 512, 2048)])
def test_gpu_sharded_selection_equals_single(G, n_list, K, nblk):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from fp4_compressed_sparse_quantize_b200 import csa2
    dev = "cuda"
    g = torch.Generator().manual_seed(G * 1000 + K)
    B, H_I, cap = len(n_list), 64, max(n_list)
    k_I = torch.randn((B, cap, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
    k_I[:, 200] = k_I[:, 100]            # exact score ties inside and across shards
    k_I[:, cap // 2 + 5] = k_I[:, 100]
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
    w = torch.rand((B, 1, H_I), generator=g).to(dev)
    n_vis = torch.tensor(n_list, dtype=torch.int32, device=dev)

    ref_idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    ref_pool = torch.empty((B, 1, nblk * 8), dtype=torch.int32, device=dev)
    ws = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, H_I, cap, K, nblk))
    csa2.index_score_topk("full", q_I, w, k_I, K, ref_idx, ws, n_vis0=n_vis, pool_out=ref_pool,
                          pool_blocks=nblk)

    cs, ci, cb, cblk = [], [], [], []
    for lo, hi in cp.shards(cap, G):
        shard = k_I[:, lo:hi].contiguous()
        idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
        pool = torch.empty((B, 1, nblk * 8), dtype=torch.int32, device=dev)
        scores = torch.zeros((B, 1, hi - lo), dtype=torch.float32, device=dev)
        wss = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, H_I, hi - lo, K, nblk))
        csa2.index_score_topk("full", q_I, w, shard, K, idx, wss,
                              n_vis0=cp.local_counts(n_vis, lo, hi), pool_out=pool,
                              pool_blocks=nblk, scores_out=scores)
        for lst, shape, dt in ((cs, K, torch.float32), (ci, K, torch.int32),
                               (cb, nblk, torch.float32), (cblk, nblk, torch.int32)):
            lst.append(torch.empty((B, 1, shape), dtype=dt, device=dev))
        csa2.cp_topk_candidates(scores, idx, lo, cs[-1], ci[-1])
        csa2.cp_pool_candidates(scores, pool, lo, cb[-1], cblk[-1])
        assert csa2.read_device_status(wss) == 0
    idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    csa2.cp_merge(torch.cat(cs, -1), torch.cat(ci, -1), idx)
    blocks = torch.empty((B, 1, nblk), dtype=torch.int32, device=dev)
    csa2.cp_merge(torch.cat(cb, -1), torch.cat(cblk, -1), blocks)
    pool = torch.empty((B, 1, nblk * 8), dtype=torch.int32, device=dev)
    csa2.cp_pool_expand(blocks, n_vis, pool)
    torch.cuda.synchronize()
    assert csa2.read_device_status(ws) == 0
    assert torch.equal(idx, ref_idx)
    assert torch.equal(pool, ref_pool)
    # and against the oracle's whole-context selection (scores over the same keys)
    from tests.helpers import bits8, check_topk
    idx_np, pool_np = idx.cpu().numpy(), pool.cpu().numpy()
    for b, n in enumerate(n_list):
        s = O.index_scores(bits8(q_I[b, 0]), w[b, 0].cpu().numpy(), bits8(k_I[b, :n]), O.E4M3)
        check_topk(idx_np[b, 0], s, np.arange(n), K, f"G={G} b={b}")
        nb = (n + 7) // 8
        bmax = np.array([s[8 * c:8 * c + 8].max() for c in range(nb)])
        got = np.unique(pool_np[b, 0][pool_np[b, 0] >= 0] // 8)
        gb = np.full(nblk, -1)
        gb[:len(got)] = got
        check_topk(gb, bmax, np.arange(nb), nblk, f"G={G} pool b={b}")


def _select_worker(port, q):
    """cp.select over a one-rank NCCL group equals the plain Full-layer call."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        from fp4_compressed_sparse_quantize_b200 import csa2
        dev = "cuda"
        g = torch.Generator().manual_seed(77)
        n_list, K, nblk, H_I = [32768, 5003], 512, 2048, 64
        B, cap = len(n_list), max(n_list)
        k_I = torch.randn((B, cap, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
        q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
        w = torch.rand((B, 1, H_I), generator=g).to(dev)
        n_vis = torch.tensor(n_list, dtype=torch.int32, device=dev)
        ws = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, H_I, cap, K, nblk))
        ref_idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
        ref_pool = torch.empty((B, 1, nblk * 8), dtype=torch.int32, device=dev)
        csa2.index_score_topk("full", q_I, w, k_I, K, ref_idx, ws, n_vis0=n_vis,
                              pool_out=ref_pool, pool_blocks=nblk)
        idx, pool = cp.select(q_I, w, k_I, n_vis, 0, K, ws, pool_blocks=nblk)
        torch.cuda.synchronize()
        q.put((bool(torch.equal(idx, ref_idx)), bool(torch.equal(pool, ref_pool)),
               csa2.read_device_status(ws)))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_gpu_select_one_rank_nccl():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_select_worker, args=(_free_port(), q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0
    assert res == (True, True, 0)


def _attend_nccl_worker(port, q):
    """cp.attend over a one-rank NCCL group: the partial path, the exchange and the merge
    kernel on a GPU, against the oracle."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        import math
        from fp4_compressed_sparse_quantize_b200 import csa2
        from tests.helpers import bits16, bits8, oracle_main_rows
        dev = "cuda"
        g = torch.Generator().manual_seed(91)
        B, H, n, K, W = 3, 64, 9000, 512, 128
        kv = (torch.randn((B, n, 512), generator=g) *
              torch.exp(torch.randn((B, 1, 512), generator=g))).to(torch.bfloat16)
        codes = torch.zeros((B, n, 256), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, n, 32), dtype=torch.uint8, device=dev)
        csa2.quantize_kv(kv.to(dev), torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
        rng = np.random.default_rng(9)
        idx = np.stack([np.sort(rng.choice(n, K, replace=False)) for _ in range(B)]).astype(np.int32)
        qh = torch.randn((B, H, 512), generator=g).to(torch.bfloat16)
        swa = torch.randn((B, W, 512), generator=g).to(torch.float8_e4m3fn)
        tau = 1 / math.sqrt(512)
        out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
        ws = csa2.new_workspace(csa2.workspace_bytes(1, B, 1, H, n, K))
        cp.attend("full", qh.to(dev), codes, scales, torch.from_numpy(idx).to(dev), 0,
                  swa.to(dev), out, ws, scale=tau)
        torch.cuda.synchronize()
        errs = []
        for b in range(B):
            rows = np.concatenate([oracle_main_rows(bits16(kv[b, idx[b]])),
                                   O.e4m3_array_to_f64(bits8(swa[b])).reshape(W, 512)])
            ref = O.attention(O.bf16_array_to_f64(bits16(qh[b])).reshape(H, 512), rows, tau)
            errs.append(float(np.max(np.abs(out[b].cpu().numpy() - ref)) /
                              math.sqrt(float(np.mean(ref * ref)))))
        q.put((errs, csa2.read_device_status(ws)))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_gpu_attend_one_rank_nccl():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_attend_nccl_worker, args=(_free_port(), q))
    p.start()
    errs, st = q.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0
    assert st == 0
    assert max(errs) <= 2e-3, errs


# ---- attention over shards: partial results merged by the log-sum-exp identity -------------

def _partial(q, rows, tau):
    """(m, l, o) of one rank's rows, natural-log units, fp64 (a plain restatement)."""
    H = q.shape[0]
    if rows.shape[0] == 0:
        return np.full(H, -np.inf), np.zeros(H), np.zeros((H, q.shape[1]))
    lg = tau * (q @ rows.T)
    m = lg.max(axis=1)
    p = np.exp(lg - m[:, None])
    return m, p.sum(axis=1), p @ rows


def _attn_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(11)
        n, K, W, H, tau = 3000, 512, 128, 8, 1 / np.sqrt(512)
        main = rng.standard_normal((n, 512)) * np.exp(rng.standard_normal(512))
        swa = rng.standard_normal((W, 512))
        qh = rng.standard_normal((H, 512))
        idx = np.sort(rng.choice(n, K, replace=False))
        lo, hi = cp.shards(n, world)[rank]
        mine = idx[(idx >= lo) & (idx < hi)]
        rows = main[mine]
        if rank == 0:
            rows = np.concatenate([rows, swa])
        m, l, o = _partial(qh, rows, tau)
        gm, gl, go = (cp.all_gather_stack(torch.from_numpy(x)).numpy() for x in (m, l, o))
        M = gm.max(axis=0)
        wgt = np.exp(gm - M)
        out = (wgt[:, :, None] * go).sum(axis=0) / (wgt * gl).sum(axis=0)[:, None]
        ref = O.attention(qh, np.concatenate([main[idx], swa]), tau)
        q.put((rank, float(np.max(np.abs(out - ref)) / np.sqrt(np.mean(ref * ref)))))
    finally:
        dist.destroy_process_group()


def test_two_rank_attention_partials_merge_to_whole():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_attn_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, rel in out:
        assert rel < 1e-12, f"rank {rank}: merged partials differ from the whole ({rel:.3g})"


@pytest.mark.gpu
@pytest.mark.parametrize("G,B,H,n,K,W", [(2, 3, 64, 20000, 512, 128), (3, 2, 40, 4001, 512, 37),
                                          (4, 32, 64, 32768, 512, 128)])
def test_gpu_sharded_attention_matches_oracle(G, B, H, n, K, W):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import math
    from fp4_compressed_sparse_quantize_b200 import csa2
    from tests.helpers import bits16, bits8, check_attention, oracle_main_rows
    dev = "cuda"
    g = torch.Generator().manual_seed(G * 7 + n)
    kv = (torch.randn((B, n, 512), generator=g) *
          torch.exp(torch.randn((B, 1, 512), generator=g))).to(torch.bfloat16)
    codes = torch.zeros((B, n, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, n, 32), dtype=torch.uint8, device=dev)
    csa2.quantize_kv(kv.to(dev), torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    rng = np.random.default_rng(n)
    idx = np.stack([np.sort(rng.choice(n, K, replace=False)) for _ in range(B)]).astype(np.int32)
    # query 0 selects only entries of the first shard: the other shards hold no row of it
    idx[0] = np.sort(rng.choice(n // G, K, replace=False))
    q = torch.randn((B, H, 512), generator=g).to(torch.bfloat16)
    swa = torch.randn((B, W, 512), generator=g).to(torch.float8_e4m3fn)
    tau = 1 / math.sqrt(512)
    tI = torch.from_numpy(idx).to(dev)
    o_parts, ml_parts = [], []
    for r, (lo, hi) in enumerate(cp.shards(n, G)):
        cs, ss = codes[:, lo:hi].contiguous(), scales[:, lo:hi].contiguous()
        local = torch.empty_like(tI)
        csa2.cp_local_idx(tI, lo, hi, local)
        o = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
        ml = torch.empty((B, 2, H), dtype=torch.float32, device=dev)
        ws = csa2.new_workspace(csa2.workspace_bytes(1, B, 1, H, hi - lo, K))
        csa2.sparse_attn_decode_partial("full", q.to(dev), cs, ss, local,
                                        swa.to(dev) if r == 0 else None, o, ml, ws, scale=tau)
        assert csa2.read_device_status(ws) == 0
        o_parts.append(o)
        ml_parts.append(ml)
    out = torch.empty((B, H, 512), dtype=torch.float32, device=dev)
    csa2.attn_merge_partials(torch.stack(o_parts), torch.stack(ml_parts), out)
    torch.cuda.synchronize()
    for b in range(min(B, 4)):
        sel = [i for i in idx[b] if i >= 0]
        rows = np.concatenate([oracle_main_rows(bits16(kv[b, sel])),
                               O.e4m3_array_to_f64(bits8(swa[b])).reshape(W, 512)])
        ref = O.attention(O.bf16_array_to_f64(bits16(q[b])).reshape(H, 512), rows, tau)
        check_attention(out[b].cpu().numpy(), ref, f"G={G} b={b}")


# ---- cp.attend on CPU ranks: the module's plumbing with the kernels stood in for --------------

class _FakeKernels:
    """CPU stand-ins (from the oracle) for the three library calls cp.attend makes, with the
    kernels' argument conventions: local indices (-1 off-shard), base-2 (maximum, sum)
    partials with the unnormalised output, and their log-sum-exp merge."""

    @staticmethod
    def cp_local_idx(idx, lo, hi, out, stream=None):
        i = idx.to(torch.int64)
        out.copy_(torch.where((i >= lo) & (i < hi), i - lo, torch.full_like(i, -1)).to(out.dtype))

    @staticmethod
    def sparse_attn_decode_partial(mode, q, codes, scales, idx, swa, o_part, ml_part, ws,
                                   scale=None, swa_valid=None, stream=None):
        B, H, D = q.shape
        for b in range(B):
            sel = [int(i) for i in idx[b] if i >= 0]
            rows = O.dequant_entries(codes[b, sel].numpy(), scales[b, sel].numpy()) if sel \
                else np.zeros((0, D))
            if swa is not None:
                rows = np.concatenate([rows, O.e4m3_array_to_f64(
                    swa[b].view(torch.uint8).numpy().ravel()).reshape(-1, D)])
            qb = O.bf16_array_to_f64(q[b].view(torch.int16).numpy().view(np.uint16)).reshape(H, D)
            if rows.shape[0] == 0:
                o_part[b] = 0
                ml_part[b, 0] = -float("inf")
                ml_part[b, 1] = 0
                continue
            lg2 = scale * (qb @ rows.T) / np.log(2.0)
            m = lg2.max(axis=1)
            p = np.exp2(lg2 - m[:, None])
            o_part[b] = torch.from_numpy(p @ rows)
            ml_part[b, 0] = torch.from_numpy(m)
            ml_part[b, 1] = torch.from_numpy(p.sum(axis=1))

    @staticmethod
    def attn_merge_partials(o_parts, ml_parts, out, stream=None):
        o = o_parts.double().numpy()
        m = ml_parts[:, :, 0].double().numpy()
        l = ml_parts[:, :, 1].double().numpy()
        M = m.max(axis=0)
        wgt = np.exp2(m - M)
        out.copy_(torch.from_numpy((wgt[..., None] * o).sum(axis=0) /
                                   (wgt * l).sum(axis=0)[..., None]))


def _attend_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for nm in ("cp_local_idx", "sparse_attn_decode_partial", "attn_merge_partials"):
            setattr(cp.csa2, nm, getattr(_FakeKernels, nm))
        g = torch.Generator().manual_seed(5)
        B, H, n, K, W, tau = 2, 8, 1000, 64, 16, 1 / np.sqrt(512)
        kv = (torch.randn((B, n, 512), generator=g) *
              torch.exp(torch.randn((B, 1, 512), generator=g))).to(torch.bfloat16)
        codes = np.zeros((B, n, 256), np.uint8)
        scales = np.zeros((B, n, 32), np.uint8)
        for b in range(B):
            codes[b], scales[b] = O.quantize_entries(
                kv[b].view(torch.int16).numpy().view(np.uint16))
        rng = np.random.default_rng(3)
        idx = np.stack([np.sort(rng.choice(n, K, replace=False)) for _ in range(B)]).astype(np.int32)
        idx[1, -5:] = -1                              # padded selection
        qh = torch.randn((B, H, 512), generator=g).to(torch.bfloat16)
        swa = torch.randn((B, W, 512), generator=g).to(torch.float8_e4m3fn)
        lo, hi = cp.shards(n, world)[rank]
        out = torch.empty((B, H, 512), dtype=torch.float32)
        cp.attend("full", qh, torch.from_numpy(codes[:, lo:hi].copy()),
                  torch.from_numpy(scales[:, lo:hi].copy()), torch.from_numpy(idx), lo,
                  swa if rank == 0 else None, out, None, scale=tau)
        errs = []
        for b in range(B):
            sel = [int(i) for i in idx[b] if i >= 0]
            rows = np.concatenate([O.dequant_entries(codes[b, sel], scales[b, sel]),
                                   O.e4m3_array_to_f64(swa[b].view(torch.uint8).numpy().ravel()
                                                       ).reshape(W, 512)])
            ref = O.attention(O.bf16_array_to_f64(qh[b].view(torch.int16).numpy()
                                                  .view(np.uint16)).reshape(H, 512), rows, tau)
            errs.append(float(np.max(np.abs(out[b].double().numpy() - ref)) /
                              np.sqrt(np.mean(ref * ref))))
        q.put((rank, errs))
    finally:
        dist.destroy_process_group()


def test_two_rank_attend_plumbing_equals_whole_context():
    """cp.attend over two gloo ranks (window rows on rank 0 only): local indices, the
    partials' exchange through all_gather_stack and the merge reproduce the oracle's
    attention over the whole selection. The three kernels are replaced by CPU stand-ins
    with the same conventions, so this tests the module, not the kernels (those are the
    GPU tests above)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_attend_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, errs in out:
        for b, e in enumerate(errs):
            # fp32 storage of the partials and of the output; a plumbing mistake (a window
            # counted twice, a lost shard, unshifted indices) is an O(1) error
            assert e < 1e-5, f"rank {rank} b={b}: {e:.3g}"
