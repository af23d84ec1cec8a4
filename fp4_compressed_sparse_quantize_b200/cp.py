"""Context parallelism of a Full layer (selection and attention) over G GPUs.

Each GPU (rank) holds one contiguous shard of every sequence's compressed entries (its own
indexer-K and main-KV cache for those positions), scans it with the ordinary Full-mode
indexer and keeps its own Top-K and candidate pool. The ranks exchange the selections as
(score, global index) and (block maximum, global block) lists with an all-gather, and every
rank merges them into the exact global selection, identical to one GPU scanning the whole
context ("DeepSeek-V4.1-Flash: A New Era in Efficient Large-Scale LLM Serving", Compressed
Sparse Attention 2 (CSA2): the Full layer keeps the 512 best entries and a candidate pool of
the 2,048 best blocks of 8 positions).

The attention follows the same split: each rank attends over the selected entries it holds
(and one rank over the window rows), leaves a partial result (maximum, sum, unnormalised
output), the ranks all-gather the partials and every rank merges them by the exact
log-sum-exp identity.

All selection and attention work runs in libcsa2's kernels (csa2.cp_*, csa2.*_partial*); this
module plans the shards and moves the lists with torch.distributed (NCCL between GPUs, gloo
on the host).
"""
import torch
import torch.distributed as dist

from . import csa2


def shards(n, g, align=csa2.POOL_BLOCK):
    """[lo, hi) of each of g shards of n entries: every lo a multiple of `align` (so pool
    blocks never straddle two shards), sizes as even as that allows."""
    if g < 1 or n < 0:
        raise ValueError("need g >= 1 and n >= 0")
    blocks = (n + align - 1) // align
    return [(min(n, blocks * r // g * align), min(n, blocks * (r + 1) // g * align))
            for r in range(g)]


def local_counts(n_vis, lo, hi):
    """Visible entries of each row that fall inside the shard [lo, hi)."""
    return (n_vis.to(torch.int64) - lo).clamp(0, hi - lo).to(torch.int32)


def all_gather_last(t, group=None):
    """Every rank's t concatenated along the last dimension, in rank order."""
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.cat(parts, dim=-1).contiguous()


def select(q_I, w, k_I_shard, n_vis, lo, K, ws, pool_blocks=0, group=None):
    """Decode Full-layer selection of every sequence, sharded over the ranks of `group`.

    q_I [B, 1, H_I, 128], w [B, 1, H_I] and n_vis int32 [B] (visible entries of the whole
    context) are the same on every rank; k_I_shard [B, cap_shard, 128] holds global entries
    [lo, lo + cap_shard) and lo is a multiple of 8. ws is a workspace for the shard's
    index_score_topk. Returns (idx [B, 1, K], pool [B, 1, pool_blocks * 8] or None) with
    global indices, the same on every rank. The shard's scores are materialised (4 bytes per
    entry) so that the selected entries can carry their scores into the exchange."""
    B, T = q_I.shape[:2]
    if T != 1:
        raise csa2.Csa2Error(csa2.ERR_UNSUPPORTED, "context-parallel selection is decode-only")
    if lo % csa2.POOL_BLOCK:
        raise csa2.Csa2Error(csa2.ERR_ARG, "a shard must start at a multiple of 8")
    cap = k_I_shard.shape[1]
    dev = q_I.device
    i32, f32 = torch.int32, torch.float32
    idx = torch.empty((B, T, K), dtype=i32, device=dev)
    scores = torch.zeros((B, T, cap), dtype=f32, device=dev)
    pool = torch.empty((B, T, pool_blocks * csa2.POOL_BLOCK), dtype=i32, device=dev) \
        if pool_blocks else None
    csa2.index_score_topk("full", q_I, w, k_I_shard, K, idx, ws,
                          n_vis0=local_counts(n_vis, lo, lo + cap), pool_out=pool,
                          pool_blocks=pool_blocks, scores_out=scores)
    cs = torch.empty((B, T, K), dtype=f32, device=dev)
    ci = torch.empty((B, T, K), dtype=i32, device=dev)
    csa2.cp_topk_candidates(scores, idx, lo, cs, ci)
    out = torch.empty((B, T, K), dtype=i32, device=dev)
    csa2.cp_merge(all_gather_last(cs, group), all_gather_last(ci, group), out)
    if not pool_blocks:
        return out, None
    cb = torch.empty((B, T, pool_blocks), dtype=f32, device=dev)
    cblk = torch.empty((B, T, pool_blocks), dtype=i32, device=dev)
    csa2.cp_pool_candidates(scores, pool, lo, cb, cblk)
    blocks = torch.empty((B, T, pool_blocks), dtype=i32, device=dev)
    csa2.cp_merge(all_gather_last(cb, group), all_gather_last(cblk, group), blocks)
    pool_out = torch.empty_like(pool)
    csa2.cp_pool_expand(blocks, n_vis.to(i32).contiguous(), pool_out)
    return out, pool_out


def all_gather_stack(t, group=None):
    """Every rank's t stacked along a new leading dimension, in rank order."""
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts).contiguous()


def attend(mode, q, codes_shard, scales_shard, idx, lo, swa, out, ws, swa_valid=None,
           scale=None, group=None):
    """Decode attention over the merged selection `idx` int32 [B, K] (global indices), with
    this rank holding main-KV entries [lo, lo + cap_shard) in codes_shard / scales_shard.
    Pass swa (and swa_valid) on exactly one rank, None elsewhere. Writes out fp32
    [B, H, 512] on every rank."""
    B, H, _ = q.shape
    cap = codes_shard.shape[1]
    dev = q.device
    local = torch.empty_like(idx)
    csa2.cp_local_idx(idx, lo, lo + cap, local)
    o = torch.empty((B, H, csa2.D_MAIN), dtype=torch.float32, device=dev)
    ml = torch.empty((B, 2, H), dtype=torch.float32, device=dev)
    csa2.sparse_attn_decode_partial(mode, q, codes_shard, scales_shard, local, swa, o, ml, ws,
                                    scale=scale, swa_valid=swa_valid)
    csa2.attn_merge_partials(all_gather_stack(o, group), all_gather_stack(ml, group), out)
