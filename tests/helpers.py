"""Shared test helpers: byte views of torch tensors, the Top-K comparison rule, and
oracle-side reconstructions of the GPU inputs (the oracle only ever sees inputs)."""
import math

import numpy as np
import torch

from oracle import oracle as O

TOPK_REL = 1e-5        # near-tie exemption of the Top-K comparison
ATTN_REL_RMS = 2e-3    # attention: max |err| <= 2e-3 * RMS(reference output)


def bits16(t):
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits8(t):
    """float8_e4m3fn / uint8 tensor -> numpy uint8."""
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def raw_qk(t):
    return bits16(t) if t.dtype == torch.bfloat16 else bits8(t)


def odt(t):
    return O.BF16 if t.dtype == torch.bfloat16 else O.E4M3


def check_topk(gpu_idx, scores, ids, K, what=""):
    """gpu_idx: int array [K] (ascending, -1 padded). scores: oracle fp64 scores of the
    valid candidates; ids: their ids. Exact set equality unless the oracle's K-th and
    (K+1)-th scores are within TOPK_REL, in which case the clear winners must be present
    and every other pick must be within TOPK_REL of the K-th score."""
    g = np.asarray(gpu_idx)
    got = g[g >= 0]
    assert np.all(np.diff(got) > 0), f"{what}: output not strictly ascending"
    assert np.all(g[len(got):] == -1), f"{what}: -1 padding not at the end"
    n = len(scores)
    if n <= K:
        assert sorted(got.tolist()) == sorted(int(i) for i in ids), f"{what}: n <= K"
        return "all"
    order = sorted(range(n), key=lambda i: (-scores[i], ids[i]))
    sK, sK1 = scores[order[K - 1]], scores[order[K]]
    expect = set(int(ids[i]) for i in order[:K])
    gs = set(got.tolist())
    assert len(got) == K, f"{what}: {len(got)} picks"
    tol = TOPK_REL * max(abs(sK), 1e-30)
    if sK - sK1 > tol:
        missing = expect - gs
        assert not missing, f"{what}: {len(missing)} picks differ (gap {sK - sK1:.3g})"
        return "exact"
    by_id = {int(ids[i]): scores[i] for i in range(n)}
    for i in range(n):
        if scores[i] > sK + tol:
            assert int(ids[i]) in gs, f"{what}: clear winner {ids[i]} missing"
    for j in gs:
        assert by_id[j] >= sK - tol, f"{what}: pick {j} below the K-th score"
    return "exempt"


def check_attention(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = math.sqrt(float(np.mean(ref * ref)))
    err = float(np.max(np.abs(gpu - ref))) if ref.size else 0.0
    assert err <= ATTN_REL_RMS * rms + 1e-30, f"{what}: max err {err:.3g} vs rms {rms:.3g}"
    return err / rms if rms > 0 else 0.0


def oracle_main_rows(kv_bits_rows):
    """Dequantised rows the oracle itself quantises from the bf16 source rows."""
    codes, scales = O.quantize_entries(kv_bits_rows)
    return O.dequant_entries(codes, scales)
