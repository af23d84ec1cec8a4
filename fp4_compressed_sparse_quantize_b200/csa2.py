"""Thin Python binding of libcsa2 (ctypes). Argument marshalling only: every step of the
CSA2 path runs in the library's CUDA kernels. torch supplies device memory and streams.

The names mirror the C ABI in include/csa2.h (csa2_quantize_kv -> quantize_kv, ...).
Importing this module does not need a GPU; calling an operation does, and raises
Csa2Error when the library is missing or reports an error. There is no fallback.
"""
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

OK, ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_DEVICE = range(6)
MODE = {"full": 0, "reindex": 1, "reuse": 2}
DTYPE = {torch.bfloat16: 0, torch.float8_e4m3fn: 1}
OP_INDEX_SCORE_TOPK, OP_SPARSE_ATTN_DECODE, OP_SPARSE_ATTN_PREFILL = 0, 1, 2
DEV_BAD_INDEX, DEV_BAD_COUNT, DEV_TIMEOUT = 1, 2, 4
D_MAIN, D_INDEX, POOL_BLOCK = 512, 128, 8
EXPORTS = ("csa2_quantize_kv", "csa2_index_score_topk", "csa2_sparse_attn_decode",
           "csa2_sparse_attn_prefill", "csa2_workspace_bytes", "csa2_status_string",
           "csa2_read_device_status", "csa2_reset_device_status", "csa2_version",
           "csa2_debug_bounded_wait", "csa2_set_stage_events",
           "csa2_index_score_topk_noalloc", "csa2_sparse_attn_decode_launches",
           "csa2_cp_topk_candidates", "csa2_cp_pool_candidates", "csa2_cp_merge",
           "csa2_cp_pool_expand", "csa2_cache_record_bytes", "csa2_cache_export",
           "csa2_cache_import", "csa2_cp_local_idx", "csa2_sparse_attn_decode_partial",
           "csa2_attn_merge_partials", "csa2_record_event", "csa2_compress_kv",
           "csa2_quantize_keys_fp4")


class Csa2Error(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib():
    """Load libcsa2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise Csa2Error(ERR_CUDA, f"{LIB_PATH} is missing; build it with "
                                      "python fp4_compressed_sparse_quantize_b200/build.py")
        L = C.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
        L.csa2_quantize_kv.argtypes = [P, i32, i32, i64, i64, P, P, P, i64, P, P]
        L.csa2_quantize_keys_fp4.argtypes = [P, i32, i32, i64, i64, P, P, i64, P, P]
        L.csa2_compress_kv.argtypes = [i32, i32, i32, P, P, i64, i64, P, i32, P, P, P, P, i64,
                                       P, P, P]
        L.csa2_index_score_topk.argtypes = [i32, i32, i32, i32, i32, P, P, P, i64, P, i32, P,
                                            i32, P, i32, P, i32, P, P, P, sz, P]
        L.csa2_sparse_attn_decode.argtypes = [i32, i32, i32, P, P, P, i64, P, i32, P, i32, P,
                                              f32, P, P, sz, P]
        L.csa2_sparse_attn_prefill.argtypes = [i32, i32, i32, P, P, P, i64, P, i32, P, i32, P,
                                               f32, P, P, sz, P]
        L.csa2_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i32, i32]
        L.csa2_workspace_bytes.restype = sz
        L.csa2_status_string.argtypes = [i32]
        L.csa2_status_string.restype = C.c_char_p
        L.csa2_read_device_status.argtypes = [P, P, P]
        L.csa2_reset_device_status.argtypes = [P, P]
        L.csa2_debug_bounded_wait.argtypes = [P, C.c_uint64, P]
        L.csa2_set_stage_events.argtypes = [P, P]
        L.csa2_record_event.argtypes = [P, P]
        L.csa2_index_score_topk_noalloc.argtypes = [i32, i32, i32, i32, i32, P, P, P, i64, P,
                                                    i32, P, i32, P, i32, P, i32, P, P, P, P]
        L.csa2_sparse_attn_decode_launches.argtypes = [i32, i32, i32]
        L.csa2_cp_topk_candidates.argtypes = [i32, P, i64, P, i32, i64, P, P, P]
        L.csa2_cp_pool_candidates.argtypes = [i32, P, i64, P, i32, i32, i64, P, P, P]
        L.csa2_cp_merge.argtypes = [i32, i32, P, P, i32, P, P]
        L.csa2_cp_pool_expand.argtypes = [i32, P, i32, P, i32, P, P]
        L.csa2_cp_local_idx.argtypes = [i64, P, i64, i64, P, P]
        L.csa2_sparse_attn_decode_partial.argtypes = [i32, i32, i32, P, P, P, i64, P, i32, P,
                                                      i32, P, f32, P, P, P, sz, P]
        L.csa2_attn_merge_partials.argtypes = [i32, i32, i32, P, P, P, P]
        L.csa2_cache_record_bytes.argtypes = [i64, i32]
        L.csa2_cache_record_bytes.restype = sz
        L.csa2_cache_export.argtypes = [P, P, P, i32, i64, i32, i64, i64, P, sz, P]
        L.csa2_cache_import.argtypes = [P, sz, P, P, P, i64, i32, P]
        for name in EXPORTS:
            if name not in ("csa2_workspace_bytes", "csa2_status_string",
                            "csa2_cache_record_bytes"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_string(status):
    return lib().csa2_status_string(int(status)).decode()


def _p(t):
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _check(status, what):
    if status != OK:
        raise Csa2Error(status, what)


def _need(t, dtype, name, dev=True):
    if t is None:
        return
    if t.dtype != dtype:
        raise Csa2Error(ERR_ARG, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise Csa2Error(ERR_ARG, f"{name} must be contiguous")
    if dev and not t.is_cuda:
        raise Csa2Error(ERR_ARG, f"{name} must be a CUDA tensor")


# ---- workspace ---------------------------------------------------------------------------

def workspace_bytes(op, B, T, H, cap, K, pool_blocks=0):
    return int(lib().csa2_workspace_bytes(int(op), int(B), int(T), int(H), int(cap), int(K),
                                          int(pool_blocks)))


def sparse_attn_decode_launches(B, K, W):
    """Kernels one sparse_attn_decode call launches on the current device (see csa2.h)."""
    return int(lib().csa2_sparse_attn_decode_launches(int(B), int(K), int(W)))


def new_workspace(nbytes, device="cuda"):
    """Zero-filled workspace (the device status word starts cleared)."""
    n = max(int(nbytes), 256)
    return torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=device)


def read_device_status(ws, stream=None):
    out = C.c_int32(0)
    st = lib().csa2_read_device_status(_p(ws), C.byref(out), _stream(stream))
    if st not in (OK, ERR_DEVICE):
        _check(st, "csa2_read_device_status")
    return out.value


def reset_device_status(ws, stream=None):
    _check(lib().csa2_reset_device_status(_p(ws), _stream(stream)), "csa2_reset_device_status")


def set_stage_events(ev_start, ev_stop):
    """Record torch.cuda.Event pair around the next indexer-scan launch of this thread."""
    a = C.c_void_p(ev_start.cuda_event) if ev_start is not None else None
    b = C.c_void_p(ev_stop.cuda_event) if ev_stop is not None else None
    _check(lib().csa2_set_stage_events(a, b), "csa2_set_stage_events")


def record_event(ev, stream=None):
    """Record torch.cuda.Event `ev` (created already: record it once beforehand) on the stream;
    inside a stream capture the record becomes an external node of the graph, so replays can
    be timed between two such events."""
    _check(lib().csa2_record_event(C.c_void_p(ev.cuda_event), _stream(stream)),
           "csa2_record_event")


def debug_bounded_wait(status_word, timeout_ns, stream=None):
    _need(status_word, torch.int32, "status_word")
    _check(lib().csa2_debug_bounded_wait(_p(status_word), int(timeout_ns), _stream(stream)),
           "csa2_debug_bounded_wait")


# ---- operations ---------------------------------------------------------------------------

def quantize_kv(kv, dst_off, codes, scales, status=None, stream=None):
    """kv bf16 [B, n_new, 512] (row stride may exceed 512); dst_off int32 [B];
    codes uint8 [B, cap, 256]; scales uint8 [B, cap, 32]."""
    _need(dst_off, torch.int32, "dst_off")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    if kv.dtype != torch.bfloat16 or kv.stride(-1) != 1 or not kv.is_cuda:
        raise Csa2Error(ERR_ARG, "kv must be a CUDA bf16 tensor with unit channel stride")
    B, n_new, D = kv.shape
    cap = codes.shape[1]
    st = lib().csa2_quantize_kv(_p(kv), B, n_new, kv.stride(1), kv.stride(0), _p(dst_off),
                                _p(codes), _p(scales), cap, _p(status), _stream(stream))
    _check(st, "csa2_quantize_kv")


def compress_kv(C, Z, ratio, w_proj, dst_off, codes, scales, k_I, latent_out=None, status=None,
                stream=None):
    """C, Z bf16 [B, ratio * n_new, 512] (unit channel stride; token and batch strides may
    be larger): source-token latents and compression logits. w_proj bf16 [128, 512];
    dst_off int32 [B]; codes uint8 [B, cap, 256]; scales uint8 [B, cap, 32]; k_I
    [B, cap, 128] E4M3 or bf16; latent_out nullable bf16 [B, n_new, 512]."""
    for t, nm in ((C, "C"), (Z, "Z")):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1 or not t.is_cuda:
            raise Csa2Error(ERR_ARG, f"{nm} must be a CUDA bf16 tensor with unit channel stride")
    if C.shape != Z.shape or C.stride() != Z.stride():
        raise Csa2Error(ERR_ARG, "C and Z must have the same shape and strides")
    _need(w_proj, torch.bfloat16, "w_proj")
    _need(dst_off, torch.int32, "dst_off")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    _need(latent_out, torch.bfloat16, "latent_out")
    if isinstance(k_I, Fp4Keys):
        kdt, kp = DTYPE_E4M3_FP4KEY, _p(k_I.buf)
    else:
        if k_I.dtype not in DTYPE:
            raise Csa2Error(ERR_ARG, "k_I must be bf16, float8_e4m3fn or Fp4Keys")
        _need(k_I, k_I.dtype, "k_I")
        kdt, kp = DTYPE[k_I.dtype], _p(k_I)
    B, n_tok, D = C.shape
    if n_tok % ratio:
        raise Csa2Error(ERR_ARG, "the token count must be a multiple of the ratio")
    st = lib().csa2_compress_kv(B, n_tok // ratio, int(ratio), _p(C), _p(Z), C.stride(1),
                                C.stride(0), _p(w_proj), kdt, _p(dst_off),
                                _p(codes), _p(scales), kp, codes.shape[1], _p(latent_out),
                                _p(status), _stream(stream))
    _check(st, "csa2_compress_kv")


DTYPE_E4M3_FP4KEY = 2
FP4KEY_CODE_BYTES = 64


class Fp4Keys:
    """Compact 68-byte indexer keys of B sequences x cap entries: one device buffer holding
    the E2M1 code plane [B, cap, 64] and then the fp32 scale plane [B, cap] (the layout of
    CSA2_DTYPE_E4M3_FP4KEY)."""

    def __init__(self, B, cap, device="cuda"):
        self.B, self.cap = int(B), int(cap)
        n = self.B * self.cap
        self.buf = torch.zeros(n * (FP4KEY_CODE_BYTES + 4), dtype=torch.uint8, device=device)
        self.codes = self.buf[:n * FP4KEY_CODE_BYTES].view(self.B, self.cap, FP4KEY_CODE_BYTES)
        self.scales = self.buf[n * FP4KEY_CODE_BYTES:].view(torch.float32).view(self.B, self.cap)


def quantize_keys_fp4(k, dst_off, keys, status=None, stream=None):
    """k bf16 [B, n_new, 128] (unit channel stride); dst_off int32 [B]; keys: Fp4Keys."""
    _need(dst_off, torch.int32, "dst_off")
    if k.dtype != torch.bfloat16 or k.stride(-1) != 1 or not k.is_cuda:
        raise Csa2Error(ERR_ARG, "k must be a CUDA bf16 tensor with unit channel stride")
    B, n_new, Di = k.shape
    st = lib().csa2_quantize_keys_fp4(_p(k), B, n_new, k.stride(1), k.stride(0), _p(dst_off),
                                      _p(keys.buf), keys.cap, _p(status), _stream(stream))
    _check(st, "csa2_quantize_keys_fp4")


def _key_args(q_I, k_I):
    """(dtype code, key pointer, cap) of index_score_topk's key argument."""
    if isinstance(k_I, Fp4Keys):
        if q_I.dtype != torch.float8_e4m3fn:
            raise Csa2Error(ERR_ARG, "compact keys take an E4M3 query")
        _need(q_I, q_I.dtype, "q_I")
        return DTYPE_E4M3_FP4KEY, _p(k_I.buf), k_I.cap
    if q_I.dtype not in DTYPE or k_I.dtype != q_I.dtype:
        raise Csa2Error(ERR_ARG, "q_I and k_I must share a dtype (bf16 or float8_e4m3fn)")
    for t, nm in ((q_I, "q_I"), (k_I, "k_I")):
        _need(t, q_I.dtype, nm)
    return DTYPE[q_I.dtype], _p(k_I), k_I.shape[1]


def index_score_topk(mode, q_I, w, k_I, K, idx_out, ws, n_vis0=None, q_pos0=None, ratio=1,
                     pool_in=None, pool_out=None, pool_blocks=0, scores_out=None, stream=None):
    """q_I [B, T, H_I, 128] (bf16 or E4M3), w fp32 [B, T, H_I], k_I [B, cap, 128] of the same
    dtype (or Fp4Keys with an E4M3 query), idx_out int32 [B, T, K]. Decode: n_vis0 int32 [B].
    Prefill: q_pos0 int32 [B] and ratio. Reindex: pool_in int32 [B, T, P]. Full with a pool:
    pool_out int32 [B, T, pool_blocks * 8]."""
    m = MODE[mode] if isinstance(mode, str) else int(mode)
    B, T, H_I, Di = q_I.shape
    dt, kp, cap = _key_args(q_I, k_I)
    _need(w, torch.float32, "w")
    _need(idx_out, torch.int32, "idx_out")
    _need(n_vis0, torch.int32, "n_vis0")
    _need(q_pos0, torch.int32, "q_pos0")
    _need(pool_in, torch.int32, "pool_in")
    _need(pool_out, torch.int32, "pool_out")
    _need(scores_out, torch.float32, "scores_out")
    P_in = pool_in.shape[-1] if pool_in is not None else 0
    st = lib().csa2_index_score_topk(
        m, B, T, H_I, dt, _p(q_I), _p(w), kp, cap, _p(n_vis0), int(ratio),
        _p(q_pos0), int(K), _p(pool_in), P_in, _p(pool_out), int(pool_blocks), _p(idx_out),
        _p(scores_out), _p(ws), ws.numel() if ws is not None else 0, _stream(stream))
    _check(st, "csa2_index_score_topk")


def index_score_topk_noalloc(mode, q_I, w, k_I, K, idx_out, n_vis0=None, q_pos0=None, ratio=1,
                             pool_in=None, pool_out=None, pool_blocks=0, scores_out=None,
                             status=None, stream=None):
    """index_score_topk without a workspace argument, for callers that cannot allocate: the
    library's fixed 16 MiB device scratch array is used instead (see include/csa2.h).
    `status` is an optional int32 CUDA tensor that receives the device status bits."""
    m = MODE[mode] if isinstance(mode, str) else int(mode)
    B, T, H_I, Di = q_I.shape
    if q_I.dtype not in DTYPE or k_I.dtype != q_I.dtype:
        raise Csa2Error(ERR_ARG, "q_I and k_I must share a dtype (bf16 or float8_e4m3fn)")
    for t, nm in ((q_I, "q_I"), (k_I, "k_I")):
        _need(t, q_I.dtype, nm)
    _need(w, torch.float32, "w")
    _need(idx_out, torch.int32, "idx_out")
    _need(n_vis0, torch.int32, "n_vis0")
    _need(q_pos0, torch.int32, "q_pos0")
    _need(pool_in, torch.int32, "pool_in")
    _need(pool_out, torch.int32, "pool_out")
    _need(scores_out, torch.float32, "scores_out")
    _need(status, torch.int32, "status")
    P_in = pool_in.shape[-1] if pool_in is not None else 0
    st = lib().csa2_index_score_topk_noalloc(
        m, B, T, H_I, DTYPE[q_I.dtype], _p(q_I), _p(w), _p(k_I), k_I.shape[1], _p(n_vis0),
        int(ratio), _p(q_pos0), int(K), _p(pool_in), P_in, _p(pool_out), int(pool_blocks),
        _p(idx_out), _p(scores_out), _p(status), _stream(stream))
    _check(st, "csa2_index_score_topk_noalloc")


def sparse_attn_decode(mode, q, codes, scales, idx, swa, out, ws, scale=None, swa_valid=None,
                       stream=None):
    """q bf16 [B, H, 512]; idx int32 [B, K]; swa E4M3 [B, W, 512]; out fp32 [B, H, 512]."""
    m = MODE[mode] if isinstance(mode, str) else int(mode)
    _need(q, torch.bfloat16, "q")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    _need(idx, torch.int32, "idx")
    _need(swa, torch.float8_e4m3fn, "swa")
    _need(out, torch.float32, "out")
    _need(swa_valid, torch.int32, "swa_valid")
    B, H, D = q.shape
    K = idx.shape[-1] if idx is not None else 0
    W = swa.shape[1] if swa is not None else 0
    sc = float(scale) if scale is not None else D_MAIN ** -0.5
    st = lib().csa2_sparse_attn_decode(m, B, H, _p(q), _p(codes), _p(scales), codes.shape[1],
                                       _p(idx), K, _p(swa), W, _p(swa_valid), sc, _p(out),
                                       _p(ws), ws.numel(), _stream(stream))
    _check(st, "csa2_sparse_attn_decode")


def sparse_attn_decode_partial(mode, q, codes, scales, idx, swa, o_part, ml_part, ws, scale=None,
                               swa_valid=None, stream=None):
    """sparse_attn_decode over the caller's rows, left as a partial: o_part fp32 [B, H, 512],
    ml_part fp32 [B, 2, H] (base-2 maximum and sum). swa may be None (no window rows)."""
    m = MODE[mode] if isinstance(mode, str) else int(mode)
    _need(q, torch.bfloat16, "q")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    _need(idx, torch.int32, "idx")
    _need(swa, torch.float8_e4m3fn, "swa")
    _need(o_part, torch.float32, "o_part")
    _need(ml_part, torch.float32, "ml_part")
    _need(swa_valid, torch.int32, "swa_valid")
    B, H, D = q.shape
    K = idx.shape[-1] if idx is not None else 0
    W = swa.shape[1] if swa is not None else 0
    sc = float(scale) if scale is not None else D_MAIN ** -0.5
    st = lib().csa2_sparse_attn_decode_partial(m, B, H, _p(q), _p(codes), _p(scales),
                                               codes.shape[1], _p(idx), K, _p(swa), W,
                                               _p(swa_valid), sc, _p(o_part), _p(ml_part),
                                               _p(ws), ws.numel(), _stream(stream))
    _check(st, "csa2_sparse_attn_decode_partial")


def attn_merge_partials(o_parts, ml_parts, out, stream=None):
    """o_parts fp32 [G, B, H, 512], ml_parts fp32 [G, B, 2, H] -> out fp32 [B, H, 512]."""
    _need(o_parts, torch.float32, "o_parts")
    _need(ml_parts, torch.float32, "ml_parts")
    _need(out, torch.float32, "out")
    G, B, H, _ = o_parts.shape
    _check(lib().csa2_attn_merge_partials(B, H, G, _p(o_parts), _p(ml_parts), _p(out),
                                          _stream(stream)), "csa2_attn_merge_partials")


def sparse_attn_prefill(q, codes, scales, idx, swa, out, ws, W, q_pos0=None, scale=None,
                        stream=None):
    """q bf16 [B, T, H, 512]; idx int32 [B, T, K]; swa E4M3 [B, W-1+T, 512];
    out fp32 [B, T, H, 512]."""
    _need(q, torch.bfloat16, "q")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    _need(idx, torch.int32, "idx")
    _need(swa, torch.float8_e4m3fn, "swa")
    _need(out, torch.float32, "out")
    _need(q_pos0, torch.int32, "q_pos0")
    B, T, H, D = q.shape
    K = idx.shape[-1]
    sc = float(scale) if scale is not None else D_MAIN ** -0.5
    st = lib().csa2_sparse_attn_prefill(B, T, H, _p(q), _p(codes), _p(scales), codes.shape[1],
                                        _p(idx), K, _p(swa), int(W), _p(q_pos0), sc, _p(out),
                                        _p(ws), ws.numel(), _stream(stream))
    _check(st, "csa2_sparse_attn_prefill")


# ---- context parallelism (one shard of every sequence's entries per GPU) -----------------

def cp_topk_candidates(scores, idx, offset, cand_score, cand_idx, stream=None):
    """A shard's Top-K as candidates: scores fp32 [rows, ld] (the shard's scores_out),
    idx int32 [rows, K] (shard-local, -1 padded), offset = global index of the shard's first
    entry -> cand_score fp32 / cand_idx int32 [rows, K] (global indices, -1 padded)."""
    for t, dt, nm in ((scores, torch.float32, "scores"), (idx, torch.int32, "idx"),
                      (cand_score, torch.float32, "cand_score"), (cand_idx, torch.int32, "cand_idx")):
        _need(t, dt, nm)
    K = idx.shape[-1]
    rows = idx.numel() // K
    ld = scores.shape[-1]
    _check(lib().csa2_cp_topk_candidates(rows, _p(scores), ld, _p(idx), K, int(offset),
                                         _p(cand_score), _p(cand_idx), _stream(stream)),
           "csa2_cp_topk_candidates")


def cp_pool_candidates(scores, pool, offset, cand_bmax, cand_block, stream=None):
    """A shard's candidate pool as (block maximum, global block) pairs: pool int32 [rows, P]
    (shard-local positions), offset a multiple of 8 -> cand_bmax fp32 / cand_block int32
    [rows, nb] (nb = the pool's block count, -1 padded)."""
    for t, dt, nm in ((scores, torch.float32, "scores"), (pool, torch.int32, "pool"),
                      (cand_bmax, torch.float32, "cand_bmax"), (cand_block, torch.int32, "cand_block")):
        _need(t, dt, nm)
    P, nb = pool.shape[-1], cand_block.shape[-1]
    rows = pool.numel() // P
    _check(lib().csa2_cp_pool_candidates(rows, _p(scores), scores.shape[-1], _p(pool), P, nb,
                                         int(offset), _p(cand_bmax), _p(cand_block),
                                         _stream(stream)), "csa2_cp_pool_candidates")


def cp_merge(cand_score, cand_idx, idx_out, stream=None):
    """The exact Top-K of every row from gathered candidates [rows, n_cand] into idx_out
    int32 [rows, K]: (score desc, index asc), written in ascending index order."""
    for t, dt, nm in ((cand_score, torch.float32, "cand_score"), (cand_idx, torch.int32, "cand_idx"),
                      (idx_out, torch.int32, "idx_out")):
        _need(t, dt, nm)
    n, K = cand_idx.shape[-1], idx_out.shape[-1]
    rows = cand_idx.numel() // n
    _check(lib().csa2_cp_merge(rows, n, _p(cand_score), _p(cand_idx), K, _p(idx_out),
                               _stream(stream)), "csa2_cp_merge")


def cp_pool_expand(blocks, n_row, pool_out, stream=None):
    """Merged pool blocks int32 [rows, nb] (ascending, -1 padded) -> entry positions int32
    [rows, P]; n_row int32 [rows] visible entries per row (None: all)."""
    for t, dt, nm in ((blocks, torch.int32, "blocks"), (n_row, torch.int32, "n_row"),
                      (pool_out, torch.int32, "pool_out")):
        _need(t, dt, nm)
    nb, P = blocks.shape[-1], pool_out.shape[-1]
    rows = blocks.numel() // nb
    _check(lib().csa2_cp_pool_expand(rows, _p(blocks), nb, _p(n_row), P, _p(pool_out),
                                     _stream(stream)), "csa2_cp_pool_expand")


# ---- persistent-cache records --------------------------------------------------------------

def _key_bytes(k_I):
    return 0 if k_I is None else k_I.shape[-1] * k_I.element_size()


def cache_record_bytes(n, key_bytes=0):
    """Bytes of a record of n entries (key_bytes 0, 128 for E4M3 keys or 256 for bf16)."""
    return int(lib().csa2_cache_record_bytes(int(n), int(key_bytes)))


def cache_export(codes, scales, b, lo, n, host, k_I=None, stream=None):
    """Entries [lo, lo + n) of sequence b (codes [B, cap, 256], scales [B, cap, 32], optional
    k_I [B, cap, 128]) into `host`, a CPU uint8 tensor of at least cache_record_bytes bytes
    (pinned for an asynchronous copy)."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    if host.dtype != torch.uint8 or host.is_cuda or not host.is_contiguous():
        raise Csa2Error(ERR_ARG, "host must be a contiguous CPU uint8 tensor")
    if k_I is not None and (not k_I.is_cuda or not k_I.is_contiguous()):
        raise Csa2Error(ERR_ARG, "k_I must be a contiguous CUDA tensor")
    _check(lib().csa2_cache_export(_p(codes), _p(scales), _p(k_I), _key_bytes(k_I),
                                   codes.shape[1], int(b), int(lo), int(n), _p(host),
                                   host.numel(), _stream(stream)), "csa2_cache_export")


def cache_import(host, codes, scales, b, k_I=None, stream=None):
    """A complete record in `host` back into sequence b of the caches, at its own lo."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    if host.dtype != torch.uint8 or host.is_cuda or not host.is_contiguous():
        raise Csa2Error(ERR_ARG, "host must be a contiguous CPU uint8 tensor")
    if k_I is not None and (not k_I.is_cuda or not k_I.is_contiguous()):
        raise Csa2Error(ERR_ARG, "k_I must be a contiguous CUDA tensor")
    _check(lib().csa2_cache_import(_p(host), host.numel(), _p(codes), _p(scales), _p(k_I),
                                   codes.shape[1], int(b), _stream(stream)), "csa2_cache_import")


def cp_local_idx(idx, lo, hi, idx_local, stream=None):
    """Global selected indices -> indices local to the shard [lo, hi), -1 elsewhere."""
    _need(idx, torch.int32, "idx")
    _need(idx_local, torch.int32, "idx_local")
    _check(lib().csa2_cp_local_idx(idx.numel(), _p(idx), int(lo), int(hi), _p(idx_local),
                                   _stream(stream)), "csa2_cp_local_idx")
