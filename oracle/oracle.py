"""ctypes front end of the CSA2 CPU oracle (test infrastructure only).

Every array crosses as a numpy array; raw bit patterns travel as uint16 (bf16) or
uint8 (E4M3, packed E2M1). The arithmetic lives in csa2_oracle.c; this file only
marshals arguments and composes the per-query steps in the order the pages describe
them (score -> Top-K / pool -> gather -> attention).
"""
import ctypes as C

import numpy as np

from . import build as _build

_lib = None

BF16, E4M3 = 0, 1
POOL_BLOCK = 8


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        d, u8, u16, i32, i64, f32 = (C.c_double, C.c_uint8, C.c_uint16, C.c_int32,
                                     C.c_int64, C.c_float)
        P = C.c_void_p
        L.orc_bf16_value.restype = d
        L.orc_bf16_value.argtypes = [u16]
        L.orc_e2m1_value.restype = d
        L.orc_e2m1_value.argtypes = [C.c_uint]
        L.orc_e4m3_value.restype = d
        L.orc_e4m3_value.argtypes = [u8]
        L.orc_e4m3_encode.restype = u8
        L.orc_e4m3_encode.argtypes = [d]
        L.orc_e2m1_encode.restype = C.c_uint
        L.orc_e2m1_encode.argtypes = [d]
        L.orc_fp4_scale_code.restype = u8
        L.orc_fp4_scale_code.argtypes = [d]
        L.orc_fp4_code.restype = C.c_uint
        L.orc_fp4_code.argtypes = [d, d]
        for nm in ("orc_fp4_scale_codes_many", "orc_e4m3_encode_many"):
            getattr(L, nm).restype = None
            getattr(L, nm).argtypes = [P, i64, P]
        L.orc_fp4_codes_many.restype = None
        L.orc_fp4_codes_many.argtypes = [P, P, i64, P]
        L.orc_quantize_block16.restype = None
        L.orc_quantize_block16.argtypes = [P, P, P]
        L.orc_quantize_entries.restype = None
        L.orc_quantize_entries.argtypes = [P, i64, i64, C.c_int, P, P]
        L.orc_dequant_entry.restype = None
        L.orc_dequant_entry.argtypes = [P, P, C.c_int, P]
        L.orc_index_scores.restype = None
        L.orc_index_scores.argtypes = [C.c_int, C.c_int, C.c_int, P, P, P, P, i64, P]
        L.orc_topk.restype = i64
        L.orc_topk.argtypes = [P, P, i64, i64, P]
        L.orc_pool.restype = i64
        L.orc_pool.argtypes = [P, i64, i64, C.c_int, P]
        L.orc_attention.restype = None
        L.orc_attention.argtypes = [C.c_int, C.c_int, P, P, i64, d, P]
        L.orc_main_entry_bytes.restype = C.c_int
        L.orc_main_entry_bytes.argtypes = [C.c_int]
        L.orc_kv_bytes_per_token.restype = d
        L.orc_kv_bytes_per_token.argtypes = [C.c_int, d, C.c_int, C.c_int, C.c_int, C.c_int]
        L.orc_num_threads.restype = C.c_int
        L.orc_num_threads.argtypes = []
        L.orc_set_num_threads.restype = None
        L.orc_set_num_threads.argtypes = [C.c_int]
        L.orc_prefill_visible.restype = i64
        L.orc_prefill_visible.argtypes = [i64, C.c_int]
        L.orc_prefill_window_rows.restype = C.c_int
        L.orc_prefill_window_rows.argtypes = [i64, C.c_int, i64, P]
        L.orc_bf16_encode.restype = u16
        L.orc_bf16_encode.argtypes = [d]
        L.orc_bf16_encode_many.restype = None
        L.orc_bf16_encode_many.argtypes = [P, i64, P]
        L.orc_compress_entries.restype = None
        L.orc_compress_entries.argtypes = [P, P, i64, C.c_int, C.c_int, i64, P]
        L.orc_project_keys.restype = None
        L.orc_project_keys.argtypes = [P, i64, C.c_int, P, C.c_int, P]
        L.orc_quantize_keys_fp4.restype = None
        L.orc_quantize_keys_fp4.argtypes = [P, i64, C.c_int, P, P]
        L.orc_dequant_key_fp4.restype = None
        L.orc_dequant_key_fp4.argtypes = [P, C.c_float, C.c_int, P]
        L.orc_index_scores_fp4key.restype = None
        L.orc_index_scores_fp4key.argtypes = [C.c_int, C.c_int, P, P, P, P, P, i64, P]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_num_threads(n):
    """Threads for the oracle's parallel loops from now on."""
    lib().orc_set_num_threads(int(n))


def num_threads():
    """Threads the oracle's parallel loops use."""
    return int(lib().orc_num_threads())


# ---- formats -------------------------------------------------------------------------

def bf16_value(bits):
    return lib().orc_bf16_value(int(bits))


def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e4m3_value(code):
    return lib().orc_e4m3_value(int(code))


def e4m3_encode(v):
    return int(lib().orc_e4m3_encode(float(v)))


def e2m1_encode(v):
    return int(lib().orc_e2m1_encode(float(v)))


def bf16_array_to_f64(bits):
    bits = _c(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_array_to_f64(codes):
    table = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return table[_c(codes, np.uint8)]


def e4m3_encode_many(v):
    v = _c(v, np.float64)
    out = np.zeros(v.shape[0], np.uint8)
    lib().orc_e4m3_encode_many(_p(v), v.shape[0], _p(out))
    return out


def fp4_scale_codes(amax):
    """Scale code step of the block quantiser for many block maxima."""
    a = _c(amax, np.float64)
    out = np.zeros(a.shape[0], np.uint8)
    lib().orc_fp4_scale_codes_many(_p(a), a.shape[0], _p(out))
    return out


def fp4_codes(x, s):
    """Element code step of the block quantiser for many (x, decoded scale) pairs."""
    x = _c(x, np.float64)
    s = _c(s, np.float64)
    out = np.zeros(x.shape[0], np.uint8)
    lib().orc_fp4_codes_many(_p(x), _p(s), x.shape[0], _p(out))
    return out


def quantize_block16(x):
    x = _c(x, np.float64)
    codes = np.zeros(16, np.uint8)
    sc = np.zeros(1, np.uint8)
    lib().orc_quantize_block16(_p(x), _p(codes), _p(sc))
    return codes, int(sc[0])


def quantize_entries(kv_bits, D=512):
    """kv_bits: uint16 [n, D] bf16 patterns -> (codes uint8 [n, D/2], scales uint8 [n, D/16])."""
    kv_bits = _c(kv_bits, np.uint16).reshape(-1, D)
    n = kv_bits.shape[0]
    codes = np.zeros((n, D // 2), np.uint8)
    scales = np.zeros((n, D // 16), np.uint8)
    lib().orc_quantize_entries(_p(kv_bits), n, D, D, _p(codes), _p(scales))
    return codes, scales


def dequant_entries(codes, scales, D=512):
    codes = _c(codes, np.uint8).reshape(-1, D // 2)
    scales = _c(scales, np.uint8).reshape(-1, D // 16)
    out = np.zeros((codes.shape[0], D), np.float64)
    for i in range(codes.shape[0]):
        row = out[i]
        lib().orc_dequant_entry(_p(codes[i]), _p(scales[i]), D, _p(row))
    return out


# ---- indexer / selection ---------------------------------------------------------------

def index_scores(q, w, k, dtype, rows=None):
    """q: [H, Di] raw (uint16 bf16 or uint8 E4M3); w: float32 [H]; k: [n_all, Di] raw.
    rows: optional int32 positions; returns float64 scores for rows (or all rows)."""
    npdt = np.uint16 if dtype == BF16 else np.uint8
    q = _c(q, npdt)
    k = _c(k, npdt)
    w = _c(w, np.float32)
    H, Di = q.shape
    if rows is None:
        n = k.shape[0]
        r = None
    else:
        r = _c(rows, np.int32)
        n = r.shape[0]
    s = np.zeros(n, np.float64)
    lib().orc_index_scores(H, Di, dtype, _p(q), _p(w), _p(k), _p(r), n, _p(s))
    return s


def topk(scores, K, ids=None):
    s = _c(scores, np.float64)
    i = _c(ids, np.int32) if ids is not None else None
    out = np.zeros(K, np.int32)
    lib().orc_topk(_p(s), _p(i), s.shape[0], K, _p(out))
    return out


def pool(scores, nblk, blk=POOL_BLOCK):
    s = _c(scores, np.float64)
    out = np.zeros(nblk * blk, np.int32)
    lib().orc_pool(_p(s), s.shape[0], nblk, blk, _p(out))
    return out


# ---- attention ---------------------------------------------------------------------

def attention(q, rows, tau):
    """q: float64 [H, D]; rows: float64 [n, D] -> float64 [H, D]."""
    q = _c(q, np.float64)
    rows = _c(rows, np.float64).reshape(-1, q.shape[1])
    H, D = q.shape
    out = np.zeros((H, D), np.float64)
    lib().orc_attention(H, D, _p(q), _p(rows), rows.shape[0], float(tau), _p(out))
    return out


def gather_rows(codes, scales, idx, D=512):
    """Dequantised main-KV rows for the indices != -1, in the order given."""
    sel = [int(i) for i in idx if i >= 0]
    if not sel:
        return np.zeros((0, D), np.float64)
    return dequant_entries(codes[sel], scales[sel], D)


def attention_decode_query(q_bits, codes, scales, idx, swa_codes, tau, swa_valid=None, D=512):
    """One decode query: q bf16 bits [H, D]; idx [K]; swa E4M3 [W, D] (last swa_valid
    rows valid when given). Returns float64 [H, D]."""
    q = bf16_array_to_f64(q_bits).reshape(-1, D)
    sel = gather_rows(codes, scales, idx, D)
    W = swa_codes.shape[0]
    v = W if swa_valid is None else int(swa_valid)
    swa = e4m3_array_to_f64(swa_codes[W - v:]).reshape(-1, D)
    rows = np.concatenate([sel, swa], axis=0)
    return attention(q, rows, tau)


# ---- prefill: causal visibility, window rows, one whole query ------------------------------

def prefill_visible(p, ratio):
    """Compressed entries visible to the token at position p (the prefix 0 .. n-1)."""
    return int(lib().orc_prefill_visible(int(p), int(ratio)))


def prefill_window_rows(q_pos0, W, t):
    """Rows of a prefill chunk's [W-1+T] window buffer that token t attends to (ascending)."""
    out = np.zeros(max(int(W), 1), np.int32)
    n = lib().orc_prefill_window_rows(int(q_pos0), int(W), int(t), _p(out))
    return out[:n].copy()


def prefill_query(qi_raw, w, k_raw, dtype, kv_bits, q_bits, swa_buf, q_pos0, t, ratio, K, W,
                  tau, D=512, idx_override=None):
    """One prefill query token t of a chunk starting at position q_pos0, step by step:
    indexer scores over the entries visible at p = q_pos0 + t, Top-K, then attention over
    the selected entries (quantised by the oracle from their bf16 source rows kv_bits
    [n, D]) plus the token's causal window rows of swa_buf (E4M3 [W-1+T, D]).
    idx_override: attend over these indices instead of the oracle's own Top-K (for picks
    that differ inside the near-tie exemption). Returns (idx [K], out float64 [H, D])."""
    if idx_override is None:
        n = prefill_visible(q_pos0 + t, ratio)
        s = index_scores(qi_raw, w, k_raw[:n], dtype)
        idx = topk(s, K)
    else:
        idx = np.asarray(idx_override, np.int32)
    sel = [int(i) for i in idx if i >= 0]
    kvb = _c(kv_bits, np.uint16).reshape(-1, D)
    if sel:
        c, sc = quantize_entries(kvb[sel], D)
        main = dequant_entries(c, sc, D)
    else:
        main = np.zeros((0, D), np.float64)
    win = e4m3_array_to_f64(_c(swa_buf, np.uint8).reshape(-1, D)[prefill_window_rows(q_pos0, W, t)])
    q = bf16_array_to_f64(q_bits).reshape(-1, D)
    return idx, attention(q, np.concatenate([main, win.reshape(-1, D)], axis=0), tau)


# ---- KV compressor and indexer-K projection ----------------------------------------------

def bf16_encode(v):
    """bf16 bit pattern of v (round to nearest, ties to even)."""
    return int(lib().orc_bf16_encode(float(v)))


def bf16_encode_many(v):
    v = _c(v, np.float64)
    out = np.zeros(v.shape, np.uint16)
    lib().orc_bf16_encode_many(_p(v), v.size, _p(out))
    return out


def compress_entries(c_bits, z_bits, r):
    """c_bits, z_bits: uint16 [r * n, D] bf16 patterns of one sequence's source tokens.
    Returns float64 [n, D]: per channel, the softmax over each entry's r tokens of the
    logits weighting their latents."""
    c_bits = _c(c_bits, np.uint16)
    z_bits = _c(z_bits, np.uint16)
    assert c_bits.shape == z_bits.shape and c_bits.shape[0] % r == 0
    n, D = c_bits.shape[0] // r, c_bits.shape[1]
    out = np.zeros((n, D), np.float64)
    lib().orc_compress_entries(_p(c_bits), _p(z_bits), n, int(r), D, D, _p(out))
    return out


def project_keys(x, w_bits):
    """x: float64 [n, D] entry latents; w_bits: uint16 [Di, D] bf16 patterns.
    Returns float64 [n, Di] = x @ W^T."""
    x = _c(x, np.float64)
    w_bits = _c(w_bits, np.uint16)
    Di, D = w_bits.shape
    out = np.zeros((x.shape[0], Di), np.float64)
    lib().orc_project_keys(_p(x), x.shape[0], D, _p(w_bits), Di, _p(out))
    return out


def compress_write(c_bits, z_bits, r, w_bits, key_dtype):
    """The whole write of one sequence's new entries: pooled latents rounded to bf16,
    their FP4 codes and scales, and the indexer keys (E4M3 codes or bf16 patterns).
    Returns (latent_bits uint16 [n, D], codes, scales, key_raw, key_exact float64)."""
    lat_bits = bf16_encode_many(compress_entries(c_bits, z_bits, r))
    codes, scales = quantize_entries(lat_bits, D=lat_bits.shape[1])
    k = project_keys(bf16_array_to_f64(lat_bits), w_bits)
    key_raw = (e4m3_encode_many(k.ravel()).reshape(k.shape) if key_dtype == E4M3
               else bf16_encode_many(k))
    return lat_bits, codes, scales, key_raw, k


# ---- compact 68-byte indexer keys -------------------------------------------------------

def quantize_keys_fp4(k_bits):
    """k_bits: uint16 [n, Di] bf16 patterns -> (codes uint8 [n, Di/2], scales float32 [n])."""
    k_bits = _c(k_bits, np.uint16)
    n, Di = k_bits.shape
    codes = np.zeros((n, Di // 2), np.uint8)
    scales = np.zeros(n, np.float32)
    lib().orc_quantize_keys_fp4(_p(k_bits), n, Di, _p(codes), _p(scales))
    return codes, scales


def dequant_keys_fp4(codes, scales):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    n, half = codes.shape
    out = np.zeros((n, 2 * half), np.float64)
    for i in range(n):
        row = out[i]
        lib().orc_dequant_key_fp4(_p(codes[i]), float(scales[i]), 2 * half, _p(row))
    return out


def index_scores_fp4key(q, w, codes, scales, rows=None):
    """q: uint8 [H, Di] E4M3; w: float32 [H]; codes uint8 [n_all, Di/2]; scales float32
    [n_all]. Returns float64 scores for rows (or all rows)."""
    q = _c(q, np.uint8)
    w = _c(w, np.float32)
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    H, Di = q.shape
    if rows is None:
        n, r = codes.shape[0], None
    else:
        r = _c(rows, np.int32)
        n = r.shape[0]
    s = np.zeros(n, np.float64)
    lib().orc_index_scores_fp4key(H, Di, _p(q), _p(w), _p(codes), _p(scales), _p(r), n, _p(s))
    return s


def bytes_per_token(D=512, indexer_entry_bytes=68.0, enc_full=3, enc_ratio=2, dec_full=1,
                    dec_ratio=1):
    return lib().orc_kv_bytes_per_token(D, float(indexer_entry_bytes), enc_full, enc_ratio,
                                        dec_full, dec_ratio)


def main_entry_bytes(D=512):
    return lib().orc_main_entry_bytes(D)
