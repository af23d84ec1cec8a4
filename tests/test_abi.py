"""CPU-side checks of the C ABI: the library loads without a GPU, exports every entry point
that include/csa2.h declares, and rejects bad arguments on the host (no device work)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp4_compressed_sparse_quantize_b200 import build
    build.build()
    from fp4_compressed_sparse_quantize_b200 import csa2
    return csa2.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "csa2.h")).read()
    return sorted(set(re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", text)))


def test_header_declares_the_four_path_calls():
    names = declared_functions()
    for n in ("csa2_quantize_kv", "csa2_index_score_topk", "csa2_sparse_attn_decode",
              "csa2_sparse_attn_prefill", "csa2_workspace_bytes", "csa2_status_string",
              "csa2_read_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    from fp4_compressed_sparse_quantize_b200 import csa2
    assert set(csa2.EXPORTS) <= set(declared_functions())


def test_status_strings(lib):
    from fp4_compressed_sparse_quantize_b200 import csa2
    for s in range(6):
        assert csa2.status_string(s)
    assert "unknown" in csa2.status_string(99)


def test_workspace_sizes(lib):
    from fp4_compressed_sparse_quantize_b200 import csa2
    a = csa2.workspace_bytes(0, 32, 1, 64, 32768, 512)
    b = csa2.workspace_bytes(0, 32, 1, 64, 65536, 512)
    assert 0 < a < b
    assert csa2.workspace_bytes(0, 4, 1, 64, 1 << 20, 512, 2048) > csa2.workspace_bytes(0, 4, 1, 64, 1 << 20, 512)
    assert csa2.workspace_bytes(0, 0, 1, 64, 1000, 512) == 0
    assert csa2.workspace_bytes(2, 2, 4096, 64, 1000, 512) == 256
    assert csa2.workspace_bytes(1, 32, 1, 64, 1000, 512) > 256


def _ptr(v):
    return C.c_void_p(v)


def test_host_validation_rejects_without_launch(lib):
    from fp4_compressed_sparse_quantize_b200 import csa2
    P = _ptr(0x10000)      # never dereferenced: validation fails first
    odd = _ptr(0x10001)
    # index_score_topk: bad mode, K > 2048, null idx, reindex without pool, misalignment
    f = lib.csa2_index_score_topk
    args = dict(mode=0, B=1, T=1, H_I=64, dt=1, q=P, w=P, k=P, cap=100, n=P, r=1, qp=None, K=8,
                pin=None, P_in=0, pout=None, pb=0, idx=P, sc=None, ws=P, wsb=1 << 30, st=None)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return f(a["mode"], a["B"], a["T"], a["H_I"], a["dt"], a["q"], a["w"], a["k"], a["cap"],
                 a["n"], a["r"], a["qp"], a["K"], a["pin"], a["P_in"], a["pout"], a["pb"],
                 a["idx"], a["sc"], a["ws"], a["wsb"], a["st"])
    assert call(mode=7) == csa2.ERR_ARG
    assert call(K=4096) == csa2.ERR_UNSUPPORTED
    assert call(idx=None) == csa2.ERR_ARG
    assert call(mode=1) == csa2.ERR_ARG                 # Reindex needs pool_in
    assert call(pin=P, P_in=16) == csa2.ERR_ARG         # Full must not get pool_in
    assert call(q=odd) == csa2.ERR_ARG
    assert call(H_I=129) == csa2.ERR_UNSUPPORTED
    assert call(T=2) == csa2.ERR_ARG                    # T > 1 needs q_pos0
    assert call(ws=None) == csa2.ERR_WORKSPACE
    assert call(wsb=16) == csa2.ERR_WORKSPACE
    assert call(pout=P, pb=5000) == csa2.ERR_ARG
    assert call(mode=2) == csa2.OK                      # Reuse: validated, nothing launched
    assert call(mode=2, pin=P) == csa2.ERR_ARG
    # attention
    g = lib.csa2_sparse_attn_decode
    assert g(0, 1, 65, P, P, P, 10, P, 4, P, 128, None, 0.1, P, P, 1 << 20, None) == csa2.ERR_UNSUPPORTED
    assert g(0, 1, 64, P, P, P, 10, P, 4, P, 2000, None, 0.1, P, P, 1 << 20, None) == csa2.ERR_UNSUPPORTED
    assert g(0, 1, 64, None, P, P, 10, P, 4, P, 128, None, 0.1, P, P, 1 << 20, None) == csa2.ERR_ARG
    assert g(0, 1, 64, P, P, P, 10, P, 4, P, 128, None, 0.1, P, None, 0, None) == csa2.ERR_WORKSPACE
    assert g(9, 1, 64, P, P, P, 10, P, 4, P, 128, None, 0.1, P, P, 1 << 20, None) == csa2.ERR_ARG
    assert g(0, 1, 64, P, P, P, 10, P, 4, P, 128, None, float("nan"), P, P, 1 << 20, None) == csa2.ERR_ARG
    h = lib.csa2_sparse_attn_prefill
    assert h(1, 4, 64, P, P, P, 10, None, 4, P, 128, None, 0.1, P, P, 1 << 20, None) == csa2.ERR_ARG
    # quantize
    q = lib.csa2_quantize_kv
    assert q(P, 1, 1, 500, 512, P, P, P, 10, None, None) == csa2.ERR_ARG   # ld_kv < 512
    assert q(odd, 1, 1, 512, 512, P, P, P, 10, None, None) == csa2.ERR_ARG
    assert q(None, 0, 1, 512, 512, P, P, P, 10, None, None) == csa2.OK     # nothing to do
    # compressor + projection: (B, n_new, r, C, Z, ld, bstride, w_proj, key_dtype, dst_off,
    # codes, scales, k_I, cap, latent_out, status, stream)
    c = lib.csa2_compress_kv
    ok = (1, 4, 2, P, P, 512, 8 * 512, P, 1, P, P, P, P, 100, None, None, None)

    def cz(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return c(*a)
    assert cz(_2=0) == csa2.ERR_ARG and cz(_2=65) == csa2.ERR_ARG      # ratio outside 1..64
    assert cz(_5=504) == csa2.ERR_ARG                                   # ld < 512
    assert cz(_3=odd) == csa2.ERR_ARG and cz(_7=None) == csa2.ERR_ARG   # misaligned C, no W
    assert cz(_8=7) == csa2.ERR_ARG                                     # unknown key type
    assert cz(_8=2, _12=_ptr(0x10010)) == csa2.ERR_ARG                  # compact keys: 32-B aligned
    assert cz(_14=odd) == csa2.ERR_ARG                                  # misaligned latent_out
    assert cz(_1=0) == csa2.OK                                          # nothing to do
    # compact-key quantiser: (k, B, n_new, ld, bstride, dst_off, keys, cap, status, stream)
    kq = lib.csa2_quantize_keys_fp4
    assert kq(P, 1, 4, 120, 1024, P, P, 100, None, None) == csa2.ERR_ARG   # ld < 128
    assert kq(odd, 1, 4, 128, 1024, P, P, 100, None, None) == csa2.ERR_ARG
    assert kq(P, 1, 4, 128, 1024, P, _ptr(0x10010), 100, None, None) == csa2.ERR_ARG
    assert kq(P, 1, 0, 128, 1024, P, P, 100, None, None) == csa2.OK
    # compact keys in index_score_topk: the key buffer must be 32-byte aligned
    assert call(dt=2, k=_ptr(0x10010)) == csa2.ERR_ARG
    assert call(dt=3) == csa2.ERR_ARG
    assert lib.csa2_read_device_status(None, None, None) == csa2.ERR_ARG
    assert lib.csa2_debug_bounded_wait(P, 0, None) == csa2.ERR_ARG
