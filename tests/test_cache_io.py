"""Persistent-cache records (csa2_cache_record_bytes / _export / _import).

CPU: the record size against the oracle's per-entry and per-token byte accounting, and the
header checks that reject a bad record before any copy is issued. GPU: export then import
moves the entries bit for bit (with and without indexer keys, E4M3 and bf16 keys) and
touches nothing else."""
import ctypes as C

import numpy as np
import pytest
import torch

from fp4_compressed_sparse_quantize_b200 import csa2
from oracle import oracle as O


def test_record_bytes_match_the_byte_accounting():
    hdr = csa2.cache_record_bytes(0)
    assert hdr == 64
    assert csa2.cache_record_bytes(1) - hdr == O.main_entry_bytes() == 288
    assert csa2.cache_record_bytes(10, 128) == hdr + 10 * (288 + 128)
    assert csa2.cache_record_bytes(10, 256) == hdr + 10 * (288 + 256)
    assert csa2.cache_record_bytes(10, 100) == 0
    assert csa2.cache_record_bytes(-1) == 0
    # 2.5 stored entry sets per token: a record entry with E4M3 keys is the oracle's
    # per-token footprint at b_I = 128 divided by 2.5
    per_entry = csa2.cache_record_bytes(1, 128) - hdr
    assert 2.5 * per_entry == O.bytes_per_token(indexer_entry_bytes=128.0) == 1040.0


def _header(magic=0x32415343, version=1, d=512, di=128, lo=0, n=4, kb=0, eb=288):
    h = np.zeros(64, np.uint8)
    h[0:16] = np.array([magic, version, d, di], np.uint32).view(np.uint8)
    h[16:32] = np.array([lo, n], np.int64).view(np.uint8)
    h[32:40] = np.array([kb, eb], np.uint32).view(np.uint8)
    return h


@pytest.mark.parametrize("bad,status", [(dict(magic=0x12345678), csa2.ERR_ARG),
                                        (dict(version=2), csa2.ERR_ARG),
                                        (dict(d=256), csa2.ERR_UNSUPPORTED),
                                        (dict(eb=300), csa2.ERR_ARG),
                                        (dict(kb=100, eb=388), csa2.ERR_ARG),
                                        (dict(lo=998), csa2.ERR_ARG),
                                        (dict(n=1000), csa2.ERR_ARG),
                                        # forged ranges whose sums or byte sizes overflow
                                        (dict(lo=2**62, n=2**62), csa2.ERR_ARG),
                                        (dict(lo=2**63 - 1, n=1), csa2.ERR_ARG),
                                        (dict(lo=-1, n=2), csa2.ERR_ARG),
                                        (dict(lo=0, n=2**60), csa2.ERR_ARG),
                                        (dict(kb=2**31 + 128, eb=416), csa2.ERR_ARG)])
def test_import_rejects_bad_records_before_copying(bad, status):
    rec = np.zeros(64 + 4 * 288, np.uint8)
    rec[:64] = _header(**bad)
    fake = C.c_void_p(256)   # never dereferenced: the header check fails first
    st = csa2.lib().csa2_cache_import(rec.ctypes.data_as(C.c_void_p), rec.nbytes, fake, fake,
                                      None, 1000, 0, None)
    assert st == status


def test_record_bytes_overflow_is_rejected():
    assert csa2.cache_record_bytes(2**62) == 0
    assert csa2.cache_record_bytes(2**62, 256) == 0


def test_export_rejects_bad_arguments():
    fake = C.c_void_p(256)
    host = np.zeros(64 + 8 * 416, np.uint8)
    hp = host.ctypes.data_as(C.c_void_p)
    L = csa2.lib()
    # range past the capacity, keys without a key cache, host buffer too small
    assert L.csa2_cache_export(fake, fake, None, 0, 100, 0, 96, 8, hp, host.nbytes, None) == csa2.ERR_ARG
    assert L.csa2_cache_export(fake, fake, None, 128, 100, 0, 0, 8, hp, host.nbytes, None) == csa2.ERR_ARG
    assert L.csa2_cache_export(fake, fake, fake, 128, 100, 0, 0, 8, hp, 64 + 8 * 300, None) == csa2.ERR_ARG
    # ranges whose end overflows int64, and a sequence offset past int64
    assert L.csa2_cache_export(fake, fake, None, 0, 100, 0, 2**63 - 1, 8, hp, host.nbytes, None) == csa2.ERR_ARG
    assert L.csa2_cache_export(fake, fake, None, 0, 2**62, 2**30, 0, 8, hp, host.nbytes, None) == csa2.ERR_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("key_dtype", [None, torch.float8_e4m3fn, torch.bfloat16])
def test_gpu_export_import_round_trip(key_dtype):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dev = "cuda"
    g = torch.Generator().manual_seed(5)
    B, cap, lo, n = 3, 1000, 100, 333
    kv = torch.randn((B, cap, 512), generator=g).to(torch.bfloat16).to(dev)
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    csa2.quantize_kv(kv, torch.zeros(B, dtype=torch.int32, device=dev), codes, scales)
    k_I = None
    if key_dtype is not None:
        k_I = torch.randn((B, cap, 128), generator=g).to(key_dtype).to(dev)
    kb = 0 if k_I is None else 128 * k_I.element_size()
    host = torch.zeros(csa2.cache_record_bytes(n, kb), dtype=torch.uint8).pin_memory()
    csa2.cache_export(codes, scales, 1, lo, n, host, k_I=k_I)
    torch.cuda.synchronize()
    h = host[:64].numpy()
    assert h[:16].view(np.uint32).tolist() == [0x32415343, 1, 512, 128]
    assert h[16:32].view(np.int64).tolist() == [lo, n]
    assert h[32:40].view(np.uint32).tolist() == [kb, 288 + kb]
    c2 = torch.zeros_like(codes)
    s2 = torch.zeros_like(scales)
    k2 = torch.zeros_like(k_I) if k_I is not None else None
    csa2.cache_import(host, c2, s2, 2, k_I=k2)
    torch.cuda.synchronize()
    assert torch.equal(c2[2, lo:lo + n], codes[1, lo:lo + n])
    assert torch.equal(s2[2, lo:lo + n], scales[1, lo:lo + n])
    assert int(c2[2, :lo].sum()) == int(c2[2, lo + n:].sum()) == int(c2[:2].sum()) == 0
    assert int(s2[2, :lo].sum()) == int(s2[:2].sum()) == 0
    if k_I is not None:
        assert torch.equal(k2[2, lo:lo + n].view(torch.uint8), k_I[1, lo:lo + n].view(torch.uint8))
        assert int(k2[:2].view(torch.uint8).sum()) == 0
    # a record with keys cannot be imported without a key cache, and vice versa
    with pytest.raises(csa2.Csa2Error):
        other = None if k_I is not None else torch.zeros((B, cap, 128), dtype=torch.uint8, device=dev)
        csa2.cache_import(host, c2, s2, 0, k_I=other)
