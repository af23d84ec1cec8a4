"""The no-allocation indexer entry point, for callers that cannot allocate device memory
(plugins inside a framework that owns every allocation, latency-critical loops where an
allocation may synchronise the device): it must give exactly what the regular entry point
gives, on two calls in a row (the library's fixed scratch array is reused between calls),
and refuse requests larger than its fixed 16 MiB scratch array.

Collected last on purpose, so that a run stopping at the first failure has already run
every other test."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
dev = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield


def _inputs(seed, B, n, H_I):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    k_I = torch.randn((B, n, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
    q_I = torch.randn((B, 1, H_I, 128), generator=g).to(torch.float8_e4m3fn).to(dev)
    w = torch.rand((B, 1, H_I), generator=g).to(dev)
    return k_I, q_I, w


def test_noalloc_matches_workspace_entry_point_twice():
    from fp4_compressed_sparse_quantize_b200 import csa2
    B, n, H_I, K, nblk = 4, 20000, 64, 512, 512
    k_I, q_I, w = _inputs(31, B, n, H_I)
    n_vis = torch.tensor([n, n - 3, 9000, 511], dtype=torch.int32, device=dev)
    # regular entry point with a caller workspace
    idx_ref = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    pool_ref = torch.empty((B, 1, nblk * 8), dtype=torch.int32, device=dev)
    ws = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, H_I, n, K, nblk))
    csa2.index_score_topk("full", q_I, w, k_I, K, idx_ref, ws, n_vis0=n_vis, pool_out=pool_ref,
                          pool_blocks=nblk)
    torch.cuda.synchronize()
    assert csa2.read_device_status(ws) == 0
    for call in range(2):
        idx = torch.full((B, 1, K), -7, dtype=torch.int32, device=dev)
        pool = torch.full((B, 1, nblk * 8), -7, dtype=torch.int32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        csa2.index_score_topk_noalloc("full", q_I, w, k_I, K, idx, n_vis0=n_vis, pool_out=pool,
                                      pool_blocks=nblk, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}"
        assert torch.equal(idx, idx_ref), f"call {call}: indices differ"
        assert torch.equal(pool, pool_ref), f"call {call}: pool differs"
    # Reindex through the no-allocation path as well
    P = nblk * 8
    idx2_ref = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    ws2 = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, H_I, P, K))
    csa2.index_score_topk("reindex", q_I, w, k_I, K, idx2_ref, ws2, n_vis0=n_vis,
                          pool_in=pool_ref)
    idx2 = torch.empty_like(idx2_ref)
    status2 = torch.zeros(1, dtype=torch.int32, device=dev)
    csa2.index_score_topk_noalloc("reindex", q_I, w, k_I, K, idx2, n_vis0=n_vis,
                                  pool_in=pool_ref, status=status2)
    torch.cuda.synchronize()
    assert csa2.read_device_status(ws2) == 0
    assert int(status2.item()) == 0, "device status of the Reindex call"
    assert torch.equal(idx2, idx2_ref)


def test_noalloc_rejects_requests_above_its_fixed_size():
    from fp4_compressed_sparse_quantize_b200 import csa2
    B, n, H_I, K = 64, 262144, 64, 512     # ~100 MB of workspace: far above 16 MiB
    assert csa2.workspace_bytes(0, B, 1, H_I, n, K) > (16 << 20)
    q_I = torch.zeros((B, 1, H_I, 128), dtype=torch.float8_e4m3fn, device=dev)
    w = torch.zeros((B, 1, H_I), device=dev)
    k_I = torch.zeros((B, 16, 128), dtype=torch.float8_e4m3fn, device=dev)
    idx = torch.empty((B, 1, K), dtype=torch.int32, device=dev)
    n_vis = torch.zeros(B, dtype=torch.int32, device=dev)
    lib = csa2.lib()
    import ctypes as C
    st = lib.csa2_index_score_topk_noalloc(
        0, B, 1, H_I, 1, C.c_void_p(q_I.data_ptr()), C.c_void_p(w.data_ptr()),
        C.c_void_p(k_I.data_ptr()), n, C.c_void_p(n_vis.data_ptr()), 1, None, K, None, 0, None,
        0, C.c_void_p(idx.data_ptr()), None, None, None)
    assert st == csa2.ERR_WORKSPACE
