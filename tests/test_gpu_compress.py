"""GPU parity of csa2_compress_kv (KV compressor + indexer-K projection + FP4 write) with the
oracle, through the C ABI.

Floating point decides two integer outputs here, and each decision is compared from the
same input on both sides:
  * the pooled latent's bf16 rounding: the GPU's fp32 softmax may land on the other side
    of a bf16 midpoint only where the oracle's exact value sits within fp32 error of it;
  * the FP4 codes and scales are then bit-exact against the oracle's quantizer applied to
    the GPU's bf16 latent;
  * the key's E4M3 (or bf16) rounding: the tensor cores accumulate in fp32, so a key may
    differ from the oracle's rounding of the exact projection of the GPU latent only where
    that exact value is within the accumulation error bound of a midpoint."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import bits16, bits8

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


def _near_midpoint_ok(got, want, exact, tol):
    """got/want/exact float64 arrays: got equals want, or exact is (within tol) equidistant
    from the two. Returns the number of accepted differences."""
    diff = got != want
    if not diff.any():
        return 0
    gap = np.abs(np.abs(got - exact) - np.abs(want - exact))
    bad = diff & (gap > 2 * tol)
    assert not bad.any(), (f"{int(bad.sum())} roundings differ away from a midpoint; first at "
                           f"{np.argwhere(bad)[0]}: got {got[bad][0]!r} want {want[bad][0]!r} "
                           f"exact {exact[bad][0]!r}")
    return int(diff.sum())


def _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent, key_dtype, n_new, skip=()):
    """Compare every written entry of every sequence with the oracle."""
    B = Cs.shape[0]
    Wb = bits16(W)
    flips = total = 0
    for b in range(B):
        if b in skip:
            continue
        cb = bits16(Cs[b, :r * n_new])
        zb = bits16(Zs[b, :r * n_new])
        exact = O.compress_entries(cb, zb, r)                      # fp64 pooled latent
        lat = bits16(latent[b]) if latent is not None else None
        # bf16 decision: tolerance = fp32 error of a convex combination of r terms
        cmax = np.abs(O.bf16_array_to_f64(cb)).reshape(n_new, r, 512).max(axis=1)
        flips += _near_midpoint_ok(O.bf16_array_to_f64(lat), O.bf16_array_to_f64(
            O.bf16_encode_many(exact)), exact, 4e-6 * cmax + 1e-30)
        total += lat.size
        # FP4 write of the GPU latent: bit-exact
        qc, qs = O.quantize_entries(lat)
        d0 = int(dst[b])
        np.testing.assert_array_equal(bits8(codes[b, d0:d0 + n_new]), qc, f"codes b={b}")
        np.testing.assert_array_equal(bits8(scales[b, d0:d0 + n_new]), qs, f"scales b={b}")
        # key: projection of the GPU latent
        lat_v = O.bf16_array_to_f64(lat)
        kx = O.project_keys(lat_v, Wb)
        tol = 1e-5 * (np.abs(lat_v) @ np.abs(O.bf16_array_to_f64(Wb)).T) + 1e-30
        if key_dtype == torch.float8_e4m3fn:
            got = O.e4m3_array_to_f64(bits8(keys[b, d0:d0 + n_new]).ravel()).reshape(kx.shape)
            want = O.e4m3_array_to_f64(O.e4m3_encode_many(kx.ravel())).reshape(kx.shape)
            # saturation: both sides clamp at 448
        else:
            got = O.bf16_array_to_f64(bits16(keys[b, d0:d0 + n_new]))
            want = O.bf16_array_to_f64(O.bf16_encode_many(kx))
        flips += _near_midpoint_ok(got, want, kx, tol)
        total += kx.size
    return flips, total


def _case(B, n_new, r, cap, dst, key_dtype, seed, ld_pad=0, zscale=2.0):
    g = _gen(seed)
    n_tok = r * n_new
    big = torch.randn((B, n_tok, 512 + ld_pad), generator=g).to(torch.bfloat16)
    Cs = big[:, :, :512]
    Zs = (torch.randn((B, n_tok, 512 + ld_pad), generator=g) * zscale).to(torch.bfloat16)[:, :, :512]
    W = (torch.randn((128, 512), generator=g) * 0.06).to(torch.bfloat16)
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    keys = torch.zeros((B, cap, 128), dtype=key_dtype, device=dev)
    latent = torch.zeros((B, n_new, 512), dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    Cd = big.to(dev)[:, :, :512]
    Zd = Zs.to(dev) if ld_pad == 0 else None
    if ld_pad:
        # Z with the same padded strides as C
        zbig = torch.zeros((B, n_tok, 512 + ld_pad), dtype=torch.bfloat16, device=dev)
        zbig[:, :, :512] = Zs.to(dev)
        Zd = zbig[:, :, :512]
    C().compress_kv(Cd, Zd, r, W.to(dev), torch.tensor(dst, dtype=torch.int32, device=dev),
                    codes, scales, keys, latent_out=latent, status=st)
    torch.cuda.synchronize()
    return Cs, Zs, W, codes.cpu(), scales.cpu(), keys.cpu(), latent.cpu(), int(st.item())


@pytest.mark.parametrize("key_dtype", [torch.float8_e4m3fn, torch.bfloat16])
def test_compress_ragged_two_tiles(key_dtype):
    B, n_new, r, cap = 2, 100, 2, 300
    dst = [5, 0]
    Cs, Zs, W, codes, scales, keys, latent, st = _case(B, n_new, r, cap, dst, key_dtype, 31)
    assert st == 0
    flips, total = _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent, key_dtype, n_new)
    assert flips <= 1e-3 * total
    # nothing outside the written rows
    assert int(codes[0, :5].sum()) == 0 and int(codes[0, 105:].sum()) == 0
    assert int(scales[1, 100:].sum()) == 0
    assert int(keys[1, 100:].view(torch.uint8).sum()) == 0


def test_compress_ratio_one_is_quantize_of_the_latents():
    B, n_new, r, cap = 3, 40, 1, 64
    dst = [0, 10, 24]
    Cs, Zs, W, codes, scales, keys, latent, st = _case(B, n_new, r, cap, dst, torch.float8_e4m3fn, 32)
    assert st == 0
    for b in range(B):
        np.testing.assert_array_equal(bits16(latent[b]), bits16(Cs[b]))   # softmax of one token
        qc, qs = O.quantize_entries(bits16(Cs[b]))
        np.testing.assert_array_equal(bits8(codes[b, dst[b]:dst[b] + n_new]), qc)
        np.testing.assert_array_equal(bits8(scales[b, dst[b]:dst[b] + n_new]), qs)
    _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent, torch.float8_e4m3fn, n_new)


def test_compress_strided_inputs_ratio_four_and_bad_offset():
    B, n_new, r, cap = 3, 37, 4, 50
    dst = [13, 40, 0]           # sequence 1 runs past cap: its last 27 entries are skipped
    Cs, Zs, W, codes, scales, keys, latent, st = _case(B, n_new, r, cap, dst, torch.float8_e4m3fn,
                                                       33, ld_pad=64)
    assert st & C().DEV_BAD_INDEX
    _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent, torch.float8_e4m3fn, n_new,
           skip=(1,))
    # sequence 1: the entries that fit are written, the rest are not
    lat1 = bits16(latent[1, :10])
    qc, qs = O.quantize_entries(lat1)
    np.testing.assert_array_equal(bits8(codes[1, 40:50]), qc)
    assert int(codes[1, :40].sum()) == 0


def test_compress_decode_shape_and_prefill_chunk():
    # decode: one entry per sequence, 32 sequences
    dst = list(range(100, 132))
    Cs, Zs, W, codes, scales, keys, latent, st = _case(32, 1, 2, 200, dst, torch.float8_e4m3fn, 34)
    assert st == 0
    flips, total = _check(Cs, Zs, 2, W, dst, 200, codes, scales, keys, latent,
                          torch.float8_e4m3fn, 1)
    assert flips <= 2e-3 * total
    # a prefill chunk's writes: 2,048 entries per sequence at ratio 2 (32 CTAs)
    dst = [65536, 65536]
    Cs, Zs, W, codes, scales, keys, latent, st = _case(2, 2048, 2, 65536 + 2048, dst,
                                                       torch.float8_e4m3fn, 35)
    assert st == 0
    flips, total = _check(Cs, Zs, 2, W, dst, 65536 + 2048, codes, scales, keys, latent,
                          torch.float8_e4m3fn, 2048)
    assert flips <= 1e-3 * total


def test_compress_ratio_above_four():
    # more than four source tokens per entry: the per-token loop instead of the single batch
    # of loads, on a ragged count with strided inputs
    B, n_new, r, cap = 2, 45, 6, 64
    dst = [3, 19]
    Cs, Zs, W, codes, scales, keys, latent, st = _case(B, n_new, r, cap, dst, torch.float8_e4m3fn,
                                                       38, ld_pad=32)
    assert st == 0
    flips, total = _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent,
                          torch.float8_e4m3fn, n_new)
    assert flips <= 1e-3 * total
    assert int(codes[0, :3].sum()) == 0 and int(codes[0, 48:].sum()) == 0


def test_compress_sixteen_entries_per_cta():
    # 1,800 entries: the launch takes 16 entries per CTA (113 CTAs), between the decode
    # shape's 8 and a long chunk's 32
    B, n_new, r, cap = 2, 900, 2, 1000
    dst = [0, 100]
    Cs, Zs, W, codes, scales, keys, latent, st = _case(B, n_new, r, cap, dst, torch.float8_e4m3fn, 37)
    assert st == 0
    flips, total = _check(Cs, Zs, r, W, dst, cap, codes, scales, keys, latent,
                          torch.float8_e4m3fn, n_new)
    assert flips <= 1e-3 * total
    assert int(codes[1, :100].sum()) == 0 and int(codes[0, 900:].sum()) == 0


def test_compress_writes_compact_keys():
    """With compact 68-byte keys the compressor stores csa2_quantize_keys_fp4's encoding of
    the bf16-rounded projection. The same call with bf16 keys yields that projection exactly
    (the MMA is deterministic), so the compact keys are compared bit for bit with the
    oracle's quantiser applied to it."""
    g = _gen(36)
    B, n_new, r, cap = 2, 300, 2, 400
    dst = [0, 57]
    Cs = torch.randn((B, r * n_new, 512), generator=g).to(torch.bfloat16).to(dev)
    Zs = (torch.randn((B, r * n_new, 512), generator=g) * 2).to(torch.bfloat16).to(dev)
    W = (torch.randn((128, 512), generator=g) * 0.06).to(torch.bfloat16).to(dev)
    d = torch.tensor(dst, dtype=torch.int32, device=dev)
    outs = []
    for kind in ("bf16", "fp4"):
        codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
        scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
        keys = (torch.zeros((B, cap, 128), dtype=torch.bfloat16, device=dev) if kind == "bf16"
                else C().Fp4Keys(B, cap))
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        C().compress_kv(Cs, Zs, r, W, d, codes, scales, keys, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append((codes.cpu(), scales.cpu(), keys))
    (c0, s0, kb), (c1, s1, kf) = outs
    assert torch.equal(c0, c1) and torch.equal(s0, s1)
    codes = kf.codes.cpu().numpy()
    kscale = kf.scales.cpu().numpy()
    for b in range(B):
        oc, os_ = O.quantize_keys_fp4(bits16(kb[b, dst[b]:dst[b] + n_new]))
        np.testing.assert_array_equal(codes[b, dst[b]:dst[b] + n_new], oc, f"codes b={b}")
        np.testing.assert_array_equal(kscale[b, dst[b]:dst[b] + n_new].view(np.uint32),
                                      os_.view(np.uint32), f"scales b={b}")
    assert codes[1, :57].sum() == 0 and kscale[0, n_new:].sum() == 0
