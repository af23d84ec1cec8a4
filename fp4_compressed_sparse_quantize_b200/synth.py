"""Seeded synthetic workloads for CSA2 decode and prefill.

This module only draws random inputs and names their shapes. It holds none of the
method's arithmetic: every cast to a storage type (bf16, E4M3) is torch's own cast,
and the FP4 main-KV cache is NOT built here (callers quantise the bf16 source with
the path under test, or with the oracle).

Every tensor is drawn from its own torch.Generator seeded with
    seed0 + 1000 * tensor_number + sequence
so one sequence of one tensor can be regenerated alone. The stream of a generator
depends on the device, so a workload must always be drawn on the same device type
(all GPU tests and the benchmark draw on "cuda").

Shapes follow the pages' workloads: 512-channel main-KV latents, Top-512 selection,
a 128-token sliding window, compression ratio 1 or 2, contexts of 4K to 1M tokens,
2,048 x 8 = 16,384-position candidate pools.
"""
from dataclasses import dataclass, field

import torch

D_MAIN = 512      # main-KV latent channels
D_IDX = 128       # indexer key / query channels
WINDOW = 128      # sliding-window rows
POOL_BLOCKS = 2048
POOL_BLOCK = 8


@dataclass
class Workload:
    name: str
    kind: str                 # "decode" or "prefill"
    B: int
    ctx: int                  # tokens of context (decode) / cached tokens (prefill)
    ratio: int
    H_I: int
    idx_dtype: str            # "bf16" or "e4m3"
    K: int
    H: int
    layers: tuple = ("full",)  # per-layer CSA2 modes, in order
    T: int = 1                # new query tokens (prefill)
    lognormal_channels: bool = False
    planted: int = 0          # planted high-score keys per sequence (recall check)
    pool: bool = False        # Full layer also builds the candidate pool
    key_format: str = "dense"  # "dense" (keys in idx_dtype) or "fp4" (compact 68-byte keys,
                               # quantised by the library from bf16 keys; E4M3 queries)
    extra: dict = field(default_factory=dict)

    @property
    def N(self):
        """Visible compressed entries per sequence at decode; cached entries at prefill."""
        return self.ctx // self.ratio

    @property
    def n_new(self):
        """Entries quantised on write per step."""
        if self.kind == "prefill":
            return (self.ctx + self.T) // self.ratio - self.ctx // self.ratio
        return 1

    @property
    def cap(self):
        if self.kind == "prefill":
            return (self.ctx + self.T) // self.ratio
        return self.N


WORKLOADS = {
    # single Full layer, batch 1, 4K context, bf16 indexer, Top-64, 16 heads
    "decode_full_b1_ctx4k": Workload("decode_full_b1_ctx4k", "decode", B=1, ctx=4096, ratio=1,
                                     H_I=8, idx_dtype="bf16", K=64, H=16),
    # Full decode, batch 32, 64K context at ratio 2, FP8 indexer, per-channel LogNormal scales
    "decode_full_b32_ctx64k_r2": Workload("decode_full_b32_ctx64k_r2", "decode", B=32,
                                          ctx=65536, ratio=2, H_I=64, idx_dtype="e4m3",
                                          K=512, H=64, lognormal_channels=True),
    # decoder group: Full then 3 Reuse, batch 64, 256K context
    "decode_group4_b64_ctx256k": Workload("decode_group4_b64_ctx256k", "decode", B=64,
                                          ctx=262144, ratio=1, H_I=64, idx_dtype="e4m3",
                                          K=512, H=64,
                                          layers=("full", "reuse", "reuse", "reuse")),
    # 1M context: Full (+ candidate pool) then Reindex, batch 4, planted keys
    "decode_pool_reindex_b4_ctx1m": Workload("decode_pool_reindex_b4_ctx1m", "decode", B=4,
                                             ctx=1048576, ratio=1, H_I=64, idx_dtype="e4m3",
                                             K=512, H=64, layers=("full", "reindex"),
                                             planted=64, pool=True),
    # chunked prefill: 4096 new tokens on 128K cached, ratio 2
    "prefill_b2_t4k_ctx128k_r2": Workload("prefill_b2_t4k_ctx128k_r2", "prefill", B=2,
                                          ctx=131072, ratio=2, H_I=64, idx_dtype="e4m3",
                                          K=512, H=64, T=4096),
    # decode_full_b32_ctx64k_r2 with compact 68-byte indexer keys (890 bytes per token)
    "decode_full_b32_ctx64k_r2_key68": Workload("decode_full_b32_ctx64k_r2_key68", "decode",
                                                B=32, ctx=65536, ratio=2, H_I=64,
                                                idx_dtype="e4m3", K=512, H=64,
                                                lognormal_channels=True, key_format="fp4"),
    # the same chunked prefill at one sequence and 1024 new tokens (profiler captures)
    "prefill_b1_t1k_ctx128k_r2": Workload("prefill_b1_t1k_ctx128k_r2", "prefill", B=1,
                                          ctx=131072, ratio=2, H_I=64, idx_dtype="e4m3",
                                          K=512, H=64, T=1024),
}


def small_workload(base: str, **over) -> Workload:
    """A reduced copy of a named workload (same structure, smaller sizes)."""
    w = WORKLOADS[base]
    d = dict(w.__dict__)
    d.update(over)
    d["name"] = base + "_small"
    return Workload(**d)


def _gen(seed0, tensor_no, seq, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed0) + 1000 * int(tensor_no) + int(seq))
    return g


def _randn(shape, seed0, tensor_no, seq, device):
    return torch.randn(shape, generator=_gen(seed0, tensor_no, seq, device), device=device,
                       dtype=torch.float32)


def _rand(shape, seed0, tensor_no, seq, device):
    return torch.rand(shape, generator=_gen(seed0, tensor_no, seq, device), device=device,
                      dtype=torch.float32)


def _cast(x, dt):
    return x.to(torch.bfloat16) if dt == "bf16" else x.to(torch.float8_e4m3fn)


def _fill_per_seq(out, B, fn):
    for b in range(B):
        out[b].copy_(fn(b))
    return out


def main_kv_source(w: Workload, seed0: int, device, n_entries=None):
    """bf16 [B, n_entries, 512] latent rows; N(0,1), times a per-channel LogNormal(0,1)
    scale fixed per sequence when the workload asks for it."""
    n = w.cap if n_entries is None else n_entries
    out = torch.empty((w.B, n, D_MAIN), dtype=torch.bfloat16, device=device)

    def one(b):
        x = _randn((n, D_MAIN), seed0, 1, b, device)
        if w.lognormal_channels:
            s = torch.exp(_randn((D_MAIN,), seed0, 2, b, device))
            x = x * s
        return x.to(torch.bfloat16)
    return _fill_per_seq(out, w.B, one)


def layer_inputs(w: Workload, layer: int, seed0: int, device):
    """Per-layer query-side inputs: indexer query + weights, main query, window KV."""
    base = 10 + 10 * layer
    T = w.T
    tdt = torch.bfloat16 if w.idx_dtype == "bf16" else torch.float8_e4m3fn
    q_I = torch.empty((w.B, T, w.H_I, D_IDX), dtype=tdt, device=device)
    _fill_per_seq(q_I, w.B, lambda b: _cast(_randn((T, w.H_I, D_IDX), seed0, base + 0, b,
                                                   device), w.idx_dtype))
    wts = torch.empty((w.B, T, w.H_I), dtype=torch.float32, device=device)
    _fill_per_seq(wts, w.B, lambda b: _rand((T, w.H_I), seed0, base + 1, b, device))
    if w.kind == "decode":
        q = torch.empty((w.B, w.H, D_MAIN), dtype=torch.bfloat16, device=device)
        _fill_per_seq(q, w.B, lambda b: _randn((w.H, D_MAIN), seed0, base + 2, b,
                                               device).to(torch.bfloat16))
        swa_rows = WINDOW
    else:
        q = torch.empty((w.B, T, w.H, D_MAIN), dtype=torch.bfloat16, device=device)
        _fill_per_seq(q, w.B, lambda b: _randn((T, w.H, D_MAIN), seed0, base + 2, b,
                                               device).to(torch.bfloat16))
        swa_rows = WINDOW - 1 + T
    swa = torch.empty((w.B, swa_rows, D_MAIN), dtype=torch.float8_e4m3fn, device=device)
    _fill_per_seq(swa, w.B, lambda b: _randn((swa_rows, D_MAIN), seed0, base + 3, b,
                                             device).to(torch.float8_e4m3fn))
    return {"q_I": q_I, "w": wts, "q": q, "swa": swa}


def indexer_keys(w: Workload, seed0: int, device, planted_dirs=None):
    """Indexer keys [B, cap, 128]; with planted keys, `planted` positions per sequence
    (each in its own 8-entry block) are overwritten by alpha * the given unit direction
    of that sequence (planted_dirs: float32 [B, 128]). Returns (keys, planted positions
    int64 [B, planted] or None). With compact keys (key_format "fp4") the keys are returned
    as bf16, for the library's key quantiser."""
    kdt = "bf16" if w.key_format == "fp4" else w.idx_dtype
    tdt = torch.bfloat16 if kdt == "bf16" else torch.float8_e4m3fn
    k = torch.empty((w.B, w.cap, D_IDX), dtype=tdt, device=device)
    _fill_per_seq(k, w.B, lambda b: _cast(_randn((w.cap, D_IDX), seed0, 3, b, device), kdt))
    pos = None
    if w.planted:
        alpha = float(w.extra.get("planted_alpha", 24.0))
        nblk = w.N // POOL_BLOCK
        pos = torch.empty((w.B, w.planted), dtype=torch.int64)
        for b in range(w.B):
            g = _gen(seed0, 4, b, "cpu")
            blocks = torch.randperm(nblk, generator=g)[: w.planted]
            off = torch.randint(0, POOL_BLOCK, (w.planted,), generator=g)
            p = torch.sort(blocks * POOL_BLOCK + off).values
            pos[b] = p
            vec = (alpha * planted_dirs[b].float()).to(device)
            k[b, p.to(device)] = _cast(vec.expand(w.planted, D_IDX).contiguous(), kdt)
    return k, pos


def planted_direction(q_I_list):
    """Unit direction aligned with every listed layer's indexer queries of a sequence:
    the normalised sum of each layer's normalised head-sum. q_I_list: tensors
    [B, T, H_I, 128]. Returns float32 [B, 128] (input construction only)."""
    acc = None
    for q in q_I_list:
        s = q.float().sum(dim=(1, 2))
        s = s / s.norm(dim=-1, keepdim=True)
        acc = s if acc is None else acc + s
    return acc / acc.norm(dim=-1, keepdim=True)


def decode_positions(w: Workload, device):
    """n_vis0 [B] int32: visible compressed entries per sequence at decode."""
    return torch.full((w.B,), w.N, dtype=torch.int32, device=device)


def prefill_positions(w: Workload, device):
    """q_pos0 [B] int32: absolute position of the first new token of each sequence."""
    return torch.full((w.B,), w.ctx, dtype=torch.int32, device=device)
