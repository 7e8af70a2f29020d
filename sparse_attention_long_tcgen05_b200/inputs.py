"""Seeded synthetic workloads for the DSA forward path.

This module draws random tensors with the shapes, dtypes and value
distributions of the five DSA workloads and nothing else: it holds no step of
the method. FP8 inputs are stored the way the indexer consumes them, as e4m3
codes plus one positive fp32 scale per token; the cast itself is torch's own
``float8_e4m3fn`` conversion (round to nearest even) after a clamp to the
format's finite range, so the GPU path and the oracle read identical bytes.

Workloads (sizes from the five configurations of the benchmark):

  0  tiny_f32_L256        fp32 everything, H_I=4, d_I=32, 8 heads, d=64, k=64
  1  prefill_L4096        FP8 indexer (64x128), bf16 576/512 MQA, 128 heads
  2  prefill_L32768_needle as 1, L=32768, 64 "needle" keys per 4096-block x3
  3  prefill_L131072      as 1, L=131072
  4  decode_B64           64 sequences, ctx ~ U[8192, 131072], 64-token pages,
                          shuffled block table, one query token each

Draw order (one torch.Generator per workload, seed 0 unless given):
prefill: q_I, k_I, w, q, kv, then needle positions (workload 2 only);
decode: ctx_lens, block-table permutation, q_I, k-cache, w, q, kv-cache.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

E4M3_MAX = 448.0
PAGE = 64


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    dtype: str           # "f32" (tiny) or "fp8_bf16"
    L: int = 0           # prefill sequence length
    B: int = 0           # decode batch
    ctx_min: int = 0
    ctx_max: int = 0
    H_I: int = 64
    d_I: int = 128
    H: int = 128
    D_K: int = 576
    D_V: int = 512
    k: int = 2048
    needles_per_block: int = 0
    needle_block: int = 4096
    needle_gain: float = 3.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D_K)


WORKLOADS = {
    0: Workload("tiny_f32_L256", "prefill", "f32", L=256, H_I=4, d_I=32, H=8,
                D_K=64, D_V=64, k=64),
    1: Workload("prefill_L4096", "prefill", "fp8_bf16", L=4096),
    2: Workload("prefill_L32768_needle", "prefill", "fp8_bf16", L=32768,
                needles_per_block=64),
    3: Workload("prefill_L131072", "prefill", "fp8_bf16", L=131072),
    4: Workload("decode_B64", "decode", "fp8_bf16", B=64, ctx_min=8192,
                ctx_max=131072),
}


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token FP8 storage of ``x`` ([T, ...] float32).

    scale[t] = amax(|x[t]|) / 448; codes = e4m3(x[t] / scale[t]) as uint8.
    """
    T = x.shape[0]
    flat = x.reshape(T, -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.float().contiguous()


@dataclass
class PrefillInputs:
    wl: Workload
    # indexer
    q_idx: torch.Tensor          # [L, H_I, d_I] uint8 codes (fp8) or float32 (tiny)
    q_scale: Optional[torch.Tensor]   # [L] float32 (fp8 only)
    k_idx: torch.Tensor          # [L, d_I] uint8 codes or float32
    k_scale: Optional[torch.Tensor]   # [L] float32
    w: torch.Tensor              # [L, H_I] float32
    # attention
    q: torch.Tensor              # [L, H, D_K] bf16 (or float32 tiny)
    kv: torch.Tensor             # [L, D_K] bf16 (or float32 tiny: K only)
    v: Optional[torch.Tensor]    # tiny only: [L, D_V] float32
    needles: Optional[torch.Tensor] = None  # [n] int64 positions scaled x3


@dataclass
class DecodeInputs:
    wl: Workload
    ctx_lens: torch.Tensor       # [B] int32
    block_table: torch.Tensor    # [B, max_pages] int32 (-1 past the sequence)
    num_pages: int
    q_idx: torch.Tensor          # [B, H_I, d_I] uint8
    q_scale: torch.Tensor        # [B] float32
    k_cache: torch.Tensor        # [num_pages, 64, d_I] uint8
    k_cache_scale: torch.Tensor  # [num_pages, 64] float32
    w: torch.Tensor              # [B, H_I] float32
    q: torch.Tensor              # [B, H, D_K] bf16
    kv_cache: torch.Tensor       # [num_pages, 64, D_K] bf16


def _randn(shape, gen, device, dtype=torch.float32, chunk_rows=8192):
    """torch.randn drawn row-chunk by row-chunk (bounded temporaries)."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n = shape[0]
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 device=device, dtype=torch.float32).to(dtype)
    return out


def make_prefill(wl: Workload, device="cpu", seed: int = 0) -> PrefillInputs:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    L = wl.L
    if wl.dtype == "f32":
        q_idx = torch.randn(L, wl.H_I, wl.d_I, generator=gen, device=device)
        k_idx = torch.randn(L, wl.d_I, generator=gen, device=device)
        w = torch.rand(L, wl.H_I, generator=gen, device=device)
        q = torch.randn(L, wl.H, wl.D_K, generator=gen, device=device)
        k = torch.randn(L, wl.D_K, generator=gen, device=device)
        v = torch.randn(L, wl.D_V, generator=gen, device=device)
        return PrefillInputs(wl, q_idx, None, k_idx, None, w, q, k, v)

    q_idx_f = _randn((L, wl.H_I, wl.d_I), gen, device)
    k_idx_f = _randn((L, wl.d_I), gen, device)
    w = torch.randn(L, wl.H_I, generator=gen, device=device) / 8.0
    q = _randn((L, wl.H, wl.D_K), gen, device, dtype=torch.bfloat16, chunk_rows=2048)
    kv = _randn((L, wl.D_K), gen, device, dtype=torch.bfloat16)
    needles = None
    if wl.needles_per_block:
        pos = []
        for b0 in range(0, L, wl.needle_block):
            perm = torch.randperm(wl.needle_block, generator=gen, device=device)
            pos.append(perm[: wl.needles_per_block] + b0)
        needles = torch.cat(pos).sort().values
        k_idx_f[needles] *= wl.needle_gain
    q_codes, q_scale = quantize_e4m3_per_token(q_idx_f)
    del q_idx_f
    k_codes, k_scale = quantize_e4m3_per_token(k_idx_f)
    return PrefillInputs(wl, q_codes, q_scale, k_codes, k_scale, w.contiguous(),
                         q, kv, None, needles)


def make_decode(wl: Workload, device="cpu", seed: int = 0, ctx_lens=None) -> DecodeInputs:
    """ctx_lens (optional list) replaces the drawn context lengths."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B = wl.B
    ctx = torch.randint(wl.ctx_min, wl.ctx_max + 1, (B,), generator=gen, device=device)
    if ctx_lens is not None:
        ctx = torch.tensor(ctx_lens, dtype=torch.int64, device=device)
        B = len(ctx_lens)
    n_pages = (ctx + PAGE - 1) // PAGE
    num_pages = int(n_pages.sum().item())
    max_pages = (wl.ctx_max + PAGE - 1) // PAGE
    perm = torch.randperm(num_pages, generator=gen, device=device).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b in range(B):
        n = int(n_pages[b].item())
        table[b, :n] = perm[off:off + n]
        off += n
    q_idx_f = torch.randn(B, wl.H_I, wl.d_I, generator=gen, device=device)
    k_cache_f = _randn((num_pages * PAGE, wl.d_I), gen, device)
    w = torch.randn(B, wl.H_I, generator=gen, device=device) / 8.0
    q = torch.randn(B, wl.H, wl.D_K, generator=gen, device=device).to(torch.bfloat16)
    kv_cache = _randn((num_pages * PAGE, wl.D_K), gen, device, dtype=torch.bfloat16)
    q_codes, q_scale = quantize_e4m3_per_token(q_idx_f)
    k_codes, k_scale = quantize_e4m3_per_token(k_cache_f)
    del k_cache_f
    return DecodeInputs(
        wl, ctx.to(torch.int32).contiguous(), table.contiguous(), num_pages,
        q_codes, q_scale, k_codes.view(num_pages, PAGE, wl.d_I),
        k_scale.view(num_pages, PAGE), w.contiguous(), q.contiguous(),
        kv_cache.view(num_pages, PAGE, wl.D_K))


def make_grad_out(n_q: int, H: int = 128, d_v: int = 512, device="cpu", seed: int = 0):
    """Seeded upstream gradient dO [n_q, H, d_v] for the attention backward:
    bf16 draws of N(0, 1), row-chunked like the other bf16 tensors."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return _randn((n_q, H, d_v), gen, device, dtype=torch.bfloat16, chunk_rows=2048)


def random_selection(n_q: int, n_keys: int, k: int, device="cpu", seed: int = 0,
                     chunk_rows: int = 8192) -> torch.Tensor:
    """Seeded valid selection in the top-k's output format, for testing the
    attention alone: query i (position p = n_keys - n_q + i) keeps every key
    0..p when p < k, else one key drawn uniformly from each of k consecutive
    strata [floor(j w), floor((j+1) w)) of 0..p, w = (p+1)/k -- k distinct keys,
    ascending, spread over the whole prefix. Padded with -1 to k columns."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    idx = torch.empty(n_q, k, dtype=torch.int32, device=device)
    j = torch.arange(k, device=device, dtype=torch.float64)
    for r0 in range(0, n_q, chunk_rows):
        r1 = min(n_q, r0 + chunk_rows)
        pos = torch.arange(n_keys - n_q + r0, n_keys - n_q + r1, device=device,
                           dtype=torch.float64)[:, None]
        w = (pos + 1.0) / k
        lo = torch.floor(j * w)
        hi = torch.floor((j + 1.0) * w)
        u = torch.rand((r1 - r0, k), generator=gen, device=device, dtype=torch.float64)
        sparse = lo + torch.floor(u * (hi - lo))
        dense = torch.where(j <= pos, j, torch.full_like(j, -1.0))
        idx[r0:r1] = torch.where(pos + 1.0 > k, sparse, dense).to(torch.int32)
    return idx


def sample_rows(L: int, n: int = 512, seed: int = 1, k: int = 2048):
    """Seeded row sample for large prefill checks: {0, k-1, k, L-1} plus
    uniform draws, sorted and unique."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    fixed = [0, k - 1, k, L - 1]
    fixed = [r for r in fixed if 0 <= r < L]
    extra = torch.randint(0, L, (4 * n,), generator=g).tolist()
    rows = list(dict.fromkeys(fixed))
    for r in extra:
        if len(rows) >= min(n, L):
            break
        if r not in rows:
            rows.append(r)
    return sorted(rows)
