"""Seeded synthetic inputs for the paged MQA-logits path.

This module only draws and encodes inputs. It holds none of the logits
arithmetic, so both the CPU oracle and the CUDA path can take their inputs
from it without sharing any of the method.

Workloads (indexer-shaped, as named by the five benchmark configurations):

  tiny     B=3,    next_n=1, H=4,  D=32,  page 16, ctx {37, 0, 70}, L=72
  decode   B=64,   next_n=1, H=64, D=128, page 64, ctx U[1024, 8192], L=8192
  stress   B=2048, next_n=1, H=64, D=128, page 64, ctx: 80% U[0, 4096],
           10% exactly 0, 10% 256*m +- 1 (m in U{1..16}) clamped to [0, 4096]; L=4096
  mtp      B=32,   next_n=2, H=64, D=128, page 64, ctx U[32768, 131072], L=131072
  fp4      B=128,  next_n=1, H=32, D=128, page 64, ctx U[512, 16384], L=16384
  nvfp4    the fp4 shapes with q in NVFP4 as well (block-scaled FP4 MMA)

Value recipe (FP8): q and k drawn from N(0, 1), clipped to +-448, rounded to
e4m3 (round-to-nearest-even, done by torch's float8_e4m3fn cast); the per-token
K scale from U[0.5, 2] (fp32); weights from N(0, 1/H) (fp32).

Value recipe (FP4): q drawn from N(0, 1) and rounded to bf16. Each K token is
drawn from N(0, 1) and quantised per 16-element block: the block scale is
e4m3_RNE(amax / 6) (the smallest positive e4m3, 2^-9, if that rounds to 0);
each element is x / scale rounded to the nearest e2m1 value (ties to even,
saturating at +-6). Two e2m1 codes share a byte, the even element in the low
nibble.

Value recipe (NVFP4 q, the block-scaled FP4 variant): as FP4, but q is
drawn from N(0, 1) and quantised like the K tokens (e4m3 scale per 16
elements, e2m1 codes). One (b, n) row of q is laid out like a page of H
tokens: [H][D/2] packed e2m1 codes, then [H][D/16] e4m3 block scales.

Paging: every row's pages are taken from one pool of
num_pages = sum_b ceil(ctx_b / page_size) pages and the pool is shuffled, so
the block table is a random permutation. Unused block-table slots hold -1.

KV page layout (one page, page_size tokens):
  FP8: [page_size][D] e4m3 K rows, then [page_size] fp32 scales.
  FP4: [page_size][D/2] packed e2m1 K rows, then [page_size][D/16] e4m3
       block scales.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

__all__ = [
    "Workload", "CONFIGS", "make_workload", "make_config", "draw_context_lens",
    "quantize_e2m1_rne", "encode_nvfp4", "fp8_page_bytes", "fp4_page_bytes",
    "nvfp4_q_row_bytes", "repage",
]


def fp8_page_bytes(page_size: int, head_dim: int) -> int:
    return page_size * (head_dim + 4)


def fp4_page_bytes(page_size: int, head_dim: int) -> int:
    return page_size * (head_dim // 2 + head_dim // 16)


def nvfp4_q_row_bytes(num_heads: int, head_dim: int) -> int:
    """Bytes of one (b, n) row of an NVFP4 q: codes, then block scales."""
    return num_heads * (head_dim // 2 + head_dim // 16)


@dataclasses.dataclass
class Workload:
    """One batch of indexer inputs, all CPU tensors.

    q           uint8 [B, next_n, H, D] (e4m3 bits) for fp8,
                int16 [B, next_n, H, D] (bf16 bits) for fp4,
                uint8 [B, next_n, H*(D/2 + D/16)] (codes, then scales) for nvfp4
    kv_cache    uint8 [num_pages, page_bytes]
    block_table int32 [B, max_pages_per_row], -1 where unused
    context_lens int32 [B]
    weights     float32 [B, next_n, H]
    """
    kind: str  # "fp8", "fp4" or "nvfp4"
    B: int
    next_n: int
    H: int
    D: int
    page_size: int
    out_len: int
    q: torch.Tensor
    kv_cache: torch.Tensor
    block_table: torch.Tensor
    context_lens: torch.Tensor
    weights: torch.Tensor
    name: str = ""

    @property
    def num_pages(self) -> int:
        return int(self.kv_cache.shape[0])

    @property
    def max_pages_per_row(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def page_bytes(self) -> int:
        return int(self.kv_cache.shape[1])

    def draft_context_lens(self) -> torch.Tensor:
        """ctx_{b,n} = clamp(ctx_b - next_n + 1 + n, 0, ctx_b), int64 [B, next_n]."""
        c = self.context_lens.to(torch.int64)[:, None]
        n = torch.arange(self.next_n, dtype=torch.int64)[None, :]
        return torch.minimum(torch.clamp(c - self.next_n + 1 + n, min=0), c)

    def tokens(self) -> int:
        """K-cache tokens scored: sum_b ctx_b."""
        return int(self.context_lens.to(torch.int64).sum())

    def algorithmic_bytes(self) -> int:
        """HBM bytes the path must move at least once: K (+ scales) of valid
        tokens, the full fp32 output, q, weights and used block-table slots."""
        ctx = self.context_lens.to(torch.int64)
        ntok = int(ctx.sum())
        if self.kind == "fp8":
            kbytes = ntok * (self.D + 4)
            qbytes = self.B * self.next_n * self.H * self.D
        elif self.kind == "fp4":
            kbytes = ntok * (self.D // 2 + self.D // 16)
            qbytes = self.B * self.next_n * self.H * self.D * 2
        else:
            kbytes = ntok * (self.D // 2 + self.D // 16)
            qbytes = self.B * self.next_n * nvfp4_q_row_bytes(self.H, self.D)
        pages_used = int(((ctx + self.page_size - 1) // self.page_size).sum())
        return (kbytes + 4 * self.B * self.next_n * self.out_len + qbytes
                + 4 * self.B * self.next_n * self.H + 4 * pages_used + 4 * self.B)

    def flops(self) -> int:
        return 2 * self.H * self.D * self.next_n * self.tokens()


CONFIGS = {
    "tiny": dict(kind="fp8", B=3, next_n=1, H=4, D=32, page_size=16, out_len=72),
    "decode": dict(kind="fp8", B=64, next_n=1, H=64, D=128, page_size=64, out_len=8192),
    "stress": dict(kind="fp8", B=2048, next_n=1, H=64, D=128, page_size=64, out_len=4096),
    "mtp": dict(kind="fp8", B=32, next_n=2, H=64, D=128, page_size=64, out_len=131072),
    "fp4": dict(kind="fp4", B=128, next_n=1, H=32, D=128, page_size=64, out_len=16384),
    # the FP4 workload with q supplied in NVFP4 too (the block-scaled MMA)
    "nvfp4": dict(kind="nvfp4", B=128, next_n=1, H=32, D=128, page_size=64, out_len=16384),
}
CONFIG_ORDER = ["tiny", "decode", "stress", "mtp", "fp4", "nvfp4"]


def draw_context_lens(name: str, B: int, gen: torch.Generator) -> torch.Tensor:
    """The per-configuration context-length distribution, int32 [B]."""
    def uni(lo, hi, n):
        return torch.randint(lo, hi + 1, (n,), generator=gen, dtype=torch.int64)
    if name == "tiny":
        c = torch.tensor([37, 0, 70], dtype=torch.int64)
    elif name == "decode":
        c = uni(1024, 8192, B)
    elif name == "stress":
        c = uni(0, 4096, B)
        perm = torch.randperm(B, generator=gen)
        n10 = B // 10
        c[perm[:n10]] = 0
        m = uni(1, 16, n10)
        pm = torch.where(torch.rand(n10, generator=gen) < 0.5, -1, 1)
        c[perm[n10:2 * n10]] = torch.clamp(256 * m + pm, 0, 4096)
    elif name == "mtp":
        c = uni(32768, 131072, B)
    elif name in ("fp4", "nvfp4"):
        c = uni(512, 16384, B)
    else:
        raise KeyError(name)
    return c.to(torch.int32)


# Midpoints between neighbouring e2m1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
_E2M1_MIDS = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=torch.float32)


def quantize_e2m1_rne(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 x to the nearest e2m1 value, ties to the even code, saturating
    at +-6. Returns the 4-bit codes (sign in bit 3) as uint8."""
    a = x.abs().to(torch.float32)
    idx = torch.bucketize(a, _E2M1_MIDS)          # a == mid goes to the lower code
    tie = (idx < 7) & (a == _E2M1_MIDS[idx.clamp(max=6)])
    idx = torch.where(tie & (idx % 2 == 1), idx + 1, idx)  # odd lower code: tie goes up
    mag = idx.to(torch.uint8)
    sign = ((x < 0) & (mag != 0)).to(torch.uint8) << 3
    return mag | sign


def encode_nvfp4(x: torch.Tensor):
    """x: fp32 [..., D/16, 16] -> (packed e2m1 codes uint8 [..., D/2], e4m3
    block scales uint8 [..., D/16]): scale = e4m3_RNE(amax / 6) (2^-9 if that
    rounds to 0), codes = e2m1_RNE(x / scale), even element in the low nibble."""
    amax = x.abs().amax(dim=-1, keepdim=True)
    sc = (amax / 6.0).to(torch.float8_e4m3fn).to(torch.float32)
    sc = torch.where(sc == 0, torch.full_like(sc, 2.0 ** -9), sc)
    codes = quantize_e2m1_rne(x / sc).reshape(*x.shape[:-2], -1)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).to(torch.uint8)
    sc8 = sc.squeeze(-1).to(torch.float8_e4m3fn).view(torch.uint8)
    return packed, sc8


def _layout_pages(ctx: torch.Tensor, page_size: int, max_pages: int,
                  gen: torch.Generator):
    """Random-permutation block table over a shared page pool."""
    B = ctx.numel()
    npg = (ctx.to(torch.int64) + page_size - 1) // page_size
    total = int(npg.sum())
    pool = torch.randperm(max(total, 1), generator=gen)[:total].to(torch.int32)
    bt = torch.full((B, max(max_pages, 1)), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        n = int(npg[b])
        bt[b, :n] = pool[off:off + n]
        off += n
    return bt, max(total, 1)


def make_workload(kind: str, B: int, next_n: int, H: int, D: int, page_size: int,
                  out_len: int, context_lens, seed: int, name: str = "",
                  max_pages_per_row: Optional[int] = None,
                  weights_nonneg: bool = False, reserve_lens=None) -> Workload:
    """Build one workload with the value recipe above from explicit shapes.
    reserve_lens (optional, per row) allocates pages for at least that many
    tokens, so context_lens can later grow up to it."""
    gen = torch.Generator().manual_seed(seed)
    ctx = torch.as_tensor(context_lens, dtype=torch.int32).clone()
    assert ctx.numel() == B
    alloc = ctx if reserve_lens is None else torch.maximum(
        ctx, torch.as_tensor(reserve_lens, dtype=torch.int32))
    if max_pages_per_row is None:
        max_pages_per_row = (max(int(alloc.max()) if B else 0, out_len) + page_size - 1) // page_size
    bt, num_pages = _layout_pages(alloc, page_size, max_pages_per_row, gen)
    w = torch.randn(B, next_n, H, generator=gen, dtype=torch.float32) / float(np.sqrt(H))
    if weights_nonneg:
        w = w.abs()
    CH = 2048  # pages drawn per chunk, to bound host memory
    if kind == "fp8":
        q = torch.randn(B, next_n, H, D, generator=gen).clamp(-448, 448)
        q = q.to(torch.float8_e4m3fn).view(torch.uint8)
        kv = torch.empty(num_pages, fp8_page_bytes(page_size, D), dtype=torch.uint8)
        for p0 in range(0, num_pages, CH):
            p1 = min(num_pages, p0 + CH)
            k = torch.randn(p1 - p0, page_size, D, generator=gen).clamp(-448, 448)
            kv[p0:p1, :page_size * D] = k.to(torch.float8_e4m3fn).view(torch.uint8).reshape(p1 - p0, -1)
        for p0 in range(0, num_pages, CH):
            p1 = min(num_pages, p0 + CH)
            s = torch.rand(p1 - p0, page_size, generator=gen, dtype=torch.float32) * 1.5 + 0.5
            kv[p0:p1, page_size * D:] = s.view(torch.uint8).reshape(p1 - p0, -1)
    elif kind in ("fp4", "nvfp4"):
        assert D % 16 == 0
        if kind == "fp4":
            q = torch.randn(B, next_n, H, D, generator=gen).to(torch.bfloat16).view(torch.int16)
        else:
            xq = torch.randn(B, next_n, H, D // 16, 16, generator=gen, dtype=torch.float32)
            qc, qs = encode_nvfp4(xq)
            q = torch.cat([qc.reshape(B, next_n, -1), qs.reshape(B, next_n, -1)], dim=-1)
        kv = torch.empty(num_pages, fp4_page_bytes(page_size, D), dtype=torch.uint8)
        for p0 in range(0, num_pages, CH):
            p1 = min(num_pages, p0 + CH)
            n = p1 - p0
            x = torch.randn(n, page_size, D // 16, 16, generator=gen, dtype=torch.float32)
            packed, sc8 = encode_nvfp4(x)
            kv[p0:p1, :page_size * D // 2] = packed.reshape(n, -1)
            kv[p0:p1, page_size * D // 2:] = sc8.reshape(n, -1)
    else:
        raise ValueError(kind)
    return Workload(kind=kind, B=B, next_n=next_n, H=H, D=D, page_size=page_size,
                    out_len=out_len, q=q.contiguous(), kv_cache=kv.contiguous(),
                    block_table=bt, context_lens=ctx, weights=w.contiguous(), name=name)


def make_config(name: str, seed: Optional[int] = None) -> Workload:
    """One of the five named workloads; seed defaults to 1234 + its index."""
    cfg = CONFIGS[name]
    if seed is None:
        seed = 1234 + CONFIG_ORDER.index(name)
    gen = torch.Generator().manual_seed(seed + 7919)
    ctx = draw_context_lens(name, cfg["B"], gen)
    return make_workload(context_lens=ctx, seed=seed, name=name, **cfg)


def repage(wl: Workload, page_size: int, seed: int) -> Workload:
    """The same logical K (token by token) stored with another page size and a
    fresh random block table. Only copies bytes."""
    B, ps0 = wl.B, wl.page_size
    D = wl.D
    if wl.kind == "fp8":
        row_k, row_s = D, 4
    else:  # fp4 and nvfp4 pages
        row_k, row_s = D // 2, D // 16
    ctx = wl.context_lens.to(torch.int64)
    gen = torch.Generator().manual_seed(seed)
    maxp = (max(int(ctx.max()) if B else 0, wl.out_len) + page_size - 1) // page_size
    bt, num_pages = _layout_pages(wl.context_lens, page_size, maxp, gen)
    kk = torch.zeros(num_pages, page_size, row_k, dtype=torch.uint8)
    ss = torch.zeros(num_pages, page_size, row_s, dtype=torch.uint8)
    src_k = wl.kv_cache[:, :ps0 * row_k].reshape(-1, ps0, row_k)
    src_s = wl.kv_cache[:, ps0 * row_k:].reshape(-1, ps0, row_s)
    for b in range(B):
        n = int(ctx[b])
        if n == 0:
            continue
        t = torch.arange(n)
        sp = wl.block_table[b].to(torch.int64)[t // ps0]
        dp = bt[b].to(torch.int64)[t // page_size]
        kk[dp, t % page_size] = src_k[sp, t % ps0]
        ss[dp, t % page_size] = src_s[sp, t % ps0]
    kv = torch.cat([kk.reshape(num_pages, -1), ss.reshape(num_pages, -1)], dim=1)
    return dataclasses.replace(wl, page_size=page_size, kv_cache=kv.contiguous(), block_table=bt)
