"""Seeded synthetic inputs for GQLA decode (shared by the tests, the bench and
the oracle checks; holds none of the method's arithmetic).

Recipe (every workload): q (nope and rope parts), the joint latent c_KV and
the decoupled RoPE key are i.i.d. N(0, 1); W_uk and W_uv are i.i.d. N(0, 1/r)
(standard deviation r**-0.5).  Values are drawn in fp32 with a seeded
``torch.Generator`` on the target device and, for bf16 workloads, rounded to
bf16 (round-to-nearest-even); the rounded tensors are the inputs of both the
CUDA path and the oracle.  Draw order: sequence lengths (ragged only), page
permutation (paged only), q, latent pool, W_uk, W_uv.

Layouts (row-major):
  q        [B, s_q, n_h, d_nope + d_rope]   nope part first
  latent   contiguous [B, capacity, r + d_rope]  or  paged [P, page, r + d_rope]
           each token row is [c_KV (r) ; k_rope (d_rope)]
  W_uk     [G, r, d_nope]      W_uv [G, r, d_v]
  block_table [B, max_blocks_per_seq] int32 physical page ids, -1 past the end
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Dims:
    n_h: int
    G: int
    d_nope: int
    d_rope: int
    d_v: int
    r: int
    s_q: int = 1
    dtype: str = "bf16"            # "f32" or "bf16"
    scale: Optional[float] = None  # default 1/sqrt(d_nope + d_rope)
    k_shared_rope: bool = False    # expanded K rows hold the RoPE key once, not per group

    @property
    def m(self) -> int:
        return self.n_h // self.G

    @property
    def d_qk(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def latent_width(self) -> int:
        return self.r + self.d_rope

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d_qk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclass
class Workload:
    name: str
    dims: Dims
    batch: int
    seq_len: Optional[int] = None          # uniform length
    ragged: Optional[tuple] = None         # (lo, hi) inclusive, uniform integers
    page_size: int = 0                     # 0 = contiguous
    seed: int = 0
    notes: str = ""


# The five workloads: tiny fp32, LLaMA-3-8B-shaped, DeepSeek-V3-shaped,
# ragged paged batch, path-crossover sweep (one point per (G, s_q, L)).
def tiny_f32() -> Workload:
    return Workload("tiny_f32", Dims(n_h=8, G=2, d_nope=32, d_rope=16, d_v=32, r=64, s_q=1,
                                     dtype="f32", scale=1.0 / math.sqrt(48.0)),
                    batch=2, seq_len=128, seed=0)


def llama3_8b(s_q: int = 1, batch: int = 32, seq_len: int = 8192) -> Workload:
    return Workload("llama3_8b_gqla", Dims(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512,
                                           s_q=s_q, dtype="bf16"),
                    batch=batch, seq_len=seq_len, seed=0)


def dsv3(seq_len: int = 8192, s_q: int = 1, batch: int = 64, G: int = 16) -> Workload:
    return Workload("dsv3_gqla", Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512,
                                      s_q=s_q, dtype="bf16"),
                    batch=batch, seq_len=seq_len, seed=0)


def ragged_paged(batch: int = 128, lo: int = 1024, hi: int = 65536, page_size: int = 64) -> Workload:
    return Workload("ragged_paged_dsv3", Dims(n_h=128, G=16, d_nope=128, d_rope=64, d_v=128,
                                              r=512, s_q=1, dtype="bf16"),
                    batch=batch, ragged=(lo, hi), page_size=page_size, seed=0)


def crossover(G: int, s_q: int, batch: int = 32, seq_len: int = 32768) -> Workload:
    return Workload("crossover", Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512,
                                      s_q=s_q, dtype="bf16"),
                    batch=batch, seq_len=seq_len, seed=0)


@dataclass
class Inputs:
    wl: Workload
    q: torch.Tensor
    latent: torch.Tensor               # contiguous [B, cap, E] or paged [P, page, E]
    W_uk: torch.Tensor
    W_uv: torch.Tensor
    seq_lens: torch.Tensor             # int32 [B] (same device)
    seq_lens_host: list
    block_table: Optional[torch.Tensor]  # int32 [B, max_blocks] or None
    capacity: int                      # contiguous: slots per sequence
    max_blocks_per_seq: int = 0
    num_pages: int = 0

    @property
    def dims(self) -> Dims:
        return self.wl.dims

    @property
    def max_seq_len(self) -> int:
        return max(self.seq_lens_host)

    def logical_latent(self, b: int) -> torch.Tensor:
        """Sequence b's token rows [L_b, E] in logical order (gathered through
        the block table for a paged pool)."""
        L = self.seq_lens_host[b]
        if self.block_table is None:
            return self.latent[b, :L]
        ps = self.wl.page_size
        nb = (L + ps - 1) // ps
        pages = self.block_table[b, :nb].long()
        return self.latent[pages].reshape(nb * ps, -1)[:L]


def make_inputs(wl: Workload, device="cpu", seq_lens=None) -> Inputs:
    d = wl.dims
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    B = wl.batch
    if seq_lens is not None:
        lens = [int(x) for x in seq_lens]
    elif wl.ragged is not None:
        lo, hi = wl.ragged
        lens = torch.randint(lo, hi + 1, (B,), generator=gen, device=dev).tolist()
    else:
        lens = [wl.seq_len] * B
    E = d.latent_width
    tdt = d.torch_dtype
    block_table = None
    mbps = 0
    n_pages = 0
    if wl.page_size > 0:
        ps = wl.page_size
        nblk = [(L + ps - 1) // ps for L in lens]
        n_pages = sum(nblk)
        mbps = max(nblk)
        perm = torch.randperm(n_pages, generator=gen, device=dev).to(torch.int32)
        block_table = torch.full((B, mbps), -1, dtype=torch.int32, device=dev)
        o = 0
        for b in range(B):
            block_table[b, :nblk[b]] = perm[o:o + nblk[b]]
            o += nblk[b]
        capacity = mbps * ps
    else:
        capacity = max(lens)
    q = torch.randn((B, d.s_q, d.n_h, d.d_qk), generator=gen, device=dev, dtype=torch.float32).to(tdt)
    if wl.page_size > 0:
        latent = _randn_chunked((n_pages, wl.page_size, E), gen, dev, tdt)
    else:
        latent = _randn_chunked((B, capacity, E), gen, dev, tdt)
    s = d.r ** -0.5
    W_uk = (torch.randn((d.G, d.r, d.d_nope), generator=gen, device=dev) * s).to(tdt)
    W_uv = (torch.randn((d.G, d.r, d.d_v), generator=gen, device=dev) * s).to(tdt)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    return Inputs(wl, q, latent, W_uk, W_uv, sl, lens, block_table, capacity, mbps, n_pages)


def _randn_chunked(shape, gen, dev, tdt, chunk_elems=1 << 28):
    """randn in fp32 then cast, a chunk of the leading axis at a time, so a
    multi-GB bf16 pool never needs a same-size fp32 temporary."""
    out = torch.empty(shape, dtype=tdt, device=dev)
    per = max(1, chunk_elems // max(1, math.prod(shape[1:])))
    for s0 in range(0, shape[0], per):
        s1 = min(shape[0], s0 + per)
        out[s0:s1] = torch.randn((s1 - s0,) + tuple(shape[1:]), generator=gen, device=dev,
                                 dtype=torch.float32).to(tdt)
    return out


def expanded_pool_shapes(inp: Inputs):
    """Shapes of the per-group expanded K and V pools with the latent pool's
    geometry: token rows [G, d_nope + d_rope] (or [G * d_nope + d_rope] when
    the RoPE key is stored once) and [G, d_v]."""
    d = inp.dims
    lead = tuple(inp.latent.shape[:2])
    k = (d.G * d.d_nope + d.d_rope,) if d.k_shared_rope else (d.G, d.d_qk)
    return lead + k, lead + (d.G, d.d_v)
