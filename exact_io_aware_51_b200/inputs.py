"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and casts them; it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed from
it without sharing any of the method.

Recipe (the same for every workload): a CPU ``torch.Generator`` seeded with
``seed`` draws float32 standard normals of shape [B, N, H, d] in the order
Q, K, V, dO (K and V with Hkv heads instead of H for grouped-query problems).  For the long-sequence workload a further ``randperm(N)`` from the
same generator picks floor(frac * N) sequence positions whose K rows (all
batches and heads) are multiplied by ``spike`` in float32, which forces large
jumps of the running row maximum in the online softmax.  The tensors are then
cast to the working dtype with round-to-nearest-even.

Paged decode inputs (``make_paged_decode``): the same generator draws Q
[B, H, d], then a page pool K, V [num_pages, page_size, Hkv, d] of standard
normals, then ``randperm(num_pages)`` which hands out the pool's pages to the
sequences in order (sequence b takes the next ceil(seqlens[b] / page_size)
entries), so a sequence's pages are scattered over the pool.  Table entries
past a sequence's last page are -1.  ``decode_lengths`` draws a batch's
sequence lengths uniformly from [lo, hi] with its own seeded generator.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, masks and which passes run."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str = "bf16"           # "bf16" or "fp32"
    causal: tuple = (False,)      # the mask settings the workload covers
    backward: bool = False        # True when dQ, dK, dV are part of it
    spike_frac: float = 0.0       # fraction of K rows scaled by ``spike``
    spike: float = 3.0
    seed: int = 0
    Hkv: int = 0                  # K/V heads (0: same as H)

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    def flops_fwd(self, causal: bool) -> float:
        """4*B*H*N^2*d, halved when causal (the usual attention count)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if causal else f


# The five problem families the method is measured on.
FP32_SMALL = Workload("fp32 fwd B1 H1 N256 d64", 1, 1, 256, 64, "fp32", (False,))
BF16_FWD_N1K = Workload("bf16 fwd B4 H16 N1024 d64", 4, 16, 1024, 64, "bf16", (False, True))
BF16_FWDBWD_N4K = Workload("bf16 fwd+bwd B2 H16 N4096 d128 causal", 2, 16, 4096, 128, "bf16",
                           (True,), backward=True)
BF16_FWDBWD_N16K = Workload("bf16 fwd+bwd B1 H32 N16384 d128 K-spike", 1, 32, 16384, 128, "bf16",
                            (False, True), backward=True, spike_frac=0.01, spike=3.0)
# The same sequence length at d = 64: the d = 64 backward kernel at a size where its
# per-tile costs, not the launch, set the time (timed by the bench's sweep).
BF16_FWDBWD_N16K_D64 = Workload("bf16 fwd+bwd B1 H32 N16384 d64", 1, 32, 16384, 64, "bf16", (False,),
                                backward=True, seed=5)
SWEEP = tuple(
    Workload(f"bf16 fwd sweep B{b} H{h} N{n} d{d}", b, h, n, d, "bf16", (False, True))
    for (b, h, n, d) in ((16, 16, 512, 64), (8, 16, 1024, 128), (4, 32, 2048, 128),
                         (2, 32, 8192, 128), (1, 16, 32768, 128))
)
# Grouped-query attention with the head grouping of the pages' example (64
# query heads sharing 8 K/V heads).
BF16_GQA_H64_KV8 = Workload("bf16 fwd+bwd GQA B1 H64 Hkv8 N4096 d128", 1, 64, 4096, 128, "bf16",
                            (False, True), backward=True, Hkv=8, seed=5)
ALL = (FP32_SMALL, BF16_FWD_N1K, BF16_FWDBWD_N4K, BF16_FWDBWD_N16K, BF16_FWDBWD_N16K_D64) + SWEEP + (BF16_GQA_H64_KV8,)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(B: int, N: int, H: int, d: int, *, seed: int = 0, dtype: str = "bf16",
                spike_frac: float = 0.0, spike: float = 3.0, with_do: bool = True, kv_heads: int | None = None):
    """Return CPU tensors (q, k, v, do) in ``dtype``: q, do [B, N, H, d]; k, v [B, N, kv_heads, d].

    ``kv_heads`` defaults to H.  ``do`` is None when ``with_do`` is False (it
    is still drawn, so Q, K, V are the same either way).
    """
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, N, H, d)
    kv_shape = (B, N, H if kv_heads is None else kv_heads, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(kv_shape, generator=g, dtype=torch.float32)
    v = torch.randn(kv_shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if spike_frac > 0 and N > 0:
        count = int(math.floor(spike_frac * N))
        if count > 0:
            idx = torch.randperm(N, generator=g)[:count]
            k[:, idx] *= float(spike)
    td = torch_dtype(dtype)
    out = [t.to(td).contiguous() for t in (q, k, v, do)]
    if not with_do:
        out[3] = None
    return tuple(out)


def workload_inputs(w: Workload, *, with_do=None):
    return make_inputs(w.B, w.N, w.H, w.d, seed=w.seed, dtype=w.dtype,
                       spike_frac=w.spike_frac, spike=w.spike,
                       with_do=w.backward if with_do is None else with_do, kv_heads=w.kv_heads)


def make_paged_decode(B: int, H: int, Hkv: int, d: int, page_size: int, seqlens, *, seed: int = 0,
                      spare_pages: int = 0, max_pages: int | None = None):
    """Return CPU tensors (q, k_cache, v_cache, block_table, seqlens) for one decode step.

    q: [B, H, d] bf16; k_cache, v_cache: [num_pages, page_size, Hkv, d] bf16 with
    num_pages = the pages the sequences need + ``spare_pages`` (never referenced);
    block_table: [B, max_pages] int32 (default: the longest sequence's page
    count), -1 past each sequence's last page; seqlens: [B] int32.
    """
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    lens = [int(x) for x in seqlens]
    need = [(n + page_size - 1) // page_size for n in lens]
    num_pages = sum(need) + int(spare_pages)
    width = max(need + [1]) if max_pages is None else int(max_pages)
    q = torch.randn((B, H, d), generator=g, dtype=torch.float32)
    k = torch.randn((num_pages, page_size, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((num_pages, page_size, Hkv, d), generator=g, dtype=torch.float32)
    order = torch.randperm(max(num_pages, 1), generator=g)[:num_pages]
    table = torch.full((B, width), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        table[b, :need[b]] = order[nxt:nxt + need[b]].to(torch.int32)
        nxt += need[b]
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(), v.to(torch.bfloat16).contiguous(),
            table, torch.tensor(lens, dtype=torch.int32))


def decode_lengths(B: int, lo: int, hi: int, *, seed: int = 0) -> list:
    """B sequence lengths drawn uniformly from [lo, hi] (a seeded CPU generator)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g)]
