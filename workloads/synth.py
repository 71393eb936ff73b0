"""Seeded synthetic inputs shaped like the pages' 7B / 70B decode workloads.

Nothing here computes attention, slots or refcounts.  A workload is:
  * context lengths drawn from the config's distribution (numpy PCG64, seeded);
  * a physical placement: a seeded permutation of the pool's block ids,
    consumed in order to fill each sequence's block table (unused table
    entries are -1);
  * fp16 ~N(0,1) q / K / V drawn with a seeded torch generator on the
    requested device (K optionally with a few seeded outlier channels x10);
  * every pool row that no sequence covers (unreferenced blocks and the rows
    past the end of each sequence's last block) holds NaN, so that a stray
    read shows up in the output.

Layouts: q [B][q_len][Hq][D]; pools [num_blocks][Hkv][bs][D]; tables int32
[B][max_blocks]; context_lens int32 [B].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Optional

import numpy as np
import torch


@dataclass(frozen=True)
class ConfigSpec:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    bs: int
    q_len: int
    lens: Callable[[np.random.Generator, int], np.ndarray]
    pool_factor: float = 1.2
    pool_blocks: Optional[int] = None
    k_outlier_channels: int = 0
    description: str = ""


def _fixed(values):
    return lambda rng, B: np.asarray(values[:B], dtype=np.int32)


def _uniform(lo, hi):
    return lambda rng, B: rng.integers(lo, hi + 1, size=B).astype(np.int32)


def _lognormal(median, sigma, cap):
    def draw(rng, B):
        z = rng.standard_normal(B)
        v = np.rint(median * np.exp(sigma * z))
        return np.clip(v, 1, cap).astype(np.int32)
    return draw


def _const(L):
    return lambda rng, B: np.full(B, L, dtype=np.int32)


CONFIGS = {
    "tiny": ConfigSpec(
        "tiny", 1, B=2, Hq=4, Hkv=4, D=64, bs=16, q_len=1, lens=_fixed([37, 64]),
        pool_blocks=16,
        description="2 sequences (37, 64 tokens), MHA 4 heads, head_dim 64, block 16, "
                    "16-block pool with permuted physical ids"),
    "llama7b_mha": ConfigSpec(
        "llama7b_mha", 2, B=64, Hq=32, Hkv=32, D=128, bs=16, q_len=1,
        lens=_uniform(512, 4096), k_outlier_channels=4,
        description="Llama-2-7B-shaped layer: 64 sequences, 32 heads MHA, head_dim 128, "
                    "block 16, lengths U[512,4096], pool 1.2x need, 4 K outlier channels x10"),
    "llama70b_gqa": ConfigSpec(
        "llama70b_gqa", 3, B=128, Hq=64, Hkv=8, D=128, bs=16, q_len=1,
        lens=_lognormal(1024, 0.8, 8192),
        description="Llama-2-70B-shaped GQA: 128 sequences, 64 query / 8 KV heads, "
                    "head_dim 128, block 16, lengths lognormal(median 1024, sigma 0.8, cap 8192)"),
    "llama70b_gqa_bs8": ConfigSpec(
        "llama70b_gqa_bs8", 3, B=128, Hq=64, Hkv=8, D=128, bs=8, q_len=1,
        lens=_lognormal(1024, 0.8, 8192),
        description="as llama70b_gqa with 8-token blocks"),
    "prefix_beam": ConfigSpec(
        "prefix_beam", 4, B=64, Hq=32, Hkv=8, D=128, bs=16, q_len=1,
        lens=_uniform(32, 512),
        description="64 requests sharing one 2048-token prefix (same physical blocks) plus "
                    "private suffixes U[32,512]; GQA 32/8, head_dim 128, block 16"),
    "beam_search": ConfigSpec(
        "beam_search", 7, B=32, Hq=32, Hkv=8, D=128, bs=16, q_len=1,
        lens=_uniform(500, 2000),
        description="beam search: 32 prompts U[500,2000] x 8 beams = 256 beams; per step the "
                    "survivors are drawn within each prompt's beams (fork / reorder of block "
                    "tables), shared partial last blocks are copied on write in one batched "
                    "call, one token is appended per beam, then decode attention; GQA 32/8, "
                    "head_dim 128, block 16"),
    "long_decode": ConfigSpec(
        "long_decode", 5, B=8, Hq=32, Hkv=8, D=128, bs=16, q_len=1, lens=_const(32768),
        description="8 sequences of 32768 tokens, GQA 32/8, head_dim 128, block 16"),
    "long_verify": ConfigSpec(
        "long_verify", 5, B=8, Hq=32, Hkv=8, D=128, bs=16, q_len=5, lens=_const(32768),
        description="as long_decode with a causal 5-token verify window per sequence "
                    "(the 5 draft tokens are the last 5 of the 32768)"),
    "prefill_chunk": ConfigSpec(
        "prefill_chunk", 6, B=8, Hq=64, Hkv=8, D=128, bs=16, q_len=512,
        lens=_uniform(1024 + 512, 4096 + 512),
        description="chunked prefill, Llama-2-70B-shaped GQA 64/8, head_dim 128, block 16: "
                    "8 sequences, a 512-token chunk on prefixes U[1024,4096] (the chunk's "
                    "K/V already in the cache)"),
}

PREFIX_TOKENS = 2048  # shared system-prompt prefix of the prefix_beam config


@dataclass
class Workload:
    spec: ConfigSpec
    lens: np.ndarray            # int32 [B]
    block_tables: np.ndarray    # int32 [B][max_blocks], -1 past each sequence's blocks
    num_blocks: int             # pool capacity in blocks
    order: np.ndarray           # int32 permutation of 0..num_blocks-1 (placement order)
    q: torch.Tensor             # fp16 [B][q_len][Hq][D]
    k_pool: torch.Tensor        # fp16 [num_blocks][Hkv][bs][D]
    v_pool: torch.Tensor
    scale: float
    extra: dict = field(default_factory=dict)

    @property
    def B(self):
        return int(self.lens.shape[0])


def normal_fp16(shape, seed: int, device="cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(shape, generator=g, device=device, dtype=torch.float16)


def fill_normal_fp16(t: torch.Tensor, seed: int) -> torch.Tensor:
    g = torch.Generator(device=t.device)
    g.manual_seed(int(seed))
    t.normal_(generator=g)
    return t


def random_distinct_slots(n: int, num_slots: int, seed: int) -> np.ndarray:
    """n distinct slot indices in [0, num_slots), seeded."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.choice(num_slots, size=n, replace=False).astype(np.int64)


def _ceil_div(a, b):
    return -(-a // b)


def make_workload(name: str, device="cpu", *, B: Optional[int] = None,
                  max_len: Optional[int] = None, lens=None, bs: Optional[int] = None,
                  q_len: Optional[int] = None, seed: Optional[int] = None,
                  Hq: Optional[int] = None, Hkv: Optional[int] = None, D: Optional[int] = None,
                  spare_blocks: int = 0, poison: bool = True) -> Workload:
    """Build config ``name``; the keyword overrides shrink or reshape it for
    oracle-sized runs.

    ``spare_blocks`` adds free blocks beyond the config's pool (room to append).
    """
    spec = CONFIGS[name]
    seed = spec.seed if seed is None else seed
    B = spec.B if B is None else B
    bs = spec.bs if bs is None else bs
    q_len = spec.q_len if q_len is None else q_len
    rng = np.random.Generator(np.random.PCG64(seed))
    if lens is None:
        lens = spec.lens(rng, B)
    lens = np.asarray(lens, dtype=np.int32)
    if max_len is not None:
        lens = np.minimum(lens, max_len).astype(np.int32)
    B = int(lens.shape[0])

    prefix_blocks = 0
    if name == "prefix_beam":
        prefix_blocks = PREFIX_TOKENS // bs
        suffix = lens
        lens = (suffix + PREFIX_TOKENS).astype(np.int32)
    need = [_ceil_div(int(L), bs) for L in lens]
    private = [n - prefix_blocks for n in need]
    total_need = prefix_blocks + sum(private)
    if spec.pool_blocks is not None and name != "prefix_beam":
        num_blocks = max(spec.pool_blocks, total_need)
    else:
        num_blocks = int(math.ceil(spec.pool_factor * total_need))
    # spare blocks go after the permuted pool, so that the placement of the
    # sequences does not depend on how much room is added for appends
    order = np.concatenate([rng.permutation(num_blocks),
                            num_blocks + np.arange(int(spare_blocks))]).astype(np.int32)
    num_blocks += int(spare_blocks)

    max_blocks = max(1, max(need) if need else 1)
    tables = np.full((B, max_blocks), -1, dtype=np.int32)
    nxt = 0
    shared = order[:prefix_blocks]
    nxt = prefix_blocks
    for s in range(B):
        tables[s, :prefix_blocks] = shared
        tables[s, prefix_blocks:need[s]] = order[nxt:nxt + private[s]]
        nxt += private[s]

    dev = torch.device(device)
    Hq = spec.Hq if Hq is None else Hq
    Hkv = spec.Hkv if Hkv is None else Hkv
    D = spec.D if D is None else D
    q = normal_fp16((B, q_len, Hq, D), seed * 1000 + 1, dev)
    k_pool = torch.empty((num_blocks, Hkv, bs, D), dtype=torch.float16, device=dev)
    v_pool = torch.empty_like(k_pool)
    fill_normal_fp16(k_pool, seed * 1000 + 2)
    fill_normal_fp16(v_pool, seed * 1000 + 3)
    extra = {}
    if spec.k_outlier_channels:
        ch = np.sort(rng.choice(D, size=spec.k_outlier_channels, replace=False))
        k_pool[..., torch.as_tensor(ch, device=dev)] *= 10.0
        extra["outlier_channels"] = ch
    if poison:
        used = np.zeros(num_blocks, dtype=bool)
        used[tables[tables >= 0]] = True
        unused = torch.as_tensor(np.nonzero(~used)[0], device=dev, dtype=torch.long)
        if unused.numel():
            k_pool[unused] = float("nan")
            v_pool[unused] = float("nan")
        for s in range(B):
            L = int(lens[s])
            if need[s] and L % bs:
                blk = int(tables[s, need[s] - 1])
                k_pool[blk, :, L % bs:, :] = float("nan")
                v_pool[blk, :, L % bs:, :] = float("nan")
    extra["prefix_blocks"] = prefix_blocks
    return Workload(spec=spec, lens=lens, block_tables=tables, num_blocks=num_blocks,
                    order=order, q=q, k_pool=k_pool, v_pool=v_pool,
                    scale=1.0 / math.sqrt(D), extra=extra)
