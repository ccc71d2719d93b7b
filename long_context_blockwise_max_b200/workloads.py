"""Seeded synthetic inputs for the Star / Pulsar two-phase attention path.

This module only draws random inputs of the shapes, value distributions and
structure of the workloads the Pulsar Attention and Star Attention pages
describe (Llama-3.1-8B attention shape, Zipf-distributed token ids, 32-token
chunks, 64-token sink).  It holds none of the method's arithmetic: no
document frequency, no scoring, no rotary embedding, no attention.  Both the
CUDA path (tests, bench) and the fp64 oracle read the arrays it returns.

Recipe
------
* Token ids: ``P(id = r - 1) ∝ r^(-s)`` for ranks ``r = 1..V`` (Zipf with
  exponent ``s`` over a vocabulary of ``V`` ids), drawn by inverse-CDF
  sampling from numpy's PCG64 stream seeded with ``seed``.  Optionally
  ``planted`` ids that the draw did not produce are written, once each, at
  ``planted`` distinct positions (both chosen from the same stream), so the
  sequence holds that many tokens with document frequency exactly 1.
* Q / K / V: standard normal N(0, 1) drawn by torch's seeded generator in
  fp32 on the requested device, then rounded to the run's dtype.

Seeds used by the named workloads: ids 1, Q 2, K 3, V 4, Phase-2 query 5,
KV cache K 6 and V 7.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_IDS, SEED_Q, SEED_K, SEED_V, SEED_QUERY, SEED_KC, SEED_VC = 1, 2, 3, 4, 5, 6, 7


def zipf_token_ids(L: int, vocab: int, s: float = 1.1, seed: int = SEED_IDS,
                   planted: int = 0) -> np.ndarray:
    """``L`` int32 token ids, Zipf(``s``) over ``vocab`` ids, plus planted singletons."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    w = ranks ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(L)
    ids = np.searchsorted(cdf, u, side="right").astype(np.int64)
    np.minimum(ids, vocab - 1, out=ids)
    if planted:
        absent = np.setdiff1d(np.arange(vocab, dtype=np.int64), np.unique(ids))
        if absent.size < planted:
            raise ValueError("vocabulary too small for the requested planted singletons")
        new_ids = rng.choice(absent, size=planted, replace=False)
        pos = rng.choice(L, size=planted, replace=False)
        ids[pos] = new_ids
    return ids.astype(np.int32)


def windowed_token_ids(n_blocks: int, block: int, spans=(1, 2, 3, 4, 8, 9, 16), seed: int = 0) -> np.ndarray:
    """Token ids whose set of blocks is fixed by construction: for every
    span v in ``spans`` (v <= n_blocks) and start block i there is one id
    that occurs exactly once in each of the v cyclically consecutive blocks
    i, i + 1, .., i + v - 1 (mod n_blocks) and nowhere else; id 0 fills the
    other positions of every block.  Every block therefore holds sum(spans)
    such ids, at positions shuffled by numpy's PCG64 stream seeded with
    ``seed``.  Id 1 + s * n_blocks + i is span number s starting at block i
    (vocabulary 1 + len(spans) * n_blocks)."""
    spans = [v for v in spans if v <= n_blocks]
    if sum(spans) > block:
        raise ValueError("block too short for the requested spans")
    rng = np.random.Generator(np.random.PCG64(seed))
    ids = np.zeros(n_blocks * block, dtype=np.int64)
    for j in range(n_blocks):
        toks = [1 + s * n_blocks + (j - o) % n_blocks for s, v in enumerate(spans) for o in range(v)]
        row = np.zeros(block, dtype=np.int64)
        row[rng.choice(block, size=len(toks), replace=False)] = toks
        ids[j * block:(j + 1) * block] = row
    return ids.astype(np.int32)


def normal(shape, seed: int, dtype: torch.dtype = torch.float32,
           device: str | torch.device = "cpu") -> torch.Tensor:
    """N(0, 1) tensor of ``shape`` from torch's generator seeded with ``seed``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    return x if dtype == torch.float32 else x.to(dtype)


@dataclass(frozen=True)
class Workload:
    """One configuration of the path: sizes, dtypes and selection budget."""
    name: str
    L: int                      # context tokens
    vocab: int
    block: int                  # tokens per block (one virtual host per block)
    sink: int = 64
    chunk: int = 32
    budget_frac: float = 0.125  # summary budget as a fraction of the block
    hq: int = 32
    hkv: int = 8
    d: int = 128
    dtype: torch.dtype = torch.bfloat16
    rope_theta: float = 500000.0
    zipf_s: float = 1.1
    planted: int = 0
    q_tokens: int = 64          # Phase-2 query length
    # Phase-2 decode shape (independent single-token queries over per-batch caches)
    decode_batch: int = 0
    decode_T: int = 0
    decode_shards: int = 0
    notes: str = field(default="", compare=False)

    @property
    def n_blocks(self) -> int:
        return self.L // self.block

    @property
    def k_chunks(self) -> int:
        return int(self.budget_frac * self.block) // self.chunk

    def token_ids(self) -> np.ndarray:
        return zipf_token_ids(self.L, self.vocab, self.zipf_s, SEED_IDS, self.planted)

    def qkv(self, device="cpu"):
        q = normal((self.L, self.hq, self.d), SEED_Q, self.dtype, device)
        k = normal((self.L, self.hkv, self.d), SEED_K, self.dtype, device)
        v = normal((self.L, self.hkv, self.d), SEED_V, self.dtype, device)
        return q, k, v

    def query(self, device="cpu"):
        """Phase-2 query [1][Tq][Hq][d] (pre-RoPE; placed right after the context)."""
        return normal((1, self.q_tokens, self.hq, self.d), SEED_QUERY, self.dtype, device)

    def decode_inputs(self, device="cpu"):
        """Decode query [B][1][Hq][d] and per-batch KV caches [B][T][Hkv][d]."""
        B, T = self.decode_batch, self.decode_T
        q = normal((B, 1, self.hq, self.d), SEED_QUERY, self.dtype, device)
        kc = normal((B, T, self.hkv, self.d), SEED_KC, self.dtype, device)
        vc = normal((B, T, self.hkv, self.d), SEED_VC, self.dtype, device)
        return q, kc, vc


TINY = Workload("tiny_2k", L=2048, vocab=1000, block=512, hq=4, hkv=2, d=64,
                dtype=torch.float32, rope_theta=10000.0, q_tokens=32,
                notes="2048 ids, 4 blocks of 512, 2 summary chunks/block, fp32")
LLAMA_32K = Workload("llama3.1-8b_attn_32k", L=32768, vocab=128256, block=8192, planted=200,
                     notes="4 blocks of 8192, 1024-token summaries, 200 planted singletons")
LLAMA_128K = Workload("llama3.1-8b_attn_128k", L=131072, vocab=128256, block=16384,
                      notes="8 blocks of 16384, 2048-token summaries")
DECODE_128K = Workload("decode_128k_b16", L=131072, vocab=128256, block=16384,
                       decode_batch=16, decode_T=131072, decode_shards=8,
                       notes="16 single-token queries, 128K bf16 cache in 8 shards")
SCALE_1M = Workload("scale_1m", L=1048576, vocab=128256, block=32768,
                    decode_batch=4, decode_T=1048576, decode_shards=32,
                    notes="1M ids, 32 blocks of 32768 (4096-token budget); decode B=4 over 1M")

WORKLOADS = {w.name: w for w in (TINY, LLAMA_32K, LLAMA_128K, DECODE_128K, SCALE_1M)}
