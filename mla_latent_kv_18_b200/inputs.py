"""Seeded synthetic inputs for MLA decode over a paged latent cache.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic. Both the oracle-based tests and the CUDA path take their
inputs from here.

Workloads (shapes from the "MLA operator design" page §3 -- DeepSeek-V3 MLA
constants 128 heads, d_hc 128, d_c 512, d_R 64, page_size 64 -- and from the
"MHA2MLA" page §3.2 -- 32 heads, head_dim 128 = nope 120 + rope 8, kv_latent 64):

  tiny      B1  n_q1 H16  L256,               identity page table
  dsv3      B16 n_q1 H128 L4096,              permuted page table
  ragged    B64 n_q1 H128 L ~ U[1024, 32768], permuted page table
  long      B16 n_q1 H128 L65536,             permuted page table
  retrofit  B32 n_q2 H32  d_n120 d_c64 d_R8 L8192, permuted page table
  prefill   B8  n_q4096 H128 L4096 (the whole prompt is queried, causal),
            permuted page table ("MLA operator design" §6: batch 8, prompt
            4096, above the prefill threshold of 256 query tokens)

Draw recipe (one torch CPU generator per workload, seed 0 by default), in this
order: seq_lens (ragged only: integers uniform on [1024, 32768]), q_c, q_r,
c_KV pool, k_R pool, W_UK, W_UV, page permutation. Activations and cache
entries are N(0, 1); weights are N(0, 1) / sqrt(d_c). Every value is drawn in
fp32 and rounded to bf16 (round to nearest even). The pool holds exactly
sum_b ceil(L_b / 64) pages; a permuted table assigns them from one random
permutation, without replacement. Unused table entries are -1.
"""
from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int
    heads: int
    d_nope: int
    d_latent: int
    d_rope: int
    d_v: int
    page_size: int
    seq_len: int = 0                 # fixed length for every sequence (0 -> ragged)
    ragged: tuple = ()               # (lo, hi) inclusive bounds when ragged
    table: str = "permuted"          # "identity" or "permuted"

    @property
    def w_std(self) -> float:
        return 1.0 / math.sqrt(self.d_latent)

    @property
    def D(self) -> int:
        return self.d_latent + self.d_rope


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 16, 128, 512, 64, 128, 64, seq_len=256, table="identity"),
    "dsv3": Workload("dsv3", 16, 1, 128, 128, 512, 64, 128, 64, seq_len=4096),
    "ragged": Workload("ragged", 64, 1, 128, 128, 512, 64, 128, 64, ragged=(1024, 32768)),
    "long": Workload("long", 16, 1, 128, 128, 512, 64, 128, 64, seq_len=65536),
    "retrofit": Workload("retrofit", 32, 2, 32, 120, 64, 8, 128, 64, seq_len=8192),
    "prefill": Workload("prefill", 8, 4096, 128, 128, 512, 64, 128, 64, seq_len=4096),
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (for reduced test sizes)."""
    return replace(WORKLOADS[name], **overrides)


def _randn_bf16(g: torch.Generator, shape, scale: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0, seq_lens=None) -> dict:
    """Draw one set of inputs on the CPU.

    seq_lens: optional explicit list of lengths (overrides the workload's rule;
    used by edge-case tests). Returns a dict of CPU tensors:
      q_c [B,n_q,H,d_nope], q_r [B,n_q,H,d_rope] (bf16)
      ckv_pool [num_pages,P,d_latent], kr_pool [num_pages,P,d_rope] (bf16)
      w_uk [H,d_nope,d_latent], w_uv [H,d_latent,d_v] (bf16)
      seq_lens [B] int32, block_table [B,max_pages] int32
    """
    g = torch.Generator().manual_seed(seed)
    B, P = w.batch, w.page_size
    if seq_lens is not None:
        lens = torch.tensor(list(seq_lens), dtype=torch.int32)
        assert lens.numel() == B
    elif w.ragged:
        lo, hi = w.ragged
        lens = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    else:
        lens = torch.full((B,), w.seq_len, dtype=torch.int32)
    pages_per_seq = [(int(l) + P - 1) // P for l in lens]
    num_pages = max(1, sum(pages_per_seq))
    max_pages = max(1, max(pages_per_seq))

    q_c = _randn_bf16(g, (B, w.n_q, w.heads, w.d_nope))
    q_r = _randn_bf16(g, (B, w.n_q, w.heads, w.d_rope))
    ckv_pool = _randn_bf16(g, (num_pages, P, w.d_latent))
    kr_pool = _randn_bf16(g, (num_pages, P, w.d_rope))
    w_uk = _randn_bf16(g, (w.heads, w.d_nope, w.d_latent), w.w_std)
    w_uv = _randn_bf16(g, (w.heads, w.d_latent, w.d_v), w.w_std)

    if w.table == "identity":
        perm = torch.arange(num_pages, dtype=torch.int64)
    else:
        perm = torch.randperm(num_pages, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    return dict(q_c=q_c, q_r=q_r, ckv_pool=ckv_pool, kr_pool=kr_pool, w_uk=w_uk, w_uv=w_uv,
                seq_lens=lens, block_table=table)


def to_device(inputs: dict, device) -> dict:
    """Copy every tensor of an input dict to ``device``."""
    return {k: v.to(device) for k, v in inputs.items()}
