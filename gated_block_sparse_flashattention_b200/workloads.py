"""Seeded synthetic inputs for SAS gated block-sparse attention.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic (no normalisation, selection or attention), so the CUDA
path and the CPU oracle can both be fed from it.

Workload shapes stand in for the Qwen3-class layers of the SAS paper (arXiv
2609.13141, §4.2.1 and §5.1: block size 64, budgets of 1024 and 2048 tokens,
GQA, 8K-64K context) and for its decode setting (§6.3, one new token per
sequence over a long KV cache). No dataset or trained weight is involved:
Q/K/V/dO are i.i.d. N(0, 1) and the selector scores follow the per-workload
distribution below.

Generation order is fixed: Q, K, V, dO, then the selector scores s (then the
planted blocks), all from one CPU ``torch.Generator`` seeded once.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": storage/compute type of Q, K, V, dO, O, dQ, dK, dV
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int                # sequence length (training) or KV-cache length (decode)
    K: int                # budget in blocks, the current block included
    block: int = 64
    s_dist: str = "normal"   # "normal", "normal2_planted3", "student_t3"
    decode: bool = False

    @property
    def NB(self) -> int:
        return (self.T + self.block - 1) // self.block

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    # Tiny fp32 fwd+bwd.
    "tiny_f32": Workload("tiny_f32", "f32", 1, 4, 1, 64, 1024, 4),
    # Qwen3-4B-like layer, budget 1024 tokens, 3 planted high-score blocks per query.
    "qwen3_4b_t8k": Workload("qwen3_4b_t8k", "bf16", 1, 32, 8, 128, 8192, 16, s_dist="normal2_planted3"),
    # Qwen3-8B-like layer, budget 2048 tokens, heavy-tailed selector scores.
    "qwen3_8b_t32k": Workload("qwen3_8b_t32k", "bf16", 2, 32, 8, 128, 32768, 32, s_dist="student_t3"),
    # Qwen3-14B-like layer, tight budget of 1024 tokens at 64K context.
    "qwen3_14b_t64k": Workload("qwen3_14b_t64k", "bf16", 1, 40, 8, 128, 65536, 16),
    # Memory-bound decode: 16 sequences, one new token each over a 32768-token cache.
    "decode_b16_l32k": Workload("decode_b16_l32k", "bf16", 16, 32, 8, 128, 32768, 16, decode=True),
    # Long-context decode over a paged cache: 8 sequences, one new token each at 512K
    # context, budget 2048 tokens (32 blocks, the current one included).
    "decode_b8_l512k_paged": Workload("decode_b8_l512k_paged", "bf16", 8, 32, 8, 128, 524288, 32, decode=True),
    # The same at 64K context (a 2 GB pool), for profiling runs.
    "decode_b8_l64k_paged": Workload("decode_b8_l64k_paged", "bf16", 8, 32, 8, 128, 65536, 32, decode=True),
}


def _selector_scores(gen, shape, dist: str, block: int):
    if dist == "normal":
        return torch.randn(shape, generator=gen, device=gen.device)
    if dist == "normal2_planted3":
        s = 2.0 * torch.randn(shape, generator=gen)
        B, Hkv, T, NB = shape
        # Three distinct historical blocks per query row (rows with at least three
        # historical blocks) get a score far above the rest.
        r = torch.rand(shape, generator=gen)
        c = (torch.arange(T) // block).view(1, 1, T, 1)
        m = torch.arange(NB).view(1, 1, 1, NB)
        r = torch.where(m < c, r, torch.full_like(r, 2.0))
        idx = torch.topk(r, 3, dim=-1, largest=False).indices
        plant = (c.expand(B, Hkv, T, 1) >= 3).expand(B, Hkv, T, 3)
        vals = torch.gather(s, -1, idx)
        s.scatter_(-1, idx, torch.where(plant, torch.full_like(vals, 10.0), vals))
        return s
    if dist == "student_t3":
        # Student-t with nu = 3: Z / sqrt(chi2_3 / 3), chi2_3 a sum of three squared normals.
        z = torch.randn(shape, generator=gen)
        chi = torch.zeros(shape)
        for _ in range(3):
            chi += torch.randn(shape, generator=gen) ** 2
        return z / torch.sqrt(chi / 3.0)
    raise ValueError(f"unknown selector-score distribution {dist!r}")


def make_training_inputs(w: Workload, seed: int = 0):
    """CPU tensors for one fwd+bwd problem.

    Returns dict with Q [B,Hq,T,d], K/V [B,Hkv,T,d], dO [B,Hq,T,d] in the
    workload's dtype, and s [B,Hkv,T,NB] float32 selector scores.
    """
    gen = torch.Generator().manual_seed(seed)
    dt = w.torch_dtype
    Q = torch.randn(w.B, w.Hq, w.T, w.d, generator=gen).to(dt)
    K = torch.randn(w.B, w.Hkv, w.T, w.d, generator=gen).to(dt)
    V = torch.randn(w.B, w.Hkv, w.T, w.d, generator=gen).to(dt)
    dO = torch.randn(w.B, w.Hq, w.T, w.d, generator=gen).to(dt)
    s = _selector_scores(gen, (w.B, w.Hkv, w.T, w.NB), w.s_dist, w.block).float()
    return {"Q": Q, "K": K, "V": V, "dO": dO, "s": s}


def make_decode_inputs(w: Workload, seed: int = 0, seqlen=None):
    """CPU tensors for one decode step.

    q [B,Hq,d], Kc/Vc [B,Hkv,Lmax,d] in the workload's dtype, seqlen [B] int32
    (default: every sequence fills the cache, the new token at position
    Lmax-1), s [B,Hkv,NBmax] float32 selector scores.
    """
    gen = torch.Generator().manual_seed(seed)
    dt = w.torch_dtype
    q = torch.randn(w.B, w.Hq, w.d, generator=gen).to(dt)
    Kc = torch.randn(w.B, w.Hkv, w.T, w.d, generator=gen).to(dt)
    Vc = torch.randn(w.B, w.Hkv, w.T, w.d, generator=gen).to(dt)
    s = _selector_scores(gen, (w.B, w.Hkv, 1, w.NB), w.s_dist, w.block).reshape(w.B, w.Hkv, w.NB).float()
    if seqlen is None:
        seqlen = torch.full((w.B,), w.T, dtype=torch.int32)
    return {"q": q, "Kc": Kc, "Vc": Vc, "s": s, "seqlen": torch.as_tensor(seqlen, dtype=torch.int32)}


def custom(name="custom", dtype="bf16", B=1, Hq=4, Hkv=1, d=64, T=256, K=3, block=64, s_dist="normal", decode=False):
    """A workload of arbitrary shape (tests and smoke use these)."""
    return Workload(name, dtype, B, Hq, Hkv, d, T, K, block, s_dist, decode)


def make_paged_decode_inputs(w: Workload, seed: int = 0, seqlen=None, pool_pages=None, device="cpu"):
    """Tensors for one decode step over a paged KV cache of one-block pages.

    q [B,Hq,d], Kp/Vp [num_pages,Hkv,block,d] in the workload's dtype,
    page_table [B,NB] int32, seqlen [B] int32, s [B,Hkv,NB] float32, all on
    ``device`` (drawn there from one generator seeded once, in the order q, s,
    page table, Kp, Vp). Without ``pool_pages`` every block a sequence reaches
    gets a page of its own, the pages in a seeded random order among a few unused
    ones; with ``pool_pages = P`` the pool holds P pages and each block names a
    seeded random one of them (pages shared, as under prefix sharing), which keeps
    long contexts small. Blocks past a sequence's end hold -1.
    """
    gen = torch.Generator(device=device).manual_seed(seed)
    dt = w.torch_dtype
    q = torch.randn(w.B, w.Hq, w.d, generator=gen, device=device).to(dt)
    s = _selector_scores(gen, (w.B, w.Hkv, 1, w.NB), w.s_dist, w.block).reshape(w.B, w.Hkv, w.NB).float()
    if seqlen is None:
        seqlen = [w.T] * w.B
    seqlen = torch.as_tensor(seqlen, dtype=torch.int32)
    n_blocks = [(int(L) + w.block - 1) // w.block for L in seqlen]
    table = torch.full((w.B, w.NB), -1, dtype=torch.int32)
    if pool_pages is None:
        used = sum(n_blocks)
        num_pages = used + max(4, used // 16)
        perm = torch.randperm(num_pages, generator=gen, device=device).to(torch.int32).cpu()
        off = 0
        for b, n in enumerate(n_blocks):
            table[b, :n] = perm[off:off + n]
            off += n
    else:
        num_pages = pool_pages
        pages = torch.randint(0, pool_pages, (w.B, w.NB), generator=gen, device=device).to(torch.int32).cpu()
        for b, n in enumerate(n_blocks):
            table[b, :n] = pages[b, :n]
    pools = []
    for _ in range(2):
        pool = torch.empty(num_pages, w.Hkv, w.block, w.d, dtype=dt, device=device)
        for p0 in range(0, num_pages, 4096):   # bounded fp32 temporaries
            p1 = min(num_pages, p0 + 4096)
            pool[p0:p1] = torch.randn(p1 - p0, w.Hkv, w.block, w.d, generator=gen, device=device).to(dt)
        pools.append(pool)
    return {"q": q, "Kp": pools[0], "Vp": pools[1], "page_table": table.to(device), "seqlen": seqlen.to(device),
            "s": s}
