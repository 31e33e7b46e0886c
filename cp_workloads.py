"""Seeded synthetic inputs and the named workloads.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic.  Both the CUDA path's tests/bench and the oracle's tests
take their inputs from here, so the two sides see bit-identical values.

Recipe: a CPU torch.Generator seeded with 1000 + workload index draws fp32
standard normals for Q, then K, then V, each of shape [b, S, H, d]; bf16
workloads cast them with round-to-nearest-even; the striped 32K workload then
multiplies K by 4 (a power of two, so exact in bf16) to widen the lse range.
The backward's output gradient dO comes from a second generator seeded with
2000 + that seed, the same way; document starts (All-Gather workload) from a third,
seeded with 3000 + that seed (uniform distinct cut points).
Head shapes follow the Llama-3 GQA table (8B: 32 query / 8 KV heads, 70B: 64 / 8).
"""
from dataclasses import dataclass, field, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: str          # "bf16" or "fp32"
    b: int
    hq: int
    hkv: int
    d: int
    S: int
    causal: bool
    layout: str         # "contiguous" | "zigzag" | "striped"
    N: int
    k_scale: float = 1.0
    n_docs: int = 1      # documents packed into the sequence (document mask when > 1)
    notes: str = field(default="")

    @property
    def seed(self):
        return 1000 + self.index

    @property
    def c(self):
        return self.S // self.N

    @property
    def scale(self):
        return self.d ** -0.5

    def doc_starts(self):
        """First position of each document (a seeded draw, see random_doc_starts)."""
        return random_doc_starts(self.S, self.n_docs, self.seed)

    def visible_pairs(self):
        """Unmasked (query, key) pairs per (batch, head): per document of length L,
        L(L+1)/2 causal, L^2 otherwise (one document: S(S+1)/2 or S^2)."""
        starts = self.doc_starts() + [self.S]
        lens = [e - a for a, e in zip(starts[:-1], starts[1:])]
        return sum(L * (L + 1) // 2 if self.causal else L * L for L in lens)

    def effective_flops(self):
        """QK^T plus PV multiply-adds, 4*d flops per visible pair per query head."""
        return 4 * self.b * self.hq * self.d * self.visible_pairs()

    def as_dict(self):
        return asdict(self)


WORKLOADS = [
    Workload("fp32_s256_contig2", 1, "fp32", 1, 2, 2, 64, 256, True, "contiguous", 2,
             notes="fp32 exactness case"),
    Workload("llama3_8b_s8k_zigzag4", 2, "bf16", 1, 32, 8, 128, 8192, True, "zigzag", 4),
    Workload("s32k_b2_striped8_kx4", 3, "bf16", 2, 32, 8, 128, 32768, True, "striped", 8,
             k_scale=4.0),
    Workload("llama3_70b_s128k_zigzag8", 4, "bf16", 1, 64, 8, 128, 131072, True, "zigzag", 8),
    Workload("noncausal_s64k_contig32", 5, "bf16", 1, 16, 16, 128, 65536, False, "contiguous", 32),
    Workload("llama3_8b_s8k_zigzag4_docs8", 6, "bf16", 1, 32, 8, 128, 8192, True, "zigzag", 4, n_docs=8,
             notes="All-Gather CP with a document mask"),
    Workload("llama3_8b_s8k_zigzag4_docs32", 7, "bf16", 1, 32, 8, 128, 8192, True, "zigzag", 4, n_docs=32,
             notes="All-Gather CP with a document mask, short documents"),
]
BY_NAME = {w.name: w for w in WORKLOADS}
# the largest workload that fits one GPU: the Llama-3-70B head shape at S = 131072
BENCH_WORKLOAD = "llama3_70b_s128k_zigzag8"


def torch_dtype(name):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def random_qkv(b, S, hq, hkv, d, dtype="bf16", seed=0, k_scale=1.0, q_zero=False):
    """Q, K, V on the CPU in original token order, [b, S, H, d], d contiguous."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((b, S, hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((b, S, hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((b, S, hkv, d), generator=g, dtype=torch.float32)
    td = torch_dtype(dtype)
    q, k, v = q.to(td), k.to(td), v.to(td)
    if k_scale != 1.0:
        k = k * k_scale
    if q_zero:
        q.zero_()
    return q, k, v


def make_inputs(w: Workload):
    return random_qkv(w.b, w.S, w.hq, w.hkv, w.d, w.dtype, w.seed, w.k_scale)


def random_doc_starts(S, n_docs, seed=0):
    """Document starts for a sequence of S tokens: 0 and n_docs - 1 distinct cut
    points drawn uniformly from 1 .. S - 1 by a CPU generator seeded with
    3000 + seed, sorted."""
    if n_docs <= 1:
        return [0]
    g = torch.Generator().manual_seed(3000 + seed)
    cuts = (torch.randperm(S - 1, generator=g)[:n_docs - 1] + 1).sort().values
    return [0] + [int(c) for c in cuts]


def random_do(b, S, hq, d, dtype="bf16", seed=0):
    """Output gradient dO [b, S, hq, d] on the CPU in original token order: fp32
    standard normals from a CPU generator seeded with 2000 + seed, cast like Q."""
    g = torch.Generator().manual_seed(2000 + seed)
    return torch.randn((b, S, hq, d), generator=g, dtype=torch.float32).to(torch_dtype(dtype))


def make_do(w: Workload):
    return random_do(w.b, w.S, w.hq, w.d, w.dtype, w.seed)
