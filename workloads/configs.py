"""Model dimensions and the five synthetic workloads.

The shapes follow the LLaTTE pages: the online ranker looks at roughly 400
recent events per source with candidate/context query tokens (huaxiaozhuan.com
LLaTTE notes, sec. 1.6.4 and 1.7.1), the upstream user model encodes
1600-token histories with user-only query tokens and a 2048-d transfer
embedding (paper-daily.com deep reading, pipeline diagram; huaxiaozhuan.com
sec. 1.6.1), and the horizon sweep uses T in {200, 400, 800, 1600}
(huaxiaozhuan.com sec. 1.5.3). Depth/width values come from the d >= 256,
L in {1,2,4,8} grid of huaxiaozhuan.com sec. 1.5.2.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple


@dataclass(frozen=True)
class Dims:
    """Sequence-module dimensions.

    d        token width
    heads    attention heads h
    d_head   per-head width d_h (attention scale is 1/sqrt(d_h))
    rank     MLA latent rank r (shared K=V latent width)
    d_ctx    width of the non-sequence context vector c (0 = none)
    n_q      query (candidate) tokens appended per user
    keep     per-layer count of most recent HISTORY rows kept as queries
             and as the next layer's sequence (non-increasing)
    d_out    readout width (0 = output the final query-token rows)
    ffn_mult FFN hidden width multiplier (hidden = ffn_mult * d)
    eps      RMSNorm epsilon
    kv_norm  1 = RMSNorm on the KV latent, 0 = plain down-projection
    dtype    storage type of activations and weights: "bf16" or "fp32"
    n_sum    sequence summaries read out of the final query tokens (0 = none)
    sum_rank hidden (low-rank) width of each summary MLP
    d_seq    width of each summary
    q_rank   rank of the low-rank query: Q = RMSNorm([x; c] W_down^Q) W_up^Q
             (0 = the full-rank query W_Q [x; c])
    d_time   hidden dims carrying the additive timestamp encoding of history
             tokens (even; 0 = none)
    attn_form which form of MLA the GPU runs (0 auto, 1 absorbed, 2 per
             head); both compute the same function, the oracle ignores it
    """

    d: int
    heads: int
    d_head: int
    rank: int
    d_ctx: int
    n_q: int
    keep: Tuple[int, ...]
    d_out: int = 0
    ffn_mult: int = 4
    eps: float = 1e-6
    kv_norm: int = 1
    dtype: str = "bf16"
    n_sum: int = 0
    sum_rank: int = 0
    d_seq: int = 0
    q_rank: int = 0
    d_time: int = 0
    attn_form: int = 0

    @property
    def n_layers(self) -> int:
        return len(self.keep)

    @property
    def d_ffn(self) -> int:
        return self.ffn_mult * self.d


@dataclass(frozen=True)
class Workload:
    """A seeded synthetic batch: dims, batch size, length law and value law.

    lengths: ("uniform", lo, hi) inclusive, ("fixed", T) or
             ("lognormal", mu, sigma, lo, hi) rounded then clipped.
    semantic: add a semantic-content term N(0,1) @ W_sem (W_sem: 128 -> d,
              entries N(0, 1/128)) to ID embeddings N(0,1).
    """

    name: str
    dims: Dims
    batch: int
    lengths: tuple
    seed: int
    semantic: bool = False
    sem_dim: int = 128
    description: str = field(default="", compare=False)


def _sweep(L: int) -> Workload:
    return Workload(
        name=f"sweep{L}",
        dims=Dims(d=256, heads=4, d_head=64, rank=128, d_ctx=64, n_q=32,
                  keep=(L, L // 2, L // 4, L // 8)),
        batch=128, lengths=("fixed", L), seed=3, semantic=True,
        description=f"sequence-length sweep at L={L}: B=128, d=256, 4 heads, r=128, "
                    "4 layers halving, 32 candidates, c in R^64")


WORKLOADS = {
    "tiny": Workload(
        name="tiny",
        dims=Dims(d=64, heads=2, d_head=32, rank=32, d_ctx=16, n_q=4, keep=(64, 32),
                  dtype="fp32"),
        batch=4, lengths=("uniform", 16, 64), seed=0,
        description="tiny fp32 case: B=4, T~U[16,64], d=64, 2 heads, r=32, 2 layers"),
    "online": Workload(
        name="online",
        dims=Dims(d=256, heads=4, d_head=64, rank=128, d_ctx=64, n_q=64,
                  keep=(400, 200, 100, 50)),
        batch=256, lengths=("uniform", 100, 400), seed=1, semantic=True,
        description="online ranker: B=256, T~U[100,400], d=256, 4 heads, r=128, "
                    "4 layers 400->200->100->50, 64 candidates, c in R^64"),
    "upstream": Workload(
        name="upstream",
        dims=Dims(d=512, heads=8, d_head=64, rank=256, d_ctx=0, n_q=0,
                  keep=(1600, 800, 400, 200, 100, 100, 100, 100), d_out=2048),
        batch=64, lengths=("fixed", 1600), seed=2,
        description="upstream user model: B=64, T=1600, d=512, 8 heads, r=256, "
                    "8 layers, mean of final rows projected to 2048"),
    "sweep200": _sweep(200),
    "sweep400": _sweep(400),
    "sweep800": _sweep(800),
    "sweep1600": _sweep(1600),
    "skewed": Workload(
        name="skewed",
        dims=Dims(d=256, heads=4, d_head=64, rank=128, d_ctx=64, n_q=256,
                  keep=tuple(512 >> l for l in range(6))),
        batch=512, lengths=("lognormal", 5.5, 0.8, 8, 1600), seed=4, semantic=True,
        description="skewed jagged batch: B=512, T~lognormal(5.5,0.8) clipped to "
                    "[8,1600], d=256, 4 heads, r=128, 6 layers keep 512>>l, 256 candidates"),
}

# Sequence summaries (the pages' LoRAMLP readout of the final query tokens):
# the same batches with k low-rank MLP summaries read out of the flattened
# final query tokens.  The pages fix neither k, the rank nor d_seq; two
# summaries of width 1024 make the 2048-wide transfer vector the upstream
# pipeline hands to downstream models.
WORKLOADS["tiny_sum"] = Workload(
    name="tiny_sum", dims=replace(WORKLOADS["tiny"].dims, n_sum=3, sum_rank=8, d_seq=12),
    batch=4, lengths=("uniform", 16, 64), seed=0,
    description="tiny fp32 case with 3 summaries (rank 8, width 12)")
# The low-rank RMSNorm'd query of the MLA parameterisation (appendix A.3,
# first display) in place of the full-rank target-aware query; the pages give
# no query rank: half the token width is taken.
WORKLOADS["tiny_lq"] = Workload(
    name="tiny_lq", dims=replace(WORKLOADS["tiny"].dims, q_rank=24),
    batch=4, lengths=("uniform", 16, 64), seed=0,
    description="tiny fp32 case with a rank-24 RMSNorm'd query")
WORKLOADS["online_lq"] = Workload(
    name="online_lq", dims=replace(WORKLOADS["online"].dims, q_rank=128),
    batch=256, lengths=("uniform", 100, 400), seed=1, semantic=True,
    description="online ranker with a rank-128 RMSNorm'd query")
WORKLOADS["upstream_lq"] = Workload(
    name="upstream_lq", dims=replace(WORKLOADS["upstream"].dims, q_rank=256),
    batch=64, lengths=("fixed", 1600), seed=2,
    description="upstream user model with a rank-256 RMSNorm'd query")
# Additive timestamp encoding on a subset of the hidden dims of the history
# tokens (appendix A.2 item 1); the pages name neither the subset nor the
# code: a quarter of the width is taken.
WORKLOADS["tiny_time"] = Workload(
    name="tiny_time", dims=replace(WORKLOADS["tiny"].dims, d_time=16),
    batch=4, lengths=("uniform", 16, 64), seed=0,
    description="tiny fp32 case with the timestamp encoding on 16 of 64 dims")
WORKLOADS["online_time"] = Workload(
    name="online_time", dims=replace(WORKLOADS["online"].dims, d_time=64),
    batch=256, lengths=("uniform", 100, 400), seed=1, semantic=True,
    description="online ranker with the timestamp encoding on 64 of 256 dims")
# The upstream batch with MLA forced into its absorbed (latent-space) form, the
# form whose attention is a dense tensor-core contraction at 4 r FLOP per
# score; "auto" runs the per-head form there (fewer FLOPs, exponential-bound).
WORKLOADS["upstream_abs"] = Workload(
    name="upstream_abs", dims=replace(WORKLOADS["upstream"].dims, attn_form=1),
    batch=64, lengths=("fixed", 1600), seed=2,
    description="upstream user model, MLA in its absorbed form")
WORKLOADS["online_sum"] = Workload(
    name="online_sum", dims=replace(WORKLOADS["online"].dims, n_sum=2, sum_rank=128, d_seq=1024),
    batch=256, lengths=("uniform", 100, 400), seed=1, semantic=True,
    description="online ranker + 2 sequence summaries: flatten(64 x 256) -> rank 128 -> 1024")


def workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None
