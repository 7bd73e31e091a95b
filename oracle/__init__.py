"""fp64 CPU oracle for the LLaTTE sequence-module forward pass.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA library.

Sources (LLaTTE notes on huaxiaozhuan.com, appendix A.2 "Sequence Module" and
A.3 "Multi-head Latent Attention"; daiwk.github.io reproduction notes,
"core formula"):
  * plan.py   - pyramidal schedule: per-layer kept counts and jagged offsets
  * model.py  - Form B: MLA absorbed into latent-space multi-query attention,
                computed per user with fp64 NumPy (the main oracle)
  * brute.py  - Form A: the non-absorbed MLA applied to the whole fused
                sequence with explicit masks, then the pages' tail slice
                (the brute force that Form B is checked against)
  * analysis.py - attention-probability statistics of the query tokens
                (cumulative attention on the most recent / the top-k keys,
                attention by hours before the request; appendix A.4)

Readings of points the pages leave open (scale 1/sqrt(d_h); candidates see all
history keys but no query token; keep counts count history rows only; RMSNorm
on the KV latent; FFN = W2 SiLU(W1 z) without biases; eps = 1e-6; mean-pool +
linear readout for the upstream workload; a sequence summary is a SiLU MLP with
a rank-r bottleneck over the row-major flattened final query tokens) are
stated where they are used.

Parity status: every function here is pinned by tests against invariants,
special cases and library routines (see tests/test_oracle.py). The numeric
forward values themselves are not printed on the pages; parity against the
pages' own numbers is unpinned for that reason.
"""
from .plan import plan_layers, LayerPlan
from .model import forward, layer_forward, absorb, rmsnorm, silu, summaries, time_encoding
from .brute import forward_brute

__all__ = ["plan_layers", "LayerPlan", "forward", "layer_forward", "absorb",
           "rmsnorm", "silu", "summaries", "time_encoding", "forward_brute"]
