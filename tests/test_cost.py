"""Checks of the FLOP / byte model behind the benchmark's roofline figures.

The per-form counts follow the two MLA displays (absorbed: scores over the
rank-r latent; per head: scores over d_h after the K | V up-projection), so
their ratios are fixed by the dimensions; the upstream total is checked
against an independent hand count of the upstream workload (3.256 TFLOP per
batch in the absorbed form), and the tokenizer's counts
against their closed forms."""
import numpy as np

from latent_attention_jagged_b200 import cost
from workloads import workload
from workloads.tokens import TOKENIZERS


def test_upstream_total_matches_independent_figure():
    dims = workload("upstream").dims
    lengths = np.full(64, 1600)
    tot = cost.total_flops(lengths, dims)
    assert abs(tot / 1e12 - 3.256) < 0.001


def test_per_head_form_ratios():
    dims = workload("upstream").dims
    lengths = np.full(8, 1600)
    L = len(dims.keep)
    absorbed = cost.layer_work(lengths, dims, 0)
    per_head = cost.layer_work(lengths, dims, (1 << L) - 1)
    hd, r = dims.heads * dims.d_head, dims.rank
    for a, p in zip(absorbed, per_head):
        # scores and weighted sums over d_h per head instead of r per head
        assert np.isclose(p.flops["attn"] / a.flops["attn"], hd / (dims.heads * r))
        # the K | V up-projection of every key row is added to the latent step
        assert np.isclose(p.flops["kv"] - a.flops["kv"], 2.0 * a.T.sum() * r * 2 * hd)
        # the projections act on h d_h instead of h r columns
        assert np.isclose(p.flops["o"] / a.flops["o"], hd / (dims.heads * r))
        # the FFN is the same in both forms
        assert p.flops["ffn1"] == a.flops["ffn1"] and p.flops["ffn2"] == a.flops["ffn2"]


def test_mixed_forms_pick_per_layer():
    dims = workload("upstream").dims
    lengths = np.full(4, 1600)
    only0 = cost.layer_work(lengths, dims, 1)
    both = cost.layer_work(lengths, dims, (1 << len(dims.keep)) - 1)
    none = cost.layer_work(lengths, dims, 0)
    assert only0[0].flops == both[0].flops
    for l in range(1, len(dims.keep)):
        assert only0[l].flops == none[l].flops


def test_tokenizer_counts_closed_form():
    t = TOKENIZERS["online"]
    # two products: [D_in -> d_hid] and [d_hid -> d], two FLOP per multiply-add
    assert cost.tokenizer_flops(t) == 2 * 256 * 256 + 2 * 256 * 256
    # ids (int32 per field) + the embedding row read + the token written, bf16
    assert cost.tokenizer_bytes(t) == 4 * 5 + 2 * 256 + 2 * 256
    tiny = TOKENIZERS["tiny"]                     # fp32 storage
    assert cost.tokenizer_bytes(tiny) == 4 * 5 + 4 * 48 + 4 * 64
