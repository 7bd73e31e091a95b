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


def test_step_bytes_closed_forms():
    """The HBM byte model on a fixed-length batch, counted by hand: one layer,
    every history row kept, bf16 storage with fp16 residual copies."""
    from workloads import Dims
    dims = Dims(d=256, heads=4, d_head=64, rank=128, d_ctx=64, n_q=8, keep=(100,))
    B, T = 3, 100
    b = cost.bytes_by_step(np.full(B, T), dims)
    d, hr, r, q = 256, 4 * 128, 128, T + 8
    rows_T, rows_q = B * T, B * q
    # gather: events + query tokens read, key rows + query rows written, row maps
    assert b["gather"] == 2 * (rows_T * d + B * 8 * d) + 2 * (rows_T * d + rows_q * d) + 4 * rows_q
    assert b["kv"] == 2 * rows_T * d + 2 * r * d + 2 * rows_T * r
    assert b["q"] == 2 * rows_q * d + 2 * hr * (d + 64) + 4 * B * hr + 2 * rows_q * hr
    assert b["attn"] == 2 * rows_q * hr + 2 * rows_T * r + 2 * rows_q * hr
    assert b["o"] == 2 * rows_q * hr + 2 * rows_q * d + 2 * d * hr + 2 * rows_q * d
    # last layer: the fp32 candidate rows are the output
    assert b["ffn"] == 2 * rows_q * d + 2 * 2 * 1024 * d + 4 * B * 8 * d
    # per-head form: the K | V rows are written by the latent step and read by attention
    p = cost.bytes_by_step(np.full(B, T), dims, per_head_layers=1)
    assert p["kv"] - b["kv"] == 2 * rows_T * r + 2 * 2 * 256 * r + 2 * rows_T * 2 * 256
    assert p["attn"] == 2 * rows_q * 256 + 2 * rows_T * 2 * 256 + 2 * rows_q * 256


def test_step_roofline_takes_the_slower_bound():
    # 1 TFLOP at 1000 TF/s = 1 ms; 1 GB at 1000 GB/s = 1 ms; measured 2 ms
    r = cost.step_roofline(1e12, 5e8, 2.0, 1000.0, 1000.0)
    assert r["bound"] == "tensor" and np.isclose(r["frac"], 0.5)
    assert np.isclose(r["frac_hbm"], 0.25)
    r = cost.step_roofline(1e9, 4e9, 8.0, 1000.0, 1000.0)
    assert r["bound"] == "hbm" and np.isclose(r["frac"], 0.5)
