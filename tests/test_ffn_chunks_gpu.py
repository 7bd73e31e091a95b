"""GPU parity of the fused FFN block at d = 256 for hidden widths other than
the 4d of the main workloads.  The fused kernel walks the hidden layer in
128-wide chunks, two TMEM buffers deep, each SM pair starting at its own
chunk and wrapping around; the number of chunks NC = hidden / 128 decides
which of its branches run (NC = 1: a single chunk per tile, no second
buffer; NC = 2: no first product issued between the second products; odd NC:
the rotation wraps unevenly).  The forward's FFN (W2 SiLU(W1 z) with the
residual, RMSNorm and pyramid scatter; LLaTTE notes, huaxiaozhuan.com,
appendix A.2 display) runs here with hidden = d, 2d and 3d, and the action
tokenizer's MLP (appendix A.2 item 1, the same kernel storing the rows as
they are) with hidden 128 and 384, each against the fp64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.tokenizer import action_tokens
from latent_attention_jagged_b200 import Tokenizer
from workloads import Workload, make_inputs, workload
from workloads.tokens import TOKENIZERS, make_token_inputs

from gpu_harness import assert_close, make_handle, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mult", [1, 2, 3])
def test_forward_fused_ffn_hidden_widths(mult):
    base = workload("online")
    inp = make_inputs(Workload(name=f"online_ffn{mult}", dims=dataclasses.replace(base.dims, ffn_mult=mult),
                               batch=40, lengths=("uniform", 100, 400), seed=31 + mult, semantic=True))
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    h.set_profiling(True)
    out = h.forward(values, offsets, ctx, cand)
    torch.cuda.synchronize()
    prof = h.profile()
    h.set_profiling(False)
    assert h.status() == 0
    # the fused kernel ran (the separate FFN-up / FFN-down GEMMs did not)
    assert prof["ffn"]["calls"] > 0 and prof["ffn1"]["calls"] == 0
    assert_close(out.cpu().numpy().astype(np.float64), oracle.forward(inp), "bf16",
                 f"fused FFN, hidden {mult}d")


@pytest.mark.parametrize("d_hid", [128, 384])
def test_tokenizer_fused_mlp_hidden_widths(d_hid):
    # the online token shapes (D_in = d = 256, bf16) with smaller item table
    dims = dataclasses.replace(TOKENIZERS["online"], d_hid=d_hid, rows=(64, 20000, 32, 256, 4096))
    n = 3 * 256 * 74 + 37                    # several tiles per SM pair and a ragged tail
    ti = make_token_inputs(dims, n, seed=23)
    tables = [torch.from_numpy(t).cuda().to(torch.bfloat16).contiguous() for t in ti.tables]
    tok = Tokenizer(tables, ti.W_a1, ti.W_a2, dtype="bf16", max_events=n)
    assert tok.uses_tensor_cores()
    x = tok(torch.from_numpy(ti.ids).cuda())
    torch.cuda.synchronize()
    assert tok.status() == 0
    ref = action_tokens(ti.ids, ti.tables, ti.W_a1, ti.W_a2)
    assert_close(x.float().cpu().numpy().astype(np.float64), ref, "bf16", f"tokenizer MLP, hidden {d_hid}")
    tok.close()
