"""GPU parity of the action tokenizer MLP_act (LLaTTE notes, appendix A.2
item 1 "Action Embeddings"): per-field embedding gather plus the two MLP
GEMMs, through the C ABI, against the fp64 oracle; then tokens fed to the
forward pass against the oracle forward on the oracle's tokens."""
import numpy as np
import pytest
import torch

import oracle
from oracle.tokenizer import action_tokens
from latent_attention_jagged_b200 import Llatte, Tokenizer
from latent_attention_jagged_b200.binding import DEV_BAD_ID
from workloads import make_inputs, workload
from workloads.tokens import TOKENIZERS, make_token_inputs

from gpu_harness import assert_close, sample_users, to_device

pytestmark = pytest.mark.gpu


def _tokenizer(ti, max_events):
    dt = torch.bfloat16 if ti.dims.dtype == "bf16" else torch.float32
    tables = [torch.from_numpy(t).cuda().to(dt).contiguous() for t in ti.tables]
    return Tokenizer(tables, ti.W_a1, ti.W_a2, dtype=ti.dims.dtype, max_events=max_events), tables


@pytest.mark.parametrize("name,n,tc", [("tiny", 517, False), ("odd_bf16", 1000, False),
                                       ("online", 64 * 1024 + 37, True)])
def test_tokens_match_oracle(name, n, tc):
    ti = make_token_inputs(TOKENIZERS[name], n, seed=21)
    tok, _tables = _tokenizer(ti, max_events=n + 100)
    assert tok.uses_tensor_cores() == tc
    ids = torch.from_numpy(ti.ids).cuda()
    x = tok(ids)
    torch.cuda.synchronize()
    assert tok.status() == 0
    ref = action_tokens(ti.ids, ti.tables, ti.W_a1, ti.W_a2)
    assert_close(x.float().cpu().numpy().astype(np.float64), ref, ti.dims.dtype, name)
    # a second call on a shorter batch (ragged tail of a tile), then n = 0
    m = n // 3 + 5
    y = tok(ids[:m].contiguous())
    z = tok(ids[:0].contiguous())
    torch.cuda.synchronize()
    assert tok.status() == 0 and z.shape == (0, ti.dims.d)
    assert torch.equal(y, x[:m])
    tok.close()


def test_bad_ids_flagged_and_read_as_zero_embeddings():
    ti = make_token_inputs(TOKENIZERS["online"], 3000, seed=22)
    tok, _tables = _tokenizer(ti, max_events=3000)
    ids = ti.ids.copy()
    bad_rows = [5, 700, 2999]
    ids[5, 1] = ti.dims.rows[1]          # one past the item table
    ids[700, 0] = -3
    ids[2999, 4] = 1 << 30
    x = tok(torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    assert tok.status() & DEV_BAD_ID
    assert tok.status() == 0             # read-and-clear
    # oracle: the offending fields index an appended zero row
    tables = [np.concatenate([t, np.zeros((1, t.shape[1]), t.dtype)]) for t in ti.tables]
    fixed = ids.copy()
    for r, f in ((5, 1), (700, 0), (2999, 4)):
        fixed[r, f] = ti.dims.rows[f]
    ref = action_tokens(fixed, tables, ti.W_a1, ti.W_a2)
    got = x.float().cpu().numpy().astype(np.float64)
    assert_close(got[bad_rows], ref[bad_rows], "bf16", "bad ids")
    assert_close(got, ref, "bf16", "all rows")
    tok.close()


def test_tokens_feed_the_forward_pass():
    inp = make_inputs(workload("online"), batch=12)
    n = int(inp.offsets[-1])
    ti = make_token_inputs(TOKENIZERS["online"], n, seed=23)
    tok, _tables = _tokenizer(ti, max_events=n)
    _, offsets, ctx, cand = to_device(inp)
    values = tok(torch.from_numpy(ti.ids).cuda())
    h = Llatte(inp.dims, inp.layers, inp.W_e, max_batch=inp.batch,
               max_len=int(inp.lengths.max()))
    out = h.forward(values, offsets, ctx, cand)
    torch.cuda.synchronize()
    assert h.status() == 0 and tok.status() == 0
    # the oracle forward on the oracle's fp64 tokens
    inp.values = action_tokens(ti.ids, ti.tables, ti.W_a1, ti.W_a2)
    users = sample_users(inp.lengths, 12)
    ref = oracle.forward(inp, users=users)
    assert_close(out.cpu().numpy().astype(np.float64)[users], ref, "bf16", "tokens -> forward")
    h.close()
    tok.close()
