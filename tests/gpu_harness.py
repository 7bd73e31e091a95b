"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the library through its C ABI, and measure the error against the oracle."""
from __future__ import annotations

import numpy as np
import torch

import parity_log
from latent_attention_jagged_b200 import Llatte

# Tolerances fixed by the target: bf16 max-abs <= 3e-2 and relative L2 <= 1e-2;
# the fp32 configuration max-abs <= 1e-4.
TOL = {"bf16": dict(max_abs=3e-2, rel_l2=1e-2), "fp32": dict(max_abs=1e-4, rel_l2=1e-5)}
# Attention-probability statistics (sums of probabilities, each in [0, 1],
# accumulated in fp32): in a bf16 forward their error comes from the scores
# the probabilities are made of (bf16 operands), not from the fp32 sums, so
# they get a bound of their own, a third of the row-output bound; the
# largest error measured on any tested workload is 2.9e-3 max-abs and 2.4e-3
# rel-L2.  The fp32 forward keeps the fp32 bound.
EXPORT_TOL = {"bf16": dict(max_abs=1e-2, rel_l2=5e-3), "fp32": TOL["fp32"]}


def to_device(inp):
    dt = torch.bfloat16 if inp.dims.dtype == "bf16" else torch.float32
    dev = "cuda"
    values = torch.from_numpy(inp.values).to(dev).to(dt).contiguous()
    offsets = torch.from_numpy(inp.offsets).to(dev)
    ctx = torch.from_numpy(inp.ctx).to(dev).to(dt).contiguous() if inp.dims.d_ctx else None
    cand = torch.from_numpy(inp.cand).to(dev).to(dt).contiguous() if inp.dims.n_q else None
    return values, offsets, ctx, cand


def make_handle(inp, max_batch=None, max_len=None, max_total=0):
    B = inp.batch
    ml = int(inp.lengths.max()) if max_len is None and B else (max_len or 1)
    return Llatte(inp.dims, inp.layers, inp.W_e, max_batch=max_batch or max(B, 1),
                  max_len=ml, max_total=max_total, summaries=inp.summaries)


def ages_on_device(inp):
    a = getattr(inp, "event_age", None)
    return torch.from_numpy(a).cuda() if a is not None else None


def run(inp, handle=None, **kw):
    h = handle or make_handle(inp, **kw)
    values, offsets, ctx, cand = to_device(inp)
    out = h.forward(values, offsets, ctx, cand, event_age=ages_on_device(inp))
    torch.cuda.synchronize()
    return h, out.cpu().numpy().astype(np.float64)


def errors(gpu: np.ndarray, ref: np.ndarray):
    diff = gpu - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.sqrt((ref ** 2).sum()))
    rel = float(np.sqrt((diff ** 2).sum()) / den) if den > 0 else float(np.sqrt((diff ** 2).sum()))
    return max_abs, rel


def assert_close(gpu, ref, dtype, what="", tol=None):
    """Max-abs and relative-L2 error of gpu against ref within the tolerance of
    the storage type (or `tol`); the errors are returned and recorded for the
    session's parity summary."""
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    ma, rl = errors(gpu, ref)
    tol = tol or TOL[dtype]
    parity_log.record(what, ma, rl, tol, dtype)
    assert ma <= tol["max_abs"] and rl <= tol["rel_l2"], \
        f"{what}: max_abs={ma:.3e} (tol {tol['max_abs']}) rel_l2={rl:.3e} (tol {tol['rel_l2']})"
    return ma, rl


def sample_users(lengths, first=8):
    """The first users, plus the longest and the shortest of the batch."""
    lengths = np.asarray(lengths)
    users = list(range(min(first, len(lengths))))
    for u in (int(np.argmax(lengths)), int(np.argmin(lengths))):
        if u not in users:
            users.append(u)
    return users
