"""Throughput benchmark of the LLaTTE sequence-module forward (user-seqs/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload online|upstream|sweepL|skewed]

One step = one whole forward pass (plan, gather, every layer's KV latent,
absorbed queries, latent attention, output projection + norm, FFN + norm,
readout) over one batch of the workload, inputs resident in HBM.  L2 is
flushed (a 256 MiB write) before every timed step, outside the timed events.
Multi-GPU: one process per GPU; a global batch of N x B users is split by
user (longest-processing-time first on per-user FLOPs), weights replicated,
no collective on the data path: weak scaling.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference there is) on
the host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import draw_lengths, make_event_ages, make_inputs, workload  # noqa: E402
from latent_attention_jagged_b200.sharding import shard_batch  # noqa: E402

# ncu-measured DRAM traffic per launch (bytes, mean over one forward's layers)
# of a dominant kernel, keyed by (step, workload, MLA form), each with the
# kernel sources it was taken on and their hash: the bench reports the figure
# only while those sources are unchanged (null otherwise).  The captures are
# summarised under profiles/.
TRAFFIC = {
    # fused FFN, online (B = 256): the four layers' launches of one forward,
    # DRAM read + write 130.6 MB in all
    ("ffn", "online", "absorbed"): {"bytes": 32.6e6, "sha16": "33cec15c170da4d5"},
    # per-head attention, upstream: captured at B = 16 (222.8 MB over the eight
    # layers' launches), scaled by the users (x 4: every launch's key and query
    # tiles grow in proportion)
    ("attn", "upstream", "per_head"): {"bytes": 111.4e6, "sha16": "f2260204a05194e5"},
}
KERNEL_SOURCES = {
    "ffn": ["ffn_pair_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
    "attn": ["attn_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
    # MLA's per-head form runs its own attention kernel
    ("attn", "per_head"): ["attn_heads_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
    "o": ["gemm_sm100.cu", "gemm_pair_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
    "ffn2": ["gemm_sm100.cu", "gemm_pair_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
    "kv": ["gemm_sm100.cu", "tc_common.cuh", "tc_epilogue.cuh"],
}


def sources_hash(step: str, form: str = "absorbed") -> str:
    import hashlib
    hsh = hashlib.sha256()
    for name in KERNEL_SOURCES.get((step, form), KERNEL_SOURCES.get(step, [])):
        with open(os.path.join(ROOT, "latent_attention_jagged_b200", "csrc", name), "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()[:16]


def traffic_of(step: str, workload_name: str, form: str):
    t = TRAFFIC.get((step, workload_name, form))
    if t is None or t["sha16"] != sources_hash(step, form):
        return None
    return t["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    # the profiling recipe's figures for this pool (burst; sustained under the power cap)
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"llatte_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "samples": len(rows),
                "reasons": reasons}


def gpu_identifier(local_rank: int) -> str:
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[local_rank] if vis else str(local_rank)


def cpu_baseline_sample(inp, budget_s: float):
    """Time the oracle on the first users until the budget is used."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    done = 0
    while done < inp.batch and time.perf_counter() - t0 < budget_s:
        oracle.forward(inp, users=[done])
        done += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "user-seqs/s", "cores": int(cores), "kind": "oracle",
            "sample": f"first {done} of {inp.batch} users of one batch, fp64 NumPy oracle "
                      f"(absorbed form), {dt:.1f} s"}


def run_reference(args, wl):
    """Reference arm: the fp64 oracle on host cores, bounded sample per step."""
    inp = make_inputs(wl)
    budget = float(os.environ.get("LLATTE_REF_STEP_S", "3.0"))
    for _ in range(args.warmup):
        cpu_baseline_sample(inp, min(budget, 1.0))
    vals, samples = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cb = cpu_baseline_sample(inp, budget)
        vals.append(cb["value"])
        samples.append(cb)
    wall = time.perf_counter() - t0
    value = float(np.mean(vals))
    cb = dict(samples[-1])
    cb["value"] = value
    line = {
        "impl": "reference", "metric": "user-seqs/s", "value": value, "unit": "user-seqs/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": wl.batch, "seq_len": wl.lengths,
                   "parallelism": "host cores"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "user-seqs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="online")
    ap.add_argument("--second", default="upstream,upstream_abs,sweep400,sweep1600,skewed",
                    help="further workloads measured in the same run, comma-separated "
                         "('' = none)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attn-form", type=int, default=None, choices=[0, 1, 2],
                    help="MLA form on the GPU: 0 auto, 1 absorbed, 2 per head (default: the "
                         "workload's)")
    ap.add_argument("--export-layer", type=int, default=-1,
                    help="also export the attention statistics of this layer in every step")
    ap.add_argument("--batch", type=int, default=None,
                    help="users per batch instead of the workload's (a smaller case for "
                         "profiler captures; the JSON line then names that batch)")
    ap.add_argument("--tokenize", action="store_true",
                    help="each step also builds the history tokens from action ids with the "
                         "MLP_act tokenizer (per-field embedding tables) before the forward")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every kernel eagerly instead of replaying one CUDA graph")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = workload(args.workload)
    if args.attn_form is not None:
        import dataclasses
        wl = dataclasses.replace(wl, dims=dataclasses.replace(wl.dims, attn_form=args.attn_form))
    if args.batch is not None:
        import dataclasses
        wl = dataclasses.replace(wl, batch=int(args.batch))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from latent_attention_jagged_b200 import Llatte, cost

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def rank_inputs(wl):
        """N = 1: the workload's batch.  N > 1: one global batch of N x B users
        (lengths from the workload's law), split by LPT on per-user FLOPs; each
        rank draws the tokens of its own users, all ranks share the weights."""
        if world == 1:
            return make_inputs(wl)
        rng = np.random.Generator(np.random.PCG64(wl.seed))
        lengths = draw_lengths(wl.lengths, wl.batch * world, rng)
        offsets = np.zeros(lengths.shape[0] + 1, dtype=np.int64)
        np.cumsum(lengths, out=offsets[1:])
        shard = shard_batch(offsets, wl.dims, world)[rank]
        inp = make_inputs(wl, lengths=lengths[shard.users], seed=wl.seed + 1000 + rank)
        shared = make_inputs(wl, lengths=np.zeros(1, dtype=np.int64), seed=wl.seed)
        inp.layers, inp.W_e, inp.summaries = shared.layers, shared.W_e, shared.summaries
        return inp

    def measure(wl, steps, warmup, sample_clocks):
        inp = rank_inputs(wl)
        dt = torch.bfloat16 if inp.dims.dtype == "bf16" else torch.float32
        h = Llatte(inp.dims, inp.layers, inp.W_e, max_batch=inp.batch,
                   max_len=int(inp.lengths.max()), summaries=inp.summaries)
        values = torch.from_numpy(inp.values).cuda().to(dt)
        offsets = torch.from_numpy(inp.offsets).cuda()
        ctx = torch.from_numpy(inp.ctx).cuda().to(dt) if inp.dims.d_ctx else None
        cand = torch.from_numpy(inp.cand).cuda().to(dt) if inp.dims.n_q else None
        out = torch.empty(h.out_shape(inp.batch), dtype=torch.float32, device="cuda")
        stream = torch.cuda.current_stream()
        # event ages: the timestamp code's input (d_time > 0), and the hour bins
        # of the optional attention statistics of one layer's query tokens
        ages = None
        if inp.event_age is not None:
            ages = torch.from_numpy(inp.event_age).cuda()
        elif args.export_layer >= 0:
            ages = torch.from_numpy(make_event_ages(inp.lengths, seed=wl.seed + 77)).cuda()

        # optional action tokenizer: the step starts from per-field ids
        tok = ids = None
        if args.tokenize:
            from latent_attention_jagged_b200 import Tokenizer
            from workloads.tokens import TOKENIZERS, make_token_inputs
            tdims = next((t for t in TOKENIZERS.values()
                          if t.d == inp.dims.d and t.dtype == inp.dims.dtype), None)
            if tdims is None:
                raise SystemExit(f"no tokenizer workload of width {inp.dims.d}")
            ti = make_token_inputs(tdims, int(inp.offsets[-1]), seed=wl.seed + 501)
            tok_tables = [torch.from_numpy(t).cuda().to(dt).contiguous() for t in ti.tables]
            tok = Tokenizer(tok_tables, ti.W_a1, ti.W_a2, dtype=tdims.dtype,
                            max_events=max(1, int(inp.offsets[-1])))
            ids = torch.from_numpy(ti.ids).cuda()

        # device buffers of one step (a second set serves the end-to-end loop)
        buf0 = dict(values=values, offsets=offsets, ctx=ctx, cand=cand, ages=ages, ids=ids,
                    out=out)

        def fwd_on(b):
            if tok is not None:
                tok(b["ids"], out=b["values"])
            if args.export_layer >= 0:
                h.forward_export(b["values"], b["offsets"], b["ctx"], b["cand"],
                                 layer=args.export_layer, n_k=11, event_age=b["ages"],
                                 n_hours=168, out=b["out"])
            else:
                h.forward(b["values"], b["offsets"], b["ctx"], b["cand"], out=b["out"],
                          event_age=b["ages"])

        def fwd():
            fwd_on(buf0)

        def capture(b):
            # the whole forward as one CUDA graph (no host work between kernels)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fwd_on(b)
            g.replay()
            torch.cuda.synchronize()
            return g

        for _ in range(warmup):
            fwd()
        torch.cuda.synchronize()
        assert h.status() == 0, "device status word set during warm-up"
        graph = capture(buf0) if args.graph else None

        def step():
            if graph is not None:
                graph.replay()
            else:
                fwd()

        # ---- device-resident timing
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        sampler = ClockSampler(gpu_identifier(local)) if sample_clocks else None
        if sampler:
            sampler.start()
        barrier()
        torch.cuda.synchronize()
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = sampler.stop() if sampler else None
        ms = sum(a.elapsed_time(b) for a, b in ev)
        ms = max_over_ranks(ms)
        users_all = inp.batch
        if world > 1:
            t = torch.tensor([inp.batch], dtype=torch.int64, device="cuda")
            dist.all_reduce(t)
            users_all = int(t.item())
        value = users_all * steps / (ms / 1e3)

        # ---- per-step timing (same loop, profiling events inside the library)
        h.profile_reset()
        h.set_profiling(True)
        prof_steps = max(3, min(steps, 50))
        for _ in range(prof_steps):
            flush.fill_(1)
            fwd()
        torch.cuda.synchronize()
        prof = h.profile()
        h.set_profiling(False)
        launches_per_fwd = sum(v["launches"] for v in prof.values()) / prof_steps
        tok_res = None
        if tok is not None:
            # the tokenizer alone, timed the same way
            evt = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(prof_steps)]
            for a, b in evt:
                flush.fill_(1)
                a.record(stream)
                tok(ids, out=values)
                b.record(stream)
            torch.cuda.synchronize()
            t_ms = sum(a.elapsed_time(b) for a, b in evt) / prof_steps
            n_ev = int(inp.offsets[-1])
            t_flops = n_ev * cost.tokenizer_flops(tdims)
            t_bytes = n_ev * cost.tokenizer_bytes(tdims)
            # the embedding gather, then the fused FFN kernel (D_in = d = 256 in
            # bf16) or two GEMMs
            fused_mlp = (tdims.dtype == "bf16" and tdims.d_in == 256 and tdims.d == 256
                         and tdims.d_hid % 128 == 0)
            tok_launches = 2 if fused_mlp else 3
            tok_res = {"ms": t_ms, "events": n_ev, "launches": tok_launches,
                       "tensor_cores": tok.uses_tensor_cores(),
                       "achieved_tflops": t_flops / (t_ms / 1e3) / 1e12,
                       "frac_of_tensor_peak": t_flops / (t_ms / 1e3) / 1e12
                       / peaks["bf16_tflops"],
                       "achieved_gbs": t_bytes / (t_ms / 1e3) / 1e9,
                       "frac_of_hbm": t_bytes / (t_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                       "algorithmic_flops": t_flops, "algorithmic_bytes": t_bytes}
            launches_per_fwd += tok_launches

        # ---- end to end: pinned host inputs -> device -> forward -> host output,
        # double-buffered: step i's inputs are copied in on a copy stream while
        # step i - 1 computes, and its result is copied out while step i + 1
        # computes.  Every step's copies are inside the timed region, which
        # runs from before the first copy-in to after the last copy-out; the L2
        # flush before each step's forward is inside it too.
        # (with the tokenizer the host sends the action ids instead of the tokens)
        def clone_set(b):
            return {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in b.items()}

        bufs = [buf0, clone_set(buf0)]
        graphs = [graph, capture(bufs[1]) if args.graph else None]
        src_names = ["ids" if tok is not None else "values", "offsets", "ctx", "cand"]
        if inp.event_age is not None:
            src_names.append("ages")
        host = {"values": torch.from_numpy(inp.values).to(dt),
                "ids": ids.cpu() if tok is not None else None,
                "offsets": torch.from_numpy(inp.offsets),
                "ctx": torch.from_numpy(inp.ctx).to(dt) if inp.dims.d_ctx else None,
                "cand": torch.from_numpy(inp.cand).to(dt) if inp.dims.n_q else None,
                "ages": torch.from_numpy(inp.event_age) if inp.event_age is not None else None}
        host = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
        hout = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        cs = torch.cuda.Stream()
        e2e_steps = max(3, min(steps, 50))
        EV = lambda: torch.cuda.Event()
        h2d_done, comp_done, d2h_done = [EV(), EV()], [EV(), EV()], [EV(), EV()]
        t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        t_begin.record(cs)
        for i in range(e2e_steps):
            k = i % 2
            b = bufs[k]
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(comp_done[k])          # step i - 2 has read these inputs
                for name in src_names:
                    if host[name] is not None and b[name] is not None:
                        b[name].copy_(host[name], non_blocking=True)
                h2d_done[k].record(cs)
            stream.wait_event(h2d_done[k])
            if i >= 2:
                stream.wait_event(d2h_done[k])           # step i - 2's result is out
            flush.fill_(1)
            if graphs[k] is not None:
                graphs[k].replay()
            else:
                fwd_on(b)
            comp_done[k].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(comp_done[k])
                hout[k].copy_(b["out"], non_blocking=True)
                d2h_done[k].record(cs)
        t_end.record(cs)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(t_begin.elapsed_time(t_end))
        h2d = sum(host[n].numel() * host[n].element_size() for n in src_names
                  if host[n] is not None)
        # the host link alone: one step's host-to-device copies (the same pinned
        # buffers, nothing else on the GPU), and one 256 MiB pinned copy
        def copy_ms(fn, reps=5):
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fn()
            torch.cuda.synchronize()
            ea.record(cs)
            for _ in range(reps):
                fn()
            eb.record(cs)
            torch.cuda.synchronize()
            return ea.elapsed_time(eb) / reps

        def step_copies():
            with torch.cuda.stream(cs):
                for name in src_names:
                    if host[name] is not None and bufs[0][name] is not None:
                        bufs[0][name].copy_(host[name], non_blocking=True)

        big_h = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
        big_d = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def big_copy():
            with torch.cuda.stream(cs):
                big_d.copy_(big_h, non_blocking=True)

        ms_h2d = copy_ms(step_copies)
        ms_big = copy_ms(big_copy, reps=3)
        del big_h, big_d
        e2e = {"value": users_all * e2e_steps / (ms_e2e / 1e3), "unit": "user-seqs/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(hout[0].numel() * 4),
               "pipeline": "double-buffered: copies of step i overlap compute of step i - 1",
               "steps": e2e_steps,
               "h2d_ms_per_step": ms_h2d, "h2d_gbs": h2d / (ms_h2d / 1e3) / 1e9,
               "link_peak_gbs": (256 << 20) / (ms_big / 1e3) / 1e9,
               "link_note": "h2d_gbs: one step's input copies alone from pinned host memory; "
                            "link_peak_gbs: one 256 MiB pinned host-to-device copy"}
        assert h.status() == 0
        for g in graphs:
            del g
        graphs = None

        # ---- roofline of every step, and of the dominant one (largest device
        # time): the slower of its algorithmic FLOPs at the burst bf16 tensor
        # peak (the kernels run at full clock inside a step of milliseconds)
        # and its algorithmic bytes at the HBM bandwidth
        ph = h.per_head_layers()              # layers in MLA's per-head form: their own work
        flops = cost.flops_by_step(inp.lengths, inp.dims, ph)
        nbytes = cost.bytes_by_step(inp.lengths, inp.dims, ph)
        peak = peaks["bf16_tflops"]
        steps_roof = {}
        for k, v in prof.items():
            if not v["calls"]:
                continue
            ms_k = v["ms"] / prof_steps
            r = cost.step_roofline(flops.get(k, 0.0), nbytes.get(k, 0.0), ms_k, peak,
                                   peaks["hbm_gbs"])
            r["launches"] = v["launches"] / prof_steps
            steps_roof[k] = {kk: (round(vv, 5) if isinstance(vv, float) else vv)
                             for kk, vv in r.items()}
        dom = max((k for k in prof if k in flops and prof[k]["calls"]),
                  key=lambda k: prof[k]["ms"])
        dom_ms = prof[dom]["ms"] / max(1, prof[dom]["calls"])       # per launch of the step
        per_launch_flops = flops[dom] / (prof[dom]["calls"] / prof_steps)
        achieved = per_launch_flops / (dom_ms / 1e3) / 1e12
        form = "per_head" if ph else "absorbed"
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peaks['source']} burst bf16 (cuBLAS, best of 10)",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "traffic": traffic_of(dom, wl.name, form),
                "traffic_sources_sha16": sources_hash(dom, form),
                "flops_per_launch": per_launch_flops, "ms_per_launch": dom_ms,
                "bytes_per_launch": nbytes.get(dom, 0.0) / (prof[dom]["calls"] / prof_steps)}
        # the sequence-summary step (bottleneck GEMM + up-projection), when the
        # workload has one, against HBM: the final rows and both projections
        # read once, the summaries written once
        summary = None
        if prof.get("summary", {}).get("calls"):
            s_ms = prof["summary"]["ms"] / prof["summary"]["calls"]
            s_bytes = cost.summary_bytes(inp.batch, inp.dims)
            summary = {"bound": "hbm", "achieved": s_bytes / (s_ms / 1e3) / 1e9,
                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": s_bytes / (s_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                       "bytes": s_bytes, "ms": s_ms, "launches": prof["summary"]["launches"]
                       / prof["summary"]["calls"],
                       "flops": cost.summary_flops(inp.batch, inp.dims)}
        total_flops = cost.total_flops(inp.lengths, inp.dims, ph)
        step_ms = ms / steps
        whole = {"achieved_tflops": total_flops / (step_ms / 1e3) / 1e12,
                 "frac_of_peak": total_flops / (step_ms / 1e3) / 1e12 / peak,
                 "peak": peak, "flops_per_step": total_flops}
        steps_ms = {k: round(v["ms"] / prof_steps, 4) for k, v in prof.items() if v["calls"]}
        res = dict(value=value, ms=step_ms, e2e=e2e, roofline=roof, whole=whole,
                   clocks=clocks, launches=launches_per_fwd, steps_ms=steps_ms, inp=inp,
                   steps_roof=steps_roof,
                   dtype=inp.dims.dtype, users_all=users_all, summary=summary,
                   per_head_layers=ph, tokenizer=tok_res)
        del graph
        h.close()
        if tok is not None:
            tok.close()
        return res

    main_res = measure(wl, args.steps, args.warmup, sample_clocks=(rank == 0))
    second = []
    for name2 in [w for w in args.second.split(",") if w and w != args.workload]:
        wl2 = workload(name2)
        s_steps = max(5, min(args.steps, 40))
        r2 = measure(wl2, s_steps, args.warmup, sample_clocks=(rank == 0))
        second.append({"workload": wl2.name, "value": r2["value"], "unit": "user-seqs/s",
                       "ms_per_step": r2["ms"], "steps": s_steps, "roofline": r2["roofline"],
                       "whole_step": r2["whole"], "e2e": r2["e2e"], "steps_ms": r2["steps_ms"],
                       "step_roofline": r2["steps_roof"], "clocks": r2["clocks"],
                       "mla_per_head_layers": r2["per_head_layers"]})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(main_res["inp"], args.cpu_budget)

    if rank == 0:
        inp = main_res["inp"]
        line = {
            "metric": "user-seqs/s", "value": main_res["value"], "unit": "user-seqs/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": main_res["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": main_res["dtype"], "data": "synthetic",
            "config": {"workload": wl.name, "global_batch": main_res["users_all"],
                       "seq_len": list(wl.lengths), "d": inp.dims.d, "layers": inp.dims.n_layers,
                       "parallelism": f"users sharded by LPT on FLOPs, dp{world}",
                       "l2": "flushed (256 MiB write) before every timed step",
                       "launch": "one CUDA graph replay per step" if args.graph else "eager",
                       "attn_export_layer": args.export_layer if args.export_layer >= 0 else None,
                       "mla_per_head_layers": main_res["per_head_layers"]},
            "roofline": main_res["roofline"],
            "whole_step": main_res["whole"],
            "cpu_baseline": cpu,
            "e2e": main_res["e2e"],
            "gpu_launches": int(round(main_res["launches"] * args.steps)),
            "clocks": main_res["clocks"],
            "steps_ms": main_res["steps_ms"],
            "step_roofline": main_res["steps_roof"],
            "summary": main_res["summary"],
            "tokenizer": main_res["tokenizer"],
            "second": second or None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
