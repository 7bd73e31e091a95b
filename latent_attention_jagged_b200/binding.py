"""ctypes binding of libllatte.so: the same entry points as include/llatte.h,
with argument marshalling from torch tensors (device memory and streams only;
every step of the forward runs in the library's kernels).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libllatte.so")
MAX_LAYERS = 16
STEPS = ("plan", "gather", "ctx_bias", "kv", "q", "attn", "o", "ffn1", "ffn2", "readout", "ffn",
         "summary", "attn_export")

LLATTE_OK, LLATTE_ERR_ARG, LLATTE_ERR_UNSUPPORTED, LLATTE_ERR_CUDA, LLATTE_ERR_OOM, \
    LLATTE_ERR_DEVICE = 0, -1, -2, -3, -4, -5
LLATTE_BF16, LLATTE_FP32 = 0, 1
DEV_BAD_OFFSETS, DEV_TOO_LONG, DEV_TOO_MANY_ROWS, DEV_TIMEOUT, DEV_BAD_ID = 1, 2, 4, 8, 16


class LlatteError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} ({code})")


class llatte_dims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("d_ctx", ctypes.c_int32), ("n_q", ctypes.c_int32),
                ("n_layers", ctypes.c_int32), ("keep", ctypes.c_int32 * MAX_LAYERS),
                ("d_out", ctypes.c_int32), ("ffn_mult", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("kv_norm", ctypes.c_int32), ("eps", ctypes.c_float),
                ("max_batch", ctypes.c_int32), ("max_len", ctypes.c_int64),
                ("max_total", ctypes.c_int64), ("n_sum", ctypes.c_int32),
                ("sum_rank", ctypes.c_int32), ("d_seq", ctypes.c_int32),
                ("q_rank", ctypes.c_int32), ("d_time", ctypes.c_int32),
                ("attn_form", ctypes.c_int32)]


LAYER_KEYS = ("W_dkv", "g_kv", "W_q", "W_uk", "W_uv", "W_o", "g1", "W1", "W2", "g2",
              "W_dq", "g_q", "W_uq")


class llatte_layer_w(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in LAYER_KEYS]


SUMMARY_KEYS = ("W_down", "W_up")


class llatte_summary_w(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in SUMMARY_KEYS]


class llatte_batch(ctypes.Structure):
    _fields_ = [("values", ctypes.c_void_p), ("offsets", ctypes.c_void_p), ("B", ctypes.c_int32),
                ("context", ctypes.c_void_p), ("cand", ctypes.c_void_p),
                ("event_age", ctypes.c_void_p)]


class llatte_tok_dims(ctypes.Structure):
    _fields_ = [("n_fields", ctypes.c_int32), ("rows", ctypes.c_int64 * 8),
                ("width", ctypes.c_int32 * 8), ("d_hid", ctypes.c_int32), ("d", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("max_events", ctypes.c_int64)]


class llatte_tok_w(ctypes.Structure):
    _fields_ = [("tables", ctypes.c_void_p * 8), ("W_a1", ctypes.c_void_p),
                ("W_a2", ctypes.c_void_p)]


class llatte_attn_export(ctypes.Structure):
    _fields_ = [("layer", ctypes.c_int32), ("n_k", ctypes.c_int32), ("n_hours", ctypes.c_int32),
                ("event_age", ctypes.c_void_p), ("recent", ctypes.c_void_p),
                ("topk", ctypes.c_void_p), ("hours", ctypes.c_void_p)]


EXPORTS = ("llatte_create", "llatte_forward", "llatte_plan_export", "llatte_get_status",
           "llatte_workspace_bytes", "llatte_error_string", "llatte_destroy",
           "llatte_set_profiling", "llatte_profile_reset", "llatte_profile_step",
           "llatte_plan_static", "llatte_exp2_eval", "llatte_forward_export",
           "llatte_forward_batch", "llatte_attn_form_mask", "llatte_tokenizer_create",
           "llatte_tokenize", "llatte_tokenizer_get_status", "llatte_tokenizer_uses_tensor_cores",
           "llatte_tokenizer_destroy", "llatte_inject_timeout")
TOK_MAX_FIELDS = 8
PLAN_STATIC_MAX_BATCH = 4096

_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Open libllatte.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with "
                           "`python -m latent_attention_jagged_b200.build`")
    lib = ctypes.CDLL(p)
    P, I32, I64, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    lib.llatte_create.argtypes = [P(VP), P(llatte_dims), P(llatte_layer_w), VP,
                                  P(llatte_summary_w), ctypes.c_int]
    lib.llatte_create.restype = ctypes.c_int
    lib.llatte_forward.argtypes = [VP, VP, VP, I32, VP, VP, VP, VP]
    lib.llatte_forward.restype = ctypes.c_int
    lib.llatte_forward_export.argtypes = [VP, VP, VP, I32, VP, VP, VP, P(llatte_attn_export), VP]
    lib.llatte_forward_export.restype = ctypes.c_int
    lib.llatte_forward_batch.argtypes = [VP, P(llatte_batch), VP, P(llatte_attn_export), VP]
    lib.llatte_forward_batch.restype = ctypes.c_int
    lib.llatte_plan_export.argtypes = [VP, VP, VP]
    lib.llatte_plan_export.restype = ctypes.c_int
    lib.llatte_get_status.argtypes = [VP, P(I32)]
    lib.llatte_get_status.restype = ctypes.c_int
    lib.llatte_workspace_bytes.argtypes = [P(llatte_dims)]
    lib.llatte_workspace_bytes.restype = ctypes.c_size_t
    lib.llatte_error_string.argtypes = [ctypes.c_int]
    lib.llatte_error_string.restype = ctypes.c_char_p
    lib.llatte_destroy.argtypes = [VP]
    lib.llatte_destroy.restype = None
    lib.llatte_set_profiling.argtypes = [VP, ctypes.c_int]
    lib.llatte_set_profiling.restype = ctypes.c_int
    lib.llatte_profile_reset.argtypes = [VP]
    lib.llatte_profile_reset.restype = ctypes.c_int
    lib.llatte_profile_step.argtypes = [VP, ctypes.c_int, P(ctypes.c_char_p),
                                        P(ctypes.c_double), P(I64), P(I64)]
    lib.llatte_profile_step.restype = ctypes.c_int
    lib.llatte_plan_static.argtypes = [P(llatte_dims), VP, I32, VP, VP, VP]
    lib.llatte_plan_static.restype = ctypes.c_int
    lib.llatte_exp2_eval.argtypes = [VP, VP, VP, I64, VP]
    lib.llatte_exp2_eval.restype = ctypes.c_int
    lib.llatte_attn_form_mask.argtypes = [VP, P(ctypes.c_uint32)]
    lib.llatte_attn_form_mask.restype = ctypes.c_int
    lib.llatte_inject_timeout.argtypes = [VP, ctypes.c_int]
    lib.llatte_inject_timeout.restype = ctypes.c_int
    lib.llatte_tokenizer_create.argtypes = [P(VP), P(llatte_tok_dims), P(llatte_tok_w),
                                            ctypes.c_int]
    lib.llatte_tokenizer_create.restype = ctypes.c_int
    lib.llatte_tokenize.argtypes = [VP, VP, I64, VP, VP]
    lib.llatte_tokenize.restype = ctypes.c_int
    lib.llatte_tokenizer_get_status.argtypes = [VP, P(I32)]
    lib.llatte_tokenizer_get_status.restype = ctypes.c_int
    lib.llatte_tokenizer_uses_tensor_cores.argtypes = [VP]
    lib.llatte_tokenizer_uses_tensor_cores.restype = ctypes.c_int
    lib.llatte_tokenizer_destroy.argtypes = [VP]
    lib.llatte_tokenizer_destroy.restype = None
    if path is None:
        _lib = lib
    return lib


def error_string(code: int) -> str:
    try:
        return load_library().llatte_error_string(code).decode()
    except Exception:
        return "unknown"


def make_dims(dims, max_batch: int, max_len: int, max_total: int = 0) -> llatte_dims:
    """Fill the C struct from any object with the Dims attributes."""
    if len(dims.keep) > MAX_LAYERS:
        raise ValueError(f"at most {MAX_LAYERS} layers")
    c = llatte_dims()
    c.d, c.heads, c.d_head, c.rank = dims.d, dims.heads, dims.d_head, dims.rank
    c.d_ctx, c.n_q, c.n_layers = dims.d_ctx, dims.n_q, len(dims.keep)
    for i, k in enumerate(dims.keep):
        c.keep[i] = int(k)
    c.d_out, c.ffn_mult = dims.d_out, dims.ffn_mult
    c.dtype = {"bf16": LLATTE_BF16, "fp32": LLATTE_FP32}[dims.dtype]
    c.kv_norm, c.eps = dims.kv_norm, float(dims.eps)
    c.max_batch, c.max_len, c.max_total = int(max_batch), int(max_len), int(max_total)
    c.n_sum = int(getattr(dims, "n_sum", 0))
    c.sum_rank = int(getattr(dims, "sum_rank", 0))
    c.d_seq = int(getattr(dims, "d_seq", 0))
    c.q_rank = int(getattr(dims, "q_rank", 0))
    c.d_time = int(getattr(dims, "d_time", 0))
    c.attn_form = int(getattr(dims, "attn_form", 0))
    return c


def torch_dtype(dims) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[dims.dtype]


def _host(a, dt: torch.dtype) -> torch.Tensor:
    t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
    return t.detach().to(device="cpu", dtype=dt).contiguous()


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


class Llatte:
    """A forward handle: weights (non-absorbed, pages' layout) are copied and
    absorbed at construction; `forward` runs the whole sequence module."""

    def __init__(self, dims, layers: Sequence[dict], W_e=None, max_batch: int = 1,
                 max_len: int = 0, max_total: int = 0, lib_path: Optional[str] = None,
                 summaries: Optional[Sequence[dict]] = None):
        self.lib = load_library(lib_path)
        self.dims = dims
        self.cdims = make_dims(dims, max_batch, max_len, max_total)
        self.dt = torch_dtype(dims)
        if len(layers) != len(dims.keep):
            raise ValueError("one weight dict per layer is required")
        keep_alive = []
        arr = (llatte_layer_w * len(layers))()
        for i, w in enumerate(layers):
            for k in LAYER_KEYS:
                if w.get(k) is None:         # W_q or the low-rank query's matrices
                    continue
                t = _host(w[k], self.dt)
                keep_alive.append(t)
                setattr(arr[i], k, t.data_ptr())
        we = None
        if dims.d_out:
            we = _host(W_e, self.dt)
            keep_alive.append(we)
        n_sum = int(getattr(dims, "n_sum", 0))
        sarr = None
        if n_sum:
            if summaries is None or len(summaries) != n_sum:
                raise ValueError(f"{n_sum} summary weight dicts are required")
            sarr = (llatte_summary_w * n_sum)()
            for i, w in enumerate(summaries):
                for k in SUMMARY_KEYS:
                    t = _host(w[k], self.dt)
                    keep_alive.append(t)
                    setattr(sarr[i], k, t.data_ptr())
        h = ctypes.c_void_p()
        rc = self.lib.llatte_create(ctypes.byref(h), ctypes.byref(self.cdims), arr,
                                    _ptr(we), sarr, 0)
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_create")
        self.h = h
        self.last_B = 0

    def per_head_layers(self) -> int:
        """Bit l set: layer l runs MLA in its per-head form on this handle."""
        m = ctypes.c_uint32(0)
        rc = self.lib.llatte_attn_form_mask(self.h, ctypes.byref(m))
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_attn_form_mask")
        return int(m.value)

    def inject_timeout(self, enable: bool = True):
        """Failure-detection aid: the forward calls that follow make a bounded
        wait of the per-head attention run out on purpose (status bit
        DEV_TIMEOUT, output unspecified) until switched off again."""
        rc = self.lib.llatte_inject_timeout(self.h, 1 if enable else 0)
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_inject_timeout")

    def workspace_bytes(self) -> int:
        return int(self.lib.llatte_workspace_bytes(ctypes.byref(self.cdims)))

    def out_shape(self, B: int):
        d = self.dims
        if getattr(d, "n_sum", 0):
            return (B, d.n_sum, d.d_seq)
        return (B, d.d_out) if d.d_out else (B, d.n_q, d.d)

    def _check_inputs(self, values, offsets, context, cand, event_age):
        d = self.dims
        B = int(offsets.numel()) - 1
        if B < 0:
            raise ValueError("offsets needs B+1 entries")
        for name, t, dt in (("values", values, self.dt), ("offsets", offsets, torch.int64),
                            ("context", context, self.dt), ("cand", cand, self.dt),
                            ("event_age", event_age, torch.float32)):
            if t is None:
                continue
            if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
        if values.dim() != 2 or values.shape[1] != d.d:
            raise ValueError(f"values must be [rows, {d.d}]")
        if d.d_ctx and (context is None or tuple(context.shape) != (B, d.d_ctx)):
            raise ValueError(f"context must be [{B}, {d.d_ctx}]")
        if d.n_q and (cand is None or tuple(cand.shape) != (B, d.n_q, d.d)):
            raise ValueError(f"cand must be [{B}, {d.n_q}, {d.d}]")
        if getattr(d, "d_time", 0) and (event_age is None or event_age.dim() != 1 or
                                        event_age.shape[0] < values.shape[0]):
            raise ValueError("event_age [rows] (hours before the request) is required")
        return B

    def _out(self, out, B, device):
        if out is None:
            return torch.empty(self.out_shape(B), dtype=torch.float32, device=device)
        if (tuple(out.shape) != self.out_shape(B) or out.dtype != torch.float32
                or not out.is_contiguous()):
            raise ValueError(f"out must be a contiguous float32 {self.out_shape(B)} tensor")
        return out

    def _run(self, values, offsets, context, cand, event_age, out, ex, stream, B):
        if ex is None and event_age is None:
            rc = self.lib.llatte_forward(self.h, _ptr(values), _ptr(offsets), B, _ptr(context),
                                         _ptr(cand), _ptr(out), _stream_ptr(stream))
            what = "llatte_forward"
        else:
            b = llatte_batch(values=values.data_ptr(), offsets=offsets.data_ptr(), B=B,
                             context=context.data_ptr() if context is not None else None,
                             cand=cand.data_ptr() if cand is not None else None,
                             event_age=event_age.data_ptr() if event_age is not None else None)
            rc = self.lib.llatte_forward_batch(self.h, ctypes.byref(b), _ptr(out),
                                               ctypes.byref(ex) if ex is not None else None,
                                               _stream_ptr(stream))
            what = "llatte_forward_batch"
        if rc != LLATTE_OK:
            raise LlatteError(rc, what)
        self.last_B = B

    def forward(self, values: torch.Tensor, offsets: torch.Tensor, context=None, cand=None,
                out: Optional[torch.Tensor] = None, stream=None, event_age=None) -> torch.Tensor:
        """One forward pass.  event_age (float32 [rows], hours before the
        request of every history event) is required when dims.d_time > 0."""
        B = self._check_inputs(values, offsets, context, cand, event_age)
        out = self._out(out, B, values.device)
        if not getattr(self.dims, "d_time", 0):
            event_age = None
        self._run(values, offsets, context, cand, event_age, out, None, stream, B)
        return out

    def forward_export(self, values: torch.Tensor, offsets: torch.Tensor, context=None,
                       cand=None, layer: int = 0, n_k: int = 8, event_age=None,
                       n_hours: int = 0, out: Optional[torch.Tensor] = None, stream=None):
        """Forward plus the attention statistics of `layer`'s query tokens:
        returns (out, recent [B, n_q, h, n_k], topk [B, n_q, h, n_k],
        hours [B, n_q, h, n_hours] or None).  event_age serves both the hour
        bins and, when dims.d_time > 0, the timestamp code."""
        d = self.dims
        B = self._check_inputs(values, offsets, context, cand, event_age)
        dev = values.device
        recent = torch.empty((B, d.n_q, d.heads, n_k), dtype=torch.float32, device=dev)
        topk = torch.empty_like(recent)
        hours = None
        if n_hours:
            if event_age is None:
                raise ValueError("event_age is required for hour bins")
            hours = torch.empty((B, d.n_q, d.heads, n_hours), dtype=torch.float32, device=dev)
        ex = llatte_attn_export(layer=layer, n_k=n_k, n_hours=n_hours,
                                event_age=event_age.data_ptr() if n_hours else None,
                                recent=recent.data_ptr(), topk=topk.data_ptr(),
                                hours=hours.data_ptr() if hours is not None else None)
        out = self._out(out, B, dev)
        self._run(values, offsets, context, cand,
                  event_age if getattr(d, "d_time", 0) else None, out, ex, stream, B)
        return out, recent, topk, hours

    def plan_export(self, stream=None) -> torch.Tensor:
        L, B = len(self.dims.keep), self.last_B
        dst = torch.empty((L, 2, B + 1), dtype=torch.int64, device="cuda")
        rc = self.lib.llatte_plan_export(self.h, _ptr(dst), _stream_ptr(stream))
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_plan_export")
        return dst

    def status(self) -> int:
        v = ctypes.c_int32(0)
        rc = self.lib.llatte_get_status(self.h, ctypes.byref(v))
        if rc not in (LLATTE_OK, LLATTE_ERR_DEVICE):
            raise LlatteError(rc, "llatte_get_status")
        return int(v.value)

    def set_profiling(self, on: bool = True):
        self.lib.llatte_set_profiling(self.h, 1 if on else 0)

    def profile_reset(self):
        self.lib.llatte_profile_reset(self.h)

    def profile(self) -> dict:
        res = {}
        for i in range(len(STEPS)):
            name = ctypes.c_char_p()
            ms = ctypes.c_double()
            nl = ctypes.c_int64()
            nc = ctypes.c_int64()
            rc = self.lib.llatte_profile_step(self.h, i, ctypes.byref(name), ctypes.byref(ms),
                                              ctypes.byref(nl), ctypes.byref(nc))
            if rc != LLATTE_OK:
                raise LlatteError(rc, "llatte_profile_step")
            res[name.value.decode()] = {"ms": ms.value, "launches": nl.value, "calls": nc.value}
        return res

    def close(self):
        if getattr(self, "h", None):
            self.lib.llatte_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def plan_static(dims, offsets: torch.Tensor, max_batch: int, max_len: int, max_total: int = 0,
                stream=None, out: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None):
    """Pyramid plan of one batch through llatte_plan_static, the entry point
    that allocates no device memory (its scratch is a fixed array inside the
    library).  Pass `out` / `status` to reuse caller-owned buffers.  Returns
    (plan [n_layers, 2, B+1] int64, status int32 tensor)."""
    lib = load_library()
    cd = make_dims(dims, max_batch, max_len, max_total)
    B = int(offsets.numel()) - 1
    if not offsets.is_cuda or offsets.dtype != torch.int64 or not offsets.is_contiguous():
        raise ValueError("offsets must be a contiguous CUDA int64 tensor")
    if out is None:
        out = torch.empty((len(dims.keep), 2, B + 1), dtype=torch.int64, device=offsets.device)
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=offsets.device)
    if tuple(out.shape) != (len(dims.keep), 2, B + 1) or out.dtype != torch.int64:
        raise ValueError("out must be int64 [n_layers, 2, B+1]")
    rc = lib.llatte_plan_static(ctypes.byref(cd), _ptr(offsets), B, _ptr(out), _ptr(status),
                                _stream_ptr(stream))
    if rc != LLATTE_OK:
        raise LlatteError(rc, "llatte_plan_static")
    return out, status


def exp2_eval(x: torch.Tensor, with_hw: bool = True, stream=None):
    """2^x through the softmax's FMA-pipe exponential (and, with `with_hw`,
    through the hardware ex2.approx) for a contiguous CUDA float32 tensor."""
    lib = load_library()
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    y_hw = torch.empty_like(x) if with_hw else None
    rc = lib.llatte_exp2_eval(_ptr(x), _ptr(y), _ptr(y_hw), x.numel(), _stream_ptr(stream))
    if rc != LLATTE_OK:
        raise LlatteError(rc, "llatte_exp2_eval")
    return (y, y_hw) if with_hw else y


class Tokenizer:
    """Action tokenizer MLP_act: x_t = W_a2 SiLU(W_a1 [E_1(id_t1); ...; E_F(id_tF)]).

    `tables` are CUDA tensors [rows_f, width_f] in the storage dtype that the
    tokenizer references (not copied): they must stay alive and unchanged.
    W_a1 [d_hid, D_in] and W_a2 [d, d_hid] are copied."""

    def __init__(self, tables, W_a1, W_a2, dtype: str = "bf16", max_events: int = 1 << 20):
        self.lib = load_library()
        self.dt = {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]
        if not 1 <= len(tables) <= TOK_MAX_FIELDS:
            raise ValueError(f"1 .. {TOK_MAX_FIELDS} tables")
        self.tables = []
        for t in tables:
            if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == self.dt
                    and t.dim() == 2 and t.is_contiguous()):
                raise ValueError("tables must be contiguous 2-D CUDA tensors of the storage dtype")
            self.tables.append(t)
        w1, w2 = _host(W_a1, self.dt), _host(W_a2, self.dt)
        c = llatte_tok_dims()
        c.n_fields = len(tables)
        for f, t in enumerate(tables):
            c.rows[f], c.width[f] = int(t.shape[0]), int(t.shape[1])
        c.d_hid, c.d = int(w1.shape[0]), int(w2.shape[0])
        if w1.shape[1] != sum(int(t.shape[1]) for t in tables) or w2.shape[1] != c.d_hid:
            raise ValueError("W_a1 must be [d_hid, sum of widths], W_a2 [d, d_hid]")
        c.dtype = LLATTE_BF16 if dtype == "bf16" else LLATTE_FP32
        c.max_events = int(max_events)
        self.cdims = c
        self.d = c.d
        w = llatte_tok_w()
        for f, t in enumerate(tables):
            w.tables[f] = t.data_ptr()
        w.W_a1, w.W_a2 = w1.data_ptr(), w2.data_ptr()
        h = ctypes.c_void_p()
        rc = self.lib.llatte_tokenizer_create(ctypes.byref(h), ctypes.byref(c), ctypes.byref(w), 0)
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_tokenizer_create")
        self.h = h

    def uses_tensor_cores(self) -> bool:
        return self.lib.llatte_tokenizer_uses_tensor_cores(self.h) == 1

    def __call__(self, ids: torch.Tensor, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """Tokens [n, d] of ids (int32 CUDA [n, n_fields])."""
        if (not ids.is_cuda or ids.dtype != torch.int32 or ids.dim() != 2
                or ids.shape[1] != self.cdims.n_fields or not ids.is_contiguous()):
            raise ValueError("ids must be a contiguous CUDA int32 [n, n_fields] tensor")
        n = int(ids.shape[0])
        if out is None:
            out = torch.empty((n, self.d), dtype=self.dt, device=ids.device)
        elif (tuple(out.shape) != (n, self.d) or out.dtype != self.dt or not out.is_contiguous()):
            raise ValueError(f"out must be a contiguous {self.dt} [{n}, {self.d}] tensor")
        rc = self.lib.llatte_tokenize(self.h, _ptr(ids), n, _ptr(out), _stream_ptr(stream))
        if rc != LLATTE_OK:
            raise LlatteError(rc, "llatte_tokenize")
        return out

    def status(self) -> int:
        v = ctypes.c_int32(0)
        rc = self.lib.llatte_tokenizer_get_status(self.h, ctypes.byref(v))
        if rc not in (LLATTE_OK, LLATTE_ERR_DEVICE):
            raise LlatteError(rc, "llatte_tokenizer_get_status")
        return int(v.value)

    def close(self):
        if getattr(self, "h", None):
            self.lib.llatte_tokenizer_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
