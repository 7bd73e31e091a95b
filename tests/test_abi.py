"""C-ABI checks that need no GPU: the library loads, exports every entry point
the public header declares, and rejects bad arguments on the host before it
touches the device."""
import ctypes
import glob
import os
import re

import pytest

from latent_attention_jagged_b200 import binding
from latent_attention_jagged_b200.build import build
from workloads import Dims, workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(hdr).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b(llatte_\w+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("llatte_create", "llatte_forward", "llatte_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(binding.EXPORTS) <= set(declared_functions())


def test_struct_layout_matches_header(lib):
    # int32 x 7, keep[16], 4 x int32, float, int32, (pad 4), int64, int64,
    # int32 x 6 (n_sum, sum_rank, d_seq, q_rank, d_time, attn_form)
    assert ctypes.sizeof(binding.llatte_dims) == 4 * (7 + 16 + 4 + 1 + 1) + 4 + 16 + 24
    assert binding.llatte_dims.attn_form.offset == binding.llatte_dims.d_time.offset + 4
    assert binding.llatte_dims.n_sum.offset == 4 * (7 + 16 + 4 + 1 + 1) + 4 + 16
    assert binding.llatte_dims.q_rank.offset == binding.llatte_dims.d_seq.offset + 4
    assert ctypes.sizeof(binding.llatte_layer_w) == 13 * ctypes.sizeof(ctypes.c_void_p)
    assert ctypes.sizeof(binding.llatte_summary_w) == 2 * ctypes.sizeof(ctypes.c_void_p)


def _cdims(**kw):
    base = workload("online").dims
    fields = dict(d=base.d, heads=base.heads, d_head=base.d_head, rank=base.rank,
                  d_ctx=base.d_ctx, n_q=base.n_q, keep=base.keep, d_out=base.d_out,
                  ffn_mult=base.ffn_mult, eps=base.eps, kv_norm=base.kv_norm, dtype=base.dtype)
    fields.update(kw)
    return binding.make_dims(Dims(**fields), max_batch=256, max_len=400)


def test_workspace_bytes_and_dim_checks(lib):
    good = _cdims()
    ws = lib.llatte_workspace_bytes(ctypes.byref(good))
    assert ws > 256 * 400 * 256 * 2          # at least the history rows
    for bad in (_cdims(keep=(100, 200)), _cdims(keep=(-1,)), _cdims(d=0), _cdims(rank=512),
                _cdims(d=12)):
        assert lib.llatte_workspace_bytes(ctypes.byref(bad)) == 0
    big = _cdims()
    big.max_total = 1000
    assert 0 < lib.llatte_workspace_bytes(ctypes.byref(big)) < ws


def test_create_rejects_bad_arguments_on_host(lib):
    h = ctypes.c_void_p()
    layers = (binding.llatte_layer_w * 4)()
    # increasing schedule: rejected before any device call
    bad = _cdims(keep=(10, 20, 30, 40))
    assert lib.llatte_create(ctypes.byref(h), ctypes.byref(bad), layers, None, None, 0) == \
        binding.LLATTE_ERR_ARG
    # null weight pointers
    good = _cdims()
    assert lib.llatte_create(ctypes.byref(h), ctypes.byref(good), layers, None, None, 0) == \
        binding.LLATTE_ERR_ARG
    assert lib.llatte_create(None, ctypes.byref(good), layers, None, None, 0) == binding.LLATTE_ERR_ARG
    # summaries: need candidates, no d_out, weights; sizes within the kernels' range
    for kw, code in ((dict(n_sum=2, sum_rank=8, d_seq=16, n_q=0), binding.LLATTE_ERR_ARG),
                     (dict(n_sum=2, sum_rank=8, d_seq=16, d_out=32), binding.LLATTE_ERR_ARG),
                     (dict(n_sum=2, sum_rank=0, d_seq=16), binding.LLATTE_ERR_ARG),
                     (dict(n_sum=17, sum_rank=8, d_seq=16), binding.LLATTE_ERR_ARG),
                     (dict(n_sum=2, sum_rank=8, d_seq=15), binding.LLATTE_ERR_UNSUPPORTED),
                     (dict(n_sum=2, sum_rank=2048, d_seq=16), binding.LLATTE_ERR_UNSUPPORTED)):
        bad = _cdims(**kw)
        assert lib.llatte_create(ctypes.byref(h), ctypes.byref(bad), layers, None, None, 0) == code
        assert lib.llatte_workspace_bytes(ctypes.byref(bad)) == 0
    for kw, code in ((dict(q_rank=-1), binding.LLATTE_ERR_ARG),
                     (dict(d_time=3), binding.LLATTE_ERR_ARG),
                     (dict(attn_form=3), binding.LLATTE_ERR_ARG),
                     (dict(attn_form=2, q_rank=64), binding.LLATTE_ERR_UNSUPPORTED),
                     (dict(attn_form=2, d_head=32, heads=8), binding.LLATTE_ERR_UNSUPPORTED),
                     (dict(d_time=512), binding.LLATTE_ERR_ARG),
                     (dict(q_rank=2048), binding.LLATTE_ERR_UNSUPPORTED)):
        bad = _cdims(**kw)
        assert lib.llatte_create(ctypes.byref(h), ctypes.byref(bad), layers, None, None, 0) == code
    ok = _cdims(n_sum=2, sum_rank=8, d_seq=16)
    assert lib.llatte_workspace_bytes(ctypes.byref(ok)) > lib.llatte_workspace_bytes(ctypes.byref(good))


def test_forward_and_status_reject_null_handle(lib):
    assert lib.llatte_forward(None, None, None, 1, None, None, None, None) == binding.LLATTE_ERR_ARG
    v = ctypes.c_int32()
    assert lib.llatte_get_status(None, ctypes.byref(v)) == binding.LLATTE_ERR_ARG
    assert lib.llatte_plan_export(None, None, None) == binding.LLATTE_ERR_ARG
    lib.llatte_destroy(None)
    assert lib.llatte_error_string(binding.LLATTE_ERR_DEVICE).startswith(b"device")


def test_tokenizer_struct_layout_and_host_checks(lib):
    # int32 (+4 pad), int64 x 8, int32 x 8, int32 x 3 (+4 pad), int64
    assert ctypes.sizeof(binding.llatte_tok_dims) == 8 + 64 + 32 + 16 + 8
    assert binding.llatte_tok_dims.max_events.offset == 120
    assert ctypes.sizeof(binding.llatte_tok_w) == 10 * ctypes.sizeof(ctypes.c_void_p)
    t = ctypes.c_void_p()
    w = binding.llatte_tok_w()

    def dims(**kw):
        c = binding.llatte_tok_dims()
        f = dict(n_fields=2, rows=(10, 20), width=(8, 8), d_hid=64, d=64,
                 dtype=binding.LLATTE_BF16, max_events=100)
        f.update(kw)
        c.n_fields = f["n_fields"]
        for i, (r, wd) in enumerate(zip(f["rows"], f["width"])):
            c.rows[i], c.width[i] = r, wd
        c.d_hid, c.d, c.dtype, c.max_events = f["d_hid"], f["d"], f["dtype"], f["max_events"]
        return c

    for kw, code in ((dict(n_fields=0), binding.LLATTE_ERR_ARG),
                     (dict(n_fields=9), binding.LLATTE_ERR_ARG),
                     (dict(rows=(0, 20)), binding.LLATTE_ERR_ARG),
                     (dict(width=(8, 4)), binding.LLATTE_ERR_UNSUPPORTED),     # 8-byte rows
                     (dict(width=(1024, 8)), binding.LLATTE_ERR_UNSUPPORTED),  # E row > 2 KB
                     (dict(d=60), binding.LLATTE_ERR_UNSUPPORTED),
                     (dict(dtype=7), binding.LLATTE_ERR_ARG),
                     (dict(max_events=-1), binding.LLATTE_ERR_ARG),
                     (dict(), binding.LLATTE_ERR_ARG)):                      # null weights
        c = dims(**kw)
        assert lib.llatte_tokenizer_create(ctypes.byref(t), ctypes.byref(c), ctypes.byref(w),
                                           0) == code
    assert lib.llatte_tokenize(None, None, 1, None, None) == binding.LLATTE_ERR_ARG
    v = ctypes.c_int32()
    assert lib.llatte_tokenizer_get_status(None, ctypes.byref(v)) == binding.LLATTE_ERR_ARG
    lib.llatte_tokenizer_destroy(None)
