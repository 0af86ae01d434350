"""GPU tests of rq_decode_attention_noalloc, the decode entry point for
callers that cannot allocate device memory (code inside a custom allocator
or memory pool, a runtime whose device memory is fully pre-reserved, a plugin
limited to the buffers it is handed).  It runs on the library's own fixed
device scratch array.  Its output must match rq_decode_attention
(caller-supplied workspace) within the tolerance the parity tests use, and
the fp64 oracle, on two calls in a row -- the second call reuses the array
the first one left behind -- and in an order where a call over fewer streams
follows one over more, so that state a larger call left in the shared array
(status word, completion counters) must not leak into a smaller one.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import all_streams, assert_close, make_cache, oracle_decode, oracle_streams, to_f32
from oracle import attention as at
from oracle import cache as ca
from quantized_decode_attention_head_b200 import _lib, workloads

pytestmark = pytest.mark.gpu


def _noalloc(cache, layer, q, out, n_splits=0):
    return _lib.lib().rq_decode_attention_noalloc(
        cache.handle, layer, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()), 0.0, n_splits,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _noalloc_status():
    st = ctypes.c_int(-1)
    assert _lib.lib().rq_decode_noalloc_read_status(ctypes.byref(st)) == 0
    return st.value


def _workload(d, g, T, L=1, B=2):
    return workloads.Workload("noalloc", n_layers=L, batch=B, n_q_heads=4 * g, n_kv_heads=4, head_dim=d,
                              context=T, n_sink=4, n_recent=32, k_sigma=1.5, allowed=(2, 3, 4, 8), avg_bits=3.0,
                              seed=11)


@pytest.mark.parametrize("d,g,splits", [(128, 4, 0), (128, 4, 7), (64, 2, 3), (128, 8, 1)])
def test_noalloc_matches_workspace_entry_point(d, g, splits):
    wl = _workload(d, g, 4 + 32 * 12 + 32 + 9, L=2)
    kb = np.array([[2, 3, 4, 8], [8, 4, 3, 2]])
    vb = np.array([[3, 2, 8, 4], [2, 8, 4, 3]])
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 8)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl))
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64),
                        [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
    # all layers, then one layer (fewer streams after more), all layers, the other layer
    for layer in (-1, 0, -1, 1):
        qq = (q[0] if layer == -1 else q[0, layer]).contiguous()
        ref = cache.rq_decode_attention(layer, qq, n_splits=splits)
        torch.cuda.synchronize()
        for call in range(2):
            out = torch.full_like(ref, float("nan"))
            assert _noalloc(cache, layer, qq, out, splits) == 0
            torch.cuda.synchronize()
            assert _noalloc_status() == 0
            got = out.cpu().numpy()
            assert_close(got, ref.cpu().numpy(), f"layer {layer} call {call} vs workspace entry point")
            for l in (range(wl.n_layers) if layer == -1 else [layer]):
                for b in range(wl.batch):
                    g_lb = got[l, b] if layer == -1 else got[b]
                    assert_close(g_lb, exp[(l, b)], f"layer {layer} call {call} ({l}, {b}) vs oracle")


def test_noalloc_rejects_calls_beyond_the_scratch_array():
    # 512 streams x 65 work items of partials do not fit the fixed array
    wl = workloads.Workload("noalloc_big", n_layers=1, batch=128, n_q_heads=16, n_kv_heads=4, head_dim=128,
                            context=4 + 32 + 32 * 64, n_sink=4, n_recent=32, k_sigma=1.0, allowed=(2,),
                            avg_bits=2.0, seed=12)
    kb = np.full((1, 4), 2)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, kb, wl.context)
    cache.rq_quantize_kv(k, v)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device="cuda")
    assert _noalloc(cache, 0, q[0, 0].contiguous(), out, 64) == 5  # RQ_ERR_WORKSPACE
    # within the limit the same cache decodes fine and matches the workspace entry point
    assert _noalloc(cache, 0, q[0, 0].contiguous(), out, 8) == 0
    ref = cache.rq_decode_attention(0, q[0, 0].contiguous(), n_splits=8)
    torch.cuda.synchronize()
    assert _noalloc_status() == 0
    assert_close(out.cpu().numpy(), ref.cpu().numpy(), "big cache, 8 splits")


def test_noalloc_automatic_plan_on_a_many_stream_call():
    """n_splits = 0 on a large many-stream call: 512 streams of 1024 tiles (8
    tile items each: no item holds more than 128 tiles) plus a 1048-token
    bf16 window (one window item of all its chunks, since the plan runs in
    several waves) at 8 query heads per kv head.  Its partials (13 items per
    stream) fit the array; the call matches the workspace entry point and
    the oracle on sampled streams.  (A call whose partials exceed the array
    is rejected: test_noalloc_rejects_calls_beyond_the_scratch_array.)"""
    wl = workloads.Workload("noalloc_many", n_layers=1, batch=64, n_q_heads=64, n_kv_heads=8, head_dim=128,
                            context=4 + 1024 + 32 * 1024 + 20, n_sink=4, n_recent=1024, k_sigma=1.0,
                            allowed=(2,), avg_bits=2.0, seed=13)
    kb = np.full((1, 8), 2)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, kb, wl.context)
    cache.rq_quantize_kv(k, v)
    sample = [(0, 0, 0), (0, wl.batch - 1, wl.n_kv_heads - 1)]
    streams = {}
    for (l, b, h) in sample:
        s = ca.StreamCache(wl.head_dim, 2, 2, wl.n_sink, wl.n_recent)
        s.prefill(to_f32(k[l, b, h]), to_f32(v[l, b, h]))
        streams[(l, b, h)] = s
    del k, v
    torch.cuda.empty_cache()
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    qq = q[0, 0].contiguous()
    ref = cache.rq_decode_attention(0, qq)
    torch.cuda.synchronize()
    G = wl.group
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(cache, 0, qq, out, 0) == 0
        torch.cuda.synchronize()
        assert _noalloc_status() == 0
        assert_close(out.cpu().numpy(), ref.cpu().numpy(), f"automatic plan call {call} vs workspace entry point")
        for (l, b, h), s in streams.items():
            kh, vh = s.dequantized()
            e = at.attend(to_f32(q[0, l, b, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
            assert_close(out[b, h * G:(h + 1) * G].cpu().numpy(), e, f"automatic plan call {call} {(l, b, h)}")
