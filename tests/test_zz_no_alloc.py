"""GPU test of rq_decode_attention_noalloc, the decode entry point for callers
that cannot allocate device memory (it runs on the library's own fixed device
scratch array).  Its output must match rq_decode_attention (caller-supplied
workspace) within the tolerance the parity tests use, on two calls in a row
-- the second call reuses the array the first one left behind.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, make_cache, to_f32
from quantized_decode_attention_head_b200 import _lib, workloads

pytestmark = pytest.mark.gpu


def _noalloc(cache, layer, q, out, n_splits=0):
    return _lib.lib().rq_decode_attention_noalloc(
        cache.handle, layer, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()), 0.0, n_splits,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


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
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    for layer in (0, 1, -1):
        qq = (q[0] if layer == -1 else q[0, layer]).contiguous()
        ref = cache.rq_decode_attention(layer, qq, n_splits=splits)
        torch.cuda.synchronize()
        for call in range(2):
            out = torch.full_like(ref, float("nan"))
            assert _noalloc(cache, layer, qq, out, splits) == 0
            torch.cuda.synchronize()
            assert_close(out.cpu().numpy(), ref.cpu().numpy(), f"layer {layer} call {call}")


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
    assert_close(out.cpu().numpy(), ref.cpu().numpy(), "big cache, 8 splits")
