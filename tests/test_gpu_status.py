"""The device timeout path, exercised without a fault: a bounded mbarrier wait
that nothing completes gives up after a short limit and the kernel records
RQ_ERR_DEVICE_TIMEOUT in the workspace status word, which the host reads;
the context stays usable afterwards (a decode on the same device matches the
oracle)."""

import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import all_streams, assert_close, make_cache, oracle_decode, oracle_streams, to_f32
from quantized_decode_attention_head_b200 import _lib, workloads
from quantized_decode_attention_head_b200.api import QuantizedKVCache

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    code = _lib.lib().rq_selftest_device_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel(), 2_000_000, stream)
    assert code == 0
    torch.cuda.synchronize()
    assert QuantizedKVCache.rq_decode_read_status(ws) == 7  # RQ_ERR_DEVICE_TIMEOUT
    assert _lib.lib().rq_decode_workspace_init(ctypes.c_void_p(ws.data_ptr()), ws.numel(), stream) == 0
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    # the device is still usable
    wl = workloads.Workload("after_timeout", n_layers=1, batch=1, n_q_heads=8, n_kv_heads=4, head_dim=128,
                            context=4 + 32 * 4 + 32 + 3, n_sink=4, n_recent=32, k_sigma=1.0, allowed=(2, 3, 4, 8),
                            avg_bits=3.0, seed=21)
    kb = np.array([[2, 3, 4, 8]])
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, kb, wl.context)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, kb, kb, to_f32(k), to_f32(v), all_streams(wl))
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    out = cache.rq_decode_attention(0, q[0, 0].contiguous()).cpu().numpy()
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(0, 0)])[(0, 0)]
    assert_close(out[0], exp, "decode after a timed-out wait")
