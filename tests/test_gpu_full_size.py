"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times (automatic split count, fused append +
decode step).

Every stream of the cache is built on the GPU; the oracle rebuilds a sample
of streams (the first and the last (layer, batch, kv-head) of the call) and
checks, for each sampled stream, the packed tile records and window rows bit
for bit and the decoded outputs of its query heads within the parity
tolerance.  The other streams are covered by the same kernels and by the
small-cache tests in test_gpu_parity.py.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, check_stream_bytes, make_cache, to_f32, workload_bits
from oracle import attention as at
from oracle import cache as ca
from quantized_decode_attention_head_b200 import workloads
from quantized_decode_attention_head_b200.api import QuantizedKVCache

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["llama3_8b", "qwen3_8b", "long_128k", "mistral_7b_b64"])
def test_full_size_sampled_streams(name):
    wl = workloads.CONFIGS[name]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    steps = 2
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + steps)
    cache.rq_quantize_kv(k, v)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    L, B, H = wl.n_layers, wl.batch, wl.n_kv_heads
    sample = [(0, 0, 0), (L - 1, B - 1, H - 1)]
    streams = {}
    for (l, b, h) in sample:
        s = ca.StreamCache(wl.head_dim, int(okb[l, h]), int(ovb[l, h]), wl.n_sink, wl.n_recent)
        s.prefill(to_f32(k[l, b, h]), to_f32(v[l, b, h]))
        streams[(l, b, h)] = s
    del k, v
    torch.cuda.empty_cache()
    ws = cache.make_workspace()
    G = wl.group
    for t in range(steps):
        out = cache.rq_decode_step(-1, q[t].contiguous(), kn[t].contiguous(), vn[t].contiguous(), workspace=ws)
        out = out.cpu().numpy()
        for (l, b, h), s in streams.items():
            s.append(to_f32(kn[t, l, b, h]), to_f32(vn[t, l, b, h]))
            kh, vh = s.dequantized()
            qh = to_f32(q[t, l, b, h * G:(h + 1) * G]).astype(np.float64)
            exp = at.attend(qh, kh, vh)
            assert_close(out[l, b, h * G:(h + 1) * G], exp, f"{name} step {t} stream {(l, b, h)}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    for key, s in streams.items():
        check_stream_bytes(cache, s, *key)
