"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times (automatic split count, fused append +
decode step), and on the long-context cache at the split counts its
workload names (64, 128, 256 per head).

Every stream of the cache is built on the GPU; the oracle rebuilds a sample
of streams and checks, for each sampled stream, the packed tile records and
window rows bit for bit and the decoded outputs of its query heads within the
parity tolerance.  The sample holds the first and the last (layer, batch,
kv-head) of the call and, for every (K bits, V bits) pair the allocation
gives, the first stream with that pair -- so every bit pair of every
workload is byte-compared at full size.  The other streams are covered by the
same kernels and by the small-cache tests in test_gpu_parity.py.
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


def sampled_streams(wl, kb, vb):
    """First and last stream of the call plus the first stream of every
    (K bits, V bits) pair (its batch element varies with the layer)."""
    L, B, H = wl.n_layers, wl.batch, wl.n_kv_heads
    sample = [(0, 0, 0), (L - 1, B - 1, H - 1)]
    seen = set()
    for l in range(L):
        for h in range(H):
            pair = (int(kb[l, h]), int(vb[l, h]))
            if pair not in seen:
                seen.add(pair)
                key = (l, l % B, h)
                if key not in sample:
                    sample.append(key)
    pairs = {(int(kb[l, h]), int(vb[l, h])) for (l, b, h) in sample}
    assert pairs == {(int(a), int(c)) for a, c in zip(kb.ravel(), vb.ravel())}
    return sample


@pytest.mark.parametrize("name", ["llama3_8b", "qwen3_8b", "long_128k", "mistral_7b_b64"])
def test_full_size_sampled_streams(name):
    wl = workloads.CONFIGS[name]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    steps = 2
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + steps)
    cache.rq_quantize_kv(k, v)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    sample = sampled_streams(wl, okb, ovb)
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


def test_long_context_named_split_counts():
    """long_128k at 64, 128 and 256 splits per head (then the combine), every
    one of its 8 streams against the oracle; the automatic plan repeated five
    times (bit-identical, within tolerance); a fused step at 256 splits."""
    wl = workloads.CONFIGS["long_128k"]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 1)
    cache.rq_quantize_kv(k, v)
    q, kn, vn = workloads.step_inputs(wl, 2, f, "cuda")
    streams = {}
    for h in range(wl.n_kv_heads):
        s = ca.StreamCache(wl.head_dim, int(okb[0, h]), int(ovb[0, h]), wl.n_sink, wl.n_recent)
        s.prefill(to_f32(k[0, 0, h]), to_f32(v[0, 0, h]))
        streams[h] = s
    del k, v
    torch.cuda.empty_cache()
    G = wl.group
    ws = cache.make_workspace(n_splits=max(wl.splits))
    exp = {}
    for h, s in streams.items():
        kh, vh = s.dequantized()
        exp[h] = at.attend(to_f32(q[0, 0, 0, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
    for splits in wl.splits:
        out = cache.rq_decode_attention(0, q[0, 0].contiguous(), n_splits=splits, workspace=ws).cpu().numpy()
        for h in streams:
            assert_close(out[0, h * G:(h + 1) * G], exp[h], f"splits {splits} kv-head {h}")
    # The automatic plan (one wave of single-CTA items, merged in two levels
    # by the last items to finish): the merge order is fixed by item index,
    # so repeated calls agree bit for bit whatever order the items finish in.
    auto = [cache.rq_decode_attention(0, q[0, 0].contiguous(), workspace=ws).cpu().numpy() for _ in range(5)]
    for o in auto[1:]:
        assert np.array_equal(o, auto[0])
    for h in streams:
        assert_close(auto[0][0, h * G:(h + 1) * G], exp[h], f"automatic plan kv-head {h}")
    out = cache.rq_decode_step(0, q[1, 0].contiguous(), kn[1, 0].contiguous(), vn[1, 0].contiguous(),
                               n_splits=max(wl.splits), workspace=ws).cpu().numpy()
    for h, s in streams.items():
        s.append(to_f32(kn[1, 0, 0, h]), to_f32(vn[1, 0, 0, h]))
        kh, vh = s.dequantized()
        e = at.attend(to_f32(q[1, 0, 0, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
        assert_close(out[0, h * G:(h + 1) * G], e, f"fused step, {max(wl.splits)} splits, kv-head {h}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    for h, s in streams.items():
        check_stream_bytes(cache, s, 0, 0, h)


def test_long_context_k_norm():
    """The long-context workload (outlier sigma 1.5) as a K-normalized cache:
    the factors, sampled streams' records and windows bit for bit, and the
    decoded heads of three streams within the parity tolerance after the
    prefill and after a fused step (24-bit query)."""
    wl = workloads.CONFIGS["long_128k"]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 1, k_norm=True)
    cache.rq_quantize_kv(k, v)
    q, kn, vn = workloads.step_inputs(wl, 2, f, "cuda")
    heads = (0, 3, 7)
    streams = {}
    for h in heads:
        s = ca.StreamCache(wl.head_dim, int(okb[0, h]), int(ovb[0, h]), wl.n_sink, wl.n_recent, k_norm=True)
        s.prefill(to_f32(k[0, 0, h]), to_f32(v[0, 0, h]))
        streams[h] = s
    del k, v
    torch.cuda.empty_cache()
    G = wl.group
    ws = cache.make_workspace()
    out = cache.rq_decode_attention(0, q[0, 0].contiguous(), workspace=ws).cpu().numpy()
    for h, s in streams.items():
        kh, vh = s.dequantized()
        e = at.attend(to_f32(q[0, 0, 0, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
        assert_close(out[0, h * G:(h + 1) * G], e, f"k_norm prefill, kv-head {h}")
    out = cache.rq_decode_step(0, q[1, 0].contiguous(), kn[1, 0].contiguous(), vn[1, 0].contiguous(),
                               workspace=ws).cpu().numpy()
    for h, s in streams.items():
        s.append(to_f32(kn[1, 0, 0, h]), to_f32(vn[1, 0, 0, h]))
        kh, vh = s.dequantized()
        e = at.attend(to_f32(q[1, 0, 0, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
        assert_close(out[0, h * G:(h + 1) * G], e, f"k_norm fused step, kv-head {h}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    for h, s in streams.items():
        check_stream_bytes(cache, s, 0, 0, h)
