"""Fused decode steps launched back to back: a CUDA graph of 80 rq_decode_step
calls on a small cache, replayed, against the same steps run one at a time
with a synchronisation after each (outputs bit for bit; both caches' bytes
against the oracle).

Back to back, each decode launch may start before the previous one ends
(programmatic dependent launch) and fetches its first tile records early; a
launch that packed the next tile ahead must therefore complete before the
launch that first reads that tile starts.  With a few tiles per stream every
split's early fetch covers the newest tile, so a missing ordering shows up
as different outputs or bytes here."""

import numpy as np
import pytest
import torch

from gpu_helpers import all_streams, check_stream_bytes, make_cache, oracle_streams, to_f32
from quantized_decode_attention_head_b200 import workloads
from quantized_decode_attention_head_b200.api import QuantizedKVCache

pytestmark = pytest.mark.gpu


def test_graph_of_fused_steps_equals_synchronised_steps():
    wl = workloads.Workload("graph_steps", n_layers=1, batch=1, n_q_heads=8, n_kv_heads=4, head_dim=128,
                            context=4 + 32 * 5 + 32 + 20, n_sink=4, n_recent=32, k_sigma=1.0, allowed=(2, 3, 4, 8),
                            avg_bits=3.0, seed=31)
    kb = np.array([[2, 3, 4, 8]])
    vb = np.array([[8, 2, 3, 4]])
    steps = 80  # three tile flushes (after steps 11, 43, 75), each packed ahead by the step before
    k, v, f = workloads.kv_inputs(wl, "cuda")
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")

    def fresh():
        c = make_cache(wl, kb, vb, wl.context + steps)
        c.rq_quantize_kv(k, v)
        return c

    eager, graphed = fresh(), fresh()
    ws_e, ws_g = eager.make_workspace(), graphed.make_workspace()
    shape = (steps, wl.batch, wl.n_q_heads, wl.head_dim)
    out_e = torch.empty(shape, dtype=torch.float32, device="cuda")
    out_g = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    # one decode without append per cache: one-time host set-up outside the capture
    eager.rq_decode_attention(0, q[0, 0], out=out_e[0], workspace=ws_e)
    graphed.rq_decode_attention(0, q[0, 0], out=out_e[0], workspace=ws_g)
    torch.cuda.synchronize()
    for t in range(steps):
        eager.rq_decode_step(0, q[t, 0], kn[t, 0], vn[t, 0], out=out_e[t], workspace=ws_e)
        torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in range(steps):
            graphed.rq_decode_step(0, q[t, 0], kn[t, 0], vn[t, 0], out=out_g[t], workspace=ws_g)
    g.replay()
    torch.cuda.synchronize()
    assert QuantizedKVCache.rq_decode_read_status(ws_e) == 0
    assert QuantizedKVCache.rq_decode_read_status(ws_g) == 0
    assert eager.length(0) == graphed.length(0) == wl.context + steps
    assert torch.equal(out_e, out_g)
    # both caches' packed tiles and window rows as the oracle's after the same appends
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl))
    knp, vnp = to_f32(kn), to_f32(vn)
    for t in range(steps):
        for (l, b, h), s in st.items():
            s.append(knp[t, l, b, h], vnp[t, l, b, h])
    for key, s in st.items():
        check_stream_bytes(eager, s, *key)
        check_stream_bytes(graphed, s, *key)
    del g
