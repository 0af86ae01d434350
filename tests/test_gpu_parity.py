"""GPU parity on small caches: packed bytes bit-exact against the oracle,
decode attention within max-abs 2e-3 / rel-L2 1e-3 of the fp64 oracle.

Sizes span several tiles with a ragged recent window; every bit width for K
and V, head_dim 64 and 128, GQA groups 1/2/4/8, split counts from 1 to one
split per tile, the all-layers call, and the short-cache edge cases."""

import numpy as np
import pytest
import torch

from gpu_helpers import (all_streams, assert_close, check_stream_bytes, make_cache, oracle_decode, oracle_streams,
                         to_f32, workload_bits)
from oracle import attention as at
from oracle import cache as ca
from oracle import quantize as qz
from quantized_decode_attention_head_b200 import workloads
from quantized_decode_attention_head_b200.api import QuantizedKVCache

pytestmark = pytest.mark.gpu


def _small(**kw):
    base = dict(name="small", n_layers=2, batch=2, n_q_heads=8, n_kv_heads=4, head_dim=128, context=4 + 32 * 6 + 32 + 13,
                n_sink=4, n_recent=32, k_sigma=1.5, allowed=(2, 3, 4, 8), avg_bits=3.0, seed=7)
    base.update(kw)
    return workloads.Workload(**base)


def _bits_grid(L, H):
    kb = np.array([[[2, 3, 4, 8][(l + h) % 4] for h in range(H)] for l in range(L)])
    vb = np.array([[[8, 2, 3, 4][(l + 2 * h) % 4] for h in range(H)] for l in range(L)])
    return kb, vb


def _build(wl, kb, vb, extra=64):
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + extra)
    cache.rq_quantize_kv(k, v)
    torch.cuda.synchronize()
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl))
    return cache, st, (k, v, f)


@pytest.mark.parametrize("d", [64, 128])
def test_quantize_all_bit_pairs_bitexact(d):
    wl = _small(head_dim=d)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    cache, st, _ = _build(wl, kb, vb)
    assert cache.length(0) == wl.context
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)


def _plant_signed_zeros(x, kind, rng):
    """Overwrite groups of a bf16 [L, B, H, T, D] tensor with zeros of both
    signs: K groups are 32 channels of a token, V groups a channel over the 32
    tokens of a tile.  Patterns: all +0, all -0, mixed zeros, a -0 minimum
    under positive values, a -0 maximum over negative values."""
    L, B, H, T, D = x.shape
    neg0 = torch.tensor(-0.0, dtype=torch.bfloat16)
    x = x.cpu().clone()
    tile0 = 4  # first tile token (n_sink = 4)
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for p in range(5):
                    t = tile0 + int(rng.integers(0, 32 * 3))  # a token of the first three tiles
                    if kind == "K":
                        g = int(rng.integers(0, D // 32))
                        idx = (l, b, h, t, slice(32 * g, 32 * g + 32))
                    else:
                        tl = (t - tile0) // 32
                        d0 = int(rng.integers(0, D))
                        idx = (l, b, h, slice(tile0 + 32 * tl, tile0 + 32 * tl + 32), d0)
                    grp = x[idx]
                    if p == 0:
                        grp.zero_()
                    elif p == 1:
                        grp.fill_(neg0)
                    elif p == 2:
                        grp.zero_()
                        grp[::3] = neg0
                    elif p == 3:
                        grp.copy_(grp.abs() + 0.125)
                        grp[int(rng.integers(0, 32))] = neg0
                        grp[int(rng.integers(0, 32))] = 0.0
                    else:
                        grp.copy_(-grp.abs() - 0.25)
                        grp[int(rng.integers(0, 32))] = neg0
                        grp[int(rng.integers(0, 32))] = 0.0
                    x[idx] = grp
    return x.cuda()


@pytest.mark.parametrize("d", [64, 128])
def test_signed_zero_groups_bitexact(d):
    """Groups whose extremes are +0 / -0 (and all-zero groups) pack to the
    oracle's bytes: a zero extreme is stored as +0 with a +0 scale whatever
    order the zeros come in."""
    wl = _small(head_dim=d, n_layers=1, context=4 + 32 * 3 + 32 + 9)
    kb, vb = _bits_grid(1, wl.n_kv_heads)
    rng = np.random.default_rng(41)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    k = _plant_signed_zeros(k, "K", rng)
    v = _plant_signed_zeros(v, "V", rng)
    cache = make_cache(wl, kb, vb, wl.context + 8)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl))
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
        for rec in s.records():
            q = qz.unpack_record(rec, s.kb, s.vb, s.d)
            for name in ("k_z", "v_z", "k_s", "v_s"):
                vals = q[name]
                assert not np.any(np.signbit(vals) & (vals == 0)), f"{key} {name}: a -0.0 was stored"
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    out = cache.rq_decode_attention(0, q[0, 0].contiguous()).cpu().numpy()
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(0, b) for b in range(wl.batch)])
    for b in range(wl.batch):
        assert_close(out[b], exp[(0, b)], f"signed zeros b {b}")


@pytest.mark.parametrize("d,g", [(64, 1), (64, 2), (64, 4), (64, 8), (128, 1), (128, 2), (128, 4), (128, 8)])
def test_decode_matches_oracle(d, g):
    wl = _small(head_dim=d, n_q_heads=4 * g, n_kv_heads=4, context=4 + 32 * 9 + 32 + 21)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    cache, st, (k, v, f) = _build(wl, kb, vb)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    ws = cache.make_workspace(n_splits=16)
    for layer in range(wl.n_layers):
        exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(layer, b) for b in range(wl.batch)])
        for splits in [1, 2, 5, 9, 0]:
            out = cache.rq_decode_attention(layer, q[0, layer].contiguous(), n_splits=splits, workspace=ws)
            got = out.cpu().numpy()
            for b in range(wl.batch):
                assert_close(got[b], exp[(layer, b)], f"layer {layer} b {b} splits {splits}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


def test_decode_all_layers_call():
    wl = _small(n_layers=3, context=4 + 32 * 5 + 32 + 3)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    cache, st, (k, v, f) = _build(wl, kb, vb)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    out = cache.rq_decode_attention(-1, q[0].contiguous(), n_splits=3)
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64),
                        [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
    got = out.cpu().numpy()
    for (l, b), e in exp.items():
        assert_close(got[l, b], e, f"layer {l} b {b}")


def test_explicit_split_count_keeps_items_short():
    """n_splits = 1 on a stream of 1024 tiles: a warp keeps P in 16-bit fixed
    point relative to its running maximum, and over 256 tiles per warp the
    rounding of the small probabilities exceeds the tolerance, so every plan
    holds an item to at most 128 tiles -- the call runs 8 splits and matches
    the oracle and the explicit 8-split call bit for bit."""
    wl = workloads.Workload("long_items", n_layers=1, batch=1, n_q_heads=16, n_kv_heads=2, head_dim=128,
                            context=4 + 32 + 32 * 1024 + 20, n_sink=4, n_recent=32, k_sigma=1.0, allowed=(2,),
                            avg_bits=2.0, seed=13)
    kb = np.full((1, 2), 2)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, kb, wl.context)
    cache.rq_quantize_kv(k, v)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    qq = q[0, 0].contiguous()
    one = cache.rq_decode_attention(0, qq, n_splits=1).cpu().numpy()
    eight = cache.rq_decode_attention(0, qq, n_splits=8).cpu().numpy()
    assert np.array_equal(one, eight)
    G = wl.group
    for h in range(wl.n_kv_heads):
        s = ca.StreamCache(wl.head_dim, 2, 2, wl.n_sink, wl.n_recent)
        s.prefill(to_f32(k[0, 0, h]), to_f32(v[0, 0, h]))
        kh, vh = s.dequantized()
        e = at.attend(to_f32(q[0, 0, 0, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
        assert_close(one[0, h * G:(h + 1) * G], e, f"n_splits=1 kv-head {h}")


def test_many_streams_single_cta_items():
    """Many streams: the automatic plan runs single-CTA work items (no
    clusters).  Every stream's output against the oracle, for the
    all-layers decode, a fused decode step and an explicit split count (which
    runs in clusters), before and after a step."""
    # 80 streams of 40 tiles: several single-CTA splits each
    wl = _small(n_layers=2, batch=10, context=4 + 32 * 40 + 32 + 11)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    cache, st, (k, v, f) = _build(wl, kb, vb)
    q, kn, vn = workloads.step_inputs(wl, 2, f, "cuda")
    which = [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)]
    ws = cache.make_workspace()
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), which)
    for splits in [0, 3]:
        got = cache.rq_decode_attention(-1, q[0].contiguous(), n_splits=splits, workspace=ws).cpu().numpy()
        for (l, b), e in exp.items():
            assert_close(got[l, b], e, f"layer {l} b {b} splits {splits}")
    got = cache.rq_decode_step(-1, q[1].contiguous(), kn[1].contiguous(), vn[1].contiguous(),
                               workspace=ws).cpu().numpy()
    for (l, b, h), s in st.items():
        s.append(to_f32(kn[1, l, b, h]), to_f32(vn[1, l, b, h]))
    exp = oracle_decode(wl, st, to_f32(q[1]).astype(np.float64), which)
    for (l, b), e in exp.items():
        assert_close(got[l, b], e, f"step: layer {l} b {b}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)


@pytest.mark.parametrize("T", [0, 1, 3, 4, 20, 36, 67, 68, 69, 100])
def test_short_caches(T):
    # T < S, T < S + R (no tiles), exactly one tile, ragged windows
    wl = _small(n_layers=1, batch=1, context=T)
    kb, vb = _bits_grid(1, wl.n_kv_heads)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, 200)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl))
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    out = cache.rq_decode_attention(0, q[0, 0].contiguous()).cpu().numpy()
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(0, 0)])[(0, 0)]
    if T == 0:
        assert np.all(out == 0)
    else:
        assert_close(out[0], exp, f"T={T}")


@pytest.mark.parametrize("S,R", [(4, 32), (0, 16), (2, 0), (6, 40)])
def test_append_across_flushes(S, R):
    wl = _small(n_layers=2, batch=2, n_sink=S, n_recent=R, context=S + R + 32 * 2 + 5)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    steps = 75
    cache, st, (k, v, f) = _build(wl, kb, vb, extra=steps)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    knp, vnp, qnp = to_f32(kn), to_f32(vn), to_f32(q).astype(np.float64)
    ws = cache.make_workspace()
    flushes = 0
    for t in range(steps):
        layer_mode = t % 3 == 0  # alternate all-layers and per-layer appends
        if layer_mode:
            cache.rq_append_token(-1, kn[t].contiguous(), vn[t].contiguous())
        else:
            for l in range(wl.n_layers):
                cache.rq_append_token(l, kn[t, l].contiguous(), vn[t, l].contiguous())
        for (l, b, h), s in st.items():
            flushes += s.append(knp[t, l, b, h], vnp[t, l, b, h])
        if t in (0, 3, 30, 31, 32, 33, 50, steps - 1):
            out = cache.rq_decode_attention(-1, q[t].contiguous(), workspace=ws).cpu().numpy()
            exp = oracle_decode(wl, st, qnp[t], [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
            for (l, b), e in exp.items():
                assert_close(out[l, b], e, f"step {t} layer {l} b {b}")
    assert flushes > 0
    assert cache.length(0) == wl.context + steps
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


@pytest.mark.parametrize("S,R,context", [(4, 32, 4 + 32 + 32 * 2 + 5), (0, 16, 16 + 31), (2, 0, 0), (6, 40, 3)])
def test_decode_step_equals_append_then_decode(S, R, context):
    """rq_decode_step (fused append + decode) gives the oracle's append-then-
    decode output at every step, across tile flushes and from a short or empty
    cache, and leaves the cache bytes (tiles, sink, ring) bit-exact."""
    wl = _small(n_layers=2, batch=2, n_sink=S, n_recent=R, context=context)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    steps = 80  # every case reaches S + R + 32 tokens: at least one tile flush
    cache, st, (k, v, f) = _build(wl, kb, vb, extra=steps)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    knp, vnp, qnp = to_f32(kn), to_f32(vn), to_f32(q).astype(np.float64)
    ws = cache.make_workspace()
    flushes = 0
    for t in range(steps):
        for (l, b, h), s in st.items():
            flushes += s.append(knp[t, l, b, h], vnp[t, l, b, h])
        if t % 2 == 0:  # all layers in one call
            out = cache.rq_decode_step(-1, q[t].contiguous(), kn[t].contiguous(), vn[t].contiguous(),
                                       workspace=ws).cpu().numpy()
        else:
            out = np.stack([cache.rq_decode_step(l, q[t, l].contiguous(), kn[t, l].contiguous(),
                                                 vn[t, l].contiguous(), workspace=ws).cpu().numpy()
                            for l in range(wl.n_layers)])
        exp = oracle_decode(wl, st, qnp[t], [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
        for (l, b), e in exp.items():
            assert_close(out[l, b], e, f"step {t} layer {l} b {b}")
    assert flushes > 0
    assert cache.length(0) == wl.context + steps
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


def test_decode_step_without_room_for_the_pack_item():
    """A workspace sized for the decode items only: the step before a tile
    flush cannot add the pack-ahead item, so it skips it and the flush step
    takes the two-launch path.  Outputs and bytes as the oracle's."""
    wl = _small(n_layers=1, batch=1, context=4 + 32 * 3 + 32 + 20)
    kb, vb = _bits_grid(1, wl.n_kv_heads)
    steps, splits = 16, 2
    cache, st, (k, v, f) = _build(wl, kb, vb, extra=steps)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    knp, vnp, qnp = to_f32(kn), to_f32(vn), to_f32(q).astype(np.float64)
    # layout: [status, counters: 64 u32 per stream][partials: streams x items x (G*D + 2G) floats];
    # the full size holds splits + 3 window items (one per chunk, the most any
    # length needs) + 1 pack item; the windows here take at most 3 chunks =
    # 2 items of 2 chunks, so splits + 2 items always decode, and the step
    # before a flush (window at S + R + 31 tokens, 2 items) has no room for
    # the pack item
    streams = wl.batch * wl.n_kv_heads
    offset = 256 + streams * 64 * 4
    part = (wl.group * wl.head_dim + 2 * wl.group) * 4
    assert cache.rq_decode_workspace_bytes(splits) == offset + streams * (splits + 3 + 1) * part
    ws = torch.zeros(offset + streams * (splits + 2) * part, dtype=torch.uint8, device="cuda")
    flushes = 0
    for t in range(steps):
        for (l, b, h), s in st.items():
            flushes += s.append(knp[t, l, b, h], vnp[t, l, b, h])
        out = cache.rq_decode_step(0, q[t, 0].contiguous(), kn[t, 0].contiguous(), vn[t, 0].contiguous(),
                                   n_splits=splits, workspace=ws).cpu().numpy()
        exp = oracle_decode(wl, st, qnp[t], [(0, 0)])[(0, 0)]
        assert_close(out[0], exp, f"step {t}")
    assert flushes > 0
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_k_norm_prefill_decode_and_steps(d):
    """Per-channel K normalization at outlier sigma 1.5 (the long-context
    workload's): factors, tile records and window rows bit for bit against
    the oracle after the prefill and after fused steps across tile flushes;
    decoded outputs (24-bit query) within the parity tolerance."""
    wl = _small(head_dim=d, n_q_heads=16, n_kv_heads=4, k_sigma=1.5, context=4 + 32 * 5 + 32 + 7)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    steps = 40
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + steps, k_norm=True)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, kb, vb, to_f32(k), to_f32(v), all_streams(wl), k_norm=True)
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    knp, vnp, qnp = to_f32(kn), to_f32(vn), to_f32(q).astype(np.float64)
    ws = cache.make_workspace()
    for t in range(steps):
        for (l, b, h), s in st.items():
            s.append(knp[t, l, b, h], vnp[t, l, b, h])
        out = cache.rq_decode_step(-1, q[t].contiguous(), kn[t].contiguous(), vn[t].contiguous(),
                                   workspace=ws).cpu().numpy()
        if t % 7 == 0 or t == steps - 1:
            exp = oracle_decode(wl, st, qnp[t], [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
            for (l, b), e in exp.items():
                assert_close(out[l, b], e, f"k_norm step {t} layer {l} b {b}")
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


def test_append_from_empty_fills_sink_then_ring():
    wl = _small(n_layers=1, batch=1, context=0)
    kb, vb = _bits_grid(1, wl.n_kv_heads)
    steps = 4 + 32 + 32 + 7
    k, v, f = workloads.kv_inputs(wl, "cuda", n_tokens=0)
    cache = make_cache(wl, kb, vb, steps)
    cache.rq_quantize_kv(k, v)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    st = {(0, 0, h): ca.StreamCache(wl.head_dim, int(kb[0, h]), int(vb[0, h]), wl.n_sink, wl.n_recent)
          for h in range(wl.n_kv_heads)}
    knp, vnp = to_f32(kn), to_f32(vn)
    for t in range(steps):
        cache.rq_append_token(0, kn[t, 0].contiguous(), vn[t, 0].contiguous())
        for (l, b, h), s in st.items():
            s.append(knp[t, l, b, h], vnp[t, l, b, h])
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    out = cache.rq_decode_attention(0, q[-1, 0].contiguous()).cpu().numpy()
    exp = oracle_decode(wl, st, to_f32(q[-1]).astype(np.float64), [(0, 0)])[(0, 0)]
    assert_close(out[0], exp)
    # capacity is checked on the host
    from quantized_decode_attention_head_b200._lib import RQError

    with pytest.raises(RQError) as e:
        cache.rq_append_token(0, kn[0, 0].contiguous(), vn[0, 0].contiguous())
    assert e.value.status == "RQ_ERR_CAPACITY"


def test_workspace_too_small_is_rejected():
    wl = _small(n_layers=1)
    kb, vb = _bits_grid(1, wl.n_kv_heads)
    cache, st, (k, v, f) = _build(wl, kb, vb)
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    from quantized_decode_attention_head_b200._lib import RQError

    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    with pytest.raises(RQError) as e:
        cache.rq_decode_attention(0, q[0, 0].contiguous(), n_splits=4, workspace=ws)
    assert e.value.status == "RQ_ERR_WORKSPACE"


def test_misaligned_device_pointers_are_rejected_before_launch():
    """The kernels move k, v, q, k_new, v_new, out and the workspace in
    16-byte vectors and bulk copies, so each must start on a 16-byte
    boundary.  A view a few bytes into a larger tensor is refused by the
    binding (ValueError) and, passed straight to the C ABI, by the host
    checks (RQ_ERR_INVALID_ARG = 1) before anything is launched: the cache
    keeps its length, and the aligned calls that follow match the oracle."""
    import ctypes

    from quantized_decode_attention_head_b200 import _lib

    P = ctypes.c_void_p
    wl = workloads.CONFIGS["tiny"]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 4)

    def shifted(t):  # the same values, starting one element past a 16-byte boundary
        buf = torch.empty(t.numel() + 16, dtype=t.dtype, device=t.device)
        view = buf[1:1 + t.numel()].view(t.shape)
        view.copy_(t)
        assert view.data_ptr() % 16 != 0
        return view

    L = _lib.lib()
    ks = shifted(k)
    with pytest.raises(ValueError):
        cache.rq_quantize_kv(ks, v)
    assert L.rq_quantize_kv(cache.handle, P(ks.data_ptr()), P(v.data_ptr()), k.shape[3], None) == 1
    assert L.rq_quantize_kv(cache.handle, P(k.data_ptr()), P(shifted(v).data_ptr()), k.shape[3], None) == 1
    assert cache.length(0) == 0
    cache.rq_quantize_kv(k, v)
    T = cache.length(0)

    q, kn, vn = workloads.step_inputs(wl, 1, f, "cuda")
    q0, kn0, vn0 = q[0, 0].contiguous(), kn[0, 0].contiguous(), vn[0, 0].contiguous()
    qs, kns, vns = shifted(q0), shifted(kn0), shifted(vn0)
    ws = cache.make_workspace()
    out = torch.empty(q0.shape, dtype=torch.float32, device="cuda")
    outs = shifted(out)
    wsb = torch.zeros(ws.numel() + 16, dtype=torch.uint8, device="cuda")[8:8 + ws.numel()]
    n = ws.numel()
    for call in (lambda: cache.rq_append_token(0, kns, vn0),
                 lambda: cache.rq_decode_attention(0, qs, workspace=ws),
                 lambda: cache.rq_decode_attention(0, q0, out=outs, workspace=ws),
                 lambda: cache.rq_decode_step(0, q0, kn0, vns, workspace=ws)):
        with pytest.raises(ValueError):
            call()
    f0 = ctypes.c_float(0.0)
    assert L.rq_append_token(cache.handle, 0, P(kns.data_ptr()), P(vn0.data_ptr()), None) == 1
    assert L.rq_append_token(cache.handle, 0, P(kn0.data_ptr()), P(vns.data_ptr()), None) == 1
    assert L.rq_decode_attention(cache.handle, 0, P(qs.data_ptr()), P(out.data_ptr()), f0, 0, P(ws.data_ptr()), n,
                                 None) == 1
    assert L.rq_decode_attention(cache.handle, 0, P(q0.data_ptr()), P(outs.data_ptr()), f0, 0, P(ws.data_ptr()), n,
                                 None) == 1
    assert L.rq_decode_attention(cache.handle, 0, P(q0.data_ptr()), P(out.data_ptr()), f0, 0, P(wsb.data_ptr()), n,
                                 None) == 1
    for a, b_, c in ((qs, kn0, vn0), (q0, kns, vn0), (q0, kn0, vns)):
        assert L.rq_decode_step(cache.handle, 0, P(a.data_ptr()), P(b_.data_ptr()), P(c.data_ptr()),
                                P(out.data_ptr()), f0, 0, P(ws.data_ptr()), n, None) == 1
    assert L.rq_decode_attention_noalloc(cache.handle, 0, P(qs.data_ptr()), P(out.data_ptr()), f0, 0, None) == 1
    assert L.rq_decode_attention_noalloc(cache.handle, 0, P(q0.data_ptr()), P(outs.data_ptr()), f0, 0, None) == 1
    assert L.rq_decode_workspace_init(P(wsb.data_ptr()), n, None) == 1
    torch.cuda.synchronize()
    assert cache.length(0) == T

    st = oracle_streams(wl, okb, ovb, to_f32(k), to_f32(v), all_streams(wl))
    cache.rq_decode_step(0, q0, kn0, vn0, out=out, workspace=ws)
    for (l, b, h), s in st.items():
        s.append(to_f32(kn[0, l, b, h]), to_f32(vn[0, l, b, h]))
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(0, 0)])[(0, 0)]
    assert_close(out.cpu().numpy()[0], exp, "aligned step after the rejected calls")
    assert cache.length(0) == T + 1
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


@pytest.mark.parametrize("scale", [0.03, 0.5])
def test_softmax_scale_argument(scale):
    """An explicit softmax scale (flatter, and four times sharper than
    1/sqrt(D) = 0.125 at head_dim 64) against the oracle's attention with the
    same scale, every stream of the small cache, through the plain and the
    fused-step calls."""
    wl = workloads.CONFIGS["tiny"]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 2)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, okb, ovb, to_f32(k), to_f32(v), all_streams(wl))
    q, kn, vn = workloads.step_inputs(wl, 2, f, "cuda")
    G = wl.group

    def check(out, qf, what):
        for (l, b, h), s in st.items():
            if l != 0:
                continue
            kh, vh = s.dequantized()
            e = at.attend(qf[0, b, h * G:(h + 1) * G].astype(np.float64), kh, vh, scale)
            assert_close(out[b, h * G:(h + 1) * G], e, f"{what} scale {scale} (b {b}, h {h})")

    out = cache.rq_decode_attention(0, q[0, 0].contiguous(), softmax_scale=scale).cpu().numpy()
    check(out, to_f32(q[0]), "decode")
    out = cache.rq_decode_step(0, q[1, 0].contiguous(), kn[1, 0].contiguous(), vn[1, 0].contiguous(),
                               softmax_scale=scale).cpu().numpy()
    for (l, b, h), s in st.items():
        if l == 0:
            s.append(to_f32(kn[1, 0, b, h]), to_f32(vn[1, 0, b, h]))
    check(out, to_f32(q[1]), "fused step")


def test_tiny_workload_end_to_end():
    wl = workloads.CONFIGS["tiny"]
    (kb, vb), (okb, ovb) = workload_bits(wl)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + wl.decode_steps)
    cache.rq_quantize_kv(k, v)
    st = oracle_streams(wl, okb, ovb, to_f32(k), to_f32(v), all_streams(wl))
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    q, kn, vn = workloads.step_inputs(wl, 1, f, "cuda")
    cache.rq_append_token(0, kn[0, 0].contiguous(), vn[0, 0].contiguous())
    for (l, b, h), s in st.items():
        s.append(to_f32(kn[0, l, b, h]), to_f32(vn[0, l, b, h]))
    out = cache.rq_decode_attention(0, q[0, 0].contiguous()).cpu().numpy()
    exp = oracle_decode(wl, st, to_f32(q[0]).astype(np.float64), [(0, 0)])[(0, 0)]
    assert_close(out[0], exp, "tiny")


@pytest.mark.parametrize("d,k_norm", [(64, False), (128, False), (128, True)])
def test_hybrid_prefill_decode_and_steps(d, k_norm):
    """Hybrid symmetric / asymmetric groups: tile records and window rows bit
    for bit against the oracle after the prefill and after fused steps across
    tile flushes, decoded outputs within the parity tolerance; both kinds of
    group occur in the data."""
    wl = _small(head_dim=d, n_q_heads=16, n_kv_heads=4, k_sigma=1.0, context=4 + 32 * 5 + 32 + 7)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    steps = 40
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + steps, k_norm=k_norm, hybrid=True)
    cache.rq_quantize_kv(k, v)
    knp0, vnp0 = to_f32(k), to_f32(v)
    st = oracle_streams(wl, kb, vb, knp0, vnp0, all_streams(wl), k_norm=k_norm, hybrid=True)
    # V groups of the prefill's tiles: one channel over 32 tokens
    vt = vnp0[:, :, :, wl.n_sink:wl.n_sink + 32 * 5].reshape(wl.n_layers, wl.batch, wl.n_kv_heads, 5, 32, d)
    sym = qz.symmetric_groups(vt.min(axis=4), vt.max(axis=4))
    assert 0 < sym.sum() < sym.size
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    q, kn, vn = workloads.step_inputs(wl, steps, f, "cuda")
    knp, vnp, qnp = to_f32(kn), to_f32(vn), to_f32(q).astype(np.float64)
    ws = cache.make_workspace()
    for t in range(steps):
        for (l, b, h), s in st.items():
            s.append(knp[t, l, b, h], vnp[t, l, b, h])
        out = cache.rq_decode_step(-1, q[t].contiguous(), kn[t].contiguous(), vn[t].contiguous(),
                                   workspace=ws).cpu().numpy()
        if t % 7 == 0 or t == steps - 1:
            exp = oracle_decode(wl, st, qnp[t], [(l, b) for l in range(wl.n_layers) for b in range(wl.batch)])
            for (l, b), e in exp.items():
                assert_close(out[l, b], e, f"hybrid step {t} layer {l} b {b}")
    for key, s in st.items():
        check_stream_bytes(cache, s, *key)
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0


def test_single_cta_items_merge_in_two_levels():
    """More than 16 single-CTA items per stream (20 streams of 1100 tiles: the
    automatic plan takes about 28 tile splits + 1 window item on a 148-SM
    device) merge in two levels: groups of 8, then the group partials.  Every
    stream's output against the cluster-merged decode at 9 splits, and
    sampled streams against the oracle."""
    wl = _small(n_layers=1, batch=5, n_q_heads=8, n_kv_heads=4, context=4 + 32 + 32 * 1100 + 11)
    kb, vb = _bits_grid(wl.n_layers, wl.n_kv_heads)
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = make_cache(wl, kb, vb, wl.context + 4)
    cache.rq_quantize_kv(k, v)
    sample = [(0, 0, 0), (0, 4, 3), (0, 2, 2)]
    st = oracle_streams(wl, kb, vb, to_f32(k[:, :, :]), to_f32(v), sample)
    del k, v
    torch.cuda.empty_cache()
    q, _, _ = workloads.step_inputs(wl, 1, f, "cuda")
    ws = cache.make_workspace(n_splits=9)
    auto = cache.rq_decode_attention(-1, q[0].contiguous(), workspace=ws).cpu().numpy()
    clus = cache.rq_decode_attention(-1, q[0].contiguous(), n_splits=9, workspace=ws).cpu().numpy()
    assert_close(auto, clus, "two-level merge vs cluster merge")
    G = wl.group
    for (l, b, h), s in st.items():
        kh, vh = s.dequantized()
        e = at.attend(to_f32(q[0, l, b, h * G:(h + 1) * G]).astype(np.float64), kh, vh)
        assert_close(auto[l, b, h * G:(h + 1) * G], e, f"two-level merge stream {(l, b, h)}")
    assert QuantizedKVCache.rq_decode_read_status(ws) == 0
