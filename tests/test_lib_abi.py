"""The C-ABI library without a GPU: it loads, exports every function that
include/rq.h declares, its host-only allocation equals the oracle's, and
argument errors come back as status codes before any CUDA call."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import allocation as al
from quantized_decode_attention_head_b200 import _lib
from quantized_decode_attention_head_b200.api import rq_allocate_bits, rq_cache_bytes

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rq.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path_calls():
    names = _declared_functions()
    for must in ["rq_allocate_bits", "rq_quantize_kv", "rq_append_token", "rq_decode_attention"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (rq_\w+)", out))
    assert set(_declared_functions()) <= exported
    # and the Python binding covers the same set
    assert set(_lib.SIGNATURES) == set(_declared_functions())


def test_status_strings():
    lib = _lib.lib()
    for code in range(8):
        assert lib.rq_status_string(code)
    assert b"librq" in lib.rq_build_info()


def _inst(rng, n):
    return rng.lognormal(0, 0.8, n), rng.uniform(0.5, 2.0, n), rng.uniform(3.6, 5.3, n)


@pytest.mark.parametrize("allowed", [(2, 3, 4, 8), (2, 4, 8), (2, 3, 4), (2, 3, 4, 5, 6, 7, 8)])
@pytest.mark.parametrize("n", [1, 4, 8, 288])
def test_host_allocation_matches_oracle(allowed, n):
    rng = np.random.default_rng(n + len(allowed))
    for avg in [min(allowed), 2.5, 3.0, 3.7, max(allowed)]:
        w, a, b = _inst(rng, n)
        ours = rq_allocate_bits(w, a, b, avg, allowed)
        ref = al.allocate(w, a, b, avg, allowed)
        assert np.allclose(ours["b_cont"], ref["b_cont"], atol=1e-9)
        assert abs(ours["b_cont"].sum() - n * avg) < 1e-8 * n
        # integer: same distortion (unique optimum on tie-free random data -> same vector)
        d_ours = al.distortion(w, a, b, ours["b_int"])
        d_ref = al.distortion(w, a, b, ref["b_int"])
        assert d_ours == pytest.approx(d_ref, rel=1e-12)
        assert np.array_equal(ours["b_int"], ref["b_int"])
        assert ours["b_int"].sum() <= ref["budget"]


def test_host_allocation_workload_budgets():
    from quantized_decode_attention_head_b200 import workloads

    for name, wl in workloads.CONFIGS.items():
        for key, (w, a, b, avg) in workloads.allocation_inputs(wl).items():
            ours = rq_allocate_bits(w, a, b, avg, wl.allowed)
            ref = al.allocate(w, a, b, avg, wl.allowed)
            assert np.array_equal(ours["b_int"], ref["b_int"]), (name, key)
    # long context floors every head at 2 bits; Qwen's V budget too (App. M.3 reading)
    w, a, b, avg = workloads.allocation_inputs(workloads.CONFIGS["long_128k"])["kv"]
    assert np.all(rq_allocate_bits(w, a, b, avg, (2, 3, 4))["b_int"] == 2)


def test_host_allocation_errors():
    w = np.ones(4)
    with pytest.raises(_lib.RQError) as e:
        rq_allocate_bits(w, 1.0, 4.4, 1.0, (2, 3, 4))
    assert e.value.status == "RQ_ERR_INFEASIBLE_BUDGET"
    with pytest.raises(_lib.RQError) as e:
        rq_allocate_bits(w, 1.0, 0.5, 3.0, (2, 3, 4))
    assert e.value.status == "RQ_ERR_INVALID_ARG"
    with pytest.raises(_lib.RQError) as e:
        rq_allocate_bits(w, 1.0, 4.4, 3.0, (2, 2, 4))
    assert e.value.status == "RQ_ERR_INVALID_ARG"


def _cfg(**kw):
    base = dict(n_layers=1, batch=1, n_q_heads=8, n_kv_heads=4, head_dim=64, n_sink=4, n_recent=32,
                max_tokens=512, k_bits=[2, 3, 4, 8], v_bits=[2, 3, 4, 8])
    base.update(kw)
    return base


def test_cache_bytes_accounting():
    c = _cfg()
    n = rq_cache_bytes(**c)
    # header + per-head tile regions + windows (bf16 rows, then D fp32 K
    # normalization factors), each region 256-aligned
    tiles = (512 - 4 - 32) // 32
    rec = {2: 4 * 128 * 2 + 512, 3: 7 * 128 * 2 + 512, 4: 8 * 128 * 2 + 512, 8: 16 * 128 * 2 + 512}
    expect = 256
    for b in (2, 3, 4, 8):
        expect += -(-(tiles * rec[b]) // 256) * 256
    expect += 4 * -(-((2 * 4 + 2 * 64) * 64 * 2 + 4 * 64) // 256) * 256
    assert n == expect


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(head_dim=96), "RQ_ERR_UNSUPPORTED"),
        (dict(k_bits=[2, 3, 5, 8]), "RQ_ERR_UNSUPPORTED"),
        (dict(n_q_heads=12), "RQ_ERR_UNSUPPORTED"),
        (dict(n_q_heads=64, n_kv_heads=4), "RQ_ERR_UNSUPPORTED"),
        (dict(batch=0), "RQ_ERR_INVALID_ARG"),
        (dict(n_sink=-1), "RQ_ERR_INVALID_ARG"),
        (dict(max_tokens=-5), "RQ_ERR_INVALID_ARG"),
    ],
)
def test_cache_config_errors(kw, status):
    with pytest.raises(_lib.RQError) as e:
        rq_cache_bytes(**_cfg(**kw))
    assert e.value.status == status


def test_cache_init_rejects_bad_arguments_before_cuda():
    lib = _lib.lib()
    from quantized_decode_attention_head_b200.api import _config

    cfg, keep = _config(**_cfg(head_dim=80))
    h = ctypes.c_void_p(0)
    assert lib.rq_cache_init(ctypes.byref(cfg), ctypes.c_void_p(4096), 1 << 20, ctypes.byref(h), None) == 2
    cfg, keep = _config(**_cfg())
    assert lib.rq_cache_init(ctypes.byref(cfg), ctypes.c_void_p(4096 + 16), 1 << 30, ctypes.byref(h), None) == 1
    assert lib.rq_cache_init(ctypes.byref(cfg), None, 1 << 30, ctypes.byref(h), None) == 1
    # null handles everywhere
    assert lib.rq_quantize_kv(None, None, None, 0, None) == 1
    assert lib.rq_append_token(None, 0, None, None, None) == 1
    assert lib.rq_decode_attention(None, 0, None, None, 0.0, 0, None, 0, None) == 1
    st = ctypes.c_int(0)
    assert lib.rq_decode_read_status(None, ctypes.byref(st)) == 1


def test_fit_distortion_matches_the_oracle():
    """Host calibration fit and fallback of the library against the oracle."""
    from oracle import calibration as cal
    from quantized_decode_attention_head_b200 import rq_fit_distortion

    rng = np.random.default_rng(11)
    bits = [2, 3, 4, 8]
    alpha = rng.uniform(0.1, 1.0, 20)
    beta = rng.uniform(3.0, 6.0, 20)
    table = alpha[:, None] * beta[:, None] ** -np.array(bits, dtype=np.float64)[None]
    table *= np.exp(rng.normal(0.0, 0.05, table.shape))  # small scatter
    table[3] = [1.0, 0.02, 0.4, 0.3]  # a poor fit
    a_l, b_l, r_l = rq_fit_distortion(bits, table)
    a_o, b_o, r_o = cal.calibrate(bits, table)
    assert np.allclose(a_l, a_o, rtol=1e-12) and np.allclose(b_l, b_o, rtol=1e-12)
    assert np.allclose(r_l, r_o, rtol=1e-12, atol=1e-12)
    assert r_l[3] < 0.96


def test_cap_weights_matches_the_oracle():
    from oracle import calibration as cal
    from quantized_decode_attention_head_b200 import rq_cap_weights

    w = np.array([0.5, 1.0, 2.0, 300.0, 1.5])
    assert np.array_equal(rq_cap_weights(w), cal.cap_weights(w))
    assert np.array_equal(rq_cap_weights(w, 2.0), cal.cap_weights(w, 2.0))


def test_timeout_selftest_rejects_bad_arguments_before_cuda():
    """Argument checks happen on the host, before any CUDA call: no workspace,
    a workspace smaller than its status block, or a limit above one second."""
    L = _lib.lib()
    assert L.rq_selftest_device_timeout(None, 4096, 1000, None) == 1
    assert L.rq_selftest_device_timeout(ctypes.c_void_p(256), 16, 1000, None) == 1
    assert L.rq_selftest_device_timeout(ctypes.c_void_p(256), 4096, 2_000_000_000, None) == 1


def test_misaligned_device_pointers_are_rejected_before_cuda():
    """A device pointer the kernels move in 16-byte vectors (the workspace,
    k, v, q, out) is refused on the host when it does not start on a 16-byte
    boundary, before any CUDA call; so are calibration samples off a 2-byte
    boundary and an fp64 result array off an 8-byte one."""
    L = _lib.lib()
    P = ctypes.c_void_p
    assert L.rq_decode_workspace_init(P(0x1008), 4096, None) == 1
    assert L.rq_selftest_device_timeout(P(0x1004), 4096, 1000, None) == 1
    bits = (ctypes.c_int * 1)(2)
    assert L.rq_measure_distortion(P(0x1001), 1, 32, 128, 0, bits, 1, P(0x2000), None) == 1
    assert L.rq_measure_distortion(P(0x1000), 1, 32, 128, 0, bits, 1, P(0x2004), None) == 1
