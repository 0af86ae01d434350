"""Python binding with the C ABI's names (include/rq.h).

PyTorch supplies device memory and streams; every computation happens in
librq.so.  Functions take torch tensors and pass their data pointers.
"""

from __future__ import annotations

import ctypes

import numpy as np

from ._lib import CacheConfig, check, lib


def _stream_ptr(stream=None, device=None):
    """The raw cudaStream_t of `stream`, or of the current stream of `device`
    (default: the current device)."""
    import torch

    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    idx = torch.cuda.current_device() if device is None else device
    return ctypes.c_void_p(torch._C._cuda_getCurrentRawStream(idx))


def _dptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _check_tensor(name, t, dtype, shape=None, device_type="cuda", align=16):
    import torch

    # one cheap test on the common path; the detailed message only on failure
    if (isinstance(t, torch.Tensor) and t.dtype is dtype and t.is_cuda == (device_type == "cuda")
            and t.is_contiguous() and (shape is None or t.shape == tuple(shape)) and t.data_ptr() % align == 0):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device.type != device_type:
        raise ValueError(f"{name} must be on {device_type}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    raise ValueError(f"{name} must start on a {align}-byte boundary (a view at an offset into a larger tensor?)")


def rq_allocate_bits(w, alpha, beta, avg_bits, allowed):
    """RateQuant allocation (host).  Returns dict(b_cont, b_int, log_lambda)."""
    w = np.ascontiguousarray(w, dtype=np.float64)
    n = w.size
    alpha = np.ascontiguousarray(np.broadcast_to(np.asarray(alpha, dtype=np.float64), (n,)))
    beta = np.ascontiguousarray(np.broadcast_to(np.asarray(beta, dtype=np.float64), (n,)))
    allowed = np.ascontiguousarray(allowed, dtype=np.int32)
    b_cont = np.zeros(n, dtype=np.float64)
    b_int = np.zeros(n, dtype=np.int32)
    nu = ctypes.c_double(0.0)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    code = lib().rq_allocate_bits(
        n,
        w.ctypes.data_as(dp),
        alpha.ctypes.data_as(dp),
        beta.ctypes.data_as(dp),
        float(avg_bits),
        allowed.ctypes.data_as(ip),
        allowed.size,
        b_cont.ctypes.data_as(dp),
        b_int.ctypes.data_as(ip),
        ctypes.byref(nu),
    )
    check("rq_allocate_bits", code)
    return {"b_cont": b_cont, "b_int": b_int.astype(np.int64), "log_lambda": nu.value}


def rq_measure_distortion(x, role, bits, stream=None):
    """Mean squared error of this library's quantizer per (head, bit width).
    x: bf16 CUDA tensor [n_heads, n_tokens, head_dim]; role "K" or "V".
    Returns a float64 numpy array [n_heads, len(bits)]."""
    import torch

    if x.dim() != 3:
        raise ValueError("x must be [n_heads, n_tokens, head_dim]")
    _check_tensor("x", x, torch.bfloat16, align=2)
    h, t, d = x.shape
    bits = np.ascontiguousarray(bits, dtype=np.int32)
    mse = torch.empty((h, bits.size), dtype=torch.float64, device=x.device)
    check("rq_measure_distortion", lib().rq_measure_distortion(
        _dptr(x), h, t, d, 0 if role == "K" else 1, bits.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), bits.size,
        _dptr(mse), _stream_ptr(stream)))
    return mse.cpu().numpy()


def rq_fit_distortion(bits, mse, r2_min=0.96):
    """Per-head (alpha, beta, r2) of D(b) = alpha * beta^-b from an
    [n_heads, n_bits] table, with the poor-fit fallback (host)."""
    bits = np.ascontiguousarray(bits, dtype=np.int32)
    mse = np.ascontiguousarray(mse, dtype=np.float64)
    n = mse.shape[0]
    alpha, beta, r2 = np.zeros(n), np.zeros(n), np.zeros(n)
    dp = ctypes.POINTER(ctypes.c_double)
    check("rq_fit_distortion", lib().rq_fit_distortion(
        n, bits.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), bits.size, mse.ctypes.data_as(dp), float(r2_min),
        alpha.ctypes.data_as(dp), beta.ctypes.data_as(dp), r2.ctypes.data_as(dp)))
    return alpha, beta, r2


def rq_cap_weights(w, factor=5.0):
    """w_i <- min(w_i, factor * mean(w)) (host)."""
    w = np.ascontiguousarray(w, dtype=np.float64)
    out = np.zeros_like(w)
    dp = ctypes.POINTER(ctypes.c_double)
    check("rq_cap_weights", lib().rq_cap_weights(w.size, w.ctypes.data_as(dp), float(factor), out.ctypes.data_as(dp)))
    return out


def _config(n_layers, batch, n_q_heads, n_kv_heads, head_dim, n_sink, n_recent, max_tokens, k_bits, v_bits, group=32,
            k_norm=False, hybrid=False):
    kb = np.ascontiguousarray(np.asarray(k_bits, dtype=np.int32).reshape(-1))
    vb = np.ascontiguousarray(np.asarray(v_bits, dtype=np.int32).reshape(-1))
    ip = ctypes.POINTER(ctypes.c_int)
    cfg = CacheConfig(
        n_layers, batch, n_q_heads, n_kv_heads, head_dim, group, n_sink, n_recent, max_tokens,
        kb.ctypes.data_as(ip), vb.ctypes.data_as(ip), int(bool(k_norm)), int(bool(hybrid)),
    )
    return cfg, (kb, vb)


def rq_cache_bytes(**cfg_kwargs) -> int:
    cfg, _keep = _config(**cfg_kwargs)
    out = ctypes.c_size_t(0)
    check("rq_cache_bytes", lib().rq_cache_bytes(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


class QuantizedKVCache:
    """Owns a device buffer (torch uint8 tensor) and the library's host handle."""

    def __init__(self, n_layers, batch, n_q_heads, n_kv_heads, head_dim, n_sink, n_recent, max_tokens,
                 k_bits, v_bits, device="cuda", group=32, k_norm=False, hybrid=False):
        import torch

        self.n_layers, self.batch = n_layers, batch
        self.n_q_heads, self.n_kv_heads, self.head_dim = n_q_heads, n_kv_heads, head_dim
        self.n_sink, self.n_recent, self.max_tokens = n_sink, n_recent, max_tokens
        self.k_bits = np.asarray(k_bits, dtype=np.int32).reshape(n_layers, n_kv_heads)
        self.v_bits = np.asarray(v_bits, dtype=np.int32).reshape(n_layers, n_kv_heads)
        cfg, keep = _config(n_layers, batch, n_q_heads, n_kv_heads, head_dim, n_sink, n_recent, max_tokens,
                            self.k_bits, self.v_bits, group, k_norm, hybrid)
        self.k_norm = bool(k_norm)
        self.hybrid = bool(hybrid)
        nbytes = ctypes.c_size_t(0)
        check("rq_cache_bytes", lib().rq_cache_bytes(ctypes.byref(cfg), ctypes.byref(nbytes)))
        self.nbytes = nbytes.value
        self.buffer = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buffer.data_ptr()) % 256
        self.buffer = self.buffer[off : off + self.nbytes]
        handle = ctypes.c_void_p(0)
        check("rq_cache_init", lib().rq_cache_init(ctypes.byref(cfg), _dptr(self.buffer), self.nbytes,
                                                   ctypes.byref(handle), _stream_ptr(None, self.buffer.get_device())))
        self.handle = handle
        # kept for the destructor, which may run while the interpreter is
        # tearing module globals down
        self._destroy = lib().rq_cache_destroy
        del keep

    def __del__(self):
        h = getattr(self, "handle", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self.handle = None

    # -- queries -----------------------------------------------------------
    def length(self, layer=0) -> int:
        t = ctypes.c_int(0)
        check("rq_cache_length", lib().rq_cache_length(self.handle, layer, ctypes.byref(t)))
        return t.value

    def k_norm_factors(self, layer, b, kv_head):
        """The stream's per-channel K normalization factors n[D] (a device view)."""
        import torch

        lay = self.stream_layout(layer, b, kv_head)
        d = self.head_dim
        rows = (2 * self.n_sink + 2 * (self.n_recent + 32)) * d * 2
        off = lay["window_offset"] + rows
        return self.buffer[off : off + 4 * d].view(torch.float32)

    def stream_layout(self, layer, b, kv_head):
        to, wo = ctypes.c_size_t(0), ctypes.c_size_t(0)
        rb, nt = ctypes.c_int(0), ctypes.c_int(0)
        check("rq_cache_stream_layout", lib().rq_cache_stream_layout(
            self.handle, layer, b, kv_head, ctypes.byref(to), ctypes.byref(rb), ctypes.byref(nt), ctypes.byref(wo)))
        return {"tile_offset": to.value, "record_bytes": rb.value, "n_tiles": nt.value, "window_offset": wo.value}

    # -- path ----------------------------------------------------------------
    def rq_quantize_kv(self, k, v, stream=None):
        import torch

        L, B, H, D = self.n_layers, self.batch, self.n_kv_heads, self.head_dim
        T = k.shape[3] if k.dim() == 5 else -1
        _check_tensor("k", k, torch.bfloat16, (L, B, H, T, D))
        _check_tensor("v", v, torch.bfloat16, (L, B, H, T, D))
        check("rq_quantize_kv", lib().rq_quantize_kv(self.handle, _dptr(k), _dptr(v), T, _stream_ptr(stream)))

    def rq_append_token(self, layer, k_new, v_new, stream=None):
        import torch

        nl = self.n_layers if layer == -1 else 1
        shape = (nl, self.batch, self.n_kv_heads, self.head_dim) if layer == -1 else (
            self.batch, self.n_kv_heads, self.head_dim)
        _check_tensor("k_new", k_new, torch.bfloat16, shape)
        _check_tensor("v_new", v_new, torch.bfloat16, shape)
        check("rq_append_token", lib().rq_append_token(self.handle, layer, _dptr(k_new), _dptr(v_new),
                                                       _stream_ptr(stream)))

    def rq_decode_workspace_bytes(self, n_splits=0) -> int:
        out = ctypes.c_size_t(0)
        check("rq_decode_workspace_bytes", lib().rq_decode_workspace_bytes(self.handle, n_splits, ctypes.byref(out)))
        return out.value

    def make_workspace(self, n_splits=0, stream=None):
        import torch

        nb = self.rq_decode_workspace_bytes(n_splits)
        ws = torch.empty(nb, dtype=torch.uint8, device=self.buffer.device)
        check("rq_decode_workspace_init", lib().rq_decode_workspace_init(_dptr(ws), nb, _stream_ptr(stream)))
        return ws

    def rq_decode_attention(self, layer, q, out=None, softmax_scale=0.0, n_splits=0, workspace=None, stream=None):
        import torch

        nl = self.n_layers if layer == -1 else 1
        shape = (nl, self.batch, self.n_q_heads, self.head_dim) if layer == -1 else (
            self.batch, self.n_q_heads, self.head_dim)
        _check_tensor("q", q, torch.bfloat16, shape)
        if out is None:
            out = torch.empty(shape, dtype=torch.float32, device=q.device)
        _check_tensor("out", out, torch.float32, shape)
        if workspace is None:
            workspace = self.make_workspace(n_splits, stream)
        check("rq_decode_attention", lib().rq_decode_attention(
            self.handle, layer, _dptr(q), _dptr(out), float(softmax_scale), int(n_splits), _dptr(workspace),
            workspace.numel(), _stream_ptr(stream, q.get_device())))
        return out

    def rq_decode_step(self, layer, q, k_new, v_new, out=None, softmax_scale=0.0, n_splits=0, workspace=None,
                       stream=None):
        """rq_append_token(layer, k_new, v_new) then rq_decode_attention(layer, q),
        in one launch (the step before a tile flush also packs that tile
        ahead); two launches only when the completed tile was not packed
        ahead by the previous step."""
        import torch

        nl = self.n_layers if layer == -1 else 1
        qshape = (nl, self.batch, self.n_q_heads, self.head_dim) if layer == -1 else (
            self.batch, self.n_q_heads, self.head_dim)
        kshape = (nl, self.batch, self.n_kv_heads, self.head_dim) if layer == -1 else (
            self.batch, self.n_kv_heads, self.head_dim)
        _check_tensor("q", q, torch.bfloat16, qshape)
        _check_tensor("k_new", k_new, torch.bfloat16, kshape)
        _check_tensor("v_new", v_new, torch.bfloat16, kshape)
        if out is None:
            out = torch.empty(qshape, dtype=torch.float32, device=q.device)
        _check_tensor("out", out, torch.float32, qshape)
        if workspace is None:
            workspace = self.make_workspace(n_splits, stream)
        check("rq_decode_step", lib().rq_decode_step(
            self.handle, layer, _dptr(q), _dptr(k_new), _dptr(v_new), _dptr(out), float(softmax_scale),
            int(n_splits), _dptr(workspace), workspace.numel(), _stream_ptr(stream, q.get_device())))
        return out

    @staticmethod
    def rq_decode_read_status(workspace) -> int:
        st = ctypes.c_int(0)
        check("rq_decode_read_status", lib().rq_decode_read_status(_dptr(workspace), ctypes.byref(st)))
        return st.value
