"""DM0 dual-expert merged-attention inference on B200 (sm_100a).

Python face of the C ABI in include/dm0.h.  `Engine` owns one dm0_ctx and
takes torch CUDA tensors (or host numpy arrays for `infer_host`); it only
passes their pointers, sizes and the current CUDA stream to the library.
"""
from __future__ import annotations

import ctypes

import numpy as np

from ._abi import (EXPORTS, LIB_PATH, SITES, Dm0Config, Dm0Error, load_library, make_config,  # noqa: F401
                   pack_weights)

__all__ = ["Engine", "Dm0Error", "pack_weights", "pack_e4m3_rows", "load_library", "EXPORTS", "LIB_PATH"]


c_int_t = ctypes.c_int


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check_cuda(t, dtype, shape, name):
    import torch
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def pack_e4m3_rows(x: np.ndarray):
    """FP8 E4M3 codes (uint8, OCP bit patterns) and one fp32 scale per row of a 2-D array, through
    dm0_pack_e4m3_rows (host code; no GPU needed)."""
    lib = load_library()
    a = np.ascontiguousarray(x, np.float32)
    if a.ndim != 2:
        raise ValueError("pack_e4m3_rows expects a 2-D array")
    codes = np.empty(a.shape, np.uint8)
    scales = np.empty(a.shape[0], np.float32)
    st = lib.dm0_pack_e4m3_rows(a.ctypes.data, a.shape[0], a.shape[1], codes.ctypes.data, scales.ctypes.data)
    if st != 0:
        raise Dm0Error(st, "dm0_pack_e4m3_rows")
    return codes, scales


class Engine:
    """One dm0_ctx on the current CUDA device."""

    def __init__(self, dims, max_batch: int, max_prefix: int, time_mod: bool = False):
        """time_mod: the time-modulated action expert (DM0.5 page, section 5.2) instead of the DM0 one."""
        self.lib = load_library()
        self.dims = dims
        self.time_mod = bool(time_mod)
        self.cfg = make_config(dims, max_batch, max_prefix, self.time_mod)
        h = ctypes.c_void_p()
        st = self.lib.dm0_create(ctypes.byref(self.cfg), ctypes.byref(h))
        if st != 0 or not h.value:
            raise Dm0Error(st, "dm0_create failed (configuration or device allocation)")
        self.h = h

    # ------------------------------------------------------------------ helpers
    def _chk(self, st: int):
        if st != 0:
            raise Dm0Error(st, self.lib.dm0_last_error(self.h).decode())

    def close(self):
        if getattr(self, "h", None) is not None and self.h.value:
            self.lib.dm0_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ API
    def weights_bytes(self) -> int:
        return int(self.lib.dm0_weights_bytes(ctypes.byref(self.cfg)))

    def load_weights(self, blob: np.ndarray):
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        self._chk(self.lib.dm0_load_weights(self.h, blob.ctypes.data_as(ctypes.c_void_p), blob.nbytes))

    def load_from(self, provider):
        self.load_weights(pack_weights(provider, self.dims.layers, self.time_mod))

    def prefill(self, prefix_emb, stream=None):
        import torch
        B, P = prefix_emb.shape[:2]
        _check_cuda(prefix_emb, torch.bfloat16, (B, P, self.dims.hidden_v), "prefix_emb")
        self._chk(self.lib.dm0_prefill(self.h, _ptr(prefix_emb), B, P, _stream(stream)))

    def prepare(self, B: int, P: int, steps: int):
        """Capture ahead of time what dm0_denoise needs for (B, P, steps) (dm0_prepare)."""
        self._chk(self.lib.dm0_prepare(self.h, B, P, steps))

    def kv_view(self):
        k, v = ctypes.c_void_p(), ctypes.c_void_p()
        self._chk(self.lib.dm0_kv_view(self.h, ctypes.byref(k), ctypes.byref(v)))
        return k.value, v.value

    def kv_commit(self, B: int, P: int):
        self._chk(self.lib.dm0_kv_commit(self.h, B, P))

    def denoise(self, noise, steps: int, actions=None, velocities=None, stream=None):
        import torch
        _check_cuda(noise, torch.float32, noise.shape, "noise")
        if actions is None:
            actions = torch.empty_like(noise)
        _check_cuda(actions, torch.float32, noise.shape, "actions")
        if velocities is not None:
            _check_cuda(velocities, torch.float32, (steps,) + tuple(noise.shape), "velocities")
        self._chk(self.lib.dm0_denoise(self.h, _ptr(noise), steps, _ptr(actions), _ptr(velocities),
                                       _stream(stream)))
        return actions

    def infer_host(self, prefix_bits: np.ndarray, noise: np.ndarray, steps: int, actions: np.ndarray = None,
                   stream=None) -> np.ndarray:
        """prefix_bits: host uint16 bf16 bit patterns [B][P][Hv]; noise: host f32 [B][S][A]."""
        B, P = prefix_bits.shape[:2]
        if actions is None:
            actions = np.empty_like(noise, dtype=np.float32)
        self._chk(self.lib.dm0_infer_host(self.h, prefix_bits.ctypes.data_as(ctypes.c_void_p),
                                          noise.ctypes.data_as(ctypes.c_void_p), B, P, steps,
                                          actions.ctypes.data_as(ctypes.c_void_p), _stream(stream)))
        return actions

    def merged_layer(self, layer, h_prefix, h_suffix, out_prefix, out_suffix, k_out, v_out, stream=None):
        import torch
        d = self.dims
        B, P = h_prefix.shape[:2]
        _check_cuda(h_prefix, torch.float32, (B, P, d.hidden_v), "h_prefix")
        _check_cuda(h_suffix, torch.float32, (B, d.chunk, d.hidden_a), "h_suffix")
        _check_cuda(out_prefix, torch.float32, (B, P, d.hidden_v), "out_prefix")
        _check_cuda(out_suffix, torch.float32, (B, d.chunk, d.hidden_a), "out_suffix")
        _check_cuda(k_out, torch.bfloat16, (B, d.n_kv, P, d.head_dim), "k_out")
        _check_cuda(v_out, torch.bfloat16, (B, d.n_kv, P, d.head_dim), "v_out")
        self._chk(self.lib.dm0_merged_layer(self.h, layer, _ptr(h_prefix), _ptr(h_suffix), B, P, _ptr(out_prefix),
                                            _ptr(out_suffix), _ptr(k_out), _ptr(v_out), _stream(stream)))

    def op_gemm(self, A, B, C, swap=0, splits=1, stream=None):
        import torch
        M, K = A.shape
        N = B.shape[0]
        _check_cuda(A, torch.bfloat16, (M, K), "A")
        _check_cuda(B, torch.bfloat16, (N, K), "B")
        _check_cuda(C, torch.float32, (N, M) if swap else (M, N), "C")
        self._chk(self.lib.dm0_op_gemm(self.h, _ptr(A), _ptr(B), _ptr(C), M, N, K, swap, splits, _stream(stream)))

    def grad_floats(self) -> int:
        return int(self.lib.dm0_grad_floats(ctypes.byref(self.cfg)))

    def train_step(self, a, eps, t, mask, grads=None, kv_grads=None, stream=None):
        """One flow-matching training step (dm0_train_step) over the context's prefix cache.

        a, eps: CUDA f32 [B][chunk][A]; t: CUDA f32 [B]; mask: CUDA uint8 [B][chunk][A].  Returns (loss
        [1], grads [grad_floats]) as CUDA f32 tensors; kv_grads, when given, is CUDA f32
        [2][layers][B][n_kv][P][head_dim] and receives the cache gradients."""
        import torch
        B = a.shape[0]
        d = self.dims
        shape = (B, d.chunk, d.action_dim)
        _check_cuda(a, torch.float32, shape, "a")
        _check_cuda(eps, torch.float32, shape, "eps")
        _check_cuda(t, torch.float32, (B,), "t")
        _check_cuda(mask, torch.uint8, shape, "mask")
        if grads is None:
            grads = torch.empty(self.grad_floats(), device=a.device, dtype=torch.float32)
        _check_cuda(grads, torch.float32, (self.grad_floats(),), "grads")
        loss = torch.empty(1, device=a.device, dtype=torch.float32)
        self._chk(self.lib.dm0_train_step(self.h, _ptr(a), _ptr(eps), _ptr(t), _ptr(mask), _ptr(loss), _ptr(grads),
                                          _ptr(kv_grads), _stream(stream)))
        return loss, grads

    def set_prefix_fp8(self, enable: bool = True, stream=None):
        """Run the VLM MLP's gate/up and down GEMMs in FP8 E4M3 (dm0_set_prefix_fp8)."""
        self._chk(self.lib.dm0_set_prefix_fp8(self.h, 1 if enable else 0, _stream(stream)))

    def op_quant_e4m3(self, x, codes, scales, gain=None, ssq=None, stream=None):
        import torch
        rows, cols = x.shape
        f32 = x.dtype == torch.float32
        _check_cuda(x, torch.float32 if f32 else torch.bfloat16, (rows, cols), "x")
        _check_cuda(codes, torch.uint8, (rows, cols), "codes")
        _check_cuda(scales, torch.float32, (rows,), "scales")
        if gain is not None:
            _check_cuda(gain, torch.float32, (cols,), "gain")
        if ssq is not None:
            _check_cuda(ssq, torch.float32, (rows,), "ssq")
        self._chk(self.lib.dm0_op_quant_e4m3(self.h, _ptr(x), int(f32), rows, cols, _ptr(gain), _ptr(ssq),
                                             _ptr(codes), _ptr(scales), _stream(stream)))

    def op_gemm_e4m3(self, A, sa, B, sb, C, stream=None):
        import torch
        M, K = A.shape
        N = B.shape[0]
        _check_cuda(A, torch.uint8, (M, K), "A")
        _check_cuda(B, torch.uint8, (N, K), "B")
        _check_cuda(sa, torch.float32, (M,), "sa")
        _check_cuda(sb, torch.float32, (N,), "sb")
        _check_cuda(C, torch.float32, (M, N), "C")
        self._chk(self.lib.dm0_op_gemm_e4m3(self.h, _ptr(A), _ptr(sa), _ptr(B), _ptr(sb), _ptr(C), M, N, K,
                                            _stream(stream)))

    def op_attention(self, q, ka, va, kb, vb, o, splits=1, stream=None):
        import torch
        for t, nm in ((q, "q"), (ka, "ka"), (va, "va"), (kb, "kb"), (vb, "vb"), (o, "o")):
            if t is not None:
                _check_cuda(t, torch.bfloat16, t.shape, nm)
        B, Tq = q.shape[:2]
        Ta = ka.shape[2]
        Tb = 0 if kb is None else kb.shape[2]
        self._chk(self.lib.dm0_op_attention(self.h, _ptr(q), _ptr(ka), _ptr(va), Ta, _ptr(kb), _ptr(vb), Tb,
                                            _ptr(o), B, Tq, splits, _stream(stream)))

    def debug_view(self, name: str) -> int:
        """Device address of an internal activation buffer (see dm0_debug_view)."""
        p = ctypes.c_void_p()
        self._chk(self.lib.dm0_debug_view(self.h, name.encode(), ctypes.byref(p)))
        return p.value

    def launch_count(self) -> int:
        return int(self.lib.dm0_launch_count(self.h))

    def probe(self, site_mask: int):
        self._chk(self.lib.dm0_probe(self.h, site_mask))

    def probe_read(self, site: int):
        n, ms = c_int_t(), ctypes.c_double()
        self._chk(self.lib.dm0_probe_read(self.h, site, ctypes.byref(n), ctypes.byref(ms)))
        return n.value, ms.value

    def selftest_timeout(self, limit_us: int = 20000, stream=None):
        self._chk(self.lib.dm0_selftest_timeout(self.h, limit_us, _stream(stream)))

    def sync(self, stream=None):
        self._chk(self.lib.dm0_sync(self.h, _stream(stream)))

    def device_error(self) -> int:
        return int(self.lib.dm0_device_error(self.h))

    def clear_error(self):
        self._chk(self.lib.dm0_clear_error(self.h))
