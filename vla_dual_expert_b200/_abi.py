"""ctypes binding of libdm0.so (include/dm0.h): argument marshalling only.

Every function here forwards device pointers, sizes and a CUDA stream to the
C ABI; all arithmetic of the path runs in the library's CUDA kernels.  If
libdm0.so is missing or fails to load, importing the binding raises: there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdm0.so")

c_int, c_float, c_size_t, c_void_p = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

STATUS = {0: "DM0_OK", -1: "DM0_EINVAL", -2: "DM0_ESHAPE", -3: "DM0_ENOMEM", -4: "DM0_ECUDA",
          -5: "DM0_EDEVICE", -6: "DM0_ESTATE"}

# every symbol include/dm0.h declares
EXPORTS = ("dm0_create", "dm0_weights_bytes", "dm0_load_weights", "dm0_prefill", "dm0_kv_view",
           "dm0_kv_commit", "dm0_denoise", "dm0_infer_host", "dm0_merged_layer", "dm0_op_gemm",
           "dm0_op_attention", "dm0_attention_noalloc", "dm0_debug_view", "dm0_launch_count", "dm0_probe",
           "dm0_probe_read", "dm0_selftest_timeout", "dm0_sync", "dm0_device_error", "dm0_clear_error", "dm0_last_error",
           "dm0_destroy", "dm0_pack_e4m3_rows", "dm0_set_prefix_fp8", "dm0_op_quant_e4m3",
           "dm0_op_gemm_e4m3", "dm0_grad_floats", "dm0_train_step", "dm0_prepare")


class Dm0Config(ctypes.Structure):
    _fields_ = [("layers", c_int), ("hidden_v", c_int), ("inter_v", c_int), ("hidden_a", c_int),
                ("inter_a", c_int), ("n_q", c_int), ("n_kv", c_int), ("head_dim", c_int),
                ("chunk", c_int), ("action_dim", c_int), ("max_batch", c_int), ("max_prefix", c_int),
                ("rope_theta", c_float), ("rms_eps", c_float), ("time_mod", c_int)]


class Dm0Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{STATUS.get(status, status)}: {what}")
        self.status = status


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libdm0.so from the package directory (raises if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m vla_dual_expert_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "dm0_create": (c_int, [ctypes.POINTER(Dm0Config), ctypes.POINTER(P)]),
        "dm0_weights_bytes": (c_size_t, [ctypes.POINTER(Dm0Config)]),
        "dm0_load_weights": (c_int, [P, P, c_size_t]),
        "dm0_prefill": (c_int, [P, P, c_int, c_int, P]),
        "dm0_kv_view": (c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P)]),
        "dm0_kv_commit": (c_int, [P, c_int, c_int]),
        "dm0_denoise": (c_int, [P, P, c_int, P, P, P]),
        "dm0_infer_host": (c_int, [P, P, P, c_int, c_int, c_int, P, P]),
        "dm0_merged_layer": (c_int, [P, c_int, P, P, c_int, c_int, P, P, P, P, P]),
        "dm0_op_gemm": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, c_int, P]),
        "dm0_op_attention": (c_int, [P, P, P, P, c_int, P, P, c_int, P, c_int, c_int, c_int, P]),
        "dm0_attention_noalloc": (c_int, [P, P, P, c_int, P, P, c_int, P, c_int, c_int, c_int, c_int, c_int, c_int,
                                          P]),
        "dm0_debug_view": (c_int, [P, ctypes.c_char_p, ctypes.POINTER(P)]),
        "dm0_launch_count": (ctypes.c_uint64, [P]),
        "dm0_probe": (c_int, [P, c_int]),
        "dm0_probe_read": (c_int, [P, c_int, ctypes.POINTER(c_int), ctypes.POINTER(ctypes.c_double)]),
        "dm0_selftest_timeout": (c_int, [P, c_int, P]),
        "dm0_sync": (c_int, [P, P]),
        "dm0_device_error": (c_int, [P]),
        "dm0_clear_error": (c_int, [P]),
        "dm0_last_error": (ctypes.c_char_p, [P]),
        "dm0_destroy": (None, [P]),
        "dm0_pack_e4m3_rows": (c_int, [P, ctypes.c_int64, ctypes.c_int64, P, P]),
        "dm0_set_prefix_fp8": (c_int, [P, c_int, P]),
        "dm0_op_quant_e4m3": (c_int, [P, P, c_int, c_int, c_int, P, P, P, P, P]),
        "dm0_op_gemm_e4m3": (c_int, [P, P, P, P, P, P, c_int, c_int, c_int, P]),
        "dm0_grad_floats": (c_size_t, [P]),
        "dm0_prepare": (c_int, [P, c_int, c_int, c_int]),
        "dm0_train_step": (c_int, [P, P, P, P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def make_config(dims, max_batch: int, max_prefix: int, time_mod: bool = False) -> Dm0Config:
    """dims: any object with the model-shape attributes (layers, hidden_v, ...); time_mod selects the
    time-modulated action expert."""
    return Dm0Config(dims.layers, dims.hidden_v, dims.inter_v, dims.hidden_a, dims.inter_a, dims.n_q,
                     dims.n_kv, dims.head_dim, dims.chunk, dims.action_dim, max_batch, max_prefix,
                     float(dims.rope_theta), float(dims.rms_eps), 1 if time_mod else 0)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


# kernel sites of dm0_probe (include/dm0.h)
SITES = ("vlm_qkv", "vlm_attn", "vlm_o", "vlm_gateup", "vlm_down", "act_qkv", "act_attn", "act_o", "act_gateup",
         "act_down", "step", "loop")

LAYER_ORDER = (("attn_norm", "f32"), ("Wq", "bf16"), ("Wk", "bf16"), ("Wv", "bf16"), ("q_norm", "f32"),
               ("k_norm", "f32"), ("Wo", "bf16"), ("mlp_norm", "f32"), ("Wg", "bf16"), ("Wu", "bf16"),
               ("Wd", "bf16"))
HEAD_ORDER = (("W_in", "bf16"), ("b_in", "f32"), ("final_norm", "f32"), ("W_out", "bf16"), ("b_out", "f32"))
# time-modulated action expert: after the head, the time MLP and final modulator, then per layer the two
# pre-norm modulators
TIME_ORDER = (("W_ti", "bf16"), ("b_ti", "f32"), ("W_to", "bf16"), ("b_to", "f32"), ("W_mf", "bf16"),
              ("b_mf", "f32"))
MOD_ORDER = (("W_ma", "bf16"), ("b_ma", "f32"), ("W_mm", "bf16"), ("b_mm", "f32"))


def pack_weights(provider, layers: int, time_mod: bool = False) -> np.ndarray:
    """Serialise parameters into the blob layout dm0_load_weights reads.

    provider.layer(branch, l) -> dict and provider.head() -> dict of fp32 arrays
    (matrices [out][in]); branch 0 = VLM, 1 = action expert.  With time_mod, provider.time() and
    provider.mod(l) give the time MLP / final modulator and layer l's modulators.
    """
    def nbytes(arr, kind):
        return arr.size * (2 if kind == "bf16" else 4)

    tensors = []
    for br in (0, 1):
        for l in range(layers):
            w = provider.layer(br, l)
            tensors += [(w[n], k) for n, k in LAYER_ORDER]
    h = provider.head()
    tensors += [(h[n], k) for n, k in HEAD_ORDER]
    if time_mod:
        t = provider.time()
        tensors += [(t[n], k) for n, k in TIME_ORDER]
        for l in range(layers):
            m = provider.mod(l)
            tensors += [(m[n], k) for n, k in MOD_ORDER]
    total = sum(nbytes(a, k) for a, k in tensors)
    out = np.empty(total, dtype=np.uint8)
    off = 0
    for a, k in tensors:
        n = nbytes(a, k)
        src = _bf16_bits(a) if k == "bf16" else np.ascontiguousarray(a, dtype=np.float32)
        out[off:off + n] = src.reshape(-1).view(np.uint8)
        off += n
    return out


def grad_layout(dims):
    """(key, shape) of every tensor of the dm0_train_step gradient buffer, in order: (l, name) for the
    action layers, ("head", name) for the head (the action-expert part of the blob order)."""
    H, I, D, A = dims.hidden_a, dims.inter_a, dims.head_dim, dims.action_dim
    shapes = {"attn_norm": (H,), "Wq": (dims.n_q * D, H), "Wk": (dims.n_kv * D, H), "Wv": (dims.n_kv * D, H),
              "q_norm": (D,), "k_norm": (D,), "Wo": (H, dims.n_q * D), "mlp_norm": (H,), "Wg": (I, H),
              "Wu": (I, H), "Wd": (H, I)}
    out = [((l, name), shapes[name]) for l in range(dims.layers) for name, _ in LAYER_ORDER]
    head = {"W_in": (H, A), "b_in": (H,), "final_norm": (H,), "W_out": (A, H), "b_out": (A,)}
    out += [(("head", name), head[name]) for name, _ in HEAD_ORDER]
    return out


def unpack_grads(flat: np.ndarray, dims) -> dict:
    """Split a host copy of the gradient buffer into arrays keyed as in grad_layout."""
    out, off = {}, 0
    for key, shape in grad_layout(dims):
        n = int(np.prod(shape))
        out[key] = flat[off:off + n].reshape(shape)
        off += n
    assert off == flat.size, (off, flat.size)
    return out
