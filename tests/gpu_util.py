"""Helpers shared by the GPU tests (device views of raw pointers, error metric)."""
import numpy as np
import torch


class _Cai:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"data": (int(ptr), False), "shape": tuple(shape), "typestr": typestr,
                                         "version": 2}


def device_view_bf16(ptr: int, shape) -> torch.Tensor:
    """Zero-copy torch view (bf16) of a device buffer the library owns."""
    return torch.as_tensor(_Cai(ptr, shape, "<u2"), device="cuda").view(torch.bfloat16)


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    """bf16-representable fp32 values -> CUDA bf16 (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def to_dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rms(x) -> float:
    return float(np.sqrt(np.mean(np.square(np.asarray(x, np.float64)))))


def rel_err(got, ref) -> float:
    """max |got - ref| / RMS(ref): the parity metric of this library's tests."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    e = float(np.max(np.abs(got - ref)) / max(rms(ref), 1e-30))
    print(f"  parity max|d|/rms = {e:.3e}  shape={ref.shape}")
    return e


def check_fp(got, ref, tol: float, what: str = ""):
    """fp32 outputs: max |got - ref| <= tol * RMS(ref)."""
    e = rel_err(got, ref)
    assert e <= tol, f"{what}: max|d|/rms {e:.3e} > {tol:.1e}"


def check_bf16(got, ref, atol_rms: float, what: str = "", rms_tol: float = 5e-3):
    """Tensors stored in bf16: |d_i| <= atol_rms * RMS(ref) + 2^-8 |ref_i| for every element
    (the second term is one bf16 rounding step of the stored value, 2^-9, doubled), and the
    RMS of the error <= rms_tol * RMS(ref)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values in GPU output"
    r = max(rms(ref), 1e-30)
    d = np.abs(got - ref)
    ratio = float(np.max(d / (atol_rms * r + 2.0 ** -8 * np.abs(ref))))
    rms_e = rms(d) / r
    print(f"  bf16 parity {what}: max ratio {ratio:.3f}, rms err {rms_e:.3e}, max|d|/rms {np.max(d) / r:.3e}")
    assert ratio <= 1.0 and rms_e <= rms_tol, f"{what}: ratio {ratio:.3f}, rms err {rms_e:.3e}"
