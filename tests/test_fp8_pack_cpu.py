"""dm0_pack_e4m3_rows (host code of the C ABI, the weight format of the FP8 prefix-MLP GEMMs)
against the oracle's E4M3 definition (reading R11): bit-exact codes and the per-row scales.

The codes are decoded with torch's float8_e4m3fn view (a library routine), so the check covers the
bit layout as well as the rounding."""
import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O


def _decode(codes):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _oracle(x):
    """Codes (as values) and scales of the oracle, from the same fp32 input."""
    q, s = O.quantize_rows(x.astype(np.float64))
    return q, s[:, 0]


@pytest.fixture(scope="module")
def pack():
    from vla_dual_expert_b200 import pack_e4m3_rows
    return pack_e4m3_rows


def test_random_rows_bit_exact(pack):
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((64, 257)) * np.exp2(rng.uniform(-20, 20, size=(64, 1)))).astype(np.float32)
    codes, scales = pack(x)
    q, s = _oracle(x)
    assert np.array_equal(_decode(codes), q)
    assert np.array_equal(scales, s.astype(np.float32))


def test_weight_like_rows_and_edge_rows(pack):
    rng = np.random.default_rng(22)
    w = (rng.standard_normal((12, 96)) * 0.02).astype(np.float32)
    w[3] = 0.0                                            # all-zero row: scale 1, codes 0
    w[4, :] = 0.0
    w[4, 7] = -3.5                                        # one nonzero: it maps to exactly -448
    w[5, :] = np.float32(2.0 ** -30) * np.arange(96)      # tiny values, wide relative range
    codes, scales = pack(w)
    q, s = _oracle(w)
    assert np.array_equal(_decode(codes), q)
    assert scales[3] == 1.0 and not codes[3].any()
    assert _decode(codes)[4, 7] == -448.0 and scales[4] == np.float32(3.5 / 448.0)
    # the dequantised matrix is within half a unit of the 3-bit mantissa of each normal entry
    deq = _decode(codes) * scales[:, None].astype(np.float64)
    big = np.abs(w / scales[:, None]) >= 2.0 ** -6
    rel = np.abs(deq - w)[big] / np.abs(w)[big]
    assert np.max(rel) <= 2.0 ** -4 + 1e-6


def test_rejects_bad_arguments(pack):
    from vla_dual_expert_b200 import Dm0Error
    with pytest.raises(Dm0Error):
        pack(np.array([[1.0, np.nan]], np.float32))
    with pytest.raises(Dm0Error):
        pack(np.array([[np.inf]], np.float32))
    with pytest.raises(ValueError):
        pack(np.zeros(4, np.float32))
