"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/dm0.h declares, sizes its weight blob like the binding
packs it, and rejects malformed configurations before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

from synth import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from vla_dual_expert_b200 import build
    build.build()
    from vla_dual_expert_b200 import _abi
    return _abi, _abi.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "dm0.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dm0_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    abi, lib = _lib()
    declared = _declared()
    assert len(declared) >= 16
    assert sorted(abi.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_blob_size_matches_packer():
    abi, lib = _lib()
    d = I.TINY
    cfg = abi.make_config(d, 1, 64)
    w = I.Weights(d, seed=0)
    blob = abi.pack_weights(w, d.layers)
    assert blob.nbytes == lib.dm0_weights_bytes(ctypes.byref(cfg))


@pytest.mark.parametrize("dims", [I.TINY, I.DM0_BASE.replace(layers=2)])
def test_time_modulated_blob_size_matches_packer(dims):
    abi, lib = _lib()
    cfg = abi.make_config(dims, 1, 64, time_mod=True)
    w = I.Weights(dims, seed=0)
    blob = abi.pack_weights(w, dims.layers, time_mod=True)
    assert blob.nbytes == lib.dm0_weights_bytes(ctypes.byref(cfg))
    plain = lib.dm0_weights_bytes(ctypes.byref(abi.make_config(dims, 1, 64)))
    Ha, L = dims.hidden_a, dims.layers
    # time MLP 2 x [Ha][Ha] bf16 + 2 biases, final modulator [2Ha][Ha] + bias, 2 x [3Ha][Ha] + biases per layer
    assert blob.nbytes - plain == 2 * (2 * Ha * Ha + 2 * Ha * Ha) + 4 * (4 * Ha) + L * (2 * 6 * Ha * Ha + 4 * 6 * Ha)


def test_time_modulated_blob_tail_layout():
    abi, _ = _lib()
    d = I.TINY
    w = I.Weights(d, seed=5)
    blob = abi.pack_weights(w, d.layers, time_mod=True)
    plain = abi.pack_weights(w, d.layers)
    assert np.array_equal(blob[:plain.nbytes], plain)
    Ha = d.hidden_a
    wti = (blob[plain.nbytes:plain.nbytes + 2 * Ha * Ha].view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_array_equal(wti.reshape(Ha, Ha), w.time()["W_ti"])
    # the last tensor is the last layer's b_mm
    np.testing.assert_array_equal(blob[-4 * 3 * Ha:].view(np.float32), w.mod(d.layers - 1)["b_mm"])


def test_blob_layout_first_tensors():
    abi, _ = _lib()
    d = I.TINY
    w = I.Weights(d, seed=3, gain_jitter=0.1)
    blob = abi.pack_weights(w, d.layers)
    l0 = w.layer(0, 0)
    H = d.hidden_v
    np.testing.assert_array_equal(blob[:4 * H].view(np.float32), l0["attn_norm"])
    wq_bits = blob[4 * H:4 * H + 2 * l0["Wq"].size].view(np.uint16)
    back = (wq_bits.astype(np.uint32) << 16).view(np.float32).reshape(l0["Wq"].shape)
    np.testing.assert_array_equal(back, l0["Wq"])


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("n_kv", 3), ("hidden_v", 200), ("action_dim", 0),
                                         ("max_batch", 0), ("inter_a", 100), ("time_mod", 2)])
def test_create_rejects_bad_config_on_host(field, value):
    abi, lib = _lib()
    d = I.TINY
    cfg = abi.make_config(d, 1, 64)
    setattr(cfg, field, value)
    h = ctypes.c_void_p()
    st = lib.dm0_create(ctypes.byref(cfg), ctypes.byref(h))
    assert st == -2 and not h.value


def test_null_arguments_rejected():
    _, lib = _lib()
    assert lib.dm0_create(None, None) == -1
    assert lib.dm0_sync(None, None) == -1
    assert lib.dm0_last_error(None) == b"null context"
    lib.dm0_destroy(None)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from vla_dual_expert_b200 import _abi
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(ImportError):
        _abi.load_library()


def test_probe_site_names_match_the_header():
    """The binding's SITES tuple names dm0.h's DM0_SITE_* enum in order, one name per site."""
    from vla_dual_expert_b200 import SITES
    src = open(os.path.join(ROOT, "include", "dm0.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    sites = dict((m.group(1), int(m.group(2))) for m in re.finditer(r"DM0_SITE_([A-Z_]+)\s*=\s*(\d+)", src))
    count = sites.pop("COUNT")
    assert count == len(SITES) == len(sites)
    assert [n.lower() for n, _ in sorted(sites.items(), key=lambda kv: kv[1])] == list(SITES)


@pytest.mark.parametrize("dims", [I.TINY, I.DM0_BASE.replace(layers=3)])
def test_gradient_buffer_layout_matches_the_oracle_parameters(dims):
    """dm0_grad_floats covers exactly the action-expert and head parameters the training oracle
    differentiates, in the blob order."""
    abi, lib = _lib()
    cfg = abi.make_config(dims, 1, 64)
    n = lib.dm0_grad_floats(ctypes.byref(cfg))
    w = I.Weights(dims, seed=0)
    want = sum(np.size(v) for l in range(dims.layers) for v in w.layer(1, l).values())
    want += sum(np.size(v) for v in w.head().values())
    assert n == want
    layout = abi.grad_layout(dims)
    for (key, shape) in layout:
        ref = w.head()[key[1]] if key[0] == "head" else w.layer(1, key[0])[key[1]]
        assert tuple(shape) == np.shape(ref), key
    g = abi.unpack_grads(np.arange(n, dtype=np.float32), dims)
    assert g[(0, "attn_norm")][0] == 0 and g[("head", "b_out")][-1] == n - 1


def test_prepare_rejects_a_null_context():
    _, lib = _lib()
    assert lib.dm0_prepare(None, 1, 64, 10) == -1
