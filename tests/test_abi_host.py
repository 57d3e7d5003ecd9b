"""Host-only checks of the C ABI: the library loads without a GPU, exports
every entry point the header declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

from kv_cache_attention_qkv_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_attention_qkv_b200 import build

    build.build()
    return binding.load_library()


def _declared_symbols():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            src = open(os.path.join(HEADER_DIR, fn)).read()
            names |= set(re.findall(r"FC_API\s+[\w\s\*]*?\b(fc_\w+)\s*\(", src))
    return names


def test_header_declares_the_boundary():
    names = _declared_symbols()
    assert {"fc_create", "fc_step", "fc_topk_tracked", "fc_destroy", "fc_get_error",
            "fc_status_str"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(binding.EXPORTED) == _declared_symbols()


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.fc_status_str(code)
    assert lib.fc_status_str(12345) == b"unknown status"


def _cfg(**over):
    base = dict(hidden=32, n_heads=2, head_dim=16, rope_theta=1e4, dtype=binding.FC_DTYPE_FP32,
                max_batch=1, max_total_q=8, max_total_k=64, max_seqlen_q=8, max_pos=64, max_topk=4)
    base.update(over)
    return binding.FcConfig(**base)


@pytest.mark.parametrize("over,expect", [
    (dict(hidden=0), -1), (dict(head_dim=15), -1), (dict(rope_theta=0.0), -1),
    (dict(rope_theta=float("nan")), -1), (dict(dtype=7), -1), (dict(max_batch=0), -1),
    (dict(max_seqlen_q=9), -1), (dict(max_topk=-1), -1), (dict(max_topk=2048), -2),
    (dict(max_pos=1 << 20), -2), (dict(max_batch=5000), -2), (dict(head_dim=512), -2),
    (dict(n_heads=300), -1),
])
def test_create_rejects_bad_config_before_touching_the_device(lib, over, expect):
    h = ctypes.c_void_p()
    st = lib.fc_create(ctypes.byref(_cfg(**over)), ctypes.c_void_p(0x1000), ctypes.byref(h))
    assert st == expect
    assert not h.value


def test_create_rejects_null_and_misaligned_weights(lib):
    h = ctypes.c_void_p()
    assert lib.fc_create(ctypes.byref(_cfg()), None, ctypes.byref(h)) == -1
    assert lib.fc_create(ctypes.byref(_cfg()), ctypes.c_void_p(0x1001), ctypes.byref(h)) == -1
    assert lib.fc_create(None, ctypes.c_void_p(0x1000), ctypes.byref(h)) == -1
    assert lib.fc_create(ctypes.byref(_cfg()), ctypes.c_void_p(0x1000), None) == -1


def test_calls_on_a_null_handle_are_rejected(lib):
    vp = ctypes.c_void_p
    assert lib.fc_step(None, None, 1, vp(16), vp(16), vp(16), vp(16), 1, 1, vp(16), vp(16),
                       vp(16), None, 0) == -1
    assert lib.fc_topk_tracked(None, None, 1, 1, vp(16), vp(16), vp(16), vp(16), None, 1, vp(16)) == -1
    w = ctypes.c_int32()
    assert lib.fc_get_error(None, ctypes.byref(w)) == -1
    assert lib.fc_last_launch_count(None) == 0
    assert lib.fc_set_option(None, 1, 0) == -1
    lib.fc_destroy(None)  # no-op


def test_valid_config_without_a_device_reports_cuda_error(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p()
    st = lib.fc_create(ctypes.byref(_cfg()), ctypes.c_void_p(0x1000), ctypes.byref(h))
    assert st == -3 and not h.value


def test_binding_refuses_to_run_without_the_library(tmp_path):
    with pytest.raises(binding.FlashCacheError):
        binding.load_library(str(tmp_path / "missing.so"))


def _mcfg(**over):
    layer = _cfg(hidden=256, n_heads=2, head_dim=128, dtype=binding.FC_DTYPE_BF16)
    base = dict(layer=layer, n_layers=2, intermediate=512, vocab=1000, max_head_rows=8,
                rms_eps=1e-5, threshold=0.9)
    base.update(over)
    return binding.FcModelConfig(**base)


def _weights(n, addr=0x1000):
    arr = (binding.FcLayerWeights * n)()
    for i in range(n):
        for name in binding.LAYER_WEIGHT_NAMES:
            setattr(arr[i], name, addr)
    return arr


@pytest.mark.parametrize("over,expect", [
    (dict(n_layers=0), -1), (dict(intermediate=0), -1), (dict(vocab=0), -1),
    (dict(max_head_rows=0), -1), (dict(rms_eps=-1.0), -1), (dict(threshold=float("nan")), -1),
    (dict(intermediate=500), -2),  # SwiGLU tiles are 128 features wide
])
def test_model_create_rejects_bad_config_before_touching_the_device(lib, over, expect):
    m = ctypes.c_void_p()
    cfg = _mcfg(**over)
    st = lib.fc_model_create(ctypes.byref(cfg), _weights(max(cfg.n_layers, 1)),
                             ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), ctypes.byref(m))
    assert st == expect and not m.value


def test_model_create_rejects_unsupported_layer_shapes(lib):
    m = ctypes.c_void_p()
    for layer in (_cfg(hidden=256, n_heads=2, head_dim=128),  # fp32
                  _cfg(hidden=256, n_heads=3, head_dim=128, dtype=binding.FC_DTYPE_BF16),
                  _cfg(hidden=320, n_heads=2, head_dim=128, dtype=binding.FC_DTYPE_BF16),
                  _cfg(hidden=256, n_heads=4, head_dim=64, dtype=binding.FC_DTYPE_BF16)):
        cfg = _mcfg(layer=layer)
        st = lib.fc_model_create(ctypes.byref(cfg), _weights(2), ctypes.c_void_p(0x1000),
                                 ctypes.c_void_p(0x1000), ctypes.byref(m))
        assert st == -2 and not m.value


def test_model_create_rejects_null_and_misaligned_weights(lib):
    m = ctypes.c_void_p()
    cfg = _mcfg()
    assert lib.fc_model_create(ctypes.byref(cfg), None, ctypes.c_void_p(0x1000),
                               ctypes.c_void_p(0x1000), ctypes.byref(m)) == -1
    assert lib.fc_model_create(ctypes.byref(cfg), _weights(2, 0x1008), ctypes.c_void_p(0x1000),
                               ctypes.c_void_p(0x1000), ctypes.byref(m)) == -1
    assert lib.fc_model_create(ctypes.byref(cfg), _weights(2), None, ctypes.c_void_p(0x1000),
                               ctypes.byref(m)) == -1


def test_noalloc_rejects_sizes_beyond_its_limits_before_any_cuda_call(lib):
    """Sizes past the static scratch, or an importance sum that could leave its
    fixed-point range (heads x query rows >= 2^23), are refused on the host."""
    vp = ctypes.c_void_p(16)
    bf16 = 0
    assert lib.fc_attention_noalloc(None, bf16, 1, 1, 128, vp, vp, vp, 1, 65536 + 1, vp, vp, vp,
                                    vp) == -2
    assert lib.fc_attention_noalloc(None, bf16, 1, 128, 128, vp, vp, vp, 65536, 16, vp, vp, vp,
                                    vp) == -2
    assert lib.fc_attention_noalloc(None, bf16, 1, 1, 257, vp, vp, vp, 1, 16, vp, vp, vp, vp) == -2
    assert lib.fc_attention_noalloc(None, 7, 1, 1, 128, vp, vp, vp, 1, 16, vp, vp, vp, vp) == -1
    assert lib.fc_attention_noalloc(None, bf16, 1, 1, 128, vp, None, vp, 1, 16, vp, vp, vp,
                                    vp) == -1


def test_model_and_host_step_calls_on_null_handles_are_rejected(lib):
    vp = ctypes.c_void_p
    arr = (ctypes.c_void_p * 2)(16, 16)
    assert lib.fc_model_step(None, None, 1, vp(16), vp(16), vp(16), vp(16), 1, 1, arr, arr, None,
                             0, None, None, None, None, None) == -1
    assert lib.fc_decode_iteration(None, None, 1, vp(16), 1, arr, arr, vp(16), 0, 1, 1, vp(16),
                                   vp(16), vp(16), vp(16), vp(16), vp(16), None) == -1
    assert lib.fc_model_lm_head(None, None, vp(16), 1, vp(16), vp(16), vp(16)) == -1
    assert lib.fc_step_host(None, None, 1, vp(16), vp(16), vp(16), vp(16), 1, 1, vp(16), vp(16),
                            vp(16), vp(16), None, 1, vp(16), vp(16)) == -1
    assert lib.fc_host_sync(None, None) == -1
    assert lib.fc_model_layer_handle(None) is None
    lib.fc_model_destroy(None)  # no-op
