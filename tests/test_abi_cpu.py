"""The C-ABI library loads on a machine without a GPU, exports every symbol the header
declares, and does its host-side sizing and validation without touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hybrid_sliding_window_swa_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return hs.load_library()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "hswa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^HSWA_API\s+(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for n in ["kv_pool_create", "swa_prefill_fwd", "full_prefill_fwd", "hybrid_decode_fwd", "window_safe_len"]:
        assert n in names
    assert set(names) == set(hs.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", hs.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in _declared_functions():
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_layout_matches_kv_bytes_formula(lib):
    for desc in [hs.PoolDesc(60, 10, 128, 8, 128, 1, (1 << 20) // 64),
                 hs.PoolDesc(6, 1, 128, 8, 128, 256, 200_000),
                 hs.PoolDesc(1, 0, 4096, 8, 128, 2, 0),
                 hs.PoolDesc(1, 1, 1, 1, 64, 3, 7)]:
        total, swa, full = hs.kv_pool_layout(desc)
        o_swa, o_full = oracle.pool_bytes(desc.n_swa_layers, desc.n_full_layers, desc.window, desc.n_kv_heads,
                                          desc.head_dim, desc.page_size, desc.max_seqs, desc.pages_per_full_layer)
        assert swa == (o_swa + 255) // 256 * 256
        assert full == (o_full + 255) // 256 * 256
        assert total == swa + full + 256


def test_fp8_layout_halves_the_entries_and_adds_the_scales(lib):
    # FP8 E4M3 entries take one byte: the KV-bytes formula with 1-byte elements, plus
    # [4][layers][Hkv] float32 scales
    for args in [(60, 10, 128, 8, 128, 1, (1 << 20) // 64), (6, 1, 128, 8, 128, 256, 200_000), (1, 1, 1, 1, 64, 3, 7)]:
        total, swa, full = hs.kv_pool_layout(hs.PoolDesc(*args, kv_format=hs.HSWA_KV_FP8_E4M3))
        o_swa, o_full = oracle.pool_bytes(*args[:5], 64, args[5], args[6], elem_bytes=1)
        assert swa == (o_swa + 255) // 256 * 256 and full == (o_full + 255) // 256 * 256
        scales = (4 * 4 * (args[0] + args[1]) * args[3] + 255) // 256 * 256
        assert total == swa + full + scales + 256
    with pytest.raises(hs.HswaError) as e:
        hs.kv_pool_layout(hs.PoolDesc(1, 1, 128, 8, 128, 1, 4, kv_format=7))
    assert e.value.code == hs.HSWA_ERR_INVALID_ARG


def test_config5_footprint_is_60W_plus_10N_slots(lib):
    n = 1 << 20
    _, swa, full = hs.kv_pool_layout(hs.PoolDesc(60, 10, 128, 8, 128, 1, n // 64))
    per_slot = 2 * 8 * 128 * 2
    assert (swa + full) == (60 * 128 + 10 * n) * per_slot
    assert abs((swa + full) / (70 * n * per_slot) - oracle.hybrid_kv_ratio(60, 10, 128, n)) < 1e-12


def test_swa_pool_bytes_do_not_depend_on_n(lib):
    a = hs.kv_pool_layout(hs.PoolDesc(60, 10, 128, 8, 128, 4, 1000))[1]
    b = hs.kv_pool_layout(hs.PoolDesc(60, 10, 128, 8, 128, 4, 1000000))[1]
    assert a == b


@pytest.mark.parametrize("field,value,code", [
    ("window", 0, hs.HSWA_ERR_INVALID_ARG),
    ("head_dim", 96, hs.HSWA_ERR_UNSUPPORTED_SHAPE),
    ("page_size", 32, hs.HSWA_ERR_UNSUPPORTED_SHAPE),
    ("n_kv_heads", 0, hs.HSWA_ERR_INVALID_ARG),
    ("n_swa_layers", -1, hs.HSWA_ERR_INVALID_ARG),
])
def test_layout_rejects_bad_descriptors(lib, field, value, code):
    kw = dict(n_swa_layers=1, n_full_layers=1, window=128, n_kv_heads=8, head_dim=128, max_seqs=1,
              pages_per_full_layer=4)
    kw[field] = value
    with pytest.raises(hs.HswaError) as e:
        hs.kv_pool_layout(hs.PoolDesc(**kw))
    assert e.value.code == code
    assert hs.hswa_last_error() != ""


def test_null_arguments_are_rejected_on_the_host(lib):
    assert lib.kv_pool_create(None, None, 0, None) == hs.HSWA_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    d = hs.PoolDesc(1, 0, 128, 1, 64, 1, 0).c()
    assert lib.kv_pool_create(ctypes.byref(d), None, 1 << 20, ctypes.byref(h)) == hs.HSWA_ERR_INVALID_ARG
    assert lib.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(0x1001), 1 << 20, ctypes.byref(h)) == \
        hs.HSWA_ERR_INVALID_ARG  # misaligned
    assert lib.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(0x100000), 16, ctypes.byref(h)) == \
        hs.HSWA_ERR_OUT_OF_MEMORY
    assert lib.swa_prefill_fwd(None, 0, None, None, None, None, 1, 1, None, None, 1, None) == \
        hs.HSWA_ERR_INVALID_ARG
    assert lib.window_safe_len(None, None, None, 0, 1, None, None) == hs.HSWA_ERR_INVALID_ARG
    assert lib.window_safe_len(None, None, None, 128, 0, None, None) == hs.HSWA_OK
    assert lib.kv_pool_destroy(None) == hs.HSWA_OK


def test_product_package_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "hybrid_sliding_window_swa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "oracle." not in txt and "liboracle" not in txt, f
