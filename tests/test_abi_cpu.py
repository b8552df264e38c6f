"""Host-side checks of the C ABI (no GPU needed): the library builds, loads
and exports every function include/mla.h declares; sizes, split planning,
status strings and argument rejection behave as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mla_split_kv_absorbed_b200 import build
    build.build()
    import mla_split_kv_absorbed_b200 as m
    return m


def header_functions():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    return re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = header_functions()
    assert set(names) == {"mla_quantize_fp8", "mla_partial_workspace_bytes", "mla_decode_partial",
                          "mla_combine", "mla_choose_splits", "mla_status_string"} | (
        set(names) - {"mla_quantize_fp8", "mla_partial_workspace_bytes", "mla_decode_partial",
                      "mla_combine", "mla_choose_splits", "mla_status_string"})
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(lib):
    handle = ctypes.CDLL(lib.LIB_PATH)
    for name in header_functions():
        assert hasattr(handle, name), name


def test_workspace_bytes(lib):
    assert lib.mla_partial_workspace_bytes(1, 1, 64, 64) == 64 * 64 * 513 * 4
    assert lib.mla_partial_workspace_bytes(16, 1, 64, 32) == 16 * 64 * 32 * 513 * 4
    assert lib.mla_partial_workspace_bytes(0, 1, 64, 32) == 0
    assert lib.mla_partial_workspace_bytes(1, 1, 64, -1) == 0


def test_status_strings(lib):
    assert lib.status_string(0) == "MLA_OK"
    assert lib.status_string(1) == "MLA_ERR_INVALID_ARG"
    assert lib.status_string(2) == "MLA_ERR_UNSUPPORTED"
    assert lib.status_string(3) == "MLA_ERR_CUDA"
    assert lib.status_string(99) == "MLA_ERR_UNKNOWN"


def test_choose_splits(lib):
    # batch 1 at 128K on 148 SMs: enough splits for about two waves
    s1 = lib.mla_choose_splits([131072], 1, 64, 148, 64)
    assert s1.tolist() == [64]
    s16 = lib.mla_choose_splits([131072] * 16, 1, 64, 148, 64)
    assert all(v == s16[0] for v in s16.tolist()) and 8 <= int(s16[0]) <= 64
    # short requests get one split, never more than max_splits, never zero
    with pytest.raises(lib.MlaError):
        lib.mla_choose_splits([1], 4, 64, 148, 64)  # seq_len below q_len
    s = lib.mla_choose_splits([4, 64, 1000, 262144], 4, 64, 148, 64).tolist()
    assert s[0] == 1 and s[1] == 1 and 1 <= s[2] <= 64 and s[3] <= 64
    # at least 16 pages per split
    s = lib.mla_choose_splits([64 * 16 * 5], 1, 16, 148, 256).tolist()
    assert s == [5]


def test_rejections_without_gpu(lib):
    h = lib.load()
    null = None
    # null pointers are rejected before any CUDA call
    assert h.mla_decode_partial(null, null, null, 0, 1.0, 1, null, 1, null, null, 1, 1, 1, 64,
                                1.0, null, null, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_combine(null, null, null, 1, 1, 1, 64, null, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_quantize_fp8(null, null, -1, 1.0, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_quantize_fp8(null, null, 0, 1.0, null) == lib.MLA_OK  # n = 0 is a no-op
    assert h.mla_choose_splits(null, 1, 1, 64, 148, 64, null) == lib.MLA_ERR_INVALID_ARG
    # unsupported shapes are reported as such (fake but aligned non-null pointers: nothing launches)
    fake = ctypes.c_void_p(1 << 20)
    args = [fake, fake, fake, 0, 1.0, 10, fake, 4, fake, fake, 4, 1]
    assert h.mla_decode_partial(*args, 5, 64, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # q_len 5
    assert h.mla_decode_partial(*args, 1, 24, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # H*q_len % 16
    assert h.mla_decode_partial(*args, 1, 256, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # H > 128
    # bad kv_dtype / bf16 with kv_scale != 1 / non-positive scale
    a2 = [fake, fake, fake, 7, 1.0, 10, fake, 4, fake, fake, 4, 1, 1, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial(*a2) == lib.MLA_ERR_INVALID_ARG
    a3 = [fake, fake, fake, 1, 0.5, 10, fake, 4, fake, fake, 4, 1, 1, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial(*a3) == lib.MLA_ERR_INVALID_ARG
    a4 = [fake, fake, fake, 0, -1.0, 10, fake, 4, fake, fake, 4, 1, 1, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial(*a4) == lib.MLA_ERR_INVALID_ARG
    # misaligned pointer
    mis = ctypes.c_void_p((1 << 20) + 4)
    a5 = [mis, fake, fake, 0, 1.0, 10, fake, 4, fake, fake, 4, 1, 1, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial(*a5) == lib.MLA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import mla_split_kv_absorbed_b200 as m
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(m, "_lib_handle", None)
    with pytest.raises(ImportError):
        m.load()


def test_partial_grid_plan(lib):
    # how mla_decode_partial lays out its CTAs (host logic, no GPU):
    # (ctas, pieces per cut unit, first cut unit, idle CTAs before the cut units)
    import mla_split_kv_absorbed_b200 as m
    FP8, BF16 = m.MLA_KV_FP8_E4M3, m.MLA_KV_BF16
    # batch 1, 64 heads, 64 splits: 64 units fill under half of 148 SMs -> every split cut in 2
    assert m.mla_partial_grid(1, 1, 64, 64, FP8, 148) == (128, 2, 0, 0)
    # a handful of units: cut in 4
    assert m.mla_partial_grid(1, 1, 64, 4, FP8, 148) == (16, 4, 0, 0)
    # batch 16, 32 splits: 512 units = 3 full waves + 68 -> the last 68 cut in 2
    assert m.mla_partial_grid(16, 1, 64, 32, FP8, 148) == (444 + 136, 2, 444, 0)
    # batch 4: 128 units, one wave more than half full -> no cut
    assert m.mla_partial_grid(4, 1, 64, 32, FP8, 148) == (128, 1, 128, 0)
    # q_len 4: 4 row groups x 64 splits x 8 -> last wave 124 > 74 -> no cut
    assert m.mla_partial_grid(8, 4, 64, 64, FP8, 148) == (2048, 1, 2048, 0)
    # odd first cut unit: one idle CTA keeps the 2-CTA clusters aligned
    assert m.mla_partial_grid(1, 1, 64, 150, FP8, 147) == (147 + 1 + 6, 2, 147, 1)
    # bf16 cache: one CTA per unit
    assert m.mla_partial_grid(1, 1, 16, 4, BF16, 148)[0] == 4
    with pytest.raises(m.MlaError):
        m.mla_partial_grid(0, 1, 64, 4, FP8, 148)
