"""Host-side checks of the C ABI (no GPU needed): the library builds, loads
and exports every function include/mla.h declares; sizes, split planning,
status strings and argument rejection behave as documented."""
import ctypes
import os
import re

import numpy as np
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
    required = {"mla_quantize_fp8", "mla_partial_workspace_bytes", "mla_decode_partial",
                "mla_combine", "mla_choose_splits", "mla_status_string", "mla_device_error_status"}
    assert required <= set(names)
    assert len(names) == len(set(names))


def test_binding_exports_match_header():
    import mla_split_kv_absorbed_b200 as m
    assert set(m.EXPORTS) == set(header_functions())


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


def test_choose_splits_follows_the_length_rule(lib):
    # the reading the ragged workload uses: about num_sms equal splits per batch
    from mla_split_kv_absorbed_b200 import workloads as wl
    rng = np.random.default_rng(7)
    lens = np.concatenate([[1, 2047, 2048, 2049, 4096, 131072, 262144],
                           rng.integers(1, 300000, size=500)]).astype(np.int32)
    for sms in (1, 148, 1000):
        got = lib.mla_choose_splits(lens, sms, 64).numpy()
        assert np.array_equal(got, np.array(wl.splits_by_length(lens.tolist(), sms, 64)))
    # the formula written out: T = max(2048, ceil(sum / max(1, SMs - B))), ceil(L / T) in [1, max]
    L64 = lens.astype(np.int64)
    for sms, max_splits in ((148, 64), (148, 7), (1000, 256), (1, 1)):
        T = max(2048, -(-int(L64.sum()) // max(1, sms - len(lens))))
        want = np.clip(-(-L64 // T), 1, max_splits)
        assert np.array_equal(lib.mla_choose_splits(lens, sms, max_splits).numpy(), want)
    assert lib.mla_choose_splits([131072], 148, 64).tolist() == [64]  # the batch-1 64-way split
    assert lib.mla_choose_splits([131072] * 16, 148, 64).tolist() == [9] * 16  # one wave
    assert lib.mla_choose_splits([1024], 148, 64).tolist() == [1]
    # at most num_sms splits (one wave at one row group) for a batch of B < SMs
    for _ in range(20):
        big = rng.integers(1, 262145, size=int(rng.integers(1, 100))).astype(np.int32)
        n = int(lib.mla_choose_splits(big, 148, 256).sum())
        assert n <= 148 or int(big.sum()) <= 2048 * len(big)
    with pytest.raises(lib.MlaError):
        lib.mla_choose_splits([0], 148, 64)  # empty request
    with pytest.raises(lib.MlaError):
        lib.mla_choose_splits([10], 0, 64)


def test_device_error_status(lib):
    assert lib.mla_device_error_status(0) == lib.MLA_OK
    for bit in (lib.DEVERR_BAD_PAGE, lib.DEVERR_BAD_SEQLEN, lib.DEVERR_TIMEOUT,
                lib.DEVERR_BAD_SPLITS, lib.DEVERR_SMEM_ALIGN, 0x7FFFFFFF, -1):
        assert lib.mla_device_error_status(bit) == lib.MLA_ERR_DEVICE
    assert lib.status_string(lib.MLA_ERR_DEVICE) == "MLA_ERR_DEVICE"


def test_rejections_without_gpu(lib):
    h = lib.load()
    null = None
    # null pointers are rejected before any CUDA call
    assert h.mla_decode_partial(null, null, null, 0, 1.0, 1, null, 1, null, null, 1, 1, 1, 64,
                                1.0, null, null, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_combine(null, null, null, 1, 1, 1, 64, null, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_quantize_fp8(null, null, -1, 1.0, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_quantize_fp8(null, null, 0, 1.0, null) == lib.MLA_OK  # n = 0 is a no-op
    assert h.mla_choose_splits(null, 1, 148, 64, null) == lib.MLA_ERR_INVALID_ARG
    # unsupported shapes are reported as such (fake but aligned non-null pointers: nothing launches)
    fake = ctypes.c_void_p(1 << 20)
    args = [fake, fake, fake, 0, 1.0, 10, fake, 4, fake, fake, 4, 1]
    assert h.mla_decode_partial(*args, 5, 64, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # q_len 5
    assert h.mla_decode_partial(*args, 1, 24, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # H*q_len % 16
    assert h.mla_decode_partial(*args, 1, 528, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # rows > 512
    assert h.mla_decode_partial(*args, 4, 144, 1.0, fake, fake, null, null) == lib.MLA_ERR_UNSUPPORTED  # q_len*H > 512
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


def test_fused_workspace_and_rejections_without_gpu(lib):
    h = lib.load()
    null = None
    # one wave of one CTA per (64-row group, split, request), at most 256 splits
    assert h.mla_fused_splits(1, 1, 64, 148) == 148
    assert h.mla_fused_splits(16, 1, 64, 148) == 9
    assert h.mla_fused_splits(2, 4, 64, 148) == 18     # 4 row groups per request
    assert h.mla_fused_splits(148, 1, 64, 148) == 1
    assert h.mla_fused_splits(149, 1, 64, 148) == 0
    assert h.mla_fused_splits(1, 1, 16, 1000) == 256
    assert h.mla_fused_splits(0, 1, 64, 148) == 0
    assert h.mla_fused_splits(1, 1, 64, 0) == 0
    # counters (256 bytes) + O (512 fp16) and LSE (fp32) per (row, split)
    per = 512 * 2 + 4
    assert h.mla_fused_workspace_bytes(1, 1, 64, 148) == 256 + 64 * 148 * per
    assert h.mla_fused_workspace_bytes(16, 1, 64, 148) == 256 + 16 * 64 * 9 * per
    assert h.mla_fused_workspace_bytes(2, 4, 16, 148) == 256 + 2 * 4 * 16 * 74 * per  # one row group
    assert h.mla_fused_workspace_bytes(149, 1, 64, 148) == 0
    assert h.mla_fused_workspace_bytes(0, 1, 64, 148) == 0
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    base = [fake, fake, fake, 0, 1.0, 10, fake, 4, fake, 1]
    # null workspace / output, misaligned workspace
    assert h.mla_decode_fused(*base, 1, 64, 1.0, null, big, fake, null, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_decode_fused(*base, 1, 64, 1.0, fake, big, null, null, null, null) == lib.MLA_ERR_INVALID_ARG
    mis = ctypes.c_void_p((1 << 20) + 8)
    assert h.mla_decode_fused(*base, 1, 64, 1.0, mis, big, fake, null, null, null) == lib.MLA_ERR_INVALID_ARG
    # a bf16 cache has no single launch
    b16 = [fake, fake, fake, 1, 1.0, 10, fake, 4, fake, 1]
    assert h.mla_decode_fused(*b16, 1, 64, 1.0, fake, big, fake, null, null, null) == lib.MLA_ERR_UNSUPPORTED
    # a workspace one byte short (the SM count without a GPU is taken as 148)
    need = h.mla_fused_workspace_bytes(1, 1, 64, 148)
    assert h.mla_decode_fused(*base, 1, 64, 1.0, fake, need - 1, fake, null, null, null) == lib.MLA_ERR_INVALID_ARG
    # the shared checks of mla_decode_partial apply
    assert h.mla_decode_fused(*base, 5, 64, 1.0, fake, big, fake, null, null, null) == lib.MLA_ERR_UNSUPPORTED


def test_merge_plan_hook_without_gpu(lib):
    h = lib.load()
    for v, gpi in [(3, 1), (4, 4), (0, 1), (8, 6), (1, 0), (-1, 2)]:
        assert h.mla_debug_merge_plan(v, gpi) == lib.MLA_ERR_INVALID_ARG
    for v in (1, 2, 4):
        for gpi in (1, 2, 3, 6):
            assert h.mla_debug_merge_plan(v, gpi) == lib.MLA_OK
    assert h.mla_debug_merge_plan(0, 0) == lib.MLA_OK


def test_q8_rejections_without_gpu(lib):
    h = lib.load()
    null = None
    fake = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    rest = [fake, 1.0, 10, fake, 4, fake, fake, 4, 1, 1, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial_q8(null, 1.0, *rest) == lib.MLA_ERR_INVALID_ARG      # no query
    assert h.mla_decode_partial_q8(mis, 1.0, *rest) == lib.MLA_ERR_INVALID_ARG       # misaligned
    assert h.mla_decode_partial_q8(fake, 0.0, *rest) == lib.MLA_ERR_INVALID_ARG      # q_scale <= 0
    assert h.mla_decode_partial_q8(fake, float("inf"), *rest) == lib.MLA_ERR_INVALID_ARG
    bad_rows = [fake, 1.0, 10, fake, 4, fake, fake, 4, 1, 5, 64, 1.0, fake, fake, null, null]
    assert h.mla_decode_partial_q8(fake, 1.0, *bad_rows) == lib.MLA_ERR_UNSUPPORTED  # q_len 5


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


def test_rope_table_matches_the_oracle_bit_for_bit(lib, oracle_lib):
    # the library's host table builder and the oracle's are separate code for
    # the same definition (angle, cosine and sine in double, rounded once)
    t_lib = lib.mla_rope_cos_sin_table(5000).numpy()
    t_ora = oracle_lib.rope_table(5000)
    assert np.array_equal(t_lib, t_ora)
    assert np.array_equal(lib.mla_rope_cos_sin_table(70, 500000.0).numpy(),
                          oracle_lib.rope_table(70, 500000.0))
    with pytest.raises(lib.MlaError):
        lib.mla_rope_cos_sin_table(0)


def test_append_rejections_without_gpu(lib):
    h = lib.load()
    null = None
    fake = ctypes.c_void_p(1 << 20)
    # null pointers, bad sizes, misalignment, bad scale: rejected before any launch
    assert h.mla_append_kv_fp8(null, fake, fake, 10, fake, 4, fake, 1, 1, 1.0, fake, 10, null,
                               null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_append_kv_fp8(fake, fake, fake, 10, fake, 4, fake, 0, 1, 1.0, fake, 10, null,
                               null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_append_kv_fp8(ctypes.c_void_p((1 << 20) + 8), fake, fake, 10, fake, 4, fake, 1, 1,
                               1.0, fake, 10, null, null) == lib.MLA_ERR_INVALID_ARG
    assert h.mla_append_kv_fp8(fake, fake, fake, 10, fake, 4, fake, 1, 1, -1.0, fake, 10, null,
                               null) == lib.MLA_ERR_INVALID_ARG
    # nothing to append is a no-op
    assert h.mla_append_kv_fp8(null, null, null, 10, null, 4, null, 1, 0, 1.0, null, 10, null,
                               null) == lib.MLA_OK
