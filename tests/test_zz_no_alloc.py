"""GPU test of mla_decode_noalloc, the allocation-free decode entry point.

Callers that cannot allocate device memory (a plugin whose host owns the
device memory pool, a loop that must not call cudaMalloc because it may
synchronise the device) pass only inputs and outputs; the split partials live
in the library's own fixed device array.  This file is collected last so a
run that stops at the first failure has run every other test first; it also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import (LSE_TOL, O_MAX_ABS, O_REL_L2, assert_attention_close, bf16_half_ulp,
                         make_case, oracle_rows, run_gpu)

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, c):
    w = c.w
    out = torch.full((w.B, w.q_len, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.q_len, w.H), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kv_dtype = 0 if c.kv_dev.dtype == torch.uint8 else 1
    fn = lib.mla_decode_noalloc
    fn.restype = ctypes.c_int
    st = fn(_p(c.dev["q_nope"]), _p(c.dev["q_rope"]), _p(c.kv_dev), ctypes.c_int(kv_dtype),
            ctypes.c_float(w.kv_scale), ctypes.c_int64(c.kv_dev.shape[0]), _p(c.dev["block_table"]),
            ctypes.c_int(c.dev["block_table"].shape[1]), _p(c.dev["seq_lens"]),
            _p(c.dev["num_splits"]), ctypes.c_int(w.max_splits), ctypes.c_int(w.B),
            ctypes.c_int(w.q_len), ctypes.c_int(w.H), ctypes.c_float(w.softmax_scale), _p(out),
            _p(lse), _p(err), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, out, lse, int(err.item())


def _assert_close(out, lse, ref_out, ref_lse):
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref_out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    max_abs = float(np.maximum(np.abs(o - r) - bf16_half_ulp(r), 0.0).max())
    rel = float(np.linalg.norm(o - r) / max(np.linalg.norm(r), 1e-30))
    assert max_abs <= O_MAX_ABS and rel <= O_REL_L2, (max_abs, rel)
    l, lr = lse.cpu().numpy().astype(np.float64), ref_lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(l), np.isneginf(lr))
    fin = np.isfinite(lr)
    assert np.all(np.abs(l[fin] - lr[fin]) <= LSE_TOL * np.maximum(1.0, np.abs(lr[fin])))


def test_noalloc_matches_partial_plus_combine_on_two_calls_in_a_row():
    import mla_split_kv_absorbed_b200 as m
    lib = m.load()
    cases = [make_case("b1_128k_fp8", seq_lens=[5000], splits=16),
             make_case("b16_128k_fp8", seq_lens=[3000, 700], splits=8, q_len=2, H=32)]
    for c in cases:  # two different calls in a row share the library's scratch array
        ref_out, ref_lse, _, _, ref_err = run_gpu(c)
        st, out, lse, err = _noalloc(lib, c)
        assert st == m.MLA_OK, m.status_string(st)
        assert err == 0 and ref_err == 0
        _assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("spec,ov", [
    # bf16 cache through the shared scratch
    ("tiny", dict(seq_lens=[777, 2000], splits=3, H=64)),
    # FP8, 128 splits x 64 heads = the whole scratch; more than half the SMs
    # are busy, so every split is one CTA (no cluster)
    ("b1_128k_fp8", dict(seq_lens=[16384], splits=128)),
])
def test_noalloc_matches_the_oracle(spec, ov):
    import mla_split_kv_absorbed_b200 as m
    lib = m.load()
    c = make_case(spec, **ov)
    w = c.w
    for _ in range(2):  # the second call reuses scratch the first one filled
        st, out, lse, err = _noalloc(lib, c)
        assert st == m.MLA_OK, m.status_string(st)
        assert err == 0
        rows = np.arange(w.B * w.q_len * w.H)
        o_ref, l_ref = oracle_rows(c, rows)
        assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                               o_ref, l_ref, what=f"noalloc {spec}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    import mla_split_kv_absorbed_b200 as m
    lib = m.load()
    fake = ctypes.c_void_p(1 << 20)
    fn = lib.mla_decode_noalloc
    fn.restype = ctypes.c_int
    # 2 x 64 heads x 65 splits = 8320 row-splits > 8192: rejected before any launch
    st = fn(fake, fake, fake, 0, ctypes.c_float(1.0), ctypes.c_int64(10), fake, 4, fake, fake, 65,
            2, 1, 64, ctypes.c_float(1.0), fake, fake, None, None)
    assert st == m.MLA_ERR_SCRATCH_LIMIT
    assert m.status_string(st) == "MLA_ERR_SCRATCH_LIMIT"
