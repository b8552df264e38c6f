"""Failure detection on the GPU without a fault.

Every wait in the partial kernel is bounded (2 s, %globaltimer).  The library's
test hook leaves one KV load of the first CTA unissued, so the waits on it
run out: the kernel must report MLA_DEVERR_TIMEOUT through the caller's error
word, return within a bounded time, and leave the CUDA context usable (the next
decode matches the oracle).  No trap, no device assert, no bad address.
"""
import time

import numpy as np
import pytest
import torch

from gpu_helpers import assert_attention_close, make_case, oracle_rows, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # 128 splits of one page each: the grid fills more than half of the SMs,
    # so every split is one CTA (no cluster), and CTA 0 is split 0
    ("b1_128k_fp8", dict(seq_lens=[8192], splits=128)),
    # 4 splits: every split is cut into 4 pieces (clusters of 4 CTAs that
    # merge through distributed shared memory); CTA 0 is piece 0 of split 0,
    # and its peers wait for it at the cluster barrier
    ("b1_128k_fp8", dict(seq_lens=[8192], splits=4)),
]


@pytest.mark.parametrize("case", CASES, ids=["one-cta-units", "cluster-cut-units"])
def test_stalled_load_times_out_and_context_survives(case):
    import mla_split_kv_absorbed_b200 as m
    c = make_case(case[0], **case[1])
    w = c.w
    part_o, part_lse = m.alloc_partials(w.B, w.q_len, w.H, w.max_splits)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    prev = m.mla_debug_inject_stall(True)
    try:
        t0 = time.perf_counter()
        m.mla_decode_partial(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale,
                             c.dev["block_table"], c.dev["seq_lens"], c.dev["num_splits"],
                             w.max_splits, w.softmax_scale, part_o, part_lse, err)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        m.mla_debug_inject_stall(prev)
    word = int(err.item())
    print(f"[failure] error word {word:#x} after {elapsed:.2f} s")
    assert word & m.DEVERR_TIMEOUT, f"timeout not reported (error word {word:#x})"
    assert elapsed < 30.0, f"kernel took {elapsed:.1f} s to give up"

    # the context is intact: the same decode without the hook is correct
    out, lse, _, _, err2 = run_gpu(c)
    assert err2 == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512),
                           lse.cpu().numpy().reshape(-1), o_ref, l_ref, what="after timeout")


def test_single_launch_with_a_stalled_piece_reports_and_resets_its_counters():
    # The single-launch path: CTA 0's stalled load runs its waits out, the
    # other CTAs wait for it at the grid barrier (also bounded), the timeout
    # is reported, the workspace counters are back at zero, and the next
    # single launch on the same workspace is correct.
    import mla_split_kv_absorbed_b200 as m
    c = make_case("b1_128k_fp8", seq_lens=[8192], splits=4)
    w = c.w
    ws = m.alloc_fused_workspace(w.B, w.q_len, w.H)
    out = torch.empty((w.B, w.q_len, w.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.q_len, w.H), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def fused():
        m.mla_decode_fused(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale,
                           c.dev["block_table"], c.dev["seq_lens"], w.softmax_scale, ws, out,
                           lse, err)

    torch.cuda.synchronize()
    prev = m.mla_debug_inject_stall(True)
    try:
        t0 = time.perf_counter()
        fused()
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        m.mla_debug_inject_stall(prev)
    word = int(err.item())
    print(f"[failure] single launch: error word {word:#x} after {elapsed:.2f} s")
    assert word & m.DEVERR_TIMEOUT, f"timeout not reported (error word {word:#x})"
    assert elapsed < 30.0
    assert torch.count_nonzero(ws[:8]).item() == 0

    err.zero_()
    fused()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512),
                           lse.cpu().numpy().reshape(-1), o_ref, l_ref, what="single launch after timeout")
