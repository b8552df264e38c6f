"""Steps A2-A9 on the GPU: mla_decode_partial + mla_combine against the oracle.

Small cases span several 128-token tiles, ragged page tails, empty splits,
q_len 1-4 with causal masking (one query position per row group, and four
positions inside one group), 16 to 128 heads and NaN-poisoned pages around
the visible range.  Small grids exercise the cluster path in which every
split is cut across 2 or 4 CTAs; one case has a partly filled last wave whose
units alone are cut, and larger grids run several waves with or without such a
cut tail.  The full-size cases run the benchmark workloads in the
benchmark's launch configuration and compare sampled rows.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import (assert_attention_close, make_case, oracle_partials, oracle_rows,
                         run_gpu)

pytestmark = pytest.mark.gpu

SMALL = [
    ("b1_128k_fp8", dict(seq_lens=[1], splits=1)),
    ("b1_128k_fp8", dict(seq_lens=[63], splits=1)),
    ("b1_128k_fp8", dict(seq_lens=[128], splits=1)),
    ("b1_128k_fp8", dict(seq_lens=[129], splits=1)),
    ("b1_128k_fp8", dict(seq_lens=[700], splits=3)),
    ("b1_128k_fp8", dict(seq_lens=[2085], splits=4)),
    ("b1_128k_fp8", dict(seq_lens=[100], splits=8)),            # more splits than pages
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 1, 777], splits=4)),
    ("verify_q4_256k_fp8", dict(seq_lens=[1000, 4], splits=2)),  # q_len 4: four row groups
    ("verify_q4_256k_fp8", dict(seq_lens=[777], splits=3, H=16)),  # 4 positions in one group
    ("b16_128k_fp8", dict(seq_lens=[3000], splits=4, H=128)),
    ("b16_128k_fp8", dict(seq_lens=[1024], splits=4, H=16)),
    ("b16_128k_fp8", dict(seq_lens=[1500, 900], splits=2, H=32, q_len=2)),
    # 5 x 32 = 160 (group, split) units on 148 SMs: the last, partly filled
    # wave (12 units) is cut into 2-CTA clusters; short splits give empty pieces
    ("b16_128k_fp8", dict(seq_lens=[5000, 3000, 64, 4100, 777], splits=32)),
    # 310 units on 148 SMs: two full waves, then 14 one-tile units cut in 2
    # whose second pieces are empty
    ("b16_128k_fp8", dict(seq_lens=[3000, 2500, 700, 4100, 64, 1800, 2222, 3333, 900, 3900],
                          splits=31)),
    # q_len 4, 4 row groups: 208 units = one full wave + 60 units cut in 2
    ("verify_q4_256k_fp8", dict(seq_lens=[3000, 2000, 900, 4100], splits=13, H=64)),
    # 396 units: two full waves + 100, no cut
    ("b16_128k_fp8", dict(seq_lens=[2100, 3000, 130, 4000, 2500, 1, 3900, 2048, 640, 3500, 1200,
                                    2900], splits=33)),
]


def _ids(c):
    spec, ov = c
    return spec + "-" + "-".join(f"{k}{v if not isinstance(v, list) else len(v)}" for k, v in ov.items())


@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_decode_small_matches_oracle(case):
    spec, ov = case
    c = make_case(spec, **ov)
    w = c.w
    out, lse, part_o, part_lse, err = run_gpu(c)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                           o_ref, l_ref, what=str(case))
    # per-split partials: same split partition, same empty splits
    po_ref, pl_ref = oracle_partials(c, rows)
    po = part_o.cpu().numpy().reshape(len(rows), w.max_splits, 512)
    pl = part_lse.cpu().numpy().reshape(len(rows), w.max_splits)
    ns = w.num_splits.cpu().numpy()[rows // (w.q_len * w.H)]
    for r in range(len(rows)):
        S = ns[r]
        assert np.array_equal(np.isneginf(pl[r, :S]), np.isneginf(pl_ref[r, :S])), r
        fin = np.isfinite(pl_ref[r, :S])
        assert np.all(np.abs(pl[r, :S][fin] - pl_ref[r, :S][fin]) <= 1e-3 * np.maximum(1, np.abs(pl_ref[r, :S][fin])))
        scale = np.maximum(1.0, np.abs(po_ref[r, :S]).max(axis=1, keepdims=True))
        assert np.all(np.abs(po[r, :S] - po_ref[r, :S]) <= 1e-2 * scale), r
        assert np.all(po[r, :S][~fin] == 0)


def test_decode_is_bitwise_deterministic():
    c = make_case("b16_128k_fp8", seq_lens=[5000, 3000], splits=3)
    a = run_gpu(c)
    b = run_gpu(c)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[2], b[2])


@pytest.mark.parametrize("splits", [1, 7, 32])
def test_decode_split_count_changes_rounding_only(splits):
    # Split count (and with it whether a split is cut across a cluster)
    # changes the accumulation order, so results are not bit-identical across
    # split counts, but each stays within the tolerance of the same oracle.
    c = make_case("b1_128k_fp8", seq_lens=[3000], splits=splits)
    w = c.w
    out, lse, _, _, err = run_gpu(c)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                           o_ref, l_ref, what=f"splits={splits}")


def test_decode_reports_bad_page_ids():
    c = make_case("b1_128k_fp8", seq_lens=[300], splits=1)
    bt = c.dev["block_table"]
    bt[0, 2] = 10 ** 6  # outside the pool
    _, _, _, _, err = run_gpu(c)
    import mla_split_kv_absorbed_b200 as m
    assert err & m.DEVERR_BAD_PAGE


BF16 = [
    ("tiny", {}),                                                   # the tiny workload as specified
    ("tiny", dict(seq_lens=[1], splits=1)),
    ("tiny", dict(seq_lens=[129], splits=2)),
    ("tiny", dict(seq_lens=[100], splits=8)),                       # more splits than pages
    ("tiny", dict(seq_lens=[777, 64, 2000], splits=3, H=64)),
    ("tiny", dict(seq_lens=[1000], splits=2, H=64, q_len=4)),       # causal, four row groups
    ("tiny", dict(seq_lens=[555], splits=3, H=16, q_len=4)),        # causal inside one group
    ("b32_ragged_bf16", dict(seq_lens=[300, 4100, 70], splits=2)),  # 128 heads: two row groups
]


@pytest.mark.parametrize("case", BF16, ids=[_ids(c) for c in BF16])
def test_decode_bf16_small_matches_oracle(case):
    spec, ov = case
    c = make_case(spec, **ov)
    w = c.w
    out, lse, part_o, part_lse, err = run_gpu(c)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                           o_ref, l_ref, what=str(case))
    po_ref, pl_ref = oracle_partials(c, rows)
    pl = part_lse.cpu().numpy().reshape(len(rows), w.max_splits)
    ns = w.num_splits.cpu().numpy()[rows // (w.q_len * w.H)]
    for r in range(len(rows)):
        S = ns[r]
        assert np.array_equal(np.isneginf(pl[r, :S]), np.isneginf(pl_ref[r, :S])), r


FULL = [("b1_128k_fp8", 64), ("b16_128k_fp8", 32), ("verify_q4_256k_fp8", 24),
        ("b32_ragged_bf16", 32)]


@pytest.mark.parametrize("spec,n_rows", FULL)
def test_decode_full_size_sampled_rows(spec, n_rows):
    # Benchmark workloads in the benchmark's launch configuration.  The rows
    # compared are the first and last, one seeded row of every request (so
    # every request's splits, including the units of a cut last wave, feed a
    # compared row) and n_rows more seeded rows.
    c = make_case(spec, gen_device="cuda")
    w = c.w
    out, lse, _, _, err = run_gpu(c)
    assert err == 0
    R = w.B * w.q_len * w.H
    per_req = w.q_len * w.H
    rng = np.random.default_rng(123)
    one_per_request = np.arange(w.B) * per_req + rng.integers(0, per_req, size=w.B)
    rows = np.unique(np.concatenate([[0, R - 1], one_per_request,
                                     rng.choice(R, size=min(n_rows, R), replace=False)]))
    assert len(np.unique(rows // per_req)) == w.B
    o_ref, l_ref = oracle_rows(c, rows)
    o = out.float().cpu().numpy().reshape(R, 512)[rows]
    l = lse.cpu().numpy().reshape(R)[rows]
    assert_attention_close(o, l, o_ref, l_ref, what=spec)
