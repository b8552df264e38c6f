"""Single-launch decode (mla_decode_fused) on the GPU against the oracle.

The fused path runs steps A2-A9 in one cooperative launch: every piece of
every unit writes its own partial, the grid meets at a barrier, and the grid
merges the partials.  It applies when the grid fits on the GPU at once (every
unit cut into 2 or 4 pieces), as at batch 1; other shapes are refused with
MLA_ERR_UNSUPPORTED.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_attention_close, make_case, oracle_rows, run_gpu

pytestmark = pytest.mark.gpu

SMALL = [
    ("b1_128k_fp8", dict(seq_lens=[2085], splits=4)),             # 4 units, 4 pieces each
    ("b1_128k_fp8", dict(seq_lens=[700], splits=3)),              # pieces of one tile and empty ones
    ("b1_128k_fp8", dict(seq_lens=[100], splits=8)),              # more splits than pages
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 1, 777], splits=4)),
    ("verify_q4_256k_fp8", dict(seq_lens=[777], splits=3, H=16)),  # q_len 4, causal
    ("verify_q4_256k_fp8", dict(seq_lens=[1000, 4], splits=2)),  # four row groups
]


def run_fused(c, workspace=None):
    import mla_split_kv_absorbed_b200 as m
    w = c.w
    if workspace is None:
        workspace = m.alloc_fused_workspace(w.B, w.q_len, w.H, w.max_splits)
    out = torch.full((w.B, w.q_len, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.q_len, w.H), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mla_decode_fused(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale, c.dev["block_table"],
                       c.dev["seq_lens"], c.dev["num_splits"], w.max_splits, w.softmax_scale,
                       workspace, out, lse, err)
    torch.cuda.synchronize()
    return out, lse, int(err.item()), workspace


def _ids(c):
    spec, ov = c
    return spec + "-" + "-".join(f"{k}{v if not isinstance(v, list) else len(v)}" for k, v in ov.items())


@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_fused_small_matches_oracle_and_two_launch_path(case):
    spec, ov = case
    c = make_case(spec, **ov)
    w = c.w
    out, lse, err, ws = run_fused(c)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                           o_ref, l_ref, what=str(case))
    # the same result as partial + combine, up to the order of the merge
    out2, lse2, _, _, err2 = run_gpu(c)
    assert err2 == 0
    d = (out.float() - out2.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * max(1.0, float(out2.float().abs().max()))
    fin = torch.isfinite(lse2)
    assert torch.equal(fin, torch.isfinite(lse))
    if bool(fin.any()):
        assert float((lse[fin] - lse2[fin]).abs().max()) <= 1e-4
    # the two counters are back at zero
    assert torch.count_nonzero(ws[:8]).item() == 0


def test_fused_is_bitwise_deterministic_and_reuses_its_workspace():
    c = make_case("b16_128k_fp8", seq_lens=[5000, 3000], splits=3)
    a = run_fused(c)
    b = run_fused(c, workspace=a[3])
    assert a[2] == 0 and b[2] == 0
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1], b[1])


def test_fused_refuses_grids_that_do_not_fit():
    import mla_split_kv_absorbed_b200 as m
    # batch 16 x 32 splits = 512 units: more than one wave
    c = make_case("b16_128k_fp8", seq_lens=[300] * 16, splits=32)
    with pytest.raises(m.MlaError) as e:
        run_fused(c)
    assert e.value.status == m.MLA_ERR_UNSUPPORTED


def test_fused_full_size_batch1_sampled_rows():
    # the batch-1 benchmark workload (64 splits, 2 pieces each: 128 CTAs)
    c = make_case("b1_128k_fp8", gen_device="cuda")
    w = c.w
    out, lse, err, ws = run_fused(c)
    assert err == 0
    R = w.B * w.q_len * w.H
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, R - 1], rng.choice(R, size=24, replace=False)]))
    o_ref, l_ref = oracle_rows(c, rows)
    o = out.float().cpu().numpy().reshape(R, 512)[rows]
    l = lse.cpu().numpy().reshape(R)[rows]
    assert_attention_close(o, l, o_ref, l_ref, what="b1 fused")
    assert torch.count_nonzero(ws[:8]).item() == 0
