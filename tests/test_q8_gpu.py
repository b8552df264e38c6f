"""FP8 query (mla_decode_partial_q8) on the GPU against the oracle.

The query is quantised with the oracle's E4M3 encoder (the GPU quantiser is
bit-exact with it, tests/test_quantize_gpu.py) and both sides use the same
codes: the oracle decodes code * q_scale in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import bf16_half_ulp, make_case

pytestmark = pytest.mark.gpu

Q_SCALE = 1.0 / 64.0


def q8_of(c):
    w = c.w
    qbits = np.concatenate([c.qn_bits, c.qr_bits], axis=-1)
    return oracle.quantize(qbits, float(np.float32(1.0) / np.float32(Q_SCALE)))


def run_q8(c, q8):
    import mla_split_kv_absorbed_b200 as m
    w = c.w
    part_o, part_lse = m.alloc_partials(w.B, w.q_len, w.H, w.max_splits)
    part_o.fill_(float("nan"))
    part_lse.fill_(float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mla_decode_partial_q8(torch.from_numpy(q8).cuda(), Q_SCALE, c.kv_dev, w.kv_scale,
                            c.dev["block_table"], c.dev["seq_lens"], c.dev["num_splits"],
                            w.max_splits, w.softmax_scale, part_o, part_lse, err)
    out = torch.empty((w.B, w.q_len, w.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.q_len, w.H), dtype=torch.float32, device="cuda")
    m.mla_combine(part_o, part_lse, c.dev["num_splits"], w.max_splits, out, lse)
    torch.cuda.synchronize()
    return part_o, part_lse, out, lse, int(err.item())


CASES = [
    ("b1_128k_fp8", dict(seq_lens=[700], splits=3)),
    ("b1_128k_fp8", dict(seq_lens=[100], splits=8)),
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 1, 777], splits=4)),
    ("verify_q4_256k_fp8", dict(seq_lens=[1000, 4], splits=2)),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{s}-{len(o['seq_lens'])}" for s, o in CASES])
def test_q8_partials_and_output_match_oracle(case):
    spec, ov = case
    c = make_case(spec, **ov)
    w = c.w
    q8 = q8_of(c)
    po, pl, out, lse, err = run_q8(c, q8)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H, dtype=np.int64)
    args = (c.kv_host, w.kv_scale, w.block_table.cpu().numpy(), w.seq_lens.cpu().numpy())
    po_ref, pl_ref = oracle.partials_rows_q8(q8, Q_SCALE, *args, w.num_splits.cpu().numpy(),
                                             w.max_splits, w.q_len, w.H, w.softmax_scale, rows)
    po = po.cpu().numpy().reshape(len(rows), w.max_splits, 512)
    pl = pl.cpu().numpy().reshape(len(rows), w.max_splits)
    ns = w.num_splits.cpu().numpy()[rows // (w.q_len * w.H)]
    for r in range(len(rows)):
        S = ns[r]
        assert np.array_equal(np.isneginf(pl[r, :S]), np.isneginf(pl_ref[r, :S])), r
        fin = np.isfinite(pl_ref[r, :S])
        assert np.all(np.abs(pl[r, :S][fin] - pl_ref[r, :S][fin]) <= 1e-3 * np.maximum(1, np.abs(pl_ref[r, :S][fin])))
        scale = np.maximum(1.0, np.abs(po_ref[r, :S]).max(axis=1, keepdims=True))
        assert np.all(np.abs(po[r, :S] - po_ref[r, :S]) <= 1e-2 * scale), r
    # the merged output against the unsplit oracle decode (one split)
    o1, l1 = oracle.partials_rows_q8(q8, Q_SCALE, *args, np.ones(w.B, np.int32), 1, w.q_len, w.H,
                                     w.softmax_scale, rows)
    o = out.float().cpu().numpy().reshape(-1, 512)
    err_o = np.maximum(np.abs(o - o1[:, 0]) - bf16_half_ulp(o1[:, 0]), 0.0)
    assert float(err_o.max()) <= 1e-2
    rel = np.linalg.norm(o - o1[:, 0]) / max(np.linalg.norm(o1[:, 0]), 1e-30)
    assert rel <= 5e-3
    fin = np.isfinite(l1[:, 0])
    assert np.all(np.abs(lse.cpu().numpy().reshape(-1)[fin] - l1[fin, 0]) <= 1e-3 * np.maximum(1, np.abs(l1[fin, 0])))
