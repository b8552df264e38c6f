"""Single-launch decode (mla_decode_fused) on the GPU against the oracle.

The fused path runs steps A2-A9 in one cooperative launch.  It cuts every
request into S = floor(SMs / (row groups x B)) equal page ranges (at most 256),
so the grid is one wave of one CTA per (row group, split, request): every CTA
writes its split's partial, the grid meets at a barrier and merges them.
Shapes with more (row group, request) pairs than SMs are refused with
MLA_ERR_UNSUPPORTED.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_attention_close, make_case, oracle_rows

pytestmark = pytest.mark.gpu

SMALL = [
    ("b1_128k_fp8", dict(seq_lens=[2085])),                 # 148 splits over 33 pages: most empty
    ("b1_128k_fp8", dict(seq_lens=[100])),                  # one page with a ragged tail
    ("b1_128k_fp8", dict(seq_lens=[64 * 148 * 2 + 5])),     # 2 pages per split, ragged last split
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 1, 777])),    # 37 splits each
    ("verify_q4_256k_fp8", dict(seq_lens=[777], H=16)),     # q_len 4, causal, one row group
    ("verify_q4_256k_fp8", dict(seq_lens=[1000, 4])),       # four row groups, 18 splits
    ("b16_128k_fp8", dict(seq_lens=[300] * 148)),           # one split per request
    ("b16_128k_fp8", dict(seq_lens=[1024], H=16)),          # 16 rows in a 64-row group
    ("b16_128k_fp8", dict(seq_lens=[3000], H=128)),         # two row groups, 74 splits
    ("b16_128k_fp8", dict(seq_lens=[1500, 900], H=32, q_len=2)),  # causal, 2 positions per group
    ("b16_128k_fp8", dict(seq_lens=[700, 5, 2200], H=16, q_len=3)),  # 48 rows, q_len 3
    ("b16_128k_fp8", dict(seq_lens=[130, 64, 1, 2000] * 25)),  # 100 requests, 1 split each
]


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def run_fused(c, workspace=None):
    import mla_split_kv_absorbed_b200 as m
    w = c.w
    if workspace is None:
        workspace = m.alloc_fused_workspace(w.B, w.q_len, w.H)
    out = torch.full((w.B, w.q_len, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.q_len, w.H), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mla_decode_fused(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale, c.dev["block_table"],
                       c.dev["seq_lens"], w.softmax_scale, workspace, out, lse, err)
    torch.cuda.synchronize()
    return out, lse, int(err.item()), workspace


def run_two_launch(c, S):
    """partial + combine with the fused call's split count S for every request."""
    import mla_split_kv_absorbed_b200 as m
    w = c.w
    ns = torch.full((w.B,), S, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = m.decode(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale,
                        c.dev["block_table"], c.dev["seq_lens"], ns, S, w.softmax_scale,
                        dev_error=err)
    torch.cuda.synchronize()
    return out, lse, int(err.item())


def _ids(c):
    spec, ov = c
    return spec + "-" + "-".join(f"{k}{v if not isinstance(v, list) else len(v)}" for k, v in ov.items())


@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_fused_small_matches_oracle_and_two_launch_path(case):
    import mla_split_kv_absorbed_b200 as m
    spec, ov = case
    c = make_case(spec, **ov)
    w = c.w
    S = m.mla_fused_splits(w.B, w.q_len, w.H, sms())
    assert S >= 1
    out, lse, err, ws = run_fused(c)
    assert err == 0
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                           o_ref, l_ref, what=str(case))
    # the same result as partial + combine with S splits, up to the order of the merge
    out2, lse2, err2 = run_two_launch(c, S)
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
    c = make_case("b16_128k_fp8", seq_lens=[5000, 3000])
    a = run_fused(c)
    b = run_fused(c, workspace=a[3])
    assert a[2] == 0 and b[2] == 0
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1], b[1])


def test_fused_refuses_shapes_without_a_single_wave_and_small_workspaces():
    import mla_split_kv_absorbed_b200 as m
    n = sms()
    # one more request than SMs: not even one split per request fits in a wave
    c = make_case("b16_128k_fp8", seq_lens=[70] * (n + 1))
    assert m.mla_fused_splits(c.w.B, 1, c.w.H, n) == 0
    with pytest.raises(m.MlaError) as e:
        run_fused(c, workspace=torch.zeros(4096, dtype=torch.uint8, device="cuda"))
    assert e.value.status == m.MLA_ERR_UNSUPPORTED
    with pytest.raises(m.MlaError) as e:
        m.alloc_fused_workspace(c.w.B, 1, c.w.H)
    assert e.value.status == m.MLA_ERR_UNSUPPORTED
    # a workspace one byte short of what the call needs
    c = make_case("b16_128k_fp8", seq_lens=[300, 200])
    need = m.mla_fused_workspace_bytes(2, 1, c.w.H, n)
    with pytest.raises(m.MlaError) as e:
        run_fused(c, workspace=torch.zeros(need - 1, dtype=torch.uint8, device="cuda"))
    assert e.value.status == m.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("spec", ["b1_128k_fp8", "b16_128k_fp8", "verify_q4_256k_fp8"])
def test_fused_full_size_sampled_rows(spec):
    # the benchmark workloads at full size, in the launch the benchmark times
    # (batch 1: 148 splits; batch 16: 9 splits, 144 CTAs; the q_len-4 verify at
    # batch 8: 4 row groups x 4 splits x 8 requests, 128 CTAs); one sampled
    # row of every (request, query position), both ends, and random extras
    c = make_case(spec, gen_device="cuda")
    w = c.w
    out, lse, err, ws = run_fused(c)
    assert err == 0
    R = w.B * w.q_len * w.H
    rng = np.random.default_rng(7)
    per = [(b * w.q_len + q) * w.H + int(rng.integers(w.H)) for b in range(w.B) for q in range(w.q_len)]
    rows = np.unique(np.concatenate([[0, R - 1], per, rng.choice(R, size=8, replace=False)]))
    o_ref, l_ref = oracle_rows(c, rows)
    o = out.float().cpu().numpy().reshape(R, 512)[rows]
    l = lse.cpu().numpy().reshape(R)[rows]
    assert_attention_close(o, l, o_ref, l_ref, what=spec + " fused")
    assert torch.count_nonzero(ws[:8]).item() == 0


@pytest.mark.parametrize("spec,ov", [
    ("b1_128k_fp8", dict(seq_lens=[64 * 148 * 2 + 5])),   # 148 entries per row
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 1, 777])),  # 37 entries per row, empty rows' splits
])
def test_every_merge_plan_matches_the_oracle(spec, ov):
    # the merge inside the single launch picks its plan from the shape; force
    # each of the twelve (dims per thread, groups per item) plans in turn
    import mla_split_kv_absorbed_b200 as m
    c = make_case(spec, **ov)
    w = c.w
    rows = np.arange(w.B * w.q_len * w.H)
    o_ref, l_ref = oracle_rows(c, rows)
    ws = m.alloc_fused_workspace(w.B, w.q_len, w.H)
    try:
        for v in (1, 2, 4):
            for gpi in (1, 2, 3, 6):
                m.mla_debug_merge_plan(v, gpi)
                out, lse, err, _ = run_fused(c, workspace=ws)
                assert err == 0
                assert_attention_close(out.float().cpu().numpy().reshape(-1, 512),
                                       lse.cpu().numpy().reshape(-1), o_ref, l_ref,
                                       what=f"{spec} plan v={v} gpi={gpi}")
                assert torch.count_nonzero(ws[:8]).item() == 0
    finally:
        m.mla_debug_merge_plan(0, 0)


def test_host_staging_round_trip_matches_device_inputs():
    # one packed host-to-device copy of the inputs, one device-to-host copy of
    # the outputs: the same bits as the call on device-resident inputs
    import mla_split_kv_absorbed_b200 as m
    c = make_case("b16_128k_fp8", seq_lens=[3000, 700, 64])
    w = c.w
    st = m.HostStaging(w.B, w.q_len, w.H, w.block_table.shape[1])
    for name in st.host:
        st.host[name].copy_(getattr(w, name).cpu())
    ws = m.alloc_fused_workspace(w.B, w.q_len, w.H)
    st.upload()
    d = st.dev
    m.mla_decode_fused(d["q_nope"], d["q_rope"], c.kv_dev, w.kv_scale, d["block_table"],
                       d["seq_lens"], w.softmax_scale, ws, st.out, st.out_lse)
    st.download()
    torch.cuda.synchronize()
    out, lse, err, _ = run_fused(c)
    assert err == 0
    assert torch.equal(st.host_out.view(torch.int16), out.cpu().view(torch.int16))
    assert torch.equal(st.host_lse, lse.cpu())
    assert st.in_bytes >= (w.q_nope.numel() + w.q_rope.numel()) * 2 + w.block_table.numel() * 4


def test_decode_graph_replays_the_host_buffer_step():
    # the captured step (upload, single launch, download) gives the same bits
    # as the call on device-resident inputs, and follows new host inputs
    import mla_split_kv_absorbed_b200 as m
    c = make_case("b16_128k_fp8", seq_lens=[3000, 700, 64])
    w = c.w
    st = m.HostStaging(w.B, w.q_len, w.H, w.block_table.shape[1])
    for name in st.host:
        st.host[name].copy_(getattr(w, name).cpu())
    g = m.DecodeGraph(st, c.kv_dev, w.kv_scale, w.softmax_scale)
    st.host_out.zero_()
    g.replay()
    torch.cuda.synchronize()
    out, lse, err, _ = run_fused(c)
    assert err == 0
    assert torch.equal(st.host_out.view(torch.int16), out.cpu().view(torch.int16))
    assert torch.equal(st.host_lse, lse.cpu())
    # new queries in the same host buffer: the next replay uses them
    st.host["q_nope"].mul_(-1)
    st.host["q_rope"].mul_(-1)
    g.replay()
    torch.cuda.synchronize()
    c.dev["q_nope"].mul_(-1)
    c.dev["q_rope"].mul_(-1)
    out2, lse2, err2, _ = run_fused(c)
    assert err2 == 0
    assert torch.equal(st.host_out.view(torch.int16), out2.cpu().view(torch.int16))
    assert not torch.equal(out2.view(torch.int16), out.view(torch.int16))
