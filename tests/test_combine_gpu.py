"""Step A9 on the GPU: mla_combine against the oracle's LSE merge."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _run(po, pl, ns_b, B, q_len, H, S):
    import mla_split_kv_absorbed_b200 as m
    out = torch.empty((B, q_len, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, q_len, H), dtype=torch.float32, device="cuda")
    m.mla_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(),
                  torch.from_numpy(ns_b).cuda(), S, out, lse)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1)


@pytest.mark.parametrize("B,q_len,H,S", [(1, 1, 16, 1), (1, 1, 64, 4), (2, 1, 64, 32), (1, 1, 64, 64),
                                         (3, 4, 16, 65), (1, 1, 128, 128), (2, 2, 16, 256)])
def test_combine_matches_oracle(B, q_len, H, S):
    rng = np.random.default_rng(B * 1000 + S)
    R = B * q_len * H
    po = rng.standard_normal((R, S, 512)).astype(np.float32)
    pl = (rng.standard_normal((R, S)) * 3 + 2).astype(np.float32)
    ns_b = rng.integers(1, S + 1, size=B).astype(np.int32)
    ns_b[0] = S
    # some empty splits inside the range
    pl[rng.random((R, S)) < 0.1] = -np.inf
    if R > 2:
        pl[1, :] = -np.inf  # a row whose splits are all empty
    got_o, got_l = _run(po.reshape(B, q_len, H, S, 512), pl.reshape(B, q_len, H, S), ns_b, B, q_len, H, S)
    n_row = np.repeat(ns_b, q_len * H)
    ref_o, ref_l = oracle.combine(po, pl, n_row)
    # bf16 rounding of an fp32 result: |err| <= 2^-8 |ref| + tiny
    err = np.abs(got_o - ref_o)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref_o) + 1e-6), float(err.max())
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(ref_l))
    np.testing.assert_allclose(got_l[fin], ref_l[fin], rtol=2e-6, atol=2e-6)
    if R > 2:
        assert np.all(got_o[1] == 0)


def test_combine_is_deterministic():
    rng = np.random.default_rng(5)
    B, q_len, H, S = 1, 1, 64, 64
    po = rng.standard_normal((B, q_len, H, S, 512)).astype(np.float32)
    pl = rng.standard_normal((B, q_len, H, S)).astype(np.float32)
    ns = np.array([S], dtype=np.int32)
    a = _run(po, pl, ns, B, q_len, H, S)
    b = _run(po, pl, ns, B, q_len, H, S)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
