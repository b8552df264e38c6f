"""Sequence-sharded decode with the library's kernels, ranks emulated on one GPU.

Every rank's work (mla_decode_partial over its page range, mla_combine_f32 of
its splits) runs in turn on one GPU; the per-rank partials are stacked in rank
order, as the all-gather lays them out, and mla_merge_rank_partials merges
them.  The result is compared with the oracle's unsharded decode.  No rank
waits on another here: the exchange itself is covered by the gloo test.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_attention_close, make_case, oracle_rows

pytestmark = pytest.mark.gpu

CASES = [
    ("b16_128k_fp8", dict(seq_lens=[5000, 130, 64, 777], splits=3)),
    ("verify_q4_256k_fp8", dict(seq_lens=[3000, 70, 4], splits=4)),      # q_len 4, causal last rank
    ("tiny", dict(seq_lens=[300, 2049], splits=2, H=64)),                 # bf16 cache
    ("b1_128k_fp8", dict(seq_lens=[131072], splits=16)),                  # 128K over the ranks
]


@pytest.mark.parametrize("n_ranks", [2, 3])
@pytest.mark.parametrize("spec,ov", CASES)
def test_sharded_decode_matches_oracle(spec, ov, n_ranks):
    import mla_split_kv_absorbed_b200 as m
    from mla_split_kv_absorbed_b200 import sharded
    c = make_case(spec, **ov)
    w = c.w
    shards = sharded.shard_plan(w.block_table, w.seq_lens, w.q_len, n_ranks)
    parts = [sharded.local_partial(c.dev["q_nope"], c.dev["q_rope"], c.kv_dev, w.kv_scale, sh,
                                   w.num_splits, w.max_splits, w.softmax_scale) for sh in shards]
    go = torch.stack([p[0] for p in parts])
    gl = torch.stack([p[1] for p in parts])
    out = torch.empty((w.B, w.q_len, w.H, 512), dtype=torch.bfloat16, device="cuda")
    out_lse = torch.empty((w.B, w.q_len, w.H), dtype=torch.float32, device="cuda")
    m.mla_merge_rank_partials(go, gl, out, out_lse)
    torch.cuda.synchronize()
    R = w.B * w.q_len * w.H
    rows = np.arange(R) if R <= 512 else np.unique(np.r_[0, R - 1, np.arange(0, R, 7)])
    o_ref, l_ref = oracle_rows(c, rows)
    assert_attention_close(out.float().cpu().numpy().reshape(R, 512)[rows],
                           out_lse.cpu().numpy().reshape(R)[rows], o_ref, l_ref,
                           what=f"{spec} x{n_ranks}")
