"""Sequence-sharded decode on CPU: the shard plan, the exchange and the merge.

Each of 2 or 3 gloo ranks decodes its page range of every request with the
oracle (the stand-in for the GPU kernels, which need no peer), all-gathers its
per-row partial (O, LSE), and merges the ranks' partials with the oracle's
log-sum-exp merge.  The result must equal the oracle's unsharded decode: this
checks the page-aligned plan (the new tokens all on the last rank), the
q_len-as-rows view of the earlier ranks, empty ranges, and the all-gather
layout ([rank][row]) that mla_merge_rank_partials reads.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    # name: (spec, overrides)
    "q1_ragged": ("b16_128k_fp8", dict(seq_lens=[5000, 130, 64, 777], splits=3, H=16)),
    "q4_causal": ("verify_q4_256k_fp8", dict(seq_lens=[1000, 70, 4], splits=2, H=16)),
    "bf16": ("tiny", dict(seq_lens=[300, 2049], splits=2, H=16)),
}


def _local_rank_partial(w, kv_host, shard, oracle):
    from mla_split_kv_absorbed_b200 import workloads as wl
    B, Q, H = w.B, w.q_len, w.H
    qn, qr = wl.bf16_bits(w.q_nope), wl.bf16_bits(w.q_rope)
    o = np.zeros((B, Q, H, 512))
    lse = np.full((B, Q, H), -np.inf)
    for b in range(B):
        L = int(shard.seq_lens[b])
        if L == 0:
            continue
        if shard.causal:
            qv, rv, ql, hv = qn[b:b + 1], qr[b:b + 1], Q, H
        else:  # every row sees every local token: rows as one query position
            qv, rv, ql, hv = qn[b:b + 1].reshape(1, 1, Q * H, 512), qr[b:b + 1].reshape(1, 1, Q * H, 64), 1, Q * H
        ob, lb = oracle.decode_rows(qv, rv, kv_host, w.kv_scale, shard.block_table[b:b + 1].numpy(),
                                    np.array([L], np.int32), ql, hv, w.softmax_scale,
                                    np.arange(Q * H))
        o[b] = ob.reshape(Q, H, 512)
        lse[b] = lb.reshape(Q, H)
    return o, lse


def _rank_main(rank, ws, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from mla_split_kv_absorbed_b200 import sharded, workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    spec, ov = CASES[case]
    w = wl.make(spec, **ov)
    kv_host = (oracle.quantize(wl.bf16_bits(w.kv_pool), w.inv_scale) if w.spec.kv_dtype == "fp8"
               else wl.bf16_bits(w.kv_pool))
    shards = sharded.shard_plan(w.block_table, w.seq_lens, w.q_len, ws)
    o, lse = _local_rank_partial(w, kv_host, shards[rank], oracle)
    go, gl = sharded.exchange(torch.from_numpy(o), torch.from_numpy(lse))
    # merge over the ranks: rank partials laid out [rank][row] -> [row][rank]
    R = w.B * w.q_len * w.H
    po = go.reshape(ws, R, 512).permute(1, 0, 2).contiguous().numpy()
    pl = gl.reshape(ws, R).permute(1, 0).contiguous().numpy()
    mo, ml = oracle.combine(po, pl, np.full(R, ws, np.int32))
    ro, rl = oracle.decode_rows(wl.bf16_bits(w.q_nope), wl.bf16_bits(w.q_rope), kv_host, w.kv_scale,
                                w.block_table.numpy(), w.seq_lens.numpy(), w.q_len, w.H,
                                w.softmax_scale, np.arange(R))
    out.put((rank, float(np.abs(mo - ro).max()), float(np.abs(ml - rl).max())))
    dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 3])
@pytest.mark.parametrize("case", sorted(CASES))
def test_sharded_merge_equals_unsharded_decode(ws, case):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, case, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, d_o, d_l in res:
        # the partials cross the exchange as fp64 and enter the merge as fp32
        assert d_o < 1e-5 and d_l < 1e-5, (rank, d_o, d_l)


def test_shard_plan_properties():
    sys.path.insert(0, ROOT)
    from mla_split_kv_absorbed_b200 import sharded
    rng = np.random.default_rng(3)
    for _ in range(200):
        L = int(rng.integers(1, 20000))
        q_len = int(rng.integers(1, min(4, L) + 1))
        n = int(rng.integers(1, 9))
        b = sharded.shard_bounds(L, q_len, n)
        pages = -(-L // 64)
        assert b[0] == 0 and b[-1] == pages and all(x <= y for x, y in zip(b, b[1:]))
        # every new token (positions L-q_len .. L-1) is on the last rank
        assert b[n - 1] * 64 <= L - q_len
    bt = torch.arange(3 * 40, dtype=torch.int32).reshape(3, 40)
    lens = [2500, 64, 1]
    shards = sharded.shard_plan(bt, lens, 1, 4)
    # the ranks' tokens tile each request exactly once, in order
    for b, L in enumerate(lens):
        got = []
        for s in shards:
            n = int(s.seq_lens[b])
            pages = -(-n // 64)
            for t in range(n):
                got.append((int(s.block_table[b, t // 64]), t % 64))
            assert int(s.starts[b]) % 64 == 0
        assert got == [(int(bt[b, t // 64]), t % 64) for t in range(L)]
    assert shards[-1].causal and not any(s.causal for s in shards[:-1])
