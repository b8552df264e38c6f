"""KV append on the GPU (mla_append_kv_fp8) against the oracle, byte for byte.

The step before the decode path: RoPE on the 64-wide key, the saturating E4M3
conversion and the write into the paged cache through the block table, in one
kernel ("Muse Spark Open" article, section "内核优化：解码吞吐 3 倍", bullet
"RoPE 与 KV 缓存写入融合"; "SGLang & Miles ... Vera Rubin" article, bullet
"原生 FP8 转换").  Every byte of the pool is compared, so rows that must not be
touched are checked too.  The (cos, sin) table comes from the library's own
host builder for the GPU and from the oracle's for the oracle; the two are
checked equal on the CPU.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _case(seed, B, n_new, lens, std=2.0, spare=3, extreme=False):
    # Block-table entries below the first new token's page all point at one
    # shared spare page (the append never reaches them), so the pool stays
    # small at 128K-256K contexts; the pages the new tokens land in are a
    # seeded permutation, and the pool starts as random bytes.
    g = torch.Generator().manual_seed(seed)
    first = [max(0, (L - n_new) // 64) for L in lens]
    last = [(L + 63) // 64 for L in lens]
    fresh = sum(l - f for f, l in zip(first, last))
    num_pages = fresh + spare
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    shared = int(perm[-1])
    bt = torch.full((B, max(last)), shared, dtype=torch.int32)
    off = 0
    for b in range(B):
        n = last[b] - first[b]
        bt[b, first[b]:last[b]] = perm[off:off + n]
        off += n
    c = (std * torch.randn((B, n_new, 512), generator=g)).to(torch.bfloat16)
    r = (std * torch.randn((B, n_new, 64), generator=g)).to(torch.bfloat16)
    if extreme:
        flat = c.view(-1)
        flat[::97] = 1e30      # saturates to +448
        flat[1::97] = -float("inf")
        flat[2::97] = 0.0
        r.view(-1)[::13] = 3e4
    pool = torch.randint(0, 256, (num_pages, 64, 576), generator=g, dtype=torch.uint8)
    return c, r, bt, torch.tensor(lens, dtype=torch.int32), pool


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _run_both(c, r, bt, sl, pool, inv_scale, max_pos, bt_dev=None):
    import mla_split_kv_absorbed_b200 as m
    n_new = c.shape[1]
    table = m.mla_rope_cos_sin_table(max_pos)
    kv = pool.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mla_append_kv_fp8(c.cuda(), r.cuda(), table.cuda(), (bt if bt_dev is None else bt_dev).cuda(),
                        sl.cuda(), inv_scale, kv, dev_error=err)
    torch.cuda.synchronize()
    ref = pool.numpy().copy()
    skipped = oracle.append_kv(_bits(c), _bits(r), oracle.rope_table(max_pos),
                               (bt if bt_dev is None else bt_dev).numpy(), sl.numpy(), n_new,
                               inv_scale, ref)
    return kv.cpu().numpy(), ref, int(err.item()), skipped


@pytest.mark.parametrize("B,n_new,lens", [
    (1, 1, [1]),                       # the first token of a request
    (3, 2, [5, 64, 130]),              # page boundary and a new page
    (16, 1, [131072] * 16),            # decode step at 128K
    (8, 4, [262144] * 8),              # speculative verify: four new tokens at 256K
    (2, 300, [300, 1000]),             # a prompt-sized append
])
def test_append_matches_oracle_bytewise(B, n_new, lens):
    c, r, bt, sl, pool = _case(B * 7 + n_new, B, n_new, lens)
    inv = float(np.float32(448.0) / np.float32(8.0))
    got, ref, err, skipped = _run_both(c, r, bt, sl, pool, inv, max(lens))
    assert err == 0 and skipped == 0
    assert np.array_equal(got, ref), f"{int((got != ref).sum())} bytes differ"


def test_append_saturates_and_never_writes_nan():
    c, r, bt, sl, pool = _case(5, 2, 8, [100, 200], extreme=True)
    got, ref, err, _ = _run_both(c, r, bt, sl, pool, 1.0, 256)
    assert err == 0
    assert np.array_equal(got, ref)
    for b in range(2):
        for j in range(8):
            pos = int(sl[b]) - 8 + j
            row = got[bt[b, pos // 64], pos % 64]
            assert not np.any((row & 0x7F) == 0x7F), "NaN code written for a finite or infinite input"


def test_append_reports_bad_positions_and_pages_and_writes_the_rest():
    import mla_split_kv_absorbed_b200 as m
    c, r, bt, sl, pool = _case(9, 3, 2, [5, 64, 130])
    bt_bad = bt.clone()
    bt_bad[1, 0] = 10 ** 6             # request 1's page id is outside the pool
    # request 2 reaches position 129, beyond a 100-entry table
    got, ref, err, skipped = _run_both(c, r, bt, sl, pool, 1.0, 100, bt_dev=bt_bad)
    assert err & m.DEVERR_BAD_PAGE and err & m.DEVERR_BAD_SEQLEN
    assert skipped == 4
    assert np.array_equal(got, ref)
