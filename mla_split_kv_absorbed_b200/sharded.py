"""Sequence-sharded decode over several GPUs (one process per GPU).

"SGLang & Miles ... Vera Rubin" article, section "Kimi K3 的 MLA", bullet
"更快的 split-KV 归约": a request's KV is cut into pieces whose partial results
(normalised O and its log-sum-exp) are merged afterwards.  Across GPUs the same
merge runs one level up: every rank holds a disjoint, page-aligned range of
each request's KV pages, computes its partials with the library's kernels,
folds them into one fp32 partial per query row, and one all-gather of those
partials (rows * 513 fp32 per rank) lets every rank merge them.

Sharding rule (host logic, no GPU needed; :func:`shard_plan`):

* a request's ``n = ceil(L / 64)`` pages are cut into ``n_ranks`` contiguous,
  page-aligned ranges, as equal as they can be, except that the last range
  always starts at or before the page of the first new token, so every one of
  the ``q_len`` new tokens lives on the last rank;
* on ranks before the last, every query row sees every token of the range, so
  those ranks decode the ``q_len * H`` rows as ``q_len = 1`` rows (the same
  memory, viewed ``[B][1][q_len * H]``), with no causal mask;
* the last rank decodes its range with the request's own ``q_len``: with local
  length ``L - start``, its causal rule (row q sees tokens up to
  ``local_len - q_len + q``) is the global one shifted by ``start``;
* a rank whose range is empty for a request contributes O = 0, LSE = -inf.

Nothing here reads a peer's memory directly: the exchange is one NCCL (or, in
the CPU tests, gloo) all-gather into this rank's own buffer.
"""
from __future__ import annotations

import dataclasses

import torch

PAGE = 64


@dataclasses.dataclass
class RankShard:
    """One rank's part of a batch: a local block table and local lengths."""
    rank: int
    n_ranks: int
    block_table: torch.Tensor   # int32 [B][max_local_pages] (entries past a request's range: 0)
    seq_lens: torch.Tensor      # int32 [B], tokens of each request on this rank (0 = none)
    starts: torch.Tensor        # int32 [B], global position of the rank's first token
    causal: bool                # True on the last rank (it holds the q_len new tokens)


def shard_bounds(L: int, q_len: int, n_ranks: int):
    """Page boundaries p_0 = 0 <= p_1 <= ... <= p_N = ceil(L/64) of one request."""
    n = -(-L // PAGE)
    last_start_max = (L - q_len) // PAGE  # page holding the first new token
    bounds = [(r * n) // n_ranks for r in range(n_ranks)] + [n]
    if bounds[n_ranks - 1] > last_start_max:
        # move the last range's start back so the new tokens all land on it
        bounds[n_ranks - 1] = last_start_max
        for r in range(n_ranks - 2, 0, -1):
            bounds[r] = min(bounds[r], bounds[r + 1])
    return bounds


def shard_plan(block_table: torch.Tensor, seq_lens, q_len: int, n_ranks: int):
    """Per-rank local block tables and lengths (CPU tensors) for a batch."""
    bt = block_table.cpu()
    lens = [int(v) for v in torch.as_tensor(seq_lens).cpu().tolist()]
    B = len(lens)
    out = []
    all_bounds = [shard_bounds(L, q_len, n_ranks) for L in lens]
    for r in range(n_ranks):
        local_pages = [all_bounds[b][r + 1] - all_bounds[b][r] for b in range(B)]
        width = max(1, max(local_pages))
        lbt = torch.zeros((B, width), dtype=torch.int32)
        lsl = torch.zeros(B, dtype=torch.int32)
        st = torch.zeros(B, dtype=torch.int32)
        for b in range(B):
            p0, p1 = all_bounds[b][r], all_bounds[b][r + 1]
            if p1 > p0:
                lbt[b, :p1 - p0] = bt[b, p0:p1]
                lsl[b] = min(lens[b], p1 * PAGE) - p0 * PAGE
            st[b] = p0 * PAGE
        out.append(RankShard(rank=r, n_ranks=n_ranks, block_table=lbt, seq_lens=lsl, starts=st,
                             causal=(r == n_ranks - 1)))
    return out


def local_partial(q_nope, q_rope, kv_pages, kv_scale, shard: RankShard, num_splits, max_splits,
                  softmax_scale, stream=None):
    """This rank's fp32 partial per query row, (O [B][q_len][H][512], LSE [B][q_len][H]),
    from the library's partial kernel and its fp32 merge of the splits."""
    import mla_split_kv_absorbed_b200 as m
    B, q_len, H, _ = q_nope.shape
    dev = q_nope.device
    o = torch.zeros((B, q_len, H, 512), dtype=torch.float32, device=dev)
    lse = torch.full((B, q_len, H), float("-inf"), dtype=torch.float32, device=dev)
    has = shard.seq_lens > 0
    if not bool(has.any()):
        return o, lse
    # requests with no tokens on this rank are left at (0, -inf): decode the others
    idx = torch.nonzero(has).flatten()
    sel = idx.to(dev)
    qn, qr = q_nope.index_select(0, sel), q_rope.index_select(0, sel)
    Bs = int(idx.numel())
    if shard.causal:
        qv, rv, ql, Hv = qn.contiguous(), qr.contiguous(), q_len, H
    else:  # every row sees every local token: the rows as one query position
        qv, rv, ql, Hv = qn.reshape(Bs, 1, q_len * H, 512), qr.reshape(Bs, 1, q_len * H, 64), 1, q_len * H
    bt = shard.block_table.index_select(0, idx).to(dev)
    sl = shard.seq_lens.index_select(0, idx).to(dev)
    ns = torch.as_tensor(num_splits, dtype=torch.int32).cpu().index_select(0, idx).to(dev)
    part_o, part_lse = m.alloc_partials(Bs, ql, Hv, max_splits, dev)
    m.mla_decode_partial(qv, rv, kv_pages, kv_scale, bt, sl, ns, max_splits, softmax_scale, part_o,
                         part_lse, stream=stream)
    po = torch.empty((Bs, ql, Hv, 512), dtype=torch.float32, device=dev)
    pl = torch.empty((Bs, ql, Hv), dtype=torch.float32, device=dev)
    m.mla_combine_f32(part_o, part_lse, ns, max_splits, po, pl, stream=stream)
    o.index_copy_(0, sel, po.reshape(Bs, q_len, H, 512))
    lse.index_copy_(0, sel, pl.reshape(Bs, q_len, H))
    return o, lse


def exchange(o, lse, group=None):
    """All-gather of every rank's (O, LSE): ([N][B][q_len][H][512], [N][B][q_len][H]).
    The gather fills this rank's own buffers (rank-major concatenation)."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    go = torch.empty((n * o.shape[0],) + tuple(o.shape[1:]), dtype=o.dtype, device=o.device)
    gl = torch.empty((n * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype, device=lse.device)
    dist.all_gather_into_tensor(go, o.contiguous(), group=group)
    dist.all_gather_into_tensor(gl, lse.contiguous(), group=group)
    return go.view((n,) + tuple(o.shape)), gl.view((n,) + tuple(lse.shape))


def sharded_decode(q_nope, q_rope, kv_pages, kv_scale, shard: RankShard, num_splits, max_splits,
                   softmax_scale, group=None, stream=None):
    """Decode one batch whose KV is sharded by sequence over the ranks of
    `group`: this rank's partial, the all-gather, and the library's merge.
    Every rank returns the full (out bf16 [B][q_len][H][512], out_lse)."""
    import mla_split_kv_absorbed_b200 as m
    o, lse = local_partial(q_nope, q_rope, kv_pages, kv_scale, shard, num_splits, max_splits,
                           softmax_scale, stream)
    go, gl = exchange(o, lse, group)
    out = torch.empty(q_nope.shape, dtype=torch.bfloat16, device=q_nope.device)
    out_lse = torch.empty(lse.shape, dtype=torch.float32, device=q_nope.device)
    m.mla_merge_rank_partials(go, gl, out, out_lse, stream=stream)
    return out, out_lse
