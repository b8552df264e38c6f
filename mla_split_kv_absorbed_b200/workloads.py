"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

Each workload fixes batch, q_len, heads, per-request KV lengths, KV storage
dtype, value distributions, page layout and split counts.  The generator
returns plain tensors: bf16 queries, the bf16 *pre-quantisation* KV values of
the whole page pool, the block table, sequence lengths and split counts.  For
an FP8 cache the caller converts the pool to E4M3 codes itself, with the
returned ``kv_scale`` (the tests use the CPU oracle's quantiser, the benchmark
uses the library's ``mla_quantize_fp8``), so this module holds no rounding or
attention arithmetic.

Layout (token t of request b lives in page ``block_table[b][t // 64]``, slot
``t % 64``)::

    q_nope   [B][q_len][H][512] bf16       q_rope [B][q_len][H][64] bf16
    kv_pool  [num_pages][64][576] bf16     (576 = 512 latent + 64 RoPE)
    block_table [B][max_pages] int32       seq_lens [B] int32 (includes q_len)
    num_splits  [B] int32

Poisoning: every pool position that no request owns (spare pages, unused
block-table entries, slots past seq_len in a request's last page) holds NaN,
so a kernel that reads outside the visible range returns NaN.

The five named workloads follow the benchmark configurations: a tiny bf16
case, batch 1 and batch 16 at 128K context with an FP8 cache, a ragged
batch-32 bf16 case with 128 heads, and a q_len-4 speculative-verify case at
256K.
"""
from __future__ import annotations

import dataclasses
import math

import torch

PAGE = 64
D_LATENT, D_ROPE, D_ROW = 512, 64, 576
SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)
NAN_BF16 = float("nan")


@dataclasses.dataclass
class Spec:
    name: str
    B: int
    q_len: int
    H: int
    seq_lens: list          # per request, or None to draw from lo/hi
    kv_dtype: str           # "fp8" or "bf16"
    kv_std: float           # KV values ~ N(0, kv_std^2)
    splits: object          # int, or "by_length"
    seed: int
    shuffle_pages: bool = True
    len_range: tuple = None  # (lo, hi) inclusive for ragged lengths
    fp8_scale: object = "amax"  # "amax" -> amax/448, or a float
    spare_pages: int = 4


def splits_by_length(lens, num_sms: int = 148, max_splits: int = 64):
    """Per-request split counts for a ragged batch: splits of at most
    T = max(2048, ceil(sum(lens) / max(1, num_sms - B))) tokens, ceil(L / T)
    per request, 1..max_splits (at most num_sms splits when B < num_sms)."""
    T = max(2048, -(-sum(int(L) for L in lens) // max(1, num_sms - len(lens))))
    return [max(1, min(max_splits, -(-int(L) // T))) for L in lens]


SPECS = {
    "tiny": Spec("tiny", B=1, q_len=1, H=16, seq_lens=[1024], kv_dtype="bf16", kv_std=1.0,
                 splits=4, seed=0, shuffle_pages=False, spare_pages=2),
    "b1_128k_fp8": Spec("b1_128k_fp8", B=1, q_len=1, H=64, seq_lens=[131072], kv_dtype="fp8",
                        kv_std=2.0, splits=64, seed=1, fp8_scale=6.0 / 448.0),
    "b16_128k_fp8": Spec("b16_128k_fp8", B=16, q_len=1, H=64, seq_lens=[131072] * 16,
                         kv_dtype="fp8", kv_std=1.0, splits=32, seed=2),
    "b32_ragged_bf16": Spec("b32_ragged_bf16", B=32, q_len=1, H=128, seq_lens=None,
                            kv_dtype="bf16", kv_std=0.5, splits="by_length", seed=3,
                            len_range=(4096, 131072)),
    # profiling size: the batch-16 shape cut to 4 requests (302 MB of KV, > L2)
    "b4_128k_fp8": Spec("b4_128k_fp8", B=4, q_len=1, H=64, seq_lens=[131072] * 4,
                        kv_dtype="fp8", kv_std=1.0, splits=32, seed=5),
    "b4_128k_bf16": Spec("b4_128k_bf16", B=4, q_len=1, H=64, seq_lens=[131072] * 4,
                         kv_dtype="bf16", kv_std=1.0, splits=32, seed=5),
    "verify_q4_256k_fp8": Spec("verify_q4_256k_fp8", B=8, q_len=4, H=64,
                               seq_lens=[262144] * 8, kv_dtype="fp8", kv_std=1.0, splits=64,
                               seed=4),
    # profiling size: the verify shape cut to 2 requests (302 MB of KV, > L2)
    "verify_q4_256k_b2_fp8": Spec("verify_q4_256k_b2_fp8", B=2, q_len=4, H=64,
                                  seq_lens=[262144] * 2, kv_dtype="fp8", kv_std=1.0, splits=64,
                                  seed=6),
}


@dataclasses.dataclass
class Workload:
    spec: Spec
    q_nope: torch.Tensor       # bf16 [B][q_len][H][512]
    q_rope: torch.Tensor       # bf16 [B][q_len][H][64]
    kv_pool: torch.Tensor      # bf16 [num_pages][64][576] (pre-quantisation values for fp8)
    block_table: torch.Tensor  # int32 [B][max_pages]
    seq_lens: torch.Tensor     # int32 [B]
    num_splits: torch.Tensor   # int32 [B]
    max_splits: int
    kv_scale: float            # dequant scale for fp8 (1.0 for bf16)
    inv_scale: float           # fp32(1/kv_scale), the quantiser's multiplier
    softmax_scale: float = SOFTMAX_SCALE

    @property
    def B(self):
        return self.spec.B

    @property
    def q_len(self):
        return self.spec.q_len

    @property
    def H(self):
        return self.spec.H

    @property
    def kv_bytes(self) -> int:
        """Algorithmic KV bytes one decode step reads: sum_b L_b * 576 * elem size."""
        esz = 1 if self.spec.kv_dtype == "fp8" else 2
        return int(self.seq_lens.to(torch.int64).sum().item()) * D_ROW * esz


def make(spec, device="cpu", seq_lens=None, B=None, H=None, q_len=None, splits=None,
         kv_dtype=None, seed=None) -> Workload:
    """Build a workload from a named spec (or a Spec), with optional overrides.

    Values are drawn in fp32 from a ``torch.Generator`` seeded with the spec's
    seed on ``device`` and rounded to bf16.  CPU and CUDA draws differ; a test
    that compares two implementations gives both the same tensors.
    """
    if isinstance(spec, str):
        spec = SPECS[spec]
    spec = dataclasses.replace(spec)
    if B is not None:
        spec.B = B
    if H is not None:
        spec.H = H
    if q_len is not None:
        spec.q_len = q_len
    if splits is not None:
        spec.splits = splits
    if kv_dtype is not None:
        spec.kv_dtype = kv_dtype
    if seed is not None:
        spec.seed = seed
    if seq_lens is not None:
        spec.seq_lens = list(seq_lens)
        spec.B = len(spec.seq_lens)

    g = torch.Generator(device=device)
    g.manual_seed(spec.seed)
    Bn, Q, Hn = spec.B, spec.q_len, spec.H

    if spec.seq_lens is None:
        lo, hi = spec.len_range
        lens = torch.randint(lo, hi + 1, (Bn,), generator=g, device=device).cpu().tolist()
    else:
        lens = list(spec.seq_lens)
    assert len(lens) == Bn and all(L >= Q for L in lens)

    if spec.splits == "by_length":
        nsp = splits_by_length(lens)
    else:
        nsp = [int(spec.splits)] * Bn
    max_splits = max(nsp)

    pages_per_req = [-(-L // PAGE) for L in lens]
    max_pages = max(pages_per_req)
    used = sum(pages_per_req)
    num_pages = used + spec.spare_pages
    if spec.shuffle_pages:
        perm = torch.randperm(num_pages, generator=g, device=device).cpu()
    else:
        perm = torch.arange(num_pages)
    spare = perm[used:]
    spare_page = int(spare[0]) if spare.numel() else int(perm[-1])
    bt = torch.full((Bn, max_pages), spare_page, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_req):
        bt[b, :n] = perm[off:off + n].to(torch.int32)
        off += n

    q_nope = torch.randn((Bn, Q, Hn, D_LATENT), generator=g, device=device).to(torch.bfloat16)
    q_rope = torch.randn((Bn, Q, Hn, D_ROPE), generator=g, device=device).to(torch.bfloat16)

    kv = torch.empty((num_pages, PAGE, D_ROW), dtype=torch.bfloat16, device=device)
    chunk = max(1, (1 << 26) // (PAGE * D_ROW))  # draw in slabs of ~64M values
    for p0 in range(0, num_pages, chunk):
        p1 = min(num_pages, p0 + chunk)
        x = torch.randn((p1 - p0, PAGE, D_ROW), generator=g, device=device)
        if spec.kv_std != 1.0:
            x.mul_(spec.kv_std)
        kv[p0:p1] = x.to(torch.bfloat16)
    # poison everything no request owns
    owned = torch.zeros(num_pages, dtype=torch.bool)
    for b, n in enumerate(pages_per_req):
        owned[bt[b, :n].long()] = True
    kv[(~owned).to(device)] = NAN_BF16
    for b, L in enumerate(lens):
        tail = L % PAGE
        if tail:
            kv[int(bt[b, pages_per_req[b] - 1]), tail:, :] = NAN_BF16

    if spec.kv_dtype == "fp8":
        if spec.fp8_scale == "amax":
            amax = 0.0
            for b, n in enumerate(pages_per_req):
                pages = bt[b, :n].long().to(device)
                amax = max(amax, float(kv[pages].float().nan_to_num(0.0).abs().max()))
            kv_scale = float(torch.tensor(amax / 448.0, dtype=torch.float32))
        else:
            kv_scale = float(torch.tensor(float(spec.fp8_scale), dtype=torch.float32))
        inv_scale = float(torch.tensor(1.0, dtype=torch.float32) / torch.tensor(kv_scale, dtype=torch.float32))
    else:
        kv_scale, inv_scale = 1.0, 1.0

    return Workload(spec=spec, q_nope=q_nope, q_rope=q_rope, kv_pool=kv,
                    block_table=bt.to(device), seq_lens=torch.tensor(lens, dtype=torch.int32, device=device),
                    num_splits=torch.tensor(nsp, dtype=torch.int32, device=device),
                    max_splits=max_splits, kv_scale=kv_scale, inv_scale=inv_scale)


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
