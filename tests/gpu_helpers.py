"""Helpers shared by the GPU parity tests.

Inputs come from the seeded workload generator; FP8 caches are quantised on
the host by the oracle's quantiser (so no oracle input comes from the CUDA
path), then copied to the device for the library.  Expected values come from
the oracle only.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from mla_split_kv_absorbed_b200 import workloads as wl

# Tolerances for attention outputs (bf16 O against the fp64 oracle):
# max-abs 1e-2 and relative L2 5e-3 on O; LSE within 1e-3 * max(1, |LSE|).
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_TOL = 1e-3


@dataclasses.dataclass
class Case:
    w: wl.Workload
    kv_host: np.ndarray        # uint8 codes or uint16 bf16 bits [num_pages][64][576]
    kv_dev: torch.Tensor       # same bytes on the device (uint8 or bf16)
    qn_bits: np.ndarray
    qr_bits: np.ndarray
    dev: dict


def make_case(spec, gen_device="cpu", **overrides) -> Case:
    w = wl.make(spec, device=gen_device, **overrides)
    pool_bits = wl.bf16_bits(w.kv_pool)
    if w.spec.kv_dtype == "fp8":
        kv_host = oracle.quantize(pool_bits, w.inv_scale)
        kv_dev = torch.from_numpy(kv_host).cuda()
    else:
        kv_host = pool_bits
        kv_dev = w.kv_pool.to("cuda", torch.bfloat16)
    dev = dict(q_nope=w.q_nope.cuda(), q_rope=w.q_rope.cuda(), block_table=w.block_table.cuda(),
               seq_lens=w.seq_lens.cuda(), num_splits=w.num_splits.cuda())
    return Case(w=w, kv_host=kv_host, kv_dev=kv_dev, qn_bits=wl.bf16_bits(w.q_nope),
                qr_bits=wl.bf16_bits(w.q_rope), dev=dev)


def run_gpu(case: Case, max_splits=None):
    import mla_split_kv_absorbed_b200 as m
    w = case.w
    S = w.max_splits if max_splits is None else max_splits
    part_o, part_lse = m.alloc_partials(w.B, w.q_len, w.H, S)
    part_o.fill_(float("nan"))
    part_lse.fill_(float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = m.decode(case.dev["q_nope"], case.dev["q_rope"], case.kv_dev, w.kv_scale,
                        case.dev["block_table"], case.dev["seq_lens"], case.dev["num_splits"], S,
                        w.softmax_scale, workspace=(part_o, part_lse), dev_error=err)
    torch.cuda.synchronize()
    return out, lse, part_o, part_lse, int(err.item())


def oracle_rows(case: Case, rows):
    w = case.w
    return oracle.decode_rows(case.qn_bits, case.qr_bits, case.kv_host, w.kv_scale,
                              w.block_table.cpu().numpy(), w.seq_lens.cpu().numpy(), w.q_len, w.H,
                              w.softmax_scale, np.asarray(rows, dtype=np.int64))


def oracle_partials(case: Case, rows, max_splits=None):
    w = case.w
    S = w.max_splits if max_splits is None else max_splits
    return oracle.partials_rows(case.qn_bits, case.qr_bits, case.kv_host, w.kv_scale,
                                w.block_table.cpu().numpy(), w.seq_lens.cpu().numpy(),
                                w.num_splits.cpu().numpy(), S, w.q_len, w.H, w.softmax_scale,
                                np.asarray(rows, dtype=np.int64))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def assert_attention_close(o_gpu_bf16: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray,
                           lse_ref: np.ndarray, what=""):
    o = o_gpu_bf16.astype(np.float64)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    # The output is bf16: even the correctly rounded value is up to half a bf16
    # ulp away from the fp64 reference (0.0156 for |O| in [4, 8)), so the
    # max-abs bound applies to the error beyond that rounding.
    err = np.maximum(np.abs(o - o_ref) - bf16_half_ulp(o_ref), 0.0)
    max_abs = float(err.max())
    rel_l2 = float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    print(f"[parity] {what}: max-abs beyond bf16 rounding {max_abs:.3e}, rel-L2 {rel_l2:.3e}")
    assert max_abs <= O_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {O_MAX_ABS}"
    assert rel_l2 <= O_REL_L2, f"{what}: rel-L2 {rel_l2:.3e} > {O_REL_L2}"
    l = lse_gpu.astype(np.float64)
    both_inf = np.isneginf(l) & np.isneginf(lse_ref)
    fin = ~both_inf
    assert np.all(np.isfinite(l[fin])) and np.all(np.isfinite(lse_ref[fin])), f"{what}: LSE -inf mismatch"
    lerr = np.abs(l[fin] - lse_ref[fin]) / np.maximum(1.0, np.abs(lse_ref[fin]))
    assert lerr.size == 0 or float(lerr.max()) <= LSE_TOL, f"{what}: LSE err {float(lerr.max()):.3e}"
    return max_abs, rel_l2
