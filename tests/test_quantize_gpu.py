"""Step A1 on the GPU: mla_quantize_fp8 must match the oracle bit for bit."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

ALL = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def _gpu_quant(bits: np.ndarray, inv: float, offset_x=0, offset_y=0):
    import mla_split_kv_absorbed_b200 as m
    n = bits.size
    xs = torch.empty(n + offset_x, dtype=torch.int16, device="cuda")
    xs[offset_x:] = torch.from_numpy(bits.view(np.int16)).cuda()
    ys = torch.full((n + offset_y,), 0xAB, dtype=torch.uint8, device="cuda")
    x = xs[offset_x:].view(torch.bfloat16)
    y = ys[offset_y:]
    m.mla_quantize_fp8(x, y, inv)
    torch.cuda.synchronize()
    out = ys.cpu().numpy()
    assert np.all(out[:offset_y] == 0xAB)  # nothing written before the output
    return out[offset_y:]


def _check(got, ref, bits, inv):
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        nan_in = np.isnan(x * np.float32(inv))
    # NaN inputs: any E4M3 NaN code is accepted (the pages do not fix its sign)
    assert np.all((got[nan_in] & 0x7F) == 0x7F)
    bad = np.nonzero(got[~nan_in] != ref[~nan_in])[0]
    assert bad.size == 0, f"{bad.size} mismatches, first input bits {bits[~nan_in][bad[:5]]}"


@pytest.mark.parametrize("scale", [1.0, 2.0 ** -3, 6.0 / 448.0, 1.0 / 3.0, 3.7 / 448.0, 4096.0, 1e-30])
def test_quantize_all_bf16_patterns_bit_exact(scale):
    inv = float(np.float32(1.0) / np.float32(scale))
    got = _gpu_quant(ALL, inv)
    _check(got, oracle.quantize(ALL, inv), ALL, inv)


@pytest.mark.parametrize("n", [1, 7, 31, 32, 33, 1000, 65537])
@pytest.mark.parametrize("offx,offy", [(0, 0), (1, 0), (0, 3), (5, 7), (8, 16)])
def test_quantize_alignment_and_tails(n, offx, offy):
    rng = np.random.default_rng(n + 31 * offx + offy)
    bits = (rng.standard_normal(n).astype(np.float32) * 50).view(np.uint32) >> 16
    bits = bits.astype(np.uint16)
    inv = float(np.float32(1.0) / np.float32(0.07))
    got = _gpu_quant(bits, inv, offx, offy)
    _check(got, oracle.quantize(bits, inv), bits, inv)


def test_quantize_large_saturating_stream():
    # 2*N(0,1) with scale 6/448: |x| > 6 saturates at +-448 (about 0.27% of values)
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(1 << 24, generator=g) * 2).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    inv = float(np.float32(1.0) / np.float32(6.0 / 448.0))
    got = _gpu_quant(bits, inv)
    ref = oracle.quantize(bits, inv)
    _check(got, ref, bits, inv)
    assert np.mean((ref & 0x7F) == 0x7E) > 1e-3  # saturation really happened
