"""Second, independent fp64 formulation in NumPy, used only to pin the C oracle.

It shares nothing with ``oracle/oracle.c``: the E4M3 value map is the
closed-form bit formula (vectorised), rounding is a brute-force argmin over
all finite codes, and attention is a dense gather + matmul + log-sum-exp.
It is meant for tiny inputs.
"""
from __future__ import annotations

import numpy as np

PAGE, D_LATENT, D_ROW = 64, 512, 576


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e.astype(np.float64) - 7))
    v = np.where(s == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, v)


_FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.int64)
_FINITE_VALS = e4m3_values(_FINITE)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 code by exhaustive argmin, ties to the even code,
    saturating to +-448; NaN -> 0x7F.  Sign of zero follows the input."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64).ravel()
    out = np.empty(x.shape, dtype=np.uint8)
    nan = np.isnan(x)
    xc = np.clip(np.nan_to_num(x, nan=0.0, posinf=1e300, neginf=-1e300), -448.0, 448.0)
    d = np.abs(xc[:, None] - _FINITE_VALS[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equally near codes prefer even codes (ties to even); among the
    # remaining (only +0 / -0 for zero) prefer the one with the input's sign
    even = (_FINITE & 1) == 0
    neg_in = np.signbit(x)[:, None]
    code_neg = (_FINITE >= 128)[None, :]
    score = cand * 4 + (cand & even[None, :]) * 2 + (cand & (code_neg == neg_in)) * 1
    out[:] = _FINITE[np.argmax(score, axis=1)]
    out[nan] = 0x7F
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequant_pool(kv_pool, kv_scale):
    if kv_pool.dtype == np.uint8:
        return e4m3_values(kv_pool) * float(kv_scale)
    return bf16_bits_to_f64(kv_pool)


def attend(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, q_len, H, softmax_scale):
    """Dense reference: returns O [B][q_len][H][512], LSE [B][q_len][H] (fp64)."""
    kv = dequant_pool(kv_pages, kv_scale)
    qn = bf16_bits_to_f64(q_nope)
    qr = bf16_bits_to_f64(q_rope)
    B = len(seq_lens)
    O = np.zeros((B, q_len, H, D_LATENT))
    LSE = np.zeros((B, q_len, H))
    for b in range(B):
        L = int(seq_lens[b])
        t = np.arange(L)
        rows = kv[np.asarray(block_table[b])[t // PAGE], t % PAGE]  # [L][576]
        for q in range(q_len):
            vis = L - q_len + q + 1
            K = rows[:vis]
            qv = np.concatenate([qn[b, q], qr[b, q]], axis=-1)  # [H][576]
            s = softmax_scale * (qv @ K.T)  # [H][vis]
            m = s.max(axis=1, keepdims=True)
            w = np.exp(s - m)
            l = w.sum(axis=1, keepdims=True)
            O[b, q] = (w @ K[:, :D_LATENT]) / l
            LSE[b, q] = (m + np.log(l))[:, 0]
    return O, LSE
