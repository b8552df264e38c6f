"""CPU oracle for absorbed MLA split-KV decode (test infrastructure only).

The oracle is a plain fp64 C implementation (``oracle.c``) of what the GPU
path computes, loaded here through ctypes.  Only the tests, the smoke check
and the benchmark's CPU-baseline leg use it; the CUDA library never imports,
links or calls it, and it never touches a GPU.

Functions (each cites its passage in ``oracle.c``):

* :func:`e4m3_value`, :func:`e4m3_encode`, :func:`quantize` — the saturating
  E4M3 conversion of the prep step ("SGLang & Miles ... Vera Rubin" article,
  bullet "原生 FP8 转换": overflow clamps to +-448, never NaN).
* :func:`decode_rows` — softmax(q k^T * scale) v over the dequantised paged
  latent cache, per listed (b, q, h) row.
* :func:`split_range`, :func:`partials_rows` — the per-split partial results
  (same article, bullet "更快的 split-KV 归约").
* :func:`combine` — the log-sum-exp merge of the partials done by the second
  kernel (same bullet).
* :func:`rope_f64`, :func:`rope_table`, :func:`append_kv` — the KV-append step
  before the path: RoPE on the 64-wide key, saturating E4M3 and the paged
  write ("Muse Spark Open" article, bullet "RoPE 与 KV 缓存写入融合").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

D_LATENT, D_ROPE, D_ROW, PAGE = 512, 64, 576, 64


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, fp64, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
               "-shared", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_quantize.argtypes = [P, P, i64, f32]
        lib.oracle_mla_decode_rows.argtypes = [P, P, P, i32, f32, P, i32, P, i32, i32, i32,
                                               f32, P, i64, P, P]
        lib.oracle_split_range.argtypes = [i64, i32, i32, i64, ctypes.POINTER(i64),
                                           ctypes.POINTER(i64)]
        lib.oracle_mla_partials_rows.argtypes = [P, P, P, i32, f32, P, i32, P, P, i32, i32,
                                                 i32, i32, f32, P, i64, P, P]
        lib.oracle_mla_partials_rows_q8.argtypes = [P, f32, P, i32, f32, P, i32, P, P, i32, i32,
                                                    i32, i32, f32, P, i64, P, P]
        lib.oracle_combine.argtypes = [P, P, P, i32, i64, P, P]
        lib.oracle_num_threads.restype = i32
        lib.oracle_rope_f64.argtypes = [P, i64, ctypes.c_double, P]
        lib.oracle_rope_table.argtypes = [i64, ctypes.c_double, P]
        lib.oracle_append_kv.argtypes = [P, P, P, i64, P, i32, P, i32, i32, f32, P, i64]
        lib.oracle_append_kv.restype = i64
        lib.oracle_set_num_threads.argtypes = [i32]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the following oracle calls (OpenMP); used to time it on one core."""
    _load().oracle_set_num_threads(int(n))


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def e4m3_encode(x: float) -> int:
    return int(_load().oracle_e4m3_encode(float(x)))


def quantize(x_bf16_bits: np.ndarray, inv_scale: float) -> np.ndarray:
    """x: uint16 bf16 bit patterns -> uint8 E4M3 codes."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    y = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_quantize(_ptr(x), _ptr(y), x.size, float(np.float32(inv_scale)))
    return y


def _kv_args(kv_pages: np.ndarray):
    if kv_pages.dtype == np.uint8:
        return 0, np.ascontiguousarray(kv_pages)
    if kv_pages.dtype == np.uint16:
        return 1, np.ascontiguousarray(kv_pages)
    raise TypeError("kv_pages must be uint8 (E4M3 codes) or uint16 (bf16 bits)")


def decode_rows(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, q_len, H,
                softmax_scale, rows):
    """Unsplit decode of the listed rows (row = (b*q_len + q)*H + h).

    q_nope/q_rope: uint16 bf16 bits [B][q_len][H][512|64]; kv_pages: uint8 E4M3
    codes or uint16 bf16 bits [num_pages][64][576]; block_table int32
    [B][max_pages]; seq_lens int32 [B].  Returns (O [n][512] f64, LSE [n] f64).
    """
    lib = _load()
    kv_dtype, kv = _kv_args(kv_pages)
    qn = np.ascontiguousarray(q_nope, dtype=np.uint16)
    qr = np.ascontiguousarray(q_rope, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    B = sl.shape[0]
    o = np.zeros((rows.size, D_LATENT), dtype=np.float64)
    lse = np.zeros(rows.size, dtype=np.float64)
    lib.oracle_mla_decode_rows(_ptr(qn), _ptr(qr), _ptr(kv), kv_dtype, float(kv_scale),
                               _ptr(bt), bt.shape[1], _ptr(sl), B, q_len, H,
                               float(softmax_scale), _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    return o, lse


def split_range(L: int, S: int, s: int, vis: int):
    t0, t1 = ctypes.c_int64(), ctypes.c_int64()
    _load().oracle_split_range(int(L), int(S), int(s), int(vis), ctypes.byref(t0), ctypes.byref(t1))
    return t0.value, t1.value


def partials_rows(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, num_splits,
                  max_splits, q_len, H, softmax_scale, rows):
    """Per-split partials for the listed rows: (O [n][max_splits][512], LSE [n][max_splits])."""
    lib = _load()
    kv_dtype, kv = _kv_args(kv_pages)
    qn = np.ascontiguousarray(q_nope, dtype=np.uint16)
    qr = np.ascontiguousarray(q_rope, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    ns = np.ascontiguousarray(num_splits, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    B = sl.shape[0]
    o = np.zeros((rows.size, max_splits, D_LATENT), dtype=np.float64)
    lse = np.zeros((rows.size, max_splits), dtype=np.float64)
    lib.oracle_mla_partials_rows(_ptr(qn), _ptr(qr), _ptr(kv), kv_dtype, float(kv_scale),
                                 _ptr(bt), bt.shape[1], _ptr(sl), _ptr(ns), int(max_splits), B,
                                 q_len, H, float(softmax_scale), _ptr(rows), rows.size, _ptr(o),
                                 _ptr(lse))
    return o, lse


def partials_rows_q8(q8, q_scale, kv_pages, kv_scale, block_table, seq_lens, num_splits,
                     max_splits, q_len, H, softmax_scale, rows):
    """partials_rows with an FP8 query: q8 uint8 E4M3 codes [B][q_len][H][576]
    (latent then RoPE dims) of value code * q_scale."""
    lib = _load()
    kv_dtype, kv = _kv_args(kv_pages)
    q = np.ascontiguousarray(q8, dtype=np.uint8)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    ns = np.ascontiguousarray(num_splits, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    B = sl.shape[0]
    o = np.zeros((rows.size, max_splits, D_LATENT), dtype=np.float64)
    lse = np.zeros((rows.size, max_splits), dtype=np.float64)
    lib.oracle_mla_partials_rows_q8(_ptr(q), float(np.float32(q_scale)), _ptr(kv), kv_dtype,
                                    float(kv_scale), _ptr(bt), bt.shape[1], _ptr(sl), _ptr(ns),
                                    int(max_splits), B, q_len, H, float(softmax_scale),
                                    _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    return o, lse


def combine(part_o: np.ndarray, part_lse: np.ndarray, n_splits: np.ndarray):
    """Merge fp32 partials [R][max_splits][512] / [R][max_splits] using n_splits[R]."""
    lib = _load()
    po = np.ascontiguousarray(part_o, dtype=np.float32)
    pl = np.ascontiguousarray(part_lse, dtype=np.float32)
    ns = np.ascontiguousarray(n_splits, dtype=np.int32)
    R, S = pl.shape
    o = np.zeros((R, D_LATENT), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    lib.oracle_combine(_ptr(po), _ptr(pl), _ptr(ns), S, R, _ptr(o), _ptr(lse))
    return o, lse


def rope_f64(x, pos: int, base: float = 10000.0) -> np.ndarray:
    """RoPE of one 64-wide key in fp64 (pairs (2i, 2i+1), theta_i = base^(-2i/64))."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.shape == (D_ROPE,)
    y = np.empty(D_ROPE, dtype=np.float64)
    _load().oracle_rope_f64(_ptr(x), int(pos), float(base), _ptr(y))
    return y


def rope_table(max_pos: int, base: float = 10000.0) -> np.ndarray:
    """fp32 [max_pos][32][2] (cos, sin) of pos * theta_i, each rounded once from fp64."""
    t = np.empty((max_pos, D_ROPE // 2, 2), dtype=np.float32)
    _load().oracle_rope_table(int(max_pos), float(base), _ptr(t))
    return t


def append_kv(c_kv_bits, k_rope_bits, cos_sin, block_table, seq_lens, n_new: int, inv_scale: float,
              kv_pages: np.ndarray) -> int:
    """Write n_new tokens per request into kv_pages (uint8 [num_pages][64][576], in
    place).  c_kv_bits uint16 [B][n_new][512], k_rope_bits uint16 [B][n_new][64]
    (bf16 bits).  Returns the number of tokens skipped as out of range."""
    lib = _load()
    c = np.ascontiguousarray(c_kv_bits, dtype=np.uint16)
    r = np.ascontiguousarray(k_rope_bits, dtype=np.uint16)
    cs = np.ascontiguousarray(cos_sin, dtype=np.float32)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert kv_pages.dtype == np.uint8 and kv_pages.flags["C_CONTIGUOUS"]
    B = bt.shape[0]
    return int(lib.oracle_append_kv(_ptr(c), _ptr(r), _ptr(cs), cs.shape[0], _ptr(bt), bt.shape[1],
                                    _ptr(sl), B, int(n_new), float(np.float32(inv_scale)),
                                    _ptr(kv_pages), kv_pages.shape[0]))
