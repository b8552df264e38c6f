"""Python binding of the B200 absorbed-MLA split-KV decode library.

A thin ctypes layer over the C ABI in include/mla.h: it checks tensor dtypes,
devices and shapes, passes raw device pointers and the current CUDA stream,
and raises :class:`MlaError` on a non-zero status.  Every step of the decode
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback: the
first call raises ImportError when the library has not been built.

Entry points (same names as the C ABI):

* ``mla_quantize_fp8(x_bf16, y_u8, inv_scale)`` — step A1, saturating E4M3.
* ``mla_decode_partial(...)`` — steps A2-A8, per-split partial O and LSE.
* ``mla_combine(...)`` — step A9, log-sum-exp merge into bf16 O and fp32 LSE.
* ``mla_decode_partial_q8(...)`` — steps A2-A8 with an FP8 query (E4M3 codes and
  one scale), an option beside the exact two-term bf16 query.
* ``mla_decode_fused(...)`` — steps A2-A9 in one cooperative launch (FP8 cache);
  it cuts every request into the same number of splits, as many as one wave of
  CTAs allows (``mla_fused_splits``); ``mla_fused_workspace_bytes`` and
  ``alloc_fused_workspace`` size and zero its workspace.
* ``mla_partial_workspace_bytes``, ``mla_choose_splits``, ``mla_status_string``.
* ``mla_append_kv_fp8(...)`` — the KV-append step before the path: RoPE on the
  64-wide key, saturating E4M3 and the paged write in one kernel;
  ``mla_rope_cos_sin_table(max_pos)`` builds its (cos, sin) table.
* ``mla_device_error_status(word)`` / ``check_device_error(dev_error)`` — fold
  the GPU's error word into MLA_ERR_DEVICE.
* ``mla_partial_grid(...)`` — host helper: the partial kernel's CTA layout for a shape.
* ``HostStaging`` — one pinned host buffer and one copy each way for a step's
  inputs and outputs (the host-buffer path); ``DecodeGraph`` — that step with
  the single launch captured as one CUDA graph.
* ``mla_debug_inject_stall(enable)`` — test hook for the bounded-wait failure path.
* ``mla_debug_merge_plan(v, gpi)`` — test hook: force the single launch's merge plan.

``mla_decode_noalloc`` (partial + merge with in-library scratch) is reached
through ``load()`` directly; its ctypes signature is in the GPU test that uses
it.

``decode(...)`` chains partial + combine with a caller-provided or freshly
allocated workspace.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_DEVICE = range(5)
MLA_ERR_SCRATCH_LIMIT = 5
MLA_KV_FP8_E4M3, MLA_KV_BF16 = 0, 1
DEVERR_BAD_PAGE, DEVERR_BAD_SEQLEN, DEVERR_TIMEOUT, DEVERR_BAD_SPLITS, DEVERR_SMEM_ALIGN = 1, 2, 4, 8, 16

EXPORTS = ("mla_quantize_fp8", "mla_partial_workspace_bytes", "mla_decode_partial",
           "mla_combine", "mla_choose_splits", "mla_device_error_status", "mla_status_string",
           "mla_decode_noalloc", "mla_partial_grid", "mla_debug_inject_stall", "mla_debug_merge_plan",
           "mla_append_kv_fp8", "mla_rope_cos_sin_table", "mla_combine_f32",
           "mla_merge_rank_partials", "mla_fused_splits", "mla_fused_workspace_bytes",
           "mla_decode_fused",
           "mla_decode_partial_q8")


class MlaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


_lib_handle = None


def load():
    """Load libmla_b200.so (raises ImportError if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load_lib()
    return _lib_handle


def _load_lib():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmla_b200.so is not built ({LIB_PATH}); run "
                          "`python -m mla_split_kv_absorbed_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.mla_quantize_fp8.argtypes = [P, P, i64, f32, P]
    lib.mla_quantize_fp8.restype = i32
    lib.mla_partial_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.mla_partial_workspace_bytes.restype = ctypes.c_size_t
    lib.mla_decode_partial.argtypes = [P, P, P, i32, f32, i64, P, i32, P, P, i32, i32, i32, i32,
                                       f32, P, P, P, P]
    lib.mla_decode_partial.restype = i32
    lib.mla_combine.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P]
    lib.mla_combine.restype = i32
    lib.mla_choose_splits.argtypes = [P, i32, i32, i32, P]
    lib.mla_choose_splits.restype = i32
    lib.mla_status_string.argtypes = [i32]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_partial_grid.argtypes = [i32, i32, i32, i32, i32, i32, P]
    lib.mla_partial_grid.restype = i32
    lib.mla_combine_f32.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P]
    lib.mla_combine_f32.restype = i32
    lib.mla_merge_rank_partials.argtypes = [P, P, i32, i32, i32, i32, P, P, P]
    lib.mla_merge_rank_partials.restype = i32
    lib.mla_append_kv_fp8.argtypes = [P, P, P, i64, P, i32, P, i32, i32, f32, P, i64, P, P]
    lib.mla_append_kv_fp8.restype = i32
    lib.mla_rope_cos_sin_table.argtypes = [P, i64, ctypes.c_double]
    lib.mla_rope_cos_sin_table.restype = i32
    lib.mla_device_error_status.argtypes = [i32]
    lib.mla_device_error_status.restype = i32
    lib.mla_debug_inject_stall.argtypes = [i32]
    lib.mla_debug_inject_stall.restype = i32
    lib.mla_debug_merge_plan.argtypes = [i32, i32]
    lib.mla_debug_merge_plan.restype = i32
    lib.mla_fused_splits.argtypes = [i32, i32, i32, i32]
    lib.mla_fused_splits.restype = i32
    lib.mla_fused_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.mla_fused_workspace_bytes.restype = ctypes.c_size_t
    lib.mla_decode_fused.argtypes = [P, P, P, i32, f32, i64, P, i32, P, i32, i32, i32,
                                     f32, P, ctypes.c_size_t, P, P, P, P]
    lib.mla_decode_fused.restype = i32
    lib.mla_decode_partial_q8.argtypes = [P, f32, P, f32, i64, P, i32, P, P, i32, i32, i32, i32,
                                          f32, P, P, P, P]
    lib.mla_decode_partial_q8.restype = i32
    return lib


class _LazyLib:
    def __getattr__(self, name):
        return getattr(load(), name)


_lib = _LazyLib()


def status_string(status: int) -> str:
    return _lib.mla_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != MLA_OK:
        raise MlaError(fn, status)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def mla_quantize_fp8(x: torch.Tensor, y: torch.Tensor, inv_scale: float, stream=None):
    """y (uint8 E4M3 codes) = saturating E4M3 of fl32(x * inv_scale); x bf16, same numel."""
    if x.numel() != y.numel():
        raise ValueError("x and y must have the same number of elements")
    _check("mla_quantize_fp8", _lib.mla_quantize_fp8(
        _dev(x, "x", torch.bfloat16), _dev(y, "y", torch.uint8), x.numel(), float(inv_scale),
        _stream(stream)))
    return y


def mla_partial_workspace_bytes(B: int, q_len: int, H: int, max_splits: int) -> int:
    return int(_lib.mla_partial_workspace_bytes(B, q_len, H, max_splits))


def alloc_partials(B, q_len, H, max_splits, device="cuda"):
    """(part_o [B][q_len][H][max_splits][512] fp32, part_lse [B][q_len][H][max_splits] fp32)."""
    po = torch.empty((B, q_len, H, max_splits, 512), dtype=torch.float32, device=device)
    pl = torch.empty((B, q_len, H, max_splits), dtype=torch.float32, device=device)
    return po, pl


def mla_decode_partial(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, num_splits,
                       max_splits, softmax_scale, part_o, part_lse, dev_error=None, stream=None):
    """Split-KV partial attention; kv_pages uint8 (E4M3) or bf16 [num_pages][64][576]."""
    B, q_len, H, dl = q_nope.shape
    if dl != 512 or tuple(q_rope.shape) != (B, q_len, H, 64):
        raise ValueError("q_nope must be [B][q_len][H][512] and q_rope [B][q_len][H][64]")
    if kv_pages.dim() != 3 or tuple(kv_pages.shape[1:]) != (64, 576):
        raise ValueError("kv_pages must be [num_pages][64][576]")
    if kv_pages.dtype == torch.uint8:
        kv_dtype = MLA_KV_FP8_E4M3
    elif kv_pages.dtype == torch.bfloat16:
        kv_dtype = MLA_KV_BF16
    else:
        raise ValueError("kv_pages must be uint8 (E4M3 codes) or bfloat16")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B][max_pages]")
    if part_o.numel() != B * q_len * H * max_splits * 512 or part_lse.numel() != B * q_len * H * max_splits:
        raise ValueError("partial buffers have the wrong size")
    _check("mla_decode_partial", _lib.mla_decode_partial(
        _dev(q_nope, "q_nope", torch.bfloat16), _dev(q_rope, "q_rope", torch.bfloat16),
        _dev(kv_pages, "kv_pages"), kv_dtype, float(kv_scale), kv_pages.shape[0],
        _dev(block_table, "block_table", torch.int32), block_table.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), _dev(num_splits, "num_splits", torch.int32),
        int(max_splits), B, q_len, H, float(softmax_scale),
        _dev(part_o, "part_o", torch.float32), _dev(part_lse, "part_lse", torch.float32),
        None if dev_error is None else _dev(dev_error, "dev_error", torch.int32), _stream(stream)))


def _device_sms(device=None) -> int:
    return torch.cuda.get_device_properties(
        torch.device("cuda") if device is None else torch.device(device)).multi_processor_count


def mla_fused_splits(B: int, q_len: int, H: int, num_sms: int) -> int:
    """Splits per request that mla_decode_fused uses on a GPU with num_sms SMs (0: none)."""
    return int(_lib.mla_fused_splits(B, q_len, H, num_sms))


def mla_fused_workspace_bytes(B: int, q_len: int, H: int, num_sms: int) -> int:
    return int(_lib.mla_fused_workspace_bytes(B, q_len, H, num_sms))


def alloc_fused_workspace(B, q_len, H, device="cuda"):
    """Workspace of mla_decode_fused on ``device``, zeroed (its two counters must start at
    zero); raises MlaError with MLA_ERR_UNSUPPORTED when the shape has no single launch."""
    n = mla_fused_workspace_bytes(B, q_len, H, _device_sms(device))
    if n == 0:
        raise MlaError("alloc_fused_workspace", MLA_ERR_UNSUPPORTED)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def mla_decode_fused(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, softmax_scale,
                     workspace, out, out_lse=None, dev_error=None, stream=None):
    """Single-launch decode over an FP8 cache, with mla_fused_splits(B, q_len, H, SMs) splits
    per request; raises MlaError with MLA_ERR_UNSUPPORTED for shapes without one."""
    B, q_len, H, dl = q_nope.shape
    if dl != 512 or tuple(q_rope.shape) != (B, q_len, H, 64):
        raise ValueError("q_nope must be [B][q_len][H][512] and q_rope [B][q_len][H][64]")
    if kv_pages.dtype != torch.uint8 or kv_pages.dim() != 3 or tuple(kv_pages.shape[1:]) != (64, 576):
        raise ValueError("kv_pages must be uint8 (E4M3 codes) [num_pages][64][576]")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B][max_pages]")
    if workspace.dtype != torch.uint8 or workspace.dim() != 1:
        raise ValueError("workspace must be a flat uint8 tensor (alloc_fused_workspace)")
    if tuple(out.shape) != (B, q_len, H, 512):
        raise ValueError("out must be [B][q_len][H][512]")
    _check("mla_decode_fused", _lib.mla_decode_fused(
        _dev(q_nope, "q_nope", torch.bfloat16), _dev(q_rope, "q_rope", torch.bfloat16),
        _dev(kv_pages, "kv_pages"), MLA_KV_FP8_E4M3, float(kv_scale), kv_pages.shape[0],
        _dev(block_table, "block_table", torch.int32), block_table.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, q_len, H, float(softmax_scale),
        _dev(workspace, "workspace"), workspace.numel(),
        _dev(out, "out", torch.bfloat16),
        None if out_lse is None else _dev(out_lse, "out_lse", torch.float32),
        None if dev_error is None else _dev(dev_error, "dev_error", torch.int32), _stream(stream)))
    return out


def mla_decode_partial_q8(q8, q_scale, kv_pages, kv_scale, block_table, seq_lens, num_splits,
                          max_splits, softmax_scale, part_o, part_lse, dev_error=None,
                          stream=None):
    """Split-KV partial attention with an FP8 query: q8 uint8 E4M3 codes
    [B][q_len][H][576] (latent then RoPE dims) of value code * q_scale."""
    B, q_len, H, dq = q8.shape
    if dq != 576 or q8.dtype != torch.uint8:
        raise ValueError("q8 must be uint8 [B][q_len][H][576]")
    if kv_pages.dtype != torch.uint8 or kv_pages.dim() != 3 or tuple(kv_pages.shape[1:]) != (64, 576):
        raise ValueError("kv_pages must be uint8 (E4M3 codes) [num_pages][64][576]")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B][max_pages]")
    if part_o.numel() != B * q_len * H * max_splits * 512 or part_lse.numel() != B * q_len * H * max_splits:
        raise ValueError("partial buffers have the wrong size")
    _check("mla_decode_partial_q8", _lib.mla_decode_partial_q8(
        _dev(q8, "q8", torch.uint8), float(q_scale), _dev(kv_pages, "kv_pages"), float(kv_scale),
        kv_pages.shape[0], _dev(block_table, "block_table", torch.int32), block_table.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), _dev(num_splits, "num_splits", torch.int32),
        int(max_splits), B, q_len, H, float(softmax_scale),
        _dev(part_o, "part_o", torch.float32), _dev(part_lse, "part_lse", torch.float32),
        None if dev_error is None else _dev(dev_error, "dev_error", torch.int32), _stream(stream)))


def mla_combine(part_o, part_lse, num_splits, max_splits, out, out_lse=None, stream=None):
    """Merge partials into out (bf16 [B][q_len][H][512]) and out_lse (fp32 [B][q_len][H])."""
    B, q_len, H, dl = out.shape
    if dl != 512:
        raise ValueError("out must be [B][q_len][H][512]")
    _check("mla_combine", _lib.mla_combine(
        _dev(part_o, "part_o", torch.float32), _dev(part_lse, "part_lse", torch.float32),
        _dev(num_splits, "num_splits", torch.int32), int(max_splits), B, q_len, H,
        _dev(out, "out", torch.bfloat16),
        None if out_lse is None else _dev(out_lse, "out_lse", torch.float32), _stream(stream)))
    return out


def mla_combine_f32(part_o, part_lse, num_splits, max_splits, out_o, out_lse, stream=None):
    """Merge one rank's split partials into one fp32 partial per row:
    out_o fp32 [B][q_len][H][512], out_lse fp32 [B][q_len][H]."""
    B, q_len, H, dl = out_o.shape
    if dl != 512 or tuple(out_lse.shape) != (B, q_len, H):
        raise ValueError("out_o must be [B][q_len][H][512] and out_lse [B][q_len][H]")
    _check("mla_combine_f32", _lib.mla_combine_f32(
        _dev(part_o, "part_o", torch.float32), _dev(part_lse, "part_lse", torch.float32),
        _dev(num_splits, "num_splits", torch.int32), int(max_splits), B, q_len, H,
        _dev(out_o, "out_o", torch.float32), _dev(out_lse, "out_lse", torch.float32),
        _stream(stream)))
    return out_o, out_lse


def mla_merge_rank_partials(rank_o, rank_lse, out, out_lse=None, stream=None):
    """Merge per-rank partials rank_o fp32 [N][B][q_len][H][512], rank_lse fp32
    [N][B][q_len][H] into out bf16 [B][q_len][H][512] (and out_lse)."""
    N = rank_o.shape[0]
    B, q_len, H, dl = out.shape
    if dl != 512 or tuple(rank_o.shape) != (N, B, q_len, H, 512) or \
            tuple(rank_lse.shape) != (N, B, q_len, H):
        raise ValueError("rank_o must be [N][B][q_len][H][512], rank_lse [N][B][q_len][H]")
    _check("mla_merge_rank_partials", _lib.mla_merge_rank_partials(
        _dev(rank_o, "rank_o", torch.float32), _dev(rank_lse, "rank_lse", torch.float32), N, B,
        q_len, H, _dev(out, "out", torch.bfloat16),
        None if out_lse is None else _dev(out_lse, "out_lse", torch.float32), _stream(stream)))
    return out


def mla_choose_splits(seq_lens_host, num_sms: int, max_splits: int):
    """Per-request split counts (host int32 tensor): one split per 2048 tokens,
    clamped to [1, max_splits]."""
    sl = torch.as_tensor(seq_lens_host, dtype=torch.int32).contiguous().cpu()
    out = torch.empty_like(sl)
    _check("mla_choose_splits", _lib.mla_choose_splits(
        ctypes.c_void_p(sl.data_ptr()), sl.numel(), num_sms, max_splits,
        ctypes.c_void_p(out.data_ptr())))
    return out


def mla_device_error_status(word: int) -> int:
    """MLA_OK for a zero device error word, MLA_ERR_DEVICE otherwise."""
    return int(_lib.mla_device_error_status(int(word)))


def check_device_error(dev_error) -> None:
    """Synchronise dev_error's stream and raise MlaError(MLA_ERR_DEVICE) if the
    GPU set any MLA_DEVERR_* bit."""
    word = int(dev_error.item())  # .item() waits for the work that writes it
    _check(f"device error word {word:#x}", mla_device_error_status(word))


def mla_rope_cos_sin_table(max_pos: int, base: float = 10000.0) -> torch.Tensor:
    """Host fp32 [max_pos][32][2] table of (cos, sin) of pos * base^(-2i/64)."""
    t = torch.empty((max_pos, 32, 2), dtype=torch.float32)
    _check("mla_rope_cos_sin_table", _lib.mla_rope_cos_sin_table(
        ctypes.c_void_p(t.data_ptr()), int(max_pos), float(base)))
    return t


def mla_append_kv_fp8(c_kv, k_rope, cos_sin, block_table, seq_lens, inv_scale, kv_pages,
                      dev_error=None, stream=None):
    """Write n_new tokens per request into the E4M3 cache kv_pages (uint8
    [num_pages][64][576]): c_kv bf16 [B][n_new][512], k_rope bf16 [B][n_new][64]
    (rotated here), cos_sin fp32 [max_pos][32][2] on the device."""
    B, n_new, dl = c_kv.shape
    if dl != 512 or tuple(k_rope.shape) != (B, n_new, 64):
        raise ValueError("c_kv must be [B][n_new][512] and k_rope [B][n_new][64]")
    if cos_sin.dim() != 3 or tuple(cos_sin.shape[1:]) != (32, 2):
        raise ValueError("cos_sin must be [max_pos][32][2]")
    if kv_pages.dim() != 3 or tuple(kv_pages.shape[1:]) != (64, 576):
        raise ValueError("kv_pages must be [num_pages][64][576]")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B][max_pages]")
    _check("mla_append_kv_fp8", _lib.mla_append_kv_fp8(
        _dev(c_kv, "c_kv", torch.bfloat16), _dev(k_rope, "k_rope", torch.bfloat16),
        _dev(cos_sin, "cos_sin", torch.float32), cos_sin.shape[0],
        _dev(block_table, "block_table", torch.int32), block_table.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, n_new, float(inv_scale),
        _dev(kv_pages, "kv_pages", torch.uint8), kv_pages.shape[0],
        None if dev_error is None else _dev(dev_error, "dev_error", torch.int32), _stream(stream)))
    return kv_pages


def mla_status_string(status: int) -> str:
    return status_string(status)


def mla_partial_grid(B: int, q_len: int, H: int, max_splits: int, kv_dtype: int, num_sms: int):
    """CTA layout mla_decode_partial uses: (ctas, pieces per cut unit, first
    cut unit, idle CTAs before the cut units)."""
    out = (ctypes.c_int32 * 4)()
    _check("mla_partial_grid", _lib.mla_partial_grid(B, q_len, H, max_splits, kv_dtype, num_sms,
                                                     ctypes.cast(out, ctypes.c_void_p)))
    return tuple(int(v) for v in out)


def mla_debug_inject_stall(enable: bool) -> bool:
    """Test hook: while enabled, FP8 partial launches leave one KV load of
    their first CTA unissued, so its bounded waits run out and the kernel
    reports MLA_DEVERR_TIMEOUT.  Returns the previous setting."""
    return bool(_lib.mla_debug_inject_stall(1 if enable else 0))


def mla_debug_merge_plan(v: int, gpi: int) -> None:
    """Test hook: later single launches merge with v dims per thread and gpi
    128-thread groups per item; (0, 0) restores the automatic choice."""
    _check("mla_debug_merge_plan", _lib.mla_debug_merge_plan(int(v), int(gpi)))


class HostStaging:
    """Host <-> device staging for one decode shape: a step's inputs (q_nope,
    q_rope, seq_lens, block_table and, optionally, num_splits) live in one
    pinned host buffer and go to the device in one copy; the outputs (O bf16
    and LSE fp32) come back in one copy.  Fill the host views (``host[name]``)
    and call ``upload()``; pass the device views (``dev[name]``) and
    ``out`` / ``out_lse`` to the decode call; ``download()`` copies the outputs
    into ``host_out`` / ``host_lse``.  Only torch copies: plumbing."""

    _ALIGN = 256

    def __init__(self, B, q_len, H, max_pages, with_num_splits=False, device="cuda"):
        spec = [("q_nope", torch.bfloat16, (B, q_len, H, 512)),
                ("q_rope", torch.bfloat16, (B, q_len, H, 64)),
                ("seq_lens", torch.int32, (B,)),
                ("block_table", torch.int32, (B, max_pages))]
        if with_num_splits:
            spec.append(("num_splits", torch.int32, (B,)))
        self.h_in, self.d_in, self.host, self.dev = self._carve(spec, device)
        self.in_bytes = self.h_in.numel()
        out_spec = [("out", torch.bfloat16, (B, q_len, H, 512)),
                    ("out_lse", torch.float32, (B, q_len, H))]
        self.h_out, self.d_out, hviews, dviews = self._carve(out_spec, device)
        self.out_bytes = self.h_out.numel()
        self.out, self.out_lse = dviews["out"], dviews["out_lse"]
        self.host_out, self.host_lse = hviews["out"], hviews["out_lse"]

    @classmethod
    def _carve(cls, spec, device):
        offs, n = [], 0
        for _, dt, shape in spec:
            nbytes = torch.empty((), dtype=dt).element_size()
            for d in shape:
                nbytes *= d
            offs.append((n, nbytes))
            n += (nbytes + cls._ALIGN - 1) // cls._ALIGN * cls._ALIGN
        h = torch.empty(n, dtype=torch.uint8).pin_memory()
        d = torch.empty(n, dtype=torch.uint8, device=device)
        hv, dv = {}, {}
        for (name, dt, shape), (o, nb) in zip(spec, offs):
            hv[name] = h[o:o + nb].view(dt).view(shape)
            dv[name] = d[o:o + nb].view(dt).view(shape)
        return h, d, hv, dv

    def upload(self, stream=None):
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.d_in.copy_(self.h_in, non_blocking=True)

    def download(self, stream=None):
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.h_out.copy_(self.d_out, non_blocking=True)


class DecodeGraph:
    """One decode step over host buffers captured as a CUDA graph: the
    HostStaging upload, the single launch (mla_decode_fused) and the download,
    replayed with one call, so the three need no host launches between them.
    The graph reads the staging buffers, the KV pool and the workspace at
    replay time: fill ``staging.host`` and call ``replay()``; the outputs land
    in ``staging.host_out`` / ``staging.host_lse`` once the stream reaches the
    end of the replay."""

    def __init__(self, staging, kv_pages, kv_scale, softmax_scale, workspace=None,
                 dev_error=None, warmup=2):
        self.st = staging
        d = staging.dev
        B, q_len, H, _ = d["q_nope"].shape
        self.workspace = alloc_fused_workspace(B, q_len, H) if workspace is None else workspace
        self.stream = torch.cuda.Stream()
        self.graph = torch.cuda.CUDAGraph()
        args = (d["q_nope"], d["q_rope"], kv_pages, kv_scale, d["block_table"], d["seq_lens"],
                softmax_scale, self.workspace, staging.out, staging.out_lse, dev_error)

        def step():
            staging.upload(self.stream)
            mla_decode_fused(*args, stream=self.stream)
            staging.download(self.stream)
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                step()
        self.stream.synchronize()
        with torch.cuda.graph(self.graph, stream=self.stream):
            step()
        self.stream.synchronize()

    def replay(self, stream=None):
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.graph.replay()


def decode(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, num_splits, max_splits,
           softmax_scale, out=None, out_lse=None, workspace=None, dev_error=None, stream=None):
    """partial + combine; returns (out bf16 [B][q_len][H][512], out_lse fp32 [B][q_len][H])."""
    B, q_len, H, _ = q_nope.shape
    dev = q_nope.device
    if workspace is None:
        workspace = alloc_partials(B, q_len, H, max_splits, dev)
    part_o, part_lse = workspace
    if out is None:
        out = torch.empty((B, q_len, H, 512), dtype=torch.bfloat16, device=dev)
    if out_lse is None:
        out_lse = torch.empty((B, q_len, H), dtype=torch.float32, device=dev)
    mla_decode_partial(q_nope, q_rope, kv_pages, kv_scale, block_table, seq_lens, num_splits,
                       max_splits, softmax_scale, part_o, part_lse, dev_error, stream)
    mla_combine(part_o, part_lse, num_splits, max_splits, out, out_lse, stream)
    return out, out_lse
