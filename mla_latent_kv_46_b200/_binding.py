"""ctypes binding of libmla.so (include/mla.h): argument marshalling only.

Every function has the C name and argument order. Tensor arguments may be torch
tensors (their data_ptr() is passed), plain integers (raw device addresses) or
None (NULL). `stream` defaults to torch's current CUDA stream. A negative status
raises MlaError carrying the status and mla_last_error().
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# MLA_LIBRARY may point at another build of the same library (e.g. an instrumented one).
LIB_PATH = os.environ.get("MLA_LIBRARY") or os.path.join(_PKG, "_lib", "libmla.so")

MLA_OK, MLA_ERR_INVALID, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE, MLA_ERR_CUDA, MLA_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
MLA_BF16, MLA_F32 = 0, 1
MLA_POLICY_AUTO, MLA_POLICY_SIMT, MLA_POLICY_TCGEN05 = 0, 1, 2

STATUS_NAMES = {0: "MLA_OK", -1: "MLA_ERR_INVALID", -2: "MLA_ERR_UNSUPPORTED", -3: "MLA_ERR_WORKSPACE",
                -4: "MLA_ERR_CUDA", -5: "MLA_ERR_TIMEOUT"}

# Every symbol include/mla.h declares.
EXPORTS = ("mla_abi_version", "mla_last_error", "mla_set_policy", "mla_set_wait_timeout_ns", "mla_set_plan_combine_cost",
           "mla_check_status", "mla_cache_append", "mla_cache_write", "mla_cache_write_workspace_size", "mla_absorb_q", "mla_plan_capacity", "mla_plan_splits",
           "mla_workspace_size", "mla_decode_attn", "mla_combine", "mla_out_proj", "mla_decode_attn_noalloc",
           "mla_debug_drop_page_load", "mla_quantize_rows_fp8", "mla_cache_append_fp8", "mla_workspace_size_fp8",
           "mla_decode_attn_fp8", "mla_prefill_workspace_size", "mla_prefill_attn")


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("Dn", ctypes.c_int32), ("Dr", ctypes.c_int32), ("Dv", ctypes.c_int32),
                ("R", ctypes.c_int32), ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32)]

    def __repr__(self):
        return (f"Dims(H={self.H}, Dn={self.Dn}, Dr={self.Dr}, Dv={self.Dv}, R={self.R}, "
                f"page_size={self.page_size}, dtype={self.dtype})")


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_items", ctypes.c_int32), ("num_units", ctypes.c_int32), ("num_slots", ctypes.c_int32),
                ("num_parts", ctypes.c_int32), ("head_groups", ctypes.c_int32), ("plan_words", ctypes.c_int32),
                ("max_pages", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python mla_latent_kv_46_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, U64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_float
    I64 = ctypes.c_int64
    D, INFO = Dims, ctypes.POINTER(PlanInfo)
    sig = {
        "mla_abi_version": (I32, []),
        "mla_last_error": (ctypes.c_char_p, []),
        "mla_set_policy": (I32, [I32]),
        "mla_set_wait_timeout_ns": (I32, [U64]),
        "mla_set_plan_combine_cost": (I32, [ctypes.c_double]),
        "mla_debug_drop_page_load": (I32, [I32]),
        "mla_check_status": (I32, [P]),
        "mla_cache_append": (I32, [P, P, P, P, I32, I32, I32, I32, D, P]),
        "mla_cache_write": (I32, [P, P, P, I32, P, P, P, I32, I32, I32, I32, P, F, F, P, SZ, D, P]),
        "mla_cache_write_workspace_size": (SZ, [I32, I32]),
        "mla_absorb_q": (I32, [P, P, P, I32, D, P]),
        "mla_plan_capacity": (SZ, [I32, I32, I32]),
        "mla_plan_splits": (I32, [P, I32, I32, I32, D, I32, P, SZ, INFO]),
        "mla_workspace_size": (SZ, [INFO, D]),
        "mla_decode_attn": (I32, [P, P, P, P, P, I32, I32, I32, I32, F, P, INFO, P, P, P, SZ, D, P]),
        "mla_combine": (I32, [P, INFO, P, SZ, P, P, D, P]),
        "mla_out_proj": (I32, [P, P, P, I32, D, P]),
        "mla_decode_attn_noalloc": (I32, [P, P, P, P, P, I32, I32, I32, I32, F, P, INFO, P, P, D, P]),
        "mla_quantize_rows_fp8": (I32, [P, P, P, I64, D, P]),
        "mla_cache_append_fp8": (I32, [P, P, P, P, P, I32, I32, I32, I32, D, P]),
        "mla_workspace_size_fp8": (SZ, [INFO, D]),
        "mla_decode_attn_fp8": (I32, [P, P, P, P, P, P, I32, I32, I32, I32, F, P, INFO, P, P, P, SZ, D, P]),
        "mla_prefill_workspace_size": (SZ, [I32, D]),
        "mla_prefill_attn": (I32, [P, P, P, P, P, P, P, I32, F, P, P, SZ, D, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status, where):
    if status != MLA_OK:
        raise MlaError(status, where, mla_last_error())


def mla_abi_version() -> int:
    return _lib.mla_abi_version()


def mla_last_error() -> str:
    return _lib.mla_last_error().decode()


def mla_set_policy(policy: int) -> None:
    _check(_lib.mla_set_policy(policy), "mla_set_policy")


def mla_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.mla_set_wait_timeout_ns(ns), "mla_set_wait_timeout_ns")


def mla_set_plan_combine_cost(pages: float) -> None:
    _check(_lib.mla_set_plan_combine_cost(float(pages)), "mla_set_plan_combine_cost")


def mla_debug_drop_page_load(ordinal: int) -> None:
    _check(_lib.mla_debug_drop_page_load(ordinal), "mla_debug_drop_page_load")


def mla_check_status(stream=None) -> None:
    _check(_lib.mla_check_status(_stream(stream)), "mla_check_status")


def mla_cache_append(kv_cache, block_table, seq_lens, new_ckr, B, q_len, max_pages, num_pages, dims, stream=None):
    _check(_lib.mla_cache_append(_ptr(kv_cache), _ptr(block_table), _ptr(seq_lens), _ptr(new_ckr), B, q_len,
                                 max_pages, num_pages, dims, _stream(stream)), "mla_cache_append")


def mla_cache_write_workspace_size(T, M) -> int:
    return _lib.mla_cache_write_workspace_size(T, M)


def mla_cache_write(hidden, W_DKV, kv_gain, M, kv_cache, block_table, seq_lens, B, q_len, max_pages, num_pages,
                    q_rope, eps, rope_base, workspace, workspace_bytes, dims, stream=None):
    _check(_lib.mla_cache_write(_ptr(hidden), _ptr(W_DKV), _ptr(kv_gain), M, _ptr(kv_cache), _ptr(block_table),
                                _ptr(seq_lens), B, q_len, max_pages, num_pages, _ptr(q_rope), eps, rope_base,
                                _ptr(workspace), workspace_bytes, dims, _stream(stream)), "mla_cache_write")


def mla_absorb_q(q_nope, W_UK, q_lat, T, dims, stream=None):
    _check(_lib.mla_absorb_q(_ptr(q_nope), _ptr(W_UK), _ptr(q_lat), T, dims, _stream(stream)), "mla_absorb_q")


def mla_plan_capacity(B, q_len, num_sms) -> int:
    return _lib.mla_plan_capacity(B, q_len, num_sms)


def mla_plan_splits(seq_lens_host, B, q_len, max_pages, dims, num_sms):
    """Returns (plan int32 numpy array of info.plan_words words, PlanInfo)."""
    lens = np.ascontiguousarray(seq_lens_host, dtype=np.int32)
    cap = mla_plan_capacity(B, q_len, num_sms)
    buf = np.zeros(max(cap, 1), dtype=np.int32)
    info = PlanInfo()
    _check(_lib.mla_plan_splits(lens.ctypes.data, B, q_len, max_pages, dims, num_sms, buf.ctypes.data, cap,
                                ctypes.byref(info)), "mla_plan_splits")
    return buf[:info.plan_words].copy(), info


def mla_workspace_size(info, dims) -> int:
    return _lib.mla_workspace_size(ctypes.byref(info), dims)


def mla_decode_attn(q_lat, q_rope, kv_cache, block_table, seq_lens, B, q_len, max_pages, num_pages, scale,
                    plan_dev, info, o_lat, lse, workspace, workspace_bytes, dims, stream=None):
    _check(_lib.mla_decode_attn(_ptr(q_lat), _ptr(q_rope), _ptr(kv_cache), _ptr(block_table), _ptr(seq_lens), B,
                                q_len, max_pages, num_pages, scale, _ptr(plan_dev), ctypes.byref(info),
                                _ptr(o_lat), _ptr(lse), _ptr(workspace), workspace_bytes, dims, _stream(stream)),
           "mla_decode_attn")


def mla_combine(plan_dev, info, workspace, workspace_bytes, o_lat, lse, dims, stream=None):
    _check(_lib.mla_combine(_ptr(plan_dev), ctypes.byref(info), _ptr(workspace), workspace_bytes, _ptr(o_lat),
                            _ptr(lse), dims, _stream(stream)), "mla_combine")


def mla_out_proj(o_lat, W_UV, out, T, dims, stream=None):
    _check(_lib.mla_out_proj(_ptr(o_lat), _ptr(W_UV), _ptr(out), T, dims, _stream(stream)), "mla_out_proj")


def mla_decode_attn_noalloc(q_lat, q_rope, kv_cache, block_table, seq_lens, B, q_len, max_pages, num_pages,
                            scale, plan_dev, info, o_lat, lse, dims, stream=None):
    _check(_lib.mla_decode_attn_noalloc(_ptr(q_lat), _ptr(q_rope), _ptr(kv_cache), _ptr(block_table),
                                        _ptr(seq_lens), B, q_len, max_pages, num_pages, scale, _ptr(plan_dev),
                                        ctypes.byref(info), _ptr(o_lat), _ptr(lse), dims, _stream(stream)),
           "mla_decode_attn_noalloc")


def dims_of(spec) -> Dims:
    """Dims from an inputs.workloads.WorkloadSpec."""
    return Dims(spec.H, spec.Dn, spec.Dr, spec.Dv, spec.R, spec.page_size,
                MLA_BF16 if spec.dtype == "bf16" else MLA_F32)


def mla_quantize_rows_fp8(rows, codes, scales, n, dims, stream=None):
    _check(_lib.mla_quantize_rows_fp8(_ptr(rows), _ptr(codes), _ptr(scales), n, dims, _stream(stream)),
           "mla_quantize_rows_fp8")


def mla_cache_append_fp8(kv_codes, kv_scales, block_table, seq_lens, new_ckr, B, q_len, max_pages, num_pages, dims,
                         stream=None):
    _check(_lib.mla_cache_append_fp8(_ptr(kv_codes), _ptr(kv_scales), _ptr(block_table), _ptr(seq_lens),
                                     _ptr(new_ckr), B, q_len, max_pages, num_pages, dims, _stream(stream)),
           "mla_cache_append_fp8")


def mla_workspace_size_fp8(info, dims) -> int:
    return _lib.mla_workspace_size_fp8(ctypes.byref(info), dims)


def mla_decode_attn_fp8(q_lat, q_rope, kv_codes, kv_scales, block_table, seq_lens, B, q_len, max_pages, num_pages,
                        scale, plan_dev, info, o_lat, lse, workspace, workspace_bytes, dims, stream=None):
    _check(_lib.mla_decode_attn_fp8(_ptr(q_lat), _ptr(q_rope), _ptr(kv_codes), _ptr(kv_scales), _ptr(block_table),
                                    _ptr(seq_lens), B, q_len, max_pages, num_pages, scale, _ptr(plan_dev),
                                    ctypes.byref(info), _ptr(o_lat), _ptr(lse), _ptr(workspace), workspace_bytes,
                                    dims, _stream(stream)), "mla_decode_attn_fp8")


def mla_prefill_workspace_size(N, dims) -> int:
    return _lib.mla_prefill_workspace_size(N, dims)


def mla_prefill_attn(ckr, q_nope, q_rope, W_UK, W_UV, cu_seqlens, cu_seqlens_host, B, scale, out, workspace,
                     workspace_bytes, dims, stream=None):
    """cu_seqlens: device int32 [B+1]; cu_seqlens_host: the same as a host numpy int32 array."""
    host = np.ascontiguousarray(cu_seqlens_host, dtype=np.int32)
    _check(_lib.mla_prefill_attn(_ptr(ckr), _ptr(q_nope), _ptr(q_rope), _ptr(W_UK), _ptr(W_UV), _ptr(cu_seqlens),
                                 host.ctypes.data, B, scale, _ptr(out), _ptr(workspace), workspace_bytes, dims,
                                 _stream(stream)), "mla_prefill_attn")
