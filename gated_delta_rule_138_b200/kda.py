"""Thin ctypes binding of libkda.so (include/kda.h), same entry-point names.

Argument marshalling only: shapes and dtypes are read off torch tensors, the
device pointers and the current CUDA stream are passed to the C ABI, and a
non-OK status raises KdaError.  Every step of the computation runs in the
library's CUDA kernels; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libkda.so"

KDA_F32, KDA_BF16 = 0, 1
_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
           3: "KDA_ERR_CUDA", 4: "KDA_ERR_DEVICE_TIMEOUT"}


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = "%s failed: %s" % (fn, _STATUS.get(status, "status %d" % status))
        if detail:
            msg += " (%s)" % detail
        super().__init__(msg)


_lib = None


def library_path() -> str:
    return os.path.join(HERE, _LIB_NAME)


def load_library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libkda.so, building it first if it is absent and nvcc is present.

    Raises KdaError if the library cannot be found or built: there is no
    non-CUDA path.
    """
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if build_if_missing:
        try:
            from . import build as _build
            path = _build.build()
        except (OSError, FileNotFoundError) as exc:
            if not os.path.exists(path):
                raise KdaError("load_library", -1, "libkda.so missing and not buildable: %s" % exc)
    if not os.path.exists(path):
        raise KdaError("load_library", -1, "libkda.so not found at %s" % path)
    lib = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.kda_forward.restype = ctypes.c_int
    lib.kda_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp,
                                i32, i64, i32, i32, i32, i32, ctypes.c_int, ctypes.c_int, vp]
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                    ctypes.c_int, ctypes.c_int, vp]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_forward_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_forward_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32]
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_last_error.argtypes = []
    lib.kda_forward_kernel_name.restype = ctypes.c_char_p
    lib.kda_forward_kernel_name.argtypes = [i32, i32, i32, ctypes.c_int, ctypes.c_int]
    lib.kda_launch_count.restype = ctypes.c_uint64
    lib.kda_launch_count.argtypes = []
    lib.kda_device_status.restype = ctypes.c_int
    lib.kda_device_status.argtypes = [vp]
    lib.kda_segment_maps.restype = ctypes.c_int
    lib.kda_segment_maps.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i64, i32, i32, i32, i32,
                                     ctypes.c_int, vp]
    lib.kda_segment_scan.restype = ctypes.c_int
    lib.kda_segment_scan.argtypes = [vp, vp, i32, vp, i32, i32, i32, i32, vp]
    lib.kda_forward_segments.restype = i32
    lib.kda_forward_segments.argtypes = [i32, i64, i32, i32]
    lib.kda_release_workspace.restype = ctypes.c_int
    lib.kda_release_workspace.argtypes = []
    lib.kda_selftest_timeout.restype = ctypes.c_int
    lib.kda_selftest_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.kda_forward_noalloc.restype = ctypes.c_int
    lib.kda_forward_noalloc.argtypes = lib.kda_forward.argtypes
    lib.kda_noalloc_status.restype = ctypes.c_int
    lib.kda_noalloc_status.argtypes = [i32, vp, vp]
    lib.kda_noalloc_selftest_timeout.restype = ctypes.c_int
    lib.kda_noalloc_selftest_timeout.argtypes = [ctypes.c_uint64, i32, vp]
    lib.kda_forward_fused.restype = ctypes.c_int
    lib.kda_forward_fused.argtypes = lib.kda_forward.argtypes
    lib.kda_decode_step_fused.restype = ctypes.c_int
    lib.kda_decode_step_fused.argtypes = lib.kda_decode_step.argtypes
    lib.kda_forward_indexed.restype = ctypes.c_int
    lib.kda_forward_indexed.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp,
                                        i32, i64, i32, i32, i32, i32, ctypes.c_int, ctypes.c_int, vp]
    lib.kda_decode_step_indexed.restype = ctypes.c_int
    lib.kda_decode_step_indexed.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                            ctypes.c_int, ctypes.c_int, vp]
    lib.kda_backward.restype = ctypes.c_int
    lib.kda_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                 i32, i64, i32, i32, i32, ctypes.c_int, vp, ctypes.c_size_t, vp]
    lib.kda_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_backward_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32, i32]
    _lib = lib
    return lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError("unsupported dtype %s (fp32 or bf16)" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        lib = load_library(False)
        raise KdaError(fn, status, lib.kda_last_error().decode())


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_forward_workspace_bytes(B: int, T: int, H: int, d_k: int, d_v: int, chunk: int = 64) -> int:
    return int(load_library().kda_forward_workspace_bytes(B, T, H, d_k, d_v, chunk))


def kda_forward_kernel_name(d_k: int, d_v: int, chunk: int, in_dtype: torch.dtype,
                            out_dtype: Optional[torch.dtype] = None) -> Optional[str]:
    """Kernel kda_forward would run for these sizes and dtypes (None = rejected)."""
    code = lambda d: KDA_F32 if d == torch.float32 else KDA_BF16
    r = load_library().kda_forward_kernel_name(d_k, d_v, chunk, code(in_dtype),
                                                code(out_dtype or in_dtype))
    return None if r is None else r.decode()


def kda_device_status(stream=None) -> None:
    """Synchronise `stream` and raise KdaError if a kernel reported a device timeout."""
    _check("kda_device_status", load_library().kda_device_status(_stream(stream)))


def kda_forward_segments(num_seqs: int, tokens_per_seq: int, H: int, num_sms: int = 0) -> int:
    """Time segments per sequence the tensor-core forward uses (1 = unsplit)."""
    return int(load_library().kda_forward_segments(num_seqs, tokens_per_seq, H, num_sms))


def kda_release_workspace() -> None:
    """Hand back the device memory the current device's split-forward workspace
    pool keeps between calls."""
    _check("kda_release_workspace", load_library().kda_release_workspace())


def kda_selftest_timeout(limit_ns: int = 1_000_000, stream=None) -> None:
    """Launch a wait that must time out (nothing arrives) and record it; check
    it with kda_device_status()."""
    _check("kda_selftest_timeout", load_library().kda_selftest_timeout(int(limit_ns), _stream(stream)))


def kda_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load_library().kda_launch_count())


def _contig(name, t):
    if t is not None and not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def kda_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                beta: torch.Tensor, S0: Optional[torch.Tensor] = None,
                cu_seqlens: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                S_final: Optional[torch.Tensor] = None, chunk: int = 64,
                out_dtype: Optional[torch.dtype] = None, want_state: bool = True,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """KDA forward (chunk-parallel) through the C ABI.

    q, k, alpha [B, T, H, d_k]; v [B, T, H, d_v]; beta [B, T, H] (fp32 or bf16,
    one dtype); S0 fp32 [N, H, d_k, d_v] or None; cu_seqlens int32 [N + 1] or
    None (packed batch, B == 1).  Returns (out [B, T, H, d_v], S_final or None).
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or alpha.shape != q.shape or v.shape != (B, T, H, dv) \
            or beta.shape != (B, T, H):
        raise ValueError("inconsistent shapes")
    dts = {q.dtype, k.dtype, v.dtype, alpha.dtype, beta.dtype}
    if len(dts) != 1:
        raise TypeError("q, k, v, alpha, beta must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("S0", S0), ("cu_seqlens", cu_seqlens)):
        _contig(name, t)
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if S0 is not None and (S0.dtype != torch.float32 or tuple(S0.shape) != (nseq, H, dk, dv)):
        raise ValueError("S0 must be fp32 [N, H, d_k, d_v]")
    od = out_dtype or q.dtype
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=od, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty(nseq, H, dk, dv, dtype=torch.float32, device=q.device)
    st = lib.kda_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                         _ptr(cu_seqlens), int(nseq), _ptr(out), _ptr(S_final),
                         int(B), int(T), int(H), int(dk), int(dv), int(chunk),
                         _dt(q), _dt(out), _stream(stream))
    _check("kda_forward", st)
    return out, S_final


def kda_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                 beta: torch.Tensor, dout: torch.Tensor, S0: Optional[torch.Tensor] = None,
                 dS_final: Optional[torch.Tensor] = None,
                 cu_seqlens: Optional[torch.Tensor] = None, want_dS0: bool = True,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients of kda_forward through the C ABI (kda_backward).

    Inputs as kda_forward plus dout (dL/d out, [B, T, H, d_v], the inputs' dtype)
    and dS_final (dL/d S_final, fp32 [N, H, d_k, d_v], or None for zero).
    Returns fp32 (dq, dk, dv, dalpha, dbeta, dS0 or None), shaped like the inputs.
    workspace: optional uint8 device tensor of at least kda_backward_workspace_bytes.
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or alpha.shape != q.shape or v.shape != (B, T, H, dv) \
            or beta.shape != (B, T, H) or dout.shape != v.shape:
        raise ValueError("inconsistent shapes")
    if len({q.dtype, k.dtype, v.dtype, alpha.dtype, beta.dtype, dout.dtype}) != 1:
        raise TypeError("q, k, v, alpha, beta, dout must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("dout", dout), ("S0", S0), ("dS_final", dS_final),
                    ("cu_seqlens", cu_seqlens), ("workspace", workspace)):
        _contig(name, t)
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    for name, t in (("S0", S0), ("dS_final", dS_final)):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (nseq, H, dk, dv)):
            raise ValueError("%s must be fp32 [N, H, d_k, d_v]" % name)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk_, dal = (torch.empty(B, T, H, dk, **f32) for _ in range(3))
    dv_ = torch.empty(B, T, H, dv, **f32)
    dbe = torch.empty(B, T, H, **f32)
    dS0 = torch.empty(nseq, H, dk, dv, **f32) if want_dS0 else None
    st = lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                          _ptr(dout), _ptr(dS_final), _ptr(cu_seqlens), int(nseq), _ptr(dq),
                          _ptr(dk_), _ptr(dv_), _ptr(dal), _ptr(dbe), _ptr(dS0), int(B), int(T),
                          int(H), int(dk), int(dv), _dt(q), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check("kda_backward", st)
    return dq, dk_, dv_, dal, dbe, dS0


def kda_backward_workspace_bytes(B: int, T: int, H: int, d_k: int, d_v: int,
                                 num_seqs: Optional[int] = None) -> int:
    """Bytes of workspace kda_backward needs (num_seqs given: a packed batch)."""
    lib = load_library()
    packed = num_seqs is not None
    return int(lib.kda_backward_workspace_bytes(int(B), int(T), int(H), int(d_k), int(d_v),
                                                1 if packed else 0, int(num_seqs or 0)))


def kda_segment_maps(k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                     cu_seqlens: Optional[torch.Tensor] = None, maps: Optional[torch.Tensor] = None,
                     chunk: int = 64, stream=None) -> torch.Tensor:
    """Affine state map [M | N] (fp32 [N, H, d_k, d_k + d_v]) of every sequence's
    tokens: S_end = M S_start + N."""
    lib = load_library()
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    for name, t in (("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("cu_seqlens", cu_seqlens), ("maps", maps)):
        _contig(name, t)
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if maps is None:
        maps = torch.empty(nseq, H, dk, dk + dv, dtype=torch.float32, device=k.device)
    st = lib.kda_segment_maps(_ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(cu_seqlens),
                              int(nseq), _ptr(maps), int(B), int(T), int(H), int(dk), int(dv),
                              int(chunk), _dt(k), _stream(stream))
    _check("kda_segment_maps", st)
    return maps


def kda_segment_scan(maps: torch.Tensor, S0: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Apply stacked segment maps [G, N, H, d_k, d_k + d_v] in order to S0 (or 0)."""
    lib = load_library()
    G, N, H, dk, w = maps.shape
    dv = w - dk
    for name, t in (("maps", maps), ("S0", S0), ("out", out)):
        _contig(name, t)
    if out is None:
        out = torch.empty(N, H, dk, dv, dtype=torch.float32, device=maps.device)
    st = lib.kda_segment_scan(_ptr(S0), _ptr(maps), int(G), _ptr(out), int(N), int(H), int(dk),
                              int(dv), _stream(stream))
    _check("kda_segment_scan", st)
    return out


def kda_forward_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                        beta: torch.Tensor, out: torch.Tensor, S_final: Optional[torch.Tensor],
                        S0: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, chunk: int = 64,
                        stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_forward without device allocation (bf16, d = 128, chunk 64 only).

    The C entry point uses a fixed scratch array compiled into the library
    instead of allocating; the caller passes the output buffers, so this
    binding allocates nothing either.
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("S0", S0), ("cu_seqlens", cu_seqlens), ("out", out), ("S_final", S_final)):
        _contig(name, t)
    st = lib.kda_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                 _ptr(cu_seqlens), int(nseq), _ptr(out), _ptr(S_final),
                                 int(B), int(T), int(H), int(dk), int(dv), int(chunk),
                                 _dt(q), _dt(out), _stream(stream))
    _check("kda_forward_noalloc", st)
    return out, S_final


def kda_noalloc_status(num_words: int, stream=None, check: bool = True) -> list:
    """Synchronise `stream` and read the first num_words status words of
    kda_forward_noalloc's fixed array (word n * H + h of the last call: 0 =
    finished, 1 = that CTA's bounded wait gave up).  Raises KdaError
    (KDA_ERR_DEVICE_TIMEOUT) if any is set and `check`; returns the words."""
    words = (ctypes.c_int32 * max(int(num_words), 1))()
    st = load_library().kda_noalloc_status(int(num_words), ctypes.cast(words, ctypes.c_void_p),
                                           _stream(stream))
    if st not in (0, 4) or (st == 4 and check):
        _check("kda_noalloc_status", st)
    return list(words)[:int(num_words)]


def kda_noalloc_selftest_timeout(limit_ns: int, word: int, stream=None) -> None:
    """A bounded wait that must give up, reported in word `word` of the fixed array."""
    _check("kda_noalloc_selftest_timeout",
           load_library().kda_noalloc_selftest_timeout(int(limit_ns), int(word), _stream(stream)))


def kda_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                    beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                    out_dtype: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """One decode step through the C ABI; S (fp32 [N, H, d_k, d_v]) is updated in place.

    q, k, alpha [N, H, d_k]; v [N, H, d_v]; beta [N, H].  Returns out [N, H, d_v].
    """
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if S.dtype != torch.float32 or tuple(S.shape) != (N, H, dk, dv):
        raise ValueError("S must be fp32 [N, H, d_k, d_v]")
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta), ("S", S)):
        _contig(name, t)
    if out is None:
        out = torch.empty(N, H, dv, dtype=out_dtype or q.dtype, device=q.device)
    st = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S),
                             _ptr(out), int(N), int(H), int(dk), int(dv), _dt(q), _dt(out),
                             _stream(stream))
    _check("kda_decode_step", st)
    return out


def kda_forward_indexed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                        beta: torch.Tensor, S_pool: torch.Tensor, slots: torch.Tensor,
                        cu_seqlens: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, chunk: int = 64,
                        out_dtype: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """kda_forward from and into pooled states: sequence n starts from, and
    leaves its final state in, S_pool[slots[n]] (fp32 [P, H, d_k, d_v]; int32
    slots, a slot outside [0, P) = padding).  Returns out [B, T, H, d_v]."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("S_pool", S_pool), ("slots", slots), ("cu_seqlens", cu_seqlens)):
        _contig(name, t)
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if slots.dtype != torch.int32 or slots.numel() != nseq:
        raise ValueError("slots must be int32 [N]")
    if S_pool.dtype != torch.float32 or tuple(S_pool.shape[1:]) != (H, dk, dv):
        raise ValueError("S_pool must be fp32 [P, H, d_k, d_v]")
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=out_dtype or q.dtype, device=q.device)
    st = lib.kda_forward_indexed(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S_pool),
                                 int(S_pool.shape[0]), _ptr(slots), _ptr(cu_seqlens), int(nseq),
                                 _ptr(out), int(B), int(T), int(H), int(dk), int(dv), int(chunk),
                                 _dt(q), _dt(out), _stream(stream))
    _check("kda_forward_indexed", st)
    return out


def kda_decode_step_indexed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            alpha: torch.Tensor, beta: torch.Tensor, S_pool: torch.Tensor,
                            slots: torch.Tensor, out: Optional[torch.Tensor] = None,
                            out_dtype: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """One decode step with the state of sequence n at S_pool[slots[n]] (in place)."""
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("S_pool", S_pool), ("slots", slots)):
        _contig(name, t)
    if slots.dtype != torch.int32 or slots.numel() != N:
        raise ValueError("slots must be int32 [N]")
    if S_pool.dtype != torch.float32 or tuple(S_pool.shape[1:]) != (H, dk, dv):
        raise ValueError("S_pool must be fp32 [P, H, d_k, d_v]")
    if out is None:
        out = torch.empty(N, H, dv, dtype=out_dtype or q.dtype, device=q.device)
    st = lib.kda_decode_step_indexed(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                     _ptr(S_pool), int(S_pool.shape[0]), _ptr(slots), _ptr(out),
                                     int(N), int(H), int(dk), int(dv), _dt(q), _dt(out),
                                     _stream(stream))
    _check("kda_decode_step_indexed", st)
    return out


def kda_forward_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      alpha_logits: torch.Tensor, beta_logits: torch.Tensor,
                      S0: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                      chunk: int = 64, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_forward from raw inputs: alpha = 1/(1 + e^x), beta = sigmoid(y), q and k
    L2-normalised per (token, head) inside the kernel (bf16, d = 128)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha_logits", alpha_logits),
                    ("beta_logits", beta_logits), ("S0", S0), ("cu_seqlens", cu_seqlens)):
        _contig(name, t)
    nseq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if S_final is None:
        S_final = torch.empty(nseq, H, dk, dv, dtype=torch.float32, device=q.device)
    st = lib.kda_forward_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha_logits), _ptr(beta_logits),
                               _ptr(S0), _ptr(cu_seqlens), int(nseq), _ptr(out), _ptr(S_final),
                               int(B), int(T), int(H), int(dk), int(dv), int(chunk), _dt(q),
                               _dt(out), _stream(stream))
    _check("kda_forward_fused", st)
    return out, S_final


def kda_decode_step_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          alpha_logits: torch.Tensor, beta_logits: torch.Tensor, S: torch.Tensor,
                          out: Optional[torch.Tensor] = None,
                          out_dtype: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """kda_decode_step from raw inputs (see kda_forward_fused); S updated in place."""
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha_logits", alpha_logits),
                    ("beta_logits", beta_logits), ("S", S)):
        _contig(name, t)
    if out is None:
        out = torch.empty(N, H, dv, dtype=out_dtype or q.dtype, device=q.device)
    st = lib.kda_decode_step_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha_logits),
                                   _ptr(beta_logits), _ptr(S), _ptr(out), int(N), int(H), int(dk),
                                   int(dv), _dt(q), _dt(out), _stream(stream))
    _check("kda_decode_step_fused", st)
    return out
