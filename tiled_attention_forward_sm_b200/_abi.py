"""ctypes binding of ``libattn_b200.so`` (see ``include/attn_b200.h``).

Argument marshalling only.  The library is loaded on first use; if it is
missing the call raises (run ``python -m tiled_attention_forward_sm_b200.build``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from .build import LIB

ATTN_OK = 0
_lib = None


class AttnOpts(ctypes.Structure):
    """Mirror of attn_opts in include/attn_b200.h."""
    _fields_ = [("exp2_poly_pairs", ctypes.c_int), ("kv_stages", ctypes.c_int),
                ("rescale_tau", ctypes.c_float)]

    def __init__(self, exp2_poly_pairs: int = -1, kv_stages: int = 0, rescale_tau: float = -1.0):
        super().__init__(exp2_poly_pairs, kv_stages, rescale_tau)


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


def library_path() -> str:
    return LIB


def library():
    """Load (once) and return the ctypes handle of the CUDA library."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(
                f"CUDA library {LIB} not built; run python -m tiled_attention_forward_sm_b200.build")
        _lib = configure(ctypes.CDLL(LIB))
    return _lib


def configure(lib):
    """Declare the C ABI's signatures on a ctypes handle of the library (or
    of one of its debugging builds, which export a subset of the entry
    points: a symbol a build does not export is left undeclared)."""
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sigs = {  # name: (return type, argument types)
        "attn_fwd": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]),
        "attn_fwd_ex": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, vp]),
        "attn_fwd_noalloc": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]),
        "attn_fwd_pair": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]),
        "attn_fwd_host": (i, [vp] * 10 + [i, i, i, i, i, f, vp]),
        "attn_selftest_wait_timeout": (i, [i, vp]),
        "attn_last_device_error": (i, [vp]),
        "attn_strerror": (ctypes.c_char_p, [i]),
        "attn_check_args": (i, [vp, vp, vp, vp, vp, i, i, i, i, f]),
        "attn_version": (i, []),
        "attn_release": (i, []),
        "attn_opts_default": (AttnOpts, []),
        "attn_fwd_chunk": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, vp]),
        "attn_fwd_varlen": (i, [vp] * 7 + [i] * 9 + [f, vp]),
        "attn_fwd_splitkv": (i, [vp] * 5 + [i] * 8 + [f, i, vp, vp, vp]),
        "attn_fwd_fp8": (i, [vp] * 5 + [i] * 5 + [f, f, f, f, vp]),
        "attn_quantize_e4m3": (i, [vp, vp, i, i, i, f, i, vp]),
        "attn_fwd_fp4": (i, [vp] * 8 + [i] * 5 + [f, f, f, f, vp]),
        "attn_quantize_nvfp4": (i, [vp, vp, vp, i, i, i, f, i, vp]),
        "attn_nvfp4_scale_bytes": (ctypes.c_longlong, [i, i]),
        "attn_kmeans_assign": (i, [vp, vp, vp, vp, vp, i, i, i, vp]),
        "attn_kmeans_workspace_floats": (ctypes.c_longlong, [i, i]),
        "attn_combine": (i, [vp, vp, i, ctypes.c_longlong, i, vp, vp, i, vp]),
    }
    for name, (restype, argtypes) in sigs.items():
        if hasattr(lib, name):
            fn = getattr(lib, name)
            fn.restype = restype
            fn.argtypes = argtypes
    return lib

def strerror(status: int) -> str:
    return library().attn_strerror(int(status)).decode()


def check_args(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int,
               B: int, H: int, N: int, d: int, scale: float) -> int:
    """The library's precondition check on raw pointer values (no CUDA call)."""
    return library().attn_check_args(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, scale)


def _stream_handle(stream, dev=None) -> int:
    """The raw handle of ``stream``; None means the current stream of ``dev``
    (or of the current device).  A torch stream of another device is
    refused: the kernel would run on one GPU against another's memory."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and isinstance(stream, torch.cuda.Stream) and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _device_of(*tensors) -> torch.device:
    """The one CUDA device every given tensor (None entries skipped) lives
    on.  Each call runs with that device current, so the library's
    tensor maps, launch and stream all refer to it."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"tensors must all be on one CUDA device, got {sorted(map(str, devs))}")
    dev = devs.pop()
    if dev.type != "cuda":
        raise ValueError(f"tensors must be CUDA tensors, got {dev}")
    return dev


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def attn_fwd_into(q, k, v, o, lse, causal: bool = False, scale: float | None = None,
                  stream=None, exp2_poly_pairs: int | None = None,
                  kv_stages: int | None = None, rescale_tau: float | None = None) -> None:
    """Enqueue the forward pass writing into ``o`` (bf16 [B,H,N,d]) and ``lse``
    (fp32 [B,H,N]).  Inputs: CUDA bf16 contiguous [B,H,N,d] tensors.
    ``exp2_poly_pairs`` (0..2), ``kv_stages`` (2..5 at d = 128) and
    ``rescale_tau`` (0..16, d <= 128) select the attn_fwd_ex tuning options."""
    B, H, N, d = _shape(q)
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16),
                        ("v", v, torch.bfloat16), ("o", o, torch.bfloat16)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {(B, H, N, d)}")
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() or \
            tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be a contiguous CUDA fp32 tensor of shape {(B, H, N)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            B, H, N, d, int(bool(causal)), float(scale))
    dev = _device_of(q, k, v, o, lse)
    if exp2_poly_pairs is None and kv_stages is None and rescale_tau is None:
        with torch.cuda.device(dev):
            rc = library().attn_fwd(*args, _stream_handle(stream, dev))
    else:
        opts = AttnOpts(-1 if exp2_poly_pairs is None else int(exp2_poly_pairs),
                        0 if kv_stages is None else int(kv_stages),
                        -1.0 if rescale_tau is None else float(rescale_tau))
        with torch.cuda.device(dev):
            rc = library().attn_fwd_ex(*args, ctypes.byref(opts), _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, stream=None,
             exp2_poly_pairs: int | None = None, kv_stages: int | None = None,
             rescale_tau: float | None = None):
    """Return ``(o, lse)`` for CUDA bf16 [B,H,N,d] inputs (enqueued on the
    current or given stream)."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd_into(q, k, v, o, lse, causal, scale, stream, exp2_poly_pairs, kv_stages, rescale_tau)
    return o, lse


def attn_fwd_noalloc_into(q, k, v, o, lse, causal: bool = False, scale: float | None = None,
                          stream=None) -> None:
    """The allocation-free entry point (see attn_fwd_noalloc in the header):
    same contract as attn_fwd_into; calls that overlap on the GPU race."""
    B, H, N, d = _shape(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or \
                tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {(B, H, N, d)}")
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() or \
            tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be a contiguous CUDA fp32 tensor of shape {(B, H, N)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = _device_of(q, k, v, o, lse)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                        _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_noalloc")


def attn_fwd_pair_into(q, k, v, o, lse, causal: bool = False, scale: float | None = None,
                       stream=None) -> None:
    """The CTA-pair kernel (attn_fwd_pair in the header: d = 128 only), with
    the contract of attn_fwd_into."""
    B, H, N, d = _shape(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or \
                tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {(B, H, N, d)}")
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() or \
            tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be a contiguous CUDA fp32 tensor of shape {(B, H, N)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = _device_of(q, k, v, o, lse)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_pair(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                     _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_pair")


def attn_fwd_pair(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Return ``(o, lse)`` from the CTA-pair kernel."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd_pair_into(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d,
                  causal: bool = False, scale: float | None = None, stream=None) -> None:
    """Forward pass on HOST tensors through the C ABI's host entry point:
    copies in, computes, copies out, and synchronises the stream.  The
    ``*_d`` tensors are the caller's device buffers of the same shapes."""
    B, H, N, d = _shape(q_h)
    for t in (q_h, k_h, v_h, o_h, lse_h):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = _device_of(q_d, k_d, v_d, o_d, lse_d)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_host(
            q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(), lse_h.data_ptr(),
            q_d.data_ptr(), k_d.data_ptr(), v_d.data_ptr(), o_d.data_ptr(), lse_d.data_ptr(),
            B, H, N, d, int(bool(causal)), float(scale), _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_host")


def selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test (see the header); the next
    last_device_error() should report the timeout status."""
    dev = _stream_device(stream)
    with torch.cuda.device(dev):
        rc = library().attn_selftest_wait_timeout(int(limit_us), _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_selftest_wait_timeout")


def _stream_device(stream) -> torch.device:
    """The device of a torch stream, else the current device."""
    if isinstance(stream, torch.cuda.Stream):
        return stream.device
    return torch.device("cuda", torch.cuda.current_device())


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word
    (of the stream's device, or of the current device)."""
    dev = _stream_device(stream)
    with torch.cuda.device(dev):
        return int(library().attn_last_device_error(_stream_handle(stream, dev)))


def _check(t, name, dtype, shape):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of shape {tuple(shape)}")


def attn_fwd_chunk_into(q, k, v, o, lse, causal: bool = False, causal_delta: int = 0,
                        scale: float | None = None, stream=None) -> None:
    """N_q queries against N_k keys per head (see attn_fwd_chunk in the
    header): q bf16 [B,H,N_q,d]; k, v bf16 [B,H_kv,N_k,d]; o [B,H,N_q,d] in
    bf16 or fp32 (fp32 keeps partial results exact for attn_combine); lse fp32
    [B,H,N_q].  Under ``causal`` key j is visible to query i iff
    j <= i + causal_delta."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    B, H, N_q, d = (int(x) for x in q.shape)
    _, H_kv, N_k, _ = (int(x) for x in k.shape)
    _check(q, "q", torch.bfloat16, (B, H, N_q, d))
    _check(k, "k", torch.bfloat16, (B, H_kv, N_k, d))
    _check(v, "v", torch.bfloat16, (B, H_kv, N_k, d))
    if o.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("o must be bf16 or fp32")
    _check(o, "o", o.dtype, (B, H, N_q, d))
    _check(lse, "lse", torch.float32, (B, H, N_q))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = _device_of(q, k, v, o, lse)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_chunk(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), B, H, H_kv, N_q, N_k, d, int(bool(causal)),
                                      int(causal_delta), float(scale),
                                      int(o.dtype == torch.float32), _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_chunk")


def attn_fwd_chunk(q, k, v, causal: bool = False, causal_delta: int = 0,
                   scale: float | None = None, out_dtype=torch.bfloat16, stream=None):
    """Return ``(o, lse)`` of attn_fwd_chunk_into."""
    B, H, N_q, d = (int(x) for x in q.shape)
    o = torch.empty((B, H, N_q, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    attn_fwd_chunk_into(q, k, v, o, lse, causal, causal_delta, scale, stream)
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    causal: bool = False, scale: float | None = None, stream=None):
    """Packed variable-length batch (see attn_fwd_varlen in the header):
    q bf16 [T_q, H, d]; k, v bf16 [T_k, H_kv, d]; cu_seqlens_* CUDA int32
    [B+1].  Returns o bf16 [T_q, H, d] and lse fp32 [H, T_q]."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q, k, v must be [tokens, heads, d]")
    T_q, H, d = (int(x) for x in q.shape)
    T_k, H_kv, _ = (int(x) for x in k.shape)
    _check(q, "q", torch.bfloat16, (T_q, H, d))
    _check(k, "k", torch.bfloat16, (T_k, H_kv, d))
    _check(v, "v", torch.bfloat16, (T_k, H_kv, d))
    B = int(cu_seqlens_q.shape[0]) - 1
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, (B + 1,))
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, (B + 1,))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((H, T_q), dtype=torch.float32, device=q.device)
    dev = _device_of(q, k, v, cu_seqlens_q, cu_seqlens_k)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       lse.data_ptr(), cu_seqlens_q.data_ptr(),
                                       cu_seqlens_k.data_ptr(), B, H, H_kv, int(max_seqlen_q),
                                       int(max_seqlen_k), T_q, T_k, d, int(bool(causal)),
                                       float(scale), _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_varlen")
    return o, lse


def splitkv_slices(N: int, n_splits: int) -> int:
    """Key slices attn_fwd_splitkv actually uses for N keys (every slice
    holds keys)."""
    tiles = (int(N) + 127) // 128
    per = (tiles + int(n_splits) - 1) // int(n_splits)
    return (tiles + per - 1) // per


def attn_fwd_splitkv(q, k, v, n_splits: int, causal: bool = False, causal_delta: int = 0,
                     scale: float | None = None, stream=None):
    """attn_fwd_chunk (bf16 O) with each head's keys cut into ``n_splits``
    slices that run as separate work items and are merged by the LSE combine
    kernel (see the header).  q bf16 [B,H,N_q,d]; k, v bf16 [B,H_kv,N_k,d].
    The fp32 scratch is allocated here from torch's allocator."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    B, H, N_q, d = (int(x) for x in q.shape)
    _, H_kv, N_k, _ = (int(x) for x in k.shape)
    _check(q, "q", torch.bfloat16, (B, H, N_q, d))
    _check(k, "k", torch.bfloat16, (B, H_kv, N_k, d))
    _check(v, "v", torch.bfloat16, (B, H_kv, N_k, d))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    used = splitkv_slices(N_k, n_splits) if n_splits >= 1 else 0
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    if used > 1:
        ws_o = torch.empty((used, B * H * N_q, d), dtype=torch.float32, device=q.device)
        ws_l = torch.empty((used, B * H * N_q), dtype=torch.float32, device=q.device)
        wp = (ws_o.data_ptr(), ws_l.data_ptr())
    else:
        wp = (None, None)
    dev = _device_of(q, k, v)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), B, H, H_kv, N_q, N_k, d, int(bool(causal)),
                                        int(causal_delta), float(scale), int(n_splits), wp[0], wp[1],
                                        _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_splitkv")
    return o, lse


def attn_combine(o_parts, lse_parts, out_dtype=torch.bfloat16, stream=None):
    """LSE merge of partial results (see attn_combine in the header):
    o_parts fp32 [G, ..., d], lse_parts fp32 [G, ...] with matching leading
    shapes.  Returns (o [..., d] in ``out_dtype``, lse fp32 [...])."""
    if o_parts.dim() < 2 or tuple(o_parts.shape[:-1]) != tuple(lse_parts.shape):
        raise ValueError("o_parts must be [G, ..., d] and lse_parts [G, ...]")
    G, d = int(o_parts.shape[0]), int(o_parts.shape[-1])
    rows = int(lse_parts[0].numel())
    _check(o_parts, "o_parts", torch.float32, o_parts.shape)
    _check(lse_parts, "lse_parts", torch.float32, lse_parts.shape)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bf16 or fp32")
    o = torch.empty(tuple(o_parts.shape[1:]), dtype=out_dtype, device=o_parts.device)
    lse = torch.empty(tuple(lse_parts.shape[1:]), dtype=torch.float32, device=o_parts.device)
    dev = _device_of(o_parts, lse_parts)
    with torch.cuda.device(dev):
        rc = library().attn_combine(o_parts.data_ptr(), lse_parts.data_ptr(), G, rows, d,
                                    o.data_ptr(), lse.data_ptr(), int(out_dtype == torch.float32),
                                    _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_combine")
    return o, lse


def kmeans_assign(x, centroids, with_best: bool = True, stream=None):
    """k-means assignment (see attn_kmeans_assign in the header): x bf16
    [N, d], centroids bf16 [K, d] on the GPU.  Returns (assign int32 [N],
    best fp32 [N] or None)."""
    if x.dim() != 2 or centroids.dim() != 2 or x.shape[1] != centroids.shape[1]:
        raise ValueError("x must be [N, d] and centroids [K, d]")
    N, d = (int(v) for v in x.shape)
    K = int(centroids.shape[0])
    _check(x, "x", torch.bfloat16, (N, d))
    _check(centroids, "centroids", torch.bfloat16, (K, d))
    lib = library()
    n_ws = int(lib.attn_kmeans_workspace_floats(N, K))
    if n_ws < 0:
        raise ValueError("bad sizes")
    ws = torch.empty(n_ws, dtype=torch.float32, device=x.device)
    assign = torch.empty(N, dtype=torch.int32, device=x.device)
    best = torch.empty(N, dtype=torch.float32, device=x.device) if with_best else None
    dev = _device_of(x, centroids)
    with torch.cuda.device(dev):
        rc = lib.attn_kmeans_assign(x.data_ptr(), centroids.data_ptr(), ws.data_ptr(),
                                    assign.data_ptr(), best.data_ptr() if with_best else None,
                                    N, K, d, _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_kmeans_assign")
    return assign, best


def attn_fwd_fp8(q, k, vt, causal: bool = False, scale: float | None = None,
                 q_descale: float = 1.0, k_descale: float = 1.0, v_descale: float = 1.0,
                 stream=None):
    """FP8 attention (see attn_fwd_fp8 in the header): q, k E4M3 [B,H,N,128]
    and vt E4M3 [B,H,128,N] (V transposed) on the GPU, as float8_e4m3fn or
    uint8 tensors.  Returns (o bf16 [B,H,N,128], lse fp32 [B,H,N])."""
    B, H, N, d = (int(x) for x in q.shape)
    for name, t, shape in (("q", q, (B, H, N, d)), ("k", k, (B, H, N, d)),
                           ("vt", vt, (B, H, d, N))):
        if t.element_size() != 1:
            raise ValueError(f"{name} must hold 8-bit values")
        _check(t, name, t.dtype, shape)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dev = _device_of(q, k, vt)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_fp8(q.data_ptr(), k.data_ptr(), vt.data_ptr(), o.data_ptr(),
                                    lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                    float(q_descale), float(k_descale), float(v_descale),
                                    _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_fp8")
    return o, lse


def quantize_e4m3(x, inv_descale: float = 1.0, transpose: bool = False, stream=None):
    """bf16 [B, H, N, d] (or [rows, d]) -> E4M3 bytes (uint8) of x * inv_descale, in the
    same layout or, with ``transpose``, as [B, H, d, N] (see attn_quantize_e4m3)."""
    if x.dim() == 2:
        BH, N, d = 1, int(x.shape[0]), int(x.shape[1])
        out_shape = (d, N) if transpose else (N, d)
    elif x.dim() == 4:
        B, H, N, d = (int(v) for v in x.shape)
        BH = B * H
        out_shape = (B, H, d, N) if transpose else (B, H, N, d)
    else:
        raise ValueError("x must be [rows, d] or [B, H, N, d]")
    _check(x, "x", torch.bfloat16, x.shape)
    out = torch.empty(out_shape, dtype=torch.uint8, device=x.device)
    dev = _device_of(x)
    with torch.cuda.device(dev):
        rc = library().attn_quantize_e4m3(x.data_ptr(), out.data_ptr(), BH, N, d,
                                          float(inv_descale), int(bool(transpose)),
                                          _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_quantize_e4m3")
    return out


def quantize_nvfp4(x, inv_descale: float = 1.0, transpose: bool = False, stream=None):
    """bf16 [B, H, N, 128] -> NVFP4 (see attn_quantize_nvfp4): returns
    (codes uint8 [B, H, N, 64], or [B, H, 128, N // 2] with ``transpose``,
    scales uint8 [B * H, ceil(N / 128), 2, 512])."""
    if x.dim() != 4:
        raise ValueError("x must be [B, H, N, d]")
    B, H, N, d = (int(v) for v in x.shape)
    _check(x, "x", torch.bfloat16, x.shape)
    codes = torch.empty((B, H, d, N // 2) if transpose else (B, H, N, d // 2), dtype=torch.uint8,
                        device=x.device)
    scales = torch.empty((B * H, (N + 127) // 128, 2, 512), dtype=torch.uint8, device=x.device)
    dev = _device_of(x)
    with torch.cuda.device(dev):
        rc = library().attn_quantize_nvfp4(x.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                           B * H, N, d, float(inv_descale), int(bool(transpose)),
                                           _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_quantize_nvfp4")
    return codes, scales


def attn_fwd_fp4(q, q_sf, k, k_sf, vt, vt_sf, causal: bool = False, scale: float | None = None,
                 q_descale: float = 1.0, k_descale: float = 1.0, v_descale: float = 1.0,
                 stream=None):
    """4-bit attention (see attn_fwd_fp4 in the header) on the outputs of
    quantize_nvfp4: q, k codes [B, H, N, 64], vt codes [B, H, 128, N // 2],
    and their scales.  Returns (o bf16 [B, H, N, 128], lse fp32 [B, H, N])."""
    B, H, N, half = (int(v) for v in q.shape)
    d = 2 * half
    for name, t, shape in (("q", q, (B, H, N, half)), ("k", k, (B, H, N, half)),
                           ("vt", vt, (B, H, d, N // 2))):
        _check(t, name, torch.uint8, shape)
    for name, t in (("q_sf", q_sf), ("k_sf", k_sf), ("vt_sf", vt_sf)):
        _check(t, name, torch.uint8, (B * H, (N + 127) // 128, 2, 512))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dev = _device_of(q, q_sf, k, k_sf, vt, vt_sf)
    with torch.cuda.device(dev):
        rc = library().attn_fwd_fp4(q.data_ptr(), q_sf.data_ptr(), k.data_ptr(), k_sf.data_ptr(),
                                    vt.data_ptr(), vt_sf.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    B, H, N, d, int(bool(causal)), float(scale), float(q_descale),
                                    float(k_descale), float(v_descale),
                                    _stream_handle(stream, dev))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_fp4")
    return o, lse
