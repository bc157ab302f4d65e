"""Oracle for the dense attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``tiled_attention_forward_sm_b200``) never imports it, and the two share
no code: no kernels, headers, helpers or constants.

Contents
--------
``attn_ref``            the plain fp64 definition (C, ``attn_ref.c``), see that
                        file's header for the formula and the pages it follows.
``attn_ref_general``    the same definition for N_q queries against N_k keys,
                        K/V heads shared by groups of query heads, and a
                        causal offset (empty rows: O = 0, LSE = -inf).
``attn_ref_varlen``     ``attn_ref_general`` applied to each sequence of a
                        packed token-major batch.
``lse_merge``           the result against a union of disjoint key sets from
                        the results against each set.
``kmeans_assign``       the k-means assignment step: nearest centroid of each
                        point and its squared distance (``kmeans_ref.c``).
``tiled_online_model``  a second fp64 formulation that follows the pages'
                        tiled algorithm step by step (tiles of K/V, a running
                        maximum and running sum, lazy rescale).  It is used to
                        check, as statements, that tiling does not change the
                        result and that a conditional rescale keeps the sums
                        consistent.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants and brute force that do not go through this code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_ref.c")
_LIB = os.path.join(_HERE, "libattn_ref.so")
_KM_SRC = os.path.join(_HERE, "kmeans_ref.c")
_KM_LIB = os.path.join(_HERE, "libkmeans_ref.so")
_lib = None
_km_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_ref.c`` and ``kmeans_ref.c`` into shared libraries
    beside them (gcc, OpenMP, -O2, no fast-math so exp/log keep their IEEE
    behaviour)."""
    for src, lib in ((_SRC, _LIB), (_KM_SRC, _KM_LIB)):
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
            cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                   "-std=c11", src, "-o", lib, "-lm"]
            subprocess.check_call(cmd)
    return _LIB


def _load_kmeans():
    global _km_lib
    if _km_lib is None:
        build()
        lib = ctypes.CDLL(_KM_LIB)
        lib.kmeans_assign_f64.restype = ctypes.c_int
        lib.kmeans_assign_f64.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_int]
        _km_lib = lib
    return _km_lib


def kmeans_assign(x_bits, c_bits, rows=None, with_dist: bool = False, nthreads: int = 0):
    """k-means assignment in fp64 (``kmeans_ref.c``): for each point the
    nearest centroid (smallest index among equal distances) and that squared
    distance.  x_bits [N, d], c_bits [K, d]: uint16 bf16 bit patterns.
    Returns (assign int32 [n], best float64 [n]) and, with ``with_dist``,
    the distance rows float64 [n, K] too."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    c_bits = np.ascontiguousarray(c_bits, dtype=np.uint16)
    N, d = x_bits.shape
    K, dc = c_bits.shape
    if dc != d:
        raise ValueError("points and centroids disagree on d")
    if rows is None:
        n, rows_p, nrows = N, None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n, rows_p, nrows = rows.shape[0], rows.ctypes.data, rows.shape[0]
    assign = np.empty(n, dtype=np.int32)
    best = np.empty(n, dtype=np.float64)
    dist = np.empty((n, K), dtype=np.float64) if with_dist else None
    rc = _load_kmeans().kmeans_assign_f64(
        x_bits.ctypes.data, c_bits.ctypes.data, N, K, d, assign.ctypes.data, best.ctypes.data,
        dist.ctypes.data if with_dist else None, rows_p, nrows, int(nthreads))
    if rc != 0:
        raise ValueError("kmeans_assign_f64 rejected its arguments")
    return (assign, best, dist) if with_dist else (assign, best)


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.attn_ref_f64.restype = ctypes.c_int
        lib.attn_ref_f64.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int, ctypes.c_double, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int64]
        lib.attn_ref_general_f64.restype = ctypes.c_int
        lib.attn_ref_general_f64.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int64]
        lib.attn_ref_max_threads.restype = ctypes.c_int
        lib.attn_ref_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the C oracle's parallel loop uses by default."""
    return int(_load().attn_ref_max_threads())


def attn_ref(q_bits, k_bits, v_bits, causal: bool, scale: float,
             rows=None, nthreads: int = 0):
    """Plain fp64 attention forward on bf16 inputs.

    q_bits, k_bits, v_bits: numpy uint16 arrays [B, H, N, d] holding bf16 bit
    patterns (the exact values the GPU sees).  ``rows``: optional 1-D array of
    flat row indices ``(b*H + h)*N + i`` to compute; default all rows.

    Returns ``(o, lse)`` as float64: o is [B, H, N, d] (or [len(rows), d]) and
    lse is [B, H, N] (or [len(rows)]), natural log.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    if q_bits.ndim != 4 or q_bits.shape != k_bits.shape or q_bits.shape != v_bits.shape:
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = q_bits.shape
    if rows is None:
        o = np.empty((B, H, N, d), dtype=np.float64)
        lse = np.empty((B, H, N), dtype=np.float64)
        rows_p, nrows = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = rows.shape[0]
        o = np.empty((nrows, d), dtype=np.float64)
        lse = np.empty((nrows,), dtype=np.float64)
        rows_p = rows.ctypes.data
    rc = _load().attn_ref_f64(
        q_bits.ctypes.data, k_bits.ctypes.data, v_bits.ctypes.data,
        o.ctypes.data, lse.ctypes.data, B, H, N, d, int(bool(causal)),
        float(scale), int(nthreads), rows_p, nrows)
    if rc != 0:
        raise ValueError("attn_ref_f64 rejected its arguments")
    return o, lse


def attn_ref_general(q_bits, k_bits, v_bits, causal: bool, delta: int, scale: float,
                     rows=None, nthreads: int = 0):
    """Plain fp64 attention of N_q queries against N_k keys (``attn_ref.c``,
    ``attn_ref_general_f64``).

    q_bits: uint16 bf16 bits [B, H, N_q, d]; k_bits, v_bits: [B, H_kv, N_k, d]
    with H a multiple of H_kv (query head h reads K/V head h // (H // H_kv)).
    Under ``causal`` key j is visible to query i iff j <= i + delta; a query
    that sees no key gets O = 0 and LSE = -inf.  ``rows``: optional flat row
    indices ``(b*H + h)*N_q + i``.  Returns ``(o, lse)`` in float64 shaped
    like ``attn_ref``'s.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    if q_bits.ndim != 4 or k_bits.ndim != 4 or k_bits.shape != v_bits.shape:
        raise ValueError("q [B,H,N_q,d]; k, v one [B,H_kv,N_k,d] shape")
    B, H, N_q, d = q_bits.shape
    Bk, H_kv, N_k, dk = k_bits.shape
    if Bk != B or dk != d:
        raise ValueError("q and k/v disagree on B or d")
    if rows is None:
        o = np.empty((B, H, N_q, d), dtype=np.float64)
        lse = np.empty((B, H, N_q), dtype=np.float64)
        rows_p, nrows = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = rows.shape[0]
        o = np.empty((nrows, d), dtype=np.float64)
        lse = np.empty((nrows,), dtype=np.float64)
        rows_p = rows.ctypes.data
    rc = _load().attn_ref_general_f64(
        q_bits.ctypes.data, k_bits.ctypes.data, v_bits.ctypes.data,
        o.ctypes.data, lse.ctypes.data, B, H, H_kv, N_q, N_k, d, int(bool(causal)),
        int(delta), float(scale), int(nthreads), rows_p, nrows)
    if rc != 0:
        raise ValueError("attn_ref_general_f64 rejected its arguments")
    return o, lse


def attn_ref_varlen(q_bits, k_bits, v_bits, cu_q, cu_k, causal: bool, scale: float):
    """``attn_ref_general`` on each sequence of a packed batch.

    q_bits [T_q, H, d], k_bits and v_bits [T_k, H_kv, d] (uint16 bf16 bits);
    sequence b owns query tokens cu_q[b]..cu_q[b+1]-1 and key tokens
    cu_k[b]..cu_k[b+1]-1.  Under ``causal`` the last query of a sequence
    sees its last key (delta = len_k - len_q).  Returns o [T_q, H, d] and
    lse [H, T_q] in float64; tokens of a sequence with no keys get O = 0 and
    LSE = -inf.
    """
    q_bits = np.asarray(q_bits, dtype=np.uint16)
    k_bits = np.asarray(k_bits, dtype=np.uint16)
    v_bits = np.asarray(v_bits, dtype=np.uint16)
    T_q, H, d = q_bits.shape
    o = np.zeros((T_q, H, d), dtype=np.float64)
    lse = np.full((H, T_q), -np.inf, dtype=np.float64)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        qs = q_bits[q0:q1].transpose(1, 0, 2)[None]
        ks = k_bits[k0:k1].transpose(1, 0, 2)[None]
        vs = v_bits[k0:k1].transpose(1, 0, 2)[None]
        ob, lb = attn_ref_general(qs, ks, vs, causal, (k1 - k0) - (q1 - q0), scale)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def lse_merge(o_parts, lse_parts):
    """Result against a union of disjoint key sets from the results against
    each set, in fp64.

    Each part's O is its keys' exp-weighted sum of V divided by exp(LSE), so
    bringing the parts to one common scale (the rule page lecompute.fr/
    kernel-perf/flashattention-4-limites-calcul-matriciel states for old and
    new contributions, section "Deplacer une partie des exponentielles") and
    adding gives LSE = log sum_g exp(LSE_g) and O = sum_g exp(LSE_g - LSE) O_g.
    A part with LSE_g = -inf (no key) has weight 0; if every part has none,
    O = 0 and LSE = -inf.

    o_parts [G, rows, d], lse_parts [G, rows].  Returns (o [rows, d], lse [rows]).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe[None, :])            # 0 for parts with no key
    total = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, total)))
    wn = np.where(empty[None, :], 0.0, w / np.where(empty, 1.0, total)[None, :])
    o = np.einsum("gr,grd->rd", wn, o_parts)
    return o, lse


def e4m3_bits_to_f64(bits) -> np.ndarray:
    """Decode OCP FP8 E4M3 (``e4m3fn``) bit patterns: sign, 4 exponent bits
    with bias 7, 3 mantissa bits; exponent 0 is subnormal (2^-6 * m/8);
    S.1111.111 is NaN; there are no infinities."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def round_e4m3(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest E4M3 value (ties to even),
    saturating at +-448 (the largest finite value)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    # spacing of the binade holding a: 2^(max(e, -6) - 3)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    q = np.exp2(e - 3.0)
    r = np.round(a / q) * q          # numpy rounds halves to even
    return np.sign(x) * np.minimum(r, 448.0)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 bit patterns of float64 values that are already E4M3 values
    (e.g. ``round_e4m3``'s results): sign bit, then exponent and mantissa
    fields (subnormals for magnitudes below 2^-6; the sign of a zero is
    kept, -0 encodes as 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 7
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    normal = a >= 2.0 ** -6
    mant_n = np.round((a / np.exp2(e.astype(np.float64)) - 1.0) * 8).astype(np.int64)
    code_n = ((e + 7) << 3) | mant_n
    code_s = np.round(a / 2.0 ** -9).astype(np.int64)  # subnormal: m * 2^-9
    code = np.where(normal, code_n, code_s)
    code = np.where(a == 0, 0, code)
    return (code | sign).astype(np.uint8)


def quantize_e4m3(x_bits, inv_descale: float):
    """E4M3 codes of bf16 values times inv_descale, rounded to nearest even
    and saturated at +-448: the conversion the FP8 path's inputs go through."""
    return e4m3_encode(round_e4m3(bf16_bits_to_f64(x_bits) * float(inv_descale)))


# ---------------------------------------------------------------- FP4 ---
# The 4-bit path reads "FP4" as NVFP4: E2M1 elements (OCP microscaling
# element type: sign, 2 exponent bits with bias 1, 1 mantissa bit; values
# 0, 0.5, 1, 1.5, 2, 3, 4, 6) with one E4M3 scale per 16 consecutive
# elements along the products' reduction dimension, and a per-tensor fp32
# descale.  Page lecompute.fr/kernel-perf/flashattention-4-limites-calcul-
# matriciel, section "Le FP4 ajoute un compromis numerique": four-bit
# arithmetic, whose data preparation and conversion eat into the gain.

NVFP4_BLOCK = 16


def e2m1_bits_to_f64(codes) -> np.ndarray:
    """Decode 4-bit E2M1 codes (the low nibble of each byte): bit 3 sign,
    bits 2..1 exponent e (bias 1), bit 0 mantissa m; e = 0 is subnormal
    (m / 2), otherwise 2^(e - 1) (1 + m / 2).  No infinities or NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, np.exp2(e - 1.0) * (1.0 + m * 0.5))
    return sign * mag


def round_e2m1(x) -> np.ndarray:
    """Nearest E2M1 value of float64 inputs, ties to the even mantissa,
    saturating at +-6.  The representable magnitudes are multiples of 0.5
    below 2, of 1 in [2, 4) and of 2 in [4, 6]; inside each of those ranges
    an even multiple has an even mantissa, so rounding the multiple to even
    is rounding the mantissa to even."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    r = np.minimum(np.round(a / step) * step, 6.0)  # numpy rounds halves to even
    return np.where(np.signbit(x), -r, r)


def e2m1_encode(x) -> np.ndarray:
    """E2M1 codes (uint8, low nibble) of values that are already E2M1
    values; the sign of a zero is kept (-0 encodes as 0x8)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    table = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    idx = np.searchsorted(table, a)
    if not np.all(table[np.minimum(idx, 7)] == a):
        raise ValueError("e2m1_encode: value not representable in E2M1")
    return (idx | (np.signbit(x).astype(np.int64) << 3)).astype(np.uint8)


def nvfp4_quantize_f32(xf):
    """NVFP4 quantisation of float32 values along their last axis (a
    multiple of 16 long), with the steps taken in float32 as written:
    per block of 16, amax = max |x|; the scale is amax / 6 rounded to E4M3
    (nearest even, saturating at 448); each element is x * (1 / scale)
    (both roundings float32) rounded to E2M1 (nearest even, saturating at
    +-6); a block whose scale rounds to 0 stores zeros.  Returns (E2M1
    codes [..., n], E4M3 scale codes [..., n / 16])."""
    xf = np.asarray(xf, dtype=np.float32)
    n = xf.shape[-1]
    if n % NVFP4_BLOCK:
        raise ValueError("nvfp4: the quantised axis must be a multiple of 16")
    blk = xf.reshape(xf.shape[:-1] + (n // NVFP4_BLOCK, NVFP4_BLOCK))
    amax = np.abs(blk).max(axis=-1)
    s = round_e4m3((amax / np.float32(6.0)).astype(np.float32).astype(np.float64))
    s32 = s.astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(s32 > 0, np.float32(1.0) / np.where(s32 > 0, s32, np.float32(1.0)),
                       np.float32(0.0)).astype(np.float32)
    q = (blk * inv[..., None]).astype(np.float32)
    codes = e2m1_encode(round_e2m1(q.astype(np.float64)))
    return codes.reshape(xf.shape), e4m3_encode(s)


def quantize_nvfp4(x_bits, inv_descale: float):
    """NVFP4 codes of bf16 values times inv_descale (the product taken in
    float32), quantised along the last axis: the conversion the 4-bit
    path's inputs go through.  Returns (codes, scale codes)."""
    xf = (bf16_bits_to_f64(x_bits).astype(np.float32) * np.float32(inv_descale)).astype(np.float32)
    return nvfp4_quantize_f32(xf)


def nvfp4_to_f64(codes, scale_codes, descale: float = 1.0) -> np.ndarray:
    """Values of NVFP4 data: E2M1 value * its block's E4M3 scale * descale."""
    v = e2m1_bits_to_f64(codes)
    s = e4m3_bits_to_f64(scale_codes)
    n = v.shape[-1]
    v = v.reshape(v.shape[:-1] + (n // NVFP4_BLOCK, NVFP4_BLOCK)) * s[..., None]
    return v.reshape(v.shape[:-2] + (n,)) * float(descale)


def round_nvfp4_rows(p) -> np.ndarray:
    """Values of float64 rows after NVFP4 quantisation of each row along its
    last axis (a multiple of 16): the rounding the 4-bit path applies to the
    softmax weights before the second product."""
    codes, sc = nvfp4_quantize_f32(np.asarray(p, dtype=np.float64).astype(np.float32))
    return nvfp4_to_f64(codes, sc)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), returned as
    float64.  Goes through float32 first; the model uses it only to predict
    the size of the kernel's P-rounding error, never as a parity reference."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def tiled_online_model(q, k, v, causal: bool, scale: float, block_n: int = 128,
                       tau: float = 8.0, round_p_bf16: bool = False, round_p=None):
    """The pages' tiled algorithm for one (b, h) pair, in fp64.

    Follows page "lecompute.fr/kernel-perf/flashattention-4-limites-calcul-
    matriciel": K/V are visited tile by tile and O is accumulated (section
    "Entre deux multiplications il faut fabriquer les poids"); a common scale
    is kept between old and new contributions, and some rescalings are skipped
    under a condition (section "Deplacer une partie des exponentielles").  The
    condition read here: the running maximum (in log2 units) is raised only
    when a tile's maximum exceeds it by more than ``tau``; otherwise the old
    maximum is kept and the tile's weights may reach 2**tau.

    q, k, v: float64 [N, d].  Returns (o [N, d], lse [N]) in float64.
    With ``round_p_bf16`` (or ``round_p="bf16"``) the weights are rounded to
    bf16 before the second product (what the kernel feeds its tensor cores);
    ``round_p="e4m3"`` rounds them to FP8 E4M3 instead (the FP8 path), and
    ``round_p="nvfp4"`` to NVFP4 per row in blocks of 16 keys (the 4-bit
    path).  The row sum stays exact.
    """
    if round_p_bf16:
        round_p = "bf16"
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    log2e = 1.0 / np.log(2.0)
    m = np.full(N, -np.inf)           # running maximum, log2 units
    l = np.zeros(N)                   # running sum of weights (scaled by 2**-m)
    acc = np.zeros((N, d))            # running unnormalised output
    rows = np.arange(N)
    for j0 in range(0, N, block_n):
        cols = np.arange(j0, min(j0 + block_n, N))
        x = (q @ k[cols].T) * (scale * log2e)          # scores in log2 units
        if causal:
            x = np.where(cols[None, :] <= rows[:, None], x, -np.inf)
        tile_max = x.max(axis=1)
        new_m = np.maximum(m, tile_max)
        raise_m = (new_m - m) > tau                    # also true while m = -inf
        m_used = np.where(raise_m, new_m, m)
        alpha = np.where(raise_m, np.exp2(m - m_used), 1.0)
        alpha = np.where(np.isneginf(m), 0.0, alpha)
        with np.errstate(invalid="ignore"):
            p = np.exp2(x - m_used[:, None])
        p = np.where(np.isneginf(x), 0.0, p)
        l = l * alpha + p.sum(axis=1)
        if round_p == "bf16":
            pv = _round_bf16(p)
        elif round_p == "e4m3":
            pv = round_e4m3(p)
        elif round_p == "nvfp4":
            pad = (-len(cols)) % NVFP4_BLOCK  # a ragged last tile: zero keys
            pv = round_nvfp4_rows(np.pad(p, ((0, 0), (0, pad))))[:, : len(cols)]
        else:
            pv = p
        acc = acc * alpha[:, None] + pv @ v[cols]
        m = m_used
    o = acc / l[:, None]
    lse = (m + np.log2(l)) / log2e
    return o, lse
