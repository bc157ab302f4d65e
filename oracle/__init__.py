"""Oracle for the dense attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``tiled_attention_forward_sm_b200``) never imports it, and the two share
no code: no kernels, headers, helpers or constants.

Contents
--------
``attn_ref``            the plain fp64 definition (C, ``attn_ref.c``), see that
                        file's header for the formula and the pages it follows.
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
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_ref.c`` into ``libattn_ref.so`` beside it (gcc, OpenMP,
    -O2, no fast-math so exp/log keep their IEEE behaviour)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


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
                       tau: float = 8.0, round_p_bf16: bool = False):
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
    With ``round_p_bf16`` the weights are rounded to bf16 before the second
    product (what the kernel feeds its tensor cores); the row sum stays exact.
    """
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
        pv = _round_bf16(p) if round_p_bf16 else p
        acc = acc * alpha[:, None] + pv @ v[cols]
        m = m_used
    o = acc / l[:, None]
    lse = (m + np.log2(l)) / log2e
    return o, lse
