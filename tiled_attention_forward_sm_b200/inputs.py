"""Seeded synthetic inputs for the attention forward pass.

This module holds no attention arithmetic.  It only draws Q, K, V (and names
the workloads); the CUDA path and the CPU oracle both take their inputs from
here, so they see the same bf16 bits.

Recipe: ``torch.Generator('cpu').manual_seed(seed)``; draw fp32 ``randn`` for
Q, then K, then V, each [B, H, N, d]; multiply Q by ``q_std``; round to bf16
(round to nearest even, torch's cast).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One attention forward problem: shapes, mask, scale and input law."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    q_std: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Reported FLOPs: 4*B*H*N^2*d (two products of 2*N^2*d each per
        head), halved under the causal mask."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    @property
    def rows(self) -> int:
        return self.B * self.H * self.N


# The five workloads the attention forward is measured and checked on.
WORKLOADS = {
    w.name: w for w in [
        Workload("b1h2n256d64", 1, 2, 256, 64, False, 1.0, 1001),
        Workload("b4h16n2048d128_causal", 4, 16, 2048, 128, True, 1.0, 1002),
        Workload("b2h32n8192d128_causal", 2, 32, 8192, 128, True, 1.0, 1003),
        Workload("b8h16n4096d128_peaky", 8, 16, 4096, 128, False, 3.0, 1004),
        Workload("b1h16n32768d128_causal", 1, 16, 32768, 128, True, 1.0, 1005),
    ]
}

# The workload bench.py times by default: the largest causal d=128 case of
# the sequence-length range the throughput target is stated for (N >= 8192).
BENCH_WORKLOAD = "b2h32n8192d128_causal"


@dataclass(frozen=True)
class GeneralWorkload:
    """A problem for the general entry points: queries and keys of different
    lengths (a block of queries at the end of a key/value cache, the last
    query seeing the last key), shared K/V heads, split keys, or a packed
    batch of sequences of different lengths (``lens_q``/``lens_k``)."""
    name: str
    kind: str           # "chunk", "splitkv" or "varlen"
    B: int
    H: int
    H_kv: int
    N_q: int            # per sequence (varlen: the longest)
    N_k: int
    d: int
    causal: bool
    seed: int
    n_splits: int = 1
    lens_q: tuple = ()
    lens_k: tuple = ()

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def _varlen_lengths(n: int, lo: int, hi: int, seed: int):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


_LENS = _varlen_lengths(16, 512, 8192, 2103)

# Problems for the general entry points (parity tests and measurement).
GENERAL_WORKLOADS = {
    w.name: w for w in [
        # 512 new queries against a 16K-token cache, 4 query heads per K/V head
        GeneralWorkload("kvcache_b4h32kv8_q512_k16384_d128", "chunk", 4, 32, 8, 512, 16384,
                        128, True, 2101),
        # a 128-query block against a 32K-token cache: 64 items without
        # splitting the keys, 512 with 8 slices
        GeneralWorkload("kvcache_b2h32kv8_q128_k32768_d128_split8", "splitkv", 2, 32, 8, 128,
                        32768, 128, True, 2102, n_splits=8),
        GeneralWorkload("kvcache_b2h32kv8_q128_k32768_d128_split1", "splitkv", 2, 32, 8, 128,
                        32768, 128, True, 2102, n_splits=1),
        # 16 sequences of 512..8192 tokens (seeded), packed without padding
        GeneralWorkload("varlen_b16h16_d128_causal", "varlen", 16, 16, 16, max(_LENS),
                        max(_LENS), 128, True, 2103, lens_q=_LENS, lens_k=_LENS),
        # head dim 256 at the bench workload's shape (the d = 256 kernel), with
        # and without the mask
        GeneralWorkload("square_b2h32n8192d256_causal", "chunk", 2, 32, 32, 8192, 8192, 256,
                        True, 2104),
        GeneralWorkload("square_b2h32n8192d256", "chunk", 2, 32, 32, 8192, 8192, 256, False,
                        2105),
    ]
}


def make_general_inputs(w: GeneralWorkload):
    """bf16 CPU tensors for a general workload: per-head [B, H, N_q, d] and
    [B, H_kv, N_k, d], or packed [T_q, H, d] and [T_k, H_kv, d] for varlen
    (same draw order: Q, then K, then V)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    if w.kind == "varlen":
        tq, tk = sum(w.lens_q), sum(w.lens_k)
        q = torch.randn((tq, w.H, w.d), generator=g, dtype=torch.float32)
        k = torch.randn((tk, w.H_kv, w.d), generator=g, dtype=torch.float32)
        v = torch.randn((tk, w.H_kv, w.d), generator=g, dtype=torch.float32)
    else:
        q = torch.randn((w.B, w.H, w.N_q, w.d), generator=g, dtype=torch.float32)
        k = torch.randn((w.B, w.H_kv, w.N_k, w.d), generator=g, dtype=torch.float32)
        v = torch.randn((w.B, w.H_kv, w.N_k, w.d), generator=g, dtype=torch.float32)
    return tuple(t.to(torch.bfloat16).contiguous() for t in (q, k, v))


@dataclass(frozen=True)
class KMeansWorkload:
    """A k-means assignment problem: N points, K centroids, dimension d.
    Recipe: ``manual_seed(seed)``; centroids ~ N(0, 1) [K, d]; each point is
    a centroid drawn uniformly plus 0.5 N(0, 1) noise; both rounded to bf16."""
    name: str
    N: int
    K: int
    d: int
    seed: int

    @property
    def flops(self) -> float:
        """2*N*K*d: the point-centroid products (the distance matrix's cost)."""
        return 2.0 * self.N * self.K * self.d


KMEANS_WORKLOADS = {
    w.name: w for w in [
        # the configuration the Flash-KMeans item quotes
        KMeansWorkload("kmeans_n65536_k1024_d128", 65536, 1024, 128, 3101),
        # a larger assignment of the same shape of problem
        KMeansWorkload("kmeans_n1048576_k4096_d128", 1048576, 4096, 128, 3102),
    ]
}


def make_kmeans_inputs(w: KMeansWorkload):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    c = torch.randn((w.K, w.d), generator=g, dtype=torch.float32)
    pick = torch.randint(0, w.K, (w.N,), generator=g)
    x = c[pick] + 0.5 * torch.randn((w.N, w.d), generator=g, dtype=torch.float32)
    return x.to(torch.bfloat16).contiguous(), c.to(torch.bfloat16).contiguous()


def make_qkv(B: int, H: int, N: int, d: int, seed: int, q_std: float = 1.0):
    """Return bf16 CPU tensors (q, k, v), each [B, H, N, d], contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q = q * q_std
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def make_workload_inputs(w: Workload):
    return make_qkv(w.B, w.H, w.N, w.d, w.seed, w.q_std)


# The bf16 kernels' default lazy-rescale threshold (log2 units), mirrored
# from the kernel source (a CPU test checks the two agree).
DEFAULT_RESCALE_TAU = 12.0

# Score offsets of the rows of make_jump_qkv (in units of the raw dot
# product; with scale = ln 2 these are log2 units): the first jump lifts a
# row's largest score by the default threshold + 2 (the rescale is taken),
# by the threshold - 0.5 (just under it), or not at all.  All exact in bf16.
JUMP_OFFSETS = (DEFAULT_RESCALE_TAU + 2.0, DEFAULT_RESCALE_TAU - 0.5, 0.0)


def jump_offset_of_rows(N: int):
    """Offset c of every query row of make_jump_qkv: a mix inside each warp
    of 32 rows, except every fourth block of 32 rows, which holds one offset
    for all its rows (a warp where every lane, or none, takes the jump)."""
    import numpy as np
    i = np.arange(N)
    mixed = (7 * i + i // 32) % 3
    uniform = (i // 128) % 3
    pick = np.where((i // 32) % 4 == 3, uniform, mixed)
    return np.asarray(JUMP_OFFSETS)[pick]


def make_jump_qkv(B: int, H: int, N: int, d: int, jump_tile: int, second_jump: bool,
                  seed: int):
    """Inputs whose largest score per row jumps by a known amount at a known
    K/V tile (128 keys per tile), for checking a lazy rescale of the running
    maximum.  Every value is exact in bf16.

    Query row i is [1, c_i, r_i, 0, ...] with c_i from jump_offset_of_rows
    and r_i uniform in [-1, 1].  Key 0 (the anchor) is [2, 0, 0, ...]: raw
    score 2.  Key 128*jump_tile is [2, 1, 0, ...]: score 2 + c_i.  With
    second_jump, key 128*(jump_tile+1) is [2, 2, 0, ...]: score 2 + 2 c_i.
    Every other key is [u_j, 0, w_j, 0, ...] with u_j in [-1, 1] and w_j in
    [-1/4, 1/4]: scores in [-1.25, 1.25], below the anchor's.  V is N(0, 1).
    The row maximum is therefore 2 until the jump key, and 2 + c_i (then
    2 + 2 c_i) from it on, for every row that sees it."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.zeros(shape, dtype=torch.float32)
    k = torch.zeros(shape, dtype=torch.float32)
    c = torch.from_numpy(jump_offset_of_rows(N)).to(torch.float32)
    q[..., 0] = 1.0
    q[..., 1] = c
    q[..., 2] = torch.rand((B, H, N), generator=g) * 2 - 1
    k[..., 0] = torch.rand((B, H, N), generator=g) * 2 - 1
    k[..., 2] = (torch.rand((B, H, N), generator=g) * 2 - 1) * 0.25
    k[..., 0, :] = 0.0
    k[..., 0, 0] = 2.0
    jumps = [(jump_tile * 128, 1.0)]
    if second_jump:
        jumps.append(((jump_tile + 1) * 128, 2.0))
    for row, c1 in jumps:
        if row < N:
            k[..., row, :] = 0.0
            k[..., row, 0] = 2.0
            k[..., row, 1] = c1
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bit patterns (no copy of
    values, just a reinterpretation)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def sample_rows(w: Workload, n_random: int = 256, seed: int = 7):
    """Deterministic row sample (flat indices (b*H+h)*N + i) for checking a
    large workload: in every (b, h), the first and last 128 rows and both rows
    at every 4th 128-row tile boundary; plus ``n_random`` seeded random rows
    over the whole problem."""
    import numpy as np
    per_bh = set(range(min(128, w.N)))
    per_bh.update(range(max(0, w.N - 128), w.N))
    for t in range(0, w.N, 4 * 128):
        for i in (t - 1, t):
            if 0 <= i < w.N:
                per_bh.add(i)
    per_bh = np.array(sorted(per_bh), dtype=np.int64)
    rows = [bh * w.N + per_bh for bh in range(w.B * w.H)]
    rng = np.random.default_rng(seed)
    rows.append(rng.integers(0, w.rows, size=n_random, dtype=np.int64))
    return np.unique(np.concatenate(rows))
