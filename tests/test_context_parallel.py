"""Context-parallel (ring) attention: the schedule, the ring over a real
process group (gloo ranks on the CPU, with the oracle standing in for the
per-pair attention and the merge), and the CUDA kernels' use of the
schedule on one GPU."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tiled_attention_forward_sm_b200 import context_parallel as cp
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv


def shard(t, rank, world, layout):
    """Rows of rank `rank` from a full [B, H, N, d] tensor."""
    n_local = t.shape[2] // world
    parts = [t[:, :, c.start:c.start + c.length] for c in cp.chunks_of(rank, world, n_local, layout)]
    return torch.cat(parts, dim=2).contiguous()


def unshard_rows(rank, world, n_local, layout):
    """Sequence positions of rank `rank`'s local rows, in local order."""
    return np.concatenate([np.arange(c.start, c.start + c.length)
                           for c in cp.chunks_of(rank, world, n_local, layout)])


# -------------------------------------------------------------- schedule ---
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world,n_local", [(1, 6), (2, 4), (3, 6), (4, 8)])
def test_schedule_covers_every_visible_pair_once(layout, causal, world, n_local):
    """Over all ring steps, each rank's tasks cover every (query, key)
    position pair its queries may see exactly once and no other pair."""
    N = world * n_local
    for rank in range(world):
        seen = np.zeros((N, N), dtype=np.int64)
        steps = cp.ring_schedule(rank, world, n_local, layout, causal)
        assert [s for s, _ in steps] == [(rank - t) % world for t in range(world)]
        for src, tasks in steps:
            src_chunks = cp.chunks_of(src, world, n_local, layout)
            for t in tasks:
                assert t.k in src_chunks
                for i in range(t.q.length):
                    for j in range(t.k.length):
                        if not t.causal or j <= i + t.delta:
                            seen[t.q.start + i, t.k.start + j] += 1
        for qpos in unshard_rows(rank, world, n_local, layout):
            want = np.zeros(N, dtype=np.int64)
            want[: (qpos + 1 if causal else N)] = 1
            np.testing.assert_array_equal(seen[qpos], want)


def test_zigzag_balances_causal_work():
    """Under the mask every rank computes the same number of visible pairs
    with the zigzag layout (and not with the contiguous one)."""
    world, n_local = 4, 16
    def work(layout):
        w = []
        for rank in range(world):
            tot = 0
            for _, tasks in cp.ring_schedule(rank, world, n_local, layout, True):
                for t in tasks:
                    i = np.arange(t.q.length)[:, None]
                    j = np.arange(t.k.length)[None, :]
                    tot += int(((j <= i + t.delta) if t.causal else np.ones_like(i + j)).sum())
            w.append(tot)
        return w
    assert len(set(work("zigzag"))) == 1
    assert len(set(work("contiguous"))) == world


# ---------------------------------------------- the ring over gloo ranks ---
def oracle_partial(q, k, v, causal, delta, scale):
    import oracle
    o, lse = oracle.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, delta, scale)
    return torch.from_numpy(o), torch.from_numpy(lse)


def oracle_merge(o_parts, lse_parts, out_dtype):
    import oracle
    G, d = o_parts.shape[0], o_parts.shape[-1]
    o, lse = oracle.lse_merge(o_parts.reshape(G, -1, d).numpy(), lse_parts.reshape(G, -1).numpy())
    return (torch.from_numpy(o).reshape(o_parts.shape[1:]),
            torch.from_numpy(lse).reshape(lse_parts.shape[1:]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ring_worker(rank, world, port, layout, causal, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, H, N, d = 1, 2, 16 * world, 8
        q, k, v = make_qkv(B, H, N, d, seed=600 + world)
        o, lse = cp.ring_attention(shard(q, rank, world, layout), shard(k, rank, world, layout),
                                   shard(v, rank, world, layout), causal=causal, scale=0.3,
                                   layout=layout, partial=oracle_partial, merge=oracle_merge)
        torch.save({"o": o.float(), "lse": lse}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("layout,causal", [("zigzag", True), ("contiguous", True),
                                           ("contiguous", False)])
def test_ring_attention_over_gloo_ranks(oracle_mod, tmp_path, world, layout, causal):
    """world gloo processes pass their K/V shards round the ring; each
    rank's merged result equals the oracle on the whole sequence for its
    rows (to the bf16 rounding of the stored O)."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, layout, causal, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a ring rank did not finish")
        assert p.exitcode == 0
    B, H, N, d = 1, 2, 16 * world, 8
    q, k, v = make_qkv(B, H, N, d, seed=600 + world)
    o_ref, l_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 0.3)
    for rank in range(world):
        got = torch.load(tmp_path / f"rank{rank}.pt")
        pos = unshard_rows(rank, world, N // world, layout)
        ref_o, ref_l = o_ref[:, :, pos], l_ref[:, :, pos]
        np.testing.assert_allclose(got["o"].numpy(), ref_o, rtol=2 ** -8, atol=1e-6)
        np.testing.assert_allclose(got["lse"].numpy(), ref_l, rtol=0, atol=1e-5)


# ---------------------------------------------- the CUDA path, one GPU ---
@pytest.mark.gpu
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_schedule_with_cuda_kernels(oracle_mod, layout, causal):
    """Four ranks' results computed on one GPU from all shards with the CUDA
    partial (attn_fwd_chunk, fp32 O) and merge (attn_combine) kernels, as
    ring_attention would on four GPUs, against the oracle on the whole
    sequence."""
    world, B, H, N, d = 4, 1, 4, 2048, 128
    q, k, v = make_qkv(B, H, N, d, seed=77)
    shards = [[shard(t, r, world, layout).cuda() for r in range(world)] for t in (q, k, v)]
    outs = cp.ring_attention_local(*shards, causal=causal, layout=layout)
    o_ref, l_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal,
                                       1 / math.sqrt(d))
    for rank, (o, lse) in enumerate(outs):
        pos = unshard_rows(rank, world, N // world, layout)
        err = np.abs(o.float().cpu().numpy() - o_ref[:, :, pos])
        assert (err <= 2e-2 + 1e-2 * np.abs(o_ref[:, :, pos])).all(), f"rank {rank}: {err.max()}"
        assert np.abs(lse.cpu().numpy() - l_ref[:, :, pos]).max() <= 1e-3
