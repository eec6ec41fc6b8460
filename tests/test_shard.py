"""Token-sharded decode, host side: two and three gloo ranks on CPU.

Each rank quantizes its own contiguous token range of one sequence with the oracle (its own key
calibration), computes the range's partial (M, L, o) at the range's absolute positions, and the
ranks exchange partials with the module's all-gather; the merged output must equal the oracle's
attention over the whole sequence (every rank's reconstruction, concatenated in order).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(w, T, lo, hi):
    import oracle as O
    import synth
    cbK = O.fit_codebook(synth.codebook_samples_k(w), w.f, w.bits)
    cbV = O.fit_codebook(synth.codebook_samples_v(w), w.f, w.bits)
    idx = (np.zeros((1, 1, 1, 1), dtype=np.int64), np.arange(lo, hi)[None, :, None, None],
           np.arange(w.Hkv)[None, None, :, None], np.arange(w.D)[None, None, None, :])
    K16, V16 = synth.gen_k(w, 0, *idx), synth.gen_v(w, 0, *idx)
    n = max(hi - lo, 1)
    c = O.QuantizedCache(1, w.Hkv, w.bits, n, w.f, 1 << 16, 1 << 16)
    if hi > lo:
        c.prefill(K16, V16, [hi - lo], cbK, cbV)
        return c.reconstruct(0, cbK, cbV)
    z = np.zeros((0, w.Hkv, w.D))
    return z, z


def _rank(rank, world, port, T, out):
    import datetime
    import torch
    import torch.distributed as dist
    import oracle as O
    import synth
    from long_context_decode_nuq_b200 import shard
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.workload("llama7b_layer_32k", Hq=4, Hkv=2)
        lo, hi = shard.token_ranges(T, world)[rank]
        Kx, Vx = _shard(w, T, lo, hi)
        q = synth.gen_q(w)[0]
        M, L, o = O.partial_attention(q, T, Kx, Vx, w.rope_theta, np.arange(lo, hi))
        ex = shard.PartialExchange(1, w.Hq, w.D, world, "cpu", dtype=torch.float64)
        ml_all, o_all = ex(torch.from_numpy(np.stack([M, L], -1)[None]),
                           torch.from_numpy(o[None]))
        merged = O.merge_partials(ml_all[:, 0, :, 0].numpy(), ml_all[:, 0, :, 1].numpy(),
                                  o_all[:, 0].numpy())
        out.put((rank, lo, hi, merged))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 700), (3, 500), (2, 40)])
def test_sharded_partials_merge_to_single_rank_attention(world, T):
    import oracle as O
    import synth
    from long_context_decode_nuq_b200 import shard
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, T, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(qq.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    ranges = [(lo, hi) for _, lo, hi, _ in res]
    assert ranges == shard.token_ranges(T, world)
    assert ranges[0][0] == 0 and ranges[-1][1] == T
    assert all(a[1] == b[0] for a, b in zip(ranges[:-1], ranges[1:]))   # contiguous, in order
    # the single-rank reference: the same per-range caches, one attention over all tokens
    w = synth.workload("llama7b_layer_32k", Hq=4, Hkv=2)
    shards = [_shard(w, T, lo, hi) for lo, hi in ranges]
    Kx = np.concatenate([s[0] for s in shards])
    Vx = np.concatenate([s[1] for s in shards])
    _, _, ref = O.decode_attention(synth.gen_q(w)[0], T, Kx, Vx, w.rope_theta)
    for _, _, _, merged in res:
        assert np.abs(merged - ref).max() < 1e-12   # every rank holds the same merged output


def test_token_ranges_and_append_rank():
    from long_context_decode_nuq_b200 import shard
    for T in (1, 63, 64, 1000, 1 << 20):
        for world in (1, 2, 3, 8):
            r = shard.token_ranges(T, world)
            assert len(r) == world and r[0][0] == 0 and r[-1][1] == T
            assert all(lo <= hi for lo, hi in r)
            assert all(lo % 64 == 0 for lo, hi in r if lo < T)
    assert shard.append_rank(8) == 7
