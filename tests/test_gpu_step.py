"""Whole-model decode step as one CUDA graph (kvq_step_*): every launch gives the same bits as
the per-layer calls it records, leaves the caches bit-identical to theirs, and matches the
oracle's binary64 attention over the oracle's own cache.

Each case runs a few layers (different synthetic data per layer) through several graph
launches, with the packed input record taken from pageable host, pinned host and device
memory in turn.
"""
import numpy as np
import pytest

import oracle as O
import synth
from kvq_testlib import gpu_cache, gpu_quantize, host_block, oracle_codebooks, to_dev_codebook

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3
CACHE_FIELDS = ("kcodes", "vcodes", "kthr", "kparams", "vparams", "kout", "vout", "kchunk",
                "vchunk", "kcount", "vcount", "len", "status")

# (workload, overrides, prefill tokens, plen, layers, launches, n_new, fused, splits)
CASES = [
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 300, None, 3, 3, 1, 0, 0),
    ("batched_8x8k", dict(B=3, Hq=4, Hkv=4, bits=2), 260, [260, 64, 1], 2, 3, 1, 0, 2),
    ("llama3_8b_gqa_128k", dict(B=2, Hq=8, Hkv=2, bits=3), 333, [333, 100], 2, 3, 1, 0, 0),
    ("batched_8x8k", dict(B=2, Hq=4, Hkv=4, bits=4), 200, None, 2, 2, 1, 0, 0),
    # more tokens per launch than the single-launch append takes: the general append path
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 256, None, 2, 2, 20, 0, 0),
    # attention only (nothing appended)
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 300, None, 2, 2, 0, 0, 0),
    # the fused attention kernel inside the graph
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4, bits=3), 300, None, 2, 3, 1, 1, 0),
]


def _record(w, ks, vs, qs, qpos):
    """The packed input record: per layer k, v, q (fp16 bytes), then qpos int32 padded to 16."""
    parts = []
    for k, v, q in zip(ks, vs, qs):
        parts += [np.ascontiguousarray(k).view(np.uint8).ravel(),
                  np.ascontiguousarray(v).view(np.uint8).ravel(),
                  np.ascontiguousarray(q).view(np.uint8).ravel()]
    qp = np.zeros((w.B * 4 + 15) // 16 * 4, dtype=np.int32)
    qp[:w.B] = qpos
    parts.append(qp.view(np.uint8))
    return np.concatenate(parts)


@pytest.mark.parametrize("name,over,T,plen,layers,launches,n_new,fused,splits", CASES)
def test_step_graph(name, over, T, plen, layers, launches, n_new, fused, splits):
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload(name, **over)
    pl = plen if plen is not None else [T] * w.B
    T_cap = T + launches * n_new + 16
    cap = 1 << 16
    data, orc, gA, gB, cbs = [], [], [], [], []
    for l in range(layers):
        K16, V16 = host_block(w, T_cap, layer=l)
        cbK, cbV = oracle_codebooks(w, l)
        o = O.QuantizedCache(w.B, w.Hkv, w.bits, T_cap, w.f, cap, cap)
        o.prefill(K16[:, :T], V16[:, :T], pl, cbK, cbV)
        dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
        a, b = gpu_cache(w, T_cap, cap, cap), gpu_cache(w, T_cap, cap, cap)
        for g in (a, b):
            gpu_quantize(g, dK, dV, K16[:, :T], V16[:, :T], plen=plen, calibrate=1)
        data.append((K16, V16, cbK, cbV))
        orc.append(o)
        gA.append(a)
        gB.append(b)
        cbs.append((dK, dV))
    cfg = gA[0].cfg
    max_len = max(pl) + launches * n_new
    in_bytes = K.kvq_step_input_bytes(cfg, layers, n_new)
    d_in = torch.empty(in_bytes, dtype=torch.uint8, device="cuda")
    outA = torch.empty((layers, w.B, w.Hq, w.D), device="cuda")
    wsA = torch.empty(K.kvq_step_workspace(cfg, n_new, max_len, splits, fused),
                      dtype=torch.uint8, device="cuda")
    step = K.kvq_step_create(cfg, gA, [c[0] for c in cbs], [c[1] for c in cbs], n_new, max_len,
                             d_in, outA, wsA, splits, fused)
    aws = torch.empty(max(16, K.kvq_quantize_workspace(cfg, max(n_new, 1), 0)),
                      dtype=torch.uint8, device="cuda")
    dws_n = (K.kvq_decode_fused_workspace if fused else K.kvq_decode_workspace)(cfg, max_len,
                                                                                  splits)
    dws = torch.empty(dws_n, dtype=torch.uint8, device="cuda")
    outB = torch.empty_like(outA)
    try:
        for s in range(launches):
            lens = [int(o.len[b]) for b in range(w.B)]
            ks, vs, qs = [], [], []
            for l in range(layers):
                K16, V16 = data[l][0], data[l][1]
                ks.append(np.stack([K16[b, lens[b]:lens[b] + n_new] for b in range(w.B)]))
                vs.append(np.stack([V16[b, lens[b]:lens[b] + n_new] for b in range(w.B)]))
                qs.append(synth.gen_q(w, layer=l, step=s))
            qpos = np.array([lens[b] + n_new - 1 if n_new else lens[b] for b in range(w.B)],
                            dtype=np.int32)
            qpos = np.maximum(qpos, 0)
            rec = torch.from_numpy(_record(w, ks, vs, qs, qpos))
            assert rec.numel() == in_bytes
            kind = s % 3
            src = rec if kind == 0 else rec.pin_memory() if kind == 1 else rec.cuda()
            outA.fill_(float("nan"))
            K.kvq_step_launch(step, src)
            # the same calls one by one on the twin caches
            dq = torch.from_numpy(qpos).cuda()
            for l in range(layers):
                if n_new:
                    K.kvq_quantize_append(gB[l], cbs[l][0], cbs[l][1],
                                          torch.from_numpy(ks[l]).cuda(),
                                          torch.from_numpy(vs[l]).cuda(), n_new, None, 0, aws)
                fn = K.kvq_decode_attention_fused if fused else K.kvq_decode_attention
                fn(gB[l], cbs[l][0], cbs[l][1], torch.from_numpy(qs[l]).cuda(), dq, max_len,
                   outB[l], dws, splits)
            torch.cuda.synchronize()
            assert np.array_equal(outA.cpu().numpy().view(np.uint32),
                                  outB.cpu().numpy().view(np.uint32)), s
            # oracle: the same appends on its own cache, binary64 attention
            for l in range(layers):
                o = orc[l]
                if n_new:
                    o.append(ks[l], vs[l], data[l][2], data[l][3])
                oa = outA[l].cpu().numpy()
                for b in range(w.B):
                    if int(o.len[b]) == 0:
                        assert not np.any(oa[b])
                        continue
                    Kx, Vx = o.reconstruct(b, data[l][2], data[l][3])
                    ref = O.decode_attention(qs[l][b], int(qpos[b]), Kx, Vx, w.rope_theta)
                    err = np.abs(oa[b].astype(np.float64) - ref[2]).max()
                    assert err <= OUT_ATOL, (s, l, b, err)
        for l in range(layers):
            for f in CACHE_FIELDS:
                a = getattr(gA[l], f).cpu().numpy().view(np.uint8)
                b = getattr(gB[l], f).cpu().numpy().view(np.uint8)
                assert np.array_equal(a, b), (l, f)
            assert K.kvq_get_status(gA[l]) == 0
            assert list(gA[l].len.cpu().numpy()) == [int(x) for x in orc[l].len]
    finally:
        torch.cuda.synchronize()
        K.kvq_step_destroy(step)


def test_step_rejects_unsupported_fused_shape():
    """A fused step needs one query head per kv head: refused at create, nothing recorded."""
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload("llama3_8b_gqa_128k", B=1, Hq=8, Hkv=2, bits=3)
    g = gpu_cache(w, 256, 1024, 1024)
    lev = torch.zeros(8, device="cuda")
    cb = K.Codebook(lev, torch.zeros(7, device="cuda"))
    d_in = torch.empty(K.kvq_step_input_bytes(g.cfg, 1, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 1, 8, 128), device="cuda")
    ws = torch.empty(K.kvq_step_workspace(g.cfg, 1, 200), dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KvqError) as ei:
        K.kvq_step_create(g.cfg, [g], [cb], [cb], 1, 200, d_in, out, ws, 0, 1)
    assert ei.value.code == -4
