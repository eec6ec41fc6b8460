"""GPU decode attention parity against the oracle's binary64 attention.

Tolerances (from the decode target): logits max_t |l - l_ref| <= 1e-3 * max(1, max_t |l_ref|),
outputs max |o - o_ref| <= 2e-3.
"""
import numpy as np
import pytest

import oracle as O
import synth
from kvq_testlib import gpu_cache, gpu_quantize, host_block, oracle_codebooks, to_dev_codebook

pytestmark = pytest.mark.gpu

LOGIT_RTOL = 1e-3
OUT_ATOL = 2e-3

CASES = [
    ("tiny_single_head", {}, 2048, None, 0),
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 700, None, 1),
    ("batched_8x8k", dict(B=3, Hq=4, Hkv=4, bits=2), 333, [333, 64, 1], 0),
    ("batched_8x8k", dict(B=2, Hq=4, Hkv=4, bits=4), 200, [200, 150], 0),
    ("llama3_8b_gqa_128k", dict(B=2, Hq=16, Hkv=4), 517, [517, 300], 0),
    ("llama7b_layer_32k", dict(Hq=32, Hkv=32), 260, None, 1),
    # four query heads over two kv heads per CTA; two query heads per CTA (shared / not)
    ("llama7b_layer_32k", dict(Hq=8, Hkv=4), 301, None, 1),
    ("llama3_8b_gqa_128k", dict(B=1, Hq=6, Hkv=3), 250, None, 0),
    ("llama3_8b_gqa_128k", dict(B=1, Hq=6, Hkv=6, bits=2), 190, None, 0),
    ("llama3_8b_gqa_128k", dict(B=2, Hq=8, Hkv=2, bits=4), 330, [330, 97], 1),
    # an empty sequence between two others (its output is defined as 0)
    ("batched_8x8k", dict(B=3, Hq=4, Hkv=4, bits=3), 260, [260, 0, 5], 0),
    # grouped-query table kernels at 2 bits: four and two query heads per kv head
    ("llama3_8b_gqa_128k", dict(B=1, Hq=8, Hkv=2, bits=2), 410, None, 1),
    ("batched_8x8k", dict(B=2, Hq=4, Hkv=2, bits=2), 300, [300, 123], 0),
]


def _setup(name, over, T, plen, appends):
    import torch
    w = synth.workload(name, **over)
    K16, V16 = host_block(w, T + 16)
    cbK, cbV = oracle_codebooks(w)
    cap = 1 << 18
    o = O.QuantizedCache(w.B, w.Hkv, w.bits, T + 16, w.f, cap, cap)
    pl = plen if plen is not None else [T] * w.B
    o.prefill(K16[:, :T], V16[:, :T], pl, cbK, cbV)
    g = gpu_cache(w, T + 16, cap, cap)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    gpu_quantize(g, dK, dV, K16[:, :T], V16[:, :T], plen=plen, calibrate=1)
    for step in range(appends):
        kt = np.stack([K16[b, int(o.len[b])] for b in range(w.B)])[:, None]
        vt = np.stack([V16[b, int(o.len[b])] for b in range(w.B)])[:, None]
        o.append(kt, vt, cbK, cbV)
        gpu_quantize(g, dK, dV, kt, vt)
    q16 = synth.gen_q(w)
    # query position: the just-appended token, or the next position when nothing was appended
    qpos = np.array([int(o.len[b]) - 1 if appends else int(o.len[b]) for b in range(w.B)],
                    dtype=np.int32)
    qpos = np.maximum(qpos, 0)
    refs = []
    for b in range(w.B):
        if o.len[b] == 0:
            refs.append(None)
            continue
        Kx, Vx = o.reconstruct(b, cbK, cbV)
        refs.append(O.decode_attention(q16[b], int(qpos[b]), Kx, Vx, w.rope_theta))
    dq = torch.from_numpy(q16).cuda()
    dpos = torch.from_numpy(qpos).cuda()
    return w, o, g, dK, dV, dq, dpos, refs, K16, V16


def _check_out(w, out, refs):
    for b in range(w.B):
        if refs[b] is None:  # no cached token: the library writes zeros
            assert not np.any(out[b]), b
            continue
        err = np.abs(out[b].astype(np.float64) - refs[b][2]).max()
        assert err <= OUT_ATOL, (b, err)


@pytest.mark.parametrize("name,over,T,plen,appends", CASES)
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_split_path(name, over, T, plen, appends, splits):
    import torch
    import long_context_decode_nuq_b200 as K
    w, o, g, dK, dV, dq, dpos, refs, _, _ = _setup(name, over, T, plen, appends)
    max_len = int(o.len.max())
    S = splits or K.kvq_decode_splits(g.cfg, max_len)
    logits = torch.full((w.B, w.Hq, g.cfg.T_max), float("nan"), device="cuda")
    stats = torch.empty((w.B, w.Hq, S, 2), device="cuda")
    ml = torch.empty((w.B, w.Hq, 2), device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    part = torch.empty((w.B, w.Hq, S, w.D), device="cuda")
    qws = torch.empty(K.kvq_decode_qk_workspace(g.cfg, max_len), dtype=torch.uint8, device="cuda")
    K.kvq_decode_qk(g, dK, dq, dpos, max_len, logits, stats, S, qws)
    K.kvq_softmax_merge(g.cfg, stats, S, ml)
    K.kvq_decode_pv(g, dV, logits, ml, max_len, out, part, S)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    mlh = ml.cpu().numpy()
    for b in range(w.B):
        L = int(o.len[b])
        if refs[b] is None:
            continue
        ref = refs[b][0]
        tol = LOGIT_RTOL * max(1.0, np.abs(ref).max())
        assert np.abs(lg[b, :, :L] - ref).max() <= tol
        # merged softmax statistics: M = max logit, L = sum exp(l - M)
        M = ref.max(axis=1)
        Ls = np.exp(ref - M[:, None]).sum(axis=1)
        assert np.allclose(mlh[b, :, 0], M, atol=tol)
        assert np.allclose(mlh[b, :, 1], Ls, rtol=2e-3)
    _check_out(w, out.cpu().numpy(), refs)
    assert K.kvq_get_status(g) == 0


@pytest.mark.parametrize("name,over,T,plen,appends", CASES)
def test_one_call_path(name, over, T, plen, appends):
    import torch
    import long_context_decode_nuq_b200 as K
    w, o, g, dK, dV, dq, dpos, refs, _, _ = _setup(name, over, T, plen, appends)
    max_len = int(o.len.max())
    for splits in (0, 2):
        ws = torch.empty(K.kvq_decode_workspace(g.cfg, max_len, splits), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty((w.B, w.Hq, w.D), device="cuda")
        K.kvq_decode_attention(g, dK, dV, dq, dpos, max_len, out, ws, splits)
        torch.cuda.synchronize()
        _check_out(w, out.cpu().numpy(), refs)


def _fused_ok(w):
    return w.Hq == w.Hkv and w.bits <= 3


@pytest.mark.parametrize("name,over,T,plen,appends", CASES)
def test_fused_path(name, over, T, plen, appends):
    """kvq_decode_attention_fused (one kernel per split, no logits in memory) where it applies;
    KVQ_ERR_UNSUPPORTED elsewhere."""
    import torch
    import long_context_decode_nuq_b200 as K
    w, o, g, dK, dV, dq, dpos, refs, _, _ = _setup(name, over, T, plen, appends)
    max_len = int(o.len.max())
    if not _fused_ok(w):
        with pytest.raises(K.KvqError):
            K.kvq_decode_fused_workspace(g.cfg, max_len, 0)
        return
    for splits in (0, 2, 5):
        ws = torch.empty(K.kvq_decode_fused_workspace(g.cfg, max_len, splits), dtype=torch.uint8,
                         device="cuda")
        assert ws.numel() < K.kvq_decode_workspace(g.cfg, max_len, splits)
        out = torch.empty((w.B, w.Hq, w.D), device="cuda")
        K.kvq_decode_attention_fused(g, dK, dV, dq, dpos, max_len, out, ws, splits)
        torch.cuda.synchronize()
        _check_out(w, out.cpu().numpy(), refs)
    assert K.kvq_get_status(g) == 0


@pytest.mark.parametrize("name,over,T,plen", [("tiny_single_head", {}, 2048, None),
                                              ("llama3_8b_gqa_128k", dict(B=2, Hq=16, Hkv=4),
                                               517, [517, 300]),
                                              ("llama7b_layer_32k", dict(Hq=8, Hkv=8), 1000,
                                               None)])
def test_fp16_comparison_kernel(name, over, T, plen):
    """The uncompressed kernel against binary64 attention over the unquantized cache."""
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload(name, **over)
    K16, V16 = host_block(w, T)
    pl = np.array(plen if plen is not None else [T] * w.B, dtype=np.int32)
    q16 = synth.gen_q(w)
    qpos = pl.copy()
    cfg = K.make_cfg(w.B, w.Hq, w.Hkv, w.bits, T, w.f, w.rope_theta, 0, 0)
    ws = torch.empty(K.kvq_decode_workspace(cfg, T, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    K.kvq_fp16_decode_attention(cfg, torch.from_numpy(K16).cuda(), torch.from_numpy(V16).cuda(),
                                T, torch.from_numpy(pl).cuda(), torch.from_numpy(q16).cuda(),
                                torch.from_numpy(qpos).cuda(), T, out, ws, 0)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    for b in range(w.B):
        _, _, ref = O.decode_attention(q16[b], int(qpos[b]), K16[b, : pl[b]], V16[b, : pl[b]],
                                       w.rope_theta)
        assert np.abs(o[b] - ref).max() <= OUT_ATOL


# many outliers (5 %), ragged lengths across several 256-token stages and 64-token chunks
HEAVY = [
    ("llama7b_layer_32k", dict(B=3, Hq=4, Hkv=4, f=0.05), 1500, [1500, 777, 3], 1),
    ("batched_8x8k", dict(B=2, Hq=2, Hkv=2, bits=2, f=0.05), 1300, [1300, 1025], 0),
]


@pytest.mark.parametrize("name,over,T,plen,appends", HEAVY)
@pytest.mark.parametrize("splits", [0, 1, 4])
def test_outlier_heavy(name, over, T, plen, appends, splits):
    import torch
    import long_context_decode_nuq_b200 as K
    w, o, g, dK, dV, dq, dpos, refs, _, _ = _setup(name, over, T, plen, appends)
    max_len = int(o.len.max())
    ws = torch.empty(K.kvq_decode_workspace(g.cfg, max_len, splits), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    K.kvq_decode_attention(g, dK, dV, dq, dpos, max_len, out, ws, splits)
    torch.cuda.synchronize()
    _check_out(w, out.cpu().numpy(), refs)
    if _fused_ok(w):   # many outliers: past the per-stage staging of the fused kernel
        K.kvq_decode_attention_fused(g, dK, dV, dq, dpos, max_len, out, ws, splits)
        torch.cuda.synchronize()
        _check_out(w, out.cpu().numpy(), refs)
    assert K.kvq_get_status(g) == 0


@pytest.mark.parametrize("name,over,T,plen,appends", [CASES[1], CASES[4], CASES[5], HEAVY[0]])
def test_decode_is_deterministic(name, over, T, plen, appends):
    """Two calls on the same inputs give the same bits: one-call path and the three calls."""
    import torch
    import long_context_decode_nuq_b200 as K
    w, o, g, dK, dV, dq, dpos, refs, _, _ = _setup(name, over, T, plen, appends)
    max_len = int(o.len.max())
    ws = torch.empty(K.kvq_decode_workspace(g.cfg, max_len, 0), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        out = torch.empty((w.B, w.Hq, w.D), device="cuda")
        ws.fill_(0x55)
        K.kvq_decode_attention(g, dK, dV, dq, dpos, max_len, out, ws, 0)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy().view(np.uint32))
    assert np.array_equal(outs[0], outs[1])
    if _fused_ok(w):
        fo = []
        for _ in range(2):
            out = torch.empty((w.B, w.Hq, w.D), device="cuda")
            ws.fill_(0x33)
            K.kvq_decode_attention_fused(g, dK, dV, dq, dpos, max_len, out, ws, 0)
            torch.cuda.synchronize()
            fo.append(out.cpu().numpy().view(np.uint32))
        assert np.array_equal(fo[0], fo[1])
    S = K.kvq_decode_splits(g.cfg, max_len)
    res = []
    for _ in range(2):
        logits = torch.zeros((w.B, w.Hq, g.cfg.T_max), device="cuda")
        stats = torch.empty((w.B, w.Hq, S, 2), device="cuda")
        ml = torch.empty((w.B, w.Hq, 2), device="cuda")
        out = torch.empty((w.B, w.Hq, w.D), device="cuda")
        part = torch.empty((w.B, w.Hq, S, w.D), device="cuda")
        qws = torch.empty(K.kvq_decode_qk_workspace(g.cfg, max_len), dtype=torch.uint8,
                          device="cuda")
        K.kvq_decode_qk(g, dK, dq, dpos, max_len, logits, stats, S, qws)
        K.kvq_softmax_merge(g.cfg, stats, S, ml)
        K.kvq_decode_pv(g, dV, logits, ml, max_len, out, part, S)
        torch.cuda.synchronize()
        res.append((logits.cpu().numpy().view(np.uint32), out.cpu().numpy().view(np.uint32)))
    assert np.array_equal(res[0][0], res[1][0])
    assert np.array_equal(res[0][1], res[1][1])
    assert K.kvq_get_status(g) == 0


@pytest.mark.parametrize("name,over,T,cut", [
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 900, 448),          # one query head per kv head
    ("llama3_8b_gqa_128k", dict(B=1, Hq=8, Hkv=2), 700, 320),    # split kernels (GQA)
    ("batched_8x8k", dict(B=1, Hq=4, Hkv=4, bits=4), 500, 500),  # second range empty
])
def test_sharded_partials(name, over, T, cut):
    """Two token ranges of one sequence in two caches (each calibrated on its own range), their
    partials at absolute positions merged by kvq_merge_partials, against the oracle's attention
    over the two ranges' reconstructions concatenated."""
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload(name, **over)
    K16, V16 = host_block(w, T)
    cbK, cbV = oracle_codebooks(w)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    cap = 1 << 16
    q16 = synth.gen_q(w)
    qpos = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    dq = torch.from_numpy(q16).cuda()
    mls, os_, recon = [], [], []
    for lo, hi in ((0, cut), (cut, T)):
        n = hi - lo
        g = gpu_cache(w, max(n, 1) + 16, cap, cap)
        oc = O.QuantizedCache(w.B, w.Hkv, w.bits, max(n, 1) + 16, w.f, cap, cap)
        if n:
            gpu_quantize(g, dK, dV, K16[:, lo:hi], V16[:, lo:hi], calibrate=1)
            oc.prefill(K16[:, lo:hi], V16[:, lo:hi], [n], cbK, cbV)
            recon.append(oc.reconstruct(0, cbK, cbV))
        ml = torch.empty((w.B, w.Hq, 2), device="cuda")
        o = torch.empty((w.B, w.Hq, w.D), device="cuda")
        ws = torch.empty(K.kvq_decode_workspace(g.cfg, max(n, 1), 0), dtype=torch.uint8,
                         device="cuda")
        K.kvq_decode_partial(g, dK, dV, dq, qpos, max(n, 1), lo, ml, o, ws, 0)
        torch.cuda.synchronize()
        assert K.kvq_get_status(g) == 0
        if not n:
            assert np.all(ml[..., 0].cpu().numpy() == -np.inf) and not o.cpu().numpy().any()
        mls.append(ml)
        os_.append(o)
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    K.kvq_merge_partials(g.cfg, 2, torch.stack(mls), torch.stack(os_), out)
    torch.cuda.synchronize()
    Kx = np.concatenate([r[0] for r in recon])
    Vx = np.concatenate([r[1] for r in recon])
    _, _, ref = O.decode_attention(q16[0], T, Kx, Vx, w.rope_theta)
    assert np.abs(out.cpu().numpy()[0] - ref).max() <= OUT_ATOL
