"""Parity at the workloads' full sizes, in the launch configuration bench.py times (split count
chosen by the library).

Inputs come from the device generator (bit-identical to the numpy one; see test_synth.py) and
are copied to the host for the oracle.  Where the oracle cannot cover a whole workload in
seconds, it covers sampled sequences, channels, tokens and heads one by one.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from kvq_testlib import compare_cache, gpu_cache, oracle_codebooks, to_dev_codebook, u16, u32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

LOGIT_RTOL = 1e-3
OUT_ATOL = 2e-3


def _device_block(w, T, layer=0):
    import torch
    from synth.gpu import DeviceGen
    g = DeviceGen(w, layer)
    K = torch.empty((w.B, T, w.Hkv, w.D), dtype=torch.float16, device="cuda")
    V = torch.empty_like(K)
    g.fill_k(K, 0, T)
    g.fill_v(V, 0, T)
    return K, V


def _device_q(w, step=0, layer=0):
    import torch
    from synth.gpu import DeviceGen
    q = torch.empty((w.B, w.Hq, w.D), dtype=torch.float16, device="cuda")
    DeviceGen(w, layer).fill_q(q, step)
    return q


def _quantize(cache, dK, dV, k, v, calibrate):
    import torch
    import long_context_decode_nuq_b200 as K
    ws = torch.empty(K.kvq_quantize_workspace(cache.cfg, k.shape[1], calibrate), dtype=torch.uint8,
                     device="cuda")
    K.kvq_quantize_append(cache, dK, dV, k.contiguous(), v.contiguous(), k.shape[1], None,
                          calibrate, ws)


def _attend(cache, dK, dV, q, qpos, max_len):
    """Both decode paths as bench.py runs them: the one-call kvq_decode_attention and the split calls."""
    import torch
    import long_context_decode_nuq_b200 as K
    cfg = cache.cfg
    S = K.kvq_decode_splits(cfg, max_len)
    ws = torch.empty(K.kvq_decode_workspace(cfg, max_len, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((cfg.B, cfg.Hq, 128), dtype=torch.float32, device="cuda")
    K.kvq_decode_attention(cache, dK, dV, q, qpos, max_len, out, ws, 0)
    logits = torch.full((cfg.B, cfg.Hq, cfg.T_max), float("nan"), device="cuda")
    stats = torch.empty((cfg.B, cfg.Hq, S, 2), device="cuda")
    ml = torch.empty((cfg.B, cfg.Hq, 2), device="cuda")
    out2 = torch.empty_like(out)
    part = torch.empty((cfg.B, cfg.Hq, S, 128), device="cuda")
    qws = torch.empty(K.kvq_decode_qk_workspace(cfg, max_len), dtype=torch.uint8, device="cuda")
    K.kvq_decode_qk(cache, dK, q, qpos, max_len, logits, stats, S, qws)
    K.kvq_softmax_merge(cfg, stats, S, ml)
    K.kvq_decode_pv(cache, dV, logits, ml, max_len, out2, part, S)
    torch.cuda.synchronize()
    assert K.kvq_get_status(cache) == 0
    return out.cpu().numpy(), out2.cpu().numpy(), logits.cpu().numpy()


def _check_attention(ref, out, out2, logits, L):
    lg_ref, _, o_ref = ref
    assert np.abs(out - o_ref).max() <= OUT_ATOL
    assert np.abs(out2 - o_ref).max() <= OUT_ATOL
    tol = LOGIT_RTOL * max(1.0, np.abs(lg_ref).max())
    assert np.abs(logits[:, :L] - lg_ref).max() <= tol


def test_llama7b_layer_32k_full():
    """One LLaMA-7B layer: 32 heads, 32768 cached tokens, a 1-token append, then attention."""
    import torch
    w = synth.workload("llama7b_layer_32k")
    T = w.T
    Kd, Vd = _device_block(w, T + 1)
    cbK, cbV = oracle_codebooks(w)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    cap = 1 << 20
    g = gpu_cache(w, T + 64, cap, cap)
    _quantize(g, dK, dV, Kd[:, :T], Vd[:, :T], 1)
    _quantize(g, dK, dV, Kd[:, T:T + 1], Vd[:, T:T + 1], 0)
    q = _device_q(w)
    qpos = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    out, out2, logits = _attend(g, dK, dV, q, qpos, T + 1)
    K16, V16 = Kd.cpu().numpy(), Vd.cpu().numpy()
    o = O.QuantizedCache(w.B, w.Hkv, w.bits, T + 64, w.f, cap, cap)
    o.prefill(K16[:, :T], V16[:, :T], [T], cbK, cbV)
    o.append(K16[:, T:T + 1], V16[:, T:T + 1], cbK, cbV)
    compare_cache(g, o, w.B)
    Kx, Vx = o.reconstruct(0, cbK, cbV)
    ref = O.decode_attention(q.cpu().numpy()[0], T, Kx, Vx, w.rope_theta)
    _check_attention(ref, out[0], out2[0], logits[0], T + 1)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_batched_8x8k_append_steps(bits):
    """8 sequences x 8192 tokens, 64 append-then-attend steps; one sequence checked per width."""
    import torch
    w = synth.workload("batched_8x8k", bits=bits)
    T, steps = w.T, w.steps
    Kd, Vd = _device_block(w, T + steps)
    cbK, cbV = oracle_codebooks(w)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    cap = 1 << 19
    g = gpu_cache(w, T + steps + 64, cap, cap)
    _quantize(g, dK, dV, Kd[:, :T], Vd[:, :T], 1)
    b = {2: 1, 3: 4, 4: 7}[bits]
    check_steps = {0, steps // 2, steps - 1}
    K16 = Kd[b:b + 1].cpu().numpy()
    V16 = Vd[b:b + 1].cpu().numpy()
    o = O.QuantizedCache(1, w.Hkv, w.bits, T + steps + 64, w.f, cap, cap)
    o.prefill(K16[:, :T], V16[:, :T], [T], cbK, cbV)
    for s in range(steps):
        t = T + s
        _quantize(g, dK, dV, Kd[:, t:t + 1], Vd[:, t:t + 1], 0)
        o.append(K16[:, t:t + 1], V16[:, t:t + 1], cbK, cbV)
        if s in check_steps:
            q = _device_q(w, step=s)
            qpos = torch.full((w.B,), t, dtype=torch.int32, device="cuda")
            out, out2, logits = _attend(g, dK, dV, q, qpos, t + 1)
            Kx, Vx = o.reconstruct(0, cbK, cbV)
            ref = O.decode_attention(q.cpu().numpy()[b], t, Kx, Vx, w.rope_theta)
            _check_attention(ref, out[b], out2[b], logits[b], t + 1)

    # the sampled sequence's whole cache after the 64 steps
    class One:  # view of sequence b of the device cache with the oracle's batch of one
        def __init__(self, c):
            for name in ("kcodes", "vcodes", "kthr", "kparams", "vparams", "kout", "vout",
                         "kchunk", "vchunk", "kcount", "vcount", "len"):
                setattr(self, name, getattr(c, name)[b:b + 1])
            self.status = c.status
    compare_cache(One(g), o, 1)


def test_llama3_8b_gqa_128k_sampled_sequence():
    """GQA 32 query heads over 8 kv heads, 4 sequences x 131072 tokens; sequence 2 checked."""
    import torch
    w = synth.workload("llama3_8b_gqa_128k")
    T = w.T
    Kd, Vd = _device_block(w, T)
    cbK, cbV = oracle_codebooks(w)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    cap = 1 << 20
    g = gpu_cache(w, T + 64, cap, cap)
    _quantize(g, dK, dV, Kd, Vd, 1)
    q = _device_q(w)
    qpos = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    out, out2, logits = _attend(g, dK, dV, q, qpos, T)
    b = 2
    o = O.QuantizedCache(1, w.Hkv, w.bits, T + 64, w.f, cap, cap)
    o.prefill(Kd[b:b + 1].cpu().numpy(), Vd[b:b + 1].cpu().numpy(), [T], cbK, cbV)
    Kx, Vx = o.reconstruct(0, cbK, cbV)
    ref = O.decode_attention(q.cpu().numpy()[b], T, Kx, Vx, w.rope_theta)
    _check_attention(ref, out[b], out2[b], logits[b], T)
    assert np.array_equal(u32(g.kcodes[b]), o.kcodes[0])
    assert np.array_equal(u32(g.vcodes[b]), o.vcodes[0])
    for s in ("k", "v"):
        for h in range(w.Hkv):
            n = int(o.out_count[s][0, h])
            assert int(u32(getattr(g, f"{s}count"))[b, h]) == n
            assert np.array_equal(u32(getattr(g, f"{s}out")[b, h, :n]), o.out[s][0, h, :n])


def _unpack_head(words, bits):
    """Codes [T, 128] of one kv head from its blocks [nq, 16*bits] (oracle unpacker)."""
    q = O.unpack_block(words, bits)            # [4, nq, 128]
    return np.transpose(q, (1, 0, 2)).reshape(-1, 128)


def _head_attention(q16, qpos, kx, vx, base, chunk=1 << 16):
    """binary64 attention of one query head over one kv head, in token chunks."""
    qr = O.rope_rotate(np.asarray(q16, dtype=np.float64)[None], qpos, base)[0]
    T = kx.shape[0]
    lg = np.empty(T)
    for a in range(0, T, chunk):
        kr = O.rope_rotate(kx[a:a + chunk], np.arange(a, min(T, a + chunk)), base)
        lg[a:a + chunk] = kr @ qr / math.sqrt(128)
    p = np.exp(lg - lg.max())
    p /= p.sum()
    out = np.zeros(128)
    for a in range(0, T, chunk):
        out += p[a:a + chunk] @ vx[a:a + chunk]
    return lg, out


def test_llama7b_1m_layer_sampled():
    """One layer of the 1M-token workload as bench.py builds it: sampled key channels and
    tokens against the oracle's quantizer, and one head's attention over all 1,048,576 tokens
    recomputed in binary64 from the device cache."""
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload("llama7b_1m_32layers", layers=1)
    T = w.T
    Kd, Vd = _device_block(w, T)
    cbK, cbV = oracle_codebooks(w)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    ceil8 = lambda x: (int(x) + 7) // 8 * 8  # noqa: E731
    capk = ceil8(T * w.f * w.D * 1.25 + 4096)
    capv = ceil8(T * 2 * math.floor(w.f * w.n / 2 + 0.5) / w.Hkv * 1.5 + 4096)
    g = gpu_cache(w, T + 64, capk, capv)
    _quantize(g, dK, dV, Kd, Vd, 1)
    torch.cuda.synchronize()
    assert K.kvq_get_status(g) == 0
    rng = np.random.default_rng(7)
    # key calibration of sampled channels: exact order statistics over the million tokens
    chans = [0, 1, 777, 2048, 4095] + rng.integers(0, w.n, 5).tolist()
    kthr = u16(g.kthr[0])
    kpar = g.kparams[0].cpu().numpy()
    for j in chans:
        col = Kd[0, :, j // 128, j % 128].cpu().numpy()
        lo, hi = O.order_stat_thresholds(col, w.f, axis=0)
        assert kthr[j, 0] == lo.view(np.uint16) and kthr[j, 1] == hi.view(np.uint16), j
        off, half = O.affine_params(lo, hi)
        assert kpar[j, 0] == off and kpar[j, 1] == half, j
    # sampled tokens: value thresholds, value codes and their outliers, key codes of the
    # sampled channels
    toks = [0, 1, 63, 64, T - 1] + rng.integers(0, T, 11).tolist()
    vpar = g.vparams[0].cpu().numpy()
    kc_all = {h: None for h in range(w.Hkv)}
    for t in toks:
        row = Vd[0, t].reshape(-1).cpu().numpy()
        lo, hi = O.order_stat_thresholds(row[None], w.f, axis=1)
        off, half = O.affine_params(lo[0], hi[0])
        assert vpar[t, 0] == off and vpar[t, 1] == half, t
        vout = (row < lo[0]) | (row > hi[0])
        codes = O.encode(O.normalize(np.where(vout, np.float16(0), row), off, half), cbV[1])
        blk = u32(g.vcodes[0, :, t // 4])              # [Hkv, 16*bits]
        got = O.unpack_block(blk, w.bits)[t % 4].reshape(-1)
        assert np.array_equal(got, codes), t
        krow = Kd[0, t].reshape(-1).cpu().numpy()
        kblk = O.unpack_block(u32(g.kcodes[0, :, t // 4]), w.bits)[t % 4].reshape(-1)
        for j in chans:
            lo_j = kthr[j, 0].view(np.float16)
            hi_j = kthr[j, 1].view(np.float16)
            x = krow[j]
            xk = np.float16(0) if (x < lo_j or x > hi_j) else x
            cj = O.encode(O.normalize(np.array([xk]), kpar[j, 0], kpar[j, 1]), cbK[1])[0]
            assert kblk[j] == cj, (t, j)
    # one head's attention over every token, from the device cache
    h = 7
    q = _device_q(w)
    qpos = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    out, out2, logits = _attend(g, dK, dV, q, qpos, T)
    kc = _unpack_head(u32(g.kcodes[0, h]), w.bits)[:T]
    vc = _unpack_head(u32(g.vcodes[0, h]), w.bits)[:T]
    levK = np.asarray(cbK[0], dtype=np.float64)
    levV = np.asarray(cbV[0], dtype=np.float64)
    kp = kpar[h * 128:(h + 1) * 128].astype(np.float64)
    vp = vpar[:T].astype(np.float64)
    kx = kp[:, 0] + kp[:, 1] * levK[kc]
    vx = vp[:, 0:1] + vp[:, 1:2] * levV[vc]
    for s, X in (("k", kx), ("v", vx)):
        n = int(u32(getattr(g, f"{s}count"))[0, h])
        ent = u32(getattr(g, f"{s}out")[0, h, :n]).astype(np.int64)
        nch = (T + 63) // 64                                      # chunks of the cached tokens
        cp = u32(getattr(g, f"{s}chunk")[0, h, :nch + 1]).astype(np.int64)
        m = np.searchsorted(cp, np.arange(n), side="right") - 1   # chunk of each entry
        t = m * 64 + ((ent >> 7) & 63)
        X[t, ent & 127] = (ent >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    for hq in (h,):
        lg_ref, o_ref = _head_attention(q.cpu().numpy()[0, hq], T, kx, vx, w.rope_theta)
        assert np.abs(out[0, hq] - o_ref).max() <= OUT_ATOL
        assert np.abs(out2[0, hq] - o_ref).max() <= OUT_ATOL
        tol = LOGIT_RTOL * max(1.0, np.abs(lg_ref).max())
        assert np.abs(logits[0, hq, :T] - lg_ref).max() <= tol
