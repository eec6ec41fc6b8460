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


def _unpack_head3(words):
    """_unpack_head for 3-bit blocks, vectorised over the 16 lane groups (a test helper for
    the 1M-token check; checked against the oracle's unpacker on sampled blocks).  Lane group
    i holds 16 six-bit fields in its three words; field 4k + s is token s ^ (i >> 2), codes of
    channels i + 16k (low 3 bits) and i + 16k + 64 (high 3 bits)."""
    nq = words.shape[0]
    W = words.reshape(nq, 16, 3).astype(np.uint64)
    A = W[..., 0] | (W[..., 1] << np.uint64(32))
    B = W[..., 2]
    F = np.empty((nq, 16, 16), dtype=np.uint8)
    for f in range(16):
        o = 6 * f
        if o + 6 <= 64:
            v = A >> np.uint64(o)
        elif o < 64:
            v = (A >> np.uint64(o)) | (B << np.uint64(64 - o))
        else:
            v = B >> np.uint64(o - 64)
        F[..., f] = (v & np.uint64(63)).astype(np.uint8)
    i = np.arange(16)[:, None, None]
    k = np.arange(4)[None, :, None]
    j = np.arange(4)[None, None, :]
    ii = np.broadcast_to(i, (16, 4, 4))
    ff = np.broadcast_to(4 * k + (j ^ (i >> 2)), (16, 4, 4))   # field of token j, channel i+16k
    src = F[:, ii, ff]                                          # [nq, 16 i, 4 k, 4 j]
    codes = np.empty((nq, 4, 128), dtype=np.uint8)
    ch = (np.arange(16)[:, None] + 16 * np.arange(4)[None, :]).reshape(-1)   # i + 16k
    lo = np.transpose(src, (0, 3, 1, 2)).reshape(nq, 4, 64)
    codes[:, :, ch] = lo & 7
    codes[:, :, ch + 64] = lo >> 3
    sample = np.random.default_rng(nq).integers(0, nq, 64)
    ref = O.unpack_block(words[sample], 3)                     # [4, 64, 128]
    assert np.array_equal(np.transpose(ref, (1, 0, 2)), codes[sample])
    return codes.reshape(-1, 128)


def _device_entries(g, s, h, m):
    """Entries of chunk m in the device list s ('k' or 'v') of (sequence 0, kv head h)."""
    cp = u32(getattr(g, f"{s}chunk")[0, h, m:m + 2])
    return u32(getattr(g, f"{s}out")[0, h, int(cp[0]):int(cp[1])])


def test_llama7b_1m_layer_sampled():
    """One layer of the 1M-token workload as bench.py builds it.

    Quantizer, against the oracle's own quantizer:
      * key calibration: thresholds and (off, half) of every channel of two kv heads, from the
        oracle's order statistics over all 1,048,576 tokens;
      * sampled 64-token chunks (several past token 131,072): key codes and key-outlier entries
        of those heads (the oracle's QuantizedCache calibrated on the head's full columns and
        quantizing the chunk), value (off, half), value codes and value-outlier entries of all
        32 kv heads (the oracle quantizing the chunk's rows).
    Attention of all 32 heads over every token, in binary64 from the device cache (whose
    sampled rows the checks above tie to the oracle), against both decode paths."""
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
    chunks = sorted({0, 1, 2047, 2048, 2049, T // 64 - 1}
                    | set(int(x) for x in rng.integers(2049, T // 64 - 1, 6)))
    kthr = u16(g.kthr[0])
    kpar = g.kparams[0].cpu().numpy()
    for h in (7, 30):
        col = Kd[0, :, h:h + 1].cpu().numpy()               # [T, 1, 128]
        ok = O.QuantizedCache(1, 1, w.bits, 64, w.f, 64 * 128, 64 * 128)
        ok.calibrate_keys(0, col)
        sl = slice(h * 128, (h + 1) * 128)
        assert np.array_equal(kthr[sl], ok.kthr[0]), h
        assert np.array_equal(kpar[sl], ok.kparams[0]), h
        for m in chunks:
            oc = O.QuantizedCache(1, 1, w.bits, 64, w.f, 64 * 128, 64 * 128)
            oc.kthr[:], oc.kparams[:] = ok.kthr, ok.kparams
            rows = slice(64 * m, 64 * m + 64)
            oc.quantize_tokens(0, 0, col[rows], Vd[0, rows, h:h + 1].cpu().numpy(), cbK, cbV)
            assert np.array_equal(u32(g.kcodes[0, h, 16 * m:16 * m + 16]), oc.kcodes[0, 0]), (h, m)
            n = int(oc.out_count["k"][0, 0])
            assert np.array_equal(_device_entries(g, "k", h, m), oc.out["k"][0, 0, :n]), (h, m)
    vpar = g.vparams[0].cpu().numpy()
    for m in chunks:
        rows = slice(64 * m, 64 * m + 64)
        ov = O.QuantizedCache(1, w.Hkv, w.bits, 64, w.f, 64 * 128, 64 * 128)
        ov.prefill(Kd[:, rows].cpu().numpy(), Vd[:, rows].cpu().numpy(), [64], cbK, cbV)
        assert np.array_equal(vpar[rows], ov.vparams[0]), m
        assert np.array_equal(u32(g.vcodes[0, :, 16 * m:16 * m + 16]), ov.vcodes[0]), m
        for h in range(w.Hkv):
            n = int(ov.out_count["v"][0, h])
            assert np.array_equal(_device_entries(g, "v", h, m), ov.out["v"][0, h, :n]), (h, m)
    # attention of every head over every token, from the device cache: the oracle's
    # decode_attention per head, heads spread over a spawn-started process pool
    q = _device_q(w)
    qpos = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    out, out2, logits = _attend(g, dK, dV, q, qpos, T)
    nch = (T + 63) // 64
    q16 = q.cpu().numpy()[0]
    jobs = []
    for h in range(w.Hkv):
        lists = {}
        for s_ in ("k", "v"):
            n = int(u32(getattr(g, f"{s_}count"))[0, h])
            lists[s_] = (u32(getattr(g, f"{s_}out")[0, h, :n]),
                         u32(getattr(g, f"{s_}chunk")[0, h, :nch + 1]))
        jobs.append((q16[h], T, u32(g.kcodes[0, h]), u32(g.vcodes[0, h]),
                     kpar[h * 128:(h + 1) * 128], vpar[:T], lists, cbK[0], cbV[0], w.rope_theta))
    for h, (lg_ref, o_ref) in enumerate(_pool_map(_head_reference, jobs)):
        assert np.abs(out[0, h] - o_ref).max() <= OUT_ATOL, h
        assert np.abs(out2[0, h] - o_ref).max() <= OUT_ATOL, h
        tol = LOGIT_RTOL * max(1.0, np.abs(lg_ref).max())
        assert np.abs(logits[0, h, :T] - lg_ref).max() <= tol, h


def _head_reference(job):
    """One kv head (one query head) of the 1M-token check: rebuild the head's exact K-hat and
    V-hat from the device codes and outlier lists (off + half L[code], outliers replaced by
    their stored value) and run the oracle's binary64 decode attention on them."""
    q16, T, kwords, vwords, kp, vp, lists, levK, levV, base = job
    kc = _unpack_head3(kwords)[:T]
    vc = _unpack_head3(vwords)[:T]
    kp = kp.astype(np.float64)
    vp = vp.astype(np.float64)
    kx = kp[:, 0] + kp[:, 1] * np.asarray(levK, dtype=np.float64)[kc]
    vx = vp[:, 0:1] + vp[:, 1:2] * np.asarray(levV, dtype=np.float64)[vc]
    del kc, vc
    for s_, X in (("k", kx), ("v", vx)):
        ent, cp = lists[s_]
        ent = ent.astype(np.int64)
        mm = np.searchsorted(cp.astype(np.int64), np.arange(len(ent)), side="right") - 1
        t = mm * 64 + ((ent >> 7) & 63)
        X[t, ent & 127] = (ent >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    lg, _, out = O.decode_attention(q16[None], T, kx[:, None], vx[:, None], base)
    return lg[0], out[0]


def _pool_map(fn, jobs):
    """Map over a process pool started with spawn (safe after CUDA use), sized to the host."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    try:
        import psutil
        mem_workers = int(psutil.virtual_memory().available // (8 << 30))
    except Exception:  # pragma: no cover
        mem_workers = 4
    n = max(1, min(len(jobs), os.cpu_count() or 1, mem_workers, 16))
    with cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(fn, jobs))
