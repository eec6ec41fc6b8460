"""GPU quantizer parity: bit-exact against the oracle (codes, outliers, params, K/V-hat)."""
import numpy as np
import pytest

import oracle as O
import synth
from kvq_testlib import (compare_cache, gpu_cache, gpu_quantize, host_block, oracle_codebooks,
                         to_dev_codebook, u16)

pytestmark = pytest.mark.gpu

CASES = [
    # (workload, overrides, prefill tokens, plen per sequence or None)
    ("tiny_single_head", {}, 2048, None),
    ("llama7b_layer_32k", dict(Hq=4, Hkv=4), 300, None),
    ("batched_8x8k", dict(B=3, Hq=4, Hkv=4, bits=2), 200, [200, 137, 0]),
    ("batched_8x8k", dict(B=2, Hq=4, Hkv=4, bits=4), 130, [130, 65]),
    ("llama3_8b_gqa_128k", dict(B=2, Hq=8, Hkv=2), 257, [257, 1]),
    ("llama7b_layer_32k", dict(Hq=32, Hkv=32, f=0.0), 100, None),
]


def _build(name, over, T, plen, extra=8, cap=1 << 18):
    w = synth.workload(name, **over)
    K16, V16 = host_block(w, T + extra)
    cbK, cbV = oracle_codebooks(w)
    o = O.QuantizedCache(w.B, w.Hkv, w.bits, T + extra, w.f, cap, cap)
    pl = plen if plen is not None else [T] * w.B
    o.prefill(K16[:, :T], V16[:, :T], pl, cbK, cbV)
    g = gpu_cache(w, T + extra, cap, cap)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    gpu_quantize(g, dK, dV, K16[:, :T], V16[:, :T], plen=plen, calibrate=1)
    return w, K16, V16, cbK, cbV, o, g, dK, dV


@pytest.mark.parametrize("name,over,T,plen", CASES)
def test_prefill_bit_exact(name, over, T, plen):
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build(name, over, T, plen)
    compare_cache(g, o, w.B)


@pytest.mark.parametrize("name,over,T,plen", CASES[:5])
def test_append_bit_exact(name, over, T, plen):
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build(name, over, T, plen)
    B = w.B
    lens = o.len.copy()
    # three single-token appends, then a block of four tokens
    for step in range(3):
        kt = np.stack([K16[b, min(lens[b] + step, T + 7)] for b in range(B)])[:, None]
        vt = np.stack([V16[b, min(lens[b] + step, T + 7)] for b in range(B)])[:, None]
        o.append(kt, vt, cbK, cbV)
        gpu_quantize(g, dK, dV, kt, vt)
        compare_cache(g, o, B)
    blk_k = np.stack([K16[b, T + 2: T + 6] for b in range(B)])
    blk_v = np.stack([V16[b, T + 2: T + 6] for b in range(B)])
    if all(int(o.len[b]) + 4 <= T + 8 for b in range(B)):
        o.append(blk_k, blk_v, cbK, cbV)
        gpu_quantize(g, dK, dV, blk_k, blk_v)
        compare_cache(g, o, B)


def test_outlier_capacity_overflow():
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build("llama7b_layer_32k", dict(Hq=4, Hkv=4), 150,
                                                  None, cap=200)
    import long_context_decode_nuq_b200 as K
    assert o.status & O.STATUS_OUTLIER_OVERFLOW
    compare_cache(g, o, w.B)
    assert K.kvq_get_status(g) & K.KVQ_STATUS_OUTLIER_OVERFLOW


def test_prefill_on_nonempty_sequence_sets_status():
    import long_context_decode_nuq_b200 as K
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build("llama7b_layer_32k", dict(Hq=4, Hkv=4), 64,
                                                  None)
    before = g.kcodes.clone()
    gpu_quantize(g, dK, dV, K16[:, :64], V16[:, :64], calibrate=1)
    assert K.kvq_get_status(g) & K.KVQ_STATUS_NOT_EMPTY
    assert bool((g.kcodes == before).all())
    # appending past T_max is skipped and flagged
    K.kvq_cache_reset(g)
    gpu_quantize(g, dK, dV, K16[:, :72], V16[:, :72], calibrate=1)
    gpu_quantize(g, dK, dV, K16[:, :1], V16[:, :1])
    assert K.kvq_get_status(g) & K.KVQ_STATUS_LEN_OVERFLOW
    assert int(g.len.cpu()[0]) == 72


@pytest.mark.parametrize("name,over,T,plen", [CASES[0], CASES[2], CASES[4]])
def test_dequantize_bit_exact(name, over, T, plen):
    import torch
    import long_context_decode_nuq_b200 as K
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build(name, over, T, plen)
    n = w.Hkv * w.D
    kh = torch.empty((w.B, T, w.Hkv, w.D), dtype=torch.float16, device="cuda")
    vh = torch.empty_like(kh)
    K.kvq_dequantize(g, dK, dV, 0, T, kh, vh)
    torch.cuda.synchronize()
    for b in range(w.B):
        L = int(o.len[b])
        Kh, Vh = o.dequantize(b, cbK, cbV)
        assert np.array_equal(u16(kh[b, :L]), Kh.view(np.uint16))
        assert np.array_equal(u16(vh[b, :L]), Vh.view(np.uint16))
        assert not u16(kh[b, L:]).any()


@pytest.mark.parametrize("name", ["tiny_single_head", "llama3_8b_gqa_128k", "llama7b_layer_32k"])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codebook_fit_matches_oracle(name, bits):
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload(name, bits=bits)
    for samples in (synth.codebook_samples_k(w), synth.codebook_samples_v(w)):
        lev_o, bnd_o = O.fit_codebook(samples, w.f, bits)
        s = torch.from_numpy(samples.view(np.uint16).astype(np.int32)).to(torch.int16).cuda()
        lev = torch.empty(1 << bits, dtype=torch.float32, device="cuda")
        bnd = torch.empty((1 << bits) - 1, dtype=torch.float32, device="cuda")
        ws = torch.empty(K.kvq_fit_workspace(*samples.shape), dtype=torch.uint8, device="cuda")
        K.kvq_fit_codebook(s, w.f, bits, lev, bnd, ws)
        torch.cuda.synchronize()
        assert np.array_equal(lev.cpu().numpy(), lev_o)
        assert np.array_equal(bnd.cpu().numpy(), bnd_o)


def test_codebook_fit_weighted():
    import torch
    import long_context_decode_nuq_b200 as K
    w = synth.workload("llama7b_layer_32k")
    samples = synth.codebook_samples_v(w)
    wts = np.random.default_rng(0).uniform(0.25, 4.0, samples.shape)
    lev_o, _ = O.fit_codebook(samples, w.f, 3, weights=wts)
    s = torch.from_numpy(samples.view(np.uint16).astype(np.int32)).to(torch.int16).cuda()
    lev = torch.empty(8, dtype=torch.float32, device="cuda")
    bnd = torch.empty(7, dtype=torch.float32, device="cuda")
    ws = torch.empty(K.kvq_fit_workspace(*samples.shape), dtype=torch.uint8, device="cuda")
    K.kvq_fit_codebook(s, w.f, 3, lev, bnd, ws, weights=torch.from_numpy(wts).cuda())
    torch.cuda.synchronize()
    # weighted sums are reduced in another order: levels agree to rounding
    assert np.allclose(lev.cpu().numpy(), lev_o, rtol=0, atol=2 ** -7 * np.abs(lev_o).max())


@pytest.mark.parametrize("name", ["tiny_single_head", "llama7b_layer_32k", "llama3_8b_gqa_128k"])
def test_device_generator_matches_numpy(name):
    import torch
    from synth.gpu import DeviceGen
    w = synth.workload(name, B=min(2, synth.workload(name).B))
    T = 96
    K16, V16 = host_block(w, T)
    g = DeviceGen(w)
    k = torch.empty((w.B, 40, w.Hkv, w.D), dtype=torch.float16, device="cuda")
    v = torch.empty_like(k)
    g.fill_k(k, 50, 40)
    g.fill_v(v, 50, 40)
    q = torch.empty((w.B, w.Hq, w.D), dtype=torch.float16, device="cuda")
    g.fill_q(q, step=3)
    torch.cuda.synchronize()
    assert np.array_equal(u16(k), K16[:, 50:90].view(np.uint16))
    assert np.array_equal(u16(v), V16[:, 50:90].view(np.uint16))
    assert np.array_equal(u16(q), synth.gen_q(w, 0, 3).view(np.uint16))


@pytest.mark.parametrize("name,over,T,plen", [CASES[1], CASES[4], CASES[2]])
def test_long_append_bit_exact(name, over, T, plen):
    """Appends longer than the short-append path takes (a block of 37, then 23 tokens): the
    general pipeline with keys encoded against the stored calibration, a first quad that is
    partly filled already, chunks that straddle the call's start."""
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build(name, over, T, plen, extra=64)
    B = w.B
    pos = 0
    for n_add in (37, 23):
        lens = o.len.copy()
        if any(int(lens[b]) + n_add > T + 64 for b in range(B)):
            break
        blk_k = np.stack([K16[b, T + pos: T + pos + n_add] for b in range(B)])
        blk_v = np.stack([V16[b, T + pos: T + pos + n_add] for b in range(B)])
        o.append(blk_k, blk_v, cbK, cbV)
        gpu_quantize(g, dK, dV, blk_k, blk_v)
        compare_cache(g, o, B)
        pos += n_add


@pytest.mark.parametrize("n_add", [1, 5, 40])
def test_append_capacity_overflow(n_add):
    """Lists that fill up during appends (short and general paths): the tokens whose outliers
    do not fit drop them, the count stops at the last kept token, the status bit is set."""
    import long_context_decode_nuq_b200 as K
    w, K16, V16, cbK, cbV, o, g, dK, dV = _build("llama7b_layer_32k", dict(Hq=4, Hkv=4), 120,
                                                  None, extra=128, cap=304)
    assert not o.status & O.STATUS_OUTLIER_OVERFLOW
    pos = 0
    while pos + n_add <= 120 and not o.status & O.STATUS_OUTLIER_OVERFLOW:
        blk_k = K16[:, 120 + pos: 120 + pos + n_add]
        blk_v = V16[:, 120 + pos: 120 + pos + n_add]
        o.append(blk_k, blk_v, cbK, cbV)
        gpu_quantize(g, dK, dV, blk_k, blk_v)
        compare_cache(g, o, w.B)
        pos += n_add
    assert o.status & O.STATUS_OUTLIER_OVERFLOW
    assert K.kvq_get_status(g) & K.KVQ_STATUS_OUTLIER_OVERFLOW


def _plant_specials(K16, V16, seed):
    """Overwrite a seeded scatter of entries with fp16 specials, and make one key channel and
    one token's value row constant (so that their half is 0)."""
    rng = np.random.default_rng(seed)
    specials = np.array([0x7E00, 0xFE00, 0x7C00, 0xFC00, 0x0000, 0x8000, 0x0001, 0x8001, 0x7BFF,
                         0xFBFF, 0x03FF, 0x3C00], dtype=np.uint16)
    for a in (K16, V16):
        flat = a.reshape(-1).view(np.uint16)
        idx = rng.choice(flat.size, size=max(1, flat.size // 400), replace=False)
        flat[idx] = specials[rng.integers(0, specials.size, idx.size)]
    K16[:, :, 0, 5] = np.float16(0.25)      # a constant key channel
    V16[:, 3] = np.float16(-1.5)           # a constant value row
    V16[:, 7, :, :64] = np.float16(np.nan)  # a row whose upper threshold is NaN
    return K16, V16


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_special_values_bit_exact(bits):
    """NaN, infinities, signed zeros, subnormals, fp16 extremes, constant channels and rows:
    prefill, a short append and a long append all match the oracle bit for bit."""
    import oracle as O2
    w = synth.workload("llama7b_layer_32k", Hq=4, Hkv=4, bits=bits)
    T, extra = 190, 64
    K16, V16 = host_block(w, T + extra)
    K16, V16 = _plant_specials(K16.copy(), V16.copy(), 7 + bits)
    cbK, cbV = oracle_codebooks(w)
    cap = 1 << 18
    o = O2.QuantizedCache(w.B, w.Hkv, w.bits, T + extra, w.f, cap, cap)
    o.prefill(K16[:, :T], V16[:, :T], [T] * w.B, cbK, cbV)
    g = gpu_cache(w, T + extra, cap, cap)
    dK, dV = to_dev_codebook(cbK), to_dev_codebook(cbV)
    gpu_quantize(g, dK, dV, K16[:, :T], V16[:, :T], calibrate=1)
    compare_cache(g, o, w.B)
    for lo, hi in ((T, T + 3), (T + 3, T + 44)):
        o.append(K16[:, lo:hi], V16[:, lo:hi], cbK, cbV)
        gpu_quantize(g, dK, dV, K16[:, lo:hi], V16[:, lo:hi])
        compare_cache(g, o, w.B)
