"""Pins for the CPU oracle: closed forms, brute force, library routines, invariants.

Each test ties one oracle function to something other than itself, chosen so a
plausible slip (an off-by-one in k, a dropped term, a wrong sign or pairing, a
transposed operand) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- thresholds (R1, R2, R4)

def test_vector_k_closed_forms():
    # k = floor(f*N/2 + 1/2) at the workloads' vector lengths
    assert O.vector_k(0.01, 2048) == 10      # tiny: key channel over 2048 tokens
    assert O.vector_k(0.01, 128) == 1        # tiny: value row of one head
    assert O.vector_k(0.01, 4096) == 20      # LLaMA-7B value row (32 x 128)
    assert O.vector_k(0.01, 1024) == 5       # Llama-3-8B value row (8 x 128)
    assert O.vector_k(0.005, 4096) == 10     # 1M-token workload value row
    assert O.vector_k(0.005, 1 << 20) == 2621
    assert O.vector_k(0.01, 8192) == 41
    assert O.vector_k(0.0, 4096) == 0
    assert O.vector_k(0.5, 5) == 1
    assert O.vector_k(1.0, 5) == 2           # floor(3.0) capped at (N-1)//2
    assert O.vector_k(0.01, 1) == 0


def test_thresholds_against_sorted_floats():
    rng = np.random.default_rng(1)
    for N, f in [(2048, 0.01), (4096, 0.01), (100, 0.1), (7, 0.3)]:
        x = rng.standard_normal(N).astype(np.float16)
        lo, hi = O.order_stat_thresholds(x, f)
        s = np.sort(x.astype(np.float64))
        k = O.vector_k(f, N)
        assert float(lo) == s[k] and float(hi) == s[N - 1 - k]
        # with distinct values exactly k entries lie strictly below / above
        if len(np.unique(x)) == N:
            assert np.sum(x < lo) == k and np.sum(x > hi) == k


def test_thresholds_total_order_on_zero():
    x = np.array([0.0, -0.0, 1.0, -1.0, 0.0], dtype=np.float16)
    lo, hi = O.order_stat_thresholds(x, 0.0)
    assert lo == np.float16(-1.0) and hi == np.float16(1.0)
    # k = 1 of N = 5: second smallest in total order is -0.0, second largest +0.0
    lo, hi = O.order_stat_thresholds(x, 0.4)
    assert lo.view(np.uint16) == 0x8000 and hi.view(np.uint16) == 0x0000


def test_affine_params_closed_form():
    off, half = O.affine_params(np.float16(-2.0), np.float16(6.0))
    assert off == np.float32(2.0) and half == np.float32(4.0)
    xn = O.normalize(np.array([-2, 6, 2, 4], dtype=np.float16), off, half)
    assert np.array_equal(xn, np.array([-1, 1, 0, 0.5], dtype=np.float32))
    assert O.normalize(np.float16(3.0), np.float32(1.0), np.float32(0.0)) == 0.0


# ---------------------------------------------------------------- encode / datatype (R6, R7)

def test_encode_is_nearest_level():
    levels = np.array([-0.9, -0.5, -0.2, 0.0, 0.15, 0.4, 0.7, 1.0], dtype=np.float32)
    bounds = ((levels[:-1].astype(np.float64) + levels[1:]) / 2).astype(np.float32)
    xn = np.random.default_rng(2).uniform(-1.2, 1.2, 100000).astype(np.float32)
    code = O.encode(xn, bounds)
    brute = np.argmin(np.abs(xn[:, None].astype(np.float64) - levels[None, :]), axis=1)
    near_mid = np.min(np.abs(xn[:, None] - bounds[None, :]), axis=1) < 1e-6
    assert np.array_equal(code[~near_mid], brute[~near_mid])
    # ties go to the lower code
    assert O.encode(bounds[3:4], bounds)[0] == 3


def test_uniform_grid_reduces_to_round_to_nearest():
    K = 8
    levels = (-1 + (2 * np.arange(K) + 1) / K).astype(np.float32)    # uniform mid-rise grid
    bounds = ((levels[:-1].astype(np.float64) + levels[1:]) / 2).astype(np.float32)
    xn = np.random.default_rng(3).uniform(-1, 1, 50000).astype(np.float32)
    code = O.encode(xn, bounds)
    rtn = np.clip(np.floor((xn.astype(np.float64) + 1) * K / 2), 0, K - 1)
    assert np.array_equal(code, rtn.astype(np.uint8))


def _dp_kmeans_cost(x, w, K):
    """Exact weighted 1-D k-means cost by dynamic programming over sorted points."""
    o = np.argsort(x)
    x, w = x[o], w[o]
    n = len(x)
    W = np.concatenate([[0], np.cumsum(w)])
    S = np.concatenate([[0], np.cumsum(w * x)])
    Q = np.concatenate([[0], np.cumsum(w * x * x)])

    def cost(i, j):  # points i..j-1
        ww = W[j] - W[i]
        s = S[j] - S[i]
        return (Q[j] - Q[i]) - s * s / ww

    INF = float("inf")
    dp = np.full((K + 1, n + 1), INF)
    dp[0, 0] = 0.0
    for k in range(1, K + 1):
        for j in range(k, n + 1):
            dp[k, j] = min(dp[k - 1, i] + cost(i, j) for i in range(k - 1, j))
    return dp[K, n]


def _lloyd_cost(x, w, c):
    d = (x[:, None] - c[None, :]) ** 2
    return float(np.sum(w * d.min(axis=1)))


def test_kmeans_against_exact_dp():
    rng = np.random.default_rng(4)
    for trial in range(4):
        x = rng.standard_normal(60)
        w = rng.uniform(0.2, 3.0, 60)
        c = O.kmeans_1d_weighted(x, w, 4)
        opt = _dp_kmeans_cost(x, w, 4)
        got = _lloyd_cost(x, w, c)
        assert got >= opt - 1e-9
        assert got <= 1.25 * opt + 1e-9          # Lloyd from quantile init stays close
    # well-separated clusters with known centres: Lloyd reaches the optimum
    centres = np.array([-3.0, -1.0, 1.5, 4.0])
    x = np.concatenate([cc + 0.05 * rng.standard_normal(40) for cc in centres])
    w = rng.uniform(0.5, 2.0, x.size)
    c = O.kmeans_1d_weighted(x, w, 4)
    assert abs(_lloyd_cost(x, w, c) - _dp_kmeans_cost(x, w, 4)) < 1e-9
    assert np.allclose(c, centres, atol=0.05)


def test_kmeans_fixed_point_and_weight_scale():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(3000)
    w = rng.uniform(0.1, 2.0, 3000)
    c = O.kmeans_1d_weighted(x, w, 8)
    a = np.argmin(np.abs(x[:, None] - c[None, :]), axis=1)
    for j in range(8):       # each centroid is the weighted mean of its own cell
        m = a == j
        assert abs(c[j] - np.dot(w[m], x[m]) / w[m].sum()) < 1e-12
    c2 = O.kmeans_1d_weighted(x, 4.0 * w, 8)    # power-of-two scale: exact invariance
    assert np.array_equal(c, c2)


def test_kmeans_uniform_closed_form():
    # k-means of U(-1, 1) with K cells: centroids at -1 + (2j+1)/K
    x = np.linspace(-1, 1, 20001)
    c = O.kmeans_1d_weighted(x, np.ones_like(x), 8, max_iter=300)
    assert np.allclose(c, -1 + (2 * np.arange(8) + 1) / 8, atol=2e-3)


def test_db16_rounding_brute_force():
    vals = np.array([(u << 16) | u for u in range(1 << 16)], dtype=np.uint32).view(np.float32)
    ok = np.isfinite(vals)
    vals64 = vals[ok].astype(np.float64)
    rng = np.random.default_rng(6)
    for x in np.concatenate([rng.uniform(-1, 1, 300), [0.0, 1e-30, -0.7]]):
        r = O.round_db16(x)
        bits = int(np.array([r], dtype=np.float32).view(np.uint32)[0])
        assert (bits >> 16) == (bits & 0xFFFF)
        d = np.abs(vals64 - x)
        assert abs(float(r) - x) == d.min()


def test_fitted_codebook_properties():
    w = synth.workload("llama7b_layer_32k")
    lev, bnd = O.fit_codebook(synth.codebook_samples_v(w), w.f, 3)
    assert lev.dtype == np.float32 and lev.size == 8 and bnd.size == 7
    assert np.all(np.diff(lev) > 0) and np.all(lev >= -1) and np.all(lev <= 1)
    assert np.all((lev[:-1] < bnd) & (bnd < lev[1:]))
    # normal-ish data normalized to [-1, 1]: roughly symmetric levels
    assert abs(lev[0] + lev[-1]) < 0.1


# ---------------------------------------------------------------- packing (R8)

def _spec(spec):
    codes = np.zeros(128, dtype=np.uint8)
    for item in spec.split(","):
        if item:
            ch, cd = item.split(":")
            codes[int(ch)] = int(cd)
    return codes


def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "pack_rows.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            kind, bits, spec = lhs.split(None, 2)
            assert kind == "b"
            words = [int(x, 16) if x.startswith("0x") else int(x) for x in rhs.split()]
            toks = [_spec(x.strip()) for x in spec.split("/")]
            assert len(toks) == 4
            rows.append((int(bits), toks, np.array(words, dtype=np.uint32)))
    return rows


def test_pack_golden_rows():
    rows = _golden_rows()
    assert sorted(r[0] for r in rows) == [2, 3, 4]
    for bits, toks, words in rows:
        got = O.pack_block(toks, bits)
        assert got.shape == (16 * bits,)
        assert np.array_equal(got, words), (bits, [hex(x) for x in got])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip_and_bit_budget(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(4, 50, 128)).astype(np.uint8)
    assert np.array_equal(O.unpack_block(O.pack_block(codes, bits), bits), codes)
    full = np.full(128, (1 << bits) - 1, dtype=np.uint8)
    assert np.all(O.pack_block([full] * 4, bits) == 0xFFFFFFFF)
    # single codes touch disjoint bits (each bit of a block is used exactly once)
    zero = np.zeros(128, dtype=np.uint8)
    acc = np.zeros(16 * bits, dtype=np.uint64)
    for ch in range(128):
        for j in range(4):
            one = zero.copy()
            one[ch] = (1 << bits) - 1
            quad = [one if jj == j else zero for jj in range(4)]
            w = O.pack_block(quad, bits).astype(np.uint64)
            assert not np.any(acc & w)
            acc |= w
            # channel c lives in the words of lane group c % 16 only
            nz = np.nonzero(w)[0]
            assert np.all(nz // bits == (ch % 64) % 16)


# ---------------------------------------------------------------- quantizer invariants

def _gen_block(w, T):
    idx = (np.arange(w.B)[:, None, None, None], np.arange(T)[None, :, None, None],
           np.arange(w.Hkv)[None, None, :, None], np.arange(w.D)[None, None, None, :])
    return synth.gen_k(w, 0, *idx), synth.gen_v(w, 0, *idx)


def _small_cache(w, T, plen=None, cap=1 << 20):
    K, V = _gen_block(w, T + 8)
    cbK = O.fit_codebook(synth.codebook_samples_k(w), w.f, w.bits)
    cbV = O.fit_codebook(synth.codebook_samples_v(w), w.f, w.bits)
    c = O.QuantizedCache(w.B, w.Hkv, w.bits, T + 8, w.f, cap, cap)
    c.prefill(K, V, plen if plen is not None else [T] * w.B, cbK, cbV)
    return c, K, V, cbK, cbV


def test_outliers_roundtrip_and_lie_outside():
    w = synth.workload("llama7b_layer_32k", Hq=4, Hkv=4)
    T = 300
    c, K, V, cbK, cbV = _small_cache(w, T)
    Kh, Vh = c.dequantize(0, cbK, cbV)
    lo = c.kthr[0, :, 0].view(np.float16)
    hi = c.kthr[0, :, 1].view(np.float16)
    ent = c.outlier_entries("k", 0)
    assert len(ent) == int(c.out_count["k"][0].sum()) > 0
    for t, j, bits in ent:
        x = K[0, t].reshape(-1)[j]
        assert x.view(np.uint16) == bits                       # stored fp16 unchanged
        assert x < lo[j] or x > hi[j]                          # strictly outside
        assert Kh[t].reshape(-1)[j].view(np.uint16) == bits    # round-trips bit-exactly
    # per-channel count: exactly 2k per key channel when its values are distinct
    Kf = K[0, :T].reshape(T, -1)
    k = O.vector_k(w.f, T)
    counts = np.bincount([j for _, j, _ in ent], minlength=c.n)
    distinct = np.array([len(np.unique(Kf[:, j])) == T for j in range(c.n)])
    assert np.all(counts[distinct] == 2 * k)
    # values: 2k_v per token when the row is distinct
    kv = O.vector_k(w.f, c.n)
    vent = c.outlier_entries("v", 0)
    vcount = np.bincount([t for t, _, _ in vent], minlength=T)
    Vf = V[0, :T].reshape(T, -1)
    dist_rows = np.array([len(np.unique(Vf[t])) == c.n for t in range(T)])
    assert np.all(vcount[dist_rows] == 2 * kv)
    for t, j, bits in vent:
        assert Vh[t].reshape(-1)[j].view(np.uint16) == bits


def test_zero_outlier_fraction_stores_none():
    w = synth.workload("tiny_single_head", f=0.0)
    c, K, V, cbK, cbV = _small_cache(w, 200)
    assert c.out_count["k"][0].sum() == 0 and c.out_count["v"][0].sum() == 0
    lo = c.kthr[0, :, 0].view(np.float16)
    assert np.array_equal(lo, K[0, :200, 0].min(axis=0))


def test_dense_error_bound_and_exact_lookup():
    w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2)
    T = 256
    c, K, V, cbK, cbV = _small_cache(w, T)
    lev = cbK[0].astype(np.float64)
    # worst normalized error: half the widest inner gap, or the distance from the
    # range ends (-1, 1) to the outer levels
    worst = max(np.max(np.diff(lev)) / 2, lev[0] + 1.0, 1.0 - lev[-1])
    Kh, _ = c.dequantize(0, cbK, cbV)
    half = c.kparams[0, :, 1].astype(np.float64)
    err = np.abs(Kh.reshape(T, -1).astype(np.float64) - K[0, :T].reshape(T, -1))
    bound = half * (worst + 1e-6) + np.abs(K[0, :T].reshape(T, -1).astype(np.float64)) * 2 ** -10
    assert np.all(err <= bound)
    # off = 0, half = 1: dequantization returns the level itself
    codes = np.arange(8)
    assert np.array_equal(O.dequant_dense(codes, np.float32(0), np.float32(1), cbK[0]),
                          cbK[0].astype(np.float16))


def test_quantizer_matches_per_element_brute_force():
    """Loops over single elements with Python floats, independent of the vectorized path."""
    w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2, f=0.02)
    T = 40
    c, K, V, cbK, cbV = _small_cache(w, T)
    n = c.n
    Kf = K[0, :T].reshape(T, n)
    Vf = V[0, :T].reshape(T, n)

    def nearest(xn, bounds):
        code = 0
        for bnd in bounds:
            if xn > bnd:
                code += 1
        return code

    f32 = np.float32
    for j in range(0, n, 17):
        col = sorted(Kf[:, j].tolist())
        k = int(math.floor(w.f * T * 0.5 + 0.5))
        lo, hi = col[k], col[T - 1 - k]
        off = (f32(lo) + f32(hi)) * f32(0.5)
        half = (f32(hi) - f32(lo)) * f32(0.5)
        for t in range(0, T, 7):
            x = Kf[t, j]
            xv = 0.0 if (x < lo or x > hi) else float(x)
            xn = (f32(xv) - off) / half
            assert c.kc[0, t, j] == nearest(xn, cbK[1])
    for t in range(0, T, 5):
        row = sorted(Vf[t].tolist())
        k = int(math.floor(w.f * n * 0.5 + 0.5))
        lo, hi = row[k], row[n - 1 - k]
        off = (f32(lo) + f32(hi)) * f32(0.5)
        half = (f32(hi) - f32(lo)) * f32(0.5)
        assert c.vparams[0, t, 0] == off and c.vparams[0, t, 1] == half
        for j in range(0, n, 13):
            x = Vf[t, j]
            xv = 0.0 if (x < lo or x > hi) else float(x)
            assert c.vc[0, t, j] == nearest((f32(xv) - off) / half, cbV[1])


def test_append_reuses_key_calibration_and_chunks():
    w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2)
    T = 130
    c, K, V, cbK, cbV = _small_cache(w, T)
    before = c.kparams.copy()
    for i in range(3):
        c.append(K[:, T + i: T + i + 1], V[:, T + i: T + i + 1], cbK, cbV)
    assert np.array_equal(before, c.kparams)
    assert c.len[0] == T + 3
    # chunk pointers are monotone and end at the count
    nch = (T + 3 + 63) // 64
    for h in range(w.Hkv):
        cp = c.chunk_ptr["k"][0, h]
        assert np.all(np.diff(cp[: nch + 1].astype(np.int64)) >= 0)
        assert cp[nch] == c.out_count["k"][0, h]
    # appending token by token equals prefill-then-quantize of the same tokens
    c2 = O.QuantizedCache(w.B, w.Hkv, w.bits, T + 8, w.f, 1 << 20, 1 << 20)
    c2.calibrate_keys(0, K[0, :T])
    c2.quantize_tokens(0, 0, K[0, : T + 3], V[0, : T + 3], cbK, cbV)
    nq = (T + 3 + 3) // 4
    assert np.array_equal(c2.kcodes[0, :nq], c.kcodes[0, :nq])
    assert np.array_equal(c2.vcodes[0, :nq], c.vcodes[0, :nq])
    for s in ("k", "v"):
        assert np.array_equal(c2.out[s][0], c.out[s][0])
        assert np.array_equal(c2.chunk_ptr[s][0, :, : nch + 1], c.chunk_ptr[s][0, :, : nch + 1])


def test_overflow_rule_prefix():
    """Per (sequence, head) list: a token's outliers are kept iff the prefix fits."""
    w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2)
    T = 100
    cap = 152
    c, K, V, cbK, cbV = _small_cache(w, T, cap=cap)
    assert c.status & O.STATUS_OUTLIER_OVERFLOW
    full, _, _, _, _ = _small_cache(w, T)
    for s in ("k", "v"):
        ent = full.outlier_entries(s, 0)
        for h in range(w.Hkv):
            per_tok = np.bincount([t for t, j, _ in ent if j // w.D == h], minlength=T)
            stop = int(np.searchsorted(np.cumsum(per_tok), cap, side="right"))
            n_kept = int(per_tok[:stop].sum())
            assert c.out_count[s][0, h] == n_kept
            assert np.array_equal(c.out[s][0, h, :n_kept], full.out[s][0, h, :n_kept])
    # the cap binds on at least one list, and a list under the cap is unaffected
    assert any(full.out_count[s][0, h] > cap for s in ("k", "v") for h in range(w.Hkv))


# ---------------------------------------------------------------- RoPE (R9)

def test_rope_closed_form_and_pairing():
    D, base = 8, 10000.0
    th = O.rope_freqs(D, base)
    assert np.allclose(th, [1.0, 0.1, 0.01, 0.001])
    x = np.zeros(D)
    x[1] = 1.0                                # first half, pair 1
    r = O.rope_rotate(x, 3.0, base)
    want = np.zeros(D)
    want[1], want[5] = math.cos(0.3), math.sin(0.3)
    assert np.allclose(r, want, atol=1e-15)
    y = np.zeros(D)
    y[5] = 1.0                                # second half of pair 1
    r = O.rope_rotate(y, 3.0, base)
    want = np.zeros(D)
    want[1], want[5] = -math.sin(0.3), math.cos(0.3)
    assert np.allclose(r, want, atol=1e-15)


def test_rope_invariants():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((5, 128))
    assert np.allclose(O.rope_rotate(x, 0, 1e4), x, atol=0)
    r = O.rope_rotate(x, 123456.0, 1e4)
    assert np.allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    d1 = O.rope_rotate(q, 1000, 1e4) @ O.rope_rotate(k, 37, 1e4)
    d2 = O.rope_rotate(q, 1500, 1e4) @ O.rope_rotate(k, 537, 1e4)
    assert abs(d1 - d2) < 1e-10


# ---------------------------------------------------------------- attention (R10)

def _brute_attention(q16, qpos, Kh, Vh, base):
    """Scalar loops: explicit 2x2 rotations per pair, math.exp softmax."""
    Hq, D = q16.shape
    T, Hkv, _ = Kh.shape
    g = Hq // Hkv
    h2 = D // 2
    out = np.zeros((Hq, D))
    logits = np.zeros((Hq, T))

    def rot(vec, pos):
        res = [0.0] * D
        for i in range(h2):
            ang = pos * base ** (-2.0 * i / D)
            a, b = float(vec[i]), float(vec[i + h2])
            res[i] = a * math.cos(ang) - b * math.sin(ang)
            res[i + h2] = a * math.sin(ang) + b * math.cos(ang)
        return res

    for hq in range(Hq):
        h = hq // g
        qr = rot(q16[hq], qpos)
        for t in range(T):
            kr = rot(Kh[t, h], t)
            logits[hq, t] = sum(a * b for a, b in zip(qr, kr)) / math.sqrt(D)
        m = max(logits[hq])
        e = [math.exp(v - m) for v in logits[hq]]
        s = sum(e)
        for t in range(T):
            for c in range(D):
                out[hq, c] += e[t] / s * float(Vh[t, h, c])
    return logits, out


def test_attention_matches_brute_force_gqa():
    rng = np.random.default_rng(9)
    T, Hkv, Hq, D = 6, 2, 4, 128
    Kh = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    Vh = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    q = rng.standard_normal((Hq, D)).astype(np.float16)
    lg, p, o = O.decode_attention(q, 9, Kh, Vh, 1e4)
    blg, bo = _brute_attention(q, 9, Kh, Vh, 1e4)
    assert np.allclose(lg, blg, atol=1e-12)
    assert np.allclose(o, bo, atol=1e-12)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)


def test_attention_against_torch_sdpa():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(10)
    T, H, D = 50, 3, 128
    Kh = rng.standard_normal((T, H, D)).astype(np.float16)
    Vh = rng.standard_normal((T, H, D)).astype(np.float16)
    q = rng.standard_normal((H, D)).astype(np.float16)
    lg, p, o = O.decode_attention(q, 50, Kh, Vh, 1e4)
    kr = np.stack([O.rope_rotate(Kh[:, h].astype(np.float64), np.arange(T), 1e4)
                   for h in range(H)])
    qr = O.rope_rotate(q.astype(np.float64), 50, 1e4)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qr)[:, None, :], torch.from_numpy(kr),
        torch.from_numpy(Vh.astype(np.float64).transpose(1, 0, 2)))
    assert np.allclose(o, ref[:, 0, :].numpy(), atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(11)
    T, D = 20, 128
    k = rng.standard_normal(D).astype(np.float16)
    Vh = rng.standard_normal((T, 1, D)).astype(np.float16)
    q = np.zeros((1, D), dtype=np.float16)        # zero query: uniform weights
    _, p, o = O.decode_attention(q, 5, np.tile(k, (T, 1))[:, None, :], Vh, 1e4)
    assert np.allclose(p, 1.0 / T, atol=1e-15)
    assert np.allclose(o[0], Vh[:, 0].astype(np.float64).mean(axis=0), atol=1e-12)
    # one key aligned with a large query dominates: output is that value row
    Kh = (0.01 * rng.standard_normal((T, 1, D))).astype(np.float16)
    Kh[7, 0] = np.float16(8.0)
    q = np.full((1, D), 8.0, dtype=np.float16)
    _, p, o = O.decode_attention(q, 7, Kh, Vh, 1e4)
    assert p[0, 7] > 1 - 1e-12
    assert np.allclose(o[0], Vh[7, 0].astype(np.float64), atol=1e-9)


def test_split_merge_independent_of_split_count():
    rng = np.random.default_rng(12)
    T, D = 333, 128
    lg = rng.standard_normal(T) * 5
    V = rng.standard_normal((T, D))
    p = np.exp(lg - lg.max())
    p /= p.sum()
    ref = p @ V
    for S in (1, 2, 7, 64, 400):
        o, M, L = O.merge_splits(lg, V, S)
        assert np.allclose(o, ref, atol=1e-12)
        assert M == lg.max()


def test_dequantize_then_attend_end_to_end():
    """Oracle pipeline on the tiny workload: quantize, dequantize, attend."""
    w = synth.workload("tiny_single_head")
    c, K, V, cbK, cbV = _small_cache(w, 512)
    Kh, Vh = c.dequantize(0, cbK, cbV)
    q = synth.gen_q(w)[0]
    lg, p, o = O.decode_attention(q, 512, Kh, Vh, w.rope_theta)
    lgx, px, ox = O.decode_attention(q, 512, K[0, :512], V[0, :512], w.rope_theta)
    assert np.isfinite(o).all() and abs(p.sum() - 1) < 1e-12
    # 3-bit + 1% outliers stays close to the unquantized attention
    assert np.corrcoef(lg[0], lgx[0])[0, 1] > 0.98


def test_reconstruct_is_exact_affine_and_rounds_to_dequantize():
    """Exact reconstruction: off + half * L in binary64; rounding it gives the fp16 dequant
    except where binary32 multiply-then-add rounding differs (double rounding), and the
    outliers are identical in both."""
    w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2)
    T = 200
    c, K, V, cbK, cbV = _small_cache(w, T)
    Kx, Vx = c.reconstruct(0, cbK, cbV)
    Kh, Vh = c.dequantize(0, cbK, cbV)
    j = 77
    t = 13
    code = int(c.kc[0, t, j])
    want = float(c.kparams[0, j, 0]) + float(c.kparams[0, j, 1]) * float(cbK[0][code])
    if not any(tt == t and jj == j for tt, jj, _ in c.outlier_entries("k", 0)):
        assert Kx.reshape(T, -1)[t, j] == want
    for X, H in ((Kx, Kh), (Vx, Vh)):
        r = X.astype(np.float32).astype(np.float16)
        assert np.mean(r == H) > 0.999
        assert np.abs(X - H.astype(np.float64)).max() <= np.abs(X).max() * 2 ** -10
    for t_, j_, bits in c.outlier_entries("v", 0):
        assert Vx.reshape(T, -1)[t_, j_] == float(np.uint16(bits).view(np.float16))


# ---------------------------------------------------------------------------------------------
# Token-range partials and their merge (the token-sharded decode)


def test_partials_of_any_split_merge_to_the_whole():
    rng = np.random.default_rng(11)
    T, Hkv, Hq, D = 300, 2, 4, 128
    Kh = rng.standard_normal((T, Hkv, D))
    Vh = rng.standard_normal((T, Hkv, D))
    q = rng.standard_normal((Hq, D)).astype(np.float16)
    _, _, ref = O.decode_attention(q, T, Kh, Vh, 1e4)
    for cuts in ([0, 300], [0, 64, 300], [0, 0, 100, 250, 300], [0, 299, 300]):
        parts = [O.partial_attention(q, T, Kh[a:b], Vh[a:b], 1e4, np.arange(a, b))
                 for a, b in zip(cuts[:-1], cuts[1:])]
        M, L, o = (np.stack(x) for x in zip(*parts))
        assert np.abs(O.merge_partials(M, L, o) - ref).max() < 1e-12
    # an empty range contributes nothing
    M, L, o = O.partial_attention(q, T, Kh[:0], Vh[:0], 1e4, np.arange(0))
    assert np.all(M == -np.inf) and not L.any() and not o.any()


def test_key_positions_shift_with_the_query():
    # RoPE logits depend only on (query position - key position)
    rng = np.random.default_rng(12)
    T, D = 50, 128
    Kh = rng.standard_normal((T, 1, D))
    Vh = rng.standard_normal((T, 1, D))
    q = rng.standard_normal((1, D)).astype(np.float16)
    a = O.decode_attention(q, T, Kh, Vh, 1e4)
    b = O.decode_attention(q, T + 1000, Kh, Vh, 1e4, kpos=np.arange(T) + 1000)
    assert np.abs(a[0] - b[0]).max() < 1e-9
    assert np.abs(a[2] - b[2]).max() < 1e-9
