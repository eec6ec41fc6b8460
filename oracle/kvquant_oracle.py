"""Plain, slow CPU oracle of the KVQuant quantized decode path (numpy).

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA library; it is
imported by ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
leg of ``bench.py`` and by nothing else.  It shares no code with the CUDA path.

Sources (pages on KVQuant, arXiv 2401.18079):
  * "KVQuant: Towards 10 Million Context Length LLM Inference with KV Cache
    Quantization" (study.space summary) -- techniques (i) per-channel key
    quantization, (ii) pre-RoPE key quantization, (iii) per-layer
    sensitivity-weighted non-uniform datatypes, (iv) per-vector
    dense-and-sparse quantization; long-context decode is memory and
    bandwidth bound.
  * "KVQuant" research note (phantomic12), Four components (1)-(4): keys are
    quantized along the channel dimension, before RoPE, onto a per-layer
    non-uniform datatype, with outliers isolated per vector rather than
    globally; 3-bit vs fp16 is a ~5.3x cache reduction.

Where the pages leave a step open the plain reading below is used; each has an
ID (R1-R10) by which the CUDA library's notes refer to it:
  R1 vector: a key vector is one channel (b, h, c) over the calibration tokens;
     a value vector is one token's full row over all kv heads (n = Hkv*D).
  R2 outlier count: k = floor(f*N/2 + 1/2) per side (capped at (N-1)//2);
     t_lo = s[k], t_hi = s[N-1-k] of the ascending sort (IEEE total order on
     fp16, so -0 < +0); an entry is an outlier iff x < t_lo or x > t_hi.
  R3 appended keys reuse the calibration thresholds and scales.
  R4 normalization: off = (t_lo + t_hi)*0.5, half = (t_hi - t_lo)*0.5,
     xn = (x - off)/half, all binary32 round-to-nearest; xn = 0 if half == 0.
  R5 dense remainder: outlier positions are set to 0 before encoding;
     reconstruction replaces them with the stored fp16 value.  The
     reconstruction used by attention is exact: x = off + half * L[code] in real
     arithmetic on the stored binary32 values (binary64 here); rounding it to
     fp16 is only the format of the dequantized-cache output.
  R6 encode: code = #{j : xn > bounds[j]} (ties go to the lower code).
  R7 codebook: weighted 1-D Lloyd k-means in binary64 (init at weighted
     quantiles (j+1/2)/K, nearest-centroid assignment with ties to the lower
     index, weighted-mean update, empty cells keep their value, stop when the
     assignment repeats or after 100 iterations); levels are then rounded to
     the nearest "DB16" binary32 value (bit pattern (u << 16) | u) and
     bounds[j] = binary32((L_j + L_{j+1})/2).
  R8 packing: see pack_block (a layout of this implementation, shared by keys
     and values: 4-token blocks per kv head).
  R9 RoPE: rotate-half pairs (i, i + D/2), theta_i = base^(-2i/D), 0-based
     positions; the query is rotated at its own position.
  R10 scale 1/sqrt(D); every cached token is visible; kv head = hq // (Hq/Hkv).
"""
from __future__ import annotations

import math

import numpy as np

CHUNK = 64                      # tokens per outlier chunk
STATUS_OUTLIER_OVERFLOW = 1     # sticky status bit: an outlier list was full

# ----------------------------------------------------------------------------------------
# Per-vector thresholds and the affine map (techniques (i) and (iv); readings R1-R4)
# ----------------------------------------------------------------------------------------


def vector_k(f: float, N: int) -> int:
    """Outliers kept per side of a vector of N values (reading R2)."""
    if N <= 0:
        return 0
    k = int(math.floor(f * N * 0.5 + 0.5))
    return min(k, (N - 1) // 2)


def fp16_order_key(bits: np.ndarray) -> np.ndarray:
    """Map fp16 bit patterns to uint16 keys whose unsigned order is IEEE total order."""
    bits = np.asarray(bits, dtype=np.uint16)
    neg = (bits & np.uint16(0x8000)) != 0
    return np.where(neg, ~bits, bits | np.uint16(0x8000)).astype(np.uint16)


def fp16_from_order_key(key: np.ndarray) -> np.ndarray:
    """Inverse of fp16_order_key (returns fp16 values)."""
    key = np.asarray(key, dtype=np.uint16)
    pos = (key & np.uint16(0x8000)) != 0
    bits = np.where(pos, key ^ np.uint16(0x8000), ~key).astype(np.uint16)
    return bits.view(np.float16)


def order_stat_thresholds(x16: np.ndarray, f: float, axis: int = -1):
    """(t_lo, t_hi) of vectors of fp16 values along ``axis``, as fp16 (reading R2)."""
    x16 = np.asarray(x16, dtype=np.float16)
    N = x16.shape[axis]
    if N == 0:
        shp = x16.shape[:axis % x16.ndim] + x16.shape[axis % x16.ndim + 1:]
        z = np.zeros(shp, dtype=np.float16)
        return z, z.copy()
    k = vector_k(f, N)
    keys = np.sort(fp16_order_key(x16.view(np.uint16)), axis=axis)
    lo = np.take(keys, k, axis=axis)
    hi = np.take(keys, N - 1 - k, axis=axis)
    return fp16_from_order_key(lo), fp16_from_order_key(hi)


def affine_params(t_lo, t_hi):
    """(off, half) in binary32 from fp16 thresholds (reading R4)."""
    lo = np.float32(t_lo)
    hi = np.float32(t_hi)
    off = (lo + hi) * np.float32(0.5)
    half = (hi - lo) * np.float32(0.5)
    return np.float32(off), np.float32(half)


def normalize(x16, off, half):
    """xn = (x - off) / half in binary32; 0 where half == 0 (reading R4)."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    off = np.asarray(off, dtype=np.float32)
    half = np.asarray(half, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        xn = (x - off) / half
    return np.where(half == np.float32(0.0), np.float32(0.0), xn).astype(np.float32)


def encode(xn, bounds):
    """NUQ code = number of decision bounds strictly below xn (reading R6)."""
    xn = np.asarray(xn, dtype=np.float32)
    b = np.asarray(bounds, dtype=np.float32)
    return (xn[..., None] > b).sum(axis=-1).astype(np.uint8)


def dequant_dense(code, off, half, levels):
    """fp16(off + half * L[code]) with binary32 multiply then add."""
    L = np.asarray(levels, dtype=np.float32)[np.asarray(code, dtype=np.int64)]
    prod = np.asarray(half, dtype=np.float32) * L
    return (np.asarray(off, dtype=np.float32) + prod).astype(np.float32).astype(np.float16)


# ----------------------------------------------------------------------------------------
# Non-uniform datatype (technique (iii); reading R7)
# ----------------------------------------------------------------------------------------


def kmeans_1d_weighted(x, w, K, max_iter=100):
    """Weighted 1-D Lloyd iterations in binary64; returns K sorted centroids."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    order = np.argsort(x, kind="stable")
    xs, ws = x[order], w[order]
    cw = np.cumsum(ws)
    W = cw[-1]
    c = np.empty(K, dtype=np.float64)
    for j in range(K):
        target = (j + 0.5) / K * W
        c[j] = xs[int(np.searchsorted(cw, target, side="left"))]
    prev = None
    for _ in range(max_iter):
        a = np.argmin(np.abs(xs[:, None] - c[None, :]), axis=1)
        if prev is not None and np.array_equal(a, prev):
            break
        for j in range(K):
            m = a == j
            if m.any():
                c[j] = np.sum(ws[m] * xs[m]) / np.sum(ws[m])
        prev = a
    return np.sort(c)


def db16_value(u: int) -> np.float32:
    """The binary32 value whose bit pattern is (u << 16) | u."""
    return np.array([(u << 16) | u], dtype=np.uint32).view(np.float32)[0]


def round_db16(x: float) -> np.float32:
    """Nearest DB16 value to x (ties to the smaller value)."""
    u0 = int(np.array([x], dtype=np.float32).view(np.uint32)[0] >> 16)
    cands = {u0, (u0 + 1) & 0xFFFF, (u0 - 1) & 0xFFFF, 0x0000, 0x8000}
    best, best_d = None, None
    for u in sorted(cands):
        if (u & 0x7F80) == 0x7F80:      # Inf/NaN patterns are not levels
            continue
        v = float(db16_value(u))
        d = abs(v - x)
        if best is None or d < best_d or (d == best_d and v < float(best)):
            best, best_d = db16_value(u), d
    return np.float32(best)


def codebook_from_centroids(c):
    """Levels (DB16 binary32, ascending) and decision bounds (binary32)."""
    levels = np.array([round_db16(v) for v in np.sort(np.asarray(c, dtype=np.float64))],
                      dtype=np.float32)
    if np.any(np.diff(levels.astype(np.float64)) <= 0):
        raise ValueError("codebook levels collapse after rounding")
    lv = levels.astype(np.float64)
    bounds = ((lv[:-1] + lv[1:]) * 0.5).astype(np.float32)
    return levels, bounds


def fit_codebook(samples16, f, bits, weights=None, max_iter=100):
    """Per-layer NUQ codebook from raw fp16 sample vectors.

    Each row of ``samples16`` is one vector; it is thresholded and normalized by
    its own order statistics (R2, R4), its outliers are dropped, and the pooled
    normalized values are fitted by weighted k-means (R7).  ``weights`` (same
    shape as ``samples16``) are the per-sample sensitivity weights; None means
    unit weights.
    """
    samples16 = np.asarray(samples16, dtype=np.float16)
    if samples16.ndim == 1:
        samples16 = samples16[None, :]
    if weights is None:
        weights = np.ones(samples16.shape, dtype=np.float64)
    xs, ws = [], []
    for row, wrow in zip(samples16, np.asarray(weights, dtype=np.float64)):
        lo, hi = order_stat_thresholds(row, f)
        off, half = affine_params(lo, hi)
        keep = (row >= lo) & (row <= hi)
        xs.append(normalize(row[keep], off, half).astype(np.float64))
        ws.append(wrow[keep])
    c = kmeans_1d_weighted(np.concatenate(xs), np.concatenate(ws), 1 << bits, max_iter)
    return codebook_from_centroids(c)


# ----------------------------------------------------------------------------------------
# Packing (reading R8)
# ----------------------------------------------------------------------------------------


def block_words(bits: int, D: int = 128) -> int:
    """Words of one code block (four tokens, one kv head)."""
    return 4 * D * bits // 32


def _field_offsets(bits):
    """Code block: (channel c < 64, token j of the quad, bit offset of its 2*bits field).

    Lane group i in [0, 16) owns words [bits*i, bits*i + bits) and the rotate-half
    pairs (c, c + 64) for c = i + 16k (k in [0, 4)).  In the group's bit string, slot
    f = 4k + s sits at bit 2*bits*f and holds the field code(4u + j, c) | code(4u + j,
    c + 64) << bits of token j = s XOR (i >> 2) (the token order within a slot row is
    rotated per lane group).  Keys and values use the same block.
    """
    return [(i + 16 * k, s ^ (i >> 2), 32 * bits * i + 2 * bits * (4 * k + s))
            for i in range(16) for k in range(4) for s in range(4)]


def _put_field(out, field, off, width):
    w, s = divmod(off, 32)
    out[..., w] |= (field << np.uint64(s)) & np.uint64(0xFFFFFFFF)
    if s + width > 32:
        out[..., w + 1] |= field >> np.uint64(32 - s)


def _get_field(words, off, width):
    w, s = divmod(off, 32)
    v = words[..., w] >> np.uint64(s)
    if s + width > 32:
        v = v | (words[..., w + 1] << np.uint64(32 - s))
    return v & np.uint64((1 << width) - 1)


def pack_block(codes, bits):
    """Code block of a token quad: codes [4, ..., 128] (token j of the quad first) ->
    [..., 16*bits] words."""
    cs = [np.asarray(c, dtype=np.uint64) for c in codes]
    assert len(cs) == 4 and all(c.shape == cs[0].shape for c in cs) and cs[0].shape[-1] == 128
    out = np.zeros(cs[0].shape[:-1] + (block_words(bits),), dtype=np.uint64)
    for c, j, off in _field_offsets(bits):
        _put_field(out, cs[j][..., c] | (cs[j][..., c + 64] << np.uint64(bits)), off, 2 * bits)
    return out.astype(np.uint32)


def unpack_block(words, bits):
    """Inverse of pack_block: words [..., 16*bits] -> codes [4, ..., 128] (uint8)."""
    words = np.asarray(words, dtype=np.uint64)
    codes = np.zeros((4,) + words.shape[:-1] + (128,), dtype=np.uint8)
    mask = np.uint64((1 << bits) - 1)
    for c, j, off in _field_offsets(bits):
        f = _get_field(words, off, 2 * bits)
        codes[j][..., c] = (f & mask).astype(np.uint8)
        codes[j][..., c + 64] = ((f >> np.uint64(bits)) & mask).astype(np.uint8)
    return codes


# ----------------------------------------------------------------------------------------
# The quantized cache (techniques (i), (ii), (iv) on the write side)
# ----------------------------------------------------------------------------------------


class QuantizedCache:
    """Mirror of the device cache arrays, filled by the oracle's quantizer.

    Code blocks are stored head-major: kcodes[b, h, u] is the block of token quad u
    of kv head h.  Outliers are kept in one list per (sequence, kv head) for keys
    and one for values.  A list holds entries sorted by (token, channel c of the
    head); an entry is the word (fp16 bits << 16) | ((t % 64) << 7) | c.
    chunk_ptr[b, h, m] .. chunk_ptr[b, h, m+1] delimit the entries of
    tokens [64m, 64m + 64).  Overflow rule, per list: within one call, token t's
    outliers in head h are stored iff the list's count at the start of the call
    plus the call's outliers in head h up to and including token t fit the
    capacity; otherwise they are dropped and the sticky status bit
    STATUS_OUTLIER_OVERFLOW is set.
    """

    def __init__(self, B, Hkv, bits, T_max, f, cap_k, cap_v, D=128):
        assert D == 128
        self.B, self.Hkv, self.D, self.bits, self.T_max, self.f = B, Hkv, D, bits, T_max, f
        self.n = Hkv * D
        self.nchunk = (T_max + CHUNK - 1) // CHUNK
        nq = (T_max + 3) // 4
        self.kcodes = np.zeros((B, Hkv, nq, block_words(bits, D)), dtype=np.uint32)
        self.vcodes = np.zeros((B, Hkv, nq, block_words(bits, D)), dtype=np.uint32)
        self.kthr = np.zeros((B, self.n, 2), dtype=np.uint16)
        self.kparams = np.zeros((B, self.n, 2), dtype=np.float32)
        self.vparams = np.zeros((B, T_max, 2), dtype=np.float32)
        self.cap = {"k": cap_k, "v": cap_v}
        self.out = {s: np.zeros((B, Hkv, cap), dtype=np.uint32) for s, cap in self.cap.items()}
        self.out_count = {s: np.zeros((B, Hkv), dtype=np.uint32) for s in self.cap}
        self.chunk_ptr = {s: np.zeros((B, Hkv, self.nchunk + 1), dtype=np.uint32) for s in self.cap}
        self.len = np.zeros(B, dtype=np.int32)
        self.status = 0
        # unpacked codes, kept for the dequantizer
        self.kc = np.zeros((B, T_max, self.n), dtype=np.uint8)
        self.vc = np.zeros((B, T_max, self.n), dtype=np.uint8)

    # -- key calibration: technique (i) per-channel, (ii) pre-RoPE -------------------------
    def calibrate_keys(self, b, K16_b):
        """K16_b: fp16 [Tp, Hkv, D] pre-RoPE keys of sequence b (reading R1 for keys)."""
        X = np.asarray(K16_b, dtype=np.float16).reshape(-1, self.n)
        lo, hi = order_stat_thresholds(X, self.f, axis=0)
        lo32, hi32 = lo.astype(np.float32), hi.astype(np.float32)
        self.kthr[b, :, 0] = lo.view(np.uint16)
        self.kthr[b, :, 1] = hi.view(np.uint16)
        self.kparams[b, :, 0] = (lo32 + hi32) * np.float32(0.5)
        self.kparams[b, :, 1] = (hi32 - lo32) * np.float32(0.5)

    # -- a block of tokens: techniques (i)-(iv) --------------------------------------------
    def quantize_tokens(self, b, t0, K16, V16, cbK, cbV):
        """Quantize tokens t0 .. t0+n-1 of sequence b (K16, V16: fp16 [n, Hkv, D])."""
        _, bndK = cbK
        _, bndV = cbV
        K = np.asarray(K16, dtype=np.float16).reshape(-1, self.n)
        V = np.asarray(V16, dtype=np.float16).reshape(-1, self.n)
        ntok = K.shape[0]
        ts = t0 + np.arange(ntok)
        assert ntok == 0 or ts[-1] < self.T_max
        # keys: the calibration thresholds and scales stay fixed (R3)
        t_lo = self.kthr[b, :, 0].view(np.float16)
        t_hi = self.kthr[b, :, 1].view(np.float16)
        kout = (K < t_lo) | (K > t_hi)
        kx = np.where(kout, np.float16(0.0), K)                   # dense remainder (R5)
        kc = encode(normalize(kx, self.kparams[b, :, 0], self.kparams[b, :, 1]), bndK)
        # values: per-token thresholds over the whole row (R1, R2, R4)
        vlo, vhi = order_stat_thresholds(V, self.f, axis=1)
        vlo32, vhi32 = vlo.astype(np.float32), vhi.astype(np.float32)
        voff = (vlo32 + vhi32) * np.float32(0.5)
        vhalf = (vhi32 - vlo32) * np.float32(0.5)
        vout = (V < vlo[:, None]) | (V > vhi[:, None])
        vx = np.where(vout, np.float16(0.0), V)
        vc = encode(normalize(vx, voff[:, None], vhalf[:, None]), bndV)
        self.vparams[b, ts, 0] = voff
        self.vparams[b, ts, 1] = vhalf
        self.kc[b, ts] = kc
        self.vc[b, ts] = vc
        # code blocks of every token quad touched; a token not yet written has code 0
        zero = np.zeros((self.Hkv, self.D), dtype=np.uint8)
        for u in sorted(set(int(t) // 4 for t in ts)):
            for arr, cc in ((self.kcodes, self.kc), (self.vcodes, self.vc)):
                quad = [cc[b, 4 * u + j].reshape(self.Hkv, self.D) if 4 * u + j < self.T_max
                        else zero for j in range(4)]
                arr[b, :, u] = pack_block(quad, self.bits)
        D = self.D
        for s, mask, X in (("k", kout, K), ("v", vout, V)):
            for h in range(self.Hkv):
                mh = mask[:, h * D:(h + 1) * D]
                per_tok = mh.sum(axis=1)
                start = int(self.out_count[s][b, h])
                # a token's outliers are kept iff the list's prefix up to it fits the capacity
                ok = start + np.cumsum(per_tok) <= self.cap[s]
                if not ok.all():
                    self.status |= STATUS_OUTLIER_OVERFLOW
                kept = np.where(ok, per_tok, 0)
                ti, ch = np.nonzero(mh & ok[:, None])          # (token, channel) order
                cnt = start + int(kept.sum())
                ent = ((X[ti, h * D + ch].view(np.uint16).astype(np.uint32) << np.uint32(16))
                       | ((ts[ti] % CHUNK).astype(np.uint32) << np.uint32(7)) | ch.astype(np.uint32))
                self.out[s][b, h, start:cnt] = ent
                # chunk_ptr[m + 1] = entries up to and including the chunk's last token of the call
                after = start + np.cumsum(kept)
                m = ts // CHUNK
                last = np.r_[m[1:] != m[:-1], True] if ntok else np.zeros(0, dtype=bool)
                self.chunk_ptr[s][b, h, m[last] + 1] = after[last]
                self.out_count[s][b, h] = cnt
        if ntok:
            self.len[b] = max(int(self.len[b]), int(ts[-1]) + 1)

    def prefill(self, K16, V16, plen, cbK, cbV):
        """K16, V16: fp16 [B, Tp, Hkv, D]; the first plen[b] tokens of sequence b are used."""
        for b in range(self.B):
            P = int(plen[b])
            assert self.len[b] == 0
            self.calibrate_keys(b, K16[b, :P])
            self.quantize_tokens(b, 0, K16[b, :P], V16[b, :P], cbK, cbV)

    def append(self, k16, v16, cbK, cbV):
        """k16, v16: fp16 [B, n_new, Hkv, D]; appended at positions len[b] onwards."""
        for b in range(self.B):
            self.quantize_tokens(b, int(self.len[b]), k16[b], v16[b], cbK, cbV)

    # -- reconstruction (R5) ---------------------------------------------------------------
    def outlier_entries(self, s, b):
        """List of (t, j = h*D + c, fp16 bits) of the lists s ('k' or 'v') of sequence b,
        head by head in stored order."""
        out = []
        nch = (int(self.len[b]) + CHUNK - 1) // CHUNK
        for h in range(self.Hkv):
            cnt = int(self.out_count[s][b, h])
            cp = self.chunk_ptr[s][b, h]
            for m in range(nch):
                for i in range(int(cp[m]), min(int(cp[m + 1]), cnt)):
                    e = int(self.out[s][b, h, i])
                    out.append((m * CHUNK + ((e >> 7) & 63), h * self.D + (e & 127), e >> 16))
        return out

    def reconstruct(self, b, cbK, cbV):
        """Exact binary64 K-hat, V-hat [T, Hkv, D] of sequence b, the attention input (R5)."""
        L = int(self.len[b])
        levK = np.asarray(cbK[0], dtype=np.float64)
        levV = np.asarray(cbV[0], dtype=np.float64)
        kp = self.kparams[b].astype(np.float64)
        vp = self.vparams[b, :L].astype(np.float64)
        Kx = kp[:, 0] + kp[:, 1] * levK[self.kc[b, :L].astype(np.int64)]
        Vx = vp[:, 0:1] + vp[:, 1:2] * levV[self.vc[b, :L].astype(np.int64)]
        for s, X in (("k", Kx), ("v", Vx)):
            for t, j, bits in self.outlier_entries(s, b):
                if t < L:
                    X[t, j] = float(np.uint16(bits).view(np.float16))
        return Kx.reshape(L, self.Hkv, self.D), Vx.reshape(L, self.Hkv, self.D)

    def dequantize(self, b, cbK, cbV, t_range=None):
        """fp16 K-hat, V-hat [T, Hkv, D] (keys pre-RoPE) of sequence b."""
        levK, _ = cbK
        levV, _ = cbV
        L = int(self.len[b])
        ts = np.arange(L) if t_range is None else np.asarray(t_range)
        kc = self.kc[b, ts].astype(np.int64)
        vc = self.vc[b, ts].astype(np.int64)
        Kh = dequant_dense(kc, self.kparams[b, :, 0], self.kparams[b, :, 1], levK)
        Vh = dequant_dense(vc, self.vparams[b, ts, 0][:, None], self.vparams[b, ts, 1][:, None],
                           levV)
        row = {int(t): i for i, t in enumerate(ts)}
        for s, Xh in (("k", Kh), ("v", Vh)):
            for t, j, bits in self.outlier_entries(s, b):
                if t in row:
                    Xh[row[t], j] = np.uint16(bits).view(np.float16)
        return Kh.reshape(len(ts), self.Hkv, self.D), Vh.reshape(len(ts), self.Hkv, self.D)


# ----------------------------------------------------------------------------------------
# RoPE and attention (technique (ii) on the read side), binary64
# ----------------------------------------------------------------------------------------


def rope_freqs(D, base):
    """theta_i = base^(-2i/D), i in [0, D/2) (reading R9)."""
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * i / D)


def rope_rotate(x, pos, base):
    """Rotate-half RoPE of x[..., D] at positions ``pos`` (broadcast over leading dims)."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_freqs(D, base)
    c, s = np.cos(ang), np.sin(ang)
    a, bb = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - bb * s, a * s + bb * c], axis=-1)


def decode_attention(q16, qpos, Kh, Vh, base, kpos=None):
    """One decode step for one sequence, binary64.

    q16: [Hq, D] pre-RoPE query; Kh, Vh: [T, Hkv, D] dequantized cache (keys
    pre-RoPE) whose row t sits at position kpos[t] (default t, reading R9).
    Returns (logits [Hq, T], probs [Hq, T], out [Hq, D]).
    """
    Hq, D = q16.shape
    T, Hkv, _ = Kh.shape
    g = Hq // Hkv
    qr = rope_rotate(np.asarray(q16, dtype=np.float64), qpos, base)
    logits = np.empty((Hq, T))
    out = np.empty((Hq, D))
    probs = np.empty((Hq, T))
    tpos = np.arange(T) if kpos is None else np.asarray(kpos)
    for h in range(Hkv):
        kr = rope_rotate(np.asarray(Kh[:, h], dtype=np.float64), tpos, base)
        vh = np.asarray(Vh[:, h], dtype=np.float64)
        for hq in range(h * g, (h + 1) * g):
            lg = kr @ qr[hq] / math.sqrt(D)
            m = lg.max()
            e = np.exp(lg - m)
            p = e / e.sum()
            logits[hq], probs[hq], out[hq] = lg, p, p @ vh
    return logits, probs, out


def merge_splits(logits, V, S):
    """Split-K softmax-weighted sum: per split (m_s, l_s, o_s), then a max/sum merge.

    logits: [T]; V: [T, D] (binary64).  Splits are S contiguous token ranges.
    """
    T = logits.shape[0]
    edges = np.linspace(0, T, S + 1).astype(int)
    parts = []
    for s in range(S):
        a, b = edges[s], edges[s + 1]
        if a == b:
            parts.append((-np.inf, 0.0, np.zeros(V.shape[1])))
            continue
        m = logits[a:b].max()
        e = np.exp(logits[a:b] - m)
        parts.append((m, e.sum(), e @ V[a:b]))
    M = max(p[0] for p in parts)
    L = sum(p[1] * math.exp(p[0] - M) for p in parts if p[1] > 0)
    o = sum(p[2] * math.exp(p[0] - M) for p in parts if p[1] > 0)
    return o / L, M, L


def partial_attention(q16, qpos, Kh, Vh, base, kpos):
    """The attention of one token range as a mergeable partial, binary64:
    M = max_t l_t, L = sum_t e^(l_t - M), o = sum_t e^(l_t - M) vhat_t (per query head).
    An empty range gives (-inf, 0, 0)."""
    Hq, D = q16.shape
    if Kh.shape[0] == 0:
        return np.full(Hq, -np.inf), np.zeros(Hq), np.zeros((Hq, D))
    lg, p, out = decode_attention(q16, qpos, Kh, Vh, base, kpos=kpos)
    M = lg.max(axis=1)
    L = np.exp(lg - M[:, None]).sum(axis=1)
    return M, L, out * L[:, None]


def merge_partials(M, L, o):
    """Softmax over the union of the ranges of partials M [P, Hq], L [P, Hq], o [P, Hq, D]
    (the same identity as the split-K merge): sum_k e^(M_k - M) o_k / sum_k e^(M_k - M) L_k."""
    M = np.asarray(M, dtype=np.float64)
    Mx = M.max(axis=0)
    w = np.where(np.asarray(L) > 0, np.exp(M - Mx[None]), 0.0)
    Ls = (w * L).sum(axis=0)
    return (w[:, :, None] * o).sum(axis=0) / Ls[:, None]

