"""Counter-based synthetic input generator (numpy side).

Definition (the CUDA side in ``gen.cu`` implements exactly the same steps):

* Random bits: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
  numbers: as easy as 1, 2, 3", SC'11), with counter ``(c0, c1, c2, c3)`` and
  key ``(k0, k1)``, ten rounds, Weyl key bump between rounds.
* Normal deviates: Box-Muller on two 32-bit words ``(w0, w1)``:
  ``u = (w0 + 1/2) 2^-32``, ``a = w1 2^-32``, ``rho = sqrt(-2 ln u)``,
  ``(z0, z1) = rho (cos 2 pi a, sin 2 pi a)``.  ``ln``, ``cos`` and ``sin`` are
  evaluated by fixed series (below) using only correctly rounded IEEE-754
  binary64 operations (+, -, *, /, sqrt, floor, frexp), one at a time, in a
  fixed order, so numpy and CUDA produce identical bits.  One Philox call
  yields four deviates (words 0,1 and 2,3).
* Student-t with 3 degrees of freedom: ``z0 / sqrt((z1^2 + z2^2 + z3^2) / 3)``
  from the four deviates of one call.
* fp16 values: ``fp16(fp32(z * scale))``, each conversion round-to-nearest-even.

Element addressing: a tensor of logical shape ``[..]`` is addressed by its flat
row-major index ``e``.  A normal element uses call ``e >> 2``, deviate
``e & 3``, counter ``(lo32(e >> 2), hi32(e >> 2), stream, 0)``.  A Student-t
element uses counter ``(lo32(e), hi32(e), stream, 1)``.  A value spike flag
uses counter ``(lo32(e >> 2), hi32(e >> 2), stream, 2)``, word ``e & 3``,
flagged when the word is below ``round(p * 2^32)``.  The key is
``(seed, layer)``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)

STREAM_K = 1
STREAM_V = 2
STREAM_Q = 3
STREAM_HEAVY = 4
STREAM_TCH = 5
STREAM_CAL_K = 6
STREAM_CAL_V = 7

# Series coefficients: 1/(2k+1), (-1)^k/(2k+1)!, (-1)^k/(2k)!  (binary64, correctly rounded).
_ATANH = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "0x1.5555555555555p-2", "0x1.999999999999ap-3",
    "0x1.2492492492492p-3", "0x1.c71c71c71c71cp-4", "0x1.745d1745d1746p-4",
    "0x1.3b13b13b13b14p-4", "0x1.1111111111111p-4", "0x1.e1e1e1e1e1e1ep-5",
    "0x1.af286bca1af28p-5", "0x1.8618618618618p-5", "0x1.642c8590b2164p-5")]
_SIN = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.5555555555555p-3", "0x1.1111111111111p-7",
    "-0x1.a01a01a01a01ap-13", "0x1.71de3a556c734p-19", "-0x1.ae64567f544e4p-26",
    "0x1.6124613a86d09p-33", "-0x1.ae7f3e733b81fp-41", "0x1.952c77030ad4ap-49",
    "-0x1.2f49b46814157p-57", "0x1.71b8ef6dcf572p-66", "-0x1.761b41316381ap-75")]
_COS = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.0000000000000p-1", "0x1.5555555555555p-5",
    "-0x1.6c16c16c16c17p-10", "0x1.a01a01a01a01ap-16", "-0x1.27e4fb7789f5cp-22",
    "0x1.1eed8eff8d898p-29", "-0x1.93974a8c07c9dp-37", "0x1.ae7f3e733b81fp-45",
    "-0x1.6827863b97d97p-53", "0x1.e542ba4020225p-62", "-0x1.0ce396db7f853p-70",
    "0x1.f2cf01972f578p-80")]
_LN2 = float.fromhex("0x1.62e42fefa39efp-1")
_HALF_PI = float.fromhex("0x1.921fb54442d18p+0")
_SQRT1_2 = float.fromhex("0x1.6a09e667f3bcdp-1")
_TWO_M32 = 2.0 ** -32


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with ten rounds; all arguments uint32-valued arrays/scalars."""
    c0, c1, c2, c3 = (np.asarray(x, dtype=np.uint64) for x in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64)
    k1 = np.asarray(k1, dtype=np.uint64)
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = _M0 * c0
        p1 = _M1 * c2
        c0, c1, c2, c3 = ((p1 >> _S32) ^ c1 ^ k0, p1 & _MASK,
                          (p0 >> _S32) ^ c3 ^ k1, p0 & _MASK)
    return c0, c1, c2, c3


def _horner(coef, z):
    p = np.full_like(z, coef[-1])
    for c in reversed(coef[:-1]):
        p = p * z
        p = p + c
    return p


def _ln_unit(u):
    """ln(u) for u in (0, 1], binary64, fixed operation order."""
    m, e = np.frexp(u)
    small = m < _SQRT1_2
    m = np.where(small, m * 2.0, m)
    e = np.where(small, e - 1, e).astype(np.float64)
    s = (m - 1.0) / (m + 1.0)
    z = s * s
    t = s * _horner(_ATANH, z)
    return e * _LN2 + (t + t)


def _cos_sin_turn(a):
    """(cos 2 pi a, sin 2 pi a) for a in [0, 1), binary64, fixed order."""
    x = a * 4.0
    q = np.floor(x)
    r = x - q
    phi = r * _HALF_PI
    z = phi * phi
    s = phi * _horner(_SIN, z)
    c = _horner(_COS, z)
    qi = q.astype(np.int64)
    cos_v = np.select([qi == 0, qi == 1, qi == 2], [c, -s, -c], s)
    sin_v = np.select([qi == 0, qi == 1, qi == 2], [s, c, -s], -c)
    return cos_v, sin_v


def _box_muller(w0, w1):
    u = (w0.astype(np.float64) + 0.5) * _TWO_M32
    a = w1.astype(np.float64) * _TWO_M32
    rho = np.sqrt(-2.0 * _ln_unit(u))
    c, s = _cos_sin_turn(a)
    return rho * c, rho * s


def _split64(x):
    x = np.asarray(x, dtype=np.uint64)
    return x & _MASK, x >> _S32


def _four_normals(lo, hi, stream, tag, seed, layer):
    w = philox4x32_10(lo, hi, np.uint64(stream), np.uint64(tag),
                      np.uint64(seed & 0xFFFFFFFF), np.uint64(layer & 0xFFFFFFFF))
    z0, z1 = _box_muller(w[0], w[1])
    z2, z3 = _box_muller(w[2], w[3])
    return z0, z1, z2, z3


def normals(seed, layer, stream, e):
    """Standard normal deviates (binary64) for flat element indices ``e``."""
    e = np.asarray(e, dtype=np.uint64)
    flat = e.ravel()
    if flat.size >= 4 and flat.size % 4 == 0 and int(flat[0]) % 4 == 0:
        groups = flat.reshape(-1, 4)
        if np.array_equal(groups - groups[:, :1], np.broadcast_to(
                np.arange(4, dtype=np.uint64), groups.shape)):
            lo, hi = _split64(groups[:, 0] >> np.uint64(2))
            z = _four_normals(lo, hi, stream, 0, seed, layer)
            return np.stack(z, axis=1).reshape(e.shape)
    lo, hi = _split64(e >> np.uint64(2))
    z = _four_normals(lo, hi, stream, 0, seed, layer)
    lane = (e & np.uint64(3)).astype(np.int64)
    return np.select([lane == 0, lane == 1, lane == 2], list(z[:3]), z[3])


def student_t3(seed, layer, stream, e):
    e = np.asarray(e, dtype=np.uint64)
    lo, hi = _split64(e)
    z0, z1, z2, z3 = _four_normals(lo, hi, stream, 1, seed, layer)
    ss = z1 * z1
    ss = ss + z2 * z2
    ss = ss + z3 * z3
    return z0 / np.sqrt(ss / 3.0)


def spike_flags(seed, layer, stream, e, p):
    e = np.asarray(e, dtype=np.uint64)
    lo, hi = _split64(e >> np.uint64(2))
    w = philox4x32_10(lo, hi, np.uint64(stream), np.uint64(2),
                      np.uint64(seed & 0xFFFFFFFF), np.uint64(layer & 0xFFFFFFFF))
    lane = (e & np.uint64(3)).astype(np.int64)
    word = np.select([lane == 0, lane == 1, lane == 2], list(w[:3]), w[3])
    return word < np.uint64(spike_threshold(p))


def spike_threshold(p):
    return int(round(p * 2.0 ** 32))


def to_fp16(z):
    """binary64 -> binary32 -> binary16, each round-to-nearest-even."""
    return np.asarray(z, dtype=np.float64).astype(np.float32).astype(np.float16)


# --------------------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int                  # cached tokens written by the prefill
    bits: int
    f: float                # outlier fraction per vector
    rope_theta: float
    seed: int
    layers: int = 1
    D: int = 128
    appends: int = 1        # decode steps that append one token before attending
    steps: int = 1          # decode steps described by the workload
    k_heavy: int = 0        # heavy key channels per kv head (scaled by k_heavy_scale)
    k_heavy_scale: float = 1.0
    k_student_t: int = 0    # Student-t(3) key channels per kv head
    v_spike_p: float = 0.0  # per-element spike probability in the values
    v_spike_scale: float = 1.0
    note: str = ""

    @property
    def T_gen(self) -> int:
        """Token extent of the generated K/V tensors (cache plus decode appends)."""
        return self.T + max(self.appends * self.steps, 1) + 63

    @property
    def n(self) -> int:
        return self.Hkv * self.D


WORKLOADS = {
    w.name: w for w in (
        Workload("tiny_single_head", B=1, Hq=1, Hkv=1, T=2048, bits=3, f=0.01,
                 rope_theta=1e4, seed=0, appends=0, k_heavy=4, k_heavy_scale=8.0,
                 note="head_dim 128, 2048 cached tokens, query at position 2048"),
        Workload("llama7b_layer_32k", B=1, Hq=32, Hkv=32, T=32768, bits=3, f=0.01,
                 rope_theta=1e4, seed=1, k_heavy=6, k_heavy_scale=10.0,
                 v_spike_p=0.001, v_spike_scale=20.0,
                 note="one LLaMA-7B layer, 1-token append then attend over 32769"),
        Workload("batched_8x8k", B=8, Hq=32, Hkv=32, T=8192, bits=3, f=0.01,
                 rope_theta=1e4, seed=2, steps=64, k_heavy=6, k_heavy_scale=10.0,
                 v_spike_p=0.001, v_spike_scale=20.0,
                 note="prefill 8192 then 64 append+attend steps; bits swept 2/3/4"),
        Workload("llama3_8b_gqa_128k", B=4, Hq=32, Hkv=8, T=131072, bits=3, f=0.01,
                 rope_theta=5e5, seed=3, appends=0, k_student_t=8,
                 note="GQA 32 query heads over 8 kv heads"),
        Workload("llama7b_1m_32layers", B=1, Hq=32, Hkv=32, T=1 << 20, bits=3, f=0.005,
                 rope_theta=1e4, seed=4, layers=32, k_heavy=6, k_heavy_scale=10.0,
                 v_spike_p=0.001, v_spike_scale=20.0,
                 note="32 layers x 1,048,576 cached tokens, one decode step"),
    )
}


def workload(name: str, **overrides) -> Workload:
    return dataclasses.replace(WORKLOADS[name], **overrides)


def _rank_channels(seed, layer, stream, Hkv, D, count):
    """Per kv head, the ``count`` channels with the smallest Philox scores."""
    out = np.zeros((Hkv, D), dtype=bool)
    if count <= 0:
        return out
    idx = np.arange(Hkv * D, dtype=np.uint64)
    w = philox4x32_10(idx, np.uint64(0), np.uint64(stream), np.uint64(3),
                      np.uint64(seed & 0xFFFFFFFF), np.uint64(layer & 0xFFFFFFFF))[0]
    score = w.reshape(Hkv, D).astype(np.int64)
    for h in range(Hkv):
        order = np.lexsort((np.arange(D), score[h]))
        out[h, order[:count]] = True
    return out


def heavy_channel_scale(w: Workload, layer: int = 0) -> np.ndarray:
    """binary64 per-channel key scale ``[Hkv, D]`` (1, or the heavy factor)."""
    mask = _rank_channels(w.seed, layer, STREAM_HEAVY, w.Hkv, w.D, w.k_heavy)
    return np.where(mask, w.k_heavy_scale, 1.0)


def student_t_channels(w: Workload, layer: int = 0) -> np.ndarray:
    """Boolean ``[Hkv, D]``: key channels drawn from Student-t(3)."""
    return _rank_channels(w.seed, layer, STREAM_TCH, w.Hkv, w.D, w.k_student_t)


def _grid(w: Workload, b, t, h, c):
    b, t, h, c = np.broadcast_arrays(*(np.asarray(x, dtype=np.uint64) for x in (b, t, h, c)))
    return ((b * np.uint64(w.T_gen) + t) * np.uint64(w.Hkv) + h) * np.uint64(w.D) + c


def gen_k(w: Workload, layer=0, b=None, t=None, h=None, c=None):
    """fp16 keys K[b, t, h, c] (pre-RoPE), any broadcastable index arrays.

    With no indices given, returns the full ``[B, T_gen, Hkv, D]`` tensor.
    """
    if b is None:
        b, t, h, c = np.meshgrid(np.arange(w.B), np.arange(w.T_gen), np.arange(w.Hkv),
                                 np.arange(w.D), indexing="ij")
    b, t, h, c = np.broadcast_arrays(*(np.asarray(x) for x in (b, t, h, c)))
    e = _grid(w, b, t, h, c)
    z = normals(w.seed, layer, STREAM_K, e)
    if w.k_student_t:
        tmask = student_t_channels(w, layer)[h, c]
        if tmask.any():
            z = np.where(tmask, student_t3(w.seed, layer, STREAM_K, e), z)
    scale = heavy_channel_scale(w, layer)[h, c]
    return to_fp16(z * scale)


def gen_v(w: Workload, layer=0, b=None, t=None, h=None, c=None):
    """fp16 values V[b, t, h, c]; with no indices the full ``[B, T_gen, Hkv, D]``."""
    if b is None:
        b, t, h, c = np.meshgrid(np.arange(w.B), np.arange(w.T_gen), np.arange(w.Hkv),
                                 np.arange(w.D), indexing="ij")
    b, t, h, c = np.broadcast_arrays(*(np.asarray(x) for x in (b, t, h, c)))
    e = _grid(w, b, t, h, c)
    z = normals(w.seed, layer, STREAM_V, e)
    if w.v_spike_p > 0:
        z = np.where(spike_flags(w.seed, layer, STREAM_V, e, w.v_spike_p),
                     z * w.v_spike_scale, z)
    return to_fp16(z)


def gen_q(w: Workload, layer=0, step=0):
    """fp16 queries ``[B, Hq, D]`` (pre-RoPE) for one decode step."""
    e = np.arange(w.B * w.Hq * w.D, dtype=np.uint64) + np.uint64(step * w.B * w.Hq * w.D)
    return to_fp16(normals(w.seed, layer, STREAM_Q, e)).reshape(w.B, w.Hq, w.D)


def codebook_samples_k(w: Workload, layer=0):
    """Raw key samples for the key codebook fit: 32 vectors x 128 values (fp16).

    Vector j stands for one key channel observed over 128 tokens; it is
    Student-t(3) for the first ``round(32 * k_student_t / D)`` vectors and
    normal otherwise (a channel's scale cancels in its per-channel
    normalization, so heavy channels need no separate treatment).
    """
    seed = w.seed + 1000
    nt = int(round(32 * w.k_student_t / w.D))
    e = np.arange(32 * 128, dtype=np.uint64)
    z = normals(seed, layer, STREAM_CAL_K, e)
    if nt:
        tz = student_t3(seed, layer, STREAM_CAL_K, e)
        z = np.where((e // np.uint64(128)) < np.uint64(nt), tz, z)
    return to_fp16(z).reshape(32, 128)


def codebook_samples_v(w: Workload, layer=0):
    """Raw value samples for the value codebook fit: 1 vector x 4096 values (fp16)."""
    seed = w.seed + 1000
    e = np.arange(4096, dtype=np.uint64)
    z = normals(seed, layer, STREAM_CAL_V, e)
    if w.v_spike_p > 0:
        z = np.where(spike_flags(seed, layer, STREAM_CAL_V, e, w.v_spike_p),
                     z * w.v_spike_scale, z)
    return to_fp16(z).reshape(1, 4096)


def _selfcheck():  # pragma: no cover - manual use
    print(philox4x32_10(0, 0, 0, 0, 0, 0))
    z = normals(0, 0, 1, np.arange(1 << 16, dtype=np.uint64))
    print(z.mean(), z.std(), math.sqrt(1.0))
