// Append-time quantizer of the KVQuant cache (write side of techniques (i)-(iv):
// per-channel pre-RoPE keys, per-token values, NUQ encode, per-vector
// dense-and-sparse outliers).
//
// Pipeline of one kvq_quantize_append call (all on one stream):
//   k_begin        per sequence: start position, token count, calibration flag
//   k_calib_*      (calibrating prefill only) per key channel: two-pass 8-bit radix
//                  select of t_lo = s[k], t_hi = s[N-1-k] over the block's tokens
//   k_key_cuts     (calibrating prefill only) per key channel: the cut table of its codes
//   k_tok_stats    per token: value thresholds (radix select in a warp's histogram), value
//                  (off, half) and cut table; outlier counts per (64-token chunk, kv head)
//   k_tok_scan     per outlier list: chunk offsets, the capacity rule, chunk pointers,
//                  counts and len
//   k_tok_write    per (64-token chunk, kv head): encode, bit-pack both blocks, write the
//                  outliers
//   k_tok_final    lists whose room ran out: count and chunk pointers
#include <mutex>

#include "kvq_common.cuh"

using namespace kvq;

namespace {

struct QuantWs {
    int32_t* t0;      // [B] first position written
    int32_t* ntok;    // [B] tokens written
    int32_t* calib;   // [B] 1: this call calibrates sequence b
    uint32_t* hist1;  // [B][n][256]
    uint32_t* sel1;   // [B][n][4]  bin_lo, rem_lo, bin_hi, rem_hi
    uint32_t* hist2;  // [B][n][512]
    uint32_t* kcut;   // [B][n/2][16] key cut pairs of adjacent channels (calibrating calls)
    uint32_t* vrec;   // [B][n_new][kVRec] per token: force-zero mask, (t_lo, t_lo), (t_hi, t_hi),
                      // then (cut_j, cut_j) for j < 2^bits - 1, fp16 pairs ready for half2 compares
    uint32_t* kcc;    // [B*Hkv][nchc] outliers of this call in chunk cl of list (b, h)
    uint32_t* vcc;
    uint32_t* kce;    // [B*Hkv][nchc] their exclusive prefix
    uint32_t* vce;
    int32_t* lst;     // [B*Hkv][8] start K/V, first overflowing chunk K/V (-1: none), kept K/V
};

constexpr int kWsParts = 13;
constexpr int kVRec = 20;  // words of a token's value record (3 + up to 15 cuts, padded)

struct WsPlan {
    size_t off[kWsParts];
    size_t total;
};

// Chunks a call's tokens can touch in one sequence (its first may be partly filled already).
inline int call_chunks(int n_new) { return n_new / kChunk + 2; }

WsPlan plan_ws(const kvq_cfg& cfg, int n_new, int calibrate) {
    using kvq_host::align_up;
    const size_t B = cfg.B, n = (size_t)cfg.Hkv * kD, T = (size_t)n_new;
    const size_t L = B * cfg.Hkv, C = (size_t)call_chunks(n_new);
    size_t sizes[kWsParts] = {B * 4, B * 4, B * 4,
                              calibrate ? B * n * 256 * 4 : 0,
                              calibrate ? B * n * 4 * 4 : 0,
                              calibrate ? B * n * 512 * 4 : 0,
                              calibrate ? B * n * 32 : 0,
                              B * T * kVRec * 4,
                              L * C * 4, L * C * 4, L * C * 4, L * C * 4,
                              L * 8 * 4};
    WsPlan p;
    size_t o = 0;
    for (int i = 0; i < kWsParts; ++i) {
        p.off[i] = o;
        o += align_up(sizes[i]);
    }
    p.total = o;
    return p;
}

QuantWs bind_ws(char* base, const WsPlan& p) {
    QuantWs w;
    w.t0 = (int32_t*)(base + p.off[0]);
    w.ntok = (int32_t*)(base + p.off[1]);
    w.calib = (int32_t*)(base + p.off[2]);
    w.hist1 = (uint32_t*)(base + p.off[3]);
    w.sel1 = (uint32_t*)(base + p.off[4]);
    w.hist2 = (uint32_t*)(base + p.off[5]);
    w.kcut = (uint32_t*)(base + p.off[6]);
    w.vrec = (uint32_t*)(base + p.off[7]);
    w.kcc = (uint32_t*)(base + p.off[8]);
    w.vcc = (uint32_t*)(base + p.off[9]);
    w.kce = (uint32_t*)(base + p.off[10]);
    w.vce = (uint32_t*)(base + p.off[11]);
    w.lst = (int32_t*)(base + p.off[12]);
    return w;
}

__device__ inline uint32_t warp_incl_scan(uint32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Exclusive block scan of one value per thread (blockDim multiple of 32, <= 1024).
__device__ uint32_t block_excl_scan(uint32_t v, uint32_t* sm, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t incl = warp_incl_scan(v);
    __syncthreads();
    if (lane == 31) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = lane < nw ? sm[lane] : 0u;
        x = warp_incl_scan(x);
        sm[lane] = x;
    }
    __syncthreads();
    const uint32_t before = warp ? sm[warp - 1] : 0u;
    *total = sm[nw - 1];
    return before + incl - v;
}

__device__ __forceinline__ uint32_t okey2(uint32_t w) {  // order keys of both halves of w
    const uint32_t s = (w >> 15) & 0x00010001u;
    return w ^ ((s * 0x7FFFu) | 0x80008000u);
}

// ---------------------------------------------------------------------------------
__global__ void k_begin(kvq_cfg cfg, kvq_cache c, const int32_t* plen, int n_new, int calibrate,
                        QuantWs ws) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= cfg.B) return;
    int nt = plen ? plen[b] : n_new;
    nt = nt < 0 ? 0 : (nt > n_new ? n_new : nt);
    const int len0 = c.len[b];
    int t0 = len0, cal = 0;
    if (calibrate) {
        if (len0 != 0) {
            set_status(c.status, KVQ_STATUS_NOT_EMPTY);
            nt = 0;
        } else {
            t0 = 0;
            cal = 1;
        }
    }
    if ((long long)t0 + nt > cfg.T_max) {
        set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        nt = 0;
        cal = 0;
    }
    ws.t0[b] = t0;
    ws.ntok[b] = nt;
    ws.calib[b] = cal;
}

// ---------------------------------------------------------------------------------
// Key channel calibration: per-channel radix select (technique (i), pre-RoPE (ii)).  A block
// takes kCalCols adjacent channels over a range of at most 65,535 tokens; lane l of each warp
// reads channels 2l and 2l + 1 of a token row (one 4-byte load, 128 bytes per warp and row),
// kCalU rows in flight per warp.  Per-channel histograms live in shared memory, 257 words per
// channel (the same bin of neighbouring channels falls in different banks), and are added to
// the global ones at the end.  Pass 1 counts the high byte of the fp16 order key (32-bit
// counters); pass 2 the low byte of the keys whose high byte is the bin of t_lo (bins 0-255)
// or of t_hi (bins 256-511), in 16-bit counters two to a word.
constexpr int kCalCols = 64;
constexpr int kCalThreads = 512;
constexpr int kCalU = 8;
constexpr int kCalStride = 257;
constexpr int kCalRows = 65535;  // rows per block at most (16-bit counters of pass 2)
constexpr int kCalSmem = kCalCols * kCalStride * 4;

template <int PASS>
__global__ void __launch_bounds__(kCalThreads) k_calib_hist(kvq_cfg cfg,
                                                            const uint16_t* __restrict__ k,
                                                            int n_new, QuantWs ws) {
    extern __shared__ uint32_t sh[];
    const int b = blockIdx.z;
    if (!ws.calib[b]) return;
    const int n = cfg.Hkv * kD;
    const int N = ws.ntok[b];
    for (int i = threadIdx.x; i < kCalCols * kCalStride; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int j0 = blockIdx.x * kCalCols + 2 * lane;  // this lane's first channel
    const int per = (N + gridDim.y - 1) / gridDim.y;
    const int i0 = blockIdx.y * per;
    const int i1 = min(N, i0 + per);
    if (j0 < n) {
        uint32_t bl0 = 0, bh0 = 0, bl1 = 0, bh1 = 0;
        if (PASS == 2) {
            const uint32_t* s0 = ws.sel1 + ((size_t)b * n + j0) * 4;
            bl0 = s0[0]; bh0 = s0[2]; bl1 = s0[4]; bh1 = s0[6];
        }

        uint32_t* h0 = sh + (2 * lane) * kCalStride;
        uint32_t* h1 = h0 + kCalStride;
        const uint16_t* src = k + (size_t)b * n_new * n + j0;
        auto count = [&](uint32_t w) {
            const uint32_t key = okey2(w);
            const uint32_t a0 = (key >> 8) & 0xFFu, a1 = key >> 24;
            if (PASS == 1) {
                atomicAdd(&h0[a0], 1u);
                atomicAdd(&h1[a1], 1u);
            } else {
                const uint32_t l0 = key & 0xFFu, l1 = (key >> 16) & 0xFFu;
                if (a0 == bl0) atomicAdd(&h0[l0 >> 1], 1u << (16 * (l0 & 1u)));
                if (a0 == bh0) atomicAdd(&h0[128 + (l0 >> 1)], 1u << (16 * (l0 & 1u)));
                if (a1 == bl1) atomicAdd(&h1[l1 >> 1], 1u << (16 * (l1 & 1u)));
                if (a1 == bh1) atomicAdd(&h1[128 + (l1 >> 1)], 1u << (16 * (l1 & 1u)));
            }
        };
        int ib = i0 + warp;
        for (; ib + (kCalU - 1) * nw < i1; ib += nw * kCalU) {
            uint32_t w[kCalU];
#pragma unroll
            for (int u = 0; u < kCalU; ++u)
                w[u] = *reinterpret_cast<const uint32_t*>(src + (size_t)(ib + u * nw) * n);
#pragma unroll
            for (int u = 0; u < kCalU; ++u) count(w[u]);
        }
        for (; ib < i1; ib += nw) count(*reinterpret_cast<const uint32_t*>(src + (size_t)ib * n));
    }
    __syncthreads();
    const int nb = PASS == 1 ? 256 : 512;
    uint32_t* gh = (PASS == 1 ? ws.hist1 : ws.hist2) + ((size_t)b * n + blockIdx.x * kCalCols) * nb;
    for (int i = threadIdx.x; i < kCalCols * nb; i += blockDim.x) {
        const int col = i / nb, r = i % nb;
        if (blockIdx.x * kCalCols + col < n) {
            const uint32_t* hc = sh + col * kCalStride;
            const uint32_t v = PASS == 1 ? hc[r] : ((hc[r >> 1] >> (16 * (r & 1))) & 0xFFFFu);
            if (v) atomicAdd(&gh[i], v);
        }
    }
}

__global__ void k_calib_select(kvq_cfg cfg, kvq_cache c, QuantWs ws, int pass) {
    const int b = blockIdx.y;
    if (!ws.calib[b]) return;
    const int n = cfg.Hkv * kD;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n) return;
    const int N = ws.ntok[b];
    const int kk = vector_k(cfg.outlier_frac, N);
    if (pass == 1) {
        if (N == 0) return;
        const uint32_t rl = kk, rh = N - 1 - kk;
        const uint32_t* h = ws.hist1 + ((size_t)b * n + j) * 256;
        uint32_t cum = 0, bl = 0, reml = 0, bh = 0, remh = 0;
        for (int q = 0; q < 256; ++q) {
            const uint32_t v = h[q];
            if (cum <= rl && rl < cum + v) { bl = q; reml = rl - cum; }
            if (cum <= rh && rh < cum + v) { bh = q; remh = rh - cum; }
            cum += v;
        }
        uint32_t* s = ws.sel1 + ((size_t)b * n + j) * 4;
        s[0] = bl; s[1] = reml; s[2] = bh; s[3] = remh;
        return;
    }
    uint32_t lo_bits = 0, hi_bits = 0;
    if (N > 0) {
        const uint32_t* s = ws.sel1 + ((size_t)b * n + j) * 4;
        const uint32_t* h = ws.hist2 + ((size_t)b * n + j) * 512;
        uint32_t cum = 0, lb = 0;
        for (int q = 0; q < 256; ++q) {
            if (cum <= s[1] && s[1] < cum + h[q]) lb = q;
            cum += h[q];
        }
        lo_bits = okey_inv((s[0] << 8) | lb);
        cum = 0;
        uint32_t hb = 0;
        for (int q = 0; q < 256; ++q) {
            if (cum <= s[3] && s[3] < cum + h[256 + q]) hb = q;
            cum += h[256 + q];
        }
        hi_bits = okey_inv((s[2] << 8) | hb);
    }
    const float lo = h2f((uint16_t)lo_bits), hi = h2f((uint16_t)hi_bits);
    c.kthr[((size_t)b * n + j) * 2 + 0] = (uint16_t)lo_bits;
    c.kthr[((size_t)b * n + j) * 2 + 1] = (uint16_t)hi_bits;
    c.kparams[((size_t)b * n + j) * 2 + 0] = __fmul_rn(__fadd_rn(lo, hi), 0.5f);
    c.kparams[((size_t)b * n + j) * 2 + 1] = __fmul_rn(__fsub_rn(hi, lo), 0.5f);
}

// ---------------------------------------------------------------------------------
// Encoding by cut tables.  For a normalization (off, half) and a decision bound b, the set of
// fp16 inputs x with normalize(x, off, half) > b is an upper range of the fp16 total order:
// the binary32 subtraction and division round monotonically, half >= 0 always (t_hi >= t_lo),
// and when off or half is not finite every input maps to NaN and the set is empty.  Its least
// element is the cut of b, so code(x) = #{j : x >= cut_j}, a comparison of fp16 values that the
// tensor of inputs supports two at a time (HSET2).  NaN inputs compare false (code 0, as the
// division gives), a cut that no input reaches is stored as a NaN, and -0 and +0 always land on
// the same side (normalize gives them equal values), so a cut is never +0.  half == 0 makes
// every input, NaN included, normalize to 0: such a channel or token is flagged in slot 15 of
// its record and its inputs are replaced by +0 before the comparison.

// Least fp16 value in the fp16 total order whose normalized value exceeds `bound` (fp16 bits);
// 0x7E00 (NaN) when none does.  The walk starts at the fp16 value nearest off + bound * half,
// which is within a step or two of the answer, and moves along the order keys until the test
// changes; the test being monotone along the keys, that is the least passing key.  A long walk
// (not expected) falls back to bisection over -inf .. +inf.
__device__ uint32_t cut_of(float bound, float off, float half) {
    auto above = [&](uint32_t key) {
        return normalize(h2f((uint16_t)okey_inv(key)), off, half) > bound;
    };
    const uint32_t kmin = 0x03FFu, kmax = 0xFC00u;
    if (!above(kmax)) return 0x7E00u;
    if (above(kmin)) return okey_inv(kmin);
    // here above(kmin) fails and above(kmax) passes
    uint32_t key = kmin + 1;
    const float x0 = __fadd_rn(off, __fmul_rn(bound, half));
    if (isfinite(x0)) {
        key = okey(__half_as_ushort(__float2half_rn(x0)));
        key = key < kmin + 1 ? kmin + 1 : (key > kmax ? kmax : key);
    }
    int steps = 0;
    if (above(key)) {
        while (above(key - 1) && ++steps < 64) --key;  // key - 1 >= kmin, which fails
    } else {
        while (!above(key) && ++steps < 64) ++key;     // stops at kmax at the latest
    }
    if (steps >= 64) {
        uint32_t lo = kmin, hi = kmax;  // above(lo) fails, above(hi) passes
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (above(mid)) hi = mid;
            else lo = mid;
        }
        key = hi;
    }
    return okey_inv(key);
}

__device__ __forceinline__ __half2 as_h2(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }
__device__ __forceinline__ uint32_t ge2(uint32_t a, uint32_t b) { return __hge2_mask(as_h2(a), as_h2(b)); }
__device__ __forceinline__ uint32_t out2(uint32_t x, uint32_t lo, uint32_t hi) {
    return __hlt2_mask(as_h2(x), as_h2(lo)) | __hgt2_mask(as_h2(x), as_h2(hi));
}

// Codes of the two fp16 inputs in x (low and high half) against the cut pairs C[0 .. 2^BITS-2]
// (cut j of each half's row or channel in the same half): a bisection over the sorted cuts in
// which each level selects the next cut per half with the masks of the levels above.
template <int BITS>
__device__ __forceinline__ uint32_t enc_pair(uint32_t x, const uint32_t* C) {
    uint32_t m[BITS];
    uint32_t code = 0;
#pragma unroll
    for (int L = 0; L < BITS; ++L) {
        uint32_t cand[1 << (BITS - 1)];
#pragma unroll
        for (int nd = 0; nd < (1 << L); ++nd) cand[nd] = C[((2 * nd + 1) << (BITS - 1 - L)) - 1];
#pragma unroll
        for (int lv = L - 1; lv >= 0; --lv) {
#pragma unroll
            for (int p = 0; p < (1 << lv); ++p)
                cand[p] = (cand[2 * p + 1] & m[lv]) | (cand[2 * p] & ~m[lv]);
        }
        m[L] = ge2(x, cand[0]);
        code |= m[L] & (0x00010001u << (BITS - 1 - L));
    }
    return code;
}

// Per pair of adjacent key channels (2m, 2m + 1), after calibration: word j of record m holds
// cut_j(2m) | cut_j(2m + 1) << 16; word 15 the force-zero flags (0xFFFF per half whose channel
// has half == 0).
__global__ void k_key_cuts(kvq_cfg cfg, kvq_cache c, kvq_codebook cbK, QuantWs ws) {
    const int n = cfg.Hkv * kD, nb = (1 << cfg.bits) - 1;
    const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (size_t)cfg.B * (n / 2) * 16) return;
    const int j = (int)(gid & 15);
    const size_t rec = gid >> 4;  // (b, m)
    const int b = (int)(rec / (n / 2));
    if (!ws.calib[b]) return;
    const int m = (int)(rec % (n / 2));
    const float* kp0 = c.kparams + ((size_t)b * n + 2 * m) * 2;
    const float* kp1 = kp0 + 2;
    uint32_t word;
    if (j < nb) {
        const float bd = cbK.bounds[j];
        word = cut_of(bd, kp0[0], kp0[1]) | (cut_of(bd, kp1[0], kp1[1]) << 16);
    } else if (j == 15) {
        word = (kp0[1] == 0.0f ? 0xFFFFu : 0u) | (kp1[1] == 0.0f ? 0xFFFF0000u : 0u);
    } else {
        word = 0x7E007E00u;
    }
    ws.kcut[gid] = word;
}

// ---------------------------------------------------------------------------------
// Per token: value thresholds over the whole row (radix select in a warp's own shared
// histogram), value (off, half) and cuts, and the outlier counts of each kv head, summed per
// (64-token chunk, kv head).  One block per (chunk, sequence); warp w takes tokens ta + w,
// ta + w + 8, ...
constexpr int kStWarps = 8;

// A full warp finds the bin of 0-based rank r in a 256-bin histogram; every lane gets it.
__device__ inline void warp_rank(const uint32_t* hist, uint32_t r, uint32_t& bin, uint32_t& rem) {
    const int lane = threadIdx.x & 31;
    const uint4 a = reinterpret_cast<const uint4*>(hist)[2 * lane];
    const uint4 bq = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
    const uint32_t loc[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
    uint32_t s = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += loc[q];
    const uint32_t incl = warp_incl_scan(s);
    uint32_t cum = incl - s, fb = 0, fr = 0;
    const bool mine = cum <= r && r < incl;
    if (mine) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (cum <= r && r < cum + loc[q]) {
                fb = lane * 8 + q;
                fr = r - cum;
            }
            cum += loc[q];
        }
    }
    int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    src = src < 0 ? 0 : src;
    bin = __shfl_sync(0xffffffffu, fb, src);
    rem = __shfl_sync(0xffffffffu, fr, src);
}

constexpr int kStRegs = 8;   // row words (16 bytes) a lane holds at once (all of it for n <= 2048)

__global__ void __launch_bounds__(kStWarps * 32, 3) k_tok_stats(kvq_cfg cfg, kvq_cache c,
                                                            kvq_codebook cbV,
                                                            const uint16_t* __restrict__ k,
                                                            const uint16_t* __restrict__ v,
                                                            int n_new, int nchc, QuantWs ws) {
    const int b = blockIdx.y, cl = blockIdx.x;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    if (nt == 0) return;
    const int chk = t0 / kChunk + cl;
    const int ta = max(chk * kChunk, t0), tb = min(chk * kChunk + kChunk, t0 + nt);
    if (ta >= tb) return;
    extern __shared__ __align__(16) uint32_t sst[];
    const int Hkv = cfg.Hkv, n = Hkv * kD, n8 = n / 8;
    uint32_t* hist = sst;                        // [kStWarps][512]
    uint4* kth = reinterpret_cast<uint4*>(sst + kStWarps * 512);  // [n8][2]: t_lo and t_hi pairs
    __shared__ uint32_t ck[64], cv[64];
    __shared__ float bnd[16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = (1 << cfg.bits) - 1;
    for (int hh = threadIdx.x; hh < 64; hh += blockDim.x) ck[hh] = cv[hh] = 0u;
    if (threadIdx.x < nb) bnd[threadIdx.x] = cbV.bounds[threadIdx.x];
    {
        // key thresholds of 8 channels per entry, as (t_lo pairs, t_hi pairs) of half2 words
        const uint4* kt4 = reinterpret_cast<const uint4*>(c.kthr + (size_t)b * n * 2);
        for (int x = threadIdx.x; x < n8; x += blockDim.x) {
            const uint4 p = kt4[2 * x], r = kt4[2 * x + 1];
            kth[2 * x] = make_uint4(__byte_perm(p.x, p.y, 0x5410), __byte_perm(p.z, p.w, 0x5410),
                                    __byte_perm(r.x, r.y, 0x5410), __byte_perm(r.z, r.w, 0x5410));
            kth[2 * x + 1] = make_uint4(__byte_perm(p.x, p.y, 0x7632), __byte_perm(p.z, p.w, 0x7632),
                                        __byte_perm(r.x, r.y, 0x7632), __byte_perm(r.z, r.w, 0x7632));
        }
    }
    __syncthreads();
    uint32_t* hw = hist + warp * 512;
    const int kk = vector_k(cfg.outlier_frac, n);
    const uint32_t rl = kk, rh = n - 1 - kk;
    const int nrep = (n8 + 32 * kStRegs - 1) / (32 * kStRegs);
    for (int t = ta + warp; t < tb; t += kStWarps) {
        const int i = t - t0;
        const uint4* vr = reinterpret_cast<const uint4*>(v + ((size_t)b * n_new + i) * n);
        const uint4* kr = reinterpret_cast<const uint4*>(k + ((size_t)b * n_new + i) * n);
        uint4 reg[kStRegs];
        auto load = [&](int rep) {
#pragma unroll
            for (int r = 0; r < kStRegs; ++r) {
                const int x = rep * 32 * kStRegs + 32 * r + lane;
                reg[r] = x < n8 ? vr[x] : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        // pass 1: the high byte of each value's order key
        for (int q = lane; q < 512; q += 32) hw[q] = 0u;
        __syncwarp();
        for (int rep = 0; rep < nrep; ++rep) {
            load(rep);
#pragma unroll
            for (int r = 0; r < kStRegs; ++r) {
                if (rep * 32 * kStRegs + 32 * r + lane >= n8) continue;
                const uint32_t ww[4] = {reg[r].x, reg[r].y, reg[r].z, reg[r].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t key = okey2(ww[e]);
                    atomicAdd(&hw[(key >> 8) & 0xFFu], 1u);
                    atomicAdd(&hw[key >> 24], 1u);
                }
            }
        }
        __syncwarp();
        uint32_t bl, reml, bh, remh;
        warp_rank(hw, rl, bl, reml);
        warp_rank(hw, rh, bh, remh);
        __syncwarp();
        for (int q = lane; q < 512; q += 32) hw[q] = 0u;
        __syncwarp();
        // pass 2: the low byte of the keys in the two selected bins
        for (int rep = 0; rep < nrep; ++rep) {
            if (nrep > 1) load(rep);
#pragma unroll
            for (int r = 0; r < kStRegs; ++r) {
                if (rep * 32 * kStRegs + 32 * r + lane >= n8) continue;
                const uint32_t ww[4] = {reg[r].x, reg[r].y, reg[r].z, reg[r].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t key = okey2(ww[e]);
                    const uint32_t h0 = (key >> 8) & 0xFFu, h1 = key >> 24;
                    if (h0 == bl) atomicAdd(&hw[key & 255u], 1u);
                    if (h0 == bh) atomicAdd(&hw[256 + (key & 255u)], 1u);
                    if (h1 == bl) atomicAdd(&hw[(key >> 16) & 255u], 1u);
                    if (h1 == bh) atomicAdd(&hw[256 + ((key >> 16) & 255u)], 1u);
                }
            }
        }
        __syncwarp();
        uint32_t lb, d0, hb, d1;
        warp_rank(hw, reml, lb, d0);
        warp_rank(hw + 256, remh, hb, d1);
        __syncwarp();
        const uint32_t lo_bits = okey_inv((bl << 8) | lb);
        const uint32_t hi_bits = okey_inv((bh << 8) | hb);
        const float vlo = h2f((uint16_t)lo_bits), vhi = h2f((uint16_t)hi_bits);
        const float off = __fmul_rn(__fadd_rn(vlo, vhi), 0.5f);
        const float half = __fmul_rn(__fsub_rn(vhi, vlo), 0.5f);
        uint32_t* rec = ws.vrec + ((size_t)b * n_new + i) * kVRec;
        if (lane == 0) {
            c.vparams[((size_t)b * cfg.T_max + t) * 2 + 0] = off;
            c.vparams[((size_t)b * cfg.T_max + t) * 2 + 1] = half;
            rec[0] = half == 0.0f ? 0xFFFFFFFFu : 0u;
            rec[1] = lo_bits | (lo_bits << 16);
            rec[2] = hi_bits | (hi_bits << 16);
        }
        if (lane < nb) {
            const uint32_t cut = cut_of(bnd[lane], off, half);
            rec[3 + lane] = cut | (cut << 16);
        }
        // outliers per kv head (entry x of the row lies in head x >> 4)
        const uint32_t lo2 = lo_bits | (lo_bits << 16), hi2 = hi_bits | (hi_bits << 16);
        for (int rep = 0; rep < nrep; ++rep) {
            if (nrep > 1) load(rep);
#pragma unroll
            for (int r = 0; r < kStRegs; ++r) {
                const int x = rep * 32 * kStRegs + 32 * r + lane;
                if (x >= n8) continue;
                const uint32_t nv = __popc(out2(reg[r].x, lo2, hi2)) + __popc(out2(reg[r].y, lo2, hi2)) +
                                    __popc(out2(reg[r].z, lo2, hi2)) + __popc(out2(reg[r].w, lo2, hi2));
                const uint4 kw = kr[x], tl = kth[2 * x], th = kth[2 * x + 1];
                const uint32_t nk = __popc(out2(kw.x, tl.x, th.x)) + __popc(out2(kw.y, tl.y, th.y)) +
                                    __popc(out2(kw.z, tl.z, th.z)) + __popc(out2(kw.w, tl.w, th.w));
                if (nv) atomicAdd(&cv[x >> 4], nv >> 4);
                if (nk) atomicAdd(&ck[x >> 4], nk >> 4);
            }
        }
    }
    __syncthreads();
    for (int hh = threadIdx.x; hh < Hkv; hh += blockDim.x) {
        const size_t li = (size_t)b * Hkv + hh;
        ws.kcc[li * nchc + cl] = ck[hh];
        ws.vcc[li * nchc + cl] = cv[hh];
    }
}

// ---------------------------------------------------------------------------------
// Per outlier list (sequence b, kv head h): exclusive prefix of the chunk counts, the capacity
// rule at chunk level, the chunk pointers and the count when nothing is dropped, len.  A token
// keeps its outliers iff the inclusive count of this call's outliers up to it fits in the
// list's room; the first chunk whose end does not fit (if any) is resolved token by token by
// k_tok_write and finished by k_tok_final.
constexpr int kScThreads = 256;

__global__ void __launch_bounds__(kScThreads) k_tok_scan(kvq_cfg cfg, kvq_cache c, int nchc,
                                                         QuantWs ws) {
    const int li = blockIdx.x, b = li / cfg.Hkv;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    if (nt == 0) return;
    const int c0 = t0 / kChunk, nch = (t0 + nt - 1) / kChunk - c0 + 1;
    const int nch1 = nchunks(cfg.T_max) + 1;
    __shared__ uint32_t sm[32];
    __shared__ int s_star;
    for (int which = 0; which < 2; ++which) {
        const uint32_t* cnt = (which ? ws.vcc : ws.kcc) + (size_t)li * nchc;
        uint32_t* ex = (which ? ws.vce : ws.kce) + (size_t)li * nchc;
        uint32_t* count = which ? c.vcount : c.kcount;
        uint32_t* chunk = (which ? c.vchunk : c.kchunk) + (size_t)li * nch1;
        const uint32_t cap = (uint32_t)(which ? cfg.out_cap_v : cfg.out_cap_k);
        const uint32_t start = count[li];
        const unsigned long long room = cap >= start ? (unsigned long long)(cap - start) : 0ull;
        if (threadIdx.x == 0) s_star = 0x7fffffff;
        __syncthreads();
        unsigned long long running = 0;
        for (int base = 0; base < nch; base += blockDim.x) {
            const int q = base + threadIdx.x;
            const uint32_t v = q < nch ? cnt[q] : 0u;
            uint32_t tot;
            const uint32_t e = block_excl_scan(v, sm, &tot);
            if (q < nch) {
                const unsigned long long E = running + e, I = E + v;
                ex[q] = E > 0xffffffffull ? 0xffffffffu : (uint32_t)E;
                if (I > room) atomicMin(&s_star, q);
                else chunk[c0 + q + 1] = start + (uint32_t)I;
            }
            running += tot;
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            const int star = s_star;
            ws.lst[li * 8 + which] = (int32_t)start;
            ws.lst[li * 8 + 2 + which] = star == 0x7fffffff ? -1 : star;
            ws.lst[li * 8 + 4 + which] = 0;
            if (star == 0x7fffffff) count[li] = start + (uint32_t)running;
            if (which == 0 && li % cfg.Hkv == 0) c.len[b] = t0 + nt;
        }
        __syncthreads();
    }
}

// The lists whose room ran out inside a chunk: count and the pointers from that chunk on.
__global__ void k_tok_final(kvq_cfg cfg, kvq_cache c, QuantWs ws) {
    const int li = blockIdx.x, b = li / cfg.Hkv;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    if (nt == 0) return;
    const int c0 = t0 / kChunk, nch = (t0 + nt - 1) / kChunk - c0 + 1;
    const int nch1 = nchunks(cfg.T_max) + 1;
    for (int which = 0; which < 2; ++which) {
        const int star = ws.lst[li * 8 + 2 + which];
        if (star < 0) continue;
        const uint32_t start = (uint32_t)ws.lst[li * 8 + which];
        const uint32_t acc = (uint32_t)ws.lst[li * 8 + 4 + which];
        uint32_t* chunk = (which ? c.vchunk : c.kchunk) + (size_t)li * nch1;
        for (int q = star + threadIdx.x; q < nch; q += blockDim.x) chunk[c0 + q + 1] = start + acc;
        if (threadIdx.x == 0) {
            (which ? c.vcount : c.kcount)[li] = start + acc;
            set_status(c.status, KVQ_STATUS_OUTLIER_OVERFLOW);
        }
    }
}

// ---------------------------------------------------------------------------------
// Encode and pack.  One warp per (64-token chunk, kv head) of a sequence, two token quads at a
// time; the rows of the two quads (keys and values of one kv head, 256 bytes per token) reach
// shared memory through a three-stage ring of 16-byte asynchronous copies, a warp's own.
//  - Encode: half-warp hw takes quad u0 + hw and lane q the channels 8q .. 8q + 7 of each of
//    its four tokens (one 16-byte shared load per row), compares them two at a time against
//    the thresholds and cuts, and stores the eight codes as bytes, row by row.
//  - Outliers: the flagged channels of a lane are contiguous in channel order, so a token's
//    entries are ranked by a prefix sum of the per-lane counts over the half-warp (the four
//    tokens of a quad in one scan, one byte each); tokens go in order, quad u0 first.
//  - Pack: lane i of half-warp hw builds the lane group i words of quad u0 + hw from the code
//    bytes: slot s holds token s ^ (i >> 2), the field of pair (c, c + 64), c = i + 16kk, is
//    code(c) | code(c + 64) << bits at bit 2 bits (4kk + s).
// Quad 1's rows and codes sit 32 and 16 bytes further on, so the two half-warps read disjoint
// banks.
constexpr int kWrWarps = 4;
constexpr int kWrStages = 3;
constexpr int kQStride = 4 * 256 + 32;
constexpr int kKVStride = 2 * kQStride;
constexpr int kStageBytes = 2 * kKVStride;
constexpr int kCQ = 4 * 128 + 16;
constexpr int kWarpSmem = kWrStages * kStageBytes + 4 * kCQ;
constexpr int kWrSmem = kWrWarps * kWarpSmem;

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int BITS, bool KCUTS>
__global__ void __launch_bounds__(kWrWarps * 32, 3) k_tok_write(kvq_cfg cfg, kvq_cache c,
                                                               kvq_codebook cbK,
                                                               const uint16_t* __restrict__ k,
                                                               const uint16_t* __restrict__ v,
                                                               int n_new, int nchc, QuantWs ws) {
    constexpr int NB = (1 << BITS) - 1;
    constexpr int W2 = 2 * BITS;
    extern __shared__ __align__(16) unsigned char wsm[];
    const int b = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int Hkv = cfg.Hkv;
    const int task = blockIdx.x * kWrWarps + warp;
    const int cl = task / Hkv, h = task % Hkv;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    if (nt == 0 || cl >= nchc) return;
    const int chk = t0 / kChunk + cl;
    const int ta = max(chk * kChunk, t0), tb = min(chk * kChunk + kChunk, t0 + nt);
    if (ta >= tb) return;
    const int n = Hkv * kD, q = lane & 15, hw = lane >> 4;
    const size_t li = (size_t)b * Hkv + h;
    unsigned char* ring = wsm + warp * kWarpSmem;
    unsigned char* codes = ring + kWrStages * kStageBytes;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const int ua = ta >> 2, ub = (tb - 1) >> 2;
    const int nit = (ub - ua) / 2 + 1;
    // stage `it`: rows of quads ua + 2it and ua + 2it + 1; piece r of a lane is (keys or
    // values) r >> 2, quad (r >> 1) & 1, token (lane >> 4) + 2 (r & 1), bytes 16 (lane & 15)
    const uint16_t* srcK = k + (size_t)b * n_new * n + h * kD + q * 8;
    const uint16_t* srcV = v + (size_t)b * n_new * n + h * kD + q * 8;
    const uint32_t dlane = (uint32_t)((lane >> 4) * 256 + q * 16);
    auto issue = [&](int it) {
        const int u0 = ua + 2 * it;
        const uint32_t sb = ring_s + (it % kWrStages) * kStageBytes + dlane;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int which = r >> 2, hq = (r >> 1) & 1, j = hw + 2 * (r & 1);
            const int t = 4 * (u0 + hq) + j;
            if (t >= ta && t < tb)
                cp16(sb + which * kKVStride + hq * kQStride + 2 * (r & 1) * 256,
                     (which ? srcV : srcK) + (size_t)(t - t0) * n);
        }
    };
#pragma unroll
    for (int p = 0; p < kWrStages - 1; ++p) {
        if (p < nit) issue(p);
        cp_commit();
    }
    // the lane's key channels 8q .. 8q + 7 as four adjacent pairs
    uint32_t KLO[4], KHI[4], KZ[4];
    uint32_t KC[4][KCUTS ? NB : 1];
    float kof[8], khf[8], bK[KCUTS ? 1 : NB];
    {
        const uint4* th = reinterpret_cast<const uint4*>(c.kthr + ((size_t)b * n + h * kD + 8 * q) * 2);
        const uint4 t0v = th[0], t1v = th[1];
        const uint32_t a[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            KLO[e] = __byte_perm(a[2 * e], a[2 * e + 1], 0x5410);
            KHI[e] = __byte_perm(a[2 * e], a[2 * e + 1], 0x7632);
        }
    }
    if constexpr (KCUTS) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint4* rec =
                reinterpret_cast<const uint4*>(ws.kcut + ((size_t)b * (n / 2) + h * 64 + 4 * q + e) * 16);
            const uint4 r0 = rec[0], r1 = rec[1], r2 = rec[2], r3 = rec[3];
            const uint32_t rw[16] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w,
                                     r2.x, r2.y, r2.z, r2.w, r3.x, r3.y, r3.z, r3.w};
#pragma unroll
            for (int j = 0; j < NB; ++j) KC[e][j] = rw[j];
            KZ[e] = rw[15];
        }
    } else {
        const float4* kp = reinterpret_cast<const float4*>(c.kparams + ((size_t)b * n + h * kD + 8 * q) * 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 p = kp[e];
            kof[2 * e] = p.x;
            khf[2 * e] = p.y;
            kof[2 * e + 1] = p.z;
            khf[2 * e + 1] = p.w;
            KZ[e] = 0u;
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) bK[j] = cbK.bounds[j];
    }
    (void)kof;
    (void)khf;
    (void)bK;
    (void)KC;
    // outlier lists: this call's outliers before the chunk, start, room
    uint32_t inc[2] = {ws.kce[li * nchc + cl], ws.vce[li * nchc + cl]};
    uint32_t room[2], start[2];
    int star[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        start[w] = (uint32_t)ws.lst[li * 8 + w];
        star[w] = ws.lst[li * 8 + 2 + w];
        const uint32_t cap = (uint32_t)(w ? cfg.out_cap_v : cfg.out_cap_k);
        room[w] = cap >= start[w] ? cap - start[w] : 0u;
    }
    uint32_t acc[2] = {inc[0], inc[1]};
    uint32_t* outl[2] = {c.kout + li * cfg.out_cap_k, c.vout + li * cfg.out_cap_v};
    const size_t blk0 = li * nquads(cfg.T_max);
    unsigned char* cq = codes + hw * kCQ;  // this half-warp's quad: key code rows, then values
    for (int it = 0; it < nit; ++it) {
        if (it + kWrStages - 1 < nit) issue(it + kWrStages - 1);
        cp_commit();
        cp_wait<kWrStages - 1>();
        __syncwarp();
        const unsigned char* sq = ring + (it % kWrStages) * kStageBytes + hw * kQStride;
        const int u0 = ua + 2 * it, u = u0 + hw;
        // ---- encode the four tokens of quad u
        uint32_t F[2] = {0u, 0u};  // flags of the lane's 8 channels, byte j per token
        uint32_t pres = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = 4 * u + j;
            const bool pr = u <= ub && t >= ta && t < tb;
            pres |= (pr ? 1u : 0u) << j;
            const uint4 xk = *reinterpret_cast<const uint4*>(sq + j * 256 + q * 16);
            const uint4 xv = *reinterpret_cast<const uint4*>(sq + kKVStride + j * 256 + q * 16);
            uint32_t VC[NB], VLO, VHI, VZ;
            {
                constexpr int NW = (3 + NB + 3) / 4;  // record words read, in 16-byte loads
                const uint4* cr = reinterpret_cast<const uint4*>(
                    ws.vrec + ((size_t)b * n_new + (pr ? t - t0 : 0)) * kVRec);
                uint32_t rw[4 * NW];
#pragma unroll
                for (int r = 0; r < NW; ++r) {
                    const uint4 x4 = cr[r];
                    rw[4 * r] = x4.x; rw[4 * r + 1] = x4.y; rw[4 * r + 2] = x4.z; rw[4 * r + 3] = x4.w;
                }
                VZ = rw[0];
                VLO = rw[1];
                VHI = rw[2];
#pragma unroll
                for (int jj = 0; jj < NB; ++jj) VC[jj] = rw[3 + jj];
            }
            const uint32_t xkw[4] = {xk.x, xk.y, xk.z, xk.w};
            const uint32_t xvw[4] = {xv.x, xv.y, xv.z, xv.w};
            uint32_t ck[4], cv[4], okk[4], okv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t ok = out2(xkw[e], KLO[e], KHI[e]);
                okk[e] = ok;
                if constexpr (KCUTS) {
                    ck[e] = enc_pair<BITS>(xkw[e] & ~(ok | KZ[e]), KC[e]);
                } else {
                    uint32_t c2[2];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const float xf = ((ok >> (16 * hf)) & 1u) ? 0.0f : h2f((uint16_t)(xkw[e] >> (16 * hf)));
                        c2[hf] = encode(normalize(xf, kof[2 * e + hf], khf[2 * e + hf]), bK, NB);
                    }
                    ck[e] = c2[0] | (c2[1] << 16);
                }
                const uint32_t ov = out2(xvw[e], VLO, VHI);
                okv[e] = ov;
                cv[e] = enc_pair<BITS>(xvw[e] & ~(ov | VZ), VC);
            }
            // flag bits (channel 8q + m at bit m), built only when the lane has an outlier
            uint32_t fk = 0, fv = 0;
            if (okk[0] | okk[1] | okk[2] | okk[3]) {
#pragma unroll
                for (int e = 0; e < 4; ++e) fk |= ((okk[e] & 1u) | ((okk[e] >> 15) & 2u)) << (2 * e);
            }
            if (okv[0] | okv[1] | okv[2] | okv[3]) {
#pragma unroll
                for (int e = 0; e < 4; ++e) fv |= ((okv[e] & 1u) | ((okv[e] >> 15) & 2u)) << (2 * e);
            }
            // code bytes of channels 8q .. 8q + 7 (zero for a token outside this call)
            const uint32_t pm = pr ? 0xFFFFFFFFu : 0u;
            *reinterpret_cast<uint2*>(cq + j * 128 + 8 * q) =
                make_uint2(__byte_perm(ck[0], ck[1], 0x6420) & pm, __byte_perm(ck[2], ck[3], 0x6420) & pm);
            *reinterpret_cast<uint2*>(cq + 2 * kCQ + j * 128 + 8 * q) =
                make_uint2(__byte_perm(cv[0], cv[1], 0x6420) & pm, __byte_perm(cv[2], cv[3], 0x6420) & pm);
            F[0] |= (fk & pm) << (8 * j);
            F[1] |= (fv & pm) << (8 * j);
        }
        // ---- outlier entries.  The list order is token by token (quad u0's four tokens, then
        // quad u0 + 1's) and channel by channel; a token's place in its list follows from the
        // per-token totals, a lane's place within the token from the prefix sum of the lanes'
        // counts.  Each lane then writes its own entries, set bit by set bit.
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            if (!__ballot_sync(0xffffffffu, F[w] != 0u)) continue;
            // per-token counts of the lane (one byte each) and their inclusive prefix over
            // the half-warp; a byte never exceeds 16 x 8
            uint32_t c4 = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) c4 |= (uint32_t)__popc((F[w] >> (8 * j)) & 0xFFu) << (8 * j);
            uint32_t in4 = c4;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, in4, o, 16);
                if (q >= o) in4 += y;
            }
            const uint32_t T0 = __shfl_sync(0xffffffffu, in4, 15);
            const uint32_t T1 = __shfl_sync(0xffffffffu, in4, 31);
            // the eight tokens in list order: running counts and the capacity rule (warp-
            // uniform); before = the list offset at the start of this half-warp's quad
            uint32_t keep4 = 0, before = 0;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (hh == hw) before = inc[w];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t tot = ((hh ? T1 : T0) >> (8 * j)) & 0xFFu;
                    const uint32_t incl = inc[w] + tot;
                    const bool kept = incl <= room[w];
                    if (kept) acc[w] = incl;
                    if (hh == hw && kept) keep4 |= 1u << j;
                    inc[w] = incl;
                }
            }
            uint32_t m = F[w];
            const unsigned char* rows = sq + (w ? kKVStride : 0) + q * 16;
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1;
                const int j = bit >> 3, ch = bit & 7;
                if (!((keep4 >> j) & 1u)) continue;
                const uint32_t tj = (hw ? T1 : T0);
                uint32_t pos = before;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) pos += jj < j ? ((tj >> (8 * jj)) & 0xFFu) : 0u;
                const uint32_t f8 = (F[w] >> (8 * j)) & 0xFFu;
                pos += ((in4 >> (8 * j)) & 0xFFu) - __popc(f8) + __popc(f8 & ((1u << ch) - 1u));
                const uint32_t x16 = *reinterpret_cast<const uint16_t*>(rows + j * 256 + 2 * ch);
                const uint32_t tloc = (uint32_t)((4 * (u0 + hw) + j) % kChunk);
                outl[w][start[w] + pos] = (x16 << 16) | (tloc << 7) | (uint32_t)(8 * q + ch);
            }
        }
        __syncwarp();  // code bytes complete
        // ---- the quad's blocks: lane group i = q
        if (u <= ub) {
            uint32_t kw[BITS], vw[BITS];
#pragma unroll
            for (int d = 0; d < BITS; ++d) kw[d] = vw[d] = 0u;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const unsigned char* rk = cq + (s ^ (q >> 2)) * 128 + q;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int off = (4 * kk + s) * W2, wd = off >> 5, bt = off & 31;
                    const uint32_t fk = (uint32_t)rk[16 * kk] | ((uint32_t)rk[16 * kk + 64] << BITS);
                    const uint32_t fv = (uint32_t)rk[2 * kCQ + 16 * kk] |
                                        ((uint32_t)rk[2 * kCQ + 16 * kk + 64] << BITS);
                    kw[wd] |= fk << bt;
                    vw[wd] |= fv << bt;
                    if (bt + W2 > 32) {
                        kw[wd + 1] |= fk >> (32 - bt);
                        vw[wd + 1] |= fv >> (32 - bt);
                    }
                }
            }
            const size_t o = (blk0 + u) * (16 * BITS) + BITS * q;
            if (4 * u >= t0) {
#pragma unroll
                for (int d = 0; d < BITS; ++d) {
                    c.kcodes[o + d] = kw[d];
                    c.vcodes[o + d] = vw[d];
                }
            } else {
                // the quad holds earlier tokens: replace only the fields of this call's tokens
                uint32_t fm[BITS];
#pragma unroll
                for (int d = 0; d < BITS; ++d) fm[d] = 0u;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint32_t m = ((pres >> (s ^ (q >> 2))) & 1u) ? ((1u << W2) - 1u) : 0u;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const int off = (4 * kk + s) * W2, wd = off >> 5, bt = off & 31;
                        fm[wd] |= m << bt;
                        if (bt + W2 > 32) fm[wd + 1] |= m >> (32 - bt);
                    }
                }
#pragma unroll
                for (int d = 0; d < BITS; ++d) {
                    c.kcodes[o + d] = (c.kcodes[o + d] & ~fm[d]) | kw[d];
                    c.vcodes[o + d] = (c.vcodes[o + d] & ~fm[d]) | vw[d];
                }
            }
        }
        __syncwarp();  // the ring slot and the code rows are free again
    }
    cp_wait<0>();
    if (lane == 0) {
#pragma unroll
        for (int w = 0; w < 2; ++w)
            if (star[w] == cl) ws.lst[li * 8 + 4 + w] = (int32_t)acc[w];
    }
}

// ---------------------------------------------------------------------------------
// Short appends (decode steps): one block per sequence does a call's few tokens one after
// another -- value statistics over the whole row with a block-wide radix select, encode by
// division, the quad's fields, outliers appended at the end of each list in channel order,
// chunk pointers, counts, len -- in a single launch and without scratch.  Half-warp h takes kv
// head h; lane i = lane & 15 is lane group i of the code block and holds channels i + 16e
// (e < 8), so the field of pair (c, c + 64), c = i + 16kk, is code(e = kk) | code(e = kk + 4)
// << bits.  The outcome is the same as the general pipeline's for the same tokens.  Used for
// appends of at most kSmallAppend tokens per sequence with at most 32 kv heads.
constexpr int kSmallAppend = 16;

template <int BITS>
__global__ void __launch_bounds__(512) k_append_small(kvq_cfg cfg, kvq_cache c,
                                                       kvq_codebook cbK, kvq_codebook cbV,
                                                       const uint16_t* __restrict__ k,
                                                       const uint16_t* __restrict__ v,
                                                       int n_new, const int32_t* plen) {
    constexpr int NB = (1 << BITS) - 1;
    constexpr int W2 = 2 * BITS;
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = threadIdx.x >> 4, i = threadIdx.x & 15;
    const int Hkv = cfg.Hkv, n = Hkv * kD;
    const bool act = h < Hkv;
    __shared__ __align__(16) uint32_t hist[512];
    __shared__ uint32_t sel[4];
    __shared__ float bK[16], bV[16];
    __shared__ int s_nt, s_t0;
    if (threadIdx.x < NB) {
        bK[threadIdx.x] = cbK.bounds[threadIdx.x];
        bV[threadIdx.x] = cbV.bounds[threadIdx.x];
    }
    if (threadIdx.x == 0) {
        int nt = plen ? plen[b] : n_new;
        nt = nt < 0 ? 0 : (nt > n_new ? n_new : nt);
        const int t0 = c.len[b];
        if ((long long)t0 + nt > cfg.T_max) {
            set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
            nt = 0;
        }
        s_nt = nt;
        s_t0 = t0;
    }
    __syncthreads();
    const int nt = s_nt, t0 = s_t0;
    if (nt == 0) return;
    const int hh = act ? h : 0;
    const size_t li = (size_t)b * Hkv + hh;
    const int nch1 = nchunks(cfg.T_max) + 1;
    // the lane's key channels: thresholds and normalization
    uint32_t kth[8];
    float kof[8], khf[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const size_t ch = (size_t)b * n + hh * kD + i + 16 * e;
        kth[e] = reinterpret_cast<const uint32_t*>(c.kthr)[ch];  // t_lo | t_hi << 16
        kof[e] = c.kparams[ch * 2];
        khf[e] = c.kparams[ch * 2 + 1];
    }
    const uint32_t cap[2] = {(uint32_t)cfg.out_cap_k, (uint32_t)cfg.out_cap_v};
    const uint32_t start[2] = {c.kcount[li], c.vcount[li]};
    const uint32_t room[2] = {cap[0] >= start[0] ? cap[0] - start[0] : 0u,
                              cap[1] >= start[1] ? cap[1] - start[1] : 0u};
    uint32_t incl[2] = {0u, 0u}, acc[2] = {0u, 0u};
    uint32_t* outl[2] = {c.kout + li * cfg.out_cap_k, c.vout + li * cfg.out_cap_v};
    uint32_t* chunk[2] = {c.kchunk + li * nch1, c.vchunk + li * nch1};
    const int kk_rank = vector_k(cfg.outlier_frac, n);
    const uint32_t hmask = (lane >> 4) ? 0xFFFF0000u : 0x0000FFFFu;
    for (int tt = 0; tt < nt; ++tt) {
        const int t = t0 + tt;
        uint32_t xk[8], xv[8];
        const size_t row = ((size_t)b * n_new + tt) * n + hh * kD + i;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xk[e] = act ? (uint32_t)__ldg(k + row + 16 * e) : 0u;
            xv[e] = act ? (uint32_t)__ldg(v + row + 16 * e) : 0u;
        }
        // value thresholds: two 8-bit passes over the row's order keys
        for (int q = threadIdx.x; q < 512; q += blockDim.x) hist[q] = 0u;
        __syncthreads();
        if (act) {
#pragma unroll
            for (int e = 0; e < 8; ++e) atomicAdd(&hist[okey(xv[e]) >> 8], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t b0, r0, b1, r1;
            warp_rank(hist, (uint32_t)kk_rank, b0, r0);
            warp_rank(hist, (uint32_t)(n - 1 - kk_rank), b1, r1);
            if (lane == 0) {
                sel[0] = b0; sel[1] = r0; sel[2] = b1; sel[3] = r1;
            }
        }
        __syncthreads();
        const uint32_t bl = sel[0], bh = sel[2], rl = sel[1], rh = sel[3];
        for (int q = threadIdx.x; q < 512; q += blockDim.x) hist[q] = 0u;
        __syncthreads();
        if (act) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t key = okey(xv[e]);
                if ((key >> 8) == bl) atomicAdd(&hist[key & 255u], 1u);
                if ((key >> 8) == bh) atomicAdd(&hist[256 + (key & 255u)], 1u);
            }
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t lb, d0, hb, d1;
            warp_rank(hist, rl, lb, d0);
            warp_rank(hist + 256, rh, hb, d1);
            if (lane == 0) {
                sel[0] = lb; sel[2] = hb;
            }
        }
        __syncthreads();
        const uint32_t lo_bits = okey_inv((bl << 8) | sel[0]);
        const uint32_t hi_bits = okey_inv((bh << 8) | sel[2]);
        __syncthreads();  // sel is rewritten by the next token
        const float vlo = h2f((uint16_t)lo_bits), vhi = h2f((uint16_t)hi_bits);
        const float voff = __fmul_rn(__fadd_rn(vlo, vhi), 0.5f);
        const float vhalf = __fmul_rn(__fsub_rn(vhi, vlo), 0.5f);
        if (threadIdx.x == 0) {
            c.vparams[((size_t)b * cfg.T_max + t) * 2 + 0] = voff;
            c.vparams[((size_t)b * cfg.T_max + t) * 2 + 1] = vhalf;
        }
        // encode, flags
        uint32_t ck[8], cv[8], fk = 0, fv = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float x = h2f((uint16_t)xk[e]);
            const bool o = act && (x < h2f((uint16_t)(kth[e] & 0xFFFFu)) || x > h2f((uint16_t)(kth[e] >> 16)));
            fk |= (o ? 1u : 0u) << e;
            ck[e] = encode(normalize(o ? 0.0f : x, kof[e], khf[e]), bK, NB);
            const float y = h2f((uint16_t)xv[e]);
            const bool p = act && (y < vlo || y > vhi);
            fv |= (p ? 1u : 0u) << e;
            cv[e] = encode(normalize(p ? 0.0f : y, voff, vhalf), bV, NB);
        }
        // the token's fields in the quad block: slot s = (t & 3) ^ (i >> 2)
        if (act) {
            const int s = (t & 3) ^ (i >> 2);
            uint32_t kw[BITS], vw[BITS], fm[BITS];
#pragma unroll
            for (int q = 0; q < BITS; ++q) kw[q] = vw[q] = fm[q] = 0u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int ss = 0; ss < 4; ++ss) {
                    if (ss != s) continue;
                    const int off = (4 * kk + ss) * W2, wd = off >> 5, bt = off & 31;
                    const uint32_t a = ck[kk] | (ck[kk + 4] << BITS);
                    const uint32_t d = cv[kk] | (cv[kk + 4] << BITS);
                    const uint32_t m = (1u << W2) - 1u;
                    kw[wd] |= a << bt;
                    vw[wd] |= d << bt;
                    fm[wd] |= m << bt;
                    if (bt + W2 > 32) {
                        kw[wd + 1] |= a >> (32 - bt);
                        vw[wd + 1] |= d >> (32 - bt);
                        fm[wd + 1] |= m >> (32 - bt);
                    }
                }
            }
            const size_t o = (li * nquads(cfg.T_max) + (t >> 2)) * (16 * BITS) + BITS * i;
            const bool fresh = (t & 3) == 0;
#pragma unroll
            for (int q = 0; q < BITS; ++q) {
                c.kcodes[o + q] = fresh ? kw[q] : ((c.kcodes[o + q] & ~fm[q]) | kw[q]);
                c.vcodes[o + q] = fresh ? vw[q] : ((c.vcodes[o + q] & ~fm[q]) | vw[q]);
            }
        }
        // outliers in channel order (channel i + 16e ranks by (e, i))
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const uint32_t f8 = w ? fv : fk;
            uint32_t bal[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                bal[e] = __ballot_sync(0xffffffffu, (f8 >> e) & 1u) & hmask;
                tot += __popc(bal[e]);
            }
            const uint32_t before = incl[w];
            incl[w] += tot;
            const bool kept = incl[w] <= room[w];
            if (kept && act) {
                const uint32_t tloc = (uint32_t)(t % kChunk);
                uint32_t r0 = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if ((f8 >> e) & 1u) {
                        const uint32_t r = r0 + __popc(bal[e] & ((1u << lane) - 1u));
                        const uint32_t x16 = w ? xv[e] : xk[e];
                        outl[w][start[w] + before + r] =
                            (x16 << 16) | (tloc << 7) | (uint32_t)(i + 16 * e);
                    }
                    r0 += __popc(bal[e]);
                }
            }
            if (kept) acc[w] = incl[w];
            if (act && i == 0 && ((t % kChunk) == kChunk - 1 || tt == nt - 1))
                chunk[w][t / kChunk + 1] = start[w] + acc[w];
        }
    }
    if (act && i == 0) {
        c.kcount[li] = start[0] + acc[0];
        c.vcount[li] = start[1] + acc[1];
        if (acc[0] < incl[0] || acc[1] < incl[1]) set_status(c.status, KVQ_STATUS_OUTLIER_OVERFLOW);
    }
    if (threadIdx.x == 0) c.len[b] = t0 + nt;
}

int launch_small(const kvq_cfg& C, const kvq_cache& K, const kvq_codebook& cbK,
                 const kvq_codebook& cbV, const uint16_t* k, const uint16_t* v, int n_new,
                 const int32_t* plen, cudaStream_t st) {
    const int threads = ((16 * C.Hkv + 31) / 32) * 32;
    switch (C.bits) {
        case 2: k_append_small<2><<<C.B, threads, 0, st>>>(C, K, cbK, cbV, k, v, n_new, plen); break;
        case 3: k_append_small<3><<<C.B, threads, 0, st>>>(C, K, cbK, cbV, k, v, n_new, plen); break;
        default: k_append_small<4><<<C.B, threads, 0, st>>>(C, K, cbK, cbV, k, v, n_new, plen); break;
    }
    return 0;
}

// The per-token kernels of a call (stats, scan, write, final).  kcuts: the key cut tables in
// the workspace are valid (calibrating calls); otherwise keys are encoded by division.
template <int BITS>
void launch_write(const kvq_cfg& C, const kvq_cache& K, const kvq_codebook& cbK,
                  const uint16_t* k, const uint16_t* v, int n_new, int nchc, bool kcuts,
                  const QuantWs& ws, cudaStream_t st) {
    const long long tasks = (long long)nchc * C.Hkv;
    dim3 gw((unsigned)((tasks + kWrWarps - 1) / kWrWarps), C.B);
    auto kern = kcuts ? k_tok_write<BITS, true> : k_tok_write<BITS, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kWrSmem);
    kern<<<gw, kWrWarps * 32, kWrSmem, st>>>(C, K, cbK, k, v, n_new, nchc, ws);
}

void launch_tokens(const kvq_cfg& C, const kvq_cache& K, const kvq_codebook& cbK,
                   const kvq_codebook& cbV, const uint16_t* k, const uint16_t* v, int n_new,
                   bool kcuts, const QuantWs& ws, cudaStream_t st) {
    const int nchc = call_chunks(n_new);
    dim3 gt(nchc, C.B);
    const int smst = (kStWarps * 512 + C.Hkv * kD / 8 * 8) * 4;
    cudaFuncSetAttribute(k_tok_stats, cudaFuncAttributeMaxDynamicSharedMemorySize, smst);
    k_tok_stats<<<gt, kStWarps * 32, smst, st>>>(C, K, cbV, k, v, n_new, nchc, ws);
    k_tok_scan<<<C.B * C.Hkv, kScThreads, 0, st>>>(C, K, nchc, ws);
    switch (C.bits) {
        case 2: launch_write<2>(C, K, cbK, k, v, n_new, nchc, kcuts, ws, st); break;
        case 3: launch_write<3>(C, K, cbK, k, v, n_new, nchc, kcuts, ws, st); break;
        default: launch_write<4>(C, K, cbK, k, v, n_new, nchc, kcuts, ws, st); break;
    }
    k_tok_final<<<C.B * C.Hkv, 128, 0, st>>>(C, K, ws);
}

}  // namespace

using namespace kvq_host;


extern "C" int kvq_quantize_workspace(const kvq_cfg* cfg, int32_t n_new, int32_t calibrate,
                                      size_t* bytes) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    if (n_new < 0) return KVQ_ERR_SHAPE;
    *bytes = plan_ws(*cfg, n_new, calibrate).total;
    return KVQ_OK;
}

extern "C" int kvq_quantize_append(const kvq_cfg* cfg, const kvq_cache* cache,
                                   const kvq_codebook* cbK, const kvq_codebook* cbV,
                                   const uint16_t* k, const uint16_t* v, int32_t n_new,
                                   const int32_t* plen, int32_t calibrate, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if ((e = check_cache(cfg, cache))) return e;
    if ((e = check_codebook(cbK)) || (e = check_codebook(cbV))) return e;
    if (n_new < 0 || n_new > cfg->T_max) return KVQ_ERR_RANGE;
    if (n_new == 0) return KVQ_OK;
    if (!k || !v || !workspace) return KVQ_ERR_NULL;
    if (!aligned16(workspace) || !aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGN;
    const int n = cfg->Hkv * kD;
    const WsPlan p = plan_ws(*cfg, n_new, calibrate);
    if (workspace_bytes < p.total) return KVQ_ERR_WORKSPACE;
    QuantWs ws = bind_ws((char*)workspace, p);
    cudaStream_t st = (cudaStream_t)stream;
    const kvq_cfg C = *cfg;
    const kvq_cache K = *cache;
    if (!calibrate && n_new <= kSmallAppend && C.Hkv <= 32) {
        launch_small(C, K, *cbK, *cbV, k, v, n_new, plen, st);
        return record_cuda(cudaGetLastError());
    }
    k_begin<<<(C.B + 127) / 128, 128, 0, st>>>(C, K, plen, n_new, calibrate, ws);
    if (calibrate) {
        cudaError_t ce;
        if ((ce = cudaMemsetAsync(ws.hist1, 0, (size_t)C.B * n * 256 * 4, st))) return record_cuda(ce);
        if ((ce = cudaMemsetAsync(ws.hist2, 0, (size_t)C.B * n * 512 * 4, st))) return record_cuda(ce);
        if ((ce = cudaFuncSetAttribute(k_calib_hist<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kCalSmem)))
            return record_cuda(ce);
        if ((ce = cudaFuncSetAttribute(k_calib_hist<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kCalSmem)))
            return record_cuda(ce);
        const int groups = (n + kCalCols - 1) / kCalCols;
        int splits = (6 * 148 + groups * C.B - 1) / (groups * C.B);
        const int maxsp = (n_new + 1023) / 1024;
        splits = splits > maxsp ? maxsp : splits;
        const int minsp = (n_new + kCalRows - 1) / kCalRows;
        splits = splits < minsp ? minsp : splits;
        splits = splits < 1 ? 1 : splits;
        dim3 gh(groups, splits, C.B);
        dim3 gs((n + 127) / 128, C.B);
        k_calib_hist<1><<<gh, kCalThreads, kCalSmem, st>>>(C, k, n_new, ws);
        k_calib_select<<<gs, 128, 0, st>>>(C, K, ws, 1);
        k_calib_hist<2><<<gh, kCalThreads, kCalSmem, st>>>(C, k, n_new, ws);
        k_calib_select<<<gs, 128, 0, st>>>(C, K, ws, 2);
        const size_t nrec = (size_t)C.B * (n / 2) * 16;
        k_key_cuts<<<(unsigned)((nrec + 255) / 256), 256, 0, st>>>(C, K, *cbK, ws);
    }
    launch_tokens(C, K, *cbK, *cbV, k, v, n_new, calibrate != 0, ws, st);
    return record_cuda(cudaGetLastError());
}

// ---------------------------------------------------------------------------------
// Append without allocation: the scratch lives in this file-scope device array.  Host code
// must not use the symbol itself as a device address; the address is looked up once per
// device (with that device current) and passed to the kernels.
static __device__ __align__(256) unsigned char g_append_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce) return record_cuda(ce);
    if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_RANGE;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        ce = cudaGetSymbolAddress(&p, g_append_scratch);
        if (ce) return record_cuda(ce);
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KVQ_OK;
}
}  // namespace

extern "C" int kvq_quantize_append_noalloc(const kvq_cfg* cfg, const kvq_cache* cache,
                                           const kvq_codebook* cbK, const kvq_codebook* cbV,
                                           const uint16_t* k, const uint16_t* v, int32_t n_new,
                                           const int32_t* plen, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if ((e = check_cache(cfg, cache))) return e;
    if ((e = check_codebook(cbK)) || (e = check_codebook(cbV))) return e;
    if (n_new < 0 || n_new > cfg->T_max) return KVQ_ERR_RANGE;
    if (n_new == 0) return KVQ_OK;
    if (!k || !v) return KVQ_ERR_NULL;
    if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGN;
    const WsPlan p = plan_ws(*cfg, n_new, 0);
    if (p.total > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if ((e = noalloc_scratch(&scratch))) return e;
    QuantWs ws = bind_ws((char*)scratch, p);
    cudaStream_t st = (cudaStream_t)stream;
    const kvq_cfg C = *cfg;
    const kvq_cache K = *cache;
    if (n_new <= kSmallAppend && C.Hkv <= 32) {
        launch_small(C, K, *cbK, *cbV, k, v, n_new, plen, st);
        return record_cuda(cudaGetLastError());
    }
    k_begin<<<(C.B + 127) / 128, 128, 0, st>>>(C, K, plen, n_new, 0, ws);
    launch_tokens(C, K, *cbK, *cbV, k, v, n_new, false, ws, st);
    return record_cuda(cudaGetLastError());
}
