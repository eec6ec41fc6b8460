// Append-time quantizer of the KVQuant cache (write side of techniques (i)-(iv):
// per-channel pre-RoPE keys, per-token values, NUQ encode, per-vector
// dense-and-sparse outliers).
//
// Pipeline of one kvq_quantize_append call (all on one stream):
//   k_begin        per sequence: start position, token count, calibration flag
//   k_calib_*      (calibrating prefill only) per key channel: two-pass 8-bit radix
//                  select of t_lo = s[k], t_hi = s[N-1-k] over the block's tokens
//   k_tok_stats    per token: value thresholds (radix select in shared memory),
//                  value (off, half), key/value outlier counts
//   k_tok_scan     per sequence: outlier offsets, the capacity rule, chunk pointers,
//                  counts and len
//   k_tok_write    per token: encode, bit-pack both rows, compact the outliers
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
    uint32_t* vthr;   // [B][n_new] fp16 t_lo | t_hi << 16
    uint32_t* kcnt;   // [B][Hkv][n_new] outliers of token i in head h
    uint32_t* vcnt;
    uint32_t* koff;   // [B][Hkv][n_new] its first entry in list (b, h), 0xffffffff if dropped
    uint32_t* voff;
};

struct WsPlan {
    size_t off[11];
    size_t total;
};

WsPlan plan_ws(const kvq_cfg& cfg, int n_new, int calibrate) {
    using kvq_host::align_up;
    const size_t B = cfg.B, n = (size_t)cfg.Hkv * kD, T = (size_t)n_new;
    size_t sizes[11] = {B * 4, B * 4, B * 4,
                        calibrate ? B * n * 256 * 4 : 0,
                        calibrate ? B * n * 4 * 4 : 0,
                        calibrate ? B * n * 512 * 4 : 0,
                        B * T * 4, B * T * cfg.Hkv * 4, B * T * cfg.Hkv * 4,
                        B * T * cfg.Hkv * 4, B * T * cfg.Hkv * 4};
    WsPlan p;
    size_t o = 0;
    for (int i = 0; i < 11; ++i) {
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
    w.vthr = (uint32_t*)(base + p.off[6]);
    w.kcnt = (uint32_t*)(base + p.off[7]);
    w.vcnt = (uint32_t*)(base + p.off[8]);
    w.koff = (uint32_t*)(base + p.off[9]);
    w.voff = (uint32_t*)(base + p.off[10]);
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

// A full warp finds the bin of 0-based rank r in a 256-bin histogram.
__device__ void warp_find_rank(const uint32_t* hist, uint32_t r, uint32_t* bin, uint32_t* rem) {
    const int lane = threadIdx.x & 31;
    uint32_t loc[8];
    uint32_t s = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        loc[q] = hist[lane * 8 + q];
        s += loc[q];
    }
    const uint32_t incl = warp_incl_scan(s);
    uint32_t cum = incl - s;
    if (cum <= r && r < incl) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (cum <= r && r < cum + loc[q]) {
                *bin = lane * 8 + q;
                *rem = r - cum;
            }
            cum += loc[q];
        }
    }
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
// Key channel calibration: per-channel radix select (technique (i), pre-RoPE (ii)).
constexpr int kCalCols = 32;

__global__ void k_calib_hist(kvq_cfg cfg, const uint16_t* __restrict__ k, int n_new, QuantWs ws,
                             int pass) {
    extern __shared__ uint32_t sh[];
    const int b = blockIdx.z;
    if (!ws.calib[b]) return;
    const int n = cfg.Hkv * kD;
    const int N = ws.ntok[b];
    const int nb = pass == 1 ? 256 : 512;
    for (int i = threadIdx.x; i < kCalCols * nb; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int j = blockIdx.x * kCalCols + lane;
    const int per = (N + gridDim.y - 1) / gridDim.y;
    const int i0 = blockIdx.y * per;
    const int i1 = min(N, i0 + per);
    if (j < n) {
        uint32_t bl = 0, bh = 0;
        if (pass == 2) {
            const uint32_t* s = ws.sel1 + ((size_t)b * n + j) * 4;
            bl = s[0];
            bh = s[2];
        }
        const uint16_t* src = k + (size_t)b * n_new * n + j;
        for (int i = i0 + warp; i < i1; i += nw) {
            const uint32_t key = okey(src[(size_t)i * n]);
            if (pass == 1) {
                atomicAdd(&sh[lane * 256 + (key >> 8)], 1u);
            } else {
                const uint32_t hb = key >> 8;
                if (hb == bl) atomicAdd(&sh[lane * 512 + (key & 255u)], 1u);
                if (hb == bh) atomicAdd(&sh[lane * 512 + 256 + (key & 255u)], 1u);
            }
        }
    }
    __syncthreads();
    uint32_t* gh = (pass == 1 ? ws.hist1 : ws.hist2) + ((size_t)b * n + blockIdx.x * kCalCols) * nb;
    for (int i = threadIdx.x; i < kCalCols * nb; i += blockDim.x) {
        const int col = i / nb;
        if (blockIdx.x * kCalCols + col < n) {
            const uint32_t v = sh[i];
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
// Per token: value thresholds over the whole row, value (off, half), outlier counts.
constexpr int kTokThreads = 512;

__global__ void __launch_bounds__(kTokThreads) k_tok_stats(kvq_cfg cfg, kvq_cache c,
                                                           const uint16_t* __restrict__ k,
                                                           const uint16_t* __restrict__ v,
                                                           int n_new, QuantWs ws) {
    const int b = blockIdx.y, i = blockIdx.x;
    if (i >= ws.ntok[b]) return;
    const int n = cfg.Hkv * kD;
    __shared__ uint32_t hist[512];
    __shared__ uint32_t sel[4];
    const uint16_t* vrow = v + ((size_t)b * n_new + i) * n;
    const uint16_t* krow = k + ((size_t)b * n_new + i) * n;
    for (int q = threadIdx.x; q < 512; q += blockDim.x) hist[q] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += blockDim.x) atomicAdd(&hist[okey(vrow[j]) >> 8], 1u);
    __syncthreads();
    const int kk = vector_k(cfg.outlier_frac, n);
    const uint32_t rl = kk, rh = n - 1 - kk;
    if (threadIdx.x < 32) {
        warp_find_rank(hist, rl, &sel[0], &sel[1]);
        warp_find_rank(hist, rh, &sel[2], &sel[3]);
    }
    __syncthreads();
    const uint32_t bl = sel[0], bh = sel[2];
    for (int q = threadIdx.x; q < 512; q += blockDim.x) hist[q] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const uint32_t key = okey(vrow[j]);
        if ((key >> 8) == bl) atomicAdd(&hist[key & 255u], 1u);
        if ((key >> 8) == bh) atomicAdd(&hist[256 + (key & 255u)], 1u);
    }
    __syncthreads();
    __shared__ uint32_t lowb[4];
    if (threadIdx.x < 32) {
        warp_find_rank(hist, sel[1], &lowb[0], &lowb[1]);
        warp_find_rank(hist + 256, sel[3], &lowb[2], &lowb[3]);
    }
    __syncthreads();
    const uint32_t lo_bits = okey_inv((bl << 8) | lowb[0]);
    const uint32_t hi_bits = okey_inv((bh << 8) | lowb[2]);
    const float vlo = h2f((uint16_t)lo_bits), vhi = h2f((uint16_t)hi_bits);
    const int t = ws.t0[b] + i;
    if (threadIdx.x == 0) {
        c.vparams[((size_t)b * cfg.T_max + t) * 2 + 0] = __fmul_rn(__fadd_rn(vlo, vhi), 0.5f);
        c.vparams[((size_t)b * cfg.T_max + t) * 2 + 1] = __fmul_rn(__fsub_rn(vhi, vlo), 0.5f);
        ws.vthr[(size_t)b * n_new + i] = lo_bits | (hi_bits << 16);
    }
    // outliers per kv head: the 32 channels of a warp's pass lie in one head
    __shared__ uint32_t hk[64], hv[64];
    for (int h = threadIdx.x; h < cfg.Hkv; h += blockDim.x) hk[h] = hv[h] = 0u;
    __syncthreads();
    const uint16_t* kt = c.kthr + (size_t)b * n * 2;
    for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + threadIdx.x;
        bool fk = false, fv = false;
        if (j < n) {
            const float xv = h2f(vrow[j]);
            fv = xv < vlo || xv > vhi;
            const float xk = h2f(krow[j]);
            fk = xk < h2f(kt[2 * j]) || xk > h2f(kt[2 * j + 1]);
        }
        const uint32_t bk = __ballot_sync(0xffffffffu, fk), bv = __ballot_sync(0xffffffffu, fv);
        if ((threadIdx.x & 31) == 0 && j < n) {
            if (bk) atomicAdd(&hk[j >> 7], (uint32_t)__popc(bk));
            if (bv) atomicAdd(&hv[j >> 7], (uint32_t)__popc(bv));
        }
    }
    __syncthreads();
    for (int h = threadIdx.x; h < cfg.Hkv; h += blockDim.x) {
        const size_t li = ((size_t)b * cfg.Hkv + h) * n_new + i;
        ws.kcnt[li] = hk[h];
        ws.vcnt[li] = hv[h];
    }
}

// ---------------------------------------------------------------------------------
// Per sequence: offsets of each token's outliers under the capacity rule.
constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;

__device__ void scan_list(int li, int nt, int t0, int n_new, const uint32_t* cnt, uint32_t* off,
                          uint32_t cap, uint32_t* count, uint32_t* chunk, int nch1,
                          int32_t* status) {
    __shared__ uint32_t sm[32];
    __shared__ unsigned long long s_acc;
    const uint32_t* cb = cnt + (size_t)li * n_new;
    uint32_t* ob = off + (size_t)li * n_new;
    const uint32_t start = count[li];
    const unsigned long long room = cap >= start ? (unsigned long long)(cap - start) : 0ull;
    if (threadIdx.x == 0) s_acc = 0;
    unsigned long long running = 0;
    const int tile = kScanThreads * kScanItems;
    for (int base = 0; base < nt; base += tile) {
        const int i0 = base + threadIdx.x * kScanItems;
        uint32_t loc[kScanItems];
        uint32_t s = 0;
#pragma unroll
        for (int q = 0; q < kScanItems; ++q) {
            loc[q] = (i0 + q < nt) ? cb[i0 + q] : 0u;
            s += loc[q];
        }
        uint32_t total;
        const uint32_t ex = block_excl_scan(s, sm, &total);
        unsigned long long incl = running + ex;
        unsigned long long best = 0;
#pragma unroll
        for (int q = 0; q < kScanItems; ++q) {
            if (i0 + q < nt) {
                incl += loc[q];
                ob[i0 + q] = incl > 0xffffffffull ? 0xffffffffu : (uint32_t)incl;
                if (incl <= room && incl > best) best = incl;
            }
        }
        if (best) atomicMax(&s_acc, best);
        running += total;
        __syncthreads();
    }
    __syncthreads();
    const unsigned long long acc = s_acc;
    for (int i = threadIdx.x; i < nt; i += blockDim.x) {
        const unsigned long long incl = ob[i];
        const bool ok = incl <= room;
        const unsigned long long ex = incl - cb[i];
        const int t = t0 + i;
        if (((t % kChunk) == kChunk - 1) || i == nt - 1) {
            const unsigned long long v = incl < acc ? incl : acc;
            chunk[(size_t)li * nch1 + t / kChunk + 1] = start + (uint32_t)v;
        }
        ob[i] = ok ? start + (uint32_t)ex : 0xffffffffu;
    }
    if (threadIdx.x == 0) {
        count[li] = start + (uint32_t)acc;
        if (acc < running) set_status(status, KVQ_STATUS_OUTLIER_OVERFLOW);
    }
    __syncthreads();
}

// One block per outlier list (sequence b, kv head h).
__global__ void __launch_bounds__(kScanThreads) k_tok_scan(kvq_cfg cfg, kvq_cache c, int n_new,
                                                           QuantWs ws) {
    const int li = blockIdx.x, b = li / cfg.Hkv;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    const int nch1 = nchunks(cfg.T_max) + 1;
    scan_list(li, nt, t0, n_new, ws.kcnt, ws.koff, (uint32_t)cfg.out_cap_k, c.kcount, c.kchunk,
              nch1, c.status);
    scan_list(li, nt, t0, n_new, ws.vcnt, ws.voff, (uint32_t)cfg.out_cap_v, c.vcount, c.vchunk,
              nch1, c.status);
    if (threadIdx.x == 0 && nt > 0 && li % cfg.Hkv == 0) c.len[b] = t0 + nt;
}

// ---------------------------------------------------------------------------------
// Per token quad (4u .. 4u+3): encode the tokens of this call in it, write their outliers,
// then the quad's key and value blocks (whole when the call starts at token 4u, else only
// the fields of this call's tokens merged into the existing block).
// Outliers of one token into the lists of its kv heads: flag/x over the n = Hkv*128 channels,
// first[h] = the token's first entry in list h (0xffffffff: dropped by the capacity rule);
// an entry is (fp16 bits << 16) | (tloc << 7) | c.  A 256-thread pass covers two heads, the
// 32 channels of a warp one quarter of a head.
__device__ void compact_outliers(int n, const uint8_t* flag, const uint16_t* x,
                                 const uint32_t* first, size_t first_stride, uint32_t tloc,
                                 uint32_t* out, size_t cap, uint32_t* sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + threadIdx.x;
        const bool f = j < n && flag[j];
        const uint32_t bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) sm[warp] = __popc(bal);
        __syncthreads();
        if (f) {
            const int h = j >> 7;
            const uint32_t f0 = first[(size_t)h * first_stride];
            if (f0 != 0xffffffffu) {
                uint32_t r = __popc(bal & ((1u << lane) - 1u));
                for (int w2 = warp & ~3; w2 < warp; ++w2) r += sm[w2];
                out[(size_t)h * cap + f0 + r] =
                    ((uint32_t)x[j] << 16) | (tloc << 7) | (uint32_t)(j & 127);
            }
        }
        __syncthreads();
    }
}

// Word `ww` of the block of kv head h from codes [4][n] of the quad's tokens; *wmask gets
// the bits of the tokens flagged in `present` (bit j = token j of the quad).
__device__ inline uint32_t block_word(const uint8_t* codes, int n, int h, int bits, int ww,
                                      uint32_t present, uint32_t* wmask) {
    const int w2 = 2 * bits, gi = ww / bits, wl = ww % bits;
    uint32_t word = 0, m = 0;
    for (int f = max(0, (32 * wl) / w2 - 1); f < 16 && f * w2 < 32 * wl + 32; ++f) {
        const int o = f * w2 - 32 * wl;
        if (o + w2 <= 0) continue;
        const int j = (f & 3) ^ (gi >> 2);   // token of slot f & 3 in lane group gi
        if (!((present >> j) & 1u)) continue;
        const int ch = h * kD + gi + 16 * (f >> 2);
        const uint32_t field =
            (uint32_t)codes[j * n + ch] | ((uint32_t)codes[j * n + ch + 64] << bits);
        const uint32_t fm = (1u << w2) - 1u;
        word |= (o >= 0) ? (field << o) : (field >> (-o));
        m |= (o >= 0) ? (fm << o) : (fm >> (-o));
    }
    *wmask = m;
    return word;
}

// One block per (token quad, sequence, kv head): the head's 128 channels of the quad's tokens.
constexpr int kWrThreads = kD;

__global__ void __launch_bounds__(kWrThreads) k_tok_write(kvq_cfg cfg, kvq_cache c,
                                                         kvq_codebook cbK, kvq_codebook cbV,
                                                         const uint16_t* __restrict__ k,
                                                         const uint16_t* __restrict__ v,
                                                         int n_new, QuantWs ws) {
    const int b = blockIdx.y, h = blockIdx.z;
    const int nt = ws.ntok[b], t0 = ws.t0[b];
    if (nt == 0) return;
    const int u = t0 / 4 + blockIdx.x;
    const int ta = max(4 * u, t0), tb = min(4 * u + 3, t0 + nt - 1);
    if (ta > tb) return;
    const int n = cfg.Hkv * kD, j = threadIdx.x, jn = h * kD + j;  // channel of the token row
    const int bits = cfg.bits, BW = block_words(bits), nbnd = (1 << bits) - 1;
    __shared__ uint8_t kc[4 * kD], vc[4 * kD];  // codes of tokens 4u .. 4u+3 (0 when absent)
    __shared__ uint8_t kf[kD], vf[kD];          // outlier flags of the current token
    __shared__ float bK[16], bV[16];
    __shared__ uint32_t sm[32];
    if (j < nbnd) {
        bK[j] = cbK.bounds[j];
        bV[j] = cbV.bounds[j];
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) kc[q * kD + j] = vc[q * kD + j] = 0;
    __syncthreads();
    const uint16_t* kt = c.kthr + ((size_t)b * n + jn) * 2;
    const float* kp = c.kparams + ((size_t)b * n + jn) * 2;
    const float klo = h2f(kt[0]), khi = h2f(kt[1]), koff = kp[0], khalf = kp[1];
    for (int t = ta; t <= tb; ++t) {
        const int i = t - t0;
        const uint16_t* vrow = v + ((size_t)b * n_new + i) * n + h * kD;
        const uint16_t* krow = k + ((size_t)b * n_new + i) * n + h * kD;
        const uint32_t vt = ws.vthr[(size_t)b * n_new + i];
        const float vlo = h2f((uint16_t)(vt & 0xffffu)), vhi = h2f((uint16_t)(vt >> 16));
        const float voff = c.vparams[((size_t)b * cfg.T_max + t) * 2 + 0];
        const float vhalf = c.vparams[((size_t)b * cfg.T_max + t) * 2 + 1];
        const float xk = h2f(krow[j]);
        const bool ok_ = xk < klo || xk > khi;
        kf[j] = ok_;
        kc[(t & 3) * kD + j] = (uint8_t)encode(normalize(ok_ ? 0.0f : xk, koff, khalf), bK, nbnd);
        const float xv = h2f(vrow[j]);
        const bool ov = xv < vlo || xv > vhi;
        vf[j] = ov;
        vc[(t & 3) * kD + j] = (uint8_t)encode(normalize(ov ? 0.0f : xv, voff, vhalf), bV, nbnd);
        __syncthreads();
        const uint32_t tloc = (uint32_t)(t % kChunk);
        const size_t li = ((size_t)b * cfg.Hkv + h) * n_new + i;  // list (b, h), token i
        compact_outliers(kD, kf, krow, ws.koff + li, 0, tloc,
                         c.kout + ((size_t)b * cfg.Hkv + h) * cfg.out_cap_k, 0, sm);
        compact_outliers(kD, vf, vrow, ws.voff + li, 0, tloc,
                         c.vout + ((size_t)b * cfg.Hkv + h) * cfg.out_cap_v, 0, sm);
    }
    // the head's key and value blocks of quad u
    uint32_t present = 0;
    for (int t = ta; t <= tb; ++t) present |= 1u << (t & 3);
    const bool fresh = (ta == 4 * u);
    const size_t blk = (((size_t)b * cfg.Hkv + h) * nquads(cfg.T_max) + u) * BW;
    for (int wi = j; wi < 2 * BW; wi += blockDim.x) {
        const int which = wi >= BW, ww = wi - which * BW;
        uint32_t m;
        const uint32_t word = block_word(which ? vc : kc, kD, 0, bits, ww, present, &m);
        uint32_t* dst = (which ? c.vcodes : c.kcodes) + blk + ww;
        *dst = fresh ? word : ((*dst & ~m) | word);
    }
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
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    const int n = cfg->Hkv * kD;
    const WsPlan p = plan_ws(*cfg, n_new, calibrate);
    if (workspace_bytes < p.total) return KVQ_ERR_WORKSPACE;
    QuantWs ws = bind_ws((char*)workspace, p);
    cudaStream_t st = (cudaStream_t)stream;
    const kvq_cfg C = *cfg;
    const kvq_cache K = *cache;
    k_begin<<<(C.B + 127) / 128, 128, 0, st>>>(C, K, plen, n_new, calibrate, ws);
    if (calibrate) {
        cudaError_t ce;
        if ((ce = cudaMemsetAsync(ws.hist1, 0, (size_t)C.B * n * 256 * 4, st))) return record_cuda(ce);
        if ((ce = cudaMemsetAsync(ws.hist2, 0, (size_t)C.B * n * 512 * 4, st))) return record_cuda(ce);
        if ((ce = cudaFuncSetAttribute(k_calib_hist, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kCalCols * 512 * 4)))
            return record_cuda(ce);
        const int groups = (n + kCalCols - 1) / kCalCols;
        int splits = (4 * 148 + groups * C.B - 1) / (groups * C.B);
        splits = splits < 1 ? 1 : splits;
        const int maxsp = (n_new + 255) / 256;
        splits = splits > maxsp ? (maxsp < 1 ? 1 : maxsp) : splits;
        dim3 gh(groups, splits, C.B);
        dim3 gs((n + 127) / 128, C.B);
        k_calib_hist<<<gh, 256, kCalCols * 256 * 4, st>>>(C, k, n_new, ws, 1);
        k_calib_select<<<gs, 128, 0, st>>>(C, K, ws, 1);
        k_calib_hist<<<gh, 256, kCalCols * 512 * 4, st>>>(C, k, n_new, ws, 2);
        k_calib_select<<<gs, 128, 0, st>>>(C, K, ws, 2);
    }
    dim3 gt(n_new, C.B);
    k_tok_stats<<<gt, kTokThreads, 0, st>>>(C, K, k, v, n_new, ws);
    k_tok_scan<<<C.B * C.Hkv, kScanThreads, 0, st>>>(C, K, n_new, ws);
    dim3 gw((n_new + 2) / 4 + 1, C.B, C.Hkv);
    k_tok_write<<<gw, kWrThreads, 0, st>>>(C, K, *cbK, *cbV, k, v, n_new, ws);
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
    const WsPlan p = plan_ws(*cfg, n_new, 0);
    if (p.total > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if ((e = noalloc_scratch(&scratch))) return e;
    QuantWs ws = bind_ws((char*)scratch, p);
    cudaStream_t st = (cudaStream_t)stream;
    const kvq_cfg C = *cfg;
    const kvq_cache K = *cache;
    k_begin<<<(C.B + 127) / 128, 128, 0, st>>>(C, K, plen, n_new, 0, ws);
    dim3 gt(n_new, C.B);
    k_tok_stats<<<gt, kTokThreads, 0, st>>>(C, K, k, v, n_new, ws);
    k_tok_scan<<<C.B * C.Hkv, kScanThreads, 0, st>>>(C, K, n_new, ws);
    dim3 gw((n_new + 2) / 4 + 1, C.B, C.Hkv);
    k_tok_write<<<gw, kWrThreads, 0, st>>>(C, K, *cbK, *cbV, k, v, n_new, ws);
    return record_cuda(cudaGetLastError());
}
