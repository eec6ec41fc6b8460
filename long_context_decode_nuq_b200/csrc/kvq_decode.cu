// Decode attention over the quantized cache (read side of techniques (i)-(iv)):
// QK with NUQ lookup + on-the-fly RoPE + key-outlier correction, split-K softmax
// statistics and merge, and the probability-weighted value sum with value-outlier
// replacement.  Also the uncompressed fp16 comparison kernel.
#include "kvq_common.cuh"

using namespace kvq;

namespace {

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kMaxG = 16;                          // query heads per kv head

__device__ inline float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Split length (multiple of 64) and effective split count for max_len and S.
__host__ __device__ inline int split_len(int max_len, int S) {
    int per = (max_len + S - 1) / S;
    per = (per + kChunk - 1) / kChunk * kChunk;
    return per < kChunk ? kChunk : per;
}

// ---------------------------------------------------------------------------------
// Packed f32x2 helpers (fma.rn.f32x2: two independent binary32 FMAs per instruction).
struct f2 {
    float x, y;
};
__device__ __forceinline__ unsigned long long pk(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ f2 upk(unsigned long long v) {
    f2 r;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

template <int BITS>
struct Fmt {
    static constexpr int FW = 2 * BITS;      // field width (two codes)
    static constexpr int NT = 1 << FW;       // pair-table entries
    static constexpr int GB = 16 * BITS;     // bits of one lane group
    static constexpr int KBW = 8 * BITS;     // words of a key block
    static constexpr int VRW = 4 * BITS;     // words of a value row
};

// First word index and bit shift of lane group j (GB bits at bit GB*j).
template <int BITS>
__device__ __forceinline__ void group_pos(int j, int& w, int& sh) {
    const int bit0 = Fmt<BITS>::GB * j;
    w = bit0 >> 5;
    sh = bit0 & 31;
}

// Align the two words of a lane group so that the group starts at bit 0 of lo.
template <int BITS>
__device__ __forceinline__ void group_align(uint32_t w0, uint32_t w1, int sh, uint32_t& lo,
                                            uint32_t& hi) {
    if (Fmt<BITS>::GB <= 32) {
        lo = w0;
        hi = 0u;
    } else {
        lo = __funnelshift_r(w0, w1, sh);
        hi = w1 >> sh;
    }
}

// A word holding the field at bit O of (hi:lo) in bits [7, 7 + FW) (other bits: junk).
template <int O>
__device__ __forceinline__ uint32_t field_at7(uint32_t lo, uint32_t hi) {
    if constexpr (O < 7) {
        return lo << (7 - O);
    } else if constexpr (O - 7 < 32) {
        return __funnelshift_r(lo, hi, O - 7);
    } else {
        return hi >> (O - 39);
    }
}

template <int BITS>
__device__ void build_pair_table(const float* levels, float2* tab) {
    constexpr int NT = Fmt<BITS>::NT;
    for (int e = threadIdx.x; e < NT * 16; e += blockDim.x) {
        const int idx = e >> 4;
        tab[e] = make_float2(levels[idx & ((1 << BITS) - 1)], levels[idx >> BITS]);
    }
}

// zhat = off + half * L[encode((0 - off)/half)]: the dense value stored at an outlier.
__device__ __forceinline__ float zero_code_value(float off, float half, const float* levels,
                                                 const float* bounds, int nb) {
    const float xn = normalize(0.0f, off, half);
    return off + half * levels[encode(xn, bounds, nb)];
}

// Pair-table load: `tab` is a shared-memory table, `off` a byte offset into it.
__device__ __forceinline__ unsigned long long tld(const unsigned long long* tab, uint32_t off) {
    return *reinterpret_cast<const unsigned long long*>(reinterpret_cast<const char*>(tab) + off);
}

// Byte offset of the pair-table entry of the field at bit O of (hi:lo): rows of 16 lane
// copies of 8 bytes (128 B per entry), copy `lane16` for this lane: (idx << 7) | lane16 << 3.
template <int BITS, int O>
__device__ __forceinline__ uint32_t tab_off(uint32_t lo, uint32_t hi, uint32_t lanebits) {
    constexpr uint32_t MASK = (uint32_t)(Fmt<BITS>::NT - 1) << 7;
    return (field_at7<O>(lo, hi) & MASK) | lanebits;
}

// One rotate-half pair m of a token pair: contribution of channels a = p, b = p + 64
// (p = j + 16m) to the two tokens' logits,
//   X = C1 + A1 La + B1 Lb,  Y = C2 + A2 La + B2 Lb,  acc += cos X + sin Y,
// evaluated for both tokens at once in the two f32x2 lanes.
template <int BITS, int M>
__device__ __forceinline__ void qk_step(const unsigned long long* tab, uint32_t lo, uint32_t hi,
                                        uint32_t lanebits, const float4* csrow,
                                        const unsigned long long* cf, unsigned long long& acc) {
    constexpr int FW = Fmt<BITS>::FW;
    const unsigned long long La = tld(tab, tab_off<BITS, FW * (2 * M)>(lo, hi, lanebits));
    const unsigned long long Lb = tld(tab, tab_off<BITS, FW * (2 * M + 1)>(lo, hi, lanebits));
    const float4 cs = csrow[16 * M];
    unsigned long long X = fma2(cf[6 * M + 0], La, cf[6 * M + 2]);
    X = fma2(cf[6 * M + 1], Lb, X);
    unsigned long long Y = fma2(cf[6 * M + 3], La, cf[6 * M + 5]);
    Y = fma2(cf[6 * M + 4], Lb, Y);
    acc = fma2(pk(cs.x, cs.y), X, acc);
    acc = fma2(pk(cs.z, cs.w), Y, acc);
}

// One value field m of a token: (o_c, o_c+64) += w * (L[code c], L[code c+64]).
template <int BITS, int M>
__device__ __forceinline__ void pv_step(const unsigned long long* tab, uint32_t lo, uint32_t hi,
                                        uint32_t lanebits, unsigned long long w,
                                        unsigned long long* o) {
    constexpr int FW = Fmt<BITS>::FW;
    o[M] = fma2(w, tld(tab, tab_off<BITS, FW * M>(lo, hi, lanebits)), o[M]);
}

// ---------------------------------------------------------------------------------
// QK: CTA = (split, sequence, group of 16 query heads); a half-warp per query head,
// lane j of it owns rotate-half pairs p = j + 16m (m < 4) of every token pair.
constexpr int kQKHeads = 16;
constexpr int kQKThreads = 256;
constexpr int kRedStride = 176;  // floats per half-warp reduction region (bank skew)

struct QKSmem {  // dynamic part (the pair table is static)
    static constexpr size_t cs4 = 0;                              // [32 token pairs][64] float4
    static constexpr size_t s8 = cs4 + 32 * 64 * 16;              // [8][64] float2 (8a*theta)
    static constexpr size_t s1 = s8 + 8 * 64 * 8;                 // [8][64] float2 (b*theta)
    static constexpr size_t b8 = s1 + 8 * 64 * 8;                 // [8][64] float2 per chunk
    static constexpr size_t qr = b8 + 8 * 64 * 8;                 // [16][128] rotated query
    static constexpr size_t zh = qr + kQKHeads * kD * 4;          // [16][128] zhat per channel
    static constexpr size_t lg = zh + kQKHeads * kD * 4;          // [64][16] chunk logits
    static constexpr size_t red = lg + 64 * kQKHeads * 4;         // reduction scratch
    static constexpr size_t base = red + (kQKThreads / 16) * kRedStride * 4;  // [64] double2
    static constexpr size_t step = base + 64 * 16;                // [64] double2 (64*theta)
    static constexpr size_t kb = step + 64 * 16;                  // bounds
    static constexpr size_t total = kb + 16 * 4;
};

template <int BITS>
__global__ void __launch_bounds__(kQKThreads, 2) k_qk2(kvq_cfg cfg, kvq_cache c, kvq_codebook cb,
                                                       const uint16_t* __restrict__ q,
                                                       const int32_t* __restrict__ qpos, int Ls,
                                                       int S, int max_len,
                                                       float* __restrict__ logits,
                                                       float2* __restrict__ stats) {
    using F = Fmt<BITS>;
    using L = QKSmem;
    __shared__ __align__(16) unsigned long long ktab[F::NT * 16];
    extern __shared__ __align__(16) uint8_t sm[];
    float4* cs4 = (float4*)(sm + L::cs4);
    float2* s8 = (float2*)(sm + L::s8);
    float2* s1 = (float2*)(sm + L::s1);
    float2* b8 = (float2*)(sm + L::b8);
    float* qr = (float*)(sm + L::qr);
    float* zh = (float*)(sm + L::zh);
    float* lg = (float*)(sm + L::lg);
    float* red = (float*)(sm + L::red);
    double2* base = (double2*)(sm + L::base);
    double2* step = (double2*)(sm + L::step);
    float* kb = (float*)(sm + L::kb);

    const int s = blockIdx.x, b = blockIdx.y, hq0 = blockIdx.z * kQKHeads;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv;
    const int nh = min(kQKHeads, Hq - hq0);
    const int tid = threadIdx.x, hh = tid >> 4, j = tid & 15;
    const bool active = hh < nh;
    const int hq = hq0 + (active ? hh : 0);
    const int h = hq / g;
    int len = c.len[b];
    if (len > max_len) {
        if (tid == 0 && s == 0 && blockIdx.z == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) {
        if (active && j == 0) stats[((size_t)b * Hq + hq) * S + s] = make_float2(-INFINITY, 0.0f);
        return;
    }
    // ---- per-CTA tables
    const int nb = (1 << BITS) - 1;
    if (tid < nb) kb[tid] = cb.bounds[tid];
    for (int e = tid; e < F::NT * 16; e += blockDim.x) {
        const int idx = e >> 4;
        ktab[e] = pk(cb.levels[idx & ((1 << BITS) - 1)], cb.levels[idx >> BITS]);
    }
    if (tid < 64) {
        const double th = rope_freq(cfg.rope_theta, tid);
        double cq, sq;
        rope_cs64((double)t_begin, th, &cq, &sq);
        base[tid] = make_double2(cq, sq);
        rope_cs64((double)kChunk, th, &cq, &sq);
        step[tid] = make_double2(cq, sq);
        // rotated, scaled query of every head of the CTA at position qpos
        rope_cs64((double)qpos[b], th, &cq, &sq);
        for (int hh2 = 0; hh2 < nh; ++hh2) {
            const uint16_t* qv = q + ((size_t)b * Hq + hq0 + hh2) * kD;
            const double qa = (double)h2f(qv[tid]), qb = (double)h2f(qv[tid + 64]);
            qr[hh2 * kD + tid] = (float)((qa * cq - qb * sq) * (double)kInvSqrtD);
            qr[hh2 * kD + tid + 64] = (float)((qa * sq + qb * cq) * (double)kInvSqrtD);
        }
        const float thf = (float)th;
        for (int a8 = 0; a8 < 8; ++a8) {
            float sn, cn;
            sincosf((float)(8 * a8) * thf, &sn, &cn);
            s8[a8 * 64 + tid] = make_float2(cn, sn);
            sincosf((float)a8 * thf, &sn, &cn);
            s1[a8 * 64 + tid] = make_float2(cn, sn);
        }
    }
    __syncthreads();
    const float* kp = c.kparams + (size_t)b * Hkv * kD * 2;
    for (int e = tid; e < nh * kD; e += blockDim.x) {
        const int hh2 = e >> 7, ch = e & 127;
        const float* p = kp + ((size_t)((hq0 + hh2) / g) * kD + ch) * 2;
        zh[e] = zero_code_value(p[0], p[1], cb.levels, kb, nb);
    }
    // ---- per-lane coefficients, duplicated into both f32x2 halves (one per token)
    unsigned long long cf[24];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int p = j + 16 * m;
        const float* pa = kp + ((size_t)h * kD + p) * 2;
        const float* pb = kp + ((size_t)h * kD + p + 64) * 2;
        const float offa = pa[0], halfa = pa[1], offb = pb[0], halfb = pb[1];
        const float qa = qr[hh * kD + p], qb = qr[hh * kD + p + 64];
        const float A1 = qa * halfa, B1 = qb * halfb, C1 = qa * offa + qb * offb;
        const float A2 = qb * halfa, B2 = -qa * halfb, C2 = qb * offa - qa * offb;
        cf[6 * m + 0] = pk(A1, A1);
        cf[6 * m + 1] = pk(B1, B1);
        cf[6 * m + 2] = pk(C1, C1);
        cf[6 * m + 3] = pk(A2, A2);
        cf[6 * m + 4] = pk(B2, B2);
        cf[6 * m + 5] = pk(C2, C2);
    }
    const int nch1 = nchunks(cfg.T_max) + 1;
    const uint32_t* chunk = c.kchunk + (size_t)b * nch1;
    const uint32_t kcount = c.kcount[b];
    const uint32_t* opos = c.kout_pos + (size_t)b * cfg.out_cap_k;
    const uint16_t* oval = c.kout_val + (size_t)b * cfg.out_cap_k;
    const size_t pair_stride = (size_t)Hkv * F::KBW;
    int gw_, gsh;
    group_pos<BITS>(j, gw_, gsh);
    const uint32_t* kb_lane =
        c.kcodes + (size_t)b * npairs(cfg.T_max) * pair_stride + (size_t)h * F::KBW + gw_;
    const uint32_t lanebits = (uint32_t)j << 3;
    float* myred = red + (tid >> 4) * kRedStride;
    float run_m = -INFINITY, run_l = 0.0f;
    uint32_t nw0[4], nw1[4];
    {
        const uint32_t* cp0 = kb_lane + (size_t)(t_begin >> 1) * pair_stride;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const bool ok = active && (t_begin + 2 * qq < t_end);
            nw0[qq] = ok ? __ldg(cp0 + (size_t)qq * pair_stride) : 0u;
            nw1[qq] = (ok && F::GB > 32) ? __ldg(cp0 + (size_t)qq * pair_stride + 1) : 0u;
        }
    }
    for (int tc = t_begin; tc < t_end; tc += kChunk) {
        // RoPE table of the chunk: cs(tc + d) = base (x) s8[d >> 3] (x) s1[d & 7]
        __syncthreads();
        for (int e = tid; e < 8 * 64; e += blockDim.x) {
            const int i = e & 63;
            const double2 bb = base[i];
            const float2 a8 = s8[e];
            const float bc = (float)bb.x, bs = (float)bb.y;
            b8[e] = make_float2(bc * a8.x - bs * a8.y, bs * a8.x + bc * a8.y);
        }
        __syncthreads();
        for (int e = tid; e < 32 * 64; e += blockDim.x) {
            const int u = e >> 6, i = e & 63;
            const int d0 = 2 * u, d1 = 2 * u + 1;
            const float2 p0 = b8[(d0 >> 3) * 64 + i], q0 = s1[(d0 & 7) * 64 + i];
            const float2 p1 = b8[(d1 >> 3) * 64 + i], q1 = s1[(d1 & 7) * 64 + i];
            cs4[e] = make_float4(p0.x * q0.x - p0.y * q0.y, p1.x * q1.x - p1.y * q1.y,
                                 p0.y * q0.x + p0.x * q0.y, p1.y * q1.x + p1.x * q1.y);
        }
        if (tid < 64) {  // advance the binary64 base angle by 64 tokens for the next chunk
            const double2 bb = base[tid], st = step[tid];
            base[tid] = make_double2(bb.x * st.x - bb.y * st.y, bb.y * st.x + bb.x * st.y);
        }
        __syncthreads();
        const int ntok = min(kChunk, t_end - tc);
        const int npr = (ntok + 1) >> 1;
        const uint32_t* cp = kb_lane + (size_t)(tc >> 1) * pair_stride;
        for (int u4 = 0; u4 < npr; u4 += 4) {
            uint32_t w0[4], w1[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                w0[qq] = nw0[qq];
                w1[qq] = nw1[qq];
                const int un = u4 + 4 + qq;
                const uint32_t* src = (un < npr) ? cp + (size_t)un * pair_stride
                                                 : cp + (size_t)(32 + qq) * pair_stride;
                const bool ok = active && ((un < npr) || (tc + kChunk + 2 * qq < t_end));
                nw0[qq] = ok ? __ldg(src) : 0u;
                nw1[qq] = (ok && F::GB > 32) ? __ldg(src + 1) : 0u;
            }
            unsigned long long acc[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t lo, hi;
                group_align<BITS>(w0[qq], w1[qq], gsh, lo, hi);
                const float4* csrow = cs4 + (u4 + qq) * 64 + j;
                unsigned long long a = 0ull;
                qk_step<BITS, 0>(ktab, lo, hi, lanebits, csrow, cf, a);
                qk_step<BITS, 1>(ktab, lo, hi, lanebits, csrow, cf, a);
                qk_step<BITS, 2>(ktab, lo, hi, lanebits, csrow, cf, a);
                qk_step<BITS, 3>(ktab, lo, hi, lanebits, csrow, cf, a);
                acc[qq] = a;
            }
            // half-warp reduction of 8 token partials over the 16 lanes (via shared memory)
            {
                float* row = myred + 8 * j + 8 * (j >> 3);
                const f2 a0 = upk(acc[0]), a1 = upk(acc[1]), a2 = upk(acc[2]), a3 = upk(acc[3]);
                *reinterpret_cast<float4*>(row) = make_float4(a0.x, a0.y, a1.x, a1.y);
                *reinterpret_cast<float4*>(row + 4) = make_float4(a2.x, a2.y, a3.x, a3.y);
                __syncwarp();
                const int col = j & 7, r0 = 8 * (j >> 3);
                float sum = 0.0f;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int r = r0 + k;
                    sum += myred[8 * r + 8 * (r >> 3) + col];
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 8);
                if (j < 8 && active) lg[(2 * u4 + col) * kQKHeads + hh] = sum;
                __syncwarp();
            }
        }
        __syncthreads();
        // key outliers of the chunk: logit += (x - zhat) * (rotated query component)
        {
            const int m = tc / kChunk;
            const uint32_t lo = min(chunk[m], kcount), hi = min(chunk[m + 1], kcount);
            const int khlo = hq0 / g, khhi = (hq0 + nh - 1) / g;
            for (uint32_t e = lo + tid; e < hi; e += blockDim.x) {
                const uint32_t p = opos[e];
                const int tl = (int)(p >> 16);
                const int jf = (int)(p & 0xffffu);
                const int kh = jf >> 7, ch = jf & 127;
                if (tl >= ntok || kh < khlo || kh > khhi) continue;
                const float x = h2f(oval[e]);
                const int i = ch & 63;
                const float4 cs = cs4[(tl >> 1) * 64 + i];
                const float cc = (tl & 1) ? cs.y : cs.x, ss = (tl & 1) ? cs.w : cs.z;
                for (int hq2 = max(kh * g, hq0); hq2 < min(kh * g + g, hq0 + nh); ++hq2) {
                    const int hh2 = hq2 - hq0;
                    const float d = x - zh[hh2 * kD + ch];
                    const float qa = qr[hh2 * kD + i], qb = qr[hh2 * kD + i + 64];
                    const float r = (ch < 64) ? (cc * qa + ss * qb) : (cc * qb - ss * qa);
                    atomicAdd(&lg[tl * kQKHeads + hh2], d * r);
                }
            }
        }
        __syncthreads();
        // logits out and the split's running softmax statistics (half-warp per head)
        {
            float mx = -INFINITY;
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int tl = j + 16 * k;
                const bool ok = active && tl < ntok;
                v[k] = ok ? lg[tl * kQKHeads + hh] : -INFINITY;
                mx = fmaxf(mx, v[k]);
                if (ok) logits[((size_t)b * Hq + hq) * cfg.T_max + tc + tl] = v[k];
            }
#pragma unroll
            for (int o = 8; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float mn = fmaxf(run_m, mx);
            float ssum = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) ssum += (v[k] > -INFINITY) ? expf(v[k] - mn) : 0.0f;
#pragma unroll
            for (int o = 8; o; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
            if (active) {
                run_l = (run_m > -INFINITY ? run_l * expf(run_m - mn) : 0.0f) + ssum;
                run_m = mn;
            }
        }
    }
    if (active && j == 0) stats[((size_t)b * Hq + hq) * S + s] = make_float2(run_m, run_l);
}

// ---------------------------------------------------------------------------------
// PV: CTA = (split, sequence, group of 16 query heads); 8 lanes per query head, lane j
// owns the value fields (c, c + 64) for c = j + 8m (m < 8) of every token.
constexpr int kPVHeads = 16;
constexpr int kPVThreads = 8 * kPVHeads;

struct PVSmem {  // dynamic part (the pair table is static)
    static constexpr size_t w2 = 0;                               // [64][16] (w, w)
    static constexpr size_t pp = w2 + 64 * kPVHeads * 8;          // [64][16] p
    static constexpr size_t corr = pp + 64 * kPVHeads * 4;        // [16][128]
    static constexpr size_t vpar = corr + kPVHeads * kD * 4;      // [64] (off, half)
    static constexpr size_t zv = vpar + 64 * 8;                   // [64]
    static constexpr size_t vb = zv + 64 * 4;                     // bounds
    static constexpr size_t total = vb + 16 * 4;
};

template <int BITS>
__global__ void __launch_bounds__(kPVThreads, 4) k_pv2(kvq_cfg cfg, kvq_cache c, kvq_codebook cb,
                                                    const float* __restrict__ logits,
                                                    const float2* __restrict__ ml, int Ls, int S,
                                                    int max_len, float* __restrict__ part) {
    using F = Fmt<BITS>;
    using L = PVSmem;
    __shared__ __align__(16) unsigned long long vtab[F::NT * 16];
    extern __shared__ __align__(16) uint8_t sm[];
    unsigned long long* w2 = (unsigned long long*)(sm + L::w2);
    float* pp = (float*)(sm + L::pp);
    float* corr = (float*)(sm + L::corr);
    float2* vpar = (float2*)(sm + L::vpar);
    float* zv = (float*)(sm + L::zv);
    float* vb = (float*)(sm + L::vb);
    const int s = blockIdx.x, b = blockIdx.y, hq0 = blockIdx.z * kPVHeads;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv;
    const int nh = min(kPVHeads, Hq - hq0);
    const int tid = threadIdx.x, hh = tid >> 3, j = tid & 7;
    const bool active = hh < nh;
    const int hq = hq0 + (active ? hh : 0);
    const int h = hq / g;
    const int len = min(c.len[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    const int nb = (1 << BITS) - 1;
    if (tid < nb) vb[tid] = cb.bounds[tid];
    for (int e = tid; e < F::NT * 16; e += blockDim.x) {
        const int idx = e >> 4;
        vtab[e] = pk(cb.levels[idx & ((1 << BITS) - 1)], cb.levels[idx >> BITS]);
    }
    for (int e = tid; e < kPVHeads * kD; e += blockDim.x) corr[e] = 0.0f;
    unsigned long long o[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m] = 0ull;
    float poff = 0.0f;
    const int nch1 = nchunks(cfg.T_max) + 1;
    const uint32_t* chunk = c.vchunk + (size_t)b * nch1;
    const uint32_t vcount = c.vcount[b];
    const uint32_t* opos = c.vout_pos + (size_t)b * cfg.out_cap_v;
    const uint16_t* oval = c.vout_val + (size_t)b * cfg.out_cap_v;
    const size_t row_stride = (size_t)Hkv * F::VRW;
    int gw_, gsh;
    group_pos<BITS>(j, gw_, gsh);
    const uint32_t* vr_lane = c.vcodes + (size_t)b * cfg.T_max * row_stride + (size_t)h * F::VRW + gw_;
    const uint32_t lanebits = (uint32_t)(tid & 15) << 3;
    const float2 mL = active ? ml[(size_t)b * Hq + hq] : make_float2(0.0f, 1.0f);
    for (int tc = t_begin; tc < t_end; tc += kChunk) {
        const int ntok = min(kChunk, t_end - tc);
        const uint32_t* rp = vr_lane + (size_t)tc * row_stride;
        // first four rows of the chunk in flight while the weights are prepared
        uint32_t nw0[4], nw1[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const bool ok = active && qq < ntok;
            nw0[qq] = ok ? __ldg(rp + (size_t)qq * row_stride) : 0u;
            nw1[qq] = (ok && F::GB > 32) ? __ldg(rp + (size_t)qq * row_stride + 1) : 0u;
        }
        __syncthreads();
        if (tid < kChunk) {
            float2 vp = make_float2(0.0f, 0.0f);
            float z = 0.0f;
            if (tid < ntok) {
                vp = *(const float2*)(c.vparams + ((size_t)b * cfg.T_max + tc + tid) * 2);
                z = zero_code_value(vp.x, vp.y, cb.levels, vb, nb);
            }
            vpar[tid] = vp;
            zv[tid] = z;
        }
        __syncthreads();
        // p_t = exp(l_t - M) / L; w = p * half_t; each of the head's 8 lanes takes 8 tokens
        {
            float po = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int dt = j + 8 * k;
                float p = 0.0f;
                if (active && dt < ntok)
                    p = expf(logits[((size_t)b * Hq + hq) * cfg.T_max + tc + dt] - mL.x) / mL.y;
                pp[dt * kPVHeads + hh] = p;
                const float w = p * vpar[dt].y;
                w2[dt * kPVHeads + hh] = pk(w, w);
                po += p * vpar[dt].x;
            }
            po += __shfl_xor_sync(0xffffffffu, po, 1);
            po += __shfl_xor_sync(0xffffffffu, po, 2);
            po += __shfl_xor_sync(0xffffffffu, po, 4);
            poff += po;
        }
        __syncthreads();
        if (active) {
            for (int d4 = 0; d4 < ntok; d4 += 4) {
                uint32_t w0[4], w1[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    w0[qq] = nw0[qq];
                    w1[qq] = nw1[qq];
                    const int dn = d4 + 4 + qq;
                    const bool ok = dn < ntok;
                    nw0[qq] = ok ? __ldg(rp + (size_t)dn * row_stride) : 0u;
                    nw1[qq] = (ok && F::GB > 32) ? __ldg(rp + (size_t)dn * row_stride + 1) : 0u;
                }
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint32_t lo, hi;
                    group_align<BITS>(w0[qq], w1[qq], gsh, lo, hi);
                    const unsigned long long w = w2[(d4 + qq) * kPVHeads + hh];
                    pv_step<BITS, 0>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 1>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 2>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 3>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 4>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 5>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 6>(vtab, lo, hi, lanebits, w, o);
                    pv_step<BITS, 7>(vtab, lo, hi, lanebits, w, o);
                }
            }
        }
        // value outliers: out += p_t * (x - zhat_t) (shared-memory atomics)
        {
            const int m = tc / kChunk;
            const uint32_t lo = min(chunk[m], vcount), hi = min(chunk[m + 1], vcount);
            const int khlo = hq0 / g, khhi = (hq0 + nh - 1) / g;
            for (uint32_t e = lo + tid; e < hi; e += blockDim.x) {
                const uint32_t p = opos[e];
                const int tl = (int)(p >> 16);
                const int jf = (int)(p & 0xffffu);
                const int kh = jf >> 7, ch = jf & 127;
                if (tl >= ntok || kh < khlo || kh > khhi) continue;
                const float d = h2f(oval[e]) - zv[tl];
                for (int hq2 = max(kh * g, hq0); hq2 < min(kh * g + g, hq0 + nh); ++hq2)
                    atomicAdd(&corr[(hq2 - hq0) * kD + ch], pp[tl * kPVHeads + (hq2 - hq0)] * d);
            }
        }
    }
    __syncthreads();
    if (active) {
        float* dst = part + (((size_t)b * Hq + hq) * S + s) * kD;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int ch = j + 8 * m;
            const f2 v = upk(o[m]);
            dst[ch] = v.x + poff + corr[hh * kD + ch];
            dst[ch + 64] = v.y + poff + corr[hh * kD + ch + 64];
        }
    }
}

__global__ void k_softmax_merge(int BH, int S, const float2* __restrict__ stats,
                                float2* __restrict__ ml) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= BH) return;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, stats[(size_t)r * S + s].x);
    float Lsum = 0.0f;
    if (M > -INFINITY)
        for (int s = 0; s < S; ++s) {
            const float2 st = stats[(size_t)r * S + s];
            if (st.y > 0.0f) Lsum += st.y * expf(st.x - M);
        }
    ml[r] = make_float2(M, Lsum);
}

__global__ void k_pv_reduce(int S, const float* __restrict__ part, float* __restrict__ out) {
    const int r = blockIdx.x, ch = threadIdx.x;
    float a = 0.0f;
    for (int s = 0; s < S; ++s) a += part[((size_t)r * S + s) * kD + ch];
    out[(size_t)r * kD + ch] = a;
}

// ---------------------------------------------------------------------------------
// Merge of per-split (m, l, o) partials: out = sum_s e^(m_s-M) o_s / sum_s e^(m_s-M) l_s.
__global__ void k_attn_merge(int S, const float2* __restrict__ st, const float* __restrict__ po,
                             float* __restrict__ out) {
    const int r = blockIdx.x, ch = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, st[(size_t)r * S + s].x);
    float Ls = 0.0f, o = 0.0f;
    if (M > -INFINITY)
        for (int s = 0; s < S; ++s) {
            const float2 x = st[(size_t)r * S + s];
            if (x.y > 0.0f) {
                const float w = expf(x.x - M);
                Ls += x.y * w;
                o += po[((size_t)r * S + s) * kD + ch] * w;
            }
        }
    out[(size_t)r * kD + ch] = Ls > 0.0f ? o / Ls : 0.0f;
}

// ---------------------------------------------------------------------------------
// fp16 comparison kernel: one CTA per (split, sequence, kv head), warps take tokens
// round-robin; lane l owns channels 2l, 2l+1 (pairs i0, i1) and their partners
// 2l+64, 2l+65.  Each lane advances its own (cos, sin) by a fixed rotation of
// 4*theta per step from a binary64 base at every chunk start.
constexpr int kF16Threads = 128;
constexpr int kF16Warps = kF16Threads / 32;

__global__ void __launch_bounds__(kF16Threads) k_fp16_attn(kvq_cfg cfg, const uint16_t* __restrict__ K,
                                                           const uint16_t* __restrict__ V, int Tst,
                                                           const int32_t* __restrict__ lens,
                                                           const uint16_t* __restrict__ q,
                                                           const int32_t* __restrict__ qpos, int Ls,
                                                           int S, int max_len, float2* __restrict__ st,
                                                           float* __restrict__ po) {
    __shared__ float wm[kF16Warps][kMaxG], wl[kF16Warps][kMaxG];
    __shared__ float wo[kF16Warps][kMaxG][kD];
    const int s = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int len = min(lens[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    const int i0 = 2 * lane, i1 = 2 * lane + 1;
    const double th0 = rope_freq(cfg.rope_theta, i0), th1 = rope_freq(cfg.rope_theta, i1);
    float qa0[kMaxG], qb0[kMaxG], qa1[kMaxG], qb1[kMaxG];
    float mst[kMaxG], lst[kMaxG], o[kMaxG][4];
    {
        double c0, s0, c1, s1;
        rope_cs64((double)qpos[b], th0, &c0, &s0);
        rope_cs64((double)qpos[b], th1, &c1, &s1);
#pragma unroll
        for (int a = 0; a < kMaxG; ++a) {
            mst[a] = -INFINITY;
            lst[a] = 0.0f;
            o[a][0] = o[a][1] = o[a][2] = o[a][3] = 0.0f;
            qa0[a] = qb0[a] = qa1[a] = qb1[a] = 0.0f;
            if (a < g) {
                const uint16_t* qv = q + ((size_t)b * Hq + h * g + a) * kD;
                const double xa0 = h2f(qv[i0]), xb0 = h2f(qv[i0 + kPairs]);
                const double xa1 = h2f(qv[i1]), xb1 = h2f(qv[i1 + kPairs]);
                qa0[a] = (float)((xa0 * c0 - xb0 * s0) * (double)kInvSqrtD);
                qb0[a] = (float)((xa0 * s0 + xb0 * c0) * (double)kInvSqrtD);
                qa1[a] = (float)((xa1 * c1 - xb1 * s1) * (double)kInvSqrtD);
                qb1[a] = (float)((xa1 * s1 + xb1 * c1) * (double)kInvSqrtD);
            }
        }
    }
    float sd0, cd0, sd1, cd1;
    {
        double c, s_;
        rope_cs64((double)kF16Warps, th0, &c, &s_);
        cd0 = (float)c; sd0 = (float)s_;
        rope_cs64((double)kF16Warps, th1, &c, &s_);
        cd1 = (float)c; sd1 = (float)s_;
    }
    for (int tc = t_begin; tc < t_end; tc += kChunk) {
        float c0, s0, c1, s1;
        {
            double c, s_;
            rope_cs64((double)(tc + warp), th0, &c, &s_);
            c0 = (float)c; s0 = (float)s_;
            rope_cs64((double)(tc + warp), th1, &c, &s_);
            c1 = (float)c; s1 = (float)s_;
        }
        for (int dt = warp; dt < kChunk; dt += kF16Warps) {
            const int t = tc + dt;
            if (t >= t_end) break;
            const size_t rb = (((size_t)b * Tst + t) * Hkv + h) * kD;
            const __half2 ka = *(const __half2*)(K + rb + i0);
            const __half2 kb = *(const __half2*)(K + rb + i0 + kPairs);
            const __half2 va = *(const __half2*)(V + rb + i0);
            const __half2 vb = *(const __half2*)(V + rb + i0 + kPairs);
            const float2 fka = __half22float2(ka), fkb = __half22float2(kb);
            const float2 fva = __half22float2(va), fvb = __half22float2(vb);
            const float ra0 = fka.x * c0 - fkb.x * s0, rb0 = fka.x * s0 + fkb.x * c0;
            const float ra1 = fka.y * c1 - fkb.y * s1, rb1 = fka.y * s1 + fkb.y * c1;
#pragma unroll
            for (int a = 0; a < kMaxG; ++a) {
                if (a < g) {
                    const float lg = warp_sum(qa0[a] * ra0 + qb0[a] * rb0 + qa1[a] * ra1 + qb1[a] * rb1);
                    const float mn = fmaxf(mst[a], lg);
                    const float sc = expf(mst[a] - mn);
                    const float pp = expf(lg - mn);
                    lst[a] = lst[a] * sc + pp;
                    o[a][0] = o[a][0] * sc + pp * fva.x;
                    o[a][1] = o[a][1] * sc + pp * fva.y;
                    o[a][2] = o[a][2] * sc + pp * fvb.x;
                    o[a][3] = o[a][3] * sc + pp * fvb.y;
                    mst[a] = mn;
                }
            }
            const float n0 = c0 * cd0 - s0 * sd0, m0 = s0 * cd0 + c0 * sd0;
            const float n1 = c1 * cd1 - s1 * sd1, m1 = s1 * cd1 + c1 * sd1;
            c0 = n0; s0 = m0; c1 = n1; s1 = m1;
        }
    }
#pragma unroll
    for (int a = 0; a < kMaxG; ++a) {
        if (a < g) {
            if (lane == 0) { wm[warp][a] = mst[a]; wl[warp][a] = lst[a]; }
            wo[warp][a][i0] = o[a][0];
            wo[warp][a][i1] = o[a][1];
            wo[warp][a][i0 + kPairs] = o[a][2];
            wo[warp][a][i1 + kPairs] = o[a][3];
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < g * kD; idx += blockDim.x) {
        const int a = idx / kD, ch = idx % kD;
        float M = -INFINITY;
        for (int w = 0; w < kF16Warps; ++w) M = fmaxf(M, wm[w][a]);
        float Ls_ = 0.0f, oo = 0.0f;
        if (M > -INFINITY)
            for (int w = 0; w < kF16Warps; ++w)
                if (wl[w][a] > 0.0f) {
                    const float sc = expf(wm[w][a] - M);
                    Ls_ += wl[w][a] * sc;
                    oo += wo[w][a][ch] * sc;
                }
        const size_t r = (size_t)b * Hq + h * g + a;
        po[(r * S + s) * kD + ch] = oo;
        if (ch == 0) st[r * S + s] = make_float2(M, Ls_);
    }
}

}  // namespace

using namespace kvq_host;

static int auto_splits(const kvq_cfg* cfg, int max_len) {
    // about four CTAs per SM over (splits x sequences x 16-query-head groups), >= 128 tokens each
    const int groups = cfg->B * ((cfg->Hq + 15) / 16);
    int S = (4 * 148 + groups - 1) / groups;
    const int maxs = (max_len + 127) / 128;
    if (S > maxs) S = maxs;
    if (S < 1) S = 1;
    if (S > 4096) S = 4096;
    return S;
}

static int resolve_splits(const kvq_cfg* cfg, int max_len, int splits, int* S, int* Ls) {
    if (splits < 0 || splits > 4096) return KVQ_ERR_RANGE;
    *S = splits ? splits : auto_splits(cfg, max_len);
    *Ls = split_len(max_len, *S);
    return KVQ_OK;
}

extern "C" int kvq_decode_splits(const kvq_cfg* cfg, int32_t max_len) {
    if (check_cfg(cfg) || max_len < 1) return 1;
    return auto_splits(cfg, max_len);
}

static int check_decode(const kvq_cfg* cfg, int max_len) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (max_len < 1 || max_len > cfg->T_max) return KVQ_ERR_RANGE;
    if (cfg->Hq / cfg->Hkv > kMaxG) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

template <int BITS>
static int launch_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                     const uint16_t* q, const int32_t* qpos, int max_len, float* logits,
                     float* stats, int S, int Ls, cudaStream_t st) {
    const size_t smem = QKSmem::total;
    cudaError_t ce = cudaFuncSetAttribute(k_qk2<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B, (cfg->Hq + kQKHeads - 1) / kQKHeads);
    k_qk2<BITS><<<grid, kQKThreads, smem, st>>>(*cfg, *cache, *cbK, q, qpos, Ls, S, max_len,
                                                 logits, (float2*)stats);
    return record_cuda(cudaGetLastError());
}

extern "C" int kvq_decode_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                             const uint16_t* q, const int32_t* qpos, int32_t max_len,
                             float* logits, float* stats, int32_t splits, void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if ((e = check_cache(cfg, cache)) || (e = check_codebook(cbK))) return e;
    if (!q || !qpos || !logits || !stats) return KVQ_ERR_NULL;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    cudaStream_t st = (cudaStream_t)stream;
    switch (cfg->bits) {
        case 2: return launch_qk<2>(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, Ls, st);
        case 3: return launch_qk<3>(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, Ls, st);
        default: return launch_qk<4>(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, Ls, st);
    }
}

extern "C" int kvq_softmax_merge(const kvq_cfg* cfg, const float* stats, int32_t splits,
                                 float* ml, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!stats || !ml) return KVQ_ERR_NULL;
    if (splits < 1 || splits > 4096) return KVQ_ERR_RANGE;
    const int BH = cfg->B * cfg->Hq;
    k_softmax_merge<<<(BH + 127) / 128, 128, 0, (cudaStream_t)stream>>>(BH, splits,
                                                                         (const float2*)stats,
                                                                         (float2*)ml);
    return record_cuda(cudaGetLastError());
}

template <int BITS>
static int launch_pv(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbV,
                     const float* logits, const float* ml, int max_len, float* part, int S,
                     int Ls, cudaStream_t st) {
    const size_t smem = PVSmem::total;
    cudaError_t ce = cudaFuncSetAttribute(k_pv2<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B, (cfg->Hq + kPVHeads - 1) / kPVHeads);
    k_pv2<BITS><<<grid, kPVThreads, smem, st>>>(*cfg, *cache, *cbV, logits, (const float2*)ml, Ls,
                                                 S, max_len, part);
    return record_cuda(cudaGetLastError());
}

extern "C" int kvq_decode_pv(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbV,
                             const float* logits, const float* ml, int32_t max_len, float* out,
                             float* part, int32_t splits, void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if ((e = check_cache(cfg, cache)) || (e = check_codebook(cbV))) return e;
    if (!logits || !ml || !out || !part) return KVQ_ERR_NULL;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    cudaStream_t st = (cudaStream_t)stream;
    switch (cfg->bits) {
        case 2: e = launch_pv<2>(cfg, cache, cbV, logits, ml, max_len, part, S, Ls, st); break;
        case 3: e = launch_pv<3>(cfg, cache, cbV, logits, ml, max_len, part, S, Ls, st); break;
        default: e = launch_pv<4>(cfg, cache, cbV, logits, ml, max_len, part, S, Ls, st); break;
    }
    if (e) return e;
    k_pv_reduce<<<cfg->B * cfg->Hq, kD, 0, st>>>(S, part, out);
    return record_cuda(cudaGetLastError());
}

static size_t split_ws_bytes(const kvq_cfg* cfg, int S, int max_len) {
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    return align_up(BH * (size_t)cfg->T_max * 4)   // logits
           + align_up(BH * S * 8)                  // stats
           + align_up(BH * 8)                      // ml
           + align_up(BH * S * kD * 4);            // partials
}

extern "C" int kvq_decode_workspace(const kvq_cfg* cfg, int32_t max_len, int32_t splits,
                                    size_t* bytes) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    *bytes = split_ws_bytes(cfg, S, max_len);
    return KVQ_OK;
}

extern "C" int kvq_decode_attention(const kvq_cfg* cfg, const kvq_cache* cache,
                                    const kvq_codebook* cbK, const kvq_codebook* cbV,
                                    const uint16_t* q, const int32_t* qpos, int32_t max_len,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    int32_t splits, void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if (!workspace || !out) return KVQ_ERR_NULL;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    if (workspace_bytes < split_ws_bytes(cfg, S, max_len)) return KVQ_ERR_WORKSPACE;
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    char* w = (char*)workspace;
    float* logits = (float*)w;
    w += align_up(BH * (size_t)cfg->T_max * 4);
    float* stats = (float*)w;
    w += align_up(BH * S * 8);
    float* ml = (float*)w;
    w += align_up(BH * 8);
    float* part = (float*)w;
    if ((e = kvq_decode_qk(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, stream))) return e;
    if ((e = kvq_softmax_merge(cfg, stats, S, ml, stream))) return e;
    return kvq_decode_pv(cfg, cache, cbV, logits, ml, max_len, out, part, S, stream);
}

extern "C" int kvq_fp16_decode_attention(const kvq_cfg* cfg, const uint16_t* K, const uint16_t* V,
                                         int32_t T_stride, const int32_t* len, const uint16_t* q,
                                         const int32_t* qpos, int32_t max_len, float* out,
                                         void* workspace, size_t workspace_bytes, int32_t splits,
                                         void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if (!K || !V || !len || !q || !qpos || !out || !workspace) return KVQ_ERR_NULL;
    if (!aligned16(K) || !aligned16(V) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
    if (T_stride < max_len) return KVQ_ERR_RANGE;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    const size_t need = align_up(BH * S * 8) + align_up(BH * S * kD * 4);
    if (workspace_bytes < need) return KVQ_ERR_WORKSPACE;
    float2* st = (float2*)workspace;
    float* po = (float*)((char*)workspace + align_up(BH * S * 8));
    cudaStream_t s = (cudaStream_t)stream;
    dim3 grid(S, cfg->B, cfg->Hkv);
    k_fp16_attn<<<grid, kF16Threads, 0, s>>>(*cfg, K, V, T_stride, len, q, qpos, Ls, S, max_len,
                                             st, po);
    k_attn_merge<<<(int)BH, kD, 0, s>>>(S, st, po, out);
    return record_cuda(cudaGetLastError());
}
