// Decode attention over the quantized cache (read side of techniques (i)-(iv)):
// QK with NUQ lookup + on-the-fly RoPE + key-outlier correction, split-K softmax
// statistics and merge, and the probability-weighted value sum with value-outlier
// replacement.  Also the uncompressed fp16 comparison kernel.
#include "kvq_common.cuh"

using namespace kvq;

namespace {

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kMaxHqSplit = 32;                    // query heads per CTA of the split QK
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

// Per-CTA RoPE tables: step[dt][i] = (cos, sin)(dt * theta_i) for dt < 64 and the
// per-chunk base (cos, sin)(t0 * theta_i) in binary64; cs = base (x) step.
__device__ void rope_step_table(const double* theta, float2* step) {
    for (int idx = threadIdx.x; idx < kChunk * kPairs; idx += blockDim.x) {
        const int dt = idx / kPairs, i = idx % kPairs;
        float s, c;
        sincosf((float)dt * (float)theta[i], &s, &c);
        step[idx] = make_float2(c, s);
    }
}

__device__ void rope_chunk_table(int t0, const double* theta, const float2* step, float2* base,
                                 float2* cs) {
    if (threadIdx.x < kPairs) {
        double c, s;
        rope_cs64((double)t0, theta[threadIdx.x], &c, &s);
        base[threadIdx.x] = make_float2((float)c, (float)s);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kChunk * kPairs; idx += blockDim.x) {
        const int i = idx % kPairs;
        const float2 a = base[i], d = step[idx];
        cs[idx] = make_float2(a.x * d.x - a.y * d.y, a.y * d.x + a.x * d.y);
    }
}

// ---------------------------------------------------------------------------------
// QK: one CTA per (split, sequence), all heads; warp per token, lanes own pairs
// (lane, lane + 32).
constexpr int kQKThreads = 256;

struct QKSm {
    size_t cs, step, coef, qr, lev, wst, base, theta, total;
};

__host__ __device__ inline QKSm qk_smem(int Hq) {
    QKSm s;
    size_t o = 0;
    s.cs = o; o += kChunk * kPairs * sizeof(float2);
    s.step = o; o += kChunk * kPairs * sizeof(float2);
    s.coef = o; o += (size_t)Hq * kPairs * 2 * sizeof(float4);
    s.qr = o; o += (size_t)Hq * kD * sizeof(float);
    s.lev = o; o += 16 * sizeof(float);
    s.wst = o; o += (size_t)(kQKThreads / 32) * Hq * sizeof(float2);
    s.base = o; o += kPairs * sizeof(float2);
    s.theta = o; o += kPairs * sizeof(double);
    s.total = o;
    return s;
}

// Rotate the query of heads [hq0, hq0 + nh) at position qpos (binary64 angles) and
// scale by 1/sqrt(D); qcs is block scratch for the 64 (cos, sin) pairs.
__device__ void rotate_query(const uint16_t* q, int b, int hq0, int nh, int Hq, int qpos,
                             const double* theta, float* qr, double2* qcs) {
    if (threadIdx.x < kPairs) {
        double c, s;
        rope_cs64((double)qpos, theta[threadIdx.x], &c, &s);
        qcs[threadIdx.x] = make_double2(c, s);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < nh * kPairs; idx += blockDim.x) {
        const int hh = idx / kPairs, i = idx % kPairs;
        const uint16_t* qv = q + ((size_t)b * Hq + hq0 + hh) * kD;
        const double c = qcs[i].x, s = qcs[i].y;
        const double qa = (double)h2f(qv[i]), qb = (double)h2f(qv[i + kPairs]);
        qr[hh * kD + i] = (float)((qa * c - qb * s) * (double)kInvSqrtD);
        qr[hh * kD + i + kPairs] = (float)((qa * s + qb * c) * (double)kInvSqrtD);
    }
}

__global__ void __launch_bounds__(kQKThreads) k_qk(kvq_cfg cfg, kvq_cache c, kvq_codebook cb,
                                                   const uint16_t* __restrict__ q,
                                                   const int32_t* __restrict__ qpos, int Ls, int S,
                                                   int max_len, float* __restrict__ logits,
                                                   float2* __restrict__ stats) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv, bits = cfg.bits, W = row_words(bits);
    const QKSm L = qk_smem(Hq);
    float2* cs = (float2*)(sm + L.cs);
    float2* step = (float2*)(sm + L.step);
    float4* coef = (float4*)(sm + L.coef);
    float* qr = (float*)(sm + L.qr);
    float* lev = (float*)(sm + L.lev);
    float2* wst = (float2*)(sm + L.wst);
    float2* base = (float2*)(sm + L.base);
    double* theta = (double*)(sm + L.theta);
    __shared__ double2 qcs[kPairs];
    const int s = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int len = c.len[b];
    if (len > max_len) {
        if (threadIdx.x == 0 && s == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (threadIdx.x < kPairs) theta[threadIdx.x] = rope_freq(cfg.rope_theta, threadIdx.x);
    if (threadIdx.x < (1 << bits)) lev[threadIdx.x] = cb.levels[threadIdx.x];
    for (int i = threadIdx.x; i < (kQKThreads / 32) * Hq; i += blockDim.x)
        wst[i] = make_float2(-INFINITY, 0.0f);
    __syncthreads();
    if (t_begin < t_end) {
        rope_step_table(theta, step);
        rotate_query(q, b, 0, Hq, Hq, qpos[b], theta, qr, qcs);
        __syncthreads();
        const float* kp = c.kparams + (size_t)b * Hkv * kD * 2;
        for (int idx = threadIdx.x; idx < Hq * kPairs; idx += blockDim.x) {
            const int hq = idx / kPairs, i = idx % kPairs, h = hq / g;
            const int ja = h * kD + i, jb = ja + kPairs;
            const float offa = kp[2 * ja], halfa = kp[2 * ja + 1];
            const float offb = kp[2 * jb], halfb = kp[2 * jb + 1];
            const float qa = qr[hq * kD + i], qb = qr[hq * kD + i + kPairs];
            coef[idx * 2 + 0] = make_float4(qa * halfa, qb * halfb, qa * offa + qb * offb, qb * halfa);
            coef[idx * 2 + 1] = make_float4(-qa * halfb, qb * offa - qa * offb, 0.0f, 0.0f);
        }
        __syncthreads();
        const int nch1 = nchunks(cfg.T_max) + 1;
        const uint32_t* chunk = c.kchunk + (size_t)b * nch1;
        const uint32_t kcount = c.kcount[b];
        const uint32_t* opos = c.kout_pos + (size_t)b * cfg.out_cap_k;
        const uint16_t* oval = c.kout_val + (size_t)b * cfg.out_cap_k;
        const uint32_t fmask = (1u << bits) - 1u;
        for (int tc = t_begin; tc < t_end; tc += kChunk) {
            rope_chunk_table(tc, theta, step, base, cs);
            __syncthreads();
            const int m = tc / kChunk;
            const uint32_t lo = min(chunk[m], kcount);
            const uint32_t hi = min(chunk[m + 1], kcount);
            for (int dt = warp; dt < kChunk; dt += kQKThreads / 32) {
                const int t = tc + dt;
                if (t >= t_end) break;
                // first entry of this token: lower bound of (dt << 16)
                uint32_t a = lo, z = hi;
                const uint32_t key0 = (uint32_t)dt << 16;
                while (a < z) {
                    const uint32_t mid = (a + z) >> 1;
                    if (opos[mid] < key0) a = mid + 1; else z = mid;
                }
                uint32_t cur = a;
                const uint32_t* rowbase = c.kcodes + ((size_t)b * cfg.T_max + t) * Hkv * W;
                const float2 cs0 = cs[dt * kPairs + lane], cs1 = cs[dt * kPairs + lane + 32];
                for (int h = 0; h < Hkv; ++h) {
                    const uint32_t* row = rowbase + h * W;
                    const uint32_t fa = k_pair_field(row, bits, lane);
                    const uint32_t fb = k_pair_field(row, bits, lane + 32);
                    const float La0 = lev[fa & fmask], Lb0 = lev[fa >> bits];
                    const float La1 = lev[fb & fmask], Lb1 = lev[fb >> bits];
                    const uint32_t lim = key0 | (uint32_t)((h + 1) * kD);
                    uint32_t segend = cur;
                    while (true) {
                        const uint32_t e = segend + lane;
                        const bool in = e < hi && opos[e] < lim;
                        const uint32_t bal = __ballot_sync(0xffffffffu, in);
                        const int nin = __popc(bal);
                        segend += nin;
                        if (nin < 32) break;
                    }
                    for (int hq = h * g; hq < h * g + g; ++hq) {
                        const float4 p0 = coef[(hq * kPairs + lane) * 2], p1 = coef[(hq * kPairs + lane) * 2 + 1];
                        const float4 r0 = coef[(hq * kPairs + lane + 32) * 2];
                        const float4 r1 = coef[(hq * kPairs + lane + 32) * 2 + 1];
                        const float X0 = p0.z + p0.x * La0 + p0.y * Lb0;
                        const float Y0 = p1.y + p0.w * La0 + p1.x * Lb0;
                        const float X1 = r0.z + r0.x * La1 + r0.y * Lb1;
                        const float Y1 = r1.y + r0.w * La1 + r1.x * Lb1;
                        float part = cs0.x * X0 + cs0.y * Y0 + cs1.x * X1 + cs1.y * Y1;
                        for (uint32_t e = cur + lane; e < segend; e += 32) {
                            const uint32_t p = opos[e];
                            const int ch = (int)(p & 0xffffu) - h * kD;
                            if (ch < 0 || ch >= kD) continue;
                            const float x = h2f(oval[e]);
                            const uint32_t code = k_code(row, bits, ch);
                            const int j = h * kD + ch;
                            const float zhat = kp[2 * j] + kp[2 * j + 1] * lev[code];
                            const int i = ch & (kPairs - 1);
                            const float2 cc = cs[dt * kPairs + i];
                            const float qa = qr[hq * kD + i], qb = qr[hq * kD + i + kPairs];
                            const float r = (ch < kPairs) ? (cc.x * qa + cc.y * qb) : (cc.x * qb - cc.y * qa);
                            part += (x - zhat) * r;
                        }
                        const float lg = warp_sum(part);
                        if (lane == 0) {
                            logits[((size_t)b * Hq + hq) * cfg.T_max + t] = lg;
                            float2 st = wst[warp * Hq + hq];
                            if (lg > st.x) {
                                st.y = st.y * expf(st.x - lg) + 1.0f;
                                st.x = lg;
                            } else {
                                st.y += expf(lg - st.x);
                            }
                            wst[warp * Hq + hq] = st;
                        }
                    }
                    cur = segend;
                }
            }
            __syncthreads();
        }
    }
    __syncthreads();
    for (int hq = threadIdx.x; hq < Hq; hq += blockDim.x) {
        float mm = -INFINITY;
        for (int w = 0; w < kQKThreads / 32; ++w) mm = fmaxf(mm, wst[w * Hq + hq].x);
        float ll = 0.0f;
        if (mm > -INFINITY)
            for (int w = 0; w < kQKThreads / 32; ++w) {
                const float2 st = wst[w * Hq + hq];
                if (st.y > 0.0f) ll += st.y * expf(st.x - mm);
            }
        stats[((size_t)b * Hq + hq) * S + s] = make_float2(mm, ll);
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

// ---------------------------------------------------------------------------------
// PV: one CTA per (split, sequence, kv head); thread = channel.
constexpr int kPVThreads = 128;

__global__ void __launch_bounds__(kPVThreads) k_pv(kvq_cfg cfg, kvq_cache c, kvq_codebook cb,
                                                   const float* __restrict__ logits,
                                                   const float2* __restrict__ ml, int Ls, int S,
                                                   int max_len, float* __restrict__ part) {
    __shared__ float p[kMaxG][kChunk];
    __shared__ float2 vpar[kChunk];
    __shared__ float ov[kChunk][kD];
    __shared__ uint8_t fl[kChunk][kD];
    __shared__ float lev[16];
    const int s = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv, bits = cfg.bits, W = row_words(bits);
    const int ch = threadIdx.x;
    const int len = min(c.len[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (threadIdx.x < (1 << bits)) lev[threadIdx.x] = cb.levels[threadIdx.x];
    float acc[kMaxG];
#pragma unroll
    for (int a = 0; a < kMaxG; ++a) acc[a] = 0.0f;
    const int nch1 = nchunks(cfg.T_max) + 1;
    const uint32_t* chunk = c.vchunk + (size_t)b * nch1;
    const uint32_t vcount = c.vcount[b];
    const uint32_t* opos = c.vout_pos + (size_t)b * cfg.out_cap_v;
    const uint16_t* oval = c.vout_val + (size_t)b * cfg.out_cap_v;
    for (int tc = t_begin; tc < t_end; tc += kChunk) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < g * kChunk; idx += blockDim.x) {
            const int a = idx / kChunk, dt = idx % kChunk, t = tc + dt;
            const int hq = h * g + a;
            float pv = 0.0f;
            if (t < t_end) {
                const float2 mL = ml[(size_t)b * Hq + hq];
                pv = expf(logits[((size_t)b * Hq + hq) * cfg.T_max + t] - mL.x) / mL.y;
            }
            p[a][dt] = pv;
        }
        for (int dt = threadIdx.x; dt < kChunk; dt += blockDim.x) {
            const int t = tc + dt;
            vpar[dt] = t < t_end ? *(const float2*)(c.vparams + ((size_t)b * cfg.T_max + t) * 2)
                                 : make_float2(0.0f, 0.0f);
        }
        for (int idx = threadIdx.x; idx < kChunk * kD; idx += blockDim.x) (&fl[0][0])[idx] = 0;
        __syncthreads();
        const int m = tc / kChunk;
        const uint32_t lo = min(chunk[m], vcount), hi = min(chunk[m + 1], vcount);
        for (uint32_t e = lo + threadIdx.x; e < hi; e += blockDim.x) {
            const uint32_t pp = opos[e];
            const int j = (int)(pp & 0xffffu);
            if (j / kD == h && (pp >> 16) < (uint32_t)kChunk) {
                const int dt = (int)(pp >> 16);
                ov[dt][j % kD] = h2f(oval[e]);
                fl[dt][j % kD] = 1;
            }
        }
        __syncthreads();
        for (int dt = 0; dt < kChunk; ++dt) {
            const int t = tc + dt;
            if (t >= t_end) break;
            const uint32_t* row = c.vcodes + (((size_t)b * cfg.T_max + t) * Hkv + h) * W;
            const uint32_t code = v_code(row, bits, ch);
            const float vv = fl[dt][ch] ? ov[dt][ch] : vpar[dt].x + vpar[dt].y * lev[code];
#pragma unroll
            for (int a = 0; a < kMaxG; ++a)
                if (a < g) acc[a] += p[a][dt] * vv;
        }
    }
#pragma unroll
    for (int a = 0; a < kMaxG; ++a)
        if (a < g) part[(((size_t)b * Hq + h * g + a) * S + s) * kD + ch] = acc[a];
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
    int S = (2 * 148 + cfg->B - 1) / cfg->B;
    const int maxs = (max_len + 255) / 256;
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

extern "C" int kvq_decode_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                             const uint16_t* q, const int32_t* qpos, int32_t max_len,
                             float* logits, float* stats, int32_t splits, void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if ((e = check_cache(cfg, cache)) || (e = check_codebook(cbK))) return e;
    if (!q || !qpos || !logits || !stats) return KVQ_ERR_NULL;
    if (cfg->Hq > kMaxHqSplit) return KVQ_ERR_UNSUPPORTED;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    const QKSm L = qk_smem(cfg->Hq);
    cudaError_t ce = cudaFuncSetAttribute(k_qk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)L.total);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B);
    k_qk<<<grid, kQKThreads, L.total, (cudaStream_t)stream>>>(*cfg, *cache, *cbK, q, qpos, Ls, S,
                                                              max_len, logits, (float2*)stats);
    return record_cuda(cudaGetLastError());
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
    dim3 grid(S, cfg->B, cfg->Hkv);
    k_pv<<<grid, kPVThreads, 0, st>>>(*cfg, *cache, *cbV, logits, (const float2*)ml, Ls, S,
                                      max_len, part);
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
