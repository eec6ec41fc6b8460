// Decode attention over the quantized cache (read side of techniques (i)-(iv)):
// QK with NUQ lookup + on-the-fly RoPE, key-outlier correction, split-K softmax
// statistics and merge, the probability-weighted value sum and the value-outlier
// correction.  Also the uncompressed fp16 comparison kernel.
//
// The two streaming kernels share one shape.  A CTA covers HPC query heads over one split of
// the tokens and walks it in 64-token chunks.  The chunk's code blocks (one contiguous run of
// 16 blocks per kv head) arrive in a ring of shared-memory stages filled by bulk copies
// (cp.async.bulk into the CTA's own shared memory, completion counted on an mbarrier) that
// the last warp issues.
// Half-warp qd of a consumer warp takes token quad qd of the chunk and lane i of the
// half-warp the rotate-half pairs (c, c + 64), c = i + 16k: exactly the lane group i of the
// code block, whose token slot s holds token s ^ (i >> 2) (the rotation that lets QK reduce
// its partials per lane across the half-warp with plain shuffles).  Consumer warps meet only
// the stage barriers.  The sparse outliers are applied by separate kernels that walk the
// outlier lists chunk by chunk: key outliers add (x - zhat) times the rotated query component
// to the logits before the softmax statistics are taken, value outliers add
// p (x - zhat) to the output after the merge.
#include <cooperative_groups.h>

#include "kvq_common.cuh"
#include "kvq_device.cuh"

using namespace kvq;

namespace {

constexpr int kThreads = 256;                      // 8 warps = 16 half-warps
constexpr int kQuads = kThreads / 16;              // token quads per chunk (64 tokens)
constexpr int kStages = 4;                         // chunks in the bulk-copy ring

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

// Consumer warps of a CTA (one more warp streams the input) and heads per consumer warp.
// With four query heads per CTA two warps share each quad pair (two heads each): twice the
// warps to hide latency, at the price of computing a lane's RoPE phases for two heads instead
// of four.
__host__ __device__ constexpr int qk_warps(int hpc) { return hpc == 4 ? 16 : 8; }
__host__ __device__ constexpr int pv_warps(int hpc) { return hpc == 4 ? 16 : 8; }
template <int HPC, int CW>
__host__ __device__ constexpr int heads_per_warp() { return HPC * 8 / CW; }
template <int HW>
__device__ __forceinline__ int out_head(int i) {
    return HW == 4 ? (i & 3) : (HW == 2 ? ((i >> 1) & 1) : 0);
}
template <int HW>
__device__ __forceinline__ bool out_owner(int i) {
    return HW == 4 ? true : (HW == 2 ? !(i & 1) : !(i & 3));
}


// ---------------------------------------------------------------------------------
// Shared-memory plans (host and device).
struct QKPlan {
    int tab, ring, pitch, stage, base, rs, qr, bar, flag, total;
};
__host__ __device__ inline QKPlan qk_plan(int bits, int hpc, int kvb) {
    QKPlan p;
    int o = 0;
    p.tab = o;  o += hpc * 64 * (1 << (2 * bits)) * 8;       // [entry][head][pair] (X, Y)
    p.pitch = kQuads * 16 * bits * 4;                         // code blocks of one kv head
    p.stage = kvb * p.pitch;
    p.ring = o; o += kStages * p.stage;
    p.base = o; o += kStages * 64 * 8;                        // [stage][64] (cos, sin) at chunk start
    p.rs = o;   o += 64 * 64 * 8;                             // [token of chunk][pair] rotation
    p.qr = o;   o += hpc * 128 * 4;                           // rotated, scaled queries
    p.bar = o;  o += 2 * kStages * 8;                         // full, empty
    p.flag = o; o += 16;
    p.total = o;
    return p;
}

struct PVPlan {
    int tab, ring, pitch, stage, wsm, bar, flag, total;
};
__host__ __device__ inline PVPlan pv_plan(int bits, int hpc, int kvb) {
    PVPlan p;
    int o = 0;
    p.tab = o;  o += (1 << (2 * bits)) * 16 * 8;              // [entry][16 lane copies] (La, Lb)
    p.pitch = kQuads * 16 * bits * 4;
    p.stage = kvb * p.pitch;
    p.ring = o;
    {
        const int ring = kStages * p.stage, red = kQuads * hpc * 128 * 4;
        o += ring > red ? ring : red;                         // reused by the final reduction
    }
    p.wsm = o;  o += kQuads * 4 * hpc * 8;                    // [quad][token][head] (w, w)
    p.bar = o;  o += 2 * kStages * 8;                         // full, empty
    p.flag = o; o += 16;
    p.total = o;
    return p;
}

// Thread 0 of the streaming warp: bulk copies of the chunk's code blocks, one contiguous run
// of 16 blocks per kv head of the CTA, into the chunk's stage (kv head k at k * pitch).
struct Streamer {
    uint8_t* ring;
    uint64_t* full;
    int pitch, stage, kvb, t_begin, t_end;
    const uint32_t* src0;  // code blocks of (sequence, first kv head), quad 0
    size_t head_stride;    // words between the blocks of consecutive kv heads
    uint32_t quad_bytes;   // bytes of one code block

    __device__ void issue(int cc) {
        const int tc = t_begin + cc * kChunk;
        const int q0 = tc >> 2, q1 = (min(tc + kChunk, t_end) + 3) >> 2;
        uint64_t* bar = full + cc % kStages;
        uint8_t* dst = ring + (size_t)(cc % kStages) * stage;
        const uint32_t bytes = (uint32_t)(q1 - q0) * quad_bytes;
        mbar_arrive_expect_tx(bar, (uint32_t)kvb * bytes);
        for (int k = 0; k < kvb; ++k)
            bulk_load(dst + k * pitch, src0 + (size_t)k * head_stride + (size_t)q0 * (quad_bytes / 4),
                      bytes, bar);
    }
};

// ---------------------------------------------------------------------------------
// Per-call tables: rotated, scaled queries qr [B][Hq][128]; trig tables hi [nhi][64] =
// (cos, sin)((256 j + pos_off) theta_p), lo [256][64] = (cos, sin)(tau theta_p), all from
// binary64, so that hi[t / 256] lo[t % 256] is the rotation of cache row t at position
// t + pos_off; the dense key value at an outlier zk [B][Hkv][128] = off + half * L[encode(
// normalize(0))].
__global__ void k_decode_prep(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const uint16_t* q,
                              const int32_t* qpos, int nhi, int pos_off, float* qr, float2* thi,
                              float2* tlo, float* zk) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int nq = cfg.B * cfg.Hq * 64, nh = nhi * 64, nl = kTrigLo * 64, nz = cfg.B * cfg.Hkv * kD;
    if (e < nq) {
        const int p = e & 63, bh = e >> 6, b = bh / cfg.Hq;
        const double th = rope_freq(cfg.rope_theta, p);
        double cq, sq;
        rope_cs64((double)qpos[b], th, &cq, &sq);
        const uint16_t* qv = q + (size_t)bh * kD;
        const double qa = (double)h2f(qv[p]), qb = (double)h2f(qv[p + 64]);
        qr[(size_t)bh * kD + p] = (float)((qa * cq - qb * sq) * (double)kInvSqrtD);
        qr[(size_t)bh * kD + p + 64] = (float)((qa * sq + qb * cq) * (double)kInvSqrtD);
    } else if (e < nq + nh) {
        const int f = e - nq, p = f & 63, j = f >> 6;
        double cc, ss;
        rope_cs64((double)j * kTrigLo + (double)pos_off, rope_freq(cfg.rope_theta, p), &cc, &ss);
        thi[f] = make_float2((float)cc, (float)ss);
    } else if (e < nq + nh + nl) {
        const int f = e - nq - nh, p = f & 63, j = f >> 6;
        double cc, ss;
        rope_cs64((double)j, rope_freq(cfg.rope_theta, p), &cc, &ss);
        tlo[f] = make_float2((float)cc, (float)ss);
    } else if (e < nq + nh + nl + nz) {
        const int f = e - nq - nh - nl;
        const int nb = (1 << cfg.bits) - 1;
        const float* kp = c.kparams + (size_t)f * 2;  // [B][Hkv*128] channels, in order
        const float xn = normalize(0.0f, kp[0], kp[1]);
        zk[f] = kp[0] + kp[1] * cb.levels[encode(xn, cb.bounds, nb)];
    }
}

// ---------------------------------------------------------------------------------
// QK.  Per query head and pair p the CTA tabulates, for every code pair e = (xa, xb),
//   X = qa (off_a + half_a L[xa]) + qb (off_b + half_b L[xb]),
//   Y = qb (off_a + half_a L[xa]) - qa (off_b + half_b L[xb])
// (q the query rotated to its own position and scaled by 1/sqrt(D)); the dense part of the
// logit of token t is then sum_p cos(t theta_p) X + sin(t theta_p) Y, one f32x2 FMA per pair
// and token.  The (cos, sin) of a lane's tokens are the chunk's base times fixed rotations.
// A consumer warp takes two token quads and HW of the CTA's heads; lane i's accumulator slot
// (token s, head h) holds token s ^ (i >> 2) and head h ^ hperm(i), so the 4*HW partials
// reduce across the half-warp by halving.  The last warp streams the chunks and the chunk
// base angles.
template <int BITS, int HPC, bool SHARE>
__global__ void __launch_bounds__(qk_warps(HPC) * 32 + 32, 1)
    k_qk(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ qr_all,
         const float2* __restrict__ thi, const float2* __restrict__ tlo, int Ls, int max_len,
         int kvb, float* __restrict__ logits) {
    using F = Fmt<BITS>;
    constexpr int CW = qk_warps(HPC), NC = CW * 32;
    constexpr int HW = heads_per_warp<HPC, CW>();
    constexpr int LH = HPC == 4 ? 2 : (HPC == 2 ? 1 : 0);
    constexpr int P = 9 + LH;  // bit of the entry index in a table byte offset
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << P;
    constexpr int NW = SHARE ? 1 : HW;
    constexpr int V = 4 * HW;  // partials per lane
    extern __shared__ __align__(128) uint8_t sm[];
    const QKPlan L = qk_plan(BITS, HPC, kvb);
    uint8_t* tab = sm + L.tab;
    uint8_t* ring = sm + L.ring;
    float2* base = (float2*)(sm + L.base);
    float2* rs = (float2*)(sm + L.rs);
    float* qr = (float*)(sm + L.qr);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x, nthr = blockDim.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5;
    const int qd = 2 * (warp & 7) + ((tid >> 4) & 1);  // token quad of the chunk
    const int hg = (warp >> 3) * HW;                     // first CTA head of the warp
    const int s = blockIdx.x, b = blockIdx.y, hq0 = blockIdx.z * HPC;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv;
    int len = c.len[b];
    if (len > max_len) {
        if (tid == 0 && s == 0 && blockIdx.z == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) return;
    const int nch = (t_end - t_begin + kChunk - 1) / kChunk;
    const int kv_first = min(hq0 / g, Hkv - kvb);
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, CW);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    // ---- per-CTA tables
    for (int e = tid; e < HPC * kD; e += nthr) qr[e] = qr_all[((size_t)b * Hq + hq0) * kD + e];
    for (int e = tid; e < 64 * 64; e += nthr) rs[e] = tlo[e];  // rotations by 0 .. 63 tokens
    __syncthreads();
    const int nb = (1 << BITS) - 1;
    const float* kp = c.kparams + (size_t)b * Hkv * kD * 2;
    for (int e = tid; e < HPC * 64 * F::NT; e += nthr) {
        const int p = e & 63, h = (e >> 6) & (HPC - 1), idx = e >> (6 + LH);
        const int kvh = (hq0 + h) / g;
        const float* pa = kp + ((size_t)kvh * kD + p) * 2;
        const float* pb = kp + ((size_t)kvh * kD + p + 64) * 2;
        const float offa = pa[0], halfa = pa[1], offb = pb[0], halfb = pb[1];
        const float qa = qr[h * kD + p], qb = qr[h * kD + p + 64];
        const float La = cb.levels[idx & nb], Lb = cb.levels[idx >> BITS];
        const float A1 = qa * halfa, B1 = qb * halfb, C1 = qa * offa + qb * offb;
        const float A2 = qb * halfa, B2 = -qa * halfb, C2 = qb * offa - qa * offb;
        const float X = fmaf(B1, Lb, fmaf(A1, La, C1));
        const float Y = fmaf(B2, Lb, fmaf(A2, La, C2));
        reinterpret_cast<unsigned long long*>(tab)[e] = pk(X, Y);
    }
    __syncthreads();  // tables complete, barriers initialised

    if (tid >= NC) {
        // ================= streaming warp
        const int pl = tid - NC;
        Streamer sr;
        sr.ring = ring;
        sr.full = full;
        sr.pitch = L.pitch;
        sr.stage = L.stage;
        sr.kvb = kvb;
        sr.t_begin = t_begin;
        sr.t_end = t_end;
        sr.src0 = c.kcodes + ((size_t)b * Hkv + kv_first) * nquads(cfg.T_max) * F::BW;
        sr.head_stride = (size_t)nquads(cfg.T_max) * F::BW;
        sr.quad_bytes = (uint32_t)F::BW * 4;
        int cc = 0;
        for (; cc < nch; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            const int tc = t_begin + cc * kChunk;
#pragma unroll
            for (int u = 0; u < 2; ++u)
                base[slot * 64 + pl + 32 * u] = trig_at(thi, tlo, tc, pl + 32 * u);
            __syncwarp();
            __threadfence_block();
            if (pl == 0) {
                fence_proxy_async();
                sr.issue(cc);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;  // chunks issued
    } else {
        // ================= consumer warps
        const int hperm = out_head<HW>(i);
        uint32_t lb[HW];
#pragma unroll
        for (int h = 0; h < HW; ++h)
            lb[h] = ((uint32_t)(hg + (h ^ hperm)) << 9) | ((uint32_t)i << 3);
        uint32_t woff[NW];
#pragma unroll
        for (int h = 0; h < NW; ++h) {
            const int kvs = SHARE ? 0 : (hq0 + hg + (h ^ hperm)) / g - kv_first;
            woff[h] = (uint32_t)(kvs * L.pitch + qd * F::BW * 4 + i * BITS * 4);
        }
        float2 RS[4][4];  // rotation from the chunk start to token 4 qd + (s ^ x), pair i + 16k
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) RS[k][sl] = rs[(4 * qd + (sl ^ x)) * 64 + i + 16 * k];
        const int hs_out = hg + hperm;  // CTA head of this lane's logit
        const bool owner = out_owner<HW>(i);
        const int tq = 4 * qd + x;
        float* lrow = logits + ((size_t)b * Hq + hq0 + hs_out) * cfg.T_max;
        for (int ch = 0; ch < nch; ++ch) {
            const int slot = ch % kStages;
            if (!mbar_wait(full + slot, (uint32_t)(ch / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[NW][BITS];
#pragma unroll
            for (int h = 0; h < NW; ++h)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[h][d] = *reinterpret_cast<const uint32_t*>(stage + woff[h] + 4 * d);
            float2 B[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) B[k] = base[slot * 64 + i + 16 * k];
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
            unsigned long long acc[4][HW];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
#pragma unroll
                for (int h = 0; h < HW; ++h) acc[sl][h] = 0ull;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    const float2 cs = cmul(B[k], RS[k][sl]);
                    const unsigned long long Pc = pk(cs.x, cs.y);
                    uint32_t fs[NW];
#pragma unroll
                    for (int h = 0; h < NW; ++h) {
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs[h] = field_to<BITS, N, P>(w[h]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                    }
#pragma unroll
                    for (int h = 0; h < HW; ++h) {
                        const uint32_t off = (fs[SHARE ? 0 : h] & MASK) | lb[h];
                        acc[sl][h] = fma2(Pc, tld(tab + 128 * k, off), acc[sl][h]);
                    }
                }
            }
            float v[V];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    const f2 a = upk(acc[sl][h]);
                    v[HW * sl + h] = a.x + a.y;
                }
            // halve across the half-warp: lane bit 3, 2, ... pairs the upper half of the partials
            int mk = 8;
#pragma unroll
            for (int half = V / 2; half >= 1; half >>= 1, mk >>= 1)
#pragma unroll
                for (int t = 0; t < half; ++t)
                    v[t] += __shfl_xor_sync(0xffffffffu, v[t + half], mk);
#pragma unroll
            for (int m2 = 16 / V / 2; m2 >= 1; m2 >>= 1)
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], m2);
            const int t = t_begin + ch * kChunk + tq;
            if (owner && t < t_end) lrow[t] = v[0];
        }
    }
    __syncthreads();
    // after an abandoned wait, copies of the last stages issued may still be in flight
    if (*flag && tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
}

// ---------------------------------------------------------------------------------
// QK with the in-quad rotation folded into the tables (one query head per CTA, kv heads of
// one query head each, codes of 2 or 3 bits).  With t = t_q + j, t_q the start of a token
// quad and j < 4, the pair term is Re(e^{i t_q theta_p} e^{i j theta_p} Z_p(code)); the
// table holds e^{i j theta_p} Z_p for each j, so a lane needs one phase per (quad, pair)
// instead of one per (token, pair).  A stage carries 256 tokens (64 quads) of the head; a
// consumer lane takes two quads and pairs i + 16 k; the reduction is the one of k_qk with
// the two quads in place of the two heads of a warp.
constexpr int kQQuads = 64;                  // token quads per stage
constexpr int kQTokens = 4 * kQQuads;        // tokens per stage
constexpr int kQWarps = 16;                  // consumer warps

// The table goes last, at the first shared-window address past `pre` that is a multiple of
// its j-slice (64 pairs x NT entries x 8 bytes): a lookup address is then one OR of the
// entry, the slice and the lane's pair, with no add of the table base.
struct QQPlan {
    int ring, stage, base, lev, bar, flag, pre, jslice, total;
};
__host__ __device__ inline QQPlan qq_plan(int bits) {
    QQPlan p;
    int o = 0;
    p.stage = kQQuads * 16 * bits * 4;                       // code blocks of 64 quads
    p.ring = o;  o += kStages * p.stage;
    p.base = o;  o += kStages * 64 * 8;                      // [stage][pair] (cos, sin) at stage start
    p.lev = o;   o += 16 * 4;                                // codebook levels
    p.bar = o;   o += 2 * kStages * 8;
    p.flag = o;  o += 16;
    p.pre = o;
    p.jslice = (1 << (2 * bits)) * 64 * 8;
    p.total = o + p.jslice + 4 * p.jslice;                   // alignment slack + [j][entry][pair]
    return p;
}

template <int BITS>
__global__ void __launch_bounds__(kQWarps * 32 + 32, 1)
    k_qk_quad(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ qr_all,
              const float2* __restrict__ thi, const float2* __restrict__ tlo, int Ls,
              int max_len, float* __restrict__ logits) {
    using F = Fmt<BITS>;
    constexpr int NC = kQWarps * 32;
    constexpr int P = 9;                         // entry bit of a table byte offset
    constexpr int JS = P + F::FW;                // j bit of a table byte offset
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << P;
    extern __shared__ __align__(128) uint8_t sm[];
    const QQPlan L = qq_plan(BITS);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t tpos = (sbase + L.pre + L.jslice - 1) & ~(uint32_t)(L.jslice - 1);
    uint8_t* tab = sm + (tpos - sbase);
    uint8_t* ring = sm + L.ring;
    float2* base = (float2*)(sm + L.base);
    float* lev = (float*)(sm + L.lev);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.x, b = blockIdx.y, hq = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, kvh = hq / (Hq / Hkv);
    int len = c.len[b];
    if (len > max_len) {
        if (tid == 0 && s == 0 && hq == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) return;
    const int nst = (t_end - t_begin + kQTokens - 1) / kQTokens;
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, kQWarps);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    // ---- tables: (X, Y) of Z_p(entry) turned by j theta_p.  Thread (p, r) of the first 512
    // holds pair p's constants and writes entries r, r + 8, ... for every j.
    if (tid < (1 << BITS)) lev[tid] = cb.levels[tid];
    __syncthreads();
    if (tid < 512) {
        const int p = tid & 63, r0 = tid >> 6;
        const float* kp = c.kparams + ((size_t)b * Hkv + kvh) * kD * 2;
        const float* qv = qr_all + ((size_t)b * Hq + hq) * kD;
        const float offa = kp[2 * p], halfa = kp[2 * p + 1];
        const float offb = kp[2 * (p + 64)], halfb = kp[2 * (p + 64) + 1];
        const float qa = qv[p], qb = qv[p + 64];
        const float A1 = qa * halfa, B1 = qb * halfb, C1 = qa * offa + qb * offb;
        const float A2 = qb * halfa, B2 = -qa * halfb, C2 = qb * offa - qa * offb;
        float2 rj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) rj[j] = tlo[j * 64 + p];
        unsigned long long* t64 = reinterpret_cast<unsigned long long*>(tab);
        for (int idx = r0; idx < F::NT; idx += 8) {
            const float La = lev[idx & ((1 << BITS) - 1)], Lb = lev[idx >> BITS];
            const float X = fmaf(B1, Lb, fmaf(A1, La, C1));
            const float Y = fmaf(B2, Lb, fmaf(A2, La, C2));
#pragma unroll
            for (int j = 0; j < 4; ++j)
                t64[(j * F::NT + idx) * 64 + p] =
                    pk(fmaf(rj[j].x, X, rj[j].y * Y), fmaf(rj[j].x, Y, -rj[j].y * X));
        }
    }
    __syncthreads();  // tables complete, barriers initialised

    if (tid >= NC) {
        // ================= streaming warp
        const int pl = tid - NC;
        const uint32_t* src = c.kcodes + ((size_t)b * Hkv + kvh) * nquads(cfg.T_max) * F::BW;
        int cc = 0;
        for (; cc < nst; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            const int tc = t_begin + cc * kQTokens;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float2 cs = trig_at(thi, tlo, tc, pl + 32 * u);
                base[slot * 64 + pl + 32 * u] = cs;
            }
            __syncwarp();
            __threadfence_block();
            if (pl == 0) {
                fence_proxy_async();
                const int q0 = tc >> 2, q1 = (min(tc + kQTokens, t_end) + 3) >> 2;
                const uint32_t bytes = (uint32_t)(q1 - q0) * F::BW * 4;
                mbar_arrive_expect_tx(full + slot, bytes);
                bulk_load(ring + (size_t)slot * L.stage, src + (size_t)q0 * F::BW, bytes,
                          full + slot);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;  // stages issued
    } else {
        // ================= consumer warps
        const int uperm = (i >> 1) & 1;     // partial u of the lane holds quad u ^ uperm
        const bool owner = !(i & 1);
        // quads 4 warp + hh and 4 warp + hh + 2 (hh the half-warp): the code words of the two
        // half-warps then sit 16 banks apart
        const int qbase = 4 * warp + ((tid >> 4) & 1);
        uint32_t lb[4], woff[2];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
            lb[sl] = tpos + ((uint32_t)(sl ^ x) << JS) + ((uint32_t)i << 3);
        // phase from the stage start to the quad, pair i + 16 k, as (c, s)
        float2 RQ[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int q = qbase + 2 * (u ^ uperm);
            woff[u] = (uint32_t)(q * F::BW + i * BITS) * 4;
#pragma unroll
            for (int k = 0; k < 4; ++k) RQ[u][k] = tlo[(4 * q) * 64 + i + 16 * k];
        }
        const int tq = 4 * (qbase + 2 * uperm) + x;
        float* lrow = logits + ((size_t)b * Hq + hq) * cfg.T_max;
        for (int st = 0; st < nst; ++st) {
            const int slot = st % kStages;
            if (!mbar_wait(full + slot, (uint32_t)(st / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[2][BITS];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[u][d] = *reinterpret_cast<const uint32_t*>(stage + woff[u] + 4 * d);
            // the stage start's (cos, sin) of pairs i + 16 k: one 8-byte read per pair
            float2 B[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) B[k] = base[slot * 64 + i + 16 * k];
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
            unsigned long long acc[4][2];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) acc[sl][0] = acc[sl][1] = 0ull;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // (c_b c_q - s_b s_q, c_b s_q + s_b c_q)
                    const float2 r = RQ[u][k];
                    const unsigned long long Pc = pk(fmaf(B[k].x, r.x, -B[k].y * r.y),
                                                     fmaf(B[k].x, r.y, B[k].y * r.x));
#pragma unroll
                    for (int sl = 0; sl < 4; ++sl) {
                        uint32_t fs;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, P>(w[u]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const uint32_t a = (fs & MASK) | lb[sl];
                        const unsigned long long T = k == 0 ? lds64<0>(a)
                                                   : k == 1 ? lds64<128>(a)
                                                   : k == 2 ? lds64<256>(a) : lds64<384>(a);
                        acc[sl][u] = fma2(Pc, T, acc[sl][u]);
                    }
                }
            }
            float v[8];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const f2 a = upk(acc[sl][u]);
                    v[2 * sl + u] = a.x + a.y;
                }
            int mk = 8;
#pragma unroll
            for (int half = 4; half >= 1; half >>= 1, mk >>= 1)
#pragma unroll
                for (int t = 0; t < half; ++t)
                    v[t] += __shfl_xor_sync(0xffffffffu, v[t + half], mk);
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
            const int t = t_begin + st * kQTokens + tq;
            if (owner && t < t_end) lrow[t] = v[0];
        }
    }
    __syncthreads();
    // after an abandoned wait, copies of the last stages issued may still be in flight
    if (*flag && tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
}

// ---------------------------------------------------------------------------------
// QK for kv heads that serve G query heads (grouped-query attention), codes of 2 or 3 bits:
// one CTA per (split, sequence, kv head).  The table holds, for each pair p and code pair, the
// dequantized key pair (off + half L[code], for channels p and p + 64) turned by j theta_p for
// the four token offsets j of a quad -- no query folded in -- so a kv head's codes are looked
// up once for all G query heads.  Per (token, pair): one lookup, the turn by the quad's phase
// (four scalar multiply-adds) and one packed multiply-add per query head.  Stages, ring,
// streaming warp and lane mapping are those of k_qk_quad.  The reduction over the 16 lane
// groups first folds the lane bits that pick a lane's token slots (slot s of lane group i
// holds token s ^ (i >> 2), so the partner's slot s ^ 2 or s ^ 1 holds the same token and no
// selection is needed), then the bits over the heads; lane i ends with token i >> 2 and head
// i & 3 (G = 4) or head (i >> 1) & 1 (G = 2).
template <int BITS, int G>
__global__ void __launch_bounds__(kQWarps * 32 + 32, 1)
    k_qk_grp(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ qr_all,
             const float2* __restrict__ thi, const float2* __restrict__ tlo, int Ls,
             int max_len, float* __restrict__ logits) {
    static_assert(G == 2 || G == 4, "two or four query heads per kv head");
    using F = Fmt<BITS>;
    constexpr int NC = kQWarps * 32;
    constexpr int P = 9;                         // entry bit of a table byte offset
    constexpr int JS = P + F::FW;                // j bit of a table byte offset
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << P;
    extern __shared__ __align__(128) uint8_t sm[];
    const QQPlan L = qq_plan(BITS);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t tpos = (sbase + L.pre + L.jslice - 1) & ~(uint32_t)(L.jslice - 1);
    uint8_t* tab = sm + (tpos - sbase);
    uint8_t* ring = sm + L.ring;
    float2* base = (float2*)(sm + L.base);
    float* lev = (float*)(sm + L.lev);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.x, b = blockIdx.y, kvh = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, hq0 = kvh * G;
    int len = c.len[b];
    if (len > max_len) {
        if (tid == 0 && s == 0 && kvh == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) return;
    const int nst = (t_end - t_begin + kQTokens - 1) / kQTokens;
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, kQWarps);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    // ---- tables: the dequantized key pair of each entry turned by j theta_p.  Thread (p, r)
    // of the first 512 writes entries r, r + 8, ... of pair p for every j.
    if (tid < (1 << BITS)) lev[tid] = cb.levels[tid];
    __syncthreads();
    if (tid < 512) {
        const int p = tid & 63, r0 = tid >> 6;
        const float* kp = c.kparams + ((size_t)b * Hkv + kvh) * kD * 2;
        const float offa = kp[2 * p], halfa = kp[2 * p + 1];
        const float offb = kp[2 * (p + 64)], halfb = kp[2 * (p + 64) + 1];
        float2 rj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) rj[j] = tlo[j * 64 + p];
        unsigned long long* t64 = reinterpret_cast<unsigned long long*>(tab);
        for (int idx = r0; idx < F::NT; idx += 8) {
            const float ka = fmaf(halfa, lev[idx & ((1 << BITS) - 1)], offa);
            const float kb = fmaf(halfb, lev[idx >> BITS], offb);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                t64[(j * F::NT + idx) * 64 + p] =
                    pk(fmaf(rj[j].x, ka, -rj[j].y * kb), fmaf(rj[j].y, ka, rj[j].x * kb));
        }
    }
    __syncthreads();  // tables complete, barriers initialised

    if (tid >= NC) {
        // ================= streaming warp (as in k_qk_quad)
        const int pl = tid - NC;
        const uint32_t* src = c.kcodes + ((size_t)b * Hkv + kvh) * nquads(cfg.T_max) * F::BW;
        int cc = 0;
        for (; cc < nst; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            const int tc = t_begin + cc * kQTokens;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float2 cs = trig_at(thi, tlo, tc, pl + 32 * u);
                base[slot * 64 + pl + 32 * u] = cs;
            }
            __syncwarp();
            __threadfence_block();
            if (pl == 0) {
                fence_proxy_async();
                const int q0 = tc >> 2, q1 = (min(tc + kQTokens, t_end) + 3) >> 2;
                const uint32_t bytes = (uint32_t)(q1 - q0) * F::BW * 4;
                mbar_arrive_expect_tx(full + slot, bytes);
                bulk_load(ring + (size_t)slot * L.stage, src + (size_t)q0 * F::BW, bytes,
                          full + slot);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;
    } else {
        // ================= consumer warps: half-warp hh takes quads 4 warp + hh and + 2
        const int qbase = 4 * warp + ((tid >> 4) & 1);
        uint32_t lb[4], woff[2];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
            lb[sl] = tpos + ((uint32_t)(sl ^ x) << JS) + ((uint32_t)i << 3);
#pragma unroll
        for (int u = 0; u < 2; ++u) woff[u] = (uint32_t)((qbase + 2 * u) * F::BW + i * BITS) * 4;
        unsigned long long Q[G][4];  // (q_p, q_{p+64}) of each query head, p = i + 16 k
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float* qv = qr_all + ((size_t)b * Hq + hq0 + h) * kD;
                Q[h][k] = pk(qv[i + 16 * k], qv[i + 16 * k + 64]);
            }
        const int hown = G == 4 ? (i & 3) : ((i >> 1) & 1);
        const bool owner = G == 4 ? true : !(i & 1);
        float* lrow = logits + ((size_t)b * Hq + hq0 + hown) * cfg.T_max;
        for (int st = 0; st < nst; ++st) {
            const int slot = st % kStages;
            if (!mbar_wait(full + slot, (uint32_t)(st / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[2][BITS];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[u][d] = *reinterpret_cast<const uint32_t*>(stage + woff[u] + 4 * d);
            float bc[4], bs[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 bq = base[slot * 64 + i + 16 * k];
                bc[k] = bq.x;
                bs[k] = bq.y;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
#pragma unroll 1
            for (int u = 0; u < 2; ++u) {
                unsigned long long acc[4][G];
#pragma unroll
                for (int sl = 0; sl < 4; ++sl)
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[sl][h] = 0ull;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // the quad's phase for pair i + 16 k: the stage start's turned by 4 q theta_p
                    // (read again each stage: an L1 hit, and no registers held across stages)
                    const float2 r = __ldg(tlo + (4 * (qbase + 2 * u)) * 64 + i + 16 * k);
                    const float pc = fmaf(bc[k], r.x, -bs[k] * r.y);
                    const float ps = fmaf(bc[k], r.y, bs[k] * r.x);
#pragma unroll
                    for (int sl = 0; sl < 4; ++sl) {
                        uint32_t fs;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, P>(w[u]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const uint32_t a = (fs & MASK) | lb[sl];
                        const unsigned long long T = k == 0 ? lds64<0>(a)
                                                   : k == 1 ? lds64<128>(a)
                                                   : k == 2 ? lds64<256>(a) : lds64<384>(a);
                        const f2 t = upk(T);
                        const unsigned long long K2 =
                            pk(fmaf(pc, t.x, -ps * t.y), fmaf(ps, t.x, pc * t.y));
#pragma unroll
                        for (int h = 0; h < G; ++h) acc[sl][h] = fma2(Q[h][k], K2, acc[sl][h]);
                    }
                }
                // token slots: fold lane bit 3 (slots 2, 3 go to the partner), then bit 2
                float v[2][G];
#pragma unroll
                for (int sl = 0; sl < 2; ++sl)
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const f2 a0 = upk(acc[sl][h]), a1 = upk(acc[sl + 2][h]);
                        v[sl][h] = (a0.x + a0.y) + __shfl_xor_sync(0xffffffffu, a1.x + a1.y, 8);
                    }
                float hv[G];
#pragma unroll
                for (int h = 0; h < G; ++h) hv[h] = v[0][h] + __shfl_xor_sync(0xffffffffu, v[1][h], 4);
                // heads: lane bit 1, then bit 0
                float r;
                if constexpr (G == 4) {
                    const bool b1 = (i >> 1) & 1, b0 = i & 1;
                    float h2[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const float keep = b1 ? hv[t + 2] : hv[t];
                        const float send = b1 ? hv[t] : hv[t + 2];
                        h2[t] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    }
                    const float keep = b0 ? h2[1] : h2[0];
                    const float send = b0 ? h2[0] : h2[1];
                    r = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                } else {
                    const bool b1 = (i >> 1) & 1;
                    const float keep = b1 ? hv[1] : hv[0];
                    const float send = b1 ? hv[0] : hv[1];
                    r = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    r += __shfl_xor_sync(0xffffffffu, r, 1);
                }
                const int t = t_begin + st * kQTokens + 4 * (qbase + 2 * u) + x;
                if (owner && t < t_end) lrow[t] = r;
            }
        }
    }
    __syncthreads();
    // after an abandoned wait, copies of the last stages issued may still be in flight
    if (*flag && tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
}

// ---------------------------------------------------------------------------------
// Outlier kernels.  A block takes up to kOutChunks 64-token chunks of one (sequence, kv head)
// list and stages their chunk pointers in shared memory; a warp walks a contiguous range of
// the block's entries, 32 kOutBatch at a time.  An entry holds only its token's offset within
// its chunk: a warp keeps the chunk of its current position and, per window, counts for each
// of its entries the chunk boundaries that fall inside the window.  A lane's kOutBatch entries
// are gathered together; lane l's u-th entry is entry E + 32u + l of the window, so slice u
// of a window is 32 consecutive entries in list order.
//
// Both kernels give the same bits on every run.  The key side gives each warp whole chunks
// (a token's entries never straddle two warps), sums each token's corrections in list order
// with a segmented scan across the lanes (a token's entries are contiguous: the list is
// sorted by token) and lets one lane add the sum to the logit: each logit receives exactly one
// addition, so the fire-and-forget atomic add gives the same bits as a read-modify-write
// without waiting on the read.  The value side adds each
// entry's term into 2^-40 fixed-point block sums with integer atomics (integer addition is
// associative, so their order does not matter), then adds each block sum once into its
// split's PV partial before the partials are summed in split order.
constexpr int kOutThreads = 256;  // threads per block of the outlier kernels
constexpr int kOutChunks = 128;   // chunks per staged window of chunk pointers
constexpr int kOutBatch = 4;      // entries a lane gathers at once
constexpr float kFixScale = 1099511627776.0f;      // 2^40
constexpr double kFixInv = 1.0 / 1099511627776.0;  // 2^-40

struct OutRange {
    uint32_t lo, hi;  // entries [lo, hi) of the staged chunks
    int m0, n;        // first chunk and number of chunks
};

// Stages min(cp[m0 + j], cnt), j <= n, n = chunks of [m0, m_end) below len (at most
// kOutChunks), in cps; ends with a block barrier.
__device__ __forceinline__ OutRange stage_chunks(const uint32_t* __restrict__ cp, uint32_t cnt,
                                                 int len, int m0, int m_end, uint32_t* cps) {
    OutRange r;
    r.m0 = m0;
    r.n = max(0, min(min((len + kChunk - 1) / kChunk, m_end) - m0, kOutChunks));
    if (r.n)
        for (int j = threadIdx.x; j <= r.n; j += blockDim.x) cps[j] = min(cp[m0 + j], cnt);
    __syncthreads();
    r.lo = r.n ? cps[0] : 0u;
    r.hi = r.n ? cps[r.n] : 0u;
    return r;
}

// A warp's walk over its entry range.  next() fills, for the lane's kOutBatch entries of the
// next window, w[u] (packed entry) and t[u] (token; -1 where the lane has no entry).
struct EntryWalker {
    static constexpr uint32_t W = 32 * kOutBatch;
    uint32_t E, Ee;
    int cur, n, m0;
    // chunk_aligned: warp w takes whole chunks [w*n/nw, (w+1)*n/nw); otherwise an even share
    // of the entries
    __device__ __forceinline__ EntryWalker(const OutRange& r, const uint32_t* cps,
                                           bool chunk_aligned) {
        const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
        n = r.n;
        m0 = r.m0;
        if (chunk_aligned) {
            const int ca = warp * n / nw, cb = (warp + 1) * n / nw;
            E = n ? cps[ca] : 0u;
            Ee = n ? cps[cb] : 0u;
            cur = ca;
        } else {
            const uint32_t span = ((r.hi - r.lo + nw - 1) / nw + 31) & ~31u;
            E = r.lo + (uint32_t)warp * span;
            Ee = min(r.hi, E + span);
            cur = 0;  // chunk of entry E: the largest j < n with cps[j] <= E
            if (E < Ee) {
#pragma unroll
                for (int step = kOutChunks / 2; step; step >>= 1)
                    if (cur + step < n && cps[cur + step] <= E) cur += step;
            }
        }
        // entries before E in the first chunk belong to an earlier warp; skip empty chunks
        while (cur + 1 < n && cps[cur + 1] <= E) ++cur;
    }
    __device__ __forceinline__ bool next(const uint32_t* cps, const uint32_t* __restrict__ ent,
                                         int (&t)[kOutBatch], uint32_t (&w)[kOutBatch]) {
        if (E >= Ee) return false;
        const uint32_t lane = threadIdx.x & 31;
        uint32_t e[kOutBatch];
        int j[kOutBatch];
#pragma unroll
        for (int u = 0; u < kOutBatch; ++u) {
            e[u] = E + lane + 32 * u;
            w[u] = e[u] < Ee ? ent[e[u]] : 0u;
            j[u] = cur;
        }
        // boundaries inside the window (warp-uniform loop)
        while (cur + 1 < n && cps[cur + 1] <= E + W - 1) {
            const uint32_t bd = cps[++cur];
#pragma unroll
            for (int u = 0; u < kOutBatch; ++u) j[u] += e[u] >= bd;
        }
#pragma unroll
        for (int u = 0; u < kOutBatch; ++u)
            t[u] = e[u] < Ee ? (m0 + j[u]) * kChunk + (int)((w[u] >> 7) & 63u) : -1;
        E += W;
        return true;
    }
};

// Inclusive scan of v over the lanes, restarted wherever the key t changes (keys contiguous).
__device__ __forceinline__ float seg_scan(float v, int t, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float vv = __shfl_up_sync(0xffffffffu, v, off);
        const int tt = __shfl_up_sync(0xffffffffu, t, off);
        if (lane >= off && tt == t) v += vv;
    }
    return v;
}

// Key outliers: logit(t, hq) += sum over the token's entries of (x - zhat) * r, r the
// component of the rotated query that meets the outlier's channel after the key is rotated to
// t.  G query heads per kv head (0: read from cfg).  The running sum of a token whose entries
// continue into the next slice is carried in carry[warp][head].
template <int G>
__global__ void __launch_bounds__(kOutThreads) k_key_outliers(
    kvq_cfg cfg, kvq_cache c, const float* __restrict__ qr, const float2* __restrict__ thi,
    const float2* __restrict__ tlo, const float* __restrict__ zk, int max_len,
    float* __restrict__ logits) {
    const int li = blockIdx.y, b = li / cfg.Hkv, h = li % cfg.Hkv;
    const int g = G ? G : cfg.Hq / cfg.Hkv;
    const int len = min(c.len[b], max_len);
    const uint32_t* cp = c.kchunk + (size_t)li * (nchunks(cfg.T_max) + 1);
    const uint32_t* ent = c.kout + (size_t)li * cfg.out_cap_k;
    __shared__ uint32_t cps[kOutChunks + 1];
    __shared__ float zks[kD];
    __shared__ float qs[(G ? G : kMaxG) * kD];
    __shared__ float carry[kOutThreads / 32][G ? G : kMaxG];
    for (int e = threadIdx.x; e < kD; e += blockDim.x) zks[e] = zk[(size_t)li * kD + e];
    for (int e = threadIdx.x; e < g * kD; e += blockDim.x)
        qs[e] = qr[((size_t)b * cfg.Hq + h * g) * kD + e];
    const int m0 = blockIdx.x * kOutChunks;
    const OutRange r = stage_chunks(cp, c.kcount[li], len, m0, m0 + kOutChunks, cps);
    float* lb0 = logits + ((size_t)b * cfg.Hq + h * g) * cfg.T_max;
    const size_t T_max = cfg.T_max;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    EntryWalker wk(r, cps, true);
    int ct = -1;  // token of the carried sums (warp-uniform)
    int t[kOutBatch];
    uint32_t w[kOutBatch];
    while (wk.next(cps, ent, t, w)) {
        float2 cs[kOutBatch];
#pragma unroll
        for (int u = 0; u < kOutBatch; ++u) {
            if ((unsigned)t[u] >= (unsigned)len) t[u] = -1;  // past the clipped length
            cs[u] = trig_at(thi, tlo, t[u] >= 0 ? t[u] : 0, (int)(w[u] & 63u));
        }
#pragma unroll
        for (int u = 0; u < kOutBatch; ++u) {
            const int tu = t[u];
            const int ch = (int)(w[u] & 127u), p = ch & 63;
            const float d = tu >= 0 ? h2f((uint16_t)(w[u] >> 16)) - zks[ch] : 0.0f;
            // rotate-half: channel c < 64 meets (cos, sin) . (q_p, q_p+64), c >= 64 the other
            const float sa = ch < 64 ? cs[u].x : -cs[u].y, sb = ch < 64 ? cs[u].y : cs[u].x;
            const int t0 = __shfl_sync(0xffffffffu, tu, 0);
            const int tn = __shfl_down_sync(0xffffffffu, tu, 1);
            const bool tail = tu >= 0 && lane < 31 && tn != tu;
            const bool flush = ct >= 0 && t0 != ct;  // the carried token ended with the last slice
            if constexpr (G > 1) {
                // all heads in one segmented scan: the token ids move once per step
                float v[G];
#pragma unroll
                for (int a = 0; a < G; ++a) {
                    v[a] = d * fmaf(sa, qs[a * kD + p], sb * qs[a * kD + p + 64]);
                    if (ct >= 0 && lane == 0) {
                        const float cv = carry[warp][a];
                        if (flush) atomicAdd(&lb0[a * T_max + ct], cv);
                        else v[a] += cv;
                    }
                }
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int tt = __shfl_up_sync(0xffffffffu, tu, off);
                    const bool same = lane >= off && tt == tu;
#pragma unroll
                    for (int a = 0; a < G; ++a) {
                        const float vv = __shfl_up_sync(0xffffffffu, v[a], off);
                        if (same) v[a] += vv;
                    }
                }
#pragma unroll
                for (int a = 0; a < G; ++a) {
                    if (tail) atomicAdd(&lb0[a * T_max + tu], v[a]);
                    if (lane == 31) carry[warp][a] = v[a];
                }
            } else {
            for (int a = 0; a < g; ++a) {
                float v = d * fmaf(sa, qs[a * kD + p], sb * qs[a * kD + p + 64]);
                if (ct >= 0 && lane == 0) {
                    const float cv = carry[warp][a];
                    if (flush) atomicAdd(&lb0[a * T_max + ct], cv);
                    else v += cv;
                }
                v = seg_scan(v, tu, lane);
                if (tail) atomicAdd(&lb0[a * T_max + tu], v);
                if (lane == 31) carry[warp][a] = v;
            }
            }
            __syncwarp();
            ct = __shfl_sync(0xffffffffu, tu, 31);
        }
    }
    if (ct >= 0 && lane == 0)
        for (int a = 0; a < g; ++a) atomicAdd(&lb0[a * T_max + ct], carry[warp][a]);
}

// ---------------------------------------------------------------------------------
// Softmax statistics of each split from the (corrected) logits: stats = (m_s, l_s), one pass
// over the split with a running (max, sum) per thread, merged across the block.
constexpr int kStatThreads = 256;  // threads of the statistics kernel
constexpr int kStatVec = 8;        // float4 loads per thread and tile
__device__ __forceinline__ void online_merge(float& m, float& l, float m2, float l2) {
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;
    l = (m > -INFINITY ? l * __expf(m - mn) : 0.0f) + (m2 > -INFINITY ? l2 * __expf(m2 - mn) : 0.0f);
    m = mn;
}

__global__ void __launch_bounds__(kStatThreads) k_logit_stats(kvq_cfg cfg, const int32_t* __restrict__ lens,
                                                     const float* __restrict__ logits, int Ls,
                                                     int S, int max_len, float2* __restrict__ stats) {
    const int s = blockIdx.x, bh = blockIdx.y, b = bh / cfg.Hq;
    const int len = min(lens[b], max_len);
    const int t0 = s * Ls, t1 = max(t0, min(len, t0 + Ls));  // empty split: t1 == t0
    const float* row = logits + (size_t)bh * cfg.T_max;
    // t0 is a multiple of 64; float4 loads when the row's address allows
    const bool vec = ((reinterpret_cast<uintptr_t>(row + t0) & 15u) == 0);
    float m = -INFINITY, l = 0.0f;
    // tiles of kStatThreads x kStatVec float4s: all loads of a tile in flight at once, then
    // its max and its sum of exponentials, merged into the running pair
    for (int tb = t0; tb < t1; tb += 4 * kStatThreads * kStatVec) {
        float x[kStatVec][4];
#pragma unroll
        for (int u = 0; u < kStatVec; ++u) {
            const int tt = tb + 4 * (threadIdx.x + kStatThreads * u);
            if (vec && tt + 3 < t1) {
                const float4 v = *reinterpret_cast<const float4*>(row + tt);
                x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[u][e] = tt + e < t1 ? row[tt + e] : -INFINITY;
            }
        }
        float mt = -INFINITY;
#pragma unroll
        for (int u = 0; u < kStatVec; ++u)
#pragma unroll
            for (int e = 0; e < 4; ++e) mt = fmaxf(mt, x[u][e]);
        if (mt > -INFINITY) {
            float lt = 0.0f;
#pragma unroll
            for (int u = 0; u < kStatVec; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) lt += __expf(x[u][e] - mt);
            online_merge(m, l, mt, lt);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        online_merge(m, l, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, l, o));
    __shared__ float2 red[kStatThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = make_float2(m, l);
    __syncthreads();
    if (threadIdx.x == 0) {
        float M = -INFINITY, Lsum = 0.0f;
        for (int w = 0; w < kStatThreads / 32; ++w) online_merge(M, Lsum, red[w].x, red[w].y);
        stats[(size_t)bh * S + s] = make_float2(M, Lsum);
    }
}

// ---------------------------------------------------------------------------------
// PV.  out_h = sum_t p_t (off_t + half_t L[code]) = sum_t p_t off_t + sum_t (p_t half_t) L[code];
// per pair (c, c + 64) and token one (La, Lb) lookup (a 16-copy table, copy = lane) and one
// f32x2 FMA with (w, w), w = p half.  A consumer warp takes two token quads and HW heads;
// lane i computes the weight of (token i >> 2 of its quad, head out_head(i) of the warp).  The
// last warp streams the chunks.
template <int BITS, int HPC, bool SHARE>
__global__ void __launch_bounds__(pv_warps(HPC) * 32 + 32, 1)
    k_pv(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ logits,
         const float2* __restrict__ ml, int Ls, int S, int max_len, int kvb,
         float* __restrict__ part) {
    using F = Fmt<BITS>;
    constexpr int CW = pv_warps(HPC), NC = CW * 32;
    constexpr int HW = heads_per_warp<HPC, CW>();
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << 7;
    constexpr int NW = SHARE ? 1 : HW;
    extern __shared__ __align__(128) uint8_t sm[];
    const PVPlan L = pv_plan(BITS, HPC, kvb);
    uint8_t* tab = sm + L.tab;
    uint8_t* ring = sm + L.ring;
    unsigned long long* wsm = (unsigned long long*)(sm + L.wsm);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x, nthr = blockDim.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5;
    const int qd = 2 * (warp & 7) + ((tid >> 4) & 1);  // token quad of the chunk
    const int hg = (warp >> 3) * HW;                     // first CTA head of the warp
    const int s = blockIdx.x, b = blockIdx.y, hq0 = blockIdx.z * HPC;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, g = Hq / Hkv;
    const int len = min(c.len[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) {
        for (int e = tid; e < HPC * kD; e += nthr)
            part[(((size_t)b * Hq + hq0 + (e >> 7)) * S + s) * kD + (e & 127)] = 0.0f;
        return;
    }
    const int nch = (t_end - t_begin + kChunk - 1) / kChunk;
    const int kv_first = min(hq0 / g, Hkv - kvb);
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, CW);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    const int nb = (1 << BITS) - 1;
    for (int e = tid; e < F::NT * 16; e += nthr) {
        const int idx = e >> 4;
        reinterpret_cast<unsigned long long*>(tab)[e] =
            pk(cb.levels[idx & nb], cb.levels[idx >> BITS]);
    }
    __syncthreads();  // tables complete, barriers initialised

    unsigned long long O[4][HW];
    float po = 0.0f;
    const int hs = hg + out_head<HW>(i);  // CTA head of this lane's weight
    const bool owner = out_owner<HW>(i);
    if (tid >= NC) {
        // ================= streaming warp
        const int pl = tid - NC;
        Streamer sr;
        sr.ring = ring;
        sr.full = full;
        sr.pitch = L.pitch;
        sr.stage = L.stage;
        sr.kvb = kvb;
        sr.t_begin = t_begin;
        sr.t_end = t_end;
        sr.src0 = c.vcodes + ((size_t)b * Hkv + kv_first) * nquads(cfg.T_max) * F::BW;
        sr.head_stride = (size_t)nquads(cfg.T_max) * F::BW;
        sr.quad_bytes = (uint32_t)F::BW * 4;
        int cc = 0;
        for (; cc < nch; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            if (pl == 0) {
                fence_proxy_async();
                sr.issue(cc);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;  // chunks issued
    } else {
        // ================= consumer warps
        const int tq = 4 * qd + x;
        const float2 mL = ml[(size_t)b * Hq + hq0 + hs];
        const float invL = mL.y > 0.0f ? 1.0f / mL.y : 0.0f;
        const float* lrow = logits + ((size_t)b * Hq + hq0 + hs) * cfg.T_max;
        const float2* vpar = reinterpret_cast<const float2*>(c.vparams) + (size_t)b * cfg.T_max;
        float lg = -INFINITY;
        float2 vp = make_float2(0.0f, 0.0f);
        auto fetch = [&](int cc) {
            const int t = t_begin + cc * kChunk + tq;
            const bool ok = owner && t < t_end;
            lg = ok ? lrow[t] : -INFINITY;
            vp = ok ? vpar[t] : make_float2(0.0f, 0.0f);
        };
        fetch(0);
        uint32_t woff[NW];
#pragma unroll
        for (int h = 0; h < NW; ++h) {
            const int kvs = SHARE ? 0 : (hq0 + hg + h) / g - kv_first;
            woff[h] = (uint32_t)(kvs * L.pitch + qd * F::BW * 4 + i * BITS * 4);
        }
        const uint32_t lanebits = (uint32_t)i << 3;
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int h = 0; h < HW; ++h) O[k][h] = 0ull;
        for (int ch = 0; ch < nch; ++ch) {
            const int slot = ch % kStages;
            {
                const float p = (lg > -INFINITY) ? expf(lg - mL.x) * invL : 0.0f;
                const float wv = p * vp.y;
                po = fmaf(p, vp.x, po);
                if (owner) wsm[(qd * 4 + x) * HPC + hs] = pk(wv, wv);
            }
            __syncwarp();
            if (ch + 1 < nch) fetch(ch + 1);
            if (!mbar_wait(full + slot, (uint32_t)(ch / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[NW][BITS];
#pragma unroll
            for (int h = 0; h < NW; ++h)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[h][d] = *reinterpret_cast<const uint32_t*>(stage + woff[h] + 4 * d);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
                unsigned long long ww[HW];
#pragma unroll
                for (int h = 0; h < HW; ++h) ww[h] = wsm[(qd * 4 + (sl ^ x)) * HPC + hg + h];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
#pragma unroll
                    for (int h = 0; h < NW; ++h) {
                        uint32_t fs = 0;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, 7>(w[h]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const unsigned long long LL = tld(tab, (fs & MASK) | lanebits);
                        if (SHARE) {
#pragma unroll
                            for (int hh = 0; hh < HW; ++hh) O[k][hh] = fma2(ww[hh], LL, O[k][hh]);
                        } else {
                            O[k][h] = fma2(ww[h], LL, O[k][h]);
                        }
                    }
                }
            }
            __syncwarp();  // wsm is rewritten for the next chunk
        }
    }
    __syncthreads();
    if (*flag) {
        if (tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
        return;
    }
    // partial sums of the 16 quads -> the split's output (the ring is idle now)
    float* red = (float*)ring;
    if (tid < NC) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int h = 0; h < HW; ++h) {
                const f2 o = upk(O[k][h]);
                red[(qd * HPC + hg + h) * kD + i + 16 * k] = o.x;
                red[(qd * HPC + hg + h) * kD + i + 16 * k + 64] = o.y;
            }
    }
    // sum_t p_t off_t per head: the owners' shares, reduced through the ring's tail region
    float* pored = red + kQuads * HPC * kD;
    if (tid < NC) pored[tid] = owner ? po : 0.0f;
    __syncthreads();
    for (int e = tid; e < HPC * kD; e += nthr) {
        const int h = e >> 7, ch2 = e & 127;
        float a = 0.0f;
        for (int qq = 0; qq < kQuads; ++qq) a += red[(qq * HPC + h) * kD + ch2];
        float o = 0.0f;
        for (int t2 = 0; t2 < NC; ++t2)
            if (((t2 >> 8) * HW + out_head<HW>(t2 & 15)) == h) o += pored[t2];
        part[(((size_t)b * Hq + hq0 + h) * S + s) * kD + ch2] = a + o;
    }
}

// ---------------------------------------------------------------------------------
// PV when every kv head serves one query head: one query head per CTA, 512-token stages of its
// value codes; half-warp hh of warp w takes the quads 8 w + 2 u + hh (u < 4), so a lane makes
// 64 (pair, token) steps per stage against one weight computation, one barrier wait and one
// stage's bookkeeping.  Lane l of warp w computes the weight of token 32 w + l of the stage;
// the warp's 32 weights sit in its own slice of shared memory.  The code words of the two
// half-warps are 16 banks apart.  Each (La, Lb) lookup reads the two levels' 16-bit patterns
// (the levels are (u << 16) | u binary32 values) from a table with one copy per lane, and two
// byte permutes rebuild the exact binary32 pair: half the table bytes of a float pair.
constexpr int kPQuads = 128;                 // token quads per stage
constexpr int kPTokens = 4 * kPQuads;        // tokens per stage

// The (La, Lb) table goes last, at a shared-window address that is a multiple of its size, so
// a lookup address is one OR of the entry and the lane's copy.
struct PQPlan {
    int ring, stage, wsm, bar, flag, pre, tsize, total;
};
__host__ __device__ inline PQPlan pq_plan(int bits, int g = 1) {
    PQPlan p;
    int o = 0;
    p.stage = kPQuads * 16 * bits * 4;
    p.ring = o;  o += kStages * p.stage;                     // reused by the final reduction
    p.wsm = o;   o += kQWarps * g * 32 * 8;                  // [warp][head][token] (w, w)
    p.bar = o;   o += 2 * kStages * 8;
    p.flag = o;  o += 16;
    p.pre = o;
    p.tsize = (1 << (2 * bits)) * 32 * 4;                    // [entry][32 lane copies] 16-bit (La, Lb)
    p.total = o + 2 * p.tsize;                               // alignment slack + table
    return p;
}

template <int BITS>
__global__ void __launch_bounds__(kQWarps * 32 + 32, 1)
    k_pv_quad(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ logits,
              const float2* __restrict__ ml, int Ls, int S, int max_len,
              float* __restrict__ part) {
    using F = Fmt<BITS>;
    constexpr int NC = kQWarps * 32;
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << 7;
    extern __shared__ __align__(128) uint8_t sm[];
    const PQPlan L = pq_plan(BITS);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t tpos = (sbase + L.pre + L.tsize - 1) & ~(uint32_t)(L.tsize - 1);
    uint8_t* tab = sm + (tpos - sbase);
    uint8_t* ring = sm + L.ring;
    unsigned long long* wsm = (unsigned long long*)(sm + L.wsm);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x, nthr = blockDim.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5, hh = (tid >> 4) & 1;
    const int s = blockIdx.x, b = blockIdx.y, hq = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, kvh = hq / (Hq / Hkv);
    float* po_out = part + (((size_t)b * Hq + hq) * S + s) * kD;
    const int len = min(c.len[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) {
        for (int e = tid; e < kD; e += nthr) po_out[e] = 0.0f;
        return;
    }
    const int nst = (t_end - t_begin + kPTokens - 1) / kPTokens;
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, kQWarps);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    const int nb = (1 << BITS) - 1;
    // (La, Lb) as the 16-bit patterns u of the (u << 16) | u levels, one copy per lane
    for (int e = tid; e < F::NT * 32; e += nthr) {
        const int idx = e >> 5;
        const uint32_t ua = __float_as_uint(cb.levels[idx & nb]);
        const uint32_t ub = __float_as_uint(cb.levels[idx >> BITS]);
        reinterpret_cast<uint32_t*>(tab)[e] = (ua & 0xFFFFu) | (ub << 16);
    }
    if (tid <= nb) {
        const uint32_t u = __float_as_uint(cb.levels[tid]);
        if ((u >> 16) != (u & 0xFFFFu)) set_status(c.status, KVQ_STATUS_CODEBOOK);
    }
    __syncthreads();  // tables complete, barriers initialised

    unsigned long long O[4] = {0ull, 0ull, 0ull, 0ull};
    float po = 0.0f;
    if (tid >= NC) {
        // ================= streaming warp
        const int pl = tid - NC;
        const uint32_t* src = c.vcodes + ((size_t)b * Hkv + kvh) * nquads(cfg.T_max) * F::BW;
        int cc = 0;
        for (; cc < nst; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            if (pl == 0) {
                fence_proxy_async();
                const int tc = t_begin + cc * kPTokens;
                const int q0 = tc >> 2, q1 = (min(tc + kPTokens, t_end) + 3) >> 2;
                const uint32_t bytes = (uint32_t)(q1 - q0) * F::BW * 4;
                mbar_arrive_expect_tx(full + slot, bytes);
                bulk_load(ring + (size_t)slot * L.stage, src + (size_t)q0 * F::BW, bytes,
                          full + slot);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;  // stages issued
    } else {
        // ================= consumer warps
        const float2 mL = ml[(size_t)b * Hq + hq];
        const float invL = mL.y > 0.0f ? 1.0f / mL.y : 0.0f;
        const float* lrow = logits + ((size_t)b * Hq + hq) * cfg.T_max;
        const float2* vpar = reinterpret_cast<const float2*>(c.vparams) + (size_t)b * cfg.T_max;
        float lg = -INFINITY;
        float2 vp = make_float2(0.0f, 0.0f);
        auto fetch = [&](int st) {
            const int t = t_begin + st * kPTokens + 32 * warp + lane;
            const bool ok = t < t_end;
            lg = ok ? lrow[t] : -INFINITY;
            vp = ok ? vpar[t] : make_float2(0.0f, 0.0f);
        };
        fetch(0);
        uint32_t woff[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            woff[u] = (uint32_t)((8 * warp + 2 * u + hh) * F::BW + i * BITS) * 4;
        const uint32_t lanebits = tpos | ((uint32_t)lane << 2);
        unsigned long long* wsw = wsm + 32 * warp;
        for (int st = 0; st < nst; ++st) {
            const int slot = st % kStages;
            {
                const float p = (lg > -INFINITY) ? __expf(lg - mL.x) * invL : 0.0f;
                const float wv = p * vp.y;
                po = fmaf(p, vp.x, po);
                wsw[lane] = pk(wv, wv);
            }
            __syncwarp();
            if (st + 1 < nst) fetch(st + 1);
            if (!mbar_wait(full + slot, (uint32_t)(st / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[4][BITS];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[u][d] = *reinterpret_cast<const uint32_t*>(stage + woff[u] + 4 * d);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    // token 4 (2 u + hh) + (sl ^ x) of the warp's 32
                    const unsigned long long ww = wsw[8 * u + 4 * hh + (sl ^ x)];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t fs = 0;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, 7>(w[u]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const uint32_t lv = lds32((fs & MASK) | lanebits);
                        const unsigned long long LL =
                            pk(__uint_as_float(__byte_perm(lv, 0u, 0x1010)),
                               __uint_as_float(__byte_perm(lv, 0u, 0x3232)));
                        O[k] = fma2(ww, LL, O[k]);
                    }
                }
            }
            __syncwarp();  // wsw is rewritten for the next stage
        }
    }
    __syncthreads();
    if (*flag) {
        if (tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
        return;
    }
    // partial sums of the 32 half-warps -> the split's output (the ring is idle now)
    float* red = (float*)ring;
    float* pored = red + 2 * kQWarps * kD;
    if (tid < NC) {
        const int row = 2 * warp + hh;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const f2 o = upk(O[k]);
            red[row * kD + i + 16 * k] = o.x;
            red[row * kD + i + 16 * k + 64] = o.y;
        }
        po = warp_sum(po);  // sum_t p_t off_t over the warp's tokens
        if (lane == 0) pored[warp] = po;
    }
    __syncthreads();
    for (int e = tid; e < kD; e += nthr) {
        float a = 0.0f;
        for (int r = 0; r < 2 * kQWarps; ++r) a += red[r * kD + e];
        float o = 0.0f;
        for (int w2 = 0; w2 < kQWarps; ++w2) o += pored[w2];
        po_out[e] = a + o;
    }
}

// ---------------------------------------------------------------------------------
// PV for kv heads that serve G query heads (grouped-query attention), codes of 2 or 3 bits:
// one CTA per (split, sequence, kv head).  Stages, ring, streaming warp, lane mapping and the
// 16-bit (La, Lb) table are those of k_pv_quad; each (La, Lb) lookup serves all G heads, one
// packed multiply-add per head with that head's weight p half of the token.  The per-warp
// weights sit in shared memory as [head][token] (w, w); the split's outputs are reduced head
// by head through the idle ring at the end.
template <int BITS, int G>
__global__ void __launch_bounds__(kQWarps * 32 + 32, 1)
    k_pv_grp(kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ logits,
             const float2* __restrict__ ml, int Ls, int S, int max_len,
             float* __restrict__ part) {
    static_assert(G == 2 || G == 4, "two or four query heads per kv head");
    using F = Fmt<BITS>;
    constexpr int NC = kQWarps * 32;
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << 7;
    extern __shared__ __align__(128) uint8_t sm[];
    const PQPlan L = pq_plan(BITS, G);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t tpos = (sbase + L.pre + L.tsize - 1) & ~(uint32_t)(L.tsize - 1);
    uint8_t* tab = sm + (tpos - sbase);
    uint8_t* ring = sm + L.ring;
    unsigned long long* wsm = (unsigned long long*)(sm + L.wsm);
    uint64_t* full = (uint64_t*)(sm + L.bar);
    uint64_t* empty = full + kStages;
    int* flag = (int*)(sm + L.flag);

    const int tid = threadIdx.x, nthr = blockDim.x;
    const int i = tid & 15, x = i >> 2, lane = tid & 31, warp = tid >> 5, hh = (tid >> 4) & 1;
    const int s = blockIdx.x, b = blockIdx.y, kvh = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, hq0 = kvh * G;
    const int len = min(c.len[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end) {
        for (int e = tid; e < G * kD; e += nthr)
            part[(((size_t)b * Hq + hq0 + e / kD) * S + s) * kD + e % kD] = 0.0f;
        return;
    }
    const int nst = (t_end - t_begin + kPTokens - 1) / kPTokens;
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(full + k, 1);
            mbar_init(empty + k, kQWarps);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    const int nb = (1 << BITS) - 1;
    for (int e = tid; e < F::NT * 32; e += nthr) {
        const int idx = e >> 5;
        const uint32_t ua = __float_as_uint(cb.levels[idx & nb]);
        const uint32_t ub = __float_as_uint(cb.levels[idx >> BITS]);
        reinterpret_cast<uint32_t*>(tab)[e] = (ua & 0xFFFFu) | (ub << 16);
    }
    if (tid <= nb) {
        const uint32_t u = __float_as_uint(cb.levels[tid]);
        if ((u >> 16) != (u & 0xFFFFu)) set_status(c.status, KVQ_STATUS_CODEBOOK);
    }
    __syncthreads();  // tables complete, barriers initialised

    unsigned long long O[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int k = 0; k < 4; ++k) O[h][k] = 0ull;
    float po[G];
#pragma unroll
    for (int h = 0; h < G; ++h) po[h] = 0.0f;
    if (tid >= NC) {
        // ================= streaming warp
        const int pl = tid - NC;
        const uint32_t* src = c.vcodes + ((size_t)b * Hkv + kvh) * nquads(cfg.T_max) * F::BW;
        int cc = 0;
        for (; cc < nst; ++cc) {
            const int slot = cc % kStages;
            if (cc >= kStages && !mbar_wait(empty + slot, (uint32_t)(cc / kStages - 1) & 1u)) {
                if (pl == 0) {
                    atomicOr(flag, 1);
                    set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (*flag) break;
            if (pl == 0) {
                fence_proxy_async();
                const int tc = t_begin + cc * kPTokens;
                const int q0 = tc >> 2, q1 = (min(tc + kPTokens, t_end) + 3) >> 2;
                const uint32_t bytes = (uint32_t)(q1 - q0) * F::BW * 4;
                mbar_arrive_expect_tx(full + slot, bytes);
                bulk_load(ring + (size_t)slot * L.stage, src + (size_t)q0 * F::BW, bytes,
                          full + slot);
            }
            __syncwarp();
        }
        if (pl == 0) flag[1] = cc;  // stages issued
    } else {
        // ================= consumer warps
        float mM[G], invL[G], lg[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float2 mL = ml[(size_t)b * Hq + hq0 + h];
            mM[h] = mL.x;
            invL[h] = mL.y > 0.0f ? 1.0f / mL.y : 0.0f;
        }
        const float* lrow0 = logits + ((size_t)b * Hq + hq0) * cfg.T_max;
        const float2* vpar = reinterpret_cast<const float2*>(c.vparams) + (size_t)b * cfg.T_max;
        float2 vp = make_float2(0.0f, 0.0f);
        auto fetch = [&](int st) {
            const int t = t_begin + st * kPTokens + 32 * warp + lane;
            const bool ok = t < t_end;
#pragma unroll
            for (int h = 0; h < G; ++h) lg[h] = ok ? lrow0[(size_t)h * cfg.T_max + t] : -INFINITY;
            vp = ok ? vpar[t] : make_float2(0.0f, 0.0f);
        };
        fetch(0);
        uint32_t woff[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            woff[u] = (uint32_t)((8 * warp + 2 * u + hh) * F::BW + i * BITS) * 4;
        const uint32_t lanebits = tpos | ((uint32_t)lane << 2);
        unsigned long long* wsw = wsm + 32 * G * warp;  // [head][32 tokens]
        for (int st = 0; st < nst; ++st) {
            const int slot = st % kStages;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = (lg[h] > -INFINITY) ? __expf(lg[h] - mM[h]) * invL[h] : 0.0f;
                const float wv = p * vp.y;
                po[h] = fmaf(p, vp.x, po[h]);
                wsw[32 * h + lane] = pk(wv, wv);
            }
            __syncwarp();
            if (st + 1 < nst) fetch(st + 1);
            if (!mbar_wait(full + slot, (uint32_t)(st / kStages) & 1u)) {
                atomicOr(flag, 1);
                set_status(c.status, KVQ_STATUS_WAIT_TIMEOUT);
            }
            if (*flag) break;
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[4][BITS];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[u][d] = *reinterpret_cast<const uint32_t*>(stage + woff[u] + 4 * d);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    // token 4 (2 u + hh) + (sl ^ x) of the warp's 32
                    unsigned long long ww[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) ww[h] = wsw[32 * h + 8 * u + 4 * hh + (sl ^ x)];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t fs = 0;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, 7>(w[u]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const uint32_t lv = lds32((fs & MASK) | lanebits);
                        const unsigned long long LL =
                            pk(__uint_as_float(__byte_perm(lv, 0u, 0x1010)),
                               __uint_as_float(__byte_perm(lv, 0u, 0x3232)));
#pragma unroll
                        for (int h = 0; h < G; ++h) O[h][k] = fma2(ww[h], LL, O[h][k]);
                    }
                }
            }
            __syncwarp();  // wsw is rewritten for the next stage
        }
    }
    __syncthreads();
    if (*flag) {
        if (tid == 0) drain_chunks(full, max(0, flag[1] - kStages), flag[1], kStages);
        return;
    }
    // per head: the two half-warps of a warp hold the same pairs; fold them, then sum the 16
    // warps' rows through the idle ring
    float* red = (float*)ring;
    float* pored = red + kQWarps * kD;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        if (tid < NC) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f2 o = upk(O[h][k]);
                o.x += __shfl_xor_sync(0xffffffffu, o.x, 16);
                o.y += __shfl_xor_sync(0xffffffffu, o.y, 16);
                if (!hh) {
                    red[warp * kD + i + 16 * k] = o.x;
                    red[warp * kD + i + 16 * k + 64] = o.y;
                }
            }
            const float pw = warp_sum(po[h]);  // sum_t p_t off_t over the warp's tokens
            if (lane == 0) pored[warp] = pw;
        }
        __syncthreads();
        for (int e = tid; e < kD; e += nthr) {
            float a = 0.0f;
            for (int r = 0; r < kQWarps; ++r) a += red[r * kD + e];
            float o = 0.0f;
            for (int w2 = 0; w2 < kQWarps; ++w2) o += pored[w2];
            part[(((size_t)b * Hq + hq0 + h) * S + s) * kD + e] = a + o;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------
// Value outliers: part(s, hq, c) += sum over the split's entries of p(t, hq) (x - zhat_t),
// p = exp(l - M) / L from the merged statistics, zhat_t = off_t + half_t L[encode(normalize(0))].
// One block per (split, sequence, kv head) walks the split's chunks kOutChunks at a time; each
// term goes into a 2^-40 fixed-point sum per (head, channel) with an integer atomic, and one
// thread adds each sum to the split's partial.  |p (x - zhat)| < 2^18 and the p of a sequence
// sum to 1, so a block's sums stay below 2^58.  G as for the key outliers.
template <int BITS, int G>
__global__ void __launch_bounds__(kOutThreads) k_value_outliers(
    kvq_cfg cfg, kvq_cache c, kvq_codebook cb, const float* __restrict__ logits,
    const float2* __restrict__ ml, int Ls, int S, int max_len, float* __restrict__ part) {
    constexpr int NB = (1 << BITS) - 1;
    // a cluster of blocks along x shares one split: block `rank` walks its share of the
    // split's chunks, and rank 0 adds the blocks' integer sums (read through distributed
    // shared memory) once into the split's partial
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const int nsub = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
    const int s = blockIdx.x / nsub, li = blockIdx.y, b = li / cfg.Hkv, h = li % cfg.Hkv;
    const int g = G ? G : cfg.Hq / cfg.Hkv;
    const int len = min(c.len[b], max_len);
    const uint32_t* cp = c.vchunk + (size_t)li * (nchunks(cfg.T_max) + 1);
    const uint32_t* ent = c.vout + (size_t)li * cfg.out_cap_v;
    __shared__ unsigned long long acc[(G ? G : kMaxG) * kD];
    __shared__ float bnd[16], lev[16];
    __shared__ float2 mls[kMaxG];  // (M, 1 / L), 1 / L = 0 for an empty row
    __shared__ uint32_t cps[kOutChunks + 1];
    if (threadIdx.x < NB) bnd[threadIdx.x] = cb.bounds[threadIdx.x];
    if (threadIdx.x <= NB) lev[threadIdx.x] = cb.levels[threadIdx.x];
    if (threadIdx.x < g) {
        const float2 v = ml[(size_t)b * cfg.Hq + h * g + threadIdx.x];
        mls[threadIdx.x] = make_float2(v.x, v.y > 0.0f ? 1.0f / v.y : 0.0f);
    }
    for (int e = threadIdx.x; e < g * kD; e += blockDim.x) acc[e] = 0ull;
    const float2* vpar = reinterpret_cast<const float2*>(c.vparams) + (size_t)b * cfg.T_max;
    const float* lrow = logits + ((size_t)b * cfg.Hq + h * g) * cfg.T_max;
    const size_t T_max = cfg.T_max;
    const int mb0 = s * (Ls / kChunk), me0 = min(mb0 + Ls / kChunk, (len + kChunk - 1) / kChunk);
    const int span = max(0, (me0 - mb0 + nsub - 1) / nsub);
    const int mb = mb0 + rank * span, me = min(me0, mb + span);
    const uint32_t cnt = c.vcount[li];
    for (int m0 = mb; m0 < me; m0 += kOutChunks) {
        __syncthreads();  // the previous window's cps are no longer read
        const OutRange r = stage_chunks(cp, cnt, len, m0, me, cps);  // barrier covers the above
        if (r.lo >= r.hi) continue;
        float bd[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) bd[j] = bnd[j];
        EntryWalker wk(r, cps, false);
        int t[kOutBatch];
        uint32_t w[kOutBatch];
        while (wk.next(cps, ent, t, w)) {
            bool ok[kOutBatch];
            float2 vp[kOutBatch];
            constexpr int GP = G ? G : 1;  // heads whose logits are gathered up front
            float l0[kOutBatch][GP];
#pragma unroll
            for (int u = 0; u < kOutBatch; ++u) {
                ok[u] = (unsigned)t[u] < (unsigned)len;
                const int tt = ok[u] ? t[u] : 0;
                vp[u] = vpar[tt];
#pragma unroll
                for (int a = 0; a < GP; ++a) l0[u][a] = lrow[a * T_max + tt];
            }
#pragma unroll
            for (int u = 0; u < kOutBatch; ++u) {
                // the dense value stored at the outlier: the code of 0 in the token's normalization
                const float xn = normalize(0.0f, vp[u].x, vp[u].y);
                int code = 0;
#pragma unroll
                for (int j = 0; j < NB; ++j) code += xn > bd[j];
                const float d = h2f((uint16_t)(w[u] >> 16)) - fmaf(vp[u].y, lev[code], vp[u].x);
                const int ch = (int)(w[u] & 127u);
                for (int a = 0; a < g; ++a) {
                    const float2 mi = mls[a];
                    const float la = a < GP ? l0[u][a < GP ? a : 0] : lrow[a * T_max + (ok[u] ? t[u] : 0)];
                    if (ok[u] && mi.y > 0.0f) {
                        const float v = __expf(la - mi.x) * mi.y * d;
                        atomicAdd(&acc[a * kD + ch], (unsigned long long)__float2ll_rn(v * kFixScale));
                    }
                }
            }
        }
    }
    cluster.sync();  // every block's sums are complete (and visible across the cluster)
    if (rank == 0) {
        for (int e = threadIdx.x; e < g * kD; e += blockDim.x) {
            long long v = 0;
            for (int r = 0; r < nsub; ++r) v += (long long)cluster.map_shared_rank(acc, r)[e];
            if (v != 0) {
                float* pp = part + (((size_t)b * cfg.Hq + h * g + e / kD) * S + s) * kD + e % kD;
                *pp += (float)((double)v * kFixInv);
            }
        }
    }
    cluster.sync();  // the other blocks' shared memory stays until rank 0 has read it
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
// With ml != nullptr the merged partial itself is written instead: ml = (M, L) and
// out = sum_s e^(m_s-M) o_s (not divided by L).
__global__ void k_attn_merge(int S, const float2* __restrict__ st, const float* __restrict__ po,
                             float* __restrict__ out, float2* __restrict__ ml = nullptr) {
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
    if (ml) {
        out[(size_t)r * kD + ch] = o;
        if (ch == 0) ml[r] = make_float2(M, Ls);
    } else {
        out[(size_t)r * kD + ch] = Ls > 0.0f ? o / Ls : 0.0f;
    }
}

// A normalized output and its (M, L) turned into a partial: o = out * L (in place).
__global__ void k_to_partial(const float2* __restrict__ ml_in, float* __restrict__ o,
                             float2* __restrict__ ml_out) {
    const int r = blockIdx.x, ch = threadIdx.x;
    const float2 m = ml_in[r];
    o[(size_t)r * kD + ch] *= m.y;
    if (ch == 0) ml_out[r] = m;
}

// Merge of partials from `parts` sources laid out [part][rows]: out = sum_r e^(M_r-M) o_r /
// sum_r e^(M_r-M) L_r, taken in part order; 0 where no source has a token.
__global__ void k_parts_merge(int parts, int rows, const float2* __restrict__ ml,
                              const float* __restrict__ o, float* __restrict__ out) {
    const int r = blockIdx.x, ch = threadIdx.x;
    float M = -INFINITY;
    for (int k = 0; k < parts; ++k) M = fmaxf(M, ml[(size_t)k * rows + r].x);
    float Ls = 0.0f, acc = 0.0f;
    if (M > -INFINITY)
        for (int k = 0; k < parts; ++k) {
            const float2 x = ml[(size_t)k * rows + r];
            if (x.y > 0.0f) {
                const float w = expf(x.x - M);
                Ls += x.y * w;
                acc += o[((size_t)k * rows + r) * kD + ch] * w;
            }
        }
    out[(size_t)r * kD + ch] = Ls > 0.0f ? acc / Ls : 0.0f;
}

// ---------------------------------------------------------------------------------
// fp16 comparison kernel (the uncompressed baseline).  CTA = (split, sequence, kv head) with
// kF16W warps; warp w takes the split's 64-token chunks w, w + kF16W, ... and walks a chunk 4
// tokens per step with all 32 lanes on each token: lane l holds channels 4 (l & 15) + e of
// the first (l < 16) or second (l >= 16) half of the rotate-half pairs p = 4 (l & 15) + e,
// e < 4, loaded 8 bytes per lane (one whole 256-byte row per warp instruction), and the rows
// of the next step are loaded before the current step is used.  RoPE turns the query instead
// of the key: the term of channel p (first half) is k (cos qa + sin qb), of channel p + 64
// k (cos qb - sin qa), with (cos, sin) of t theta_p from the per-call tables at each chunk
// start and advanced by one token's rotation within the chunk.  Each warp keeps an online
// softmax per query head; the warps are merged in order at the end.
constexpr int kF16W = 8;

__global__ void k_fp16_prep(kvq_cfg cfg, const uint16_t* q, const int32_t* qpos, int nhi,
                            float* qr, float2* thi, float2* tlo) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int nq = cfg.B * cfg.Hq * 64, nh = nhi * 64, nl = kTrigLo * 64;
    if (e < nq) {
        const int p = e & 63, bh = e >> 6, b = bh / cfg.Hq;
        double cq, sq;
        rope_cs64((double)qpos[b], rope_freq(cfg.rope_theta, p), &cq, &sq);
        const uint16_t* qv = q + (size_t)bh * kD;
        const double qa = (double)h2f(qv[p]), qb = (double)h2f(qv[p + 64]);
        qr[(size_t)bh * kD + p] = (float)((qa * cq - qb * sq) * (double)kInvSqrtD);
        qr[(size_t)bh * kD + p + 64] = (float)((qa * sq + qb * cq) * (double)kInvSqrtD);
    } else if (e < nq + nh) {
        const int f = e - nq, p = f & 63, j = f >> 6;
        double cc, ss;
        rope_cs64((double)j * kTrigLo, rope_freq(cfg.rope_theta, p), &cc, &ss);
        thi[f] = make_float2((float)cc, (float)ss);
    } else if (e < nq + nh + nl) {
        const int f = e - nq - nh, p = f & 63, j = f >> 6;
        double cc, ss;
        rope_cs64((double)j, rope_freq(cfg.rope_theta, p), &cc, &ss);
        tlo[f] = make_float2((float)cc, (float)ss);
    }
}

__device__ __forceinline__ void half4_to_float(uint2 r, float (&f)[4]) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

template <int G>
__global__ void __launch_bounds__(kF16W * 32) k_fp16_attn(
    kvq_cfg cfg, const uint16_t* __restrict__ K, const uint16_t* __restrict__ V, int Tst,
    const int32_t* __restrict__ lens, const float* __restrict__ qr, const float2* __restrict__ thi,
    const float2* __restrict__ tlo, int Ls, int S, int max_len, float2* __restrict__ st,
    float* __restrict__ po) {
    __shared__ float wm[kF16W][G], wl[kF16W][G];
    __shared__ float wo[kF16W][G][kD];
    const int s = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4, e0 = 4 * (lane & 15);
    const int len = min(lens[b], max_len);
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    float U[G][4], W[G][4];
#pragma unroll
    for (int a = 0; a < G; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float* qv = qr + ((size_t)b * Hq + h * G + a) * kD;
            const float qa = qv[e0 + e], qb = qv[e0 + e + 64];
            U[a][e] = half ? qb : qa;
            W[a][e] = half ? -qa : qb;
        }
    float2 R1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) R1[e] = tlo[64 + e0 + e];  // one token's rotation
    float m[G], l[G], o[G][4];
#pragma unroll
    for (int a = 0; a < G; ++a) {
        m[a] = -INFINITY;
        l[a] = 0.0f;
        o[a][0] = o[a][1] = o[a][2] = o[a][3] = 0.0f;
    }
    const size_t rs = (size_t)Hkv * kD;  // elements between consecutive tokens
    const uint16_t* Kb = K + ((size_t)b * Tst * Hkv + h) * kD + e0 + 64 * half;
    const uint16_t* Vb = V + ((size_t)b * Tst * Hkv + h) * kD + e0 + 64 * half;
    const int jt = 2 * half + ((lane >> 3) & 1);  // token of the step this lane's logit ends on
    for (int cc = warp;; cc += kF16W) {
        const int tc = t_begin + cc * kChunk;
        if (tc >= t_end) break;
        const int n = min(kChunk, t_end - tc);
        float2 ph[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) ph[e] = trig_at(thi, tlo, tc, e0 + e);
        uint2 kr[4], vr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool ok = j < n;
            kr[j] = ok ? *reinterpret_cast<const uint2*>(Kb + (size_t)(tc + j) * rs) : make_uint2(0, 0);
            vr[j] = ok ? *reinterpret_cast<const uint2*>(Vb + (size_t)(tc + j) * rs) : make_uint2(0, 0);
        }
        for (int j0 = 0; j0 < n; j0 += 4) {
            uint2 kn[4], vn[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool ok = j0 + 4 + j < n;
                kn[j] = ok ? *reinterpret_cast<const uint2*>(Kb + (size_t)(tc + j0 + 4 + j) * rs)
                           : make_uint2(0, 0);
                vn[j] = ok ? *reinterpret_cast<const uint2*>(Vb + (size_t)(tc + j0 + 4 + j) * rs)
                           : make_uint2(0, 0);
            }
            float lp[G][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float kf[4];
                half4_to_float(kr[j], kf);
#pragma unroll
                for (int a = 0; a < G; ++a) {
                    float acc = 0.0f;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc = fmaf(kf[e], fmaf(ph[e].x, U[a][e], ph[e].y * W[a][e]), acc);
                    lp[a][j] = acc;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) ph[e] = cmul(ph[e], R1[e]);
            }
            const bool b3 = (lane >> 3) & 1;
            const bool valid = tc + j0 + jt < t_end;
            float pj[G][4];
#pragma unroll
            for (int a = 0; a < G; ++a) {
                // transposed reduction over the 32 lanes: lane ends with token jt's logit
                const float x0 = (half ? lp[a][2] : lp[a][0]) +
                                 __shfl_xor_sync(0xffffffffu, half ? lp[a][0] : lp[a][2], 16);
                const float x1 = (half ? lp[a][3] : lp[a][1]) +
                                 __shfl_xor_sync(0xffffffffu, half ? lp[a][1] : lp[a][3], 16);
                float y = (b3 ? x1 : x0) + __shfl_xor_sync(0xffffffffu, b3 ? x0 : x1, 8);
                y += __shfl_xor_sync(0xffffffffu, y, 4);
                y += __shfl_xor_sync(0xffffffffu, y, 2);
                y += __shfl_xor_sync(0xffffffffu, y, 1);
                const float lg = valid ? y : -INFINITY;
                float mx = lg;
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                if (mx > m[a]) {
                    const float sc = m[a] == -INFINITY ? 0.0f : __expf(m[a] - mx);
                    l[a] *= sc;
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[a][e] *= sc;
                    m[a] = mx;
                }
                const float p = valid ? __expf(lg - m[a]) : 0.0f;
                if ((lane & 7) == 0) l[a] += p;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    pj[a][j] = __shfl_sync(0xffffffffu, p, (j >> 1) * 16 + (j & 1) * 8);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float vf[4];
                half4_to_float(vr[j], vf);
#pragma unroll
                for (int a = 0; a < G; ++a)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[a][e] = fmaf(pj[a][j], vf[e], o[a][e]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kr[j] = kn[j];
                vr[j] = vn[j];
            }
        }
    }
#pragma unroll
    for (int a = 0; a < G; ++a) {
        // l: the owner lanes (lane & 7 == 0) summed in lane order
        float lt = l[a];
#pragma unroll
        for (int off = 8; off < 32; off <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, off);
        if (lane == 0) {
            wm[warp][a] = m[a];
            wl[warp][a] = lt;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) wo[warp][a][e0 + e + 64 * half] = o[a][e];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
        const int a = idx / kD, ch = idx % kD;
        float M = -INFINITY;
        for (int w2 = 0; w2 < kF16W; ++w2) M = fmaxf(M, wm[w2][a]);
        float Ls_ = 0.0f, oo = 0.0f;
        if (M > -INFINITY)
            for (int w2 = 0; w2 < kF16W; ++w2)
                if (wm[w2][a] > -INFINITY) {
                    const float sc = expf(wm[w2][a] - M);
                    Ls_ = fmaf(wl[w2][a], sc, Ls_);
                    oo = fmaf(wo[w2][a][ch], sc, oo);
                }
        const size_t r = (size_t)b * Hq + h * G + a;
        po[(r * S + s) * kD + ch] = oo;
        if (ch == 0) st[r * S + s] = make_float2(M, Ls_);
    }
}

}  // namespace

using namespace kvq_host;

// Query heads per CTA of the streaming kernels and the number of kv heads they span.
static int hpc_of(const kvq_cfg* cfg) { return cfg->Hq % 4 == 0 ? 4 : (cfg->Hq % 2 == 0 ? 2 : 1); }
static int kvb_of(const kvq_cfg* cfg, int hpc) {
    const int g = cfg->Hq / cfg->Hkv;
    int m = 1;
    for (int hq0 = 0; hq0 < cfg->Hq; hq0 += hpc) {
        const int span = (hq0 + hpc - 1) / g - hq0 / g + 1;
        m = span > m ? span : m;
    }
    return m;
}

// Splits of the decode grid.  The CTAs of a split are one per (sequence, kv head) for the
// table kernels of 2- and 3-bit codes with 1, 2 or 4 query heads per kv head, else one per
// (sequence, group of hpc query heads); each CTA holds an SM.  The count minimises
// waves x (setup + stages): waves of 148 CTAs, stages of 256 tokens per CTA, and a setup
// (tables, barriers) worth about two stages -- so short caches get few long splits instead of
// many CTAs that mostly build tables.
static int auto_splits(const kvq_cfg* cfg, int max_len) {
    const int g = cfg->Hq / cfg->Hkv;
    const bool tab = cfg->bits <= 3 && (g == 1 || g == 2 || g == 4);
    const long long groups = tab ? (long long)cfg->B * cfg->Hkv : (long long)cfg->B * (cfg->Hq / hpc_of(cfg));
    int maxs = (max_len + 255) / 256;
    if (maxs > 4096) maxs = 4096;
    if (maxs < 1) maxs = 1;
    long long best = -1;
    int bestS = 1;
    for (int S = 1; S <= maxs; ++S) {
        const long long waves = (S * groups + 147) / 148;
        const long long stages = (((long long)max_len + S - 1) / S + 255) / 256;
        const long long cost = waves * (2 + stages);
        if (best < 0 || cost < best) {
            best = cost;
            bestS = S;
        }
    }
    return bestS;
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

// Per-call tables of the QK path (kvq_decode_qk's workspace).
struct QKTables {
    float* qr;     // [B][Hq][128]
    float2* thi;   // [nhi][64]
    float2* tlo;   // [256][64]
    float* zk;     // [B][Hkv][128]
    int nhi;
    size_t bytes;
};
static QKTables qk_tables(const kvq_cfg* cfg, int max_len, void* ws) {
    QKTables t;
    t.nhi = (max_len + kTrigLo - 1) / kTrigLo;
    const size_t sq = align_up((size_t)cfg->B * cfg->Hq * kD * 4);
    const size_t sh = align_up((size_t)t.nhi * 64 * 8);
    const size_t sl = align_up((size_t)kTrigLo * 64 * 8);
    const size_t sz = align_up((size_t)cfg->B * cfg->Hkv * kD * 4);
    char* w = (char*)ws;
    t.qr = (float*)w;
    t.thi = (float2*)(w + sq);
    t.tlo = (float2*)(w + sq + sh);
    t.zk = (float*)(w + sq + sh + sl);
    t.bytes = sq + sh + sl + sz;
    return t;
}

typedef void (*QKKernel)(kvq_cfg, kvq_cache, kvq_codebook, const float*, const float2*,
                         const float2*, int, int, int, float*);
typedef void (*QKQKernel)(kvq_cfg, kvq_cache, kvq_codebook, const float*, const float2*,
                          const float2*, int, int, float*);
typedef void (*PVQKernel)(kvq_cfg, kvq_cache, kvq_codebook, const float*, const float2*, int,
                          int, int, float*);
typedef void (*PVKernel)(kvq_cfg, kvq_cache, kvq_codebook, const float*, const float2*, int, int,
                         int, int, float*);

template <int BITS>
static QKKernel qk_kernel(int hpc, bool share) {
    if constexpr (BITS == 4) {
        return k_qk<4, 1, true>;  // one head's 256-entry pair tables already take 128 KB
    } else {
        if (hpc == 4) return share ? k_qk<BITS, 4, true> : k_qk<BITS, 4, false>;
        if (hpc == 2) return share ? k_qk<BITS, 2, true> : k_qk<BITS, 2, false>;
        return k_qk<BITS, 1, true>;
    }
}

template <int BITS>
static PVKernel pv_kernel(int hpc, bool share) {
    if (hpc == 4) return share ? k_pv<BITS, 4, true> : k_pv<BITS, 4, false>;
    if (hpc == 2) return share ? k_pv<BITS, 2, true> : k_pv<BITS, 2, false>;
    return k_pv<BITS, 1, true>;
}

// QK over the quantized cache into logits, key-outlier corrections, split statistics.
static int run_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                  const uint16_t* q, const int32_t* qpos, int max_len, float* logits,
                  float* stats, int S, int Ls, const QKTables& T, cudaStream_t st,
                  int pos_off = 0) {
    {
        const int n = cfg->B * cfg->Hq * 64 + T.nhi * 64 + kTrigLo * 64 + cfg->B * cfg->Hkv * kD;
        k_decode_prep<<<(n + 255) / 256, 256, 0, st>>>(*cfg, *cache, *cbK, q, qpos, T.nhi,
                                                        pos_off, T.qr, T.thi, T.tlo, T.zk);
    }
    const int g = cfg->Hq / cfg->Hkv;
    if (cfg->bits <= 3 && (g == 1 || g == 2 || g == 4)) {
        QKQKernel kq = g == 1 ? (cfg->bits == 2 ? k_qk_quad<2> : k_qk_quad<3>)
                     : g == 2 ? (cfg->bits == 2 ? k_qk_grp<2, 2> : k_qk_grp<3, 2>)
                              : (cfg->bits == 2 ? k_qk_grp<2, 4> : k_qk_grp<3, 4>);
        const int smem = qq_plan(cfg->bits).total;
        cudaError_t ce = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (ce) return record_cuda(ce);
        dim3 grid(S, cfg->B, cfg->Hkv);
        kq<<<grid, kQWarps * 32 + 32, smem, st>>>(*cfg, *cache, *cbK, T.qr, T.thi, T.tlo, Ls,
                                                    max_len, logits);
    } else {
    const int hpc = cfg->bits == 4 ? 1 : hpc_of(cfg);
    const int kvb = kvb_of(cfg, hpc);
    QKKernel kern = cfg->bits == 2 ? qk_kernel<2>(hpc, kvb == 1)
                  : cfg->bits == 3 ? qk_kernel<3>(hpc, kvb == 1)
                                   : qk_kernel<4>(hpc, kvb == 1);
    const int smem = qk_plan(cfg->bits, hpc, kvb).total;
    cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B, cfg->Hq / hpc);
    kern<<<grid, qk_warps(hpc) * 32 + 32, smem, st>>>(*cfg, *cache, *cbK, T.qr, T.thi, T.tlo,
                                                            Ls, max_len, kvb, logits);
    }
    const int nch = (max_len + kChunk - 1) / kChunk;
    dim3 go((nch + kOutChunks - 1) / kOutChunks, cfg->B * cfg->Hkv);
    const int gq = cfg->Hq / cfg->Hkv;
    auto ko = gq == 1 ? k_key_outliers<1> : gq == 2 ? k_key_outliers<2>
            : gq == 4 ? k_key_outliers<4> : k_key_outliers<0>;
    ko<<<go, kOutThreads, 0, st>>>(*cfg, *cache, T.qr, T.thi, T.tlo, T.zk, max_len, logits);
    dim3 gs(S, cfg->B * cfg->Hq);
    k_logit_stats<<<gs, kStatThreads, 0, st>>>(*cfg, cache->len, logits, Ls, S, max_len, (float2*)stats);
    return record_cuda(cudaGetLastError());
}

extern "C" int kvq_decode_qk_workspace(const kvq_cfg* cfg, int32_t max_len, size_t* bytes) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    *bytes = qk_tables(cfg, max_len, nullptr).bytes;
    return KVQ_OK;
}

extern "C" int kvq_decode_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                             const uint16_t* q, const int32_t* qpos, int32_t max_len,
                             float* logits, float* stats, int32_t splits, void* workspace,
                             size_t workspace_bytes, void* stream) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if ((e = check_cache(cfg, cache)) || (e = check_codebook(cbK))) return e;
    if (!q || !qpos || !logits || !stats || !workspace) return KVQ_ERR_NULL;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    const QKTables T = qk_tables(cfg, max_len, workspace);
    if (workspace_bytes < T.bytes) return KVQ_ERR_WORKSPACE;
    return run_qk(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, Ls, T, (cudaStream_t)stream);
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

// PV over the quantized cache into per-split partials, their sum, value-outlier corrections.
static int run_pv(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbV,
                  const float* logits, const float* ml, int max_len, float* out, float* part,
                  int S, int Ls, cudaStream_t st) {
    if (cfg->Hq == cfg->Hkv) {
        PVQKernel kq = cfg->bits == 2 ? k_pv_quad<2> : cfg->bits == 3 ? k_pv_quad<3> : k_pv_quad<4>;
        const int smem = pq_plan(cfg->bits).total;
        cudaError_t ce = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (ce) return record_cuda(ce);
        dim3 grid(S, cfg->B, cfg->Hq);
        kq<<<grid, kQWarps * 32 + 32, smem, st>>>(*cfg, *cache, *cbV, logits, (const float2*)ml, Ls,
                                                    S, max_len, part);
    } else if (cfg->Hq == 2 * cfg->Hkv || cfg->Hq == 4 * cfg->Hkv) {
        const int g = cfg->Hq / cfg->Hkv;
        PVQKernel kg = g == 2 ? (cfg->bits == 2 ? k_pv_grp<2, 2> : cfg->bits == 3 ? k_pv_grp<3, 2> : k_pv_grp<4, 2>)
                              : (cfg->bits == 2 ? k_pv_grp<2, 4> : cfg->bits == 3 ? k_pv_grp<3, 4> : k_pv_grp<4, 4>);
        const int smem = pq_plan(cfg->bits, g).total;
        cudaError_t ce = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (ce) return record_cuda(ce);
        dim3 grid(S, cfg->B, cfg->Hkv);
        kg<<<grid, kQWarps * 32 + 32, smem, st>>>(*cfg, *cache, *cbV, logits, (const float2*)ml, Ls,
                                                    S, max_len, part);
    } else {
    const int hpc = hpc_of(cfg);
    const int kvb = kvb_of(cfg, hpc);
    PVKernel kern = cfg->bits == 2 ? pv_kernel<2>(hpc, kvb == 1)
                  : cfg->bits == 3 ? pv_kernel<3>(hpc, kvb == 1)
                                   : pv_kernel<4>(hpc, kvb == 1);
    const int smem = pv_plan(cfg->bits, hpc, kvb).total;
    cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B, cfg->Hq / hpc);
    kern<<<grid, pv_warps(hpc) * 32 + 32, smem, st>>>(*cfg, *cache, *cbV, logits,
                                                            (const float2*)ml, Ls, S, max_len,
                                                            kvb, part);
    }

    const bool mha = cfg->Hq == cfg->Hkv;
    const int gq = cfg->Hq / cfg->Hkv;
    auto vo = cfg->bits == 2 ? (mha ? k_value_outliers<2, 1> : gq == 2 ? k_value_outliers<2, 2> : gq == 4 ? k_value_outliers<2, 4> : k_value_outliers<2, 0>)
            : cfg->bits == 3 ? (mha ? k_value_outliers<3, 1> : gq == 2 ? k_value_outliers<3, 2> : gq == 4 ? k_value_outliers<3, 4> : k_value_outliers<3, 0>)
                             : (mha ? k_value_outliers<4, 1> : gq == 2 ? k_value_outliers<4, 2> : gq == 4 ? k_value_outliers<4, 4> : k_value_outliers<4, 0>);
    {
        // blocks per split: enough for about four per SM, at most a portable cluster of 8
        const long long base = (long long)S * cfg->B * cfg->Hkv;
        int nsub = (int)((4 * 148 + base - 1) / base);
        nsub = nsub < 1 ? 1 : (nsub > 8 ? 8 : nsub);
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(S * nsub, cfg->B * cfg->Hkv);
        lc.blockDim = dim3(kOutThreads);
        lc.dynamicSmemBytes = 0;
        lc.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = nsub;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        lc.attrs = at;
        lc.numAttrs = 1;
        cudaError_t ce = cudaLaunchKernelEx(&lc, vo, *cfg, *cache, *cbV, logits, (const float2*)ml,
                                            Ls, S, max_len, part);
        if (ce) return record_cuda(ce);
    }
    k_pv_reduce<<<cfg->B * cfg->Hq, kD, 0, st>>>(S, part, out);
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
    return run_pv(cfg, cache, cbV, logits, ml, max_len, out, part, S, Ls, (cudaStream_t)stream);
}

// The fused path's workspace: the split path's without the [B][Hq][T_max] logits.
static size_t fused_ws_bytes(const kvq_cfg* cfg, int S, int max_len) {
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    return align_up(BH * S * 8) + align_up(BH * 8) + align_up(BH * S * kD * 4) +
           qk_tables(cfg, max_len, nullptr).bytes;
}

static size_t split_ws_bytes(const kvq_cfg* cfg, int S, int max_len) {
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    return align_up(BH * (size_t)cfg->T_max * 4)   // logits
           + align_up(BH * S * 8)                  // stats
           + align_up(BH * 8)                      // ml
           + align_up(BH * S * kD * 4)             // partials
           + qk_tables(cfg, max_len, nullptr).bytes;
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

// Decode over a cache whose row t sits at position t + pos_off.  With ml_part == nullptr,
// out receives the normalized attention output; otherwise out receives the unnormalized
// partial o = sum_t e^(l_t - M) vhat_t and ml_part its (M, L).
static int decode_core(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                       const kvq_codebook* cbV, const uint16_t* q, const int32_t* qpos,
                       int32_t max_len, int32_t pos_off, float* out, float2* ml_part,
                       void* workspace, size_t workspace_bytes, int32_t splits, void* stream,
                       bool fused = false) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if ((e = check_cache(cfg, cache)) || (e = check_codebook(cbK)) || (e = check_codebook(cbV)))
        return e;
    if (!workspace || !out || !q || !qpos) return KVQ_ERR_NULL;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    if (pos_off < 0 || (int64_t)pos_off + max_len > (int64_t)1 << 30) return KVQ_ERR_RANGE;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    if (fused && !fused_supported(cfg)) return KVQ_ERR_UNSUPPORTED;
    if (workspace_bytes < (fused ? fused_ws_bytes(cfg, S, max_len) : split_ws_bytes(cfg, S, max_len)))
        return KVQ_ERR_WORKSPACE;
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    char* w = (char*)workspace;
    float* logits = (float*)w;
    if (!fused) w += align_up(BH * (size_t)cfg->T_max * 4);
    float* stats = (float*)w;
    w += align_up(BH * S * 8);
    float* ml = (float*)w;
    w += align_up(BH * 8);
    float* part = (float*)w;
    w += align_up(BH * S * kD * 4);
    const QKTables T = qk_tables(cfg, max_len, w);
    cudaStream_t st = (cudaStream_t)stream;
    if (fused) {
        // one pass: per-call tables, the fused kernel's per-split (m, l, o), the split merge
        const int n = cfg->B * cfg->Hq * 64 + T.nhi * 64 + kTrigLo * 64 + cfg->B * cfg->Hkv * kD;
        k_decode_prep<<<(n + 255) / 256, 256, 0, st>>>(*cfg, *cache, *cbK, q, qpos, T.nhi,
                                                        pos_off, T.qr, T.thi, T.tlo, T.zk);
        if ((e = record_cuda(cudaGetLastError()))) return e;
        if ((e = run_fused(cfg, cache, cbK, cbV, T.qr, T.thi, T.tlo, T.zk, max_len, S, Ls,
                           (float2*)stats, part, st)))
            return e;
        k_attn_merge<<<(int)BH, kD, 0, st>>>(S, (const float2*)stats, part, out, ml_part);
        return record_cuda(cudaGetLastError());
    }
    if ((e = run_qk(cfg, cache, cbK, q, qpos, max_len, logits, stats, S, Ls, T, st, pos_off)))
        return e;
    if ((e = kvq_softmax_merge(cfg, stats, S, ml, stream))) return e;
    if ((e = run_pv(cfg, cache, cbV, logits, ml, max_len, out, part, S, Ls, st))) return e;
    if (ml_part) {
        k_to_partial<<<(int)BH, kD, 0, st>>>((const float2*)ml, out, ml_part);
        return record_cuda(cudaGetLastError());
    }
    return KVQ_OK;
}

extern "C" int kvq_decode_attention(const kvq_cfg* cfg, const kvq_cache* cache,
                                    const kvq_codebook* cbK, const kvq_codebook* cbV,
                                    const uint16_t* q, const int32_t* qpos, int32_t max_len,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    int32_t splits, void* stream) {
    return decode_core(cfg, cache, cbK, cbV, q, qpos, max_len, 0, out, nullptr, workspace,
                       workspace_bytes, splits, stream);
}

extern "C" int kvq_decode_fused_workspace(const kvq_cfg* cfg, int32_t max_len, int32_t splits,
                                          size_t* bytes) {
    int e = check_decode(cfg, max_len);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    if (!fused_supported(cfg)) return KVQ_ERR_UNSUPPORTED;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    *bytes = fused_ws_bytes(cfg, S, max_len);
    return KVQ_OK;
}

extern "C" int kvq_decode_attention_fused(const kvq_cfg* cfg, const kvq_cache* cache,
                                          const kvq_codebook* cbK, const kvq_codebook* cbV,
                                          const uint16_t* q, const int32_t* qpos, int32_t max_len,
                                          float* out, void* workspace, size_t workspace_bytes,
                                          int32_t splits, void* stream) {
    return decode_core(cfg, cache, cbK, cbV, q, qpos, max_len, 0, out, nullptr, workspace,
                       workspace_bytes, splits, stream, true);
}

extern "C" int kvq_decode_partial(const kvq_cfg* cfg, const kvq_cache* cache,
                                  const kvq_codebook* cbK, const kvq_codebook* cbV,
                                  const uint16_t* q, const int32_t* qpos, int32_t max_len,
                                  int32_t pos_offset, float* ml, float* o, void* workspace,
                                  size_t workspace_bytes, int32_t splits, void* stream) {
    if (!ml) return KVQ_ERR_NULL;
    return decode_core(cfg, cache, cbK, cbV, q, qpos, max_len, pos_offset, o, (float2*)ml,
                       workspace, workspace_bytes, splits, stream);
}

extern "C" int kvq_merge_partials(const kvq_cfg* cfg, int32_t parts, const float* ml,
                                  const float* o, float* out, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!ml || !o || !out) return KVQ_ERR_NULL;
    if (parts < 1 || parts > 4096) return KVQ_ERR_RANGE;
    const int rows = cfg->B * cfg->Hq;
    k_parts_merge<<<rows, kD, 0, (cudaStream_t)stream>>>(parts, rows, (const float2*)ml, o, out);
    return record_cuda(cudaGetLastError());
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
    const int g = cfg->Hq / cfg->Hkv;
    if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_UNSUPPORTED;
    int S, Ls;
    if ((e = resolve_splits(cfg, max_len, splits, &S, &Ls))) return e;
    const size_t BH = (size_t)cfg->B * cfg->Hq;
    const size_t a0 = align_up(BH * S * 8), a1 = align_up(BH * S * kD * 4);
    const QKTables T = qk_tables(cfg, max_len, (char*)workspace + a0 + a1);
    if (workspace_bytes < a0 + a1 + T.bytes) return KVQ_ERR_WORKSPACE;
    float2* st = (float2*)workspace;
    float* po = (float*)((char*)workspace + a0);
    cudaStream_t s = (cudaStream_t)stream;
    const int n = cfg->B * cfg->Hq * 64 + T.nhi * 64 + kTrigLo * 64;
    k_fp16_prep<<<(n + 255) / 256, 256, 0, s>>>(*cfg, q, qpos, T.nhi, T.qr, T.thi, T.tlo);
    dim3 grid(S, cfg->B, cfg->Hkv);
    auto kern = g == 1 ? k_fp16_attn<1> : g == 2 ? k_fp16_attn<2> : g == 4 ? k_fp16_attn<4>
                       : k_fp16_attn<8>;
    kern<<<grid, kF16W * 32, 0, s>>>(*cfg, K, V, T_stride, len, T.qr, T.thi, T.tlo, Ls, S, max_len,
                                     st, po);
    k_attn_merge<<<(int)BH, kD, 0, s>>>(S, st, po, out);
    return record_cuda(cudaGetLastError());
}
