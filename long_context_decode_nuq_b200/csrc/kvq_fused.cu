// Fused single-pass decode attention over the quantized cache, for kv heads that serve one
// query head each (multi-head attention) and 2- or 3-bit codes: QK with NUQ lookup and RoPE,
// the key-outlier correction, the softmax, PV and the value-outlier correction in one kernel
// per (split, sequence, head), with no logits in memory.  (The decode side of techniques
// (i)-(iv): study.space summary, custom kernels for memory- and bandwidth-bound decode;
// phantomic12 research note, components (1)-(4).)
//
// A CTA has 16 consumer warps and three helper warps and walks its split in 256-token stages
// through a ring of kFSlots shared-memory slots.
//  - Issuing warp: per stage, bulk copies (cp.async.bulk, completion counted on an mbarrier;
//    one destination CTA) of the key code blocks, the tokens' value (off, half), and the stage's key-
//    and value-outlier entries (up to kFEnt of each; entries past that are read from global
//    memory).  It waits only for the slot to be released, so copies run a full ring ahead.
//  - Key warp: per stage, the (cos, sin) of the stage start for the 64 RoPE pairs and, once
//    the stage's copies have landed, the key-outlier correction of every token,
//    kc[tau] = sum over the token's entries of (x - zhat_c) r, r the rotated query component
//    that meets channel c at the token, each term added in 2^-32 fixed point with an integer
//    atomic (associative, so the sum is the same on every run).
//  - Value helper: per stage, once its copies have landed, the dense value the cache holds at
//    a value outlier of each token, zv = off + half L[code of 0], and the first value-outlier
//    entry of each 16-token slice of the stage.
//  - Consumer warp w owns tokens [16 w, 16 w + 16) of every stage and keeps its own online
//    softmax state (running max m, sum l, sum of p off, and the value accumulators).  Per
//    stage: QK over its four quads from the key ring (tables of e^{i j theta_p} Z_p(code) for
//    the four token offsets j of a quad, one phase per quad and pair, as in the split-path QK
//    kernel), plus kc; its max, a rescale when it rises, p = exp(l - m); PV over the same
//    quads with value codes read straight from global memory one stage ahead, each (La, Lb)
//    pair looked up as two 16-bit level patterns (the levels are (u << 16) | u binary32
//    values, so two byte permutes rebuild them exactly); the value outliers of its slice,
//    p (x - zv), added per channel in entry order.
// At the end the 16 warp states are merged in warp order into the split's (m, l, o); the
// splits are merged afterwards (k_attn_merge).
#include "kvq_common.cuh"
#include "kvq_device.cuh"

using namespace kvq;

namespace {

constexpr int kFW = 16;                   // consumer warps
constexpr int kFCons = kFW * 32;          // consumer threads
constexpr int kFThreads = kFCons + 96;    // + issuing, key and value-helper warps
constexpr int kFQuads = 64;               // token quads per stage
constexpr int kFTok = 4 * kFQuads;        // tokens per stage (the lo trig table spans a stage)
constexpr int kFSlots = 3;                // stages in flight
constexpr uint32_t kFAnchor = 32768;      // shared-window address of the QK tables
constexpr int kFEnt = 512;                // outlier entries of each kind staged per slot
constexpr int kFSide = 16;                // words of a slot's side record
constexpr float kKcScale = 4294967296.0f;           // 2^32
constexpr double kKcInv = 1.0 / 4294967296.0;       // 2^-32
static_assert(kFTok == kTrigLo, "the in-stage rotation comes from the lo trig table");

// Shared-memory plan.  The small buffers sit from the window base up to the PV table, which
// ends at kFAnchor; the QK tables start at kFAnchor (a multiple of their j-slice and of the
// PV table's size, so a lookup address is one OR); the key ring and the per-warp value
// accumulators follow the tables.  `total` is the dynamic size for a window base of 0; a
// kernel whose window base leaves too little room below the PV table reports
// KVQ_STATUS_SMEM_LAYOUT and writes nothing.
struct FusedPlan {
    int base, kc, zv, vsl, side, wsm, wp, scr, zk, qv, levk, levv, bar, flag, small;
    int pv, jslice;
    int stage, ring, vps, kent, vent, accv, post;
    int total;
};
__host__ __device__ inline FusedPlan fused_plan(int bits) {
    FusedPlan p;
    int o = 0;
    p.base = o; o += kFSlots * 64 * 16;   // [slot][pair] (c, c, s, s) at the stage start
    p.kc = o;   o += kFSlots * kFTok * 8; // [slot][token] key-outlier correction, 2^-32 fixed point
    p.zv = o;   o += kFSlots * kFTok * 4; // [slot][token] dense value at a value outlier
    p.vsl = o;  o += kFSlots * 32 * 4;    // [slot][slice] first value entry (17 used)
    p.side = o; o += kFSlots * kFSide * 4;  // [slot] staged entry ranges and value-param count
    p.wsm = o;  o += kFW * 16 * 8;        // [warp][token] (w, w), w = p half
    p.wp = o;   o += kFW * 16 * 4;        // [warp][token] p
    p.scr = o;  o += kFW * 32 * 4;        // [warp][lane] scratch
    p.zk = o;   o += kD * 4;              // dense key value at a key outlier, per channel
    p.qv = o;   o += kD * 4;              // rotated, scaled query
    p.levk = o; o += 16 * 4;
    p.levv = o; o += 16 * 4;
    p.bar = o;  o += 3 * kFSlots * 8;     // copy, full, empty
    p.flag = o; o += 16;
    p.small = o;
    p.pv = (1 << (2 * bits)) * 32 * 4;    // [entry][32 lane copies] 16-bit level pair
    p.jslice = (1 << (2 * bits)) * 64 * 8;
    o = 0;
    p.stage = kFQuads * 16 * bits * 4;
    p.ring = o; o += kFSlots * p.stage;
    p.vps = o;  o += kFSlots * kFTok * 8; // [slot][token] value (off, half)
    p.kent = o; o += kFSlots * kFEnt * 4; // [slot] key-outlier entries of the stage
    p.vent = o; o += kFSlots * kFEnt * 4; // [slot] value-outlier entries of the stage
    p.accv = o; o += kFW * kD * 4;        // [warp][channel] value-outlier sums
    p.post = o;
    p.total = (int)kFAnchor + 4 * p.jslice + p.post;
    return p;
}

// acc[ch] += v for the lanes with ok, in lane order per channel (the lowest lane of each
// group of equal channels sums the group's values through scr).
__device__ __forceinline__ void add_ordered(float* acc, float* scr, int ch, float v, bool ok,
                                            int lane) {
    const unsigned grp = __match_any_sync(0xffffffffu, ok ? ch : -1 - lane);
    scr[lane] = v;
    __syncwarp();
    if (ok && __ffs(grp) - 1 == lane) {
        float sum = 0.0f;
        for (unsigned gg = grp; gg; gg &= gg - 1) sum += scr[__ffs(gg) - 1];
        acc[ch] += sum;
    }
    __syncwarp();
}

// Bounded wait by every lane, made warp-uniform; false (and the abort flag set) on a timeout
// or when another warp has aborted.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* flag,
                                          int32_t* status) {
    const bool ok = mbar_wait(bar, parity);
    if (__any_sync(0xffffffffu, !ok)) {
        if ((threadIdx.x & 31) == 0) {
            atomicOr(flag, 1);
            set_status(status, KVQ_STATUS_WAIT_TIMEOUT);
        }
        return false;
    }
    return __shfl_sync(0xffffffffu, *(volatile int*)flag, 0) == 0;
}

template <int BITS>
__global__ void __launch_bounds__(kFThreads, 1)
    k_attn_quad(kvq_cfg cfg, kvq_cache c, kvq_codebook cbK, kvq_codebook cbV,
                const float* __restrict__ qr_all, const float2* __restrict__ thi,
                const float2* __restrict__ tlo, const float* __restrict__ zk_all, int Ls, int S,
                int max_len, float2* __restrict__ st_out, float* __restrict__ po_out) {
    using F = Fmt<BITS>;
    constexpr int NB = (1 << BITS) - 1;
    constexpr int P = 9;                  // entry bit of a QK table byte offset
    constexpr int JS = P + F::FW;         // j bit of a QK table byte offset
    constexpr uint32_t MASK = (uint32_t)(F::NT - 1) << P;
    constexpr uint32_t PVMASK = (uint32_t)(F::NT - 1) << 7;  // 32 copies x 4 bytes per entry
    extern __shared__ __align__(128) uint8_t sm[];
    const FusedPlan L = fused_plan(BITS);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.x, b = blockIdx.y, hq = blockIdx.z;
    const int Hq = cfg.Hq, Hkv = cfg.Hkv, kvh = hq / (Hq / Hkv);
    const size_t row = (size_t)b * Hq + hq;
    const size_t li = (size_t)b * Hkv + kvh;
    int len = c.len[b];
    if (len > max_len) {
        if (tid == 0 && s == 0 && hq == 0) set_status(c.status, KVQ_STATUS_LEN_OVERFLOW);
        len = max_len;
    }
    const int t_begin = s * Ls, t_end = min(len, t_begin + Ls);
    if (t_begin >= t_end || sbase + (uint32_t)L.small > kFAnchor - (uint32_t)L.pv) {
        if (t_begin < t_end && tid == 0) set_status(c.status, KVQ_STATUS_SMEM_LAYOUT);
        if (tid < kD) po_out[(row * S + s) * kD + tid] = 0.0f;
        if (tid == 0) st_out[row * S + s] = make_float2(-INFINITY, 0.0f);
        return;
    }
    float4* base = reinterpret_cast<float4*>(sm + L.base);
    unsigned long long* kc = reinterpret_cast<unsigned long long*>(sm + L.kc);
    float* zv = reinterpret_cast<float*>(sm + L.zv);
    uint32_t* vsl = reinterpret_cast<uint32_t*>(sm + L.vsl);
    unsigned long long* wsm = reinterpret_cast<unsigned long long*>(sm + L.wsm);
    float* wp = reinterpret_cast<float*>(sm + L.wp);
    float* scr = reinterpret_cast<float*>(sm + L.scr);
    float* zks = reinterpret_cast<float*>(sm + L.zk);
    float* qs = reinterpret_cast<float*>(sm + L.qv);
    float* levk = reinterpret_cast<float*>(sm + L.levk);
    float* levv = reinterpret_cast<float*>(sm + L.levv);
    uint64_t* bcopy = reinterpret_cast<uint64_t*>(sm + L.bar);
    uint64_t* full = bcopy + kFSlots;
    uint64_t* empty = full + kFSlots;
    int* flag = reinterpret_cast<int*>(sm + L.flag);
    uint8_t* pvt = sm + (kFAnchor - (uint32_t)L.pv - sbase);
    uint8_t* tab = sm + (kFAnchor - sbase);
    uint8_t* post = tab + 4 * L.jslice;
    uint8_t* ring = post + L.ring;
    float* accv = reinterpret_cast<float*>(post + L.accv);
    const int nst = (t_end - t_begin + kFTok - 1) / kFTok;

    if (tid == 0) {
        for (int k = 0; k < kFSlots; ++k) {
            mbar_init(bcopy + k, 1);
            mbar_init(full + k, 2);   // key warp, value helper
            mbar_init(empty + k, kFW);
        }
        flag[0] = 0;
        flag[1] = 0;
        fence_mbar_init();
    }
    if (tid < kD) {
        zks[tid] = zk_all[li * kD + tid];
        qs[tid] = qr_all[row * kD + tid];
    }
    if (tid < 16) {
        levk[tid] = tid <= NB ? cbK.levels[tid] : 0.0f;
        levv[tid] = tid <= NB ? cbV.levels[tid] : 0.0f;
        if (tid <= NB) {
            // the PV table keeps 16 bits per level: the levels must be (u << 16) | u values
            const uint32_t u = __float_as_uint(cbV.levels[tid]);
            if ((u >> 16) != (u & 0xFFFFu)) set_status(c.status, KVQ_STATUS_CODEBOOK);
        }
    }
    for (int e = tid; e < kFW * kD; e += kFThreads) accv[e] = 0.0f;
    __syncthreads();
    // ---- QK tables: (X, Y) of Z_p(entry) turned by j theta_p (threads 0 .. 511)
    if (tid < 512) {
        const int p = tid & 63, r0 = tid >> 6;
        const float* kp = c.kparams + li * kD * 2;
        const float offa = kp[2 * p], halfa = kp[2 * p + 1];
        const float offb = kp[2 * (p + 64)], halfb = kp[2 * (p + 64) + 1];
        const float qa = qs[p], qb = qs[p + 64];
        const float A1 = qa * halfa, B1 = qb * halfb, C1 = qa * offa + qb * offb;
        const float A2 = qb * halfa, B2 = -qa * halfb, C2 = qb * offa - qa * offb;
        float2 rj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) rj[j] = tlo[j * 64 + p];
        unsigned long long* t64 = reinterpret_cast<unsigned long long*>(tab);
        for (int idx = r0; idx < F::NT; idx += 8) {
            const float La = levk[idx & NB], Lb = levk[idx >> BITS];
            const float X = fmaf(B1, Lb, fmaf(A1, La, C1));
            const float Y = fmaf(B2, Lb, fmaf(A2, La, C2));
#pragma unroll
            for (int j = 0; j < 4; ++j)
                t64[(j * F::NT + idx) * 64 + p] =
                    pk(fmaf(rj[j].x, X, rj[j].y * Y), fmaf(rj[j].x, Y, -rj[j].y * X));
        }
    }
    // ---- PV table: the 16-bit patterns of (L[xa], L[xb]) per entry, one copy per lane
    for (int e = tid; e < F::NT * 32; e += kFThreads) {
        const int idx = e >> 5;
        const uint32_t ua = __float_as_uint(levv[idx & NB]), ub = __float_as_uint(levv[idx >> BITS]);
        reinterpret_cast<uint32_t*>(pvt)[e] = (ua & 0xFFFFu) | (ub << 16);
    }
    __syncthreads();  // tables complete, barriers initialised

    const int i = lane & 15, hh = lane >> 4;
    unsigned long long O[4] = {0ull, 0ull, 0ull, 0ull};  // consumer lanes: (o[c], o[c + 64]), c = i + 16 k
    const float2* vpar = reinterpret_cast<const float2*>(c.vparams) + (size_t)b * cfg.T_max;
    const uint32_t* kent = c.kout + li * cfg.out_cap_k;
    const uint32_t* vent = c.vout + li * cfg.out_cap_v;
    uint32_t* side = reinterpret_cast<uint32_t*>(sm + L.side);  // [slot][kFSide]
    float2* vps = reinterpret_cast<float2*>(post + L.vps);
    uint32_t* kents = reinterpret_cast<uint32_t*>(post + L.kent);
    uint32_t* vents = reinterpret_cast<uint32_t*>(post + L.vent);
    // side[slot][]: 0 kB, 1 kN (staged key entries [kB, kB + kN)), 2 kE0, 3 kE1 (the stage's key
    // entries), 4..6 the key chunk boundaries, 7 the stage's chunks, 8 vB, 9 vN, 10 vE0, 11 vE1,
    // 12..14 the value chunk boundaries, 15 value params staged
    if (warp == kFW) {
        // ================= issuing warp: the stage's side record and its bulk copies
        const uint32_t* ksrc = c.kcodes + li * nquads(cfg.T_max) * F::BW;
        const uint32_t* kcp = c.kchunk + li * (nchunks(cfg.T_max) + 1);
        const uint32_t* vcp = c.vchunk + li * (nchunks(cfg.T_max) + 1);
        const uint32_t kcnt = c.kcount[li], vcnt = c.vcount[li];
        uint32_t kcpl = 0, vcpl = 0;  // chunk pointers of the next stage to issue (lanes 0 .. 4)
        auto load_cp = [&](int st) {
            const int tc = t_begin + st * kFTok, m0 = tc >> 6;
            const int nm = min(4, ((t_end + 63) >> 6) - m0);
            kcpl = lane <= nm ? min(kcp[m0 + lane], kcnt) : 0u;
            vcpl = lane <= nm ? min(vcp[m0 + lane], vcnt) : 0u;
        };
        load_cp(0);
        int issued = 0;
        for (int cc = 0; cc < nst; ++cc) {
            const int slot = cc % kFSlots;
            if (cc >= kFSlots &&
                !warp_wait(empty + slot, (uint32_t)(cc / kFSlots - 1) & 1u, flag, c.status))
                break;
            if (__shfl_sync(0xffffffffu, *(volatile int*)flag, 0)) break;
            const int tc = t_begin + cc * kFTok;
            const int nm = min(4, ((t_end + 63) >> 6) - (tc >> 6));
            const int n = min(kFTok, t_end - tc);
            // value params: an even count from a 16-byte aligned start, so the copy is a
            // whole number of 16-byte units; none staged when the row starts mid-unit (the
            // readers then load them from global memory)
            const bool va = (((size_t)b * cfg.T_max + tc) & 1) == 0;
            const int nv = !va ? 0 : !(n & 1) ? n : (tc + n + 1 <= cfg.T_max ? n + 1 : n - 1);
            uint32_t sv[kFSide];
            sv[2] = __shfl_sync(0xffffffffu, kcpl, 0);
            sv[3] = __shfl_sync(0xffffffffu, kcpl, nm);
            sv[10] = __shfl_sync(0xffffffffu, vcpl, 0);
            sv[11] = __shfl_sync(0xffffffffu, vcpl, nm);
#pragma unroll
            for (int k = 1; k < 4; ++k) {
                sv[3 + k] = __shfl_sync(0xffffffffu, kcpl, k);
                sv[11 + k] = __shfl_sync(0xffffffffu, vcpl, k);
            }
            sv[7] = (uint32_t)nm;
            sv[15] = (uint32_t)nv;
            sv[0] = sv[2] & ~3u;
            sv[1] = min(((sv[3] + 3u) & ~3u) - sv[0], (uint32_t)kFEnt);
            sv[8] = sv[10] & ~3u;
            sv[9] = min(((sv[11] + 3u) & ~3u) - sv[8], (uint32_t)kFEnt);
            if (sv[3] == sv[2]) sv[1] = 0;
            if (sv[11] == sv[10]) sv[9] = 0;
            if (lane == 0) {
#pragma unroll
                for (int k = 0; k < kFSide; ++k) side[slot * kFSide + k] = sv[k];
            }
            __syncwarp();  // the side record is complete before the copies are announced
            if (lane == 0) {
                fence_proxy_async();
                const int q0 = tc >> 2, q1 = (min(tc + kFTok, t_end) + 3) >> 2;
                const uint32_t kbytes = (uint32_t)(q1 - q0) * F::BW * 4;
                mbar_arrive_expect_tx(bcopy + slot,
                                      kbytes + 8u * (uint32_t)nv + 4u * (sv[1] + sv[9]));
                bulk_load(ring + (size_t)slot * L.stage, ksrc + (size_t)q0 * F::BW, kbytes,
                          bcopy + slot);
                if (nv) bulk_load(vps + slot * kFTok, vpar + tc, 8u * nv, bcopy + slot);
                if (sv[1]) bulk_load(kents + slot * kFEnt, kent + sv[0], 4u * sv[1], bcopy + slot);
                if (sv[9]) bulk_load(vents + slot * kFEnt, vent + sv[8], 4u * sv[9], bcopy + slot);
            }
            issued = cc + 1;
            if (cc + 1 < nst) load_cp(cc + 1);
        }
        if (lane == 0) flag[1] = issued;  // stages whose copies were issued
    } else if (warp == kFW + 1) {
        // ================= key warp: the stage's start phases and key-outlier corrections
        float2 thv[2], tlv[2];  // (cos, sin) tables of the next stage
        auto load_tr = [&](int st) {
            const int tc = t_begin + st * kFTok;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                thv[u] = thi[(tc / kTrigLo) * 64 + lane + 32 * u];
                tlv[u] = tlo[(tc % kTrigLo) * 64 + lane + 32 * u];
            }
        };
        load_tr(0);
        for (int cc = 0; cc < nst; ++cc) {
            const int ps = cc % kFSlots;
            if (cc >= kFSlots &&
                !warp_wait(empty + ps, (uint32_t)(cc / kFSlots - 1) & 1u, flag, c.status))
                break;
            {
                float4* bsw = base + ps * 64;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float2 cs = cmul(thv[u], tlv[u]);
                    bsw[lane + 32 * u] = make_float4(cs.x, cs.x, cs.y, cs.y);
                }
            }
            if (cc + 1 < nst) load_tr(cc + 1);
            if (!warp_wait(bcopy + ps, (uint32_t)(cc / kFSlots) & 1u, flag, c.status)) break;
            __syncwarp();
            const uint32_t* sd = side + ps * kFSide;
            const uint32_t kB = sd[0], kN = sd[1], E0 = sd[2], E1 = sd[3];
            const uint32_t bd1 = sd[4], bd2 = sd[5], bd3 = sd[6];
            const int nm = (int)sd[7];
            const int tc = t_begin + cc * kFTok;
            const float4* bs = base + ps * 64;
            const uint32_t* se = kents + ps * kFEnt;
            unsigned long long* kcs = kc + ps * kFTok;
            for (int j = lane; j < kFTok; j += 32) kcs[j] = 0ull;
            __syncwarp();
            // each entry's term in 2^-32 fixed point, added with an integer atomic: the sum
            // of a token's terms does not depend on their order.  A term is below 2^17 *
            // |q| in magnitude (|x - zhat| < 2^17), far inside the 2^31 range.
            constexpr int kKB = 8;
            for (uint32_t EW = E0; EW < E1; EW += 32 * kKB) {
                uint32_t wv[kKB];
                int kv[kKB];
                float2 rv[kKB];
#pragma unroll
                for (int u = 0; u < kKB; ++u) {
                    const uint32_t e = EW + 32 * u + lane;
                    wv[u] = e < E1 ? (e - kB < kN ? se[e - kB] : kent[e]) : 0u;
                    const int mc =
                        (nm > 1 && e >= bd1) + (nm > 2 && e >= bd2) + (nm > 3 && e >= bd3);
                    const int tau = mc * kChunk + (int)((wv[u] >> 7) & 63u);
                    kv[u] = (e < E1 && tc + tau < t_end) ? tau : -1;
                    rv[u] = tlo[(kv[u] >= 0 ? kv[u] : 0) * 64 + (int)(wv[u] & 63u)];
                }
#pragma unroll
                for (int u = 0; u < kKB; ++u) {
                    if (kv[u] < 0) continue;
                    const uint32_t w = wv[u];
                    const int ch = (int)(w & 127u), p = ch & 63;
                    const float d = h2f((uint16_t)(w >> 16)) - zks[ch];
                    const float4 bq = bs[p];
                    const float2 cs = cmul(make_float2(bq.x, bq.z), rv[u]);
                    // rotate-half: channel c < 64 meets (cos, sin) . (q_p, q_p+64), c >= 64 the other
                    const float sa = ch < 64 ? cs.x : -cs.y, sb = ch < 64 ? cs.y : cs.x;
                    const float v = d * fmaf(sa, qs[p], sb * qs[p + 64]);
                    atomicAdd(kcs + kv[u], (unsigned long long)__float2ll_rn(v * kKcScale));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(full + ps);
        }
    } else if (warp == kFW + 2) {
        // ================= value helper: zv per token, first value entry per 16-token slice
        float bd[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) bd[j] = cbV.bounds[j];
        for (int cc = 0; cc < nst; ++cc) {
            const int slot = cc % kFSlots;
            if (cc >= kFSlots &&
                !warp_wait(empty + slot, (uint32_t)(cc / kFSlots - 1) & 1u, flag, c.status))
                break;
            if (!warp_wait(bcopy + slot, (uint32_t)(cc / kFSlots) & 1u, flag, c.status)) break;
            const uint32_t* sd = side + slot * kFSide;
            const uint32_t vB = sd[8], vN = sd[9], E0 = sd[10], E1 = sd[11];
            const uint32_t bd1 = sd[12], bd2 = sd[13], bd3 = sd[14];
            const int nm = (int)sd[7], nv = (int)sd[15];
            const int tc = t_begin + cc * kFTok;
            const float2* vs_ = vps + slot * kFTok;
            float* zs = zv + slot * kFTok;
#pragma unroll
            for (int j = lane; j < kFTok; j += 32) {
                const int t = tc + j;
                float z = 0.0f;
                if (t < t_end) {
                    // the dense value stored at an outlier: the code of 0 in the token's normalization
                    const float2 vp = j < nv ? vs_[j] : vpar[t];
                    const float xn = normalize(0.0f, vp.x, vp.y);
                    int code = 0;
#pragma unroll
                    for (int jj = 0; jj < NB; ++jj) code += xn > bd[jj];
                    z = fmaf(vp.y, levv[code], vp.x);
                }
                zs[j] = z;
            }
            uint32_t* vs = vsl + slot * 32;
            const uint32_t* se = vents + slot * kFEnt;
            int qprev = -1;  // slice of the entry before the window
            for (uint32_t E = E0; E < E1; E += 32) {
                const uint32_t e = E + lane;
                const uint32_t w = e < E1 ? (e - vB < vN ? se[e - vB] : vent[e]) : 0u;
                const int mc = (nm > 1 && e >= bd1) + (nm > 2 && e >= bd2) + (nm > 3 && e >= bd3);
                const int tau = mc * kChunk + (int)((w >> 7) & 63u);
                const int q = (e < E1 && tc + tau < t_end) ? (tau >> 4) : 16;
                int qp = __shfl_up_sync(0xffffffffu, q, 1);
                if (lane == 0) qp = qprev;
                if (e < E1)
                    for (int r = qp + 1; r <= q; ++r) vs[r] = e;
                qprev = __shfl_sync(0xffffffffu, q, min(31, (int)(E1 - 1 - E)));
            }
            for (int r = qprev + 1 + lane; r <= 16; r += 32) vs[r] = E1;
            __syncwarp();
            if (lane == 0) mbar_arrive(full + slot);
        }
    } else {
        // ================= consumer warps
        const int x = i >> 2;
        const int uperm = (i >> 1) & 1;   // QK partial u of the lane holds quad u ^ uperm
        const bool owner = !(i & 1);
        const int qbase = 4 * warp + hh;  // quads qbase and qbase + 2 of the stage
        const int tl = 4 * (hh + 2 * uperm) + x;  // this lane's token among the warp's 16
        uint32_t lb[4], woff[2];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
            lb[sl] = kFAnchor + ((uint32_t)(sl ^ x) << JS) + ((uint32_t)i << 3);
        unsigned long long RQ[2][4], RQp[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int q = qbase + 2 * (u ^ uperm);
            woff[u] = (uint32_t)(q * F::BW + i * BITS) * 4;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 r = tlo[(4 * q) * 64 + i + 16 * k];
                RQ[u][k] = pk(r.x, r.y);
                RQp[u][k] = pk(-r.y, r.x);
            }
        }
        const uint32_t pvlane = (kFAnchor - (uint32_t)L.pv) | ((uint32_t)lane << 2);
        const uint32_t* vsrc = c.vcodes + li * nquads(cfg.T_max) * F::BW + i * BITS;
        auto load_v = [&](int st, uint32_t (&dst)[2][BITS]) {
            const int q0 = (t_begin + st * kFTok) >> 2;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int q = q0 + qbase + 2 * u;
                const bool ok = 4 * q < t_end;
#pragma unroll
                for (int d = 0; d < BITS; ++d) dst[u][d] = ok ? vsrc[(size_t)q * F::BW + d] : 0u;
            }
        };
        float m_w = -INFINITY, l_w = 0.0f, po_w = 0.0f;
        float* accw = accv + warp * kD;
        unsigned long long* wsw = wsm + warp * 16;
        float* wpw = wp + warp * 16;
        float* scw = scr + warp * 32;
        // one stage: vw holds its value codes; the next stage's go into vwn, first read one
        // stage later (the two buffers alternate), so their loads are in flight for a stage
        auto stage_fn = [&](int st, const uint32_t (&vw)[2][BITS], uint32_t (&vwn)[2][BITS]) -> bool {
            const int slot = st % kFSlots;
            const uint32_t par = (uint32_t)(st / kFSlots) & 1u;
            if (!warp_wait(bcopy + slot, par, flag, c.status)) return false;
            if (!warp_wait(full + slot, par, flag, c.status)) return false;
            if (st + 1 < nst) load_v(st + 1, vwn);
            const uint32_t* sd = side + slot * kFSide;
            const uint32_t vB = sd[8], vN = sd[9];
            const int nv = (int)sd[15];
            const uint32_t ea = vsl[slot * 32 + warp], eb = vsl[slot * 32 + warp + 1];
            const uint32_t* se = vents + slot * kFEnt;
            // ---- QK over quads qbase + 2 (u ^ uperm)
            const uint8_t* stage = ring + (size_t)slot * L.stage;
            uint32_t w[2][BITS];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int d = 0; d < BITS; ++d)
                    w[u][d] = *reinterpret_cast<const uint32_t*>(stage + woff[u] + 4 * d);
            unsigned long long Bc[4], Bs[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 bq = base[slot * 64 + i + 16 * k];
                Bc[k] = pk(bq.x, bq.y);
                Bs[k] = pk(bq.z, bq.w);
            }
            unsigned long long acc[4][2];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) acc[sl][0] = acc[sl][1] = 0ull;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const unsigned long long Pc = fma2(Bc[k], RQ[u][k], mul2(Bs[k], RQp[u][k]));
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
            // ---- logit, the warp's online softmax
            const int tst = 16 * warp + tl;  // token within the stage
            const int tabs = t_begin + st * kFTok + tst;
            const float lg =
                tabs < t_end ? v[0] + (float)((double)(long long)kc[slot * kFTok + tst] * kKcInv)
                             : -INFINITY;
            const float2 vp = tabs < t_end ? (tst < nv ? vps[slot * kFTok + tst] : vpar[tabs])
                                           : make_float2(0.0f, 0.0f);
            float mx = lg;
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (mx > m_w) {
                const float sc = m_w == -INFINITY ? 0.0f : __expf(m_w - mx);
                const unsigned long long sc2 = pk(sc, sc);
#pragma unroll
                for (int k = 0; k < 4; ++k) O[k] = mul2(O[k], sc2);
                l_w *= sc;
                po_w *= sc;
                for (int j = lane; j < kD; j += 32) accw[j] *= sc;
                m_w = mx;
            }
            const float p = lg > -INFINITY ? __expf(lg - m_w) : 0.0f;
            const float wv = p * vp.y;
            if (owner) {
                l_w += p;
                po_w = fmaf(p, vp.x, po_w);
                wsw[tl] = pk(wv, wv);
                wpw[tl] = p;
            }
            __syncwarp();
            // ---- PV over quads qbase + 2u
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    const unsigned long long ww = wsw[4 * (hh + 2 * u) + (sl ^ x)];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t fs = 0;
                        switch (4 * k + sl) {
#define KVQ_FS(N) case N: fs = field_to<BITS, N, 7>(vw[u]); break;
                            KVQ_FS(0) KVQ_FS(1) KVQ_FS(2) KVQ_FS(3) KVQ_FS(4) KVQ_FS(5)
                            KVQ_FS(6) KVQ_FS(7) KVQ_FS(8) KVQ_FS(9) KVQ_FS(10) KVQ_FS(11)
                            KVQ_FS(12) KVQ_FS(13) KVQ_FS(14) KVQ_FS(15)
#undef KVQ_FS
                        }
                        const uint32_t lv = lds32((fs & PVMASK) | pvlane);
                        const unsigned long long LL =
                            pk(__uint_as_float(__byte_perm(lv, 0u, 0x1010)),
                               __uint_as_float(__byte_perm(lv, 0u, 0x3232)));
                        O[k] = fma2(ww, LL, O[k]);
                    }
                }
            }
            // ---- value outliers of the warp's 16 tokens: p (x - zv), in entry order per channel
            for (uint32_t E = ea; E < eb; E += 32) {
                const uint32_t e = E + lane;
                const bool ok = e < eb;
                const uint32_t we = ok ? (e - vB < vN ? se[e - vB] : vent[e]) : 0u;
                const int tau = (int)((we >> 7) & 15u);  // token within the slice
                const int ch = (int)(we & 127u);
                float val = 0.0f;
                if (ok)
                    val = wpw[tau] * (h2f((uint16_t)(we >> 16)) - zv[slot * kFTok + 16 * warp + tau]);
                add_ordered(accw, scw, ch, val, ok, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the stage may be refilled
            return true;
        };
        uint32_t vA[2][BITS], vB[2][BITS];
        load_v(0, vA);
        for (int st = 0; st < nst; st += 2) {
            if (!stage_fn(st, vA, vB)) break;
            if (st + 1 < nst && !stage_fn(st + 1, vB, vA)) break;
        }
        // the warp's state: l and sum p off over the owner lanes
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            l_w += __shfl_xor_sync(0xffffffffu, l_w, o);
            po_w += __shfl_xor_sync(0xffffffffu, po_w, o);
        }
        __syncwarp();
        if (lane == 0) {
            scw[0] = m_w;
            scw[1] = l_w;
            scw[2] = po_w;
        }
    }
    __syncthreads();
    if (*(volatile int*)flag) {
        // after an abandoned wait, bulk copies of the last stages issued may still be in flight
        if (tid == 0) drain_chunks(bcopy, max(0, flag[1] - kFSlots), flag[1], kFSlots);
        return;
    }
    // ---- merge of the 16 warp states in warp order (the ring is idle now)
    float* red = reinterpret_cast<float*>(ring);  // [half-warp][channel]
    if (tid < kFCons) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const f2 o = upk(O[k]);
            red[(2 * warp + hh) * kD + i + 16 * k] = o.x;
            red[(2 * warp + hh) * kD + i + 16 * k + 64] = o.y;
        }
    }
    __syncthreads();
    if (tid < kD) {
        float M = -INFINITY;
        for (int w2 = 0; w2 < kFW; ++w2) M = fmaxf(M, scr[w2 * 32]);
        float o = 0.0f, Lt = 0.0f;
        if (M > -INFINITY)
            for (int w2 = 0; w2 < kFW; ++w2) {
                const float mw = scr[w2 * 32];
                if (mw == -INFINITY) continue;
                const float f = expf(mw - M);
                o = fmaf(f, red[(2 * w2) * kD + tid] + red[(2 * w2 + 1) * kD + tid] +
                                accv[w2 * kD + tid] + scr[w2 * 32 + 2], o);
                Lt = fmaf(f, scr[w2 * 32 + 1], Lt);
            }
        po_out[(row * S + s) * kD + tid] = o;
        if (tid == 0) st_out[row * S + s] = make_float2(M, Lt);
    }
}

}  // namespace

namespace kvq_host {

int fused_supported(const kvq_cfg* cfg) { return cfg->Hq == cfg->Hkv && cfg->bits <= 3; }

// Launch of the fused kernel: per-split (m, l, o) into st / po ([B][Hq][S], [B][Hq][S][D]).
int run_fused(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
              const kvq_codebook* cbV, const float* qr, const float2* thi, const float2* tlo,
              const float* zk, int max_len, int S, int Ls, float2* st, float* po,
              cudaStream_t stream) {
    auto kern = cfg->bits == 2 ? k_attn_quad<2> : k_attn_quad<3>;
    const int smem = fused_plan(cfg->bits).total;
    cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (ce) return record_cuda(ce);
    dim3 grid(S, cfg->B, cfg->Hq);
    kern<<<grid, kFThreads, smem, stream>>>(*cfg, *cache, *cbK, *cbV, qr, thi, tlo, zk, Ls, S,
                                            max_len, st, po);
    return record_cuda(cudaGetLastError());
}

}  // namespace kvq_host
