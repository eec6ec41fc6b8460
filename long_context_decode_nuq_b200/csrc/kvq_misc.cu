// Dequantization of cache rows (test support) and the device fit of the per-layer
// NUQ datatype (technique (iii): per-layer non-uniform datatype from a weighted
// 1-D k-means over normalized samples).
#include "kvq_common.cuh"

using namespace kvq;

namespace {

// ---------------------------------------------------------------------------------
// Dense dequantization: fp16(off + half * L[code]); rows past len[b] are zero.
__global__ void k_dequant_dense(kvq_cfg cfg, kvq_cache c, kvq_codebook cbK, kvq_codebook cbV,
                                int t0, int nt, uint16_t* khat, uint16_t* vhat) {
    const int b = blockIdx.z, it = blockIdx.y;
    const int n = cfg.Hkv * kD;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n) return;
    const int t = t0 + it;
    const size_t o = ((size_t)b * nt + it) * n + j;
    if (t >= c.len[b]) {
        khat[o] = 0;
        vhat[o] = 0;
        return;
    }
    const int h = j / kD, ch = j % kD, BW = block_words(cfg.bits);
    const size_t blk = (((size_t)b * cfg.Hkv + h) * nquads(cfg.T_max) + t / 4) * BW;
    const float* kp = c.kparams + ((size_t)b * n + j) * 2;
    const float* vp = c.vparams + ((size_t)b * cfg.T_max + t) * 2;
    const float lk = cbK.levels[block_code(c.kcodes + blk, cfg.bits, ch, t & 3)];
    const float lv = cbV.levels[block_code(c.vcodes + blk, cfg.bits, ch, t & 3)];
    khat[o] = __half_as_ushort(__float2half_rn(__fadd_rn(kp[0], __fmul_rn(kp[1], lk))));
    vhat[o] = __half_as_ushort(__float2half_rn(__fadd_rn(vp[0], __fmul_rn(vp[1], lv))));
}

// Outlier replacement: entries of tokens in [t0, t0 + nt).
// Outlier replacement: entries of tokens in [t0, t0 + nt) of list (b, h) = blockIdx.y.
__global__ void k_dequant_outliers(kvq_cfg cfg, kvq_cache c, int t0, int nt, uint16_t* khat,
                                   uint16_t* vhat, int which) {
    const int li = blockIdx.y, b = li / cfg.Hkv, h = li % cfg.Hkv;
    const int n = cfg.Hkv * kD;
    const int nch1 = nchunks(cfg.T_max) + 1;
    const uint32_t* chunk = (which ? c.vchunk : c.kchunk) + (size_t)li * nch1;
    const uint32_t cnt = (which ? c.vcount : c.kcount)[li];
    const int cap = which ? cfg.out_cap_v : cfg.out_cap_k;
    const uint32_t* ent = (which ? c.vout : c.kout) + (size_t)li * cap;
    uint16_t* dst = which ? vhat : khat;
    const int len = c.len[b];
    const int tend = min(t0 + nt, len);
    if (tend <= t0) return;
    const int m0 = t0 / kChunk, m1 = (tend - 1) / kChunk;
    const uint32_t lo = chunk[m0];
    const uint32_t hi = min(chunk[m1 + 1], cnt);
    for (uint32_t e = lo + blockIdx.x * blockDim.x + threadIdx.x; e < hi;
         e += gridDim.x * blockDim.x) {
        // the chunk of entry e: the last m in [m0, m1] with chunk[m] <= e
        int a = m0, z = m1;
        while (a < z) {
            const int mid = (a + z + 1) >> 1;
            if (chunk[mid] <= e) a = mid; else z = mid - 1;
        }
        const uint32_t p = ent[e];
        const int t = a * kChunk + (int)((p >> 7) & 63u);
        const int ch = (int)(p & 127u);
        if (t < t0 || t >= tend) continue;
        dst[((size_t)b * nt + (t - t0)) * n + h * kD + ch] = (uint16_t)(p >> 16);
    }
}

// ---------------------------------------------------------------------------------
// Codebook fit (one block).
constexpr int kFitThreads = 1024;
constexpr int kFitMax = 16384;

__device__ inline uint32_t warp_incl(uint32_t v) {
    const int lane = threadIdx.x & 31;
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__device__ uint32_t blk_excl(uint32_t v, uint32_t* sm, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t incl = warp_incl(v);
    __syncthreads();
    if (lane == 31) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = lane < nw ? sm[lane] : 0u;
        sm[lane] = warp_incl(x);
    }
    __syncthreads();
    *total = sm[nw - 1];
    return (warp ? sm[warp - 1] : 0u) + incl - v;
}

__device__ inline double warp_sum_d(double v) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ inline float db16(uint32_t u) { return __uint_as_float((u << 16) | u); }

__device__ float round_db16(double x) {
    const uint32_t u0 = __float_as_uint((float)x) >> 16;
    const uint32_t cands[5] = {0x0000u, 0x8000u, (u0 - 1u) & 0xffffu, u0, (u0 + 1u) & 0xffffu};
    bool have = false;
    float best = 0.0f;
    double bd = 0.0;
    for (int q = 0; q < 5; ++q) {
        const uint32_t u = cands[q];
        if ((u & 0x7f80u) == 0x7f80u) continue;
        const float v = db16(u);
        const double d = fabs((double)v - x);
        if (!have || d < bd || (d == bd && v < best)) {
            have = true;
            best = v;
            bd = d;
        }
    }
    return best;
}

// Workspace: xs[kFitMax] double, wsum scratch; x/w live in global memory.
__global__ void __launch_bounds__(kFitThreads) k_fit(const uint16_t* samples, int n_vec, int L,
                                                     double f, const double* weights, int bits,
                                                     int max_iter, float* levels, float* bounds,
                                                     double* gx, double* gw) {
    extern __shared__ double sx[];            // [npad] sorted x
    uint16_t* sidx = (uint16_t*)(sx + kFitMax);  // [npad] original index
    __shared__ uint32_t hist[512];
    __shared__ uint32_t sel[4], lowb[4];
    __shared__ uint32_t sm[32];
    __shared__ uint32_t s_count;
    __shared__ double cent[16];
    __shared__ double red_sx[32][16], red_sw[32][16];
    __shared__ int s_changed;
    const int K = 1 << bits;
    const int tid = threadIdx.x;
    if (tid == 0) s_count = 0;
    __syncthreads();
    // 1. per vector: thresholds, normalization, drop outliers; append (index order)
    for (int vv = 0; vv < n_vec; ++vv) {
        const uint16_t* row = samples + (size_t)vv * L;
        for (int q = tid; q < 512; q += blockDim.x) hist[q] = 0;
        __syncthreads();
        for (int j = tid; j < L; j += blockDim.x) atomicAdd(&hist[okey(row[j]) >> 8], 1u);
        __syncthreads();
        const int kk = vector_k(f, L);
        if (tid < 32) {
            // warp-level rank search, 8 bins per lane
            for (int which = 0; which < 2; ++which) {
                const uint32_t r = which ? (uint32_t)(L - 1 - kk) : (uint32_t)kk;
                uint32_t loc[8], s = 0;
                for (int q = 0; q < 8; ++q) { loc[q] = hist[tid * 8 + q]; s += loc[q]; }
                const uint32_t incl = warp_incl(s);
                uint32_t cum = incl - s;
                for (int q = 0; q < 8; ++q) {
                    if (cum <= r && r < cum + loc[q]) { sel[2 * which] = tid * 8 + q; sel[2 * which + 1] = r - cum; }
                    cum += loc[q];
                }
            }
        }
        __syncthreads();
        for (int q = tid; q < 512; q += blockDim.x) hist[q] = 0;
        __syncthreads();
        for (int j = tid; j < L; j += blockDim.x) {
            const uint32_t key = okey(row[j]);
            if ((key >> 8) == sel[0]) atomicAdd(&hist[key & 255u], 1u);
            if ((key >> 8) == sel[2]) atomicAdd(&hist[256 + (key & 255u)], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            for (int which = 0; which < 2; ++which) {
                const uint32_t r = sel[2 * which + 1];
                const uint32_t* hh = hist + 256 * which;
                uint32_t loc[8], s = 0;
                for (int q = 0; q < 8; ++q) { loc[q] = hh[tid * 8 + q]; s += loc[q]; }
                const uint32_t incl = warp_incl(s);
                uint32_t cum = incl - s;
                for (int q = 0; q < 8; ++q) {
                    if (cum <= r && r < cum + loc[q]) lowb[2 * which] = tid * 8 + q;
                    cum += loc[q];
                }
            }
        }
        __syncthreads();
        const float lo = h2f((uint16_t)okey_inv((sel[0] << 8) | lowb[0]));
        const float hi = h2f((uint16_t)okey_inv((sel[2] << 8) | lowb[2]));
        const float off = __fmul_rn(__fadd_rn(lo, hi), 0.5f);
        const float half = __fmul_rn(__fsub_rn(hi, lo), 0.5f);
        // compaction in index order: per-thread contiguous ranges
        const int per = (L + blockDim.x - 1) / blockDim.x;
        const int j0 = tid * per;
        uint32_t cnt = 0;
        for (int j = j0; j < j0 + per && j < L; ++j) {
            const float x = h2f(row[j]);
            cnt += (x >= lo && x <= hi) ? 1u : 0u;
        }
        uint32_t total;
        uint32_t r = blk_excl(cnt, sm, &total);
        const uint32_t base = s_count;
        for (int j = j0; j < j0 + per && j < L; ++j) {
            const float x = h2f(row[j]);
            if (x >= lo && x <= hi) {
                gx[base + r] = (double)normalize(x, off, half);
                gw[base + r] = weights ? weights[(size_t)vv * L + j] : 1.0;
                ++r;
            }
        }
        __syncthreads();
        if (tid == 0) s_count = base + total;
        __syncthreads();
    }
    const int N = (int)s_count;
    int npad = 1;
    while (npad < N) npad <<= 1;
    // 2. sort (x, index) ascending: bitonic, padding with +inf
    for (int i = tid; i < npad; i += blockDim.x) {
        sx[i] = i < N ? gx[i] : INFINITY;
        sidx[i] = (uint16_t)(i < N ? i : 0);
    }
    __syncthreads();
    for (int size = 2; size <= npad; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < npad / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = ((lo & size) == 0);
                const double a = sx[lo], bb = sx[hi];
                const uint16_t ia = sidx[lo], ib = sidx[hi];
                const bool gt = (a > bb) || (a == bb && ia > ib);
                if (gt == up) {
                    sx[lo] = bb; sx[hi] = a;
                    sidx[lo] = ib; sidx[hi] = ia;
                }
            }
            __syncthreads();
        }
    }
    // sorted weights into gx's second half region (reuse gw as sorted copy in place)
    for (int i = tid; i < N; i += blockDim.x) gx[i] = gw[sidx[i]];
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) gw[i] = gx[i];
    __syncthreads();
    // 3. weighted quantile init (sequential cumulative sum, one thread)
    if (tid == 0 && N == 0) {
        for (int j = 0; j < K; ++j) cent[j] = 0.0;
    } else if (tid == 0) {
        double W = 0.0;
        for (int i = 0; i < N; ++i) W += gw[i];
        for (int j = 0; j < K; ++j) {
            const double target = ((double)j + 0.5) / (double)K * W;
            double cw = 0.0;
            int idx = N - 1;
            for (int i = 0; i < N; ++i) {
                cw += gw[i];
                if (cw >= target) { idx = i; break; }
            }
            cent[j] = sx[idx];
        }
    }
    __syncthreads();
    // 4. Lloyd iterations; assignment kept in the top bits of gx (as a byte array)
    uint8_t* assign = (uint8_t*)gx;
    const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    for (int it = 0; it < max_iter; ++it) {
        if (tid == 0) s_changed = 0;
        __syncthreads();
        double ls[16], lw[16];
        for (int j = 0; j < 16; ++j) { ls[j] = 0.0; lw[j] = 0.0; }
        int changed = 0;
        for (int i = tid; i < N; i += blockDim.x) {
            const double x = sx[i];
            int a = 0;
            double bd = fabs(x - cent[0]);
            for (int j = 1; j < K; ++j) {
                const double d = fabs(x - cent[j]);
                if (d < bd) { bd = d; a = j; }
            }
            if (it == 0 || assign[i] != (uint8_t)a) changed = 1;
            assign[i] = (uint8_t)a;
            const double w = gw[i];
            for (int j = 0; j < 16; ++j) {
                if (j == a) { ls[j] += w * x; lw[j] += w; }
            }
        }
        if (changed) s_changed = 1;
        for (int j = 0; j < K; ++j) {
            const double a = warp_sum_d(ls[j]);
            const double bw = warp_sum_d(lw[j]);
            if (lane == 0) { red_sx[warp][j] = a; red_sw[warp][j] = bw; }
        }
        __syncthreads();
        if (it > 0 && !s_changed) break;
        if (tid < K) {
            double a = 0.0, bw = 0.0;
            for (int w = 0; w < nw; ++w) { a += red_sx[w][tid]; bw += red_sw[w][tid]; }
            if (bw > 0.0) cent[tid] = a / bw;
        }
        __syncthreads();
    }
    // 5. sort centroids, round, bounds
    if (tid == 0) {
        for (int a = 1; a < K; ++a) {
            const double key = cent[a];
            int z = a - 1;
            while (z >= 0 && cent[z] > key) { cent[z + 1] = cent[z]; --z; }
            cent[z + 1] = key;
        }
        float lv[16];
        for (int j = 0; j < K; ++j) { lv[j] = round_db16(cent[j]); levels[j] = lv[j]; }
        for (int j = 0; j + 1 < K; ++j)
            bounds[j] = (float)(((double)lv[j] + (double)lv[j + 1]) * 0.5);
    }
}

}  // namespace

using namespace kvq_host;

extern "C" int kvq_dequantize(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                              const kvq_codebook* cbV, int32_t t0, int32_t nt, uint16_t* khat,
                              uint16_t* vhat, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if ((e = check_cache(cfg, cache))) return e;
    if ((e = check_codebook(cbK)) || (e = check_codebook(cbV))) return e;
    if (!khat || !vhat) return KVQ_ERR_NULL;
    if (t0 < 0 || nt < 0 || (long long)t0 + nt > cfg->T_max) return KVQ_ERR_RANGE;
    if (nt == 0) return KVQ_OK;
    if (nt > 65535) return KVQ_ERR_RANGE;
    cudaStream_t st = (cudaStream_t)stream;
    const int n = cfg->Hkv * kD;
    dim3 g((n + 127) / 128, nt, cfg->B);
    k_dequant_dense<<<g, 128, 0, st>>>(*cfg, *cache, *cbK, *cbV, t0, nt, khat, vhat);
    dim3 go(16, cfg->B * cfg->Hkv);
    k_dequant_outliers<<<go, 256, 0, st>>>(*cfg, *cache, t0, nt, khat, vhat, 0);
    k_dequant_outliers<<<go, 256, 0, st>>>(*cfg, *cache, t0, nt, khat, vhat, 1);
    return record_cuda(cudaGetLastError());
}

extern "C" int kvq_fit_workspace(int32_t n_vec, int32_t vec_len, size_t* bytes) {
    if (!bytes) return KVQ_ERR_NULL;
    if (n_vec < 1 || vec_len < 1 || (long long)n_vec * vec_len > kFitMax) return KVQ_ERR_SHAPE;
    *bytes = 2 * (size_t)kFitMax * sizeof(double);
    return KVQ_OK;
}

extern "C" int kvq_fit_codebook(const uint16_t* samples, int32_t n_vec, int32_t vec_len, double f,
                                const double* weights, int32_t bits, int32_t max_iter,
                                float* levels, float* bounds, void* workspace,
                                size_t workspace_bytes, void* stream) {
    if (!samples || !levels || !bounds || !workspace) return KVQ_ERR_NULL;
    if (bits < 2 || bits > 4) return KVQ_ERR_UNSUPPORTED;
    if (n_vec < 1 || vec_len < 1 || (long long)n_vec * vec_len > kFitMax) return KVQ_ERR_SHAPE;
    if (!(f >= 0.0 && f <= 1.0) || max_iter < 1) return KVQ_ERR_SHAPE;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    if (workspace_bytes < 2 * (size_t)kFitMax * sizeof(double)) return KVQ_ERR_WORKSPACE;
    const size_t smem = (size_t)kFitMax * (sizeof(double) + sizeof(uint16_t));
    cudaError_t ce = cudaFuncSetAttribute(k_fit, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
    if (ce) return record_cuda(ce);
    double* gx = (double*)workspace;
    double* gw = gx + kFitMax;
    k_fit<<<1, kFitThreads, smem, (cudaStream_t)stream>>>(samples, n_vec, vec_len, f, weights,
                                                         bits, max_iter, levels, bounds, gx, gw);
    return record_cuda(cudaGetLastError());
}
