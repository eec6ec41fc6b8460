// GPU side of the seeded synthetic input generator (see philox.py for the
// definition).  Every floating-point step is a single correctly rounded binary64
// operation issued through the _rn intrinsics, in the same order as the numpy
// side, so both produce identical fp16 bits.  No quantization or attention
// arithmetic lives here.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ inline void philox(uint32_t c[4], uint32_t k0, uint32_t k1) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
        const uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
}

__constant__ double kAtanh[12] = {
    0x1.0000000000000p+0, 0x1.5555555555555p-2, 0x1.999999999999ap-3, 0x1.2492492492492p-3,
    0x1.c71c71c71c71cp-4, 0x1.745d1745d1746p-4, 0x1.3b13b13b13b14p-4, 0x1.1111111111111p-4,
    0x1.e1e1e1e1e1e1ep-5, 0x1.af286bca1af28p-5, 0x1.8618618618618p-5, 0x1.642c8590b2164p-5};
__constant__ double kSin[12] = {
    0x1.0000000000000p+0, -0x1.5555555555555p-3, 0x1.1111111111111p-7, -0x1.a01a01a01a01ap-13,
    0x1.71de3a556c734p-19, -0x1.ae64567f544e4p-26, 0x1.6124613a86d09p-33, -0x1.ae7f3e733b81fp-41,
    0x1.952c77030ad4ap-49, -0x1.2f49b46814157p-57, 0x1.71b8ef6dcf572p-66, -0x1.761b41316381ap-75};
__constant__ double kCos[13] = {
    0x1.0000000000000p+0, -0x1.0000000000000p-1, 0x1.5555555555555p-5, -0x1.6c16c16c16c17p-10,
    0x1.a01a01a01a01ap-16, -0x1.27e4fb7789f5cp-22, 0x1.1eed8eff8d898p-29, -0x1.93974a8c07c9dp-37,
    0x1.ae7f3e733b81fp-45, -0x1.6827863b97d97p-53, 0x1.e542ba4020225p-62, -0x1.0ce396db7f853p-70,
    0x1.f2cf01972f578p-80};
constexpr double kLn2 = 0x1.62e42fefa39efp-1;
constexpr double kHalfPi = 0x1.921fb54442d18p+0;
constexpr double kSqrt1_2 = 0x1.6a09e667f3bcdp-1;
constexpr double kTwoM32 = 0x1p-32;

__device__ inline double horner(const double* coef, int n, double z) {
    double p = coef[n - 1];
    for (int i = n - 2; i >= 0; --i) {
        p = __dmul_rn(p, z);
        p = __dadd_rn(p, coef[i]);
    }
    return p;
}

__device__ inline double ln_unit(double u) {
    int e;
    double m = frexp(u, &e);
    if (m < kSqrt1_2) {
        m = __dmul_rn(m, 2.0);
        e -= 1;
    }
    const double s = __ddiv_rn(__dsub_rn(m, 1.0), __dadd_rn(m, 1.0));
    const double z = __dmul_rn(s, s);
    const double t = __dmul_rn(s, horner(kAtanh, 12, z));
    return __dadd_rn(__dmul_rn((double)e, kLn2), __dadd_rn(t, t));
}

__device__ inline void cos_sin_turn(double a, double* cv, double* sv) {
    const double x = __dmul_rn(a, 4.0);
    const double q = floor(x);
    const double r = __dsub_rn(x, q);
    const double phi = __dmul_rn(r, kHalfPi);
    const double z = __dmul_rn(phi, phi);
    const double s = __dmul_rn(phi, horner(kSin, 12, z));
    const double c = horner(kCos, 13, z);
    const int qi = (int)q;
    if (qi == 0) { *cv = c; *sv = s; }
    else if (qi == 1) { *cv = -s; *sv = c; }
    else if (qi == 2) { *cv = -c; *sv = -s; }
    else { *cv = s; *sv = -c; }
}

__device__ inline void box_muller(uint32_t w0, uint32_t w1, double* z0, double* z1) {
    const double u = __dmul_rn(__dadd_rn((double)w0, 0.5), kTwoM32);
    const double a = __dmul_rn((double)w1, kTwoM32);
    const double rho = __dsqrt_rn(__dmul_rn(-2.0, ln_unit(u)));
    double c, s;
    cos_sin_turn(a, &c, &s);
    *z0 = __dmul_rn(rho, c);
    *z1 = __dmul_rn(rho, s);
}

__device__ inline void four_normals(uint64_t ctr, uint32_t stream, uint32_t tag, uint32_t seed,
                                    uint32_t layer, double z[4]) {
    uint32_t c[4] = {(uint32_t)ctr, (uint32_t)(ctr >> 32), stream, tag};
    philox(c, seed, layer);
    box_muller(c[0], c[1], &z[0], &z[1]);
    box_muller(c[2], c[3], &z[2], &z[3]);
}

__device__ inline uint16_t to_fp16(double z) {
    return __half_as_ushort(__float2half_rn(__double2float_rn(z)));
}

struct FillArgs {
    uint32_t seed, layer, stream;
    int B, T_gen, Hkv, D;
    int t0, nt;                 // token range written
    const double* scale;        // [Hkv*D] or NULL (1.0)
    const uint8_t* tmask;       // [Hkv*D] or NULL: Student-t(3) channels
    uint32_t spike_thresh;      // 0: no spikes
    double spike_scale;
};

// One thread per group of four consecutive elements of the logical tensor
// [B][T_gen][Hkv][D] restricted to tokens [t0, t0 + nt); out is [B][nt][Hkv][D].
__global__ void k_fill(FillArgs a, uint16_t* __restrict__ out) {
    const uint64_t row = (uint64_t)a.Hkv * a.D;
    const uint64_t per_b = (uint64_t)a.nt * row;
    const uint64_t total = (uint64_t)a.B * per_b;
    for (uint64_t g4 = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; g4 * 4 < total;
         g4 += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t o0 = g4 * 4;
        const uint64_t b = o0 / per_b;
        const uint64_t rem = o0 - b * per_b;
        const uint64_t tt = rem / row;
        const uint64_t hc = rem - tt * row;      // multiple of 4 (D % 4 == 0)
        const uint64_t e0 = (b * (uint64_t)a.T_gen + (uint64_t)(a.t0 + tt)) * row + hc;
        double z[4];
        four_normals(e0 >> 2, a.stream, 0u, a.seed, a.layer, z);
        uint32_t sw[4] = {0, 0, 0, 0};
        if (a.spike_thresh) {
            sw[0] = (uint32_t)(e0 >> 2);
            sw[1] = (uint32_t)((e0 >> 2) >> 32);
            sw[2] = a.stream;
            sw[3] = 2u;
            philox(sw, a.seed, a.layer);
        }
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const uint64_t ch = hc + l;
            double v = z[l];
            if (a.tmask && a.tmask[ch]) {
                double t[4];
                four_normals(e0 + l, a.stream, 1u, a.seed, a.layer, t);
                double ss = __dmul_rn(t[1], t[1]);
                ss = __dadd_rn(ss, __dmul_rn(t[2], t[2]));
                ss = __dadd_rn(ss, __dmul_rn(t[3], t[3]));
                v = __ddiv_rn(t[0], __dsqrt_rn(__ddiv_rn(ss, 3.0)));
            }
            if (a.scale) v = __dmul_rn(v, a.scale[ch]);
            if (a.spike_thresh && sw[l] < a.spike_thresh) v = __dmul_rn(v, a.spike_scale);
            out[o0 + l] = to_fp16(v);
        }
    }
}

// Plain normals (queries): out[i] = fp16(N(0,1) at element e_base + i).
__global__ void k_fill_normal(uint32_t seed, uint32_t layer, uint32_t stream, uint64_t e_base,
                              uint64_t n, uint16_t* __restrict__ out) {
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t e = e_base + i;
        double z[4];
        four_normals(e >> 2, stream, 0u, seed, layer, z);
        out[i] = to_fp16(z[e & 3]);
    }
}

}  // namespace

extern "C" {

// Fill out (device, fp16 [B][nt][Hkv][D]) with tokens [t0, t0+nt) of the K or V tensor.
int kvqsynth_fill_kv(uint32_t seed, uint32_t layer, uint32_t stream, int B, int T_gen, int Hkv,
                     int D, int t0, int nt, const double* scale, const uint8_t* tmask,
                     uint32_t spike_thresh, double spike_scale, uint16_t* out, void* cuda_stream) {
    if (!out || B < 1 || Hkv < 1 || D % 4 != 0 || nt < 0 || t0 < 0 || t0 + nt > T_gen) return -1;
    if (nt == 0) return 0;
    FillArgs a{seed, layer, stream, B, T_gen, Hkv, D, t0, nt, scale, tmask, spike_thresh,
               spike_scale};
    const uint64_t groups = (uint64_t)B * nt * Hkv * D / 4;
    uint64_t blocks = (groups + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    k_fill<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(a, out);
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

int kvqsynth_fill_normal(uint32_t seed, uint32_t layer, uint32_t stream, uint64_t e_base,
                         uint64_t n, uint16_t* out, void* cuda_stream) {
    if (!out) return -1;
    if (n == 0) return 0;
    uint64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    k_fill_normal<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(seed, layer, stream,
                                                                            e_base, n, out);
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

}  // extern "C"
