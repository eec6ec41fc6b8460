// Shared device/host helpers of libkvq (layouts, order keys, status bits).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int kD = 128;          // head dimension (the only one supported)
constexpr int kPairs = kD / 2;   // rotate-half pairs (p, p + 64)
constexpr int kChunk = KVQ_CHUNK;

__host__ __device__ inline int row_words(int bits) { return 4 * bits; }
__host__ __device__ inline int nchunks(int T_max) { return (T_max + kChunk - 1) / kChunk; }

// Outliers kept per side of an N-value vector: floor(f*N/2 + 1/2), capped at (N-1)/2.
__host__ __device__ inline int vector_k(double f, int N) {
    if (N <= 0) return 0;
    double x = f * (double)N * 0.5 + 0.5;
    int k = (int)floor(x);
    int cap = (N - 1) / 2;
    return k < cap ? k : cap;
}

// fp16 bit pattern <-> 16-bit key whose unsigned order is IEEE total order.
__host__ __device__ inline uint32_t okey(uint32_t bits) {
    return (bits & 0x8000u) ? (~bits & 0xFFFFu) : (bits | 0x8000u);
}
__host__ __device__ inline uint32_t okey_inv(uint32_t key) {
    return (key & 0x8000u) ? (key ^ 0x8000u) : (~key & 0xFFFFu);
}

__device__ inline float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Affine normalization (binary32, round to nearest, no contraction).
__device__ inline float normalize(float x, float off, float half) {
    if (half == 0.0f) return 0.0f;
    return __fdiv_rn(__fsub_rn(x, off), half);
}

// Number of decision bounds strictly below xn.
__device__ inline uint32_t encode(float xn, const float* bounds, int nb) {
    uint32_t c = 0;
    for (int j = 0; j < nb; ++j) c += (xn > bounds[j]) ? 1u : 0u;
    return c;
}

// ---- key row layout: pair p = (p, p+64) is a 2*bits field in pair-group p/16 ----
__device__ inline uint32_t k_pair_field(const uint32_t* row, int bits, int p) {
    const int g = p >> 4, j = p & 15;
    const int o = 2 * bits * j;
    const int w = o >> 5, s = o & 31;
    const uint32_t* gw = row + g * bits;
    uint32_t v = gw[w] >> s;
    if (s + 2 * bits > 32) v |= gw[w + 1] << (32 - s);
    return v & ((1u << (2 * bits)) - 1u);
}

// ---- value row layout: channel c = 32g + k in nibble format ----
// Bit position (word within the group, bit) of bit m of code k.
__host__ __device__ inline void v_bitpos(int bits, int k, int m, int* word, int* bit) {
    if (bits == 3) {
        if (k < 24) { *word = k >> 3; *bit = 4 * (k & 7) + m; }
        else { *word = m; *bit = 4 * (k - 24) + 3; }
    } else if (bits == 2) {
        const int w = k >> 4, kk = k & 15;
        *word = w; *bit = 4 * (kk & 7) + 2 * (kk >> 3) + m;
    } else {
        *word = k >> 3; *bit = 4 * (k & 7) + m;
    }
}

__device__ inline uint32_t v_code(const uint32_t* row, int bits, int c) {
    const int g = c >> 5, k = c & 31;
    const uint32_t* gw = row + g * bits;
    if (bits == 3) {
        if (k < 24) return (gw[k >> 3] >> (4 * (k & 7))) & 7u;
        const int sh = 4 * (k - 24) + 3;
        return ((gw[0] >> sh) & 1u) | (((gw[1] >> sh) & 1u) << 1) | (((gw[2] >> sh) & 1u) << 2);
    }
    if (bits == 2) {
        const int kk = k & 15;
        return (gw[k >> 4] >> (4 * (kk & 7) + 2 * (kk >> 3))) & 3u;
    }
    return (gw[k >> 3] >> (4 * (k & 7))) & 15u;
}

__device__ inline uint32_t k_code(const uint32_t* row, int bits, int c) {
    const uint32_t f = k_pair_field(row, bits, c & 63);
    return (c < 64) ? (f & ((1u << bits) - 1u)) : (f >> bits);
}

__device__ inline void set_status(int32_t* status, int bit) { atomicOr(status, bit); }

// RoPE frequency theta_i = base^(-2i/D) in binary64.
__device__ inline double rope_freq(double base, int i) {
    return pow(base, -2.0 * (double)i / (double)kD);
}

// (cos, sin) of t * theta in binary64 with the angle reduced modulo 2*pi first.
__device__ inline void rope_cs64(double t, double theta, double* c, double* s) {
    const double two_pi = 6.283185307179586476925286766559;
    double a = t * theta;
    a = a - two_pi * floor(a / two_pi);
    sincos(a, s, c);
}

}  // namespace kvq

// Host-side helpers shared by the entry points.
namespace kvq_host {
int record_cuda(cudaError_t e);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int check_cfg(const kvq_cfg* cfg);
int check_cache(const kvq_cfg* cfg, const kvq_cache* c);
int check_codebook(const kvq_codebook* cb);
size_t align_up(size_t x);
}  // namespace kvq_host
