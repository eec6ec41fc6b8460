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

__host__ __device__ inline int row_words(int bits) { return 4 * bits; }    // value row
__host__ __device__ inline int block_words(int bits) { return 8 * bits; }  // key block (2 tokens)
__host__ __device__ inline int nchunks(int T_max) { return (T_max + kChunk - 1) / kChunk; }
__host__ __device__ inline int npairs(int T_max) { return (T_max + 1) / 2; }

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

// ---- key block (token pair 2u, 2u+1; one kv head): channel c = j + 16m + 64s
// (j in [0,16), m in [0,4), s in {0,1}) has the 2*bits field
// code(2u, c) | code(2u+1, c) << bits at bit 16*bits*j + 2*bits*(2m + s).
__host__ __device__ inline int k_field_index(int c) {
    return 8 * (c & 15) + 2 * ((c & 63) >> 4) + (c >> 6);
}
// ---- value row (one token, one kv head): channel c < 64 and c + 64 share the field
// code(c) | code(c+64) << bits at bit 16*bits*j + 2*bits*m for c = j + 8m.
__host__ __device__ inline int v_field_index(int c) { return 8 * (c & 7) + ((c & 63) >> 3); }
// channel of field f (key block: f = 8j + 2m + s; value row: f = 8j + m, channel < 64)
__host__ __device__ inline int k_field_channel(int f) { return (f >> 3) + 16 * ((f >> 1) & 3) + 64 * (f & 1); }
__host__ __device__ inline int v_field_channel(int f) { return (f >> 3) + 8 * (f & 7); }

__device__ inline uint32_t get_field(const uint32_t* w, int f, int width) {
    const int off = f * width;
    const int wi = off >> 5, s = off & 31;
    uint32_t v = w[wi] >> s;
    if (s + width > 32) v |= w[wi + 1] << (32 - s);
    return v & ((1u << width) - 1u);
}

// Code of channel c of token (2u + parity) from a key block.
__device__ inline uint32_t k_code(const uint32_t* block, int bits, int c, int parity) {
    const uint32_t f = get_field(block, k_field_index(c), 2 * bits);
    return parity ? (f >> bits) : (f & ((1u << bits) - 1u));
}

// Code of channel c from a value row.
__device__ inline uint32_t v_code(const uint32_t* row, int bits, int c) {
    const uint32_t f = get_field(row, v_field_index(c), 2 * bits);
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
