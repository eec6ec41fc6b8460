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

__host__ __device__ inline int block_words(int bits) { return 16 * bits; }  // code block (4 tokens)
__host__ __device__ inline int nchunks(int T_max) { return (T_max + kChunk - 1) / kChunk; }
__host__ __device__ inline int nquads(int T_max) { return (T_max + 3) / 4; }

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

// ---- code block (token quad 4u .. 4u+3; one kv head; keys and values alike): lane group
// i in [0,16) owns words [bits*i, bits*i + bits) and the rotate-half pairs (c, c + 64) for
// c = i + 16k (k in [0,4)); the 2*bits field code(4u+j, c) | code(4u+j, c+64) << bits of
// token j sits in slot s = j ^ (i >> 2), at bit 2*bits*(4k + s) of the group's bit string.
__host__ __device__ inline int field_offset(int bits, int c, int j) {
    const int i = c & 15;
    return 32 * bits * i + 2 * bits * (4 * (c >> 4) + (j ^ (i >> 2)));
}

__device__ inline uint32_t get_bits(const uint32_t* w, int off, int width) {
    const int wi = off >> 5, s = off & 31;
    uint32_t v = w[wi] >> s;
    if (s + width > 32) v |= w[wi + 1] << (32 - s);
    return v & ((1u << width) - 1u);
}

// Code of channel c (0 .. 127) of token j of the quad.
__device__ inline uint32_t block_code(const uint32_t* block, int bits, int c, int j) {
    const uint32_t f = get_bits(block, field_offset(bits, c & 63, j), 2 * bits);
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
// Fused single-pass decode (kvq_fused.cu): shapes it covers, and its launch.
int fused_supported(const kvq_cfg* cfg);
int run_fused(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
              const kvq_codebook* cbV, const float* qr, const float2* thi, const float2* tlo,
              const float* zk, int max_len, int S, int Ls, float2* st, float* po,
              cudaStream_t stream);
}  // namespace kvq_host
