// Device helpers shared by the decode kernels: mbarriers and bulk copies (PTX), packed f32x2
// arithmetic, code-field extraction and the per-call RoPE tables.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kMaxG = 16;                          // query heads per kv head
constexpr uint32_t kWaitLimit = 1u << 24;          // mbarrier polls before giving up
constexpr int kTrigLo = 256;                       // trig tables: t = 256 * hi + lo

// ---------------------------------------------------------------------------------
// mbarrier + bulk copy (PTX).
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Adds `bytes` to the transaction count the current phase waits for, without an arrival.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
// Bounded wait for the phase with the given parity; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t it = 0; it < kWaitLimit; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
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
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
template <int BITS>
struct Fmt {
    static constexpr int FW = 2 * BITS;  // field width (codes of c and c + 64)
    static constexpr int NT = 1 << FW;   // entries of a pair table
    static constexpr int BW = 16 * BITS; // words of a code block
};

// A word holding slot F's field (bit FW*F of the lane group's string w[0 .. BITS)) at bit P
// (the other bits are junk, masked by the caller).
template <int BITS, int F, int P>
__device__ __forceinline__ uint32_t field_to(const uint32_t (&w)[BITS]) {
    constexpr int FW = 2 * BITS;
    constexpr int O = FW * F;
    constexpr int wi = O >> 5, sh = O & 31;
    if constexpr (sh + FW <= 32) {
        if constexpr (sh >= P)
            return w[wi] >> (sh - P);
        else
            return w[wi] << (P - sh);
    } else {
        static_assert(sh >= P, "a field that crosses words starts above bit P");
        return __funnelshift_r(w[wi], w[wi + 1], sh - P);
    }
}

// Shared-memory load at a 32-bit shared-window address plus an immediate byte offset.
template <int IMM>
__device__ __forceinline__ unsigned long long lds64(uint32_t addr) {
    unsigned long long d;
    asm("ld.shared.b64 %0, [%1+%2];" : "=l"(d) : "r"(addr), "n"(IMM));
    return d;
}

// 32-bit shared-memory load at a shared-window address.
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t d;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(d) : "r"(addr));
    return d;
}

// Shared-memory table load at a byte offset.
__device__ __forceinline__ unsigned long long tld(const uint8_t* tab, uint32_t off) {
    return *reinterpret_cast<const unsigned long long*>(tab + off);
}


__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// After an abandoned wait: let every copy still in flight land before the CTA exits.
__device__ inline void drain_chunks(uint64_t* bars, int from, int to, int nslots) {
    for (int cc = from; cc < to; ++cc) mbar_wait(bars + cc % nslots, (cc / nslots) & 1);
}

// (cos, sin) of t * theta_p from the per-call tables: hi[t / 256] rotated by lo[t % 256].
__device__ __forceinline__ float2 trig_at(const float2* thi, const float2* tlo, int t, int p) {
    return cmul(thi[(t / kTrigLo) * 64 + p], tlo[(t % kTrigLo) * 64 + p]);
}


}  // namespace kvq
