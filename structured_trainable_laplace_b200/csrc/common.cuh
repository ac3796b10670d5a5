// Shared device helpers for the LAPLEX kernels (sm_100a).
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda_runtime.h>

namespace laplex {

constexpr int32_t kStatusNonFinite = 4;
constexpr int32_t kStatusTimeout = 5;

// Upper bound on the polls of one lookback wait.  Each poll is an L2 round trip
// plus a short sleep, so the bound is well under a second; past it the waiting
// tile records kStatusTimeout, treats the missing value as zero and finishes.
constexpr uint32_t kSpinLimit = 1u << 20;

// Sentinel anchors for "before the first row" / "after the last row" and for
// padding rows of a partial tile.  Finite, so that differences of two sentinels
// are 0 (never inf - inf).
constexpr float kLowAnchor = -FLT_MAX;
constexpr float kHighAnchor = FLT_MAX;

__device__ __forceinline__ void raise_status(int32_t* st, int32_t code) {
    if (st != nullptr) atomicCAS(st, 0, code);
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Relaxed (unordered) 64-bit load at gpu scope: several can be in flight at once.
// For words that carry their own status bits no further ordering is needed.
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Relaxed 64-bit store at gpu scope, for words that carry their own status bits.
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Order-preserving map from fp32 to uint32 (ascending floats -> ascending keys);
// -0.0 maps to the key of +0.0.
__device__ __forceinline__ uint32_t float_to_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ bool is_nonfinite(float f) {
    return (__float_as_uint(f) & 0x7f800000u) == 0x7f800000u;
}

}  // namespace laplex
