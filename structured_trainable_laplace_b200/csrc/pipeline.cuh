// Asynchronous staging of sorted tiles into shared memory (cp.async), used by
// the range-walking scan kernels: the sorted anchors and the permutation of a
// tile, then the rows it gathers through the permutation.
#pragma once

#include "scan_tile.cuh"

namespace laplex {

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Wait until at most N of this thread's most recent copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Geometry of a tile of R rows x C channels walked by NT threads, K = NT / C
// segments of E rows per channel.  Staged values live at k*SEG + e*C + c with
// SEG = E*C + PAD: the padding spreads the column reads of a warp over distinct
// banks (PAD = C when a warp spans segments of all channels, PAD = channels per
// warp when each warp owns whole channels).
template <int C_, int NT_, int E_, int PAD_ = C_>
struct TileGeo {
    static constexpr int C = C_;
    static constexpr int NT = NT_;
    static constexpr int E = E_;
    static constexpr int K = NT / C;
    static constexpr int R = K * E;
    static constexpr int SEG = E * C + PAD_;
    static constexpr int XS = K * SEG;  // floats of one staged vector tile
    static constexpr int SS = R + 8;    // anchors: [4 + r] holds row r, r in [-1, R]
    // widest copy (floats) that keeps every staged row chunk aligned
    static constexpr int VW = (SEG % 4 == 0 && C % 4 == 0) ? 4 : ((SEG % 2 == 0 && C % 2 == 0) ? 2 : 1);
    __device__ static __forceinline__ int xidx(int r, int c) { return (r / E) * SEG + (r % E) * C + c; }
};

// Start copying the anchors s[lo-1 .. lo+R] and the permutation perm[lo .. lo+R-1]
// of one tile; rows outside [0, n) get sentinels (plain stores).
template <class G>
__device__ __forceinline__ void stage_meta(const float* __restrict__ s, const uint32_t* __restrict__ perm, int64_t n,
                                           int64_t lo, float* s_buf, uint32_t* p_buf) {
    for (int r = threadIdx.x; r < G::R; r += G::NT) {
        const int64_t g = lo + r;
        if (g < n) {
            cp_async4(s_buf + 4 + r, s + g);
            cp_async4(p_buf + r, perm + g);
        } else {
            s_buf[4 + r] = kHighAnchor;
            p_buf[r] = 0u;
        }
    }
    if (threadIdx.x == 0) {
        if (lo > 0)
            cp_async4(s_buf + 3, s + lo - 1);
        else
            s_buf[3] = kLowAnchor;
    }
    if (threadIdx.x == G::NT - 1) {
        if (lo + G::R < n)
            cp_async4(s_buf + 4 + G::R, s + lo + G::R);
        else
            s_buf[4 + G::R] = kHighAnchor;
    }
}

// Start gathering channels [ch0, ch0 + C) of the rows perm[lo + r] of v [n][B].
// Copies of G::VW floats (16 or 8 bytes) when the rows of v keep that alignment,
// else 4 bytes.
template <class G>
__device__ __forceinline__ void stage_rows(const float* __restrict__ v, int B, int ch0, int64_t n, int64_t lo,
                                           const uint32_t* p_buf, float* x_buf) {
    if (G::VW > 1 && (B % G::VW) == 0) {
        constexpr int W = G::VW > 1 ? G::VW : 2;
        constexpr int Q = G::C >= W ? G::C / W : 1;
        for (int i = threadIdx.x; i < G::R * Q; i += G::NT) {
            const int r = i / Q, c = (i % Q) * W;
            float* dst = x_buf + G::xidx(r, c);
            if (lo + r < n && ch0 + c < B) {
                const uint32_t row = min(p_buf[r], (uint32_t)(n - 1));
                if (W == 4)
                    cp_async16(dst, v + (int64_t)row * B + ch0 + c);
                else
                    cp_async8(dst, v + (int64_t)row * B + ch0 + c);
            } else {
#pragma unroll
                for (int q = 0; q < W; ++q) dst[q] = 0.f;
            }
        }
    } else {
        for (int i = threadIdx.x; i < G::R * G::C; i += G::NT) {
            const int r = i / G::C, c = i % G::C;
            float* dst = x_buf + G::xidx(r, c);
            if (lo + r < n && ch0 + c < B) {
                const uint32_t row = min(p_buf[r], (uint32_t)(n - 1));
                cp_async4(dst, v + (int64_t)row * B + ch0 + c);
            } else {
                *dst = 0.f;
            }
        }
    }
}

// Encoded decay between two oriented anchors uA <= uB: exp(uA - uB) when uB > uA
// (a break), -1 when they are equal (a tie: decay 1, no break).
__device__ __forceinline__ float enc_decay(float uA, float uB) { return (uB > uA) ? expf(uA - uB) : -1.f; }

// One recurrence step from a stored decay (see lp_step).
__device__ __forceinline__ LP lp_step_d(LP s, float dv, float l, float t) {
    const float d = fabsf(dv);
    LP o;
    o.P = fmaf(d, s.P, l + t);
    o.L = (dv >= 0.f) ? fmaf(d, s.P, l) : (s.L + l);
    return o;
}

// A then B with the decay e = exp(u_A - u_B) and the break flag u_B > u_A given.
__device__ __forceinline__ LP combine_e(LP A, LP B, float e, bool brk) {
    LP o;
    o.P = fmaf(e, A.P, B.P);
    o.L = brk ? fmaf(e, A.P, B.L) : (A.L + B.L);
    return o;
}

// A then B from an encoded decay (see enc_decay).
__device__ __forceinline__ LP combine_v(LP A, LP B, float ev) { return combine_e(A, B, fabsf(ev), ev >= 0.f); }

__device__ __forceinline__ double2 combine_ed(double2 A, double2 B, double e, bool brk) {
    double2 o;  // x = L, y = P
    o.y = fma(e, A.y, B.y);
    o.x = brk ? fma(e, A.y, B.x) : (A.x + B.x);
    return o;
}

}  // namespace laplex
