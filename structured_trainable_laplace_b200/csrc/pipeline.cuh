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

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Geometry of a tile of R rows x C channels walked by NT threads, thread (c, k)
// owning rows k*E .. k*E+E-1 of channel c.  Staged values live at
// k*SEG + e*C + c: one padding row per segment keeps the column reads of a warp
// on distinct banks.
template <int C_, int NT_, int E_>
struct TileGeo {
    static constexpr int C = C_;
    static constexpr int NT = NT_;
    static constexpr int E = E_;
    static constexpr int K = NT / C;
    static constexpr int R = K * E;
    static constexpr int SEG = (E + 1) * C;
    static constexpr int XS = K * SEG;  // floats of one staged vector tile
    static constexpr int SS = R + 8;    // anchors: [4 + r] holds row r, r in [-1, R]
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
// 16-byte copies when four channels stay contiguous and aligned, else 4-byte.
template <class G>
__device__ __forceinline__ void stage_rows(const float* __restrict__ v, int B, int ch0, int64_t n, int64_t lo,
                                           const uint32_t* p_buf, float* x_buf) {
    if (G::C % 4 == 0 && (B & 3) == 0) {
        constexpr int Q = G::C >= 4 ? G::C / 4 : 1;
        for (int i = threadIdx.x; i < G::R * Q; i += G::NT) {
            const int r = i / Q, c = (i % Q) * 4;
            float* dst = x_buf + G::xidx(r, c);
            if (lo + r < n && ch0 + c < B) {
                const uint32_t row = min(p_buf[r], (uint32_t)(n - 1));
                cp_async16(dst, v + (int64_t)row * B + ch0 + c);
            } else {
                *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
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

// Per-row decays of a staged tile: dl[r] = exp(a(r-1) - a(r)) for r in [0, R],
// stored as -1 when a(r) == a(r-1) (tie: decay 1, no break).  The right-to-left
// direction uses dl[r+1] for row r.
template <class G>
__device__ __forceinline__ void tile_decays(const float* s_buf, float* dl) {
    for (int r = threadIdx.x; r <= G::R; r += G::NT) {
        const float prev = s_buf[3 + r], cur = s_buf[4 + r];
        dl[r] = (cur > prev) ? expf(prev - cur) : -1.f;
    }
}

// One recurrence step from a stored decay (see lp_step).
__device__ __forceinline__ LP lp_step_d(LP s, float dv, float l, float t) {
    const float d = fabsf(dv);
    LP o;
    o.P = fmaf(d, s.P, l + t);
    o.L = (dv >= 0.f) ? fmaf(d, s.P, l) : (s.L + l);
    return o;
}

}  // namespace laplex
