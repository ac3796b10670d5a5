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

// L2 eviction priorities (createpolicy).  Data streamed through once is marked
// evict-first, so that lines written piecewise elsewhere (scattered 4-byte
// gradient rows) stay in L2 until they are complete instead of being written back
// half-filled.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, uint64_t pol) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;" ::"r"(s), "l"(gmem), "l"(pol) : "memory");
}

__device__ __forceinline__ void cp_async8(void* smem, const void* gmem, uint64_t pol) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 8, %2;" ::"r"(s), "l"(gmem), "l"(pol) : "memory");
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint64_t pol) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_hint(float* p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_hint(float2* p, float2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_hint(float4* p, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
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
                                           int64_t lo, float* s_buf, uint32_t* p_buf, uint64_t pol) {
    for (int r = threadIdx.x; r < G::R; r += G::NT) {
        const int64_t g = lo + r;
        if (g < n) {
            cp_async4(s_buf + 4 + r, s + g, pol);
            cp_async4(p_buf + r, perm + g, pol);
        } else {
            s_buf[4 + r] = kHighAnchor;
            p_buf[r] = 0u;
        }
    }
    if (threadIdx.x == 0) {
        if (lo > 0)
            cp_async4(s_buf + 3, s + lo - 1, pol);
        else
            s_buf[3] = kLowAnchor;
    }
    if (threadIdx.x == G::NT - 1) {
        if (lo + G::R < n)
            cp_async4(s_buf + 4 + G::R, s + lo + G::R, pol);
        else
            s_buf[4 + G::R] = kHighAnchor;
    }
}

// Per-thread walk over the (row, chunk) copies of one tile: W floats per copy, Q
// copies per row, thread tid handles chunk tid % Q of rows tid / Q + it * RPI.
template <class G, int W>
struct RowWalk {
    static constexpr int Q = G::C >= W ? G::C / W : 1;
    static_assert(G::NT % Q == 0, "threads must cover whole rows");
    static constexpr int RPI = G::NT / Q;  // rows per iteration
    static constexpr int ITER = (G::R + RPI - 1) / RPI;
    int r0, c;
    __device__ __forceinline__ RowWalk() : r0(threadIdx.x / Q), c((threadIdx.x % Q) * W) {}
    __device__ __forceinline__ int row(int it) const { return r0 + it * RPI; }
    __device__ __forceinline__ int off(int it) const {  // offset of the copy in the staged layout
        if constexpr (RPI % G::E == 0)
            return G::xidx(r0, c) + it * (RPI / G::E) * G::SEG;
        else
            return G::xidx(row(it), c);
    }
};

// Start gathering channels [ch0, ch0 + C) of the rows perm[lo + r] of v [n][B].
// Copies of G::VW floats (16 or 8 bytes) when the rows of v keep that alignment,
// else 4 bytes.  Rows past n and channels past B are staged as zero.
template <class G, int W>
__device__ __forceinline__ void stage_rows_w(const float* __restrict__ v, int B, int ch0, int64_t n, int64_t lo,
                                             const uint32_t* p_buf, float* x_buf, uint64_t pol) {
    const RowWalk<G, W> wk;
    const int rem = (int)((n - lo) < (int64_t)G::R ? (n - lo) : (int64_t)G::R);
    const uint32_t last = (uint32_t)(n - 1);
    const bool cok = ch0 + wk.c < B;
    const float* src0 = v + ch0 + wk.c;
#pragma unroll
    for (int it = 0; it < RowWalk<G, W>::ITER; ++it) {
        const int r = wk.row(it);
        if (G::R % RowWalk<G, W>::RPI != 0 && r >= G::R) break;
        float* dst = x_buf + wk.off(it);
        if (r < rem && cok) {
            const float* src = src0 + (size_t)min(p_buf[r], last) * B;
            if constexpr (W == 4)
                cp_async16(dst, src, pol);
            else if constexpr (W == 2)
                cp_async8(dst, src, pol);
            else
                cp_async4(dst, src, pol);
        } else {
#pragma unroll
            for (int q = 0; q < W; ++q) dst[q] = 0.f;
        }
    }
}

template <class G>
__device__ __forceinline__ void stage_rows(const float* __restrict__ v, int B, int ch0, int64_t n, int64_t lo,
                                           const uint32_t* p_buf, float* x_buf, uint64_t pol) {
    if (G::VW > 1 && (B % G::VW) == 0)
        stage_rows_w<G, G::VW>(v, B, ch0, n, lo, p_buf, x_buf, pol);
    else
        stage_rows_w<G, 1>(v, B, ch0, n, lo, p_buf, x_buf, pol);
}

// Store a staged tile back to the rows perm[lo + r] of out [n][B] (the inverse
// of stage_rows; rows past n and channels past B are skipped).
template <class G, int W>
__device__ __forceinline__ void store_rows_w(float* __restrict__ out, int B, int ch0, int64_t n, int64_t lo,
                                             const uint32_t* p_buf, const float* x_buf, uint64_t pol) {
    const RowWalk<G, W> wk;
    const int rem = (int)((n - lo) < (int64_t)G::R ? (n - lo) : (int64_t)G::R);
    const uint32_t last = (uint32_t)(n - 1);
    if (ch0 + wk.c >= B) return;
    float* dst0 = out + ch0 + wk.c;
#pragma unroll
    for (int it = 0; it < RowWalk<G, W>::ITER; ++it) {
        const int r = wk.row(it);
        if (r >= rem || (G::R % RowWalk<G, W>::RPI != 0 && r >= G::R)) break;
        float* dst = dst0 + (size_t)min(p_buf[r], last) * B;
        const float* sp = x_buf + wk.off(it);
        if constexpr (W == 4)
            st_hint(reinterpret_cast<float4*>(dst), *reinterpret_cast<const float4*>(sp), pol);
        else if constexpr (W == 2)
            st_hint(reinterpret_cast<float2*>(dst), *reinterpret_cast<const float2*>(sp), pol);
        else
            st_hint(dst, *sp, pol);
    }
}

template <class G>
__device__ __forceinline__ void store_rows(float* __restrict__ out, int B, int ch0, int64_t n, int64_t lo,
                                           const uint32_t* p_buf, const float* x_buf, uint64_t pol) {
    if (G::VW > 1 && (B % G::VW) == 0)
        store_rows_w<G, G::VW>(out, B, ch0, n, lo, p_buf, x_buf, pol);
    else
        store_rows_w<G, 1>(out, B, ch0, n, lo, p_buf, x_buf, pol);
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

// One step with a single input t sitting at the row (no interval part): the
// common case of the symmetric scans.  Written without the zero interval input so
// that no addition of +0 (which IEEE arithmetic may not drop) is issued.
__device__ __forceinline__ LP lp_step_x(LP s, float dv, float t) {
    const float d = fabsf(dv);
    LP o;
    o.P = fmaf(d, s.P, t);
    o.L = (dv >= 0.f) ? d * s.P : s.L;
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
