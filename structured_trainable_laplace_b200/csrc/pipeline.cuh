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

// Shared scratch of block_scan2 for NV vectors, both directions.
template <int C, int NT, int NV>
struct Scan2Smem {
    static constexpr int NW = NT / 32;
    LP wtL[NW][NV][C], wtR[NW][NV][C];  // warp totals
    LP wxL[NW][NV][C], wxR[NW][NV][C];  // exclusive prefixes over warps
    float wuL[NW], wuR[NW];             // oriented anchors of each warp's last row
};

// In-tile scan of NV vectors in both directions at once (one barrier pair).
// Thread (c, k) = (tid % C, tid / C) owns segment k of channel c; left
// processing order is k ascending, right is k descending.  segL/segR are the
// segment summaries, anchored at uL_end = a(last row) and uR_end = -a(first row);
// uL_before / uR_before are the oriented anchors of the row just before the
// segment in each direction.  Returns the in-tile exclusive prefixes (anchored
// at uL_before / uR_before) with has-flags.  on_total(c, totL, totR) runs once
// per channel, after the tile totals are known and before the final barrier,
// so it can publish tile carries to shared memory for every thread.
template <int C, int NT, int NV, class F>
__device__ __forceinline__ void block_scan2(const LP (&segL)[NV], const LP (&segR)[NV], float uL_end, float uL_before,
                                            float uR_end, float uR_before, Scan2Smem<C, NT, NV>& sm, LP (&exL)[NV],
                                            LP (&exR)[NV], bool& hL, bool& hR, F&& on_total) {
    constexpr int SW = 32 / C;
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, c = threadIdx.x % C;
    const int ql = lane / C, qr = SW - 1 - ql;
    LP incL[NV], incR[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        incL[v] = segL[v];
        incR[v] = segR[v];
    }
#pragma unroll
    for (int off = 1; off < SW; off <<= 1) {
        const int sL = (lane - off * C) & 31, sR = (lane + off * C) & 31;
        const float uoL = __shfl_sync(0xffffffffu, uL_end, sL), uoR = __shfl_sync(0xffffffffu, uR_end, sR);
        const float eL = expf(uoL - uL_end), eR = expf(uoR - uR_end);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            LP oL, oR;
            oL.L = __shfl_sync(0xffffffffu, incL[v].L, sL);
            oL.P = __shfl_sync(0xffffffffu, incL[v].P, sL);
            oR.L = __shfl_sync(0xffffffffu, incR[v].L, sR);
            oR.P = __shfl_sync(0xffffffffu, incR[v].P, sR);
            if (ql >= off) incL[v] = combine_e(oL, incL[v], eL, uL_end > uoL);
            if (qr >= off) incR[v] = combine_e(oR, incR[v], eR, uR_end > uoR);
        }
    }
    {
        const int sL = (lane - C) & 31, sR = (lane + C) & 31;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            exL[v].L = __shfl_sync(0xffffffffu, incL[v].L, sL);
            exL[v].P = __shfl_sync(0xffffffffu, incL[v].P, sL);
            exR[v].L = __shfl_sync(0xffffffffu, incR[v].L, sR);
            exR[v].P = __shfl_sync(0xffffffffu, incR[v].P, sR);
        }
        hL = ql >= 1;
        hR = qr >= 1;
    }
    if (ql == SW - 1) {
#pragma unroll
        for (int v = 0; v < NV; ++v) sm.wtL[w][v][c] = incL[v];
        if (c == 0) sm.wuL[w] = uL_end;
    }
    if (qr == SW - 1) {
#pragma unroll
        for (int v = 0; v < NV; ++v) sm.wtR[w][v][c] = incR[v];
        if (c == 0) sm.wuR[w] = uR_end;
    }
    __syncthreads();
    if (threadIdx.x < C * NW) {
        const int cc = threadIdx.x % C, jp = threadIdx.x / C;
        LP aL[NV], aR[NV];
        // left: fold warps 0 .. jp-1
        for (int j = 0; j < jp; ++j) {
            const float e = (j > 0) ? expf(sm.wuL[j - 1] - sm.wuL[j]) : 0.f;
            const bool brk = (j > 0) && sm.wuL[j] > sm.wuL[j - 1];
#pragma unroll
            for (int v = 0; v < NV; ++v) aL[v] = (j == 0) ? sm.wtL[0][v][cc] : combine_e(aL[v], sm.wtL[j][v][cc], e, brk);
        }
        // right: fold warps NW-1 .. NW-jp (processing order)
        for (int j = 0; j < jp; ++j) {
            const int wj = NW - 1 - j;
            const float e = (j > 0) ? expf(sm.wuR[wj + 1] - sm.wuR[wj]) : 0.f;
            const bool brk = (j > 0) && sm.wuR[wj] > sm.wuR[wj + 1];
#pragma unroll
            for (int v = 0; v < NV; ++v) aR[v] = (j == 0) ? sm.wtR[wj][v][cc] : combine_e(aR[v], sm.wtR[wj][v][cc], e, brk);
        }
        if (jp > 0) {
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                sm.wxL[jp][v][cc] = aL[v];
                sm.wxR[NW - 1 - jp][v][cc] = aR[v];
            }
        }
        if (jp == NW - 1) {
            LP tL[NV], tR[NV];
            const float eL = (NW > 1) ? expf(sm.wuL[NW - 2] - sm.wuL[NW - 1]) : 0.f;
            const bool bL = (NW > 1) && sm.wuL[NW - 1] > sm.wuL[NW - 2];
            const float eR = (NW > 1) ? expf(sm.wuR[1] - sm.wuR[0]) : 0.f;
            const bool bR = (NW > 1) && sm.wuR[0] > sm.wuR[1];
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                tL[v] = (NW > 1) ? combine_e(aL[v], sm.wtL[NW - 1][v][cc], eL, bL) : sm.wtL[0][v][cc];
                tR[v] = (NW > 1) ? combine_e(aR[v], sm.wtR[0][v][cc], eR, bR) : sm.wtR[0][v][cc];
            }
            on_total(cc, tL, tR);
        }
    }
    __syncthreads();
    if (w > 0) {
        const float uwe = sm.wuL[w - 1];
        const float e = expf(uwe - uL_before);
        const bool brk = uL_before > uwe;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const LP we = sm.wxL[w][v][c];
            exL[v] = hL ? combine_e(we, exL[v], e, brk) : we;
        }
        hL = true;
    }
    if (w < NW - 1) {
        const float uwe = sm.wuR[w + 1];
        const float e = expf(uwe - uR_before);
        const bool brk = uR_before > uwe;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const LP we = sm.wxR[w][v][c];
            exR[v] = hR ? combine_e(we, exR[v], e, brk) : we;
        }
        hR = true;
    }
}

}  // namespace laplex
