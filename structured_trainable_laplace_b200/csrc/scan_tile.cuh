// Tile-level pieces of the LAPLEX scans: the linear-recurrence monoid, the
// in-tile block scan over thread segments, and the decoupled lookback between
// tiles ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary
// section 2.2, "Exact scan algebra": after sorting, each triangular part of the
// kernel matrix is a prefix or suffix scan of y_(r) = x_(r) + exp(a_(r-1) - a_(r)) y_(r-1)).
//
// A scan direction walks rows in processing order with ORIENTED anchors u
// (u = a for the left-to-right direction, u = -a for right-to-left), so u never
// decreases along the walk and every decay exp(u_prev - u) lies in [0, 1].
// Each row r carries two inputs: l_r, contributions whose source anchor lies
// strictly before u_r (already weighted to u_r), and t_r, contributions sitting
// exactly at u_r.  The state at row r is the pair
//     P_r = sum of everything up to and including u_r, weighted exp(u_src - u_r)
//     L_r = the part of P_r whose source lies strictly before u_r
// with the recurrence (d = exp(u_(r-1) - u_r))
//     P_r = d P_(r-1) + l_r + t_r
//     L_r = u_r > u_(r-1) ? d P_(r-1) + l_r : L_(r-1) + l_r.
// P gives the products; L (strict sums, ties excluded) gives the anchor
// gradients with sign(0) = 0.  Decays are always exp of an anchor difference
// between two rows, never a product of many decays and never exp(a) alone.
//
// A segment summary (L, P) is the state at the segment's last row computed from
// a zero incoming state; it is anchored at that row's u.  Summaries compose:
//   A then B:  P = e P_A + P_B,  L = u_B > u_A ? e P_A + L_B : L_A + L_B,  e = exp(u_A - u_B).
#pragma once

#include "common.cuh"

namespace laplex {

struct LP {
    float L, P;
};

__device__ __forceinline__ LP lp_step(LP s, float u_prev, float u, float l, float t) {
    const float d = expf(u_prev - u);
    LP o;
    o.P = fmaf(d, s.P, l + t);
    o.L = (u > u_prev) ? fmaf(d, s.P, l) : (s.L + l);
    return o;
}

__device__ __forceinline__ LP lp_combine(LP A, float uA, LP B, float uB) {
    const float e = expf(uA - uB);
    LP o;
    o.P = fmaf(e, A.P, B.P);
    o.L = (uB > uA) ? fmaf(e, A.P, B.L) : (A.L + B.L);
    return o;
}

__device__ __forceinline__ double2 lpd_combine(double2 A, float uA, double2 B, float uB) {
    // fp64 carries between tiles: x = L, y = P
    const double e = exp((double)uA - (double)uB);
    double2 o;
    o.y = fma(e, A.y, B.y);
    o.x = (uB > uA) ? fma(e, A.y, B.x) : (A.x + B.x);
    return o;
}

// Shared scratch of one block scan (one direction) with NW warps, C channels.
template <int C, int NW>
struct ScanSmem {
    LP wtot[NW][C];
    LP wexcl[NW][C];
    float wu[NW];
    LP tot[C];
};

// In-tile scan over thread segments.  Thread (c, k) = (tid % C, tid / C) owns
// segment k of channel c.  In processing order, segment k's predecessor is k-1
// (REV = false) or k+1 (REV = true).
//   seg:      the segment summary, anchored at u_end
//   u_before: oriented anchor of the row just before the segment in processing order
// Returns in (excl, has_excl) the composition of all earlier segments of the tile,
// anchored at u_before.  On return sm.tot[c] is the tile total (anchored at the
// tile's last row in processing order).  Contains two __syncthreads; every thread
// of the block must call it.
template <int C, int NT, bool REV>
__device__ __forceinline__ void block_scan_dir(LP seg, float u_end, float u_before, ScanSmem<C, NT / 32>& sm,
                                               LP& excl, bool& has_excl) {
    constexpr int SW = 32 / C;
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int c = threadIdx.x % C;
    const int q = REV ? (SW - 1 - lane / C) : (lane / C);

    LP inc = seg;
#pragma unroll
    for (int off = 1; off < SW; off <<= 1) {
        const int src = (REV ? lane + off * C : lane - off * C) & 31;
        LP o;
        o.L = __shfl_sync(0xffffffffu, inc.L, src);
        o.P = __shfl_sync(0xffffffffu, inc.P, src);
        const float uo = __shfl_sync(0xffffffffu, u_end, src);
        if (q >= off) inc = lp_combine(o, uo, inc, u_end);
    }
    {
        const int src = (REV ? lane + C : lane - C) & 31;
        excl.L = __shfl_sync(0xffffffffu, inc.L, src);
        excl.P = __shfl_sync(0xffffffffu, inc.P, src);
        has_excl = (q >= 1);
    }
    if (q == SW - 1) {
        sm.wtot[w][c] = inc;
        if (c == 0) sm.wu[w] = u_end;
    }
    __syncthreads();
    if (threadIdx.x < C * NW) {
        const int cc = threadIdx.x % C;
        const int jp = threadIdx.x / C;  // processing position of the target warp
        LP acc = {0.f, 0.f};
        float uacc = 0.f;
        for (int j = 0; j < jp; ++j) {
            const int wj = REV ? NW - 1 - j : j;
            const LP v = sm.wtot[wj][cc];
            const float uv = sm.wu[wj];
            acc = (j == 0) ? v : lp_combine(acc, uacc, v, uv);
            uacc = uv;
        }
        const int wt = REV ? NW - 1 - jp : jp;
        sm.wexcl[wt][cc] = acc;
        if (jp == NW - 1) {
            const LP v = sm.wtot[wt][cc];
            sm.tot[cc] = (jp == 0) ? v : lp_combine(acc, uacc, v, sm.wu[wt]);
        }
    }
    __syncthreads();
    const int wpos = REV ? NW - 1 - w : w;
    if (wpos > 0) {
        const LP we = sm.wexcl[w][c];
        const float uwe = sm.wu[REV ? w + 1 : w - 1];
        excl = has_excl ? lp_combine(we, uwe, excl, u_before) : we;
        has_excl = true;
    }
}

// One decoupled-lookback chain: per tile a status flag (0 none, 1 aggregate,
// 2 inclusive) and fp64 (L, P) values per channel.
struct Chain {
    int* flags;    // [T]
    double2* agg;  // [T][C]
    double2* inc;  // [T][C]  inclusive state at the tile's last row (processing order)
};

// The chains of all channel groups of one scan: group g's arrays start at
// g * T (flags) and g * T * C (values).
struct ChainSet {
    int* flags;
    double2* agg;
    double2* inc;
    int64_t T;
    int C;
    __device__ __forceinline__ Chain chain(int g) const {
        return Chain{flags + (int64_t)g * T, agg + (int64_t)g * T * C, inc + (int64_t)g * T * C};
    }
};

// Shared scratch of a block-wide lookback (NT threads, C channels).  A window
// holds W predecessors: thread (c, g) = (tid % C, tid / C) takes channel c of
// slots g, g + NT / C, ... (Q of them), so a window's states are read with one
// round of independent loads whatever its width.
template <int C, int NT>
struct LookbackSmem {
    static constexpr int Q = (128 * C / NT) > 1 ? 128 * C / NT : 1;
    static constexpr int W = NT / C * Q;
    double2 part[NT / 32][C];
    double2 run[C];
    double e[W];
    int flag[W];
    int stop[2];
    bool brk[W];
};

// Publish tile t's total and look back over its predecessors (t-1, t-2, ... or
// t+1, t+2, ... when REV).  Called by every thread of the block; thread c < C
// passes channel c's tile total in tot (anchored at u_tile_end).  u_before_tile:
// oriented anchor of the last row of the predecessor tile.  Returns, to every
// thread, the incoming carry of channel tid % C (anchored at u_before_tile), and
// whether one exists.
//
// A window is W predecessors: thread i < W polls the flag of the i-th and reads
// the anchor at its end, the nearest one that holds an inclusive state bounds
// the window, and once every tile up to it has published, the block sums the
// window's states and the next window is read only if none was inclusive.
// Waits are bounded: past kSpinLimit polls the tile records kStatusTimeout and
// proceeds with what it has.
template <int C, bool REV, int NT>
__device__ __forceinline__ double2 block_lookback(Chain ch, int64_t t, int64_t T, const float* s, int64_t n, int64_t R,
                                                  LP tot, float u_tile_end, float u_before_tile, int32_t* status,
                                                  LookbackSmem<C, NT>& sm, bool& has_carry) {
    using S = LookbackSmem<C, NT>;
    constexpr int Q = S::Q, W = S::W, SG = NT / C;
    const int tid = threadIdx.x, c = tid % C, g = tid / C;
    const bool first = REV ? (t == T - 1) : (t == 0);
    const double2 totd = make_double2((double)tot.L, (double)tot.P);
    // only the threads that wrote a value fence before the block barrier that
    // precedes the flag's release
    if (first) {
        if (tid < C) {
            ch.inc[t * C + tid] = totd;
            __threadfence();
        }
        __syncthreads();
        if (tid == 0) st_release(&ch.flags[t], 2);
        has_carry = false;
        return make_double2(0.0, 0.0);
    }
    if (tid == 0) sm.stop[0] = sm.stop[1] = W;
    if (tid < C) {
        ch.agg[t * C + tid] = totd;
        sm.run[tid] = make_double2(0.0, 0.0);
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) st_release(&ch.flags[t], 1);
    bool have = false;
    int64_t jb = REV ? t + 1 : t - 1;  // nearest predecessor of the window
    uint32_t spins = 0;
    bool timed_out = false;
    for (int it = 0;; ++it) {
        // Every state taken is weighted to the same anchor (the end of the nearest
        // predecessor), so the carry is a plain sum of independent terms: slot i
        // adds e_i P_i to P and, to L, e_i P_i when its end lies strictly before
        // that anchor, else its own strict part L_i.  A slot still unpublished
        // after the bound counts as zero.
        for (int i = tid; i < W; i += NT) {
            const int64_t jl = REV ? jb + i : jb - i;
            const bool exists = REV ? (jl < T) : (jl >= 0);
            // 3 marks a slot past the end tile (which always publishes an
            // inclusive state, so the window never reaches one)
            const int f = exists ? ld_acquire(&ch.flags[jl]) : 3;
            const float uj = exists ? (REV ? -s[jl * R] : s[min(n, (jl + 1) * R) - 1]) : 0.f;
            const bool brk = u_before_tile > uj;
            sm.flag[i] = f;
            sm.brk[i] = brk;
            sm.e[i] = brk ? exp((double)uj - (double)u_before_tile) : 1.0;
            if (f >= 2) atomicMin(&sm.stop[it & 1], i);
        }
        __syncthreads();
        const int stop = sm.stop[it & 1];  // last window slot to take
        if (tid == 0) sm.stop[(it + 1) & 1] = W;
        bool zero = false;
        for (int i = tid; i <= stop && i < W; i += NT) zero = zero || (sm.flag[i] == 0);
        if (__syncthreads_or(zero) && !timed_out) {
            if (++spins > kSpinLimit) {
                if (tid == 0) raise_status(status, kStatusTimeout);
                timed_out = true;
            } else {
                __nanosleep(64);
            }
            continue;
        }
        double2 vk[Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int i = g + q * SG;
            const int f = (i <= stop) ? sm.flag[i] : 0;
            const int64_t ji = REV ? jb + i : jb - i;
            vk[q] = make_double2(0.0, 0.0);
            if (f == 1) vk[q] = __ldcg(&ch.agg[ji * C + c]);
            if (f == 2) vk[q] = __ldcg(&ch.inc[ji * C + c]);
        }
        double2 part = make_double2(0.0, 0.0);
        bool took = false;
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int i = g + q * SG;
            const int f = (i <= stop) ? sm.flag[i] : 0;
            if (f == 1 || f == 2) {
                const double e = sm.e[i];
                part.y = fma(e, vk[q].y, part.y);
                part.x = sm.brk[i] ? fma(e, vk[q].y, part.x) : part.x + vk[q].x;
                took = true;
            }
        }
#pragma unroll
        for (int off = C; off < 32; off <<= 1) {
            part.x += __shfl_xor_sync(0xffffffffu, part.x, off);
            part.y += __shfl_xor_sync(0xffffffffu, part.y, off);
        }
        if ((tid & 31) < C) sm.part[tid >> 5][tid & 31] = part;
        have = __syncthreads_or(took) || have;
        if (tid < C) {
            double2 r = sm.run[tid];
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) {
                r.x += sm.part[w][tid].x;
                r.y += sm.part[w][tid].y;
            }
            sm.run[tid] = r;
        }
        if (stop < W || timed_out) break;
        jb = REV ? jb + W : jb - W;
    }
    __syncthreads();
    const double2 run = sm.run[c];
    if (tid < C) {
        ch.inc[t * C + tid] = have ? lpd_combine(run, u_before_tile, totd, u_tile_end) : totd;
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) st_release(&ch.flags[t], 2);
    has_carry = have;
    return run;
}

// Incoming state of a segment: the tile carry (anchored at u_tile) followed by
// the in-tile exclusive prefix (anchored at u_seg).
__device__ __forceinline__ LP seg_incoming(bool has_carry, LP carry, float u_tile, bool has_excl, LP excl,
                                           float u_seg) {
    if (has_carry && has_excl) return lp_combine(carry, u_tile, excl, u_seg);
    if (has_carry) return carry;
    if (has_excl) return excl;
    return LP{0.f, 0.f};
}

// Channels per group of a scan over Cb channels: the next power of two, at most 32.
inline int choose_channels(int64_t Cb) {
    int C = 1;
    while (C < Cb && C < 32) C <<= 1;
    return C;
}

// Stage the tile's sorted anchors (one before, R rows, one after; sentinels
// outside [0, n)) and its permutation entries in shared memory.
template <int R>
__device__ __forceinline__ void load_tile_meta(const float* __restrict__ s, const uint32_t* __restrict__ perm, int64_t n,
                                               int64_t lo, float* s_sm, uint32_t* p_sm) {
    for (int i = threadIdx.x; i < R + 2; i += blockDim.x) {
        const int64_t r = lo - 1 + i;
        s_sm[i] = (r < 0) ? kLowAnchor : (r < n ? __ldg(s + r) : kHighAnchor);
    }
    if (p_sm != nullptr)
        for (int i = threadIdx.x; i < R; i += blockDim.x) {
            const int64_t r = lo + i;
            p_sm[i] = r < n ? min(__ldg(perm + r), (uint32_t)(n - 1)) : 0u;  // clamp: never index past the rows
        }
}

}  // namespace laplex
