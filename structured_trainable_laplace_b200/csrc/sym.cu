// Symmetric LAPLEX operator y = K x, K_ij = exp(-|a_i - a_j|), and its backward
// ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary section 2.2,
// "symmetric case": after sorting, the lower triangle is the prefix scan
// P_r = x_r + exp(a_(r-1) - a_(r)) P_(r-1), the upper triangle the mirrored suffix
// scan S_r, and y = P + S - x because both contain the diagonal).
//
// Both directions of the scan are needed at every row, and the vectors do not
// fit on chip, so each product reads its input twice.  The two reads are made
// free of inter-tile waits by partitioning the sorted rows into P contiguous
// base ranges of tiles:
//   k_sym_agg    walks its ranges right to left and writes, per tile, the fp64
//                suffix state of the base range from that tile's first row on
//                (RS), and each base range's aggregates in both directions;
//   k_sym_carry_direct  gives each base range its fp64 carries from the
//                left/right as sums of the other ranges' aggregates, each
//                weighted straight to the range's boundary;
//   k_sym_sweep  walks its ranges left to right, folding the left state tile by
//                tile and taking the right state from RS and the range carry,
//                evaluates both directions inside each tile and writes
//                y = P + S - x through the permutation (forward), or, over x and
//                g at once, gx = K g = P_g + S_g - g and
//                ga = sum_c g (R_x - L_x) + x (R_g - L_g) from the strict sums
//                (ties excluded: sign(0) = 0); x's RS and carries come from the
//                forward (the `saved` buffer) or are recomputed.
// Each persistent CTA walks m consecutive base ranges, m chosen per kernel so
// that its grid is one full wave at that kernel's occupancy.
//
// Inside a CTA each warp owns whole channels of the tile: lane (cs, k) holds the
// k-th segment of E rows of one channel, so the in-tile scan is a shuffle scan
// over the lanes of that channel and the fp64 range fold runs in the channel's
// first lane.  The only block barriers are the one that publishes a staged tile
// and the one before the coalesced output stores.  Tiles are staged with
// cp.async: the gathered rows AHEAD tiles ahead, anchors, permutation and
// carries one tile further; per-row decays and the fp64 decays of the tile folds
// are computed one tile ahead.  No kernel waits on another CTA.
#include <mutex>

#include <cuda.h>

#include "laplex.h"
#include "laplex_internal.h"
#include "pipeline.cuh"

namespace laplex {

namespace {

constexpr int kE = 16;
constexpr int kMaxRanges = 8192;   // base ranges per channel group
constexpr int kRangesPerSM = 6;    // base ranges per SM (divisible by the usual occupancies)
constexpr int kAheadAgg = 2;       // prefetch distance of the gathered rows (aggregate pass)
constexpr int kAheadFwd = 1;       // of the streamed sorted tiles: forward sweep
constexpr int kAheadBwd = 1;       // backward sweep (two streamed vectors)

template <int C>
struct SymGeo {
    static constexpr int NW = C < 8 ? C : 8;  // warps per CTA
    static constexpr int NT = NW * 32;
    static constexpr int CW = C / NW;  // channels per warp
    static constexpr int SK = 32 / CW;  // segments per channel = lanes per channel group
    // staged rows padded by CW floats per segment (conflict-free column reads), or
    // by 4 when CW = 2, which keeps the rows 16-byte aligned for 16-byte copies at
    // the price of 2-way conflicts
    using G = TileGeo<C, NT, kE, (CW == 2 ? 4 : CW)>;
    static constexpr int R = G::R;  // rows per tile (SK * E)
};

// Single channel (B = 1): tiles of k1NT threads x k1E rows, loaded straight into
// registers (see the one-channel kernels below).
constexpr int k1NT = 256, k1E = 16, k1NW = k1NT / 32, k1R = k1NT * k1E;
// Above this many rows (a 64 MB single-channel output) the one-channel sweeps
// write sorted-order outputs and launch_unpermute places them.
constexpr int64_t kUnpermuteMinRows = 1ll << 24;

inline int64_t rows_per_tile(int C) {
    return C == 1 ? k1R : (C <= 8 ? 32 * kE : (32 * kE * 8) / C);
}

template <int C>
__host__ __device__ constexpr int tile_rows() {
    return C == 1 ? k1R : SymGeo<C>::R;
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Decays of one staged tile of SK segments, all encoded as by enc_decay and
// computed once per tile (one tile ahead) instead of once per lane:
//   d[k][e]   row k*E+e from the row before it, e in [0, E] (the last entry repeats
//             the next segment's first, so each segment's row has E+1 entries
//             and the SK lanes of a channel read distinct banks);
//   gL/gR[j]  the step of width 2^j of the scans over segments (left: from the
//             last row of segment k - 2^j to that of k; right: from -first row of
//             k + 2^j to -first row of k);
//   iL/iR[k]  from the tile carry to the state before segment k (left: row
//             before the tile to the row before segment k; right: -row after the
//             tile to -row after segment k).
template <int SK>
struct SegTab {
    static constexpr int LOG = ilog2(SK) > 0 ? ilog2(SK) : 1;
    float d[SK][kE + 1];
    float gL[LOG][SK], gR[LOG][SK];
    float iL[SK], iR[SK];
};

template <int SK, int NT>
__device__ __forceinline__ void seg_tables(const float* sb, SegTab<SK>& tb) {
    constexpr int E = kE, R = SK * E, LOG = ilog2(SK);
    constexpr int N1 = SK * (E + 1), N2 = N1 + LOG * SK, N3 = N2 + SK;
    for (int i = threadIdx.x; i < N3; i += NT) {
        if (i < N1) {
            const int k = i / (E + 1), e = i % (E + 1), r = k * E + e;
            tb.d[k][e] = enc_decay(sb[3 + r], sb[4 + r]);
        } else if (i < N2) {
            const int j = (i - N1) / SK, k = (i - N1) % SK, off = 1 << j;
            tb.gL[j][k] = (k >= off) ? enc_decay(sb[4 + (k - off) * E + E - 1], sb[4 + k * E + E - 1]) : -1.f;
            tb.gR[j][k] = (k + off < SK) ? enc_decay(-sb[4 + (k + off) * E], -sb[4 + k * E]) : -1.f;
        } else {
            const int k = i - N2;
            tb.iL[k] = enc_decay(sb[3], sb[3 + k * E]);
            tb.iR[k] = enc_decay(-sb[4 + R], -sb[4 + (k + 1) * E]);
        }
    }
}

// State entering a segment: the tile carry (if any) followed by the exclusive
// scan over the segments before it (if any); ev is the decay between the two.
__device__ __forceinline__ LP seg_in(bool has_carry, LP carry, bool has_excl, LP excl, float ev) {
    if (has_carry && has_excl) return combine_v(carry, excl, ev);
    if (has_carry) return carry;
    if (has_excl) return excl;
    return LP{0.f, 0.f};
}

// Sum of v[E] over the CW lanes of a row group (lanes SK apart) by recursive
// halving: afterwards lane cs holds in v[0, E/CW) the sums for rows
// seg_rows_base<CW>(cs) + [0, E/CW) of its segment.
template <int CW, int SK>
__device__ __forceinline__ void reduce_scatter(float (&v)[kE], int cs) {
    int len = kE;
#pragma unroll
    for (int o = 1; o < CW; o <<= 1) {
        len >>= 1;
        const bool upper = (cs & o) != 0;
#pragma unroll
        for (int i = 0; i < kE / 2; ++i) {
            if (i < len) {
                const float keep = upper ? v[i + len] : v[i];
                const float send = upper ? v[i] : v[i + len];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o * SK);
            }
        }
    }
}

template <int CW>
__device__ __forceinline__ int seg_rows_base(int cs) {
    int base = 0, len = kE;
#pragma unroll
    for (int o = 1; o < CW; o <<= 1) {
        len >>= 1;
        if (cs & o) base += len;
    }
    return base;
}

struct SymScan {
    const float* s;
    const uint32_t* perm;
    int64_t n;
    int B;
    int64_t T;    // tiles per channel group
    int P;        // base ranges per channel group
    int64_t tpr;  // tiles per base range
    int m;        // base ranges walked by one CTA
};

// fp64 scan state of one vector, per channel group, base range J, tile t, channel c
struct RangeState {
    double2* RS;    // [G][T][C]  right state from tile t's first row to its base range's end
    double2* Lagg;  // [G][P][C]  range aggregate, left direction (anchored at its last row)
    double2* Ragg;  // [G][P][C]  range aggregate, right direction (anchored at -its first row)
    double2* Lin;   // [G][P][C]  carry from the ranges before (anchored at the row before)
    double2* Rin;   // [G][P][C]  carry from the ranges after (anchored at -the row after)
};

// Shared memory of the aggregate pass, which gathers rows through the permutation.
template <int C, int AHEAD>
struct AggSmem {
    using G = typename SymGeo<C>::G;
    static constexpr int MA = AHEAD + 2;  // anchors and permutation are staged MA tiles ahead
    static constexpr int MS = MA + 1;     // anchor / permutation slots
    static constexpr int VS = AHEAD + 1;  // gathered-row slots
    float s[MS][G::SS];
    uint32_t p[MS][G::R];
    float v[1][VS][G::XS];
    SegTab<SymGeo<C>::SK> tab[2];  // decay tables of the current and the next tile
    double ed[2][2];               // fp64 decays of the two tile-level folds, current and next tile
};

// Shared memory of the sweeps, which stream the sorted copies written by the
// aggregate pass (see SortedTile) instead of gathering rows.
template <int C, int NV, int AHEAD>
struct SweepSmem {
    using SG = SymGeo<C>;
    using G = typename SG::G;
    static constexpr int MS = AHEAD + 2;      // anchor / permutation / carry slots
    static constexpr int VS = AHEAD + 1;      // sorted-tile slots
    static constexpr int KS = C * kE + 4;     // floats per staged segment (4 of padding)
    static constexpr int TS = SG::SK * KS;    // floats per staged sorted tile
    float s[MS][G::SS];
    uint32_t p[MS][G::R];
    double2 rs[MS][NV][C];   // RS[t+1]
    double2 rin[MS][NV][C];  // carry entering the tile's base range from the right
    alignas(16) float v[NV][VS][TS];
    float o[G::XS];          // output rows (y or gx) in the gathered layout, for the scatter
    SegTab<SG::SK> tab[2];   // decay tables of the current and the next tile
    double ed[2][2];         // fp64 decays of the two tile-level folds, current and next tile
    // backward: per-warp sums of the ga shares of the warp's channels, rows padded
    // as in SegTab::d
    float gp[NV == 2 ? SG::NW : 1][NV == 2 ? SG::SK * (kE + 1) : 1];
};

// Sorted copy of one vector: tile t of channel group grp is R*C contiguous floats
// holding the value of sorted row k*E + e, channel c, at [k][c][e], so that each
// lane's E values are contiguous.  Rows past n and channels past B hold zero.
template <class F>
__device__ __forceinline__ F* sorted_tile(F* vs, int grp, int64_t T, int64_t t, int R, int C) {
    return vs + ((int64_t)grp * T + t) * (int64_t)R * C;
}

// Start copying one sorted tile into the staged segment-major layout (16-byte
// copies; KS-float segment stride keeps the lanes' 16-byte reads conflict-free).
template <int C>
__device__ __forceinline__ void stage_sorted(const float* __restrict__ src, float* dst, uint64_t pol) {
    using SG = SymGeo<C>;
    constexpr int SEGF = C * kE, KS = SEGF + 4, NCOPY = SG::SK * SEGF / 4;
    static_assert(NCOPY % SG::NT == 0, "whole copies per thread");
#pragma unroll
    for (int q = 0; q < NCOPY / SG::NT; ++q) {
        const int f = 4 * (threadIdx.x + q * SG::NT), k = f / SEGF;
        cp_async16(dst + k * KS + (f - k * SEGF), src + f, pol);
    }
}

__device__ __forceinline__ int64_t tile_lo(int64_t t, int R) { return t * (int64_t)R; }

__device__ __forceinline__ double2 to_d2(LP v) { return make_double2((double)v.L, (double)v.P); }

__device__ __forceinline__ LP shfl_lp(LP v, int src, int width) {
    LP o;
    o.L = __shfl_sync(0xffffffffu, v.L, src, width);
    o.P = __shfl_sync(0xffffffffu, v.P, src, width);
    return o;
}

// Inclusive scans over the SK segments of one channel (the SK lanes of a group),
// both directions, NV vectors.  tb: the tile's decay tables; k: this lane's segment.
template <int SK, int NV>
__device__ __forceinline__ void group_scan(LP (&incL)[NV], LP (&incR)[NV], const SegTab<SK>& tb, int k) {
#pragma unroll
    for (int j = 0, off = 1; off < SK; ++j, off <<= 1) {
        const float evL = tb.gL[j][k], evR = tb.gR[j][k];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            LP oL, oR;
            oL.L = __shfl_up_sync(0xffffffffu, incL[v].L, off, SK);
            oL.P = __shfl_up_sync(0xffffffffu, incL[v].P, off, SK);
            oR.L = __shfl_down_sync(0xffffffffu, incR[v].L, off, SK);
            oR.P = __shfl_down_sync(0xffffffffu, incR[v].P, off, SK);
            if (k >= off) incL[v] = combine_v(oL, incL[v], evL);
            if (k + off < SK) incR[v] = combine_v(oR, incR[v], evR);
        }
    }
}

// The same scans for the inclusive sums P alone (the forward product).
template <int SK>
__device__ __forceinline__ void group_scan_p(float& pl, float& pr, const SegTab<SK>& tb, int k) {
#pragma unroll
    for (int j = 0, off = 1; off < SK; ++j, off <<= 1) {
        const float oL = __shfl_up_sync(0xffffffffu, pl, off, SK);
        const float oR = __shfl_down_sync(0xffffffffu, pr, off, SK);
        if (k >= off) pl = fmaf(fabsf(tb.gL[j][k]), oL, pl);
        if (k + off < SK) pr = fmaf(fabsf(tb.gR[j][k]), oR, pr);
    }
}

__device__ __forceinline__ float seg_in_p(bool has_carry, float carry, bool has_excl, float excl, float ev) {
    if (has_carry && has_excl) return fmaf(fabsf(ev), carry, excl);
    if (has_carry) return carry;
    if (has_excl) return excl;
    return 0.f;
}

// Tiles walked by CTA blockIdx.x: those of base ranges [J0, J1).
struct CtaTiles {
    int J0, J1;
    int64_t tb, te;
};

__device__ __forceinline__ CtaTiles cta_tiles(const SymScan& a) {
    CtaTiles w;
    w.J0 = blockIdx.x * a.m;
    w.J1 = min(a.P, w.J0 + a.m);
    w.tb = (int64_t)w.J0 * a.tpr;
    w.te = min(a.T, (int64_t)w.J1 * a.tpr);
    return w;
}

// ------------------------------------------------------------------ pass A

// Walks tiles te-1 .. tb.  Per tile: the right total extends the running suffix of
// its base range (RS[t]), the left total is prepended to the range's running left
// aggregate; both restart at each base range's last tile and are written out at
// its first.
template <int C, int AHEAD>
__global__ void __launch_bounds__(SymGeo<C>::NT, (SymGeo<C>::NT == 256 ? 3 : 1))
    k_sym_agg(SymScan a, const float* __restrict__ v, RangeState st, float* __restrict__ vs) {
    using SG = SymGeo<C>;
    using G = typename SG::G;
    using SM = AggSmem<C, AHEAD>;
    constexpr int E = kE, R = G::R, SK = SG::SK, CW = SG::CW, MS = SM::MS, VS = SM::VS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SM& sm = *reinterpret_cast<SM*>(smem_raw);
    const int grp = blockIdx.y;
    const CtaTiles w = cta_tiles(a);
    const int nt = (int)(w.te - w.tb);
    const int lane = threadIdx.x & 31, cs = lane / SK, k = lane % SK;
    const int c = (threadIdx.x >> 5) * CW + cs, ch0 = grp * C;
    auto tile_of = [&](int i) { return w.te - 1 - i; };
    // anchors, permutation and the sorted copy stream through once; the gathered
    // rows keep normal priority (the other row of a 128-byte line may follow soon)
    const uint64_t pol_f = l2_evict_first(), pol_n = l2_evict_normal();
    // anchor of the last row of base range J
    auto range_end = [&](int64_t J) { return __ldg(a.s + min(a.n, (J + 1) * a.tpr * (int64_t)R) - 1); };
    // fp64 decays of the tile folds, negative for a tie (decay 1, no break): [0] right
    // fold (-row after the tile -> -its first row), [1] left fold (the tile's last row
    // -> its base range's last row)
    // Thread 0 computes [0], thread 32 (another warp) [1], in parallel; thread 32
    // keeps the current range's end anchor and reloads it only when the range changes.
    int64_t J_ue = -1;
    float ue_c = 0.f;
    auto tile_ed = [&](const float* sb, int64_t t, double* ed) {
        if (threadIdx.x == 0) {
            ed[0] = (sb[4 + R] > sb[4]) ? exp((double)sb[4] - (double)sb[4 + R]) : -1.0;
        } else if (threadIdx.x == 32) {
            const int64_t J = t / a.tpr;
            if (J != J_ue) {
                J_ue = J;
                ue_c = range_end(J);
            }
            ed[1] = (ue_c > sb[4 + R - 1]) ? exp((double)sb[4 + R - 1] - (double)ue_c) : -1.0;
        }
    };
    // cp.async groups, in commit order: anchors+permutation of tiles 0 .. MA-1
    // (waited for at once), rows of tiles 0 .. AHEAD-1, then per iteration j the
    // anchors+permutation of tile j+MA and the rows of tile j+AHEAD.  At the top
    // of iteration i at most WAIT groups may stay pending: the rows of tile i have
    // at least AHEAD-1 groups after them and the permutation of tile i+AHEAD
    // (read when its rows are staged) has three.
    constexpr int MA = SM::MA, WAIT = (AHEAD - 1 < 3) ? AHEAD - 1 : 3;
    static_assert(AHEAD >= 1, "at least one tile of prefetch");
#pragma unroll
    for (int q = 0; q < MA; ++q) {
        if (q < nt) stage_meta<G>(a.s, a.perm, a.n, tile_lo(tile_of(q), R), sm.s[q % MS], sm.p[q % MS], pol_f);
        cp_async_commit();
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int q = 0; q < AHEAD; ++q) {
        if (q < nt) stage_rows<G>(v, a.B, ch0, a.n, tile_lo(tile_of(q), R), sm.p[q % MS], sm.v[0][q % VS], pol_n);
        cp_async_commit();
    }
    seg_tables<SK, SG::NT>(sm.s[0], sm.tab[0]);
    tile_ed(sm.s[0], tile_of(0), sm.ed[0]);
    double2 runR = make_double2(0.0, 0.0), runL = make_double2(0.0, 0.0);
    for (int i = 0; i < nt; ++i) {
        const int64_t t = tile_of(i);
        const int64_t J = t / a.tpr;
        cp_async_wait<WAIT>();  // this tile's rows and the anchors of the tiles ahead are in
        __syncthreads();
        if (i + MA < nt)
            stage_meta<G>(a.s, a.perm, a.n, tile_lo(tile_of(i + MA), R), sm.s[(i + MA) % MS], sm.p[(i + MA) % MS],
                          pol_f);
        cp_async_commit();
        if (i + AHEAD < nt)
            stage_rows<G>(v, a.B, ch0, a.n, tile_lo(tile_of(i + AHEAD), R), sm.p[(i + AHEAD) % MS],
                          sm.v[0][(i + AHEAD) % VS], pol_n);
        cp_async_commit();
        if (i + 1 < nt) {
            seg_tables<SK, SG::NT>(sm.s[(i + 1) % MS], sm.tab[(i + 1) & 1]);
            tile_ed(sm.s[(i + 1) % MS], tile_of(i + 1), sm.ed[(i + 1) & 1]);
        }
        const float* sb = sm.s[i % MS];
        const SegTab<SK>& tb = sm.tab[i & 1];
        const float* dk = tb.d[k];
        const float* xb = sm.v[0][i % VS] + k * G::SEG + c;
        float xv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) xv[e] = xb[e * C];
        {  // this lane's E values of the sorted copy
            float4* dst = reinterpret_cast<float4*>(sorted_tile(vs, grp, a.T, t, R, C) + (k * C + c) * E);
#pragma unroll
            for (int q = 0; q < E / 4; ++q)
                st_hint(dst + q, make_float4(xv[4 * q], xv[4 * q + 1], xv[4 * q + 2], xv[4 * q + 3]), pol_f);
        }
        LP sr[1] = {{0.f, 0.f}}, sl[1] = {{0.f, 0.f}};
#pragma unroll
        for (int e = E - 1; e >= 0; --e) sr[0] = lp_step_x(sr[0], dk[e + 1], xv[e]);
#pragma unroll
        for (int e = 0; e < E; ++e) sl[0] = lp_step_x(sl[0], dk[e], xv[e]);
        group_scan<SK, 1>(sl, sr, tb, k);
        const LP tl = shfl_lp(sl[0], SK - 1, SK);  // tile totals: left at the last segment, right at the first
        if (k == 0) {
            const double* ed = sm.ed[i & 1];
            const bool last_of_range = (t + 1 == min(a.T, (J + 1) * a.tpr));  // the first one walked
            const double2 trd = to_d2(sr[0]), tld = to_d2(tl);
            runR = last_of_range ? trd : combine_ed(runR, trd, fabs(ed[0]), ed[0] >= 0.0);
            st.RS[((int64_t)grp * a.T + t) * C + c] = runR;
            runL = last_of_range ? tld : combine_ed(tld, runL, fabs(ed[1]), ed[1] >= 0.0);
            if (t == J * a.tpr) {  // first tile of the base range: its aggregates are complete
                st.Lagg[((int64_t)grp * a.P + J) * C + c] = runL;
                st.Ragg[((int64_t)grp * a.P + J) * C + c] = runR;
            }
        }
    }
}

// ------------------------------------------------------------------ pass B

// The carries entering each base range, from the range aggregates, in direct form:
// one CTA per base range J (grid P x G).  The carry from the left is the sum over
// the ranges J' < J of their left aggregates,
// each weighted by the fp64 decay from its end straight to the row before J (a
// range whose end ties with that row adds its strict part L to L), and mirrored
// from the right.  The anchors are sorted, so the weights fall with the distance:
// ranges are taken in windows of kDirW nearest ones per side, and the walk stops
// at the first weight that underflows to zero (every farther one does too).  No
// chain of dependent folds: a window is one round of loads and a block reduction.
constexpr int kDirNT = 128;
constexpr int kDirW = 64;

template <int C>
__global__ void __launch_bounds__(kDirNT) k_sym_carry_direct(SymScan a, RangeState st) {
    constexpr int SG = kDirNT / C;  // slot groups
    __shared__ double s_e[2][kDirW];
    __shared__ bool s_brk[2][kDirW];
    __shared__ double2 s_part[2][kDirNT / 32][C];
    __shared__ int s_more;
    const int J = blockIdx.x, grp = blockIdx.y, P = a.P;
    const int tid = threadIdx.x, c = tid % C, g = tid / C;
    const int64_t RR = a.tpr * (int64_t)tile_rows<C>();  // rows per range
    auto uL = [&](int jj) { return __ldg(a.s + min(a.n, (jj + 1) * RR) - 1); };  // left aggregate's anchor
    auto uR = [&](int jj) { return -__ldg(a.s + jj * RR); };                    // right aggregate's anchor
    const float ubL = J > 0 ? uL(J - 1) : 0.f;       // the row before range J
    const float ubR = J + 1 < P ? uR(J + 1) : 0.f;   // -(the row after range J)
    const double2* Lagg = st.Lagg + (int64_t)grp * P * C;
    const double2* Ragg = st.Ragg + (int64_t)grp * P * C;
    double2 accL = make_double2(0.0, 0.0), accR = make_double2(0.0, 0.0);
    for (int base = 0;; base += kDirW) {
        // weights of this window: slot i is range J-1-base-i (left) / J+1+base+i (right)
        if (tid < 2 * kDirW) {
            const int side = tid / kDirW, i = tid % kDirW;
            const int jj = side ? J + 1 + base + i : J - 1 - base - i;
            double e = 0.0;
            bool brk = true;
            if (jj >= 0 && jj < P) {
                const float uj = side ? uR(jj) : uL(jj), ub = side ? ubR : ubL;
                brk = ub > uj;
                e = brk ? exp((double)uj - (double)ub) : 1.0;
            }
            s_e[side][i] = e;
            s_brk[side][i] = brk;
        }
        if (tid == 0) s_more = 0;
        __syncthreads();
#pragma unroll
        for (int side = 0; side < 2; ++side) {
            const double2* agg = side ? Ragg : Lagg;
            double2& acc = side ? accR : accL;
            for (int i = g; i < kDirW; i += SG) {
                const double e = s_e[side][i];
                if (e == 0.0) continue;  // underflowed (or past the ends): adds nothing
                const int jj = side ? J + 1 + base + i : J - 1 - base - i;
                const double2 v = __ldcg(agg + (int64_t)jj * C + c);
                acc.y = fma(e, v.y, acc.y);
                acc.x = s_brk[side][i] ? fma(e, v.y, acc.x) : acc.x + v.x;
            }
        }
        // another window only while the farthest range of this one still contributes
        if (tid == 0 && ((s_e[0][kDirW - 1] != 0.0 && J - 1 - base - kDirW >= 0) ||
                         (s_e[1][kDirW - 1] != 0.0 && J + 1 + base + kDirW < P)))
            s_more = 1;
        __syncthreads();
        const bool more = s_more != 0;
        __syncthreads();  // the window's weights are read before the next one writes them
        if (!more) break;
    }
#pragma unroll
    for (int off = C; off < 32; off <<= 1) {
        accL.x += __shfl_xor_sync(0xffffffffu, accL.x, off);
        accL.y += __shfl_xor_sync(0xffffffffu, accL.y, off);
        accR.x += __shfl_xor_sync(0xffffffffu, accR.x, off);
        accR.y += __shfl_xor_sync(0xffffffffu, accR.y, off);
    }
    if ((tid & 31) < C) {
        s_part[0][tid >> 5][tid & 31] = accL;
        s_part[1][tid >> 5][tid & 31] = accR;
    }
    __syncthreads();
    if (tid < 2 * C) {
        const int side = tid / C, cc = tid % C;
        double2 r = make_double2(0.0, 0.0);
#pragma unroll
        for (int w = 0; w < kDirNT / 32; ++w) {
            r.x += s_part[side][w][cc].x;
            r.y += s_part[side][w][cc].y;
        }
        // zero (unused) for the first range's left and the last range's right carry
        (side ? st.Rin : st.Lin)[((int64_t)grp * P + J) * C + cc] = r;
    }
}

// ------------------------------------------------------------------ pass C

// Start copying, for tile t, RS[t+1] (if t+1 is in the same base range) and the
// right carry of t's base range, for each vector.
template <int C, int NV>
__device__ __forceinline__ void stage_carries(const SymScan& a, const RangeState& sx, const RangeState& sg, int grp,
                                              int64_t t,
                                              double2 (*rs_dst)[C], double2 (*rin_dst)[C]) {
    const int64_t J = t / a.tpr;
    const bool more = t + 1 < min(a.T, (J + 1) * a.tpr);
    const bool hasRin = J + 1 < a.P;
    for (int i = threadIdx.x; i < NV * C; i += SymGeo<C>::NT) {
        const int w = i / C, c = i % C;
        const double2* RS = (w == 0) ? sx.RS : sg.RS;
        const double2* Rin = (w == 0) ? sx.Rin : sg.Rin;
        if (more) cp_async16(&rs_dst[w][c], RS + ((int64_t)grp * a.T + t + 1) * C + c);
        if (hasRin) cp_async16(&rin_dst[w][c], Rin + ((int64_t)grp * a.P + J) * C + c);
    }
}

// NV = 1: forward (x -> y = out).  NV = 2: backward (x, g -> gx = out, ga).
// xs / gs are the sorted copies of x and g that the aggregate passes wrote.
template <int C, int NV, int AHEAD>
__global__ void __launch_bounds__(SymGeo<C>::NT, (SymGeo<C>::NT == 256 ? (NV == 1 ? 3 : 2) : 1)) k_sym_sweep(
    SymScan a, const float* __restrict__ xs, const float* __restrict__ gs, RangeState sx, RangeState sg,
    float* __restrict__ out, float* __restrict__ ga, int ga_atomic) {
    using SG = SymGeo<C>;
    using G = typename SG::G;
    using SM = SweepSmem<C, NV, AHEAD>;
    constexpr int E = kE, R = G::R, SK = SG::SK, CW = SG::CW, NT = SG::NT, MS = SM::MS, VS = SM::VS, KS = SM::KS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SM& sm = *reinterpret_cast<SM*>(smem_raw);
    const int grp = blockIdx.y;
    const CtaTiles cw = cta_tiles(a);
    const int nt = (int)(cw.te - cw.tb);
    const int lane = threadIdx.x & 31, cs = lane / SK, k = lane % SK;
    const int c = (threadIdx.x >> 5) * CW + cs, ch0 = grp * C;
    // oriented anchor of the row after base range J (where its right carry is anchored)
    auto u_rin = [&](int64_t J) { return -__ldg(a.s + min(a.n - 1, (J + 1) * a.tpr * (int64_t)R)); };
    // fp64 decays of the tile folds, negative for a tie (decay 1, no break):
    // [0] left fold (row before the tile -> its last row), [1] right carry (the row
    // after the base range -> the row after the tile)
    // Thread 0 computes [0], thread 32 (another warp) [1], in parallel; thread 32
    // keeps the current range's right anchor and reloads it only when the range changes.
    int64_t J_ur = -1;
    float ur_c = 0.f;
    auto tile_ed = [&](const float* sb, int64_t t, double* ed) {
        if (threadIdx.x == 0) {
            ed[0] = (sb[4 + R - 1] > sb[3]) ? exp((double)sb[3] - (double)sb[4 + R - 1]) : -1.0;
        } else if (threadIdx.x == 32) {
            const int64_t J = t / a.tpr;
            if (J != J_ur) {
                J_ur = J;
                ur_c = u_rin(J);
            }
            ed[1] = (-sb[4 + R] > ur_c) ? exp((double)ur_c + (double)sb[4 + R]) : -1.0;
        }
    };
    // everything but the scattered 4-byte ga rows streams through L2 once
    const uint64_t pol_f = l2_evict_first(), pol_l = l2_evict_last();
    // cp.async groups per iteration j: anchors+permutation+carries of tile j+AHEAD+1,
    // then the sorted tiles of tile j+AHEAD; waiting until AHEAD-1 groups remain
    // leaves the current tile's data and the next tile's anchors complete when
    // AHEAD <= 2
    static_assert(AHEAD >= 1 && AHEAD <= 2, "prefetch distance of the sweeps");
    auto stage_vecs = [&](int64_t tt, int slot) {
#pragma unroll
        for (int w = 0; w < NV; ++w)
            stage_sorted<C>(sorted_tile(w == 0 ? xs : gs, grp, a.T, tt, R, C), sm.v[w][slot], pol_f);
    };
#pragma unroll
    for (int q = 0; q <= AHEAD; ++q) {
        if (q < nt) {
            stage_meta<G>(a.s, a.perm, a.n, tile_lo(cw.tb + q, R), sm.s[q % MS], sm.p[q % MS], pol_f);
            stage_carries<C, NV>(a, sx, sg, grp, cw.tb + q, sm.rs[q % MS], sm.rin[q % MS]);
        }
        cp_async_commit();
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int q = 0; q < AHEAD; ++q) {
        if (q < nt) stage_vecs(cw.tb + q, q % VS);
        cp_async_commit();
    }
    seg_tables<SK, NT>(sm.s[0], sm.tab[0]);
    tile_ed(sm.s[0], cw.tb, sm.ed[0]);

    // fp64 left folds of channel c, kept by the channel's first lane (k == 0)
    double2 runL[NV];
    bool hasL = (cw.J0 > 0);
    const int64_t rng = ((int64_t)grp * a.P + cw.J0) * C + c;
#pragma unroll
    for (int w = 0; w < NV; ++w) runL[w] = hasL ? (w == 0 ? sx.Lin : sg.Lin)[rng] : make_double2(0.0, 0.0);

    for (int i = 0; i < nt; ++i) {
        const int64_t t = cw.tb + i, lo = tile_lo(t, R);
        const int64_t J = t / a.tpr;
        cp_async_wait<AHEAD - 1>();
        __syncthreads();
        if (i + AHEAD + 1 < nt) {
            stage_meta<G>(a.s, a.perm, a.n, tile_lo(t + AHEAD + 1, R), sm.s[(i + AHEAD + 1) % MS],
                          sm.p[(i + AHEAD + 1) % MS], pol_f);
            stage_carries<C, NV>(a, sx, sg, grp, t + AHEAD + 1, sm.rs[(i + AHEAD + 1) % MS],
                                 sm.rin[(i + AHEAD + 1) % MS]);
        }
        cp_async_commit();
        if (i + AHEAD < nt) stage_vecs(t + AHEAD, (i + AHEAD) % VS);
        cp_async_commit();
        if (i + 1 < nt) {
            seg_tables<SK, NT>(sm.s[(i + 1) % MS], sm.tab[(i + 1) & 1]);
            tile_ed(sm.s[(i + 1) % MS], t + 1, sm.ed[(i + 1) & 1]);
        }
        const SegTab<SK>& tb = sm.tab[i & 1];
        const float* dk = tb.d[k];
        float* ob = sm.o + k * G::SEG + c;  // this lane's output column (gathered layout)
        const bool more = (t + 1 < min(a.T, (J + 1) * a.tpr)), hasRin = (J + 1 < a.P);
        const bool hl_tile = hasL, hr_tile = hasRin || more;
        const double* ed = sm.ed[i & 1];
        hasL = true;
        // this lane's E values of each vector (segment k, channel c)
        float xr[NV][E];
#pragma unroll
        for (int w = 0; w < NV; ++w) {
            const float4* src = reinterpret_cast<const float4*>(sm.v[w][i % VS] + k * KS + c * E);
#pragma unroll
            for (int q = 0; q < E / 4; ++q) {
                const float4 f = src[q];
                xr[w][4 * q] = f.x;
                xr[w][4 * q + 1] = f.y;
                xr[w][4 * q + 2] = f.z;
                xr[w][4 * q + 3] = f.w;
            }
        }
        if constexpr (NV == 1) {
            // forward: y = P + S - x needs only the inclusive sums (ties enter with decay 1)
            float pr = 0.f, pl = 0.f;
#pragma unroll
            for (int e = E - 1; e >= 0; --e) pr = fmaf(fabsf(dk[e + 1]), pr, xr[0][e]);
#pragma unroll
            for (int e = 0; e < E; ++e) pl = fmaf(fabsf(dk[e]), pl, xr[0][e]);
            group_scan_p<SK>(pl, pr, tb, k);
            // tile carries: the channel's first lane folds in fp64, then broadcasts
            const float tl = __shfl_sync(0xffffffffu, pl, SK - 1, SK);
            float cl = 0.f, cr = 0.f;
            if (k == 0) {
                double crd = hasRin ? sm.rin[i % MS][0][c].y : 0.0;
                if (more) {
                    const double rsn = sm.rs[i % MS][0][c].y;
                    crd = hasRin ? fma(fabs(ed[1]), crd, rsn) : rsn;
                }
                cl = (float)runL[0].y;
                cr = (float)crd;
                runL[0].y = hl_tile ? fma(fabs(ed[0]), runL[0].y, (double)tl) : (double)tl;
            }
            cl = __shfl_sync(0xffffffffu, cl, 0, SK);
            cr = __shfl_sync(0xffffffffu, cr, 0, SK);
            // incoming state of this segment: tile carry, then the segments before it
            const float exl = __shfl_sync(0xffffffffu, pl, (lane - 1) & 31);
            const float exr = __shfl_sync(0xffffffffu, pr, (lane + 1) & 31);
            float Pr = seg_in_p(hr_tile, cr, k + 1 < SK, exr, tb.iR[k]);
            float Pl = seg_in_p(hl_tile, cl, k >= 1, exl, tb.iL[k]);
            // pass 2
            float yv[E];
#pragma unroll
            for (int e = E - 1; e >= 0; --e) {
                Pr = fmaf(fabsf(dk[e + 1]), Pr, xr[0][e]);
                yv[e] = Pr - xr[0][e];
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                Pl = fmaf(fabsf(dk[e]), Pl, xr[0][e]);
                ob[e * C] = yv[e] + Pl;
            }
        } else {
            // backward: the strict sums L (and R) are needed for ga, so both scans
            // carry (L, P)
            LP sr[NV], sl[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                sr[w] = LP{0.f, 0.f};
                sl[w] = LP{0.f, 0.f};
#pragma unroll
                for (int e = E - 1; e >= 0; --e) sr[w] = lp_step_x(sr[w], dk[e + 1], xr[w][e]);
#pragma unroll
                for (int e = 0; e < E; ++e) sl[w] = lp_step_x(sl[w], dk[e], xr[w][e]);
            }
            group_scan<SK, NV>(sl, sr, tb, k);  // now inclusive over segments 0..k (left) / k..SK-1 (right)
            LP cL[NV], cR[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                const LP tl = shfl_lp(sl[w], SK - 1, SK);
                cL[w] = LP{0.f, 0.f};
                cR[w] = LP{0.f, 0.f};
                if (k == 0) {
                    const double2 cl = runL[w];
                    double2 cr = hasRin ? sm.rin[i % MS][w][c] : make_double2(0.0, 0.0);
                    if (more) {
                        const double2 rsn = sm.rs[i % MS][w][c];
                        cr = hasRin ? combine_ed(cr, rsn, fabs(ed[1]), ed[1] >= 0.0) : rsn;
                    }
                    cL[w] = LP{(float)cl.x, (float)cl.y};
                    cR[w] = LP{(float)cr.x, (float)cr.y};
                    const double2 tld = to_d2(tl);
                    runL[w] = hl_tile ? combine_ed(runL[w], tld, fabs(ed[0]), ed[0] >= 0.0) : tld;
                }
                cL[w] = shfl_lp(cL[w], 0, SK);
                cR[w] = shfl_lp(cR[w], 0, SK);
            }
            const float evl = tb.iL[k], evr = tb.iR[k];
            LP inR[NV], inL[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                const LP exL = shfl_lp(sl[w], (lane - 1) & 31, 32), exR = shfl_lp(sr[w], (lane + 1) & 31, 32);
                inL[w] = seg_in(hl_tile, cL[w], k >= 1, exL, evl);
                inR[w] = seg_in(hr_tile, cR[w], k + 1 < SK, exR, evr);
            }
            // pass 2: gx to the output rows, ga to the per-warp sums
            float gap[E], gxr[E];
            LP ax = inR[0], ag = inR[NV - 1];
#pragma unroll
            for (int e = E - 1; e >= 0; --e) {
                const float xe = xr[0][e], ge = xr[NV - 1][e], dv = dk[e + 1];
                ax = lp_step_x(ax, dv, xe);
                ag = lp_step_x(ag, dv, ge);
                gxr[e] = ag.P - ge;                  // gx, right part
                gap[e] = fmaf(ge, ax.L, xe * ag.L);  // strict right sums
            }
            ax = inL[0];
            ag = inL[NV - 1];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float xe = xr[0][e], ge = xr[NV - 1][e], dv = dk[e];
                ax = lp_step_x(ax, dv, xe);
                ag = lp_step_x(ag, dv, ge);
                ob[e * C] = gxr[e] + ag.P;                    // gx
                gap[e] = fmaf(-ge, ax.L, fmaf(-xe, ag.L, gap[e]));  // this channel's share of ga
            }
            // sum over the warp's channels, then one padded row per warp in shared memory
            reduce_scatter<CW, SK>(gap, cs);
            const int rb = seg_rows_base<CW>(cs);
            float* gpw = sm.gp[threadIdx.x >> 5] + k * (E + 1) + rb;
#pragma unroll
            for (int e = 0; e < E / CW; ++e) gpw[e] = gap[e];
        }
        __syncthreads();
        // coalesced stores of whole rows through the permutation
        const uint32_t* pb = sm.p[i % MS];
        if (out != nullptr) store_rows<G>(out, a.B, ch0, a.n, lo, pb, sm.o, pol_f);
        if (NV == 2 && ga != nullptr) {
            for (int r = threadIdx.x; r < R; r += NT) {
                if (lo + r >= a.n) continue;
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < SG::NW; ++q) acc += sm.gp[q][r + r / E];  // channels past B hold zero
                const int64_t row = min(pb[r], (uint32_t)(a.n - 1));
                if (ga_atomic)
                    atomicAdd(ga + row, acc);
                else
                    st_hint(ga + row, acc, pol_l);  // kept in L2 until its lines are complete
            }
        }
    }
}

// ------------------------------------------------------- one channel (B = 1)
//
// With a single channel every row carries 4 bytes, so staging tiles in shared
// memory would cost as much as the rows themselves and would cap the CTAs per
// SM.  Instead thread q of a tile owns rows lo + q*k1E .. + k1E - 1: it loads
// their anchors and permutation entries with 16-byte loads, gathers (aggregate
// pass) or streams (sweeps) their values into registers, and scatters its
// outputs through the permutation itself; many tiles' gathers are in flight per
// SM.  The tile's scans: a sequential pass per thread, a shuffle scan over the
// warp's 32 segments, and a pass over the k1NW warp totals in shared memory.
// The base ranges, range aggregates, carries and the saved state are those of
// the multi-channel kernels with C = 1 and tiles of k1R rows.

struct Rows1 {
    float a[k1E];       // anchors, kHighAnchor past n
    uint32_t p[k1E];    // permutation entries (clamped), 0 past n
    float ap, an;       // anchors of the rows just before / after the segment
    int64_t row0;
};

// WITH_PERM false: the permutation entries are not needed (outputs in sorted
// order) and are not read.
template <bool WITH_PERM = true>
__device__ __forceinline__ void load_rows1(const float* __restrict__ s, const uint32_t* __restrict__ perm, int64_t n,
                                           int64_t row0, Rows1& r) {
    r.row0 = row0;
    const uint32_t last = (uint32_t)(n - 1);
    if (row0 + k1E <= n) {
#pragma unroll
        for (int q = 0; q < k1E / 4; ++q) {
            const float4 av = __ldg(reinterpret_cast<const float4*>(s + row0) + q);
            r.a[4 * q] = av.x, r.a[4 * q + 1] = av.y, r.a[4 * q + 2] = av.z, r.a[4 * q + 3] = av.w;
            if (WITH_PERM) {
                const uint4 pv = __ldg(reinterpret_cast<const uint4*>(perm + row0) + q);
                r.p[4 * q] = min(pv.x, last), r.p[4 * q + 1] = min(pv.y, last);
                r.p[4 * q + 2] = min(pv.z, last), r.p[4 * q + 3] = min(pv.w, last);
            } else {
                r.p[4 * q] = r.p[4 * q + 1] = r.p[4 * q + 2] = r.p[4 * q + 3] = 0u;
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < k1E; ++e) {
            const bool in = row0 + e < n;
            r.a[e] = in ? __ldg(s + row0 + e) : kHighAnchor;
            r.p[e] = (in && WITH_PERM) ? min(__ldg(perm + row0 + e), last) : 0u;
        }
    }
    r.ap = (row0 == 0) ? kLowAnchor : (row0 - 1 < n ? __ldg(s + row0 - 1) : kHighAnchor);
    r.an = (row0 + k1E < n) ? __ldg(s + row0 + k1E) : kHighAnchor;
}

// Encoded decays into each row from the row before it (d[0] from ap), and d[k1E]
// from the last row to the row after the segment (see enc_decay).
__device__ __forceinline__ void decays1(const Rows1& r, float (&d)[k1E + 1]) {
    d[0] = enc_decay(r.ap, r.a[0]);
#pragma unroll
    for (int e = 1; e < k1E; ++e) d[e] = enc_decay(r.a[e - 1], r.a[e]);
    d[k1E] = enc_decay(r.a[k1E - 1], r.an);
}

// Inclusive shuffle scans over the 32 segments of a warp, left (over lanes
// 0..lane, anchored at the lane's last row) and right (lanes lane..31, anchored
// at -its first row), NV vectors.
template <int NV>
__device__ __forceinline__ void warp_scan1(LP (&l)[NV], LP (&rr)[NV], float ul, float ur) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float uo_l = __shfl_up_sync(0xffffffffu, ul, off);
        const float uo_r = __shfl_down_sync(0xffffffffu, ur, off);
        const float evl = enc_decay(uo_l, ul), evr = enc_decay(uo_r, ur);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            LP ol, orr;
            ol.L = __shfl_up_sync(0xffffffffu, l[v].L, off);
            ol.P = __shfl_up_sync(0xffffffffu, l[v].P, off);
            orr.L = __shfl_down_sync(0xffffffffu, rr[v].L, off);
            orr.P = __shfl_down_sync(0xffffffffu, rr[v].P, off);
            if (lane >= off) l[v] = combine_v(ol, l[v], evl);
            if (lane + off < 32) rr[v] = combine_v(orr, rr[v], evr);
        }
    }
}

// Cross-warp scratch of one tile.
template <int NV>
struct Cross1 {
    LP wl[NV][k1NW], wr[NV][k1NW];  // warp inclusive totals
    float ul[k1NW], ur[k1NW];       // left: anchor of the warp's last row; right: -anchor of its first row
    LP xl[NV][k1NW], xr[NV][k1NW];  // exclusive states entering each warp (from the warps before / after)
    LP tl[NV], tr[NV];              // tile totals
    LP cl[NV], cr[NV];              // tile carries (sweeps)
    bool hl, hr;                    // carries present
};

// Warp totals -> exclusive states per warp and the tile totals.  Threads 0 ..
// k1NW-1 each serve one warp; one __syncthreads inside, the caller syncs after.
template <int NV>
__device__ __forceinline__ void cross_warps1(Cross1<NV>& cx) {
    __syncthreads();
    const int w = threadIdx.x;
    if (w < k1NW) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            LP acc = {0.f, 0.f};
            float ua = 0.f;
            for (int j = 0; j < w; ++j) {
                acc = (j == 0) ? cx.wl[v][0] : lp_combine(acc, ua, cx.wl[v][j], cx.ul[j]);
                ua = cx.ul[j];
            }
            cx.xl[v][w] = acc;
            if (w == k1NW - 1) cx.tl[v] = (w == 0) ? cx.wl[v][w] : lp_combine(acc, ua, cx.wl[v][w], cx.ul[w]);
            acc = LP{0.f, 0.f};
            for (int j = k1NW - 1; j > w; --j) {
                acc = (j == k1NW - 1) ? cx.wr[v][j] : lp_combine(acc, ua, cx.wr[v][j], cx.ur[j]);
                ua = cx.ur[j];
            }
            cx.xr[v][w] = acc;
            if (w == 0) cx.tr[v] = (k1NW == 1) ? cx.wr[v][0] : lp_combine(acc, ua, cx.wr[v][0], cx.ur[0]);
        }
    }
}

// Aggregate pass for one channel: walks its base ranges' tiles right to left,
// writes the sorted copy, RS and the range aggregates (as k_sym_agg).
// SORTED_IN: the sorted copy vs already holds the values in sorted order (placed
// there through the inverse permutation); it is read, the permutation is not.
template <bool SORTED_IN>
__global__ void __launch_bounds__(k1NT, 3) k_sym1_agg(SymScan a, const float* __restrict__ v, RangeState st,
                                                     float* __restrict__ vs) {
    __shared__ Cross1<1> cx;
    const CtaTiles w = cta_tiles(a);
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    auto range_end = [&](int64_t J) { return __ldg(a.s + min(a.n, (J + 1) * a.tpr * (int64_t)k1R) - 1); };
    double2 runR = make_double2(0.0, 0.0), runL = make_double2(0.0, 0.0);
    for (int64_t t = w.te - 1; t >= w.tb; --t) {
        const int64_t lo = t * (int64_t)k1R, J = t / a.tpr;
        Rows1 r;
        load_rows1<!SORTED_IN>(a.s, a.perm, a.n, lo + threadIdx.x * k1E, r);
        float x[k1E];
        if (SORTED_IN) {
            if (r.row0 + k1E <= a.n) {
                const float4* src = reinterpret_cast<const float4*>(vs + r.row0);
#pragma unroll
                for (int q = 0; q < k1E / 4; ++q) {
                    const float4 f = __ldcs(src + q);
                    x[4 * q] = f.x, x[4 * q + 1] = f.y, x[4 * q + 2] = f.z, x[4 * q + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < k1E; ++e) x[e] = (r.row0 + e < a.n) ? __ldcs(vs + r.row0 + e) : 0.f;
            }
        } else {
#pragma unroll
            for (int e = 0; e < k1E; ++e) x[e] = (r.row0 + e < a.n) ? __ldg(v + r.p[e]) : 0.f;
            float4* dst = reinterpret_cast<float4*>(vs + r.row0);
#pragma unroll
            for (int q = 0; q < k1E / 4; ++q) __stcs(dst + q, make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
        }
        float d[k1E + 1];
        decays1(r, d);
        LP sl[1] = {{0.f, 0.f}}, sr[1] = {{0.f, 0.f}};
#pragma unroll
        for (int e = k1E - 1; e >= 0; --e) sr[0] = lp_step_x(sr[0], d[e + 1], x[e]);
#pragma unroll
        for (int e = 0; e < k1E; ++e) sl[0] = lp_step_x(sl[0], d[e], x[e]);
        warp_scan1<1>(sl, sr, r.a[k1E - 1], -r.a[0]);
        if (lane == 31) {
            cx.wl[0][wp] = sl[0];
            cx.ul[wp] = r.a[k1E - 1];
        }
        if (lane == 0) {
            cx.wr[0][wp] = sr[0];
            cx.ur[wp] = -r.a[0];
        }
        cross_warps1<1>(cx);
        __syncthreads();
        if (threadIdx.x == 0) {
            const float f0 = __ldg(a.s + lo);                                    // the tile's first row
            const float fa = (lo + k1R < a.n) ? __ldg(a.s + lo + k1R) : kHighAnchor;  // the row after it
            const float fl = (lo + k1R <= a.n) ? __ldg(a.s + lo + k1R - 1) : kHighAnchor;  // its last row
            const float ue = range_end(J);
            const bool last_of_range = (t + 1 == min(a.T, (J + 1) * a.tpr));
            const double2 trd = to_d2(cx.tr[0]), tld = to_d2(cx.tl[0]);
            const bool br = fa > f0, bl = ue > fl;
            runR = last_of_range ? trd : combine_ed(runR, trd, br ? exp((double)f0 - (double)fa) : 1.0, br);
            st.RS[t] = runR;
            runL = last_of_range ? tld : combine_ed(tld, runL, bl ? exp((double)fl - (double)ue) : 1.0, bl);
            if (t == J * a.tpr) {
                st.Lagg[J] = runL;
                st.Ragg[J] = runR;
            }
        }
        __syncthreads();  // cx is rewritten by the next tile
    }
}

// A thread's 16 outputs: scattered through the permutation, or (sorted_out) in
// sorted order with 16-byte stores, for a later bucketed unpermute.
__device__ __forceinline__ void put_rows1(float* __restrict__ dst, const float (&val)[k1E], const Rows1& r, int64_t n,
                                          int sorted_out) {
    if (sorted_out) {
        if (r.row0 + k1E <= n) {
            float4* d4 = reinterpret_cast<float4*>(dst + r.row0);
#pragma unroll
            for (int q = 0; q < k1E / 4; ++q)
                __stcs(d4 + q, make_float4(val[4 * q], val[4 * q + 1], val[4 * q + 2], val[4 * q + 3]));
        } else {
#pragma unroll
            for (int e = 0; e < k1E; ++e)
                if (r.row0 + e < n) dst[r.row0 + e] = val[e];
        }
    } else {
#pragma unroll
        for (int e = 0; e < k1E; ++e)
            if (r.row0 + e < n) __stcs(dst + r.p[e], val[e]);
    }
}

// Sweep for one channel: NV = 1 forward (xs -> y), NV = 2 backward (xs, gs -> gx,
// ga), from the sorted copies, RS and the range carries (as k_sym_sweep).
// SORTED: the outputs are written in sorted order (for launch_unpermute) and the
// permutation is not read.
template <int NV, bool SORTED>
__global__ void __launch_bounds__(k1NT, NV == 1 ? 3 : 2) k_sym1_sweep(SymScan a, const float* __restrict__ xs,
                                                       const float* __restrict__ gs, RangeState sx, RangeState sg,
                                                       float* __restrict__ out, float* __restrict__ ga) {
    __shared__ Cross1<NV> cx;
    __shared__ double2 s_runL[NV];
    const CtaTiles cw = cta_tiles(a);
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    if (threadIdx.x < NV) {
        const RangeState& sv = (threadIdx.x == 0) ? sx : sg;
        s_runL[threadIdx.x] = (cw.J0 > 0) ? sv.Lin[cw.J0] : make_double2(0.0, 0.0);
    }
    bool hasL = (cw.J0 > 0);
    __syncthreads();
    for (int64_t t = cw.tb; t < cw.te; ++t) {
        const int64_t lo = t * (int64_t)k1R, J = t / a.tpr;
        const bool more = (t + 1 < min(a.T, (J + 1) * a.tpr)), hasRin = (J + 1 < a.P);
        Rows1 r;
        load_rows1<!SORTED>(a.s, a.perm, a.n, lo + threadIdx.x * k1E, r);
        float xv[NV][k1E];
#pragma unroll
        for (int vv = 0; vv < NV; ++vv) {
            const float4* src = reinterpret_cast<const float4*>((vv == 0 ? xs : gs) + r.row0);
#pragma unroll
            for (int q = 0; q < k1E / 4; ++q) {
                const float4 f = __ldcs(src + q);
                xv[vv][4 * q] = f.x, xv[vv][4 * q + 1] = f.y, xv[vv][4 * q + 2] = f.z, xv[vv][4 * q + 3] = f.w;
            }
        }
        // tile carries (thread 0, fp64): left = the running fold, right = RS of the
        // next tile of the range after the range's own right carry
        if (threadIdx.x == 0) {
            const float fa = (lo + k1R < a.n) ? __ldg(a.s + lo + k1R) : kHighAnchor;
            const float ur = -__ldg(a.s + min(a.n - 1, (J + 1) * a.tpr * (int64_t)k1R));
            const bool brr = -fa > ur;
            const double er = brr ? exp((double)ur + (double)fa) : 1.0;
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) {
                const RangeState& sv = (vv == 0) ? sx : sg;
                double2 crd = hasRin ? sv.Rin[J] : make_double2(0.0, 0.0);
                if (more) {
                    const double2 rsn = sv.RS[t + 1];
                    crd = hasRin ? combine_ed(crd, rsn, er, brr) : rsn;
                }
                cx.cr[vv] = LP{(float)crd.x, (float)crd.y};
                cx.cl[vv] = LP{(float)s_runL[vv].x, (float)s_runL[vv].y};
            }
            cx.hl = hasL;
            cx.hr = hasRin || more;
        }
        float d[k1E + 1];
        decays1(r, d);
        LP sl[NV], sr[NV];
#pragma unroll
        for (int vv = 0; vv < NV; ++vv) {
            sl[vv] = LP{0.f, 0.f};
            sr[vv] = LP{0.f, 0.f};
#pragma unroll
            for (int e = k1E - 1; e >= 0; --e) sr[vv] = lp_step_x(sr[vv], d[e + 1], xv[vv][e]);
#pragma unroll
            for (int e = 0; e < k1E; ++e) sl[vv] = lp_step_x(sl[vv], d[e], xv[vv][e]);
        }
        warp_scan1<NV>(sl, sr, r.a[k1E - 1], -r.a[0]);
        if (lane == 31) {
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) cx.wl[vv][wp] = sl[vv];
            cx.ul[wp] = r.a[k1E - 1];
        }
        if (lane == 0) {
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) cx.wr[vv][wp] = sr[vv];
            cx.ur[wp] = -r.a[0];
        }
        cross_warps1<NV>(cx);
        __syncthreads();
        // incoming states of this thread's segment: tile carry, then the warps
        // before (after), then the lanes before (after) in this warp
        const float u_tile_l = (lo > 0) ? __ldg(a.s + lo - 1) : kLowAnchor;          // row before the tile
        const float u_tile_r = -((lo + k1R < a.n) ? __ldg(a.s + lo + k1R) : kHighAnchor);  // -row after it
        const float u_warp_l = (wp > 0) ? cx.ul[wp - 1] : u_tile_l;
        const float u_warp_r = (wp + 1 < k1NW) ? cx.ur[wp + 1] : u_tile_r;
        LP inL[NV], inR[NV];
#pragma unroll
        for (int vv = 0; vv < NV; ++vv) {
            // left
            bool h = cx.hl;
            LP acc = cx.cl[vv];
            if (wp > 0) {
                acc = h ? lp_combine(acc, u_tile_l, cx.xl[vv][wp], u_warp_l) : cx.xl[vv][wp];
                h = true;
            }
            const LP exl = shfl_lp(sl[vv], (lane - 1) & 31, 32);
            if (lane > 0) {
                acc = h ? lp_combine(acc, u_warp_l, exl, r.ap) : exl;
                h = true;
            }
            inL[vv] = h ? acc : LP{0.f, 0.f};
            // right
            h = cx.hr;
            acc = cx.cr[vv];
            if (wp + 1 < k1NW) {
                acc = h ? lp_combine(acc, u_tile_r, cx.xr[vv][wp], u_warp_r) : cx.xr[vv][wp];
                h = true;
            }
            const LP exr = shfl_lp(sr[vv], (lane + 1) & 31, 32);
            if (lane < 31) {
                acc = h ? lp_combine(acc, u_warp_r, exr, -r.an) : exr;
                h = true;
            }
            inR[vv] = h ? acc : LP{0.f, 0.f};
        }
        // the fold of the tile's left total into the running carry (thread 0, after
        // every thread has read the carries above)
        const LP tl0 = cx.tl[0], tl1 = cx.tl[NV - 1];
        if (NV == 1) {
            float pr = inR[0].P, pl = inL[0].P;
            float yv[k1E];
#pragma unroll
            for (int e = k1E - 1; e >= 0; --e) {
                pr = fmaf(fabsf(d[e + 1]), pr, xv[0][e]);
                yv[e] = pr - xv[0][e];
            }
#pragma unroll
            for (int e = 0; e < k1E; ++e) {
                pl = fmaf(fabsf(d[e]), pl, xv[0][e]);
                yv[e] += pl;
            }
            put_rows1(out, yv, r, a.n, SORTED);
        } else {
            LP ax = inR[0], ag = inR[NV - 1];
            float gxr[k1E], gap[k1E];
#pragma unroll
            for (int e = k1E - 1; e >= 0; --e) {
                const float xe = xv[0][e], ge = xv[NV - 1][e], dv = d[e + 1];
                ax = lp_step_x(ax, dv, xe);
                ag = lp_step_x(ag, dv, ge);
                gxr[e] = ag.P - ge;
                gap[e] = fmaf(ge, ax.L, xe * ag.L);  // strict right sums
            }
            ax = inL[0];
            ag = inL[NV - 1];
#pragma unroll
            for (int e = 0; e < k1E; ++e) {
                const float xe = xv[0][e], ge = xv[NV - 1][e], dv = d[e];
                ax = lp_step_x(ax, dv, xe);
                ag = lp_step_x(ag, dv, ge);
                gxr[e] += ag.P;
                gap[e] = fmaf(-ge, ax.L, fmaf(-xe, ag.L, gap[e]));
            }
            if (out != nullptr) put_rows1(out, gxr, r, a.n, SORTED);
            if (ga != nullptr) put_rows1(ga, gap, r, a.n, SORTED);
        }
        if (threadIdx.x == 0) {
            const float fl = (lo + k1R <= a.n) ? __ldg(a.s + lo + k1R - 1) : kHighAnchor;
            const bool bl = fl > u_tile_l;
            const double el = bl ? exp((double)u_tile_l - (double)fl) : 1.0;
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) {
                const LP tlv = (vv == 0) ? tl0 : tl1;
                s_runL[vv] = hasL ? combine_ed(s_runL[vv], to_d2(tlv), el, bl) : to_d2(tlv);
            }
        }
        hasL = true;
        __syncthreads();  // cx and s_runL are rewritten by the next tile
    }
}

// ------------------------------------------------------------------ host side

struct SymPlan {
    int C, G, P;
    int64_t R, T, tpr;
    size_t rs_elems, rng_elems;  // double2 counts of one RS array / one range array
    size_t state_bytes;          // RS, Lin, Rin, Lagg, Ragg of one vector
    size_t saved_state_bytes;    // RS, Lin, Rin of one vector
    size_t sorted_bytes;         // sorted copy of one vector (G * T * R * C floats)
    bool bucketed;               // one channel past the L2: outputs leave through launch_unpermute and the
                                 // inputs enter through the inverse permutation (launch_place)
    size_t unperm_bytes;         // two sorted-order outputs + the unpermute scratch
    size_t inv_bytes;            // the inverse permutation (bucketed only)
    size_t total;
};

SymPlan plan_sym(int64_t n, int64_t B, int sms) {
    SymPlan p;
    p.C = choose_channels(B);
    p.G = (int)((B + p.C - 1) / p.C);
    p.R = rows_per_tile(p.C);
    p.T = (n + p.R - 1) / p.R;
    const int64_t want = std::max<int64_t>(1, ((int64_t)sms * kRangesPerSM + p.G - 1) / p.G);
    const int64_t P0 = std::min<int64_t>(std::min<int64_t>(p.T, want), kMaxRanges);
    p.tpr = (p.T + P0 - 1) / P0;
    p.P = (int)((p.T + p.tpr - 1) / p.tpr);
    p.rs_elems = (size_t)p.G * p.T * p.C;
    p.rng_elems = (size_t)p.G * kMaxRanges * p.C;
    p.state_bytes = align_up(sizeof(double2) * (p.rs_elems + 4 * p.rng_elems), 256);
    p.saved_state_bytes = align_up(sizeof(double2) * (p.rs_elems + 2 * p.rng_elems), 256);
    p.sorted_bytes = align_up(sizeof(float) * (size_t)p.G * p.T * p.R * p.C, 256);
    // per vector (x, g): the scan state and the sorted copy
    p.total = 2 * (p.state_bytes + p.sorted_bytes);
    // single floats scattered through the permutation into an output far larger
    // than the L2 are written in sorted order and regrouped by destination instead
    p.bucketed = (p.C == 1 && n > kUnpermuteMinRows);
    p.unperm_bytes = p.bucketed ? 2 * align_up(sizeof(float) * (size_t)n, 256) + unpermute_workspace_bytes(n) : 0;
    p.inv_bytes = p.bucketed ? align_up(sizeof(uint32_t) * (size_t)n, 256) : 0;
    p.total += p.unperm_bytes + p.inv_bytes;  // the inverse permutation here when there is no saved buffer
    return p;
}

// The sorted-order outputs and the unpermute scratch (after the scan state and
// the sorted copies in the workspace).
float* unperm_outputs(const SymPlan& p, void* ws) { return (float*)((char*)ws + 2 * (p.state_bytes + p.sorted_bytes)); }
void* unperm_scratch(const SymPlan& p, void* ws, int64_t n) {
    return (char*)unperm_outputs(p, ws) + 2 * align_up(sizeof(float) * (size_t)n, 256);
}
// The second sorted-order output slot, free while the inputs are placed: the
// placement's second-split values.
float* place_scratch(const SymPlan& p, void* ws, int64_t n) { return unperm_outputs(p, ws) + align_up((size_t)n, 64); }
// The inverse permutation: after the saved state and sorted copy of the saved
// buffer, or at the end of the workspace.
uint32_t* inv_slot(const SymPlan& p, void* ws, void* saved, int64_t n) {
    if (saved != nullptr) return (uint32_t*)((char*)saved + p.saved_state_bytes + p.sorted_bytes);
    return (uint32_t*)((char*)unperm_scratch(p, ws, n) + unpermute_workspace_bytes(n));
}

RangeState carve(const SymPlan& p, double2* base, bool with_aggs) {
    RangeState st;
    st.RS = base;
    st.Lin = base + p.rs_elems;
    st.Rin = st.Lin + p.rng_elems;
    st.Lagg = with_aggs ? st.Rin + p.rng_elems : nullptr;
    st.Ragg = with_aggs ? st.Lagg + p.rng_elems : nullptr;
    return st;
}

int device_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Opt a kernel into its dynamic shared memory and return its resident CTAs per SM
// (cached per device).
template <class F>
int prepare(F* f, int threads, size_t smem, int& cached) {
    if (cached > 0) return cached;
    int occ = 1;
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, f, threads, smem) != cudaSuccess)
        occ = 1;
    cached = std::max(occ, 1);
    return cached;
}

// Base ranges per CTA so that the grid is one wave at occupancy `occ`.
SymScan scan_args(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, int64_t B, int sms, int occ) {
    SymScan a;
    a.s = s;
    a.perm = perm;
    a.n = n;
    a.B = (int)B;
    a.T = p.T;
    a.P = p.P;
    a.tpr = p.tpr;
    const int64_t slots = std::max<int64_t>(1, (int64_t)sms * occ / p.G);
    a.m = (int)std::max<int64_t>(1, (p.P + slots - 1) / slots);
    return a;
}

// Pass A + pass B for one vector.
// sorted_in (one channel): vs already holds v in sorted order (launch_place); the
// pass reads it instead of gathering v through the permutation.
template <int C>
cudaError_t sym_ranges_t(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, int64_t B, int sms,
                         const float* v, RangeState st, float* vs, cudaStream_t stream, bool sorted_in = false) {
    if constexpr (C == 1) {
        static PerDevice occ_cache[2];
        const int occ = sorted_in ? prepare(k_sym1_agg<true>, k1NT, 0, occ_cache[1].here())
                                  : prepare(k_sym1_agg<false>, k1NT, 0, occ_cache[0].here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), 1u);
        if (sorted_in)
            LAPLEX_TIMED("sym_agg", stream, k_sym1_agg<true><<<grid, k1NT, 0, stream>>>(a, v, st, vs));
        else
            LAPLEX_TIMED("sym_agg", stream, k_sym1_agg<false><<<grid, k1NT, 0, stream>>>(a, v, st, vs));
    } else {
        using SM = AggSmem<C, kAheadAgg>;
        static PerDevice occ_cache;
        const int occ = prepare(k_sym_agg<C, kAheadAgg>, SymGeo<C>::NT, sizeof(SM), occ_cache.here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), (unsigned)p.G);
        LAPLEX_TIMED("sym_agg", stream,
                     k_sym_agg<C, kAheadAgg><<<grid, SymGeo<C>::NT, sizeof(SM), stream>>>(a, v, st, vs));
    }
    const SymScan a = scan_args(p, s, perm, n, B, sms, 1);
    LAPLEX_TIMED("sym_carry", stream,
                 k_sym_carry_direct<C><<<dim3((unsigned)p.P, (unsigned)p.G), kDirNT, 0, stream>>>(a, st));
    return cudaGetLastError();
}

#define LAPLEX_TRY_SYM(expr)                 \
    do {                                     \
        cudaError_t e_ = (expr);             \
        if (e_ != cudaSuccess) return e_;    \
    } while (0)

// The forward sweep (y from the sorted copy, RS and the range carries).
template <int C>
cudaError_t launch_sym_sweep_fwd(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, int64_t B, int sms,
                                 const float* xs, const RangeState& sx, float* y, cudaStream_t st,
                                 void* ws = nullptr) {
    if constexpr (C == 1) {
        static PerDevice occ_cache[2];
        const bool bucketed = p.bucketed && ws != nullptr;
        const int occ = bucketed ? prepare(k_sym1_sweep<1, true>, k1NT, 0, occ_cache[1].here())
                                 : prepare(k_sym1_sweep<1, false>, k1NT, 0, occ_cache[0].here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), 1u);
        if (bucketed) {
            float* ys = unperm_outputs(p, ws);
            LAPLEX_TIMED("sym_fwd", st,
                         k_sym1_sweep<1, true><<<grid, k1NT, 0, st>>>(a, xs, nullptr, sx, sx, ys, nullptr));
            return launch_unpermute(perm, ys, n, y, unperm_scratch(p, ws, n), st);
        }
        LAPLEX_TIMED("sym_fwd", st, k_sym1_sweep<1, false><<<grid, k1NT, 0, st>>>(a, xs, nullptr, sx, sx, y, nullptr));
    } else {
        using SM = SweepSmem<C, 1, kAheadFwd>;
        static PerDevice occ_cache;
        const int occ = prepare(k_sym_sweep<C, 1, kAheadFwd>, SymGeo<C>::NT, sizeof(SM), occ_cache.here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), (unsigned)p.G);
        LAPLEX_TIMED("sym_fwd", st,
                     k_sym_sweep<C, 1, kAheadFwd>
                     <<<grid, SymGeo<C>::NT, sizeof(SM), st>>>(a, xs, nullptr, sx, sx, y, nullptr, 0));
    }
    return cudaGetLastError();
}

// One channel past 2^24 rows: v enters the sorted copy vs through the inverse
// permutation, vs[inv[i]] = v[i] (a bucketed placement that reads v in order,
// instead of one random 4-byte gather per row); the rows of the last tile past n
// are zeroed, as the gathering pass would have written them.
cudaError_t place_sorted1(const SymPlan& p, const uint32_t* inv, int64_t n, const float* v, float* vs, void* ws,
                          cudaStream_t st) {
    cudaError_t e = launch_place(inv, v, n, vs, unperm_scratch(p, ws, n), place_scratch(p, ws, n), st);
    if (e != cudaSuccess) return e;
    const int64_t padded = p.T * p.R;
    if (padded > n) e = cudaMemsetAsync(vs + n, 0, sizeof(float) * (size_t)(padded - n), st);
    return e;
}

template <int C>
cudaError_t sym_forward_t(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B, float* y,
                          void* saved, void* ws, cudaStream_t st) {
    const int sms = device_sms();
    const SymPlan p = plan_sym(n, B, sms);
    RangeState sx = carve(p, (double2*)ws, true);
    float* xs = (float*)((char*)ws + 2 * p.state_bytes);
    if (saved != nullptr) {  // RS, carries and the sorted copy go to the caller's buffer
        const RangeState sv = carve(p, (double2*)saved, false);
        sx.RS = sv.RS;
        sx.Lin = sv.Lin;
        sx.Rin = sv.Rin;
        xs = (float*)((char*)saved + p.saved_state_bytes);
    }
    cudaError_t e;
    if (C == 1 && p.bucketed) {
        // the inverse permutation (kept with the saved state for the backward), then
        // x placed into sorted order
        uint32_t* inv = inv_slot(p, ws, saved, n);
        e = launch_inverse_perm(perm, n, inv, unperm_scratch(p, ws, n), place_scratch(p, ws, n), st);
        if (e == cudaSuccess) e = place_sorted1(p, inv, n, x, xs, ws, st);
        if (e == cudaSuccess) e = sym_ranges_t<C>(p, s, perm, n, B, sms, x, sx, xs, st, true);
    } else {
        e = sym_ranges_t<C>(p, s, perm, n, B, sms, x, sx, xs, st);
    }
    if (e != cudaSuccess) return e;
    return launch_sym_sweep_fwd<C>(p, s, perm, n, B, sms, xs, sx, y, st, ws);
}

template <int C>
cudaError_t sym_backward_t(const float* s, const uint32_t* perm, int64_t n, const float* x, const float* g, int64_t B,
                           const void* saved, float* gx, float* ga, void* ws, cudaStream_t st) {
    const int sms = device_sms();
    const SymPlan p = plan_sym(n, B, sms);
    RangeState sx = carve(p, (double2*)ws, true);
    const RangeState sg = carve(p, (double2*)((char*)ws + p.state_bytes), true);
    float* xs = (float*)((char*)ws + 2 * p.state_bytes);
    float* gs = (float*)((char*)xs + p.sorted_bytes);
    if (saved != nullptr) {
        const RangeState sv = carve(p, (double2*)saved, false);
        sx.RS = sv.RS;
        sx.Lin = sv.Lin;
        sx.Rin = sv.Rin;
        xs = (float*)((char*)saved + p.saved_state_bytes);
    }
    cudaError_t e;
    if (ga != nullptr && p.G > 1) {
        e = cudaMemsetAsync(ga, 0, sizeof(float) * n, st);
        if (e != cudaSuccess) return e;
    }
    if (C == 1 && p.bucketed) {
        // the forward's inverse permutation (saved), or a new one; x (without a saved
        // buffer) and g placed into sorted order
        uint32_t* inv = inv_slot(p, ws, const_cast<void*>(saved), n);
        if (saved == nullptr) {
            e = launch_inverse_perm(perm, n, inv, unperm_scratch(p, ws, n), place_scratch(p, ws, n), st);
            if (e == cudaSuccess) e = place_sorted1(p, inv, n, x, xs, ws, st);
            if (e == cudaSuccess) e = sym_ranges_t<C>(p, s, perm, n, B, sms, x, sx, xs, st, true);
            if (e != cudaSuccess) return e;
        }
        e = place_sorted1(p, inv, n, g, gs, ws, st);
        if (e == cudaSuccess) e = sym_ranges_t<C>(p, s, perm, n, B, sms, g, sg, gs, st, true);
        if (e != cudaSuccess) return e;
    } else {
        if (saved == nullptr) {
            e = sym_ranges_t<C>(p, s, perm, n, B, sms, x, sx, xs, st);
            if (e != cudaSuccess) return e;
        }
        e = sym_ranges_t<C>(p, s, perm, n, B, sms, g, sg, gs, st);
        if (e != cudaSuccess) return e;
    }
    if constexpr (C == 1) {
        static PerDevice occ_cache[2];
        const int occ = p.bucketed ? prepare(k_sym1_sweep<2, true>, k1NT, 0, occ_cache[1].here())
                                   : prepare(k_sym1_sweep<2, false>, k1NT, 0, occ_cache[0].here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), 1u);
        float* gxs = p.bucketed && gx ? unperm_outputs(p, ws) : gx;
        float* gas = p.bucketed && ga ? unperm_outputs(p, ws) + align_up((size_t)n, 64) : ga;
        if (p.bucketed)
            LAPLEX_TIMED("sym_bwd", st, k_sym1_sweep<2, true><<<grid, k1NT, 0, st>>>(a, xs, gs, sx, sg, gxs, gas));
        else
            LAPLEX_TIMED("sym_bwd", st, k_sym1_sweep<2, false><<<grid, k1NT, 0, st>>>(a, xs, gs, sx, sg, gxs, gas));
        if (p.bucketed) {
            void* scratch = unperm_scratch(p, ws, n);
            if (gx && ga)  // both through one placement (the sorted copy of g is free by now)
                LAPLEX_TRY_SYM(launch_unpermute2(perm, gxs, gas, n, gx, ga, gs, scratch, st));
            else if (gx)
                LAPLEX_TRY_SYM(launch_unpermute(perm, gxs, n, gx, scratch, st));
            else if (ga)
                LAPLEX_TRY_SYM(launch_unpermute(perm, gas, n, ga, scratch, st));
        }
    } else {
        using SM = SweepSmem<C, 2, kAheadBwd>;
        static PerDevice occ_cache;
        const int occ = prepare(k_sym_sweep<C, 2, kAheadBwd>, SymGeo<C>::NT, sizeof(SM), occ_cache.here());
        const SymScan a = scan_args(p, s, perm, n, B, sms, occ);
        const dim3 grid((unsigned)((p.P + a.m - 1) / a.m), (unsigned)p.G);
        LAPLEX_TIMED("sym_bwd", st,
                     k_sym_sweep<C, 2, kAheadBwd>
                     <<<grid, SymGeo<C>::NT, sizeof(SM), st>>>(a, xs, gs, sx, sg, gx, ga, p.G > 1 ? 1 : 0));
    }
    return cudaGetLastError();
}

}  // namespace

size_t sym_workspace_bytes(int64_t n, int64_t B) { return plan_sym(n, B, 1).total; }

size_t sym_saved_bytes(int64_t n, int64_t B) {
    const SymPlan p = plan_sym(n, B, 1);
    return p.saved_state_bytes + p.sorted_bytes + p.inv_bytes;
}

#define LAPLEX_SYM_DISPATCH(C_, CALL) \
    switch (C_) {                     \
        case 1: return CALL(1);       \
        case 2: return CALL(2);       \
        case 4: return CALL(4);       \
        case 8: return CALL(8);       \
        case 16: return CALL(16);     \
        default: return CALL(32);     \
    }

cudaError_t launch_sym_forward(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B, float* y,
                               void* saved, void* ws, int32_t* status, cudaStream_t st) {
    (void)status;  // no kernel of this path waits on another CTA
#define CALL(C) sym_forward_t<C>(s, perm, n, x, B, y, saved, ws, st)
    LAPLEX_SYM_DISPATCH(choose_channels(B), CALL)
#undef CALL
}

cudaError_t launch_sym_backward(const float* s, const uint32_t* perm, int64_t n, const float* x, const float* g,
                                int64_t B, const void* saved, float* gx, float* ga, void* ws, int32_t* status,
                                cudaStream_t st) {
    (void)status;
#define CALL(C) sym_backward_t<C>(s, perm, n, x, g, B, saved, gx, ga, ws, st)
    LAPLEX_SYM_DISPATCH(choose_channels(B), CALL)
#undef CALL
}

// ------------------------------------------------------- static-scratch forward

// Scratch of laplex_apply_sym_noalloc: part of the library's static device
// memory (one copy per device, created with the module), so that entry point
// takes no workspace and allocates nothing.  LAPLEX_NOALLOC_SCRATCH_BYTES covers
// every problem with n * sym_padded_batch(B) <= LAPLEX_NOALLOC_MAX_ELEMS on a GPU
// of up to about 300 SMs (the range arrays grow with the SM count);
// sym_noalloc_fits checks the actual plan on the current device before any launch.
// Nothing in it has to start at zero: every word the kernels read is written
// earlier in the same call.  Calls whose work overlaps on one device (two
// streams, or two host threads) share the array and corrupt each other.
static __device__ __align__(256) unsigned char g_sym_scratch[LAPLEX_NOALLOC_SCRATCH_BYTES];

namespace {

// The device address of g_sym_scratch belongs to the CUDA context that loaded the
// module: a new context on the same device (after cudaDeviceReset, or another
// context made current) loads the module again, possibly elsewhere.  The address
// is therefore cached per device together with the unique id of the context it
// was looked up in, and looked up again when the current context's id differs.
// The context calls come from the driver through the runtime's entry-point query,
// so the library needs no link to the driver library.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchCache {
    unsigned long long ctx_id = 0;  // 0: nothing cached (context ids start at 1)
    void* ptr = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
ScratchCache g_scratch[kMaxDevices];
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;

cudaError_t current_context_id(unsigned long long* id) {
    if (g_ctx_current == nullptr || g_ctx_id == nullptr) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1);
        if (e == cudaSuccess) e = cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2);
        if (e != cudaSuccess) return e;
        if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return cudaErrorNotSupported;
        g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    if (g_ctx_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// Device address of g_sym_scratch in the current context, looked up the first
// time a context is used on a device (the only setup step; later calls in the same
// context reuse it).
cudaError_t sym_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    e = cudaFree(nullptr);  // makes the device's primary context current (allocates nothing)
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    unsigned long long id = 0;
    e = current_context_id(&id);
    if (e != cudaSuccess) return e;
    ScratchCache& c = g_scratch[dev];
    if (c.ptr == nullptr || c.ctx_id != id) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_sym_scratch);
        if (e != cudaSuccess) return e;
        c.ptr = p;
        c.ctx_id = id;
    }
    *out = c.ptr;
    return cudaSuccess;
}

// Plan of the static-scratch forward: the plan of sym_forward_t with the range
// arrays sized for this device's ranges only and no saved state; the bytes it
// carves from g_sym_scratch.
SymPlan plan_sym_static(int64_t n, int64_t B, int sms, size_t* state_bytes) {
    SymPlan p = plan_sym(n, B, sms);
    p.rng_elems = (size_t)p.G * p.P * p.C;
    *state_bytes = align_up(sizeof(double2) * (p.rs_elems + 4 * p.rng_elems), 256);
    return p;
}

template <int C>
cudaError_t sym_forward_static_t(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B, float* y,
                                 cudaStream_t st) {
    void* scratch = nullptr;
    cudaError_t e = sym_scratch(&scratch);
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    size_t state = 0;
    const SymPlan p = plan_sym_static(n, B, sms, &state);
    // checked before the call by sym_noalloc_fits; kept as a guard
    if (state + p.sorted_bytes > (size_t)LAPLEX_NOALLOC_SCRATCH_BYTES) return cudaErrorInvalidValue;
    const RangeState sx = carve(p, (double2*)scratch, true);
    float* xs = (float*)((char*)scratch + state);
    e = sym_ranges_t<C>(p, s, perm, n, B, sms, x, sx, xs, st);
    if (e != cudaSuccess) return e;
    return launch_sym_sweep_fwd<C>(p, s, perm, n, B, sms, xs, sx, y, st);
}

}  // namespace

int64_t sym_padded_batch(int64_t B) {
    const int64_t C = choose_channels(B);
    return (B + C - 1) / C * C;
}

bool sym_noalloc_fits(int64_t n, int64_t B) {
    if (n > LAPLEX_NOALLOC_MAX_ELEMS / sym_padded_batch(B)) return false;
    size_t state = 0;
    const SymPlan p = plan_sym_static(n, B, device_sms(), &state);
    return state + p.sorted_bytes <= (size_t)LAPLEX_NOALLOC_SCRATCH_BYTES;
}

cudaError_t launch_sym_forward_noalloc(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B,
                                       float* y, int32_t* status, cudaStream_t st) {
    (void)status;
#define CALL(C) sym_forward_static_t<C>(s, perm, n, x, B, y, st)
    LAPLEX_SYM_DISPATCH(choose_channels(B), CALL)
#undef CALL
}

}  // namespace laplex
