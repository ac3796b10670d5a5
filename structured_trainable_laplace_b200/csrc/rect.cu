// Rectangular LAPLEX operators: out = E(O, I) x with E_ij = exp(-|o_i - q_j|),
// optionally times cos(theta_O,i - theta_I,j), their backward, and the Gram apply
// ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary sections
// 2.1 and 2.2: "general case a != b", the phased operator, "Gram operators").
//
// O is the output anchor set, I the input anchor set, both sorted.  The product
// is one scan over the merged sorted sequence of O and I: the state just left
// of an output o is the prefix over the inputs q <= o, the state right of it the
// suffix over q > o, and out(o) = prefix + suffix.  It is evaluated in whichever
// of two ways keeps the scan on the SMALLER side:
//   expand (|I| <= |O|): scan the inputs over sorted I (prefix P and suffix S per
//       input row), then every output reads the states of its two neighbours in
//       I:  out(o) = exp(q_(m'-1) - o) P_(m'-1) + exp(o - q_(m')) S_(m'),
//       m' = number of inputs <= o.
//   reduce (|I| > |O|): sum every input into the interval of sorted O it falls
//       in -- u (strictly left of the next output, weighted to it), v (strictly
//       right of the previous output, weighted to it) and ties t -- then carry
//       the interval sums across O with the same scan and read out = P + R.
// The phased operator runs as the cos/sin split cos(tO) cos(tI) + sin(tO) sin(tI):
// 2B scan channels (cos part, then sin part) per B input channels.
//
// Kernels:
//   k_side_totals / k_side_apply  scan over the small side of up to 1024 tiles
//       with no wait between CTAs (tile totals, then per tile direct weighted
//       sums of the other tiles' totals and the tile's evaluation); inputs:
//       gathered rows x phase weights, or fp64 interval sums; outputs: per-row
//       states (P, S) or parts (strict L, strict R, full).
//   k_side_right / k_side_left  the same scan for larger small sides, by bounded
//       decoupled lookback.
//   k_large  one streaming pass over the large side: interval sums into fp64
//       bins (reduce), neighbour lookups (expand), and the fused anchor / phase
//       gradients of that side.
//   k_finish  per small-side row: combine the cos/sin parts into outputs and
//       gradients.
//   k_gram_mid_sorted / k_gram_mid2  the middle of the Gram apply and backward
//       (D w, D u, gD) between its two rectangular products.
#include "laplex_internal.h"
#include "pipeline.cuh"

namespace laplex {

namespace {

constexpr int kTileValues = 4096;
constexpr int kSideNT = 512;
constexpr int kSideE = kTileValues / kSideNT;

// ------------------------------------------------------------------ side scan

struct SideScan {
    const float* s;        // sorted anchors [m]
    const uint32_t* perm;  // gather index of sorted row r (values mode)
    const float* theta;    // phases, original order (values mode), or nullptr
    int64_t m;
    const float* X;  // values mode: rows [m][B], original order
    int B;
    int Cb;            // scan channels: B, or 2B when phased
    const double* U;   // bins mode: strict-left interval sums   [m][Cb]
    const double* TL;  //            ties, at the first row of a tie run
    const double* V;   //            strict-right interval sums
    const double* TR;  //            ties, at the last row of a tie run
    float* o0;         // values mode: P (inclusive prefix); bins mode: strict L
    float* o1;         // values mode: S (inclusive suffix); bins mode: strict R
    float* o2;         // bins mode: full = P + R
    int64_t T;
};

template <int R>
__device__ __forceinline__ void side_meta(const SideScan& a, int64_t lo, float* s_sm, uint32_t* p_sm, float* cw,
                                          float* sw, bool bins, bool phase_smem) {
    for (int i = threadIdx.x; i < R + 2; i += blockDim.x) {
        const int64_t r = lo - 1 + i;
        s_sm[i] = (r < 0) ? kLowAnchor : (r < a.m ? __ldg(a.s + r) : kHighAnchor);
    }
    if (!bins)
        for (int i = threadIdx.x; i < R; i += blockDim.x) {
            const int64_t r = lo + i;
            const uint32_t src = (r < a.m) ? min(a.perm ? __ldg(a.perm + r) : (uint32_t)r, (uint32_t)(a.m - 1)) : 0u;
            p_sm[i] = src;
            if (a.theta != nullptr && phase_smem) {
                float sn = 0.f, cs = 1.f;
                if (r < a.m) sincosf(__ldg(a.theta + src), &sn, &cs);
                cw[i] = cs;
                sw[i] = sn;
            }
        }
}

// Inputs of row r (tile-local), channel cb: left (l, t), right (rr, tp).
template <bool BINS>
__device__ __forceinline__ void side_inputs(const SideScan& a, int64_t lo, int r, int cb, const uint32_t* p_sm,
                                            const float* cw, const float* sw, float& l, float& t, float& rr,
                                            float& tp) {
    l = t = rr = tp = 0.f;
    if (lo + r >= a.m || cb >= a.Cb) return;
    if (BINS) {
        const int64_t idx = (lo + r) * (int64_t)a.Cb + cb;
        l = (float)__ldcg(a.U + idx);
        t = (float)__ldcg(a.TL + idx);
        rr = (float)__ldcg(a.V + idx);
        tp = (float)__ldcg(a.TR + idx);
    } else {
        const int part = cb / a.B, c = cb - part * a.B;
        float v = __ldg(a.X + (int64_t)p_sm[r] * a.B + c);
        if (a.theta != nullptr) v *= part ? sw[r] : cw[r];
        t = tp = v;
    }
}

template <int C, bool BINS>
__global__ void __launch_bounds__(kSideNT) k_side_right(SideScan a, ChainSet cs, unsigned* counters,
                                                        int32_t* status) {
    constexpr int NT = kSideNT, E = kSideE, R = kTileValues / C;
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[BINS ? 1 : R];
    // phases need two scan channels per input channel, so C == 1 never carries them
    __shared__ float cw[(BINS || C == 1) ? 1 : R], sw[(BINS || C == 1) ? 1 : R];
    __shared__ ScanSmem<C, NT / 32> sm;
    __shared__ LookbackSmem<C, NT> lb;
    __shared__ int64_t s_tile;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = a.T - 1 - (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    side_meta<R>(a, lo, s_sm, p_sm, cw, sw, BINS, !(BINS || C == 1));
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int cb = grp * C + c;
    float rin[E], tin[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        float l, tt;
        side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, l, tt, rin[e], tin[e]);
    }
    LP st = {0.f, 0.f};
    float up = -s_sm[(k + 1) * E + 1];
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, rin[e], tin[e]);
        up = u;
    }
    LP excl;
    bool has;
    block_scan_dir<C, NT, true>(st, -s_sm[k * E + 1], -s_sm[(k + 1) * E + 1], sm, excl, has);
    bool hc;
    const LP tot = threadIdx.x < C ? sm.tot[threadIdx.x] : LP{0.f, 0.f};
    (void)block_lookback<C, true, NT>(cs.chain(grp), t, a.T, a.s, a.m, R, tot, -s_sm[1], -s_sm[R + 1], status, lb, hc);
}

// The inputs are read twice (the summaries, then the final sweeps; the second
// read hits L2) so that none is held through the lookback: two CTAs fit per SM.
template <int C, bool BINS>
__global__ void __launch_bounds__(kSideNT, 2) k_side_left(SideScan a, ChainSet left, ChainSet right,
                                                          unsigned* counters, int32_t* status) {
    constexpr int NT = kSideNT, E = kSideE, R = kTileValues / C;
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[BINS ? 1 : R];
    __shared__ float cw[(BINS || C == 1) ? 1 : R], sw[(BINS || C == 1) ? 1 : R];
    __shared__ ScanSmem<C, NT / 32> smL, smR;
    __shared__ LookbackSmem<C, NT> lb;
    __shared__ int64_t s_tile;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int cb = grp * C + c;
    // the right scan's inclusive state of the next tile (written by the previous launch)
    const bool hasr = (t + 1 < a.T);
    const double2 crd = hasr ? __ldcg(&right.chain(grp).inc[(t + 1) * C + c]) : make_double2(0.0, 0.0);
    side_meta<R>(a, lo, s_sm, p_sm, cw, sw, BINS, !(BINS || C == 1));
    __syncthreads();
    const float ub_r = -s_sm[(k + 1) * E + 1];
    const float ub_l = s_sm[k * E];
    LP str = {0.f, 0.f}, stl = {0.f, 0.f};
    {
        float lin[E], tin[E], rin[E], tpin[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, lin[e], tin[e], rin[e], tpin[e]);
        float up = ub_r;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) {
            const float u = -s_sm[k * E + e + 1];
            str = lp_step(str, up, u, rin[e], tpin[e]);
            up = u;
        }
        up = ub_l;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float u = s_sm[k * E + e + 1];
            stl = lp_step(stl, up, u, lin[e], tin[e]);
            up = u;
        }
    }
    LP exr, exl;
    bool hr, hl;
    block_scan_dir<C, NT, true>(str, -s_sm[k * E + 1], ub_r, smR, exr, hr);
    block_scan_dir<C, NT, false>(stl, s_sm[k * E + E], ub_l, smL, exl, hl);
    bool hcl;
    const LP tot = threadIdx.x < C ? smL.tot[threadIdx.x] : LP{0.f, 0.f};
    const double2 cin =
        block_lookback<C, false, NT>(left.chain(grp), t, a.T, a.s, a.m, R, tot, s_sm[R], s_sm[0], status, lb, hcl);
    const LP cl = {(float)cin.x, (float)cin.y};
    const LP left_in = seg_incoming(hcl, cl, s_sm[0], hl, exl, ub_l);
    const LP cr = {(float)crd.x, (float)crd.y};
    const LP right_in = seg_incoming(hasr, cr, -s_sm[R + 1], hr, exr, ub_r);
    float rres[E];  // values: S; bins: strict R
    LP st = right_in;
    float up = ub_r;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        float l, tt, r, tp;
        side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, l, tt, r, tp);
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, r, tp);
        rres[e] = BINS ? st.L : st.P;
        up = u;
    }
    st = left_in;
    up = ub_l;
    const bool cval = cb < a.Cb;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        float l, tt, rr, tp;
        side_inputs<BINS>(a, lo, r, cb, p_sm, cw, sw, l, tt, rr, tp);
        const float u = s_sm[r + 1];
        st = lp_step(st, up, u, l, tt);
        up = u;
        if (cval && lo + r < a.m) {
            const int64_t idx = (lo + r) * (int64_t)a.Cb + cb;
            if (BINS) {
                a.o0[idx] = st.L;
                a.o1[idx] = rres[e];
                a.o2[idx] = st.P + rres[e];
            } else {
                a.o0[idx] = st.P;
                a.o1[idx] = rres[e];
            }
        }
    }
}

// ---------------------------------------------- side scan without waits (T small)
//
// When the small side has few tiles the scan runs as two launches with no wait
// between CTAs: k_side_totals writes each tile's totals in both directions
// (chain agg arrays), and k_side_apply gives each tile its incoming states
// directly as sums over all its predecessors' / successors' totals, every term
// weighted straight to the tile's boundary anchor (the sum form of the
// recurrence, as in the lookback), then evaluates the tile.  Each apply CTA reads
// (T - 1) * C totals, so the form is used while T * C stays small.
constexpr int64_t kSideDirectMaxTiles = 1024;
constexpr int64_t kSideDirectMaxValues = 8192;  // T * C

template <int C, bool BINS>
__global__ void __launch_bounds__(kSideNT, 2) k_side_totals(SideScan a, ChainSet left, ChainSet right) {
    constexpr int NT = kSideNT, E = kSideE, R = kTileValues / C;
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[BINS ? 1 : R];
    __shared__ float cw[(BINS || C == 1) ? 1 : R], sw[(BINS || C == 1) ? 1 : R];
    __shared__ ScanSmem<C, NT / 32> smL, smR;
    const int grp = blockIdx.y;
    const int64_t t = blockIdx.x, lo = t * R;
    side_meta<R>(a, lo, s_sm, p_sm, cw, sw, BINS, !(BINS || C == 1));
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int cb = grp * C + c;
    const float ub_r = -s_sm[(k + 1) * E + 1];
    const float ub_l = s_sm[k * E];
    LP str = {0.f, 0.f}, stl = {0.f, 0.f};
    {
        float lin[E], tin[E], rin[E], tpin[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, lin[e], tin[e], rin[e], tpin[e]);
        float up = ub_r;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) {
            const float u = -s_sm[k * E + e + 1];
            str = lp_step(str, up, u, rin[e], tpin[e]);
            up = u;
        }
        up = ub_l;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float u = s_sm[k * E + e + 1];
            stl = lp_step(stl, up, u, lin[e], tin[e]);
            up = u;
        }
    }
    LP exr, exl;
    bool hr, hl;
    block_scan_dir<C, NT, true>(str, -s_sm[k * E + 1], ub_r, smR, exr, hr);
    block_scan_dir<C, NT, false>(stl, s_sm[k * E + E], ub_l, smL, exl, hl);
    if (threadIdx.x < C) {
        const LP tl = smL.tot[threadIdx.x], tr = smR.tot[threadIdx.x];
        left.chain(grp).agg[t * C + threadIdx.x] = make_double2((double)tl.L, (double)tl.P);
        right.chain(grp).agg[t * C + threadIdx.x] = make_double2((double)tr.L, (double)tr.P);
    }
}

// Shared scratch of the direct carries: per other tile its fp64 weight and
// whether its end lies strictly before the anchor, then the per-warp sums.
template <int C, int NT>
struct DirectSmem {
    double e[kSideDirectMaxTiles];
    bool brk[kSideDirectMaxTiles];
    double2 part[2][NT / 32][C];
    double2 carry[2][C];
};

// Incoming states of tile t (every thread of the block): left = sum over tiles
// j < t of their left totals weighted to the row before the tile, right = sum over
// j > t of their right totals weighted to -(the row after the tile).  A term with
// decay 1 (its end tied with the anchor) adds its strict part L to L, every other
// term adds e P to both.  Returns channel tid % C's carries.
template <int C, int NT>
__device__ __forceinline__ void direct_carries(const SideScan& a, Chain left, Chain right, int64_t t, int64_t R,
                                               float u_left, float u_right, DirectSmem<C, NT>& sm, double2& cl,
                                               double2& cr) {
    const int64_t T = a.T;
    const int tid = threadIdx.x, c = tid % C, g = tid / C;
    constexpr int SG = NT / C;
    // slot i in [0, T - 1) is tile j = i (< t: left) or i + 1 (> t: right)
    for (int64_t i = tid; i < T - 1; i += NT) {
        const int64_t j = i < t ? i : i + 1;
        const bool isl = j < t;
        const float uj = isl ? __ldg(a.s + min(a.m, (j + 1) * R) - 1) : -__ldg(a.s + j * R);
        const float ub = isl ? u_left : u_right;
        const bool brk = ub > uj;
        sm.e[i] = brk ? exp((double)uj - (double)ub) : 1.0;
        sm.brk[i] = brk;
    }
    __syncthreads();
    double2 pl = make_double2(0.0, 0.0), pr = make_double2(0.0, 0.0);
#pragma unroll 4
    for (int64_t i = g; i < T - 1; i += SG) {
        const double e = sm.e[i];
        if (e == 0.0) continue;  // underflowed: the tile adds nothing
        const int64_t j = i < t ? i : i + 1;
        const bool isl = j < t;
        const double2 v = __ldcg(&(isl ? left : right).agg[j * C + c]);
        double2& acc = isl ? pl : pr;
        acc.y = fma(e, v.y, acc.y);
        acc.x = sm.brk[i] ? fma(e, v.y, acc.x) : acc.x + v.x;
    }
#pragma unroll
    for (int off = C; off < 32; off <<= 1) {
        pl.x += __shfl_xor_sync(0xffffffffu, pl.x, off);
        pl.y += __shfl_xor_sync(0xffffffffu, pl.y, off);
        pr.x += __shfl_xor_sync(0xffffffffu, pr.x, off);
        pr.y += __shfl_xor_sync(0xffffffffu, pr.y, off);
    }
    if ((tid & 31) < C) {
        sm.part[0][tid >> 5][tid & 31] = pl;
        sm.part[1][tid >> 5][tid & 31] = pr;
    }
    __syncthreads();
    if (tid < 2 * C) {
        const int d = tid / C, cc = tid % C;
        double2 r = make_double2(0.0, 0.0);
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) {
            r.x += sm.part[d][w][cc].x;
            r.y += sm.part[d][w][cc].y;
        }
        sm.carry[d][cc] = r;
    }
    __syncthreads();
    cl = sm.carry[0][c];
    cr = sm.carry[1][c];
}

template <int C, bool BINS>
__global__ void __launch_bounds__(kSideNT, 2) k_side_apply(SideScan a, ChainSet left, ChainSet right) {
    constexpr int NT = kSideNT, E = kSideE, R = kTileValues / C;
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[BINS ? 1 : R];
    __shared__ float cw[(BINS || C == 1) ? 1 : R], sw[(BINS || C == 1) ? 1 : R];
    __shared__ ScanSmem<C, NT / 32> smL, smR;
    __shared__ DirectSmem<C, NT> dsm;
    const int grp = blockIdx.y;
    const int64_t t = blockIdx.x, lo = t * R;
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int cb = grp * C + c;
    const bool hasl = t > 0, hasr = t + 1 < a.T;
    side_meta<R>(a, lo, s_sm, p_sm, cw, sw, BINS, !(BINS || C == 1));
    __syncthreads();
    double2 cld, crd;
    direct_carries<C, NT>(a, left.chain(grp), right.chain(grp), t, R, s_sm[0], -s_sm[R + 1], dsm, cld, crd);
    const float ub_r = -s_sm[(k + 1) * E + 1];
    const float ub_l = s_sm[k * E];
    LP str = {0.f, 0.f}, stl = {0.f, 0.f};
    {
        float lin[E], tin[E], rin[E], tpin[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, lin[e], tin[e], rin[e], tpin[e]);
        float up = ub_r;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) {
            const float u = -s_sm[k * E + e + 1];
            str = lp_step(str, up, u, rin[e], tpin[e]);
            up = u;
        }
        up = ub_l;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float u = s_sm[k * E + e + 1];
            stl = lp_step(stl, up, u, lin[e], tin[e]);
            up = u;
        }
    }
    LP exr, exl;
    bool hr, hl;
    block_scan_dir<C, NT, true>(str, -s_sm[k * E + 1], ub_r, smR, exr, hr);
    block_scan_dir<C, NT, false>(stl, s_sm[k * E + E], ub_l, smL, exl, hl);
    const LP left_in = seg_incoming(hasl, LP{(float)cld.x, (float)cld.y}, s_sm[0], hl, exl, ub_l);
    const LP right_in = seg_incoming(hasr, LP{(float)crd.x, (float)crd.y}, -s_sm[R + 1], hr, exr, ub_r);
    float rres[E];  // values: S; bins: strict R
    LP st = right_in;
    float up = ub_r;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        float l, tt, r, tp;
        side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, l, tt, r, tp);
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, r, tp);
        rres[e] = BINS ? st.L : st.P;
        up = u;
    }
    st = left_in;
    up = ub_l;
    const bool cval = cb < a.Cb;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        float l, tt, rr, tp;
        side_inputs<BINS>(a, lo, r, cb, p_sm, cw, sw, l, tt, rr, tp);
        const float u = s_sm[r + 1];
        st = lp_step(st, up, u, l, tt);
        up = u;
        if (cval && lo + r < a.m) {
            const int64_t idx = (lo + r) * (int64_t)a.Cb + cb;
            if (BINS) {
                a.o0[idx] = st.L;
                a.o1[idx] = rres[e];
                a.o2[idx] = st.P + rres[e];
            } else {
                a.o0[idx] = st.P;
                a.o1[idx] = rres[e];
            }
        }
    }
}

// ------------------------------------------------------------------ large pass

constexpr int kLmExpand = 1;  // write output rows from the small side's states
constexpr int kLmAccum = 2;   // sum the rows into the small side's interval bins
constexpr int kLmGrad = 4;    // anchor / phase gradients of the large side

struct LargePass {
    const float* s;  // large side, sorted anchors
    const uint32_t* perm;
    const float* theta;
    int64_t m;
    const float* sp;  // small side, sorted anchors
    int64_t ms;
    const float* rows;   // [m][Bs] original order: accumulated (accum) and h (grad)
    const float* rows2;  // nullptr, or the source of channels [Bs, B) ([m][Bs]) of a paired pass
    int Bs;              // row stride of rows / rows2: B, or B / 2 for a paired pass
    int B;
    int Cb;
    const float* Pst;  // small side states [ms][Cb]
    const float* Sst;
    double* U;  // small side bins [ms][Cb]
    double* TL;
    double* V;
    double* TR;
    float* out;  // [m][B] original order
    float* g_anchor;
    float* g_phase;
    int64_t rows_per_group;
    int lpr;
    int chunk_atomic;
    int accumulate;  // add the anchor / phase gradients into g_anchor / g_phase
};

__device__ __forceinline__ int64_t lower_bound_f(const float* a, int64_t n, float v) {
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(a + mid) < v)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

__device__ __forceinline__ int64_t upper_bound_f(const float* a, int64_t n, float v) {
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(a + mid) <= v)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

template <int VEC>
__device__ __forceinline__ void load_vec(const float* p, float (&v)[VEC]) {
    if (VEC == 4) {
        const float4 q = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = q.x;
        v[1] = q.y;
        v[2] = q.z;
        v[3] = q.w;
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) v[i] = __ldg(p + i);
    }
}

template <int VEC>
__device__ __forceinline__ void store_vec(float* p, const float (&v)[VEC]) {
    if (VEC == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) p[i] = v[i];
    }
}

// Rows per prefetch batch of k_large (gathered rows in flight per group).
template <int VEC, bool PHASED, int MODE>
constexpr int kLargeBatch = 8;

// Each group of `lpr` lanes walks a contiguous range of sorted large-side rows;
// lane gl of the group owns channels c0 .. c0+VEC-1 of every row.
template <int VEC, bool PHASED, int MODE>
__global__ void __launch_bounds__(256, 2) k_large(LargePass A) {
    constexpr int NP = PHASED ? 2 : 1;
    constexpr bool EXPAND = (MODE & kLmExpand) != 0;
    constexpr bool ACCUM = (MODE & kLmAccum) != 0;
    constexpr bool GRAD = (MODE & kLmGrad) != 0;
    constexpr bool STATES = EXPAND || GRAD;
    constexpr bool ROWS = ACCUM || GRAD;
    const int lane = threadIdx.x & 31;
    const int lpr = A.lpr;
    const int gl = lane & (lpr - 1);
    const unsigned gmask = (lpr == 32) ? 0xffffffffu : (((1u << lpr) - 1u) << (lane & ~(lpr - 1)));
    const int64_t gid = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * (32 / lpr) + lane / lpr;
    const int c0 = (blockIdx.y * lpr + gl) * VEC;
    const bool cval = c0 < A.B;
    const int64_t r0 = gid * A.rows_per_group;
    const int64_t r1 = min(A.m, r0 + A.rows_per_group);
    if (r0 >= r1) return;  // the whole group leaves together
    const int64_t ms = A.ms;
    const int B = A.B, Cb = A.Cb;

    int64_t m = lower_bound_f(A.sp, ms, __ldg(A.s + r0));
    int64_t mp = upper_bound_f(A.sp, ms, __ldg(A.s + r0));
    const int64_t m_first = m;
    const int64_t m_last = ACCUM ? lower_bound_f(A.sp, ms, __ldg(A.s + r1 - 1)) : 0;

    // interval sums of the current bin: fp32 for up to 16 rows, then folded into
    // fp64 partials kept in shared memory (slot i of thread t at [i][t]: touched
    // only at folds and flushes, so they cost no registers)
    constexpr int ND = ACCUM ? 2 * NP * VEC : 1;
    // dynamic shared memory: the fp64 partials [ND][256], then (wide groups in
    // modes that gather rows) the per-warp ring of two sub-batch slots
    extern __shared__ __align__(16) unsigned char large_smem[];
    double(*s_dacc)[256] = reinterpret_cast<double(*)[256]>(large_smem);
    float* s_rows = reinterpret_cast<float*>(large_smem + sizeof(double) * ND * 256);
    int64_t cur = m;
    float fu[NP][VEC], fv[NP][VEC];
    int cnt = 0;  // rows in the fp32 partials (wide groups: the same in every lane)
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int v = 0; v < VEC; ++v) fu[p][v] = fv[p][v] = 0.f;
#pragma unroll
    for (int i = 0; i < ND; ++i) s_dacc[i][threadIdx.x] = 0.0;
    auto du = [&](int p, int v) -> double& { return s_dacc[(p * VEC + v) % ND][threadIdx.x]; };
    auto dv = [&](int p, int v) -> double& { return s_dacc[(NP * VEC + p * VEC + v) % ND][threadIdx.x]; };

    auto fold = [&]() {
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                du(p, v) += (double)fu[p][v];
                dv(p, v) += (double)fv[p][v];
                fu[p][v] = fv[p][v] = 0.f;
            }
        cnt = 0;
    };
    auto flush = [&](int64_t bin) {
        fold();
        if (cval) {
            const bool owner = bin > m_first && bin < m_last;  // no other group touches this bin
#pragma unroll
            for (int p = 0; p < NP; ++p)
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const int ch = p * B + c0 + v;
                    const double su = du(p, v), sv = dv(p, v);
                    if (bin < ms) {
                        double* dst = A.U + bin * Cb + ch;
                        if (owner)
                            *dst = su;
                        else if (su != 0.0)
                            atomicAdd(dst, su);
                    }
                    if (bin >= 1) {
                        double* dst = A.V + (bin - 1) * Cb + ch;
                        if (owner)
                            *dst = sv;
                        else if (sv != 0.0)
                            atomicAdd(dst, sv);
                    }
                    du(p, v) = 0.0;
                    dv(p, v) = 0.0;
                }
        }
    };

    int64_t st_m = -1, st_mp = -1;
    float Pm1[NP][VEC], Pmp[NP][VEC], Smp[NP][VEC];

    constexpr int U = kLargeBatch<VEC, PHASED, MODE>;
    const bool wide = lpr >= U;  // group-uniform, and warp-uniform when wide
    // this lane's channels of gathered row pr (a paired pass takes channels past Bs
    // from the second source; Bs is a multiple of VEC, so no chunk straddles)
    auto row_src = [&](uint32_t pr) -> const float* {
        return (A.rows2 != nullptr && c0 >= A.Bs) ? A.rows2 + (int64_t)pr * A.Bs + (c0 - A.Bs)
                                                  : A.rows + (int64_t)pr * A.Bs + c0;
    };

    // One row: q's bins m (small-side anchors < q) and mp (<= q), the decays eL / eR
    // to the neighbouring small-side anchors, phase weights (w0, w1) = (cos, sin),
    // the gathered row h.  Returns the row's anchor / phase gradient shares of this
    // lane's channels in ga / gp.
    auto row = [&](uint32_t pr, float w0, float w1, float eL, float eR, int64_t mr, int64_t mpr, const float* h,
                   float& ga, float& gp) {
        const float w[2] = {w0, w1};
        const bool tie = mpr > mr;
        const float eLf = tie ? 1.f : eL;
        if (ACCUM) {
            if (mr != cur) {
                flush(cur);
                cur = mr;
            }
            if (!tie) {
                // untied rows feed the interval sums u (weighted to the right
                // neighbour) and v (to the left one)
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    const float wr = eR * w[p], wl = eL * w[p];
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        fu[p][v] = fmaf(wr, h[v], fu[p][v]);
                        fv[p][v] = fmaf(wl, h[v], fv[p][v]);
                    }
                }
            } else if (cval) {
                // a row tied with a run of small-side anchors enters that run only
                // (TL, TR); the neighbours beyond it receive it through the scan
#pragma unroll
                for (int p = 0; p < NP; ++p)
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        const double val = (double)(w[p] * h[v]);
                        atomicAdd(A.TL + mr * Cb + p * B + c0 + v, val);
                        atomicAdd(A.TR + (mpr - 1) * Cb + p * B + c0 + v, val);
                    }
            }
            if (wide && ++cnt == 16) fold();  // narrow groups fold on a fixed schedule instead
        }
        if (STATES) {
            if (mr != st_m || mpr != st_mp) {
#pragma unroll
                for (int p = 0; p < NP; ++p)
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        const int ch = p * B + c0 + v;
                        Pm1[p][v] = (GRAD && cval && mr > 0) ? __ldg(A.Pst + (mr - 1) * Cb + ch) : 0.f;
                        Pmp[p][v] = (cval && mpr > 0) ? __ldg(A.Pst + (mpr - 1) * Cb + ch) : 0.f;
                        Smp[p][v] = (cval && mpr < ms) ? __ldg(A.Sst + mpr * Cb + ch) : 0.f;
                    }
                st_m = mr;
                st_mp = mpr;
            }
            // out = sum_p w_p (eLf P_(mp-1) + eR S_mp); the strict left part of the
            // prefix is eL P_(m-1) (ties excluded)
            float fl[NP], fr[NP], dl[NP];
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                fl[p] = eLf * w[p];
                fr[p] = eR * w[p];
                dl[p] = eL * w[p];
            }
            float o[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                o[v] = 0.f;
                float t = 0.f;
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    o[v] = fmaf(fl[p], Pmp[p][v], fmaf(fr[p], Smp[p][v], o[v]));
                    if (GRAD) t = fmaf(fr[p], Smp[p][v], fmaf(-dl[p], Pm1[p][v], t));
                }
                if (GRAD) {
                    ga = fmaf(h[v], t, ga);  // strict right - strict left
                    if (PHASED) {
                        // d/dtheta of (cos, sin) is (-sin, cos)
                        const float f0 = fmaf(eLf, Pmp[0][v], eR * Smp[0][v]);
                        const float f1 = fmaf(eLf, Pmp[NP - 1][v], eR * Smp[NP - 1][v]);
                        gp = fmaf(h[v], fmaf(w0, f1, -w1 * f0), gp);
                    }
                }
            }
            if (EXPAND && A.out != nullptr && cval) store_vec<VEC>(A.out + (int64_t)pr * B + c0, o);
        }
    };
    auto put_grad = [&](float* dst, uint32_t pr, float v) {
        if (dst == nullptr) return;
        if (A.chunk_atomic)
            atomicAdd(dst + pr, v);
        else if (A.accumulate)
            dst[pr] += v;  // every row is visited once per launch
        else
            dst[pr] = v;
    };

    if (wide) {
        // Wide groups.  Rows are taken in batches of lpr: lane gl computes the
        // scalars of row rb + gl (permutation entry, phase weights, bins, decays),
        // so every row's scalar work is done once; the group then walks the batch in
        // sub-batches of U rows, taking each row's scalars from the lane that
        // computed them.  Bins are below 2^32.  The gathered rows go through a
        // per-warp ring of two sub-batch slots in shared memory: each lane copies
        // its own VEC floats of the next sub-batch's rows with cp.async while the
        // current one is processed (and reads back only what it copied, so no
        // warp barrier is needed).  The next batch's scalars are computed one
        // sub-batch early, from the bins reached so far (a lower bound).
        struct Scal {
            uint32_t pr, mm, mmp;
            float cs, sn, eL, eR;
        };
        auto batch_scalars = [&](int64_t rb, int nb, Scal& S) {
            const int64_t rme = rb + min(gl, nb - 1);
            const float q_me = __ldg(A.s + rme);
            S.pr = min(__ldg(A.perm + rme), (uint32_t)(A.m - 1));
            S.cs = 1.f;
            S.sn = 0.f;
            if (PHASED) sincosf(__ldg(A.theta + S.pr), &S.sn, &S.cs);
            int64_t mm = m;
            while (mm < ms && __ldg(A.sp + mm) < q_me) ++mm;
            int64_t mmp = max(mp, mm);
            while (mmp < ms && __ldg(A.sp + mmp) <= q_me) ++mmp;
            S.eL = (mm > 0) ? expf(__ldg(A.sp + mm - 1) - q_me) : 0.f;
            S.eR = (mmp < ms) ? expf(q_me - __ldg(A.sp + mmp)) : 0.f;
            S.mm = (uint32_t)mm;
            S.mmp = (uint32_t)mmp;
        };
        float* ring = s_rows + (threadIdx.x >> 5) * (2 * U * 32 * VEC) + lane * VEC;  // this lane's slots
        auto stage = [&](const Scal& S, int j, int nb, int slot) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t pr = __shfl_sync(gmask, S.pr, min(j + u, nb - 1), lpr);
                if (ROWS) {
                    float* dst = ring + (slot * U + u) * (32 * VEC);
                    if (cval) {
                        if constexpr (VEC == 4)
                            cp_async16(dst, row_src(pr));
                        else
                            cp_async4(dst, row_src(pr));
                    } else {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) dst[v] = 0.f;  // channels past B read as zero
                    }
                }
            }
            cp_async_commit();
        };
        Scal S;
        int slot = 0;
        batch_scalars(r0, (int)min((int64_t)lpr, r1 - r0), S);
        stage(S, 0, (int)min((int64_t)lpr, r1 - r0), 0);
        for (int64_t rb = r0; rb < r1; rb += lpr) {
            const int nb = (int)min((int64_t)lpr, r1 - rb);
            Scal Sn = S;
            for (int j = 0; j < nb; j += U) {
                if (j + U < nb) {
                    stage(S, j + U, nb, slot ^ 1);
                } else if (rb + lpr < r1) {
                    const int nbn = (int)min((int64_t)lpr, r1 - rb - lpr);
                    batch_scalars(rb + lpr, nbn, Sn);
                    stage(Sn, 0, nbn, slot ^ 1);
                } else {
                    cp_async_commit();  // keep one group per sub-batch
                }
                cp_async_wait<1>();  // this sub-batch's copies are in
                // the rows are read from the ring inside the row body
                const float* hrow0 = ring + slot * U * (32 * VEC);
                constexpr int hstep = 32 * VEC;
                const float cs_me = S.cs, sn_me = S.sn, eL_me = S.eL, eR_me = S.eR;
                const uint32_t mm32 = S.mm, mmp32 = S.mmp;
                float gpart[GRAD ? 2 * U : 1];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int src = min(j + u, nb - 1);
                    const float w0 = __shfl_sync(gmask, cs_me, src, lpr);
                    const float w1 = PHASED ? __shfl_sync(gmask, sn_me, src, lpr) : 0.f;
                    const float eL = __shfl_sync(gmask, eL_me, src, lpr);
                    const float eR = __shfl_sync(gmask, eR_me, src, lpr);
                    m = __shfl_sync(gmask, mm32, src, lpr);
                    mp = __shfl_sync(gmask, mmp32, src, lpr);
                    float ga = 0.f, gp = 0.f;
                    const uint32_t pru = __shfl_sync(gmask, S.pr, src, lpr);
                    if (j + u < nb) row(pru, w0, w1, eL, eR, m, mp, hrow0 + u * hstep, ga, gp);  // group-uniform
                    if (GRAD) {
                        gpart[u] = ga;
                        gpart[U + u] = gp;
                    }
                }
                if (GRAD) {
                    // sum the 2U partials over the group's lanes by recursive halving
                    // (halves fixed at compile time, the group width at run time);
                    // lane gl ends with the totals of value indices base .. base + vc - 1
                    constexpr int NV = 2 * U;
                    int vc = NV, base = 0, hl = 0;
#pragma unroll
                    for (int L = 0; (NV >> L) > 1; ++L) {
                        const int o = lpr >> (L + 1);
                        if (o >= 1) {
                            const bool upper = (gl & o) != 0;
#pragma unroll
                            for (int i = 0; i < (NV >> (L + 1)); ++i) {
                                const float keep = upper ? gpart[i + (NV >> (L + 1))] : gpart[i];
                                const float send = upper ? gpart[i] : gpart[i + (NV >> (L + 1))];
                                gpart[i] = keep + __shfl_xor_sync(gmask, send, o, lpr);
                            }
                            if (upper) base += NV >> (L + 1);
                            vc = NV >> (L + 1);
                            hl = L + 1;
                        }
                    }
                    // the remaining levels add whole totals: lanes that differ only in
                    // those bits hold the same totals, and the lowest of them writes
                    const int dup = lpr >> hl;
                    for (int o = dup >> 1; o >= 1; o >>= 1) gpart[0] += __shfl_xor_sync(gmask, gpart[0], o, lpr);
                    const bool writer = (gl & (dup - 1)) == 0;
#pragma unroll
                    for (int i = 0; i < NV; ++i) {
                        if (i >= vc) break;
                        const int idx = base + i, u = idx % U;
                        const uint32_t pr = __shfl_sync(gmask, S.pr, min(j + u, nb - 1), lpr);
                        if (writer && j + u < nb) put_grad(idx < U ? A.g_anchor : (PHASED ? A.g_phase : nullptr), pr,
                                                          gpart[i]);
                    }
                }
                slot ^= 1;
            }
            S = Sn;
        }
        cp_async_wait_all();
    } else {
        // Narrow groups: the group walks its rows in batches of U, loading the
        // batch's anchors and permutation entries, then its phases and gathered rows
        // (U rows in flight), then processing the rows in order.  Rows past r1 in
        // the last batch repeat row r1-1 for the loads and are skipped.
        for (int64_t rb = r0; rb < r1; rb += U) {
            float qv[U], tv[U];
            uint32_t pv[U];
            float hv[U][VEC];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = min(rb + u, r1 - 1);
                qv[u] = __ldg(A.s + r);
                pv[u] = min(__ldg(A.perm + r), (uint32_t)(A.m - 1));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                tv[u] = PHASED ? __ldg(A.theta + pv[u]) : 0.f;
#pragma unroll
                for (int v = 0; v < VEC; ++v) hv[u][v] = 0.f;
                if (ROWS && cval) load_vec<VEC>(row_src(pv[u]), hv[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (rb + u >= r1) break;
                const float q = qv[u];
                float sn = 0.f, cs = 1.f;
                if (PHASED) sincosf(tv[u], &sn, &cs);
                while (m < ms && __ldg(A.sp + m) < q) ++m;
                if (mp < m) mp = m;
                while (mp < ms && __ldg(A.sp + mp) <= q) ++mp;
                const float eL = (m > 0) ? expf(__ldg(A.sp + m - 1) - q) : 0.f;
                const float eR = (mp < ms) ? expf(q - __ldg(A.sp + mp)) : 0.f;
                float ga = 0.f, gp = 0.f;
                row(pv[u], cs, sn, eL, eR, m, mp, hv[u], ga, gp);
                if (GRAD) {
                    for (int off = lpr >> 1; off >= 1; off >>= 1) {
                        ga += __shfl_xor_sync(gmask, ga, off);
                        if (PHASED) gp += __shfl_xor_sync(gmask, gp, off);
                    }
                    if (gl == 0) {
                        put_grad(A.g_anchor, pv[u], ga);
                        if (PHASED) put_grad(A.g_phase, pv[u], gp);
                    }
                }
            }
            // fp32 interval partials cover at most 16 rows; the schedule is the same
            // for every group of the warp, so the fold never diverges
            if (ACCUM && (((rb - r0) / U) & 1)) fold();
        }
    }
    if (ACCUM) flush(cur);
}

// The interval-sum pass (accumulate only) for full 32-lane groups, 16-byte
// slices: one warp per contiguous run of sorted rows, lane l owning channels
// c0 .. c0+3 of every row (as k_large with lpr = 32, VEC = 4, MODE = kLmAccum, and the
// same interval sums, tie sums, fp32-then-fp64 partials and owner-or-atomic
// flushes).  Per batch of 32 rows, lane l computes the scalars of row rb + l (its
// permutation entry, its bins among the small-side anchors, and the four weights
// e_R w_p, e_L w_p of its phase weights w_p and decays to the neighbouring
// small-side anchors) into a per-warp slot in shared memory; the warp then walks
// the batch reading each row's scalars with two broadcast loads and its 512-byte
// row with one coalesced load per lane, issued four rows ahead of their use.
struct AccumSlot {
    float4 w;  // (e_R w_0, e_R w_1, e_L w_0, e_L w_1), or (w_0, w_1, 0, 0) for a row tied with the small side
    uint4 ib;  // permutation entry, bin m (anchors < q), bin mp (anchors <= q), unused
};

// Rows per batch of a group of LPR lanes (at least 8, so that narrow groups too take
// a batch of rows per pair of warp barriers) and the slots of a warp.
template <int LPR>
constexpr int kLeanBatch = LPR >= 8 ? LPR : 8;
template <int LPR>
constexpr int kLeanSlots = (32 / LPR) * kLeanBatch<LPR>;

template <int LPR, bool PHASED>
__global__ void __launch_bounds__(256, 3) k_large_accum_w(LargePass A) {
    constexpr int NP = PHASED ? 2 : 1, VEC = 4, ND = 2 * NP * VEC, S = kLeanBatch<LPR>, PF = S < 4 ? S : 4;
    extern __shared__ __align__(16) unsigned char accum_smem[];
    double(*s_dacc)[256] = reinterpret_cast<double(*)[256]>(accum_smem);
    AccumSlot* slots = reinterpret_cast<AccumSlot*>(accum_smem + sizeof(double) * ND * 256);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gl = lane % LPR, gw = lane / LPR;
    const unsigned gmask = (LPR == 32) ? 0xffffffffu : (((1u << LPR) - 1u) << (gw * LPR));
    AccumSlot* ws = slots + warp * kLeanSlots<LPR> + gw * S;
    const int64_t gid = ((int64_t)blockIdx.x * 8 + warp) * (32 / LPR) + gw;
    const int c0 = (blockIdx.y * LPR + gl) * VEC;
    const bool cval = c0 < A.B;
    const int64_t r0 = gid * A.rows_per_group;
    const int64_t r1 = min(A.m, r0 + A.rows_per_group);
    if (r0 >= r1) return;  // the whole group leaves together; no block barrier follows
    const int64_t ms = A.ms;
    const int B = A.B, Cb = A.Cb;
    // this lane's slice of a row: channels [0, Bs) from rows, [Bs, B) from rows2
    const float* src = (A.rows2 != nullptr && c0 >= A.Bs) ? A.rows2 + (c0 - A.Bs) : A.rows + c0;
    const int64_t stride = A.Bs;

#pragma unroll
    for (int i = 0; i < ND; ++i) s_dacc[i][threadIdx.x] = 0.0;
    int64_t m_run = lower_bound_f(A.sp, ms, __ldg(A.s + r0));
    int64_t mp_run = upper_bound_f(A.sp, ms, __ldg(A.s + r0));
    const int64_t m_first = m_run;
    const int64_t m_last = lower_bound_f(A.sp, ms, __ldg(A.s + r1 - 1));
    int64_t cur = m_run;
    float fu[NP][VEC], fv[NP][VEC];
#pragma unroll
    for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int v = 0; v < VEC; ++v) fu[q][v] = fv[q][v] = 0.f;
    int cnt = 0;
    auto fold = [&]() {
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                s_dacc[q * VEC + v][threadIdx.x] += (double)fu[q][v];
                s_dacc[NP * VEC + q * VEC + v][threadIdx.x] += (double)fv[q][v];
                fu[q][v] = fv[q][v] = 0.f;
            }
        cnt = 0;
    };
    auto flush = [&](int64_t bin) {
        fold();
        if (!cval) return;
        const bool owner = bin > m_first && bin < m_last;  // no other warp touches this bin
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                const int ch = q * B + c0 + v;
                double& du = s_dacc[q * VEC + v][threadIdx.x];
                double& dv = s_dacc[NP * VEC + q * VEC + v][threadIdx.x];
                if (bin < ms) {
                    double* dst = A.U + bin * Cb + ch;
                    if (owner)
                        *dst = du;
                    else if (du != 0.0)
                        atomicAdd(dst, du);
                }
                if (bin >= 1) {
                    double* dst = A.V + (bin - 1) * Cb + ch;
                    if (owner)
                        *dst = dv;
                    else if (dv != 0.0)
                        atomicAdd(dst, dv);
                }
                du = 0.0;
                dv = 0.0;
            }
    };

    for (int64_t rb = r0; rb < r1; rb += S) {
        const int nb = (int)min((int64_t)S, r1 - rb);
        __syncwarp(gmask);  // the previous batch's slots have been read
        for (int j = gl; j < nb; j += LPR) {
            const int64_t r = rb + j;
            const float q = __ldg(A.s + r);
            AccumSlot sl;
            const uint32_t pr = min(__ldg(A.perm + r), (uint32_t)(A.m - 1));
            float w0 = 1.f, w1 = 0.f;
            if (PHASED) sincosf(__ldg(A.theta + pr), &w1, &w0);
            int64_t mm = m_run;
            while (mm < ms && __ldg(A.sp + mm) < q) ++mm;
            int64_t mmp = max(mp_run, mm);
            while (mmp < ms && __ldg(A.sp + mmp) <= q) ++mmp;
            const float eL = (mm > 0) ? expf(__ldg(A.sp + mm - 1) - q) : 0.f;
            const float eR = (mmp < ms) ? expf(q - __ldg(A.sp + mmp)) : 0.f;
            sl.w = (mmp > mm) ? make_float4(w0, w1, 0.f, 0.f) : make_float4(eR * w0, eR * w1, eL * w0, eL * w1);
            sl.ib = make_uint4(pr, (uint32_t)mm, (uint32_t)mmp, 0u);
            ws[j] = sl;
        }
        __syncwarp(gmask);
        {
            const uint4 last = ws[nb - 1].ib;  // where the next batch's searches start
            m_run = last.y;
            mp_run = last.z;
        }
        for (int u0 = 0; u0 < nb; u0 += PF) {
            float4 h[PF];
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                h[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (u0 + i < nb && cval) h[i] = __ldg(reinterpret_cast<const float4*>(src + (int64_t)ws[u0 + i].ib.x * stride));
            }
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                if (u0 + i >= nb) break;
                const float4 w = ws[u0 + i].w;
                const uint4 ib = ws[u0 + i].ib;
                const int64_t mr = ib.y, mpr = ib.z;
                if (mr != cur) {
                    flush(cur);
                    cur = mr;
                }
                const float hv[4] = {h[i].x, h[i].y, h[i].z, h[i].w};
                if (mpr == mr) {
                    // untied rows feed the interval sums u (weighted to the right
                    // neighbour) and v (to the left one)
                    const float wr[2] = {w.x, w.y}, wl[2] = {w.z, w.w};
#pragma unroll
                    for (int q = 0; q < NP; ++q)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            fu[q][v] = fmaf(wr[q], hv[v], fu[q][v]);
                            fv[q][v] = fmaf(wl[q], hv[v], fv[q][v]);
                        }
                } else if (cval) {
                    // a row tied with a run of small-side anchors enters that run only
                    const float wt[2] = {w.x, w.y};
#pragma unroll
                    for (int q = 0; q < NP; ++q)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            const double val = (double)(wt[q] * hv[v]);
                            atomicAdd(A.TL + mr * Cb + q * B + c0 + v, val);
                            atomicAdd(A.TR + (mpr - 1) * Cb + q * B + c0 + v, val);
                        }
                }
                if (++cnt == 16) fold();
            }
        }
    }
    flush(cur);
}

// The neighbour-state pass (expand and / or gradients) for full 32-lane groups,
// 16-byte slices: the per-warp scalar slots of k_large_accum_w, then per row
//   out = sum_p w_p (eLf P_(mp-1) + eR S_mp)          (EXPAND; eLf = 1 for a tie)
//   ga  = sum_c h_c sum_p w_p (eR S_mp - eL P_(m-1))   (GRAD: strict right - left)
//   gph = sum_c h_c (w_0 f_1 - w_1 f_0),  f_p = eLf P_(mp-1) + eR S_mp   (GRAD, phased)
// from the small side's states P, S (reloaded only when the row's bins change) and
// the gathered row h; the gradient shares of four rows are summed over the warp by
// recursive halving.  The arithmetic is that of k_large's row body.
struct ExpandSlot {
    float4 w;  // (w_0, w_1, eL, eR)
    uint4 ib;  // permutation entry, bin m (anchors < q), bin mp (anchors <= q), unused
};

template <int LPR, bool PHASED, bool EXPAND, bool GRAD>
__global__ void __launch_bounds__(256, 3) k_large_expand_w(LargePass A) {
    static_assert(!GRAD || LPR == 32, "the gradient reduction is written for full warps");
    constexpr int NP = PHASED ? 2 : 1, VEC = 4, U = 4, S = kLeanBatch<LPR>;
    __shared__ ExpandSlot slots[8][kLeanSlots<LPR>];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gl = lane % LPR, gw = lane / LPR;
    const unsigned gmask = (LPR == 32) ? 0xffffffffu : (((1u << LPR) - 1u) << (gw * LPR));
    ExpandSlot* ws = slots[warp] + gw * S;
    const int64_t gid = ((int64_t)blockIdx.x * 8 + warp) * (32 / LPR) + gw;
    const int c0 = (blockIdx.y * LPR + gl) * VEC;
    const bool cval = c0 < A.B;
    const int64_t r0 = gid * A.rows_per_group;
    const int64_t r1 = min(A.m, r0 + A.rows_per_group);
    if (r0 >= r1) return;  // the whole group leaves together; no block barrier follows
    const int64_t ms = A.ms;
    const int B = A.B, Cb = A.Cb;
    const float* src = (A.rows2 != nullptr && c0 >= A.Bs) ? A.rows2 + (c0 - A.Bs) : A.rows + c0;
    const int64_t stride = A.Bs;
    int64_t m_run = lower_bound_f(A.sp, ms, __ldg(A.s + r0));
    int64_t mp_run = upper_bound_f(A.sp, ms, __ldg(A.s + r0));
    int64_t st_m = -1, st_mp = -1;
    float Pm1[NP][VEC], Pmp[NP][VEC], Smp[NP][VEC];
    auto put_grad = [&](float* dst, uint32_t pr, float v) {
        if (dst == nullptr) return;
        if (A.chunk_atomic)
            atomicAdd(dst + pr, v);
        else if (A.accumulate)
            dst[pr] += v;  // every row is visited once per launch
        else
            dst[pr] = v;
    };

    for (int64_t rb = r0; rb < r1; rb += S) {
        const int nb = (int)min((int64_t)S, r1 - rb);
        __syncwarp(gmask);  // the previous batch's slots have been read
        for (int j = gl; j < nb; j += LPR) {
            const int64_t r = rb + j;
            const float q = __ldg(A.s + r);
            const uint32_t pr = min(__ldg(A.perm + r), (uint32_t)(A.m - 1));
            float w0 = 1.f, w1 = 0.f;
            if (PHASED) sincosf(__ldg(A.theta + pr), &w1, &w0);
            int64_t mm = m_run;
            while (mm < ms && __ldg(A.sp + mm) < q) ++mm;
            int64_t mmp = max(mp_run, mm);
            while (mmp < ms && __ldg(A.sp + mmp) <= q) ++mmp;
            const float eL = (mm > 0) ? expf(__ldg(A.sp + mm - 1) - q) : 0.f;
            const float eR = (mmp < ms) ? expf(q - __ldg(A.sp + mmp)) : 0.f;
            ExpandSlot sl;
            sl.w = make_float4(w0, w1, eL, eR);
            sl.ib = make_uint4(pr, (uint32_t)mm, (uint32_t)mmp, 0u);
            ws[j] = sl;
        }
        __syncwarp(gmask);
        {
            const uint4 last = ws[nb - 1].ib;
            m_run = last.y;
            mp_run = last.z;
        }
        for (int u0 = 0; u0 < nb; u0 += U) {
            float4 h[U];
#pragma unroll
            for (int i = 0; i < U; ++i) {
                h[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (GRAD && u0 + i < nb && cval)
                    h[i] = __ldg(reinterpret_cast<const float4*>(src + (int64_t)ws[u0 + i].ib.x * stride));
            }
            float gpart[GRAD ? 2 * U : 1];
#pragma unroll
            for (int i = 0; i < U; ++i) {
                float ga = 0.f, gph = 0.f;
                if (u0 + i < nb) {
                    const float4 w = ws[u0 + i].w;
                    const uint4 ib = ws[u0 + i].ib;
                    const int64_t mr = ib.y, mpr = ib.z;
                    if (mr != st_m || mpr != st_mp) {
#pragma unroll
                        for (int q = 0; q < NP; ++q)
#pragma unroll
                            for (int v = 0; v < VEC; ++v) {
                                const int ch = q * B + c0 + v;
                                Pm1[q][v] = (GRAD && cval && mr > 0) ? __ldg(A.Pst + (mr - 1) * Cb + ch) : 0.f;
                                Pmp[q][v] = (cval && mpr > 0) ? __ldg(A.Pst + (mpr - 1) * Cb + ch) : 0.f;
                                Smp[q][v] = (cval && mpr < ms) ? __ldg(A.Sst + mpr * Cb + ch) : 0.f;
                            }
                        st_m = mr;
                        st_mp = mpr;
                    }
                    const float wp[2] = {w.x, w.y};
                    const float eL = w.z, eR = w.w, eLf = (mpr > mr) ? 1.f : eL;
                    const float hv[4] = {h[i].x, h[i].y, h[i].z, h[i].w};
                    float o[VEC];
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        o[v] = 0.f;
                        float t = 0.f;
#pragma unroll
                        for (int q = 0; q < NP; ++q) {
                            const float fl = eLf * wp[q], fr = eR * wp[q], dl = eL * wp[q];
                            o[v] = fmaf(fl, Pmp[q][v], fmaf(fr, Smp[q][v], o[v]));
                            if (GRAD) t = fmaf(fr, Smp[q][v], fmaf(-dl, Pm1[q][v], t));
                        }
                        if (GRAD) {
                            ga = fmaf(hv[v], t, ga);
                            if (PHASED) {
                                const float f0 = fmaf(eLf, Pmp[0][v], eR * Smp[0][v]);
                                const float f1 = fmaf(eLf, Pmp[NP - 1][v], eR * Smp[NP - 1][v]);
                                gph = fmaf(hv[v], fmaf(wp[0], f1, -wp[1] * f0), gph);
                            }
                        }
                    }
                    if (EXPAND && A.out != nullptr && cval)
                        *reinterpret_cast<float4*>(A.out + (int64_t)ib.x * B + c0) = make_float4(o[0], o[1], o[2], o[3]);
                }
                if (GRAD) {
                    gpart[i] = ga;
                    gpart[U + i] = gph;
                }
            }
            if (GRAD) {
                // sum the 2U shares over the 32 lanes by recursive halving: after the
                // halving rounds lane l holds the total of value index base, then the
                // remaining rounds add whole totals
                constexpr int NV = 2 * U;
                int base = 0;
#pragma unroll
                for (int L = 0; (NV >> L) > 1; ++L) {
                    const int o = 16 >> L;
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < (NV >> (L + 1)); ++i) {
                        const float keep = upper ? gpart[i + (NV >> (L + 1))] : gpart[i];
                        const float send = upper ? gpart[i] : gpart[i + (NV >> (L + 1))];
                        gpart[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                    if (upper) base += NV >> (L + 1);
                }
                constexpr int HL = (NV == 8) ? 3 : 0;  // halving rounds taken (log2 NV)
                static_assert(NV == 8, "four rows per reduction");
                for (int o = (32 >> HL) >> 1; o >= 1; o >>= 1) gpart[0] += __shfl_xor_sync(0xffffffffu, gpart[0], o);
                const bool writer = (lane & ((32 >> HL) - 1)) == 0;
                const int u = base % U;
                if (writer && u0 + u < nb) {
                    const uint32_t pr = ws[u0 + u].ib.x;
                    put_grad(base < U ? A.g_anchor : (PHASED ? A.g_phase : nullptr), pr, gpart[0]);
                }
            }
        }
    }
}

// Interval sums and anchor / phase gradients in one pass (kLmAccum | kLmGrad: the
// backward over a larger output side) for groups of 2-16 lanes of 16-byte slices
// (instantiated unphased; the phased form would spill):
// the per-group row slots and interval sums of k_large_accum_w, plus per row the
// gradient shares of k_large's row body from the cached small-side states, summed
// over the group's lanes by xor-shuffles and written by its first lane.
struct AccGradSlot {
    float4 f;  // (e_R w_0, e_R w_1, e_L w_0, e_L w_1)
    float4 x;  // (w_0, w_1, e_L, e_R)
    uint4 ib;  // permutation entry, bin m (anchors < q), bin mp (anchors <= q), unused
};

template <int LPR, bool PHASED>
__global__ void __launch_bounds__(256, 3) k_large_accgrad_n(LargePass A) {
    static_assert(LPR >= 2 && LPR <= 16, "narrow groups");
    constexpr int NP = PHASED ? 2 : 1, VEC = 4, ND = 2 * NP * VEC, S = kLeanBatch<LPR>, PF = 4;
    extern __shared__ __align__(16) unsigned char accgrad_smem[];
    double(*s_dacc)[256] = reinterpret_cast<double(*)[256]>(accgrad_smem);
    AccGradSlot* slots = reinterpret_cast<AccGradSlot*>(accgrad_smem + sizeof(double) * ND * 256);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gl = lane % LPR, gw = lane / LPR;
    const unsigned gmask = ((1u << LPR) - 1u) << (gw * LPR);
    AccGradSlot* ws = slots + warp * kLeanSlots<LPR> + gw * S;
    const int64_t gid = ((int64_t)blockIdx.x * 8 + warp) * (32 / LPR) + gw;
    const int c0 = (blockIdx.y * LPR + gl) * VEC;
    const bool cval = c0 < A.B;
    const int64_t r0 = gid * A.rows_per_group;
    const int64_t r1 = min(A.m, r0 + A.rows_per_group);
    if (r0 >= r1) return;  // the whole group leaves together; no block barrier follows
    const int64_t ms = A.ms;
    const int B = A.B, Cb = A.Cb;
    const float* src = (A.rows2 != nullptr && c0 >= A.Bs) ? A.rows2 + (c0 - A.Bs) : A.rows + c0;
    const int64_t stride = A.Bs;

#pragma unroll
    for (int i = 0; i < ND; ++i) s_dacc[i][threadIdx.x] = 0.0;
    int64_t m_run = lower_bound_f(A.sp, ms, __ldg(A.s + r0));
    int64_t mp_run = upper_bound_f(A.sp, ms, __ldg(A.s + r0));
    const int64_t m_first = m_run;
    const int64_t m_last = lower_bound_f(A.sp, ms, __ldg(A.s + r1 - 1));
    int64_t cur = m_run, st_m = -1, st_mp = -1;
    float fu[NP][VEC], fv[NP][VEC], Pm1[NP][VEC], Pmp[NP][VEC], Smp[NP][VEC];
#pragma unroll
    for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int v = 0; v < VEC; ++v) fu[q][v] = fv[q][v] = 0.f;
    int cnt = 0;
    auto fold = [&]() {
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                s_dacc[q * VEC + v][threadIdx.x] += (double)fu[q][v];
                s_dacc[NP * VEC + q * VEC + v][threadIdx.x] += (double)fv[q][v];
                fu[q][v] = fv[q][v] = 0.f;
            }
        cnt = 0;
    };
    auto flush = [&](int64_t bin) {
        fold();
        if (!cval) return;
        const bool owner = bin > m_first && bin < m_last;  // no other group touches this bin
#pragma unroll
        for (int q = 0; q < NP; ++q)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                const int ch = q * B + c0 + v;
                double& du = s_dacc[q * VEC + v][threadIdx.x];
                double& dv = s_dacc[NP * VEC + q * VEC + v][threadIdx.x];
                if (bin < ms) {
                    double* dst = A.U + bin * Cb + ch;
                    if (owner)
                        *dst = du;
                    else if (du != 0.0)
                        atomicAdd(dst, du);
                }
                if (bin >= 1) {
                    double* dst = A.V + (bin - 1) * Cb + ch;
                    if (owner)
                        *dst = dv;
                    else if (dv != 0.0)
                        atomicAdd(dst, dv);
                }
                du = 0.0;
                dv = 0.0;
            }
    };
    auto put_grad = [&](float* dst, uint32_t pr, float v) {
        if (dst == nullptr) return;
        if (A.chunk_atomic)
            atomicAdd(dst + pr, v);
        else if (A.accumulate)
            dst[pr] += v;  // every row is visited once per launch
        else
            dst[pr] = v;
    };

    for (int64_t rb = r0; rb < r1; rb += S) {
        const int nb = (int)min((int64_t)S, r1 - rb);
        __syncwarp(gmask);  // the previous batch's slots have been read
        for (int j = gl; j < nb; j += LPR) {
            const int64_t r = rb + j;
            const float q = __ldg(A.s + r);
            const uint32_t pr = min(__ldg(A.perm + r), (uint32_t)(A.m - 1));
            float w0 = 1.f, w1 = 0.f;
            if (PHASED) sincosf(__ldg(A.theta + pr), &w1, &w0);
            int64_t mm = m_run;
            while (mm < ms && __ldg(A.sp + mm) < q) ++mm;
            int64_t mmp = max(mp_run, mm);
            while (mmp < ms && __ldg(A.sp + mmp) <= q) ++mmp;
            const float eL = (mm > 0) ? expf(__ldg(A.sp + mm - 1) - q) : 0.f;
            const float eR = (mmp < ms) ? expf(q - __ldg(A.sp + mmp)) : 0.f;
            AccGradSlot sl;
            sl.f = make_float4(eR * w0, eR * w1, eL * w0, eL * w1);
            sl.x = make_float4(w0, w1, eL, eR);
            sl.ib = make_uint4(pr, (uint32_t)mm, (uint32_t)mmp, 0u);
            ws[j] = sl;
        }
        __syncwarp(gmask);
        {
            const uint4 last = ws[nb - 1].ib;  // where the next batch's searches start
            m_run = last.y;
            mp_run = last.z;
        }
        for (int u0 = 0; u0 < nb; u0 += PF) {
            float4 h[PF];
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                h[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (u0 + i < nb && cval)
                    h[i] = __ldg(reinterpret_cast<const float4*>(src + (int64_t)ws[u0 + i].ib.x * stride));
            }
#pragma unroll
            for (int i = 0; i < PF; ++i) {
                if (u0 + i >= nb) break;
                const float4 f = ws[u0 + i].f, x = ws[u0 + i].x;
                const uint4 ib = ws[u0 + i].ib;
                const int64_t mr = ib.y, mpr = ib.z;
                const bool tie = mpr > mr;
                const float hv[4] = {h[i].x, h[i].y, h[i].z, h[i].w};
                const float fr[2] = {f.x, f.y}, dl[2] = {f.z, f.w}, wp[2] = {x.x, x.y};
                // interval sums
                if (mr != cur) {
                    flush(cur);
                    cur = mr;
                }
                if (!tie) {
#pragma unroll
                    for (int q = 0; q < NP; ++q)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            fu[q][v] = fmaf(fr[q], hv[v], fu[q][v]);
                            fv[q][v] = fmaf(dl[q], hv[v], fv[q][v]);
                        }
                } else if (cval) {
#pragma unroll
                    for (int q = 0; q < NP; ++q)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            const double val = (double)(wp[q] * hv[v]);
                            atomicAdd(A.TL + mr * Cb + q * B + c0 + v, val);
                            atomicAdd(A.TR + (mpr - 1) * Cb + q * B + c0 + v, val);
                        }
                }
                if (++cnt == 16) fold();
                // gradient shares from the small side's states
                if (mr != st_m || mpr != st_mp) {
#pragma unroll
                    for (int q = 0; q < NP; ++q)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            const int ch = q * B + c0 + v;
                            Pm1[q][v] = (cval && mr > 0) ? __ldg(A.Pst + (mr - 1) * Cb + ch) : 0.f;
                            Pmp[q][v] = (cval && mpr > 0) ? __ldg(A.Pst + (mpr - 1) * Cb + ch) : 0.f;
                            Smp[q][v] = (cval && mpr < ms) ? __ldg(A.Sst + mpr * Cb + ch) : 0.f;
                        }
                    st_m = mr;
                    st_mp = mpr;
                }
                const float eL = x.z, eR = x.w, eLf = tie ? 1.f : eL;
                float ga = 0.f, gph = 0.f;
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    float t = 0.f;
#pragma unroll
                    for (int q = 0; q < NP; ++q) t = fmaf(fr[q], Smp[q][v], fmaf(-dl[q], Pm1[q][v], t));
                    ga = fmaf(hv[v], t, ga);  // strict right - strict left
                    if (PHASED) {
                        const float f0 = fmaf(eLf, Pmp[0][v], eR * Smp[0][v]);
                        const float f1 = fmaf(eLf, Pmp[NP - 1][v], eR * Smp[NP - 1][v]);
                        gph = fmaf(hv[v], fmaf(wp[0], f1, -wp[1] * f0), gph);
                    }
                }
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) {
                    ga += __shfl_xor_sync(gmask, ga, o);
                    if (PHASED) gph += __shfl_xor_sync(gmask, gph, o);
                }
                if (gl == 0) {
                    put_grad(A.g_anchor, ib.x, ga);
                    if (PHASED) put_grad(A.g_phase, ib.x, gph);
                }
            }
        }
    }
    flush(cur);
}

// ------------------------------------------------------------------ finish

struct Finish {
    const uint32_t* perm;  // small side
    const float* theta;
    int64_t m;
    const float* ZL;  // parts [m][Cb], sorted order
    const float* ZR;
    const float* ZF;
    int B;
    int Cb;
    const float* h;  // [m][B] original order (for gradients), or sorted order when h_sorted
    bool h_sorted;
    float* out;      // [m][B] original order: sum_p w_p ZF
    float* g_anchor;  // sum_c h sum_p w_p (ZR - ZL)
    float* g_phase;   // sum_c h sum_p w'_p ZF
    int accumulate;   // add into g_anchor / g_phase instead of writing
};

template <bool PHASED>
__global__ void __launch_bounds__(256) k_finish(Finish F) {
    constexpr int NP = PHASED ? 2 : 1;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= F.m) return;
    const int lane = threadIdx.x & 31;
    const uint32_t pr = min(__ldg(F.perm + r), (uint32_t)(F.m - 1));
    float w[NP], wd[NP];
    if (PHASED) {
        float sn, cs;
        sincosf(__ldg(F.theta + pr), &sn, &cs);
        w[0] = cs;
        w[NP - 1] = sn;
        wd[0] = -sn;
        wd[NP - 1] = cs;
    } else {
        w[0] = 1.f;
        wd[0] = 0.f;
    }
    float ga = 0.f, gp = 0.f;
    for (int c = lane; c < F.B; c += 32) {
        const float hv = F.h ? __ldg(F.h + (int64_t)(F.h_sorted ? r : pr) * F.B + c) : 0.f;
        float o = 0.f;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const int64_t idx = r * F.Cb + p * F.B + c;
            const float zf = __ldg(F.ZF + idx);
            o = fmaf(w[p], zf, o);
            if (F.g_anchor) ga = fmaf(hv * w[p], __ldg(F.ZR + idx) - __ldg(F.ZL + idx), ga);
            if (PHASED) gp = fmaf(hv * wd[p], zf, gp);
        }
        if (F.out) F.out[(int64_t)pr * F.B + c] = o;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        ga += __shfl_xor_sync(0xffffffffu, ga, off);
        gp += __shfl_xor_sync(0xffffffffu, gp, off);
    }
    if (lane == 0) {
        if (F.g_anchor) F.g_anchor[pr] = F.accumulate ? F.g_anchor[pr] + ga : ga;
        if (PHASED && F.g_phase) F.g_phase[pr] = F.accumulate ? F.g_phase[pr] + gp : gp;
    }
}

// The middle of the Gram apply, one warp per small-side row j: w2 = D_j w_j (the
// input of the second pass), w_saved = w_j (optional), and gD_j = <wg_j, w_j> when
// wg is given.  w and wg are rows of ld floats (a paired pass stores them side by
// side in one [k][2B] array).
__global__ void __launch_bounds__(256) k_gram_mid(const float* __restrict__ D, const float* __restrict__ w, int ld,
                                                  const float* __restrict__ wg, float* __restrict__ w2,
                                                  float* __restrict__ w_saved, float* __restrict__ gD, int64_t k, int B) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= k) return;
    const int lane = threadIdx.x & 31;
    const float d = __ldg(D + r);
    float acc = 0.f;
    for (int c = lane; c < B; c += 32) {
        const float wv = __ldg(w + r * ld + c);
        w2[r * B + c] = d * wv;
        if (w_saved != nullptr) w_saved[r * B + c] = wv;
        if (wg != nullptr) acc = fmaf(__ldg(wg + r * ld + c), wv, acc);
    }
    if (gD != nullptr) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) gD[r] = acc;
    }
}

// The middle of the Gram operator straight from the paired reduce pass's full parts
// (sorted order, rows of ld floats: w = A^T v in [0, B), u = A^T g in [B, 2B)).
// LPR lanes per sorted row j, original row p = perm[j]: x[j] = D_p w, followed by
// D_p u when WITH_U (rows of x_ld floats, sorted order, so that the next scan reads
// them without the permutation), w_saved[p] = w (optional) and gD[p] = <u, w>
// (optional).
template <int LPR, bool WITH_U>
__global__ void __launch_bounds__(256) k_gram_mid_sorted(const uint32_t* __restrict__ perm, const float* __restrict__ D,
                                                         const float* __restrict__ ZF, int ld, float* __restrict__ x,
                                                         int x_ld, float* __restrict__ w_saved, float* __restrict__ gD,
                                                         int64_t k, int B) {
    const int64_t j = (int64_t)blockIdx.x * (256 / LPR) + threadIdx.x / LPR;
    const int q = threadIdx.x % LPR;
    const bool in = j < k;
    const int64_t jj = in ? j : 0;
    const uint32_t pr = min(__ldg(perm + jj), (uint32_t)(k - 1));
    const float d = __ldg(D + pr);
    float acc = 0.f;
    if (in)
        for (int c = q; c < B; c += LPR) {
            const float wv = __ldg(ZF + jj * ld + c), uv = __ldg(ZF + jj * ld + B + c);
            x[jj * x_ld + c] = d * wv;
            if (WITH_U) x[jj * x_ld + B + c] = d * uv;
            if (w_saved != nullptr) w_saved[(int64_t)pr * B + c] = wv;
            acc = fmaf(uv, wv, acc);
        }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in && q == 0 && gD != nullptr) gD[pr] = acc;
}

template <bool WITH_U>
cudaError_t launch_gram_mid_sorted(const uint32_t* perm, const float* D, const float* ZF, int ld, float* x, int x_ld,
                                   float* w_saved, float* gD, int64_t k, int64_t B, cudaStream_t st) {
#define GRAM_MID_CASE(LP)                                                                                       \
    LAPLEX_TIMED("gram_mid", st,                                                                              \
                 (k_gram_mid_sorted<LP, WITH_U><<<(unsigned)((k + (256 / LP) - 1) / (256 / LP)), 256, 0, st>>>( \
                     perm, D, ZF, ld, x, x_ld, w_saved, gD, k, (int)B)))
    if (B <= 4)
        GRAM_MID_CASE(4);
    else if (B <= 8)
        GRAM_MID_CASE(8);
    else if (B <= 16)
        GRAM_MID_CASE(16);
    else
        GRAM_MID_CASE(32);
#undef GRAM_MID_CASE
    return cudaGetLastError();
}

// ------------------------------------------------------------------ host side

struct RectPlan {
    int64_t ms;  // rows of the small side
    int Cb, C, G;
    int64_t R, T;
    unsigned* counters;  // [2][G]
    int* flags;          // [2][G][T]
    size_t memset_bytes;
    double2* agg;  // [2][G][T][C]
    double2* inc;
    double* bins;  // U, TL, V, TR: [4][ms][Cb]
    float* bufA;   // [3][ms][Cb]
    float* bufB;   // [3][ms][Cb]
    float* rows3;  // gram scratch [3][k][B]
    size_t total;
};

RectPlan plan_rect(int64_t n_out, int64_t n_in, int64_t B, bool phased, void* ws, int64_t gram_k = 0) {
    RectPlan p;
    p.ms = std::min(n_out, n_in);
    p.Cb = (int)(phased ? 2 * B : B);
    p.C = choose_channels(p.Cb);
    p.G = (p.Cb + p.C - 1) / p.C;
    p.R = kTileValues / p.C;
    p.T = (p.ms + p.R - 1) / p.R;
    char* base = (char*)ws;
    size_t off = 0;
    p.counters = (unsigned*)(base + off);
    off += align_up(sizeof(unsigned) * 2 * p.G, 256);
    p.flags = (int*)(base + off);
    off += align_up(sizeof(int) * 2 * p.G * p.T, 256);
    p.memset_bytes = off;
    p.agg = (double2*)(base + off);
    off += align_up(sizeof(double2) * 2 * p.G * p.T * p.C, 256);
    p.inc = (double2*)(base + off);
    off += align_up(sizeof(double2) * 2 * p.G * p.T * p.C, 256);
    p.bins = (double*)(base + off);
    off += align_up(sizeof(double) * 4 * p.ms * p.Cb, 256);
    p.bufA = (float*)(base + off);
    off += align_up(sizeof(float) * 3 * p.ms * p.Cb, 256);
    p.bufB = (float*)(base + off);
    off += align_up(sizeof(float) * 3 * p.ms * p.Cb, 256);
    p.rows3 = (float*)(base + off);
    off += align_up(sizeof(float) * 3 * gram_k * B, 256);
    p.total = off;
    return p;
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int C, bool BINS>
cudaError_t side_scan_t(const RectPlan& p, SideScan a, int32_t* status, cudaStream_t st) {
    ChainSet cr{p.flags, p.agg, p.inc, p.T, p.C};
    ChainSet cl{p.flags + (int64_t)p.G * p.T, p.agg + (int64_t)p.G * p.T * p.C, p.inc + (int64_t)p.G * p.T * p.C,
                p.T, p.C};
    const dim3 grid((unsigned)p.T, (unsigned)p.G);
    if (p.T <= kSideDirectMaxTiles && p.T * C <= kSideDirectMaxValues) {
        LAPLEX_TIMED("side_totals", st, k_side_totals<C, BINS><<<grid, kSideNT, 0, st>>>(a, cl, cr));
        LAPLEX_TIMED("side_apply", st, k_side_apply<C, BINS><<<grid, kSideNT, 0, st>>>(a, cl, cr));
        return cudaGetLastError();
    }
    // the lookback kernels claim tiles from counters and wait on flags: both start at zero
    const cudaError_t e = cudaMemsetAsync(p.counters, 0, p.memset_bytes, st);
    if (e != cudaSuccess) return e;
    LAPLEX_TIMED("side_right", st, k_side_right<C, BINS><<<grid, kSideNT, 0, st>>>(a, cr, p.counters, status));
    LAPLEX_TIMED("side_left", st, k_side_left<C, BINS><<<grid, kSideNT, 0, st>>>(a, cl, cr, p.counters + p.G, status));
    return cudaGetLastError();
}

cudaError_t side_scan(const RectPlan& p, SideScan a, bool bins, int32_t* status, cudaStream_t st) {
    a.T = p.T;
    a.Cb = p.Cb;
#define SIDE_CASE(CC)                                                                                  \
    case CC:                                                                                           \
        return bins ? side_scan_t<CC, true>(p, a, status, st) : side_scan_t<CC, false>(p, a, status, st);
    switch (p.C) {
        SIDE_CASE(1)
        SIDE_CASE(2)
        SIDE_CASE(4)
        SIDE_CASE(8)
        SIDE_CASE(16)
        default:
            return bins ? side_scan_t<32, true>(p, a, status, st) : side_scan_t<32, false>(p, a, status, st);
    }
#undef SIDE_CASE
}

#define LAPLEX_TRY(expr)                     \
    do {                                     \
        cudaError_t e_ = (expr);             \
        if (e_ != cudaSuccess) return e_;    \
    } while (0)

// One launch of k_large<VEC, PHASED, MODE>: a grid of one wave at the kernel's
// occupancy (resident blocks per SM are queried once per instantiation), each
// group walking an equal contiguous run of rows, at least kLargeMinRows of them.
constexpr int64_t kLargeMinRows = 64;

// One warp as tile 1 of a two-tile chain whose tile 0 never publishes: the
// lookback must give up after its bound and record the timeout.
__global__ void __launch_bounds__(32) k_check_wait_bound(Chain ch, const float* s, int32_t* status) {
    __shared__ LookbackSmem<1, 32> lb;
    bool has = false;
    (void)block_lookback<1, false, 32>(ch, 1, 2, s, 2, 1, LP{1.f, 1.f}, s[1], s[0], status, lb, has);
}

// Dynamic shared memory of k_large<VEC, PHASED, MODE>: the fp64 partials, plus the
// staging ring when the groups are wide and the mode gathers rows.
template <int VEC, bool PHASED, int MODE>
size_t large_smem_bytes(bool wide) {
    constexpr int NP = PHASED ? 2 : 1;
    constexpr int ND = (MODE & kLmAccum) ? 2 * NP * VEC : 1;
    constexpr bool ROWS = (MODE & (kLmAccum | kLmGrad)) != 0;
    const size_t ring = (wide && ROWS) ? sizeof(float) * 8 * 2 * kLargeBatch<VEC, PHASED, MODE> * 32 * VEC : 0;
    return sizeof(double) * ND * 256 + ring;
}

template <int VEC, bool PHASED, int MODE>
cudaError_t launch_large(LargePass A, int chunks, const char* name, cudaStream_t st) {
    const bool wide = A.lpr >= kLargeBatch<VEC, PHASED, MODE>;
    const size_t smem = large_smem_bytes<VEC, PHASED, MODE>(wide);
    static PerDevice occ_dev[2];
    int& occ_w = occ_dev[wide].here();
    if (occ_w == 0) {
        int o = 1;
        cudaFuncSetAttribute(k_large<VEC, PHASED, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)large_smem_bytes<VEC, PHASED, MODE>(true));
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k_large<VEC, PHASED, MODE>, 256, smem) != cudaSuccess)
            o = 1;
        occ_w = std::max(o, 1);
    }
    const int occ_here = occ_w;
    const int64_t groups_per_block = 8 * (32 / A.lpr);
    const int64_t wave = std::max<int64_t>(1, (int64_t)sm_count() * occ_here / chunks);
    const int64_t need = (A.m + groups_per_block * kLargeMinRows - 1) / (groups_per_block * kLargeMinRows);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(wave, need));
    A.rows_per_group = (A.m + blocks * groups_per_block - 1) / (blocks * groups_per_block);
    const dim3 grid((unsigned)blocks, (unsigned)chunks);
    LAPLEX_TIMED(name, st, k_large<VEC, PHASED, MODE><<<grid, 256, smem, st>>>(A));
    return cudaGetLastError();
}

template <int VEC, bool PHASED>
cudaError_t large_mode(LargePass A, int mode, int chunks, cudaStream_t st) {
    switch (mode) {
        case kLmExpand: return launch_large<VEC, PHASED, kLmExpand>(A, chunks, "large_expand", st);
        case kLmAccum: return launch_large<VEC, PHASED, kLmAccum>(A, chunks, "large_accum", st);
        case kLmGrad: return launch_large<VEC, PHASED, kLmGrad>(A, chunks, "large_grad", st);
        case kLmExpand | kLmGrad:
            return launch_large<VEC, PHASED, kLmExpand | kLmGrad>(A, chunks, "large_expand_grad", st);
        case kLmAccum | kLmGrad:
            return launch_large<VEC, PHASED, kLmAccum | kLmGrad>(A, chunks, "large_accum_grad", st);
        default: return cudaErrorInvalidValue;
    }
}

// Grid of the lean large-side kernels: one wave at the kernel's occupancy, each
// group of LPR lanes walking an equal contiguous run of at least kLargeMinRows rows.
int64_t lean_grid(LargePass& A, int lpr, int chunks, int occ) {
    const int64_t groups_per_block = 8 * (32 / lpr);
    const int64_t wave = std::max<int64_t>(1, (int64_t)sm_count() * occ / chunks);
    const int64_t need = (A.m + groups_per_block * kLargeMinRows - 1) / (groups_per_block * kLargeMinRows);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(wave, need));
    A.rows_per_group = (A.m + blocks * groups_per_block - 1) / (blocks * groups_per_block);
    return blocks;
}

template <int LPR, bool PHASED>
cudaError_t launch_large_accum_w(LargePass A, int chunks, cudaStream_t st) {
    constexpr int NP = PHASED ? 2 : 1;
    const size_t smem = sizeof(double) * 2 * NP * 4 * 256 + sizeof(AccumSlot) * 8 * kLeanSlots<LPR>;
    static PerDevice occ_dev;
    int& occ = occ_dev.here();
    if (occ == 0) {
        int o = 1;
        cudaFuncSetAttribute(k_large_accum_w<LPR, PHASED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k_large_accum_w<LPR, PHASED>, 256, smem) != cudaSuccess)
            o = 1;
        occ = std::max(o, 1);
    }
    const int64_t blocks = lean_grid(A, LPR, chunks, occ);
    const dim3 grid((unsigned)blocks, (unsigned)chunks);
    LAPLEX_TIMED("large_accum", st, k_large_accum_w<LPR, PHASED><<<grid, 256, smem, st>>>(A));
    return cudaGetLastError();
}

template <int LPR, bool PHASED, bool EXPAND, bool GRAD>
cudaError_t launch_large_expand_w(LargePass A, int chunks, const char* name, cudaStream_t st) {
    static PerDevice occ_dev;
    int& occ = occ_dev.here();
    if (occ == 0) {
        int o = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k_large_expand_w<LPR, PHASED, EXPAND, GRAD>, 256, 0) !=
            cudaSuccess)
            o = 1;
        occ = std::max(o, 1);
    }
    const int64_t blocks = lean_grid(A, LPR, chunks, occ);
    const dim3 grid((unsigned)blocks, (unsigned)chunks);
    LAPLEX_TIMED(name, st, k_large_expand_w<LPR, PHASED, EXPAND, GRAD><<<grid, 256, 0, st>>>(A));
    return cudaGetLastError();
}

template <int LPR>
cudaError_t lean_accum(LargePass A, bool phased, int chunks, cudaStream_t st) {
    return phased ? launch_large_accum_w<LPR, true>(A, chunks, st) : launch_large_accum_w<LPR, false>(A, chunks, st);
}

template <int LPR>
cudaError_t lean_expand(LargePass A, bool phased, int chunks, cudaStream_t st) {
    return phased ? launch_large_expand_w<LPR, true, true, false>(A, chunks, "large_expand", st)
                  : launch_large_expand_w<LPR, false, true, false>(A, chunks, "large_expand", st);
}

template <int LPR, bool PHASED>
cudaError_t launch_large_accgrad_n(LargePass A, int chunks, cudaStream_t st) {
    constexpr int NP = PHASED ? 2 : 1;
    const size_t smem = sizeof(double) * 2 * NP * 4 * 256 + sizeof(AccGradSlot) * 8 * kLeanSlots<LPR>;
    static PerDevice occ_dev;
    int& occ = occ_dev.here();
    if (occ == 0) {
        int o = 1;
        cudaFuncSetAttribute(k_large_accgrad_n<LPR, PHASED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k_large_accgrad_n<LPR, PHASED>, 256, smem) !=
            cudaSuccess)
            o = 1;
        occ = std::max(o, 1);
    }
    const int64_t blocks = lean_grid(A, LPR, chunks, occ);
    const dim3 grid((unsigned)blocks, (unsigned)chunks);
    LAPLEX_TIMED("large_accum_grad", st, k_large_accgrad_n<LPR, PHASED><<<grid, 256, smem, st>>>(A));
    return cudaGetLastError();
}

template <int LPR>
cudaError_t lean_accgrad(LargePass A, int chunks, cudaStream_t st) {
    return launch_large_accgrad_n<LPR, false>(A, chunks, st);
}

cudaError_t large_pass(LargePass A, int mode, cudaStream_t st) {
    const bool phased = A.theta != nullptr;
    if (A.Bs == 0) A.Bs = A.B;
    const int vec = (A.B % 4 == 0 && A.Bs % 4 == 0) ? 4 : 1;
    int lpr = 1;
    while (lpr < 32 && lpr * vec < A.B) lpr <<= 1;
    const int chunks = (A.B + lpr * vec - 1) / (lpr * vec);
    A.lpr = lpr;
    A.chunk_atomic = chunks > 1 ? 1 : 0;
    if ((mode & kLmGrad) && A.chunk_atomic && !A.accumulate) {
        if (A.g_anchor) LAPLEX_TRY(cudaMemsetAsync(A.g_anchor, 0, sizeof(float) * A.m, st));
        if (A.g_phase) LAPLEX_TRY(cudaMemsetAsync(A.g_phase, 0, sizeof(float) * A.m, st));
    }
    if (mode == kLmAccum && vec == 4) {  // the lean interval-sum pass, every group width
        switch (lpr) {
            case 1: break;  // one lane per row: k_large
            case 2: return lean_accum<2>(A, phased, chunks, st);
            case 4: return lean_accum<4>(A, phased, chunks, st);
            case 8: return lean_accum<8>(A, phased, chunks, st);
            case 16: return lean_accum<16>(A, phased, chunks, st);
            default: return lean_accum<32>(A, phased, chunks, st);
        }
    }
    // the lean sums + gradients pass, narrow unphased groups (the phased one holds three
    // more state arrays and would spill: k_large)
    if (mode == (kLmAccum | kLmGrad) && vec == 4 && !phased) {
        switch (lpr) {
            case 2: return lean_accgrad<2>(A, chunks, st);
            case 4: return lean_accgrad<4>(A, chunks, st);
            case 8: return lean_accgrad<8>(A, chunks, st);
            case 16: return lean_accgrad<16>(A, chunks, st);
            default: break;  // one lane per row, or full warps: k_large
        }
    }
    // the lean output pass for full-warp groups (narrow groups measured faster in k_large:
    // Gram image y = A (D w), two lanes per row, 0.090 against 0.081 ms)
    if (mode == kLmExpand && vec == 4 && lpr == 32) return lean_expand<32>(A, phased, chunks, st);
    if (vec == 4 && lpr == 32 && (mode & kLmAccum) == 0) {  // full-warp groups: the lean gradient pass
        switch (mode | (phased ? 8 : 0)) {
            case kLmGrad: return launch_large_expand_w<32, false, false, true>(A, chunks, "large_grad", st);
            case kLmExpand | kLmGrad:
                return launch_large_expand_w<32, false, true, true>(A, chunks, "large_expand_grad", st);
            case 8 | kLmGrad: return launch_large_expand_w<32, true, false, true>(A, chunks, "large_grad", st);
            case 8 | kLmExpand | kLmGrad:
                return launch_large_expand_w<32, true, true, true>(A, chunks, "large_expand_grad", st);
            default: return cudaErrorInvalidValue;
        }
    }
    if (vec == 4) return phased ? large_mode<4, true>(A, mode, chunks, st) : large_mode<4, false>(A, mode, chunks, st);
    return phased ? large_mode<1, true>(A, mode, chunks, st) : large_mode<1, false>(A, mode, chunks, st);
}

cudaError_t finish(Finish F, cudaStream_t st) {
    const unsigned blocks = (unsigned)((F.m + 7) / 8);
    if (F.theta)
        LAPLEX_TIMED("finish", st, k_finish<true><<<blocks, 256, 0, st>>>(F));
    else
        LAPLEX_TIMED("finish", st, k_finish<false><<<blocks, 256, 0, st>>>(F));
    return cudaGetLastError();
}

SideScan values_scan(Side S, const float* X, int64_t B, float* P, float* Sout) {
    SideScan a{};
    a.s = S.s;
    a.perm = S.rows_sorted ? nullptr : S.perm;  // no permutation: row r is sorted row r
    a.theta = S.theta;
    a.m = S.m;
    a.X = X;
    a.B = (int)B;
    a.o0 = P;
    a.o1 = Sout;
    return a;
}

SideScan bins_scan(Side S, const RectPlan& p, int64_t B, float* ZL, float* ZR, float* ZF) {
    SideScan a{};
    a.s = S.s;
    a.perm = S.perm;
    a.m = S.m;
    a.B = (int)B;
    const int64_t sz = p.ms * (int64_t)p.Cb;
    a.U = p.bins;
    a.TL = p.bins + sz;
    a.V = p.bins + 2 * sz;
    a.TR = p.bins + 3 * sz;
    a.o0 = ZL;
    a.o1 = ZR;
    a.o2 = ZF;
    return a;
}

LargePass large_args(Side L, Side Sm, const RectPlan& p, int64_t B) {
    LargePass A{};
    A.s = L.s;
    A.perm = L.perm;
    A.theta = L.theta;
    A.m = L.m;
    A.sp = Sm.s;
    A.ms = Sm.m;
    A.B = (int)B;
    A.Bs = (int)B;
    A.rows2 = nullptr;
    A.Cb = p.Cb;
    const int64_t sz = p.ms * (int64_t)p.Cb;
    A.U = p.bins;
    A.TL = p.bins + sz;
    A.V = p.bins + 2 * sz;
    A.TR = p.bins + 3 * sz;
    return A;
}


// Reduce path of the forward: interval sums of x (at I) into O's bins, scan over
// O, parts written to ZL/ZR/ZF.
cudaError_t reduce_parts(const RectPlan& p, Side O, Side I, const float* x, int64_t B, float* ZL, float* ZR, float* ZF,
                         int32_t* status, cudaStream_t st, const float* x2 = nullptr) {
    LAPLEX_TRY(cudaMemsetAsync(p.bins, 0, sizeof(double) * 4 * p.ms * p.Cb, st));
    LargePass A = large_args(I, O, p, B);
    A.rows = x;
    if (x2 != nullptr) {  // paired pass: channels [0, B/2) from x, [B/2, B) from x2
        A.rows2 = x2;
        A.Bs = (int)(B / 2);
    }
    LAPLEX_TRY(large_pass(A, kLmAccum, st));
    return side_scan(p, bins_scan(O, p, B, ZL, ZR, ZF), true, status, st);
}

}  // namespace

size_t rect_workspace_bytes(int64_t n_out, int64_t n_in, int64_t B, bool phased) {
    return plan_rect(n_out, n_in, B, phased, nullptr).total;
}

size_t rect_saved_bytes(int64_t n_out, int64_t n_in, int64_t B, bool phased) {
    const int64_t Cb = phased ? 2 * B : B;
    return (n_in <= n_out) ? sizeof(float) * 2 * n_in * Cb : sizeof(float) * 3 * n_out * Cb;
}

cudaError_t launch_rect_forward(Side O, Side I, const float* x, int64_t B, float* out, void* saved, void* ws,
                                int32_t* status, cudaStream_t st) {
    const RectPlan p = plan_rect(O.m, I.m, B, O.theta != nullptr, ws);
    const int64_t sz = p.ms * (int64_t)p.Cb;
    if (I.m <= O.m) {  // expand
        float* P = saved ? (float*)saved : p.bufA;
        float* S = P + sz;
        LAPLEX_TRY(side_scan(p, values_scan(I, x, B, P, S), false, status, st));
        LargePass A = large_args(O, I, p, B);
        A.Pst = P;
        A.Sst = S;
        A.out = out;
        return large_pass(A, kLmExpand, st);
    }
    float* ZL = saved ? (float*)saved : p.bufA;  // reduce
    LAPLEX_TRY(reduce_parts(p, O, I, x, B, ZL, ZL + sz, ZL + 2 * sz, status, st));
    Finish F{};
    F.perm = O.perm;
    F.theta = O.theta;
    F.m = O.m;
    F.ZL = ZL;
    F.ZR = ZL + sz;
    F.ZF = ZL + 2 * sz;
    F.B = (int)B;
    F.Cb = p.Cb;
    F.out = out;
    return finish(F, st);
}

cudaError_t launch_rect_backward(Side O, Side I, const float* x, const float* g, int64_t B, const void* saved,
                                 float* gx, float* gO, float* gI, float* gtO, float* gtI, void* ws, int32_t* status,
                                 cudaStream_t st, bool accumulate, const float* g2) {
    const bool phased = O.theta != nullptr;
    // paired rows: only the pass over a larger output side takes them
    if (g2 != nullptr && (O.m <= I.m || phased || (B % 2) != 0 || gx != nullptr)) return cudaErrorInvalidValue;
    const RectPlan p = plan_rect(O.m, I.m, B, phased, ws);
    const int64_t sz = p.ms * (int64_t)p.Cb;
    if (!phased) gtO = gtI = nullptr;
    const bool needI = gx || gI || gtI;  // quantities at the input side
    const bool needO = gO || gtO;        // quantities at the output side
    if (O.m <= I.m) {
        if (needI) {  // C = E(I, O)(w_O g): scan g over O, expand over I
            float* P = p.bufB;
            float* S = P + sz;
            LAPLEX_TRY(side_scan(p, values_scan(O, g, B, P, S), false, status, st));
            LargePass A = large_args(I, O, p, B);
            A.rows = x;
            A.Pst = P;
            A.Sst = S;
            A.out = gx;
            A.g_anchor = gI;
            A.g_phase = gtI;
            A.accumulate = accumulate;
            const int mode = (gx ? kLmExpand : 0) | ((gI || gtI) ? kLmGrad : 0);
            LAPLEX_TRY(large_pass(A, mode, st));
        }
        if (needO) {
            if (I.m > O.m) {  // the forward reduced: parts of E(O, I) x at O
                const float* Z = (const float*)saved;
                if (Z == nullptr) {
                    LAPLEX_TRY(reduce_parts(p, O, I, x, B, p.bufA, p.bufA + sz, p.bufA + 2 * sz, status, st));
                    Z = p.bufA;
                }
                Finish F{};
                F.perm = O.perm;
                F.theta = O.theta;
                F.m = O.m;
                F.ZL = Z;
                F.ZR = Z + sz;
                F.ZF = Z + 2 * sz;
                F.B = (int)B;
                F.Cb = p.Cb;
                F.h = g;
                F.h_sorted = O.rows_sorted;
                F.g_anchor = gO;
                F.g_phase = gtO;
                F.accumulate = accumulate;
                if (gO == nullptr) {
                    // k_finish keys the anchor sums on g_anchor; phase-only still needs a target
                    F.g_anchor = nullptr;
                }
                LAPLEX_TRY(finish(F, st));
            } else {  // equal sizes: the forward expanded over O from states at I
                const float* Pst = (const float*)saved;
                if (Pst == nullptr) {
                    LAPLEX_TRY(side_scan(p, values_scan(I, x, B, p.bufA, p.bufA + sz), false, status, st));
                    Pst = p.bufA;
                }
                LargePass A = large_args(O, I, p, B);
                A.rows = g;
                A.Pst = Pst;
                A.Sst = Pst + sz;
                A.g_anchor = gO;
                A.g_phase = gtO;
                A.accumulate = accumulate;
                LAPLEX_TRY(large_pass(A, kLmGrad, st));
            }
        }
        return cudaSuccess;
    }
    // O larger than I: one pass over O sums g into I's bins and, with the states of
    // x at I, forms the output-side gradients; then scan over I and finish there.
    const float* Pst = (const float*)saved;
    if (needO && Pst == nullptr) {
        LAPLEX_TRY(side_scan(p, values_scan(I, x, B, p.bufA, p.bufA + sz), false, status, st));
        Pst = p.bufA;
    }
    if (needI) LAPLEX_TRY(cudaMemsetAsync(p.bins, 0, sizeof(double) * 4 * sz, st));
    const int mode = (needI ? kLmAccum : 0) | (needO ? kLmGrad : 0);
    if (mode != 0) {
        LargePass A = large_args(O, I, p, B);
        A.rows = g;
        if (g2 != nullptr) {  // channels [0, B/2) of a row from g, [B/2, B) from g2
            A.rows2 = g2;
            A.Bs = (int)(B / 2);
        }
        A.Pst = Pst;
        A.Sst = Pst ? Pst + sz : nullptr;
        A.g_anchor = gO;
        A.g_phase = gtO;
        A.accumulate = accumulate;
        LAPLEX_TRY(large_pass(A, mode, st));
    }
    if (needI) {
        float* CL = p.bufB;
        LAPLEX_TRY(side_scan(p, bins_scan(I, p, B, CL, CL + sz, CL + 2 * sz), true, status, st));
        Finish F{};
        F.perm = I.perm;
        F.theta = I.theta;
        F.m = I.m;
        F.ZL = CL;
        F.ZR = CL + sz;
        F.ZF = CL + 2 * sz;
        F.B = (int)B;
        F.Cb = p.Cb;
        F.h = x;
        F.h_sorted = I.rows_sorted;
        F.out = gx;
        F.g_anchor = gI;
        F.g_phase = gtI;
        F.accumulate = accumulate;
        LAPLEX_TRY(finish(F, st));
    }
    return cudaSuccess;
}

cudaError_t launch_check_wait_bound(void* ws, int32_t* status, cudaStream_t st) {
    // ws: flags [2] | agg [2] | inc [2] | anchors [2]
    char* b = (char*)ws;
    LAPLEX_TRY(cudaMemsetAsync(b, 0, 256, st));
    Chain ch{(int*)b, (double2*)(b + 64), (double2*)(b + 128)};
    const float* s = (const float*)(b + 192);  // anchors 0, 0 (zeroed)
    LAPLEX_TIMED("check_wait_bound", st, k_check_wait_bound<<<1, 32, 0, st>>>(ch, s, status));
    return cudaGetLastError();
}

// The middle of the Gram backward after separate passes, one warp per small-side
// row j (original order): x1 = D_j w_j, x2 = D_j u_j (the inputs of the general
// products A (D w) and A (D u)) and gD_j = <u_j, w_j>.  w and u are rows of ld floats.
__global__ void __launch_bounds__(256) k_gram_mid2(const float* __restrict__ D, const float* __restrict__ w,
                                                   const float* __restrict__ u, int ld, float* __restrict__ x1,
                                                   float* __restrict__ x2, float* __restrict__ gD, int64_t k, int B) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= k) return;
    const int lane = threadIdx.x & 31;
    const float d = __ldg(D + r);
    float acc = 0.f;
    for (int c = lane; c < B; c += 32) {
        const float wv = __ldg(w + r * ld + c), uv = __ldg(u + r * ld + c);
        x1[r * B + c] = d * wv;
        x2[r * B + c] = d * uv;
        acc = fmaf(uv, wv, acc);
    }
    if (gD != nullptr) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) gD[r] = acc;
    }
}

// Workspace of the Gram apply: the rectangular scratch sized for the paired pass
// (2B channels), then three [k][2B] row buffers.
size_t gram_workspace_bytes(int64_t n, int64_t k, int64_t B) {
    return plan_rect(n, k, 2 * B, false, nullptr, k).total;
}

cudaError_t launch_gram(Side A, Side Bs, const float* D, const float* v, int64_t B, float* y, float* w_saved,
                        const float* g, float* gD, void* ws, int32_t* status, cudaStream_t st) {
    const RectPlan p2 = plan_rect(A.m, Bs.m, 2 * B, false, ws, Bs.m);  // layout: rows3 after the paired scratch
    const int64_t kb = Bs.m * B;
    float* wpair = p2.rows3;      // [k][2B]: A^T v | A^T g (separate passes)
    float* w2 = p2.rows3 + 2 * kb;  // [k][B]: D (A^T v); in b's sorted order after the paired pass
    if (g != nullptr && gD != nullptr && A.m > Bs.m) {
        // A^T v and A^T g in one reduce pass over the pixel side (2B channels)
        const RectPlan pp = plan_rect(Bs.m, A.m, 2 * B, false, ws);
        const int64_t sz = pp.ms * (int64_t)pp.Cb;
        LAPLEX_TRY(reduce_parts(pp, Bs, A, v, 2 * B, pp.bufA, pp.bufA + sz, pp.bufA + 2 * sz, status, st, g));
        // w2 = D w in b's sorted order, so the expand reads b's side without the permutation
        LAPLEX_TRY(launch_gram_mid_sorted<false>(Bs.perm, D, pp.bufA + 2 * sz, pp.Cb, w2, (int)B, w_saved, gD, Bs.m,
                                                 B, st));
        const Side Bss{Bs.s, Bs.perm, nullptr, Bs.m, true};
        return launch_rect_forward(A, Bss, w2, B, y, nullptr, ws, status, st);  // y = A (D w)
    }
    float* w = w_saved ? w_saved : wpair;
    float* wg = wpair + kb;
    LAPLEX_TRY(launch_rect_forward(Bs, A, v, B, w, nullptr, ws, status, st));  // w = A^T v
    if (g != nullptr && gD != nullptr)
        LAPLEX_TRY(launch_rect_forward(Bs, A, g, B, wg, nullptr, ws, status, st));  // A^T g
    LAPLEX_TIMED("gram_mid", st,
                 k_gram_mid<<<(unsigned)((Bs.m + 7) / 8), 256, 0, st>>>(D, w, B, (g && gD) ? wg : nullptr, w2,
                                                                       nullptr, (g && gD) ? gD : nullptr, Bs.m, (int)B));
    LAPLEX_TRY(cudaGetLastError());
    return launch_rect_forward(A, Bs, w2, B, y, nullptr, ws, status, st);  // y = A (D w)
}

// Every gradient of l = <g, A diag(D) A^T v>: with w = A^T v and u = A^T g,
// gv = A (D u), gD = sum_c u w, and ga, gb the anchor gradients of the general
// products A (D w) read by g and A (D u) read by v (dl/dA_ij = D_j sum_c (g_ic w_jc
// + v_ic u_jc)); the second backward adds into the first's ga, gb.
cudaError_t launch_gram_backward(Side A, Side Bs, const float* D, const float* v, const float* g, int64_t B,
                                 float* gv, float* ga, float* gb, float* gD, void* ws, int32_t* status,
                                 cudaStream_t st) {
    const RectPlan p2 = plan_rect(A.m, Bs.m, 2 * B, false, ws, Bs.m);
    const int64_t kb = Bs.m * B;
    float* wpair = p2.rows3;           // w | u ([k][B] each, separate passes)
    float* x1 = p2.rows3 + 2 * kb;     // [k][B]  D w
    float* x2 = p2.rows3 + 3 * kb;     // [k][B]  D u
    float* xp = p2.rows3 + 4 * kb;     // [k][2B] D w | D u in b's sorted order (paired pass)
    const bool need_ab = ga != nullptr || gb != nullptr;
    if (A.m > Bs.m) {
        // A^T v and A^T g in one paired reduce pass; then D w | D u (and gD) in b's
        // sorted order, and the scan states of D w | D u over b, once: the paired
        // backward reads them, and their second half (D u) gives gv = A (D u)
        const RectPlan pp = plan_rect(Bs.m, A.m, 2 * B, false, ws);
        const int64_t sz = pp.ms * (int64_t)pp.Cb;
        LAPLEX_TRY(reduce_parts(pp, Bs, A, v, 2 * B, pp.bufA, pp.bufA + sz, pp.bufA + 2 * sz, status, st, g));
        LAPLEX_TRY(launch_gram_mid_sorted<true>(Bs.perm, D, pp.bufA + 2 * sz, pp.Cb, xp, (int)(2 * B), nullptr, gD,
                                                Bs.m, B, st));
        if (gv == nullptr && !need_ab) return cudaSuccess;
        const Side Bss{Bs.s, Bs.perm, nullptr, Bs.m, true};
        const RectPlan pb = plan_rect(A.m, Bs.m, 2 * B, false, ws);
        const int64_t szb = pb.ms * (int64_t)pb.Cb;
        float* P = pb.bufA;
        LAPLEX_TRY(side_scan(pb, values_scan(Bss, xp, 2 * B, P, P + szb), false, status, st));
        if (gv != nullptr) {
            LargePass E = large_args(A, Bss, pb, B);  // B channels, states with the 2B-channel stride
            E.Pst = P + B;
            E.Sst = P + szb + B;
            E.out = gv;
            LAPLEX_TRY(large_pass(E, kLmExpand, st));
        }
        // both general products in one backward over 2B channels: inputs D w | D u at
        // b, rows g | v at a (ga sums over all 2B channels, and so does gb)
        if (need_ab)
            LAPLEX_TRY(launch_rect_backward(A, Bss, xp, g, 2 * B, P, nullptr, ga, gb, nullptr, nullptr, ws, status, st,
                                            false, v));
        return cudaSuccess;
    }
    LAPLEX_TRY(launch_rect_forward(Bs, A, v, B, wpair, nullptr, ws, status, st));       // w = A^T v
    LAPLEX_TRY(launch_rect_forward(Bs, A, g, B, wpair + kb, nullptr, ws, status, st));  // u = A^T g
    LAPLEX_TIMED("gram_mid", st,
                 k_gram_mid2<<<(unsigned)((Bs.m + 7) / 8), 256, 0, st>>>(D, wpair, wpair + kb, (int)B, x1, x2, gD,
                                                                        Bs.m, (int)B));
    LAPLEX_TRY(cudaGetLastError());
    if (gv != nullptr) LAPLEX_TRY(launch_rect_forward(A, Bs, x2, B, gv, nullptr, ws, status, st));  // gv = A (D u)
    if (need_ab) {
        LAPLEX_TRY(launch_rect_backward(A, Bs, x1, g, B, nullptr, nullptr, ga, gb, nullptr, nullptr, ws, status, st,
                                        false));
        LAPLEX_TRY(launch_rect_backward(A, Bs, x2, v, B, nullptr, nullptr, ga, gb, nullptr, nullptr, ws, status, st,
                                        true));
    }
    return cudaSuccess;
}

}  // namespace laplex
