// Symmetric LAPLEX operator y = K x, K_ij = exp(-|a_i - a_j|), and its backward
// ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary section 2.2,
// "symmetric case": after sorting, the lower triangle is the prefix scan
// P_r = x_r + exp(a_(r-1) - a_(r)) P_(r-1), the upper triangle the mirrored suffix
// scan S_r, and y = P + S - x because both contain the diagonal).
//
// Both directions of the scan are needed at every row, and the vectors do not
// fit on chip, so each product reads its input twice.  The two reads are made
// free of inter-tile waits by partitioning the sorted rows into P contiguous
// ranges of tiles, one persistent CTA per (range, channel group):
//   k_sym_agg    walks its range right to left and writes, per tile, the fp64
//                suffix state of the range from that tile's first row on (RS),
//                and the range's aggregates in both directions;
//   k_sym_carry  scans the P range aggregates (one CTA per channel group) into
//                the fp64 carries entering each range from the left and right;
//   k_sym_sweep  walks its range left to right, folding the left state tile by
//                tile and taking the right state from RS and the range carry,
//                evaluates both directions inside each tile and writes
//                y = P + S - x through the permutation (forward), or, over x and
//                g at once, gx = K g = P_g + S_g - g and
//                ga = sum_c g (R_x - L_x) + x (R_g - L_g) from the strict sums
//                (ties excluded: sign(0) = 0); x's RS and carries come from the
//                forward (the `saved` buffer) or are recomputed.
// Every tile is staged with cp.async: anchors and permutation two tiles ahead,
// the gathered rows one tile ahead, so the gathers of the next tile overlap the
// arithmetic of the current one.  No kernel waits on another CTA.
#include "laplex_internal.h"
#include "pipeline.cuh"

namespace laplex {

namespace {

constexpr int kNT = 256;
constexpr int kMaxRanges = 1024;  // per channel group
constexpr int kRangesPerSM = 3;

template <int C>
using SymGeo = TileGeo<C, kNT, (C == 1 ? 8 : 16)>;

struct SymScan {
    const float* s;
    const uint32_t* perm;
    int64_t n;
    int B;
    int64_t T;    // tiles per channel group
    int P;        // ranges per channel group
    int64_t tpr;  // tiles per range
};

// fp64 scan state of one vector, per channel group, range j, tile t and channel c
struct RangeState {
    double2* RS;    // [G][T][C]  right state from tile t's first row to the range's end
    double2* Lagg;  // [G][P][C]  range aggregate, left direction (anchored at its last row)
    double2* Ragg;  // [G][P][C]  range aggregate, right direction (anchored at -its first row)
    double2* Lin;   // [G][P][C]  carry from the ranges before (anchored at the row before)
    double2* Rin;   // [G][P][C]  carry from the ranges after (anchored at -the row after)
};

template <int C, int NV>
struct SymSmem {
    using G = SymGeo<C>;
    float s[3][G::SS];
    uint32_t p[3][G::R];
    float v[NV][2][G::XS];
    float dl[G::R + 4];
    ScanSmem<C, kNT / 32> sc[2 * NV];
    double2 carry[2 * NV][C];
    int has[2 * NV];
};

__device__ __forceinline__ int64_t tile_lo(int64_t t, int R) { return t * (int64_t)R; }

// ------------------------------------------------------------------ pass A

template <int C>
__global__ void __launch_bounds__(kNT, 3) k_sym_agg(SymScan a, const float* __restrict__ v, RangeState st) {
    using G = SymGeo<C>;
    constexpr int E = G::E, R = G::R;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SymSmem<C, 1>& sm = *reinterpret_cast<SymSmem<C, 1>*>(smem_raw);
    const int grp = blockIdx.y, j = blockIdx.x;
    const int64_t tb = (int64_t)j * a.tpr, te = min(a.T, tb + a.tpr);
    const int nt = (int)(te - tb);
    const int c = threadIdx.x % C, k = threadIdx.x / C, ch0 = grp * C;
    // walk t = te-1, te-2, ..., tb
    stage_meta<G>(a.s, a.perm, a.n, tile_lo(te - 1, R), sm.s[0], sm.p[0]);
    cp_async_commit();
    if (nt > 1) stage_meta<G>(a.s, a.perm, a.n, tile_lo(te - 2, R), sm.s[1], sm.p[1]);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    stage_rows<G>(v, a.B, ch0, a.n, tile_lo(te - 1, R), sm.p[0], sm.v[0][0]);
    cp_async_commit();
    double2 runR = make_double2(0.0, 0.0), runL = make_double2(0.0, 0.0);
    float uRunR = 0.f, uRunL = 0.f;
    for (int i = 0; i < nt; ++i) {
        const int64_t t = te - 1 - i;
        cp_async_wait_all();
        __syncthreads();
        if (i + 1 < nt) stage_rows<G>(v, a.B, ch0, a.n, tile_lo(t - 1, R), sm.p[(i + 1) % 3], sm.v[0][(i + 1) & 1]);
        cp_async_commit();
        if (i + 2 < nt) stage_meta<G>(a.s, a.perm, a.n, tile_lo(t - 2, R), sm.s[(i + 2) % 3], sm.p[(i + 2) % 3]);
        cp_async_commit();
        const float* sb = sm.s[i % 3];
        const float* xb = sm.v[0][i & 1] + k * G::SEG + c;
        tile_decays<G>(sb, sm.dl);
        __syncthreads();
        LP str = {0.f, 0.f}, stl = {0.f, 0.f};
#pragma unroll
        for (int e = E - 1; e >= 0; --e) str = lp_step_d(str, sm.dl[k * E + e + 1], 0.f, xb[e * C]);
#pragma unroll
        for (int e = 0; e < E; ++e) stl = lp_step_d(stl, sm.dl[k * E + e], 0.f, xb[e * C]);
        LP ex;
        bool hx;
        block_scan_dir<C, kNT, true>(str, -sb[4 + k * E], -sb[4 + k * E + E], sm.sc[0], ex, hx);
        block_scan_dir<C, kNT, false>(stl, sb[4 + k * E + E - 1], sb[4 + k * E - 1], sm.sc[1], ex, hx);
        if (threadIdx.x < C) {
            const LP tr = sm.sc[0].tot[c], tl = sm.sc[1].tot[c];
            const double2 trd = make_double2(tr.L, tr.P), tld = make_double2(tl.L, tl.P);
            const float u_first = -sb[4], u_last = sb[4 + R - 1];
            runR = (i == 0) ? trd : lpd_combine(runR, uRunR, trd, u_first);
            uRunR = u_first;
            st.RS[((int64_t)grp * a.T + t) * C + c] = runR;
            if (i == 0) {
                runL = tld;
                uRunL = u_last;
            } else {
                runL = lpd_combine(tld, u_last, runL, uRunL);
            }
        }
    }
    if (threadIdx.x < C) {
        st.Lagg[((int64_t)grp * a.P + j) * C + c] = runL;
        st.Ragg[((int64_t)grp * a.P + j) * C + c] = runR;
    }
}

// ------------------------------------------------------------------ pass B

// One CTA per channel group.  Thread (c, q), q < QS, folds a contiguous block of
// ranges; the blocks are then composed serially (at most QS steps) and re-walked
// to produce the carry entering every range.
template <int C>
__global__ void __launch_bounds__(kNT) k_sym_carry(SymScan a, RangeState st) {
    constexpr int QS = (kNT / C) < 16 ? (kNT / C) : 16;
    __shared__ double2 segL[QS][C], segR[QS][C];
    const int grp = blockIdx.x;
    const int c = threadIdx.x % C, q = threadIdx.x / C;
    const int P = a.P;
    const int PS = (P + QS - 1) / QS;
    const int j0 = min(P, q * PS), j1 = min(P, j0 + PS);
    const int64_t RR = a.tpr * (int64_t)SymGeo<C>::R;  // rows per range
    auto uL = [&](int jj) { return __ldg(a.s + min(a.n, (jj + 1) * RR) - 1); };  // left anchor of range jj
    auto uR = [&](int jj) { return -__ldg(a.s + jj * RR); };                    // right anchor of range jj
    const int64_t base = (int64_t)grp * P * C + c;
    const bool mine = q < QS && j0 < j1;
    if (mine) {
        double2 fl = st.Lagg[base + (int64_t)j0 * C];
        for (int jj = j0 + 1; jj < j1; ++jj) fl = lpd_combine(fl, uL(jj - 1), st.Lagg[base + (int64_t)jj * C], uL(jj));
        double2 fr = st.Ragg[base + (int64_t)(j1 - 1) * C];
        for (int jj = j1 - 2; jj >= j0; --jj)
            fr = lpd_combine(fr, uR(jj + 1), st.Ragg[base + (int64_t)jj * C], uR(jj));
        segL[q][c] = fl;
        segR[q][c] = fr;
    }
    __syncthreads();
    if (mine) {
        bool hl = false;  // carry entering block q from the left: blocks 0 .. q-1
        double2 cl = make_double2(0.0, 0.0);
        for (int qq = 0; qq < q; ++qq) {
            const int a0 = qq * PS, a1 = min(P, a0 + PS);
            if (a0 >= a1) continue;
            cl = hl ? lpd_combine(cl, uL(a0 - 1), segL[qq][c], uL(a1 - 1)) : segL[qq][c];
            hl = true;
        }
        bool hr = false;  // from the right: blocks QS-1 .. q+1
        double2 cr = make_double2(0.0, 0.0);
        for (int qq = QS - 1; qq > q; --qq) {
            const int a0 = qq * PS, a1 = min(P, a0 + PS);
            if (a0 >= a1) continue;
            cr = hr ? lpd_combine(cr, uR(a1), segR[qq][c], uR(a0)) : segR[qq][c];
            hr = true;
        }
        for (int jj = j0; jj < j1; ++jj) {
            st.Lin[base + (int64_t)jj * C] = cl;  // zero (unused) for the first range
            const double2 ag = st.Lagg[base + (int64_t)jj * C];
            cl = hl ? lpd_combine(cl, uL(jj - 1), ag, uL(jj)) : ag;
            hl = true;
        }
        for (int jj = j1 - 1; jj >= j0; --jj) {
            st.Rin[base + (int64_t)jj * C] = cr;  // zero (unused) for the last range
            const double2 ag = st.Ragg[base + (int64_t)jj * C];
            cr = hr ? lpd_combine(cr, uR(jj + 1), ag, uR(jj)) : ag;
            hr = true;
        }
    }
}

// ------------------------------------------------------------------ pass C

// NV = 1: forward (x -> y = out).  NV = 2: backward (x, g -> gx = out, ga).
template <int C, int NV>
__global__ void __launch_bounds__(kNT, (NV == 1 ? 3 : 2)) k_sym_sweep(SymScan a, const float* __restrict__ x, const float* __restrict__ g,
                                                   RangeState sx, RangeState sg, float* __restrict__ out,
                                                   float* __restrict__ ga, int ga_atomic) {
    using G = SymGeo<C>;
    constexpr int E = G::E, R = G::R;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SymSmem<C, NV>& sm = *reinterpret_cast<SymSmem<C, NV>*>(smem_raw);
    const int grp = blockIdx.y, j = blockIdx.x;
    const int64_t tb = (int64_t)j * a.tpr, te = min(a.T, tb + a.tpr);
    const int nt = (int)(te - tb);
    const int c = threadIdx.x % C, k = threadIdx.x / C, ch0 = grp * C;
    const int ch = ch0 + c;
    const bool cval = ch < a.B;
    const float* src[2] = {x, g};
    const RangeState* rs[2] = {&sx, &sg};

    stage_meta<G>(a.s, a.perm, a.n, tile_lo(tb, R), sm.s[0], sm.p[0]);
    cp_async_commit();
    if (nt > 1) stage_meta<G>(a.s, a.perm, a.n, tile_lo(tb + 1, R), sm.s[1], sm.p[1]);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int w = 0; w < NV; ++w) stage_rows<G>(src[w], a.B, ch0, a.n, tile_lo(tb, R), sm.p[0], sm.v[w][0]);
    cp_async_commit();

    // the left folds start from the carries entering the range
    double2 runL[NV], rin[NV];
    bool hasL = (j > 0);
    const bool hasRin = (j + 1 < a.P);
    const int64_t rng = ((int64_t)grp * a.P + j) * C + c;
#pragma unroll
    for (int w = 0; w < NV; ++w) {
        runL[w] = (hasL && threadIdx.x < C) ? rs[w]->Lin[rng] : make_double2(0.0, 0.0);
        rin[w] = (hasRin && threadIdx.x < C) ? rs[w]->Rin[rng] : make_double2(0.0, 0.0);
    }
    const float uRin = hasRin ? -__ldg(a.s + min(a.n - 1, te * (int64_t)R)) : 0.f;

    for (int i = 0; i < nt; ++i) {
        const int64_t t = tb + i, lo = tile_lo(t, R);
        cp_async_wait_all();
        __syncthreads();
        if (i + 1 < nt) {
#pragma unroll
            for (int w = 0; w < NV; ++w)
                stage_rows<G>(src[w], a.B, ch0, a.n, tile_lo(t + 1, R), sm.p[(i + 1) % 3], sm.v[w][(i + 1) & 1]);
        }
        cp_async_commit();
        if (i + 2 < nt) stage_meta<G>(a.s, a.perm, a.n, tile_lo(t + 2, R), sm.s[(i + 2) % 3], sm.p[(i + 2) % 3]);
        cp_async_commit();
        const float* sb = sm.s[i % 3];
        const uint32_t* pb = sm.p[i % 3];
        tile_decays<G>(sb, sm.dl);
        __syncthreads();
        const float ub_r = -sb[4 + k * E + E], ub_l = sb[4 + k * E - 1];
        LP exR[NV], exL[NV];
        bool hR[NV], hL[NV];
#pragma unroll
        for (int w = 0; w < NV; ++w) {
            const float* vb = sm.v[w][i & 1] + k * G::SEG + c;
            LP str = {0.f, 0.f}, stl = {0.f, 0.f};
#pragma unroll
            for (int e = E - 1; e >= 0; --e) str = lp_step_d(str, sm.dl[k * E + e + 1], 0.f, vb[e * C]);
#pragma unroll
            for (int e = 0; e < E; ++e) stl = lp_step_d(stl, sm.dl[k * E + e], 0.f, vb[e * C]);
            block_scan_dir<C, kNT, true>(str, -sb[4 + k * E], ub_r, sm.sc[2 * w], exR[w], hR[w]);
            block_scan_dir<C, kNT, false>(stl, sb[4 + k * E + E - 1], ub_l, sm.sc[2 * w + 1], exL[w], hL[w]);
        }
        // tile carries (threads < C), then fold the tile into the left state
        if (threadIdx.x < C) {
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                sm.carry[2 * w + 1][c] = runL[w];
                // right: the range carry (farther right) followed by the in-range suffix RS[t+1]
                double2 cr = rin[w];
                bool hr = hasRin;
                if (t + 1 < te) {
                    const double2 rsn = rs[w]->RS[((int64_t)grp * a.T + t + 1) * C + c];
                    cr = hr ? lpd_combine(rin[w], uRin, rsn, -sb[4 + R]) : rsn;
                    hr = true;
                }
                sm.carry[2 * w][c] = cr;
                if (c == 0) {
                    sm.has[2 * w] = hr;
                    sm.has[2 * w + 1] = hasL;
                }
                const LP tl = sm.sc[2 * w + 1].tot[c];
                const double2 tld = make_double2(tl.L, tl.P);
                runL[w] = hasL ? lpd_combine(runL[w], sb[3], tld, sb[4 + R - 1]) : tld;
            }
        }
        __syncthreads();
        hasL = true;
        // second pass: both directions from the true incoming states
        LP inR[NV], inL[NV];
#pragma unroll
        for (int w = 0; w < NV; ++w) {
            const double2 cr = sm.carry[2 * w][c], cl = sm.carry[2 * w + 1][c];
            inR[w] = seg_incoming(sm.has[2 * w], LP{(float)cr.x, (float)cr.y}, -sb[4 + R], hR[w], exR[w], ub_r);
            inL[w] = seg_incoming(sm.has[2 * w + 1], LP{(float)cl.x, (float)cl.y}, sb[3], hL[w], exL[w], ub_l);
        }
        if (NV == 1) {
            const float* vb = sm.v[0][i & 1] + k * G::SEG + c;
            float yv[E];
            LP s2 = inR[0];
#pragma unroll
            for (int e = E - 1; e >= 0; --e) {
                const float xe = vb[e * C];
                s2 = lp_step_d(s2, sm.dl[k * E + e + 1], 0.f, xe);
                yv[e] = s2.P - xe;
            }
            s2 = inL[0];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int r = k * E + e;
                s2 = lp_step_d(s2, sm.dl[r], 0.f, vb[e * C]);
                if (cval && lo + r < a.n) out[(int64_t)min(pb[r], (uint32_t)(a.n - 1)) * a.B + ch] = yv[e] + s2.P;
            }
        } else {
            const float* xv = sm.v[0][i & 1] + k * G::SEG + c;
            const float* gv = sm.v[NV - 1][i & 1] + k * G::SEG + c;
            float gxp[E], gap[E];
            LP ax = inR[0], ag = inR[NV - 1];
#pragma unroll
            for (int e = E - 1; e >= 0; --e) {
                const float xe = xv[e * C], ge = gv[e * C], dv = sm.dl[k * E + e + 1];
                ax = lp_step_d(ax, dv, 0.f, xe);
                ag = lp_step_d(ag, dv, 0.f, ge);
                gxp[e] = ag.P - ge;
                gap[e] = fmaf(ge, ax.L, xe * ag.L);  // strict right sums
            }
            ax = inL[0];
            ag = inL[NV - 1];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int r = k * E + e;
                const float xe = xv[e * C], ge = gv[e * C], dv = sm.dl[r];
                ax = lp_step_d(ax, dv, 0.f, xe);
                ag = lp_step_d(ag, dv, 0.f, ge);
                const bool valid = lo + r < a.n;
                const int64_t row = min(pb[r], (uint32_t)(a.n - 1));
                if (out != nullptr && cval && valid) out[row * a.B + ch] = gxp[e] + ag.P;
                float part = gap[e] - fmaf(ge, ax.L, xe * ag.L);  // minus strict left sums
#pragma unroll
                for (int off = C / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (ga != nullptr && c == 0 && valid) {
                    if (ga_atomic)
                        atomicAdd(ga + row, part);
                    else
                        ga[row] = part;
                }
            }
        }
    }
}

// ------------------------------------------------------------------ host side

struct SymPlan {
    int C, G, P;
    int64_t R, T, tpr;
    size_t rs_elems, rng_elems;  // double2 counts of one RS array / one range array
    size_t total;
};

SymPlan plan_sym(int64_t n, int64_t B, int sms) {
    SymPlan p;
    p.C = choose_channels(B);
    p.G = (int)((B + p.C - 1) / p.C);
    p.R = (int64_t)kNT / p.C * (p.C == 1 ? 8 : 16);
    p.T = (n + p.R - 1) / p.R;
    const int64_t want = std::max<int64_t>(1, ((int64_t)sms * kRangesPerSM + p.G - 1) / p.G);
    const int64_t P0 = std::min<int64_t>(std::min<int64_t>(p.T, want), kMaxRanges);
    p.tpr = (p.T + P0 - 1) / P0;
    p.P = (int)((p.T + p.tpr - 1) / p.tpr);
    p.rs_elems = (size_t)p.G * p.T * p.C;
    p.rng_elems = (size_t)p.G * kMaxRanges * p.C;
    // per vector: RS, Lin, Rin, Lagg, Ragg; two vectors (x, g)
    p.total = 2 * align_up(sizeof(double2) * (p.rs_elems + 4 * p.rng_elems), 256);
    return p;
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

template <class F>
cudaError_t set_smem(F* f, size_t bytes) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Pass A + pass B for one vector.
template <int C>
cudaError_t sym_ranges_t(const SymScan& a, const SymPlan& p, const float* v, RangeState st, cudaStream_t s) {
    const dim3 grid((unsigned)p.P, (unsigned)p.G);
    const size_t smA = sizeof(SymSmem<C, 1>);
    cudaError_t e = set_smem(k_sym_agg<C>, smA);
    if (e != cudaSuccess) return e;
    LAPLEX_TIMED("sym_agg", s, k_sym_agg<C><<<grid, kNT, smA, s>>>(a, v, st));
    LAPLEX_TIMED("sym_carry", s, k_sym_carry<C><<<p.G, kNT, 0, s>>>(a, st));
    return cudaGetLastError();
}

template <int C>
cudaError_t sym_forward_t(const SymScan& a, const SymPlan& p, const float* x, float* y, RangeState sx, cudaStream_t s) {
    cudaError_t e = sym_ranges_t<C>(a, p, x, sx, s);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)p.P, (unsigned)p.G);
    const size_t smC = sizeof(SymSmem<C, 1>);
    e = set_smem(k_sym_sweep<C, 1>, smC);
    if (e != cudaSuccess) return e;
    LAPLEX_TIMED("sym_fwd", s, k_sym_sweep<C, 1><<<grid, kNT, smC, s>>>(a, x, nullptr, sx, sx, y, nullptr, 0));
    return cudaGetLastError();
}

template <int C>
cudaError_t sym_backward_t(const SymScan& a, const SymPlan& p, const float* x, const float* g, float* gx, float* ga,
                           RangeState sx, bool have_x, RangeState sg, cudaStream_t s) {
    cudaError_t e;
    if (!have_x) {
        e = sym_ranges_t<C>(a, p, x, sx, s);
        if (e != cudaSuccess) return e;
    }
    e = sym_ranges_t<C>(a, p, g, sg, s);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)p.P, (unsigned)p.G);
    const size_t smC = sizeof(SymSmem<C, 2>);
    e = set_smem(k_sym_sweep<C, 2>, smC);
    if (e != cudaSuccess) return e;
    LAPLEX_TIMED("sym_bwd", s, k_sym_sweep<C, 2><<<grid, kNT, smC, s>>>(a, x, g, sx, sg, gx, ga, p.G > 1 ? 1 : 0));
    return cudaGetLastError();
}

SymScan scan_args(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, int64_t B) {
    SymScan a;
    a.s = s;
    a.perm = perm;
    a.n = n;
    a.B = (int)B;
    a.T = p.T;
    a.P = p.P;
    a.tpr = p.tpr;
    return a;
}

}  // namespace

size_t sym_workspace_bytes(int64_t n, int64_t B) { return plan_sym(n, B, 1).total; }

size_t sym_saved_bytes(int64_t n, int64_t B) {
    const SymPlan p = plan_sym(n, B, 1);
    return sizeof(double2) * (p.rs_elems + 2 * p.rng_elems);
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
    const SymPlan p = plan_sym(n, B, device_sms());
    const SymScan a = scan_args(p, s, perm, n, B);
    RangeState sx = carve(p, (double2*)ws, true);
    if (saved != nullptr) {  // RS and carries go to the caller's buffer; aggregates stay in ws
        const RangeState sv = carve(p, (double2*)saved, false);
        sx.RS = sv.RS;
        sx.Lin = sv.Lin;
        sx.Rin = sv.Rin;
    }
#define CALL(C) sym_forward_t<C>(a, p, x, y, sx, st)
    LAPLEX_SYM_DISPATCH(p.C, CALL)
#undef CALL
}

cudaError_t launch_sym_backward(const float* s, const uint32_t* perm, int64_t n, const float* x, const float* g,
                                int64_t B, const void* saved, float* gx, float* ga, void* ws, int32_t* status,
                                cudaStream_t st) {
    (void)status;
    const SymPlan p = plan_sym(n, B, device_sms());
    const SymScan a = scan_args(p, s, perm, n, B);
    const size_t half = align_up(sizeof(double2) * (p.rs_elems + 4 * p.rng_elems), 256);
    RangeState sx = carve(p, (double2*)ws, true);
    const RangeState sg = carve(p, (double2*)((char*)ws + half), true);
    if (saved != nullptr) {
        const RangeState sv = carve(p, (double2*)saved, false);
        sx.RS = sv.RS;
        sx.Lin = sv.Lin;
        sx.Rin = sv.Rin;
    }
    if (ga != nullptr && p.G > 1) {
        const cudaError_t e = cudaMemsetAsync(ga, 0, sizeof(float) * n, st);
        if (e != cudaSuccess) return e;
    }
#define CALL(C) sym_backward_t<C>(a, p, x, g, gx, ga, sx, saved != nullptr, sg, st)
    LAPLEX_SYM_DISPATCH(p.C, CALL)
#undef CALL
}

}  // namespace laplex
