// Rectangular LAPLEX operators: out = E(O, I) x with E_ij = exp(-|o_i - q_j|),
// optionally times cos(theta_O,i - theta_I,j), their backward, and the Gram apply
// ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary sections
// 2.1 and 2.2: "general case a != b", the phased operator, "Gram operators").
//
// O is the output anchor set, I the input anchor set, both sorted.  The product
// is one scan over the merged sorted sequence of O and I: the state just left
// of an output o is the prefix over the inputs q <= o, the state right of it the
// suffix over q > o, and out(o) = prefix + suffix.  It is evaluated in whichever
// of two ways keeps the lookback scan on the SMALLER side:
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
//   k_side_right / k_side_left  bounded decoupled-lookback scan over the small
//       side (inputs: gathered rows x phase weights, or fp64 interval sums),
//       writing per-row states (P, S) or parts (strict L, strict R, full).
//   k_large  one streaming pass over the large side: interval sums into fp64
//       bins (reduce), neighbour lookups (expand), and the fused anchor / phase
//       gradients of that side.
//   k_finish  per small-side row: combine the cos/sin parts into outputs and
//       gradients.
#include "laplex_internal.h"
#include "scan_tile.cuh"

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
    if (threadIdx.x < 32) {
        bool hc;
        const LP tot = threadIdx.x < C ? sm.tot[threadIdx.x] : LP{0.f, 0.f};
        lookback<C, true>(cs.chain(grp), t, a.T, a.s, a.m, R, tot, -s_sm[1], -s_sm[R + 1], status, hc);
    }
}

template <int C, bool BINS>
__global__ void __launch_bounds__(kSideNT) k_side_left(SideScan a, ChainSet left, ChainSet right, unsigned* counters,
                                                       int32_t* status) {
    constexpr int NT = kSideNT, E = kSideE, R = kTileValues / C;
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[BINS ? 1 : R];
    __shared__ float cw[(BINS || C == 1) ? 1 : R], sw[(BINS || C == 1) ? 1 : R];
    __shared__ ScanSmem<C, NT / 32> smL, smR;
    __shared__ double2 s_carry[C];
    __shared__ int64_t s_tile;
    __shared__ bool s_has;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    side_meta<R>(a, lo, s_sm, p_sm, cw, sw, BINS, !(BINS || C == 1));
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int cb = grp * C + c;
    float lin[E], tin[E], rin[E], tpin[E];
#pragma unroll
    for (int e = 0; e < E; ++e) side_inputs<BINS>(a, lo, k * E + e, cb, p_sm, cw, sw, lin[e], tin[e], rin[e], tpin[e]);
    const float ub_r = -s_sm[(k + 1) * E + 1];
    const float ub_l = s_sm[k * E];
    LP str = {0.f, 0.f}, stl = {0.f, 0.f};
    {
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
    if (threadIdx.x < 32) {
        bool hc;
        const LP tot = threadIdx.x < C ? smL.tot[threadIdx.x] : LP{0.f, 0.f};
        const double2 cin = lookback<C, false>(left.chain(grp), t, a.T, a.s, a.m, R, tot, s_sm[R], s_sm[0], status, hc);
        if (threadIdx.x < C) s_carry[threadIdx.x] = cin;
        if (threadIdx.x == 0) s_has = hc;
    }
    __syncthreads();
    const LP cl = {(float)s_carry[c].x, (float)s_carry[c].y};
    const LP left_in = seg_incoming(s_has, cl, s_sm[0], hl, exl, ub_l);
    LP cr = {0.f, 0.f};
    const bool hasr = (t + 1 < a.T);
    if (hasr) {
        const double2 v = __ldcg(&right.chain(grp).inc[(t + 1) * C + c]);
        cr = LP{(float)v.x, (float)v.y};
    }
    const LP right_in = seg_incoming(hasr, cr, -s_sm[R + 1], hr, exr, ub_r);
    float rres[E];  // values: S; bins: strict R
    LP st = right_in;
    float up = ub_r;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, rin[e], tpin[e]);
        rres[e] = BINS ? st.L : st.P;
        up = u;
    }
    st = left_in;
    up = ub_l;
    const bool cval = cb < a.Cb;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        const float u = s_sm[r + 1];
        st = lp_step(st, up, u, lin[e], tin[e]);
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
    const float* rows;  // [m][B] original order: accumulated (accum) and h (grad)
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

// Each group of `lpr` lanes walks a contiguous range of sorted large-side rows;
// lane gl of the group owns channels c0 .. c0+VEC-1 of every row.
template <int VEC, bool PHASED, int MODE>
__global__ void __launch_bounds__(256) k_large(LargePass A) {
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

    // interval sums of the current bin: fp32 for up to 16 rows, then folded into fp64
    int64_t cur = m;
    float fu[NP][VEC], fv[NP][VEC];
    double du[NP][VEC], dv[NP][VEC];
    int cnt = 0;
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int v = 0; v < VEC; ++v) fu[p][v] = fv[p][v] = 0.f, du[p][v] = dv[p][v] = 0.0;

    auto fold = [&]() {
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                du[p][v] += (double)fu[p][v];
                dv[p][v] += (double)fv[p][v];
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
                    if (bin < ms) {
                        double* dst = A.U + bin * Cb + ch;
                        if (owner)
                            *dst = du[p][v];
                        else if (du[p][v] != 0.0)
                            atomicAdd(dst, du[p][v]);
                    }
                    if (bin >= 1) {
                        double* dst = A.V + (bin - 1) * Cb + ch;
                        if (owner)
                            *dst = dv[p][v];
                        else if (dv[p][v] != 0.0)
                            atomicAdd(dst, dv[p][v]);
                    }
                    du[p][v] = dv[p][v] = 0.0;
                }
        }
    };

    int64_t st_m = -1, st_mp = -1;
    float Pm1[NP][VEC], Pmp[NP][VEC], Smp[NP][VEC];

    for (int64_t r = r0; r < r1; ++r) {
        const float q = __ldg(A.s + r);
        const uint32_t pr = min(__ldg(A.perm + r), (uint32_t)(A.m - 1));
        float w[NP], wd[NP];
        if (PHASED) {
            float sn, cs;
            sincosf(__ldg(A.theta + pr), &sn, &cs);
            w[0] = cs;
            w[NP - 1] = sn;
            wd[0] = -sn;
            wd[NP - 1] = cs;
        } else {
            w[0] = 1.f;
            wd[0] = 0.f;
        }
        while (m < ms && __ldg(A.sp + m) < q) ++m;
        if (mp < m) mp = m;
        while (mp < ms && __ldg(A.sp + mp) <= q) ++mp;
        const bool tie = mp > m;
        const float eL = (m > 0) ? expf(__ldg(A.sp + m - 1) - q) : 0.f;
        const float eR = (mp < ms) ? expf(q - __ldg(A.sp + mp)) : 0.f;
        const float eLf = tie ? 1.f : eL;
        float h[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) h[v] = 0.f;
        if (ROWS && cval) load_vec<VEC>(A.rows + (int64_t)pr * B + c0, h);
        if (ACCUM) {
            if (m != cur) {
                flush(cur);
                cur = m;
            }
#pragma unroll
            for (int p = 0; p < NP; ++p)
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const float val = w[p] * h[v];
                    // A row tied with a run of small-side anchors enters that run only
                    // (TL, TR); the neighbours beyond it receive it through the scan.
                    if (!tie) {
                        fu[p][v] = fmaf(eR, val, fu[p][v]);
                        fv[p][v] = fmaf(eL, val, fv[p][v]);
                    } else if (cval) {
                        atomicAdd(A.TL + m * Cb + p * B + c0 + v, (double)val);
                        atomicAdd(A.TR + (mp - 1) * Cb + p * B + c0 + v, (double)val);
                    }
                }
            if (++cnt == 16) fold();
        }
        if (STATES) {
            if (m != st_m || mp != st_mp) {
#pragma unroll
                for (int p = 0; p < NP; ++p)
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        const int ch = p * B + c0 + v;
                        Pm1[p][v] = (GRAD && cval && m > 0) ? __ldg(A.Pst + (m - 1) * Cb + ch) : 0.f;
                        Pmp[p][v] = (cval && mp > 0) ? __ldg(A.Pst + (mp - 1) * Cb + ch) : 0.f;
                        Smp[p][v] = (cval && mp < ms) ? __ldg(A.Sst + mp * Cb + ch) : 0.f;
                    }
                st_m = m;
                st_mp = mp;
            }
            float o[VEC];
            float ga = 0.f, gp = 0.f;
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                o[v] = 0.f;
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    const float full = fmaf(eLf, Pmp[p][v], eR * Smp[p][v]);
                    o[v] = fmaf(w[p], full, o[v]);
                    if (GRAD) {
                        const float diff = fmaf(eR, Smp[p][v], -eL * Pm1[p][v]);  // strict right - strict left
                        ga = fmaf(h[v] * w[p], diff, ga);
                        if (PHASED) gp = fmaf(h[v] * wd[p], full, gp);
                    }
                }
            }
            if (EXPAND && A.out != nullptr && cval) store_vec<VEC>(A.out + (int64_t)pr * B + c0, o);
            if (GRAD) {
                for (int off = lpr >> 1; off >= 1; off >>= 1) {
                    ga += __shfl_xor_sync(gmask, ga, off);
                    if (PHASED) gp += __shfl_xor_sync(gmask, gp, off);
                }
                if (gl == 0) {
                    if (A.g_anchor != nullptr) {
                        if (A.chunk_atomic)
                            atomicAdd(A.g_anchor + pr, ga);
                        else
                            A.g_anchor[pr] = ga;
                    }
                    if (PHASED && A.g_phase != nullptr) {
                        if (A.chunk_atomic)
                            atomicAdd(A.g_phase + pr, gp);
                        else
                            A.g_phase[pr] = gp;
                    }
                }
            }
        }
    }
    if (ACCUM) flush(cur);
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
    const float* h;  // [m][B] original order (for gradients)
    float* out;      // [m][B] original order: sum_p w_p ZF
    float* g_anchor;  // sum_c h sum_p w_p (ZR - ZL)
    float* g_phase;   // sum_c h sum_p w'_p ZF
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
        const float hv = F.h ? __ldg(F.h + (int64_t)pr * F.B + c) : 0.f;
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
        if (F.g_anchor) F.g_anchor[pr] = ga;
        if (PHASED && F.g_phase) F.g_phase[pr] = gp;
    }
}

__global__ void k_scale_rows(const float* __restrict__ D, const float* __restrict__ w, float* __restrict__ out,
                             int64_t k, int B) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < k * B) out[i] = __ldg(D + i / B) * __ldg(w + i);
}

__global__ void k_row_dot(const float* __restrict__ a, const float* __restrict__ b, float* __restrict__ out, int64_t k,
                          int B) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= k) return;
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    for (int c = lane; c < B; c += 32) acc = fmaf(__ldg(a + r * B + c), __ldg(b + r * B + c), acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) out[r] = acc;
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
    LAPLEX_TIMED("side_right", st, k_side_right<C, BINS><<<grid, kSideNT, 0, st>>>(a, cr, p.counters, status));
    LAPLEX_TIMED("side_left", st, k_side_left<C, BINS><<<grid, kSideNT, 0, st>>>(a, cl, cr, p.counters + p.G, status));
    return cudaGetLastError();
}

cudaError_t side_scan(const RectPlan& p, SideScan a, bool bins, int32_t* status, cudaStream_t st) {
    a.T = p.T;
    a.Cb = p.Cb;
    cudaError_t e = cudaMemsetAsync(p.counters, 0, p.memset_bytes, st);
    if (e != cudaSuccess) return e;
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

template <int VEC, bool PHASED>
cudaError_t large_mode(LargePass A, int mode, dim3 grid, cudaStream_t st) {
    switch (mode) {
        case kLmExpand: LAPLEX_TIMED("large_expand", st, k_large<VEC, PHASED, kLmExpand><<<grid, 256, 0, st>>>(A)); break;
        case kLmAccum: LAPLEX_TIMED("large_accum", st, k_large<VEC, PHASED, kLmAccum><<<grid, 256, 0, st>>>(A)); break;
        case kLmGrad: LAPLEX_TIMED("large_grad", st, k_large<VEC, PHASED, kLmGrad><<<grid, 256, 0, st>>>(A)); break;
        case kLmExpand | kLmGrad: LAPLEX_TIMED("large_expand_grad", st, k_large<VEC, PHASED, kLmExpand | kLmGrad><<<grid, 256, 0, st>>>(A)); break;
        case kLmAccum | kLmGrad: LAPLEX_TIMED("large_accum_grad", st, k_large<VEC, PHASED, kLmAccum | kLmGrad><<<grid, 256, 0, st>>>(A)); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t large_pass(LargePass A, int mode, cudaStream_t st) {
    const bool phased = A.theta != nullptr;
    const int vec = (A.B % 4 == 0) ? 4 : 1;
    int lpr = 1;
    while (lpr < 32 && lpr * vec < A.B) lpr <<= 1;
    const int chunks = (A.B + lpr * vec - 1) / (lpr * vec);
    A.lpr = lpr;
    A.chunk_atomic = chunks > 1 ? 1 : 0;
    const int64_t groups_per_block = 8 * (32 / lpr);
    // enough groups to fill the GPU, each walking a contiguous run of rows
    const int64_t min_rows = 64;
    int64_t blocks = std::min<int64_t>((int64_t)sm_count() * 4, (A.m + groups_per_block * min_rows - 1) /
                                                                     (groups_per_block * min_rows));
    blocks = std::max<int64_t>(blocks, 1);
    A.rows_per_group = (A.m + blocks * groups_per_block - 1) / (blocks * groups_per_block);
    if ((mode & kLmGrad) && A.chunk_atomic) {
        if (A.g_anchor) cudaMemsetAsync(A.g_anchor, 0, sizeof(float) * A.m, st);
        if (A.g_phase) cudaMemsetAsync(A.g_phase, 0, sizeof(float) * A.m, st);
    }
    const dim3 grid((unsigned)blocks, (unsigned)chunks);
    if (vec == 4) return phased ? large_mode<4, true>(A, mode, grid, st) : large_mode<4, false>(A, mode, grid, st);
    return phased ? large_mode<1, true>(A, mode, grid, st) : large_mode<1, false>(A, mode, grid, st);
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
    a.perm = S.perm;
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
    A.Cb = p.Cb;
    const int64_t sz = p.ms * (int64_t)p.Cb;
    A.U = p.bins;
    A.TL = p.bins + sz;
    A.V = p.bins + 2 * sz;
    A.TR = p.bins + 3 * sz;
    return A;
}

#define LAPLEX_TRY(expr)                     \
    do {                                     \
        cudaError_t e_ = (expr);             \
        if (e_ != cudaSuccess) return e_;    \
    } while (0)

// Reduce path of the forward: interval sums of x (at I) into O's bins, scan over
// O, parts written to ZL/ZR/ZF.
cudaError_t reduce_parts(const RectPlan& p, Side O, Side I, const float* x, int64_t B, float* ZL, float* ZR, float* ZF,
                         int32_t* status, cudaStream_t st) {
    LAPLEX_TRY(cudaMemsetAsync(p.bins, 0, sizeof(double) * 4 * p.ms * p.Cb, st));
    LargePass A = large_args(I, O, p, B);
    A.rows = x;
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
                                 cudaStream_t st) {
    const bool phased = O.theta != nullptr;
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
                F.g_anchor = gO;
                F.g_phase = gtO;
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
        A.Pst = Pst;
        A.Sst = Pst ? Pst + sz : nullptr;
        A.g_anchor = gO;
        A.g_phase = gtO;
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
        F.out = gx;
        F.g_anchor = gI;
        F.g_phase = gtI;
        LAPLEX_TRY(finish(F, st));
    }
    return cudaSuccess;
}

size_t gram_workspace_bytes(int64_t n, int64_t k, int64_t B) {
    return plan_rect(n, k, B, false, nullptr, k).total;
}

cudaError_t launch_gram(Side A, Side Bs, const float* D, const float* v, int64_t B, float* y, float* w_saved,
                        const float* g, float* gD, void* ws, int32_t* status, cudaStream_t st) {
    const RectPlan p = plan_rect(A.m, Bs.m, B, false, ws, Bs.m);
    const int64_t kb = Bs.m * B;
    float* w = w_saved ? w_saved : p.rows3;
    float* w2 = p.rows3 + kb;
    float* wg = p.rows3 + 2 * kb;
    LAPLEX_TRY(launch_rect_forward(Bs, A, v, B, w, nullptr, ws, status, st));  // w = A^T v
    LAPLEX_TIMED("scale_rows", st, k_scale_rows<<<(unsigned)((kb + 255) / 256), 256, 0, st>>>(D, w, w2, Bs.m, (int)B));
    LAPLEX_TRY(cudaGetLastError());
    LAPLEX_TRY(launch_rect_forward(A, Bs, w2, B, y, nullptr, ws, status, st));  // y = A (D w)
    if (g != nullptr && gD != nullptr) {
        LAPLEX_TRY(launch_rect_forward(Bs, A, g, B, wg, nullptr, ws, status, st));  // A^T g
        LAPLEX_TIMED("row_dot", st, k_row_dot<<<(unsigned)((Bs.m + 7) / 8), 256, 0, st>>>(wg, w, gD, Bs.m, (int)B));
        LAPLEX_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace laplex
