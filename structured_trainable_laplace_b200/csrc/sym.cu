// Symmetric LAPLEX operator y = K x, K_ij = exp(-|a_i - a_j|), and its backward
// ("LAPLEX: The FFT of Learnable Laplace Kernels", technical summary section 2.2,
// "symmetric case": after sorting, the lower triangle is the prefix scan
// P_r = x_r + exp(a_(r-1) - a_(r)) P_(r-1), the upper triangle the mirrored suffix
// scan S_r, and y = P + S - x because both contain the diagonal).
//
// Rows are the sorted anchors; a tile is R = 4096 / C rows by C channels (one
// channel group).  Three kernels:
//   k_sym_right  walks tiles from the right end with a bounded decoupled
//                lookback and publishes, per tile, the fp64 suffix state of
//                everything from the tile's first row to the end.
//   k_sym_left   walks tiles from the left end: lookback for the prefix state,
//                reads the suffix carry of the next tile, and in the same sweep
//                evaluates both directions inside the tile and writes
//                y = P + S - x through the permutation.
//   k_sym_bwd    the backward in one sweep: gx = K g = P_g + S_g - g and
//                ga = sum_c g (R_x - L_x) + x (R_g - L_g) from the strict sums
//                (ties excluded: sign(0) = 0), with the x carries from the
//                forward and the g prefix by lookback.
// k_sym_left runs its tiles left to right right after k_sym_right finished at
// the left end, so the first tiles it gathers are still in L2.
#include "laplex_internal.h"
#include "scan_tile.cuh"

namespace laplex {

namespace {

constexpr int kTileValues = 4096;  // rows x channels per tile

template <int C, int NT, int E>
__global__ void __launch_bounds__(NT) k_sym_right(const float* __restrict__ s, const uint32_t* __restrict__ perm,
                                                  int64_t n, const float* __restrict__ x, int B, int64_t T,
                                                  ChainSet cs, unsigned* counters, int32_t* status) {
    constexpr int K = NT / C;
    constexpr int R = K * E;
    static_assert(R * C == kTileValues, "tile geometry");
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[R];
    __shared__ ScanSmem<C, NT / 32> sm;
    __shared__ int64_t s_tile;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = T - 1 - (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    load_tile_meta<R>(s, perm, n, lo, s_sm, p_sm);
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int ch = grp * C + c;
    const bool cval = ch < B;
    float xv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        xv[e] = (cval && lo + r < n) ? __ldg(x + (int64_t)p_sm[r] * B + ch) : 0.f;
    }
    LP st = {0.f, 0.f};
    float up = -s_sm[(k + 1) * E + 1];
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, 0.f, xv[e]);
        up = u;
    }
    LP excl;
    bool has;
    block_scan_dir<C, NT, true>(st, -s_sm[k * E + 1], -s_sm[(k + 1) * E + 1], sm, excl, has);
    if (threadIdx.x < 32) {
        bool hc;
        const LP tot = threadIdx.x < C ? sm.tot[threadIdx.x] : LP{0.f, 0.f};
        lookback<C, true>(cs.chain(grp), t, T, s, n, R, tot, -s_sm[1], -s_sm[R + 1], status, hc);
    }
}

template <int C, int NT, int E, bool WRITE_Y>
__global__ void __launch_bounds__(NT) k_sym_left(const float* __restrict__ s, const uint32_t* __restrict__ perm,
                                                 int64_t n, const float* __restrict__ x, int B, int64_t T,
                                                 ChainSet left, ChainSet right, unsigned* counters,
                                                 float* __restrict__ y, int32_t* status) {
    constexpr int K = NT / C;
    constexpr int R = K * E;
    static_assert(R * C == kTileValues, "tile geometry");
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[R];
    __shared__ ScanSmem<C, NT / 32> smL, smR;
    __shared__ double2 s_carry[C];
    __shared__ int64_t s_tile;
    __shared__ bool s_has;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    load_tile_meta<R>(s, perm, n, lo, s_sm, p_sm);
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int ch = grp * C + c;
    const bool cval = ch < B;
    float xv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        xv[e] = (cval && lo + r < n) ? __ldg(x + (int64_t)p_sm[r] * B + ch) : 0.f;
    }
    const float ub_r = -s_sm[(k + 1) * E + 1];  // right direction: anchor before the segment
    const float ub_l = s_sm[k * E];             // left direction: anchor before the segment
    LP str = {0.f, 0.f}, stl = {0.f, 0.f};
    {
        float up = ub_r;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) {
            const float u = -s_sm[k * E + e + 1];
            str = lp_step(str, up, u, 0.f, xv[e]);
            up = u;
        }
        up = ub_l;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float u = s_sm[k * E + e + 1];
            stl = lp_step(stl, up, u, 0.f, xv[e]);
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
        const double2 cin = lookback<C, false>(left.chain(grp), t, T, s, n, R, tot, s_sm[R], s_sm[0], status, hc);
        if (threadIdx.x < C) s_carry[threadIdx.x] = cin;
        if (threadIdx.x == 0) s_has = hc;
    }
    __syncthreads();
    if (!WRITE_Y) return;
    LP cl = {(float)s_carry[c].x, (float)s_carry[c].y};
    const LP left_in = seg_incoming(s_has, cl, s_sm[0], hl, exl, ub_l);
    LP cr = {0.f, 0.f};
    const bool hasr = (t + 1 < T);
    if (hasr) {
        const double2 v = __ldcg(&right.chain(grp).inc[(t + 1) * C + c]);
        cr = LP{(float)v.x, (float)v.y};
    }
    const LP right_in = seg_incoming(hasr, cr, -s_sm[R + 1], hr, exr, ub_r);
    float yv[E];
    LP st = right_in;
    float up = ub_r;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const float u = -s_sm[k * E + e + 1];
        st = lp_step(st, up, u, 0.f, xv[e]);
        yv[e] = st.P - xv[e];
        up = u;
    }
    st = left_in;
    up = ub_l;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float u = s_sm[k * E + e + 1];
        st = lp_step(st, up, u, 0.f, xv[e]);
        yv[e] += st.P;
        up = u;
    }
    if (cval) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int r = k * E + e;
            if (lo + r < n) y[(int64_t)p_sm[r] * B + ch] = yv[e];
        }
    }
}

template <int C, int NT, int E>
__global__ void __launch_bounds__(NT) k_sym_bwd(const float* __restrict__ s, const uint32_t* __restrict__ perm,
                                                int64_t n, const float* __restrict__ x, const float* __restrict__ g,
                                                int B, int64_t T, ChainSet xl, ChainSet xr, ChainSet gl, ChainSet gr,
                                                unsigned* counters, float* __restrict__ gx, float* __restrict__ ga,
                                                int ga_atomic, int32_t* status) {
    constexpr int K = NT / C;
    constexpr int R = K * E;
    static_assert(R * C == kTileValues, "tile geometry");
    __shared__ float s_sm[R + 2];
    __shared__ uint32_t p_sm[R];
    __shared__ ScanSmem<C, NT / 32> sm_xr, sm_gr, sm_xl, sm_gl;
    __shared__ double2 s_carry[C];
    __shared__ int64_t s_tile;
    __shared__ bool s_has;
    const int grp = blockIdx.y;
    if (threadIdx.x == 0) s_tile = (int64_t)atomicAdd(&counters[grp], 1u);
    __syncthreads();
    const int64_t t = s_tile, lo = t * R;
    load_tile_meta<R>(s, perm, n, lo, s_sm, p_sm);
    __syncthreads();
    const int c = threadIdx.x % C, k = threadIdx.x / C;
    const int ch = grp * C + c;
    const bool cval = ch < B;
    float xv[E], gv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        const bool ok = cval && lo + r < n;
        const int64_t off = (int64_t)p_sm[r] * B + ch;
        xv[e] = ok ? __ldg(x + off) : 0.f;
        gv[e] = ok ? __ldg(g + off) : 0.f;
    }
    const float ub_r = -s_sm[(k + 1) * E + 1];
    const float ub_l = s_sm[k * E];
    LP axr = {0.f, 0.f}, agr = {0.f, 0.f}, axl = {0.f, 0.f}, agl = {0.f, 0.f};
    {
        float up = ub_r;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) {
            const float u = -s_sm[k * E + e + 1];
            axr = lp_step(axr, up, u, 0.f, xv[e]);
            agr = lp_step(agr, up, u, 0.f, gv[e]);
            up = u;
        }
        up = ub_l;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float u = s_sm[k * E + e + 1];
            axl = lp_step(axl, up, u, 0.f, xv[e]);
            agl = lp_step(agl, up, u, 0.f, gv[e]);
            up = u;
        }
    }
    LP exr, egr, exl, egl;
    bool hxr, hgr, hxl, hgl;
    block_scan_dir<C, NT, true>(axr, -s_sm[k * E + 1], ub_r, sm_xr, exr, hxr);
    block_scan_dir<C, NT, true>(agr, -s_sm[k * E + 1], ub_r, sm_gr, egr, hgr);
    block_scan_dir<C, NT, false>(axl, s_sm[k * E + E], ub_l, sm_xl, exl, hxl);
    block_scan_dir<C, NT, false>(agl, s_sm[k * E + E], ub_l, sm_gl, egl, hgl);
    if (threadIdx.x < 32) {
        bool hc;
        const LP tot = threadIdx.x < C ? sm_gl.tot[threadIdx.x] : LP{0.f, 0.f};
        const double2 cin = lookback<C, false>(gl.chain(grp), t, T, s, n, R, tot, s_sm[R], s_sm[0], status, hc);
        if (threadIdx.x < C) s_carry[threadIdx.x] = cin;
        if (threadIdx.x == 0) s_has = hc;
    }
    __syncthreads();
    const bool hasl = (t > 0), hasr = (t + 1 < T);
    LP cxl = {0.f, 0.f}, cxr = {0.f, 0.f}, cgr = {0.f, 0.f};
    if (hasl) {
        const double2 v = __ldcg(&xl.chain(grp).inc[(t - 1) * C + c]);
        cxl = LP{(float)v.x, (float)v.y};
    }
    if (hasr) {
        const double2 v = __ldcg(&xr.chain(grp).inc[(t + 1) * C + c]);
        const double2 w = __ldcg(&gr.chain(grp).inc[(t + 1) * C + c]);
        cxr = LP{(float)v.x, (float)v.y};
        cgr = LP{(float)w.x, (float)w.y};
    }
    const LP cgl = {(float)s_carry[c].x, (float)s_carry[c].y};
    const float ut_l = s_sm[0], ut_r = -s_sm[R + 1];
    LP ax = seg_incoming(hasr, cxr, ut_r, hxr, exr, ub_r);
    LP ag = seg_incoming(hasr, cgr, ut_r, hgr, egr, ub_r);
    float gxp[E], gap[E];
    float up = ub_r;
#pragma unroll
    for (int e = E - 1; e >= 0; --e) {
        const float u = -s_sm[k * E + e + 1];
        ax = lp_step(ax, up, u, 0.f, xv[e]);
        ag = lp_step(ag, up, u, 0.f, gv[e]);
        gxp[e] = ag.P - gv[e];
        gap[e] = fmaf(gv[e], ax.L, xv[e] * ag.L);  // strict right sums
        up = u;
    }
    ax = seg_incoming(hasl, cxl, ut_l, hxl, exl, ub_l);
    ag = seg_incoming(s_has, cgl, ut_l, hgl, egl, ub_l);
    up = ub_l;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int r = k * E + e;
        const float u = s_sm[r + 1];
        ax = lp_step(ax, up, u, 0.f, xv[e]);
        ag = lp_step(ag, up, u, 0.f, gv[e]);
        up = u;
        const bool valid = lo + r < n;
        const int64_t row = p_sm[r];
        if (gx != nullptr && cval && valid) gx[row * B + ch] = gxp[e] + ag.P;
        float part = gap[e] - fmaf(gv[e], ax.L, xv[e] * ag.L);  // minus strict left sums
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

struct SymPlan {
    int C, G;
    int64_t R, T;
    // workspace pieces
    unsigned* counters;  // [4][G]
    int* flags;          // [4][G][T]
    double2* agg;        // [4][G][T][C]
    double2* inc;        // [4][G][T][C]
    size_t memset_bytes;
    size_t total;
};

SymPlan plan_sym(int64_t n, int64_t B, void* ws) {
    SymPlan p;
    p.C = choose_channels(B);
    p.G = (int)((B + p.C - 1) / p.C);
    p.R = kTileValues / p.C;
    p.T = (n + p.R - 1) / p.R;
    char* base = (char*)ws;
    size_t off = 0;
    p.counters = (unsigned*)(base + off);
    off += align_up(sizeof(unsigned) * 4 * p.G, 256);
    p.flags = (int*)(base + off);
    off += align_up(sizeof(int) * 4 * p.G * p.T, 256);
    p.memset_bytes = off;
    p.agg = (double2*)(base + off);
    off += align_up(sizeof(double2) * 4 * p.G * p.T * p.C, 256);
    p.inc = (double2*)(base + off);
    off += align_up(sizeof(double2) * 4 * p.G * p.T * p.C, 256);
    p.total = off;
    return p;
}

// chain ids: 0 x-right, 1 x-left, 2 g-right, 3 g-left
ChainSet chain_set(const SymPlan& p, int id, double2* inc_override) {
    ChainSet cs;
    cs.flags = p.flags + (int64_t)id * p.G * p.T;
    cs.agg = p.agg + (int64_t)id * p.G * p.T * p.C;
    cs.inc = inc_override ? inc_override : p.inc + (int64_t)id * p.G * p.T * p.C;
    cs.T = p.T;
    cs.C = p.C;
    return cs;
}

template <int C>
cudaError_t sym_forward_t(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, const float* x, int B,
                          float* y, double2* saved_l, double2* saved_r, int32_t* status, cudaStream_t st,
                          bool write_y, int chain_r, int chain_l) {
    const dim3 grid((unsigned)p.T, (unsigned)p.G);
    ChainSet cr = chain_set(p, chain_r, saved_r), cl = chain_set(p, chain_l, saved_l);
    LAPLEX_TIMED("sym_right", st, k_sym_right<C, 256, kTileValues / 256><<<grid, 256, 0, st>>>(s, perm, n, x, B, p.T, cr, p.counters + chain_r * p.G,
                                                                 status));
    if (write_y)
        LAPLEX_TIMED("sym_left", st, k_sym_left<C, 256, kTileValues / 256, true><<<grid, 256, 0, st>>>(s, perm, n, x, B, p.T, cl, cr,
                                                                          p.counters + chain_l * p.G, y, status));
    else
        LAPLEX_TIMED("sym_left_carry", st, k_sym_left<C, 256, kTileValues / 256, false><<<grid, 256, 0, st>>>(s, perm, n, x, B, p.T, cl, cr,
                                                                           p.counters + chain_l * p.G, y, status));
    return cudaGetLastError();
}

template <int C>
cudaError_t sym_backward_t(const SymPlan& p, const float* s, const uint32_t* perm, int64_t n, const float* x,
                           const float* g, int B, double2* saved_l, double2* saved_r, float* gx, float* ga,
                           int32_t* status, cudaStream_t st) {
    const dim3 grid((unsigned)p.T, (unsigned)p.G);
    cudaError_t e;
    if (saved_l == nullptr) {
        // no saved forward state: recompute the x carries (chains 0, 1)
        e = sym_forward_t<C>(p, s, perm, n, x, B, nullptr, nullptr, nullptr, status, st, false, 0, 1);
        if (e != cudaSuccess) return e;
    }
    ChainSet cxr = chain_set(p, 0, saved_r), cxl = chain_set(p, 1, saved_l);
    ChainSet cgr = chain_set(p, 2, nullptr), cgl = chain_set(p, 3, nullptr);
    LAPLEX_TIMED("sym_right", st, k_sym_right<C, 256, kTileValues / 256><<<grid, 256, 0, st>>>(s, perm, n, g, B, p.T, cgr, p.counters + 2 * p.G,
                                                                 status));
    LAPLEX_TIMED("sym_bwd", st, k_sym_bwd<C, 512, kTileValues / 512><<<grid, 512, 0, st>>>(s, perm, n, x, g, B, p.T, cxl, cxr, cgl, cgr,
                                                               p.counters + 3 * p.G, gx, ga, p.G > 1 ? 1 : 0,
                                                               status));
    return cudaGetLastError();
}

}  // namespace

size_t sym_workspace_bytes(int64_t n, int64_t B) { return plan_sym(n, B, nullptr).total; }

size_t sym_saved_bytes(int64_t n, int64_t B) {
    const SymPlan p = plan_sym(n, B, nullptr);
    return 2 * sizeof(double2) * (size_t)p.G * p.T * p.C;
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
    const SymPlan p = plan_sym(n, B, ws);
    cudaError_t e = cudaMemsetAsync(ws, 0, p.memset_bytes, st);
    if (e != cudaSuccess) return e;
    double2* sl = saved ? (double2*)saved : nullptr;
    double2* sr = saved ? (double2*)saved + (int64_t)p.G * p.T * p.C : nullptr;
#define CALL(C) sym_forward_t<C>(p, s, perm, n, x, (int)B, y, sl, sr, status, st, true, 0, 1)
    LAPLEX_SYM_DISPATCH(p.C, CALL)
#undef CALL
}

cudaError_t launch_sym_backward(const float* s, const uint32_t* perm, int64_t n, const float* x, const float* g,
                                int64_t B, const void* saved, float* gx, float* ga, void* ws, int32_t* status,
                                cudaStream_t st) {
    const SymPlan p = plan_sym(n, B, ws);
    cudaError_t e = cudaMemsetAsync(ws, 0, p.memset_bytes, st);
    if (e != cudaSuccess) return e;
    if (ga != nullptr && p.G > 1) {
        e = cudaMemsetAsync(ga, 0, sizeof(float) * n, st);
        if (e != cudaSuccess) return e;
    }
    double2* sl = saved ? (double2*)saved : nullptr;
    double2* sr = saved ? (double2*)saved + (int64_t)p.G * p.T * p.C : nullptr;
#define CALL(C) sym_backward_t<C>(p, s, perm, n, x, g, (int)B, sl, sr, gx, ga, status, st)
    LAPLEX_SYM_DISPATCH(p.C, CALL)
#undef CALL
}

}  // namespace laplex
