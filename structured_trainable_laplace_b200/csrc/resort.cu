// Warm-start re-sort: the anchors were sorted before (perm_prev) and have moved a
// little since, as they do between two training steps ("LAPLEX: The FFT of
// Learnable Laplace Kernels", technical summary section 2.2: the scan algebra
// starts from the sorted anchors, and the anchors are trainable parameters).
//
// The result is the same unique stable order as the full sort: ascending by the
// composite c = (key(a), index).  Gather the moved anchors through perm_prev:
// c_r = (key(a[perm_prev[r]]), perm_prev[r]).  An element with c_r above every
// composite before it and below every composite after it is at its final rank
// already (exactly r composites are smaller): it is KEPT.  Every other element is
// DISPLACED; sorting the displaced ones among themselves and writing them, in
// order, into the displaced positions completes the sorted order.  So:
//
//   1. gather: keys of the moved anchors in the old order, each tile's max and min;
//   2. tile carries: exclusive prefix max / suffix min over the tiles (one CTA);
//   3. classify: kept elements are written out; displaced positions go to a
//      position bitmap, their indices to an index bitmap;
//   4. count: set bits of the index bitmap per tile;
//   5. offsets (one CTA): scans of both counts; decide the path on the device;
//   6. compact: displaced positions in position order, displaced (anchor, index)
//      in index order;
//   7. the full radix sort on the displaced anchors (stable, so equal keys keep
//      ascending index), then place them;
//   8. the full radix sort of all anchors instead when too many are displaced or
//      perm_prev is not a permutation (the two bitmap counts differ).
// The path is decided on the device; the sorts run with device-side counts, so
// the call never synchronises.
#include "laplex_internal.h"

namespace laplex {

namespace {

constexpr int kNT = 256;
constexpr int kItems = 16;
constexpr int kTile = kNT * kItems;   // 4096 positions per tile
constexpr int kWords = kTile / 32;    // bitmap words per tile
constexpr int kScanNT = 1024;         // the one-CTA scans
// above this share of displaced anchors the full sort runs instead
constexpr int64_t kMaxDisplacedDen = 2;

__device__ __forceinline__ uint64_t comp(uint32_t key, uint32_t idx) { return ((uint64_t)key << 32) | idx; }

__device__ __forceinline__ uint64_t shfl_up_u64(uint64_t v, int d) {
    const uint32_t lo = __shfl_up_sync(0xffffffffu, (uint32_t)v, d);
    const uint32_t hi = __shfl_up_sync(0xffffffffu, (uint32_t)(v >> 32), d);
    return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_down_u64(uint64_t v, int d) {
    const uint32_t lo = __shfl_down_sync(0xffffffffu, (uint32_t)v, d);
    const uint32_t hi = __shfl_down_sync(0xffffffffu, (uint32_t)(v >> 32), d);
    return ((uint64_t)hi << 32) | lo;
}

// Exclusive max over the threads before this one and exclusive min over the
// threads after it, for a block of NT threads (identities 0 and ~0).
template <int NT>
__device__ __forceinline__ void block_excl_max_min(uint64_t vmax, uint64_t vmin, uint64_t* s_max, uint64_t* s_min,
                                                   uint64_t& before_max, uint64_t& after_min) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint64_t inc_max = vmax, inc_min = vmin;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint64_t o = shfl_up_u64(inc_max, d);
        if (lane >= d) inc_max = max(inc_max, o);
        const uint64_t u = shfl_down_u64(inc_min, d);
        if (lane + d < 32) inc_min = min(inc_min, u);
    }
    if (lane == 31) s_max[w] = inc_max;
    if (lane == 0) s_min[w] = inc_min;
    __syncthreads();
    uint64_t bm = 0, am = ~0ull;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
        if (j < w) bm = max(bm, s_max[j]);
        if (j > w) am = min(am, s_min[j]);
    }
    __syncthreads();
    const uint64_t pm = shfl_up_u64(inc_max, 1), nm = shfl_down_u64(inc_min, 1);
    before_max = lane > 0 ? max(bm, pm) : bm;
    after_min = lane < 31 ? min(am, nm) : am;
}

// Exclusive sum of one value per thread over an NT-thread block; *total gets the sum.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_sum(uint32_t v, uint32_t* s_w, uint32_t* total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += o;
    }
    if (lane == 31) s_w[w] = inc;
    __syncthreads();
    uint32_t base = 0, tot = 0;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
        const uint32_t x = s_w[j];
        if (j < w) base += x;
        tot += x;
    }
    __syncthreads();
    *total = tot;
    return base + inc - v;
}

struct ResortWs {
    uint32_t* keys;       // [n] keys of the moved anchors in the old order
    uint32_t* pos_bits;   // [T * kWords] displaced positions
    uint32_t* idx_bits;   // [T * kWords] displaced indices
    uint64_t* tile_max;   // [T] -> exclusive prefix max over tiles (in place)
    uint64_t* tile_min;   // [T] -> exclusive suffix min over tiles (in place)
    uint32_t* pos_cnt;    // [T] displaced positions per tile -> exclusive offsets
    uint32_t* idx_cnt;    // [T] displaced indices per tile -> exclusive offsets
    int64_t* counts;      // [0] displaced count to sort (0: none), [1] full-sort count (0 or n)
    uint32_t* disp_pos;   // [n / 2] displaced positions, ascending
    uint32_t* disp_idx;   // [n / 2] displaced indices, ascending
    float* disp_a;        // [n / 2] a[disp_idx]
    float* disp_sorted;   // [n / 2] sorted displaced anchors
    uint32_t* disp_perm;  // [n / 2] their ranks into disp_idx
    void* disp_ws;        // workspace of the displaced sort
    void* full_ws;        // workspace of the full sort (overlaps the rest: it runs last)
};

// Layout: [ warm-path buffers | ... ] overlapped by the full sort's workspace
// (it runs last, after the rest is consumed), then the two counts, which both
// paths read, in a slot of their own.
size_t resort_shared_bytes(int64_t n, ResortWs* w, char* ws) {
    const int64_t T = (n + kTile - 1) / kTile, h = (n + 1) / 2;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* q = ws ? ws + off : nullptr;
        off += align_up(bytes, 256);
        return (void*)q;
    };
    ResortWs v;
    v.full_ws = ws;
    v.keys = (uint32_t*)take((size_t)n * 4);
    v.pos_bits = (uint32_t*)take((size_t)T * kWords * 4);
    v.idx_bits = (uint32_t*)take((size_t)T * kWords * 4);
    v.tile_max = (uint64_t*)take((size_t)T * 8);
    v.tile_min = (uint64_t*)take((size_t)T * 8);
    v.pos_cnt = (uint32_t*)take((size_t)T * 4);
    v.idx_cnt = (uint32_t*)take((size_t)T * 4);
    v.disp_pos = (uint32_t*)take((size_t)h * 4);
    v.disp_idx = (uint32_t*)take((size_t)h * 4);
    v.disp_a = (float*)take((size_t)h * 4);
    v.disp_sorted = (float*)take((size_t)h * 4);
    v.disp_perm = (uint32_t*)take((size_t)h * 4);
    v.disp_ws = take(sort_workspace_bytes(h));
    off = std::max(off, align_up(sort_workspace_bytes(n), 256));
    v.counts = ws ? (int64_t*)(ws + off) : nullptr;
    off += 256;
    if (w) *w = v;
    return off;
}

// 1. keys[r] = key(a[perm_prev[r]]) (indices clamped to n - 1), the tile's max and
// min composite; non-finite anchors raise the status.
__global__ void __launch_bounds__(kNT) k_resort_gather(const float* __restrict__ a, const uint32_t* __restrict__ perm_prev,
                                                       int64_t n, ResortWs w, int32_t* status) {
    __shared__ uint64_t s_max[kNT / 32], s_min[kNT / 32];
    const int64_t base = (int64_t)blockIdx.x * kTile;
    const uint32_t last = (uint32_t)(n - 1);
    // item i of thread t: position base + (i / 4) * 4 * kNT + 4 t + i % 4, moved 16
    // bytes at a time in full tiles (the tile's max and min do not depend on order)
    const bool full = base + kTile <= n;
    auto pos = [&](int i) { return base + (int64_t)(i / 4) * 4 * kNT + 4 * threadIdx.x + (i % 4); };
    uint32_t idx[kItems];
    float f[kItems];
#pragma unroll
    for (int q = 0; q < kItems / 4; ++q) {
        if (full) {
            const uint4 p4 = __ldcs(reinterpret_cast<const uint4*>(perm_prev + pos(4 * q)));
            idx[4 * q] = p4.x, idx[4 * q + 1] = p4.y, idx[4 * q + 2] = p4.z, idx[4 * q + 3] = p4.w;
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) idx[4 * q + u] = pos(4 * q + u) < n ? __ldcs(perm_prev + pos(4 * q + u)) : 0u;
        }
    }
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
        idx[i] = min(idx[i], last);
        f[i] = pos(i) < n ? __ldg(a + idx[i]) : 0.f;
    }
    uint64_t mx = 0, mn = ~0ull;
    bool bad = false;
    uint32_t k[kItems];
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
        k[i] = float_to_key(f[i]);
        if (pos(i) < n) {
            bad |= is_nonfinite(f[i]);
            const uint64_t c = comp(k[i], idx[i]);
            mx = max(mx, c);
            mn = min(mn, c);
        }
    }
#pragma unroll
    for (int q = 0; q < kItems / 4; ++q) {
        if (full) {
            __stcs(reinterpret_cast<uint4*>(w.keys + pos(4 * q)),
                   make_uint4(k[4 * q], k[4 * q + 1], k[4 * q + 2], k[4 * q + 3]));
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (pos(4 * q + u) < n) w.keys[pos(4 * q + u)] = k[4 * q + u];
        }
    }
    if (bad) raise_status(status, kStatusNonFinite);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        mx = max(mx, shfl_down_u64(mx, d));
        mn = min(mn, shfl_down_u64(mn, d));
    }
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    if (lane == 0) {
        s_max[wp] = mx;
        s_min[wp] = mn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int j = 1; j < kNT / 32; ++j) {
            mx = max(mx, s_max[j]);
            mn = min(mn, s_min[j]);
        }
        w.tile_max[blockIdx.x] = mx;
        w.tile_min[blockIdx.x] = mn;
    }
}

// 2. One CTA: tile_max[t] <- max over tiles < t, tile_min[t] <- min over tiles > t.
__global__ void __launch_bounds__(kScanNT) k_resort_tile_carries(int64_t T, ResortWs w) {
    __shared__ uint64_t s_max[kScanNT / 32], s_min[kScanNT / 32];
    const int64_t per = (T + kScanNT - 1) / kScanNT;
    const int64_t t0 = min(T, (int64_t)threadIdx.x * per), t1 = min(T, t0 + per);
    uint64_t mx = 0, mn = ~0ull;
    for (int64_t t = t0; t < t1; ++t) {
        mx = max(mx, w.tile_max[t]);
        mn = min(mn, w.tile_min[t]);
    }
    uint64_t before, after;
    block_excl_max_min<kScanNT>(mx, mn, s_max, s_min, before, after);
    for (int64_t t = t0; t < t1; ++t) {
        const uint64_t v = w.tile_max[t];
        w.tile_max[t] = before;
        before = max(before, v);
    }
    for (int64_t t = t1 - 1; t >= t0; --t) {
        const uint64_t v = w.tile_min[t];
        w.tile_min[t] = after;
        after = min(after, v);
    }
}

// 3. Classify one tile.  Thread j holds positions base + 16 j .. + 15 (16-byte
// loads); the in-tile exclusive max before each position and min after it come
// from a thread-local pass and a block scan, then the tile carries.  Every
// position gets a_sorted/perm from the old order (displaced ones are overwritten
// later); displaced positions set their bit in pos_bits, displaced indices theirs
// in idx_bits (atomically: indices are scattered).
__global__ void __launch_bounds__(kNT) k_resort_classify(const uint32_t* __restrict__ perm_prev, int64_t n, ResortWs w,
                                                         float* __restrict__ a_sorted, uint32_t* __restrict__ perm) {
    __shared__ uint64_t s_max[kNT / 32], s_min[kNT / 32];
    __shared__ uint32_t s_scan[kNT / 32];
    const int64_t base = (int64_t)blockIdx.x * kTile;
    const int64_t r0 = base + (int64_t)threadIdx.x * kItems;
    const uint32_t last = (uint32_t)(n - 1);
    uint32_t key[kItems], idx[kItems];
    if (r0 + kItems <= n) {
        const uint4* k4 = reinterpret_cast<const uint4*>(w.keys + r0);
        const uint4* p4 = reinterpret_cast<const uint4*>(perm_prev + r0);
#pragma unroll
        for (int q = 0; q < kItems / 4; ++q) {
            const uint4 kv = __ldcs(k4 + q), pv = __ldcs(p4 + q);
            key[4 * q] = kv.x, key[4 * q + 1] = kv.y, key[4 * q + 2] = kv.z, key[4 * q + 3] = kv.w;
            idx[4 * q] = pv.x, idx[4 * q + 1] = pv.y, idx[4 * q + 2] = pv.z, idx[4 * q + 3] = pv.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < kItems; ++e) {
            key[e] = r0 + e < n ? w.keys[r0 + e] : 0xffffffffu;
            idx[e] = r0 + e < n ? perm_prev[r0 + e] : 0xffffffffu;
        }
    }
    uint64_t mx = 0, mn = ~0ull;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
        idx[e] = min(idx[e], last);
        if (r0 + e < n) {
            const uint64_t c = comp(key[e], idx[e]);
            mx = max(mx, c);
            mn = min(mn, c);
        }
    }
    uint64_t before, after;
    block_excl_max_min<kNT>(mx, mn, s_max, s_min, before, after);
    before = max(before, w.tile_max[blockIdx.x]);
    after = min(after, w.tile_min[blockIdx.x]);
    // after-min per element: a backward pass over the thread's items
    uint64_t amin[kItems];
    {
        uint64_t m = after;
#pragma unroll
        for (int e = kItems - 1; e >= 0; --e) {
            amin[e] = m;
            if (r0 + e < n) m = min(m, comp(key[e], idx[e]));
        }
    }
    uint32_t bits = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
        if (r0 + e < n) {
            const uint64_t c = comp(key[e], idx[e]);
            if (!(c > before && c < amin[e])) {
                bits |= 1u << e;
                atomicOr(w.idx_bits + (idx[e] >> 5), 1u << (idx[e] & 31));
            }
            before = max(before, c);
        }
    }
    if (r0 + kItems <= n) {
        float4* a4 = reinterpret_cast<float4*>(a_sorted + r0);
        uint4* p4 = reinterpret_cast<uint4*>(perm + r0);
#pragma unroll
        for (int q = 0; q < kItems / 4; ++q) {
            __stcs(a4 + q, make_float4(key_to_float(key[4 * q]), key_to_float(key[4 * q + 1]),
                                       key_to_float(key[4 * q + 2]), key_to_float(key[4 * q + 3])));
            __stcs(p4 + q, make_uint4(idx[4 * q], idx[4 * q + 1], idx[4 * q + 2], idx[4 * q + 3]));
        }
    } else {
#pragma unroll
        for (int e = 0; e < kItems; ++e)
            if (r0 + e < n) {
                a_sorted[r0 + e] = key_to_float(key[e]);
                perm[r0 + e] = idx[e];
            }
    }
    // two threads make one bitmap word (16 positions each)
    const uint32_t other = __shfl_down_sync(0xffffffffu, bits, 1);
    if ((threadIdx.x & 1) == 0) w.pos_bits[(size_t)blockIdx.x * kWords + (threadIdx.x >> 1)] = bits | (other << 16);
    uint32_t tot;
    block_excl_sum<kNT>((uint32_t)__popc(bits), s_scan, &tot);
    if (threadIdx.x == 0) w.pos_cnt[blockIdx.x] = tot;
}

// 4. Set bits of the index bitmap per tile (one warp per tile).
__global__ void __launch_bounds__(kNT) k_resort_count_idx(int64_t T, ResortWs w) {
    const int64_t t = (int64_t)blockIdx.x * (kNT / 32) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const uint4 v = reinterpret_cast<const uint4*>(w.idx_bits + t * kWords)[lane];
    uint32_t c = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) c += __shfl_down_sync(0xffffffffu, c, d);
    if (lane == 0) w.idx_cnt[t] = c;
}

// 5. One CTA: exclusive offsets of both counts, and the path.
__global__ void __launch_bounds__(kScanNT) k_resort_offsets(int64_t n, int64_t T, ResortWs w, int32_t* path) {
    __shared__ uint32_t s_scan[kScanNT / 32];
    const int64_t per = (T + kScanNT - 1) / kScanNT;
    const int64_t t0 = min(T, (int64_t)threadIdx.x * per), t1 = min(T, t0 + per);
    uint32_t sp = 0, si = 0;
    for (int64_t t = t0; t < t1; ++t) {
        sp += w.pos_cnt[t];
        si += w.idx_cnt[t];
    }
    uint32_t mp, mi;
    uint32_t bp = block_excl_sum<kScanNT>(sp, s_scan, &mp);
    uint32_t bi = block_excl_sum<kScanNT>(si, s_scan, &mi);
    for (int64_t t = t0; t < t1; ++t) {
        const uint32_t cp = w.pos_cnt[t], ci = w.idx_cnt[t];
        w.pos_cnt[t] = bp;
        w.idx_cnt[t] = bi;
        bp += cp;
        bi += ci;
    }
    if (threadIdx.x == 0) {
        // a permutation has as many distinct displaced indices as displaced positions
        const bool full = mp != mi || (int64_t)mp > n / kMaxDisplacedDen;
        w.counts[0] = full ? 0 : (int64_t)mp;
        w.counts[1] = full ? n : 0;
        if (path != nullptr) *path = mp == 0 && !full ? kResortSorted : (full ? kResortFull : kResortRepaired);
    }
}

// 6. Compact one tile of each bitmap: threads 0..127 the position words, 128..255
// the index words (each set bit in ascending order); the displaced anchors are
// gathered with their indices.
__global__ void __launch_bounds__(kNT) k_resort_compact(const float* __restrict__ a, ResortWs w) {
    __shared__ uint32_t s_scan[kNT / 32];
    if (w.counts[0] == 0) return;
    const int t = blockIdx.x;
    const bool is_idx = threadIdx.x >= kWords;
    const int j = threadIdx.x & (kWords - 1);
    const uint32_t word = (is_idx ? w.idx_bits : w.pos_bits)[(size_t)t * kWords + j];
    __shared__ uint32_t s_half;
    uint32_t tot;
    uint32_t off = block_excl_sum<kNT>((uint32_t)__popc(word), s_scan, &tot);
    // the index half starts after the position half's total: the offset at thread kWords
    if (threadIdx.x == kWords) s_half = off;
    __syncthreads();
    if (is_idx) off -= s_half;
    const uint32_t g = (is_idx ? w.idx_cnt[t] : w.pos_cnt[t]) + off;
    const uint32_t first = (uint32_t)t * kTile + (uint32_t)j * 32;
    uint32_t m = word, q = 0;
    while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t v = first + (uint32_t)b;
        if (is_idx) {
            w.disp_idx[g + q] = v;
            w.disp_a[g + q] = __ldg(a + v);
        } else {
            w.disp_pos[g + q] = v;
        }
        ++q;
    }
}

// 7. Place the sorted displaced anchors into the displaced positions.
__global__ void __launch_bounds__(kNT) k_resort_place(ResortWs w, float* __restrict__ a_sorted,
                                                      uint32_t* __restrict__ perm) {
    const int64_t m = w.counts[0];
    for (int64_t t = (int64_t)blockIdx.x * kNT + threadIdx.x; t < m; t += (int64_t)gridDim.x * kNT) {
        const uint32_t p = w.disp_pos[t];
        a_sorted[p] = w.disp_sorted[t];
        perm[p] = w.disp_idx[w.disp_perm[t]];
    }
}

}  // namespace

size_t resort_workspace_bytes(int64_t n) { return resort_shared_bytes(n, nullptr, nullptr); }

cudaError_t launch_resort(const float* a, int64_t n, const uint32_t* perm_prev, float* a_sorted, uint32_t* perm,
                          void* ws, int32_t* status, int32_t* path, cudaStream_t stream) {
    const int64_t T = (n + kTile - 1) / kTile, h = (n + 1) / 2;
    ResortWs w;
    resort_shared_bytes(n, &w, (char*)ws);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaMemsetAsync(w.idx_bits, 0, (size_t)T * kWords * 4, stream);
    if (e != cudaSuccess) return e;
    LAPLEX_TIMED("resort_gather", stream, k_resort_gather<<<(unsigned)T, kNT, 0, stream>>>(a, perm_prev, n, w, status));
    LAPLEX_TIMED("resort_scan", stream, k_resort_tile_carries<<<1, kScanNT, 0, stream>>>(T, w));
    LAPLEX_TIMED("resort_classify", stream,
                 k_resort_classify<<<(unsigned)T, kNT, 0, stream>>>(perm_prev, n, w, a_sorted, perm));
    LAPLEX_TIMED("resort_scan", stream,
                 k_resort_count_idx<<<(unsigned)((T + kNT / 32 - 1) / (kNT / 32)), kNT, 0, stream>>>(T, w));
    LAPLEX_TIMED("resort_scan", stream, k_resort_offsets<<<1, kScanNT, 0, stream>>>(n, T, w, path));
    LAPLEX_TIMED("resort_compact", stream, k_resort_compact<<<(unsigned)T, kNT, 0, stream>>>(a, w));
    e = launch_sort(w.disp_a, h, w.disp_sorted, w.disp_perm, w.disp_ws, status, stream, w.counts + 0);
    if (e != cudaSuccess) return e;
    const int pblocks = (int)std::max<int64_t>(1, std::min<int64_t>((h + kNT - 1) / kNT, (int64_t)sms * 4));
    LAPLEX_TIMED("resort_place", stream, k_resort_place<<<pblocks, kNT, 0, stream>>>(w, a_sorted, perm));
    // the full sort last: its workspace overlaps everything above
    return launch_sort(a, n, a_sorted, perm, w.full_ws, status, stream, w.counts + 1);
}

}  // namespace laplex
