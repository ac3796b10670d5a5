// Stable key-index radix sort of fp32 anchors ("LAPLEX: The FFT of Learnable
// Laplace Kernels", technical summary section 2.2: the scan algebra starts by
// sorting the anchors).
//
// Keys are the order-preserving uint32 images of the anchors (-0 folded onto
// +0), values the original indices.  Least-significant digit first, 4 passes of
// 8 bits.  Each pass is one kernel over tiles of 3840 keys claimed in order from
// an atomic counter: the tile ranks its keys stably inside each warp (the lanes
// sharing a digit found through per-digit lane words in shared memory), publishes
// its per-digit counts, looks back over the tiles
// before it for their per-digit prefixes (bounded waits), and scatters through
// shared memory so that runs of equal digits leave as contiguous stores.
// A histogram kernel computes the four global digit histograms in one read of
// the anchors and flags non-finite anchors.
#include "laplex_internal.h"

namespace laplex {

namespace {

constexpr int kNT = 256;
constexpr int kItems = 15;  // 3840-key tiles: with the values loaded late, four CTAs per SM
constexpr int kTile = kNT * kItems;
// Up to kShortMax keys a sort can take tiles of kItemsShort keys per thread
// instead, when its grid is a few waves and the smaller tiles end the last wave
// sooner (see sort_items); its workspace is sized for the smaller tiles.
constexpr int kItemsShort = 11;
constexpr int kTileShort = kNT * kItemsShort;
constexpr int64_t kShortMax = 1ll << 23;
constexpr int kNW = kNT / 32;
constexpr int kRadix = 256;
constexpr unsigned long long kValMask = (1ull << 62) - 1;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan of one value per thread over a 256-thread block.  Returns the
// exclusive prefix; *total receives the sum.
__device__ __forceinline__ uint32_t block_excl_scan_256(uint32_t v, uint32_t* s_warp, uint32_t* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) s_warp[w] = inc;
    __syncthreads();
    uint32_t base = 0, tot = 0;
#pragma unroll
    for (int j = 0; j < kNW; ++j) {
        uint32_t x = s_warp[j];
        if (j < w) base += x;
        tot += x;
    }
    __syncthreads();
    *total = tot;
    return base + inc - v;
}

__global__ void __launch_bounds__(kNT) k_radix_hist(const float* __restrict__ a, int64_t n, const int64_t* n_dev,
                                                    int tile_keys, uint32_t* hist, unsigned long long* look0,
                                                    int32_t* status) {
    __shared__ uint32_t s_hist[kNW][4][kRadix];  // one histogram set per warp: fewer colliding atomics
    if (n_dev != nullptr) n = min(n, *n_dev);  // count known only on the device (<= the launch bound)
    if (n <= 0) return;
    const int64_t look_words = (n + tile_keys - 1) / tile_keys * kRadix;
    for (int i = threadIdx.x; i < kNW * 4 * kRadix; i += kNT) (&s_hist[0][0][0])[i] = 0;
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * kNT;
    // zero the first pass's lookback region
    for (int64_t i = (int64_t)blockIdx.x * kNT + threadIdx.x; i < look_words; i += stride) look0[i] = 0ull;
    uint32_t(*wh)[kRadix] = s_hist[threadIdx.x >> 5];
    bool bad = false;
    auto add = [&](float f) {
        bad |= is_nonfinite(f);
        const uint32_t key = float_to_key(f);
        atomicAdd(&wh[0][key & 0xffu], 1u);
        atomicAdd(&wh[1][(key >> 8) & 0xffu], 1u);
        atomicAdd(&wh[2][(key >> 16) & 0xffu], 1u);
        atomicAdd(&wh[3][key >> 24], 1u);
    };
    const int64_t n4 = n / 4;  // the anchors are 16-byte aligned (ABI)
    const float4* a4 = reinterpret_cast<const float4*>(a);
    for (int64_t i = (int64_t)blockIdx.x * kNT + threadIdx.x; i < n4; i += stride) {
        const float4 v = __ldg(a4 + i);
        add(v.x);
        add(v.y);
        add(v.z);
        add(v.w);
    }
    for (int64_t i = n4 * 4 + (int64_t)blockIdx.x * kNT + threadIdx.x; i < n; i += stride) add(__ldg(a + i));
    if (bad) raise_status(status, kStatusNonFinite);
    __syncthreads();
    for (int i = threadIdx.x; i < 4 * kRadix; i += kNT) {
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < kNW; ++w) v += (&s_hist[w][0][0])[i];
        if (v) atomicAdd(hist + i, v);
    }
}

// One LSD pass.  MODE 0: keys from the fp32 anchors, values = indices.
// MODE 1: keys/values from the previous pass.  MODE 2: like 1, and the keys
// leave as fp32 anchors (last pass).
template <int MODE, int ITEMS>
__global__ void __launch_bounds__(kNT, 4) k_radix_pass(const float* __restrict__ a, const uint32_t* __restrict__ keys_in,
                                                    const uint32_t* __restrict__ vals_in, uint32_t* __restrict__ keys_out,
                                                    uint32_t* __restrict__ vals_out, int64_t n, const int64_t* n_dev,
                                                    int shift, const uint32_t* __restrict__ hist, uint32_t* counter,
                                                    unsigned long long* look, unsigned long long* look_next,
                                                    int32_t* status) {
    constexpr int TILE = kNT * ITEMS;
    __shared__ uint32_t s_whist[kNW][kRadix];
    __shared__ uint32_t s_keys[TILE];
    __shared__ uint32_t s_vals[TILE];
    __shared__ uint32_t s_base[kRadix];   // global destination of the tile's first key per digit
    __shared__ uint32_t s_start[kRadix];  // tile-local start of each digit
    __shared__ uint32_t s_scan[kNW];
    __shared__ int64_t s_tile;
    // during the ranking, the lanes of the current item holding each digit (and a
    // word for rows past n), per warp; the key buffer is free until the placement
    static_assert(kNW * (kRadix + 1) <= TILE, "peer words fit in the key buffer");
    uint32_t(*s_peer)[kRadix + 1] = reinterpret_cast<uint32_t(*)[kRadix + 1]>(s_keys);

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (n_dev != nullptr) {
        // count known only on the device (<= the launch bound): the first
        // ceil(n / TILE) CTAs claim one tile each, the others leave at once
        n = min(n, *n_dev);
        if ((int64_t)blockIdx.x * TILE >= n) return;
    }
    if (tid == 0) s_tile = atomicAdd(counter, 1u);
    for (int i = tid; i < kNW * kRadix; i += kNT) (&s_whist[0][0])[i] = 0;
    for (int i = tid; i < kNW * (kRadix + 1); i += kNT) (&s_peer[0][0])[i] = 0;
    __syncthreads();
    const int64_t tile = s_tile;
    const int64_t base = tile * TILE;
    if (base >= n) return;  // the tiles of a smaller device-side count (uniform per CTA)
    look_next[tile * kRadix + tid] = 0ull;  // the pass after next reuses this region

    // global exclusive digit offsets for this pass
    uint32_t gtot;
    const uint32_t gexcl = block_excl_scan_256(__ldg(hist + tid), s_scan, &gtot);

    // keys now; the values are loaded only when they are placed (fewer live
    // registers: four CTAs per SM)
    uint32_t key[ITEMS], rank[ITEMS];
    const int64_t wbase = base + (int64_t)w * 32 * ITEMS;
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
        const int64_t idx = wbase + i * 32 + lane;
        if (idx < n) {
            if (MODE == 0)
                key[i] = float_to_key(__ldg(a + idx));
            else
                key[i] = __ldg(keys_in + idx);
        } else {
            key[i] = 0xffffffffu;
        }
    }
    // stable rank inside the warp, items in (i, lane) order = index order.  For each
    // item the lanes holding the same digit are found in shared memory: every lane
    // ORs its lane bit into the warp's word for its digit (rows past n into a word
    // of their own), reads the word back, and the lowest of those lanes advances
    // the warp's running count of the digit and clears the word for the next item.
    // rank = running count before the item + the lanes below in the word.
    // rows of this warp's slice below n (32-bit from here on: a slice holds 32 * ITEMS)
    const int wn = (int)max((int64_t)0, min((int64_t)(32 * ITEMS), n - wbase));
    const uint32_t my_bit = 1u << lane, lt = lanemask_lt();
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
        const bool valid = i * 32 + lane < wn;
        const uint32_t d = valid ? ((key[i] >> shift) & 0xffu) : (uint32_t)kRadix;
        atomicOr(&s_peer[w][d], my_bit);
        __syncwarp();
        const uint32_t peers = s_peer[w][d];
        const uint32_t before = valid ? s_whist[w][d] : 0u;
        rank[i] = before + __popc(peers & lt);
        __syncwarp();
        if (lane == __ffs(peers) - 1) {
            if (valid) s_whist[w][d] = before + __popc(peers);
            s_peer[w][d] = 0u;
        }
        __syncwarp();
    }
    __syncthreads();
    // per-digit: warp offsets and tile count (thread tid handles digit tid)
    uint32_t cnt = 0;
#pragma unroll
    for (int j = 0; j < kNW; ++j) {
        const uint32_t c = s_whist[j][tid];
        s_whist[j][tid] = cnt;
        cnt += c;
    }
    // publish this tile's count for digit tid (tile 0's is already its inclusive prefix);
    // a lookback word carries its own status bits and nothing else is read on the
    // strength of it, so relaxed stores and loads suffice
    unsigned long long* mine = look + tile * kRadix + tid;
    st_relaxed_u64(mine, ((tile == 0 ? 2ull : 1ull) << 62) | cnt);
    uint32_t ttot;
    s_start[tid] = block_excl_scan_256(cnt, s_scan, &ttot);
    __syncthreads();
    // place keys in shared memory in (digit, rank) order
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
        if (i * 32 + lane < wn) {
            const int64_t idx = wbase + i * 32 + lane;
            const uint32_t d = (key[i] >> shift) & 0xffu;
            const uint32_t p = s_start[d] + s_whist[w][d] + rank[i];
            s_keys[p] = key[i];
            s_vals[p] = (MODE == 0) ? (uint32_t)idx : __ldg(vals_in + idx);
        }
    }
    // decoupled lookback over earlier tiles for digit tid
    {
        unsigned long long excl = 0;
        if (tile > 0) {
            // read a window of kWin predecessors per round trip, newest first, and add
            // their counts until one holds an inclusive prefix (tile 0 always does)
            constexpr int kWin = 16;
            int64_t j = tile - 1;
            bool done = false;
            while (!done) {
                unsigned long long v[kWin];
#pragma unroll
                for (int q = 0; q < kWin; ++q) v[q] = (j - q >= 0) ? ld_relaxed_u64(look + (j - q) * kRadix + tid) : (2ull << 62);
#pragma unroll
                for (int q = 0; q < kWin; ++q) {
                    if (done) break;
                    unsigned long long vv = v[q];
                    uint32_t spins = 0;
                    while ((vv >> 62) == 0) {  // not yet published: poll this one (bounded)
                        if (++spins > kSpinLimit) {
                            raise_status(status, kStatusTimeout);
                            vv = 2ull << 62;
                            break;
                        }
                        __nanosleep(32);
                        vv = ld_relaxed_u64(look + (j - q) * kRadix + tid);
                    }
                    excl += vv & kValMask;
                    done = (vv >> 62) == 2;
                }
                j -= kWin;
            }
            st_relaxed_u64(mine, (2ull << 62) | (excl + cnt));
        }
        s_base[tid] = gexcl + (uint32_t)excl;
    }
    __syncthreads();
    const int valid_count = (n - base) < TILE ? (int)(n - base) : TILE;
    for (int p = tid; p < valid_count; p += kNT) {
        const uint32_t k = s_keys[p];
        const uint32_t d = (k >> shift) & 0xffu;
        const uint32_t dst = s_base[d] + (uint32_t)(p - s_start[d]);
        if ((int64_t)dst < n) {  // always true for consistent counts; a bad count never writes out of range
            keys_out[dst] = (MODE == 2) ? __float_as_uint(key_to_float(k)) : k;
            vals_out[dst] = s_vals[p];
        }
    }
}

// ---------------------------------------------------------- small n
//
// Up to kSmallMax anchors: rank by counting.  The composites c_i = (key_i << 32 | i)
// are distinct and ordered as the stable sort orders the anchors, so the position
// of anchor i is the number of composites below c_i.  Each CTA holds all n
// composites in shared memory and ranks kRankPer of them (kRankParts threads per
// anchor, each counting over every kRankParts-th composite: consecutive words, no
// bank conflicts), then writes those anchors to their positions.  One launch of
// ceil(n / kRankPer) CTAs instead of five; the result equals the radix sort's.

constexpr int kSmallMax = 8192;
constexpr int kRankParts = 8;
constexpr int kRankPer = 32;
constexpr int kRankNT = kRankParts * kRankPer;

__global__ void __launch_bounds__(kRankNT) k_sort_small(const float* __restrict__ a, int n,
                                                        float* __restrict__ a_sorted, uint32_t* __restrict__ perm,
                                                        int32_t* status) {
    extern __shared__ unsigned long long s_c[];  // n composites
    for (int i = threadIdx.x; i < n; i += kRankNT)
        s_c[i] = ((unsigned long long)float_to_key(__ldg(a + i)) << 32) | (unsigned)i;
    __syncthreads();
    const int el = blockIdx.x * kRankPer + threadIdx.x / kRankParts, part = threadIdx.x % kRankParts;
    const unsigned long long mine = el < n ? s_c[el] : 0ull;
    int below = 0;
    for (int q = part; q < n; q += kRankParts) below += s_c[q] < mine;
#pragma unroll
    for (int d = 1; d < kRankParts; d <<= 1) below += __shfl_xor_sync(0xffffffffu, below, d);
    if (part == 0 && el < n) {
        if (is_nonfinite(__ldg(a + el))) raise_status(status, kStatusNonFinite);
        a_sorted[below] = key_to_float((uint32_t)(mine >> 32));
        perm[below] = (uint32_t)mine;
    }
}

// ---------------------------------------------------------- unpermute
//
// out[perm[r]] = v[r] for vectors whose rows are single floats and too large for
// the L2.  A direct scatter makes every 4-byte store a separate sector request
// (about 23 G stores/s fully random on a B200, 34 G/s inside 16 MB windows,
// 93 G/s inside 64 KB windows), so the (destination, value) pairs are regrouped
// instead: two split passes group them by 16 bits of the destination (8 bits
// each), so that window q holds exactly the destinations [q << s, (q + 1) << s)
// (its size and where its pairs go follow from n alone: no histogram, no lookback,
// and the order inside a window is free), then one CTA per window places its
// values in shared memory and writes the window out contiguously.

constexpr int kSplitItems = 16;
constexpr int kSplitTile = kNT * kSplitItems;
constexpr int kPlaceMaxWindow = 1 << 14;  // floats of a window placed in shared memory

// One tile of pairs: the bucket of p is p >> shift; the tile's pairs all share
// its bits above the lowest 8 (the first pass has at most 256 buckets, and the
// second pass's tiles lie inside one first-pass bucket).  Per-bucket counts
// (shared atomics), a block scan into per-bucket starts, one global cursor claim
// per bucket, then runs of equal buckets leave as contiguous stores.
// IOTA: the values are the pairs' own positions (their uint32 bits in a float
// slot), not read from v_in: out[p[i]] = i builds the inverse permutation.
// TWO: a second value per destination travels along (vb_in -> vb_out), read when
// the tile is placed in shared memory (dynamic shared memory: kSplitTile floats).
template <bool IOTA, bool TWO>
__global__ void __launch_bounds__(kNT, 4) k_bucket_split(const uint32_t* __restrict__ p_in, const float* __restrict__ v_in,
                                                      int64_t n, int shift, uint32_t* cursor, uint32_t* __restrict__ p_out,
                                                      float* __restrict__ v_out, const float* __restrict__ vb_in,
                                                      float* __restrict__ vb_out) {
    __shared__ uint32_t s_cnt[kRadix], s_start[kRadix], s_base[kRadix], s_scan[kNW];
    __shared__ uint32_t s_p[kSplitTile];
    __shared__ float s_v[kSplitTile];
    extern __shared__ float s_vb[];  // TWO only
    const int tid = threadIdx.x;
    const int64_t base = (int64_t)blockIdx.x * kSplitTile;
    s_cnt[tid] = 0;
    __syncthreads();
    const uint32_t last = (uint32_t)(n - 1);
    uint32_t pv[kSplitItems], rk[kSplitItems];
    float vv[kSplitItems];
    // item i of thread tid: position base + (i / 4) * 4 * kNT + 4 * tid + i % 4 (the
    // order inside a bucket is free), loaded 16 bytes at a time in full tiles
    const bool full = base + kSplitTile <= n;
#pragma unroll
    for (int q = 0; q < kSplitItems / 4; ++q) {
        const int64_t idx0 = base + (int64_t)q * 4 * kNT + 4 * tid;
        if (full) {
            const uint4 p4 = __ldcs(reinterpret_cast<const uint4*>(p_in + idx0));
            pv[4 * q] = p4.x, pv[4 * q + 1] = p4.y, pv[4 * q + 2] = p4.z, pv[4 * q + 3] = p4.w;
            if (!IOTA) {
                const float4 v4 = __ldcs(reinterpret_cast<const float4*>(v_in + idx0));
                vv[4 * q] = v4.x, vv[4 * q + 1] = v4.y, vv[4 * q + 2] = v4.z, vv[4 * q + 3] = v4.w;
            }
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                pv[4 * q + u] = idx0 + u < n ? __ldcs(p_in + idx0 + u) : 0u;
                if (!IOTA) vv[4 * q + u] = idx0 + u < n ? __ldcs(v_in + idx0 + u) : 0.f;
            }
        }
        if (IOTA) {
#pragma unroll
            for (int u = 0; u < 4; ++u) vv[4 * q + u] = __uint_as_float((uint32_t)(idx0 + u));
        }
    }
#pragma unroll
    for (int i = 0; i < kSplitItems; ++i) {
        const int64_t idx = base + (int64_t)(i / 4) * 4 * kNT + 4 * tid + (i % 4);
        if (idx < n) {
            pv[i] = min(pv[i], last);
            rk[i] = atomicAdd(&s_cnt[(pv[i] >> shift) & 0xffu], 1u);
        }
    }
    __syncthreads();
    const uint32_t hi = ((min(__ldg(p_in + base), last)) >> shift) & ~0xffu;  // the tile's common upper bits
    uint32_t tot;
    const uint32_t cnt = s_cnt[tid];
    s_start[tid] = block_excl_scan_256(cnt, s_scan, &tot);
    if (cnt) s_base[tid] = atomicAdd(cursor + (hi | tid), cnt);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kSplitItems; ++i) {
        const int64_t idx = base + (int64_t)(i / 4) * 4 * kNT + 4 * tid + (i % 4);
        if (idx < n) {
            const uint32_t q = s_start[(pv[i] >> shift) & 0xffu] + rk[i];
            s_p[q] = pv[i];
            s_v[q] = vv[i];
            if (TWO) s_vb[q] = __ldcs(vb_in + idx);
        }
    }
    __syncthreads();
    const int count = (n - base) < kSplitTile ? (int)(n - base) : kSplitTile;
    for (int q = tid; q < count; q += kNT) {
        const uint32_t p = s_p[q], b = (p >> shift) & 0xffu;
        const int64_t dst = (int64_t)s_base[b] + (q - (int)s_start[b]);
        if (dst < n) {  // always, for a permutation; a bad perm never writes out of range
            p_out[dst] = p;
            v_out[dst] = s_v[q];
            if (TWO) vb_out[dst] = s_vb[q];
        }
    }
}

__global__ void k_bucket_cursors(uint32_t* cursor, int64_t count, int shift) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < count) cursor[i] = (uint32_t)(i << shift);
}

// One CTA per window of W = 1 << shift destinations: its pairs (contiguous after
// the splits) go to a shared-memory copy of the window, which then leaves with
// contiguous stores.  TWO: a second value per destination (vb -> outb), placed in a
// second window copy (dynamic shared memory 2 W floats).
template <bool TWO>
__global__ void __launch_bounds__(kNT) k_place_window(const uint32_t* __restrict__ p, const float* __restrict__ v,
                                                      int64_t n, int shift, float* __restrict__ out,
                                                      const float* __restrict__ vb, float* __restrict__ outb) {
    extern __shared__ float s_win[];
    float* s_win2 = s_win + ((size_t)1 << shift);
    constexpr int U = 8;  // pairs in flight per thread
    const int64_t w0 = (int64_t)blockIdx.x << shift;
    const int cnt = (int)min((int64_t)1 << shift, n - w0);
    for (int i0 = threadIdx.x; i0 < cnt; i0 += kNT * U) {
        uint32_t pp[U];
        float vv[U], wb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kNT;
            pp[u] = i < cnt ? __ldcs(p + w0 + i) : 0xffffffffu;
            vv[u] = i < cnt ? __ldcs(v + w0 + i) : 0.f;
            if (TWO) wb[u] = i < cnt ? __ldcs(vb + w0 + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t d = (int64_t)pp[u] - w0;
            if (i0 + u * kNT < cnt && d >= 0 && d < cnt) {
                s_win[d] = vv[u];
                if (TWO) s_win2[d] = wb[u];
            }
        }
    }
    __syncthreads();
    // windows start at multiples of 2^shift >= 512 floats: 16-byte aligned
    float4* o4 = reinterpret_cast<float4*>(out + w0);
    const float4* w4 = reinterpret_cast<const float4*>(s_win);
    for (int i = threadIdx.x; i < cnt / 4; i += kNT) __stcs(o4 + i, w4[i]);
    for (int i = (cnt / 4) * 4 + threadIdx.x; i < cnt; i += kNT) __stcs(out + w0 + i, s_win[i]);
    if (TWO) {
        float4* ob4 = reinterpret_cast<float4*>(outb + w0);
        const float4* wb4 = reinterpret_cast<const float4*>(s_win2);
        for (int i = threadIdx.x; i < cnt / 4; i += kNT) __stcs(ob4 + i, wb4[i]);
        for (int i = (cnt / 4) * 4 + threadIdx.x; i < cnt; i += kNT) __stcs(outb + w0 + i, s_win2[i]);
    }
}

// out[p[i]] = v[i] (v null: the position i itself, as uint32 bits), i in order,
// for windows too large for shared memory.
__global__ void __launch_bounds__(kNT) k_scatter_pairs(const uint32_t* __restrict__ p, const float* __restrict__ v,
                                                       int64_t n, float* __restrict__ out,
                                                       const float* __restrict__ vb = nullptr,
                                                       float* __restrict__ outb = nullptr) {
    const int64_t stride = (int64_t)gridDim.x * kNT * 4;
    for (int64_t i0 = (int64_t)blockIdx.x * kNT * 4 + threadIdx.x; i0 < n; i0 += stride) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * kNT;
            if (i < n) {
                const uint32_t d = __ldcs(p + i);
                if ((int64_t)d < n) {
                    out[d] = v != nullptr ? __ldcs(v + i) : __uint_as_float((uint32_t)i);
                    if (vb != nullptr) outb[d] = __ldcs(vb + i);
                }
            }
        }
    }
}

}  // namespace

size_t unpermute_workspace_bytes(int64_t n) {
    return 3 * align_up((size_t)n * 4, 256) + (size_t)4 * 65536;
}

cudaError_t launch_unpermute(const uint32_t* perm, float* v, int64_t n, float* out, void* ws, cudaStream_t stream) {
    return launch_place(perm, v, n, out, ws, v, stream);
}

cudaError_t launch_unpermute2(const uint32_t* perm, float* va, float* vb, int64_t n, float* outa, float* outb,
                              float* v1b, void* ws, cudaStream_t stream) {
    return launch_place(perm, va, n, outa, ws, va, stream, vb, outb, v1b, vb);
}

cudaError_t launch_inverse_perm(const uint32_t* perm, int64_t n, uint32_t* inv, void* ws, float* v2,
                                cudaStream_t stream) {
    return launch_place(perm, nullptr, n, reinterpret_cast<float*>(inv), ws, v2, stream);
}

cudaError_t launch_place(const uint32_t* perm, const float* v, int64_t n, float* out, void* ws, float* v2,
                         cudaStream_t stream, const float* vb, float* outb, float* v1b, float* v2b) {
    if (n <= 0) return cudaSuccess;
    const bool two = vb != nullptr;
    if (two && (v == nullptr || outb == nullptr || v1b == nullptr || v2b == nullptr)) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const auto scatter_grid = [&](int64_t m) {
        return (int)std::max<int64_t>(1, std::min<int64_t>((m + kNT * 4 - 1) / (kNT * 4), (int64_t)sms * 8));
    };
    int bits = 0;
    while ((1ll << bits) < n) ++bits;
    // two 8-bit levels above the window bits s2 (windows of 2^s2 destinations)
    const int s2 = bits > 16 ? bits - 16 : 0, s1 = s2 + 8;
    if (s1 < 12) {  // second-level tiles would straddle first-level buckets: one plain scatter
        LAPLEX_TIMED("unpermute_place", stream,
                     k_scatter_pairs<<<scatter_grid(n), kNT, 0, stream>>>(perm, v, n, out, vb, outb));
        return cudaGetLastError();
    }
    char* q = (char*)ws;
    uint32_t* p1 = (uint32_t*)q;
    q += align_up((size_t)n * 4, 256);
    float* v1 = (float*)q;
    q += align_up((size_t)n * 4, 256);
    uint32_t* p2 = (uint32_t*)q;
    q += align_up((size_t)n * 4, 256);
    uint32_t* cursor = (uint32_t*)q;  // 65536 entries
    // v2 (the second split's values) may be v itself: v is read only by the first split
    const int64_t tiles = (n + kSplitTile - 1) / kSplitTile;
    const int64_t nb1 = ((n - 1) >> s1) + 1, nb2 = ((n - 1) >> s2) + 1;  // buckets of each level
    static PerDevice ready;
    if (!ready.here()) {
        cudaError_t e = cudaFuncSetAttribute(k_place_window<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(float) * kPlaceMaxWindow));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_place_window<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(2 * sizeof(float) * kPlaceMaxWindow));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_bucket_split<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(sizeof(float) * kSplitTile));
        if (e != cudaSuccess) return e;
        ready.here() = 1;
    }
    const size_t sb = two ? sizeof(float) * kSplitTile : 0;
    LAPLEX_TIMED("unpermute_split", stream, k_bucket_cursors<<<1, kRadix, 0, stream>>>(cursor, nb1, s1));
    if (v == nullptr)
        LAPLEX_TIMED("unpermute_split", stream,
                     k_bucket_split<true, false><<<(unsigned)tiles, kNT, 0, stream>>>(perm, nullptr, n, s1, cursor, p1,
                                                                                     v1, nullptr, nullptr));
    else if (two)
        LAPLEX_TIMED("unpermute_split", stream,
                     k_bucket_split<false, true><<<(unsigned)tiles, kNT, sb, stream>>>(perm, v, n, s1, cursor, p1, v1,
                                                                                      vb, v1b));
    else
        LAPLEX_TIMED("unpermute_split", stream,
                     k_bucket_split<false, false><<<(unsigned)tiles, kNT, 0, stream>>>(perm, v, n, s1, cursor, p1, v1,
                                                                                      nullptr, nullptr));
    // bucket q of the first level fills [q << s1, (q + 1) << s1) and 2^s1 is a
    // multiple of the tile, so every second-level tile lies inside one of them
    LAPLEX_TIMED("unpermute_split", stream,
                 k_bucket_cursors<<<(unsigned)((nb2 + kNT - 1) / kNT), kNT, 0, stream>>>(cursor, nb2, s2));
    if (two)
        LAPLEX_TIMED("unpermute_split", stream,
                     k_bucket_split<false, true><<<(unsigned)tiles, kNT, sb, stream>>>(p1, v1, n, s2, cursor, p2, v2,
                                                                                      v1b, v2b));
    else
        LAPLEX_TIMED("unpermute_split", stream,
                     k_bucket_split<false, false><<<(unsigned)tiles, kNT, 0, stream>>>(p1, v1, n, s2, cursor, p2, v2,
                                                                                      nullptr, nullptr));
    if ((1ll << s2) <= kPlaceMaxWindow) {
        if (two)
            LAPLEX_TIMED("unpermute_place", stream,
                         k_place_window<true><<<(unsigned)nb2, kNT, 2 * (sizeof(float) << s2), stream>>>(
                             p2, v2, n, s2, out, v2b, outb));
        else
            LAPLEX_TIMED("unpermute_place", stream,
                         k_place_window<false><<<(unsigned)nb2, kNT, sizeof(float) << s2, stream>>>(p2, v2, n, s2, out,
                                                                                                   nullptr, nullptr));
    } else {
        LAPLEX_TIMED("unpermute_place", stream,
                     k_scatter_pairs<<<scatter_grid(n), kNT, 0, stream>>>(p2, v2, n, out, two ? v2b : nullptr, outb));
    }
    return cudaGetLastError();
}

// Tiles of a sort of n keys at the smallest tile sort_items may choose for it (the
// lookback regions are sized by this count).
int64_t sort_max_tiles(int64_t n) {
    const int tile = n <= kShortMax ? kTileShort : kTile;
    return (n + tile - 1) / tile;
}

// Keys per thread of the radix passes.  The tiles run as about ceil(T / slots)
// rounds of the resident CTAs (four per SM), each round lasting about one tile's
// keys per thread: when that estimate is at least 10 % lower for the short tiles,
// a sort of up to kShortMax keys takes them (n = 3 145 728: 819 tiles of 3840 keys
// are two rounds of 15, 1117 tiles of 2816 two rounds of 11).
int sort_items(int64_t n, int sms) {
    if (n > kShortMax) return kItems;
    const int64_t slots = 4ll * sms;
    auto rounds = [&](int tile) { return ((n + tile - 1) / tile + slots - 1) / slots; };
    return 10 * rounds(kTileShort) * kItemsShort <= 9 * rounds(kTile) * kItems ? kItemsShort : kItems;
}

size_t sort_workspace_bytes(int64_t n) {
    const int64_t T = sort_max_tiles(n);
    size_t b = 0;
    b += align_up((size_t)n * 4, 256);            // keys_alt
    b += align_up((size_t)n * 4, 256);            // vals_alt
    b += align_up(4 * kRadix * 4 + 64, 256);      // hist + counters
    b += 2 * align_up((size_t)T * kRadix * 8, 256);  // two lookback regions
    return b;
}

// The four LSD passes over T tiles of ITEMS keys per thread.
// pass 0: a -> alt; pass 1: alt -> out; pass 2: out -> alt; pass 3: alt -> out
template <int ITEMS>
cudaError_t launch_passes(const float* a, int64_t n, const int64_t* n_dev, int64_t T, uint32_t* keys_alt,
                          uint32_t* vals_alt, float* a_sorted, uint32_t* perm, const uint32_t* hist,
                          uint32_t* counters, unsigned long long* const* look, int32_t* status, cudaStream_t stream) {
    uint32_t* ka = (uint32_t*)a_sorted;
    const dim3 grid((unsigned)T);
    LAPLEX_TIMED("radix_pass", stream,
                 (k_radix_pass<0, ITEMS><<<grid, kNT, 0, stream>>>(a, nullptr, nullptr, keys_alt, vals_alt, n, n_dev, 0,
                                                                   hist + 0 * kRadix, counters + 0, look[0], look[1],
                                                                   status)));
    LAPLEX_TIMED("radix_pass", stream,
                 (k_radix_pass<1, ITEMS><<<grid, kNT, 0, stream>>>(nullptr, keys_alt, vals_alt, ka, perm, n, n_dev, 8,
                                                                   hist + 1 * kRadix, counters + 1, look[1], look[0],
                                                                   status)));
    LAPLEX_TIMED("radix_pass", stream,
                 (k_radix_pass<1, ITEMS><<<grid, kNT, 0, stream>>>(nullptr, ka, perm, keys_alt, vals_alt, n, n_dev, 16,
                                                                   hist + 2 * kRadix, counters + 2, look[0], look[1],
                                                                   status)));
    LAPLEX_TIMED("radix_pass", stream,
                 (k_radix_pass<2, ITEMS><<<grid, kNT, 0, stream>>>(nullptr, keys_alt, vals_alt, ka, perm, n, n_dev, 24,
                                                                   hist + 3 * kRadix, counters + 3, look[1], look[0],
                                                                   status)));
    return cudaGetLastError();
}

cudaError_t launch_sort(const float* a, int64_t n, float* a_sorted, uint32_t* perm, void* ws, int32_t* status,
                        cudaStream_t stream, const int64_t* n_dev) {
    if (n_dev == nullptr && n <= kSmallMax) {
        static PerDevice ready;
        if (!ready.here()) {
            const cudaError_t e = cudaFuncSetAttribute(k_sort_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)(sizeof(unsigned long long) * kSmallMax));
            if (e != cudaSuccess) return e;
            ready.here() = 1;
        }
        LAPLEX_TIMED("sort_small", stream,
                     k_sort_small<<<(unsigned)((n + kRankPer - 1) / kRankPer), kRankNT,
                                    sizeof(unsigned long long) * n, stream>>>(a, (int)n, a_sorted, perm, status));
        return cudaGetLastError();
    }
    char* p = (char*)ws;
    uint32_t* keys_alt = (uint32_t*)p;
    p += align_up((size_t)n * 4, 256);
    uint32_t* vals_alt = (uint32_t*)p;
    p += align_up((size_t)n * 4, 256);
    uint32_t* hist = (uint32_t*)p;
    uint32_t* counters = hist + 4 * kRadix;
    p += align_up(4 * kRadix * 4 + 64, 256);
    unsigned long long* look[2];
    look[0] = (unsigned long long*)p;
    p += align_up((size_t)sort_max_tiles(n) * kRadix * 8, 256);
    look[1] = (unsigned long long*)p;

    cudaError_t e = cudaMemsetAsync(hist, 0, 4 * kRadix * 4 + 64, stream);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int items = sort_items(n, sms);
    const int tile_keys = kNT * items;
    const int64_t want = (n + kNT * 8 - 1) / (kNT * 8);
    const int hblocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
    LAPLEX_TIMED("radix_hist", stream,
                 k_radix_hist<<<hblocks, kNT, 0, stream>>>(a, n, n_dev, tile_keys, hist, look[0], status));
    const int64_t T = (n + tile_keys - 1) / tile_keys;
    return items == kItemsShort ? launch_passes<kItemsShort>(a, n, n_dev, T, keys_alt, vals_alt, a_sorted, perm, hist,
                                                            counters, look, status, stream)
                                : launch_passes<kItems>(a, n, n_dev, T, keys_alt, vals_alt, a_sorted, perm, hist,
                                                       counters, look, status, stream);
}

}  // namespace laplex
