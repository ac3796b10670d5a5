// Internal launchers behind the C ABI (include/laplex.h).  All pointers are
// device pointers; all launches go to `stream`; nothing synchronises.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace laplex {

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A value cached once per device (kernel attributes and occupancies belong to a
// device, and one process may drive several).  Devices past kMaxDevices get no
// cache: here() returns a fresh zero each time, so the setup simply reruns.
struct PerDevice {
    static constexpr int kMaxDevices = 64;
    int v[kMaxDevices] = {};
    int& here() {
        int d = 0;
        if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) {
            static thread_local int none;
            none = 0;
            return none;
        }
        return v[d];
    }
};

// profile.cu: optional CUDA-event bracket around each kernel launch.
bool profiling();
void* profile_begin(const char* name, cudaStream_t stream);
void profile_end(void* token, cudaStream_t stream);
struct ProfScope {
    void* token;
    cudaStream_t stream;
    ProfScope(const char* name, cudaStream_t st) : token(profile_begin(name, st)), stream(st) {}
    ~ProfScope() { profile_end(token, stream); }
};
#define LAPLEX_TIMED(name, stream, ...)        \
    do {                                       \
        ::laplex::ProfScope ps_(name, stream); \
        __VA_ARGS__;                           \
    } while (0)

// sort.cu
size_t sort_workspace_bytes(int64_t n);
// n_dev (optional): the count to sort, read on the device (<= n, which sizes the
// launches and the workspace); 0 makes every kernel return at once.
cudaError_t launch_sort(const float* a, int64_t n, float* a_sorted, uint32_t* perm, void* ws, int32_t* status,
                        cudaStream_t stream, const int64_t* n_dev = nullptr);

// resort.cu: warm-start re-sort from a previous permutation; *path (optional,
// device) gets which way the sorted order was reached.
constexpr int32_t kResortSorted = 0, kResortRepaired = 1, kResortFull = 2;
size_t resort_workspace_bytes(int64_t n);
cudaError_t launch_resort(const float* a, int64_t n, const uint32_t* perm_prev, float* a_sorted, uint32_t* perm,
                          void* ws, int32_t* status, int32_t* path, cudaStream_t stream);

// out[perm[r]] = v[r] (4-byte rows) through destination buckets (sort.cu); v is
// overwritten (it holds the regrouped values of the last split).
size_t unpermute_workspace_bytes(int64_t n);
cudaError_t launch_unpermute(const uint32_t* perm, float* v, int64_t n, float* out, void* ws, cudaStream_t stream);
// The same placement out[dest[i]] = v[i] with v left alone: v2 (n floats) holds the
// second split's values.  v == nullptr places the positions themselves (v[i] = i,
// uint32 bits in the float slots).
// vb, outb (both or neither): a second value per destination placed along with v
// (outb[dest[i]] = vb[i]); v1b, v2b: n floats each for its split levels (v2b may be
// vb itself).
cudaError_t launch_place(const uint32_t* dest, const float* v, int64_t n, float* out, void* ws, float* v2,
                         cudaStream_t stream, const float* vb = nullptr, float* outb = nullptr, float* v1b = nullptr,
                         float* v2b = nullptr);
// launch_unpermute of two vectors through the same permutation at once (va and vb
// are overwritten; v1b: n floats of scratch).
cudaError_t launch_unpermute2(const uint32_t* perm, float* va, float* vb, int64_t n, float* outa, float* outb,
                              float* v1b, void* ws, cudaStream_t stream);
// inv[perm[r]] = r: the inverse permutation, by the same placement (v2: n floats
// of scratch).  With it a gather v[perm[r]] into sorted order becomes the placement
// out[inv[i]] = v[i], which reads v in order.
cudaError_t launch_inverse_perm(const uint32_t* perm, int64_t n, uint32_t* inv, void* ws, float* v2,
                                cudaStream_t stream);

// sym.cu
size_t sym_workspace_bytes(int64_t n, int64_t B);
size_t sym_saved_bytes(int64_t n, int64_t B);
cudaError_t launch_sym_forward(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B, float* y,
                               void* saved, void* ws, int32_t* status, cudaStream_t stream);
cudaError_t launch_sym_backward(const float* s, const uint32_t* perm, int64_t n, const float* x, const float* g,
                                int64_t B, const void* saved, float* gx, float* ga, void* ws, int32_t* status,
                                cudaStream_t stream);
// The symmetric forward on the library's static scratch (laplex_apply_sym_noalloc):
// B rounded up to whole channel groups; whether the plan of (n, B) on the current
// device fits the scratch (checked before any launch); the launcher, which returns
// cudaErrorInvalidValue if the problem does not fit.
int64_t sym_padded_batch(int64_t B);
bool sym_noalloc_fits(int64_t n, int64_t B);
cudaError_t launch_sym_forward_noalloc(const float* s, const uint32_t* perm, int64_t n, const float* x, int64_t B,
                                       float* y, int32_t* status, cudaStream_t stream);

// rect.cu: rectangular operators in canonical form.  The "output side" O and the
// "input side" I are each a sorted anchor set with its permutation and optional
// phases (original order).
struct Side {
    const float* s;        // sorted anchors
    const uint32_t* perm;  // s[r] = anchors[perm[r]]
    const float* theta;    // phases in original order, or nullptr
    int64_t m;             // number of anchors
    // the vector rows read at this side (the input of a scan over it, the h of its
    // finish) are stored in sorted order, row r at sorted position r; outputs are
    // still placed through perm.  Only without phases.
    bool rows_sorted = false;
};

size_t rect_workspace_bytes(int64_t n_out, int64_t n_in, int64_t B, bool phased);
size_t rect_saved_bytes(int64_t n_out, int64_t n_in, int64_t B, bool phased);
// out[O] = E(O, I) x[I], x [n_in][B], out [n_out][B].
cudaError_t launch_rect_forward(Side O, Side I, const float* x, int64_t B, float* out, void* saved, void* ws,
                                int32_t* status, cudaStream_t stream);
// Gradients of <g, out> for launch_rect_forward (g at O):
//   gx [n_in][B], gO/gI anchor gradients, gtO/gtI phase gradients (each nullable).
// accumulate: add the anchor and phase gradients into gO, gI, gtO, gtI instead of
// writing them (gx is always written).
// g2 (nullable): paired rows -- channels [0, B/2) of each output-side row come from g
// and [B/2, B) from g2 (both [m_O][B/2]), so that two products with the same anchors
// share one backward (output side larger than the input side, unphased, no gx).
cudaError_t launch_rect_backward(Side O, Side I, const float* x, const float* g, int64_t B, const void* saved,
                                 float* gx, float* gO, float* gI, float* gtO, float* gtI, void* ws, int32_t* status,
                                 cudaStream_t stream, bool accumulate = false, const float* g2 = nullptr);

// The bounded lookback against a predecessor that never publishes (failure-
// detection self-check): ws holds the chain, zeroed here.
cudaError_t launch_check_wait_bound(void* ws, int32_t* status, cudaStream_t stream);

size_t gram_workspace_bytes(int64_t n, int64_t k, int64_t B);
// Every gradient of <g, A diag(D) A^T v> (each output nullable): gv [n][B] = A D A^T g,
// ga [n], gb [k] the anchor gradients, gD [k].
cudaError_t launch_gram_backward(Side A, Side Bs, const float* D, const float* v, const float* g, int64_t B,
                                 float* gv, float* ga, float* gb, float* gD, void* ws, int32_t* status,
                                 cudaStream_t stream);
cudaError_t launch_gram(Side A, Side Bs, const float* D, const float* v, int64_t B, float* y, float* w_saved,
                        const float* g, float* gD, void* ws, int32_t* status, cudaStream_t stream);

}  // namespace laplex
