// extern "C" entry points of liblaplex.so (declared and documented in
// include/laplex.h).  Host-side argument checks happen here, before anything is
// launched; the work itself is enqueued by the launchers in sort.cu, sym.cu and
// rect.cu.
#include <cstdio>

#include "laplex.h"
#include "laplex_internal.h"

using namespace laplex;

namespace {

struct Range {
    const void* p;
    size_t bytes;
};

bool overlaps(Range a, Range b) {
    if (a.p == nullptr || b.p == nullptr || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = (uintptr_t)a.p, a1 = a0 + a.bytes, b0 = (uintptr_t)b.p, b1 = b0 + b.bytes;
    return a0 < b1 && b0 < a1;
}

bool aligned(const void* p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

bool size_ok(int64_t v) { return v >= 1 && v <= LAPLEX_MAX_N; }

bool batch_ok(int64_t B) { return B >= 1 && B <= LAPLEX_MAX_B; }

// Every output must be disjoint from every input and from every other output.
laplex_status check_ranges(std::initializer_list<Range> ins, std::initializer_list<Range> outs) {
    for (const Range& o : outs) {
        if (!aligned(o.p)) return LAPLEX_ERR_ALIGN;
        for (const Range& i : ins)
            if (overlaps(o, i)) return LAPLEX_ERR_ARG;
    }
    for (const Range& i : ins)
        if (!aligned(i.p)) return LAPLEX_ERR_ALIGN;
    const Range* ob = outs.begin();
    for (size_t a = 0; a < outs.size(); ++a)
        for (size_t b = a + 1; b < outs.size(); ++b)
            if (overlaps(ob[a], ob[b])) return LAPLEX_ERR_ARG;
    return LAPLEX_OK;
}

laplex_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return LAPLEX_OK;
    std::fprintf(stderr, "laplex: CUDA error: %s\n", cudaGetErrorString(e));
    return LAPLEX_ERR_CUDA;
}

size_t fbytes(int64_t count) { return sizeof(float) * (size_t)count; }

// Canonical sides of a rectangular op: the output set O and the input set I.
void rect_sides(laplex_op op, const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi, Side& O, Side& I) {
    const bool phased = (op == LAPLEX_OP_PHASED || op == LAPLEX_OP_PHASED_TRANSPOSE);
    const bool transpose = (op == LAPLEX_OP_TRANSPOSE || op == LAPLEX_OP_PHASED_TRANSPOSE);
    Side A{a_sorted, perm_a, phased ? phi : nullptr, n};
    Side Bs{b_sorted, perm_b, phased ? psi : nullptr, k};
    O = transpose ? Bs : A;
    I = transpose ? A : Bs;
}

bool is_rect(laplex_op op) {
    return op == LAPLEX_OP_GENERAL || op == LAPLEX_OP_TRANSPOSE || op == LAPLEX_OP_PHASED ||
           op == LAPLEX_OP_PHASED_TRANSPOSE;
}

laplex_status rect_apply(laplex_op op, const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                         const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi, const float* x,
                         int64_t B, float* out, void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                         laplex_stream_t stream) {
    const bool phased = (op == LAPLEX_OP_PHASED || op == LAPLEX_OP_PHASED_TRANSPOSE);
    if (!size_ok(n) || !size_ok(k) || !batch_ok(B)) return LAPLEX_ERR_ARG;
    if (!a_sorted || !perm_a || !b_sorted || !perm_b || !x || !out || !ws) return LAPLEX_ERR_ARG;
    if (phased && (!phi || !psi)) return LAPLEX_ERR_ARG;
    Side O, I;
    rect_sides(op, a_sorted, perm_a, n, phi, b_sorted, perm_b, k, psi, O, I);
    if (ws_bytes < rect_workspace_bytes(O.m, I.m, B, phased)) return LAPLEX_ERR_WORKSPACE;
    const size_t sbytes = saved ? rect_saved_bytes(O.m, I.m, B, phased) : 0;
    laplex_status s = check_ranges(
        {{a_sorted, fbytes(n)}, {perm_a, fbytes(n)}, {b_sorted, fbytes(k)}, {perm_b, fbytes(k)},
         {phased ? phi : nullptr, fbytes(n)}, {phased ? psi : nullptr, fbytes(k)}, {x, fbytes(I.m * B)}},
        {{out, fbytes(O.m * B)}, {saved, sbytes}, {ws, ws_bytes}, {d_status, sizeof(int32_t)}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_rect_forward(O, I, x, B, out, saved, ws, d_status, (cudaStream_t)stream));
}

}  // namespace

extern "C" {

const char* laplex_status_string(laplex_status s) {
    switch (s) {
        case LAPLEX_OK: return "ok";
        case LAPLEX_ERR_ARG: return "invalid argument";
        case LAPLEX_ERR_ALIGN: return "pointer not 16-byte aligned";
        case LAPLEX_ERR_WORKSPACE: return "workspace too small";
        case LAPLEX_ERR_NONFINITE: return "non-finite anchor";
        case LAPLEX_ERR_TIMEOUT: return "lookback wait exceeded its bound";
        case LAPLEX_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

laplex_status laplex_read_status(const int32_t* d_status, laplex_stream_t stream, int32_t* h_status) {
    if (!d_status || !h_status) return LAPLEX_ERR_ARG;
    cudaError_t e = cudaMemcpyAsync(h_status, d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
    return (laplex_status)*h_status;
}

laplex_status laplex_check_wait_bound(void* ws, size_t ws_bytes, int32_t* d_status, laplex_stream_t stream) {
    if (!ws || !d_status) return LAPLEX_ERR_ARG;
    if (ws_bytes < LAPLEX_CHECK_WAIT_WS_BYTES) return LAPLEX_ERR_WORKSPACE;
    laplex_status s = check_ranges({}, {{ws, ws_bytes}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_check_wait_bound(ws, d_status, (cudaStream_t)stream));
}

size_t laplex_sort_workspace_size(int64_t n) { return size_ok(n) ? sort_workspace_bytes(n) : 0; }

laplex_status laplex_sort_anchors(const float* a, int64_t n, float* a_sorted, uint32_t* perm, void* ws,
                                  size_t ws_bytes, int32_t* d_status, laplex_stream_t stream) {
    if (!size_ok(n) || !a || !a_sorted || !perm || !ws) return LAPLEX_ERR_ARG;
    if (ws_bytes < sort_workspace_bytes(n)) return LAPLEX_ERR_WORKSPACE;
    laplex_status s = check_ranges({{a, fbytes(n)}},
                                   {{a_sorted, fbytes(n)}, {perm, fbytes(n)}, {ws, ws_bytes}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_sort(a, n, a_sorted, perm, ws, d_status, (cudaStream_t)stream));
}

size_t laplex_resort_workspace_size(int64_t n) { return size_ok(n) ? resort_workspace_bytes(n) : 0; }

laplex_status laplex_resort_anchors(const float* a, int64_t n, const uint32_t* perm_prev, float* a_sorted,
                                    uint32_t* perm, void* ws, size_t ws_bytes, int32_t* d_status, int32_t* d_path,
                                    laplex_stream_t stream) {
    if (!size_ok(n) || !a || !perm_prev || !a_sorted || !perm || !ws) return LAPLEX_ERR_ARG;
    if (ws_bytes < resort_workspace_bytes(n)) return LAPLEX_ERR_WORKSPACE;
    laplex_status s = check_ranges({{a, fbytes(n)}, {perm_prev, fbytes(n)}},
                                   {{a_sorted, fbytes(n)}, {perm, fbytes(n)}, {ws, ws_bytes}, {d_status, 4}, {d_path, 4}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_resort(a, n, perm_prev, a_sorted, perm, ws, d_status, d_path, (cudaStream_t)stream));
}

size_t laplex_workspace_size(laplex_op op, int64_t n, int64_t k, int64_t B) {
    if (!size_ok(n) || !batch_ok(B)) return 0;
    if (op == LAPLEX_OP_SYM) return sym_workspace_bytes(n, B);
    if (!size_ok(k)) return 0;
    if (op == LAPLEX_OP_GRAM) return gram_workspace_bytes(n, k, B);
    if (!is_rect(op)) return 0;
    const bool phased = (op == LAPLEX_OP_PHASED || op == LAPLEX_OP_PHASED_TRANSPOSE);
    const bool transpose = (op == LAPLEX_OP_TRANSPOSE || op == LAPLEX_OP_PHASED_TRANSPOSE);
    return transpose ? rect_workspace_bytes(k, n, B, phased) : rect_workspace_bytes(n, k, B, phased);
}

size_t laplex_saved_size(laplex_op op, int64_t n, int64_t k, int64_t B) {
    if (!size_ok(n) || !batch_ok(B)) return 0;
    if (op == LAPLEX_OP_SYM) return sym_saved_bytes(n, B);
    if (!size_ok(k) || !is_rect(op)) return 0;
    const bool phased = (op == LAPLEX_OP_PHASED || op == LAPLEX_OP_PHASED_TRANSPOSE);
    const bool transpose = (op == LAPLEX_OP_TRANSPOSE || op == LAPLEX_OP_PHASED_TRANSPOSE);
    return transpose ? rect_saved_bytes(k, n, B, phased) : rect_saved_bytes(n, k, B, phased);
}

laplex_status laplex_apply_sym(const float* a_sorted, const uint32_t* perm, int64_t n, const float* x, int64_t B,
                               float* y, void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                               laplex_stream_t stream) {
    if (!size_ok(n) || !batch_ok(B) || !a_sorted || !perm || !x || !y || !ws) return LAPLEX_ERR_ARG;
    if (ws_bytes < sym_workspace_bytes(n, B)) return LAPLEX_ERR_WORKSPACE;
    const size_t sbytes = saved ? sym_saved_bytes(n, B) : 0;
    laplex_status s = check_ranges({{a_sorted, fbytes(n)}, {perm, fbytes(n)}, {x, fbytes(n * B)}},
                                   {{y, fbytes(n * B)}, {saved, sbytes}, {ws, ws_bytes}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_sym_forward(a_sorted, perm, n, x, B, y, saved, ws, d_status, (cudaStream_t)stream));
}

laplex_status laplex_apply_sym_noalloc(const float* a_sorted, const uint32_t* perm, int64_t n, const float* x,
                                       int64_t B, float* y, int32_t* d_status, laplex_stream_t stream) {
    if (!size_ok(n) || !batch_ok(B) || !a_sorted || !perm || !x || !y) return LAPLEX_ERR_ARG;
    if (n > LAPLEX_NOALLOC_MAX_ELEMS / sym_padded_batch(B)) return LAPLEX_ERR_WORKSPACE;
    if (!sym_noalloc_fits(n, B)) return LAPLEX_ERR_WORKSPACE;  // the plan on this device's SM count
    laplex_status s = check_ranges({{a_sorted, fbytes(n)}, {perm, fbytes(n)}, {x, fbytes(n * B)}},
                                   {{y, fbytes(n * B)}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    return cuda_status(launch_sym_forward_noalloc(a_sorted, perm, n, x, B, y, d_status, (cudaStream_t)stream));
}

laplex_status laplex_apply_general(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                   const uint32_t* perm_b, int64_t k, const float* x, int64_t B, float* y,
                                   void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                                   laplex_stream_t stream) {
    return rect_apply(LAPLEX_OP_GENERAL, a_sorted, perm_a, n, nullptr, b_sorted, perm_b, k, nullptr, x, B, y, saved,
                      ws, ws_bytes, d_status, stream);
}

laplex_status laplex_apply_transpose(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                     const uint32_t* perm_b, int64_t k, const float* x, int64_t B, float* z,
                                     void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                                     laplex_stream_t stream) {
    return rect_apply(LAPLEX_OP_TRANSPOSE, a_sorted, perm_a, n, nullptr, b_sorted, perm_b, k, nullptr, x, B, z, saved,
                      ws, ws_bytes, d_status, stream);
}

laplex_status laplex_apply_phased(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                                  const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi,
                                  int transpose, const float* x, int64_t B, float* out, void* saved, void* ws,
                                  size_t ws_bytes, int32_t* d_status, laplex_stream_t stream) {
    return rect_apply(transpose ? LAPLEX_OP_PHASED_TRANSPOSE : LAPLEX_OP_PHASED, a_sorted, perm_a, n, phi, b_sorted,
                      perm_b, k, psi, x, B, out, saved, ws, ws_bytes, d_status, stream);
}

laplex_status laplex_backward(laplex_op op, const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                              const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi,
                              const float* x, const float* g, int64_t B, const void* saved, float* gx, float* ga,
                              float* gb, float* gphi, float* gpsi, void* ws, size_t ws_bytes, int32_t* d_status,
                              laplex_stream_t stream) {
    if (!size_ok(n) || !batch_ok(B) || !a_sorted || !perm_a || !x || !g || !ws) return LAPLEX_ERR_ARG;
    if (op == LAPLEX_OP_SYM) {
        if (ws_bytes < sym_workspace_bytes(n, B)) return LAPLEX_ERR_WORKSPACE;
        const size_t sbytes = saved ? sym_saved_bytes(n, B) : 0;
        laplex_status s = check_ranges(
            {{a_sorted, fbytes(n)}, {perm_a, fbytes(n)}, {x, fbytes(n * B)}, {g, fbytes(n * B)}, {saved, sbytes}},
            {{gx, fbytes(n * B)}, {ga, fbytes(n)}, {ws, ws_bytes}, {d_status, 4}});
        if (s != LAPLEX_OK) return s;
        return cuda_status(
            launch_sym_backward(a_sorted, perm_a, n, x, g, B, saved, gx, ga, ws, d_status, (cudaStream_t)stream));
    }
    if (!is_rect(op)) return LAPLEX_ERR_ARG;
    const bool phased = (op == LAPLEX_OP_PHASED || op == LAPLEX_OP_PHASED_TRANSPOSE);
    const bool transpose = (op == LAPLEX_OP_TRANSPOSE || op == LAPLEX_OP_PHASED_TRANSPOSE);
    if (!size_ok(k) || !b_sorted || !perm_b) return LAPLEX_ERR_ARG;
    if (phased && (!phi || !psi)) return LAPLEX_ERR_ARG;
    Side O, I;
    rect_sides(op, a_sorted, perm_a, n, phi, b_sorted, perm_b, k, psi, O, I);
    if (ws_bytes < rect_workspace_bytes(O.m, I.m, B, phased)) return LAPLEX_ERR_WORKSPACE;
    const size_t sbytes = saved ? rect_saved_bytes(O.m, I.m, B, phased) : 0;
    if (!phased) gphi = gpsi = nullptr;
    laplex_status s = check_ranges({{a_sorted, fbytes(n)}, {perm_a, fbytes(n)}, {b_sorted, fbytes(k)},
                                    {perm_b, fbytes(k)}, {phased ? phi : nullptr, fbytes(n)},
                                    {phased ? psi : nullptr, fbytes(k)}, {x, fbytes(I.m * B)},
                                    {g, fbytes(O.m * B)}, {saved, sbytes}},
                                   {{gx, fbytes(I.m * B)}, {ga, fbytes(n)}, {gb, fbytes(k)}, {gphi, fbytes(n)},
                                    {gpsi, fbytes(k)}, {ws, ws_bytes}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    float* gO = transpose ? gb : ga;
    float* gI = transpose ? ga : gb;
    float* gtO = transpose ? gpsi : gphi;
    float* gtI = transpose ? gphi : gpsi;
    return cuda_status(
        launch_rect_backward(O, I, x, g, B, saved, gx, gO, gI, gtO, gtI, ws, d_status, (cudaStream_t)stream));
}

laplex_status laplex_gram_apply(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                const uint32_t* perm_b, int64_t k, const float* D, const float* v, int64_t B,
                                float* y, float* w_saved, const float* g, float* gD, void* ws, size_t ws_bytes,
                                int32_t* d_status, laplex_stream_t stream) {
    if (!size_ok(n) || !size_ok(k) || !batch_ok(B)) return LAPLEX_ERR_ARG;
    if (!a_sorted || !perm_a || !b_sorted || !perm_b || !D || !v || !y || !ws) return LAPLEX_ERR_ARG;
    if ((g == nullptr) != (gD == nullptr)) return LAPLEX_ERR_ARG;
    if (ws_bytes < gram_workspace_bytes(n, k, B)) return LAPLEX_ERR_WORKSPACE;
    laplex_status s = check_ranges({{a_sorted, fbytes(n)}, {perm_a, fbytes(n)}, {b_sorted, fbytes(k)},
                                    {perm_b, fbytes(k)}, {D, fbytes(k)}, {v, fbytes(n * B)}, {g, fbytes(n * B)}},
                                   {{y, fbytes(n * B)}, {w_saved, fbytes(k * B)}, {gD, fbytes(k)}, {ws, ws_bytes},
                                    {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    Side A{a_sorted, perm_a, nullptr, n}, Bs{b_sorted, perm_b, nullptr, k};
    return cuda_status(launch_gram(A, Bs, D, v, B, y, w_saved, g, gD, ws, d_status, (cudaStream_t)stream));
}


laplex_status laplex_gram_backward(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                   const uint32_t* perm_b, int64_t k, const float* D, const float* v, const float* g,
                                   int64_t B, float* gv, float* ga, float* gb, float* gD, void* ws, size_t ws_bytes,
                                   int32_t* d_status, laplex_stream_t stream) {
    if (!size_ok(n) || !size_ok(k) || !batch_ok(B)) return LAPLEX_ERR_ARG;
    if (!a_sorted || !perm_a || !b_sorted || !perm_b || !D || !v || !g || !ws) return LAPLEX_ERR_ARG;
    if (!gv && !ga && !gb && !gD) return LAPLEX_ERR_ARG;
    if (ws_bytes < gram_workspace_bytes(n, k, B)) return LAPLEX_ERR_WORKSPACE;
    laplex_status s = check_ranges({{a_sorted, fbytes(n)}, {perm_a, fbytes(n)}, {b_sorted, fbytes(k)},
                                    {perm_b, fbytes(k)}, {D, fbytes(k)}, {v, fbytes(n * B)}, {g, fbytes(n * B)}},
                                   {{gv, fbytes(n * B)}, {ga, fbytes(n)}, {gb, fbytes(k)}, {gD, fbytes(k)},
                                    {ws, ws_bytes}, {d_status, 4}});
    if (s != LAPLEX_OK) return s;
    Side A{a_sorted, perm_a, nullptr, n}, Bs{b_sorted, perm_b, nullptr, k};
    return cuda_status(
        launch_gram_backward(A, Bs, D, v, g, B, gv, ga, gb, gD, ws, d_status, (cudaStream_t)stream));
}

}  // extern "C"
