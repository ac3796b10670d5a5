/*
 * laplex.h -- C ABI of the B200 (sm_100a) LAPLEX operator library, liblaplex.so.
 *
 * LAPLEX ("LAPLEX: The FFT of Learnable Laplace Kernels", Struski, Blazhko,
 * Kubaty, Tabor) is the dense matrix
 *
 *     E(a, b)_ij = exp(-|a_i - b_j|)                         (technical summary, section 2.1)
 *     E(a, phi; b, psi)_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j)   (section 2.1, phased form)
 *
 * defined by learnable 1-D anchors a (n), b (k) and optional phases phi (n),
 * psi (k).  This library applies it, its transpose, its gradients and the
 * weighted Gram operator A diag(D) A^T (section 2.2, "Gram operators") to
 * vectors without ever forming the matrix: the anchors are sorted once, after
 * which every product is a pair of linear-recurrence scans (prefix and suffix)
 * over the sorted order (section 2.2, "Exact scan algebra").  The results are
 * exact in exact arithmetic; in fp32 every output o satisfies
 * |o - o_exact| <= 1e-5 * twin(o) + 1e-30, where twin(o) is the same expression
 * evaluated with every input replaced by its absolute value.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.   Every array pointer is a DEVICE pointer to caller-owned memory.
 *             The library allocates nothing and frees nothing.  Inputs are
 *             read-only; outputs must not overlap any input or each other
 *             (LAPLEX_ERR_ARG if they do).  Every pointer must be 16-byte
 *             aligned (LAPLEX_ERR_ALIGN).
 * Layout.     Vectors are feature-major, row-major [rows][B] fp32, rows
 *             contiguous (row i holds the B batch values of feature i, the
 *             leading dimension is B).  B = 1 is a plain vector.
 * Order.      x, y, g, gradients and phases are in ORIGINAL index order.  Anchors
 *             are passed SORTED together with their permutation, exactly as
 *             laplex_sort_anchors returns them: a_sorted[r] = a[perm[r]],
 *             ascending, ties by ascending original index.  A sort can be reused
 *             while the anchors do not change.
 * Sizes.      1 <= n, k <= LAPLEX_MAX_N; 1 <= B <= LAPLEX_MAX_B.
 * Workspace.  Scratch memory is passed as (ws, ws_bytes); query the size with
 *             the matching *_workspace_size function (LAPLEX_ERR_WORKSPACE if
 *             too small).  It holds nothing between calls.
 * Saved.      Forward calls may fill an optional caller buffer `saved` (size from
 *             laplex_saved_size) that the matching laplex_backward call reads,
 *             so that the backward does not recompute the forward's scans.
 *             NULL means "do not save" (forward) / "recompute" (backward).  Its
 *             contents are opaque and only valid for the same sorted anchors.
 * Streams.    Every call enqueues its work on `stream` (a cudaStream_t; NULL is
 *             the legacy default stream) and returns without synchronising.
 * Errors.     Argument errors are returned at once, before anything is launched.
 *             Errors found by the kernels (non-finite anchors, a lookback wait
 *             that exceeded its bound) are written to the optional device word
 *             *d_status (first error wins; the caller zeroes it); read it with
 *             laplex_read_status.  After any error the outputs are unspecified.
 *             A failed launch returns LAPLEX_ERR_CUDA.
 */
#ifndef LAPLEX_H
#define LAPLEX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (same underlying type). */
typedef struct CUstream_st* laplex_stream_t;

#define LAPLEX_MAX_N 4294967295LL /* 2^32 - 1: permutations are uint32 */
#define LAPLEX_MAX_B 1024

typedef enum laplex_status {
    LAPLEX_OK = 0,
    LAPLEX_ERR_ARG = 1,       /* bad size, NULL pointer, overlap, bad op */
    LAPLEX_ERR_ALIGN = 2,     /* a pointer is not 16-byte aligned */
    LAPLEX_ERR_WORKSPACE = 3, /* ws_bytes smaller than the *_workspace_size answer */
    LAPLEX_ERR_NONFINITE = 4, /* an anchor (or phase) is NaN or infinite (device word) */
    LAPLEX_ERR_TIMEOUT = 5,   /* a bounded lookback wait gave up (device word) */
    LAPLEX_ERR_CUDA = 6       /* a CUDA launch or runtime call failed */
} laplex_status;

/* Operator selector for laplex_workspace_size, laplex_saved_size, laplex_backward. */
typedef enum laplex_op {
    LAPLEX_OP_SYM = 0,              /* y = K x, K = E(a, a)                      x [n][B] -> y [n][B] */
    LAPLEX_OP_GENERAL = 1,          /* y = E(a, b) x                             x [k][B] -> y [n][B] */
    LAPLEX_OP_TRANSPOSE = 2,        /* z = E(a, b)^T x                           x [n][B] -> z [k][B] */
    LAPLEX_OP_PHASED = 3,           /* y = E(a, phi; b, psi) x                   x [k][B] -> y [n][B] */
    LAPLEX_OP_PHASED_TRANSPOSE = 4, /* z = E(a, phi; b, psi)^T x                 x [n][B] -> z [k][B] */
    LAPLEX_OP_GRAM = 5              /* y = A diag(D) A^T v, A = E(a, b)          v [n][B] -> y [n][B] */
} laplex_op;

/* Human-readable name of a status code (static string). */
const char* laplex_status_string(laplex_status s);

/* Synchronise `stream`, then copy *d_status to *h_status and return it as a
 * laplex_status (LAPLEX_ERR_CUDA if the copy fails). */
laplex_status laplex_read_status(const int32_t* d_status, laplex_stream_t stream, int32_t* h_status);

/* ------------------------------------------------------------------ sort */

/* Bytes of workspace laplex_sort_anchors needs for n anchors. */
size_t laplex_sort_workspace_size(int64_t n);

/* Sort the anchors (technical summary, section 2.2: "after sorting the anchors").
 *   a         [n] fp32, original order (read only).
 *   a_sorted  [n] fp32 out: the anchors ascending; -0.0 is returned as +0.0.
 *   perm      [n] uint32 out: a_sorted[r] == a[perm[r]]; equal anchors keep
 *             ascending original index, so perm is unique (stable sort).
 * A least-significant-digit radix sort of an order-preserving uint32 key
 * (4 passes of 8 bits); up to 8192 anchors, one launch that ranks each anchor by
 * counting the (key, index) pairs below its own.  Both give the same unique order.
 * NaN or infinite anchors set LAPLEX_ERR_NONFINITE. */
laplex_status laplex_sort_anchors(const float* a, int64_t n, float* a_sorted, uint32_t* perm, void* ws,
                                  size_t ws_bytes, int32_t* d_status, laplex_stream_t stream);

/* Bytes of workspace laplex_resort_anchors needs for n anchors. */
size_t laplex_resort_workspace_size(int64_t n);

/* laplex_resort_anchors *d_path values. */
#define LAPLEX_RESORT_SORTED 0   /* a[perm_prev] was already in the stable order */
#define LAPLEX_RESORT_REPAIRED 1 /* the displaced anchors were sorted and placed */
#define LAPLEX_RESORT_FULL 2     /* the full radix sort ran */

/* Warm-start re-sort: the same output as laplex_sort_anchors(a, ...), bit for bit,
 * starting from the permutation of an earlier sort of anchors that have moved
 * since (trainable anchors between two steps; technical summary section 2.2:
 * the scans run over the sorted anchors).
 *   a          [n] fp32, original order (read only), the anchors as they are now.
 *   perm_prev  [n] uint32 (read only): any array; the fast path applies when it
 *              is a permutation of 0..n-1 that nearly sorts a.  Entries >= n are
 *              clamped to n - 1 (and then send the call to the full sort).
 *   a_sorted, perm [n] out: as laplex_sort_anchors.
 *   d_path     optional device int32 out: LAPLEX_RESORT_SORTED / _REPAIRED / _FULL.
 * An anchor whose composite (anchor, index) exceeds every one before it in the
 * order perm_prev gives and is below every one after it is already at its final
 * rank; the others (the displaced ones) are sorted by the radix sort and written
 * into the positions they leave free.  When more than half are displaced, or
 * perm_prev is not a permutation, the full radix sort of a runs instead.  The
 * choice is made on the device: the call does not synchronise.  NaN or infinite
 * anchors set LAPLEX_ERR_NONFINITE (on the fast path, those perm_prev reaches). */
laplex_status laplex_resort_anchors(const float* a, int64_t n, const uint32_t* perm_prev, float* a_sorted,
                                    uint32_t* perm, void* ws, size_t ws_bytes, int32_t* d_status, int32_t* d_path,
                                    laplex_stream_t stream);

/* ------------------------------------------------------------ operators */

/* Bytes of workspace for the forward and the backward of `op` (the larger of
 * the two).  k is ignored for LAPLEX_OP_SYM. */
size_t laplex_workspace_size(laplex_op op, int64_t n, int64_t k, int64_t B);

/* Bytes of the optional `saved` buffer that forwards of `op` fill. */
size_t laplex_saved_size(laplex_op op, int64_t n, int64_t k, int64_t B);

/* Symmetric operator (section 2.2, "symmetric case a = b"): y = K x with
 * K_ij = exp(-|a_i - a_j|), computed as the prefix scan P_r = x_r + exp(a_(r-1) - a_(r)) P_(r-1)
 * plus the mirrored suffix scan S_r, minus the diagonal counted twice:
 * y = P + S - x, in sorted order, scattered back through perm.
 *   a_sorted, perm [n]: from laplex_sort_anchors.   x [n][B] in, y [n][B] out. */
laplex_status laplex_apply_sym(const float* a_sorted, const uint32_t* perm, int64_t n, const float* x, int64_t B,
                               float* y, void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                               laplex_stream_t stream);

/* laplex_apply_sym without a workspace.  This entry point has no counterpart in
 * the paper: it is an interface convenience for callers that cannot hand the
 * library scratch memory -- code that owns no device allocator (a plain C host
 * program that only holds device pointers to its inputs and outputs), or a loop
 * that must not allocate or grow buffers between its calls.  Its scratch is a
 * static device array inside the library (LAPLEX_NOALLOC_SCRATCH_BYTES, one copy
 * per device), so the call allocates and frees nothing.  Contract:
 *   - the same arguments and result as laplex_apply_sym with saved = NULL;
 *   - size limit: n * Bp <= LAPLEX_NOALLOC_MAX_ELEMS, where Bp is B rounded up to
 *     the next of 1, 2, 4, 8, 16, 32, or to a multiple of 32 above 32 (B = 16
 *     allows n up to 65536); larger problems return LAPLEX_ERR_WORKSPACE before
 *     anything is launched -- use laplex_apply_sym for them;
 *   - the first call in each CUDA context performs a one-time setup (it looks up
 *     the device address of the static array in that context), so make it before
 *     any stream capture; a new context on the same device (after
 *     cudaDeviceReset, or another context made current) gets its own setup on
 *     its first call, since the array may then sit at another address;
 *   - on a device with many more SMs than a B200 the per-SM scan state can
 *     exceed the array at sizes below the limit: such calls also return
 *     LAPLEX_ERR_WORKSPACE before anything is launched;
 *   - calls must not overlap on one device: two calls in flight at once (on two
 *     streams, or from two host threads) share the scratch and race;
 *   - nothing has to be zeroed beforehand. */
#define LAPLEX_NOALLOC_MAX_ELEMS (1LL << 20)
#define LAPLEX_NOALLOC_SCRATCH_BYTES (8LL << 20)
laplex_status laplex_apply_sym_noalloc(const float* a_sorted, const uint32_t* perm, int64_t n, const float* x,
                                       int64_t B, float* y, int32_t* d_status, laplex_stream_t stream);

/* General rectangular operator (section 2.2, "general case a != b"): y = E x,
 * E_ij = exp(-|a_i - b_j|), x [k][B] at the b anchors, y [n][B] at the a anchors.
 * The inputs are scanned over sorted b and every a reads the state of its
 * neighbours in the merged order. */
laplex_status laplex_apply_general(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                   const uint32_t* perm_b, int64_t k, const float* x, int64_t B, float* y,
                                   void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                                   laplex_stream_t stream);

/* Transposed rectangular operator: z = E^T x, x [n][B] at a, z [k][B] at b.  The
 * inputs are summed into the intervals of sorted b (strict-left sums u, strict-
 * right sums v, ties t), then propagated across the intervals by the scan. */
laplex_status laplex_apply_transpose(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                     const uint32_t* perm_b, int64_t k, const float* x, int64_t B, float* z,
                                     void* saved, void* ws, size_t ws_bytes, int32_t* d_status,
                                     laplex_stream_t stream);

/* Phased operator (section 2.1): E_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j),
 * evaluated as the cos/sin split cos phi_i cos psi_j + sin phi_i sin psi_j (two
 * scan channels per input channel).  phi [n], psi [k] in original order.
 * transpose = 0: x [k][B] -> out [n][B];  transpose = 1: x [n][B] -> out [k][B]. */
laplex_status laplex_apply_phased(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                                  const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi,
                                  int transpose, const float* x, int64_t B, float* out, void* saved, void* ws,
                                  size_t ws_bytes, int32_t* d_status, laplex_stream_t stream);

/* Backward pass of any operator above (the anchors are trainable: abstract and
 * section 2.3, "differentiability with respect to the anchors").  Given the
 * forward's input x and the upstream gradient g (shape of the forward's output),
 * writes the gradients of <g, out>:
 *   gx   (shape of x)  = E^T g (the adjoint product),
 *   ga [n], gb [k]     anchor gradients from sign-split sums: for an output row i,
 *                      sum over the columns to its right minus the columns to
 *                      its left, d|t|/dt = sign(t) with sign(0) = 0 (tied anchors
 *                      contribute nothing),
 *   gphi [n], gpsi [k] phase gradients (phased ops only).
 * Any output pointer may be NULL to skip it; for LAPLEX_OP_SYM gb, gphi, gpsi,
 * b_sorted, perm_b, psi and phi are ignored (ga holds the whole anchor gradient).
 * `saved` is the buffer the matching forward filled, or NULL.
 * LAPLEX_OP_GRAM is not accepted here: use laplex_gram_apply. */
laplex_status laplex_backward(laplex_op op, const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* phi,
                              const float* b_sorted, const uint32_t* perm_b, int64_t k, const float* psi,
                              const float* x, const float* g, int64_t B, const void* saved, float* gx, float* ga,
                              float* gb, float* gphi, float* gpsi, void* ws, size_t ws_bytes, int32_t* d_status,
                              laplex_stream_t stream);

/* Weighted Gram operator (section 2.2, "Gram operators": M = A diag(D) A^T):
 * y = A diag(D) A^T v with A_ij = exp(-|a_i - b_j|), v, y [n][B], D [k], as two
 * rectangular scan passes (w = A^T v at b, then y = A (D w) at a).
 *   w_saved [k][B] (nullable): receives w = A^T v.
 *   g [n][B], gD [k] (both NULL or both set): also the gradient of <g, y> with
 *   respect to D, gD_j = sum_c (A^T g)_jc (A^T v)_jc. */
laplex_status laplex_gram_apply(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                const uint32_t* perm_b, int64_t k, const float* D, const float* v, int64_t B,
                                float* y, float* w_saved, const float* g, float* gD, void* ws, size_t ws_bytes,
                                int32_t* d_status, laplex_stream_t stream);

/* Every gradient of the Gram apply (section 2.2, "Gram operators"; the covariance
 * factor is trainable, abstract and section 4.2): for l = <g, A diag(D) A^T v>,
 * A_ij = exp(-|a_i - b_j|), with w = A^T v and u = A^T g,
 *   gv [n][B] = A diag(D) A^T g                 (the operator is symmetric),
 *   ga [n]    = sum_c g_ic (R - L)[D w]_ic + v_ic (R - L)[D u]_ic,
 *   gb [k]    = D_j sum_c w_jc (R' - L')[g]_jc + u_jc (R' - L')[v]_jc,
 *   gD [k]    = sum_c u_jc w_jc,
 * where (R - L)[z]_i is the sum over the b anchors strictly right of a_i minus the
 * sum over those strictly left, each weighted exp(-|a_i - b_j|) (sign(0) = 0), and
 * (R' - L')[h]_j the same over the a anchors relative to b_j.  Any output may be
 * NULL to skip it (at least one must be set); v, g [n][B] in original order.
 * Workspace: laplex_workspace_size(LAPLEX_OP_GRAM, n, k, B). */
laplex_status laplex_gram_backward(const float* a_sorted, const uint32_t* perm_a, int64_t n, const float* b_sorted,
                                   const uint32_t* perm_b, int64_t k, const float* D, const float* v, const float* g,
                                   int64_t B, float* gv, float* ga, float* gb, float* gD, void* ws, size_t ws_bytes,
                                   int32_t* d_status, laplex_stream_t stream);

/* -------------------------------------------------------- diagnostics */

/* Bytes of device workspace laplex_check_wait_bound needs. */
#define LAPLEX_CHECK_WAIT_WS_BYTES 1024

/* Failure-detection self-check (no counterpart on the pages).  Runs one warp of the
 * small-side scan's lookback against a predecessor whose status flag nothing ever
 * sets: the bounded wait must give up (after about 2^20 polls, well under a second
 * on a B200), write LAPLEX_ERR_TIMEOUT to *d_status and let the kernel finish, so
 * the context stays usable.  ws: at least LAPLEX_CHECK_WAIT_WS_BYTES of device
 * memory (overwritten); d_status: required, zeroed by the caller.  Returns
 * LAPLEX_ERR_ARG / LAPLEX_ERR_ALIGN / LAPLEX_ERR_WORKSPACE for bad arguments,
 * LAPLEX_ERR_CUDA if the launch fails, else LAPLEX_OK (read the outcome with
 * laplex_read_status). */
laplex_status laplex_check_wait_bound(void* ws, size_t ws_bytes, int32_t* d_status, laplex_stream_t stream);

/* ------------------------------------------------------------- tracing */

/* Per-kernel timing aid (no counterpart on the pages; a measurement tool).
 * laplex_profile_enable(1) clears the record and starts bracketing every kernel
 * the library launches with a pair of CUDA events recorded on the launch
 * stream; laplex_profile_enable(0) stops.  Adds one event pair per launch. */
void laplex_profile_enable(int on);

/* Synchronise on the recorded events and write, for up to max_kernels kernel
 * names, the name (NUL-terminated, at most name_len bytes, into names +
 * i * name_len), the number of launches and the summed device time in ms.
 * Clears the record.  Returns the number of distinct kernel names, or -1 if an
 * event query failed.  Any output pointer may be NULL. */
int laplex_profile_report(int max_kernels, char* names, int name_len, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* LAPLEX_H */
