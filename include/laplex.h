/*
 * laplex.h -- C ABI of liblaplex.so, the exact LAPLEX Laplace-kernel operator on
 * NVIDIA B200 (sm_100a).
 *
 * The operator (page "Riepilogo Tecnico: LAPLEX - La FFT dei Nuclei di Laplace
 * Apprendibili", gist.science technical summary of arXiv 2605.24584, §2.1
 * "L'Operatore"; same text in the French summary, §2.1):
 *
 *     K_ij = exp(-|a_i - b_j|),      a in R^n, b in R^k (learnable 1-D anchors)
 *     K_ij = exp(-|a_i - b_j|) * cos(phi_i - psi_j)     (phased variant)
 *
 * and its exact O(n log n) products (same page, §2.2 "Algebra di Scansione
 * Esatta"): sort the anchors, then evaluate the lower and upper triangular
 * parts as prefix and suffix recurrences, L_{i+1} = x_{i+1} + exp(a_i - a_{i+1}) L_i,
 * never forming K.
 *
 * Common conventions
 * ------------------
 *  - Every pointer except `bytes` in laplex_workspace_size is a DEVICE pointer
 *    on the current CUDA device, owned by the caller.  The library never
 *    allocates, frees or retains memory; it keeps no state between calls.
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *    void*; NULL is the legacy default stream).  No call synchronises, except
 *    laplex_get_device_status.
 *  - dtype LAPLEX_F32: every floating array is float; LAPLEX_F64: double.
 *    The kernels compute in that type.
 *  - Vectors with B columns are row-major [len, B], contiguous.
 *  - Every array must be 16-byte aligned; the workspace 256-byte aligned.
 *  - Sizes: 0 <= n, k < 2^31; B >= 1.  Outputs must not overlap inputs.
 *  - "sorted" anchors: ascending.  perm[r] (int32) is the caller-order index of
 *    the r-th sorted anchor, as written by laplex_sort_anchors.  When a perm
 *    pointer is non-NULL every per-anchor vector on that side (x, y, phi, ...)
 *    is in the caller's original order and the kernels gather and scatter
 *    through perm; when it is NULL those vectors are in sorted order.
 *  - Workspace: `ws` of at least laplex_workspace_size(...) bytes.  Its first
 *    256 bytes are a header holding a sticky device status word; zero the
 *    header once before first use (laplex_workspace_init).  One workspace must
 *    not be used by two calls that may run at the same time.
 *  - Errors found on the host (bad argument, workspace too small, a failed CUDA
 *    launch) return immediately with nothing enqueued, or, for a launch failure,
 *    with earlier kernels of the call possibly enqueued; laplex_last_error()
 *    then holds a message.  Errors found on the device (a non-finite anchor, an
 *    inter-block wait that ran out) are recorded in the workspace header and
 *    reported by laplex_get_device_status.  No call aborts or throws.
 */
#ifndef LAPLEX_H
#define LAPLEX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LAPLEX_OK = 0,
    LAPLEX_EINVAL = 1,      /* invalid argument (NULL, size, alignment, dtype) */
    LAPLEX_ENONFINITE = 2,  /* an anchor was NaN or +-Inf (device-detected)    */
    LAPLEX_EWORKSPACE = 3,  /* ws_bytes below laplex_workspace_size()           */
    LAPLEX_ECUDA = 4,       /* a CUDA runtime call or launch failed             */
    LAPLEX_ETIMEOUT = 5     /* a bounded inter-block wait expired (device)      */
} laplex_status;

typedef enum { LAPLEX_F32 = 0, LAPLEX_F64 = 1 } laplex_dtype;

typedef enum {
    LAPLEX_OP_SORT = 0,
    LAPLEX_OP_MATVEC_SYM = 1,
    LAPLEX_OP_MATVEC_GENERAL = 2,
    LAPLEX_OP_MATVEC_PHASED = 3,
    LAPLEX_OP_GRAM = 4,
    LAPLEX_OP_BACKWARD = 5,
    LAPLEX_OP_BACKWARD_GENERAL = 6,
    LAPLEX_OP_GRAM_MATRIX = 7,
    LAPLEX_OP_BACKWARD_PHASED = 8,
    LAPLEX_OP_PERMUTE = 9,           /* laplex_permute and laplex_invert_perm (n elements) */
    LAPLEX_OP_MATVEC_SYM_PLANNED = 10,
    LAPLEX_OP_SORT_CARRY = 11,       /* laplex_sort_anchors_carry (n anchors and values) */
    LAPLEX_OP_MATVEC_SYM_UNSORTED = 12
} laplex_op;

/* Library ABI version (major*10000 + minor*100 + patch). */
int laplex_version(void);

/* How the library was built: LAPLEX_BUILD_ACCURATE_EXP set when the fp32
 * decays use CUDA's expf (more accurate, slower) instead of the hardware
 * base-2 exponential.  No side effects; callable without a GPU. */
#define LAPLEX_BUILD_ACCURATE_EXP 1
int laplex_build_flags(void);

/* Human-readable name of a status code (static string). */
const char* laplex_status_string(laplex_status s);

/* Message of the last host-side error on the calling thread ("" if none). */
const char* laplex_last_error(void);

/*
 * Workspace bytes needed by `op` for these sizes (host only, no device work).
 * n: anchors of a; k: anchors of b (0 for symmetric ops and the sort);
 * B: columns of x (1 for the sort and the backward pass).
 * For LAPLEX_OP_SORT, n is the number of keys.  The result covers every
 * variant of the op (with or without perm, transposed or not) and includes
 * the 256-byte header.  Errors: EINVAL for negative/oversized sizes or NULL bytes.
 */
laplex_status laplex_workspace_size(laplex_op op, int64_t n, int64_t k, int64_t B,
                                    laplex_dtype dtype, size_t* bytes);

/* Zero the workspace header (async on stream).  Call once per new workspace. */
laplex_status laplex_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Wait for `stream`, read the sticky device status of `ws`, clear it, and
 * return it: LAPLEX_OK, LAPLEX_ENONFINITE or LAPLEX_ETIMEOUT (ECUDA if the
 * wait or the read fails).  The only call that synchronises.
 */
laplex_status laplex_get_device_status(void* ws, void* stream);

/*
 * Sort the anchors (the recurrences run over them in sorted order, summary
 * §2.2; the O(n log n) term of the method, §2.2 and §3).
 *   a      [n]   caller's anchors (read only).
 *   sorted [n]   out: the anchors ascending.  -0.0 is stored as +0.0.
 *   perm   [n]   out: int32, sorted[r] == a[perm[r]] (numerically); ties in
 *                ascending caller index, so perm is unique.
 * Stable LSD radix sort of the IEEE bit patterns.  A NaN or +-Inf anchor sets
 * LAPLEX_ENONFINITE in the device status (outputs then unspecified).
 * Workspace: laplex_workspace_size(LAPLEX_OP_SORT, n, 0, 1, dtype, ...).
 */
laplex_status laplex_sort_anchors(const void* a, int64_t n, laplex_dtype dtype,
                                  void* sorted, int32_t* perm,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * Sort the anchors and carry a value per anchor along (summary §2.2: the
 * recurrences run over the anchors in sorted order, and so over the entries of
 * the vector they weigh).  As laplex_sort_anchors, and
 *   x  [n]  in: one value per anchor, caller order (dtype).
 *   xs [n]  out: xs[r] == x[perm[r]], bit for bit.
 * fp32: the value rides through the digit passes beside the index payload, so
 * it reaches sorted order with coalesced writes (no random gather).  fp64: the
 * sort, then xs by laplex_invert_perm and laplex_permute inside the call.
 * sorted, perm, xs must not overlap a, x or each other.
 * Workspace: laplex_workspace_size(LAPLEX_OP_SORT_CARRY, n, 0, 1, dtype, ...).
 */
laplex_status laplex_sort_anchors_carry(const void* a, const void* x, int64_t n, laplex_dtype dtype,
                                        void* sorted, int32_t* perm, void* xs,
                                        void* ws, size_t ws_bytes, void* stream);

/*
 * Symmetric product y = K x on anchors in the caller's order, in one call
 * (B = 1; summary §2.2: sort, then the two recurrences): the sort carrying x
 * (laplex_sort_anchors_carry), the streaming product in sorted order, and y
 * back to caller order by laplex_permute(y', perm).
 *   a [n], x [n]: caller order.    y [n]: out, caller order.
 *   sorted [n], perm [n]: out, as laplex_sort_anchors writes them (for the
 *   backward pass or later products).
 * Same result as laplex_sort_anchors followed by laplex_matvec_sym(sorted, perm, ...).
 * Workspace: laplex_workspace_size(LAPLEX_OP_MATVEC_SYM_UNSORTED, n, 0, 1, dtype, ...).
 */
laplex_status laplex_matvec_sym_unsorted(const void* a, const void* x, int64_t n, laplex_dtype dtype, void* y,
                                         void* sorted, int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/*
 * Permutation by buckets (no counterpart in the paper beyond the sort itself:
 * the recurrences of summary §2.2 run over the anchors in sorted order, and a
 * caller whose vectors are in its own order moves them into and out of that
 * order).  dst[idx[i]] = src[i] for 0 <= i < n.
 *   src  [n]  elements of 4 bytes (dtype LAPLEX_F32; any 4-byte type, moved
 *             as bits) or 8 bytes (LAPLEX_F64).
 *   idx  [n]  int32 destinations, a permutation of 0..n-1; entries outside
 *             [0, n) are skipped, positions that no entry names keep their
 *             contents, and for a repeated entry one of its sources is written
 *             (which one is unspecified).
 *   dst  [n]  output; must not overlap src or idx.
 * Writing single elements at random positions of a large array moves a
 * partial 32-byte sector each; instead, stable radix digit passes over the
 * group number idx >> 14 (idx >> 13 for 8-byte elements; none for n up to one
 * group, two up to n = 2^30) order the elements by the group of 64 KiB of
 * dst they land in, and one block per group fills the group in shared memory
 * and stores it whole.
 * Workspace: laplex_workspace_size(LAPLEX_OP_PERMUTE, n, 0, 1, dtype, ...).
 */
laplex_status laplex_permute(const void* src, const int32_t* idx, int64_t n, laplex_dtype dtype,
                             void* dst, void* ws, size_t ws_bytes, void* stream);

/*
 * Inverse of a permutation: inv[perm[r]] = r (laplex_permute of the indices
 * 0..n-1).  With (sorted, perm, inv) a caller holds a plan: vectors in its
 * own order enter sorted order by laplex_permute(x, inv) and leave it by
 * laplex_permute(y, perm), both bucketed scatters, instead of the random
 * gather and scatter of the perm argument of the products.
 * Workspace: laplex_workspace_size(LAPLEX_OP_PERMUTE, n, 0, 1, LAPLEX_F32, ...).
 */
laplex_status laplex_invert_perm(const int32_t* perm, int64_t n, int32_t* inv, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * Symmetric product with a plan, y = K x for x, y in the caller's order
 * (B = 1): x moves into sorted order by laplex_permute(x, inv), the product
 * runs on the streaming path, and y moves back by laplex_permute(y', perm).
 * Same result as laplex_matvec_sym(sorted, perm, ...).
 *   sorted [n], perm [n], inv [n]: from laplex_sort_anchors and laplex_invert_perm.
 *   x [n], y [n]: caller order.
 * Workspace: laplex_workspace_size(LAPLEX_OP_MATVEC_SYM_PLANNED, n, 0, 1, dtype, ...).
 */
laplex_status laplex_matvec_sym_planned(const void* sorted, const int32_t* perm, const int32_t* inv, int64_t n,
                                        const void* x, void* y, laplex_dtype dtype, void* ws, size_t ws_bytes,
                                        void* stream);

/*
 * Symmetric product y = K x, K_ij = exp(-|a_i - a_j|) (summary §2.2, "Caso
 * Simmetrico": lower part by the prefix recurrence, upper part by the suffix
 * recurrence, y = L + U - x so that the diagonal counts once).
 *   sorted [n]      anchors ascending (from laplex_sort_anchors, or already sorted).
 *   perm   [n]|NULL see conventions: non-NULL -> x, y in caller order.
 *   x      [n, B]   input;  y [n, B] output.
 */
laplex_status laplex_matvec_sym(const void* sorted, const int32_t* perm, int64_t n,
                                const void* x, void* y, int64_t B, laplex_dtype dtype,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * General product, a != b (summary §2.2, "Caso Generale": the b-anchors'
 * contributions are collected in the intervals cut by the sorted a-anchors and
 * propagated by the symmetric recurrences; here done by one scan over the
 * merged sorted sequence of a and b).
 *   transpose = 0:  y = K x,    x [k, B] on the b side, y [n, B] on the a side.
 *   transpose = 1:  y = K^T x,  x [n, B] on the a side, y [k, B] on the b side.
 *   sa [n], pa|NULL: sorted a and its perm;  sb [k], pb|NULL: same for b.
 */
laplex_status laplex_matvec_general(const void* sa, const int32_t* pa, int64_t n,
                                    const void* sb, const int32_t* pb, int64_t k,
                                    const void* x, void* y, int64_t B, int transpose,
                                    laplex_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Phased product with K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j) (summary §2.1),
 * computed as two unphased channels through cos(p - q) = cos p cos q + sin p sin q.
 *   sb == NULL: symmetric case (b = a, psi = phi); k, pb, psi ignored.
 *   phi [n] on the a side, psi [k] on the b side (same order convention as x, y).
 *   transpose = 0: y = K x (x on the b side, y on the a side); 1: y = K^T x.
 *   x, y: [len, B].
 */
laplex_status laplex_matvec_phased(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                                   const void* sb, const int32_t* pb, const void* psi, int64_t k,
                                   const void* x, void* y, int64_t B, int transpose,
                                   laplex_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Gram operator z = K^T diag(D) K v (summary §2.2 "Operatori di Gram"; the
 * abstract lists a fast Gram operator), as two chained products through the
 * workspace.
 *   phi == NULL: unphased K; otherwise the phased K (psi used when sb != NULL).
 *   sb == NULL: symmetric (b = a): v, z [n, B], D [n] or NULL (D = 1).
 *   sb != NULL: v, z [k, B] on the b side, D [n] on the a side or NULL.
 */
laplex_status laplex_gram(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                          const void* sb, const int32_t* pb, const void* psi, int64_t k,
                          const void* D, const void* v, void* z, int64_t B,
                          laplex_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward pass of L = <g, K x>, K = K(a, a), w.r.t. x and the anchors
 * (differentiability in the anchors: summary §2.3 and §4.1):
 *   dx = K^T g = K g,
 *   da_i = -g_i sum_j sign(a_i - a_j) K_ij x_j - x_i sum_j sign(a_i - a_j) K_ij g_j,
 * with sign(0) = 0 for tied anchors.  x, g, dx, da: [n] (B = 1).
 */
laplex_status laplex_backward(const void* sorted, const int32_t* perm, int64_t n,
                              const void* x, const void* g, void* dx, void* da,
                              laplex_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward pass of the general product: L = <g, K x>, K_ij = exp(-|a_i - b_j|),
 * a in R^n, b in R^k, with respect to x and both anchor sets (learnable
 * anchors: summary §2.3):
 *   dx = K^T g,
 *   da_i = -g_i sum_j sign(a_i - b_j) K_ij x_j,
 *   db_j = -x_j sum_i sign(b_j - a_i) K_ij g_i,      sign(0) = 0.
 *   sa [n], pa [n]|NULL, sb [k], pb [k]|NULL: sorted anchors and perms as in
 *              laplex_matvec_general; g, da [n] follow pa, x, dx, db [k] follow pb.
 *   B = 1.  Workspace: laplex_workspace_size(LAPLEX_OP_BACKWARD_GENERAL, n, k, 1, ...).
 * n = 0 or k = 0: the outputs on the other side are zero.
 */
laplex_status laplex_backward_general(const void* sa, const int32_t* pa, int64_t n,
                                      const void* sb, const int32_t* pb, int64_t k,
                                      const void* x, const void* g, void* dx, void* da,
                                      void* db, laplex_dtype dtype, void* ws, size_t ws_bytes,
                                      void* stream);

/*
 * Backward pass of the phased product: L = <g, K x>,
 * K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j) (summary §2.1; anchors and phases
 * trainable, §2.3), with respect to x, the phases and the anchors:
 *   dx_j   = sum_i K_ij g_i,
 *   dphi_i = -g_i sum_j exp(-|a_i - b_j|) sin(phi_i - psi_j) x_j,
 *   dpsi_j =  x_j sum_i exp(-|a_i - b_j|) sin(phi_i - psi_j) g_i,
 *   da_i   = -g_i sum_j sign(a_i - b_j) K_ij x_j,
 *   db_j   = -x_j sum_i sign(b_j - a_i) K_ij g_i,        sign(0) = 0.
 *   sa [n], pa [n]|NULL, sb [k], pb [k]|NULL: sorted anchors and perms as in
 *              laplex_matvec_general; phi, g, dphi, da [n] follow pa; psi, x, dx,
 *              dpsi, db [k] follow pb.
 *   sb == NULL: symmetric case (b = a, psi = phi, k = n; k, pb, psi, dpsi, db
 *              ignored).  The anchors and phases are shared, so dphi and da
 *              receive the total gradients (both sides' terms); dx = K g.
 *   Any of dx, dphi, dpsi, da, db may be NULL: that output is not computed.
 *   B = 1.  Workspace: laplex_workspace_size(LAPLEX_OP_BACKWARD_PHASED, n, k, 1, ...).
 * n = 0 or k = 0: the outputs on the other side are zero.
 */
laplex_status laplex_backward_phased(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                                     const void* sb, const int32_t* pb, const void* psi, int64_t k,
                                     const void* x, const void* g, void* dx, void* dphi, void* dpsi,
                                     void* da, void* db, laplex_dtype dtype, void* ws,
                                     size_t ws_bytes, void* stream);

/*
 * Weighted Gram matrix M = A diag(D) A^T, A_ij = exp(-|a_i - b_j|) (summary
 * §2.2 "Operatori di Gram"), in O(n^2 + k log n): per a-point one-sided sums
 * over b and fp64 prefix sums of D, then
 *   M_ij = exp(a_i - a_j) (Lw_i + sum_{a_i < b <= a_j} D_b + Rw_j)   (a_i <= a_j).
 *   sa [n], pa [n]|NULL, sb [k], pb [k]|NULL: sorted anchors and perms.
 *   D [k]|NULL: weights on b (follow pb); NULL means 1.
 *   M [n, ldm] row-major, ldm >= n: rows and columns follow pa (sorted order
 *   when pa is NULL).  Every entry in the first n columns is written.
 *   Workspace: laplex_workspace_size(LAPLEX_OP_GRAM_MATRIX, n, k, 1, ...).
 */
laplex_status laplex_gram_matrix(const void* sa, const int32_t* pa, int64_t n, const void* sb,
                                 const int32_t* pb, int64_t k, const void* D, void* M, int64_t ldm,
                                 laplex_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Profiling hook (no counterpart in the paper): for the following calls on the
 * calling thread, record the CUDA events `before` and `after` (cudaEvent_t
 * passed as void*, created by the caller) on the call's stream immediately
 * before and after the call's dominant kernel: the tile-local scan of the
 * symmetric product and of the backward pass, the four digit passes of the
 * sort, the merged scan of the general product.  NULL, NULL switches it off.
 * Host-only bookkeeping; no synchronisation.  Returns LAPLEX_OK.
 */
laplex_status laplex_set_profile_events(void* before, void* after);

/*
 * Test hook for the bounded waits (no counterpart in the paper).  For the
 * following laplex_sort_anchors calls on the calling thread: `polls` bounds
 * every wait of the sort's digit passes for a bulk copy into shared memory
 * (0 restores the default, 2^20 polls), and a non-zero `force_expiry` leaves
 * the first copy of every block of a digit pass unissued, so that its wait
 * runs to the bound.  An expired wait sets LAPLEX_ETIMEOUT in the device
 * status, and the block lets its other copies land (bounded) and stops; the
 * outputs are then unspecified, and nothing is written outside them.  It
 * exists so that tests can check that an expired wait ends with an error
 * instead of hanging.  Host-only bookkeeping.  Returns LAPLEX_OK.
 */
laplex_status laplex_test_set_sort_wait(uint32_t polls, int force_expiry);

/*
 * Allocation-free symmetric product, y = K x (fp32, B = 1).  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate device
 * memory -- code running where cudaMalloc is unavailable or forbidden (inside
 * another library's allocator-free hot path, a real-time loop that must not
 * allocate, or a host that owns a fixed memory budget) -- and so cannot
 * provide the workspace laplex_matvec_sym needs.
 *   sorted [n], perm [n]|NULL, x [n], y [n]: as in laplex_matvec_sym (fp32, B = 1).
 *   stream: as elsewhere.
 * Scratch: a fixed array of 4 MiB + 4 KiB compiled into the library as a
 * __device__ variable (per tile its edge anchors and totals, then the carries
 * into it; per group of 2048 tiles its totals); every GPU that loads the
 * library holds it until the process exits.
 * It bounds n to 2^30 (2^18 tiles of 4096 anchors); larger n returns
 * LAPLEX_EINVAL with a message.  The call allocates and frees nothing.
 * The first call on each device looks up the array's device address (with that
 * device current), so make that first call before any stream capture.  A
 * device reset (cudaDeviceReset) gives the device a new context; the first
 * call after it looks the address up again and, likewise, belongs before any
 * stream capture.
 * Every call shares the one array per device and leaves its last contents
 * there; each call writes every scratch entry before reading it, so nothing
 * needs clearing, but calls that overlap on the GPU (several streams or host
 * threads on one device) race on it and must be serialised by the caller.
 * Errors: LAPLEX_EINVAL (sizes, NULL or misaligned pointers), LAPLEX_ECUDA
 * (set-up or launch failure); laplex_last_error() holds the message.
 */
laplex_status laplex_matvec_sym_noalloc(const float* sorted, const int32_t* perm, int64_t n,
                                        const float* x, float* y, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LAPLEX_H */
