// capi.cu -- the extern "C" boundary of liblaplex.so (declared in include/laplex.h).
//
// Host-side argument checks, workspace carving and dispatch to the kernel files.
// No call allocates, frees, synchronises (except laplex_get_device_status) or
// throws; host-detected errors return before anything is enqueued.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <type_traits>

#include "laplex.h"
#include "laplex_impl.h"

namespace {

thread_local char g_err[512] = "";

laplex_status fail(laplex_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

laplex_status ok() {
    g_err[0] = '\0';
    return LAPLEX_OK;
}

laplex_status cuda_fail(cudaError_t e, const char* where) {
    return fail(LAPLEX_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int64_t MAXN = (int64_t)1 << 31;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define REQ(cond, ...)                                      \
    do {                                                    \
        if (!(cond)) return fail(LAPLEX_EINVAL, __VA_ARGS__); \
    } while (0)

#define REQ_PTR(p, need)                                                              \
    do {                                                                              \
        if (need) {                                                                   \
            REQ((p) != nullptr, "%s is NULL", #p);                                    \
            REQ(aligned((p), 16), "%s is not 16-byte aligned", #p);                   \
        }                                                                             \
    } while (0)

laplex_status check_sizes(int64_t n, int64_t k, int64_t B) {
    REQ(n >= 0 && n < MAXN, "n = %lld out of range [0, 2^31)", (long long)n);
    REQ(k >= 0 && k < MAXN, "k = %lld out of range [0, 2^31)", (long long)k);
    REQ(B >= 1 && B < MAXN, "B = %lld must be >= 1", (long long)B);
    return LAPLEX_OK;
}

laplex_status check_dtype(laplex_dtype dt) {
    REQ(dt == LAPLEX_F32 || dt == LAPLEX_F64, "dtype %d is not LAPLEX_F32 or LAPLEX_F64", (int)dt);
    return LAPLEX_OK;
}

// the sort carrying a value: fp32 in the digit passes; fp64 as the sort, then
// inv (n int32) and the permutation of x by inv
size_t sort_carry_body(int64_t n, int f64) {
    if (!f64) return lx::sort_carry_ws_bytes(n);
    return lx::Carve::need((size_t)n, 4) + std::max(lx::sort_ws_bytes(n, 1), lx::permute_ws_bytes(n, 8));
}

size_t body_bytes(laplex_op op, int64_t n, int64_t k, int64_t B, int f64) {
    switch (op) {
        case LAPLEX_OP_SORT: return lx::sort_ws_bytes(n, f64);
        case LAPLEX_OP_MATVEC_SYM: return lx::sym_ws_bytes(n, B, false, f64);
        case LAPLEX_OP_MATVEC_GENERAL: {
            size_t a = lx::gen_ws_bytes(n, k, B, false, f64), b = lx::gen_ws_bytes(k, n, B, false, f64);
            return a > b ? a : b;
        }
        case LAPLEX_OP_MATVEC_PHASED: {
            size_t s = lx::sym_ws_bytes(n, B, true, f64);
            size_t a = lx::gen_ws_bytes(n, k, B, true, f64), b = lx::gen_ws_bytes(k, n, B, true, f64);
            size_t m = a > b ? a : b;
            return s > m ? s : m;
        }
        case LAPLEX_OP_GRAM: {
            // intermediate u on the a side + the larger of the two passes (phased covers unphased)
            const size_t es = f64 ? 8 : 4;
            size_t u = lx::Carve::need((size_t)(n * B), es);
            size_t s = lx::sym_ws_bytes(n, B, true, f64);
            size_t a = lx::gen_ws_bytes(n, k, B, true, f64), b = lx::gen_ws_bytes(k, n, B, true, f64);
            size_t m = a > b ? a : b;
            m = m > s ? m : s;
            return u + m;
        }
        case LAPLEX_OP_BACKWARD: return lx::bwd_ws_bytes(n, f64);
        case LAPLEX_OP_BACKWARD_GENERAL: {
            // K^T g first (the general product's workspace), then the two signed
            // sums one after the other (each over one side)
            const size_t g = std::max(lx::gen_ws_bytes(n, k, 1, false, f64), lx::gen_ws_bytes(k, n, 1, false, f64));
            const size_t sg = std::max(lx::sgen_ws_bytes(n, f64), lx::sgen_ws_bytes(k, f64));
            return std::max(g, sg);
        }
        case LAPLEX_OP_GRAM_MATRIX: return lx::grammat_ws_bytes(n, k, f64);
        case LAPLEX_OP_BACKWARD_PHASED: return std::max(lx::pbwd_ws_bytes(n, f64), lx::pbwd_ws_bytes(k, f64));
        case LAPLEX_OP_PERMUTE: return lx::permute_ws_bytes(n, f64 ? 8 : 4);
        case LAPLEX_OP_SORT_CARRY: return sort_carry_body(n, f64);
        case LAPLEX_OP_MATVEC_SYM_UNSORTED: {
            // xs and y' in sorted order, then the larger of the sort, the product and the permutation
            const size_t es = f64 ? 8 : 4;
            return 2 * lx::Carve::need((size_t)n, es) +
                   std::max(sort_carry_body(n, f64),
                            std::max(lx::permute_ws_bytes(n, (int)es), lx::stream_ws_bytes(n, f64)));
        }
        case LAPLEX_OP_MATVEC_SYM_PLANNED: {
            // x and y in sorted order, then the larger of the permutation and the product
            const size_t es = f64 ? 8 : 4;
            return 2 * lx::Carve::need((size_t)n, es) +
                   std::max(lx::permute_ws_bytes(n, (int)es), lx::stream_ws_bytes(n, f64));
        }
    }
    return 0;
}

laplex_status check_ws(laplex_op op, int64_t n, int64_t k, int64_t B, laplex_dtype dt, void* ws,
                       size_t ws_bytes) {
    REQ(ws != nullptr, "workspace is NULL");
    REQ(aligned(ws, 256), "workspace is not 256-byte aligned");
    const size_t need = lx::HEADER_BYTES + body_bytes(op, n, k, B, dt == LAPLEX_F64);
    if (ws_bytes < need)
        return fail(LAPLEX_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    return LAPLEX_OK;
}

void* ws_body(void* ws) { return static_cast<char*>(ws) + lx::HEADER_BYTES; }
uint32_t* ws_status(void* ws) { return static_cast<uint32_t*>(ws); }

}  // namespace

namespace {
thread_local lx::ProfileEvents g_prof = {nullptr, nullptr};
}

const lx::ProfileEvents& lx::profile_events() { return g_prof; }

void lx::set_last_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

extern "C" {

int laplex_version(void) { return 10100; }

int laplex_build_flags(void) {
#ifdef LX_ACCURATE_EXP
    return LAPLEX_BUILD_ACCURATE_EXP;
#else
    return 0;
#endif
}

const char* laplex_status_string(laplex_status s) {
    switch (s) {
        case LAPLEX_OK: return "LAPLEX_OK";
        case LAPLEX_EINVAL: return "LAPLEX_EINVAL";
        case LAPLEX_ENONFINITE: return "LAPLEX_ENONFINITE";
        case LAPLEX_EWORKSPACE: return "LAPLEX_EWORKSPACE";
        case LAPLEX_ECUDA: return "LAPLEX_ECUDA";
        case LAPLEX_ETIMEOUT: return "LAPLEX_ETIMEOUT";
    }
    return "LAPLEX_UNKNOWN";
}

const char* laplex_last_error(void) { return g_err; }

laplex_status laplex_set_profile_events(void* before, void* after) {
    g_prof.before = (cudaEvent_t)before;
    g_prof.after = (cudaEvent_t)after;
    return ok();
}

laplex_status laplex_permute(const void* src, const int32_t* idx, int64_t n, laplex_dtype dt, void* dst,
                             void* ws, size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(src, n > 0);
    REQ_PTR(idx, n > 0);
    REQ_PTR(dst, n > 0);
    if ((st = check_ws(LAPLEX_OP_PERMUTE, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    cudaError_t e = dt == LAPLEX_F32
                        ? lx::permute_run<int32_t>((const int32_t*)src, idx, n, (int32_t*)dst, ws_body(ws), body,
                                                   ws_status(ws), (cudaStream_t)stream)
                        : lx::permute_run<int64_t>((const int64_t*)src, idx, n, (int64_t*)dst, ws_body(ws), body,
                                                   ws_status(ws), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_permute");
    return ok();
}

laplex_status laplex_invert_perm(const int32_t* perm, int64_t n, int32_t* inv, void* ws, size_t ws_bytes,
                                 void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    REQ_PTR(perm, n > 0);
    REQ_PTR(inv, n > 0);
    if ((st = check_ws(LAPLEX_OP_PERMUTE, n, 0, 1, LAPLEX_F32, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e = lx::permute_run<int32_t>(nullptr, perm, n, inv, ws_body(ws), ws_bytes - lx::HEADER_BYTES,
                                             ws_status(ws), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_invert_perm");
    return ok();
}

laplex_status laplex_test_set_sort_wait(uint32_t polls, int force_expiry) {
    lx::set_sort_wait(polls, force_expiry);
    return ok();
}

laplex_status laplex_workspace_size(laplex_op op, int64_t n, int64_t k, int64_t B, laplex_dtype dt,
                                    size_t* bytes) {
    REQ(bytes != nullptr, "bytes is NULL");
    laplex_status st = check_sizes(n, k, B);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ(op >= LAPLEX_OP_SORT && op <= LAPLEX_OP_MATVEC_SYM_UNSORTED, "unknown op %d", (int)op);
    *bytes = lx::HEADER_BYTES + body_bytes(op, n, k, B, dt == LAPLEX_F64);
    return ok();
}

laplex_status laplex_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    REQ(ws != nullptr && ws_bytes >= lx::HEADER_BYTES, "workspace NULL or below the header size");
    cudaError_t e = cudaMemsetAsync(ws, 0, lx::HEADER_BYTES, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_workspace_init");
    return ok();
}

laplex_status laplex_get_device_status(void* ws, void* stream) {
    REQ(ws != nullptr, "workspace is NULL");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_get_device_status");
    if (word != 0) {
        e = cudaMemsetAsync(ws, 0, sizeof(word), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "laplex_get_device_status (clear)");
    }
    if (word & lx::ST_NONFINITE) return fail(LAPLEX_ENONFINITE, "a non-finite anchor was found");
    if (word & lx::ST_TIMEOUT) return fail(LAPLEX_ETIMEOUT, "a bounded inter-block wait expired");
    return ok();
}

laplex_status laplex_sort_anchors(const void* a, int64_t n, laplex_dtype dt, void* sorted,
                                  int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(a, n > 0);
    REQ_PTR(sorted, n > 0);
    REQ_PTR(perm, n > 0);
    if ((st = check_ws(LAPLEX_OP_SORT, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e;
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    if (dt == LAPLEX_F32)
        e = lx::sort_run<float>((const float*)a, n, (float*)sorted, perm, ws_body(ws), body,
                                ws_status(ws), (cudaStream_t)stream);
    else
        e = lx::sort_run<double>((const double*)a, n, (double*)sorted, perm, ws_body(ws), body,
                                 ws_status(ws), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_sort_anchors");
    return ok();
}

}  // extern "C"

template <typename T>
static cudaError_t run_sym(const void* sorted, const int32_t* perm, int64_t n, const void* x,
                           void* y, int64_t B, const void* phi, const void* D, void* ws,
                           size_t ws_bytes, cudaStream_t st, bool phased) {
    lx::SymArgs<T> A;
    A.s = (const T*)sorted;
    A.n = n;
    A.x = (const T*)x;
    A.pin = perm;
    A.ldx = B;
    A.y = (T*)y;
    A.pout = perm;
    A.ldy = B;
    A.phi = (const T*)phi;
    A.D = (const T*)D;
    A.paux = perm;
    A.col0 = 0;
    A.ncol = 1;
    A.status = ws_status(ws);
    return lx::sym_run<T>(A, B, phased, ws_body(ws), ws_bytes - lx::HEADER_BYTES, st);
}

extern "C" {

laplex_status laplex_matvec_sym(const void* sorted, const int32_t* perm, int64_t n, const void* x,
                                void* y, int64_t B, laplex_dtype dt, void* ws, size_t ws_bytes,
                                void* stream) {
    laplex_status st = check_sizes(n, 0, B);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sorted, n > 0);
    REQ_PTR(x, n > 0);
    REQ_PTR(y, n > 0);
    if (perm) REQ_PTR(perm, n > 0);
    if ((st = check_ws(LAPLEX_OP_MATVEC_SYM, n, 0, B, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e = dt == LAPLEX_F32
                        ? run_sym<float>(sorted, perm, n, x, y, B, nullptr, nullptr, ws, ws_bytes,
                                         (cudaStream_t)stream, false)
                        : run_sym<double>(sorted, perm, n, x, y, B, nullptr, nullptr, ws, ws_bytes,
                                          (cudaStream_t)stream, false);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_matvec_sym");
    return ok();
}

}  // extern "C"

// xs[r] = x[perm[r]] with the sort (see sort_carry_body for the layout)
static cudaError_t run_sort_carry(const void* a, const void* x, int64_t n, bool f64, void* sorted, int32_t* perm,
                                  void* xs, void* body, size_t body_bytes, uint32_t* status, cudaStream_t st) {
    if (!f64)
        return lx::sort_carry_run((const float*)a, (const float*)x, n, (float*)sorted, perm, (float*)xs, body,
                                  body_bytes, status, st);
    lx::Carve cv(body, body_bytes);
    int32_t* inv = cv.take<int32_t>(n);
    if (!cv.ok) return cudaErrorInvalidValue;
    void* rest = cv.base + cv.off;
    const size_t rest_bytes = cv.cap - cv.off;
    cudaError_t e = lx::sort_run<double>((const double*)a, n, (double*)sorted, perm, rest, rest_bytes, status, st);
    if (e == cudaSuccess) e = lx::permute_run<int32_t>(nullptr, perm, n, inv, rest, rest_bytes, status, st);
    if (e == cudaSuccess)
        e = lx::permute_run<int64_t>((const int64_t*)x, inv, n, (int64_t*)xs, rest, rest_bytes, status, st);
    return e;
}

extern "C" laplex_status laplex_sort_anchors_carry(const void* a, const void* x, int64_t n, laplex_dtype dt,
                                                   void* sorted, int32_t* perm, void* xs, void* ws, size_t ws_bytes,
                                                   void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(a, n > 0);
    REQ_PTR(x, n > 0);
    REQ_PTR(sorted, n > 0);
    REQ_PTR(perm, n > 0);
    REQ_PTR(xs, n > 0);
    if ((st = check_ws(LAPLEX_OP_SORT_CARRY, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e = run_sort_carry(a, x, n, dt == LAPLEX_F64, sorted, perm, xs, ws_body(ws),
                                   ws_bytes - lx::HEADER_BYTES, ws_status(ws), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_sort_anchors_carry");
    return ok();
}

template <typename T>
static cudaError_t run_sym_unsorted(const void* a, const void* x, int64_t n, void* y, void* sorted, int32_t* perm,
                                    void* ws, size_t ws_bytes, cudaStream_t st) {
    using V = typename std::conditional<sizeof(T) == 8, int64_t, int32_t>::type;
    lx::Carve cv(ws_body(ws), ws_bytes - lx::HEADER_BYTES);
    T* xs = cv.take<T>(n);
    T* ys = cv.take<T>(n);
    if (!cv.ok) return cudaErrorInvalidValue;
    void* rest = cv.base + cv.off;
    const size_t rest_bytes = cv.cap - cv.off;
    cudaError_t e = run_sort_carry(a, x, n, sizeof(T) == 8, sorted, perm, xs, rest, rest_bytes, ws_status(ws), st);
    if (e == cudaSuccess)
        e = lx::stream_run<T>((const T*)sorted, xs, ys, nullptr, n, rest, rest_bytes, ws_status(ws), st);
    if (e == cudaSuccess) e = lx::permute_run<V>((const V*)ys, perm, n, (V*)y, rest, rest_bytes, ws_status(ws), st);
    return e;
}

extern "C" laplex_status laplex_matvec_sym_unsorted(const void* a, const void* x, int64_t n, laplex_dtype dt,
                                                    void* y, void* sorted, int32_t* perm, void* ws, size_t ws_bytes,
                                                    void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(a, n > 0);
    REQ_PTR(x, n > 0);
    REQ_PTR(y, n > 0);
    REQ_PTR(sorted, n > 0);
    REQ_PTR(perm, n > 0);
    if ((st = check_ws(LAPLEX_OP_MATVEC_SYM_UNSORTED, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e = dt == LAPLEX_F32
                        ? run_sym_unsorted<float>(a, x, n, y, sorted, perm, ws, ws_bytes, (cudaStream_t)stream)
                        : run_sym_unsorted<double>(a, x, n, y, sorted, perm, ws, ws_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_matvec_sym_unsorted");
    return ok();
}

template <typename T>
static cudaError_t run_sym_planned(const void* sorted, const int32_t* perm, const int32_t* inv, int64_t n,
                                   const void* x, void* y, void* ws, size_t ws_bytes, cudaStream_t st) {
    using V = typename std::conditional<sizeof(T) == 8, int64_t, int32_t>::type;
    lx::Carve cv(ws_body(ws), ws_bytes - lx::HEADER_BYTES);
    T* xs = cv.take<T>(n);
    T* ys = cv.take<T>(n);
    if (!cv.ok) return cudaErrorInvalidValue;
    void* rest = cv.base + cv.off;
    const size_t rest_bytes = cv.cap - cv.off;
    cudaError_t e = lx::permute_run<V>((const V*)x, inv, n, (V*)xs, rest, rest_bytes, ws_status(ws), st);
    if (e == cudaSuccess)
        e = lx::stream_run<T>((const T*)sorted, xs, ys, nullptr, n, rest, rest_bytes, ws_status(ws), st);
    if (e == cudaSuccess) e = lx::permute_run<V>((const V*)ys, perm, n, (V*)y, rest, rest_bytes, ws_status(ws), st);
    return e;
}

extern "C" laplex_status laplex_matvec_sym_planned(const void* sorted, const int32_t* perm, const int32_t* inv,
                                                   int64_t n, const void* x, void* y, laplex_dtype dt, void* ws,
                                                   size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sorted, n > 0);
    REQ_PTR(perm, n > 0);
    REQ_PTR(inv, n > 0);
    REQ_PTR(x, n > 0);
    REQ_PTR(y, n > 0);
    if ((st = check_ws(LAPLEX_OP_MATVEC_SYM_PLANNED, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaError_t e = dt == LAPLEX_F32
                        ? run_sym_planned<float>(sorted, perm, inv, n, x, y, ws, ws_bytes, (cudaStream_t)stream)
                        : run_sym_planned<double>(sorted, perm, inv, n, x, y, ws, ws_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_matvec_sym_planned");
    return ok();
}

template <typename T>
static cudaError_t run_gen(const void* sa, const int32_t* pa, int64_t n, const void* sb,
                           const int32_t* pb, int64_t k, const void* x, void* y, int64_t B,
                           int transpose, const void* phi, const void* psi, const void* D,
                           const int32_t* pD, void* ws, size_t ws_bytes, cudaStream_t st,
                           bool phased) {
    // y lives on the "out" side, x on the "in" side; transpose swaps the sides.
    lx::GenArgs<T> A;
    const bool tr = transpose != 0;
    A.sa = (const T*)(tr ? sb : sa);
    A.pa = tr ? pb : pa;
    A.n = tr ? k : n;
    A.sb = (const T*)(tr ? sa : sb);
    A.pb = tr ? pa : pb;
    A.k = tr ? n : k;
    A.x = (const T*)x;
    A.ldx = B;
    A.y = (T*)y;
    A.ldy = B;
    A.pout = A.pa;
    A.pin = A.pb;
    A.phi = (const T*)(tr ? psi : phi);
    A.pphi = A.pa;
    A.psi = (const T*)(tr ? phi : psi);
    A.ppsi = A.pb;
    A.D = (const T*)D;
    A.pD = pD;
    A.col0 = 0;
    A.ncol = 1;
    A.status = ws_status(ws);
    return lx::gen_run<T>(A, B, phased, ws_body(ws), ws_bytes - lx::HEADER_BYTES, st);
}

extern "C" {

laplex_status laplex_matvec_general(const void* sa, const int32_t* pa, int64_t n, const void* sb,
                                    const int32_t* pb, int64_t k, const void* x, void* y, int64_t B,
                                    int transpose, laplex_dtype dt, void* ws, size_t ws_bytes,
                                    void* stream) {
    laplex_status st = check_sizes(n, k, B);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    const int64_t nin = transpose ? n : k, nout = transpose ? k : n;
    REQ_PTR(sa, n > 0);
    REQ_PTR(sb, k > 0);
    REQ_PTR(x, nin > 0);
    REQ_PTR(y, nout > 0);
    if (pa) REQ_PTR(pa, n > 0);
    if (pb) REQ_PTR(pb, k > 0);
    if ((st = check_ws(LAPLEX_OP_MATVEC_GENERAL, n, k, B, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (nout == 0) return ok();
    cudaError_t e = dt == LAPLEX_F32
                        ? run_gen<float>(sa, pa, n, sb, pb, k, x, y, B, transpose, nullptr, nullptr,
                                         nullptr, nullptr, ws, ws_bytes, (cudaStream_t)stream, false)
                        : run_gen<double>(sa, pa, n, sb, pb, k, x, y, B, transpose, nullptr,
                                          nullptr, nullptr, nullptr, ws, ws_bytes,
                                          (cudaStream_t)stream, false);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_matvec_general");
    return ok();
}

laplex_status laplex_matvec_phased(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                                   const void* sb, const int32_t* pb, const void* psi, int64_t k,
                                   const void* x, void* y, int64_t B, int transpose,
                                   laplex_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    const bool symm = sb == nullptr;
    if (symm) k = 0;
    laplex_status st = check_sizes(n, k, B);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sa, n > 0);
    REQ_PTR(phi, n > 0);
    if (pa) REQ_PTR(pa, n > 0);
    if (!symm) {
        REQ_PTR(psi, k > 0);
        if (pb) REQ_PTR(pb, k > 0);
    }
    const int64_t nin = symm ? n : (transpose ? n : k), nout = symm ? n : (transpose ? k : n);
    REQ_PTR(x, nin > 0);
    REQ_PTR(y, nout > 0);
    if ((st = check_ws(LAPLEX_OP_MATVEC_PHASED, n, k, B, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (nout == 0) return ok();
    cudaError_t e;
    cudaStream_t s = (cudaStream_t)stream;
    if (symm) {
        e = dt == LAPLEX_F32 ? run_sym<float>(sa, pa, n, x, y, B, phi, nullptr, ws, ws_bytes, s, true)
                             : run_sym<double>(sa, pa, n, x, y, B, phi, nullptr, ws, ws_bytes, s, true);
    } else {
        e = dt == LAPLEX_F32
                ? run_gen<float>(sa, pa, n, sb, pb, k, x, y, B, transpose, phi, psi, nullptr,
                                 nullptr, ws, ws_bytes, s, true)
                : run_gen<double>(sa, pa, n, sb, pb, k, x, y, B, transpose, phi, psi, nullptr,
                                  nullptr, ws, ws_bytes, s, true);
    }
    if (e != cudaSuccess) return cuda_fail(e, "laplex_matvec_phased");
    return ok();
}

laplex_status laplex_gram(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                          const void* sb, const int32_t* pb, const void* psi, int64_t k,
                          const void* D, const void* v, void* z, int64_t B, laplex_dtype dt,
                          void* ws, size_t ws_bytes, void* stream) {
    const bool symm = sb == nullptr;
    const bool phased = phi != nullptr;
    if (symm) k = 0;
    laplex_status st = check_sizes(n, k, B);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    const int64_t nv = symm ? n : k;
    REQ_PTR(sa, n > 0);
    if (pa) REQ_PTR(pa, n > 0);
    if (phased) REQ_PTR(phi, n > 0);
    if (!symm) {
        REQ_PTR(sb, k > 0);
        if (pb) REQ_PTR(pb, k > 0);
        if (phased) REQ_PTR(psi, k > 0);
    }
    if (D) REQ_PTR(D, n > 0);
    REQ_PTR(v, nv > 0);
    REQ_PTR(z, nv > 0);
    if ((st = check_ws(LAPLEX_OP_GRAM, n, k, B, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (nv == 0) return ok();
    cudaStream_t s = (cudaStream_t)stream;
    const size_t es = dt == LAPLEX_F64 ? 8 : 4;
    // u = K v on the a side, kept in sorted-a order in the workspace.
    char* body = static_cast<char*>(ws_body(ws));
    const size_t ubytes = lx::Carve::need((size_t)(n * B), es);
    void* u = body;
    // a sub-workspace that starts after u but keeps the header of ws for the status word
    const size_t rest = ws_bytes - lx::HEADER_BYTES - ubytes;
    cudaError_t e = cudaSuccess;
    auto pass = [&](auto tag) -> cudaError_t {
        using T = decltype(tag);
        if (symm) {
            lx::SymArgs<T> A;
            A.s = (const T*)sa; A.n = n; A.status = ws_status(ws); A.col0 = 0; A.ncol = 1;
            A.phi = (const T*)phi; A.paux = pa;
            // pass 1: u = K v (v in caller order, u in sorted order)
            A.x = (const T*)v; A.pin = pa; A.ldx = B; A.y = (T*)u; A.pout = nullptr; A.ldy = B;
            A.D = nullptr;
            cudaError_t r = lx::sym_run<T>(A, B, phased, body + ubytes, rest, s);
            if (r != cudaSuccess) return r;
            // pass 2: z = K (D u)
            A.x = (const T*)u; A.pin = nullptr; A.y = (T*)z; A.pout = pa; A.D = (const T*)D;
            return lx::sym_run<T>(A, B, phased, body + ubytes, rest, s);
        } else {
            // pass 1: u = K v, v on the b side (caller order), u on the a side (sorted order)
            lx::GenArgs<T> A;
            A.sa = (const T*)sa; A.pa = pa; A.n = n; A.sb = (const T*)sb; A.pb = pb; A.k = k;
            A.x = (const T*)v; A.ldx = B; A.pin = pb; A.y = (T*)u; A.ldy = B; A.pout = nullptr;
            A.phi = (const T*)phi; A.pphi = pa; A.psi = (const T*)psi; A.ppsi = pb;
            A.D = nullptr; A.pD = nullptr; A.col0 = 0; A.ncol = 1; A.status = ws_status(ws);
            cudaError_t r = lx::gen_run<T>(A, B, phased, body + ubytes, rest, s);
            if (r != cudaSuccess) return r;
            // pass 2: z = K^T (D u): out side b, in side a (u sorted, D caller order via pa)
            lx::GenArgs<T> Bq;
            Bq.sa = (const T*)sb; Bq.pa = pb; Bq.n = k; Bq.sb = (const T*)sa; Bq.pb = pa; Bq.k = n;
            Bq.x = (const T*)u; Bq.ldx = B; Bq.pin = nullptr; Bq.y = (T*)z; Bq.ldy = B; Bq.pout = pb;
            Bq.phi = (const T*)psi; Bq.pphi = pb; Bq.psi = (const T*)phi; Bq.ppsi = pa;
            Bq.D = (const T*)D; Bq.pD = pa; Bq.col0 = 0; Bq.ncol = 1; Bq.status = ws_status(ws);
            return lx::gen_run<T>(Bq, B, phased, body + ubytes, rest, s);
        }
    };
    e = dt == LAPLEX_F32 ? pass(float()) : pass(double());
    if (e != cudaSuccess) return cuda_fail(e, "laplex_gram");
    return ok();
}

laplex_status laplex_backward(const void* sorted, const int32_t* perm, int64_t n, const void* x,
                              const void* g, void* dx, void* da, laplex_dtype dt, void* ws,
                              size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, 0, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sorted, n > 0);
    REQ_PTR(x, n > 0);
    REQ_PTR(g, n > 0);
    REQ_PTR(dx, n > 0);
    REQ_PTR(da, n > 0);
    if (perm) REQ_PTR(perm, n > 0);
    if ((st = check_ws(LAPLEX_OP_BACKWARD, n, 0, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    cudaStream_t s = (cudaStream_t)stream;
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    cudaError_t e =
        dt == LAPLEX_F32
            ? lx::bwd_run<float>((const float*)sorted, perm, n, (const float*)x, (const float*)g,
                                 (float*)dx, (float*)da, ws_body(ws), body, ws_status(ws), s)
            : lx::bwd_run<double>((const double*)sorted, perm, n, (const double*)x,
                                  (const double*)g, (double*)dx, (double*)da, ws_body(ws), body,
                                  ws_status(ws), s);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_backward");
    return ok();
}

laplex_status laplex_backward_general(const void* sa, const int32_t* pa, int64_t n, const void* sb,
                                      const int32_t* pb, int64_t k, const void* x, const void* g,
                                      void* dx, void* da, void* db, laplex_dtype dt, void* ws,
                                      size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, k, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sa, n > 0);
    REQ_PTR(sb, k > 0);
    REQ_PTR(g, n > 0);
    REQ_PTR(da, n > 0);
    REQ_PTR(x, k > 0);
    REQ_PTR(dx, k > 0);
    REQ_PTR(db, k > 0);
    if (pa) REQ_PTR(pa, n > 0);
    if (pb) REQ_PTR(pb, k > 0);
    if ((st = check_ws(LAPLEX_OP_BACKWARD_GENERAL, n, k, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0 && k == 0) return ok();
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    // dx = K^T g (the transposed general product; zero when n = 0)
    if (k > 0) {
        e = dt == LAPLEX_F32
                ? run_gen<float>(sa, pa, n, sb, pb, k, g, dx, 1, 1, nullptr, nullptr, nullptr, nullptr,
                                 ws, ws_bytes, s, false)
                : run_gen<double>(sa, pa, n, sb, pb, k, g, dx, 1, 1, nullptr, nullptr, nullptr, nullptr,
                                  ws, ws_bytes, s, false);
        if (e != cudaSuccess) return cuda_fail(e, "laplex_backward_general (K^T g)");
    }
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    e = dt == LAPLEX_F32
            ? lx::sgen_run<float>((const float*)sa, pa, n, (const float*)sb, pb, k, (const float*)x,
                                  (const float*)g, (float*)da, (float*)db, ws_body(ws), body, s)
            : lx::sgen_run<double>((const double*)sa, pa, n, (const double*)sb, pb, k,
                                   (const double*)x, (const double*)g, (double*)da, (double*)db,
                                   ws_body(ws), body, s);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_backward_general (signed sums)");
    return ok();
}

laplex_status laplex_backward_phased(const void* sa, const int32_t* pa, const void* phi, int64_t n,
                                     const void* sb, const int32_t* pb, const void* psi, int64_t k,
                                     const void* x, const void* g, void* dx, void* dphi, void* dpsi,
                                     void* da, void* db, laplex_dtype dt, void* ws, size_t ws_bytes,
                                     void* stream) {
    const bool sym = sb == nullptr;
    if (sym) {
        k = n;
        pb = nullptr;
        psi = nullptr;
        dpsi = nullptr;
        db = nullptr;
    }
    laplex_status st = check_sizes(n, k, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ_PTR(sa, n > 0);
    REQ_PTR(phi, n > 0);
    REQ_PTR(g, n > 0);
    REQ_PTR(x, k > 0);
    if (!sym) {
        REQ_PTR(sb, k > 0);
        REQ_PTR(psi, k > 0);
    }
    if (pa) REQ_PTR(pa, n > 0);
    if (pb) REQ_PTR(pb, k > 0);
    if (dphi) REQ_PTR(dphi, n > 0);
    if (da) REQ_PTR(da, n > 0);
    if (dx) REQ_PTR(dx, k > 0);
    if (dpsi) REQ_PTR(dpsi, k > 0);
    if (db) REQ_PTR(db, k > 0);
    if ((st = check_ws(LAPLEX_OP_BACKWARD_PHASED, n, k, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0 && k == 0) return ok();
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    cudaStream_t s = (cudaStream_t)stream;
    const cudaError_t e =
        dt == LAPLEX_F32
            ? lx::pbwd_run<float>((const float*)sa, pa, (const float*)phi, n, (const float*)sb, pb,
                                  (const float*)psi, k, (const float*)x, (const float*)g, (float*)dx,
                                  (float*)dphi, (float*)dpsi, (float*)da, (float*)db, ws_body(ws), body, s)
            : lx::pbwd_run<double>((const double*)sa, pa, (const double*)phi, n, (const double*)sb, pb,
                                   (const double*)psi, k, (const double*)x, (const double*)g, (double*)dx,
                                   (double*)dphi, (double*)dpsi, (double*)da, (double*)db, ws_body(ws), body,
                                   s);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_backward_phased");
    return ok();
}

laplex_status laplex_gram_matrix(const void* sa, const int32_t* pa, int64_t n, const void* sb,
                                 const int32_t* pb, int64_t k, const void* D, void* M, int64_t ldm,
                                 laplex_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    laplex_status st = check_sizes(n, k, 1);
    if (st != LAPLEX_OK) return st;
    if ((st = check_dtype(dt)) != LAPLEX_OK) return st;
    REQ(ldm >= n, "ldm = %lld below n = %lld", (long long)ldm, (long long)n);
    REQ_PTR(sa, n > 0);
    REQ_PTR(sb, k > 0);
    REQ_PTR(M, n > 0);
    if (pa) REQ_PTR(pa, n > 0);
    if (pb) REQ_PTR(pb, k > 0);
    if (D) REQ_PTR(D, k > 0);
    if ((st = check_ws(LAPLEX_OP_GRAM_MATRIX, n, k, 1, dt, ws, ws_bytes)) != LAPLEX_OK) return st;
    if (n == 0) return ok();
    const size_t body = ws_bytes - lx::HEADER_BYTES;
    cudaStream_t s = (cudaStream_t)stream;
    const cudaError_t e =
        dt == LAPLEX_F32
            ? lx::grammat_run<float>((const float*)sa, pa, n, (const float*)sb, pb, k, (const float*)D,
                                     (float*)M, ldm, ws_body(ws), body, s)
            : lx::grammat_run<double>((const double*)sa, pa, n, (const double*)sb, pb, k, (const double*)D,
                                      (double*)M, ldm, ws_body(ws), body, s);
    if (e != cudaSuccess) return cuda_fail(e, "laplex_gram_matrix");
    return ok();
}

}  // extern "C"
