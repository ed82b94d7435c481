// signed.cu -- signed general sums and the general-case backward pass.
//
// For anchors a (n of them) and b (k of them) and values v on b,
//     S(a <- b, v)_i = sum_j sign(a_i - b_j) exp(-|a_i - b_j|) v_j,   sign(0) = 0,
// the derivative of the kernel exp(-|a_i - b_j|) in the anchors ("LAPLEX - La
// FFT dei Nuclei di Laplace Apprendibili", technical summary §2.3: learnable
// anchors).  The backward pass of L = <g, K x> with K_ij = exp(-|a_i - b_j|) is
//     dx = K^T g,   da_i = -g_i S(a <- b, x)_i,   db_j = -x_j S(b <- a, g)_j.
//
// S splits into the b strictly below a_i minus the b strictly above it.  Both
// are read off two one-sided scans over the sorted b,
//     F_m = sum_{l <= m} exp(b_l - b_m) v_l,   G_m = sum_{l >= m} exp(b_m - b_l) v_l,
// (the wait-free scheme of threepass.cuh, policy OneSidedTP), at
// lb = #{b < a_i} and ub = #{b <= a_i}:
//     S_i = F_{lb-1} exp(b_{lb-1} - a_i) - G_{ub} exp(a_i - b_{ub})
// (one exp of an anchor gap each; a k_signed_query thread per a_i finds lb, ub
// by binary search).
#include <algorithm>

#include "laplex_impl.h"
#include "threepass.cuh"

namespace lx {

constexpr int OS_NT = 256;

// Policy of threepass.cuh: one channel, the values gathered through perm, the
// prefix F and the suffix G written (sorted order) instead of L + U - v.
template <typename T_, int E_>
struct OneSidedTP {
    using T = T_;
    static constexpr int C = 1, CT = 0, E = E_, NT = OS_NT;
    static constexpr int H = sizeof(T_) == 4 ? 192 : 0;  // as the symmetric products
    int64_t n;
    const T* s;
    const int32_t* perm;
    const T* v;          // NULL: every value 1
    T* F;
    T* G;
    struct Aux {};
    __device__ __forceinline__ void load(int64_t r0, T (&sv)[E], T (&vv)[E][C], Aux&) const {
        constexpr int VN = V16<T>::N;
        const bool full = r0 + E <= n;
        if (full) {
#pragma unroll
            for (int i = 0; i < E; i += VN) ld16_stream<T>(s + r0 + i, &sv[i]);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) sv[i] = s[min(r0 + i, n - 1)];
        }
        if (v == nullptr) {
#pragma unroll
            for (int i = 0; i < E; ++i) vv[i][0] = r0 + i < n ? T(1) : T(0);
        } else if (full && perm == nullptr) {
            T t[E];
#pragma unroll
            for (int i = 0; i < E; i += VN) ld16_stream<T>(v + r0 + i, &t[i]);
#pragma unroll
            for (int i = 0; i < E; ++i) vv[i][0] = t[i];
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const int64_t r = r0 + i;
                vv[i][0] = r < n ? v[perm ? (int64_t)perm[r] : r] : T(0);
            }
        }
    }
    __device__ __forceinline__ void load1(int64_t j, T& sj, T (&vj)[C]) const {
        sj = s[j];
        vj[0] = v == nullptr ? T(1) : v[perm ? (int64_t)perm[j] : j];
    }
    __device__ __forceinline__ void finish(int64_t r0, const T (&sv)[E], const T (&vv)[E][C],
                                           T (&dl)[E], T eprev, const T (&Lp)[C], T enext,
                                           const T (&Un)[C], Aux&) const {
        constexpr int VN = V16<T>::N;
        T fo[E], go[E];
        T L = Lp[0];
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const T d = i == 0 ? dexp<T>(eprev - sv[0]) : dl[i];
            L = dfma<T>(d, L, vv[i][0]);
            fo[i] = L;
        }
        T U = Un[0];
#pragma unroll
        for (int i = E - 1; i >= 0; --i) {
            const T d = i == E - 1 ? dexp<T>(sv[E - 1] - enext) : dl[i + 1];
            U = dfma<T>(d, U, vv[i][0]);
            go[i] = U;
        }
        if (r0 + E <= n) {
#pragma unroll
            for (int i = 0; i < E; i += VN) {
                st16<T>(F + r0 + i, &fo[i]);
                st16<T>(G + r0 + i, &go[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i)
                if (r0 + i < n) {
                    F[r0 + i] = fo[i];
                    G[r0 + i] = go[i];
                }
        }
    }
};

static constexpr int os_E(int es) { return es == 4 ? 12 : 6; }

// first index in [0, k) with sp[index] >= q (strict = false) or > q (strict =
// true); k < 2^31, so 32-bit indices, and selects instead of branches
template <typename T>
__device__ __forceinline__ int64_t bound(const T* __restrict__ sp, int64_t k, T q, bool strict) {
    uint32_t lo = 0, len = (uint32_t)k;
    while (len > 0) {
        const uint32_t half = len >> 1;
        const T v = sp[lo + half];
        const bool go = strict ? v <= q : v < q;
        lo = go ? lo + half + 1 : lo;
        len = go ? len - half - 1 : half;
    }
    return (int64_t)lo;
}

// #{b < q} (upper: #{b <= q}) over ascending b[0..k), by one warp: each round
// probes 32 points of the remaining range at once (4 rounds of dependent loads
// for k = 2^20, against 20 for a binary search).  lane: this thread's lane.
template <typename T>
__device__ __forceinline__ int64_t warp_bound(const T* __restrict__ b, int64_t k, T q, bool upper, int lane) {
    int64_t lo = 0, hi = k;  // the first index whose element fails the test
    while (lo < hi) {
        const int64_t span = hi - lo, mid = lo + span * lane / 32;
        const T v = b[mid];
        const unsigned m = __ballot_sync(FULL, upper ? v <= q : v < q);
        const int c = __popc(m);  // probes 0..c-1 pass, c..31 fail
        const int64_t nlo = c == 0 ? lo : lo + span * (c - 1) / 32 + 1;
        const int64_t nhi = c == 32 ? hi : lo + span * c / 32;
        lo = nlo;
        hi = nhi;
    }
    return lo;
}

// The queries are ascending, so a block takes them in chunks of QCH consecutive
// ones and first finds the window [lo, hi) of sp that holds the bounds of all of
// them: lo = #{sp < sq[r0]}, hi = #{sp <= sq[r1 - 1]}.  Each query then searches
// only that window.  Contains block barriers: every thread of the block calls it.
constexpr int QCH = 256;

template <typename T>
__device__ __forceinline__ void chunk_window(const T* __restrict__ sq, const T* __restrict__ sp, int64_t k,
                                             int64_t r0, int64_t r1, int64_t& lo, int64_t& hi) {
    __shared__ int64_t win[2];
    __syncthreads();  // the previous chunk's threads have read win
    // warps 0 and 1 each search the whole of sp, 32 probes per round
    const int wq = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (wq < 2) {
        const int64_t v = warp_bound<T>(sp, k, sq[wq == 0 ? r0 : r1 - 1], wq == 1, lane);
        if (lane == 0) win[wq] = v;
    }
    __syncthreads();
    lo = win[0];
    hi = win[1];
}

// A window of at most QWIN points of sp is copied to shared memory, and the
// queries search it there (a few shared loads instead of dependent global ones).
constexpr int QWIN = 2048;

template <typename T>
__device__ __forceinline__ void stage_window(const T* __restrict__ sp, int64_t lo, int64_t hi, T* swin) {
    if (hi - lo <= QWIN)
        for (int64_t j = threadIdx.x; j < hi - lo; j += blockDim.x) swin[j] = sp[lo + j];
    __syncthreads();
}

// lb = #{sp < q}, ub = #{sp <= q} for a query whose bounds lie in [lo, hi]
template <typename T>
__device__ __forceinline__ void window_bounds(const T* __restrict__ sp, int64_t lo, int64_t hi, const T* swin, T q,
                                              int64_t& lb, int64_t& ub) {
    const T* base = hi - lo <= QWIN ? swin : sp + lo;
    lb = lo + bound<T>(base, hi - lo, q, false);
    ub = lo + bound<T>(base, hi - lo, q, true);
}

// out[row_r] = -w[row_r] S_r for the sorted query anchors sq (rows through pq)
template <typename T>
__global__ void __launch_bounds__(QCH) k_signed_query(const T* __restrict__ sq, const int32_t* __restrict__ pq,
                                                      int64_t m, const T* __restrict__ sp, int64_t k,
                                                      const T* __restrict__ F, const T* __restrict__ G,
                                                      const T* __restrict__ w, T* __restrict__ out) {
    __shared__ T swin[QWIN];
    const int64_t nch = (m + QCH - 1) / QCH;
    for (int64_t c = blockIdx.x; c < nch; c += gridDim.x) {
        const int64_t r0 = c * QCH, r1 = min(r0 + QCH, m);
        int64_t lo, hi;
        chunk_window<T>(sq, sp, k, r0, r1, lo, hi);
        stage_window<T>(sp, lo, hi, swin);
        const int64_t r = r0 + threadIdx.x;
        if (r >= r1) continue;
        const T q = sq[r];
        int64_t lb, ub;
        window_bounds<T>(sp, lo, hi, swin, q, lb, ub);
        T S = T(0);
        if (lb > 0) S = F[lb - 1] * dexp<T>(sp[lb - 1] - q);
        if (ub < k) S -= G[ub] * dexp<T>(q - sp[ub]);
        const int64_t row = pq ? (int64_t)pq[r] : r;
        out[row] = -w[row] * S;
    }
}

// workspace of one signed sum over a side of `len` anchors: F and G, then the
// scan's per-tile records (tp_ws_bytes)
size_t sgen_ws_bytes(int64_t len, int f64) {
    const size_t es = f64 ? 8 : 4;
    const int64_t tile = (int64_t)OS_NT * os_E((int)es);
    const int64_t ntiles = std::max<int64_t>(1, (len + tile - 1) / tile);
    return 2 * Carve::need((size_t)std::max<int64_t>(len, 1), es) + tp_ws_bytes(ntiles, 1, es);
}

// out = -w * S(q <- p, v): p anchors (sorted, perm pp, values v), q anchors
// (sorted, perm pq, weights w and out in the order pq says)
template <typename T>
static cudaError_t signed_pass(const T* sp, const int32_t* pp, int64_t k, const T* v, const T* sq,
                               const int32_t* pq, int64_t m, const T* w, T* out, void* ws,
                               size_t ws_bytes, cudaStream_t st) {
    if (m == 0) return cudaSuccess;
    if (k == 0) return cudaMemsetAsync(out, 0, sizeof(T) * (size_t)m, st);
    Carve cv(ws, ws_bytes);
    T* F = cv.take<T>(k);
    T* G = cv.take<T>(k);
    if (!cv.ok) return cudaErrorInvalidValue;
    OneSidedTP<T, os_E((int)sizeof(T))> p;
    p.n = k;
    p.s = sp;
    p.perm = pp;
    p.v = v;
    p.F = F;
    p.G = G;
    cudaError_t e = tp_run(p, cv.base + cv.off, cv.cap - cv.off, st);
    if (e != cudaSuccess) return e;
    int dev_ = 0, sms = 0;
    e = tp_sm_count(dev_, sms);
    if (e != cudaSuccess) return e;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((m + 255) / 256, (int64_t)sms * 16));
    k_signed_query<T><<<(unsigned)blocks, QCH, 0, st>>>(sq, pq, m, sp, k, F, G, w, out);
    return cudaGetLastError();
}

template <typename T>
cudaError_t sgen_run(const T* sa, const int32_t* pa, int64_t n, const T* sb, const int32_t* pb,
                     int64_t k, const T* x, const T* g, T* da, T* db, void* ws, size_t ws_bytes,
                     cudaStream_t st) {
    // da = -g S(a <- b, x), then db = -x S(b <- a, g); the workspace is reused
    cudaError_t e = signed_pass<T>(sb, pb, k, x, sa, pa, n, g, da, ws, ws_bytes, st);
    if (e != cudaSuccess) return e;
    return signed_pass<T>(sa, pa, n, g, sb, pb, k, x, db, ws, ws_bytes, st);
}

// ------------------------------------------------------------------ phased backward
// L = <g, K x> with K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j) (summary §2.1;
// trainable anchors and phases, §2.3).  By cos(p - q) = cos p cos q + sin p sin q
// and sin(p - q) = sin p cos q - cos p sin q, with the two channels
//     P(a <- b) = sum_j exp(-|a - b_j|) (cos psi_j x_j, sin psi_j x_j)
//     S(a <- b) = sum_j sign(a - b_j) exp(-|a - b_j|) (cos psi_j x_j, sin psi_j x_j)
// at an a-point with phase phi and weight g:
//     dphi = g (cos phi P1 - sin phi P0),   da = -g (cos phi S0 + sin phi S1),
// and, with the roles of the sides swapped (channels cos phi g, sin phi g seen
// from a b-point with phase psi and weight x):
//     dx = cos psi P0 + sin psi P1,  dpsi = x (cos psi P1 - sin psi P0),
//     db = -x (cos psi S0 + sin psi S1).
// P and S come from the one-sided scans F, G of the two channels (as the signed
// sums above): P = F_{ub-1} exp(b_{ub-1} - a) + G_{ub} exp(a - b_{ub}),
// S = F_{lb-1} exp(b_{lb-1} - a) - G_{ub} exp(a - b_{ub}).


// Policy of threepass.cuh: channels cos(ph) v and sin(ph) v (v and ph gathered
// through perm), prefix F and suffix G written interleaved, [n][2], sorted order.
template <typename T_, int E_>
struct OneSidedPhasedTP {
    using T = T_;
    static constexpr int C = 2, CT = 0, E = E_, NT = OS_NT;
    static constexpr int H = sizeof(T_) == 4 ? 192 : 0;
    int64_t n;
    const T* s;
    const int32_t* perm;
    const T* v;
    const T* ph;
    T* F;
    T* G;
    struct Aux {};
    __device__ __forceinline__ void value(int64_t r, T (&vj)[C]) const {
        const int64_t o = perm ? (int64_t)perm[r] : r;
        T sn, cs;
        psincos(ph[o], &sn, &cs);
        const T x = v[o];
        vj[0] = cs * x;
        vj[1] = sn * x;
    }
    __device__ __forceinline__ void load(int64_t r0, T (&sv)[E], T (&vv)[E][C], Aux&) const {
        constexpr int VN = V16<T>::N;
        if (r0 + E <= n) {
#pragma unroll
            for (int i = 0; i < E; i += VN) ld16_stream<T>(s + r0 + i, &sv[i]);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) sv[i] = s[min(r0 + i, n - 1)];
        }
#pragma unroll
        for (int i = 0; i < E; ++i) {
            if (r0 + i < n) {
                value(r0 + i, vv[i]);
            } else {
                vv[i][0] = T(0);
                vv[i][1] = T(0);
            }
        }
    }
    __device__ __forceinline__ void load1(int64_t j, T& sj, T (&vj)[C]) const {
        sj = s[j];
        value(j, vj);
    }
    __device__ __forceinline__ void finish(int64_t r0, const T (&sv)[E], const T (&vv)[E][C],
                                           T (&dl)[E], T eprev, const T (&Lp)[C], T enext,
                                           const T (&Un)[C], Aux&) const {
        constexpr int VN = V16<T>::N;
        T fo[2 * E], go[2 * E];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            T L = Lp[c];
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const T d = i == 0 ? dexp<T>(eprev - sv[0]) : dl[i];
                L = dfma<T>(d, L, vv[i][c]);
                fo[2 * i + c] = L;
            }
            T U = Un[c];
#pragma unroll
            for (int i = E - 1; i >= 0; --i) {
                const T d = i == E - 1 ? dexp<T>(sv[E - 1] - enext) : dl[i + 1];
                U = dfma<T>(d, U, vv[i][c]);
                go[2 * i + c] = U;
            }
        }
        if (r0 + E <= n) {
#pragma unroll
            for (int i = 0; i < 2 * E; i += VN) {
                st16<T>(F + 2 * r0 + i, &fo[i]);
                st16<T>(G + 2 * r0 + i, &go[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 2 * E; ++i)
                if (r0 + i / 2 < n) {
                    F[2 * r0 + i] = fo[i];
                    G[2 * r0 + i] = go[i];
                }
        }
    }
};

static constexpr int pb_E(int es) { return es == 4 ? 8 : 4; }

// [lb, ub): the run of entries equal to sp[r] around index r (ascending sp of
// length k), by galloping outward from r and bisecting the last step: O(log of
// the run length) loads instead of a search over the whole array.
template <typename T>
__device__ __forceinline__ void tie_run(const T* __restrict__ sp, int64_t k, int64_t r, int64_t& lb, int64_t& ub) {
    const T q = sp[r];
    int64_t in = r, out = r, step = 1;  // sp[in] == q; out: below the run, or -1
    for (;;) {
        out = r - step;
        if (out < 0) {
            out = -1;
            break;
        }
        if (sp[out] < q) break;
        in = out;
        step <<= 1;
    }
    while (in - out > 1) {
        const int64_t mid = out + ((in - out) >> 1);
        if (sp[mid] < q) out = mid;
        else in = mid;
    }
    lb = in;
    in = r;
    step = 1;
    for (;;) {  // out: above the run, or k
        out = r + step;
        if (out >= k) {
            out = k;
            break;
        }
        if (sp[out] > q) break;
        in = out;
        step <<= 1;
    }
    while (out - in > 1) {
        const int64_t mid = in + ((out - in) >> 1);
        if (sp[mid] > q) out = mid;
        else in = mid;
    }
    ub = in + 1;
}

// Per sorted query anchor r (row pq[r]; phase th and weight w in row order):
//     prod = cos th P0 + sin th P1,  dph = w (cos th P1 - sin th P0),
//     dan = -w (cos th S0 + sin th S1),
// each where its pointer is not NULL: prod written, dph and dan written (acc = 0)
// or added (acc = 1).  k = 0 gives P = S = 0.  self_q: the queries are the
// p-side anchors themselves (sq == sp, m == k), so the bounds are the tie run
// around r.
template <typename T>
__global__ void __launch_bounds__(QCH) k_phased_query(const T* __restrict__ sq, const int32_t* __restrict__ pq,
                                                      int64_t m, const T* __restrict__ th,
                                                      const T* __restrict__ w, const T* __restrict__ sp,
                                                      int64_t k, const T* __restrict__ F,
                                                      const T* __restrict__ G, T* prod, T* dph, T* dan,
                                                      int acc, int self_q) {
    __shared__ T swin[QWIN];
    const int64_t nch = (m + QCH - 1) / QCH;
    for (int64_t c = blockIdx.x; c < nch; c += gridDim.x) {
        const int64_t r0 = c * QCH, r1 = min(r0 + QCH, m);
        int64_t lo = 0, hi = k;
        if (!self_q) {  // self_q: the same for the whole grid
            chunk_window<T>(sq, sp, k, r0, r1, lo, hi);
            stage_window<T>(sp, lo, hi, swin);
        }
        const int64_t r = r0 + threadIdx.x;
        if (r >= r1) continue;
        const T q = sq[r];
        int64_t lb, ub;
        if (self_q) {
            tie_run<T>(sp, k, r, lb, ub);
        } else {
            window_bounds<T>(sp, lo, hi, swin, q, lb, ub);
        }
        T P0 = T(0), P1 = T(0), S0 = T(0), S1 = T(0);
        if (ub > 0) {
            const T f = dexp<T>(sp[ub - 1] - q);
            P0 = F[2 * (ub - 1)] * f;
            P1 = F[2 * (ub - 1) + 1] * f;
        }
        if (lb == ub) {
            S0 = P0;
            S1 = P1;
        } else if (lb > 0) {
            const T f = dexp<T>(sp[lb - 1] - q);
            S0 = F[2 * (lb - 1)] * f;
            S1 = F[2 * (lb - 1) + 1] * f;
        }
        if (ub < k) {
            const T f = dexp<T>(q - sp[ub]);
            const T g0 = G[2 * ub] * f, g1 = G[2 * ub + 1] * f;
            P0 += g0;
            P1 += g1;
            S0 -= g0;
            S1 -= g1;
        }
        const int64_t row = pq ? (int64_t)pq[r] : r;
        T sn, cs;
        psincos(th[row], &sn, &cs);
        if (prod) prod[row] = cs * P0 + sn * P1;
        if (dph || dan) {
            const T wr = w[row];
            if (dph) {
                const T v = wr * (cs * P1 - sn * P0);
                dph[row] = acc ? dph[row] + v : v;
            }
            if (dan) {
                const T v = -wr * (cs * S0 + sn * S1);
                dan[row] = acc ? dan[row] + v : v;
            }
        }
    }
}

// workspace of one phased pass over a side of `len` anchors: F and G of the two
// channels, then the scan's per-tile records (tp_ws_bytes)
size_t pbwd_ws_bytes(int64_t len, int f64) {
    const size_t es = f64 ? 8 : 4;
    const int64_t tile = (int64_t)OS_NT * pb_E((int)es);
    const int64_t ntiles = std::max<int64_t>(1, (len + tile - 1) / tile);
    return 2 * Carve::need((size_t)std::max<int64_t>(2 * len, 1), es) + tp_ws_bytes(ntiles, 2, es);
}

// The channels of (p-side anchors sp, perm pp, values v, phases php) seen from
// the query side (sq, pq, phases thq, weights w): prod, dph, dan as in
// k_phased_query.
template <typename T>
static cudaError_t phased_pass(const T* sp, const int32_t* pp, int64_t k, const T* v, const T* php,
                               const T* sq, const int32_t* pq, int64_t m, const T* thq, const T* w,
                               T* prod, T* dph, T* dan, int acc, void* ws, size_t ws_bytes,
                               cudaStream_t st) {
    if (m == 0 || (prod == nullptr && dph == nullptr && dan == nullptr)) return cudaSuccess;
    Carve cv(ws, ws_bytes);
    T* F = cv.take<T>(2 * std::max<int64_t>(k, 1));
    T* G = cv.take<T>(2 * std::max<int64_t>(k, 1));
    if (!cv.ok) return cudaErrorInvalidValue;
    cudaError_t e;
    if (k > 0) {
        OneSidedPhasedTP<T, pb_E((int)sizeof(T))> p;
        p.n = k;
        p.s = sp;
        p.perm = pp;
        p.v = v;
        p.ph = php;
        p.F = F;
        p.G = G;
        e = tp_run(p, cv.base + cv.off, cv.cap - cv.off, st);
        if (e != cudaSuccess) return e;
    }
    int dev_ = 0, sms = 0;
    e = tp_sm_count(dev_, sms);
    if (e != cudaSuccess) return e;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((m + 255) / 256, (int64_t)sms * 16));
    const int self_q = sq == sp && m == k ? 1 : 0;
    k_phased_query<T><<<(unsigned)blocks, QCH, 0, st>>>(sq, pq, m, thq, w, sp, k, F, G, prod, dph, dan, acc,
                                                        self_q);
    return cudaGetLastError();
}

template <typename T>
cudaError_t pbwd_run(const T* sa, const int32_t* pa, const T* phi, int64_t n, const T* sb,
                     const int32_t* pb, const T* psi, int64_t k, const T* x, const T* g, T* dx, T* dphi,
                     T* dpsi, T* da, T* db, void* ws, size_t ws_bytes, cudaStream_t st) {
    // sb == NULL: b = a, psi = phi; the b-side gradients are added to the a-side ones
    const bool sym = sb == nullptr;
    if (sym) {
        sb = sa;
        pb = pa;
        psi = phi;
        k = n;
        dpsi = dphi;
        db = da;
    }
    // a-side: dphi, da from the channels of (x, psi) on b
    cudaError_t e = phased_pass<T>(sb, pb, k, x, psi, sa, pa, n, phi, g, nullptr, dphi, da, 0, ws, ws_bytes, st);
    if (e != cudaSuccess) return e;
    // b-side: dx, dpsi, db from the channels of (g, phi) on a (the workspace is reused)
    return phased_pass<T>(sa, pa, n, g, phi, sb, pb, k, psi, x, dx, dpsi, db, sym ? 1 : 0, ws, ws_bytes, st);
}

// ------------------------------------------------------------------ weighted Gram matrix
// M = A diag(D) A^T, A_ij = exp(-|a_i - b_j|) (summary §2.2 "Operatori di
// Gram").  For a_i <= a_j the terms split at a_i and a_j:
//     b <= a_i:        D_b exp(-(a_i - b)) exp(-(a_j - b)) = e^{a_i - a_j} D_b e^{-2(a_i - b)}
//     a_i < b <= a_j:  D_b exp(-(b - a_i)) exp(-(a_j - b)) = e^{a_i - a_j} D_b
//     b > a_j:         D_b exp(-(b - a_i)) exp(-(b - a_j)) = e^{a_i - a_j} D_b e^{-2(b - a_j)}
// so M_ij = e^{a_i - a_j} (Lw_i + (P_j - P_i) + Rw_j) with, per a-point,
// Lw = sum_{b <= a} D e^{-2(a - b)}, Rw = sum_{b > a} D e^{-2(b - a)} (one-sided
// scans over 2b) and P = sum_{b <= a} D (fp64 prefix sums: their difference
// must not cancel).  Work: O(k) scans, O(n log k) searches, O(n^2) fill.

constexpr int PS_NT = 256, PS_PT = 16, PS_BT = PS_NT * PS_PT;  // prefix sums: elements per block

template <typename T>
__global__ void __launch_bounds__(PS_NT) k_psum_blocks(const T* __restrict__ D, const int32_t* __restrict__ pb,
                                                       int64_t k, double* __restrict__ bsum) {
    __shared__ double red[PS_NT / 32];
    const int64_t b0 = (int64_t)blockIdx.x * PS_BT + (int64_t)threadIdx.x * PS_PT;
    double acc = 0.0;
    for (int i = 0; i < PS_PT; ++i) {
        const int64_t r = b0 + i;
        if (r < k) acc += D ? (double)D[pb ? (int64_t)pb[r] : r] : 1.0;
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(FULL, acc, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < PS_NT / 32; ++w) t += red[w];
        bsum[blockIdx.x] = t;
    }
}

// exclusive prefix of the block sums, one block (each thread a run of them)
__global__ void __launch_bounds__(1024) k_psum_scan(double* __restrict__ bsum, int64_t nb) {
    __shared__ double part[1024];
    const int64_t per = (nb + 1023) / 1024;
    const int64_t b0 = (int64_t)threadIdx.x * per;
    double acc = 0.0;
    for (int64_t i = 0; i < per && b0 + i < nb; ++i) acc += bsum[b0 + i];
    part[threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double run = 0.0;
        for (int t = 0; t < 1024; ++t) {
            const double v = part[t];
            part[t] = run;
            run += v;
        }
    }
    __syncthreads();
    double run = part[threadIdx.x];
    for (int64_t i = 0; i < per && b0 + i < nb; ++i) {
        const double v = bsum[b0 + i];
        bsum[b0 + i] = run;
        run += v;
    }
}

// P[r] = sum_{l <= r} D_l (sorted order)
template <typename T>
__global__ void __launch_bounds__(PS_NT) k_psum_apply(const T* __restrict__ D, const int32_t* __restrict__ pb,
                                                      int64_t k, const double* __restrict__ boff,
                                                      double* __restrict__ P) {
    __shared__ double part[PS_NT];
    const int64_t b0 = (int64_t)blockIdx.x * PS_BT + (int64_t)threadIdx.x * PS_PT;
    double v[PS_PT], acc = 0.0;
    for (int i = 0; i < PS_PT; ++i) {
        const int64_t r = b0 + i;
        v[i] = r < k ? (D ? (double)D[pb ? (int64_t)pb[r] : r] : 1.0) : 0.0;
        acc += v[i];
    }
    part[threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double run = boff[blockIdx.x];
        for (int t = 0; t < PS_NT; ++t) {
            const double x = part[t];
            part[t] = run;
            run += x;
        }
    }
    __syncthreads();
    double run = part[threadIdx.x];
    for (int i = 0; i < PS_PT; ++i) {
        run += v[i];
        if (b0 + i < k) P[b0 + i] = run;
    }
}

template <typename T>
__global__ void __launch_bounds__(256) k_double(const T* __restrict__ s, int64_t k, T* __restrict__ s2) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < k; r += stride) s2[r] = T(2) * s[r];
}

// per sorted a-point (one warp each): Lw, Rw, P (and the inverse of pa)
template <typename T>
__global__ void __launch_bounds__(256) k_gram_points(const T* __restrict__ sa, const int32_t* __restrict__ pa,
                                                     int64_t n, const T* __restrict__ sb, int64_t k,
                                                     const T* __restrict__ F, const T* __restrict__ G,
                                                     const double* __restrict__ P, T* __restrict__ Lw,
                                                     T* __restrict__ Rw, double* __restrict__ Pa,
                                                     int32_t* __restrict__ inv) {
    const int lane = threadIdx.x & 31;
    const int64_t wstride = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; i < n; i += wstride) {
        const T q = sa[i];
        const int64_t ub = warp_bound<T>(sb, k, q, true, lane);  // #{b <= a_i}
        if (lane == 0) {
            Lw[i] = ub > 0 ? F[ub - 1] * dexp<T>(T(2) * (sb[ub - 1] - q)) : T(0);
            Rw[i] = ub < k ? G[ub] * dexp<T>(T(2) * (q - sb[ub])) : T(0);
            Pa[i] = ub > 0 ? P[ub - 1] : 0.0;
            if (pa) inv[pa[i]] = (int32_t)i;
        }
    }
}

// M[r][c], a block per row r (rows and columns in the order of pa, or sorted
// order without it)
template <typename T>
__global__ void __launch_bounds__(256) k_gram_fill(const T* __restrict__ sa, const int32_t* __restrict__ inv,
                                                   int64_t n, const T* __restrict__ Lw, const T* __restrict__ Rw,
                                                   const double* __restrict__ Pa, T* __restrict__ M, int64_t ldm) {
    const int64_t r = blockIdx.x;
    const int64_t i = inv ? (int64_t)inv[r] : r;
    const T ai = sa[i], Li = Lw[i], Ri = Rw[i];
    const double Pi = Pa[i];
    T* row = M + r * ldm;
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
        const int64_t j = inv ? (int64_t)inv[c] : c;
        const T aj = sa[j];
        T v;
        if (j >= i) v = dexp<T>(ai - aj) * (Li + (T)(Pa[j] - Pi) + Rw[j]);
        else v = dexp<T>(aj - ai) * (Lw[j] + (T)(Pi - Pa[j]) + Ri);
        row[c] = v;
    }
}

size_t grammat_ws_bytes(int64_t n, int64_t k, int f64) {
    const size_t es = f64 ? 8 : 4;
    const int64_t nb = std::max<int64_t>(1, (k + PS_BT - 1) / PS_BT);
    return Carve::need((size_t)std::max<int64_t>(k, 1), es) + sgen_ws_bytes(k, f64) +
           Carve::need((size_t)std::max<int64_t>(k, 1), 8) + Carve::need((size_t)nb, 8) +
           2 * Carve::need((size_t)std::max<int64_t>(n, 1), es) + Carve::need((size_t)std::max<int64_t>(n, 1), 8) +
           Carve::need((size_t)std::max<int64_t>(n, 1), 4);
}

template <typename T>
cudaError_t grammat_run(const T* sa, const int32_t* pa, int64_t n, const T* sb, const int32_t* pb, int64_t k,
                        const T* D, T* M, int64_t ldm, void* ws, size_t ws_bytes, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    Carve cv(ws, ws_bytes);
    T* s2 = cv.take<T>(std::max<int64_t>(k, 1));
    T* F = cv.take<T>(std::max<int64_t>(k, 1));
    T* G = cv.take<T>(std::max<int64_t>(k, 1));
    double* P = cv.take<double>(std::max<int64_t>(k, 1));
    const int64_t nb = std::max<int64_t>(1, (k + PS_BT - 1) / PS_BT);
    double* bsum = cv.take<double>(nb);
    T* Lw = cv.take<T>(n);
    T* Rw = cv.take<T>(n);
    double* Pa = cv.take<double>(n);
    int32_t* inv = cv.take<int32_t>(n);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev_ = 0, sms = 0;
    cudaError_t e = tp_sm_count(dev_, sms);
    if (e != cudaSuccess) return e;
    const int64_t gb = std::max<int64_t>(1, (int64_t)sms * 8);
    if (k > 0) {
        k_double<T><<<(unsigned)std::min<int64_t>(gb, (k + 255) / 256), 256, 0, st>>>(sb, k, s2);
        OneSidedTP<T, os_E((int)sizeof(T))> p;
        p.n = k;
        p.s = s2;
        p.perm = pb;
        p.v = D;
        p.F = F;
        p.G = G;
        e = tp_run(p, cv.base + cv.off, cv.cap - cv.off, st);
        if (e != cudaSuccess) return e;
        k_psum_blocks<T><<<(unsigned)nb, PS_NT, 0, st>>>(D, pb, k, bsum);
        k_psum_scan<<<1, 1024, 0, st>>>(bsum, nb);
        k_psum_apply<T><<<(unsigned)nb, PS_NT, 0, st>>>(D, pb, k, bsum, P);
    }
    k_gram_points<T><<<(unsigned)std::max<int64_t>(1, std::min<int64_t>(gb * 8, (n + 7) / 8)), 256, 0, st>>>(sa, pa, n, sb, k, F, G, P,
                                                                                      Lw, Rw, Pa, inv);
    k_gram_fill<T><<<(unsigned)n, 256, 0, st>>>(sa, pa ? inv : nullptr, n, Lw, Rw, Pa, M, ldm);  // a block per row
    return cudaGetLastError();
}

template cudaError_t grammat_run<float>(const float*, const int32_t*, int64_t, const float*, const int32_t*,
                                        int64_t, const float*, float*, int64_t, void*, size_t, cudaStream_t);
template cudaError_t grammat_run<double>(const double*, const int32_t*, int64_t, const double*, const int32_t*,
                                         int64_t, const double*, double*, int64_t, void*, size_t, cudaStream_t);

template cudaError_t sgen_run<float>(const float*, const int32_t*, int64_t, const float*, const int32_t*,
                                     int64_t, const float*, const float*, float*, float*, void*, size_t,
                                     cudaStream_t);
template cudaError_t sgen_run<double>(const double*, const int32_t*, int64_t, const double*,
                                      const int32_t*, int64_t, const double*, const double*, double*,
                                      double*, void*, size_t, cudaStream_t);

template cudaError_t pbwd_run<float>(const float*, const int32_t*, const float*, int64_t, const float*,
                                     const int32_t*, const float*, int64_t, const float*, const float*, float*,
                                     float*, float*, float*, float*, void*, size_t, cudaStream_t);
template cudaError_t pbwd_run<double>(const double*, const int32_t*, const double*, int64_t, const double*,
                                      const int32_t*, const double*, int64_t, const double*, const double*,
                                      double*, double*, double*, double*, double*, void*, size_t, cudaStream_t);

}  // namespace lx
