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

// first index in [0, k) with sp[index] >= q (strict = false) or > q (strict = true)
template <typename T>
__device__ __forceinline__ int64_t bound(const T* __restrict__ sp, int64_t k, T q, bool strict) {
    int64_t lo = 0, hi = k;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        const T v = sp[mid];
        if (strict ? v <= q : v < q) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// out[row_r] = -w[row_r] S_r for the sorted query anchors sq (rows through pq)
template <typename T>
__global__ void __launch_bounds__(256) k_signed_query(const T* __restrict__ sq, const int32_t* __restrict__ pq,
                                                      int64_t m, const T* __restrict__ sp, int64_t k,
                                                      const T* __restrict__ F, const T* __restrict__ G,
                                                      const T* __restrict__ w, T* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < m; r += stride) {
        const T q = sq[r];
        const int64_t lb = bound<T>(sp, k, q, false), ub = bound<T>(sp, k, q, true);
        T S = T(0);
        if (lb > 0) S = F[lb - 1] * dexp<T>(sp[lb - 1] - q);
        if (ub < k) S -= G[ub] * dexp<T>(q - sp[ub]);
        const int64_t row = pq ? (int64_t)pq[r] : r;
        out[row] = -w[row] * S;
    }
}

// workspace of one signed sum over a side of `len` anchors: F, G and the scan's
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
    int sms = 0;
    e = tp_sm_count(sms);
    if (e != cudaSuccess) return e;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((m + 255) / 256, (int64_t)sms * 16));
    k_signed_query<T><<<(unsigned)blocks, 256, 0, st>>>(sq, pq, m, sp, k, F, G, w, out);
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

template cudaError_t sgen_run<float>(const float*, const int32_t*, int64_t, const float*, const int32_t*,
                                     int64_t, const float*, const float*, float*, float*, void*, size_t,
                                     cudaStream_t);
template cudaError_t sgen_run<double>(const double*, const int32_t*, int64_t, const double*,
                                      const int32_t*, int64_t, const double*, const double*, double*,
                                      double*, void*, size_t, cudaStream_t);

}  // namespace lx
