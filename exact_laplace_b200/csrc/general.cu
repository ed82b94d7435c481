// general.cu -- the general LAPLEX product, a != b ("LAPLEX - La FFT dei Nuclei
// di Laplace Apprendibili", technical summary §2.2 "Caso Generale"), and its
// phased variant (§2.1).
//
//   y_i = sum_j exp(-|a_i - b_j|) x_j            (a: n output anchors, b: k input anchors)
//   y_i = sum_j exp(-|a_i - b_j|) cos(phi_i - psi_j) x_j
//
// The page gathers the b-contributions into the intervals cut by the sorted a
// and propagates the summaries with the symmetric scan.  Here the same sums
// are taken by ONE scan over the merged sorted sequence of a and b: b-points
// carry x_j (phased: cos psi_j x_j and sin psi_j x_j), a-points carry 0, and at
// every a-point y = L + U (the a-point itself adds nothing, and each b-point
// sits either before or after it, so every pair is counted once; equal anchors
// weigh exp(0) = 1 on either side).  Merge order: a_i before b_j iff a_i < b_j.
//
// Kernels: k_merge_partition (merge-path split of the merged sequence into
// tiles), k_gen_onepass (single pass, onepass.cuh carries), k_suffix_carries +
// k_gen_fixup (only for tiles whose look-ahead was deferred).  K^T is the same
// product with the roles of a and b exchanged (done by the caller).
#include <algorithm>

#include "laplex_impl.h"
#include "onepass.cuh"

namespace lx {

constexpr int GEN_NT = 256;

template <typename T> __device__ __forceinline__ void gsincos(T a, T* s, T* c);
template <> __device__ __forceinline__ void gsincos<float>(float a, float* s, float* c) { sincosf(a, s, c); }
template <> __device__ __forceinline__ void gsincos<double>(double a, double* s, double* c) { sincos(a, s, c); }

// ia[t] = number of a-points among the first min(t*tile, n+k) merged elements.
template <typename T>
__global__ void k_merge_partition(const T* __restrict__ a, int64_t n, const T* __restrict__ b,
                                  int64_t k, int64_t tile, int64_t ntiles, int64_t* __restrict__ ia) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t > ntiles) return;
    const int64_t p = min(t * tile, n + k);
    int64_t lo = max((int64_t)0, p - k), hi = min(p, n);
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (a[mid] < b[p - 1 - mid]) lo = mid + 1;
        else hi = mid;
    }
    ia[t] = lo;
}

template <typename T, int NCOL, bool PHASED, int E, int NT>
__global__ void __launch_bounds__(NT) k_gen_onepass(GenArgs<T> A, OnePassWs<T> W,
                                                    const int64_t* __restrict__ ia, int64_t ntiles) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    constexpr int TILE = NT * E;
    __shared__ T sh_anc[TILE];          // a-part [0, na), b-part [na, na + nb)
    __shared__ T sh_val[TILE * C];      // channel values of the b-part
    __shared__ BlockScanSmem<T, C, NT> smf, smb;
    __shared__ int64_t sh_tile;
    __shared__ T sh_e[2];
    __shared__ T sh_c[2][C];
    if (threadIdx.x == 0) sh_tile = (int64_t)atomicAdd(&W.ctrl[0], 1u);
    __syncthreads();
    const int64_t t = sh_tile;
    const int64_t n = A.n, k = A.k, N = n + k;
    const int64_t p0 = t * TILE, p1 = min(p0 + TILE, N);
    const int64_t i0 = ia[t], i1 = ia[t + 1];
    const int64_t j0 = p0 - i0, j1 = p1 - i1;
    const int na = (int)(i1 - i0), nb = (int)(j1 - j0), cnt = na + nb;
    for (int q = threadIdx.x; q < na; q += NT) sh_anc[q] = A.sa[i0 + q];
    for (int q = threadIdx.x; q < nb; q += NT) {
        const int64_t j = j0 + q;
        sh_anc[na + q] = A.sb[j];
        const int64_t row = A.pin ? (int64_t)A.pin[j] : j;
        const T dsc = A.D ? A.D[A.pD ? (int64_t)A.pD[j] : j] : T(1);
        T cs = T(1), sn = T(0);
        if (PHASED) gsincos<T>(A.psi[A.ppsi ? (int64_t)A.ppsi[j] : j], &sn, &cs);
        const T* xr = A.x + row * A.ldx + A.col0;
#pragma unroll
        for (int c = 0; c < NCOL; ++c) {
            const T val = (c < A.ncol ? xr[c] : T(0)) * dsc;
            if (PHASED) {
                sh_val[q * C + 2 * c] = cs * val;
                sh_val[q * C + 2 * c + 1] = sn * val;
            } else {
                sh_val[q * C + c] = val;
            }
        }
    }
    __syncthreads();
    const T* Aa = sh_anc;
    const T* Bb = sh_anc + na;
    // this thread's merged range [d0, d0 + E) within the tile: merge-path search
    const int d0 = min((int)threadIdx.x * E, cnt);
    int lo = max(0, d0 - nb), hi = min(d0, na);
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (Aa[mid] < Bb[d0 - 1 - mid]) lo = mid + 1;
        else hi = mid;
    }
    int ai = lo, bi = d0 - lo;
    const T padA = cnt > 0 ? (na > 0 && (nb == 0 || Aa[na - 1] >= Bb[nb - 1]) ? Aa[na - 1] : Bb[nb - 1])
                           : T(0);
    T s[E], v[E][C], dl[E], fV[C], bW[C];
    int aidx[E];  // local a index for a-points, -1 otherwise
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const bool valid = d0 + e < cnt;
        const bool takeA = valid && ai < na && (bi >= nb || Aa[ai] < Bb[bi]);
        if (!valid) {
            s[e] = padA;
            aidx[e] = -1;
#pragma unroll
            for (int c = 0; c < C; ++c) v[e][c] = T(0);
        } else if (takeA) {
            s[e] = Aa[ai];
            aidx[e] = ai;
            ++ai;
#pragma unroll
            for (int c = 0; c < C; ++c) v[e][c] = T(0);
        } else {
            s[e] = Bb[bi];
            aidx[e] = -1;
#pragma unroll
            for (int c = 0; c < C; ++c) v[e][c] = sh_val[bi * C + c];
            ++bi;
        }
    }
    chunk_aggregates<T, C, E>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    block_excl_fwd<T, C, NT>(s[E - 1], fV, hf, pe, pV, te, tV, smf);
    block_excl_bwd<T, C, NT>(s[0], bW, hb, nf, nW, tf, tW, smb);
    if (threadIdx.x == 0) {
        // anchors of the merged elements just before and just after this tile
        T eT = padA, fT = padA;
        if (p0 > 0) {
            if (i0 > 0 && j0 > 0) eT = max(A.sa[i0 - 1], A.sb[j0 - 1]);
            else eT = i0 > 0 ? A.sa[i0 - 1] : A.sb[j0 - 1];
        } else if (cnt > 0) {
            eT = s[0];
        }
        if (p1 < N) {
            if (i1 < n && j1 < k) fT = min(A.sa[i1], A.sb[j1]);
            else fT = i1 < n ? A.sa[i1] : A.sb[j1];
        }
        T acc[C], accb[C];
        onepass_carries<T, C>(W, t, ntiles, tf, tW, te, tV, eT, fT, acc, accb, A.status);
        sh_e[0] = eT;
        sh_e[1] = fT;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            sh_c[0][c] = acc[c];
            sh_c[1][c] = accb[c];
        }
    }
    __syncthreads();
    T VT[C], WT[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        VT[c] = sh_c[0][c];
        WT[c] = sh_c[1][c];
    }
    T eprev, Lprev[C], enext, Unext[C], out[E][C];
    apply_carry_fwd<T, C>(hf, pe, pV, sh_e[0], VT, eprev, Lprev);
    apply_carry_bwd<T, C>(hb, nf, nW, sh_e[1], WT, enext, Unext);
    chunk_final<T, C, E>(s, v, dl, eprev, Lprev, enext, Unext, out);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (aidx[e] < 0) continue;
        const int64_t i = i0 + aidx[e];
        const int64_t row = A.pout ? (int64_t)A.pout[i] : i;
        T* yr = A.y + row * A.ldy + A.col0;
        if (PHASED) {
            T sp, cp;
            gsincos<T>(A.phi[A.pphi ? (int64_t)A.pphi[i] : i], &sp, &cp);
#pragma unroll
            for (int c = 0; c < NCOL; ++c)
                if (c < A.ncol) yr[c] = cp * out[e][2 * c] + sp * out[e][2 * c + 1];
        } else {
#pragma unroll
            for (int c = 0; c < NCOL; ++c)
                if (c < A.ncol) yr[c] = out[e][c];
        }
    }
}

// y_i += exp(a_i - fT) * carB[t] for the a-points of each deferred tile.
template <typename T, int NCOL, bool PHASED, int NT>
__global__ void __launch_bounds__(NT) k_gen_fixup(GenArgs<T> A, OnePassWs<T> W,
                                                  const int64_t* __restrict__ ia, int64_t tile) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    const uint32_t nfix = W.ctrl[1];
    for (uint32_t q = blockIdx.x; q < nfix; q += gridDim.x) {
        const int64_t t = W.fix[q];
        const int64_t n = A.n, k = A.k, N = n + k;
        const int64_t p1 = min((t + 1) * tile, N);
        if (p1 >= N) continue;
        const int64_t i0 = ia[t], i1 = ia[t + 1], j1 = p1 - i1;
        T fT;
        if (i1 < n && j1 < k) fT = min(A.sa[i1], A.sb[j1]);
        else fT = i1 < n ? A.sa[i1] : A.sb[j1];
        T cr[C];
#pragma unroll
        for (int c = 0; c < C; ++c) cr[c] = W.carB[t * C + c];
        for (int64_t i = i0 + threadIdx.x; i < i1; i += NT) {
            const T f = dexp<T>(A.sa[i] - fT);
            if (f == T(0)) continue;
            const int64_t row = A.pout ? (int64_t)A.pout[i] : i;
            T* yr = A.y + row * A.ldy + A.col0;
            if (PHASED) {
                T sp, cp;
                gsincos<T>(A.phi[A.pphi ? (int64_t)A.pphi[i] : i], &sp, &cp);
                for (int c = 0; c < A.ncol; ++c) yr[c] += f * (cp * cr[2 * c] + sp * cr[2 * c + 1]);
            } else {
                for (int c = 0; c < A.ncol; ++c) yr[c] += f * cr[c];
            }
        }
    }
}

// ------------------------------------------------------------------ host side
struct GenPlan {
    int ncol, C, E;
    int64_t tile, ntiles, groups;
};

// elements per thread: keeps the staged b-values of a tile within 48 KB of shared memory
constexpr int gen_E(int C, int es) { return C * es <= 4 ? 8 : (C * es <= 16 ? 4 : 2); }

static GenPlan gen_plan(int64_t n, int64_t k, int64_t B, bool phased, int es) {
    GenPlan p;
    const int maxcol = phased ? 4 : 8;
    int nc = 1;
    while (nc < B && nc < maxcol) nc <<= 1;
    p.ncol = nc;
    p.C = phased ? 2 * nc : nc;
    p.E = gen_E(p.C, es);
    p.tile = (int64_t)GEN_NT * p.E;
    p.ntiles = std::max<int64_t>(1, (n + k + p.tile - 1) / p.tile);
    p.groups = (B + nc - 1) / nc;
    return p;
}

size_t gen_ws_bytes(int64_t n, int64_t k, int64_t B, bool phased, int f64) {
    const GenPlan p = gen_plan(n, k, B, phased, f64 ? 8 : 4);
    return Carve::need((size_t)(p.ntiles + 1), 8) + onepass_ws_bytes(p.ntiles, p.C, f64 ? 8 : 4);
}

template <typename T, int NCOL, bool PHASED>
static cudaError_t gen_launch(const GenArgs<T>& A, const GenPlan& p, const OnePassWs<T>& W,
                              const int64_t* ia, cudaStream_t st) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    constexpr int E = gen_E(C, (int)sizeof(T));
    cudaError_t e = onepass_reset(W, p.ntiles, st);
    if (e != cudaSuccess) return e;
    profile_before(st);
    k_gen_onepass<T, NCOL, PHASED, E, GEN_NT><<<(unsigned)p.ntiles, GEN_NT, 0, st>>>(A, W, ia, p.ntiles);
    profile_after(st);
    k_suffix_carries<T, C, 1024><<<1, 1024, 0, st>>>(W, p.ntiles);
    k_gen_fixup<T, NCOL, PHASED, GEN_NT><<<FIXUP_BLOCKS, GEN_NT, 0, st>>>(A, W, ia, p.tile);
    return cudaGetLastError();
}

template <typename T>
cudaError_t gen_run(GenArgs<T> A, int64_t B, bool phased, void* ws, size_t ws_bytes,
                    cudaStream_t st) {
    if (A.n == 0) return cudaSuccess;
    if (A.k == 0)  // no input anchors: every output row is zero
        return cudaMemsetAsync(A.y, 0, sizeof(T) * (size_t)(A.n * A.ldy), st);
    const GenPlan p = gen_plan(A.n, A.k, B, phased, (int)sizeof(T));
    Carve cv(ws, ws_bytes);
    int64_t* ia = cv.take<int64_t>(p.ntiles + 1);
    OnePassWs<T> W = onepass_carve<T>(cv, p.ntiles, p.C);
    if (!cv.ok) return cudaErrorInvalidValue;
    {
        const unsigned blocks = (unsigned)((p.ntiles + 1 + 255) / 256);
        k_merge_partition<T><<<blocks, 256, 0, st>>>(A.sa, A.n, A.sb, A.k, p.tile, p.ntiles, ia);
    }
    for (int64_t g = 0; g < p.groups; ++g) {
        A.col0 = g * p.ncol;
        A.ncol = (int)std::min<int64_t>(p.ncol, B - A.col0);
        cudaError_t e;
        if (!phased) {
            switch (p.ncol) {
                case 1: e = gen_launch<T, 1, false>(A, p, W, ia, st); break;
                case 2: e = gen_launch<T, 2, false>(A, p, W, ia, st); break;
                case 4: e = gen_launch<T, 4, false>(A, p, W, ia, st); break;
                default: e = gen_launch<T, 8, false>(A, p, W, ia, st); break;
            }
        } else {
            switch (p.ncol) {
                case 1: e = gen_launch<T, 1, true>(A, p, W, ia, st); break;
                case 2: e = gen_launch<T, 2, true>(A, p, W, ia, st); break;
                default: e = gen_launch<T, 4, true>(A, p, W, ia, st); break;
            }
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template cudaError_t gen_run<float>(GenArgs<float>, int64_t, bool, void*, size_t, cudaStream_t);
template cudaError_t gen_run<double>(GenArgs<double>, int64_t, bool, void*, size_t, cudaStream_t);

}  // namespace lx
