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
// Kernels (the wait-free scheme of threepass.cuh on the merged sequence):
// k_merge_partition (merge-path split into tiles), k_gen_local (tile-local
// scan, outputs at the a-points), k_tp_carry_blocks + k_tp_carry_tiles (exact
// tile carries), k_gen_headtail (carries added to the a-points of each tile's
// head and tail reach).  K^T is the same product with the roles of a and b
// exchanged (done by the caller).
#include <algorithm>

#include "laplex_impl.h"
#include "threepass.cuh"

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

// Tile-local scan of the merged sequence with zero carries from outside the
// tile (threepass.cuh pass 1 for the merged case).  Outputs go to the
// a-points; the tile's totals and its reach in a-points (a-points within CUT
// of the tile's first / last merged anchor) go to the workspace.
template <typename T, int NCOL, bool PHASED, int E, int NT>
__global__ void __launch_bounds__(NT) k_gen_local(GenArgs<T> A, TPWs<T, PHASED ? 2 * NCOL : NCOL> W,
                                                  const int64_t* __restrict__ ia) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    constexpr int TILE = NT * E;
    __shared__ T sh_anc[TILE];      // a-part [0, na), b-part [na, na + nb)
    __shared__ T sh_val[TILE * C];  // channel values of the b-part
    __shared__ BlockScan2Smem<T, C, NT> sm2;
    const int64_t t = blockIdx.x;
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
    const T first = na > 0 && (nb == 0 || Aa[0] <= Bb[0]) ? Aa[0] : Bb[0];
    const T padA = na > 0 && (nb == 0 || Aa[na - 1] >= Bb[nb - 1]) ? Aa[na - 1] : Bb[nb - 1];
    const int d0 = min((int)threadIdx.x * E, cnt);
    int lo = max(0, d0 - nb), hi = min(d0, na);
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (Aa[mid] < Bb[d0 - 1 - mid]) lo = mid + 1;
        else hi = mid;
    }
    int ai = lo, bi = d0 - lo;
    T s[E], v[E][C], dl[E], fV[C], bW[C];
    int aidx[E];
    int h = 0, q = 0;
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
            h += (Aa[ai] - first < ExpCut<T>::v) ? 1 : 0;
            q += (padA - Aa[ai] < ExpCut<T>::v) ? 1 : 0;
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
    const int hq[2] = {h, q};
    int reach[2];
    (void)block_excl_both_counted<T, C, NT, 0, true>(s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf,
                                                     nW, tf, tW, hq, reach, false, sm2);
    if (threadIdx.x == 0) {
        W.tfirst[t] = tf;
        W.tlast[t] = te;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            W.fagg[t * C + c] = tV[c];
            W.bagg[t * C + c] = tW[c];
        }
        W.st[t].head = reach[0];
        W.st[t].tail = reach[1];
    }
    T eprev = hf ? pe : s[0], enext = hb ? nf : s[E - 1];
    T Lprev[C], Unext[C], out[E][C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        Lprev[c] = hf ? pV[c] : T(0);
        Unext[c] = hb ? nW[c] : T(0);
    }
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

// Carries into the a-points of each tile's head and tail reach (a warp per tile).
template <typename T, int NCOL, bool PHASED>
__global__ void __launch_bounds__(256) k_gen_headtail(GenArgs<T> A, TPWs<T, PHASED ? 2 * NCOL : NCOL> W,
                                                      const int64_t* __restrict__ ia, int64_t tile,
                                                      int64_t ntiles) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    const int lane = threadIdx.x & 31;
    const int64_t n = A.n, k = A.k, N = n + k;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < ntiles;
         t += warps) {
        const int64_t p0 = t * tile, p1 = min(p0 + tile, N);
        const int64_t i0 = ia[t], i1 = ia[t + 1], j0 = p0 - i0, j1 = p1 - i1;
        const TPStats stt = W.st[t];
        for (int side = 0; side < 2; ++side) {
            const bool left = side == 0;
            if (left ? t == 0 : t == ntiles - 1) continue;
            T c[C];
            bool nz = false;
#pragma unroll
            for (int q = 0; q < C; ++q) {
                c[q] = (left ? W.carF : W.carB)[t * C + q];
                nz |= c[q] != T(0);
            }
            if (!nz) continue;
            T edge;  // merged anchor just before (left) or just after (right) the tile
            if (left) {
                if (i0 > 0 && j0 > 0) edge = max(A.sa[i0 - 1], A.sb[j0 - 1]);
                else edge = i0 > 0 ? A.sa[i0 - 1] : A.sb[j0 - 1];
            } else {
                if (i1 < n && j1 < k) edge = min(A.sa[i1], A.sb[j1]);
                else edge = i1 < n ? A.sa[i1] : A.sb[j1];
            }
            const int64_t len = left ? stt.head : stt.tail;
            for (int64_t q = lane; q < len; q += 32) {
                const int64_t i = left ? i0 + q : i1 - 1 - q;
                const T f = dexp<T>(left ? edge - A.sa[i] : A.sa[i] - edge);
                if (f == T(0)) continue;
                const int64_t row = A.pout ? (int64_t)A.pout[i] : i;
                T* yr = A.y + row * A.ldy + A.col0;
                if (PHASED) {
                    T sp, cp;
                    gsincos<T>(A.phi[A.pphi ? (int64_t)A.pphi[i] : i], &sp, &cp);
                    for (int q2 = 0; q2 < A.ncol; ++q2) yr[q2] += f * (cp * c[2 * q2] + sp * c[2 * q2 + 1]);
                } else {
                    for (int q2 = 0; q2 < A.ncol; ++q2) yr[q2] += f * c[q2];
                }
            }
            __syncwarp();
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
    return Carve::need((size_t)(p.ntiles + 1), 8) + tp_ws_bytes(p.ntiles, p.C, f64 ? 8 : 4);
}

template <typename T, int NCOL, bool PHASED>
static cudaError_t gen_launch(const GenArgs<T>& A, const GenPlan& p, void* wsbody, size_t wsb,
                              const int64_t* ia, cudaStream_t st) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    constexpr int E = gen_E(C, (int)sizeof(T));
    Carve cv(wsbody, wsb);
    TPWs<T, C> W = tp_carve<T, C>(cv, p.ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    W.redo_count = nullptr;  // every tile takes the carries (reach read-modify-write)
    const int64_t nb = (p.ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    profile_before(st);
    k_gen_local<T, NCOL, PHASED, E, GEN_NT><<<(unsigned)p.ntiles, GEN_NT, 0, st>>>(A, W, ia);
    profile_after(st);
    k_tp_carry_blocks<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, p.ntiles);
    k_tp_carry_tiles<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, p.ntiles, nb);
    const int64_t htb = std::max<int64_t>(1, std::min<int64_t>((p.ntiles + 7) / 8, 148 * 8));
    k_gen_headtail<T, NCOL, PHASED><<<(unsigned)htb, 256, 0, st>>>(A, W, ia, p.tile, p.ntiles);
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
    if (!cv.ok) return cudaErrorInvalidValue;
    void* wsbody = cv.base + cv.off;
    const size_t wsb = cv.cap - cv.off;
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
                case 1: e = gen_launch<T, 1, false>(A, p, wsbody, wsb, ia, st); break;
                case 2: e = gen_launch<T, 2, false>(A, p, wsbody, wsb, ia, st); break;
                case 4: e = gen_launch<T, 4, false>(A, p, wsbody, wsb, ia, st); break;
                default: e = gen_launch<T, 8, false>(A, p, wsbody, wsb, ia, st); break;
            }
        } else {
            switch (p.ncol) {
                case 1: e = gen_launch<T, 1, true>(A, p, wsbody, wsb, ia, st); break;
                case 2: e = gen_launch<T, 2, true>(A, p, wsbody, wsb, ia, st); break;
                default: e = gen_launch<T, 4, true>(A, p, wsbody, wsb, ia, st); break;
            }
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template cudaError_t gen_run<float>(GenArgs<float>, int64_t, bool, void*, size_t, cudaStream_t);
template cudaError_t gen_run<double>(GenArgs<double>, int64_t, bool, void*, size_t, cudaStream_t);

}  // namespace lx
