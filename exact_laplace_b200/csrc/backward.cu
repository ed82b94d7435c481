// backward.cu -- backward pass of L = <g, K x>, K_ij = exp(-|a_i - a_j|), with
// respect to x and the anchors (differentiability in the anchors: "LAPLEX - La
// FFT dei Nuclei di Laplace Apprendibili", technical summary §2.3 and §4.1).
//
//   dx   = K^T g = K g
//   da_i = -g_i D(x)_i - x_i D(g)_i,   D(v)_i = sum_j sign(a_i - a_j) exp(-|a_i - a_j|) v_j
//
// with sign(0) = 0.  In sorted order D(v)_r is the strictly-lower minus the
// strictly-upper exp-weighted sum:  D(v)_r = (L^v_r - P^v_r) - (U^v_r - Q^v_r),
// where L, U are the inclusive prefix/suffix scans of the symmetric product and
// P, Q the inclusive prefix/suffix sums over the run of anchors equal to a_r
// (scan_core.cuh "tie channels").  One single-pass scan of four channels
// (x, g with exp decay; x, g with tie decay) reads s, x, g once and writes
// dx, da once: 20 bytes per anchor in fp32.
#include <algorithm>

#include "laplex_impl.h"
#include "onepass.cuh"

namespace lx {

constexpr int BWD_NT = 256;

template <typename T, int E, int NT>
__global__ void __launch_bounds__(NT) k_bwd_onepass(const T* __restrict__ s_, const int32_t* __restrict__ perm,
                                                    int64_t n, const T* __restrict__ x_,
                                                    const T* __restrict__ g_, T* __restrict__ dx_,
                                                    T* __restrict__ da_, OnePassWs<T> W, int64_t ntiles,
                                                    uint32_t* status) {
    constexpr int C = 4, CT = 2;
    constexpr int VN = V16<T>::N;
    constexpr int64_t TILE = (int64_t)NT * E;
    __shared__ BlockScanSmem<T, C, NT> smf, smb;
    __shared__ int64_t sh_tile;
    __shared__ T sh_e[2];
    __shared__ T sh_c[2][C];
    if (threadIdx.x == 0) sh_tile = (int64_t)atomicAdd(&W.ctrl[0], 1u);
    __syncthreads();
    const int64_t t = sh_tile;
    const int64_t tile0 = t * TILE;
    const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
    const bool full = r0 + E <= n;
    T s[E], xv[E], gv[E];
    if (full) {
#pragma unroll
        for (int i = 0; i < E; i += VN) ld16_stream<T>(s_ + r0 + i, &s[i]);
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = s_[min(r0 + i, n - 1)];
    }
    if (full && perm == nullptr) {
#pragma unroll
        for (int i = 0; i < E; i += VN) {
            ld16_stream<T>(x_ + r0 + i, &xv[i]);
            ld16_stream<T>(g_ + r0 + i, &gv[i]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const int64_t r = r0 + i;
            if (r < n) {
                const int64_t row = perm ? (int64_t)perm[r] : r;
                xv[i] = x_[row];
                gv[i] = g_[row];
            } else {
                xv[i] = T(0);
                gv[i] = T(0);
            }
        }
    }
    T v[E][C], dl[E], fV[C], bW[C];
#pragma unroll
    for (int i = 0; i < E; ++i) {
        v[i][0] = xv[i];
        v[i][1] = gv[i];
        v[i][2] = xv[i];
        v[i][3] = gv[i];
    }
    chunk_aggregates<T, C, E, CT>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    block_excl_fwd<T, C, NT, CT>(s[E - 1], fV, hf, pe, pV, te, tV, smf);
    block_excl_bwd<T, C, NT, CT>(s[0], bW, hb, nf, nW, tf, tW, smb);
    if (threadIdx.x == 0) {
        const T eT = t == 0 ? s_[0] : s_[tile0 - 1];
        const T fT = tile0 + TILE < n ? s_[tile0 + TILE] : s_[n - 1];
        T acc[C], accb[C];
        onepass_carries<T, C, CT>(W, t, ntiles, tf, tW, te, tV, eT, fT, acc, accb, status);
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
    T eprev, Lprev[C], enext, Unext[C];
    apply_carry_fwd<T, C, CT>(hf, pe, pV, sh_e[0], VT, eprev, Lprev);
    apply_carry_bwd<T, C, CT>(hb, nf, nW, sh_e[1], WT, enext, Unext);
    // forward: L (exp) and P (tie) at every element
    T Lo[E][C];
    {
        T L[C];
#pragma unroll
        for (int c = 0; c < C; ++c) L[c] = Lprev[c];
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const T pv = i == 0 ? eprev : s[i - 1];
            const T de = i == 0 ? dexp<T>(eprev - s[0]) : dl[i];
            const T dt = pv == s[i] ? T(1) : T(0);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                L[c] = dfma<T>(c < 2 ? de : dt, L[c], v[i][c]);
                Lo[i][c] = L[c];
            }
        }
    }
    // backward: U (exp) and Q (tie), and the outputs
    T dxo[E], dao[E];
    {
        T U[C];
#pragma unroll
        for (int c = 0; c < C; ++c) U[c] = Unext[c];
#pragma unroll
        for (int i = E - 1; i >= 0; --i) {
            const T nx = i == E - 1 ? enext : s[i + 1];
            const T de = i == E - 1 ? dexp<T>(s[E - 1] - enext) : dl[i + 1];
            const T dt = s[i] == nx ? T(1) : T(0);
#pragma unroll
            for (int c = 0; c < C; ++c) U[c] = dfma<T>(c < 2 ? de : dt, U[c], v[i][c]);
            dxo[i] = Lo[i][1] + U[1] - gv[i];
            const T Dx = (Lo[i][0] - Lo[i][2]) - (U[0] - U[2]);
            const T Dg = (Lo[i][1] - Lo[i][3]) - (U[1] - U[3]);
            dao[i] = -(gv[i] * Dx + xv[i] * Dg);
        }
    }
    if (full && perm == nullptr) {
#pragma unroll
        for (int i = 0; i < E; i += VN) {
            st16_stream<T>(dx_ + r0 + i, &dxo[i]);
            st16_stream<T>(da_ + r0 + i, &dao[i]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const int64_t r = r0 + i;
            if (r < n) {
                const int64_t row = perm ? (int64_t)perm[r] : r;
                dx_[row] = dxo[i];
                da_[row] = dao[i];
            }
        }
    }
}

// Deferred tiles: add the suffix carry (U^x, U^g by exp(s_r - fT), Q^x, Q^g by
// [s_r == fT]) to dx and da of the tile's anchors.
template <typename T, int NT>
__global__ void __launch_bounds__(NT) k_bwd_fixup(const T* __restrict__ s_, const int32_t* __restrict__ perm,
                                                  int64_t n, const T* __restrict__ x_,
                                                  const T* __restrict__ g_, T* __restrict__ dx_,
                                                  T* __restrict__ da_, OnePassWs<T> W, int64_t tile) {
    const uint32_t nfix = W.ctrl[1];
    for (uint32_t q = blockIdx.x; q < nfix; q += gridDim.x) {
        const int64_t t = W.fix[q];
        const int64_t b = t * tile, e = min(b + tile, n);
        if (e >= n) continue;
        const T fT = s_[e];
        const T cx = W.carB[t * 4 + 0], cg = W.carB[t * 4 + 1];
        const T qx = W.carB[t * 4 + 2], qg = W.carB[t * 4 + 3];
        for (int64_t r = b + threadIdx.x; r < e; r += NT) {
            const T f = dexp<T>(s_[r] - fT);
            const T qq = s_[r] == fT ? T(1) : T(0);
            if (f == T(0) && qq == T(0)) continue;
            const int64_t row = perm ? (int64_t)perm[r] : r;
            const T dUx = f * cx, dUg = f * cg, dQx = qq * qx, dQg = qq * qg;
            dx_[row] += dUg;
            da_[row] += g_[row] * (dUx - dQx) + x_[row] * (dUg - dQg);
        }
    }
}

static constexpr int bwd_E(int es) { return es == 4 ? 8 : 4; }

size_t bwd_ws_bytes(int64_t n, int f64) {
    const int64_t tile = (int64_t)BWD_NT * bwd_E(f64 ? 8 : 4);
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    return onepass_ws_bytes(ntiles, 4, f64 ? 8 : 4);
}

template <typename T>
cudaError_t bwd_run(const T* s, const int32_t* perm, int64_t n, const T* x, const T* g, T* dx,
                    T* da, void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    constexpr int E = bwd_E((int)sizeof(T));
    const int64_t tile = (int64_t)BWD_NT * E;
    const int64_t ntiles = (n + tile - 1) / tile;
    Carve cv(ws, ws_bytes);
    OnePassWs<T> W = onepass_carve<T>(cv, ntiles, 4);
    if (!cv.ok) return cudaErrorInvalidValue;
    cudaError_t e = onepass_reset(W, ntiles, st);
    if (e != cudaSuccess) return e;
    k_bwd_onepass<T, E, BWD_NT><<<(unsigned)ntiles, BWD_NT, 0, st>>>(s, perm, n, x, g, dx, da, W,
                                                                     ntiles, status);
    k_suffix_carries<T, 4, 1024, 2><<<1, 1024, 0, st>>>(W, ntiles);
    k_bwd_fixup<T, BWD_NT><<<FIXUP_BLOCKS, BWD_NT, 0, st>>>(s, perm, n, x, g, dx, da, W, tile);
    return cudaGetLastError();
}

template cudaError_t bwd_run<float>(const float*, const int32_t*, int64_t, const float*,
                                    const float*, float*, float*, void*, size_t, uint32_t*,
                                    cudaStream_t);
template cudaError_t bwd_run<double>(const double*, const int32_t*, int64_t, const double*,
                                     const double*, double*, double*, void*, size_t, uint32_t*,
                                     cudaStream_t);

}  // namespace lx
