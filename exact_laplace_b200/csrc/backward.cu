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
// (scan_core.cuh "tie channels").  One scan of four channels (x, g with exp
// decay; x, g with tie decay) reads s, x, g once and writes dx, da once
// (20 bytes per anchor in fp32), in the wait-free scheme of threepass.cuh.
#include <algorithm>

#include "laplex_impl.h"
#include "threepass.cuh"

namespace lx {

// elements per thread (fp32: LX_BWD_E32) and resident blocks per SM of the ring pass
#ifndef LX_BWD_E32
#define LX_BWD_E32 12
#endif
#ifndef LX_BWD_MINB
#define LX_BWD_MINB 2
#endif
#ifndef LX_BWD_S
#define LX_BWD_S 2
#endif
constexpr int BWD_NT = 256;

// Policy of threepass.cuh (wait-free: tile-local scans, exact tile carries,
// carries added to the heads and tails of the tiles).  Channels: x and g with
// exp decay (L, U), then x and g with tie decay (P, Q).
template <typename T_, int E_>
struct BwdTP {
    using T = T_;
    static constexpr int C = 4, CT = 2, E = E_, NT = BWD_NT;
    // halos of 192 (fp32: they span CUT = 88 at spacings above 0.47, and
    // across runs of up to 64 equal anchors; fp64, CUT = 746, would need
    // several times more: none).  Streamed pass 1 (inputs in sorted order):
    // s, x, g in a 2-stage ring.
    static constexpr int H = sizeof(T_) == 4 ? 192 : 0;
    static constexpr int NIN = 2, S = LX_BWD_S, MINB = LX_BWD_MINB;
    int64_t n;
    const T* s;
    const int32_t* perm;
    const T* x;
    const T* g;
    T* dx;
    T* da;
    struct Aux {};
    __device__ __forceinline__ void load(int64_t r0, T (&sv)[E], T (&v)[E][C], Aux&) const {
        constexpr int VN = V16<T>::N;
        const bool full = r0 + E <= n;
        T xv[E], gv[E];
        if (full) {
#pragma unroll
            for (int i = 0; i < E; i += VN) ld16_stream<T>(s + r0 + i, &sv[i]);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) sv[i] = s[min(r0 + i, n - 1)];
        }
        if (full && perm == nullptr) {
#pragma unroll
            for (int i = 0; i < E; i += VN) {
                ld16_stream<T>(x + r0 + i, &xv[i]);
                ld16_stream<T>(g + r0 + i, &gv[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const int64_t r = r0 + i;
                const int64_t row = r < n ? (perm ? (int64_t)perm[r] : r) : 0;
                xv[i] = r < n ? x[row] : T(0);
                gv[i] = r < n ? g[row] : T(0);
            }
        }
#pragma unroll
        for (int i = 0; i < E; ++i) {
            v[i][0] = xv[i];
            v[i][1] = gv[i];
            v[i][2] = xv[i];
            v[i][3] = gv[i];
        }
    }
    __device__ __forceinline__ const T* ring_in(int a) const { return a == 0 ? x : g; }
    __device__ __forceinline__ void value(const T (&xe)[NIN], T (&vv)[C]) const {
        vv[0] = xe[0];
        vv[1] = xe[1];
        vv[2] = xe[0];
        vv[3] = xe[1];
    }
    __device__ __forceinline__ void value_chunk(const T (&xe)[NIN], T (&vv)[C], Aux&, int) const { value(xe, vv); }
    __device__ __forceinline__ void finish(int64_t r0, const T (&sv)[E], const T (&v)[E][C],
                                           T (&dl)[E], T eprev, const T (&Lp)[C], T enext,
                                           const T (&Un)[C], Aux&) const {
        constexpr int VN = V16<T>::N;
        T Lo[E][C];
        {
            T L[C];
#pragma unroll
            for (int c = 0; c < C; ++c) L[c] = Lp[c];
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const T pv = i == 0 ? eprev : sv[i - 1];
                const T de = i == 0 ? dexp<T>(eprev - sv[0]) : dl[i];
                const T dt = pv == sv[i] ? T(1) : T(0);
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    L[c] = dfma<T>(c < 2 ? de : dt, L[c], v[i][c]);
                    Lo[i][c] = L[c];
                }
            }
        }
        T dxo[E], dao[E];
        {
            T U[C];
#pragma unroll
            for (int c = 0; c < C; ++c) U[c] = Un[c];
#pragma unroll
            for (int i = E - 1; i >= 0; --i) {
                const T nx = i == E - 1 ? enext : sv[i + 1];
                const T de = i == E - 1 ? dexp<T>(sv[E - 1] - enext) : dl[i + 1];
                const T dt = sv[i] == nx ? T(1) : T(0);
#pragma unroll
                for (int c = 0; c < C; ++c) U[c] = dfma<T>(c < 2 ? de : dt, U[c], v[i][c]);
                dxo[i] = Lo[i][1] + U[1] - v[i][1];
                const T Dx = (Lo[i][0] - Lo[i][2]) - (U[0] - U[2]);
                const T Dg = (Lo[i][1] - Lo[i][3]) - (U[1] - U[3]);
                dao[i] = -(v[i][1] * Dx + v[i][0] * Dg);
            }
        }
        if (r0 + E <= n && perm == nullptr) {
#pragma unroll
            for (int i = 0; i < E; i += VN) {
                st16_stream<T>(dx + r0 + i, &dxo[i]);
                st16_stream<T>(da + r0 + i, &dao[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const int64_t r = r0 + i;
                if (r < n) {
                    const int64_t row = perm ? (int64_t)perm[r] : r;
                    dx[row] = dxo[i];
                    da[row] = dao[i];
                }
            }
        }
    }
    __device__ __forceinline__ void load1(int64_t j, T& sj, T (&vv)[C]) const {
        sj = s[j];
        const int64_t row = perm ? (int64_t)perm[j] : j;
        const T xe[NIN] = {x[row], g[row]};
        value(xe, vv);
    }
};

static constexpr int bwd_E(int es) { return es == 4 ? LX_BWD_E32 : 4; }

size_t bwd_ws_bytes(int64_t n, int f64) {
    const int64_t tile = (int64_t)BWD_NT * bwd_E(f64 ? 8 : 4);
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    return tp_ws_bytes(ntiles, 4, f64 ? 8 : 4);
}

template <typename T>
cudaError_t bwd_run(const T* s, const int32_t* perm, int64_t n, const T* x, const T* g, T* dx,
                    T* da, void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    BwdTP<T, bwd_E((int)sizeof(T))> p;
    p.n = n;
    p.s = s;
    p.perm = perm;
    p.x = x;
    p.g = g;
    p.dx = dx;
    p.da = da;
    if (perm == nullptr) return tp_run_ring(p, ws, ws_bytes, status, st);
    return tp_run(p, ws, ws_bytes, st);
}

template cudaError_t bwd_run<float>(const float*, const int32_t*, int64_t, const float*,
                                    const float*, float*, float*, void*, size_t, uint32_t*,
                                    cudaStream_t);
template cudaError_t bwd_run<double>(const double*, const int32_t*, int64_t, const double*,
                                     const double*, double*, double*, void*, size_t, uint32_t*,
                                     cudaStream_t);

}  // namespace lx
