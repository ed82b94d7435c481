// cols.cuh -- the symmetric product y = K x with B columns ("LAPLEX - La FFT
// dei Nuclei di Laplace Apprendibili", technical summary §2.2 "Caso
// Simmetrico", applied to every column of x), for x, y row-major [n, B] in
// sorted order, B in {2, 4, 8, 16, 32}.
//
// Column-parallel layout: a warp holds 32 / B runs of E consecutive rows, each
// run spread over B lanes, one column per lane.  A lane's sequential
// recurrences carry one column, so the scans between runs move one value per
// lane (shuffles at stride B inside the warp, shared memory across warps)
// instead of B values per thread; a warp's loads of x fetch whole rows (B
// consecutive values per run).  Every lane evaluates the decays of its rows
// (B-fold redundant exponentials, cheap next to the memory traffic).
//
// Three launches, exact for any anchor density (no halos):
//   k_cols<.., false>  per tile, the zero-carry forward total at its last row
//                      and backward total at its first row, per column
//   k_tp_carry_blocks, k_tp_carry_tiles   the exact carries into every tile
//                      (threepass.cuh, from the tiles' edge anchors and totals)
//   k_cols<.., true>   the tile again with its carries: y = L + U - x
//
// Included by sym.cu.
#pragma once
#include <algorithm>

#include "common.cuh"
#include "laplex_impl.h"
#include "scan_core.cuh"
#include "threepass.cuh"

namespace lx {

#ifndef LX_COLS_NT
#define LX_COLS_NT 256
#endif
constexpr int COLS_NT = LX_COLS_NT;  // 256 measured faster than 512 at n = 2^24, B = 8
constexpr int COLS_NW = COLS_NT / 32;

template <typename T> struct ColsE;
template <> struct ColsE<float> { static constexpr int E = 16; };
template <> struct ColsE<double> { static constexpr int E = 8; };

// Forward pair (anchor, value): the value is a decayed sum at the anchor.
// (e1, v1) then (e2, v2) -> (e2, v1 exp(e1 - e2) + v2); the backward mirror
// keeps the earlier anchor: (f1, w1) after (f2, w2) -> (f1, w2 exp(f1 - f2) + w1).
template <typename T>
__device__ __forceinline__ void fwd_join(T e1, T v1, T& e2, T& v2) {
    v2 = dfma<T>(dexp<T>(e1 - e2), v1, v2);
}
template <typename T>
__device__ __forceinline__ void bwd_join(T& f1, T& w1, T f2, T w2) {
    w1 = dfma<T>(dexp<T>(f1 - f2), w2, w1);
}

template <typename T, int B, int E, bool FINAL>
__global__ void __launch_bounds__(COLS_NT) k_cols(const T* __restrict__ s, int64_t n, const T* __restrict__ x,
                                                  T* __restrict__ y, TPWs<T, B> W) {
    constexpr int RPW = 32 / B;              // runs per warp
    constexpr int NR = COLS_NW * RPW;        // runs per tile
    constexpr int64_t TILE = (int64_t)NR * E;
    constexpr int VN = V16<T>::N;
    static_assert(32 % B == 0 && E % VN == 0, "B divides 32; E whole 16-byte units");
    __shared__ T wfe[COLS_NW][B], wfv[COLS_NW][B], wbf[COLS_NW][B], wbv[COLS_NW][B];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c = lane % B, rw = lane / B;   // column, run within the warp
    const int64_t t = blockIdx.x, tile0 = t * TILE;
    const int64_t r0 = tile0 + (int64_t)(w * RPW + rw) * E;
    // rows of this run (past the end: the last anchor, value 0)
    T sv[E], xv[E];
    if (r0 + E <= n) {
#pragma unroll
        for (int i = 0; i < E; i += VN) ld16<T>(s + r0 + i, &sv[i]);
#pragma unroll
        for (int i = 0; i < E; ++i) xv[i] = x[(r0 + i) * B + c];
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const int64_t r = r0 + i;
            sv[i] = s[min(r, n - 1)];
            xv[i] = r < n ? x[r * B + c] : T(0);
        }
    }
    // decays inside the run and the run's zero-carry totals
    T dl[E];
    dl[0] = T(1);
#pragma unroll
    for (int i = 1; i < E; ++i) dl[i] = dexp<T>(sv[i - 1] - sv[i]);
    T F = xv[0];
#pragma unroll
    for (int i = 1; i < E; ++i) F = dfma<T>(dl[i], F, xv[i]);
    T G = xv[E - 1];
#pragma unroll
    for (int i = E - 2; i >= 0; --i) G = dfma<T>(dl[i + 1], G, xv[i]);
    // inclusive scans over the warp's runs of this column (lanes at stride B)
    T fe = sv[E - 1], fv = F, bf = sv[0], bv = G;
#pragma unroll
    for (int off = 1; off < RPW; off <<= 1) {
        const T oe = __shfl_up_sync(FULL, fe, off * B), ov = __shfl_up_sync(FULL, fv, off * B);
        const T of = __shfl_down_sync(FULL, bf, off * B), ow = __shfl_down_sync(FULL, bv, off * B);
        if (rw >= off) fwd_join<T>(oe, ov, fe, fv);
        if (rw + off < RPW) bwd_join<T>(bf, bv, of, ow);
    }
    // exclusive (forward) and exclusive-from-the-right (backward) within the warp
    T pe = __shfl_up_sync(FULL, fe, B), pv = __shfl_up_sync(FULL, fv, B);
    T nf = __shfl_down_sync(FULL, bf, B), nw = __shfl_down_sync(FULL, bv, B);
    bool hasP = rw > 0, hasN = rw + 1 < RPW;
    // warp totals of this column: the last run's inclusive forward, the first run's backward
    if (rw == RPW - 1) {
        wfe[w][c] = fe;
        wfv[w][c] = fv;
    }
    if (rw == 0) {
        wbf[w][c] = bf;
        wbv[w][c] = bv;
    }
    __syncthreads();
    // the earlier warps' forward totals and the later warps' backward totals
    {
        bool h = false;
        T ae = T(0), av = T(0);
        for (int ww = 0; ww < w; ++ww) {
            if (h) {
                T e2 = wfe[ww][c], v2 = wfv[ww][c];
                fwd_join<T>(ae, av, e2, v2);
                ae = e2;
                av = v2;
            } else {
                ae = wfe[ww][c];
                av = wfv[ww][c];
                h = true;
            }
        }
        if (h) {
            if (hasP) fwd_join<T>(ae, av, pe, pv);
            else {
                pe = ae;
                pv = av;
            }
            hasP = true;
        }
        h = false;
        T af = T(0), aw = T(0);
        for (int ww = COLS_NW - 1; ww > w; --ww) {
            if (h) {
                T f1 = wbf[ww][c], w1 = wbv[ww][c];
                bwd_join<T>(f1, w1, af, aw);
                af = f1;
                aw = w1;
            } else {
                af = wbf[ww][c];
                aw = wbv[ww][c];
                h = true;
            }
        }
        if (h) {
            if (hasN) bwd_join<T>(nf, nw, af, aw);
            else {
                nf = af;
                nw = aw;
            }
            hasN = true;
        }
    }
    if constexpr (!FINAL) {
        // the tile's totals: thread of the last run (forward), of the first run (backward)
        if (w == COLS_NW - 1 && rw == RPW - 1) {
            T te = pe, tv = pv;
            if (hasP) {
                T e2 = sv[E - 1], v2 = F;
                fwd_join<T>(te, tv, e2, v2);
                tv = v2;
            } else {
                tv = F;
            }
            W.fagg[t * B + c] = tv;
        }
        if (w == 0 && rw == 0) {
            T f1 = sv[0], w1 = G;
            if (hasN) bwd_join<T>(f1, w1, nf, nw);
            W.bagg[t * B + c] = w1;
        }
        if (threadIdx.x == 0) {
            W.tfirst[t] = s[tile0];
            W.tlast[t] = s[min(tile0 + TILE, n) - 1];
        }
    } else {
        // carries into the tile: L at the row before it, U at the row after it
        const int64_t ntiles = (n + TILE - 1) / TILE;
        if (t > 0) {
            const T eT = s[tile0 - 1], cv = W.carF[t * B + c];
            if (hasP) {
                fwd_join<T>(eT, cv, pe, pv);
            } else {
                pe = eT;
                pv = cv;
                hasP = true;
            }
        }
        if (t < ntiles - 1) {
            const T fT = s[tile0 + TILE], cw = W.carB[t * B + c];
            if (hasN) {
                T f1 = nf, w1 = nw;
                bwd_join<T>(f1, w1, fT, cw);
                nw = w1;
            } else {
                nf = fT;
                nw = cw;
                hasN = true;
            }
        }
        // the run's outputs: L forward, then U backward and y = L + U - x
        T L[E];
        T acc = hasP ? dexp<T>(pe - sv[0]) * pv : T(0);
        L[0] = acc + xv[0];
#pragma unroll
        for (int i = 1; i < E; ++i) L[i] = dfma<T>(dl[i], L[i - 1], xv[i]);
        T U = (hasN ? dexp<T>(sv[E - 1] - nf) * nw : T(0)) + xv[E - 1];
        T out[E];
        out[E - 1] = L[E - 1] + U - xv[E - 1];
#pragma unroll
        for (int i = E - 2; i >= 0; --i) {
            U = dfma<T>(dl[i + 1], U, xv[i]);
            out[i] = L[i] + U - xv[i];
        }
        if (r0 + E <= n) {
#pragma unroll
            for (int i = 0; i < E; ++i) y[(r0 + i) * B + c] = out[i];
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i)
                if (r0 + i < n) y[(r0 + i) * B + c] = out[i];
        }
    }
}

// ------------------------------------------------------------------ host side
template <typename T, int B>
constexpr int64_t cols_tile() { return (int64_t)COLS_NW * (32 / B) * ColsE<T>::E; }

inline bool cols_supported(int64_t B) { return B == 2 || B == 4 || B == 8; }

inline size_t cols_ws_bytes(int64_t n, int64_t B, int f64) {
    if (!cols_supported(B)) return 0;
    const int64_t tile = (int64_t)COLS_NW * (32 / B) * (f64 ? ColsE<double>::E : ColsE<float>::E);
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    return tp_ws_bytes(ntiles, (int)B, f64 ? 8 : 4);
}

template <typename T, int B>
cudaError_t cols_launch(const T* s, int64_t n, const T* x, T* y, void* ws, size_t ws_bytes, cudaStream_t st) {
    constexpr int E = ColsE<T>::E;
    constexpr int64_t TILE = cols_tile<T, B>();
    const int64_t ntiles = (n + TILE - 1) / TILE;
    Carve cv(ws, ws_bytes);
    TPWs<T, B> W = tp_carve<T, B>(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    cudaError_t e = cudaMemsetAsync(W.redo_count, 1, sizeof(uint32_t), st);  // the carry kernels always run
    if (e != cudaSuccess) return e;
    profile_before(st);
    k_cols<T, B, E, false><<<(unsigned)ntiles, COLS_NT, 0, st>>>(s, n, x, y, W);
    // the per-block totals are read only when there is more than one carry block
    if (nb > 1) k_tp_carry_blocks<T, B, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles);
    k_tp_carry_tiles<T, B, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles, nb);
    k_cols<T, B, E, true><<<(unsigned)ntiles, COLS_NT, 0, st>>>(s, n, x, y, W);
    profile_after(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t cols_run(const T* s, int64_t n, const T* x, T* y, int64_t B, void* ws, size_t ws_bytes,
                     cudaStream_t st) {
    switch (B) {
        case 2: return cols_launch<T, 2>(s, n, x, y, ws, ws_bytes, st);
        case 4: return cols_launch<T, 4>(s, n, x, y, ws, ws_bytes, st);
        default: return cols_launch<T, 8>(s, n, x, y, ws, ws_bytes, st);
    }
}

}  // namespace lx
