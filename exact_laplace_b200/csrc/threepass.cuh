// threepass.cuh -- wait-free scheme for the LAPLEX scans, generic over the
// operation (a policy) and its channels.
//
//   1. first pass, k_tp_local<P, 0> (one block per tile, register loads) or
//      k_tp_ring<P> (persistent, TMA ring; inputs in sorted order): each tile
//      is scanned with the carries from its halos, H elements on each side.
//      A carry from outside the tile reaches element r with a factor exp(-d),
//      d >= the distance from r to the tile's edge anchor, and exp(-d) is
//      exactly 0 for d >= CUT; tie factors are 0 for any d > 0.  So when both
//      halos span at least CUT (or the tile is at an end of the array) the
//      halo sums are the exact carries and the tile writes its final outputs.
//      Otherwise it writes nothing and is appended to the redo list.  Every
//      tile stores its first/last anchors and its zero-carry totals.
//   2. k_tp_carry_blocks, k_tp_carry_tiles (skipped when the list is empty):
//      the exact carries into every tile from the tile totals.
//   3. k_tp_local<P, 1>: the listed tiles again, with those carries.
// No kernel waits on another block.
//
// A policy P provides
//   using T;  static constexpr int C, CT, E, NT, H;   (CT trailing tie channels;
//                                                      halo H: 0, or a multiple
//                                                      of 32 up to a tile)
//   int64_t n;  const T* s;
//   struct Aux { ... }                                  per-thread extra state
//   __device__ void load(int64_t r0, T (&s)[E], T (&v)[E][C], Aux& a) const
//        the chunk [r0, r0 + E), padded with the last anchor and value 0
//   __device__ void load1(int64_t j, T& s, T (&v)[C]) const      one element
//   __device__ void finish(int64_t r0, const T (&s)[E], const T (&v)[E][C], T (&dl)[E],
//                          T eprev, const T (&Lp)[C], T enext, const T (&Un)[C], Aux& a) const
//        writes the outputs of the chunk from the state around it
#pragma once
#include <algorithm>

#include "bulk.cuh"
#include "devcache.h"
#include "laplex_impl.h"
#include "scan_core.cuh"

namespace lx {

constexpr int TP_CARRY_NT = 256;
constexpr int TP_CARRY_PT = 8;
constexpr int TP_CARRY_BT = TP_CARRY_NT * TP_CARRY_PT;

struct TPStats {  // reach of a tile (general product): elements within CUT of each edge
    int32_t head;
    int32_t tail;
};

template <typename T, int C>
struct TPWs {
    T* tfirst;   // [ntiles]
    T* tlast;    // [ntiles]
    T* fagg;     // [ntiles*C] L at the tile's last element, tile only
    T* bagg;     // [ntiles*C] U at the tile's first element, tile only
    TPStats* st;           // [ntiles] reach (general product)
    int32_t* redo;         // [ntiles] tiles left for the redo pass, any order
    uint32_t* redo_count;  // their number (zeroed before pass 1)
    T* bfe;      // [nb] last anchor of each carry block
    T* bfv;      // [nb*C]
    T* bbf;      // [nb] first anchor of each carry block
    T* bbv;      // [nb*C]
    T* carF;     // [ntiles*C] L at the element before tile t
    T* carB;     // [ntiles*C] U at the element after tile t
};

inline size_t tp_ws_bytes(int64_t ntiles, int C, size_t es) {
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    return 2 * Carve::need((size_t)ntiles, es) + 4 * Carve::need((size_t)(ntiles * C), es) +
           Carve::need((size_t)ntiles, sizeof(TPStats)) + Carve::need((size_t)ntiles, 4) + Carve::need(1, 4) +
           2 * Carve::need((size_t)nb, es) + 2 * Carve::need((size_t)(nb * C), es);
}

template <typename T, int C>
inline TPWs<T, C> tp_carve(Carve& cv, int64_t ntiles) {
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    TPWs<T, C> W;
    W.tfirst = cv.take<T>(ntiles);
    W.tlast = cv.take<T>(ntiles);
    W.fagg = cv.take<T>(ntiles * C);
    W.bagg = cv.take<T>(ntiles * C);
    W.st = cv.take<TPStats>(ntiles);
    W.redo = cv.take<int32_t>(ntiles);
    W.redo_count = cv.take<uint32_t>(1);
    W.bfe = cv.take<T>(nb);
    W.bfv = cv.take<T>(nb * C);
    W.bbf = cv.take<T>(nb);
    W.bbv = cv.take<T>(nb * C);
    W.carF = cv.take<T>(ntiles * C);
    W.carB = cv.take<T>(ntiles * C);
    return W;
}

// ------------------------------------------------------------------ pass 1 and 3
// Halo terms of thread q of a tile: the halo elements k = q + m NT < 2H
// (k < H: left halo, H <= k < 2H: right halo), summed per side, and the checks
// that each halo spans CUT.  A side needs no carry at an end of the array, and
// a halo that reaches the end of the array needs no check.  Contains a block
// barrier: every thread of the block calls it.
template <class P>
__device__ __forceinline__ void tp_halo_terms(const P& p, int64_t t, int64_t tile0, int64_t tile1,
                                              typename P::T (&hvL)[P::C], typename P::T (&hvU)[P::C],
                                              int (&bad)[2]) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT, H = P::H, NT = P::NT;
    const int64_t n = p.n;
    const int q = (int)threadIdx.x;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        hvL[c] = T(0);
        hvU[c] = T(0);
    }
    bad[0] = bad[1] = 0;
    if (H == 0) {
        if (q == 0) bad[0] = (t > 0 || tile1 < n) ? 1 : 0;  // no halos: final only if alone
        return;
    }
    const bool needL = t > 0, needR = tile1 < n;
    // the left halo is always in the array (tile0 >= TILE >= H); a right halo
    // cut short by the end of the array holds every element to the right.
    // Thread 0 checks from two anchors whether both halos can be exact; only
    // then are they summed (dense anchors skip the loads).
    const bool fullR = tile1 + H <= n;
    __shared__ int sh_ok;
    if (q == 0) {
        const bool okL = !needL || p.s[tile0 - 1] - p.s[tile0 - H] >= ExpCut<T>::v;
        const bool okR = !needR || !fullR || p.s[tile1 + H - 1] - p.s[tile1] >= ExpCut<T>::v;
        sh_ok = (okL ? 1 : 0) | (okR ? 2 : 0);
    }
    __syncthreads();
    const int ok = sh_ok;
    if (q == 0) {
        bad[0] = (ok & 1) ? 0 : 1;
        bad[1] = (ok & 2) ? 0 : 1;
    }
    if (ok != 3) return;
    const T eL = needL ? p.s[tile0 - 1] : T(0), eR = needR ? p.s[tile1] : T(0);
#pragma unroll
    for (int m = 0; m * NT < 2 * H; ++m) {
        const int k = q + m * NT;
        if (k >= 2 * H) break;
        const bool left = k < H;
        if (!(left ? needL : needR)) continue;
        const int64_t j = left ? tile0 - H + k : tile1 + (k - H);
        if (j >= n) continue;
        const T edge = left ? eL : eR;
        T sj, vj[C];
        p.load1(j, sj, vj);
        const Decay<T, C, CT> d = left ? Decay<T, C, CT>(sj, edge) : Decay<T, C, CT>(edge, sj);
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (left) hvL[c] += d[c] * vj[c];
            else hvU[c] += d[c] * vj[c];
        }
    }
}

// One tile.  MODE 0: carries from the halos; a tile whose halos fall short is
// listed for MODE 1 and writes nothing.  MODE 1: carries from the carry kernels.
template <class P, int MODE>
__device__ __forceinline__ void tp_tile(const P& p, const TPWs<typename P::T, P::C>& W, int64_t t,
                                        int64_t ntiles, BlockScan2Smem<typename P::T, P::C, P::NT>& sm2) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT, E = P::E, NT = P::NT, H = MODE == 0 ? P::H : 0;
    constexpr int64_t TILE = (int64_t)NT * E;
    const int64_t n = p.n;
    const int64_t tile0 = t * TILE, tile1 = min(tile0 + TILE, n);
    const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
    const bool needL = t > 0, needR = tile1 < n;
    T s[E], v[E][C];
    typename P::Aux aux;
    p.load(r0, s, v, aux);
    T hvL[C], hvU[C];
    int bad[2] = {0, 0};
#pragma unroll
    for (int c = 0; c < C; ++c) hvL[c] = hvU[c] = T(0);
    if (MODE == 0) tp_halo_terms<P>(p, t, tile0, tile1, hvL, hvU, bad);
    T dl[E], fV[C], bW[C];
    chunk_aggregates<T, C, E, CT>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    int nbad[2];
    T hL[C], hU[C];
    (void)block_excl_both_counted<T, C, NT, CT, true, 2, H, C>(
        s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf, nW, tf, tW, bad, nbad, false, sm2, hvL, hvU, hL, hU);
    bool out = true;
    T eT = hf ? pe : s[0], fT = hb ? nf : s[E - 1], Lc[C], Uc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        Lc[c] = T(0);
        Uc[c] = T(0);
    }
    if (MODE == 0) {
        out = nbad[0] == 0 && nbad[1] == 0;
        if (threadIdx.x == 0) {
            W.tfirst[t] = tf;
            W.tlast[t] = te;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                W.fagg[t * C + c] = tV[c];
                W.bagg[t * C + c] = tW[c];
            }
            if (!out) W.redo[atomicAdd(W.redo_count, 1u)] = (int32_t)t;
        }
        if (!out) return;
        if (H > 0 && needL) {
            eT = p.s[tile0 - 1];
#pragma unroll
            for (int c = 0; c < C; ++c) Lc[c] = hL[c];
        }
        if (H > 0 && needR) {
            fT = p.s[tile1];
#pragma unroll
            for (int c = 0; c < C; ++c) Uc[c] = hU[c];
        }
    } else {
        if (needL) {
            eT = p.s[tile0 - 1];
#pragma unroll
            for (int c = 0; c < C; ++c) Lc[c] = W.carF[t * C + c];
        }
        if (needR) {
            fT = p.s[tile1];
#pragma unroll
            for (int c = 0; c < C; ++c) Uc[c] = W.carB[t * C + c];
        }
    }
    T eprev, Lprev[C], enext, Unext[C];
    apply_carry_fwd<T, C, CT>(hf, pe, pV, eT, Lc, eprev, Lprev);
    apply_carry_bwd<T, C, CT>(hb, nf, nW, fT, Uc, enext, Unext);
    p.finish(r0, s, v, dl, eprev, Lprev, enext, Unext, aux);
}

// pass 1: one block per tile
template <class P>
__global__ void __launch_bounds__(P::NT) k_tp_local(P p, TPWs<typename P::T, P::C> W, int64_t ntiles) {
    __shared__ BlockScan2Smem<typename P::T, P::C, P::NT> sm2;
    tp_tile<P, 0>(p, W, (int64_t)blockIdx.x, ntiles, sm2);
}

// pass 3: the listed tiles, a grid-stride loop over the list
template <class P>
__global__ void __launch_bounds__(P::NT) k_tp_redo(P p, TPWs<typename P::T, P::C> W, int64_t ntiles) {
    __shared__ BlockScan2Smem<typename P::T, P::C, P::NT> sm2;
    const int64_t listed = (int64_t)*(volatile uint32_t*)W.redo_count;
    for (int64_t k = blockIdx.x; k < listed; k += gridDim.x) {
        tp_tile<P, 1>(p, W, (int64_t)W.redo[k], ntiles, sm2);
        __syncthreads();  // sm2 is reused by the next tile
    }
}

// ------------------------------------------------------------------ pass 1, streamed
// Persistent variant of pass 1 for inputs already in sorted order: s and the
// policy's NIN value arrays come into a shared-memory ring of S stages by 1-D
// bulk copies (TMA), each full tile with a halo of H elements on both sides
// (thread q takes the halo elements q, q + NT, ... < 2H, as in k_tp_local).  The ragged last
// tile goes through the policy's register loads.
//
// Extra policy members:
//   static constexpr int NIN, S, MINB;         (value arrays, stages, blocks/SM)
//   __device__ const T* ring_in(int a) const  value array a, sorted order
//   __device__ void value(const T (&xin)[NIN], T (&v)[C]) const   channels of one element
//   __device__ void value_chunk(const T (&xin)[NIN], T (&v)[C], Aux& a, int k) const
//        the same for element k of this thread's chunk, also filling Aux
template <class P>
__global__ void __launch_bounds__(P::NT, P::MINB) k_tp_ring(P p, TPWs<typename P::T, P::C> W,
                                                            int64_t ntiles, uint32_t* status) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT, E = P::E, NT = P::NT, S = P::S, H = P::H, NIN = P::NIN;
    constexpr int VN = V16<T>::N, NA = NIN + 1;
    constexpr int64_t TILE = (int64_t)NT * E, STAGE = TILE + 2 * H;
    static_assert(E % VN == 0, "E: whole 16-byte units");
    static_assert(H % 32 == 0 && H <= TILE, "halo: whole warps, at most a tile");
    extern __shared__ __align__(128) unsigned char dyn[];
    T* ring = reinterpret_cast<T*>(dyn);  // stage st, array a (0 = s) at ring + (st * NA + a) * STAGE
    __shared__ __align__(8) uint64_t full[S];
    __shared__ BlockScan2Smem<T, C, NT> sm2;
    const int64_t n = p.n;
    const int64_t G = gridDim.x;

    auto issue = [&](int st, int64_t t) {  // one thread
        const int64_t b = t * TILE, e = b + TILE;
        if (e <= n) {
            const int64_t hl = (H > 0 && t > 0) ? H : 0;
            const int64_t hr = (H > 0 && e + H <= n) ? H : 0;
            const int64_t lo = b - hl, cnt = hl + TILE + hr;
            const uint32_t bytes = (uint32_t)(cnt * sizeof(T));
            mbar_expect_tx(&full[st], (uint32_t)NA * bytes);
            bulk_g2s(ring + (int64_t)(st * NA) * STAGE + (H - hl), p.s + lo, bytes, &full[st]);
#pragma unroll
            for (int a = 0; a < NIN; ++a)
                bulk_g2s(ring + (int64_t)(st * NA + 1 + a) * STAGE + (H - hl), p.ring_in(a) + lo, bytes,
                         &full[st]);
        } else {
            mbar_arrive(&full[st]);  // ragged tile: register loads
        }
    };
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) mbar_init(&full[st], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int st = 0; st < S; ++st) {
            const int64_t t = blockIdx.x + st * G;
            if (t < ntiles) issue(st, t);
        }
    }
    __syncthreads();
    for (int64_t i = 0;; ++i) {
        const int64_t t = blockIdx.x + i * G;
        if (t >= ntiles) break;
        const int st = (int)(i % S);
        const bool landed = mbar_wait(&full[st], (uint32_t)((i / S) & 1));
        const int64_t tile0 = t * TILE, tile1 = min(tile0 + TILE, n);
        const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
        const bool ragged = tile0 + TILE > n;
        const bool needL = t > 0, needR = tile1 < n;
        const T* S0 = ring + (int64_t)(st * NA) * STAGE;  // [left halo | tile | right halo]
        T s[E], v[E][C];
        typename P::Aux aux;
        if (!landed) {  // reported at the block scan's first barrier
#pragma unroll
            for (int k = 0; k < E; ++k) {
                s[k] = T(0);
#pragma unroll
                for (int c = 0; c < C; ++c) v[k][c] = T(0);
            }
        } else if (!ragged) {
#pragma unroll
            for (int k = 0; k < E; k += VN) ld16<T>(S0 + H + threadIdx.x * E + k, &s[k]);
            T xin[NIN][E];
#pragma unroll
            for (int a = 0; a < NIN; ++a)
#pragma unroll
                for (int k = 0; k < E; k += VN) ld16<T>(S0 + (a + 1) * STAGE + H + threadIdx.x * E + k, &xin[a][k]);
#pragma unroll
            for (int k = 0; k < E; ++k) {
                T xe[NIN];
#pragma unroll
                for (int a = 0; a < NIN; ++a) xe[a] = xin[a][k];
                p.value_chunk(xe, v[k], aux, k);
            }
        } else {
            p.load(r0, s, v, aux);
        }
        // halo terms of this thread (elements k = q + m NT < 2H), the span
        // checks, the edge anchors.  A halo comes from the ring when the copy
        // brought it, else through the policy's single-element load (the
        // ragged last tile; a right halo cut short by the end of the array,
        // which then holds every element to the right and needs no check).
        T hvL[C], hvU[C], ringL = T(0), ringR = T(0);
        int bad[2] = {0, 0};
#pragma unroll
        for (int c = 0; c < C; ++c) hvL[c] = hvU[c] = T(0);
        {
            const int q = (int)threadIdx.x;
            const bool fullR = tile1 + H <= n;
            const bool ringH = !ragged;
            if (H == 0) {
                if (q == 0) bad[0] = (needL || needR) ? 1 : 0;
            } else if (landed) {
                if (needL) ringL = ringH ? S0[H - 1] : p.s[tile0 - 1];
                if (needR) ringR = ringH && fullR ? S0[H + TILE] : p.s[tile1];
#pragma unroll
                for (int m = 0; m * NT < 2 * H; ++m) {
                    const int k = q + m * NT;
                    if (k >= 2 * H) break;
                    const bool left = k < H;
                    if (!(left ? needL : needR)) continue;
                    const int64_t jg = left ? tile0 - H + k : tile1 + (k - H);
                    if (!left && jg >= n) continue;
                    const bool inring = ringH && (left || fullR);
                    const int j = left ? k : (int)TILE + k;  // ring index
                    const T edge = left ? ringL : ringR;
                    T sj, vj[C];
                    if (inring) {
                        sj = S0[j];
                        T xe[NIN];
#pragma unroll
                        for (int a = 0; a < NIN; ++a) xe[a] = S0[(a + 1) * STAGE + j];
                        p.value(xe, vj);
                    } else {
                        p.load1(jg, sj, vj);
                    }
                    const Decay<T, C, CT> d = left ? Decay<T, C, CT>(sj, edge) : Decay<T, C, CT>(edge, sj);
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        if (left) hvL[c] += d[c] * vj[c];
                        else hvU[c] += d[c] * vj[c];
                    }
                    if (k == 0) bad[0] = edge - sj >= ExpCut<T>::v ? 0 : 1;
                    if (k == H && fullR)
                        bad[1] = (inring ? S0[2 * H + TILE - 1] : p.s[tile1 + H - 1]) - edge >= ExpCut<T>::v ? 0 : 1;
                }
            }
        }
        // this thread's reads of stage st are ordered before the TMA writes
        // that refill it, issued after the block scan's barriers
        fence_proxy_async();
        T dl[E], fV[C], bW[C];
        chunk_aggregates<T, C, E, CT>(s, v, dl, fV, bW);
        bool hf, hb;
        T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
        int nbad[2];
        T hL[C], hU[C];
        if (block_excl_both_counted<T, C, NT, CT, true, 2, H, C>(
                s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf, nW, tf, tW, bad, nbad, !landed, sm2, hvL,
                hvU, hL, hU)) {
            // a copy never completed: report, let the copies in flight land, stop
            if (threadIdx.x == 0) {
                set_status(status, ST_TIMEOUT);
                for (int k = 0; k < S; ++k) {
                    const int64_t t2 = blockIdx.x + (i + k) * G;
                    if (t2 < ntiles) mbar_wait(&full[(i + k) % S], (uint32_t)(((i + k) / S) & 1));
                }
            }
            return;
        }
        const bool out = nbad[0] == 0 && nbad[1] == 0;
        if (threadIdx.x == 0) {
            const int64_t t2 = t + S * G;
            if (t2 < ntiles) issue(st, t2);
            W.tfirst[t] = tf;
            W.tlast[t] = te;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                W.fagg[t * C + c] = tV[c];
                W.bagg[t * C + c] = tW[c];
            }
            if (!out) W.redo[atomicAdd(W.redo_count, 1u)] = (int32_t)t;
        }
        if (!out) continue;
        T eT = hf ? pe : s[0], fT = hb ? nf : s[E - 1], Lc[C], Uc[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            Lc[c] = needL ? hL[c] : T(0);
            Uc[c] = needR ? hU[c] : T(0);
        }
        if (needL) eT = ringL;
        if (needR) fT = ringR;
        T eprev, Lprev[C], enext, Unext[C];
        apply_carry_fwd<T, C, CT>(hf, pe, pV, eT, Lc, eprev, Lprev);
        apply_carry_bwd<T, C, CT>(hb, nf, nW, fT, Uc, enext, Unext);
        p.finish(r0, s, v, dl, eprev, Lprev, enext, Unext, aux);
    }
}

// ------------------------------------------------------------------ pass 2
// The records of a thread's TP_CARRY_PT consecutive tiles, loaded at once (the
// loads are independent; entries past the last tile are 0 and never used).
// Only the thread's own tiles are read, so k_tp_carry_tiles may write the
// carries over the totals (carF == fagg, carB == bagg), as the fixed-scratch
// product does.
template <typename T, int C>
struct TPSeg {
    T tl[TP_CARRY_PT], tf[TP_CARRY_PT];
    T fa[TP_CARRY_PT][C], ba[TP_CARRY_PT][C];
    __device__ __forceinline__ void load(const TPWs<T, C>& W, int64_t t0, int64_t ntiles) {
#pragma unroll
        for (int k = 0; k < TP_CARRY_PT; ++k) {
            const int64_t t = t0 + k;
            const bool in = t < ntiles;  // only this thread's own tiles are read
            tl[k] = in ? W.tlast[t] : T(0);
            tf[k] = in ? W.tfirst[t] : T(0);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                fa[k][c] = in ? W.fagg[t * C + c] : T(0);
                ba[k][c] = in ? W.bagg[t * C + c] : T(0);
            }
        }
    }
};

// The thread's segment summaries: forward (fe, fv) and backward (bf, bv);
// a thread with no tile holds the neutral summary (the last anchor, 0).
template <typename T, int C, int CT>
__device__ __forceinline__ void tp_segment(const TPSeg<T, C>& g, int64_t t0, int64_t ntiles, T pad, T& fe,
                                           T (&fv)[C], T& bf, T (&bv)[C]) {
    fe = pad;
    bf = pad;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        fv[c] = T(0);
        bv[c] = T(0);
    }
    bool any = false;
#pragma unroll
    for (int k = 0; k < TP_CARRY_PT; ++k) {
        if (t0 + k >= ntiles) break;
        const T e = g.tl[k];
        const Decay<T, C, CT> d(fe, e);
#pragma unroll
        for (int c = 0; c < C; ++c) fv[c] = dfma<T>(any ? d[c] : T(0), fv[c], g.fa[k][c]);
        fe = e;
        any = true;
    }
    any = false;
#pragma unroll
    for (int k = TP_CARRY_PT - 1; k >= 0; --k) {
        if (t0 + k >= ntiles) continue;
        const T f = g.tf[k];
        const Decay<T, C, CT> d(f, bf);
#pragma unroll
        for (int c = 0; c < C; ++c) bv[c] = dfma<T>(any ? d[c] : T(0), bv[c], g.ba[k][c]);
        bf = f;
        any = true;
    }
}

template <typename T, int C, int CT>
__global__ void __launch_bounds__(TP_CARRY_NT) k_tp_carry_blocks(TPWs<T, C> W, int64_t ntiles) {
    if (*(volatile uint32_t*)W.redo_count == 0) return;  // every tile final
    __shared__ BlockScan2Smem<T, C, TP_CARRY_NT> sm2;
    const int64_t t0 = (int64_t)blockIdx.x * TP_CARRY_BT + (int64_t)threadIdx.x * TP_CARRY_PT;
    TPSeg<T, C> g;
    g.load(W, t0, ntiles);
    T fe, fv[C], bf, bv[C];
    tp_segment<T, C, CT>(g, t0, ntiles, W.tlast[ntiles - 1], fe, fv, bf, bv);
    bool hf, hb;
    T pe, pv[C], te, tv[C], nf, nv[C], tf, tw[C];
    block_excl_both<T, C, TP_CARRY_NT, CT>(fe, fv, bf, bv, hf, pe, pv, te, tv, hb, nf, nv, tf, tw, sm2);
    if (threadIdx.x == 0) {
        W.bfe[blockIdx.x] = te;
        W.bbf[blockIdx.x] = tf;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            W.bfv[blockIdx.x * C + c] = tv[c];
            W.bbv[blockIdx.x * C + c] = tw[c];
        }
    }
}

template <typename T, int C, int CT>
__global__ void __launch_bounds__(TP_CARRY_NT) k_tp_carry_tiles(TPWs<T, C> W, int64_t ntiles,
                                                                 int64_t nblocks) {
    if (*(volatile uint32_t*)W.redo_count == 0) return;  // every tile final
    __shared__ BlockScan2Smem<T, C, TP_CARRY_NT> sm2;
    __shared__ T sh_c[2][C];
    const int64_t bidx = blockIdx.x;
    if (threadIdx.x == 0) {
        // carries into this block from the block totals: direct decays from the
        // block's own edge anchor, stopping where every factor is exactly 0
        T acc[C], accb[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            acc[c] = T(0);
            accb[c] = T(0);
        }
        if (bidx > 0) {
            const T eb = W.bfe[bidx - 1];
            for (int64_t j = bidx - 1; j >= 0; --j) {
                const Decay<T, C, CT> d(W.bfe[j], eb);
                if (d.e == T(0) && (CT == 0 || d.t == T(0))) break;
#pragma unroll
                for (int c = 0; c < C; ++c) acc[c] = dfma<T>(d[c], W.bfv[j * C + c], acc[c]);
            }
        }
        if (bidx + 1 < nblocks) {
            const T fb = W.bbf[bidx + 1];
            for (int64_t j = bidx + 1; j < nblocks; ++j) {
                const Decay<T, C, CT> d(fb, W.bbf[j]);
                if (d.e == T(0) && (CT == 0 || d.t == T(0))) break;
#pragma unroll
                for (int c = 0; c < C; ++c) accb[c] = dfma<T>(d[c], W.bbv[j * C + c], accb[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < C; ++c) {
            sh_c[0][c] = acc[c];
            sh_c[1][c] = accb[c];
        }
    }
    const int64_t t0 = bidx * TP_CARRY_BT + (int64_t)threadIdx.x * TP_CARRY_PT;
    TPSeg<T, C> g;
    g.load(W, t0, ntiles);
    T fe, fv[C], bf, bv[C];
    tp_segment<T, C, CT>(g, t0, ntiles, W.tlast[ntiles - 1], fe, fv, bf, bv);
    bool hf, hb;
    T pe, pv[C], te, tv[C], nf, nv[C], tf, tw[C];
    block_excl_both<T, C, TP_CARRY_NT, CT>(fe, fv, bf, bv, hf, pe, pv, te, tv, hb, nf, nv, tf, tw,
                                           sm2);  // barriers publish sh_c
    // forward: carry at the end of the previous tile
    const T eBlk = bidx > 0 ? W.bfe[bidx - 1] : W.tlast[0];
    T ce, cv[C];
    if (hf) {
        ce = pe;
        const Decay<T, C, CT> d(eBlk, pe);
#pragma unroll
        for (int c = 0; c < C; ++c) cv[c] = dfma<T>(d[c], sh_c[0][c], pv[c]);
    } else {
        ce = eBlk;
#pragma unroll
        for (int c = 0; c < C; ++c) cv[c] = sh_c[0][c];
    }
#pragma unroll
    for (int k = 0; k < TP_CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
#pragma unroll
        for (int c = 0; c < C; ++c) W.carF[t * C + c] = t == 0 ? T(0) : cv[c];
        const T e = g.tl[k];
        const Decay<T, C, CT> d(ce, e);
#pragma unroll
        for (int c = 0; c < C; ++c) cv[c] = dfma<T>(d[c], cv[c], g.fa[k][c]);
        ce = e;
    }
    const T fBlk = bidx + 1 < nblocks ? W.bbf[bidx + 1] : W.tlast[ntiles - 1];
    T cf, cw[C];
    if (hb) {
        cf = nf;
        const Decay<T, C, CT> d(nf, fBlk);
#pragma unroll
        for (int c = 0; c < C; ++c) cw[c] = dfma<T>(d[c], sh_c[1][c], nv[c]);
    } else {
        cf = fBlk;
#pragma unroll
        for (int c = 0; c < C; ++c) cw[c] = sh_c[1][c];
    }
#pragma unroll
    for (int k = TP_CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
#pragma unroll
        for (int c = 0; c < C; ++c) W.carB[t * C + c] = t == ntiles - 1 ? T(0) : cw[c];
        const T f = g.tf[k];
        const Decay<T, C, CT> d(f, cf);
#pragma unroll
        for (int c = 0; c < C; ++c) cw[c] = dfma<T>(d[c], cw[c], g.ba[k][c]);
        cf = f;
    }
}

template <class P>
inline int64_t tp_ntiles(int64_t n) {
    const int64_t tile = (int64_t)P::NT * P::E;
    return std::max<int64_t>(1, (n + tile - 1) / tile);
}

// Passes 2 and 3 after pass 1 (shared by tp_run and tp_run_ring).
template <class P>
cudaError_t tp_finish(const P& p, TPWs<typename P::T, P::C> W, int64_t ntiles, int sms, cudaStream_t st) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT;
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    // the per-block totals are read only when there is more than one carry block
    if (nb > 1) k_tp_carry_blocks<T, C, CT><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles);
    k_tp_carry_tiles<T, C, CT><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles, nb);
    const int64_t rb = std::max<int64_t>(1, std::min<int64_t>(ntiles, (int64_t)sms * 4));
    k_tp_redo<P><<<(unsigned)rb, P::NT, 0, st>>>(p, W, ntiles);
    return cudaGetLastError();
}

inline cudaError_t tp_sm_count(int& dev, int& sms) { return current_device_sms(&dev, &sms); }

// The streamed pass 1 (k_tp_ring) for inputs in sorted order, then passes 2-3.
template <class P>
cudaError_t tp_run_ring(const P& p, void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    using T = typename P::T;
    constexpr int C = P::C;
    if (p.n == 0) return cudaSuccess;
    const int64_t ntiles = tp_ntiles<P>(p.n);
    Carve cv(ws, ws_bytes);
    TPWs<T, C> W = tp_carve<T, C>(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = tp_sm_count(dev, sms);
    if (e != cudaSuccess) return e;
    constexpr size_t smem = (size_t)P::S * (P::NIN + 1) * ((size_t)P::NT * P::E + 2 * P::H) * sizeof(T);
    int per_sm = 0;  // resident blocks per SM, cached per device
    e = blocks_per_sm<k_tp_ring<P>>(dev, P::NT, smem, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ntiles, (int64_t)per_sm * sms);
    e = cudaMemsetAsync(W.redo_count, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    profile_before(st);
    k_tp_ring<P><<<(unsigned)grid, P::NT, smem, st>>>(p, W, ntiles, status);
    profile_after(st);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return tp_finish(p, W, ntiles, sms, st);
}

template <class P>
cudaError_t tp_run(const P& p, void* ws, size_t ws_bytes, cudaStream_t st) {
    using T = typename P::T;
    constexpr int C = P::C;
    if (p.n == 0) return cudaSuccess;
    const int64_t ntiles = tp_ntiles<P>(p.n);
    Carve cv(ws, ws_bytes);
    TPWs<T, C> W = tp_carve<T, C>(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = tp_sm_count(dev, sms);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(W.redo_count, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    profile_before(st);
    k_tp_local<P><<<(unsigned)ntiles, P::NT, 0, st>>>(p, W, ntiles);
    profile_after(st);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return tp_finish(p, W, ntiles, sms, st);
}

}  // namespace lx
