// threepass.cuh -- wait-free three-kernel scheme for the LAPLEX scans, generic
// over the operation (a policy) and its channels.
//
//   1. k_tp_local: one block per tile; the policy loads the tile (with any
//      gather through perm), the tile is scanned with zero carries from outside
//      and the policy writes its outputs.  The tile's first/last anchors, its
//      forward/backward totals (C channels) and its reach (elements within CUT
//      of either end anchor) go to the workspace.
//   2. k_tp_carry_blocks, k_tp_carry_tiles: exact carries into every tile.
//   3. k_tp_headtail: the policy adds the carries to the elements in each
//      tile's head and tail reach.  Beyond the reach every carry factor is
//      exactly 0 (exp of a gap >= CUT underflows; tie factors are 0 for any
//      gap > 0), so the result equals adding them everywhere.
// No kernel waits on another block.
//
// A policy P provides
//   using T;  static constexpr int C, CT, E, NT;   (CT trailing tie channels)
//   int64_t n;  const T* s;
//   struct Aux { ... }                                  per-thread extra state
//   __device__ void load(int64_t r0, T (&s)[E], T (&v)[E][C], Aux& a) const
//   __device__ void finish(int64_t r0, const T (&s)[E], const T (&v)[E][C], T (&dl)[E],
//                          T eprev, const T (&Lp)[C], T enext, const T (&Un)[C], Aux& a) const
//   __device__ void carry_in(int64_t r, T fe, T ft, const T* c, bool from_left) const
//        adds, at element r (sorted index), a carry c[C] arriving with the exp
//        factor fe and the tie factor ft, from the left (prefix) or the right.
#pragma once
#include <algorithm>

#include "laplex_impl.h"
#include "scan_core.cuh"

namespace lx {

template <typename T> struct TPCut;
template <> struct TPCut<float> { static constexpr float v = 104.0f; };   // exp(-104) == 0 in fp32
template <> struct TPCut<double> { static constexpr double v = 746.0; };  // exp(-746) == 0 in fp64

struct TPStats {
    int32_t head;
    int32_t tail;
};

constexpr int TP_CARRY_NT = 256;
constexpr int TP_CARRY_PT = 8;
constexpr int TP_CARRY_BT = TP_CARRY_NT * TP_CARRY_PT;

template <typename T, int C>
struct TPWs {
    T* tfirst;   // [ntiles]
    T* tlast;    // [ntiles]
    T* fagg;     // [ntiles*C] L at the tile's last element, tile only
    T* bagg;     // [ntiles*C] U at the tile's first element, tile only
    TPStats* st; // [ntiles]
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
           Carve::need((size_t)ntiles, sizeof(TPStats)) + 2 * Carve::need((size_t)nb, es) +
           2 * Carve::need((size_t)(nb * C), es);
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
    W.bfe = cv.take<T>(nb);
    W.bfv = cv.take<T>(nb * C);
    W.bbf = cv.take<T>(nb);
    W.bbv = cv.take<T>(nb * C);
    W.carF = cv.take<T>(ntiles * C);
    W.carB = cv.take<T>(ntiles * C);
    return W;
}

// ------------------------------------------------------------------ pass 1
template <class P>
__global__ void __launch_bounds__(P::NT) k_tp_local(P p, TPWs<typename P::T, P::C> W) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT, E = P::E, NT = P::NT;
    constexpr int64_t TILE = (int64_t)NT * E;
    __shared__ BlockScan2Smem<T, C, NT> sm2;
    __shared__ int cnt_head, cnt_tail;
    __shared__ T sh_first, sh_last;
    const int64_t n = p.n;
    const int64_t t = blockIdx.x;
    const int64_t tile0 = t * TILE;
    const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
    T s[E], v[E][C];
    typename P::Aux aux;
    p.load(r0, s, v, aux);
    if (threadIdx.x == 0) {
        cnt_head = 0;
        cnt_tail = 0;
        sh_first = s[0];
        sh_last = p.s[min(tile0 + TILE, n) - 1];
    }
    T dl[E], fV[C], bW[C];
    chunk_aggregates<T, C, E, CT>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    block_excl_both<T, C, NT, CT>(s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf, nW, tf, tW,
                                  sm2);  // its barriers publish sh_first / sh_last
    {
        const T first = sh_first, lastv = sh_last;
        const int valid = (int)min((int64_t)E, max((int64_t)0, n - r0));
        int h = 0, q = 0;
        if (valid > 0) {
            T sl = s[0];
#pragma unroll
            for (int k = 1; k < E; ++k)
                if (k < valid) sl = s[k];
            if (sl - first < TPCut<T>::v) h = valid;
            else if (s[0] - first < TPCut<T>::v)
#pragma unroll
                for (int k = 0; k < E; ++k) h += (k < valid && s[k] - first < TPCut<T>::v) ? 1 : 0;
            if (lastv - s[0] < TPCut<T>::v) q = valid;
            else if (lastv - sl < TPCut<T>::v)
#pragma unroll
                for (int k = 0; k < E; ++k) q += (k < valid && lastv - s[k] < TPCut<T>::v) ? 1 : 0;
        }
        if (h) atomicAdd(&cnt_head, h);
        if (q) atomicAdd(&cnt_tail, q);
    }
    // zero carries from outside the tile (k_tp_headtail adds them)
    T eprev = hf ? pe : s[0], enext = hb ? nf : s[E - 1];
    T Lprev[C], Unext[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        Lprev[c] = hf ? pV[c] : T(0);
        Unext[c] = hb ? nW[c] : T(0);
    }
    p.finish(r0, s, v, dl, eprev, Lprev, enext, Unext, aux);
    __syncthreads();
    if (threadIdx.x == 0) {
        W.tfirst[t] = tf;
        W.tlast[t] = te;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            W.fagg[t * C + c] = tV[c];
            W.bagg[t * C + c] = tW[c];
        }
        W.st[t].head = cnt_head;
        W.st[t].tail = cnt_tail;
    }
}

// ------------------------------------------------------------------ pass 2
template <typename T, int C, int CT>
__device__ __forceinline__ void tp_segment(const TPWs<T, C>& W, int64_t t0, int64_t ntiles, T& fe,
                                           T (&fv)[C], T& bf, T (&bv)[C]) {
    const T pad = W.tlast[ntiles - 1];
    fe = pad;
    bf = pad;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        fv[c] = T(0);
        bv[c] = T(0);
    }
    bool any = false;
    for (int k = 0; k < TP_CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
        const T e = W.tlast[t];
        const Decay<T, C, CT> d(fe, e);
#pragma unroll
        for (int c = 0; c < C; ++c) fv[c] = dfma<T>(any ? d[c] : T(0), fv[c], W.fagg[t * C + c]);
        fe = e;
        any = true;
    }
    any = false;
    for (int k = TP_CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
        const T f = W.tfirst[t];
        const Decay<T, C, CT> d(f, bf);
#pragma unroll
        for (int c = 0; c < C; ++c) bv[c] = dfma<T>(any ? d[c] : T(0), bv[c], W.bagg[t * C + c]);
        bf = f;
        any = true;
    }
}

template <typename T, int C, int CT>
__global__ void __launch_bounds__(TP_CARRY_NT) k_tp_carry_blocks(TPWs<T, C> W, int64_t ntiles) {
    __shared__ BlockScan2Smem<T, C, TP_CARRY_NT> sm2;
    const int64_t t0 = (int64_t)blockIdx.x * TP_CARRY_BT + (int64_t)threadIdx.x * TP_CARRY_PT;
    T fe, fv[C], bf, bv[C];
    tp_segment<T, C, CT>(W, t0, ntiles, fe, fv, bf, bv);
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
    T fe, fv[C], bf, bv[C];
    tp_segment<T, C, CT>(W, t0, ntiles, fe, fv, bf, bv);
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
    for (int k = 0; k < TP_CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
#pragma unroll
        for (int c = 0; c < C; ++c) W.carF[t * C + c] = t == 0 ? T(0) : cv[c];
        const T e = W.tlast[t];
        const Decay<T, C, CT> d(ce, e);
#pragma unroll
        for (int c = 0; c < C; ++c) cv[c] = dfma<T>(d[c], cv[c], W.fagg[t * C + c]);
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
    for (int k = TP_CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
#pragma unroll
        for (int c = 0; c < C; ++c) W.carB[t * C + c] = t == ntiles - 1 ? T(0) : cw[c];
        const T f = W.tfirst[t];
        const Decay<T, C, CT> d(f, cf);
#pragma unroll
        for (int c = 0; c < C; ++c) cw[c] = dfma<T>(d[c], cw[c], W.bagg[t * C + c]);
        cf = f;
    }
}

// ------------------------------------------------------------------ pass 3
// One warp per tile at a time (persistent grid).
template <class P>
__global__ void __launch_bounds__(256) k_tp_headtail(P p, TPWs<typename P::T, P::C> W, int64_t ntiles) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT;
    constexpr int64_t TILE = (int64_t)P::NT * P::E;
    const int lane = threadIdx.x & 31;
    const int64_t n = p.n;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < ntiles;
         t += warps) {
        const int64_t b = t * TILE, e = min(b + TILE, n);
        const TPStats stt = W.st[t];
        if (t > 0) {
            T c[C];
            bool nz = false;
#pragma unroll
            for (int k = 0; k < C; ++k) {
                c[k] = W.carF[t * C + k];
                nz |= c[k] != T(0);
            }
            if (nz) {
                const T eT = p.s[b - 1];
                for (int64_t r = b + lane; r < b + stt.head; r += 32) {
                    const Decay<T, C, CT> d(eT, p.s[r]);
                    if (d.e != T(0) || (CT > 0 && d.t != T(0))) p.carry_in(r, d.e, CT > 0 ? d.t : T(0), c, true);
                }
            }
        }
        __syncwarp();
        if (t < ntiles - 1) {
            T c[C];
            bool nz = false;
#pragma unroll
            for (int k = 0; k < C; ++k) {
                c[k] = W.carB[t * C + k];
                nz |= c[k] != T(0);
            }
            if (nz) {
                const T fT = p.s[e];
                for (int64_t r = e - 1 - lane; r >= e - stt.tail; r -= 32) {
                    const Decay<T, C, CT> d(p.s[r], fT);
                    if (d.e != T(0) || (CT > 0 && d.t != T(0))) p.carry_in(r, d.e, CT > 0 ? d.t : T(0), c, false);
                }
            }
        }
        __syncwarp();
    }
}

template <class P>
inline int64_t tp_ntiles(int64_t n) {
    const int64_t tile = (int64_t)P::NT * P::E;
    return std::max<int64_t>(1, (n + tile - 1) / tile);
}

template <class P>
cudaError_t tp_run(const P& p, void* ws, size_t ws_bytes, cudaStream_t st) {
    using T = typename P::T;
    constexpr int C = P::C, CT = P::CT;
    if (p.n == 0) return cudaSuccess;
    const int64_t ntiles = tp_ntiles<P>(p.n);
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    Carve cv(ws, ws_bytes);
    TPWs<T, C> W = tp_carve<T, C>(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    static int sms_cache[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (sms_cache[dev] == 0) {
        e = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    profile_before(st);
    k_tp_local<P><<<(unsigned)ntiles, P::NT, 0, st>>>(p, W);
    profile_after(st);
    k_tp_carry_blocks<T, C, CT><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles);
    k_tp_carry_tiles<T, C, CT><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles, nb);
    const int64_t htb = std::max<int64_t>(1, std::min<int64_t>((ntiles + 7) / 8, (int64_t)sms_cache[dev] * 8));
    k_tp_headtail<P><<<(unsigned)htb, 256, 0, st>>>(p, W, ntiles);
    return cudaGetLastError();
}

}  // namespace lx
