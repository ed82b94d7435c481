// sym_stream.cu -- the symmetric product for contiguous single-column input
// (x in sorted order): y = K x, K_ij = exp(-|s_i - s_j|) ("LAPLEX - La FFT dei
// Nuclei di Laplace Apprendibili", technical summary, §2.2 "Caso Simmetrico").
// x in sorted order, or in the caller's order with perm (gathered on load, y
// scattered back); several columns, phases or a scale use sym.cu.
//
// Three passes, none of which waits for another block:
//   1. k_tile_local<..., 0> (streams s and x once; persistent blocks, every
//      tile's s and x brought into a 2-stage shared-memory ring by 1-D bulk
//      copies (TMA), the next tiles loading while one is computed).  The copy
//      of a tile also brings a halo of H elements on each side.  A carry from
//      outside the tile reaches element r with a factor exp(-d), d >= the
//      distance from r to the tile's edge anchor, and exp(-d) is exactly 0 for
//      d >= CUT (ExpCut in common.cuh: fp32 88, fp64 746).  So when
//      a halo spans at least CUT, the carry summed over the halo is the exact
//      carry, and the tile writes its final outputs.  A tile whose halos do
//      not span CUT (dense anchors) writes nothing and is listed for pass 3.
//      Every tile records its first and last anchors and its zero-carry
//      forward/backward totals.
//   2. k_carry_blocks, k_carry_tiles (only when a tile was listed): the exact
//      carries into every tile from the tile totals (block totals, then
//      per-tile carries; the carry into a block is a walk over the block totals
//      that stops where exp of the gap is exactly 0).
//   3. k_tile_local<..., 1>: the listed tiles again, with those carries.
// Sparse anchors (spacing around 1 unit, as in a ~ U(0, n)) finish in pass 1:
// 12 bytes per element.  Dense anchors take passes 1 and 3: 8 + 12 bytes.
#include <algorithm>

#include "laplex_impl.h"
#include "bulk.cuh"
#include "devcache.h"
#include "scan_core.cuh"

namespace lx {

// tile shape of k_tile_local (fp32): threads per block, elements per thread,
// halo per side, resident blocks per SM
#ifndef LX_LT_NT
#define LX_LT_NT 256
#endif
#ifndef LX_LT_E
#define LX_LT_E 12
#endif
#ifndef LX_LT_H
#define LX_LT_H 192
#endif
#ifndef LX_LT_MINB
#define LX_LT_MINB 4
#endif
constexpr int LT_NT = LX_LT_NT;  // threads per tile block
constexpr int CARRY_NT = 256;  // threads per carry block
constexpr int CARRY_PT = 8;    // tiles per carry thread
constexpr int CARRY_BT = CARRY_NT * CARRY_PT;

template <typename T> struct LocalE;
template <> struct LocalE<float> { static constexpr int E = LX_LT_E; };  // 3 x 16 bytes
template <> struct LocalE<double> { static constexpr int E = 6; };   // 3 x 16 bytes
// halo elements per side: a span of CUT needs about CUT / spacing elements;
// fp64 (CUT 746) would need several times more, so its tiles have none
template <typename T> struct LocalH;
template <> struct LocalH<float> { static constexpr int H = LX_LT_H; };
template <> struct LocalH<double> { static constexpr int H = 0; };
constexpr int LT_STAGES = 2;

template <typename T>
struct LocalWs {
    T* tfirst;
    T* tlast;
    T* fagg;  // L at the tile's last element, tile only
    T* bagg;  // U at the tile's first element, tile only
    int32_t* redo;        // tiles the first pass left for the redo pass (any order)
    uint32_t* redo_count; // their number (zeroed before the first pass)
    T* bfe;   // per carry-block forward total: last anchor of the block, value
    T* bfv;
    T* bbf;   // per carry-block backward total: first anchor of the block, value
    T* bbv;
    T* carF;  // L at the element before tile t
    T* carB;  // U at the element after tile t
};

// Persistent: block b handles tiles b, b + G, b + 2G, ... (MODE 1: only the
// tiles of that sequence marked for the redo pass).  The tile of iteration i
// sits in ring stage i % S, and the stage is refilled with the block's tile
// S iterations later as soon as every thread has read it (after the block
// scan's barriers), so S tiles are in flight while one is computed.  Each
// thread owns E consecutive elements, an odd number of 16-byte units, so
// 128-bit shared loads of a warp touch distinct banks.  Two block barriers per
// tile, both inside the block scan, which also sums the halo terms and checks
// and carries the copy-timeout flag.
//
// MODE 0 (first pass).  The copy of a full tile also brings H elements on each
// side (halos).  Thread q takes the halo elements q, q + NT, ... < 2H: their
// terms of the carry from the left, L_{b-1} = sum_j exp(s_j - s_{b-1}) x_j, or
// from the right, U_e.  When both halos span at least CUT (or the tile is at an end of the
// array, or the halo reaches the end of the array) these sums are the exact
// carries and the tile's outputs are final.  Otherwise (dense anchors, H = 0)
// nothing is written and the tile is marked for the redo pass.  Every tile publishes its first
// and last anchors and its zero-carry totals for the carry kernels.
// MODE 1 (redo pass): the marked tiles again, with the exact carries from the
// carry kernels.
// GATHER: x is in the caller's order and y goes back to it through perm (the
// ring then holds s and perm; x is gathered from global memory).
template <typename T, int E, int NT, int S, int H, bool GATHER, int MODE>
__global__ void __launch_bounds__(NT, LX_LT_MINB) k_tile_local(const T* __restrict__ s_, const T* __restrict__ x_,
                                                      T* __restrict__ y_, const int32_t* __restrict__ perm,
                                                      int64_t n, int64_t ntiles, LocalWs<T> W,
                                                      uint32_t* status) {
    constexpr int VN = V16<T>::N;
    constexpr int64_t TILE = (int64_t)NT * E;
    constexpr int HH = MODE == 0 ? H : 0;     // halo brought by the copies
    constexpr int64_t STAGE = TILE + 2 * H;   // elements per array per stage
    static_assert(((E / VN) & 1) == 1, "E must be an odd number of 16-byte units");
    static_assert(H % 32 == 0 && H <= TILE, "halo: whole warps, at most a tile");
    extern __shared__ __align__(128) unsigned char dyn[];
    T* ring_s = reinterpret_cast<T*>(dyn);
    T* ring_x = ring_s + S * STAGE;                              // !GATHER
    int32_t* ring_p = reinterpret_cast<int32_t*>(ring_s + S * STAGE);  // GATHER
    __shared__ __align__(8) uint64_t full[S];
    __shared__ int64_t slot_tile[S];  // tile of each stage, -1: the block is done
    __shared__ int sh_timeout;
    __shared__ BlockScan2Smem<T, 1, NT> sm2;
    const int64_t G = gridDim.x;
    // thread 0: next candidate tile (MODE 0) or redo-list entry (MODE 1)
    int64_t cursor = blockIdx.x, listed = 0;

    auto issue = [&](int st, int64_t t) {  // one thread
        const int64_t b = t * TILE, e = b + TILE;
        if (e <= n) {
            const int64_t hl = (HH > 0 && t > 0) ? HH : 0;
            const int64_t hr = (HH > 0 && e + HH <= n) ? HH : 0;
            const int64_t lo = b - hl, cnt = hl + TILE + hr;
            const int64_t off = st * STAGE + (H - hl);
            if constexpr (GATHER) {
                mbar_expect_tx(&full[st], (uint32_t)(cnt * (sizeof(T) + sizeof(int32_t))));
                bulk_g2s(ring_s + off, s_ + lo, (uint32_t)(cnt * sizeof(T)), &full[st]);
                bulk_g2s(ring_p + off, perm + lo, (uint32_t)(cnt * sizeof(int32_t)), &full[st]);
            } else {
                mbar_expect_tx(&full[st], (uint32_t)(2 * cnt * sizeof(T)));
                bulk_g2s(ring_s + off, s_ + lo, (uint32_t)(cnt * sizeof(T)), &full[st]);
                bulk_g2s(ring_x + off, x_ + lo, (uint32_t)(cnt * sizeof(T)), &full[st]);
            }
        } else {
            mbar_arrive(&full[st]);  // ragged tile: read from global
        }
    };
    // thread 0: the block's next tile into stage st (or the end mark)
    auto next = [&](int st) {
        int64_t t = -1;
        if (MODE == 0 ? cursor < ntiles : cursor < listed) t = MODE == 0 ? cursor : (int64_t)W.redo[cursor];
        cursor += G;
        slot_tile[st] = t;
        if (t >= 0) issue(st, t);
        else mbar_arrive(&full[st]);
    };
    if (threadIdx.x == 0) {
        sh_timeout = 0;
        if (MODE == 1) listed = (int64_t)*(volatile uint32_t*)W.redo_count;
        for (int st = 0; st < S; ++st) mbar_init(&full[st], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int st = 0; st < S; ++st) next(st);
    }
    __syncthreads();
    for (int64_t i = 0;; ++i) {
        const int st = (int)(i % S);
        const bool landed = mbar_wait(&full[st], (uint32_t)((i / S) & 1));
        // the stage's tile (written before the arrive that completed the
        // phase); a thread whose wait ran out records it, and the block leaves
        // the loop together at the block scan's first barrier
        if (!landed) sh_timeout = 1;
        const int64_t t = landed ? slot_tile[st] : -1;
        const bool live = t >= 0;
        const int64_t tile0 = t * TILE;
        const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
        const bool ragged = tile0 + TILE > n;
        const T* S0 = ring_s + st * STAGE;  // [left halo | tile | right halo]
        // MODE 1: the exact carries into the tile (zero at the array's ends)
        T cL = T(0), cU = T(0), aL = T(0), aU = T(0);
        if (MODE == 1 && live) {
            if (t > 0) {
                cL = W.carF[t];
                aL = s_[tile0 - 1];
            }
            if (t < ntiles - 1) {
                cU = W.carB[t];
                aU = s_[tile0 + TILE];
            }
        }
        T s[E], v[E][1];
        int32_t pr[GATHER ? E : 1];
        {
            T xv[E];
            if (!live) {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    s[k] = T(0);
                    xv[k] = T(0);
                    if constexpr (GATHER) pr[k] = 0;
                }
            } else if (!ragged) {
                const T* ps = S0 + H + threadIdx.x * E;
#pragma unroll
                for (int k = 0; k < E; k += VN) ld16<T>(ps + k, &s[k]);
                if constexpr (GATHER) {
                    const int32_t* pp = ring_p + st * STAGE + H + threadIdx.x * E;
#pragma unroll
                    for (int k = 0; k < E; ++k) pr[k] = pp[k];
#pragma unroll
                    for (int k = 0; k < E; ++k) xv[k] = __ldg(x_ + pr[k]);
                } else {
                    const T* px = ring_x + st * STAGE + H + threadIdx.x * E;
#pragma unroll
                    for (int k = 0; k < E; k += VN) ld16<T>(px + k, &xv[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const int64_t r = r0 + k;
                    s[k] = s_[min(r, n - 1)];  // padded with the last anchor
                    if constexpr (GATHER) {
                        pr[k] = r < n ? perm[r] : 0;
                        xv[k] = r < n ? x_[pr[k]] : T(0);
                    } else {
                        xv[k] = r < n ? x_[r] : T(0);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < E; ++k) v[k][0] = xv[k];
        }
        // MODE 0: the halo terms of this thread (halo element k = q + m NT;
        // k < H: left, H <= k < 2H: right), and the checks that each halo
        // spans CUT (by the threads holding k = 0 and k = H).  A halo comes
        // from the ring when the copy brought it, else from global memory (the
        // ragged last tile; a right halo cut short by the end of the array,
        // which then holds every element to the right and needs no check).
        T hvL = T(0), hvU = T(0), ringL = T(0), ringR = T(0);  // s_{b-1}, s_e
        int bad[2] = {0, 0};
        if constexpr (MODE == 0) {
            const int q = (int)threadIdx.x;
            const int64_t e = min(tile0 + TILE, n);
            if constexpr (H > 0) {
                const bool needL = t > 0, needR = e < n;
                const bool ringH = !ragged;                    // halos copied with the tile
                const bool fullR = e + H <= n;                 // a right halo of H elements
                if (live) {
                    if (needL) ringL = ringH ? S0[H - 1] : s_[tile0 - 1];
                    if (needR) ringR = ringH && fullR ? S0[H + TILE] : s_[e];
#pragma unroll
                    for (int m = 0; m * NT < 2 * H; ++m) {
                        const int k = q + m * NT;
                        if (k >= 2 * H) break;
                        const bool left = k < H;
                        if (!(left ? needL : needR)) continue;
                        const int64_t jg = left ? tile0 - H + k : e + (k - H);  // global index
                        if (!left && jg >= n) continue;                      // past the end
                        const bool inring = ringH && (left || fullR);
                        const int j = left ? k : (int)(TILE + k);            // ring index
                        T sj, xj;
                        if (inring) {
                            sj = S0[j];
                            if constexpr (GATHER) xj = __ldg(x_ + ring_p[st * STAGE + j]);
                            else xj = ring_x[st * STAGE + j];
                        } else {
                            sj = s_[jg];
                            if constexpr (GATHER) xj = __ldg(x_ + perm[jg]);
                            else xj = x_[jg];
                        }
                        const T edge = left ? ringL : ringR;
                        const T term = dexp<T>(left ? sj - edge : edge - sj) * xj;
                        if (left) hvL += term;
                        else hvU += term;
                        if (k == 0) bad[0] = edge - sj >= ExpCut<T>::v ? 0 : 1;
                        if (k == H && fullR)
                            bad[1] = (inring ? S0[2 * H + TILE - 1] : s_[e + H - 1]) - edge >= ExpCut<T>::v ? 0 : 1;
                    }
                }
            } else {
                if (q == 0) bad[0] = (t > 0 || tile0 + TILE < n) ? 1 : 0;  // no halos: final only if alone
            }
        }
        // this thread's reads of stage st are ordered before the TMA writes that
        // refill it (generic -> async proxy); the refill is issued after the
        // block scan's barriers
        fence_proxy_async();
        T dl[E], fV[1], bW[1];
        chunk_aggregates<T, 1, E>(s, v, dl, fV, bW);
        bool hf, hb;
        T pe, pV[1], te, tV[1], nf, nW[1], tf, tW[1];
        int nbad[2];
        T hL = T(0), hU = T(0);
        if (block_excl_both_counted<T, 1, NT, 0, true, 2, (MODE == 0 ? H : 0)>(
                s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf, nW, tf, tW, bad, nbad, !live, sm2, &hvL,
                &hvU, &hL, &hU)) {
            // the block's last tile is done, or a copy never completed: then
            // report it and let the copies in flight land before leaving
            if (threadIdx.x == 0 && sh_timeout) {
                set_status(status, ST_TIMEOUT);
                for (int k = 0; k < S; ++k)
                    if (slot_tile[(i + k) % S] >= 0)
                        mbar_wait(&full[(i + k) % S], (uint32_t)(((i + k) / S) & 1));
            }
            return;
        }
        // the carries into the tile, and whether this pass writes it
        bool out = true;
        T eT = hf ? pe : s[0], Lc = T(0), fT = hb ? nf : s[E - 1], Uc = T(0);
        if (MODE == 0) {
            out = nbad[0] == 0 && nbad[1] == 0;
            if (H > 0 && out && t > 0) {
                eT = ringL;
                Lc = hL;
            }
            if (H > 0 && out && tile0 + TILE < n) {
                fT = ringR;
                Uc = hU;
            }
        } else {
            if (t > 0) {
                eT = aL;
                Lc = cL;
            }
            if (t < ntiles - 1) {
                fT = aU;
                Uc = cU;
            }
        }
        if (threadIdx.x == 0) {
            if (MODE == 0) {
                W.tfirst[t] = tf;
                W.tlast[t] = te;
                W.fagg[t] = tV[0];
                W.bagg[t] = tW[0];
                if (!out) W.redo[atomicAdd(W.redo_count, 1u)] = (int32_t)t;
            }
            next(st);
        }
        if (!out) continue;
        T eprev, Lprev[1], enext, Unext[1];
        {
            const T VT[1] = {Lc}, WT[1] = {Uc};
            apply_carry_fwd<T, 1>(hf, pe, pV, eT, VT, eprev, Lprev);
            apply_carry_bwd<T, 1>(hb, nf, nW, fT, WT, enext, Unext);
        }
        T o4[E][1];
        chunk_final<T, 1, E>(s, v, dl, eprev, Lprev, enext, Unext, o4);
        T o[E];
#pragma unroll
        for (int k = 0; k < E; ++k) o[k] = o4[k][0];
        if constexpr (GATHER) {
#pragma unroll
            for (int k = 0; k < E; ++k)
                if (r0 + k < n) y_[pr[k]] = o[k];
        } else if (!ragged) {
#pragma unroll
            for (int k = 0; k < E; k += VN) st16_stream<T>(y_ + r0 + k, &o[k]);
        } else {
#pragma unroll
            for (int k = 0; k < E; ++k)
                if (r0 + k < n) y_[r0 + k] = o[k];
        }
    }
}

// The records of this thread's CARRY_PT tiles, loaded in one round of
// independent loads (a tile past the end repeats the last one; it is skipped).
template <typename T>
struct CarrySeg {
    T tl[CARRY_PT], tf[CARRY_PT], fa[CARRY_PT], ba[CARRY_PT];
    __device__ __forceinline__ void load(const LocalWs<T>& W, int64_t t0, int64_t ntiles) {
#pragma unroll
        for (int k = 0; k < CARRY_PT; ++k) {
            const int64_t t = min(t0 + k, ntiles - 1);
            tl[k] = W.tlast[t];
            tf[k] = W.tfirst[t];
            fa[k] = W.fagg[t];
            ba[k] = W.bagg[t];
        }
    }
};

// This thread's forward and backward totals over its CARRY_PT tiles.
template <typename T>
__device__ __forceinline__ void carry_segment(const CarrySeg<T>& g, int64_t t0, int64_t ntiles, T pad,
                                              T& fe, T (&fv)[1], T& bf, T (&bv)[1]) {
    fe = pad;
    bf = pad;
    fv[0] = T(0);
    bv[0] = T(0);
    bool any = false;
#pragma unroll
    for (int k = 0; k < CARRY_PT; ++k) {
        if (t0 + k >= ntiles) break;
        const T e = g.tl[k];
        fv[0] = dfma<T>(any ? dexp<T>(fe - e) : T(0), fv[0], g.fa[k]);
        fe = e;
        any = true;
    }
    any = false;
#pragma unroll
    for (int k = CARRY_PT - 1; k >= 0; --k) {
        if (t0 + k >= ntiles) continue;
        const T f = g.tf[k];
        bv[0] = dfma<T>(any ? dexp<T>(f - bf) : T(0), bv[0], g.ba[k]);
        bf = f;
        any = true;
    }
}

template <typename T>
__global__ void __launch_bounds__(CARRY_NT) k_carry_blocks(LocalWs<T> W, int64_t ntiles) {
    if (*(volatile uint32_t*)W.redo_count == 0) return;  // every tile final
    __shared__ BlockScanSmem<T, 1, CARRY_NT> smf, smb;
    const int64_t t0 = (int64_t)blockIdx.x * CARRY_BT + (int64_t)threadIdx.x * CARRY_PT;
    CarrySeg<T> g;
    g.load(W, t0, ntiles);
    T fe, fv[1], bf, bv[1];
    carry_segment<T>(g, t0, ntiles, W.tlast[ntiles - 1], fe, fv, bf, bv);
    bool h;
    T pe, pv[1], te, tv[1], nf, nv[1], tf, tw[1];
    block_excl_fwd<T, 1, CARRY_NT>(fe, fv, h, pe, pv, te, tv, smf);
    block_excl_bwd<T, 1, CARRY_NT>(bf, bv, h, nf, nv, tf, tw, smb);
    if (threadIdx.x == 0) {
        W.bfe[blockIdx.x] = te;
        W.bfv[blockIdx.x] = tv[0];
        W.bbf[blockIdx.x] = tf;
        W.bbv[blockIdx.x] = tw[0];
    }
}

template <typename T>
__global__ void __launch_bounds__(CARRY_NT) k_carry_tiles(LocalWs<T> W, int64_t ntiles, int64_t nblocks) {
    if (*(volatile uint32_t*)W.redo_count == 0) return;  // every tile final
    __shared__ BlockScanSmem<T, 1, CARRY_NT> smf, smb;
    __shared__ T sh_c[2];
    const int64_t bidx = blockIdx.x;
    if (threadIdx.x == 0) {
        T acc = T(0);  // L at the element before this block
        if (bidx > 0) {
            const T eb = W.bfe[bidx - 1];
            for (int64_t j = bidx - 1; j >= 0; --j) {
                const T f = dexp<T>(W.bfe[j] - eb);
                if (f == T(0)) break;
                acc = dfma<T>(f, W.bfv[j], acc);
            }
        }
        T accb = T(0);  // U at the element after this block
        if (bidx + 1 < nblocks) {
            const T fb = W.bbf[bidx + 1];
            for (int64_t j = bidx + 1; j < nblocks; ++j) {
                const T f = dexp<T>(fb - W.bbf[j]);
                if (f == T(0)) break;
                accb = dfma<T>(f, W.bbv[j], accb);
            }
        }
        sh_c[0] = acc;
        sh_c[1] = accb;
    }
    const int64_t t0 = bidx * CARRY_BT + (int64_t)threadIdx.x * CARRY_PT;
    CarrySeg<T> g;
    g.load(W, t0, ntiles);
    T fe, fv[1], bf, bv[1];
    carry_segment<T>(g, t0, ntiles, W.tlast[ntiles - 1], fe, fv, bf, bv);
    bool hf, hb;
    T pe, pv[1], te, tv[1], nf, nv[1], tf, tw[1];
    block_excl_fwd<T, 1, CARRY_NT>(fe, fv, hf, pe, pv, te, tv, smf);  // its barriers publish sh_c
    block_excl_bwd<T, 1, CARRY_NT>(bf, bv, hb, nf, nv, tf, tw, smb);
    const T eBlk = bidx > 0 ? W.bfe[bidx - 1] : W.tlast[0];
    T ce, cv;
    if (hf) {
        ce = pe;
        cv = dfma<T>(dexp<T>(eBlk - pe), sh_c[0], pv[0]);
    } else {
        ce = eBlk;
        cv = sh_c[0];
    }
#pragma unroll
    for (int k = 0; k < CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
        W.carF[t] = t == 0 ? T(0) : cv;
        const T e = g.tl[k];
        cv = dfma<T>(dexp<T>(ce - e), cv, g.fa[k]);
        ce = e;
    }
    const T fBlk = bidx + 1 < nblocks ? W.bbf[bidx + 1] : W.tlast[ntiles - 1];
    T cf, cw;
    if (hb) {
        cf = nf;
        cw = dfma<T>(dexp<T>(nf - fBlk), sh_c[1], nv[0]);
    } else {
        cf = fBlk;
        cw = sh_c[1];
    }
#pragma unroll
    for (int k = CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
        W.carB[t] = t == ntiles - 1 ? T(0) : cw;
        const T f = g.tf[k];
        cw = dfma<T>(dexp<T>(f - cf), cw, g.ba[k]);
        cf = f;
    }
}

// ------------------------------------------------------------------ host side
template <typename T>
static int64_t local_ntiles(int64_t n) {
    const int64_t tile = (int64_t)LT_NT * LocalE<T>::E;
    return std::max<int64_t>(1, (n + tile - 1) / tile);
}

template <typename T>
static LocalWs<T> local_carve(Carve& cv, int64_t ntiles) {
    const int64_t nb = (ntiles + CARRY_BT - 1) / CARRY_BT;
    LocalWs<T> W;
    W.tfirst = cv.take<T>(ntiles);
    W.tlast = cv.take<T>(ntiles);
    W.fagg = cv.take<T>(ntiles);
    W.bagg = cv.take<T>(ntiles);
    W.redo = cv.take<int32_t>(ntiles);
    W.redo_count = cv.take<uint32_t>(1);
    W.bfe = cv.take<T>(nb);
    W.bfv = cv.take<T>(nb);
    W.bbf = cv.take<T>(nb);
    W.bbv = cv.take<T>(nb);
    W.carF = cv.take<T>(ntiles);
    W.carB = cv.take<T>(ntiles);
    return W;
}

size_t stream_ws_bytes(int64_t n, int f64) {
    const int64_t ntiles = f64 ? local_ntiles<double>(n) : local_ntiles<float>(n);
    const int64_t nb = (ntiles + CARRY_BT - 1) / CARRY_BT;
    const size_t es = f64 ? 8 : 4;
    return 6 * Carve::need((size_t)ntiles, es) + Carve::need((size_t)ntiles, 4) + Carve::need(1, 4) +
           4 * Carve::need((size_t)nb, es);
}

// One persistent launch of a k_tile_local variant: as many blocks as fit on
// the device (resident blocks per SM cached per device and variant), or one per
// tile; `timed` records the profiling events around it.
template <auto KERN, typename T>
static cudaError_t launch_tiles(int dev, int sms, size_t smem, bool timed, cudaStream_t st, const T* s,
                                const T* x, T* y, const int32_t* pp, int64_t n, int64_t ntiles,
                                const LocalWs<T>& W, uint32_t* status) {
    int per = 0;
    cudaError_t e = blocks_per_sm<KERN>(dev, LT_NT, smem, &per);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ntiles, (int64_t)per * sms);
    if (timed) profile_before(st);
    KERN<<<(unsigned)grid, LT_NT, smem, st>>>(s, x, y, pp, n, ntiles, W, status);
    if (timed) profile_after(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t stream_run(const T* s, const T* x, T* y, const int32_t* pout, int64_t n, void* ws,
                       size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    constexpr int E = LocalE<T>::E;
    constexpr int H = LocalH<T>::H;
    constexpr int TILE = LT_NT * E;
    constexpr size_t STAGE = (size_t)TILE + 2 * H;
    const int64_t ntiles = local_ntiles<T>(n);
    const int64_t nb = (ntiles + CARRY_BT - 1) / CARRY_BT;
    Carve cv(ws, ws_bytes);
    LocalWs<T> W = local_carve<T>(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = current_device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(W.redo_count, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    const size_t smem_x = (size_t)LT_STAGES * STAGE * (2 * sizeof(T));
    const size_t smem_p = (size_t)LT_STAGES * STAGE * (sizeof(T) + sizeof(int32_t));
    if (pout == nullptr)
        e = launch_tiles<k_tile_local<T, E, LT_NT, LT_STAGES, H, false, 0>>(dev, sms, smem_x, true, st, s, x, y, nullptr, n, ntiles, W, status);
    else
        e = launch_tiles<k_tile_local<T, E, LT_NT, LT_STAGES, H, true, 0>>(dev, sms, smem_p, true, st, s, x, y, pout, n, ntiles, W, status);
    if (e != cudaSuccess) return e;
    // the per-block totals are read only when there is more than one carry block
    if (nb > 1) k_carry_blocks<T><<<(unsigned)nb, CARRY_NT, 0, st>>>(W, ntiles);
    k_carry_tiles<T><<<(unsigned)nb, CARRY_NT, 0, st>>>(W, ntiles, nb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (pout == nullptr)
        e = launch_tiles<k_tile_local<T, E, LT_NT, LT_STAGES, H, false, 1>>(dev, sms, smem_x, false, st, s, x, y, nullptr, n, ntiles, W, status);
    else
        e = launch_tiles<k_tile_local<T, E, LT_NT, LT_STAGES, H, true, 1>>(dev, sms, smem_p, false, st, s, x, y, pout, n, ntiles, W, status);
    return e;
}

template cudaError_t stream_run<float>(const float*, const float*, float*, const int32_t*, int64_t,
                                       void*, size_t, uint32_t*, cudaStream_t);
template cudaError_t stream_run<double>(const double*, const double*, double*, const int32_t*,
                                        int64_t, void*, size_t, uint32_t*, cudaStream_t);

}  // namespace lx
