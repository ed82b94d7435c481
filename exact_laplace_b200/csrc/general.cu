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
// k_merge_partition (merge-path split into tiles), k_gen_local (tile scan with
// the carries from halos of b-points, outputs at the a-points), k_tp_carry_blocks
// + k_tp_carry_tiles (exact tile carries, only when some tile's halos fell
// short), k_gen_headtail (those carries added to the a-points of such a tile's
// head and tail reach: on dense anchors a read-modify-write of the output
// side only, cheaper than scanning the merged tile again).  K^T is the same product with
// the roles of a and b exchanged (done by the caller).
#include <algorithm>

#include "laplex_impl.h"
#include "threepass.cuh"

namespace lx {

constexpr int GEN_NT = 256;


// ia[t] = number of a-points among the first min(t*tile, n+k) merged elements
// (the merge path of a before b on ties).  One warp per diagonal: each round
// probes 32 points of the remaining range at once (the test a[i] < b[p-1-i]
// is true, then false, along it), so a search over 2^20 points takes 4 rounds
// of dependent loads instead of 20.
template <typename T>
__global__ void k_merge_partition(const T* __restrict__ a, int64_t n, const T* __restrict__ b,
                                  int64_t k, int64_t tile, int64_t ntiles, int64_t* __restrict__ ia) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // uniform per warp
    if (t > ntiles) return;
    const int64_t p = min(t * tile, n + k);
    int64_t lo = max((int64_t)0, p - k), hi = min(p, n);  // the answer is in [lo, hi]
    while (lo < hi) {
        const int64_t span = hi - lo;
        const int64_t mid = lo + span * lane / 32;
        const unsigned m = __ballot_sync(FULL, a[mid] < b[p - 1 - mid]);
        const int c = __popc(m);  // probes 0..c-1 hold the test, c..31 do not
        const int64_t nlo = c == 0 ? lo : lo + span * (c - 1) / 32 + 1;
        const int64_t nhi = c == 32 ? hi : lo + span * c / 32;
        lo = nlo;
        hi = nhi;
    }
    if (lane == 0) ia[t] = lo;
}

// Channel values of b-point j (x_j times the scale; phased: cos psi_j and
// sin psi_j times that).
template <typename T, int NCOL, bool PHASED>
__device__ __forceinline__ void gen_bvalue(const GenArgs<T>& A, int64_t j, T (&vj)[PHASED ? 2 * NCOL : NCOL]) {
    const int64_t row = A.pin ? (int64_t)A.pin[j] : j;
    const T dsc = A.D ? A.D[A.pD ? (int64_t)A.pD[j] : j] : T(1);
    T cs = T(1), sn = T(0);
    if (PHASED) psincos<T>(A.psi[A.ppsi ? (int64_t)A.ppsi[j] : j], &sn, &cs);
    const T* xr = A.x + row * A.ldx + A.col0;
#pragma unroll
    for (int c = 0; c < NCOL; ++c) {
        const T val = (c < A.ncol ? xr[c] : T(0)) * dsc;
        if (PHASED) {
            vj[2 * c] = cs * val;
            vj[2 * c + 1] = sn * val;
        } else {
            vj[c] = val;
        }
    }
}

// One tile of the merged sequence (merged positions [p0, p1)).  The carries
// come from halos of H b-points on each side (a-points carry 0, so the b-points
// alone make the halo): the left one, b[j0 - H, j0), gives L at the merged
// element before the tile as sum_j exp(b_j - eT) x_j, the right one,
// b[j1, j1 + H), gives U at the element after it.  They are exact when they
// span CUT or reach the end of b; then the tile's outputs are final and its
// reach is stored as 0.  Otherwise the outputs are written with zero carries,
// the tile is counted (so the carry kernels run) and its reach -- the a-points
// within CUT of its first / last merged anchor -- is stored for k_gen_headtail.
// Every tile stores its edge anchors and zero-carry totals.
template <typename T, int NCOL, bool PHASED, int E, int NT, int H>
__device__ __forceinline__ void gen_tile(const GenArgs<T>& A, const TPWs<T, PHASED ? 2 * NCOL : NCOL>& W,
                                         const int64_t* __restrict__ ia, int64_t t, T* sh_anc, T* sh_val,
                                         BlockScan2Smem<T, PHASED ? 2 * NCOL : NCOL, NT>& sm2) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    constexpr int TILE = NT * E;
    constexpr int HH = H;
    const int64_t n = A.n, k = A.k, N = n + k;
    const int64_t p0 = t * TILE, p1 = min(p0 + TILE, N);
    const int64_t i0 = ia[t], i1 = ia[t + 1];
    const int64_t j0 = p0 - i0, j1 = p1 - i1;
    const int na = (int)(i1 - i0), nb = (int)(j1 - j0), cnt = na + nb;
    const bool needL = p0 > 0, needR = p1 < N;
    // merged anchors just before and just after the tile
    T eT = T(0), fT = T(0);
    if (needL) eT = (i0 > 0 && j0 > 0) ? max(A.sa[i0 - 1], A.sb[j0 - 1]) : (i0 > 0 ? A.sa[i0 - 1] : A.sb[j0 - 1]);
    if (needR) fT = (i1 < n && j1 < k) ? min(A.sa[i1], A.sb[j1]) : (i1 < n ? A.sa[i1] : A.sb[j1]);
    // thread 0 checks from two anchors whether the halos can be exact (they
    // span CUT or reach the end of b); the halos are only summed when both can
    __shared__ int sh_ok;
    if (threadIdx.x == 0) {
        bool okL = !needL || HH == 0 ? !needL : (j0 - HH <= 0 || eT - A.sb[j0 - HH] >= ExpCut<T>::v);
        bool okR = !needR || HH == 0 ? !needR : (j1 + HH >= k || A.sb[j1 + HH - 1] - fT >= ExpCut<T>::v);
        sh_ok = (okL ? 1 : 0) | (okR ? 2 : 0);
    }
    for (int q = threadIdx.x; q < na; q += NT) sh_anc[q] = A.sa[i0 + q];
    for (int q = threadIdx.x; q < nb; q += NT) {
        const int64_t j = j0 + q;
        sh_anc[na + q] = A.sb[j];
        T vj[C];
        gen_bvalue<T, NCOL, PHASED>(A, j, vj);
#pragma unroll
        for (int c = 0; c < C; ++c) sh_val[q * C + c] = vj[c];
    }
    __syncthreads();
    const int ok = sh_ok;
    // halo terms of this thread (halo element m = q + r NT < 2H; m < H: left,
    // H <= m < 2H: right), when both halos are exact
    T hvL[C], hvU[C];
    int bad[2] = {0, 0};
    if (threadIdx.x == 0) {
        bad[0] = (ok & 1) ? 0 : 1;
        bad[1] = (ok & 2) ? 0 : 1;
    }
#pragma unroll
    for (int c = 0; c < C; ++c) hvL[c] = hvU[c] = T(0);
    if (HH > 0 && ok == 3) {
        const int q = (int)threadIdx.x;
#pragma unroll
        for (int r = 0; r * NT < 2 * HH; ++r) {
            const int m = q + r * NT;
            if (m >= 2 * HH) break;
            const bool left = m < HH;
            if (!(left ? needL : needR)) continue;
            const int64_t j = left ? j0 - HH + m : j1 + (m - HH);
            if (j < 0 || j >= k) continue;  // the halo reaches the end of b
            const T bj = A.sb[j];
            T vj[C];
            gen_bvalue<T, NCOL, PHASED>(A, j, vj);
            const T f = dexp<T>(left ? bj - eT : fT - bj);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                if (left) hvL[c] += f * vj[c];
                else hvU[c] += f * vj[c];
            }
        }
    }
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
    int cnt4[4] = {bad[0], bad[1], 0, 0};  // span checks, then the reach in a-points
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
            cnt4[2] += (Aa[ai] - first < ExpCut<T>::v) ? 1 : 0;
            cnt4[3] += (padA - Aa[ai] < ExpCut<T>::v) ? 1 : 0;
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
    int tot4[4];
    T hL[C], hU[C];
    (void)block_excl_both_counted<T, C, NT, 0, true, 4, HH, C>(s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb,
                                                                nf, nW, tf, tW, cnt4, tot4, false, sm2, hvL,
                                                                hvU, hL, hU);
    const bool fin = tot4[0] == 0 && tot4[1] == 0;
    if (threadIdx.x == 0) {
        W.tfirst[t] = tf;
        W.tlast[t] = te;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            W.fagg[t * C + c] = tV[c];
            W.bagg[t * C + c] = tW[c];
        }
        W.st[t].head = fin ? 0 : tot4[2];
        W.st[t].tail = fin ? 0 : tot4[3];
        if (!fin) atomicAdd(W.redo_count, 1u);  // the carry kernels are needed
    }
    T Lc[C], Uc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        Lc[c] = fin && HH > 0 && needL ? hL[c] : T(0);
        Uc[c] = fin && HH > 0 && needR ? hU[c] : T(0);
    }
    const T eA = fin && needL ? eT : (hf ? pe : s[0]), fA = fin && needR ? fT : (hb ? nf : s[E - 1]);
    T eprev, Lprev[C], enext, Unext[C], o[E][C];
    apply_carry_fwd<T, C>(hf, pe, pV, eA, Lc, eprev, Lprev);
    apply_carry_bwd<T, C>(hb, nf, nW, fA, Uc, enext, Unext);
    chunk_final<T, C, E>(s, v, dl, eprev, Lprev, enext, Unext, o);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (aidx[e] < 0) continue;
        const int64_t i = i0 + aidx[e];
        const int64_t row = A.pout ? (int64_t)A.pout[i] : i;
        T* yr = A.y + row * A.ldy + A.col0;
        if (PHASED) {
            T sp, cp;
            psincos<T>(A.phi[A.pphi ? (int64_t)A.pphi[i] : i], &sp, &cp);
#pragma unroll
            for (int c = 0; c < NCOL; ++c)
                if (c < A.ncol) yr[c] = cp * o[e][2 * c] + sp * o[e][2 * c + 1];
        } else {
#pragma unroll
            for (int c = 0; c < NCOL; ++c)
                if (c < A.ncol) yr[c] = o[e][c];
        }
    }
}

// one block per merged tile
template <typename T, int NCOL, bool PHASED, int E, int NT, int H>
__global__ void __launch_bounds__(NT) k_gen_local(GenArgs<T> A, TPWs<T, PHASED ? 2 * NCOL : NCOL> W,
                                                  const int64_t* __restrict__ ia) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    __shared__ T sh_anc[NT * E];      // a-part [0, na), b-part [na, na + nb)
    __shared__ T sh_val[NT * E * C];  // channel values of the b-part
    __shared__ BlockScan2Smem<T, C, NT> sm2;
    gen_tile<T, NCOL, PHASED, E, NT, H>(A, W, ia, (int64_t)blockIdx.x, sh_anc, sh_val, sm2);
}

// Carries into the a-points of each tile's head and tail reach (a warp per tile).
template <typename T, int NCOL, bool PHASED>
__global__ void __launch_bounds__(256) k_gen_headtail(GenArgs<T> A, TPWs<T, PHASED ? 2 * NCOL : NCOL> W,
                                                      const int64_t* __restrict__ ia, int64_t tile,
                                                      int64_t ntiles) {
    // One block per tile.  Both carries are added in one read-modify-write of
    // each a-point of the head or tail reach (on dense anchors both reaches
    // are the whole tile), U = 4 independent a-points per thread and round so
    // that their loads are in flight together.
    constexpr int C = PHASED ? 2 * NCOL : NCOL, U = 4;
    const int64_t n = A.n, k = A.k, N = n + k;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t p0 = t * tile, p1 = min(p0 + tile, N);
        const int64_t i0 = ia[t], i1 = ia[t + 1], j0 = p0 - i0, j1 = p1 - i1, na = i1 - i0;
        const TPStats stt = W.st[t];
        T cL[C], cR[C];
        bool nzL = false, nzR = false;
#pragma unroll
        for (int q = 0; q < C; ++q) {
            cL[q] = t > 0 ? W.carF[t * C + q] : T(0);
            cR[q] = t < ntiles - 1 ? W.carB[t * C + q] : T(0);
            nzL |= cL[q] != T(0);
            nzR |= cR[q] != T(0);
        }
        const int64_t hl = nzL ? min((int64_t)stt.head, na) : 0;   // a-points [0, hl) take the left carry
        const int64_t tl = nzR ? min((int64_t)stt.tail, na) : 0;   // a-points [na - tl, na) the right one
        if (hl == 0 && tl == 0) continue;
        // merged anchors just before and just after the tile
        T eL = T(0), eR = T(0);
        if (hl > 0) eL = (i0 > 0 && j0 > 0) ? max(A.sa[i0 - 1], A.sb[j0 - 1]) : (i0 > 0 ? A.sa[i0 - 1] : A.sb[j0 - 1]);
        if (tl > 0) eR = (i1 < n && j1 < k) ? min(A.sa[i1], A.sb[j1]) : (i1 < n ? A.sa[i1] : A.sb[j1]);
        // the a-points of the reaches: [0, hl) and [max(hl, na - tl), na)
        const int64_t gap0 = hl, gap1 = max(hl, na - tl), tot = hl + (na - gap1);
        for (int64_t q0 = threadIdx.x; q0 < tot; q0 += (int64_t)U * blockDim.x) {
            int64_t iu[U];
            T au[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t q = q0 + (int64_t)u * blockDim.x;
                const int64_t qq = q < gap0 ? q : q - gap0 + gap1;  // skip the middle
                iu[u] = q < tot ? i0 + qq : -1;
                au[u] = iu[u] >= 0 ? A.sa[iu[u]] : T(0);
            }
            if constexpr (NCOL == 1 && !PHASED) {
                // one column: all loads of the round first, then the stores
                T* yp[U];
                T yv[U], dv[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    dv[u] = T(0);
                    yp[u] = nullptr;
                    if (iu[u] < 0) continue;
                    const int64_t q = iu[u] - i0;
                    const T fL = q < hl ? dexp<T>(eL - au[u]) : T(0);
                    const T fR = q >= na - tl ? dexp<T>(au[u] - eR) : T(0);
                    if (fL == T(0) && fR == T(0)) continue;
                    dv[u] = fL * cL[0] + fR * cR[0];
                    const int64_t row = A.pout ? (int64_t)A.pout[iu[u]] : iu[u];
                    yp[u] = A.y + row * A.ldy + A.col0;
                }
#pragma unroll
                for (int u = 0; u < U; ++u) yv[u] = yp[u] ? *yp[u] : T(0);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (yp[u]) *yp[u] = yv[u] + dv[u];
                continue;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (iu[u] < 0) continue;
                const int64_t q = iu[u] - i0;
                const T fL = q < hl ? dexp<T>(eL - au[u]) : T(0);
                const T fR = q >= na - tl ? dexp<T>(au[u] - eR) : T(0);
                if (fL == T(0) && fR == T(0)) continue;
                const int64_t row = A.pout ? (int64_t)A.pout[iu[u]] : iu[u];
                T* yr = A.y + row * A.ldy + A.col0;
                if (PHASED) {
                    T sp, cp;
                    psincos<T>(A.phi[A.pphi ? (int64_t)A.pphi[iu[u]] : iu[u]], &sp, &cp);
                    for (int q2 = 0; q2 < A.ncol; ++q2)
                        yr[q2] += fL * (cp * cL[2 * q2] + sp * cL[2 * q2 + 1]) +
                                  fR * (cp * cR[2 * q2] + sp * cR[2 * q2 + 1]);
                } else {
                    for (int q2 = 0; q2 < A.ncol; ++q2) yr[q2] += fL * cL[q2] + fR * cR[q2];
                }
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
// (one fp32 channel: 12, measured fastest on the C3 product among 4, 8, 12, 16)
#ifndef LX_GEN_E1
#define LX_GEN_E1 12
#endif
constexpr int gen_E(int C, int es) { return C * es <= 4 ? LX_GEN_E1 : (C * es <= 16 ? 4 : 2); }

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
    const int64_t nb = (p.ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    int dev_ = 0, sms = 0;
    cudaError_t e = tp_sm_count(dev_, sms);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(W.redo_count, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    constexpr int H = sizeof(T) == 4 ? 192 : 0;  // as the symmetric products
    profile_before(st);
    k_gen_local<T, NCOL, PHASED, E, GEN_NT, H><<<(unsigned)p.ntiles, GEN_NT, 0, st>>>(A, W, ia);
    profile_after(st);
    // the per-block totals are read only when there is more than one carry block
    if (nb > 1) k_tp_carry_blocks<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, p.ntiles);
    k_tp_carry_tiles<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, p.ntiles, nb);
    const int64_t htb = std::max<int64_t>(1, std::min<int64_t>(p.ntiles, (int64_t)sms * 8));
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
        const unsigned blocks = (unsigned)(((p.ntiles + 1) * 32 + 255) / 256);  // a warp per diagonal
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
