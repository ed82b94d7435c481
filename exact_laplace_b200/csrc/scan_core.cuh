// scan_core.cuh -- the first-order linear-recurrence scan of the LAPLEX products.
//
// With anchors ascending, the lower part L_i = sum_{j<=i} exp(s_j - s_i) x_j and
// the upper part U_i = sum_{j>=i} exp(s_i - s_j) x_j obey
//     L_i = x_i + exp(s_{i-1} - s_i) L_{i-1},   U_i = x_i + exp(s_i - s_{i+1}) U_{i+1}
// ("LAPLEX - La FFT dei Nuclei di Laplace Apprendibili", technical summary, §2.2).
// A run of elements is summarised by a pair: forward (e, V) = "V is L at the
// element whose anchor is e, counting only that run"; backward (f, W) = "W is
// U at the element whose anchor is f".  Runs combine associatively:
//     forward   P (+) A  = (e_A, V_A + exp(e_P - e_A) V_P)      P left of A
//     backward  A (+) S  = (f_A, W_A + exp(f_A - f_S) W_S)      A left of S
// Between two runs the decay is one exp of the difference of their edge
// anchors, so between tiles and between warps of a block fp32 error does not
// grow with the distance; inside a warp's shuffle scan a decay is a product of
// at most five rounded factors (see the warp level below).  Elements past the end are padded with the last
// anchor and value 0, which is neutral in both directions.
//
// The last CT channels ("tie channels") use the decay [e_P == e_A] instead of
// exp(e_P - e_A): with sorted anchors that is the product of the per-step
// indicators, so those channels sum over runs of equal anchors only (used by
// the backward pass for the sign(0) = 0 terms).
#pragma once
#include "common.cuh"

namespace lx {

// decay applied to channel c of a combine across anchors p <= q
template <typename T, int C, int CT>
struct Decay {
    T e;   // exp(p - q)
    T t;   // [p == q]
    __device__ __forceinline__ Decay(const T p, const T q) {
        e = dexp<T>(p - q);
        if (CT > 0) t = (p == q) ? T(1) : T(0);
    }
    __device__ __forceinline__ T operator[](int c) const { return (CT > 0 && c >= C - CT) ? t : e; }
};

// ---------------------------------------------------------------- warp level
// Inclusive scans over the lanes.  At step off a lane combines the partial of
// lane l - off, whose edge anchor is e_{l-off}, with the decay
// d_off(l) = exp(e_{l-off} - e_l) (tie channels: [e_{l-off} == e_l]).  Only
// d_1 takes an exp; d_2off(l) = d_off(l - off) d_off(l) is the product of the
// previous level's two decays (at most five rounded products; each factor is
// at least the product, so nothing at or above FLT_MIN is flushed).
template <typename T, int C, int CT = 0>
__device__ __forceinline__ void warp_incl_fwd(const T e, T (&V)[C], const int lane) {
    Decay<T, C, CT> d(__shfl_up_sync(FULL, e, 1), e);  // lane 0: exp(0), unused
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        T Vo[C];
#pragma unroll
        for (int c = 0; c < C; ++c) Vo[c] = __shfl_up_sync(FULL, V[c], off);
        const T de = __shfl_up_sync(FULL, d.e, off);
        const T dt = CT > 0 ? __shfl_up_sync(FULL, d.t, off) : T(0);
        if (lane >= off) {
#pragma unroll
            for (int c = 0; c < C; ++c) V[c] = dfma<T>(d[c], Vo[c], V[c]);
        }
        d.e *= de;
        if (CT > 0) d.t *= dt;
    }
}

template <typename T, int C, int CT = 0>
__device__ __forceinline__ void warp_incl_bwd(const T f, T (&W)[C], const int lane) {
    Decay<T, C, CT> d(f, __shfl_down_sync(FULL, f, 1));  // lane 31: exp(0), unused
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        T Wo[C];
#pragma unroll
        for (int c = 0; c < C; ++c) Wo[c] = __shfl_down_sync(FULL, W[c], off);
        const T de = __shfl_down_sync(FULL, d.e, off);
        const T dt = CT > 0 ? __shfl_down_sync(FULL, d.t, off) : T(0);
        if (lane + off < 32) {
#pragma unroll
            for (int c = 0; c < C; ++c) W[c] = dfma<T>(d[c], Wo[c], W[c]);
        }
        d.e *= de;
        if (CT > 0) d.t *= dt;
    }
}

// ---------------------------------------------------------------- block level
template <typename T, int C, int NT>
struct BlockScanSmem {
    static constexpr int NW = NT / 32;
    T we[NW];
    T wV[NW][C];
    T pe[NW];      // exclusive prefix (forward) / suffix (backward) of each warp
    T pV[NW][C];
    T te;          // block total
    T tV[C];
};

// Exclusive forward scan over the threads of the block, in thread order.
// In: this thread's run summary (e, V).  Out: has (false for thread 0), the
// summary (pe, pV) of all runs of lower threads, and the block total (te, tV).
template <typename T, int C, int NT, int CT = 0>
__device__ __forceinline__ void block_excl_fwd(const T e, const T (&V)[C], bool& has, T& pe,
                                               T (&pV)[C], T& te, T (&tV)[C],
                                               BlockScanSmem<T, C, NT>& sm) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    T iV[C];
#pragma unroll
    for (int c = 0; c < C; ++c) iV[c] = V[c];
    warp_incl_fwd<T, C, CT>(e, iV, lane);
    if (lane == 31) {
        sm.we[w] = e;
#pragma unroll
        for (int c = 0; c < C; ++c) sm.wV[w][c] = iV[c];
    }
    __syncthreads();
    if (w == 0) {
        T ge = lane < NW ? sm.we[lane] : T(0);
        T gV[C];
#pragma unroll
        for (int c = 0; c < C; ++c) gV[c] = lane < NW ? sm.wV[lane][c] : T(0);
#pragma unroll
        for (int off = 1; off < NW; off <<= 1) {
            const T eo = __shfl_up_sync(FULL, ge, off);
            T Vo[C];
#pragma unroll
            for (int c = 0; c < C; ++c) Vo[c] = __shfl_up_sync(FULL, gV[c], off);
            if (lane >= off && lane < NW) {
                const Decay<T, C, CT> d(eo, ge);
#pragma unroll
                for (int c = 0; c < C; ++c) gV[c] = dfma<T>(d[c], Vo[c], gV[c]);
            }
        }
        const T xe = __shfl_up_sync(FULL, ge, 1);
        T xV[C];
#pragma unroll
        for (int c = 0; c < C; ++c) xV[c] = __shfl_up_sync(FULL, gV[c], 1);
        if (lane > 0 && lane < NW) {
            sm.pe[lane] = xe;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.pV[lane][c] = xV[c];
        }
        if (lane == NW - 1) {
            sm.te = ge;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.tV[c] = gV[c];
        }
    }
    __syncthreads();
    const T le = __shfl_up_sync(FULL, e, 1);
    T lV[C];
#pragma unroll
    for (int c = 0; c < C; ++c) lV[c] = __shfl_up_sync(FULL, iV[c], 1);
    if (w > 0 && lane > 0) {
        has = true;
        pe = le;
        const Decay<T, C, CT> d(sm.pe[w], le);
#pragma unroll
        for (int c = 0; c < C; ++c) pV[c] = dfma<T>(d[c], sm.pV[w][c], lV[c]);
    } else if (w > 0) {
        has = true;
        pe = sm.pe[w];
#pragma unroll
        for (int c = 0; c < C; ++c) pV[c] = sm.pV[w][c];
    } else if (lane > 0) {
        has = true;
        pe = le;
#pragma unroll
        for (int c = 0; c < C; ++c) pV[c] = lV[c];
    } else {
        has = false;
        pe = T(0);
#pragma unroll
        for (int c = 0; c < C; ++c) pV[c] = T(0);
    }
    te = sm.te;
#pragma unroll
    for (int c = 0; c < C; ++c) tV[c] = sm.tV[c];
}

// Exclusive backward scan (suffix over higher threads), mirror of block_excl_fwd.
template <typename T, int C, int NT, int CT = 0>
__device__ __forceinline__ void block_excl_bwd(const T f, const T (&W)[C], bool& has, T& nf,
                                               T (&nW)[C], T& tf, T (&tW)[C],
                                               BlockScanSmem<T, C, NT>& sm) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    T iW[C];
#pragma unroll
    for (int c = 0; c < C; ++c) iW[c] = W[c];
    warp_incl_bwd<T, C, CT>(f, iW, lane);
    if (lane == 0) {
        sm.we[w] = f;
#pragma unroll
        for (int c = 0; c < C; ++c) sm.wV[w][c] = iW[c];
    }
    __syncthreads();
    if (w == 0) {
        T gf = lane < NW ? sm.we[lane] : T(0);
        T gW[C];
#pragma unroll
        for (int c = 0; c < C; ++c) gW[c] = lane < NW ? sm.wV[lane][c] : T(0);
#pragma unroll
        for (int off = 1; off < NW; off <<= 1) {
            const T fo = __shfl_down_sync(FULL, gf, off);
            T Wo[C];
#pragma unroll
            for (int c = 0; c < C; ++c) Wo[c] = __shfl_down_sync(FULL, gW[c], off);
            if (lane + off < NW) {
                const Decay<T, C, CT> d(gf, fo);
#pragma unroll
                for (int c = 0; c < C; ++c) gW[c] = dfma<T>(d[c], Wo[c], gW[c]);
            }
        }
        const T xf = __shfl_down_sync(FULL, gf, 1);
        T xW[C];
#pragma unroll
        for (int c = 0; c < C; ++c) xW[c] = __shfl_down_sync(FULL, gW[c], 1);
        if (lane < NW - 1) {
            sm.pe[lane] = xf;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.pV[lane][c] = xW[c];
        }
        if (lane == 0) {
            sm.te = gf;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.tV[c] = gW[c];
        }
    }
    __syncthreads();
    const T lf = __shfl_down_sync(FULL, f, 1);
    T lW[C];
#pragma unroll
    for (int c = 0; c < C; ++c) lW[c] = __shfl_down_sync(FULL, iW[c], 1);
    if (w < NW - 1 && lane < 31) {
        has = true;
        nf = lf;
        const Decay<T, C, CT> d(lf, sm.pe[w]);
#pragma unroll
        for (int c = 0; c < C; ++c) nW[c] = dfma<T>(d[c], sm.pV[w][c], lW[c]);
    } else if (w < NW - 1) {
        has = true;
        nf = sm.pe[w];
#pragma unroll
        for (int c = 0; c < C; ++c) nW[c] = sm.pV[w][c];
    } else if (lane < 31) {
        has = true;
        nf = lf;
#pragma unroll
        for (int c = 0; c < C; ++c) nW[c] = lW[c];
    } else {
        has = false;
        nf = T(0);
#pragma unroll
        for (int c = 0; c < C; ++c) nW[c] = T(0);
    }
    tf = sm.te;
#pragma unroll
    for (int c = 0; c < C; ++c) tW[c] = sm.tV[c];
}

// Both exclusive scans of one channel set at once (forward prefix over lower
// threads, backward suffix over higher threads), sharing two barriers.
template <typename T, int C, int NT>
struct BlockScan2Smem {
    static constexpr int NW = NT / 32;
    T fe[NW];
    T fV[NW][C];
    T be[NW];
    T bV[NW][C];
    T pfe[NW];
    T pfV[NW][C];
    T pbe[NW];
    T pbV[NW][C];
    T tfe, tbe;
    T tfV[C], tbV[C];
    int wcnt[NW][4];  // per-warp sums of integer counts (block_excl_both_counted)
    int tcnt[4];
    T whL[NW][C];     // per-warp halo sums (left, right; one per channel)
    T whU[NW][C];
    T thL[C], thU[C]; // and their totals
};

// block_excl_both_counted: the two scans; it also sums NI <= 4 integer counts
// over the block (cnt in, tot out, read by every thread) and ORs a flag: if any
// thread passes bad, the function returns true right after its first barrier,
// in every thread, with the outputs unset.  COUNTED = false drops the counts
// and the flag.  HH > 0 (halo elements per side) also sums two sets of HC <= C
// values per thread, hvL and hvU, into the block totals hL and hU.  The halo
// element k of the tile (k < HH: left, HH <= k < 2 HH: right) belongs to
// thread k mod NT, so a warp holds left terms only if one of its k < HH, and
// right terms only if one of its k lies in [HH, 2 HH).
template <typename T, int C, int NT, int CT, bool COUNTED, int NI = 2, int HH = 0, int HC = 1>
__device__ __forceinline__ bool block_excl_both_counted(
    const T e, const T (&V)[C], const T f, const T (&W)[C], bool& hasf, T& pe, T (&pV)[C], T& te,
    T (&tV)[C], bool& hasb, T& nf, T (&nW)[C], T& tf, T (&tW)[C], const int (&cnt)[NI], int (&tot)[NI],
    const bool bad, BlockScan2Smem<T, C, NT>& sm, const T* hvL = nullptr, const T* hvU = nullptr,
    T* hL = nullptr, T* hU = nullptr) {
    constexpr int NW = NT / 32;
    static_assert(NW <= 32, "one warp scans the warp totals");
    static_assert(NI >= 1 && NI <= 4, "at most four counts");
    static_assert(HH % 32 == 0, "halo: whole warps");
    static_assert(HC >= 1 && HC <= C, "halo channels");
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    T iV[C], iW[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        iV[c] = V[c];
        iW[c] = W[c];
    }
    warp_incl_fwd<T, C, CT>(e, iV, lane);
    warp_incl_bwd<T, C, CT>(f, iW, lane);
    if (lane == 31) {
        sm.fe[w] = e;
#pragma unroll
        for (int c = 0; c < C; ++c) sm.fV[w][c] = iV[c];
    }
    if (COUNTED) {
#pragma unroll
        for (int q = 0; q < NI; ++q) {
            const int cq = (int)__reduce_add_sync(FULL, (unsigned)cnt[q]);
            if (lane == 0) sm.wcnt[w][q] = cq;
        }
    }
    if (HH > 0) {
        bool hasL = false, hasR = false;
#pragma unroll
        for (int m = 0; m * NT < 2 * HH; ++m) {
            const int lo = 32 * w + m * NT;
            if (lo < HH) hasL = true;
            else if (lo < 2 * HH) hasR = true;
        }
#pragma unroll
        for (int c = 0; c < HC; ++c) {
            T hl = hasL ? hvL[c] : T(0), hu = hasR ? hvU[c] : T(0);
            if (hasL) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) hl += __shfl_xor_sync(FULL, hl, off);
            }
            if (hasR) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) hu += __shfl_xor_sync(FULL, hu, off);
            }
            if (lane == 0) {
                sm.whL[w][c] = hl;
                sm.whU[w][c] = hu;
            }
        }
    }
    if (lane == 0) {
        sm.be[w] = f;
#pragma unroll
        for (int c = 0; c < C; ++c) sm.bV[w][c] = iW[c];
    }
    if (COUNTED) {
        if (__syncthreads_or(bad)) return true;
    } else {
        __syncthreads();
    }
    // the serial middle step, split: warp 0 scans the warp totals forward and
    // sums the counts, warp 1 scans them backward and sums the halo terms
    constexpr int WB = NW > 1 ? 1 : 0;
    if (w == 0) {
        if (COUNTED) {
#pragma unroll
            for (int q = 0; q < NI; ++q) {
                const int cq = (int)__reduce_add_sync(FULL, lane < NW ? (unsigned)sm.wcnt[lane][q] : 0u);
                if (lane == 0) sm.tcnt[q] = cq;
            }
        }
        T ge = lane < NW ? sm.fe[lane] : T(0), gV[C];
#pragma unroll
        for (int c = 0; c < C; ++c) gV[c] = lane < NW ? sm.fV[lane][c] : T(0);
#pragma unroll
        for (int off = 1; off < NW; off <<= 1) {
            const T eo = __shfl_up_sync(FULL, ge, off);
            T Vo[C];
#pragma unroll
            for (int c = 0; c < C; ++c) Vo[c] = __shfl_up_sync(FULL, gV[c], off);
            if (lane >= off && lane < NW) {
                const Decay<T, C, CT> d(eo, ge);
#pragma unroll
                for (int c = 0; c < C; ++c) gV[c] = dfma<T>(d[c], Vo[c], gV[c]);
            }
        }
        const T xe = __shfl_up_sync(FULL, ge, 1);
        T xV[C];
#pragma unroll
        for (int c = 0; c < C; ++c) xV[c] = __shfl_up_sync(FULL, gV[c], 1);
        if (lane > 0 && lane < NW) {
            sm.pfe[lane] = xe;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.pfV[lane][c] = xV[c];
        }
        if (lane == NW - 1) {
            sm.tfe = ge;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.tfV[c] = gV[c];
        }
    }
    if (w == WB) {
        if (HH > 0) {
            // warp sums added in a fixed butterfly over the lanes
#pragma unroll
            for (int c = 0; c < HC; ++c) {
                T sl = lane < NW ? sm.whL[lane][c] : T(0), su = lane < NW ? sm.whU[lane][c] : T(0);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sl += __shfl_xor_sync(FULL, sl, off);
                    su += __shfl_xor_sync(FULL, su, off);
                }
                if (lane == 0) {
                    sm.thL[c] = sl;
                    sm.thU[c] = su;
                }
            }
        }
        T gf = lane < NW ? sm.be[lane] : T(0), gW[C];
#pragma unroll
        for (int c = 0; c < C; ++c) gW[c] = lane < NW ? sm.bV[lane][c] : T(0);
#pragma unroll
        for (int off = 1; off < NW; off <<= 1) {
            const T fo = __shfl_down_sync(FULL, gf, off);
            T Wo[C];
#pragma unroll
            for (int c = 0; c < C; ++c) Wo[c] = __shfl_down_sync(FULL, gW[c], off);
            if (lane + off < NW) {
                const Decay<T, C, CT> d(gf, fo);
#pragma unroll
                for (int c = 0; c < C; ++c) gW[c] = dfma<T>(d[c], Wo[c], gW[c]);
            }
        }
        const T xf = __shfl_down_sync(FULL, gf, 1);
        T xW[C];
#pragma unroll
        for (int c = 0; c < C; ++c) xW[c] = __shfl_down_sync(FULL, gW[c], 1);
        if (lane < NW - 1) {
            sm.pbe[lane] = xf;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.pbV[lane][c] = xW[c];
        }
        if (lane == 0) {
            sm.tbe = gf;
#pragma unroll
            for (int c = 0; c < C; ++c) sm.tbV[c] = gW[c];
        }
    }
    __syncthreads();
    // forward: lanes below, then warps below
    {
        const T le = __shfl_up_sync(FULL, e, 1);
        T lV[C];
#pragma unroll
        for (int c = 0; c < C; ++c) lV[c] = __shfl_up_sync(FULL, iV[c], 1);
        if (w > 0 && lane > 0) {
            hasf = true;
            pe = le;
            const Decay<T, C, CT> d(sm.pfe[w], le);
#pragma unroll
            for (int c = 0; c < C; ++c) pV[c] = dfma<T>(d[c], sm.pfV[w][c], lV[c]);
        } else if (w > 0) {
            hasf = true;
            pe = sm.pfe[w];
#pragma unroll
            for (int c = 0; c < C; ++c) pV[c] = sm.pfV[w][c];
        } else if (lane > 0) {
            hasf = true;
            pe = le;
#pragma unroll
            for (int c = 0; c < C; ++c) pV[c] = lV[c];
        } else {
            hasf = false;
            pe = T(0);
#pragma unroll
            for (int c = 0; c < C; ++c) pV[c] = T(0);
        }
        te = sm.tfe;
#pragma unroll
        for (int c = 0; c < C; ++c) tV[c] = sm.tfV[c];
    }
    // backward: lanes above, then warps above
    {
        const T lf = __shfl_down_sync(FULL, f, 1);
        T lW[C];
#pragma unroll
        for (int c = 0; c < C; ++c) lW[c] = __shfl_down_sync(FULL, iW[c], 1);
        if (w < NW - 1 && lane < 31) {
            hasb = true;
            nf = lf;
            const Decay<T, C, CT> d(lf, sm.pbe[w]);
#pragma unroll
            for (int c = 0; c < C; ++c) nW[c] = dfma<T>(d[c], sm.pbV[w][c], lW[c]);
        } else if (w < NW - 1) {
            hasb = true;
            nf = sm.pbe[w];
#pragma unroll
            for (int c = 0; c < C; ++c) nW[c] = sm.pbV[w][c];
        } else if (lane < 31) {
            hasb = true;
            nf = lf;
#pragma unroll
            for (int c = 0; c < C; ++c) nW[c] = lW[c];
        } else {
            hasb = false;
            nf = T(0);
#pragma unroll
            for (int c = 0; c < C; ++c) nW[c] = T(0);
        }
        tf = sm.tbe;
#pragma unroll
        for (int c = 0; c < C; ++c) tW[c] = sm.tbV[c];
    }
    if (COUNTED) {
#pragma unroll
        for (int q = 0; q < NI; ++q) tot[q] = sm.tcnt[q];
    }
    if (HH > 0) {
#pragma unroll
        for (int c = 0; c < HC; ++c) {
            hL[c] = sm.thL[c];
            hU[c] = sm.thU[c];
        }
    }
    return false;
}

template <typename T, int C, int NT, int CT = 0>
__device__ __forceinline__ void block_excl_both(const T e, const T (&V)[C], const T f, const T (&W)[C],
                                                bool& hasf, T& pe, T (&pV)[C], T& te, T (&tV)[C],
                                                bool& hasb, T& nf, T (&nW)[C], T& tf, T (&tW)[C],
                                                BlockScan2Smem<T, C, NT>& sm) {
    const int cnt[2] = {0, 0};
    int tot[2];
    (void)block_excl_both_counted<T, C, NT, CT, false>(e, V, f, W, hasf, pe, pV, te, tV, hasb, nf, nW,
                                                       tf, tW, cnt, tot, false, sm);
}

// ---------------------------------------------------------------- chunk level
// A thread owns E consecutive elements: anchors s[E], values v[E][C].
// dl[i] = exp(s[i-1] - s[i]) for i = 1..E-1 (dl[0] is set in chunk_final).
template <typename T, int C, int E, int CT = 0>
__device__ __forceinline__ void chunk_aggregates(const T (&s)[E], const T (&v)[E][C], T (&dl)[E],
                                                 T (&fV)[C], T (&bW)[C]) {
#pragma unroll
    for (int i = 1; i < E; ++i) dl[i] = dexp<T>(s[i - 1] - s[i]);
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const bool tie = CT > 0 && c >= C - CT;
        T a = v[0][c];
#pragma unroll
        for (int i = 1; i < E; ++i) {
            const T d = tie ? (s[i - 1] == s[i] ? T(1) : T(0)) : dl[i];
            a = dfma<T>(d, a, v[i][c]);
        }
        fV[c] = a;
        T b = v[E - 1][c];
#pragma unroll
        for (int i = E - 2; i >= 0; --i) {
            const T d = tie ? (s[i] == s[i + 1] ? T(1) : T(0)) : dl[i + 1];
            b = dfma<T>(d, b, v[i][c]);
        }
        bW[c] = b;
    }
}

// Given the state just before the chunk (anchor eprev, value Lprev) and just
// after it (anchor enext, value Unext), out[i][c] = L_i + U_i - v_i, formed as
// L_i + exp(s_i - s_{i+1}) U_{i+1} (U_i without its own term).
template <typename T, int C, int E>
__device__ __forceinline__ void chunk_final(const T (&s)[E], const T (&v)[E][C], T (&dl)[E],
                                            const T eprev, const T (&Lprev)[C], const T enext,
                                            const T (&Unext)[C], T (&out)[E][C]) {
    dl[0] = dexp<T>(eprev - s[0]);
    const T dn = dexp<T>(s[E - 1] - enext);
#pragma unroll
    for (int c = 0; c < C; ++c) {
        T L = Lprev[c];
#pragma unroll
        for (int i = 0; i < E; ++i) {
            L = dfma<T>(dl[i], L, v[i][c]);
            out[i][c] = L;
        }
        T U = Unext[c];
#pragma unroll
        for (int i = E - 1; i >= 0; --i) {
            const T d = i == E - 1 ? dn : dl[i + 1];
            out[i][c] = dfma<T>(d, U, out[i][c]);
            U = dfma<T>(d, U, v[i][c]);
        }
    }
}

// Combine a thread's in-tile exclusive prefix with the tile's carry-in.
template <typename T, int C, int CT = 0>
__device__ __forceinline__ void apply_carry_fwd(const bool has, const T pe, const T (&pV)[C],
                                                const T eT, const T (&VT)[C], T& eprev,
                                                T (&Lprev)[C]) {
    if (has) {
        eprev = pe;
        const Decay<T, C, CT> d(eT, pe);
#pragma unroll
        for (int c = 0; c < C; ++c) Lprev[c] = dfma<T>(d[c], VT[c], pV[c]);
    } else {
        eprev = eT;
#pragma unroll
        for (int c = 0; c < C; ++c) Lprev[c] = VT[c];
    }
}

template <typename T, int C, int CT = 0>
__device__ __forceinline__ void apply_carry_bwd(const bool has, const T nf, const T (&nW)[C],
                                                const T fT, const T (&WT)[C], T& enext,
                                                T (&Unext)[C]) {
    if (has) {
        enext = nf;
        const Decay<T, C, CT> d(nf, fT);
#pragma unroll
        for (int c = 0; c < C; ++c) Unext[c] = dfma<T>(d[c], WT[c], nW[c]);
    } else {
        enext = fT;
#pragma unroll
        for (int c = 0; c < C; ++c) Unext[c] = WT[c];
    }
}

}  // namespace lx
