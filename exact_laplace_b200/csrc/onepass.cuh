// onepass.cuh -- carries between tiles of a single-pass LAPLEX scan.
//
// A launch walks the (sorted or merged) sequence in tiles taken in order from
// an atomic ticket.  Each tile
//   1. scans itself and publishes its first/last anchors and its forward and
//      backward totals (flag 1),
//   2. looks back over the tiles to its left for the prefix carry, using an
//      inclusive prefix (flag 2) where one is published, and stopping as soon
//      as the decay exp(e_j - e_T) is exactly 0 (every term further left is
//      then exactly 0 too); then publishes its inclusive prefix,
//   3. looks ahead over at most LOOKAHEAD_TILES tiles to its right for the
//      suffix carry in the same way; then publishes its inclusive suffix,
//   4. finishes and writes its elements.
// A tile publishes its totals before it waits for anything and tiles start in
// ticket order, so a wait on a left neighbour always ends (that tile is
// running); a wait on a right neighbour ends while the look-ahead is shorter
// than the number of co-resident blocks.  Every wait is bounded: an expired
// look-back sets ST_TIMEOUT; a look-ahead that is too deep or expires marks the
// tile instead, and k_suffix_carries + a fix-up kernel complete it exactly.
#pragma once
#include "scan_core.cuh"

namespace lx {

constexpr uint32_t LOOKBACK_POLLS = 1u << 25;
constexpr uint32_t LOOKAHEAD_POLLS = 1u << 16;
constexpr int LOOKAHEAD_TILES = 64;

template <typename T>
struct OnePassWs {
    uint32_t* ctrl;   // [0] ticket, [1] number of marked tiles, then the flags below
    uint32_t* fflag;  // [ntiles] forward: 1 totals, 2 inclusive
    uint32_t* bflag;  // [ntiles] backward: 1 totals, 2 inclusive
    uint32_t* fix;    // [ntiles] list of deferred tiles (first ctrl[1] entries)
    T* tfirst;        // [ntiles] first anchor of each tile
    T* tlast;         // [ntiles] last anchor of each tile
    T* fagg;          // [ntiles*C] forward total (L at the tile's last element)
    T* finc;          // [ntiles*C] inclusive prefix at the tile's last element
    T* bagg;          // [ntiles*C] backward total (U at the tile's first element)
    T* binc;          // [ntiles*C] inclusive suffix at the tile's first element
    T* carB;          // [ntiles*C] exact suffix carry after each tile (marked tiles)
};

// Bytes of workspace OnePassWs needs (same carving order as onepass_carve).
inline size_t onepass_ws_bytes(int64_t ntiles, int C, size_t es) {
    return Carve::need((size_t)(2 + 3 * ntiles), 4) + 2 * Carve::need((size_t)ntiles, es) +
           5 * Carve::need((size_t)(ntiles * C), es);
}

template <typename T>
inline OnePassWs<T> onepass_carve(Carve& cv, int64_t ntiles, int C) {
    OnePassWs<T> W;
    W.ctrl = cv.take<uint32_t>(2 + 3 * ntiles);
    W.fflag = W.ctrl + 2;
    W.bflag = W.fflag + ntiles;
    W.fix = W.bflag + ntiles;
    W.tfirst = cv.take<T>(ntiles);
    W.tlast = cv.take<T>(ntiles);
    W.fagg = cv.take<T>(ntiles * C);
    W.finc = cv.take<T>(ntiles * C);
    W.bagg = cv.take<T>(ntiles * C);
    W.binc = cv.take<T>(ntiles * C);
    W.carB = cv.take<T>(ntiles * C);
    return W;
}

template <typename T>
inline cudaError_t onepass_reset(const OnePassWs<T>& W, int64_t ntiles, cudaStream_t st) {
    return cudaMemsetAsync(W.ctrl, 0, sizeof(uint32_t) * (2 + 3 * ntiles), st);
}

// Record tile t as deferred: its suffix carry is added after the scan.
template <typename T>
__device__ __forceinline__ void onepass_defer(const OnePassWs<T>& W, int64_t t) {
    const uint32_t slot = atomicAdd(&W.ctrl[1], 1u);
    W.fix[slot] = (uint32_t)t;
}

// Fix-up launches use a small fixed grid that walks the deferred-tile list.
constexpr int FIXUP_BLOCKS = 296;

// Run by ONE thread of the block owning tile t after the tile's local scan.
//   (tf, tW): first anchor and backward total;  (te, tV): last anchor and forward total
//   eT: anchor of the element before the tile;  fT: anchor of the element after it
// Out: acc = L at the element before the tile, accb = U at the element after it
// (zero and the tile marked when the look-ahead is deferred).
template <typename T, int C, int CT = 0>
__device__ __forceinline__ void onepass_carries(const OnePassWs<T>& W, const int64_t t,
                                                const int64_t ntiles, const T tf, const T (&tW)[C],
                                                const T te, const T (&tV)[C], const T eT,
                                                const T fT, T (&acc)[C], T (&accb)[C],
                                                uint32_t* status) {
    const bool first = t == 0, last = t == ntiles - 1;
    W.tfirst[t] = tf;
    W.tlast[t] = te;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        W.fagg[t * C + c] = tV[c];
        W.bagg[t * C + c] = tW[c];
        if (first) W.finc[c] = tV[c];
        if (last) W.binc[t * C + c] = tW[c];
    }
    st_release(&W.fflag[t], first ? 2u : 1u);
    st_release(&W.bflag[t], last ? 2u : 1u);
    // ---- look-back
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = T(0);
    for (int64_t j = t - 1; j >= 0; --j) {
        const uint32_t fl = wait_flag(&W.fflag[j], 1u, LOOKBACK_POLLS);
        if (fl == 0u) {
            set_status(status, ST_TIMEOUT);
            break;
        }
        const Decay<T, C, CT> f(__ldcg(&W.tlast[j]), eT);
        if (f.e == T(0) && (CT == 0 || f.t == T(0))) break;
        const T* src = (fl == 2u ? W.finc : W.fagg) + j * C;
#pragma unroll
        for (int c = 0; c < C; ++c) acc[c] = dfma<T>(f[c], __ldcg(src + c), acc[c]);
        if (fl == 2u) break;
    }
    if (!first) {
        const Decay<T, C, CT> d(eT, te);
#pragma unroll
        for (int c = 0; c < C; ++c) W.finc[t * C + c] = dfma<T>(d[c], acc[c], tV[c]);
        st_release(&W.fflag[t], 2u);
    }
    // ---- look-ahead
#pragma unroll
    for (int c = 0; c < C; ++c) accb[c] = T(0);
    bool defer = false;
    int depth = 0;
    for (int64_t j = t + 1; j < ntiles; ++j) {
        if (++depth > LOOKAHEAD_TILES) {
            defer = true;
            break;
        }
        const uint32_t fl = wait_flag(&W.bflag[j], 1u, LOOKAHEAD_POLLS);
        if (fl == 0u) {
            defer = true;
            break;
        }
        const Decay<T, C, CT> f(fT, __ldcg(&W.tfirst[j]));
        if (f.e == T(0) && (CT == 0 || f.t == T(0))) break;
        const T* src = (fl == 2u ? W.binc : W.bagg) + j * C;
#pragma unroll
        for (int c = 0; c < C; ++c) accb[c] = dfma<T>(f[c], __ldcg(src + c), accb[c]);
        if (fl == 2u) break;
    }
    if (defer) {
#pragma unroll
        for (int c = 0; c < C; ++c) accb[c] = T(0);
        onepass_defer(W, t);
    } else if (!last) {
        const Decay<T, C, CT> d(tf, fT);
#pragma unroll
        for (int c = 0; c < C; ++c) W.binc[t * C + c] = dfma<T>(d[c], accb[c], tW[c]);
        st_release(&W.bflag[t], 2u);
    }
}

// Exact suffix carries carB[t] = U at the first element of tile t+1, from the
// published backward totals and first anchors; one block, segments of tiles
// per thread, the block-wide backward scan across segments.  Exits at once
// when no tile is marked.
template <typename T, int C, int NT, int CT = 0>
__global__ void __launch_bounds__(NT) k_suffix_carries(OnePassWs<T> W, int64_t ntiles) {
    if (W.ctrl[1] == 0u) return;
    __shared__ BlockScanSmem<T, C, NT> smb;
    const int64_t per = (ntiles + NT - 1) / NT;
    const int64_t t0 = min((int64_t)threadIdx.x * per, ntiles);
    const int64_t t1 = min(t0 + per, ntiles);
    const T pad = W.tlast[ntiles - 1];
    T bf = pad, bW[C];
#pragma unroll
    for (int c = 0; c < C; ++c) bW[c] = T(0);
    for (int64_t t = t1 - 1; t >= t0; --t) {
        const T f = W.tfirst[t];
        const Decay<T, C, CT> d(f, bf);
#pragma unroll
        for (int c = 0; c < C; ++c)
            bW[c] = dfma<T>(t == t1 - 1 ? T(0) : d[c], bW[c], W.bagg[t * C + c]);
        bf = f;
    }
    bool has;
    T nf, nW[C], tf, tW[C];
    block_excl_bwd<T, C, NT, CT>(bf, bW, has, nf, nW, tf, tW, smb);
    T cf = has ? nf : pad, cw[C];
#pragma unroll
    for (int c = 0; c < C; ++c) cw[c] = has ? nW[c] : T(0);
    for (int64_t t = t1 - 1; t >= t0; --t) {
#pragma unroll
        for (int c = 0; c < C; ++c) W.carB[t * C + c] = cw[c];
        const T f = W.tfirst[t];
        const Decay<T, C, CT> d(f, cf);
#pragma unroll
        for (int c = 0; c < C; ++c) cw[c] = dfma<T>(d[c], cw[c], W.bagg[t * C + c]);
        cf = f;
    }
}

}  // namespace lx
