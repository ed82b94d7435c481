// sym_stream.cu -- the symmetric product for contiguous single-column input
// (x in sorted order): y = K x, K_ij = exp(-|s_i - s_j|) ("LAPLEX - La FFT dei
// Nuclei di Laplace Apprendibili", technical summary, §2.2 "Caso Simmetrico").
// This is the path of a pre-sorted product; inputs that need a gather through
// perm, several columns or phases use sym.cu.
//
// Three kernels, none of which waits for another block:
//   1. k_tile_local (streams s and x once, writes y once): each tile scans
//      itself with zero carries and writes y = Lloc + Uloc - x.  It records its
//      first and last anchors, its forward/backward totals and its reach: how
//      many elements from each end lie within CUT of that end's anchor.  A carry
//      from outside the tile reaches element r with a factor exp(-d), d >= the
//      distance from r to the tile's end anchor, and exp(-d) is exactly 0 for
//      d >= CUT (fp32: 104, below the smallest subnormal; fp64: 746), so
//      elements beyond the reach are untouched by the carries, bit for bit.
//   2. k_carry_blocks, k_carry_tiles: the exact carries into every tile from
//      the tile totals (block totals, then per-tile carries; the carry into a
//      block is a walk over the block totals that stops where exp of the gap is
//      exactly 0).
//   3. k_headtail: y_r += exp(eT - s_r) L_carry over each tile's head reach and
//      y_r += exp(s_r - fT) U_carry over its tail reach (read-modify-write of a
//      few percent of y; one warp per tile at a time).
#include <algorithm>

#include "laplex_impl.h"
#include "scan_core.cuh"

namespace lx {

constexpr int LT_NT = 512;     // threads per tile block
constexpr int CARRY_NT = 256;  // threads per carry block
constexpr int CARRY_PT = 8;    // tiles per carry thread
constexpr int CARRY_BT = CARRY_NT * CARRY_PT;
constexpr int HT_BLOCKS_PER_SM = 8;

template <typename T> struct LocalE;
template <> struct LocalE<float> { static constexpr int E = 16; };
template <> struct LocalE<double> { static constexpr int E = 8; };

template <typename T> struct Cut;
template <> struct Cut<float> { static constexpr float v = 104.0f; };
template <> struct Cut<double> { static constexpr double v = 746.0; };

struct TileStats {
    int32_t head;  // elements from the tile start within CUT of the first anchor
    int32_t tail;  // elements from the tile end within CUT of the last anchor
};

template <typename T>
struct LocalWs {
    T* tfirst;
    T* tlast;
    T* fagg;  // L at the tile's last element, tile only
    T* bagg;  // U at the tile's first element, tile only
    TileStats* st;
    T* bfe;   // per carry-block forward total: last anchor of the block, value
    T* bfv;
    T* bbf;   // per carry-block backward total: first anchor of the block, value
    T* bbv;
    T* carF;  // L at the element before tile t
    T* carB;  // U at the element after tile t
};

template <typename T, int E, int NT>
__global__ void __launch_bounds__(NT) k_tile_local(const T* __restrict__ s_, const T* __restrict__ x_,
                                                   T* __restrict__ y_, const int32_t* __restrict__ pout,
                                                   int64_t n, LocalWs<T> W) {
    constexpr int VN = V16<T>::N;
    constexpr int64_t TILE = (int64_t)NT * E;
    __shared__ BlockScanSmem<T, 1, NT> smf, smb;
    __shared__ int cnt_head, cnt_tail;
    __shared__ T sh_first, sh_last;
    const int64_t t = blockIdx.x;
    const int64_t tile0 = t * TILE;
    const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
    const bool full = r0 + E <= n;
    T s[E], v[E][1];
    {
        T xv[E];
        if (full) {
#pragma unroll
            for (int i = 0; i < E; i += VN) {
                ld16_stream<T>(s_ + r0 + i, &s[i]);
                ld16_stream<T>(x_ + r0 + i, &xv[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                s[i] = s_[min(r0 + i, n - 1)];
                xv[i] = r0 + i < n ? x_[r0 + i] : T(0);
            }
        }
#pragma unroll
        for (int i = 0; i < E; ++i) v[i][0] = xv[i];
    }
    if (threadIdx.x == 0) {
        cnt_head = 0;
        cnt_tail = 0;
        sh_first = s[0];
        sh_last = s_[min(tile0 + TILE, n) - 1];
    }
    T dl[E], fV[1], bW[1];
    chunk_aggregates<T, 1, E>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[1], te, tV[1], nf, nW[1], tf, tW[1];
    block_excl_fwd<T, 1, NT>(s[E - 1], fV, hf, pe, pV, te, tV, smf);  // its barriers publish sh_*
    block_excl_bwd<T, 1, NT>(s[0], bW, hb, nf, nW, tf, tW, smb);
    {
        int h = 0, q = 0;
        const T first = sh_first, lastv = sh_last;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const bool valid = r0 + i < n;
            h += (valid && s[i] - first < Cut<T>::v) ? 1 : 0;
            q += (valid && lastv - s[i] < Cut<T>::v) ? 1 : 0;
        }
        if (h) atomicAdd(&cnt_head, h);
        if (q) atomicAdd(&cnt_tail, q);
    }
    const T zero[1] = {T(0)};  // carries are added by k_headtail
    T eprev, Lprev[1], enext, Unext[1], out[E][1];
    apply_carry_fwd<T, 1>(hf, pe, pV, s[0], zero, eprev, Lprev);
    apply_carry_bwd<T, 1>(hb, nf, nW, s[E - 1], zero, enext, Unext);
    chunk_final<T, 1, E>(s, v, dl, eprev, Lprev, enext, Unext, out);
    T o[E];
#pragma unroll
    for (int i = 0; i < E; ++i) o[i] = out[i][0];
    if (full && pout == nullptr) {
#pragma unroll
        for (int i = 0; i < E; i += VN) st16_stream<T>(y_ + r0 + i, &o[i]);
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i)
            if (r0 + i < n) y_[pout ? (int64_t)pout[r0 + i] : r0 + i] = o[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        W.tfirst[t] = tf;
        W.tlast[t] = te;
        W.fagg[t] = tV[0];
        W.bagg[t] = tW[0];
        W.st[t].head = cnt_head;
        W.st[t].tail = cnt_tail;
    }
}

// This thread's forward and backward totals over its CARRY_PT tiles.
template <typename T>
__device__ __forceinline__ void carry_segment(const LocalWs<T>& W, int64_t t0, int64_t ntiles,
                                              T& fe, T (&fv)[1], T& bf, T (&bv)[1]) {
    const T pad = W.tlast[ntiles - 1];
    fe = pad;
    bf = pad;
    fv[0] = T(0);
    bv[0] = T(0);
    bool any = false;
    for (int k = 0; k < CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
        const T e = W.tlast[t];
        fv[0] = dfma<T>(any ? dexp<T>(fe - e) : T(0), fv[0], W.fagg[t]);
        fe = e;
        any = true;
    }
    any = false;
    for (int k = CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
        const T f = W.tfirst[t];
        bv[0] = dfma<T>(any ? dexp<T>(f - bf) : T(0), bv[0], W.bagg[t]);
        bf = f;
        any = true;
    }
}

template <typename T>
__global__ void __launch_bounds__(CARRY_NT) k_carry_blocks(LocalWs<T> W, int64_t ntiles) {
    __shared__ BlockScanSmem<T, 1, CARRY_NT> smf, smb;
    const int64_t t0 = (int64_t)blockIdx.x * CARRY_BT + (int64_t)threadIdx.x * CARRY_PT;
    T fe, fv[1], bf, bv[1];
    carry_segment<T>(W, t0, ntiles, fe, fv, bf, bv);
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
    T fe, fv[1], bf, bv[1];
    carry_segment<T>(W, t0, ntiles, fe, fv, bf, bv);
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
    for (int k = 0; k < CARRY_PT; ++k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) break;
        W.carF[t] = t == 0 ? T(0) : cv;
        const T e = W.tlast[t];
        cv = dfma<T>(dexp<T>(ce - e), cv, W.fagg[t]);
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
    for (int k = CARRY_PT - 1; k >= 0; --k) {
        const int64_t t = t0 + k;
        if (t >= ntiles) continue;
        W.carB[t] = t == ntiles - 1 ? T(0) : cw;
        const T f = W.tfirst[t];
        cw = dfma<T>(dexp<T>(f - cf), cw, W.bagg[t]);
        cf = f;
    }
}

template <typename T, int TILE>
__global__ void __launch_bounds__(256) k_headtail(const T* __restrict__ s_, T* __restrict__ y_,
                                                  const int32_t* __restrict__ pout, int64_t n,
                                                  LocalWs<T> W, int64_t ntiles) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < ntiles;
         t += warps) {
        const int64_t b = t * TILE, e = min(b + (int64_t)TILE, n);
        const TileStats stt = W.st[t];
        if (t > 0) {
            const T c = W.carF[t];
            if (c != T(0)) {
                const T eT = s_[b - 1];
                for (int64_t r = b + lane; r < b + stt.head; r += 32) {
                    const T f = dexp<T>(eT - s_[r]);
                    if (f != T(0)) y_[pout ? (int64_t)pout[r] : r] += f * c;
                }
            }
        }
        __syncwarp();
        if (t < ntiles - 1) {
            const T c = W.carB[t];
            if (c != T(0)) {
                const T fT = s_[e];
                for (int64_t r = e - 1 - lane; r >= e - stt.tail; r -= 32) {
                    const T f = dexp<T>(s_[r] - fT);
                    if (f != T(0)) y_[pout ? (int64_t)pout[r] : r] += f * c;
                }
            }
        }
        __syncwarp();
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
    W.st = cv.take<TileStats>(ntiles);
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
    return 6 * Carve::need((size_t)ntiles, es) + Carve::need((size_t)ntiles, sizeof(TileStats)) +
           4 * Carve::need((size_t)nb, es);
}

template <typename T>
cudaError_t stream_run(const T* s, const T* x, T* y, const int32_t* pout, int64_t n, void* ws,
                       size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    (void)status;  // no inter-block waits, nothing to report
    if (n == 0) return cudaSuccess;
    constexpr int E = LocalE<T>::E;
    constexpr int TILE = LT_NT * E;
    const int64_t ntiles = local_ntiles<T>(n);
    const int64_t nb = (ntiles + CARRY_BT - 1) / CARRY_BT;
    Carve cv(ws, ws_bytes);
    LocalWs<T> W = local_carve<T>(cv, ntiles);
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
    k_tile_local<T, E, LT_NT><<<(unsigned)ntiles, LT_NT, 0, st>>>(s, x, y, pout, n, W);
    k_carry_blocks<T><<<(unsigned)nb, CARRY_NT, 0, st>>>(W, ntiles);
    k_carry_tiles<T><<<(unsigned)nb, CARRY_NT, 0, st>>>(W, ntiles, nb);
    const int64_t htb =
        std::max<int64_t>(1, std::min<int64_t>((ntiles + 7) / 8, (int64_t)sms_cache[dev] * HT_BLOCKS_PER_SM));
    k_headtail<T, TILE><<<(unsigned)htb, 256, 0, st>>>(s, y, pout, n, W, ntiles);
    return cudaGetLastError();
}

template cudaError_t stream_run<float>(const float*, const float*, float*, const int32_t*, int64_t,
                                       void*, size_t, uint32_t*, cudaStream_t);
template cudaError_t stream_run<double>(const double*, const double*, double*, const int32_t*,
                                        int64_t, void*, size_t, uint32_t*, cudaStream_t);

}  // namespace lx
