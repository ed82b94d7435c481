// sym_stream.cu -- the symmetric product for contiguous single-column input
// (x in sorted order): y = K x, K_ij = exp(-|s_i - s_j|) ("LAPLEX - La FFT dei
// Nuclei di Laplace Apprendibili", technical summary, §2.2 "Caso Simmetrico").
// x in sorted order, or in the caller's order with perm (gathered on load, y
// scattered back); several columns, phases or a scale use sym.cu.
//
// Three kernels, none of which waits for another block:
//   1. k_tile_local (streams s and x once, writes y once; persistent blocks,
//      every tile's s and x brought into a 2-stage shared-memory ring by 1-D
//      bulk copies (TMA), the next tile loading while one is computed): each tile scans
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
template <> struct LocalE<float> { static constexpr int E = 12; };   // 3 x 16 bytes
template <> struct LocalE<double> { static constexpr int E = 6; };   // 3 x 16 bytes
constexpr int LT_STAGES = 2;

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

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}
constexpr uint32_t MBAR_POLLS = 1u << 20;
// bounded wait for phase `parity` of *bar; false if it never completed
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t it = 0; it < MBAR_POLLS; ++it)
        if (mbar_test(bar, parity)) return true;
    return false;
}
// orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses to the same memory
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Persistent: block b handles tiles b, b + G, b + 2G, ...; the tile of
// iteration i sits in ring stage i % S.  Each thread owns E consecutive
// elements, an odd number of 16-byte units, so 128-bit shared loads of a warp
// touch distinct banks.  The ragged last tile (if any) is read from global.
// GATHER: x is in the caller's order and y goes back to it through perm (the
// ring then holds s and perm; x is gathered from global memory).
template <typename T, int E, int NT, int S, bool GATHER>
__global__ void __launch_bounds__(NT, 2) k_tile_local(const T* __restrict__ s_, const T* __restrict__ x_,
                                                      T* __restrict__ y_, const int32_t* __restrict__ perm,
                                                      int64_t n, int64_t ntiles, LocalWs<T> W,
                                                      uint32_t* status) {
    constexpr int VN = V16<T>::N;
    constexpr int64_t TILE = (int64_t)NT * E;
    static_assert(((E / VN) & 1) == 1, "E must be an odd number of 16-byte units");
    extern __shared__ __align__(128) unsigned char dyn[];
    T* ring_s = reinterpret_cast<T*>(dyn);
    T* ring_x = ring_s + S * TILE;                              // !GATHER
    int32_t* ring_p = reinterpret_cast<int32_t*>(ring_s + S * TILE);  // GATHER
    const int32_t* pout = perm;
    __shared__ __align__(8) uint64_t full[S];
    __shared__ BlockScan2Smem<T, 1, NT> sm2;
    __shared__ int cnt_head, cnt_tail;
    __shared__ T sh_first, sh_last;
    const int64_t G = gridDim.x;

    auto issue = [&](int st, int64_t t) {  // one thread
        if ((t + 1) * TILE <= n) {
            if constexpr (GATHER) {
                mbar_expect_tx(&full[st], (uint32_t)(TILE * (sizeof(T) + sizeof(int32_t))));
                bulk_g2s(ring_s + st * TILE, s_ + t * TILE, (uint32_t)(TILE * sizeof(T)), &full[st]);
                bulk_g2s(ring_p + st * TILE, perm + t * TILE, (uint32_t)(TILE * sizeof(int32_t)), &full[st]);
            } else {
                mbar_expect_tx(&full[st], (uint32_t)(2 * TILE * sizeof(T)));
                bulk_g2s(ring_s + st * TILE, s_ + t * TILE, (uint32_t)(TILE * sizeof(T)), &full[st]);
                bulk_g2s(ring_x + st * TILE, x_ + t * TILE, (uint32_t)(TILE * sizeof(T)), &full[st]);
            }
        } else {
            mbar_arrive(&full[st]);  // ragged tile: read from global
        }
    };
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) mbar_init(&full[st], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int st = 0; st < S - 1; ++st) {
            const int64_t t = blockIdx.x + st * G;
            if (t < ntiles) issue(st, t);
        }
    }
    __syncthreads();
    for (int64_t i = 0;; ++i) {
        const int64_t t = blockIdx.x + i * G;
        if (t >= ntiles) break;
        const int st = (int)(i % S);
        const uint32_t ph = (uint32_t)((i / S) & 1);
        const bool landed = mbar_wait(&full[st], ph);
        if (__syncthreads_or(!landed)) {  // a copy never completed: report and stop
            if (threadIdx.x == 0) {
                set_status(status, ST_TIMEOUT);
                for (int k = 1; k < S - 1; ++k) {
                    const int64_t t2 = blockIdx.x + (i + k) * G;
                    if (t2 < ntiles) mbar_wait(&full[(i + k) % S], (uint32_t)(((i + k) / S) & 1));
                }
            }
            return;
        }
        const int64_t tile0 = t * TILE;
        const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
        const bool ragged = tile0 + TILE > n;
        T s[E], v[E][1];
        int32_t pr[GATHER ? E : 1];
        {
            T xv[E];
            if (!ragged) {
                const T* ps = ring_s + st * TILE + threadIdx.x * E;
#pragma unroll
                for (int k = 0; k < E; k += VN) ld16<T>(ps + k, &s[k]);
                if constexpr (GATHER) {
                    const int32_t* pp = ring_p + st * TILE + threadIdx.x * E;
#pragma unroll
                    for (int k = 0; k < E; ++k) pr[k] = pp[k];
#pragma unroll
                    for (int k = 0; k < E; ++k) xv[k] = __ldg(x_ + pr[k]);
                } else {
                    const T* px = ring_x + st * TILE + threadIdx.x * E;
#pragma unroll
                    for (int k = 0; k < E; k += VN) ld16<T>(px + k, &xv[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const int64_t r = r0 + k;
                    s[k] = s_[min(r, n - 1)];
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
        if (threadIdx.x == 0) {
            cnt_head = 0;
            cnt_tail = 0;
            sh_first = ragged ? s_[tile0] : ring_s[st * TILE];
            sh_last = ragged ? s_[n - 1] : ring_s[st * TILE + TILE - 1];
        }
        // Every thread's reads of earlier stages are ordered before the TMA
        // writes that refill them (generic -> async proxy).  The stage refilled
        // now is the one of the previous iteration, read before at least one
        // earlier barrier; the stage just read is refilled one iteration later.
        fence_proxy_async();
        __syncthreads();
        if (threadIdx.x == 0) {
            const int64_t t2 = blockIdx.x + (i + S - 1) * G;
            if (t2 < ntiles) issue((int)((i + S - 1) % S), t2);
        }
        T dl[E], fV[1], bW[1];
        chunk_aggregates<T, 1, E>(s, v, dl, fV, bW);
        bool hf, hb;
        T pe, pV[1], te, tV[1], nf, nW[1], tf, tW[1];
        block_excl_both<T, 1, NT>(s[E - 1], fV, s[0], bW, hf, pe, pV, te, tV, hb, nf, nW, tf, tW, sm2);
        {
            // reach counts; the chunk is sorted, so only a chunk that straddles
            // the cut needs a per-element count
            const T first = sh_first, lastv = sh_last;
            const int valid = (int)min((int64_t)E, max((int64_t)0, n - r0));
            int h = 0, q = 0;
            if (valid > 0) {
                T sl = s[0];  // last valid anchor of the chunk (static indexing only)
#pragma unroll
                for (int k = 1; k < E; ++k)
                    if (k < valid) sl = s[k];
                if (sl - first < Cut<T>::v) h = valid;
                else if (s[0] - first < Cut<T>::v)
#pragma unroll
                    for (int k = 0; k < E; ++k) h += (k < valid && s[k] - first < Cut<T>::v) ? 1 : 0;
                if (lastv - s[0] < Cut<T>::v) q = valid;
                else if (lastv - sl < Cut<T>::v)
#pragma unroll
                    for (int k = 0; k < E; ++k) q += (k < valid && lastv - s[k] < Cut<T>::v) ? 1 : 0;
            }
            if (h) atomicAdd(&cnt_head, h);
            if (q) atomicAdd(&cnt_tail, q);
        }
        // no carries from outside the tile here (k_headtail adds them): a thread
        // without a neighbour on one side starts that recurrence from 0
        T eprev = hf ? pe : s[0], Lprev[1] = {hf ? pV[0] : T(0)};
        T enext = hb ? nf : s[E - 1], Unext[1] = {hb ? nW[0] : T(0)};
        T out[E][1];
        chunk_final<T, 1, E>(s, v, dl, eprev, Lprev, enext, Unext, out);
        T o[E];
#pragma unroll
        for (int k = 0; k < E; ++k) o[k] = out[k][0];
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
        __syncthreads();  // the reach counters are complete
        if (threadIdx.x == 0) {
            W.tfirst[t] = tf;
            W.tlast[t] = te;
            W.fagg[t] = tV[0];
            W.bagg[t] = tW[0];
            W.st[t].head = cnt_head;
            W.st[t].tail = cnt_tail;
        }
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
    {
        auto launch = [&](auto kern, size_t smem, const int32_t* pp) -> cudaError_t {
            static int per_sm[64][2] = {{0}};
            const int which = pp ? 1 : 0;
            if (per_sm[dev][which] == 0) {
                cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (r != cudaSuccess) return r;
                int per = 0;
                r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, LT_NT, smem);
                if (r != cudaSuccess) return r;
                per_sm[dev][which] = std::max(1, per);
            }
            const int64_t grid = std::min<int64_t>(ntiles, (int64_t)per_sm[dev][which] * sms_cache[dev]);
            profile_before(st);
            kern<<<(unsigned)grid, LT_NT, smem, st>>>(s, x, y, pp, n, ntiles, W, status);
            profile_after(st);
            return cudaGetLastError();
        };
        if (pout == nullptr)
            e = launch(k_tile_local<T, E, LT_NT, LT_STAGES, false>,
                       (size_t)LT_STAGES * TILE * (2 * sizeof(T)), nullptr);
        else
            e = launch(k_tile_local<T, E, LT_NT, LT_STAGES, true>,
                       (size_t)LT_STAGES * TILE * (sizeof(T) + sizeof(int32_t)), pout);
        if (e != cudaSuccess) return e;
    }
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
