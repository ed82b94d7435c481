// sym.cu -- symmetric and phased-symmetric LAPLEX products on sorted anchors.
//
//   y = K x,   K_ij = exp(-|s_i - s_j|)                      (summary §2.1, §2.2)
//   y = K x,   K_ij = exp(-|s_i - s_j|) cos(phi_i - phi_j)   (phased, §2.1)
//
// The phased product runs two unphased channels, cos(phi) x and sin(phi) x, and
// recombines them with cos(phi_i) and sin(phi_i) (cos(p - q) = cos p cos q +
// sin p sin q).  Each channel is the recurrence pair of scan_core.cuh.
//
// Paths:
//   * one column, x in sorted order or gathered through perm: sym_stream.cu;
//   * several columns, phases or a scale: the wait-free three-kernel scheme of
//     threepass.cuh with the SymTP policy below;
//   * laplex_matvec_sym_noalloc: the three-phase reduce-then-scan below
//     (k_sym_reduce, the carry kernels of threepass.cuh, k_sym_final) with a
//     fixed scratch array.
#include <algorithm>

#include "laplex_impl.h"
#include "threepass.cuh"

namespace lx {

constexpr int SYM_NT = 256;


// Load the chunk [r0, r0 + E) : anchors, channel values, and (phased) cos/sin.
template <typename T, int NCOL, bool PHASED, int E>
__device__ __forceinline__ void sym_load(const SymArgs<T>& A, const int64_t r0, T (&s)[E],
                                         T (&v)[E][PHASED ? 2 * NCOL : NCOL], T (&cph)[E],
                                         T (&sph)[E]) {
    constexpr int VN = V16<T>::N;
    const int64_t n = A.n;
    const bool full = r0 + E <= n;
    if (full) {
#pragma unroll
        for (int i = 0; i < E; i += VN) ld16_stream<T>(A.s + r0 + i, &s[i]);
    } else {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = A.s[min(r0 + i, n - 1)];
    }
    if (!PHASED && NCOL == 1 && full && A.pin == nullptr && A.D == nullptr && A.ldx == 1) {
        T t[E];
#pragma unroll
        for (int i = 0; i < E; i += VN) ld16_stream<T>(A.x + r0 + i, &t[i]);
#pragma unroll
        for (int i = 0; i < E; ++i) v[i][0] = t[i];
        return;
    }
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int64_t r = r0 + i;
        if (r < n) {
            const int64_t row = A.pin ? (int64_t)A.pin[r] : r;
            const int64_t ar = A.paux ? (int64_t)A.paux[r] : r;
            const T dsc = A.D ? A.D[ar] : T(1);
            if (PHASED) psincos<T>(A.phi[ar], &sph[i], &cph[i]);
            const T* xr = A.x + row * A.ldx + A.col0;
            T xv[NCOL];
            if (NCOL >= VN && (NCOL % VN) == 0 && A.ncol == NCOL && (A.ldx % VN) == 0 &&
                (A.col0 % VN) == 0) {
#pragma unroll
                for (int c = 0; c < NCOL; c += VN) ld16<T>(xr + c, &xv[c]);
            } else {
#pragma unroll
                for (int c = 0; c < NCOL; ++c) xv[c] = c < A.ncol ? xr[c] : T(0);
            }
#pragma unroll
            for (int c = 0; c < NCOL; ++c) {
                const T val = xv[c] * dsc;
                if (PHASED) {
                    v[i][2 * c] = cph[i] * val;
                    v[i][2 * c + 1] = sph[i] * val;
                } else {
                    v[i][c] = val;
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < (PHASED ? 2 * NCOL : NCOL); ++c) v[i][c] = T(0);
            cph[i] = T(0);
            sph[i] = T(0);
        }
    }
}

template <typename T, int NCOL, bool PHASED, int E>
__device__ __forceinline__ void sym_store(const SymArgs<T>& A, const int64_t r0,
                                          const T (&out)[E][PHASED ? 2 * NCOL : NCOL],
                                          const T (&cph)[E], const T (&sph)[E]) {
    constexpr int VN = V16<T>::N;
    const int64_t n = A.n;
    const bool full = r0 + E <= n;
    if (!PHASED && NCOL == 1 && full && A.pout == nullptr && A.ldy == 1) {
        T t[E];
#pragma unroll
        for (int i = 0; i < E; ++i) t[i] = out[i][0];
#pragma unroll
        for (int i = 0; i < E; i += VN) st16_stream<T>(A.y + r0 + i, &t[i]);
        return;
    }
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int64_t r = r0 + i;
        if (r < n) {
            const int64_t row = A.pout ? (int64_t)A.pout[r] : r;
            T* yr = A.y + row * A.ldy + A.col0;
            T yv[NCOL];
#pragma unroll
            for (int c = 0; c < NCOL; ++c)
                yv[c] = PHASED ? cph[i] * out[i][2 * c] + sph[i] * out[i][2 * c + 1] : out[i][c];
            if (NCOL >= VN && (NCOL % VN) == 0 && A.ncol == NCOL && (A.ldy % VN) == 0 &&
                (A.col0 % VN) == 0) {
#pragma unroll
                for (int c = 0; c < NCOL; c += VN) st16<T>(yr + c, &yv[c]);
            } else {
#pragma unroll
                for (int c = 0; c < NCOL; ++c)
                    if (c < A.ncol) yr[c] = yv[c];
            }
        }
    }
}

template <typename T, int NCOL, bool PHASED, int E, int NT>
__global__ void __launch_bounds__(NT) k_sym_reduce(SymArgs<T> A, TPWs<T, PHASED ? 2 * NCOL : NCOL> W) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    __shared__ BlockScanSmem<T, C, NT> smf, smb;
    const int64_t r0 = (int64_t)blockIdx.x * (NT * E) + (int64_t)threadIdx.x * E;
    T s[E], v[E][C], cph[E], sph[E], dl[E], fV[C], bW[C];
    sym_load<T, NCOL, PHASED, E>(A, r0, s, v, cph, sph);
    chunk_aggregates<T, C, E>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    block_excl_fwd<T, C, NT>(s[E - 1], fV, hf, pe, pV, te, tV, smf);
    block_excl_bwd<T, C, NT>(s[0], bW, hb, nf, nW, tf, tW, smb);
    if (threadIdx.x == 0) {
        W.tfirst[blockIdx.x] = tf;
        W.tlast[blockIdx.x] = te;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            W.fagg[(int64_t)blockIdx.x * C + c] = tV[c];
            W.bagg[(int64_t)blockIdx.x * C + c] = tW[c];
        }
        if (blockIdx.x == 0) *W.redo_count = 1u;  // every tile takes the carry kernels
    }
}

}  // namespace lx

#include "cols.cuh"

namespace lx {

template <typename T, int NCOL, bool PHASED, int E, int NT>
__global__ void __launch_bounds__(NT) k_sym_final(SymArgs<T> A, const T* __restrict__ carF,
                                                  const T* __restrict__ carB) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    __shared__ BlockScanSmem<T, C, NT> smf, smb;
    const int64_t tile0 = (int64_t)blockIdx.x * (NT * E);
    const int64_t r0 = tile0 + (int64_t)threadIdx.x * E;
    T s[E], v[E][C], cph[E], sph[E], dl[E], fV[C], bW[C];
    sym_load<T, NCOL, PHASED, E>(A, r0, s, v, cph, sph);
    chunk_aggregates<T, C, E>(s, v, dl, fV, bW);
    bool hf, hb;
    T pe, pV[C], te, tV[C], nf, nW[C], tf, tW[C];
    block_excl_fwd<T, C, NT>(s[E - 1], fV, hf, pe, pV, te, tV, smf);
    block_excl_bwd<T, C, NT>(s[0], bW, hb, nf, nW, tf, tW, smb);
    const int64_t n = A.n;
    const T eT = tile0 > 0 ? A.s[tile0 - 1] : A.s[0];
    const T fT = tile0 + NT * E < n ? A.s[tile0 + NT * E] : A.s[n - 1];
    T VT[C], WT[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        VT[c] = carF[(int64_t)blockIdx.x * C + c];
        WT[c] = carB[(int64_t)blockIdx.x * C + c];
    }
    T eprev, Lprev[C], enext, Unext[C], out[E][C];
    apply_carry_fwd<T, C>(hf, pe, pV, eT, VT, eprev, Lprev);
    apply_carry_bwd<T, C>(hb, nf, nW, fT, WT, enext, Unext);
    chunk_final<T, C, E>(s, v, dl, eprev, Lprev, enext, Unext, out);
    sym_store<T, NCOL, PHASED, E>(A, r0, out, cph, sph);
}


// ------------------------------------------------------------------ wait-free path
// Policy of threepass.cuh for the symmetric/phased product with B columns,
// an optional scale D and gather/scatter through perm (sym_load/sym_store).
template <typename T_, int NCOL_, bool PHASED_, int E_, int NT_>
struct SymTP {
    using T = T_;
    static constexpr int NCOL = NCOL_, C = PHASED_ ? 2 * NCOL_ : NCOL_, CT = 0, E = E_, NT = NT_;
    // halos of 192 (fp32: they span CUT = 88 at spacings above 0.47, and
    // across runs of up to 64 equal anchors); fp64 (CUT = 746) would need
    // several times more: none
    static constexpr int H = sizeof(T_) == 4 ? 192 : 0;
    // streamed first pass (k_tp_ring: one column in sorted order, no scale):
    // the value arrays x (and phi), 2 stages, 3 blocks per SM (fp64: 2)
    static constexpr int NIN = PHASED_ ? 2 : 1, S = 2, MINB = sizeof(T_) == 8 ? 2 : 3;
    SymArgs<T> A;
    int64_t n;
    const T* s;
    struct Aux {
        T cph[E], sph[E];
    };
    __device__ __forceinline__ const T* ring_in(int a) const { return a == 0 ? A.x : A.phi; }
    __device__ __forceinline__ void value(const T (&xe)[NIN], T (&vv)[C]) const {
        if constexpr (PHASED_) {
            T sp, cp;
            psincos<T>(xe[1], &sp, &cp);
            vv[0] = cp * xe[0];
            vv[1] = sp * xe[0];
        } else {
            vv[0] = xe[0];
        }
    }
    __device__ __forceinline__ void value_chunk(const T (&xe)[NIN], T (&vv)[C], Aux& a, int k) const {
        if constexpr (PHASED_) {
            T sp, cp;
            psincos<T>(xe[1], &sp, &cp);
            a.cph[k] = cp;
            a.sph[k] = sp;
            vv[0] = cp * xe[0];
            vv[1] = sp * xe[0];
        } else {
            vv[0] = xe[0];
        }
    }
    __device__ __forceinline__ void load(int64_t r0, T (&sv)[E], T (&v)[E][C], Aux& a) const {
        sym_load<T, NCOL, PHASED_, E>(A, r0, sv, v, a.cph, a.sph);
    }
    __device__ __forceinline__ void finish(int64_t r0, const T (&sv)[E], const T (&v)[E][C],
                                           T (&dl)[E], T eprev, const T (&Lp)[C], T enext,
                                           const T (&Un)[C], Aux& a) const {
        T out[E][C];
        chunk_final<T, C, E>(sv, v, dl, eprev, Lp, enext, Un, out);
        sym_store<T, NCOL, PHASED_, E>(A, r0, out, a.cph, a.sph);
    }
    __device__ __forceinline__ void load1(int64_t j, T& sj, T (&vj)[C]) const {
        sj = A.s[j];
        const int64_t row = A.pin ? (int64_t)A.pin[j] : j;
        const int64_t ar = A.paux ? (int64_t)A.paux[j] : j;
        const T dsc = A.D ? A.D[ar] : T(1);
        T sp = T(0), cp = T(1);
        if (PHASED_) psincos<T>(A.phi[ar], &sp, &cp);
        const T* xr = A.x + row * A.ldx + A.col0;
#pragma unroll
        for (int c = 0; c < NCOL; ++c) {
            const T val = (c < A.ncol ? xr[c] : T(0)) * dsc;
            if (PHASED_) {
                vj[2 * c] = cp * val;
                vj[2 * c + 1] = sp * val;
            } else {
                vj[c] = val;
            }
        }
    }
};

// ------------------------------------------------------------------ host side
// elements per thread of the products with four or more channels
#ifndef LX_SYM_E_WIDE
#define LX_SYM_E_WIDE 4
#endif
struct SymPlan {
    int ncol;  // template columns per pass
    int C;     // channels per pass
    int E;     // elements per thread
    int64_t tile;
    int64_t ntiles;
    int64_t groups;
};

static SymPlan sym_plan(int64_t n, int64_t B, bool phased, int f64) {
    SymPlan p;
    const int maxcol = phased ? 4 : 8;
    int nc = 1;
    while (nc < B && nc < maxcol) nc <<= 1;
    p.ncol = nc;
    p.C = phased ? 2 * nc : nc;
    if (p.C == 1) p.E = f64 ? 8 : 16;
    else if (p.C == 2) p.E = 8;
    else p.E = LX_SYM_E_WIDE;
    p.tile = (int64_t)SYM_NT * p.E;
    p.ntiles = (n + p.tile - 1) / p.tile;
    p.groups = (B + nc - 1) / nc;
    return p;
}

size_t sym_ws_bytes(int64_t n, int64_t B, bool phased, int f64) {
    const SymPlan p = sym_plan(n, B, phased, f64);
    const size_t a = tp_ws_bytes(p.ntiles, p.C, f64 ? 8 : 4);
    const size_t b = (!phased && B == 1) ? stream_ws_bytes(n, f64) : 0;
    const size_t c = phased ? 0 : cols_ws_bytes(n, B, f64);
    return std::max(a, std::max(b, c));
}

template <typename T, int NCOL, bool PHASED, int E>
static cudaError_t sym_launch(const SymArgs<T>& A, int64_t ntiles, TPWs<T, PHASED ? 2 * NCOL : NCOL> W,
                              cudaStream_t st) {
    constexpr int C = PHASED ? 2 * NCOL : NCOL;
    const int64_t nb = (ntiles + TP_CARRY_BT - 1) / TP_CARRY_BT;
    k_sym_reduce<T, NCOL, PHASED, E, SYM_NT><<<(unsigned)ntiles, SYM_NT, 0, st>>>(A, W);
    // the per-block totals are read only when there is more than one carry block
    if (nb > 1) k_tp_carry_blocks<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles);
    k_tp_carry_tiles<T, C, 0><<<(unsigned)nb, TP_CARRY_NT, 0, st>>>(W, ntiles, nb);
    k_sym_final<T, NCOL, PHASED, E, SYM_NT><<<(unsigned)ntiles, SYM_NT, 0, st>>>(A, W.carF, W.carB);
    return cudaGetLastError();
}

template <typename T>
cudaError_t sym_run(SymArgs<T> A, int64_t B, bool phased, void* ws, size_t ws_bytes,
                    cudaStream_t st) {
    if (A.n == 0) return cudaSuccess;
    // single-column input in sorted order, or gathered through perm: the wait-free kernels
    if (!phased && B == 1 && A.pin == A.pout && A.D == nullptr && A.ldx == 1 && A.ldy == 1)
        return stream_run<T>(A.s, A.x, A.y, A.pout, A.n, ws, ws_bytes, A.status, st);
    // 2, 4 or 8 columns in sorted order without a scale: the column-parallel kernels
    if (!phased && cols_supported(B) && A.pin == nullptr && A.pout == nullptr && A.D == nullptr && A.ldx == B &&
        A.ldy == B)
        return cols_run<T>(A.s, A.n, A.x, A.y, B, ws, ws_bytes, st);
    const SymPlan p = sym_plan(A.n, B, phased, sizeof(T) == 8);
    for (int64_t g = 0; g < p.groups; ++g) {
        A.col0 = g * p.ncol;
        A.ncol = (int)std::min<int64_t>(p.ncol, B - A.col0);
        cudaError_t e;
        constexpr bool D = sizeof(T) == 8;
        // one column in sorted order without a scale: the streamed (TMA ring) first pass
        const bool ring = p.ncol == 1 && B == 1 && A.pin == nullptr && A.pout == nullptr && A.paux == nullptr &&
                          A.D == nullptr && A.ldx == 1 && A.ldy == 1;
        auto run = [&](auto pol) {
            pol.A = A;
            pol.n = A.n;
            pol.s = A.s;
            if constexpr (decltype(pol)::NCOL == 1)
                if (ring) return tp_run_ring(pol, ws, ws_bytes, A.status, st);
            return tp_run(pol, ws, ws_bytes, st);
        };
        if (!phased) {
            switch (p.ncol) {
                case 1: e = run(SymTP<T, 1, false, D ? 8 : 16, SYM_NT>{}); break;
                case 2: e = run(SymTP<T, 2, false, 8, SYM_NT>{}); break;
                case 4: e = run(SymTP<T, 4, false, LX_SYM_E_WIDE, SYM_NT>{}); break;
                default: e = run(SymTP<T, 8, false, LX_SYM_E_WIDE, SYM_NT>{}); break;
            }
        } else {
            switch (p.ncol) {
                case 1: e = run(SymTP<T, 1, true, 8, SYM_NT>{}); break;
                case 2: e = run(SymTP<T, 2, true, LX_SYM_E_WIDE, SYM_NT>{}); break;
                default: e = run(SymTP<T, 4, true, LX_SYM_E_WIDE, SYM_NT>{}); break;
            }
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template cudaError_t sym_run<float>(SymArgs<float>, int64_t, bool, void*, size_t, cudaStream_t);
template cudaError_t sym_run<double>(SymArgs<double>, int64_t, bool, void*, size_t, cudaStream_t);

}  // namespace lx

// ------------------------------------------------------------------ no-alloc variant
// laplex_matvec_sym_noalloc: the three-phase symmetric product (fp32, B = 1)
// with its per-tile scratch in a fixed device array instead of a caller
// workspace, for callers that cannot allocate device memory.
#include <cuda.h>

#include <mutex>

#include "laplex.h"

namespace lx {

constexpr int64_t NOALLOC_TILE = (int64_t)SYM_NT * 16;           // elements per tile (fp32, B = 1)
constexpr int64_t NOALLOC_MAX_TILES = (int64_t)1 << 18;          // n <= 2^30
constexpr int64_t NOALLOC_MAX_CBLK = NOALLOC_MAX_TILES / TP_CARRY_BT;  // carry blocks
constexpr size_t NOALLOC_BYTES = 4 * NOALLOC_MAX_TILES * sizeof(float) + 4096;  // 4 MiB + 4 KiB
static_assert(4 * NOALLOC_MAX_CBLK * sizeof(float) + sizeof(uint32_t) <= 4096, "carry-block records");

// Per tile: first and last anchor, forward and backward totals (the carry
// kernels overwrite the totals with the carries into each tile, in place);
// per carry block: its four totals; one gate word.  Every call writes each
// entry it reads, so nothing here needs clearing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[NOALLOC_MAX_DEVICES];
static CUcontext g_noalloc_ctx[NOALLOC_MAX_DEVICES];

// The current context (NULL if none or unknown), through the driver entry
// point that the runtime hands out, so the library needs no link to the driver.
static CUcontext current_context() {
    using GetCtx = CUresult (*)(CUcontext*);
    static GetCtx fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<GetCtx>(f);
    }();
    CUcontext ctx = nullptr;
    if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    return ctx;
}

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up with
// cudaGetSymbolAddress, once per device and context: a device reset gives the
// device a new primary context (and reloads the module), and the first call in
// the new context looks the address up again.
static cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    CUcontext ctx = current_context();
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the primary context current
        if (e != cudaSuccess) return e;
        ctx = current_context();
        g_noalloc_ptr[dev] = p;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace lx

extern "C" laplex_status laplex_matvec_sym_noalloc(const float* sorted, const int32_t* perm,
                                                   int64_t n, const float* x, float* y,
                                                   void* stream) {
    using namespace lx;
    if (n < 0 || n > NOALLOC_MAX_TILES * NOALLOC_TILE) {
        set_last_error("laplex_matvec_sym_noalloc: n = %lld outside [0, 2^30] (the fixed "
                                 "scratch holds 2^18 tiles of 4096 anchors)", (long long)n);
        return LAPLEX_EINVAL;
    }
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (n > 0 && (!sorted || !x || !y || !al(sorted) || !al(x) || !al(y) || (perm && !al(perm)))) {
        set_last_error("laplex_matvec_sym_noalloc: sorted, x and y must be non-NULL and "
                                 "16-byte aligned (perm too, when given)");
        return LAPLEX_EINVAL;
    }
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) {
        set_last_error("laplex_matvec_sym_noalloc: scratch set-up: %s", cudaGetErrorString(e));
        return LAPLEX_ECUDA;
    }
    if (n == 0) {
        set_last_error("");
        return LAPLEX_OK;
    }
    const int64_t ntiles = (n + NOALLOC_TILE - 1) / NOALLOC_TILE;
    float* base = static_cast<float*>(scratch);
    TPWs<float, 1> W;
    W.tfirst = base;
    W.tlast = base + NOALLOC_MAX_TILES;
    W.fagg = base + 2 * NOALLOC_MAX_TILES;
    W.bagg = base + 3 * NOALLOC_MAX_TILES;
    W.carF = W.fagg;  // each carry thread reads its tiles' totals before it writes their carries
    W.carB = W.bagg;
    W.bfe = base + 4 * NOALLOC_MAX_TILES;
    W.bfv = W.bfe + NOALLOC_MAX_CBLK;
    W.bbf = W.bfv + NOALLOC_MAX_CBLK;
    W.bbv = W.bbf + NOALLOC_MAX_CBLK;
    W.redo_count = reinterpret_cast<uint32_t*>(W.bbv + NOALLOC_MAX_CBLK);
    W.st = nullptr;
    W.redo = nullptr;
    SymArgs<float> A;
    A.s = sorted;
    A.n = n;
    A.x = x;
    A.pin = perm;
    A.ldx = 1;
    A.y = y;
    A.pout = perm;
    A.ldy = 1;
    A.phi = nullptr;
    A.D = nullptr;
    A.paux = perm;
    A.col0 = 0;
    A.ncol = 1;
    A.status = nullptr;
    e = sym_launch<float, 1, false, 16>(A, ntiles, W, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        set_last_error("laplex_matvec_sym_noalloc: %s", cudaGetErrorString(e));
        return LAPLEX_ECUDA;
    }
    set_last_error("");
    return LAPLEX_OK;
}
