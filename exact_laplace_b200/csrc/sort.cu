// sort.cu -- stable LSD radix sort of the anchors with an index payload
// ("after sorting the anchors": "LAPLEX - La FFT dei Nuclei di Laplace
// Apprendibili", technical summary §2.2; the sort is the O(n log n) term).
//
// Key map (monotone, bijective on finite values after -0.0 -> +0.0):
//     u = bits(a);  u = (u == -0.0) ? +0.0 : u;
//     key = sign(u) ? ~u : u | signbit
// so unsigned key order is numeric order.  Each pass sorts by one 8-bit digit
// and is stable, so equal anchors keep ascending index order and the output
// permutation is unique.  A NaN or Inf anchor sets ST_NONFINITE.
//
// One pass = three kernels:
//   k_radix_upsweep   : digit counts of each contiguous segment of keys
//   k_radix_scan      : exclusive scan of the counts, digit-major -> start of
//                       every (digit, segment) run in the output
//   k_radix_downsweep : each block walks its segment tile by tile in order,
//                       ranks keys stably inside the tile (warp match + per-warp
//                       counters), stages them in shared memory in digit order
//                       and writes them to their runs (runs are contiguous, so
//                       the writes coalesce).
// Pass 0 reads the anchors and generates the index payload; the last pass
// writes the anchors back as values and the payload as perm.
#include <algorithm>

#include "common.cuh"
#include "laplex_impl.h"

namespace lx {

constexpr int RADIX = 256;
constexpr int SORT_NT = 256;

template <typename T> struct KeyOf;
template <> struct KeyOf<float> { using K = uint32_t; };
template <> struct KeyOf<double> { using K = uint64_t; };

__device__ __forceinline__ uint32_t to_key(float f, bool& bad) {
    uint32_t u = __float_as_uint(f);
    bad |= (u & 0x7F800000u) == 0x7F800000u;
    if (u == 0x80000000u) u = 0u;
    return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t to_key(double f, bool& bad) {
    uint64_t u = (uint64_t)__double_as_longlong(f);
    bad |= (u & 0x7FF0000000000000ull) == 0x7FF0000000000000ull;
    if (u == 0x8000000000000000ull) u = 0ull;
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ uint32_t key_to_bits(uint32_t k) {
    return (k >> 31) ? (k ^ 0x80000000u) : ~k;
}
__device__ __forceinline__ uint64_t key_to_bits(uint64_t k) {
    return (k >> 63) ? (k ^ 0x8000000000000000ull) : ~k;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// exclusive scan of one uint32 per thread over a block of NT threads
template <int NT>
__device__ __forceinline__ uint32_t block_excl_sum(uint32_t v, uint32_t* sm /*NT/32 + 1*/,
                                                   uint32_t& total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t o = __shfl_up_sync(FULL, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) sm[w] = inc;
    __syncthreads();
    if (w == 0) {
        uint32_t t = lane < NT / 32 ? sm[lane] : 0u;
        uint32_t ti = t;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            uint32_t o = __shfl_up_sync(FULL, ti, off);
            if (lane >= off) ti += o;
        }
        if (lane < NT / 32) sm[lane] = ti - t;
        if (lane == 31) sm[NT / 32] = ti;
    }
    __syncthreads();
    const uint32_t r = sm[w] + inc - v;
    total = sm[NT / 32];
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(SORT_NT) k_radix_upsweep(const T* __restrict__ a,
                                                           const typename KeyOf<T>::K* __restrict__ ksrc,
                                                           int64_t n, int shift, int64_t seg, int G,
                                                           uint32_t* __restrict__ counts,
                                                           uint32_t* status, int first) {
    using K = typename KeyOf<T>::K;
    __shared__ uint32_t hist[RADIX];
    hist[threadIdx.x] = 0;
    __syncthreads();
    const int64_t beg = (int64_t)blockIdx.x * seg;
    const int64_t end = min(beg + seg, n);
    bool bad = false;
    for (int64_t i = beg + threadIdx.x; i < end; i += SORT_NT) {
        const K k = first ? to_key(a[i], bad) : ksrc[i];
        atomicAdd(&hist[(unsigned)(k >> shift) & (RADIX - 1)], 1u);
    }
    if (bad) set_status(status, ST_NONFINITE);
    __syncthreads();
    counts[(int64_t)threadIdx.x * G + blockIdx.x] = hist[threadIdx.x];
}

// in-place exclusive scan of counts[0 .. total) (one block of 1024 threads)
__global__ void __launch_bounds__(1024) k_radix_scan(uint32_t* __restrict__ counts, int64_t total) {
    __shared__ uint32_t sm[1024 / 32 + 1];
    const int64_t per = (total + 1023) / 1024;
    const int64_t b = min((int64_t)threadIdx.x * per, total);
    const int64_t e = min(b + per, total);
    uint32_t s = 0;
    for (int64_t i = b; i < e; ++i) s += counts[i];
    uint32_t tot;
    uint32_t run = block_excl_sum<1024>(s, sm, tot);
    for (int64_t i = b; i < e; ++i) {
        const uint32_t c = counts[i];
        counts[i] = run;
        run += c;
    }
}

template <typename T, int KPT>
__global__ void __launch_bounds__(SORT_NT) k_radix_downsweep(
    const T* __restrict__ a, const typename KeyOf<T>::K* __restrict__ ksrc,
    const int32_t* __restrict__ vsrc, int64_t n, int shift, int64_t seg, int G,
    const uint32_t* __restrict__ offsets, typename KeyOf<T>::K* __restrict__ kdst,
    int32_t* __restrict__ vdst, int first, int last) {
    using K = typename KeyOf<T>::K;
    constexpr int NT = SORT_NT, NW = NT / 32, TILE = NT * KPT;
    __shared__ K skey[TILE];
    __shared__ int32_t sval[TILE];
    __shared__ uint32_t wcnt[NW][RADIX];
    __shared__ uint32_t dstart[RADIX], dcount[RADIX], run[RADIX];
    __shared__ uint32_t scan_sm[NT / 32 + 1];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t beg = (int64_t)blockIdx.x * seg;
    const int64_t end = min(beg + seg, n);
    run[threadIdx.x] = offsets[(int64_t)threadIdx.x * G + blockIdx.x];
    const unsigned ltmask = lanemask_lt();
    for (int64_t tb = beg; tb < end; tb += TILE) {
        for (int j = threadIdx.x; j < NW * RADIX; j += NT) (&wcnt[0][0])[j] = 0u;
        __syncthreads();
        K k[KPT];
        int32_t v[KPT];
        int dg[KPT];
        uint32_t rk[KPT];
        bool bad = false;
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const int64_t idx = tb + (int64_t)w * 32 * KPT + i * 32 + lane;
            if (idx < end) {
                k[i] = first ? to_key(a[idx], bad) : ksrc[idx];
                v[i] = first ? (int32_t)idx : vsrc[idx];
                dg[i] = (int)((unsigned)(k[i] >> shift) & (RADIX - 1));
            } else {
                k[i] = 0;
                v[i] = 0;
                dg[i] = RADIX;  // padding: never placed
            }
        }
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const int d = dg[i];
            const unsigned peers = __match_any_sync(FULL, d);
            const uint32_t lower = __popc(peers & ltmask);
            rk[i] = d < RADIX ? wcnt[w][d] + lower : 0u;
            __syncwarp();
            if (d < RADIX && lower == 0) wcnt[w][d] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        {
            const int d = threadIdx.x;  // NT == RADIX
            uint32_t c = 0;
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) {
                const uint32_t t = wcnt[ww][d];
                wcnt[ww][d] = c;
                c += t;
            }
            dcount[d] = c;
            uint32_t tot;
            dstart[d] = block_excl_sum<NT>(c, scan_sm, tot);
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const int d = dg[i];
            if (d < RADIX) {
                const uint32_t pos = dstart[d] + wcnt[w][d] + rk[i];
                skey[pos] = k[i];
                sval[pos] = v[i];
            }
        }
        __syncthreads();
        const int cnt = (int)(end - tb < (int64_t)TILE ? end - tb : (int64_t)TILE);
        for (int q = threadIdx.x; q < cnt; q += NT) {
            const K kk = skey[q];
            const int d = (int)((unsigned)(kk >> shift) & (RADIX - 1));
            const int64_t gpos = (int64_t)run[d] + (q - (int)dstart[d]);
            kdst[gpos] = last ? key_to_bits(kk) : kk;
            vdst[gpos] = sval[q];
        }
        __syncthreads();
        run[threadIdx.x] += dcount[threadIdx.x];
        __syncthreads();
    }
}

// ------------------------------------------------------------------ host side
struct SortPlan {
    int kpt;
    int64_t tile, seg;
    int G;
};

static SortPlan sort_plan(int64_t n, int f64) {
    SortPlan p;
    p.kpt = f64 ? 8 : 16;
    p.tile = (int64_t)SORT_NT * p.kpt;
    const int64_t tiles = std::max<int64_t>(1, (n + p.tile - 1) / p.tile);
    const int64_t G0 = std::min<int64_t>(tiles, 148 * 4);
    const int64_t per_tiles = (tiles + G0 - 1) / G0;
    p.seg = per_tiles * p.tile;
    p.G = (int)std::max<int64_t>(1, (n + p.seg - 1) / p.seg);
    return p;
}

size_t sort_ws_bytes(int64_t n, int f64) {
    const SortPlan p = sort_plan(n, f64);
    const size_t ks = f64 ? 8 : 4;
    return Carve::need((size_t)n, ks) + Carve::need((size_t)n, 4) +
           Carve::need((size_t)RADIX * p.G, 4);
}

template <typename T>
cudaError_t sort_run(const T* a, int64_t n, T* sorted, int32_t* perm, void* ws, size_t ws_bytes,
                     uint32_t* status, cudaStream_t st) {
    using K = typename KeyOf<T>::K;
    if (n == 0) return cudaSuccess;
    const int f64 = sizeof(T) == 8;
    const SortPlan p = sort_plan(n, f64);
    Carve cv(ws, ws_bytes);
    K* kws = cv.take<K>(n);
    int32_t* vws = cv.take<int32_t>(n);
    uint32_t* counts = cv.take<uint32_t>((size_t)RADIX * p.G);
    if (!cv.ok) return cudaErrorInvalidValue;
    K* kout = reinterpret_cast<K*>(sorted);
    const int passes = (int)(sizeof(K) * 8 / 8);
    const K* ksrc = nullptr;
    const int32_t* vsrc = nullptr;
    for (int pass = 0; pass < passes; ++pass) {
        const bool to_out = ((passes - 1 - pass) % 2) == 0;
        K* kdst = to_out ? kout : kws;
        int32_t* vdst = to_out ? perm : vws;
        const int shift = 8 * pass;
        const int first = pass == 0, last = pass == passes - 1;
        k_radix_upsweep<T><<<p.G, SORT_NT, 0, st>>>(a, ksrc, n, shift, p.seg, p.G, counts, status,
                                                     first);
        k_radix_scan<<<1, 1024, 0, st>>>(counts, (int64_t)RADIX * p.G);
        constexpr int KPT = sizeof(T) == 8 ? 8 : 16;
        k_radix_downsweep<T, KPT><<<p.G, SORT_NT, 0, st>>>(a, ksrc, vsrc, n, shift, p.seg, p.G,
                                                           counts, kdst, vdst, first, last);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ksrc = kdst;
        vsrc = vdst;
    }
    return cudaSuccess;
}

template cudaError_t sort_run<float>(const float*, int64_t, float*, int32_t*, void*, size_t,
                                     uint32_t*, cudaStream_t);
template cudaError_t sort_run<double>(const double*, int64_t, double*, int32_t*, void*, size_t,
                                      uint32_t*, cudaStream_t);

}  // namespace lx
