// sort.cu -- stable LSD radix sort of the anchors with an index payload (the
// recurrences run over the anchors in sorted order: "LAPLEX - La FFT dei
// Nuclei di Laplace Apprendibili", technical summary §2.2; the sort is the
// O(n log n) term).
//
// Key map (monotone, bijective on finite values after -0.0 -> +0.0):
//     u = bits(a);  u = (u == -0.0) ? +0.0 : u;
//     key = sign(u) ? ~u : u | signbit
// so unsigned key order is numeric order.  Each pass sorts by one 8-bit digit
// and is stable, so equal anchors keep ascending index order and the output
// permutation is unique.  A NaN or Inf anchor sets ST_NONFINITE.
//
// Onesweep (Adinets & Merrill, "Onesweep: A Faster Least Significant Digit
// Radix Sort for GPUs", 2022):
//   k_radix_hist    : one read of the keys counts every digit of every pass
//   k_radix_offsets : exclusive scan of each pass's 256 counts
//   k_onesweep      : one kernel per pass.  Tiles are taken in ticket order;
//                     each ranks its keys stably (warp match + per-warp
//                     counters), publishes its 256 digit counts, and finds how
//                     many keys of each digit lie in earlier tiles by a
//                     decoupled look-back over 64-bit records (pass tag in the
//                     high word, so one memset per call serves every pass).
//                     Keys are staged in shared memory in digit order, so the
//                     writes to each digit's run coalesce.
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

// A look-back record is one 64-bit word (tag in the high half, count in the
// low half) written and read whole, and nothing else is read on the strength
// of it, so relaxed accesses suffice and a window of loads can be in flight.
__device__ __forceinline__ void st_relaxed64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Counts of every digit of every pass in one read of the keys.
template <typename T>
__global__ void __launch_bounds__(SORT_NT) k_radix_hist(const T* __restrict__ a, int64_t n,
                                                        uint32_t* __restrict__ hist,
                                                        uint32_t* status) {
    using K = typename KeyOf<T>::K;
    constexpr int P = sizeof(K);
    __shared__ uint32_t h[P][RADIX];
    for (int j = threadIdx.x; j < P * RADIX; j += SORT_NT) (&h[0][0])[j] = 0u;
    __syncthreads();
    bool bad = false;
    const int64_t stride = (int64_t)gridDim.x * SORT_NT;
    for (int64_t i = (int64_t)blockIdx.x * SORT_NT + threadIdx.x; i < n; i += stride) {
        const K k = to_key(a[i], bad);
#pragma unroll
        for (int p = 0; p < P; ++p) atomicAdd(&h[p][(unsigned)(k >> (8 * p)) & (RADIX - 1)], 1u);
    }
    if (bad) set_status(status, ST_NONFINITE);
    __syncthreads();
    for (int j = threadIdx.x; j < P * RADIX; j += SORT_NT) {
        const uint32_t c = (&h[0][0])[j];
        if (c) atomicAdd(&hist[j], c);
    }
}

// hist[p][d] <- number of keys with a smaller digit d in pass p (one block per pass)
__global__ void __launch_bounds__(SORT_NT) k_radix_offsets(uint32_t* __restrict__ hist) {
    __shared__ uint32_t sm[SORT_NT / 32 + 1];
    uint32_t* h = hist + (int64_t)blockIdx.x * RADIX;
    uint32_t tot;
    const uint32_t ex = block_excl_sum<SORT_NT>(h[threadIdx.x], sm, tot);
    h[threadIdx.x] = ex;
}

constexpr uint32_t SORT_POLLS = 1u << 25;

template <typename T, int KPT>
__global__ void __launch_bounds__(SORT_NT, 3) k_onesweep(
    const T* __restrict__ a, const typename KeyOf<T>::K* __restrict__ ksrc,
    const int32_t* __restrict__ vsrc, int64_t n, int pass, const uint32_t* __restrict__ offsets,
    uint64_t* __restrict__ rec, uint32_t* __restrict__ ticket, typename KeyOf<T>::K* __restrict__ kdst,
    int32_t* __restrict__ vdst, int last, uint32_t* status) {
    using K = typename KeyOf<T>::K;
    constexpr int NT = SORT_NT, NW = NT / 32, TILE = NT * KPT;
    static_assert(KPT % 4 == 0, "digits are packed four to a word");
    __shared__ K skey[TILE];
    __shared__ int32_t sval[TILE];
    __shared__ uint32_t wcnt[NW][RADIX];
    __shared__ uint32_t dstart[RADIX];
    __shared__ int64_t gofs[RADIX];  // global position of staged key q: gofs[digit] + q
    __shared__ uint32_t scan_sm[NT / 32 + 1];
    __shared__ int64_t sh_tile;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int shift = 8 * pass;
    const bool first = pass == 0;
    if (threadIdx.x == 0) sh_tile = (int64_t)atomicAdd(ticket, 1u);
    for (int j = threadIdx.x; j < NW * RADIX; j += NT) (&wcnt[0][0])[j] = 0u;
    __syncthreads();
    const int64_t t = sh_tile;
    const int64_t tb = t * TILE;
    const int64_t end = min(tb + TILE, n);
    const unsigned ltmask = lanemask_lt();
    // key i of this thread is element lane0 + 32 i of the tile (coalesced per i)
    const int64_t lane0 = tb + (int64_t)w * 32 * KPT + lane;
    const int nvalid = (int)max((int64_t)0, min((int64_t)KPT, (end - lane0 + 31) / 32));
    K k[KPT];
    uint32_t dg[KPT / 4];  // the digits, four per word
    uint32_t rk[KPT];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int64_t idx = lane0 + i * 32;
        k[i] = i < nvalid ? (first ? to_key(a[idx], bad) : ksrc[idx]) : K(0);
    }
#pragma unroll
    for (int i = 0; i < KPT; i += 4) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) word |= ((uint32_t)(k[i + b] >> shift) & (RADIX - 1)) << (8 * b);
        dg[i / 4] = word;
    }
    auto digit = [&](int i) -> int { return (int)((dg[i / 4] >> (8 * (i % 4))) & (RADIX - 1)); };
    // stable rank among the keys of this warp with the same digit: lanes in
    // order within a round, rounds in order.  The lowest lane of each group of
    // equal digits adds the group to the warp's counter and hands the old
    // count to the group with one shuffle.
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const bool valid = i < nvalid;
        const int d = valid ? digit(i) : RADIX;  // padding ranks apart
        const unsigned peers = __match_any_sync(FULL, d);
        const int leader = __ffs(peers) - 1;
        uint32_t base = 0;
        if (valid && lane == leader) base = atomicAdd(&wcnt[w][d], (uint32_t)__popc(peers));
        base = __shfl_sync(FULL, base, leader);
        rk[i] = base + __popc(peers & ltmask);
    }
    __syncthreads();
    const int d = threadIdx.x;  // NT == RADIX: one digit per thread from here on
    uint32_t c = 0;  // this tile's count of digit d; wcnt[.][d] becomes the warps' exclusive offsets
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) {
        const uint32_t x = wcnt[ww][d];
        wcnt[ww][d] = c;
        c += x;
    }
    // publish this tile's count of digit d early; its prefix over earlier tiles
    // is looked up after the tile is staged, when they have had time to finish
    const uint64_t tagA = (uint64_t)(2 * pass + 2) << 32, tagI = (uint64_t)(2 * pass + 3) << 32;
    uint64_t* my = rec + t * RADIX + d;
    st_relaxed64(my, (t == 0 ? tagI : tagA) | c);
    uint32_t tot;
    dstart[d] = block_excl_sum<NT>(c, scan_sm, tot);  // its barriers publish wcnt
    __syncthreads();                                   // and this one dstart
    // stage the keys in digit order (rk becomes the staging position), then
    // the payloads, loaded only now to keep the ranking's registers free
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
        if (i < nvalid) {
            const int di = digit(i);
            rk[i] += dstart[di] + wcnt[w][di];
            skey[rk[i]] = k[i];
        }
    }
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int64_t idx = lane0 + i * 32;
        if (i < nvalid) sval[rk[i]] = first ? (int32_t)idx : vsrc[idx];
    }
    // keys of digit d in all earlier tiles: walk back LB records at a time
    // (loads in flight together), adding counts up to and including the first
    // inclusive record
    uint64_t excl = 0;
    if (t > 0) {
        constexpr int LB = 8;
        bool done = false;
        for (int64_t j0 = t - 1; !done; j0 -= LB) {
            uint64_t val[LB];
#pragma unroll
            for (int q = 0; q < LB; ++q)
                val[q] = j0 - q >= 0 ? ld_relaxed64(rec + (j0 - q) * RADIX + d) : tagI;
#pragma unroll
            for (int q = 0; q < LB; ++q) {
                if (done) break;
                uint32_t it = 0;
                while ((val[q] & 0xFFFFFFFF00000000ull) < tagA) {
                    if (++it > SORT_POLLS) break;
                    __nanosleep(64);
                    val[q] = ld_relaxed64(rec + (j0 - q) * RADIX + d);
                }
                if ((val[q] & 0xFFFFFFFF00000000ull) < tagA) {
                    set_status(status, ST_TIMEOUT);
                    done = true;
                    break;
                }
                excl += val[q] & 0xFFFFFFFFull;
                if ((val[q] & 0xFFFFFFFF00000000ull) == tagI) done = true;
            }
        }
        st_relaxed64(my, tagI | (excl + c));
    }
    (void)bad;  // non-finite anchors are reported by k_radix_hist
    gofs[d] = (int64_t)offsets[d] + (int64_t)excl - (int64_t)dstart[d];
    __syncthreads();
    const int cnt = (int)(end - tb);
    for (int q = threadIdx.x; q < cnt; q += NT) {
        const K kk = skey[q];
        const int64_t gpos = gofs[(unsigned)(kk >> shift) & (RADIX - 1)] + q;
        kdst[gpos] = last ? key_to_bits(kk) : kk;
        vdst[gpos] = sval[q];
    }
}

// ------------------------------------------------------------------ host side
template <typename T> constexpr int sort_kpt() { return sizeof(T) == 8 ? 8 : 16; }

size_t sort_ws_bytes(int64_t n, int f64) {
    const int kpt = f64 ? 8 : 16;
    const int64_t tile = (int64_t)SORT_NT * kpt;
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    const size_t ks = f64 ? 8 : 4;
    const int P = f64 ? 8 : 4;
    return Carve::need((size_t)n, ks) + Carve::need((size_t)n, 4) +
           Carve::need((size_t)(16 + P * RADIX), 4) + Carve::need((size_t)(ntiles * RADIX), 8);
}

template <typename T>
cudaError_t sort_run(const T* a, int64_t n, T* sorted, int32_t* perm, void* ws, size_t ws_bytes,
                     uint32_t* status, cudaStream_t st) {
    using K = typename KeyOf<T>::K;
    if (n == 0) return cudaSuccess;
    constexpr int KPT = sort_kpt<T>();
    constexpr int P = sizeof(K);
    const int64_t tile = (int64_t)SORT_NT * KPT;
    const int64_t ntiles = (n + tile - 1) / tile;
    Carve cv(ws, ws_bytes);
    K* kws = cv.take<K>(n);
    int32_t* vws = cv.take<int32_t>(n);
    uint32_t* ctl = cv.take<uint32_t>(16 + P * RADIX);  // [0..P) tickets, [16..) histograms
    uint64_t* rec = cv.take<uint64_t>(ntiles * RADIX);
    if (!cv.ok) return cudaErrorInvalidValue;
    uint32_t* tickets = ctl;
    uint32_t* hist = ctl + 16;
    cudaError_t e = cudaMemsetAsync(ctl, 0, sizeof(uint32_t) * (16 + P * RADIX), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(rec, 0, sizeof(uint64_t) * ntiles * RADIX, st);
    if (e != cudaSuccess) return e;
    {
        const int64_t blocks = std::min<int64_t>((n + SORT_NT - 1) / SORT_NT, 148 * 8);
        k_radix_hist<T><<<(unsigned)blocks, SORT_NT, 0, st>>>(a, n, hist, status);
        k_radix_offsets<<<P, SORT_NT, 0, st>>>(hist);
    }
    K* kout = reinterpret_cast<K*>(sorted);
    const K* ksrc = nullptr;
    const int32_t* vsrc = nullptr;
    profile_before(st);
    for (int pass = 0; pass < P; ++pass) {
        const bool to_out = ((P - 1 - pass) % 2) == 0;
        K* kdst = to_out ? kout : kws;
        int32_t* vdst = to_out ? perm : vws;
        k_onesweep<T, KPT><<<(unsigned)ntiles, SORT_NT, 0, st>>>(
            a, ksrc, vsrc, n, pass, hist + pass * RADIX, rec, tickets + pass, kdst, vdst,
            pass == P - 1, status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ksrc = kdst;
        vsrc = vdst;
    }
    profile_after(st);
    return cudaSuccess;
}

template cudaError_t sort_run<float>(const float*, int64_t, float*, int32_t*, void*, size_t,
                                     uint32_t*, cudaStream_t);
template cudaError_t sort_run<double>(const double*, int64_t, double*, int32_t*, void*, size_t,
                                      uint32_t*, cudaStream_t);

}  // namespace lx
