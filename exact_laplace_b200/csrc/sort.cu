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
// Every pass is a reduce-then-scan over tiles of 6144 keys (fp32; 2048 fp64),
// three launches without any wait between blocks:
//   k_count      : per tile, the count of each digit; each block walks a
//                  contiguous range of tiles and keeps running sums, so it
//                  writes per tile the counts of the earlier tiles of its
//                  range, and at the end its range's totals
//   k_count_scan : one block: per digit, the exclusive sums over the ranges,
//                  plus the digit's start (the exclusive sum over smaller digits)
//   k_scatter    : persistent blocks, each over a contiguous range of tiles; the tiles'
//                  keys (and payloads) arrive in a ring of shared-memory stages
//                  by 1-D bulk copies (TMA), the next ones in flight while one
//                  is ranked: a stable rank per warp (equal digits found by
//                  warp match or ballots, one shared atomic per group), staging
//                  in digit order, then coalesced runs written per digit at the
//                  offsets k_count_scan gave.
// The count pass reads the keys once more (4 bytes per key) but leaves the
// scatter free of the serial look-back of a single-pass sort, whose chain of
// dependent L2 round trips bounded the tile rate on this GPU.
// Pass 0 reads the anchors and generates the index payload; the last pass
// writes the anchors back as values and the payload as perm.
#include <algorithm>
#include <type_traits>

#include "bulk.cuh"
#include "common.cuh"
#include "devcache.h"
#include "laplex_impl.h"

// ranking of equal digits in a warp: 0 = warp match, 1 = eight ballots,
// 3 = shared-memory match masks; 2 = chosen per pass from the digit histogram
// between the warp match and LX_SORT_HI (1 or 3)
#ifndef LX_SORT_RANK
#define LX_SORT_RANK 2
#endif
#ifndef LX_SORT_HI
#define LX_SORT_HI 3
#endif
// keys per thread (fp32 keys), input stages and resident blocks per SM of
// k_scatter (24 keys per thread, 2 blocks: measured fastest at n = 2^24 to 2^30)
#ifndef LX_SORT_KPT
#define LX_SORT_KPT 24
#endif
#ifndef LX_SORT_S
#define LX_SORT_S 1
#endif
#ifndef LX_SORT_MINB
#define LX_SORT_MINB 2
#endif
// k_scatter: contiguous tiles per block (1) or round robin (0)
#ifndef LX_SORT_BLOCKED
#define LX_SORT_BLOCKED 1
#endif
// k_count: one atomic for all lanes sharing lane 0's digit (1) or one per key (0: measured
// faster on B200, the high exponent digits included)
#ifndef LX_COUNT_AGG
#define LX_COUNT_AGG 0
#endif

namespace lx {

constexpr int RADIX = 256;
constexpr int SORT_NT = 256;  // threads per block: one digit per thread in the per-digit steps
constexpr int SORT_NW = SORT_NT / 32;

// bounded wait for phase `parity` of *bar with a caller-chosen bound
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t polls) {
    for (uint32_t it = 0; it < polls; ++it)
        if (mbar_test(bar, parity)) return true;
    return false;
}

template <typename T> struct KeyOf;
template <> struct KeyOf<float> { using K = uint32_t; };
template <> struct KeyOf<double> { using K = uint64_t; };

// keys per thread and input stages (ring of bulk-copy destinations) per block
template <typename T> struct SortShape;
template <> struct SortShape<float> { static constexpr int KPT = LX_SORT_KPT, S = LX_SORT_S; };
template <> struct SortShape<double> { static constexpr int KPT = 8, S = 1; };

__device__ __forceinline__ uint32_t key_of_bits(uint32_t u) {
    if (u == 0x80000000u) u = 0u;
    return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t key_of_bits(uint64_t u) {
    if (u == 0x8000000000000000ull) u = 0ull;
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ bool non_finite_bits(uint32_t u) { return (u & 0x7F800000u) == 0x7F800000u; }
__device__ __forceinline__ bool non_finite_bits(uint64_t u) {
    return (u & 0x7FF0000000000000ull) == 0x7FF0000000000000ull;
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

// Lanes of the warp holding the same digit (0..255; 256 marks padding, which
// groups only with padding).  Three ways:
//  - RANK_MATCH: the warp match instruction, whose cost grows with the number
//    of distinct digits among the 32 lanes (cheap for the few values of an
//    exponent byte, slow on uniformly spread digits);
//  - RANK_BALLOT: one ballot per digit bit, a fixed cost;
//  - RANK_MASK: match masks in shared memory (wmask: this warp's RADIX + 1
//    words, zero on entry): every lane ors its bit into its digit's word and
//    reads the word back; the group's highest lane clears the word at the next
//    call (clr: the previous call's word, RADIX + 1 for none).
// The shared-memory and rank steps are single PTX blocks, so that no branch
// (and no reconvergence point) surrounds the warp-wide steps.
enum : int { RANK_MATCH = 0, RANK_BALLOT = 1, RANK_MASK = 3 };

template <bool RAGGED>
__device__ __forceinline__ unsigned ballot_peers(uint32_t dig) {
    unsigned m = FULL;
#pragma unroll
    for (int b = 0; b < (RAGGED ? 9 : 8); ++b) {
        const bool on = (dig >> b) & 1u;
        const unsigned bb = __ballot_sync(FULL, on);
        m &= on ? bb : ~bb;
    }
    return m;
}

__device__ __forceinline__ unsigned mask_peers(uint32_t dig, uint32_t* wmask, uint32_t& clr, uint32_t lanebit,
                                               uint32_t gtmask) {
    unsigned peers;
    asm volatile(
        "{\n"
        " .reg .b32 a;\n"
        " .reg .pred pc;\n"
        " setp.le.u32 pc, %2, 256;\n"
        " mad.lo.u32 a, %2, 4, %3;\n"
        " @pc st.shared.u32 [a], 0;\n"
        " bar.warp.sync 0xffffffff;\n"
        " mad.lo.u32 a, %1, 4, %3;\n"
        " red.shared.or.b32 [a], %4;\n"
        " bar.warp.sync 0xffffffff;\n"
        " ld.shared.u32 %0, [a];\n"
        "}\n"
        : "=r"(peers)
        : "r"(dig), "r"(clr), "r"(smem_u32(wmask)), "r"(lanebit)
        : "memory");
    clr = (peers & gtmask) == 0u ? dig : (uint32_t)(RADIX + 1);
    return peers;
}

// Stable rank of this lane's key among the warp's keys of its digit in this
// and the earlier rounds: the group's highest lane adds the group's size to
// the warp's counter of the digit and hands the old count to the group.
__device__ __forceinline__ uint32_t group_rank(unsigned peers, uint32_t dig, bool valid, uint32_t* wcnt_w,
                                               unsigned ltmask) {
    uint32_t r;
    asm volatile(
        "{\n"
        " .reg .b32 pc, ltb, lt, old, hi, a, b;\n"
        " .reg .pred ld;\n"
        " popc.b32 pc, %1;\n"
        " and.b32 ltb, %1, %4;\n"
        " popc.b32 lt, ltb;\n"
        " add.u32 a, lt, 1;\n"
        " setp.eq.u32 ld, a, pc;\n"
        " setp.ne.and.u32 ld, %3, 0, ld;\n"
        " and.b32 a, %2, 255;\n"
        " mad.lo.u32 a, a, 4, %5;\n"
        " mov.b32 old, 0;\n"
        " @ld atom.shared.add.u32 old, [a], pc;\n"
        " bfind.u32 hi, %1;\n"
        " shfl.sync.idx.b32 b, old, hi, 0x1f, 0xffffffff;\n"
        " add.u32 %0, b, lt;\n"
        "}\n"
        : "=r"(r)
        : "r"(peers), "r"(dig), "r"((uint32_t)valid), "r"(ltmask), "r"(smem_u32(wcnt_w))
        : "memory");
    return r;
}

// The expected number of distinct digits among 32 keys drawn from a pass's
// digit histogram below which the warp match ranks faster than the ballots
// (measured on B200: about 3 distinct values, match 1.6x faster; about 30,
// ballots 1.4x faster).
constexpr float MATCH_BELOW_DISTINCT = 12.0f;

// A predicated shared-memory add without a result, as one instruction.
__device__ __forceinline__ void red_add_shared_if(bool pred, uint32_t* p, uint32_t v) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %2, 0;\n @q red.shared.add.u32 [%0], %1;\n}\n" ::"r"(
                     smem_u32(p)),
                 "r"(v), "r"((uint32_t)pred)
                 : "memory");
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
    return r;  // sm is written again only after the caller's next barriers
}

// ------------------------------------------------------------------ count
// grid bound of k_count (sizes its per-block totals in the workspace)
constexpr int COUNT_MAX_BLOCKS = 4096;
constexpr int COUNT_BLOCKS_PER_SM = 4;

template <typename K>
struct CountArgs {
    const K* keys;                     // this pass's keys (sort pass 0: the anchor bits)
    int64_t n, ntiles, R;              // R: tiles per block
    int shift;
    uint32_t* tile_pre;                // [ntiles][RADIX] counts of the earlier tiles of the range
    uint32_t* blk_tot;                 // [G][RADIX] totals of each range
    uint32_t* status;
};

// one key of this warp into the tile histogram; lane 0's digit is counted by
// one atomic for all lanes that share it (the high digits of real anchors
// take few values, and same-address shared atomics serialise)
// key maps of a digit pass's input keys
enum : int {
    KM_NONE = 0,
    KM_ANCHOR = 1,  // anchor bits -> sort key (and a finiteness check)
    KM_CLAMP = 2,   // index: one outside [0, n) becomes (n - 1) | 2^31 (sorts with the last
                    // group while its digits below bit 31 are read, and is dropped at the end)
};

template <int KM, typename K>
__device__ __forceinline__ K map_key(K kb, int64_t n) {
    if constexpr (KM == KM_ANCHOR) return key_of_bits(kb);
    else if constexpr (KM == KM_CLAMP) return (int64_t)kb < n ? kb : (K)((uint64_t)(n - 1) | 0x80000000ull);
    else return kb;
}

// One key per lane into the tile histogram hb (dig = RADIX: no key).  The
// lanes holding lane 0's digit are counted by one add of lane 0 (the high
// digits of real anchors take few values, and same-address shared atomics
// serialise), the others add 1 each.  Written as one PTX block so that no
// branch, and no reconvergence point, surrounds the warp-wide steps.
__device__ __forceinline__ void count_digit(uint32_t dig, uint32_t* hb, uint32_t lane0) {
    asm volatile(
        "{\n"
        " .reg .b32 d0, same, cnt, a0, a1;\n"
        " .reg .pred p, np, q, r;\n"
        " shfl.sync.idx.b32 d0, %0, 0, 0x1f, 0xffffffff;\n"
        " setp.eq.u32 p, %0, d0;\n"
        " vote.sync.ballot.b32 same, p, 0xffffffff;\n"
        " popc.b32 cnt, same;\n"
        " setp.lt.u32 q, d0, 256;\n"
        " setp.ne.and.u32 q, %2, 0, q;\n"
        " mad.lo.u32 a0, d0, 4, %1;\n"
        " @q red.shared.add.u32 [a0], cnt;\n"
        " not.pred np, p;\n"
        " setp.lt.and.u32 r, %0, 256, np;\n"
        " mad.lo.u32 a1, %0, 4, %1;\n"
        " @r red.shared.add.u32 [a1], 1;\n"
        "}\n" ::"r"(dig),
        "r"(smem_u32(hb)), "r"(lane0)
        : "memory");
}

template <int KM, typename K>
__device__ __forceinline__ void count_key(K kb, bool valid, int shift, uint32_t* hb, bool& bad, int64_t n,
                                          uint32_t lane0) {
    if constexpr (KM == KM_ANCHOR) bad |= valid & non_finite_bits(kb);
    const K k = map_key<KM>(kb, n);
    const uint32_t dig = valid ? ((uint32_t)(k >> shift) & (RADIX - 1)) : (uint32_t)RADIX;
#if LX_COUNT_AGG
    count_digit(dig, hb, lane0);
#else
    red_add_shared_if(valid, &hb[dig & (RADIX - 1)], 1u);
#endif
}

// KM: the map of the input keys (KM_ANCHOR: anchor bits, also checked finite).
template <typename K, int KPT, int KM>
__global__ void __launch_bounds__(SORT_NT) k_count(CountArgs<K> A) {
    constexpr int NT = SORT_NT, TILE = NT * KPT;
    constexpr int KPV = 16 / sizeof(K);          // keys per 16-byte vector
    constexpr int VPT = TILE / KPV / NT;         // vectors per thread per tile
    static_assert(VPT * KPV * NT == TILE, "a tile is whole vectors per thread");
    __shared__ uint32_t h[2][RADIX];  // two tiles' histograms: one barrier per tile
    const int d = threadIdx.x;
    const uint32_t lane0 = (threadIdx.x & 31) == 0 ? 1u : 0u;
    h[0][d] = 0u;
    h[1][d] = 0u;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * A.R, t1 = std::min(t0 + A.R, A.ntiles);
    const uint4* src = reinterpret_cast<const uint4*>(A.keys);
    auto full_tile = [&](int64_t t) { return (t + 1) * TILE <= A.n; };
    auto load = [&](int64_t t, uint4* v) {
#pragma unroll
        for (int j = 0; j < VPT; ++j) v[j] = __ldcs(src + t * (TILE / KPV) + j * NT + threadIdx.x);
    };
    bool bad = false;
    uint32_t run = 0;
    uint4 v[VPT];
    if (t0 < t1 && full_tile(t0)) load(t0, v);
    for (int64_t t = t0; t < t1; ++t) {
        uint4 nx[VPT];
        const bool nfull = t + 1 < t1 && full_tile(t + 1);
        if (nfull) load(t + 1, nx);
        uint32_t* hb = h[t & 1];
        if (full_tile(t)) {
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const K* kv = reinterpret_cast<const K*>(&v[j]);
#pragma unroll
                for (int e = 0; e < KPV; ++e) count_key<KM>(kv[e], true, A.shift, hb, bad, A.n, lane0);
            }
        } else {  // the ragged last tile
            for (int j = 0; j < TILE / NT; ++j) {
                const int64_t idx = t * TILE + j * NT + threadIdx.x;
                const bool valid = idx < A.n;
                count_key<KM>(valid ? A.keys[idx] : K(0), valid, A.shift, hb, bad, A.n, lane0);
            }
        }
        __syncthreads();
        const uint32_t c = hb[d];
        hb[d] = 0u;  // counted into again two tiles later, after this tile's barrier
        A.tile_pre[t * RADIX + d] = run;
        run += c;
        if (nfull) {
#pragma unroll
            for (int j = 0; j < VPT; ++j) v[j] = nx[j];
        }
    }
    A.blk_tot[(int64_t)blockIdx.x * RADIX + d] = run;
    if (KM == KM_ANCHOR && bad) set_status(A.status, ST_NONFINITE);
}

// One block of 1024 threads: blk_pre[b][d] = start of digit d + the count of
// digit d in the ranges before b.  Thread (g, c) owns the four digits 4g..4g+3
// (16-byte loads) and the c-th of 16 chunks of the ranges; the ranges' rows
// are read with 8 loads in flight per thread.
__global__ void __launch_bounds__(1024) k_count_scan(const uint32_t* __restrict__ blk_tot,
                                                     uint32_t* __restrict__ blk_pre, int G,
                                                     uint32_t* __restrict__ use_match) {
    constexpr int CH = 16, U = 8;
    __shared__ uint4 part[CH][RADIX / 4];
    __shared__ uint32_t base[RADIX];
    const int g = threadIdx.x & (RADIX / 4 - 1), c = threadIdx.x >> 6;
    const int rc = (G + CH - 1) / CH, r0 = std::min(G, c * rc), r1 = std::min(G, r0 + rc);
    const uint4* tot4 = reinterpret_cast<const uint4*>(blk_tot);
    uint4* pre4 = reinterpret_cast<uint4*>(blk_pre);
    uint4 sum = make_uint4(0u, 0u, 0u, 0u);
    for (int r = r0; r < r1; r += U) {
        uint4 x[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            x[u] = r + u < r1 ? tot4[(int64_t)(r + u) * (RADIX / 4) + g] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            sum.x += x[u].x;
            sum.y += x[u].y;
            sum.z += x[u].z;
            sum.w += x[u].w;
        }
    }
    part[c][g] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {  // warp 0: exclusive scan of the 256 digit totals, 8 per lane
        const int lane = threadIdx.x;
        const uint32_t* pw = reinterpret_cast<const uint32_t*>(&part[0][0]);
        uint32_t tot[8], acc = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int dd = lane * 8 + u;
            uint32_t t = 0;
#pragma unroll
            for (int cc = 0; cc < CH; ++cc) t += pw[cc * RADIX + dd];
            tot[u] = t;
            acc += t;
        }
        uint32_t inc = acc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(FULL, inc, off);
            if (lane >= off) inc += o;
        }
        uint32_t ex = inc - acc;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            base[lane * 8 + u] = ex;
            ex += tot[u];
        }
        // expected distinct digits among 32 keys: sum over d of 1 - (1 - p_d)^32
        const float all = (float)__shfl_sync(FULL, inc, 31);
        float ed = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float q = 1.f - (float)tot[u] / fmaxf(all, 1.f);
#pragma unroll
            for (int k = 0; k < 5; ++k) q *= q;  // q^32
            ed += 1.f - q;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ed += __shfl_xor_sync(FULL, ed, off);
        if (lane == 0) *use_match = ed < MATCH_BELOW_DISTINCT ? 1u : 0u;
    }
    __syncthreads();
    uint4 pre = make_uint4(base[4 * g], base[4 * g + 1], base[4 * g + 2], base[4 * g + 3]);
    for (int cc = 0; cc < c; ++cc) {
        const uint4 p = part[cc][g];
        pre.x += p.x;
        pre.y += p.y;
        pre.z += p.z;
        pre.w += p.w;
    }
    for (int r = r0; r < r1; r += U) {
        uint4 x[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            x[u] = r + u < r1 ? tot4[(int64_t)(r + u) * (RADIX / 4) + g] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (r + u < r1) pre4[(int64_t)(r + u) * (RADIX / 4) + g] = pre;
            pre.x += x[u].x;
            pre.y += x[u].y;
            pre.z += x[u].z;
            pre.w += x[u].w;
        }
    }
}

// ------------------------------------------------------------------ scatter
// what a k_scatter launch does besides the digit pass
enum : int {
    F_KEYMAP = 1,  // the keys are anchor bits: map them to sort keys
    F_IOTA = 2,    // the payload of key i is its index i (no payload input)
    F_UNMAP = 4,   // write the keys back as anchor bits
    F_CLAMP = 8,   // the keys are indices: map them to min(index, n)
    F_PAIR = 16,   // a second 4-byte payload array rides along (v2src -> v2dst), staged in a
                   // second round through the staging area after the keys and payloads
};

template <typename K, typename V>
struct ScatterArgs {
    const K* ksrc;                     // this pass's keys (with F_KEYMAP: the anchor bits)
    const V* vsrc;                     // and payloads (not read with F_IOTA)
    K* kdst;                           // the keys in digit order (with F_UNMAP: anchor bits)
    V* vdst;                           // and their payloads
    const uint32_t* v2src;             // with F_PAIR: the second payload, in and out
    uint32_t* v2dst;
    int64_t n, ntiles, R;              // R: tiles per k_count block
    int shift;
    const uint32_t* tile_pre;
    const uint32_t* blk_pre;
    const uint32_t* use_match;         // ranking of this pass (k_count_scan's choice)
    uint32_t* status;
    uint32_t polls;                    // bound of each copy wait
    int force_expiry;                  // test hook: every block's first copy is never issued
};

// Dynamic shared memory of one k_scatter block.
template <typename K, typename V, int KPT, int S, int F>
constexpr size_t scatter_smem() {
    constexpr size_t TILE = (size_t)SORT_NT * KPT;
    return S * TILE * sizeof(K) + ((F & F_IOTA) ? 0 : S * TILE * sizeof(V)) + TILE * (sizeof(K) + sizeof(V)) +
           (size_t)SORT_NW * RADIX * 4;
}

template <typename K, typename V, int KPT, int S, int F>
__global__ void __launch_bounds__(SORT_NT, LX_SORT_MINB) k_scatter(ScatterArgs<K, V> A) {
    constexpr bool IOTA = F & F_IOTA, UNMAP = F & F_UNMAP, PAIR = F & F_PAIR;
    constexpr int KM = (F & F_KEYMAP) ? KM_ANCHOR : (F & F_CLAMP) ? KM_CLAMP : KM_NONE;
    constexpr int NT = SORT_NT, NW = SORT_NW, TILE = NT * KPT;
    static_assert(TILE * (sizeof(K) + sizeof(V)) >= NW * (RADIX + 1) * 4, "the staging area holds the match masks");
    static_assert(!PAIR || (sizeof(K) == 4 && sizeof(V) == 4), "a second payload rides with 4-byte keys and payloads");
    extern __shared__ __align__(128) unsigned char dyn[];
    K* stage_k = reinterpret_cast<K*>(dyn);                    // [S][TILE] (F_KEYMAP: anchor bits)
    V* stage_v = reinterpret_cast<V*>(stage_k + S * TILE);     // [S][TILE] (not with F_IOTA)
    K* out_k = reinterpret_cast<K*>(stage_v + (IOTA ? 0 : S * TILE));  // [TILE] in digit order
    V* out_v = reinterpret_cast<V*>(out_k + TILE);             // [TILE]
    uint32_t* wcnt = reinterpret_cast<uint32_t*>(out_v + TILE);  // [NW][RADIX]
    __shared__ __align__(8) uint64_t full[S];
    __shared__ int32_t gofs[RADIX];   // output position of staged key q of digit d: gofs[d] + q
    __shared__ uint32_t scan_sm[NW + 1];
    __shared__ int sh_abort;

    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int d = threadIdx.x;  // the digit of this thread in the per-digit steps
    const int shift = A.shift;
    const unsigned ltmask = lanemask_lt();
    const uint32_t lanebit = 1u << lane, gtmask = ~(ltmask | lanebit);
    const int64_t G = gridDim.x;
    const bool use_match = *A.use_match != 0u;
    // The block's i-th tile (-1 past its share).  Blocked: block b owns the
    // contiguous tiles [b per, (b + 1) per), so that the tiles in work at one
    // time are spread over the whole array and so are the runs they write
    // into each digit's region (round robin would have them all write at one
    // offset of every region; for digits of equal counts the regions are a
    // power of two apart, and the concurrent writes then crowd a few DRAM
    // channels).  Tiles may go in any order: their offsets come precomputed.
    const int64_t per = (A.ntiles + G - 1) / G;
    auto tile_of = [&](int64_t i) -> int64_t {
#if LX_SORT_BLOCKED
        const int64_t t = (int64_t)blockIdx.x * per + i;
        return i < per && t < A.ntiles ? t : -1;
#else
        const int64_t t = (int64_t)blockIdx.x + i * G;
        return t < A.ntiles ? t : -1;
#endif
    };

    // thread 0: tile t into stage st (a bulk copy for a full tile; a plain
    // arrive for the ragged last tile, which is read from global memory)
    auto refill = [&](int st, int64_t t) {
        if (t < 0) return;
        const int64_t tb = t * TILE;
        if (tb + TILE <= A.n) {
            constexpr uint32_t kb = TILE * sizeof(K), vb = IOTA ? 0u : TILE * (uint32_t)sizeof(V);
            mbar_expect_tx(&full[st], kb + vb);
            bulk_g2s(stage_k + st * TILE, A.ksrc + tb, kb, &full[st]);
            if constexpr (!IOTA) bulk_g2s(stage_v + st * TILE, A.vsrc + tb, vb, &full[st]);
        } else {
            mbar_arrive(&full[st]);
        }
    };

    if (threadIdx.x == 0) {
        sh_abort = 0;
        for (int st = 0; st < S; ++st) mbar_init(&full[st], 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int st = 0; st < S; ++st)
            if (!(A.force_expiry && st == 0)) refill(st, tile_of(st));
    }
    for (int j = threadIdx.x; j < NW * RADIX; j += NT) wcnt[j] = 0u;
    __syncthreads();

    for (int64_t i = 0;; ++i) {
        const int64_t t = tile_of(i);
        if (t < 0) return;  // every copy this block issued has been waited for
        const int st = (int)(i % S);
        // this tile's output offset of digit d, loaded while its copy lands
        const uint32_t off = A.blk_pre[(t / A.R) * RADIX + d] + A.tile_pre[t * RADIX + d];
        // an expired wait is acted on at the first barrier below, together
        if (!mbar_wait_bounded(&full[st], (uint32_t)((i / S) & 1), A.polls)) sh_abort = 1;
        const int64_t tb = t * TILE;
        const int cnt = (int)std::min<int64_t>((int64_t)TILE, A.n - tb);

        auto body = [&](auto full_c, auto rank_c) -> bool {
            constexpr bool FT = decltype(full_c)::value;  // a full tile, staged by the bulk copy
            constexpr int RM = decltype(rank_c)::value;   // how equal digits are found
            const int seg = w * 32 * KPT + lane;          // key i of this thread: seg + 32 i
            K k[KPT];
#pragma unroll
            for (int e = 0; e < KPT; ++e) {
                const int q = seg + 32 * e;
                K raw;
                if constexpr (FT) raw = stage_k[st * TILE + q];
                else raw = q < cnt ? A.ksrc[tb + q] : K(0);
                k[e] = map_key<KM>(raw, A.n);
            }
            // stable rank among the warp's keys of the same digit: rounds in
            // order, lanes in order within a round.  The match masks, if used,
            // live in the staging area (free until the staging below; only
            // generic-proxy accesses touch it, so no proxy fence is needed).
            uint32_t* wmask = reinterpret_cast<uint32_t*>(out_k) + w * (RADIX + 1);
            if constexpr (RM == RANK_MASK) {
                __syncwarp();
                for (int j = lane; j <= RADIX; j += 32) wmask[j] = 0u;
            }
            uint32_t clr = RADIX + 1;
            uint32_t rk[KPT];
#pragma unroll
            for (int e = 0; e < KPT; ++e) {
                const bool valid = FT || seg + 32 * e < cnt;
                const uint32_t dig = valid ? ((uint32_t)(k[e] >> shift) & (RADIX - 1)) : (uint32_t)RADIX;
                unsigned peers;
                if constexpr (RM == RANK_MATCH) peers = __match_any_sync(FULL, dig);
                else if constexpr (RM == RANK_MASK) peers = mask_peers(dig, wmask, clr, lanebit, gtmask);
                else peers = ballot_peers<!FT>(dig);
                rk[e] = group_rank(peers, dig, valid, wcnt + w * RADIX, ltmask);
            }
            __syncthreads();
            if (sh_abort) return false;
            // per digit: the tile's count; wcnt[.][d] becomes the warps' offsets
            // inside the tile's digit-ordered staging (one read and one write
            // of each count: the warps' counts stay in registers across the scan)
            uint32_t xw[NW], c = 0;
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) {
                xw[ww] = wcnt[ww * RADIX + d];
                c += xw[ww];
            }
            uint32_t tot;
            const uint32_t ds = block_excl_sum<NT>(c, scan_sm, tot);
            {
                uint32_t pre = ds;
#pragma unroll
                for (int ww = 0; ww < NW; ++ww) {
                    wcnt[ww * RADIX + d] = pre;
                    pre += xw[ww];
                }
            }
            gofs[d] = (int32_t)(off - ds);
            __syncthreads();
            auto value_of = [&](int q) -> V {
                if constexpr (IOTA) return (V)((int32_t)tb + q);  // n < 2^31
                else if constexpr (FT) return stage_v[st * TILE + q];
                else return A.vsrc[tb + q];
            };
            // 4-byte keys and payloads are staged as one 8-byte pair: one
            // shared store per key, one shared load per key in the write-out
            constexpr bool PACK = sizeof(K) == 4 && sizeof(V) == 4;
            uint2* out_kv = reinterpret_cast<uint2*>(out_k);  // out_k and out_v are contiguous
            if constexpr (PACK) {
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const int q = seg + 32 * e;
                    if (FT || q < cnt) {
                        rk[e] += wcnt[w * RADIX + ((uint32_t)(k[e] >> shift) & (RADIX - 1))];
                        out_kv[rk[e]] = make_uint2((uint32_t)k[e], (uint32_t)value_of(q));
                    }
                }
            } else {
                // stage keys, then payloads, in digit order
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const int q = seg + 32 * e;
                    if (FT || q < cnt) {
                        rk[e] += wcnt[w * RADIX + ((uint32_t)(k[e] >> shift) & (RADIX - 1))];
                        out_k[rk[e]] = k[e];
                    }
                }
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const int q = seg + 32 * e;
                    if (FT || q < cnt) out_v[rk[e]] = value_of(q);
                }
            }
            __syncthreads();
            // the stage is consumed: the copy of this block's tile S rounds
            // later runs while this one is written out
            if (threadIdx.x == 0) {
                fence_proxy_async();
                refill(st, tile_of(i + S));
            }
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) wcnt[ww * RADIX + d] = 0u;
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const int q = (int)threadIdx.x + j * NT;
                if (FT || q < cnt) {
                    K kk;
                    V vv;
                    if constexpr (PACK) {
                        const uint2 kv = out_kv[q];
                        kk = (K)kv.x;
                        vv = (V)kv.y;
                    } else {
                        kk = out_k[q];
                        vv = out_v[q];
                    }
                    const int64_t g = (int64_t)gofs[(uint32_t)(kk >> shift) & (RADIX - 1)] + q;
                    A.kdst[g] = UNMAP ? key_to_bits(kk) : kk;
                    A.vdst[g] = vv;
                    // F_PAIR: position q's output offset replaces its key (read only by this thread)
                    if constexpr (PAIR) out_kv[q].x = (uint32_t)g;  // n < 2^31
                }
            }
            if constexpr (PAIR) {
                // second round: the second payload (read from global memory,
                // coalesced) into the payload slots of the staging area, at the
                // same positions; each slot pairs it with its output offset
                __syncthreads();  // the first round's payloads have been read
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const int q = seg + 32 * e;
                    if (FT || q < cnt) out_kv[rk[e]].y = __ldcs(A.v2src + tb + q);
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < KPT; ++j) {
                    const int q = (int)threadIdx.x + j * NT;
                    if (FT || q < cnt) {
                        const uint2 gw = out_kv[q];
                        A.v2dst[gw.x] = gw.y;
                    }
                }
            }
            __syncthreads();  // out_k, out_v, gofs, wcnt are the next tile's
            return true;
        };
        // the ranking of this pass (uniform over the grid), and full or ragged tile
        using HiRank = std::integral_constant<int, LX_SORT_RANK == 2 ? LX_SORT_HI : LX_SORT_RANK>;
        using MatchRank = std::integral_constant<int, LX_SORT_RANK == 2 ? RANK_MATCH : LX_SORT_RANK>;
        bool ok;
        if (cnt == TILE) ok = use_match ? body(std::true_type{}, MatchRank{}) : body(std::true_type{}, HiRank{});
        else ok = use_match ? body(std::false_type{}, MatchRank{}) : body(std::false_type{}, HiRank{});
        if (!ok) {
            // a copy never landed: report it, give this block's copies in
            // flight (this one included) a bounded time to land, and leave
            if (threadIdx.x == 0) {
                set_status(A.status, ST_TIMEOUT);
                for (int64_t j = 0; j < S; ++j)
                    if (tile_of(i + j) >= 0)
                        (void)mbar_wait_bounded(&full[(i + j) % S], (uint32_t)(((i + j) / S) & 1), A.polls);
            }
            return;
        }
    }
}

// ------------------------------------------------------------------ host side
namespace {
thread_local uint32_t g_sort_polls = MBAR_POLLS;
thread_local int g_sort_force_expiry = 0;
}  // namespace

void set_sort_wait(uint32_t polls, int force_expiry) {
    g_sort_polls = polls ? polls : MBAR_POLLS;
    g_sort_force_expiry = force_expiry;
}

template <typename T> constexpr int sort_tile() { return SORT_NT * SortShape<T>::KPT; }

// Workspace shared by the digit passes over one array: per-tile counts,
// per-range totals and prefixes, and the pass's ranking choice.
struct PassWs {
    uint32_t* tile_pre;
    uint32_t* blk_tot;
    uint32_t* blk_pre;
    uint32_t* mode;
};
static size_t pass_ws_bytes(int64_t ntiles) {
    return Carve::need((size_t)(ntiles * RADIX), 4) + 2 * Carve::need((size_t)COUNT_MAX_BLOCKS * RADIX, 4) +
           Carve::need(1, 4);
}
static PassWs pass_carve(Carve& cv, int64_t ntiles) {
    PassWs W;
    W.tile_pre = cv.take<uint32_t>((size_t)(ntiles * RADIX));
    W.blk_tot = cv.take<uint32_t>((size_t)COUNT_MAX_BLOCKS * RADIX);
    W.blk_pre = cv.take<uint32_t>((size_t)COUNT_MAX_BLOCKS * RADIX);
    W.mode = cv.take<uint32_t>(1);
    return W;
}

// One stable digit pass, (key >> shift) & 255, of n keys ksrc with payloads
// vsrc into kdst, vdst: k_count, k_count_scan, k_scatter.
template <typename K, typename V, int KPT, int S, int F>
static cudaError_t digit_pass(const K* ksrc, const V* vsrc, K* kdst, V* vdst, int64_t n, int shift,
                              const PassWs& W, uint32_t* status, int dev, int sms, cudaStream_t st,
                              const uint32_t* v2src = nullptr, uint32_t* v2dst = nullptr) {
    const int64_t tile = (int64_t)SORT_NT * KPT;
    const int64_t ntiles = (n + tile - 1) / tile;
    // k_count: contiguous ranges of R >= 4 tiles (fewer ranges keep k_count_scan
    // short on small arrays), every block non-empty
    const int64_t gmax = std::max<int64_t>(
        1, std::min<int64_t>(std::min<int64_t>((int64_t)COUNT_BLOCKS_PER_SM * sms, COUNT_MAX_BLOCKS), ntiles / 4));
    const int64_t R = (ntiles + gmax - 1) / gmax;
    const int64_t Gc = (ntiles + R - 1) / R;
    CountArgs<K> C;
    C.keys = ksrc;
    C.n = n;
    C.ntiles = ntiles;
    C.R = R;
    C.shift = shift;
    C.tile_pre = W.tile_pre;
    C.blk_tot = W.blk_tot;
    C.status = status;
    k_count<K, KPT, (F & F_KEYMAP) ? KM_ANCHOR : (F & F_CLAMP) ? KM_CLAMP : KM_NONE><<<(unsigned)Gc, SORT_NT, 0, st>>>(C);
    k_count_scan<<<1, 1024, 0, st>>>(W.blk_tot, W.blk_pre, (int)Gc, W.mode);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ScatterArgs<K, V> A;
    A.ksrc = ksrc;
    A.vsrc = vsrc;
    A.kdst = kdst;
    A.vdst = vdst;
    A.v2src = v2src;
    A.v2dst = v2dst;
    A.n = n;
    A.ntiles = ntiles;
    A.R = R;
    A.shift = shift;
    A.tile_pre = W.tile_pre;
    A.blk_pre = W.blk_pre;
    A.use_match = W.mode;
    A.status = status;
    A.polls = g_sort_polls;
    A.force_expiry = g_sort_force_expiry;
    constexpr auto kern = k_scatter<K, V, KPT, S, F>;
    constexpr size_t smem = scatter_smem<K, V, KPT, S, F>();
    int per = 0;
    e = blocks_per_sm<kern>(dev, SORT_NT, smem, &per);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ntiles, (int64_t)per * sms);
    kern<<<(unsigned)grid, SORT_NT, smem, st>>>(A);
    return cudaGetLastError();
}

size_t sort_ws_bytes(int64_t n, int f64) {
    const int64_t tile = f64 ? sort_tile<double>() : sort_tile<float>();
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    const size_t ks = f64 ? 8 : 4;
    return Carve::need((size_t)n, ks) + Carve::need((size_t)n, 4) + pass_ws_bytes(ntiles);
}

template <typename T>
cudaError_t sort_run(const T* a, int64_t n, T* sorted, int32_t* perm, void* ws, size_t ws_bytes,
                     uint32_t* status, cudaStream_t st) {
    using K = typename KeyOf<T>::K;
    if (n == 0) return cudaSuccess;
    constexpr int P = sizeof(K), KPT = SortShape<T>::KPT, S = SortShape<T>::S;
    const int64_t tile = sort_tile<T>();
    const int64_t ntiles = (n + tile - 1) / tile;
    Carve cv(ws, ws_bytes);
    K* kws = cv.take<K>(n);
    int32_t* vws = cv.take<int32_t>(n);
    const PassWs W = pass_carve(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = current_device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    K* kout = reinterpret_cast<K*>(sorted);
    const K* ksrc = reinterpret_cast<const K*>(a);
    const int32_t* vsrc = nullptr;
    profile_before(st);
    for (int pass = 0; pass < P; ++pass) {
        const bool to_out = ((P - 1 - pass) % 2) == 0;  // the last pass lands in the outputs
        K* kdst = to_out ? kout : kws;
        int32_t* vdst = to_out ? perm : vws;
        if (pass == 0)
            e = digit_pass<K, int32_t, KPT, S, F_KEYMAP | F_IOTA>(ksrc, vsrc, kdst, vdst, n, 8 * pass, W, status,
                                                                  dev, sms, st);
        else if (pass == P - 1)
            e = digit_pass<K, int32_t, KPT, S, F_UNMAP>(ksrc, vsrc, kdst, vdst, n, 8 * pass, W, status, dev, sms, st);
        else
            e = digit_pass<K, int32_t, KPT, S, 0>(ksrc, vsrc, kdst, vdst, n, 8 * pass, W, status, dev, sms, st);
        if (e != cudaSuccess) return e;
        ksrc = kdst;
        vsrc = vdst;
    }
    profile_after(st);
    return cudaSuccess;
}

// ------------------------------------------------------------------ sort carrying a value
// The fp32 sort with a second payload: the value x[i] of each anchor rides
// through the digit passes beside its index, so that the values arrive in
// sorted order (xs[r] = x[perm[r]]) with coalesced writes, instead of a random
// gather after the sort.  Each pass stages the keys with the indices, then the
// values through the same staging area (the same shared memory as the plain sort).
#ifndef LX_CARRY_KPT
#define LX_CARRY_KPT 24
#endif
constexpr int CARRY_KPT = LX_CARRY_KPT;

size_t sort_carry_ws_bytes(int64_t n) {
    const int64_t tile = (int64_t)SORT_NT * CARRY_KPT;
    const int64_t ntiles = std::max<int64_t>(1, (n + tile - 1) / tile);
    return 3 * Carve::need((size_t)n, 4) + pass_ws_bytes(ntiles);
}

cudaError_t sort_carry_run(const float* a, const float* x, int64_t n, float* sorted, int32_t* perm, float* xs,
                           void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    constexpr int P = 4, KPT = CARRY_KPT;
    const int64_t tile = (int64_t)SORT_NT * KPT;
    const int64_t ntiles = (n + tile - 1) / tile;
    Carve cv(ws, ws_bytes);
    uint32_t* kws = cv.take<uint32_t>(n);
    int32_t* vws = cv.take<int32_t>(n);
    uint32_t* wws = cv.take<uint32_t>(n);
    const PassWs W = pass_carve(cv, ntiles);
    if (!cv.ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = current_device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    const uint32_t* ksrc = reinterpret_cast<const uint32_t*>(a);
    const int32_t* vsrc = nullptr;
    const uint32_t* wsrc = reinterpret_cast<const uint32_t*>(x);
    profile_before(st);
    for (int pass = 0; pass < P; ++pass) {
        const bool to_out = ((P - 1 - pass) % 2) == 0;  // the last pass lands in the outputs
        uint32_t* kdst = to_out ? reinterpret_cast<uint32_t*>(sorted) : kws;
        int32_t* vdst = to_out ? perm : vws;
        uint32_t* wdst = to_out ? reinterpret_cast<uint32_t*>(xs) : wws;
        if (pass == 0)
            e = digit_pass<uint32_t, int32_t, KPT, 1, F_KEYMAP | F_IOTA | F_PAIR>(ksrc, vsrc, kdst, vdst, n, 0, W,
                                                                                  status, dev, sms, st, wsrc, wdst);
        else if (pass == P - 1)
            e = digit_pass<uint32_t, int32_t, KPT, 1, F_UNMAP | F_PAIR>(ksrc, vsrc, kdst, vdst, n, 8 * pass, W,
                                                                        status, dev, sms, st, wsrc, wdst);
        else
            e = digit_pass<uint32_t, int32_t, KPT, 1, F_PAIR>(ksrc, vsrc, kdst, vdst, n, 8 * pass, W, status, dev,
                                                              sms, st, wsrc, wdst);
        if (e != cudaSuccess) return e;
        ksrc = kdst;
        vsrc = vdst;
        wsrc = wdst;
    }
    profile_after(st);
    return cudaSuccess;
}

// ------------------------------------------------------------------ permutation
// dst[idx[i]] = src[i] (IOTA: dst[idx[i]] = i) for i < n.  Writing 4 or 8
// bytes at random positions of a large array costs a partial 32-byte sector
// write each, which the L2 cache does not merge well (measured: 3.3x the
// bytes written to DRAM, even with the targets grouped into a window of a few
// MB).  So the elements are first ordered by the group of 2^PERM_GB targets
// they land in, with stable radix digit passes over the group number
// (index >> PERM_GB; one pass up to 256 groups, two up to 65536, which covers
// n <= 2^30 with 4-byte elements), and each block of k_place_group then fills
// one group's 2^PERM_GB outputs in shared memory and writes them out with
// whole-sector stores.  Entries of idx outside [0, n) are clamped to n, sort
// last and are dropped; a position that no entry names is left untouched
// (a bitmap of the written positions guards the store).
// keys per thread of the permutation's digit passes: 24 with 4-byte elements
// (the plain sort's shape), 16 with 8-byte ones (shared memory for two blocks per SM)
template <typename V> struct PermKPT { static constexpr int v = sizeof(V) == 4 ? 24 : 16; };
template <typename V> struct PermGB { static constexpr int v = sizeof(V) == 8 ? 13 : 14; };  // 64 KB of outputs

// group_lo[q] = first position of the ordered keys whose group (index below
// bit 31, >> gb) is >= q, for q <= ngroups; with ordered == 0 (no digit pass
// ran: one group) just {0, m}.
__global__ void __launch_bounds__(256) k_group_bounds(const uint32_t* __restrict__ tk, int64_t m, int gb,
                                                      int64_t ngroups, int ordered, int64_t* __restrict__ group_lo) {
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q > ngroups) return;
    if (!ordered) {
        group_lo[q] = q == 0 ? 0 : m;
        return;
    }
    int64_t lo = 0, hi = m;  // first i with group(tk[i]) >= q
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if ((int64_t)((tk[mid] & 0x7FFFFFFFu) >> gb) < q) lo = mid + 1;
        else hi = mid;
    }
    group_lo[q] = lo;
}

template <typename V, int GB, bool IOTA>
__global__ void __launch_bounds__(1024) k_place_group(const uint32_t* __restrict__ tk, const V* __restrict__ tv,
                                                      const int64_t* __restrict__ group_lo, int64_t n,
                                                      V* __restrict__ dst) {
    constexpr int GS = 1 << GB;
    extern __shared__ __align__(128) unsigned char dyn[];
    V* buf = reinterpret_cast<V*>(dyn);                       // [GS]
    uint32_t* wrote = reinterpret_cast<uint32_t*>(buf + GS);  // [GS / 32]
    const int64_t q = blockIdx.x;
    const int64_t base = q << GB;
    const int64_t lo = group_lo[q], hi = group_lo[q + 1];
    for (int j = threadIdx.x; j < GS / 32; j += blockDim.x) wrote[j] = 0u;
    __syncthreads();
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
        const uint32_t j = __ldcs(tk + i);
        if ((int64_t)j < n) {
            const int p = (int)(j - base);
            buf[p] = IOTA ? (V)i : __ldcs(tv + i);
            atomicOr(&wrote[p >> 5], 1u << (p & 31));
        }
    }
    __syncthreads();
    const int cnt = (int)std::min<int64_t>(GS, n - base);
    for (int p = threadIdx.x; p < cnt; p += blockDim.x)
        if ((wrote[p >> 5] >> (p & 31)) & 1u) __stcs(dst + base + p, buf[p]);
}

template <typename V>
static int64_t perm_groups(int64_t n) {
    return ((n + ((int64_t)1 << PermGB<V>::v) - 1) >> PermGB<V>::v);
}

// digit passes over the group number (of the valid indices 0..n-1)
template <typename V>
static int perm_passes(int64_t n) {
    const int64_t top = (n - 1) >> PermGB<V>::v;  // the largest group number
    int bits = 0;
    while (bits < 32 && (top >> bits) > 0) ++bits;
    return (bits + 7) / 8;
}

size_t permute_ws_bytes(int64_t n, int vbytes) {
    const int P = vbytes == 8 ? perm_passes<int64_t>(n) : perm_passes<int32_t>(n);
    const int64_t ng = vbytes == 8 ? perm_groups<int64_t>(n) : perm_groups<int32_t>(n);
    const int64_t ptile = (int64_t)SORT_NT * (vbytes == 8 ? PermKPT<int64_t>::v : PermKPT<int32_t>::v);
    const int64_t ntiles = (n + ptile - 1) / ptile;
    const int bufs = P == 0 ? 0 : (P == 1 ? 1 : 2);
    return bufs * (Carve::need((size_t)n, 4) + Carve::need((size_t)n, (size_t)vbytes)) + pass_ws_bytes(ntiles) +
           Carve::need((size_t)(ng + 2), 8);
}

template <typename V>
cudaError_t permute_run(const V* src, const int32_t* idx, int64_t n, V* dst, void* ws, size_t ws_bytes,
                        uint32_t* status, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    constexpr int GB = PermGB<V>::v;
    int dev = 0, sms = 0;
    cudaError_t e = current_device_sms(&dev, &sms);
    if (e != cudaSuccess) return e;
    const bool iota = src == nullptr;
    const int P = perm_passes<V>(n);
    const int64_t ng = perm_groups<V>(n);
    constexpr int PERM_KPT = PermKPT<V>::v;
    const int64_t ntiles = (n + (int64_t)SORT_NT * PERM_KPT - 1) / ((int64_t)SORT_NT * PERM_KPT);
    Carve cv(ws, ws_bytes);
    uint32_t* tk[2] = {nullptr, nullptr};
    V* tv[2] = {nullptr, nullptr};
    for (int b = 0; b < (P == 0 ? 0 : (P == 1 ? 1 : 2)); ++b) {
        tk[b] = cv.take<uint32_t>(n);
        tv[b] = cv.take<V>(n);
    }
    const PassWs W = pass_carve(cv, ntiles);
    int64_t* group_lo = cv.take<int64_t>(ng + 2);
    if (!cv.ok) return cudaErrorInvalidValue;
    const uint32_t* ksrc = reinterpret_cast<const uint32_t*>(idx);
    const V* vsrc = src;
    bool vio = iota;  // the payloads are still the indices i, not read from memory
    for (int p = 0; p < P; ++p) {
        uint32_t* kd = tk[p & 1];
        V* vd = tv[p & 1];
        const int shift = GB + 8 * p;
        if (p == 0 && vio)
            e = digit_pass<uint32_t, V, PERM_KPT, 1, F_CLAMP | F_IOTA>(ksrc, nullptr, kd, vd, n, shift, W, status,
                                                                       dev, sms, st);
        else if (p == 0)
            e = digit_pass<uint32_t, V, PERM_KPT, 1, F_CLAMP>(ksrc, vsrc, kd, vd, n, shift, W, status, dev, sms, st);
        else
            e = digit_pass<uint32_t, V, PERM_KPT, 1, 0>(ksrc, vsrc, kd, vd, n, shift, W, status, dev, sms, st);
        if (e != cudaSuccess) return e;
        ksrc = kd;
        vsrc = vd;
        vio = false;
    }
    // group boundaries of the ordered keys (with no pass: one group, all of idx)
    k_group_bounds<<<(unsigned)((ng + 1 + 255) / 256), 256, 0, st>>>(ksrc, n, GB, ng, P > 0 ? 1 : 0, group_lo);
    constexpr size_t smem = ((size_t)1 << GB) * sizeof(V) + ((size_t)1 << GB) / 8;
    auto place = [&](auto kc) -> cudaError_t {
        constexpr auto kern = decltype(kc)::value;
        int per = 0;  // raises the kernel's shared-memory limit once per device (no per-call host state)
        cudaError_t r = blocks_per_sm<kern>(dev, 1024, smem, &per);
        if (r != cudaSuccess) return r;
        kern<<<(unsigned)ng, 1024, smem, st>>>(ksrc, vsrc, group_lo, n, dst);
        return cudaGetLastError();
    };
    return vio ? place(std::integral_constant<decltype(&k_place_group<V, GB, true>), &k_place_group<V, GB, true>>{})
               : place(std::integral_constant<decltype(&k_place_group<V, GB, false>), &k_place_group<V, GB, false>>{});
}

template cudaError_t permute_run<int32_t>(const int32_t*, const int32_t*, int64_t, int32_t*, void*, size_t,
                                          uint32_t*, cudaStream_t);
template cudaError_t permute_run<int64_t>(const int64_t*, const int32_t*, int64_t, int64_t*, void*, size_t,
                                          uint32_t*, cudaStream_t);

template cudaError_t sort_run<float>(const float*, int64_t, float*, int32_t*, void*, size_t,
                                     uint32_t*, cudaStream_t);
template cudaError_t sort_run<double>(const double*, int64_t, double*, int32_t*, void*, size_t,
                                      uint32_t*, cudaStream_t);

}  // namespace lx
