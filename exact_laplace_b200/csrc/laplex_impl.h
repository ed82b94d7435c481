// laplex_impl.h -- internal host-side interface between the C ABI (capi.cu)
// and the kernel files.  Not installed; not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lx {

// sticky device status bits, kept in the first word of the workspace header
constexpr uint32_t ST_NONFINITE = 1u;
constexpr uint32_t ST_TIMEOUT = 2u;
constexpr size_t HEADER_BYTES = 256;

// Sets the calling thread's message returned by laplex_last_error() (capi.cu).
void set_last_error(const char* fmt, ...);

// Optional events recorded around a call's dominant kernel (capi.cu, thread-local).
struct ProfileEvents {
    cudaEvent_t before;
    cudaEvent_t after;
};
const ProfileEvents& profile_events();
inline void profile_before(cudaStream_t st) {
    if (profile_events().before) cudaEventRecord(profile_events().before, st);
}
inline void profile_after(cudaStream_t st) {
    if (profile_events().after) cudaEventRecord(profile_events().after, st);
}

// Bump allocator over the caller's workspace (256-byte granules).
struct Carve {
    char* base;
    size_t off;
    size_t cap;
    bool ok;
    Carve(void* b, size_t c) : base(static_cast<char*>(b)), off(0), cap(c), ok(true) {}
    template <typename U>
    U* take(size_t count) {
        size_t bytes = (count * sizeof(U) + 255) / 256 * 256;
        if (off + bytes > cap) { ok = false; return nullptr; }
        U* p = reinterpret_cast<U*>(base + off);
        off += bytes;
        return p;
    }
    static size_t need(size_t count, size_t elem) { return (count * elem + 255) / 256 * 256; }
};

// -------------------------------------------------------------- symmetric / phased
template <typename T>
struct SymArgs {
    const T* s;           // sorted anchors [n]
    int64_t n;
    const T* x;           // input rows
    const int32_t* pin;   // gather rows of x through pin (NULL: sorted order)
    int64_t ldx;
    T* y;                 // output rows
    const int32_t* pout;  // scatter rows of y through pout (NULL: sorted order)
    int64_t ldy;
    const T* phi;         // phases (phased only), indexed through paux
    const T* D;           // optional per-anchor scale of the input, through paux
    const int32_t* paux;
    int64_t col0;         // first column of this pass
    int ncol;             // columns in this pass
    uint32_t* status;
};

size_t sym_ws_bytes(int64_t n, int64_t B, bool phased, int f64);
template <typename T>
cudaError_t sym_run(SymArgs<T> A, int64_t B, bool phased, void* ws, size_t ws_bytes,
                    cudaStream_t st);

// streaming path of the symmetric product (x in sorted order, one column)
size_t stream_ws_bytes(int64_t n, int f64);
template <typename T>
cudaError_t stream_run(const T* s, const T* x, T* y, const int32_t* pout, int64_t n, void* ws,
                       size_t ws_bytes, uint32_t* status, cudaStream_t st);

// -------------------------------------------------------------- sort
size_t sort_ws_bytes(int64_t n, int f64);
// bound of each bulk-copy wait of the calling thread's later sorts (0: the
// default, 2^20 polls), and a test switch under which the first copy of every
// block of a digit pass is never issued, so that its wait runs to the bound
void set_sort_wait(uint32_t polls, int force_expiry);
template <typename T>
cudaError_t sort_run(const T* a, int64_t n, T* sorted, int32_t* perm, void* ws,
                     size_t ws_bytes, uint32_t* status, cudaStream_t st);

// fp32 sort whose values x ride along: xs[r] = x[perm[r]]
size_t sort_carry_ws_bytes(int64_t n);
cudaError_t sort_carry_run(const float* a, const float* x, int64_t n, float* sorted, int32_t* perm, float* xs,
                           void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st);

// -------------------------------------------------------------- permutation
// dst[idx[i]] = src[i] for i < n (src NULL: dst[idx[i]] = i); V is a 4- or
// 8-byte element moved as bits.  Entries of idx outside [0, n) are dropped.
size_t permute_ws_bytes(int64_t n, int vbytes);
template <typename V>
cudaError_t permute_run(const V* src, const int32_t* idx, int64_t n, V* dst, void* ws, size_t ws_bytes,
                        uint32_t* status, cudaStream_t st);

// -------------------------------------------------------------- general (merged)
template <typename T>
struct GenArgs {
    const T* sa; const int32_t* pa; int64_t n;     // output side anchors (sorted) + perm
    const T* sb; const int32_t* pb; int64_t k;     // input side anchors (sorted) + perm
    const T* x; int64_t ldx;                       // input rows on the b side
    T* y; int64_t ldy;                             // output rows on the a side
    const int32_t* pout;                           // scatter of y (NULL: sorted a order)
    const int32_t* pin;                            // gather of x (NULL: sorted b order)
    const T* phi; const int32_t* pphi;             // output-side phases (a side)
    const T* psi; const int32_t* ppsi;             // input-side phases (b side)
    const T* D; const int32_t* pD;                 // input-side scale (b side)
    int64_t col0;
    int ncol;
    uint32_t* status;
};
size_t gen_ws_bytes(int64_t n, int64_t k, int64_t B, bool phased, int f64);
template <typename T>
cudaError_t gen_run(GenArgs<T> A, int64_t B, bool phased, void* ws, size_t ws_bytes,
                    cudaStream_t st);

// -------------------------------------------------------------- backward
size_t bwd_ws_bytes(int64_t n, int f64);
template <typename T>
cudaError_t bwd_run(const T* s, const int32_t* perm, int64_t n, const T* x, const T* g, T* dx,
                    T* da, void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st);

// -------------------------------------------------------------- general backward
size_t sgen_ws_bytes(int64_t len, int f64);
size_t grammat_ws_bytes(int64_t n, int64_t k, int f64);
template <typename T>
cudaError_t grammat_run(const T* sa, const int32_t* pa, int64_t n, const T* sb, const int32_t* pb, int64_t k,
                        const T* D, T* M, int64_t ldm, void* ws, size_t ws_bytes, cudaStream_t st);
size_t pbwd_ws_bytes(int64_t len, int f64);
template <typename T>
cudaError_t pbwd_run(const T* sa, const int32_t* pa, const T* phi, int64_t n, const T* sb,
                     const int32_t* pb, const T* psi, int64_t k, const T* x, const T* g, T* dx, T* dphi,
                     T* dpsi, T* da, T* db, void* ws, size_t ws_bytes, cudaStream_t st);
template <typename T>
cudaError_t sgen_run(const T* sa, const int32_t* pa, int64_t n, const T* sb, const int32_t* pb,
                     int64_t k, const T* x, const T* g, T* da, T* db, void* ws, size_t ws_bytes,
                     cudaStream_t st);

}  // namespace lx
