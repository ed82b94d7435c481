// common.cuh -- shared device helpers of liblaplex (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "laplex_impl.h"

namespace lx {

constexpr unsigned FULL = 0xffffffffu;

template <typename T> __device__ __forceinline__ T dexp(T v);
// fp32: the hardware exp2 path (__expf).  A decay exp(d) with d <= 0 only ever
// multiplies an already-summed value, and terms below FLT_MIN are flushed.
template <> __device__ __forceinline__ float dexp<float>(float v) { return __expf(v); }
template <> __device__ __forceinline__ double dexp<double>(double v) { return exp(v); }

template <typename T> __device__ __forceinline__ T dfma(T a, T b, T c) { return fma(a, b, c); }

__device__ __forceinline__ void set_status(uint32_t* st, uint32_t bits) {
    if (st) atomicOr(st, bits);
}

// 16-byte vector type for T
template <typename T> struct V16;
template <> struct V16<float> { using type = float4; static constexpr int N = 4; };
template <> struct V16<double> { using type = double2; static constexpr int N = 2; };

template <typename T>
__device__ __forceinline__ void ld16(const T* p, T* out) {
    using VT = typename V16<T>::type;
    VT v = *reinterpret_cast<const VT*>(p);
    const T* q = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int i = 0; i < V16<T>::N; ++i) out[i] = q[i];
}

template <typename T>
__device__ __forceinline__ void st16(T* p, const T* in) {
    using VT = typename V16<T>::type;
    VT v;
    T* q = reinterpret_cast<T*>(&v);
#pragma unroll
    for (int i = 0; i < V16<T>::N; ++i) q[i] = in[i];
    *reinterpret_cast<VT*>(p) = v;
}

// streaming (evict-first) variants for data touched exactly once
template <typename T>
__device__ __forceinline__ void ld16_stream(const T* p, T* out) {
    using VT = typename V16<T>::type;
    VT v = __ldcs(reinterpret_cast<const VT*>(p));
    const T* q = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int i = 0; i < V16<T>::N; ++i) out[i] = q[i];
}

template <typename T>
__device__ __forceinline__ void st16_stream(T* p, const T* in) {
    using VT = typename V16<T>::type;
    VT v;
    T* q = reinterpret_cast<T*>(&v);
#pragma unroll
    for (int i = 0; i < V16<T>::N; ++i) q[i] = in[i];
    __stcs(reinterpret_cast<VT*>(p), v);
}

}  // namespace lx
