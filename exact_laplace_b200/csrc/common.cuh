// common.cuh -- shared device helpers of liblaplex (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "laplex_impl.h"

namespace lx {

constexpr unsigned FULL = 0xffffffffu;

template <typename T> __device__ __forceinline__ T dexp(T v);
// fp32: exp(v) = 2^(v log2 e) on the hardware base-2 exponential in
// flush-to-zero mode (ex2.approx.ftz: relative error about 2^-22; a result
// below FLT_MIN is 0).  Every factor of the scans is at most 1 and at least
// the kernel value exp(-|a_i - b_j|) of each term it carries, so a term whose
// kernel value is >= FLT_MIN is never flushed; only terms below FLT_MIN can
// be lost (at most their |x|-weighted mass).
// Built with LX_ACCURATE_EXP (and --ftz=true): CUDA's expf, whose smaller
// error takes the scan's error below the dense fp32 product's, for a slower
// product; the flush of results below FLT_MIN, and so the cut below, hold.
#ifdef LX_ACCURATE_EXP
template <> __device__ __forceinline__ float dexp<float>(float v) { return expf(v); }
#else
template <> __device__ __forceinline__ float dexp<float>(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v * 1.44269504088896341f));
    return r;
}
#endif
template <> __device__ __forceinline__ double dexp<double>(double v) { return exp(v); }

// A distance beyond which dexp(-d) is exactly 0: fp32, 2^(-88 log2 e) =
// 2^-126.96 < FLT_MIN is flushed (the approximation error of about 2^-22 cannot
// lift it to FLT_MIN); fp64, exp(-746) rounds to 0 (below the smallest
// subnormal).  Carries between tiles are cut off there, bit for bit.
template <typename T> struct ExpCut;
template <> struct ExpCut<float> { static constexpr float v = 88.0f; };
template <> struct ExpCut<double> { static constexpr double v = 746.0; };

template <typename T> __device__ __forceinline__ T dfma(T a, T b, T c) { return fma(a, b, c); }

// sin and cos of a phase.  fp32: the phase is first reduced to [-pi, pi] by
// Cody and Waite's two-constant reduction (t - k 2pi with 2pi split into the
// nearest float and its remainder, each step one fused multiply-add), then the
// hardware sine and cosine (absolute error about 2^-21 on [-pi, pi]); fp64:
// sincos.
template <typename T> __device__ __forceinline__ void psincos(T t, T* s, T* c);
template <> __device__ __forceinline__ void psincos<float>(float t, float* s, float* c) {
    constexpr float TWO_PI_HI = 6.28318548202514648f;   // the float nearest 2 pi
    constexpr float TWO_PI_LO = -1.7484555314695172e-7f;  // 2 pi - TWO_PI_HI
    const float k = rintf(t * 0.159154943091895336f);     // t / (2 pi), rounded
    const float r = fmaf(-k, TWO_PI_LO, fmaf(-k, TWO_PI_HI, t));
    __sincosf(r, s, c);
}
template <> __device__ __forceinline__ void psincos<double>(double t, double* s, double* c) { sincos(t, s, c); }

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
