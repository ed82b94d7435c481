// pending.cu -- entry points whose kernels are not written yet report
// cudaErrorNotSupported (mapped to LAPLEX_ECUDA by the C ABI).
#include "laplex_impl.h"
namespace lx {
size_t gen_ws_bytes(int64_t, int64_t, int64_t, bool, int) { return 0; }
template <typename T>
cudaError_t gen_run(GenArgs<T>, int64_t, bool, void*, size_t, cudaStream_t) { return cudaErrorNotSupported; }
template cudaError_t gen_run<float>(GenArgs<float>, int64_t, bool, void*, size_t, cudaStream_t);
template cudaError_t gen_run<double>(GenArgs<double>, int64_t, bool, void*, size_t, cudaStream_t);
size_t bwd_ws_bytes(int64_t, int) { return 0; }
template <typename T>
cudaError_t bwd_run(const T*, const int32_t*, int64_t, const T*, const T*, T*, T*, void*, size_t, uint32_t*, cudaStream_t) { return cudaErrorNotSupported; }
template cudaError_t bwd_run<float>(const float*, const int32_t*, int64_t, const float*, const float*, float*, float*, void*, size_t, uint32_t*, cudaStream_t);
template cudaError_t bwd_run<double>(const double*, const int32_t*, int64_t, const double*, const double*, double*, double*, void*, size_t, uint32_t*, cudaStream_t);
}
