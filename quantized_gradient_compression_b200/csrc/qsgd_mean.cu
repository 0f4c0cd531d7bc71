// The last step of the mean of K received streams: out[i] <- fl(out[i] / K).
//
// Method: the data-parallel use of the definition paragraph of "QSGD (Quantized
// Stochastic Gradient Descent) with Elias Coding" (AIMech curated entry): each node
// averages the K decoded gradients it receives.  The sum is the decode-accumulate
// kernels' (left to right); this pass divides it, one IEEE division per coordinate.
#include <cuda_runtime.h>

#include <algorithm>

#include "qsgd_internal.h"

namespace qsgd {
namespace {

constexpr int kDivBlock = 256;

template <bool kVec4>
__global__ void __launch_bounds__(kDivBlock) div_by(float* out, uint64_t n, float k) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kDivBlock;
    const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * kDivBlock + threadIdx.x;
    if (kVec4) {
        const uint64_t n4 = n / 4;
        for (uint64_t j = t0; j < n4; j += stride) {
            float4 v = reinterpret_cast<float4*>(out)[j];
            v.x = __fdiv_rn(v.x, k);
            v.y = __fdiv_rn(v.y, k);
            v.z = __fdiv_rn(v.z, k);
            v.w = __fdiv_rn(v.w, k);
            reinterpret_cast<float4*>(out)[j] = v;
        }
        for (uint64_t i = 4 * n4 + t0; i < n; i += stride) out[i] = __fdiv_rn(out[i], k);
    } else {
        for (uint64_t i = t0; i < n; i += stride) out[i] = __fdiv_rn(out[i], k);
    }
}

}  // namespace

cudaError_t launch_div(float* out, uint64_t n, uint32_t K, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool vec4 = (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
    const uint64_t items = vec4 ? n / 4 + 1 : n;
    const int grid = static_cast<int>(
        std::max<uint64_t>(1, std::min<uint64_t>((items + kDivBlock - 1) / kDivBlock, static_cast<uint64_t>(sms) * 8)));
    const float k = static_cast<float>(K);  // K <= 2^24: exact
    if (vec4)
        div_by<true><<<grid, kDivBlock, 0, stream>>>(out, n, k);
    else
        div_by<false><<<grid, kDivBlock, 0, stream>>>(out, n, k);
    return cudaGetLastError();
}

}  // namespace qsgd
