// Sums of states across sequence parts: the exchange step of a prefill whose
// sequence is split over several devices.
//
// The state after a sequence is the sum of its parts' states ("Kernelized
// Linear Attention: Breaking the Capacity Wall with Symmetric Cones", s2.3:
// the state propagates across blocks as a prefix sum), so part r starts from
// the exclusive prefix carry_r = sum_{r' < r} state_r'.
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

// out[z] = in[0] + ... + in[z - 1] (out[0] = 0) for z = 0 .. nparts - 1,
// four floats per thread, summed in part order.
__global__ void __launch_bounds__(256) exclusive_prefix_kernel(const float4 *__restrict__ in,
                                                               int nparts, long n4,
                                                               float4 *__restrict__ out) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
         i += (long)gridDim.x * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int z = 0; z < nparts; ++z) {
            out[(size_t)z * n4 + i] = acc;
            const float4 x = in[(size_t)z * n4 + i];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
    }
}

}  // namespace

cudaError_t exclusive_prefix(const float *in, int nparts, size_t n, float *out,
                             cudaStream_t stream) {
    const long n4 = (long)(n / 4);
    const int blocks = (int)((n4 + 255) / 256 < 4 * 148 ? (n4 + 255) / 256 : 4 * 148);
    exclusive_prefix_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(in),
                                                        nparts, n4,
                                                        reinterpret_cast<float4 *>(out));
    return after_launch();
}

}  // namespace kata
