// Device helpers shared by the libkata kernels.
//
// Packed feature layout (rank-one PSD feature of "Kernelized Linear Attention:
// Breaking the Capacity Wall with Symmetric Cones", s2.2): phi(x) is the upper
// triangle of x x^T, row (a) major. Entry (a, b), a <= b, sits at
// r = a*d - a(a-1)/2 + (b - a) and carries sqrt(2) when a < b, so that
// <phi(x), phi(y)> = (x.y)^2.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kata {

constexpr float kSqrt2 = 1.41421356237309515f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__host__ __device__ __forceinline__ int packed_dim(int d) { return d * (d + 1) / 2; }
__host__ __device__ __forceinline__ int packed_row_base(int a, int d) {
    return a * d - a * (a - 1) / 2;
}

// Packed row r -> (a << 8) | b. One pass over a by the calling threads.
__device__ __forceinline__ void build_pair_table(uint16_t *tab, int d) {
    for (int a = threadIdx.x; a < d; a += blockDim.x) {
        const int base = packed_row_base(a, d);
        for (int b = a; b < d; ++b) tab[base + b - a] = (uint16_t)((a << 8) | b);
    }
}

// phi entry for pair `ab` of the fp32 vector x.
__device__ __forceinline__ float phi_entry(const float *x, uint16_t ab) {
    const int a = ab >> 8, b = ab & 255;
    const float p = x[a] * x[b];
    return a == b ? p : p * kSqrt2;
}

// Device-side error codes written to the per-device error word.
enum : unsigned int { kErrNone = 0, kErrTimeout = 1 };

}  // namespace kata
