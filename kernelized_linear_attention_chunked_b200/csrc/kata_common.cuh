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

// Multi-factor features ("Kernelized Linear Attention", s2.3 "Variants":
// KATA-Mg, several PSD factors; KATA-Sigma-g, summed PSD factors). The head
// vector x is cut into g sub-vectors x_r of p = d/g values, each giving the
// rank-one factor x_r x_r^T; Mg keeps the factors apart (g packed p x p
// triangles one after another, kernel sum_r (q_r.k_r)^2), Sigma-g sums them
// into one p x p matrix (kernel sum_{r,t} (q_r.k_t)^2). kFeatRank1 is the
// single factor of s2.2.
enum : int { kFeatRank1 = 0, kFeatMg = 1, kFeatSigmaG = 2 };

__host__ __device__ __forceinline__ int feature_dim(int d, int feature, int g) {
    const int p = d / g;
    return feature == kFeatRank1 ? packed_dim(d)
                                 : (feature == kFeatMg ? g * packed_dim(p) : packed_dim(p));
}

// Pair (a, b), a <= b < p, of packed row r of a p x p triangle.
__device__ __forceinline__ void unpack_pair(int r, int p, int &a, int &b) {
    a = 0;
    while (packed_row_base(a + 1, p) <= r) ++a;
    b = a + r - packed_row_base(a, p);
}

// Feature row r of x for Mg / Sigma-g (p = d / g), with sqrt(2) off the diagonal.
template <int FK>
__device__ __forceinline__ float factor_feature(const float *x, int r, int g, int p) {
    const int Dp = packed_dim(p);
    int a, b;
    if (FK == kFeatMg) {
        const int f = r / Dp;
        unpack_pair(r - f * Dp, p, a, b);
        const float v = x[f * p + a] * x[f * p + b];
        return a == b ? v : v * kSqrt2;
    }
    unpack_pair(r, p, a, b);
    float v = 0.f;
    for (int t = 0; t < g; ++t) v = fmaf(x[t * p + a], x[t * p + b], v);
    return a == b ? v : v * kSqrt2;
}

// kappa(q, k) = <psi(q), psi(k)> from the sub-vectors' dot products.
template <int FK>
__device__ __forceinline__ float factor_kernel(const float *q, const float *k, int d, int g) {
    if (FK == kFeatRank1) {
        float dot = 0.f;
        for (int a = 0; a < d; ++a) dot = fmaf(q[a], k[a], dot);
        return dot * dot;
    }
    const int p = d / g;
    float sum = 0.f;
    for (int r = 0; r < g; ++r)
        for (int t = 0; t < g; ++t) {
            if (FK == kFeatMg && t != r) continue;
            float dot = 0.f;
            for (int a = 0; a < p; ++a) dot = fmaf(q[r * p + a], k[t * p + a], dot);
            sum = fmaf(dot, dot, sum);
        }
    return sum;
}

// Device-side error codes written to the per-device error word. Codes
// kErrBoundsFirst .. kErrBoundsLast are bounds-check sites of the debug build.
enum : unsigned int { kErrNone = 0, kErrTimeout = 1, kErrBoundsFirst = 0xB000, kErrBoundsLast = 0xBFFF };

}  // namespace kata

// ------------------------------------------------------------ debug build --
// Bounds checks of the debug library (compiled with -DKATA_DEBUG): a check
// that fails records its site code (0xB000 and up) in the device error word,
// which kata_sync_status reports as KATA_ERR_BOUNDS, and the caller skips the
// access instead of faulting. In the normal library KATA_CHECK is the
// constant true and costs nothing. Each translation unit holds its own copy of
// the pointer to the word; KATA_DEBUG_BIND() (in its launchers, after
// kata_internal.h) points it at this device's word.
#ifdef KATA_DEBUG
static __constant__ unsigned int *kata_dbg_word;
__device__ __forceinline__ bool kata_dbg_check(bool ok, unsigned int code) {
    if (!ok && kata_dbg_word) atomicCAS(kata_dbg_word, 0u, code);
    return ok;
}
#define KATA_CHECK(cond, code) kata_dbg_check((cond), (code))
#define KATA_DEBUG_BIND()                                                     \
    do {                                                                      \
        unsigned int *kata_dbg_p = ::kata::device_error_word();               \
        cudaMemcpyToSymbol(kata_dbg_word, &kata_dbg_p, sizeof(kata_dbg_p));   \
    } while (0)
#else
#define KATA_CHECK(cond, code) true
#define KATA_DEBUG_BIND() \
    do {                  \
    } while (0)
#endif
