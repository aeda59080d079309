// One decode step of causal kernelized linear attention, HBM-bandwidth bound.
//
// "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
// Cones", s1 (constant-time recurrent inference with a fixed-size state) and
// s2.2 (phi(x) = x x^T):
//   H += phi(k) v^T;  s += phi(k);  o = phi(q)^T H / (phi(q)^T s + eps)
// with the update applied before the readout.
//
// One CTA per (b, h) streams that head's packed fp32 state exactly once:
// every H row (d floats) is read with 128-bit loads, updated, written back
// with 128-bit stores (both with the streaming cache hint, the state is not
// reused by this launch), and folded into the readout while still in
// registers. The readout is reduced with warp shuffles and one shared-memory
// pass. phi(q) and phi(k) are built once per CTA in shared memory.
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

constexpr int kThreads = 256;

template <typename Tin, int DH>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              float eps, float *__restrict__ Hst, float *__restrict__ s,
              float *__restrict__ o) {
    constexpr int D = DH * (DH + 1) / 2;
    constexpr int CG = DH / 4;           // float4 groups per row
    constexpr int RPP = kThreads / CG;   // rows per pass
    constexpr int NW = kThreads / 32;
    __shared__ float pq[D], pk[D];
    __shared__ float xs[3][DH];
    __shared__ float4 red[NW][CG];
    __shared__ float zred[NW];

    const int bh = blockIdx.x, tid = threadIdx.x;
    if (tid < DH) {
        xs[0][tid] = to_f32(q[(size_t)bh * DH + tid]);
        xs[1][tid] = to_f32(k[(size_t)bh * DH + tid]);
        xs[2][tid] = to_f32(v[(size_t)bh * DH + tid]);
    }
    __syncthreads();
    for (int a = tid; a < DH; a += kThreads) {  // one thread per triangle row
        const int base = packed_row_base(a, DH);
        const float qa = xs[0][a], ka = xs[1][a];
        for (int b = a; b < DH; ++b) {
            const float w = (a == b) ? 1.f : kSqrt2;
            pq[base + b - a] = (qa * xs[0][b]) * w;
            pk[base + b - a] = (ka * xs[1][b]) * w;
        }
    }
    __syncthreads();

    const int cg = tid % CG, rsub = tid / CG;
    const float4 vv = reinterpret_cast<const float4 *>(xs[2])[cg];
    float4 *H4 = reinterpret_cast<float4 *>(Hst + (size_t)bh * D * DH);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int r = rsub; r < D; r += RPP) {
        float4 h = __ldcs(H4 + (size_t)r * CG + cg);
        const float kk = pk[r], qq = pq[r];
        h.x = fmaf(kk, vv.x, h.x);
        h.y = fmaf(kk, vv.y, h.y);
        h.z = fmaf(kk, vv.z, h.z);
        h.w = fmaf(kk, vv.w, h.w);
        __stcs(H4 + (size_t)r * CG + cg, h);
        acc.x = fmaf(qq, h.x, acc.x);
        acc.y = fmaf(qq, h.y, acc.y);
        acc.z = fmaf(qq, h.z, acc.z);
        acc.w = fmaf(qq, h.w, acc.w);
    }
    float4 *s4 = reinterpret_cast<float4 *>(s + (size_t)bh * D);
    float z = 0.f;
    for (int r4 = tid; r4 < D / 4; r4 += kThreads) {
        float4 sv = __ldcs(s4 + r4);
        const int r = r4 * 4;
        sv.x += pk[r];
        sv.y += pk[r + 1];
        sv.z += pk[r + 2];
        sv.w += pk[r + 3];
        __stcs(s4 + r4, sv);
        z = fmaf(pq[r], sv.x, z);
        z = fmaf(pq[r + 1], sv.y, z);
        z = fmaf(pq[r + 2], sv.z, z);
        z = fmaf(pq[r + 3], sv.w, z);
    }
    // lanes with equal cg hold partial sums of the same 4 outputs
#pragma unroll
    for (int off = CG; off < 32; off <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    const int warp = tid / 32, lane = tid % 32;
    if (lane < CG) red[warp][lane] = acc;
    if (lane == 0) zred[warp] = z;
    __syncthreads();
    if (tid < DH) {
        float zt = 0.f, num = 0.f;
        for (int w = 0; w < NW; ++w) {
            zt += zred[w];
            const float4 p = red[w][tid / 4];
            const int c = tid % 4;
            num += c == 0 ? p.x : c == 1 ? p.y : c == 2 ? p.z : p.w;
        }
        o[(size_t)bh * DH + tid] = num / (zt + eps);
    }
}

template <typename Tin>
cudaError_t launch(const void *q, const void *k, const void *v, int B, int H, int d, float eps,
                   float *Hst, float *s, float *o, cudaStream_t stream) {
    dim3 grid(B * H);
    const Tin *qq = static_cast<const Tin *>(q), *kk = static_cast<const Tin *>(k),
              *vv = static_cast<const Tin *>(v);
    switch (d) {
        case 16: decode_kernel<Tin, 16><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o); break;
        case 32: decode_kernel<Tin, 32><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o); break;
        case 64: decode_kernel<Tin, 64><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o); break;
        default: return cudaErrorInvalidValue;
    }
    return after_launch();
}

}  // namespace

cudaError_t decode_step(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int d, float eps, float *Hst, float *s, float *o, cudaStream_t stream) {
    return dtype == 0 ? launch<float>(q, k, v, B, H, d, eps, Hst, s, o, stream)
                      : launch<__nv_bfloat16>(q, k, v, B, H, d, eps, Hst, s, o, stream);
}

}  // namespace kata
