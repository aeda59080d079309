// One decode step of causal kernelized linear attention, HBM-bandwidth bound.
//
// "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
// Cones", s1 (constant-time recurrent inference with a fixed-size state) and
// s2.2 (phi(x) = x x^T):
//   H += phi(k) v^T;  s += phi(k);  o = phi(q)^T H / (phi(q)^T s + eps)
// with the update applied before the readout.
//
// A cluster of two CTAs per (b, h) streams that head's packed fp32 state
// exactly once: the CTAs take alternate blocks of rows (4 KB apart at d = 64,
// which keeps twice as many independent streams in flight as one CTA per head
// and measured 7 % more DRAM throughput for this read-modify-write pattern);
// every H row (d floats) is read with 128-bit loads, updated, written back
// with 128-bit stores (both with the streaming cache hint, the state is not
// reused by this launch), and folded into the readout while still in
// registers. The readout is reduced with warp shuffles and one shared-memory
// pass per CTA; the second CTA then adds its partial numerators and
// denominator into the first one's shared memory (distributed shared memory)
// and the first writes o. phi(q) and phi(k) are built by all threads of each
// CTA in shared memory.
//
// The multi-factor features of s2.3 "Variants" (KATA-Mg, KATA-Sigma-g;
// kata_common.cuh) run through the same kernel with their own feature rows
// (the state has D_f = feature_dim rows instead of D).
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Split cluster barrier, first half: this CTA is running (no memory ordering).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
// Second half: every CTA of the cluster has arrived, so every CTA has started
// and its shared memory may be written through distributed shared memory.
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// All threads of every CTA of the cluster: release this CTA's shared-memory
// writes, acquire the others'.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store v to the same shared-memory variable in CTA `cta` of the cluster.
__device__ __forceinline__ void st_cluster(float *local, uint32_t cta, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(ra)
                 : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(cta));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <typename Tin, int DH, int FK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              float eps, float *__restrict__ Hst, float *__restrict__ s,
              float *__restrict__ o, int g) {
    constexpr int DM = DH * (DH + 1) / 2;  // the largest feature dimension (one factor)
    const int D = FK == kFeatRank1 ? DM : feature_dim(DH, FK, g);
    constexpr int CG = DH / 4;           // float4 groups per row
    constexpr int RPP = kThreads / CG;   // rows per pass
    constexpr int NW = kThreads / 32;
    __shared__ float pq[DM], pk[DM];
    __shared__ float xs[3][DH];
    __shared__ float4 red[NW][CG];
    __shared__ float zred[NW];
    __shared__ float xnum[DH], xz;  // the second CTA's partial readout

    const int bh = blockIdx.x / 2, tid = threadIdx.x;
    const uint32_t cr = cluster_ctarank();  // 0 or 1: which row blocks this CTA takes
    if (tid < DH) {
        xs[0][tid] = to_f32(q[(size_t)bh * DH + tid]);
        xs[1][tid] = to_f32(k[(size_t)bh * DH + tid]);
        xs[2][tid] = to_f32(v[(size_t)bh * DH + tid]);
    }
    __syncthreads();
    if (FK == kFeatRank1) {
        for (int idx = tid; idx < DH * DH; idx += kThreads) {  // entry (a, b) of x x^T, b >= a
            const int a = idx / DH, b = idx % DH;
            if (b < a) continue;
            const int at = packed_row_base(a, DH) + b - a;
            const float w = (a == b) ? 1.f : kSqrt2;
            pq[at] = (xs[0][a] * xs[0][b]) * w;
            pk[at] = (xs[1][a] * xs[1][b]) * w;
        }
    } else {
        for (int r = tid; r < D; r += kThreads) {
            pq[r] = factor_feature<FK>(xs[0], r, g, DH / g);
            pk[r] = factor_feature<FK>(xs[1], r, g, DH / g);
        }
    }
    __syncthreads();
    // announce that this CTA runs; the partner waits for it before writing into
    // this CTA's shared memory (the wait comes after the streaming loop, so the
    // barrier costs nothing on the loop)
    cluster_arrive_relaxed();

    const int cg = tid % CG, rsub = tid / CG;
    const float4 vv = reinterpret_cast<const float4 *>(xs[2])[cg];
    float4 *H4 = reinterpret_cast<float4 *>(Hst + (size_t)bh * D * DH);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int r = rsub + RPP * (int)cr; r < D; r += 2 * RPP) {
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
    for (int r4 = tid + kThreads * (int)cr; r4 < D / 4; r4 += 2 * kThreads) {
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
    cluster_wait();  // both CTAs of the cluster have started
    float zt = 0.f, num = 0.f;
    if (tid < DH) {
        for (int w = 0; w < NW; ++w) {
            zt += zred[w];
            const float4 p = red[w][tid / 4];
            const int c = tid % 4;
            num += c == 0 ? p.x : c == 1 ? p.y : c == 2 ? p.z : p.w;
        }
        if (cr == 1) {
            st_cluster(&xnum[tid], 0, num);
            if (tid == 0) st_cluster(&xz, 0, zt);
        }
    }
    cluster_sync();
    if (cr == 0 && tid < DH) o[(size_t)bh * DH + tid] = (num + xnum[tid]) / (zt + xz + eps);
}

template <typename Tin, int FK>
cudaError_t launch(const void *q, const void *k, const void *v, int B, int H, int d, float eps,
                   float *Hst, float *s, float *o, int g, cudaStream_t stream) {
    dim3 grid(2 * B * H);  // clusters of two CTAs per head
    const Tin *qq = static_cast<const Tin *>(q), *kk = static_cast<const Tin *>(k),
              *vv = static_cast<const Tin *>(v);
    switch (d) {
        case 16: decode_kernel<Tin, 16, FK><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o, g); break;
        case 32: decode_kernel<Tin, 32, FK><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o, g); break;
        case 64: decode_kernel<Tin, 64, FK><<<grid, kThreads, 0, stream>>>(qq, kk, vv, eps, Hst, s, o, g); break;
        default: return cudaErrorInvalidValue;
    }
    return after_launch();
}

template <typename Tin>
cudaError_t launch_feature(const void *q, const void *k, const void *v, int B, int H, int d,
                           float eps, float *Hst, float *s, float *o, int feature, int g,
                           cudaStream_t stream) {
    switch (feature) {
        case kFeatRank1: return launch<Tin, kFeatRank1>(q, k, v, B, H, d, eps, Hst, s, o, 1, stream);
        case kFeatMg: return launch<Tin, kFeatMg>(q, k, v, B, H, d, eps, Hst, s, o, g, stream);
        case kFeatSigmaG: return launch<Tin, kFeatSigmaG>(q, k, v, B, H, d, eps, Hst, s, o, g, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t decode_step(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int d, float eps, float *Hst, float *s, float *o, cudaStream_t stream,
                        int feature, int g) {
    return dtype == 0
               ? launch_feature<float>(q, k, v, B, H, d, eps, Hst, s, o, feature, g, stream)
               : launch_feature<__nv_bfloat16>(q, k, v, B, H, d, eps, Hst, s, o, feature, g,
                                               stream);
}

}  // namespace kata
