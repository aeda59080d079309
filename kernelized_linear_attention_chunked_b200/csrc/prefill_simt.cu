// Causal chunked prefill on the CUDA cores, fp32 arithmetic.
//
// "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
// Cones", s2.3 (chunked parallelism) with the feature of s2.2: for chunk c,
//   o_i = [ sum_{j<=i in c} (q_i.k_j)^2 v_j + phi(q_i)^T H_{c-1} ]
//       / [ sum_{j<=i in c} (q_i.k_j)^2     + phi(q_i)^T s_{c-1} + eps ]
//   H_c = H_{c-1} + phi(K_c)^T V_c,   s_c = s_{c-1} + phi(K_c)^T 1.
//
// This is the accuracy path (fp32 inputs) and the path for shapes the tensor
// core kernel does not take. One CTA owns one head and a 16-column slice of
// the value dimension; its slice of the state (D x 16 fp32) and the whole
// normaliser s (D fp32) stay in shared memory for the whole sequence, so the
// carry across chunks never leaves the SM. Every CTA of a head keeps an
// identical copy of s (same operations in the same order).
//
// The same kernel runs the multi-factor features of s2.3 "Variants" (KATA-Mg,
// KATA-Sigma-g; kata_common.cuh): only the feature rows and the intra-chunk
// kernel change.
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

constexpr int kThreads = 256;
constexpr int kE = 16;   // value columns per CTA
constexpr int kRT = 16;  // packed rows per phi tile
constexpr int kRTP = kRT + 1;
constexpr int kCS = 64;  // tokens per inner chunk

size_t simt_smem_bytes(int d, int D) {
    const size_t floats = (size_t)D * kE + D + 2 * (size_t)kCS * (d + 1) + (size_t)kCS * kE +
                          2 * (size_t)kCS * kRTP;
    return floats * sizeof(float) + ((size_t)D * sizeof(uint16_t) + 15) / 16 * 16;
}

template <typename Tin, int FK>
__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const Tin *__restrict__ v, int T, int d, int cs, float eps,
                    const float *__restrict__ H_in, const float *__restrict__ s_in,
                    float *__restrict__ o, float *__restrict__ H_out,
                    float *__restrict__ s_out, int g) {
    const int D = feature_dim(d, FK, g);
    const int fp = d / g;  // values per factor
    const int NE = d / kE;
    const int bh = blockIdx.x / NE;
    const int e0 = (blockIdx.x % NE) * kE;
    const int dp = d + 1;
    const int tid = threadIdx.x;

    extern __shared__ float4 smem4[];
    float *Hs = reinterpret_cast<float *>(smem4);  // [D][kE]
    float *sv = Hs + (size_t)D * kE;               // [D]
    float *Qs = sv + D;                            // [kCS][d+1]
    float *Ks = Qs + kCS * dp;                     // [kCS][d+1]
    float *Vs = Ks + kCS * dp;                     // [kCS][kE]
    float *PQ = Vs + kCS * kE;                     // [kCS][kRTP]
    float *PK = PQ + kCS * kRTP;                   // [kCS][kRTP]
    uint16_t *tab = reinterpret_cast<uint16_t *>(PK + kCS * kRTP);

    if (FK == kFeatRank1) build_pair_table(tab, d);
    const size_t hoff = (size_t)bh * D * d;
    for (int idx = tid; idx < D * kE; idx += kThreads) {
        const int r = idx / kE, e = idx % kE;
        Hs[idx] = H_in ? H_in[hoff + (size_t)r * d + e0 + e] : 0.f;
    }
    for (int r = tid; r < D; r += kThreads) sv[r] = s_in ? s_in[(size_t)bh * D + r] : 0.f;

    const int row = tid >> 2;       // query row inside the chunk
    const int eq = (tid & 3) * 4;   // 4 value columns of the slice
    const size_t xoff = (size_t)bh * T * d;

    for (int t0 = 0; t0 < T; t0 += cs) {
        __syncthreads();
        for (int idx = tid; idx < cs * d; idx += kThreads) {
            const int i = idx / d, a = idx % d;
            Qs[i * dp + a] = to_f32(q[xoff + (size_t)(t0 + i) * d + a]);
            Ks[i * dp + a] = to_f32(k[xoff + (size_t)(t0 + i) * d + a]);
        }
        for (int idx = tid; idx < cs * kE; idx += kThreads) {
            const int i = idx / kE, e = idx % kE;
            Vs[idx] = to_f32(v[xoff + (size_t)(t0 + i) * d + e0 + e]);
        }
        __syncthreads();

        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, z = 0.f;
        if (row < cs) {  // intra-chunk masked (q.k)^2 contraction
            const float *qi = Qs + row * dp;
            for (int j = 0; j <= row; ++j) {
                const float w = factor_kernel<FK>(qi, Ks + j * dp, d, g);
                z += w;
                const float *vj = Vs + j * kE + eq;
                acc0 = fmaf(w, vj[0], acc0);
                acc1 = fmaf(w, vj[1], acc1);
                acc2 = fmaf(w, vj[2], acc2);
                acc3 = fmaf(w, vj[3], acc3);
            }
        }
        for (int r0 = 0; r0 < D; r0 += kRT) {
            for (int idx = tid; idx < cs * kRT; idx += kThreads) {
                const int i = idx / kRT, rr = idx % kRT, r = r0 + rr;
                float pq = 0.f, pk = 0.f;
                if (r < D) {
                    if (FK == kFeatRank1) {
                        pq = phi_entry(Qs + i * dp, tab[r]);
                        pk = phi_entry(Ks + i * dp, tab[r]);
                    } else {
                        pq = factor_feature<FK>(Qs + i * dp, r, g, fp);
                        pk = factor_feature<FK>(Ks + i * dp, r, g, fp);
                    }
                }
                PQ[i * kRTP + rr] = pq;
                PK[i * kRTP + rr] = pk;
            }
            __syncthreads();
            if (row < cs) {  // inter-chunk readout against the previous state
                const int rmax = min(kRT, D - r0);
                for (int rr = 0; rr < rmax; ++rr) {
                    const float p = PQ[row * kRTP + rr];
                    const float *hr = Hs + (size_t)(r0 + rr) * kE + eq;
                    z = fmaf(p, sv[r0 + rr], z);
                    acc0 = fmaf(p, hr[0], acc0);
                    acc1 = fmaf(p, hr[1], acc1);
                    acc2 = fmaf(p, hr[2], acc2);
                    acc3 = fmaf(p, hr[3], acc3);
                }
            }
            __syncthreads();
            {  // state update with this chunk's keys and values
                const int rr = tid >> 4, e = tid & 15, r = r0 + rr;
                if (r < D) {
                    float hsum = 0.f, ssum = 0.f;
                    for (int i = 0; i < cs; ++i) {
                        const float p = PK[i * kRTP + rr];
                        hsum = fmaf(p, Vs[i * kE + e], hsum);
                        ssum += p;
                    }
                    Hs[(size_t)r * kE + e] += hsum;
                    if (e == 0) sv[r] += ssum;
                }
            }
            __syncthreads();
        }
        if (o && row < cs && KATA_CHECK(t0 + row < T, 0xB101u)) {
            const float inv = 1.f / (z + eps);
            float *orow = o + xoff + (size_t)(t0 + row) * d + e0 + eq;
            orow[0] = acc0 * inv;
            orow[1] = acc1 * inv;
            orow[2] = acc2 * inv;
            orow[3] = acc3 * inv;
        }
    }
    __syncthreads();
    if (H_out) {
        for (int idx = tid; idx < D * kE; idx += kThreads) {
            const int r = idx / kE, e = idx % kE;
            H_out[hoff + (size_t)r * d + e0 + e] = Hs[idx];
        }
    }
    if (s_out && e0 == 0)
        for (int r = tid; r < D; r += kThreads) s_out[(size_t)bh * D + r] = sv[r];
}

template <typename Tin, int FK>
cudaError_t launch_simt(const PrefillArgs &a, cudaStream_t stream) {
    const size_t smem = simt_smem_bytes(a.d, feature_dim(a.d, FK, a.g));
    cudaError_t err = cudaFuncSetAttribute(prefill_simt_kernel<Tin, FK>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const int cs = a.chunk < kCS ? a.chunk : kCS;
    dim3 grid(a.B * a.H * (a.d / kE));
    prefill_simt_kernel<Tin, FK><<<grid, kThreads, smem, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
        static_cast<const Tin *>(a.v), a.T, a.d, cs, a.eps, a.H_in, a.s_in, a.o, a.H_out,
        a.s_out, a.g);
    return after_launch();
}

template <typename Tin>
cudaError_t launch_feature(const PrefillArgs &a, cudaStream_t stream) {
    switch (a.feature) {
        case kFeatRank1: return launch_simt<Tin, kFeatRank1>(a, stream);
        case kFeatMg: return launch_simt<Tin, kFeatMg>(a, stream);
        case kFeatSigmaG: return launch_simt<Tin, kFeatSigmaG>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t prefill_simt(const PrefillArgs &a, cudaStream_t stream) {
    KATA_DEBUG_BIND();
    return a.dtype == 0 ? launch_feature<float>(a, stream)
                        : launch_feature<__nv_bfloat16>(a, stream);
}

}  // namespace kata
