// LoLA sparse-cache pieces on the CUDA cores, fp32 arithmetic.
//
// "LoLA: Low-Rank Linear Attention with Sparse Caching":
//  - "Self-Recall Error": SRE(k, v | H, s) = || phi(k)^T H / phi(k)^T s - v ||^2
//    (eps added to the denominator, as in every readout here);
//  - "Inference strategy" 1-3: score the pairs leaving the window together
//    with the cached pairs, keep the highest SRE in the cache, merge the rest
//    into the linear state by outer-product updates;
//  - "Inference strategy" 4 / Methodology 1-3: the output combines window
//    softmax attention, sparse-cache attention and the linear-state readout.
// phi is the rank-one PSD feature of "Kernelized Linear Attention: Breaking
// the Capacity Wall with Symmetric Cones", s2.2.
//
// Kernels:
//  state_partial  phi(x_i)^T [H | s] for many rows x_i, split over slices of
//                 the packed dimension (one CTA per head x slice x 64 rows);
//                 partial sums go to the workspace and are reduced in a fixed
//                 order by the consumer, so results are run-to-run identical.
//  sre_select     reduce partials, SRE per candidate, rank-based top-k (every
//                 thread counts the candidates ranked before it), kept slots
//                 in ascending position, list of slots to merge.
//  merge          H_dst = H_src + sum_{j merged} phi(k_j) v_j^T per slice.
//  hybrid_finish  window + cache softmax terms, plus the state partials, one
//                 shared denominator.
//  append/compact the cache bookkeeping of the schedule.
#include <mutex>

#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;
constexpr int kMaxSlice = 512;
constexpr int kTargetCtas = 296;  // two CTAs per SM on a 148-SM part

int num_slices(int nh, int n, int d) {
    const int D = packed_dim(d);
    const int rb = (n + kRows - 1) / kRows;
    const int pmin = (D + kMaxSlice - 1) / kMaxSlice;
    const int pmax = (D + 63) / 64;
    int p = (kTargetCtas + nh * rb - 1) / (nh * rb);
    if (p < pmin) p = pmin;
    if (p > pmax) p = pmax;
    return p;
}

size_t partial_floats(int nh, int n, int d) {
    return (size_t)num_slices(nh, n, d) * nh * n * (d + 1);
}

// Register-blocked scoring: each thread owns kCB candidates x kEB output
// columns; the state slice streams through shared memory kRC rows at a time
// and phi of those rows is built once per chunk for all the CTA's candidates.
// Asynchronous global -> shared copies (16 or 4 bytes), grouped per commit.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

constexpr int kRC = 32;  // state rows per chunk
constexpr int kCB = 4;   // candidates per thread
constexpr int kEB = 16;  // output columns per thread

// candidates one CTA scores in one pass over its slice
int partial_pass(int d, int n, int zsplit) {
    const int neb = d / kEB;
    const int cap = kThreads / neb * kCB;
    const int per = (n + zsplit - 1) / zsplit;
    const int p4 = (per + kCB - 1) / kCB * kCB;
    return p4 < cap ? p4 : cap;
}

size_t state_partial_smem(int d, int pass) {
    const int D = packed_dim(d);
    // candidates, phi of a chunk, two state chunks (H rows and s)
    return ((size_t)pass * (d + 1) + (size_t)kRC * pass + 2 * ((size_t)kRC * d + kRC)) *
               sizeof(float) +
           align_up((size_t)D * sizeof(uint16_t), 16);
}

// part[p][h][i][e] = sum_{r in slice p} phi(x_i)_r H[r][e]; part[..][d] uses s.
// CTA (h, p, z) scores candidates [z * per, (z + 1) * per) against slice p of
// head h's state, `pass` candidates at a time; with many heads the launch uses
// z = 1, so every slice of the state is read once.
template <typename Tin, int DH>
__global__ void __launch_bounds__(kThreads)
state_partial_kernel(const Tin *__restrict__ X, long x_head_stride, int n,
                     const float *__restrict__ Hst, const float *__restrict__ s, int P,
                     int pass, float *__restrict__ part) {
    constexpr int D = DH * (DH + 1) / 2;
    constexpr int NEB = DH / kEB;  // column blocks
    const int h = blockIdx.x, p = blockIdx.y, nh = gridDim.x;
    const int slice = (D + P - 1) / P;
    const int r0 = p * slice, r1 = min(D, r0 + slice);
    const int per = (n + gridDim.z - 1) / gridDim.z;
    const int c0 = blockIdx.z * per, c1 = min(n, c0 + per);
    const int tid = threadIdx.x;
    const int ej = tid % NEB, cg = tid / NEB;  // column block, candidate group

    extern __shared__ float4 smem4[];
    float *Xs = reinterpret_cast<float *>(smem4);  // [pass][DH+1]
    float *Ph = Xs + (size_t)pass * (DH + 1);       // [kRC][pass]
    float *Hc = Ph + (size_t)kRC * pass;            // [2][kRC][DH]: chunk k in buffer k % 2
    float *sc = Hc + 2 * kRC * DH;                  // [2][kRC]
    uint16_t *tab = reinterpret_cast<uint16_t *>(sc + 2 * kRC);

    build_pair_table(tab, DH);
    const Tin *Xh = X + (size_t)h * x_head_stride;
    const float *Hh = Hst + (size_t)h * D * DH;
    const float *sh = s + (size_t)h * D;
    const bool active = cg * kCB < pass;

    for (int pc0 = c0; pc0 < c1; pc0 += pass) {
        const int pn = min(pass, c1 - pc0);
        __syncthreads();  // the previous pass is done with Xs
        for (int idx = tid; idx < pass * DH; idx += kThreads) {
            const int i = idx / DH, a = idx % DH;
            Xs[i * (DH + 1) + a] = i < pn ? to_f32(Xh[(size_t)(pc0 + i) * DH + a]) : 0.f;
        }
        float acc[kCB][kEB];
        float den[kCB];
#pragma unroll
        for (int c = 0; c < kCB; ++c) {
            den[c] = 0.f;
#pragma unroll
            for (int e = 0; e < kEB; ++e) acc[c][e] = 0.f;
        }
        // the slice streams through two shared-memory chunk buffers: the copy
        // of chunk k + 1 is in flight while chunk k's phi is built and used
        const int nchunk = (r1 - r0 + kRC - 1) / kRC;
        auto issue = [&](int k) {
            const int rc = r0 + k * kRC, nr = min(kRC, r1 - rc);
            float *hb = Hc + (k & 1) * kRC * DH;
            float *sb = sc + (k & 1) * kRC;
            for (int idx = tid; idx < nr * DH / 4; idx += kThreads)
                cp_async16(hb + 4 * idx, Hh + (size_t)rc * DH + 4 * idx);
            for (int idx = tid; idx < nr; idx += kThreads) cp_async4(sb + idx, sh + rc + idx);
            cp_async_commit();
        };
        if (nchunk > 0) issue(0);
        for (int k = 0; k < nchunk; ++k) {
            const int rc = r0 + k * kRC, nr = min(kRC, r1 - rc);
            const float *hb = Hc + (k & 1) * kRC * DH;
            const float *sb = sc + (k & 1) * kRC;
            cp_async_wait_all();  // this thread's copies of chunk k have landed
            // every copy of chunk k is visible; every thread is done with chunk
            // k - 1 (its buffer and Ph), and Xs is written
            __syncthreads();
            if (k + 1 < nchunk) issue(k + 1);
            for (int idx = tid; idx < nr * pass; idx += kThreads) {
                const int rr = idx / pass, i = idx % pass;
                Ph[rr * pass + i] = phi_entry(Xs + i * (DH + 1), tab[rc + rr]);
            }
            __syncthreads();
            if (active) {
                for (int rr = 0; rr < nr; ++rr) {
                    const float4 ph = *reinterpret_cast<const float4 *>(Ph + rr * pass + cg * kCB);
                    const float pv[kCB] = {ph.x, ph.y, ph.z, ph.w};
                    // columns 4 (q NEB + ej) .. +3: neighbouring threads read
                    // neighbouring 16-byte chunks (no bank conflicts)
                    const float4 *hv = reinterpret_cast<const float4 *>(hb + rr * DH);
#pragma unroll
                    for (int q = 0; q < kEB / 4; ++q) {
                        const float4 hq = hv[q * NEB + ej];
#pragma unroll
                        for (int c = 0; c < kCB; ++c) {
                            acc[c][4 * q + 0] = fmaf(pv[c], hq.x, acc[c][4 * q + 0]);
                            acc[c][4 * q + 1] = fmaf(pv[c], hq.y, acc[c][4 * q + 1]);
                            acc[c][4 * q + 2] = fmaf(pv[c], hq.z, acc[c][4 * q + 2]);
                            acc[c][4 * q + 3] = fmaf(pv[c], hq.w, acc[c][4 * q + 3]);
                        }
                    }
                    if (ej == 0) {
                        const float sr = sb[rr];
#pragma unroll
                        for (int c = 0; c < kCB; ++c) den[c] = fmaf(pv[c], sr, den[c]);
                    }
                }
            }
        }
        if (active) {
#pragma unroll
            for (int c = 0; c < kCB; ++c) {
                const int i = pc0 + cg * kCB + c;
                if (i < c1) {
                    float *dst = part + (((size_t)p * nh + h) * n + i) * (DH + 1);
#pragma unroll
                    for (int q = 0; q < kEB / 4; ++q)
#pragma unroll
                        for (int k = 0; k < 4; ++k) dst[4 * (q * NEB + ej) + k] = acc[c][4 * q + k];
                    if (ej == 0) dst[DH] = den[c];
                }
            }
        }
    }
}

template <typename Tin>
cudaError_t launch_state_partial(const Tin *X, long x_head_stride, int nh, int n, int d,
                                 const float *Hst, const float *s, int P, float *part,
                                 cudaStream_t stream) {
    // enough (head, slice) CTAs to fill the GPU twice over: one CTA per slice
    // reads it once; otherwise split the candidates too
    const int rb = (n + kRows - 1) / kRows;
    const int zsplit = nh * P >= 2 * kTargetCtas ? 1 : rb;
    const int pass = partial_pass(d, n, zsplit);
    const size_t smem = state_partial_smem(d, pass);
    dim3 grid(nh, P, zsplit);
    cudaError_t err;
#define KATA_LAUNCH_PARTIAL(DH)                                                               \
    err = cudaFuncSetAttribute(state_partial_kernel<Tin, DH>,                                 \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);      \
    if (err != cudaSuccess) return err;                                                       \
    state_partial_kernel<Tin, DH><<<grid, kThreads, smem, stream>>>(X, x_head_stride, n, Hst, \
                                                                     s, P, pass, part);
    switch (d) {
        case 16: KATA_LAUNCH_PARTIAL(16) break;
        case 32: KATA_LAUNCH_PARTIAL(32) break;
        case 64: KATA_LAUNCH_PARTIAL(64) break;
        default: return cudaErrorInvalidValue;
    }
#undef KATA_LAUNCH_PARTIAL
    return after_launch();
}

// Candidate i is retained before candidate j: higher SRE, then smaller
// position, then smaller slot.
__device__ __forceinline__ bool retained_before(float si, int pi, int i, float sj, int pj,
                                                int j) {
    if (si != sj) return si > sj;
    if (pi != pj) return pi < pj;
    return i < j;
}

template <typename Tin>
__global__ void __launch_bounds__(1024)
sre_select_kernel(const float *__restrict__ part, int P, int n, int d,
                  const Tin *__restrict__ vc, long cand_head_stride,
                  const int *__restrict__ pos, long pos_head_stride, int keep, float eps,
                  float *__restrict__ scores, int *__restrict__ keep_idx,
                  int *__restrict__ mlist, int *__restrict__ mcount) {
    __shared__ float sc[1024];
    __shared__ int ps[1024];
    __shared__ unsigned char kept[1024];
    const int h = blockIdx.x, nh = gridDim.x, j = threadIdx.x;
    const int m = keep < n ? keep : n;
    // SRE of every candidate: one warp per candidate, lanes across the columns
    // of its partial sums (coalesced), summed over the slices in slice order
    {
        const int warp = j >> 5, lane = j & 31, nwarps = blockDim.x >> 5;
        const size_t pstride = (size_t)nh * n * (d + 1);
        for (int c = warp; c < n; c += nwarps) {
            const float *pc = part + ((size_t)h * n + c) * (d + 1);
            float den = 0.f;
            if (lane == 0) {
#pragma unroll 4
                for (int p = 0; p < P; ++p) den += pc[p * pstride + d];
            }
            den = __shfl_sync(0xFFFFFFFFu, den, 0);
            const float inv = 1.f / (den + eps);
            const Tin *vj = vc + (size_t)h * cand_head_stride + (size_t)c * d;
            float err = 0.f;
            for (int e = lane; e < d; e += 32) {
                float num = 0.f;
#pragma unroll 4
                for (int p = 0; p < P; ++p) num += pc[p * pstride + e];
                const float diff = num * inv - to_f32(vj[e]);
                err = fmaf(diff, diff, err);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) err += __shfl_xor_sync(0xFFFFFFFFu, err, o);
            if (lane == 0) {
                sc[c] = isnan(err) ? -INFINITY : err;  // a total order even for 0/0 scores
                ps[c] = pos[(size_t)h * pos_head_stride + c];
            }
        }
    }
    __syncthreads();
    bool isk = false;
    if (j < n) {
        int rank = 0;
        for (int i = 0; i < n; ++i) rank += retained_before(sc[i], ps[i], i, sc[j], ps[j], j);
        isk = rank < m;
        kept[j] = isk;
    }
    __syncthreads();
    if (j < n) {
        if (isk) {
            int pr = 0;
            for (int i = 0; i < n; ++i)
                pr += kept[i] && (ps[i] < ps[j] || (ps[i] == ps[j] && i < j));
            if (pr < m) keep_idx[(size_t)h * m + pr] = j;
        } else {
            int mr = 0;
            for (int i = 0; i < j; ++i) mr += !kept[i];
            if (mr < n - m) mlist[(size_t)h * n + mr] = j;
        }
        if (scores) scores[(size_t)h * n + j] = sc[j];
    }
    if (j == 0) mcount[h] = n - m;
}

// Merge: Hdst[r][e] = Hsrc[r][e] + sum_{c merged} phi(k_c)_r v_c[e], and the
// same for s. CTA (h, 256-row block); thread = 4 rows x 16 columns of the
// block, accumulating over the merged candidates kMC at a time (phi of the
// block's rows built once per chunk in shared memory); the state is read and
// written once with 16-byte accesses. Hdst may alias Hsrc.
constexpr int kMR = 256;  // state rows per CTA
constexpr int kMC = 16;   // merged candidates per shared-memory chunk

template <typename Tin, int DH>
__global__ void __launch_bounds__(kThreads)
merge_kernel(const float *Hsrc, const float *ssrc, float *Hdst, float *sdst,
             const Tin *__restrict__ kc, const Tin *__restrict__ vc, long cand_head_stride,
             const int *__restrict__ mlist, const int *__restrict__ mcount, int n) {
    constexpr int D = DH * (DH + 1) / 2;
    constexpr int NEB = DH / kEB;  // column blocks
    __shared__ float Ks[kMC][DH + 1];
    __shared__ __align__(16) float Vs[kMC][DH];
    __shared__ __align__(16) float Pk[kMC][kMR];
    __shared__ uint16_t tab[D];
    const int h = blockIdx.x, rb0 = blockIdx.y * kMR, tid = threadIdx.x;
    const int m = mcount[h];
    const bool active = tid < (kMR / 4) * NEB;
    const int rg = tid / NEB, ej = tid % NEB;
    build_pair_table(tab, DH);
    const Tin *kh = kc + (size_t)h * cand_head_stride;
    const Tin *vh = vc + (size_t)h * cand_head_stride;
    float acc[4][kEB];
    float sacc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        sacc[r] = 0.f;
#pragma unroll
        for (int e = 0; e < kEB; ++e) acc[r][e] = 0.f;
    }
    for (int mc = 0; mc < m; mc += kMC) {
        const int nb = min(kMC, m - mc);
        __syncthreads();  // the previous chunk's readers are done
        for (int idx = tid; idx < kMC * DH; idx += kThreads) {
            const int ii = idx / DH, a = idx % DH;
            float kx = 0.f, vx = 0.f;
            if (ii < nb) {
                const int j = mlist[(size_t)h * n + mc + ii];
                if (KATA_CHECK(j >= 0 && j < n, 0xB304u)) {
                    kx = to_f32(kh[(size_t)j * DH + a]);
                    vx = to_f32(vh[(size_t)j * DH + a]);
                }
            }
            Ks[ii][a] = kx;
            Vs[ii][a] = vx;
        }
        __syncthreads();
        for (int idx = tid; idx < kMC * kMR; idx += kThreads) {
            const int ii = idx / kMR, rr = idx % kMR;
            Pk[ii][rr] = rb0 + rr < D ? phi_entry(Ks[ii], tab[rb0 + rr]) : 0.f;
        }
        __syncthreads();
        if (active) {
            for (int ii = 0; ii < nb; ++ii) {
                const float4 p4 = *reinterpret_cast<const float4 *>(&Pk[ii][rg * 4]);
                const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
                // columns 4 (q NEB + ej) .. +3 (neighbouring threads, neighbouring chunks)
                const float4 *vv = reinterpret_cast<const float4 *>(&Vs[ii][0]);
#pragma unroll
                for (int q = 0; q < kEB / 4; ++q) {
                    const float4 vq = vv[q * NEB + ej];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        acc[r][4 * q + 0] = fmaf(pr[r], vq.x, acc[r][4 * q + 0]);
                        acc[r][4 * q + 1] = fmaf(pr[r], vq.y, acc[r][4 * q + 1]);
                        acc[r][4 * q + 2] = fmaf(pr[r], vq.z, acc[r][4 * q + 2]);
                        acc[r][4 * q + 3] = fmaf(pr[r], vq.w, acc[r][4 * q + 3]);
                    }
                }
                if (ej == 0) {
#pragma unroll
                    for (int r = 0; r < 4; ++r) sacc[r] += pr[r];
                }
            }
        }
    }
    if (!active) return;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int row = rb0 + rg * 4 + r;
        if (row >= D) break;
        const size_t base = ((size_t)h * D + row) * DH;
        const float4 *src = reinterpret_cast<const float4 *>(Hsrc + base);
        float4 *dst = reinterpret_cast<float4 *>(Hdst + base);
#pragma unroll
        for (int q = 0; q < kEB / 4; ++q) {
            float4 x = src[q * NEB + ej];
            x.x += acc[r][4 * q + 0];
            x.y += acc[r][4 * q + 1];
            x.z += acc[r][4 * q + 2];
            x.w += acc[r][4 * q + 3];
            dst[q * NEB + ej] = x;
        }
        if (ej == 0) sdst[(size_t)h * D + row] = ssrc[(size_t)h * D + row] + sacc[r];
    }
}

// One warp per query: window and cache softmax terms plus the state partials.
template <typename Tin, int DH>
__global__ void __launch_bounds__(kThreads)
hybrid_finish_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                     const Tin *__restrict__ v, int T, int seg0, int nq, int w0,
                     const Tin *__restrict__ ck, const Tin *__restrict__ cv, int nc, int cap,
                     const float *__restrict__ part, int P, float eps, float tau,
                     float *__restrict__ o) {
    constexpr int PL = (DH + 31) / 32;  // elements per lane
    const int h = blockIdx.x, nh = gridDim.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int r = blockIdx.y * (kThreads / 32) + warp;
    if (r >= nq) return;
    const int i = seg0 + r;
    const size_t hoff = (size_t)h * T * DH;
    float qv[PL], num[PL];
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        const int a = lane + 32 * c;
        qv[c] = a < DH ? to_f32(q[hoff + (size_t)i * DH + a]) : 0.f;
        num[c] = 0.f;
    }
    // The softmax weights are taken relative to m = max(0, max_j tau q.k_j)
    // (raised on the fly, rescaling what was summed so far), and the state
    // terms and eps are scaled by exp(-m) to match: the same quotient, with no
    // exp overflow however large tau q.k gets.
    float den = 0.f, mx = 0.f;
    const int nw = i - w0 + 1;
    for (int jj = 0; jj < nw + nc; ++jj) {
        const Tin *kj, *vj;
        if (jj < nw) {
            kj = k + hoff + (size_t)(w0 + jj) * DH;
            vj = v + hoff + (size_t)(w0 + jj) * DH;
        } else {
            kj = ck + ((size_t)h * cap + (jj - nw)) * DH;
            vj = cv + ((size_t)h * cap + (jj - nw)) * DH;
        }
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const int a = lane + 32 * c;
            if (a < DH) dot = fmaf(qv[c], to_f32(kj[a]), dot);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float t = tau * dot;
        if (t > mx) {
            const float r = expf(mx - t);
            den *= r;
#pragma unroll
            for (int c = 0; c < PL; ++c) num[c] *= r;
            mx = t;
        }
        const float w = expf(t - mx);
        den += w;
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const int a = lane + 32 * c;
            if (a < DH) num[c] = fmaf(w, to_f32(vj[a]), num[c]);
        }
    }
    float sden = 0.f, snum[PL];
#pragma unroll
    for (int c = 0; c < PL; ++c) snum[c] = 0.f;
    for (int p = 0; p < P; ++p) {
        const float *src = part + (((size_t)p * nh + h) * nq + r) * (DH + 1);
        sden += src[DH];
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const int a = lane + 32 * c;
            if (a < DH) snum[c] += src[a];
        }
    }
    const float sc = mx > 0.f ? expf(-mx) : 1.f;
#pragma unroll
    for (int c = 0; c < PL; ++c) num[c] = fmaf(snum[c], sc, num[c]);
    const float inv = 1.f / (fmaf(sden + eps, sc, den));
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        const int a = lane + 32 * c;
        if (a < DH) o[hoff + (size_t)i * DH + a] = num[c] * inv;
    }
}

template <typename Tin>
__global__ void lola_append_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v, int T,
                                   int d, int pstart, int U, Tin *cand_k, Tin *cand_v,
                                   int *cand_pos, int cap, int nc) {
    const int h = blockIdx.x;
    for (int idx = threadIdx.x; idx < U * d; idx += blockDim.x) {
        const int u = idx / d, a = idx % d;
        if (!KATA_CHECK(nc + u < cap, 0xB301u) || !KATA_CHECK(pstart + u < T, 0xB302u)) continue;
        const size_t src = ((size_t)h * T + pstart + u) * d + a;
        const size_t dst = ((size_t)h * cap + nc + u) * d + a;
        cand_k[dst] = k[src];
        cand_v[dst] = v[src];
        if (a == 0) cand_pos[(size_t)h * cap + nc + u] = pstart + u;
    }
}

template <typename Tin>
__global__ void lola_compact_kernel(const Tin *__restrict__ src_k, const Tin *__restrict__ src_v,
                                    const int *__restrict__ src_pos, Tin *__restrict__ dst_k,
                                    Tin *__restrict__ dst_v, int *__restrict__ dst_pos,
                                    const int *__restrict__ keep_idx, int m, int cap, int d,
                                    int *__restrict__ kept_pos, int cache) {
    const int h = blockIdx.x;
    for (int idx = threadIdx.x; idx < m * d; idx += blockDim.x) {
        const int rr = idx / d, a = idx % d;
        const int j = keep_idx[(size_t)h * m + rr];
        if (!KATA_CHECK(j >= 0 && j < cap, 0xB303u)) continue;
        dst_k[((size_t)h * cap + rr) * d + a] = src_k[((size_t)h * cap + j) * d + a];
        dst_v[((size_t)h * cap + rr) * d + a] = src_v[((size_t)h * cap + j) * d + a];
        if (a == 0) dst_pos[(size_t)h * cap + rr] = src_pos[(size_t)h * cap + j];
    }
    if (kept_pos)
        for (int rr = threadIdx.x; rr < cache; rr += blockDim.x)
            kept_pos[(size_t)h * cache + rr] =
                rr < m ? src_pos[(size_t)h * cap + keep_idx[(size_t)h * m + rr]] : -1;
}

size_t elem_size(int dtype) { return dtype == 0 ? 4 : 2; }

struct SreWs {
    float *part;
    int *mlist, *mcount;
};

SreWs carve_sre(void *ws, int nh, int n, int d) {
    char *p = static_cast<char *>(ws);
    SreWs w;
    w.part = reinterpret_cast<float *>(p);
    p += align_up(partial_floats(nh, n, d) * sizeof(float), 256);
    w.mlist = reinterpret_cast<int *>(p);
    p += align_up((size_t)nh * n * sizeof(int), 256);
    w.mcount = reinterpret_cast<int *>(p);
    return w;
}

template <typename Tin>
cudaError_t sre_impl(const float *Hst, const float *s, const Tin *kc, const Tin *vc,
                     const int *pos, int nh, int d, int n, int cand_stride, int keep, float eps,
                     int merge, float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                     void *ws, cudaStream_t stream) {
    const int P = num_slices(nh, n, d);
    SreWs w = carve_sre(ws, nh, n, d);
    const long cstride = (long)cand_stride * d;
    cudaError_t err = launch_state_partial<Tin>(kc, cstride, nh, n, d, Hst, s, P, w.part, stream);
    if (err != cudaSuccess) return err;
    // 32 warps share the per-candidate reductions; the ranking uses one thread
    // per candidate (n <= 1024)
    const int threads = 1024;
    sre_select_kernel<Tin><<<nh, threads, 0, stream>>>(w.part, P, n, d, vc, cstride, pos,
                                                       cand_stride, keep, eps, scores, keep_idx,
                                                       w.mlist, w.mcount);
    if ((err = after_launch()) != cudaSuccess) return err;
    if (!merge || keep >= n) {
        if (merge && (Hst_mut != Hst || s_mut != s)) {  // nothing to merge: copy through
            const int D = packed_dim(d);
            if ((err = cudaMemcpyAsync(Hst_mut, Hst, (size_t)nh * D * d * 4,
                                       cudaMemcpyDeviceToDevice, stream)) != cudaSuccess)
                return err;
            if ((err = cudaMemcpyAsync(s_mut, s, (size_t)nh * D * 4, cudaMemcpyDeviceToDevice,
                                       stream)) != cudaSuccess)
                return err;
        }
        return cudaSuccess;
    }
    const int D = packed_dim(d);
    dim3 grid(nh, (D + kMR - 1) / kMR);
    switch (d) {
        case 16: merge_kernel<Tin, 16><<<grid, kThreads, 0, stream>>>(Hst, s, Hst_mut, s_mut, kc, vc, cstride, w.mlist, w.mcount, n); break;
        case 32: merge_kernel<Tin, 32><<<grid, kThreads, 0, stream>>>(Hst, s, Hst_mut, s_mut, kc, vc, cstride, w.mlist, w.mcount, n); break;
        case 64: merge_kernel<Tin, 64><<<grid, kThreads, 0, stream>>>(Hst, s, Hst_mut, s_mut, kc, vc, cstride, w.mlist, w.mcount, n); break;
        default: return cudaErrorInvalidValue;
    }
    return after_launch();
}

template <typename Tin>
cudaError_t readout_impl(const Tin *q, const Tin *k, const Tin *v, int nh, int T, int d,
                         int seg0, int nq, int w0, const Tin *ck, const Tin *cv, int nc,
                         int cap, const float *Hst, const float *s, float eps, float tau,
                         float *o, void *ws, cudaStream_t stream) {
    const int P = num_slices(nh, nq, d);
    float *part = static_cast<float *>(ws);
    cudaError_t err = launch_state_partial<Tin>(q + (size_t)seg0 * d, (long)T * d, nh, nq, d,
                                                Hst, s, P, part, stream);
    if (err != cudaSuccess) return err;
    dim3 grid(nh, (nq + 7) / 8);
    switch (d) {
        case 16: hybrid_finish_kernel<Tin, 16><<<grid, kThreads, 0, stream>>>(q, k, v, T, seg0, nq, w0, ck, cv, nc, cap, part, P, eps, tau, o); break;
        case 32: hybrid_finish_kernel<Tin, 32><<<grid, kThreads, 0, stream>>>(q, k, v, T, seg0, nq, w0, ck, cv, nc, cap, part, P, eps, tau, o); break;
        case 64: hybrid_finish_kernel<Tin, 64><<<grid, kThreads, 0, stream>>>(q, k, v, T, seg0, nq, w0, ck, cv, nc, cap, part, P, eps, tau, o); break;
        default: return cudaErrorInvalidValue;
    }
    return after_launch();
}

// The schedule scores between 1 and cap candidates; the slice count (and so
// the partial-sum buffer) depends on the count, so size for the largest.
size_t max_sre_workspace_bytes(int nh, int d, int cap) {
    size_t m = 0;
    for (int n = 1; n <= cap; ++n) {
        const size_t b = sre_workspace_bytes(nh, 1, d, n);
        if (b > m) m = b;
    }
    return m;
}

struct LolaWs {
    void *ck[2], *cv[2];
    int *cpos[2];
    int *keep_idx;
    void *sre_ws;
    void *readout_ws;
};

LolaWs carve_lola(void *ws, int nh, int T, int d, int window, int cache, int dtype) {
    const int cap = cache + window;
    const size_t es = elem_size(dtype);
    char *p = static_cast<char *>(ws);
    LolaWs w;
    for (int b = 0; b < 2; ++b) {
        w.ck[b] = p;
        p += align_up((size_t)nh * cap * d * es, 256);
        w.cv[b] = p;
        p += align_up((size_t)nh * cap * d * es, 256);
        w.cpos[b] = reinterpret_cast<int *>(p);
        p += align_up((size_t)nh * cap * sizeof(int), 256);
    }
    w.keep_idx = reinterpret_cast<int *>(p);
    p += align_up((size_t)nh * cap * sizeof(int), 256);
    w.sre_ws = p;
    p += align_up(max_sre_workspace_bytes(nh, d, cap), 256);
    w.readout_ws = p;
    (void)T;
    return w;
}

template <typename Tin>
cudaError_t lola_impl(const Tin *q, const Tin *k, const Tin *v, int dtype, int nh, int T, int d,
                      int window, int cache, float eps, float tau, float *o, float *Hst,
                      float *s, int *kept_pos, void *ws, cudaStream_t stream) {
    const int U = window, cap = cache + window, G = T / U;
    LolaWs w = carve_lola(ws, nh, T, d, window, cache, dtype);
    int cur = 0, nc = 0;
    cudaError_t err;
    for (int g = 0; g < G; ++g) {
        err = readout_impl<Tin>(q, k, v, nh, T, d, g * U, U, g >= 1 ? U * (g - 1) : 0,
                                static_cast<const Tin *>(w.ck[cur]),
                                static_cast<const Tin *>(w.cv[cur]), nc, cap, Hst, s, eps, tau,
                                o, w.readout_ws, stream);
        if (err != cudaSuccess) return err;
        if (g < 1) continue;
        lola_append_kernel<Tin><<<nh, 256, 0, stream>>>(
            k, v, T, d, U * (g - 1), U, static_cast<Tin *>(w.ck[cur]),
            static_cast<Tin *>(w.cv[cur]), w.cpos[cur], cap, nc);
        if ((err = after_launch()) != cudaSuccess) return err;
        const int n = nc + U;
        const int m = cache < n ? cache : n;
        err = sre_score_topk(Hst, s, w.ck[cur], w.cv[cur], w.cpos[cur], dtype, nh, 1, d, n, cap,
                             cache, eps, 1, nullptr, w.keep_idx, Hst, s, w.sre_ws, 0, stream);
        if (err != cudaSuccess) return err;
        lola_compact_kernel<Tin><<<nh, 256, 0, stream>>>(
            static_cast<const Tin *>(w.ck[cur]), static_cast<const Tin *>(w.cv[cur]),
            w.cpos[cur], static_cast<Tin *>(w.ck[1 - cur]), static_cast<Tin *>(w.cv[1 - cur]),
            w.cpos[1 - cur], w.keep_idx, m, cap, d,
            kept_pos ? kept_pos + (size_t)(g - 1) * nh * cache : nullptr, cache);
        if ((err = after_launch()) != cudaSuccess) return err;
        cur = 1 - cur;
        nc = m;
    }
    return cudaSuccess;
}

}  // namespace

size_t sre_workspace_bytes(int B, int H, int d, int n_cand) {
    const int nh = B * H;
    return align_up(partial_floats(nh, n_cand, d) * sizeof(float), 256) +
           align_up((size_t)nh * n_cand * sizeof(int), 256) +
           align_up((size_t)nh * sizeof(int), 256);
}

size_t readout_workspace_bytes(int B, int H, int d, int nq) {
    return align_up(partial_floats(B * H, nq, d) * sizeof(float), 256);
}

size_t lola_workspace_bytes(int B, int H, int T, int d, int window, int cache) {
    const int nh = B * H, cap = cache + window;
    const size_t es = 4;  // sized for the wider input type
    size_t b = 0;
    for (int i = 0; i < 2; ++i)
        b += 2 * align_up((size_t)nh * cap * d * es, 256) +
             align_up((size_t)nh * cap * sizeof(int), 256);
    b += align_up((size_t)nh * cap * sizeof(int), 256);
    b += align_up(max_sre_workspace_bytes(nh, d, cap), 256);
    b += readout_workspace_bytes(nh, 1, d, window);
    (void)T;
    return b;
}

cudaError_t sre_score_topk(const float *Hst, const float *s, const void *kc, const void *vc,
                           const int *pos, int dtype, int B, int H, int d, int n_cand,
                           int cand_stride, int keep, float eps, int merge, float *scores,
                           int *keep_idx, float *Hst_mut, float *s_mut, void *ws,
                           size_t ws_bytes, cudaStream_t stream) {
    KATA_DEBUG_BIND();
    (void)ws_bytes;
    const int nh = B * H;
    if (sre_tc_applies(dtype, d, n_cand, Hst, s, Hst_mut, s_mut, kc, vc))
        return sre_tc(Hst, s, kc, vc, pos, nh, d, n_cand, cand_stride, keep, eps, merge, scores,
                      keep_idx, Hst_mut, s_mut, device_error_word(), stream);
    if (dtype == 0)
        return sre_impl<float>(Hst, s, static_cast<const float *>(kc),
                               static_cast<const float *>(vc), pos, nh, d, n_cand, cand_stride,
                               keep, eps, merge, scores, keep_idx, Hst_mut, s_mut, ws, stream);
    return sre_impl<__nv_bfloat16>(Hst, s, static_cast<const __nv_bfloat16 *>(kc),
                                   static_cast<const __nv_bfloat16 *>(vc), pos, nh, d, n_cand,
                                   cand_stride, keep, eps, merge, scores, keep_idx, Hst_mut,
                                   s_mut, ws, stream);
}

cudaError_t hybrid_readout(const void *q, const void *k, const void *v, int dtype, int B,
                           int H, int T, int d, int seg0, int nq, int w0, const void *ck,
                           const void *cv, int nc, int cap, const float *Hst, const float *s,
                           float eps, float tau, float *o, void *ws, size_t ws_bytes,
                           cudaStream_t stream) {
    KATA_DEBUG_BIND();
    (void)ws_bytes;
    const int nh = B * H;
    if (dtype == 0)
        return readout_impl<float>(static_cast<const float *>(q), static_cast<const float *>(k),
                                   static_cast<const float *>(v), nh, T, d, seg0, nq, w0,
                                   static_cast<const float *>(ck),
                                   static_cast<const float *>(cv), nc, cap, Hst, s, eps, tau, o,
                                   ws, stream);
    using bf = __nv_bfloat16;
    return readout_impl<bf>(static_cast<const bf *>(q), static_cast<const bf *>(k),
                            static_cast<const bf *>(v), nh, T, d, seg0, nq, w0,
                            static_cast<const bf *>(ck), static_cast<const bf *>(cv), nc, cap,
                            Hst, s, eps, tau, o, ws, stream);
}

cudaError_t lola_run(const void *q, const void *k, const void *v, int dtype, int B, int H,
                     int T, int d, int window, int cache, float eps, float tau, float *o,
                     float *Hst, float *s, int *kept_pos, void *ws, size_t ws_bytes,
                     cudaStream_t stream) {
    KATA_DEBUG_BIND();
    (void)ws_bytes;
    const int nh = B * H;
    if (dtype == 0)
        return lola_impl<float>(static_cast<const float *>(q), static_cast<const float *>(k),
                                static_cast<const float *>(v), dtype, nh, T, d, window, cache,
                                eps, tau, o, Hst, s, kept_pos, ws, stream);
    using bf = __nv_bfloat16;
    return lola_impl<bf>(static_cast<const bf *>(q), static_cast<const bf *>(k),
                         static_cast<const bf *>(v), dtype, nh, T, d, window, cache, eps, tau, o,
                         Hst, s, kept_pos, ws, stream);
}

}  // namespace kata

namespace kata {

// ---------------------------------------------------------------------------
// SRE scoring + top-k with a fixed scratch area instead of a caller workspace.
//
// Some callers cannot allocate device memory at the point where they score
// candidates: code running under an allocator that must not grow (a serving
// loop with a pre-sized memory pool), or a host program that has no allocator
// of its own for device scratch. For them the scratch lives in one file-scope
// device array of kNoAllocScratchBytes, created when the library is loaded on
// a device and kept until the process exits.
//
// Set-up: the array's device address is looked up once per device, with that
// device current, by the first call on that device. Make that first call
// before any stream capture.
// Sharing: every call uses the same array and it keeps the last call's
// contents. Nothing in it needs to start at zero (every value the kernels read
// is written earlier in the same call). Calls whose kernels overlap on the GPU
// (other streams, other host threads) race on the array; serialise them.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 128;  // device ordinals the address cache covers
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kMaxDevices] = {nullptr};

cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

}  // namespace

size_t sre_noalloc_capacity() { return kNoAllocScratchBytes; }

cudaError_t sre_score_topk_noalloc(const float *Hst, const float *s, const void *kc,
                                   const void *vc, const int *pos, int dtype, int B, int H,
                                   int d, int n_cand, int keep, float eps, int merge,
                                   float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                                   cudaStream_t stream) {
    void *scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    return sre_score_topk(Hst, s, kc, vc, pos, dtype, B, H, d, n_cand, n_cand, keep, eps,
                          merge, scores, keep_idx, Hst_mut, s_mut, scratch,
                          kNoAllocScratchBytes, stream);
}

}  // namespace kata
