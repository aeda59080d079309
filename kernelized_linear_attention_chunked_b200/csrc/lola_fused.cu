// The whole LoLA schedule in one launch: one cluster of NCL CTAs per head
// keeps that head's fp32 state on chip for the entire sequence.
//
// "LoLA: Low-Rank Linear Attention with Sparse Caching":
//  - Methodology 1-3: a sliding window of recent pairs (full-rank softmax), the
//    linear state H_t = sum phi(k) v^T with normaliser s_t = sum phi(k), and a
//    sparse cache of pairs the state recalls badly;
//  - "Self-Recall Error": SRE(k, v | H, s) = || phi(k)^T H / phi(k)^T s - v ||^2
//    (eps added to the denominator, as in every readout here);
//  - "Inference strategy" 1-4: segment by segment, the pairs leaving the window
//    and the cached pairs are scored against the current state, the highest
//    SRE stay cached, the rest are merged into the state by outer products,
//    and the output combines the window, the cache and the state.
// phi is the rank-one PSD feature of "Kernelized Linear Attention: Breaking
// the Capacity Wall with Symmetric Cones", s2.2, in the canonical packed
// layout (upper triangle, sqrt(2) on off-diagonal entries).
//
// Segment g (W tokens; the window of its queries starts at W(g-1)) runs:
//   A. X^T: the segment's queries, the keys leaving the window (segment g-1),
//      the cached keys and the segment's own keys, transposed into shared
//      memory (in the input type: the values are used as stored).
//   B. phi(x)^T [H | s] over this CTA's rows of the state for the queries and
//      the keys leaving the window (each CTA owns D/NCL rows of [H | s];
//      partial sums go to a global scratch, summed in CTA order afterwards).
//   C. After a cluster barrier each CTA finishes every NCL-th query (state
//      terms plus the window and cache softmax terms, max-shifted, one shared
//      denominator) and 1/NCL of the candidates: phi(k)^T [H | s] of a cached
//      candidate is carried from the update that kept it (below), that of a
//      new one is the sum of the partials; then its SRE.
//   D. After a second cluster barrier every CTA ranks all candidates (higher
//      SRE first, an exact tie to the smaller position) and derives the same
//      kept set and merge list.
//   E. Each CTA adds the merged pairs' phi(k) v^T and phi(k) to its rows, and
//      carries the kept candidates' phi(k)^T [H | s] forward by the same merged
//      pairs: phi(k_j)^T (H + sum_m phi(k_m) v_m^T) =
//      phi(k_j)^T H + sum_m (k_j . k_m)^2 v_m^T (the PSD kernel identity), so a
//      cached candidate is never rescored against the whole state.
// The state is written back once at the end.
//
// The cluster size NCL (8 down to 6) is the largest for which every head's
// cluster is resident at once (a head whose cluster waits for a second wave
// doubles the time of the whole launch).
#include <atomic>

#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {
namespace {

constexpr int kFT = 352;          // threads: a state row each in the merge (up to 352 rows);
                                  // warps 0-7 score the H columns, warp 8 the s column
constexpr int kRC = 32;           // state rows per phi chunk
constexpr int kNSMax = 128;       // scoring vectors per segment (queries + new candidates)
constexpr int kNKMax = 256;       // softmax keys per segment (window + cache)
constexpr int kWMax = 64;         // longest segment
constexpr int kQMax = 16;         // queries per CTA (a segment over at least 4 CTAs)
constexpr int kNclMin = 6;        // fewest CTAs per head: D / 6 rows fit one pass of kFT threads
constexpr int kVPT = 4;           // scoring vectors per thread of the s column
constexpr int kVPH = 8;           // scoring vectors per thread of the H columns (x 8 columns)

__device__ __forceinline__ float xv(const float *p) { return *p; }
__device__ __forceinline__ float xv(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// Eight consecutive values (16-byte aligned) as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// Eight consecutive values (16-byte aligned), kept in the input type.
__device__ __forceinline__ void raw8(const __nv_bfloat16 *p, __nv_bfloat16 (&x)[8]) {
    *reinterpret_cast<uint4 *>(x) = *reinterpret_cast<const uint4 *>(p);
}
__device__ __forceinline__ void raw8(const float *p, float (&x)[8]) { load8(p, x); }
// Two consecutive values (8-byte aligned for fp32, 4-byte for bf16) as fp32.
__device__ __forceinline__ float2 load2(const __nv_bfloat16 *p) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float2 load2(const float *p) {
    return *reinterpret_cast<const float2 *>(p);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster: release this thread's earlier
// memory operations (global and shared) to the cluster, acquire the others'.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <typename Tin, int DH, int NCL>
struct FusedCfg {
    static constexpr int D = DH * (DH + 1) / 2;
    static constexpr int R = (D + NCL - 1) / NCL;          // state rows per CTA
    static constexpr int RP = (R + 3) / 4 * 4;
    static constexpr int NCOL = kWMax + kNKMax;            // X^T columns (upper bound)
    // X^T pitch in elements: odd in 32-bit words, so column reads down a row
    // of pairs and row writes across columns spread over the banks
    static constexpr int P = sizeof(Tin) == 4 ? NCOL + 1 : NCOL + 2;
    static constexpr int XT_FLOATS = ((DH * P * (int)sizeof(Tin) + 15) / 16) * 4;
    static constexpr int PHI_FLOATS = kRC * kNSMax;
    static constexpr int VST_FLOATS = (kNKMax * DH * (int)sizeof(Tin) + 3) / 4;
    static constexpr int BUF = PHI_FLOATS > VST_FLOATS ? PHI_FLOATS : VST_FLOATS;
    static constexpr int RED = kQMax * (DH + 1);
    static constexpr int VM = kWMax * DH;                  // merged pairs' values, fp32
    // in floats: Hs, ss, tab (ints), XT, buf, red, vm, logits, then the ints
    static constexpr int OFF_SS = R * DH;
    static constexpr int OFF_TAB = OFF_SS + RP;
    static constexpr int OFF_XT = OFF_TAB + RP;
    static constexpr int OFF_BUF = OFF_XT + XT_FLOATS;
    static constexpr int OFF_RED = OFF_BUF + BUF;
    static constexpr int OFF_VM = OFF_RED + RED;
    static constexpr int OFF_LOG = OFF_VM + VM;
    static constexpr int OFF_INT = OFF_LOG + kQMax * kNKMax;
    static constexpr int NINT = 6 * kNKMax + 2 * kQMax;
    static constexpr size_t BYTES = (size_t)(OFF_INT + NINT) * 4;
    static_assert(OFF_SS % 4 == 0 && RED % 4 == 0 && BUF % 4 == 0, "16-byte alignment");
    static_assert(R <= kFT, "one state row per thread in the merge");
    static_assert((DH / 16) * ((R + DH / 16 - 1) / (DH / 16)) <= kFT,
                  "one (row group, column group) tile per thread in the merge");
};

// Global scratch per head: partial sums [NCL][kNSMax][DH+1], the full
// phi(k)^T [H | s] of this segment's candidates [kNKMax][DH+1], the carried
// values of the cached pairs [kNKMax][DH+1], and the scores [kNKMax].
template <int DH>
__host__ __device__ constexpr size_t fused_scratch_floats() {
    return (size_t)8 * kNSMax * (DH + 1) + 2 * (size_t)kNKMax * (DH + 1) + kNKMax;
}

// Candidate i is retained before candidate j: higher SRE, then smaller
// position, then smaller slot.
__device__ __forceinline__ bool kept_before(float si, int pi, int i, float sj, int pj, int j) {
    if (si != sj) return si > sj;
    if (pi != pj) return pi < pj;
    return i < j;
}

template <typename Tin, int DH, int NCL>
__global__ void __launch_bounds__(kFT, 1)
lola_fused_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                  const Tin *__restrict__ v, int T, int W, int cache, float eps, float tau,
                  float *__restrict__ o, float *Hst, float *s, int *__restrict__ kept_pos,
                  float *__restrict__ scratch) {
    using C = FusedCfg<Tin, DH, NCL>;
    constexpr int D = C::D, R = C::R, P = C::P;
    constexpr int CG = DH / 8;   // column groups of the scoring GEMM (8 columns per thread)
    constexpr int E1 = DH + 1;   // [H | s] columns
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    float *Hs = sm;                                           // [R][DH]
    float *ss = sm + C::OFF_SS;                               // [R]
    int *tab = reinterpret_cast<int *>(sm + C::OFF_TAB);      // [R] pair of each row
    Tin *XT = reinterpret_cast<Tin *>(sm + C::OFF_XT);        // [DH][P]
    float *buf = sm + C::OFF_BUF;                             // phi chunk / staged values
    float *red = sm + C::OFF_RED;                             // [kQMax][DH+1]
    float *vm = sm + C::OFF_VM;                               // [nm][DH] merged values
    float *logit = sm + C::OFF_LOG;                           // [kQMax][kNKMax]
    int *ip = reinterpret_cast<int *>(sm + C::OFF_INT);
    int *cpos0 = ip, *cpos1 = ip + kNKMax;                    // cache positions (two buffers)
    int *cand_pos = ip + 2 * kNKMax;                          // candidate positions
    int *kflag = ip + 3 * kNKMax;                             // kept flags
    int *klist = ip + 4 * kNKMax;                             // kept candidates, slot order
    int *mlist = ip + 5 * kNKMax;                             // merged candidates
    float *qmax = reinterpret_cast<float *>(ip + 6 * kNKMax); // [kQMax]
    float *qden = qmax + kQMax;
    float *scs = logit;  // the scores reuse the logits' space after the readout

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cr = (int)cluster_rank();
    const int head = blockIdx.x / NCL, nh = gridDim.x / NCL;
    const int r0 = cr * R;
    const int nrows = D - r0 < R ? (D - r0 > 0 ? D - r0 : 0) : R;
    const size_t hoff = (size_t)head * T * DH;
    const Tin *qh = q + hoff, *kh = k + hoff, *vh = v + hoff;
    float *Hh = Hst + (size_t)head * D * DH;
    float *sh = s + (size_t)head * D;
    float *part = scratch + (size_t)head * fused_scratch_floats<DH>();  // [NCL][kNSMax][E1]
    float *cand_num = part + (size_t)8 * kNSMax * E1;                    // [kNKMax][E1]
    float *cache_num = cand_num + (size_t)kNKMax * E1;                   // [kNKMax][E1]
    float *score_g = cache_num + (size_t)kNKMax * E1;                    // [kNKMax]
    Tin *vst = reinterpret_cast<Tin *>(buf);                             // [nk][DH]

    // the pair (a, b) of each of this CTA's rows, and the initial state slice
    for (int rr = tid; rr < R; rr += kFT) {
        const int r = r0 + rr;
        int e = -1;
        if (r < D) {
            int a = 0;
            while (packed_row_base(a + 1, DH) <= r) ++a;
            const int b = a + r - packed_row_base(a, DH);
            e = a | (b << 8) | ((a != b) << 16);
        }
        tab[rr] = e;
        ss[rr] = r < D ? sh[r] : 0.f;
    }
    for (int idx = tid; idx < R * DH / 4; idx += kFT) {
        const int rr = idx / (DH / 4);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r0 + rr < D) x = reinterpret_cast<const float4 *>(Hh + (size_t)r0 * DH)[idx];
        reinterpret_cast<float4 *>(Hs)[idx] = x;
    }

    const int G = T / W;
    const int nq = cr < W ? (W - cr + NCL - 1) / NCL : 0;  // this CTA's queries: cr, cr + NCL, ...
    int nc = 0;  // cached pairs (the same in every CTA)
    int *cpos = cpos0, *cnext = cpos1;
    for (int g = 0; g < G; ++g) {
        const int seg0 = g * W;
        const int nE = g >= 1 ? W : 0;   // pairs leaving the window: segment g-1
        const int ncand = nc + nE;       // candidates: the cache, then segment g-1
        const int nsc = W + nE;          // scored against the state: queries, segment g-1
        const int nk = nE + nc + W;      // softmax keys: segment g-1, the cache, segment g
        // X^T columns: [0, W) queries, [W, W + nE) segment g-1 keys (also softmax
        // keys 0 .. nE-1), then the cached keys and segment g's keys; softmax
        // key t is column W + t
        auto key_pos = [&](int t) -> int {
            return t < nE ? seg0 - W + t : (t < nE + nc ? cpos[t - nE] : seg0 + (t - nE - nc));
        };
        // candidate j (slot order: cached pairs, then segment g-1) -> softmax key
        auto cand_key = [&](int j) -> int { return j < nc ? nE + j : j - nc; };

        __syncthreads();  // the previous segment is done with X^T, buf and the lists
        // ---- A: X^T (the stored values, transposed) ----
        for (int idx = tid; idx < (W + nk) * (DH / 8); idx += kFT) {
            const int col = idx / (DH / 8), a0 = 8 * (idx % (DH / 8));
            const Tin *src = col < W ? qh + (size_t)(seg0 + col) * DH
                                     : kh + (size_t)key_pos(col - W) * DH;
            Tin x[8];
            raw8(src + a0, x);
#pragma unroll
            for (int i = 0; i < 8; ++i) XT[(a0 + i) * P + col] = x[i];
        }
        __syncthreads();

        // ---- B: phi(x)^T [H | s] over this CTA's rows, x = queries + new candidates ----
        {
            // H threads: 8 vectors x 8 columns (4cg..4cg+3 and 4(CG+cg)..+3) each,
            // so one 16-byte read of shared memory feeds 16 multiply-adds
            const bool hthr = tid < (kNSMax / kVPH) * CG;
            const bool sthr = warp == 8;      // the s column: 4 vectors per lane
            const int nvt = hthr ? kVPH : kVPT;     // vectors per thread
            const int vg = hthr ? tid / CG : lane;  // vectors nvt vg .. nvt vg + nvt - 1
            const int cg = tid % CG;
            const bool act = (hthr || sthr) && nvt * vg < nsc;
            const int bx = tid & (kNSMax - 1), brs = tid >> 7;  // phi builder: column, row phase
            float acc[kVPH][8];
#pragma unroll
            for (int i = 0; i < kVPH; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
            for (int c0 = 0; c0 < nrows; c0 += kRC) {
                const int nr = nrows - c0 < kRC ? nrows - c0 : kRC;
                __syncthreads();  // the previous chunk is consumed
                if (tid < 2 * kNSMax && bx < nsc) {
#pragma unroll 4
                    for (int rr = brs; rr < kRC; rr += 2) {
                        float val = 0.f;
                        if (rr < nr) {
                            const int e = tab[c0 + rr];
                            const float p = xv(XT + (e & 255) * P + bx) * xv(XT + ((e >> 8) & 255) * P + bx);
                            val = (e >> 16) ? p * kSqrt2 : p;
                        }
                        buf[rr * kNSMax + bx] = val;
                    }
                }
                __syncthreads();
                if (act) {
                    const float *prow = buf + nvt * vg;
                    if (hthr) {
                        const float4 *hrow = reinterpret_cast<const float4 *>(Hs + c0 * DH);
#pragma unroll 2
                        for (int rr = 0; rr < nr; ++rr) {
                            const float4 p4 = *reinterpret_cast<const float4 *>(prow + rr * kNSMax);
                            const float4 p5 = *reinterpret_cast<const float4 *>(prow + rr * kNSMax + 4);
                            const float pv[kVPH] = {p4.x, p4.y, p4.z, p4.w, p5.x, p5.y, p5.z, p5.w};
                            const float4 h0 = hrow[rr * (DH / 4) + cg];
                            const float4 h1 = hrow[rr * (DH / 4) + CG + cg];
                            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                            for (int i = 0; i < kVPH; ++i)
#pragma unroll
                                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(pv[i], hv[j], acc[i][j]);
                        }
                    } else {
#pragma unroll 4
                        for (int rr = 0; rr < nr; ++rr) {
                            const float4 p4 = *reinterpret_cast<const float4 *>(prow + rr * kNSMax);
                            const float sv = ss[c0 + rr];
                            acc[0][0] = fmaf(p4.x, sv, acc[0][0]);
                            acc[1][0] = fmaf(p4.y, sv, acc[1][0]);
                            acc[2][0] = fmaf(p4.z, sv, acc[2][0]);
                            acc[3][0] = fmaf(p4.w, sv, acc[3][0]);
                        }
                    }
                }
            }
            if (act) {
                float *dst0 = part + (size_t)cr * kNSMax * E1;
#pragma unroll
                for (int i = 0; i < kVPH; ++i) {
                    if (i >= nvt) break;
                    const int x = nvt * vg + i;
                    if (x >= nsc) break;
                    float *dst = dst0 + (size_t)x * E1;
                    if (hthr) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            dst[4 * cg + j] = acc[i][j];
                            dst[4 * (CG + cg) + j] = acc[i][4 + j];
                        }
                    } else {
                        dst[DH] = acc[i][0];
                    }
                }
            }
        }
        cluster_barrier();  // every partial sum of this head is written

        // ---- C: this CTA's queries and candidates ----
        // values of the softmax keys, 16 bytes at a time
        constexpr int VCH = 16 / (int)sizeof(Tin);
        for (int idx = tid; idx < nk * (DH / VCH); idx += kFT) {
            const int t = idx / (DH / VCH), a0 = VCH * (idx % (DH / VCH));
            *reinterpret_cast<uint4 *>(vst + (size_t)t * DH + a0) =
                *reinterpret_cast<const uint4 *>(vh + (size_t)key_pos(t) * DH + a0);
        }
        const int cpc = (ncand + NCL - 1) / NCL;
        const int cc0 = cr * cpc < ncand ? cr * cpc : ncand;
        const int cc1 = cc0 + cpc < ncand ? cc0 + cpc : ncand;
        // the queries' state terms: partial sums in CTA order
        for (int idx = tid; idx < nq * E1; idx += kFT) {
            const int m = idx / E1, e = idx % E1;
            const int x = cr + NCL * m;
            float a = 0.f;
#pragma unroll
            for (int c = 0; c < NCL; ++c) a += __ldcg(part + ((size_t)c * kNSMax + x) * E1 + e);
            red[m * E1 + e] = a;
        }
        // the candidates' phi(k)^T [H | s]: carried for cached pairs, summed for new ones
        for (int idx = tid; idx < (cc1 - cc0) * E1; idx += kFT) {
            const int j = cc0 + idx / E1, e = idx % E1;
            float a = 0.f;
            if (j < nc) {
                a = __ldcg(cache_num + (size_t)j * E1 + e);
            } else {
                const int x = W + (j - nc);
#pragma unroll
                for (int c = 0; c < NCL; ++c) a += __ldcg(part + ((size_t)c * kNSMax + x) * E1 + e);
            }
            cand_num[(size_t)j * E1 + e] = a;
        }
        // logits of this CTA's queries against every key (causal inside segment g)
        for (int t = tid; t < nk; t += kFT) {
            float dot[kQMax];
#pragma unroll
            for (int i = 0; i < kQMax; ++i) dot[i] = 0.f;
#pragma unroll 2
            for (int a = 0; a < DH; ++a) {
                const Tin *xa = XT + a * P;
                const float kv = xv(xa + W + t);
#pragma unroll
                for (int i = 0; i < kQMax; ++i)
                    if (i < nq) dot[i] = fmaf(xv(xa + cr + NCL * i), kv, dot[i]);
            }
            const int kp = key_pos(t);
#pragma unroll
            for (int i = 0; i < kQMax; ++i)
                if (i < nq)
                    logit[i * kNKMax + t] = kp <= seg0 + cr + NCL * i ? tau * dot[i] : -INFINITY;
        }
        __syncthreads();  // logits, staged values, red and cand_num (this CTA's part) ready
        // softmax weights relative to m = max(0, max logit); one warp per query
        for (int i = warp; i < nq; i += kFT / 32) {
            float *L = logit + i * kNKMax;
            float mx = 0.f;
            for (int t = lane; t < nk; t += 32) mx = fmaxf(mx, L[t]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            float den = 0.f;
            for (int t = lane; t < nk; t += 32) {
                const float w = expf(L[t] - mx);
                L[t] = w;
                den += w;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
            if (lane == 0) {
                qmax[i] = mx;
                qden[i] = den;
            }
        }
        // SRE of this CTA's candidates: one warp each, lanes over the columns
        for (int m = warp; m < cc1 - cc0; m += kFT / 32) {
            const int j = cc0 + m;
            const float *cn = cand_num + (size_t)j * E1;
            const float inv = 1.f / (__ldcg(cn + DH) + eps);
            const Tin *vj = vst + (size_t)cand_key(j) * DH;
            float err = 0.f;
            for (int e = lane; e < DH; e += 32) {
                const float diff = __ldcg(cn + e) * inv - xv(vj + e);
                err = fmaf(diff, diff, err);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) err += __shfl_xor_sync(0xffffffffu, err, off);
            if (lane == 0) score_g[j] = isnan(err) ? -INFINITY : err;  // a total order
        }
        __syncthreads();
        // outputs: window + cache softmax terms plus the state terms scaled by exp(-m)
        for (int idx = tid; idx < nq * DH / 2; idx += kFT) {
            const int i = idx / (DH / 2), e = 2 * (idx % (DH / 2));
            const float *L = logit + i * kNKMax;
            float n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f;  // two keys at a time
            int t = 0;
            for (; t + 1 < nk; t += 2) {
                const float2 x = load2(vst + (size_t)t * DH + e);
                const float2 y = load2(vst + (size_t)(t + 1) * DH + e);
                n0 = fmaf(L[t], x.x, n0);
                n1 = fmaf(L[t], x.y, n1);
                n2 = fmaf(L[t + 1], y.x, n2);
                n3 = fmaf(L[t + 1], y.y, n3);
            }
            if (t < nk) {
                const float2 x = load2(vst + (size_t)t * DH + e);
                n0 = fmaf(L[t], x.x, n0);
                n1 = fmaf(L[t], x.y, n1);
            }
            const float mx = qmax[i];
            const float sc = mx > 0.f ? expf(-mx) : 1.f;
            const float *rv = red + i * E1;
            const float inv = 1.f / fmaf(rv[DH] + eps, sc, qden[i]);
            *reinterpret_cast<float2 *>(o + hoff + (size_t)(seg0 + cr + NCL * i) * DH + e) =
                make_float2(fmaf(rv[e], sc, n0 + n2) * inv, fmaf(rv[e + 1], sc, n1 + n3) * inv);
        }
        cluster_barrier();  // every score and candidate value of this head is written

        if (ncand == 0) continue;  // segment 0: nothing leaves the window yet
        // ---- D: the kept set, the same in every CTA ----
        const int keep = cache < ncand ? cache : ncand;
        for (int j = tid; j < ncand; j += kFT) {
            scs[j] = __ldcg(score_g + j);
            cand_pos[j] = key_pos(cand_key(j));
        }
        __syncthreads();
        for (int j = tid; j < ncand; j += kFT) {
            int rank = 0;
            if (keep < ncand) {
                const float sj = scs[j];
                const int pj = cand_pos[j];
                for (int i = 0; i < ncand; ++i) rank += kept_before(scs[i], cand_pos[i], i, sj, pj, j);
            }
            kflag[j] = rank < keep;
        }
        __syncthreads();
        for (int j = tid; j < ncand; j += kFT) {
            int before = 0;
            for (int i = 0; i < j; ++i) before += kflag[i];
            if (kflag[j]) {
                if (KATA_CHECK(before < keep, 0xB501u)) {
                    klist[before] = j;
                    cnext[before] = cand_pos[j];  // candidates are in ascending position
                }
            } else if (KATA_CHECK(j - before < ncand - keep, 0xB502u)) {
                mlist[j - before] = j;
            }
        }
        __syncthreads();
        const int nm = ncand - keep;
        if (cr == 0 && kept_pos)
            for (int t = tid; t < cache; t += kFT)
                kept_pos[((size_t)(g - 1) * nh + head) * cache + t] = t < keep ? cnext[t] : -1;

        // ---- E: merge into this CTA's rows; carry the kept candidates' values ----
        for (int idx = tid; idx < nm * (DH / 8); idx += kFT) {  // merged values, fp32
            const int mm = idx / (DH / 8), a0 = 8 * (idx % (DH / 8));
            float x[8];
            load8(vst + (size_t)cand_key(mlist[mm]) * DH + a0, x);
            *reinterpret_cast<float4 *>(vm + mm * DH + a0) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4 *>(vm + mm * DH + a0 + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
        __syncthreads();
        // H[r] += sum_m phi_r(k_m) v_m, s[r] += sum_m phi_r(k_m): each thread a tile
        // of RT rows x 16 columns (the pairs in list order, as one row at a time
        // would add them), so a merged value read from shared memory feeds RT
        // multiply-adds
        {
            constexpr int NCG = DH / 16, RT = DH / 16;  // column groups, rows per thread
            const int cg = tid % NCG, rg = tid / NCG;
            if (nm > 0 && RT * rg < nrows) {
                int ea[RT], eb[RT];
                float wgt[RT];
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const int e = RT * rg + i < nrows ? tab[RT * rg + i] : 0;
                    ea[i] = e & 255;
                    eb[i] = (e >> 8) & 255;
                    wgt[i] = (e >> 16) ? kSqrt2 : 1.f;
                }
                float acc[RT][16], sacc[RT];
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    sacc[i] = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) acc[i][c] = 0.f;
                }
#pragma unroll 2
                for (int mm = 0; mm < nm; ++mm) {
                    const int col = W + cand_key(mlist[mm]);
                    float pv[RT];
#pragma unroll
                    for (int i = 0; i < RT; ++i)
                        pv[i] = xv(XT + ea[i] * P + col) * xv(XT + eb[i] * P + col) * wgt[i];
                    const float4 *vr = reinterpret_cast<const float4 *>(vm + mm * DH + 16 * cg);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float4 x = vr[c];
#pragma unroll
                        for (int i = 0; i < RT; ++i) {
                            acc[i][4 * c] = fmaf(pv[i], x.x, acc[i][4 * c]);
                            acc[i][4 * c + 1] = fmaf(pv[i], x.y, acc[i][4 * c + 1]);
                            acc[i][4 * c + 2] = fmaf(pv[i], x.z, acc[i][4 * c + 2]);
                            acc[i][4 * c + 3] = fmaf(pv[i], x.w, acc[i][4 * c + 3]);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < RT; ++i) sacc[i] += pv[i];
                }
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const int rr = RT * rg + i;
                    if (rr >= nrows) break;
                    float4 *hr = reinterpret_cast<float4 *>(Hs + rr * DH + 16 * cg);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float4 h = hr[c];
                        h.x += acc[i][4 * c];
                        h.y += acc[i][4 * c + 1];
                        h.z += acc[i][4 * c + 2];
                        h.w += acc[i][4 * c + 3];
                        hr[c] = h;
                    }
                    if (cg == 0) ss[rr] += sacc[i];
                }
            }
        }
        // kept candidate n (of this CTA's share): phi(k)^T [H | s] after the merge
        {
            const int kpc = (keep + NCL - 1) / NCL;
            const int n0 = cr * kpc < keep ? cr * kpc : keep;
            const int n1 = n0 + kpc < keep ? n0 + kpc : keep;
            for (int n = n0 + warp; n < n1; n += kFT / 32) {
                const int j = klist[n];
                const int colj = W + cand_key(j);
                float add[(DH + 31) / 32];
                float sadd = 0.f;
#pragma unroll
                for (int c = 0; c < (DH + 31) / 32; ++c) add[c] = 0.f;
                for (int m0 = 0; m0 < nm; m0 += 32) {
                    // lane: (k_j . k_m)^2 of merged pair m0 + lane
                    float w = 0.f;
                    if (m0 + lane < nm) {
                        const int colm = W + cand_key(mlist[m0 + lane]);
                        float d0 = 0.f, d1 = 0.f;
                        for (int a = 0; a < DH; a += 2) {
                            d0 = fmaf(xv(XT + a * P + colj), xv(XT + a * P + colm), d0);
                            d1 = fmaf(xv(XT + (a + 1) * P + colj), xv(XT + (a + 1) * P + colm), d1);
                        }
                        w = (d0 + d1) * (d0 + d1);
                    }
                    const int cnt = nm - m0 < 32 ? nm - m0 : 32;
                    for (int u = 0; u < cnt; ++u) {
                        const float wu = __shfl_sync(0xffffffffu, w, u);
                        const float *vr = vm + (m0 + u) * DH;
#pragma unroll
                        for (int c = 0; c < (DH + 31) / 32; ++c)
                            if (lane + 32 * c < DH) add[c] = fmaf(wu, vr[lane + 32 * c], add[c]);
                        sadd += wu;
                    }
                }
                const float *src = cand_num + (size_t)j * E1;
                float *dst = cache_num + (size_t)n * E1;
#pragma unroll
                for (int c = 0; c < (DH + 31) / 32; ++c)
                    if (lane + 32 * c < DH) dst[lane + 32 * c] = __ldcg(src + lane + 32 * c) + add[c];
                if (lane == 0) dst[DH] = __ldcg(src + DH) + sadd;
            }
        }
        nc = keep;
        int *t = cpos;
        cpos = cnext;
        cnext = t;
    }

    // the final state slice
    __syncthreads();
    for (int idx = tid; idx < R * DH / 4; idx += kFT) {
        const int rr = idx / (DH / 4);
        if (r0 + rr < D) reinterpret_cast<float4 *>(Hh + (size_t)r0 * DH)[idx] =
            reinterpret_cast<const float4 *>(Hs)[idx];
    }
    for (int rr = tid; rr < nrows; rr += kFT) sh[r0 + rr] = ss[rr];
}

constexpr int kMaxDev = 128;

// Clusters of NCL CTAs of this kernel that can be resident at once on the
// current device (looked up once per device).
template <typename Tin, int DH, int NCL>
int max_clusters() {
    using C = FusedCfg<Tin, DH, NCL>;
    static std::atomic<int> cached[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c != 0) return c > 0 ? c : 0;
    int n = 0;
    if (cudaFuncSetAttribute(lola_fused_kernel<Tin, DH, NCL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::BYTES) == cudaSuccess) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(NCL, 1, 1);
        cfg.blockDim = dim3(kFT, 1, 1);
        cfg.dynamicSmemBytes = C::BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = NCL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, lola_fused_kernel<Tin, DH, NCL>, &cfg) !=
            cudaSuccess)
            n = 0;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    cached[dev].store(n > 0 ? n : -1, std::memory_order_relaxed);
    return n;
}

template <typename Tin, int DH, int NCL>
cudaError_t launch_ncl(const Tin *q, const Tin *k, const Tin *v, int nh, int T, int W, int cache,
                       float eps, float tau, float *o, float *Hst, float *s, int *kept_pos,
                       float *scratch, cudaStream_t stream) {
    using C = FusedCfg<Tin, DH, NCL>;
    static_assert(C::BYTES <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(lola_fused_kernel<Tin, DH, NCL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nh * NCL, 1, 1);
    cfg.blockDim = dim3(kFT, 1, 1);
    cfg.dynamicSmemBytes = C::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NCL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, lola_fused_kernel<Tin, DH, NCL>, q, k, v, T, W, cache, eps, tau,
                           o, Hst, s, kept_pos, scratch);
    if (e != cudaSuccess) return e;
    return after_launch();
}

// The largest cluster (8 down to 6 CTAs per head) that keeps every head's
// cluster resident at once; 8 when none does.
template <typename Tin, int DH>
int choose_ncl(int nh) {
    static_assert(kNclMin == 6, "the candidates below");
    if (max_clusters<Tin, DH, 8>() >= nh) return 8;
    if (max_clusters<Tin, DH, 7>() >= nh) return 7;
    if (max_clusters<Tin, DH, 6>() >= nh) return 6;
    return 8;
}

template <typename Tin, int DH>
cudaError_t launch_fused(const Tin *q, const Tin *k, const Tin *v, int nh, int T, int W,
                         int cache, float eps, float tau, float *o, float *Hst, float *s,
                         int *kept_pos, float *scratch, int ncl, cudaStream_t stream) {
    if (ncl <= 0) ncl = choose_ncl<Tin, DH>(nh);
    switch (ncl) {
        case 8: return launch_ncl<Tin, DH, 8>(q, k, v, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, stream);
        case 7: return launch_ncl<Tin, DH, 7>(q, k, v, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, stream);
        case 6: return launch_ncl<Tin, DH, 6>(q, k, v, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t fused_dispatch(const void *q, const void *k, const void *v, int nh, int T, int d,
                           int W, int cache, float eps, float tau, float *o, float *Hst,
                           float *s, int *kept_pos, float *scratch, int ncl,
                           cudaStream_t stream) {
    const Tin *qq = static_cast<const Tin *>(q), *kk = static_cast<const Tin *>(k),
              *vv = static_cast<const Tin *>(v);
    switch (d) {
        case 16: return launch_fused<Tin, 16>(qq, kk, vv, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, ncl, stream);
        case 32: return launch_fused<Tin, 32>(qq, kk, vv, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, ncl, stream);
        case 64:
            // fp32 rows of 64 values do not leave room for the staged values
            if constexpr (sizeof(Tin) * 64 <= 128)
                return launch_fused<Tin, 64>(qq, kk, vv, nh, T, W, cache, eps, tau, o, Hst, s, kept_pos, scratch, ncl, stream);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool lola_fused_applies(int dtype, int d, int window, int cache) {
    const int es = dtype == 0 ? 4 : 2;
    return (d == 16 || d == 32 || d == 64) && es * d <= 128 && window % 8 == 0 &&
           window <= kWMax && 2 * window <= kNSMax && 2 * window + cache <= kNKMax &&
           cache >= 0;
}

size_t lola_fused_scratch_bytes(int nh, int d) {
    const size_t f = d == 16 ? fused_scratch_floats<16>() : d == 32 ? fused_scratch_floats<32>()
                                                                    : fused_scratch_floats<64>();
    return align_up((size_t)nh * f * sizeof(float), 256);
}

cudaError_t lola_fused(const void *q, const void *k, const void *v, int dtype, int nh, int T,
                       int d, int window, int cache, float eps, float tau, float *o, float *Hst,
                       float *s, int *kept_pos, void *scratch, int ncl, cudaStream_t stream) {
    KATA_DEBUG_BIND();
    float *sc = static_cast<float *>(scratch);
    if (dtype == 0)
        return fused_dispatch<float>(q, k, v, nh, T, d, window, cache, eps, tau, o, Hst, s,
                                     kept_pos, sc, ncl, stream);
    return fused_dispatch<__nv_bfloat16>(q, k, v, nh, T, d, window, cache, eps, tau, o, Hst, s,
                                         kept_pos, sc, ncl, stream);
}

}  // namespace kata
