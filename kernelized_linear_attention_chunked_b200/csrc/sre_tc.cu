// SRE scoring, top-k retention and merge on the tcgen05 tensor cores, with
// split bf16 operands so that the scores keep fp32-level accuracy.
//
// "LoLA: Low-Rank Linear Attention with Sparse Caching", "Self-Recall Error":
//   SRE_j = || phi(k_j)^T H / (phi(k_j)^T s + eps) - v_j ||^2,
// and its inference strategy (keep the candidates with the highest SRE, fold
// the rest into the state as outer products). phi is the rank-one PSD feature
// of "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
// Cones", s2.2, in the packed layout: row r is the pair (a, b), a <= b, and
// phi(x)_r = w_r x_a x_b with w_r = sqrt(2) off the diagonal.
//
// One CTA per head (bf16 candidates, d = 32 or 64, at most 256 of them):
//  1. Scores. For 32 packed rows at a time, D[m][c] += A[m][r] B[c][r] with
//     A = (w [H | s])^T (m < d: a value column; m = d: the normaliser) and
//     B[c][r] = k_c[a_r] k_c[b_r]. The product of two bf16 values is exact in
//     fp32 and splits exactly into two bf16 parts (hi + lo); w [H | s] splits
//     into hi + lo with a relative residual below 2^-16. Three MMAs per step
//     (hi.hi, hi.lo, lo.hi) accumulate in fp32 tensor memory; what is dropped
//     is below 2^-16 of each term, and the SRE, a distance of order |v|^2, is
//     insensitive to that (1e-7 relative on the synthetic candidates). The
//     state streams from HBM once, in 64-row bulk copies, three in flight.
//  2. The SRE of every candidate from D (numerator lanes, normaliser lane),
//     then the kept set (higher SRE, then smaller position, then slot) in
//     ascending position, and the list of candidates to merge.
//  3. Merge, 128 packed rows at a time: D2[r][e] = sum_m k_m[a_r] k_m[b_r]
//     [v_m | 1][e] with exact products (two bf16 parts times bf16 values and
//     ones), then H[r] += w_r D2[r][0..d-1] and s[r] += w_r D2[r][d] in fp32:
//     the state is read and written once more, as 16-byte accesses.
#include "kata_common.cuh"
#include "kata_internal.h"
#include "sm100.cuh"
#include "tc_tiles.cuh"

namespace kata {
namespace {

using namespace sm100;
using tc::warp_wait;

constexpr int kST = 512;     // threads (16 warps)
constexpr int kKR = 32;      // packed rows per score step (the MMA K extent)
constexpr int kLR = 64;      // packed rows per staging copy
constexpr int kStages = 3;   // staging copies in flight
constexpr int kNMax = 256;   // candidates per head
constexpr int kMR = 128;     // packed rows per merge tile
constexpr int kMK = 32;      // merged candidates per merge step
constexpr float kSqrt2f = 1.41421356237309515f;

// Byte offset of 16-byte chunk `chunk` of row `row` in a K-major tile with
// 64-byte rows (32 bf16 along K) under the 64-byte swizzle: chunk c of row r
// is stored at chunk c ^ ((r >> 1) & 3). Tiles start on a 1024-byte boundary.
__device__ __forceinline__ uint32_t sw64_chunk(int row, int chunk) {
    return (uint32_t)(row * 64 + (((chunk ^ (row >> 1)) & 3) << 4));
}
// Descriptor of such a tile at K-step kk (16 elements, 32 bytes).
__device__ __forceinline__ uint64_t kmaj64_desc(uint32_t base, int kk) {
    return smem_desc(base + 32 * kk, 16, 512, kSwizzle64);
}

__device__ __forceinline__ uint32_t bf16_bits(float x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(x);
    return (uint32_t)*reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float bits_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Eight values -> two 16-byte rows of bf16 parts, x = hi + lo (+ the residual
// of a value with more than 16 significant bits).
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[8], l[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        h[u] = bf16_bits(x[u]);
        l[u] = bf16_bits(x[u] - bits_f32(h[u]));
    }
    hi = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
    lo = make_uint4(l[0] | (l[1] << 16), l[2] | (l[3] << 16), l[4] | (l[5] << 16), l[6] | (l[7] << 16));
}

__device__ __forceinline__ float row_weight(uint16_t ab) {
    return (ab >> 8) != (ab & 255) ? kSqrt2f : 1.f;
}

enum SreBar {
    kBLoad = 0,                 // kStages: a staging copy landed
    kBMma = kBLoad + kStages,   // 2: the score MMAs reading operand buffer i completed
    kBFinal = kBMma + 2,        // every score MMA completed
    kBM2 = kBFinal + 1,         // 2: the merge MMAs reading operand buffer i completed
    kBDrain = kBM2 + 2,         // teardown: every MMA completed
    kBCount = kBDrain + 1
};

template <int DH>
struct SreCfg {
    static constexpr int D = DH * (DH + 1) / 2;
    static constexpr int N2 = DH + 16;                       // merge MMA N: [v | 1 | 0]
    static constexpr int STG = ((kLR * DH + kLR) * 4 + 1023) / 1024 * 1024;
    static constexpr int ATILE = 128 * 64;                   // 128 rows x 32 bf16
    static constexpr int BTILE = kNMax * 64;                 // 256 rows x 32 bf16
    static constexpr int B2TILE = N2 * 64;                   // a multiple of 1024
    static constexpr int OFF_STG = 0;                        // phase 3: k of merged [256][DH]
    static constexpr int OFF_A = OFF_STG + kStages * STG;    // [2 buffers][hi, lo]
    static constexpr int OFF_B = OFF_A + 2 * 2 * ATILE;      // [2 buffers][hi, lo]; phase 3: B2
    static constexpr int OFF_KT = OFF_B + 2 * 2 * BTILE;     // k^T [DH][256] bf16
    static constexpr int OFF_TAB = OFF_KT + DH * kNMax * 2;  // pair of each packed row
    static constexpr int OFF_SC = OFF_TAB + (D * 2 + 15) / 16 * 16;
    static constexpr int OFF_BAR = OFF_SC + 5 * kNMax * 4;   // five per-candidate arrays
    static constexpr int BYTES = OFF_BAR + kBCount * 8 + 16 + 1024;
    static_assert(B2TILE % 1024 == 0, "merge operand tiles stay 1024-aligned");
    static_assert(8 * B2TILE <= 2 * 2 * BTILE, "merge operand fits the score operand area");
    static_assert(kNMax * (DH + 1) * 4 <= 2 * 2 * (ATILE + BTILE), "squared errors fit");
    static_assert(kNMax * DH * 2 <= kStages * STG, "merged keys fit the staging area");
    static_assert(BYTES <= 227 * 1024, "shared memory");
};

template <int DH>
__global__ void __launch_bounds__(kST, 1)
sre_tc_kernel(const float *Hst, const float *s, const __nv_bfloat16 *__restrict__ kc,
              const __nv_bfloat16 *__restrict__ vc, long cand_head_stride,
              const int *__restrict__ pos, long pos_head_stride, int n, int keep, float eps,
              int merge, float *__restrict__ scores, int *__restrict__ keep_idx,
              float *Hst_mut, float *s_mut, unsigned int *errw) {
    using L = SreCfg<DH>;
    constexpr int D = L::D;
    constexpr int NCH = (D + kKR - 1) / kKR;  // score steps
    constexpr int NL = (D + kLR - 1) / kLR;   // staging copies
    constexpr int N2 = L::N2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::OFF_BAR + kBCount * 8);
    uint16_t *kT = reinterpret_cast<uint16_t *>(sm + L::OFF_KT);
    uint16_t *tab = reinterpret_cast<uint16_t *>(sm + L::OFF_TAB);
    float *sc = reinterpret_cast<float *>(sm + L::OFF_SC);
    float *den = sc + kNMax;
    int *cpos = reinterpret_cast<int *>(den + kNMax);
    int *kflag = cpos + kNMax;
    int *mlist = kflag + kNMax;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int NP = (n + 15) & ~15;  // score MMA N: candidates padded to 16
    const ErrCtx err{errw};
    const float *Hh = Hst + (size_t)h * D * DH;
    const float *sh = s + (size_t)h * D;
    const __nv_bfloat16 *kh = kc + (size_t)h * cand_head_stride;
    const __nv_bfloat16 *vh = vc + (size_t)h * cand_head_stride;

    if (tid == 0) {
        for (int i = 0; i < kBCount; ++i) mbar_init(&bar[i], 1);
        cta_abort_clear();
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    int issued = 0;  // staging copies issued (thread 0)
    auto issue_load = [&](int j) {
        const int r0 = j * kLR, rows = D - r0 < kLR ? D - r0 : kLR;
        uint8_t *dst = sm + L::OFF_STG + (j % kStages) * L::STG;
        const uint32_t hb = (uint32_t)(rows * DH * 4), sb = (uint32_t)(rows * 4);
        mbar_arrive_expect_tx(&bar[kBLoad + j % kStages], hb + sb);
        bulk_load(dst, Hh + (size_t)r0 * DH, hb, &bar[kBLoad + j % kStages]);
        bulk_load(dst + kLR * DH * 4, sh + r0, sb, &bar[kBLoad + j % kStages]);
        ++issued;
    };
    __syncthreads();  // barriers initialised
    if (tid == 0)
        for (int j = 0; j < kStages && j < NL; ++j) issue_load(j);
    // pair table; k^T with zeros past n; rows d+1 .. 127 of the A operands are
    // zero in both buffers and both parts
    for (int r = tid; r < D; r += kST) {
        int a = 0;
        while (packed_row_base(a + 1, DH) <= r) ++a;
        tab[r] = (uint16_t)((a << 8) | (a + r - packed_row_base(a, DH)));
    }
    for (int idx = tid; idx < kNMax * DH; idx += kST) {
        const int c = idx / DH, a = idx % DH;
        kT[a * kNMax + c] = c < n ? reinterpret_cast<const uint16_t *>(kh)[(size_t)c * DH + a] : 0;
    }
    {
        constexpr int z0 = (DH + 1) * 64, zq = (L::ATILE - z0) / 16;
        for (int idx = tid; idx < 4 * zq; idx += kST)
            *reinterpret_cast<uint4 *>(sm + L::OFF_A + (idx / zq) * L::ATILE + z0 +
                                       (idx % zq) * 16) = make_uint4(0, 0, 0, 0);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    // ---------------- 1. scores ----------------
    const uint32_t id_s = idesc_bf16(128, NP, 0, 0);
    bool ok = true;
    for (int i = 0; i < NCH; ++i) {
        const int j = i >> 1, half = i & 1, buf = i & 1;
        const float *stg = reinterpret_cast<const float *>(sm + L::OFF_STG + (j % kStages) * L::STG);
        uint8_t *Ah = sm + L::OFF_A + buf * 2 * L::ATILE, *Al = Ah + L::ATILE;
        uint8_t *Bh = sm + L::OFF_B + buf * 2 * L::BTILE, *Bl = Bh + L::BTILE;
        // this step's rows have landed; the MMAs of step i - 2 (the last
        // readers of operand buffer buf) have completed
        ok = warp_wait(&bar[kBLoad + j % kStages], (j / kStages) & 1, err, 0x701) && ok;
        if (i >= 2) ok = warp_wait(&bar[kBMma + buf], ((i - 2) >> 1) & 1, err, 0x702) && ok;
        // A: row m (a value column, or the normaliser at m = DH), 8 packed rows
        // per task
        for (int idx = tid; idx < 4 * (DH + 1); idx += kST) {
            const int m = idx < 4 * DH ? idx % DH : DH;
            const int kg = idx < 4 * DH ? idx / DH : idx - 4 * DH;
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int rr = kg * 8 + u, r = i * kKR + rr, lr = half * kKR + rr;
                x[u] = r < D ? row_weight(tab[r]) * (m < DH ? stg[lr * DH + m] : stg[kLR * DH + lr])
                             : 0.f;
            }
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4 *>(Ah + sw64_chunk(m, kg)) = hi;
            *reinterpret_cast<uint4 *>(Al + sw64_chunk(m, kg)) = lo;
        }
        // B: row c (a candidate), 8 packed rows of k_c[a] k_c[b] per task
        for (int idx = tid; idx < 4 * NP; idx += kST) {
            const int c = idx % NP, kg = idx / NP;
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = i * kKR + kg * 8 + u;
                float p = 0.f;
                if (r < D) {
                    const int ab = tab[r];
                    p = bits_f32(kT[(ab >> 8) * kNMax + c]) * bits_f32(kT[(ab & 255) * kNMax + c]);
                }
                x[u] = p;
            }
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4 *>(Bh + sw64_chunk(c, kg)) = hi;
            *reinterpret_cast<uint4 *>(Bl + sw64_chunk(c, kg)) = lo;
        }
        fence_proxy_async_smem();
        ok = bar_sync_and(1, kST, ok);
        if (!ok) break;
        if (tid == 0) {
            // both halves of staging copy j are converted: refill its buffer
            if (half == 1 && j + kStages < NL) issue_load(j + kStages);
            tc_fence_after();
            const uint32_t ah = smem_u32(Ah), al = smem_u32(Al);
            const uint32_t bh = smem_u32(Bh), bl = smem_u32(Bl);
#pragma unroll
            for (int kk = 0; kk < kKR / 16; ++kk) {
                mma_ss(tmem, kmaj64_desc(ah, kk), kmaj64_desc(bh, kk), id_s, (i > 0 || kk > 0) ? 1u : 0u);
                mma_ss(tmem, kmaj64_desc(ah, kk), kmaj64_desc(bl, kk), id_s, 1u);
                mma_ss(tmem, kmaj64_desc(al, kk), kmaj64_desc(bh, kk), id_s, 1u);
            }
            mma_commit(&bar[kBMma + buf]);
        }
    }
    if (tid == 0) mma_commit(&bar[kBFinal]);
    ok = warp_wait(&bar[kBFinal], 0, err, 0x703) && ok;
    tc_fence_after();
    ok = bar_sync_and(1, kST, ok);

    // ---------------- 2. SRE and the kept set ----------------
    const int m_keep = keep < n ? keep : n;
    const int nm = n - m_keep;
    if (ok) {
        if (warp == DH / 32) {  // tensor-memory lane DH: the normaliser of every candidate
            for (int c0 = 0; c0 < NP; c0 += 16) {
                uint32_t r16[16];
                tmem_ld16(tmem + lane_base + c0, r16);
                tmem_ld_wait();
                if (lane == 0)
#pragma unroll
                    for (int u = 0; u < 16; ++u) den[c0 + u] = __uint_as_float(r16[u]);
            }
        }
        __syncthreads();
        // squared differences, one value column per thread of warps 0 .. DH/32 - 1,
        // staged as sq[c][e] (pitch DH + 1) over the free operand buffers
        float *sq = reinterpret_cast<float *>(sm + L::OFF_A);
        if (warp < DH / 32) {
            const int e = tid;
            for (int c0 = 0; c0 < NP; c0 += 16) {
                uint32_t r16[16];
                tmem_ld16(tmem + lane_base + c0, r16);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int c = c0 + u;
                    if (c < n) {
                        const float diff = __uint_as_float(r16[u]) / (den[c] + eps) -
                                           __bfloat162float(vh[(size_t)c * DH + e]);
                        sq[c * (DH + 1) + e] = diff * diff;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid < n) {
            float acc = 0.f;
            for (int e = 0; e < DH; ++e) acc += sq[tid * (DH + 1) + e];
            sc[tid] = isnan(acc) ? -INFINITY : acc;  // a total order even for 0/0 scores
            cpos[tid] = pos[(size_t)h * pos_head_stride + tid];
            if (scores) scores[(size_t)h * n + tid] = sc[tid];
        }
        __syncthreads();
        if (tid < n) {
            const float si = sc[tid];
            const int pi = cpos[tid];
            int rank = 0;
            for (int c = 0; c < n; ++c) {
                const float sj = sc[c];
                const int pj = cpos[c];
                rank += sj > si || (sj == si && (pj < pi || (pj == pi && c < tid)));
            }
            kflag[tid] = rank < m_keep;
        }
        __syncthreads();
        if (tid < n) {
            const int pi = cpos[tid];
            if (kflag[tid]) {
                int pr = 0;
                for (int c = 0; c < n; ++c)
                    pr += kflag[c] && (cpos[c] < pi || (cpos[c] == pi && c < tid));
                if (pr < m_keep) keep_idx[(size_t)h * m_keep + pr] = tid;
            } else {
                int mr = 0;
                for (int c = 0; c < tid; ++c) mr += !kflag[c];
                mlist[mr] = tid;
            }
        }
        __syncthreads();
    }

    // ---------------- 3. merge ----------------
    if (ok && merge && nm > 0) {
        const int nk2 = (nm + kMK - 1) / kMK;
        constexpr int NT2 = (D + kMR - 1) / kMR;
        // keys of the merged candidates, row-major [mi][DH], zero past nm
        uint16_t *kM = reinterpret_cast<uint16_t *>(sm + L::OFF_STG);
        for (int idx = tid; idx < nk2 * kMK * DH; idx += kST) {
            const int mi = idx / DH, a = idx % DH;
            kM[idx] = mi < nm ? reinterpret_cast<const uint16_t *>(kh)[(size_t)mlist[mi] * DH + a] : 0;
        }
        // B2 (K-major), step q: row e < DH is v[e] of merged candidates
        // 32 q .. 32 q + 31, row DH is 1, rows above are 0 (zero past nm)
        uint8_t *B2 = sm + L::OFF_B;
        for (int idx = tid; idx < nk2 * N2 * 4; idx += kST) {
            const int q = idx / (N2 * 4), rem = idx % (N2 * 4);
            const int kg = rem / N2, e = rem % N2;
            uint32_t b[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int mi = q * kMK + kg * 8 + u;
                uint32_t val = 0;
                if (mi < nm) {
                    if (e < DH)
                        val = reinterpret_cast<const uint16_t *>(vh)[(size_t)mlist[mi] * DH + e];
                    else if (e == DH)
                        val = 0x3F80u;  // 1.0 in bf16
                }
                b[u] = val;
            }
            *reinterpret_cast<uint4 *>(B2 + q * L::B2TILE + sw64_chunk(e, kg)) =
                make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16),
                           b[6] | (b[7] << 16));
        }
        __syncthreads();  // the merged keys are read by other threads below
        const uint32_t id_m = idesc_bf16(128, N2, 0, 0);
        // epilogue share of each thread: tile row 32 (warp % 4) + lane, the
        // column group warp / 4 (16 columns at DH = 64, 8 at 32)
        constexpr int EC = DH / 4;
        const int cg = warp >> 2;
        float4 hreg[EC / 4];
        float sreg = 0.f;
        const int nsteps = NT2 * nk2;
        for (int st = 0; st < nsteps; ++st) {
            const int t = st / nk2, q = st % nk2, buf = st & 1;
            const int row = t * kMR + (warp & 3) * 32 + lane;
            if (q == 0 && row < D) {  // this tile's state, read early
                const float4 *src = reinterpret_cast<const float4 *>(Hh + (size_t)row * DH + cg * EC);
#pragma unroll
                for (int u = 0; u < EC / 4; ++u) hreg[u] = src[u];
                if (cg == 0) sreg = sh[row];
            }
            uint8_t *Ah = sm + L::OFF_A + buf * 2 * L::ATILE, *Al = Ah + L::ATILE;
            if (st >= 2) ok = warp_wait(&bar[kBM2 + buf], ((st - 2) >> 1) & 1, err, 0x704) && ok;
            {   // A2: tile row rr, merged candidates 32 q + 8 kg .. +7 (kg warp-uniform)
                const int rr = tid & 127, kg = tid >> 7;
                const int r = t * kMR + rr;
                float x[8];
                int a = 0, b = 0;
                if (r < D) {
                    const int ab = tab[r];
                    a = ab >> 8;
                    b = ab & 255;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int mi = q * kMK + kg * 8 + u;
                    x[u] = r < D ? bits_f32(kM[mi * DH + a]) * bits_f32(kM[mi * DH + b]) : 0.f;
                }
                uint4 hi, lo;
                split8(x, hi, lo);
                *reinterpret_cast<uint4 *>(Ah + sw64_chunk(rr, kg)) = hi;
                *reinterpret_cast<uint4 *>(Al + sw64_chunk(rr, kg)) = lo;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            ok = bar_sync_and(1, kST, ok);
            if (!ok) break;
            if (tid == 0) {
                tc_fence_after();
                const uint32_t ah = smem_u32(Ah), al = smem_u32(Al);
                const uint32_t b2 = smem_u32(B2 + q * L::B2TILE);
#pragma unroll
                for (int kk = 0; kk < kMK / 16; ++kk) {
                    mma_ss(tmem, kmaj64_desc(ah, kk), kmaj64_desc(b2, kk), id_m, (q > 0 || kk > 0) ? 1u : 0u);
                    mma_ss(tmem, kmaj64_desc(al, kk), kmaj64_desc(b2, kk), id_m, 1u);
                }
                mma_commit(&bar[kBM2 + buf]);
            }
            if (q == nk2 - 1) {  // H[r] += w_r D2[r], s[r] += w_r D2[r][DH]
                ok = warp_wait(&bar[kBM2 + buf], (st >> 1) & 1, err, 0x705) && ok;
                tc_fence_after();
                uint32_t v16[16], s16[16];
                tmem_ld16(tmem + lane_base + cg * EC, v16);
                if (cg == 0) tmem_ld16(tmem + lane_base + DH, s16);
                tmem_ld_wait();
                if (ok && row < D) {
                    const float w = row_weight(tab[row]);
                    float4 *dst = reinterpret_cast<float4 *>(Hst_mut + ((size_t)h * D + row) * DH + cg * EC);
#pragma unroll
                    for (int u = 0; u < EC / 4; ++u) {
                        float4 x = hreg[u];
                        x.x = fmaf(w, __uint_as_float(v16[4 * u + 0]), x.x);
                        x.y = fmaf(w, __uint_as_float(v16[4 * u + 1]), x.y);
                        x.z = fmaf(w, __uint_as_float(v16[4 * u + 2]), x.z);
                        x.w = fmaf(w, __uint_as_float(v16[4 * u + 3]), x.w);
                        dst[u] = x;
                    }
                    if (cg == 0) s_mut[(size_t)h * D + row] = fmaf(w, __uint_as_float(s16[0]), sreg);
                }
                tc_fence_before();
            }
        }
    }

    // teardown: every copy and MMA this CTA issued has completed
    if (tid == 0) {
        for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
            mbar_drain(&bar[kBLoad + j % kStages], (j / kStages) & 1, err, 0x706);
        mma_commit(&bar[kBDrain]);
        mbar_drain(&bar[kBDrain], 0, err, 0x707);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <int DH>
cudaError_t launch(const float *Hst, const float *s, const __nv_bfloat16 *kc,
                   const __nv_bfloat16 *vc, const int *pos, int nh, int n, int cand_stride,
                   int keep, float eps, int merge, float *scores, int *keep_idx, float *Hst_mut,
                   float *s_mut, unsigned int *err, cudaStream_t stream) {
    const int bytes = SreCfg<DH>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(sre_tc_kernel<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    sre_tc_kernel<DH><<<nh, kST, bytes, stream>>>(Hst, s, kc, vc, (long)cand_stride * DH, pos,
                                                  cand_stride, n, keep, eps, merge, scores,
                                                  keep_idx, Hst_mut, s_mut, err);
    return after_launch();
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool sre_tc_applies(int dtype, int d, int n, const float *Hst, const float *s,
                    const float *Hst_mut, const float *s_mut) {
    return dtype == 1 && (d == 32 || d == 64) && n >= 1 && n <= kNMax && aligned16(Hst) &&
           aligned16(s) && aligned16(Hst_mut) && aligned16(s_mut);
}

cudaError_t sre_tc(const float *Hst, const float *s, const void *kc, const void *vc,
                   const int *pos, int nh, int d, int n, int cand_stride, int keep, float eps,
                   int merge, float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                   unsigned int *err, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const bf *k = static_cast<const bf *>(kc), *v = static_cast<const bf *>(vc);
    cudaError_t e;
    if (d == 64)
        e = launch<64>(Hst, s, k, v, pos, nh, n, cand_stride, keep, eps, merge, scores, keep_idx,
                       Hst_mut, s_mut, err, stream);
    else if (d == 32)
        e = launch<32>(Hst, s, k, v, pos, nh, n, cand_stride, keep, eps, merge, scores, keep_idx,
                       Hst_mut, s_mut, err, stream);
    else
        return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    if (merge && keep >= n && (Hst_mut != Hst || s_mut != s)) {  // nothing to merge: copy through
        const size_t D = (size_t)d * (d + 1) / 2;
        if ((e = cudaMemcpyAsync(Hst_mut, Hst, (size_t)nh * D * d * 4, cudaMemcpyDeviceToDevice,
                                 stream)) != cudaSuccess)
            return e;
        e = cudaMemcpyAsync(s_mut, s, (size_t)nh * D * 4, cudaMemcpyDeviceToDevice, stream);
    }
    return e;
}

}  // namespace kata
