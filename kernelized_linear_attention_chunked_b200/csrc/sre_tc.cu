// SRE scoring, top-k retention and merge on the tcgen05 tensor cores.
//
// "LoLA: Low-Rank Linear Attention with Sparse Caching", "Self-Recall Error":
//   SRE_j = || phi(k_j)^T H / (phi(k_j)^T s + eps) - v_j ||^2,
// and its inference strategy (keep the candidates with the highest SRE, fold
// the rest into the state as outer products). phi is the rank-one PSD feature
// of "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
// Cones", s2.2, in the packed layout: row r is the pair (a, b), a <= b, and
// phi(x)_r = w_r x_a x_b with w_r = sqrt(2) off the diagonal.
//
// Scores as a quadratic form. With U_a[m][b] = w_(a,b) [H | s][r(a, b)][m] for
// b >= a (zero for b < a),
//   phi(k)^T [H | s][:, m] = sum_a k[a] sum_b k[b] U_a[m][b],
// so for every a one MMA D_a[c][m] = sum_b k_c[b] U_a[m][b] takes the bf16
// candidate keys as they are (exact) and U_a split into two bf16 parts
// (hi + lo, relative residual below 2^-16), and the epilogue accumulates
// k_c[a] D_a[c][m] in fp32 registers. Every state value is converted once, and
// the state streams from HBM once. The SRE is a distance of order |v|^2 and
// keeps fp32-level accuracy (1e-7 relative on the synthetic candidates).
//
// Merge, 128 packed rows at a time: D2[r][e] = sum_m k_m[a_r] k_m[b_r]
// [v_m | 1][e] with exact products (the product of two bf16 values splits
// exactly into two bf16 parts), then H[r] += w_r D2[r][0..d-1] and
// s[r] += w_r D2[r][d] in fp32, added by bulk reductions (the bulk-copy
// engine reads the update from shared memory and adds it in L2). The kernel
// merges in place; the host copies the state first for an out-of-place call.
//
// One CTA per head (bf16 candidates, d = 32 or 64, at most 256 of them), 32
// warps in four roles that hand work over through mbarrier rings (every wait
// bounded): 16 epilogue warps (warp w reads tensor-memory lanes 32 (w % 4) ..
// and a quarter of the columns), 14 builder warps (operand conversion), a
// producer warp (bulk copies of the state) and an MMA warp (one lane issues).
// Conversion, MMAs and epilogues of consecutive indices overlap.
#include "kata_common.cuh"
#include "kata_internal.h"
#include "sm100.cuh"
#include "tc_tiles.cuh"

namespace kata {
namespace {

using namespace sm100;
using tc::warp_wait;

constexpr int kEpiWarps = 16;           // epilogue warps: TMEM lane quadrant x column group
constexpr int kBuildWarps = 14;         // operand builder warps
constexpr int kEpi = kEpiWarps * 32;
constexpr int kBuild = kBuildWarps * 32;
constexpr int kProducerWarp = kEpiWarps + kBuildWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kLR = 64;                 // packed rows per staging copy
constexpr int kNMax = 256;              // candidates per head
constexpr int kMR = 128;                // packed rows per merge tile
constexpr int kMK = 32;                 // merged candidates per merge K chunk
constexpr int kNB = 3;                  // U_a operand buffers
constexpr int kND = 3;                  // D_a accumulators in tensor memory
constexpr int kNA = 2;                  // merge operand buffers
constexpr int kStSlots = 10;            // staging copies in flight, at most
constexpr int kKmtPitch = 264;          // merged keys, transposed: row pitch (bank spread)
constexpr float kSqrt2f = 1.41421356237309515f;

// K-major operand tiles with RB-byte rows (RB = 128: 128-byte swizzle, RB =
// 64: 64-byte swizzle): byte offset of 16-byte chunk `chunk` of row `row`, and
// the descriptor at K-step ks (16 elements, 32 bytes). Tiles start on a
// 1024-byte boundary.
template <int RB>
__device__ __forceinline__ uint32_t kmaj_off(int row, int chunk) {
    if constexpr (RB == 128)
        return (uint32_t)(row * 128 + (((chunk ^ row) & 7) << 4));
    else
        return (uint32_t)(row * 64 + (((chunk ^ (row >> 1)) & 3) << 4));
}
template <int RB>
__device__ __forceinline__ uint64_t kmaj_desc_rb(uint32_t base, int ks) {
    return smem_desc(base + 32 * ks, 16, RB * 8, RB == 128 ? kSwizzle128 : kSwizzle64);
}

// Eight values -> two 16-byte rows of bf16 parts, x = hi + lo (+ the residual
// of a value with more than 16 significant bits); pairs convert together.
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        h[p] = pack_bf16x2(x[2 * p], x[2 * p + 1]);
        l[p] = pack_bf16x2(x[2 * p] - __uint_as_float(h[p] << 16),
                           x[2 * p + 1] - __uint_as_float(h[p] & 0xFFFF0000u));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// The two bf16 values of a packed pair as fp32.
__device__ __forceinline__ float lo_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float row_weight(uint16_t ab) {
    return (ab >> 8) != (ab & 255) ? kSqrt2f : 1.f;
}

// Hint: bring [p, p + bytes) into L2 (16-byte aligned, a multiple of 16 bytes).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
                 "r"(bytes)
                 : "memory");
}

// dst (global) += src (shared), elementwise fp32, by the bulk-copy engine; the
// reduction runs in L2. Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_reduce_add_f32(float *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(dst)),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// At most one bulk group of this thread is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_one() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// 32 lanes x 8 or 1 consecutive 32-bit tensor-memory columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t &r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}

enum SreBar {
    kStFull = 0,                     // kStSlots: a staging copy landed (tx count)
    kStEmpty = kStFull + kStSlots,   // kStSlots: every builder warp is done with a copy
    kBbFull = kStEmpty + kStSlots,   // kNB: U_a written (builder warps)
    kBbEmpty = kBbFull + kNB, // kNB: the MMAs reading U_a completed
    kDFull = kBbEmpty + kNB,  // kND: D_a complete
    kDEmpty = kDFull + kND,   // kND: D_a read (epilogue warps)
    kA2Full = kDEmpty + kND,  // kNA: a merge operand chunk written (builder warps)
    kA2Empty = kA2Full + kNA, // kNA: the MMAs reading it completed
    kD2Full = kA2Empty + kNA, // 2: a merge tile's D2 complete
    kD2Empty = kD2Full + 2,   // 2: D2 read (epilogue warps)
    kDrain = kD2Empty + 2,    // teardown: every MMA completed
    kBarCount = kDrain + 1
};

template <int DH>
struct SreCfg {
    static constexpr int D = DH * (DH + 1) / 2;
    static constexpr int RB = 2 * DH;           // K-major rows of DH bf16
    static constexpr int KS = DH / 16;          // K-steps over b
    static constexpr int NCH = DH / 8;          // 16-byte chunks per row
    static constexpr int N1 = DH + 16;          // score MMA N: [H | s | 0] columns
    static constexpr int N2 = DH + 16;          // merge MMA N: [v | 1 | 0]
    static constexpr int EC = DH / 4;           // epilogue columns per epilogue warp
    static constexpr int NST = DH == 64 ? 6 : 10;
    static constexpr int NL = (D + kLR - 1) / kLR;  // staging copies
    static constexpr int STG = ((kLR * DH + kLR) * 4 + 1023) / 1024 * 1024;
    static constexpr int KA_BYTES = kNMax * RB;
    static constexpr int BPART = (N1 * RB + 1023) / 1024 * 1024;
    static constexpr int A2PART = kMR * 64;
    static constexpr int B2TILE = N2 * 64;
    static constexpr int OFF_KA = 0;
    static constexpr int OFF_STG = OFF_KA + KA_BYTES;
    static constexpr int OFF_BB = OFF_STG + NST * STG;  // [kNB][hi, lo]
    // merge: two images of a tile's state update (w_r D2, rows of DH then the
    // normaliser column), over the key operand and the staging copies, then B2,
    // the A2 ring and the transposed merged keys
    static constexpr int DHB = (kMR * DH * 4 + kMR * 4 + 1023) / 1024 * 1024;
    static constexpr int OFF_DH = OFF_KA;
    static constexpr int OFF_B2 = OFF_DH + 2 * DHB;
    static constexpr int OFF_A2 = OFF_B2 + (kNMax / kMK) * B2TILE;  // [kNA][hi, lo]
    static constexpr int OFF_KMT = OFF_A2 + kNA * 2 * A2PART;  // merge: keys [DH][kKmtPitch]
    static constexpr int OFF_TAB = OFF_BB + kNB * 2 * BPART;
    static constexpr int OFF_SC = OFF_TAB + (D * 2 + 15) / 16 * 16;
    static constexpr int OFF_BAR = OFF_SC + 9 * kNMax * 4;  // 5 arrays + 4 partial sums
    static constexpr int BYTES = OFF_BAR + kBarCount * 8 + 16 + 1024;
    static_assert(NST <= kStSlots, "barrier slots");
    static_assert(B2TILE % 1024 == 0 && BPART % 1024 == 0 && STG % 1024 == 0, "alignment");
    static_assert(OFF_KMT + DH * kKmtPitch * 2 <= OFF_TAB, "merge operands fit");
    static_assert(BYTES <= 227 * 1024, "shared memory");
    static_assert(kND * 2 * N1 <= 512 && 128 + N2 <= 512, "tensor memory");
};

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
sre_tc_kernel(const float *Hst, const float *s, const __nv_bfloat16 *__restrict__ kc,
              const __nv_bfloat16 *__restrict__ vc, long cand_head_stride,
              const int *__restrict__ pos, long pos_head_stride, int n, int keep, float eps,
              int merge, float *__restrict__ scores, int *__restrict__ keep_idx,
              float *Hst_mut, float *s_mut, unsigned int *errw) {
    using L = SreCfg<DH>;
    constexpr int D = L::D, RB = L::RB, N1 = L::N1, N2 = L::N2, EC = L::EC, NST = L::NST;
    constexpr int NL = L::NL;
    constexpr int NT2 = (D + kMR - 1) / kMR;  // merge tiles
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::OFF_BAR + kBarCount * 8);
    uint8_t *KA = sm + L::OFF_KA;
    uint16_t *tab = reinterpret_cast<uint16_t *>(sm + L::OFF_TAB);
    float *sc = reinterpret_cast<float *>(sm + L::OFF_SC);
    float *den = sc + kNMax;
    int *cpos = reinterpret_cast<int *>(den + kNMax);
    int *kflag = cpos + kNMax;
    int *mlist = kflag + kNMax;
    float *sqp = reinterpret_cast<float *>(mlist + kNMax);  // [4][256]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int nmt = n > 128 ? 2 : 1;  // 128-candidate M tiles
    const ErrCtx err{errw};
    const float *Hh = Hst + (size_t)h * D * DH;
    const float *sh = s + (size_t)h * D;
    const __nv_bfloat16 *kh = kc + (size_t)h * cand_head_stride;
    const __nv_bfloat16 *vh = vc + (size_t)h * cand_head_stride;
    const bool epi = warp < kEpiWarps;
    const bool builder = warp >= kEpiWarps && warp < kEpiWarps + kBuildWarps;
    const int btid = tid - kEpi;                   // builder thread index
    const int qd = warp & 3, g = (warp >> 2) & 3;  // epilogue: lane quadrant, column group
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;

    // ---------------- set-up ----------------
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&bar[kStFull + i], 1);
            mbar_init(&bar[kStEmpty + i], kBuildWarps);
        }
        for (int i = 0; i < kNB; ++i) {
            mbar_init(&bar[kBbFull + i], kBuildWarps);
            mbar_init(&bar[kBbEmpty + i], 1);
        }
        for (int i = 0; i < kND; ++i) {
            mbar_init(&bar[kDFull + i], 1);
            mbar_init(&bar[kDEmpty + i], kEpiWarps);
        }
        for (int i = 0; i < kNA; ++i) {
            mbar_init(&bar[kA2Full + i], kBuildWarps);
            mbar_init(&bar[kA2Empty + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[kD2Full + i], 1);
            mbar_init(&bar[kD2Empty + i], kEpiWarps);
        }
        mbar_init(&bar[kDrain], 1);
        cta_abort_clear();
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    build_pair_table(tab, DH);
    if (epi || builder) {
        constexpr int nt = kEpi + kBuild;
        // candidate keys as the score MMA's A operand (zero rows past n)
        for (int idx = tid; idx < nmt * 128 * L::NCH; idx += nt) {
            const int c = idx / L::NCH, ch = idx % L::NCH;
            uint4 x = make_uint4(0, 0, 0, 0);
            if (c < n) x = *reinterpret_cast<const uint4 *>(kh + (size_t)c * DH + ch * 8);
            *reinterpret_cast<uint4 *>(KA + kmaj_off<RB>(c, ch)) = x;
        }
        // rows DH + 1 .. N1 - 1 of every U_a buffer and part stay zero
        constexpr int zrows = N1 - DH - 1;
        for (int idx = tid; idx < kNB * 2 * zrows * L::NCH; idx += nt) {
            const int part = idx / (zrows * L::NCH), rem = idx % (zrows * L::NCH);
            const int row = DH + 1 + rem / L::NCH, ch = rem % L::NCH;
            *reinterpret_cast<uint4 *>(sm + L::OFF_BB + part * L::BPART + kmaj_off<RB>(row, ch)) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    int issued = 0;  // staging copies issued (producer warp)

    // ---------------- 1. scores ----------------
    float acc[2][EC];
    float sacc[2] = {0.f, 0.f};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int i = 0; i < EC; ++i) acc[mt][i] = 0.f;

    if (warp == kProducerWarp) {
        for (int st = 0; st < NL; ++st) {
            const int slot = st % NST, use = st / NST;
            if (use >= 1) ok = warp_wait(&bar[kStEmpty + slot], (use - 1) & 1, err, 0x711) && ok;
            if (!ok) break;
            if (lane == 0) {
                const int r0 = st * kLR, rows = D - r0 < kLR ? D - r0 : kLR;
                uint8_t *dst = sm + L::OFF_STG + slot * L::STG;
                const uint32_t hb = (uint32_t)(rows * DH * 4), sb = (uint32_t)(rows * 4);
                mbar_arrive_expect_tx(&bar[kStFull + slot], hb + sb);
                bulk_load(dst, Hh + (size_t)r0 * DH, hb, &bar[kStFull + slot]);
                bulk_load(dst + kLR * DH * 4, sh + r0, sb, &bar[kStFull + slot]);
            }
            ++issued;
            __syncwarp();
        }
    } else if (warp == kMmaWarp) {
        const uint32_t id1 = idesc_bf16(128, N1, 0, 0);
        const uint32_t ka0 = smem_u32(KA);
        for (int a = 0; a < DH; ++a) {
            const int i = a % kNB, j = a % kND;
            ok = warp_wait(&bar[kBbFull + i], (a / kNB) & 1, err, 0x712) && ok;
            if (a >= kND) ok = warp_wait(&bar[kDEmpty + j], ((a / kND) - 1) & 1, err, 0x713) && ok;
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t bh = smem_u32(sm + L::OFF_BB + i * 2 * L::BPART), bl = bh + L::BPART;
                const int ks0 = a / 16;
                for (int mt = 0; mt < nmt; ++mt) {
                    const uint32_t d = tmem + (uint32_t)((j * nmt + mt) * N1);
                    const uint32_t ka = ka0 + (uint32_t)(mt * 128 * RB);
                    for (int ks = ks0; ks < L::KS; ++ks) {
                        mma_ss(d, kmaj_desc_rb<RB>(ka, ks), kmaj_desc_rb<RB>(bh, ks), id1,
                               ks > ks0 ? 1u : 0u);
                        mma_ss(d, kmaj_desc_rb<RB>(ka, ks), kmaj_desc_rb<RB>(bl, ks), id1, 1u);
                    }
                }
                mma_commit(&bar[kBbEmpty + i]);
                mma_commit(&bar[kDFull + j]);
            }
            __syncwarp();
        }
    } else if (builder) {
        int waited = 0, released = 0;  // staging copies waited for / released (warp-uniform)
        for (int a = 0; a < DH && ok; ++a) {  // U_a: rows m (value columns, the normaliser), K = b
            const int i = a % kNB;
            const int first = packed_row_base(a, DH), last = first + DH - 1 - a;
            while (waited <= last / kLR && ok) {
                ok = warp_wait(&bar[kStFull + waited % NST], (waited / NST) & 1, err, 0x714) && ok;
                ++waited;
            }
            if (a >= kNB) ok = warp_wait(&bar[kBbEmpty + i], ((a / kNB) - 1) & 1, err, 0x715) && ok;
            if (!ok) break;
            uint8_t *Bh = sm + L::OFF_BB + i * 2 * L::BPART, *Bl = Bh + L::BPART;
            const int ch0 = (a / 16) * 2, ntask = (DH + 1) * (L::NCH - ch0);
            for (int idx = btid; idx < ntask; idx += kBuild) {
                const int m = idx % (DH + 1), ch = ch0 + idx / (DH + 1);
                // rows of b = 8 ch .. 8 ch + 7 (those with b < a are zero):
                // consecutive packed rows, in at most two staging copies
                const int b0 = ch * 8, rs = first + (b0 > a ? b0 - a : 0);
                const int st0 = rs / kLR, lr0 = rs - st0 * kLR;
                const float *p0 = reinterpret_cast<const float *>(sm + L::OFF_STG + (st0 % NST) * L::STG);
                float x[8];
                if (b0 > a && lr0 + 7 < kLR) {
                    // common case: eight rows of one staging copy, all off the diagonal
                    if (m < DH) {
                        const float *pp = p0 + lr0 * DH + m;
#pragma unroll
                        for (int u = 0; u < 8; ++u) x[u] = kSqrt2f * pp[u * DH];
                    } else {
                        const float *pp = p0 + kLR * DH + lr0;
#pragma unroll
                        for (int u = 0; u < 8; ++u) x[u] = kSqrt2f * pp[u];
                    }
                } else {
                    const float *p1 = reinterpret_cast<const float *>(sm + L::OFF_STG + ((st0 + 1) % NST) * L::STG);
                    const int col = m < DH ? m : kLR * DH;  // value column, or the normaliser
                    const int rstride = m < DH ? DH : 1;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int b = b0 + u, bb = b > a ? b : a;  // rows b < a are not read
                        const int lr = first + bb - a - st0 * kLR;  // row inside copy st0 (or past it)
                        const float *pp = lr < kLR ? p0 + lr * rstride : p1 + (lr - kLR) * rstride;
                        const float val = pp[col];
                        x[u] = b > a ? kSqrt2f * val : (b == a ? val : 0.f);
                    }
                }
                uint4 hi, lo;
                split8(x, hi, lo);
                *reinterpret_cast<uint4 *>(Bh + kmaj_off<RB>(m, ch)) = hi;
                *reinterpret_cast<uint4 *>(Bl + kmaj_off<RB>(m, ch)) = lo;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kBbFull + i]);
            // staging copies whose rows all come before the next index
            const int lim = a == DH - 1 ? NL : packed_row_base(a + 1, DH) / kLR;
            for (; released < lim; ++released)
                if (lane == 0) mbar_arrive(&bar[kStEmpty + released % NST]);
        }
    } else if (epi) {
        for (int a = 0; a < DH && ok; ++a) {  // acc += k_c[a] D_a[c][columns of this warp]
            const int j = a % kND;
            ok = warp_wait(&bar[kDFull + j], (a / kND) & 1, err, 0x716) && ok;
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                if (mt >= nmt) break;
                if (mt * 128 + qd * 32 >= n) continue;  // no candidate in these lanes
                const uint32_t col = (uint32_t)((j * nmt + mt) * N1);
                uint32_t v[EC], sv = 0u;
                if constexpr (EC == 16) tmem_ld16(tmem + lane_base + col + EC * g, v);
                else tmem_ld8(tmem + lane_base + col + EC * g, v);
                if (g == 0) tmem_ld1(tmem + lane_base + col + DH, sv);
                const int c = mt * 128 + qd * 32 + lane;
                const uint16_t kb = *reinterpret_cast<const uint16_t *>(
                    KA + kmaj_off<RB>(c, a >> 3) + (a & 7) * 2);
                tmem_ld_wait();
                const float kca = lo_f32(kb);
#pragma unroll
                for (int u = 0; u < EC; ++u)
                    acc[mt][u] = fmaf(kca, __uint_as_float(v[u]), acc[mt][u]);
                sacc[mt] = fmaf(kca, __uint_as_float(sv), sacc[mt]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kDEmpty + j]);
        }
    }
    ok = bar_sync_and(0, kThreads, ok);

    // ---------------- 2. SRE and the kept set (epilogue warps) ----------------
    const int m_keep = keep < n ? keep : n;
    const int nm = n - m_keep;
    if (ok && epi) {
        if (g == 0) {
            den[qd * 32 + lane] = sacc[0];
            if (nmt > 1) den[128 + qd * 32 + lane] = sacc[1];
        }
        bar_sync_and(1, kEpi, true);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int c = mt * 128 + qd * 32 + lane;
            if (mt < nmt && c < n) {
                const float inv_den = 1.f / (den[c] + eps);
                const uint4 *vr = reinterpret_cast<const uint4 *>(vh + (size_t)c * DH + EC * g);
                float part = 0.f;
#pragma unroll
                for (int q4 = 0; q4 < EC / 8; ++q4) {
                    const uint4 w4 = vr[q4];
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float vv = (u & 1) ? hi_f32(wv[u >> 1]) : lo_f32(wv[u >> 1]);
                        const float diff = acc[mt][q4 * 8 + u] * inv_den - vv;
                        part = fmaf(diff, diff, part);
                    }
                }
                sqp[g * kNMax + c] = part;
            }
        }
        bar_sync_and(1, kEpi, true);
        if (tid < n) {
            const float e2 = (sqp[tid] + sqp[kNMax + tid]) + (sqp[2 * kNMax + tid] + sqp[3 * kNMax + tid]);
            sc[tid] = isnan(e2) ? -INFINITY : e2;  // a total order even for 0/0 scores
            cpos[tid] = pos[(size_t)h * pos_head_stride + tid];
            if (scores) scores[(size_t)h * n + tid] = sc[tid];
        }
        bar_sync_and(1, kEpi, true);
        {   // rank among all candidates: two threads per candidate, each half of the others
            const int c = tid >> 1, hf = tid & 1, j0 = hf ? n / 2 : 0, j1 = hf ? n : n / 2;
            int rank = 0;
            if (c < n) {
                const float si = sc[c];
                const int pi = cpos[c];
#pragma unroll 4
                for (int jj = j0; jj < j1; ++jj) {
                    const float sj = sc[jj];
                    const int pj = cpos[jj];
                    rank += sj > si || (sj == si && (pj < pi || (pj == pi && jj < c)));
                }
            }
            rank += __shfl_xor_sync(0xFFFFFFFFu, rank, 1);
            if (c < n && hf == 0) kflag[c] = rank < m_keep;
            bar_sync_and(1, kEpi, true);
            // kept: rank by position among the kept; merged: rank by slot among the merged
            int cnt = 0;
            bool kept = false;
            if (c < n) {
                kept = kflag[c] != 0;
                const int pi = cpos[c];
#pragma unroll 4
                for (int jj = j0; jj < j1; ++jj) {
                    const int kj = kflag[jj];
                    cnt += kept ? (kj && (cpos[jj] < pi || (cpos[jj] == pi && jj < c)))
                                : (!kj && jj < c);
                }
            }
            cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, 1);
            if (c < n && hf == 0) {
                if (kept) {
                    if (cnt < m_keep) keep_idx[(size_t)h * m_keep + cnt] = c;
                } else if (KATA_CHECK(cnt < nm, 0xB402u)) {
                    mlist[cnt] = c;
                }
            }
        }
    }
    if (ok && merge && nm > 0 && warp == kProducerWarp && lane == 0) {
        // the merge reads the state again: ask L2 for it while the epilogue warps rank
        for (int t = 0; t < NT2; ++t) {
            const int rows = D - t * kMR < kMR ? D - t * kMR : kMR;
            prefetch_l2(Hh + (size_t)t * kMR * DH, (uint32_t)(rows * DH * 4));
        }
        prefetch_l2(sh, (uint32_t)(D * 4));
    }
    __syncthreads();

    // ---------------- 3. merge ----------------
    if (ok && merge && nm > 0) {
        const int nk2 = (nm + kMK - 1) / kMK;
        uint8_t *B2 = sm + L::OFF_B2;
        uint16_t *kmT = reinterpret_cast<uint16_t *>(sm + L::OFF_KMT);
        if (warp == kMmaWarp) {
            const uint32_t id2 = idesc_bf16(128, N2, 0, 0);
            for (int t = 0; t < NT2 && ok; ++t) {
                for (int q = 0; q < nk2; ++q) {
                    const int ci = t * nk2 + q, slot = ci % kNA;
                    ok = warp_wait(&bar[kA2Full + slot], (ci / kNA) & 1, err, 0x721) && ok;
                    if (q == 0 && t >= 2)
                        ok = warp_wait(&bar[kD2Empty + (t & 1)], ((t >> 1) - 1) & 1, err, 0x722) && ok;
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t d2 = tmem + (uint32_t)((t & 1) * 128);
                        const uint32_t ah = smem_u32(sm + L::OFF_A2 + slot * 2 * L::A2PART);
                        const uint32_t al = ah + L::A2PART;
                        const uint32_t b2 = smem_u32(B2 + q * L::B2TILE);
#pragma unroll
                        for (int kk = 0; kk < kMK / 16; ++kk) {
                            mma_ss(d2, kmaj_desc_rb<64>(ah, kk), kmaj_desc_rb<64>(b2, kk), id2,
                                   (q > 0 || kk > 0) ? 1u : 0u);
                            mma_ss(d2, kmaj_desc_rb<64>(al, kk), kmaj_desc_rb<64>(b2, kk), id2, 1u);
                        }
                        mma_commit(&bar[kA2Empty + slot]);
                        if (q == nk2 - 1) mma_commit(&bar[kD2Full + (t & 1)]);
                    }
                    __syncwarp();
                }
            }
        } else if (builder) {
            // merged keys, transposed: kmT[a][mi] (zero past nm)
            for (int idx = btid; idx < L::NCH * nk2 * kMK; idx += kBuild) {
                const int mi = idx % (nk2 * kMK), a8 = idx / (nk2 * kMK);
                uint4 x = make_uint4(0, 0, 0, 0);
                if (mi < nm && KATA_CHECK(mlist[mi] >= 0 && mlist[mi] < n, 0xB401u))
                    x = *reinterpret_cast<const uint4 *>(KA + kmaj_off<RB>(mlist[mi], a8));
                const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    kmT[(a8 * 8 + u) * kKmtPitch + mi] = (uint16_t)(xw[u >> 1] >> ((u & 1) * 16));
            }
            // B2 (K-major), chunk q: row e < DH is v[e] of merged candidates
            // 32 q .. 32 q + 31, row DH is 1, rows above are 0 (zero past nm)
            for (int idx = btid; idx < nk2 * N2 * 4; idx += kBuild) {
                const int q = idx / (N2 * 4), rem = idx % (N2 * 4);
                const int kg = rem / N2, e = rem % N2;
                uint32_t bv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int mi = q * kMK + kg * 8 + u;
                    uint32_t val = 0;
                    if (mi < nm && KATA_CHECK(mlist[mi] >= 0 && mlist[mi] < n, 0xB403u)) {
                        if (e < DH)
                            val = reinterpret_cast<const uint16_t *>(vh)[(size_t)mlist[mi] * DH + e];
                        else if (e == DH)
                            val = 0x3F80u;  // 1.0 in bf16
                    }
                    bv[u] = val;
                }
                *reinterpret_cast<uint4 *>(B2 + q * L::B2TILE + kmaj_off<64>(e, kg)) =
                    make_uint4(bv[0] | (bv[1] << 16), bv[2] | (bv[3] << 16),
                               bv[4] | (bv[5] << 16), bv[6] | (bv[7] << 16));
            }
            bar_sync_and(2, kBuild, true);  // kmT complete
            for (int t = 0; t < NT2 && ok; ++t) {
                for (int q = 0; q < nk2; ++q) {
                    const int ci = t * nk2 + q, slot = ci % kNA;
                    if (ci >= kNA)
                        ok = warp_wait(&bar[kA2Empty + slot], ((ci / kNA) - 1) & 1, err, 0x723) && ok;
                    if (!ok) break;
                    uint8_t *Ah = sm + L::OFF_A2 + slot * 2 * L::A2PART, *Al = Ah + L::A2PART;
                    // tile row rr, merged candidates 32 q + 8 kg .. +7
                    for (int idx = btid; idx < 4 * kMR; idx += kBuild) {
                        const int rr = idx & (kMR - 1), kg = idx >> 7;
                        const int r = t * kMR + rr;
                        float x[8];
                        if (r < D) {
                            const int ab = tab[r], col = q * kMK + kg * 8;
                            const uint4 ka = *reinterpret_cast<const uint4 *>(kmT + (ab >> 8) * kKmtPitch + col);
                            const uint4 kb = *reinterpret_cast<const uint4 *>(kmT + (ab & 255) * kKmtPitch + col);
                            const uint32_t aw[4] = {ka.x, ka.y, ka.z, ka.w}, bw[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
                            for (int p = 0; p < 4; ++p) {
                                x[2 * p] = lo_f32(aw[p]) * lo_f32(bw[p]);
                                x[2 * p + 1] = hi_f32(aw[p]) * hi_f32(bw[p]);
                            }
                        } else {
#pragma unroll
                            for (int u = 0; u < 8; ++u) x[u] = 0.f;
                        }
                        uint4 hi, lo;
                        split8(x, hi, lo);
                        *reinterpret_cast<uint4 *>(Ah + kmaj_off<64>(rr, kg)) = hi;
                        *reinterpret_cast<uint4 *>(Al + kmaj_off<64>(rr, kg)) = lo;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[kA2Full + slot]);
                }
            }
        } else if (epi) {
            // w_r D2[r] of tile t goes to a shared-memory image of the tile's state
            // rows (row-major, as in HBM; the normaliser column after them); one
            // thread adds the image to the state with bulk reductions in L2, so
            // no thread reads the state
            for (int t = 0; t < NT2; ++t) {
                const int b = t & 1, rr = qd * 32 + lane, row = t * kMR + rr;
                float *img = reinterpret_cast<float *>(sm + L::OFF_DH + b * L::DHB);
                ok = warp_wait(&bar[kD2Full + b], (t >> 1) & 1, err, 0x724) && ok;
                tc_fence_after();
                uint32_t v[EC], sv = 0;
                if (ok) {
                    const uint32_t col = (uint32_t)(b * 128);
                    if constexpr (EC == 16) tmem_ld16(tmem + lane_base + col + EC * g, v);
                    else tmem_ld8(tmem + lane_base + col + EC * g, v);
                    if (g == 0) tmem_ld1(tmem + lane_base + col + DH, sv);
                    tmem_ld_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && ok) mbar_arrive(&bar[kD2Empty + b]);
                // the reduction that read this image two tiles ago is done reading
                if (tid == 0 && t >= 2) bulk_wait_read_one();
                ok = bar_sync_and(1, kEpi, ok);
                if (!ok) break;
                const float w = row < D ? row_weight(tab[row]) : 0.f;
                float4 *dst = reinterpret_cast<float4 *>(img + rr * DH + EC * g);
#pragma unroll
                for (int u = 0; u < EC / 4; ++u)
                    dst[u] = make_float4(w * __uint_as_float(v[4 * u + 0]), w * __uint_as_float(v[4 * u + 1]),
                                         w * __uint_as_float(v[4 * u + 2]), w * __uint_as_float(v[4 * u + 3]));
                if (g == 0) img[kMR * DH + rr] = w * __uint_as_float(sv);
                fence_proxy_async_smem();
                bar_sync_and(1, kEpi, true);
                if (tid == 0) {
                    const int rows = D - t * kMR < kMR ? D - t * kMR : kMR;
                    bulk_reduce_add_f32(Hst_mut + ((size_t)h * D + (size_t)t * kMR) * DH, img,
                                        (uint32_t)(rows * DH * 4));
                    bulk_reduce_add_f32(s_mut + (size_t)h * D + (size_t)t * kMR, img + kMR * DH,
                                        (uint32_t)(rows * 4));
                    bulk_commit();
                }
            }
            if (tid == 0) bulk_wait_all();  // the reductions are complete before the CTA exits
        }
    }

    // teardown: every copy and MMA this CTA issued has completed
    __syncthreads();
    if (warp == kProducerWarp && lane == 0)
        for (int st = issued > NST ? issued - NST : 0; st < issued; ++st)
            mbar_drain(&bar[kStFull + st % NST], (st / NST) & 1, err, 0x731);
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(&bar[kDrain]);
        mbar_drain(&bar[kDrain], 0, err, 0x732);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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
    sre_tc_kernel<DH><<<nh, kThreads, bytes, stream>>>(Hst, s, kc, vc, (long)cand_stride * DH,
                                                       pos, cand_stride, n, keep, eps, merge,
                                                       scores, keep_idx, Hst_mut, s_mut, err);
    return after_launch();
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool sre_tc_applies(int dtype, int d, int n, const float *Hst, const float *s,
                    const float *Hst_mut, const float *s_mut, const void *kc, const void *vc) {
    return dtype == 1 && (d == 32 || d == 64) && n >= 1 && n <= kNMax && aligned16(Hst) &&
           aligned16(s) && aligned16(Hst_mut) && aligned16(s_mut) && aligned16(kc) &&
           aligned16(vc);
}

cudaError_t sre_tc(const float *Hst, const float *s, const void *kc, const void *vc,
                   const int *pos, int nh, int d, int n, int cand_stride, int keep, float eps,
                   int merge, float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                   unsigned int *err, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const bf *k = static_cast<const bf *>(kc), *v = static_cast<const bf *>(vc);
    KATA_DEBUG_BIND();
    cudaError_t e;
    if (merge && (Hst_mut != Hst || s_mut != s)) {
        // the kernel merges in place: an out-of-place call works on a copy of the
        // state in the output buffers (scored there: the same values)
        const size_t D = (size_t)d * (d + 1) / 2;
        if ((e = cudaMemcpyAsync(Hst_mut, Hst, (size_t)nh * D * d * 4, cudaMemcpyDeviceToDevice,
                                 stream)) != cudaSuccess)
            return e;
        if ((e = cudaMemcpyAsync(s_mut, s, (size_t)nh * D * 4, cudaMemcpyDeviceToDevice,
                                 stream)) != cudaSuccess)
            return e;
        Hst = Hst_mut;
        s = s_mut;
    }
    if (d == 64)
        e = launch<64>(Hst, s, k, v, pos, nh, n, cand_stride, keep, eps, merge, scores, keep_idx,
                       Hst_mut, s_mut, err, stream);
    else if (d == 32)
        e = launch<32>(Hst, s, k, v, pos, nh, n, cand_stride, keep, eps, merge, scores, keep_idx,
                       Hst_mut, s_mut, err, stream);
    else
        return cudaErrorInvalidValue;
    return e;
}

}  // namespace kata
