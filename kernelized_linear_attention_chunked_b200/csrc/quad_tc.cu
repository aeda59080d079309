// Tensor-core (tcgen05) quadratic form of causal kernelized attention for
// bf16 inputs, d = 32 or 64 (no state).
//
// What it computes ("Kernelized Linear Attention: Breaking the Capacity Wall
// with Symmetric Cones", §2.2: the rank-one PSD feature makes the kernel the
// squared inner product, so the attention matrix is (Q K^T)^2 taken
// elementwise; the quadratic form and the chunked state form give the same
// outputs):
//
//   o_i = sum_{j<=i} (q_i.k_j)^2 v_j / (sum_{j<=i} (q_i.k_j)^2 + eps).
//
// It does O(T^2 d) work instead of the chunked form's O(T d^3), with no
// sequential carry: every 128-query tile is independent. It is the faster
// form of an output-only prefill while T is small next to D = d(d+1)/2.
//
// One CTA per (head, 128-query tile), heaviest tiles first. Warp roles: four
// workers, one issuer for the S MMAs, one for the P [V | 1] MMAs, one TMA
// producer. For each 64-key half up to the diagonal:
//   S = Q K^T            tcgen05 SS MMA into tensor memory (fp32), K = d,
//   P = S^2 (causal mask on the diagonal tile), bf16, written back to tensor
//       memory by the four worker warps (thread = query row = TMEM lane),
//   [N | Z] += P [V | 1] tcgen05 TS MMA; the [V | 1] operand is the V tile
//                        followed by an all-ones block, so the accumulator's
//                        columns d.. hold the denominator Z.
// S is double-buffered (d = 32) and P always is, so the MMAs of one half run
// while the workers square the next. o = N / (Z + eps) in the epilogue.
#include "kata_internal.h"
#include "tc_tiles.cuh"

namespace kata {
namespace {

using namespace tc;

struct QuadParams {
    int nch;  // 128-token tiles per head
    float eps;
    float *o;
    unsigned int *err;
    // test hook, 0 in every product call: the P [V | 1] issuer first waits at
    // most `stall` polls on a barrier that nothing arrives at, so the CTA's
    // bounded waits run out and it tears down through its error path
    unsigned int stall;
};

enum QuadBar {
    kQbQFull = 0,
    kQbKFull = 1,   // 2 stages: K tile landed
    kQbKFree = 3,   // 2: both halves' S MMAs read it
    kQbVFull = 5,   // 2: V tile landed
    kQbVFree = 7,   // 2: both halves' P [V | 1] MMAs read it
    kQbSFull = 9,   // S buffers: the scores are in tensor memory
    kQbSFree = 11,  // S buffers: the workers read them (4 warp arrivals)
    kQbPFull = 13,  // 2 P slots: the squared scores are written (4 warp arrivals)
    kQbPFree = 15,  // 2 P slots: the MMAs that read them completed
    kQbODone = 17,
    kQbSDrain = 18,  // the S issuer's MMAs completed (teardown)
    kQbPDrain = 19,  // the P [V | 1] issuer's MMAs completed (teardown)
    kQbNever = 20,   // nothing arrives here (the test hook's stall)
    kQbCount = 21
};

// Square two fp32 scores (one packed f32x2 multiply, round to nearest) and
// round the squares to a bf16 pair (first score in the low half).
__device__ __forceinline__ uint32_t sq_pack(uint32_t x0, uint32_t x1) {
    uint32_t d;
    asm("{\n\t.reg .b64 a;\n\t.reg .f32 l, h;\n\t"
        "mov.b64 a, {%1, %2};\n\t"
        "mul.rn.f32x2 a, a, a;\n\t"
        "mov.b64 {l, h}, a;\n\t"
        "cvt.rn.bf16x2.f32 %0, h, l;\n\t}"
        : "=r"(d)
        : "r"(x0), "r"(x1));
    return d;
}

template <int DH>
struct QuadCfg {
    using S = Shape<DH>;
    // tensor memory (256 columns): the [N | Z] accumulator, NSB S buffers of
    // 64 fp32 columns, NP P slots of 32 columns (64 bf16 keys)
    static constexpr int NSB = DH == 64 ? 1 : 2;
    static constexpr int NP = 2;
    static constexpr uint32_t S_COL = S::ACC_PITCH;
    static constexpr uint32_t P_COL = S_COL + 64 * NSB;
    static_assert(P_COL + 32 * NP <= 256, "tensor-memory budget");
    // shared memory: Q tile, two K stages, two V stages, the all-ones block
    static constexpr int Q = 0;
    static constexpr int K0 = kTileBytes;
    static constexpr int V0 = 3 * kTileBytes;
    static constexpr int ONES = V0 + 2 * S::VBYTES;
    static constexpr int BAR = ONES + 2048;
    static constexpr int SLOT = BAR + kQbCount * 8;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr int ISSUER_WARP = 4;  // S = Q K^T issuer (allocates tensor memory)
    static constexpr int PV_WARP = 5;      // P [V | 1] issuer
    static constexpr int TMA_WARP = 6;
    static constexpr int THREADS = 224;
};

template <int DH>
__global__ void __launch_bounds__(QuadCfg<DH>::THREADS, 2)
    quad_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, QuadParams p) {
    using S = Shape<DH>;
    using L = QuadCfg<DH>;
    constexpr int NSB = L::NSB, NP = L::NP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x;
    const int m = p.nch - 1 - (int)blockIdx.y;  // query tile: the longest rows launch first
    const int nh = 2 * (m + 1);                 // 64-key halves up to the diagonal
    const long row0 = (long)head * p.nch * kTile;
    const ErrCtx err{p.err};

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQbCount; ++i) {
            const bool four = (i >= kQbSFree && i < kQbSFree + 2) || (i >= kQbPFull && i < kQbPFull + 2);
            mbar_init(&bar[i], four ? 4 : 1);
        }
        cta_abort_clear();
        fence_barrier_init();
    }
    if (warp == L::ISSUER_WARP) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == L::TMA_WARP) {
        // ---------------- TMA producer: Q once, K and V tiles in two stages ----------------
        if (lane == 0) {
            prefetch_tensormap(&mq);
            prefetch_tensormap(&mk);
            prefetch_tensormap(&mv);
            mbar_arrive_expect_tx(&bar[kQbQFull], kTileBytes);
            tma_load_2d(sm + L::Q, &mq, 0, (int)(row0 + (long)m * kTile), &bar[kQbQFull]);
            int nk = 0, nv = 0;  // K and V tiles issued
            for (int u = 0; u <= m; ++u) {
                const int st = u & 1;
                const int y = (int)(row0 + (long)u * kTile);
                if (u >= 2 && !mbar_wait(&bar[kQbKFree + st], ((u >> 1) - 1) & 1, err, 0x601)) break;
                mbar_arrive_expect_tx(&bar[kQbKFull + st], kTileBytes);
                tma_load_2d(sm + L::K0 + st * kTileBytes, &mk, 0, y, &bar[kQbKFull + st]);
                ++nk;
                if (u >= 2 && !mbar_wait(&bar[kQbVFree + st], ((u >> 1) - 1) & 1, err, 0x602)) break;
                mbar_arrive_expect_tx(&bar[kQbVFull + st], S::VBYTES);
                tma_load_2d(sm + L::V0 + st * S::VBYTES, &mv, 0, y, &bar[kQbVFull + st]);
                ++nv;
            }
            // no copy may still be in flight when the CTA exits. A tile is only
            // issued once the previous phase of its barrier completed, so the
            // last tile issued on each barrier is the only one to wait for.
            mbar_drain(&bar[kQbQFull], 0, err, 0x603);
            for (int u = nk - 2 < 0 ? 0 : nk - 2; u < nk; ++u)
                mbar_drain(&bar[kQbKFull + (u & 1)], (u >> 1) & 1, err, 0x604);
            for (int u = nv - 2 < 0 ? 0 : nv - 2; u < nv; ++u)
                mbar_drain(&bar[kQbVFull + (u & 1)], (u >> 1) & 1, err, 0x605);
        }
    } else if (warp == L::ISSUER_WARP) {
        // ---------------- S issuer: S = Q K^T for half j into buffer j % NSB ----------------
        if (lane == 0) {
            const uint32_t i_s = idesc_bf16(128, 64, 0, 0);
            const uint32_t q_a = smem_u32(sm + L::Q), k_a = smem_u32(sm + L::K0);
            const bool ok = mbar_wait(&bar[kQbQFull], 0, err, 0x614);
            for (int j = 0; ok && j < nh; ++j) {
                const int u = j >> 1, h = j & 1, st = u & 1, b = j % NSB;
                // the workers read this buffer's previous scores
                if (j >= NSB && !mbar_wait(&bar[kQbSFree + b], (j / NSB - 1) & 1, err, 0x610)) break;
                if (h == 0 && !mbar_wait(&bar[kQbKFull + st], (u >> 1) & 1, err, 0x611)) break;
                tc_fence_after();
                const uint32_t kb = k_a + st * kTileBytes + h * 64 * 128;
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    mma_ss(tmem + L::S_COL + 64 * b, kmaj_desc(q_a, kk), kmaj_desc(kb, kk), i_s,
                           kk > 0);
                mma_commit(&bar[kQbSFull + b]);
                if (h == 1) mma_commit(&bar[kQbKFree + st]);
            }
            // every MMA this thread issued has completed before the teardown
            mma_commit(&bar[kQbSDrain]);
            mbar_drain(&bar[kQbSDrain], 0, err, 0x615);
        }
    } else if (warp == L::PV_WARP) {
        // ---------------- P [V | 1] issuer: [N | Z] += P [V | 1] for half j ----------------
        if (lane == 0) {
            const uint32_t i_av = idesc_bf16(128, S::NACC, 0, 1);
            const uint32_t v_a = smem_u32(sm + L::V0), ones = smem_u32(sm + L::ONES);
            bool ok = p.stall == 0u || mbar_wait(&bar[kQbNever], 0, err, 0x6FF, p.stall);
            for (int j = 0; ok && j < nh; ++j) {
                const int u = j >> 1, h = j & 1, st = u & 1, ps = j % NP;
                ok = mbar_wait(&bar[kQbPFull + ps], (j / NP) & 1, err, 0x612) &&
                     (h != 0 || mbar_wait(&bar[kQbVFull + st], (u >> 1) & 1, err, 0x613));
                if (!ok) break;
                tc_fence_after();
                const uint32_t vb = v_a + st * S::VBYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem, tmem + L::P_COL + 32 * ps + 8 * kk,
                           vones_desc<DH>(vb, ones, 64 * h + 16 * kk), i_av, (j > 0 || kk > 0));
                mma_commit(&bar[kQbPFree + ps]);
                if (h == 1) mma_commit(&bar[kQbVFree + st]);
            }
            if (ok) mma_commit(&bar[kQbODone]);
            mma_commit(&bar[kQbPDrain]);
            mbar_drain(&bar[kQbPDrain], 0, err, 0x616);
        }
    } else {
        // ---------------- workers: thread = query row = tensor-memory lane ----------------
        const int i = threadIdx.x;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // the all-ones block; the first P-full arrival publishes it to the MMAs
        fill_ones(sm + L::ONES, i, kWorkers);
        bool ok = true;
        for (int j = 0; j < nh; ++j) {
            const int h = j & 1, b = j % NSB, ps = j % NP;
            const bool diag = (j >> 1) == m;
            if (!(ok = warp_wait(&bar[kQbSFull + b], (j / NSB) & 1, err, 0x620))) break;
            tc_fence_after();
            float sv[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[16];
                tmem_ld16(tmem + lane_base + L::S_COL + 64 * b + 16 * c, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[16 * c + e] = __uint_as_float(r[e]);
            }
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kQbSFree + b]);
            // squared scores; key 64 h + e of the diagonal tile is masked past row i
            uint32_t pk[32];
            if (diag) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int k0 = 64 * h + 2 * e;
                    const float a0 = k0 > i ? 0.f : sv[2 * e] * sv[2 * e];
                    const float a1 = k0 + 1 > i ? 0.f : sv[2 * e + 1] * sv[2 * e + 1];
                    pk[e] = pack_bf16x2(a0, a1);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    pk[e] = sq_pack(__float_as_uint(sv[2 * e]), __float_as_uint(sv[2 * e + 1]));
            }
            if (j >= NP && !(ok = warp_wait(&bar[kQbPFree + ps], (j / NP - 1) & 1, err, 0x621)))
                break;
            tc_fence_after();
            {
                uint32_t r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = pk[e];
                tmem_st16(tmem + lane_base + L::P_COL + 32 * ps, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = pk[16 + e];
                tmem_st16(tmem + lane_base + L::P_COL + 32 * ps + 16, r);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kQbPFull + ps]);
        }
        // epilogue: o = N / (Z + eps)
        if (ok) ok = warp_wait(&bar[kQbODone], 0, err, 0x622);
        tc_fence_after();
        uint32_t r[DH / 16 + 1][16];
#pragma unroll
        for (int c = 0; c <= DH / 16; ++c) tmem_ld16(tmem + lane_base + 16 * c, r[c]);
        tmem_ld_wait();
        const float inv = 1.f / (__uint_as_float(r[DH / 16][0]) + p.eps);
        float4 *dst = reinterpret_cast<float4 *>(p.o + (row0 + (long)m * kTile + i) * DH);
#pragma unroll
        for (int n = 0; ok && n < DH; n += 4)
            dst[n / 4] = make_float4(__uint_as_float(r[n / 16][n % 16]) * inv,
                                     __uint_as_float(r[n / 16][n % 16 + 1]) * inv,
                                     __uint_as_float(r[n / 16][n % 16 + 2]) * inv,
                                     __uint_as_float(r[n / 16][n % 16 + 3]) * inv);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == L::ISSUER_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <int DH>
cudaError_t launch(const PrefillArgs &a, cudaStream_t stream, unsigned int stall) {
    using L = QuadCfg<DH>;
    const int nheads = a.B * a.H, nch = a.T / kTile;
    CUtensorMap mq, mk, mv;
    if (!make_qkv_maps(&mq, &mk, &mv, a.q, a.k, a.v, DH, (long)nheads * a.T))
        return cudaErrorInvalidValue;
    QuadParams qp{nch, a.eps, a.o, a.err, stall};
    cudaError_t e = set_smem_once<quad_kernel<DH>>(L::BYTES);
    if (e != cudaSuccess) return e;
    quad_kernel<DH><<<dim3(nheads, nch), L::THREADS, L::BYTES, stream>>>(mq, mk, mv, qp);
    return after_launch();
}

}  // namespace

bool quad_tc_shape_ok(int dtype, int B, int H, int T, int d) {
    return dtype == 1 && (d == 64 || d == 32) && T > 0 && T % kTile == 0 &&
           T / kTile <= 65535 && (long)B * H * T < (1L << 31) && (long)B * H <= 0x7FFFFFFFL;
}

cudaError_t quad_tc(const PrefillArgs &a, cudaStream_t stream, unsigned int stall) {
    if (!quad_tc_shape_ok(a.dtype, a.B, a.H, a.T, a.d) || a.o == nullptr)
        return cudaErrorNotSupported;
    return a.d == 64 ? launch<64>(a, stream, stall) : launch<32>(a, stream, stall);
}

}  // namespace kata
