// Tensor-core (tcgen05) chunked prefill for bf16 inputs, d = 32 or 64.
//
// What it computes ("Kernelized Linear Attention: Breaking the Capacity Wall
// with Symmetric Cones", technical summary §2.2 rank-one PSD cone and §2.3
// chunked parallelism with the exact chunked state form):
//
//   o_i = phi(q_i)^T H_i / (phi(q_i)^T s_i + eps),   H_i = sum_{j<=i} phi(k_j) v_j^T,
//   s_i = sum_{j<=i} phi(k_j),   <phi(q), phi(k)> = (q.k)^2.
//
// Two kernels, split along the dependency structure of the chunked form:
//
//  1. state_kernel — the carry across chunks (§2.3's inter-chunk state
//     propagation). One CTA owns one 128-row tile of the feature space of one
//     head and walks the sequence chunk by chunk (128 tokens), accumulating
//     dH = Phi(K_c)^T [V_c | 1] on the tensor cores into fp32 tensor memory.
//     Every L tokens it writes the exclusive prefix state (the state before
//     the interval) as a bf16 snapshot laid out as the readout's MMA operand.
//     Feature rows are independent, so a head's tiles run as separate CTAs
//     with no communication.
//  2. readout_kernel — fully parallel over (head, 128-query tile):
//       inter part  Phi(Q) [H | s](snapshot at the start of the interval),
//       intra part  ((Q K^T)^2 masked causally) [V | 1] over the keys from
//                   the interval start to the query (the quadratic form),
//     both accumulated in one fp32 tensor-memory tile, then normalised.
//
// Feature space. phi(x) x phi(y) = (x.y)^2 is expanded over 8x8 blocks of the
// outer product x x^T: an off-diagonal block (A < B) holds x_a x_b for a in
// block A, b in block B (each unordered pair once, weight 2 on the query side);
// a diagonal block (A, A) holds all 64 ordered products (weight 1, so a pair
// a != b inside it counts twice, a = b once). Every block is one 64-feature
// slice: d = 32 has 10 slices, d = 64 has 36. The state is stored without the
// sqrt(2) of the canonical packed layout; kata_prefill's H_in/H_out use the
// canonical one and the state kernel converts at both ends.
//
// Column layout of the fp32 accumulators (state and output), N = d + 16
// columns: 0..d-1 hold H (or the numerator), d..d+15 all hold s (or the
// denominator), because the [V | 1] operand is the V tile (one swizzle atom of
// d columns: 128-byte swizzle for d = 64, 64-byte for d = 32) followed by an
// all-ones block. The snapshot slices hold rows 0..d-1 = H and d..d+15 = s.
#include "kata_internal.h"
#include "tc_tiles.cuh"

namespace kata {
namespace {

using namespace tc;

// Block pair (A, B), A <= B, of slice s: slices run A-major, B ascending.
__device__ __forceinline__ void slice_blocks(int s, int nb, int &A, int &B) {
    A = 0;
    while (s >= nb - A) {
        s -= nb - A;
        ++A;
    }
    B = A + s;
}

// Canonical packed index of the unordered pair {a, b} (upper triangle, a-major).
__device__ __forceinline__ int canon_index(int a, int b, int d) {
    const int lo = a < b ? a : b, hi = a < b ? b : a;
    return lo * d - lo * (lo - 1) / 2 + (hi - lo);
}

__device__ __forceinline__ uint32_t hmul2(uint32_t x, uint32_t y) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
    return r;
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t x) { return (x & 0xFFFFu) * 0x10001u; }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t x) { return (x >> 16) * 0x10001u; }

__device__ __forceinline__ void worker_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(kWorkers) : "memory");
}

// worker_sync that also tells every worker whether all of them are still fine
// (a worker whose bounded wait ran out passes false; all then stop together,
// so none is left waiting at a later worker barrier).
__device__ __forceinline__ bool worker_vote(bool ok) { return bar_sync_and(1, kWorkers, ok); }

// Element offset of 16-byte chunk `c` of row `r` in a tile with 128-byte rows
// and the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------------------
// State kernel
// ---------------------------------------------------------------------------

struct StateParams {
    int nch;        // chunks per head
    int cpi;        // chunks per snapshot interval
    int nint;       // snapshot intervals per head
    int seg_len;    // chunks per sequence segment (grid z): segment z starts at
                    // chunk z * seg_len; with several segments there are no
                    // snapshots and segment z writes its own partial state at
                    // H_out + z * heads * D * d, s_out + z * heads * D
    const float *H_in, *s_in;
    float *H_out, *s_out;
    uint8_t *snap;  // [heads][nint][NS][NSNAP][128 B], or null: no snapshots
    unsigned int *err;
    // Scan mode (several segments that write snapshots; seg_len a multiple of
    // cpi): segment z >= 1 starts from the sum of the earlier segments' states,
    // carry_H + (z - 1) * heads * D * d and carry_s + (z - 1) * heads * D,
    // numbers its snapshot intervals from its first chunk's, and only the last
    // segment writes H_out, s_out (the final state, not a partial).
    const float *carry_H = nullptr, *carry_s = nullptr;
    int scan = 0;
};

enum StateBar {
    kSbKFull = 0,    // 4: K tile landed
    kSbKFree = 4,    // 4: the workers transposed it (4 warp arrivals)
    kSbVFull = 8,    // 2: V tile landed
    kSbVFree = 10,   // 2: the chunk's MMAs finished reading it (one commit per issuer)
    kSbAFull = 12,   // NA: Phi(K)^T tile written to tensor memory (4 warp arrivals)
    kSbDone = 14,    // NA: the MMAs of the chunk that used this A slot completed
    kSbSnap = 16,    // the workers read the accumulators at an interval end
    kSbDrain = 17,   // 2: an issuer's MMAs completed (teardown)
    kSbCount = 19
};

// Transposed K tile: row a holds k[t][a] for the 128 tokens of the chunk as
// 16 chunks of 16 bytes; chunk j of row a sits at j ^ kt_swz(a), which keeps
// both the 8x8 block transpose writes and the per-feature row reads free of
// shared-memory bank conflicts.
__device__ __forceinline__ uint32_t kt_offset(int row, int chunk) {
    return (uint32_t)(row * 256 + ((chunk ^ ((row + (row >> 3)) & 7)) << 4));
}

template <int DH, int NI, int NA>
struct StateCfg {
    static constexpr int KR = DH == 64 ? 2 : 3;  // K tiles in flight
    static constexpr int K0 = 0;
    static constexpr int V0 = KR * kTileBytes;    // 2 x V tile
    static constexpr int ONES = V0 + 2 * Shape<DH>::VBYTES;
    static constexpr int KT = ONES + 2048;
    static constexpr int STAGE = KT + DH * 256;   // snapshot staging: 2 slices
    static constexpr int BAR = STAGE + 2 * Shape<DH>::SLICE_BYTES;
    static constexpr int SLOT = BAR + kSbCount * 8;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr int THREADS = 32 * (5 + NI);  // workers, NI issuers, TMA
    // NI accumulators, then NA Phi(K)^T slots of 64 columns
    static constexpr uint32_t A_COL = (NI * Shape<DH>::ACC_PITCH + 63) / 64 * 64;
    static constexpr uint32_t TMEM_COLS = A_COL + 64u * NA <= 256 ? 256 : 512;
    __host__ __device__ static constexpr uint32_t acc_col(int i) {
        return (uint32_t)(Shape<DH>::ACC_PITCH * i);
    }
};

template <int DH, int NI, int NA>
__global__ void __launch_bounds__(StateCfg<DH, NI, NA>::THREADS,
                                  StateCfg<DH, NI, NA>::TMEM_COLS == 256 ? 2 : 1)
    state_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                 StateParams p) {
    using S = Shape<DH>;
    using L = StateCfg<DH, NI, NA>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, head = blockIdx.y;
    const ErrCtx err{p.err};
    constexpr int kTmaWarp = 4 + NI;

    if (threadIdx.x == 0) {
        cta_abort_clear();
        for (int i = 0; i < 2; ++i) mbar_init(&bar[kSbDrain + i], 1);
        for (int i = 0; i < L::KR; ++i) {
            mbar_init(&bar[kSbKFull + i], 1);
            mbar_init(&bar[kSbKFree + i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[kSbVFull + i], 1);
            mbar_init(&bar[kSbVFree + i], NI);
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&bar[kSbAFull + i], 4);
            mbar_init(&bar[kSbDone + i], NI);
        }
        mbar_init(&bar[kSbSnap], 4);
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // this CTA's chunks: [c0, c0 + nch) of its head
    const int c0 = (int)blockIdx.z * p.seg_len;
    const int nch = p.nch - c0 < p.seg_len ? p.nch - c0 : p.seg_len;
    const long row0 = ((long)head * p.nch + c0) * kTile;  // first token row of this CTA
    constexpr int D = DH * (DH + 1) / 2;
    const int z = (int)blockIdx.z;
    float *H_out, *s_out;
    const float *H_in, *s_in;
    if (p.scan) {
        // scan mode: the state before chunk c0 comes in as this segment's
        // initial state; the last segment's final state is the call's
        const bool last = z == (int)gridDim.z - 1;
        H_out = last ? p.H_out : nullptr;
        s_out = last ? p.s_out : nullptr;
        H_in = z == 0 ? p.H_in : p.carry_H + (size_t)(z - 1) * gridDim.y * D * DH;
        s_in = z == 0 ? p.s_in : p.carry_s + (size_t)(z - 1) * gridDim.y * D;
    } else {
        H_out = p.H_out ? p.H_out + (size_t)z * gridDim.y * D * DH : nullptr;
        s_out = p.s_out ? p.s_out + (size_t)z * gridDim.y * D : nullptr;
        // the initial state enters through the first segment only
        H_in = z == 0 ? p.H_in : nullptr;
        s_in = z == 0 ? p.s_in : nullptr;
    }
    const int g0 = c0 / p.cpi;  // this segment's first snapshot interval
    // the readout kernel may start its setup and intra-chunk work now; it waits
    // for this grid's completion before it reads a snapshot
    if (threadIdx.x == 0) launch_dependents();

    if (warp == kTmaWarp) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&mk);
            prefetch_tensormap(&mv);
            // K and V tiles are freed by different consumers (the transposing
            // workers, the MMAs): issue whichever slot frees first
            int nk = 0, nv = 0;
            uint32_t idle = 0;
            while ((nk < nch || nv < nch) && idle < (1u << 24)) {
                bool moved = false;
                if (nk < nch) {
                    const int ks = nk % L::KR, kn = nk / L::KR;
                    if (kn == 0 || mbar_test_wait(&bar[kSbKFree + ks], (kn - 1) & 1)) {
                        mbar_arrive_expect_tx(&bar[kSbKFull + ks], kTileBytes);
                        tma_load_2d(sm + L::K0 + ks * kTileBytes, &mk, 0,
                                    (int)(row0 + (long)nk * kTile), &bar[kSbKFull + ks]);
                        ++nk;
                        moved = true;
                    }
                }
                if (nv < nch) {
                    const int s = nv & 1, n = nv >> 1;
                    if (n == 0 || mbar_test_wait(&bar[kSbVFree + s], (n - 1) & 1)) {
                        mbar_arrive_expect_tx(&bar[kSbVFull + s], S::VBYTES);
                        tma_load_2d(sm + L::V0 + s * S::VBYTES, &mv, 0,
                                    (int)(row0 + (long)nv * kTile), &bar[kSbVFull + s]);
                        ++nv;
                        moved = true;
                    }
                }
                if (!moved) {
                    __nanosleep(32);
                    if ((++idle & 1023u) == 0u && cta_aborted(err)) break;
                }
            }
            if (nk < nch || nv < nch) report_timeout(err, 0x401u);
            // no copy may still be in flight when the CTA exits. A tile is only
            // issued once the previous phase of its barrier completed, so the
            // last tile issued on each barrier is the only one to wait for.
            for (int c = nk - L::KR < 0 ? 0 : nk - L::KR; c < nk; ++c)
                mbar_drain(&bar[kSbKFull + c % L::KR], (c / L::KR) & 1, err, 0x403);
            for (int c = nv - 2 < 0 ? 0 : nv - 2; c < nv; ++c)
                mbar_drain(&bar[kSbVFull + (c & 1)], (c >> 1) & 1, err, 0x404);
        }
    } else if (warp >= 4) {
        // ---------------- MMA issuer `ii`: K-steps ii, ii + NI, ... ----------------
        const int ii = warp - 4;
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, S::NACC, 0, 1);
            const uint32_t ones = smem_u32(sm + L::ONES);
            const uint32_t acc = tmem + L::acc_col(ii);
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1, sa = c % NA;
                if (!mbar_wait(&bar[kSbVFull + s], (c >> 1) & 1, err, 0x412)) break;
                if (!mbar_wait(&bar[kSbAFull + sa], (c / NA) & 1, err, 0x410)) break;
                // the state at an interval end must be read before it moves on
                if (c > 0 && c % p.cpi == 0 &&
                    !mbar_wait(&bar[kSbSnap], (c / p.cpi - 1) & 1, err, 0x411))
                    break;
                tc_fence_after();
                const uint32_t v = smem_u32(sm + L::V0 + s * S::VBYTES);
#pragma unroll
                for (int kk = ii; kk < kTile / 16; kk += NI)
                    mma_ts(acc, tmem + L::A_COL + 64 * sa + 8 * kk,
                           vones_desc<DH>(v, ones, 16 * kk), idesc, 1);
                mma_commit(&bar[kSbVFree + s]);
                mma_commit(&bar[kSbDone + sa]);
            }
            // every MMA this thread issued has completed before the teardown
            mma_commit(&bar[kSbDrain + ii]);
            mbar_drain(&bar[kSbDrain + ii], 0, err, 0x413);
        }
    } else {
        // ---------------- workers: one thread per feature row ----------------
        const int f = threadIdx.x;  // tensor-memory lane = row of this state tile
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int slice = 2 * tile + (f >> 6);
        const bool valid = slice < S::NS;
        const int nvalid = S::NS - 2 * tile < 2 ? S::NS - 2 * tile : 2;
        int ra = 0, rb = 0;
        if (valid) {
            int A, B;
            slice_blocks(slice, S::NB, A, B);
            ra = 8 * A + ((f & 63) >> 3);
            rb = 8 * B + (f & 7);
        }
        uint8_t *kt = sm + L::KT;
        uint8_t *stage = sm + L::STAGE;

        // 16-row all-ones block of the [V | 1] operand
        {
            uint4 *o4 = reinterpret_cast<uint4 *>(sm + L::ONES);
            for (int i = f; i < 2048 / 16; i += kWorkers)
                o4[i] = make_uint4(kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2);
            fence_proxy_async_smem();
        }

        // initial state: H_in in the internal scaling (no sqrt 2) in accumulator 0
        float init[DH + 1];
        {
            const bool have = valid && H_in != nullptr;
            const int ci = valid ? canon_index(ra, rb, DH) : 0;
            const float w = (ra != rb) ? 0.70710678118654752f : 1.f;
            const size_t hb = ((size_t)head * (DH * (DH + 1) / 2) + ci);
#pragma unroll
            for (int n = 0; n < DH; ++n) init[n] = have ? H_in[hb * DH + n] * w : 0.f;
            init[DH] = have ? s_in[hb] * w : 0.f;
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < S::NACC / 16; ++j) {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int col = 16 * j + e;
                    r[e] = __float_as_uint(col < DH ? init[col] : init[DH]);
                }
                tmem_st16(tmem + lane_base + L::acc_col(0) + 16 * j, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = 0u;
#pragma unroll
                for (int i = 1; i < NI; ++i) tmem_st16(tmem + lane_base + L::acc_col(i) + 16 * j, r);
            }
            tmem_st_wait();
        }
        // snapshot: staged in shared memory as the readout's K-major operand
        // (row n < DH = column n of H, rows DH.. = s), then one bulk store
        // (thread 0 waits for the previous bulk store's read of the staging
        // buffer before the first worker sync of each chunk)
        auto write_snapshot = [&](int g, const float (&x)[DH + 1], bool ok) -> bool {
            if (p.snap == nullptr) return ok;
            if (ok && valid) {
                uint8_t *row = stage + (f >> 6) * S::SLICE_BYTES;
                const int fl = f & 63;
#pragma unroll
                for (int n = 0; n < S::NSNAP; ++n)
                    *reinterpret_cast<__nv_bfloat16 *>(row + n * 128 +
                                                       (((fl >> 3) ^ (n & 7)) << 4) +
                                                       (fl & 7) * 2) =
                        __float2bfloat16_rn(n < DH ? x[n] : x[DH]);
            }
            fence_proxy_async_smem();
            if (!worker_vote(ok)) return false;
            if (f == 0)
                bulk_store(p.snap + (((size_t)head * p.nint + g) * S::NS + 2 * tile) *
                                        S::SLICE_BYTES,
                           stage, nvalid * S::SLICE_BYTES);
            return true;
        };
        bool ok = true;  // warp-uniform: every wait of this warp so far succeeded
        if (H_in) ok = write_snapshot(g0, init, ok);
        if (f == 0) bulk_wait_read();
        // the state: sum of the issuers' accumulators, columns 0..DH-1 and s
        auto read_acc = [&](float (&x)[DH + 1]) {
#pragma unroll
            for (int n = 0; n <= DH; ++n) x[n] = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const uint32_t acc = tmem + lane_base + L::acc_col(i);
                uint32_t r[DH / 16 + 1][16];
#pragma unroll
                for (int j = 0; j < DH / 16; ++j) tmem_ld16(acc + 16 * j, r[j]);
                tmem_ld16(acc + S::SCOL, r[DH / 16]);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < DH / 16; ++j)
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[16 * j + e] += __uint_as_float(r[j][e]);
                x[DH] += __uint_as_float(r[DH / 16][0]);
            }
        };

        constexpr int NCB = DH / 8;  // 8-column blocks of a K row
        // every worker reaches every worker_vote below (no worker leaves the
        // loop on its own), so a failed wait never strands the others there
        for (int c = 0; c < nch; ++c) {
            const int sa = c % NA, ks = c % L::KR;
            // transpose the K tile in 8 x 8 blocks (8 tokens x 8 columns per thread)
            ok = ok && warp_wait(&bar[kSbKFull + ks], (c / L::KR) & 1, err, 0x420);
            if (ok && f < 16 * NCB) {
                const uint8_t *kb = sm + L::K0 + ks * kTileBytes;
                const int tb = f / NCB, cb = f % NCB;
                uint32_t x[8][4];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(kb + sw128_chunk(8 * tb + r, cb));
                    x[r][0] = v.x;
                    x[r][1] = v.y;
                    x[r][2] = v.z;
                    x[r][3] = v.w;
                }
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint32_t sel = (cc & 1) ? 0x7632u : 0x5410u;
                    uint4 y;
                    y.x = __byte_perm(x[0][cc >> 1], x[1][cc >> 1], sel);
                    y.y = __byte_perm(x[2][cc >> 1], x[3][cc >> 1], sel);
                    y.z = __byte_perm(x[4][cc >> 1], x[5][cc >> 1], sel);
                    y.w = __byte_perm(x[6][cc >> 1], x[7][cc >> 1], sel);
                    *reinterpret_cast<uint4 *>(kt + kt_offset(8 * cb + cc, tb)) = y;
                }
            }
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(&bar[kSbKFree + ks]);
            if (f == 0) bulk_wait_read();  // staging buffer free for the next snapshot
            if (!(ok = worker_vote(ok))) break;  // K^T complete
            // Phi(K)^T row of feature (ra, rb): 128 tokens, two per 32-bit column
            uint32_t a_row[64];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint4 x = *reinterpret_cast<const uint4 *>(kt + kt_offset(ra, j));
                const uint4 y = *reinterpret_cast<const uint4 *>(kt + kt_offset(rb, j));
                a_row[4 * j + 0] = valid ? hmul2(x.x, y.x) : 0u;
                a_row[4 * j + 1] = valid ? hmul2(x.y, y.y) : 0u;
                a_row[4 * j + 2] = valid ? hmul2(x.z, y.z) : 0u;
                a_row[4 * j + 3] = valid ? hmul2(x.w, y.w) : 0u;
            }
            worker_sync();  // K^T free for the next chunk
            // A slot sa was last read by chunk c - NA
            if (c >= NA) ok = warp_wait(&bar[kSbDone + sa], (c / NA - 1) & 1, err, 0x421);
            tc_fence_after();
            if (ok) {
                uint32_t r[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[e] = a_row[16 * j + e];
                    tmem_st16(tmem + lane_base + L::A_COL + 64 * sa + 16 * j, r);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(&bar[kSbAFull + sa]);
            // chunk c opens interval g: the state after chunk c - 1 is snapshot g
            // (A(c) is already published, so the issuers wait only for this read)
            if (c > 0 && c % p.cpi == 0) {
                // after a failed wait this one gives up at once (the CTA's abort
                // flag is set), and reading the allocated tensor memory is
                // harmless: both stay unconditional, which keeps x in registers
                ok = warp_wait(&bar[kSbDone + (c - 1) % NA], ((c - 1) / NA) & 1, err, 0x422) && ok;
                tc_fence_after();
                float x[DH + 1];
                read_acc(x);
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&bar[kSbSnap]);
                ok = write_snapshot(g0 + c / p.cpi, x, ok);
            }
        }
        // final state, converted to the canonical layout
        if (ok) ok = warp_wait(&bar[kSbDone + (nch - 1) % NA], ((nch - 1) / NA) & 1, err, 0x423);
        tc_fence_after();
        if (ok && H_out) {
            float fin[DH + 1];
            read_acc(fin);
            if (valid && ra <= rb) {
                const int ci = canon_index(ra, rb, DH);
                const float w = (ra != rb) ? 1.41421356237309505f : 1.f;
                const size_t hb = (size_t)head * (DH * (DH + 1) / 2) + ci;
                float4 *dst = reinterpret_cast<float4 *>(H_out + hb * DH);
#pragma unroll
                for (int n = 0; n < DH; n += 4)
                    dst[n / 4] = make_float4(fin[n] * w, fin[n + 1] * w, fin[n + 2] * w,
                                             fin[n + 3] * w);
                s_out[hb] = fin[DH] * w;
            }
        }
        if (f == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Readout kernel
// ---------------------------------------------------------------------------

constexpr int kRP = 4;      // snapshot slices in flight
constexpr int kRQMax = 3;   // A-operand slots in tensor memory (at most)

struct ReadParams {
    int nch;     // query tiles (= chunks) per head
    int cpi;     // chunks per snapshot interval
    int nint;    // snapshot intervals per head
    int has_in;  // an initial state was given: snapshot 0 exists
    const uint8_t *snap;
    float *o;
    float eps;
    unsigned int *err;
};

enum ReadBar {
    kRbQFull = 0,
    kRbKFull = 1,
    kRbKFree = 2,
    kRbVFull = 3,
    kRbVFree = 4,
    kRbSFull = 5,
    kRbSFree = 6,  // 4 warp arrivals
    kRbODone = 7,
    kRbPFull = 8,
    kRbPFree = kRbPFull + kRP,
    kRbAqFull = kRbPFree + kRP,  // 4 warp arrivals
    kRbAqFree = kRbAqFull + kRQMax,
    kRbDrain = kRbAqFree + kRQMax,  // 2: an issuer's MMAs completed (teardown)
    kRbCount = kRbDrain + 2
};

template <int DH, int NIR>
struct ReadCfg {
    static constexpr int Q = 0;
    static constexpr int K = kTileBytes;
    static constexpr int V = 2 * kTileBytes;
    static constexpr int ONES = 3 * kTileBytes;   // 16-row all-ones block
    static constexpr int P = 3 * kTileBytes + 2048;  // kRP snapshot slices
    static constexpr int BAR = P + kRP * Shape<DH>::SLICE_BYTES;
    static constexpr int SLOT = BAR + kRbCount * 8;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr int THREADS = 32 * (5 + NIR);  // workers, NIR issuers, TMA
    static constexpr int TMA_WARP = 4 + NIR;
    // tensor memory (256 columns): NIR output accumulators, S (64 keys), then
    // RQ A-operand slots of 32 columns
    static constexpr uint32_t S_COL = (NIR * Shape<DH>::ACC_PITCH + 31) / 32 * 32;
    static constexpr uint32_t AQ_COL = S_COL + 64;
    static constexpr int RQ = (256 - AQ_COL) / 32 < kRQMax ? (256 - AQ_COL) / 32 : kRQMax;
    __host__ __device__ static constexpr uint32_t o_col(int i) {
        return (uint32_t)(Shape<DH>::ACC_PITCH * i);
    }
    static_assert(RQ >= 2 && RQ % NIR == 0, "tensor-memory budget");
    // every snapshot slot is consumed by one issuer only (slices s, s + kRP, ...)
    static_assert(kRP % NIR == 0, "snapshot ring must divide among the issuers");
};

template <int DH, int NIR>
__global__ void __launch_bounds__(ReadCfg<DH, NIR>::THREADS, 2)
    readout_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, ReadParams p) {
    using S = Shape<DH>;
    using L = ReadCfg<DH, NIR>;
    constexpr int RQ = L::RQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::SLOT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m = blockIdx.x, head = blockIdx.y;  // query tile, (batch, head)
    const ErrCtx err{p.err};

    const int g = m / p.cpi;               // snapshot interval of this query tile
    const int kt0 = g * p.cpi;             // first key tile of the interval
    const int n_half = 2 * (m - kt0 + 1);  // intra items: 64-key halves
    const int n_inter = (g > 0 || p.has_in) ? S::NS : 0;
    const int n_items = n_half + n_inter;
    const long row0 = (long)head * p.nch * kTile;
    // item -> issuer: the intra items (and S) on issuer 0, inter slices round-robin.
    // Each issuer owns SPI of the A-operand slots, so every slot's barriers are
    // consumed in phase order by one issuer (a parity wait only tells the
    // current phase from the one before it).
    constexpr int SPI = RQ / NIR;
    auto issuer_of = [&](int it) { return it < n_half ? 0 : (it - n_half) % NIR; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRbCount; ++i) {
            const bool four = i == kRbSFree || (i >= kRbAqFull && i < kRbAqFull + kRQMax);
            mbar_init(&bar[i], four ? 4 : (i == kRbODone ? NIR : 1));
        }
        cta_abort_clear();
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint8_t *snap =
        p.snap + ((size_t)head * p.nint + g) * S::NS * (size_t)S::SLICE_BYTES;

    if (warp == L::TMA_WARP) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&mq);
            prefetch_tensormap(&mk);
            prefetch_tensormap(&mv);
            int nk = 0, nv = 0, np = 0;  // tiles and slices issued
            auto load_p = [&](int s) -> bool {
                const int slot = s % kRP;
                if (s >= kRP && !mbar_wait(&bar[kRbPFree + slot], ((s / kRP) - 1) & 1, err, 0x501))
                    return false;
                mbar_arrive_expect_tx(&bar[kRbPFull + slot], S::SLICE_BYTES);
                bulk_load(sm + L::P + slot * S::SLICE_BYTES, snap + (size_t)s * S::SLICE_BYTES,
                          S::SLICE_BYTES, &bar[kRbPFull + slot]);
                ++np;
                return true;
            };
            auto load_kv = [&](int u) -> bool {
                const int y = (int)(row0 + (long)(kt0 + u) * kTile);
                if (u > 0 && !mbar_wait(&bar[kRbKFree], (u - 1) & 1, err, 0x502)) return false;
                mbar_arrive_expect_tx(&bar[kRbKFull], kTileBytes);
                tma_load_2d(sm + L::K, &mk, 0, y, &bar[kRbKFull]);
                ++nk;
                if (u > 0 && !mbar_wait(&bar[kRbVFree], (u - 1) & 1, err, 0x503)) return false;
                mbar_arrive_expect_tx(&bar[kRbVFull], S::VBYTES);
                tma_load_2d(sm + L::V, &mv, 0, y, &bar[kRbVFull]);
                ++nv;
                return true;
            };
            mbar_arrive_expect_tx(&bar[kRbQFull], kTileBytes);
            tma_load_2d(sm + L::Q, &mq, 0, (int)(row0 + (long)m * kTile), &bar[kRbQFull]);
            bool ok = load_kv(0);
            // the snapshots are written by the state kernel just before this one
            if (ok && n_inter > 0) grid_dependency_wait();
            const int first_p = n_inter < kRP ? n_inter : kRP;
            for (int s = 0; ok && s < first_p; ++s) ok = load_p(s);
            for (int u = 1; ok && u < n_half / 2; ++u) ok = load_kv(u);
            for (int s = first_p; ok && s < n_inter; ++s) ok = load_p(s);
            // no copy may still be in flight when the CTA exits. A copy is only
            // issued once the previous phase of its barrier completed, so the
            // last copy issued on each barrier is the only one to wait for.
            mbar_drain(&bar[kRbQFull], 0, err, 0x504);
            if (nk > 0) mbar_drain(&bar[kRbKFull], (nk - 1) & 1, err, 0x505);
            if (nv > 0) mbar_drain(&bar[kRbVFull], (nv - 1) & 1, err, 0x506);
            for (int s = np - kRP < 0 ? 0 : np - kRP; s < np; ++s)
                mbar_drain(&bar[kRbPFull + s % kRP], (s / kRP) & 1, err, 0x507);
        }
    } else if (warp >= 4) {
        // ---------------- MMA issuer `ii` ----------------
        const int ii = warp - 4;
        if (lane == 0) {
            const uint32_t i_s = idesc_bf16(128, 64, 0, 0);
            const uint32_t i_av = idesc_bf16(128, S::NACC, 0, 1);
            const uint32_t i_p = idesc_bf16(128, S::NSNAP, 0, 0);
            const uint32_t q_a = smem_u32(sm + L::Q), k_a = smem_u32(sm + L::K);
            const uint32_t v_a = smem_u32(sm + L::V), ones = smem_u32(sm + L::ONES);
            const uint32_t o_acc = tmem + L::o_col(ii);
            auto issue_s = [&](int j) -> bool {  // S = Q K^T for 64-key half j
                const int u = j >> 1, h = j & 1;
                if (h == 0 && !mbar_wait(&bar[kRbKFull], u & 1, err, 0x510)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    mma_ss(tmem + L::S_COL, kmaj_desc(q_a, kk), kmaj_desc(k_a + h * 64 * 128, kk),
                           i_s, kk > 0);
                mma_commit(&bar[kRbSFull]);
                if (h == 1) mma_commit(&bar[kRbKFree]);
                return true;
            };
            bool ok = true;
            if (ii == 0) ok = mbar_wait(&bar[kRbQFull], 0, err, 0x511) && issue_s(0);
            int uses = 0;  // this issuer's items so far
            for (int it = 0; ok && it < n_items; ++it) {
                if (issuer_of(it) != ii) continue;
                const int u = uses++;
                const int slot = ii * SPI + u % SPI;
                const uint32_t ph = (uint32_t)(u / SPI) & 1u;
                if (it < n_half) {
                    const int j = it, h = j & 1;
                    if (j + 1 < n_half &&
                        !(mbar_wait(&bar[kRbSFree], j & 1, err, 0x512) && issue_s(j + 1))) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&bar[kRbAqFull + slot], ph, err, 0x513) ||
                        (h == 0 && !mbar_wait(&bar[kRbVFull], (j >> 1) & 1, err, 0x514))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(o_acc, tmem + L::AQ_COL + 32 * slot + 8 * kk,
                               vones_desc<DH>(v_a, ones, 64 * h + 16 * kk), i_av, 1);
                    mma_commit(&bar[kRbAqFree + slot]);
                    if (h == 1) mma_commit(&bar[kRbVFree]);
                } else {
                    const int s = it - n_half, ps = s % kRP;
                    if (!mbar_wait(&bar[kRbPFull + ps], (s / kRP) & 1, err, 0x516) ||
                        !mbar_wait(&bar[kRbAqFull + slot], ph, err, 0x515)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t pa = smem_u32(sm + L::P + ps * S::SLICE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(o_acc, tmem + L::AQ_COL + 32 * slot + 8 * kk, kmaj_desc(pa, kk),
                               i_p, 1);
                    mma_commit(&bar[kRbAqFree + slot]);
                    mma_commit(&bar[kRbPFree + ps]);
                }
            }
            if (ok) mma_commit(&bar[kRbODone]);
            // every MMA this thread issued has completed before the teardown
            mma_commit(&bar[kRbDrain + ii]);
            mbar_drain(&bar[kRbDrain + ii], 0, err, 0x517);
        }
    } else {
        // ---------------- workers: one thread per query row ----------------
        const int i = threadIdx.x;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        {
            uint32_t z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll
            for (int a = 0; a < NIR; ++a)
#pragma unroll
                for (int j = 0; j < S::NACC / 16; ++j)
                    tmem_st16(tmem + lane_base + L::o_col(a) + 16 * j, z);
            tmem_st_wait();
            uint4 *o4 = reinterpret_cast<uint4 *>(sm + L::ONES);
            for (int x = i; x < 2048 / 16; x += kWorkers)
                o4[x] = make_uint4(kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2);
            fence_proxy_async_smem();
        }
        bool ok = warp_wait(&bar[kRbQFull], 0, err, 0x520);
        int uses0 = 0, uses1 = 0;  // items so far of issuer 0 and issuer 1
        for (int it = 0; ok && it < n_items; ++it) {
            const int iss = issuer_of(it);
            const int u = iss == 0 ? uses0++ : uses1++;
            const int slot = iss * SPI + u % SPI;
            uint32_t pk[32];
            if (it < n_half) {
                // intra: squared scores of 64 keys, causal mask on the diagonal tile
                const int j = it, h = j & 1, u = j >> 1;
                const bool diag = kt0 + u == m;
                if (!(ok = warp_wait(&bar[kRbSFull], j & 1, err, 0x521))) break;
                tc_fence_after();
                float sv[64];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_base + L::S_COL + 16 * q4, r);
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[16 * q4 + e] = __uint_as_float(r[e]);
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kRbSFree]);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int k0 = 64 * h + 2 * e;
                    const float a0 = (diag && k0 > i) ? 0.f : sv[2 * e] * sv[2 * e];
                    const float a1 = (diag && k0 + 1 > i) ? 0.f : sv[2 * e + 1] * sv[2 * e + 1];
                    pk[e] = pack_bf16x2(a0, a1);
                }
            } else {
                // inter: Phi(Q) for slice s, block pair (A, B); q[8A..8A+7] and
                // q[8B..8B+7] are 16-byte chunks A and B of this row of the Q tile
                int A, B;
                slice_blocks(it - n_half, S::NB, A, B);
                const uint32_t wgt = A < B ? 0x40004000u : 0x3F803F80u;  // 2 or 1
                const uint4 xa = *reinterpret_cast<const uint4 *>(sm + L::Q + sw128_chunk(i, A));
                const uint4 xb = *reinterpret_cast<const uint4 *>(sm + L::Q + sw128_chunk(i, B));
                const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w};
                const uint32_t wb[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const uint32_t qa =
                        hmul2((a & 1) ? bcast_hi(wa[a >> 1]) : bcast_lo(wa[a >> 1]), wgt);
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) pk[4 * a + bb] = hmul2(qa, wb[bb]);
                }
            }
            if (u >= SPI && !(ok = warp_wait(&bar[kRbAqFree + slot], (u / SPI - 1) & 1, err, 0x522)))
                break;
            tc_fence_after();
            {
                uint32_t r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = pk[e];
                tmem_st16(tmem + lane_base + L::AQ_COL + 32 * slot, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = pk[16 + e];
                tmem_st16(tmem + lane_base + L::AQ_COL + 32 * slot + 16, r);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kRbAqFull + slot]);
        }
        // epilogue: o = numerator / (denominator + eps), summed over the issuers
        if (ok) ok = warp_wait(&bar[kRbODone], 0, err, 0x523);
        tc_fence_after();
        float num[DH], den = 0.f;
#pragma unroll
        for (int n = 0; n < DH; ++n) num[n] = 0.f;
#pragma unroll
        for (int a = 0; a < NIR; ++a) {
            uint32_t r[DH / 16 + 1][16];
#pragma unroll
            for (int j = 0; j <= DH / 16; ++j) tmem_ld16(tmem + lane_base + L::o_col(a) + 16 * j, r[j]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < DH / 16; ++j)
#pragma unroll
                for (int e = 0; e < 16; ++e) num[16 * j + e] += __uint_as_float(r[j][e]);
            den += __uint_as_float(r[DH / 16][0]);
        }
        const float inv = 1.f / (den + p.eps);
        float4 *dst =
            reinterpret_cast<float4 *>(p.o + ((size_t)head * p.nch * kTile + (size_t)m * kTile + i) * DH);
#pragma unroll
        for (int n = 0; ok && n < DH; n += 4)
            dst[n / 4] = make_float4(num[n] * inv, num[n + 1] * inv, num[n + 2] * inv,
                                     num[n + 3] * inv);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Chunks per snapshot interval: longer intervals mean fewer snapshot bytes
// and more quadratic intra work per query tile.
int chunks_per_interval(int d, int nch) {
    int c = d == 64 ? 4 : 2;
    while (c > 1 && nch % c) c >>= 1;
    return c;
}

template <int DH>
size_t snapshot_bytes(long nheads, int nch) {
    const int nint = nch / chunks_per_interval(DH, nch);
    return (size_t)nheads * nint * Shape<DH>::NS * Shape<DH>::SLICE_BYTES;
}

// Sequence segments of a final-state-only pass: as many (tile, head, segment)
// CTAs as fit in one wave of two per SM (a second, partial wave costs more than
// the split saves), at most 8 segments and one chunk per segment.
int state_segments(int d, long nheads, int nch) {
    const long ctas = (long)(d == 64 ? Shape<64>::NT : Shape<32>::NT) * nheads;
    long seg = (2 * 148) / ctas;
    if (seg > 8) seg = 8;
    if (seg > nch) seg = nch;
    return seg < 1 ? 1 : (int)seg;
}

// Partial states of the segments: H then s of each segment, 256-byte aligned.
size_t partial_state_bytes(int d, long nheads, int nseg) {
    if (nseg <= 1) return 0;
    const size_t D = (size_t)d * (d + 1) / 2;
    return align_up((size_t)nseg * nheads * D * d * 4, 256) +
           align_up((size_t)nseg * nheads * D * 4, 256);
}

// out[i] = sum over the segments z = 0, 1, ... of part[z * n + i] (in that
// order), four floats per thread.
__global__ void __launch_bounds__(256) state_sum_kernel(const float4 *__restrict__ part, int nseg,
                                                        long n4, float4 *__restrict__ out) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
         i += (long)gridDim.x * blockDim.x) {
        float4 acc = part[i];
        for (int z = 1; z < nseg; ++z) {
            const float4 x = part[(size_t)z * n4 + i];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        out[i] = acc;
    }
}

cudaError_t launch_state_sum(const float *part, int nseg, size_t n, float *out,
                             cudaStream_t stream) {
    const long n4 = (long)(n / 4);
    const int blocks = (int)((n4 + 255) / 256 < 4 * 148 ? (n4 + 255) / 256 : 4 * 148);
    state_sum_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(part), nseg,
                                                 n4, reinterpret_cast<float4 *>(out));
    return after_launch();
}

// In place over the segments' partial states part[z] (z = 0 .. nseg - 1, n4
// float4s each): part[z] = part[0] + ... + part[z] for z < nseg - 1, in
// segment order, so part[z - 1] becomes the state before segment z. The last
// partial is not needed (the carry pass recomputes that segment from its carry).
__global__ void __launch_bounds__(256) state_scan_kernel(float4 *__restrict__ part, int nseg,
                                                         long n4) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
         i += (long)gridDim.x * blockDim.x) {
        float4 acc = part[i];
        for (int z = 1; z < nseg - 1; ++z) {
            const float4 x = part[(size_t)z * n4 + i];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
            part[(size_t)z * n4 + i] = acc;
        }
    }
}

cudaError_t launch_state_scan(float *part, int nseg, size_t n, cudaStream_t stream) {
    const long n4 = (long)(n / 4);
    const int blocks = (int)((n4 + 255) / 256 < 4 * 148 ? (n4 + 255) / 256 : 4 * 148);
    state_scan_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<float4 *>(part), nseg, n4);
    return after_launch();
}

// Sequence segments and their length for a call that writes snapshots (the
// scan mode): whole snapshot intervals per segment, at least two segments.
int scan_segments(int d, long nheads, int nch, int cpi, int &seg_len) {
    const int want = state_segments(d, nheads, nch);
    const int nint = nch / cpi;
    if (want < 2 || nint < 2) return 1;
    const int ipseg = (nint + want - 1) / want;  // intervals per segment
    seg_len = ipseg * cpi;
    return (nch + seg_len - 1) / seg_len;
}

template <int DH>
cudaError_t launch_state(const CUtensorMap &mk, const CUtensorMap &mv, const StateParams &sp,
                         int nheads, int nseg, cudaStream_t stream) {
    // two issuers halve the MMA issue chain of a chunk; with d = 32 the
    // accumulators are narrow enough to keep two Phi(K)^T slots as well
    constexpr int NA = DH == 64 ? 1 : 2;
    using L = StateCfg<DH, 2, NA>;
    cudaError_t e = set_smem_once<state_kernel<DH, 2, NA>>(L::BYTES);
    if (e != cudaSuccess) return e;
    state_kernel<DH, 2, NA><<<dim3(Shape<DH>::NT, nheads, nseg), L::THREADS, L::BYTES, stream>>>(
        mk, mv, sp);
    return after_launch();
}

template <int DH>
cudaError_t launch(const PrefillArgs &a, cudaStream_t stream) {
    const int nheads = a.B * a.H, nch = a.T / kTile;
    const int cpi = chunks_per_interval(DH, nch), nint = nch / cpi;
    const long rows = (long)nheads * a.T;
    const bool want_o = a.o != nullptr;
    const size_t D = (size_t)DH * (DH + 1) / 2;
    const size_t snap_bytes = want_o ? align_up(snapshot_bytes<DH>(nheads, nch), 256) : 0;
    uint8_t *snap = want_o ? static_cast<uint8_t *>(a.ws) : nullptr;
    if (want_o && a.ws_bytes < snap_bytes) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_qkv_maps(&mq, &mk, &mv, a.q, a.k, a.v, DH, rows)) return cudaErrorInvalidValue;

    StateParams sp{nch, cpi, nint, nch, a.H_in, a.s_in, a.H_out, a.s_out, snap, a.err};
    // The sequence splits into segments across CTAs when the (tile, head) CTAs
    // alone leave SMs idle and the workspace holds the segments' partial
    // states (after the snapshots, if any):
    //  - final state only: every segment accumulates its chunks from zero (the
    //    first from H_in) and the partials are summed;
    //  - with snapshots (the scan of the KATA page's s2.3, two-level): a first
    //    pass computes each segment's partial state, an exclusive prefix over
    //    the segments gives each segment the state before it, and a second pass
    //    starts every segment from that carry and writes its snapshots.
    int nseg = 1, seg_len = nch;
    if (!want_o) {
        sp.cpi = nch;
        sp.nint = 1;
        const int want = state_segments(DH, nheads, nch);
        if (want > 1) {
            seg_len = (nch + want - 1) / want;
            nseg = (nch + seg_len - 1) / seg_len;  // no empty segment
        }
    } else {
        nseg = scan_segments(DH, nheads, nch, cpi, seg_len);
    }
    float *pH = nullptr, *ps = nullptr;
    if (nseg > 1) {
        const bool room = a.ws && a.ws_bytes >= snap_bytes + partial_state_bytes(DH, nheads, nseg);
        // with snapshots, segment 0 rereads H_in in the second pass while the
        // last segment writes H_out: an H_out that aliases H_in keeps one pass
        const bool alias = want_o && a.H_in && a.H_out == a.H_in;
        if (!room || alias || (!want_o && !a.H_out)) {
            nseg = 1;
            seg_len = nch;
        } else {
            uint8_t *base = static_cast<uint8_t *>(a.ws) + snap_bytes;
            pH = reinterpret_cast<float *>(base);
            ps = reinterpret_cast<float *>(base + align_up((size_t)nseg * nheads * D * DH * 4, 256));
        }
    }
    sp.seg_len = seg_len;
    cudaError_t e;
    if (nseg > 1) {
        // pass 1: each segment's partial state (no snapshots)
        StateParams p1 = sp;
        p1.cpi = nch;
        p1.nint = 1;
        p1.snap = nullptr;
        p1.H_out = pH;
        p1.s_out = ps;
        if ((e = launch_state<DH>(mk, mv, p1, nheads, nseg, stream)) != cudaSuccess) return e;
        if (!want_o) {
            if ((e = launch_state_sum(pH, nseg, (size_t)nheads * D * DH, a.H_out, stream)) !=
                cudaSuccess)
                return e;
            return launch_state_sum(ps, nseg, (size_t)nheads * D, a.s_out, stream);
        }
        // the state before each segment, then pass 2 from those carries
        if ((e = launch_state_scan(pH, nseg, (size_t)nheads * D * DH, stream)) != cudaSuccess ||
            (e = launch_state_scan(ps, nseg, (size_t)nheads * D, stream)) != cudaSuccess)
            return e;
        sp.scan = 1;
        sp.carry_H = pH;
        sp.carry_s = ps;
    }
    if ((e = launch_state<DH>(mk, mv, sp, nheads, nseg, stream)) != cudaSuccess) return e;
    if (!want_o) return cudaSuccess;
    ReadParams rp{nch, cpi, nint, a.H_in != nullptr ? 1 : 0, snap, a.o, a.eps, a.err};
    // two issuers where the accumulators leave room for them (d = 32)
    constexpr int NIR = DH == 64 ? 1 : 2;
    using R = ReadCfg<DH, NIR>;
    auto kern = readout_kernel<DH, NIR>;
    e = set_smem_once<readout_kernel<DH, NIR>>(R::BYTES);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: overlap this grid's setup and intra-chunk
    // work with the end of the state kernel
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nch, nheads, 1);
    cfg.blockDim = dim3(R::THREADS, 1, 1);
    cfg.dynamicSmemBytes = R::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, rp);
    if (e != cudaSuccess) return e;
    return after_launch();
}

}  // namespace

bool prefill_tc_supported(const PrefillArgs &a) {
    return a.dtype == 1 && (a.d == 64 || a.d == 32) && a.T % kTile == 0 &&
           (long)a.B * a.H * a.T < (1L << 31) && a.B * a.H <= 65535 &&
           (reinterpret_cast<uintptr_t>(a.q) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(a.k) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(a.v) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(a.ws) & 15) == 0;
}

size_t prefill_tc_workspace_bytes(int B, int H, int T, int d, int) {
    if (T % kTile || (d != 32 && d != 64)) return 0;
    const long nheads = (long)B * H;
    const int nch = T / kTile;
    // a final-state-only call: the segments' partial states; a call with o:
    // the snapshots, then the partial states of the scan's segments
    const size_t snaps = align_up(d == 32 ? snapshot_bytes<32>(nheads, nch)
                                          : snapshot_bytes<64>(nheads, nch), 256);
    const size_t parts = partial_state_bytes(d, nheads, state_segments(d, nheads, nch));
    int seg_len = nch;
    const int nscan = scan_segments(d, nheads, nch, chunks_per_interval(d, nch), seg_len);
    const size_t with_o = snaps + (nscan > 1 ? partial_state_bytes(d, nheads, nscan) : 0);
    return with_o > parts ? with_o : parts;
}

cudaError_t prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
    return a.d == 64 ? launch<64>(a, stream) : launch<32>(a, stream);
}

}  // namespace kata
