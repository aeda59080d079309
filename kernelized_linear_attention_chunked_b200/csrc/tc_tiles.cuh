// Tile shapes, operand descriptors and tensor maps shared by the tcgen05
// prefill kernels (prefill_tc.cu: the chunked form; quad_tc.cu: the quadratic
// form). bf16 q, k, v rows of d = 32 or 64 elements, 128-token tiles.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "sm100.cuh"

namespace kata {
namespace tc {

using namespace sm100;

constexpr int kTile = 128;         // tokens per chunk / query tile; rows per state tile
constexpr int kTileBytes = 16384;  // one 128 x 64 bf16 tile, 128-byte swizzle
constexpr int kWorkers = 128;      // 4 warps: one thread per tensor-memory lane
constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;

template <int DH>
struct Shape {
    static constexpr int NB = DH / 8;             // 8-wide index blocks
    static constexpr int NS = NB * (NB + 1) / 2;  // 64-feature slices
    static constexpr int NT = (NS + 1) / 2;       // 128-row state tiles
    static constexpr int NSNAP = DH + 16;         // snapshot rows: H | s x 16
    static constexpr int SLICE_BYTES = NSNAP * 128;
    static constexpr int NACC = DH + 16;          // accumulator columns: H | s x 16
    static constexpr int SCOL = DH;               // first accumulator column holding s
    static constexpr int ACC_PITCH = DH == 64 ? 96 : 64;  // tensor-memory columns per accumulator
    static constexpr int VROW = 2 * DH;           // bytes per V row (one swizzle atom)
    static constexpr int VBYTES = kTile * VROW;
    static constexpr uint32_t VSW = DH == 64 ? kSwizzle128 : kSwizzle64;
};

// One warp-uniform wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const ErrCtx &err,
                                          unsigned int code) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err, code) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    return ok != 0;
}

// MN-major [V | 1] operand for 16 tokens starting at row `row0` of the V tile:
// the V tile (d bf16 per row) is the first atom; the second atom is a 16-row
// all-ones block, reached through the leading byte offset from this K-step's
// start (every row of it is the same).
template <int DH>
__device__ __forceinline__ uint64_t vones_desc(uint32_t v, uint32_t ones, int row0) {
    using S = Shape<DH>;
    const uint32_t start = v + row0 * S::VROW;
    return smem_desc(start, ones - start, 8 * S::VROW, S::VSW);
}

// K-major operand: 128-byte rows, 16 K-elements at byte offset 32 * kk.
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int kk) {
    return smem_desc(base + 32 * kk, 16, 1024, kSwizzle128);
}

// Fill the 2 KB all-ones block of the [V | 1] operand (threads 0..n-1 of the
// calling group) and make it visible to the tensor cores' operand reads.
__device__ __forceinline__ void fill_ones(uint8_t *ones, int t, int n) {
    uint4 *o4 = reinterpret_cast<uint4 *>(ones);
    for (int i = t; i < 2048 / 16; i += n)
        o4[i] = make_uint4(kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2);
    fence_proxy_async_smem();
}

// ------------------------------------------------------------------ host --

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Raise `Kern`'s dynamic shared-memory limit to `bytes` once per device (the
// attribute is per device; setting it on every launch costs host time).
template <auto Kern>
inline cudaError_t set_smem_once(int bytes) {
    static std::atomic<unsigned long long> done{0};  // one bit per device ordinal < 64
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// [rows, d] bf16 rows in boxes of 128 rows x box_x columns. Q and K use
// box_x = 64 with the 128-byte swizzle (for d = 32 the box reaches past the row
// and the extra columns are zero-filled); V uses box_x = d, one swizzle atom
// (128-byte swizzle for d = 64, 64-byte for d = 32).
inline bool make_map(CUtensorMap *m, const void *base, int d, long rows, int box_x,
                     CUtensorMapSwizzle sw) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)kTile};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The three maps of a q, k, v set of `rows` rows of d elements.
inline bool make_qkv_maps(CUtensorMap *mq, CUtensorMap *mk, CUtensorMap *mv, const void *q,
                          const void *k, const void *v, int d, long rows) {
    const CUtensorMapSwizzle vsw = d == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return make_map(mq, q, d, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map(mk, k, d, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map(mv, v, d, rows, d, vsw);
}

}  // namespace tc
}  // namespace kata
