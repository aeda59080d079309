// Host-side interfaces between the C ABI (kata_abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace kata {

struct PrefillArgs {
    const void *q, *k, *v;
    int dtype;  // 0 = fp32, 1 = bf16
    int B, H, T, d, chunk;
    float eps;
    const float *H_in, *s_in;
    float *o, *H_out, *s_out;
    void *ws;
    size_t ws_bytes;
    unsigned int *err;  // per-device error word
    int feature = 0;    // kFeatRank1, kFeatMg or kFeatSigmaG (kata_common.cuh)
    int g = 1;          // factors of a multi-factor feature
};

// fp32 CUDA-core path: any supported d and chunk, fp32 or bf16 inputs.
cudaError_t prefill_simt(const PrefillArgs &a, cudaStream_t stream);

// tcgen05 tensor-core path (bf16 inputs). Returns cudaErrorNotSupported when
// the shape is not one it takes; the caller then uses the CUDA-core path.
bool prefill_tc_supported(const PrefillArgs &a);
size_t prefill_tc_workspace_bytes(int B, int H, int T, int d, int chunk);
cudaError_t prefill_tc(const PrefillArgs &a, cudaStream_t stream);

// tcgen05 quadratic form: o only, from a zero state; H_in, H_out, ws are
// ignored. quad_tc_shape_ok tells the sizes it takes (bf16, d = 32 or 64, T a
// multiple of 128); the caller checks that q, k, v, o are 16-byte aligned.
// `stall` > 0 is the forced-timeout test hook (the kernel's error path runs
// after a wait of at most `stall` polls on a barrier nothing arrives at).
bool quad_tc_shape_ok(int dtype, int B, int H, int T, int d);
cudaError_t quad_tc(const PrefillArgs &a, cudaStream_t stream, unsigned int stall = 0);

// One decode step; feature / g select a multi-factor feature (kFeatRank1: s2.2's).
cudaError_t decode_step(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int d, float eps, float *Hst, float *s, float *o, cudaStream_t stream,
                        int feature = 0, int g = 1);

// LoLA pieces (lola.cu).
size_t sre_workspace_bytes(int B, int H, int d, int n_cand);
cudaError_t sre_score_topk(const float *Hst, const float *s, const void *kc, const void *vc,
                           const int *pos, int dtype, int B, int H, int d, int n_cand,
                           int cand_stride, int keep, float eps, int merge, float *scores,
                           int *keep_idx, float *Hst_mut, float *s_mut, void *ws,
                           size_t ws_bytes, cudaStream_t stream);
// Same as sre_score_topk with scratch in a fixed device array (no caller
// workspace); sre_noalloc_capacity() is that array's size in bytes.
size_t sre_noalloc_capacity();
cudaError_t sre_score_topk_noalloc(const float *Hst, const float *s, const void *kc,
                                   const void *vc, const int *pos, int dtype, int B, int H,
                                   int d, int n_cand, int keep, float eps, int merge,
                                   float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                                   cudaStream_t stream);
size_t readout_workspace_bytes(int B, int H, int d, int nq);
// The SRE step on the tensor cores (sre_tc.cu): bf16 candidates, d = 32 or
// 64, 1 <= n <= 256, 16-byte aligned state and candidate buffers; no workspace.
bool sre_tc_applies(int dtype, int d, int n, const float *Hst, const float *s,
                    const float *Hst_mut, const float *s_mut, const void *kc, const void *vc);
cudaError_t sre_tc(const float *Hst, const float *s, const void *kc, const void *vc,
                   const int *pos, int nh, int d, int n, int cand_stride, int keep, float eps,
                   int merge, float *scores, int *keep_idx, float *Hst_mut, float *s_mut,
                   unsigned int *err, cudaStream_t stream);
// This device's error word (kata_abi.cu): kernels record a timed-out wait there.
unsigned int *device_error_word();
cudaError_t hybrid_readout(const void *q, const void *k, const void *v, int dtype, int B,
                           int H, int T, int d, int seg0, int nq, int w0, const void *ck,
                           const void *cv, int nc, int cap, const float *Hst, const float *s,
                           float eps, float tau, float *o, void *ws, size_t ws_bytes,
                           cudaStream_t stream);
size_t lola_workspace_bytes(int B, int H, int T, int d, int window, int cache);
// The schedule as segment-by-segment launches (any supported size).
cudaError_t lola_run(const void *q, const void *k, const void *v, int dtype, int B, int H,
                     int T, int d, int window, int cache, float eps, float tau, float *o,
                     float *Hst, float *s, int *kept_pos, void *ws, size_t ws_bytes,
                     cudaStream_t stream);

// The schedule as one launch, a cluster of CTAs per head holding the state on
// chip (lola_fused.cu): the sizes lola_fused_applies() accepts; the scratch is
// lola_fused_scratch_bytes() of device memory. ncl = CTAs per head (6 to 8), or
// 0: the largest that keeps every head's cluster resident at once.
bool lola_fused_applies(int dtype, int d, int window, int cache);
size_t lola_fused_scratch_bytes(int nh, int d);
cudaError_t lola_fused(const void *q, const void *k, const void *v, int dtype, int nh, int T,
                       int d, int window, int cache, float eps, float tau, float *o, float *Hst,
                       float *s, int *kept_pos, void *scratch, int ncl, cudaStream_t stream);

// out[z] = in[0] + ... + in[z - 1] over nparts parts of n floats (n % 4 == 0,
// 16-byte aligned), summed in part order (state_ops.cu).
cudaError_t exclusive_prefix(const float *in, int nparts, size_t n, float *out,
                             cudaStream_t stream);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Called right after every kernel launch: counts it (kata_launch_count) and
// returns the launch status.
cudaError_t after_launch();

}  // namespace kata
