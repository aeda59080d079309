/*
 * kata.h -- C ABI of libkata.so: causal kernelized linear attention with the
 * rank-one PSD feature phi(x) = x x^T, and the LoLA self-recall-error sparse
 * cache, on NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section):
 *   [KATA] "Kernelized Linear Attention: Breaking the Capacity Wall with
 *          Symmetric Cones": s1 (fixed-size recurrent state, constant-time
 *          recurrent inference), s2.1 (the normalising denominator is a
 *          parameter-free convex output gate), s2.2 (psi(u) = u u^T, whose
 *          inner products are squared raw inner products), s2.3 (chunked
 *          parallelism: tensor cores inside a chunk, state propagated across
 *          chunks; the chunked state form is exact).
 *   [LoLA] "LoLA: Low-Rank Linear Attention with Sparse Caching":
 *          Methodology 1-3 (sliding window, recurrent state H_t with
 *          normaliser s_t, sparse global cache), "Self-Recall Error",
 *          "Inference strategy" steps 1-4.
 *
 * Conventions shared by every entry point
 *   - Shapes are row-major (C order). B = batch, H = heads, T = tokens,
 *     d = head dimension (keys, queries and values all have d columns),
 *     D = d(d+1)/2 = packed feature dimension.
 *   - Packed state layout (the checkpoint format): phi(x) is the upper
 *     triangle of x x^T, row (a) major; entry (a, b), a <= b, sits at index
 *     a*d - a(a-1)/2 + (b - a) and carries a factor sqrt(2) when a < b, so
 *     that <phi(x), phi(y)> = (x.y)^2 exactly. The state is
 *     H [B, H, D, d] fp32 = sum_j phi(k_j) v_j^T and s [B, H, D] fp32 =
 *     sum_j phi(k_j).
 *   - Causality is inclusive: output i sees tokens j <= i. eps is added to
 *     every denominator.
 *   - Pointers named *_dev (and every pointer unless stated) are device
 *     pointers; *_host pointers are host pointers (pinned memory gives
 *     asynchronous copies). The caller owns every buffer; the library never
 *     allocates or frees memory and never synchronises the stream, except
 *     kata_sync_status.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream). Arguments are validated on the host before any
 *     launch; an invalid call returns a status and launches nothing.
 *   - Device pointers must be 16-byte aligned; d must be 16, 32 or 64.
 *   - Errors: the return value is a kata_status. kata_last_error() gives a
 *     one-line, thread-local description of the last failure on this thread.
 *     Device-side failures (a bounded wait that ran out) set a per-device
 *     error word that kata_sync_status() reads back and clears.
 */
#ifndef KATA_H
#define KATA_H

#include <stddef.h>

#if defined(__GNUC__)
#define KATA_API __attribute__((visibility("default")))
#else
#define KATA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KATA_OK = 0,
    KATA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
    KATA_ERR_UNSUPPORTED = 2, /* valid but not built: d, chunk or dtype */
    KATA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    KATA_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out */
    KATA_ERR_WORKSPACE = 5,   /* workspace missing or too small */
    KATA_ERR_BOUNDS = 6       /* debug library only: a device-side bounds check failed */
} kata_status;

typedef enum { KATA_F32 = 0, KATA_BF16 = 1 } kata_dtype; /* dtype of q, k, v */

/* Library version (major*10000 + minor*100 + patch). */
KATA_API int kata_version(void);
/* Short name of a status code. */
KATA_API const char *kata_status_string(int status);
/* Description of the last failure on the calling thread ("" if none). */
KATA_API const char *kata_last_error(void);
/* D = d(d+1)/2. */
KATA_API long kata_packed_dim(int d);
/* Number of kernels this library has launched in this process (all devices,
 * all threads); a diagnostic for counting launches inside a timed region. */
KATA_API unsigned long long kata_launch_count(void);

/*
 * Synchronise `stream`, then read and clear this device's error word.
 * Returns KATA_OK, KATA_ERR_TIMEOUT (a kernel's bounded wait ran out and the
 * kernel returned early: its outputs are invalid) or KATA_ERR_CUDA.
 */
KATA_API int kata_sync_status(void *stream);

/* --------------------------------------------------------------- prefill -- */

/* Device workspace bytes kata_prefill needs for these sizes (may be 0). */
KATA_API size_t kata_prefill_workspace_bytes(int B, int H, int T, int d, int chunk, int dtype);

/*
 * Causal chunked prefill [KATA s2.2, s2.3]:
 *   o_i = phi(q_i)^T H_i / (phi(q_i)^T s_i + eps),
 *   H_i = H_in + sum_{j<=i} phi(k_j) v_j^T,  s_i = s_in + sum_{j<=i} phi(k_j),
 * computed chunk by chunk (chunk tokens at a time): inside a chunk the masked
 * (Q K^T)^2 [V | 1] contraction, across chunks the carried state.
 *
 *   q, k, v   [B, H, T, d], dtype KATA_F32 or KATA_BF16.
 *   H_in, s_in  initial state [B, H, D, d] / [B, H, D] fp32, packed layout;
 *             both NULL = zero state; both or neither.
 *   o         [B, H, T, d] fp32 output (NULL: state only).
 *   H_out, s_out  final state, packed layout (NULL: not written; both or
 *             neither). May alias H_in / s_in.
 *   chunk     16, 32, 64 or 128; T must be a positive multiple of chunk.
 *   workspace device scratch of at least kata_prefill_workspace_bytes().
 * bf16 inputs run on the tcgen05 tensor cores (bf16 operands, fp32
 * accumulation and state); fp32 inputs run in fp32 on the CUDA cores.
 * An output-only bf16 call (no H_in, no H_out) with T up to
 * kata_quadratic_max_tokens(d) runs the quadratic form instead (see
 * kata_prefill_ex); the result is the same up to rounding.
 */
KATA_API int kata_prefill(const void *q, const void *k, const void *v, int dtype, int B, int H, int T,
                 int d, int chunk, float eps, const float *H_in, const float *s_in, float *o,
                 float *H_out, float *s_out, void *workspace, size_t ws_bytes, void *stream);

/* Which kernel the chunked form runs for these sizes: 1 = tcgen05 tensor
 * cores, 0 = CUDA cores, -1 = invalid or unsupported arguments. */
KATA_API int kata_prefill_path(int B, int H, int T, int d, int chunk, int dtype);

/*
 * Test hook for failure detection (no counterpart on the pages). Runs the
 * quadratic form of kata_prefill (bf16 q, k, v [B, H, T, d], d = 32 or 64,
 * T a multiple of 128, zero initial state) with one deliberate fault: in
 * every CTA, the warp that issues the P [V | 1] MMAs first waits on a barrier
 * that nothing ever arrives at, giving up after `polls` polls (1 .. 2^20).
 * The CTA then takes its error path: every role stops waiting, drains the
 * copies and MMAs it issued, frees its tensor memory and exits; o is not
 * valid. The next kata_sync_status() on this device returns
 * KATA_ERR_TIMEOUT with the site code 0x6FF (kata_last_error()), and the
 * context stays usable for the calls that follow.
 */
KATA_API int kata_test_forced_timeout(const void *q, const void *k, const void *v, int B, int H,
                                      int T, int d, float eps, float *o, unsigned int polls,
                                      void *stream);

/*
 * The debug library (libkata_debug.so, the same sources built with
 * -DKATA_DEBUG; no counterpart on the pages) adds device-side bounds checks
 * where an index comes from device data or a size another kernel produced:
 * candidate slots, kept and merged lists, cache rows, output rows. A check
 * that fails records its site code (0xB000 .. 0xBFFF) in the device error
 * word and the access is skipped, so a bad index turns into a status instead
 * of a memory fault: the next kata_sync_status() returns KATA_ERR_BOUNDS with
 * the code in kata_last_error(), and the outputs of that call are invalid.
 * kata_debug_build() returns 1 in the debug library and 0 in libkata.so.
 */
KATA_API int kata_debug_build(void);

/*
 * Test hook of the debug library: launches one tiny kernel whose checked store
 * targets index 7 of a 4-element device array, so the check fails, records
 * site code 0xB001 and skips the store. The next kata_sync_status() returns
 * KATA_ERR_BOUNDS. The normal library returns KATA_ERR_UNSUPPORTED and
 * launches nothing (its checks are compiled out).
 */
KATA_API int kata_test_bounds_check(void *stream);

/* The two exact forms of a prefill. */
enum { KATA_FORM_AUTO = 0, KATA_FORM_CHUNKED = 1, KATA_FORM_QUADRATIC = 2 };

/*
 * kata_prefill with the form chosen by the caller.
 *   KATA_FORM_CHUNKED    the chunked state form described at kata_prefill.
 *   KATA_FORM_QUADRATIC  o by the quadratic form [KATA s2.2: the rank-one PSD
 *                        feature makes the kernel (q.k)^2]:
 *                          o_i = sum_{j<=i} (q_i.k_j)^2 v_j / (sum_{j<=i} (q_i.k_j)^2 + eps),
 *                        O(T^2 d) work on the tcgen05 tensor cores with no
 *                        state (bf16 (q.k)^2 operands, fp32 accumulation). It
 *                        takes bf16 inputs, d = 32 or 64, T a multiple of 128,
 *                        o non-NULL and H_in, s_in NULL; other calls return
 *                        KATA_ERR_UNSUPPORTED. With H_out, s_out the final
 *                        state is computed by the chunked form's state pass
 *                        at the same time, on a second stream the library
 *                        forks from `stream` and joins back to it with events
 *                        (one per device, shared by the calling threads; a
 *                        call made while `stream` is being captured into a
 *                        CUDA graph brings the side stream into the capture,
 *                        so no other thread may use this form on the same
 *                        device during the capture). workspace is not used
 *                        (may be NULL, ws_bytes 0).
 *   KATA_FORM_AUTO       what kata_prefill does: the quadratic form for a call
 *                        without H_in and H_out when it applies and
 *                        T <= kata_quadratic_max_tokens(d), the chunked form
 *                        otherwise.
 * Both forms give the same result up to rounding.
 */
KATA_API int kata_prefill_ex(const void *q, const void *k, const void *v, int dtype, int B, int H,
                    int T, int d, int chunk, float eps, const float *H_in, const float *s_in,
                    float *o, float *H_out, float *s_out, void *workspace, size_t ws_bytes,
                    void *stream, int form);

/* Largest T for which KATA_FORM_AUTO takes the quadratic form (0: never). */
KATA_API int kata_quadratic_max_tokens(int d);

/* The form KATA_FORM_AUTO takes for these sizes: KATA_FORM_CHUNKED or
 * KATA_FORM_QUADRATIC; with_state = H_in or H_out given (such calls take the
 * chunked form). -1 = invalid or unsupported arguments. */
KATA_API int kata_prefill_auto_form(int B, int H, int T, int d, int chunk, int dtype,
                                    int with_state);

/* Device workspace for kata_prefill_host: staging for q, k, v and o plus
 * kata_prefill_workspace_bytes(). */
KATA_API size_t kata_prefill_host_workspace_bytes(int B, int H, int T, int d, int chunk, int dtype);

/*
 * kata_prefill with host inputs and output: copies q_host, k_host, v_host to
 * device staging inside `workspace`, runs kata_prefill from a zero state, and
 * copies o back to o_host. The heads are processed in two pieces of
 * consecutive heads (each head is independent), one on `stream` and one on a
 * second stream the library keeps per device, so the host-to-device
 * copies of one piece overlap the kernels and the device-to-host copy of
 * another; `stream` is made to wait for the second stream before the call
 * returns. Everything is asynchronous with respect to the host: the caller
 * synchronises `stream` before reading o_host, and pinned host buffers are
 * needed for the copies to overlap. The result equals kata_prefill's on the
 * same inputs (the same kernels per head; the chunked form may split a
 * piece's sequence differently, which changes fp32 rounding only).
 */
KATA_API int kata_prefill_host(const void *q_host, const void *k_host, const void *v_host, int dtype,
                      int B, int H, int T, int d, int chunk, float eps, float *o_host,
                      void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------ multi-factor features -- */

/*
 * The feature variants of [KATA s2.3 "Variants"]: KATA-Mg (several PSD
 * factors) and KATA-Sigma-g (summed PSD factors). The page does not say how
 * the factors are formed; this library reads them as follows. The head vector
 * x (d values) is cut into g contiguous sub-vectors x_r of p = d/g values, and
 * each gives the rank-one PSD factor x_r x_r^T of s2.2:
 *   KATA_FEATURE_RANK1   psi(x) = x x^T (g = 1)          kernel (q.k)^2
 *   KATA_FEATURE_MG      psi(x) = the g factors apart     kernel sum_r (q_r.k_r)^2
 *   KATA_FEATURE_SIGMAG  psi(x) = sum_r x_r x_r^T         kernel sum_{r,t} (q_r.k_t)^2
 * State layout: each symmetric p x p block as the packed upper triangle
 * (sqrt(2) off the diagonal, as for the rank-one feature); Mg stores its g
 * blocks one after another. The state has kata_feature_dim(d, feature, g)
 * rows: d(d+1)/2, g p(p+1)/2 or p(p+1)/2. g must divide d with p >= 8.
 */
enum { KATA_FEATURE_RANK1 = 0, KATA_FEATURE_MG = 1, KATA_FEATURE_SIGMAG = 2 };

/* Rows of the state of a feature (0: invalid d, feature or g). */
KATA_API long kata_feature_dim(int d, int feature, int g);

/*
 * kata_prefill with a multi-factor feature: o_i = psi(q_i)^T H_i /
 * (psi(q_i)^T s_i + eps), H_i = H_in + sum_{j<=i} psi(k_j) v_j^T, computed in
 * the chunked form (intra-chunk kernel sum plus the carried state) on the CUDA
 * cores in fp32, for fp32 or bf16 inputs. Arguments as kata_prefill, with
 * H_in/H_out [B, H, Df, d] and s_in/s_out [B, H, Df], Df = kata_feature_dim().
 * workspace: needed only when s_out aliases s_in (B*H*Df floats).
 * KATA_FEATURE_RANK1 is kata_prefill itself.
 */
KATA_API int kata_prefill_feature(const void *q, const void *k, const void *v, int dtype, int B,
                                  int H, int T, int d, int chunk, float eps, int feature, int g,
                                  const float *H_in, const float *s_in, float *o, float *H_out,
                                  float *s_out, void *workspace, size_t ws_bytes, void *stream);

/* kata_decode_step with a multi-factor feature (state [B, H, Df, d], [B, H, Df]). */
KATA_API int kata_decode_step_feature(const void *q, const void *k, const void *v, int dtype,
                                      int B, int H, int d, float eps, int feature, int g,
                                      float *Hst, float *s, float *o, void *stream);

/* ------------------------------------------------- split sequences ------ */

/*
 * Exclusive prefix sums of states over the parts of a sequence [KATA s2.3:
 * the state propagates across blocks as a prefix sum]. For a prefill whose
 * sequence is split into nparts consecutive parts (one per device, say):
 *   H_prefix[z] = H_parts[0] + ... + H_parts[z-1],  H_prefix[0] = 0,
 * and the same for s, summed in part order; part z then runs kata_prefill
 * with H_in = H_prefix[z], s_in = s_prefix[z] and gets the outputs and state
 * of the whole sequence up to its end. H_parts, H_prefix [nparts, B, H, Df, d]
 * and s_parts, s_prefix [nparts, B, H, Df] fp32, Df =
 * kata_feature_dim(d, feature, g); the prefixes must not overwrite the parts.
 */
KATA_API int kata_state_prefix(const float *H_parts, const float *s_parts, int nparts, int B,
                               int H, int d, int feature, int g, float *H_prefix,
                               float *s_prefix, void *stream);

/* ---------------------------------------------------------------- decode -- */

/*
 * One decode step per (b, h) [KATA s1 "constant-time recurrent inference"]:
 *   H += phi(k) v^T;  s += phi(k);  o = phi(q)^T H / (phi(q)^T s + eps)
 * (update first, then read out). The state is updated IN PLACE.
 *   q, k, v   [B, H, d], dtype KATA_F32 or KATA_BF16.
 *   Hst, s    [B, H, D, d] / [B, H, D] fp32, packed layout, read and written.
 *   o         [B, H, d] fp32.
 */
KATA_API int kata_decode_step(const void *q, const void *k, const void *v, int dtype, int B, int H,
                     int d, float eps, float *Hst, float *s, float *o, void *stream);

/*
 * kata_decode_step with host q, k, v and o: staging (3 * B*H*d elements of
 * dtype, then B*H*d fp32, each part 256-byte aligned) lives in `workspace`;
 * the state stays on the device.
 */
KATA_API int kata_decode_step_host(const void *q_host, const void *k_host, const void *v_host,
                          int dtype, int B, int H, int d, float eps, float *Hst, float *s,
                          float *o_host, void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------ LoLA -- */

/* Device workspace bytes lola_sre_score_topk needs. */
KATA_API size_t lola_sre_workspace_bytes(int B, int H, int d, int n_cand);

/*
 * Self-recall error and top-k retention [LoLA "Self-Recall Error",
 * "Inference strategy" steps 1-3]:
 *   SRE_j = || phi(k_j)^T H / (phi(k_j)^T s + eps) - v_j ||^2
 * for the n_cand candidates of every (b, h), scored against (Hst, s). The
 * min(keep, n_cand) highest scores are kept (an exact tie goes to the smaller
 * position); with merge = 1 every other candidate is added to the state,
 * H += phi(k_j) v_j^T, s += phi(k_j).
 *   Hst, s     [B, H, D, d] / [B, H, D] fp32 state to score against.
 *   kc, vc     [B, H, n_cand, d] candidates, dtype KATA_F32 or KATA_BF16.
 *   pos        [B, H, n_cand] int32 token positions, distinct within a head.
 *   scores     [B, H, n_cand] fp32 SRE (NULL: not written).
 *   keep_idx   [B, H, min(keep, n_cand)] int32 kept candidate slots in
 *              ascending position.
 *   Hst_mut, s_mut  merged state (merge = 1; may alias Hst / s; ignored when
 *              merge = 0).
 *   1 <= n_cand <= 1024, 0 <= keep.
 */
KATA_API int lola_sre_score_topk(const float *Hst, const float *s, const void *kc, const void *vc,
                        const int *pos, int dtype, int B, int H, int d, int n_cand, int keep,
                        float eps, int merge, float *scores, int *keep_idx, float *Hst_mut,
                        float *s_mut, void *workspace, size_t ws_bytes, void *stream);

/*
 * lola_sre_score_topk without a workspace argument. (The pages have no
 * counterpart: this is a calling convenience of this library.)
 *
 * For callers that cannot allocate device memory when they score candidates,
 * for example a serving loop whose memory pool is sized once and must not
 * grow, or a host program with no device allocator of its own. The scratch
 * the scoring needs comes from one fixed array of 8 MiB of device memory that
 * the library holds on every GPU it is loaded on, until the process exits.
 * This call allocates nothing.
 *
 * Arguments, results and errors are those of lola_sre_score_topk. Sizes whose
 * scratch would exceed 8 MiB (lola_sre_workspace_bytes() > 8 MiB; for d = 64
 * and 192 candidates, up to 33 heads B*H) return KATA_ERR_WORKSPACE with the
 * numbers in kata_last_error().
 *
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture. Every call
 * shares the one array and it keeps what the last call left there (nothing in
 * it needs to start at zero). Two calls whose kernels overlap on the GPU, from
 * different streams or host threads, race on the array: serialise them.
 */
KATA_API int lola_sre_score_topk_noalloc(const float *Hst, const float *s, const void *kc,
                                         const void *vc, const int *pos, int dtype, int B,
                                         int H, int d, int n_cand, int keep, float eps,
                                         int merge, float *scores, int *keep_idx,
                                         float *Hst_mut, float *s_mut, void *stream);

/* Device workspace bytes lola_hybrid_readout needs. */
KATA_API size_t lola_readout_workspace_bytes(int B, int H, int d, int nq);

/*
 * Hybrid readout of one segment [LoLA "Inference strategy" step 4,
 * Methodology 1-3], one shared denominator:
 *   o_i = [ sum_{j in W_i u S} exp(tau q_i.k_j) v_j + phi(q_i)^T H ]
 *       / [ sum_{j in W_i u S} exp(tau q_i.k_j) + phi(q_i)^T s + eps ]
 * for queries i = seg0 .. seg0+nq-1, window W_i = positions [w0, i] of k, v,
 * sparse cache S = the first nc pairs of ck, cv.
 *   q, k, v    [B, H, T, d] whole sequences, dtype KATA_F32 or KATA_BF16.
 *   ck, cv     [B, H, cap, d] cache pairs, same dtype (nc <= cap).
 *   Hst, s     state, packed layout.
 *   o          [B, H, T, d] fp32; rows seg0 .. seg0+nq-1 are written.
 *   0 <= w0 <= seg0, seg0 + nq <= T, 1 <= nq <= 256, seg0 + nq - w0 <= 1024.
 */
KATA_API int lola_hybrid_readout(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int T, int d, int seg0, int nq, int w0, const void *ck,
                        const void *cv, int nc, int cap, const float *Hst, const float *s,
                        float eps, float tau, float *o, void *workspace, size_t ws_bytes,
                        void *stream);

/* Device workspace bytes lola_prefill needs. */
KATA_API size_t lola_prefill_workspace_bytes(int B, int H, int T, int d, int window, int cache);

/*
 * The whole LoLA schedule over a sequence [LoLA "Inference strategy" 1-4],
 * segment by segment (segment length = window):
 *   for g = 0, 1, ...: read out segment g (lola_hybrid_readout with window
 *   start max(0, window*(g-1))); then, for g >= 1, segment g-1 leaves the
 *   window: its pairs and the cached pairs are scored by SRE against the
 *   current state, the `cache` highest stay cached and the rest are merged.
 *   q, k, v    [B, H, T, d]; T a positive multiple of window.
 *   window     1..256; cache 0..1024 (window + cache <= 1024).
 *   tau        softmax scale for window and cache pairs (1/sqrt(d) usual).
 *   o          [B, H, T, d] fp32.
 *   Hst, s     state in/out, packed layout (zero it for a fresh sequence).
 *   kept_pos   optional [T/window - 1, B, H, cache] int32: the cached token
 *              positions after each update, ascending, -1 padded (NULL: not
 *              written).
 */
KATA_API int lola_prefill(const void *q, const void *k, const void *v, int dtype, int B, int H, int T,
                 int d, int window, int cache, float eps, float tau, float *o, float *Hst,
                 float *s, int *kept_pos, void *workspace, size_t ws_bytes, void *stream);

/* How lola_prefill runs the schedule. */
enum { LOLA_RUN_AUTO = 0, LOLA_RUN_SEGMENTS = 1, LOLA_RUN_FUSED = 2 };
/* LOLA_RUN_FUSED with exactly n CTAs per (b, h), n = 6 .. 8 (tests, tuning). */
#define LOLA_RUN_FUSED_NCL(n) (10 + (n))

/*
 * lola_prefill with the execution chosen by the caller; the results are the
 * same up to fp32 rounding.
 *   LOLA_RUN_SEGMENTS  a few launches per segment (readout, SRE scoring,
 *                      top-k, merge, cache bookkeeping); any size above.
 *   LOLA_RUN_FUSED     one launch for the whole sequence: a cluster of n CTAs
 *                      per (b, h) keeps that head's fp32 state in shared memory
 *                      (each CTA 1/n of the packed rows) from the first segment
 *                      to the last, and writes it back once; n is the largest of
 *                      8, 7, 6 for which every head's cluster is resident at
 *                      once on the device (8 if none is). A cached pair's
 *                      phi(k)^T [H | s] is carried from update to update by the
 *                      merged pairs, (k . k_m)^2 v_m [KATA s2.2], instead of
 *                      being recomputed against the whole state. Sizes:
 *                      window a multiple of 8 up to 64, 2*window + cache <= 256,
 *                      d * element size <= 128 bytes (bf16 d <= 64, fp32 d <= 32);
 *                      other sizes return KATA_ERR_UNSUPPORTED.
 *   LOLA_RUN_AUTO      fused when the sizes allow it, segments otherwise
 *                      (what lola_prefill does).
 * lola_prefill_workspace_bytes() covers both.
 */
KATA_API int lola_prefill_ex(const void *q, const void *k, const void *v, int dtype, int B, int H,
                             int T, int d, int window, int cache, float eps, float tau, float *o,
                             float *Hst, float *s, int *kept_pos, void *workspace,
                             size_t ws_bytes, void *stream, int run);

/* 1 if LOLA_RUN_FUSED takes these sizes (LOLA_RUN_AUTO then runs it), else 0. */
KATA_API int lola_prefill_fused_applies(int dtype, int d, int window, int cache);

#ifdef __cplusplus
}
#endif

#endif /* KATA_H */
