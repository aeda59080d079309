// C ABI of libkata.so: argument validation, dispatch, status reporting.
// The declarations and the contract of every entry point are in include/kata.h.
#include <atomic>
#include <mutex>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "../../include/kata.h"
#include "kata_common.cuh"
#include "kata_internal.h"

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(KATA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

__device__ unsigned int g_error_word;

// Per-device caches below cover device ordinals 0 .. kMaxDevices - 1.
constexpr int kMaxDevices = 128;

// Address of this device's error word (looked up once per device, with the
// device current; the lookup is serialised across host threads).
unsigned int *error_word() {
    static std::atomic<unsigned int *> addr[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned int *a = addr[dev].load(std::memory_order_acquire);
    if (a) return a;
    std::lock_guard<std::mutex> lock(mu);
    a = addr[dev].load(std::memory_order_relaxed);
    if (!a) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        a = static_cast<unsigned int *>(p);
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

std::atomic<unsigned long long> g_launches{0};

// A second stream per device for work that runs beside the caller's stream
// within one call, forked from and joined back to it with events. Slot 0
// serves the quadratic form's state pass, slot 1 the host-buffer prefill (so
// neither holds the other's lock).
struct SideStream {
    std::mutex mu;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream *side_stream(int slot = 0) {
    static SideStream sides[2][kMaxDevices];
    int dev = 0;
    if (slot < 0 || slot > 1 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    SideStream &sd = sides[slot][dev];
    std::lock_guard<std::mutex> lock(sd.mu);
    if (!sd.stream) {
        cudaStream_t st = nullptr;
        cudaEvent_t f = nullptr, j = nullptr;
        if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
            cudaStreamDestroy(st);
            return nullptr;
        }
        sd.stream = st;
        sd.fork = f;
        sd.join = j;
    }
    return &sd;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int dtype, int B, int H, int d) {
    if (dtype != KATA_F32 && dtype != KATA_BF16)
        return fail(KATA_ERR_UNSUPPORTED, "dtype %d is not KATA_F32 or KATA_BF16", dtype);
    if (B <= 0 || H <= 0) return fail(KATA_ERR_INVALID_ARG, "B=%d H=%d must be positive", B, H);
    if (d != 16 && d != 32 && d != 64)
        return fail(KATA_ERR_UNSUPPORTED, "d=%d: only 16, 32 and 64 are built", d);
    if ((long)B * H > (1L << 20)) return fail(KATA_ERR_INVALID_ARG, "B*H=%ld too large", (long)B * H);
    return KATA_OK;
}

#define KATA_REQUIRE_PTR(p)                                                        \
    do {                                                                           \
        if (!(p)) return fail(KATA_ERR_INVALID_ARG, "%s must not be NULL", #p);    \
        if (!aligned16(p))                                                         \
            return fail(KATA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);    \
    } while (0)

#define KATA_OPTIONAL_PTR(p)                                                       \
    do {                                                                           \
        if ((p) && !aligned16(p))                                                  \
            return fail(KATA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);    \
    } while (0)

size_t elem_bytes(int dtype) { return dtype == KATA_F32 ? 4 : 2; }

}  // namespace

unsigned int *kata::device_error_word() { return error_word(); }

cudaError_t kata::after_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

extern "C" {

unsigned long long kata_launch_count(void) { return g_launches.load(); }

int kata_version(void) { return 100; }

const char *kata_status_string(int status) {
    switch (status) {
        case KATA_OK: return "KATA_OK";
        case KATA_ERR_INVALID_ARG: return "KATA_ERR_INVALID_ARG";
        case KATA_ERR_UNSUPPORTED: return "KATA_ERR_UNSUPPORTED";
        case KATA_ERR_CUDA: return "KATA_ERR_CUDA";
        case KATA_ERR_TIMEOUT: return "KATA_ERR_TIMEOUT";
        case KATA_ERR_WORKSPACE: return "KATA_ERR_WORKSPACE";
        case KATA_ERR_BOUNDS: return "KATA_ERR_BOUNDS";
        default: return "KATA_ERR_UNKNOWN";
    }
}

const char *kata_last_error(void) { return g_last_error; }

long kata_packed_dim(int d) { return (long)d * (d + 1) / 2; }

int kata_sync_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int *w = error_word();
    if (!w) return fail(KATA_ERR_CUDA, "error word unavailable");
    unsigned int h = 0;
    e = cudaMemcpy(&h, w, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read error word");
    if (h != kata::kErrNone) {
        unsigned int zero = 0;
        e = cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "clear error word");
        if (h >= kata::kErrBoundsFirst && h <= kata::kErrBoundsLast)
            return fail(KATA_ERR_BOUNDS, "a device-side bounds check failed (site 0x%X)", h);
        return fail(KATA_ERR_TIMEOUT, "a kernel's bounded wait ran out (code 0x%X)", h);
    }
    return KATA_OK;
}

/* ------------------------------------------------------------- prefill --- */

static int check_prefill(int dtype, int B, int H, int T, int d, int chunk) {
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128)
        return fail(KATA_ERR_UNSUPPORTED, "chunk=%d: only 16, 32, 64, 128", chunk);
    if (T <= 0 || T % chunk)
        return fail(KATA_ERR_INVALID_ARG, "T=%d must be a positive multiple of chunk=%d", T, chunk);
    if ((long)T > (1L << 24)) return fail(KATA_ERR_INVALID_ARG, "T=%d too large", T);
    return KATA_OK;
}

static size_t prefill_ws_bytes(int B, int H, int T, int d, int chunk, int dtype) {
    // a copy of s_in, used when s_out aliases it
    size_t b = kata::align_up((size_t)B * H * kata::packed_dim(d) * sizeof(float), 256);
    if (dtype == KATA_BF16) b += kata::prefill_tc_workspace_bytes(B, H, T, d, chunk);
    return b;
}

size_t kata_prefill_workspace_bytes(int B, int H, int T, int d, int chunk, int dtype) {
    if (check_prefill(dtype, B, H, T, d, chunk)) return 0;
    return prefill_ws_bytes(B, H, T, d, chunk, dtype);
}

int kata_quadratic_max_tokens(int d) {
    // measured crossover of the output-only prefill on B200: below it the
    // quadratic form's O(T^2 d) work beats the chunked form's state carry
    return d == 32 ? 4096 : d == 64 ? 8192 : 0;
}

// The quadratic form computes o from a zero initial state.
static bool quadratic_applies(int dtype, int B, int H, int T, int d, bool from_initial_state) {
    return !from_initial_state && kata::quad_tc_shape_ok(dtype, B, H, T, d);
}

// KATA_FORM_AUTO: the quadratic form for output-only calls up to the
// crossover. With a final state the chunked form stays: running the state pass
// beside the quadratic kernel measured no faster at d = 32 (57 vs 56 us at
// B4 H8 T2048) and only wins at d = 64 for short T.
static bool auto_quadratic(int dtype, int B, int H, int T, int d, bool with_state) {
    return !with_state && quadratic_applies(dtype, B, H, T, d, false) &&
           T <= kata_quadratic_max_tokens(d);
}

int kata_prefill_auto_form(int B, int H, int T, int d, int chunk, int dtype, int with_state) {
    if (check_prefill(dtype, B, H, T, d, chunk)) return -1;
    return auto_quadratic(dtype, B, H, T, d, with_state != 0) ? KATA_FORM_QUADRATIC
                                                              : KATA_FORM_CHUNKED;
}

// o by the quadratic form; with H_out, the final state by the chunked form's
// state kernel (no snapshots) on the side stream at the same time.
static int prefill_quadratic(const void *q, const void *k, const void *v, int dtype, int B,
                             int H, int T, int d, int chunk, float eps, float *o, float *H_out,
                             float *s_out, cudaStream_t s) {
    unsigned int *err = error_word();
    if (!err) return fail(KATA_ERR_CUDA, "error word unavailable");
    kata::PrefillArgs a{q, k, v, dtype, B, H, T, d, chunk, eps, nullptr, nullptr, o,
                        nullptr, nullptr, nullptr, 0, err};
    if (!H_out) {
        cudaError_t e = kata::quad_tc(a, s);
        if (e != cudaSuccess) return cuda_fail(e, "kata_prefill (quadratic form) launch");
        return KATA_OK;
    }
    kata::PrefillArgs st{q, k, v, dtype, B, H, T, d, chunk, eps, nullptr, nullptr, nullptr,
                         H_out, s_out, nullptr, 0, err};
    if (!kata::prefill_tc_supported(st))
        return fail(KATA_ERR_UNSUPPORTED, "final state beside the quadratic form: not supported");
    SideStream *sd = side_stream();
    if (!sd) return fail(KATA_ERR_CUDA, "side stream unavailable");
    cudaError_t e;
    {
        std::lock_guard<std::mutex> lock(sd->mu);
        if ((e = cudaEventRecord(sd->fork, s)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(sd->stream, sd->fork, 0)) != cudaSuccess)
            return cuda_fail(e, "fork to the side stream");
        e = kata::prefill_tc(st, sd->stream);
        cudaError_t ej = cudaEventRecord(sd->join, sd->stream);
        if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, sd->join, 0);
        if (e != cudaSuccess) return cuda_fail(e, "kata_prefill (state kernel) launch");
        if (ej != cudaSuccess) return cuda_fail(ej, "join from the side stream");
    }
    e = kata::quad_tc(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "kata_prefill (quadratic form) launch");
    return KATA_OK;
}

int kata_prefill(const void *q, const void *k, const void *v, int dtype, int B, int H, int T,
                 int d, int chunk, float eps, const float *H_in, const float *s_in, float *o,
                 float *H_out, float *s_out, void *workspace, size_t ws_bytes, void *stream) {
    return kata_prefill_ex(q, k, v, dtype, B, H, T, d, chunk, eps, H_in, s_in, o, H_out, s_out,
                           workspace, ws_bytes, stream, KATA_FORM_AUTO);
}

int kata_prefill_ex(const void *q, const void *k, const void *v, int dtype, int B, int H, int T,
                    int d, int chunk, float eps, const float *H_in, const float *s_in, float *o,
                    float *H_out, float *s_out, void *workspace, size_t ws_bytes, void *stream,
                    int form) {
    g_last_error[0] = 0;
    int st = check_prefill(dtype, B, H, T, d, chunk);
    if (st) return st;
    if (form != KATA_FORM_AUTO && form != KATA_FORM_CHUNKED && form != KATA_FORM_QUADRATIC)
        return fail(KATA_ERR_INVALID_ARG, "form=%d: 0 (auto), 1 (chunked) or 2 (quadratic)", form);
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_OPTIONAL_PTR(o);
    KATA_OPTIONAL_PTR(H_in);
    KATA_OPTIONAL_PTR(s_in);
    KATA_OPTIONAL_PTR(H_out);
    KATA_OPTIONAL_PTR(s_out);
    if (!H_in != !s_in) return fail(KATA_ERR_INVALID_ARG, "H_in and s_in: both or neither");
    if (!H_out != !s_out) return fail(KATA_ERR_INVALID_ARG, "H_out and s_out: both or neither");
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const bool init = H_in != nullptr;
    if (form == KATA_FORM_AUTO)
        form = o && auto_quadratic(dtype, B, H, T, d, init || H_out) ? KATA_FORM_QUADRATIC
                                                                      : KATA_FORM_CHUNKED;
    if (form == KATA_FORM_QUADRATIC) {
        if (!o || !quadratic_applies(dtype, B, H, T, d, init))
            return fail(KATA_ERR_UNSUPPORTED, "quadratic form: bf16, d = 32 or 64, T a multiple "
                                              "of 128, o given, no initial state");
        return prefill_quadratic(q, k, v, dtype, B, H, T, d, chunk, eps, o, H_out, s_out,
                                 static_cast<cudaStream_t>(stream));
    }
    const size_t need = prefill_ws_bytes(B, H, T, d, chunk, dtype);
    if (ws_bytes < need || (need && !workspace))
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_OPTIONAL_PTR(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int *err = error_word();
    if (!err) return fail(KATA_ERR_CUDA, "error word unavailable");

    const size_t s_bytes = (size_t)B * H * kata::packed_dim(d) * sizeof(float);
    char *ws = static_cast<char *>(workspace);
    if (s_in && s_out == s_in) {  // every CTA of a head reads s_in: keep a copy
        cudaError_t e = cudaMemcpyAsync(ws, s_in, s_bytes, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "copy s_in");
        s_in = reinterpret_cast<const float *>(ws);
    }
    kata::PrefillArgs a{q, k, v, dtype, B, H, T, d, chunk, eps, H_in, s_in, o, H_out, s_out,
                        ws + kata::align_up(s_bytes, 256), ws_bytes - kata::align_up(s_bytes, 256),
                        err};
    cudaError_t e;
    if (dtype == KATA_BF16 && kata::prefill_tc_supported(a))
        e = kata::prefill_tc(a, s);
    else
        e = kata::prefill_simt(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "kata_prefill launch");
    return KATA_OK;
}

int kata_prefill_path(int B, int H, int T, int d, int chunk, int dtype) {
    if (check_prefill(dtype, B, H, T, d, chunk)) return -1;
    kata::PrefillArgs a{};
    a.dtype = dtype;
    a.B = B;
    a.H = H;
    a.T = T;
    a.d = d;
    a.chunk = chunk;
    return dtype == KATA_BF16 && kata::prefill_tc_supported(a) ? 1 : 0;
}

static int check_feature(int d, int feature, int g) {
    if (feature == KATA_FEATURE_RANK1) {
        if (g != 1) return fail(KATA_ERR_INVALID_ARG, "g=%d: the rank-one feature has g = 1", g);
        return KATA_OK;
    }
    if (feature != KATA_FEATURE_MG && feature != KATA_FEATURE_SIGMAG)
        return fail(KATA_ERR_UNSUPPORTED, "feature=%d: 0 (rank one), 1 (Mg) or 2 (Sigma-g)",
                    feature);
    if (g < 1 || d % g || d / g < 8)
        return fail(KATA_ERR_UNSUPPORTED, "g=%d: must divide d=%d into factors of >= 8 values",
                    g, d);
    return KATA_OK;
}

long kata_feature_dim(int d, int feature, int g) {
    if (d != 16 && d != 32 && d != 64) return 0;
    if (check_feature(d, feature, g)) return 0;
    return kata::feature_dim(d, feature, g);
}

int kata_prefill_feature(const void *q, const void *k, const void *v, int dtype, int B, int H,
                         int T, int d, int chunk, float eps, int feature, int g,
                         const float *H_in, const float *s_in, float *o, float *H_out,
                         float *s_out, void *workspace, size_t ws_bytes, void *stream) {
    g_last_error[0] = 0;
    int st = check_prefill(dtype, B, H, T, d, chunk);
    if (st) return st;
    if ((st = check_feature(d, feature, g))) return st;
    if (feature == KATA_FEATURE_RANK1)
        return kata_prefill_ex(q, k, v, dtype, B, H, T, d, chunk, eps, H_in, s_in, o, H_out,
                               s_out, workspace, ws_bytes, stream, KATA_FORM_AUTO);
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_OPTIONAL_PTR(o);
    KATA_OPTIONAL_PTR(H_in);
    KATA_OPTIONAL_PTR(s_in);
    KATA_OPTIONAL_PTR(H_out);
    KATA_OPTIONAL_PTR(s_out);
    if (!H_in != !s_in) return fail(KATA_ERR_INVALID_ARG, "H_in and s_in: both or neither");
    if (!H_out != !s_out) return fail(KATA_ERR_INVALID_ARG, "H_out and s_out: both or neither");
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const size_t s_bytes = (size_t)B * H * kata::feature_dim(d, feature, g) * sizeof(float);
    const bool alias = s_in && s_out == s_in;
    if (alias && (!workspace || ws_bytes < s_bytes))
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, s_bytes);
    KATA_OPTIONAL_PTR(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int *err = error_word();
    if (!err) return fail(KATA_ERR_CUDA, "error word unavailable");
    if (alias) {  // every CTA of a head reads s_in: keep a copy
        cudaError_t e = cudaMemcpyAsync(workspace, s_in, s_bytes, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "copy s_in");
        s_in = static_cast<const float *>(workspace);
    }
    kata::PrefillArgs a{q, k, v, dtype, B, H, T, d, chunk, eps, H_in, s_in, o, H_out, s_out,
                        nullptr, 0, err};
    a.feature = feature;
    a.g = g;
    cudaError_t e = kata::prefill_simt(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "kata_prefill_feature launch");
    return KATA_OK;
}

int kata_state_prefix(const float *H_parts, const float *s_parts, int nparts, int B, int H,
                      int d, int feature, int g, float *H_prefix, float *s_prefix,
                      void *stream) {
    g_last_error[0] = 0;
    int st = check_common(KATA_F32, B, H, d);
    if (st) return st;
    if ((st = check_feature(d, feature, g))) return st;
    if (nparts < 1 || nparts > 65536)
        return fail(KATA_ERR_INVALID_ARG, "nparts=%d must be in [1, 65536]", nparts);
    KATA_REQUIRE_PTR(H_parts);
    KATA_REQUIRE_PTR(s_parts);
    KATA_REQUIRE_PTR(H_prefix);
    KATA_REQUIRE_PTR(s_prefix);
    if (H_prefix == H_parts || s_prefix == s_parts)
        return fail(KATA_ERR_INVALID_ARG, "the prefixes must not overwrite the parts");
    const size_t Df = (size_t)kata::feature_dim(d, feature, g);
    const size_t nH = (size_t)B * H * Df * d, ns = (size_t)B * H * Df;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = kata::exclusive_prefix(H_parts, nparts, nH, H_prefix, s);
    if (e == cudaSuccess) e = kata::exclusive_prefix(s_parts, nparts, ns, s_prefix, s);
    if (e != cudaSuccess) return cuda_fail(e, "kata_state_prefix launch");
    return KATA_OK;
}

int kata_test_forced_timeout(const void *q, const void *k, const void *v, int B, int H, int T,
                             int d, float eps, float *o, unsigned int polls, void *stream) {
    g_last_error[0] = 0;
    int st = check_prefill(KATA_BF16, B, H, T, d, 128);
    if (st) return st;
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_REQUIRE_PTR(o);
    if (!quadratic_applies(KATA_BF16, B, H, T, d, false))
        return fail(KATA_ERR_UNSUPPORTED, "the forced timeout runs the quadratic form: d = 32 or "
                                          "64, T a multiple of 128");
    if (polls < 1 || polls > (1u << 20))
        return fail(KATA_ERR_INVALID_ARG, "polls=%u must be in [1, 2^20]", polls);
    unsigned int *err = error_word();
    if (!err) return fail(KATA_ERR_CUDA, "error word unavailable");
    kata::PrefillArgs a{q, k, v, KATA_BF16, B, H, T, d, 128, eps, nullptr, nullptr, o,
                        nullptr, nullptr, nullptr, 0, err};
    cudaError_t e = kata::quad_tc(a, static_cast<cudaStream_t>(stream), polls);
    if (e != cudaSuccess) return cuda_fail(e, "kata_test_forced_timeout launch");
    return KATA_OK;
}

#ifdef KATA_DEBUG
namespace {
__device__ int g_bounds_probe[4];
// One checked store past the end of a 4-element array: the check records
// 0xB001 and the store is skipped.
__global__ void bounds_probe_kernel(int idx) {
    if (threadIdx.x == 0 && KATA_CHECK(idx >= 0 && idx < 4, 0xB001u)) g_bounds_probe[idx] = 1;
}
}  // namespace
#endif

int kata_debug_build(void) {
#ifdef KATA_DEBUG
    return 1;
#else
    return 0;
#endif
}

int kata_test_bounds_check(void *stream) {
    g_last_error[0] = 0;
#ifdef KATA_DEBUG
    KATA_DEBUG_BIND();
    bounds_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(7);
    const cudaError_t e = kata::after_launch();
    if (e != cudaSuccess) return cuda_fail(e, "kata_test_bounds_check launch");
    return KATA_OK;
#else
    (void)stream;
    return fail(KATA_ERR_UNSUPPORTED, "bounds checks are compiled into libkata_debug.so only");
#endif
}

// A host-buffer prefill runs in pieces of consecutive heads (every head is
// independent): piece i's copies in, kernels and copy out go to the caller's
// stream or the side stream by turns, so the host-to-device copies of one
// piece overlap the kernels and the device-to-host copy of another.
// Two pieces measured best at B4 H8 T2048 d32 (394 us per call against 424 us
// in one piece, 414 us in four, 473 us in eight): the host link, not the
// kernels, sets the pace, and each piece adds four copies and a launch.
static int host_pieces(long heads) { return heads >= 2 ? 2 : 1; }
static void host_piece(long heads, int np, int i, long &h0, long &h1) {
    h0 = heads * i / np;
    h1 = heads * (i + 1) / np;
}
// kata_prefill workspace of every piece, each 256-byte aligned
static size_t host_pieces_ws_bytes(int B, int H, int T, int d, int chunk, int dtype) {
    const long heads = (long)B * H;
    const int np = host_pieces(heads);
    size_t b = 0;
    for (int i = 0; i < np; ++i) {
        long h0, h1;
        host_piece(heads, np, i, h0, h1);
        b += kata::align_up(prefill_ws_bytes(1, (int)(h1 - h0), T, d, chunk, dtype), 256);
    }
    return b;
}

size_t kata_prefill_host_workspace_bytes(int B, int H, int T, int d, int chunk, int dtype) {
    if (check_prefill(dtype, B, H, T, d, chunk)) return 0;
    const size_t n = (size_t)B * H * T * d;
    return 3 * kata::align_up(n * elem_bytes(dtype), 256) + kata::align_up(n * 4, 256) +
           host_pieces_ws_bytes(B, H, T, d, chunk, dtype);
}

int kata_prefill_host(const void *q_host, const void *k_host, const void *v_host, int dtype,
                      int B, int H, int T, int d, int chunk, float eps, float *o_host,
                      void *workspace, size_t ws_bytes, void *stream) {
    g_last_error[0] = 0;
    int st = check_prefill(dtype, B, H, T, d, chunk);
    if (st) return st;
    if (!q_host || !k_host || !v_host || !o_host)
        return fail(KATA_ERR_INVALID_ARG, "host pointers must not be NULL");
    const size_t need = kata_prefill_host_workspace_bytes(B, H, T, d, chunk, dtype);
    if (!workspace || ws_bytes < need)
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_REQUIRE_PTR(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = (size_t)B * H * T * d, xb = n * elem_bytes(dtype);
    char *w = static_cast<char *>(workspace);
    char *qd = w, *kd = qd + kata::align_up(xb, 256), *vd = kd + kata::align_up(xb, 256);
    float *od = reinterpret_cast<float *>(vd + kata::align_up(xb, 256));
    char *rest = reinterpret_cast<char *>(od) + kata::align_up(n * 4, 256);
    SideStream *sd = side_stream(1);
    if (!sd) return fail(KATA_ERR_CUDA, "side stream unavailable");
    const long heads = (long)B * H;
    const int np = host_pieces(heads);
    const size_t hx = (size_t)T * d * elem_bytes(dtype), ho = (size_t)T * d * 4;  // bytes per head
    std::lock_guard<std::mutex> lock(sd->mu);
    cudaError_t e;
    if ((e = cudaEventRecord(sd->fork, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(sd->stream, sd->fork, 0)) != cudaSuccess)
        return cuda_fail(e, "fork to the side stream");
    const char *qh = static_cast<const char *>(q_host), *kh = static_cast<const char *>(k_host),
               *vh = static_cast<const char *>(v_host);
    char *oh = reinterpret_cast<char *>(o_host), *od8 = reinterpret_cast<char *>(od);
    st = KATA_OK;
    for (int i = 0; i < np && st == KATA_OK; ++i) {
        long h0, h1;
        host_piece(heads, np, i, h0, h1);
        cudaStream_t ps = (i & 1) ? sd->stream : s;
        const size_t x0 = (size_t)h0 * hx, nx = (size_t)(h1 - h0) * hx;
        const size_t wsi = kata::align_up(prefill_ws_bytes(1, (int)(h1 - h0), T, d, chunk, dtype), 256);
        if ((e = cudaMemcpyAsync(qd + x0, qh + x0, nx, cudaMemcpyHostToDevice, ps)) != cudaSuccess ||
            (e = cudaMemcpyAsync(kd + x0, kh + x0, nx, cudaMemcpyHostToDevice, ps)) != cudaSuccess ||
            (e = cudaMemcpyAsync(vd + x0, vh + x0, nx, cudaMemcpyHostToDevice, ps)) != cudaSuccess) {
            st = cuda_fail(e, "host-to-device copy");
            break;
        }
        st = kata_prefill(qd + x0, kd + x0, vd + x0, dtype, 1, (int)(h1 - h0), T, d, chunk, eps,
                          nullptr, nullptr, reinterpret_cast<float *>(od8 + (size_t)h0 * ho),
                          nullptr, nullptr, rest, wsi, ps);
        if (st) break;
        rest += wsi;
        if ((e = cudaMemcpyAsync(oh + (size_t)h0 * ho, od8 + (size_t)h0 * ho,
                                 (size_t)(h1 - h0) * ho, cudaMemcpyDeviceToHost, ps)) != cudaSuccess)
            st = cuda_fail(e, "device-to-host copy");
    }
    // the caller's stream waits for the side stream's pieces, also after an error
    cudaError_t ej = cudaEventRecord(sd->join, sd->stream);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, sd->join, 0);
    if (st) return st;
    if (ej != cudaSuccess) return cuda_fail(ej, "join from the side stream");
    return KATA_OK;
}

/* -------------------------------------------------------------- decode --- */

int kata_decode_step(const void *q, const void *k, const void *v, int dtype, int B, int H,
                     int d, float eps, float *Hst, float *s, float *o, void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_REQUIRE_PTR(o);
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    cudaError_t e = kata::decode_step(q, k, v, dtype, B, H, d, eps, Hst, s, o,
                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kata_decode_step launch");
    return KATA_OK;
}

int kata_decode_step_feature(const void *q, const void *k, const void *v, int dtype, int B,
                             int H, int d, float eps, int feature, int g, float *Hst, float *s,
                             float *o, void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if ((st = check_feature(d, feature, g))) return st;
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_REQUIRE_PTR(o);
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    cudaError_t e = kata::decode_step(q, k, v, dtype, B, H, d, eps, Hst, s, o,
                                      static_cast<cudaStream_t>(stream), feature, g);
    if (e != cudaSuccess) return cuda_fail(e, "kata_decode_step_feature launch");
    return KATA_OK;
}

int kata_decode_step_host(const void *q_host, const void *k_host, const void *v_host,
                          int dtype, int B, int H, int d, float eps, float *Hst, float *s,
                          float *o_host, void *workspace, size_t ws_bytes, void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if (!q_host || !k_host || !v_host || !o_host)
        return fail(KATA_ERR_INVALID_ARG, "host pointers must not be NULL");
    const size_t n = (size_t)B * H * d, xb = n * elem_bytes(dtype);
    const size_t need = 3 * kata::align_up(xb, 256) + kata::align_up(n * 4, 256);
    if (!workspace || ws_bytes < need)
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_REQUIRE_PTR(workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char *qd = static_cast<char *>(workspace), *kd = qd + kata::align_up(xb, 256);
    char *vd = kd + kata::align_up(xb, 256);
    float *od = reinterpret_cast<float *>(vd + kata::align_up(xb, 256));
    cudaError_t e;
    if ((e = cudaMemcpyAsync(qd, q_host, xb, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(kd, k_host, xb, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(vd, v_host, xb, cudaMemcpyHostToDevice, cs)) != cudaSuccess)
        return cuda_fail(e, "host-to-device copy");
    st = kata_decode_step(qd, kd, vd, dtype, B, H, d, eps, Hst, s, od, stream);
    if (st) return st;
    if ((e = cudaMemcpyAsync(o_host, od, n * 4, cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
        return cuda_fail(e, "device-to-host copy");
    return KATA_OK;
}

/* ---------------------------------------------------------------- LoLA --- */

size_t lola_sre_workspace_bytes(int B, int H, int d, int n_cand) {
    if (check_common(KATA_F32, B, H, d) || n_cand < 1 || n_cand > 1024) return 0;
    return kata::sre_workspace_bytes(B, H, d, n_cand);
}

int lola_sre_score_topk(const float *Hst, const float *s, const void *kc, const void *vc,
                        const int *pos, int dtype, int B, int H, int d, int n_cand, int keep,
                        float eps, int merge, float *scores, int *keep_idx, float *Hst_mut,
                        float *s_mut, void *workspace, size_t ws_bytes, void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if (n_cand < 1 || n_cand > 1024)
        return fail(KATA_ERR_INVALID_ARG, "n_cand=%d must be in [1, 1024]", n_cand);
    if (keep < 0) return fail(KATA_ERR_INVALID_ARG, "keep=%d must be >= 0", keep);
    if (merge != 0 && merge != 1) return fail(KATA_ERR_INVALID_ARG, "merge must be 0 or 1");
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_REQUIRE_PTR(kc);
    KATA_REQUIRE_PTR(vc);
    KATA_REQUIRE_PTR(pos);
    KATA_OPTIONAL_PTR(scores);
    if (keep > 0) KATA_REQUIRE_PTR(keep_idx);
    if (merge) {
        KATA_REQUIRE_PTR(Hst_mut);
        KATA_REQUIRE_PTR(s_mut);
    }
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const size_t need = kata::sre_workspace_bytes(B, H, d, n_cand);
    if (!workspace || ws_bytes < need)
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_REQUIRE_PTR(workspace);
    cudaError_t e = kata::sre_score_topk(Hst, s, kc, vc, pos, dtype, B, H, d, n_cand, n_cand,
                                         keep, eps, merge, scores, keep_idx, Hst_mut, s_mut,
                                         workspace, ws_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "lola_sre_score_topk launch");
    return KATA_OK;
}

int lola_sre_score_topk_noalloc(const float *Hst, const float *s, const void *kc,
                                const void *vc, const int *pos, int dtype, int B, int H, int d,
                                int n_cand, int keep, float eps, int merge, float *scores,
                                int *keep_idx, float *Hst_mut, float *s_mut, void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if (n_cand < 1 || n_cand > 1024)
        return fail(KATA_ERR_INVALID_ARG, "n_cand=%d must be in [1, 1024]", n_cand);
    if (keep < 0) return fail(KATA_ERR_INVALID_ARG, "keep=%d must be >= 0", keep);
    if (merge != 0 && merge != 1) return fail(KATA_ERR_INVALID_ARG, "merge must be 0 or 1");
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_REQUIRE_PTR(kc);
    KATA_REQUIRE_PTR(vc);
    KATA_REQUIRE_PTR(pos);
    KATA_OPTIONAL_PTR(scores);
    if (keep > 0) KATA_REQUIRE_PTR(keep_idx);
    if (merge) {
        KATA_REQUIRE_PTR(Hst_mut);
        KATA_REQUIRE_PTR(s_mut);
    }
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const size_t need = kata::sre_workspace_bytes(B, H, d, n_cand);
    const size_t cap = kata::sre_noalloc_capacity();
    if (need > cap)
        return fail(KATA_ERR_WORKSPACE,
                    "B=%d H=%d d=%d n_cand=%d needs %zu bytes of scratch but the fixed scratch "
                    "holds %zu; call lola_sre_score_topk with a workspace instead",
                    B, H, d, n_cand, need, cap);
    cudaError_t e = kata::sre_score_topk_noalloc(Hst, s, kc, vc, pos, dtype, B, H, d, n_cand,
                                                 keep, eps, merge, scores, keep_idx, Hst_mut,
                                                 s_mut, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "lola_sre_score_topk_noalloc");
    return KATA_OK;
}

size_t lola_readout_workspace_bytes(int B, int H, int d, int nq) {
    if (check_common(KATA_F32, B, H, d) || nq < 1 || nq > 256) return 0;
    return kata::readout_workspace_bytes(B, H, d, nq);
}

int lola_hybrid_readout(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int T, int d, int seg0, int nq, int w0, const void *ck,
                        const void *cv, int nc, int cap, const float *Hst, const float *s,
                        float eps, float tau, float *o, void *workspace, size_t ws_bytes,
                        void *stream) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    if (T <= 0 || nq < 1 || nq > 256 || seg0 < 0 || seg0 + nq > T || w0 < 0 || w0 > seg0 ||
        seg0 + nq - w0 > 1024)
        return fail(KATA_ERR_INVALID_ARG, "bad segment T=%d seg0=%d nq=%d w0=%d", T, seg0, nq, w0);
    if (nc < 0 || cap < nc || cap > 4096)
        return fail(KATA_ERR_INVALID_ARG, "bad cache nc=%d cap=%d", nc, cap);
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_REQUIRE_PTR(o);
    if (nc > 0) {
        KATA_REQUIRE_PTR(ck);
        KATA_REQUIRE_PTR(cv);
    }
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const size_t need = kata::readout_workspace_bytes(B, H, d, nq);
    if (!workspace || ws_bytes < need)
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_REQUIRE_PTR(workspace);
    cudaError_t e = kata::hybrid_readout(q, k, v, dtype, B, H, T, d, seg0, nq, w0, ck, cv, nc,
                                         cap, Hst, s, eps, tau, o, workspace, ws_bytes,
                                         static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "lola_hybrid_readout launch");
    return KATA_OK;
}

size_t lola_prefill_workspace_bytes(int B, int H, int T, int d, int window, int cache) {
    if (check_common(KATA_F32, B, H, d) || window < 1 || window > 256 || cache < 0 ||
        window + cache > 1024)
        return 0;
    const size_t seg = kata::lola_workspace_bytes(B, H, T, d, window, cache);
    const size_t fused = kata::lola_fused_scratch_bytes(B * H, d);
    return seg > fused ? seg : fused;
}

int lola_prefill_fused_applies(int dtype, int d, int window, int cache) {
    return kata::lola_fused_applies(dtype, d, window, cache) ? 1 : 0;
}

int lola_prefill(const void *q, const void *k, const void *v, int dtype, int B, int H, int T,
                 int d, int window, int cache, float eps, float tau, float *o, float *Hst,
                 float *s, int *kept_pos, void *workspace, size_t ws_bytes, void *stream) {
    return lola_prefill_ex(q, k, v, dtype, B, H, T, d, window, cache, eps, tau, o, Hst, s,
                           kept_pos, workspace, ws_bytes, stream, LOLA_RUN_AUTO);
}

int lola_prefill_ex(const void *q, const void *k, const void *v, int dtype, int B, int H,
                    int T, int d, int window, int cache, float eps, float tau, float *o,
                    float *Hst, float *s, int *kept_pos, void *workspace, size_t ws_bytes,
                    void *stream, int run) {
    g_last_error[0] = 0;
    int st = check_common(dtype, B, H, d);
    if (st) return st;
    int ncl = 0;  // CTAs per head of the fused run (0: chosen by occupancy)
    if (run >= LOLA_RUN_FUSED_NCL(6) && run <= LOLA_RUN_FUSED_NCL(8)) {
        ncl = run - LOLA_RUN_FUSED_NCL(0);
        run = LOLA_RUN_FUSED;
    }
    if (run != LOLA_RUN_AUTO && run != LOLA_RUN_SEGMENTS && run != LOLA_RUN_FUSED)
        return fail(KATA_ERR_INVALID_ARG,
                    "run=%d: 0 (auto), 1 (segments), 2 (fused) or LOLA_RUN_FUSED_NCL(6..8)", run);
    if (window < 1 || window > 256 || cache < 0 || window + cache > 1024)
        return fail(KATA_ERR_INVALID_ARG, "window=%d cache=%d out of range", window, cache);
    if (T <= 0 || T % window)
        return fail(KATA_ERR_INVALID_ARG, "T=%d must be a positive multiple of window=%d", T, window);
    KATA_REQUIRE_PTR(q);
    KATA_REQUIRE_PTR(k);
    KATA_REQUIRE_PTR(v);
    KATA_REQUIRE_PTR(o);
    KATA_REQUIRE_PTR(Hst);
    KATA_REQUIRE_PTR(s);
    KATA_OPTIONAL_PTR(kept_pos);
    if (!(eps >= 0.f)) return fail(KATA_ERR_INVALID_ARG, "eps must be >= 0");
    const bool fused_ok = kata::lola_fused_applies(dtype, d, window, cache);
    if (run == LOLA_RUN_FUSED && !fused_ok)
        return fail(KATA_ERR_UNSUPPORTED, "fused LoLA schedule: window a multiple of 8 up to 64, "
                                          "2*window + cache <= 256, d*elem_size <= 128");
    const bool fused = run == LOLA_RUN_FUSED || (run == LOLA_RUN_AUTO && fused_ok);
    const size_t need = fused ? kata::lola_fused_scratch_bytes(B * H, d)
                              : kata::lola_workspace_bytes(B, H, T, d, window, cache);
    if (!workspace || ws_bytes < need)
        return fail(KATA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    KATA_REQUIRE_PTR(workspace);
    cudaError_t e =
        fused ? kata::lola_fused(q, k, v, dtype, B * H, T, d, window, cache, eps, tau, o, Hst, s,
                                 kept_pos, workspace, ncl, static_cast<cudaStream_t>(stream))
              : kata::lola_run(q, k, v, dtype, B, H, T, d, window, cache, eps, tau, o, Hst, s,
                               kept_pos, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "lola_prefill launch");
    return KATA_OK;
}

}  // extern "C"
