// C ABI of libkda (declared in include/kda.h): argument validation, the
// device error word, and dispatch to the kernels.  All argument errors are
// reported before anything is launched.
#include "kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"

#include <atomic>
#include <mutex>

namespace {

// One error area per device context, in this library's own device memory:
// word 0 = error bits, word 1 = epoch of the latest launch that timed out
// (kda_common.cuh).  Kernels receive its device address as an argument.
__device__ uint32_t g_kda_error_word[2];

std::atomic<uint32_t> g_epoch{0};

constexpr int kMaxDevices = 64;
uint32_t *g_err_ptr[kMaxDevices];
std::mutex g_err_mu;

uint32_t *error_word_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<uint32_t *>(p);
    }
    return g_err_ptr[dev];
}

bool supported_dim(int dk, int dv) { return dk == dv && (dk == 64 || dk == 128); }

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// ---- kernel timing (kda_profile_enable / kda_profile_last)
constexpr int kMaxMarks = 16;
struct ProfState {
    bool enabled = false;
    int device = -1;
    cudaEvent_t ev[kMaxMarks] = {};
    int n = 0;   // events recorded in the current record
};
ProfState g_prof;
std::mutex g_prof_mu;

}  // namespace

namespace kda {

uint32_t next_launch_epoch() {
    uint32_t e;
    do {
        e = g_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    } while (e == 0);   // 0 is the word's initial value: never an epoch
    return e;
}

void Profiler::begin(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.n = 0;
    if (!g_prof.enabled) return;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != g_prof.device) return;
    if (cudaEventRecord(g_prof.ev[0], st) == cudaSuccess) g_prof.n = 1;
}

void Profiler::mark(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof.enabled || g_prof.n == 0 || g_prof.n >= kMaxMarks) return;
    if (cudaEventRecord(g_prof.ev[g_prof.n], st) == cudaSuccess) ++g_prof.n;
}

__global__ void selftest_wait_kernel(uint64_t limit_ns, uint32_t *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: phase 0 never completes, the bounded
    // wait gives up after `limit_ns` and records the timeout.
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, err, limit_ns)) atomicOr(err, ERR_SELFTEST);
}

cudaError_t launch_selftest_wait(uint64_t timeout_us, uint32_t *err, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(timeout_us * 1000ull, err);
    return cudaGetLastError();
}

}  // namespace kda

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_INPUT_RANGE: return "KDA_ERR_INPUT_RANGE";
    }
    return "KDA_ERR_UNKNOWN";
}

size_t kda_chunk_prefill_workspace_bytes(int64_t rows, int N, int H, int dk, int dv,
                                         kda_dtype dtype) {
    if (rows < 0 || N < 0 || H <= 0 || !supported_dim(dk, dv)) return 0;
    if (dtype != KDA_BF16) return 0;
    return kda::prefill_tc_workspace_bytes(rows, N, H, dk);
}

}  // extern "C"

namespace {
kda_status prefill_impl(const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *state_in, const int32_t *cu_seqlens,
                        int B, int64_t T, int N, int H, int dk, int dv, kda_dtype dtype, void *o,
                        float *state_out, void *workspace, size_t workspace_bytes, void *stream,
                        int64_t ckpt_interval, float *ckpt, int64_t ckpt_capacity,
                        uint32_t flags) {
    if (B < 0 || T < 0 || N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens ? B != 1 : N != B) return KDA_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * T;
    if (rows > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)N * H > (int64_t)INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    const size_t need = kda_chunk_prefill_workspace_bytes(rows, N, H, dk, dv, dtype);
    if (need > 0 && (!workspace || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return KDA_ERR_INVALID_ARG;
    // the tensor-core path reads q, k, g and v as TMA tiles: 16-byte aligned bases,
    // row coordinates that fit in int32
    if (dtype == KDA_BF16 && dk == 128 && rows > 0) {
        for (const void *p : {q, k, g, v})
            if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return KDA_ERR_INVALID_ARG;
        if (rows > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    }
    if (N == 0) return KDA_OK;

    uint32_t *err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::PrefillArgs a{q, k, v, g, beta, state_in, cu_seqlens, B, T, N, H, dk, dv,
                       o, state_out, workspace, workspace_bytes, err,
                       ckpt_interval, ckpt, ckpt_capacity, flags, kda::next_launch_epoch()};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // debug input scan (not with gate logits in g: every logit is a valid input)
    if (kda::debug_checks_enabled() && !(flags & KDA_PREP_GATE_LOGIT)) {
        const cudaError_t e = kda::launch_input_scan(g, rows, H, dk, dtype == KDA_BF16,
                                                     cu_seqlens, N, err, st);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    kda::Profiler::begin(st);
    // the tensor-core path is for bf16 at d = 128; fp32, and bf16 at d = 64, take the
    // fp32 SIMT kernel (which reads either input type)
    if (dtype == KDA_F32 || dk != 128)
        return from_cuda(kda::launch_prefill_simt(a, dtype == KDA_BF16, st));
    return from_cuda(kda::launch_prefill_tc(a, st));
}
}  // namespace

extern "C" {

kda_status kda_chunk_prefill(const void *q, const void *k, const void *v, const void *g,
                             const void *beta, const float *state_in,
                             const int32_t *cu_seqlens, int B, int64_t T, int N, int H,
                             int dk, int dv, kda_dtype dtype, void *o, float *state_out,
                             void *workspace, size_t workspace_bytes, void *stream) {
    return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, B, T, N, H, dk, dv, dtype, o,
                        state_out, workspace, workspace_bytes, stream, 0, nullptr, 0, 0u);
}

kda_status kda_chunk_prefill_ex(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, const float *state_in,
                                const int32_t *cu_seqlens, int B, int64_t T, int N, int H,
                                int dk, int dv, kda_dtype dtype, uint32_t flags, void *o,
                                float *state_out, int64_t ckpt_interval, float *ckpt,
                                int64_t ckpt_capacity, void *workspace, size_t workspace_bytes,
                                void *stream) {
    if ((flags & ~(uint32_t)(KDA_PREP_GATE_LOGIT | KDA_PREP_L2NORM_QK)) != 0)
        return KDA_ERR_INVALID_ARG;
    if (ckpt_interval < 0 || ckpt_capacity < 0 || (ckpt_capacity > 0 && !ckpt))
        return KDA_ERR_INVALID_ARG;
    if ((flags != 0 || ckpt_interval > 0) && (dtype != KDA_BF16 || dk != 128))
        return KDA_ERR_UNSUPPORTED;
    if (ckpt_interval > 0 && ckpt_interval % 64 != 0) return KDA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(ckpt) & 15u) != 0) return KDA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, B, T, N, H, dk, dv, dtype, o,
                        state_out, workspace, workspace_bytes, stream, ckpt_interval,
                        ckpt_interval > 0 ? ckpt : nullptr, ckpt_capacity, flags);
}

int64_t kda_prefill_checkpoint_count(const int32_t *cu_seqlens_host, int B, int64_t T, int N,
                                     int64_t interval) {
    if (B < 0 || T < 0 || N < 0 || interval <= 0) return -1;
    if (cu_seqlens_host ? B != 1 : N != B) return -1;
    if (!cu_seqlens_host) return T > 0 ? (int64_t)N * ((T - 1) / interval) : 0;
    // the same clamping as the device: offsets into [0, T], made non-decreasing
    int64_t total = 0, prev = 0;
    for (int i = 0; i <= N; ++i) {
        int64_t x = cu_seqlens_host[i];
        x = x < 0 ? 0 : (x > T ? T : x);
        if (x < prev) x = prev;
        if (i > 0 && x > prev) total += (x - prev - 1) / interval;
        prev = x;
    }
    return total;
}

kda_status kda_chunk_prefill_checkpointed(const void *q, const void *k, const void *v,
                                          const void *g, const void *beta,
                                          const float *state_in, const int32_t *cu_seqlens,
                                          int B, int64_t T, int N, int H, int dk, int dv,
                                          kda_dtype dtype, void *o, float *state_out,
                                          int64_t interval, float *ckpt, int64_t ckpt_capacity,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream) {
    if (interval <= 0 || ckpt_capacity < 0 || (ckpt_capacity > 0 && !ckpt))
        return KDA_ERR_INVALID_ARG;
    if (interval % 64 != 0 || dtype != KDA_BF16 || dk != 128) return KDA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(ckpt) & 15u) != 0) return KDA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, g, beta, state_in, cu_seqlens, B, T, N, H, dk, dv, dtype, o,
                        state_out, workspace, workspace_bytes, stream, interval, ckpt,
                        ckpt_capacity, 0u);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *g,
                           const void *beta, float *state, int N, int H, int dk, int dv,
                           kda_dtype dtype, void *o, void *stream) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!q || !k || !v || !g || !beta || !state || !o)) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)N * H > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if ((reinterpret_cast<uintptr_t>(state) & 15u) != 0) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kda::debug_checks_enabled()) {
        uint32_t *err = error_word_ptr();
        if (!err) return KDA_ERR_CUDA;
        if (kda::launch_input_scan(g, N, H, dk, dtype == KDA_BF16, nullptr, N, err, st) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    kda::Profiler::begin(st);
    return from_cuda(kda::launch_decode(q, k, v, g, beta, state, N, H, dk, dtype == KDA_BF16, o,
                                        nullptr, N, nullptr, st));
}

kda_status kda_decode_step_indexed(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, float *state_pool, const int32_t *slots,
                                   int N, int P, int H, int dk, int dv, kda_dtype dtype, void *o,
                                   void *stream) {
    if (N < 0 || P < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!q || !k || !v || !g || !beta || !state_pool || !slots || !o))
        return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)N * H > (int64_t)INT32_MAX || (int64_t)P * H > (int64_t)INT32_MAX)
        return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if ((reinterpret_cast<uintptr_t>(state_pool) & 15u) != 0) return KDA_ERR_INVALID_ARG;
    uint32_t *err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kda::debug_checks_enabled() &&
        kda::launch_input_scan(g, N, H, dk, dtype == KDA_BF16, nullptr, N, err, st) != cudaSuccess)
        return KDA_ERR_CUDA;
    kda::Profiler::begin(st);
    return from_cuda(kda::launch_decode(q, k, v, g, beta, state_pool, N, H, dk,
                                        dtype == KDA_BF16, o, slots, P, err, st));
}

size_t kda_backward_workspace_bytes(int64_t rows, int N, int H, int dk, int dv) {
    if (rows < 0 || N < 0 || H <= 0 || !supported_dim(dk, dv)) return 0;
    return kda::backward_workspace_bytes(rows, N, H, dk);
}

kda_status kda_backward(const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *state_in, const int32_t *cu_seqlens,
                        int B, int64_t T, int N, int H, int dk, int dv, kda_dtype dtype,
                        const float *dout, const float *dstate_out, float *dq, float *dk_out,
                        float *dv_out, float *dg, float *dbeta, float *dstate_in,
                        void *workspace, size_t workspace_bytes, void *stream) {
    if (B < 0 || T < 0 || N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens ? B != 1 : N != B) return KDA_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * T;
    if (rows > 0 && (!q || !k || !v || !g || !beta || !dout || !dq || !dk_out || !dv_out || !dg ||
                     !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)N * H > (int64_t)INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    for (const void *p : {(const void *)state_in, (const void *)dstate_out, (const void *)dstate_in})
        if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return KDA_ERR_INVALID_ARG;
    const size_t need = kda_backward_workspace_bytes(rows, N, H, dk, dv);
    const bool chunked = dtype == KDA_BF16 && dk == 128;   // through the tensor-core forward
    if (N > 0 && (!workspace || workspace_bytes < need ||
                  (reinterpret_cast<uintptr_t>(workspace) & (chunked ? 255u : 15u)) != 0))
        return KDA_ERR_INVALID_ARG;
    if (chunked && rows > 0) {
        for (const void *p : {q, k, g, v, (const void *)dout, (const void *)dv_out})
            if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return KDA_ERR_INVALID_ARG;
        if (rows > (int64_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    }
    if (N == 0) return KDA_OK;
    uint32_t *err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::BackwardArgs a{q, k, v, g, beta, state_in, cu_seqlens, rows, T, N, H, dk, dout,
                        dstate_out, dq, dk_out, dv_out, dg, dbeta, dstate_in, workspace,
                        err, kda::next_launch_epoch()};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    kda::Profiler::begin(st);
    return from_cuda(kda::launch_backward(a, dtype == KDA_BF16, st));
}

kda_status kda_check_device_error(void *stream) {
    uint32_t *err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpyFromSymbol(&word, g_kda_error_word, sizeof(word)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word == 0) return KDA_OK;
    // One condition per call, most severe first; only the reported bits are
    // cleared, so a following call reports the next one.
    uint32_t bits;
    kda_status s;
    if (word & (kda::ERR_WAIT_TIMEOUT | kda::ERR_SELFTEST)) {
        bits = kda::ERR_WAIT_TIMEOUT | kda::ERR_SELFTEST;
        s = KDA_ERR_TIMEOUT;
    } else if (word & kda::ERR_BAD_INDEX) {
        bits = kda::ERR_BAD_INDEX;
        s = KDA_ERR_INVALID_ARG;
    } else if (word & kda::ERR_INPUT_RANGE) {
        bits = kda::ERR_INPUT_RANGE;
        s = KDA_ERR_INPUT_RANGE;
    } else {
        bits = word;
        s = KDA_ERR_TIMEOUT;
    }
    const uint32_t rest = word & ~bits;
    if (cudaMemcpyToSymbol(g_kda_error_word, &rest, sizeof(rest)) != cudaSuccess)
        return KDA_ERR_CUDA;
    return s;
}

kda_status kda_profile_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.n = 0;
    if (!enable) {
        g_prof.enabled = false;
        return KDA_OK;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (g_prof.device != dev) {
        for (int i = 0; i < kMaxMarks; ++i)
            if (g_prof.ev[i]) {
                cudaEventDestroy(g_prof.ev[i]);
                g_prof.ev[i] = nullptr;
            }
        for (int i = 0; i < kMaxMarks; ++i)
            if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return KDA_ERR_CUDA;
        g_prof.device = dev;
    }
    g_prof.enabled = true;
    return KDA_OK;
}

kda_status kda_profile_last(float *ms, int capacity, int *count) {
    if (!ms || !count || capacity < 0) return KDA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    *count = 0;
    if (g_prof.n < 2) return KDA_OK;
    if (cudaEventSynchronize(g_prof.ev[g_prof.n - 1]) != cudaSuccess) return KDA_ERR_CUDA;
    int c = 0;
    for (int i = 1; i < g_prof.n && c < capacity; ++i, ++c)
        if (cudaEventElapsedTime(&ms[c], g_prof.ev[i - 1], g_prof.ev[i]) != cudaSuccess)
            return KDA_ERR_CUDA;
    *count = c;
    return KDA_OK;
}

kda_status kda_selftest_bounded_wait(int64_t timeout_us, void *stream) {
    if (timeout_us < 1 || timeout_us > 10000000) return KDA_ERR_INVALID_ARG;
    uint32_t *err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    return from_cuda(kda::launch_selftest_wait((uint64_t)timeout_us, err,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
