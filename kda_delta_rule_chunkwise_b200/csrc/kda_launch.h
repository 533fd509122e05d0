// Internal launch interface between the C ABI (kda_abi.cu) and the kernel
// translation units.  Not part of the public header.
#pragma once

#include <cuda_runtime.h>

#include "kda.h"
#include <stddef.h>
#include <stdint.h>

namespace kda {

struct PrefillArgs {
    const void *q, *k, *v, *g, *beta;
    const float *state_in;
    const int32_t *cu_seqlens;   // device, N+1 entries, or nullptr
    int B;
    int64_t T;                   // rows per batch entry (packed rows when cu_seqlens)
    int N, H, dk, dv;
    void *o;
    float *state_out;
    void *workspace;
    size_t workspace_bytes;
    uint32_t *err;               // device error word
    // intermediate states: every ckpt_interval tokens (a multiple of the chunk
    // length; 0 = none) inside each sequence, into ckpt [ckpt_capacity, H, dk, dv]
    int64_t ckpt_interval = 0;
    float *ckpt = nullptr;
    int64_t ckpt_capacity = 0;
    uint32_t flags = 0;          // KDA_PREP_* input preprocessing (kda.h)
    uint32_t epoch = 0;          // this launch's nonzero epoch (see kda_common.cuh)
};

// A fresh nonzero epoch for one launch of kernels that use bounded waits.
uint32_t next_launch_epoch();

// Optional per-kernel event recording (see kda_profile_enable).  Launchers
// call mark() before their first kernel and after each kernel.
struct Profiler {
    static void begin(cudaStream_t st);   // start a new record
    static void mark(cudaStream_t st);    // event after a kernel
};

cudaError_t launch_prefill_simt(const PrefillArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st);
size_t prefill_tc_workspace_bytes(int64_t rows, int N, int H, int d);
// slots == nullptr: request n owns state entry n; otherwise entry slots[n] of P.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *g,
                          const void *beta, float *state, int N, int H, int d, bool bf16,
                          void *o, const int32_t *slots, int P, uint32_t *err, cudaStream_t st);
// Debug input scan (kda_debug.cu): sets ERR_INPUT_RANGE when a log-decay of
// rows [cu[0], cu[N]) (all rows when cu is null) lies outside [-5, 0] or is NaN.
cudaError_t launch_input_scan(const void *g, int64_t rows, int H, int dk, bool bf16,
                              const int32_t *cu, int N, uint32_t *err, cudaStream_t st);
// True when the environment variable KDA_DEBUG_CHECKS is set to 1 (read per call).
bool debug_checks_enabled();
cudaError_t launch_selftest_wait(uint64_t timeout_us, uint32_t *err, cudaStream_t st);

// Backward (kda_backward.cu).  Gradients are fp32; inputs fp32 or bf16.
struct BackwardArgs {
    const void *q, *k, *v, *g, *beta;
    const float *state_in;
    const int32_t *cu_seqlens;
    int64_t rows, T;
    int N, H, d;
    const float *dout, *dstate_out;
    float *dq, *dk, *dv, *dg, *dbeta, *dstate_in;
    void *workspace;
    uint32_t *err = nullptr;     // device error word (the chunked path's forward waits)
    uint32_t epoch = 0;
};
size_t backward_workspace_bytes(int64_t rows, int N, int H, int d);
cudaError_t launch_backward(const BackwardArgs &a, bool bf16, cudaStream_t st);
// Backward through the chunked form (kda_backward_chunked.cu): bf16 inputs, d = 128.
size_t backward_chunked_workspace_bytes(int64_t rows, int N, int H);
cudaError_t launch_backward_chunked(const BackwardArgs &a, cudaStream_t st);

}  // namespace kda
