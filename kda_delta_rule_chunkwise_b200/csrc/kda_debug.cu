// Debug input scan (KDA_DEBUG_CHECKS=1): reports log-decays outside the
// contract before a prefill or decode step reads them.
//
// The contract is g in [-5, 0]: the lower bound is the one neurohive.io "Kimi
// K3 ... overview", section "Sequence length: hybrid KDA and Gated MLA
// attention", puts on the log-decay so that every rescaling factor of the
// chunked form stays in range; a positive log-decay would make the state
// grow.  The kernels clamp g below at -5 and use g > 0 as given, so neither
// is an error for them; this scan only tells the caller that its inputs left
// the contract (or hold a NaN).  It sets ERR_INPUT_RANGE in the device error
// word, which kda_check_device_error reports as KDA_ERR_INPUT_RANGE; it never
// traps and changes no output.
#include <cuda_bf16.h>
#include <cstdlib>

#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

namespace {

__device__ __forceinline__ bool out_of_range(float x) { return !(x >= -5.f && x <= 0.f); }

// Rows [r0, r1) of g [rows, H*dk]; for packed sequences r0 = clamp(cu[0]) and
// r1 = clamp(cu[N]) are read here (rows outside every sequence are not inputs).
template <typename Tin>
__global__ void __launch_bounds__(256)
input_scan_kernel(const Tin *__restrict__ g, int64_t rows, int64_t row_elems,
                  const int32_t *__restrict__ cu, int N, uint32_t *err) {
    int64_t r0 = 0, r1 = rows;
    if (cu) {
        auto clampT = [&](int64_t x) { return x < 0 ? (int64_t)0 : (x > rows ? rows : x); };
        r0 = clampT(cu[0]);
        r1 = clampT(cu[N]);
        if (r1 < r0) r1 = r0;
    }
    const int64_t e0 = r0 * row_elems, e1 = r1 * row_elems;
    bool bad = false;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = e0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < e1; i += stride)
        bad |= out_of_range(to_f32(g[i]));
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, ERR_INPUT_RANGE);
}

}  // namespace

cudaError_t launch_input_scan(const void *g, int64_t rows, int H, int dk, bool bf16,
                              const int32_t *cu, int N, uint32_t *err, cudaStream_t st) {
    if (rows <= 0 || !g || !err) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t elems = rows * H * dk;
    int64_t blocks = (elems + 255) / 256;
    if (blocks > 8LL * sms) blocks = 8LL * sms;
    if (bf16)
        input_scan_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)g, rows, (int64_t)H * dk, cu, N, err);
    else
        input_scan_kernel<float><<<(unsigned)blocks, 256, 0, st>>>((const float *)g, rows,
                                                                   (int64_t)H * dk, cu, N, err);
    return cudaGetLastError();
}

bool debug_checks_enabled() {
    const char *e = getenv("KDA_DEBUG_CHECKS");
    return e && e[0] == '1';
}

}  // namespace kda
