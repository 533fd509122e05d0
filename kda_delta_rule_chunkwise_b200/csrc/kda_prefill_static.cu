// Allocation-free prefill entry point (kda_chunk_prefill_static_scratch).
//
// For callers that cannot allocate device memory, the bf16 path's scratch is
// a file-scope device array owned by the library.  Host code must not pass
// the array's name to a kernel: in host code that name is a host-side
// stand-in, not a device address.  Its device address is looked up once per
// device with cudaGetSymbolAddress (no allocation) and cached.
#include <mutex>

#include "kda.h"
#include "kda_launch.h"

namespace {

__device__ __align__(256) uint8_t g_kda_static_scratch[KDA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_dev_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device; the first call
// on a device does the lookup.  Returns nullptr on failure.
void *static_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_dev_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_static_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_dev_ptr[dev] = p;
    }
    return g_scratch_dev_ptr[dev];
}

}  // namespace

extern "C" kda_status kda_chunk_prefill_static_scratch(
    const void *q, const void *k, const void *v, const void *g, const void *beta,
    const float *state_in, const int32_t *cu_seqlens, int B, int64_t T, int N, int H, int dk,
    int dv, kda_dtype dtype, void *o, float *state_out, void *stream) {
    if (B < 0 || T < 0 || N < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    const size_t need = kda_chunk_prefill_workspace_bytes((int64_t)B * T, N, H, dk, dv, dtype);
    if (need > KDA_STATIC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        ws = static_scratch_ptr();
        if (!ws) return KDA_ERR_CUDA;
    }
    return kda_chunk_prefill(q, k, v, g, beta, state_in, cu_seqlens, B, T, N, H, dk, dv, dtype, o,
                             state_out, ws, need > 0 ? KDA_STATIC_SCRATCH_BYTES : 0, stream);
}
