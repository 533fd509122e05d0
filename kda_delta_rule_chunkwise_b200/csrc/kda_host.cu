// Prefill from host buffers: kda_chunk_prefill_host (declared in include/kda.h).
//
// The sequence axis is cut into segments; segment s's inputs go host -> device
// on one stream while segment s - 1 is computed on the caller's stream and
// segment s - 2's outputs go device -> host on a third, so the PCIe traffic in
// both directions overlaps itself and the kernels.  Segments chain through the
// state (segment s starts from segment s - 1's final state), which is exact:
// the recurrence is sequential in tokens and the prefill of a segment is the
// prefill of that part of the sequence from that state.  Inputs and outputs
// are double-buffered in the caller's device workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kda.h"
#include "kda_launch.h"

namespace {

constexpr int64_t kDefaultSegment = 4096;

struct HostLayout {
    int64_t seg;                 // tokens per segment
    size_t in_elem, in_tok;      // element size; bytes of q|k|g per (batch, token) row = H dk elem
    size_t v_tok, b_tok, o_tok;  // bytes per (batch, token): v, beta, o (fp32)
    size_t in_buf, o_buf, state, pre_ws;
    size_t off_in[2], off_o[2], off_state[2], off_pre, total;
};

bool host_layout(int B, int64_t T, int H, int dk, int dv, kda_dtype dtype, int64_t segment,
                 HostLayout &L) {
    if (B <= 0 || T <= 0 || H <= 0 || dk != dv || (dk != 64 && dk != 128)) return false;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return false;
    L.seg = segment > 0 ? segment : kDefaultSegment;
    if (L.seg % 64 != 0) return false;
    if (L.seg > T) L.seg = (T + 63) / 64 * 64;
    L.in_elem = dtype == KDA_BF16 ? 2 : 4;
    L.in_tok = (size_t)H * dk * L.in_elem;
    L.v_tok = (size_t)H * dv * L.in_elem;
    L.b_tok = (size_t)H * L.in_elem;
    L.o_tok = (size_t)H * dv * 4;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t rows = (size_t)B * L.seg;
    // q, k, g, v, beta of one segment, each 256-byte aligned
    L.in_buf = 3 * al(rows * L.in_tok) + al(rows * L.v_tok) + al(rows * L.b_tok);
    L.o_buf = al(rows * L.o_tok);
    L.state = al((size_t)B * H * dk * dv * 4);
    L.pre_ws = al(kda_chunk_prefill_workspace_bytes((int64_t)rows, B, H, dk, dv, dtype));
    size_t off = 0;
    for (int i = 0; i < 2; ++i) { L.off_in[i] = off; off += L.in_buf; }
    for (int i = 0; i < 2; ++i) { L.off_o[i] = off; off += L.o_buf; }
    for (int i = 0; i < 2; ++i) { L.off_state[i] = off; off += L.state; }
    L.off_pre = off;
    off += L.pre_ws;
    L.total = off;
    return true;
}

// `height` rows of `width` bytes at the given pitches: one pitched copy, or one
// copy per row when a pitch is above what a pitched copy accepts.
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, size_t width,
                      int height, cudaMemcpyKind kind, cudaStream_t st) {
    if (height == 1) return cudaMemcpyAsync(dst, src, width, kind, st);
    constexpr size_t kMaxPitch = 0x7fffffff;
    if (dpitch <= kMaxPitch && spitch <= kMaxPitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, kind, st);
    for (int r = 0; r < height; ++r) {
        const cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t *>(dst) + r * dpitch,
                                              static_cast<const uint8_t *>(src) + r * spitch,
                                              width, kind, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// The two side streams and nine events of the copy pipeline, created once per
// device on first use and kept until the process exits (creating and
// destroying them on every call is driver work on a path that runs at the PCIe
// limit).  One call at a time enqueues on them: the mutex is held while a call
// enqueues its copies and kernels.  Reusing an event across calls is safe:
// every wait a call enqueues refers to the record made before it.
struct CopyPipeline {
    std::mutex mu;
    bool ready = false;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[9] = {};   // start, in_ready[2], in_free[2], out_ready[2], out_free[2]
};
constexpr int kMaxDevices = 64;
CopyPipeline g_pipes[kMaxDevices];

// The current device's pipeline with its mutex locked (in `lk`), or nullptr.
CopyPipeline *pipeline_for_current_device(std::unique_lock<std::mutex> &lk) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    CopyPipeline &p = g_pipes[dev];
    lk = std::unique_lock<std::mutex>(p.mu);
    if (p.ready) return &p;
    bool ok = cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) == cudaSuccess;
    for (auto &e : p.ev)
        ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        for (auto &e : p.ev)
            if (e) cudaEventDestroy(e), e = nullptr;
        if (p.s_in) cudaStreamDestroy(p.s_in), p.s_in = nullptr;
        if (p.s_out) cudaStreamDestroy(p.s_out), p.s_out = nullptr;
        return nullptr;
    }
    p.ready = true;
    return &p;
}

}  // namespace

extern "C" {

size_t kda_prefill_host_workspace_bytes(int B, int64_t T, int H, int dk, int dv, kda_dtype dtype,
                                        int64_t segment) {
    HostLayout L;
    return host_layout(B, T, H, dk, dv, dtype, segment, L) ? L.total : 0;
}

kda_status kda_chunk_prefill_host(const void *q, const void *k, const void *v, const void *g,
                                  const void *beta, const float *state_in, int B, int64_t T,
                                  int H, int dk, int dv, kda_dtype dtype, float *o,
                                  float *state_out, int64_t segment, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (segment < 0) return KDA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128)) return KDA_ERR_UNSUPPORTED;
    HostLayout L;
    if (!host_layout(B, T, H, dk, dv, dtype, segment, L)) return KDA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return KDA_ERR_INVALID_ARG;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    std::unique_lock<std::mutex> lk;
    CopyPipeline *pipe = pipeline_for_current_device(lk);
    if (!pipe) return KDA_ERR_CUDA;
    cudaStream_t s_in = pipe->s_in, s_out = pipe->s_out;
    cudaEvent_t *ev = pipe->ev;
    kda_status st = KDA_OK;
    auto ok = [&](cudaError_t e) {
        if (e != cudaSuccess && st == KDA_OK) st = KDA_ERR_CUDA;
        return st == KDA_OK;
    };
    cudaEvent_t start = ev[0], *in_ready = ev + 1, *in_free = ev + 3, *out_ready = ev + 5,
                *out_free = ev + 7;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };

    // the side streams start after everything the caller queued before this call
    if (st == KDA_OK) {
        ok(cudaEventRecord(start, cs));
        ok(cudaStreamWaitEvent(s_in, start, 0));
        ok(cudaStreamWaitEvent(s_out, start, 0));
    }
    const size_t state_bytes = (size_t)B * H * dk * dv * 4;
    float *state[2] = {reinterpret_cast<float *>(ws + L.off_state[0]),
                       reinterpret_cast<float *>(ws + L.off_state[1])};
    if (st == KDA_OK && state_in)
        ok(cudaMemcpyAsync(state[0], state_in, state_bytes, cudaMemcpyHostToDevice, cs));

    const int64_t nseg = (T + L.seg - 1) / L.seg;
    for (int64_t s = 0; s < nseg && st == KDA_OK; ++s) {
        const int b2 = (int)(s & 1);
        const int64_t t0 = s * L.seg, len = (T - t0) < L.seg ? (T - t0) : L.seg;
        uint8_t *ib = ws + L.off_in[b2];
        const size_t rows_seg = (size_t)B * L.seg;
        uint8_t *dq = ib, *dk_ = dq + al(rows_seg * L.in_tok), *dg = dk_ + al(rows_seg * L.in_tok);
        uint8_t *dv_ = dg + al(rows_seg * L.in_tok), *db = dv_ + al(rows_seg * L.v_tok);
        float *dout = reinterpret_cast<float *>(ws + L.off_o[b2]);
        // host -> device: rows t0 .. t0 + len of every batch entry (pitched copies)
        if (s >= 2) ok(cudaStreamWaitEvent(s_in, in_free[b2], 0));
        auto h2d = [&](uint8_t *dst, const void *src, size_t tok_bytes) {
            return ok(copy_rows(dst, len * tok_bytes,
                                static_cast<const uint8_t *>(src) + t0 * tok_bytes,
                                (size_t)T * tok_bytes, len * tok_bytes, B,
                                cudaMemcpyHostToDevice, s_in));
        };
        if (!h2d(dq, q, L.in_tok) || !h2d(dk_, k, L.in_tok) || !h2d(dg, g, L.in_tok) ||
            !h2d(dv_, v, L.v_tok) || !h2d(db, beta, L.b_tok))
            break;
        ok(cudaEventRecord(in_ready[b2], s_in));
        // compute: this segment from the previous segment's state
        ok(cudaStreamWaitEvent(cs, in_ready[b2], 0));
        if (s >= 2) ok(cudaStreamWaitEvent(cs, out_free[b2], 0));
        const float *sin = (s == 0 && !state_in) ? nullptr : state[s & 1];
        float *sout = state[(s + 1) & 1];
        if (st == KDA_OK) {
            const kda_status r = kda_chunk_prefill(dq, dk_, dv_, dg, db, sin, nullptr, B, len, B, H,
                                                   dk, dv, dtype, dout, sout, ws + L.off_pre,
                                                   L.pre_ws, cs);
            if (r != KDA_OK) st = r;
        }
        ok(cudaEventRecord(in_free[b2], cs));
        ok(cudaEventRecord(out_ready[b2], cs));
        // device -> host: o of this segment
        ok(cudaStreamWaitEvent(s_out, out_ready[b2], 0));
        ok(copy_rows(reinterpret_cast<uint8_t *>(o) + t0 * L.o_tok, (size_t)T * L.o_tok, dout,
                     len * L.o_tok, len * L.o_tok, B, cudaMemcpyDeviceToHost, s_out));
        ok(cudaEventRecord(out_free[b2], s_out));
    }
    if (st == KDA_OK && state_out)
        ok(cudaMemcpyAsync(state_out, state[nseg & 1], state_bytes, cudaMemcpyDeviceToHost, cs));
    // The caller's stream is ordered after every copy this call queued, also
    // when it stopped early on an error, so that the caller may free its
    // buffers once its stream is done.
    for (cudaStream_t side : {s_in, s_out}) {
        if (cudaEventRecord(in_free[0], side) == cudaSuccess)
            cudaStreamWaitEvent(cs, in_free[0], 0);
        else
            cudaStreamSynchronize(side);
    }
    return st;
}

}  // extern "C"
