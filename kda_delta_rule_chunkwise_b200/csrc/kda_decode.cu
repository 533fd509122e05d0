// KDA single-token decode step, state updated in place.
//
// Per (sequence n, head h), with a = exp(max(g, -5)):
//     S' = Diag(a) S;  p = S'^T k;  y = S'^T q;  delta = beta (v - p)
//     S  = S' + k delta^T;  o = S^T q = y + (k.q) delta
// This is one step of S_t = (I - beta k k^T) Diag(exp g) S_{t-1} + beta k v^T,
// o_t = S_t^T q_t: the fixed-size, single-copy-per-request KDA state of
// neurohive.io "Kimi K3 ... overview", section "Training and inference
// infrastructure", advanced by one token.
//
// o is written in fp32 for either input dtype (the step accumulates in fp32).
// The step is bound by HBM: each (n, h) state (dk*dv fp32, 64 KiB at d=128)
// is read once and written once; everything else is ~1 KiB.
//
// Indexed form (continuous batching over a state pool): request n's state is
// pool entry slots[n] of P, so the per-request state stays a single copy that
// the step updates in place wherever the serving layer keeps it.  A slot
// outside [0, P) is not touched: the unit is skipped and ERR_BAD_INDEX is
// recorded in the device error word.  One CTA of 256
// threads per (n, h).  Each thread keeps a (DK/RG) x 4 block of S in
// registers (loaded as coalesced 16-byte vectors, a warp covering whole rows),
// reduces p and y over its rows, the CTA reduces across row groups through
// shared memory, then every thread applies the rank-1 update to its block and
// streams it back.  Loads and stores use the streaming cache hint: the state
// is touched once per step and is far larger than L2.
#include "kda_common.cuh"

namespace kda {

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(256, 2)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const Tin *__restrict__ g, const Tin *__restrict__ beta, float *__restrict__ state,
              float *__restrict__ o, int units, int H, const int32_t *__restrict__ slots, int P,
              uint32_t *err) {
    constexpr int NT = 256;
    constexpr int CG = DV / 4;        // 16-byte column groups per row
    constexpr int RG = NT / CG;       // row groups
    constexpr int RPT = DK / RG;      // rows per thread
    static_assert(DK % RG == 0, "rows must split evenly");
    const int unit = blockIdx.x;
    if (unit >= units) return;
    const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;

    __shared__ float ks[DK], qs[DK], as[DK], vs[DV];
    __shared__ float4 red_p[RG][CG], red_y[RG][CG];
    __shared__ float dl[DV];
    __shared__ float kq_sh, b_sh;

    size_t sunit = (size_t)unit;   // state entry of this (request, head)
    if (slots != nullptr) {
        const int n = unit / H, slot = slots[n];
        if (slot < 0 || slot >= P) {
            if (tid == 0 && err) atomicOr(err, ERR_BAD_INDEX);
            return;
        }
        sunit = (size_t)slot * H + (unit - n * H);
    }
    float4 *S4 = reinterpret_cast<float4 *>(state + sunit * DK * DV);

    // issue the state loads first: they are the long pole
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(S4 + (size_t)(rg + i * RG) * CG + cg);

    for (int c = tid; c < DK; c += NT) {
        const size_t off = (size_t)unit * DK + c;
        ks[c] = to_f32(k[off]);
        qs[c] = to_f32(q[off]);
        as[c] = expf(fmaxf(to_f32(g[off]), -5.f));
    }
    for (int j = tid; j < DV; j += NT) vs[j] = to_f32(v[(size_t)unit * DV + j]);
    if (tid == 0) b_sh = to_f32(beta[unit]);
    __syncthreads();
    if (tid < 32) {
        float a = 0.f;
        for (int c = tid; c < DK; c += 32) a = fmaf(ks[c], qs[c], a);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) a += __shfl_xor_sync(0xffffffffu, a, m);
        if (tid == 0) kq_sh = a;
    }

    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), y = p;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg + i * RG;
        const float a = as[r], kr = ks[r], qr = qs[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        p.x = fmaf(s[i].x, kr, p.x); p.y = fmaf(s[i].y, kr, p.y);
        p.z = fmaf(s[i].z, kr, p.z); p.w = fmaf(s[i].w, kr, p.w);
        y.x = fmaf(s[i].x, qr, y.x); y.y = fmaf(s[i].y, qr, y.y);
        y.z = fmaf(s[i].z, qr, y.z); y.w = fmaf(s[i].w, qr, y.w);
    }
    red_p[rg][cg] = p;
    red_y[rg][cg] = y;
    __syncthreads();
    if (tid < DV) {
        const int c4 = tid >> 2, e = tid & 3;
        float pj = 0.f, yj = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            pj += reinterpret_cast<const float *>(&red_p[r][c4])[e];
            yj += reinterpret_cast<const float *>(&red_y[r][c4])[e];
        }
        const float d = b_sh * (vs[tid] - pj);
        dl[tid] = d;
        o[(size_t)unit * DV + tid] = fmaf(kq_sh, d, yj);
    }
    __syncthreads();
    const float4 d4 = reinterpret_cast<const float4 *>(dl)[cg];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg + i * RG;
        const float kr = ks[r];
        s[i].x = fmaf(kr, d4.x, s[i].x); s[i].y = fmaf(kr, d4.y, s[i].y);
        s[i].z = fmaf(kr, d4.z, s[i].z); s[i].w = fmaf(kr, d4.w, s[i].w);
        __stcs(S4 + (size_t)r * CG + cg, s[i]);
    }
}

}  // namespace kda

#include "kda_launch.h"

namespace kda {

template <int D, typename Tin>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, float *state, void *o, int units, int H,
                                   const int32_t *slots, int P, uint32_t *err, cudaStream_t st) {
    decode_kernel<D, D, Tin><<<units, 256, 0, st>>>(
        (const Tin *)q, (const Tin *)k, (const Tin *)v, (const Tin *)g, (const Tin *)beta,
        state, (float *)o, units, H, slots, P, err);
    cudaError_t e = cudaGetLastError();
    Profiler::mark(st);
    return e;
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *g,
                          const void *beta, float *state, int N, int H, int d, bool bf16,
                          void *o, const int32_t *slots, int P, uint32_t *err, cudaStream_t st) {
    const int units = N * H;
    if (units == 0) return cudaSuccess;
    if (d == 64)
        return bf16 ? launch_decode_t<64, __nv_bfloat16>(q, k, v, g, beta, state, o, units, H,
                                                         slots, P, err, st)
                    : launch_decode_t<64, float>(q, k, v, g, beta, state, o, units, H, slots, P,
                                                 err, st);
    return bf16 ? launch_decode_t<128, __nv_bfloat16>(q, k, v, g, beta, state, o, units, H, slots,
                                                      P, err, st)
                : launch_decode_t<128, float>(q, k, v, g, beta, state, o, units, H, slots, P,
                                              err, st);
}

}  // namespace kda
