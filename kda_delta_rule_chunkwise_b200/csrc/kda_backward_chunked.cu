// KDA backward through the chunked (WY) form, bf16 inputs, d = 128.
//
// The forward runs in its chunked form (kda_prefill_bf16.cu) with a snapshot of
// the state at every chunk start, which leaves the per-chunk factors
// T = (I + Akk)^-1 Diag(beta), R = Aqk T, W = T (K*Gamma), P = Q*Gamma - R (K*Gamma),
// Khat = K*exp(G_L - G) and Gamma_L in the workspace slots.  With dS' the
// gradient of a chunk's end state and dO of its outputs, the adjoint splits
// (the delta rule with per-channel retention of neurohive.io "Kimi K3 ...
// overview", section "Sequence length: hybrid KDA and Gated MLA attention";
// the pages give no formulas for its gradient):
//
//   chain, chunks in reverse (bwd_chain_kernel, per (sequence, head, dv-slice)):
//       dU = Khat dS',   dS = Diag(Gamma_L) dS' + P^T dO - W^T dU
//   per chunk, independently (bwd_factor_kernel):
//       U = T V - W S,  dV = T^T dU + R^T dO,  dT = dU V^T,  dR = dO V^T,
//       dW = -dU S^T,  dP = dO S^T,  dKhat = U dS'^T,  dGamma_L = rowsum(dS' * S)
//   per chunk, independently and without the state (bwd_recompute_kernel,
//   bwd_pullback_kernel, bwd_assemble_kernel): the factor gradients pulled back
//   to q, k, g, beta through the chunk's construction (decay-rescaled Akk / Aqk,
//   the UT solve, R, W, P, Khat).
//
// All of them run fp32 SIMT products on shared-memory tiles; the factors come
// from the forward's fp16 slots.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "sm100.cuh"

namespace kda {
namespace cbw {

using namespace sm100;

constexpr int C = 64, D = 128, NT = 256;

// four consecutive elements as fp32 (p aligned to 4 elements)
__device__ __forceinline__ float4 load4_f32(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// asks the memory system to bring [p, p + bytes) into L2 (p 16-byte aligned,
// bytes a multiple of 16); nothing waits for it
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---- the forward's slot layout (kda_prefill_bf16.cu), read here
constexpr uint32_t kSlotWP = 0, kSlotTR = 32768, kSlotKh = 49152, kSlotGam = 65536;
constexpr uint32_t kSlotBytes = 66560;

__device__ __forceinline__ float h2f(const uint8_t *base, uint32_t off) {
    return __half2float(*reinterpret_cast<const __half *>(base + off));
}
// [-W; P]: 128 rows (0..63 = -W, 64..127 = P) x 128 channels, K-major, 128-byte
// swizzle, 64-channel blocks 16 KiB apart
__device__ __forceinline__ uint32_t wp_off(int r, int c) {
    return (uint32_t)(kSlotWP + (c >> 6) * 16384 + (r >> 3) * 1024 + (r & 7) * 128 +
                      ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}
// [T; R]: 128 rows (0..63 = T, 64..127 = R) x 64 columns, K-major, 128-byte swizzle
__device__ __forceinline__ uint32_t tr_off(int r, int s) {
    return (uint32_t)(kSlotTR + (r >> 3) * 1024 + (r & 7) * 128 + (((s >> 3) ^ (r & 7)) << 4) + (s & 7) * 2);
}
// Khat (token t, channel c): channel contiguous, 128-byte swizzle, 64-channel blocks 8 KiB apart
__device__ __forceinline__ uint32_t kh_off(int t, int c) {
    return (uint32_t)(kSlotKh + (c >> 6) * 8192 + (t >> 3) * 1024 + (t & 7) * 128 +
                      ((((c & 63) >> 3) ^ (t & 7)) << 4) + (c & 7) * 2);
}

// out(i, j, sum_k A(i, k) B(k, j)) for an M x N result, on 256 threads as a
// 16 x 16 grid: thread (ty, tx) owns rows ty + 16 a and columns tx + 16 b.  A, B
// and out are functors; the sums run over k in order (fp32 FMA), so a result
// is the same on every run.
template <int M, int N, int K, typename FA, typename FB, typename FO>
__device__ __forceinline__ void smm(FA A, FB B, FO out) {
    constexpr int TM = M / 16, TN = N / 16;
    static_assert(M % 16 == 0 && N % 16 == 0, "tile");
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float r[TM][TN];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) r[a][b] = 0.f;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        float av[TM], bv[TN];
#pragma unroll
        for (int a = 0; a < TM; ++a) av[a] = A(ty + 16 * a, k);
#pragma unroll
        for (int b = 0; b < TN; ++b) bv[b] = B(k, tx + 16 * b);
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
            for (int b = 0; b < TN; ++b) r[a][b] = fmaf(av[a], bv[b], r[a][b]);
    }
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) out(ty + 16 * a, tx + 16 * b, r[a][b]);
}

// 64-row products whose terms vanish outside a band of k that depends on the
// row: thread (ty, tx) owns the four consecutive rows 4 ty .. 4 ty + 3 (so warp w
// owns rows 8w .. 8w + 7) and columns tx + 16 b, and sums
//   out(i, j, sum_{k in [lo1, hi1)} A1(i, k) B1(k, j) + sum_{k in [lo2, hi2)} A2(i, k) B2(k, j))
// with the ranges taken per warp (range(w, lo1, hi1, lo2, hi2)), in order of k.
template <int N, typename FA1, typename FB1, typename FA2, typename FB2, typename FR, typename FO>
__device__ __forceinline__ void smm_rows2(FA1 A1, FB1 B1, FA2 A2, FB2 B2, FR range, FO out) {
    constexpr int TM = 4, TN = N / 16;
    static_assert(N % 16 == 0, "tile");
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    int lo1, hi1, lo2, hi2;
    range(threadIdx.x >> 5, lo1, hi1, lo2, hi2);
    float r[TM][TN];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) r[a][b] = 0.f;
    auto run = [&](auto A, auto B, int lo, int hi) {
#pragma unroll 4
        for (int k = lo; k < hi; ++k) {
            float av[TM], bv[TN];
#pragma unroll
            for (int a = 0; a < TM; ++a) av[a] = A(TM * ty + a, k);
#pragma unroll
            for (int b = 0; b < TN; ++b) bv[b] = B(k, tx + 16 * b);
#pragma unroll
            for (int a = 0; a < TM; ++a)
#pragma unroll
                for (int b = 0; b < TN; ++b) r[a][b] = fmaf(av[a], bv[b], r[a][b]);
        }
    };
    run(A1, B1, lo1, hi1);
    run(A2, B2, lo2, hi2);
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) out(TM * ty + a, tx + 16 * b, r[a][b]);
}
// The same banded sums with row-major fp32 right operands (ldb a multiple of 4):
// thread (ty, tx) owns rows 4 ty .. 4 ty + 3 and the four consecutive columns
// 4 tx + 64 b + e, read as one 16-byte load per k and b (as smm_pb).
template <int N, typename FA1, typename FA2, typename FR, typename FO>
__device__ __forceinline__ void smm_rows2_pb(FA1 A1, const float *B1, int ldb1, FA2 A2, const float *B2,
                                             int ldb2, FR range, FO out, const int lt = (int)threadIdx.x) {
    constexpr int TM = 4, NB = N / 64;
    static_assert(N % 64 == 0, "tile");
    const int tx = lt & 15, ty = lt >> 4;
    int lo1, hi1, lo2, hi2;
    range(lt >> 5, lo1, hi1, lo2, hi2);
    float r[TM][NB][4];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) r[a][b][e] = 0.f;
    auto run = [&](auto A, const float *B, int ldb, int lo, int hi) {
#pragma unroll 4
        for (int k = lo; k < hi; ++k) {
            float av[TM];
            float4 bv[NB];
#pragma unroll
            for (int a = 0; a < TM; ++a) av[a] = A(TM * ty + a, k);
#pragma unroll
            for (int b = 0; b < NB; ++b) bv[b] = *reinterpret_cast<const float4 *>(B + k * ldb + 64 * b + 4 * tx);
#pragma unroll
            for (int a = 0; a < TM; ++a)
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    r[a][b][0] = fmaf(av[a], bv[b].x, r[a][b][0]);
                    r[a][b][1] = fmaf(av[a], bv[b].y, r[a][b][1]);
                    r[a][b][2] = fmaf(av[a], bv[b].z, r[a][b][2]);
                    r[a][b][3] = fmaf(av[a], bv[b].w, r[a][b][3]);
                }
        }
    };
    run(A1, B1, ldb1, lo1, hi1);
    run(A2, B2, ldb2, lo2, hi2);
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) out(TM * ty + a, 64 * b + 4 * tx + e, r[a][b][e]);
}

// one product: the second pair is empty
template <int N, typename FA, typename FB, typename FR, typename FO>
__device__ __forceinline__ void smm_rows(FA A, FB B, FR range, FO out) {
    smm_rows2<N>(A, B, A, B,
                 [&](int w, int &lo1, int &hi1, int &lo2, int &hi2) {
                     range(w, lo1, hi1);
                     lo2 = hi2 = 0;
                 },
                 out);
}

// The same product when both operands are row-major fp32 with K contiguous:
// out(i, j, sum_k A[i][k] B[j][k]) (A times B transposed), four k at a time as
// 16-byte loads (lda, ldb multiples of 4, K a multiple of 4).  Same thread
// mapping and summation order as smm.
// LOWER: only the 16 x 16 blocks on and below the diagonal are summed; the
// blocks above it come out as 0.
template <int M, int N, int K, bool LOWER = false, typename FO>
__device__ __forceinline__ void smm_nt(const float *A, int lda, const float *B, int ldb, FO out,
                                       const int lt = (int)threadIdx.x) {
    constexpr int TM = M / 16, TN = N / 16;
    static_assert(M % 16 == 0 && N % 16 == 0 && K % 4 == 0, "tile");
    const int tx = lt & 15, ty = lt >> 4;
    float r[TM][TN];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) r[a][b] = 0.f;
#pragma unroll 2
    for (int k = 0; k < K; k += 4) {
        float4 av[TM], bv[TN];
#pragma unroll
        for (int a = 0; a < TM; ++a) av[a] = *reinterpret_cast<const float4 *>(A + (ty + 16 * a) * lda + k);
#pragma unroll
        for (int b = 0; b < TN; ++b) bv[b] = *reinterpret_cast<const float4 *>(B + (tx + 16 * b) * ldb + k);
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
            for (int b = 0; b < TN; ++b) {
                if (LOWER && b > a) continue;
                float x = r[a][b];
                x = fmaf(av[a].x, bv[b].x, x);
                x = fmaf(av[a].y, bv[b].y, x);
                x = fmaf(av[a].z, bv[b].z, x);
                r[a][b] = fmaf(av[a].w, bv[b].w, x);
            }
    }
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TN; ++b) out(ty + 16 * a, tx + 16 * b, (LOWER && b > a) ? 0.f : r[a][b]);
}

// The product with a row-major fp32 right operand B (ldb a multiple of 4):
// out(i, j, sum_k A(i, k) B[k][j]).  Thread (ty, tx) owns rows ty + 16 a and the
// four consecutive columns 4 tx + 64 b + e, read as one 16-byte load per k and b.
// The sums run over k in order, as in smm.
template <int M, int N, int K, typename FA, typename FO>
__device__ __forceinline__ void smm_pb(FA A, const float *B, int ldb, FO out, const int lt = (int)threadIdx.x) {
    constexpr int TM = M / 16, NB = N / 64;
    static_assert(M % 16 == 0 && N % 64 == 0, "tile");
    const int tx = lt & 15, ty = lt >> 4;
    float r[TM][NB][4];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) r[a][b][e] = 0.f;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        float av[TM];
        float4 bv[NB];
#pragma unroll
        for (int a = 0; a < TM; ++a) av[a] = A(ty + 16 * a, k);
#pragma unroll
        for (int b = 0; b < NB; ++b) bv[b] = *reinterpret_cast<const float4 *>(B + k * ldb + 64 * b + 4 * tx);
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                r[a][b][0] = fmaf(av[a], bv[b].x, r[a][b][0]);
                r[a][b][1] = fmaf(av[a], bv[b].y, r[a][b][1]);
                r[a][b][2] = fmaf(av[a], bv[b].z, r[a][b][2]);
                r[a][b][3] = fmaf(av[a], bv[b].w, r[a][b][3]);
            }
    }
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) out(ty + 16 * a, 64 * b + 4 * tx + e, r[a][b][e]);
}

// rows [a, b) of sequence n: equal-length batch, or the chunk table's clamped offsets
__device__ __forceinline__ void seq_rows(const int32_t *hdr, bool packed, int64_t T, int N, int n,
                                         int64_t &a, int64_t &b) {
    if (packed) {
        a = hdr[(N + 1) + n];
        b = hdr[(N + 1) + n + 1];
    } else {
        a = (int64_t)n * T;
        b = a + T;
    }
}
__device__ __forceinline__ int first_chunk(const int32_t *hdr, bool packed, int64_t T, int n) {
    return packed ? hdr[n] : n * (int)((T + C - 1) / C);
}
// state at the start of chunk j of sequence n: state_in (j = 0, or zero), else the
// forward's snapshot after j C tokens
__device__ __forceinline__ const float *chunk_state(const int32_t *hdr, bool packed, int64_t T, int N,
                                                    int H, int n, int h, int j, const float *state_in,
                                                    const float *snaps) {
    if (j == 0) return state_in ? state_in + ((size_t)n * H + h) * D * D : nullptr;
    const int64_t e = packed ? (int64_t)hdr[2 * (N + 1) + n] + j - 1
                             : (int64_t)n * ((T - 1) / C) + j - 1;
    return snaps + ((size_t)e * H + h) * D * D;
}

// ======================================================================
// chain: dU_j = Khat_j dS'_j, dS_j = Diag(Gamma_L) dS'_j + P_j^T dO_j - W_j^T dU_j
// one CTA per (sequence, head, 32-column slice), chunks in reverse
// ======================================================================
constexpr int CH_DVS = 32;
constexpr int CH_LD = CH_DVS + 4;
constexpr uint32_t CH_SLOT = 0;                                   // 2 slot images (66 560 B each)
constexpr uint32_t CH_DS = 2 * kSlotBytes;                        // dS' [128][CH_LD] fp32
constexpr uint32_t CH_Y = CH_DS + 128 * CH_LD * 4;                // dU  [64][CH_LD]
constexpr uint32_t CH_DO = CH_Y + 64 * CH_LD * 4;                 // dO  2 x [64][CH_LD]
constexpr uint32_t CH_BAR = CH_DO + 2 * 64 * CH_LD * 4;           // one slot-copy mbarrier per image
constexpr uint32_t CH_SMEM = CH_BAR + 16;
static_assert(CH_SMEM <= 227 * 1024, "chain kernel shared memory");
static_assert(kSlotBytes % 16 == 0, "slot images start on 16-byte boundaries");
static_assert(CH_DVS == 32 && NT == 256, "chain kernel thread map: 32 x 8 threads, four columns each");

// four consecutive fp16 channels of a slot image (8 bytes at byte offset off)
__device__ __forceinline__ float4 h4(const uint8_t *img, uint32_t off) {
    const uint2 u = *reinterpret_cast<const uint2 *>(img + off);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__global__ void __launch_bounds__(NT, 1)
bwd_chain_kernel(const uint8_t *__restrict__ fws, const int32_t *__restrict__ cu, int64_t T, int N,
                 int H, const float *__restrict__ dout, const float *dstate_out,
                 float *__restrict__ ws_dS, float *__restrict__ ws_dU, float *dstate_in,
                 uint32_t hdr_bytes, uint32_t *err) {
    constexpr int NSL = D / CH_DVS;
    extern __shared__ __align__(16) uint8_t sm[];
    const int slice = blockIdx.x % NSL, unit = blockIdx.x / NSL;
    const int n = unit / H, h = unit % H;
    if (n >= N) return;
    const int tid = threadIdx.x;
    const int j0 = slice * CH_DVS;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(fws);
    const bool packed = cu != nullptr;
    int64_t ra, rb;
    seq_rows(hdr, packed, T, N, n, ra, rb);
    const int nch = (int)((rb - ra + C - 1) / C);
    const int c0 = first_chunk(hdr, packed, T, n);
    float *dS = reinterpret_cast<float *>(sm + CH_DS);
    float *Y = reinterpret_cast<float *>(sm + CH_Y);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + CH_BAR);
    const size_t sbase = ((size_t)n * H + h) * D * D;
    // The products read Khat, -W, P and Gamma_L straight from the fp16 slot image
    // (8 bytes = 4 channels of one row per load; the 128-byte swizzle keeps a
    // piece's 8 channels together). Two images: the next chunk's comes in by one
    // bulk copy (completing on its own barrier) and its dO rows by cp.async into
    // the other dO buffer while this chunk runs.
    auto img_of = [&](int step) { return sm + CH_SLOT + (uint32_t)(step & 1) * kSlotBytes; };
    auto issue_slot = [&](int jn, int step) {
        if (tid == 0) {
            fence_async_smem();   // the previous readers of this image come first
            mbar_arrive_expect_tx(&bar[step & 1], kSlotBytes);
            bulk_g2s(img_of(step), fws + hdr_bytes + ((size_t)(c0 + jn) * H + h) * kSlotBytes, kSlotBytes,
                     &bar[step & 1]);
        }
    };
    auto issue_dO = [&](int jn, int step) {
        float *buf = reinterpret_cast<float *>(sm + CH_DO) + (step & 1) * 64 * CH_LD;
        const int64_t tn = ra + (int64_t)jn * C;
        const int Ln = (int)((rb - tn) < C ? (rb - tn) : C);
        for (int i = tid; i < 64 * (CH_DVS / 4); i += NT) {   // 16-byte pieces
            const int t = i / (CH_DVS / 4), p4 = i % (CH_DVS / 4);
            const float *src = dout + ((size_t)(tn + (t < Ln ? t : 0)) * H + h) * D + j0 + 4 * p4;
            cp_async16(buf + t * CH_LD + 4 * p4, src, t < Ln ? 16u : 0u);
        }
        cp_async_commit();
    };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_fence_init();
    }
    // dS' of the last chunk = dL/dS_final
    for (int i = tid; i < 128 * (CH_DVS / 4); i += NT) {
        const int c = i / (CH_DVS / 4), jj = (i % (CH_DVS / 4)) * 4;
        *reinterpret_cast<float4 *>(dS + c * CH_LD + jj) =
            dstate_out ? *reinterpret_cast<const float4 *>(dstate_out + sbase + (size_t)c * D + j0 + jj)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    if (nch > 0) {
        issue_slot(nch - 1, 0);
        issue_dO(nch - 1, 0);
    }
    bool ok = true;
    int iss0 = nch > 0 ? 1 : 0, iss1 = 0, wt0 = 0, wt1 = 0;   // slot copies issued / waited for, per image
    // thread (q, cq), q = 4 warp + lane / 8, cq = lane % 8, owns columns
    // 4 cq .. 4 cq + 3 of the slice
    const int cq = tid & 7, q = tid >> 3;
    for (int step = 0; step < nch; ++step) {
        const int j = nch - 1 - step;
        const size_t item = (size_t)(c0 + j) * H + h;
        const uint8_t *img = img_of(step);
        const float *dO = reinterpret_cast<const float *>(sm + CH_DO) + (step & 1) * 64 * CH_LD;
        // the next chunk's image and dO, into the buffers the previous step released
        if (j > 0 && ok) {
            issue_slot(j - 1, step + 1);
            issue_dO(j - 1, step + 1);
            if ((step + 1) & 1) ++iss1; else ++iss0;
        }
        // dS' of this chunk, for the factor kernel
        for (int i = tid; i < 128 * (CH_DVS / 4); i += NT) {
            const int c = i / (CH_DVS / 4), jj = (i % (CH_DVS / 4)) * 4;
            *reinterpret_cast<float4 *>(ws_dS + (item * D + c) * D + j0 + jj) =
                *reinterpret_cast<const float4 *>(dS + c * CH_LD + jj);
        }
        bool got = false;   // this chunk's image has landed
        if (ok) {
            got = mbar_wait(&bar[step & 1], (step >> 1) & 1, err);
            if (got) {
                if (step & 1) ++wt1; else ++wt0;
            }
        }
        if (j > 0 && ok) cp_async_wait_group1(); else cp_async_wait_all();   // this thread's dO pieces
        ok = __syncthreads_and(got) != 0;
        if (!ok) break;
        // dU = Khat dS': rows 2q, 2q + 1, four channels at a time
        {
            float r[2][4];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int e = 0; e < 4; ++e) r[x][e] = 0.f;
#pragma unroll 2
            for (int c = 0; c < 128; c += 4) {
                const float4 a0 = h4(img, kh_off(2 * q, c)), a1 = h4(img, kh_off(2 * q + 1, c));
                const float av0[4] = {a0.x, a0.y, a0.z, a0.w}, av1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float4 b = *reinterpret_cast<const float4 *>(dS + (c + kk) * CH_LD + 4 * cq);
                    r[0][0] = fmaf(av0[kk], b.x, r[0][0]); r[0][1] = fmaf(av0[kk], b.y, r[0][1]);
                    r[0][2] = fmaf(av0[kk], b.z, r[0][2]); r[0][3] = fmaf(av0[kk], b.w, r[0][3]);
                    r[1][0] = fmaf(av1[kk], b.x, r[1][0]); r[1][1] = fmaf(av1[kk], b.y, r[1][1]);
                    r[1][2] = fmaf(av1[kk], b.z, r[1][2]); r[1][3] = fmaf(av1[kk], b.w, r[1][3]);
                }
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const float4 o = make_float4(r[x][0], r[x][1], r[x][2], r[x][3]);
                *reinterpret_cast<float4 *>(Y + (2 * q + x) * CH_LD + 4 * cq) = o;
                *reinterpret_cast<float4 *>(ws_dU + (item * 64 + 2 * q + x) * D + j0 + 4 * cq) = o;
            }
        }
        __syncthreads();
        // dS = Diag(Gamma_L) dS' + P^T dO + (-W)^T dU   (the slot holds -W): channels
        // 4q .. 4q + 3; each thread overwrites only the elements it alone reads
        {
            float r[4][4];
            const float4 gm4 = *reinterpret_cast<const float4 *>(img + kSlotGam + 16 * q);
            const float gmv[4] = {gm4.x, gm4.y, gm4.z, gm4.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float4 d = *reinterpret_cast<const float4 *>(dS + (4 * q + x) * CH_LD + 4 * cq);
                r[x][0] = gmv[x] * d.x; r[x][1] = gmv[x] * d.y; r[x][2] = gmv[x] * d.z; r[x][3] = gmv[x] * d.w;
            }
#pragma unroll 4
            for (int t = 0; t < 64; ++t) {
                const float4 pw = h4(img, wp_off(64 + t, 4 * q));
                const float4 wn = h4(img, wp_off(t, 4 * q));
                const float4 o = *reinterpret_cast<const float4 *>(dO + t * CH_LD + 4 * cq);
                const float4 y = *reinterpret_cast<const float4 *>(Y + t * CH_LD + 4 * cq);
                const float pv[4] = {pw.x, pw.y, pw.z, pw.w}, wv[4] = {wn.x, wn.y, wn.z, wn.w};
                const float ov[4] = {o.x, o.y, o.z, o.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int e = 0; e < 4; ++e) r[x][e] = fmaf(pv[x], ov[e], fmaf(wv[x], yv[e], r[x][e]));
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
                *reinterpret_cast<float4 *>(dS + (4 * q + x) * CH_LD + 4 * cq) =
                    make_float4(r[x][0], r[x][1], r[x][2], r[x][3]);
        }
        __syncthreads();   // dS, Y, this image and this dO buffer are consumed
    }
    // copies given up on (after a timeout) land before exit
    if (tid == 0) {
        for (; wt0 < iss0; ++wt0) mbar_wait(&bar[0], wt0 & 1, err, 1ull << 28);
        for (; wt1 < iss1; ++wt1) mbar_wait(&bar[1], wt1 & 1, err, 1ull << 28);
    }
    cp_async_wait_all();
    __syncthreads();
    if (dstate_in && ok)
        for (int i = tid; i < 128 * (CH_DVS / 4); i += NT) {
            const int c = i / (CH_DVS / 4), jj = (i % (CH_DVS / 4)) * 4;
            *reinterpret_cast<float4 *>(dstate_in + sbase + (size_t)c * D + j0 + jj) =
                *reinterpret_cast<const float4 *>(dS + c * CH_LD + jj);
        }
}


// ======================================================================
// factor gradients, one CTA per (chunk, head):
//   U = T V - W S,  dV = T^T dU + R^T dO (the final dv),  dT = dU V^T,  dR = dO V^T,
//   dW = -dU S^T,  dP = dO S^T,  dKhat = U dS'^T,  dGamma_L = rowsum(dS' * S)
// ======================================================================
constexpr int LD = 132;                                  // fp32 row stride of 128-wide tiles
constexpr uint32_t FG_FLOATS = 64 * 64 * 2 + 64 * 128 * 3 + 128;
constexpr uint32_t FG_DT = 0, FG_DR = 4096, FG_DW = 8192, FG_DP = 16384, FG_DKH = 24576, FG_DGL = 32768;
constexpr int L6 = 68;                                   // fp32 row stride of 64-wide tiles
constexpr uint32_t F_R0 = 0;                             // V [64][LD] + T, R [64][L6] | S [128][LD]
constexpr uint32_t F_T = 64 * LD * 4;                    //   T [64][L6] after V
constexpr uint32_t F_RR = F_T + 64 * L6 * 4;             //   R [64][L6]
constexpr uint32_t F_R1 = F_RR + 64 * L6 * 4;           // dU [64][LD] + dO [64][LD] | dS' [128][LD]
constexpr uint32_t F_R2 = F_R1 + 128 * LD * 4;           // U [64][LD] (dV first)
constexpr uint32_t F_WN = F_R2 + 64 * LD * 4;            // -W [64][LD]
constexpr uint32_t F_BAR = F_WN + 64 * LD * 4;             // 3 mbarriers: dU + dO, S, dS'
constexpr uint32_t F_SMEM = F_BAR + 32;
static_assert(128 * LD * 4 <= F_R1, "factor kernel layout: S fits the first region");
static_assert(F_SMEM <= 227 * 1024, "factor kernel shared memory");

// (sequence, chunk within it) of a global chunk index: equal-length arithmetic,
// or the last sequence whose first chunk is <= cidx (binary search)
__device__ __forceinline__ void locate_chunk(const int32_t *hdr, bool packed, int64_t T, int N,
                                             int cidx, int &n, int &j) {
    if (!packed) {
        const int cps = (int)((T + C - 1) / C);
        n = cidx / cps;
        j = cidx - n * cps;
        return;
    }
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (hdr[mid] <= cidx) lo = mid; else hi = mid - 1;
    }
    n = lo;
    j = cidx - hdr[lo];
}

// 512 threads: two groups of 256 run independent products side by side (the
// products' 16 x 16 thread grids are per group), so that each SM has 16 warps
// to hide shared-memory and load latency with the same per-thread tiles.
constexpr int FNT = 2 * NT;
__device__ __forceinline__ void group_bar(int id) { asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory"); }

template <typename Tin>
__global__ void __launch_bounds__(FNT, 1)
bwd_factor_kernel(const uint8_t *__restrict__ fws, const int32_t *__restrict__ cu, int64_t T, int N,
                  int H, const Tin *__restrict__ v, const float *state_in,
                  const float *__restrict__ snaps, const float *__restrict__ dout,
                  const float *__restrict__ ws_dS, const float *__restrict__ ws_dU,
                  float *__restrict__ fg, float *__restrict__ dv, uint32_t hdr_bytes, uint32_t *err) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(fws);
    const bool packed = cu != nullptr;
    const int total = packed ? hdr[N] : N * (int)((T + C - 1) / C);
    const int cidx = blockIdx.x / H, h = blockIdx.x % H;
    if (cidx >= total) return;
    int n, j;
    locate_chunk(hdr, packed, T, N, cidx, n, j);
    int64_t ra, rb;
    seq_rows(hdr, packed, T, N, n, ra, rb);
    const int64_t t0 = ra + (int64_t)j * C;
    const int L = (int)((rb - t0) < C ? (rb - t0) : C);
    const size_t item = (size_t)cidx * H + h;
    const uint8_t *slot = fws + hdr_bytes + item * kSlotBytes;
    float *V = reinterpret_cast<float *>(sm + F_R0);
    float *Tf = reinterpret_cast<float *>(sm + F_T);
    float *Rf = reinterpret_cast<float *>(sm + F_RR);
    float *dU = reinterpret_cast<float *>(sm + F_R1);
    float *dO = dU + 64 * LD;
    float *U = reinterpret_cast<float *>(sm + F_R2);
    float *Wnf = reinterpret_cast<float *>(sm + F_WN);
    float *out = fg + item * FG_FLOATS;

    const float *Sg = chunk_state(hdr, packed, T, N, H, n, h, j, state_in, snaps);
    const float *dSg = ws_dS + item * D * D;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + F_BAR);
    if (tid == 0) {
        // S and dS' (64 KB each) are read in phases 2 and 3: start them toward L2
        if (Sg) prefetch_l2(Sg, D * D * 4);
        prefetch_l2(dSg, D * D * 4);
        for (int b = 0; b < 3; ++b) mbar_init(&bars[b], 1);
        mbar_fence_init();
    }
    __syncthreads();
    // The fp32 operands dU, dO, S and dS' come in by bulk copies, one per 512-byte
    // row, each group completing on its own barrier; the issuing threads fence
    // against the generic accesses the region saw before (barrier first).
    auto copy_rows = [&](float *dst, const float *src, size_t src_stride, int rows, int t_lo, uint64_t *bar) {
        const int t = tid - t_lo;
        if (t >= 0 && t < rows) {
            fence_async_smem();
            bulk_g2s(dst + t * LD, src + (size_t)t * src_stride, 512, bar);
        }
    };
    // ---- phase 1: dU, dO (rows past the chunk's end are zero) by bulk copies;
    // V, [T; R] and -W by 16-byte loads (rows of 128 channels; every base is
    // 16-byte aligned)
    const int grp = tid >> 8, lt = tid & 255;   // product group, thread within it
    if (tid == 0) mbar_arrive_expect_tx(&bars[0], (uint32_t)(64 + L) * 512u);
    copy_rows(dU, ws_dU + item * 64 * D, D, 64, 0, &bars[0]);
    copy_rows(dO, dout + ((size_t)t0 * H + h) * D, (size_t)H * D, L, 64, &bars[0]);
    for (int i = tid; i < 64 * 32; i += FNT) {
        const int t = i >> 5, c = (i & 31) * 4;
        const size_t off = ((size_t)(t0 + t) * H + h) * D + c;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(V + t * LD + c) = t < L ? load4_f32(v + off) : z;
        if (t >= L) *reinterpret_cast<float4 *>(dO + t * LD + c) = z;
    }
    // [T; R] and -W out of the slot by 16-byte pieces (8 fp16 of one row; the
    // swizzle permutes whole pieces within a row)
    auto unpack_h8 = [](uint4 u, float *dst) {
        const __half2 *hp = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(hp[e]);
            dst[2 * e] = f.x;
            dst[2 * e + 1] = f.y;
        }
    };
    for (int i = tid; i < 128 * 8; i += FNT) {   // [T; R]: 128 rows x 8 pieces
        const int r = i >> 3, pc = i & 7, lc = pc ^ (r & 7);
        const uint4 u = *reinterpret_cast<const uint4 *>(slot + kSlotTR + (r >> 3) * 1024 + (r & 7) * 128 + pc * 16);
        unpack_h8(u, r < 64 ? Tf + r * L6 + 8 * lc : Rf + (r - 64) * L6 + 8 * lc);
    }
    for (int i = tid; i < 64 * 16; i += FNT) {   // -W: rows 0..63 of [-W; P], 2 x 8 pieces per row
        const int r = i >> 4, kb = (i >> 3) & 1, pc = i & 7, lc = pc ^ (r & 7);
        const uint4 u = *reinterpret_cast<const uint4 *>(slot + kSlotWP + kb * 16384 + (r >> 3) * 1024 +
                                                         (r & 7) * 128 + pc * 16);
        unpack_h8(u, Wnf + r * LD + 64 * kb + 8 * lc);
    }
    // a copy given up on (after a timeout) lands before the CTA exits; the item's
    // results are then not written (the error word says why)
    auto drain = [&](int nb) {
        if (tid == 0)
            for (int b = 0; b < nb; ++b)
                if (b != 1 || Sg) mbar_wait(&bars[b], 0, err, 1ull << 28);
        __syncthreads();
    };
    if (!__syncthreads_and(mbar_wait(&bars[0], 0, err))) {
        drain(1);
        return;
    }
    auto Tm = [&](int r, int s2) { return Tf[r * L6 + s2]; };   // T[r][s]
    auto Rm = [&](int r, int s2) { return Rf[r * L6 + s2]; };   // R[r][s]
    if (grp == 0) {
        // dV = T^T dU + R^T dO (into U's buffer, then the rows of the chunk out); T
        // and R are lower triangular, so row s sums t >= s only
        smm_rows2_pb<128>([&](int s, int t) { return Tm(t, s); }, dU, LD, [&](int s, int t) { return Rm(t, s); },
                          dO, LD,
                          [](int w, int &lo1, int &hi1, int &lo2, int &hi2) { lo1 = lo2 = 8 * w; hi1 = hi2 = 64; },
                          [&](int s, int c, float x) { U[s * LD + c] = x; }, lt);
        group_bar(1);
        for (int i = lt; i < 64 * 32; i += NT) {
            const int s = i >> 5, c = (i & 31) * 4;
            if (s < L)
                *reinterpret_cast<float4 *>(dv + ((size_t)(t0 + s) * H + h) * D + c) =
                    *reinterpret_cast<const float4 *>(U + s * LD + c);
        }
        group_bar(1);   // U's buffer (dV) is read out
        // U = T V (row t sums s <= t)
        smm_rows2_pb<128>([&](int t, int s) { return Tm(t, s); }, V, LD, [&](int t, int s) { return Tm(t, s); }, V,
                          LD,
                          [](int w, int &lo1, int &hi1, int &lo2, int &hi2) { lo1 = 0; hi1 = 8 * w + 8; lo2 = hi2 = 0; },
                          [&](int t, int c, float x) { U[t * LD + c] = x; }, lt);
    } else {
        // dT = dU V^T, dR = dO V^T
        // (only the blocks on and below the diagonal matter: T and R are lower
        // triangular, and the pull-back reads no entry of dT or dR above it)
        smm_nt<64, 64, 128, true>(dU, LD, V, LD, [&](int t, int s, float x) { out[FG_DT + t * 64 + s] = x; }, lt);
        smm_nt<64, 64, 128, true>(dO, LD, V, LD, [&](int t, int s, float x) { out[FG_DR + t * 64 + s] = x; }, lt);
    }
    __syncthreads();   // V and [T; R] are consumed

    // ---- phase 2: S (zero without an initial state)
    float *S = reinterpret_cast<float *>(sm + F_R0);
    if (Sg) {
        if (tid == 0) mbar_arrive_expect_tx(&bars[1], 128u * 512u);
        copy_rows(S, Sg, D, 128, 0, &bars[1]);
    } else {
        for (int i = tid; i < 128 * 32; i += FNT)
            *reinterpret_cast<float4 *>(S + (i >> 5) * LD + (i & 31) * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (!__syncthreads_and(Sg ? mbar_wait(&bars[1], 0, err) : true)) {
        drain(2);
        return;
    }
    // group 0: U += (-W) S (the slot holds -W); group 1: dW = -dU S^T; each group
    // then half of dP = dO S^T (key channels 64 g .. 64 g + 63)
    if (grp == 0)
        smm_pb<64, 128, 128>([&](int t, int c) { return Wnf[t * LD + c]; }, S, LD,
                             [&](int t, int jj, float x) { U[t * LD + jj] += x; }, lt);
    else
        smm_nt<64, 128, 128>(dU, LD, S, LD, [&](int t, int c, float x) { out[FG_DW + t * 128 + c] = -x; }, lt);
    smm_nt<64, 64, 128>(dO, LD, S + 64 * grp * LD, LD,
                        [&](int t, int c, float x) { out[FG_DP + t * 128 + 64 * grp + c] = x; }, lt);
    __syncthreads();   // dU and dO are consumed

    // ---- phase 3: dS'
    float *dSp = reinterpret_cast<float *>(sm + F_R1);
    if (tid == 0) mbar_arrive_expect_tx(&bars[2], 128u * 512u);
    copy_rows(dSp, dSg, D, 128, 0, &bars[2]);
    if (!__syncthreads_and(mbar_wait(&bars[2], 0, err))) {
        drain(3);
        return;
    }
    if (tid < 128) {
        float a = 0.f;
        for (int jj = 0; jj < 128; ++jj) a = fmaf(dSp[tid * LD + jj], S[tid * LD + jj], a);
        out[FG_DGL + tid] = a;
    }
    // dKhat = U dS'^T (key channels 64 g .. 64 g + 63 per group)
    smm_nt<64, 64, 128>(U, LD, dSp + 64 * grp * LD, LD,
                        [&](int t, int c, float x) { out[FG_DKH + t * 128 + 64 * grp + c] = x; }, lt);
}


// ======================================================================
// input side, one CTA per (chunk, head), in three kernels with the chunk's
// 64 x 64 intermediates in the workspace (IW_* offsets, floats per item):
//   recompute   Aqk, M (decay-rescaled, the forward's 16-row references)
//   pullback    X = (I + Diag(beta) M)^-1, T, R, K*Gamma;
//               dR' = dR - dP (K*Gamma)^T,  dKt = T^T dW - R^T dP,
//               dT' = dT + Aqk^T dR' + dW (K*Gamma)^T,  dAqk = tril(dR' T^T),
//               dbeta = colsum(X * dT') + rowsum(dAkk * M),
//               dAkk = strict_tril(-X^T (dT' Diag(beta)) X^T),  dM = Diag(beta) dAkk
//   assemble    the decayed adjoints of Aqk (q, k) and M (k, k), then
//               dq = dP Gamma + da_q,
//               dk = dKt Gamma + dKhat Gamma_L / Gamma + db_qk + da_k + db_kk,
//               dG = (Q*Gamma) dP + (K*Gamma) dKt - Khat dKhat + q da_q - k db_qk
//                    + k da_k - k db_kk  (+ sum_r Khat dKhat + Gamma_L dGamma_L at row L-1),
//               dg = reverse cumsum of dG over the rows, 0 where g < -5
// A decayed form F[r,s] = sum_c a_r b_s exp(G_r - G_s) (s <= r) has
//   da_r = E1_r sum_s dF[r,s] b_s exp(R_a - G_s)          (a = block of r)
//   db_s = sum_a exp(R_a - G_s) sum_{r in a} dF[r,s] a_r E1_r
// with E1_r = exp(G_r - R_a) in [e^-80, 1] and exp(R_a - G_s) <= e^80: the
// factorisation the forward uses, in fp32.
// ======================================================================
constexpr uint32_t IW_AQK = 0, IW_M = 4096, IW_DAQK = 8192, IW_DM = 12288, IW_DKT = 16384,
                   IW_DB = 16384 + 8192, IW_FLOATS = 16384 + 8192 + 64;

// G = cumsum(max(g, -5)) over the chunk's rows (rows past L decay by nothing), and
// the block references R_a = G at the end of block a - 1 (R_0 = 0), per channel
// (all threads: the rows load in parallel, then one thread per channel scans them
// in shared memory; G is complete after the caller's next barrier)
template <typename Tin>
__device__ __forceinline__ void chunk_cumsum(const Tin *g, int64_t t0, int H, int h, int L, float *G,
                                             float *Rref) {
    const int tid = threadIdx.x;
    for (int i = tid; i < 64 * 32; i += NT) {   // 4 channels per load
        const int r = i >> 5, c = (i & 31) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < L) {
            x = load4_f32(g + ((size_t)(t0 + r) * H + h) * D + c);
            x = make_float4(fmaxf(x.x, -5.f), fmaxf(x.y, -5.f), fmaxf(x.z, -5.f), fmaxf(x.w, -5.f));
        }
        *reinterpret_cast<float4 *>(G + r * LD + c) = x;
    }
    __syncthreads();
    if (tid < 128) {
        float acc = 0.f;
        for (int r = 0; r < 64; ++r) {
            acc += G[r * LD + tid];
            G[r * LD + tid] = acc;
            if ((r & 15) == 15 && r < 63) Rref[((r + 1) >> 4) * 128 + tid] = acc;
        }
        Rref[tid] = 0.f;
    }
}

constexpr int RC_LDK = 136;   // row stride (elements) of the staged k rows: 16-byte aligned rows
template <typename Tin>
__global__ void __launch_bounds__(NT, 2)
bwd_recompute_kernel(const uint8_t *__restrict__ fws, const int32_t *__restrict__ cu, int64_t T,
                     int N, int H, const Tin *__restrict__ q, const Tin *__restrict__ k,
                     const Tin *__restrict__ g, float *__restrict__ iw) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(fws);
    const bool packed = cu != nullptr;
    const int total = packed ? hdr[N] : N * (int)((T + C - 1) / C);
    const int cidx = blockIdx.x / H, h = blockIdx.x % H;
    if (cidx >= total) return;
    int n, j;
    locate_chunk(hdr, packed, T, N, cidx, n, j);
    int64_t ra, rb;
    seq_rows(hdr, packed, T, N, n, ra, rb);
    const int64_t t0 = ra + (int64_t)j * C;
    const int L = (int)((rb - t0) < C ? (rb - t0) : C);
    float *G = reinterpret_cast<float *>(sm);              // [64][LD]
    float *KF = G + 64 * LD;                               // [64][LD]: k_s exp(R_a - G_s), block a's
    float *QE = KF + 64 * LD;                              // [16][LD]: q_r E1_r, rows of block a
    float *KE = QE + 16 * LD;                              // [16][LD]: k_r E1_r
    float *Rref = KE + 16 * LD;                            // [4][128]
    static_assert(sizeof(Tin) == 2, "the recompute kernel's shared memory is sized for 16-bit k");
    Tin *Kb = reinterpret_cast<Tin *>(Rref + 4 * 128);     // [64][RC_LDK]: k as given (0 past the end)
    float *out = iw + ((size_t)cidx * H + h) * IW_FLOATS;
    chunk_cumsum(g, t0, H, h, L, G, Rref);
    {
        constexpr int PR = 128 * (int)sizeof(Tin) / 16;   // 16-byte pieces per row
        for (int i = tid; i < 64 * PR; i += NT) {
            const int r = i / PR, pc = i % PR;
            const uint4 u = r < L ? *reinterpret_cast<const uint4 *>(k + ((size_t)(t0 + r) * H + h) * D + pc * (16 / sizeof(Tin)))
                                  : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(Kb + r * RC_LDK + pc * (16 / sizeof(Tin))) = u;
        }
    }
    const int tx = tid & 15, ty = tid >> 4;   // output (row 16a + ty, columns tx + 16 b)
    // block a of rows needs columns s <= 16a + 15 only (both forms are lower triangular)
    auto block = [&](auto ac) {
        constexpr int A = decltype(ac)::value, NS = 16 * (A + 1), NB = A + 1;
        __syncthreads();
        // k_s exp(R_a - G_s) for s < NS, row-major like k
        for (int i = tid; i < NS * 32; i += NT) {
            const int s2 = i >> 5, c = (i & 31) * 4;
            const float4 kr = load4_f32(Kb + s2 * RC_LDK + c);
            const float4 g4 = *reinterpret_cast<const float4 *>(G + s2 * LD + c);
            const float4 rf = *reinterpret_cast<const float4 *>(Rref + A * 128 + c);
            *reinterpret_cast<float4 *>(KF + s2 * LD + c) =
                make_float4(kr.x * __expf(rf.x - g4.x), kr.y * __expf(rf.y - g4.y),
                            kr.z * __expf(rf.z - g4.z), kr.w * __expf(rf.w - g4.w));
        }
        // q_r E1_r and k_r E1_r, E1_r = exp(G_r - R_a), for the 16 rows of block a
        for (int i = tid; i < 16 * 32; i += NT) {
            const int r = i >> 5, c = (i & 31) * 4, rr = 16 * A + r;
            const float4 g4 = *reinterpret_cast<const float4 *>(G + rr * LD + c);
            const float4 rf = *reinterpret_cast<const float4 *>(Rref + A * 128 + c);
            const float4 e = make_float4(__expf(g4.x - rf.x), __expf(g4.y - rf.y), __expf(g4.z - rf.z),
                                         __expf(g4.w - rf.w));
            const float4 q4 = rr < L ? load4_f32(q + ((size_t)(t0 + rr) * H + h) * D + c)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 k4 = load4_f32(Kb + rr * RC_LDK + c);
            *reinterpret_cast<float4 *>(QE + r * LD + c) = make_float4(q4.x * e.x, q4.y * e.y, q4.z * e.z, q4.w * e.w);
            *reinterpret_cast<float4 *>(KE + r * LD + c) = make_float4(k4.x * e.x, k4.y * e.y, k4.z * e.z, k4.w * e.w);
        }
        __syncthreads();
        // rows 16a .. 16a + 15 of Aqk (s <= r) and of M (s < r) in one pass over the
        // channels (the two share the decayed k operand); sums over c in order
        float ra_[NB], rm_[NB];
#pragma unroll
        for (int b2 = 0; b2 < NB; ++b2) ra_[b2] = rm_[b2] = 0.f;
        const float *qe = QE + ty * LD, *ke = KE + ty * LD;
#pragma unroll 2
        for (int c = 0; c < 128; c += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(qe + c);
            const float4 y = *reinterpret_cast<const float4 *>(ke + c);
#pragma unroll
            for (int b2 = 0; b2 < NB; ++b2) {
                const float4 kf = *reinterpret_cast<const float4 *>(KF + (tx + 16 * b2) * LD + c);
                ra_[b2] = fmaf(x.w, kf.w, fmaf(x.z, kf.z, fmaf(x.y, kf.y, fmaf(x.x, kf.x, ra_[b2]))));
                rm_[b2] = fmaf(y.w, kf.w, fmaf(y.z, kf.z, fmaf(y.y, kf.y, fmaf(y.x, kf.x, rm_[b2]))));
            }
        }
        const int r = 16 * A + ty;
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) {
            const int s2 = tx + 16 * b2;
            const float va = b2 < NB ? ra_[b2 < NB ? b2 : 0] : 0.f, vm = b2 < NB ? rm_[b2 < NB ? b2 : 0] : 0.f;
            out[IW_AQK + r * 64 + s2] = s2 <= r ? va : 0.f;
            out[IW_M + r * 64 + s2] = s2 < r ? vm : 0.f;
        }
    };
    block(std::integral_constant<int, 0>{});
    block(std::integral_constant<int, 1>{});
    block(std::integral_constant<int, 2>{});
    block(std::integral_constant<int, 3>{});
}

// Shared memory of the pull-back: five 64 x 64 regions (reused as the phases
// free them) and two 64 x 32 channel-quarter tiles, 104 KB: two CTAs per SM.
constexpr int PB_LQ = 36;                                   // fp32 row stride of 32-wide tiles
constexpr uint32_t PB_SMEM = 5 * 64 * L6 * 4 + 2 * 64 * PB_LQ * 4 + 8 * 32 * 4 + 64 * 4;

template <typename Tin>
__global__ void __launch_bounds__(NT, 2)
bwd_pullback_kernel(const uint8_t *__restrict__ fws, const int32_t *__restrict__ cu, int64_t T,
                    int N, int H, const Tin *__restrict__ k, const Tin *__restrict__ g,
                    const Tin *__restrict__ beta, const float *__restrict__ fg,
                    float *__restrict__ iw) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(fws);
    const bool packed = cu != nullptr;
    const int total = packed ? hdr[N] : N * (int)((T + C - 1) / C);
    const int cidx = blockIdx.x / H, h = blockIdx.x % H;
    if (cidx >= total) return;
    int n, j;
    locate_chunk(hdr, packed, T, N, cidx, n, j);
    int64_t ra, rb;
    seq_rows(hdr, packed, T, N, n, ra, rb);
    const int64_t t0 = ra + (int64_t)j * C;
    const int L = (int)((rb - t0) < C ? (rb - t0) : C);
    const size_t item = (size_t)cidx * H + h;
    float *io = iw + item * IW_FLOATS;
    const float *fgi = fg + item * FG_FLOATS;
    // regions [64][L6]: 0 Aqk, then dR'; 1 M, then dT'; 2 X; 3 R, then Aqk again;
    // 4 the X scratch, then K*Gamma of a channel quarter, then Wk
    float *Rg0 = reinterpret_cast<float *>(sm);
    float *Rg1 = Rg0 + 64 * L6, *Rg2 = Rg1 + 64 * L6, *Rg3 = Rg2 + 64 * L6, *Rg4 = Rg3 + 64 * L6;
    float *dPq = Rg4 + 64 * L6;                            // dP, dW of a channel quarter [64][PB_LQ]
    float *dWq = dPq + 64 * PB_LQ;
    float *gsum = dWq + 64 * PB_LQ;                        // [8][32] row-group sums of the quarter's g
    float *bs = gsum + 8 * 32;                             // beta [64]
    float *Aq = Rg0, *Mm = Rg1, *X = Rg2, *Rm = Rg3, *Wk = Rg4;
    // ---- phase 1: X = (I + Diag(beta) M)^-1, R = Aqk T
    for (int i = tid; i < 64 * 16; i += NT) {
        const int r = i >> 4, s = (i & 15) * 4;
        *reinterpret_cast<float4 *>(Aq + r * L6 + s) = *reinterpret_cast<const float4 *>(io + IW_AQK + r * 64 + s);
        *reinterpret_cast<float4 *>(Mm + r * L6 + s) = *reinterpret_cast<const float4 *>(io + IW_M + r * 64 + s);
        *reinterpret_cast<float4 *>(X + r * L6 + s) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < 64) bs[tid] = tid < L ? to_f32(beta[(size_t)(t0 + tid) * H + h]) : 0.f;
    __syncthreads();
    // X = (I + A)^-1, A = Diag(beta) M (strictly lower), by 16 x 16 blocks: the
    // diagonal blocks by forward substitution (thread = block a, column j), then
    // block row i from the rows above: X[i, 0:i] = -X_ii (A[i, 0:i] X[0:i, 0:i])
    if (tid < 64) {
        const int a = tid >> 4, jc = tid & 15, o = 16 * a;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = r == jc ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) acc = fmaf(-bs[o + r] * Mm[(o + r) * L6 + o + m], x[m], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) X[(o + r) * L6 + o + jc] = x[r];
    }
    __syncthreads();
    auto block_row = [&](auto ic) {
        constexpr int I = decltype(ic)::value, W = 16 * I;
        // Wk[r][m] = sum_{p < W} A[16I + r][p] X[p][m]
        smm<16, W, W>([&](int r, int p) { return bs[16 * I + r] * Mm[(16 * I + r) * L6 + p]; },
                      [&](int p, int m) { return X[p * L6 + m]; },
                      [&](int r, int m, float v) { Wk[r * L6 + m] = v; });
        __syncthreads();
        smm<16, W, 16>([&](int r, int p) { return X[(16 * I + r) * L6 + 16 * I + p]; },
                       [&](int p, int m) { return Wk[p * L6 + m]; },
                       [&](int r, int m, float v) { X[(16 * I + r) * L6 + m] = -v; });
        __syncthreads();
    };
    block_row(std::integral_constant<int, 1>{});
    block_row(std::integral_constant<int, 2>{});
    block_row(std::integral_constant<int, 3>{});
    // The lower-triangular factors (Aqk, X, T, R) make most of the sums below
    // run over a band of k: a warp's rows 8w .. 8w + 7 need k <= 8w + 7 or k >= 8w.
    auto k_upto = [](int w, int &lo, int &hi) { lo = 0; hi = 8 * w + 8; };
    auto k_from = [](int w, int &lo, int &hi) { lo = 8 * w; hi = 64; };
    // R = Aqk T, T = X Diag(beta): R[r][s] sums m in [s, r]
    smm_rows<64>([&](int r, int m) { return Aq[r * L6 + m]; }, [&](int m, int s) { return X[m * L6 + s] * bs[s]; },
                 k_upto, [&](int r, int s, float x) { Rm[r * L6 + s] = x; });
    __syncthreads();   // Aqk and M are consumed (Aqk comes back in phase 3, M from the workspace)

    // ---- phase 2, by quarters of 32 channels: K*Gamma, dR' = dR - dP (K Gamma)^T,
    // dT'_0 = dT + dW (K Gamma)^T (both summed over the quarters in order), and
    // dKt = T^T dW - R^T dP -> workspace (sums t >= s)
    float *dRp = Rg0, *dTp = Rg1, *Ktq = Rg4;   // Ktq: [64][PB_LQ]
    for (int i = tid; i < 64 * 16; i += NT) {
        const int r = i >> 4, s = (i & 15) * 4;
        *reinterpret_cast<float4 *>(dRp + r * L6 + s) = *reinterpret_cast<const float4 *>(fgi + FG_DR + r * 64 + s);
        *reinterpret_cast<float4 *>(dTp + r * L6 + s) = *reinterpret_cast<const float4 *>(fgi + FG_DT + r * 64 + s);
    }
    for (int qd = 0; qd < 4; ++qd) {
        const int cb = 32 * qd;
        __syncthreads();   // the previous quarter's products are done with its tiles
        // the quarter's dP, dW, g (clamped; 0 past the chunk's end) and k
        float4 kq[2];
        for (int i = tid, it = 0; i < 64 * 8; i += NT, ++it) {
            const int r = i >> 3, c = (i & 7) * 4;
            *reinterpret_cast<float4 *>(dPq + r * PB_LQ + c) = *reinterpret_cast<const float4 *>(fgi + FG_DP + r * 128 + cb + c);
            *reinterpret_cast<float4 *>(dWq + r * PB_LQ + c) = *reinterpret_cast<const float4 *>(fgi + FG_DW + r * 128 + cb + c);
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
            if (r < L) {
                const size_t off = ((size_t)(t0 + r) * H + h) * D + cb + c;
                x = load4_f32(g + off);
                x = make_float4(fmaxf(x.x, -5.f), fmaxf(x.y, -5.f), fmaxf(x.z, -5.f), fmaxf(x.w, -5.f));
                y = load4_f32(k + off);
            }
            *reinterpret_cast<float4 *>(Ktq + r * PB_LQ + c) = x;
            kq[it] = y;
        }
        __syncthreads();
        // Gamma = exp(cumsum over rows): thread (group gr of 8 rows, channel cc) sums
        // its rows, the group offsets come from the groups above
        {
            const int cc = tid & 31, gr = tid >> 5;
            float run = 0.f, loc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                run += Ktq[(8 * gr + e) * PB_LQ + cc];
                loc[e] = run;
            }
            gsum[gr * 32 + cc] = run;
            __syncthreads();
            float off = 0.f;
            for (int g2 = 0; g2 < gr; ++g2) off += gsum[g2 * 32 + cc];
#pragma unroll
            for (int e = 0; e < 8; ++e) Ktq[(8 * gr + e) * PB_LQ + cc] = __expf(off + loc[e]);
        }
        __syncthreads();
        for (int i = tid, it = 0; i < 64 * 8; i += NT, ++it) {   // K * Gamma (the same rows as the load)
            const int r = i >> 3, c = (i & 7) * 4;
            float4 *p4 = reinterpret_cast<float4 *>(Ktq + r * PB_LQ + c);
            const float4 e = *p4;
            *p4 = make_float4(kq[it].x * e.x, kq[it].y * e.y, kq[it].z * e.z, kq[it].w * e.w);
        }
        __syncthreads();
        // (the blocks above the diagonal of dR' and dT' reach no output: they stay 0)
        smm_nt<64, 64, 32, true>(dPq, PB_LQ, Ktq, PB_LQ, [&](int t, int s, float x) { dRp[t * L6 + s] -= x; });
        smm_nt<64, 64, 32, true>(dWq, PB_LQ, Ktq, PB_LQ, [&](int t, int s, float x) { dTp[t * L6 + s] += x; });
        smm_rows2<32>([&](int s, int t) { return X[t * L6 + s] * bs[s]; }, [&](int t, int c) { return dWq[t * PB_LQ + c]; },
                      [&](int s, int t) { return -Rm[t * L6 + s]; }, [&](int t, int c) { return dPq[t * PB_LQ + c]; },
                      [](int w, int &lo1, int &hi1, int &lo2, int &hi2) { lo1 = lo2 = 8 * w; hi1 = hi2 = 64; },
                      [&](int s, int c, float x) { io[IW_DKT + s * 128 + cb + c] = x; });
    }
    __syncthreads();   // R is consumed: its region takes Aqk again

    // ---- phase 3
    Aq = Rg3;
    for (int i = tid; i < 64 * 16; i += NT) {
        const int r = i >> 4, s = (i & 15) * 4;
        *reinterpret_cast<float4 *>(Aq + r * L6 + s) = *reinterpret_cast<const float4 *>(io + IW_AQK + r * 64 + s);
    }
    __syncthreads();
    // dT' += Aqk^T dR' (sums m >= r)
    smm_rows<64>([&](int r, int m) { return Aq[m * L6 + r]; }, [&](int m, int s) { return dRp[m * L6 + s]; },
                 k_from, [&](int r, int s, float x) { dTp[r * L6 + s] += x; });
    // dAqk = tril(dR' T^T) -> workspace, as its transpose: dAqk[r][s] = sum_{m <= s}
    // T[s][m] dR'[r][m], rows s
    smm_rows<64>([&](int s2, int m) { return X[s2 * L6 + m] * bs[m]; }, [&](int m, int r) { return dRp[r * L6 + m]; },
                 k_upto, [&](int s2, int r, float x) { io[IW_DAQK + r * 64 + s2] = s2 <= r ? x : 0.f; });
    __syncthreads();
    // Wk = X^T (dT' Diag(beta)) (sums m >= r)
    smm_rows<64>([&](int r, int m) { return X[m * L6 + r]; }, [&](int m, int s) { return dTp[m * L6 + s] * bs[s]; },
                 k_from, [&](int r, int s, float x) { Wk[r * L6 + s] = x; });
    __syncthreads();
    // dAkk = strict_tril(-Wk X^T), dM = Diag(beta) dAkk -> workspace, as the
    // transpose: dAkk[r][s] = -sum_{m <= s} X[s][m] Wk[r][m], rows s (into dR''s region)
    float *dAkk = Rg0;
    smm_rows<64>([&](int s2, int m) { return X[s2 * L6 + m]; }, [&](int m, int r) { return Wk[r * L6 + m]; },
                 k_upto,
                 [&](int s2, int r, float x) {
                     const float d = s2 < r ? -x : 0.f;
                     dAkk[r * L6 + s2] = d;
                     io[IW_DM + r * 64 + s2] = bs[r] * d;
                 });
    __syncthreads();
    // dbeta_s = sum_r X[r,s] dT'[r,s] + sum_t dAkk[s,t] M[s,t]
    if (tid < 64) {
        float a = 0.f, b = 0.f;
        for (int r = 0; r < 64; ++r) {
            a = fmaf(X[r * L6 + tid], dTp[r * L6 + tid], a);
            b = fmaf(dAkk[tid * L6 + r], io[IW_M + tid * 64 + r], b);
        }
        io[IW_DB + tid] = a + b;
    }
}

// One CTA per (chunk, head, 32-channel slice): every step below is independent
// per key channel except the 64 x 64 adjoint tiles dAqk and dM, which each slice
// reads whole.  Slices keep the shared memory at 75 KB, so that three CTAs share
// an SM.
constexpr int AS_CW = 32;                 // channels per CTA
constexpr int AS_LS = AS_CW + 4;          // fp32 row stride
constexpr uint32_t AS_SMEM = (6 * 64 * AS_LS + 16 * AS_LS + 64 * L6 + 4 * AS_CW + 64) * 4;

template <typename Tin>
__global__ void __launch_bounds__(NT, 3)
bwd_assemble_kernel(const uint8_t *__restrict__ fws, const int32_t *__restrict__ cu, int64_t T,
                    int N, int H, const Tin *__restrict__ q, const Tin *__restrict__ k,
                    const Tin *__restrict__ g, const float *__restrict__ fg,
                    const float *__restrict__ iw, float *__restrict__ dq, float *__restrict__ dk,
                    float *__restrict__ dg, float *__restrict__ dbeta) {
    extern __shared__ __align__(16) uint8_t sm[];
    constexpr int CW = AS_CW, LS = AS_LS, NSL = D / CW;
    const int tid = threadIdx.x;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(fws);
    const bool packed = cu != nullptr;
    const int total = packed ? hdr[N] : N * (int)((T + C - 1) / C);
    const int slice = blockIdx.x % NSL, itm = blockIdx.x / NSL;
    const int cidx = itm / H, h = itm % H;
    if (cidx >= total) return;
    const int cb = slice * CW;   // first channel of the slice
    int n, j;
    locate_chunk(hdr, packed, T, N, cidx, n, j);
    int64_t ra, rb;
    seq_rows(hdr, packed, T, N, n, ra, rb);
    const int64_t t0 = ra + (int64_t)j * C;
    const int L = (int)((rb - t0) < C ? (rb - t0) : C);
    const size_t item = (size_t)cidx * H + h;
    const float *io = iw + item * IW_FLOATS;
    const float *fgi = fg + item * FG_FLOATS;
    float *G = reinterpret_cast<float *>(sm);             // [64][LS] chunk-local cumsum
    float *KK = G + 64 * LS;                               // k_s exp(R_a - G_s), block a's
    float *dG = KK + 64 * LS;                              // dG accumulator
    float *Dq = dG + 64 * LS;                              // dq accumulator
    float *Dk = Dq + 64 * LS;                              // dk accumulator
    float *Ks = Dk + 64 * LS;                              // k (0 past the chunk's end)
    float *AE = Ks + 64 * LS;                              // a_r E1_r for the 16 rows of block a
    float *dFs = AE + 16 * LS;                             // dAqk, then dM  [64][L6]
    float *Rref = dFs + 64 * L6;                           // [4][CW]
    uint32_t *below = reinterpret_cast<uint32_t *>(Rref + 4 * CW);   // [64]: bit cc set where g < -5
    // chunk-local cumsum of this slice's channels and the 16-row references: the
    // rows load in parallel (clamped, with the rows below the clamp flagged for
    // dg), then one thread per channel scans them in shared memory
    if (tid < 64) below[tid] = 0u;
    __syncthreads();
    for (int i = tid; i < 64 * (CW / 4); i += NT) {   // 4 channels per load
        const int r = i / (CW / 4), cc = (i % (CW / 4)) * 4;
        const size_t off = ((size_t)(t0 + r) * H + h) * D + cb + cc;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
        if (r < L) {
            x = load4_f32(g + off);
            y = load4_f32(k + off);
            const uint32_t m = (!(x.x >= -5.f) ? 1u : 0u) | (!(x.y >= -5.f) ? 2u : 0u) |
                               (!(x.z >= -5.f) ? 4u : 0u) | (!(x.w >= -5.f) ? 8u : 0u);
            if (m) atomicOr(&below[r], m << cc);
            x = make_float4(fmaxf(x.x, -5.f), fmaxf(x.y, -5.f), fmaxf(x.z, -5.f), fmaxf(x.w, -5.f));
        }
        *reinterpret_cast<float4 *>(G + r * LS + cc) = x;
        *reinterpret_cast<float4 *>(Ks + r * LS + cc) = y;
    }
    __syncthreads();
    if (tid < CW) {
        float acc = 0.f;
        for (int r = 0; r < 64; ++r) {
            acc += G[r * LS + tid];
            G[r * LS + tid] = acc;
            if ((r & 15) == 15 && r < 63) Rref[((r + 1) >> 4) * CW + tid] = acc;
        }
        Rref[tid] = 0.f;
    }
    __syncthreads();
    auto qv = [&](int r, int cc) {
        return r < L ? to_f32(q[((size_t)(t0 + r) * H + h) * D + cb + cc]) : 0.f;
    };
    auto kv = [&](int r, int cc) { return Ks[r * LS + cc]; };
    const float *gl = G + 63 * LS;   // G at the last row = G_L (rows past L add nothing)
    // the elementwise terms
    for (int i = tid; i < 64 * (CW / 4); i += NT) {   // 4 channels per load
        const int r = i / (CW / 4), cc0 = (i % (CW / 4)) * 4, c0 = cb + cc0;
        const float4 q4 = r < L ? load4_f32(q + ((size_t)(t0 + r) * H + h) * D + c0)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 dP4 = *reinterpret_cast<const float4 *>(fgi + FG_DP + r * 128 + c0);
        const float4 dKt4 = *reinterpret_cast<const float4 *>(io + IW_DKT + r * 128 + c0);
        const float4 dKh4 = *reinterpret_cast<const float4 *>(fgi + FG_DKH + r * 128 + c0);
        const float qa[4] = {q4.x, q4.y, q4.z, q4.w}, dPa[4] = {dP4.x, dP4.y, dP4.z, dP4.w};
        const float dKta[4] = {dKt4.x, dKt4.y, dKt4.z, dKt4.w}, dKha[4] = {dKh4.x, dKh4.y, dKh4.z, dKh4.w};
        // shared-memory rows by 16-byte pieces (a quarter-warp covers one row)
        const float4 G4 = *reinterpret_cast<const float4 *>(G + r * LS + cc0);
        const float4 gl4 = *reinterpret_cast<const float4 *>(gl + cc0);
        const float4 k4 = *reinterpret_cast<const float4 *>(Ks + r * LS + cc0);
        const float Ga[4] = {G4.x, G4.y, G4.z, G4.w}, gla[4] = {gl4.x, gl4.y, gl4.z, gl4.w};
        const float ka[4] = {k4.x, k4.y, k4.z, k4.w};
        float dq4[4], dk4[4], dg4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float gam = __expf(Ga[e]), kh_f = __expf(gla[e] - Ga[e]);
            dq4[e] = dPa[e] * gam;
            dk4[e] = dKta[e] * gam + dKha[e] * kh_f;
            dg4[e] = qa[e] * gam * dPa[e] + ka[e] * gam * dKta[e] - ka[e] * kh_f * dKha[e];
        }
        *reinterpret_cast<float4 *>(Dq + r * LS + cc0) = make_float4(dq4[0], dq4[1], dq4[2], dq4[3]);
        *reinterpret_cast<float4 *>(Dk + r * LS + cc0) = make_float4(dk4[0], dk4[1], dk4[2], dk4[3]);
        *reinterpret_cast<float4 *>(dG + r * LS + cc0) = make_float4(dg4[0], dg4[1], dg4[2], dg4[3]);
    }
    // decayed adjoints: first Aqk with (a, b) = (q, k), then M with (k, k).  dF is
    // lower triangular, so block a's sums run over s <= 16a + 15 only.
    const int warp = tid >> 5, lane = tid & 31;
    auto block = [&](auto ac, int form) {
        constexpr int A = decltype(ac)::value, NS = 16 * (A + 1), KQ = NS / 4;
        const float *dF = dFs;
        __syncthreads();   // the previous block's products are done with KK and AE
        for (int i = tid; i < NS * CW; i += NT) {
            const int s = i / CW, cc = i % CW;
            KK[s * LS + cc] = Ks[s * LS + cc] * __expf(Rref[A * CW + cc] - G[s * LS + cc]);
        }
        for (int i = tid; i < 16 * CW; i += NT) {
            const int r = i / CW, cc = i % CW, rr = 16 * A + r;
            AE[r * LS + cc] = (form == 0 ? qv(rr, cc) : kv(rr, cc)) * __expf(G[rr * LS + cc] - Rref[A * CW + cc]);
        }
        __syncthreads();
        // da_r (rows of block a) = E1_r sum_s dF[r,s] k_s exp(R_a - G_s): warp w takes
        // rows 16a + 2w, 16a + 2w + 1; lane = 8 kq + cq sums s in the kq-th quarter of
        // [0, NS) for columns 4 cq .. 4 cq + 3, then the quarters are added across lanes
        {
            float acc[2][4];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
            const int kq = lane >> 3, cq = lane & 7;
            const float *d0 = dF + (16 * A + 2 * warp) * L6;
#pragma unroll 4
            for (int s2 = kq * KQ; s2 < kq * KQ + KQ; ++s2) {
                const float x0 = d0[s2], x1 = d0[L6 + s2];
                const float4 b = *reinterpret_cast<const float4 *>(KK + s2 * LS + 4 * cq);
                acc[0][0] = fmaf(x0, b.x, acc[0][0]); acc[0][1] = fmaf(x0, b.y, acc[0][1]);
                acc[0][2] = fmaf(x0, b.z, acc[0][2]); acc[0][3] = fmaf(x0, b.w, acc[0][3]);
                acc[1][0] = fmaf(x1, b.x, acc[1][0]); acc[1][1] = fmaf(x1, b.y, acc[1][1]);
                acc[1][2] = fmaf(x1, b.z, acc[1][2]); acc[1][3] = fmaf(x1, b.w, acc[1][3]);
            }
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    acc[x][y] += __shfl_xor_sync(0xffffffffu, acc[x][y], 8);
                    acc[x][y] += __shfl_xor_sync(0xffffffffu, acc[x][y], 16);
                }
            // every lane of a quarter group holds the sums; lane kq finishes row
            // 2w + (kq >> 1), columns 4 cq + 2 (kq & 1) + e (the second row takes its
            // two columns in the other order, so that the rows fall on different banks)
            const int rsel = kq >> 1, csel = kq & 1, rr = 16 * A + 2 * warp + rsel;
#pragma unroll
            for (int e0 = 0; e0 < 2; ++e0) {
                const int e = rsel ? 1 - e0 : e0;
                const float x = rsel ? (csel ? (e ? acc[1][3] : acc[1][2]) : (e ? acc[1][1] : acc[1][0]))
                                     : (csel ? (e ? acc[0][3] : acc[0][2]) : (e ? acc[0][1] : acc[0][0]));
                const int cc = 4 * cq + 2 * csel + e;
                const float da = x * __expf(G[rr * LS + cc] - Rref[A * CW + cc]);
                if (form == 0) Dq[rr * LS + cc] += da; else Dk[rr * LS + cc] += da;
                dG[rr * LS + cc] += x * AE[(rr - 16 * A) * LS + cc];   // a_r da_r = x a_r E1_r
            }
        }
        __syncthreads();   // block a's rows of Dk and dG take db next
        // db_s += exp(R_a - G_s) sum_{r in a} dF[r,s] a_r E1_r, for s < NS: thread
        // (rg = tid / 8, cq = tid % 8) takes rows rg and rg + 32 (those below NS) and
        // columns 4 cq .. 4 cq + 3, read as 16-byte pieces
        {
            constexpr int NR = NS > 32 ? 2 : 1;
            const int rg = tid >> 3, cq = tid & 7;
            if (rg < NS) {
                const bool two = NR == 2 && rg + 32 < NS;
                float acc[NR][4];
#pragma unroll
                for (int x = 0; x < NR; ++x)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[x][e] = 0.f;
#pragma unroll 4
                for (int r = 0; r < 16; ++r) {
                    const float4 b4 = *reinterpret_cast<const float4 *>(AE + r * LS + 4 * cq);
#pragma unroll
                    for (int x = 0; x < NR; ++x) {
                        const float av = (x == 0 || two) ? dF[(16 * A + r) * L6 + rg + 32 * x] : 0.f;
                        acc[x][0] = fmaf(av, b4.x, acc[x][0]); acc[x][1] = fmaf(av, b4.y, acc[x][1]);
                        acc[x][2] = fmaf(av, b4.z, acc[x][2]); acc[x][3] = fmaf(av, b4.w, acc[x][3]);
                    }
                }
#pragma unroll
                for (int x = 0; x < NR; ++x) {
                    if (x == 1 && !two) break;
                    const int s2 = rg + 32 * x, o = s2 * LS + 4 * cq;
                    const float4 g4 = *reinterpret_cast<const float4 *>(G + o);
                    const float4 rf = *reinterpret_cast<const float4 *>(Rref + A * CW + 4 * cq);
                    const float4 k4 = *reinterpret_cast<const float4 *>(Ks + o);
                    float4 dk4 = *reinterpret_cast<const float4 *>(Dk + o);
                    float4 dg4 = *reinterpret_cast<const float4 *>(dG + o);
                    const float d0 = acc[x][0] * __expf(rf.x - g4.x), d1 = acc[x][1] * __expf(rf.y - g4.y);
                    const float d2 = acc[x][2] * __expf(rf.z - g4.z), d3 = acc[x][3] * __expf(rf.w - g4.w);
                    dk4.x += d0; dk4.y += d1; dk4.z += d2; dk4.w += d3;
                    dg4.x -= k4.x * d0; dg4.y -= k4.y * d1; dg4.z -= k4.z * d2; dg4.w -= k4.w * d3;
                    *reinterpret_cast<float4 *>(Dk + o) = dk4;
                    *reinterpret_cast<float4 *>(dG + o) = dg4;
                }
            }
        }
    };
    for (int form = 0; form < 2; ++form) {
        __syncthreads();   // the previous form's products are done with dFs
        for (int i = tid; i < 64 * 16; i += NT)
            *reinterpret_cast<float4 *>(dFs + (i >> 4) * L6 + (i & 15) * 4) =
                *reinterpret_cast<const float4 *>(io + (form == 0 ? IW_DAQK : IW_DM) + i * 4);
        block(std::integral_constant<int, 0>{}, form);
        block(std::integral_constant<int, 1>{}, form);
        block(std::integral_constant<int, 2>{}, form);
        block(std::integral_constant<int, 3>{}, form);
    }
    __syncthreads();
    // row L-1 also carries G_L's gradient: sum_r Khat dKhat + Gamma_L dGamma_L (the
    // sum by 8-row groups over all threads, into KK, which is free now); then dg =
    // reverse cumsum of dG, 0 where g < -5
    {
        const int cc = tid % CW, rg = tid / CW;   // NT / CW = 8 groups of 8 rows
        float part = 0.f;
#pragma unroll
        for (int r = 8 * rg; r < 8 * rg + 8; ++r)
            if (r < L)
                part = fmaf(kv(r, cc) * __expf(gl[cc] - G[r * LS + cc]), fgi[FG_DKH + r * 128 + cb + cc], part);
        KK[rg * LS + cc] = part;
    }
    __syncthreads();
    if (tid < CW && L > 0) {
        const int cc = tid, c = cb + tid;
        float s_kh = 0.f;
        for (int rg = 0; rg < NT / CW; ++rg) s_kh += KK[rg * LS + cc];
        dG[(L - 1) * LS + cc] += s_kh + __expf(gl[cc]) * fgi[FG_DGL + c];
        float acc = 0.f;
        for (int r = L - 1; r >= 0; --r) {
            acc += dG[r * LS + cc];
            dg[((size_t)(t0 + r) * H + h) * D + c] = (below[r] >> cc) & 1u ? 0.f : acc;
        }
    }
    for (int i = tid; i < 64 * CW; i += NT) {
        const int r = i / CW, cc = i % CW;
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + cb + cc;
            dq[off] = Dq[r * LS + cc];
            dk[off] = Dk[r * LS + cc];
        }
    }
    if (slice == 0 && tid < L) dbeta[(size_t)(t0 + tid) * H + h] = io[IW_DB + tid];
}

}  // namespace cbw

// ======================================================================
// host side
// ======================================================================
namespace {
struct CwLayout {
    int64_t max_chunks;
    size_t fws, o, snaps, sout, dS, dU, fg, iw, total;
};
size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
CwLayout cw_layout(int64_t rows, int N, int H) {
    CwLayout L;
    L.max_chunks = (rows + cbw::C - 1) / cbw::C + N;
    const size_t mch = (size_t)L.max_chunks * H, dd = (size_t)cbw::D * cbw::D;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off += al256(bytes); return o; };
    L.fws = take(prefill_tc_workspace_bytes(rows, N, H, cbw::D));
    L.o = take((size_t)rows * H * cbw::D * 4);
    L.snaps = take(mch * dd * 4);
    L.sout = take((size_t)N * H * dd * 4);
    L.dS = take(mch * dd * 4);
    L.dU = take(mch * 64 * cbw::D * 4);
    L.fg = take(mch * cbw::FG_FLOATS * 4);
    L.iw = take(mch * cbw::IW_FLOATS * 4);
    L.total = off;
    return L;
}
template <typename K>
cudaError_t set_smem(K kern, uint32_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}
}  // namespace

size_t backward_chunked_workspace_bytes(int64_t rows, int N, int H) {
    return cw_layout(rows, N, H).total;
}

cudaError_t launch_backward_chunked(const BackwardArgs &a, cudaStream_t st) {
    using namespace cbw;
    using bf = __nv_bfloat16;
    const CwLayout L = cw_layout(a.rows, a.N, a.H);
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    uint8_t *fws = ws + L.fws;
    float *snaps = reinterpret_cast<float *>(ws + L.snaps);
    // 1. the forward in its chunked form, with a snapshot at every chunk start
    PrefillArgs f{};
    f.q = a.q; f.k = a.k; f.v = a.v; f.g = a.g; f.beta = a.beta;
    f.state_in = a.state_in;
    f.cu_seqlens = a.cu_seqlens;
    f.B = a.cu_seqlens ? 1 : (a.T > 0 ? (int)(a.rows / a.T) : a.N);
    f.T = a.T;
    f.N = a.N; f.H = a.H; f.dk = D; f.dv = D;
    f.o = ws + L.o;
    f.state_out = reinterpret_cast<float *>(ws + L.sout);
    f.workspace = fws;
    f.workspace_bytes = prefill_tc_workspace_bytes(a.rows, a.N, a.H, D);
    f.err = a.err;
    f.ckpt_interval = C;
    f.ckpt = snaps;
    f.ckpt_capacity = L.max_chunks;
    f.epoch = a.epoch;
    cudaError_t e = launch_prefill_tc(f, st);
    if (e != cudaSuccess) return e;
    const uint32_t hb = (uint32_t)(((size_t)(a.N + 1) * 16 + 1023) & ~(size_t)1023);
    float *dS = reinterpret_cast<float *>(ws + L.dS), *dU = reinterpret_cast<float *>(ws + L.dU);
    float *fg = reinterpret_cast<float *>(ws + L.fg), *iw = reinterpret_cast<float *>(ws + L.iw);
    // 2. the chain, chunks in reverse
    if ((e = set_smem(bwd_chain_kernel, CH_SMEM)) != cudaSuccess) return e;
    bwd_chain_kernel<<<(unsigned)(a.N * a.H * (D / CH_DVS)), NT, CH_SMEM, st>>>(
        fws, a.cu_seqlens, a.T, a.N, a.H, a.dout, a.dstate_out, dS, dU, a.dstate_in, hb, a.err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    Profiler::mark(st);
    // 3.-6. per chunk: factor gradients (and dv), recompute, pull-back, assembly
    const unsigned items = (unsigned)(L.max_chunks * a.H);
    if ((e = set_smem(bwd_factor_kernel<bf>, F_SMEM)) != cudaSuccess) return e;
    bwd_factor_kernel<bf><<<items, FNT, F_SMEM, st>>>(fws, a.cu_seqlens, a.T, a.N, a.H, (const bf *)a.v,
                                                     a.state_in, snaps, a.dout, dS, dU, fg, a.dv, hb, a.err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    Profiler::mark(st);
    // G, KF, QE and KE of one row block, Rref, k (bf16): two CTAs per SM
    constexpr uint32_t RC_SMEM = (2 * 64 + 2 * 16) * LD * 4 + 4 * 128 * 4 + 64 * RC_LDK * 2;
    static_assert(2 * (RC_SMEM + 1024) <= 228 * 1024, "recompute: two CTAs per SM");
    if ((e = set_smem(bwd_recompute_kernel<bf>, RC_SMEM)) != cudaSuccess) return e;
    bwd_recompute_kernel<bf><<<items, NT, RC_SMEM, st>>>(fws, a.cu_seqlens, a.T, a.N, a.H, (const bf *)a.q,
                                                         (const bf *)a.k, (const bf *)a.g, iw);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    Profiler::mark(st);
    static_assert(2 * (PB_SMEM + 1024) <= 228 * 1024, "pull-back: two CTAs per SM");
    if ((e = set_smem(bwd_pullback_kernel<bf>, PB_SMEM)) != cudaSuccess) return e;
    bwd_pullback_kernel<bf><<<items, NT, PB_SMEM, st>>>(fws, a.cu_seqlens, a.T, a.N, a.H, (const bf *)a.k,
                                                        (const bf *)a.g, (const bf *)a.beta, fg, iw);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    Profiler::mark(st);
    static_assert(3 * (cbw::AS_SMEM + 1024) <= 228 * 1024, "assembly: three CTAs per SM");
    if ((e = set_smem(bwd_assemble_kernel<bf>, cbw::AS_SMEM)) != cudaSuccess) return e;
    bwd_assemble_kernel<bf><<<items * (cbw::D / cbw::AS_CW), NT, cbw::AS_SMEM, st>>>(fws, a.cu_seqlens, a.T, a.N, a.H, (const bf *)a.q,
                                                        (const bf *)a.k, (const bf *)a.g, fg, iw, a.dq,
                                                        a.dk, a.dg, a.dbeta);
    e = cudaGetLastError();
    Profiler::mark(st);
    return e;
}

}  // namespace kda
