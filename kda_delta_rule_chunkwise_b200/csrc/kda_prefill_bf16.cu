// KDA chunked prefill, bf16 path: tcgen05 (TMEM) tensor-core kernels for sm_100a.
//
// The recurrence S_t = (I - beta k k^T) Diag(exp g) S_{t-1} + beta k v^T,
// o_t = S_t^T q_t (the delta rule with per-channel retention of neurohive.io
// "Kimi K3 ... overview", section "Sequence length: hybrid KDA and Gated MLA
// attention") is evaluated in chunks of C = 64 tokens in two kernels:
//
// Phase A, intra_chunk_kernel (one CTA per (chunk, head), all in parallel):
//   G     chunk-local inclusive cumsum of max(g, -5)                     (fp32)
//   Akk, Aqk  decay-rescaled intra-chunk products on tensor cores.  The
//         pairwise decay exp(G_r - G_s) is split as
//         exp(G_r - R_a) * exp(R_a - G_s), R_a = G at the end of the
//         previous 16-row block a.  Both factors stay inside the bf16
//         exponent range because g >= -5: the first is in [e^-80, 1], the
//         second <= e^75.  That bound is what lets every tile (diagonal ones
//         included) run as a dense bf16 MMA; it is the point of the lower
//         bound on the log-decay in the section cited above.
//   T     = (I + Akk)^-1 Diag(beta): blocked unit-lower-triangular inverse,
//         fp32 (the UT/WY step that turns the sequential delta rule into
//         matrix products)
//   R     = Aqk T;   W = T (K * exp(G));   P = Q * exp(G) - R (K * exp(G))
//   Khat  = K * exp(G_L - G),  Gamma_L = exp(G_L)
//   These are written to a per-(chunk, head) workspace slot, already in the
//   shared-memory layouts the state pass feeds to its MMAs.
//
// Phase B, state_pass_kernel (one CTA per (sequence, head, dv-slice),
// sequential over that sequence's chunks; the fp32 state lives in TMEM):
//   [U; O] = [T; R] V + [-W; P] S        (one accumulator, 128 rows)
//   S     <- Diag(Gamma_L) S + Khat^T U
// With U = T V - W S this is the WY form: U are the chunk's pseudo-values and
// O = Q*exp(G) S + Aqk U, the chunk's outputs.
//
// Roles in phase B: warp 0 = producer (1-D bulk copy of the slot, V slice
// converted to fp16), warp 1 = MMA issuer and TMEM owner, warps 4-7 = U/O
// epilogue (TMEM -> registers), warps 8-11 = state epilogue (Gamma scaling
// of the TMEM state, fp16 copy of S for the next chunk's MMA).
//
// Precision.  Inputs are bf16; every product accumulates in fp32 (TMEM); the
// state and the outputs o are fp32.  The decay-rescaled operands of Akk/Aqk
// need the fp32 exponent range (factors down to e^-80 and up to e^75), so
// those MMAs run in tf32.  Every other stored operand is O(1) in magnitude
// and is kept in fp16, whose 11-bit significand is what the error bound
// max|do|/rms(o) <= 2e-2 needs on heavy-tailed outputs (8-bit bf16
// intermediates alone cost about 3e-2 there).  The fp16 operands assume
// |v| and |state| stay below 65504.
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int C = 64;      // chunk length
constexpr int D = 128;     // dk = dv on this path

// ---- workspace slot (one per (chunk, head)), offsets in bytes
constexpr uint32_t kSlotWP = 0;          // [-W; P]: 128 rows x 128 bf16, K-major SW128, 2 K-blocks
constexpr uint32_t kSlotTR = 32768;      // [T; R] : 128 rows x 64 bf16, K-major SW128
constexpr uint32_t kSlotKh = 49152;      // Khat   : MN-major SW128 (M = channel, K = token)
constexpr uint32_t kSlotGam = 65536;     // Gamma_L: 128 fp32
constexpr uint32_t kSlotBytes = 66560;   // 65 KiB, keeps every slot 1024-aligned
constexpr uint32_t kWPKBlock = 16384;    // bytes between the two 64-column K-blocks of [-W;P]
constexpr uint32_t kKhMNBlock = 8192;    // bytes between the two 64-channel MN-blocks of Khat

// Workspace header: int32 chunk_off[N+1] (first chunk of each sequence, total
// in chunk_off[N]) followed by int32 bound[N+1] (the row offsets actually used:
// cu_seqlens clamped to [0, T] and made non-decreasing by a running maximum,
// so that sequences never overlap and the chunk total never exceeds the
// workspace bound).  Then the slots, 1024-aligned.
__host__ __device__ inline uint32_t header_bytes(int N) {
    return (uint32_t)(((size_t)(N + 1) * 8 + 1023) & ~(size_t)1023);
}

// ======================================================================
// chunk table (one block of 1024 threads)
// ======================================================================
__global__ void __launch_bounds__(1024)
chunk_table_kernel(const int32_t *__restrict__ cu, int64_t T, int N, int32_t *__restrict__ hdr) {
    __shared__ int64_t part[1024];
    int32_t *chunk_off = hdr;
    int32_t *bound = hdr + (N + 1);
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (N + 1 + nt - 1) / nt;             // offsets 0..N, contiguous per thread
    const int i0 = tid * per, i1 = min(N + 1, i0 + per);
    auto clampT = [&](int64_t x) -> int64_t { return x < 0 ? 0 : (x > T ? T : x); };
    if (cu) {
        // running maximum of the clamped offsets
        int64_t m = 0;
        for (int i = i0; i < i1; ++i) m = max(m, clampT(cu[i]));
        part[tid] = m;
        __syncthreads();
        if (tid == 0) {
            int64_t run = 0;
            for (int i = 0; i < nt; ++i) {
                const int64_t v = part[i];
                part[i] = run;
                run = max(run, v);
            }
        }
        __syncthreads();
        int64_t run = part[tid];
        for (int i = i0; i < i1; ++i) {
            run = max(run, clampT(cu[i]));
            bound[i] = (int32_t)run;
        }
        __syncthreads();
    }
    __threadfence_block();
    // chunks per sequence, exclusive sum
    auto nchunks = [&](int n) -> int64_t {
        const int64_t len = cu ? (int64_t)bound[n + 1] - bound[n] : T;
        return (len + C - 1) / C;
    };
    const int pn = (N + nt - 1) / nt;
    const int n0 = tid * pn, n1 = min(N, n0 + pn);
    int64_t sum = 0;
    for (int n = n0; n < n1; ++n) sum += nchunks(n);
    part[tid] = sum;
    __syncthreads();
    if (tid == 0) {
        int64_t acc = 0;
        for (int i = 0; i < nt; ++i) {
            const int64_t v = part[i];
            part[i] = acc;
            acc += v;
        }
        chunk_off[N] = (int32_t)acc;
    }
    __syncthreads();
    int64_t acc = part[tid];
    for (int n = n0; n < n1; ++n) {
        chunk_off[n] = (int32_t)acc;
        acc += nchunks(n);
    }
}

// Rows [a, b) of sequence n (bound[] from the header when packed).
__device__ __forceinline__ void seq_rows(const int32_t *hdr, bool packed, int64_t T, int N, int n,
                                         int64_t &a, int64_t &b) {
    if (packed) {
        const int32_t *bound = hdr + (N + 1);
        a = bound[n];
        b = bound[n + 1];
    } else {
        a = (int64_t)n * T;
        b = a + T;
    }
}

// eight fp32 values -> eight fp16 (round to nearest) in one 16-byte word
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    uint4 u;
    __half2 t;
    t = __floats2half2_rn(x[0], x[1]); u.x = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2half2_rn(x[2], x[3]); u.y = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2half2_rn(x[4], x[5]); u.z = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2half2_rn(x[6], x[7]); u.w = *reinterpret_cast<uint32_t *>(&t);
    return u;
}

// four fp32 values rounded to tf32, as one 16-byte word
__device__ __forceinline__ float4 pack4_tf32(float a, float b, float c, float d) {
    return make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

__device__ __forceinline__ void unpack8(uint4 u, float (&x)[8]) {
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// ======================================================================
// Phase A
// ======================================================================
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t A_G = 0;            // fp32 [64][128] G (cumsum)              32 KiB
constexpr uint32_t A_BT = 32768;       // bf16 B tiles [Q'_a; K'_a], 128 rows    32 KiB
constexpr uint32_t A_AT = 65536;       // bf16 A tiles K^(a), 20 row-groups      40 KiB
constexpr uint32_t A_ATKB = 20480;     //   bytes between its two K-blocks
// reused after the Akk/Aqk MMAs have completed:
constexpr uint32_t A_AK = 32768;       // fp32 [64][64] Akk                      16 KiB
constexpr uint32_t A_AQ = 49152;       // bf16 Aqk, K-major SW128 64x64            8 KiB
constexpr uint32_t A_TR = 57344;       // bf16 [T; R], K-major SW128 128x64       16 KiB
constexpr uint32_t A_KT = 73728;       // bf16 K*exp(G), MN-major SW128           16 KiB
constexpr uint32_t A_XS = 90112;       // fp32 [64][64] X = (I+Akk)^-1 (+ scratch) 16 KiB
constexpr uint32_t A_MISC = 106496;    // beta[64], Rref[4][128], GL[128], barriers
constexpr uint32_t A_SMEM = A_MISC + 4096 + 1024;   // + alignment slack
// first row-group of the packed K^(a) tile: 0, 2, 6, 12
__device__ __forceinline__ int at_group(int a) { return a * (a + 1); }

__global__ void __launch_bounds__(256, 2)
intra_chunk_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ g, const __nv_bfloat16 *__restrict__ beta,
                   const int32_t *__restrict__ cu, int64_t T, int N, int H,
                   uint8_t *__restrict__ ws, uint32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + A_G);
    float *AK = reinterpret_cast<float *>(sm + A_AK);
    float *XS = reinterpret_cast<float *>(sm + A_XS);
    float *bs = reinterpret_cast<float *>(sm + A_MISC);          // [64]
    float *Rref = bs + 64;                                        // [4][128]
    float *GL = Rref + 4 * 128;                                   // [128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(GL + 128);      // [4]
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 4);
    volatile uint32_t *abort_flag = tmem_ptr + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    const int32_t *chunk_off = reinterpret_cast<const int32_t *>(ws);
    const int cidx = blockIdx.x;
    const int total = chunk_off[N];
    if (cidx >= total) return;
    // sequence owning this chunk: last n with chunk_off[n] <= cidx
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= cidx) lo = mid; else hi = mid - 1;
    }
    const int n = lo;
    int64_t ra, rb;
    seq_rows(chunk_off, cu != nullptr, T, N, n, ra, rb);
    const int64_t t0 = ra + (int64_t)(cidx - chunk_off[n]) * C;
    const int L = (int)((rb - t0) < C ? (rb - t0) : C);
    uint8_t *slot = ws + header_bytes(N) + ((size_t)cidx * H + h) * kSlotBytes;

    if (warp == 0) {
        tmem_alloc(tmem_ptr, 256);
        tmem_relinquish();
        tc_fence_before();
    }
    if (tid == 32) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        *abort_flag = 0u;
    }

    // ---- A0: beta and the chunk-local cumsum of the clamped log-decay
    if (tid < 64) bs[tid] = tid < L ? __bfloat162float(beta[(size_t)(t0 + tid) * H + h]) : 0.f;
    {
        const int c = tid & 127, half = tid >> 7;
        float gv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = half * 32 + i;
            gv[i] = r < L ? fmaxf(__bfloat162float(g[((size_t)(t0 + r) * H + h) * D + c]), -5.f)
                          : 0.f;
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            acc += gv[i];
            Gs[(half * 32 + i) * D + c] = acc;
        }
    }
    __syncthreads();
    if (tid >= 128) {
        const int c = tid & 127;
        const float base = Gs[31 * D + c];
        for (int i = 32; i < 64; ++i) Gs[i * D + c] += base;
    }
    __syncthreads();
    if (tid < 128) {
        const int c = tid;
        GL[c] = L > 0 ? Gs[(L - 1) * D + c] : 0.f;
        Rref[c] = 0.f;
        Rref[128 + c] = Gs[15 * D + c];
        Rref[256 + c] = Gs[31 * D + c];
        Rref[384 + c] = Gs[47 * D + c];
    }
    __syncthreads();

    // ---- A1: Akk / Aqk on tensor cores, tf32 operands (K-major, 128B swizzle),
    // accumulated over two 64-channel halves that reuse one operand buffer.
    // B tiles: row 32a + i      = q_r * exp(G_r - R_a),  r = 16a + i
    //          row 32a + 16 + i = k_r * exp(G_r - R_a)
    // A tiles: K^(a) row s (s <= 16a+15) = k_s * exp(R_a - G_s), packed from
    //          row-group at_group(a)
    // D^(a) (M=64 rows s, N=32: the 16 q-rows and 16 k-rows of block a) goes to
    // TMEM columns 32a.
    const uint32_t tmem_hold = 0;  // (TMEM base read after the first barrier below)
    (void)tmem_hold;
    bool ok = true;
    for (int hf = 0; hf < 2; ++hf) {
        const int c0 = 64 * hf;
        if (ok) {
            for (int task = tid; task < 128 * 16; task += 256) {
                const int row = task >> 4, ch = task & 15;   // ch: 4-channel chunk of this half
                const int a = row >> 5, isk = (row >> 4) & 1, r = 16 * a + (row & 15);
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (r < L) {
                    const __nv_bfloat16 *src =
                        (isk ? k : q) + ((size_t)(t0 + r) * H + h) * D + c0 + ch * 4;
                    const uint2 u = *reinterpret_cast<const uint2 *>(src);
                    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
                    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
                    const int c = c0 + ch * 4;
                    const float *gr = Gs + r * D + c, *ra = Rref + a * 128 + c;
                    x = pack4_tf32(f0.x * __expf(gr[0] - ra[0]), f0.y * __expf(gr[1] - ra[1]),
                                   f1.x * __expf(gr[2] - ra[2]), f1.y * __expf(gr[3] - ra[3]));
                }
                *reinterpret_cast<float4 *>(sm + A_BT + sw128_kmajor_off32(row, ch * 4, 16384)) = x;
            }
            for (int task = tid; task < 160 * 16; task += 256) {
                const int prow = task >> 4, ch = task & 15;
                int a = 3;
                if (prow < 16) a = 0; else if (prow < 48) a = 1; else if (prow < 96) a = 2;
                const int s = prow - at_group(a) * 8;
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s < L) {
                    const __nv_bfloat16 *src = k + ((size_t)(t0 + s) * H + h) * D + c0 + ch * 4;
                    const uint2 u = *reinterpret_cast<const uint2 *>(src);
                    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
                    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
                    const int c = c0 + ch * 4;
                    const float *gs = Gs + s * D + c, *ra = Rref + a * 128 + c;
                    x = pack4_tf32(f0.x * __expf(ra[0] - gs[0]), f0.y * __expf(ra[1] - gs[1]),
                                   f1.x * __expf(ra[2] - gs[2]), f1.y * __expf(ra[3] - gs[3]));
                }
                *reinterpret_cast<float4 *>(sm + A_AT + sw128_kmajor_off32(prow, ch * 4, A_ATKB)) = x;
            }
        }
        fence_async_smem();
        __syncthreads();
        tc_fence_after();
        if (ok && tid == 0) {
            const uint32_t tm = *tmem_ptr;
            const uint32_t id = idesc(FMT_TF32, 64, 32, 0, 0);
            for (int a = 0; a < 4; ++a)
                for (int kk = 0; kk < 8; ++kk) {          // 8 steps of K=8 over 64 channels
                    const uint32_t koff = kk >> 2, kin = (kk & 3) * 32;
                    const uint64_t ad = smem_desc(
                        sbase + A_AT + at_group(a) * 1024 + koff * A_ATKB + kin, 16, 1024, SW_128B);
                    const uint64_t bd = smem_desc(sbase + A_BT + (4 * a) * 1024 + koff * 16384 + kin,
                                                  16, 1024, SW_128B);
                    mma_tf32(tm + 32 * a, ad, bd, id, (hf > 0 || kk > 0) ? 1u : 0u);
                }
            mma_commit(&bars[hf]);
        }
        if (ok) ok = mbar_wait_abortable(&bars[hf], 0, err, abort_flag);
        tc_fence_after();
    }
    const uint32_t tmem = *tmem_ptr;

    // ---- A2: Akk (fp32, beta applied, strictly lower) and Aqk (fp16, lower incl. diagonal)
    if (ok && warp < 4) {
        const int s = 16 * warp + (lane & 15);
        for (int a = 0; a < 4; ++a) {
            float vq[16], vk[16];
            tmem_ld16(taddr(tmem, 32 * warp, 32 * a), vq);
            tmem_ld16(taddr(tmem, 32 * warp, 32 * a + 16), vk);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = 16 * a + j;
                    AK[r * 64 + s] = (s < r && r < L) ? bs[r] * vk[j] : 0.f;
                    const float aq = (s <= r && r < L) ? vq[j] : 0.f;
                    reinterpret_cast<__half *>(sm + A_AQ + sw128_kmajor_off(r, s, 0))[0] =
                        __float2half_rn(aq);
                }
            }
        }
    }
    // K*exp(G) as the MN-major B operand of W = T (K*exp(G)) (region freed by the MMA above)
    if (ok && warp >= 4) {
        for (int task = tid - 128; task < 64 * 16; task += 128) {
            const int s = task >> 4, ch = task & 15;
            float x[8];
            if (s < L) {
                const __nv_bfloat16 *src = k + ((size_t)(t0 + s) * H + h) * D + ch * 8;
                unpack8(*reinterpret_cast<const uint4 *>(src), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= __expf(Gs[s * D + ch * 8 + e]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            *reinterpret_cast<uint4 *>(sm + A_KT + sw128_mnmajor_off(ch * 8, s, kKhMNBlock)) =
                pack8(x);
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- A3: X = (I + Akk)^-1, blocked over 16x16 blocks, fp32
    // (every __syncthreads below is reached by all threads, whatever `ok` is)
    // diagonal blocks by forward substitution: thread (a, j) owns column j of block a
    if (ok && tid < 64) {
        const int a = tid >> 4, j = tid & 15, o = 16 * a;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) acc = fmaf(-AK[(o + i) * 64 + o + m], x[m], acc);
            x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) XS[(o + i) * 64 + o + j] = x[i];
    }
    __syncthreads();
    // off-diagonal blocks, by distance d = a - b:
    //   Y_ab = sum_{m=b}^{a-1} A_am X_mb ;  X_ab = -X_aa Y_ab
    // Y_ab is parked in the (unused) upper-triangular block (b, a) of XS.
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;   // blocks at this distance
        if (ok) {
            for (int e = tid; e < nb * 256; e += 256) {
                const int b = e >> 8, a = b + d, i = (e >> 4) & 15, j = e & 15;
                float acc = 0.f;
                for (int m = b; m < a; ++m)
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        acc = fmaf(AK[(16 * a + i) * 64 + 16 * m + t],
                                   XS[(16 * m + t) * 64 + 16 * b + j], acc);
                XS[(16 * b + i) * 64 + 16 * a + j] = acc;
            }
        }
        __syncthreads();
        if (ok) {
            for (int e = tid; e < nb * 256; e += 256) {
                const int b = e >> 8, a = b + d, i = (e >> 4) & 15, j = e & 15;
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    acc = fmaf(XS[(16 * a + i) * 64 + 16 * a + t],
                               XS[(16 * b + t) * 64 + 16 * a + j], acc);
                XS[(16 * a + i) * 64 + 16 * b + j] = -acc;
            }
        }
        __syncthreads();
    }
    // T = X Diag(beta) into rows 0..63 of [T; R] (bf16, K-major SW128)
    if (ok) {
        for (int task = tid; task < 64 * 8; task += 256) {
            const int r = task >> 3, ch = task & 7;
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int s = ch * 8 + e;
                const float xv = (s == r) ? 1.f : (s < r ? XS[r * 64 + s] : 0.f);
                x[e] = xv * bs[s];
            }
            *reinterpret_cast<uint4 *>(sm + A_TR + sw128_kmajor_off(r, ch * 8, 0)) = pack8(x);
        }
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();

    // ---- A4: R = Aqk T  (M=64, N=64, K=64) into TMEM columns 128..191
    if (ok && tid == 0) {
        const uint32_t id = idesc(FMT_F16, 64, 64, 0, 1);
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(sbase + A_AQ + kk * 32, 16, 1024, SW_128B);
            const uint64_t bd = smem_desc(sbase + A_TR + kk * 2048, 8192, 1024, SW_128B);
            mma_f16(tmem + 128, ad, bd, id, kk > 0);
        }
        mma_commit(&bars[2]);
    }
    if (ok) ok = mbar_wait_abortable(&bars[2], 0, err, abort_flag);
    tc_fence_after();
    if (ok && warp < 4) {
        const int r = 16 * warp + (lane & 15);
        float x[64];
        tmem_ld16(taddr(tmem, 32 * warp, 128), *reinterpret_cast<float(*)[16]>(x));
        tmem_ld16(taddr(tmem, 32 * warp, 144), *reinterpret_cast<float(*)[16]>(x + 16));
        tmem_ld16(taddr(tmem, 32 * warp, 160), *reinterpret_cast<float(*)[16]>(x + 32));
        tmem_ld16(taddr(tmem, 32 * warp, 176), *reinterpret_cast<float(*)[16]>(x + 48));
        tmem_wait_ld();
        if (lane < 16) {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = x[ch * 8 + e];
                *reinterpret_cast<uint4 *>(sm + A_TR + sw128_kmajor_off(64 + r, ch * 8, 0)) =
                    pack8(y);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- A5: D1 = [T; R] (K*exp(G))  (M=128, N=128, K=64) into TMEM columns 0..127
    if (ok && tid == 0) {
        const uint32_t id = idesc(FMT_F16, 128, 128, 0, 1);
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(sbase + A_TR + kk * 32, 16, 1024, SW_128B);
            const uint64_t bd = smem_desc(sbase + A_KT + kk * 2048, kKhMNBlock, 1024, SW_128B);
            mma_f16(tmem, ad, bd, id, kk > 0);
        }
        mma_commit(&bars[3]);
    }
    // [T; R] is final: copy it to the slot while the MMA runs (reads only)
    if (ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(sm + A_TR);
        uint4 *dst = reinterpret_cast<uint4 *>(slot + kSlotTR);
        for (int i = tid; i < 16384 / 16; i += 256) dst[i] = src[i];
        // Khat and Gamma_L straight to the slot
        for (int task = tid; task < 64 * 16; task += 256) {
            const int s = task >> 4, ch = task & 15;
            float x[8];
            if (s < L) {
                const __nv_bfloat16 *srck = k + ((size_t)(t0 + s) * H + h) * D + ch * 8;
                unpack8(*reinterpret_cast<const uint4 *>(srck), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = ch * 8 + e;
                    x[e] *= __expf(GL[c] - Gs[s * D + c]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            *reinterpret_cast<uint4 *>(slot + kSlotKh + sw128_mnmajor_off(ch * 8, s, kKhMNBlock)) =
                pack8(x);
        }
        if (tid < 128) reinterpret_cast<float *>(slot + kSlotGam)[tid] = __expf(GL[tid]);
    }
    if (ok) ok = mbar_wait_abortable(&bars[3], 0, err, abort_flag);
    tc_fence_after();

    // ---- A6: rows 0..63 -> -W, rows 64..127 -> P = Q*exp(G) - R (K*exp(G))
    if (ok) {
        const int quad = warp & 3, chalf = warp >> 2;
        const int row = 32 * quad + lane;
        float x[64];
#pragma unroll
        for (int p = 0; p < 4; ++p)
            tmem_ld16(taddr(tmem, 32 * quad, 64 * chalf + 16 * p),
                      *reinterpret_cast<float(*)[16]>(x + 16 * p));
        tmem_wait_ld();
        const int r = row & 63;
        if (row < 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i) x[i] = -x[i];
        } else {
            if (r < L) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float qv[8];
                    unpack8(*reinterpret_cast<const uint4 *>(
                                q + ((size_t)(t0 + r) * H + h) * D + 64 * chalf + ch * 8),
                            qv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = 64 * chalf + ch * 8 + e;
                        x[ch * 8 + e] = qv[e] * __expf(Gs[r * D + c]) - x[ch * 8 + e];
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) x[i] = 0.f;
            }
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = x[ch * 8 + e];
            *reinterpret_cast<uint4 *>(slot + kSlotWP +
                                       sw128_kmajor_off(row, 64 * chalf + ch * 8, kWPKBlock)) =
                pack8(y);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ======================================================================
// Phase B
// ======================================================================
template <int DVS>
struct BLayout {
    static constexpr uint32_t kVBytes = 64 * DVS * 2;          // V slice tile
    static constexpr uint32_t kStage = kSlotBytes + kVBytes;   // slot image + V
    static constexpr uint32_t kSB = 128 * DVS * 2;             // bf16 S  (K=128 x N=DVS)
    static constexpr uint32_t kUB = 64 * DVS * 2;              // bf16 U  (K=64 x N=DVS)
    static constexpr uint32_t kKGroup = (DVS / 8) * 128;       // k-group stride, interleaved MN-major
    static constexpr uint32_t oStage0 = 0;
    static constexpr uint32_t oStage1 = (kStage + 1023) & ~1023u;
    static constexpr uint32_t oSB = oStage1 + ((kStage + 1023) & ~1023u);
    static constexpr uint32_t oUB = oSB + kSB;
    static constexpr uint32_t oBar = oUB + kUB;
    static constexpr uint32_t kBytes = oBar + 256 + 1024;      // + barriers + alignment slack
    static constexpr uint32_t kTmemCols = DVS == 32 ? 128 : (DVS == 64 ? 256 : 512);
};

enum BBar {
    FULL0 = 0, FULL1, EMPTY0, EMPTY1, TDFULL0, TDFULL1, TDEMPTY0, TDEMPTY1,
    SBREADY, TSSCALED, UBREADY, TSFULL, DRAIN, NBARS
};

template <int DVS>
__global__ void __launch_bounds__(384, 1)
state_pass_kernel(const __nv_bfloat16 *__restrict__ v, const float *state_in,
                  const int32_t *__restrict__ cu, int64_t T, int N, int H,
                  const uint8_t *__restrict__ ws, float *__restrict__ o,
                  float *state_out, uint32_t *err) {
    using Lay = BLayout<DVS>;
    constexpr int NSL = D / DVS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::oBar);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + NBARS);
    volatile uint32_t *abort_flag = tmem_ptr + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = blockIdx.x % NSL;
    const int unit = blockIdx.x / NSL;
    const int n = unit / H, h = unit % H;
    if (n >= N) return;
    const int32_t *chunk_off = reinterpret_cast<const int32_t *>(ws);
    int64_t ra, rb;
    seq_rows(chunk_off, cu != nullptr, T, N, n, ra, rb);
    const int nch = (int)((rb - ra + C - 1) / C);
    const int c0 = chunk_off[n];
    const uint8_t *slots = ws + header_bytes(N);
    const int j0 = slice * DVS;   // first value channel of this slice

    if (warp == 1) {
        tmem_alloc(tmem_ptr, Lay::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars[FULL0], 33);
        mbar_init(&bars[FULL1], 33);
        mbar_init(&bars[EMPTY0], 1);
        mbar_init(&bars[EMPTY1], 1);
        mbar_init(&bars[TDFULL0], 1);
        mbar_init(&bars[TDFULL1], 1);
        mbar_init(&bars[TDEMPTY0], 4);
        mbar_init(&bars[TDEMPTY1], 4);
        mbar_init(&bars[SBREADY], 4);
        mbar_init(&bars[TSSCALED], 4);
        mbar_init(&bars[UBREADY], 2);
        mbar_init(&bars[TSFULL], 1);
        mbar_init(&bars[DRAIN], 1);
        mbar_fence_init();
        *abort_flag = 0u;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t tTD0 = tmem, tTD1 = tmem + DVS, tTS = tmem + 2 * DVS;

    if (warp == 0) {
        // ------------------------------------------------ producer
        int issued_last = -1;
        for (int j = 0; j < nch; ++j) {
            const int st = j & 1;
            if (j >= 2 && !mbar_wait_abortable(&bars[EMPTY0 + st], ((j >> 1) + 1) & 1, err,
                                               abort_flag))
                break;
            uint8_t *stg = sm + (st ? Lay::oStage1 : Lay::oStage0);
            const uint8_t *src = slots + ((size_t)(c0 + j) * H + h) * kSlotBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[FULL0 + st], kSlotBytes);
                bulk_g2s(stg, src, kSlotBytes, &bars[FULL0 + st]);
            }
            const int64_t t0 = ra + (int64_t)j * C;
            const int L = (int)((rb - t0) < C ? (rb - t0) : C);
            // V slice -> fp16 MMA operand (MN-major, interleaved core matrices);
            // rows past the end of the sequence are zero
            uint8_t *vt = stg + kSlotBytes;
            constexpr int CPR = DVS / 8;   // 16-byte chunks per row
            for (int task = lane; task < 64 * CPR; task += 32) {
                const int r = task / CPR, ch = task % CPR;
                float x[8];
                if (r < L) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                        v + ((size_t)(t0 + r) * H + h) * D + j0 + ch * 8));
                    unpack8(u, x);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = 0.f;
                }
                *reinterpret_cast<uint4 *>(vt + interleave_mnmajor_off(ch * 8, r, Lay::kKGroup)) =
                    pack8(x);
            }
            fence_async_smem();
            mbar_arrive(&bars[FULL0 + st]);
            issued_last = j;
        }
        // drain: never leave the CTA with bulk copies still landing in its shared memory
        for (int j = issued_last - 1; j <= issued_last; ++j)
            if (j >= 0) mbar_wait(&bars[FULL0 + (j & 1)], (j >> 1) & 1, err, 1u << 22);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_nn = idesc(FMT_F16, 128, DVS, 0, 1);   // A K-major, B MN-major
            const uint32_t id_mm = idesc(FMT_F16, 128, DVS, 1, 1);   // A MN-major, B MN-major
            for (int j = 0; j < nch; ++j) {
                const int st = j & 1, b = j & 1;
                const uint32_t stg = sbase + (st ? Lay::oStage1 : Lay::oStage0);
                const uint32_t tTD = b ? tTD1 : tTD0;
                if (!mbar_wait_abortable(&bars[FULL0 + st], (j >> 1) & 1, err, abort_flag)) break;
                if (j >= 2 && !mbar_wait_abortable(&bars[TDEMPTY0 + b], ((j >> 1) + 1) & 1, err,
                                                   abort_flag))
                    break;
                tc_fence_after();
                // [U; O] = [T; R] V
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(stg + kSlotTR + kk * 32, 16, 1024, SW_128B);
                    const uint64_t bd = smem_desc(stg + kSlotBytes + kk * 2 * Lay::kKGroup,
                                                  Lay::kKGroup, 128, SW_NONE);
                    mma_f16(tTD, ad, bd, id_nn, kk > 0);
                }
                if (!mbar_wait_abortable(&bars[SBREADY], j & 1, err, abort_flag)) break;
                tc_fence_after();
                // [U; O] += [-W; P] S
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = smem_desc(
                        stg + kSlotWP + (kk >> 2) * kWPKBlock + (kk & 3) * 32, 16, 1024, SW_128B);
                    const uint64_t bd = smem_desc(sbase + Lay::oSB + kk * 2 * Lay::kKGroup,
                                                  Lay::kKGroup, 128, SW_NONE);
                    mma_f16(tTD, ad, bd, id_nn, 1);
                }
                mma_commit(&bars[TDFULL0 + b]);
                if (!mbar_wait_abortable(&bars[UBREADY], j & 1, err, abort_flag)) break;
                if (!mbar_wait_abortable(&bars[TSSCALED], j & 1, err, abort_flag)) break;
                tc_fence_after();
                // S += Khat^T U
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc(stg + kSlotKh + kk * 2048, kKhMNBlock, 1024,
                                                  SW_128B);
                    const uint64_t bd = smem_desc(sbase + Lay::oUB + kk * 2 * Lay::kKGroup,
                                                  Lay::kKGroup, 128, SW_NONE);
                    mma_f16(tTS, ad, bd, id_mm, 1);
                }
                mma_commit(&bars[TSFULL]);
                mma_commit(&bars[EMPTY0 + st]);
            }
            // drain: every MMA issued above has completed before TMEM is released
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, err, 1u << 22);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ U / O epilogue
        const int quad = warp - 4;
        const int row = 32 * quad + lane;
        for (int j = 0; j < nch; ++j) {
            const int b = j & 1;
            const uint32_t tTD = b ? tTD1 : tTD0;
            if (!mbar_wait_abortable(&bars[TDFULL0 + b], (j >> 1) & 1, err, abort_flag)) break;
            tc_fence_after();
            const int64_t t0 = ra + (int64_t)j * C;
            const int L = (int)((rb - t0) < C ? (rb - t0) : C);
            const int r = row - 64;
#pragma unroll
            for (int p = 0; p < DVS / 16; ++p) {
                float x[16];
                tmem_ld16(taddr(tTD, 32 * quad, 16 * p), x);
                tmem_wait_ld();
                float y0[8], y1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    y0[e] = x[e];
                    y1[e] = x[8 + e];
                }
                if (quad < 2) {
                    // U rows -> bf16 B operand (MN-major, interleaved core matrices)
                    *reinterpret_cast<uint4 *>(
                        sm + Lay::oUB + interleave_mnmajor_off(16 * p, row, Lay::kKGroup)) = pack8(y0);
                    *reinterpret_cast<uint4 *>(
                        sm + Lay::oUB + interleave_mnmajor_off(16 * p + 8, row, Lay::kKGroup)) =
                        pack8(y1);
                } else if (r < L) {
                    float4 *dst = reinterpret_cast<float4 *>(o + ((size_t)(t0 + r) * H + h) * D + j0 +
                                                             16 * p);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
                }
            }
            if (quad < 2) {
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[UBREADY]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[TDEMPTY0 + b]);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------ state epilogue
        const int quad = warp - 8;
        const int c = 32 * quad + lane;   // key channel = TMEM lane
        const uint32_t tS = taddr(tTS, 32 * quad, 0);
        const size_t srow = (((size_t)n * H + h) * D + c) * D + j0;
        uint8_t *sbp = sm + Lay::oSB;
        auto put_sb = [&](int p, const float (&x)[16]) {
            float y0[8], y1[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                y0[e] = x[e];
                y1[e] = x[8 + e];
            }
            *reinterpret_cast<uint4 *>(sbp + interleave_mnmajor_off(16 * p, c, Lay::kKGroup)) =
                pack8(y0);
            *reinterpret_cast<uint4 *>(sbp + interleave_mnmajor_off(16 * p + 8, c, Lay::kKGroup)) =
                pack8(y1);
        };
        auto signal = [&](int which) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[which]);
        };
        auto stage_gamma = [&](int j, float &gam) -> bool {
            const int st = j & 1;
            if (!mbar_wait_abortable(&bars[FULL0 + st], (j >> 1) & 1, err, abort_flag))
                return false;
            gam = reinterpret_cast<const float *>(sm + (st ? Lay::oStage1 : Lay::oStage0) +
                                                  kSlotGam)[c];
            return true;
        };
        if (nch == 0) {
            // empty sequence: the state passes through unchanged
            if (state_out)
                for (int i = 0; i < DVS / 4; ++i)
                    reinterpret_cast<float4 *>(state_out + srow)[i] =
                        state_in ? reinterpret_cast<const float4 *>(state_in + srow)[i]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            // S_0: bf16 copy for the first MMA, fp32 copy (already scaled by Gamma_0) into TMEM
            float gam = 0.f;
            bool ok = true;
            for (int p = 0; p < DVS / 16; ++p) {
                float x[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = state_in
                        ? reinterpret_cast<const float4 *>(state_in + srow)[4 * p + i]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
                }
                put_sb(p, x);
            }
            fence_async_smem();
            signal(SBREADY);
            ok = stage_gamma(0, gam);
            if (ok) {
                for (int p = 0; p < DVS / 16; ++p) {
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 f = state_in
                            ? reinterpret_cast<const float4 *>(state_in + srow)[4 * p + i]
                            : make_float4(0.f, 0.f, 0.f, 0.f);
                        x[4 * i] = f.x * gam; x[4 * i + 1] = f.y * gam;
                        x[4 * i + 2] = f.z * gam; x[4 * i + 3] = f.w * gam;
                    }
                    tmem_st16(tS + 16 * p, x);
                }
                tmem_wait_st();
                tc_fence_before();
                signal(TSSCALED);
            }
            for (int j = 0; ok && j < nch; ++j) {
                if (!mbar_wait_abortable(&bars[TSFULL], j & 1, err, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (j + 1 == nch) break;
                // S_{j+1}: bf16 copy for the next chunk's MMA (critical path) ...
                for (int p = 0; p < DVS / 16; ++p) {
                    float x[16];
                    tmem_ld16(tS + 16 * p, x);
                    tmem_wait_ld();
                    put_sb(p, x);
                }
                fence_async_smem();
                signal(SBREADY);
                // ... then the fp32 copy scaled by Gamma_{j+1} for the next state update
                if (!stage_gamma(j + 1, gam)) { ok = false; break; }
                for (int p = 0; p < DVS / 16; ++p) {
                    float x[16];
                    tmem_ld16(tS + 16 * p, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] *= gam;
                    tmem_st16(tS + 16 * p, x);
                }
                tmem_wait_st();
                tc_fence_before();
                signal(TSSCALED);
            }
            if (ok && state_out && !*abort_flag) {
                for (int p = 0; p < DVS / 16; ++p) {
                    float x[16];
                    tmem_ld16(tS + 16 * p, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        reinterpret_cast<float4 *>(state_out + srow)[4 * p + i] =
                            make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}

}  // namespace tc

// ======================================================================
// host side
// ======================================================================
size_t prefill_tc_workspace_bytes(int64_t rows, int N, int H, int d) {
    if (d != tc::D) return 0;
    const int64_t max_chunks = (rows + tc::C - 1) / tc::C + N;
    return (size_t)tc::header_bytes(N) + (size_t)max_chunks * H * tc::kSlotBytes;
}

template <int DVS>
static cudaError_t launch_state_pass(const PrefillArgs &a, cudaStream_t st) {
    using Lay = tc::BLayout<DVS>;
    auto kern = tc::state_pass_kernel<DVS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lay::kBytes);
    if (e != cudaSuccess) return e;
    const int grid = a.N * a.H * (tc::D / DVS);
    kern<<<grid, 384, Lay::kBytes, st>>>((const __nv_bfloat16 *)a.v, a.state_in, a.cu_seqlens,
                                         a.T, a.N, a.H, (const uint8_t *)a.workspace,
                                         (float *)a.o, a.state_out, a.err);
    e = cudaGetLastError();
    Profiler::mark(st);
    return e;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    if (a.dk != tc::D || a.dv != tc::D) return cudaErrorInvalidValue;
    uint8_t *ws = (uint8_t *)a.workspace;
    tc::chunk_table_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.T, a.N,
                                               reinterpret_cast<int32_t *>(ws));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Profiler::mark(st);
    const int64_t rows = (int64_t)a.B * a.T;
    const int64_t max_chunks =
        a.cu_seqlens ? (rows + tc::C - 1) / tc::C + a.N : (int64_t)a.N * ((a.T + tc::C - 1) / tc::C);
    if (max_chunks > 0) {
        e = cudaFuncSetAttribute(tc::intra_chunk_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::A_SMEM);
        if (e != cudaSuccess) return e;
        if (max_chunks > INT32_MAX || a.H > 65535) return cudaErrorInvalidValue;
        dim3 grid((unsigned)max_chunks, (unsigned)a.H);
        tc::intra_chunk_kernel<<<grid, 256, tc::A_SMEM, st>>>(
            (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.g,
            (const __nv_bfloat16 *)a.beta, a.cu_seqlens, a.T, a.N, a.H, ws, a.err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    Profiler::mark(st);
    // dv-slices: enough CTAs to cover the SMs when there are few (sequence, head) units
    const int64_t units = (int64_t)a.N * a.H;
    if (units <= 74) return launch_state_pass<32>(a, st);
    if (units <= 148) return launch_state_pass<64>(a, st);
    return launch_state_pass<128>(a, st);
}

}  // namespace kda
