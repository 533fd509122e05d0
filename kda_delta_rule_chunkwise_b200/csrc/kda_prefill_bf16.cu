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
// Decay factors.  With G the chunk-local cumsum and R_a = G at the end of the
// 16-row block before block a (R_0 = 0), every decay term is built from
//   E1[r] = exp(G_r - R_a(r))        in [e^-80, 1]   (one exp per element)
// and per-channel block tables (one exp per channel and block):
//   ER[a]    = exp(R_a)               Gamma_r          = E1[r] ER[a(r)]
//   EL[a]    = exp(G_L - R_a)         exp(G_L - G_s)   = EL[a(s)] / E1[s]
//   PF[a][b] = exp(R_a - R_b), b < a  exp(R_a - G_s)   = PF[a][b(s)] / E1[s]
// Every product above is of two factors that are each <= 1 or each within
// [e^-80, e^80], so none of them overflows, and a factor underflows only where
// the exact value is itself negligible.
//
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t A_E1 = 0;          // fp32 [64][128]: G, then E1 in place          32 KiB
constexpr uint32_t A_MISC = 32768;    // beta, GL, Rref, ER, EL, PF, barriers         10 KiB
constexpr uint32_t A_OPS = 43008;     // operand region (two uses, below)
// before the Akk/Aqk MMAs (one 32-channel round at a time, tf32, K-major SW128):
constexpr uint32_t A_BT = A_OPS;              // [Q'_a; K'_a], 128 rows x 128 B   16 KiB
constexpr uint32_t A_AT = A_OPS + 16384;      // packed K^(a), 160 rows x 128 B   20 KiB
// after them:
constexpr uint32_t A_AK = A_OPS;              // fp32 [64][64] Akk, then X in place 16 KiB
constexpr uint32_t A_AQ = A_OPS + 16384;      // fp16 Aqk, MN-major SW128 64x64      8 KiB
constexpr uint32_t A_TR = A_OPS + 24576;      // fp16 [T; R], K-major SW128 128x64  16 KiB
constexpr uint32_t A_KT = A_OPS + 40960;      // fp16 K*Gamma, MN-major SW128       16 KiB
constexpr uint32_t A_Y = A_OPS + 57344;       // fp32 [16][16] solve scratch          1 KiB
constexpr uint32_t A_SMEM = A_OPS + 58368 + 1024;   // + alignment slack (= 102400)
// first row-group of the packed K^(a) tile: 0, 2, 6, 12
__device__ __forceinline__ int at_group(int a) { return a * (a + 1); }
// index of the block pair (a, b), b < a, in PF
__device__ __forceinline__ int pf_index(int a, int b) { return a * (a - 1) / 2 + b; }

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
__device__ __forceinline__ float4 bf4(uint2 u) {   // four bf16 -> fp32
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(f0.x, f0.y, f1.x, f1.y);
}
__device__ __forceinline__ float4 tf4(float4 a) {
    return make_float4(to_tf32(a.x), to_tf32(a.y), to_tf32(a.z), to_tf32(a.w));
}

__global__ void __launch_bounds__(256, 2)
intra_chunk_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ g, const __nv_bfloat16 *__restrict__ beta,
                   const int32_t *__restrict__ cu, int64_t T, int N, int H,
                   uint8_t *__restrict__ ws, uint32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    float *E1 = reinterpret_cast<float *>(sm + A_E1);
    float *bs = reinterpret_cast<float *>(sm + A_MISC);   // [64]
    float *GL = bs + 64;                                   // [128]
    float *Rref = GL + 128;                                // [4][128]
    float *ER = Rref + 4 * 128;                            // [4][128]
    float *EL = ER + 4 * 128;                              // [4][128]
    float *PF = EL + 4 * 128;                              // [6][128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(PF + 6 * 128);   // [8]
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 8);
    volatile uint32_t *abort_flag = tmem_ptr + 1;
    float *AK = reinterpret_cast<float *>(sm + A_AK);
    float *Yb = reinterpret_cast<float *>(sm + A_Y);

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
    auto row_ptr = [&](const __nv_bfloat16 *base, int r) {
        return base + ((size_t)(t0 + r) * H + h) * D;
    };

    if (warp == 0) {
        tmem_alloc(tmem_ptr, 256);
        tmem_relinquish();
        tc_fence_before();
    }
    if (tid == 32) {
        for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        *abort_flag = 0u;
    }

    // ---- A0: beta and the chunk-local cumsum G of the clamped log-decay (fp32)
    if (tid < 64) bs[tid] = tid < L ? __bfloat162float(beta[(size_t)(t0 + tid) * H + h]) : 0.f;
    {
        const int c = tid & 127, half = tid >> 7;
        float gv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = half * 32 + i;
            gv[i] = r < L ? fmaxf(__bfloat162float(row_ptr(g, r)[c]), -5.f) : 0.f;
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            acc += gv[i];
            E1[(half * 32 + i) * D + c] = acc;
        }
    }
    __syncthreads();
    if (tid >= 128) {
        const int c = tid & 127;
        const float base = E1[31 * D + c];
        for (int i = 32; i < 64; ++i) E1[i * D + c] += base;
    }
    __syncthreads();
    if (tid < 128) {
        const int c = tid;
        const float gl = L > 0 ? E1[(L - 1) * D + c] : 0.f;
        float rr[4] = {0.f, E1[15 * D + c], E1[31 * D + c], E1[47 * D + c]};
        GL[c] = gl;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            Rref[a * 128 + c] = rr[a];
            ER[a * 128 + c] = __expf(rr[a]);
            EL[a * 128 + c] = __expf(gl - rr[a]);
        }
#pragma unroll
        for (int a = 1; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < a; ++b) PF[pf_index(a, b) * 128 + c] = __expf(rr[a] - rr[b]);
    }
    __syncthreads();
    // E1 in place: exp(G_r - R_a(r)), one row per warp-iteration, float4 per lane
    for (int r = warp; r < 64; r += 8) {
        float4 gr = ld4(E1 + r * D + 4 * lane);
        const float4 rf = ld4(Rref + (r >> 4) * 128 + 4 * lane);
        gr = make_float4(__expf(gr.x - rf.x), __expf(gr.y - rf.y), __expf(gr.z - rf.z),
                         __expf(gr.w - rf.w));
        *reinterpret_cast<float4 *>(E1 + r * D + 4 * lane) = gr;
    }
    __syncthreads();

    // ---- A1: Akk / Aqk on tensor cores (tf32), four rounds of 32 channels.
    // B tile row 32a + i      = q_r E1[r]      (r = 16a + i)
    //        row 32a + 16 + i = k_r E1[r]
    // A tile (packed from row-group at_group(a)) row s, s <= 16a+15:
    //        k_s exp(R_a - G_s) = k_s / E1[s]             (s in block a)
    //                           = k_s PF[a][b(s)] / E1[s]  (s in an earlier block)
    // D^(a) = K^(a) [Q'_a; K'_a]^T (M=64 rows s, N=32) accumulates in TMEM columns 32a.
    // Task: (token row r, 4-channel piece p of the round); lane -> (row group, piece).
    bool ok = true;
    const int p_l = lane & 7, rsub = lane >> 3;   // 8 pieces x 4 rows per warp
    for (int rd = 0; rd < 4; ++rd) {
        const int c0 = 32 * rd + 4 * p_l;
        if (ok) {
            uint2 qv[2], kv[2];
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int r = 32 * it + 4 * warp + rsub;
                if (r < L) {
                    qv[it] = __ldg(reinterpret_cast<const uint2 *>(row_ptr(q, r) + c0));
                    kv[it] = __ldg(reinterpret_cast<const uint2 *>(row_ptr(k, r) + c0));
                } else {
                    qv[it] = make_uint2(0u, 0u);
                    kv[it] = make_uint2(0u, 0u);
                }
            }
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int r = 32 * it + 4 * warp + rsub;
                const int a = r >> 4, i = r & 15;
                const float4 e = ld4(E1 + r * D + c0);
                const float4 qf = bf4(qv[it]), kf = bf4(kv[it]);
                const float4 inv = make_float4(__frcp_rn(e.x), __frcp_rn(e.y), __frcp_rn(e.z),
                                               __frcp_rn(e.w));
                *reinterpret_cast<float4 *>(sm + A_BT + sw128_kmajor_off32(32 * a + i, 4 * p_l, 0)) =
                    tf4(mul4(qf, e));
                *reinterpret_cast<float4 *>(sm + A_BT +
                                            sw128_kmajor_off32(32 * a + 16 + i, 4 * p_l, 0)) =
                    tf4(mul4(kf, e));
                const float4 ki = mul4(kf, inv);
                *reinterpret_cast<float4 *>(sm + A_AT + sw128_kmajor_off32(8 * at_group(a) + r, 4 * p_l, 0)) =
                    tf4(ki);
                for (int a2 = a + 1; a2 < 4; ++a2) {
                    const float4 pf = ld4(PF + pf_index(a2, a) * 128 + c0);
                    *reinterpret_cast<float4 *>(
                        sm + A_AT + sw128_kmajor_off32(8 * at_group(a2) + r, 4 * p_l, 0)) =
                        tf4(mul4(ki, pf));
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        tc_fence_after();
        if (ok && tid == 0) {
            const uint32_t tm = *tmem_ptr;
            const uint32_t id = idesc(FMT_TF32, 64, 32, 0, 0);
            for (int a = 0; a < 4; ++a)
                for (int kk = 0; kk < 4; ++kk) {          // 4 steps of K=8 over 32 channels
                    const uint64_t ad = smem_desc(sbase + A_AT + at_group(a) * 1024 + kk * 32, 16,
                                                  1024, SW_128B);
                    const uint64_t bd = smem_desc(sbase + A_BT + (4 * a) * 1024 + kk * 32, 16,
                                                  1024, SW_128B);
                    mma_tf32(tm + 32 * a, ad, bd, id, (rd > 0 || kk > 0) ? 1u : 0u);
                }
            mma_commit(&bars[rd]);
        }
        if (ok) ok = mbar_wait_abortable(&bars[rd], 0, err, abort_flag);
        tc_fence_after();
    }
    const uint32_t tmem = *tmem_ptr;

    // ---- A2: Akk (fp32, beta applied, strictly lower) and Aqk (fp16, lower incl. diagonal,
    // MN-major: element (r, s) at (s, r) of a 64-wide MN block, so a thread's 16 rows are
    // 32 contiguous bytes)
    if (ok && warp < 4) {
        const int s = 16 * warp + (lane & 15);
        for (int a = 0; a < 4; ++a) {
            float vq[16], vk[16];
            tmem_ld16(taddr(tmem, 32 * warp, 32 * a), vq);
            tmem_ld16(taddr(tmem, 32 * warp, 32 * a + 16), vk);
            tmem_wait_ld();
            if (lane < 16) {
                float y0[8], y1[8];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = 16 * a + j;
                    AK[r * 64 + s] = (s < r && r < L) ? bs[r] * vk[j] : 0.f;
                    const float aq = (s <= r && r < L) ? vq[j] : 0.f;
                    if (j < 8) y0[j] = aq; else y1[j - 8] = aq;
                }
                *reinterpret_cast<uint4 *>(sm + A_AQ + sw128_mnmajor_off(16 * a, s, 0)) = pack8(y0);
                *reinterpret_cast<uint4 *>(sm + A_AQ + sw128_mnmajor_off(16 * a + 8, s, 0)) =
                    pack8(y1);
            }
        }
    }
    // K*Gamma = k E1 ER as the MN-major B operand of W = T (K*Gamma)
    if (ok && warp >= 4) {
        for (int task = tid - 128; task < 64 * 16; task += 128) {
            const int s = task >> 4, ch = task & 15, c = ch * 8;
            float x[8];
            if (s < L) {
                unpack8(__ldg(reinterpret_cast<const uint4 *>(row_ptr(k, s) + c)), x);
                const float4 e0 = ld4(E1 + s * D + c), e1 = ld4(E1 + s * D + c + 4);
                const float4 r0 = ld4(ER + (s >> 4) * 128 + c), r1 = ld4(ER + (s >> 4) * 128 + c + 4);
                x[0] *= e0.x * r0.x; x[1] *= e0.y * r0.y; x[2] *= e0.z * r0.z; x[3] *= e0.w * r0.w;
                x[4] *= e1.x * r1.x; x[5] *= e1.y * r1.y; x[6] *= e1.z * r1.z; x[7] *= e1.w * r1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            *reinterpret_cast<uint4 *>(sm + A_KT + sw128_mnmajor_off(c, s, kKhMNBlock)) = pack8(x);
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- A3: X = (I + Akk)^-1 in place over AK, blocked over 16x16 blocks, fp32.
    // (every __syncthreads below is reached by all threads, whatever `ok` is)
    // diagonal blocks by forward substitution, thread (a, j) owns column j of block a
    {
        float x[16];
        const int a = tid >> 4, j = tid & 15, o = 16 * a;
        if (ok && tid < 64) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc = fmaf(-AK[(o + i) * 64 + o + m], x[m], acc);
                x[i] = acc;
            }
        }
        __syncthreads();
        if (ok && tid < 64) {
#pragma unroll
            for (int i = 0; i < 16; ++i) AK[(o + i) * 64 + o + j] = x[i];
        }
    }
    __syncthreads();
    // off-diagonal blocks, row by row, b increasing (so A_am, m >= b, is still unmodified):
    //   Y = sum_{m=b}^{a-1} A_am X_mb ;   X_ab = -X_aa Y  (written over A_ab)
    for (int a = 1; a < 4; ++a)
        for (int b = 0; b < a; ++b) {
            const int i = tid >> 4, j = tid & 15;
            if (ok) {
                float acc = 0.f;
                for (int m = b; m < a; ++m)
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        acc = fmaf(AK[(16 * a + i) * 64 + 16 * m + t], AK[(16 * m + t) * 64 + 16 * b + j],
                                   acc);
                Yb[i * 16 + j] = acc;
            }
            __syncthreads();
            if (ok) {
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    acc = fmaf(AK[(16 * a + i) * 64 + 16 * a + t], Yb[t * 16 + j], acc);
                AK[(16 * a + i) * 64 + 16 * b + j] = -acc;
            }
            __syncthreads();
        }
    // T = X Diag(beta) into rows 0..63 of [T; R] (fp16, K-major SW128)
    if (ok) {
        for (int task = tid; task < 64 * 8; task += 256) {
            const int r = task >> 3, ch = task & 7;
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int s = ch * 8 + e;
                x[e] = (s <= r) ? AK[r * 64 + s] * bs[s] : 0.f;
            }
            *reinterpret_cast<uint4 *>(sm + A_TR + sw128_kmajor_off(r, ch * 8, 0)) = pack8(x);
        }
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();

    // ---- A4: R = Aqk T  (M=64, N=64, K=64; A MN-major, B MN-major) into TMEM columns 128..191
    if (ok && tid == 0) {
        const uint32_t id = idesc(FMT_F16, 64, 64, 1, 1);
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(sbase + A_AQ + kk * 2048, 8192, 1024, SW_128B);
            const uint64_t bd = smem_desc(sbase + A_TR + kk * 2048, 8192, 1024, SW_128B);
            mma_f16(tmem + 128, ad, bd, id, kk > 0);
        }
        mma_commit(&bars[4]);
    }
    if (ok) ok = mbar_wait_abortable(&bars[4], 0, err, abort_flag);
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

    // ---- A5: D1 = [T; R] (K*Gamma)  (M=128, N=128, K=64) into TMEM columns 0..127
    if (ok && tid == 0) {
        const uint32_t id = idesc(FMT_F16, 128, 128, 0, 1);
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(sbase + A_TR + kk * 32, 16, 1024, SW_128B);
            const uint64_t bd = smem_desc(sbase + A_KT + kk * 2048, kKhMNBlock, 1024, SW_128B);
            mma_f16(tmem, ad, bd, id, kk > 0);
        }
        mma_commit(&bars[5]);
    }
    // [T; R] is final: copy it to the slot while the MMA runs (reads only);
    // Khat = k EL / E1 and Gamma_L straight to the slot
    if (ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(sm + A_TR);
        uint4 *dst = reinterpret_cast<uint4 *>(slot + kSlotTR);
        for (int i = tid; i < 16384 / 16; i += 256) dst[i] = src[i];
        for (int task = tid; task < 64 * 16; task += 256) {
            const int s = task >> 4, ch = task & 15, c = ch * 8;
            float x[8];
            if (s < L) {
                unpack8(__ldg(reinterpret_cast<const uint4 *>(row_ptr(k, s) + c)), x);
                const float *e1 = E1 + s * D + c, *el = EL + (s >> 4) * 128 + c;
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= el[e] * __frcp_rn(e1[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            *reinterpret_cast<uint4 *>(slot + kSlotKh + sw128_mnmajor_off(c, s, kKhMNBlock)) =
                pack8(x);
        }
        if (tid < 128) reinterpret_cast<float *>(slot + kSlotGam)[tid] = __expf(GL[tid]);
    }
    if (ok) ok = mbar_wait_abortable(&bars[5], 0, err, abort_flag);
    tc_fence_after();

    // ---- A6: rows 0..63 -> -W, rows 64..127 -> P = q E1 ER - R (K*Gamma)
    if (ok) {
        const int quad = warp & 3, chalf = warp >> 2;
        const int row = 32 * quad + lane;
        const int r = row & 63;
        float x[64];
#pragma unroll
        for (int p = 0; p < 4; ++p)
            tmem_ld16(taddr(tmem, 32 * quad, 64 * chalf + 16 * p),
                      *reinterpret_cast<float(*)[16]>(x + 16 * p));
        tmem_wait_ld();
        if (row < 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i) x[i] = -x[i];
        } else if (r < L) {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const int c = 64 * chalf + ch * 8;
                float qv[8];
                unpack8(__ldg(reinterpret_cast<const uint4 *>(row_ptr(q, r) + c)), qv);
                const float *e1 = E1 + r * D + c, *er = ER + (r >> 4) * 128 + c;
#pragma unroll
                for (int e = 0; e < 8; ++e) x[ch * 8 + e] = qv[e] * e1[e] * er[e] - x[ch * 8 + e];
            }
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) x[i] = 0.f;
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
            // V slice -> fp16 MMA operand (MN-major, interleaved core matrices).
            // All 16-byte pieces are fetched asynchronously straight into their
            // operand positions (rows past the end of the sequence zero-filled),
            // then each lane converts the pieces it fetched from bf16 to fp16 in place.
            uint8_t *vt = stg + kSlotBytes;
            constexpr int CPR = DVS / 8;   // 16-byte pieces per row
            for (int task = lane; task < 64 * CPR; task += 32) {
                const int r = task / CPR, ch = task % CPR;
                const int rr = r < L ? r : 0;
                cp_async16(vt + interleave_mnmajor_off(ch * 8, r, Lay::kKGroup),
                           v + ((size_t)(t0 + rr) * H + h) * D + j0 + ch * 8, r < L ? 16u : 0u);
            }
            cp_async_wait_all();
            for (int task = lane; task < 64 * CPR; task += 32) {
                const int r = task / CPR, ch = task % CPR;
                uint4 *pc = reinterpret_cast<uint4 *>(vt + interleave_mnmajor_off(ch * 8, r, Lay::kKGroup));
                float x[8];
                unpack8(*pc, x);
                *pc = pack8(x);
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
