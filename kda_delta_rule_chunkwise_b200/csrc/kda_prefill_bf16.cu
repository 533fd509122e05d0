// KDA chunked prefill, bf16 path: tcgen05 (TMEM) tensor-core kernels for sm_100a.
//
// The recurrence S_t = (I - beta k k^T) Diag(exp g) S_{t-1} + beta k v^T,
// o_t = S_t^T q_t (the delta rule with per-channel retention of neurohive.io
// "Kimi K3 ... overview", section "Sequence length: hybrid KDA and Gated MLA
// attention") is evaluated in chunks of C = 64 tokens in two kernels:
//
// Phase A, intra_chunk_kernel (persistent: two CTAs per SM walk the
// (chunk, head) items; the next item's rows are prefetched while one finishes):
//   G     chunk-local inclusive cumsum of max(g, -5)                     (fp32)
//   Akk, Aqk  decay-rescaled intra-chunk products on tensor cores.  The
//         pairwise decay exp(G_r - G_s) is split as
//         exp(G_r - R_a) * exp(R_a - G_s), R_a = G at the end of the
//         previous 16-row block a.  Because g >= -5 the first factor is in
//         [e^-80, 1] and the second at most e^80, inside the fp32 exponent
//         range of tf32 operands.  That bound is what lets every tile
//         (diagonal ones included) run as a dense MMA; it is the point of the
//         lower bound on the log-decay in the section cited above.
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
// Roles in phase B: warp 0 = producer (1-D bulk copy of the slot, cp.async of
// the V slice), warp 1 = TMEM owner, warps 2-3 convert V to fp16 in place,
// warps 4-7 = U/O epilogue (TMEM -> registers; its elected thread issues the
// state update), warps 8-11 = state epilogue (fp16 copy of S, Gamma scaling of
// the TMEM state; its elected thread issues the chunk products).  Each chunk
// costs two hand-offs: state copy -> chunk products -> U copy -> state update.
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

#include <cstring>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tma.h"
#include "sm100.cuh"

namespace kda {
namespace tc {

// Pause of a phase A CTA between items when its SM also runs a state-pass chain
// in the one-launch form. The chain bounds that launch, and a phase A CTA next
// to it slows it by sharing issue slots, shared memory and TMEM. Measured at
// T=65536, H=32: 3.04 ms without a pause, 2.93 ms for 5-8 us (one item takes
// about 18 us), 3.00 ms at 10 us. With the gate and norms computed inside, the
// pause made the step slower (3.24 -> 3.42 ms), so that form does not pause.
constexpr unsigned kChainYieldNs = 6000;

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
// in chunk_off[N]), int32 bound[N+1] (the row offsets actually used:
// cu_seqlens clamped to [0, T] and made non-decreasing by a running maximum,
// so that sequences never overlap and the chunk total never exceeds the
// workspace bound), int32 ckpt_off[N+1] (first intermediate-state entry of
// each sequence, total in ckpt_off[N]) and int32 order[N+1] (the sequences by
// decreasing chunk count, so that the state pass starts the longest chains
// first; identity order past kOrderMaxN sequences).  Then the slots, 1024-aligned.
constexpr int kOrderMaxN = 8192;
// Ready words of the one-launch form: one per (chunk, head) item, head-major with
// each head's row padded to a multiple of 8 words (32 bytes), so that eight
// consecutive chunks of a head are read by two aligned 16-byte loads.
__host__ __device__ inline int ready_stride(int chunks) { return (chunks + 7) & ~7; }
__host__ __device__ inline uint32_t header_bytes(int N) {
    return (uint32_t)(((size_t)(N + 1) * 16 + 1023) & ~(size_t)1023);
}

// ======================================================================
// chunk table (one block of 1024 threads)
// ======================================================================
__global__ void __launch_bounds__(1024)
chunk_table_kernel(const int32_t *__restrict__ cu, int64_t T, int N, int64_t ckpt_interval,
                   int32_t *__restrict__ hdr) {
    __shared__ int64_t part[1024];
    int32_t *chunk_off = hdr;
    int32_t *bound = hdr + (N + 1);
    int32_t *ckpt_off = hdr + 2 * (N + 1);
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
    // chunks and intermediate states per sequence, exclusive sums
    auto seqlen = [&](int n) -> int64_t { return cu ? (int64_t)bound[n + 1] - bound[n] : T; };
    auto nchunks = [&](int n) -> int64_t { return (seqlen(n) + C - 1) / C; };
    auto nckpt = [&](int n) -> int64_t {   // states after m * interval tokens, m >= 1, inside
        const int64_t len = seqlen(n);
        return (ckpt_interval > 0 && len > 0) ? (len - 1) / ckpt_interval : 0;
    };
    const int pn = (N + nt - 1) / nt;
    const int n0 = tid * pn, n1 = min(N, n0 + pn);
    auto exclusive_sum = [&](auto count, int32_t *out) {
        int64_t sum = 0;
        for (int n = n0; n < n1; ++n) sum += count(n);
        part[tid] = sum;
        __syncthreads();
        if (tid == 0) {
            int64_t acc = 0;
            for (int i = 0; i < nt; ++i) {
                const int64_t v = part[i];
                part[i] = acc;
                acc += v;
            }
            out[N] = (int32_t)acc;
        }
        __syncthreads();
        int64_t acc = part[tid];
        for (int n = n0; n < n1; ++n) {
            out[n] = (int32_t)acc;
            acc += count(n);
        }
        __syncthreads();
    };
    exclusive_sum(nchunks, chunk_off);
    exclusive_sum(nckpt, ckpt_off);
    // longest first: the rank of sequence n among all by (chunk count descending,
    // index ascending) is its position in the order (a strict total order)
    int32_t *order = hdr + 3 * (N + 1);
    for (int n = tid; n < N; n += nt) {
        if (N > kOrderMaxN) {
            order[n] = n;
            continue;
        }
        const int32_t cn = chunk_off[n + 1] - chunk_off[n];
        int rank = 0;
        for (int m = 0; m < N; ++m) {
            const int32_t cm = chunk_off[m + 1] - chunk_off[m];
            rank += (cm > cn || (cm == cn && m < n)) ? 1 : 0;
        }
        order[rank] = n;
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

// eight fp16 -> fp32
__device__ __forceinline__ void unpack8h(uint4 u, float (&x)[8]) {
    const __half2 *p = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
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
//   E1[r] = exp(G_r - R_a(r))    in [e^-80, 1]   (one exp per element)
// and per-channel block factors
//   F_m   = exp(R_{m+1} - R_m)   (the decay of block m, <= 1), m = 0, 1, 2
//   EL[a] = exp(G_L - R_a)       (<= 1 for every block holding a valid row)
// as
//   Gamma_r         = E1[r] * prod_{m < a(r)} F_m
//   exp(G_L - G_s)  = EL[a(s)] / E1[s]
//   exp(R_a - G_s)  = (prod_{m = b(s)}^{a-1} F_m) / E1[s]       (a >= b(s))
// Each product is of factors that are all <= 1, or of one factor <= 1 and
// 1/E1 <= e^80 whose product is <= 1, so nothing overflows, and a factor
// underflows only where the exact value is itself negligible.
//
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t A_E1 = 0;          // fp32 [64][128] E1                           32 KiB
constexpr uint32_t A_MISC = 32768;    // beta, F, EL, Gamma_L, barriers, TMEM address  5 KiB
constexpr uint32_t A_M_BETA = 0;      //   fp32 [64]
constexpr uint32_t A_M_F = 256;       //   fp32 [3][128]
constexpr uint32_t A_M_EL = 1792;     //   fp32 [4][128]
constexpr uint32_t A_M_PF = 3840;     //   fp32 [2][128]: F_0 F_1 and F_0 F_1 F_2
constexpr uint32_t A_M_BARS = 4864;   //   8 mbarriers
constexpr uint32_t A_M_TMEM = 4928;   //   TMEM base address + abort flag
constexpr uint32_t A_M_NEXT = 4936;   //   next item (from the device counter)
constexpr uint32_t A_M_END = 4940;
constexpr uint32_t A_OPS = 37888;     // operand region (two uses, below)
static_assert(A_MISC + A_M_END <= A_OPS, "phase A misc region overflows into the operands");
static_assert(A_M_BARS % 8 == 0 && A_M_F % 16 == 0 && A_M_EL % 16 == 0 && A_M_PF % 16 == 0,
              "misc alignment");
// before the Akk/Aqk MMAs: two buffers of one 32-channel round (tf32, K-major SW128)
constexpr uint32_t A_RBUF = 36864;            // bytes per round buffer
constexpr uint32_t A_BT = 0;                  //   + [Q'_a; K'_a], 128 rows x 128 B    16 KiB
constexpr uint32_t A_AT = 16384;              //   + packed K^(a), 160 rows x 128 B    20 KiB
// after them:
constexpr uint32_t A_AK = A_OPS;              // fp32 [64][64] Akk, then X in place    16 KiB
constexpr uint32_t A_AQ = A_OPS + 16384;      // fp16 Aqk, MN-major SW128 64x64         8 KiB
constexpr uint32_t A_TR = A_OPS + 24576;      // fp16 [T; R], K-major SW128 128x64     16 KiB
constexpr uint32_t A_KT = A_OPS + 40960;      // fp16 K*Gamma, MN-major SW128          16 KiB
constexpr uint32_t A_Y = A_OPS + 57344;       // fp32 solve scratch (32 x 32)               4 KiB
// next item's rows, loaded by TMA as soon as D1 has completed: the regions of AK (dead
// after the solve), K*Gamma (dead after D1) and the solve scratch with the tail; none
// overlaps [T; R], which a bulk store may still be reading.  Each tile is the TMA box
// layout of stage_off(): two 64-channel blocks of 64 rows x 128 B.
constexpr uint32_t A_QST = A_AK;              // bf16 q [64][128]                            16 KiB
constexpr uint32_t A_KST = A_KT;              // bf16 k                                      16 KiB
constexpr uint32_t A_GST = A_Y;               // bf16 g                                      16 KiB
// A0 scratch (block sums, G_L), in the Aqk region (free until A2)
constexpr uint32_t A_A0S = A_AQ;
constexpr uint32_t A_SMEM = A_OPS + 2 * A_RBUF + 1024;   // + alignment slack (= 112640)
static_assert(A_Y + 4096 <= A_OPS + 2 * A_RBUF, "phase A post-MMA region overflows");
static_assert(A_GST + 16384 <= A_OPS + 2 * A_RBUF, "staging area");
static_assert((A_QST >= A_TR + 16384 || A_QST + 16384 <= A_TR) && (A_KST >= A_TR + 16384 || A_KST + 16384 <= A_TR) &&
              (A_GST >= A_TR + 16384 || A_GST + 16384 <= A_TR), "staging must not overlap [T; R]");
static_assert(3 * 128 * 4 + 128 * 4 <= 8192, "A0 scratch (tot, G_L) fits the Aqk region");
static_assert(A_OPS % 1024 == 0 && A_RBUF % 1024 == 0 && A_AQ % 1024 == 0 && A_TR % 1024 == 0 &&
              A_KT % 1024 == 0, "swizzled tiles need 1024-byte alignment");
// E1 is stored [64][128] fp32 with its 16-byte pieces (4 channels) permuted per
// row: piece p of row r sits at p ^ (r % 32).  Reads of the same channels in
// consecutive rows (one row per lane) then spread over all banks.
__device__ __forceinline__ int e1_at(int row, int col4) {   // col4: multiple of 4
    return row * 128 + (((col4 >> 2) ^ (row & 31)) << 2);
}
// Byte offset of (row, channel) in a staged [64][128] bf16 input tile as the TMA
// box loads land: channels [0, 64) and [64, 128) in two blocks 8 KiB apart, each
// 64 lines of 128 B with the 128-byte swizzle (16-byte piece index XOR row % 8).
__device__ __forceinline__ uint32_t stage_off(int row, int ch) {
    return (uint32_t)((ch >> 6) * 8192 + row * 128 + ((((ch & 63) >> 3) ^ (row & 7)) << 4) +
                      (ch & 7) * 2);
}
// first row-group of the packed K^(a) tile: 0, 2, 6, 12
__device__ __forceinline__ int at_group(int a) { return a * (a + 1); }

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {   // two packed f32x2 multiplies
    const float2 lo = __fmul2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fmul2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 bf4(uint2 u) {   // four bf16 -> fp32
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(f0.x, f0.y, f1.x, f1.y);
}
// round to tf32 (nearest, ties away from zero) for a tf32 MMA operand: add half an
// ulp of the 10-bit significand to the magnitude; the tensor core reads only the
// 19 high bits of each 32-bit operand, which completes the rounding (finite
// inputs far from the fp32 maximum only)
__device__ __forceinline__ float tf32r(float x) {
    return __uint_as_float(__float_as_uint(x) + 0x1000u);
}
__device__ __forceinline__ float4 tf4(float4 a) {
    return make_float4(tf32r(a.x), tf32r(a.y), tf32r(a.z), tf32r(a.w));
}
// approximate reciprocal (about 1 ulp): enough for operands rounded to tf32/fp16 next
__device__ __forceinline__ float rcpa(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float4 rcp4(float4 a) {
    return make_float4(rcpa(a.x), rcpa(a.y), rcpa(a.z), rcpa(a.w));
}

// PREP: the input-preprocessing variant (flags at run time); the plain variant
// compiles without any of it.
// q, k and g arrive as TMA tiles (tensor maps over [rows, H, 128] bf16, boxes of
// 64 channels x 64 rows); beta is read per row.
//
// The body runs in two kernels.  cta and ncta are this CTA's index among the
// CTAs that run phase A and their number.  sched == nullptr: the CTA takes
// items cta, cta + ncta, ...; otherwise each item comes from the device counter
// *sched (zero before the launch), so items go out in increasing order, chunk
// by chunk, to whichever CTA is free.  ready != nullptr: once an item's slot is
// complete in device memory it is published by a release store of the launch's
// epoch into ready[item].
template <bool PREP>
__device__ __forceinline__ void intra_chunk_body(
    const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_g,
    const __nv_bfloat16 *__restrict__ beta, const int32_t *__restrict__ cu, int64_t T, int N, int H,
    uint32_t flags, uint8_t *__restrict__ ws, uint32_t *err, uint32_t epoch, uint8_t *sm, int cta,
    int ncta, uint32_t *sched, uint32_t *ready) {
    const uint32_t sbase = smem_u32(sm);
    float *E1 = reinterpret_cast<float *>(sm + A_E1);
    float *bs = reinterpret_cast<float *>(sm + A_MISC + A_M_BETA);    // [64]
    float *Fb = reinterpret_cast<float *>(sm + A_MISC + A_M_F);       // [3][128] block decays F_m
    float *EL = reinterpret_cast<float *>(sm + A_MISC + A_M_EL);      // [4][128]
    float *PF = reinterpret_cast<float *>(sm + A_MISC + A_M_PF);      // [2][128] F_0 F_1 (F_2)
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + A_MISC + A_M_BARS);   // [8]
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(sm + A_MISC + A_M_TMEM);
    volatile uint32_t *abort_flag = tmem_ptr + 1;
    volatile int *s_next = reinterpret_cast<volatile int *>(sm + A_MISC + A_M_NEXT);
    // used only inside A0, before any operand round: parked in the operand region
    float *tot = reinterpret_cast<float *>(sm + A_A0S);              // [3][128] half sums
    float *GLv = tot + 3 * 128;                                       // [128] G_L
    float *AK = reinterpret_cast<float *>(sm + A_AK);
    float *Yb = reinterpret_cast<float *>(sm + A_Y);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t *chunk_off = reinterpret_cast<const int32_t *>(ws);
    // items are (chunk, head) pairs, item = chunk * H + head, which is also the
    // index of the item's workspace slot
    const int64_t cps = (T + C - 1) / C;
    const int64_t n_items = (cu == nullptr ? (int64_t)N * cps : (int64_t)chunk_off[N]) * H;
    // first row and length of an item's chunk
    auto locate = [&](int64_t item, int64_t &t0_, int &L_) {
        const int64_t cidx = item / H;
        if (cu == nullptr) {
            // equal-length batch: chunk -> (sequence, start) by arithmetic, no table read
            const int64_t n = cidx / cps, j = cidx - n * cps;
            t0_ = n * T + j * C;
            L_ = (int)((T - j * C) < C ? (T - j * C) : C);
        } else {
            // sequence owning this chunk: last n with chunk_off[n] <= cidx
            int lo = 0, hi = N - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (chunk_off[mid] <= cidx) lo = mid; else hi = mid - 1;
            }
            int64_t ra, rb;
            seq_rows(chunk_off, true, T, N, lo, ra, rb);
            t0_ = ra + (cidx - chunk_off[lo]) * C;
            L_ = (int)((rb - t0_) < C ? (rb - t0_) : C);
        }
    };

    // round task: lane -> 4-channel piece p_l of the round and two token rows, one
    // in the first and one in the second half of the chunk, paired so that every
    // warp writes the same number of packed K^(a) copies (rows of block b have
    // 4 - b of them): warps 0-3 take blocks 0 and 3, warps 4-7 blocks 1 and 2
    const int p_l = lane & 7, rsub = lane >> 3;
    auto a1_row = [&](int it) { return it == 0 ? 4 * warp + rsub : 32 + 4 * (warp ^ 4) + rsub; };

    // Next item's q, k, g rows go to the staging area as six TMA boxes (one thread
    // issues them; their bytes complete bars[6]) while the current item finishes;
    // beta into a register.  Rows past the chunk's end are zeroed once the tiles
    // have landed (the boxes read the next rows of the tensor there, or zeros past
    // its end).
    __nv_bfloat16 bnext = __float2bfloat16(0.f);   // raw: converted where it is used
    int loads_issued = 0, items_done = 0;   // tile loads issued / consumed by this CTA
    auto prefetch = [&](int64_t item) {
        int64_t t0n;
        int Ln;
        locate(item, t0n, Ln);
        const int hn = (int)(item % H);
        if (tid == 0) {
            fence_async_smem();   // earlier generic writes to the staging regions come first
            mbar_arrive_expect_tx(&bars[6], 3 * 16384);
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                tma_load_3d(sm + A_QST + blk * 8192, tm_q, 64 * blk, hn, (int)t0n, &bars[6]);
                tma_load_3d(sm + A_KST + blk * 8192, tm_k, 64 * blk, hn, (int)t0n, &bars[6]);
                tma_load_3d(sm + A_GST + blk * 8192, tm_g, 64 * blk, hn, (int)t0n, &bars[6]);
            }
        }
        ++loads_issued;
        bnext = (tid < Ln) ? beta[(size_t)(t0n + (tid < 64 ? tid : 0)) * H + hn] : __float2bfloat16(0.f);
    };

    if (warp == 0) {
        tmem_alloc(tmem_ptr, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 4);   // operand rounds: four issuers
        for (int i = 4; i < 8; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        *abort_flag = 0u;
        *s_next = sched ? (int)atomicAdd(sched, 1u) : cta;
    }
    __syncthreads();
    const int first_item = *s_next;
    if ((int64_t)first_item < n_items) prefetch(first_item);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    // publish a finished item: the slot's generic stores (all threads, ordered by
    // the CTA barrier before this call) and this thread's bulk store of [T; R]
    // are complete before the release store of the epoch
    auto publish = [&](int it) {
        bulk_wait_all();
        fence_proxy_async_global();
        st_release_gpu(ready + (size_t)(it % H) * ready_stride((int)(n_items / H)) + it / H, epoch);
    };
    uint32_t ph = 0;   // mbarrier phase parity: each barrier completes once per item
    int prev_item = -1, next_item = 0;
    // (items fit in int32: the host checks max_chunks * H against INT32_MAX)
    for (int item = first_item; item < (int)n_items; item = next_item, ph ^= 1u) {
    int64_t t0;
    int L;
    locate(item, t0, L);
    uint8_t *slot = ws + header_bytes(N) + (size_t)item * kSlotBytes;
    // the next item from the counter (its value is needed only after a barrier)
    const int claimed = (sched && tid == 0) ? (int)atomicAdd(sched, 1u) : 0;

    // ---- this item's rows have landed; rows past the chunk's end are zeroed
    const bool landed = mbar_wait_abortable(&bars[6], ph, err, epoch, abort_flag);
    if (landed) ++items_done;
    if (landed && L < C) {
        for (int task = tid; task < (C - L) * 3 * 2; task += 256) {
            const int r = L + task / 6, which = task % 6;
            const uint32_t base = (which >> 1) == 0 ? A_QST : ((which >> 1) == 1 ? A_KST : A_GST);
            uint4 *line = reinterpret_cast<uint4 *>(sm + base + (which & 1) * 8192 + r * 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) line[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    if (__syncthreads_or(*abort_flag != 0u)) break;
    if (ready && tid == 0 && prev_item >= 0) publish(prev_item);
    // one launch: a phase A CTA on an SM that also runs a state-pass chain pauses
    // between items (its other threads wait at the barrier below), leaving the
    // SM's issue slots, shared memory and TMEM to the chain, which bounds the
    // launch (the SMs that run chains are marked in the scheduler area).  Not
    // with preprocessing inside: its longer items make phase A the bound.
    if (!PREP && sched && tid == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        if ((smid >> 5) < 8u &&
            ((*reinterpret_cast<volatile const uint32_t *>(sched + 8 + (smid >> 5)) >> (smid & 31)) & 1u))
            __nanosleep(kChainYieldNs);
    }
    prev_item = item;
    const int c = tid & 127, half = tid >> 7;
    float p[32];   // clamped log-decay of rows 32*half + i, then its prefix sums
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x = __bfloat162float(
            *reinterpret_cast<const __nv_bfloat16 *>(sm + A_GST + stage_off(half * 32 + i, c)));
        // gate from a logit: g = -5 sigmoid(x), inside (-5, 0) by construction.  Rows
        // past the chunk's end decay by nothing (their staged x is 0, which the
        // gate would map to -2.5): the block factors and EL then stay <= 1.
        if (PREP) {
            const float gv = (flags & KDA_PREP_GATE_LOGIT) ? -5.f / (1.f + __expf(-x)) : fmaxf(x, -5.f);
            p[i] = (half * 32 + i < L) ? gv : 0.f;
        } else {
            p[i] = fmaxf(x, -5.f);   // rows past the end are staged as zero
        }
    }
    if (tid < 64) bs[tid] = __bfloat162float(bnext);
    if (tid == 0) *s_next = sched ? claimed : item + ncta;
    __syncthreads();
    // the g staging is free now: it holds 1 / |q_r| and 1 / |k_r| when q, k are to be
    // normalised here (two threads per row; a zero row stays zero)
    float *inv_norm = reinterpret_cast<float *>(sm + A_GST);   // [2][64]: q rows, then k rows
    if (PREP && (flags & KDA_PREP_L2NORM_QK)) {
        const int which = tid >> 7, row = (tid >> 1) & 63, hf = tid & 1;
        const uint8_t *src = sm + (which ? A_KST : A_QST);
        float ss = 0.f;
#pragma unroll
        for (int pc = 8 * hf; pc < 8 * hf + 8; ++pc) {
            float x[8];
            unpack8(*reinterpret_cast<const uint4 *>(src + stage_off(row, pc * 8)), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (hf == 0) inv_norm[which * 64 + row] = ss > 0.f ? rsqrtf(ss) : 0.f;
    }

    // ---- A0: chunk-local cumsum (fp32) and E1 = exp(G - R_a), per channel c and half
    // G_r - R_a(r) = p_i for the first 16 rows of a half and p_i - p_15 for the
    // last 16 (R of the half's first block is the base the half starts from).
#pragma unroll
    for (int i = 1; i < 32; ++i) p[i] += p[i - 1];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x = i < 16 ? p[i] : p[i] - p[15];
        E1[e1_at(half * 32 + i, c & ~3) + (c & 3)] = __expf(x);
    }
    if (half == 0) {
        tot[c] = p[31];
        tot[128 + c] = p[15];
        Fb[c] = __expf(p[15]);                 // F_0
        Fb[128 + c] = __expf(p[31] - p[15]);   // F_1
    } else {
        tot[256 + c] = p[15];
        Fb[256 + c] = __expf(p[15]);           // F_2
    }
    __syncthreads();
    {
        // G_L: the owner half of row L-1 writes it
        const int lr = L - 1;
        if (lr >= 0 && (lr >> 5) == half) {
            const float base = half ? tot[c] : 0.f;
            // multiply-add selection keeps p[] in registers (no indexed access)
            const int li = lr & 31;
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) v = fmaf(i == li ? 1.f : 0.f, p[i], v);
            GLv[c] = base + v;
        }
        if (L <= 0 && half == 0) GLv[c] = 0.f;
    }
    __syncthreads();
    if (tid < 128) {
        const float gl = GLv[c];
        const float r1 = tot[128 + c], r2 = tot[c], r3 = tot[c] + tot[256 + c];
        EL[c] = __expf(gl);
        EL[128 + c] = __expf(gl - r1);
        EL[256 + c] = __expf(gl - r2);
        EL[384 + c] = __expf(gl - r3);
        PF[c] = Fb[c] * Fb[128 + c];
        PF[128 + c] = PF[c] * Fb[256 + c];
    }
    // q, k of the operand rounds into registers; the staging area is free after the barrier
    float qn[2] = {1.f, 1.f}, kn[2] = {1.f, 1.f};   // row scales (normalisation)
    if (PREP && (flags & KDA_PREP_L2NORM_QK)) {
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            qn[it] = inv_norm[a1_row(it)];
            kn[it] = inv_norm[64 + a1_row(it)];
        }
    }
    uint2 qv[4][2], kv[4][2];
#pragma unroll
    for (int rd = 0; rd < 4; ++rd)
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int r = a1_row(it);
            const int c0 = 32 * rd + 4 * p_l;   // four channels: one 8-byte half of a 16-byte piece
            const uint32_t sw = stage_off(r, c0);
            qv[rd][it] = *reinterpret_cast<const uint2 *>(sm + A_QST + sw);
            kv[rd][it] = *reinterpret_cast<const uint2 *>(sm + A_KST + sw);
        }
    // the previous item's bulk store of [T; R] has read its source before the
    // operand rounds below overwrite that region
    if (tid == 0) bulk_wait_read();
    __syncthreads();

    // ---- A1: Akk / Aqk on tensor cores (tf32), four double-buffered rounds of 32 channels.
    // B tile row 32a + i      = q_r E1[r]      (r = 16a + i)
    //        row 32a + 16 + i = k_r E1[r]
    // A tile (packed from row-group at_group(a)) row s, s <= 16a+15:
    //        k_s exp(R_a - G_s) = k_s (prod_{m=b(s)}^{a-1} F_m) / E1[s]
    // D^(a) = K^(a) [Q'_a; K'_a]^T (M=64 rows s, N=32) accumulates in TMEM columns 32a.
    bool ok = true;
#pragma unroll
    for (int rd = 0; rd < 4; ++rd) {
        const uint32_t buf = A_OPS + (rd & 1) * A_RBUF;
        if (rd >= 2 && ok) ok = mbar_wait_abortable(&bars[rd - 2], ph, err, epoch, abort_flag);
        if (ok) {
            const int c0 = 32 * rd + 4 * p_l;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int r = a1_row(it);
                const int a = r >> 4, i = r & 15;
                // every row this task writes is congruent to r mod 8: one swizzled chunk offset
                const uint32_t co = (r & 7) * 128 + ((p_l ^ (r & 7)) << 4);
                uint8_t *bt = sm + buf + A_BT + co, *at = sm + buf + A_AT + co;
                float *e1p = E1 + e1_at(r, c0);
                const float4 e = ld4(e1p);
                float4 qf = bf4(qv[rd][it]), kf = bf4(kv[rd][it]);
                if (PREP && (flags & KDA_PREP_L2NORM_QK)) {
                    qf = make_float4(qf.x * qn[it], qf.y * qn[it], qf.z * qn[it], qf.w * qn[it]);
                    kf = make_float4(kf.x * kn[it], kf.y * kn[it], kf.z * kn[it], kf.w * kn[it]);
                }
                const float4 qe = mul4(qf, e), ke = mul4(kf, e);
                *reinterpret_cast<float4 *>(bt + ((32 * a + i) >> 3) * 1024) = tf4(qe);
                *reinterpret_cast<float4 *>(bt + ((32 * a + 16 + i) >> 3) * 1024) = tf4(ke);
                {   // Q*Gamma and K*Gamma = (q, k) E1 prod_{m<a} F_m as fp16 pairs (low: Q*Gamma,
                    // high: K*Gamma), in place of this task's E1 values, read by nobody else
                    const float4 pf = a == 0 ? make_float4(1.f, 1.f, 1.f, 1.f)
                                             : ld4((a == 1 ? Fb : PF + (a - 2) * 128) + c0);
                    const float4 qg = mul4(qe, pf), kg = mul4(ke, pf);
                    __half2 p0 = __floats2half2_rn(qg.x, kg.x), p1 = __floats2half2_rn(qg.y, kg.y);
                    __half2 p2 = __floats2half2_rn(qg.z, kg.z), p3 = __floats2half2_rn(qg.w, kg.w);
                    *reinterpret_cast<uint4 *>(e1p) =
                        make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                                   *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
                }
                float4 ki = mul4(kf, rcp4(e));
                *reinterpret_cast<float4 *>(at + ((8 * at_group(a) + r) >> 3) * 1024) = tf4(ki);
                {   // Khat = k EL / E1 straight to the slot (fp16, MN-major, 4 channels)
                    const float4 kh = mul4(ki, ld4(EL + a * 128 + c0));
                    __half2 h0 = __floats2half2_rn(kh.x, kh.y), h1 = __floats2half2_rn(kh.z, kh.w);
                    *reinterpret_cast<uint2 *>(slot + kSlotKh + sw128_mnmajor_off(c0, r, kKhMNBlock)) =
                        make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
                }
                for (int a2 = a + 1; a2 < 4; ++a2) {
                    ki = mul4(ki, ld4(Fb + (a2 - 1) * 128 + c0));
                    *reinterpret_cast<float4 *>(at + ((8 * at_group(a2) + r) >> 3) * 1024) = tf4(ki);
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        tc_fence_after();
        // row block a's chain is issued by lane 0 of warp 2a: a tcgen05.mma costs
        // its issuing thread tens of cycles, so four issuers keep that off any
        // one warp's path (each commits; the round's barrier counts four)
        if (ok && lane == 0 && (warp & 1) == 0) {
            const int a = warp >> 1;
            // descriptors advance by their start-address field (address / 16)
            const uint64_t ad0 = smem_desc(sbase + buf + A_AT + at_group(a) * 1024, 16, 1024, SW_128B);
            const uint64_t bd0 = smem_desc(sbase + buf + A_BT + 4 * a * 1024, 16, 1024, SW_128B);
            const uint32_t id = idesc(FMT_TF32, 64, 32, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)            // 4 steps of K=8 over 32 channels
                mma_tf32(tmem + 32 * a, ad0 + (uint64_t)((kk * 32) >> 4), bd0 + (uint64_t)((kk * 32) >> 4),
                         id, (rd > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars[rd]);
        }
    }
    if (ok) ok = mbar_wait_abortable(&bars[3], ph, err, epoch, abort_flag);
    tc_fence_after();

    // ---- A2: K*Gamma (the high halves of the packed pairs) into the MN-major B operand of
    // W = T (K*Gamma)
    if (ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int task = tid + 256 * i, s = task >> 4, cc = (task & 15) * 8;
            const uint4 u0 = *reinterpret_cast<const uint4 *>(E1 + e1_at(s, cc));
            const uint4 u1 = *reinterpret_cast<const uint4 *>(E1 + e1_at(s, cc + 4));
            const uint4 kg = make_uint4(__byte_perm(u0.x, u0.y, 0x7632), __byte_perm(u0.z, u0.w, 0x7632),
                                        __byte_perm(u1.x, u1.y, 0x7632), __byte_perm(u1.z, u1.w, 0x7632));
            *reinterpret_cast<uint4 *>(sm + A_KT + sw128_mnmajor_off(cc, s, kKhMNBlock)) = kg;
        }
    }
    // and Akk (fp32, beta applied, strictly lower) and Aqk (fp16, lower incl. diagonal,
    // MN-major: element (r, s) at (mn = r, k = s), so a thread's 16 rows are 32 contiguous
    // bytes) out of TMEM.  Warps w and w + 4 share TMEM lanes 32 (w % 4) ...; the first
    // takes row blocks a = 0, 1 and the second a = 2, 3.
    if (ok) {
        const int quad = warp & 3, s = 16 * quad + (lane & 15);
        const int a0 = 2 * (warp >> 2);
        for (int a = a0; a < a0 + 2; ++a) {
            float vq[16], vk[16];
            tmem_ld16(taddr(tmem, 32 * quad, 32 * a), vq);
            tmem_ld16(taddr(tmem, 32 * quad, 32 * a + 16), vk);
            tmem_wait_ld();
            if (lane < 16) {
                float y0[8], y1[8];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    // (rows r >= L are zero already: their q, k and beta are zero)
                    const int r = 16 * a + j;
                    AK[r * 64 + s] = s < r ? bs[r] * vk[j] : 0.f;
                    const float aq = s <= r ? vq[j] : 0.f;
                    if (j < 8) y0[j] = aq; else y1[j - 8] = aq;
                }
                *reinterpret_cast<uint4 *>(sm + A_AQ + sw128_mnmajor_off(16 * a, s, 0)) = pack8(y0);
                *reinterpret_cast<uint4 *>(sm + A_AQ + sw128_mnmajor_off(16 * a + 8, s, 0)) =
                    pack8(y1);
            }
        }
    }
    tc_fence_before();
    __syncthreads();


    // ---- A3: X = (I + Akk)^-1 in place over AK (fp32), by 2x2 block merges:
    //   inv([[L11, 0], [L21, L22]]) = [[X11, 0], [-X22 (L21 X11), X22]]
    // 16x16 diagonal blocks by forward substitution, then two merges 16 -> 32
    // (in parallel), then one merge 32 -> 64.  The strictly upper part of AK is
    // zero throughout.  (Every __syncthreads below is reached by all threads.)
    {
        float x[16];
        const int a = tid >> 4, j = tid & 15, o = 16 * a;
        if (ok && tid >= 128) reinterpret_cast<float *>(slot + kSlotGam)[tid - 128] = EL[tid - 128];
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
    // merge 16 -> 32 for diagonal pairs p = 0, 1 (rows/cols 32p .. 32p+31):
    //   Y = A_{2p+1,2p} X_{2p,2p};  X_{2p+1,2p} = -X_{2p+1,2p+1} Y
    // thread: pair pr, column j, rows i and i + 8 (row operands as float4, the
    // column operand shared by both rows)
    {
        const int pr = tid >> 7, j = tid & 15, i = (tid >> 4) & 7;
        const int o = 32 * pr;
        const float *r0 = AK + (o + 16 + i) * 64 + o, *r1 = r0 + 8 * 64;
        if (ok) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
                const float4 a0 = ld4(r0 + 4 * t4), a1 = ld4(r1 + 4 * t4);
                const float x0 = AK[(o + 4 * t4) * 64 + o + j], x1 = AK[(o + 4 * t4 + 1) * 64 + o + j];
                const float x2 = AK[(o + 4 * t4 + 2) * 64 + o + j], x3 = AK[(o + 4 * t4 + 3) * 64 + o + j];
                acc0 = fmaf(a0.x, x0, fmaf(a0.y, x1, fmaf(a0.z, x2, fmaf(a0.w, x3, acc0))));
                acc1 = fmaf(a1.x, x0, fmaf(a1.y, x1, fmaf(a1.z, x2, fmaf(a1.w, x3, acc1))));
            }
            Yb[pr * 256 + i * 16 + j] = acc0;
            Yb[pr * 256 + (i + 8) * 16 + j] = acc1;
        }
        __syncthreads();
        if (ok) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
                const float4 a0 = ld4(r0 + 16 + 4 * t4), a1 = ld4(r1 + 16 + 4 * t4);
                const float *yc = Yb + pr * 256 + 64 * t4 + j;
                const float y0 = yc[0], y1 = yc[16], y2 = yc[32], y3 = yc[48];
                acc0 = fmaf(a0.x, y0, fmaf(a0.y, y1, fmaf(a0.z, y2, fmaf(a0.w, y3, acc0))));
                acc1 = fmaf(a1.x, y0, fmaf(a1.y, y1, fmaf(a1.z, y2, fmaf(a1.w, y3, acc1))));
            }
            AK[(o + 16 + i) * 64 + o + j] = -acc0;
            AK[(o + 24 + i) * 64 + o + j] = -acc1;
        }
        __syncthreads();
    }
    // merge 32 -> 64:  Z = A21 X11 (32x32);  X21 = -X22 Z
    // thread (i0 = warp, j = lane) computes rows i0 + 8q, q = 0..3, of column j;
    // the row operands are warp-uniform (broadcast float4 loads), the zero upper
    // triangles make the fixed trip counts exact
    {
        const int j = lane, i0 = warp;
        if (ok) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
                float xv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) xv[u] = AK[(4 * t4 + u) * 64 + j];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const float4 av = ld4(AK + (32 + i0 + 8 * qq) * 64 + 4 * t4);
                    acc[qq] = fmaf(av.x, xv[0], fmaf(av.y, xv[1], fmaf(av.z, xv[2], fmaf(av.w, xv[3], acc[qq]))));
                }
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) Yb[(i0 + 8 * qq) * 32 + j] = acc[qq];
        }
        __syncthreads();
        if (ok) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
                float zv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) zv[u] = Yb[(4 * t4 + u) * 32 + j];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    // X22 is lower triangular: row i0 + 8 qq has no terms past column
                    // i0 + 8 qq (a warp-uniform bound, so whole blocks are skipped)
                    if (t4 <= (i0 >> 2) + 2 * qq) {
                        const float4 av = ld4(AK + (32 + i0 + 8 * qq) * 64 + 32 + 4 * t4);
                        acc[qq] = fmaf(av.x, zv[0], fmaf(av.y, zv[1], fmaf(av.z, zv[2], fmaf(av.w, zv[3], acc[qq]))));
                    }
                }
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) AK[(32 + i0 + 8 * qq) * 64 + j] = -acc[qq];
        }
        __syncthreads();
    }
    // T = X Diag(beta) into rows 0..63 of [T; R] (fp16, K-major SW128)
    if (ok) {
        for (int task = tid; task < 64 * 8; task += 256) {
            const int r = task >> 3, ch = task & 7;
            const float4 xa = ld4(AK + r * 64 + ch * 8), xb = ld4(AK + r * 64 + ch * 8 + 4);
            const float4 ba = ld4(bs + ch * 8), bb = ld4(bs + ch * 8 + 4);
            const float xv[8] = {xa.x * ba.x, xa.y * ba.y, xa.z * ba.z, xa.w * ba.w,
                                 xb.x * bb.x, xb.y * bb.y, xb.z * bb.z, xb.w * bb.w};
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (ch * 8 + e <= r) ? xv[e] : 0.f;
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
    if (ok) ok = mbar_wait_abortable(&bars[4], ph, err, epoch, abort_flag);
    tc_fence_after();
    if (ok && warp < 4) {
        const int r = 16 * warp + (lane & 15);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x[32];
            tmem_ld16(taddr(tmem, 32 * warp, 128 + 32 * hh), *reinterpret_cast<float(*)[16]>(x));
            tmem_ld16(taddr(tmem, 32 * warp, 144 + 32 * hh), *reinterpret_cast<float(*)[16]>(x + 16));
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = x[ch * 8 + e];
                    *reinterpret_cast<uint4 *>(sm + A_TR + sw128_kmajor_off(64 + r, 32 * hh + ch * 8, 0)) =
                        pack8(y);
                }
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
    const int quad = warp & 3, chalf = warp >> 2;
    const int row6 = 32 * quad + lane, r6 = row6 & 63;
    // [T; R] is final: one bulk store to the slot while the MMA runs
    if (ok && tid == 0) {
        bulk_s2g(slot + kSlotTR, sm + A_TR, 16384);
        bulk_commit();
    }
    if (ok) ok = mbar_wait_abortable(&bars[5], ph, err, epoch, abort_flag);
    tc_fence_after();
    // the staging regions are free once D1 has completed: the next item's rows go
    // out now (the bulk store of [T; R] is waited for before the next item's
    // operand rounds overwrite it)
    next_item = *s_next;
    if (ok && (int64_t)next_item < n_items) prefetch(next_item);

    // ---- A6: rows 0..63 -> -W, rows 64..127 -> P = Q*Gamma - R (K*Gamma), in two
    // halves of 32 columns (fewer live registers)
    if (ok) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x[32];
            tmem_ld16(taddr(tmem, 32 * quad, 64 * chalf + 32 * hh), *reinterpret_cast<float(*)[16]>(x));
            tmem_ld16(taddr(tmem, 32 * quad, 64 * chalf + 32 * hh + 16),
                      *reinterpret_cast<float(*)[16]>(x + 16));
            tmem_wait_ld();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float y[8];
                uint4 u;
                if (row6 < 64) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = x[ch * 8 + e];
                    u = pack8(y);
                    u.x ^= 0x80008000u; u.y ^= 0x80008000u;   // -W: flip the fp16 signs
                    u.z ^= 0x80008000u; u.w ^= 0x80008000u;
                } else {
                    const int cc = 8 * (8 * chalf + 4 * hh + ch);
                    // Q*Gamma: the low halves of the packed pairs
                    const uint4 u0 = *reinterpret_cast<const uint4 *>(E1 + e1_at(r6, cc));
                    const uint4 u1 = *reinterpret_cast<const uint4 *>(E1 + e1_at(r6, cc + 4));
                    float qg[8];
                    unpack8h(make_uint4(__byte_perm(u0.x, u0.y, 0x5410), __byte_perm(u0.z, u0.w, 0x5410),
                                        __byte_perm(u1.x, u1.y, 0x5410), __byte_perm(u1.z, u1.w, 0x5410)),
                             qg);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = qg[e] - x[ch * 8 + e];
                    u = pack8(y);
                }
                *reinterpret_cast<uint4 *>(
                    slot + kSlotWP + sw128_kmajor_off(row6, 64 * chalf + 32 * hh + ch * 8, kWPKBlock)) = u;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    }   // item loop
    // a load issued for an item this CTA will not process (the loop left early on an
    // abort) must land before the CTA's shared memory is released (bounded wait)
    if (tid == 0 && loads_issued > items_done)
        mbar_wait(&bars[6], (uint32_t)(items_done & 1), err, 1ull << 28);
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (ready && tid == 0 && prev_item >= 0 && !*abort_flag) publish(prev_item);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <bool PREP>
__global__ void __launch_bounds__(256, 2)
intra_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16 *__restrict__ beta,
                   const int32_t *__restrict__ cu, int64_t T, int N, int H, uint32_t flags,
                   uint8_t *__restrict__ ws, uint32_t *err, uint32_t epoch) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    intra_chunk_body<PREP>(&tm_q, &tm_k, &tm_g, beta, cu, T, N, H, flags, ws, err, epoch, sm,
                           (int)blockIdx.x, (int)gridDim.x, nullptr, nullptr);
}

// ======================================================================
// Phase B
// ======================================================================
template <int DVS>
struct BLayout {
    static constexpr int NST = DVS == 32 ? 3 : 2;              // slot ring depth (smem bound)
    static constexpr uint32_t kVBytes = 64 * DVS * 2;          // V slice tile
    static constexpr uint32_t kStage = kSlotBytes + kVBytes;   // slot image + V
    static constexpr uint32_t kStageR = (kStage + 1023) & ~1023u;
    static constexpr uint32_t kSB = 128 * DVS * 2;             // fp16 S  (K=128 x N=DVS)
    static constexpr uint32_t kUB = 64 * DVS * 2;              // fp16 U  (K=64 x N=DVS)
    static constexpr uint32_t kKGroup = (DVS / 8) * 128;       // k-group stride, interleaved MN-major
    static constexpr uint32_t oSB = NST * kStageR;
    static constexpr uint32_t oUB = oSB + kSB;
    static constexpr uint32_t oBar = oUB + kUB;
    static constexpr uint32_t kBytes = oBar + 256 + 1024;      // + barriers + alignment slack
    static constexpr uint32_t kTmemCols = DVS == 32 ? 128 : (DVS == 64 ? 256 : 512);
    // V slice as its TMA boxes land: 64 rows of DVS channels, MN-major (channel
    // contiguous) with the swizzle that matches the line length: 64-byte lines and
    // the 64-byte swizzle for DVS = 32; 128-byte lines and the 128-byte swizzle
    // otherwise, in 64-channel blocks 8 KiB apart.  These are the canonical UMMA
    // MN-major swizzled layouts of the [T; R] V operand.
    static constexpr uint32_t kVLine = DVS == 32 ? 64 : 128;
    static constexpr Swizzle kVSwz = DVS == 32 ? SW_64B : SW_128B;
    static constexpr uint32_t kVSbo = 8 * kVLine;            // 8-row (k) groups
    static constexpr uint32_t kVLbo = 64 * kVLine;           // 64-channel blocks
    static constexpr uint32_t kVKstep = 16 * kVLine;         // 16 rows: one K step of an MMA
    static_assert(kBytes <= 227 * 1024, "state pass shared memory");
};

enum BBar {
    FULL0 = 0,       // [NST] slot image landed (bulk copy tx)
    EMPTY0 = 3,      // [NST] every MMA reading the stage has completed
    VRAW0 = 6,       // [NST] the producer lanes' cp.async of the V slice have landed
    VREADY0 = 9,     // [NST] V slice converted to fp16 in place
    TDFULL0 = 12, TDFULL1, TDEMPTY0, TDEMPTY1,
    TSSCALED, TSFULL, DRAIN_S, DRAIN_U, NBARS
};
static_assert(NBARS * 8 + 16 <= 256, "phase B barrier area");

__device__ __forceinline__ void named_bar(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Roles (384 threads): warp 0 producer; warp 1 owns the TMEM allocation;
// warps 2-3 convert each V slice from bf16 to fp16 in place; warps 4-7 U/O
// epilogue, whose elected thread (warp 4, lane 0) issues the state update
// S += Khat^T U; warps 8-11 state epilogue, whose elected thread (warp 8,
// lane 0) issues [U; O] = [T; R] V + [-W; P] S.  Every bar.sync below is
// executed by all threads of its group in every iteration (a failed bounded
// wait only skips work), so a timeout can never leave a barrier half-joined.
template <int DVS>
__global__ void __launch_bounds__(384, 1)
state_pass_kernel(const __grid_constant__ CUtensorMap tm_v, const float *state_in,
                  const int32_t *__restrict__ cu, int64_t T, int N, int H,
                  const uint8_t *__restrict__ ws, float *__restrict__ o,
                  float *state_out, int64_t ckpt_interval, float *ckpt, int64_t ckpt_capacity,
                  uint32_t *err, uint32_t epoch) {
    using Lay = BLayout<DVS>;
    constexpr int NSL = D / DVS;
    constexpr int CPR = DVS / 8;   // 16-byte pieces per V row
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::oBar);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + NBARS);
    volatile uint32_t *abort_flag = tmem_ptr + 1;
    volatile uint32_t *s_grp_ok = tmem_ptr + 2;   // elected state thread -> state warps

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = blockIdx.x % NSL;
    const int unit = blockIdx.x / NSL;
    const int32_t *chunk_off = reinterpret_cast<const int32_t *>(ws);
    if (unit / H >= N) return;
    // packed sequences run longest first (order[] from the chunk table)
    const int n = cu ? chunk_off[3 * (N + 1) + unit / H] : unit / H, h = unit % H;
    int64_t ra, rb;
    seq_rows(chunk_off, cu != nullptr, T, N, n, ra, rb);
    const int nch = (int)((rb - ra + C - 1) / C);
    // first chunk of the sequence: from the table for packed sequences, else n chunks
    // of T each (no table is built for equal-length batches)
    const int c0 = cu ? chunk_off[n] : n * (int)((T + C - 1) / C);
    // first intermediate-state entry of the sequence, likewise
    const int64_t ck0 = cu ? (int64_t)chunk_off[2 * (N + 1) + n]
                           : (int64_t)n * ((T > 0 && ckpt_interval > 0) ? (T - 1) / ckpt_interval : 0);
    const uint8_t *slots = ws + header_bytes(N);
    const int j0 = slice * DVS;   // first value channel of this slice

    if (warp == 1) {
        tmem_alloc(tmem_ptr, Lay::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < Lay::NST; ++i) {
            mbar_init(&bars[FULL0 + i], 1);
            mbar_init(&bars[EMPTY0 + i], 1);
            mbar_init(&bars[VRAW0 + i], 1);
            mbar_init(&bars[VREADY0 + i], 1);
        }
        mbar_init(&bars[TDFULL0], 1);
        mbar_init(&bars[TDFULL1], 1);
        mbar_init(&bars[TDEMPTY0], 4);
        mbar_init(&bars[TDEMPTY1], 4);
        mbar_init(&bars[TSSCALED], 1);
        mbar_init(&bars[TSFULL], 1);
        mbar_init(&bars[DRAIN_S], 1);
        mbar_init(&bars[DRAIN_U], 1);
        mbar_fence_init();
        *abort_flag = 0u;
        *s_grp_ok = 1u;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t tTD0 = tmem, tTD1 = tmem + DVS, tTS = tmem + 2 * DVS;
    constexpr int NST = Lay::NST;
    auto stage_addr = [&](int st) { return sbase + st * Lay::kStageR; };
    auto full_par = [&](int j) { return (uint32_t)((j / NST) & 1); };          // FULL[j % NST]
    auto empty_par = [&](int j) { return (uint32_t)(((j / NST) + 1) & 1); };   // EMPTY before reuse
    auto chunk_len = [&](int j) {
        const int64_t t0 = ra + (int64_t)j * C;
        return (int)((rb - t0) < C ? (rb - t0) : C);
    };

    if (warp == 0) {
        // ------------------------------------------------ producer
        // Chunk j's slot image goes in with one bulk copy; its V slice as TMA boxes
        // straight into the operand layout (rows past the chunk's end are zeroed by
        // the converters).  Both complete on mbarriers by their bytes, so nothing
        // here waits for a copy and loads run NST chunks ahead.
        int issued = 0;
        for (int j = 0; j < nch; ++j) {
            const int st = j % NST;
            if (j >= NST &&
                !mbar_wait_abortable(&bars[EMPTY0 + st], empty_par(j), err, epoch, abort_flag))
                break;
            uint8_t *stg = sm + st * Lay::kStageR;
            const uint8_t *src = slots + ((size_t)(c0 + j) * H + h) * kSlotBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[FULL0 + st], kSlotBytes);
                bulk_g2s(stg, src, kSlotBytes, &bars[FULL0 + st]);
                const int t0 = (int)(ra + (int64_t)j * C);
                mbar_arrive_expect_tx(&bars[VRAW0 + st], Lay::kVBytes);
#pragma unroll
                for (int blk = 0; blk < (DVS + 63) / 64; ++blk)
                    tma_load_3d(stg + kSlotBytes + blk * 8192, &tm_v, j0 + 64 * blk, h, t0,
                                &bars[VRAW0 + st]);
            }
            issued = j + 1;
        }
        // drain: never leave the CTA with copies still landing in its shared memory
        for (int j = issued - NST; j < issued; ++j)
            if (j >= 0) {
                mbar_wait(&bars[FULL0 + j % NST], full_par(j), err, 1ull << 28);
                mbar_wait(&bars[VRAW0 + j % NST], full_par(j), err, 1ull << 28);
            }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------ V converters (64 threads)
        // bf16 -> fp16 in place; each 16-byte piece holds 8 values of one row (the
        // swizzle only permutes pieces within a line).  Rows past the chunk's end
        // hold the next rows of the tensor (or zeros past its end): they become 0.
        const int ct = tid - 64;
        bool ok = true;
        for (int j = 0; j < nch; ++j) {
            const int st = j % NST;
            if (ok) ok = mbar_wait_abortable(&bars[VRAW0 + st], full_par(j), err, epoch, abort_flag);
            if (ok) {
                uint8_t *vt = sm + st * Lay::kStageR + kSlotBytes;
                const int L = chunk_len(j);
#pragma unroll
                for (int i = 0; i < CPR; ++i) {
                    const int idx = ct + 64 * i;
                    const int row = ((idx * 16) % 8192) / (int)Lay::kVLine;
                    uint4 *pc = reinterpret_cast<uint4 *>(vt) + idx;
                    if (row < L) {
                        float x[8];
                        unpack8(*pc, x);
                        *pc = pack8(x);
                    } else {
                        *pc = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            fence_async_smem();
            named_bar(3, 64);
            if (ct == 0 && ok) mbar_arrive(&bars[VREADY0 + st]);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ U / O epilogue (+ state-update issue)
        const int quad = warp - 4;
        const int row = 32 * quad + lane;
        // one thread issues the whole state update: its K steps then accumulate in
        // a fixed order and the result is the same on every run
        const bool issuer = (warp == 4 && lane == 0);
        const uint32_t id_mm = idesc(FMT_F16, 128, DVS, 1, 1);   // A MN-major, B MN-major
        bool ok = true;
        for (int j = 0; j < nch; ++j) {
            const int b = j & 1, st = j % NST;
            const uint32_t tTD = b ? tTD1 : tTD0;
            if (ok) ok = mbar_wait_abortable(&bars[TDFULL0 + b], (j >> 1) & 1, err, epoch, abort_flag);
            tc_fence_after();
            const int64_t t0 = ra + (int64_t)j * C;
            const int L = chunk_len(j);
            const int r = row - 64;
            if (ok) {
                float xa[DVS];
#pragma unroll
                for (int p = 0; p < DVS / 16; ++p)
                    tmem_ld16(taddr(tTD, 32 * quad, 16 * p), *reinterpret_cast<float(*)[16]>(xa + 16 * p));
                tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < DVS / 16; ++p) {
                    const float *x = xa + 16 * p;
                    float y0[8], y1[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        y0[e] = x[e];
                        y1[e] = x[8 + e];
                    }
                    if (quad < 2) {
                        // U rows -> fp16 B operand (MN-major, interleaved core matrices)
                        *reinterpret_cast<uint4 *>(
                            sm + Lay::oUB + interleave_mnmajor_off(16 * p, row, Lay::kKGroup)) = pack8(y0);
                        *reinterpret_cast<uint4 *>(
                            sm + Lay::oUB + interleave_mnmajor_off(16 * p + 8, row, Lay::kKGroup)) =
                            pack8(y1);
                    } else if (r < L) {
                        float4 *dst = reinterpret_cast<float4 *>(o + ((size_t)(t0 + r) * H + h) * D +
                                                                 j0 + 16 * p);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
                    }
                }
            }
            if (quad < 2) {
                fence_async_smem();
                named_bar(1, 64);   // both U warps (4 and 5) have written their rows
                if (issuer && ok) {
                    // and the state is scaled by Gamma_j (normally long since)
                    ok = mbar_wait_abortable(&bars[TSSCALED], j & 1, err, epoch, abort_flag);
                    if (ok) {
                        tc_fence_after();
                        // S += Khat^T U   (descriptors advance by their start-address field)
                        const uint64_t ad0 = smem_desc(stage_addr(st) + kSlotKh, kKhMNBlock, 1024, SW_128B);
                        const uint64_t bd0 = smem_desc(sbase + Lay::oUB, Lay::kKGroup, 128, SW_NONE);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(tTS, ad0 + (uint64_t)(kk * 2048 / 16),
                                    bd0 + (uint64_t)(kk * 2 * Lay::kKGroup / 16), id_mm, 1);
                        mma_commit(&bars[TSFULL]);
                        mma_commit(&bars[EMPTY0 + st]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[TDEMPTY0 + b]);
        }
        if (issuer) {
            // every MMA this thread issued has completed before TMEM is released
            mma_commit(&bars[DRAIN_U]);
            mbar_wait(&bars[DRAIN_U], 0, err, 1ull << 28);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------ state epilogue (+ chunk-product issue)
        const int quad = warp - 8;
        const int c = 32 * quad + lane;   // key channel = TMEM lane
        // one thread issues the V and state terms: their K steps then accumulate in a
        // fixed order and the result is the same on every run
        const bool issuer = (warp == 8 && lane == 0);
        const uint32_t tS = taddr(tTS, 32 * quad, 0);
        const size_t srow = (((size_t)n * H + h) * D + c) * D + j0;
        const uint32_t id_nn = idesc(FMT_F16, 128, DVS, 0, 1);   // A K-major, B MN-major
        uint8_t *sbp = sm + Lay::oSB;
        // fp16 copy of S (B operand of the state term) and TS <- Gamma * S (the
        // base the state update accumulates onto), from the fp32 S in xa
        auto put_state = [&](const float *xa, float gam) {
#pragma unroll
            for (int p = 0; p < DVS / 16; ++p) {
                const float *x = xa + 16 * p;
                float y0[8], y1[8], z[16];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    y0[e] = x[e];
                    y1[e] = x[8 + e];
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = x[e] * gam;
                tmem_st16(tS + 16 * p, z);
                *reinterpret_cast<uint4 *>(sbp + interleave_mnmajor_off(16 * p, c, Lay::kKGroup)) =
                    pack8(y0);
                *reinterpret_cast<uint4 *>(sbp + interleave_mnmajor_off(16 * p + 8, c, Lay::kKGroup)) =
                    pack8(y1);
            }
            tmem_wait_st();
        };
        // [T; R]_j V_j into TD[j % 2] (the V term; independent of the state)
        int v_issued = -1;   // highest chunk whose V term has been issued (issuer only)
        auto issue_vterm = [&](int j) {
            const int st = j % NST;
            const uint32_t tTD = (j & 1) ? tTD1 : tTD0;
            const uint64_t ad0 = smem_desc(stage_addr(st) + kSlotTR, 16, 1024, SW_128B);
            const uint64_t bd0 =
                smem_desc(stage_addr(st) + kSlotBytes, Lay::kVLbo, Lay::kVSbo, Lay::kVSwz);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tTD, ad0 + (uint64_t)(kk * 32 / 16),
                        bd0 + (uint64_t)(kk * Lay::kVKstep / 16), id_nn, kk > 0);
            v_issued = j;
        };
        auto vterm_ready = [&](int j) {   // one poll: slot, V slice and accumulator free
            return mbar_try_wait(&bars[FULL0 + j % NST], full_par(j)) &&
                   mbar_try_wait(&bars[VREADY0 + j % NST], full_par(j)) &&
                   (j < 2 || mbar_try_wait(&bars[TDEMPTY0 + (j & 1)], ((j >> 1) + 1) & 1));
        };
        // After the fp16 copy of S_j and the scaled TS are in place: the elected
        // thread releases the state update of chunk j (TSSCALED), issues
        // [U; O]_j = [T; R]_j V_j + [-W; P]_j S_j into TD[j % 2] and tells the
        // group whether it succeeded.  When the next chunk's slot, V slice and
        // accumulator are already free it also issues that chunk's V term: the
        // pipe then runs it while the U warps copy U out, and only the state
        // term remains on the chunk-to-chunk path.
        // (ok_in: the elected thread's own status; the group status travels in
        // s_grp_ok, written only between the two barriers below)
        auto issue_chunk = [&](int j, bool ok_in) {
            const int st = j % NST, b = j & 1;
            fence_async_smem();
            tc_fence_before();
            named_bar(2, 128);
            if (issuer) {
                bool okk = ok_in;
                if (okk) mbar_arrive(&bars[TSSCALED]);
                if (okk && v_issued < j) {
                    okk = mbar_wait_abortable(&bars[FULL0 + st], full_par(j), err, epoch, abort_flag);
                    if (okk) okk = mbar_wait_abortable(&bars[VREADY0 + st], full_par(j), err, epoch, abort_flag);
                    if (okk && j >= 2)
                        okk = mbar_wait_abortable(&bars[TDEMPTY0 + b], ((j >> 1) + 1) & 1, err,
                                                  epoch, abort_flag);
                    if (okk) {
                        tc_fence_after();
                        issue_vterm(j);
                    }
                }
                if (okk) {
                    tc_fence_after();
                    const uint32_t tTD = b ? tTD1 : tTD0;
                    const uint64_t ad0 = smem_desc(stage_addr(st) + kSlotWP, 16, 1024, SW_128B);
                    const uint64_t bd0 = smem_desc(sbase + Lay::oSB, Lay::kKGroup, 128, SW_NONE);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16(tTD, ad0 + (uint64_t)(((kk >> 2) * kWPKBlock + (kk & 3) * 32) / 16),
                                bd0 + (uint64_t)(kk * 2 * Lay::kKGroup / 16), id_nn, 1);
                    mma_commit(&bars[TDFULL0 + b]);
                    // early V term of chunk j + 1, only if nothing has to be waited for
                    const int jn = j + 1;
                    if (jn < nch && vterm_ready(jn)) {
                        tc_fence_after();
                        issue_vterm(jn);
                    }
                }
                *s_grp_ok = okk ? 1u : 0u;
            }
            named_bar(2, 128);
            return *s_grp_ok != 0u;
        };
        auto gamma_of = [&](int j, bool &ok) {
            if (ok) ok = mbar_wait_abortable(&bars[FULL0 + j % NST], full_par(j), err, epoch, abort_flag);
            return ok ? reinterpret_cast<const float *>(sm + (j % NST) * Lay::kStageR + kSlotGam)[c]
                      : 0.f;
        };
        if (nch == 0) {
            // empty sequence: the state passes through unchanged
            if (state_out)
                for (int i = 0; i < DVS / 4; ++i)
                    reinterpret_cast<float4 *>(state_out + srow)[i] =
                        state_in ? reinterpret_cast<const float4 *>(state_in + srow)[i]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            bool ok = true;
            // xa = S_j in registers (fp32).  Per chunk: S_j -> fp16 copy and
            // TS = Gamma_j S_j, the chunk products are issued, and the state
            // update S_{j+1} = TS + Khat_j^T U_j lands in TS.
            float xa[DVS];
            for (int p = 0; p < DVS / 16; ++p)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = state_in
                        ? reinterpret_cast<const float4 *>(state_in + srow)[4 * p + i]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    xa[16 * p + 4 * i] = f.x; xa[16 * p + 4 * i + 1] = f.y;
                    xa[16 * p + 4 * i + 2] = f.z; xa[16 * p + 4 * i + 3] = f.w;
                }
            {
                const float gam = gamma_of(0, ok);
                if (ok) put_state(xa, gam);
                ok = issue_chunk(0, ok) && ok;
            }
            for (int j = 0; j < nch; ++j) {
                // S_{j+1} = TS after the state update of chunk j
                if (ok) ok = mbar_wait_abortable(&bars[TSFULL], j & 1, err, epoch, abort_flag);
                tc_fence_after();
                if (ok) {
#pragma unroll
                    for (int p = 0; p < DVS / 16; ++p)
                        tmem_ld16(tS + 16 * p, *reinterpret_cast<float(*)[16]>(xa + 16 * p));
                    tmem_wait_ld();
                }
                if (j + 1 == nch) break;
                const float gam = gamma_of(j + 1, ok);
                if (ok) put_state(xa, gam);
                const bool ok2 = issue_chunk(j + 1, ok);
                ok = ok && ok2;
                // intermediate state: S after (j + 1) C tokens, when that is a multiple of
                // the interval strictly inside the sequence.  Written here, after the next
                // chunk's products are issued, so the stores overlap the wait for the next
                // state update instead of delaying it (xa still holds that state).
                if (ckpt_interval > 0 && ok) {
                    const int64_t done = (int64_t)(j + 1) * C;
                    if (done % ckpt_interval == 0 && done < rb - ra) {
                        const int64_t e = ck0 + done / ckpt_interval - 1;
                        if (e < ckpt_capacity) {
                            float4 *dst = reinterpret_cast<float4 *>(
                                ckpt + (((size_t)e * H + h) * D + c) * D + j0);
#pragma unroll
                            for (int i = 0; i < DVS / 4; ++i)
                                dst[i] = make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
                        } else if (lane == 0) {
                            atomicOr(err, ERR_BAD_INDEX);   // the caller's array is too small
                        }
                    }
                }
            }
            if (ok && state_out && !*abort_flag) {
#pragma unroll
                for (int i = 0; i < DVS / 4; ++i)
                    reinterpret_cast<float4 *>(state_out + srow)[i] =
                        make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
            }
            if (issuer) {
                mma_commit(&bars[DRAIN_S]);
                mbar_wait(&bars[DRAIN_S], 0, err, 1ull << 28);
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


// ======================================================================
// One launch for both phases
// ======================================================================
// With few (sequence, head) units the state pass needs few CTAs, and run after
// phase A it holds the GPU alone, latency-bound, for 40 % of the step.  In
// prefill_fused_kernel the first CTAs run the state pass while the others run
// phase A, taking items from a device counter in chunk order; phase A publishes
// each finished slot (release store of the launch's epoch into its ready word)
// and the state pass copies a slot in only after an acquire load has seen that
// word.  Phase A never waits on the state pass, so the launch finishes whether
// or not all of its CTAs are resident at once; every wait is bounded.
//
// The state pass here fits the launch's 256 threads and phase A's shared
// memory: one copy of each slot part, in regions that free at different times
// so that each is refilled while the chain works on something else:
//   [T; R]: free once the V term [T; R] V has run (VDONE; the V term is issued
//     as soon as its operands are in, ahead of the state), refilled during the
//     rest of the chunk;
//   the V slice (an input, read from device memory): two copies, loaded two
//     chunks ahead;
//   Gamma_L: two copies (the state copy of chunk j reads its own while chunk
//     j + 1's lands);
//   [-W; P]: free once the chunk products have completed (TDFULL), refilled
//     during the U copy-out, the state update and the next state copy;
//   Khat: free once the state update has completed (TSFULL), refilled during
//     the state copy, the chunk products and the U copy-out.
template <int DVS>
struct FLayout {
    static constexpr uint32_t oWP = 0;                   // slot bytes [0, 32768)
    static constexpr uint32_t oTR = kSlotTR;             // slot bytes [32768, 49152)
    static constexpr uint32_t oV = 49152;                // V slices, 2 x 64 rows x DVS
    static constexpr uint32_t kVBytes = 64 * DVS * 2;
    static constexpr uint32_t oGam = oV + 2 * kVBytes;   // Gamma_L, 2 x 128 fp32
    static constexpr uint32_t kTTx = 16384 + 512;        // tx of one [T; R] + Gamma_L fill
    static constexpr uint32_t oKh = (oGam + 1024 + 1023) & ~1023u;
    static constexpr uint32_t oSB = oKh + 16384;         // fp16 S  (K=128 x N=DVS)
    static constexpr uint32_t oUB = oSB + 128 * DVS * 2; // fp16 U  (K=64 x N=DVS)
    static constexpr uint32_t oBar = oUB + 64 * DVS * 2;
    static constexpr uint32_t kBytes = oBar + 256;
    static constexpr uint32_t kKGroup = (DVS / 8) * 128;
    static constexpr uint32_t kVLine = DVS == 32 ? 64 : 128;
    static constexpr Swizzle kVSwz = DVS == 32 ? SW_64B : SW_128B;
    static constexpr uint32_t kVSbo = 8 * kVLine;
    static constexpr uint32_t kVLbo = 64 * kVLine;
    static constexpr uint32_t kVKstep = 16 * kVLine;
    static constexpr uint32_t kTmemCols = DVS == 32 ? 128 : 256;   // TD0, TD1, TS
    static_assert(DVS == 32 || DVS == 64, "one-launch state pass slice");
    static_assert(kBytes + 1024 <= A_SMEM, "state pass must fit phase A's shared memory");
    static_assert(oV % 1024 == 0 && kVBytes % 512 == 0 && oKh % 1024 == 0 && oSB % 128 == 0 &&
                  oUB % 128 == 0, "operand alignment");
};

enum FBar { F_WFULL = 0, F_TFULL, F_VFULL0, F_VFULL1, F_VDONE, F_YFULL, F_TD0, F_TD1, F_TSFULL,
            F_DRAIN_S, F_DRAIN_U, F_NBARS };
static_assert(F_NBARS * 8 + 5 * 4 <= 256, "one-launch state pass barrier area");

// Roles (256 threads): warps 0-3 state group (TMEM lane = key channel; fp16
// copy of S, Gamma scaling; thread 0 issues the state term [-W; P] S and every
// copy); warps 4-7 U group (TMEM lane = row of [U; O]; V conversion, U
// copy-out, O to device memory; thread 128 issues the V term [T; R] V as soon
// as its operands are in, and the state update).
// Each barrier completes once per chunk, and no copy into a region is issued
// before every waiter has passed the region's previous phase, so a parity wait
// never meets a barrier two phases ahead.
template <int DVS>
__device__ __forceinline__ void state_pass_role(
    const CUtensorMap *tm_v, const float *state_in, const int32_t *__restrict__ cu, int64_t T,
    int N, int H, const uint8_t *__restrict__ ws, const uint32_t *ready, float *__restrict__ o,
    float *state_out, int64_t ckpt_interval, float *ckpt, int64_t ckpt_capacity, uint32_t *err,
    uint32_t epoch, uint8_t *sm, int cta) {
    using Lay = FLayout<DVS>;
    constexpr int NSL = D / DVS;
    constexpr int CPR = DVS / 8;   // 16-byte pieces per V row
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::oBar);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + F_NBARS);
    volatile uint32_t *abort_flag = tmem_ptr + 1;
    volatile uint32_t *s_grp_ok = tmem_ptr + 2;   // state-group leader -> group
    volatile uint32_t *s_u_ok = tmem_ptr + 3;     // U-group leader -> group
    // highest chunk (launch index) whose ready word the U-group leader has seen
    volatile uint32_t *s_seen = tmem_ptr + 4;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = cta % NSL, unit = cta / NSL;
    const int32_t *chunk_off = reinterpret_cast<const int32_t *>(ws);
    if (unit / H >= N) return;
    const int n = cu ? chunk_off[3 * (N + 1) + unit / H] : unit / H, h = unit % H;
    int64_t ra, rb;
    seq_rows(chunk_off, cu != nullptr, T, N, n, ra, rb);
    const int nch = (int)((rb - ra + C - 1) / C);
    const int c0 = cu ? chunk_off[n] : n * (int)((T + C - 1) / C);
    const int64_t ck0 = cu ? (int64_t)chunk_off[2 * (N + 1) + n]
                           : (int64_t)n * ((T > 0 && ckpt_interval > 0) ? (T - 1) / ckpt_interval : 0);
    const uint8_t *slots = ws + header_bytes(N);
    const int j0 = slice * DVS;
    const int nct_total = cu ? chunk_off[N] : N * (int)((T + C - 1) / C);   // chunks of the launch

    if (warp == 0) {
        tmem_alloc(tmem_ptr, Lay::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < F_NBARS; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        *abort_flag = 0u;
        *s_grp_ok = 1u;
        *s_u_ok = 1u;
        *s_seen = (uint32_t)(c0 - 1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t tTD0 = tmem, tTD1 = tmem + DVS, tTS = tmem + 2 * DVS;
    auto chunk_len = [&](int j) {
        const int64_t t0 = ra + (int64_t)j * C;
        return (int)((rb - t0) < C ? (rb - t0) : C);
    };
    auto slot_of = [&](int j) { return slots + ((size_t)(c0 + j) * H + h) * kSlotBytes; };
    auto gam_buf = [&](int j) { return reinterpret_cast<float *>(sm + Lay::oGam + (j & 1) * 512); };
    auto v_off = [&](int j) { return Lay::oV + (uint32_t)(j & 1) * Lay::kVBytes; };   // V slice of chunk j

    if (warp < 4) {
        // ------------------------------------------------ state group
        // Only thread 0 (the leader) polls barriers and ready words; the group
        // waits for it at named barriers, which take no issue slots from the
        // phase A CTA that shares the SM.
        const int c = tid;   // key channel = TMEM lane
        const bool issuer = tid == 0;
        const uint32_t tS = taddr(tTS, 32 * warp, 0);
        const size_t srow = (((size_t)n * H + h) * D + c) * D + j0;
        const uint32_t id_nn = idesc(FMT_F16, 128, DVS, 0, 1);   // A K-major, B MN-major
        uint8_t *sbp = sm + Lay::oSB;
        // issuer bookkeeping: copies issued per region, V terms issued, ready words seen
        int t_loads = 0, v_loads = 0, w_loads = 0, y_loads = 0, seen = c0 - 1;
        const uint32_t *rrow = ready + (size_t)h * ready_stride(nct_total);
        // chunk j's ready word observed (acquire) before any copy of its slot: as a
        // rule by the U-group leader ahead of time (handed over in s_seen); else here,
        // eight words (consecutive chunks of this head) per 32-byte acquire load, one
        // acquire load of the word itself when they are not all set
        auto ensure_ready = [&](int j) {
            const int cc = c0 + j;
            if (cc <= seen) return true;
            const int sv = (int)ld_acquire_cta_shared(s_seen);
            if (cc <= sv) {
                seen = sv;
                return true;
            }
            const int g = cc & ~7;
            uint32_t w[8];
            ld_acquire_gpu_v8(rrow + g, w);
            int m = cc - 1;
            bool run = true;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int ci = g + i;
                if (run && ci >= cc && ci < c0 + nch) {
                    if (w[i] == epoch) m = ci; else run = false;
                }
            }
            if (m >= cc) {
                seen = m;
                return true;
            }
            if (!word_wait_abortable(rrow + cc, epoch, err, epoch, abort_flag)) return false;
            seen = cc;
            return true;
        };
        // [T; R] and Gamma_L of chunk j by bulk copy, after its ready word
        auto load_t = [&](int j) {
            if (!ensure_ready(j)) return false;
            fence_proxy_async_global();
            const uint8_t *src = slot_of(j);
            mbar_arrive_expect_tx(&bars[F_TFULL], Lay::kTTx);
            bulk_g2s(sm + Lay::oTR, src + kSlotTR, 16384, &bars[F_TFULL]);
            bulk_g2s(gam_buf(j), src + kSlotGam, 512, &bars[F_TFULL]);
            ++t_loads;
            return true;
        };
        // the V slice of chunk j (an input: no ready word) into its copy by TMA
        auto load_vs = [&](int j) {
            uint64_t *bar = &bars[(j & 1) ? F_VFULL1 : F_VFULL0];
            mbar_arrive_expect_tx(bar, Lay::kVBytes);
            tma_load_3d(sm + v_off(j), tm_v, j0, h, (int)(ra + (int64_t)j * C), bar);
            ++v_loads;
        };
        // [-W; P] and Khat of chunk j (its ready word was seen by load_t(j))
        auto load_w = [&](int j) {
            mbar_arrive_expect_tx(&bars[F_WFULL], 32768);
            bulk_g2s(sm + Lay::oWP, slot_of(j), 32768, &bars[F_WFULL]);
            ++w_loads;
        };
        auto load_y = [&](int j) {
            mbar_arrive_expect_tx(&bars[F_YFULL], 16384);
            bulk_g2s(sm + Lay::oKh, slot_of(j) + kSlotKh, 16384, &bars[F_YFULL]);
            ++y_loads;
        };
        // fp16 copy of S (B operand of the state term)
        auto put_state = [&](const float *xa) {
#pragma unroll
            for (int p = 0; p < DVS / 16; ++p) {
                const float *x = xa + 16 * p;
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
            }
        };
        // S_{j+1} = Gamma_j S_j + D_j in registers, D_j = Khat_j^T U_j from TS (the
        // state update accumulates into a fresh tile: no scaled state goes back to TMEM)
        auto advance_state = [&](float *xa, float gam) {
#pragma unroll
            for (int hp = 0; hp < DVS / 32; ++hp) {
                float d[32];
                tmem_ld16(tS + 32 * hp, *reinterpret_cast<float(*)[16]>(d));
                tmem_ld16(tS + 32 * hp + 16, *reinterpret_cast<float(*)[16]>(d + 16));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) xa[32 * hp + e] = fmaf(gam, xa[32 * hp + e], d[e]);
            }
        };
        // leader, after the group's state copy: [U; O]_j += [-W; P]_j S_j onto the V term
        // [T; R]_j V_j, which the U-group leader issued (its completion orders the two)
        auto issue_products = [&](int j) {
            if (!mbar_wait_abortable(&bars[F_TFULL], j & 1, err, epoch, abort_flag)) return false;
            if (!mbar_wait_abortable(&bars[F_VDONE], j & 1, err, epoch, abort_flag)) return false;
            if (!mbar_wait_abortable(&bars[F_WFULL], j & 1, err, epoch, abort_flag)) return false;
            tc_fence_after();
            const uint32_t tTD = (j & 1) ? tTD1 : tTD0;
            const uint64_t ad0 = smem_desc(sbase + Lay::oWP, 16, 1024, SW_128B);
            const uint64_t bd0 = smem_desc(sbase + Lay::oSB, Lay::kKGroup, 128, SW_NONE);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_f16(tTD, ad0 + (uint64_t)(((kk >> 2) * kWPKBlock + (kk & 3) * 32) / 16),
                        bd0 + (uint64_t)(kk * 2 * Lay::kKGroup / 16), id_nn, 1);
            mma_commit(&bars[(j & 1) ? F_TD1 : F_TD0]);
            return true;
        };
        if (nch == 0) {
            if (state_out)
                for (int i = 0; i < DVS / 4; ++i)
                    reinterpret_cast<float4 *>(state_out + srow)[i] =
                        state_in ? reinterpret_cast<const float4 *>(state_in + srow)[i]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            bool ok = true;
            float xa[DVS];
#pragma unroll
            for (int i = 0; i < DVS / 4; ++i) {
                const float4 f = state_in ? reinterpret_cast<const float4 *>(state_in + srow)[i]
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                xa[4 * i] = f.x; xa[4 * i + 1] = f.y; xa[4 * i + 2] = f.z; xa[4 * i + 3] = f.w;
            }
            if (issuer) {
                load_vs(0);
                if (nch > 1) load_vs(1);
                ok = load_t(0);
                if (ok) {
                    load_w(0);
                    load_y(0);
                    ok = mbar_wait_abortable(&bars[F_TFULL], 0, err, epoch, abort_flag);
                }
                *s_grp_ok = ok ? 1u : 0u;
            }
            named_bar(2, 128);
            ok = *s_grp_ok != 0u;
            if (ok) put_state(xa);
            fence_async_smem();
            tc_fence_before();
            named_bar(2, 128);
            if (issuer && ok) ok = issue_products(0);
            for (int j = 0; j < nch; ++j) {
                const bool more = j + 1 < nch;
                if (issuer) {
                    if (ok && more) {
                        // once the V term of chunk j has run (the whole group has read
                        // Gamma_j: the state term of j was issued after it): [T; R] of
                        // chunk j + 1, and the V slice of chunk j + 2 into V_j's copy
                        ok = mbar_wait_abortable(&bars[F_VDONE], j & 1, err, epoch, abort_flag);
                        if (ok && j + 2 < nch) load_vs(j + 2);
                        if (ok) ok = load_t(j + 1);
                        // [-W; P] of chunk j + 1 once the chunk products of j have completed
                        if (ok)
                            ok = mbar_wait_abortable(&bars[(j & 1) ? F_TD1 : F_TD0], (j >> 1) & 1, err,
                                                     epoch, abort_flag);
                        if (ok) load_w(j + 1);
                    }
                    // the state update of chunk j has landed in TS; then Khat is free.
                    // ([T; R] and Gamma_L of chunk j + 1 are waited for only before the
                    // V term: the state copy-out below needs Gamma_j, which is in.)
                    if (ok) ok = mbar_wait_abortable(&bars[F_TSFULL], j & 1, err, epoch, abort_flag);
                    if (ok && more) load_y(j + 1);
                    *s_grp_ok = ok ? 1u : 0u;
                }
                named_bar(2, 128);
                ok = *s_grp_ok != 0u;
                tc_fence_after();
                if (ok) advance_state(xa, gam_buf(j)[c]);
                if (!more) break;
                if (ok) put_state(xa);
                fence_async_smem();
                tc_fence_before();
                named_bar(2, 128);
                if (issuer && ok) ok = issue_products(j + 1);
                // intermediate state: S after (j + 1) C tokens, when that is a multiple of
                // the interval strictly inside the sequence (the stores overlap the
                // chunk products)
                if (ckpt_interval > 0 && ok) {
                    const int64_t done = (int64_t)(j + 1) * C;
                    if (done % ckpt_interval == 0 && done < rb - ra) {
                        const int64_t e = ck0 + done / ckpt_interval - 1;
                        if (e < ckpt_capacity) {
                            float4 *dst = reinterpret_cast<float4 *>(
                                ckpt + (((size_t)e * H + h) * D + c) * D + j0);
#pragma unroll
                            for (int i = 0; i < DVS / 4; ++i)
                                dst[i] = make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
                        } else if (lane == 0) {
                            atomicOr(err, ERR_BAD_INDEX);
                        }
                    }
                }
            }
            if (ok && state_out && !*abort_flag) {
#pragma unroll
                for (int i = 0; i < DVS / 4; ++i)
                    reinterpret_cast<float4 *>(state_out + srow)[i] =
                        make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
            }
            if (issuer) {
                mma_commit(&bars[F_DRAIN_S]);
                mbar_wait(&bars[F_DRAIN_S], 0, err, 1ull << 28);
                // copies issued and never consumed (after an abort) land before exit
                if (t_loads > 0) mbar_wait(&bars[F_TFULL], (t_loads - 1) & 1, err, 1ull << 28);
                for (int jl = v_loads - 2; jl < v_loads; ++jl)
                    if (jl >= 0)
                        mbar_wait(&bars[(jl & 1) ? F_VFULL1 : F_VFULL0], (jl >> 1) & 1, err, 1ull << 28);
                if (w_loads > 0) mbar_wait(&bars[F_WFULL], (w_loads - 1) & 1, err, 1ull << 28);
                if (y_loads > 0) mbar_wait(&bars[F_YFULL], (y_loads - 1) & 1, err, 1ull << 28);
            }
        }
    } else {
        // ------------------------------------------------ U group (leader: thread 128)
        const int quad = warp - 4;
        const int row = 32 * quad + lane;   // TMEM lane: U rows 0..63, O rows 64..127
        const int ct = tid - 128;
        const bool issuer = tid == 128;
        const uint32_t id_mm = idesc(FMT_F16, 128, DVS, 1, 1);   // A MN-major, B MN-major
        const uint32_t id_nn = idesc(FMT_F16, 128, DVS, 0, 1);   // A K-major, B MN-major
        const uint32_t *urow = ready + (size_t)h * ready_stride(nct_total);
        int useen = c0 - 1;   // leader: highest chunk whose ready word it has seen
        bool ok = true;
        for (int j = 0; j < nch; ++j) {
            // V slice of chunk j: bf16 -> fp16 in place, rows past the chunk's end -> 0
            if (issuer) {
                if (ok)
                    ok = mbar_wait_abortable(&bars[(j & 1) ? F_VFULL1 : F_VFULL0], (j >> 1) & 1, err, epoch,
                                             abort_flag);
                *s_u_ok = ok ? 1u : 0u;
            }
            named_bar(1, 128);
            ok = *s_u_ok != 0u;
            if (ok) {
                uint8_t *vt = sm + v_off(j);
                const int L = chunk_len(j);
#pragma unroll
                for (int i = 0; i < CPR / 2; ++i) {
                    const int idx = ct + 128 * i;
                    const int vrow = ((idx * 16) % 8192) / (int)Lay::kVLine;
                    uint4 *pc = reinterpret_cast<uint4 *>(vt) + idx;
                    if (vrow < L) {
                        float x[8];
                        unpack8(*pc, x);
                        *pc = pack8(x);
                    } else {
                        *pc = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            fence_async_smem();
            named_bar(1, 128);
            // [U; O]_j out of TMEM once the chunk products have completed
            const int b = j & 1;
            const uint32_t tTD = b ? tTD1 : tTD0;
            if (issuer) {
                // the V term [T; R]_j V_j into TD[j % 2] (free: the U copy-out of chunk
                // j - 2 read it before the state update of j - 2 was issued)
                if (ok) ok = mbar_wait_abortable(&bars[F_TFULL], j & 1, err, epoch, abort_flag);
                if (ok) {
                    tc_fence_after();
                    const uint64_t ad0 = smem_desc(sbase + Lay::oTR, 16, 1024, SW_128B);
                    const uint64_t bd0 = smem_desc(sbase + v_off(j), Lay::kVLbo, Lay::kVSbo, Lay::kVSwz);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tTD, ad0 + (uint64_t)(kk * 32 / 16),
                                bd0 + (uint64_t)(kk * Lay::kVKstep / 16), id_nn, kk > 0);
                    mma_commit(&bars[F_VDONE]);
                    // while the chunk products run: the next ready words (eight chunks
                    // of this head per 32-byte acquire load, never waiting), handed
                    // to the state-group leader
                    if (useen < c0 + nch - 1 && useen < c0 + j + 16) {
                        const int g = (useen + 1) & ~7;
                        uint32_t w[8];
                        ld_acquire_gpu_v8(urow + g, w);
                        int m = useen;
                        bool run = true;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int ci = g + i;
                            if (run && ci > useen && ci < c0 + nch) {
                                if (w[i] == epoch) m = ci; else run = false;
                            }
                        }
                        if (m > useen) {
                            useen = m;
                            st_release_cta_shared(s_seen, (uint32_t)m);
                        }
                    }
                    ok = mbar_wait_abortable(&bars[b ? F_TD1 : F_TD0], (j >> 1) & 1, err, epoch, abort_flag);
                }
                *s_u_ok = ok ? 1u : 0u;
            }
            named_bar(1, 128);
            ok = *s_u_ok != 0u;
            tc_fence_after();
            const int64_t t0 = ra + (int64_t)j * C;
            const int L = chunk_len(j);
            float xa[DVS];
            if (ok) {
#pragma unroll
                for (int p = 0; p < DVS / 16; ++p)
                    tmem_ld16(taddr(tTD, 32 * quad, 16 * p), *reinterpret_cast<float(*)[16]>(xa + 16 * p));
                tmem_wait_ld();
                if (quad < 2) {
#pragma unroll
                    for (int p = 0; p < DVS / 16; ++p) {
                        float y0[8], y1[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            y0[e] = xa[16 * p + e];
                            y1[e] = xa[16 * p + 8 + e];
                        }
                        *reinterpret_cast<uint4 *>(
                            sm + Lay::oUB + interleave_mnmajor_off(16 * p, row, Lay::kKGroup)) = pack8(y0);
                        *reinterpret_cast<uint4 *>(
                            sm + Lay::oUB + interleave_mnmajor_off(16 * p + 8, row, Lay::kKGroup)) =
                            pack8(y1);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_bar(1, 128);
            if (issuer && ok) {
                // D_j = Khat_j^T U_j into TS (the state group has read D_{j-1}: the
                // chunk products of j were issued after it)
                ok = mbar_wait_abortable(&bars[F_YFULL], j & 1, err, epoch, abort_flag);
                if (ok) {
                    tc_fence_after();
                    const uint64_t ad0 = smem_desc(sbase + Lay::oKh, kKhMNBlock, 1024, SW_128B);
                    const uint64_t bd0 = smem_desc(sbase + Lay::oUB, Lay::kKGroup, 128, SW_NONE);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tTS, ad0 + (uint64_t)(kk * 2048 / 16),
                                bd0 + (uint64_t)(kk * 2 * Lay::kKGroup / 16), id_mm, kk > 0);
                    mma_commit(&bars[F_TSFULL]);
                }
            }
            // O rows to device memory (fp32), after the state update is on its way
            const int r = row - 64;
            if (ok && quad >= 2 && r < L) {
                float4 *dst = reinterpret_cast<float4 *>(o + ((size_t)(t0 + r) * H + h) * D + j0);
#pragma unroll
                for (int i = 0; i < DVS / 4; ++i)
                    dst[i] = make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
            }
        }
        if (issuer) {
            mma_commit(&bars[F_DRAIN_U]);
            mbar_wait(&bars[F_DRAIN_U], 0, err, 1ull << 28);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}

// The first n_state CTAs run the state pass (DVS value columns each), the rest
// phase A.
template <bool PREP, int DVS>
__global__ void __launch_bounds__(256, 2)
prefill_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                     const __nv_bfloat16 *__restrict__ beta, const int32_t *__restrict__ cu,
                     int64_t T, int N, int H, uint32_t flags, uint8_t *__restrict__ ws,
                     const float *state_in, float *__restrict__ o, float *state_out,
                     int64_t ckpt_interval, float *ckpt, int64_t ckpt_capacity, uint32_t *sched,
                     uint32_t *ready, int n_state, uint32_t *err, uint32_t epoch) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    if ((int)blockIdx.x < n_state) {
        if (threadIdx.x == 0) {   // mark this SM as running a chain (words 8 .. 15 of the scheduler area)
            uint32_t smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            if ((smid >> 5) < 8u) atomicOr(sched + 8 + (smid >> 5), 1u << (smid & 31));
        }
        state_pass_role<DVS>(&tm_v, state_in, cu, T, N, H, ws, ready, o, state_out, ckpt_interval,
                             ckpt, ckpt_capacity, err, epoch, sm, (int)blockIdx.x);
    } else {
        intra_chunk_body<PREP>(&tm_q, &tm_k, &tm_g, beta, cu, T, N, H, flags, ws, err, epoch, sm,
                               (int)blockIdx.x - n_state, (int)gridDim.x - n_state, sched, ready);
    }
}

}  // namespace tc

// ======================================================================
// host side
// ======================================================================
// Workspace: header, slots, then (for the one-launch form) a 256-byte area
// holding phase A's item counter and one ready word per (chunk, head) item.
static size_t sched_offset(int64_t rows, int N, int H) {
    const int64_t max_chunks = (rows + tc::C - 1) / tc::C + N;
    return (size_t)tc::header_bytes(N) + (size_t)max_chunks * H * tc::kSlotBytes;
}

size_t prefill_tc_workspace_bytes(int64_t rows, int N, int H, int d) {
    if (d != tc::D) return 0;
    const int64_t max_chunks = (rows + tc::C - 1) / tc::C + N;
    return sched_offset(rows, N, H) + 256 +
           (((size_t)tc::ready_stride((int)max_chunks) * H * 4 + 255) & ~(size_t)255);
}

template <int DVS>
static cudaError_t launch_state_pass(const PrefillArgs &a, cudaStream_t st) {
    using Lay = tc::BLayout<DVS>;
    auto kern = tc::state_pass_kernel<DVS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lay::kBytes);
    if (e != cudaSuccess) return e;
    // TMA boxes of the V slice: DVS (at most 64) channels x 64 rows of one head
    CUtensorMap tv;
    const int64_t rows = (int64_t)a.B * a.T;
    if (rows > 0 && !make_rows_heads_tmap(&tv, a.v, rows, a.H, tc::D, DVS < 64 ? DVS : 64, tc::C,
                                          DVS == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (rows == 0) memset(&tv, 0, sizeof(tv));   // no chunk: the map is never used
    const int grid = a.N * a.H * (tc::D / DVS);
    kern<<<grid, 384, Lay::kBytes, st>>>(tv, a.state_in, a.cu_seqlens,
                                         a.T, a.N, a.H, (const uint8_t *)a.workspace,
                                         (float *)a.o, a.state_out, a.ckpt_interval, a.ckpt,
                                         a.ckpt_capacity, a.err, a.epoch);
    e = cudaGetLastError();
    Profiler::mark(st);
    return e;
}

// One launch for both phases (tc::prefill_fused_kernel) when the state pass
// needs at most kFusedMaxStateCtas CTAs of kFusedDVS value columns; otherwise
// the two-kernel form.  The choice depends on the shapes only, so a call with
// intermediate states runs the same kernels as one without (its o and final
// state are the same bit for bit).  The grid assumes two CTAs per SM (phase A's shared
// memory and 128 registers per thread); correctness does not depend on it.
constexpr int kFusedDVS = 64;
constexpr int64_t kFusedMaxStateCtas = 74;

static cudaError_t launch_fused(const PrefillArgs &a, int64_t rows, int64_t max_chunks,
                                cudaStream_t st) {
    auto kern = a.flags ? tc::prefill_fused_kernel<true, kFusedDVS>
                        : tc::prefill_fused_kernel<false, kFusedDVS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc::A_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n_state = (int64_t)a.N * a.H * (tc::D / kFusedDVS);
    const int64_t items = max_chunks * a.H;
    if (items > INT32_MAX - 65536 || rows > INT32_MAX) return cudaErrorInvalidValue;
    int64_t n_a = 2 * (int64_t)sms - n_state;
    if (n_a > items) n_a = items;
    if (n_a < 1) n_a = 1;
    CUtensorMap tq, tk, tg, tv;
    if (!make_rows_heads_tmap(&tq, a.q, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_rows_heads_tmap(&tk, a.k, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_rows_heads_tmap(&tg, a.g, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_rows_heads_tmap(&tv, a.v, rows, a.H, tc::D, kFusedDVS, tc::C,
                              CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    uint8_t *ws = (uint8_t *)a.workspace;
    uint32_t *sched = reinterpret_cast<uint32_t *>(ws + sched_offset(rows, a.N, a.H));
    uint32_t *ready = sched + 64;
    // the counter and every ready word start at zero (epochs are nonzero)
    e = cudaMemsetAsync(sched, 0, 256 + (size_t)tc::ready_stride((int)max_chunks) * a.H * 4, st);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(n_state + n_a), 256, tc::A_SMEM, st>>>(
        tq, tk, tg, tv, (const __nv_bfloat16 *)a.beta, a.cu_seqlens, a.T, a.N, a.H, a.flags, ws,
        a.state_in, (float *)a.o, a.state_out, a.ckpt_interval, a.ckpt, a.ckpt_capacity, sched,
        ready, (int)n_state, a.err, a.epoch);
    e = cudaGetLastError();
    Profiler::mark(st);
    return e;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    if (a.dk != tc::D || a.dv != tc::D) return cudaErrorInvalidValue;
    uint8_t *ws = (uint8_t *)a.workspace;
    cudaError_t e = cudaSuccess;
    if (a.cu_seqlens) {
        // packed sequences: row bounds and first chunks per sequence (both kernels
        // below compute them by arithmetic for an equal-length batch)
        tc::chunk_table_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.T, a.N, a.ckpt_interval,
                                                   reinterpret_cast<int32_t *>(ws));
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        Profiler::mark(st);
    }
    const int64_t rows = (int64_t)a.B * a.T;
    const int64_t max_chunks =
        a.cu_seqlens ? (rows + tc::C - 1) / tc::C + a.N : (int64_t)a.N * ((a.T + tc::C - 1) / tc::C);
    const int64_t units = (int64_t)a.N * a.H;
    if (max_chunks > 0 && units * (tc::D / kFusedDVS) <= kFusedMaxStateCtas) {
        return launch_fused(a, rows, max_chunks, st);
    }
    if (max_chunks > 0) {
        auto kern = a.flags ? tc::intra_chunk_kernel<true> : tc::intra_chunk_kernel<false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::A_SMEM);
        if (e != cudaSuccess) return e;
        // persistent: two CTAs per SM walk the (chunk, head) items
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t items = max_chunks * a.H;
        if (items > INT32_MAX - 65536) return cudaErrorInvalidValue;
        const int64_t ctas = items < 2 * (int64_t)sms ? items : 2 * (int64_t)sms;
        // TMA tiles of q, k, g: 64 channels x 64 rows of one head per box
        CUtensorMap tq, tk, tg;
        if (rows > INT32_MAX ||
            !make_rows_heads_tmap(&tq, a.q, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_rows_heads_tmap(&tk, a.k, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_rows_heads_tmap(&tg, a.g, rows, a.H, tc::D, 64, tc::C, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        kern<<<(unsigned)ctas, 256, tc::A_SMEM, st>>>(
            tq, tk, tg, (const __nv_bfloat16 *)a.beta, a.cu_seqlens, a.T, a.N, a.H, a.flags, ws,
            a.err, a.epoch);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    Profiler::mark(st);
    // dv-slices: enough CTAs to cover the SMs when there are few (sequence, head) units
    if (units <= 74) return launch_state_pass<32>(a, st);
    if (units <= 148) return launch_state_pass<64>(a, st);
    return launch_state_pass<128>(a, st);
}

}  // namespace kda
