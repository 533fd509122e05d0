// KDA backward: gradients of the recurrence
//     S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = S_t^T q_t,   a_t = exp(max(g_t, -5))
// with respect to q, k, v, g, beta and the initial state, given dL/do and
// dL/dS_T (the training use of the delta rule with per-channel retention of
// neurohive.io "Kimi K3 ... overview", section "Sequence length: hybrid KDA
// and Gated MLA attention"; the pages give no formulas for it).
//
// Per token, with S' = Diag(a) S_{t-1}, p = S'^T k, delta = beta (v - p),
// S_t = S' + k delta^T, and dS the gradient flowing into S_t:
//     dS  += q do^T;            dq = S_t do
//     dd   = dS^T k;            dbeta = dd . (v - p);   dv = beta dd
//     dp   = -beta dd;          dk = dS delta + S' dp
//     dS'  = dS + k dp^T;       da = rowsum(dS' * S_{t-1})
//     dg   = da * a  (0 where g < -5);   dS_{t-1} = Diag(a) dS'
//
// One CTA of 256 threads per (sequence, head, value-column slice), fp32
// throughout (bf16 inputs are read exactly).  Every step above is local to a
// set of value columns (the recurrence updates the columns of S
// independently) except the sums over columns: dq, dk, da and dbeta.  So a
// few units are cut into NSL column slices, one CTA each, and the slices
// write those four as partial sums that a second kernel adds up in slice
// order (deterministic); with many units NSL = 1 and the CTA writes them
// directly.  Each thread keeps a (D / RG) x 4 block of its slice of S and of
// dS in registers; column sums over rows and row sums over columns go through
// shared memory.  Pass 1 runs the recurrence forward and stores the state at
// every chunk start (C = 64 tokens) in the workspace.  Pass 2 walks the chunks
// backwards: it reruns the chunk forward from its stored start state, storing
// the state before each token, then applies the token steps above in reverse.
// Reads and writes are sequential per (sequence, head); the work is the
// recurrence's ~12 dk dv flops per token three times over.  This is the
// straightforward form of the backward, not a tensor-core chunked one.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "sm100.cuh"

namespace kda {
namespace bwd {

using sm100::cp_async16;
using sm100::cp_async_commit;
using sm100::cp_async_wait_all;

constexpr int C = 64;     // tokens per stored chunk state
constexpr int NT = 256;   // threads per CTA

template <int D, int DVS>
struct Lay {
    static constexpr int CG = DVS / 4;       // column groups of 4
    static constexpr int RG = NT / CG;       // row groups
    static constexpr int RPT = D / RG;       // rows per thread
    static constexpr int PW = 3 * D + 4;     // partial sums per (token, head): dq, dk, da, dbeta
    static_assert(D % RG == 0 && RPT >= 1, "rows must split evenly");
};

// column slices per (sequence, head): enough CTAs to cover the SMs when there
// are few units
__host__ __device__ inline int slices_for(int64_t units) {
    return units <= 37 ? 4 : (units <= 74 ? 2 : 1);
}

// rows [a, b) of sequence n: equal-length batch, or the packed offsets clamped
// to [0, T] and made non-decreasing (the prefill's rule)
__device__ __forceinline__ void rows_of(const int32_t *cu, int64_t T, int n, int64_t &a, int64_t &b) {
    if (!cu) {
        a = (int64_t)n * T;
        b = a + T;
        return;
    }
    auto cl = [&](int64_t x) { return x < 0 ? 0 : (x > T ? T : x); };
    int64_t run = 0;
    for (int i = 0; i <= n; ++i) run = max(run, cl(cu[i]));
    a = run;
    b = max(run, cl(cu[n + 1]));
}

// index of sequence n's first stored chunk state: chunks of sequences 0..n-1
__device__ __forceinline__ int64_t chunk_base(const int32_t *cu, int64_t T, int n) {
    if (!cu) return (int64_t)n * ((T + C - 1) / C);
    int64_t acc = 0, a, b;
    for (int i = 0; i < n; ++i) {
        rows_of(cu, T, i, a, b);
        acc += (b - a + C - 1) / C;
    }
    return acc;
}

template <int D, int DVS, typename Tin>
__global__ void __launch_bounds__(NT, 1)
backward_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                const Tin *__restrict__ g, const Tin *__restrict__ beta, const float *state_in,
                const int32_t *__restrict__ cu, int64_t T, int N, int H, int64_t rows,
                const float *__restrict__ dout, const float *dstate_out,
                float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                float *__restrict__ dg, float *__restrict__ dbeta, float *dstate_in,
                float *__restrict__ ws_chunks, float *__restrict__ ws_tokens,
                float *__restrict__ part) {
    using L = Lay<D, DVS>;
    constexpr int CG = L::CG, RG = L::RG, RPT = L::RPT, PW = L::PW;
    constexpr int NSL = D / DVS;
    const int unit = blockIdx.x / NSL, slice = blockIdx.x % NSL;
    const int n = unit / H, h = unit % H;
    if (n >= N) return;
    const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
    const int j0 = slice * DVS;          // first value column of this slice

    extern __shared__ float shm[];
    // per key channel (D): q, k, a, clamp mask, a k; per value column of the slice (DVS):
    // v, do, p, delta, v - p, dd, dp
    float *qs = shm, *ks = qs + D, *as = ks + D, *ms = as + D;
    float *aks = ms + D;                 // a * k (the column weights of p = (Diag(a) S)^T k)
    float *vs = aks + D, *dos = vs + DVS, *pv = dos + DVS, *dl = pv + DVS, *vp = dl + DVS;
    float *ddv = vp + DVS, *dpv = ddv + DVS;
    float *red_c = dpv + DVS;            // [RG][DVS] column partials (sums over a thread's rows)
    // [2][D][CG + 1] row partials (sums over a thread's columns), rows padded by one
    // word so that both the writes (one row, consecutive column groups) and the
    // reads (one row per thread) are free of bank conflicts
    constexpr int RS = CG + 1;
    float *red_r = red_c + RG * DVS;
    __shared__ float bsh;

    int64_t ra, rb;
    rows_of(cu, T, n, ra, rb);
    const int64_t len = rb - ra;
    const int nch = (int)((len + C - 1) / C);
    float *chunks = ws_chunks + (size_t)(chunk_base(cu, T, n) * H + (int64_t)h * nch) * D * D;
    float *toks = ws_tokens + (size_t)unit * C * D * D;
    const size_t sbase = ((size_t)n * H + h) * D * D;

    // this thread's block of a D x D state: rows rg + RG i, columns j0 + 4 cg .. + 3
    auto ld_block = [&](const float *src, float4 (&x)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            x[i] = src ? reinterpret_cast<const float4 *>(src + (size_t)(rg + RG * i) * D + j0)[cg]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto st_block = [&](float *dst, const float4 (&x)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            reinterpret_cast<float4 *>(dst + (size_t)(rg + RG * i) * D + j0)[cg] = x[i];
    };
    // partial sums of token t (slices > 1): [NSL][rows][H][PW]
    auto part_of = [&](int64_t t) { return part + (((size_t)slice * rows + (ra + t)) * H + h) * PW; };
    auto tok_off = [&](int64_t t, int d) { return ((size_t)(ra + t) * H + h) * d; };
    // Token inputs travel one token ahead: fetch() issues the global loads of a
    // token into registers (thread c < D holds channel c), stage() moves the
    // fetched values into shared memory (k, v, a = exp(max(g, -5)), the clamp
    // mask, a k, beta; q and do when the backward needs them), so each step's
    // loads land while the previous step computes.
    struct Tok { float k, v, g, q, dout, b; };
    auto fetch = [&](int64_t t, bool with_q) {
        Tok x{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (t < 0 || t >= len) return x;
        if (tid < D) {
            x.k = to_f32(k[tok_off(t, D) + tid]);
            x.g = to_f32(g[tok_off(t, D) + tid]);
            if (with_q) x.q = to_f32(q[tok_off(t, D) + tid]);
        }
        if (tid < DVS) {
            x.v = to_f32(v[tok_off(t, D) + j0 + tid]);
            if (with_q) x.dout = dout[tok_off(t, D) + j0 + tid];
        }
        if (tid == 0) x.b = to_f32(beta[(size_t)(ra + t) * H + h]);
        return x;
    };
    auto stage = [&](const Tok &x, bool with_q) {
        if (tid < D) {
            ks[tid] = x.k;
            const float a = expf(fmaxf(x.g, -5.f));
            as[tid] = a;
            ms[tid] = x.g >= -5.f ? 1.f : 0.f;
            aks[tid] = a * x.k;
            if (with_q) qs[tid] = x.q;
        }
        if (tid < DVS) {
            vs[tid] = x.v;
            if (with_q) dos[tid] = x.dout;
        }
        if (tid == 0) bsh = x.b;
    };
    // column sums over rows of x[r][j] * w[r], result into out[j]
    auto col_sum = [&](const float4 (&x)[RPT], const float *w, float *out) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float wr = w[rg + RG * i];
            s.x = fmaf(x[i].x, wr, s.x); s.y = fmaf(x[i].y, wr, s.y);
            s.z = fmaf(x[i].z, wr, s.z); s.w = fmaf(x[i].w, wr, s.w);
        }
        reinterpret_cast<float4 *>(red_c + rg * DVS)[cg] = s;
        __syncthreads();
        if (tid < DVS) {
            float acc = 0.f;
#pragma unroll 8
            for (int r = 0; r < RG; ++r) acc += red_c[r * DVS + tid];
            out[tid] = acc;
        }
        __syncthreads();
    };
    // one forward token step on the block S: S <- Diag(a) S + k delta^T
    auto fwd_step = [&](float4 (&S)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float a = as[rg + RG * i];
            S[i].x *= a; S[i].y *= a; S[i].z *= a; S[i].w *= a;
        }
        col_sum(S, ks, pv);                           // p = S'^T k
        if (tid < DVS) dl[tid] = bsh * (vs[tid] - pv[tid]);
        __syncthreads();
        const float4 d4 = reinterpret_cast<const float4 *>(dl)[cg];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kr = ks[rg + RG * i];
            S[i].x = fmaf(kr, d4.x, S[i].x); S[i].y = fmaf(kr, d4.y, S[i].y);
            S[i].z = fmaf(kr, d4.z, S[i].z); S[i].w = fmaf(kr, d4.w, S[i].w);
        }
    };

    // ---- pass 1: forward, storing the state at every chunk start
    float4 S[RPT];
    ld_block(state_in ? state_in + sbase : nullptr, S);
    Tok nx = fetch(0, false);
    for (int64_t t = 0; t < len; ++t) {
        if ((t % C) == 0) st_block(chunks + (size_t)(t / C) * D * D, S);
        __syncthreads();
        stage(nx, false);
        nx = fetch(t + 1, false);
        __syncthreads();
        fwd_step(S);
    }

    // ---- pass 2: chunks in reverse
    float4 dS[RPT];
    ld_block(dstate_out ? dstate_out + sbase : nullptr, dS);
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int64_t t0 = (int64_t)ci * C;
        const int cl = (int)((len - t0) < C ? (len - t0) : C);
        ld_block(chunks + (size_t)ci * D * D, S);
        Tok fx = fetch(t0, false);
        for (int u = 0; u < cl; ++u) {   // rerun the chunk, keeping S before each token
            st_block(toks + (size_t)u * D * D, S);
            __syncthreads();
            stage(fx, false);
            fx = fetch(t0 + u + 1 < t0 + cl ? t0 + u + 1 : -1, false);
            __syncthreads();
            fwd_step(S);
        }
        Tok bx = fetch(t0 + cl - 1, true);
        for (int u = cl - 1; u >= 0; --u) {
            const int64_t t = t0 + u;
            float4 Sp[RPT];                       // S_{t-1}; S' = Diag(a) S_{t-1} is formed inline
            ld_block(toks + (size_t)u * D * D, Sp);
            __syncthreads();
            stage(bx, true);
            bx = fetch(u > 0 ? t - 1 : -1, true);
            __syncthreads();
            col_sum(Sp, aks, pv);                 // p = S'^T k
            if (tid < DVS) {
                vp[tid] = vs[tid] - pv[tid];
                dl[tid] = bsh * vp[tid];          // delta
            }
            __syncthreads();
            const float4 d4 = reinterpret_cast<const float4 *>(dl)[cg];
            const float4 do4 = reinterpret_cast<const float4 *>(dos)[cg];
            // dS += q do^T; row partials of dq = S_t do; column partials of dd = dS^T k
            float4 cs = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int r = rg + RG * i;
                const float qr = qs[r], kr = ks[r], a = as[r];
                dS[i].x = fmaf(qr, do4.x, dS[i].x); dS[i].y = fmaf(qr, do4.y, dS[i].y);
                dS[i].z = fmaf(qr, do4.z, dS[i].z); dS[i].w = fmaf(qr, do4.w, dS[i].w);
                const float4 St = make_float4(fmaf(kr, d4.x, a * Sp[i].x), fmaf(kr, d4.y, a * Sp[i].y),
                                              fmaf(kr, d4.z, a * Sp[i].z), fmaf(kr, d4.w, a * Sp[i].w));
                red_r[r * RS + cg] = St.x * do4.x + St.y * do4.y + St.z * do4.z + St.w * do4.w;
                cs.x = fmaf(dS[i].x, kr, cs.x); cs.y = fmaf(dS[i].y, kr, cs.y);
                cs.z = fmaf(dS[i].z, kr, cs.z); cs.w = fmaf(dS[i].w, kr, cs.w);
            }
            reinterpret_cast<float4 *>(red_c + rg * DVS)[cg] = cs;
            __syncthreads();
            if (tid < D) {
                float aq = 0.f;
                for (int x = 0; x < CG; ++x) aq += red_r[tid * RS + x];
                if (NSL == 1) dq[tok_off(t, D) + tid] = aq;
                else part_of(t)[tid] = aq;
            }
            if (tid < DVS) {
                float ad = 0.f;
#pragma unroll 8
                for (int x = 0; x < RG; ++x) ad += red_c[x * DVS + tid];
                ddv[tid] = ad;                                   // dd
                dv[tok_off(t, D) + j0 + tid] = bsh * ad;
                dpv[tid] = -bsh * ad;                            // dp
            }
            __syncthreads();
            if (tid < 32) {                                      // dbeta = dd . (v - p)
                float s = 0.f;
                for (int c = tid; c < DVS; c += 32) s = fmaf(ddv[c], vp[c], s);
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
                if (tid == 0) {
                    if (NSL == 1) dbeta[(size_t)(ra + t) * H + h] = s;
                    else part_of(t)[3 * D] = s;
                }
            }
            const float4 dp4 = reinterpret_cast<const float4 *>(dpv)[cg];
            // row partials of dk = dS delta + S' dp and of da = rowsum(dS' * S_{t-1}),
            // with dS' = dS + k dp^T; then dS <- Diag(a) dS'
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int r = rg + RG * i;
                const float kr = ks[r], a = as[r];
                red_r[r * RS + cg] = dS[i].x * d4.x + dS[i].y * d4.y + dS[i].z * d4.z + dS[i].w * d4.w +
                                    a * (Sp[i].x * dp4.x + Sp[i].y * dp4.y + Sp[i].z * dp4.z +
                                         Sp[i].w * dp4.w);
                dS[i].x = fmaf(kr, dp4.x, dS[i].x); dS[i].y = fmaf(kr, dp4.y, dS[i].y);
                dS[i].z = fmaf(kr, dp4.z, dS[i].z); dS[i].w = fmaf(kr, dp4.w, dS[i].w);
                red_r[RS * D + r * RS + cg] = dS[i].x * Sp[i].x + dS[i].y * Sp[i].y +
                                             dS[i].z * Sp[i].z + dS[i].w * Sp[i].w;
                dS[i].x *= a; dS[i].y *= a; dS[i].z *= a; dS[i].w *= a;
            }
            __syncthreads();
            if (tid < D) {
                float akk = 0.f, aa = 0.f;
                for (int x = 0; x < CG; ++x) {
                    akk += red_r[tid * RS + x];
                    aa += red_r[RS * D + tid * RS + x];
                }
                if (NSL == 1) {
                    dk[tok_off(t, D) + tid] = akk;
                    dg[tok_off(t, D) + tid] = aa * as[tid] * ms[tid];
                } else {
                    part_of(t)[D + tid] = akk;
                    part_of(t)[2 * D + tid] = aa;   // da; the reduction applies a and the mask
                }
            }
        }
    }
    __syncthreads();
    if (dstate_in) st_block(dstate_in + sbase, dS);
}

// Sliced form (DVS <= 64 value columns per CTA): warp w owns the columns
// j0 + 4 w .. + 3 of the slice, lane l the key rows l + 32 i.  Column sums
// (p, dd) are warp shuffles.  Token inputs move in batches of TB tokens: the
// raw rows of the next batch are copied into shared memory (cp.async, double
// buffered) while the current batch is computed, so the loads' latency is
// paid once per batch instead of once per token.  The sums over columns (dq,
// dk, da, dbeta) of a batch's tokens are added up once per batch.
template <int D, int DVS, typename Tin>
struct BwdBatch {
    static constexpr int NW = DVS / 4;              // warps: 4 value columns each
    static constexpr int NTH = 32 * NW;
    static constexpr int RPT = D / 32;              // key rows per lane
    static constexpr int TB = NW <= 8 ? 8 : 4;      // tokens per batch
    static constexpr int ES = (int)sizeof(Tin);
    // one token's raw inputs in shared memory (bytes): k, g, q rows; v, do slices; beta
    static constexpr int RK = 0, RG = D * ES, RQ = 2 * D * ES, RV = 3 * D * ES;
    static constexpr int RDO = RV + DVS * ES, RB = RDO + DVS * 4;
    static constexpr int TOKB = (RB + 4 + 15) / 16 * 16;
    static constexpr int PK = D * ES / 16, PV = DVS * ES / 16, PD = DVS * 4 / 16;
    static constexpr int STG = 2 * TB * TOKB;       // two batch buffers
    static constexpr int RED = TB * (3 * NW * D + NW) * 4;   // a batch's row partials
    static constexpr int SMEM = STG + RED;
    static_assert(NTH >= D && RV % 16 == 0 && RDO % 16 == 0, "layout");
};

template <int D, int DVS, typename Tin>
__global__ void __launch_bounds__(8 * DVS, 1)
backward_sliced_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                       const Tin *__restrict__ g, const Tin *__restrict__ beta, const float *state_in,
                       const int32_t *__restrict__ cu, int64_t T, int N, int H, int64_t rows,
                       const float *__restrict__ dout, const float *dstate_out,
                       float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                       float *__restrict__ dg, float *__restrict__ dbeta, float *dstate_in,
                       float *__restrict__ ws_chunks, float *__restrict__ ws_tokens,
                       float *__restrict__ part) {
    using B = BwdBatch<D, DVS, Tin>;
    constexpr int NW = B::NW, NTH = B::NTH, RPT = B::RPT, TB = B::TB, TOKB = B::TOKB;
    constexpr int NSL = D / DVS;
    constexpr int PW = 3 * D + 4;
    const int unit = blockIdx.x / NSL, slice = blockIdx.x % NSL;
    const int n = unit / H, h = unit % H;
    if (n >= N) return;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int j0 = slice * DVS;                  // first value column of this slice
    const int jc = j0 + 4 * w;                   // this warp's first value column

    extern __shared__ __align__(16) uint8_t smb[];
    uint8_t *stg = smb;                                              // [2][TB][TOKB]
    float *red = reinterpret_cast<float *>(smb + B::STG);            // [TB][3 NW D + NW]

    int64_t ra, rb;
    rows_of(cu, T, n, ra, rb);
    const int64_t len = rb - ra;
    const int nch = (int)((len + C - 1) / C);
    float *chunks = ws_chunks + (size_t)(chunk_base(cu, T, n) * H + (int64_t)h * nch) * D * D;
    float *toks = ws_tokens + (size_t)unit * C * D * D;
    const size_t sbase = ((size_t)n * H + h) * D * D;
    auto tok_off = [&](int64_t t, int d) { return ((size_t)(ra + t) * H + h) * d; };

    // this thread's block of a D x D state: rows lane + 32 i, columns jc .. jc + 3
    auto ld_block = [&](const float *src, float4 (&x)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            x[i] = src ? *reinterpret_cast<const float4 *>(src + (size_t)(lane + 32 * i) * D + jc)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto st_block = [&](float *dst, const float4 (&x)[RPT]) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) *reinterpret_cast<float4 *>(dst + (size_t)(lane + 32 * i) * D + jc) = x[i];
    };
    // sum over the 32 lanes (the key rows) of four column partials
    auto warp_sum4 = [&](float4 x) {
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            x.x += __shfl_xor_sync(0xffffffffu, x.x, m);
            x.y += __shfl_xor_sync(0xffffffffu, x.y, m);
            x.z += __shfl_xor_sync(0xffffffffu, x.z, m);
            x.w += __shfl_xor_sync(0xffffffffu, x.w, m);
        }
        return x;
    };
    // Copies of the raw inputs of tokens t_first + dir * tau (tau < cnt) into
    // batch buffer buf, with beta into a register of thread tau.
    float breg = 0.f;
    auto issue = [&](int buf, int64_t t_first, int cnt, int dir, bool bwd) {
        constexpr int PK = B::PK, PV = B::PV, PD = B::PD;
        const int cpt = bwd ? 3 * PK + PV + PD : 2 * PK + PV;
        for (int task = tid; task < cnt * cpt; task += NTH) {
            const int tau = task / cpt;
            int pc = task % cpt;
            const int64_t t = t_first + (int64_t)dir * tau;
            uint8_t *dst = stg + (size_t)(buf * TB + tau) * TOKB;
            const uint8_t *src;
            if (pc < PK) {
                src = reinterpret_cast<const uint8_t *>(k + tok_off(t, D)) + 16 * pc;
                dst += B::RK + 16 * pc;
            } else if ((pc -= PK) < PK) {
                src = reinterpret_cast<const uint8_t *>(g + tok_off(t, D)) + 16 * pc;
                dst += B::RG + 16 * pc;
            } else if ((pc -= PK) < PV) {
                src = reinterpret_cast<const uint8_t *>(v + tok_off(t, D) + j0) + 16 * pc;
                dst += B::RV + 16 * pc;
            } else if ((pc -= PV) < PK) {
                src = reinterpret_cast<const uint8_t *>(q + tok_off(t, D)) + 16 * pc;
                dst += B::RQ + 16 * pc;
            } else {
                pc -= PK;
                src = reinterpret_cast<const uint8_t *>(dout + tok_off(t, D) + j0) + 16 * pc;
                dst += B::RDO + 16 * pc;
            }
            cp_async16(dst, src, 16u);
        }
        cp_async_commit();
        if (tid < cnt) breg = to_f32(beta[(size_t)(ra + t_first + (int64_t)dir * tid) * H + h]);
    };
    // the landed batch becomes visible (beta from the registers of its threads)
    auto land = [&](int buf, int cnt) {
        cp_async_wait_all();
        if (tid < cnt) *reinterpret_cast<float *>(stg + (size_t)(buf * TB + tid) * TOKB + B::RB) = breg;
        __syncthreads();
    };
    auto kval = [&](const uint8_t *tb, int c) { return to_f32(reinterpret_cast<const Tin *>(tb + B::RK)[c]); };
    auto qval = [&](const uint8_t *tb, int c) { return to_f32(reinterpret_cast<const Tin *>(tb + B::RQ)[c]); };
    auto gval = [&](const uint8_t *tb, int c) { return to_f32(reinterpret_cast<const Tin *>(tb + B::RG)[c]); };
    auto vval4 = [&](const uint8_t *tb) {
        const Tin *p = reinterpret_cast<const Tin *>(tb + B::RV) + 4 * w;
        return make_float4(to_f32(p[0]), to_f32(p[1]), to_f32(p[2]), to_f32(p[3]));
    };
    // forward token step on S from the token's raw inputs: S <- Diag(a) S + k delta^T
    auto fwd_step = [&](float4 (&S)[RPT], const uint8_t *tb) {
        float kr[RPT], ar[RPT];
        float4 pp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = lane + 32 * i;
            kr[i] = kval(tb, r);
            ar[i] = expf(fmaxf(gval(tb, r), -5.f));
            const float ak = ar[i] * kr[i];
            pp.x = fmaf(ak, S[i].x, pp.x); pp.y = fmaf(ak, S[i].y, pp.y);
            pp.z = fmaf(ak, S[i].z, pp.z); pp.w = fmaf(ak, S[i].w, pp.w);
        }
        pp = warp_sum4(pp);                                           // p = S'^T k
        const float b = *reinterpret_cast<const float *>(tb + B::RB);
        const float4 vv = vval4(tb);
        const float4 dl = make_float4(b * (vv.x - pp.x), b * (vv.y - pp.y), b * (vv.z - pp.z),
                                      b * (vv.w - pp.w));
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            S[i].x = fmaf(kr[i], dl.x, ar[i] * S[i].x); S[i].y = fmaf(kr[i], dl.y, ar[i] * S[i].y);
            S[i].z = fmaf(kr[i], dl.z, ar[i] * S[i].z); S[i].w = fmaf(kr[i], dl.w, ar[i] * S[i].w);
        }
    };
    // forward over tokens t_begin .. t_begin + count - 1, storing the state before
    // token u to dst: at chunk starts (u % C == 0, slot u / C) or, with every_token, always
    // (slot u)
    auto forward = [&](int64_t t_begin, int64_t count, float4 (&S)[RPT], float *dst, bool every_token) {
        __syncthreads();   // both batch buffers are free
        const int64_t nb = (count + TB - 1) / TB;
        if (nb > 0) issue(0, t_begin, (int)(count < TB ? count : TB), 1, false);
        for (int64_t bi = 0; bi < nb; ++bi) {
            const int buf = (int)(bi & 1);
            const int64_t u0 = bi * TB;
            const int cnt = (int)((count - u0) < TB ? (count - u0) : TB);
            land(buf, cnt);
            if (bi + 1 < nb) {
                const int64_t u1 = u0 + TB;
                issue(buf ^ 1, t_begin + u1, (int)((count - u1) < TB ? (count - u1) : TB), 1, false);
            }
            for (int tau = 0; tau < cnt; ++tau) {
                const int64_t u = u0 + tau;
                if (every_token) st_block(dst + (size_t)u * D * D, S);
                else if ((u % C) == 0) st_block(dst + (size_t)(u / C) * D * D, S);
                fwd_step(S, stg + (size_t)(buf * TB + tau) * TOKB);
            }
        }
    };

    // ---- pass 1: forward, storing the state at every chunk start
    float4 S[RPT];
    ld_block(state_in ? state_in + sbase : nullptr, S);
    forward(0, len, S, chunks, false);

    // ---- pass 2: chunks in reverse
    float4 dS[RPT];
    ld_block(dstate_out ? dstate_out + sbase : nullptr, dS);
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int64_t t0 = (int64_t)ci * C;
        const int cl = (int)((len - t0) < C ? (len - t0) : C);
        // rerun the chunk, keeping the state before each token
        ld_block(chunks + (size_t)ci * D * D, S);
        forward(t0, cl, S, toks, true);
        // the token steps in reverse, batch by batch (tokens t_hi, t_hi - 1, ...)
        __syncthreads();
        const int nb = (cl + TB - 1) / TB;
        issue(0, t0 + cl - 1, cl < TB ? cl : TB, -1, true);
        float4 Sp[RPT], Spn[RPT];                 // S_{t-1} of this step and of the next
        ld_block(toks + (size_t)(cl - 1) * D * D, Sp);
        for (int bi = 0; bi < nb; ++bi) {
            const int buf = bi & 1;
            const int hi = cl - 1 - bi * TB;                       // highest token (in chunk) of this batch
            const int cnt = hi + 1 < TB ? hi + 1 : TB;
            land(buf, cnt);
            if (bi + 1 < nb) {
                const int hi1 = hi - TB;
                issue(buf ^ 1, t0 + hi1, hi1 + 1 < TB ? hi1 + 1 : TB, -1, true);
            }
            for (int tau = 0; tau < cnt; ++tau) {
                const int u = hi - tau;
                const int64_t t = t0 + u;
                const uint8_t *tb = stg + (size_t)(buf * TB + tau) * TOKB;
                float *rq = red + (size_t)tau * (3 * NW * D + NW);  // this token's row partials
                if (u > 0) ld_block(toks + (size_t)(u - 1) * D * D, Spn);
                float kr[RPT], ar[RPT], qr[RPT];
                float4 pp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const int r = lane + 32 * i;
                    kr[i] = kval(tb, r);
                    qr[i] = qval(tb, r);
                    ar[i] = expf(fmaxf(gval(tb, r), -5.f));
                    const float ak = ar[i] * kr[i];
                    pp.x = fmaf(ak, Sp[i].x, pp.x); pp.y = fmaf(ak, Sp[i].y, pp.y);
                    pp.z = fmaf(ak, Sp[i].z, pp.z); pp.w = fmaf(ak, Sp[i].w, pp.w);
                }
                pp = warp_sum4(pp);                                 // p = S'^T k
                const float b = *reinterpret_cast<const float *>(tb + B::RB);
                const float4 vv = vval4(tb);
                const float4 do4 = *reinterpret_cast<const float4 *>(tb + B::RDO + 16 * w);
                const float4 vp = make_float4(vv.x - pp.x, vv.y - pp.y, vv.z - pp.z, vv.w - pp.w);
                const float4 dl = make_float4(b * vp.x, b * vp.y, b * vp.z, b * vp.w);
                // dS += q do^T; row partials of dq = S_t do; column partials of dd = dS^T k
                float4 cs = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const int r = lane + 32 * i;
                    dS[i].x = fmaf(qr[i], do4.x, dS[i].x); dS[i].y = fmaf(qr[i], do4.y, dS[i].y);
                    dS[i].z = fmaf(qr[i], do4.z, dS[i].z); dS[i].w = fmaf(qr[i], do4.w, dS[i].w);
                    const float4 St = make_float4(fmaf(kr[i], dl.x, ar[i] * Sp[i].x),
                                                  fmaf(kr[i], dl.y, ar[i] * Sp[i].y),
                                                  fmaf(kr[i], dl.z, ar[i] * Sp[i].z),
                                                  fmaf(kr[i], dl.w, ar[i] * Sp[i].w));
                    rq[w * D + r] = St.x * do4.x + St.y * do4.y + St.z * do4.z + St.w * do4.w;
                    cs.x = fmaf(dS[i].x, kr[i], cs.x); cs.y = fmaf(dS[i].y, kr[i], cs.y);
                    cs.z = fmaf(dS[i].z, kr[i], cs.z); cs.w = fmaf(dS[i].w, kr[i], cs.w);
                }
                const float4 dd = warp_sum4(cs);
                if (lane == 0) {
                    *reinterpret_cast<float4 *>(dv + tok_off(t, D) + jc) =
                        make_float4(b * dd.x, b * dd.y, b * dd.z, b * dd.w);
                    rq[3 * NW * D + w] = dd.x * vp.x + dd.y * vp.y + dd.z * vp.z + dd.w * vp.w;
                }
                const float4 dp = make_float4(-b * dd.x, -b * dd.y, -b * dd.z, -b * dd.w);
                // row partials of dk = dS delta + S' dp and of da = rowsum(dS' * S_{t-1}),
                // with dS' = dS + k dp^T; then dS <- Diag(a) dS'
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const int r = lane + 32 * i;
                    rq[NW * D + w * D + r] =
                        dS[i].x * dl.x + dS[i].y * dl.y + dS[i].z * dl.z + dS[i].w * dl.w +
                        ar[i] * (Sp[i].x * dp.x + Sp[i].y * dp.y + Sp[i].z * dp.z + Sp[i].w * dp.w);
                    dS[i].x = fmaf(kr[i], dp.x, dS[i].x); dS[i].y = fmaf(kr[i], dp.y, dS[i].y);
                    dS[i].z = fmaf(kr[i], dp.z, dS[i].z); dS[i].w = fmaf(kr[i], dp.w, dS[i].w);
                    rq[2 * NW * D + w * D + r] = dS[i].x * Sp[i].x + dS[i].y * Sp[i].y +
                                                dS[i].z * Sp[i].z + dS[i].w * Sp[i].w;
                    dS[i].x *= ar[i]; dS[i].y *= ar[i]; dS[i].z *= ar[i]; dS[i].w *= ar[i];
                }
#pragma unroll
                for (int i = 0; i < RPT; ++i) Sp[i] = Spn[i];
            }
            __syncthreads();
            // sums over the warps' columns, token by token
            if (tid < D) {
                for (int tau = 0; tau < cnt; ++tau) {
                    const int64_t t = t0 + hi - tau;
                    const float *rq = red + (size_t)tau * (3 * NW * D + NW);
                    float aq = 0.f, akk = 0.f, aa = 0.f;
#pragma unroll
                    for (int x = 0; x < NW; ++x) {
                        aq += rq[x * D + tid];
                        akk += rq[NW * D + x * D + tid];
                        aa += rq[2 * NW * D + x * D + tid];
                    }
                    if (NSL == 1) {
                        const float gv = gval(stg + (size_t)(buf * TB + tau) * TOKB, tid);
                        dq[tok_off(t, D) + tid] = aq;
                        dk[tok_off(t, D) + tid] = akk;
                        dg[tok_off(t, D) + tid] = aa * expf(fmaxf(gv, -5.f)) * (gv >= -5.f ? 1.f : 0.f);
                    } else {
                        float *pt = part + (((size_t)slice * rows + (ra + t)) * H + h) * PW;
                        pt[tid] = aq;
                        pt[D + tid] = akk;
                        pt[2 * D + tid] = aa;
                    }
                }
            }
            if (tid < cnt) {
                const int64_t t = t0 + hi - tid;
                const float *rq = red + (size_t)tid * (3 * NW * D + NW);
                float sb = 0.f;
#pragma unroll
                for (int x = 0; x < NW; ++x) sb += rq[3 * NW * D + x];
                if (NSL == 1) dbeta[(size_t)(ra + t) * H + h] = sb;
                else part[(((size_t)slice * rows + (ra + t)) * H + h) * PW + 3 * D] = sb;
            }
        }
    }
    if (dstate_in) st_block(dstate_in + sbase, dS);
}

// Sums of the column slices' partials, in slice order: dq, dk, dbeta, and
// dg = da a (0 where g < -5).  CTA (unit, i) takes rows i, i + G, ... of its
// sequence, one key channel per thread.
template <int D, int NSL, typename Tin>
__global__ void __launch_bounds__(D)
backward_reduce_kernel(const Tin *__restrict__ g, const int32_t *__restrict__ cu, int64_t T, int N,
                       int H, int64_t rows, int G, const float *__restrict__ part,
                       float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dg,
                       float *__restrict__ dbeta) {
    constexpr int PW = 3 * D + 4;
    const int unit = blockIdx.x / G, gi = blockIdx.x % G;
    const int n = unit / H, h = unit % H;
    if (n >= N) return;
    int64_t ra, rb;
    rows_of(cu, T, n, ra, rb);
    const int c = threadIdx.x;
    for (int64_t t = ra + gi; t < rb; t += G) {
        const size_t th = (size_t)t * H + h;
        float sq = 0.f, sk = 0.f, sa = 0.f, sb = 0.f;
#pragma unroll
        for (int s = 0; s < NSL; ++s) {
            const float *p = part + ((size_t)s * rows * H + th) * PW;
            sq += p[c];
            sk += p[D + c];
            sa += p[2 * D + c];
            if (c == 0) sb += p[3 * D];
        }
        const float gv = to_f32(g[th * D + c]);
        dq[th * D + c] = sq;
        dk[th * D + c] = sk;
        dg[th * D + c] = sa * expf(fmaxf(gv, -5.f)) * (gv >= -5.f ? 1.f : 0.f);
        if (c == 0) dbeta[th] = sb;
    }
}

}  // namespace bwd

size_t backward_workspace_bytes(int64_t rows, int N, int H, int d) {
    const int64_t chunk_states = ((rows + bwd::C - 1) / bwd::C + N) * (int64_t)H;
    const int64_t token_states = (int64_t)N * H * bwd::C;
    const int nsl = bwd::slices_for((int64_t)N * H);
    const int64_t partials = nsl > 1 ? (int64_t)nsl * rows * H * (3 * d + 4) : 0;
    const size_t simt = (size_t)(chunk_states + token_states) * d * d * sizeof(float) +
                        (size_t)partials * sizeof(float);
    // d = 128 may take the chunked path (bf16 inputs): room for either
    if (d != 128) return simt;
    const size_t chunked = backward_chunked_workspace_bytes(rows, N, H);
    return simt > chunked ? simt : chunked;
}

template <int D, int NSL, typename Tin>
static cudaError_t launch_bwd_t(const BackwardArgs &a, cudaStream_t st) {
    constexpr int DVS = D / NSL;
    const int64_t units = (int64_t)a.N * a.H;
    const int64_t chunk_states = ((a.rows + bwd::C - 1) / bwd::C + a.N) * (int64_t)a.H;
    const int64_t token_states = units * bwd::C;
    float *ws = (float *)a.workspace;
    float *part = ws + (size_t)(chunk_states + token_states) * D * D;
    cudaError_t e;
    if constexpr (DVS <= 64) {
        // warp-per-column-group form with batched token inputs
        using BB = bwd::BwdBatch<D, DVS, Tin>;
        const size_t smem = BB::SMEM;
        auto kern = bwd::backward_sliced_kernel<D, DVS, Tin>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)(units * NSL), BB::NTH, smem, st>>>(
            (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v, (const Tin *)a.g,
            (const Tin *)a.beta, a.state_in, a.cu_seqlens, a.T, a.N, a.H, a.rows, a.dout,
            a.dstate_out, a.dq, a.dk, a.dv, a.dg, a.dbeta, a.dstate_in, ws,
            ws + (size_t)chunk_states * D * D, part);
    } else {
        using L = bwd::Lay<D, DVS>;
        const size_t smem =
            (size_t)(5 * D + 7 * DVS + L::RG * DVS + 2 * (L::CG + 1) * D) * sizeof(float);
        auto kern = bwd::backward_kernel<D, DVS, Tin>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)(units * NSL), bwd::NT, smem, st>>>(
            (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v, (const Tin *)a.g,
            (const Tin *)a.beta, a.state_in, a.cu_seqlens, a.T, a.N, a.H, a.rows, a.dout,
            a.dstate_out, a.dq, a.dk, a.dv, a.dg, a.dbeta, a.dstate_in, ws,
            ws + (size_t)chunk_states * D * D, part);
    }
    e = cudaGetLastError();
    Profiler::mark(st);
    if constexpr (NSL > 1) {
        if (e != cudaSuccess) return e;
        // about eight CTAs per SM for the reduction
        const int G = (int)(units >= 1184 ? 1 : 1184 / units);
        bwd::backward_reduce_kernel<D, NSL, Tin><<<(unsigned)(units * G), D, 0, st>>>(
            (const Tin *)a.g, a.cu_seqlens, a.T, a.N, a.H, a.rows, G, part, a.dq, a.dk, a.dg,
            a.dbeta);
        e = cudaGetLastError();
        Profiler::mark(st);
    }
    return e;
}

template <int D, typename Tin>
static cudaError_t launch_bwd_d(const BackwardArgs &a, cudaStream_t st) {
    switch (bwd::slices_for((int64_t)a.N * a.H)) {
    case 4: return launch_bwd_t<D, 4, Tin>(a, st);
    case 2: return launch_bwd_t<D, 2, Tin>(a, st);
    default: return launch_bwd_t<D, 1, Tin>(a, st);
    }
}

cudaError_t launch_backward(const BackwardArgs &a, bool bf16, cudaStream_t st) {
    if (a.N * (int64_t)a.H == 0) return cudaSuccess;
    // bf16 at d = 128: through the chunked form on top of the tensor-core forward
    if (bf16 && a.d == 128) return launch_backward_chunked(a, st);
    if (a.d == 64)
        return bf16 ? launch_bwd_d<64, __nv_bfloat16>(a, st) : launch_bwd_d<64, float>(a, st);
    return bf16 ? launch_bwd_d<128, __nv_bfloat16>(a, st) : launch_bwd_d<128, float>(a, st);
}

}  // namespace kda
