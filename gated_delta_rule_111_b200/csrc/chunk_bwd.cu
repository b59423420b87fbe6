// Chunkwise backward of the Gated DeltaNet-2 recurrence, FP32 arithmetic on CUDA cores.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Token processing and parallel training": training
// needs the gradient of the chunkwise form with the channel-wise decay and the
// separate erase (b) and write (w) gates carried through every factor.  Per
// chunk of C = 64 tokens with start state S, log-decay g_t = sum_{j<=t} ln alpha_j
// (per key channel, relative to the chunk start), e = b k, z = w v,
//   Etil_t = e_t exp(g_t),  Qtil_t = q_t exp(g_t),  Khat_s = k_s exp(g_n - g_s),
//   A[t,s] = sum_i e_ti k_si exp(g_ti - g_si)  (s < t),   P[t,s] likewise with q (s <= t),
//   T = (I + A)^{-1},  U = T (Z - Etil S),  O = Qtil S + P U,  S' = diag(exp g_n) S + Khat^T U.
// With dO the chunk's output gradient and dS' the gradient of its end state:
//   dU = P^T dO + Khat dS',  dR = T^T dU,
//   dS = Qtil^T dO + diag(exp g_n) dS' - Etil^T dR            (carried to the previous chunk)
//   dP = dO U^T (s <= t),  dA = -dR U^T (s < t)
//   dq_t = exp(g_t) S dO_t + sum_{s<=t} dP[t,s] k_s exp(g_t - g_s)
//   de_t = -exp(g_t) S dR_t + sum_{s<t} dA[t,s] k_s exp(g_t - g_s)
//   dk_s = sum_{t>s} dA[t,s] e_t exp(g_t - g_s) + sum_{t>=s} dP[t,s] q_t exp(g_t - g_s)
//          + exp(g_n - g_s) dS' U_s + de_s b_s
//   db = de k,  dw = dR v,  dv = dR w,
//   dlog gamma_t = de_t e_t + dq_t q_t - (dk_t - de_t b_t) k_t, plus at the chunk's last
//          token exp(g_n) rowsum(S * dS') + sum_s Khat_s * (dS' U_s),
//   dalpha_j = (sum over the chunk's tokens t >= j of dlog gamma_t) / alpha_j.
// Every decay factor here is the exponential of a difference g_t - g_s <= 0 (or of
// g_t <= 0), so nothing overflows for any alpha in (0, 1].  alpha is taken as
// max(alpha, 2^-64), the value the prefill kernels compute with.  The cumulative
// log-decays are kept base 2 and as compensated (hi, lo) pairs, so a difference
// g_t - g_s keeps its own precision however large |g| has grown in the chunk.
//
// Three launches on the caller's stream:
//   prep   grid (chunk, sequence x head): A and P from differences of logs, T by
//          column-parallel forward substitution; T and P to the workspace.
//   state  grid (sequence x head, 32-column slice of d_v), serial over chunks: the
//          forward recurrence again (every chunk's start state and U to the
//          workspace), then the dS recurrence backwards (dR and every chunk's dS'
//          to the workspace, dS0 out).  Each CTA carries only its value columns.
//   grad   grid (chunk, sequence x head), independent CTAs: the contractions over
//          the value columns and the per-token gradients.
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kC = 64;            // chunk length
constexpr int kCS = 32;           // value columns per CTA of the state kernel
constexpr int kThreads = 256;
constexpr int LDT = kC + 1;       // row stride of 64 x 64 tiles in shared memory
constexpr int LDZ = kCS + 1;      // row stride of column-slice tiles
constexpr float kAlphaMin = 5.42101086e-20f;   // 2^-64

// log2 of the clamped decay, to an ulp (the exponentials below are base 2)
__device__ __forceinline__ float log2_alpha(const float *p) { return log2f(fmaxf(__ldg(p), kAlphaMin)); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// s = fl(a + b) and err with a + b = s + err exactly (Knuth's TwoSum).
__device__ __forceinline__ float two_sum(float a, float b, float &err) {
    const float s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    err = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
    return s;
}

// (hi_t + lo_t) - (hi_s + lo_s), the high parts subtracted first
__device__ __forceinline__ float gdiff(float ht, float lt, float hs, float ls) { return (ht - hs) + (lt - ls); }

// In place over a [64][ld] tile of NCH channels: hi holds log2(alpha) per token on
// entry (0 on padding rows); on exit hi + lo is the compensated prefix sum from the
// chunk start.  Each (channel, half of the chunk) runs over 32 tokens, then the
// second half adds the first half's total.  Ends with __syncthreads().
template <int NCH>
__device__ void comp_cumsum(float *hi, float *lo, int ld) {
    for (int idx = threadIdx.x; idx < 2 * NCH; idx += kThreads) {
        const int i = idx % NCH, half = idx / NCH;
        float run = 0.f, comp = 0.f, err;
        for (int t = half * 32; t < half * 32 + 32; ++t) {
            run = two_sum(run, hi[t * ld + i], err);
            comp += err;
            hi[t * ld + i] = run;
            lo[t * ld + i] = comp;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 32 * NCH; idx += kThreads) {
        const int t = 32 + idx / NCH, i = idx % NCH;
        float err;
        const float h = two_sum(hi[31 * ld + i], hi[t * ld + i], err);
        lo[t * ld + i] += lo[31 * ld + i] + err;
        hi[t * ld + i] = h;
    }
    __syncthreads();
}

// Workspace views (FP32).  nch = ceil(T / 64), units = B * H.
//   Sc  [units][nch][dk][dv]   state at the start of every chunk
//   dSc [units][nch][dk][dv]   gradient of every chunk's end state
//   TP  [units][nch][2][64][64]  T = (I + A)^{-1}, then P
//   U, dR [B][T][H][dv]        per token, laid out like o
struct Ws {
    float *Sc, *dSc, *TP, *U, *dR;
};

// acc[r][c] += sum_k A(m, k) B(k, n) on shared-memory operands, with A(m, k) at
// A[m*sam + k*sak] and B(k, n) at B[k*sbk + n*sbn].  Thread tid owns the outputs
// m = mg + r*MG, n = ng + c*NG (interleaved, so a warp's loads fall in distinct
// banks for the strides used here).
template <int M, int N, int TM, int TN>
struct Mm {
    static constexpr int NG = N / TN, MG = M / TM;
    static_assert(MG * NG == kThreads, "one output micro-tile per thread");
    __device__ static int mg() { return threadIdx.x / NG; }
    __device__ static int ng() { return threadIdx.x % NG; }
    __device__ static void zero(float (&acc)[TM][TN]) {
#pragma unroll
        for (int r = 0; r < TM; ++r)
#pragma unroll
            for (int c = 0; c < TN; ++c) acc[r][c] = 0.f;
    }
    __device__ static void run(float (&acc)[TM][TN], const float *A, int sam, int sak, const float *B, int sbk,
                               int sbn, int K) {
        const int m0 = mg(), n0 = ng();
#pragma unroll 4
        for (int kk = 0; kk < K; ++kk) {
            float a[TM], b[TN];
#pragma unroll
            for (int r = 0; r < TM; ++r) a[r] = A[(m0 + r * MG) * sam + kk * sak];
#pragma unroll
            for (int c = 0; c < TN; ++c) b[c] = B[kk * sbk + (n0 + c * NG) * sbn];
#pragma unroll
            for (int r = 0; r < TM; ++r)
#pragma unroll
                for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
    }
};

// ---------------------------------------------------------------------------
// prep: A, P, T of one chunk.
template <int DK>
struct PrepSmem {
    static constexpr int LB = 33;
    static constexpr size_t floats = 5 * (size_t)kC * LB + 3 * (size_t)kC * LDT;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kThreads)
bwd_prep_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const float *__restrict__ alpha,
                const float *__restrict__ bgate, float *TP, int T, int H) {
    constexpr int LB = PrepSmem<DK>::LB;
    extern __shared__ float smem[];
    float *cg = smem, *cl = cg + kC * LB, *ck = cl + kC * LB, *ce = ck + kC * LB, *cq = ce + kC * LB;
    float *sA = cq + kC * LB, *sP = sA + kC * LDT, *sT = sP + kC * LDT;
    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;

    // thread owns (t = tid/64 + 4r, s = tid%64), r = 0..15
    float a[16], p[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) a[r] = p[r] = 0.f;
    const int s = tid & 63, tb = tid >> 6;
    for (int ib = 0; ib < DK; ib += 32) {
        __syncthreads();
        for (int idx = tid; idx < kC * 32; idx += kThreads) {
            const int t = idx >> 5, i = idx & 31;
            float g = 0.f, kk = 0.f, qq = 0.f, ee = 0.f;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DK + ib + i;
                g = log2_alpha(alpha + off);
                kk = Elem<TIn>::load(k + off);
                qq = Elem<TIn>::load(q + off);
                ee = __ldg(bgate + off) * kk;
            }
            cg[t * LB + i] = g; ck[t * LB + i] = kk; cq[t * LB + i] = qq; ce[t * LB + i] = ee;
        }
        __syncthreads();
        comp_cumsum<32>(cg, cl, LB);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int t = tb + 4 * r;
            if (s <= t) {
                const float *gt = cg + t * LB, *gs = cg + s * LB, *lt = cl + t * LB, *ls = cl + s * LB,
                            *ks = ck + s * LB, *et = ce + t * LB, *qt = cq + t * LB;
                float aa = a[r], pp = p[r];
#pragma unroll 8
                for (int i = 0; i < 32; ++i) {
                    const float kd = ks[i] * ex2(gdiff(gt[i], lt[i], gs[i], ls[i]));
                    aa = fmaf(et[i], kd, aa);
                    pp = fmaf(qt[i], kd, pp);
                }
                a[r] = aa; p[r] = pp;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int t = tb + 4 * r;
        sA[t * LDT + s] = (s < t) ? a[r] : 0.f;
        sP[t * LDT + s] = (s <= t) ? p[r] : 0.f;
    }
    __syncthreads();
    // T = (I + A)^{-1}: column j by four lanes, x_t = -sum_{j<=s<t} A[t,s] x_s
    {
        const int j = tid >> 2, part = tid & 3;
        for (int t = 0; t < kC; ++t) {
            float acc = 0.f;
            if (t > j)
                for (int u = j + part; u < t; u += 4) acc = fmaf(sA[t * LDT + u], sT[u * LDT + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (part == 0) sT[t * LDT + j] = (t < j) ? 0.f : (t == j ? 1.f : -acc);
            __syncwarp();
        }
    }
    __syncthreads();
    float *dst = TP + ((size_t)unit * nch + c) * 2 * kC * kC;
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
        const int t = idx >> 6, u = idx & 63;
        dst[idx] = sT[t * LDT + u];
        dst[kC * kC + idx] = sP[t * LDT + u];
    }
}

// ---------------------------------------------------------------------------
// state: the two serial sweeps for one (sequence, head, column slice).
template <int DK>
struct StateSmem {
    static constexpr int LD = DK + 1;
    static constexpr size_t floats =
        3 * (size_t)kC * LD + 2 * (size_t)kC * LDT + 3 * (size_t)kC * LDZ + 2 * (size_t)DK * LDZ + 2 * DK;
    static constexpr size_t bytes = floats * sizeof(float);
};

// Loads the key side of chunk [c0, c0 + n): G = cumulative log2 alpha (hi in Qt,
// lo in Et), then Et = b k 2^G, Kh = k 2^(g_n - G), and (with_q) Qt = q 2^G;
// gl = (hi, lo) of g_n.  Padding rows are zero and hold G at its last value.
template <typename TIn, int DK>
__device__ void state_key_side(const TIn *q, const TIn *k, const float *alpha, const float *bgate, size_t tok0,
                               int n, int H, int h, float *Et, float *Kh, float *Qt, float *gl, bool with_q) {
    constexpr int LD = DK + 1;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < kC * DK; idx += kThreads) {
        const int t = idx / DK, i = idx % DK;
        Qt[t * LD + i] = (t < n) ? log2_alpha(alpha + ((tok0 + t) * H + h) * DK + i) : 0.f;
    }
    __syncthreads();
    comp_cumsum<DK>(Qt, Et, LD);
    for (int idx = tid; idx < DK; idx += kThreads) {
        gl[idx] = Qt[(kC - 1) * LD + idx];
        gl[DK + idx] = Et[(kC - 1) * LD + idx];
    }
    __syncthreads();
    for (int idx = tid; idx < kC * DK; idx += kThreads) {
        const int t = idx / DK, i = idx % DK;
        const float gh = Qt[t * LD + i], glo = Et[t * LD + i];
        float kk = 0.f, bb = 0.f, qq = 0.f;
        if (t < n) {
            const size_t off = ((tok0 + t) * H + h) * DK + i;
            kk = Elem<TIn>::load(k + off);
            bb = __ldg(bgate + off);
            if (with_q) qq = Elem<TIn>::load(q + off);
        }
        const float f = ex2(gh + glo);
        Et[t * LD + i] = bb * kk * f;
        Kh[t * LD + i] = kk * ex2(gdiff(gl[i], gl[DK + i], gh, glo));
        if (with_q) Qt[t * LD + i] = qq * f;
    }
}

template <typename TIn, int DK>
__global__ void __launch_bounds__(kThreads, 1)
bwd_state_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                 const float *__restrict__ alpha, const float *__restrict__ bgate, const float *__restrict__ wgate,
                 const float *S0, const TIn *__restrict__ dO, const float *dST, float *dS0, Ws ws, int T, int H,
                 int dv) {
    constexpr int LD = DK + 1;
    using M64 = Mm<kC, kCS, 4, 2>;          // 64 x 32 outputs
    using MDK = Mm<DK, kCS, DK / 16, 2>;    // DK x 32 outputs
    extern __shared__ float smem[];
    float *Et = smem, *Kh = Et + kC * LD, *Qt = Kh + kC * LD;
    float *Tm = Qt + kC * LD, *Pm = Tm + kC * LDT;
    float *Z = Pm + kC * LDT, *U = Z + kC * LDZ, *W = U + kC * LDZ;
    float *Sst = W + kC * LDZ, *dS = Sst + DK * LDZ, *gl = dS + DK * LDZ;     // gl: [2][DK]

    const int unit = blockIdx.x, seq = unit / H, h = unit % H;
    const int col0 = blockIdx.y * kCS, tid = threadIdx.x;
    const size_t tokb = (size_t)seq * T;
    const int nch = (T + kC - 1) / kC;
    const size_t soff = (size_t)unit * DK * dv;
    const int m64 = M64::mg(), n64 = M64::ng(), mdk = MDK::mg(), ndk = MDK::ng();

    for (int idx = tid; idx < DK * kCS; idx += kThreads) {
        const int i = idx / kCS, j = idx % kCS;
        Sst[i * LDZ + j] = S0 ? S0[soff + (size_t)i * dv + col0 + j] : 0.f;
    }
    // ---------------- forward sweep: chunk start states and U
    for (int c = 0; c < nch; ++c) {
        const int c0 = c * kC, n = min(kC, T - c0);
        const size_t chunk = (size_t)unit * nch + c;
        __syncthreads();
        for (int idx = tid; idx < DK * kCS; idx += kThreads) {
            const int i = idx / kCS, j = idx % kCS;
            ws.Sc[chunk * DK * dv + (size_t)i * dv + col0 + j] = Sst[i * LDZ + j];
        }
        state_key_side<TIn, DK>(q, k, alpha, bgate, tokb + c0, n, H, h, Et, Kh, Qt, gl, false);
        const float *tp = ws.TP + chunk * 2 * kC * kC;
        for (int idx = tid; idx < kC * kC; idx += kThreads) Tm[(idx >> 6) * LDT + (idx & 63)] = tp[idx];
        for (int idx = tid; idx < kC * kCS; idx += kThreads) {
            const int t = idx / kCS, j = idx % kCS;
            float zz = 0.f;
            if (t < n) {
                const size_t off = ((tokb + c0 + t) * H + h) * dv + col0 + j;
                zz = __ldg(wgate + off) * Elem<TIn>::load(v + off);
            }
            Z[t * LDZ + j] = zz;
        }
        __syncthreads();
        {   // W = Z - Et S
            float acc[4][2];
            M64::zero(acc);
            M64::run(acc, Et, LD, 1, Sst, LDZ, 1, DK);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int t = m64 + r * 16, j = n64 + cc * 16;
                    W[t * LDZ + j] = Z[t * LDZ + j] - acc[r][cc];
                }
        }
        __syncthreads();
        {   // U = T W
            float acc[4][2];
            M64::zero(acc);
            M64::run(acc, Tm, LDT, 1, W, LDZ, 1, kC);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int t = m64 + r * 16, j = n64 + cc * 16;
                    U[t * LDZ + j] = acc[r][cc];
                    if (t < n) ws.U[((tokb + c0 + t) * H + h) * dv + col0 + j] = acc[r][cc];
                }
        }
        __syncthreads();
        {   // S <- diag(exp g_n) S + Kh^T U
            float acc[DK / 16][2];
            MDK::zero(acc);
            MDK::run(acc, Kh, 1, LD, U, LDZ, 1, kC);
#pragma unroll
            for (int r = 0; r < DK / 16; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int i = mdk + r * 16, j = ndk + cc * 16;
                    Sst[i * LDZ + j] = fmaf(ex2(gl[i] + gl[DK + i]), Sst[i * LDZ + j], acc[r][cc]);
                }
        }
    }
    // ---------------- backward sweep: the dS recurrence
    __syncthreads();
    for (int idx = tid; idx < DK * kCS; idx += kThreads) {
        const int i = idx / kCS, j = idx % kCS;
        dS[i * LDZ + j] = dST ? dST[soff + (size_t)i * dv + col0 + j] : 0.f;
    }
    for (int c = nch - 1; c >= 0; --c) {
        const int c0 = c * kC, n = min(kC, T - c0);
        const size_t chunk = (size_t)unit * nch + c;
        __syncthreads();
        for (int idx = tid; idx < DK * kCS; idx += kThreads) {
            const int i = idx / kCS, j = idx % kCS;
            ws.dSc[chunk * DK * dv + (size_t)i * dv + col0 + j] = dS[i * LDZ + j];
        }
        state_key_side<TIn, DK>(q, k, alpha, bgate, tokb + c0, n, H, h, Et, Kh, Qt, gl, true);
        const float *tp = ws.TP + chunk * 2 * kC * kC;
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            Tm[(idx >> 6) * LDT + (idx & 63)] = tp[idx];
            Pm[(idx >> 6) * LDT + (idx & 63)] = tp[kC * kC + idx];
        }
        for (int idx = tid; idx < kC * kCS; idx += kThreads) {
            const int t = idx / kCS, j = idx % kCS;
            float d = 0.f;
            if (t < n) d = Elem<TIn>::load(dO + ((tokb + c0 + t) * H + h) * dv + col0 + j);
            Z[t * LDZ + j] = d;
        }
        __syncthreads();
        {   // dU = P^T dO + Kh dS
            float acc[4][2];
            M64::zero(acc);
            M64::run(acc, Pm, 1, LDT, Z, LDZ, 1, kC);
            M64::run(acc, Kh, LD, 1, dS, LDZ, 1, DK);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) W[(m64 + r * 16) * LDZ + n64 + cc * 16] = acc[r][cc];
        }
        __syncthreads();
        {   // dR = T^T dU
            float acc[4][2];
            M64::zero(acc);
            M64::run(acc, Tm, 1, LDT, W, LDZ, 1, kC);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int t = m64 + r * 16, j = n64 + cc * 16;
                    U[t * LDZ + j] = acc[r][cc];
                    if (t < n) ws.dR[((tokb + c0 + t) * H + h) * dv + col0 + j] = acc[r][cc];
                }
        }
        __syncthreads();
        {   // dS <- diag(exp g_n) dS + Qt^T dO - Et^T dR
            float acc[DK / 16][2], neg[DK / 16][2];
            MDK::zero(acc);
            MDK::zero(neg);
            MDK::run(acc, Qt, 1, LD, Z, LDZ, 1, kC);
            MDK::run(neg, Et, 1, LD, U, LDZ, 1, kC);
#pragma unroll
            for (int r = 0; r < DK / 16; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int i = mdk + r * 16, j = ndk + cc * 16;
                    dS[i * LDZ + j] = fmaf(ex2(gl[i] + gl[DK + i]), dS[i * LDZ + j], acc[r][cc] - neg[r][cc]);
                }
        }
    }
    __syncthreads();
    if (dS0) {
        for (int idx = tid; idx < DK * kCS; idx += kThreads) {
            const int i = idx / kCS, j = idx % kCS;
            dS0[soff + (size_t)i * dv + col0 + j] = dS[i * LDZ + j];
        }
    }
}

// ---------------------------------------------------------------------------
// grad: per-token gradients of one chunk.  Key channels in blocks of 32.
template <int DV>
struct GradSmem {
    static constexpr int LDV = DV + 1, LB = 33;
    static constexpr size_t floats = 3 * (size_t)kC * LDV + 2 * (size_t)kC * LDT + 2 * 32 * (size_t)LDV +
                                     7 * (size_t)kC * LB + 32;
    static_assert(2 * 32 * LDV >= kC * LB, "the lo tile fits where S and dS' were");
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_grad_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                const float *__restrict__ alpha, const float *__restrict__ bgate, const float *__restrict__ wgate,
                const TIn *__restrict__ dO, Ws ws, TIn *dq, TIn *dk, TIn *dvv, float *dalpha, float *db,
                float *dw, int T, int H) {
    constexpr int LDV = GradSmem<DV>::LDV, LB = GradSmem<DV>::LB;
    using MP = Mm<kC, kC, 4, 4>;     // 64 x 64 outputs
    using MX = Mm<kC, 32, 4, 2>;     // 64 x 32 outputs
    extern __shared__ float smem[];
    float *sO = smem, *sU = sO + kC * LDV, *sR = sU + kC * LDV;
    float *dP = sR + kC * LDV, *dA = dP + kC * LDT;
    float *sS = dA + kC * LDT, *sD = sS + 32 * LDV;
    float *cg = sD + 32 * LDV, *ck = cg + kC * LB, *cq = ck + kC * LB, *ce = cq + kC * LB;
    float *X1 = ce + kC * LB, *X2 = X1 + kC * LB, *Y = X2 + kC * LB;
    float *rs = Y + kC * LB;
    float *cl = sS;                     // lo parts of the cumulative log decay, once sS, sD are consumed

    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;
    const size_t chunk = (size_t)unit * nch + c;

    for (int idx = tid; idx < kC * DV; idx += kThreads) {
        const int t = idx / DV, j = idx % DV;
        float o = 0.f, u = 0.f, r = 0.f;
        if (t < n) {
            const size_t off = ((tok0 + t) * H + h) * DV + j;
            o = Elem<TIn>::load(dO + off);
            u = ws.U[off];
            r = ws.dR[off];
            dw[off] = r * Elem<TIn>::load(v + off);
            Elem<TIn>::store(dvv + off, r * __ldg(wgate + off));
        }
        sO[t * LDV + j] = o; sU[t * LDV + j] = u; sR[t * LDV + j] = r;
    }
    __syncthreads();
    {   // dP = dO U^T (s <= t), dA = -dR U^T (s < t)
        float ap[4][4], aa[4][4];
        MP::zero(ap);
        MP::zero(aa);
        MP::run(ap, sO, LDV, 1, sU, 1, LDV, DV);
        MP::run(aa, sR, LDV, 1, sU, 1, LDV, DV);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int t = MP::mg() + r * 16, s = MP::ng() + cc * 16;
                dP[t * LDT + s] = (s <= t) ? ap[r][cc] : 0.f;
                dA[t * LDT + s] = (s < t) ? -aa[r][cc] : 0.f;
            }
    }
    for (int ib = 0; ib < DK; ib += 32) {
        __syncthreads();
        const float *sc = ws.Sc + chunk * DK * DV + (size_t)ib * DV;
        const float *dsc = ws.dSc + chunk * DK * DV + (size_t)ib * DV;
        for (int idx = tid; idx < 32 * DV; idx += kThreads) {
            const int i = idx / DV, j = idx % DV;
            sS[i * LDV + j] = sc[idx];
            sD[i * LDV + j] = dsc[idx];
        }
        for (int idx = tid; idx < kC * 32; idx += kThreads) {
            const int t = idx >> 5, i = idx & 31;
            float g = 0.f, kk = 0.f, qq = 0.f, ee = 0.f;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DK + ib + i;
                g = log2_alpha(alpha + off);
                kk = Elem<TIn>::load(k + off);
                qq = Elem<TIn>::load(q + off);
                ee = __ldg(bgate + off) * kk;
            }
            cg[t * LB + i] = g; ck[t * LB + i] = kk; cq[t * LB + i] = qq; ce[t * LB + i] = ee;
        }
        __syncthreads();
        if (tid < 32) {                 // row sums of S * dS'
            float acc = 0.f;
            for (int j = 0; j < DV; ++j) acc = fmaf(sS[tid * LDV + j], sD[tid * LDV + j], acc);
            rs[tid] = acc;
        }
        {   // X1 = S dO, X2 = S dR, Y = dS' U, as [token][channel]
            float x1[4][2], x2[4][2], y[4][2];
            MX::zero(x1);
            MX::zero(x2);
            MX::zero(y);
            MX::run(x1, sO, LDV, 1, sS, 1, LDV, DV);
            MX::run(x2, sR, LDV, 1, sS, 1, LDV, DV);
            MX::run(y, sU, LDV, 1, sD, 1, LDV, DV);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int t = MX::mg() + r * 16, i = MX::ng() + cc * 16;
                    X1[t * LB + i] = x1[r][cc]; X2[t * LB + i] = x2[r][cc]; Y[t * LB + i] = y[r][cc];
                }
        }
        __syncthreads();
        comp_cumsum<32>(cg, cl, LB);        // S and dS' are consumed: cl takes their place
        float dlg[kC * 32 / kThreads];
#pragma unroll
        for (int e = 0; e < kC * 32 / kThreads; ++e) {
            const int idx = tid + e * kThreads, t = idx >> 5, i = idx & 31;
            const float gt = cg[t * LB + i], lt = cl[t * LB + i];
            const float gnh = cg[(kC - 1) * LB + i], gnl = cl[(kC - 1) * LB + i];
            float sq = 0.f, se = 0.f, sk = 0.f;
            for (int s = 0; s <= t; ++s) {          // dq, de: earlier keys of the chunk
                const float r = ck[s * LB + i] * ex2(gdiff(gt, lt, cg[s * LB + i], cl[s * LB + i]));
                sq = fmaf(dP[t * LDT + s], r, sq);
                se = fmaf(dA[t * LDT + s], r, se);
            }
            for (int u = t; u < kC; ++u) {          // dk: later tokens of the chunk
                const float r = ex2(gdiff(cg[u * LB + i], cl[u * LB + i], gt, lt));
                sk = fmaf(fmaf(dA[u * LDT + t], ce[u * LB + i], dP[u * LDT + t] * cq[u * LB + i]), r, sk);
            }
            const float ft = ex2(gt + lt);
            const float dqv = fmaf(ft, X1[t * LB + i], sq);
            const float dev = fmaf(-ft, X2[t * LB + i], se);
            const float kkey = fmaf(ex2(gdiff(gnh, gnl, gt, lt)), Y[t * LB + i], sk);
            const float kk = ck[t * LB + i];
            float l = dev * ce[t * LB + i] + dqv * cq[t * LB + i] - kkey * kk;
            if (t == n - 1) {               // through g_n: diag(exp g_n) S and every Khat_s
                float kh = 0.f;
                for (int s2 = 0; s2 < n; ++s2)
                    kh = fmaf(ck[s2 * LB + i] * ex2(gdiff(gnh, gnl, cg[s2 * LB + i], cl[s2 * LB + i])), Y[s2 * LB + i], kh);
                l += fmaf(ex2(gnh + gnl), rs[i], kh);
            }
            dlg[e] = (t < n) ? l : 0.f;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DK + ib + i;
                Elem<TIn>::store(dq + off, dqv);
                db[off] = dev * kk;
                Elem<TIn>::store(dk + off, fmaf(dev, __ldg(bgate + off), kkey));
            }
        }
        __syncthreads();                    // X2 is free now: it takes dlog gamma
#pragma unroll
        for (int e = 0; e < kC * 32 / kThreads; ++e) {
            const int idx = tid + e * kThreads;
            X2[(idx >> 5) * LB + (idx & 31)] = dlg[e];
        }
        __syncthreads();
        if (tid < 32) {                     // dalpha = reverse cumulative sum / alpha
            float run = 0.f;
            for (int t = n - 1; t >= 0; --t) {
                run += X2[t * LB + tid];
                const size_t off = ((tok0 + t) * H + h) * DK + ib + tid;
                dalpha[off] = run / fmaxf(__ldg(alpha + off), kAlphaMin);
            }
        }
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename TIn, int DK, int DV>
cudaError_t launch_bwd_typed(const void *q_, const void *k_, const void *v_, const float *alpha, const float *b,
                             const float *w, const float *S0, const void *dO_, const float *dST, void *dq, void *dk,
                             void *dv, float *dalpha, float *db, float *dw, float *dS0, Ws ws, int B, int T, int H,
                             cudaStream_t stream) {
    const TIn *q = static_cast<const TIn *>(q_), *k = static_cast<const TIn *>(k_),
              *v = static_cast<const TIn *>(v_), *dO = static_cast<const TIn *>(dO_);
    const int nch = (T + kC - 1) / kC, units = B * H;
    auto kp = bwd_prep_kernel<TIn, DK>;
    auto ks = bwd_state_kernel<TIn, DK>;
    auto kg = bwd_grad_kernel<TIn, DK, DV>;
    cudaError_t err;
    if ((err = set_smem(kp, PrepSmem<DK>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(ks, StateSmem<DK>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(kg, GradSmem<DV>::bytes)) != cudaSuccess) return err;
    kp<<<dim3((unsigned)nch, (unsigned)units), kThreads, PrepSmem<DK>::bytes, stream>>>(q, k, alpha, b, ws.TP, T, H);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    ks<<<dim3((unsigned)units, (unsigned)(DV / kCS)), kThreads, StateSmem<DK>::bytes, stream>>>(
        q, k, v, alpha, b, w, S0, dO, dST, dS0, ws, T, H, DV);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    kg<<<dim3((unsigned)nch, (unsigned)units), kThreads, GradSmem<DV>::bytes, stream>>>(
        q, k, v, alpha, b, w, dO, ws, static_cast<TIn *>(dq), static_cast<TIn *>(dk), static_cast<TIn *>(dv), dalpha,
        db, dw, T, H);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_bwd_dt(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                          const float *w, const float *S0, const void *dO, const float *dST, void *dq, void *dk,
                          void *dv, float *dalpha, float *db, float *dw, float *dS0, Ws ws, int B, int T, int H,
                          int d_k, int d_v, cudaStream_t s) {
#define GDN2_BWD(DK_, DV_)                                                                                        \
    if (d_k == DK_ && d_v == DV_)                                                                                 \
        return launch_bwd_typed<TIn, DK_, DV_>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, \
                                               ws, B, T, H, s);
    GDN2_BWD(128, 128)
    GDN2_BWD(128, 64)
    GDN2_BWD(64, 128)
    GDN2_BWD(64, 64)
#undef GDN2_BWD
    return cudaErrorInvalidValue;
}

}  // namespace

size_t chunk_bwd_workspace_floats(int B, int T, int H, int dk, int dv) {
    const size_t nch = (size_t)(T + kC - 1) / kC, units = (size_t)B * H;
    return 2 * units * nch * dk * dv + units * nch * 2 * kC * kC + 2 * (size_t)B * T * H * dv;
}

cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                             const float *w, const float *S0, const void *dO, const float *dST, void *dq, void *dk,
                             void *dv, float *dalpha, float *db, float *dw, float *dS0, float *workspace, int B,
                             int T, int H, int d_k, int d_v, gdn2_dtype dt, cudaStream_t stream) {
    const size_t nch = (size_t)(T + kC - 1) / kC, units = (size_t)B * H;
    Ws ws;
    ws.Sc = workspace;
    ws.dSc = ws.Sc + units * nch * d_k * d_v;
    ws.TP = ws.dSc + units * nch * d_k * d_v;
    ws.U = ws.TP + units * nch * 2 * kC * kC;
    ws.dR = ws.U + (size_t)B * T * H * d_v;
    if (dt == GDN2_BF16)
        return launch_bwd_dt<__nv_bfloat16>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, ws, B,
                                            T, H, d_k, d_v, stream);
    return launch_bwd_dt<float>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, ws, B, T, H, d_k,
                                d_v, stream);
}

}  // namespace gdn2
