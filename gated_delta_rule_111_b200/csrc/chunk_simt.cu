// Chunkwise prefill of the Gated DeltaNet-2 recurrence on CUDA cores, in FP32.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Token processing and parallel training": the
// sequence is cut into 64-token blocks; the per-channel decay accumulated since
// the block start is folded into the erase-side and key-side factors, so each
// block costs one unit-triangular system plus matrix products; decay, state and
// the triangular system are carried in FP32.
//
// This kernel is the FP32 path (q/k/v in FP32, tolerance 1e-4) and the path for
// every head size the tensor-core kernel does not cover.  Within a chunk of n
// tokens starting from state S (d_k x d_v), with g_t = sum_{j<=t} ln alpha_j
// (per key channel, inclusive) and e = b*k, z = w*v:
//   A[t,s] = sum_i e_t[i] k_s[i] exp(g_t[i] - g_s[i])   (s < t)
//   P[t,s] = sum_i q_t[i] k_s[i] exp(g_t[i] - g_s[i])   (s <= t)
//   (I + A) U = Z - Etil S,           Etil_t = e_t * exp(g_t)
//   O = Qtil S + P U,                 Qtil_t = q_t * exp(g_t)
//   S <- diag(exp(g_n)) S + Khat^T U, Khat_s = k_s * exp(g_n - g_s)
// Every exponent in A, P and Khat is of a difference g_t - g_s <= 0, so no
// factor can overflow for any alpha in (0, 1].  U holds the per-token
// corrections u_t = z_t - (diag(alpha_t) S_{t-1})^T e_t of the token recurrence.
//
// Grid: one CTA per (sequence*head, 32-column slice of d_v); the value columns
// of the recurrence evolve independently given the key-side quantities.  A
// sequence is either row block s of B sequences of T tokens, or, for packed
// variable-length batches, tokens cu_seqlens[s] .. cu_seqlens[s+1] - 1.
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kC = 64;        // chunk length
constexpr int kDVS = 32;      // value columns per CTA
constexpr int kThreads = 256;

template <int DK>
struct SimtSmem {
    static constexpr int LD = DK + 1;  // padded row stride: conflict-free column walks
    static constexpr int LDC = kC + 1;
    static constexpr size_t floats = 4 * (size_t)kC * LD + 2 * (size_t)kC * LDC + 2 * (size_t)kC * kDVS +
                                     (size_t)DK * kDVS + DK;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kThreads, 1)
chunk_simt_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                  const float *__restrict__ alpha, const float *__restrict__ bgate,
                  const float *__restrict__ wgate, const float *S0, TIn *__restrict__ o, float *S_T,
                  const int *cu_seqlens, int T, int H, int dv) {
    using SM = SimtSmem<DK>;
    constexpr int LD = SM::LD, LDC = SM::LDC;
    extern __shared__ float smem[];
    float *G = smem;                    // [kC][LD]  cumulative log-decay
    float *Kk = G + kC * LD;            // [kC][LD]  k, then Khat
    float *E = Kk + kC * LD;            // [kC][LD]  b*k, then Etil
    float *Qq = E + kC * LD;            // [kC][LD]  q, then Qtil
    float *A = Qq + kC * LD;            // [kC][LDC] strictly lower Gram
    float *P = A + kC * LDC;            // [kC][LDC] lower Gram incl. diagonal
    float *Z = P + kC * LDC;            // [kC][kDVS]
    float *U = Z + kC * kDVS;           // [kC][kDVS]
    float *Sst = U + kC * kDVS;         // [DK][kDVS] state slice
    float *gl = Sst + DK * kDVS;        // [DK] g at the chunk's last token

    const int head = blockIdx.x;        // sequence * H + h
    const int seq = head / H, h = head % H;
    // Tokens [tb, te) of the flat token index (seq * T + t, or packed offsets).
    int tb = seq * T, te = tb + T;
    if (cu_seqlens) {
        tb = min(max(cu_seqlens[seq], 0), T);
        te = min(max(cu_seqlens[seq + 1], tb), T);
    }
    const int len = te - tb;
    const int col0 = blockIdx.y * kDVS;
    const int tid = threadIdx.x;

    const size_t state_off = (size_t)head * DK * dv;
    for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
        const int i = idx / kDVS, j = idx % kDVS;
        Sst[idx] = S0 ? S0[state_off + (size_t)i * dv + col0 + j] : 0.f;
    }

    for (int c0 = 0; c0 < len; c0 += kC) {
        const int n = min(kC, len - c0);
        __syncthreads();
        // 1. Load the chunk; padding tokens act as k = q = e = z = 0, alpha = 1.
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            float g = 0.f, kk = 0.f, ee = 0.f, qq = 0.f;
            if (t < n) {
                const size_t off = ((size_t)(tb + c0 + t) * H + h) * DK + i;
                g = logf(clamp_alpha(__ldg(alpha + off)));
                kk = Elem<TIn>::load(k + off);
                ee = __ldg(bgate + off) * kk;
                qq = Elem<TIn>::load(q + off);
            }
            G[t * LD + i] = g; Kk[t * LD + i] = kk; E[t * LD + i] = ee; Qq[t * LD + i] = qq;
        }
        for (int idx = tid; idx < kC * kDVS; idx += kThreads) {
            const int t = idx / kDVS, j = idx % kDVS;
            float zz = 0.f;
            if (t < n) {
                const size_t off = ((size_t)(tb + c0 + t) * H + h) * dv + col0 + j;
                zz = __ldg(wgate + off) * Elem<TIn>::load(v + off);
            }
            Z[idx] = zz;
        }
        __syncthreads();
        // 2. Inclusive cumulative sum of ln alpha along the chunk, per key channel.
        if (tid < DK) {
            float run = 0.f;
            for (int t = 0; t < kC; ++t) { run += G[t * LD + tid]; G[t * LD + tid] = run; }
            gl[tid] = run;
        }
        __syncthreads();
        // 3. Gram matrices with the decay ratio formed from a difference of logs.
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int t = idx / kC, s = idx % kC;
            float a = 0.f, p = 0.f;
            if (s <= t) {
                const float *gt = G + t * LD, *gs = G + s * LD, *ks = Kk + s * LD;
                const float *et = E + t * LD, *qt = Qq + t * LD;
                for (int i = 0; i < DK; ++i) {
                    const float ks_d = ks[i] * expf(gt[i] - gs[i]);
                    a = fmaf(et[i], ks_d, a);
                    p = fmaf(qt[i], ks_d, p);
                }
            }
            A[t * LDC + s] = (s < t) ? a : 0.f;
            P[t * LDC + s] = p;
        }
        __syncthreads();
        // 4. Scale by the decay from the chunk start: Etil, Qtil; Khat from the chunk end.
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int t = idx / DK, i = idx % DK;
            const float g = G[t * LD + i];
            const float fwd = expf(g);
            E[t * LD + i] *= fwd;
            Qq[t * LD + i] *= fwd;
            Kk[t * LD + i] *= expf(gl[i] - g);
        }
        __syncthreads();
        // 5. Right-hand side Z - Etil S.
        for (int idx = tid; idx < kC * kDVS; idx += kThreads) {
            const int t = idx / kDVS, j = idx % kDVS;
            const float *et = E + t * LD;
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(et[i], Sst[i * kDVS + j], acc);
            U[idx] = Z[idx] - acc;
        }
        __syncthreads();
        // 6. Forward substitution (I + A) U = RHS, one thread per value column.
        if (tid < kDVS) {
            for (int t = 1; t < kC; ++t) {
                const float *at = A + t * LDC;
                float acc = U[t * kDVS + tid];
                for (int s = 0; s < t; ++s) acc = fmaf(-at[s], U[s * kDVS + tid], acc);
                U[t * kDVS + tid] = acc;
            }
        }
        __syncthreads();
        // 7. Outputs O = Qtil S + P U for the valid tokens.
        for (int idx = tid; idx < kC * kDVS; idx += kThreads) {
            const int t = idx / kDVS, j = idx % kDVS;
            if (t >= n) continue;
            const float *qt = Qq + t * LD, *pt = P + t * LDC;
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(qt[i], Sst[i * kDVS + j], acc);
            for (int s = 0; s <= t; ++s) acc = fmaf(pt[s], U[s * kDVS + j], acc);
            const size_t off = ((size_t)(tb + c0 + t) * H + h) * dv + col0 + j;
            Elem<TIn>::store(o + off, acc);
        }
        __syncthreads();
        // 8. State carry S <- diag(exp(g_n)) S + Khat^T U.
        for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
            const int i = idx / kDVS, j = idx % kDVS;
            float acc = expf(gl[i]) * Sst[idx];
            for (int s = 0; s < kC; ++s) acc = fmaf(Kk[s * LD + i], U[s * kDVS + j], acc);
            Sst[idx] = acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < DK * kDVS; idx += kThreads) {
            const int i = idx / kDVS, j = idx % kDVS;
            S_T[state_off + (size_t)i * dv + col0 + j] = Sst[idx];
        }
    }
}

template <typename TIn, int DK>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                         const float *w, const float *S0, void *o, float *S_T, int B, int T, int H, int dv,
                         const int *cu_seqlens, cudaStream_t stream) {
    auto kern = chunk_simt_kernel<TIn, DK>;
    const size_t smem = SimtSmem<DK>::bytes;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)B * (unsigned)H, (unsigned)(dv / kDVS));
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const TIn *>(q), static_cast<const TIn *>(k),
                                           static_cast<const TIn *>(v), alpha, b, w, S0,
                                           static_cast<TIn *>(o), S_T, cu_seqlens, T, H, dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *alpha,
                              const float *b, const float *w, const float *S0, void *o, float *S_T,
                              int B, int T, int H, int dk, int dv, gdn2_dtype dt, const int *cu_seqlens,
                              cudaStream_t stream) {
    if (dt == GDN2_BF16) {
        if (dk == 128)
            return launch_typed<__nv_bfloat16, 128>(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, dv, cu_seqlens, stream);
        return launch_typed<__nv_bfloat16, 64>(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, dv, cu_seqlens, stream);
    }
    if (dk == 128) return launch_typed<float, 128>(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, dv, cu_seqlens, stream);
    return launch_typed<float, 64>(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, dv, cu_seqlens, stream);
}

}  // namespace gdn2
