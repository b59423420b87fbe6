// Fused single-token decode step of the Gated DeltaNet-2 recurrence.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Independent decisions on two axes":
//   Sbar = diag(alpha) S;  e = b*k;  z = w*v;  r = Sbar^T e;  S' = Sbar + k (z - r)^T;  o = S'^T q.
// The recurrent mode for decode is named on the mindpattern.ai DeltaNet trail
// (fused recurrent for decode, chunkwise for training, identical mathematics).
//
// One CTA per (batch, head).  The state (d_k x d_v FP32, 64 KiB at d = 128) is
// read exactly once into registers with 16-byte streaming loads, and written
// exactly once.  Between the two, the CTA forms both column reductions it needs
// in the same sweep over the decayed rows:
//   r = Sbar^T e  and  p = Sbar^T q,
// and then o = S'^T q = p + (k . q)(z - r), so the updated state is never
// re-read.  Work per head: 2 d_k d_v FLOP-pairs; bytes per head: 2 * 4 d_k d_v
// plus the token vectors -- HBM-bound by a wide margin.
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
recurrent_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                      const float *__restrict__ alpha, const float *__restrict__ bgate,
                      const float *__restrict__ wgate, float *__restrict__ S, TIn *__restrict__ o) {
    constexpr int TPR = DV / 4;              // threads per state row (one float4 each)
    constexpr int RPP = kThreads / TPR;      // rows per pass
    constexpr int PASSES = DK / RPP;         // rows held per thread
    static_assert(DK % RPP == 0, "row tiling");
    static_assert(DK <= kThreads && DV <= kThreads, "one thread per channel in the prologue");

    __shared__ float s_alpha[DK], s_e[DK], s_q[DK], s_k[DK];
    __shared__ float s_z[DV], s_u[DV];
    __shared__ float s_red_r[RPP][DV], s_red_p[RPP][DV];
    __shared__ float s_kq[kThreads / 32];

    const int head = blockIdx.x;                    // b * H + h
    const int tid = threadIdx.x;
    const int cg = tid % TPR;                       // column group: columns 4cg .. 4cg+3
    const int rg = tid / TPR;                       // row group: rows rg + RPP * p
    float4 *Sh = reinterpret_cast<float4 *>(S + (size_t)head * DK * DV);

    // 1. Issue every state load first so the whole head is in flight at once.
    float4 s[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) s[p] = ld_stream(Sh + (rg + RPP * p) * TPR + cg);

    // 2. Token vectors: one thread per key channel, then one per value channel.
    float kq = 0.f;
    if (tid < DK) {
        const size_t off = (size_t)head * DK + tid;
        const float kk = Elem<TIn>::load(k + off), qq = Elem<TIn>::load(q + off);
        s_alpha[tid] = clamp_alpha(__ldg(alpha + off));
        s_e[tid] = __ldg(bgate + off) * kk;
        s_q[tid] = qq;
        s_k[tid] = kk;
        kq = kk * qq;
    }
    if (tid < DV) {
        const size_t off = (size_t)head * DV + tid;
        s_z[tid] = __ldg(wgate + off) * Elem<TIn>::load(v + off);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, m);
    if ((tid & 31) == 0) s_kq[tid >> 5] = kq;
    __syncthreads();

    // 3. Decay the rows in registers and accumulate both column reductions.
    float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), p4 = r4;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int i = rg + RPP * p;
        const float a = s_alpha[i], ei = s_e[i], qi = s_q[i];
        float4 x = s[p];
        x.x *= a; x.y *= a; x.z *= a; x.w *= a;
        s[p] = x;
        r4.x = fmaf(x.x, ei, r4.x); r4.y = fmaf(x.y, ei, r4.y); r4.z = fmaf(x.z, ei, r4.z); r4.w = fmaf(x.w, ei, r4.w);
        p4.x = fmaf(x.x, qi, p4.x); p4.y = fmaf(x.y, qi, p4.y); p4.z = fmaf(x.z, qi, p4.z); p4.w = fmaf(x.w, qi, p4.w);
    }
    reinterpret_cast<float4 *>(&s_red_r[rg][0])[cg] = r4;
    reinterpret_cast<float4 *>(&s_red_p[rg][0])[cg] = p4;
    __syncthreads();

    // 4. Finish the reductions: u = z - r, o = p + (k . q) u.
    if (tid < DV) {
        float r = 0.f, pp = 0.f;
#pragma unroll
        for (int g = 0; g < RPP; ++g) { r += s_red_r[g][tid]; pp += s_red_p[g][tid]; }
        float kqs = 0.f;
#pragma unroll
        for (int wv = 0; wv < (DK + 31) / 32; ++wv) kqs += s_kq[wv];
        const float u = s_z[tid] - r;
        s_u[tid] = u;
        Elem<TIn>::store(o + (size_t)head * DV + tid, fmaf(kqs, u, pp));
    }
    __syncthreads();

    // 5. Rank-1 delta write from registers: S' = Sbar + k u^T.
    const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const float ki = s_k[rg + RPP * p];
        float4 x = s[p];
        x.x = fmaf(ki, u4.x, x.x); x.y = fmaf(ki, u4.y, x.y); x.z = fmaf(ki, u4.z, x.z); x.w = fmaf(ki, u4.w, x.w);
        st_stream(Sh + (rg + RPP * p) * TPR + cg, x);
    }
}

template <typename TIn, int DK, int DV>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                         const float *w, float *S, void *o, int B, int H, cudaStream_t stream) {
    const unsigned grid = (unsigned)B * (unsigned)H;
    recurrent_step_kernel<TIn, DK, DV><<<grid, kThreads, 0, stream>>>(
        static_cast<const TIn *>(q), static_cast<const TIn *>(k), static_cast<const TIn *>(v), alpha, b, w, S,
        static_cast<TIn *>(o));
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_dims(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                        const float *w, float *S, void *o, int B, int H, int dk, int dv, cudaStream_t st) {
    if (dk == 128 && dv == 128) return launch_typed<TIn, 128, 128>(q, k, v, alpha, b, w, S, o, B, H, st);
    if (dk == 64 && dv == 64) return launch_typed<TIn, 64, 64>(q, k, v, alpha, b, w, S, o, B, H, st);
    if (dk == 128 && dv == 64) return launch_typed<TIn, 128, 64>(q, k, v, alpha, b, w, S, o, B, H, st);
    return launch_typed<TIn, 64, 128>(q, k, v, alpha, b, w, S, o, B, H, st);
}

}  // namespace

cudaError_t launch_recurrent_step(const void *q, const void *k, const void *v, const float *alpha,
                                  const float *b, const float *w, float *S, void *o, int B, int H,
                                  int dk, int dv, gdn2_dtype dt, cudaStream_t stream) {
    if (dt == GDN2_BF16)
        return launch_dims<__nv_bfloat16>(q, k, v, alpha, b, w, S, o, B, H, dk, dv, stream);
    return launch_dims<float>(q, k, v, alpha, b, w, S, o, B, H, dk, dv, stream);
}

}  // namespace gdn2
