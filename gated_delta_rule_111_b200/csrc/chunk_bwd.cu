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
// Five launches on the caller's stream.  Everything that does not depend on the
// carried state is computed for all chunks in parallel first, so the serial part
// is two matrix products per chunk and direction:
//   prep   grid (chunk, sequence x head): A and P from differences of logs, T by
//          column-parallel forward substitution; Etil, Khat, Qtil and 2^(g_n).
//   prep2  grid (chunk, sequence x head): T Etil, T^T Khat, T Z, T^T P^T dO and
//          Qtil^T dO, so that per chunk
//            U  = (T Z) - (T Etil) S,              S'  = diag(2^g_n) S + Khat^T U,
//            dR = (T^T P^T dO) + (T^T Khat) dS',   dS  = diag(2^g_n) dS' + Qtil^T dO - Etil^T dR.
//   state  grid (sequence x head, 32-column slice of d_v), serial over chunks: the
//          forward sweep (every chunk's start state and U to the workspace), then
//          the backward sweep (every chunk's dS' and dR, and dS0).  The next
//          chunk's operand tiles stream into a second shared-memory buffer
//          (cp.async) while the current chunk computes.
//   grad   grid (chunk, sequence x head), independent CTAs: the contractions over
//          the value columns and the per-token gradients.
#include "common.cuh"
#include "mma_sync.cuh"

namespace gdn2 {
namespace {

constexpr int kC = 64;            // chunk length
constexpr int kCS = 32;           // value columns per CTA of the state kernel
constexpr int kThreads = 256;
constexpr int kThreadsB = 512;   // the gradient gathers (grad_b): 16 warps, to hide their load latency
constexpr int LDT = kC + 1;       // row stride of 64 x 64 tiles in shared memory
constexpr float kAlphaMin = 5.42101086e-20f;   // 2^-64; log2f of the clamped decay is accurate to an ulp

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
template <int NCH, int NT = kThreads>
__device__ void comp_cumsum(float *hi, float *lo, int ld) {
    for (int idx = threadIdx.x; idx < 2 * NCH; idx += NT) {
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
    for (int idx = threadIdx.x; idx < 32 * NCH; idx += NT) {
        const int t = 32 + idx / NCH, i = idx % NCH;
        float err;
        const float h = two_sum(hi[31 * ld + i], hi[t * ld + i], err);
        lo[t * ld + i] += lo[31 * ld + i] + err;
        hi[t * ld + i] = h;
    }
    __syncthreads();
}

// 16-byte asynchronous global -> shared copies (completion by wait_group: no spin loop).
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// rows x cols floats (cols a multiple of 4; both row strides multiples of 4 floats), by NT threads.
template <int NT = kThreads>
__device__ __forceinline__ void copy_tile_async(float *dst, int dst_ld, const float *src, size_t src_ld, int rows,
                                                int cols) {
    const int per = cols >> 2;
    for (int idx = threadIdx.x; idx < rows * per; idx += NT) {
        const int r = idx / per, c4 = (idx - r * per) << 2;
        cp_async16(dst + r * dst_ld + c4, src + r * src_ld + c4);
    }
}

// Per-chunk key block of the workspace (FP32, rows padded by 4 floats):
//   Et, Kh, Qt, TEt = T Et, TKh = T^T Kh    [64][DK + 4] each
//   TZ = T Z, TPdO = T^T P^T dO              [64][DV + 4] each
//   QdO = Qt^T dO                            [DK][DV + 4]
//   gnf = 2^(g_n)                            [DK]
template <int DK, int DV>
struct Kb {
    static constexpr int LK = DK + 4, LV = DV + 4;
    static constexpr size_t ET = 0, KH = ET + kC * LK, QT = KH + kC * LK, TET = QT + kC * LK, TKH = TET + kC * LK,
                            TZ = TKH + kC * LK, TPDO = TZ + kC * LV, QDO = TPDO + kC * LV, GNF = QDO + DK * LV,
                            floats = GNF + DK;
    static_assert(floats % 4 == 0, "16-byte aligned blocks");
};

// Workspace views (FP32).  nch = ceil(T / 64), units = B * H.
//   Sc  [units][nch][dk][dv]   state at the start of every chunk
//   dSc [units][nch][dk][dv]   gradient of every chunk's end state
//   TP  [units][nch][2][64][64]  T = (I + A)^{-1}, then P
//   U, dR [B][T][H][dv]        per token, laid out like o
//   KB  [units][nch][Kb::floats]  the key block above
//   DPA [units][nch][2][64][64]   dP, then dA (masked)
//   XS  [units][nch][3][64][dk]   S dO, S dR, dS' U as [token][channel]
//   RS  [units][nch][dk]          row sums of S * dS'
struct Ws {
    float *Sc, *dSc, *TP, *U, *dR, *KB, *DPA, *XS, *RS;
};

// ---------------------------------------------------------------------------
// prep: A, P, T of one chunk.  The chunk is cut into four 16-token blocks.  For a
// key s in an earlier block than the row t, the decay 2^(G_t - G_s) is split at
// the first token r of t's block into 2^(G_t - G_r) 2^(G_r - G_s), both at most 1
// (s < r <= t), so those entries are products of scaled tiles on the tensor cores;
// the four 16 x 16 diagonal blocks take each pair's decay directly.
template <int DK>
struct PrepSmem {
    static constexpr int LB = 33, LE = 36;
    // per channel block: cg, cl, ck, ce, cq [64][LB]; Er, Qr [48][LE]; Kr [96][LE]
    static constexpr size_t blk = 5 * (size_t)kC * LB + (48 + 48 + 96) * (size_t)LE;
    // after the channel loop: A, P, T [64][LDT], over the same memory
    static constexpr size_t fin = 3 * (size_t)kC * LDT;
    static constexpr size_t floats = blk > fin ? blk : fin;
    static constexpr size_t bytes = floats * sizeof(float);
};

// Rows of Kr: block tau = 1, 2, 3 holds the keys s < 16 tau scaled to reference 16 tau.
__device__ __forceinline__ int kr_offset(int tau) { return tau == 1 ? 0 : (tau == 2 ? 16 : 48); }

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kThreads)
bwd_prep_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const float *__restrict__ alpha,
                const float *__restrict__ bgate, float *TP, float *KB, int T, int H) {
    using L = Kb<DK, DV>;
    constexpr int LB = PrepSmem<DK>::LB, LE = PrepSmem<DK>::LE;
    extern __shared__ float smem[];
    float *cg = smem, *cl = cg + kC * LB, *ck = cl + kC * LB, *ce = ck + kC * LB, *cq = ce + kC * LB;
    float *Er = cq + kC * LB, *Qr = Er + 48 * LE, *Kr = Qr + 48 * LE;
    float *sA = smem, *sP = sA + kC * LDT, *sT = sP + kC * LDT;     // after the channel loop
    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int warp = tid >> 5;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;
    float *kb = KB + ((size_t)unit * nch + c) * L::floats;

    // Off-diagonal blocks: 12 n8 column blocks per matrix (tau = 1: 2, tau = 2: 4, tau = 3: 6);
    // warps 0-3 build A from Er, warps 4-7 build P from Qr, three column blocks each.
    Wt<1, 1> off[3];
    int off_tau[3], off_nb[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int b = (warp & 3) * 3 + j;
        off_tau[j] = b < 2 ? 1 : (b < 6 ? 2 : 3);
        off_nb[j] = b - (off_tau[j] == 1 ? 0 : (off_tau[j] == 2 ? 2 : 6));
        off[j].zero();
    }
    // Diagonal blocks: pair p = tid + 256 j of 4 x 136 (s <= t inside one 16-token block).
    int pt[3], ps[3];
    float pa[3], pp[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int p = tid + j * kThreads;
        const int blk = p / 136, qd = p - blk * 136;
        int tt = (int)((sqrtf(8.f * qd + 1.f) - 1.f) * 0.5f);
        while ((tt + 1) * (tt + 2) / 2 <= qd) ++tt;
        while (tt * (tt + 1) / 2 > qd) --tt;
        pt[j] = p < 4 * 136 ? blk * 16 + tt : -1;
        ps[j] = p < 4 * 136 ? blk * 16 + qd - tt * (tt + 1) / 2 : -1;
        pa[j] = pp[j] = 0.f;
    }

    for (int ib = 0; ib < DK; ib += 32) {
        __syncthreads();
        {   // all loads first, then the transforms
            constexpr int E = kC * 32 / kThreads;
            float ra[E], rk[E], rq[E], rb[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int idx = tid + e * kThreads, t = idx >> 5, i = idx & 31;
                ra[e] = 1.f; rk[e] = rq[e] = rb[e] = 0.f;
                if (t < n) {
                    const size_t off2 = ((tok0 + t) * H + h) * DK + ib + i;
                    ra[e] = __ldg(alpha + off2);
                    rk[e] = Elem<TIn>::load(k + off2);
                    rq[e] = Elem<TIn>::load(q + off2);
                    rb[e] = __ldg(bgate + off2);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int idx = tid + e * kThreads, t = idx >> 5, i = idx & 31;
                cg[t * LB + i] = log2f(fmaxf(ra[e], kAlphaMin));
                ck[t * LB + i] = rk[e];
                cq[t * LB + i] = rq[e];
                ce[t * LB + i] = rb[e] * rk[e];
            }
        }
        __syncthreads();
        comp_cumsum<32>(cg, cl, LB);
        // Etil = e 2^g, Khat = k 2^(g_n - g), Qtil = q 2^g, 2^(g_n) for this channel block
        for (int idx = tid; idx < kC * 32; idx += kThreads) {
            const int t = idx >> 5, i = idx & 31;
            const float gh = cg[t * LB + i], gl = cl[t * LB + i];
            const float f = ex2(gh + gl);
            const float kh = ck[t * LB + i] * ex2(gdiff(cg[(kC - 1) * LB + i], cl[(kC - 1) * LB + i], gh, gl));
            kb[L::ET + t * L::LK + ib + i] = ce[t * LB + i] * f;
            kb[L::KH + t * L::LK + ib + i] = kh;
            kb[L::QT + t * L::LK + ib + i] = cq[t * LB + i] * f;
            if (t == kC - 1) kb[L::GNF + ib + i] = f;
        }
        // scaled tiles: Er, Qr rows t = 16..63 to reference r = 16 (t / 16); Kr as above
        for (int idx = tid; idx < 48 * 32; idx += kThreads) {
            const int t = 16 + (idx >> 5), i = idx & 31, r = t & ~15;
            const float f = ex2(gdiff(cg[t * LB + i], cl[t * LB + i], cg[r * LB + i], cl[r * LB + i]));
            Er[(t - 16) * LE + i] = ce[t * LB + i] * f;
            Qr[(t - 16) * LE + i] = cq[t * LB + i] * f;
        }
        for (int idx = tid; idx < 96 * 32; idx += kThreads) {
            const int row = idx >> 5, i = idx & 31;
            const int tau = row < 16 ? 1 : (row < 48 ? 2 : 3), s2 = row - kr_offset(tau), r = 16 * tau;
            Kr[row * LE + i] = ck[s2 * LB + i] * ex2(gdiff(cg[r * LB + i], cl[r * LB + i], cg[s2 * LB + i], cl[s2 * LB + i]));
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 3; ++j) {       // off-diagonal blocks on the tensor cores
            const float *Am = (warp < 4 ? Er : Qr) + (off_tau[j] - 1) * 16 * LE;
            off[j].run(Am, LE, 1, Kr, 1, LE, 32, 0, kr_offset(off_tau[j]) + off_nb[j] * 8);
        }
#pragma unroll
        for (int j = 0; j < 3; ++j) {       // diagonal blocks, pair by pair
            if (pt[j] < 0) continue;
            const int t = pt[j], s2 = ps[j];
            const float *gt = cg + t * LB, *gs = cg + s2 * LB, *lt = cl + t * LB, *ls = cl + s2 * LB,
                        *ks = ck + s2 * LB, *et = ce + t * LB, *qt = cq + t * LB;
            float aa = pa[j], qq = pp[j];
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const float kd = ks[i] * ex2(gdiff(gt[i], lt[i], gs[i], ls[i]));
                aa = fmaf(et[i], kd, aa);
                qq = fmaf(qt[i], kd, qq);
            }
            pa[j] = aa; pp[j] = qq;
        }
    }
    __syncthreads();                        // sA, sP, sT now take the channel tiles' memory
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
        const int t = idx >> 6, s2 = idx & 63;
        if (s2 >= t) {                      // above the diagonal (and A's diagonal): zero
            sA[t * LDT + s2] = 0.f;
            if (s2 > t) sP[t * LDT + s2] = 0.f;
        }
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int tau = off_tau[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 16 * tau + off[j].row(0, 0, i), s2 = off[j].col(off_nb[j] * 8, 0, i);
            (warp < 4 ? sA : sP)[t * LDT + s2] = off[j].c[0][0][i];
        }
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        if (pt[j] < 0) continue;
        if (ps[j] < pt[j]) sA[pt[j] * LDT + ps[j]] = pa[j];
        sP[pt[j] * LDT + ps[j]] = pp[j];
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
// prep2: the products with T and with dO that do not involve the carried state.
template <int DV>
struct Prep2Smem {
    static constexpr int LT = kC + 8, LDV = DV + 8, LB = 40;
    static constexpr size_t floats = 2 * (size_t)kC * LT + 3 * (size_t)kC * LDV + 3 * (size_t)kC * LB;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_prep2_kernel(const TIn *__restrict__ v, const float *__restrict__ wgate, const TIn *__restrict__ dO,
                 const float *TP, float *KB, int T, int H) {
    using L = Kb<DK, DV>;
    constexpr int LT = Prep2Smem<DV>::LT, LDV = Prep2Smem<DV>::LDV, LB = Prep2Smem<DV>::LB;
    constexpr int VN = DV / 32;             // n8 blocks per warp over DV / 4 columns
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5;
    float *Tm = smem, *Pm = Tm + kC * LT;
    float *sO = Pm + kC * LT, *sZ = sO + kC * LDV, *sW = sZ + kC * LDV;
    float *b1 = sW + kC * LDV, *b2 = b1 + kC * LB, *b3 = b2 + kC * LB;
    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;
    const size_t chunk = (size_t)unit * nch + c;
    float *kb = KB + chunk * L::floats;

    const float *tp = TP + chunk * 2 * kC * kC;
    copy_tile_async(Tm, LT, tp, kC, kC, kC);
    copy_tile_async(Pm, LT, tp + kC * kC, kC, kC, kC);
    cp_async_commit();
    for (int base = 0; base < kC * DV; base += 8 * kThreads) {     // eight loads in flight per thread
        float ro[8], rw[8], rv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads, t = idx / DV, j = idx % DV;
            ro[e] = rw[e] = rv[e] = 0.f;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DV + j;
                ro[e] = Elem<TIn>::load(dO + off);
                rw[e] = __ldg(wgate + off);
                rv[e] = Elem<TIn>::load(v + off);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads, t = idx / DV, j = idx % DV;
            sO[t * LDV + j] = ro[e];
            sZ[t * LDV + j] = rw[e] * rv[e];
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    const int vm0 = (warp >> 2) * 32, vn0 = (warp & 3) * (DV / 4);   // 64 x DV outputs: 32 x DV/4 per warp
    {   // W = P^T dO
        Wt<2, VN> w;
        w.zero();
        w.run(Pm, 1, LT, sO, LDV, 1, kC, vm0, vn0);
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < VN; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) sW[w.row(vm0, a, i) * LDV + w.col(vn0, b, i)] = w.c[a][b][i];
    }
    __syncthreads();
    {   // TPdO = T^T W, TZ = T Z
        Wt<2, VN> w1, w2;
        w1.zero();
        w2.zero();
        w1.run(Tm, 1, LT, sW, LDV, 1, kC, vm0, vn0);
        w2.run(Tm, LT, 1, sZ, LDV, 1, kC, vm0, vn0);
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < VN; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = w1.row(vm0, a, i), j = w1.col(vn0, b, i);
                    kb[L::TPDO + t * L::LV + j] = w1.c[a][b][i];
                    kb[L::TZ + t * L::LV + j] = w2.c[a][b][i];
                }
    }
    for (int ib = 0; ib < DK; ib += 32) {
        __syncthreads();
        copy_tile_async(b1, LB, kb + L::ET + ib, L::LK, kC, 32);
        copy_tile_async(b2, LB, kb + L::KH + ib, L::LK, kC, 32);
        copy_tile_async(b3, LB, kb + L::QT + ib, L::LK, kC, 32);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        {   // TEt = T Et, TKh = T^T Kh on this channel block (64 x 32: 16 x 16 per warp)
            const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;
            Wt<1, 2> w1, w2;
            w1.zero();
            w2.zero();
            w1.run(Tm, LT, 1, b1, LB, 1, kC, m0, n0);
            w2.run(Tm, 1, LT, b2, LB, 1, kC, m0, n0);
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = w1.row(m0, 0, i), ic = w1.col(n0, b, i);
                    kb[L::TET + t * L::LK + ib + ic] = w1.c[0][b][i];
                    kb[L::TKH + t * L::LK + ib + ic] = w2.c[0][b][i];
                }
        }
        {   // QdO rows of this channel block = Qt^T dO (32 x DV: 16 x DV/4 per warp)
            const int m0 = (warp >> 2) * 16, n0 = (warp & 3) * (DV / 4);
            Wt<1, VN> w3;
            w3.zero();
            w3.run(b3, 1, LB, sO, LDV, 1, kC, m0, n0);
#pragma unroll
            for (int b = 0; b < VN; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    kb[L::QDO + (size_t)(ib + w3.row(m0, 0, i)) * L::LV + w3.col(n0, b, i)] = w3.c[0][b][i];
        }
    }
}

// ---------------------------------------------------------------------------
// state: the two serial sweeps for one (sequence, head, column slice).
template <int DK>
struct StateSmem {
    // X1 is read row-major, X2 transposed: row strides 4 and 8 mod 32 floats
    static constexpr int LK = DK + 4, LK2 = DK + 8, LZ = kCS + 8;
    // one operand buffer: X1 [64][LK], X2 [64][LK2], Zs [64][LZ], Qs [DK][LZ], gnf [DK]
    static constexpr size_t buf = (size_t)kC * LK + (size_t)kC * LK2 + (size_t)kC * LZ + (size_t)DK * LZ + DK;
    static constexpr size_t floats = 2 * buf + (size_t)DK * LZ + (size_t)kC * LZ;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_state_kernel(const float *S0, const float *dST, float *dS0, Ws ws, int T, int H) {
    using L = Kb<DK, DV>;
    using SM = StateSmem<DK>;
    constexpr int LK = SM::LK, LK2 = SM::LK2, LZ = SM::LZ;
    constexpr int SN = DK == 128 ? 4 : 2;   // DK x 32 outputs: 16 x (8 SN) per warp
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5;
    const int um0 = (warp >> 1) * 16, un0 = (warp & 1) * 16;                          // 64 x 32 outputs
    const int sm0 = DK == 128 ? warp * 16 : (warp >> 1) * 16, sn0 = DK == 128 ? 0 : (warp & 1) * 16;
    float *St = smem + 2 * SM::buf, *Us = St + DK * LZ;

    const int unit = blockIdx.x, seq = unit / H, h = unit % H;
    const int col0 = blockIdx.y * kCS, tid = threadIdx.x;
    const size_t tokb = (size_t)seq * T;
    const int nch = (T + kC - 1) / kC, steps = 2 * nch;
    const size_t soff = (size_t)unit * DK * DV;

    // step k < nch: forward over chunk k; step k >= nch: backward over chunk 2 nch - 1 - k
    auto issue = [&](int kstep) {
        float *b = smem + (kstep & 1) * SM::buf;
        float *X1 = b, *X2 = X1 + kC * LK, *Zs = X2 + kC * LK2, *Qs = Zs + kC * LZ, *gnf = Qs + DK * LZ;
        const bool fwd = kstep < nch;
        const int c = fwd ? kstep : steps - 1 - kstep;
        const float *kb = ws.KB + ((size_t)unit * nch + c) * L::floats;
        copy_tile_async(X1, LK, kb + (fwd ? L::TET : L::TKH), L::LK, kC, DK);
        copy_tile_async(X2, LK2, kb + (fwd ? L::KH : L::ET), L::LK, kC, DK);
        copy_tile_async(Zs, LZ, kb + (fwd ? L::TZ : L::TPDO) + col0, L::LV, kC, kCS);
        if (!fwd) copy_tile_async(Qs, LZ, kb + L::QDO + col0, L::LV, DK, kCS);
        copy_tile_async(gnf, DK, kb + L::GNF, DK, 1, DK);
        cp_async_commit();
    };

    for (int idx = tid; idx < DK * kCS; idx += kThreads) {
        const int i = idx / kCS, j = idx % kCS;
        St[i * LZ + j] = S0 ? S0[soff + (size_t)i * DV + col0 + j] : 0.f;
    }
    issue(0);
    for (int kstep = 0; kstep < steps; ++kstep) {
        if (kstep + 1 < steps) {
            issue(kstep + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        const bool fwd = kstep < nch;
        const int c = fwd ? kstep : steps - 1 - kstep;
        const int n = min(kC, T - c * kC);
        const size_t chunk = (size_t)unit * nch + c;
        if (kstep == nch) {             // the backward sweep starts from dST
            for (int idx = tid; idx < DK * kCS; idx += kThreads) {
                const int i = idx / kCS, j = idx % kCS;
                St[i * LZ + j] = dST ? dST[soff + (size_t)i * DV + col0 + j] : 0.f;
            }
        }
        __syncthreads();
        const float *b = smem + (kstep & 1) * SM::buf;
        const float *X1 = b, *X2 = X1 + kC * LK, *Zs = X2 + kC * LK2, *Qs = Zs + kC * LZ, *gnf = Qs + DK * LZ;
        float *save = (fwd ? ws.Sc : ws.dSc) + chunk * DK * DV + col0;
        for (int idx = tid; idx < DK * kCS; idx += kThreads) {
            const int i = idx / kCS, j = idx % kCS;
            save[(size_t)i * DV + j] = St[i * LZ + j];
        }
        {   // forward: U = TZ - TEt S;  backward: dR = TPdO + TKh dS
            Wt<1, 2> w;
            w.zero();
            w.run(X1, LK, 1, St, LZ, 1, DK, um0, un0);
            float *out = fwd ? ws.U : ws.dR;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = w.row(um0, 0, i), j = w.col(un0, b, i);
                    const float u = fwd ? Zs[t * LZ + j] - w.c[0][b][i] : Zs[t * LZ + j] + w.c[0][b][i];
                    Us[t * LZ + j] = u;
                    if (t < n) out[((tokb + c * kC + t) * H + h) * DV + col0 + j] = u;
                }
        }
        __syncthreads();
        {   // forward: S = gnf S + Kh^T U;  backward: dS = gnf dS + QdO - Et^T dR
            Wt<1, SN> w;
            w.zero();
            w.run(X2, 1, LK2, Us, LZ, 1, kC, sm0, sn0);
#pragma unroll
            for (int b = 0; b < SN; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = w.row(sm0, 0, i), j = w.col(sn0, b, i);
                    const float carried = gnf[r] * St[r * LZ + j];
                    St[r * LZ + j] = fwd ? carried + w.c[0][b][i] : carried + Qs[r * LZ + j] - w.c[0][b][i];
                }
        }
        __syncthreads();                // buffer kstep & 1 is refilled by the next issue()
    }
    if (dS0) {
        for (int idx = tid; idx < DK * kCS; idx += kThreads) {
            const int i = idx / kCS, j = idx % kCS;
            dS0[soff + (size_t)i * DV + col0 + j] = St[i * LZ + j];
        }
    }
}

// ---------------------------------------------------------------------------
// grad_a: the contractions over the value columns of one chunk.
template <int DV>
struct GradASmem {
    static constexpr int LDV = DV + 4;
    static constexpr size_t floats = 3 * (size_t)kC * LDV + 2 * 32 * (size_t)LDV;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_grada_kernel(const TIn *__restrict__ v, const float *__restrict__ wgate, const TIn *__restrict__ dO, Ws ws,
                 TIn *dvv, float *dw, int T, int H) {
    constexpr int LDV = GradASmem<DV>::LDV;
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5;
    float *sO = smem, *sU = sO + kC * LDV, *sR = sU + kC * LDV;
    float *sS = sR + kC * LDV, *sD = sS + 32 * LDV;
    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;
    const size_t chunk = (size_t)unit * nch + c;

    // U, dR of the chunk's valid rows (asynchronously), dO through registers; padding rows zero
    for (int idx = tid; idx < kC * (DV / 4); idx += kThreads) {
        const int t = idx / (DV / 4), j4 = (idx % (DV / 4)) * 4;
        if (t < n) {
            const size_t off = ((tok0 + t) * H + h) * DV + j4;
            cp_async16(sU + t * LDV + j4, ws.U + off);
            cp_async16(sR + t * LDV + j4, ws.dR + off);
        } else {
            *reinterpret_cast<float4 *>(sU + t * LDV + j4) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(sR + t * LDV + j4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    cp_async_commit();
    for (int base = 0; base < kC * DV; base += 8 * kThreads) {
        float ro[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads, t = idx / DV, j = idx % DV;
            ro[e] = t < n ? Elem<TIn>::load(dO + ((tok0 + t) * H + h) * DV + j) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads;
            sO[(idx / DV) * LDV + idx % DV] = ro[e];
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    for (int base = 0; base < kC * DV; base += 8 * kThreads) {   // dw = dR v, dv = dR w
        float rv[8], rw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads, t = idx / DV, j = idx % DV;
            rv[e] = rw[e] = 0.f;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DV + j;
                rv[e] = Elem<TIn>::load(v + off);
                rw[e] = __ldg(wgate + off);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = base + tid + e * kThreads, t = idx / DV, j = idx % DV;
            if (t < n) {
                const size_t off = ((tok0 + t) * H + h) * DV + j;
                const float r = sR[t * LDV + j];
                dw[off] = r * rv[e];
                Elem<TIn>::store(dvv + off, r * rw[e]);
            }
        }
    }
    {   // dP = dO U^T (s <= t), dA = -dR U^T (s < t); 64 x 64, 32 x 16 per warp
        const int m0 = (warp >> 2) * 32, n0 = (warp & 3) * 16;
        Wt<2, 2> wp, wa;
        wp.zero();
        wa.zero();
        wp.run(sO, LDV, 1, sU, 1, LDV, DV, m0, n0);
        wa.run(sR, LDV, 1, sU, 1, LDV, DV, m0, n0);
        float *dpa = ws.DPA + chunk * 2 * kC * kC;
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = wp.row(m0, a, i), s2 = wp.col(n0, b, i);
                    dpa[t * kC + s2] = (s2 <= t) ? wp.c[a][b][i] : 0.f;
                    dpa[kC * kC + t * kC + s2] = (s2 < t) ? -wa.c[a][b][i] : 0.f;
                }
    }
    float *xs = ws.XS + chunk * 3 * kC * DK;
    for (int ib = 0; ib < DK; ib += 32) {
        copy_tile_async(sS, LDV, ws.Sc + chunk * DK * DV + (size_t)ib * DV, DV, 32, DV);
        copy_tile_async(sD, LDV, ws.dSc + chunk * DK * DV + (size_t)ib * DV, DV, 32, DV);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        {   // row sums of S * dS': eight lanes per row
            const int i = tid >> 3, part = tid & 7;
            float acc = 0.f;
            for (int j = part; j < DV; j += 8) acc = fmaf(sS[i * LDV + j], sD[i * LDV + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            if (part == 0) ws.RS[chunk * DK + ib + i] = acc;
        }
        {   // X1 = S dO, X2 = S dR, Y = dS' U, as [token][channel]; 64 x 32, 16 x 16 per warp
            const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;
            Wt<1, 2> x1, x2, y;
            x1.zero();
            x2.zero();
            y.zero();
            x1.run(sO, LDV, 1, sS, 1, LDV, DV, m0, n0);
            x2.run(sR, LDV, 1, sS, 1, LDV, DV, m0, n0);
            y.run(sU, LDV, 1, sD, 1, LDV, DV, m0, n0);
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = x1.row(m0, 0, i), ic = ib + x1.col(n0, b, i);
                    xs[t * DK + ic] = x1.c[0][b][i];
                    xs[kC * DK + t * DK + ic] = x2.c[0][b][i];
                    xs[2 * kC * DK + t * DK + ic] = y.c[0][b][i];
                }
        }
        __syncthreads();                    // sS, sD are refilled by the next block
    }
}

// ---------------------------------------------------------------------------
// grad_b: the per-token gradients of one chunk, key channels in blocks of 32.
// The decay-weighted sums over pairs of tokens use the 16-token block split of
// the prep kernel: pairs in different blocks go through scaled tiles on the
// tensor cores, pairs inside one block are summed directly.
//   rows:    sum_{s < r} dP[t,s] k_s 2^(G_t - G_s) = 2^(G_t - G_r) (dP Kr)[t]      (r: first token of t's block)
//   columns: sum_{t in tau} (dA[t,s] e_t + dP[t,s] q_t) 2^(G_t - G_s)
//          = 2^(G_r - G_s) (dA^T Er + dP^T Qr)[s]                                  (r: first token of block tau > s's)
struct GradBSmem {
    static constexpr int LP = kC + 4, LB = 36, LE = 40;
    // dP, dA [64][LP]; per block: cg, cl, ck, cq, ce, X1, X2, Y, OQ, OE, OK [64][LB];
    // Er, Qr [48][LE]; Kr, F [96][LE]; rs [32]
    static constexpr size_t floats = 2 * (size_t)kC * LP + 11 * (size_t)kC * LB + (48 * 2 + 96 * 2) * (size_t)LE + 32;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kThreadsB, 1)
bwd_gradb_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const float *__restrict__ alpha,
                 const float *__restrict__ bgate, Ws ws, TIn *dq, TIn *dk, float *dalpha, float *db, int T, int H) {
    constexpr int LP = GradBSmem::LP, LB = GradBSmem::LB, LE = GradBSmem::LE;
    extern __shared__ __align__(16) float smem[];
    float *dP = smem, *dA = dP + kC * LP;
    float *cg = dA + kC * LP, *cl = cg + kC * LB, *ck = cl + kC * LB, *cq = ck + kC * LB, *ce = cq + kC * LB;
    float *X1 = ce + kC * LB, *X2 = X1 + kC * LB, *Y = X2 + kC * LB;
    float *OQ = Y + kC * LB, *OE = OQ + kC * LB, *OK = OE + kC * LB;
    float *Er = OK + kC * LB, *Qr = Er + 48 * LE, *Kr = Qr + 48 * LE, *F = Kr + 96 * LE;
    float *rs = F + 96 * LE;
    const int c = blockIdx.x, unit = blockIdx.y, seq = unit / H, h = unit % H, tid = threadIdx.x;
    const int warp = tid >> 5;
    const int nch = gridDim.x, c0 = c * kC, n = min(kC, T - c0);
    const size_t tok0 = (size_t)seq * T + c0;
    const size_t chunk = (size_t)unit * nch + c;

    copy_tile_async<kThreadsB>(dP, LP, ws.DPA + chunk * 2 * kC * kC, kC, kC, kC);
    copy_tile_async<kThreadsB>(dA, LP, ws.DPA + chunk * 2 * kC * kC + kC * kC, kC, kC, kC);
    cp_async_commit();
    const float *xs = ws.XS + chunk * 3 * kC * DK;
    for (int ib = 0; ib < DK; ib += 32) {
        __syncthreads();
        copy_tile_async<kThreadsB>(X1, LB, xs + ib, DK, kC, 32);
        copy_tile_async<kThreadsB>(X2, LB, xs + kC * DK + ib, DK, kC, 32);
        copy_tile_async<kThreadsB>(Y, LB, xs + 2 * kC * DK + ib, DK, kC, 32);
        copy_tile_async<kThreadsB>(rs, 32, ws.RS + chunk * DK + ib, 32, 1, 32);
        cp_async_commit();
        {   // this block's key side: all loads first, then the transforms
            constexpr int E = kC * 32 / kThreadsB;
            float ra[E], rk[E], rq[E], rb[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int idx = tid + e * kThreadsB, t = idx >> 5, i = idx & 31;
                ra[e] = 1.f; rk[e] = rq[e] = rb[e] = 0.f;
                if (t < n) {
                    const size_t off = ((tok0 + t) * H + h) * DK + ib + i;
                    ra[e] = __ldg(alpha + off);
                    rk[e] = Elem<TIn>::load(k + off);
                    rq[e] = Elem<TIn>::load(q + off);
                    rb[e] = __ldg(bgate + off);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int idx = tid + e * kThreadsB, t = idx >> 5, i = idx & 31;
                cg[t * LB + i] = log2f(fmaxf(ra[e], kAlphaMin));
                ck[t * LB + i] = rk[e];
                cq[t * LB + i] = rq[e];
                ce[t * LB + i] = rb[e] * rk[e];
            }
        }
        __syncthreads();
        comp_cumsum<32, kThreadsB>(cg, cl, LB);
        // scaled tiles (both factors of every split decay are at most 1)
        for (int idx = tid; idx < 48 * 32; idx += kThreadsB) {
            const int t = 16 + (idx >> 5), i = idx & 31, r = t & ~15;
            const float f = ex2(gdiff(cg[t * LB + i], cl[t * LB + i], cg[r * LB + i], cl[r * LB + i]));
            Er[(t - 16) * LE + i] = ce[t * LB + i] * f;
            Qr[(t - 16) * LE + i] = cq[t * LB + i] * f;
        }
        for (int idx = tid; idx < 96 * 32; idx += kThreadsB) {
            const int row = idx >> 5, i = idx & 31;
            const int tau = row < 16 ? 1 : (row < 48 ? 2 : 3), s2 = row - kr_offset(tau), r = 16 * tau;
            const float f = ex2(gdiff(cg[r * LB + i], cl[r * LB + i], cg[s2 * LB + i], cl[s2 * LB + i]));
            F[row * LE + i] = f;
            Kr[row * LE + i] = ck[s2 * LB + i] * f;
        }
        for (int idx = tid; idx < 16 * 32; idx += kThreadsB) {     // no earlier block for rows 0-15,
            const int t = idx >> 5, i = idx & 31;                 // no later block for keys 48-63
            OQ[t * LB + i] = 0.f;
            OE[t * LB + i] = 0.f;
            OK[(48 + t) * LB + i] = 0.f;
        }
        cp_async_wait<0>();
        __syncthreads();
        if (warp < 6) {
            {   // rows of block tau = 1 + warp / 2 against all earlier keys: warp & 1 ? dA : dP
                const int tau = 1 + (warp >> 1);
                Wt<1, 4> w;
                w.zero();
                w.run((warp & 1 ? dA : dP) + 16 * tau * LP, LP, 1, Kr + kr_offset(tau) * LE, LE, 1, 16 * tau, 0, 0);
                float *out = warp & 1 ? OE : OQ;
#pragma unroll
                for (int b = 0; b < 4; ++b)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int t = 16 * tau + w.row(0, 0, i), ic = w.col(0, b, i), r = 16 * tau;
                        out[t * LB + ic] = w.c[0][b][i] *
                            ex2(gdiff(cg[t * LB + ic], cl[t * LB + ic], cg[r * LB + ic], cl[r * LB + ic]));
                    }
            }
        }
        if (warp >= 6 && warp < 12) {
            const int cw = warp - 6;
            {   // keys of block sigma = cw / 2, channels 16 (cw & 1) ..: every later block tau
                const int sigma = cw >> 1, n0 = 16 * (cw & 1);
                float acc[2][4];
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;
                for (int tau = sigma + 1; tau < 4; ++tau) {
                    Wt<1, 2> w;
                    w.zero();
                    w.run(dA + 16 * tau * LP, 1, LP, Er + 16 * (tau - 1) * LE, LE, 1, 16, 16 * sigma, n0);
                    w.run(dP + 16 * tau * LP, 1, LP, Qr + 16 * (tau - 1) * LE, LE, 1, 16, 16 * sigma, n0);
#pragma unroll
                    for (int b = 0; b < 2; ++b)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int s2 = w.row(16 * sigma, 0, i), ic = w.col(n0, b, i);
                            acc[b][i] = fmaf(F[(kr_offset(tau) + s2) * LE + ic], w.c[0][b][i], acc[b][i]);
                        }
                }
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int s2 = 16 * sigma + ((threadIdx.x & 31) >> 2) + (i >> 1) * 8;
                        const int ic = n0 + b * 8 + 2 * (threadIdx.x & 3) + (i & 1);
                        OK[s2 * LB + ic] = acc[b][i];
                    }
            }
        }
        __syncthreads();
        float dlg[kC * 32 / kThreadsB];
#pragma unroll
        for (int e = 0; e < kC * 32 / kThreadsB; ++e) {
            const int idx = tid + e * kThreadsB, t = idx >> 5, i = idx & 31;
            const int r = t & ~15;
            const float gt = cg[t * LB + i], lt = cl[t * LB + i];
            const float gnh = cg[(kC - 1) * LB + i], gnl = cl[(kC - 1) * LB + i];
            float sq = OQ[t * LB + i], se = OE[t * LB + i], sk = OK[t * LB + i];
            for (int s2 = r; s2 <= t; ++s2) {       // dq, de: earlier keys of t's own block
                const float f = ck[s2 * LB + i] * ex2(gdiff(gt, lt, cg[s2 * LB + i], cl[s2 * LB + i]));
                sq = fmaf(dP[t * LP + s2], f, sq);
                se = fmaf(dA[t * LP + s2], f, se);
            }
            for (int u = t; u < r + 16; ++u) {      // dk: later tokens of t's own block
                const float f = ex2(gdiff(cg[u * LB + i], cl[u * LB + i], gt, lt));
                sk = fmaf(fmaf(dA[u * LP + t], ce[u * LB + i], dP[u * LP + t] * cq[u * LB + i]), f, sk);
            }
            const float ft = ex2(gt + lt);
            const float dqv = fmaf(ft, X1[t * LB + i], sq);
            const float dev = fmaf(-ft, X2[t * LB + i], se);
            const float kkey = fmaf(ex2(gdiff(gnh, gnl, gt, lt)), Y[t * LB + i], sk);
            const float kk = ck[t * LB + i];
            float l = dev * ce[t * LB + i] + dqv * cq[t * LB + i] - kkey * kk;
            if (t == n - 1) {               // through g_n: diag(2^g_n) S and every Khat_s
                float kh = 0.f;
                for (int s2 = 0; s2 < n; ++s2)
                    kh = fmaf(ck[s2 * LB + i] * ex2(gdiff(gnh, gnl, cg[s2 * LB + i], cl[s2 * LB + i])),
                              Y[s2 * LB + i], kh);
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
        for (int e = 0; e < kC * 32 / kThreadsB; ++e) {
            const int idx = tid + e * kThreadsB;
            X2[(idx >> 5) * LB + (idx & 31)] = dlg[e];
        }
        __syncthreads();
        {   // dalpha = reverse cumulative sum of dlog gamma / alpha: (channel, 4-token segment) per thread
            constexpr int SEG = kC * 32 / kThreadsB, NSEG = kC / SEG;
            const int i = tid & 31, seg = tid >> 5;
            float ra[SEG];
#pragma unroll
            for (int u = 0; u < SEG; ++u) {
                const int t = seg * SEG + u;
                ra[u] = t < n ? __ldg(alpha + ((tok0 + t) * H + h) * DK + ib + i) : 1.f;
            }
            float tot = 0.f;
#pragma unroll
            for (int u = 0; u < SEG; ++u) tot += X2[(seg * SEG + u) * LB + i];
            X1[seg * LB + i] = tot;             // X1 is free: segment totals
            __syncthreads();
            float run = 0.f;
            for (int s2 = seg + 1; s2 < NSEG; ++s2) run += X1[s2 * LB + i];
#pragma unroll
            for (int u = SEG - 1; u >= 0; --u) {
                const int t = seg * SEG + u;
                run += X2[t * LB + i];
                if (t < n) dalpha[((tok0 + t) * H + h) * DK + ib + i] = run / fmaxf(ra[u], kAlphaMin);
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
    auto kp = bwd_prep_kernel<TIn, DK, DV>;
    auto kp2 = bwd_prep2_kernel<TIn, DK, DV>;
    auto ks = bwd_state_kernel<DK, DV>;
    auto kga = bwd_grada_kernel<TIn, DK, DV>;
    auto kgb = bwd_gradb_kernel<TIn, DK>;
    cudaError_t err;
    if ((err = set_smem(kp, PrepSmem<DK>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(kp2, Prep2Smem<DV>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(ks, StateSmem<DK>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(kga, GradASmem<DV>::bytes)) != cudaSuccess) return err;
    if ((err = set_smem(kgb, GradBSmem::bytes)) != cudaSuccess) return err;
    const dim3 grid_c((unsigned)nch, (unsigned)units);
    kp<<<grid_c, kThreads, PrepSmem<DK>::bytes, stream>>>(q, k, alpha, b, ws.TP, ws.KB, T, H);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    kp2<<<grid_c, kThreads, Prep2Smem<DV>::bytes, stream>>>(v, w, dO, ws.TP, ws.KB, T, H);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    ks<<<dim3((unsigned)units, (unsigned)(DV / kCS)), kThreads, StateSmem<DK>::bytes, stream>>>(S0, dST, dS0, ws, T,
                                                                                                 H);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    kga<<<grid_c, kThreads, GradASmem<DV>::bytes, stream>>>(v, w, dO, ws, static_cast<TIn *>(dv), dw, T, H);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    kgb<<<grid_c, kThreadsB, GradBSmem::bytes, stream>>>(q, k, alpha, b, ws, static_cast<TIn *>(dq),
                                                         static_cast<TIn *>(dk), dalpha, db, T, H);
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

static size_t kb_floats(int dk, int dv) {
    if (dk == 128) return dv == 128 ? Kb<128, 128>::floats : Kb<128, 64>::floats;
    return dv == 128 ? Kb<64, 128>::floats : Kb<64, 64>::floats;
}

size_t chunk_bwd_workspace_floats(int B, int T, int H, int dk, int dv) {
    const size_t nch = (size_t)(T + kC - 1) / kC, units = (size_t)B * H;
    return 2 * units * nch * dk * dv + units * nch * 2 * kC * kC + 2 * (size_t)B * T * H * dv +
           units * nch * kb_floats(dk, dv) + units * nch * (2 * kC * kC + 3 * kC * dk + dk);
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
    ws.KB = ws.dR + (size_t)B * T * H * d_v;
    ws.DPA = ws.KB + units * nch * kb_floats(d_k, d_v);
    ws.XS = ws.DPA + units * nch * 2 * kC * kC;
    ws.RS = ws.XS + units * nch * 3 * kC * d_k;
    if (dt == GDN2_BF16)
        return launch_bwd_dt<__nv_bfloat16>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, ws, B,
                                            T, H, d_k, d_v, stream);
    return launch_bwd_dt<float>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, ws, B, T, H, d_k,
                                d_v, stream);
}

}  // namespace gdn2
