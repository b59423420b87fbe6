// Chunkwise prefill of the Gated DeltaNet-2 recurrence on the sm_100a tensor
// cores (tcgen05, TF32 operands, FP32 accumulation in Tensor Memory).
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Token processing and parallel training":
// 64-token chunks, the cumulative channel-wise decay absorbed into asymmetric
// erase factors, triangular solves and dense products inside each chunk, FP32
// decay and state/solve precision.  Per chunk of n tokens from state S:
//
//   gamma_t = prod_{j<=t} alpha_j,  rho_t = 1/gamma_t          (per key channel, FP32)
//   Etil = b*k*gamma,  Qtil = q*gamma,  Ktil = k*rho,  Z = w*v   (gate prep)
//   [A | Etil S] and [P | Qtil S] = [Etil; Qtil] [Ktil; S^T]^T  (one tensor-core product)
//   A <- strict_tril(A),  P <- tril(P),  T = (I + A)^{-1}        (FP32 blocked solve)
//   R = Z - Etil S                                               (FP32 epilogue)
//   U = T R                                                      (tensor core)
//   O = Qtil S + P U                                             (tensor core, accumulated)
//   S <- diag(gamma_n) (S + Ktil^T U)                            (tensor core + FP32 epilogue)
//
// The state path (R, U and Ktil in the state update) is computed with split
// TF32 operands: x = x_hi + x_lo, both TF32, and
//   T R = T R_hi + T R_lo,   Ktil^T U = Ktil_hi^T U_hi + Ktil_hi^T U_lo + Ktil_lo^T U_hi,
// which carries about 21 bits of each operand.  With plain TF32 there the
// carried state drifts by ~0.7% of its RMS over 16K tokens; split, ~0.03%.
//
// U holds the per-token corrections z_t - r_t of the token recurrence, so this
// is the same arithmetic as the token loop, re-associated.
//
// Precision: tensor-core operands are rounded to TF32 (10-bit mantissa);
// accumulation, decay, solve, R and the carried state are FP32.  BF16 operands
// lose too much here: the read r = Sbar^T e nearly cancels the write z in the
// delta rule, and products of decay-scaled factors carry that error into o and
// S.  The key factor Ktil = k / gamma grows within a chunk as
// exp(-sum ln alpha); it must stay below ~1e34 (sum of -ln alpha over one chunk
// <= 78 per key channel), as documented in gdn2.h.
//
// Layout: one CTA per (batch, head, 64-column half of d_v); 256 threads (8
// warps) run the phases of a chunk in turn; thread 0 issues TMA loads and MMAs.
// Every shared-memory operand is K-major with the 128-byte swizzle.  Operands
// needed transposed (Ktil^T, [T; P]) are written to Tensor Memory and read from
// there as the A operand.  alpha, b and w are TMA-loaded straight into the
// tiles they become and transformed in place; the next chunk's loads are
// issued as soon as each tile is consumed.
#include <cudaTypedefs.h>
#include <stdio.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn2 {

__device__ unsigned int g_device_error = 0;  // nonzero: a bounded wait in a kernel gave up

namespace tc {

using namespace sm100;

constexpr int kC = 64;            // chunk length (tokens)
constexpr int kDK = 128;          // key channels
constexpr int kDVS = 64;          // value columns per CTA
constexpr int kThreads = 256;
constexpr long long kWaitLimit = 4000000000ll;   // ~2 s of SM cycles per wait

// Shared-memory map (bytes from a 1024-aligned base).  Tiles hold FP32/TF32,
// 32 elements per 128-byte swizzled row, K-major:
//   X1  rows 0-63 Etil[t][i], rows 64-127 Qtil[t][i]     4 atoms x 16 KB (i = key channel)
//   KS  rows 0-63 Ktil[s][i], rows 64-127 S[i][j] as [j][i]   4 atoms x 16 KB
//   RU  R_hi, later U_hi, as [j][t]                       2 atoms x 8 KB (t = token)
//   RL  R_lo, later U_lo, as [j][t]                       2 atoms x 8 KB
//   ZW  w, then Z = w*v, as [t][j] (FP32, epilogue only)   2 atoms x 8 KB
// and unswizzled BF16 staging of q, k (64 x 128) and v (64 x 64).
constexpr uint32_t OFF_X1 = 0;
constexpr uint32_t OFF_KS = OFF_X1 + 65536;
constexpr uint32_t OFF_RU = OFF_KS + 65536;
constexpr uint32_t OFF_RL = OFF_RU + 16384;
constexpr uint32_t OFF_ZW = OFF_RL + 16384;
constexpr uint32_t OFF_RQ = OFF_ZW + 16384;
constexpr uint32_t OFF_RK = OFF_RQ + 16384;
constexpr uint32_t OFF_RV = OFF_RK + 16384;
constexpr uint32_t OFF_GN = OFF_RV + 8192;      // float[128]   decay over the chunk
constexpr uint32_t OFF_PART = OFF_GN + 512;     // float[2][128] half-chunk decay products
constexpr uint32_t OFF_BAR = OFF_PART + 1024;   // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 64;     // tmem base, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack
// Solve scratch inside the q/k/v staging (free between prep and the next load).
constexpr int LDA = 65, LDX = 33;
constexpr uint32_t OFF_AS = OFF_RQ;                     // float[64][65] A, strictly lower
constexpr uint32_t OFF_TS = OFF_AS + 16896;             // float[64][65] T
constexpr uint32_t OFF_XS = OFF_TS + 16896;             // float[32][33] block products
static_assert(OFF_XS + 32 * LDX * 4 <= OFF_GN, "solve scratch overflows the staging area");

// Tensor Memory columns (512 allocated).
constexpr uint32_t TM_G = 0;      // [Etil;Qtil] Ktil^T : lanes 0-63 A, lanes 64-127 P   (64 cols)
constexpr uint32_t TM_X = 64;     // [Etil;Qtil] S, then + [T;P] U : lanes 64-127 -> O    (64 cols)
constexpr uint32_t TM_U = 128;    // [T;P] R : lanes 0-63 U                               (64 cols)
constexpr uint32_t TM_D = 192;    // Ktil^T U                                             (64 cols)
constexpr uint32_t TM_KT = 256;   // A operand Ktil^T: lane i, column s                   (64 cols)
constexpr uint32_t TM_TP = 320;   // A operand [T;P]: lane t (P at 64+t), column s        (64 cols)
constexpr uint32_t TM_KL = 384;   // A operand Ktil_lo^T (low TF32 part of Ktil^T)        (64 cols)
constexpr uint32_t TM_COLS = 512;

enum { BAR_QKV = 0, BAR_A, BAR_B, BAR_W, BAR_MMA, NBARS };

constexpr uint32_t TX_QKV = 16384 + 16384 + 8192;
constexpr uint32_t TX_A = 4 * 8192;
constexpr uint32_t TX_B = 4 * 8192;
constexpr uint32_t TX_W = 2 * 8192;

// Element byte offsets inside the tiles.
__device__ __forceinline__ uint32_t x_off(uint32_t r, uint32_t i) { return (i >> 5) * 16384u + swz128(r, (i & 31u) * 4u); }
__device__ __forceinline__ uint32_t ru_off(uint32_t j, uint32_t t) { return (t >> 5) * 8192u + swz128(j, (t & 31u) * 4u); }
__device__ __forceinline__ uint32_t zw_off(uint32_t t, uint32_t j) { return (j >> 5) * 8192u + swz128(t, (j & 31u) * 4u); }

struct Maps {
    CUtensorMap q, k, v, alpha, b, w;
};

struct Ctx {
    uint8_t *sm;          // 1024-aligned shared base (generic pointer)
    uint32_t sa;          // same, shared-window address
    uint32_t bar[NBARS];
};

__device__ __forceinline__ float *fptr(const Ctx &c, uint32_t off) { return reinterpret_cast<float *>(c.sm + off); }
__device__ __forceinline__ float &at(const Ctx &c, uint32_t off) { return *reinterpret_cast<float *>(c.sm + off); }

// TMA loads of one chunk's inputs (thread 0 only).
__device__ __forceinline__ void load_qkv(const Ctx &c, const Maps &m, int h, int t0, int bidx, int col0) {
    mbar_expect_tx(c.bar[BAR_QKV], TX_QKV);
    tma_load_4d(c.sa + OFF_RQ, &m.q, 0, h, t0, bidx, c.bar[BAR_QKV]);
    tma_load_4d(c.sa + OFF_RK, &m.k, 0, h, t0, bidx, c.bar[BAR_QKV]);
    tma_load_4d(c.sa + OFF_RV, &m.v, col0, h, t0, bidx, c.bar[BAR_QKV]);
}
__device__ __forceinline__ void load_alpha(const Ctx &c, const Maps &m, int h, int t0, int bidx) {
    mbar_expect_tx(c.bar[BAR_A], TX_A);   // rows 0-63 of each KS atom
    for (int a = 0; a < 4; ++a) tma_load_4d(c.sa + OFF_KS + a * 16384, &m.alpha, 32 * a, h, t0, bidx, c.bar[BAR_A]);
}
__device__ __forceinline__ void load_b(const Ctx &c, const Maps &m, int h, int t0, int bidx) {
    mbar_expect_tx(c.bar[BAR_B], TX_B);   // rows 0-63 of each X1 atom
    for (int a = 0; a < 4; ++a) tma_load_4d(c.sa + OFF_X1 + a * 16384, &m.b, 32 * a, h, t0, bidx, c.bar[BAR_B]);
}
__device__ __forceinline__ void load_w(const Ctx &c, const Maps &m, int h, int t0, int bidx, int col0) {
    mbar_expect_tx(c.bar[BAR_W], TX_W);
    for (int a = 0; a < 2; ++a) tma_load_4d(c.sa + OFF_ZW + a * 8192, &m.w, col0 + 32 * a, h, t0, bidx, c.bar[BAR_W]);
}

__device__ __forceinline__ float ldbf(const uint8_t *p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p)); }

// ---------------------------------------------------------------------------
// Gate prep.  Thread (lane quarter qd, half th, lane l) owns key channel
// i = 32 qd + l for tokens [32 th, 32 th + 32).  Cumulative decay is a running
// FP32 product (exp of the cumulative log-decay up to rounding).  Padding tokens
// (t >= n) have zero q, k, b, w, v from the TMA bounds fill and alpha forced to 1.
__device__ __forceinline__ void prep(const Ctx &c, uint32_t tmem, int tid, int qd, int th, int lane, int n) {
    const int i = 32 * qd + lane;
    float *part = fptr(c, OFF_PART);
    float pa = 1.f;
    for (int t = 32 * th; t < 32 * th + 32; ++t)
        if (t < n) pa *= clamp_alpha(at(c, OFF_KS + x_off(t, i)));
    part[th * 128 + i] = pa;
    __syncthreads();
    const float p0 = part[i], p1 = part[128 + i];
    if (th == 0) fptr(c, OFF_GN)[i] = p0 * p1;
    float g = th ? p0 : 1.f;
    float r = 1.f / g;
    float kt[32], kl[32];
#pragma unroll
    for (int tt = 0; tt < 32; ++tt) {
        const int t = 32 * th + tt;
        const uint32_t o = x_off(t, i);
        float a = (t < n) ? clamp_alpha(at(c, OFF_KS + o)) : 1.f;
        g *= a;
        r *= __fdividef(1.f, a);
        const float kk = ldbf(c.sm + OFF_RK + t * 256 + i * 2);
        const float qq = ldbf(c.sm + OFF_RQ + t * 256 + i * 2);
        const float bb = at(c, OFF_X1 + o);
        at(c, OFF_X1 + o) = to_tf32(bb * kk * g);
        at(c, OFF_X1 + x_off(64 + t, i)) = to_tf32(qq * g);
        const float kf = kk * r;
        kt[tt] = to_tf32(kf);
        kl[tt] = to_tf32(kf - kt[tt]);
        at(c, OFF_KS + o) = kt[tt];
    }
    tmem_st32(tmem + ((uint32_t)(32 * qd) << 16) + TM_KT + 32 * th, kt);
    tmem_st32(tmem + ((uint32_t)(32 * qd) << 16) + TM_KL + 32 * th, kl);
    // Z = w * v in place over w (FP32; used only by the R epilogue).
    const int j2 = tid & 31, tg = tid >> 5;
    for (int m = 0; m < 8; ++m) {
        const int t = tg + 8 * m;
        float2 *pz = reinterpret_cast<float2 *>(c.sm + OFF_ZW + zw_off(t, 2 * j2));
        const float2 w = *pz;
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(c.sm + OFF_RV + t * 128 + j2 * 4);
        const float2 vf = __bfloat1622float2(v);
        *pz = make_float2(w.x * vf.x, w.y * vf.y);
    }
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1}, A strictly lower 64 x 64 (FP32, As), result in Ts (FP32,
// zero above the diagonal).  16 x 16 diagonal blocks by forward substitution,
// then T_ab = -T_aa (sum_c A_ac T_cb) for the 16- and 32-wide off-diagonal blocks.
__device__ __forceinline__ void solve(const Ctx &c, int tid) {
    const float *As = fptr(c, OFF_AS);
    float *Ts = fptr(c, OFF_TS);
    float *Xs = fptr(c, OFF_XS);
    if (tid < 64) {
        const int a = tid >> 4, j = tid & 15, base = 16 * a;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
            for (int l = 0; l < i; ++l) acc = fmaf(-As[(base + i) * LDA + base + l], x[l], acc);
            x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Ts[(base + i) * LDA + base + j] = x[i];
    } else {
        // zero the blocks above the diagonal: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
        for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
            const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
            const int a = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int b = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            Ts[(16 * a + i) * LDA + 16 * b + j] = 0.f;
        }
    }
    __syncthreads();
    // T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22
    for (int e = tid; e < 512; e += kThreads) {
        const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(As[(16 * a + i) * LDA + 16 * b + l], Ts[(16 * b + l) * LDA + 16 * b + j], acc);
        Xs[blk * 16 * LDX + i * LDX + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 512; e += kThreads) {
        const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(Ts[(16 * a + i) * LDA + 16 * a + l], Xs[blk * 16 * LDX + l * LDX + j], acc);
        Ts[(16 * a + i) * LDA + 16 * b + j] = -acc;
    }
    __syncthreads();
    // lower-left 32 x 32 block: T_BA = -T_BB A_BA T_AA
    for (int e = tid; e < 1024; e += kThreads) {
        const int i = e >> 5, j = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc = fmaf(As[(32 + i) * LDA + l], Ts[l * LDA + j], acc);
        Xs[i * LDX + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += kThreads) {
        const int i = e >> 5, j = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc = fmaf(Ts[(32 + i) * LDA + 32 + l], Xs[l * LDX + j], acc);
        Ts[(32 + i) * LDA + j] = -acc;
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ Maps maps, const float *S0, __nv_bfloat16 *__restrict__ o, float *S_T,
                int T, int H) {
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    c.sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    c.sa = smem_u32(c.sm);
    for (int i = 0; i < NBARS; ++i) c.bar[i] = c.sa + OFF_BAR + 8 * i;
    uint32_t *misc = reinterpret_cast<uint32_t *>(c.sm + OFF_MISC);
    volatile uint32_t *abort_flag = misc + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, chh = warp >> 2;          // TMEM lane quarter, column half
    const int head = blockIdx.x >> 1, half = blockIdx.x & 1;
    const int bidx = head / H, h = head % H;
    const int col0 = half * kDVS;
    const int nchunks = (T + kC - 1) / kC;
    const int srow = 32 * qd + lane;                    // the TMEM lane this thread reads

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(c.bar[i], 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_map(&maps.q); tma_prefetch_map(&maps.k); tma_prefetch_map(&maps.v);
        tma_prefetch_map(&maps.alpha); tma_prefetch_map(&maps.b); tma_prefetch_map(&maps.w);
    }
    if (warp == 0) {
        tmem_alloc(c.sa + OFF_MISC, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const uint32_t tlane = tmem + ((uint32_t)(32 * qd) << 16);   // this warp's lane quarter
    if (tid == 0) {
        load_qkv(c, maps, h, 0, bidx, col0);
        load_alpha(c, maps, h, 0, bidx);
        load_b(c, maps, h, 0, bidx);
        load_w(c, maps, h, 0, bidx, col0);
    }

    // State slice owned by this thread: key channel i = srow, value columns
    // col0 + 32*chh + [0, 32).  FP32 in registers across all chunks; its TF32
    // copy is KS rows 64 + j (j = local column), channel i.
    float S[32];
    {
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * chh;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + off + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) at(c, OFF_KS + x_off(64 + 32 * chh + j, srow)) = to_tf32(S[j]);
    }

    uint32_t mma_phase = 0;
    bool ok = true;
    auto wait_all = [&](int which, uint32_t parity) {
        if (!mbar_wait(c.bar[which], parity, kWaitLimit)) {
            *abort_flag = 1;
            atomicExch(&g_device_error, 1u + (unsigned)which);
        }
        __syncthreads();
        return *abort_flag == 0;
    };
    auto mma_wait = [&]() {
        const bool r = wait_all(BAR_MMA, mma_phase);
        mma_phase ^= 1u;
        tc_fence_after();
        return r;
    };
    auto sync_for_mma = [&]() {   // make this phase's smem / TMEM writes visible to the tensor core
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    };

    for (int ck = 0; ck < nchunks && ok; ++ck) {
        const int t0 = ck * kC;
        const int n = min(kC, T - t0);
        const uint32_t ph = ck & 1;
        const bool more = ck + 1 < nchunks;
        // ---- gate prep
        if (!(ok = wait_all(BAR_QKV, ph) && wait_all(BAR_A, ph) && wait_all(BAR_B, ph) && wait_all(BAR_W, ph))) break;
        prep(c, tmem, tid, qd, chh, lane, n);
        sync_for_mma();
        // ---- [Etil; Qtil] x [Ktil; S^T]^T -> TM_G (Gram) and TM_X (Etil S, Qtil S)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 128, 0, 0);
            for (int kk = 0; kk < 16; ++kk) {
                const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_tf32(tmem + TM_G, sdesc_sw128(c.sa + OFF_X1 + koff, 16, 1024),
                         sdesc_sw128(c.sa + OFF_KS + koff, 16, 1024), id, kk > 0);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (tid == 0 && more) {     // X1 and the Ktil rows of KS are consumed: next b and alpha
            load_alpha(c, maps, h, t0 + kC, bidx);
            load_b(c, maps, h, t0 + kC, bidx);
        }
        {
            float g[32];
            tmem_ld32(tlane + TM_G + 32 * chh, g);
            if (srow < 64) {        // A row (strictly lower) and R = Z - Etil S
                float *As = fptr(c, OFF_AS);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * chh + j;
                    As[srow * LDA + s] = (s < srow) ? g[j] : 0.f;
                }
                float x[32];
                tmem_ld32(tlane + TM_X + 32 * chh, x);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int col = 32 * chh + j;
                    const float rr = at(c, OFF_ZW + zw_off(srow, col)) - x[j];
                    const float hi = to_tf32(rr);
                    at(c, OFF_RU + ru_off(col, srow)) = hi;
                    at(c, OFF_RL + ru_off(col, srow)) = to_tf32(rr - hi);
                }
            } else {                // P row (lower incl. diagonal) -> A operand in TMEM
                const int t = srow - 64;
#pragma unroll
                for (int j = 0; j < 32; ++j) g[j] = (32 * chh + j <= t) ? to_tf32(g[j]) : 0.f;
                tmem_st32(tlane + TM_TP + 32 * chh, g);
            }
        }
        sync_for_mma();
        if (tid == 0 && more) load_w(c, maps, h, t0 + kC, bidx, col0);   // Z consumed
        solve(c, tid);
        if (srow < 64) {            // T rows -> A operand in TMEM
            float tv[32];
            const float *Ts = fptr(c, OFF_TS);
#pragma unroll
            for (int j = 0; j < 32; ++j) tv[j] = to_tf32(Ts[srow * LDA + 32 * chh + j]);
            tmem_st32(tlane + TM_TP + 32 * chh, tv);
        }
        sync_for_mma();
        // ---- U = [T; P] R (lanes 0-63)
        if (tid == 0) {
            if (more) load_qkv(c, maps, h, t0 + kC, bidx, col0);         // staging free again
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_tf32_ts(tmem + TM_U, tmem + TM_TP + 8 * kk, sdesc_sw128(c.sa + OFF_RU + koff, 16, 1024), id, kk > 0);
                mma_tf32_ts(tmem + TM_U, tmem + TM_TP + 8 * kk, sdesc_sw128(c.sa + OFF_RL + koff, 16, 1024), id, 1);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (srow < 64) {            // U -> RU (transposed)
            float u[32];
            tmem_ld32(tlane + TM_U + 32 * chh, u);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float hi = to_tf32(u[j]);
                at(c, OFF_RU + ru_off(32 * chh + j, srow)) = hi;
                at(c, OFF_RL + ru_off(32 * chh + j, srow)) = to_tf32(u[j] - hi);
            }
        }
        sync_for_mma();
        // ---- Ktil^T U -> TM_D;  [T; P] U accumulated onto TM_X (lanes 64-127 become O)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
                const uint64_t uh = sdesc_sw128(c.sa + OFF_RU + koff, 16, 1024);
                const uint64_t ul = sdesc_sw128(c.sa + OFF_RL + koff, 16, 1024);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, uh, id, kk > 0);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, ul, id, 1);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KL + 8 * kk, uh, id, 1);
            }
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_tf32_ts(tmem + TM_X, tmem + TM_TP + 8 * kk, sdesc_sw128(c.sa + OFF_RU + koff, 16, 1024), id, 1);
                mma_tf32_ts(tmem + TM_X, tmem + TM_TP + 8 * kk, sdesc_sw128(c.sa + OFF_RL + koff, 16, 1024), id, 1);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        {   // state: S <- gamma_n (S + Ktil^T U); TF32 operand copy for the next chunk
            float d[32];
            tmem_ld32(tlane + TM_D + 32 * chh, d);
            const float gn = fptr(c, OFF_GN)[srow];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                S[j] = gn * (S[j] + d[j]);
                at(c, OFF_KS + x_off(64 + 32 * chh + j, srow)) = to_tf32(S[j]);
            }
        }
        if (srow >= 64) {           // outputs from lanes 64-127 of TM_X
            float v[32];
            tmem_ld32(tlane + TM_X + 32 * chh, v);
            const int t = srow - 64;
            if (t < n) {
                __nv_bfloat16 *dst = o + (((size_t)bidx * T + t0 + t) * H + h) * 128 + col0 + 32 * chh;
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint4 pk;
                    __nv_bfloat162 p0 = __floats2bfloat162_rn(v[j], v[j + 1]);
                    __nv_bfloat162 p1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
                    __nv_bfloat162 p2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]);
                    __nv_bfloat162 p3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
                    pk.x = *reinterpret_cast<uint32_t *>(&p0);
                    pk.y = *reinterpret_cast<uint32_t *>(&p1);
                    pk.z = *reinterpret_cast<uint32_t *>(&p2);
                    pk.w = *reinterpret_cast<uint32_t *>(&p3);
                    *reinterpret_cast<uint4 *>(dst + j) = pk;
                }
            }
        }
        sync_for_mma();
    }

    if (ok && S_T) {
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * chh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(S_T + off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (!ok && tid == 0) {
        // Drain copies still in flight (bounded) before the CTA releases its shared memory.
        for (int i = 0; i < NBARS; ++i) (void)mbar_wait(c.bar[i], 0, kWaitLimit / 8);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (driver entry point fetched through the runtime).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [B][T][H][d] tensor; box = {box_d, 1, 64, 1}.
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, size_t es, int B, int T, int H, int d,
              int box_d, bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)T * H * d * es};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, dt, 4, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc

bool chunk_tc_supported(int dk, int dv, gdn2_dtype dt) { return dk == 128 && dv == 128 && dt == GDN2_BF16; }

cudaError_t read_device_error(unsigned int *value, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                            const float *w, const float *S0, void *o, float *S_T, int B, int T, int H,
                            cudaStream_t stream) {
    using namespace tc;
    Maps m;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!make_map(&m.q, q, BF, 2, B, T, H, kDK, 128, false) || !make_map(&m.k, k, BF, 2, B, T, H, kDK, 128, false) ||
        !make_map(&m.v, v, BF, 2, B, T, H, 128, 64, false) ||
        !make_map(&m.alpha, alpha, F32, 4, B, T, H, kDK, 32, true) ||
        !make_map(&m.b, b, F32, 4, B, T, H, kDK, 32, true) || !make_map(&m.w, w, F32, 4, B, T, H, 128, 32, true))
        return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const unsigned grid = 2u * (unsigned)B * (unsigned)H;
    chunk_tc_kernel<<<grid, kThreads, SMEM_BYTES, stream>>>(m, S0, static_cast<__nv_bfloat16 *>(o), S_T, T, H);
    return cudaGetLastError();
}

}  // namespace gdn2
