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
//   Etil = b*k*gamma,  Qtil = q*gamma,  Ktil = k*rho            (gate prep)
//   [A | Etil S] and [P | Qtil S] = [Etil; Qtil] [Ktil; S^T]^T  (one tensor-core product)
//   R = w*v - Etil S                                             (FP32 epilogue)
//   (I + strict_tril(A)) U = R                                   (FP32 blocked forward substitution)
//   O = Qtil S + tril(P) U                                       (tensor core, accumulated)
//   S <- diag(gamma_n) (S + Ktil^T U)                            (tensor core + FP32 epilogue)
//
// U holds the per-token corrections z_t - r_t of the token recurrence, so this
// is the token loop's arithmetic, re-associated.
//
// Precision: tensor-core operands are TF32 (10-bit mantissa); accumulation,
// decay, R, the solve and the carried state are FP32.  The state update uses
// split operands, x = x_hi + x_lo with both parts TF32:
//   Ktil^T U = Ktil_hi^T U_hi + Ktil_hi^T U_lo + Ktil_lo^T U_hi,
// which carries about 21 bits of each operand (plain TF32 there lets the state
// drift by ~0.7% of its RMS over 16K tokens; split, ~0.03%).  BF16 operands lose
// too much: the read r = Sbar^T e nearly cancels the write z in the delta rule.
// The key factor Ktil = k / gamma grows within a chunk as exp(-sum ln alpha); it
// must stay below ~1e34 (sum of -ln alpha over one chunk <= 78 per key channel),
// as documented in gdn2.h.
//
// Layout: one CTA per (batch, head, 64-column half of d_v); 256 threads (8
// warps) run the phases of a chunk in turn; thread 0 issues TMA loads and MMAs.
// Every shared-memory MMA operand is K-major with the 128-byte swizzle.  The
// operands needed transposed (Ktil^T, P) are written to Tensor Memory and read
// from there as the A operand.  alpha, b and w are TMA-loaded straight into the
// tiles they become and transformed in place; each next-chunk load is issued as
// soon as its tile is consumed.
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

// Shared-memory map (bytes from a 1024-aligned base).  MMA tiles hold TF32,
// 32 elements per 128-byte swizzled row, K-major:
//   X1  rows 0-63 Etil[t][i], rows 64-127 Qtil[t][i]         4 atoms x 16 KB (i = key channel)
//   KS  rows 0-63 Ktil_hi[s][i], rows 64-127 S[i][j] as [j][i]  4 atoms x 16 KB
//   UH  U_hi as [j][t]                                        2 atoms x 8 KB (t = token)
//   UL  U_lo as [j][t]                                        2 atoms x 8 KB
//   ZW  w, then R, then U, as [t][j] (FP32, same swizzle)     2 atoms x 8 KB
// and unswizzled BF16 staging of q, k (64 x 128) and v (64 x 64).
constexpr uint32_t OFF_X1 = 0;
constexpr uint32_t OFF_KS = OFF_X1 + 65536;
constexpr uint32_t OFF_UH = OFF_KS + 65536;
constexpr uint32_t OFF_UL = OFF_UH + 16384;
constexpr uint32_t OFF_ZW = OFF_UL + 16384;
constexpr uint32_t OFF_RQ = OFF_ZW + 16384;
constexpr uint32_t OFF_RK = OFF_RQ + 16384;
constexpr uint32_t OFF_RV = OFF_RK + 16384;
constexpr uint32_t OFF_GN = OFF_RV + 8192;      // float[128]   decay over the chunk
constexpr uint32_t OFF_PART = OFF_GN + 512;     // float[2][128] half-chunk decay products
constexpr uint32_t OFF_BAR = OFF_PART + 1024;   // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 64;     // tmem base, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack
// Solve scratch inside the q/k staging (free between prep and the next load).
constexpr int LDA = 65, LDD = 17;
constexpr uint32_t OFF_AS = OFF_RQ;             // float[64][65]    A, strictly lower
constexpr uint32_t OFF_DS = OFF_AS + 16896;     // float[4][16][17] inverses of the diagonal blocks
static_assert(OFF_DS + 4 * 16 * LDD * 4 <= OFF_RV, "solve scratch overlaps the v staging");

// Tensor Memory columns (512 allocated).
constexpr uint32_t TM_G = 0;      // [Etil;Qtil] Ktil^T : lanes 0-63 A, lanes 64-127 P   (64 cols)
constexpr uint32_t TM_X = 64;     // [Etil;Qtil] S, then + P U : lanes 64-127 -> O        (64 cols)
constexpr uint32_t TM_D = 128;    // Ktil^T U                                             (64 cols)
constexpr uint32_t TM_KT = 192;   // A operand Ktil_hi^T: lane i, column s                (64 cols)
constexpr uint32_t TM_KL = 256;   // A operand Ktil_lo^T                                  (64 cols)
constexpr uint32_t TM_P = 320;    // A operand: lanes 64-127 tril(P), lanes 0-63 zero     (64 cols)
constexpr uint32_t TM_COLS = 512;

enum { BAR_QKV = 0, BAR_A, BAR_B, BAR_W, BAR_MMA, NBARS };

constexpr uint32_t TX_QKV = 16384 + 16384 + 8192;
constexpr uint32_t TX_A = 4 * 8192;
constexpr uint32_t TX_B = 4 * 8192;
constexpr uint32_t TX_W = 2 * 8192;

// Element byte offsets inside the tiles.
__device__ __forceinline__ uint32_t x_off(uint32_t r, uint32_t i) { return (i >> 5) * 16384u + swz128(r, (i & 31u) * 4u); }
__device__ __forceinline__ uint32_t u_off(uint32_t j, uint32_t t) { return (t >> 5) * 8192u + swz128(j, (t & 31u) * 4u); }
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
__device__ __forceinline__ float4 &at4(const Ctx &c, uint32_t off) { return *reinterpret_cast<float4 *>(c.sm + off); }

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
// (t >= n) have zero q, k, b from the TMA bounds fill and alpha forced to 1.
// Tokens go in groups of 8; a group's loads are issued before the previous
// group's stores so the in-place writes never stall the reads.
__device__ __forceinline__ void prep(const Ctx &c, uint32_t tlane, int qd, int th, int lane, int n) {
    const int i = 32 * qd + lane;
    float *part = fptr(c, OFF_PART);
    const uint32_t ci = (i >> 5) * 16384u;       // atom of channel i
    const uint32_t cb = (i & 31) * 4u;           // byte in row
    float pa = 1.f;
#pragma unroll
    for (int tt = 0; tt < 32; ++tt) {
        const int t = 32 * th + tt;
        const float a = at(c, OFF_KS + ci + swz128(t, cb));
        pa *= (t < n) ? clamp_alpha(a) : 1.f;
    }
    part[th * 128 + i] = pa;
    __syncthreads();
    const float p0 = part[i], p1 = part[128 + i];
    if (th == 0) fptr(c, OFF_GN)[i] = p0 * p1;
    float g = th ? p0 : 1.f;
    float r = 1.f / g;
    float av[8], kv[8], qv[8], bv[8];
    auto load_group = [&](int g8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = 32 * th + 8 * g8 + u;
            av[u] = at(c, OFF_KS + ci + swz128(t, cb));
            bv[u] = at(c, OFF_X1 + ci + swz128(t, cb));
            kv[u] = ldbf(c.sm + OFF_RK + t * 256 + i * 2);
            qv[u] = ldbf(c.sm + OFF_RQ + t * 256 + i * 2);
        }
    };
    load_group(0);
#pragma unroll
    for (int g8 = 0; g8 < 4; ++g8) {
        float e[8], qt[8], kh[8], kl[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = 32 * th + 8 * g8 + u;
            const float a = (t < n) ? clamp_alpha(av[u]) : 1.f;
            g *= a;
            r *= __fdividef(1.f, a);
            e[u] = to_tf32(bv[u] * kv[u] * g);
            qt[u] = to_tf32(qv[u] * g);
            const float kf = kv[u] * r;
            kh[u] = to_tf32(kf);
            kl[u] = to_tf32(kf - kh[u]);
        }
        if (g8 < 3) load_group(g8 + 1);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = 32 * th + 8 * g8 + u;
            at(c, OFF_X1 + ci + swz128(t, cb)) = e[u];
            at(c, OFF_X1 + ci + swz128(64 + t, cb)) = qt[u];
            at(c, OFF_KS + ci + swz128(t, cb)) = kh[u];
        }
        tmem_st8(tlane + TM_KT + 32 * th + 8 * g8, kh);
        tmem_st8(tlane + TM_KL + 32 * th + 8 * g8, kl);
    }
}

// ---------------------------------------------------------------------------
// Solve (I + A) U = R in FP32, A strictly lower 64 x 64 (As), R and U in the ZW
// tile ([t][j], 64 value columns).  The inverses D_b of the four 16 x 16
// diagonal blocks come first (forward substitution, one thread per column);
// then, block by block, R'_b = R_b - sum_{c<b} A_bc U_c and U_b = D_b R'_b.
// Thread (i, cg) owns row 16 b + i, columns 4 cg .. 4 cg + 3 of each block.
__device__ __forceinline__ void fma4(float4 &acc, float a, const float4 &x) {
    acc.x = fmaf(a, x.x, acc.x); acc.y = fmaf(a, x.y, acc.y); acc.z = fmaf(a, x.z, acc.z); acc.w = fmaf(a, x.w, acc.w);
}

__device__ __forceinline__ void solve_u(const Ctx &c, int tid) {
    const float *As = fptr(c, OFF_AS);
    float *Ds = fptr(c, OFF_DS);
    if (tid < 64) {
        const int b = tid >> 4, j = tid & 15, base = 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
            for (int l = 0; l < i; ++l) acc = fmaf(-As[(base + i) * LDA + base + l], x[l], acc);
            x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Ds[(b * 16 + i) * LDD + j] = x[i];
    }
    __syncthreads();
    const int i = tid >> 4, cg = tid & 15;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int row = 16 * b + i;
        const uint32_t my = OFF_ZW + zw_off(row, 4 * cg);
        float4 acc = at4(c, my);
#pragma unroll
        for (int l = 0; l < 16 * b; ++l) fma4(acc, -As[row * LDA + l], at4(c, OFF_ZW + zw_off(l, 4 * cg)));
        at4(c, my) = acc;
        __syncthreads();
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m <= i) fma4(u, Ds[(b * 16 + i) * LDD + m], at4(c, OFF_ZW + zw_off(16 * b + m, 4 * cg)));
        __syncthreads();
        at4(c, my) = u;
        __syncthreads();
    }
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
    if (srow < 64) {   // rows 0-63 of the P operand stay zero
        float z[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = 0.f;
        tmem_st32(tlane + TM_P + 32 * chh, z);
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
        if (!(ok = wait_all(BAR_QKV, ph) && wait_all(BAR_A, ph) && wait_all(BAR_B, ph))) break;
        prep(c, tlane, qd, chh, lane, n);
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
        if (!(ok = mma_wait() && wait_all(BAR_W, ph))) break;
        if (tid == 0 && more) {     // X1 and the Ktil rows of KS are consumed: next b and alpha
            load_alpha(c, maps, h, t0 + kC, bidx);
            load_b(c, maps, h, t0 + kC, bidx);
        }
        {
            float g[32];
            tmem_ld32(tlane + TM_G + 32 * chh, g);
            if (srow < 64) {        // A row (strictly lower) and R = w*v - Etil S, in place over w
                float *As = fptr(c, OFF_AS);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * chh + j;
                    As[srow * LDA + s] = (s < srow) ? g[j] : 0.f;
                }
                float x[32];
                tmem_ld32(tlane + TM_X + 32 * chh, x);
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int col = 32 * chh + j;
                    float4 &wr = at4(c, OFF_ZW + zw_off(srow, col));
                    const float4 w = wr;
                    const uint2 vb = *reinterpret_cast<const uint2 *>(c.sm + OFF_RV + srow * 128 + col * 2);
                    const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.x));
                    const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.y));
                    wr = make_float4(w.x * v01.x - x[j], w.y * v01.y - x[j + 1], w.z * v23.x - x[j + 2],
                                     w.w * v23.y - x[j + 3]);
                }
            } else {                // P row (lower incl. diagonal) -> A operand in TMEM
                const int t = srow - 64;
#pragma unroll
                for (int j = 0; j < 32; ++j) g[j] = (32 * chh + j <= t) ? to_tf32(g[j]) : 0.f;
                tmem_st32(tlane + TM_P + 32 * chh, g);
            }
        }
        __syncthreads();
        solve_u(c, tid);
        // U (FP32, ZW) -> U_hi, U_lo tiles as [j][t]
        {
            const int t = srow >> 1;                       // token row; two threads per row
            const int j0 = 32 * (srow & 1) + 16 * chh;     // 16 columns each
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 u = at4(c, OFF_ZW + zw_off(t, j0 + j));
                const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float hi = to_tf32(uu[e]);
                    at(c, OFF_UH + u_off(j0 + j + e, t)) = hi;
                    at(c, OFF_UL + u_off(j0 + j + e, t)) = to_tf32(uu[e] - hi);
                }
            }
        }
        sync_for_mma();
        // ---- Ktil^T U -> TM_D (split);  P U_hi accumulated onto TM_X (lanes 64-127 become O)
        if (tid == 0) {
            if (more) {                  // solve scratch and ZW consumed: next q, k, v and w
                load_qkv(c, maps, h, t0 + kC, bidx, col0);
                load_w(c, maps, h, t0 + kC, bidx, col0);
            }
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
                const uint64_t uh = sdesc_sw128(c.sa + OFF_UH + koff, 16, 1024);
                const uint64_t ul = sdesc_sw128(c.sa + OFF_UL + koff, 16, 1024);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, uh, id, kk > 0);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, ul, id, 1);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KL + 8 * kk, uh, id, 1);
                mma_tf32_ts(tmem + TM_X, tmem + TM_P + 8 * kk, uh, id, 1);
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
