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
//   A = strict_tril(Etil Ktil^T),  P = tril(Qtil Ktil^T)         (Gram, tensor core)
//   T = (I + A)^{-1}                                            (FP32 blocked solve)
//   W = T Etil,  Y = T Z                                        (tensor core)
//   U = Y - W S                                                 (tensor core + epilogue)
//   O = Qtil S + P U                                            (tensor core)
//   S <- diag(gamma_n) (S + Ktil^T U)                           (tensor core + FP32 epilogue)
//
// Precision: every operand is rounded to TF32 (10-bit mantissa); accumulation,
// decay, solve and the carried state are FP32.  With BF16 operands the products
// of decay-scaled factors lose too much (the read r = Sbar^T e nearly cancels
// the write z in the delta rule), so TF32 is used throughout.  The key factor
// Ktil = k / gamma grows within a chunk as exp(-sum ln alpha); the kernel
// requires that growth to stay below ~1e34 (sum of -ln alpha over one chunk
// <= 78 per key channel), documented in gdn2.h.
//
// Layout: one CTA per (batch, head, 64-column half of d_v); 256 threads (8
// warps) run the phases of a chunk in turn; thread 0 issues TMA loads and MMAs.
// alpha, b and w are TMA-loaded (128-byte swizzle) straight into the operand
// tiles they become (Ktil, Etil, Z) and transformed in place, so a chunk needs
// ~220 KB of shared memory.  Tensor Memory: 512 columns.
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

// Shared-memory map (bytes from a 1024-aligned base).  128-byte-swizzled tiles
// of FP32/TF32 elements, 32 elements per 128-byte row:
//   X1  [Etil -> W ; Qtil]  K-major, 128 rows x 128 channels, 4 atoms of 16 KB
//   KT  Ktil                 64 tokens x 128 channels, 4 atoms of 8 KB
//   ZU  Z, later U           64 tokens x 64 columns, 2 atoms of 8 KB
//   TP  [T ; P]              K-major, 128 rows x 64 tokens, 2 atoms of 16 KB
//   ST  S (operand copy)     128 channels x 64 columns, 2 atoms of 16 KB
// Raw (unswizzled) BF16 staging for q, k (64 x 128) and v (64 x 64).
constexpr uint32_t OFF_X1 = 0;
constexpr uint32_t OFF_KT = OFF_X1 + 65536;
constexpr uint32_t OFF_ZU = OFF_KT + 32768;
constexpr uint32_t OFF_TP = OFF_ZU + 16384;
constexpr uint32_t OFF_ST = OFF_TP + 32768;
constexpr uint32_t OFF_RQ = OFF_ST + 32768;
constexpr uint32_t OFF_RK = OFF_RQ + 16384;
constexpr uint32_t OFF_RV = OFF_RK + 16384;
constexpr uint32_t OFF_GN = OFF_RV + 8192;      // float[128]   decay over the chunk
constexpr uint32_t OFF_PART = OFF_GN + 512;     // float[4][128] partial decay products
constexpr uint32_t OFF_BAR = OFF_PART + 2048;   // 6 mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 64;     // tmem base, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack
// Solve scratch, inside the q/k staging (free between prep and the next load).
constexpr uint32_t OFF_AS = OFF_RQ;             // float[64][65]  A (strictly lower)
constexpr uint32_t OFF_XS = OFF_RQ + 16896;     // float[32][33]  block-product scratch
constexpr int LDA = 65, LDX = 33;

// Tensor Memory columns.
constexpr uint32_t TM_G = 0;      // Gram: lanes 0-63 A, lanes 64-127 P          (64 cols)
constexpr uint32_t TM_W = 64;     // W = T Etil (lanes 0-63)                      (128 cols)
constexpr uint32_t TM_Y = 192;    // Y = T Z   (lanes 0-63)                       (64 cols)
constexpr uint32_t TM_X = 256;    // lanes 0-63 W S, lanes 64-127 Qtil S + P U    (64 cols)
constexpr uint32_t TM_D = 320;    // Ktil^T U                                     (64 cols)
constexpr uint32_t TM_COLS = 512;

enum { BAR_QKV = 0, BAR_A, BAR_B, BAR_W, BAR_MMA, NBARS };

// TMA byte counts per chunk.
constexpr uint32_t TX_QKV = 16384 + 16384 + 8192;
constexpr uint32_t TX_A = 4 * 8192;
constexpr uint32_t TX_B = 4 * 8192;
constexpr uint32_t TX_W = 2 * 8192;

// Element byte offsets inside the tiles.
__device__ __forceinline__ uint32_t x1_off(uint32_t r, uint32_t i) { return (i >> 5) * 16384u + swz128(r, (i & 31u) * 4u); }
__device__ __forceinline__ uint32_t kt_off(uint32_t t, uint32_t i) { return (i >> 5) * 8192u + swz128(t, (i & 31u) * 4u); }
__device__ __forceinline__ uint32_t zu_off(uint32_t t, uint32_t j) { return (j >> 5) * 8192u + swz128(t, (j & 31u) * 4u); }
__device__ __forceinline__ uint32_t tp_off(uint32_t r, uint32_t s) { return (s >> 5) * 16384u + swz128(r, (s & 31u) * 4u); }
__device__ __forceinline__ uint32_t st_off(uint32_t i, uint32_t j) { return (j >> 5) * 16384u + swz128(i, (j & 31u) * 4u); }

struct Maps {
    CUtensorMap q, k, v, alpha, b, w;
};

struct Ctx {
    uint8_t *sm;          // 1024-aligned shared base (generic pointer)
    uint32_t sa;          // same, shared-window address
    uint32_t bar[NBARS];
};

__device__ __forceinline__ float *fptr(const Ctx &c, uint32_t off) { return reinterpret_cast<float *>(c.sm + off); }

// Issue the TMA loads of one chunk's inputs (thread 0 only).
__device__ __forceinline__ void load_qkv(const Ctx &c, const Maps &m, int h, int t0, int bidx, int col0) {
    mbar_expect_tx(c.bar[BAR_QKV], TX_QKV);
    tma_load_4d(c.sa + OFF_RQ, &m.q, 0, h, t0, bidx, c.bar[BAR_QKV]);
    tma_load_4d(c.sa + OFF_RK, &m.k, 0, h, t0, bidx, c.bar[BAR_QKV]);
    tma_load_4d(c.sa + OFF_RV, &m.v, col0, h, t0, bidx, c.bar[BAR_QKV]);
}
__device__ __forceinline__ void load_alpha(const Ctx &c, const Maps &m, int h, int t0, int bidx) {
    mbar_expect_tx(c.bar[BAR_A], TX_A);
    for (int a = 0; a < 4; ++a) tma_load_4d(c.sa + OFF_KT + a * 8192, &m.alpha, 32 * a, h, t0, bidx, c.bar[BAR_A]);
}
__device__ __forceinline__ void load_b(const Ctx &c, const Maps &m, int h, int t0, int bidx) {
    mbar_expect_tx(c.bar[BAR_B], TX_B);
    for (int a = 0; a < 4; ++a) tma_load_4d(c.sa + OFF_X1 + a * 16384, &m.b, 32 * a, h, t0, bidx, c.bar[BAR_B]);
}
__device__ __forceinline__ void load_w(const Ctx &c, const Maps &m, int h, int t0, int bidx, int col0) {
    mbar_expect_tx(c.bar[BAR_W], TX_W);
    for (int a = 0; a < 2; ++a) tma_load_4d(c.sa + OFF_ZU + a * 8192, &m.w, col0 + 32 * a, h, t0, bidx, c.bar[BAR_W]);
}

__device__ __forceinline__ float2 ldbf2(const uint8_t *p) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(p);
    return __bfloat1622float2(x);
}
__device__ __forceinline__ void st_tf32x2(uint8_t *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(to_tf32(a), to_tf32(b));
}
__device__ __forceinline__ void st_tf32x4(uint8_t *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// ---------------------------------------------------------------------------
// Gate prep: cumulative decay along the chunk (running FP32 products, equal to
// exp of the cumulative log-decay up to rounding) and the operand factors,
// written in place over the loaded gates.  Padding tokens (t >= n) have zero
// q, k, b, w, v from the TMA bounds fill and alpha forced to 1.
__device__ __forceinline__ void prep(const Ctx &c, int tid, int n) {
    const int cp = tid & 63, tq = tid >> 6;        // channel pair, token quarter
    const uint32_t ch = 2u * cp;
    float *part = fptr(c, OFF_PART);
    float2 pa = make_float2(1.f, 1.f);
    for (int t = 16 * tq; t < 16 * tq + 16; ++t) {
        if (t < n) {
            const float2 a = *reinterpret_cast<const float2 *>(c.sm + OFF_KT + kt_off(t, ch));
            pa.x *= clamp_alpha(a.x);
            pa.y *= clamp_alpha(a.y);
        }
    }
    part[tq * 128 + ch] = pa.x;
    part[tq * 128 + ch + 1] = pa.y;
    __syncthreads();
    float g0 = 1.f, g1 = 1.f, tot0 = 1.f, tot1 = 1.f;
    for (int q2 = 0; q2 < 4; ++q2) {
        const float p0 = part[q2 * 128 + ch], p1 = part[q2 * 128 + ch + 1];
        if (q2 < tq) { g0 *= p0; g1 *= p1; }
        tot0 *= p0; tot1 *= p1;
    }
    if (tq == 0) {
        float *gn = fptr(c, OFF_GN);
        gn[ch] = tot0;
        gn[ch + 1] = tot1;
    }
    float r0 = 1.f / g0, r1 = 1.f / g1;
    for (int t = 16 * tq; t < 16 * tq + 16; ++t) {
        uint8_t *pk = c.sm + OFF_KT + kt_off(t, ch);
        uint8_t *pe = c.sm + OFF_X1 + x1_off(t, ch);
        uint8_t *pq = c.sm + OFF_X1 + x1_off(64 + t, ch);
        float2 a = *reinterpret_cast<const float2 *>(pk);
        if (t >= n) a = make_float2(1.f, 1.f);
        a.x = clamp_alpha(a.x);
        a.y = clamp_alpha(a.y);
        g0 *= a.x; g1 *= a.y;
        r0 *= __fdividef(1.f, a.x);
        r1 *= __fdividef(1.f, a.y);
        const float2 kk = ldbf2(c.sm + OFF_RK + t * 256 + ch * 2);
        const float2 qq = ldbf2(c.sm + OFF_RQ + t * 256 + ch * 2);
        const float2 bb = *reinterpret_cast<const float2 *>(pe);
        st_tf32x2(pe, bb.x * kk.x * g0, bb.y * kk.y * g1);
        st_tf32x2(pq, qq.x * g0, qq.y * g1);
        st_tf32x2(pk, kk.x * r0, kk.y * r1);
    }
    // Z = w * v in place over w.
    const int j2 = tid & 31, tg = tid >> 5;
    for (int m = 0; m < 8; ++m) {
        const int t = tg + 8 * m;
        uint8_t *pz = c.sm + OFF_ZU + zu_off(t, 2 * j2);
        const float2 w = *reinterpret_cast<const float2 *>(pz);
        const float2 v = ldbf2(c.sm + OFF_RV + t * 128 + j2 * 4);
        st_tf32x2(pz, w.x * v.x, w.y * v.y);
    }
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1}, A strictly lower 64 x 64 in As (FP32).  Blocked: 16 x 16
// diagonal blocks by forward substitution, then the 16- and 32-wide
// off-diagonal blocks by T_ab = -T_aa (sum_c A_ac T_cb).  T (FP32, zero above
// the diagonal) is written into rows 0-63 of the TP tile.
__device__ __forceinline__ float tget(const Ctx &c, int r, int s) {
    return *reinterpret_cast<const float *>(c.sm + OFF_TP + tp_off(r, s));
}
__device__ __forceinline__ void tset(const Ctx &c, int r, int s, float x) {
    *reinterpret_cast<float *>(c.sm + OFF_TP + tp_off(r, s)) = x;
}

__device__ __forceinline__ void solve(const Ctx &c, int tid) {
    const float *As = fptr(c, OFF_AS);
    float *Xs = fptr(c, OFF_XS);
    // 1. Diagonal 16 x 16 blocks (64 threads: block a, column j); zero the upper blocks.
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
        for (int i = 0; i < 16; ++i) tset(c, base + i, base + j, x[i]);
    } else {
        // upper off-diagonal blocks (a < b): 6 blocks x 256 elements over 192 threads
        for (int e = tid - 64; e < 6 * 256; e += 192) {
            const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
            // blocks (a, b), a < b, in the order (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
            const int a = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int b = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            tset(c, 16 * a + i, 16 * b + j, 0.f);
        }
    }
    __syncthreads();
    // 2. T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22.
    for (int e = tid; e < 512; e += kThreads) {
        const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(As[(16 * a + i) * LDA + 16 * b + l], tget(c, 16 * b + l, 16 * b + j), acc);
        Xs[blk * 16 * LDX + i * LDX + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 512; e += kThreads) {
        const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(tget(c, 16 * a + i, 16 * a + l), Xs[blk * 16 * LDX + l * LDX + j], acc);
        tset(c, 16 * a + i, 16 * b + j, -acc);
    }
    __syncthreads();
    // 3. Lower-left 32 x 32 block: T_BA = -T_BB A_BA T_AA.
    for (int e = tid; e < 1024; e += kThreads) {
        const int i = e >> 5, j = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc = fmaf(As[(32 + i) * LDA + l], tget(c, l, j), acc);
        Xs[i * LDX + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += kThreads) {
        const int i = e >> 5, j = e & 31;
        float acc = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) acc = fmaf(tget(c, 32 + i, 32 + l), Xs[l * LDX + j], acc);
        tset(c, 32 + i, j, -acc);
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
    if (tid == 0) {
        load_qkv(c, maps, h, 0, bidx, col0);
        load_alpha(c, maps, h, 0, bidx);
        load_b(c, maps, h, 0, bidx);
        load_w(c, maps, h, 0, bidx, col0);
    }

    // State slice owned by this thread: key channel i = 32*qd + lane, value
    // columns col0 + 32*chh + [0, 32).  FP32 in registers across all chunks.
    const int srow = 32 * qd + lane;
    float S[32];
    {
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * chh;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + off + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            st_tf32x4(c.sm + OFF_ST + st_off(srow, 32 * chh + j), S[j], S[j + 1], S[j + 2], S[j + 3]);
    }

    const uint32_t tq_lane = (uint32_t)(32 * qd) << 16;   // TMEM lane field of this warp
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

    for (int ck = 0; ck < nchunks && ok; ++ck) {
        const int t0 = ck * kC;
        const int n = min(kC, T - t0);
        const uint32_t ph = ck & 1;
        const bool more = ck + 1 < nchunks;
        // ---- gate prep
        if (!(ok = wait_all(BAR_QKV, ph) && wait_all(BAR_A, ph) && wait_all(BAR_B, ph) && wait_all(BAR_W, ph))) break;
        prep(c, tid, n);
        fence_proxy_async_smem();
        __syncthreads();
        // ---- Gram: [Etil; Qtil] Ktil^T -> TM_G
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
            for (int kk = 0; kk < 16; ++kk) {
                const uint64_t a = sdesc_sw128(c.sa + OFF_X1 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(c.sa + OFF_KT + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                mma_tf32(tmem + TM_G, a, b, id, kk > 0);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        {   // A (rows 0-63, strictly lower, FP32 for the solve) and P (rows 64-127, lower, TF32)
            float v[32];
            tmem_ld32(tmem + tq_lane + TM_G + 32 * chh, v);
            const int r = srow;
            if (r < 64) {
                float *As = fptr(c, OFF_AS);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * chh + j;
                    As[r * LDA + s] = (s < r) ? v[j] : 0.f;
                }
            } else {
                const int t = r - 64;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int s = 32 * chh + j;
                    st_tf32x4(c.sm + OFF_TP + tp_off(r, s), (s <= t) ? v[j] : 0.f, (s + 1 <= t) ? v[j + 1] : 0.f,
                              (s + 2 <= t) ? v[j + 2] : 0.f, (s + 3 <= t) ? v[j + 3] : 0.f);
                }
            }
        }
        __syncthreads();
        solve(c, tid);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- next chunk's q, k, v may land now; W = T Etil, Y = T Z
        if (tid == 0) {
            if (more) load_qkv(c, maps, h, t0 + kC, bidx, col0);
            tc_fence_after();
            const uint32_t idw = idesc_tf32(128, 128, 0, 1), idy = idesc_tf32(128, 64, 0, 1);
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t a = sdesc_sw128(c.sa + OFF_TP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bw = sdesc_sw128(c.sa + OFF_X1 + kk * 1024, 16384, 1024);
                const uint64_t by = sdesc_sw128(c.sa + OFF_ZU + kk * 1024, 8192, 1024);
                mma_tf32(tmem + TM_W, a, bw, idw, kk > 0);
                mma_tf32(tmem + TM_Y, a, by, idy, kk > 0);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (qd < 2) {   // W rows (lanes 0-63) -> X1 rows 0-63, channels [64*chh, 64*chh + 64)
            float v[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c0 = 64 * chh + 32 * hh;
                tmem_ld32(tmem + tq_lane + TM_W + c0, v);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    st_tf32x4(c.sm + OFF_X1 + x1_off(srow, c0 + j), v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- [W; Qtil] S -> TM_X
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 1);
            for (int kk = 0; kk < 16; ++kk) {
                const uint64_t a = sdesc_sw128(c.sa + OFF_X1 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(c.sa + OFF_ST + kk * 1024, 16384, 1024);
                mma_tf32(tmem + TM_X, a, b, id, kk > 0);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (tid == 0 && more) load_b(c, maps, h, t0 + kC, bidx);   // X1 rows 0-63 are free again
        if (qd < 2) {   // U = Y - W S (lanes 0-63) -> ZU tile
            float ws[32], y[32];
            tmem_ld32(tmem + tq_lane + TM_X + 32 * chh, ws);
            tmem_ld32(tmem + tq_lane + TM_Y + 32 * chh, y);
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                st_tf32x4(c.sm + OFF_ZU + zu_off(srow, 32 * chh + j), y[j] - ws[j], y[j + 1] - ws[j + 1],
                          y[j + 2] - ws[j + 2], y[j + 3] - ws[j + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- Ktil^T U -> TM_D;  [T; P] U accumulated onto TM_X (lanes 64-127 become O)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idd = idesc_tf32(128, 64, 1, 1), ido = idesc_tf32(128, 64, 0, 1);
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t ak = sdesc_sw128(c.sa + OFF_KT + kk * 1024, 8192, 1024);
                const uint64_t at = sdesc_sw128(c.sa + OFF_TP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bu = sdesc_sw128(c.sa + OFF_ZU + kk * 1024, 8192, 1024);
                mma_tf32(tmem + TM_D, ak, bu, idd, kk > 0);
                mma_tf32(tmem + TM_X, at, bu, ido, 1);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (tid == 0 && more) {    // Ktil and Z/U tiles are free: next alpha and w
            load_alpha(c, maps, h, t0 + kC, bidx);
            load_w(c, maps, h, t0 + kC, bidx, col0);
        }
        {   // state: S <- gamma_n (S + Ktil^T U); operand copy for the next chunk
            float d[32];
            tmem_ld32(tmem + tq_lane + TM_D + 32 * chh, d);
            const float gn = fptr(c, OFF_GN)[srow];
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = gn * (S[j] + d[j]);
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                st_tf32x4(c.sm + OFF_ST + st_off(srow, 32 * chh + j), S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (qd >= 2) {   // outputs: lanes 64-127 of TM_X
            float v[32];
            tmem_ld32(tmem + tq_lane + TM_X + 32 * chh, v);
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
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (ok && S_T) {
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * chh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(S_T + off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (!ok && tid == 0) {
        // Drain any copies still in flight (bounded) before the CTA releases its shared memory.
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
