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
//   T = (I + strict_tril(A))^{-1}                                (FP32 blocked inversion)
//   R = w*v - Etil S                                             (FP32 epilogue)
//   U = T R                                                      (tensor core)
//   O = Qtil S + tril(P) U                                       (tensor core, accumulated)
//   S <- diag(gamma_n) (S + Ktil^T U)                            (tensor core + FP32 epilogue)
//
// U holds the per-token corrections z_t - r_t of the token recurrence, so this
// is the token loop's arithmetic, re-associated.
//
// Precision: tensor-core operands are TF32 (10-bit mantissa); accumulation,
// decay, R, T and the carried state are FP32.  The state path uses split
// operands, x = x_hi + x_lo with both parts TF32:
//   T R = T R_hi + T R_lo,  Ktil^T U = Ktil_hi^T U_hi + Ktil_hi^T U_lo + Ktil_lo^T U_hi,
// which carries about 21 bits of each operand (plain TF32 there lets the state
// drift by ~0.7% of its RMS over 16K tokens; split, ~0.03%).  BF16 operands lose
// too much: the read r = Sbar^T e nearly cancels the write z in the delta rule.
// The key factor Ktil = k / gamma grows within a chunk as exp(-sum ln alpha); it
// must stay below ~1e34 (sum of -ln alpha over one chunk <= 78 per key channel),
// as documented in gdn2.h.
//
// Layout: one CTA per (batch, head, 64-column half of d_v); 512 threads (16
// warps) run the phases of a chunk in turn; thread 0 issues TMA loads and MMAs.
// Warp w reads Tensor Memory lanes 32 (w % 4) .. +31 and owns the 16-column
// quarter w / 4 of every 64-column accumulator.  Every shared-memory MMA operand
// is K-major with the 128-byte swizzle; the operands needed transposed (Ktil^T,
// [T; P]) are written to Tensor Memory and read from there as the A operand.
// alpha, b and w are TMA-loaded straight into the tiles they become and
// transformed in place; each next-chunk load is issued as soon as its tile is
// consumed.
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
constexpr int kThreads = 512;
constexpr long long kWaitLimit = 4000000000ll;   // ~2 s of SM cycles per wait

// Shared-memory map (bytes from a 1024-aligned base).  MMA tiles hold TF32,
// 32 elements per 128-byte swizzled row, K-major:
//   X1  rows 0-63 Etil[t][i], rows 64-127 Qtil[t][i]         4 atoms x 16 KB (i = key channel)
//   KS  rows 0-63 Ktil_hi[s][i], rows 64-127 S[i][j] as [j][i]  4 atoms x 16 KB
//   UH  R_hi, later U_hi, as [j][t]                           2 atoms x 8 KB (t = token)
//   UL  R_lo, later U_lo, as [j][t]                           2 atoms x 8 KB
//   ZW  w as [t][j] (FP32, same swizzle; TMA destination)     2 atoms x 8 KB
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
constexpr uint32_t OFF_PART = OFF_GN + 512;     // float[4][128] quarter-chunk decay products
constexpr uint32_t OFF_BAR = OFF_PART + 2048;   // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 64;     // tmem base, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack
// Inversion scratch inside the q/k/v staging (A is written after the prep has
// consumed q and k; T only after the R epilogue has consumed v).
constexpr int LDT = 66;
constexpr uint32_t OFF_AT = OFF_RQ;                     // float[64][66]  A transposed: AT[s][t] = A[t][s]
constexpr uint32_t OFF_TS = OFF_AT + 64 * LDT * 4;      // float[64][66]  T
constexpr uint32_t OFF_XS = OFF_TS + 64 * LDT * 4;      // float[32][34]  block products
constexpr int LDX = 34;
static_assert(OFF_AT + 64 * LDT * 4 <= OFF_RV, "A scratch overlaps the v staging");
static_assert(OFF_XS + 32 * LDX * 4 <= OFF_GN, "inversion scratch overflows the staging area");

// Tensor Memory columns (512 allocated).
constexpr uint32_t TM_G = 0;      // [Etil;Qtil] Ktil^T : lanes 0-63 A, lanes 64-127 P   (64 cols)
constexpr uint32_t TM_X = 64;     // [Etil;Qtil] S, then + P U : lanes 64-127 -> O        (64 cols)
constexpr uint32_t TM_U = 128;    // [T;P] R : lanes 0-63 U                               (64 cols)
constexpr uint32_t TM_D = 192;    // Ktil^T U                                             (64 cols)
constexpr uint32_t TM_KT = 256;   // A operand Ktil_hi^T: lane i, column s                (64 cols)
constexpr uint32_t TM_KL = 320;   // A operand Ktil_lo^T                                  (64 cols)
constexpr uint32_t TM_TP = 384;   // A operand [T; P]: lane t (P at 64 + t), column s     (64 cols)
constexpr uint32_t TM_COLS = 512;

enum { BAR_QKV = 0, BAR_A, BAR_B, BAR_W, BAR_MMA, NBARS };

constexpr uint32_t TX_QKV = 16384 + 16384 + 8192;
constexpr uint32_t TX_A = 4 * 8192;
constexpr uint32_t TX_B = 4 * 8192;
constexpr uint32_t TX_W = 2 * 8192;

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
__device__ __forceinline__ float2 &at2(const Ctx &c, uint32_t off) { return *reinterpret_cast<float2 *>(c.sm + off); }
__device__ __forceinline__ float4 &at4(const Ctx &c, uint32_t off) { return *reinterpret_cast<float4 *>(c.sm + off); }

// Swizzled offsets of one fixed 4-byte column position in a tile with 128-byte
// rows: element (row, byte cb) is at row*128 + sw[row % 8].  Indexing sw[] with
// a compile-time row keeps the XOR out of the inner loops.
struct Swz {
    uint32_t o[8];
    __device__ __forceinline__ explicit Swz(uint32_t cb) {
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = ((((cb >> 4) ^ k) & 7u) << 4) | (cb & 15u);
    }
};

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
// Gate prep.  Thread (lane quarter qd, token quarter cq, lane l) owns key
// channel i = 32 qd + l for tokens [16 cq, 16 cq + 16).  Cumulative decay is a
// running FP32 product (exp of the cumulative log-decay up to rounding).
// Padding tokens (t >= n) have zero q, k, b from the TMA bounds fill and alpha
// forced to 1.  All loads of the 16 tokens precede the in-place stores.
__device__ __forceinline__ void prep(const Ctx &c, uint32_t tlane, int qd, int cq, int lane, int n) {
    const int i = 32 * qd + lane;
    const Swz sw((i & 31) * 4u);
    const uint32_t rbase = (i >> 5) * 16384u + cq * 16 * 128;   // atom of channel i, first row of the quarter
    float *part = fptr(c, OFF_PART);
    float av[16], bv[16], kv[16], qv[16];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
        const uint32_t o = rbase + tt * 128 + sw.o[tt & 7];
        av[tt] = at(c, OFF_KS + o);
        bv[tt] = at(c, OFF_X1 + o);
        const int t = 16 * cq + tt;
        kv[tt] = ldbf(c.sm + OFF_RK + t * 256 + i * 2);
        qv[tt] = ldbf(c.sm + OFF_RQ + t * 256 + i * 2);
    }
    float pa = 1.f;
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
        av[tt] = (16 * cq + tt < n) ? clamp_alpha(av[tt]) : 1.f;
        pa *= av[tt];
    }
    part[cq * 128 + i] = pa;
    __syncthreads();
    float g = 1.f, tot = 1.f;
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
        const float p = part[q2 * 128 + i];
        g = (q2 < cq) ? g * p : g;
        tot *= p;
    }
    if (cq == 0) fptr(c, OFF_GN)[i] = tot;
    float r = 1.f / g;
    float kh[16], kl[16];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
        g *= av[tt];
        r *= __fdividef(1.f, av[tt]);
        const uint32_t o = rbase + tt * 128 + sw.o[tt & 7];
        at(c, OFF_X1 + o) = to_tf32(bv[tt] * kv[tt] * g);
        at(c, OFF_X1 + o + 64 * 128) = to_tf32(qv[tt] * g);      // Qtil: rows 64-127, same swizzle phase
        const float kf = kv[tt] * r;
        kh[tt] = to_tf32(kf);
        kl[tt] = to_tf32(kf - kh[tt]);
        at(c, OFF_KS + o) = kh[tt];
    }
    tmem_st16(tlane + TM_KT + 16 * cq, kh);
    tmem_st16(tlane + TM_KL + 16 * cq, kl);
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1} in FP32, A strictly lower 64 x 64 given transposed (AT[s][t]).
// 16 x 16 diagonal blocks D_b by forward substitution; then T_10 = -D_1 A_10 D_0,
// T_32 = -D_3 A_32 D_2; then the lower-left 32 x 32 block T_BA = -T_BB A_BA T_AA.
// Result in Ts (row-major, zero above the diagonal).
__device__ __forceinline__ void invert(const Ctx &c, int tid) {
    const float *AT = fptr(c, OFF_AT);
    float *Ts = fptr(c, OFF_TS);
    float *Xs = fptr(c, OFF_XS);
    if (tid < 64) {
        const int b = tid >> 4, j = tid & 15, base = 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
            for (int l = 0; l < i; ++l) acc = fmaf(-AT[(base + l) * LDT + base + i], x[l], acc);
            x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Ts[(base + i) * LDT + base + j] = x[i];
    } else {
        // zero the blocks above the diagonal: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
        for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
            const int blk = e >> 8, i = (e >> 4) & 15, j = e & 15;
            const int a = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int b = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            Ts[(16 * a + i) * LDT + 16 * b + j] = 0.f;
        }
    }
    __syncthreads();
    {   // X = A_{a,a-1} D_{a-1} for a = 1, 3 (one output per thread)
        const int blk = tid >> 8, i = (tid >> 4) & 15, j = tid & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(AT[(16 * b + l) * LDT + 16 * a + i], Ts[(16 * b + l) * LDT + 16 * b + j], acc);
        Xs[blk * 16 * LDX + i * LDX + j] = acc;
    }
    __syncthreads();
    {   // T_{a,a-1} = -D_a X
        const int blk = tid >> 8, i = (tid >> 4) & 15, j = tid & 15;
        const int a = blk ? 3 : 1, b = a - 1;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(Ts[(16 * a + i) * LDT + 16 * a + l], Xs[blk * 16 * LDX + l * LDX + j], acc);
        Ts[(16 * a + i) * LDT + 16 * b + j] = -acc;
    }
    __syncthreads();
    // Y = A_BA T_AA (32 x 32): 256 threads, 2 x 2 outputs each
    if (tid < 256) {
        const int i = 2 * (tid >> 4), j = 2 * (tid & 15);
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {
            const float2 a = *reinterpret_cast<const float2 *>(AT + l * LDT + 32 + i);   // A[32+i][l], A[33+i][l]
            const float2 t = *reinterpret_cast<const float2 *>(Ts + l * LDT + j);         // T[l][j], T[l][j+1]
            y00 = fmaf(a.x, t.x, y00); y01 = fmaf(a.x, t.y, y01);
            y10 = fmaf(a.y, t.x, y10); y11 = fmaf(a.y, t.y, y11);
        }
        *reinterpret_cast<float2 *>(Xs + i * LDX + j) = make_float2(y00, y01);
        *reinterpret_cast<float2 *>(Xs + (i + 1) * LDX + j) = make_float2(y10, y11);
    }
    __syncthreads();
    // T_BA = -T_BB Y
    if (tid < 256) {
        const int i = 2 * (tid >> 4), j = 2 * (tid & 15);
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {
            const float a0 = Ts[(32 + i) * LDT + 32 + l], a1 = Ts[(33 + i) * LDT + 32 + l];
            const float2 y = *reinterpret_cast<const float2 *>(Xs + l * LDX + j);
            y00 = fmaf(a0, y.x, y00); y01 = fmaf(a0, y.y, y01);
            y10 = fmaf(a1, y.x, y10); y11 = fmaf(a1, y.y, y11);
        }
        *reinterpret_cast<float2 *>(Ts + (32 + i) * LDT + j) = make_float2(-y00, -y01);
        *reinterpret_cast<float2 *>(Ts + (33 + i) * LDT + j) = make_float2(-y10, -y11);
    }
    __syncthreads();
}

// Split x into TF32 hi + lo parts and store both into the [j][t] tiles UH / UL
// at token t (this thread's TMEM lane), columns 16 cq .. 16 cq + 15.
__device__ __forceinline__ void store_split_jt(const Ctx &c, const float (&x)[16], int t, int cq) {
    const Swz sw((t & 31) * 4u);
    const uint32_t base = (t >> 5) * 8192u + cq * 16 * 128;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint32_t o = base + j * 128 + sw.o[j & 7];
        const float hi = to_tf32(x[j]);
        at(c, OFF_UH + o) = hi;
        at(c, OFF_UL + o) = to_tf32(x[j] - hi);
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
    const int qd = warp & 3, cq = warp >> 2;            // TMEM lane quarter, 16-column quarter
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
    // col0 + 16 cq + [0, 16).  FP32 in registers across all chunks; its TF32
    // copy is KS rows 64 + j (j = local column), channel i.
    const Swz ssw((srow & 31) * 4u);
    const uint32_t sbase = OFF_KS + (srow >> 5) * 16384u + (64 + 16 * cq) * 128;
    float S[16];
    {
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 16 * cq;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + off + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) at(c, sbase + j * 128 + ssw.o[j & 7]) = to_tf32(S[j]);
    }

    // Shared-memory descriptors (start address advanced per K step).
    const uint64_t dX1 = sdesc_sw128(c.sa + OFF_X1, 16, 1024), dKS = sdesc_sw128(c.sa + OFF_KS, 16, 1024);
    const uint64_t dUH = sdesc_sw128(c.sa + OFF_UH, 16, 1024), dUL = sdesc_sw128(c.sa + OFF_UL, 16, 1024);

    uint32_t mma_phase = 0;
    bool ok = true;
    // One lane polls the mbarrier; the other warps wait at the CTA barrier, which
    // costs them no issue slots.  The barrier also publishes the TMA-written data.
    auto wait_all = [&](int which, uint32_t parity) {
        if (tid == 0 && !mbar_wait(c.bar[which], parity, kWaitLimit)) {
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
        prep(c, tlane, qd, cq, lane, n);
        sync_for_mma();
        // ---- [Etil; Qtil] x [Ktil; S^T]^T -> TM_G (Gram) and TM_X (Etil S, Qtil S)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 128, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const uint32_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                mma_tf32(tmem + TM_G, dX1 + koff, dKS + koff, id, kk > 0);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait() && wait_all(BAR_W, ph))) break;
        if (tid == 0 && more) {     // X1 and the Ktil rows of KS are consumed: next b and alpha
            load_alpha(c, maps, h, t0 + kC, bidx);
            load_b(c, maps, h, t0 + kC, bidx);
        }
        {
            float g[16];
            tmem_ld16(tlane + TM_G + 16 * cq, g);
            if (srow < 64) {        // A row (strictly lower, transposed into AT) and R = w*v - Etil S
                float *AT = fptr(c, OFF_AT);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int s = 16 * cq + j;
                    AT[s * LDT + srow] = (s < srow) ? g[j] : 0.f;
                }
                float x[16];
                tmem_ld16(tlane + TM_X + 16 * cq, x);
                const int ch = (16 * cq) >> 2;          // first 16-byte chunk of this quarter's columns
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int cc = ch + m;              // chunk among the 16 of a row (two 8-chunk atoms)
                    const uint32_t zo = (cc >> 3) * 8192u + srow * 128 + ((((cc & 7) ^ (srow & 7))) << 4);
                    const float4 w = at4(c, OFF_ZW + zo);
                    const uint2 vb = *reinterpret_cast<const uint2 *>(c.sm + OFF_RV + srow * 128 + (4 * cc) * 2);
                    const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.x));
                    const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.y));
                    x[4 * m] = w.x * v01.x - x[4 * m];
                    x[4 * m + 1] = w.y * v01.y - x[4 * m + 1];
                    x[4 * m + 2] = w.z * v23.x - x[4 * m + 2];
                    x[4 * m + 3] = w.w * v23.y - x[4 * m + 3];
                }
                store_split_jt(c, x, srow, cq);
            } else {                // P row (lower incl. diagonal) -> A operand in TMEM
                const int t = srow - 64;
#pragma unroll
                for (int j = 0; j < 16; ++j) g[j] = (16 * cq + j <= t) ? to_tf32(g[j]) : 0.f;
                tmem_st16(tlane + TM_TP + 16 * cq, g);
            }
        }
        __syncthreads();
        if (tid == 0 && more) load_w(c, maps, h, t0 + kC, bidx, col0);   // w consumed
        invert(c, tid);
        if (srow < 64) {            // T rows -> A operand in TMEM
            float tv[16];
            const float *Ts = fptr(c, OFF_TS);
#pragma unroll
            for (int j = 0; j < 16; ++j) tv[j] = to_tf32(Ts[srow * LDT + 16 * cq + j]);
            tmem_st16(tlane + TM_TP + 16 * cq, tv);
        }
        sync_for_mma();
        // ---- U = [T; P] (R_hi + R_lo) -> TM_U (lanes 0-63)
        if (tid == 0) {
            if (more) load_qkv(c, maps, h, t0 + kC, bidx, col0);         // inversion scratch free
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                mma_tf32_ts(tmem + TM_U, tmem + TM_TP + 8 * kk, dUH + koff, id, kk > 0);
                mma_tf32_ts(tmem + TM_U, tmem + TM_TP + 8 * kk, dUL + koff, id, 1);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        if (srow < 64) {            // U -> U_hi, U_lo
            float u[16];
            tmem_ld16(tlane + TM_U + 16 * cq, u);
            store_split_jt(c, u, srow, cq);
        }
        sync_for_mma();
        // ---- Ktil^T U -> TM_D (split);  P U_hi accumulated onto TM_X (lanes 64-127 become O)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, dUH + koff, id, kk > 0);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KT + 8 * kk, dUL + koff, id, 1);
                mma_tf32_ts(tmem + TM_D, tmem + TM_KL + 8 * kk, dUH + koff, id, 1);
                mma_tf32_ts(tmem + TM_X, tmem + TM_TP + 8 * kk, dUH + koff, id, 1);
            }
            mma_commit(c.bar[BAR_MMA]);
        }
        if (!(ok = mma_wait())) break;
        {   // state: S <- gamma_n (S + Ktil^T U); TF32 operand copy for the next chunk
            float d[16];
            tmem_ld16(tlane + TM_D + 16 * cq, d);
            const float gn = fptr(c, OFF_GN)[srow];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                S[j] = gn * (S[j] + d[j]);
                at(c, sbase + j * 128 + ssw.o[j & 7]) = to_tf32(S[j]);
            }
        }
        if (srow >= 64) {           // outputs from lanes 64-127 of TM_X
            float v[16];
            tmem_ld16(tlane + TM_X + 16 * cq, v);
            const int t = srow - 64;
            if (t < n) {
                __nv_bfloat16 *dst = o + (((size_t)bidx * T + t0 + t) * H + h) * 128 + col0 + 16 * cq;
#pragma unroll
                for (int j = 0; j < 16; j += 8) {
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
        const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 16 * cq;
#pragma unroll
        for (int j = 0; j < 16; j += 4)
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
