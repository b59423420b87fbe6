// Chunkwise prefill of the Gated DeltaNet-2 recurrence on the sm_100a tensor
// cores (tcgen05, TF32 operands, FP32 accumulation in Tensor Memory).
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Token processing and parallel training": the
// sequence is cut into 64-token blocks; the per-channel decay accumulated since
// the block start is folded into the erase-side and key-side factors, so each
// block costs one unit-triangular system plus matrix products; decay, state and
// the triangular system are carried in FP32.  Per chunk of n tokens from state S:
//
//   gamma_t = prod_{j<=t} alpha_j,  rho_t = 1/gamma_t          (per key channel, FP32)
//   Etil = b*k*gamma,  Qtil = q*gamma,  Ktil = k*rho            (gate prep)
//   [A; P] = [Etil; Qtil] Ktil^T                                 (Gram, tensor core)
//   T = (I + strict_tril(A))^{-1}                                (FP32 blocked inversion)
//   [Etil S; Qtil S]                                             (tensor core)
//   R = w*v - Etil S                                             (FP32 epilogue)
//   U = T R                                                      (tensor core)
//   O = Qtil S + tril(P) U                                       (tensor core, accumulated)
//   S <- diag(gamma_n) (S + Ktil^T U)                            (tensor core + FP32 epilogue)
//
// U holds the per-token corrections z_t - r_t of the token recurrence, so this
// is the token loop's arithmetic, re-associated.
//
// Precision: tensor-core operands are TF32 (10-bit mantissa); accumulation,
// decay, R, T and the carried state are FP32.  R and U enter their products as
// split operands, x = x_hi + x_lo with both parts TF32 (T R = T R_hi + T R_lo,
// Ktil^T U = Ktil^T U_hi + Ktil^T U_lo), which keeps the carried state within
// ~0.3% of its RMS over 16K tokens (plain TF32 there: ~0.7%).  BF16 operands
// lose too much: the read r = Sbar^T e nearly cancels the write z in the delta
// rule.  The key factor Ktil = k / gamma grows within a chunk as
// exp(-sum ln alpha); it must stay below ~1e34 (sum of -ln alpha over one chunk
// <= 78 per key channel), as documented in gdn2.h.
//
// Organisation: one CTA per (batch, head, 64-column half of d_v), 18 warps in
// four roles that run concurrently and hand work over through mbarriers:
//   warp 0      TMA producer (alpha, b into their operand tiles; q, k into a
//               BF16 staging tile; L2 prefetch of the next chunk's tiles)
//   warp 1      MMA issuer (one thread, every tcgen05 instruction)
//   warps 2-9   key side: gate prep, Gram epilogue, the diagonal 32 x 32
//               blocks of T = (I + A)^{-1}
//   warps 10-17 state side: R epilogue (w, v read straight from global memory
//               into registers), the off-diagonal block of T and its copy into
//               Tensor Memory, U, state and output epilogues
// The key side of chunk c+1 runs while the state chain of chunk c runs; the
// key factor Ktil^T and [T; P] are double-buffered in Tensor Memory for that.
// The FP32 state itself lives in Tensor Memory: the state-update MMA
// accumulates Ktil^T U onto it, the epilogue scales it by the chunk decay and
// writes the TF32 copy that the next chunk's MMAs read.
// Shared-memory MMA operands are K-major with the 128-byte swizzle; operands
// needed transposed (Ktil^T, [T; P]) are read from Tensor Memory as operand A.
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
constexpr int kThreads = 576;     // 18 warps
constexpr int kGroup = 256;       // threads in each of the two compute groups
constexpr uint32_t kBarK = 1, kBarS = 2;   // named hardware barriers of the groups
constexpr long long kWaitLimit = 4000000000ll;   // ~2 s of SM cycles per wait

// Shared-memory map (bytes from a 1024-aligned base).  MMA tiles hold TF32,
// 32 elements per 128-byte swizzled row, K-major:
//   X1  rows 0-63 Etil[t][i], rows 64-127 Qtil[t][i]         4 atoms x 16 KB (i = key channel)
//   KS  rows 0-63 Ktil[s][i], rows 64-127 S[i][j] as [j][i]    4 atoms x 16 KB
//   UH  R_hi, later U_hi, as [j][t]                           2 atoms x 8 KB (t = token)
//   UL  R_lo, later U_lo, as [j][t]                           2 atoms x 8 KB
//   QK  q, k as BF16 [a][t][32] (a = channel block of 32), 16 KB each: TMA
//       destinations, read by the gate prep
//   AS  A, then T in place (FP32 [64][66]);  XS block products (FP32 [32][34])
constexpr uint32_t OFF_X1 = 0;
constexpr uint32_t OFF_KS = OFF_X1 + 65536;
constexpr uint32_t OFF_UH = OFF_KS + 65536;
constexpr uint32_t OFF_UL = OFF_UH + 16384;
constexpr uint32_t OFF_GN = OFF_UL + 16384;            // float[2][128] decay over the chunk (by buffer)
constexpr uint32_t OFF_PART = OFF_GN + 1024;           // float[2][128] half-chunk decay products
constexpr uint32_t OFF_BAR = OFF_PART + 1024;          // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 256;           // tmem base, abort flag
constexpr int LDA = 66, LDX = 34;
constexpr uint32_t OFF_QK = (OFF_MISC + 16 + 1023) / 1024 * 1024;
constexpr uint32_t OFF_AS = OFF_QK + 32768;
constexpr uint32_t OFF_XS = OFF_AS + 64 * LDA * 4;
constexpr uint32_t SMEM_USED = OFF_XS + 32 * LDX * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;      // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

// Tensor Memory columns (512 allocated).
constexpr uint32_t TM_G = 0;        // Gram: lanes 0-63 A, lanes 64-127 P                 (64 cols)
constexpr uint32_t TM_X = 64;       // [Etil;Qtil] S, then + P U: lanes 64-127 -> O       (64 cols)
constexpr uint32_t TM_U = 128;      // U = T R (lanes 0-63)                                (64 cols)
constexpr uint32_t TM_KT = 192;     // 2 buffers: A operand Ktil^T, lane i, column s      (2 x 64 cols)
constexpr uint32_t TM_TP = 320;     // 2 buffers: A operand [T; P], lane t, column s      (2 x 64 cols)
constexpr uint32_t TM_S = 448;      // FP32 state S[i][j], lane i, column j               (64 cols)
constexpr uint32_t TM_COLS = 512;

enum {
    B_FULL_AB = 0, B_FULL_QK, B_X1_FREE, B_KPREP, B_G_FULL, B_DIAG_DONE, B_TP_READY, B_S_READY,
    B_X_FULL, B_R_READY, B_U_FULL, B_U_READY, B_D_FULL, B_O_FULL, B_KT_FREE0, B_KT_FREE1, B_DRAIN, NBARS
};

constexpr uint32_t TX_AB = 8 * 8192;
constexpr uint32_t TX_QK = 8 * 4096;

struct Maps {
    CUtensorMap q, k, v, alpha, b, w;
};

struct Ctx {
    uint8_t *sm;          // 1024-aligned shared base (generic pointer)
    uint32_t sa;          // same, shared-window address
    volatile uint32_t *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return sa + OFF_BAR + 8 * i; }
};

__device__ __forceinline__ float *fptr(const Ctx &c, uint32_t off) { return reinterpret_cast<float *>(c.sm + off); }
__device__ __forceinline__ float &at(const Ctx &c, uint32_t off) { return *reinterpret_cast<float *>(c.sm + off); }
__device__ __forceinline__ float4 &at4(const Ctx &c, uint32_t off) { return *reinterpret_cast<float4 *>(c.sm + off); }

// Swizzled offsets of one fixed 4-byte column position in a tile with 128-byte
// rows: element (row, byte cb) is at row*128 + o[row % 8].
struct Swz {
    uint32_t o[8];
    __device__ __forceinline__ explicit Swz(uint32_t cb) {
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = ((((cb >> 4) ^ k) & 7u) << 4) | (cb & 15u);
    }
};

// A wait whose outcome is uniform across a compute group: one thread polls the
// mbarrier (bounded), the group meets at its named barrier, all read the flag.
__device__ __forceinline__ bool group_wait(const Ctx &c, int which, uint32_t parity, bool elected, uint32_t bar_id) {
    if (elected && *c.abort_flag == 0 && !mbar_wait(c.bar(which), parity, kWaitLimit)) {
        *c.abort_flag = 1;
        atomicExch(&g_device_error, 1u + (unsigned)which);
    }
    named_bar(bar_id, kGroup);
    return *c.abort_flag == 0;
}
// Bounded wait for a single thread (producer, MMA issuer).
__device__ __forceinline__ bool solo_wait(const Ctx &c, int which, uint32_t parity) {
    if (*c.abort_flag) return false;
    if (!mbar_wait(c.bar(which), parity, kWaitLimit)) {
        *c.abort_flag = 1;
        atomicExch(&g_device_error, 1u + (unsigned)which);
        return false;
    }
    return true;
}

// ---------------------------------------------------------------------------
// Key side.  Thread (lane quarter qd, half kh, lane l) owns key channel
// i = 32 qd + l for tokens [32 kh, 32 kh + 32) in the gate prep, and TMEM lane
// 32 qd + l, columns [32 kh, 32 kh + 32) in the Gram epilogue.
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// Gate prep: cumulative decay as running FP32 products (exp of the cumulative
// log-decay up to rounding); Etil, Qtil into X1, Ktil into KS (rows 0-63) and
// its transpose into Tensor Memory.  Padding tokens (t >= n): zero b from the
// TMA bounds fill, zero q, k, alpha forced to 1.  prep_decay forms each
// thread's product of alpha over its 32 tokens (needs only alpha).  kFull: the
// chunk has all 64 tokens, so no token needs the padding test.
template <bool kFull>
__device__ __forceinline__ void prep_decay(const Ctx &c, int qd, int kh, int lane, int n) {
    const int i = 32 * qd + lane;
    const Swz sw((i & 31) * 4u);
    const uint32_t rbase = (i >> 5) * 16384u + kh * 32 * 128;
    float pa = 1.f;
#pragma unroll
    for (int tt = 0; tt < 32; ++tt) {
        const float a = at(c, OFF_KS + rbase + tt * 128 + sw.o[tt & 7]);
        pa *= (kFull || 32 * kh + tt < n) ? clamp_alpha(a) : 1.f;
    }
    fptr(c, OFF_PART)[kh * 128 + i] = pa;
}

// Gate prep proper (after prep_decay and a group barrier).
template <bool kFull>
__device__ __forceinline__ void prep(const Ctx &c, uint32_t tlane, uint32_t kt_col, int kb, int qd, int kh,
                                     int lane, int n) {
    const int i = 32 * qd + lane;
    const Swz sw((i & 31) * 4u);
    const uint32_t rbase = (i >> 5) * 16384u + kh * 32 * 128;
    const float *part = fptr(c, OFF_PART);
    const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(c.sm + OFF_QK) + (i >> 5) * 2048 + kh * 1024 + (i & 31);
    const __nv_bfloat16 *ks = qs + 8192;
    const float p0 = part[i], p1 = part[128 + i];
    if (kh == 0) fptr(c, OFF_GN)[kb * 128 + i] = p0 * p1;
    float g = kh ? p0 : 1.f;
    float r = 1.f / g;
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
        float av[8], bv[8], kt[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t o = rbase + (8 * grp + u) * 128 + sw.o[u];
            av[u] = at(c, OFF_KS + o);
            bv[u] = at(c, OFF_X1 + o);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int tt = 8 * grp + u;
            const float a = (kFull || 32 * kh + tt < n) ? clamp_alpha(av[u]) : 1.f;
            g *= a;
            r *= __fdividef(1.f, a);
            const float qq = __bfloat162float(qs[tt * 32]), kk = __bfloat162float(ks[tt * 32]);
            const uint32_t o = rbase + tt * 128 + sw.o[u];
            at(c, OFF_X1 + o) = to_tf32(bv[u] * kk * g);
            at(c, OFF_X1 + o + 64 * 128) = to_tf32(qq * g);          // Qtil rows 64-127, same swizzle phase
            kt[u] = to_tf32(kk * r);
            at(c, OFF_KS + o) = kt[u];
        }
        tmem_st8_nowait(tlane + kt_col + 32 * kh + 8 * grp, kt);
    }
}

// T = (I + A)^{-1} in FP32, in place in AS (A strictly lower, zero above the
// diagonal), in two parts.  invert_diag (key side): the 32 x 32 diagonal
// blocks T_AA, T_BB by forward substitution (right-looking: column j of a block
// per thread, each step's dependency one FMA).  invert_offdiag (state side,
// which is otherwise waiting for T): T_BA = -T_BB A_BA T_AA.
__device__ __forceinline__ void invert_diag(const Ctx &c, int ktid) {
    float *As = fptr(c, OFF_AS);
    if (ktid < 64) {
        const int base = 32 * (ktid >> 5), j = ktid & 31;
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < 31; ++l) {
            const float xl = x[l];
#pragma unroll
            for (int i = l + 1; i < 32; ++i) x[i] = fmaf(-As[(base + i) * LDA + base + l], xl, x[i]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32; ++i) As[(base + i) * LDA + base + j] = x[i];
    }
}
// gtid: thread index within the 256-thread group that runs this; bar_id: its barrier.
__device__ __forceinline__ void invert_offdiag(const Ctx &c, int gtid, uint32_t bar_id) {
    float *As = fptr(c, OFF_AS);
    float *Xs = fptr(c, OFF_XS);
    // Y = A_BA T_AA (32 x 32), 2 x 2 outputs per thread
    {
        const int i = 2 * (gtid >> 4), jj = 2 * (gtid & 15);
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {
            const float a0 = As[(32 + i) * LDA + l], a1 = As[(33 + i) * LDA + l];
            const float2 t = *reinterpret_cast<const float2 *>(As + l * LDA + jj);
            y00 = fmaf(a0, t.x, y00); y01 = fmaf(a0, t.y, y01);
            y10 = fmaf(a1, t.x, y10); y11 = fmaf(a1, t.y, y11);
        }
        *reinterpret_cast<float2 *>(Xs + i * LDX + jj) = make_float2(y00, y01);
        *reinterpret_cast<float2 *>(Xs + (i + 1) * LDX + jj) = make_float2(y10, y11);
    }
    named_bar(bar_id, kGroup);
    // T_BA = -T_BB Y
    {
        const int i = 2 * (gtid >> 4), jj = 2 * (gtid & 15);
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {
            const float a0 = As[(32 + i) * LDA + 32 + l], a1 = As[(33 + i) * LDA + 32 + l];
            const float2 y = *reinterpret_cast<const float2 *>(Xs + l * LDX + jj);
            y00 = fmaf(a0, y.x, y00); y01 = fmaf(a0, y.y, y01);
            y10 = fmaf(a1, y.x, y10); y11 = fmaf(a1, y.y, y11);
        }
        *reinterpret_cast<float2 *>(As + (32 + i) * LDA + jj) = make_float2(-y00, -y01);
        *reinterpret_cast<float2 *>(As + (33 + i) * LDA + jj) = make_float2(-y10, -y11);
    }
    named_bar(bar_id, kGroup);
}

// Split 32 values into TF32 hi + lo parts and store both into the [j][t] tiles
// UH / UL at token t, columns 32 sh .. 32 sh + 31.  hi keeps the top 10
// mantissa bits (a TF32 value exactly), lo = x - hi is exact in FP32 and
// below one TF32 unit of x; the tensor core reads lo to TF32 by dropping its
// low bits, so hi + lo carries x to within 2^-20 of |x|.
__device__ __forceinline__ void store_split_jt(const Ctx &c, const float (&x)[32], int t, int sh) {
    const Swz sw((t & 31) * 4u);
    const uint32_t base = (t >> 5) * 8192u + sh * 32 * 128;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t o = base + j * 128 + sw.o[j & 7];
        const float hi = __uint_as_float(__float_as_uint(x[j]) & 0xFFFFE000u);
        at(c, OFF_UH + o) = hi;
        at(c, OFF_UL + o) = x[j] - hi;
    }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ Maps maps, const float *__restrict__ wg,
                const __nv_bfloat16 *__restrict__ vg, const float *S0, __nv_bfloat16 *__restrict__ o, float *S_T,
                int T, int H) {
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    // Align by offsetting the __shared__ array itself (not through an integer
    // cast) so that the compiler keeps every access in the shared window.
    c.sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    c.sa = smem_u32(c.sm);
    uint32_t *misc = reinterpret_cast<uint32_t *>(c.sm + OFF_MISC);
    c.abort_flag = misc + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x >> 1, half = blockIdx.x & 1;
    const int bidx = head / H, h = head % H;
    const int col0 = half * kDVS;
    const int nchunks = (T + kC - 1) / kC;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(c.bar(i), 1);
        fence_mbar_init();
        *c.abort_flag = 0;
        tma_prefetch_map(&maps.q); tma_prefetch_map(&maps.k);
        tma_prefetch_map(&maps.v); tma_prefetch_map(&maps.alpha);
        tma_prefetch_map(&maps.b); tma_prefetch_map(&maps.w);
    }
    if (warp == 0) {
        tmem_alloc(c.sa + OFF_MISC, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // Each lane finally waits (bounded) for the last copy it issued, so that no copy
        // into shared memory is still in flight when the CTA ends, also after a give-up.
        if (lane == 0) {            // alpha -> KS rows 0-63, b -> X1 rows 0-63
            int last = -1;
            for (int ck = 0; ck < nchunks; ++ck) {
                if (ck > 0 && !solo_wait(c, B_X1_FREE, (ck - 1) & 1)) break;
                const uint32_t fb = c.bar(B_FULL_AB);
                mbar_expect_tx(fb, TX_AB);
                last = ck;
                for (int a = 0; a < 4; ++a) {
                    tma_load_4d(c.sa + OFF_KS + a * 16384, &maps.alpha, 32 * a, h, ck * kC, bidx, fb);
                    tma_load_4d(c.sa + OFF_X1 + a * 16384, &maps.b, 32 * a, h, ck * kC, bidx, fb);
                }
                if (ck + 1 < nchunks) {     // the next chunk's tiles into L2 while this one is processed
                    for (int a = 0; a < 4; ++a) {
                        tma_prefetch_4d(&maps.alpha, 32 * a, h, (ck + 1) * kC, bidx);
                        tma_prefetch_4d(&maps.b, 32 * a, h, (ck + 1) * kC, bidx);
                    }
                    for (int a = 0; a < 2; ++a) tma_prefetch_4d(&maps.w, col0 + 32 * a, h, (ck + 1) * kC, bidx);
                    tma_prefetch_4d(&maps.v, col0, h, (ck + 1) * kC, bidx);
                }
            }
            if (last >= 0) (void)mbar_wait(c.bar(B_FULL_AB), last & 1, kWaitLimit / 8);
        } else if (lane == 1) {     // q, k -> QK once the gate prep has consumed the previous chunk's
            int last = -1;
            for (int ck = 0; ck < nchunks; ++ck) {
                if (ck > 0 && !solo_wait(c, B_KPREP, (ck - 1) & 1)) break;
                const uint32_t fb = c.bar(B_FULL_QK);
                mbar_expect_tx(fb, TX_QK);
                last = ck;
                for (int a = 0; a < 4; ++a) {
                    tma_load_4d(c.sa + OFF_QK + a * 4096, &maps.q, 32 * a, h, ck * kC, bidx, fb);
                    tma_load_4d(c.sa + OFF_QK + 16384 + a * 4096, &maps.k, 32 * a, h, ck * kC, bidx, fb);
                }
                if (ck + 1 < nchunks)
                    for (int a = 0; a < 4; ++a) {
                        tma_prefetch_4d(&maps.q, 32 * a, h, (ck + 1) * kC, bidx);
                        tma_prefetch_4d(&maps.k, 32 * a, h, (ck + 1) * kC, bidx);
                    }
            }
            if (last >= 0) (void)mbar_wait(c.bar(B_FULL_QK), last & 1, kWaitLimit / 8);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t dX1 = sdesc_sw128(c.sa + OFF_X1, 16, 1024);
            const uint64_t dKK = sdesc_sw128(c.sa + OFF_KS, 16, 1024);           // Ktil rows
            const uint64_t dKSt = sdesc_sw128(c.sa + OFF_KS + 8192, 16, 1024);   // S rows
            const uint64_t dUH = sdesc_sw128(c.sa + OFF_UH, 16, 1024), dUL = sdesc_sw128(c.sa + OFF_UL, 16, 1024);
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
            for (int ck = 0; ck < nchunks; ++ck) {
                const uint32_t ph = ck & 1;
                const uint32_t kt = tmem + TM_KT + 64 * ph, tp = tmem + TM_TP + 64 * ph;
                // Gram [Etil; Qtil] Ktil^T
                if (!solo_wait(c, B_KPREP, ph)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint32_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                    mma_tf32(tmem + TM_G, dX1 + koff, dKK + koff, id, kk > 0);
                }
                mma_commit(c.bar(B_G_FULL));
                // [Etil; Qtil] S
                if (!solo_wait(c, B_S_READY, ph)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint32_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                    mma_tf32(tmem + TM_X, dX1 + koff, dKSt + koff, id, kk > 0);
                }
                mma_commit(c.bar(B_X_FULL));
                mma_commit(c.bar(B_X1_FREE));
                // U = [T; P] (R_hi + R_lo)
                if (!solo_wait(c, B_R_READY, ph) || !solo_wait(c, B_TP_READY, ph)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                    mma_tf32_ts(tmem + TM_U, tp + 8 * kk, dUH + koff, id, kk > 0);
                    mma_tf32_ts(tmem + TM_U, tp + 8 * kk, dUL + koff, id, 1);
                }
                mma_commit(c.bar(B_U_FULL));
                // S + Ktil^T (U_hi + U_lo) accumulated onto the state;  then P U_hi onto TM_X
                if (!solo_wait(c, B_U_READY, ph)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                    mma_tf32_ts(tmem + TM_S, kt + 8 * kk, dUH + koff, id, 1);
                    mma_tf32_ts(tmem + TM_S, kt + 8 * kk, dUL + koff, id, 1);
                }
                mma_commit(c.bar(B_D_FULL));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                    mma_tf32_ts(tmem + TM_X, tp + 8 * kk, dUH + koff, id, 1);
                }
                mma_commit(c.bar(B_O_FULL));
                mma_commit(c.bar(ph ? B_KT_FREE1 : B_KT_FREE0));     // Ktil^T and [T; P] of this parity
            }
            // Every MMA issued above has completed before Tensor Memory is released (bounded).
            mma_commit(c.bar(B_DRAIN));
            (void)mbar_wait(c.bar(B_DRAIN), 0, kWaitLimit / 8);
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------ key side
        const int ktid = tid - 64, qd = warp & 3, kh = (warp - 2) >> 2;
        const int srow = 32 * qd + lane;
        const uint32_t tlane = tmem + ((uint32_t)(32 * qd) << 16);
        const bool el = ktid == 0;
        for (int ck = 0; ck < nchunks; ++ck) {
            const uint32_t ph = ck & 1;
            const int t0 = ck * kC, n = min(kC, T - t0);
            if (!group_wait(c, B_FULL_AB, ph, el, kBarK)) break;
            if (n == kC) prep_decay<true>(c, qd, kh, lane, n);
            else prep_decay<false>(c, qd, kh, lane, n);
            if (!group_wait(c, B_FULL_QK, ph, el, kBarK)) break;
            if (ck >= 2 && !group_wait(c, ph ? B_KT_FREE1 : B_KT_FREE0, ((ck - 2) >> 1) & 1, el, kBarK)) break;
            if (n == kC) prep<true>(c, tlane, TM_KT + 64 * ph, ph, qd, kh, lane, n);
            else prep<false>(c, tlane, TM_KT + 64 * ph, ph, qd, kh, lane, n);
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarK, kGroup);
            if (el) mbar_arrive(c.bar(B_KPREP));
            // Gram epilogue: A (rows 0-63, strictly lower) -> AS; P (rows 64-127) -> [T; P] operand.
            // AS is free once the state side has copied out the previous chunk's T.
            if (!group_wait(c, B_G_FULL, ph, el, kBarK)) break;
            if (ck >= 1 && !group_wait(c, B_TP_READY, (ck - 1) & 1, el, kBarK)) break;
            tc_fence_after();
            {
                float g[32];
                tmem_ld32(tlane + TM_G + 32 * kh, g);
                if (srow < 64) {
                    // The diagonal 32 x 32 blocks are only read strictly below their diagonal and are
                    // then overwritten by T_AA, T_BB; A_BA lies wholly below the diagonal.  Only the
                    // block above the diagonal (rows 0-31, columns 32-63) needs its zeros.
                    float2 *dst = reinterpret_cast<float2 *>(fptr(c, OFF_AS) + srow * LDA + 32 * kh);
                    const bool upper = srow < 32 && kh == 1;
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 2)
                        dst[jj >> 1] = upper ? make_float2(0.f, 0.f) : make_float2(g[jj], g[jj + 1]);
                } else {
                    const int t = srow - 64;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) g[jj] = (32 * kh + jj <= t) ? to_tf32(g[jj]) : 0.f;
                    tmem_st32_nowait(tlane + TM_TP + 64 * ph + 32 * kh, g);
                }
            }
            named_bar(kBarK, kGroup);
            invert_diag(c, ktid);
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarK, kGroup);
            if (el) mbar_arrive(c.bar(B_DIAG_DONE));
        }
    } else {
        // ------------------------------------------------ state side
        const int stid = tid - 320, qd = warp & 3, sh = (warp - 10) >> 2;
        const int srow = 32 * qd + lane;
        const uint32_t tlane = tmem + ((uint32_t)(32 * qd) << 16);
        const uint32_t ts = tlane + TM_S + 32 * sh;        // this thread's state row, 32 columns
        const bool el = stid == 0;
        const Swz ssw((srow & 31) * 4u);
        const uint32_t sbase = OFF_KS + (srow >> 5) * 16384u + (64 + 32 * sh) * 128;   // S rows of KS
        {   // S0 -> Tensor Memory and its TF32 copy
            float S[32];
            const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * sh;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                float4 x = S0 ? *reinterpret_cast<const float4 *>(S0 + off + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) at(c, sbase + j * 128 + ssw.o[j & 7]) = to_tf32(S[j]);
            tmem_st32_nowait(ts, S);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar(kBarS, kGroup);
        if (el) mbar_arrive(c.bar(B_S_READY));
        bool done_ok = true;
        for (int ck = 0; ck < nchunks; ++ck) {
            const uint32_t ph = ck & 1;
            const int t0 = ck * kC, n = min(kC, T - t0);
            // w, v of this thread's token (lanes 0-63) and columns, straight into registers;
            // the loads complete while the MMA below runs.  Padding tokens read as zero.
            float4 wr[8];
            uint4 vr[4];
            if (srow < 64) {
                if (srow < n) {
                    const size_t row = (((size_t)bidx * T + t0 + srow) * H + h) * 128 + col0 + 32 * sh;
                    const float4 *wp = reinterpret_cast<const float4 *>(wg + row);
                    const uint4 *vp = reinterpret_cast<const uint4 *>(vg + row);
#pragma unroll
                    for (int m = 0; m < 8; ++m) wr[m] = __ldg(wp + m);
#pragma unroll
                    for (int m = 0; m < 4; ++m) vr[m] = __ldg(vp + m);
                } else {
#pragma unroll
                    for (int m = 0; m < 8; ++m) wr[m] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int m = 0; m < 4; ++m) vr[m] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            // R = w*v - Etil S (lanes 0-63) -> R_hi, R_lo
            if (!group_wait(c, B_X_FULL, ph, el, kBarS)) { done_ok = false; break; }
            tc_fence_after();
            if (srow < 64) {
                float x[32];
                tmem_ld32(tlane + TM_X + 32 * sh, x);
#pragma unroll
                for (int p = 0; p < 4; ++p) {                  // columns 32 sh + 8 p .. + 7
                    const uint4 vb = vr[p];
                    const float4 w0 = wr[2 * p], w1 = wr[2 * p + 1];
                    float *xp = x + 8 * p;
                    xp[0] = w0.x * bf_lo(vb.x) - xp[0];
                    xp[1] = w0.y * bf_hi(vb.x) - xp[1];
                    xp[2] = w0.z * bf_lo(vb.y) - xp[2];
                    xp[3] = w0.w * bf_hi(vb.y) - xp[3];
                    xp[4] = w1.x * bf_lo(vb.z) - xp[4];
                    xp[5] = w1.y * bf_hi(vb.z) - xp[5];
                    xp[6] = w1.z * bf_lo(vb.w) - xp[6];
                    xp[7] = w1.w * bf_hi(vb.w) - xp[7];
                }
                store_split_jt(c, x, srow, sh);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarS, kGroup);
            if (el) mbar_arrive(c.bar(B_R_READY));
            // finish T = (I + A)^{-1} and copy it, TF32, into rows 0-63 of the [T; P] operand
            if (!group_wait(c, B_DIAG_DONE, ph, el, kBarS)) { done_ok = false; break; }
            tc_fence_after();
            invert_offdiag(c, stid, kBarS);
            if (srow < 64) {        // AS holds exact zeros above the diagonal of T
                float tv[32];
                const float *As = fptr(c, OFF_AS) + srow * LDA + 32 * sh;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) tv[jj] = to_tf32(As[jj]);
                tmem_st32_nowait(tlane + TM_TP + 64 * ph + 32 * sh, tv);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarS, kGroup);
            if (el) mbar_arrive(c.bar(B_TP_READY));
            // U -> U_hi, U_lo
            if (!group_wait(c, B_U_FULL, ph, el, kBarS)) { done_ok = false; break; }
            tc_fence_after();
            if (srow < 64) {
                float u[32];
                tmem_ld32(tlane + TM_U + 32 * sh, u);
                store_split_jt(c, u, srow, sh);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarS, kGroup);
            if (el) mbar_arrive(c.bar(B_U_READY));
            // state S <- gamma_n (S + Ktil^T U), in Tensor Memory, and its TF32 copy
            if (!group_wait(c, B_D_FULL, ph, el, kBarS)) { done_ok = false; break; }
            tc_fence_after();
            {
                float d[32];
                tmem_ld32(ts, d);
                const float gn = fptr(c, OFF_GN)[ph * 128 + srow];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    d[j] *= gn;
                    at(c, sbase + j * 128 + ssw.o[j & 7]) = to_tf32(d[j]);
                }
                tmem_st32_nowait(ts, d);
            }
            // outputs: lanes 64-127 of TM_X
            if (!group_wait(c, B_O_FULL, ph, el, kBarS)) { done_ok = false; break; }
            tc_fence_after();
            if (srow >= 64) {
                float v[32];
                tmem_ld32(tlane + TM_X + 32 * sh, v);
                const int t = srow - 64;
                if (t < n) {
                    __nv_bfloat16 *dst = o + (((size_t)bidx * T + t0 + t) * H + h) * 128 + col0 + 32 * sh;
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
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarS, kGroup);
            if (el) mbar_arrive(c.bar(B_S_READY));
        }
        if (done_ok && *c.abort_flag == 0 && S_T) {
            float S[32];
            tmem_ld32(ts, S);
            const size_t off = ((size_t)head * kDK + srow) * 128 + col0 + 32 * sh;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4 *>(S_T + off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }

    // Every role has finished or given up, and the producer and MMA lanes have seen
    // their last copy and MMA complete: release Tensor Memory.
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
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
    if (!make_map(&m.q, q, BF, 2, B, T, H, kDK, 32, false) || !make_map(&m.k, k, BF, 2, B, T, H, kDK, 32, false) ||
        !make_map(&m.v, v, BF, 2, B, T, H, 128, 64, true) ||
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
    chunk_tc_kernel<<<grid, kThreads, SMEM_BYTES, stream>>>(m, w, static_cast<const __nv_bfloat16 *>(v), S0,
                                                            static_cast<__nv_bfloat16 *>(o), S_T, T, H);
    return cudaGetLastError();
}

}  // namespace gdn2
