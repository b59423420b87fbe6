// Chunkwise prefill of the Gated DeltaNet-2 recurrence on the sm_100a tensor
// cores (tcgen05, TF32 operands, FP32 accumulation in Tensor Memory).
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Token processing and parallel training": the
// sequence is cut into blocks of up to 64 tokens; the per-channel decay
// accumulated since the block start is folded into the erase-side and key-side
// factors, so each block costs one unit-triangular system plus matrix
// products; decay, state and the triangular system are carried in FP32.  Per
// chunk of n tokens from state S:
//
//   gamma_t = prod_{j<=t} alpha_j                                (per key channel, FP32)
//   Etil = b*k*gamma,  Qtil = q*gamma,  Ktil = k / gamma          (gate prep)
//   [A; P] = [Etil; Qtil] Ktil^T                                  (Gram, tensor core)
//   T = (I + strict_tril(A))^{-1}                                 (FP32 blocked inversion)
//   [Etil S; Qtil S]                                              (tensor core)
//   R = w*v - Etil S                                              (FP32 epilogue)
//   U = T R                                                       (tensor core)
//   O = Qtil S + tril(P) U                                        (tensor core, accumulated)
//   S <- diag(gamma_n) (S + Ktil^T U)                             (tensor core + FP32 epilogue)
//
// U holds the per-token corrections z_t - r_t of the token recurrence, so this
// is the token loop's arithmetic, re-associated.
//
// Chunk length.  Ktil = k / gamma grows inside a chunk as the decay deepens.
// A chunk is therefore cut short, to n <= 64 tokens, where the decay
// accumulated since its first token would fall below 2^-64 in some key
// channel; the next chunk starts at the cut.  Every factor then stays within
// [2^-64, 2^64] of its input, for every alpha in (0, 1] (values of alpha below
// 2^-64 are taken as 2^-64, which changes a decayed state row by less than
// 2^-64 of its size).  On ordinary gates (a few to some tens of nats of decay
// per 64 tokens) no chunk is cut; a chunk of one token is always exact.
//
// Precision: tensor-core operands are TF32 (10-bit mantissa); accumulation,
// decay, R, T and the carried state are FP32.  R and U enter their products as
// split operands, x = x_hi + x_lo with both parts TF32, which keeps the carried
// state within a few 1e-3 of its RMS over 16K tokens.
//
// Organisation: one CTA per (sequence, head, 64-column half of d_v), 17 warps
// in three roles that run concurrently and hand work over through mbarriers:
//   warp 0      MMA issuer: the warp decides, one elected lane issues every
//               tcgen05 instruction, in whichever order their inputs become ready
//   warps 1-8   key side, one chunk ahead of the state side.  alpha, b, q, k
//               arrive by TMA in 128-byte-swizzled tiles; a thread per key
//               channel forms the decay products and the chunk length and
//               turns the tiles in place into Qtil and Etil (the A operand
//               [Etil; Qtil] of the Gram and X products, read from shared
//               memory) and writes Ktil (the Gram's B operand); while the Gram
//               runs, Ktil^T goes into Tensor Memory (the state update's A
//               operand, two buffers); Gram epilogue; the whole inversion
//               T = (I + A)^{-1}
//   warps 9-16  state side: R epilogue (w, v straight from global memory into
//               registers), U, state and output epilogues; once X has read the
//               chunk's [Etil; Qtil] it issues the next chunk's alpha, b load
// The state chain of a chunk is X -> R -> U -> state update; everything that
// does not depend on the state (gate prep, Gram, T) is done one chunk ahead.
// The FP32 state lives in Tensor Memory: the state-update MMA accumulates
// Ktil^T U onto it, the epilogue scales it by the chunk decay and writes the
// TF32 copy that the next chunk's X product reads.
//
// Logits variant (kLogits): every input arrives as BF16 pre-activation logits.
// alpha and b land as BF16 tiles in the first half of AT and BT; the decay pass
// reads every raw alpha and b value before it writes any tile, forms the FP32
// gates (alpha = exp(-softplus(x)) = 1 / (1 + e^x), b = sigmoid(x)) in
// registers, and applies SiLU and the L2 norm over each token's 128 channels (a
// warp holds whole token rows) to q and k in FP32 as it reads them.  The state
// side forms z = sigmoid(x_w) silu(x_v) from BF16 loads.  The rest of the kernel
// is unchanged.
#include <cudaTypedefs.h>
#include <stdio.h>

#include <atomic>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn2 {

__device__ unsigned int g_device_error = 0;  // nonzero: a bounded wait in a kernel gave up

namespace tc {

using namespace sm100;

constexpr int kC = 64;            // longest chunk (tokens)
constexpr int kDK = 128;          // key channels
constexpr int kDV = 128;          // value channels of a head
constexpr int kDVS = 64;          // value columns per CTA
constexpr int kThreads = 544;     // 17 warps
constexpr int kGroup = 256;       // threads in each of the two compute groups
constexpr uint32_t kBarK = 1, kBarS = 2;        // named hardware barriers of the groups
constexpr float kGammaMin = 5.42101086e-20f;   // 2^-64: floor of the decay spanned by one chunk
constexpr long long kDrainLimit = 4000000000ll; // ~2 s: end-of-kernel waits for in-flight MMAs

// Shared-memory map (bytes from a 1024-aligned base).  Tiles hold 64 rows of
// 128 swizzled bytes per block (8 KB):
//   AT  alpha[t][i] as TMA delivers it (4 channel blocks of FP32), turned in
//       place into Qtil (TF32)
//   BT  b[t][i], turned in place into Etil (TF32)
//   QT  q[t][i], KT  k[t][i] (BF16, 2 blocks of 64 channels each)
//   KG  Ktil[s][i] (TF32, 4 channel blocks): B operand of the Gram (K-major)
//   SC  S[i][j] as [j][i] (TF32, 4 channel blocks): B operand of the X product
//   UH  R_hi, later U_hi, as [j][t] (2 token blocks);  UL  R_lo, later U_lo
//   AS  A, then T in place (FP32 [64][68]);  XS block products (FP32 [32][36])
constexpr uint32_t TILE = 8192;
constexpr uint32_t OFF_EQS = 0;     // Etil / b and Qtil / alpha blocks interleaved: E0 Q0 E1 Q1 E2 Q2 E3 Q3
__host__ __device__ constexpr uint32_t OFF_E(int blk) { return OFF_EQS + 2u * blk * TILE; }
__host__ __device__ constexpr uint32_t OFF_Q(int blk) { return OFF_EQS + (2u * blk + 1u) * TILE; }
constexpr uint32_t OFF_QT = OFF_EQS + 8 * TILE;
constexpr uint32_t OFF_KT = OFF_QT + 2 * TILE;
constexpr uint32_t OFF_KG = OFF_KT + 2 * TILE;
constexpr uint32_t OFF_SC = OFF_KG + 4 * TILE;
constexpr uint32_t OFF_UH = OFF_SC + 4 * TILE;
constexpr uint32_t OFF_UL = OFF_UH + 2 * TILE;
constexpr int LDA = 68, LDX = 36;   // padded row strides (float4-aligned)
constexpr uint32_t OFF_AS = OFF_UL + 2 * TILE;
constexpr uint32_t OFF_XS = OFF_AS + 64 * LDA * 4;
// Per-chunk record handed from the key side to the issuer and the state side.
struct ChunkRec {
    int t0, n, last, pad;
    float gn[kDK];                // decay over the chunk, per key channel
};
constexpr int kRecSlots = 4;
constexpr uint32_t OFF_REC = OFF_XS + 32 * LDX * 4;
constexpr uint32_t OFF_PART = OFF_REC + kRecSlots * sizeof(ChunkRec);   // float[8][128]
constexpr uint32_t OFF_BAR = OFF_PART + 4096;                            // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 256;   // [0] tmem base, [1] abort flag, [2] first cut
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;      // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert(OFF_REC % 16 == 0 && sizeof(ChunkRec) % 16 == 0, "record alignment");
constexpr uint32_t TX_AB = 8 * TILE;                   // alpha and b of one chunk
constexpr uint32_t TX_AB_LOGITS = 4 * TILE;            // their BF16 logits
constexpr uint32_t TX_QK = 4 * TILE;                   // q and k of one chunk

// Tensor Memory columns (512 allocated).
constexpr uint32_t TM_X = 0;        // [Etil;Qtil] S, then + P U: lanes 64-127 -> O                     (64 cols)
constexpr uint32_t TM_U = 64;       // U = T R (lanes 0-63)                                             (64 cols)
constexpr uint32_t TM_S = 128;      // FP32 state S[i][j], lane i, column j                             (64 cols)
constexpr uint32_t TM_TP = 192;     // 2 buffers: the Gram [A; P], then the A operand [T; P]            (2 x 64 cols)
constexpr uint32_t TM_KH = 320;     // 2 buffers: A operand Ktil^T, lane i, column s                    (2 x 64 cols)
constexpr uint32_t TM_COLS = 512;

enum {
    B_G_FULL = 0, B_S_READY, B_X_FULL, B_R_READY, B_TP_READY0, B_TP_READY1, B_U_FULL, B_U_READY,
    B_D_FULL, B_O_FULL, B_KH_READY0, B_KH_READY1, B_KH_FREE0, B_KH_FREE1, B_TP_FREE0, B_TP_FREE1, B_RR0, B_RR1,
    B_RR2, B_RR3,
    B_FULL_AB, B_FULL_QK, B_DRAIN, B_GRAM_GO, NBARS
};
static_assert(NBARS * 8 <= 256, "barrier area");

// Flat token index space: token t of sequence s is row (tok * H + h) of every
// per-token tensor, tok = s * T + t (fixed length) or the packed index (varlen).
struct Maps {
    CUtensorMap q, k, v, alpha, b, w;    // 3-D {channel, head, token}, used for L2 prefetch
};
struct Params {
    const __nv_bfloat16 *q, *k, *v;
    const void *alpha, *b, *w;    // float gates, or BF16 logits in the logits variant
    const float *S0;
    __nv_bfloat16 *o;
    float *S_T;
    const int *cu_seqlens;    // nullptr: nseq sequences of T tokens; else packed offsets [nseq + 1]
    const int4 *ranges;       // else (non-null): sequence i is tokens [x, y) of the flat axis, and z != 0 makes
                              // its written values zero (the state's transition over the range alone)
    int nst;                  // sequences with an index below this write S_T
    int T, H;
    long long wait_limit;     // SM cycles before a pipeline wait gives up
};

struct Ctx {
    uint8_t *sm;          // 1024-aligned shared base (generic pointer)
    uint32_t sa;          // same, shared-window address
    volatile uint32_t *abort_flag;
    long long limit;
    __device__ __forceinline__ uint32_t bar(int i) const { return sa + OFF_BAR + 8 * i; }
};

__device__ __forceinline__ float *fptr(const Ctx &c, uint32_t off) { return reinterpret_cast<float *>(c.sm + off); }
__device__ __forceinline__ float &at(const Ctx &c, uint32_t off) { return *reinterpret_cast<float *>(c.sm + off); }
__device__ __forceinline__ ChunkRec &rec(const Ctx &c, int ck) {
    return reinterpret_cast<ChunkRec *>(c.sm + OFF_REC)[ck & (kRecSlots - 1)];
}

// Swizzled offsets of one fixed 4-byte column position in a tile with 128-byte
// rows: element (row, byte cb) is at row*128 + o[row % 8].
struct Swz {
    uint32_t o[8];
    __device__ __forceinline__ explicit Swz(uint32_t cb) {
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = ((((cb >> 4) ^ k) & 7u) << 4) | (cb & 15u);
    }
};

__device__ __forceinline__ void record_abort(const Ctx &c, int which) {
    *c.abort_flag = 1;
    atomicExch(&g_device_error, 1u + (unsigned)which);
}
// A wait whose outcome is uniform across a compute group: one thread polls the
// mbarrier (bounded), and the group's barrier ORs the failure over all of it.
__device__ __forceinline__ bool group_wait(const Ctx &c, int which, uint32_t parity, bool elected, uint32_t bar_id) {
    bool fail = false;
    if (elected) {
        if (*c.abort_flag) fail = true;
        else if (!mbar_wait(c.bar(which), parity, c.limit)) { record_abort(c, which); fail = true; }
    }
    return !named_bar_or(bar_id, kGroup, fail);
}
// Bounded wait for a single thread (the MMA issuer).
__device__ __forceinline__ bool solo_wait(const Ctx &c, int which, uint32_t parity) {
    if (*c.abort_flag) return false;
    if (!mbar_wait(c.bar(which), parity, c.limit)) {
        record_abort(c, which);
        return false;
    }
    return true;
}

__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// Key side, pass A: thread (cg, tg) owns key channels 4 cg .. 4 cg + 3 of
// tokens 8 tg .. 8 tg + 7 (a warp covers one group of 8 tokens, a lane four
// channels, so every access is one 16-byte piece of a swizzled row).  Decay
// products from the alpha tile, the chunk length, then in place alpha -> Qtil
// and b -> Etil, and Ktil into KG.  Tokens past the chunk become padding (no
// decay, zero rows).  Returns the chunk length n (uniform across the group).
template <bool kLogits>
__device__ __forceinline__ int key_decay(const Ctx &c, int ktid, int t0, int navail, int te, ChunkRec &r, bool el) {
    const int cg = ktid & 31, tg = ktid >> 5, lane = ktid & 31;
    const int tl0 = 8 * tg;
    float p[8][4];
    uint2 braw[kLogits ? 8 : 1];     // logits: b's raw BF16 values, read before any tile is rewritten
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        float4 a;
        if constexpr (kLogits) {     // alpha = exp(-softplus(x)) = 1 / (1 + e^x) from the BF16 logit
            const uint32_t s16 = swz128(tl0 + u, (cg & 15) * 8);
            const uint2 ar = *reinterpret_cast<const uint2 *>(c.sm + OFF_Q(cg >> 4) + s16);
            braw[u] = *reinterpret_cast<const uint2 *>(c.sm + OFF_E(cg >> 4) + s16);
            a = make_float4(sigmoid_fast(-bf_lo(ar.x)), sigmoid_fast(-bf_hi(ar.x)), sigmoid_fast(-bf_lo(ar.y)),
                            sigmoid_fast(-bf_hi(ar.y)));
        } else {
            a = *reinterpret_cast<const float4 *>(c.sm + OFF_Q(cg >> 3) + swz128(tl0 + u, (cg & 7) * 16));
        }
        const bool v = tl0 + u < navail;
        p[u][0] = v ? fmaxf(a.x, kGammaMin) : 1.f;
        p[u][1] = v ? fmaxf(a.y, kGammaMin) : 1.f;
        p[u][2] = v ? fmaxf(a.z, kGammaMin) : 1.f;
        p[u][3] = v ? fmaxf(a.w, kGammaMin) : 1.f;
    }
#pragma unroll
    for (int u = 1; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) p[u][e] *= p[u - 1][e];
    float *part = fptr(c, OFF_PART);                // [token group][channel]: product over the group
    int *nfirst = reinterpret_cast<int *>(c.sm + OFF_MISC + 8);
    *reinterpret_cast<float4 *>(part + tg * kDK + 4 * cg) = make_float4(p[7][0], p[7][1], p[7][2], p[7][3]);
    named_bar(kBarK, kGroup);
    float carry[4] = {1.f, 1.f, 1.f, 1.f};
    for (int g = 0; g < tg; ++g) {
        const float4 q4 = *reinterpret_cast<const float4 *>(part + g * kDK + 4 * cg);
        carry[0] *= q4.x; carry[1] *= q4.y; carry[2] *= q4.z; carry[3] *= q4.w;
    }
    // first token whose decay since the chunk start is below the floor in any of the four channels
    int first = 8;
#pragma unroll
    for (int u = 7; u >= 0; --u)
        if (fminf(fminf(carry[0] * p[u][0], carry[1] * p[u][1]), fminf(carry[2] * p[u][2], carry[3] * p[u][3])) < kGammaMin)
            first = u;
    int cut = first < 8 ? tl0 + first : kC;
    cut = __reduce_min_sync(0xffffffffu, cut);
    if (lane == 0 && cut < kC) atomicMin(nfirst, cut);
    named_bar(kBarK, kGroup);
    const int n = min(navail, *nfirst);
    if (n < navail) {
        // Cut chunk: tokens from n on belong to the next chunk (no decay here).
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (tl0 + u >= n)
#pragma unroll
                for (int e = 0; e < 4; ++e) p[u][e] = u ? p[u - 1][e] : 1.f;
        *reinterpret_cast<float4 *>(part + tg * kDK + 4 * cg) = make_float4(p[7][0], p[7][1], p[7][2], p[7][3]);
        named_bar(kBarK, kGroup);
#pragma unroll
        for (int e = 0; e < 4; ++e) carry[e] = 1.f;
        for (int g = 0; g < tg; ++g) {
            const float4 q4 = *reinterpret_cast<const float4 *>(part + g * kDK + 4 * cg);
            carry[0] *= q4.x; carry[1] *= q4.y; carry[2] *= q4.z; carry[3] *= q4.w;
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int t = tl0 + u;
        const uint32_t s32 = swz128(t, (cg & 7) * 16);
        const uint32_t o16 = (cg >> 4) * TILE + swz128(t, (cg & 15) * 8);
        const bool valid = t < n;
        const uint2 kr = valid ? *reinterpret_cast<const uint2 *>(c.sm + OFF_KT + o16) : make_uint2(0u, 0u);
        const uint2 qr = valid ? *reinterpret_cast<const uint2 *>(c.sm + OFF_QT + o16) : make_uint2(0u, 0u);
        float4 b4;
        if constexpr (kLogits)
            b4 = make_float4(sigmoid_fast(bf_lo(braw[u].x)), sigmoid_fast(bf_hi(braw[u].x)),
                             sigmoid_fast(bf_lo(braw[u].y)), sigmoid_fast(bf_hi(braw[u].y)));
        else
            b4 = *reinterpret_cast<const float4 *>(c.sm + OFF_E(cg >> 3) + s32);
        float kk[4] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y)};
        float qq[4] = {bf_lo(qr.x), bf_hi(qr.x), bf_lo(qr.y), bf_hi(qr.y)};
        if constexpr (kLogits) {     // q, k = silu(x) / ||silu(x)||, in FP32 from the raw logits;
            float sk = 0.f, sq = 0.f; // the warp holds token t's 128 channels
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kk[e] *= sigmoid_fast(kk[e]);
                qq[e] *= sigmoid_fast(qq[e]);
                sk = fmaf(kk[e], kk[e], sk);
                sq = fmaf(qq[e], qq[e], sq);
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, m);
                sq += __shfl_xor_sync(0xffffffffu, sq, m);
            }
            const float ik = sk > 0.f ? rsqrtf(sk) : 0.f, iq = sq > 0.f ? rsqrtf(sq) : 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kk[e] *= ik;
                qq[e] *= iq;
            }
        }
        const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
        float e4[4], q4[4], k4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float g = carry[e] * p[u][e];
            e4[e] = to_tf32(bb[e] * kk[e] * g);
            q4[e] = to_tf32(qq[e] * g);
            k4[e] = to_tf32(__fdividef(kk[e], g));
        }
        *reinterpret_cast<float4 *>(c.sm + OFF_E(cg >> 3) + s32) = make_float4(e4[0], e4[1], e4[2], e4[3]);
        *reinterpret_cast<float4 *>(c.sm + OFF_Q(cg >> 3) + s32) = make_float4(q4[0], q4[1], q4[2], q4[3]);
        *reinterpret_cast<float4 *>(c.sm + OFF_KG + (cg >> 3) * TILE + s32) = make_float4(k4[0], k4[1], k4[2], k4[3]);
    }
    if (tg == 7)
        *reinterpret_cast<float4 *>(r.gn + 4 * cg) =
            make_float4(carry[0] * p[7][0], carry[1] * p[7][1], carry[2] * p[7][2], carry[3] * p[7][3]);
    if (el) {
        r.t0 = t0;
        r.n = n;
        r.last = (t0 + n >= te) ? 1 : 0;
    }
    return n;
}



// Key side: Ktil^T of the chunk from KG into Tensor Memory (thread per key
// channel i and token half, lane i), the A operand of the state update.
__device__ __forceinline__ void key_kt(const Ctx &c, uint32_t tmem, int warp, int lane, int buf) {
    const int cb = warp & 3, hh = (warp - 1) >> 2;
    const int i = 32 * cb + lane;
    const Swz sw((i & 31) * 4u);
    const uint32_t fb = OFF_KG + (uint32_t)cb * TILE + hh * 32 * 128;
    float x[32];
#pragma unroll
    for (int tt = 0; tt < 32; ++tt) x[tt] = at(c, fb + tt * 128 + sw.o[tt & 7]);
    tmem_st32_nowait(tmem + TM_KH + 64 * buf + ((uint32_t)(32 * cb) << 16) + 32 * hh, x);
}

// The chunk's alpha and b tiles (or q and k) by TMA.
// FP32 gates: four 32-channel blocks each.  Logits: two 64-channel BF16 blocks each,
// at the start of the same regions (the decay pass reads them as logits).
template <bool kLogits>
__device__ __forceinline__ void load_ab(const Ctx &c, const Maps &m, int h, int t0) {
    const uint32_t fb = c.bar(B_FULL_AB);
    mbar_expect_tx(fb, kLogits ? TX_AB_LOGITS : TX_AB);
    for (int a = 0; a < (kLogits ? 2 : 4); ++a) {
        const int x = kLogits ? 64 * a : 32 * a;
        tma_load_3d(c.sa + OFF_Q(a), &m.alpha, x, h, t0, fb);
        tma_load_3d(c.sa + OFF_E(a), &m.b, x, h, t0, fb);
    }
}
__device__ __forceinline__ void load_qk(const Ctx &c, const Maps &m, int h, int t0) {
    const uint32_t fb = c.bar(B_FULL_QK);
    mbar_expect_tx(fb, TX_QK);
    for (int a = 0; a < 2; ++a) {
        tma_load_3d(c.sa + OFF_QT + a * TILE, &m.q, 64 * a, h, t0, fb);
        tma_load_3d(c.sa + OFF_KT + a * TILE, &m.k, 64 * a, h, t0, fb);
    }
}

// T = (I + A)^{-1} in FP32, in place in AS, by the 256 key-side threads (A is
// strictly lower and AS holds exact zeros on and above its diagonal).  Three
// levels: the four 16 x 16 diagonal blocks by forward substitution (column j of
// a block per thread, each step's dependency one FMA); then the 16 x 16 blocks
// below them, T_10 = -T_11 A_10 T_00, in both 32 x 32 halves; then the 32 x 32
// block T_BA = -T_BB A_BA T_AA.  Products keep a 1 x 4 or 2 x 4 block of outputs
// per thread in registers (half the group; the other half's warps share the
// sub-partitions with the state side's epilogues).
__device__ __forceinline__ void invert_t(const Ctx &c, int ktid, uint32_t bar_id) {
    float *As = fptr(c, OFF_AS);
    float *Xs = fptr(c, OFF_XS);
    if (ktid < 64) {                                         // 16 x 16 diagonal blocks
        const int base = 16 * (ktid >> 4), j = ktid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < 15; ++l) {
            const float xl = x[l];
#pragma unroll
            for (int i = l + 1; i < 16; ++i) x[i] = fmaf(-As[(base + i) * LDA + base + l], xl, x[i]);
        }
        __syncwarp();                                        // the warp's blocks are read before written
#pragma unroll
        for (int i = 0; i < 16; ++i) As[(base + i) * LDA + base + j] = x[i];
    }
    named_bar(bar_id, kGroup);
    if (ktid < 128) {                                        // Y = A_10 T_00 in both halves (16 x 16 x 16)
        const int base = 32 * (ktid >> 6), r = (ktid & 63) >> 2, cq = 4 * (ktid & 3);
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = As[(base + 16 + r) * LDA + base + k];
            const float4 t = *reinterpret_cast<const float4 *>(As + (base + k) * LDA + base + cq);
            y.x = fmaf(a, t.x, y.x); y.y = fmaf(a, t.y, y.y); y.z = fmaf(a, t.z, y.z); y.w = fmaf(a, t.w, y.w);
        }
        *reinterpret_cast<float4 *>(Xs + (ktid >> 6) * 16 * LDX + r * LDX + cq) = y;
    }
    named_bar(bar_id, kGroup);
    if (ktid < 128) {                                        // T_10 = -T_11 Y
        const int base = 32 * (ktid >> 6), r = (ktid & 63) >> 2, cq = 4 * (ktid & 3);
        const float *Y = Xs + (ktid >> 6) * 16 * LDX;
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = As[(base + 16 + r) * LDA + base + 16 + k];
            const float4 y = *reinterpret_cast<const float4 *>(Y + k * LDX + cq);
            z.x = fmaf(a, y.x, z.x); z.y = fmaf(a, y.y, z.y); z.z = fmaf(a, y.z, z.z); z.w = fmaf(a, y.w, z.w);
        }
        *reinterpret_cast<float4 *>(As + (base + 16 + r) * LDA + base + cq) = make_float4(-z.x, -z.y, -z.z, -z.w);
    }
    named_bar(bar_id, kGroup);
    const int ri = 2 * (ktid >> 3), ci = 4 * (ktid & 7);     // rows ri, ri + 1; columns ci .. ci + 3
    if (ktid < 128) {                                        // Y = A_BA T_AA (32 x 32 x 32)
        float4 y0 = make_float4(0.f, 0.f, 0.f, 0.f), y1 = y0;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a0 = As[(32 + ri) * LDA + k], a1 = As[(33 + ri) * LDA + k];
            const float4 t = *reinterpret_cast<const float4 *>(As + k * LDA + ci);
            y0.x = fmaf(a0, t.x, y0.x); y0.y = fmaf(a0, t.y, y0.y); y0.z = fmaf(a0, t.z, y0.z); y0.w = fmaf(a0, t.w, y0.w);
            y1.x = fmaf(a1, t.x, y1.x); y1.y = fmaf(a1, t.y, y1.y); y1.z = fmaf(a1, t.z, y1.z); y1.w = fmaf(a1, t.w, y1.w);
        }
        *reinterpret_cast<float4 *>(Xs + ri * LDX + ci) = y0;
        *reinterpret_cast<float4 *>(Xs + (ri + 1) * LDX + ci) = y1;
    }
    named_bar(bar_id, kGroup);
    if (ktid < 128) {                                        // T_BA = -T_BB Y
        float4 z0 = make_float4(0.f, 0.f, 0.f, 0.f), z1 = z0;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a0 = As[(32 + ri) * LDA + 32 + k], a1 = As[(33 + ri) * LDA + 32 + k];
            const float4 y = *reinterpret_cast<const float4 *>(Xs + k * LDX + ci);
            z0.x = fmaf(a0, y.x, z0.x); z0.y = fmaf(a0, y.y, z0.y); z0.z = fmaf(a0, y.z, z0.z); z0.w = fmaf(a0, y.w, z0.w);
            z1.x = fmaf(a1, y.x, z1.x); z1.y = fmaf(a1, y.y, z1.y); z1.z = fmaf(a1, y.z, z1.z); z1.w = fmaf(a1, y.w, z1.w);
        }
        *reinterpret_cast<float4 *>(As + (32 + ri) * LDA + ci) = make_float4(-z0.x, -z0.y, -z0.z, -z0.w);
        *reinterpret_cast<float4 *>(As + (33 + ri) * LDA + ci) = make_float4(-z1.x, -z1.y, -z1.z, -z1.w);
    }
    named_bar(bar_id, kGroup);
}

// Split 32 values into TF32 hi + lo parts and store both into the [j][t] tiles
// UH / UL at token t, columns 32 sh .. 32 sh + 31.  hi keeps the top 10
// mantissa bits (a TF32 value exactly), lo = x - hi is exact in FP32 and below
// one TF32 unit of x; the tensor core reads lo to TF32 by dropping its low
// bits, so hi + lo carries x to within 2^-20 of |x|.
__device__ __forceinline__ void store_split_jt(const Ctx &c, const float (&x)[32], int t, int sh) {
    const Swz sw((t & 31) * 4u);
    const uint32_t base = (t >> 5) * TILE + sh * 32 * 128;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t o = base + j * 128 + sw.o[j & 7];
        const float hi = __uint_as_float(__float_as_uint(x[j]) & 0xFFFFE000u);
        at(c, OFF_UH + o) = hi;
        at(c, OFF_UL + o) = x[j] - hi;
    }
}

// Descriptor offset (16-byte units) of K-step kk (8 TF32 = 32 bytes) in a
// K-major tile of 64-row blocks: 4 K-steps per 128-byte row, then the next block.
__device__ __forceinline__ uint32_t kstep(int kk) { return ((kk >> 2) * TILE + (kk & 3) * 32) >> 4; }
// The same for the 128-row A operand [Etil; Qtil]: its channel blocks are E/Q tile pairs (2 tiles apart).
__device__ __forceinline__ uint32_t eq_step(int kk) { return ((kk >> 2) * 2 * TILE + (kk & 3) * 32) >> 4; }

// A bounded mbarrier test whose outcome is the same in every lane of the warp
// (a phase, once complete, stays complete, so any lane's yes is everyone's).
__device__ __forceinline__ bool warp_test(const Ctx &c, int which, uint32_t parity) {
    return __any_sync(0xffffffffu, mbar_test(c.bar(which), parity));
}

// The MMA issuer (warp 0).  Four streams of work, each in chunk order: the Gram
// of chunk cg, the X product of chunk cx, U of chunk cu, the state update and
// output of chunk cs.  Whichever has its inputs ready is issued, the state
// chain first.  The whole warp runs the loop and takes every decision by vote,
// so that descriptors and counters stay warp-uniform; one elected lane (always
// the same, the lowest) issues the tcgen05 instructions.  A separate function
// keeps its few live values out of the other roles' register allocation.
__device__ __noinline__ void issuer_role(const Ctx &c, uint32_t tmem) {
    // B descriptors as (low, high) halves; the K-step offset is added inside each MMA's asm.
    const uint64_t dSC = sdesc_sw128(c.sa + OFF_SC, 16, 1024), dKG = sdesc_sw128(c.sa + OFF_KG, 16, 1024);
    // [Etil; Qtil] in shared memory: rows 0-63 from an E block, rows 64-127 from the Q block after it
    const uint32_t eq = (uint32_t)sdesc_sw128(c.sa + OFF_EQS, 16, 1024);
    const uint64_t dUH = sdesc_sw128(c.sa + OFF_UH, 16, 1024), dUL = sdesc_sw128(c.sa + OFF_UL, 16, 1024);
    const uint32_t hi = (uint32_t)(dSC >> 32);      // identical for every tile (layout, SBO, version)
    const uint32_t sc = (uint32_t)dSC, kg = (uint32_t)dKG, uh = (uint32_t)dUH, ul = (uint32_t)dUL;
    const uint32_t id = idesc_tf32(128, 64, 0, 0);
    const bool lane0 = (threadIdx.x & 31) == 0;
    int cg = 0, cx = 0, cu = 0, cs = 0, lastc = 0x7fffffff;
    long long t_prog = clock64();
    while (cs <= lastc) {
        if (cs < cu && warp_test(c, B_U_READY, cs & 1) &&
            warp_test(c, (cs & 1) ? B_KH_READY1 : B_KH_READY0, (cs >> 1) & 1)) {
            // S + Ktil^T (U_hi + U_lo) onto the state;  P U_hi onto TM_X (-> O)
            const uint32_t tp = tmem + TM_TP + 64 * (cs & 1), kh = tmem + TM_KH + 64 * (cs & 1);
            if (elect_one_sync()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_tf32_ts_off(tmem + TM_S, kh + 8 * kk, uh, hi, kstep(kk), id, 1);
                    mma_tf32_ts_off(tmem + TM_S, kh + 8 * kk, ul, hi, kstep(kk), id, 1);
                }
                mma_commit(c.bar(B_D_FULL));
                mma_commit(c.bar((cs & 1) ? B_KH_FREE1 : B_KH_FREE0));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) mma_tf32_ts_off(tmem + TM_X, tp + 8 * kk, uh, hi, kstep(kk), id, 1);
                mma_commit(c.bar(B_O_FULL));
                mma_commit(c.bar((cs & 1) ? B_TP_FREE1 : B_TP_FREE0));
            }
            __syncwarp();
            ++cs;
        } else if (cu < cx && warp_test(c, B_R_READY, cu & 1) &&
                   warp_test(c, (cu & 1) ? B_TP_READY1 : B_TP_READY0, (cu >> 1) & 1)) {
            // U = [T; P] (R_hi + R_lo)
            const uint32_t tp = tmem + TM_TP + 64 * (cu & 1);
            if (elect_one_sync()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_tf32_ts_off(tmem + TM_U, tp + 8 * kk, uh, hi, kstep(kk), id, kk > 0);
                    mma_tf32_ts_off(tmem + TM_U, tp + 8 * kk, ul, hi, kstep(kk), id, 1);
                }
                mma_commit(c.bar(B_U_FULL));
            }
            __syncwarp();
            ++cu;
        } else if (cx < cg && warp_test(c, B_S_READY, cx & 1)) {
            // [Etil; Qtil] S, A from the shared-memory tiles (the Gram of the chunk found them ready)
            if (elect_one_sync()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    mma_tf32_ss_off(tmem + TM_X, eq, eq_step(kk), sc, kstep(kk), hi, id, kk > 0);
                mma_commit(c.bar(B_X_FULL));
            }
            __syncwarp();
            ++cx;
        } else if (cg <= lastc && warp_test(c, B_GRAM_GO, cg & 1) &&
                   (cg < 2 || warp_test(c, (cg & 1) ? B_TP_FREE1 : B_TP_FREE0, ((cg - 2) >> 1) & 1))) {
            // Gram [Etil; Qtil] Ktil^T into the chunk's [T; P] buffer
            if (__any_sync(0xffffffffu, rec(c, cg).last != 0)) lastc = cg;
            const uint32_t tp = tmem + TM_TP + 64 * (cg & 1);
            if (elect_one_sync()) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) mma_tf32_ss_off(tp, eq, eq_step(kk), kg, kstep(kk), hi, id, kk > 0);
                mma_commit(c.bar(B_G_FULL));
            }
            __syncwarp();
            ++cg;
        } else {
            if (__any_sync(0xffffffffu, *c.abort_flag != 0)) break;
            if (__any_sync(0xffffffffu, clock64() - t_prog > c.limit)) {
                if (lane0) record_abort(c, B_DRAIN);
                break;
            }
            continue;
        }
        t_prog = clock64();
    }
    // Every MMA issued above has completed before Tensor Memory is released (bounded).
    if (elect_one_sync()) mma_commit(c.bar(B_DRAIN));
    __syncwarp();
    (void)mbar_wait(c.bar(B_DRAIN), 0, kDrainLimit);
}

// ---------------------------------------------------------------------------
template <bool kLogits>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    // Align by offsetting the __shared__ array itself (not through an integer
    // cast) so that the compiler keeps every access in the shared window.
    c.sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    c.sa = smem_u32(c.sm);
    uint32_t *misc = reinterpret_cast<uint32_t *>(c.sm + OFF_MISC);
    c.abort_flag = misc + 1;
    c.limit = p.wait_limit;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x >> 1, half = blockIdx.x & 1;   // unit = sequence * H + head
    const int seq = unit / p.H, h = unit % p.H;
    int tb, te;
    bool zero_z = false;
    if (p.ranges) {             // explicit token ranges, clamped to the T tokens there are
        const int4 rg = p.ranges[seq];
        tb = min(max(rg.x, 0), p.T);
        te = min(max(rg.y, tb), p.T);
        zero_z = rg.z != 0;
    } else if (p.cu_seqlens) {  // packed offsets, clamped to the T tokens there are
        tb = min(max(p.cu_seqlens[seq], 0), p.T);
        te = min(max(p.cu_seqlens[seq + 1], tb), p.T);
    } else {
        tb = seq * p.T;
        te = tb + p.T;
    }
    const bool empty = te <= tb;
    const int col0 = half * kDVS;
    const size_t soff = (size_t)unit * kDK * kDV;

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
        // ------------------------------------------------ MMA issuer
        if (!empty) issuer_role(c, tmem);
        __syncwarp();
    } else if (warp <= 8) {
        // ------------------------------------------------ key side
        const int ktid = tid - 32;
        const bool el = ktid == 0;
        const int lq = warp & 3, ch = (warp - 1) >> 2;
        const int srow = 32 * lq + lane;                       // TMEM lane in the epilogues
        const uint32_t tlane = tmem + ((uint32_t)(32 * lq) << 16);
        int t0 = tb;
        if (el && !empty) {
            load_ab<kLogits>(c, maps, h, t0);
            load_qk(c, maps, h, t0);
        }
        int pend_ab = empty ? -1 : 0, pend_qk = pend_ab;   // chunk whose loads are in flight, not yet awaited
        for (int ck = 0; !empty; ++ck) {
            const uint32_t ph = ck & 1;
            const int navail = min(kC, te - t0);
            ChunkRec &r = rec(c, ck);
            if (!group_wait(c, B_FULL_AB, ph, el, kBarK)) break;
            pend_ab = -1;
            if (!group_wait(c, B_FULL_QK, ph, el, kBarK)) break;
            pend_qk = -1;
            if (el) {
                *reinterpret_cast<volatile int *>(c.sm + OFF_MISC + 8) = kC;
                const int tn = t0 + kC;
                if (tn < te) {      // the next chunk's w, v (state side) and alpha, b (its TMA load) into L2
                    for (int a = 0; a < (kLogits ? 1 : 2); ++a) tma_prefetch_3d(&maps.w, col0 + 32 * a, h, tn);
                    tma_prefetch_3d(&maps.v, col0, h, tn);
                    for (int a = 0; a < (kLogits ? 2 : 4); ++a) {
                        tma_prefetch_3d(&maps.alpha, kLogits ? 64 * a : 32 * a, h, tn);
                        tma_prefetch_3d(&maps.b, kLogits ? 64 * a : 32 * a, h, tn);
                    }
                }
            }
            const int n = key_decay<kLogits>(c, ktid, t0, navail, te, r, el);
            const bool last = t0 + n >= te;
            fence_proxy_async_smem();
            named_bar(kBarK, kGroup);
            if (el) {
                mbar_arrive(c.bar(B_RR0 + (ck & 3)));
                mbar_arrive(c.bar(B_GRAM_GO));         // the Gram reads [Etil; Qtil] from shared memory
                if (!last) {
                    load_qk(c, maps, h, t0 + n);       // q, k consumed: the next chunk's
                    pend_qk = ck + 1;
                }
            }
            // While the Gram runs: Ktil^T into Tensor Memory (buffer ck & 1) once the state
            // update two chunks back has read that buffer
            if (ck >= 2 && !group_wait(c, ph ? B_KH_FREE1 : B_KH_FREE0, ((ck - 2) >> 1) & 1, el, kBarK)) break;
            tc_fence_after();
            key_kt(c, tmem, warp, lane, ph);
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarK, kGroup);
            if (el) mbar_arrive(c.bar(ph ? B_KH_READY1 : B_KH_READY0));
            // Gram epilogue: A (rows 0-63, strictly lower) -> AS; P (rows 64-127) masked in place.
            if (!group_wait(c, B_G_FULL, ph, el, kBarK)) break;
            tc_fence_after();
            {
                const uint32_t tp = tlane + TM_TP + 64 * ph + 32 * ch;
                float g[32];
                tmem_ld32(tp, g);
                if (srow < 64) {      // A strictly lower; exact zeros on and above the diagonal
                    float4 *dst = reinterpret_cast<float4 *>(fptr(c, OFF_AS) + srow * LDA + 32 * ch);
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 4) {
                        const int s0 = 32 * ch + jj;
                        dst[jj >> 2] = make_float4(s0 < srow ? g[jj] : 0.f, s0 + 1 < srow ? g[jj + 1] : 0.f,
                                                   s0 + 2 < srow ? g[jj + 2] : 0.f, s0 + 3 < srow ? g[jj + 3] : 0.f);
                    }
                } else {
                    const int t = srow - 64;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) g[jj] = (32 * ch + jj <= t) ? to_tf32(g[jj]) : 0.f;
                    tmem_st32_nowait(tp, g);
                }
            }
            named_bar(kBarK, kGroup);
            invert_t(c, ktid, kBarK);
            if (srow < 64) {        // AS holds exact zeros above the diagonal of T (TF32 copy)
                float tv[32];
                const float *As = fptr(c, OFF_AS) + srow * LDA + 32 * ch;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) tv[jj] = to_tf32(As[jj]);
                tmem_st32_nowait(tlane + TM_TP + 64 * ph + 32 * ch, tv);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarK, kGroup);
            if (el) mbar_arrive(c.bar(ph ? B_TP_READY1 : B_TP_READY0));
            if (last) break;
            t0 += n;
        }
        // No copy into shared memory may still be in flight when the CTA ends (bounded).
        if (el && pend_ab >= 0) (void)mbar_wait(c.bar(B_FULL_AB), pend_ab & 1, kDrainLimit);
        if (el && pend_qk >= 0) (void)mbar_wait(c.bar(B_FULL_QK), pend_qk & 1, kDrainLimit);
    } else {
        // ------------------------------------------------ state side
        const int stid = tid - 288, lq = warp & 3, sh = (warp - 9) >> 2;
        const int srow = 32 * lq + lane;
        const uint32_t tlane = tmem + ((uint32_t)(32 * lq) << 16);
        const uint32_t ts = tlane + TM_S + 32 * sh;        // this thread's state row, 32 columns
        const bool el = stid == 0;
        const Swz ssw((srow & 31) * 4u);
        const uint32_t sbase = OFF_SC + (srow >> 5) * TILE + 32 * sh * 128;   // S[i][j] at [j][i]
        const size_t srow_off = soff + (size_t)srow * kDV + col0 + 32 * sh;
        const bool write_st = p.S_T != nullptr && seq < p.nst;
        if (empty) {
            if (write_st) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 x = p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + srow_off + j)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(p.S_T + srow_off + j) = x;
                }
            }
        } else {
            {   // S0 -> Tensor Memory and its TF32 copy
                float S[32];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 x = p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + srow_off + j)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
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
            int pend_ab = -1;      // chunk whose alpha, b load this side issued, not yet known to be complete
            for (int ck = 0;; ++ck) {
                const uint32_t ph = ck & 1;
                if (!group_wait(c, B_RR0 + (ck & 3), (ck >> 2) & 1, el, kBarS)) { done_ok = false; break; }
                const ChunkRec &r = rec(c, ck);
                const int t0 = r.t0, n = r.n;
                const bool last = r.last != 0;
                // w, v of this thread's token (lanes 0-63) and columns, straight into registers;
                // the loads complete while the MMA below runs.  Tokens past the chunk read as zero.
                float z[32];
                if (srow < 64) {
                    if (srow < n && !zero_z) {
                        const size_t row = ((size_t)(t0 + srow) * p.H + h) * kDV + col0 + 32 * sh;
                        const uint4 *vp = reinterpret_cast<const uint4 *>(p.v + row);
                        if constexpr (kLogits) {      // z = sigmoid(xw) silu(xv)
                            const uint4 *wp = reinterpret_cast<const uint4 *>(
                                static_cast<const __nv_bfloat16 *>(p.w) + row);
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const uint4 vb = __ldg(vp + m), wb = __ldg(wp + m);
                                const float vv[8] = {bf_lo(vb.x), bf_hi(vb.x), bf_lo(vb.y), bf_hi(vb.y),
                                                     bf_lo(vb.z), bf_hi(vb.z), bf_lo(vb.w), bf_hi(vb.w)};
                                const float ww[8] = {bf_lo(wb.x), bf_hi(wb.x), bf_lo(wb.y), bf_hi(wb.y),
                                                     bf_lo(wb.z), bf_hi(wb.z), bf_lo(wb.w), bf_hi(wb.w)};
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    z[8 * m + e] = sigmoid_fast(ww[e]) * vv[e] * sigmoid_fast(vv[e]);
                            }
                        } else {
                            const float4 *wp = reinterpret_cast<const float4 *>(
                                static_cast<const float *>(p.w) + row);
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const uint4 vb = __ldg(vp + m);
                                const float4 w0 = __ldg(wp + 2 * m), w1 = __ldg(wp + 2 * m + 1);
                                float *zp = z + 8 * m;
                                zp[0] = w0.x * bf_lo(vb.x); zp[1] = w0.y * bf_hi(vb.x);
                                zp[2] = w0.z * bf_lo(vb.y); zp[3] = w0.w * bf_hi(vb.y);
                                zp[4] = w1.x * bf_lo(vb.z); zp[5] = w1.y * bf_hi(vb.z);
                                zp[6] = w1.z * bf_lo(vb.w); zp[7] = w1.w * bf_hi(vb.w);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) z[j] = 0.f;
                    }
                }
                // R = w*v - Etil S (lanes 0-63) -> R_hi, R_lo
                if (!group_wait(c, B_X_FULL, ph, el, kBarS)) { done_ok = false; break; }
                if (el && !last) {     // the Gram and X have read Qtil and Etil: the next chunk's alpha, b over them
                    load_ab<kLogits>(c, maps, h, t0 + n);
                    pend_ab = ck + 1;
                }
                tc_fence_after();
                if (srow < 64) {
                    float x[32];
                    tmem_ld32(tlane + TM_X + 32 * sh, x);
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = z[j] - x[j];
                    store_split_jt(c, x, srow, sh);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(kBarS, kGroup);
                if (el) mbar_arrive(c.bar(B_R_READY));
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
                    const float gn = r.gn[srow];
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
                    if (t < n && p.o) {
                        __nv_bfloat16 *dst = p.o + ((size_t)(t0 + t) * p.H + h) * kDV + col0 + 32 * sh;
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
                if (last) break;
            }
            // No copy into shared memory may still be in flight when the CTA ends (bounded).
            if (el && pend_ab >= 0) (void)mbar_wait(c.bar(B_FULL_AB), pend_ab & 1, kDrainLimit);
            if (done_ok && *c.abort_flag == 0 && write_st) {
                float S[32];
                tmem_ld32(ts, S);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(p.S_T + srow_off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
        }
    }

    // Every role has finished or given up, and the MMA lane has seen its last MMA
    // complete: release Tensor Memory.
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
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
    if (!f) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
            fn.store(f);
        }
    }
    return f;
}

// Flat [NT][H][d] tensor; box = {box_d, 1, 64}, rows of 128 bytes swizzled as the MMA tiles are.
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, size_t es, long long NT, int H, int d,
              int box_d, bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)NT};
    cuuint64_t strides[2] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es};
    cuuint32_t box[3] = {(cuuint32_t)box_d, 1, (cuuint32_t)kC};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

std::atomic<long long> g_wait_limit{4000000000ll};
std::atomic<unsigned long long> g_attr_set{0};   // bit d: the shared-memory attribute is set on device d

}  // namespace tc

bool chunk_tc_supported(int dk, int dv, gdn2_dtype dt) { return dk == 128 && dv == 128 && dt == GDN2_BF16; }

void set_wait_limit(long long cycles) { tc::g_wait_limit.store(cycles); }

cudaError_t read_device_error(unsigned int *value, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

// nseq sequences: of T tokens each (cu_seqlens and ranges null), packed with
// device offsets cu_seqlens[0..nseq] into T_total = T tokens, or given as device
// token ranges ranges[0..nseq) of T_total = T tokens (z != 0: written values
// taken as zero).  o may be null (no output written); only sequences below nst
// (all, when nst < 0) write S_T.
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *alpha, const void *b,
                            const void *w, const float *S0, void *o, float *S_T, int nseq, int T, int H,
                            const int *cu_seqlens, bool logits, cudaStream_t stream, const int4 *ranges,
                            int nst) {
    using namespace tc;
    const bool packed = cu_seqlens != nullptr || ranges != nullptr;
    const long long NT = packed ? (long long)T : (long long)nseq * T;
    if (NT <= 0 && !packed) return cudaSuccess;
    Maps m;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const long long NTm = NT > 0 ? NT : 1;
    if (!make_map(&m.q, q, BF, 2, NTm, H, kDK, 64, true) || !make_map(&m.k, k, BF, 2, NTm, H, kDK, 64, true) ||
        !make_map(&m.v, v, BF, 2, NTm, H, kDV, 64, false) ||
        !make_map(&m.alpha, alpha, logits ? BF : F32, logits ? 2 : 4, NTm, H, kDK, logits ? 64 : 32, true) ||
        !make_map(&m.b, b, logits ? BF : F32, logits ? 2 : 4, NTm, H, kDK, logits ? 64 : 32, true) ||
        !make_map(&m.w, w, logits ? BF : F32, logits ? 2 : 4, NTm, H, kDV, logits ? 64 : 32, false))
        return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (!bit || !(g_attr_set.load() & bit)) {
        e = cudaFuncSetAttribute(chunk_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(chunk_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (bit) g_attr_set.fetch_or(bit);
    }
    Params prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.k = static_cast<const __nv_bfloat16 *>(k);
    prm.v = static_cast<const __nv_bfloat16 *>(v);
    prm.alpha = alpha;
    prm.b = b;
    prm.w = w;
    prm.S0 = S0;
    prm.o = static_cast<__nv_bfloat16 *>(o);
    prm.S_T = S_T;
    prm.cu_seqlens = cu_seqlens;
    prm.ranges = ranges;
    prm.nst = nst < 0 ? nseq : nst;
    prm.T = T;
    prm.H = H;
    prm.wait_limit = g_wait_limit.load();
    const unsigned grid = 2u * (unsigned)nseq * (unsigned)H;
    if (logits)
        chunk_tc_kernel<true><<<grid, kThreads, SMEM_BYTES, stream>>>(m, prm);
    else
        chunk_tc_kernel<false><<<grid, kThreads, SMEM_BYTES, stream>>>(m, prm);
    return cudaGetLastError();
}

}  // namespace gdn2
