// Segment-parallel prefill for long sequences.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (iplexlaw.co.kr analysis), "Independent decisions on two axes": per token the
// state is decayed per key channel, the erase reads r = S^T e from it and the
// write adds k (z - r)^T, so
//   S_t = (I - k_t e_t^T) diag(alpha_t) S_{t-1} + k_t z_t^T,
// an affine map of the previous state.  Over a range of tokens therefore
//   S_end = M S_start + C,
// with C the end state from a zero start and M (d_k x d_k) the end state from
// S_start = I with every written value z taken as zero (the product of the
// tokens' transitions).  A sequence cut into P segments runs as
//   1. one launch of the chunkwise kernel over 2 (P - 1) independent token
//      ranges: segments 0 .. P-2 from a zero state (S_T -> C_s) and again with
//      z = 0 from the identity (S_T -> M_s); no outputs;
//   2. S_start(0) = S0 and S_start(s + 1) = M_s S_start(s) + C_s, in FP32, here;
//   3. one launch over all P segments from their start states: o, and S_T from
//      the last segment.
// About three times the sequential chunk work, over 4 (P - 1) + 2 P CTAs per
// (sequence, head) instead of 2: it pays when few (sequence, head) pairs are
// long ("What was compared": the fixed-size state carries the whole history, so
// a long sequence is otherwise one serial chain).
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kD = 128;                      // d_k = d_v on the tensor-core path
constexpr size_t kState = (size_t)kD * kD;   // floats of one (sequence, head) state
constexpr int kCols = 32;                    // value columns per combine CTA

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct SegLayout {
    size_t ranges_ab, ranges_d, wab, sd, total;
};
SegLayout seg_layout(int B, int H, int P) {
    SegLayout l;
    const size_t nab = 2 * (size_t)B * (P - 1), nd = (size_t)B * P;
    l.ranges_ab = 0;
    l.ranges_d = align256(nab * sizeof(int4));
    l.wab = l.ranges_d + align256(nd * sizeof(int4));
    l.sd = l.wab + align256(nab * H * kState * sizeof(float));
    l.total = l.sd + align256(nd * H * kState * sizeof(float));
    return l;
}

// Position of segment s of sequence b in the final launch: the last segments
// first (their S_T is the result), then the others in order.
__host__ __device__ __forceinline__ int final_index(int b, int s, int B, int P) {
    return s == P - 1 ? b : B + b * (P - 1) + s;
}

// Token ranges of both launches, and the start states of the first one: zero
// for the C runs (ranges 0 .. B(P-1)-1), the identity for the M runs.
__global__ void seg_init_kernel(int4 *ranges_ab, int4 *ranges_d, float *wab, int B, int T, int H, int P, int L) {
    const int nseg = B * (P - 1);
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = tid; i < (size_t)2 * nseg; i += stride) {
        const int j = (int)(i % nseg), b = j / (P - 1), s = j % (P - 1);
        const int tb = b * T + s * L;
        ranges_ab[i] = make_int4(tb, tb + L, i >= (size_t)nseg ? 1 : 0, 0);
    }
    for (size_t i = tid; i < (size_t)B * P; i += stride) {
        const int b = (int)(i / P), s = (int)(i % P);
        const int tb = b * T + s * L, te = s == P - 1 ? (b + 1) * T : tb + L;
        ranges_d[final_index(b, s, B, P)] = make_int4(tb, te, 0, 0);
    }
    const size_t n = (size_t)2 * nseg * H * kState;
    for (size_t i = tid; i < n; i += stride) {
        const size_t within = i % kState;
        wab[i] = (i >= n / 2 && within / kD == within % kD) ? 1.f : 0.f;
    }
}

// S_start(s + 1) = M_s S_start(s) + C_s for one (sequence, head) and 32 value
// columns, s = 0 .. P-2, in FP32; every S_start goes to its place among the
// final launch's start states.  Thread (warp w, lane j) keeps rows 16 w ..
// 16 w + 15 of column j.
__global__ void __launch_bounds__(256) seg_combine_kernel(const float *S0, const float *wab, float *sd, int B, int H,
                                                          int P) {
    extern __shared__ float smem[];
    constexpr int LDM = kD + 1;
    float *Ms = smem, *Ss = Ms + kD * LDM;     // M_s [kD][kD + 1]; S_start columns [kD][kCols]
    const int bh = blockIdx.x, b = bh / H, h = bh % H, col0 = blockIdx.y * kCols;
    const int tid = threadIdx.x, j = tid & 31, r0 = (tid >> 5) * 16;
    const int nseg = B * (P - 1);
    auto put = [&](int s) {
        float *dst = sd + ((size_t)final_index(b, s, B, P) * H + h) * kState + col0;
        for (int idx = tid; idx < kD * kCols; idx += 256) dst[(idx >> 5) * kD + (idx & 31)] = Ss[idx];
    };
    for (int idx = tid; idx < kD * kCols; idx += 256) {
        const int i = idx >> 5, jj = idx & 31;
        Ss[idx] = S0 ? S0[((size_t)b * H + h) * kState + (size_t)i * kD + col0 + jj] : 0.f;
    }
    __syncthreads();
    put(0);
    for (int s = 0; s + 1 < P; ++s) {
        const float *C = wab + ((size_t)(b * (P - 1) + s) * H + h) * kState;
        const float *M = wab + ((size_t)(nseg + b * (P - 1) + s) * H + h) * kState;
        for (int idx = tid; idx < kD * kD; idx += 256) Ms[(idx / kD) * LDM + idx % kD] = M[idx];
        __syncthreads();
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = C[(size_t)(r0 + r) * kD + col0 + j];
        for (int l = 0; l < kD; ++l) {
            const float sv = Ss[l * kCols + j];
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = fmaf(Ms[(r0 + r) * LDM + l], sv, acc[r]);
        }
        __syncthreads();                       // every read of S_start(s) and M_s is done
#pragma unroll
        for (int r = 0; r < 16; ++r) Ss[(r0 + r) * kCols + j] = acc[r];
        __syncthreads();
        put(s + 1);
    }
}

constexpr size_t kCombineSmem = ((size_t)kD * (kD + 1) + (size_t)kD * kCols) * sizeof(float);

}  // namespace

size_t segmented_workspace_bytes(int B, int H, int P) { return P <= 1 ? 0 : seg_layout(B, H, P).total; }

cudaError_t launch_chunk_segmented(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                                   const float *w, const float *S0, void *o, float *S_T, int B, int T, int H,
                                   int P, int L, void *workspace, cudaStream_t stream) {
    const SegLayout lay = seg_layout(B, H, P);
    char *base = static_cast<char *>(workspace);
    int4 *ranges_ab = reinterpret_cast<int4 *>(base + lay.ranges_ab);
    int4 *ranges_d = reinterpret_cast<int4 *>(base + lay.ranges_d);
    float *wab = reinterpret_cast<float *>(base + lay.wab);
    float *sd = reinterpret_cast<float *>(base + lay.sd);
    const int T_total = B * T;

    seg_init_kernel<<<296, 256, 0, stream>>>(ranges_ab, ranges_d, wab, B, T, H, P, L);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // 1. C_s (zero start) and M_s (identity start, z = 0) of segments 0 .. P-2, in place over their start states
    e = launch_chunk_tc(q, k, v, alpha, b, w, wab, nullptr, wab, 2 * B * (P - 1), T_total, H, nullptr, false, stream,
                        ranges_ab, -1);
    if (e != cudaSuccess) return e;
    // 2. the start state of every segment
    e = cudaFuncSetAttribute(seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCombineSmem);
    if (e != cudaSuccess) return e;     // set on every call: the attribute belongs to the current device
    seg_combine_kernel<<<dim3((unsigned)(B * H), kD / kCols), 256, kCombineSmem, stream>>>(S0, wab, sd, B, H, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. every segment from its start state: o, and S_T from the last segment of each sequence
    return launch_chunk_tc(q, k, v, alpha, b, w, sd, o, S_T, B * P, T_total, H, nullptr, false, stream, ranges_d,
                           S_T ? B : 0);
}

}  // namespace gdn2
