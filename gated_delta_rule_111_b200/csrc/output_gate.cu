// Output epilogue of the Gated DeltaNet-2 layer: per (token, head) row of d_v
// channels,
//   y = o / sqrt(mean_j(o_j^2) + eps) * weight * sigmoid(g)
// ("Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
// iplexlaw.co.kr analysis, "Token processing and parallel training": after the
// recurrent update come RMS normalisation and a separate output gate, distinct
// from the write gate, before the output projection).  The RMS norm runs over
// one head's channels with a per-channel weight; the gate is a sigmoid of its own
// logits, like the layer's other gates.
//
// Memory-bound: one read of o and g and one write of y per element.  A warp owns
// a row; each warp issues the loads of four rows before it reduces any of them.
#include "common.cuh"

namespace gdn2 {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kThreads = 256;

template <typename T, int DV> struct Vec;
template <> struct Vec<__nv_bfloat16, 128> {      // 4 channels per lane: 8 bytes
    using raw = uint2;
    static __device__ __forceinline__ void unpack(raw r, float (&x)[4]) {
        x[0] = __uint_as_float(r.x << 16); x[1] = __uint_as_float(r.x & 0xFFFF0000u);
        x[2] = __uint_as_float(r.y << 16); x[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
    static __device__ __forceinline__ raw pack(const float (&x)[4]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
        return make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
    }
    static constexpr int N = 4;
};
template <> struct Vec<__nv_bfloat16, 64> {       // 2 channels per lane: 4 bytes
    using raw = uint32_t;
    static __device__ __forceinline__ void unpack(raw r, float (&x)[2]) {
        x[0] = __uint_as_float(r << 16); x[1] = __uint_as_float(r & 0xFFFF0000u);
    }
    static __device__ __forceinline__ raw pack(const float (&x)[2]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        return *reinterpret_cast<const uint32_t *>(&a);
    }
    static constexpr int N = 2;
};
template <> struct Vec<float, 128> {              // 4 channels per lane: 16 bytes
    using raw = float4;
    static __device__ __forceinline__ void unpack(raw r, float (&x)[4]) { x[0] = r.x; x[1] = r.y; x[2] = r.z; x[3] = r.w; }
    static __device__ __forceinline__ raw pack(const float (&x)[4]) { return make_float4(x[0], x[1], x[2], x[3]); }
    static constexpr int N = 4;
};
template <> struct Vec<float, 64> {               // 2 channels per lane: 8 bytes
    using raw = float2;
    static __device__ __forceinline__ void unpack(raw r, float (&x)[2]) { x[0] = r.x; x[1] = r.y; }
    static __device__ __forceinline__ raw pack(const float (&x)[2]) { return make_float2(x[0], x[1]); }
    static constexpr int N = 2;
};

template <typename T, int DV>
__global__ void __launch_bounds__(kThreads)
output_gate_kernel(const T *o, const T *g, const float *__restrict__ weight, float eps, T *y, long long rows) {
    using V = Vec<T, DV>;
    constexpr int N = V::N;
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
    float wt[N];
#pragma unroll
    for (int e = 0; e < N; ++e) wt[e] = __ldg(weight + lane * N + e);
    for (long long r0 = warp0 * kRowsPerWarp; r0 < rows; r0 += nwarps * kRowsPerWarp) {
        typename V::raw ro[kRowsPerWarp], rg[kRowsPerWarp];
#pragma unroll
        for (int u = 0; u < kRowsPerWarp; ++u) {
            if (r0 + u < rows) {
                const size_t off = (size_t)(r0 + u) * (DV / N) + lane;
                ro[u] = reinterpret_cast<const typename V::raw *>(o)[off];
                rg[u] = reinterpret_cast<const typename V::raw *>(g)[off];
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerWarp; ++u) {
            if (r0 + u >= rows) break;
            float x[N], gv[N];
            V::unpack(ro[u], x);
            V::unpack(rg[u], gv);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < N; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const float inv = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
            for (int e = 0; e < N; ++e) x[e] = x[e] * inv * wt[e] * __fdividef(1.f, 1.f + __expf(-gv[e]));
            reinterpret_cast<typename V::raw *>(y)[(size_t)(r0 + u) * (DV / N) + lane] = V::pack(x);
        }
    }
}

template <typename T, int DV>
cudaError_t launch_typed(const void *o, const void *g, const float *weight, float eps, void *y, long long rows,
                         cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long need = (rows + kRowsPerWarp * (kThreads / 32) - 1) / (kRowsPerWarp * (kThreads / 32));
    const long long cap = (long long)sms * 8;        // eight 256-thread blocks per SM, grid-stride beyond
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    output_gate_kernel<T, DV><<<grid, kThreads, 0, stream>>>(static_cast<const T *>(o), static_cast<const T *>(g),
                                                             weight, eps, static_cast<T *>(y), rows);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_output_gate(const void *o, const void *g, const float *weight, float eps, void *y,
                               long long rows, int dv, gdn2_dtype dt, cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    if (dt == GDN2_BF16)
        return dv == 128 ? launch_typed<__nv_bfloat16, 128>(o, g, weight, eps, y, rows, stream)
                         : launch_typed<__nv_bfloat16, 64>(o, g, weight, eps, y, rows, stream);
    return dv == 128 ? launch_typed<float, 128>(o, g, weight, eps, y, rows, stream)
                     : launch_typed<float, 64>(o, g, weight, eps, y, rows, stream);
}

}  // namespace gdn2
