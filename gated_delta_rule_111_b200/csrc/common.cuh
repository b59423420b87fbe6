// Internal helpers shared by the libgdn2 kernels (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn2.h"

namespace gdn2 {

// Element type of q, k, v, o.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// alpha below FLT_MIN is treated as FLT_MIN (documented precondition: alpha > 0).
__device__ __forceinline__ float clamp_alpha(float a) { return fmaxf(a, 1.17549435e-38f); }

// Streaming (read-once / write-once) 16-byte accesses for the decode state.
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

// Host-side launchers (one per kernel family); each returns cudaGetLastError().
cudaError_t launch_recurrent_step(const void *q, const void *k, const void *v, const float *alpha,
                                  const float *b, const float *w, float *S, void *o, int B, int H,
                                  int dk, int dv, gdn2_dtype dt, cudaStream_t stream);

// B sequences of T tokens (cu_seqlens == nullptr), or B packed sequences with device
// offsets cu_seqlens[0..B] into T tokens in all.
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *alpha,
                              const float *b, const float *w, const float *S0, void *o, float *S_T,
                              int B, int T, int H, int dk, int dv, gdn2_dtype dt, const int *cu_seqlens,
                              cudaStream_t stream);

// Chunkwise prefill on the tensor cores (BF16 q/k/v, d_k = d_v = 128): nseq
// sequences of T tokens each; or packed, with device offsets cu_seqlens[0..nseq]
// or device token ranges ranges[0..nseq) (x, y: tokens [x, y) of the flat axis;
// z != 0: written values taken as zero) into T tokens in all.  o may be null;
// only sequences below nst (all when nst < 0) write S_T.
bool chunk_tc_supported(int dk, int dv, gdn2_dtype dt);
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *alpha, const void *b,
                            const void *w, const float *S0, void *o, float *S_T, int nseq, int T, int H,
                            const int *cu_seqlens, bool logits, cudaStream_t stream, const int4 *ranges = nullptr,
                            int nst = -1);

// Segment-parallel prefill of B sequences of T tokens cut into P segments of L
// tokens (the last shorter): workspace of segmented_workspace_bytes(B, H, P).
size_t segmented_workspace_bytes(int B, int H, int P);
cudaError_t launch_chunk_segmented(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                                   const float *w, const float *S0, void *o, float *S_T, int B, int T, int H,
                                   int P, int L, void *workspace, cudaStream_t stream);

// Chunkwise backward: prep, state and gradient launches.  workspace holds
// chunk_bwd_workspace_floats(B, T, H, dk, dv) floats.
size_t chunk_bwd_workspace_floats(int B, int T, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                             const float *w, const float *S0, const void *dO, const float *dST, void *dq, void *dk,
                             void *dv, float *dalpha, float *db, float *dw, float *dS0, float *workspace, int B,
                             int T, int H, int d_k, int d_v, gdn2_dtype dt, cudaStream_t stream);

// Output epilogue: rows = B*T*H rows of dv channels (dv 64 or 128).
cudaError_t launch_output_gate(const void *o, const void *g, const float *weight, float eps, void *y,
                               long long rows, int dv, gdn2_dtype dt, cudaStream_t stream);

}  // namespace gdn2
