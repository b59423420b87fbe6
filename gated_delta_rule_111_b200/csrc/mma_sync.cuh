// Split-TF32 products on the warp-level tensor-core MMA (mma.sync m16n8k8), shared
// by the kernels that need FP32-level accuracy from small shared-memory products
// (the backward's chunk products, the prefill's blocked inversion).
#pragma once

#include <stdint.h>

namespace gdn2 {

// Products on shared-memory operands with the warp-level tensor-core MMA
// (mma.sync m16n8k8, TF32 inputs, FP32 accumulation), three products per step:
// each operand is split into a TF32 high part and a TF32 remainder, and
// a_lo b_hi + a_hi b_lo + a_hi b_hi keeps FP32-level accuracy (the dropped
// a_lo b_lo term is below 2^-22 of the product).
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float rest = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(rest));
}

__device__ __forceinline__ void mma_16x8x8(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One warp's (16 WM) x (8 WN) block of C += A B, A(m, k) at A[m*sam + k*sak] and
// B(k, n) at B[k*sbk + n*sbn], rows from m0 and columns from n0; K a multiple of 8.
// Fragment layout of m16n8k8 (lane = 4 g + tg): A rows g, g + 8 and columns tg,
// tg + 4; B rows tg, tg + 4 and column g; C rows g, g + 8 and columns 2 tg, 2 tg + 1.
// Shared-memory banks: a row-major operand (unit column step) wants a row stride
// of 4 mod 32 floats, a transposed one (unit row step) 8 mod 32.
template <int WM, int WN>
struct Wt {
    float c[WM][WN][4];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int a = 0; a < WM; ++a)
#pragma unroll
            for (int b = 0; b < WN; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) c[a][b][i] = 0.f;
    }
    __device__ __forceinline__ void run(const float *A, int sam, int sak, const float *B, int sbk, int sbn, int K,
                                        int m0, int n0) {
        const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
#pragma unroll 2
        for (int k0 = 0; k0 < K; k0 += 8) {
            uint32_t ah[WM][4], al[WM][4], bh[WN][2], bl[WN][2];
#pragma unroll
            for (int a = 0; a < WM; ++a) {
                const float *p = A + (m0 + a * 16 + g) * sam + (k0 + tg) * sak;
                split_tf32(p[0], ah[a][0], al[a][0]);
                split_tf32(p[8 * sam], ah[a][1], al[a][1]);
                split_tf32(p[4 * sak], ah[a][2], al[a][2]);
                split_tf32(p[8 * sam + 4 * sak], ah[a][3], al[a][3]);
            }
#pragma unroll
            for (int b = 0; b < WN; ++b) {
                const float *p = B + (k0 + tg) * sbk + (n0 + b * 8 + g) * sbn;
                split_tf32(p[0], bh[b][0], bl[b][0]);
                split_tf32(p[4 * sbk], bh[b][1], bl[b][1]);
            }
#pragma unroll
            for (int a = 0; a < WM; ++a)
#pragma unroll
                for (int b = 0; b < WN; ++b) {
                    mma_16x8x8(c[a][b], al[a], bh[b]);
                    mma_16x8x8(c[a][b], ah[a], bl[b]);
                    mma_16x8x8(c[a][b], ah[a], bh[b]);
                }
        }
    }
    // Row and column of accumulator entry c[a][b][i].
    __device__ __forceinline__ static int row(int m0, int a, int i) {
        return m0 + a * 16 + ((threadIdx.x & 31) >> 2) + (i >> 1) * 8;
    }
    __device__ __forceinline__ static int col(int n0, int b, int i) {
        return n0 + b * 8 + 2 * (threadIdx.x & 3) + (i & 1);
    }
};


}  // namespace gdn2
