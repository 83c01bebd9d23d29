// gdn_inverse.cuh -- T = (I + A)^-1 for the 64 x 64 unit-lower-triangular
// factor of a chunk's WY representation ("Gated Attention Architectures",
// section 2: the UT transform), shared by the kernels that invert chunk
// factors outside the state loop (gdn_chunk_inv.cu, gdn_kda_tc.cu,
// gdn_backward_tc.cu).
//
// Divide and conquer on the block structure
//   [[X, 0], [C, Z]]^-1 = [[X^-1, 0], [-Z^-1 C X^-1, Z^-1]]:
// the four 16 x 16 diagonal blocks by forward substitution in fp32 (one
// thread per column), then the 16 -> 32 and 32 -> 64 levels as warp-level
// tf32 products with fp32 accumulation.  Where T is rounded to bf16
// afterwards the 10-bit tf32 mantissa is ample; the gradients, which keep T
// to about 16 bits, take the exact form (kExact), whose products split each
// operand into a tf32 value and a tf32 residual (x = hi + lo, three
// products hi hi + hi lo + lo hi: near-fp32 results).
#pragma once

#include "gdn_sm100.cuh"

namespace gdn {

constexpr int kLdA = 68;  // fp32 row stride of A / T (16-byte aligned rows, 4 mod 8 against bank conflicts)
constexpr int kLdY = 36;  // fp32 row stride of the block-product scratch

// c += X Z as tile_mma, each operand split into tf32 value + residual.
__device__ __forceinline__ void tile_mma3(float (&c)[4], const float *X, int ldx, const float *Z, int ldz, int n0,
                                          int nk, int lane) {
    using namespace sm100;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        if (s >= nk) break;
        const int k = 8 * s;
        const float af[4] = {X[g * ldx + k + t], X[(g + 8) * ldx + k + t], X[g * ldx + k + t + 4],
                             X[(g + 8) * ldx + k + t + 4]};
        const float bf[2] = {Z[(k + t) * ldz + n0 + g], Z[(k + t + 4) * ldz + n0 + g]};
        uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            ah[e] = to_tf32(af[e]);
            al[e] = to_tf32(af[e] - __uint_as_float(ah[e]));
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            bh[e] = to_tf32(bf[e]);
            bl[e] = to_tf32(bf[e] - __uint_as_float(bh[e]));
        }
        mma_tf32_16x8x8(c, al, bh);
        mma_tf32_16x8x8(c, ah, bl);
        mma_tf32_16x8x8(c, ah, bh);
    }
}

template <bool kExact>
__device__ __forceinline__ void inv_tile(float (&c)[4], const float *X, int ldx, const float *Z, int ldz, int n0,
                                         int nk, int lane) {
    if constexpr (kExact) tile_mma3(c, X, ldx, Z, ldz, n0, nk, lane);
    else sm100::tile_mma(c, X, ldx, Z, ldz, n0, nk, lane);
}

// T = (I + A)^-1 in place for the 64 x 64 strictly lower A in Af (everything
// on and above the diagonal zero).  Called by all kThreads threads.
template <bool kExact = false>
__device__ __forceinline__ void invert_in_place(float *Af, float *Y, int t) {
    using namespace sm100;
    const int w = t >> 5, lane = t & 31;
    // the four 16 x 16 diagonal blocks: thread (b, c) solves column c of block b
    float x[16];
    if (t < 64) {
        const int b = t >> 4, c = t & 15;
        const float *Ab = Af + (16 * b) * kLdA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float a[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) load4(Ab + r * kLdA + 4 * q, a + 4 * q);
            float acc0 = (r == c) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < r; ++jj) {
                if (jj & 1) acc1 = fmaf(-a[jj], x[jj], acc1);
                else acc0 = fmaf(-a[jj], x[jj], acc0);
            }
            x[r] = acc0 + acc1;
        }
    }
    __syncthreads();  // every diagonal block of A has been read
    if (t < 64) {
        const int b = t >> 4, c = t & 15;
        float *Tb = Af + (16 * b) * kLdA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * kLdA + c] = x[r];
    }
    __syncthreads();
    // 16 -> 32: in each 32 x 32 half p, Y = A21 T11, then T21 = -T22 Y
    if (w < 4) {
        const int p = w >> 1, n0 = 8 * (w & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        inv_tile<kExact>(c, Af + (32 * p + 16) * kLdA + 32 * p, kLdA, Af + (32 * p) * kLdA + 32 * p, kLdA, n0, 2, lane);
        tile_store(Y + (16 * p) * kLdY, kLdY, 0, n0, c, 1.f, lane);
    }
    __syncthreads();
    if (w < 4) {
        const int p = w >> 1, n0 = 8 * (w & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        inv_tile<kExact>(c, Af + (32 * p + 16) * kLdA + 32 * p + 16, kLdA, Y + (16 * p) * kLdY, kLdY, n0, 2, lane);
        tile_store(Af + (32 * p + 16) * kLdA + 32 * p, kLdA, 0, n0, c, -1.f, lane);
    }
    __syncthreads();
    // 32 -> 64: Y = A21 T11 (32 x 32), then T21 = -T22 Y
    {
        const int m0 = 16 * (w >> 2), n0 = 8 * (w & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        inv_tile<kExact>(c, Af + (32 + m0) * kLdA, kLdA, Af, kLdA, n0, 4, lane);
        tile_store(Y, kLdY, m0, n0, c, 1.f, lane);
    }
    __syncthreads();
    {
        const int m0 = 16 * (w >> 2), n0 = 8 * (w & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        inv_tile<kExact>(c, Af + (32 + m0) * kLdA + 32, kLdA, Y, kLdY, n0, 4, lane);
        tile_store(Af + 32 * kLdA, kLdA, m0, n0, c, -1.f, lane);  // rows 32 + m0 .., columns n0 ..
    }
    __syncthreads();
}

}  // namespace gdn
