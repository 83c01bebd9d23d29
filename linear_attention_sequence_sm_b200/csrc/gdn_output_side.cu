// gdn_output_side.cu -- the mixer's output side as a pass over o in place:
// every (token, value head) row o of d_v values becomes
//   y_i = o_i / sqrt(mean_j(o_j^2) + eps) * s_i * act(z_i)
// (RMS normalisation of the mixer output, "Architecture Thread I", "Modern
// Architecture Improvements"; the gated form of the Gated DeltaNet code
// listing in "Gated Attention Architectures").  The tensor-core prefill and
// the decode kernels apply it in their own epilogues; this pass serves the
// CUDA-core prefill, whose blocks each own a 32-row slice of d_v and so never
// hold a whole output row.  One warp per row; d_v <= 128 (lane l holds
// elements l, l + 32, ...).  Reads o and z once and writes o once.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kOutWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kOutWarps * 32)
output_side_kernel(T *__restrict__ o, int64_t rows, int32_t hv, int32_t dv, const OutSide os) {
    const int lane = threadIdx.x & 31;
    const int64_t row = int64_t(blockIdx.x) * kOutWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int h = int(row % hv);
    T *x = o + row * dv;
    const T *z = os.z ? static_cast<const T *>(os.z) + row * dv : nullptr;
    float v[4];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = lane + 32 * e;
        v[e] = i < dv ? to_f32(x[i]) : 0.f;
        ss = fmaf(v[e], v[e], ss);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float inv_rms = rsqrtf(ss / float(dv) + os.eps);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = lane + 32 * e;
        if (i >= dv) continue;
        const float gz = z ? out_gate(os.flags, to_f32(z[i])) : 1.f;
        x[i] = from_f32<T>(v[e] * inv_rms * out_scale(os, h, i, dv) * gz);
    }
}

cudaError_t launch_output_side(void *o, int32_t tokens, int32_t hv, int32_t dv, int32_t dtype, const OutSide &os,
                               cudaStream_t stream) {
    const int64_t rows = int64_t(tokens) * hv;
    if (rows <= 0) return cudaSuccess;
    if (dv > 128) return cudaErrorInvalidValue;
    const int64_t blocks = (rows + kOutWarps - 1) / kOutWarps;
    if (blocks > INT32_MAX) return cudaErrorInvalidValue;
    if (dtype == GDN_DTYPE_BF16)
        output_side_kernel<__nv_bfloat16><<<unsigned(blocks), kOutWarps * 32, 0, stream>>>(
            static_cast<__nv_bfloat16 *>(o), rows, hv, dv, os);
    else
        output_side_kernel<float><<<unsigned(blocks), kOutWarps * 32, 0, stream>>>(static_cast<float *>(o), rows,
                                                                                   hv, dv, os);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
