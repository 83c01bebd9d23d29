// gdn_mtp.cu -- several decode tokens per sequence in one pass, with the
// state after every token kept, for verifying draft tokens (multi-token
// prediction drafts a few tokens ahead and the model confirms several at
// once: "Architecture Thread I", the Qwen3-Next passage).
//
// For each (sequence, value head) the block reads S once, applies the K
// draft tokens in order with the decode step's row form
//   p_i = s_i . k, r_i = s_i . q, u_i = beta (v_i - alpha p_i),
//   s_i <- alpha s_i + u_i k^T, o_i = alpha r_i + u_i (k . q),
// and after token j writes o_j and the state snapshot S_j.  S itself is not
// modified: once the drafts are checked, gdn_decode_commit copies the
// snapshot of the accepted prefix into it.  Traffic per (sequence, head):
// one read of S and K snapshot writes, against K reads and K writes for K
// separate decode steps.
//
// d_k = 128: a warp owns whole state rows, lane l holds s_i[4l .. 4l+3]; the
// block's four warps take rows round-robin in batches of kMtpRows.  The K
// tokens' q, k (normalised if asked), alpha, beta and k . q are prepared
// once per block in shared memory.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kMtpWarps = 4;
constexpr int kMtpRows = 4;      // state rows per warp and batch
constexpr int kMtpMaxTok = 16;   // draft tokens per call

__device__ __forceinline__ float mtp_warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

template <typename T, uint32_t flags>
__global__ void __launch_bounds__(kMtpWarps * 32)
decode_multi_kernel(int32_t ntok, int32_t hk, int32_t hv, int32_t dv, const T *__restrict__ q,
                    const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, const float *__restrict__ state, float *__restrict__ snap,
                    T *__restrict__ o) {
    constexpr int dk = 128;
    constexpr bool kL2 = (flags & GDN_FLAG_QK_L2NORM) != 0;
    constexpr bool kLogits = (flags & GDN_FLAG_GATE_LOGITS) != 0;
    __shared__ __align__(16) float sk[kMtpMaxTok][dk], sq[kMtpMaxTok][dk];
    __shared__ float sal[kMtpMaxTok], sb[kMtpMaxTok], skq[kMtpMaxTok];
    const int unit = blockIdx.x;  // sequence * hv + head
    const int n = unit / hv, h = unit % hv;
    const int hq = h / (hv / hk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // the K tokens' inputs, one warp per token
    for (int j = warp; j < ntok; j += kMtpWarps) {
        const size_t qk = ((size_t(n) * ntok + j) * hk + hq) * dk + 4 * lane;
        float kf[4], qf[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kf[e] = to_f32(k[qk + e]);
            qf[e] = to_f32(q[qk + e]);
        }
        if constexpr (kL2) {
            const float ik = inv_l2(mtp_warp_sum(kf[0] * kf[0] + kf[1] * kf[1] + kf[2] * kf[2] + kf[3] * kf[3]));
            const float iq = inv_l2(mtp_warp_sum(qf[0] * qf[0] + qf[1] * qf[1] + qf[2] * qf[2] + qf[3] * qf[3]));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kf[e] *= ik;
                qf[e] *= iq;
            }
        }
        const float kq = mtp_warp_sum(kf[0] * qf[0] + kf[1] * qf[1] + kf[2] * qf[2] + kf[3] * qf[3]);
        *reinterpret_cast<float4 *>(&sk[j][4 * lane]) = make_float4(kf[0], kf[1], kf[2], kf[3]);
        *reinterpret_cast<float4 *>(&sq[j][4 * lane]) = make_float4(qf[0], qf[1], qf[2], qf[3]);
        if (lane == 0) {
            const size_t gb = (size_t(n) * ntok + j) * hv + h;
            sal[j] = __expf(fmaxf(kLogits ? log_sigmoid(g[gb]) : g[gb], kGFloor));
            sb[j] = kLogits ? sigmoid(beta[gb]) : beta[gb];
            skq[j] = kq;
        }
    }
    __syncthreads();

    const float *S = state + size_t(unit) * dv * dk;
    for (int i0 = warp * kMtpRows; i0 < dv; i0 += kMtpWarps * kMtpRows) {
        float4 s[kMtpRows];
#pragma unroll
        for (int r = 0; r < kMtpRows; ++r)
            if (i0 + r < dv) s[r] = __ldcs(reinterpret_cast<const float4 *>(S + size_t(i0 + r) * dk + 4 * lane));
        for (int j = 0; j < ntok; ++j) {
            const float4 kf = *reinterpret_cast<const float4 *>(&sk[j][4 * lane]);
            const float4 qf = *reinterpret_cast<const float4 *>(&sq[j][4 * lane]);
            const float alpha = sal[j], b = sb[j], kq = skq[j];
            const size_t tv = (size_t(n) * ntok + j) * hv + h;  // (sequence, token, head)
            float p[kMtpRows], rq[kMtpRows], vr[kMtpRows];
#pragma unroll
            for (int r = 0; r < kMtpRows; ++r) {
                vr[r] = (i0 + r < dv) ? to_f32(v[tv * dv + i0 + r]) : 0.f;
                p[r] = s[r].x * kf.x + s[r].y * kf.y + s[r].z * kf.z + s[r].w * kf.w;
                rq[r] = s[r].x * qf.x + s[r].y * qf.y + s[r].z * qf.z + s[r].w * qf.w;
            }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1)
#pragma unroll
                for (int r = 0; r < kMtpRows; ++r) {
                    p[r] += __shfl_xor_sync(0xffffffffu, p[r], m);
                    rq[r] += __shfl_xor_sync(0xffffffffu, rq[r], m);
                }
            float *Sj = snap + tv * size_t(dv) * dk;
#pragma unroll
            for (int r = 0; r < kMtpRows; ++r) {
                if (i0 + r >= dv) continue;
                const float u = b * (vr[r] - alpha * p[r]);
                s[r].x = fmaf(alpha, s[r].x, u * kf.x);
                s[r].y = fmaf(alpha, s[r].y, u * kf.y);
                s[r].z = fmaf(alpha, s[r].z, u * kf.z);
                s[r].w = fmaf(alpha, s[r].w, u * kf.w);
                __stcs(reinterpret_cast<float4 *>(Sj + size_t(i0 + r) * dk + 4 * lane), s[r]);
                if (lane == r) o[tv * dv + i0 + r] = from_f32<T>(fmaf(alpha, rq[r], u * kq));
            }
        }
    }
}

// state[n, h] <- snapshot (n, accepted[n] - 1, h) for accepted[n] in 1..K;
// accepted[n] = 0 keeps the state; other values leave it and are counted in
// *bad (if not NULL).  One block per (sequence, head), float4 copies.
__global__ void decode_commit_kernel(int32_t ntok, int32_t hv, int32_t elems4, const float4 *__restrict__ snap,
                                     const int32_t *__restrict__ accepted, float4 *__restrict__ state,
                                     int32_t *bad) {
    const int unit = blockIdx.x;
    const int n = unit / hv, h = unit % hv;
    const int a = accepted[n];
    if (a < 0 || a > ntok) {
        if (threadIdx.x == 0 && h == 0 && bad) atomicAdd(bad, 1);
        return;
    }
    if (a == 0) return;
    const float4 *src = snap + ((size_t(n) * ntok + (a - 1)) * hv + h) * size_t(elems4);
    float4 *dst = state + size_t(unit) * elems4;
    for (int i = threadIdx.x; i < elems4; i += blockDim.x) dst[i] = src[i];
}

template <uint32_t F>
static void launch_multi_as(unsigned grid, int32_t ntok, int32_t hk, int32_t hv, int32_t dv, int32_t dtype,
                            const void *q, const void *k, const void *v, const float *g, const float *beta,
                            const float *state, float *snap, void *o, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    if (dtype == GDN_DTYPE_BF16)
        decode_multi_kernel<bf, F><<<grid, kMtpWarps * 32, 0, stream>>>(
            ntok, hk, hv, dv, static_cast<const bf *>(q), static_cast<const bf *>(k), static_cast<const bf *>(v), g,
            beta, state, snap, static_cast<bf *>(o));
    else
        decode_multi_kernel<float, F><<<grid, kMtpWarps * 32, 0, stream>>>(
            ntok, hk, hv, dv, static_cast<const float *>(q), static_cast<const float *>(k),
            static_cast<const float *>(v), g, beta, state, snap, static_cast<float *>(o));
}

cudaError_t launch_decode_multi(int32_t n, int32_t ntok, int32_t hk, int32_t hv, int32_t dk, int32_t dv,
                                int32_t dtype, const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *state, float *snap, void *o, uint32_t flags,
                                cudaStream_t stream) {
    const int64_t units = int64_t(n) * hv;
    if (units <= 0) return cudaSuccess;
    if (units > INT32_MAX || dk != 128 || ntok < 1 || ntok > kMtpMaxTok) return cudaErrorInvalidValue;
    const unsigned grid = unsigned(units);
    switch (flags & (GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS)) {
        case 0: launch_multi_as<0>(grid, ntok, hk, hv, dv, dtype, q, k, v, g, beta, state, snap, o, stream); break;
        case GDN_FLAG_QK_L2NORM:
            launch_multi_as<GDN_FLAG_QK_L2NORM>(grid, ntok, hk, hv, dv, dtype, q, k, v, g, beta, state, snap, o,
                                                stream);
            break;
        case GDN_FLAG_GATE_LOGITS:
            launch_multi_as<GDN_FLAG_GATE_LOGITS>(grid, ntok, hk, hv, dv, dtype, q, k, v, g, beta, state, snap, o,
                                                  stream);
            break;
        default:
            launch_multi_as<GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS>(grid, ntok, hk, hv, dv, dtype, q, k, v, g,
                                                                      beta, state, snap, o, stream);
            break;
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_decode_commit(int32_t n, int32_t ntok, int32_t hv, int32_t dk, int32_t dv, const float *snap,
                                 const int32_t *accepted, float *state, int32_t *bad, cudaStream_t stream) {
    const int64_t units = int64_t(n) * hv;
    if (units <= 0) return cudaSuccess;
    if (units > INT32_MAX || (int64_t(dv) * dk) % 4 != 0) return cudaErrorInvalidValue;
    decode_commit_kernel<<<unsigned(units), 256, 0, stream>>>(ntok, hv, int32_t(int64_t(dv) * dk / 4),
                                                             reinterpret_cast<const float4 *>(snap), accepted,
                                                             reinterpret_cast<float4 *>(state), bad);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
