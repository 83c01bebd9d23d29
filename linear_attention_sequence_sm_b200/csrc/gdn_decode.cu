// gdn_decode.cu -- one decode token per sequence, state updated in place.
//
// Per value head and per state row i (s_i = row i of S, length d_k):
//   p_i = s_i . k,  r_i = s_i . q                 (the two dot products)
//   u_i = beta (v_i - alpha p_i)                  (error-corrected write)
//   s_i <- alpha s_i + u_i k^T
//   o_i = alpha r_i + u_i (k . q)                 (= s_i,new . q)
// which is the gated delta rule S_t = S_{t-1}(alpha(I - beta k k^T)) +
// beta v k^T, o = S_t q ("Architecture Thread I", section "Gated DeltaNet";
// "Gated Attention Architectures", section 3) written so that S is read once
// and written once.  Decode is bound by that traffic ("The Transformer Isn't
// Alone Anymore": the recurrent state is read and updated every step).
//
// With the output side (gdn_decode_step_out) the d_v outputs of the block's
// (sequence, head) wait in shared memory; one block reduction gives their
// root mean square, and y = o / rms * s * act(z) is written once.
//
// d_k = 128: a warp owns whole rows; lane l holds s_i[4l .. 4l+3] as one
// float4 (a row is one coalesced 512-byte segment).  Each warp keeps
// kRowBatch rows of loads in flight before reducing, for memory-level
// parallelism.  Other d_k (<= 256): a generic warp-per-row kernel.
#include "gdn_internal.cuh"

namespace gdn {

#ifndef GDN_DECODE_ROWS
#define GDN_DECODE_ROWS 8
#endif
#ifndef GDN_DECODE_MINBLOCKS
#define GDN_DECODE_MINBLOCKS 1
#endif
constexpr int kDecodeWarps = 4;     // warps per block; a block owns one (sequence, head)
constexpr int kRowBatch = GDN_DECODE_ROWS;  // rows in flight per warp
// Template bit (beside the GDN_FLAG_* input-side bits): the output side is
// applied in the kernel.  The rows of o then wait in shared memory until the
// whole vector is known, for its root mean square.
constexpr uint32_t kDecOut = 1u << 8;
constexpr int kDecOutMaxDv = 256;
// Template bit: Kimi Delta Attention, g holds one log-decay per key channel
// ([N, Hv, d_k]): each row becomes s' = alpha .* s, p = s' . k, r = s' . q,
// u = beta (v - p), s <- s' + u k, o = r + u (k . q) ("Gated Attention
// Architectures", section 8; with all alpha[c] equal, the gated delta rule).
constexpr uint32_t kDecKda = 1u << 9;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

__device__ __forceinline__ float4 load4(const float *p) { return __ldcs(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ void store4(float *p, float4 x) { __stcs(reinterpret_cast<float4 *>(p), x); }

__device__ __forceinline__ void load_vec4(const float *p, float out[4]) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
}
__device__ __forceinline__ void load_vec4(const __nv_bfloat16 *p, float out[4]) {
    const uint2 x = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&x.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&x.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    out[0] = fa.x; out[1] = fa.y; out[2] = fb.x; out[3] = fb.y;
}

template <typename T, uint32_t flags>
__global__ void __launch_bounds__(kDecodeWarps * 32, GDN_DECODE_MINBLOCKS)
decode_d128_kernel(int32_t hk, int32_t hv, int32_t dv, const T *__restrict__ q, const T *__restrict__ k,
                   const T *__restrict__ v, const float *__restrict__ g, const float *__restrict__ beta,
                   float *__restrict__ state, T *__restrict__ o, const OutSide os) {
    constexpr int dk = 128;
    constexpr bool kOut = (flags & kDecOut) != 0;
    __shared__ float ob[kOut ? kDecOutMaxDv : 1], red[kDecodeWarps];
    const int unit = blockIdx.x;            // sequence * hv + head
    const int n = unit / hv, h = unit % hv;
    const int hq = h / (hv / hk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float kf[4], qf[4];
    load_vec4(k + (size_t(n) * hk + hq) * dk + 4 * lane, kf);
    load_vec4(q + (size_t(n) * hk + hq) * dk + 4 * lane, qf);
    if constexpr ((flags & GDN_FLAG_QK_L2NORM) != 0) {
        const float ik = inv_l2(warp_sum(kf[0] * kf[0] + kf[1] * kf[1] + kf[2] * kf[2] + kf[3] * kf[3]));
        const float iq = inv_l2(warp_sum(qf[0] * qf[0] + qf[1] * qf[1] + qf[2] * qf[2] + qf[3] * qf[3]));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kf[e] *= ik;
            qf[e] *= iq;
        }
    }
    const float kq = warp_sum(kf[0] * qf[0] + kf[1] * qf[1] + kf[2] * qf[2] + kf[3] * qf[3]);
    constexpr bool logits = (flags & GDN_FLAG_GATE_LOGITS) != 0;
    constexpr bool kKda = (flags & kDecKda) != 0;
    // GDN: one decay alpha; KDA: al[e] for this lane's channels, and the dot
    // products take alpha .* k and alpha .* q
    float alpha = 1.f, al[4], ak[4], aq[4];
    if constexpr (kKda) {
        float gg[4];
        load_vec4(g + size_t(unit) * dk + 4 * lane, gg);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            al[e] = __expf(fmaxf(logits ? log_sigmoid(gg[e]) : gg[e], kGFloor));
            ak[e] = al[e] * kf[e];
            aq[e] = al[e] * qf[e];
        }
    } else {
        alpha = __expf(fmaxf(logits ? log_sigmoid(g[unit]) : g[unit], kGFloor));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            al[e] = alpha;
            ak[e] = kf[e];
            aq[e] = qf[e];
        }
    }
    const float b = logits ? sigmoid(beta[unit]) : beta[unit];

    float *S = state + size_t(unit) * dv * dk;
    const T *vrow = v + size_t(unit) * dv;
    T *orow = o + size_t(unit) * dv;

    for (int i0 = warp * kRowBatch; i0 < dv; i0 += kDecodeWarps * kRowBatch) {
        float4 s[kRowBatch];
#pragma unroll
        for (int r = 0; r < kRowBatch; ++r)
            if (i0 + r < dv) s[r] = load4(S + size_t(i0 + r) * dk + 4 * lane);
        float vr[kRowBatch];
#pragma unroll
        for (int r = 0; r < kRowBatch; ++r) vr[r] = (i0 + r < dv) ? to_f32(vrow[i0 + r]) : 0.f;
        float p[kRowBatch], rq[kRowBatch];
#pragma unroll
        for (int r = 0; r < kRowBatch; ++r) {
            if (i0 + r < dv) {
                p[r] = s[r].x * ak[0] + s[r].y * ak[1] + s[r].z * ak[2] + s[r].w * ak[3];
                rq[r] = s[r].x * aq[0] + s[r].y * aq[1] + s[r].z * aq[2] + s[r].w * aq[3];
            } else {
                p[r] = rq[r] = 0.f;
            }
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
#pragma unroll
            for (int r = 0; r < kRowBatch; ++r) {
                p[r] += __shfl_xor_sync(0xffffffffu, p[r], m);
                rq[r] += __shfl_xor_sync(0xffffffffu, rq[r], m);
            }
        }
#pragma unroll
        for (int r = 0; r < kRowBatch; ++r) {
            if (i0 + r >= dv) continue;
            // GDN: p and rq are undecayed, alpha applies here; KDA: already decayed
            const float u = kKda ? b * (vr[r] - p[r]) : b * (vr[r] - alpha * p[r]);
            float4 sn;
            sn.x = fmaf(al[0], s[r].x, u * kf[0]);
            sn.y = fmaf(al[1], s[r].y, u * kf[1]);
            sn.z = fmaf(al[2], s[r].z, u * kf[2]);
            sn.w = fmaf(al[3], s[r].w, u * kf[3]);
            store4(S + size_t(i0 + r) * dk + 4 * lane, sn);
            if (lane == r) {
                const float ov = kKda ? fmaf(u, kq, rq[r]) : fmaf(alpha, rq[r], u * kq);
                if constexpr (kOut) ob[i0 + r] = ov;
                else orow[i0 + r] = from_f32<T>(ov);
            }
        }
    }
    if constexpr (kOut) decode_output_side(ob, red, dv, unit, h, os, orow);
}

// Output side over the block's d_v outputs in shared memory (kDecOut).
template <typename T>
__device__ __forceinline__ void decode_output_side(const float *ob, float *red, int dv, int unit, int h,
                                                   const OutSide &os, T *orow) {
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float ss = 0.f;
    for (int i = threadIdx.x; i < dv; i += kDecodeWarps * 32) ss = fmaf(ob[i], ob[i], ss);
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) tot += red[w];
    const float inv_rms = rsqrtf(tot / float(dv) + os.eps);
    const T *z = os.z ? static_cast<const T *>(os.z) + size_t(unit) * dv : nullptr;
    for (int i = threadIdx.x; i < dv; i += kDecodeWarps * 32) {
        const float gz = z ? out_gate(os.flags, to_f32(z[i])) : 1.f;
        orow[i] = from_f32<T>(ob[i] * inv_rms * out_scale(os, h, i, dv) * gz);
    }
}

// Generic d_k <= 256: warp per row, lane l holds elements l, l+32, ...
template <typename T, uint32_t flags>
__global__ void __launch_bounds__(kDecodeWarps * 32)
decode_generic_kernel(int32_t hk, int32_t hv, int32_t dk, int32_t dv, const T *__restrict__ q,
                      const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ g,
                      const float *__restrict__ beta, float *__restrict__ state, T *__restrict__ o,
                      const OutSide os) {
    constexpr int kMaxPer = 8;  // 8 * 32 = 256 elements
    constexpr bool kOut = (flags & kDecOut) != 0;
    __shared__ float ob[kOut ? kDecOutMaxDv : 1], red[kDecodeWarps];
    const int unit = blockIdx.x;
    const int n = unit / hv, h = unit % hv;
    const int hq = h / (hv / hk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float kf[kMaxPer], qf[kMaxPer];
    float kk = 0.f, qq = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e) {
        const int j = lane + 32 * e;
        kf[e] = j < dk ? to_f32(k[(size_t(n) * hk + hq) * dk + j]) : 0.f;
        qf[e] = j < dk ? to_f32(q[(size_t(n) * hk + hq) * dk + j]) : 0.f;
        kk += kf[e] * kf[e];
        qq += qf[e] * qf[e];
    }
    if constexpr ((flags & GDN_FLAG_QK_L2NORM) != 0) {
        const float ik = inv_l2(warp_sum(kk)), iq = inv_l2(warp_sum(qq));
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) {
            kf[e] *= ik;
            qf[e] *= iq;
        }
    }
    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e) kq += kf[e] * qf[e];
    kq = warp_sum(kq);
    constexpr bool logits = (flags & GDN_FLAG_GATE_LOGITS) != 0;
    constexpr bool kKda = (flags & kDecKda) != 0;
    float alpha = 1.f, al[kMaxPer];
    if constexpr (kKda) {
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) {
            const int j = lane + 32 * e;
            const float gg = j < dk ? g[size_t(unit) * dk + j] : 0.f;
            al[e] = __expf(fmaxf(logits ? log_sigmoid(gg) : gg, kGFloor));
        }
    } else {
        alpha = __expf(fmaxf(logits ? log_sigmoid(g[unit]) : g[unit], kGFloor));
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) al[e] = alpha;
    }
    const float b = logits ? sigmoid(beta[unit]) : beta[unit];
    float *S = state + size_t(unit) * dv * dk;
    for (int i = warp; i < dv; i += kDecodeWarps) {
        float s[kMaxPer];
        float p = 0.f, rq = 0.f;
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) {
            const int j = lane + 32 * e;
            s[e] = j < dk ? S[size_t(i) * dk + j] : 0.f;
            const float sd = kKda ? al[e] * s[e] : s[e];  // KDA: the decayed row
            p += sd * kf[e];
            rq += sd * qf[e];
        }
        p = warp_sum(p);
        rq = warp_sum(rq);
        const float u = kKda ? b * (to_f32(v[size_t(unit) * dv + i]) - p)
                             : b * (to_f32(v[size_t(unit) * dv + i]) - alpha * p);
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) {
            const int j = lane + 32 * e;
            if (j < dk) S[size_t(i) * dk + j] = fmaf(al[e], s[e], u * kf[e]);
        }
        if (lane == 0) {
            const float ov = kKda ? fmaf(u, kq, rq) : fmaf(alpha, rq, u * kq);
            if constexpr (kOut) ob[i] = ov;
            else o[size_t(unit) * dv + i] = from_f32<T>(ov);
        }
    }
    if constexpr (kOut) decode_output_side(ob, red, dv, unit, h, os, o + size_t(unit) * dv);
}

template <uint32_t F>
static void launch_decode_as(dim3 grid, dim3 block, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                             const void *q, const void *k, const void *v, const float *g, const float *beta,
                             float *state, void *o, const OutSide &os, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    if (dk == 128) {
        if (dtype == GDN_DTYPE_BF16)
            decode_d128_kernel<bf, F><<<grid, block, 0, stream>>>(
                hk, hv, dv, static_cast<const bf *>(q), static_cast<const bf *>(k), static_cast<const bf *>(v), g,
                beta, state, static_cast<bf *>(o), os);
        else
            decode_d128_kernel<float, F><<<grid, block, 0, stream>>>(
                hk, hv, dv, static_cast<const float *>(q), static_cast<const float *>(k),
                static_cast<const float *>(v), g, beta, state, static_cast<float *>(o), os);
    } else {
        if (dtype == GDN_DTYPE_BF16)
            decode_generic_kernel<bf, F><<<grid, block, 0, stream>>>(
                hk, hv, dk, dv, static_cast<const bf *>(q), static_cast<const bf *>(k), static_cast<const bf *>(v),
                g, beta, state, static_cast<bf *>(o), os);
        else
            decode_generic_kernel<float, F><<<grid, block, 0, stream>>>(
                hk, hv, dk, dv, static_cast<const float *>(q), static_cast<const float *>(k),
                static_cast<const float *>(v), g, beta, state, static_cast<float *>(o), os);
    }
}

static cudaError_t launch_decode_any(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                     const void *q, const void *k, const void *v, const float *g,
                                     const float *beta, float *state, void *o, uint32_t flags, const OutSide &os,
                                     bool kda, cudaStream_t stream) {
    const int64_t units = int64_t(n) * hv;
    if (units > INT32_MAX) return cudaErrorInvalidValue;
    if (os.flags && dv > kDecOutMaxDv) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(units)), block(kDecodeWarps * 32);
    constexpr uint32_t L2 = GDN_FLAG_QK_L2NORM, LG = GDN_FLAG_GATE_LOGITS;
    const uint32_t f = (flags & (L2 | LG)) | (os.flags ? kDecOut : 0u) | (kda ? kDecKda : 0u);
#define GDN_DECODE_CASE(F)                                                                                  \
    case F: launch_decode_as<F>(grid, block, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, os, stream); \
        break;
    switch (f) {
        GDN_DECODE_CASE(0u)
        GDN_DECODE_CASE(L2)
        GDN_DECODE_CASE(LG)
        GDN_DECODE_CASE(L2 | LG)
        GDN_DECODE_CASE(kDecOut)
        GDN_DECODE_CASE(kDecOut | L2)
        GDN_DECODE_CASE(kDecOut | LG)
        GDN_DECODE_CASE(kDecOut | L2 | LG)
        GDN_DECODE_CASE(kDecKda)
        GDN_DECODE_CASE(kDecKda | L2)
        GDN_DECODE_CASE(kDecKda | LG)
        GDN_DECODE_CASE(kDecKda | L2 | LG)
        GDN_DECODE_CASE(kDecKda | kDecOut)
        GDN_DECODE_CASE(kDecKda | kDecOut | L2)
        GDN_DECODE_CASE(kDecKda | kDecOut | LG)
        GDN_DECODE_CASE(kDecKda | kDecOut | L2 | LG)
        default: return cudaErrorInvalidValue;
    }
#undef GDN_DECODE_CASE
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_decode(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                          const void *q, const void *k, const void *v, const float *g, const float *beta,
                          float *state, void *o, uint32_t flags, const OutSide &os, cudaStream_t stream) {
    return launch_decode_any(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, flags, os, false, stream);
}

cudaError_t launch_kda_decode(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                              const void *q, const void *k, const void *v, const float *g, const float *beta,
                              float *state, void *o, uint32_t flags, const OutSide &os, cudaStream_t stream) {
    return launch_decode_any(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, flags, os, true, stream);
}

}  // namespace gdn
