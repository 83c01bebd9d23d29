// gdn_kda.cu -- Kimi Delta Attention (one decay per key channel) prefill on
// CUDA cores.
//
// "Gated Attention Architectures", section 8 (Kimi Delta Attention),
// "Mathematical Formulation": S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} +
// beta_t k_t v_t^T, o_t = S_t^T q_t with D_t = diag(alpha_t) holding one decay
// per key channel.  With the state stored d_v x d_k (the transpose of that
// page's) the update is S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t
// k_t^T and o_t = S_t q_t; row i of S evolves as
//     s' = alpha_t .* s,   u_i = beta_t (v_i - s' . k_t),   s <- s' + u_i k_t,
//     o_i = s . q_t = s' . q_t + u_i (k_t . q_t).
// With every alpha_t[c] equal this is the gated delta rule.
//
// The kernel walks the tokens in order with the state in registers: a block
// of four warps owns one (sequence, value head, 32-row slice of d_v); a warp
// owns 8 rows, lane l holds key channels l, l + 32, l + 64, l + 96.  Per
// token the 16 dot products of a warp (s' . k and s' . q for its 8 rows) are
// reduced together (column sums across the warp, then a broadcast), and the
// next token's inputs are already in registers.  The chunked tensor-core
// form for this rule needs decay-masked key products, which are not plain
// matrix products (the page's DPLR remark); this kernel is the CUDA-core
// path.  Blocks take the sequences longest first from the schedule.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kKdaWarps = 4;
constexpr int kKdaRows = 8;                       // state rows per warp
constexpr int kKdaSlice = kKdaWarps * kKdaRows;   // rows of d_v per block
constexpr int kKdaMaxE = 4;                       // key channels per lane (d_k <= 128)

__device__ __forceinline__ float kda_warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// One token's inputs as a lane holds them.
struct KdaTok {
    float k[kKdaMaxE], q[kKdaMaxE], g[kKdaMaxE], v[kKdaRows], beta;
};

template <typename T>
__device__ __forceinline__ void kda_load(KdaTok &x, const T *__restrict__ k, const T *__restrict__ q,
                                         const float *__restrict__ g, const T *__restrict__ v,
                                         const float *__restrict__ beta, size_t qk_off, size_t g_off, size_t v_off,
                                         size_t b_off, int lane, int dk, int nrows) {
#pragma unroll
    for (int e = 0; e < kKdaMaxE; ++e) {
        const int c = lane + 32 * e;
        const bool ok = c < dk;
        x.k[e] = ok ? to_f32(k[qk_off + c]) : 0.f;
        x.q[e] = ok ? to_f32(q[qk_off + c]) : 0.f;
        x.g[e] = ok ? g[g_off + c] : 0.f;
    }
#pragma unroll
    for (int rr = 0; rr < kKdaRows; ++rr) x.v[rr] = rr < nrows ? to_f32(v[v_off + rr]) : 0.f;
    x.beta = beta[b_off];
}

template <typename T, uint32_t flags>
__global__ void __launch_bounds__(kKdaWarps * 32, 4)
kda_prefill_kernel(const PrefillArgs a, int n_slices) {
    if (a.sched.hdr->status != GDN_OK) return;
    constexpr bool kL2 = (flags & GDN_FLAG_QK_L2NORM) != 0;
    constexpr bool kLogits = (flags & GDN_FLAG_GATE_LOGITS) != 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hv = a.hv, hk = a.hk, dk = a.dk, dv = a.dv;
    const int bid = blockIdx.x;
    const int rank = bid / (hv * n_slices);
    const int h = (bid / n_slices) % hv;
    const int slice = bid % n_slices;
    const int seq = a.sched.order[rank];
    const int t0 = a.sched.start[seq], len = a.sched.len[seq];
    const int hq = h / (hv / hk);
    const int row0 = slice * kKdaSlice + warp * kKdaRows;
    const int nrows = max(0, min(kKdaRows, dv - row0));
    const size_t sbase = (size_t(seq) * hv + h) * size_t(dv) * dk;
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    T *o = static_cast<T *>(a.o);

    float s[kKdaRows][kKdaMaxE];
#pragma unroll
    for (int rr = 0; rr < kKdaRows; ++rr)
#pragma unroll
        for (int e = 0; e < kKdaMaxE; ++e) {
            const int c = lane + 32 * e;
            s[rr][e] = (a.s0 && rr < nrows && c < dk) ? a.s0[sbase + size_t(row0 + rr) * dk + c] : 0.f;
        }

    auto load_token = [&](KdaTok &x, int t) {
        const size_t tok = size_t(t0 + t);
        kda_load(x, k, q, a.g, v, a.beta, (tok * hk + hq) * dk, (tok * hv + h) * dk, (tok * hv + h) * dv + row0,
                 tok * hv + h, lane, dk, nrows);
    };
    KdaTok cur, nxt;
    if (len > 0) load_token(cur, 0);
    for (int t = 0; t < len; ++t) {
        if (t + 1 < len) load_token(nxt, t + 1);
        float kf[kKdaMaxE], qf[kKdaMaxE], al[kKdaMaxE];
#pragma unroll
        for (int e = 0; e < kKdaMaxE; ++e) {
            kf[e] = cur.k[e];
            qf[e] = cur.q[e];
        }
        if constexpr (kL2) {
            float kk = 0.f, qq = 0.f;
#pragma unroll
            for (int e = 0; e < kKdaMaxE; ++e) {
                kk = fmaf(kf[e], kf[e], kk);
                qq = fmaf(qf[e], qf[e], qq);
            }
            const float ik = inv_l2(kda_warp_sum(kk)), iq = inv_l2(kda_warp_sum(qq));
#pragma unroll
            for (int e = 0; e < kKdaMaxE; ++e) {
                kf[e] *= ik;
                qf[e] *= iq;
            }
        }
#pragma unroll
        for (int e = 0; e < kKdaMaxE; ++e) {
            const float lg = kLogits ? log_sigmoid(cur.g[e]) : cur.g[e];
            al[e] = __expf(fmaxf(lg, kGFloor));
        }
        const float b = kLogits ? sigmoid(cur.beta) : cur.beta;
        float kq = 0.f;
#pragma unroll
        for (int e = 0; e < kKdaMaxE; ++e) kq = fmaf(kf[e], qf[e], kq);
        kq = kda_warp_sum(kq);
        // decayed rows and their partial dot products with k and q
        float red[16];
#pragma unroll
        for (int rr = 0; rr < kKdaRows; ++rr) {
            float p = 0.f, r = 0.f;
#pragma unroll
            for (int e = 0; e < kKdaMaxE; ++e) {
                const float sd = al[e] * s[rr][e];
                s[rr][e] = sd;
                p = fmaf(sd, kf[e], p);
                r = fmaf(sd, qf[e], r);
            }
            red[rr] = p;
            red[kKdaRows + rr] = r;
        }
        const float tot = warp_colsum16(red, lane);  // lanes 2j, 2j + 1: the warp's total of red[j]
        float ov = 0.f;
#pragma unroll
        for (int rr = 0; rr < kKdaRows; ++rr) {
            const float P = __shfl_sync(0xffffffffu, tot, 2 * rr);
            const float R = __shfl_sync(0xffffffffu, tot, 2 * (kKdaRows + rr));
            const float u = b * (cur.v[rr] - P);
#pragma unroll
            for (int e = 0; e < kKdaMaxE; ++e) s[rr][e] = fmaf(u, kf[e], s[rr][e]);
            if (lane == rr) ov = fmaf(u, kq, R);
        }
        if (lane < nrows) o[(size_t(t0 + t) * hv + h) * dv + row0 + lane] = from_f32<T>(ov);
        cur = nxt;
    }
    if (a.s_final) {
#pragma unroll
        for (int rr = 0; rr < kKdaRows; ++rr)
#pragma unroll
            for (int e = 0; e < kKdaMaxE; ++e) {
                const int c = lane + 32 * e;
                if (rr < nrows && c < dk) a.s_final[sbase + size_t(row0 + rr) * dk + c] = s[rr][e];
            }
    }
}

// ---- staged variant: inputs through shared memory, 16 tokens at a time ----
// The direct kernel above waits on each token's loads (an L2 round trip per
// token).  Here the block copies chunks of kKdaTok tokens -- k, q, the
// per-channel g, its 32 rows of v and beta -- into shared memory with
// cp.async one chunk ahead (double-buffered), and each token reads them back
// as short vector loads.  Lane l holds the 4 contiguous channels 4l .. 4l+3.
// Taken when every copy is 16-byte aligned: d_k and d_v multiples of 8.
constexpr int kKdaTok = 16;

template <typename T>
struct KdaStageLayout {
    int k, q, g, v, b, bytes;
    __host__ __device__ KdaStageLayout(int dk) {
        const int esz = int(sizeof(T));
        k = 0;
        q = k + kKdaTok * dk * esz;
        g = q + kKdaTok * dk * esz;
        v = g + kKdaTok * dk * 4;
        b = v + kKdaTok * kKdaSlice * esz;
        bytes = (b + kKdaTok * 4 + 15) / 16 * 16;
    }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void load4v(const float *p, float x[4]) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
__device__ __forceinline__ void load4v(const __nv_bfloat16 *p, float x[4]) {
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

template <typename T, uint32_t flags>
__global__ void __launch_bounds__(kKdaWarps * 32, 4)
kda_prefill_staged_kernel(const PrefillArgs a, int n_slices) {
    if (a.sched.hdr->status != GDN_OK) return;
    extern __shared__ __align__(16) unsigned char kda_smem[];
    constexpr bool kL2 = (flags & GDN_FLAG_QK_L2NORM) != 0;
    constexpr bool kLogits = (flags & GDN_FLAG_GATE_LOGITS) != 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hv = a.hv, hk = a.hk, dk = a.dk, dv = a.dv;
    const int bid = blockIdx.x;
    const int rank = bid / (hv * n_slices);
    const int h = (bid / n_slices) % hv;
    const int slice = bid % n_slices;
    const int seq = a.sched.order[rank];
    const int t0 = a.sched.start[seq], len = a.sched.len[seq];
    const int hq = h / (hv / hk);
    const int rows_blk = min(kKdaSlice, dv - slice * kKdaSlice);  // rows of this block (multiple of 8)
    const int row0 = slice * kKdaSlice + warp * kKdaRows;
    const int nrows = max(0, min(kKdaRows, dv - row0));
    const bool lane_on = 4 * lane < dk;
    const size_t sbase = (size_t(seq) * hv + h) * size_t(dv) * dk;
    const KdaStageLayout<T> L(dk);
    const uint32_t sm0 = uint32_t(__cvta_generic_to_shared(kda_smem));
    const char *qg = static_cast<const char *>(a.q);
    const char *kg = static_cast<const char *>(a.k);
    const char *vg = static_cast<const char *>(a.v);
    const char *gg = reinterpret_cast<const char *>(a.g);
    T *o = static_cast<T *>(a.o);
    constexpr int esz = int(sizeof(T));

    // chunk c (tokens c*kKdaTok ..) of this sequence into stage st
    auto load_chunk = [&](int c, int st) {
        const int tc0 = c * kKdaTok, n = min(kKdaTok, len - tc0);
        const uint32_t base = sm0 + uint32_t(st * L.bytes);
        const int kp = dk * esz / 16, gp = dk * 4 / 16, vp = rows_blk * esz / 16;
        for (int i = tid; i < n * kp; i += kKdaWarps * 32) {
            const int tt = i / kp, pc = i % kp;
            const size_t off = (size_t(t0 + tc0 + tt) * hk + hq) * size_t(dk) * esz + size_t(pc) * 16;
            cp_async16(base + L.k + (tt * dk * esz) + pc * 16, kg + off);
            cp_async16(base + L.q + (tt * dk * esz) + pc * 16, qg + off);
        }
        for (int i = tid; i < n * gp; i += kKdaWarps * 32) {
            const int tt = i / gp, pc = i % gp;
            cp_async16(base + L.g + tt * dk * 4 + pc * 16,
                       gg + (size_t(t0 + tc0 + tt) * hv + h) * size_t(dk) * 4 + size_t(pc) * 16);
        }
        for (int i = tid; i < n * vp; i += kKdaWarps * 32) {
            const int tt = i / vp, pc = i % vp;
            cp_async16(base + L.v + tt * kKdaSlice * esz + pc * 16,
                       vg + ((size_t(t0 + tc0 + tt) * hv + h) * size_t(dv) + slice * kKdaSlice) * esz + size_t(pc) * 16);
        }
        if (tid < n) cp_async4(base + L.b + tid * 4, a.beta + size_t(t0 + tc0 + tid) * hv + h);
    };

    float s[kKdaRows][4];
#pragma unroll
    for (int rr = 0; rr < kKdaRows; ++rr)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = 4 * lane + e;
            s[rr][e] = (a.s0 && rr < nrows && c < dk) ? a.s0[sbase + size_t(row0 + rr) * dk + c] : 0.f;
        }

    const int nch = (len + kKdaTok - 1) / kKdaTok;
    if (nch > 0) load_chunk(0, 0);
    cp_async_commit();
    for (int c = 0; c < nch; ++c) {
        if (c + 1 < nch) load_chunk(c + 1, (c + 1) & 1);
        cp_async_commit();
        cp_async_wait_one();  // chunk c has landed (this thread's copies)
        __syncthreads();      // ... and everyone's
        const unsigned char *stg = kda_smem + (c & 1) * L.bytes;
        const T *sk = reinterpret_cast<const T *>(stg + L.k);
        const T *sq = reinterpret_cast<const T *>(stg + L.q);
        const float *sgt = reinterpret_cast<const float *>(stg + L.g);
        const T *sv = reinterpret_cast<const T *>(stg + L.v);
        const float *sbt = reinterpret_cast<const float *>(stg + L.b);
        const int n = min(kKdaTok, len - c * kKdaTok);
        for (int tt = 0; tt < n; ++tt) {
            float kf[4] = {0.f, 0.f, 0.f, 0.f}, qf[4] = {0.f, 0.f, 0.f, 0.f}, gv[4] = {0.f, 0.f, 0.f, 0.f};
            if (lane_on) {
                load4v(sk + tt * dk + 4 * lane, kf);
                load4v(sq + tt * dk + 4 * lane, qf);
                load4v(sgt + tt * dk + 4 * lane, gv);
            }
            float vr[kKdaRows];
#pragma unroll
            for (int rr = 0; rr < kKdaRows; ++rr) vr[rr] = rr < nrows ? to_f32(sv[tt * kKdaSlice + warp * kKdaRows + rr]) : 0.f;
            const float bt = sbt[tt];
            if constexpr (kL2) {
                float kk = 0.f, qq = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kk = fmaf(kf[e], kf[e], kk);
                    qq = fmaf(qf[e], qf[e], qq);
                }
                const float ik = inv_l2(kda_warp_sum(kk)), iq = inv_l2(kda_warp_sum(qq));
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[e] *= ik;
                    qf[e] *= iq;
                }
            }
            float al[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) al[e] = lane_on ? __expf(fmaxf(kLogits ? log_sigmoid(gv[e]) : gv[e], kGFloor)) : 0.f;
            const float b = kLogits ? sigmoid(bt) : bt;
            float kq = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) kq = fmaf(kf[e], qf[e], kq);
            kq = kda_warp_sum(kq);
            float red[16];
#pragma unroll
            for (int rr = 0; rr < kKdaRows; ++rr) {
                float p = 0.f, r = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float sd = al[e] * s[rr][e];
                    s[rr][e] = sd;
                    p = fmaf(sd, kf[e], p);
                    r = fmaf(sd, qf[e], r);
                }
                red[rr] = p;
                red[kKdaRows + rr] = r;
            }
            const float tot = warp_colsum16(red, lane);
            float ov = 0.f;
#pragma unroll
            for (int rr = 0; rr < kKdaRows; ++rr) {
                const float P = __shfl_sync(0xffffffffu, tot, 2 * rr);
                const float R = __shfl_sync(0xffffffffu, tot, 2 * (kKdaRows + rr));
                const float u = b * (vr[rr] - P);
#pragma unroll
                for (int e = 0; e < 4; ++e) s[rr][e] = fmaf(u, kf[e], s[rr][e]);
                if (lane == rr) ov = fmaf(u, kq, R);
            }
            if (lane < nrows) o[(size_t(t0 + c * kKdaTok + tt) * hv + h) * dv + row0 + lane] = from_f32<T>(ov);
        }
        __syncthreads();  // stage c & 1 is free for chunk c + 2
    }
    if (a.s_final) {
#pragma unroll
        for (int rr = 0; rr < kKdaRows; ++rr)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = 4 * lane + e;
                if (rr < nrows && c < dk) a.s_final[sbase + size_t(row0 + rr) * dk + c] = s[rr][e];
            }
    }
}

template <typename T, uint32_t F>
static void launch_kda_as(const PrefillArgs &a, int n_slices, unsigned grid, cudaStream_t stream) {
    if (a.dk % 8 == 0 && a.dv % 8 == 0) {
        const int bytes = 2 * KdaStageLayout<T>(a.dk).bytes;
        cudaFuncSetAttribute(kda_prefill_staged_kernel<T, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        kda_prefill_staged_kernel<T, F><<<grid, kKdaWarps * 32, bytes, stream>>>(a, n_slices);
    } else {
        kda_prefill_kernel<T, F><<<grid, kKdaWarps * 32, 0, stream>>>(a, n_slices);
    }
}

template <typename T>
static void launch_kda_t(const PrefillArgs &a, int n_slices, unsigned grid, cudaStream_t stream) {
    switch (a.flags & (GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS)) {
        case 0: launch_kda_as<T, 0>(a, n_slices, grid, stream); break;
        case GDN_FLAG_QK_L2NORM: launch_kda_as<T, GDN_FLAG_QK_L2NORM>(a, n_slices, grid, stream); break;
        case GDN_FLAG_GATE_LOGITS: launch_kda_as<T, GDN_FLAG_GATE_LOGITS>(a, n_slices, grid, stream); break;
        default: launch_kda_as<T, GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS>(a, n_slices, grid, stream); break;
    }
}

cudaError_t launch_kda_prefill(const PrefillArgs &a, cudaStream_t stream) {
    if (a.dk > kKdaMaxE * 32) return cudaErrorInvalidValue;
    const int n_slices = (a.dv + kKdaSlice - 1) / kKdaSlice;
    const int64_t blocks = int64_t(a.num_seqs) * a.hv * n_slices;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > INT32_MAX) return cudaErrorInvalidValue;
    if (a.dtype == GDN_DTYPE_BF16)
        launch_kda_t<__nv_bfloat16>(a, n_slices, unsigned(blocks), stream);
    else
        launch_kda_t<float>(a, n_slices, unsigned(blocks), stream);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
