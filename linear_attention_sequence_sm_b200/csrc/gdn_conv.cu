// gdn_conv.cu -- the input side's short causal convolution with SiLU
// ("Architecture Thread I", "Modern Architecture Improvements": after the
// projections, q and k pass through a short convolution, SiLU and L2
// normalisation, v through a short convolution and SiLU).
//
// Causal and depthwise: one filter of W taps per channel,
//     y[t, c] = act( sum_{j<W} w[c, j] x[t - (W-1) + j, c] ),
// the last tap on the current token.  Inputs before a sequence's first token
// come from its conv state (its W-1 preceding inputs, oldest first) or are
// zero; the state after each sequence (its last W-1 inputs) is returned so
// that decode can continue.
//
// HBM-bound: one read of x and one write of y.  The work is spread for
// memory-level parallelism: a thread owns kConvTok consecutive tokens of the
// packed layout and 4 consecutive channels (one 8- or 16-byte vector per
// token; consecutive threads take consecutive channel groups, so a warp reads
// whole rows), loads its W-1+kConvTok input rows at once (the W-1 halo rows
// come again from L1/L2, not from HBM), and finds the sequence of each of its
// tokens by binary search over the sequence starts, stepping on at sequence
// boundaries.  A tap before its token's sequence start reads the sequence's
// conv state (or zero).  The thread holding a sequence's last token writes
// the sequence's conv state, its last W-1 inputs (reaching into the incoming
// state when the sequence is shorter); a small second kernel passes the state
// of empty sequences through.  Weights of width 4 arrive as one 16-byte load
// per channel: the load/store pipe, not DRAM, is what this kernel runs out of
// first, so it is fed few and wide instructions.  Every index is bounded by
// the sizes, so contents of cu_seqlens that break its contract give
// unspecified values, never an access out of bounds.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kConvTok = 8;         // tokens per thread
constexpr int kConvThreads = 256;
struct ConvArgs {
    const int32_t *cu;  // [N + 1], or NULL: N sequences of seq_len tokens
    int32_t n, seq_len, tokens, channels;
    const void *x;
    const float *w;         // [channels, W]
    const float *state_in;  // [N, channels, W-1] or NULL
    float *state_out;       // [N, channels, W-1] or NULL
    void *y;
    int silu;
};

__device__ __forceinline__ int32_t conv_cu(const ConvArgs &a, int32_t i) {
    return a.cu ? a.cu[i] : i * a.seq_len;
}

// One token's CPT consecutive channels, as loaded: fp32 values, or bf16 kept
// packed (two per 32-bit word) until used.  A row is one 16-byte access
// (8 bytes for bf16 with 4 channels).
template <typename T, int CPT>
struct Row;
template <>
struct Row<float, 4> {
    float v[4];
    __device__ __forceinline__ void load(const float *p) {
        const float4 f = *reinterpret_cast<const float4 *>(p);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
    __device__ __forceinline__ void zero() { v[0] = v[1] = v[2] = v[3] = 0.f; }
    __device__ __forceinline__ float get(int e) const { return v[e]; }
};
template <int CPT>
struct Row<__nv_bfloat16, CPT> {
    uint32_t u[CPT / 2];
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
        if constexpr (CPT == 8) {
            const uint4 q = *reinterpret_cast<const uint4 *>(p);
            u[0] = q.x; u[1] = q.y; u[2] = q.z; u[3] = q.w;
        } else {
            const uint2 q = *reinterpret_cast<const uint2 *>(p);
            u[0] = q.x; u[1] = q.y;
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < CPT / 2; ++i) u[i] = 0u;
    }
    __device__ __forceinline__ float get(int e) const {  // e compile-time in the unrolled loops
        return __uint_as_float((e & 1) ? (u[e >> 1] & 0xffff0000u) : (u[e >> 1] << 16));
    }
};

template <int CPT>
__device__ __forceinline__ void store_row(float *p, const float (&v)[CPT]) {
#pragma unroll
    for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4 *>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
template <int CPT>
__device__ __forceinline__ void store_row(__nv_bfloat16 *p, const float (&v)[CPT]) {
    uint32_t w[CPT / 2];
#pragma unroll
    for (int i = 0; i < CPT / 2; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    if constexpr (CPT == 8) *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    else *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
}

// xr[i].get(e) for a row index known only at run time (the boundary path; the
// compiler keeps the array in registers and selects)
template <typename RowT, int R>
__device__ __forceinline__ float xr_at(const RowT (&xr)[R], int i, int e) {
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < R; ++k) v = (k == i) ? xr[k].get(e) : v;
    return v;
}

// CPT channels per thread (4).
template <typename T, int W, int CPT>
__global__ void __launch_bounds__(kConvThreads, 3) short_conv_kernel(const ConvArgs a) {
    constexpr int H = W - 1, R = H + kConvTok;
    const int64_t cgs = a.channels / CPT;
    const int64_t idx = int64_t(blockIdx.x) * kConvThreads + threadIdx.x;
    const int64_t tg = idx / cgs;
    const int64_t c0 = (idx - tg * cgs) * CPT;
    const int64_t t0 = tg * kConvTok;
    if (t0 >= a.tokens) return;
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y);
    const int64_t C = a.channels;

    // input rows t0 - H .. t0 + kConvTok - 1 (zeros outside 0 .. tokens - 1), all loads first
    Row<T, CPT> xr[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int64_t u = t0 - H + i;
        if (u >= 0 && u < a.tokens) xr[i].load(x + u * C + c0);
        else xr[i].zero();
    }
    float w[CPT][W];
    if constexpr (W == 4) {  // one 16-byte load per channel (rows of 4 taps are 16-byte aligned)
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
            const float4 f = *reinterpret_cast<const float4 *>(a.w + (c0 + e) * 4);
            w[e][0] = f.x; w[e][1] = f.y; w[e][2] = f.z; w[e][3] = f.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < CPT; ++e)
#pragma unroll
            for (int j = 0; j < W; ++j) w[e][j] = a.w[(c0 + e) * W + j];
    }

    // the sequence of the first token: the last n with cu[n] <= t0 (first entry above t0, minus one)
    int32_t lo = 0, hi = a.n + 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi) >> 1;
        if (conv_cu(a, mid) <= t0) lo = mid + 1;
        else hi = mid;
    }
    int32_t n = min(max(lo - 1, 0), a.n - 1);
    int64_t start = conv_cu(a, n), next = conv_cu(a, n + 1);

    auto silu_inplace = [&](float (&out)[CPT]) {
        // SiLU: x / (1 + e^-x) with the fast exponential and division (relative
        // error a few ulp of fp32, far inside the output's rounding; for x below
        // about -88 the denominator is infinite and the result the limit 0)
        if (a.silu)
#pragma unroll
            for (int e = 0; e < CPT; ++e) out[e] = __fdividef(out[e], 1.f + __expf(-out[e]));
    };
    if (t0 - H >= start && t0 + kConvTok <= next && t0 + kConvTok <= a.tokens) {
        // the common case: every token of the group, with all its taps, inside one sequence
        T *yb = y + t0 * C + c0;
#pragma unroll
        for (int p = 0; p < kConvTok; ++p) {
            float out[CPT];
#pragma unroll
            for (int e = 0; e < CPT; ++e) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < W; ++j) acc = fmaf(w[e][j], xr[p + j].get(e), acc);
                out[e] = acc;
            }
            silu_inplace(out);
            store_row<CPT>(yb + int64_t(p) * C, out);
        }
        if (a.state_out && H > 0 && t0 + kConvTok == next)  // the sequence's last H inputs: rows kConvTok ..
#pragma unroll
            for (int e = 0; e < CPT; ++e)
#pragma unroll
                for (int i = 0; i < H; ++i) a.state_out[(int64_t(n) * C + c0 + e) * H + i] = xr[kConvTok + i].get(e);
        return;
    }
    for (int p = 0; p < kConvTok; ++p) {
        const int64_t t = t0 + p;
        if (t >= a.tokens) break;
        while (t >= next && n < a.n - 1) {  // a sequence starts at or before t
            ++n;
            start = next;
            next = conv_cu(a, n + 1);
        }
        float out[CPT];
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const int64_t u = t - H + j;  // tap j of token t
                float v;
                if (u >= start) {
                    v = xr_at(xr, p + j, e);
                } else {
                    const int64_t si = H - (start - u);  // oldest first in the conv state
                    v = (a.state_in && si >= 0 && si < H) ? a.state_in[(int64_t(n) * C + c0 + e) * H + si] : 0.f;
                }
                acc = fmaf(w[e][j], v, acc);
            }
            out[e] = acc;
        }
        silu_inplace(out);
        store_row<CPT>(y + t * C + c0, out);
        if (a.state_out && H > 0 && t == next - 1) {  // the sequence's last H inputs, oldest first
#pragma unroll
            for (int e = 0; e < CPT; ++e)
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const int64_t u = t - H + 1 + i;
                    float v;
                    if (u >= start) {
                        v = xr_at(xr, p + 1 + i, e);
                    } else {
                        const int64_t si = H - (start - u);
                        v = (a.state_in && si >= 0 && si < H) ? a.state_in[(int64_t(n) * C + c0 + e) * H + si] : 0.f;
                    }
                    a.state_out[(int64_t(n) * C + c0 + e) * H + i] = v;
                }
        }
    }
}

// Empty sequences (no thread of the convolution sees them): the conv state
// passes through (zeros without an incoming state).
__global__ void short_conv_empty_kernel(const ConvArgs a, int32_t H) {
    const int32_t n = blockIdx.x;
    if (conv_cu(a, n + 1) != conv_cu(a, n)) return;
    const int64_t per = int64_t(a.channels) * H;
    for (int64_t i = threadIdx.x; i < per; i += blockDim.x)
        a.state_out[int64_t(n) * per + i] = a.state_in ? a.state_in[int64_t(n) * per + i] : 0.f;
}

template <typename T, int CPT>
static cudaError_t launch_conv_as(const ConvArgs &a, int32_t width, cudaStream_t stream) {
    const int64_t threads = (int64_t(a.tokens) + kConvTok - 1) / kConvTok * (a.channels / CPT);
    const unsigned grid = unsigned((threads + kConvThreads - 1) / kConvThreads);
    switch (width) {
        case 1: short_conv_kernel<T, 1, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 2: short_conv_kernel<T, 2, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 3: short_conv_kernel<T, 3, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 4: short_conv_kernel<T, 4, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 5: short_conv_kernel<T, 5, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 6: short_conv_kernel<T, 6, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 7: short_conv_kernel<T, 7, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
        default: short_conv_kernel<T, 8, CPT><<<grid, kConvThreads, 0, stream>>>(a); break;
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_short_conv(int32_t n, int32_t seq_len, const int32_t *cu, int32_t tokens, int32_t channels,
                              int32_t width, int32_t dtype, const void *x, const float *w, const float *state_in,
                              float *state_out, void *y, bool silu, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    if (width < 1 || width > 8 || channels <= 0 || channels % 4 != 0 || tokens < 0) return cudaErrorInvalidValue;
    const int64_t threads = (int64_t(tokens) + kConvTok - 1) / kConvTok * (channels / 4);
    if ((threads + kConvThreads - 1) / kConvThreads > int64_t(0x7fffffff)) return cudaErrorInvalidValue;
    ConvArgs a{cu, n, seq_len, tokens, channels, x, w, state_in, state_out, y, silu ? 1 : 0};
    cudaError_t e = cudaSuccess;
    if (tokens > 0) {
        // (8 bf16 channels per thread measured slower: the registers for 16-byte rows
        // halve the resident warps)
        e = dtype == GDN_DTYPE_BF16 ? launch_conv_as<__nv_bfloat16, 4>(a, width, stream)
                                    : launch_conv_as<float, 4>(a, width, stream);
        if (e != cudaSuccess) return e;
    }
    // (the batched layout has empty sequences only when seq_len is 0)
    if (state_out && width > 1 && (cu || seq_len == 0)) {
        short_conv_empty_kernel<<<unsigned(n), 256, 0, stream>>>(a, width - 1);
        count_launch();
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace gdn
