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
// HBM-bound: one read of x and one write of y.  A thread owns a segment of
// kConvSeg tokens of the packed layout and 4 consecutive channels (one 8- or
// 16-byte vector per token, coalesced across the warp).  It finds the
// sequence of its first token by binary search over the sequence starts,
// fills its W-1 token history from the inputs before the segment (or the
// state), and walks its tokens, resetting the history at each sequence start
// and writing the state after each sequence's last token.  Loads run
// kConvPre tokens ahead.  Empty sequences pass their state through in a
// second, small kernel.  Every index is bounded by the sizes, so contents of
// cu_seqlens that break its contract give unspecified values, never an
// access out of bounds.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kConvSeg = 64;      // tokens per thread
constexpr int kConvPre = 8;       // tokens loaded ahead
constexpr int kConvThreads = 128; // 4 channels each: 512 channels per block

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

__device__ __forceinline__ void load4(const float *p, float (&v)[4]) {
    const float4 f = *reinterpret_cast<const float4 *>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void store4(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t *>(&a);
    u.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}

template <typename T, int W>
__global__ void __launch_bounds__(kConvThreads) short_conv_kernel(const ConvArgs a) {
    constexpr int H = W - 1;
    const int64_t c0 = (int64_t(blockIdx.y) * kConvThreads + threadIdx.x) * 4;
    if (c0 >= a.channels) return;
    const int32_t t0 = int32_t(blockIdx.x) * kConvSeg;
    if (t0 >= a.tokens) return;
    const int32_t t1 = min(t0 + kConvSeg, a.tokens);
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y);
    const int64_t C = a.channels;

    float w[4][W];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int j = 0; j < W; ++j) w[e][j] = a.w[(c0 + e) * W + j];

    // the sequence of the first token: the last n with cu[n] <= t0 (first entry above t0, minus one)
    int32_t lo = 0, hi = a.n + 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi) >> 1;
        if (conv_cu(a, mid) <= t0) lo = mid + 1;
        else hi = mid;
    }
    int32_t n = min(max(lo - 1, 0), a.n - 1);
    int32_t start = conv_cu(a, n), next = conv_cu(a, n + 1);

    // history: the W-1 inputs before t0, oldest first
    float hist[H > 0 ? H : 1][4];
#pragma unroll
    for (int i = 0; i < H; ++i) {
        const int32_t u = t0 - H + i;
        if (u >= start && u >= 0) {
            load4(x + int64_t(u) * C + c0, hist[i]);
        } else {
            const int32_t si = H - (start - u);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                hist[i][e] = (a.state_in && si >= 0 && si < H) ? a.state_in[(int64_t(n) * C + c0 + e) * H + si] : 0.f;
        }
    }

    for (int32_t tb = t0; tb < t1; tb += kConvPre) {
        float xv[kConvPre][4];
#pragma unroll
        for (int p = 0; p < kConvPre; ++p)
            if (tb + p < t1) load4(x + int64_t(tb + p) * C + c0, xv[p]);
#pragma unroll
        for (int p = 0; p < kConvPre; ++p) {
            const int32_t t = tb + p;
            if (t >= t1) break;
            while (t >= next && n < a.n - 1) {  // a sequence starts at t: reset from its state
                ++n;
                start = next;
                next = conv_cu(a, n + 1);
#pragma unroll
                for (int i = 0; i < H; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hist[i][e] = a.state_in ? a.state_in[(int64_t(n) * C + c0 + e) * H + i] : 0.f;
            }
            float out[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float acc = w[e][H] * xv[p][e];
#pragma unroll
                for (int j = 0; j < H; ++j) acc = fmaf(w[e][j], hist[j][e], acc);
                out[e] = a.silu ? acc / (1.f + expf(-acc)) : acc;
            }
            store4(y + int64_t(t) * C + c0, out);
#pragma unroll
            for (int i = 0; i + 1 < H; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) hist[i][e] = hist[i + 1][e];
            if (H > 0)
#pragma unroll
                for (int e = 0; e < 4; ++e) hist[H > 0 ? H - 1 : 0][e] = xv[p][e];
            if (t == next - 1 && a.state_out)
#pragma unroll
                for (int i = 0; i < H; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) a.state_out[(int64_t(n) * C + c0 + e) * H + i] = hist[i][e];
        }
    }
}

// empty sequences: state_out = state_in (zeros without one)
__global__ void short_conv_empty_kernel(const ConvArgs a, int32_t hist) {
    const int32_t n = blockIdx.x;
    if (conv_cu(a, n + 1) != conv_cu(a, n)) return;
    const int64_t per = int64_t(a.channels) * hist;
    for (int64_t i = threadIdx.x; i < per; i += blockDim.x)
        a.state_out[int64_t(n) * per + i] = a.state_in ? a.state_in[int64_t(n) * per + i] : 0.f;
}

template <typename T>
static cudaError_t launch_conv_as(const ConvArgs &a, int32_t width, cudaStream_t stream) {
    const dim3 grid(unsigned((a.tokens + kConvSeg - 1) / kConvSeg),
                    unsigned((a.channels / 4 + kConvThreads - 1) / kConvThreads));
    switch (width) {
        case 1: short_conv_kernel<T, 1><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 2: short_conv_kernel<T, 2><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 3: short_conv_kernel<T, 3><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 4: short_conv_kernel<T, 4><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 5: short_conv_kernel<T, 5><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 6: short_conv_kernel<T, 6><<<grid, kConvThreads, 0, stream>>>(a); break;
        case 7: short_conv_kernel<T, 7><<<grid, kConvThreads, 0, stream>>>(a); break;
        default: short_conv_kernel<T, 8><<<grid, kConvThreads, 0, stream>>>(a); break;
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_short_conv(int32_t n, int32_t seq_len, const int32_t *cu, int32_t tokens, int32_t channels,
                              int32_t width, int32_t dtype, const void *x, const float *w, const float *state_in,
                              float *state_out, void *y, bool silu, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    if (width < 1 || width > 8 || channels <= 0 || channels % 4 != 0 || tokens < 0) return cudaErrorInvalidValue;
    if (int64_t(channels) / 4 > int64_t(65535) * kConvThreads) return cudaErrorInvalidValue;
    ConvArgs a{cu, n, seq_len, tokens, channels, x, w, state_in, state_out, y, silu ? 1 : 0};
    cudaError_t e = cudaSuccess;
    if (tokens > 0) {
        e = dtype == GDN_DTYPE_BF16 ? launch_conv_as<__nv_bfloat16>(a, width, stream)
                                    : launch_conv_as<float>(a, width, stream);
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
