// gdn_internal.cuh -- declarations shared by the translation units of
// libgdn.so (host launch layer and kernels).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Floor applied to the log-decay g inside the kernels: exp(-20) ~ 2.1e-9 is
// below fp32 resolution relative to the state, and the floor keeps the
// chunk-local prefix sums of g finite (g = -inf would give -inf - -inf).
constexpr float kGFloor = -20.0f;

// The input side of the mixer (GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM):
// log sigmoid(a) as -log1p(e^-a) for a >= 0 and a - log1p(e^a) below (the same
// function, each form free of overflow); sigmoid(b); and the reciprocal of
// max(||x||_2, 1e-12) from the sum of squares.
__device__ __forceinline__ float log_sigmoid(float a) { return a >= 0.f ? -log1pf(expf(-a)) : a - log1pf(expf(a)); }
__device__ __forceinline__ float sigmoid(float b) { return 1.f / (1.f + expf(-b)); }
__device__ __forceinline__ float inv_l2(float sum_sq) { return 1.f / fmaxf(sqrtf(sum_sq), 1e-12f); }
// The same two gates with the fast exponential and logarithm intrinsics, for
// the bf16 tensor-core path: their absolute error in log sigmoid is about
// 1e-7, far below that path's bf16 rounding.
__device__ __forceinline__ float log_sigmoid_fast(float a) {
    return a >= 0.f ? -__logf(1.f + __expf(-a)) : a - __logf(1.f + __expf(a));
}
__device__ __forceinline__ float sigmoid_fast(float b) { return __fdividef(1.f, 1.f + __expf(-b)); }

// ---------------------------------------------------------------------------
// Workspace layout of gdn_chunk_forward (all offsets 256-byte aligned).
//   [0, 256)              WsHeader
//   seq_order [N]         sequences, longest first (ties by index)
//   seq_start [N]         first token of each sequence
//   seq_len   [N]         tokens of each sequence
// ---------------------------------------------------------------------------
struct WsHeader {
    int32_t status;        // GDN_OK or GDN_ERR_DEVICE_CHECK
    int32_t bad_index;     // first offending cu_seqlens index (diagnostics)
    uint32_t next_unit;    // work counter of the persistent prefill kernels
    int32_t num_seqs;
    int32_t total_chunks;  // chunks of all sequences (the two-kernel path: chunk_base filled)
    int32_t pad[59];
};
static_assert(sizeof(WsHeader) == 256, "header must be 256 bytes");

struct WsLayout {
    size_t order_off, start_off, len_off, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int32_t num_seqs) {
    WsLayout L;
    size_t off = 256;
    L.order_off = off; off = align256(off + 4 * size_t(num_seqs));
    L.start_off = off; off = align256(off + 4 * size_t(num_seqs));
    L.len_off = off;   off = align256(off + 4 * size_t(num_seqs));
    L.total = off;
    return L;
}

// The two-kernel tensor-core path appends to the schedule tables
//   chunk_base [N + 1]    first chunk of each sequence in the chunk order
//                         (sequence by sequence, chunks in token order);
//                         chunk_base[N] = total chunks
//   tinv                  per (chunk, value head) T' = T diag(beta gamma) and
//                         T'' = T diag(beta) of the chunk's WY factor
//                         T = (I + A)^-1, bf16 row-major, [max_chunks][Hv][2][64][64]
//   gcum                  per (chunk, value head) the chunk-local prefix sums G
//                         of the log-decay (tokens past the end carry g = 0),
//                         fp32 [max_chunks][Hv][64]
// max_chunks bounds the chunk count for the shape: (tokens + 63 N) / 64 (each
// sequence adds at most one partial chunk).
struct SplitLayout {
    WsLayout sched;
    size_t cbase_off, tinv_off, gcum_off, total;
    int64_t max_chunks;
};

inline int64_t max_chunks_bound(const gdn_shape_t &s) {
    // sum over sequences of ceil(L_n / 64) <= (sum L_n + 63 N) / 64 (also
    // covers the batched layout: B ceil(T / 64) <= (B T + 63 B) / 64)
    return (int64_t(s.batch) * s.seq_len + 63 * int64_t(s.num_seqs)) / 64;
}

inline SplitLayout split_layout(const gdn_shape_t &s) {
    SplitLayout L;
    L.sched = ws_layout(s.num_seqs);
    size_t off = L.sched.total;
    L.cbase_off = off; off = align256(off + 4 * (size_t(s.num_seqs) + 1));
    off = (off + 1023) & ~size_t(1023);
    L.tinv_off = off;
    L.max_chunks = max_chunks_bound(s);
    off += size_t(L.max_chunks) * size_t(s.num_v_heads) * 2 * 64 * 64 * 2;
    L.gcum_off = off;
    off += size_t(L.max_chunks) * size_t(s.num_v_heads) * 64 * 4;
    L.total = align256(off);
    return L;
}

// Sequence n holding global chunk gc: the largest n < N with chunk_base[n] <= gc.
__device__ __forceinline__ int chunk_sequence(const int32_t *chunk_base, int num_seqs, int gc) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_base[mid] <= gc) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Workspace of the tensor-core KDA prefill (gdn_kda_tc.cu): the schedule
// tables, chunk_base, then per (chunk, value head) the chunk loop's operands
// (K+, Q+, K^, T'', P as bf16 tiles and e^G_last), 66,048 bytes each.
struct KdaLayout {
    WsLayout sched;
    size_t cbase_off, items_off, total;
    int64_t max_chunks;
};
KdaLayout kda_layout(const gdn_shape_t &s);
bool kda_tc_supported(const gdn_shape_t &s);

// Pointers into the workspace, as the kernels see them.
struct Sched {
    WsHeader *hdr;
    const int32_t *order;
    const int32_t *start;
    const int32_t *len;
    const int32_t *chunk_base;  // two-kernel path only (else NULL)
};

// Element access for the two storage types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Sets the per-thread error text returned by gdn_last_error_message
// (defined in gdn_api.cu) and returns `st`.
gdn_status_t set_error(gdn_status_t st, const char *text);

// Launch counter (defined in gdn_api.cu).
void count_launch();

// Prefill schedule: validates cu_seqlens (or synthesises the batched layout)
// and fills the workspace tables (with chunk_base when it is not NULL).  One
// block.
cudaError_t launch_schedule(const gdn_shape_t &s, const int32_t *cu_seqlens, void *workspace,
                            cudaStream_t stream, int32_t *chunk_base = nullptr);

// Column sums over a warp of 16 values per lane, transposed: afterwards lanes
// 2t and 2t + 1 return the sum over all 32 lanes of x[t] (t = 0..15).  Four
// halving exchanges (each lane keeps the half of its values selected by its
// lane bit and adds its partner's copy of that half) and a final pairwise
// add: 16 shuffles instead of the 80 of 16 separate reductions.
__device__ __forceinline__ float warp_colsum16(float (&x)[16], int lane) {
#pragma unroll
    for (int n = 8, bit = 16; n >= 1; n >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int m = 0; m < n; ++m) {
            const float send = up ? x[m] : x[m + n];
            const float keep = up ? x[m + n] : x[m];
            x[m] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    return x[0] + __shfl_xor_sync(0xffffffffu, x[0], 1);
}

// The output side as the kernels see it (gdn_output_side_t plus an enable
// bit): y = o / sqrt(mean(o^2) + eps) * s * act(z).
constexpr uint32_t kOutOn = 1u << 31;
struct OutSide {
    const float *w;   // scale, or NULL
    const void *z;    // gate, or NULL
    float eps;
    uint32_t flags;   // GDN_OUT_* | kOutOn; 0 = no output side
};

// The scale s_i of row channel i of value head h.
__device__ __forceinline__ float out_scale(const OutSide &os, int h, int i, int dv) {
    const float w = os.w ? os.w[((os.flags & GDN_OUT_WEIGHT_PER_HEAD) ? size_t(h) * dv : 0) + i]
                         : ((os.flags & GDN_OUT_ZERO_CENTRED) ? 0.f : 1.f);
    return (os.flags & GDN_OUT_ZERO_CENTRED) ? 1.f + w : w;
}

// act(z) for the gate kinds (1 without a gate).
__device__ __forceinline__ float out_gate(uint32_t flags, float z) {
    if (flags & GDN_OUT_GATE_SILU) return z * sigmoid(z);
    if (flags & GDN_OUT_GATE_SIGMOID) return sigmoid(z);
    return 1.f;
}

// The same for bf16 outputs, with sigmoid(z) = 1/2 + tanh(z/2)/2 through the
// hardware tanh approximation (one special-function instruction instead of an
// exponential and a reciprocal): absolute error in sigmoid about 2^-12, below
// the bf16 rounding of the result.
__device__ __forceinline__ float out_gate_fast(uint32_t flags, float z) {
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(0.5f * z));
    const float sg = fmaf(0.5f, th, 0.5f);
    if (flags & GDN_OUT_GATE_SILU) return z * sg;
    if (flags & GDN_OUT_GATE_SIGMOID) return sg;
    return 1.f;
}

struct PrefillArgs {
    int32_t num_seqs, hk, hv, dk, dv, chunk, dtype;
    int32_t tokens;  // rows of q, k, v, o (B * T, or the packed total)
    uint32_t flags;  // GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS (input side in the kernels)
    const void *q, *k, *v;
    const float *g, *beta, *s0;
    void *o;
    float *s_final;
    Sched sched;
    OutSide out;     // output side (flags 0: none)
};

// fp32 CUDA-core chunkwise kernel (any dtype, d_k, d_v <= 128, C in {16,32,64}).
cudaError_t launch_chunk_simt(const PrefillArgs &a, cudaStream_t stream, int num_sms);

// Tensor maps (gdn_tma.cu): gates [tokens, heads] fp32 in boxes of 4 heads x
// 64 tokens; [tokens, heads, 128] bf16 in boxes of 64 x 1 x 64, 128-byte
// swizzle (out: 128 x 1 x 64, no swizzle); rows x 64 bf16 tiles of 64 rows,
// 128-byte swizzle.
bool make_gate_map(CUtensorMap *map, const float *base, int heads, int tokens);
bool make_map(CUtensorMap *map, const void *base, int heads, int tokens, bool out = false);
bool make_tile_map(CUtensorMap *map, const void *base, int64_t rows);

// Tensor-core chunkwise kernel (bf16, d = 128, C = 64) as one kernel.
cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t stream, int num_sms);
bool chunk_tc_supported(const gdn_shape_t &s);

// The two-kernel tensor-core path (bf16, d = 128, C = 64, any head counts):
// the chunk inverses T for all chunks (gdn_chunk_inv.cu), then the
// state-carrying chunk loop that reads them (gdn_chunk_chain.cu).  Both are
// programmatic dependents of the schedule kernel, which fills chunk_base.
bool chunk_split_supported(const gdn_shape_t &s);
cudaError_t launch_chunk_inverse(const PrefillArgs &a, __nv_bfloat16 *tinv, float *gcum, int64_t max_chunks,
                                 cudaStream_t stream, int num_sms);
cudaError_t launch_chunk_chain(const PrefillArgs &a, const __nv_bfloat16 *tinv, const float *gcum,
                               int64_t max_chunks, cudaStream_t stream, int num_sms);
// The tensor-core KDA prefill: factor kernel, then chunk loop (gdn_kda_tc.cu).
cudaError_t launch_kda_tc(const PrefillArgs &a, unsigned char *items, cudaStream_t stream, int num_sms);

// The tensor-core backward (gdn_backward_tc.cu; bf16, d_k = d_v = 128): the
// schedule tables, chunk_base, then per (chunk, value head) the factor item
// (212,992 bytes) and two checkpoints (65,536 bytes each).
struct BwdTcLayout {
    WsLayout sched;
    size_t cbase_off, items_off, ck_s_off, ck_ds_off, total;
    int64_t max_chunks;
};
bool backward_tc_supported(const gdn_shape_t &s);
BwdTcLayout bwd_tc_layout(const gdn_shape_t &s);
// Factors, chains and gradients after the schedule kernel (which must fill
// chunk_base); s_final, if not NULL, receives the final states.
cudaError_t launch_backward_tc(const PrefillArgs &a, const void *dO, const float *dSf, float *dq, float *dk,
                               float *dv, float *dg, float *dbeta, float *dS0, float *s_final, unsigned char *ws,
                               const BwdTcLayout &L, cudaStream_t stream, int num_sms);

// The output side as its own pass over o, in place (for the CUDA-core prefill,
// whose blocks each own a slice of d_v).
cudaError_t launch_output_side(void *o, int32_t tokens, int32_t hv, int32_t dv, int32_t dtype, const OutSide &os,
                               cudaStream_t stream);

// Kimi Delta Attention: prefill (token order, CUDA cores) and decode.
cudaError_t launch_kda_prefill(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_kda_decode(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                              const void *q, const void *k, const void *v, const float *g, const float *beta,
                              float *state, void *o, uint32_t flags, const OutSide &os, cudaStream_t stream);

// Multi-token decode (draft verification) and its commit.
cudaError_t launch_decode_multi(int32_t n, int32_t ntok, int32_t hk, int32_t hv, int32_t dk, int32_t dv,
                                int32_t dtype, const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *state, float *snap, void *o, uint32_t flags,
                                cudaStream_t stream);
cudaError_t launch_decode_commit(int32_t n, int32_t ntok, int32_t hv, int32_t dk, int32_t dv, const float *snap,
                                 const int32_t *accepted, float *state, int32_t *bad, cudaStream_t stream);

// The input side's short causal convolution (+ SiLU) and its conv states.
cudaError_t launch_short_conv(int32_t n, int32_t seq_len, const int32_t *cu, int32_t tokens, int32_t channels,
                              int32_t width, int32_t dtype, const void *x, const float *w, const float *state_in,
                              float *state_out, void *y, bool silu, cudaStream_t stream);

// Backward (training): checkpoint bytes and the kernel.
size_t backward_ckpt_bytes(int32_t tokens, int32_t num_seqs, int32_t hv, int32_t dk, int32_t dv);
cudaError_t launch_chunk_backward(const PrefillArgs &a, const void *dO, const float *dSf, float *dq, float *dk,
                                  float *dv, float *dg, float *dbeta, float *dS0, float *ckpt, cudaStream_t stream);

// Decode step.
cudaError_t launch_decode(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                          const void *q, const void *k, const void *v, const float *g, const float *beta,
                          float *state, void *o, uint32_t flags, const OutSide &os, cudaStream_t stream);

}  // namespace gdn
