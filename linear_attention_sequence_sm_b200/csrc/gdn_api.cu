// gdn_api.cu -- the extern "C" entry points of libgdn.so: argument checks,
// path selection and stream-ordered launches.  No allocation, no sync
// (except gdn_read_device_status, documented as synchronising).
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "gdn_internal.cuh"

namespace gdn {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static thread_local char g_msg[512] = "";

static gdn_status_t fail(gdn_status_t st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return st;
}

// Records the per-thread error text for entry points defined in other files.
gdn_status_t set_error(gdn_status_t st, const char *text) {
    snprintf(g_msg, sizeof(g_msg), "%s", text);
    return st;
}

static gdn_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(GDN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int device_sm_count(int *major) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (major && cudaDeviceGetAttribute(major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
    return sms;
}

static gdn_status_t check_shape(const gdn_shape_t *s) {
    if (!s) return fail(GDN_ERR_INVALID_ARGUMENT, "shape is NULL");
    if (s->batch < 0 || s->seq_len < 0 || s->num_seqs < 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "negative batch/seq_len/num_seqs");
    if (s->num_qk_heads <= 0 || s->num_v_heads <= 0 || s->head_dim_k <= 0 || s->head_dim_v <= 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "heads and head dims must be positive");
    if (s->num_v_heads % s->num_qk_heads != 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "num_v_heads (%d) must be a multiple of num_qk_heads (%d)",
                    s->num_v_heads, s->num_qk_heads);
    if (s->dtype != GDN_DTYPE_F32 && s->dtype != GDN_DTYPE_BF16)
        return fail(GDN_ERR_INVALID_ARGUMENT, "dtype %d is not GDN_DTYPE_F32 or GDN_DTYPE_BF16", s->dtype);
    if ((s->flags & GDN_FLAG_ONE_KERNEL) && (s->flags & GDN_FLAG_SPLIT))
        return fail(GDN_ERR_INVALID_ARGUMENT, "GDN_FLAG_ONE_KERNEL and GDN_FLAG_SPLIT are both set");
    if (s->flags &
        ~(GDN_FLAG_FORCE_SIMT | GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS | GDN_FLAG_ONE_KERNEL | GDN_FLAG_SPLIT))
        return fail(GDN_ERR_INVALID_ARGUMENT, "unknown flag bits 0x%x", s->flags);
    if (s->chunk_size != 16 && s->chunk_size != 32 && s->chunk_size != 64)
        return fail(GDN_ERR_UNSUPPORTED, "chunk_size %d not in {16, 32, 64}", s->chunk_size);
    if (s->head_dim_k > 128 || s->head_dim_v > 128)
        return fail(GDN_ERR_UNSUPPORTED, "head dims above 128 are not supported (d_k=%d, d_v=%d)",
                    s->head_dim_k, s->head_dim_v);
    int64_t tokens = int64_t(s->batch) * s->seq_len;
    if (tokens > INT32_MAX) return fail(GDN_ERR_UNSUPPORTED, "more than 2^31-1 tokens");
    if (int64_t(tokens) * s->num_v_heads * s->head_dim_v > (int64_t(1) << 40))
        return fail(GDN_ERR_UNSUPPORTED, "problem too large");
    return GDN_OK;
}

// Validates an output-side descriptor (NULL = none) and converts it for the
// kernels.
// The two-kernel tensor-core form: asked for with GDN_FLAG_SPLIT, else taken
// where the single kernel does not apply (value heads not a multiple of 4).
static bool wants_split(const gdn_shape_t &s) {
    if (!chunk_split_supported(s) || (s.flags & (GDN_FLAG_ONE_KERNEL | GDN_FLAG_FORCE_SIMT))) return false;
    return (s.flags & GDN_FLAG_SPLIT) || !chunk_tc_supported(s);
}

// The kernel path of a prefill call (GDN kernels; KDA has its own).  One
// function serves the call and the path query, so the two cannot disagree.
static int32_t select_path(const gdn_shape_t &s, int major, bool out_side, size_t workspace_bytes) {
    const int64_t tokens = int64_t(s.batch) * s.seq_len;
    const bool tc_arch = major == 10 && !(s.flags & GDN_FLAG_FORCE_SIMT);
    // the two-kernel form needs the full queried workspace (it keeps every
    // chunk's factors there) and has no output side
    if (tc_arch && tokens > 0 && !out_side && wants_split(s) && workspace_bytes >= split_layout(s).total)
        return GDN_PATH_TC_SPLIT;
    if (tc_arch && chunk_tc_supported(s)) return GDN_PATH_TC_ONE_KERNEL;
    return GDN_PATH_SIMT;
}

static gdn_status_t check_output_side(const gdn_output_side_t *os, OutSide *out) {
    *out = OutSide{nullptr, nullptr, 0.f, 0u};
    if (!os) return GDN_OK;
    const uint32_t known = GDN_OUT_GATE_SILU | GDN_OUT_GATE_SIGMOID | GDN_OUT_ZERO_CENTRED | GDN_OUT_WEIGHT_PER_HEAD;
    if (os->flags & ~known) return fail(GDN_ERR_INVALID_ARGUMENT, "unknown output-side flag bits 0x%x", os->flags);
    const uint32_t gates = os->flags & (GDN_OUT_GATE_SILU | GDN_OUT_GATE_SIGMOID);
    if (os->gate && gates != GDN_OUT_GATE_SILU && gates != GDN_OUT_GATE_SIGMOID)
        return fail(GDN_ERR_INVALID_ARGUMENT, "an output gate needs exactly one of GDN_OUT_GATE_SILU, "
                                              "GDN_OUT_GATE_SIGMOID");
    if (!os->gate && gates) return fail(GDN_ERR_INVALID_ARGUMENT, "a gate activation is set but gate is NULL");
    if (!(os->eps > 0.f) || !(os->eps < 3.0e38f))
        return fail(GDN_ERR_INVALID_ARGUMENT, "output-side eps must be finite and > 0");
    if (os->gate && !aligned16(os->gate)) return fail(GDN_ERR_MISALIGNED, "output gate is not 16-byte aligned");
    if (os->weight && !aligned16(os->weight))
        return fail(GDN_ERR_MISALIGNED, "output-side weight is not 16-byte aligned");
    *out = OutSide{os->weight, os->gate, os->eps, os->flags | kOutOn};
    return GDN_OK;
}

static gdn_status_t chunk_forward_impl(const gdn_shape_t *s, const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, const float *initial_state,
                                       const int32_t *cu_seqlens, const gdn_output_side_t *out_side, void *o,
                                       float *final_state, void *workspace, size_t workspace_bytes,
                                       void *stream_, bool kda = false);
static gdn_status_t decode_impl(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                const void *q, const void *k, const void *v, const float *g, const float *beta,
                                float *state, const gdn_output_side_t *out_side, void *o, uint32_t flags,
                                void *stream_, bool kda);

}  // namespace gdn

using namespace gdn;

extern "C" {

const char *gdn_status_string(gdn_status_t st) {
    switch (st) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARGUMENT: return "GDN_ERR_INVALID_ARGUMENT";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_MISALIGNED: return "GDN_ERR_MISALIGNED";
        case GDN_ERR_WORKSPACE_TOO_SMALL: return "GDN_ERR_WORKSPACE_TOO_SMALL";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_DEVICE_CHECK: return "GDN_ERR_DEVICE_CHECK";
    }
    return "GDN_ERR_UNKNOWN";
}

const char *gdn_last_error_message(void) { return g_msg; }

uint64_t gdn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

gdn_status_t gdn_chunk_forward_workspace_size(const gdn_shape_t *s, size_t *bytes) {
    g_msg[0] = 0;
    if (!bytes) return fail(GDN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    *bytes = wants_split(*s) ? split_layout(*s).total : ws_layout(s->num_seqs).total;
    return GDN_OK;
}

gdn_status_t gdn_chunk_forward_path(const gdn_shape_t *s, size_t workspace_bytes, int32_t *path) {
    g_msg[0] = 0;
    if (!path) return fail(GDN_ERR_INVALID_ARGUMENT, "path is NULL");
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    const size_t need = ws_layout(s->num_seqs).total;
    if (workspace_bytes < need)
        return fail(GDN_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
    int major = 0;
    if (device_sm_count(&major) <= 0) return fail(GDN_ERR_CUDA, "no usable CUDA device");
    *path = select_path(*s, major, false, workspace_bytes);
    return GDN_OK;
}

gdn_status_t gdn_chunk_forward(const gdn_shape_t *s, const void *q, const void *k, const void *v,
                               const float *g, const float *beta, const float *initial_state,
                               const int32_t *cu_seqlens, void *o, float *final_state, void *workspace,
                               size_t workspace_bytes, void *stream_) {
    return chunk_forward_impl(s, q, k, v, g, beta, initial_state, cu_seqlens, nullptr, o, final_state, workspace,
                              workspace_bytes, stream_);
}

gdn_status_t gdn_chunk_forward_out(const gdn_shape_t *s, const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, const float *initial_state,
                                   const int32_t *cu_seqlens, const gdn_output_side_t *out_side, void *o,
                                   float *final_state, void *workspace, size_t workspace_bytes, void *stream_) {
    return chunk_forward_impl(s, q, k, v, g, beta, initial_state, cu_seqlens, out_side, o, final_state, workspace,
                              workspace_bytes, stream_);
}

gdn_status_t gdn_kda_forward_workspace_size(const gdn_shape_t *s, size_t *bytes) {
    g_msg[0] = 0;
    if (!bytes) return fail(GDN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    const bool tc = kda_tc_supported(*s) && !(s->flags & GDN_FLAG_FORCE_SIMT);
    *bytes = tc ? kda_layout(*s).total : ws_layout(s->num_seqs).total;
    return GDN_OK;
}

gdn_status_t gdn_kda_forward(const gdn_shape_t *s, const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                             const gdn_output_side_t *out_side, void *o, float *final_state, void *workspace,
                             size_t workspace_bytes, void *stream_) {
    return chunk_forward_impl(s, q, k, v, g, beta, initial_state, cu_seqlens, out_side, o, final_state, workspace,
                              workspace_bytes, stream_, true);
}

}  // extern "C"

namespace gdn {

static gdn_status_t chunk_forward_impl(const gdn_shape_t *s, const void *q, const void *k, const void *v,
                                       const float *g, const float *beta, const float *initial_state,
                                       const int32_t *cu_seqlens, const gdn_output_side_t *out_side, void *o,
                                       float *final_state, void *workspace, size_t workspace_bytes,
                                       void *stream_, bool kda) {
    g_msg[0] = 0;
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    OutSide out;
    st = check_output_side(out_side, &out);
    if (st != GDN_OK) return st;
    const int64_t tokens = int64_t(s->batch) * s->seq_len;
    if (cu_seqlens) {
        if (s->batch != 1) return fail(GDN_ERR_INVALID_ARGUMENT, "batch must be 1 with cu_seqlens");
    } else if (s->num_seqs != s->batch) {
        return fail(GDN_ERR_INVALID_ARGUMENT, "num_seqs (%d) must equal batch (%d) without cu_seqlens",
                    s->num_seqs, s->batch);
    }
    if (tokens > 0 && (!q || !k || !v || !g || !beta || !o))
        return fail(GDN_ERR_INVALID_ARGUMENT, "q, k, v, g, beta and o must be non-NULL");
    if (!workspace) return fail(GDN_ERR_INVALID_ARGUMENT, "workspace is NULL");
    const WsLayout L = ws_layout(s->num_seqs);
    if (workspace_bytes < L.total)
        return fail(GDN_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
    const void *ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, o, final_state};
    const char *names[] = {"q", "k", "v", "g", "beta", "initial_state", "cu_seqlens", "o", "final_state"};
    for (int i = 0; i < 9; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(GDN_ERR_MISALIGNED, "workspace is not 256-byte aligned");

    int major = 0;
    const int sms = device_sm_count(&major);
    if (sms <= 0) return fail(GDN_ERR_CUDA, "no usable CUDA device");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);

    cudaError_t e = cudaSuccess;

    PrefillArgs a;
    a.num_seqs = s->num_seqs;
    a.hk = s->num_qk_heads;
    a.hv = s->num_v_heads;
    a.dk = s->head_dim_k;
    a.dv = s->head_dim_v;
    a.chunk = s->chunk_size;
    a.dtype = s->dtype;
    a.tokens = int32_t(tokens);
    a.flags = s->flags & (GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS);
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.s0 = initial_state; a.o = o; a.s_final = final_state;
    a.out = out;
    char *ws = static_cast<char *>(workspace);
    a.sched.hdr = reinterpret_cast<WsHeader *>(ws);
    a.sched.order = reinterpret_cast<const int32_t *>(ws + L.order_off);
    a.sched.start = reinterpret_cast<const int32_t *>(ws + L.start_off);
    a.sched.len = reinterpret_cast<const int32_t *>(ws + L.len_off);
    a.sched.chunk_base = nullptr;
    if (s->num_seqs == 0) {  // nothing to compute; the status word still reads GDN_OK
        e = launch_schedule(*s, cu_seqlens, workspace, stream);
        return e == cudaSuccess ? GDN_OK : cuda_fail(e, "schedule kernel launch");
    }

    if (kda) {
        // bf16 with d_k = d_v = 128 and C = 64 runs on the tensor cores when the
        // workspace holds the chunk operands; otherwise the token-order kernel
        const bool kda_tc = major == 10 && tokens > 0 && !(s->flags & GDN_FLAG_FORCE_SIMT) &&
                            kda_tc_supported(*s) && workspace_bytes >= kda_layout(*s).total;
        if (kda_tc) {
            const KdaLayout KL = kda_layout(*s);
            int32_t *cbase = reinterpret_cast<int32_t *>(ws + KL.cbase_off);
            e = launch_schedule(*s, cu_seqlens, workspace, stream, cbase);
            if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
            a.sched.chunk_base = cbase;
            e = launch_kda_tc(a, reinterpret_cast<unsigned char *>(ws + KL.items_off), stream, sms);
            if (e != cudaSuccess) return cuda_fail(e, "tensor-core KDA prefill launch");
        } else {
            e = launch_schedule(*s, cu_seqlens, workspace, stream);
            if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
            e = launch_kda_prefill(a, stream);
            if (e != cudaSuccess) return cuda_fail(e, "KDA prefill launch");
        }
        if (out.flags) {
            e = launch_output_side(o, int32_t(tokens), s->num_v_heads, s->head_dim_v, s->dtype, out, stream);
            if (e != cudaSuccess) return cuda_fail(e, "output-side launch");
        }
        return GDN_OK;
    }
    const int32_t path = select_path(*s, major, out.flags != 0, workspace_bytes);
    const bool use_split = path == GDN_PATH_TC_SPLIT, use_tc = path == GDN_PATH_TC_ONE_KERNEL;
    if (use_split) {
        const SplitLayout SL = split_layout(*s);
        int32_t *cbase = reinterpret_cast<int32_t *>(ws + SL.cbase_off);
        __nv_bfloat16 *tinv = reinterpret_cast<__nv_bfloat16 *>(ws + SL.tinv_off);
        float *gcum = reinterpret_cast<float *>(ws + SL.gcum_off);
        e = launch_schedule(*s, cu_seqlens, workspace, stream, cbase);
        if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
        a.sched.chunk_base = cbase;
        e = launch_chunk_inverse(a, tinv, gcum, SL.max_chunks, stream, sms);
        if (e != cudaSuccess) return cuda_fail(e, "chunk inverse launch");
        e = launch_chunk_chain(a, tinv, gcum, SL.max_chunks, stream, sms);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core chunk loop launch");
        return GDN_OK;
    }
    e = launch_schedule(*s, cu_seqlens, workspace, stream);
    if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
    e = use_tc ? launch_chunk_tc(a, stream, sms) : launch_chunk_simt(a, stream, sms);
    if (e != cudaSuccess) return cuda_fail(e, use_tc ? "tensor-core prefill launch" : "prefill launch");
    // the tensor-core kernel applies the output side itself (with tokens to load)
    if (out.flags && !(use_tc && tokens > 0)) {
        e = launch_output_side(o, int32_t(tokens), s->num_v_heads, s->head_dim_v, s->dtype, out, stream);
        if (e != cudaSuccess) return cuda_fail(e, "output-side launch");
    }
    return GDN_OK;
}

}  // namespace gdn

extern "C" {

gdn_status_t gdn_read_device_status(const void *workspace, int32_t *device_status, void *stream_) {
    g_msg[0] = 0;
    if (!workspace || !device_status) return fail(GDN_ERR_INVALID_ARGUMENT, "NULL argument");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    WsHeader h;
    cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    *device_status = h.status;
    if (h.status != GDN_OK)
        fail(GDN_ERR_DEVICE_CHECK, "cu_seqlens rejected on the device at index %d", h.bad_index);
    return GDN_OK;
}

gdn_status_t gdn_decode_step(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                             const void *q, const void *k, const void *v, const float *g, const float *beta,
                             float *state, void *o, void *stream_) {
    return gdn_decode_step_ex(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, 0u, stream_);
}

gdn_status_t gdn_decode_step_ex(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                const void *q, const void *k, const void *v, const float *g, const float *beta,
                                float *state, void *o, uint32_t flags, void *stream_) {
    return gdn_decode_step_out(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, nullptr, o, flags, stream_);
}

gdn_status_t gdn_decode_step_out(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                 const void *q, const void *k, const void *v, const float *g, const float *beta,
                                 float *state, const gdn_output_side_t *out_side, void *o, uint32_t flags,
                                 void *stream_) {
    return decode_impl(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, out_side, o, flags, stream_, false);
}

gdn_status_t gdn_kda_decode_step(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                 const void *q, const void *k, const void *v, const float *g, const float *beta,
                                 float *state, const gdn_output_side_t *out_side, void *o, uint32_t flags,
                                 void *stream_) {
    return decode_impl(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, out_side, o, flags, stream_, true);
}

}  // extern "C"

namespace gdn {

static gdn_status_t decode_impl(int32_t n, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                                const void *q, const void *k, const void *v, const float *g, const float *beta,
                                float *state, const gdn_output_side_t *out_side, void *o, uint32_t flags,
                                void *stream_, bool kda) {
    g_msg[0] = 0;
    OutSide out;
    gdn_status_t st = check_output_side(out_side, &out);
    if (st != GDN_OK) return st;
    if (flags & ~(GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS))
        return fail(GDN_ERR_INVALID_ARGUMENT, "unknown decode flag bits 0x%x", flags);
    if (n < 0 || hk <= 0 || hv <= 0 || dk <= 0 || dv <= 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "bad decode shape");
    if (hv % hk != 0) return fail(GDN_ERR_INVALID_ARGUMENT, "num_v_heads must be a multiple of num_qk_heads");
    if (dtype != GDN_DTYPE_F32 && dtype != GDN_DTYPE_BF16)
        return fail(GDN_ERR_INVALID_ARGUMENT, "dtype %d is not GDN_DTYPE_F32 or GDN_DTYPE_BF16", dtype);
    if (dk > 256) return fail(GDN_ERR_UNSUPPORTED, "decode supports d_k <= 256 (got %d)", dk);
    if (out.flags && dv > 256)
        return fail(GDN_ERR_UNSUPPORTED, "decode with an output side supports d_v <= 256 (got %d)", dv);
    if (n == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !o)
        return fail(GDN_ERR_INVALID_ARGUMENT, "decode pointers must be non-NULL");
    const void *ptrs[] = {q, k, v, g, beta, state, o};
    const char *names[] = {"q", "k", "v", "g", "beta", "state", "o"};
    for (int i = 0; i < 7; ++i)
        if (!aligned16(ptrs[i])) return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if (int64_t(n) * hv * dv * dk > (int64_t(1) << 40)) return fail(GDN_ERR_UNSUPPORTED, "state too large");
    cudaError_t e = kda ? launch_kda_decode(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, flags, out,
                                            static_cast<cudaStream_t>(stream_))
                        : launch_decode(n, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, o, flags, out,
                                        static_cast<cudaStream_t>(stream_));
    if (e != cudaSuccess) return cuda_fail(e, kda ? "KDA decode launch" : "decode launch");
    return GDN_OK;
}

}  // namespace gdn

extern "C" {

gdn_status_t gdn_decode_multi(int32_t n, int32_t ntok, int32_t hk, int32_t hv, int32_t dk, int32_t dv, int32_t dtype,
                              const void *q, const void *k, const void *v, const float *g, const float *beta,
                              const float *state, float *snapshots, void *o, uint32_t flags, void *stream_) {
    g_msg[0] = 0;
    if (flags & ~(GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS))
        return fail(GDN_ERR_INVALID_ARGUMENT, "unknown flag bits 0x%x", flags);
    if (n < 0 || hk <= 0 || hv <= 0 || dk <= 0 || dv <= 0 || ntok <= 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "bad multi-token decode shape");
    if (hv % hk != 0) return fail(GDN_ERR_INVALID_ARGUMENT, "num_v_heads must be a multiple of num_qk_heads");
    if (dtype != GDN_DTYPE_F32 && dtype != GDN_DTYPE_BF16)
        return fail(GDN_ERR_INVALID_ARGUMENT, "dtype %d is not GDN_DTYPE_F32 or GDN_DTYPE_BF16", dtype);
    if (dk != 128) return fail(GDN_ERR_UNSUPPORTED, "multi-token decode supports d_k = 128 (got %d)", dk);
    if (ntok > 16) return fail(GDN_ERR_UNSUPPORTED, "multi-token decode takes at most 16 tokens (got %d)", ntok);
    if (n == 0) return GDN_OK;
    const void *ptrs[] = {q, k, v, g, beta, state, snapshots, o};
    const char *names[] = {"q", "k", "v", "g", "beta", "state", "snapshots", "o"};
    for (int i = 0; i < 8; ++i) {
        if (!ptrs[i]) return fail(GDN_ERR_INVALID_ARGUMENT, "%s is NULL", names[i]);
        if (!aligned16(ptrs[i])) return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    }
    if (int64_t(n) * ntok * hv * dv * dk > (int64_t(1) << 40)) return fail(GDN_ERR_UNSUPPORTED, "too large");
    cudaError_t e = launch_decode_multi(n, ntok, hk, hv, dk, dv, dtype, q, k, v, g, beta, state, snapshots, o,
                                        flags, static_cast<cudaStream_t>(stream_));
    if (e != cudaSuccess) return cuda_fail(e, "multi-token decode launch");
    return GDN_OK;
}

gdn_status_t gdn_decode_commit(int32_t n, int32_t ntok, int32_t hv, int32_t dk, int32_t dv, const float *snapshots,
                               const int32_t *accepted, float *state, int32_t *bad_count, void *stream_) {
    g_msg[0] = 0;
    if (n < 0 || hv <= 0 || dk <= 0 || dv <= 0 || ntok <= 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "bad commit shape");
    if ((int64_t(dv) * dk) % 4 != 0) return fail(GDN_ERR_UNSUPPORTED, "d_v * d_k must be a multiple of 4");
    if (n == 0) return GDN_OK;
    if (!snapshots || !accepted || !state) return fail(GDN_ERR_INVALID_ARGUMENT, "NULL argument");
    if (!aligned16(snapshots) || !aligned16(state)) return fail(GDN_ERR_MISALIGNED, "state or snapshots misaligned");
    cudaError_t e = launch_decode_commit(n, ntok, hv, dk, dv, snapshots, accepted, state, bad_count,
                                         static_cast<cudaStream_t>(stream_));
    if (e != cudaSuccess) return cuda_fail(e, "commit launch");
    return GDN_OK;
}

}  // extern "C"

extern "C" {

static size_t bwd_sched_bytes(const gdn_shape_t *s) { return (ws_layout(s->num_seqs).total + 255) / 256 * 256; }

gdn_status_t gdn_chunk_backward_workspace_size(const gdn_shape_t *s, size_t *bytes) {
    g_msg[0] = 0;
    if (!bytes) return fail(GDN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    const int64_t tokens = int64_t(s->batch) * s->seq_len;
    if (backward_tc_supported(*s) && !(s->flags & GDN_FLAG_FORCE_SIMT)) {
        *bytes = bwd_tc_layout(*s).total;
        return GDN_OK;
    }
    *bytes = bwd_sched_bytes(s) +
             backward_ckpt_bytes(int32_t(tokens), s->num_seqs, s->num_v_heads, s->head_dim_k, s->head_dim_v);
    return GDN_OK;
}

gdn_status_t gdn_chunk_backward(const gdn_shape_t *s, const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                                const void *d_o, const float *d_final_state, float *dq, float *dk, float *dv,
                                float *dg, float *dbeta, float *d_initial_state, void *workspace,
                                size_t workspace_bytes, void *stream_) {
    g_msg[0] = 0;
    gdn_status_t st = check_shape(s);
    if (st != GDN_OK) return st;
    if (s->flags & (GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS))
        return fail(GDN_ERR_UNSUPPORTED, "the backward takes prepared inputs (no input-side flags)");
    if (s->flags & (GDN_FLAG_ONE_KERNEL | GDN_FLAG_SPLIT))
        return fail(GDN_ERR_UNSUPPORTED, "GDN_FLAG_ONE_KERNEL and GDN_FLAG_SPLIT select forward paths");
    const int64_t tokens = int64_t(s->batch) * s->seq_len;
    if (cu_seqlens) {
        if (s->batch != 1) return fail(GDN_ERR_INVALID_ARGUMENT, "batch must be 1 with cu_seqlens");
    } else if (s->num_seqs != s->batch) {
        return fail(GDN_ERR_INVALID_ARGUMENT, "num_seqs (%d) must equal batch (%d) without cu_seqlens",
                    s->num_seqs, s->batch);
    }
    if (tokens > 0 && (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta))
        return fail(GDN_ERR_INVALID_ARGUMENT, "inputs, d_o and the gradient outputs must be non-NULL");
    if (!workspace) return fail(GDN_ERR_INVALID_ARGUMENT, "workspace is NULL");
    size_t need = 0;
    gdn_chunk_backward_workspace_size(s, &need);
    if (workspace_bytes < need)
        return fail(GDN_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
    const void *ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state, dq, dk, dv, dg, dbeta,
                          d_initial_state};
    const char *names[] = {"q", "k", "v", "g", "beta", "initial_state", "cu_seqlens", "d_o", "d_final_state",
                           "dq", "dk", "dv", "dg", "dbeta", "d_initial_state"};
    for (int i = 0; i < 15; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(GDN_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    int major = 0;
    const int sms = device_sm_count(&major);
    if (sms <= 0) return fail(GDN_ERR_CUDA, "no usable CUDA device");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // the tensor-core form (bf16, d = 128) on sm_100 unless GDN_FLAG_FORCE_SIMT; its
    // workspace size is what gdn_chunk_backward_workspace_size reports for such shapes
    const bool tc = major == 10 && backward_tc_supported(*s) && !(s->flags & GDN_FLAG_FORCE_SIMT);
    const BwdTcLayout TL = bwd_tc_layout(*s);
    char *ws = static_cast<char *>(workspace);
    cudaError_t e = tc ? launch_schedule(*s, cu_seqlens, workspace, stream, reinterpret_cast<int32_t *>(ws + TL.cbase_off))
                       : launch_schedule(*s, cu_seqlens, workspace, stream);
    if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
    if (tokens > 0) {
        const size_t qk = size_t(tokens) * s->num_qk_heads * s->head_dim_k * sizeof(float);
        const size_t gb = size_t(tokens) * s->num_v_heads * sizeof(float);
        // the tensor-core form writes dq and dk whole (one CTA per chunk and q/k head)
        if ((!tc && ((e = cudaMemsetAsync(dq, 0, qk, stream)) != cudaSuccess ||
                     (e = cudaMemsetAsync(dk, 0, qk, stream)) != cudaSuccess)) ||
            (e = cudaMemsetAsync(dg, 0, gb, stream)) != cudaSuccess ||
            (e = cudaMemsetAsync(dbeta, 0, gb, stream)) != cudaSuccess)
            return cuda_fail(e, "clearing the gradient accumulators");
    }
    const WsLayout L = ws_layout(s->num_seqs);
    PrefillArgs a;
    a.num_seqs = s->num_seqs;
    a.hk = s->num_qk_heads;
    a.hv = s->num_v_heads;
    a.dk = s->head_dim_k;
    a.dv = s->head_dim_v;
    a.chunk = s->chunk_size;
    a.dtype = s->dtype;
    a.tokens = int32_t(tokens);
    a.flags = 0;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.s0 = initial_state; a.o = nullptr; a.s_final = nullptr;
    a.out = OutSide{nullptr, nullptr, 0.f, 0u};
    a.sched.hdr = reinterpret_cast<WsHeader *>(ws);
    a.sched.order = reinterpret_cast<const int32_t *>(ws + L.order_off);
    a.sched.start = reinterpret_cast<const int32_t *>(ws + L.start_off);
    a.sched.len = reinterpret_cast<const int32_t *>(ws + L.len_off);
    a.sched.chunk_base = nullptr;
    if (s->num_seqs == 0) return GDN_OK;
    if (tc) {
        a.sched.chunk_base = reinterpret_cast<const int32_t *>(ws + TL.cbase_off);
        e = launch_backward_tc(a, d_o, d_final_state, dq, dk, dv, dg, dbeta, d_initial_state, nullptr,
                               reinterpret_cast<unsigned char *>(ws), TL, stream, sms);
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
        return GDN_OK;
    }
    float *ckpt = reinterpret_cast<float *>(ws + bwd_sched_bytes(s));
    e = launch_chunk_backward(a, d_o, d_final_state, dq, dk, dv, dg, dbeta, d_initial_state, ckpt, stream);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return GDN_OK;
}

}  // extern "C"

extern "C" {

gdn_status_t gdn_short_conv(int32_t num_seqs, int32_t seq_len, const int32_t *cu_seqlens, int64_t tokens,
                            int32_t channels, int32_t width, int32_t dtype, const void *x, const float *weight,
                            const float *state_in, float *state_out, void *y, uint32_t flags, void *stream_) {
    g_msg[0] = 0;
    if (flags & ~GDN_CONV_SILU) return fail(GDN_ERR_INVALID_ARGUMENT, "unknown convolution flag bits 0x%x", flags);
    if (num_seqs < 0 || tokens < 0 || channels <= 0)
        return fail(GDN_ERR_INVALID_ARGUMENT, "bad convolution shape");
    if (dtype != GDN_DTYPE_F32 && dtype != GDN_DTYPE_BF16)
        return fail(GDN_ERR_INVALID_ARGUMENT, "dtype %d is not GDN_DTYPE_F32 or GDN_DTYPE_BF16", dtype);
    if (width < 1 || width > 8) return fail(GDN_ERR_UNSUPPORTED, "convolution width %d not in 1..8", width);
    if (channels % 4 != 0) return fail(GDN_ERR_UNSUPPORTED, "channels (%d) must be a multiple of 4", channels);
    if (tokens > INT32_MAX) return fail(GDN_ERR_UNSUPPORTED, "more than 2^31-1 tokens");
    // at most one thread per token and 4 channels, 256 threads a block, in a 1-D grid
    if (tokens * (int64_t(channels) / 4) / 256 >= int64_t(INT32_MAX))
        return fail(GDN_ERR_UNSUPPORTED, "too many (token, channel) groups: %lld tokens x %d channels",
                    static_cast<long long>(tokens), channels);
    if (!cu_seqlens && int64_t(num_seqs) * seq_len != tokens)
        return fail(GDN_ERR_INVALID_ARGUMENT, "tokens (%lld) must equal num_seqs * seq_len without cu_seqlens",
                    (long long)tokens);
    if (num_seqs == 0 && tokens > 0) return fail(GDN_ERR_INVALID_ARGUMENT, "tokens without sequences");
    if (num_seqs == 0) return GDN_OK;
    if (!weight || (tokens > 0 && (!x || !y)))
        return fail(GDN_ERR_INVALID_ARGUMENT, "x, weight and y must be non-NULL");
    if (tokens > 0 && x == y) return fail(GDN_ERR_INVALID_ARGUMENT, "y must not alias x");
    if (width > 1 && state_in && state_in == state_out)
        return fail(GDN_ERR_INVALID_ARGUMENT, "state_out must not alias state_in");
    const void *ptrs[] = {x, weight, state_in, state_out, y, cu_seqlens};
    const char *names[] = {"x", "weight", "state_in", "state_out", "y", "cu_seqlens"};
    for (int i = 0; i < 6; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if (device_sm_count(nullptr) <= 0) return fail(GDN_ERR_CUDA, "no usable CUDA device");
    cudaError_t e = launch_short_conv(num_seqs, seq_len, cu_seqlens, int32_t(tokens), channels, width, dtype, x,
                                      weight, state_in, state_out, y, (flags & GDN_CONV_SILU) != 0,
                                      static_cast<cudaStream_t>(stream_));
    if (e != cudaSuccess) return cuda_fail(e, "short convolution launch");
    return GDN_OK;
}

}  // extern "C"
