// gdn_kda_tc.cu -- Kimi Delta Attention prefill on the tensor cores, in the
// chunkwise WY form ("Gated Attention Architectures", section 8, "Mathematical
// Formulation": DeltaNet's WY representation with the channel-wise decay
// absorbed into the keys).
//
// Per chunk of L <= 64 tokens with start state S (d_v x d_k) and the
// per-channel cumulative log-decay G_r[c] = g_0[c] + ... + g_r[c]:
//   A_rj = beta_r sum_c k_r[c] k_j[c] e^(G_r[c] - G_j[c])        (j < r)
//   P_rj =        sum_c q_r[c] k_j[c] e^(G_r[c] - G_j[c])        (j <= r)
//   T = (I + A)^-1,  K+ = K (.) e^G,  Q+ = Q (.) e^G,  K^ = K (.) e^(G_last - G)
//   W = T diag(beta) K+,  U~ = T diag(beta) V,  U = U~ - W S^T
//   O = Q+ S^T + P U,   S <- S diag(e^G_last) + U^T K^
// (the oracle's chunkwise KDA, term by term).  Two kernels:
//
// The factor kernel, over all (chunk, value head) items at once: G from the
// gates; [K+; Q+] (K, Q scaled by e^G) and K- = K (.) e^-G for the channels
// whose decay over the chunk stays above e^-80, so that one tcgen05 product
// [K+; Q+] K-^T gives A and P (every kept entry is a bounded e^(G_r - G_j)
// with j <= r; entries above the diagonal, which may be huge, are masked by
// selection); the rare channels that decay faster are added entry by entry
// in fp32 with the exact exponent.  Then T (the shared divide-and-conquer
// inverse), and the loop's operands -- K+, Q+, K^, T'' = T diag(beta), P and
// e^G_last -- written in the 128-byte-swizzled layout the loop's products
// read, so that plain bulk copies move them.
//
// The chunk loop, one CTA per (sequence, value head) unit: the products of
// the gated delta rule's loop with the decays folded into the operands
//   (W)   W^T  = K+^T T''^T           128 x 64 x 64     warp 14
//   (U~)  U~^T = V^T T''^T            128 x 64 x 64     warp 13
//   (XU)  U^T  = U~^T - S W^T         128 x 64 x 128    warp 12
//   (S7)  S   += U^T K^                128 x 128 x 64    warp 12
//   (X1)  X1' = -S Q+^T               128 x 64 x 128    warp 15
//   (X6)  X2   = U^T P^T              128 x 64 x 64     warp 15
// O^T = X2 - X1'; the state pass scales column c of S by e^(G_last[c]).
// Roles as in the gated delta rule's two-kernel loop (state, epilogue, W^T
// epilogue, four issuers); every wait is bounded and a timeout records
// GDN_ERR_DEVICE_CHECK (bad_index -4 in the factor kernel, -5 in the loop).
#include "gdn_internal.cuh"
#include "gdn_inverse.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

// ---------------------------------------------------------------------------
// One (chunk, value head) item of the workspace, written by the factor kernel
// and bulk-copied by the chunk loop.  Tiles are bf16 in the 128-byte swizzle:
// K+, Q+, K^ as 2 atom columns x 64 token rows, T'' and P as one atom of 64
// rows; then e^G_last, 128 fp32.
constexpr uint32_t kItKp = 0, kItQp = 16384, kItKh = 32768, kItT = 49152, kItP = 57344, kItGam = 65536;
constexpr uint32_t kItemBytes = 66048;
constexpr float kMildFloor = -80.f;  // e^-G stays finite in fp32 while G >= -80

// ---------------------------------------------------------------- factors
constexpr int kFThreads = 256;
constexpr uint32_t kFOffA = 0;                             // [K+; Q+]: 2 atoms x 128 rows (32 KB)
constexpr uint32_t kFOffB = 32768;                         // K-: 2 atoms x 64 rows (16 KB)
constexpr uint32_t kFOffG = 49152;                         // G, fp32 [64 tokens][128 channels]
constexpr uint32_t kFOffAf = kFOffG + 64 * 128 * 4;        // A, inverted into T: 64 x kLdA fp32
constexpr uint32_t kFOffY = kFOffAf + 64 * kLdA * 4;       // 32 x kLdY fp32
constexpr uint32_t kFOffVec = kFOffY + 32 * kLdY * 4;      // per-token and per-channel vectors
constexpr int kFVB = 0, kFVIk = 64, kFVIq = 128, kFVGl = 192, kFVList = 320, kFVCount = 448, kFVecFloats = 512;
constexpr uint32_t kFOffBar = kFOffVec + kFVecFloats * 4;  // mbarrier, tensor-memory slot
constexpr uint32_t kFSmem = kFOffBar + 64 + 1024;
static_assert(kFSmem <= 116 * 1024, "two factor CTAs per SM");

template <bool kL2, bool kLogits>
__global__ void __launch_bounds__(kFThreads, 2)
kda_factor_kernel(const PrefillArgs a, unsigned char *items) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *G = reinterpret_cast<float *>(smem + kFOffG);
    float *Af = reinterpret_cast<float *>(smem + kFOffAf);
    float *Yb = reinterpret_cast<float *>(smem + kFOffY);
    float *vec = reinterpret_cast<float *>(smem + kFOffVec);
    int *list = reinterpret_cast<int *>(vec + kFVList);
    const uint32_t bar = sb + kFOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kFOffBar + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader *hdr = a.sched.hdr;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();  // the schedule (chunk_base, status) is written
    bool aborted = hdr->status != GDN_OK;
    const int hk = a.hk, hv = a.hv, group = hv / hk;
    const int64_t total = aborted ? 0 : int64_t(hdr->total_chunks) * hv;
    const __nv_bfloat16 *kp = static_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *qp = static_cast<const __nv_bfloat16 *>(a.q);
    const uint32_t id_gram = idesc_bf16(128, 64, false, false);
    uint32_t ph = 0;

    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
        const int gc = int(item / hv), h = int(item - int64_t(gc) * hv), hq = h / group;
        const int n = chunk_sequence(a.sched.chunk_base, a.num_seqs, gc);
        const int c0 = gc - a.sched.chunk_base[n];
        const int t0 = a.sched.start[n] + 64 * c0;
        const int L = min(64, a.sched.len[n] - 64 * c0);
        unsigned char *it = items + size_t(item) * kItemBytes;

        // 1. the log-decays of the chunk (floored; logits through log sigmoid; rows
        //    past the end 0), beta, and the rows' 1/||k||, 1/||q||
        for (int e = tid; e < 64 * 32; e += kFThreads) {
            const int r = e >> 5, q4 = e & 31;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < L) {
                v = *reinterpret_cast<const float4 *>(a.g + (size_t(t0 + r) * hv + h) * 128 + 4 * q4);
                if (kLogits) {
                    v.x = log_sigmoid_fast(v.x); v.y = log_sigmoid_fast(v.y);
                    v.z = log_sigmoid_fast(v.z); v.w = log_sigmoid_fast(v.w);
                }
                v.x = fmaxf(v.x, kGFloor); v.y = fmaxf(v.y, kGFloor);
                v.z = fmaxf(v.z, kGFloor); v.w = fmaxf(v.w, kGFloor);
            }
            *reinterpret_cast<float4 *>(G + r * 128 + 4 * q4) = v;
        }
        if (tid < 64) {
            float b = 0.f;
            if (tid < L) {
                b = a.beta[size_t(t0 + tid) * hv + h];
                if (kLogits) b = sigmoid_fast(b);
            }
            vec[kFVB + tid] = b;
        }
        if constexpr (kL2) {
            if (tid >= 128) {  // rows of K (0-63) and Q (64-127)
                const int R = tid - 128, r = R & 63;
                float ss = 0.f;
                if (r < L) {
                    const uint4 *src = reinterpret_cast<const uint4 *>((R < 64 ? kp : qp) + (size_t(t0 + r) * hk + hq) * 128);
#pragma unroll 4
                    for (int p = 0; p < 16; ++p) {
                        const uint4 w = src[p];
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                        }
                    }
                }
                vec[(R < 64 ? kFVIk : kFVIq) + r] = inv_l2(ss);
            }
        }
        __syncthreads();
        // 2. prefix sums per channel, in place: each half of the tokens by its own
        //    thread, then the second half offset by the first half's total
        {
            const int c = tid & 127, r0 = (tid >> 7) * 32;
            float acc = 0.f;
#pragma unroll 8
            for (int r = r0; r < r0 + 32; ++r) {
                acc += G[r * 128 + c];
                G[r * 128 + c] = acc;
            }
        }
        __syncthreads();
        if (tid >= 128) {
            const int c = tid - 128;
            const float base = G[31 * 128 + c];
#pragma unroll 8
            for (int r = 32; r < 64; ++r) G[r * 128 + c] += base;
            const float gl = G[63 * 128 + c];
            vec[kFVGl + c] = gl;  // G_63 = G_(L-1): rows past the end carry g = 0
            reinterpret_cast<float *>(it + kItGam)[c] = __expf(gl);
        }
        __syncthreads();
        if (warp == 0) {
            int count = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = 32 * q + lane;
                const bool strong = vec[kFVGl + c] < kMildFloor;
                const uint32_t m = __ballot_sync(0xffffffffu, strong);
                if (strong) list[count + __popc(m & ((1u << lane) - 1u))] = c;
                count += __popc(m);
            }
            if (lane == 0) reinterpret_cast<int *>(vec)[kFVCount] = count;
        }
        // 3. operands: [K+; Q+] and K- for the product, K+, Q+, K^ for the loop
        for (int e = tid; e < 64 * 16; e += kFThreads) {
            const int r = e >> 4, cc = e & 15, ch = cc & 7;
            const uint32_t atom = uint32_t(cc >> 3);
            uint4 kw = make_uint4(0, 0, 0, 0), qw = make_uint4(0, 0, 0, 0);
            if (r < L) {
                kw = *reinterpret_cast<const uint4 *>(kp + (size_t(t0 + r) * hk + hq) * 128 + 8 * cc);
                qw = *reinterpret_cast<const uint4 *>(qp + (size_t(t0 + r) * hk + hq) * 128 + 8 * cc);
            }
            const float sk = kL2 ? vec[kFVIk + r] : 1.f, sq = kL2 ? vec[kFVIq + r] : 1.f;
            const uint32_t kws[4] = {kw.x, kw.y, kw.z, kw.w}, qws[4] = {qw.x, qw.y, qw.z, qw.w};
            float kpv[8], kmv[8], khv[8], qpv[8];
            float grv[8], glv[8];
            load4(G + r * 128 + 8 * cc, grv);
            load4(G + r * 128 + 8 * cc + 4, grv + 4);
            load4(vec + kFVGl + 8 * cc, glv);
            load4(vec + kFVGl + 8 * cc + 4, glv + 4);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float gr = grv[u], gl = glv[u];
                const float kv = sk * __uint_as_float((u & 1) ? (kws[u >> 1] & 0xffff0000u) : (kws[u >> 1] << 16));
                const float qv = sq * __uint_as_float((u & 1) ? (qws[u >> 1] & 0xffff0000u) : (qws[u >> 1] << 16));
                const float eg = __expf(gr);
                kpv[u] = kv * eg;
                qpv[u] = qv * eg;
                kmv[u] = gl >= kMildFloor ? kv * __fdividef(1.f, eg) : 0.f;
                khv[u] = kv * __expf(gl - gr);
            }
            const uint4 kpp = pack_bf16x8(kpv), qpp = pack_bf16x8(qpv), kmp = pack_bf16x8(kmv), khp = pack_bf16x8(khv);
            const uint32_t off = sw128_offset(r, ch);
            st_shared_v4(sb + kFOffA + atom * 16384 + off, kpp);
            st_shared_v4(sb + kFOffA + atom * 16384 + 8192 + off, qpp);
            st_shared_v4(sb + kFOffB + atom * 8192 + off, kmp);
            *reinterpret_cast<uint4 *>(it + kItKp + atom * 8192 + off) = kpp;
            *reinterpret_cast<uint4 *>(it + kItQp + atom * 8192 + off) = qpp;
            *reinterpret_cast<uint4 *>(it + kItKh + atom * 8192 + off) = khp;
        }
        fence_proxy_async_shared();  // the operand stores, before the tensor cores read them
        __syncthreads();
        // 4. [K+; Q+] K-^T: rows 0-63 the Gram of A, rows 64-127 that of P
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t atom = uint32_t(s >> 2), kk = uint32_t(s & 3) * 32;
                mma_bf16(tmem, smem_desc(sb + kFOffA + atom * 16384 + kk, 16, 1024),
                         smem_desc(sb + kFOffB + atom * 8192 + kk, 16, 1024), id_gram, s > 0);
            }
            mma_commit(bar);
        }
        {
            const bool ok = warp != 0 || mbar_wait(bar, ph);
            ph ^= 1u;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        tc_fence_after();
        // 5. A (fp32, for the inverse) and P (bf16, to the item) with the strong
        //    channels added exactly; entries above the diagonal are selected away
        if (warp < 4) {
            const int R = warp * 32 + lane, r = R & 63;
            const bool is_a = R < 64;
            const int count = reinterpret_cast<const int *>(vec)[kFVCount];
            const float br = vec[kFVB + r];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {  // 32 columns at a time (registers)
                const int j0 = 32 * half;
                float v[32];
                tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(j0), v);
                tmem_wait_ld();
                if (count > 0 && r < L && j0 <= r) {
                    const __nv_bfloat16 *xrow = (is_a ? kp : qp) + (size_t(t0 + r) * hk + hq) * 128;
                    const float sx = kL2 ? vec[(is_a ? kFVIk : kFVIq) + r] : 1.f;
                    for (int i = 0; i < count; ++i) {
                        const int c = list[i];
                        const float xr = sx * __bfloat162float(xrow[c]), gr = G[r * 128 + c];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {  // (unrolled: v stays in registers)
                            const int j = j0 + jj;
                            if (j <= r) {                  // j <= r < L: rows of this sequence
                                const float kj = (kL2 ? vec[kFVIk + j] : 1.f) *
                                                 __bfloat162float(kp[(size_t(t0 + j) * hk + hq) * 128 + c]);
                                v[jj] = fmaf(xr * kj, __expf(gr - G[j * 128 + c]), v[jj]);
                            }
                        }
                    }
                }
                if (is_a) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int j = j0 + 4 * q;
                        *reinterpret_cast<float4 *>(Af + r * kLdA + j) =
                            make_float4(j < r ? br * v[4 * q] : 0.f, j + 1 < r ? br * v[4 * q + 1] : 0.f,
                                        j + 2 < r ? br * v[4 * q + 2] : 0.f, j + 3 < r ? br * v[4 * q + 3] : 0.f);
                    }
                } else {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float x[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) x[u] = (j0 + 8 * ch + u <= r) ? v[8 * ch + u] : 0.f;
                        *reinterpret_cast<uint4 *>(it + kItP + sw128_offset(r, j0 / 8 + ch)) = pack_bf16x8(x);
                    }
                }
            }
        }
        tc_fence_before();  // the tensor-memory reads, before the next item's product
        __syncthreads();
        // 6. T = (I + A)^-1, then T'' = T diag(beta) to the item
        invert_in_place(Af, Yb, tid);
        {
            const int r = tid >> 2, cq = (tid & 3) * 16;
            float x[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) x[u] = Af[r * kLdA + cq + u] * vec[kFVB + cq + u];
            *reinterpret_cast<uint4 *>(it + kItT + sw128_offset(r, cq / 8)) = pack_bf16x8(x);
            *reinterpret_cast<uint4 *>(it + kItT + sw128_offset(r, cq / 8 + 1)) = pack_bf16x8(x + 8);
        }
        __syncthreads();  // Af, G and the vectors are reused by the next item
    }
    if (aborted && tid == 0 && total > 0) {
        // let this thread's tensor-core work drain (bounded) before the tensor
        // memory is freed
        mma_commit(bar);
        (void)mbar_wait(bar, ph);
        hdr->bad_index = -4;
        atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------- chunk loop
constexpr int kThreads = 512;
constexpr int kWarpEpi = 4, kWarpPrep = 8, kWarpA = 12, kWarpB = 13, kWarpW = 14;
constexpr int kBarState = 1, kBarEpi = 2, kBarPrep = 3;
constexpr int kSpCols = 96;

constexpr uint32_t kSlotKQ = 49152, kKQ_Kp = 0, kKQ_Qp = 16384, kKQ_Kh = 32768;  // [2]: K+, Q+, K^
constexpr uint32_t kOffKQ = 0;
constexpr uint32_t kSlotT = 17408, kT_T = 0, kT_P = 8192, kT_Gam = 16384;       // [2]: T'', P, e^G_last
constexpr uint32_t kOffT = kOffKQ + 2 * kSlotKQ;                                  // 98304
constexpr uint32_t kOffW = kOffT + 2 * kSlotT;                                    // 133120: W^T [2]
constexpr uint32_t kOffV = kOffW + 2 * 16384;                                     // 165888
constexpr uint32_t kOffOst = kOffV + 16384;                                       // 182272
constexpr uint32_t kOffBar = kOffOst + 16384;                                     // 198656
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");
constexpr uint32_t kBytesKQ = 49152, kBytesT = 16384 + 512, kBytesV = 16384;

enum {
    kBKQ = 0,     // [2] K+, Q+, K^ of a chunk landed
    kBT = 2,      // [2] T'', P, e^G_last landed
    kBV = 4,      // V landed
    kBW = 5,      // W^T done
    kBFull = 6,   // [2] W^T of a chunk in shared memory
    kBU = 8,      // U~ done
    kBSp = 9,     // state pass done (count 2)
    kBXU = 10,    // (XU) done
    kBX1 = 11,    // (X1) done
    kBUe = 12,    // bf16 U^T written
    kBS7 = 13,    // (S7) done
    kBX6 = 14,    // (X6) done
    kBOut = 15,   // X1', X2 read by the output epilogue
    kBWFree = 16, // [2] W^T of a stage read by (XU)
    kNumBars = 18
};

constexpr uint32_t kColW = 0, kColU = 64, kColX1 = 128, kColS = 192, kColX2 = 320, kColSb = 384, kColUb = 448;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ bool group_wait(bool poller, uint32_t bar, uint32_t parity, int bar_id, int count) {
    const bool ok = !poller || mbar_wait(bar, parity);
    return !named_sync_or(bar_id, count, !ok);
}

// The state pass over columns [c0, c0 + 32 kSlices) of this thread's row: the
// bf16 copy (A operand of (XU), (X1)) and S[:, c] <- e^(G_last[c]) S[:, c].
template <int kSlices>
__device__ __forceinline__ void kda_state_pass(uint32_t tmem_row, int c0, const float *gam) {
#pragma unroll
    for (int p = 0; p < kSlices; ++p) {
        const int c = c0 + 32 * p;
        float v[32];
        tmem_ld32(tmem_row + kColS + uint32_t(c), v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
        tmem_st16u(tmem_row + kColSb + uint32_t(c / 2), pk);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float gq[4];
            load4(gam + c + 4 * q, gq);
#pragma unroll
            for (int u = 0; u < 4; ++u) v[4 * q + u] *= gq[u];
        }
        tmem_st32(tmem_row + kColS + uint32_t(c), v);
    }
    tmem_wait_st();
}
template <int kSlices>
__device__ __forceinline__ void kda_state_in(uint32_t tmem_row, const float *src, int c0) {
#pragma unroll
    for (int p = 0; p < kSlices; ++p) {
        float v[32];
        if (src) {
#pragma unroll
            for (int c = 0; c < 8; ++c) load4(src + c0 + 32 * p + 4 * c, v + 4 * c);
        } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = 0.f;
        }
        tmem_st32(tmem_row + kColS + uint32_t(c0 + 32 * p), v);
    }
    tmem_wait_st();
}
template <int kSlices>
__device__ __forceinline__ void kda_state_out(uint32_t tmem_row, float *dst, int c0) {
#pragma unroll
    for (int p = 0; p < kSlices; ++p) {
        float v[32];
        tmem_ld32(tmem_row + kColS + uint32_t(c0 + 32 * p), v);
        tmem_wait_ld();
        if (dst) {
            float4 *d4 = reinterpret_cast<float4 *>(dst + c0 + 32 * p);
#pragma unroll
            for (int c = 0; c < 8; ++c) d4[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
kda_chain_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const PrefillArgs a, const unsigned char *items) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    const uint32_t bars = sb + kOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * kNumBars);
    int *s_unit = reinterpret_cast<int *>(smem + kOffBar + 8 * kNumBars + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_bits = uint32_t((warp & 3) * 32) << 16;
    WsHeader *hdr = a.sched.hdr;
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    auto gam_of = [&](uint32_t gc) {  // e^G_last of chunk gc, in its T slot
        return reinterpret_cast<const float *>(smem + kOffT + (gc & 1u) * kSlotT + kT_Gam);
    };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), i == kBSp ? 2 : 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();  // the schedule and the items are written
    bool aborted = hdr->status != GDN_OK;

    const int hv = a.hv;
    const int total_units = aborted ? 0 : a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);

    const uint32_t id_w = idesc_bf16(128, 64, true, false);         // W^T and U~^T (A MN-major)
    const uint32_t id_xu = idesc_bf16(128, 64, false, true, true);  // -S W^T
    const uint32_t id_x1 = idesc_bf16(128, 64, false, false, true); // -S Q+^T
    const uint32_t id_s7 = idesc_bf16(128, 128, false, true);       // U^T K^
    const uint32_t id_x6 = idesc_bf16(128, 64, false, false);       // U^T P^T

    uint32_t gn = 0;
    for (;;) {
        if (__syncthreads_or(aborted)) break;
        if (tid == 0) *s_unit = int(atomicAdd(&hdr->next_unit, 1u));
        __syncthreads();
        const int unit = *s_unit;
        if (unit >= total_units) break;
        const int seq = a.sched.order[unit / hv];
        const int h = unit % hv;
        const int t0 = a.sched.start[seq], len = a.sched.len[seq];
        const int nchunks = (len + 63) / 64;
        const int cbase = a.sched.chunk_base[seq];
        const size_t sbase = (size_t(seq) * hv + h) * 128 * 128;
        auto item_of = [&](int c) { return items + (size_t(cbase + c) * hv + h) * kItemBytes; };

        auto load_kq = [&](int c) {  // K+, Q+, K^ of chunk c
            const uint32_t gc = gn + uint32_t(c), i = gc & 1u;
            const uint32_t b = bar(kBKQ + int(i));
            mbar_arrive_expect_tx(b, kBytesKQ);
            bulk_load(sb + kOffKQ + i * kSlotKQ, item_of(c) + kItKp, kBytesKQ, b);
        };
        auto load_t = [&](int c) {  // T'', P and e^G_last of chunk c
            const uint32_t gc = gn + uint32_t(c), i = gc & 1u;
            const uint32_t b = bar(kBT + int(i));
            mbar_arrive_expect_tx(b, kBytesT);
            bulk_load(sb + kOffT + i * kSlotT, item_of(c) + kItT, kBytesT, b);
        };
        auto load_v = [&](int c) {
            mbar_arrive_expect_tx(bar(kBV), kBytesV);
            tma_load_3d(sb + kOffV, &tm_v, 0, h, t0 + 64 * c, bar(kBV));
            tma_load_3d(sb + kOffV + 8192, &tm_v, 64, h, t0 + 64 * c, bar(kBV));
        };

        if (warp < kWarpEpi) {
            // ============ state warps: thread = state row, columns 0 .. kSpCols-1 ============
            const int row = (warp & 3) * 32 + lane;
            const uint32_t trow = tmem + lane_bits;
            if (nchunks == 0) {
                if (a.s_final) {
                    float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128);
                    const float4 *src = a.s0 ? reinterpret_cast<const float4 *>(a.s0 + sbase + size_t(row) * 128)
                                             : nullptr;
                    for (int c = 0; c < 32; ++c) dst[c] = src ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
                kda_state_in<kSpCols / 32>(trow, a.s0 ? a.s0 + sbase + size_t(row) * 128 : nullptr, 0);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n);
                    // this chunk's decays have landed (W^T, which needed them, is done), and the
                    // previous chunk's (S7) and (X1) -- the readers of S and its bf16 copy
                    bool ok = true;
                    if (warp == 0) {
                        ok = mbar_wait(bar(kBFull + int(gc & 1u)), (gc >> 1) & 1u);
                        if (ok && n > 0) ok = mbar_wait(bar(kBS7), (gc - 1) & 1u) && mbar_wait(bar(kBX1), (gc - 1) & 1u);
                    }
                    if (named_sync_or(kBarState, 128, !ok)) { aborted = true; break; }
                    tc_fence_after();
                    kda_state_pass<kSpCols / 32>(trow, 0, gam_of(gc));
                    tc_fence_before();
                    named_sync(kBarState, 128);
                    if (tid == 0) mbar_arrive(bar(kBSp));
                }
                if (!aborted) {
                    const uint32_t gl = gn + uint32_t(nchunks) - 1u;
                    if (!group_wait(warp == 0, bar(kBS7), gl & 1u, kBarState, 128)) {
                        aborted = true;
                    } else {
                        tc_fence_after();
                        kda_state_out<kSpCols / 32>(trow, a.s_final ? a.s_final + sbase + size_t(row) * 128 : nullptr, 0);
                        tc_fence_before();
                    }
                }
            }
        } else if (warp < kWarpPrep) {
            // ==================== epilogue warps: thread = value row i ====================
            const int row = (warp & 3) * 32 + lane;
            const uint32_t trow = tmem + lane_bits;
            const bool poller = warp == kWarpEpi;
            const int et = tid - 32 * kWarpEpi;
            float *sf_row = a.s_final ? a.s_final + sbase + size_t(row) * 128 : nullptr;
            if (nchunks > 0) {
                kda_state_in<(128 - kSpCols) / 32>(trow, a.s0 ? a.s0 + sbase + size_t(row) * 128 : nullptr, kSpCols);
                if (!group_wait(poller, bar(kBFull + int(gn & 1u)), (gn >> 1) & 1u, kBarEpi, 128)) {
                    aborted = true;
                } else {
                    tc_fence_after();
                    kda_state_pass<(128 - kSpCols) / 32>(trow, kSpCols, gam_of(gn));
                    tc_fence_before();
                    named_sync(kBarEpi, 128);
                    if (et == 0) mbar_arrive(bar(kBSp));
                }
            }
            for (int n = 0; n < nchunks && !aborted; ++n) {
                const uint32_t gc = gn + uint32_t(n);
                const int c0 = t0 + 64 * n, L = min(64, len - 64 * n);
                // U^T -> bf16, the A operand of (X6) and (S7)
                if (!group_wait(poller, bar(kBXU), gc & 1u, kBarEpi, 128)) { aborted = true; break; }
                tc_fence_after();
                {
                    float v[2][32];
                    tmem_ld32(trow + kColU, v[0]);
                    tmem_ld32(trow + kColU + 32, v[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        uint32_t pu[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) pu[j] = pack_bf16x2(v[p][2 * j], v[p][2 * j + 1]);
                        tmem_st16u(trow + kColUb + 16 * p, pu);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                named_sync(kBarEpi, 128);
                if (et == 0) mbar_arrive(bar(kBUe));
                // O^T = X2 - X1', staged token-major (rows of 256 bytes)
                {
                    bool ok = true;
                    if (poller) ok = mbar_wait(bar(kBX1), gc & 1u) && mbar_wait(bar(kBX6), gc & 1u);
                    if (named_sync_or(kBarEpi, 128, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                if (et == 0) bulk_wait_read();  // the previous chunk's output store has read the tile
                named_sync(kBarEpi, 128);
                {
                    __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffOst);
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        float x1[32], x2[32];
                        tmem_ld32(trow + kColX1 + 32 * p, x1);
                        tmem_ld32(trow + kColX2 + 32 * p, x2);
                        tmem_wait_ld();
#pragma unroll
                        for (int r = 0; r < 32; ++r) Ot[(32 * p + r) * 128 + row] = __float2bfloat16_rn(x2[r] - x1[r]);
                    }
                }
                tc_fence_before();
                fence_proxy_async_shared();
                named_sync(kBarEpi, 128);
                if (et == 0) {
                    mbar_arrive(bar(kBOut));
                    if (L == 64) {
                        tma_store_3d(&tm_o, sb + kOffOst, 0, h, c0);
                        bulk_commit();
                    }
                }
                if (L < 64) {
                    for (int e = et; e < 64 * 16; e += 128) {
                        const int r = e >> 4, c = e & 15;
                        if (r < L) {
                            const uint4 val = *reinterpret_cast<const uint4 *>(smem + kOffOst + r * 256 + c * 16);
                            *reinterpret_cast<uint4 *>(o + (size_t(c0 + r) * hv + h) * 128 + c * 8) = val;
                        }
                    }
                }
                // the state pass of columns kSpCols..127 for the next chunk, or this
                // unit's final state of those columns
                {
                    const uint32_t g1 = gc + 1u;
                    bool ok = true;
                    if (poller) {
                        ok = mbar_wait(bar(kBS7), gc & 1u);
                        if (ok && n + 1 < nchunks) ok = mbar_wait(bar(kBFull + int(g1 & 1u)), (g1 >> 1) & 1u);
                    }
                    if (named_sync_or(kBarEpi, 128, !ok)) { aborted = true; break; }
                    tc_fence_after();
                    if (n + 1 < nchunks) {
                        kda_state_pass<(128 - kSpCols) / 32>(trow, kSpCols, gam_of(g1));
                        tc_fence_before();
                        named_sync(kBarEpi, 128);
                        if (et == 0) mbar_arrive(bar(kBSp));
                    } else {
                        kda_state_out<(128 - kSpCols) / 32>(trow, sf_row, kSpCols);
                        tc_fence_before();
                    }
                }
            }
        } else if (warp < kWarpA) {
            // ============ prep warps: the epilogue of W^T (MN-major operand of (XU)) ============
            const int pt = tid - 32 * kWarpPrep;
            const bool poller = warp == kWarpPrep;
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                const uint32_t wst = sb + kOffW + b * 16384;
                // the stage was read by (XU) of the chunk two back, and W^T is done
                if (!group_wait(poller && gc >= 2, bar(kBWFree + int(b)), ((gc >> 1) - 1) & 1u, kBarPrep, 128)) {
                    aborted = true;
                    break;
                }
                if (!group_wait(poller, bar(kBW), gc & 1u, kBarPrep, 128)) { aborted = true; break; }
                tc_fence_after();
                {
                    const int c = (warp & 3) * 32 + lane;  // d_k index = tensor-memory lane
                    const uint32_t base = wst + uint32_t(c) * 128;
                    float v[2][32];
                    tmem_ld32(tmem + lane_bits + kColW, v[0]);
                    tmem_ld32(tmem + lane_bits + kColW + 32, v[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            st_shared_v4(base + (uint32_t((4 * p + q) ^ (c & 7)) << 4), pack_bf16x8(v[p] + 8 * q));
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarPrep, 128);
                if (pt == 0) mbar_arrive(bar(kBFull + int(b)));
            }
        } else if (warp == kWarpA) {
            // ============ warp 12: (XU) and (S7), the state's critical path ============
            if (lane == 0) {
                if (nchunks > 0) load_kq(0);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t wst = sb + kOffW + b * 16384;
                    const uint32_t kq = sb + kOffKQ + b * kSlotKQ;
                    bool ok = mbar_wait(bar(kBFull + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBSp), gc & 1u) &&
                              mbar_wait(bar(kBU), gc & 1u);
                    if (!ok) { aborted = true; break; }
                    // the previous chunk's readers of its slot are done (the state pass waited
                    // for its (S7) and (X1), and its W^T was made before): the next chunk's
                    // operands take it
                    if (n + 1 < nchunks) load_kq(n + 1);
                    tc_fence_after();
                    // (XU): U^T = U~^T - S W^T
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        mma_bf16_ts(tmem + kColU, tmem + kColSb + 8 * s,
                                    smem_desc(wst, 8192, 1024) + uint64_t((s * 2048) >> 4), id_xu, 1);
                    mma_commit(bar(kBXU));
                    mma_commit(bar(kBWFree + int(b)));
                    if (!mbar_wait(bar(kBUe), gc & 1u)) { aborted = true; break; }
                    if (!mbar_wait(bar(kBKQ + int(b)), (gc >> 1) & 1u)) { aborted = true; break; }
                    tc_fence_after();
                    // (S7): S += U^T K^ (B = K^ MN-major)
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColS, tmem + kColUb + 8 * s,
                                    smem_desc(kq + kKQ_Kh, 8192, 1024) + uint64_t((s * 2048) >> 4), id_s7, 1);
                    mma_commit(bar(kBS7));
                }
            }
        } else if (warp == kWarpB) {
            // ========================= warp 13: U~^T = V^T T''^T =========================
            if (lane == 0) {
                if (nchunks > 0) { load_t(0); load_v(0); }
                if (nchunks > 1) load_t(1);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t tt = sb + kOffT + b * kSlotT;
                    bool ok = mbar_wait(bar(kBT + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBV), gc & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBUe), (gc - 1) & 1u);  // the previous U has been read
                    if (!ok) { aborted = true; break; }
                    // the previous chunk's T slot: its U~ and W^T are done, its P read by (X6)
                    // and its decays by both state passes: the next chunk takes it
                    if (n >= 1 && n + 1 < nchunks) {
                        if (!mbar_wait(bar(kBX6), (gc - 1) & 1u)) { aborted = true; break; }
                        load_t(n + 1);
                    }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColU, smem_desc(sb + kOffV, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(tt + kT_T, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBU));
                    if (n + 1 < nchunks) {
                        if (!mbar_wait(bar(kBU), gc & 1u)) { aborted = true; break; }
                        load_v(n + 1);
                    }
                }
            }
        } else if (warp == kWarpW) {
            // ======================== warp 14: W^T = K+^T T''^T ========================
            if (lane == 0) {
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t kq = sb + kOffKQ + b * kSlotKQ;
                    const uint32_t tt = sb + kOffT + b * kSlotT;
                    bool ok = mbar_wait(bar(kBKQ + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBT + int(b)), (gc >> 1) & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBFull + int((gc - 1) & 1u)), ((gc - 1) >> 1) & 1u);
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColW, smem_desc(kq + kKQ_Kp, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(tt + kT_T, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBW));
                }
            }
        } else {
            // ============ warp 15: (X1) X1' = -S Q+^T and (X6) X2 = U^T P^T ============
            if (lane == 0) {
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t kq = sb + kOffKQ + b * kSlotKQ;
                    const uint32_t tt = sb + kOffT + b * kSlotT;
                    bool ok = mbar_wait(bar(kBFull + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBSp), gc & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBOut), (gc - 1) & 1u);  // X1', X2 read
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t koff = (s >> 2) * 8192 + (s & 3) * 32;
                        mma_bf16_ts(tmem + kColX1, tmem + kColSb + 8 * s,
                                    smem_desc(kq + kKQ_Qp, 16, 1024) + uint64_t(koff >> 4), id_x1, s > 0);
                    }
                    mma_commit(bar(kBX1));
                    if (!mbar_wait(bar(kBUe), gc & 1u)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColX2, tmem + kColUb + 8 * s,
                                    smem_desc(tt + kT_P, 16, 1024) + uint64_t((s * 32) >> 4), id_x6, s > 0);
                    mma_commit(bar(kBX6));
                }
            }
        }
        gn += uint32_t(nchunks);
    }

    if (warp >= kWarpEpi && warp < kWarpPrep && tid == 32 * kWarpEpi) bulk_wait_all();
    if (aborted) {
        if (warp >= kWarpA && lane == 0) {
            const int bi = warp == kWarpA ? kBS7 : (warp == kWarpB ? kBU : (warp == kWarpW ? kBW : kBX6));
            mma_commit(bar(bi));
            (void)mbar_wait(bar(bi), 0u);
            (void)mbar_wait(bar(bi), 1u);
        }
        if (tid == 0) {
            hdr->bad_index = -5;
            atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool kda_tc_supported(const gdn_shape_t &s) {
    return s.dtype == GDN_DTYPE_BF16 && s.head_dim_k == 128 && s.head_dim_v == 128 && s.chunk_size == 64;
}

KdaLayout kda_layout(const gdn_shape_t &s) {
    KdaLayout L;
    L.sched = ws_layout(s.num_seqs);
    size_t off = L.sched.total;
    L.cbase_off = off;
    off = align256(off + 4 * (size_t(s.num_seqs) + 1));
    off = (off + 1023) & ~size_t(1023);
    L.items_off = off;
    L.max_chunks = max_chunks_bound(s);
    off += size_t(L.max_chunks) * size_t(s.num_v_heads) * kItemBytes;
    L.total = align256(off);
    return L;
}

cudaError_t launch_kda_tc(const PrefillArgs &a, unsigned char *items, cudaStream_t stream, int num_sms) {
    const bool l2 = a.flags & GDN_FLAG_QK_L2NORM, logits = a.flags & GDN_FLAG_GATE_LOGITS;
    using FactorFn = void (*)(PrefillArgs, unsigned char *);
    static const FactorFn ftable[4] = {kda_factor_kernel<false, false>, kda_factor_kernel<false, true>,
                                       kda_factor_kernel<true, false>, kda_factor_kernel<true, true>};
    const FactorFn fk = ftable[(l2 ? 2 : 0) + (logits ? 1 : 0)];
    cudaError_t e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kFSmem));
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(unsigned(2 * num_sms));  // persistent; items come from the schedule on the device
        cfg.blockDim = dim3(kFThreads);
        cfg.dynamicSmemBytes = kFSmem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, fk, a, items);
        count_launch();
        if (e != cudaSuccess) return e;
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mv, mo;
    if (!make_map(&mv, a.v, a.hv, a.tokens) || !make_map(&mo, a.o, a.hv, a.tokens, true)) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kda_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t(a.num_seqs) * a.hv;
    const int grid = int(units < num_sms ? units : num_sms);
    if (grid <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kda_chain_kernel, mv, mo, a, static_cast<const unsigned char *>(items));
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
