// gdn_chunk_inv.cu -- first kernel of the two-kernel tensor-core prefill.
//
// For every (chunk, value head) it forms the chunk's triangular factor of the
// WY representation ("Gated Attention Architectures", section 2: the UT
// transform of the product of generalised Householder transitions; section 3:
// the same with the per-chunk cumulative decay products),
//
//   A_rj = beta_r Gamma_rj (k_r . k_j)  for j < r (else 0),
//   Gamma_rj = e^(G_r - G_j),  G = chunk-local prefix sums of g,
//   T = (I + A)^-1   (unit lower triangular, 64 x 64),
//
// and stores the two column scalings the chunk loop multiplies by, T' = T
// diag(beta gamma) and T'' = T diag(beta) (gamma = e^G), as bf16, each
// rounded once from the fp32 T.  None of this depends on the state, so it runs over
// the chunks of all sequences at once, before the kernel that carries the
// state (gdn_chunk_chain.cu), which reads T instead of inverting on its
// critical path.  Tokens past a sequence's end take beta = g = 0, so A is zero
// there and T is the identity.
//
// One work item is a (chunk, q/k head) pair: its K tile arrives by TMA (double
// buffered, one item ahead), the Gram K K^T is one tcgen05.mma group of
// M = 64 (fp32 in tensor memory), and each of the q/k head's value heads then
// masks the Gram into A (fp32, shared memory) and inverts it in place: the
// four 16 x 16 diagonal blocks by forward substitution in fp32, then the
// 16 -> 32 and 32 -> 64 block levels
//   [[X, 0], [C, Z]]^-1 = [[X^-1, 0], [-Z^-1 C X^-1, Z^-1]]
// as warp-level tf32 products with fp32 accumulation (T is rounded to bf16
// afterwards, so the 10-bit tf32 mantissa is ample).  With GDN_FLAG_QK_L2NORM
// the keys are normalised inside the mask (A_rj carries 1 / (||k_r|| ||k_j||)),
// so T is the factor of the normalised keys.  Every wait is bounded; a timeout
// records GDN_ERR_DEVICE_CHECK (bad_index -3) in the workspace status word.
#include "gdn_internal.cuh"
#include "gdn_inverse.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kTileK = 16384;  // one K tile: 2 atom columns x 64 rows x 128 bytes
constexpr uint32_t kOffK0 = 0, kOffK1 = kTileK;
constexpr uint32_t kOffA = 2 * kTileK;                 // A, inverted in place into T
constexpr uint32_t kOffY = kOffA + 64 * kLdA * 4;      // 32 x kLdY fp32
constexpr uint32_t kOffVec = kOffY + 32 * kLdY * 4;    // per-token vectors (below)
constexpr int kMaxGatedHeads = 8;                      // value heads per q/k head whose gates are prefetched
constexpr uint32_t kOffGst = kOffVec + 6 * 64 * 4;     // gates by cp.async: [2 items][kMaxGatedHeads][g, beta][64]
constexpr uint32_t kOffBar = kOffGst + 2 * kMaxGatedHeads * 2 * 64 * 4;  // mbarriers, tensor-memory slot
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;   // + alignment slack
constexpr int kVecG = 0, kVecB = 64, kVecRow = 128, kVecCol = 192, kVecIk = 256, kVecTp = 320;
constexpr int kBarK = 0, kBarMma = 2;  // K tile barriers (2 buffers), Gram completion
constexpr uint32_t kTmemCols = 64;

template <bool kL2, bool kLogits>
__global__ void __launch_bounds__(kThreads, 3)
chunk_inverse_kernel(const __grid_constant__ CUtensorMap tm_k, const PrefillArgs a, __nv_bfloat16 *tinv,
                     float *gcum) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *Af = reinterpret_cast<float *>(smem + kOffA);
    float *Yb = reinterpret_cast<float *>(smem + kOffY);
    float *vec = reinterpret_cast<float *>(smem + kOffVec);
    const uint32_t bars = sb + kOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 24);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader *hdr = a.sched.hdr;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(bars + 8 * i, 1);
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
    grid_dep_wait();  // the schedule (chunk_base, status) is written
    bool aborted = hdr->status != GDN_OK;
    const int hk = a.hk, hv = a.hv, group = hv / hk;
    const int total = aborted ? 0 : hdr->total_chunks * hk;
    const uint32_t id_gram = idesc_bf16(64, 64, false, false);

    // item -> (chunk, q/k head, first token, tokens)
    auto locate = [&](int item, int &gc, int &hq, int &t0, int &L) {
        gc = item / hk;
        hq = item - gc * hk;
        const int n = chunk_sequence(a.sched.chunk_base, a.num_seqs, gc);
        const int c = gc - a.sched.chunk_base[n];
        t0 = a.sched.start[n] + 64 * c;
        L = min(64, a.sched.len[n] - 64 * c);
    };
    auto load_k = [&](uint32_t buf, int hq, int t0, uint32_t bar) {
        mbar_arrive_expect_tx(bar, kTileK);
        tma_load_3d(buf, &tm_k, 0, hq, t0, bar);
        tma_load_3d(buf + 8192, &tm_k, 64, hq, t0, bar);
    };
    // the gates of an item's value heads (g, beta for 64 tokens; zeros past the end) by
    // cp.async into buffer `buf`, one group per item; with more than kMaxGatedHeads value
    // heads per q/k head the gates are read from global memory instead
    const bool prefetch = group <= kMaxGatedHeads;
    auto load_gates = [&](uint32_t buf, int hq, int t0, int L) {
        if (prefetch) {
            const uint32_t dst = sb + kOffGst + buf * (kMaxGatedHeads * 512);
            for (int e = tid; e < group * 128; e += kThreads) {
                const int j = e >> 7, isb = (e >> 6) & 1, r = e & 63;
                const size_t i = size_t(t0 + min(r, L - 1)) * hv + hq * group + j;
                cp_async_4(dst + uint32_t(e) * 4, (isb ? a.beta : a.g) + i, r < L);
            }
        }
        cp_async_commit();
    };

    int item = blockIdx.x;
    int gc = 0, hq = 0, t0 = 0, L = 0;
    if (item < total) {
        locate(item, gc, hq, t0, L);
        if (tid == 0) load_k(sb + kOffK0, hq, t0, bars + 8 * kBarK);
        load_gates(0, hq, t0, L);
    }
    uint32_t ph_k[2] = {0u, 0u}, ph_m = 0u;
    for (uint32_t it = 0; item < total; ++it, item += gridDim.x) {
        const uint32_t buf = it & 1u;
        const uint32_t ktile = sb + (buf ? kOffK1 : kOffK0);
        // the next item's K tile comes in while this one is worked on
        const int nitem = item + int(gridDim.x);
        int ngc = 0, nhq = 0, nt0 = 0, nL = 0;
        if (nitem < total) {
            locate(nitem, ngc, nhq, nt0, nL);
            if (tid == 0) load_k(sb + (buf ? kOffK0 : kOffK1), nhq, nt0, bars + 8 * (kBarK + (buf ^ 1u)));
            load_gates(buf ^ 1u, nhq, nt0, nL);
            cp_async_wait_1();  // this item's gates (the next item's may still be in flight)
        } else {
            cp_async_wait_all();
        }
        {
            const bool ok = warp != 0 || mbar_wait(bars + 8 * (kBarK + buf), ph_k[buf]);
            ph_k[buf] ^= 1u;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        // Gram K K^T (M = 64: row r of the result sits in tensor-memory lane
        // (r % 16) + 32 (r / 16)), one thread issues
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t d = smem_desc(ktile + (s >> 2) * 8192, 16, 1024) + uint64_t(((s & 3) * 32) >> 4);
                mma_bf16(tmem, d, d, id_gram, s > 0);
            }
            mma_commit(bars + 8 * kBarMma);
        }
        if constexpr (kL2) {
            // 1 / max(||k_r||, 1e-12) of the tile's 64 rows (rows past L are zeros
            // or the next sequence's keys; their A entries are masked by beta = 0)
            if (tid < 64) {
                const int R = tid;
                float ss = 0.f;
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const uint4 wv = ld_shared_v4(ktile + c * 8192 + R * 128 + (uint32_t(p ^ (R & 7)) << 4));
                        const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                        }
                    }
                vec[kVecIk + R] = inv_l2(ss);
            }
        }
        for (int j = 0; j < group; ++j) {
            const int h = hq * group + j;
            // gates of head h and their chunk-local prefix sums (warp 0, two tokens
            // per lane); tokens past the end get g = beta = 0
            if (warp == 0) {
                const bool ok0 = 2 * lane < L, ok1 = 2 * lane + 1 < L;
                float ga, gb, ba, bb;
                if (prefetch) {
                    const float *gs = reinterpret_cast<const float *>(smem + kOffGst) + buf * (kMaxGatedHeads * 128) + j * 128;
                    ga = gs[2 * lane]; gb = gs[2 * lane + 1]; ba = gs[64 + 2 * lane]; bb = gs[64 + 2 * lane + 1];
                } else {
                    const size_t i0 = size_t(t0 + 2 * lane) * hv + h, i1 = i0 + hv;
                    ga = ok0 ? a.g[i0] : 0.f; gb = ok1 ? a.g[i1] : 0.f;
                    ba = ok0 ? a.beta[i0] : 0.f; bb = ok1 ? a.beta[i1] : 0.f;
                }
                const float g0 = ok0 ? fmaxf(kLogits ? log_sigmoid_fast(ga) : ga, kGFloor) : 0.f;
                const float g1 = ok1 ? fmaxf(kLogits ? log_sigmoid_fast(gb) : gb, kGFloor) : 0.f;
                vec[kVecB + 2 * lane] = ok0 ? (kLogits ? sigmoid_fast(ba) : ba) : 0.f;
                vec[kVecB + 2 * lane + 1] = ok1 ? (kLogits ? sigmoid_fast(bb) : bb) : 0.f;
                float incl = g0 + g1;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float tt = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += tt;
                }
                const float excl = incl - (g0 + g1);
                vec[kVecG + 2 * lane] = excl + g0;
                vec[kVecG + 2 * lane + 1] = excl + g0 + g1;
                // the chunk loop takes its decays from these same sums
                reinterpret_cast<float2 *>(gcum + (size_t(gc) * hv + h) * 64)[lane] =
                    make_float2(excl + g0, excl + g0 + g1);
            }
            __syncthreads();
            // row and column scales of the mask.  While the chunk's total log-decay
            // is at least -80, Gamma is the rank-1 product e^(G_r) e^(-G_j):
            // row scale beta_r e^(G_r) (/||k_r||), column scale e^(-G_j) (/||k_j||);
            // otherwise row beta_r (/||k_r||), column (1/||k_j||) and the exponential
            // of the difference per entry.
            const bool rank1 = vec[kVecG + 63] >= -80.f;
            if (tid < 64) {
                const float G = vec[kVecG + tid], bt = vec[kVecB + tid];
                const float ik = kL2 ? vec[kVecIk + tid] : 1.f;
                vec[kVecRow + tid] = rank1 ? bt * __expf(G) * ik : bt * ik;
                vec[kVecCol + tid] = rank1 ? __expf(-G) * ik : ik;
                vec[kVecTp + tid] = bt * __expf(G) * ik;  // T' column scale beta gamma (/||k||)
            }
            if (j == 0) {  // the Gram is complete
                const bool ok = warp != 0 || mbar_wait(bars + 8 * kBarMma, ph_m);
                ph_m ^= 1u;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
                tc_fence_after();
            } else {
                __syncthreads();
            }
            // A from the Gram: warp w reads its lane quarter (rows 16 (w % 4) ..
            // + 15 in lanes 0-15) and 32 of the 64 columns; slices entirely above
            // the diagonal are zeros without a tensor-memory read
            {
                const int quarter = warp & 3, half = warp >> 2;
                const int r = 16 * quarter + (lane & 15);
                const bool valid = lane < 16;
                const float rs = vec[kVecRow + r], Gr = vec[kVecG + r];
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    const int j0 = 32 * half + 16 * sl;
                    float xo[16];
                    if (j0 / 16 > quarter) {  // warp-uniform: every entry has j > r
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) xo[jj] = 0.f;
                    } else {
                        float v[16], cs[16];
                        tmem_ld16(tmem + (uint32_t(32 * quarter) << 16) + uint32_t(j0), v);
#pragma unroll
                        for (int q = 0; q < 4; ++q) load4(vec + kVecCol + j0 + 4 * q, cs + 4 * q);
                        tmem_wait_ld();
                        if (rank1) {  // uniform across the CTA
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
                                xo[jj] = (j0 + jj < r) ? rs * cs[jj] * v[jj] : 0.f;
                        } else {
                            float gj[16];
#pragma unroll
                            for (int q = 0; q < 4; ++q) load4(vec + kVecG + j0 + 4 * q, gj + 4 * q);
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
                                xo[jj] = (j0 + jj < r) ? rs * cs[jj] * __expf(fminf(Gr - gj[jj], 0.f)) * v[jj] : 0.f;
                        }
                    }
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<float4 *>(Af + r * kLdA + j0 + 4 * q) =
                                make_float4(xo[4 * q], xo[4 * q + 1], xo[4 * q + 2], xo[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();  // the tensor-memory reads are ordered before the next item's Gram
            __syncthreads();
            invert_in_place(Af, Yb, tid);
            // T' = T diag(beta gamma (/||k||)) and T'' = T diag(beta) (bf16, row-major, T' then
            // T'') to the (chunk, head) slot: thread t stores 16 entries of row t / 4 of each
            {
                const int r = tid >> 2, c0 = (tid & 3) * 16;
                const float *src = Af + r * kLdA + c0;
                uint4 *dst = reinterpret_cast<uint4 *>(tinv + ((size_t(gc) * hv + h) * 128 + r) * 64 + c0);
                float tp[16], tpp[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float x[4], sp[4], sb[4];
                    load4(src + 4 * q, x);
                    load4(vec + kVecTp + c0 + 4 * q, sp);
                    load4(vec + kVecB + c0 + 4 * q, sb);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        tp[4 * q + u] = x[u] * sp[u];
                        tpp[4 * q + u] = x[u] * sb[u];
                    }
                }
                dst[0] = pack_bf16x8(tp);
                dst[1] = pack_bf16x8(tp + 8);
                dst[64 * 64 / 8] = pack_bf16x8(tpp);  // T'' tile: 64 x 64 entries on
                dst[64 * 64 / 8 + 1] = pack_bf16x8(tpp + 8);
            }
            __syncthreads();  // Af and the vectors are reused by the next head
        }
        if (aborted) break;
        // this item's K tile was read through the generic proxy too (norms): order
        // those reads before the tile buffer is refilled by the next prefetch
        fence_proxy_async_shared();
        __syncthreads();
        gc = ngc; hq = nhq; t0 = nt0; L = nL;
    }
    cp_async_wait_all();
    if (aborted && tid == 0 && total > 0) {
        // let this thread's tensor-core work drain (bounded) before the tensor
        // memory is freed
        mma_commit(bars + 8 * kBarMma);
        (void)mbar_wait(bars + 8 * kBarMma, ph_m);
        hdr->bad_index = -3;
        atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_chunk_inverse(const PrefillArgs &a, __nv_bfloat16 *tinv, float *gcum, int64_t max_chunks,
                                 cudaStream_t stream, int num_sms) {
    CUtensorMap mk;
    if (!make_map(&mk, a.k, a.hk, a.tokens)) return cudaErrorInvalidValue;
    const bool l2 = a.flags & GDN_FLAG_QK_L2NORM, logits = a.flags & GDN_FLAG_GATE_LOGITS;
    using KernFn = void (*)(CUtensorMap, PrefillArgs, __nv_bfloat16 *, float *);
    static const KernFn table[4] = {chunk_inverse_kernel<false, false>, chunk_inverse_kernel<false, true>,
                                    chunk_inverse_kernel<true, false>, chunk_inverse_kernel<true, true>};
    const KernFn kern = table[(l2 ? 2 : 0) + (logits ? 1 : 0)];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    if (e != cudaSuccess) return e;
    const int64_t items = max_chunks * a.hk;
    const int64_t cap = int64_t(num_sms) * 3;
    const int grid = int(items < cap ? items : cap);
    if (grid <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mk, a, tinv, gcum);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
