// gdn_chunk_chain.cu -- second kernel of the two-kernel tensor-core prefill:
// the state-carrying chunk loop, with the chunks' triangular factors T read
// from the first kernel (gdn_chunk_inv.cu) instead of inverted on the spot.
//
// Chunk algebra (chunk of L <= 64 tokens, start state S, everything as in the
// single-kernel path): G = prefix sums of g, gamma = e^G, Gamma_rj =
// e^(G_r - G_j), lambda_j = e^(G_(L-1) - G_j);
//   W = T diag(beta gamma) K,   U~ = T diag(beta) V,   U = U~ - W S^T,
//   O = diag(gamma) Q S^T + (Q K^T (.) Gamma) U,
//   S <- gamma_(L-1) S + U^T diag(lambda) K
// ("Gated Attention Architectures", sections 2 and 3: the WY representation
// with per-chunk cumulative decay; section 1: the decay-masked chunk output).
//
// Only two products carry the state from chunk to chunk, so they are the
// whole critical path, one instruction stream each (M = 128 rows = the value
// index of the state, accumulators in tensor memory):
//   (XU) [X1 | U^T] = [0 | U~^T] - S [-gamma Q; W]^T     N = 128, K = d_k
//        i.e. X1 = S (gamma Q)^T and U^T = U~^T - S W^T   (A = bf16 S, negated)
//   (SO) [S | X1] += U^T [diag(lambda) K | P^T]         N = 192, K = 64
//        i.e. S += U^T diag(lambda) K and X1 += U^T P^T = O^T,  P = Q K^T (.) Gamma
// so the output O^T ends in X1 and the state update and the output share one
// A operand (bf16 U^T in tensor memory).  Around them:
//   state warps (0-3)     before (XU): S -> bf16 copy, S <- gamma_(L-1) S
//   epilogue warps (4-7)  after (XU): U^T -> bf16; after (SO): O out (staged,
//                         one TMA store) and X1 zeroed
//   prep warps (8-15)     one chunk ahead, state-independent: gates, the
//                         Gram Q K^T (M = 64) and the mask P, T' = T diag(beta
//                         gamma) and T'' = T diag(beta), W^T = K^T T'^T (MMA)
//                         and its epilogue, the scaled copies -gamma Q and
//                         diag(lambda) K
//   warp 16 lane 0        issues (XU) and (SO)
//   warp 17 lane 0        issues U~^T = V^T T''^T (into U's columns, once the
//                         previous chunk's U has been read)
// Roles hand over through mbarriers; every wait is bounded, and a timeout
// records GDN_ERR_DEVICE_CHECK (bad_index -2) and ends the kernel after its
// own tensor-core work has drained.  With GDN_FLAG_QK_L2NORM the normalising
// factors 1/||q_r||, 1/||k_r|| are folded into -gamma Q, P, T' and
// diag(lambda) K (and T is the factor of the normalised keys).
//
// One CTA per SM (its shared memory and all 512 tensor-memory columns) takes
// (sequence, value head) units longest sequence first from an atomic counter.
#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThreads = 576;
constexpr int kWarpEpi = 4, kWarpPrep = 8, kWarpMmaA = 16, kWarpMmaB = 17;
constexpr int kBarState = 1, kBarEpi = 2, kBarPrep = 3;  // named barriers (128, 128, 256 threads)
constexpr int kPrepIssuer = 7 * 32;                      // prep thread index (warp 15 lane 0) issuing its MMAs and loads

// Shared memory (bytes from a 1024-byte-aligned base).  128-byte-swizzled
// tiles throughout ("atom columns" of 64 bf16 per 128-byte row).
//   slots (2, by chunk parity; TMA):  K 16 KB, Q 16 KB (two atom columns of
//     64 token rows each), T 8 KB (64 x 64; the prep scales it into T' in place)
//   stages (2, by chunk parity; written by the prep warps):
//     GQW  32 KB: per atom column of d_k, 64 rows of -gamma Q then 64 rows of W
//          (the N = 128 B operand of (XU), K-major); after (XU) the output tile
//          of the chunk is staged in its first 16 KB
//     KP   24 KB: diag(lambda) K (two N atoms of d_k, K = tokens) and P^T (one N
//          atom of output tokens): the N = 192 B operand of (SO), MN-major
//   T''  8 KB, V 16 KB (TMA), per-stage token vectors, barriers
constexpr uint32_t kSlotBytes = 40960, kSlotK = 0, kSlotQ = 16384, kSlotT = 32768;
constexpr uint32_t kOffSlot0 = 0;
constexpr uint32_t kStageBytes = 57344, kStGQW = 0, kStKP = 32768;
constexpr uint32_t kOffStage0 = 2 * kSlotBytes;                    // 81920
constexpr uint32_t kOffTpp = kOffStage0 + 2 * kStageBytes;         // 196608
constexpr uint32_t kOffV = kOffTpp + 8192;                         // 204800
constexpr uint32_t kOffVec0 = kOffV + 16384;                       // 221184
constexpr int kVecFloats = 12 * 64;
constexpr uint32_t kOffBar = kOffVec0 + 2 * kVecFloats * 4;        // 227328
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");
// per-token vectors of a stage (floats)
constexpr int kVecG = 0, kVecB = 64, kVecGam = 128, kVecTp = 192, kVecTpp = 256, kVecQs = 320, kVecKs = 384,
              kVecPr = 448, kVecPc = 512, kVecIk = 576, kVecIq = 640, kVecGr = 704;

// mbarriers
enum {
    kBSlot = 0,      // [2] TMA: K, Q, T of a chunk landed
    kBV = 2,         // TMA: V landed
    kBGram = 3,      // prep MMA: Gram done
    kBW = 4,         // prep MMA: W^T done
    kBTpp = 5,       // prep -> warp 17: T'' ready
    kBFull = 6,      // [2] prep -> chain: stage ready
    kBU = 8,         // U~ done
    kBSp = 9,        // state pass done
    kBX1 = 10,       // X1 zeroed (epilogue)
    kBXU = 11,       // (XU) done
    kBUe = 12,       // U^T -> bf16 done
    kBSO = 13,       // (SO) done
    kBStFree = 14,   // [2] stage free again (its output tile has left)
    kNumBars = 16
};

// Tensor-memory columns (128 lanes each)
constexpr uint32_t kColGram = 0;   // Q K^T, M = 64: row r in lane (r % 16) + 32 (r / 16)
constexpr uint32_t kColW = 64;     // W^T (fp32, 64 token columns)
constexpr uint32_t kColSb = 192;   // bf16 S (64 columns), then bf16 U^T in its first 32
constexpr uint32_t kColS = 256;    // fp32 S (128)
constexpr uint32_t kColX1 = 384;   // X1 = O^T (64), contiguous after S for (SO)
constexpr uint32_t kColU = 448;    // U^T (64), contiguous after X1 for (XU)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesSlot = 16384 + 16384 + 8192;
constexpr uint32_t kBytesV = 16384;

// A bounded wait by one polling warp of a group, then the group's named
// barrier (which also ORs the failure across the group).
__device__ __forceinline__ bool group_wait(bool poller, uint32_t bar, uint32_t parity, int bar_id, int count) {
    const bool ok = !poller || mbar_wait(bar, parity);
    return !named_sync_or(bar_id, count, !ok);
}

template <bool kL2, bool kLogits>
__global__ void __launch_bounds__(kThreads, 1)
chunk_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_t, const PrefillArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    const uint32_t bars = sb + kOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * kNumBars);
    int *s_unit = reinterpret_cast<int *>(smem + kOffBar + 8 * kNumBars + 4);
    // the chunks' total decays gamma_(L-1) for the state pass, by chunk index mod 4
    // (the prep warps run at most two chunks ahead of the state warps)
    float *gc_ring = reinterpret_cast<float *>(smem + kOffBar + 8 * kNumBars + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_bits = uint32_t((warp & 3) * 32) << 16;
    WsHeader *hdr = a.sched.hdr;
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
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
    grid_dep_wait();  // the schedule and the chunk inverses are written
    bool aborted = hdr->status != GDN_OK;

    const int hv = a.hv, hk = a.hk, group = hv / hk;
    const int total_units = aborted ? 0 : a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);

    // X1 starts at zero (afterwards each output epilogue leaves it zeroed)
    if (warp >= kWarpEpi && warp < kWarpPrep) {
        uint32_t z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st16u(tmem + lane_bits + kColX1 + 16 * c, z);
        tmem_wait_st();
        tc_fence_before();
        named_sync(kBarEpi, 128);
        if (tid == 32 * kWarpEpi) mbar_arrive(bar(kBX1));
    }

    const uint32_t id_gram = idesc_bf16(64, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 64, true, false);
    const uint32_t id_xu = idesc_bf16(128, 128, false, false, true);
    const uint32_t id_so = idesc_bf16(128, 192, false, true);

    uint32_t gn = 0;  // chunks this CTA has processed (selects slots, stages and barrier phases)
    for (;;) {
        if (__syncthreads_or(aborted)) break;
        if (tid == 0) *s_unit = int(atomicAdd(&hdr->next_unit, 1u));
        __syncthreads();
        const int unit = *s_unit;
        if (unit >= total_units) break;
        const int seq = a.sched.order[unit / hv];
        const int h = unit % hv, hq = h / group;
        const int t0 = a.sched.start[seq], len = a.sched.len[seq];
        const int nchunks = (len + 63) / 64;
        const int cbase = a.sched.chunk_base[seq];
        const size_t sbase = (size_t(seq) * hv + h) * 128 * 128;

        auto load_slot = [&](int c) {  // K, Q, T of chunk c of this unit
            const uint32_t s = (gn + uint32_t(c)) & 1u;
            const uint32_t dst = sb + kOffSlot0 + s * kSlotBytes;
            const uint32_t b = bar(kBSlot + int(s));
            mbar_arrive_expect_tx(b, kBytesSlot);
            const int tok = t0 + 64 * c;
            tma_load_3d(dst + kSlotK, &tm_k, 0, hq, tok, b);
            tma_load_3d(dst + kSlotK + 8192, &tm_k, 64, hq, tok, b);
            tma_load_3d(dst + kSlotQ, &tm_q, 0, hq, tok, b);
            tma_load_3d(dst + kSlotQ + 8192, &tm_q, 64, hq, tok, b);
            tma_load_2d(dst + kSlotT, &tm_t, 0, ((cbase + c) * hv + h) * 64, b);
        };
        auto load_v = [&](int c) {
            mbar_arrive_expect_tx(bar(kBV), kBytesV);
            tma_load_3d(sb + kOffV, &tm_v, 0, h, t0 + 64 * c, bar(kBV));
            tma_load_3d(sb + kOffV + 8192, &tm_v, 64, h, t0 + 64 * c, bar(kBV));
        };

        if (warp < kWarpEpi) {
            // ======================= state warps: thread = state row =======================
            const int row = (warp & 3) * 32 + lane;
            if (nchunks == 0) {
                // no tokens: the final state is the initial state
                if (a.s_final) {
                    float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128);
                    const float4 *src = reinterpret_cast<const float4 *>(a.s0 + sbase + size_t(row) * 128);
                    for (int c = 0; c < 32; ++c) dst[c] = a.s0 ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float v[32];
                    if (a.s0) {
                        const float *src = a.s0 + sbase + size_t(row) * 128 + 32 * c4;
#pragma unroll
                        for (int c = 0; c < 8; ++c) load4(src + 4 * c, v + 4 * c);
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) v[c] = 0.f;
                    }
                    tmem_st32(tmem + lane_bits + kColS + 32 * c4, v);
                }
                tmem_wait_st();
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    // this chunk's decay (prep) and the state after the previous chunk
                    if (!group_wait(warp == 0, bar(kBFull + int(b)), (gc >> 1) & 1u, kBarState, 128)) {
                        aborted = true;
                        break;
                    }
                    if (n > 0 && !group_wait(warp == 0, bar(kBSO), (gc - 1) & 1u, kBarState, 128)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                    const float gC = gc_ring[gc & 3u];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        float v[32];
                        tmem_ld32(tmem + lane_bits + kColS + 32 * p, v);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                        tmem_st16u(tmem + lane_bits + kColSb + 16 * p, pk);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= gC;
                        tmem_st32(tmem + lane_bits + kColS + 32 * p, v);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    named_sync(kBarState, 128);
                    if (tid == 0) mbar_arrive(bar(kBSp));
                }
                if (!aborted) {
                    // final state after the last chunk's update
                    const uint32_t gl = gn + uint32_t(nchunks) - 1u;
                    if (!group_wait(warp == 0, bar(kBSO), gl & 1u, kBarState, 128)) {
                        aborted = true;
                    } else {
                        tc_fence_after();
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            float v[32];
                            tmem_ld32(tmem + lane_bits + kColS + 32 * c4, v);
                            tmem_wait_ld();
                            if (a.s_final) {
                                float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128 + 32 * c4);
#pragma unroll
                                for (int c = 0; c < 8; ++c)
                                    dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                            }
                        }
                        tc_fence_before();
                    }
                }
            }
        } else if (warp < kWarpPrep) {
            // ==================== epilogue warps: thread = value row i ====================
            const int row = (warp & 3) * 32 + lane;
            const bool poller = warp == kWarpEpi;
            const int et = tid - 32 * kWarpEpi;  // 0..127
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                const int c0 = t0 + 64 * n, L = min(64, len - 64 * n);
                const uint32_t stage = sb + kOffStage0 + b * kStageBytes;
                // U^T -> bf16 A operand of (SO), in the first 32 columns of the bf16 S copy
                if (!group_wait(poller, bar(kBXU), gc & 1u, kBarEpi, 128)) { aborted = true; break; }
                tc_fence_after();
                {
                    float v[32];
                    uint32_t pk[16];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        tmem_ld32(tmem + lane_bits + kColU + 32 * p, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                        tmem_st16u(tmem + lane_bits + kColSb + 16 * p, pk);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                named_sync(kBarEpi, 128);
                if (et == 0) mbar_arrive(bar(kBUe));
                // O^T from X1 after (SO); X1 zeroed for the next (XU)
                if (!group_wait(poller, bar(kBSO), gc & 1u, kBarEpi, 128)) { aborted = true; break; }
                tc_fence_after();
                float o0[32], o1[32];
                {
                    uint32_t z[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) z[j] = 0u;
                    tmem_ld32(tmem + lane_bits + kColX1, o0);
                    tmem_ld32(tmem + lane_bits + kColX1 + 32, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c) tmem_st16u(tmem + lane_bits + kColX1 + 16 * c, z);
                    tmem_wait_st();
                }
                tc_fence_before();
                named_sync(kBarEpi, 128);
                if (et == 0) mbar_arrive(bar(kBX1));
                // stage the chunk's output token-major (rows of 256 bytes) in the GQW
                // region, which (XU) has finished reading
                {
                    __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffStage0 + b * kStageBytes + kStGQW);
#pragma unroll
                    for (int r = 0; r < 32; ++r) Ot[r * 128 + row] = __float2bfloat16_rn(o0[r]);
#pragma unroll
                    for (int r = 0; r < 32; ++r) Ot[(32 + r) * 128 + row] = __float2bfloat16_rn(o1[r]);
                }
                fence_proxy_async_shared();
                named_sync(kBarEpi, 128);
                if (L == 64) {
                    if (et == 0) {
                        tma_store_3d(&tm_o, stage + kStGQW, 0, h, c0);
                        bulk_commit();
                        bulk_wait_read();  // the tile has been read: the stage may be rewritten
                        mbar_arrive(bar(kBStFree + int(b)));
                    }
                } else {
                    for (int e = et; e < 64 * 16; e += 128) {
                        const int r = e >> 4, c = e & 15;
                        if (r < L) {
                            const uint4 val = *reinterpret_cast<const uint4 *>(smem + kOffStage0 + b * kStageBytes +
                                                                              kStGQW + r * 256 + c * 16);
                            *reinterpret_cast<uint4 *>(o + (size_t(c0 + r) * hv + h) * 128 + c * 8) = val;
                        }
                    }
                    named_sync(kBarEpi, 128);
                    if (et == 0) mbar_arrive(bar(kBStFree + int(b)));
                }
            }
        } else if (warp < kWarpMmaA) {
            // ============ prep warps: chunk n's state-independent operands ============
            const int pt = tid - 32 * kWarpPrep;  // 0..255
            const bool poller = warp == kWarpPrep;
            if (pt == kPrepIssuer && nchunks > 0) {
                load_slot(0);
                if (nchunks > 1) load_slot(1);
            }
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                const int c0 = t0 + 64 * n, L = min(64, len - 64 * n);
                float *vec = reinterpret_cast<float *>(smem + kOffVec0) + b * kVecFloats;
                const uint32_t slot = sb + kOffSlot0 + b * kSlotBytes;
                const uint32_t stage = sb + kOffStage0 + b * kStageBytes;
                if (!group_wait(poller, bar(kBSlot + int(b)), (gc >> 1) & 1u, kBarPrep, 256)) {
                    aborted = true;
                    break;
                }
                // Gram Q K^T (M = 64), one thread issues
                if (pt == kPrepIssuer) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t koff = (s >> 2) * 8192 + (s & 3) * 32;
                        mma_bf16(tmem + kColGram, smem_desc(slot + kSlotQ, 16, 1024) + uint64_t(koff >> 4),
                                 smem_desc(slot + kSlotK, 16, 1024) + uint64_t(koff >> 4), id_gram, s > 0);
                    }
                    mma_commit(bar(kBGram));
                }
                // gates and their chunk-local prefix sums (tokens past the end: g = beta = 0)
                if (warp == kWarpPrep) {
                    const bool ok0 = 2 * lane < L, ok1 = 2 * lane + 1 < L;
                    const size_t i0 = size_t(c0 + 2 * lane) * hv + h, i1 = i0 + hv;
                    const float ga = ok0 ? a.g[i0] : 0.f, gb = ok1 ? a.g[i1] : 0.f;
                    const float ba = ok0 ? a.beta[i0] : 0.f, bb = ok1 ? a.beta[i1] : 0.f;
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
                }
                if constexpr (kL2) {
                    // 1 / max(||x||, 1e-12) of the 64 k rows (pt 32..95) and q rows (pt 96..159)
                    if (pt >= 32 && pt < 160) {
                        const int R = (pt - 32) & 63;
                        const uint32_t tile = slot + (pt < 96 ? kSlotK : kSlotQ);
                        float ss = 0.f;
#pragma unroll
                        for (int c = 0; c < 2; ++c)
#pragma unroll
                            for (int p = 0; p < 8; ++p) {
                                const uint4 wv = ld_shared_v4(tile + c * 8192 + R * 128 + (uint32_t(p ^ (R & 7)) << 4));
                                const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                                }
                            }
                        vec[(pt < 96 ? kVecIk : kVecIq) + R] = inv_l2(ss);
                    }
                }
                named_sync(kBarPrep, 256);
                // per-token scales (tokens past the end: lambda = beta = 0)
                if (pt < 64) {
                    const float G = vec[kVecG + pt], bt = vec[kVecB + pt], gam = __expf(G);
                    const float ik = kL2 ? vec[kVecIk + pt] : 1.f, iq = kL2 ? vec[kVecIq + pt] : 1.f;
                    const float lam = pt < L ? __expf(vec[kVecG + L - 1] - G) : 0.f;
                    const bool rank1 = vec[kVecG + 63] >= -80.f;
                    vec[kVecGam + pt] = gam;
                    vec[kVecTp + pt] = bt * gam * ik;
                    vec[kVecTpp + pt] = bt;
                    vec[kVecQs + pt] = -gam * iq;
                    vec[kVecKs + pt] = lam * ik;
                    vec[kVecPr + pt] = rank1 ? gam * iq : iq;
                    vec[kVecPc + pt] = rank1 ? __expf(-G) * ik : ik;
                    vec[kVecGr + pt] = G;
                    if (pt == 63) gc_ring[gc & 3u] = gam;  // padded rows carry g = 0: G_63 = G_(L-1)
                }
                // T'' may be rewritten once the previous chunk's U~ is done; the stage once
                // its previous chunk's output has left
                {
                    bool ok = true;
                    if (poller) {
                        if (gc >= 1) ok = mbar_wait(bar(kBU), (gc - 1) & 1u);
                        if (ok && gc >= 2) ok = mbar_wait(bar(kBStFree + int(b)), ((gc >> 1) - 1) & 1u);
                    }
                    if (named_sync_or(kBarPrep, 256, !ok)) { aborted = true; break; }
                }
                // T' = T diag(beta gamma / ||k||) in place, T'' = T diag(beta): thread = 16 entries of row pt / 4
                {
                    const int r = pt >> 2;
                    uint4 w0[2];
                    uint32_t off[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int ch = (pt & 3) * 2 + q;
                        off[q] = uint32_t(r) * 128 + (uint32_t(ch ^ (r & 7)) << 4);
                        w0[q] = ld_shared_v4(slot + kSlotT + off[q]);
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int cb = ((pt & 3) * 2 + q) * 8;
                        const uint32_t ws[4] = {w0[q].x, w0[q].y, w0[q].z, w0[q].w};
                        float tp[8], tpp[8];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                            tp[2 * u] = lo * vec[kVecTp + cb + 2 * u];
                            tp[2 * u + 1] = hi * vec[kVecTp + cb + 2 * u + 1];
                            tpp[2 * u] = lo * vec[kVecTpp + cb + 2 * u];
                            tpp[2 * u + 1] = hi * vec[kVecTpp + cb + 2 * u + 1];
                        }
                        st_shared_v4(slot + kSlotT + off[q], pack_bf16x8(tp));
                        st_shared_v4(sb + kOffTpp + off[q], pack_bf16x8(tpp));
                    }
                }
                // diag(lambda / ||k||) K into the stage's KP region (same layout as the K tile)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = pt + 256 * i;  // 16-byte chunk: atom, row, chunk
                    const int atom = e >> 9, r = (e >> 3) & 63, ch = e & 7;
                    const uint32_t off = uint32_t(atom) * 8192 + uint32_t(r) * 128 + (uint32_t(ch ^ (r & 7)) << 4);
                    const uint4 wv = ld_shared_v4(slot + kSlotK + off);
                    const float sc = vec[kVecKs + r];
                    const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
                    float x[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        x[2 * u] = __uint_as_float(ws[u] << 16) * sc;
                        x[2 * u + 1] = __uint_as_float(ws[u] & 0xffff0000u) * sc;
                    }
                    st_shared_v4(stage + kStKP + off, pack_bf16x8(x));
                }
                fence_proxy_async_shared();
                named_sync(kBarPrep, 256);
                if (pt == 0) mbar_arrive(bar(kBTpp));
                // W^T = K^T T'^T (A = K MN-major, B = T' K-major), one thread issues
                if (pt == kPrepIssuer) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColW, smem_desc(slot + kSlotK, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(slot + kSlotT, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBW));
                }
                // P = Q K^T (.) Gamma (j <= r), stored transposed (P^T, MN-major B of (SO))
                if (!group_wait(poller, bar(kBGram), gc & 1u, kBarPrep, 256)) { aborted = true; break; }
                tc_fence_after();
                {
                    const int quarter = warp & 3, half = (warp - kWarpPrep) >> 2;
                    const int r = 16 * quarter + (lane & 15);  // query token (row of P)
                    const bool valid = lane < 16;
                    const bool rank1 = vec[kVecG + 63] >= -80.f;
                    const float pr = vec[kVecPr + r], Gr = vec[kVecGr + r];
                    const uint32_t pbase = stage + kStKP + 16384;
#pragma unroll
                    for (int sl = 0; sl < 2; ++sl) {
                        const int j0 = 32 * half + 16 * sl;
                        float v[16], pc[16], gj[16];
                        tmem_ld16(tmem + lane_bits + kColGram + uint32_t(j0), v);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            load4(vec + kVecPc + j0 + 4 * q, pc + 4 * q);
                            load4(vec + kVecGr + j0 + 4 * q, gj + 4 * q);
                        }
                        tmem_wait_ld();
                        if (valid) {
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) {
                                const int j = j0 + jj;  // key token (row of P^T)
                                const float keep = (j <= r) ? 1.f : 0.f;
                                const float x = rank1 ? keep * pr * pc[jj] * v[jj]
                                                      : keep * pr * pc[jj] * __expf(fminf(Gr - gj[jj], 0.f)) * v[jj];
                                st_shared_b16(pbase + uint32_t(j) * 128 + (uint32_t((r >> 3) ^ (j & 7)) << 4) +
                                                  uint32_t(r & 7) * 2,
                                              x);
                            }
                        }
                    }
                }
                // -gamma Q / ||q|| into the stage's GQW rows 0-63 (the Gram has read Q)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = pt + 256 * i;
                    const int atom = e >> 9, r = (e >> 3) & 63, ch = e & 7;
                    const uint32_t soff = uint32_t(atom) * 8192 + uint32_t(r) * 128 + (uint32_t(ch ^ (r & 7)) << 4);
                    const uint32_t doff = uint32_t(atom) * 16384 + uint32_t(r) * 128 + (uint32_t(ch ^ (r & 7)) << 4);
                    const uint4 wv = ld_shared_v4(slot + kSlotQ + soff);
                    const float sc = vec[kVecQs + r];
                    const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
                    float x[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        x[2 * u] = __uint_as_float(ws[u] << 16) * sc;
                        x[2 * u + 1] = __uint_as_float(ws[u] & 0xffff0000u) * sc;
                    }
                    st_shared_v4(stage + kStGQW + doff, pack_bf16x8(x));
                }
                // W rows (token-major, d_k contiguous) into the stage's GQW rows 64-127
                if (!group_wait(poller, bar(kBW), gc & 1u, kBarPrep, 256)) { aborted = true; break; }
                tc_fence_after();
                {
                    const int half = (warp - kWarpPrep) >> 2;
                    const int c = (warp & 3) * 32 + lane;  // d_k index = tensor-memory lane
                    float v[32];
                    tmem_ld32(tmem + lane_bits + kColW + 32 * half, v);
                    tmem_wait_ld();
                    const uint32_t wb = stage + kStGQW + uint32_t(c >> 6) * 16384 + uint32_t(c & 7) * 2;
                    const uint32_t c8 = uint32_t(c & 63) >> 3;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int r = 32 * half + j;
                        st_shared_b16(wb + uint32_t(64 + r) * 128 + ((c8 ^ uint32_t(r & 7)) << 4), v[j]);
                    }
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarPrep, 256);
                if (pt == 0) mbar_arrive(bar(kBFull + int(b)));
                // every read of this slot is done (Gram, W^T, the copies): chunk n + 2 may come in
                if (pt == kPrepIssuer && n + 2 < nchunks) load_slot(n + 2);
            }
        } else if (warp == kWarpMmaA) {
            // ==================== warp 16: the state-carrying products ====================
            if (lane == 0) {
                if (nchunks > 0) load_v(0);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t stage = sb + kOffStage0 + b * kStageBytes;
                    bool ok = mbar_wait(bar(kBFull + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBSp), gc & 1u) &&
                              mbar_wait(bar(kBU), gc & 1u) && mbar_wait(bar(kBX1), gc & 1u);
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
                    // (XU): [X1 | U^T] = [0 | U~^T] - S [-gamma Q; W]^T
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                        mma_bf16_ts(tmem + kColX1, tmem + kColSb + 8 * s,
                                    smem_desc(stage + kStGQW, 16, 1024) + uint64_t(off >> 4), id_xu, 1);
                    }
                    mma_commit(bar(kBXU));
                    // U~ of this chunk is done: V of the next may come in
                    if (n + 1 < nchunks) load_v(n + 1);
                    if (!mbar_wait(bar(kBUe), gc & 1u)) { aborted = true; break; }
                    tc_fence_after();
                    // (SO): [S | X1] += U^T [diag(lambda) K | P^T]
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColS, tmem + kColSb + 8 * s,
                                    smem_desc(stage + kStKP, 8192, 1024) + uint64_t((s * 2048) >> 4), id_so, 1);
                    mma_commit(bar(kBSO));
                }
            }
        } else {
            // ========================= warp 17: U~^T = V^T T''^T =========================
            if (lane == 0) {
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n);
                    bool ok = mbar_wait(bar(kBTpp), gc & 1u) && mbar_wait(bar(kBV), gc & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBUe), (gc - 1) & 1u);  // the previous U has been read
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColU, smem_desc(sb + kOffV, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(sb + kOffTpp, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBU));
                }
            }
        }
        gn += uint32_t(nchunks);
    }

    if (warp >= kWarpEpi && warp < kWarpPrep && tid == 32 * kWarpEpi) bulk_wait_all();
    if (aborted) {
        // let this thread's own tensor-core work drain (bounded) before the tensor
        // memory is freed
        if ((warp == kWarpMmaA || warp == kWarpMmaB) && lane == 0) {
            mma_commit(bar(warp == kWarpMmaA ? kBSO : kBU));
            (void)mbar_wait(bar(warp == kWarpMmaA ? kBSO : kBU), 0u);
            (void)mbar_wait(bar(warp == kWarpMmaA ? kBSO : kBU), 1u);
        }
        if (tid == 32 * kWarpPrep + kPrepIssuer) {
            mma_commit(bar(kBW));
            (void)mbar_wait(bar(kBW), 0u);
            (void)mbar_wait(bar(kBW), 1u);
        }
        if (tid == 0) {
            hdr->bad_index = -2;
            atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool chunk_split_supported(const gdn_shape_t &s) {
    return s.dtype == GDN_DTYPE_BF16 && s.head_dim_k == 128 && s.head_dim_v == 128 && s.chunk_size == 64;
}

cudaError_t launch_chunk_chain(const PrefillArgs &a, const __nv_bfloat16 *tinv, int64_t max_chunks,
                               cudaStream_t stream, int num_sms) {
    CUtensorMap mq, mk, mv, mo, mt;
    if (!make_map(&mq, a.q, a.hk, a.tokens) || !make_map(&mk, a.k, a.hk, a.tokens) ||
        !make_map(&mv, a.v, a.hv, a.tokens) || !make_map(&mo, a.o, a.hv, a.tokens, true) ||
        !make_tile_map(&mt, tinv, max_chunks * a.hv * 64))
        return cudaErrorInvalidValue;
    const bool l2 = a.flags & GDN_FLAG_QK_L2NORM, logits = a.flags & GDN_FLAG_GATE_LOGITS;
    using KernFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, PrefillArgs);
    static const KernFn table[4] = {chunk_chain_kernel<false, false>, chunk_chain_kernel<false, true>,
                                    chunk_chain_kernel<true, false>, chunk_chain_kernel<true, true>};
    const KernFn kern = table[(l2 ? 2 : 0) + (logits ? 1 : 0)];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t(a.num_seqs) * a.hv;
    const int grid = int(units < num_sms ? units : num_sms);
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
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, mt, a);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
