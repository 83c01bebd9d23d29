// gdn_chunk_chain.cu -- second kernel of the two-kernel tensor-core prefill:
// the state-carrying chunk loop, with the chunks' scaled WY factors
// T' = T diag(beta gamma) and T'' = T diag(beta) read from the first kernel
// (gdn_chunk_inv.cu) instead of inverted on the spot.
//
// Chunk algebra (chunk of L <= 64 tokens, start state S, everything as in the
// single-kernel path): G = prefix sums of g, gamma = e^G, Gamma_rj =
// e^(G_r - G_j), lambda_j = e^(G_(L-1) - G_j);
//   W = T' K,   U~ = T'' V,   U = U~ - W S^T,
//   O = diag(gamma) Q S^T + (Q K^T (.) Gamma) U,
//   S <- gamma_(L-1) S + U^T diag(lambda) K
// ("Gated Attention Architectures", sections 2 and 3: the WY representation
// with per-chunk cumulative decay; section 1: the decay-masked chunk output).
//
// Every product is one tcgen05.mma stream with M = 128 rows (the value index
// of the state, or the key index for W), fp32 accumulators in tensor memory:
//   (W)   W^T  = K^T T'^T             128 x 64 x 64     warp 14
//   (U~)  U~^T = V^T T''^T            128 x 64 x 64     warp 13
//   (XU)  U^T  = U~^T - S W^T         128 x 64 x 128    warp 12   } the state's
//   (S7)  S   += (U^T diag(lambda)) K 128 x 128 x 64    warp 12   } critical path
//   (X1)  X1' = -S Q^T                128 x 64 x 128    warp 15
//   (X6)  X2   = U^T P^T              128 x 64 x 64     warp 15
// and the Gram Q K^T (M = 64) for P = Q K^T (.) Gamma.  O^T = X2 - X1' diag(gamma).
// Operands come straight from the TMA tiles wherever their layout allows: K
// and Q (token-major, 128-byte swizzle) serve as the K-major and MN-major
// operands they are; W^T is written by its epilogue in the MN-major layout of
// the (XU) operand (16-byte stores), P row by row K-major.  The bf16 copies of
// S, U^T and U^T diag(lambda) are A operands in tensor memory.
//
// Roles (16 warps):
//   state warps (0-3)     before (XU): S -> bf16 copy, S <- gamma_(L-1) S
//                         (state columns 0-95)
//   epilogue warps (4-7)  after (XU): U^T -> bf16, U^T diag(lambda) -> bf16;
//                         after (X1), (X6): O staged and stored by TMA; then the
//                         state pass of columns 96-127 for the next chunk
//   prep warps (8-11)     one chunk ahead, state-independent: per-token scales
//                         from the chunk's prefix sums G (computed by the factor
//                         kernel, which took the same sums for T'; they arrive
//                         with T' and T''), the mask P from the Gram, the
//                         epilogue of W^T
//   warps 12, 13, 14, 15  lane 0 issues the products above (14: Gram and W)
// Tiles: K and Q in a ring of three chunks, T' and T'' in two, W^T and P in
// two, V in one.  Tensor-memory loads of a role are issued together and waited
// for once.  Roles hand over through mbarriers; every wait is bounded,
// and a timeout records GDN_ERR_DEVICE_CHECK (bad_index -2) and ends the
// kernel after its own tensor-core work has drained.  With
// GDN_FLAG_QK_L2NORM the factors 1/||q_r||, 1/||k_r|| are folded into P, the
// U^T diag(lambda) copy and the output combination (T' carries its own).
//
// One CTA per SM (its shared memory and all 512 tensor-memory columns) takes
// (sequence, value head) units longest sequence first from an atomic counter.
#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThreads = 512;
constexpr int kWarpEpi = 4, kWarpPrep = 8, kWarpA = 12, kWarpB = 13, kWarpP = 14, kWarpC = 15;
constexpr int kBarState = 1, kBarEpi = 2, kBarPrep = 3;  // named barriers (128 threads each)
constexpr int kSpCols = 96;  // state columns the state warps pass; the epilogue warps take the rest

// Shared memory (bytes from a 1024-byte-aligned base).  128-byte-swizzled tiles
// ("atom columns" of 64 bf16 per 128-byte row).
constexpr uint32_t kKQBytes = 32768, kKQ_K = 0, kKQ_Q = 16384;       // [3]: K, Q (2 atoms x 64 token rows)
constexpr uint32_t kOffKQ = 0;
constexpr uint32_t kTBytes = 16384, kT_P = 0, kT_PP = 8192;           // [2]: T', T'' (64 x 64)
constexpr uint32_t kOffT = kOffKQ + 3 * kKQBytes;                     // 98304
constexpr uint32_t kWPBytes = 24576, kWP_W = 0, kWP_P = 16384;        // [2]: W^T (128 d_k rows x 64 tokens), P
constexpr uint32_t kOffWP = kOffT + 2 * kTBytes;                      // 131072
constexpr uint32_t kOffV = kOffWP + 2 * kWPBytes;                     // 180224: V (2 atoms x 64 rows)
constexpr uint32_t kOffOst = kOffV + 16384;                           // 196608: output tile, 64 tokens x 256 B
constexpr uint32_t kOffVec = kOffOst + 16384;                         // 212992: token vectors [4]
constexpr int kVecFloats = 10 * 64;
constexpr uint32_t kOffBar = kOffVec + 4 * kVecFloats * 4;            // 223232
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");
// token vectors of a chunk (floats)
constexpr int kVecG = 0, kVecGam = 128, kVecLam = 192, kVecPr = 256, kVecPc = 320, kVecGo = 384,
              kVecIk = 448, kVecIq = 512, kVecRank1 = 576;

// mbarriers (arrival count 1 unless noted)
enum {
    kBKQ = 0,     // [3] TMA: K and Q of a chunk landed
    kBT = 3,      // [2] TMA: T', T'' of a chunk landed
    kBV = 5,      // TMA: V landed
    kBGram = 6,   // Gram done
    kBGFree = 7,  // prep -> warp 14: Gram read
    kBW = 8,      // W^T done
    kBFull = 9,   // [2] prep -> chain: W^T, P and the token vectors of a chunk ready
    kBU = 11,     // U~ done
    kBSp = 12,    // state pass done (count 2: state and epilogue warps)
    kBXU = 13,    // (XU) done
    kBX1 = 14,    // (X1) done
    kBUe = 15,    // bf16 U^T copies written
    kBS7 = 16,    // (S7) done
    kBX6 = 17,    // (X6) done
    kBOut = 18,   // X1' and X2 read by the output epilogue
    kBWPFree = 19,  // [2] W^T and P of a stage read
    kNumBars = 21
};

// Tensor-memory columns (128 lanes each)
constexpr uint32_t kColGram = 0;   // Q K^T, M = 64: row r in lane (r % 16) + 32 (r / 16)
constexpr uint32_t kColW = 64;     // W^T (fp32, 64 token columns)
constexpr uint32_t kColU = 128;    // U^T
constexpr uint32_t kColX1 = 192;   // X1'
constexpr uint32_t kColS = 256;    // fp32 S (128)
constexpr uint32_t kColX2 = 384;   // X2
constexpr uint32_t kColSb = 448;   // bf16 S (64 columns); then bf16 U^T (32) and U^T diag(lambda) (32)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesKQ = 32768, kBytesT = 16384, kBytesV = 16384;

// A bounded wait by one polling warp of a group, then the group's named
// barrier (which also ORs the failure across the group).
__device__ __forceinline__ bool group_wait(bool poller, uint32_t bar, uint32_t parity, int bar_id, int count) {
    const bool ok = !poller || mbar_wait(bar, parity);
    return !named_sync_or(bar_id, count, !ok);
}

// The state pass of columns [c0, c0 + 32 kSlices) of this thread's state row:
// the bf16 copy (A operand of (XU), (X1)) and S <- gC S in place.  Slices are
// read two at a time, with one wait per pair.
__device__ __forceinline__ void state_slice(uint32_t tmem_row, int c, float gC, float (&v)[32]) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
    tmem_st16u(tmem_row + kColSb + uint32_t(c / 2), pk);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= gC;
    tmem_st32(tmem_row + kColS + uint32_t(c), v);
}
template <int kSlices>
__device__ __forceinline__ void state_pass(uint32_t tmem_row, int c0, float gC) {
#pragma unroll
    for (int p = 0; p < kSlices; p += 2) {
        float v0[32], v1[32];
        tmem_ld32(tmem_row + kColS + uint32_t(c0 + 32 * p), v0);
        if (p + 1 < kSlices) tmem_ld32(tmem_row + kColS + uint32_t(c0 + 32 * p + 32), v1);
        tmem_wait_ld();
        state_slice(tmem_row, c0 + 32 * p, gC, v0);
        if (p + 1 < kSlices) state_slice(tmem_row, c0 + 32 * p + 32, gC, v1);
    }
    tmem_wait_st();
}

// State columns [c0, c0 + 32 kSlices) of this row between global and tensor memory.
template <int kSlices>
__device__ __forceinline__ void state_in(uint32_t tmem_row, const float *src, int c0) {
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
__device__ __forceinline__ void state_out(uint32_t tmem_row, float *dst, int c0) {
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

template <bool kL2>
__global__ void __launch_bounds__(kThreads, 1)
chunk_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_t, const PrefillArgs a, const float *gcum) {
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
    auto vecs = [&](uint32_t gc) { return reinterpret_cast<float *>(smem + kOffVec) + (gc & 3u) * kVecFloats; };

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
    grid_dep_wait();  // the schedule and the chunk factors are written
    bool aborted = hdr->status != GDN_OK;

    const int hv = a.hv, hk = a.hk, group = hv / hk;
    const int total_units = aborted ? 0 : a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);

    const uint32_t id_gram = idesc_bf16(64, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 64, true, false);      // also U~ (A = V MN-major)
    const uint32_t id_xu = idesc_bf16(128, 64, false, true, true);
    const uint32_t id_x1 = idesc_bf16(128, 64, false, false, true);
    const uint32_t id_s7 = idesc_bf16(128, 128, false, true);
    const uint32_t id_x6 = idesc_bf16(128, 64, false, false);

    uint32_t gn = 0;  // chunks this CTA has processed (selects buffers and barrier phases)
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

        auto load_kq = [&](int c) {  // K, Q of chunk c of this unit
            const uint32_t gc = gn + uint32_t(c), i = gc % 3u;
            const uint32_t dst = sb + kOffKQ + i * kKQBytes;
            const uint32_t b = bar(kBKQ + int(i));
            mbar_arrive_expect_tx(b, kBytesKQ);
            const int tok = t0 + 64 * c;
            tma_load_3d(dst + kKQ_K, &tm_k, 0, hq, tok, b);
            tma_load_3d(dst + kKQ_K + 8192, &tm_k, 64, hq, tok, b);
            tma_load_3d(dst + kKQ_Q, &tm_q, 0, hq, tok, b);
            tma_load_3d(dst + kKQ_Q + 8192, &tm_q, 64, hq, tok, b);
        };
        auto load_t = [&](int c) {  // T', T'' and the prefix sums G of chunk c
            const uint32_t gc = gn + uint32_t(c), i = gc & 1u;
            const uint32_t dst = sb + kOffT + i * kTBytes;
            const uint32_t b = bar(kBT + int(i));
            mbar_arrive_expect_tx(b, kBytesT + 256);
            const int row = ((cbase + c) * hv + h) * 128;
            tma_load_2d(dst + kT_P, &tm_t, 0, row, b);
            tma_load_2d(dst + kT_PP, &tm_t, 0, row + 64, b);
            bulk_load(sb + kOffVec + (gc & 3u) * (kVecFloats * 4) + kVecG * 4,
                      gcum + (size_t(cbase + c) * hv + h) * 64, 256, b);
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
                // no tokens: the final state is the initial state
                if (a.s_final) {
                    float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128);
                    const float4 *src = a.s0 ? reinterpret_cast<const float4 *>(a.s0 + sbase + size_t(row) * 128)
                                             : nullptr;
                    for (int c = 0; c < 32; ++c) dst[c] = src ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
                state_in<kSpCols / 32>(trow, a.s0 ? a.s0 + sbase + size_t(row) * 128 : nullptr, 0);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n);
                    // this chunk's decay (prep), the state after the previous chunk and the
                    // bf16 region free again (both products of the previous chunk done)
                    bool ok = true;
                    if (warp == 0) {
                        ok = mbar_wait(bar(kBFull + int(gc & 1u)), (gc >> 1) & 1u);
                        if (ok && n > 0) ok = mbar_wait(bar(kBS7), (gc - 1) & 1u) && mbar_wait(bar(kBX6), (gc - 1) & 1u);
                    }
                    if (named_sync_or(kBarState, 128, !ok)) { aborted = true; break; }
                    tc_fence_after();
                    state_pass<kSpCols / 32>(trow, 0, vecs(gc)[kVecGam + 63]);
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
                        state_out<kSpCols / 32>(trow, a.s_final ? a.s_final + sbase + size_t(row) * 128 : nullptr, 0);
                        tc_fence_before();
                    }
                }
            }
        } else if (warp < kWarpPrep) {
            // ==================== epilogue warps: thread = value row i ====================
            const int row = (warp & 3) * 32 + lane;
            const uint32_t trow = tmem + lane_bits;
            const bool poller = warp == kWarpEpi;
            const int et = tid - 32 * kWarpEpi;  // 0..127
            float *sf_row = a.s_final ? a.s_final + sbase + size_t(row) * 128 : nullptr;
            if (nchunks > 0) {
                // the initial state of columns kSpCols..127 and their state pass for chunk 0
                state_in<(128 - kSpCols) / 32>(trow, a.s0 ? a.s0 + sbase + size_t(row) * 128 : nullptr, kSpCols);
                if (!group_wait(poller, bar(kBFull + int(gn & 1u)), (gn >> 1) & 1u, kBarEpi, 128)) {
                    aborted = true;
                } else {
                    tc_fence_after();
                    state_pass<(128 - kSpCols) / 32>(trow, kSpCols, vecs(gn)[kVecGam + 63]);
                    tc_fence_before();
                    named_sync(kBarEpi, 128);
                    if (et == 0) mbar_arrive(bar(kBSp));
                }
            }
            for (int n = 0; n < nchunks && !aborted; ++n) {
                const uint32_t gc = gn + uint32_t(n);
                const int c0 = t0 + 64 * n, L = min(64, len - 64 * n);
                const float *vec = vecs(gc);
                // U^T and U^T diag(lambda (/||k||)) -> bf16 A operands of (X6) and (S7), over
                // the bf16 S that (XU) and (X1) read
                {
                    bool ok = true;
                    if (poller) ok = mbar_wait(bar(kBXU), gc & 1u) && mbar_wait(bar(kBX1), gc & 1u);
                    if (named_sync_or(kBarEpi, 128, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                {
                    float v[2][32];
                    tmem_ld32(trow + kColU, v[0]);
                    tmem_ld32(trow + kColU + 32, v[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        uint32_t pu[16], pl[16];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float l[4];
                            load4(vec + kVecLam + 32 * p + 4 * q, l);
                            pu[2 * q] = pack_bf16x2(v[p][4 * q], v[p][4 * q + 1]);
                            pu[2 * q + 1] = pack_bf16x2(v[p][4 * q + 2], v[p][4 * q + 3]);
                            pl[2 * q] = pack_bf16x2(l[0] * v[p][4 * q], l[1] * v[p][4 * q + 1]);
                            pl[2 * q + 1] = pack_bf16x2(l[2] * v[p][4 * q + 2], l[3] * v[p][4 * q + 3]);
                        }
                        tmem_st16u(trow + kColSb + 16 * p, pu);
                        tmem_st16u(trow + kColSb + 32 + 16 * p, pl);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                named_sync(kBarEpi, 128);
                if (et == 0) mbar_arrive(bar(kBUe));
                // O^T = X2 - X1' diag(gamma (/||q||)), staged token-major (rows of 256 bytes)
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
                        for (int r = 0; r < 32; ++r)
                            Ot[(32 * p + r) * 128 + row] = __float2bfloat16_rn(fmaf(-vec[kVecGo + 32 * p + r], x1[r], x2[r]));
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
                        state_pass<(128 - kSpCols) / 32>(trow, kSpCols, vecs(g1)[kVecGam + 63]);
                        tc_fence_before();
                        named_sync(kBarEpi, 128);
                        if (et == 0) mbar_arrive(bar(kBSp));
                    } else {
                        state_out<(128 - kSpCols) / 32>(trow, sf_row, kSpCols);
                        tc_fence_before();
                    }
                }
            }
        } else if (warp < kWarpA) {
            // ============ prep warps: chunk n's state-independent operands ============
            const int pt = tid - 32 * kWarpPrep;  // 0..127
            const bool poller = warp == kWarpPrep;
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                const int L = min(64, len - 64 * n);
                float *vec = vecs(gc);
                const uint32_t kq = sb + kOffKQ + (gc % 3u) * kKQBytes;
                const uint32_t wp = sb + kOffWP + b * kWPBytes;
                // the chunk's prefix sums G arrive with its T' and T''
                if (!group_wait(poller, bar(kBT + int(b)), (gc >> 1) & 1u, kBarPrep, 128)) { aborted = true; break; }
                if constexpr (kL2) {
                    // 1 / max(||x||, 1e-12) of the 64 k rows (pt 0..63) and q rows (pt 64..127)
                    if (!group_wait(warp == kWarpPrep + 1, bar(kBKQ + int(gc % 3u)), (gc / 3u) & 1u, kBarPrep, 128)) {
                        aborted = true;
                        break;
                    }
                    {
                        const int R = pt & 63;
                        const uint32_t tile = kq + (pt < 64 ? kKQ_K : kKQ_Q);
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
                        vec[(pt < 64 ? kVecIk : kVecIq) + R] = inv_l2(ss);
                    }
                    named_sync(kBarPrep, 128);
                }
                // per-token scales (tokens past the end: lambda = 0)
                if (pt < 64) {
                    const float G = vec[kVecG + pt], gam = __expf(G);
                    const float ik = kL2 ? vec[kVecIk + pt] : 1.f, iq = kL2 ? vec[kVecIq + pt] : 1.f;
                    const float lam = pt < L ? __expf(vec[kVecG + L - 1] - G) : 0.f;
                    const bool rank1 = vec[kVecG + 63] >= -80.f;
                    vec[kVecGam + pt] = gam;  // G_63 = G_(L-1): padded rows carry g = 0
                    vec[kVecLam + pt] = lam * ik;
                    vec[kVecGo + pt] = gam * iq;
                    vec[kVecPr + pt] = rank1 ? gam * iq : iq;
                    vec[kVecPc + pt] = rank1 ? __expf(-G) * ik : ik;
                    if (pt == 63) vec[kVecRank1] = rank1 ? 1.f : 0.f;
                }
                // the stage's W^T and P were read by the chunk two back
                if (!group_wait(poller && gc >= 2, bar(kBWPFree + int(b)), ((gc >> 1) - 1) & 1u, kBarPrep, 128)) {
                    aborted = true;
                    break;
                }
                // P = Q K^T (.) Gamma (j <= r), row by row (K-major B of (X6)); slices with
                // every j above the quarter's rows are zeros without a tensor-memory read
                if (!group_wait(poller, bar(kBGram), gc & 1u, kBarPrep, 128)) { aborted = true; break; }
                tc_fence_after();
                {
                    const int quarter = warp & 3;
                    const int r = 16 * quarter + (lane & 15);  // query token (row of P)
                    const bool valid = lane < 16;
                    const bool rank1 = vec[kVecRank1] != 0.f;
                    const float pr = vec[kVecPr + r], Gr = vec[kVecG + r];
                    // the warp's slices two at a time: both tensor-memory loads, one wait
#pragma unroll
                    for (int s2 = 0; s2 < 4; s2 += 2) {
                        float v[2][16];
#pragma unroll
                        for (int u = 0; u < 2; ++u)
                            if (s2 + u <= quarter) tmem_ld16(tmem + lane_bits + kColGram + uint32_t(16 * (s2 + u)), v[u]);
                        if (s2 <= quarter) tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int sl = s2 + u, j0 = 16 * sl;
                            float x[16];
                            if (sl > quarter) {  // warp-uniform: every entry has j > r
#pragma unroll
                                for (int jj = 0; jj < 16; ++jj) x[jj] = 0.f;
                            } else {
                                float pc[16];
#pragma unroll
                                for (int q = 0; q < 4; ++q) load4(vec + kVecPc + j0 + 4 * q, pc + 4 * q);
                                if (rank1) {
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj) x[jj] = (j0 + jj <= r) ? pr * pc[jj] * v[u][jj] : 0.f;
                                } else {
                                    float gj[16];
#pragma unroll
                                    for (int q = 0; q < 4; ++q) load4(vec + kVecG + j0 + 4 * q, gj + 4 * q);
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj)
                                        x[jj] = (j0 + jj <= r) ? pr * pc[jj] * __expf(fminf(Gr - gj[jj], 0.f)) * v[u][jj]
                                                               : 0.f;
                                }
                            }
                            if (valid) {
                                const uint32_t base = wp + kWP_P + uint32_t(r) * 128;
                                st_shared_v4(base + (uint32_t((2 * sl) ^ (r & 7)) << 4), pack_bf16x8(x));
                                st_shared_v4(base + (uint32_t((2 * sl + 1) ^ (r & 7)) << 4), pack_bf16x8(x + 8));
                            }
                        }
                    }
                }
                tc_fence_before();
                // W^T rows (d_k index, 64 tokens) in the MN-major layout of the (XU) operand
                if (!group_wait(poller, bar(kBW), gc & 1u, kBarPrep, 128)) { aborted = true; break; }
                if (pt == 0) mbar_arrive(bar(kBGFree));  // the Gram has been read
                tc_fence_after();
                {
                    const int c = (warp & 3) * 32 + lane;  // d_k index = tensor-memory lane
                    const uint32_t base = wp + kWP_W + uint32_t(c) * 128;
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
                if (nchunks > 1) load_kq(1);
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t wp = sb + kOffWP + b * kWPBytes;
                    const uint32_t kq = sb + kOffKQ + (gc % 3u) * kKQBytes;
                    bool ok = mbar_wait(bar(kBFull + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBSp), gc & 1u) &&
                              mbar_wait(bar(kBU), gc & 1u);
                    if (!ok) { aborted = true; break; }
                    // the previous chunk's products are done (the state pass waited for them):
                    // its K, Q buffer takes chunk n + 2
                    if (n + 2 < nchunks) load_kq(n + 2);
                    tc_fence_after();
                    // (XU): U^T = U~^T - S W^T (A = bf16 S negated, B = W^T MN-major)
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        mma_bf16_ts(tmem + kColU, tmem + kColSb + 8 * s,
                                    smem_desc(wp + kWP_W, 8192, 1024) + uint64_t((s * 2048) >> 4), id_xu, 1);
                    mma_commit(bar(kBXU));
                    if (!mbar_wait(bar(kBUe), gc & 1u)) { aborted = true; break; }
                    tc_fence_after();
                    // (S7): S += (U^T diag(lambda)) K (B = K MN-major)
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColS, tmem + kColSb + 32 + 8 * s,
                                    smem_desc(kq + kKQ_K, 8192, 1024) + uint64_t((s * 2048) >> 4), id_s7, 1);
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
                    const uint32_t tt = sb + kOffT + b * kTBytes;
                    bool ok = mbar_wait(bar(kBT + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBV), gc & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBUe), (gc - 1) & 1u);  // the previous U has been read
                    if (!ok) { aborted = true; break; }
                    // the previous chunk's T' and T'' are no longer read (its U~ and W^T are
                    // done): that buffer takes chunk n + 1
                    if (n >= 1 && n + 1 < nchunks) load_t(n + 1);
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColU, smem_desc(sb + kOffV, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(tt + kT_PP, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBU));
                    // V has been read once U~ is done: the next chunk's V takes its place
                    if (n + 1 < nchunks) {
                        if (!mbar_wait(bar(kBU), gc & 1u)) { aborted = true; break; }
                        load_v(n + 1);
                    }
                }
            }
        } else if (warp == kWarpP) {
            // ============ warp 14: the Gram Q K^T (M = 64) and W^T = K^T T'^T ============
            if (lane == 0) {
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t kq = sb + kOffKQ + (gc % 3u) * kKQBytes;
                    const uint32_t tt = sb + kOffT + b * kTBytes;
                    bool ok = mbar_wait(bar(kBKQ + int(gc % 3u)), (gc / 3u) & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBGFree), (gc - 1) & 1u);
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t koff = (s >> 2) * 8192 + (s & 3) * 32;
                        mma_bf16(tmem + kColGram, smem_desc(kq + kKQ_Q, 16, 1024) + uint64_t(koff >> 4),
                                 smem_desc(kq + kKQ_K, 16, 1024) + uint64_t(koff >> 4), id_gram, s > 0);
                    }
                    mma_commit(bar(kBGram));
                    // W^T once T' has landed and the previous W^T has been read (the previous
                    // stage is full)
                    ok = mbar_wait(bar(kBT + int(b)), (gc >> 1) & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBFull + int((gc - 1) & 1u)), ((gc - 1) >> 1) & 1u);
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColW, smem_desc(kq + kKQ_K, 8192, 1024) + uint64_t((s * 2048) >> 4),
                                 smem_desc(tt + kT_P, 16, 1024) + uint64_t((s * 32) >> 4), id_w, s > 0);
                    mma_commit(bar(kBW));
                }
            }
        } else {
            // ============ warp 15: (X1) X1' = -S Q^T and (X6) X2 = U^T P^T ============
            if (lane == 0) {
                for (int n = 0; n < nchunks; ++n) {
                    const uint32_t gc = gn + uint32_t(n), b = gc & 1u;
                    const uint32_t wp = sb + kOffWP + b * kWPBytes;
                    const uint32_t kq = sb + kOffKQ + (gc % 3u) * kKQBytes;
                    bool ok = mbar_wait(bar(kBFull + int(b)), (gc >> 1) & 1u) && mbar_wait(bar(kBSp), gc & 1u);
                    if (ok && gc >= 1) ok = mbar_wait(bar(kBOut), (gc - 1) & 1u);  // X1', X2 read
                    if (!ok) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t koff = (s >> 2) * 8192 + (s & 3) * 32;
                        mma_bf16_ts(tmem + kColX1, tmem + kColSb + 8 * s,
                                    smem_desc(kq + kKQ_Q, 16, 1024) + uint64_t(koff >> 4), id_x1, s > 0);
                    }
                    mma_commit(bar(kBX1));
                    if (!mbar_wait(bar(kBUe), gc & 1u)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColX2, tmem + kColSb + 8 * s,
                                    smem_desc(wp + kWP_P, 16, 1024) + uint64_t((s * 32) >> 4), id_x6, s > 0);
                    mma_commit(bar(kBX6));
                    mma_commit(bar(kBWPFree + int(b)));
                }
            }
        }
        gn += uint32_t(nchunks);
    }

    if (warp >= kWarpEpi && warp < kWarpPrep && tid == 32 * kWarpEpi) bulk_wait_all();
    if (aborted) {
        // let this thread's own tensor-core work drain (bounded) before the tensor
        // memory is freed
        if (warp >= kWarpA && lane == 0) {
            const int bi = warp == kWarpA ? kBS7 : (warp == kWarpB ? kBU : (warp == kWarpP ? kBW : kBX6));
            mma_commit(bar(bi));
            (void)mbar_wait(bar(bi), 0u);
            (void)mbar_wait(bar(bi), 1u);
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

cudaError_t launch_chunk_chain(const PrefillArgs &a, const __nv_bfloat16 *tinv, const float *gcum,
                               int64_t max_chunks, cudaStream_t stream, int num_sms) {
    CUtensorMap mq, mk, mv, mo, mt;
    if (!make_map(&mq, a.q, a.hk, a.tokens) || !make_map(&mk, a.k, a.hk, a.tokens) ||
        !make_map(&mv, a.v, a.hv, a.tokens) || !make_map(&mo, a.o, a.hv, a.tokens, true) ||
        !make_tile_map(&mt, tinv, max_chunks * a.hv * 128))
        return cudaErrorInvalidValue;
    // (the gate logits were turned into decays by the chunk-factor kernel, which
    // hands over the prefix sums G)
    const bool l2 = a.flags & GDN_FLAG_QK_L2NORM;
    using KernFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, PrefillArgs,
                            const float *);
    const KernFn kern = l2 ? chunk_chain_kernel<true> : chunk_chain_kernel<false>;
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
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, mt, a, gcum);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
