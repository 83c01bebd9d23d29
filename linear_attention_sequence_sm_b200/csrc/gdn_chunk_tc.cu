// gdn_chunk_tc.cu -- chunkwise gated delta rule on the 5th-generation tensor
// cores (tcgen05.mma, fp32 accumulators in tensor memory), bf16 inputs,
// d_k = d_v = 128, chunk C = 64.
//
// Chunk algebra (per chunk of L <= 64 tokens r, j with start state S, as in
// the fp32 kernel): G = prefix sums of g, gamma = e^G,
// Gamma_rj = e^(G_r - G_j); A_rj = beta_r Gamma_rj (k_r.k_j) (j < r);
// T = (I + A)^-1; W = T diag(beta gamma) K; U~ = T diag(beta) V;
// U = U~ - W S^T; O = diag(gamma) Q S^T + (Q K^T (.) Gamma) U;
// S <- gamma_C S + U^T diag(e^(G_C - G)) K.  This is the WY representation of
// the DeltaNet transitions with per-chunk cumulative decay ("Gated Attention
// Architectures", sections 2 and 3) and the decay-masked chunk output of its
// section 1, applied to the corrected values U.
//
// Mapping to the tensor cores.  Every contraction is issued with M = 128 so
// that the accumulator row is the tensor-memory lane:
//   (1) [K;Q] K^T      -> Gram (lanes 0-63: K K^T, 64-127: Q K^T)   128x64x128
//   (2) W^T = K^T T'^T  (T' = T diag(beta gamma))                   128x64x64
//   (3) U~^T = V^T T''^T (T'' = T diag(beta))                       128x64x64
//   (4)+(5) [X1' | U^T] = [0 | U~^T] - S [Q; W]^T                   128x128x128
//       (one product with A negated: X1' = -S Q^T, U^T = U~^T - S W^T)
//   (6) X2 = U^T P^T,  P = Q K^T (.) Gamma                           128x64x64
//   (7) S += (U^T diag(lambda)) K,  lambda_j = e^(G_C - G_j)         128x128x64
// O[r][i] = X2[i][r] - gamma_r X1'[i][r].  A tcgen05.mma of M = 128 costs
// about the same whether N is 64 or 128, so (4) and (5), which share the
// operand S, run as one instruction stream of N = 128.  B operands are bf16 in
// 128-byte-swizzled shared memory (q, k, v tiles by TMA, no multicast; W is
// written token-major next to Q); the A operands S, U^T and U^T diag(lambda)
// are bf16 copies in tensor memory.  The fp32 state S lives in tensor memory
// as the accumulator of (7); once per chunk it is read, copied to bf16 for
// (4)+(5), and rescaled by gamma_C in place.
//
// Warp specialisation.  Only (4), (7) and the state pass depend on the state
// carried from the previous chunk; everything else in a chunk does not.  So a
// CTA runs two warp groups on one (sequence, value head) unit:
//   chain  (warps 0-7):  (2)+(3) under the state pass, W epilogue, (4)+(5),
//                        U epilogue, (6)+(7), output
//   intra  (warps 8-15): gates and their prefix sums, (1), decay masks A and
//                        P, the triangular inverse (fp32 diagonal blocks,
//                        tf32 block products) writing T' and T'' as its
//                        blocks become final -- one chunk ahead.
// They hand chunks over through mbarriers: "full[b]" (intra -> chain: T',
// T'', P and the per-token vectors of buffer b are ready), "empty[b]"
// (chain -> intra: buffer b may be refilled), "t_free" (T' and T'' have been
// consumed by (2) and (3); the intra group waits for it just before its
// inverse).  q/k tiles are double-buffered; the chain refills a buffer two
// chunks ahead as soon as its last reader (7) completes.  Each group
// synchronises internally with its own named barrier, and one warp of each
// group polls the mbarriers.  A full chunk of output leaves through one TMA
// store of the staged tile.
//
// With the output side (a template instance of its own), each output row is
// RMS-normalised, scaled and gated before it is stored: after (6)+(7) the
// chain leaves O in fp32 in X2's columns, and the row reductions, scale, gate
// and store of that chunk run under the next chunk's merged product (4)+(5).
// The gate tile arrives by TMA one chunk ahead.
//
// One CTA per SM (shared memory and the 512 tensor-memory columns force it)
// takes units longest sequence first from an atomic counter.  Every wait is
// bounded; a timeout records GDN_ERR_DEVICE_CHECK (bad_index -2) in the
// workspace status word, and the CTA frees its tensor memory and exits.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThreads = 512;      // warps 0-7: chain group; warps 8-15: intra group
constexpr int kChain = 256, kIntra = 256;
constexpr int kBarChain = 1, kBarIntra = 2;  // named barrier ids (0 is __syncthreads)
// The intra group's Gram MMAs are issued from its last warp, which does none of
// the gate scan or the first inverse phase: an issue that stalls behind the
// chain's tensor-core work then delays no other intra work.
constexpr int kIntraIssuer = 224;
constexpr int kLdA = 68;  // fp32 row stride of the A and T scratch matrices (16-byte aligned rows)
constexpr int kLdY = 36;  // fp32 row stride of the inverse's 32 x 32 scratch

// Shared-memory map (bytes from a 1024-byte-aligned base).  Tiles are
// 128-byte-swizzled: "atom columns" of 64 bf16 (128 bytes) per row.
// A chunk buffer holds, per atom column, 64 rows each of K, Q and W (token-major):
// [K;Q] is the Gram's A operand and [Q;W] the B operand of the merged (4)+(5).
constexpr uint32_t kAtomKQ = 24576;   // one atom column of a chunk buffer: K, Q, W rows
constexpr uint32_t kOffKQ0 = 0;       // chunk buffer 0: 2 atom columns
constexpr uint32_t kOffKQ1 = 49152;   // chunk buffer 1
constexpr uint32_t kOffV = 98304;     // V: 2 atom columns x 64 rows
constexpr uint32_t kOffP0 = 114688;   // P = Q K^T (.) Gamma, buffer 0: 64 x 64
constexpr uint32_t kOffP1 = 122880;   // P, buffer 1
constexpr uint32_t kOffOst = 131072;  // output staging: 64 tokens x 128 bf16, token-major (one TMA store)
constexpr uint32_t kOffAf = 147456;   // A, fp32 64 x kLdA (intra group)
constexpr uint32_t kOffTf = kOffAf + 64 * kLdA * 4;  // T, fp32 64 x kLdA
constexpr uint32_t kOffY = kOffTf + 64 * kLdA * 4;   // inverse scratch, 32 x kLdY fp32
constexpr uint32_t kOffVec0 = kOffY + 32 * kLdY * 4;  // per-token vectors of buffer 0 (10 x 64 fp32)
constexpr uint32_t kOffVec1 = kOffVec0 + 10 * 64 * 4; // buffer 1
constexpr uint32_t kOffNrm = kOffVec1 + 10 * 64 * 4;  // 1/||k_r|| (0-63), 1/||q_r|| (64-127) of the next chunk
constexpr uint32_t kOffGst = kOffNrm + 128 * 4;       // gates by TMA, per [K;Q] buffer: g, beta as 64 tokens x 4 heads
constexpr uint32_t kOffTp = (kOffGst + 2 * 2048 + 1023) / 1024 * 1024;  // T' = T diag(beta gamma), bf16 64 x 64
constexpr uint32_t kOffTpp = kOffTp + 8192;                               // T'' = T diag(beta)
constexpr uint32_t kOffBar = kOffTpp + 8192;          // mbarriers, tensor-memory slot, unit slot
constexpr uint32_t kSmemBytes = kOffBar + 128 + 1024; // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");
// With the output side: the chunk's gate tile z (64 tokens x 128 bf16,
// token-major, by TMA one chunk ahead) and the per-token partial sums of
// squares after the barriers.
constexpr uint32_t kOffZ = (kOffBar + 128 + 1023) / 1024 * 1024;
constexpr uint32_t kBytesZ = 64 * 128 * 2;
constexpr uint32_t kOffRed = kOffZ + kBytesZ;  // per token, 4 partial sums of squares (fp32 64 x 4)
constexpr uint32_t kSmemBytesOut = kOffRed + 64 * 4 * 4 + 1024;
static_assert(kSmemBytesOut <= 232448, "shared memory over the sm_100 per-block limit");
// per-token vectors inside a buffer (floats)
constexpr int kVecG = 0, kVecB = 64, kVecGam = 128, kVecBG = 192, kVecLam = 256, kVecIGam = 320;
// per-token scales through which GDN_FLAG_QK_L2NORM normalises the raw q and k
// (the plain instantiation reads beta and gamma instead): A rows beta / ||k||^2,
// P rows 1 / ||q||, T'' columns beta / ||k||, output gamma / ||q||; the T'
// columns (kVecBG) then carry beta gamma / ||k||^2.  With N_k = diag(||k||):
// T = N_k (I + diag(beta / ||k||^2) M)^-1 N_k^-1 for M = strict(K K^T (.) Gamma)
// of the raw K, so W = N_k W' and U~ = N_k U~' with the scaled T', T''; U =
// N_k U', the state update U'^T diag(lambda) K needs no scale, and the output
// is diag(gamma / ||q||) Q S^T + diag(1 / ||q||) (Q K^T (.) Gamma) U'.
constexpr int kVecSa = 384, kVecSp = 448, kVecTpp = 512, kVecGo = 576;
// mbarrier slots
constexpr int kBarTKQ = 0, kBarTV = 2, kBarI = 3, kBarC = 4, kBarFull = 5, kBarEmpty = 7, kBarWT = 9, kBarZ = 10,
              kNumBars = 11;
// (kBarWT: "T' and T'' consumed", chain -> intra; kBarZ: gate tile landed)
static_assert(8 * kNumBars + 8 <= 128, "barrier slots overflow their region");

// Tensor-memory columns (128 lanes each): fp32 accumulators, and bf16 A
// operands packed two elements per column: the copy of S for (4) and (5), and
// U^T and U^T diag(lambda) for (6) and (7), which reuse the W^T accumulator's
// columns once its epilogue has read them.
constexpr uint32_t kColGram = 0, kColW = 64, kColX1 = 128, kColU = 192, kColSb = 256, kColX2 = 320, kColS = 384;
constexpr uint32_t kColUb = kColW, kColUlb = kColW + 32;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesKQ = 4 * 8192 + 2 * 1024;  // four 64 x 64 bf16 boxes and two 64 x 4 fp32 gate boxes
constexpr uint32_t kBytesV = 2 * 8192;

// T' = T diag(beta gamma) and T'' = T diag(beta) entries (R, C), (R, C + 1) as
// bf16 pairs in the 128-byte-swizzled 64 x 64 operand tiles at tp and tpp.
__device__ __forceinline__ void st_tt_pair(uint32_t tp, uint32_t tpp, int R, int C, float v0, float v1,
                                           const float *bg, const float *bb) {
    const uint32_t off = uint32_t(R) * 128 + ((uint32_t((C >> 3) ^ (R & 7))) << 4) + uint32_t(C & 7) * 2;
    st_shared_u32(tp + off, pack_bf16x2(v0 * bg[C], v1 * bg[C + 1]));
    st_shared_u32(tpp + off, pack_bf16x2(v0 * bb[C], v1 * bb[C + 1]));
}

// T = (I + A)^-1 for the 64 x 64 unit-lower-triangular system, fp32, in
// shared memory, by divide and conquer on the block structure
//   [[X, 0], [C, Z]]^-1 = [[X^-1, 0], [-Z^-1 C X^-1, Z^-1]]:
// the four 16 x 16 diagonal blocks by row-wise forward substitution (one
// thread per column, fp32), then the two 32 x 32 halves (two 16 x 16
// products each) and the 64 x 64 matrix (two 32 x 32 products) as warp-level
// tf32 products with fp32 accumulation (T is rounded to bf16 afterwards, so
// the 10-bit tf32 mantissa is ample).
// Everything of Tf above the diagonal must be zero on entry (it is zeroed once
// and never written).  Called by the 256 threads of the intra group (t = 0..255).
//
// The bf16 operands T' and T'' (column scales bg = beta gamma, bb = beta) are
// written as each block of T becomes final:
// the diagonal 16 x 16 blocks from the forward substitution, the 16 x 16 and
// 32 x 32 lower blocks from the tf32 products; the idle threads of the first
// phase zero the blocks above the diagonal.  The fp32 copy of the last block
// is not needed and not written.  Ends with every thread's operand writes
// fenced for the tensor cores and a group barrier.
__device__ void invert_to_operands(const float *Af, float *Tf, float *Y, int t, uint32_t tp, uint32_t tpp,
                                   const float *bg, const float *bb) {
    if (t < 64) {
        const int b = t >> 4, c = t & 15;
        const float *Ab = Af + (16 * b) * kLdA + 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float a[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) load4(Ab + r * kLdA + 4 * q, a + 4 * q);
            float acc0 = (r == c) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < r; ++jj) {
                if (jj & 1) acc1 = fmaf(-a[jj], x[jj], acc1);
                else acc0 = fmaf(-a[jj], x[jj], acc0);
            }
            x[r] = acc0 + acc1;
        }
        float *Tb = Tf + (16 * b) * kLdA + 16 * b;
        const int C = 16 * b + c;
        const float sg = bg[C], sb = bb[C];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            Tb[r * kLdA + c] = x[r];
            const int R = 16 * b + r;
            const uint32_t off = uint32_t(R) * 128 + ((uint32_t((C >> 3) ^ (R & 7))) << 4) + uint32_t(C & 7) * 2;
            st_shared_b16(tp + off, x[r] * sg);
            st_shared_b16(tpp + off, x[r] * sb);
        }
    } else {
        // zero the six 16 x 16 blocks above the diagonal of both tiles:
        // 2 tiles x 6 blocks x 16 rows x 2 sixteen-byte chunks = 384 stores
        for (int e = t - 64; e < 384; e += 192) {
            const int tile = e / 192, w = e % 192, blk = w >> 5, rr = (w >> 1) & 15, half = w & 1;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            const int R = 16 * bi + rr, ck = 2 * bj + half;
            st_shared_v4((tile ? tpp : tp) + uint32_t(R) * 128 + (uint32_t(ck ^ (R & 7)) << 4), make_uint4(0, 0, 0, 0));
        }
    }
    named_sync(kBarIntra, kIntra);
    const int w = t >> 5, lane = t & 31;
    const int g = lane >> 2, tq = lane & 3;
    if (w < 4) {
        const int p = w >> 1, n0 = 8 * (w & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma(c, Af + (32 * p + 16) * kLdA + 32 * p, kLdA, Tf + (32 * p) * kLdA + 32 * p, kLdA, n0, 2, lane);
        tile_store(Y + (16 * p) * kLdY, kLdY, 0, n0, c, 1.f, lane);
    }
    named_sync(kBarIntra, kIntra);
    if (w < 4) {
        const int p = w >> 1, n0 = 8 * (w & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma(c, Tf + (32 * p + 16) * kLdA + 32 * p + 16, kLdA, Y + (16 * p) * kLdY, kLdY, n0, 2, lane);
        tile_store(Tf + (32 * p + 16) * kLdA + 32 * p, kLdA, 0, n0, c, -1.f, lane);
        const int R = 32 * p + 16 + g, C = 32 * p + n0 + 2 * tq;
        st_tt_pair(tp, tpp, R, C, -c[0], -c[1], bg, bb);
        st_tt_pair(tp, tpp, R + 8, C, -c[2], -c[3], bg, bb);
    }
    named_sync(kBarIntra, kIntra);
    {
        const int m0 = 16 * (w >> 2), n0 = 8 * (w & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma(c, Af + (32 + m0) * kLdA, kLdA, Tf, kLdA, n0, 4, lane);
        tile_store(Y, kLdY, m0, n0, c, 1.f, lane);
    }
    named_sync(kBarIntra, kIntra);
    {
        const int m0 = 16 * (w >> 2), n0 = 8 * (w & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_mma(c, Tf + (32 + m0) * kLdA + 32, kLdA, Y, kLdY, n0, 4, lane);
        const int R = 32 + m0 + g, C = n0 + 2 * tq;
        st_tt_pair(tp, tpp, R, C, -c[0], -c[1], bg, bb);
        st_tt_pair(tp, tpp, R + 8, C, -c[2], -c[3], bg, bb);
    }
    fence_proxy_async_shared();
    named_sync(kBarIntra, kIntra);
}

// Loads chunk `c0` of q and k for q/k head `hq` into a [K;Q] buffer, and the
// chunk's g and beta for the four value heads around `h` into `gst`.
__device__ __forceinline__ void load_kq(uint32_t dst, uint32_t bar, const CUtensorMap *tk, const CUtensorMap *tq,
                                        int hq, int c0, uint32_t gst, const CUtensorMap *tg, const CUtensorMap *tb,
                                        int h) {
    mbar_arrive_expect_tx(bar, kBytesKQ);
    tma_load_2d(gst, tg, h & ~3, c0, bar);
    tma_load_2d(gst + 1024, tb, h & ~3, c0, bar);
    tma_load_3d(dst, tk, 0, hq, c0, bar);
    tma_load_3d(dst + 8192, tq, 0, hq, c0, bar);
    tma_load_3d(dst + kAtomKQ, tk, 64, hq, c0, bar);
    tma_load_3d(dst + kAtomKQ + 8192, tq, 64, hq, c0, bar);
}

__device__ __forceinline__ void load_v(uint32_t dst, uint32_t bar, const CUtensorMap *tv, int h, int c0) {
    mbar_arrive_expect_tx(bar, kBytesV);
    tma_load_3d(dst, tv, 0, h, c0, bar);
    tma_load_3d(dst + 8192, tv, 64, h, c0, bar);
}

// The output side's gate tile of chunk c0, value head h (rows past the last
// token read as zeros).
__device__ __forceinline__ void load_z(uint32_t dst, uint32_t bar, const CUtensorMap *tz, int h, int c0) {
    mbar_arrive_expect_tx(bar, kBytesZ);
    tma_load_3d(dst, tz, 0, h, c0, bar);
}

// kL2: GDN_FLAG_QK_L2NORM; kLogits: GDN_FLAG_GATE_LOGITS; kOut: the output
// side in the output epilogue (compile-time, so the plain path carries none
// of the input- or output-side work)
template <bool kL2, bool kLogits, bool kOut>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_z, const PrefillArgs a) {
    extern __shared__ unsigned char smem_raw[];
    // Align to 1024 bytes with a byte offset on the shared array itself (not
    // through an integer cast), so that the compiler keeps every access below in
    // the shared address space (ld.shared / st.shared, not generic loads).
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *Af = reinterpret_cast<float *>(smem + kOffAf);
    float *Tf = reinterpret_cast<float *>(smem + kOffTf);
    float *Yb = reinterpret_cast<float *>(smem + kOffY);
    float *nrm = reinterpret_cast<float *>(smem + kOffNrm);
    const uint32_t bars = sb + kOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * kNumBars);
    int *s_unit = reinterpret_cast<int *>(smem + kOffBar + 8 * kNumBars + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool is_chain = warp < 8;
    // One warp per group polls each mbarrier; the rest of the group blocks in the
    // named barrier that follows every wait, so the spinning costs the shared-
    // memory pipe one warp's requests instead of eight.
    const bool chain_poll = warp == 0, intra_poll = warp == 8;
    const uint32_t lane_bits = uint32_t((warp & 3) * 32) << 16;  // this warp's tensor-memory lane quarter
    WsHeader *hdr = a.sched.hdr;

    // Set-up that needs nothing from the schedule kernel runs while it finishes
    // (this kernel is launched as its programmatic dependent).
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bars + 8 * i, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), kTmemCols);
        tmem_relinquish();
    }
    // T starts all zero: the inverse writes only the lower-triangular blocks
    // (and zeros above the diagonal inside the diagonal blocks), so everything
    // above the diagonal reads as zero for the rest of the kernel.
    if (!is_chain)
        for (int e = tid - kChain; e < 64 * kLdA; e += kIntra) Tf[e] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();  // the schedule and the workspace status word are written
    if (hdr->status != GDN_OK) {
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, kTmemCols);
        return;
    }

    const int hv = a.hv, hk = a.hk, group = hv / hk;
    const int total_units = a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
    uint32_t gn = 0;  // chunks this CTA has processed so far (selects buffers and barrier phases)
    uint32_t ph_full = 0, ph_empty = 0, ph_tkq = 0, ph_v = 0, ph_i = 0, ph_c = 0, ph_wt = 0, ph_z = 0;
    bool aborted = false;

    const uint32_t id_gram = idesc_bf16(128, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 64, true, false);
    const uint32_t id_qw = idesc_bf16(128, 128, false, false, true);  // [X1' | U^T] -= S [Q; W]^T
    const uint32_t id_x = idesc_bf16(128, 64, false, false);
    const uint32_t id_ds = idesc_bf16(128, 128, false, true);  // state update, accumulates into S

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
        const size_t sbase = (size_t(seq) * hv + h) * 128 * 128;
        if (tid == 0 && nchunks > 0) {
            load_kq(sb + ((gn & 1) ? kOffKQ1 : kOffKQ0), bars + 8 * (kBarTKQ + (gn & 1)), &tm_k, &tm_q, hq, t0,
                    sb + kOffGst + (gn & 1) * 2048, &tm_g, &tm_b, h);
            if (nchunks > 1)
                load_kq(sb + (((gn + 1) & 1) ? kOffKQ1 : kOffKQ0), bars + 8 * (kBarTKQ + ((gn + 1) & 1)), &tm_k,
                        &tm_q, hq, t0 + 64, sb + kOffGst + ((gn + 1) & 1) * 2048, &tm_g, &tm_b, h);
            load_v(sb + kOffV, bars + 8 * kBarTV, &tm_v, h, t0);
            if (kOut && a.out.z) load_z(sb + kOffZ, bars + 8 * kBarZ, &tm_z, h, t0);
        }

        if (is_chain) {
            // ============ chain group: thread = (state row, half of the columns) ============
            const int row = (warp & 3) * 32 + lane;
            const int ch = warp >> 2;
            // output side: this thread's channel scale, and whether a gate tile comes
            const float out_s = kOut ? out_scale(a.out, h, row, 128) : 0.f;
            const bool zgate = kOut && a.out.z != nullptr;
            // initial state into tensor memory
#pragma unroll
            for (int c4 = 2 * ch; c4 < 2 * ch + 2; ++c4) {
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
            {  // X1' accumulates onto zero
                uint32_t z[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) z[j] = 0u;
                tmem_st16u(tmem + lane_bits + kColX1 + 32 * ch, z);
                tmem_st16u(tmem + lane_bits + kColX1 + 32 * ch + 16, z);
            }
            tmem_wait_st();
            // Output side, second half, for the chunk whose O (fp32) waits in X2's
            // columns (tokens cp .. cp + Lp - 1): per token the root mean square
            // over the 128 value rows (column sums of O^2 per warp, then 4 partial
            // sums per token), scale, gate, stage and store; then the gate tile of
            // the chunk at cz may come in.  It runs while the tensor cores work on
            // the next chunk's merged product (4)+(5), which leaves X2 alone.
            auto out_deferred = [&](int cp, int Lp, bool load_next, int cz) -> bool {
                __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffOst);
                float *red = reinterpret_cast<float *>(smem + kOffRed);
                const __nv_bfloat16 *Zt = reinterpret_cast<const __nv_bfloat16 *>(smem + kOffZ);
                float ov[2][16];
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) tmem_ld16(tmem + lane_bits + kColX2 + 32 * ch + 16 * sl, ov[sl]);
                tmem_wait_ld();
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    float sq[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) sq[j] = ov[sl][j] * ov[sl][j];
                    const float part = warp_colsum16(sq, lane);
                    if ((lane & 1) == 0) red[(32 * ch + 16 * sl + (lane >> 1)) * 4 + (warp & 3)] = part;
                }
                bool ok = true;
                if (zgate) {
                    ok = mbar_wait(bars + 8 * kBarZ, ph_z);
                    ph_z ^= 1u;
                }
                // (also orders the staging writes after tid 0's wait for the last store)
                if (named_sync_or(kBarChain, kChain, !ok)) return false;
                float inv_rms;  // of token 32 ch + lane
                {
                    const float4 pr = *reinterpret_cast<const float4 *>(red + 4 * (32 * ch + lane));
                    inv_rms = rsqrtf(((pr.x + pr.y) + (pr.z + pr.w)) * (1.f / 128.f) + a.out.eps);
                }
                const uint32_t oflags = a.out.flags;
#pragma unroll
                for (int sl = 0; sl < 2; ++sl)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int r = 32 * ch + 16 * sl + j;
                        float y = ov[sl][j] * out_s * __shfl_sync(0xffffffffu, inv_rms, 16 * sl + j);
                        if (zgate) y *= out_gate_fast(oflags, __bfloat162float(Zt[r * 128 + row]));
                        Ot[r * 128 + row] = __float2bfloat16_rn(y);
                    }
                fence_proxy_async_shared();
                named_sync(kBarChain, kChain);
                if (Lp == 64) {
                    if (tid == 0) {
                        tma_store_3d(&tm_o, sb + kOffOst, 0, h, cp);
                        bulk_commit();
                    }
                } else {
                    for (int e = tid; e < 64 * 16; e += kChain) {
                        const int r = e >> 4, c = e & 15;
                        if (r < Lp) {
                            const uint4 val = *reinterpret_cast<const uint4 *>(smem + kOffOst + r * 256 + c * 16);
                            *reinterpret_cast<uint4 *>(o + (size_t(cp + r) * hv + h) * 128 + c * 8) = val;
                        }
                    }
                    named_sync(kBarChain, kChain);
                }
                // the gate tile has been read by every thread (barriers above)
                if (load_next && zgate && tid == 0) load_z(sb + kOffZ, bars + 8 * kBarZ, &tm_z, h, cz);
                return true;
            };
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gcn = gn + n, b = gcn & 1;
                const int c0 = t0 + n * 64, L = min(64, len - n * 64);
                const float *vec = reinterpret_cast<const float *>(smem + (b ? kOffVec1 : kOffVec0));
                const uint32_t kq = sb + (b ? kOffKQ1 : kOffKQ0);
                const uint32_t pt = sb + (b ? kOffP1 : kOffP0);
                const uint32_t colU = kColU;
                {
                    const bool ok = !chain_poll || (mbar_wait(bars + 8 * (kBarFull + b), (ph_full >> b) & 1u) &&
                                    mbar_wait(bars + 8 * kBarTV, ph_v));
                    ph_full ^= 1u << b;
                    ph_v ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // (2) W^T = K^T T'^T and (3) U~^T = V^T T''^T, running under the state pass
                if (tid == 0) {
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColW, (smem_desc(kq, kAtomKQ, 1024) + uint64_t((s * 2048) >> 4)),
                                 (smem_desc(sb, 16, 1024) + uint64_t((kOffTp + s * 32) >> 4)), id_w, s > 0);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + colU, (smem_desc(sb, 8192, 1024) + uint64_t((kOffV + s * 2048) >> 4)),
                                 (smem_desc(sb, 16, 1024) + uint64_t((kOffTpp + s * 32) >> 4)), id_w, s > 0);
                    mma_commit(bars + 8 * kBarC);
                }
                // state pass: S_n -> bf16 operand, S <- gamma_C S_n in place
                {
                    const float gC = vec[kVecGam + 63];  // padded rows carry g = 0, so G_63 = G_{L-1}
#pragma unroll
                    for (int p2 = 0; p2 < 2; ++p2) {
                        float v0[32];
                        tmem_ld32(tmem + lane_bits + kColS + 64 * ch + 32 * p2, v0);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(v0[2 * j], v0[2 * j + 1]);
                        tmem_st16u(tmem + lane_bits + kColSb + 32 * ch + 16 * p2, pk);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v0[j] *= gC;
                        tmem_st32(tmem + lane_bits + kColS + 64 * ch + 32 * p2, v0);
                    }
                    tmem_wait_st();
                }
                {
                    const bool ok = !chain_poll || mbar_wait(bars + 8 * kBarC, ph_c);
                    ph_c ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                if (tid == 0) {
                    mbar_arrive(bars + 8 * kBarWT);  // T' and T'' consumed: the intra group may overwrite them
                    if (n + 1 < nchunks) load_v(sb + kOffV, bars + 8 * kBarTV, &tm_v, h, c0 + 64);
                }
                {
                    float v[32];
                    tmem_ld32(tmem + lane_bits + kColW + 32 * ch, v);
                    tmem_wait_ld();
                    // W[r][i] (token-major, d_k contiguous) for this thread's d_k index
                    // i = row and tokens r = 32 ch + j, in the W rows of atom column i / 64
                    const uint32_t wb = kq + (row >> 6) * kAtomKQ + 16384 + (row & 7) * 2;
                    const uint32_t c8 = (row & 63) >> 3;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int r = 32 * ch + j;
                        st_shared_b16(wb + r * 128 + ((c8 ^ uint32_t(r & 7)) << 4), v[j]);
                    }
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarChain, kChain);
                // (4) and (5) as one product of N = 128 with A negated:
                // [X1' | U^T] = [0 | U~^T] - S [Q; W]^T, so X1' = -S Q^T (its columns
                // were zeroed after the previous output) and U^T = U~^T - S W^T
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t off = (s >> 2) * kAtomKQ + (s & 3) * 32;
                        mma_bf16_ts(tmem + kColX1, tmem + kColSb + 8 * s,
                                    (smem_desc(kq + 8192, 16, 1024) + uint64_t(off >> 4)), id_qw, 1);
                    }
                    mma_commit(bars + 8 * kBarC);
                    bulk_wait_read();  // the previous chunk's output store has read the staging tile
                }
                // output side: the previous chunk (a full one: only a sequence's last
                // chunk is ragged) finishes under this product; its gate tile then
                // makes room for this chunk's
                if constexpr (kOut)
                    if (n > 0 && !out_deferred(c0 - 64, 64, true, c0)) { aborted = true; break; }
                {
                    const bool ok = !chain_poll || mbar_wait(bars + 8 * kBarC, ph_c);
                    ph_c ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // U epilogue: U^T rows to bf16 A operands of (6) and (7), plain and
                // lambda-scaled, in the W accumulator's columns (consumed above)
                {
                    float v[32], l[32];
                    tmem_ld32(tmem + lane_bits + colU + 32 * ch, v);
#pragma unroll
                    for (int q = 0; q < 8; ++q) load4(vec + kVecLam + 32 * ch + 4 * q, l + 4 * q);
                    tmem_wait_ld();
                    uint32_t pu[16], pl[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        pu[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                        pl[j] = pack_bf16x2(l[2 * j] * v[2 * j], l[2 * j + 1] * v[2 * j + 1]);
                    }
                    tmem_st16u(tmem + lane_bits + kColUb + 16 * ch, pu);
                    tmem_st16u(tmem + lane_bits + kColUlb + 16 * ch, pl);
                    tmem_wait_st();
                }
                tc_fence_before();
                named_sync(kBarChain, kChain);
                // (6) X2 = U^T P^T and (7) S += U^T diag(lambda) K
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColX2, tmem + kColUb + 8 * s,
                                    (smem_desc(pt, 16, 1024) + uint64_t((s * 32) >> 4)), id_x, s > 0);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_ts(tmem + kColS, tmem + kColUlb + 8 * s,
                                    (smem_desc(kq, kAtomKQ, 1024) + uint64_t((s * 2048) >> 4)), id_ds, 1);
                    mma_commit(bars + 8 * kBarC);
                }
                {
                    const bool ok = !chain_poll || mbar_wait(bars + 8 * kBarC, ph_c);
                    ph_c ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // the [K;Q] buffer is free: refill it two chunks ahead
                if (tid == 0 && n + 2 < nchunks)
                    load_kq(kq, bars + 8 * (kBarTKQ + b), &tm_k, &tm_q, hq, c0 + 128, sb + kOffGst + b * 2048, &tm_g,
                            &tm_b, h);
                // output O[r][i] = gamma_r X1[i][r] + X2[i][r] = X2[i][r] - gamma_r X1'[i][r],
                // staged token-major (rows of 256 bytes); a full chunk leaves in one
                // TMA store, a ragged last chunk row by row.  X1' is zeroed for the
                // next chunk's merged product.
                if constexpr (!kOut) {
                    __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffOst);
                    uint32_t z[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll
                    for (int sl = 0; sl < 2; ++sl) {
                        const int r0 = 32 * ch + 16 * sl;
                        float x1[16], x2[16], gm[16];
                        tmem_ld16(tmem + lane_bits + kColX1 + r0, x1);
                        tmem_ld16(tmem + lane_bits + kColX2 + r0, x2);
#pragma unroll
                        for (int q = 0; q < 4; ++q) load4(vec + (kL2 ? kVecGo : kVecGam) + r0 + 4 * q, gm + 4 * q);
                        tmem_wait_ld();
                        tmem_st16u(tmem + lane_bits + kColX1 + r0, z);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            Ot[(r0 + j) * 128 + row] = __float2bfloat16_rn(fmaf(-gm[j], x1[j], x2[j]));
                    }
                    tmem_wait_st();
                }
                else {
                    // output side, first half: O = X2 - gamma X1' (fp32) into X2's columns and
                    // X1' zeroed; the rest runs under the next chunk's merged product
#pragma unroll
                    for (int sl = 0; sl < 2; ++sl) {
                        const int r0 = 32 * ch + 16 * sl;
                        float x1[16], x2[16], gm[16];
                        tmem_ld16(tmem + lane_bits + kColX1 + r0, x1);
                        tmem_ld16(tmem + lane_bits + kColX2 + r0, x2);
#pragma unroll
                        for (int q = 0; q < 4; ++q) load4(vec + (kL2 ? kVecGo : kVecGam) + r0 + 4 * q, gm + 4 * q);
                        tmem_wait_ld();
                        uint32_t ob[16], zr[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            ob[j] = __float_as_uint(fmaf(-gm[j], x1[j], x2[j]));
                            zr[j] = 0u;
                        }
                        tmem_st16u(tmem + lane_bits + kColX1 + r0, zr);
                        tmem_st16u(tmem + lane_bits + kColX2 + r0, ob);
                    }
                    tmem_wait_st();
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarChain, kChain);
                if constexpr (!kOut) {
                    if (L == 64) {
                        if (tid == 0) {
                            tma_store_3d(&tm_o, sb + kOffOst, 0, h, c0);
                            bulk_commit();
                        }
                    } else {
                        for (int e = tid; e < 64 * 16; e += kChain) {
                            const int r = e >> 4, c = e & 15;
                            if (r < L) {
                                const uint4 val =
                                    *reinterpret_cast<const uint4 *>(smem + kOffOst + r * 256 + c * 16);
                                *reinterpret_cast<uint4 *>(o + (size_t(c0 + r) * hv + h) * 128 + c * 8) = val;
                            }
                        }
                        named_sync(kBarChain, kChain);
                    }
                }
                if (tid == 0) mbar_arrive(bars + 8 * (kBarEmpty + b));  // buffers b may be refilled
            }
            if constexpr (kOut) {
                if (!aborted && nchunks > 0) {
                    const int cl = t0 + (nchunks - 1) * 64;
                    if (tid == 0) bulk_wait_read();  // the previous store has read the staging tile
                    if (!out_deferred(cl, len - (nchunks - 1) * 64, false, 0)) aborted = true;
                    tc_fence_before();
                }
            }
            if (!aborted) {
                // final state out of tensor memory
#pragma unroll
                for (int c4 = 2 * ch; c4 < 2 * ch + 2; ++c4) {
                    float v[32];
                    tmem_ld32(tmem + lane_bits + kColS + 32 * c4, v);
                    tmem_wait_ld();
                    if (a.s_final) {
                        float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128 + 32 * c4);
#pragma unroll
                        for (int c = 0; c < 8; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    }
                }
                tc_fence_before();
            }
        } else {
            // ================= intra group: next chunk's state-independent work =================
            const int it = tid - kChain;                 // 0..255
            const int irow = (warp & 3) * 32 + lane;     // tensor-memory lane of this thread
            const int ih = (warp - 8) >> 2;              // which 32-column half of a 64-column tile
            // (1) for the chunk whose [K;Q] tile is at kqb, by one thread
            auto issue_gram = [&](uint32_t kqb) {
                tc_fence_after();
                const uint64_t dk = smem_desc(kqb, 16, 1024);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t d = dk + uint64_t(((s >> 2) * kAtomKQ + (s & 3) * 32) >> 4);
                    mma_bf16(tmem + kColGram, d, d, id_gram, s > 0);
                }
                mma_commit(bars + 8 * kBarI);
            };
            // gates of the chunk in buffer bb (arrived with its q and k) and their
            // chunk-local prefix sums, by one warp; tokens past the sequence end get
            // g = beta = 0 (the identity on S)
            auto chunk_gates = [&](uint32_t bb, int Lc) {
                float *vv = reinterpret_cast<float *>(smem + (bb ? kOffVec1 : kOffVec0));
                const float *stg = reinterpret_cast<const float *>(smem + kOffGst + bb * 2048);
                const int hc = h & 3;
                const bool ok0 = 2 * lane < Lc, ok1 = 2 * lane + 1 < Lc;
                constexpr bool logits = kLogits;
                const float ga = stg[(2 * lane) * 4 + hc], gb = stg[(2 * lane + 1) * 4 + hc];
                const float ba = stg[256 + (2 * lane) * 4 + hc], bb2 = stg[256 + (2 * lane + 1) * 4 + hc];
                const float g0 = ok0 ? fmaxf(logits ? log_sigmoid_fast(ga) : ga, kGFloor) : 0.f;
                const float g1 = ok1 ? fmaxf(logits ? log_sigmoid_fast(gb) : gb, kGFloor) : 0.f;
                vv[kVecB + 2 * lane] = ok0 ? (logits ? sigmoid_fast(ba) : ba) : 0.f;
                vv[kVecB + 2 * lane + 1] = ok1 ? (logits ? sigmoid_fast(bb2) : bb2) : 0.f;
                float incl = g0 + g1;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float tt = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += tt;
                }
                const float excl = incl - (g0 + g1);
                vv[kVecG + 2 * lane] = excl + g0;
                vv[kVecG + 2 * lane + 1] = excl + g0 + g1;
            };
            // 1 / max(||row||, 1e-12) of the 64 k rows and 64 q rows of the [K;Q]
            // tile at kqb (GDN_FLAG_QK_L2NORM), one row per thread of warps 9-12
            constexpr bool l2 = kL2;
            auto chunk_norms = [&](uint32_t kqb) {
                const int R = it - 32;  // tile row: k rows 0-63, q rows 64-127
                float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        // piece p of the row in swizzled order: the 8 lanes that share a
                        // shared-memory phase hit 8 different 16-byte bank groups
                        const uint4 w = ld_shared_v4(kqb + c * kAtomKQ + R * 128 + (uint32_t(p ^ (R & 7)) << 4));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                            ss[u] = fmaf(lo, lo, fmaf(hi, hi, ss[u]));
                        }
                    }
                nrm[R] = inv_l2((ss[0] + ss[1]) + (ss[2] + ss[3]));
            };
            // per-token vectors gamma, beta gamma, lambda and 1/gamma, and the operand scales (threads 0-63)
            auto chunk_vectors = [&](uint32_t bb, int Lc) {
                float *vv = reinterpret_cast<float *>(smem + (bb ? kOffVec1 : kOffVec0));
                const float G = vv[kVecG + it], bt = vv[kVecB + it], gam = __expf(G);
                vv[kVecGam + it] = gam;
                vv[kVecLam + it] = it < Lc ? __expf(vv[kVecG + Lc - 1] - G) : 0.f;
                vv[kVecIGam + it] = __expf(-G);
                if constexpr (kL2) {
                    const float ik = nrm[it], iq = nrm[64 + it];  // 1/||k_it||, 1/||q_it||
                    vv[kVecBG + it] = bt * gam * ik * ik;
                    vv[kVecSa + it] = bt * ik * ik;
                    vv[kVecSp + it] = iq;
                    vv[kVecTpp + it] = bt * ik;
                    vv[kVecGo + it] = gam * iq;
                } else {
                    vv[kVecBG + it] = bt * gam;
                }
            };
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gcn = gn + n, b = gcn & 1;
                const int L = min(64, len - n * 64);
                float *vec = reinterpret_cast<float *>(smem + (b ? kOffVec1 : kOffVec0));
                float *gs = vec + kVecG, *bs = vec + kVecB;
                const uint32_t kq = sb + (b ? kOffKQ1 : kOffKQ0);
                const uint32_t pt = sb + (b ? kOffP1 : kOffP0);
                if (n == 0) {  // later chunks are prepared at the end of the previous one
                    bool ok = true;
                    if (intra_poll) {
                        if (gcn >= 2) ok = mbar_wait(bars + 8 * (kBarEmpty + b), (ph_empty >> b) & 1u);
                        ok = ok && mbar_wait(bars + 8 * (kBarTKQ + b), (ph_tkq >> b) & 1u);
                    }
                    if (gcn >= 2) ph_empty ^= 1u << b;
                    ph_tkq ^= 1u << b;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                    if (it == kIntraIssuer) issue_gram(kq);
                    if (warp == 8) chunk_gates(b, L);
                    if (l2 && it >= 32 && it < 160) chunk_norms(kq);
                    named_sync(kBarIntra, kIntra);
                    if (it < 64) chunk_vectors(b, L);
                }
                {
                    const bool ok = !intra_poll || mbar_wait(bars + 8 * kBarI, ph_i);
                    ph_i ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // A (fp32, for the inverse) and P (bf16 operand) from the Gram, in
                // slices of 16 columns
                {
                    const int r = irow & 63;
                    const bool is_a = irow < 64;
                    float scale;
                    if constexpr (kL2) scale = vec[(is_a ? kVecSa : kVecSp) + r];
                    else scale = is_a ? bs[r] : 1.f;
                    const int lim = is_a ? r : r + 1;  // A: j < r;  P: j <= r
                    // Gamma_rj = e^(G_r - G_j).  While the chunk's total log-decay is
                    // at least -80, e^(-G_j) stays finite in fp32 and Gamma is the
                    // rank-1 product e^(G_r) e^(-G_j) (64 exponentials, not 4096).
                    const bool rank1 = gs[63] >= -80.f;
                    const float sg = scale * vec[kVecGam + r], Gr = gs[r];
#pragma unroll
                    for (int sl = 0; sl < 2; ++sl) {
                        const int j0 = 32 * ih + 16 * sl;
                        float v[16], e[16], x[16];
                        tmem_ld16(tmem + lane_bits + kColGram + j0, v);
#pragma unroll
                        for (int q = 0; q < 4; ++q) load4((rank1 ? vec + kVecIGam : gs) + j0 + 4 * q, e + 4 * q);
                        tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            // branch-free: a 0/1 factor masks the strictly upper part
                            const float keep = (j0 + jj < lim) ? 1.f : 0.f;
                            x[jj] = rank1 ? keep * sg * e[jj] * v[jj]
                                          : keep * scale * __expf(fminf(Gr - e[jj], 0.f)) * v[jj];
                        }
                        if (is_a) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<float4 *>(Af + r * kLdA + j0 + 4 * q) =
                                    make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                        } else {
                            store_row_bf16(pt, r, j0 / 8, x, 2);
                        }
                    }
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarIntra, kIntra);
                if (gcn >= 1) {  // the chain has consumed the previous chunk's T' and T''
                    const bool ok = !intra_poll || mbar_wait(bars + 8 * kBarWT, ph_wt);
                    ph_wt ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                invert_to_operands(Af, Tf, Yb, it, sb + kOffTp, sb + kOffTpp, vec + kVecBG, kL2 ? vec + kVecTpp : bs);
                if (it == 0) mbar_arrive(bars + 8 * (kBarFull + b));  // chunk gcn ready for the chain
                // the next chunk: once its q and k are in, warp 15 starts its Gram (the
                // Gram accumulator was consumed by this chunk's decay masks) while warp
                // 8 waits for its buffers and scans its gates
                if (n + 1 < nchunks) {
                    const uint32_t nb = b ^ 1u;
                    const int L1 = min(64, len - (n + 1) * 64);
                    const bool ok = !intra_poll || mbar_wait(bars + 8 * (kBarTKQ + nb), (ph_tkq >> nb) & 1u);
                    ph_tkq ^= 1u << nb;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                    if (it == kIntraIssuer) issue_gram(sb + (nb ? kOffKQ1 : kOffKQ0));
                    bool ok2 = true;
                    if (warp == 8) {
                        if (gcn + 1 >= 2) ok2 = mbar_wait(bars + 8 * (kBarEmpty + nb), (ph_empty >> nb) & 1u);
                        if (ok2) chunk_gates(nb, L1);
                    }
                    if (l2 && it >= 32 && it < 160) chunk_norms(sb + (nb ? kOffKQ1 : kOffKQ0));
                    if (gcn + 1 >= 2) ph_empty ^= 1u << nb;
                    if (named_sync_or(kBarIntra, kIntra, !ok2)) { aborted = true; break; }
                    if (it < 64) chunk_vectors(nb, L1);
                }
            }
        }
        gn += uint32_t(nchunks);
    }

    if (tid == 0) bulk_wait_all();  // output stores complete before the CTA's shared memory goes away
    if (aborted) {
        // let this thread's own tensor-core work drain (bounded) before freeing tensor memory
        if (tid == 0 || tid == kChain + kIntraIssuer) {
            const uint32_t bar = bars + 8 * (tid == 0 ? kBarC : kBarI);
            mma_commit(bar);
            (void)mbar_wait(bar, tid == 0 ? ph_c : ph_i);
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

bool chunk_tc_supported(const gdn_shape_t &s) {
    // value heads in multiples of 4: the gates arrive as boxes of 4 heads
    return s.dtype == GDN_DTYPE_BF16 && s.head_dim_k == 128 && s.head_dim_v == 128 && s.chunk_size == 64 &&
           s.num_v_heads % 4 == 0;
}

cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t stream, int num_sms) {
    // With no tokens at all there is nothing to load; the fp32 kernel writes
    // the final states (= initial states) of the empty sequences.
    if (a.tokens <= 0) return launch_chunk_simt(a, stream, num_sms);
    CUtensorMap mq, mk, mv, mo, mg, mb, mz;
    if (!make_map(&mq, a.q, a.hk, a.tokens) || !make_map(&mk, a.k, a.hk, a.tokens) ||
        !make_map(&mv, a.v, a.hv, a.tokens) || !make_map(&mo, a.o, a.hv, a.tokens, true) ||
        !make_gate_map(&mg, a.g, a.hv, a.tokens) || !make_gate_map(&mb, a.beta, a.hv, a.tokens))
        return cudaErrorInvalidValue;
    mz = mo;  // not read unless the output side has a gate
    if (a.out.flags && a.out.z && !make_map(&mz, a.out.z, a.hv, a.tokens, true)) return cudaErrorInvalidValue;
    const bool l2 = a.flags & GDN_FLAG_QK_L2NORM, logits = a.flags & GDN_FLAG_GATE_LOGITS;
    const bool out = a.out.flags != 0;
    using KernFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                            PrefillArgs);
    static const KernFn table[8] = {
        chunk_tc_kernel<false, false, false>, chunk_tc_kernel<false, true, false>,
        chunk_tc_kernel<true, false, false>,  chunk_tc_kernel<true, true, false>,
        chunk_tc_kernel<false, false, true>,  chunk_tc_kernel<false, true, true>,
        chunk_tc_kernel<true, false, true>,   chunk_tc_kernel<true, true, true>,
    };
    const KernFn kern = table[(out ? 4 : 0) + (l2 ? 2 : 0) + (logits ? 1 : 0)];
    const uint32_t smem_bytes = out ? kSmemBytesOut : kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_bytes));
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t(a.num_seqs) * a.hv;
    const int grid = int(units < num_sms ? units : num_sms);
    if (grid <= 0) return cudaSuccess;
    // launched as a programmatic dependent of the schedule kernel: its set-up
    // overlaps the schedule, and it waits for the schedule's results on device
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, mg, mb, mz, a);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
