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
//   (4) U^T = U~^T - S W^T   (accumulates into (3), A negated)      128x64x128
//   (5) X1 = S Q^T                                                   128x64x128
//   (6) X2 = U^T P^T,  P = Q K^T (.) Gamma                           128x64x64
//   (7) S += (U^T diag(lambda)) K,  lambda_j = e^(G_C - G_j)         128x128x64
// O[r][i] = gamma_r X1[i][r] + X2[i][r].  Operands are bf16 in
// 128-byte-swizzled shared memory; q, k, v tiles arrive by TMA (no
// multicast).  The fp32 state S lives in tensor memory as the accumulator of
// (7); once per chunk it is read, staged as the bf16 operand of (4) and (5),
// and rescaled by gamma_C in place.
//
// Warp specialisation.  Only (4), (7) and the state pass depend on the state
// carried from the previous chunk; everything else in a chunk does not.  So a
// CTA runs two warp groups on one (sequence, value head) unit:
//   chain  (warps 0-3):  state pass, (4)+(5), U epilogue, (6)+(7), output
//   intra  (warps 4-11): gates and their prefix sums, (1), decay masks A and
//                        P, the triangular inverse (CUDA cores, fp32), T'
//                        and T'', (2)+(3), W^T epilogue -- one chunk ahead.
// They hand chunks over through mbarriers: "full[b]" (intra -> chain: W^T,
// P, U~ in tensor memory and the per-token vectors of buffer b are ready),
// "empty[b]" (chain -> intra: buffer b may be refilled), "wt_free" (the
// single W^T tile has been consumed).  q/k tiles are double-buffered; the
// chain refills a buffer two chunks ahead as soon as its last reader (7)
// completes.  Each group synchronises internally with its own named barrier.
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

constexpr int kThreads = 384;      // warps 0-3: chain group; warps 4-11: intra group
constexpr int kChain = 128, kIntra = 256;
constexpr int kBarChain = 1, kBarIntra = 2;  // named barrier ids (0 is __syncthreads)
constexpr int kLdA = 68;  // fp32 row stride of the A and T scratch matrices (16-byte aligned rows)
constexpr int kLdY = 36;  // fp32 row stride of the inverse's 32 x 32 scratch

// Shared-memory map (bytes from a 1024-byte-aligned base).  Tiles are
// 128-byte-swizzled: "atom columns" of 64 bf16 (128 bytes) per row.
constexpr uint32_t kOffKQ0 = 0;       // [K;Q] buffer 0: 2 atom columns x 128 rows (K 0-63, Q 64-127)
constexpr uint32_t kOffKQ1 = 32768;   // [K;Q] buffer 1
constexpr uint32_t kOffV = 65536;     // V: 2 atom columns x 64 rows (intra only)
constexpr uint32_t kOffWT = 81920;    // W^T: 128 rows (d_k) x 64 tokens
constexpr uint32_t kOffP0 = 98304;    // P = Q K^T (.) Gamma, buffer 0: 64 x 64
constexpr uint32_t kOffP1 = 106496;   // P, buffer 1
constexpr uint32_t kOffS = 114688;    // S operand (bf16): 2 atom columns x 128 rows (chain only)
constexpr uint32_t kOffUT = 147456;   // U^T: 128 rows (d_v) x 64 tokens; then the output staging tile
constexpr uint32_t kOffUTl = 163840;  // U^T diag(lambda)
constexpr uint32_t kOffAf = 180224;   // A, fp32 64 x kLdA; after the inverse: T' (8 KB) and T'' (8 KB)
constexpr uint32_t kOffTp = kOffAf, kOffTpp = kOffAf + 8192;
constexpr uint32_t kOffTf = kOffAf + 64 * kLdA * 4;  // T, fp32 64 x kLdA
constexpr uint32_t kOffY = kOffTf + 64 * kLdA * 4;   // inverse scratch, 32 x kLdY fp32
constexpr uint32_t kOffVec0 = kOffY + 32 * kLdY * 4;  // per-token vectors of buffer 0 (6 x 64 fp32)
constexpr uint32_t kOffVec1 = kOffVec0 + 6 * 64 * 4;  // buffer 1
constexpr uint32_t kOffBar = kOffVec1 + 6 * 64 * 4;   // mbarriers, tensor-memory slot, unit slot
constexpr uint32_t kSmemBytes = kOffBar + 128 + 1024; // + alignment slack
static_assert(kOffTpp + 8192 <= kOffTf, "T' and T'' must fit in the A scratch");
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");
// per-token vectors inside a buffer (floats)
constexpr int kVecG = 0, kVecB = 64, kVecGam = 128, kVecBG = 192, kVecLam = 256, kVecIGam = 320;
// mbarrier slots
constexpr int kBarTKQ = 0, kBarTV = 2, kBarI = 3, kBarC = 4, kBarFull = 5, kBarEmpty = 7, kBarWT = 9, kNumBars = 10;

// Tensor-memory columns (fp32, 128 lanes each).
constexpr uint32_t kColGram = 0, kColW = 64, kColU0 = 128, kColU1 = 192, kColX1 = 256, kColX2 = 320, kColS = 384;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesKQ = 4 * 8192;  // four 64 x 64 bf16 boxes
constexpr uint32_t kBytesV = 2 * 8192;

__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier over one warp group that also ORs a predicate across it.
__device__ __forceinline__ bool named_sync_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void store_row_bf16(uint32_t tile, int row, int chunk0, const float *x, int nchunks) {
#pragma unroll
    for (int c = 0; c < nchunks; ++c) st_shared_v4(tile + sw128_offset(row, chunk0 + c), pack_bf16x8(x + 8 * c));
}

__device__ __forceinline__ void load4(const float *p, float *x) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}

// T = (I + A)^-1 for the 64 x 64 unit-lower-triangular system, fp32, in
// shared memory, by divide and conquer on the block structure
//   [[X, 0], [C, Z]]^-1 = [[X^-1, 0], [-Z^-1 C X^-1, Z^-1]]:
// the four 16 x 16 diagonal blocks by row-wise forward substitution (one
// thread per column), then the two 32 x 32 halves (two 16 x 16 products each),
// then the 64 x 64 matrix (two 32 x 32 products, 2 x 2 outputs per thread).
// Everything of Tf above the diagonal must be zero on entry (it is zeroed once
// and never written).  Called by the 256 threads of the intra group (t = 0..255).
__device__ void invert_unit_lower(const float *Af, float *Tf, float *Y, int t) {
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
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * kLdA + c] = x[r];
    }
    named_sync(kBarIntra, kIntra);
    // 32 x 32 halves p = 0, 1: Y_p = A[32p+16.., 32p..] B_{2p}, T[32p+16.., 32p..] = -B_{2p+1} Y_p
    const int p = t >> 7, e = t & 127, r1 = e >> 3, c1 = (e & 7) * 2;
    {
        const float *Arow = Af + (32 * p + 16 + r1) * kLdA + 32 * p;
        const float *Bm = Tf + (32 * p) * kLdA + 32 * p;
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float av = Arow[m];
            const float2 tv = *reinterpret_cast<const float2 *>(Bm + m * kLdA + c1);
            z0 = fmaf(av, tv.x, z0);
            z1 = fmaf(av, tv.y, z1);
        }
        *reinterpret_cast<float2 *>(Y + (16 * p + r1) * kLdY + c1) = make_float2(z0, z1);
    }
    named_sync(kBarIntra, kIntra);
    {
        const float *Brow = Tf + (32 * p + 16 + r1) * kLdA + 32 * p + 16;
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float bm = Brow[m];  // zero above the diagonal
            const float2 tv = *reinterpret_cast<const float2 *>(Y + (16 * p + m) * kLdY + c1);
            z0 = fmaf(bm, tv.x, z0);
            z1 = fmaf(bm, tv.y, z1);
        }
        *reinterpret_cast<float2 *>(Tf + (32 * p + 16 + r1) * kLdA + 32 * p + c1) = make_float2(-z0, -z1);
    }
    named_sync(kBarIntra, kIntra);
    // 64 x 64: Y = A[32.., 0..32] T_a, T[32.., 0..32] = -T_b Y
    const int r0 = (t >> 4) * 2, c0 = (t & 15) * 2;
    {
        const float *A0 = Af + (32 + r0) * kLdA, *A1 = A0 + kLdA;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            float a0v[4], a1v[4];
            load4(A0 + 4 * k4, a0v);
            load4(A1 + 4 * k4, a1v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 tv = *reinterpret_cast<const float2 *>(Tf + (4 * k4 + u) * kLdA + c0);
                y00 = fmaf(a0v[u], tv.x, y00); y01 = fmaf(a0v[u], tv.y, y01);
                y10 = fmaf(a1v[u], tv.x, y10); y11 = fmaf(a1v[u], tv.y, y11);
            }
        }
        *reinterpret_cast<float2 *>(Y + r0 * kLdY + c0) = make_float2(y00, y01);
        *reinterpret_cast<float2 *>(Y + (r0 + 1) * kLdY + c0) = make_float2(y10, y11);
    }
    named_sync(kBarIntra, kIntra);
    {
        const float *B0 = Tf + (32 + r0) * kLdA + 32, *B1 = B0 + kLdA;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            float b0v[4], b1v[4];
            load4(B0 + 4 * k4, b0v);
            load4(B1 + 4 * k4, b1v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 tv = *reinterpret_cast<const float2 *>(Y + (4 * k4 + u) * kLdY + c0);
                y00 = fmaf(b0v[u], tv.x, y00); y01 = fmaf(b0v[u], tv.y, y01);
                y10 = fmaf(b1v[u], tv.x, y10); y11 = fmaf(b1v[u], tv.y, y11);
            }
        }
        *reinterpret_cast<float2 *>(Tf + (32 + r0) * kLdA + c0) = make_float2(-y00, -y01);
        *reinterpret_cast<float2 *>(Tf + (32 + r0 + 1) * kLdA + c0) = make_float2(-y10, -y11);
    }
    named_sync(kBarIntra, kIntra);
}

// Loads chunk `c0` of q and k for q/k head `hq` into a [K;Q] buffer.
__device__ __forceinline__ void load_kq(uint32_t dst, uint32_t bar, const CUtensorMap *tk, const CUtensorMap *tq,
                                        int hq, int c0) {
    mbar_arrive_expect_tx(bar, kBytesKQ);
    tma_load_3d(dst, tk, 0, hq, c0, bar);
    tma_load_3d(dst + 8192, tq, 0, hq, c0, bar);
    tma_load_3d(dst + 16384, tk, 64, hq, c0, bar);
    tma_load_3d(dst + 24576, tq, 64, hq, c0, bar);
}

__device__ __forceinline__ void load_v(uint32_t dst, uint32_t bar, const CUtensorMap *tv, int h, int c0) {
    mbar_arrive_expect_tx(bar, kBytesV);
    tma_load_3d(dst, tv, 0, h, c0, bar);
    tma_load_3d(dst + 8192, tv, 64, h, c0, bar);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
    extern __shared__ unsigned char smem_raw[];
    // Align to 1024 bytes with a byte offset on the shared array itself (not
    // through an integer cast), so that the compiler keeps every access below in
    // the shared address space (ld.shared / st.shared, not generic loads).
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *Af = reinterpret_cast<float *>(smem + kOffAf);
    float *Tf = reinterpret_cast<float *>(smem + kOffTf);
    float *Yb = reinterpret_cast<float *>(smem + kOffY);
    const uint32_t bars = sb + kOffBar;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 8 * kNumBars);
    int *s_unit = reinterpret_cast<int *>(smem + kOffBar + 8 * kNumBars + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool is_chain = warp < 4;
    const uint32_t lane_bits = uint32_t((warp & 3) * 32) << 16;  // this warp's tensor-memory lane quarter
    WsHeader *hdr = a.sched.hdr;
    if (hdr->status != GDN_OK) return;

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

    const int hv = a.hv, hk = a.hk, group = hv / hk;
    const int total_units = a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
    uint32_t gn = 0;  // chunks this CTA has processed so far (selects buffers and barrier phases)
    uint32_t ph_full = 0, ph_empty = 0, ph_tkq = 0, ph_v = 0, ph_i = 0, ph_c = 0, ph_wt = 0;
    bool aborted = false;

    const uint32_t id_gram = idesc_bf16(128, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 64, true, false);
    const uint32_t id_u = idesc_bf16(128, 64, false, true, true);
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
            load_kq(sb + ((gn & 1) ? kOffKQ1 : kOffKQ0), bars + 8 * (kBarTKQ + (gn & 1)), &tm_k, &tm_q, hq, t0);
            if (nchunks > 1)
                load_kq(sb + (((gn + 1) & 1) ? kOffKQ1 : kOffKQ0), bars + 8 * (kBarTKQ + ((gn + 1) & 1)), &tm_k,
                        &tm_q, hq, t0 + 64);
            load_v(sb + kOffV, bars + 8 * kBarTV, &tm_v, h, t0);
        }

        if (is_chain) {
            // ================= chain group: one thread per state row =================
            const int row = tid;
            // initial state into tensor memory
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
                const uint32_t gcn = gn + n, b = gcn & 1;
                const int c0 = t0 + n * 64, L = min(64, len - n * 64);
                const float *vec = reinterpret_cast<const float *>(smem + (b ? kOffVec1 : kOffVec0));
                const uint32_t kq = sb + (b ? kOffKQ1 : kOffKQ0);
                const uint32_t pt = sb + (b ? kOffP1 : kOffP0);
                const uint32_t colU = b ? kColU1 : kColU0;
                {
                    const bool ok = mbar_wait(bars + 8 * (kBarFull + b), (ph_full >> b) & 1u);
                    ph_full ^= 1u << b;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // state pass: S_n -> bf16 operand, S <- gamma_C S_n in place
                {
                    const float gC = vec[kVecGam + 63];  // padded rows carry g = 0, so G_63 = G_{L-1}
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float v0[32], v1[32];
                        tmem_ld32(tmem + lane_bits + kColS + 64 * hh, v0);
                        tmem_ld32(tmem + lane_bits + kColS + 64 * hh + 32, v1);
                        tmem_wait_ld();
                        store_row_bf16(sb + kOffS + hh * 16384, row, 0, v0, 4);
                        store_row_bf16(sb + kOffS + hh * 16384, row, 4, v1, 4);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            v0[j] *= gC;
                            v1[j] *= gC;
                        }
                        tmem_st32(tmem + lane_bits + kColS + 64 * hh, v0);
                        tmem_st32(tmem + lane_bits + kColS + 64 * hh + 32, v1);
                    }
                    tmem_wait_st();
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarChain, kChain);
                // (4) U^T = U~^T - S W^T and (5) X1 = S Q^T
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                        mma_bf16(tmem + colU, smem_desc(sb + kOffS + off, 16, 1024),
                                 smem_desc(sb + kOffWT + s * 2048, 16384, 1024), id_u, 1);
                    }
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                        mma_bf16(tmem + kColX1, smem_desc(sb + kOffS + off, 16, 1024),
                                 smem_desc(kq + 8192 + off, 16, 1024), id_x, s > 0);
                    }
                    mma_commit(bars + 8 * kBarC);
                }
                {
                    const bool ok = mbar_wait(bars + 8 * kBarC, ph_c);
                    ph_c ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                if (tid == 0) mbar_arrive(bars + 8 * kBarWT);  // W^T consumed
                // U epilogue: U^T rows to bf16 operands (plain and lambda-scaled)
                {
                    float v0[32], v1[32];
                    tmem_ld32(tmem + lane_bits + colU, v0);
                    tmem_ld32(tmem + lane_bits + colU + 32, v1);
                    float l0[32], l1[32];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        load4(vec + kVecLam + 4 * q, l0 + 4 * q);
                        load4(vec + kVecLam + 32 + 4 * q, l1 + 4 * q);
                    }
                    tmem_wait_ld();
                    store_row_bf16(sb + kOffUT, row, 0, v0, 4);
                    store_row_bf16(sb + kOffUT, row, 4, v1, 4);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        l0[j] *= v0[j];
                        l1[j] *= v1[j];
                    }
                    store_row_bf16(sb + kOffUTl, row, 0, l0, 4);
                    store_row_bf16(sb + kOffUTl, row, 4, l1, 4);
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarChain, kChain);
                // (6) X2 = U^T P^T and (7) S += U^T diag(lambda) K
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColX2, smem_desc(sb + kOffUT + s * 32, 16, 1024),
                                 smem_desc(pt + s * 32, 16, 1024), id_x, s > 0);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColS, smem_desc(sb + kOffUTl + s * 32, 16, 1024),
                                 smem_desc(kq + s * 2048, 16384, 1024), id_ds, 1);
                    mma_commit(bars + 8 * kBarC);
                }
                {
                    const bool ok = mbar_wait(bars + 8 * kBarC, ph_c);
                    ph_c ^= 1u;
                    if (named_sync_or(kBarChain, kChain, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // the [K;Q] buffer is free: refill it two chunks ahead
                if (tid == 0 && n + 2 < nchunks) load_kq(kq, bars + 8 * (kBarTKQ + b), &tm_k, &tm_q, hq, c0 + 128);
                // output O[r][i] = gamma_r X1[i][r] + X2[i][r], staged through the
                // U^T tile so that each token row leaves as contiguous 16-byte stores
                {
                    __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffUT);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float x1[32], x2[32];
                        tmem_ld32(tmem + lane_bits + kColX1 + 32 * hh, x1);
                        tmem_ld32(tmem + lane_bits + kColX2 + 32 * hh, x2);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int r = 32 * hh + j;
                            Ot[r * 128 + row] = __float2bfloat16_rn(fmaf(vec[kVecGam + r], x1[j], x2[j]));
                        }
                    }
                }
                tc_fence_before();
                named_sync(kBarChain, kChain);
                for (int e = tid; e < 64 * 16; e += kChain) {
                    const int r = e >> 4, c = e & 15;
                    if (r < L) {
                        const uint4 val = *reinterpret_cast<const uint4 *>(smem + kOffUT + r * 256 + c * 16);
                        *reinterpret_cast<uint4 *>(o + (size_t(c0 + r) * hv + h) * 128 + c * 8) = val;
                    }
                }
                named_sync(kBarChain, kChain);
                if (tid == 0) mbar_arrive(bars + 8 * (kBarEmpty + b));  // buffers b may be refilled
            }
            if (!aborted) {
                // final state out of tensor memory
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
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
            const int ih = (warp - 4) >> 2;              // which 32-column half of a 64-column tile
            float g_next = 0.f, b_next = 0.f;            // gates kept one chunk in flight (it < 64)
            if (it < 64 && it < len) {
                g_next = a.g[size_t(t0 + it) * hv + h];
                b_next = a.beta[size_t(t0 + it) * hv + h];
            }
            for (int n = 0; n < nchunks; ++n) {
                const uint32_t gcn = gn + n, b = gcn & 1;
                const int c0 = t0 + n * 64, L = min(64, len - n * 64);
                float *vec = reinterpret_cast<float *>(smem + (b ? kOffVec1 : kOffVec0));
                float *gs = vec + kVecG, *bs = vec + kVecB;
                const uint32_t kq = sb + (b ? kOffKQ1 : kOffKQ0);
                const uint32_t pt = sb + (b ? kOffP1 : kOffP0);
                const uint32_t colU = b ? kColU1 : kColU0;
                if (gcn >= 2) {  // buffers b were last used by chunk gcn - 2
                    const bool ok = mbar_wait(bars + 8 * (kBarEmpty + b), (ph_empty >> b) & 1u);
                    ph_empty ^= 1u << b;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                if (it < 64) {
                    gs[it] = it < L ? fmaxf(g_next, kGFloor) : 0.f;
                    bs[it] = it < L ? b_next : 0.f;
                    if (n + 1 < nchunks && it < min(64, len - (n + 1) * 64)) {
                        const size_t off = size_t(c0 + 64 + it) * hv + h;
                        g_next = a.g[off];
                        b_next = a.beta[off];
                    }
                }
                {
                    const bool ok = mbar_wait(bars + 8 * (kBarTKQ + b), (ph_tkq >> b) & 1u);
                    ph_tkq ^= 1u << b;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                // (1) Gram
                if (it == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                        mma_bf16(tmem + kColGram, smem_desc(kq + off, 16, 1024), smem_desc(kq + off, 16, 1024),
                                 id_gram, s > 0);
                    }
                    mma_commit(bars + 8 * kBarI);
                }
                // chunk-local prefix sums of g (first intra warp) while the Gram runs
                if (warp == 4) {
                    const float g0 = gs[2 * lane], g1 = gs[2 * lane + 1];
                    float incl = g0 + g1;
#pragma unroll
                    for (int d = 1; d < 32; d <<= 1) {
                        const float tt = __shfl_up_sync(0xffffffffu, incl, d);
                        if (lane >= d) incl += tt;
                    }
                    const float excl = incl - (g0 + g1);
                    gs[2 * lane] = excl + g0;
                    gs[2 * lane + 1] = excl + g0 + g1;
                }
                named_sync(kBarIntra, kIntra);
                if (it < 64) {
                    const float G = gs[it];
                    vec[kVecGam + it] = __expf(G);
                    vec[kVecBG + it] = bs[it] * __expf(G);
                    vec[kVecLam + it] = it < L ? __expf(gs[L - 1] - G) : 0.f;
                    vec[kVecIGam + it] = __expf(-G);
                }
                {
                    const bool ok = mbar_wait(bars + 8 * kBarI, ph_i);
                    ph_i ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                // A (fp32, for the inverse) and P (bf16 operand) from the Gram
                {
                    float v[32], x[32];
                    tmem_ld32(tmem + lane_bits + kColGram + 32 * ih, v);
                    const int r = irow & 63;
                    const bool is_a = irow < 64;
                    const float scale = is_a ? bs[r] : 1.f;
                    const int lim = is_a ? r : r + 1;  // A: j < r;  P: j <= r
                    // Gamma_rj = e^(G_r - G_j).  While the chunk's total log-decay is
                    // at least -80, e^(-G_j) stays finite in fp32 and Gamma is the
                    // rank-1 product e^(G_r) e^(-G_j) (64 exponentials, not 4096).
                    if (gs[63] >= -80.f) {
                        float ig[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) load4(vec + kVecIGam + 32 * ih + 4 * q, ig + 4 * q);
                        const float sg = scale * vec[kVecGam + r];
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float keep = (32 * ih + j < lim) ? 1.f : 0.f;
                            x[j] = keep * sg * ig[j] * v[j];
                        }
                    } else {
                        float gj[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) load4(gs + 32 * ih + 4 * q, gj + 4 * q);
                        const float Gr = gs[r];
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            // branch-free: every lane evaluates the exponential, a 0/1 factor masks it
                            const float keep = (32 * ih + j < lim) ? 1.f : 0.f;
                            x[j] = keep * scale * __expf(fminf(Gr - gj[j], 0.f)) * v[j];
                        }
                    }
                    if (is_a) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4 *>(Af + r * kLdA + 32 * ih + 4 * q) =
                                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                    } else {
                        store_row_bf16(pt, r, 4 * ih, x, 4);
                    }
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarIntra, kIntra);
                invert_unit_lower(Af, Tf, Yb, it);
                // T' = T diag(beta gamma) and T'' = T diag(beta) as bf16 operands (over A)
                for (int e = it; e < 64 * 8; e += kIntra) {
                    const int r = e >> 3, c8 = e & 7;
                    float tv[8], b1[8], b2[8], x1[8], x2[8];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        load4(Tf + r * kLdA + 8 * c8 + 4 * q, tv + 4 * q);  // zero above the diagonal
                        load4(vec + kVecBG + 8 * c8 + 4 * q, b1 + 4 * q);
                        load4(bs + 8 * c8 + 4 * q, b2 + 4 * q);
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        x1[u] = tv[u] * b1[u];
                        x2[u] = tv[u] * b2[u];
                    }
                    st_shared_v4(sb + kOffTp + sw128_offset(r, c8), pack_bf16x8(x1));
                    st_shared_v4(sb + kOffTpp + sw128_offset(r, c8), pack_bf16x8(x2));
                }
                fence_proxy_async_shared();
                {
                    const bool ok = mbar_wait(bars + 8 * kBarTV, ph_v);
                    ph_v ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                // (2) W^T and (3) U~^T
                if (it == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + kColW, smem_desc(kq + s * 2048, 16384, 1024),
                                 smem_desc(sb + kOffTp + s * 32, 16, 1024), id_w, s > 0);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(tmem + colU, smem_desc(sb + kOffV + s * 2048, 8192, 1024),
                                 smem_desc(sb + kOffTpp + s * 32, 16, 1024), id_w, s > 0);
                    mma_commit(bars + 8 * kBarI);
                }
                {
                    const bool ok = mbar_wait(bars + 8 * kBarI, ph_i);
                    ph_i ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                tc_fence_after();
                if (it == 0 && n + 1 < nchunks) load_v(sb + kOffV, bars + 8 * kBarTV, &tm_v, h, c0 + 64);
                if (gcn >= 1) {  // the chain has consumed the previous chunk's W^T
                    const bool ok = mbar_wait(bars + 8 * kBarWT, ph_wt);
                    ph_wt ^= 1u;
                    if (named_sync_or(kBarIntra, kIntra, !ok)) { aborted = true; break; }
                }
                {
                    float v[32];
                    tmem_ld32(tmem + lane_bits + kColW + 32 * ih, v);
                    tmem_wait_ld();
                    store_row_bf16(sb + kOffWT, irow, 4 * ih, v, 4);
                }
                fence_proxy_async_shared();
                tc_fence_before();
                named_sync(kBarIntra, kIntra);
                if (it == 0) mbar_arrive(bars + 8 * (kBarFull + b));  // chunk gcn ready for the chain
            }
        }
        gn += uint32_t(nchunks);
    }

    if (aborted) {
        // let this thread's own tensor-core work drain (bounded) before freeing tensor memory
        if (tid == 0 || tid == kChain) {
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [tokens, heads, 128] bf16 viewed as a 3-D tensor (d fastest), boxes of
// 64 (d) x 1 (head) x 64 (tokens), 128-byte swizzle; rows past the last token
// read as zeros.
bool make_map(CUtensorMap *map, const void *base, int heads, int tokens) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, cuuint64_t(heads), cuuint64_t(tokens)};
    const cuuint64_t strides[2] = {128 * 2, cuuint64_t(heads) * 128 * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(const gdn_shape_t &s) {
    return s.dtype == GDN_DTYPE_BF16 && s.head_dim_k == 128 && s.head_dim_v == 128 && s.chunk_size == 64;
}

cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t stream, int num_sms) {
    // With no tokens at all there is nothing to load; the fp32 kernel writes
    // the final states (= initial states) of the empty sequences.
    if (a.tokens <= 0) return launch_chunk_simt(a, stream, num_sms);
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.hk, a.tokens) || !make_map(&mk, a.k, a.hk, a.tokens) ||
        !make_map(&mv, a.v, a.hv, a.tokens))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    if (e != cudaSuccess) return e;
    const int64_t units = int64_t(a.num_seqs) * a.hv;
    const int grid = int(units < num_sms ? units : num_sms);
    if (grid <= 0) return cudaSuccess;
    chunk_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(mq, mk, mv, a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
