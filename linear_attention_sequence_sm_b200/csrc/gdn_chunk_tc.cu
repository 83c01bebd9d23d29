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
//   (7) dS = (U^T diag(lambda)) K,  lambda_j = e^(G_C - G_j)         128x128x64
// O[r][i] = gamma_r X1[i][r] + X2[i][r];  S <- gamma_C S + dS.
// Operands are bf16 in 128-byte-swizzled shared memory; q, k, v tiles arrive
// by TMA (no multicast); the fp32 state S lives in registers (thread = state
// row, half of the key columns) and is re-staged as a bf16 operand each
// chunk.  The triangular inverse runs on the CUDA cores in fp32 (16 x 16
// diagonal blocks by forward substitution, then the off-diagonal blocks).
//
// One CTA per SM (the shared-memory footprint forces it) owns a unit
// (sequence, value head) at a time, taking units longest sequence first from
// an atomic counter, and walks the unit's chunks in order.  Every wait on an
// mbarrier is bounded; a timeout records GDN_ERR_DEVICE_CHECK (bad_index -2)
// in the workspace status word and the CTA frees its tensor memory and exits.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThreads = 256;
constexpr int kLdA = 68;  // fp32 row stride of the A and T scratch matrices (16-byte aligned rows)
constexpr int kLdY = 36;  // fp32 row stride of the inverse's 32 x 32 scratch

// Shared-memory map (bytes from a 1024-byte-aligned base).  Tiles are
// 128-byte-swizzled: "atom columns" of 64 bf16 (128 bytes) per row.
constexpr uint32_t kOffKQ0 = 0;       // [K;Q] chunk buffer 0: 2 atom columns x 128 rows (K 0-63, Q 64-127)
constexpr uint32_t kOffKQ1 = 32768;   // [K;Q] chunk buffer 1
constexpr uint32_t kOffV = 65536;     // V: 2 atom columns x 64 rows
constexpr uint32_t kOffS = 81920;     // S operand (bf16): 2 atom columns x 128 rows (d_v)
constexpr uint32_t kOffTp = 114688;   // T diag(beta gamma): 64 x 64
constexpr uint32_t kOffTpp = 122880;  // T diag(beta): 64 x 64
constexpr uint32_t kOffWT = 131072;   // W^T: 128 rows (d_k) x 64 tokens
constexpr uint32_t kOffP = 147456;    // P: 64 x 64
constexpr uint32_t kOffUT = 155648;   // U^T: 128 rows (d_v) x 64 tokens
constexpr uint32_t kOffUTl = 172032;  // U^T diag(lambda)
constexpr uint32_t kOffAf = 188416;   // A, fp32 64 x kLdA
constexpr uint32_t kOffTf = kOffAf + 64 * kLdA * 4;  // T, fp32 64 x kLdA
constexpr uint32_t kOffY = kOffTf + 64 * kLdA * 4;   // inverse scratch, 32 x kLdY fp32
constexpr uint32_t kOffVec = kOffY + 32 * kLdY * 4;  // per-token vectors, 8 x 64 fp32
constexpr uint32_t kOffBar = kOffVec + 8 * 64 * 4;   // 4 mbarriers + tensor-memory slot
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024; // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 per-block limit");

// Tensor-memory columns (fp32, 128 lanes each).  The state S (d_v lanes x
// d_k columns) lives at kColS for the whole unit and is the accumulator of
// the state-update product.
constexpr uint32_t kColGram = 0, kColW = 64, kColU = 128, kColX1 = 192, kColX2 = 256, kColS = 320;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesKQ = 4 * 8192;  // four 64 x 64 bf16 boxes
constexpr uint32_t kBytesV = 2 * 8192;

__device__ __forceinline__ void store_row_bf16(uint32_t tile, int row, int chunk0, const float *x, int nchunks) {
#pragma unroll
    for (int c = 0; c < nchunks; ++c) st_shared_v4(tile + sw128_offset(row, chunk0 + c), pack_bf16x8(x + 8 * c));
}

// T = (I + A)^-1 for the 64 x 64 unit-lower-triangular system, fp32, in
// shared memory, by divide and conquer on the block structure
//   [[X, 0], [C, Z]]^-1 = [[X^-1, 0], [-Z^-1 C X^-1, Z^-1]]:
// the four 16 x 16 diagonal blocks by row-wise forward substitution (one
// thread per column), then the two 32 x 32 halves (two 16 x 16 products each),
// then the 64 x 64 matrix (two 32 x 32 products, 2 x 2 outputs per thread).
// The strictly-upper 16 x 16 blocks inside each 32 x 32 half must be zero in
// Tf on entry (they are zeroed once and never written).  All threads call it.
__device__ void invert_unit_lower(const float *Af, float *Tf, float *Y, int tid) {
    if (tid < 64) {
        const int b = tid >> 4, c = tid & 15;
        const float *Ab = Af + (16 * b) * kLdA + 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float a[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 t = *reinterpret_cast<const float4 *>(Ab + r * kLdA + 4 * q);
                a[4 * q] = t.x; a[4 * q + 1] = t.y; a[4 * q + 2] = t.z; a[4 * q + 3] = t.w;
            }
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
    __syncthreads();
    // 32 x 32 halves p = 0, 1: Y_p = A[32p+16.., 32p..] B_{2p}, T[32p+16.., 32p..] = -B_{2p+1} Y_p
    const int p = tid >> 7, e = tid & 127, r1 = e >> 3, c1 = (e & 7) * 2;
    {
        const float *Arow = Af + (32 * p + 16 + r1) * kLdA + 32 * p;
        const float *Bm = Tf + (32 * p) * kLdA + 32 * p;
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float a = Arow[m];
            const float2 t = *reinterpret_cast<const float2 *>(Bm + m * kLdA + c1);
            z0 = fmaf(a, t.x, z0);
            z1 = fmaf(a, t.y, z1);
        }
        *reinterpret_cast<float2 *>(Y + (16 * p + r1) * kLdY + c1) = make_float2(z0, z1);
    }
    __syncthreads();
    {
        const float *Brow = Tf + (32 * p + 16 + r1) * kLdA + 32 * p + 16;
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float bm = Brow[m];  // zero above the diagonal
            const float2 t = *reinterpret_cast<const float2 *>(Y + (16 * p + m) * kLdY + c1);
            z0 = fmaf(bm, t.x, z0);
            z1 = fmaf(bm, t.y, z1);
        }
        *reinterpret_cast<float2 *>(Tf + (32 * p + 16 + r1) * kLdA + 32 * p + c1) = make_float2(-z0, -z1);
    }
    __syncthreads();
    // 64 x 64: Y = A[32.., 0..32] T_a, T[32.., 0..32] = -T_b Y
    const int r0 = (tid >> 4) * 2, c0 = (tid & 15) * 2;
    {
        const float *A0 = Af + (32 + r0) * kLdA, *A1 = A0 + kLdA;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 a0 = *reinterpret_cast<const float4 *>(A0 + 4 * k4);
            const float4 a1 = *reinterpret_cast<const float4 *>(A1 + 4 * k4);
            const float a0v[4] = {a0.x, a0.y, a0.z, a0.w}, a1v[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 t = *reinterpret_cast<const float2 *>(Tf + (4 * k4 + u) * kLdA + c0);
                y00 = fmaf(a0v[u], t.x, y00); y01 = fmaf(a0v[u], t.y, y01);
                y10 = fmaf(a1v[u], t.x, y10); y11 = fmaf(a1v[u], t.y, y11);
            }
        }
        *reinterpret_cast<float2 *>(Y + r0 * kLdY + c0) = make_float2(y00, y01);
        *reinterpret_cast<float2 *>(Y + (r0 + 1) * kLdY + c0) = make_float2(y10, y11);
    }
    __syncthreads();
    {
        const float *B0 = Tf + (32 + r0) * kLdA + 32, *B1 = B0 + kLdA;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 b0 = *reinterpret_cast<const float4 *>(B0 + 4 * k4);
            const float4 b1 = *reinterpret_cast<const float4 *>(B1 + 4 * k4);
            const float b0v[4] = {b0.x, b0.y, b0.z, b0.w}, b1v[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 t = *reinterpret_cast<const float2 *>(Y + (4 * k4 + u) * kLdY + c0);
                y00 = fmaf(b0v[u], t.x, y00); y01 = fmaf(b0v[u], t.y, y01);
                y10 = fmaf(b1v[u], t.x, y10); y11 = fmaf(b1v[u], t.y, y11);
            }
        }
        *reinterpret_cast<float2 *>(Tf + (32 + r0) * kLdA + c0) = make_float2(-y00, -y01);
        *reinterpret_cast<float2 *>(Tf + (32 + r0 + 1) * kLdA + c0) = make_float2(-y10, -y11);
    }
    __syncthreads();
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
    float *gs = reinterpret_cast<float *>(smem + kOffVec);  // g, then its prefix sums G
    float *bs = gs + 64;                                   // beta
    float *gam = gs + 128;                                 // gamma = e^G
    float *bg = gs + 192;                                  // beta gamma
    float *lam = gs + 256;                                 // e^(G_C - G), 0 past the sequence end
    float *igam = gs + 320;                                // e^(-G), used when the chunk's decay is mild
    const uint32_t bar_kq0 = sb + kOffBar, bar_kq1 = sb + kOffBar + 8, bar_v = sb + kOffBar + 16,
                   bar_mma = sb + kOffBar + 24;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kOffBar + 32);
    int *s_unit = reinterpret_cast<int *>(smem + kOffBar + 40);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;  // tensor-memory lane = accumulator row of this thread
    const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
    WsHeader *hdr = a.sched.hdr;
    if (hdr->status != GDN_OK) return;

    if (tid == 0) {
        mbar_init(bar_kq0, 1);
        mbar_init(bar_kq1, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
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
    // T starts all zero: the inverse writes only the lower-triangular blocks
    // (and zeros above the diagonal inside the diagonal blocks), so everything
    // above the diagonal reads as zero for the rest of the kernel.
    for (int e = tid; e < 64 * kLdA; e += kThreads) Tf[e] = 0.f;
    __syncthreads();

    const int hv = a.hv, hk = a.hk, group = hv / hk;
    const int total_units = a.num_seqs * hv;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
    uint32_t ph_kq0 = 0, ph_kq1 = 0, ph_v = 0, ph_mma = 0;
    uint32_t pending = 0;  // (tid 0) bit 0/1: KQ buffer load in flight, bit 2: V load in flight
    bool aborted = false;

    const uint32_t id_gram = idesc_bf16(128, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 64, true, false);
    const uint32_t id_u = idesc_bf16(128, 64, false, true, true);
    const uint32_t id_x = idesc_bf16(128, 64, false, false);
    const uint32_t id_ds = idesc_bf16(128, 128, false, true);  // state update, accumulates into S

    for (;;) {
        if (tid == 0) *s_unit = int(atomicAdd(&hdr->next_unit, 1u));
        __syncthreads();
        const int unit = *s_unit;
        __syncthreads();
        if (unit >= total_units) break;
        const int seq = a.sched.order[unit / hv];
        const int h = unit % hv, hq = h / group;
        const int t0 = a.sched.start[seq], len = a.sched.len[seq];
        const int nchunks = (len + 63) / 64;
        const size_t sbase = (size_t(seq) * hv + h) * 128 * 128;

        if (tid == 0 && nchunks > 0) {
            mbar_arrive_expect_tx(bar_kq0, kBytesKQ);
            tma_load_3d(sb + kOffKQ0, &tm_k, 0, hq, t0, bar_kq0);
            tma_load_3d(sb + kOffKQ0 + 8192, &tm_q, 0, hq, t0, bar_kq0);
            tma_load_3d(sb + kOffKQ0 + 16384, &tm_k, 64, hq, t0, bar_kq0);
            tma_load_3d(sb + kOffKQ0 + 24576, &tm_q, 64, hq, t0, bar_kq0);
            mbar_arrive_expect_tx(bar_v, kBytesV);
            tma_load_3d(sb + kOffV, &tm_v, 0, h, t0, bar_v);
            tma_load_3d(sb + kOffV + 8192, &tm_v, 64, h, t0, bar_v);
            pending |= 1u | 4u;
        }
        // gates of the first chunk (threads 0-63 keep one chunk of g, beta in flight)
        float g_next = 0.f, b_next = 0.f;
        if (tid < 64 && tid < len) {
            g_next = a.g[size_t(t0 + tid) * hv + h];
            b_next = a.beta[size_t(t0 + tid) * hv + h];
        }
        // initial state into tensor memory (this thread: lane `row`, 64 key columns)
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
            float v[32];
            if (a.s0) {
                const float4 *src =
                    reinterpret_cast<const float4 *>(a.s0 + sbase + size_t(row) * 128 + 64 * half + 32 * p2);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 x = src[c];
                    v[4 * c] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = 0.f;
            }
            tmem_st32(tmem + lane_bits + kColS + 64 * half + 32 * p2, v);
        }
        tmem_wait_st();

        for (int n = 0; n < nchunks; ++n) {
            const int c0 = t0 + n * 64;
            const int L = min(64, len - n * 64);
            const int buf = n & 1;
            const uint32_t kq = sb + (buf ? kOffKQ1 : kOffKQ0);
            if (tid < 64) {
                gs[tid] = tid < L ? fmaxf(g_next, kGFloor) : 0.f;
                bs[tid] = tid < L ? b_next : 0.f;
                // prefetch the next chunk's gates; they are consumed one chunk later
                if (n + 1 < nchunks && tid < min(64, len - (n + 1) * 64)) {
                    const size_t off = size_t(c0 + 64 + tid) * hv + h;
                    g_next = a.g[off];
                    b_next = a.beta[off];
                }
            }
            // (1) Gram, once this chunk's K and Q are in
            {
                const bool ok = mbar_wait(buf ? bar_kq1 : bar_kq0, buf ? ph_kq1 : ph_kq0);
                if (buf) ph_kq1 ^= 1; else ph_kq0 ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            if (tid == 0) {
                pending &= ~(1u << buf);
                if (n + 1 < nchunks) {
                    const uint32_t nb = buf ? kOffKQ0 : kOffKQ1, nbar = buf ? bar_kq0 : bar_kq1;
                    mbar_arrive_expect_tx(nbar, kBytesKQ);
                    tma_load_3d(sb + nb, &tm_k, 0, hq, c0 + 64, nbar);
                    tma_load_3d(sb + nb + 8192, &tm_q, 0, hq, c0 + 64, nbar);
                    tma_load_3d(sb + nb + 16384, &tm_k, 64, hq, c0 + 64, nbar);
                    tma_load_3d(sb + nb + 24576, &tm_q, 64, hq, c0 + 64, nbar);
                    pending |= 1u << (buf ^ 1);
                }
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_bf16(tmem + kColGram, smem_desc(kq + off, 16, 1024), smem_desc(kq + off, 16, 1024), id_gram,
                             s > 0);
                }
                mma_commit(bar_mma);
            }
            // chunk-local prefix sums of g (warp 0) while the Gram runs
            if (warp == 0) {
                const float g0 = gs[2 * lane], g1 = gs[2 * lane + 1];
                float incl = g0 + g1;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float t = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += t;
                }
                const float excl = incl - (g0 + g1);
                gs[2 * lane] = excl + g0;
                gs[2 * lane + 1] = excl + g0 + g1;
            }
            __syncthreads();
            if (tid < 64) {
                const float G = gs[tid];
                gam[tid] = __expf(G);
                bg[tid] = bs[tid] * __expf(G);
                lam[tid] = tid < L ? __expf(gs[L - 1] - G) : 0.f;
                igam[tid] = __expf(-G);
            }
            // S pass: the chunk-start state S_n becomes the bf16 operand, and the
            // fp32 state in tensor memory is decayed to gamma_C S_n so that the
            // state-update product can accumulate onto it.  Padded rows carry
            // g = 0, so G_63 = G_{L-1}.
            {
                const float gC = __expf(gs[63]);
                float v0[32], v1[32];
                tmem_ld32(tmem + lane_bits + kColS + 64 * half, v0);
                tmem_ld32(tmem + lane_bits + kColS + 64 * half + 32, v1);
                tmem_wait_ld();
                store_row_bf16(sb + kOffS + half * 16384, row, 0, v0, 4);
                store_row_bf16(sb + kOffS + half * 16384, row, 4, v1, 4);
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    v0[jj] *= gC;
                    v1[jj] *= gC;
                }
                tmem_st32(tmem + lane_bits + kColS + 64 * half, v0);
                tmem_st32(tmem + lane_bits + kColS + 64 * half + 32, v1);
                tmem_wait_st();
            }
            fence_proxy_async_shared();
            {
                const bool ok = mbar_wait(bar_mma, ph_mma);
                ph_mma ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            tc_fence_after();
            // A (fp32, for the inverse) and P (bf16 operand) from the Gram
            {
                float v[32], gj[32];
                tmem_ld32(tmem + lane_bits + kColGram + 32 * half, v);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 t = *reinterpret_cast<const float4 *>(gs + 32 * half + 4 * q);
                    gj[4 * q] = t.x; gj[4 * q + 1] = t.y; gj[4 * q + 2] = t.z; gj[4 * q + 3] = t.w;
                }
                const int r = row & 63;
                const float Gr = gs[r];
                const bool is_a = row < 64;
                const float scale = is_a ? bs[r] : 1.f;
                const int lim = is_a ? r : r + 1;  // A: j < r;  P: j <= r
                float x[32];
                // Gamma_rj = e^(G_r - G_j).  While the chunk's total log-decay is
                // at least -80, e^(-G_j) stays finite in fp32 and Gamma is the
                // rank-1 product e^(G_r) e^(-G_j) (64 exponentials, not 4096).
                if (gs[63] >= -80.f) {
                    float ig[32];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 t = *reinterpret_cast<const float4 *>(igam + 32 * half + 4 * q);
                        ig[4 * q] = t.x; ig[4 * q + 1] = t.y; ig[4 * q + 2] = t.z; ig[4 * q + 3] = t.w;
                    }
                    const float sg = scale * gam[r];
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const float keep = (32 * half + jj < lim) ? 1.f : 0.f;
                        x[jj] = keep * sg * ig[jj] * v[jj];
                    }
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        // branch-free: every lane evaluates the exponential, a 0/1 factor masks it
                        const float keep = (32 * half + jj < lim) ? 1.f : 0.f;
                        x[jj] = keep * scale * __expf(fminf(Gr - gj[jj], 0.f)) * v[jj];
                    }
                }
                if (is_a) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(Af + r * kLdA + 32 * half + 4 * q) =
                            make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                } else {
                    store_row_bf16(sb + kOffP, r, 4 * half, x, 4);
                }
            }
            fence_proxy_async_shared();
            tc_fence_before();
            __syncthreads();
            invert_unit_lower(Af, Tf, Yb, tid);
            for (int e = tid; e < 64 * 8; e += kThreads) {
                const int r = e >> 3, c8 = e & 7;
                float t[8], b1[8], b2[8], x1[8], x2[8];
#pragma unroll
                for (int hq4 = 0; hq4 < 2; ++hq4) {
                    const float4 tv = *reinterpret_cast<const float4 *>(Tf + r * kLdA + 8 * c8 + 4 * hq4);  // zero above the diagonal
                    const float4 bv = *reinterpret_cast<const float4 *>(bg + 8 * c8 + 4 * hq4);
                    const float4 sv = *reinterpret_cast<const float4 *>(bs + 8 * c8 + 4 * hq4);
                    t[4 * hq4] = tv.x; t[4 * hq4 + 1] = tv.y; t[4 * hq4 + 2] = tv.z; t[4 * hq4 + 3] = tv.w;
                    b1[4 * hq4] = bv.x; b1[4 * hq4 + 1] = bv.y; b1[4 * hq4 + 2] = bv.z; b1[4 * hq4 + 3] = bv.w;
                    b2[4 * hq4] = sv.x; b2[4 * hq4 + 1] = sv.y; b2[4 * hq4 + 2] = sv.z; b2[4 * hq4 + 3] = sv.w;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    x1[u] = t[u] * b1[u];
                    x2[u] = t[u] * b2[u];
                }
                st_shared_v4(sb + kOffTp + sw128_offset(r, c8), pack_bf16x8(x1));
                st_shared_v4(sb + kOffTpp + sw128_offset(r, c8), pack_bf16x8(x2));
            }
            fence_proxy_async_shared();
            {
                const bool ok = mbar_wait(bar_v, ph_v);
                ph_v ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            // (2) W^T, (3) U~^T, (5) X1 = S Q^T
            if (tid == 0) {
                pending &= ~4u;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kColW, smem_desc(kq + s * 2048, 16384, 1024),
                             smem_desc(sb + kOffTp + s * 32, 16, 1024), id_w, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kColU, smem_desc(sb + kOffV + s * 2048, 8192, 1024),
                             smem_desc(sb + kOffTpp + s * 32, 16, 1024), id_w, s > 0);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_bf16(tmem + kColX1, smem_desc(sb + kOffS + off, 16, 1024),
                             smem_desc(kq + 8192 + off, 16, 1024), id_x, s > 0);
                }
                mma_commit(bar_mma);
            }
            {
                const bool ok = mbar_wait(bar_mma, ph_mma);
                ph_mma ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            tc_fence_after();
            if (tid == 0 && n + 1 < nchunks) {
                mbar_arrive_expect_tx(bar_v, kBytesV);
                tma_load_3d(sb + kOffV, &tm_v, 0, h, c0 + 64, bar_v);
                tma_load_3d(sb + kOffV + 8192, &tm_v, 64, h, c0 + 64, bar_v);
                pending |= 4u;
            }
            {
                float v[32];
                tmem_ld32(tmem + lane_bits + kColW + 32 * half, v);
                tmem_wait_ld();
                store_row_bf16(sb + kOffWT, row, 4 * half, v, 4);
            }
            fence_proxy_async_shared();
            tc_fence_before();
            __syncthreads();
            // (4) U^T = U~^T - S W^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_bf16(tmem + kColU, smem_desc(sb + kOffS + off, 16, 1024),
                             smem_desc(sb + kOffWT + s * 2048, 16384, 1024), id_u, 1);
                }
                mma_commit(bar_mma);
            }
            {
                const bool ok = mbar_wait(bar_mma, ph_mma);
                ph_mma ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            tc_fence_after();
            {
                float v[32], w[32];
                tmem_ld32(tmem + lane_bits + kColU + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) w[jj] = v[jj] * lam[32 * half + jj];
                store_row_bf16(sb + kOffUT, row, 4 * half, v, 4);
                store_row_bf16(sb + kOffUTl, row, 4 * half, w, 4);
            }
            fence_proxy_async_shared();
            tc_fence_before();
            __syncthreads();
            // (6) X2 = U^T P^T, (7) S += U^T diag(lambda) K
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kColX2, smem_desc(sb + kOffUT + s * 32, 16, 1024),
                             smem_desc(sb + kOffP + s * 32, 16, 1024), id_x, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kColS, smem_desc(sb + kOffUTl + s * 32, 16, 1024),
                             smem_desc(kq + s * 2048, 16384, 1024), id_ds, 1);
                mma_commit(bar_mma);
            }
            {
                const bool ok = mbar_wait(bar_mma, ph_mma);
                ph_mma ^= 1;
                if (__syncthreads_or(!ok)) { aborted = true; break; }
            }
            tc_fence_after();
            // O[r][i] = gamma_r X1[i][r] + X2[i][r], staged through shared memory
            // (over the inverse's scratch) so that each token row leaves as
            // contiguous 16-byte stores
            {
                float x1[32], x2[32];
                tmem_ld32(tmem + lane_bits + kColX1 + 32 * half, x1);
                tmem_ld32(tmem + lane_bits + kColX2 + 32 * half, x2);
                tmem_wait_ld();
                __nv_bfloat16 *Ot = reinterpret_cast<__nv_bfloat16 *>(smem + kOffAf);
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int r = 32 * half + jj;
                    Ot[r * 128 + row] = __float2bfloat16_rn(fmaf(gam[r], x1[jj], x2[jj]));
                }
            }
            tc_fence_before();
            __syncthreads();
            for (int e = tid; e < 64 * 16; e += kThreads) {
                const int r = e >> 4, c = e & 15;
                if (r < L) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(smem + kOffAf + r * 256 + c * 16);
                    *reinterpret_cast<uint4 *>(o + (size_t(c0 + r) * hv + h) * 128 + c * 8) = val;
                }
            }
            __syncthreads();
        }
        if (aborted) break;
        // final state out of tensor memory
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
            float v[32];
            tmem_ld32(tmem + lane_bits + kColS + 64 * half + 32 * p2, v);
            tmem_wait_ld();
            if (a.s_final) {
                float4 *dst = reinterpret_cast<float4 *>(a.s_final + sbase + size_t(row) * 128 + 64 * half + 32 * p2);
#pragma unroll
                for (int c = 0; c < 8; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
        }
        tc_fence_before();
    }

    if (aborted && tid == 0) {
        // let this CTA's own asynchronous work drain (bounded) before freeing tensor memory
        mma_commit(bar_mma);
        (void)mbar_wait(bar_mma, ph_mma);
        if (pending & 1u) (void)mbar_wait(bar_kq0, ph_kq0);
        if (pending & 2u) (void)mbar_wait(bar_kq1, ph_kq1);
        if (pending & 4u) (void)mbar_wait(bar_v, ph_v);
        hdr->bad_index = -2;
        atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
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
