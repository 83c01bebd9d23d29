// gdn_backward_tc.cu -- gradients of the gated delta rule on the tensor cores
// (bf16 inputs, d_k = d_v = 128, chunks of C = 64 tokens).
//
// The pages train the layer through the chunked form ("Architecture Thread
// I", the Gated DeltaNet section; "Gated Attention Architectures", sections 2
// and 3).  Per chunk, with start state S_c and G, gamma, lambda, Gamma, A, T,
// W, U~, U, P as in the forward (U = U~ - W S_c^T), the two state
// recurrences each become one product per chunk:
//   S_{c+1} = gamma_L S_c + U^T diag(lambda) K = S_c M'_c + U~^T diag(lambda) K,
//       M'_c = gamma_L I - W^T diag(lambda) K                      (d_k x d_k)
//   dS_c = gamma_L dS_{c+1} + dO^T diag(gamma) Q - dU^T W = dS_{c+1} M'_c^T + dO^T X_c,
//       X_c = diag(gamma) Q - P W,  dU = diag(lambda) K dS_{c+1}^T + P^T dO
// (dS_{c+1} is the gradient of the chunk's end state).  Three kernels after
// the schedule kernel (which fills chunk_base):
//   1. factors, every (chunk, value head) item at once: T, W, U~, P from the
//      chunk alone; writes M'_c, U~ diag(lambda), X_c, W, T, T diag(beta)
//      and T diag(beta gamma) to the item;
//   2. chains, one CTA per (sequence, value head) and direction: the state
//      recurrence forward, keeping every chunk's start state, and the
//      state-gradient recurrence backward, keeping every chunk's end-state
//      gradient (and returning dS_0);
//   3. gradients, every (chunk, value head, half of d_v) at once: the rest of
//      the reverse mode of the chunk from its S_c and dS_{c+1}:
//        U^T  = V^T T''^T - S_c W^T,   dU^T = lambda Z^T + dO^T P,  Z^T = dS K^T
//        dQ   = diag(gamma) dO S_c + (dP (.) Gamma) K,   dP = dO U^T (lower)
//        dK   = diag(lambda) U dS + (dP (.) Gamma)^T Q + (T diag(beta gamma))^T dW + (dKK + dKK^T) K
//        dW   = -dU S_c,  dV = (T diag(beta))^T dU,
//        dT   = dW K^T diag(beta gamma) + dU V^T diag(beta)  (lower),
//        dA   = -T^T (dT T^T),  dKK = dA (.) beta Gamma  (strictly lower),
//      the decay and beta gradients as row and column sums of these
//      products, and dg as reverse prefix sums of dG inside the chunk.
// Every d_v row enters dS, dU and dv alone and the shared gradients (dq, dk,
// dg, dbeta) linearly, so the two halves of d_v are independent units.  A CTA
// takes the units of one (chunk, q/k head) in turn and sums their dq and dk
// shares in registers; dg and dbeta shares are added with atomics.
//
// Precision: the tensor cores take bf16 operands.  q, k, v and dO are exact
// in bf16; every fp32 operand is split into a bf16 value and a bf16
// residual, x = hi + lo (about 16 mantissa bits), and a product with one
// split operand takes two instructions (hi, lo), with two split operands
// three (hi hi + hi lo + lo hi), accumulating in fp32 in tensor memory.  The
// chunk inverse runs in fp32 with split-tf32 block products.
//
// Every wait is bounded; a timeout records GDN_ERR_DEVICE_CHECK with
// bad_index -6 (factors), -7 (chains) or -8 (gradients).
#include "gdn_internal.cuh"
#include "gdn_inverse.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int kThr = 256;

// ---------------------------------------------------------------------------
// One (chunk, value head) item, written by the factor kernel.  Tiles are bf16
// in the 128-byte swizzle (rows of 64 elements per atom, atoms of a tile at a
// fixed stride), each as a value part then a residual part.
//   M'   [128][128]  2 atoms of 16 KB a part              (d_k x d_k)
//   Ul   [64][128]   U~ diag(lambda), tokens x d_v         2 atoms of 8 KB
//   X    [64][128]   X_c, tokens x d_k
//   W    [64][128]   W, tokens x d_k
//   T, Tb, Tbg [64][64]  T, T diag(beta), T diag(beta gamma), 8 KB a part
// A checkpoint (chunk start state, or end-state gradient) is a [128][128]
// tile pair laid out as M'.
// ---------------------------------------------------------------------------
constexpr uint32_t kIMp = 0, kIUl = 65536, kIX = 98304, kIW = 131072, kIT = 163840, kITb = 180224,
                   kITbg = 196608;
constexpr uint32_t kItemBytes = 212992;
constexpr uint32_t kCkBytes = 65536;

// x = hi + lo for 8 values: hi the bf16 rounding, lo the bf16 rounding of the rest.
__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
    float h[8], l[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        h[u] = __bfloat162float(__float2bfloat16_rn(x[u]));
        l[u] = x[u] - h[u];
    }
    hi = pack_bf16x8(h);
    lo = pack_bf16x8(l);
}

__device__ __forceinline__ void unpack8(uint4 w, float *x) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        x[2 * u] = __uint_as_float(ws[u] << 16);
        x[2 * u + 1] = __uint_as_float(ws[u] & 0xffff0000u);
    }
}

// 8 values of a split pair (hi + lo) from shared memory.
__device__ __forceinline__ void ld_pair8(uint32_t hi_addr, uint32_t lo_addr, float *x) {
    float h[8], l[8];
    unpack8(ld_shared_v4(hi_addr), h);
    unpack8(ld_shared_v4(lo_addr), l);
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = h[u] + l[u];
}

// Operand descriptors for k-step s (16 elements of K) of a tile in the
// 128-byte swizzle.  K-major: the tile's rows are M (or N), K runs along the
// row; 64 K-elements per atom.  MN-major: the tile's rows are K, M (or N)
// runs along the row, 64 per atom, atoms `atom` bytes apart; a k-step is 16
// rows (2048 bytes).
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, uint32_t atom, int s) {
    return smem_desc(tile + uint32_t(s >> 2) * atom + uint32_t(s & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mdesc(uint32_t tile, uint32_t atom, int s) {
    return smem_desc(tile + uint32_t(s) * 2048, atom, 1024);
}

// One operand of a product: tile address, byte distance between its value
// and residual parts (0: a single exact bf16 part), atom stride, K- or MN-major.
struct Opd {
    uint32_t tile, part, atom;
    bool mn;
    __device__ __forceinline__ uint64_t desc(int s, int p) const {
        const uint32_t t = tile + uint32_t(p) * part;
        return mn ? mdesc(t, atom, s) : kdesc(t, atom, s);
    }
};

// Start-address step (16-byte units, the descriptor's low field) of k-step s.
__device__ __forceinline__ uint64_t kstep(const Opd &X, int s) {
    return X.mn ? uint64_t(s) * 128u : uint64_t((uint32_t(s >> 2) * X.atom + uint32_t(s & 3) * 32) >> 4);
}

// D (+)= A B over nk k-steps, split parts combined as hi hi + hi lo + lo hi
// (or hi, lo against an exact operand).  One thread issues; each part's
// descriptor is built once and stepped through K by its start address.
__device__ __forceinline__ void product(uint32_t d, const Opd &A, const Opd &B, int M, int N, int nk, bool neg,
                                        bool accumulate) {
    const uint32_t id = idesc_bf16(M, N, A.mn, B.mn, neg);
    const uint64_t a0 = A.desc(0, 0), a1 = A.desc(0, 1), b0 = B.desc(0, 0), b1 = B.desc(0, 1);
    const bool pa = A.part != 0, pb = B.part != 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        if (s >= nk) break;
        const uint64_t da = kstep(A, s), db = kstep(B, s);
        mma_bf16(d, a0 + da, b0 + db, id, (accumulate || s > 0) ? 1u : 0u);
        if (pb) mma_bf16(d, a0 + da, b1 + db, id, 1);
        if (pa) mma_bf16(d, a1 + da, b0 + db, id, 1);
    }
}

// Tensor-memory address of this warp's lane quarter at column `col`.  For an
// M = 64 accumulator, row r sits in lane (r % 16) + 32 (r / 16): lanes 0-15 of
// each quarter hold rows 16 q .. 16 q + 15.
__device__ __forceinline__ uint32_t tlane(uint32_t tmem, int warp, int col) {
    return tmem + (uint32_t((warp & 3) * 32) << 16) + uint32_t(col);
}

// Shared -> global bulk copy (one thread; completion through the bulk group).
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

// Adds to the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Reads of an M = 64 accumulator with every lane busy (16x32bx2 shape):
// threads 0-15 read lanes 0-15 of the warp's quarter (rows 16 (warp % 4) +
// lane) at column `col`, threads 16-31 the same rows at `col + 32`.
__device__ __forceinline__ void tmem_ld_h16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_h32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Column sums over the 16 lanes of each half-warp, 16 values per lane: four
// halving exchanges leave lane l with the sum of column l % 16; added into
// dst[l % 16] (dst: this half-warp's columns).
__device__ __forceinline__ void colsum16_add(float (&x)[16], float *dst, int lane) {
#pragma unroll
    for (int n = 8, bit = 8; n >= 1; n >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int m = 0; m < n; ++m) {
            const float send = up ? x[m] : x[m + n];
            const float keep = up ? x[m + n] : x[m];
            x[m] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    atomicAdd(dst + (lane & 15), x[0]);
}

// Waits on an mbarrier phase with every thread polling (bounded); true on
// success for the whole block.
__device__ __forceinline__ bool block_wait(uint32_t bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return !__syncthreads_or(!ok);
}

// Records a device-side timeout.
__device__ __forceinline__ void record_abort(WsHeader *hdr, int code) {
    hdr->bad_index = code;
    atomicExch(&hdr->status, int(GDN_ERR_DEVICE_CHECK));
}

// The chunk's floored log-decays (0 past the end) and beta (0 past the end)
// into g[64], b[64]; then G (inclusive prefix sums), gamma, lambda and beta
// gamma.  Threads 0-63 load, warp 0 scans; ends with a block barrier.
struct ChunkVec {
    float *G, *gam, *lam, *beta, *bg;
};
__device__ __forceinline__ void chunk_vectors(const PrefillArgs &a, int t0, int L, int h, const ChunkVec &cv,
                                              int tid) {
    if (tid < 64) {
        float g = 0.f, b = 0.f;
        if (tid < L) {
            const size_t o = size_t(t0 + tid) * a.hv + h;
            g = fmaxf(a.g[o], kGFloor);
            b = a.beta[o];
        }
        cv.G[tid] = g;
        cv.beta[tid] = b;
    }
    __syncthreads();
    if (tid < 32) {
        const float g0 = cv.G[2 * tid], g1 = cv.G[2 * tid + 1];
        float s = g0 + g1;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, m);
            if (tid >= m) s += y;
        }
        const float G1 = s, G0 = s - g1;
        const float Gl = __shfl_sync(0xffffffffu, s, 31);  // G_63 = G_(L-1): rows past the end carry g = 0
        cv.G[2 * tid] = G0;
        cv.G[2 * tid + 1] = G1;
        const float e0 = __expf(G0), e1 = __expf(G1);
        cv.gam[2 * tid] = e0;
        cv.gam[2 * tid + 1] = e1;
        cv.lam[2 * tid] = __expf(Gl - G0);
        cv.lam[2 * tid + 1] = __expf(Gl - G1);
        cv.bg[2 * tid] = cv.beta[2 * tid] * e0;
        cv.bg[2 * tid + 1] = cv.beta[2 * tid + 1] * e1;
    }
    __syncthreads();
}

// ===========================================================================
// 1. Factors.  256 threads, one CTA per SM, over all items.
// ===========================================================================
constexpr uint32_t kAK = 0, kAQ = 16384, kAV = 32768;  // K, Q, V tiles [64][128] (TMA)
constexpr uint32_t kAP = 49152;                          // P pair [64][64]
constexpr uint32_t kATbg = 65536, kATb = 81920;          // T diag(beta gamma), T diag(beta) pairs
constexpr uint32_t kAW = 98304, kAWl = 131072;           // W, W diag(lambda) pairs [64][128]
constexpr uint32_t kAAf = 163840;                        // A, inverted into T: 64 x kLdA fp32
constexpr uint32_t kAY = kAAf + 64 * kLdA * 4;           // 32 x kLdY fp32
constexpr uint32_t kAVec = kAY + 32 * kLdY * 4;          // G, gamma, lambda, beta, beta gamma
constexpr uint32_t kABar = kAVec + 5 * 64 * 4;           // load and product mbarriers, tensor-memory slot
constexpr uint32_t kAT = (kABar + 64 + 1023) & ~1023u;   // T pair, staged for its copy to the item
constexpr uint32_t kASmem = kAT + 16384 + 1024;
// The item's tiles leave through shared memory as bulk copies: T, T diag(beta), T diag(beta gamma)
// from their slots; W from kAW and U~ diag(lambda) from kATbg (its 32 KB span kATbg and kATb);
// M' from kAW (with kAWl) and X from kATbg once the products that read those slots are done.
static_assert(kASmem <= 232448, "factor kernel shared memory");
// tensor memory (512 columns): K K^T 0, Q K^T 64 (M = 64); then W 128, U~ 256
// (M = 64, 128 columns); then (W diag(lambda))^T K 384 (M = 128) and P W 0.
constexpr int kTKK = 0, kTQK = 64, kTW = 128, kTU = 256, kTM = 384, kTPW = 0;

__global__ void __launch_bounds__(kThr, 1)
bwd_factor_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tq,
                  const __grid_constant__ CUtensorMap tv, unsigned char *items) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *Af = reinterpret_cast<float *>(smem + kAAf);
    float *Yb = reinterpret_cast<float *>(smem + kAY);
    float *vec = reinterpret_cast<float *>(smem + kAVec);
    const ChunkVec cv{vec, vec + 64, vec + 128, vec + 192, vec + 256};
    const uint32_t lbar = sb + kABar, mbar = sb + kABar + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kABar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader *hdr = a.sched.hdr;
    if (tid == 0) {
        mbar_init(lbar, 1);
        mbar_init(mbar, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();
    bool aborted = hdr->status != GDN_OK;
    const int hv = a.hv, group = hv / a.hk;
    const int64_t total = aborted ? 0 : int64_t(hdr->total_chunks) * hv;
    uint32_t lph = 0, mph = 0;
    const int q4 = warp & 3, half = warp >> 2;
    // M = 64 accumulators, read with every lane busy: row rr; of a 64-column one the
    // 16 columns cb .. cb + 15, of a 128-column one the 32 columns 64 half + cb2 ..
    const int rr = 16 * q4 + (lane & 15);
    const int cb = 16 * half + 32 * (lane >> 4), cb2 = 32 * (lane >> 4);

    // an item's (value head, q/k head, first token, tokens)
    auto decode = [&](int64_t item, int &h, int &hq, int &t0, int &L) {
        const int gc = int(item / hv);
        h = int(item - int64_t(gc) * hv);
        hq = h / group;
        const int n = chunk_sequence(a.sched.chunk_base, a.num_seqs, gc);
        const int c0 = gc - a.sched.chunk_base[n];
        t0 = a.sched.start[n] + 64 * c0;
        L = min(64, a.sched.len[n] - 64 * c0);
    };
    // K and V of an item (once the previous item's products are done), then Q (after its last reader)
    auto load_kv = [&](int h, int hq, int t0) {
        mbar_expect_tx(lbar, 2 * 16384);
        tma_load_3d(sb + kAK, &tk, 0, hq, t0, lbar);
        tma_load_3d(sb + kAK + 8192, &tk, 64, hq, t0, lbar);
        tma_load_3d(sb + kAV, &tv, 0, h, t0, lbar);
        tma_load_3d(sb + kAV + 8192, &tv, 64, h, t0, lbar);
    };
    auto load_q = [&](int hq, int t0) {
        mbar_arrive_expect_tx(lbar, 16384);
        tma_load_3d(sb + kAQ, &tq, 0, hq, t0, lbar);
        tma_load_3d(sb + kAQ + 8192, &tq, 64, hq, t0, lbar);
    };
    bool pending = false;  // a load phase is open (thread 0)
    if (tid == 0 && total > int64_t(blockIdx.x)) {
        int h, hq, t0, L;
        decode(blockIdx.x, h, hq, t0, L);
        load_kv(h, hq, t0);
        load_q(hq, t0);
        pending = true;
    }

    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
        int h, hq, t0, L;
        decode(item, h, hq, t0, L);
        unsigned char *it = items + size_t(item) * kItemBytes;
        const int64_t next = item + gridDim.x;
        const bool has_next = next < total;
        int nh = 0, nhq = 0, nt0 = 0, nL = 0;
        if (tid == 0 && has_next) decode(next, nh, nhq, nt0, nL);

        chunk_vectors(a, t0, L, h, cv, tid);
        if (!block_wait(lbar, lph)) { aborted = true; break; }
        lph ^= 1u;
        if (tid == 0) pending = false;
        // K K^T and Q K^T (exact bf16 operands)
        if (tid == 0) {
            tc_fence_after();
            const Opd K{sb + kAK, 0, 8192, false}, Q{sb + kAQ, 0, 8192, false};
            product(tmem + kTKK, K, K, 64, 64, 8, false, false);
            product(tmem + kTQK, Q, K, 64, 64, 8, false, false);
            mma_commit(mbar);
        }
        if (!block_wait(mbar, mph)) { aborted = true; break; }
        mph ^= 1u;
        tc_fence_after();
        // A (fp32, strictly lower) from K K^T; P = Q K^T (.) Gamma (lower, rows < L) as a split pair
        {
            float v[16];
            tmem_ld_h16(tlane(tmem, warp, kTKK + 16 * half), v);
            tmem_wait_ld();
            const float br = cv.beta[rr], Gr = cv.G[rr];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = cb + 4 * q + u;
                    x[u] = j < rr ? br * __expf(Gr - cv.G[j]) * v[4 * q + u] : 0.f;
                }
                *reinterpret_cast<float4 *>(Af + rr * kLdA + cb + 4 * q) = make_float4(x[0], x[1], x[2], x[3]);
            }
            tmem_ld_h16(tlane(tmem, warp, kTQK + 16 * half), v);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = cb + u;
                v[u] = (j <= rr && rr < L) ? __expf(Gr - cv.G[j]) * v[u] : 0.f;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint4 hi, lo;
                split8(v + 8 * c, hi, lo);
                st_shared_v4(sb + kAP + sw128_offset(rr, cb / 8 + c), hi);
                st_shared_v4(sb + kAP + 8192 + sw128_offset(rr, cb / 8 + c), lo);
            }
        }
        tc_fence_before();
        __syncthreads();
        invert_in_place<true>(Af, Yb, tid);
        // T, T diag(beta), T diag(beta gamma) as split pairs to shared memory; copied to the item
        // while W and U~ run
        const int tr = tid >> 2, tcq = (tid & 3) * 16;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float t[8], tb[8], tbg[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = tcq + 8 * c + u;
                t[u] = Af[tr * kLdA + j];
                tb[u] = t[u] * cv.beta[j];
                tbg[u] = t[u] * cv.bg[j];
            }
            const uint32_t off = sw128_offset(tr, tcq / 8 + c);
            uint4 hi, lo;
            split8(t, hi, lo);
            st_shared_v4(sb + kAT + off, hi);
            st_shared_v4(sb + kAT + 8192 + off, lo);
            split8(tb, hi, lo);
            st_shared_v4(sb + kATb + off, hi);
            st_shared_v4(sb + kATb + 8192 + off, lo);
            split8(tbg, hi, lo);
            st_shared_v4(sb + kATbg + off, hi);
            st_shared_v4(sb + kATbg + 8192 + off, lo);
        }
        fence_proxy_async_shared();
        __syncthreads();
        // W = (T diag(beta gamma)) K and U~ = (T diag(beta)) V   (M = 64, N = 128, K = 64)
        if (tid == 0) {
            bulk_store(it + kIT, sb + kAT, 16384);
            bulk_store(it + kITb, sb + kATb, 16384);
            bulk_store(it + kITbg, sb + kATbg, 16384);
            bulk_commit();
            tc_fence_after();
            const Opd Tbg{sb + kATbg, 8192, 8192, false}, Tb{sb + kATb, 8192, 8192, false};
            const Opd Kmn{sb + kAK, 0, 8192, true}, Vmn{sb + kAV, 0, 8192, true};
            product(tmem + kTW, Tbg, Kmn, 64, 128, 4, false, false);
            product(tmem + kTU, Tb, Vmn, 64, 128, 4, false, false);
            mma_commit(mbar);
        }
        if (!block_wait(mbar, mph)) { aborted = true; break; }
        mph ^= 1u;
        tc_fence_after();
        // W, W diag(lambda) and U~ diag(lambda) as split pairs to shared memory (columns 64 half +
        // cb2 ..: atom `half`); W and U~ diag(lambda) copied to the item while the last products run
        if (tid == 0) bulk_wait_read();  // the T copies have read kATb, kATbg
        __syncthreads();
        {
            const uint32_t watom = uint32_t(half) * 8192;
            const float lr = cv.lam[rr];
            float v[32];
            tmem_ld_h32(tlane(tmem, warp, kTW + 64 * half), v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = watom + sw128_offset(rr, cb2 / 8 + c);
                float wl[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) wl[u] = lr * v[8 * c + u];
                uint4 hi, lo;
                split8(v + 8 * c, hi, lo);
                st_shared_v4(sb + kAW + off, hi);
                st_shared_v4(sb + kAW + 16384 + off, lo);
                split8(wl, hi, lo);
                st_shared_v4(sb + kAWl + off, hi);
                st_shared_v4(sb + kAWl + 16384 + off, lo);
            }
            tmem_ld_h32(tlane(tmem, warp, kTU + 64 * half), v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = watom + sw128_offset(rr, cb2 / 8 + c);
                float ul[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) ul[u] = lr * v[8 * c + u];
                uint4 hi, lo;
                split8(ul, hi, lo);
                st_shared_v4(sb + kATbg + off, hi);
                st_shared_v4(sb + kATbg + 16384 + off, lo);
            }
        }
        fence_proxy_async_shared();
        tc_fence_before();
        __syncthreads();
        // (W diag(lambda))^T K (M = 128, N = 128, K = 64) and P W (M = 64, N = 128, K = 64)
        if (tid == 0) {
            bulk_store(it + kIW, sb + kAW, 32768);
            bulk_store(it + kIUl, sb + kATbg, 32768);
            bulk_commit();
            tc_fence_after();
            const Opd Wl{sb + kAWl, 16384, 8192, true}, Kmn{sb + kAK, 0, 8192, true};
            const Opd P{sb + kAP, 8192, 8192, false}, Wmn{sb + kAW, 16384, 8192, true};
            product(tmem + kTM, Wl, Kmn, 128, 128, 4, false, false);
            product(tmem + kTPW, P, Wmn, 64, 128, 4, false, false);
            mma_commit(mbar);
        }
        if (!block_wait(mbar, mph)) { aborted = true; break; }
        mph ^= 1u;
        tc_fence_after();
        if (tid == 0 && has_next) {  // K and V are free (their last products are done)
            load_kv(nh, nhq, nt0);
            pending = true;
        }
        if (tid == 0) bulk_wait_read();  // the W and U~ diag(lambda) copies have read kAW, kATbg
        __syncthreads();
        // M' = gamma_L I - (W diag(lambda))^T K: row y = 32 (warp % 4) + lane, 64 columns;
        // as a pair in kAW .. (value 32 KB, then residual 32 KB over kAWl)
        {
            const int y = 32 * q4 + lane;
            const float gl = cv.gam[63];
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                float v[32];
                tmem_ld32(tmem + (uint32_t(32 * q4) << 16) + uint32_t(kTM + 64 * half + 32 * p), v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float x[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int xcol = 64 * half + 32 * p + 8 * c + u;
                        x[u] = (xcol == y ? gl : 0.f) - v[8 * c + u];
                    }
                    uint4 hi, lo;
                    split8(x, hi, lo);
                    const uint32_t off = uint32_t(half) * 16384 + sw128_offset(y, 4 * p + c);
                    st_shared_v4(sb + kAW + off, hi);
                    st_shared_v4(sb + kAW + 32768 + off, lo);
                }
            }
        }
        // X = diag(gamma) Q - P W (rows < L), as a pair in kATbg ..
        {
            const uint32_t atom = uint32_t(half) * 8192;
            float v[32];
            tmem_ld_h32(tlane(tmem, warp, kTPW + 64 * half), v);
            tmem_wait_ld();
            const float gr = rr < L ? cv.gam[rr] : 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = atom + sw128_offset(rr, cb2 / 8 + c);
                float qv[8], x[8];
                unpack8(ld_shared_v4(sb + kAQ + off), qv);
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = rr < L ? fmaf(gr, qv[u], -v[8 * c + u]) : 0.f;
                uint4 hi, lo;
                split8(x, hi, lo);
                st_shared_v4(sb + kATbg + off, hi);
                st_shared_v4(sb + kATbg + 16384 + off, lo);
            }
        }
        fence_proxy_async_shared();
        __syncthreads();
        if (tid == 0) {
            bulk_store(it + kIMp, sb + kAW, 65536);
            bulk_store(it + kIX, sb + kATbg, 32768);
            bulk_commit();
            bulk_wait_read();  // the next item reuses these slots
        }
        fence_proxy_async_shared();
        tc_fence_before();
        __syncthreads();  // tensor memory and shared memory are reused by the next item
        if (tid == 0 && has_next) load_q(nhq, nt0);  // Q's last reader (X) is done
    }
    if (aborted && tid == 0 && total > 0) {
        mma_commit(mbar);
        (void)mbar_wait(mbar, mph);
        if (pending) {  // loads in flight into this CTA's shared memory: let them land
            mbar_arrive(lbar);
            (void)mbar_wait(lbar, lph);
        }
        record_abort(hdr, -6);
    }
    if (tid == 0) bulk_wait_all();  // the item copies have landed
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}


// ===========================================================================
// 2. Chains.  256 threads, one CTA per (sequence, value head, direction):
//    forward  S_{c+1}  = S_c M'_c + (U~ diag(lambda))^T K,    keeps S_c,
//    backward dS_c     = dS_{c+1} M'_c^T + dO^T X_c,          keeps dS_{c+1}.
// The state lives in registers (thread: row 32 (warp % 4) + lane, 64 columns
// of half warp / 4); each chunk it is split into a pair in shared memory
// (the product's A operand, bulk-copied to the checkpoint as is), one
// product of K = 128 + 64 gives the next state in tensor memory.
// ===========================================================================
constexpr uint32_t kCA = 0;        // state pair [128][128]: 2 parts x 2 atoms of 16 KB
constexpr uint32_t kCM = 65536;    // M' pair
constexpr uint32_t kC2 = 131072;   // forward: U~ diag(lambda) pair [64][128]; backward: X pair
constexpr uint32_t kC3 = 163840;   // forward: K [64][128]; backward: dO [64][128] (TMA)
constexpr uint32_t kCBar = 180224;
constexpr uint32_t kCSmem = kCBar + 64 + 1024;
static_assert(kCSmem <= 232448, "chain kernel shared memory");

__global__ void __launch_bounds__(kThr, 1)
bwd_chain_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tdo,
                 const unsigned char *items, unsigned char *ck_s, unsigned char *ck_ds, const float *dS_final,
                 float *dS0_out, float *s_final_out) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    const uint32_t lbar = sb + kCBar, mbar = sb + kCBar + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kCBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader *hdr = a.sched.hdr;
    if (tid == 0) {
        mbar_init(lbar, 1);
        mbar_init(mbar, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();
    const int hv = a.hv, group = hv / a.hk;
    const bool fwd = (blockIdx.x & 1u) == 0;  // even: forward, odd: backward, longest sequences first
    const int u = int(blockIdx.x >> 1);
    bool aborted = hdr->status != GDN_OK;
    const int h = u % hv, hq = h / group;
    // (the tables are read only once the schedule has validated the sequences)
    const int n = aborted ? 0 : a.sched.order[u / hv];
    const int t0 = aborted ? 0 : a.sched.start[n], len = aborted ? 0 : a.sched.len[n];
    const int nch = (len + 63) / 64, cb = aborted ? 0 : a.sched.chunk_base[n];
    const int row = 32 * (warp & 3) + lane, half = warp >> 2;
    const size_t sbase = ((size_t(n) * hv + h) * 128 + row) * 128 + 64 * half;

    // the state's first value: S_0 (forward) or dS_N (backward), zeros for NULL
    float st[64];
    {
        const float *src = aborted ? nullptr : (fwd ? a.s0 : dS_final);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 x = src ? *reinterpret_cast<const float4 *>(src + sbase + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
            st[4 * q] = x.x; st[4 * q + 1] = x.y; st[4 * q + 2] = x.z; st[4 * q + 3] = x.w;
        }
    }
    uint32_t lph = 0, mph = 0;
    for (int k = 0; k < nch && !aborted; ++k) {
        const int c = fwd ? k : nch - 1 - k;
        const size_t item = size_t(cb + c) * hv + h;
        const unsigned char *it = items + item * kItemBytes;
        unsigned char *ck = (fwd ? ck_s : ck_ds) + item * kCkBytes;
        if (tid == 0) {
            // the chunk's operands (the previous product, their last reader, has completed)
            mbar_arrive_expect_tx(lbar, 65536 + 32768 + 16384);
            for (int q = 0; q < 4; ++q) bulk_load(sb + kCM + 16384 * q, it + kIMp + 16384 * q, 16384, lbar);
            const uint32_t src2 = fwd ? kIUl : kIX;
            for (int q = 0; q < 2; ++q) bulk_load(sb + kC2 + 16384 * q, it + src2 + 16384 * q, 16384, lbar);
            if (fwd) {
                tma_load_3d(sb + kC3, &tk, 0, hq, t0 + 64 * c, lbar);
                tma_load_3d(sb + kC3 + 8192, &tk, 64, hq, t0 + 64 * c, lbar);
            } else {
                tma_load_3d(sb + kC3, &tdo, 0, h, t0 + 64 * c, lbar);
                tma_load_3d(sb + kC3 + 8192, &tdo, 64, h, t0 + 64 * c, lbar);
            }
            bulk_wait_read();  // the previous checkpoint copy has read the state pair
        }
        __syncthreads();
        // the state as a split pair: row `row`, columns 64 half .. + 63 (atom `half`)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint4 hi, lo;
            split8(st + 8 * ch, hi, lo);
            const uint32_t off = uint32_t(half) * 16384 + sw128_offset(row, ch);
            st_shared_v4(sb + kCA + off, hi);
            st_shared_v4(sb + kCA + 32768 + off, lo);
        }
        fence_proxy_async_shared();
        __syncthreads();
        if (tid == 0) {
            for (int q = 0; q < 4; ++q)
                asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                             ::"l"(ck + 16384 * q), "r"(sb + kCA + 16384 * q), "r"(16384) : "memory");
            bulk_commit();
        }
        if (!block_wait(lbar, lph)) { aborted = true; break; }
        lph ^= 1u;
        if (tid == 0) {
            tc_fence_after();
            const Opd S{sb + kCA, 32768, 16384, false};
            const Opd M{sb + kCM, 32768, 16384, fwd};  // forward S M': MN-major; backward dS M'^T: K-major
            product(tmem, S, M, 128, 128, 8, false, false);
            if (fwd) {
                const Opd Ul{sb + kC2, 16384, 8192, true}, K{sb + kC3, 0, 8192, true};
                product(tmem, Ul, K, 128, 128, 4, false, true);
            } else {
                const Opd dO{sb + kC3, 0, 8192, true}, X{sb + kC2, 16384, 8192, true};
                product(tmem, dO, X, 128, 128, 4, false, true);
            }
            mma_commit(mbar);
        }
        if (!block_wait(mbar, mph)) { aborted = true; break; }
        mph ^= 1u;
        tc_fence_after();
        {
            float v[32];
            tmem_ld32(tmem + (uint32_t(32 * (warp & 3)) << 16) + uint32_t(64 * half), v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) st[q] = v[q];
            tmem_ld32(tmem + (uint32_t(32 * (warp & 3)) << 16) + uint32_t(64 * half + 32), v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) st[32 + q] = v[q];
        }
        tc_fence_before();
    }
    if (!aborted) {
        float *dst = fwd ? s_final_out : dS0_out;
        if (dst)
#pragma unroll
            for (int q = 0; q < 16; ++q)
                *reinterpret_cast<float4 *>(dst + sbase + 4 * q) =
                    make_float4(st[4 * q], st[4 * q + 1], st[4 * q + 2], st[4 * q + 3]);
    }
    if (tid == 0) {
        bulk_wait_all();
        if (aborted) {
            mma_commit(mbar);
            (void)mbar_wait(mbar, mph);
            record_abort(hdr, -7);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ===========================================================================
// 3. Gradients.  256 threads, one CTA per SM, over groups of units: a
//    (chunk, q/k head) with its value heads' two halves of d_v in turn.
//    Products are M = 64 (rows: tokens or the half's d_v rows), read with
//    every lane busy: threads 0-15 and 16-31 of warp w take rows 16 (w % 4)
//    .. + 15 at columns 32 apart, warp group w / 4 its own 16 (or 64) columns.
// ===========================================================================
constexpr uint32_t kDK = 0, kDQ = 16384;        // K, Q [64][128] (TMA)
constexpr uint32_t kDV = 32768, kDO = 40960;    // V, dO: the half's 64 columns [64][64] (TMA)
constexpr uint32_t kDT = 49152, kDTb = 65536, kDTbg = 81920;  // T, T diag(beta), T diag(beta gamma) pairs
constexpr uint32_t kDS0 = 98304;   // S_c half pair [64][128]
constexpr uint32_t kDdS = 131072;  // dS_{c+1} half pair; then dU^T (+0) and dP (.) Gamma (+16384) pairs
constexpr uint32_t kDR1 = 163840;  // W pair; then U^T (+0) and (U diag(lambda))^T (+16384); then dW pair
constexpr uint32_t kDgO = 196608;  // diag(gamma) dO pair [64][64]; then P, dT, M = dT T^T and dKK in turn
// The next unit's inputs are loaded while this one finishes, each into its
// buffer once the buffer's last reader has completed: after the third group
// of products S_c, dS, Q, V, dO and T diag(beta); after the fourth W and
// T diag(beta gamma); after the sixth T; after the seventh K.
constexpr uint32_t kDVec = 212992;
constexpr uint32_t kDBar = kDVec + 4096;
constexpr uint32_t kDSmem = kDBar + 64 + 1024;
static_assert(kDSmem <= 232448, "gradient kernel shared memory");
// vectors (64 floats each) after G, gamma, lambda, beta, beta gamma
enum { kVll = 5, kVgg, kVrs, kVcs, kVbg, kVyv, kVab, kVG2, kVNum };  // + 2 scalars at kVNum * 64
// tensor memory (512 columns): dK 0; dW 128 (Q K^T 192 before it, dT1 192 and K K^T 128 after it);
// dQ 256; scratch A 384 and B 448 (64 columns each)
constexpr int kTdK = 0, kTdW = 128, kTKK2 = 128, kTQK2 = 192, kTdT1 = 192, kTdQ = 256, kTSA = 384, kTSB = 448;

__global__ void __launch_bounds__(kThr, 1)
bwd_grad_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tq,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                const unsigned char *items, const unsigned char *ck_s, const unsigned char *ck_ds, float *dq,
                float *dk, float *dv, float *dg, float *dbeta) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);
    float *vec = reinterpret_cast<float *>(smem + kDVec);
    const ChunkVec cv{vec, vec + 64, vec + 128, vec + 192, vec + 256};
    float *dll = vec + 64 * kVll, *dgg = vec + 64 * kVgg, *rs = vec + 64 * kVrs, *cs = vec + 64 * kVcs;
    float *dbgv = vec + 64 * kVbg, *dyv = vec + 64 * kVyv, *dab = vec + 64 * kVab, *dG = vec + 64 * kVG2;
    float *scal = vec + 64 * kVNum;  // [0] <dS, S_c> over the half, [1] sum of dlambda lambda
    const uint32_t lbar = sb + kDBar, mbar = sb + kDBar + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kDBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader *hdr = a.sched.hdr;
    if (tid == 0) {
        mbar_init(lbar, 1);
        mbar_init(mbar, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_wait();
    bool aborted = hdr->status != GDN_OK;
    const int hv = a.hv, hk = a.hk, group = hv / hk;
    // Units come in groups of one (chunk, q/k head): its value heads' two halves of d_v in turn,
    // so that dq and dk add up in registers and are written once, and K and Q (per group) and
    // T, T diag(beta), T diag(beta gamma) (per value head) are loaded once.
    const int upg = 2 * group;  // units per group
    const int64_t groups = aborted ? 0 : int64_t(hdr->total_chunks) * hk;
    const int64_t my_units = groups > int64_t(blockIdx.x) ? ((groups - 1 - blockIdx.x) / gridDim.x + 1) * upg : 0;
    uint32_t lph = 0, mph = 0;
    // accumulator reads: row rr of an M = 64 accumulator; of a 64-column one the 16
    // columns cb .. cb + 15, of a 128-column one the 32 columns cb2 .. cb2 + 31
    // (warp group wg = warp / 4 takes columns 64 wg ..)
    const int wg = warp >> 2, rr = 16 * (warp & 3) + (lane & 15);
    const int cb = 16 * wg + 32 * (lane >> 4), cb2 = 32 * (lane >> 4);

    // every thread waits for the group of products last committed
    auto group_wait = [&]() -> bool {
        const bool ok = block_wait(mbar, mph);
        mph ^= 1u;
        tc_fence_after();
        return ok;
    };
    auto group_done = [&]() -> bool {
        if (tid == 0) mma_commit(mbar);
        return group_wait();
    };
    // the staged operands are visible to the tensor cores, the accumulator reads are done
    auto stage_done = [&]() {
        fence_proxy_async_shared();
        tc_fence_before();
        __syncthreads();
    };
    // 16 values (row r, columns c0 .. c0 + 15 of a 64-column tile) as a split pair
    auto stage16 = [&](uint32_t tile, int r, int c0, const float *x) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint4 hi, lo;
            split8(x + 8 * c, hi, lo);
            const uint32_t off = sw128_offset(r, c0 / 8 + c);
            st_shared_v4(tile + off, hi);
            st_shared_v4(tile + 8192 + off, lo);
        }
    };

    // the k-th unit of this CTA
    struct Unit {
        int sh, i0, h, hq, t0, L, pos;
        const unsigned char *it, *cs0, *cds;
    };
    auto decode = [&](int64_t k) {
        Unit U;
        const int64_t gi = blockIdx.x + (k / upg) * gridDim.x;
        U.pos = int(k % upg);
        U.sh = U.pos & 1;
        U.i0 = 64 * U.sh;
        const int gc = int(gi / hk);
        U.hq = int(gi - int64_t(gc) * hk);
        U.h = U.hq * group + (U.pos >> 1);
        const int64_t item = int64_t(gc) * hv + U.h;
        const int n = chunk_sequence(a.sched.chunk_base, a.num_seqs, gc);
        const int c0 = gc - a.sched.chunk_base[n];
        U.t0 = a.sched.start[n] + 64 * c0;
        U.L = min(64, a.sched.len[n] - 64 * c0);
        U.it = items + size_t(item) * kItemBytes;
        U.cs0 = ck_s + size_t(item) * kCkBytes;
        U.cds = ck_ds + size_t(item) * kCkBytes;
        return U;
    };
    // the unit's inputs, in the four sets the prefetch uses (thread 0; set 3 arrives).  Q and
    // K only for a group's first unit, the three T tiles only for a value head's first half.
    auto load_set = [&](const Unit &U, int set) {
        const bool new_group = U.pos == 0, new_head = U.sh == 0;
        if (set == 0) {
            mbar_expect_tx(lbar, 2 * 32768 + 2 * 8192 + (new_group ? 16384 : 0) + (new_head ? 16384 : 0));
            for (int q = 0; q < 4; ++q) {  // rows i0 .. i0 + 63 of each atom of the two checkpoint pairs
                const uint32_t src = uint32_t(q) * 16384 + uint32_t(U.sh) * 8192, dst = uint32_t(q) * 8192;
                bulk_load(sb + kDS0 + dst, U.cs0 + src, 8192, lbar);
                bulk_load(sb + kDdS + dst, U.cds + src, 8192, lbar);
            }
            if (new_group) {
                tma_load_3d(sb + kDQ, &tq, 0, U.hq, U.t0, lbar);
                tma_load_3d(sb + kDQ + 8192, &tq, 64, U.hq, U.t0, lbar);
            }
            tma_load_3d(sb + kDV, &tv, U.i0, U.h, U.t0, lbar);
            tma_load_3d(sb + kDO, &tdo, U.i0, U.h, U.t0, lbar);
            if (new_head) bulk_load(sb + kDTb, U.it + kITb, 16384, lbar);
        } else if (set == 1) {
            mbar_expect_tx(lbar, 32768 + (new_head ? 16384 : 0));
            bulk_load(sb + kDR1, U.it + kIW, 32768, lbar);
            if (new_head) bulk_load(sb + kDTbg, U.it + kITbg, 16384, lbar);
        } else if (set == 2) {
            if (new_head) {
                mbar_expect_tx(lbar, 16384);
                bulk_load(sb + kDT, U.it + kIT, 16384, lbar);
            }
        } else {
            mbar_arrive_expect_tx(lbar, new_group ? 16384 : 0);
            if (new_group) {
                tma_load_3d(sb + kDK, &tk, 0, U.hq, U.t0, lbar);
                tma_load_3d(sb + kDK + 8192, &tk, 64, U.hq, U.t0, lbar);
            }
        }
    };
    bool pending = false;  // a load phase is open (thread 0)
    if (tid == 0 && my_units > 0) {
        const Unit U = decode(0);
        for (int set = 0; set < 4; ++set) load_set(U, set);
        pending = true;
    }
    float accq[32], acck[32];  // this thread's 32 columns of dq and dk, summed over the group

    for (int64_t k = 0; k < my_units; ++k) {
        const Unit U = decode(k);
        const int i0 = U.i0, h = U.h, hq = U.hq, t0 = U.t0, L = U.L;
        const bool has_next = k + 1 < my_units;
        Unit N{};
        if (tid == 0 && has_next) N = decode(k + 1);
        if (U.pos == 0) {
#pragma unroll
            for (int q = 0; q < 32; ++q) accq[q] = acck[q] = 0.f;
        }
        if (tid < 64)
            for (int v = kVll; v < kVNum; ++v) vec[64 * v + tid] = 0.f;
        if (tid < 2) scal[tid] = 0.f;
        chunk_vectors(a, t0, L, h, cv, tid);
        if (!block_wait(lbar, lph)) { aborted = true; break; }
        lph ^= 1u;
        if (tid == 0) pending = false;
        // diag(gamma) dO (rows < L) as a split pair
        for (int e = tid; e < 64 * 8; e += kThr) {
            const int r = e >> 3, ch = e & 7;
            const uint32_t off = sw128_offset(r, ch);
            float x[8];
            unpack8(ld_shared_v4(sb + kDO + off), x);
            const float gr = r < L ? cv.gam[r] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] *= gr;
            uint4 hi, lo;
            split8(x, hi, lo);
            st_shared_v4(sb + kDgO + off, hi);
            st_shared_v4(sb + kDgO + 8192 + off, lo);
        }
        stage_done();
        // ---- G1: U^T, Z^T = dS K^T, Q K^T, dQ <- diag(gamma) dO S_c
        if (tid == 0) {
            tc_fence_after();
            const Opd Vmn{sb + kDV, 0, 8192, true}, Tb{sb + kDTb, 8192, 8192, false};
            const Opd S0{sb + kDS0, 16384, 8192, false}, W{sb + kDR1, 16384, 8192, false};
            const Opd dS{sb + kDdS, 16384, 8192, false}, K{sb + kDK, 0, 8192, false}, Q{sb + kDQ, 0, 8192, false};
            const Opd gO{sb + kDgO, 8192, 8192, false}, S0mn{sb + kDS0, 16384, 8192, true};
            product(tmem + kTSA, Vmn, Tb, 64, 64, 4, false, false);
            product(tmem + kTSA, S0, W, 64, 64, 8, true, true);
            product(tmem + kTSB, dS, K, 64, 64, 8, false, false);
            product(tmem + kTQK2, Q, K, 64, 64, 8, false, false);
            product(tmem + kTdQ, gO, S0mn, 64, 128, 4, false, false);
        }
        if (!group_done()) { aborted = true; break; }
        // ---- E1.  Every 64-column accumulator is read by all eight warps, 16 columns a
        // thread (columns cb .. cb + 15 of row rr); 128-column ones 32 a thread (cb2 ..).
        float zl[16];  // lambda_j Z_ij, kept for dU^T
        float pr[16];  // U_ij lambda_j Z_ij, for dlambda lambda
        {
            float u[16], ul[16];
            tmem_ld_h16(tlane(tmem, warp, kTSA + 16 * wg), u);
            tmem_ld_h16(tlane(tmem, warp, kTSB + 16 * wg), zl);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = cb + q;
                const float lj = j < L ? cv.lam[j] : 0.f;
                zl[q] *= lj;
                pr[q] = u[q] * zl[q];
                ul[q] = lj * u[q];
            }
            stage16(sb + kDR1, rr, cb, u);
            stage16(sb + kDR1 + 16384, rr, cb, ul);
            // P = Q K^T (.) Gamma (lower, rows < L)
            tmem_ld_h16(tlane(tmem, warp, kTQK2 + 16 * wg), u);
            tmem_wait_ld();
            const float Gr = cv.G[rr];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = cb + q;
                u[q] = (j <= rr && rr < L) ? __expf(Gr - cv.G[j]) * u[q] : 0.f;
            }
            stage16(sb + kDgO, rr, cb, u);
        }
        stage_done();
        // ---- G2: dO^T P, dP = dO U^T, dK = (U diag(lambda)) dS
        if (tid == 0) {
            tc_fence_after();
            const Opd dOmn{sb + kDO, 0, 8192, true}, Pmn{sb + kDgO, 8192, 8192, true};
            const Opd dO{sb + kDO, 0, 8192, false}, Utmn{sb + kDR1, 8192, 8192, true};
            const Opd Ulmn{sb + kDR1 + 16384, 8192, 8192, true}, dSmn{sb + kDdS, 16384, 8192, true};
            product(tmem + kTSB, dOmn, Pmn, 64, 64, 4, false, false);
            product(tmem + kTSA, dO, Utmn, 64, 64, 4, false, false);
            product(tmem + kTdK, Ulmn, dSmn, 64, 128, 4, false, false);
            mma_commit(mbar);
        }
        // (while G2 runs) dlambda lambda column sums; gamma_r dgamma_r; <dS_{c+1}, S_c>
        {
            colsum16_add(pr, dll + cb, lane);
            float y[32], part = 0.f;
            tmem_ld_h32(tlane(tmem, warp, kTdQ + 64 * wg), y);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float qv[8];
                unpack8(ld_shared_v4(sb + kDQ + uint32_t(wg) * 8192 + sw128_offset(rr, cb2 / 8 + c)), qv);
#pragma unroll
                for (int e = 0; e < 8; ++e) part = fmaf(y[8 * c + e], qv[e], part);
            }
            atomicAdd(dgg + rr, part);
            float dot = 0.f;
            for (int e = tid; e < 64 * 16; e += kThr) {
                const int r = e >> 4, a8 = (e >> 3) & 1, ch = e & 7;
                const uint32_t off = uint32_t(a8) * 8192 + sw128_offset(r, ch);
                float x[8], w8[8];
                ld_pair8(sb + kDS0 + off, sb + kDS0 + 16384 + off, x);
                ld_pair8(sb + kDdS + off, sb + kDdS + 16384 + off, w8);
#pragma unroll
                for (int q = 0; q < 8; ++q) dot = fmaf(x[q], w8[q], dot);
            }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, m);
            if (lane == 0) atomicAdd(scal, dot);
        }
        tc_fence_before();
        if (!group_wait()) { aborted = true; break; }
        // ---- E2: dU^T = lambda Z^T + dO^T P (columns < L); dP (.) Gamma and its dGamma sums
        float e2[16], rsum = 0.f;
        {
            float x[16];
            tmem_ld_h16(tlane(tmem, warp, kTSB + 16 * wg), x);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) x[q] = cb + q < L ? x[q] + zl[q] : 0.f;
            stage16(sb + kDdS, rr, cb, x);
            tmem_ld_h16(tlane(tmem, warp, kTSA + 16 * wg), x);    // dP: rows r, columns j
            tmem_ld_h16(tlane(tmem, warp, kTQK2 + 16 * wg), e2);  // Q K^T
            tmem_wait_ld();
            const float Gr = cv.G[rr];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = cb + q;
                const bool ok = j <= rr && rr < L;
                const float gm = ok ? __expf(Gr - cv.G[j]) : 0.f;
                x[q] = ok ? x[q] * gm : 0.f;  // dP (.) Gamma
                e2[q] = x[q] * e2[q];         // dGamma_rj Gamma_rj (the P part)
                rsum += e2[q];
            }
            stage16(sb + kDdS + 16384, rr, cb, x);
        }
        stage_done();
        // ---- G3: dQ += (dP (.) Gamma) K, dK += (dP (.) Gamma)^T Q, dW = -dU S_c, dT2 = dU V^T, dV = T''^T dU
        if (tid == 0) {
            tc_fence_after();
            const Opd dPG{sb + kDdS + 16384, 8192, 8192, false}, dPGmn{sb + kDdS + 16384, 8192, 8192, true};
            const Opd Kmn{sb + kDK, 0, 8192, true}, Qmn{sb + kDQ, 0, 8192, true};
            const Opd dUtmn{sb + kDdS, 8192, 8192, true}, dUt{sb + kDdS, 8192, 8192, false};
            const Opd S0mn{sb + kDS0, 16384, 8192, true}, V{sb + kDV, 0, 8192, false};
            const Opd Tbmn{sb + kDTb, 8192, 8192, true};
            product(tmem + kTdQ, dPG, Kmn, 64, 128, 4, false, true);
            product(tmem + kTdK, dPGmn, Qmn, 64, 128, 4, false, true);
            product(tmem + kTdW, dUtmn, S0mn, 64, 128, 4, true, false);
            product(tmem + kTSA, dUtmn, V, 64, 64, 4, false, false);
            product(tmem + kTSB, Tbmn, dUt, 64, 64, 4, false, false);
            mma_commit(mbar);
        }
        atomicAdd(rs + rr, rsum);
        colsum16_add(e2, cs + cb, lane);
        if (!group_wait()) { aborted = true; break; }
        if (tid == 0 && has_next) {
            load_set(N, 0);
            pending = true;
        }
        // ---- E3: dW as a split pair; dv (this half's columns, rows < L) while G4 runs
        {
            float y[32];
            tmem_ld_h32(tlane(tmem, warp, kTdW + 64 * wg), y);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 hi, lo;
                split8(y + 8 * c, hi, lo);
                const uint32_t off = uint32_t(wg) * 8192 + sw128_offset(rr, cb2 / 8 + c);
                st_shared_v4(sb + kDR1 + off, hi);
                st_shared_v4(sb + kDR1 + 16384 + off, lo);
            }
        }
        stage_done();
        // ---- G4: dT1 = dW K^T, dK += (T diag(beta gamma))^T dW
        if (tid == 0) {
            tc_fence_after();
            const Opd dW{sb + kDR1, 16384, 8192, false}, K{sb + kDK, 0, 8192, false};
            const Opd Tbgmn{sb + kDTbg, 8192, 8192, true}, dWmn{sb + kDR1, 16384, 8192, true};
            product(tmem + kTdT1, dW, K, 64, 64, 8, false, false);
            product(tmem + kTdK, Tbgmn, dWmn, 64, 128, 4, false, true);
            mma_commit(mbar);
        }
        {
            float y[32];
            tmem_ld_h32(tlane(tmem, warp, kTdQ + 64 * wg), y);  // dQ: complete after G3
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) accq[q] += y[q];
        }
        {
            float x[16];
            tmem_ld_h16(tlane(tmem, warp, kTSB + 16 * wg), x);
            tmem_wait_ld();
            if (rr < L) {
                float *dst = dv + (size_t(t0 + rr) * hv + h) * 128 + i0 + cb;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(dst + 4 * q) = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            }
        }
        tc_fence_before();
        if (!group_wait()) { aborted = true; break; }
        if (tid == 0 && has_next) load_set(N, 1);
        // ---- E4: dT (lower, rows < L) as a split pair; T (.) dT1 and T (.) dT2 column sums
        {
            float x1[16], x2[16], t[16];
            tmem_ld_h16(tlane(tmem, warp, kTdT1 + 16 * wg), x1);
            tmem_ld_h16(tlane(tmem, warp, kTSA + 16 * wg), x2);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const uint32_t off = sw128_offset(rr, cb / 8 + c);
                ld_pair8(sb + kDT + off, sb + kDT + 8192 + off, t + 8 * c);
            }
            tmem_wait_ld();
            const bool ok = rr < L;
            float p1[16], p2[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = cb + q;
                const float tv = ok ? t[q] : 0.f;
                p1[q] = tv * x1[q];
                p2[q] = tv * x2[q];
                x1[q] = (ok && j <= rr) ? fmaf(cv.bg[j], x1[q], cv.beta[j] * x2[q]) : 0.f;
            }
            stage16(sb + kDgO, rr, cb, x1);
            stage_done();
            // ---- G5: M = dT T^T
            if (tid == 0) {
                tc_fence_after();
                const Opd dT{sb + kDgO, 8192, 8192, false}, T{sb + kDT, 8192, 8192, false};
                product(tmem + kTSA, dT, T, 64, 64, 4, false, false);
                mma_commit(mbar);
            }
            colsum16_add(p1, dbgv + cb, lane);
            colsum16_add(p2, dyv + cb, lane);
        }
        if (!group_wait()) { aborted = true; break; }
        {
            float x[16];
            tmem_ld_h16(tlane(tmem, warp, kTSA + 16 * wg), x);
            tmem_wait_ld();
            stage16(sb + kDgO, rr, cb, x);  // M (dT, its operand, is consumed)
        }
        stage_done();
        // ---- G6: dA = -T^T M, K K^T
        if (tid == 0) {
            tc_fence_after();
            const Opd Tmn{sb + kDT, 8192, 8192, true}, Mmn{sb + kDgO, 8192, 8192, true};
            const Opd K{sb + kDK, 0, 8192, false};
            product(tmem + kTSB, Tmn, Mmn, 64, 64, 4, true, false);
            product(tmem + kTKK2, K, K, 64, 64, 8, false, false);
        }
        if (!group_done()) { aborted = true; break; }
        if (tid == 0 && has_next) load_set(N, 2);
        // ---- E6: from dA (strictly lower, rows < L): dbeta, dGamma, dKK
        {
            float da[16], kk[16];
            tmem_ld_h16(tlane(tmem, warp, kTSB + 16 * wg), da);
            tmem_ld_h16(tlane(tmem, warp, kTKK2 + 16 * wg), kk);
            tmem_wait_ld();
            const int j = rr;
            const float Gj = cv.G[j], bj = cv.beta[j];
            float sab = 0.f, srs = 0.f, e[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int m = cb + q;
                const bool ok = m < j && j < L;
                const float gm = ok ? __expf(Gj - cv.G[m]) : 0.f;
                const float d = ok ? da[q] : 0.f;
                sab = fmaf(d * gm, kk[q], sab);
                e[q] = d * bj * kk[q] * gm;
                srs += e[q];
                da[q] = d * bj * gm;  // dKK
            }
            stage16(sb + kDgO, j, cb, da);  // dKK (M is consumed)
            stage_done();
            // ---- G7: dK += dKK K + dKK^T K
            if (tid == 0) {
                tc_fence_after();
                const Opd dKK{sb + kDgO, 8192, 8192, false}, dKKmn{sb + kDgO, 8192, 8192, true};
                const Opd Kmn{sb + kDK, 0, 8192, true};
                product(tmem + kTdK, dKK, Kmn, 64, 128, 4, false, true);
                product(tmem + kTdK, dKKmn, Kmn, 64, 128, 4, false, true);
                mma_commit(mbar);
            }
            atomicAdd(dab + j, sab);
            atomicAdd(rs + j, srs);
            colsum16_add(e, cs + cb, lane);
        }
        if (!group_wait()) { aborted = true; break; }
        if (tid == 0 && has_next) load_set(N, 3);
        // ---- E7: dK into the register sums; after the group's last unit dq and dk stored (rows < L)
        {
            float x[32];
            tmem_ld_h32(tlane(tmem, warp, kTdK + 64 * wg), x);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) acck[q] += x[q];
            if (U.pos == upg - 1 && rr < L) {
                const size_t o = (size_t(t0 + rr) * hk + hq) * 128 + 64 * wg + 32 * (lane >> 4);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    *reinterpret_cast<float4 *>(dq + o + 4 * q) =
                        make_float4(accq[4 * q], accq[4 * q + 1], accq[4 * q + 2], accq[4 * q + 3]);
                    *reinterpret_cast<float4 *>(dk + o + 4 * q) =
                        make_float4(acck[4 * q], acck[4 * q + 1], acck[4 * q + 2], acck[4 * q + 3]);
                }
            }
        }
        if (tid < 64) {
            const int r = tid;
            const float gam = cv.gam[r], bt = cv.beta[r];
            const bool ok = r < L;
            const float db = dyv[r] + dbgv[r] * gam + dab[r];
            dG[r] = ok ? dgg[r] + dbgv[r] * bt * gam - dll[r] + rs[r] - cs[r] : 0.f;
            if (ok) atomicAdd(dbeta + size_t(t0 + r) * hv + h, db);
            float sl = ok ? dll[r] : 0.f;
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, m);
            if (lane == 0) atomicAdd(scal + 1, sl);
        }
        __syncthreads();
        if (tid < 32) {
            // gamma_L = e^(G_L) and every lambda_j = e^(G_L - G_j) also reach G_L, the last token's
            const float extra = scal[0] * cv.gam[63] + scal[1];
            const int r0 = 2 * tid, r1 = r0 + 1;
            const float a0 = dG[r0] + (r0 == L - 1 ? extra : 0.f), a1 = dG[r1] + (r1 == L - 1 ? extra : 0.f);
            float run = a0 + a1;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, run, m);
                if (tid + m < 32) run += y;
            }
            // d max(g, floor) / dg: zero below the floor
            if (r0 < L && a.g[size_t(t0 + r0) * hv + h] >= kGFloor) atomicAdd(dg + size_t(t0 + r0) * hv + h, run);
            if (r1 < L && a.g[size_t(t0 + r1) * hv + h] >= kGFloor) atomicAdd(dg + size_t(t0 + r1) * hv + h, run - a0);
        }
        tc_fence_before();
        __syncthreads();  // tensor memory, shared memory and the vectors are reused by the next unit
    }
    if (aborted && tid == 0 && my_units > 0) {
        mma_commit(mbar);
        (void)mbar_wait(mbar, mph);
        if (pending) {  // loads in flight into this CTA's shared memory: let them land
            mbar_arrive(lbar);
            (void)mbar_wait(lbar, lph);
        }
        record_abort(hdr, -8);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}
}  // namespace

bool backward_tc_supported(const gdn_shape_t &s) {
    return s.dtype == GDN_DTYPE_BF16 && s.head_dim_k == 128 && s.head_dim_v == 128 && s.num_qk_heads > 0 &&
           s.num_v_heads % s.num_qk_heads == 0;
}

BwdTcLayout bwd_tc_layout(const gdn_shape_t &s) {
    BwdTcLayout L;
    L.sched = ws_layout(s.num_seqs);
    size_t off = L.sched.total;
    L.cbase_off = off;
    off = align256(off + 4 * (size_t(s.num_seqs) + 1));
    off = (off + 1023) & ~size_t(1023);
    L.max_chunks = max_chunks_bound(s);
    const size_t n_items = size_t(L.max_chunks) * size_t(s.num_v_heads);
    L.items_off = off;
    off += n_items * kItemBytes;
    L.ck_s_off = off;
    off += n_items * kCkBytes;
    L.ck_ds_off = off;
    off += n_items * kCkBytes;
    L.total = align256(off);
    return L;
}

cudaError_t launch_backward_tc(const PrefillArgs &a, const void *dO, const float *dSf, float *dq, float *dk,
                               float *dv, float *dg, float *dbeta, float *dS0, float *s_final, unsigned char *ws,
                               const BwdTcLayout &L, cudaStream_t stream, int num_sms) {
    CUtensorMap mk, mq, mv, mdo;
    if (!make_map(&mk, a.k, a.hk, a.tokens) || !make_map(&mq, a.q, a.hk, a.tokens) ||
        !make_map(&mv, a.v, a.hv, a.tokens) || !make_map(&mdo, dO, a.hv, a.tokens))
        return cudaErrorInvalidValue;
    unsigned char *items = ws + L.items_off, *cks = ws + L.ck_s_off, *ckd = ws + L.ck_ds_off;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    auto config = [&](int grid, uint32_t smem) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(unsigned(grid));
        cfg.blockDim = dim3(kThr);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cfg;
    };
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bwd_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kASmem))) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kCSmem))) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kDSmem))) !=
            cudaSuccess)
        return e;
    // the item counts come from the schedule on the device: persistent grids
    {
        cudaLaunchConfig_t cfg = config(num_sms, kASmem);
        e = cudaLaunchKernelEx(&cfg, bwd_factor_kernel, a, mk, mq, mv, items);
        count_launch();
        if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int64_t ctas = 2 * int64_t(a.num_seqs) * a.hv;
        if (ctas > INT32_MAX) return cudaErrorInvalidValue;
        cudaLaunchConfig_t cfg = config(int(ctas), kCSmem);
        e = cudaLaunchKernelEx(&cfg, bwd_chain_kernel, a, mk, mdo, static_cast<const unsigned char *>(items), cks, ckd,
                               dSf, dS0, s_final);
        count_launch();
        if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        cudaLaunchConfig_t cfg = config(num_sms, kDSmem);
        e = cudaLaunchKernelEx(&cfg, bwd_grad_kernel, a, mk, mq, mv, mdo, static_cast<const unsigned char *>(items),
                               static_cast<const unsigned char *>(cks), static_cast<const unsigned char *>(ckd), dq,
                               dk, dv, dg, dbeta);
        count_launch();
        if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdn
