// gdn_backward.cu -- gradients of the chunked gated delta rule (training),
// fp32 arithmetic: products as split-bf16 tensor-core tiles for bf16 inputs,
// as CUDA-core tiles for fp32 inputs.
//
// The pages present the chunked form as the way to train the layer
// ("Architecture Thread I", the Gated DeltaNet section; "Gated Attention
// Architectures", sections 2 and 3).  For upstream gradients dO and dS_T,
// the kernel returns the gradients of L = sum dO . O + sum dS_T . S_T with
// respect to q, k, v, g, beta and the initial state.
//
// Per chunk of C tokens with start state S0 (G, gamma, Gamma, lambda, A, T,
// W, U~, U, P as in the forward):
//   S_C = gamma_L S0 + U^T diag(lambda) K,  O = diag(gamma) Q S0^T + P U,
//   U = U~ - W S0^T,  W = T diag(beta gamma) K,  U~ = T diag(beta) V,
//   T = (I + A)^-1,  A = strict(diag(beta)(K K^T (.) Gamma)),  P = Q K^T (.) Gamma.
// Reverse mode through these, for the chunk's end-state gradient dS:
//   dS0 = gamma_L dS + dO^T diag(gamma) Q - dU^T W        (the previous chunk's dS)
//   dU = diag(lambda) K dS^T + P^T dO,   dP = dO U^T (lower, with diagonal)
//   dW = -dU S0,  dT = dW (diag(bg) K)^T + dU (diag(beta) V)^T,  dA = -T^T dT T^T
//   dq, dk, dv, dbeta from the products; dg from the decays through the prefix sums G.
// Every row slice of d_v enters dS, dU, dv and dS0 alone, and dq, dk, dbeta
// and dg linearly, so a block owns (sequence, value head, 32 rows of d_v)
// and adds its share of the shared gradients with atomics.
//
// Pass 1 runs the chunks forward and stores each chunk's start state (the
// block's rows) in the workspace; pass 2 walks the chunks backward,
// recomputing the chunk's forward quantities from its stored start state.
#include <type_traits>

#include "gdn_internal.cuh"

namespace gdn {

constexpr int kBwdThreads = 256;
constexpr int kBwdC = 32;    // tokens per chunk
constexpr int kBwdRows = 32; // rows of d_v per block

struct BwdSmem {
    int ldk, ldc, ldv;
    size_t k, q, w, dw, dq, dk, s0, ds, v, u, du, dO, t, gm, kk, qk, dt, da, sm, se, vec, total;
};

// Row strides (floats) of the shared arrays.  The CUDA-core tiles (tc = false)
// read a row per lane, so an odd stride puts the 32 lanes in 32 banks.  The
// tensor-core tiles read fragment element (g, 2t) of lane 4g + t, as row g or
// as column g: a stride of 4 mod 8 maps the column form to bank 8t + g (all
// distinct) and the row form to at most 2 lanes a bank, where an odd stride
// gives g + 2t (up to 4 a bank) in both.
__host__ __device__ inline BwdSmem bwd_smem(int dk, bool tc) {
    BwdSmem s;
    s.ldk = tc ? dk + (12 - dk % 8) % 8 : dk + 1;
    s.ldc = kBwdC + (tc ? 4 : 1);
    s.ldv = kBwdRows + (tc ? 4 : 1);
    size_t off = 0;
    auto take = [&](size_t n) { size_t o = off; off += n; return o; };
    s.k = take(size_t(kBwdC) * s.ldk);
    s.q = take(size_t(kBwdC) * s.ldk);
    s.w = take(size_t(kBwdC) * s.ldk);
    s.dw = take(size_t(kBwdC) * s.ldk);
    s.dq = take(size_t(kBwdC) * s.ldk);
    s.dk = take(size_t(kBwdC) * s.ldk);
    s.s0 = take(size_t(kBwdRows) * s.ldk);
    s.ds = take(size_t(kBwdRows) * s.ldk);
    s.v = take(size_t(kBwdC) * s.ldv);
    s.u = take(size_t(kBwdC) * s.ldv);
    s.du = take(size_t(kBwdC) * s.ldv);
    s.dO = take(size_t(kBwdC) * s.ldv);
    s.t = take(size_t(kBwdC) * s.ldc);
    s.gm = take(size_t(kBwdC) * s.ldc);
    s.kk = take(size_t(kBwdC) * s.ldc);
    s.qk = take(size_t(kBwdC) * s.ldc);
    s.dt = take(size_t(kBwdC) * s.ldc);
    s.da = take(size_t(kBwdC) * s.ldc);
    s.sm = take(size_t(kBwdC) * s.ldc);  // C x C scratch: dT T^T
    s.se = take(size_t(kBwdC) * s.ldc);  // C x C scratch: the dbeta terms of dA
    s.vec = take(size_t(16) * kBwdC);
    s.total = off;
    return s;
}

// per-token vectors inside the vec block
enum { kVG = 0, kVGam, kVLam, kVB, kVBG, kVDG, kVDGam, kVDLam, kVDBG, kVDB, kVNum };

__device__ __forceinline__ float bwd_warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// floats kept per (chunk, value head, row slice) for pass 2: K K^T, Q K^T, T, W, U
__host__ __device__ inline size_t bwd_keep_floats(int dk) {
    return size_t(3) * kBwdC * kBwdC + size_t(kBwdC) * dk + size_t(kBwdC) * kBwdRows;
}

// checkpoint slot of chunk c of the sequence starting at token t0, sequence n:
// floor(t0 / C) + n + c never collides between sequences
__device__ __forceinline__ size_t bwd_slot(int t0, int n, int c) { return size_t(t0 / kBwdC + n + c); }

// out(m, n, sum_k a(m, k) b(k, n)) for m < M <= 32, n < N <= 32 TN, over the
// block's 256 threads: warp w takes rows 4w .. 4w + 3 and lane l the columns
// l + 32 i (i < TN), so b's reads are consecutive across a warp and a's are
// broadcasts; 4 TN multiply-adds per 4 + TN shared-memory loads.  a and b are
// element accessors, so scales, transposes and stacked operands need no copy.
// A given (M, N, TN) always maps an output element to the same thread, so
// products of one shape that accumulate into one array need no barrier
// between them.
template <int TN, class FA, class FB, class FO>
__device__ __forceinline__ void bgemm(int M, int N, int K, FA a, FB b, FO out) {
    const int m0 = 4 * (threadIdx.x >> 5), l = threadIdx.x & 31;
    if (m0 >= M) return;
    float acc[4][TN];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < TN; ++i) acc[j][i] = 0.f;
    for (int kk = 0; kk < K; ++kk) {
        float av[4], bv[TN];
#pragma unroll
        for (int j = 0; j < 4; ++j) av[j] = (m0 + j < M) ? a(m0 + j, kk) : 0.f;
#pragma unroll
        for (int i = 0; i < TN; ++i) bv[i] = (l + 32 * i < N) ? b(kk, l + 32 * i) : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < TN; ++i) acc[j][i] = fmaf(av[j], bv[i], acc[j][i]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < TN; ++i)
            if (m0 + j < M && l + 32 * i < N) out(m0 + j, l + 32 * i, acc[j][i]);
}

// The same contract on the tensor cores: 16 x 8 output tiles per warp
// (mma.sync m16n8k16, fp32 accumulation), tiles dealt to the 8 warps in a
// fixed order, so again a given (M, N) always maps an element to the same
// thread.  Each fp32 operand is split into a bf16 value and a bf16 residual,
// x = hi + lo, and a b is formed as hi hi + hi lo + lo hi: about 16
// mantissa bits, near the fp32 products of the CUDA-core path (the
// gradients of the decays are sums with heavy cancellation, which a plain
// bf16 product does not resolve).
__device__ __forceinline__ void bwd_split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ void bwd_mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <class FA, class FB, class FO>
__device__ __forceinline__ void tgemm(int M, int N, int K, FA a, FB b, FO out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int mt = (M + 15) / 16, nt = (N + 7) / 8;
    for (int tile = warp; tile < mt * nt; tile += kBwdThreads / 32) {
        const int m0 = (tile % mt) * 16, n0 = (tile / mt) * 8;
        // three independent accumulators, so the three products of a step do not wait on each other
        float d[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < K; k0 += 16) {
            auto A = [&](int r, int c) {
                const int m = m0 + r, kk = k0 + c;
                return (m < M && kk < K) ? a(m, kk) : 0.f;
            };
            auto B = [&](int r, int c) {
                const int kk = k0 + r, n = n0 + c;
                return (kk < K && n < N) ? b(kk, n) : 0.f;
            };
            uint32_t ah[4], al[4], bh[2], bl[2];
            bwd_split2(A(g, 2 * t), A(g, 2 * t + 1), ah[0], al[0]);
            bwd_split2(A(g + 8, 2 * t), A(g + 8, 2 * t + 1), ah[1], al[1]);
            bwd_split2(A(g, 2 * t + 8), A(g, 2 * t + 9), ah[2], al[2]);
            bwd_split2(A(g + 8, 2 * t + 8), A(g + 8, 2 * t + 9), ah[3], al[3]);
            bwd_split2(B(2 * t, g), B(2 * t + 1, g), bh[0], bl[0]);
            bwd_split2(B(2 * t + 8, g), B(2 * t + 9, g), bh[1], bl[1]);
            bwd_mma(d1, al, bh);
            bwd_mma(d2, ah, bl);
            bwd_mma(d, ah, bh);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] += d1[e] + d2[e];
        const int r0 = m0 + g, c0 = n0 + 2 * t;
        if (r0 < M && c0 < N) out(r0, c0, d[0]);
        if (r0 < M && c0 + 1 < N) out(r0, c0 + 1, d[1]);
        if (r0 + 8 < M && c0 < N) out(r0 + 8, c0, d[2]);
        if (r0 + 8 < M && c0 + 1 < N) out(r0 + 8, c0 + 1, d[3]);
    }
}

// bf16 inputs: tensor-core tiles with split operands; fp32 inputs: fp32 CUDA-core tiles.
template <bool kTC, int TN, class FA, class FB, class FO>
__device__ __forceinline__ void prod(int M, int N, int K, FA a, FB b, FO out) {
    if constexpr (kTC) tgemm(M, N, K, a, b, out);
    else bgemm<TN>(M, N, K, a, b, out);
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads, 1)
chunk_backward_kernel(const PrefillArgs a, const void *dO_, const float *dSf, float *dq, float *dk, float *dv,
                      float *dg, float *dbeta, float *dS0_out, float *ckpt, float *keep, int n_slices) {
    if (a.sched.hdr->status != GDN_OK) return;
    extern __shared__ float smem[];
    constexpr bool kTC = std::is_same<T, __nv_bfloat16>::value;
    const int dkd = a.dk, dvd = a.dv, hv = a.hv, hk = a.hk;
    const BwdSmem L = bwd_smem(dkd, kTC);
    const int ldk = L.ldk, ldc = L.ldc, ldv = L.ldv;
    float *K = smem + L.k, *Q = smem + L.q, *W = smem + L.w, *dW = smem + L.dw, *dQ = smem + L.dq,
          *dK = smem + L.dk, *S0 = smem + L.s0, *dS = smem + L.ds, *V = smem + L.v, *U = smem + L.u,
          *dU = smem + L.du, *dOs = smem + L.dO, *Tm = smem + L.t, *Gm = smem + L.gm, *KK = smem + L.kk,
          *QK = smem + L.qk, *dT = smem + L.dt, *dA = smem + L.da, *sM = smem + L.sm, *sE = smem + L.se,
          *vec = smem + L.vec;
    float *vG = vec + kVG * kBwdC, *vGam = vec + kVGam * kBwdC, *vLam = vec + kVLam * kBwdC,
          *vB = vec + kVB * kBwdC, *vBG = vec + kVBG * kBwdC, *vdG = vec + kVDG * kBwdC,
          *vdGam = vec + kVDGam * kBwdC, *vdLam = vec + kVDLam * kBwdC, *vdBG = vec + kVDBG * kBwdC,
          *vdB = vec + kVDB * kBwdC;
    __shared__ float red[kBwdThreads / 32];
    const int tid = threadIdx.x;
    // rows x d_k loops without a division: thread t takes column t & 127 of rows (t >> 7), (t >> 7) + 2, ...
    auto rows_dk = [&](int nrows, auto &&f) {
        const int x = tid & 127;
        if (x < dkd)
            for (int r = tid >> 7; r < nrows; r += kBwdThreads / 128) f(r, x);
    };
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    const T *dO = static_cast<const T *>(dO_);

    const int blk = blockIdx.x;
    const int rank = blk / (hv * n_slices);
    const int h = (blk / n_slices) % hv;
    const int slice = blk % n_slices;
    const int seq = a.sched.order[rank];
    const int t0 = a.sched.start[seq], len = a.sched.len[seq];
    const int hq = h / (hv / hk);
    const int i0 = slice * kBwdRows;
    const int nr = min(kBwdRows, dvd - i0);
    const size_t sbase = (size_t(seq) * hv + h) * size_t(dvd) * dkd;
    const int nch = (len + kBwdC - 1) / kBwdC;
    auto ck = [&](int c) { return ckpt + (bwd_slot(t0, seq, c) * hv + h) * size_t(dvd) * dkd + size_t(i0) * dkd; };
    // pass 1 keeps the chunk's K K^T, Q K^T, T, W and U (this block's rows) for pass 2
    const size_t keep_sz = bwd_keep_floats(dkd);
    auto kp = [&](int c) { return keep + ((bwd_slot(t0, seq, c) * hv + h) * n_slices + slice) * keep_sz; };

    // one chunk's inputs, prefix sums, per-token decays and Gamma.  Every
    // thread issues all of its global loads before its first shared-memory
    // store, so a group of loads costs about one memory latency, not one per row.
    constexpr int C = kBwdC, R = kBwdRows;
    static_assert(C == 32 && kBwdThreads % 128 == 0, "one warp spans a chunk; d_k columns map to 128 threads");
    constexpr int kRowStep = kBwdThreads / 128;     // rows apart of one thread's d_k-wide elements
    constexpr int kRowsPer = C / kRowStep;          // C x d_k elements per thread
    constexpr int kVPer = C * R / kBwdThreads;      // C x R elements per thread
    const int colx = tid & 127, row0 = tid >> 7;
    auto chunk_inputs = [&](int c, int Lc) {
        const int c0 = t0 + c * C;
        float kr[kRowsPer], qr[kRowsPer], vr[kVPer], gr = 0.f, br = 0.f;
#pragma unroll
        for (int e = 0; e < kRowsPer; ++e) {
            const int r = row0 + e * kRowStep;
            const bool ok = r < Lc && colx < dkd;
            const size_t o = (size_t(c0 + r) * hk + hq) * dkd + colx;
            kr[e] = ok ? to_f32(k[o]) : 0.f;
            qr[e] = ok ? to_f32(q[o]) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < kVPer; ++e) {
            const int idx = tid + e * kBwdThreads, r = idx / R, i = idx % R;
            vr[e] = (r < Lc && i < nr) ? to_f32(v[(size_t(c0 + r) * hv + h) * dvd + i0 + i]) : 0.f;
        }
        if (tid < Lc) {
            const size_t gb = size_t(c0 + tid) * hv + h;
            gr = fmaxf(a.g[gb], kGFloor);
            br = a.beta[gb];
        }
        if (colx < dkd)
#pragma unroll
            for (int e = 0; e < kRowsPer; ++e) {
                const int r = row0 + e * kRowStep;
                K[r * ldk + colx] = kr[e];
                Q[r * ldk + colx] = qr[e];
            }
#pragma unroll
        for (int e = 0; e < kVPer; ++e) {
            const int idx = tid + e * kBwdThreads;
            V[(idx / R) * ldv + idx % R] = vr[e];
        }
        if (tid < C) {  // the first warp: inclusive prefix sums G of the clamped gates
            const int l = tid;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, gr, m);
                if (l >= m) gr += y;
            }
            vG[l] = gr;
            vB[l] = br;
        }
        __syncthreads();
        if (tid < C) {
            const float gam = __expf(vG[tid]);
            vGam[tid] = gam;
            vLam[tid] = tid < Lc ? __expf(vG[Lc - 1] - vG[tid]) : 0.f;
            vBG[tid] = vB[tid] * gam;
        }
        for (int p = tid; p < C * C; p += kBwdThreads) {
            const int r = p / C, j = p % C;
            Gm[r * ldc + j] = j <= r ? __expf(vG[r] - vG[j]) : 0.f;
        }
        __syncthreads();
    };
    // the chunk's products: K K^T, Q K^T, T, W, U (after chunk_inputs)
    auto chunk_products = [&]() {
        // K K^T and Q K^T (lower, with the diagonal)
        prod<kTC, 1>(C, C, dkd, [&](int r, int x) { return K[r * ldk + x]; }, [&](int x, int j) { return K[j * ldk + x]; },
                 [&](int r, int j, float acc) { KK[r * ldc + j] = j <= r ? acc : 0.f; });
        prod<kTC, 1>(C, C, dkd, [&](int r, int x) { return Q[r * ldk + x]; }, [&](int x, int j) { return K[j * ldk + x]; },
                 [&](int r, int j, float acc) { QK[r * ldc + j] = j <= r ? acc : 0.f; });
        __syncthreads();
        // T = (I + A)^-1, A_rj = beta_r Gamma_rj KK_rj (j < r): A formed by the block, then one column
        // per thread by forward substitution with the column in registers (entries above the diagonal
        // come out as exact zeros, the diagonal as 1)
        for (int p = tid; p < C * C; p += kBwdThreads) {
            const int r = p / C, j = p % C;
            sM[r * ldc + j] = j < r ? vB[r] * Gm[r * ldc + j] * KK[r * ldc + j] : 0.f;
        }
        __syncthreads();
        if (tid < C) {
            const int col = tid;
            float xs[C];
#pragma unroll
            for (int r = 0; r < C; ++r) {
                float acc[4] = {r == col ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < r; ++j) acc[j & 3] = fmaf(-sM[r * ldc + j], xs[j], acc[j & 3]);
                xs[r] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                Tm[r * ldc + col] = xs[r];
            }
        }
        __syncthreads();
        // W = T diag(beta gamma) K
        prod<kTC, 4>(C, dkd, C, [&](int r, int j) { return Tm[r * ldc + j] * vBG[j]; },
                 [&](int j, int x) { return K[j * ldk + x]; }, [&](int r, int x, float acc) { W[r * ldk + x] = acc; });
        __syncthreads();
        // U = T diag(beta) V - W S0^T
        prod<kTC, 1>(C, R, C, [&](int r, int j) { return Tm[r * ldc + j] * vB[j]; },
                 [&](int j, int i) { return V[j * ldv + i]; }, [&](int r, int i, float acc) { U[r * ldv + i] = acc; });
        prod<kTC, 1>(C, R, dkd, [&](int r, int x) { return -W[r * ldk + x]; },
                 [&](int x, int i) { return S0[i * ldk + x]; }, [&](int r, int i, float acc) { U[r * ldv + i] += acc; });
        __syncthreads();
    };

    // K K^T, Q K^T, T (C x C each), W (C x d_k), U (C x 32) to the workspace
    auto keep_store = [&](float *base) {
        for (int e = tid; e < 3 * C * C; e += kBwdThreads) {
            const int m = e / (C * C), r = (e / C) % C, j = e % C;
            base[e] = (m == 0 ? KK : (m == 1 ? QK : Tm))[r * ldc + j];
        }
        float *bw = base + 3 * C * C;
        rows_dk(C, [&](int r, int x) { bw[r * dkd + x] = W[r * ldk + x]; });
        float *bu = bw + C * dkd;
        for (int e = tid; e < C * R; e += kBwdThreads) bu[e] = U[(e / R) * ldv + e % R];
    };
    // and back, with the chunk's dO rows in the same group of loads
    static_assert((C * C) % kBwdThreads == 0, "a thread's C x C elements stay in one matrix per step");
    auto keep_load = [&](const float *base, int c0, int Lc) {
        constexpr int kCC = 3 * C * C / kBwdThreads;
        float cc[kCC], wr[kRowsPer], ur[kVPer], orow[kVPer];
        const float *bw = base + 3 * C * C, *bu = bw + C * dkd;
#pragma unroll
        for (int e = 0; e < kCC; ++e) cc[e] = base[tid + e * kBwdThreads];
#pragma unroll
        for (int e = 0; e < kRowsPer; ++e)
            wr[e] = colx < dkd ? bw[size_t(row0 + e * kRowStep) * dkd + colx] : 0.f;
#pragma unroll
        for (int e = 0; e < kVPer; ++e) {
            const int idx = tid + e * kBwdThreads, r = idx / R, i = idx % R;
            ur[e] = bu[idx];
            orow[e] = (r < Lc && i < nr) ? to_f32(dO[(size_t(c0 + r) * hv + h) * dvd + i0 + i]) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < kCC; ++e) {
            const int idx = tid + e * kBwdThreads, r = (idx / C) % C, j = idx % C;
            constexpr int kPerMat = C * C / kBwdThreads;
            float *mat = e / kPerMat == 0 ? KK : (e / kPerMat == 1 ? QK : Tm);
            mat[r * ldc + j] = cc[e];
        }
        if (colx < dkd)
#pragma unroll
            for (int e = 0; e < kRowsPer; ++e) W[(row0 + e * kRowStep) * ldk + colx] = wr[e];
#pragma unroll
        for (int e = 0; e < kVPer; ++e) {
            const int idx = tid + e * kBwdThreads, r = idx / R, i = idx % R;
            U[r * ldv + i] = ur[e];
            dOs[r * ldv + i] = orow[e];
        }
    };
    // R rows of d_k floats (row stride d_k; rows >= nvalid, or all rows for a null source, are zeros)
    static_assert(kBwdRows == kBwdC, "state row slices use the chunk's row mapping");
    auto load_rows = [&](float *dst, const float *src, int nvalid) {
        float t[kRowsPer];
#pragma unroll
        for (int e = 0; e < kRowsPer; ++e) {
            const int r = row0 + e * kRowStep;
            t[e] = (src && r < nvalid && colx < dkd) ? src[size_t(r) * dkd + colx] : 0.f;
        }
        if (colx < dkd)
#pragma unroll
            for (int e = 0; e < kRowsPer; ++e) dst[(row0 + e * kRowStep) * ldk + colx] = t[e];
    };

    // ---- pass 1: chunk start states into the workspace ----
    load_rows(S0, a.s0 ? a.s0 + sbase + size_t(i0) * dkd : nullptr, nr);
    __syncthreads();
    for (int c = 0; c < nch; ++c) {
        const int Lc = min(C, len - c * C);
        float *dst = ck(c);
        rows_dk(nr, [&](int i, int x) { dst[i * dkd + x] = S0[i * ldk + x]; });
        chunk_inputs(c, Lc);
        chunk_products();
        keep_store(kp(c));
        const float gl = __expf(vG[Lc - 1]);
        // S <- gamma_L S + U^T diag(lambda) K
        prod<kTC, 4>(R, dkd, Lc, [&](int i, int j) { return U[j * ldv + i] * vLam[j]; },
                 [&](int j, int x) { return K[j * ldk + x]; },
                 [&](int i, int x, float acc) { S0[i * ldk + x] = fmaf(gl, S0[i * ldk + x], acc); });
        __syncthreads();
    }

    // ---- pass 2: backward over the chunks ----
    load_rows(dS, dSf ? dSf + sbase + size_t(i0) * dkd : nullptr, nr);
    for (int c = nch - 1; c >= 0; --c) {
        const int Lc = min(C, len - c * C);
        const int c0 = t0 + c * C;
        load_rows(S0, ck(c), nr);
        chunk_inputs(c, Lc);
        keep_load(kp(c), c0, Lc);
        rows_dk(C, [&](int r, int x) {
            dQ[r * ldk + x] = 0.f;
            dK[r * ldk + x] = 0.f;
        });
        if (tid < C) vdGam[tid] = vdLam[tid] = vdBG[tid] = vdB[tid] = vdG[tid] = 0.f;
        // dgamma_L = <dS, S0> over the block's rows
        float part = 0.f;
        rows_dk(R, [&](int i, int x) { part = fmaf(dS[i * ldk + x], S0[i * ldk + x], part); });
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
        if ((tid & 31) == 0) red[tid >> 5] = part;
        __syncthreads();
        float dgl = 0.f;
        for (int w = 0; w < kBwdThreads / 32; ++w) dgl += red[w];
        // from the end state: Z_ji = dS_i . k_j, dU = diag(lambda) Z, dlambda_j = sum_i U_ji Z_ji
        prod<kTC, 1>(C, R, dkd, [&](int j, int x) { return K[j * ldk + x]; }, [&](int x, int i) { return dS[i * ldk + x]; },
                 [&](int j, int i, float z) {
                     dU[j * ldv + i] = vLam[j] * z;
                     dT[j * ldc + i] = U[j * ldv + i] * z;  // scratch, summed below
                 });
        // dK_j += lambda_j dS^T u_j;  Y_r = dO_r S0: dQ_r += gamma_r Y_r, dgamma_r += Y_r . q_r
        prod<kTC, 4>(C, dkd, R, [&](int j, int i) { return U[j * ldv + i]; }, [&](int i, int x) { return dS[i * ldk + x]; },
                 [&](int j, int x, float acc) { dK[j * ldk + x] += vLam[j] * acc; });
        prod<kTC, 4>(C, dkd, R, [&](int r, int i) { return dOs[r * ldv + i]; }, [&](int i, int x) { return S0[i * ldk + x]; },
                 [&](int r, int x, float y) {
                     dQ[r * ldk + x] += vGam[r] * y;
                     dW[r * ldk + x] = y * Q[r * ldk + x];  // scratch for dgamma
                 });
        __syncthreads();
        for (int r = tid >> 5; r < C; r += kBwdThreads / 32) {  // a warp per row, lanes over the columns
            const int l = tid & 31;
            float sl = l < R ? dT[r * ldc + l] : 0.f, sg = 0.f;
            for (int x = l; x < dkd; x += 32) sg += dW[r * ldk + x];
            sl = bwd_warp_sum(sl);
            sg = bwd_warp_sum(sg);
            if (l == 0) {
                vdLam[r] = sl;
                vdGam[r] += sg;
            }
        }
        __syncthreads();
        // dP_rj = dO_r . u_j (j <= r), kept in dT's storage
        prod<kTC, 1>(C, C, R, [&](int r, int i) { return dOs[r * ldv + i]; }, [&](int i, int j) { return U[j * ldv + i]; },
                 [&](int r, int j, float acc) { dT[r * ldc + j] = j <= r ? acc : 0.f; });
        __syncthreads();
        // dU_j += sum_r P_rj dO_r;  P = Q K^T (.) Gamma: dQ, dK and dGamma (in dA)
        prod<kTC, 1>(C, R, C, [&](int j, int r) { return Gm[r * ldc + j] * QK[r * ldc + j]; },
                 [&](int r, int i) { return dOs[r * ldv + i]; }, [&](int j, int i, float acc) { dU[j * ldv + i] += acc; });
        prod<kTC, 4>(C, dkd, C, [&](int r, int j) { return dT[r * ldc + j] * Gm[r * ldc + j]; },
                 [&](int j, int x) { return K[j * ldk + x]; }, [&](int r, int x, float acc) { dQ[r * ldk + x] += acc; });
        prod<kTC, 4>(C, dkd, C, [&](int r, int i) { return dT[i * ldc + r] * Gm[i * ldc + r]; },
                 [&](int i, int x) { return Q[i * ldk + x]; }, [&](int r, int x, float acc) { dK[r * ldk + x] += acc; });
        for (int p = tid; p < C * C; p += kBwdThreads) {
            const int r = p / C, j = p % C;
            dA[r * ldc + j] = j <= r ? dT[r * ldc + j] * QK[r * ldc + j] : 0.f;  // dGamma so far
        }
        __syncthreads();
        // dW = -dU S0;  dS0 = gamma_L dS + dO^T diag(gamma) Q - dU^T W (over dS)
        const float gL = __expf(vG[Lc - 1]);
        prod<kTC, 4>(C, dkd, R, [&](int r, int i) { return -dU[r * ldv + i]; }, [&](int i, int x) { return S0[i * ldk + x]; },
                 [&](int r, int x, float acc) { dW[r * ldk + x] = acc; });
        prod<kTC, 4>(R, dkd, C, [&](int i, int r) { return dOs[r * ldv + i] * vGam[r]; },
                 [&](int r, int x) { return Q[r * ldk + x]; },
                 [&](int i, int x, float acc) { dS[i * ldk + x] = fmaf(gL, dS[i * ldk + x], acc); });
        prod<kTC, 4>(R, dkd, C, [&](int i, int r) { return -dU[r * ldv + i]; }, [&](int r, int x) { return W[r * ldk + x]; },
                 [&](int i, int x, float acc) { dS[i * ldk + x] += acc; });
        __syncthreads();
        // dT_rj = dW_r . (bg_j k_j) + dU_r . (beta_j v_j), j <= r
        prod<kTC, 1>(C, C, dkd, [&](int r, int x) { return dW[r * ldk + x]; },
                 [&](int x, int j) { return K[j * ldk + x] * vBG[j]; },
                 [&](int r, int j, float acc) { dT[r * ldc + j] = j <= r ? acc : 0.f; });
        prod<kTC, 1>(C, C, R, [&](int r, int i) { return dU[r * ldv + i]; }, [&](int i, int j) { return V[j * ldv + i] * vB[j]; },
                 [&](int r, int j, float acc) {
                     if (j <= r) dT[r * ldc + j] += acc;
                 });
        __syncthreads();
        // dX = T^T dW: dK_j += bg_j dX_j, dbg_j = dX_j . k_j;  dY = T^T dU: dv_j = beta_j dY_j, dbeta_j += dY_j . v_j
        prod<kTC, 4>(C, dkd, C, [&](int j, int r) { return Tm[r * ldc + j]; }, [&](int r, int x) { return dW[r * ldk + x]; },
                 [&](int j, int x, float dx) {
                     dK[j * ldk + x] = fmaf(vBG[j], dx, dK[j * ldk + x]);
                     Q[j * ldk + x] = dx * K[j * ldk + x];  // scratch for dbg (Q is no longer needed)
                 });
        prod<kTC, 1>(C, R, C, [&](int j, int r) { return Tm[r * ldc + j]; }, [&](int r, int i) { return dU[r * ldv + i]; },
                 [&](int j, int i, float dy) {
                     if (j < Lc && i < nr) dv[(size_t(c0 + j) * hv + h) * dvd + i0 + i] = vB[j] * dy;
                     U[j * ldv + i] = dy * V[j * ldv + i];  // scratch for dbeta (U is no longer needed)
                 });
        __syncthreads();
        for (int r = tid >> 5; r < C; r += kBwdThreads / 32) {  // a warp per row, lanes over the columns
            const int l = tid & 31;
            float su = l < R ? U[r * ldv + l] : 0.f, sb = 0.f;
            for (int x = l; x < dkd; x += 32) sb += Q[r * ldk + x];
            sb = bwd_warp_sum(sb);
            su = bwd_warp_sum(su);
            if (l == 0) {
                vdBG[r] = sb;
                vdB[r] = su;
            }
        }
        // dA = -T^T dT T^T (strictly lower): M = dT T^T first
        prod<kTC, 1>(C, C, C, [&](int r, int m) { return dT[r * ldc + m]; }, [&](int m, int j) { return Tm[j * ldc + m]; },
                 [&](int r, int j, float acc) { sM[r * ldc + j] = acc; });
        __syncthreads();
        // A_rj = beta_r Gamma_rj KK_rj: dbeta_r terms (sE), dGamma_rj (dA), dKK_rj (dT)
        prod<kTC, 1>(C, C, C, [&](int r, int m) { return Tm[m * ldc + r]; }, [&](int m, int j) { return sM[m * ldc + j]; },
                 [&](int r, int j, float acc) {
                     const float da = -acc;
                     const bool low = j < r;
                     dT[r * ldc + j] = low ? da * vB[r] * Gm[r * ldc + j] : 0.f;
                     if (low) dA[r * ldc + j] += da * vB[r] * KK[r * ldc + j];
                     sE[r * ldc + j] = low ? da * Gm[r * ldc + j] * KK[r * ldc + j] : 0.f;
                 });
        __syncthreads();
        if (tid < C) {
            float sv = 0.f;
            for (int j = 0; j < tid; ++j) sv += sE[tid * ldc + j];
            vdB[tid] += sv;
        }
        // dK_r += sum_j (dKK_rj + dKK_jr) k_j
        prod<kTC, 4>(C, dkd, C, [&](int r, int j) { return j < r ? dT[r * ldc + j] : (j > r ? dT[j * ldc + r] : 0.f); },
                 [&](int j, int x) { return K[j * ldk + x]; }, [&](int r, int x, float acc) { dK[r * ldk + x] += acc; });
        __syncthreads();
        // decays: beta gamma, gamma, lambda, gamma_L and Gamma through G, then dg = reverse prefix
        // sums of dG (the first warp, a lane per token; gamma_L = e^(G_L) and every lambda_j =
        // e^(G_L - G_j) also reach G_L, the last token's)
        if (tid < C) {
            const int r = tid;
            vdB[r] = fmaf(vdBG[r], vGam[r], vdB[r]);
            const float dgam = fmaf(vdBG[r], vB[r], vdGam[r]);
            float dG = dgam * vGam[r] - vdLam[r] * vLam[r];
            for (int j = 0; j <= r; ++j) dG = fmaf(dA[r * ldc + j], Gm[r * ldc + j], dG);
            for (int i = r; i < C; ++i) dG = fmaf(-dA[i * ldc + r], Gm[i * ldc + r], dG);
            const float extra = dgl * gL + bwd_warp_sum(r < Lc ? vdLam[r] * vLam[r] : 0.f);
            float run = r < Lc ? dG + (r == Lc - 1 ? extra : 0.f) : 0.f;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, run, m);
                if (r + m < 32) run += y;
            }
            vdG[r] = run;
        }
        __syncthreads();
        // the block's share of the shared gradients
        rows_dk(Lc, [&](int r, int x) {
            const size_t o = (size_t(c0 + r) * hk + hq) * dkd + x;
            atomicAdd(dq + o, dQ[r * ldk + x]);
            atomicAdd(dk + o, dK[r * ldk + x]);
        });
        if (tid < Lc) {
            // d max(g, floor) / dg: zero below the floor
            if (a.g[size_t(c0 + tid) * hv + h] >= kGFloor) atomicAdd(dg + size_t(c0 + tid) * hv + h, vdG[tid]);
            atomicAdd(dbeta + size_t(c0 + tid) * hv + h, vdB[tid]);
        }
        __syncthreads();
    }
    if (dS0_out)
        rows_dk(nr, [&](int i, int x) { dS0_out[sbase + size_t(i0 + i) * dkd + x] = dS[i * ldk + x]; });
}

static size_t bwd_slots(int32_t tokens, int32_t num_seqs) { return size_t(tokens) / kBwdC + size_t(num_seqs) + 1; }

// chunk start states, then the kept per-chunk quantities (256-byte aligned)
size_t backward_ckpt_bytes(int32_t tokens, int32_t num_seqs, int32_t hv, int32_t dk, int32_t dv) {
    const size_t slots = bwd_slots(tokens, num_seqs);
    const size_t states = (slots * size_t(hv) * size_t(dv) * size_t(dk) * sizeof(float) + 255) / 256 * 256;
    const size_t n_slices = (size_t(dv) + kBwdRows - 1) / kBwdRows;
    return states + slots * size_t(hv) * n_slices * bwd_keep_floats(dk) * sizeof(float);
}

cudaError_t launch_chunk_backward(const PrefillArgs &a, const void *dO, const float *dSf, float *dq, float *dk,
                                  float *dv, float *dg, float *dbeta, float *dS0, float *ckpt, cudaStream_t stream) {
    const int n_slices = (a.dv + kBwdRows - 1) / kBwdRows;
    const int64_t blocks = int64_t(a.num_seqs) * a.hv * n_slices;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > INT32_MAX || a.dk > 128 || a.dv > 128) return cudaErrorInvalidValue;
    const size_t bytes = bwd_smem(a.dk, a.dtype == GDN_DTYPE_BF16).total * sizeof(float);
    const size_t slots = bwd_slots(a.tokens, a.num_seqs);
    float *keep = ckpt + (slots * size_t(a.hv) * size_t(a.dv) * size_t(a.dk) * sizeof(float) + 255) / 256 * 256 /
                             sizeof(float);
    cudaError_t e;
    if (a.dtype == GDN_DTYPE_BF16) {
        e = cudaFuncSetAttribute(chunk_backward_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(bytes));
        if (e != cudaSuccess) return e;
        chunk_backward_kernel<__nv_bfloat16><<<unsigned(blocks), kBwdThreads, bytes, stream>>>(
            a, dO, dSf, dq, dk, dv, dg, dbeta, dS0, ckpt, keep, n_slices);
    } else {
        e = cudaFuncSetAttribute(chunk_backward_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(bytes));
        if (e != cudaSuccess) return e;
        chunk_backward_kernel<float><<<unsigned(blocks), kBwdThreads, bytes, stream>>>(a, dO, dSf, dq, dk, dv, dg,
                                                                                      dbeta, dS0, ckpt, keep,
                                                                                      n_slices);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
