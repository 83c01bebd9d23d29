// gdn_chunk_simt.cu -- chunkwise gated delta rule on CUDA cores, fp32
// arithmetic throughout.  Serves fp32 inputs (whose 1e-4 accuracy bar the
// 10-bit-mantissa tensor-core formats cannot meet) and every shape the
// tensor-core kernel does not take (d_k, d_v <= 128, C in {16, 32, 64}).
//
// Chunk algebra (per chunk of L <= C tokens, start state S0, rows r, j):
//   G_r = g_0 + ... + g_r, gamma_r = exp(G_r), Gamma_rj = exp(G_r - G_j)
//   A_rj = beta_r Gamma_rj (k_r . k_j), j < r;     T = (I + A)^-1
//   W = T diag(beta gamma) K,  U~ = T diag(beta) V,  U = U~ - W S0^T
//   O = diag(gamma) Q S0^T + (Q K^T (.) Gamma) U     (Gamma incl. diagonal)
//   S <- gamma_{L-1} S0 + U^T diag(exp(G_{L-1} - G)) K
// -- the WY representation of the DeltaNet transitions with per-chunk
// cumulative decay ("Gated Attention Architectures", sections 2 and 3) and
// the decay-aware masked chunk output of its section 1 (GLA), applied to
// the corrected values U.
//
// One block owns a unit (sequence, value head, 32-row slice of d_v) and
// walks the sequence's chunks in order; units are handed out longest
// sequence first through an atomic counter (persistent grid).
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kSimtDvs = 32;  // rows of S (value index) per block

struct SimtSmem {
    int C, dk, ldk, ldc, ldv;
    size_t kc, qc, wc, vc, uc, am, tm, pm, st, gg, bb, bg, lam, total_floats;
};

__host__ __device__ inline SimtSmem simt_smem(int C, int dk) {
    SimtSmem s;
    s.C = C; s.dk = dk;
    s.ldk = dk + 1;       // padded row strides avoid shared-memory bank conflicts
    s.ldc = C + 1;
    s.ldv = kSimtDvs + 1;
    size_t off = 0;
    s.kc = off; off += size_t(C) * s.ldk;
    s.qc = off; off += size_t(C) * s.ldk;
    s.wc = off; off += size_t(C) * s.ldk;
    s.vc = off; off += size_t(C) * s.ldv;
    s.uc = off; off += size_t(C) * s.ldv;
    s.am = off; off += size_t(C) * s.ldc;
    s.tm = off; off += size_t(C) * s.ldc;
    s.pm = off; off += size_t(C) * s.ldc;
    s.st = off; off += size_t(kSimtDvs) * s.ldk;
    s.gg = off; off += C;
    s.bb = off; off += C;
    s.bg = off; off += C;
    s.lam = off; off += C;
    s.total_floats = off;
    return s;
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(PrefillArgs a, int n_slices) {
    extern __shared__ float smem[];
    __shared__ int s_unit;
    const SimtSmem L = simt_smem(a.chunk, a.dk);
    float *Kc = smem + L.kc, *Qc = smem + L.qc, *Wc = smem + L.wc, *Vc = smem + L.vc, *Uc = smem + L.uc;
    float *Am = smem + L.am, *Tm = smem + L.tm, *Pm = smem + L.pm, *St = smem + L.st;
    float *Gc = smem + L.gg, *Bc = smem + L.bb, *BGc = smem + L.bg, *Lam = smem + L.lam;
    const int C = a.chunk, dk = a.dk, dv = a.dv, hv = a.hv, hk = a.hk;
    const int ldk = L.ldk, ldc = L.ldc, ldv = L.ldv;
    const int tid = threadIdx.x;
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    T *o = static_cast<T *>(a.o);
    if (a.sched.hdr->status != GDN_OK) return;
    const int total_units = a.num_seqs * hv * n_slices;

    for (;;) {
        if (tid == 0) s_unit = int(atomicAdd(&a.sched.hdr->next_unit, 1u));
        __syncthreads();
        const int unit = s_unit;
        __syncthreads();
        if (unit >= total_units) break;
        const int rank = unit / (hv * n_slices);
        const int h = (unit / n_slices) % hv;
        const int slice = unit % n_slices;
        const int seq = a.sched.order[rank];
        const int t0 = a.sched.start[seq], len = a.sched.len[seq];
        const int hq = h / (hv / hk);
        const int i0 = slice * kSimtDvs;
        const size_t sbase = (size_t(seq) * hv + h) * dv * dk;

        for (int idx = tid; idx < kSimtDvs * dk; idx += kSimtThreads) {
            const int i = idx / dk, x = idx % dk;
            St[i * ldk + x] = (a.s0 && i0 + i < dv) ? a.s0[sbase + size_t(i0 + i) * dk + x] : 0.f;
        }
        __syncthreads();

        for (int c0 = 0; c0 < len; c0 += C) {
            const int Lc = min(C, len - c0);
            // 1. this chunk's rows (zero beyond the sequence end)
            for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
                const int r = idx / dk, x = idx % dk;
                float kv = 0.f, qv = 0.f;
                if (r < Lc) {
                    const size_t off = (size_t(t0 + c0 + r) * hk + hq) * dk + x;
                    kv = to_f32(k[off]);
                    qv = to_f32(q[off]);
                }
                Kc[r * ldk + x] = kv;
                Qc[r * ldk + x] = qv;
            }
            for (int idx = tid; idx < C * kSimtDvs; idx += kSimtThreads) {
                const int r = idx / kSimtDvs, i = idx % kSimtDvs;
                Vc[r * ldv + i] = (r < Lc && i0 + i < dv) ? to_f32(v[(size_t(t0 + c0 + r) * hv + h) * dv + i0 + i])
                                                          : 0.f;
            }
            if (tid < C) {
                const size_t off = size_t(t0 + c0 + tid) * hv + h;
                const bool logits = a.flags & GDN_FLAG_GATE_LOGITS;
                Gc[tid] = tid < Lc ? fmaxf(logits ? log_sigmoid(a.g[off]) : a.g[off], kGFloor) : 0.f;
                Bc[tid] = tid < Lc ? (logits ? sigmoid(a.beta[off]) : a.beta[off]) : 0.f;
            }
            __syncthreads();
            if (a.flags & GDN_FLAG_QK_L2NORM) {
                // raw q and k: each row scaled by 1 / max(||row||, 1e-12), a warp per row
                const int warp = tid >> 5, lane = tid & 31;
                for (int rr = warp; rr < 2 * C; rr += kSimtThreads / 32) {
                    float *row = (rr < C ? Kc + rr * ldk : Qc + (rr - C) * ldk);
                    float ss = 0.f;
                    for (int x = lane; x < dk; x += 32) ss = fmaf(row[x], row[x], ss);
#pragma unroll
                    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float inv = inv_l2(ss);
                    for (int x = lane; x < dk; x += 32) row[x] *= inv;
                }
                __syncthreads();
            }
            // 2. cumulative log-decay inside the chunk
            if (tid == 0) {
                float run = 0.f;
                for (int r = 0; r < C; ++r) {
                    run += Gc[r];
                    Gc[r] = run;
                }
            }
            __syncthreads();
            if (tid < C) {
                BGc[tid] = Bc[tid] * __expf(Gc[tid]);
                Lam[tid] = tid < Lc ? __expf(Gc[Lc - 1] - Gc[tid]) : 0.f;
            }
            // 3. A (strictly lower) and P = Q K^T (.) Gamma (lower incl. diagonal)
            for (int p = tid; p < C * C; p += kSimtThreads) {
                const int r = p / C, j = p % C;
                float kk = 0.f, qk = 0.f;
                if (j <= r) {
                    for (int x = 0; x < dk; ++x) {
                        const float kj = Kc[j * ldk + x];
                        kk = fmaf(Kc[r * ldk + x], kj, kk);
                        qk = fmaf(Qc[r * ldk + x], kj, qk);
                    }
                }
                const float gam = j <= r ? __expf(Gc[r] - Gc[j]) : 0.f;
                Am[r * ldc + j] = j < r ? Bc[r] * gam * kk : 0.f;
                Pm[r * ldc + j] = gam * qk;
            }
            __syncthreads();
            // 4. T = (I + A)^-1, one column per thread: (I + A) t_c = e_c
            if (tid < C) {
                const int c = tid;
                for (int r = 0; r < C; ++r) {
                    float x;
                    if (r < c) {
                        x = 0.f;
                    } else if (r == c) {
                        x = 1.f;
                    } else {
                        x = 0.f;
                        for (int j = c; j < r; ++j) x = fmaf(-Am[r * ldc + j], Tm[j * ldc + c], x);
                    }
                    Tm[r * ldc + c] = x;
                }
            }
            __syncthreads();
            // 5. W = T diag(beta gamma) K and U~ = T diag(beta) V
            for (int idx = tid; idx < C * dk; idx += kSimtThreads) {
                const int r = idx / dk, x = idx % dk;
                float acc = 0.f;
                for (int j = 0; j <= r; ++j) acc = fmaf(Tm[r * ldc + j] * BGc[j], Kc[j * ldk + x], acc);
                Wc[r * ldk + x] = acc;
            }
            for (int idx = tid; idx < C * kSimtDvs; idx += kSimtThreads) {
                const int r = idx / kSimtDvs, i = idx % kSimtDvs;
                float acc = 0.f;
                for (int j = 0; j <= r; ++j) acc = fmaf(Tm[r * ldc + j] * Bc[j], Vc[j * ldv + i], acc);
                Uc[r * ldv + i] = acc;
            }
            __syncthreads();
            // 6. U = U~ - W S0^T
            for (int idx = tid; idx < C * kSimtDvs; idx += kSimtThreads) {
                const int r = idx / kSimtDvs, i = idx % kSimtDvs;
                float acc = 0.f;
                for (int x = 0; x < dk; ++x) acc = fmaf(Wc[r * ldk + x], St[i * ldk + x], acc);
                Uc[r * ldv + i] -= acc;
            }
            __syncthreads();
            // 7. O = diag(gamma) Q S0^T + P U
            for (int idx = tid; idx < C * kSimtDvs; idx += kSimtThreads) {
                const int r = idx / kSimtDvs, i = idx % kSimtDvs;
                if (r >= Lc || i0 + i >= dv) continue;
                float inter = 0.f;
                for (int x = 0; x < dk; ++x) inter = fmaf(Qc[r * ldk + x], St[i * ldk + x], inter);
                float intra = 0.f;
                for (int j = 0; j <= r; ++j) intra = fmaf(Pm[r * ldc + j], Uc[j * ldv + i], intra);
                o[(size_t(t0 + c0 + r) * hv + h) * dv + i0 + i] = from_f32<T>(fmaf(__expf(Gc[r]), inter, intra));
            }
            __syncthreads();
            // 8. S <- gamma_{L-1} S0 + U^T diag(exp(G_{L-1} - G)) K
            const float gl = __expf(Gc[Lc - 1]);
            for (int idx = tid; idx < kSimtDvs * dk; idx += kSimtThreads) {
                const int i = idx / dk, x = idx % dk;
                float acc = 0.f;
                for (int j = 0; j < Lc; ++j) acc = fmaf(Uc[j * ldv + i] * Lam[j], Kc[j * ldk + x], acc);
                St[i * ldk + x] = fmaf(gl, St[i * ldk + x], acc);
            }
            __syncthreads();
        }
        if (a.s_final) {
            for (int idx = tid; idx < kSimtDvs * dk; idx += kSimtThreads) {
                const int i = idx / dk, x = idx % dk;
                if (i0 + i < dv) a.s_final[sbase + size_t(i0 + i) * dk + x] = St[i * ldk + x];
            }
        }
        __syncthreads();
    }
}

cudaError_t launch_chunk_simt(const PrefillArgs &a, cudaStream_t stream, int num_sms) {
    const SimtSmem L = simt_smem(a.chunk, a.dk);
    const size_t bytes = L.total_floats * sizeof(float);
    const int n_slices = (a.dv + kSimtDvs - 1) / kSimtDvs;
    const int64_t units = int64_t(a.num_seqs) * a.hv * n_slices;
    cudaError_t e;
    if (a.dtype == GDN_DTYPE_BF16)
        e = cudaFuncSetAttribute(chunk_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(bytes));
    else
        e = cudaFuncSetAttribute(chunk_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e != cudaSuccess) return e;
    const int per_sm = bytes > 110 * 1024 ? 1 : (bytes > 72 * 1024 ? 2 : 4);
    const int64_t grid = units < int64_t(num_sms) * per_sm ? units : int64_t(num_sms) * per_sm;
    if (grid <= 0) return cudaSuccess;
    if (a.dtype == GDN_DTYPE_BF16)
        chunk_simt_kernel<__nv_bfloat16><<<unsigned(grid), kSimtThreads, bytes, stream>>>(a, n_slices);
    else
        chunk_simt_kernel<float><<<unsigned(grid), kSimtThreads, bytes, stream>>>(a, n_slices);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
