// gdn_sched.cu -- prefill schedule: checks cu_seqlens on the device and fills
// the workspace tables the prefill kernels read (sequence starts, lengths and
// a longest-first order for greedy scheduling of (sequence, head) units).
#include "gdn_internal.cuh"

namespace gdn {

constexpr int kSchedThreads = 1024;
// Above this many sequences the longest-first ranking (quadratic in N) is
// skipped and sequences keep their given order.
constexpr int kMaxRankedSeqs = 8192;

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(int32_t num_seqs, int32_t tokens, int32_t batched_len, const int32_t *__restrict__ cu,
                WsHeader *hdr, int32_t *order, int32_t *start, int32_t *len, int32_t *chunk_base) {
    __shared__ int bad;
    __shared__ int part[kSchedThreads];
    // the prefill kernel that follows may start its own set-up now; it waits for
    // this kernel's results (griddepcontrol.wait) before reading them
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        bad = -1;
        hdr->status = GDN_OK;
        hdr->bad_index = -1;
        hdr->next_unit = 0;
        hdr->num_seqs = num_seqs;
        hdr->total_chunks = 0;
    }
    __syncthreads();
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        int s0, s1;
        if (cu) {
            s0 = cu[n];
            s1 = cu[n + 1];
            const bool ok = s1 >= s0 && s0 >= 0 && s1 <= tokens && (n != 0 || s0 == 0) &&
                            (n != num_seqs - 1 || s1 == tokens);
            if (!ok) atomicMax(&bad, n);
        } else {
            s0 = n * batched_len;
            s1 = s0 + batched_len;
        }
        start[n] = s0;
        len[n] = max(s1 - s0, 0);
    }
    __syncthreads();
    if (bad >= 0) {
        if (threadIdx.x == 0) {
            hdr->status = GDN_ERR_DEVICE_CHECK;
            hdr->bad_index = bad;
        }
        return;
    }
    if (chunk_base) {
        // chunk_base = exclusive prefix sums of ceil(L_n / 64): each thread sums a
        // contiguous run of sequences, the block scans the run totals, and each
        // thread then writes its run's prefixes
        const int per = (num_seqs + kSchedThreads - 1) / kSchedThreads;
        const int n0 = min(num_seqs, int(threadIdx.x) * per), n1 = min(num_seqs, n0 + per);
        int local = 0;
        for (int n = n0; n < n1; ++n) local += (len[n] + 63) / 64;
        part[threadIdx.x] = local;
        __syncthreads();
        for (int d = 1; d < kSchedThreads; d <<= 1) {  // inclusive Hillis-Steele scan
            const int add = threadIdx.x >= unsigned(d) ? part[threadIdx.x - d] : 0;
            __syncthreads();
            part[threadIdx.x] += add;
            __syncthreads();
        }
        int run = part[threadIdx.x] - local;
        for (int n = n0; n < n1; ++n) {
            chunk_base[n] = run;
            run += (len[n] + 63) / 64;
        }
        if (threadIdx.x == kSchedThreads - 1) {
            chunk_base[num_seqs] = part[kSchedThreads - 1];
            hdr->total_chunks = part[kSchedThreads - 1];
        }
    }
    // longest first, ties by index: rank(n) = #{m : L_m > L_n or (L_m == L_n and m < n)}
    const bool rank_it = cu != nullptr && num_seqs <= kMaxRankedSeqs;
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        if (!rank_it) {
            order[n] = n;
            continue;
        }
        const int ln = len[n];
        int r = 0;
        for (int m = 0; m < num_seqs; ++m) {
            const int lm = len[m];
            r += (lm > ln) || (lm == ln && m < n);
        }
        order[r] = n;
    }
}

cudaError_t launch_schedule(const gdn_shape_t &s, const int32_t *cu_seqlens, void *workspace,
                            cudaStream_t stream, int32_t *chunk_base) {
    const WsLayout L = ws_layout(s.num_seqs);
    char *ws = static_cast<char *>(workspace);
    const int32_t tokens = s.batch * s.seq_len;
    schedule_kernel<<<1, kSchedThreads, 0, stream>>>(
        s.num_seqs, tokens, cu_seqlens ? 0 : s.seq_len, cu_seqlens, reinterpret_cast<WsHeader *>(ws),
        reinterpret_cast<int32_t *>(ws + L.order_off), reinterpret_cast<int32_t *>(ws + L.start_off),
        reinterpret_cast<int32_t *>(ws + L.len_off), chunk_base);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
