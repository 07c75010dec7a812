// Token-to-expert permutation: a stable counting sort of the T*k (token, rank)
// pairs by expert, then a gather of the activation rows into expert order.
//
// The pages only say a token's activations go to a few routed experts
// (winzheng.com page, section "Why Now of All Times"); this is the dispatch that
// makes the grouped expert GEMM possible. All integer outputs are exact and
// deterministic (no atomics decide an order):
//   count   : per 1024-pair chunk, a shared-memory histogram -> counts[c][e]
//   scan    : one block: offsets = exclusive scan of the totals, and the base of
//             every (chunk, expert) = offsets[e] + counts of earlier chunks
//   scatter : per chunk, the rank of a pair among equal experts of earlier
//             pairs (warp match + per-warp counts), giving its row
//   gather  : x_perm[r] = x[sorted_pair[r] / k], 16 bytes per thread, with the
//             8-column groups stored in the operand order 0,4,1,5,2,6,3,7
#include "common.cuh"
#include "internal.h"
#include "permute_small.cuh"

namespace moe {

constexpr int kChunk = 1024;

size_t permute_ws_bytes(int T, int k, int E) {
    const int P = T * k;
    const int C = (P + kChunk - 1) / kChunk;
    return align_up((size_t)C * E * sizeof(int32_t), 256) * 2;   // counts + bases
}

__global__ void __launch_bounds__(kChunk) perm_count_kernel(const int32_t *__restrict__ idx, int P, int E,
                                                           int32_t *__restrict__ counts) {
    extern __shared__ int32_t hist[];
    pdl_wait();
    pdl_release();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int p = blockIdx.x * kChunk + threadIdx.x;
    if (p < P) {
        const int e = idx[p];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else flag_error(2);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One block. Thread e walks the chunks of expert e; a block scan gives offsets.
__global__ void __launch_bounds__(kMaxExperts) perm_scan_kernel(const int32_t *__restrict__ counts, int C, int E,
                                                               int P, int32_t *__restrict__ bases,
                                                               int32_t *__restrict__ offsets) {
    __shared__ int32_t tot[kMaxExperts];
    __shared__ int32_t warp_sums[32];
    pdl_wait();
    pdl_release();
    const int e = threadIdx.x;
    int run = 0;
    if (e < E) {
        for (int c = 0; c < C; ++c) {
            bases[(int64_t)c * E + e] = run;
            run += counts[(int64_t)c * E + e];
        }
    }
    // exclusive scan of run over e
    const int lane = e & 31, wid = e >> 5;
    int incl = (e < E) ? run : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int ws = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ws, d);
            if (lane >= d) ws += v;
        }
        warp_sums[lane] = ws;   // inclusive
    }
    __syncthreads();
    const int excl = incl - ((e < E) ? run : 0) + (wid > 0 ? warp_sums[wid - 1] : 0);
    if (e < E) {
        offsets[e] = excl;
        tot[e] = excl;
    }
    if (e == 0) offsets[E] = P;
    __syncthreads();
    if (e < E)
        for (int c = 0; c < C; ++c) bases[(int64_t)c * E + e] += tot[e];
}

__global__ void __launch_bounds__(kChunk) perm_scatter_kernel(const int32_t *__restrict__ idx, int P, int E,
                                                             const int32_t *__restrict__ bases,
                                                             int32_t *__restrict__ sorted_pair,
                                                             int32_t *__restrict__ pair_row) {
    extern __shared__ int32_t wcnt[];   // [32 warps][E]
    pdl_wait();
    pdl_release();
    const int nw = kChunk / 32;
    for (int i = threadIdx.x; i < nw * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int p = blockIdx.x * kChunk + threadIdx.x;
    int e = (p < P) ? idx[p] : -1 - lane;   // padding lanes never match a real expert
    if (p < P && (e < 0 || e >= E)) e = -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank_w == 0) wcnt[wid * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
        int rank = rank_w;
        for (int w2 = 0; w2 < wid; ++w2) rank += wcnt[w2 * E + e];
        const int dst = bases[(int64_t)blockIdx.x * E + e] + rank;
        sorted_pair[dst] = p;
        pair_row[p] = dst;
    }
}

// Small batches (P <= kSmallP, E <= kSmallE): the whole counting sort in one
// block of kChunk threads (permute_small.cuh).
__global__ void __launch_bounds__(kChunk) perm_small_kernel(const int32_t *__restrict__ idx, int P, int E,
                                                           int32_t *__restrict__ offsets,
                                                           int32_t *__restrict__ sorted_pair,
                                                           int32_t *__restrict__ pair_row) {
    __shared__ SmallPermuteSmem<kChunk> sm;
    extern __shared__ int32_t sidx[];   // [P]
    pdl_wait();
    pdl_release();
    small_permute<kChunk>(idx, P, E, offsets, sorted_pair, pair_row, sm, sidx);
}

// Workspace bytes launch_permute actually uses for these sizes: none on the
// one-block path, else the per-chunk counters and bases.
size_t permute_scratch_bytes(int T, int k, int E) {
    const int64_t P = (int64_t)T * k;
    if (P == 0 || (P <= kSmallP && E <= kSmallE)) return 0;
    const int64_t C = (P + kChunk - 1) / kChunk;
    return align_up((size_t)C * E * sizeof(int32_t), 256) * 2;
}

__global__ void __launch_bounds__(256) perm_gather_kernel(const uint4 *__restrict__ x, int H8, int k,
                                                         const int32_t *__restrict__ sorted_pair, int P,
                                                         uint4 *__restrict__ x_perm, int natural) {
    pdl_wait();
    pdl_release();
    const int64_t total = (int64_t)P * H8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / H8;
        const int c = (int)(i - r * H8);
        const int t = sorted_pair[r] / k;
        const uint4 v = x[(int64_t)t * H8 + c];
        x_perm[i] = natural ? v : interleave8(v);
    }
}

moe_status launch_permute(const int32_t *idx, int T, int k, int E, const void *x, int H, int32_t *offsets,
                          int32_t *sorted_pair, int32_t *pair_row, void *x_perm, void *ws, size_t ws_bytes,
                          cudaStream_t st, int natural) {
    const int P = T * k;
    if (P == 0) {
        cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "memset offsets");
    }
    cudaError_t e;
    if (P <= kSmallP && E <= kSmallE) {
        e = ensure_max_smem<perm_small_kernel>((int)(kSmallP * sizeof(int32_t)));
        if (e == cudaSuccess)
            e = launch_pdl(perm_small_kernel, dim3(1), dim3(kChunk), (size_t)P * sizeof(int32_t), st, idx, P, E,
                           offsets, sorted_pair, pair_row);
        if (e != cudaSuccess) return set_cuda_error(e, "permute launch");
    } else {
        const int C = (P + kChunk - 1) / kChunk;
        const size_t half = align_up((size_t)C * E * sizeof(int32_t), 256);
        if (ws_bytes < 2 * half) return set_error(MOE_ERR_OOM, "permute workspace too small");
        int32_t *counts = reinterpret_cast<int32_t *>(ws);
        int32_t *bases = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + half);
        e = launch_pdl(perm_count_kernel, dim3(C), dim3(kChunk), E * sizeof(int32_t), st, idx, P, E, counts);
        if (e == cudaSuccess)
            e = launch_pdl(perm_scan_kernel, dim3(1), dim3(kMaxExperts), 0, st, (const int32_t *)counts, C, E, P, bases,
                           offsets);
        if (e != cudaSuccess) return set_cuda_error(e, "permute launch");
        const size_t sm_scatter = (size_t)(kChunk / 32) * E * sizeof(int32_t);
        if (sm_scatter > 48 * 1024) {
            e = cudaFuncSetAttribute(perm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sm_scatter);
            if (e != cudaSuccess) return set_cuda_error(e, "scatter smem attribute");
        }
        e = launch_pdl(perm_scatter_kernel, dim3(C), dim3(kChunk), sm_scatter, st, idx, P, E, (const int32_t *)bases,
                       sorted_pair, pair_row);
        if (e != cudaSuccess) return set_cuda_error(e, "permute launch");
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "permute launch");
    if (x_perm) {
        const int H8 = H / 8;
        const int64_t total = (int64_t)P * H8;
        int blocks = (int)((total + 255) / 256);
        if (blocks > 148 * 16) blocks = 148 * 16;
        e = launch_pdl(perm_gather_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4 *>(x), H8, k,
                       (const int32_t *)sorted_pair, P, reinterpret_cast<uint4 *>(x_perm), natural);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return set_cuda_error(e, "gather launch");
    }
    return MOE_OK;
}

}  // namespace moe
