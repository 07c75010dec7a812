// One-block counting sort of the token-to-expert pairs (the permutation step),
// for P <= kSmallP pairs and E <= kSmallE experts, run by every thread of one
// block of NT threads (NT a multiple of 32, NT >= E). Used by perm_small_kernel
// and by the router's last cluster when the layer fuses routing and
// permutation.
//
// idx is read from global memory once, into sidx (shared, P entries). Histogram,
// exclusive scan over the experts, then the pairs in chunks of NT in order: each pair lands at its expert's running position + its rank among the
// equal experts of earlier warps of the chunk + its rank inside its warp, which
// is the stable order (by pair index) within every expert.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kSmallP = 8192;
constexpr int kSmallE = 256;

// Shared scratch of small_permute for a block of NT threads.
template <int NT>
struct SmallPermuteSmem {
    int32_t cnt[kSmallE];
    int32_t run[kSmallE];
    int32_t wsum[32];
    int32_t wcnt[NT / 32][kSmallE];
};

// idx is read through L2 (__ldcg): in the fused case other CTAs of the same
// kernel wrote it. Entries outside [0, E) set the device error word and are
// left out (sidx holds -1 for them).
template <int NT>
__device__ void small_permute(const int32_t *idx, int P, int E, int32_t *__restrict__ offsets,
                              int32_t *__restrict__ sorted_pair, int32_t *__restrict__ pair_row,
                              SmallPermuteSmem<NT> &s, int32_t *sidx) {
    static_assert(NT % 32 == 0 && NT >= kSmallE && NT <= 1024, "block size");
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // into shared memory, up to 8 loads per thread in flight; the counters are cleared
    // meanwhile (the histogram starts after the barrier)
    for (int p0 = 0; p0 < P; p0 += 8 * NT) {
        int ev[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int p = p0 + tid + i * NT;
            ev[i] = p < P ? __ldcg(idx + p) : 0;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int p = p0 + tid + i * NT;
            if (p < P) sidx[p] = ev[i];
        }
    }
    for (int e = tid; e < E; e += NT) s.cnt[e] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += NT) {
        const int e = sidx[p];
        if (e >= 0 && e < E) {
            atomicAdd(&s.cnt[e], 1);
        } else {
            flag_error(2);
            sidx[p] = -1;
        }
    }
    __syncthreads();
    // exclusive scan over experts (E <= NT: one expert per thread)
    const int c = (tid < E) ? s.cnt[tid] : 0;
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) s.wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int t = lane < NT / 32 ? s.wsum[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += v;
        }
        s.wsum[lane] = t;   // inclusive over warps
    }
    __syncthreads();
    if (tid < E) {
        const int excl = incl - c + (wid > 0 ? s.wsum[wid - 1] : 0);
        offsets[tid] = excl;
        s.run[tid] = excl;
    }
    if (tid == 0) offsets[E] = P;
    for (int c0 = 0; c0 < P; c0 += NT) {
        for (int i = tid; i < (NT / 32) * E; i += NT) s.wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int p = c0 + tid;
        int e = (p < P) ? sidx[p] : -1;
        if (e < 0) e = -1 - lane;   // never matches a real expert
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank_w = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && rank_w == 0) s.wcnt[wid][e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int rank = s.run[e] + rank_w;
            for (int w2 = 0; w2 < wid; ++w2) rank += s.wcnt[w2][e];
            sorted_pair[rank] = p;
            pair_row[p] = rank;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += NT) {
            int add = 0;
            for (int w2 = 0; w2 < NT / 32; ++w2) add += s.wcnt[w2][ee];
            s.run[ee] += add;
        }
        __syncthreads();
    }
}

}  // namespace moe
