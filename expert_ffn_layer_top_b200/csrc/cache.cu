// Device LRU expert cache with host->device streaming of misses and of the
// next layer's experts.
//
// Source: winzheng.com page, sections "Why Now of All Times" (most experts stay
// in host memory and are loaded on demand) and "FreeToken's Three-Layer
// Mechanism" (double-buffered streaming overlapped with compute, a global LRU
// expert cache reusing high-frequency experts, transfers sized to the bandwidth
// measured); aimodeling.com English page, section "Three Engineering Cores"
// (full-layer double-buffered prefill streaming, the global LRU cache, elastic
// memory management without weight reloads).
//
// Pool. A reserved virtual address range (the device's memory size) backed by
// physical chunks mapped on demand, so the pool grows and shrinks in place; a
// slot holds one expert's w13 codes, w13 scales, w2 codes and w2 scales at
// fixed 256-byte-aligned offsets, and the grouped FFN reads cached experts
// through the same strided descriptor as resident ones, with expert_map = the
// slot of each expert. Where reserved addresses are not available the pool is
// one ordinary allocation and resizing stays within it.
//
// Table (device): slot_of[L*E], owner, an intrusive LRU list (prev/next, head =
// least recent), ref_call (index of the last call that referenced the slot), a
// free-slot bitmap, per-layer bitmaps and pair counts of the experts used at
// the last step (the prefetch prediction) and counters. One warp runs a call:
// lanes build the request bitmap, the pair counts and the next layer's
// prefetch request; lane 0 walks the request in ascending expert order:
//   hit  -> move to the most-recent end;
//   miss -> lowest free slot, else the least recent slot not referenced by
//           this call or the previous one (those may still be in use);
// a call that cannot fit fails with CACHE_FULL before changing anything.
// The (expert, slot) loads go to page-locked mapped host memory; the host
// reads them after one event wait and issues one cudaMemcpyAsync per array
// on the cache's copy stream. The layer's GEMM waits on an event recorded
// after its own loads; the loads for the next layer are issued behind it on
// the copy stream, so they overlap this layer's GEMMs (the double buffering:
// the layer being computed and the layer being filled).
#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "lru_table.cuh"

namespace moe {

// Timing records: one per cached call, kTimedKinds events each, in a fixed ring
// created at init (no event is created on the hot path).
enum { TK_COPY_B = 0, TK_COPY_E, TK_TABLE_B, TK_TABLE_E, TK_COMP_B, TK_COMP_E, kTimedKinds };
constexpr int kTimerRing = 64;

// Driver entry points of the virtual memory management API.
struct VmmApi {
    CUresult (*reserve)(CUdeviceptr *, size_t, size_t, CUdeviceptr, unsigned long long) = nullptr;
    CUresult (*free_va)(CUdeviceptr, size_t) = nullptr;
    CUresult (*create)(CUmemGenericAllocationHandle *, size_t, const CUmemAllocationProp *,
                       unsigned long long) = nullptr;
    CUresult (*release)(CUmemGenericAllocationHandle) = nullptr;
    CUresult (*map)(CUdeviceptr, size_t, size_t, CUmemGenericAllocationHandle, unsigned long long) = nullptr;
    CUresult (*unmap)(CUdeviceptr, size_t) = nullptr;
    CUresult (*set_access)(CUdeviceptr, size_t, const CUmemAccessDesc *, size_t) = nullptr;
    CUresult (*granularity)(size_t *, const CUmemAllocationProp *, CUmemAllocationGranularity_flags) = nullptr;
    bool ok = false;
};

static const VmmApi &vmm_api() {
    static VmmApi api;
    static std::once_flag once;
    std::call_once(once, [] {
        auto get = [](const char *name, void **fn) {
            cudaDriverEntryPointQueryResult q;
            return cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess && *fn;
        };
        bool ok = true;
        ok &= get("cuMemAddressReserve", reinterpret_cast<void **>(&api.reserve));
        ok &= get("cuMemAddressFree", reinterpret_cast<void **>(&api.free_va));
        ok &= get("cuMemCreate", reinterpret_cast<void **>(&api.create));
        ok &= get("cuMemRelease", reinterpret_cast<void **>(&api.release));
        ok &= get("cuMemMap", reinterpret_cast<void **>(&api.map));
        ok &= get("cuMemUnmap", reinterpret_cast<void **>(&api.unmap));
        ok &= get("cuMemSetAccess", reinterpret_cast<void **>(&api.set_access));
        ok &= get("cuMemGetAllocationGranularity", reinterpret_cast<void **>(&api.granularity));
        api.ok = ok;
    });
    return api;
}

}  // namespace moe

struct expert_cache {
    int device = 0, n_layers = 0, E = 0, H = 0, I = 0, fmt = 0, layout = 0;
    size_t sz[4] = {0, 0, 0, 0};      // per-expert bytes: w13, w13 scales, w2, w2 scales
    size_t off[4] = {0, 0, 0, 0};     // offsets inside a slot
    size_t slot_bytes = 0;
    int n_slots = 0, max_slots = 0;
    // pool: reserved range with mapped chunks, or one plain allocation
    uint8_t *pool = nullptr;
    bool vmm = false;
    size_t va_bytes = 0, chunk_bytes = 0;
    std::vector<CUmemGenericAllocationHandle> chunks;   // mapped chunk i at pool + i * chunk_bytes
    // device table (one allocation starting at d_slot_of)
    int32_t *d_slot_of = nullptr, *d_owner = nullptr, *d_prev = nullptr, *d_next = nullptr, *d_ref = nullptr;
    uint32_t *d_free = nullptr, *d_last = nullptr;    // free bitmap [Smax/32], last-used bitmaps [L][E/32]
    int32_t *d_lastcnt = nullptr;                       // pairs per expert at the last resolve [L][E]
    int32_t *d_state = nullptr;                         // head, tail, calls, free_count, hint, last_nref
    unsigned long long *d_counts = nullptr;             // hits, misses
    float *d_ts13 = nullptr, *d_ts2 = nullptr;          // NVFP4 tensor scales [L][E]
    size_t table_bytes = 0;
    // mapped host buffers
    int32_t *h_io = nullptr, *d_io = nullptr;           // loads out / ids in
    int32_t *h_ev = nullptr, *d_ev = nullptr;           // eviction list of a rollback
    std::vector<moe_experts> layers;                    // host descriptions (host pointers)
    cudaStream_t cs = nullptr;
    cudaEvent_t ev_lru = nullptr, ev_res = nullptr;
    // prefetch policy
    int pf_policy = MOE_PREFETCH_PREDICTED, pf_depth = -1, last_depth = -1;
    // timing ring (see TK_*): event k of record r is ring[r * kTimedKinds + k]
    cudaEvent_t ev_ref = nullptr;
    std::vector<cudaEvent_t> ring;
    std::vector<unsigned> ring_mask;
    std::vector<uint64_t> ring_bytes;                   // bytes copied in the record
    int cur = -1, ring_head = 0, ring_used = 0;
    double last_comp_b = -1.0, last_comp_e = -1.0;      // previous compute interval (ms from ev_ref)
    std::vector<std::pair<double, double>> pending_copy;   // copy intervals later computes may overlap
    // counters
    uint64_t bytes_h2d = 0, copies = 0, calls = 0, prefetched = 0, moved = 0;
    double copy_s = 0.0, table_s = 0.0, compute_s = 0.0, overlap_s = 0.0, host_wait_s = 0.0, issue_s = 0.0;
    double bw_ewma = 0.0, comp_ewma = 0.0;              // bytes/s and seconds
    long fault_h2d_at = -1;                             // host fault injection: fail this copy (1-based)
};

namespace moe {

static double now_s() {
    return std::chrono::duration<double>(std::chrono::steady_clock::now().time_since_epoch()).count();
}

// Next-layer prefetch request for `layer` (bitmap pf[ceil(E/32)]), computed by the
// warp with the rule of lru_predict: every expert when `full`, else the first `depth`
// experts of the layer's prediction by rank key (depth < 0: all of it).
__device__ void lru_predict_warp(const LruTable &t, int layer, int depth, bool full, uint32_t *pf, uint32_t *keys) {
    const int lane = threadIdx.x & 31;
    const int words = (t.E + 31) / 32;
    const uint32_t *pred = t.last + layer * words;
    for (int w = lane; w < words; w += 32) {
        const int rem = t.E - w * 32;
        const uint32_t all = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        pf[w] = full ? all : (depth < 0 ? pred[w] : 0u);
    }
    __syncwarp();
    if (full || depth <= 0) return;
    // keys of the predicted experts (0 for the others), lane l holding experts l, l + 32, ...
    for (int e = lane; e < t.E; e += 32)
        keys[e] = ((pred[e >> 5] >> (e & 31)) & 1u) ? lru_rank_key(t.lastcnt[layer * t.E + e], e) : 0u;
    __syncwarp();
    uint32_t bound = 0xffffffffu;
    for (int j = 0; j < depth; ++j) {
        uint32_t best = 0u;
        for (int e = lane; e < t.E; e += 32) {
            const uint32_t k = keys[e];
            if (k < bound && k > best) best = k;
        }
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        if (m == 0u) break;
        const int be = 2047 - (int)(m & 2047u);
        if (lane == 0) pf[be >> 5] |= 1u << (be & 31);
        bound = m;
    }
    __syncwarp();
}

// Shared-memory image of the table for one update: the parts a call can touch (every
// layer's slot_of, last and lastcnt; owner, prev, next, ref and the free bitmap of the S
// slots in use; the state and counters), each padded to 16 bytes. The update then makes
// its dependent reads (about ten per requested expert) in shared memory.
struct LruStage {
    int n[10];        // words of each part: slot_of owner prev next ref freeb last lastcnt st counts
    int off[10];      // word offset of each part in the image
    int total;        // words
};
constexpr int kLruStageThreads = 512;
constexpr int kLruStageMaxBytes = 200 * 1024;

__host__ __device__ inline LruStage lru_stage(int L, int E, int S) {
    LruStage g;
    const int lw = (E + 31) / 32;
    const int n[10] = {L * E, S, S, S, S, (S + 31) / 32, L * lw, L * E, ST_N, 4};
    int o = 0;
    for (int i = 0; i < 10; ++i) {
        g.n[i] = (n[i] + 3) & ~3;
        g.off[i] = o;
        o += g.n[i];
    }
    g.total = o;
    return g;
}

// The table's arrays in the order of LruStage (base pointers).
__device__ inline void lru_parts(const LruTable &t, uint32_t **p) {
    p[0] = reinterpret_cast<uint32_t *>(t.slot_of);
    p[1] = reinterpret_cast<uint32_t *>(t.owner);
    p[2] = reinterpret_cast<uint32_t *>(t.prev);
    p[3] = reinterpret_cast<uint32_t *>(t.next);
    p[4] = reinterpret_cast<uint32_t *>(t.ref);
    p[5] = t.freeb;
    p[6] = t.last;
    p[7] = reinterpret_cast<uint32_t *>(t.lastcnt);
    p[8] = reinterpret_cast<uint32_t *>(t.st);
    p[9] = reinterpret_cast<uint32_t *>(t.counts);
}

// Global address of 16-byte chunk j of the image (j < g.total / 4).
__device__ inline uint4 *lru_stage_src(const LruStage &g, uint32_t *const *gp, int j) {
    int i = 0;
    while (i < 9 && j >= g.off[i + 1] / 4) ++i;
    return reinterpret_cast<uint4 *>(gp[i]) + (j - g.off[i] / 4);
}

// Copies the image in (in = true) or back, over all parts as one range of 16-byte chunks,
// eight in flight per thread. The parts start 256-byte aligned in global memory with room
// past each used end (their allocations are padded to 256 bytes, or hold max_slots >= S
// entries), and a word read past the end is written back unchanged.
__device__ inline void lru_stage_copy(const LruStage &g, uint32_t *const *gp, uint4 *img, bool in) {
    constexpr int kU = 8;
    const int n4 = g.total / 4;
    for (int j0 = threadIdx.x; j0 < n4; j0 += kU * blockDim.x) {
        uint4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * blockDim.x;
            if (j < n4) v[u] = in ? *lru_stage_src(g, gp, j) : img[j];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * blockDim.x;
            if (j < n4) {
                if (in) img[j] = v[u];
                else *lru_stage_src(g, gp, j) = v[u];
            }
        }
    }
}

// The update by one warp (lane = thread index): the request bitmap and pair counts of the
// call, the prediction of the next layer, then lane 0 runs the table's policy.
__device__ void lru_update_warp(LruTable &t, int layer, const int32_t *idx, int P, int mode, int pf_mode,
                                int depth, int32_t *io, uint32_t *req, uint32_t *pf, int32_t *cnt, uint32_t *keys) {
    const int lane = threadIdx.x;
    const int words = (t.E + 31) / 32;
    for (int w = lane; w < words; w += 32) req[w] = 0;
    for (int e = lane; e < t.E; e += 32) cnt[e] = 0;
    __syncwarp();
    int nids = 0;
    if (mode == 1) nids = io[0];
    __syncwarp();
    if (mode == 0) {
        for (int p = lane; p < P; p += 32) {
            const int e = idx[p];
            if (e >= 0 && e < t.E) {
                atomicOr(&req[e >> 5], 1u << (e & 31));
                atomicAdd(&cnt[e], 1);
            }
        }
    } else {
        for (int i = lane; i < nids; i += 32) {
            const int e = io[1 + i];
            if (e >= 0 && e < t.E) atomicOr(&req[e >> 5], 1u << (e & 31));
        }
    }
    __syncwarp();
    const bool pfn = mode == 0 && pf_mode != 0 && layer + 1 < t.L;
    if (pfn) lru_predict_warp(t, layer + 1, depth, pf_mode == 2, pf, keys);
    __syncwarp();
    if (lane == 0) lru_run(t, layer, req, mode == 0 ? cnt : nullptr, mode, pfn ? pf : nullptr, io);
}

// mode 0: resolve `layer` from idx[P]; then, unless pf_mode is 0, prefetch layer+1
//         (pf_mode 1: the first `depth` of its prediction, depth < 0 all; 2: every expert)
// mode 1: prefetch `layer` with the explicit ids in io (count io[0], ids io[1..])
// Output in io: [0] status (0 ok, 6 cache full), [1] n resolve loads, [2] n prefetch loads
// (-1 = not run or full), then the pairs.
// staged: the block (kLruStageThreads threads) copies the table into dynamic shared
// memory (lru_stage), warp 0 updates it there, and the block copies it back; otherwise
// one warp updates the table in global memory. The table was last written by the update
// before (several kernels back), so it is read before the wait on the kernel just before,
// which writes idx.
__global__ void __launch_bounds__(kLruStageThreads) lru_kernel(LruTable tg, int layer, const int32_t *idx, int P,
                                                               int mode, int pf_mode, int depth, int32_t *io,
                                                               int staged) {
    __shared__ uint32_t req[kMaxExperts / 32];
    __shared__ uint32_t pf[kMaxExperts / 32];
    __shared__ int32_t cnt[kMaxExperts];
    __shared__ uint32_t keys[kMaxExperts];
    extern __shared__ uint4 img[];
    LruTable t = tg;
    LruStage g;
    uint32_t *gp[10];
    if (staged) {
        g = lru_stage(tg.L, tg.E, tg.S);
        lru_parts(tg, gp);
        lru_stage_copy(g, gp, img, true);
        uint32_t *w = reinterpret_cast<uint32_t *>(img);
        t.slot_of = reinterpret_cast<int32_t *>(w + g.off[0]);
        t.owner = reinterpret_cast<int32_t *>(w + g.off[1]);
        t.prev = reinterpret_cast<int32_t *>(w + g.off[2]);
        t.next = reinterpret_cast<int32_t *>(w + g.off[3]);
        t.ref = reinterpret_cast<int32_t *>(w + g.off[4]);
        t.freeb = w + g.off[5];
        t.last = w + g.off[6];
        t.lastcnt = reinterpret_cast<int32_t *>(w + g.off[7]);
        t.st = reinterpret_cast<int32_t *>(w + g.off[8]);
        t.counts = reinterpret_cast<unsigned long long *>(w + g.off[9]);
    }
    pdl_wait();
    if (staged) __syncthreads();
    if (threadIdx.x < 32) lru_update_warp(t, layer, idx, P, mode, pf_mode, depth, io, req, pf, cnt, keys);
    if (staged) {
        __syncthreads();
        lru_stage_copy(g, gp, img, false);
    }
}

__global__ void lru_init_kernel(LruTable t) { lru_init_one(t, blockIdx.x * blockDim.x + threadIdx.x); }

// Free slots matching (layer, ids) (see lru_evict).
__global__ void lru_evict_kernel(LruTable t, int layer, const int32_t *io) {
    if (threadIdx.x == 0) lru_evict(t, layer, io);
}

// Table pointers inside a table block at `b` (device block or its host copy).
static LruTable table_at(const expert_cache *c, uint8_t *b) {
    const int L = c->n_layers, E = c->E, lw = (E + 31) / 32;
    const size_t Sm = (size_t)c->max_slots;
    size_t p = 0;
    auto take = [&](size_t bytes) { uint8_t *r = b + p; p += align_up(bytes, 256); return r; };
    LruTable t;
    t.slot_of = reinterpret_cast<int32_t *>(take((size_t)L * E * 4));
    t.owner = reinterpret_cast<int32_t *>(take(Sm * 4));
    t.prev = reinterpret_cast<int32_t *>(take(Sm * 4));
    t.next = reinterpret_cast<int32_t *>(take(Sm * 4));
    t.ref = reinterpret_cast<int32_t *>(take(Sm * 4));
    t.freeb = reinterpret_cast<uint32_t *>(take((Sm + 31) / 32 * 4));
    t.last = reinterpret_cast<uint32_t *>(take((size_t)L * lw * 4));
    t.lastcnt = reinterpret_cast<int32_t *>(take((size_t)L * E * 4));
    t.st = reinterpret_cast<int32_t *>(take(256));
    t.counts = reinterpret_cast<unsigned long long *>(take(256));
    t.S = c->n_slots;
    t.E = E;
    t.L = L;
    t.Smax = c->max_slots;
    return t;
}

static size_t table_block_bytes(int L, int E, int Smax) {
    const size_t lw = (size_t)(E + 31) / 32, Sm = (size_t)Smax;
    size_t tb = 0;
    tb += align_up((size_t)L * E * 4, 256);            // slot_of
    tb += 4 * align_up(Sm * 4, 256);                    // owner prev next ref
    tb += align_up((Sm + 31) / 32 * 4, 256);            // free bitmap
    tb += align_up((size_t)L * lw * 4, 256);            // last-used bitmaps
    tb += align_up((size_t)L * E * 4, 256);             // last pair counts
    tb += 256 + 256;                                    // state, counters
    return tb;
}

static LruTable table_of(expert_cache *c) { return table_at(c, reinterpret_cast<uint8_t *>(c->d_slot_of)); }

// Launches the table update: staged in shared memory when the image fits, else one warp
// on the table in global memory.
static cudaError_t launch_lru(expert_cache *c, int layer, const int32_t *idx, int P, int mode, int pf_mode,
                              int depth, cudaStream_t st) {
    const LruTable t = table_of(c);
    const size_t bytes = (size_t)lru_stage(t.L, t.E, t.S).total * 4;
    cudaError_t e;
    if (bytes <= (size_t)kLruStageMaxBytes && ensure_max_smem<lru_kernel>((int)bytes) == cudaSuccess)
        e = launch_pdl(lru_kernel, dim3(1), dim3(kLruStageThreads), bytes, st, t, layer, idx, P, mode, pf_mode, depth,
                       c->d_io, 1);
    else
        e = launch_pdl(lru_kernel, dim3(1), dim3(32), 0, st, t, layer, idx, P, mode, pf_mode, depth, c->d_io, 0);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

static size_t part_bytes(int fmt, int rows, int K, bool scale) {
    if (scale) return (size_t)rows * scale_rowbytes(fmt, K);
    const size_t n = (size_t)rows * K;
    return fmt == MOE_BF16 ? 2 * n : fmt == MOE_FP8_E4M3_K128 ? n : n / 2;
}

static int64_t host_stride(const moe_experts &x, int part, size_t dense) {
    const int64_t s[4] = {x.w13_estride, x.w13s_estride, x.w2_estride, x.w2s_estride};
    return s[part] ? s[part] : (int64_t)dense;
}

// ------------------------------------------------------------------ pool chunks

static size_t mapped_bytes(const expert_cache *c) { return c->chunks.size() * c->chunk_bytes; }

// Map chunks until `bytes` of the range are backed. On failure the chunks mapped by
// this call are released again.
static moe_status map_to(expert_cache *c, size_t bytes) {
    const VmmApi &v = vmm_api();
    const size_t had = c->chunks.size();
    CUmemAllocationProp prop = {};
    prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
    prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    prop.location.id = c->device;
    CUmemAccessDesc acc = {};
    acc.location = prop.location;
    acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;
    while (mapped_bytes(c) < bytes) {
        const CUdeviceptr at = reinterpret_cast<CUdeviceptr>(c->pool) + mapped_bytes(c);
        CUmemGenericAllocationHandle h;
        CUresult r = v.create(&h, c->chunk_bytes, &prop, 0);
        if (r == CUDA_SUCCESS) {
            r = v.map(at, c->chunk_bytes, 0, h, 0);
            if (r == CUDA_SUCCESS) {
                r = v.set_access(at, c->chunk_bytes, &acc, 1);
                if (r != CUDA_SUCCESS) v.unmap(at, c->chunk_bytes);
            }
            if (r != CUDA_SUCCESS) v.release(h);
        }
        if (r != CUDA_SUCCESS) {
            while (c->chunks.size() > had) {
                const CUdeviceptr a = reinterpret_cast<CUdeviceptr>(c->pool) + (c->chunks.size() - 1) * c->chunk_bytes;
                v.unmap(a, c->chunk_bytes);
                v.release(c->chunks.back());
                c->chunks.pop_back();
            }
            return set_error(r == CUDA_ERROR_OUT_OF_MEMORY ? MOE_ERR_OOM : MOE_ERR_CUDA,
                             "mapping pool chunk %zu failed (%d)", c->chunks.size(), (int)r);
        }
        c->chunks.push_back(h);
    }
    return MOE_OK;
}

// Unmap the chunks wholly past `bytes` (no kernel or copy may be using them).
static void unmap_past(expert_cache *c, size_t bytes) {
    const VmmApi &v = vmm_api();
    const size_t keep = (bytes + c->chunk_bytes - 1) / c->chunk_bytes;
    while (c->chunks.size() > keep) {
        const CUdeviceptr a = reinterpret_cast<CUdeviceptr>(c->pool) + (c->chunks.size() - 1) * c->chunk_bytes;
        v.unmap(a, c->chunk_bytes);
        v.release(c->chunks.back());
        c->chunks.pop_back();
    }
}

// ------------------------------------------------------------------ timing

// Milliseconds from the reference event to event `kind` of record `rec` (positions, for
// the overlap), and between two events of a record (durations, at full resolution).
static double ev_ms(expert_cache *c, int rec, int kind) {
    float ms = 0.f;
    cudaEventElapsedTime(&ms, c->ev_ref, c->ring[rec * kTimedKinds + kind]);
    return (double)ms;
}
static double ev_dur_ms(expert_cache *c, int rec, int kb, int ke) {
    float ms = 0.f;
    cudaEventElapsedTime(&ms, c->ring[rec * kTimedKinds + kb], c->ring[rec * kTimedKinds + ke]);
    return (double)ms;
}

static void add_overlap(expert_cache *c, double cb, double ce) {
    for (auto &iv : c->pending_copy) {
        const double lo = std::max(iv.first, cb), hi = std::min(iv.second, ce);
        if (hi > lo) c->overlap_s += (hi - lo) * 1e-3;
    }
    // compute intervals arrive in time order: a copy that ended before this one
    // began cannot overlap a later one
    c->pending_copy.erase(std::remove_if(c->pending_copy.begin(), c->pending_copy.end(),
                                         [&](const std::pair<double, double> &iv) { return iv.second <= cb; }),
                          c->pending_copy.end());
}

// Read back the oldest records whose events have all completed (or, with `block`, the
// oldest one in any case).
static void harvest(expert_cache *c, bool block) {
    while (c->ring_used > 0) {
        const int r = c->ring_head;
        if (r == c->cur) break;   // still being recorded
        const unsigned m = c->ring_mask[r];
        bool done = true;
        for (int k = 0; k < kTimedKinds && done; ++k) {
            if (!(m & (1u << k))) continue;
            cudaEvent_t ev = c->ring[r * kTimedKinds + k];
            if (block) cudaEventSynchronize(ev);
            done = cudaEventQuery(ev) == cudaSuccess;
        }
        if (!done) break;
        block = false;
        const unsigned copy = (1u << TK_COPY_B) | (1u << TK_COPY_E);
        const unsigned table = (1u << TK_TABLE_B) | (1u << TK_TABLE_E);
        const unsigned comp = (1u << TK_COMP_B) | (1u << TK_COMP_E);
        if ((m & table) == table) c->table_s += ev_dur_ms(c, r, TK_TABLE_B, TK_TABLE_E) * 1e-3;
        if ((m & copy) == copy) {
            const double d = ev_dur_ms(c, r, TK_COPY_B, TK_COPY_E);
            const double b = ev_ms(c, r, TK_COPY_B), e = b + d;
            if (d > 0) {
                c->copy_s += d * 1e-3;
                if (c->ring_bytes[r] > 0) {
                    const double bw = c->ring_bytes[r] / (d * 1e-3);
                    c->bw_ewma = c->bw_ewma > 0 ? 0.75 * c->bw_ewma + 0.25 * bw : bw;
                }
                // an earlier call's compute may still have been running when these copies began
                if (c->last_comp_e > b) {
                    const double lo = std::max(b, c->last_comp_b), hi = std::min(e, c->last_comp_e);
                    if (hi > lo) c->overlap_s += (hi - lo) * 1e-3;
                }
                c->pending_copy.emplace_back(b, e);
            }
        }
        if ((m & comp) == comp) {
            const double d = ev_dur_ms(c, r, TK_COMP_B, TK_COMP_E);
            const double b = ev_ms(c, r, TK_COMP_B), e = b + d;
            if (d > 0) {
                c->compute_s += d * 1e-3;
                c->comp_ewma = c->comp_ewma > 0 ? 0.75 * c->comp_ewma + 0.25 * d * 1e-3 : d * 1e-3;
                add_overlap(c, b, e);
                c->last_comp_b = b;
                c->last_comp_e = e;
            }
        }
        c->ring_head = (c->ring_head + 1) % kTimerRing;
        --c->ring_used;
    }
    if (c->pending_copy.size() > 256) c->pending_copy.erase(c->pending_copy.begin(), c->pending_copy.end() - 256);
}

// Open the timing record of a call (the oldest record is read back first if the ring is full).
static void timer_open(expert_cache *c) {
    if (c->ring_used == kTimerRing) harvest(c, true);
    if (c->ring_used == kTimerRing) { c->cur = -1; return; }
    c->cur = (c->ring_head + c->ring_used) % kTimerRing;
    ++c->ring_used;
    c->ring_mask[c->cur] = 0;
    c->ring_bytes[c->cur] = 0;
}

static void timer_mark(expert_cache *c, int kind, cudaStream_t st) {
    if (c->cur < 0) return;
    if (cudaEventRecord(c->ring[c->cur * kTimedKinds + kind], st) == cudaSuccess) c->ring_mask[c->cur] |= 1u << kind;
}

static void timer_close(expert_cache *c) { c->cur = -1; }

// ------------------------------------------------------------------ loads

// Issue the copies of `n` loads (pairs e, slot) of `layer` on the copy stream.
// *done: loads whose copies were all enqueued.
static moe_status issue_loads(expert_cache *c, int layer, const int32_t *pairs, int n, int *done) {
    const moe_experts &x = c->layers[layer];
    const void *src[4] = {x.w13, x.w13_scale, x.w2, x.w2_scale};
    *done = 0;
    for (int i = 0; i < n; ++i) {
        const int e = pairs[2 * i], s = pairs[2 * i + 1];
        for (int part = 0; part < 4; ++part) {
            if (!c->sz[part]) continue;
            ++c->copies;
            if (c->fault_h2d_at > 0 && (long)c->copies == c->fault_h2d_at)
                return set_error(MOE_ERR_CUDA, "injected host-to-device copy failure (copy %lu)", (unsigned long)c->copies);
            const uint8_t *from = reinterpret_cast<const uint8_t *>(src[part]) + (int64_t)e * host_stride(x, part, c->sz[part]);
            uint8_t *to = c->pool + (size_t)s * c->slot_bytes + c->off[part];
            cudaError_t er = cudaMemcpyAsync(to, from, c->sz[part], cudaMemcpyHostToDevice, c->cs);
            if (er != cudaSuccess) return set_cuda_error(er, "expert copy");
            c->bytes_h2d += c->sz[part];
            if (c->cur >= 0) c->ring_bytes[c->cur] += c->sz[part];
        }
        *done = i + 1;
    }
    return MOE_OK;
}

// After a failed load: free the table entries of the loads whose copies were not all
// enqueued (pairs[from..n) of `layer`), so no later call takes their slots for resident.
static void rollback(expert_cache *c, int layer, const int32_t *pairs, int from, int n, cudaStream_t st) {
    if (from >= n || layer >= c->n_layers) return;
    c->h_ev[0] = n - from;
    for (int i = from; i < n; ++i) c->h_ev[1 + i - from] = pairs[2 * i];
    count_launch();
    lru_evict_kernel<<<1, 32, 0, st>>>(table_of(c), layer, c->d_ev);
    if (cudaGetLastError() == cudaSuccess) cudaStreamSynchronize(st);
}

moe_status cache_resolve_and_map(expert_cache *c, int layer, const int32_t *idx, int T, int k,
                                 const moe_experts *shape, moe_experts *view, cudaStream_t st) {
    if (layer < 0 || layer >= c->n_layers) return set_error(MOE_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (shape->E != c->E || shape->H != c->H || shape->I != c->I || shape->fmt != c->fmt)
        return set_error(MOE_ERR_INVALID_ARG, "layer shape differs from the cache's");
    bool full = false, none = false;
    const double expert_bytes = (double)(c->sz[0] + c->sz[1] + c->sz[2] + c->sz[3]);
    int depth = lru_prefetch_plan(c->pf_policy, c->pf_depth, T, k, c->E, c->bw_ewma, c->comp_ewma, expert_bytes,
                                  &full, &none);
    c->last_depth = none ? 0 : (full ? c->E : depth);
    const int pf_mode = none ? 0 : (full ? 2 : 1);
    harvest(c, false);
    timer_open(c);
    ++c->calls;
    timer_mark(c, TK_TABLE_B, st);
    cudaError_t e = launch_lru(c, layer, idx, T * k, 0, pf_mode, depth, st);
    timer_mark(c, TK_TABLE_E, st);
    const double t0 = now_s();
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_lru, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_lru);
    const double t1 = now_s();
    c->host_wait_s += t1 - t0;
    if (e != cudaSuccess) { timer_close(c); return set_cuda_error(e, "cache table update"); }
    const int32_t *io = c->h_io;
    if (io[0] == MOE_ERR_CACHE_FULL) {
        timer_close(c);
        return set_error(MOE_ERR_CACHE_FULL, "layer %d needs more slots than the cache can free", layer);
    }
    const int na = io[1], nb = io[2];
    // keep the pairs: a rollback reuses the mapped buffers
    std::vector<int32_t> pairs(io + 3, io + 3 + 2 * (na + (nb > 0 ? nb : 0)));
    moe_status r = MOE_OK;
    int done_a = 0, done_b = 0;
    timer_mark(c, TK_COPY_B, c->cs);
    r = issue_loads(c, layer, pairs.data(), na, &done_a);
    if (r == MOE_OK && (e = cudaEventRecord(c->ev_res, c->cs)) != cudaSuccess) r = set_cuda_error(e, "event");
    if (r == MOE_OK && nb > 0) {
        r = issue_loads(c, layer + 1, pairs.data() + 2 * na, nb, &done_b);
        c->prefetched += (uint64_t)done_b;
    }
    timer_mark(c, TK_COPY_E, c->cs);
    c->issue_s += now_s() - t1;
    if (r != MOE_OK) {
        timer_close(c);
        const std::string msg = moe_last_error_string();
        rollback(c, layer, pairs.data(), done_a, na, st);
        if (nb > 0) rollback(c, layer + 1, pairs.data() + 2 * na, done_b, nb, st);
        return set_error(r, "%s", msg.c_str());
    }
    if ((e = cudaStreamWaitEvent(st, c->ev_res, 0)) != cudaSuccess) {
        timer_close(c);
        return set_cuda_error(e, "stream wait");
    }
    *view = *shape;
    view->w13 = c->pool + c->off[0];
    view->w13_scale = c->sz[1] ? c->pool + c->off[1] : nullptr;
    view->w2 = c->pool + c->off[2];
    view->w2_scale = c->sz[3] ? c->pool + c->off[3] : nullptr;
    view->w13_estride = view->w13s_estride = view->w2_estride = view->w2s_estride = (int64_t)c->slot_bytes;
    view->expert_map = c->d_slot_of + (size_t)layer * c->E;
    view->n_entries = c->n_slots;
    view->layout = c->layout;
    if (c->fmt == MOE_NVFP4) {
        view->w13_tscale = c->d_ts13 + (size_t)layer * c->E;
        view->w2_tscale = c->d_ts2 + (size_t)layer * c->E;
    }
    timer_mark(c, TK_COMP_B, st);
    return MOE_OK;
}

// Called by the layer forward once the cached layer's FFN and combine are enqueued.
void cache_compute_end(expert_cache *c, cudaStream_t st) {
    timer_mark(c, TK_COMP_E, st);
    timer_close(c);
}

int cache_layout(const struct expert_cache *c) { return c->layout; }

}  // namespace moe

using namespace moe;

extern "C" {

moe_status expert_cache_init(struct expert_cache **out, size_t capacity_bytes, int n_layers,
                             const moe_experts *host_layers, int device) {
    if (!out || !host_layers || n_layers <= 0) return set_error(MOE_ERR_INVALID_ARG, "bad cache arguments");
    *out = nullptr;
    const moe_experts &l0 = host_layers[0];
    if (l0.fmt < MOE_BF16 || l0.fmt > MOE_NVFP4 || l0.E <= 0 || l0.E > kMaxExperts || l0.H <= 0 || l0.I <= 0 ||
        l0.H % 256 || l0.I % 256)
        return set_error(MOE_ERR_UNSUPPORTED, "unsupported layer shape for the cache");
    for (int l = 1; l < n_layers; ++l) {
        const moe_experts &x = host_layers[l];
        if (x.fmt != l0.fmt || x.E != l0.E || x.H != l0.H || x.I != l0.I || x.layout != l0.layout)
            return set_error(MOE_ERR_INVALID_ARG, "cache layers must share format and shape");
    }
    const char *fault = getenv("MOE_FAULT");
    if (fault && strcmp(fault, "pin_alloc") == 0) return set_error(MOE_ERR_OOM, "injected page-locked allocation failure");
    cudaError_t e = cudaSetDevice(device);
    if (e != cudaSuccess) return set_cuda_error(e, "set device");
    expert_cache *c = new expert_cache();
    c->device = device;
    c->n_layers = n_layers;
    c->E = l0.E;
    c->H = l0.H;
    c->I = l0.I;
    c->fmt = l0.fmt;
    c->layers.assign(host_layers, host_layers + n_layers);
    if (fault && strncmp(fault, "h2d_fail@", 9) == 0) c->fault_h2d_at = atol(fault + 9);
    const int fmt = l0.fmt;
    c->layout = l0.layout;
    if (c->layout == MOE_LAYOUT_TILED) {   // scales travel inside the prepacked blobs
        c->sz[0] = prepacked_expert_bytes(fmt, c->H, c->I, 0);
        c->sz[2] = prepacked_expert_bytes(fmt, c->H, c->I, 1);
    } else {
        c->sz[0] = part_bytes(fmt, 2 * c->I, c->H, false);
        c->sz[1] = fmt == MOE_BF16 ? 0 : part_bytes(fmt, 2 * c->I, c->H, true);
        c->sz[2] = part_bytes(fmt, c->H, c->I, false);
        c->sz[3] = fmt == MOE_BF16 ? 0 : part_bytes(fmt, c->H, c->I, true);
    }
    size_t o = 0;
    for (int i = 0; i < 4; ++i) {
        c->off[i] = o;
        o += align_up(c->sz[i], 256);
    }
    c->slot_bytes = o;
    const size_t S = capacity_bytes / c->slot_bytes;
    if (S < 1) {
        const size_t need = c->slot_bytes;
        delete c;
        return set_error(MOE_ERR_CACHE_FULL, "capacity below one expert (%zu bytes)", need);
    }
    c->n_slots = (int)S;
    const int L = n_layers, E = c->E;
    auto fail = [&](cudaError_t er, const char *what) {
        moe_status r = set_cuda_error(er, what);
        expert_cache_destroy(c);
        return r;
    };
    // Pool: reserve the device's memory size of addresses and map the capacity.
    const VmmApi &v = vmm_api();
    size_t total = 0, freeb = 0;
    if (v.ok && cudaMemGetInfo(&freeb, &total) == cudaSuccess) {
        CUmemAllocationProp prop = {};
        prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
        prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
        prop.location.id = device;
        size_t gran = 0;
        if (v.granularity(&gran, &prop, CU_MEM_ALLOC_GRANULARITY_RECOMMENDED) == CUDA_SUCCESS && gran > 0) {
            c->chunk_bytes = align_up((size_t)256 << 20, gran);
            c->va_bytes = align_up(std::max(total, c->slot_bytes * S), c->chunk_bytes);
            CUdeviceptr va = 0;
            if (v.reserve(&va, c->va_bytes, c->chunk_bytes, 0, 0) == CUDA_SUCCESS) {
                c->pool = reinterpret_cast<uint8_t *>(va);
                c->vmm = true;
            }
        }
    }
    if (c->vmm) {
        moe_status r = map_to(c, c->slot_bytes * S);
        if (r != MOE_OK) {
            const std::string msg = moe_last_error_string();
            expert_cache_destroy(c);
            return set_error(r, "slot pool: %s", msg.c_str());
        }
        // the table has room for the larger of 8x the initial slots and 65536, within the range
        c->max_slots = (int)std::min<size_t>(c->va_bytes / c->slot_bytes, std::max<size_t>(8 * S, 65536));
    } else {
        if ((e = cudaMalloc(&c->pool, c->slot_bytes * S)) != cudaSuccess) return fail(e, "slot pool");
        c->max_slots = (int)S;
    }
    c->table_bytes = table_block_bytes(L, E, c->max_slots) + 2 * align_up((size_t)L * E * 4, 256);
    uint8_t *tbuf = nullptr;
    if ((e = cudaMalloc(&tbuf, c->table_bytes)) != cudaSuccess) return fail(e, "cache table");
    c->d_slot_of = reinterpret_cast<int32_t *>(tbuf);
    const LruTable t = table_of(c);
    c->d_owner = t.owner;
    c->d_prev = t.prev;
    c->d_next = t.next;
    c->d_ref = t.ref;
    c->d_free = t.freeb;
    c->d_last = t.last;
    c->d_lastcnt = t.lastcnt;
    c->d_state = t.st;
    c->d_counts = t.counts;
    const size_t tsb = table_block_bytes(L, E, c->max_slots);
    c->d_ts13 = reinterpret_cast<float *>(tbuf + tsb);
    c->d_ts2 = reinterpret_cast<float *>(tbuf + tsb + align_up((size_t)L * E * 4, 256));
    // io buffer: status + counts + up to 2 * (2E) pairs, or an id list; eviction list
    const size_t io_bytes = (size_t)(3 + 4 * E + 16) * 4;
    if ((e = cudaHostAlloc(&c->h_io, io_bytes, cudaHostAllocMapped)) != cudaSuccess) return fail(e, "mapped io buffer");
    if ((e = cudaHostGetDevicePointer(&c->d_io, c->h_io, 0)) != cudaSuccess) return fail(e, "mapped io pointer");
    if ((e = cudaHostAlloc(&c->h_ev, (size_t)(E + 16) * 4, cudaHostAllocMapped)) != cudaSuccess)
        return fail(e, "mapped eviction buffer");
    if ((e = cudaHostGetDevicePointer(&c->d_ev, c->h_ev, 0)) != cudaSuccess) return fail(e, "mapped eviction pointer");
    if ((e = cudaStreamCreateWithFlags(&c->cs, cudaStreamNonBlocking)) != cudaSuccess) return fail(e, "copy stream");
    // the host spins on this event (the table update is short; a blocking wait adds wake-up latency)
    if ((e = cudaEventCreateWithFlags(&c->ev_lru, cudaEventDisableTiming)) != cudaSuccess) return fail(e, "event");
    if ((e = cudaEventCreateWithFlags(&c->ev_res, cudaEventDisableTiming)) != cudaSuccess) return fail(e, "event");
    if ((e = cudaEventCreate(&c->ev_ref)) != cudaSuccess) return fail(e, "event");
    c->ring.assign((size_t)kTimerRing * kTimedKinds, nullptr);
    for (auto &ev : c->ring)
        if ((e = cudaEventCreate(&ev)) != cudaSuccess) return fail(e, "timing events");
    c->ring_mask.assign(kTimerRing, 0u);
    c->ring_bytes.assign(kTimerRing, 0u);
    if (fmt == MOE_NVFP4) {
        for (int l = 0; l < L; ++l) {
            const moe_experts &x = host_layers[l];
            if (!x.w13_tscale || !x.w2_tscale) {
                expert_cache_destroy(c);
                return set_error(MOE_ERR_INVALID_ARG, "NVFP4 layer %d without tensor scales", l);
            }
            cudaMemcpy(c->d_ts13 + (size_t)l * E, x.w13_tscale, E * 4, cudaMemcpyDefault);
            if ((e = cudaMemcpy(c->d_ts2 + (size_t)l * E, x.w2_tscale, E * 4, cudaMemcpyDefault)) != cudaSuccess)
                return fail(e, "tensor scales");
        }
    }
    const int lw = (E + 31) / 32;
    const int n = (int)std::max<size_t>(std::max<size_t>((size_t)L * E, (size_t)c->max_slots), (size_t)L * lw);
    count_launch();
    lru_init_kernel<<<(n + 255) / 256, 256>>>(table_of(c));
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return fail(e, "cache init");
    if ((e = cudaEventRecord(c->ev_ref, c->cs)) != cudaSuccess) return fail(e, "event");
    *out = c;
    return MOE_OK;
}

moe_status expert_cache_prefetch(struct expert_cache *c, int layer, const int32_t *ids, int n, moe_stream_t stream) {
    if (!c || layer < 0 || layer >= c->n_layers || n < 0 || n > c->E || (n && !ids))
        return set_error(MOE_ERR_INVALID_ARG, "bad prefetch arguments");
    if (n == 0) return MOE_OK;
    cudaStream_t st = (cudaStream_t)stream;
    // the previous call's readback is complete (it was synchronised), so io is free
    c->h_io[0] = n;
    memcpy(c->h_io + 1, ids, sizeof(int32_t) * n);
    cudaError_t e = launch_lru(c, layer, nullptr, 0, 1, 0, 0, st);
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_lru, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_lru);
    if (e != cudaSuccess) return set_cuda_error(e, "prefetch table update");
    if (c->h_io[0] == MOE_ERR_CACHE_FULL) return set_error(MOE_ERR_CACHE_FULL, "prefetch does not fit");
    const int na = c->h_io[1];
    std::vector<int32_t> pairs(c->h_io + 3, c->h_io + 3 + 2 * na);
    harvest(c, false);
    timer_open(c);
    timer_mark(c, TK_COPY_B, c->cs);
    int done = 0;
    moe_status r = issue_loads(c, layer, pairs.data(), na, &done);
    timer_mark(c, TK_COPY_E, c->cs);
    timer_close(c);
    if (r != MOE_OK) {
        const std::string msg = moe_last_error_string();
        rollback(c, layer, pairs.data(), done, na, st);
        return set_error(r, "%s", msg.c_str());
    }
    return MOE_OK;
}

moe_status expert_cache_evict(struct expert_cache *c, int layer, const int32_t *ids, int n) {
    if (!c || layer < -1 || layer >= c->n_layers || n > c->E || (n > 0 && !ids))
        return set_error(MOE_ERR_INVALID_ARG, "bad evict arguments");
    cudaError_t e = cudaStreamSynchronize(c->cs);   // no copy may still target a freed slot
    if (e != cudaSuccess) return set_cuda_error(e, "copy stream");
    c->h_io[0] = (layer < 0 || n < 0) ? -1 : n;
    if (layer >= 0 && n > 0) memcpy(c->h_io + 1, ids, sizeof(int32_t) * n);
    count_launch();
    lru_evict_kernel<<<1, 32>>>(table_of(c), layer, c->d_io);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "evict");
}

moe_status expert_cache_set_prefetch(struct expert_cache *c, int policy, int depth) {
    if (!c || policy < MOE_PREFETCH_NONE || policy > MOE_PREFETCH_ADAPTIVE)
        return set_error(MOE_ERR_INVALID_ARG, "bad prefetch policy");
    c->pf_policy = policy;
    c->pf_depth = depth;
    return MOE_OK;
}

moe_status expert_cache_resize(struct expert_cache *c, size_t capacity_bytes) {
    if (!c) return set_error(MOE_ERR_INVALID_ARG, "cache is NULL");
    const size_t S_new = capacity_bytes / c->slot_bytes;
    if (S_new < 1) return set_error(MOE_ERR_CACHE_FULL, "capacity below one expert (%zu bytes)", c->slot_bytes);
    if (S_new > (size_t)c->max_slots)
        return set_error(MOE_ERR_UNSUPPORTED, "%zu slots exceed the %d the pool's address range holds", S_new,
                         c->max_slots);
    // no kernel or copy may use the slots while the table and the pool change
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return set_cuda_error(e, "device synchronize");
    harvest(c, false);
    if (c->vmm && S_new > (size_t)c->n_slots) {
        moe_status r = map_to(c, c->slot_bytes * S_new);
        if (r != MOE_OK) return r;
    }
    // the table update runs on a host copy of the table block, with the same code
    std::vector<uint8_t> host(table_block_bytes(c->n_layers, c->E, c->max_slots));
    if ((e = cudaMemcpy(host.data(), c->d_slot_of, host.size(), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return set_cuda_error(e, "table read");
    LruTable t = table_at(c, host.data());
    std::vector<int32_t> moves(2 * S_new + 2);
    const int nm = lru_resize(t, (int)S_new, moves.data());
    if (nm < 0) return set_error(MOE_ERR_INVALID_ARG, "resize to %zu slots", S_new);
    for (int i = 0; i < nm; ++i) {
        const uint8_t *from = c->pool + (size_t)moves[2 * i] * c->slot_bytes;
        uint8_t *to = c->pool + (size_t)moves[2 * i + 1] * c->slot_bytes;
        if ((e = cudaMemcpyAsync(to, from, c->slot_bytes, cudaMemcpyDeviceToDevice, c->cs)) != cudaSuccess)
            return set_cuda_error(e, "slot move");
    }
    if ((e = cudaMemcpyAsync(c->d_slot_of, host.data(), host.size(), cudaMemcpyHostToDevice, c->cs)) != cudaSuccess)
        return set_cuda_error(e, "table write");
    if ((e = cudaStreamSynchronize(c->cs)) != cudaSuccess) return set_cuda_error(e, "copy stream");
    c->moved += (uint64_t)nm;
    c->n_slots = (int)S_new;
    if (c->vmm) unmap_past(c, c->slot_bytes * S_new);
    return MOE_OK;
}

moe_status expert_cache_stats(struct expert_cache *c, uint64_t *hits, uint64_t *misses, uint64_t *bytes_h2d,
                              double *copy_s) {
    if (!c) return set_error(MOE_ERR_INVALID_ARG, "cache is NULL");
    cudaError_t e = cudaStreamSynchronize(c->cs);
    if (e != cudaSuccess) return set_cuda_error(e, "copy stream");
    unsigned long long cnt[2] = {0, 0};
    e = cudaMemcpy(cnt, c->d_counts, sizeof(cnt), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return set_cuda_error(e, "counters");
    harvest(c, false);
    if (hits) *hits = cnt[0];
    if (misses) *misses = cnt[1];
    if (bytes_h2d) *bytes_h2d = c->bytes_h2d;
    if (copy_s) *copy_s = c->copy_s;
    return MOE_OK;
}

moe_status expert_cache_report(struct expert_cache *c, moe_cache_report *out) {
    if (!c || !out) return set_error(MOE_ERR_INVALID_ARG, "NULL argument");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return set_cuda_error(e, "device synchronize");
    harvest(c, false);
    memset(out, 0, sizeof(*out));
    out->table_s = c->table_s;
    out->host_wait_s = c->host_wait_s;
    out->issue_s = c->issue_s;
    out->copy_s = c->copy_s;
    out->compute_s = c->compute_s;
    out->overlap_s = c->overlap_s;
    out->h2d_gbs = c->bw_ewma * 1e-9;
    out->calls = c->calls;
    out->prefetched = c->prefetched;
    out->moved = c->moved;
    out->n_slots = c->n_slots;
    out->last_depth = c->last_depth;
    return MOE_OK;
}

moe_status expert_cache_slot_of(struct expert_cache *c, int layer, int e, int32_t *slot) {
    if (!c || !slot || layer < 0 || layer >= c->n_layers || e < 0 || e >= c->E)
        return set_error(MOE_ERR_INVALID_ARG, "bad slot_of arguments");
    cudaError_t er = cudaMemcpy(slot, c->d_slot_of + (size_t)layer * c->E + e, 4, cudaMemcpyDeviceToHost);
    return er == cudaSuccess ? MOE_OK : set_cuda_error(er, "slot_of");
}

moe_status expert_cache_destroy(struct expert_cache *c) {
    if (!c) return MOE_OK;
    cudaDeviceSynchronize();   // no kernel may still read the pool or the table
    for (cudaEvent_t ev : c->ring)
        if (ev) cudaEventDestroy(ev);
    if (c->ev_ref) cudaEventDestroy(c->ev_ref);
    if (c->ev_lru) cudaEventDestroy(c->ev_lru);
    if (c->ev_res) cudaEventDestroy(c->ev_res);
    if (c->cs) cudaStreamDestroy(c->cs);
    if (c->h_io) cudaFreeHost(c->h_io);
    if (c->h_ev) cudaFreeHost(c->h_ev);
    if (c->d_slot_of) cudaFree(c->d_slot_of);   // start of the table block
    if (c->vmm) {
        unmap_past(c, 0);
        vmm_api().free_va(reinterpret_cast<CUdeviceptr>(c->pool), c->va_bytes);
    } else if (c->pool) {
        cudaFree(c->pool);
    }
    delete c;
    return MOE_OK;
}

}  // extern "C"
