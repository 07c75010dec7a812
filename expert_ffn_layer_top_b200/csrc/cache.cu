// Device LRU expert cache with host->device streaming of misses.
//
// Source: winzheng.com page, sections "Why Now of All Times" (most experts stay
// in host memory and are loaded on demand) and "FreeToken's Three-Layer
// Mechanism" (double-buffered streaming overlapped with compute, a global LRU
// expert cache reusing high-frequency experts); aimodeling.com English page,
// section "Three Engineering Cores" (the same).
//
// Layout. One device allocation of n_slots slots; a slot holds one expert's
// w13 codes, w13 scales, w2 codes and w2 scales at fixed 256-byte-aligned
// offsets, so the grouped FFN reads cached experts through the same strided
// descriptor as resident ones, with expert_map = the slot of each expert.
//
// Table (device): slot_of[L*E], owner[S], an intrusive LRU list (prev/next,
// head = least recent), ref_call[S] (index of the last call that referenced
// the slot), a free-slot bitmap, per-layer bitmaps of the experts used at the
// last step (the prefetch prediction) and counters. One warp runs a call:
// lanes build the request bitmap, lane 0 walks it in ascending expert order:
//   hit  -> move to the most-recent end;
//   miss -> lowest free slot, else the least recent slot not referenced by
//           this call or the previous one (those may still be in use);
// a call that cannot fit fails with CACHE_FULL before changing anything.
// The (expert, slot) loads go to page-locked mapped host memory; the host
// reads them after one event wait and issues one cudaMemcpyAsync per array
// on the cache's copy stream. The layer's GEMM waits on an event recorded
// after its own loads; the loads for the next layer's predicted experts are
// issued behind it on the copy stream, so they overlap this layer's GEMMs
// (the double buffering: the layer being computed and the layer being filled).
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "lru_table.cuh"

struct expert_cache {
    int device = 0, n_layers = 0, E = 0, H = 0, I = 0, fmt = 0, layout = 0;
    size_t sz[4] = {0, 0, 0, 0};      // per-expert bytes: w13, w13 scales, w2, w2 scales
    size_t off[4] = {0, 0, 0, 0};     // offsets inside a slot
    size_t slot_bytes = 0;
    int n_slots = 0;
    uint8_t *pool = nullptr;
    // device table
    int32_t *d_slot_of = nullptr, *d_owner = nullptr, *d_prev = nullptr, *d_next = nullptr, *d_ref = nullptr;
    uint32_t *d_free = nullptr, *d_last = nullptr;   // free bitmap [S/32], last-used bitmaps [L][E/32]
    int32_t *d_state = nullptr;                        // head, tail, calls, free_count, hint, last_nref
    unsigned long long *d_counts = nullptr;            // hits, misses
    float *d_ts13 = nullptr, *d_ts2 = nullptr;         // NVFP4 tensor scales [L][E]
    // mapped host buffers
    int32_t *h_io = nullptr, *d_io = nullptr;          // loads out / ids in
    std::vector<moe_experts> layers;                   // host descriptions (host pointers)
    cudaStream_t cs = nullptr;
    cudaEvent_t ev_lru = nullptr, ev_res = nullptr;
    std::vector<cudaEvent_t> timers;                   // start/stop pairs on the copy stream
    uint64_t bytes_h2d = 0;
    uint64_t copies = 0;
    double copy_s = 0.0;
    long fault_h2d_at = -1;                            // host fault injection: fail this copy (1-based)
};

namespace moe {

// mode 0: resolve `layer` from idx[P] (+ prefetch layer+1's prediction if prefetch_next)
// mode 1: prefetch `layer` with the explicit ids in io (count io[0], ids io[1..])
// Output in io: [0] status (0 ok, 6 cache full), [1] n resolve loads, [2] n prefetch loads
// (-1 = not run or full), then the pairs.
__global__ void __launch_bounds__(32) lru_kernel(LruTable t, int layer, const int32_t *idx, int P, int mode,
                                                  int prefetch_next, int32_t *io) {
    __shared__ uint32_t req[kMaxExperts / 32];
    const int lane = threadIdx.x;
    const int words = (t.E + 31) / 32;
    for (int w = lane; w < words; w += 32) req[w] = 0;
    __syncwarp();
    int nids = 0;
    if (mode == 1) nids = io[0];
    __syncwarp();
    if (mode == 0) {
        for (int p = lane; p < P; p += 32) {
            const int e = idx[p];
            if (e >= 0 && e < t.E) atomicOr(&req[e >> 5], 1u << (e & 31));
        }
    } else {
        for (int i = lane; i < nids; i += 32) {
            const int e = io[1 + i];
            if (e >= 0 && e < t.E) atomicOr(&req[e >> 5], 1u << (e & 31));
        }
    }
    __syncwarp();
    if (lane != 0) return;
    lru_run(t, layer, req, mode, prefetch_next, io);
}

__global__ void lru_init_kernel(LruTable t) { lru_init_one(t, blockIdx.x * blockDim.x + threadIdx.x); }

// Free slots matching (layer, ids) (see lru_evict).
__global__ void lru_evict_kernel(LruTable t, int layer, const int32_t *io) {
    if (threadIdx.x == 0) lru_evict(t, layer, io);
}

static LruTable table_of(expert_cache *c) {
    LruTable t;
    t.slot_of = c->d_slot_of;
    t.owner = c->d_owner;
    t.prev = c->d_prev;
    t.next = c->d_next;
    t.ref = c->d_ref;
    t.freeb = c->d_free;
    t.last = c->d_last;
    t.st = c->d_state;
    t.counts = c->d_counts;
    t.S = c->n_slots;
    t.E = c->E;
    t.L = c->n_layers;
    return t;
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

// Issue the copies of `n` loads (pairs e, slot) of `layer` on the copy stream.
static moe_status issue_loads(expert_cache *c, int layer, const int32_t *pairs, int n) {
    const moe_experts &x = c->layers[layer];
    const void *src[4] = {x.w13, x.w13_scale, x.w2, x.w2_scale};
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
        }
    }
    return MOE_OK;
}

static moe_status timed_begin(expert_cache *c) {
    cudaEvent_t a;
    cudaError_t e = cudaEventCreate(&a);
    if (e == cudaSuccess) e = cudaEventRecord(a, c->cs);
    if (e != cudaSuccess) return set_cuda_error(e, "copy timer");
    c->timers.push_back(a);
    return MOE_OK;
}

static moe_status timed_end(expert_cache *c) { return timed_begin(c); }

static void harvest_timers(expert_cache *c) {
    // pairs (start, stop); accumulate the finished ones
    size_t i = 0;
    for (; i + 1 < c->timers.size(); i += 2) {
        if (cudaEventQuery(c->timers[i + 1]) != cudaSuccess) break;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, c->timers[i], c->timers[i + 1]) == cudaSuccess) c->copy_s += ms * 1e-3;
        cudaEventDestroy(c->timers[i]);
        cudaEventDestroy(c->timers[i + 1]);
    }
    c->timers.erase(c->timers.begin(), c->timers.begin() + i);
}

moe_status cache_resolve_and_map(expert_cache *c, int layer, const int32_t *idx, int T, int k,
                                 const moe_experts *shape, moe_experts *view, cudaStream_t st) {
    if (layer < 0 || layer >= c->n_layers) return set_error(MOE_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (shape->E != c->E || shape->H != c->H || shape->I != c->I || shape->fmt != c->fmt)
        return set_error(MOE_ERR_INVALID_ARG, "layer shape differs from the cache's");
    count_launch();
    lru_kernel<<<1, 32, 0, st>>>(table_of(c), layer, idx, T * k, 0, 1, c->d_io);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_lru, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_lru);
    if (e != cudaSuccess) return set_cuda_error(e, "cache table update");
    const int32_t *io = c->h_io;
    if (io[0] == MOE_ERR_CACHE_FULL)
        return set_error(MOE_ERR_CACHE_FULL, "layer %d needs more slots than the cache can free", layer);
    const int na = io[1], nb = io[2];
    moe_status r;
    if ((r = timed_begin(c)) != MOE_OK) return r;
    if ((r = issue_loads(c, layer, io + 3, na)) != MOE_OK) return r;
    if ((e = cudaEventRecord(c->ev_res, c->cs)) != cudaSuccess) return set_cuda_error(e, "event");
    if (nb > 0 && (r = issue_loads(c, layer + 1, io + 3 + 2 * na, nb)) != MOE_OK) return r;
    if ((r = timed_end(c)) != MOE_OK) return r;
    if ((e = cudaStreamWaitEvent(st, c->ev_res, 0)) != cudaSuccess) return set_cuda_error(e, "stream wait");
    harvest_timers(c);
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
    return MOE_OK;
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
    const int L = n_layers, E = c->E, lw = (E + 31) / 32;
    auto fail = [&](cudaError_t er, const char *what) {
        moe_status r = set_cuda_error(er, what);
        expert_cache_destroy(c);
        return r;
    };
    if ((e = cudaMalloc(&c->pool, c->slot_bytes * S)) != cudaSuccess) return fail(e, "slot pool");
    size_t tb = 0;
    tb += align_up((size_t)L * E * 4, 256);             // slot_of
    tb += 4 * align_up(S * 4, 256);                      // owner prev next ref
    tb += align_up((S + 31) / 32 * 4, 256);              // free bitmap
    tb += align_up((size_t)L * lw * 4, 256);             // last-used bitmaps
    tb += 256 + 256;                                     // state, counters
    tb += 2 * align_up((size_t)L * E * 4, 256);          // tensor scales
    uint8_t *tbuf = nullptr;
    if ((e = cudaMalloc(&tbuf, tb)) != cudaSuccess) return fail(e, "cache table");
    size_t p = 0;
    auto take = [&](size_t bytes) { uint8_t *r = tbuf + p; p += align_up(bytes, 256); return r; };
    c->d_slot_of = reinterpret_cast<int32_t *>(take((size_t)L * E * 4));
    c->d_owner = reinterpret_cast<int32_t *>(take(S * 4));
    c->d_prev = reinterpret_cast<int32_t *>(take(S * 4));
    c->d_next = reinterpret_cast<int32_t *>(take(S * 4));
    c->d_ref = reinterpret_cast<int32_t *>(take(S * 4));
    c->d_free = reinterpret_cast<uint32_t *>(take((S + 31) / 32 * 4));
    c->d_last = reinterpret_cast<uint32_t *>(take((size_t)L * lw * 4));
    c->d_state = reinterpret_cast<int32_t *>(take(256));
    c->d_counts = reinterpret_cast<unsigned long long *>(take(256));
    c->d_ts13 = reinterpret_cast<float *>(take((size_t)L * E * 4));
    c->d_ts2 = reinterpret_cast<float *>(take((size_t)L * E * 4));
    // io buffer: status + counts + up to 2 * (2E) pairs, or an id list
    const size_t io_bytes = (size_t)(3 + 4 * E + 16) * 4;
    if ((e = cudaHostAlloc(&c->h_io, io_bytes, cudaHostAllocMapped)) != cudaSuccess) return fail(e, "mapped io buffer");
    if ((e = cudaHostGetDevicePointer(&c->d_io, c->h_io, 0)) != cudaSuccess) return fail(e, "mapped io pointer");
    if ((e = cudaStreamCreateWithFlags(&c->cs, cudaStreamNonBlocking)) != cudaSuccess) return fail(e, "copy stream");
    if ((e = cudaEventCreateWithFlags(&c->ev_lru, cudaEventBlockingSync | cudaEventDisableTiming)) != cudaSuccess)
        return fail(e, "event");
    if ((e = cudaEventCreateWithFlags(&c->ev_res, cudaEventDisableTiming)) != cudaSuccess) return fail(e, "event");
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
    const int n = (int)std::max<size_t>(std::max<size_t>((size_t)L * E, S), (size_t)L * lw);
    count_launch();
    lru_init_kernel<<<(n + 255) / 256, 256>>>(table_of(c));
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return fail(e, "cache init");
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
    count_launch();
    lru_kernel<<<1, 32, 0, st>>>(table_of(c), layer, nullptr, 0, 1, 0, c->d_io);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_lru, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_lru);
    if (e != cudaSuccess) return set_cuda_error(e, "prefetch table update");
    if (c->h_io[0] == MOE_ERR_CACHE_FULL) return set_error(MOE_ERR_CACHE_FULL, "prefetch does not fit");
    moe_status r;
    if ((r = timed_begin(c)) != MOE_OK) return r;
    if ((r = issue_loads(c, layer, c->h_io + 3, c->h_io[1])) != MOE_OK) return r;
    if ((r = timed_end(c)) != MOE_OK) return r;
    harvest_timers(c);
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

moe_status expert_cache_stats(struct expert_cache *c, uint64_t *hits, uint64_t *misses, uint64_t *bytes_h2d,
                              double *copy_s) {
    if (!c) return set_error(MOE_ERR_INVALID_ARG, "cache is NULL");
    cudaError_t e = cudaStreamSynchronize(c->cs);
    if (e != cudaSuccess) return set_cuda_error(e, "copy stream");
    unsigned long long cnt[2] = {0, 0};
    e = cudaMemcpy(cnt, c->d_counts, sizeof(cnt), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return set_cuda_error(e, "counters");
    harvest_timers(c);
    if (hits) *hits = cnt[0];
    if (misses) *misses = cnt[1];
    if (bytes_h2d) *bytes_h2d = c->bytes_h2d;
    if (copy_s) *copy_s = c->copy_s;
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
    if (c->cs) cudaStreamSynchronize(c->cs);
    for (cudaEvent_t ev : c->timers) cudaEventDestroy(ev);
    if (c->ev_lru) cudaEventDestroy(c->ev_lru);
    if (c->ev_res) cudaEventDestroy(c->ev_res);
    if (c->cs) cudaStreamDestroy(c->cs);
    if (c->h_io) cudaFreeHost(c->h_io);
    if (c->d_slot_of) cudaFree(c->d_slot_of);   // start of the table block
    if (c->pool) cudaFree(c->pool);
    delete c;
    return MOE_OK;
}

}  // extern "C"
