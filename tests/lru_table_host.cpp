// Host build of the expert cache's table functions (lru_table.cuh) for the CPU
// tests: the same code the cache runs on the device, driven one call at a time
// through a small C interface. Test infrastructure only.
#include <algorithm>
#include <vector>

#include "../expert_ffn_layer_top_b200/csrc/lru_table.cuh"

using namespace moe;

namespace {

struct HostLru {
    std::vector<int32_t> slot_of, owner, prev, next, ref, st;
    std::vector<uint32_t> freeb, last;
    unsigned long long counts[2] = {0, 0};
    LruTable t{};
};

// The request bitmap, built as the device kernel builds it: each id in [0, E) once.
std::vector<uint32_t> request(const LruTable &t, const int32_t *ids, int n) {
    std::vector<uint32_t> req((t.E + 31) / 32, 0u);
    for (int i = 0; i < n; ++i)
        if (ids[i] >= 0 && ids[i] < t.E) req[ids[i] >> 5] |= 1u << (ids[i] & 31);
    return req;
}

}  // namespace

extern "C" {

void *lru_host_create(int S, int L, int E) {
    HostLru *h = new HostLru();
    const int sw = (S + 31) / 32, lw = (E + 31) / 32;
    h->slot_of.assign((size_t)L * E, 0);
    h->owner.assign(S, 0);
    h->prev.assign(S, 0);
    h->next.assign(S, 0);
    h->ref.assign(S, 0);
    h->st.assign(ST_N, 0);
    h->freeb.assign(sw, 0u);
    h->last.assign((size_t)L * lw, 0u);
    LruTable &t = h->t;
    t.slot_of = h->slot_of.data();
    t.owner = h->owner.data();
    t.prev = h->prev.data();
    t.next = h->next.data();
    t.ref = h->ref.data();
    t.freeb = h->freeb.data();
    t.last = h->last.data();
    t.st = h->st.data();
    t.counts = h->counts;
    t.S = S;
    t.E = E;
    t.L = L;
    const int n = std::max(std::max(L * E, S), L * lw);
    for (int i = 0; i < n; ++i) lru_init_one(t, i);
    return h;
}

void lru_host_destroy(void *p) { delete static_cast<HostLru *>(p); }

// A layer's resolve from its routed expert ids idx[P] (mode 0 of the device kernel).
// io: at least 3 + 4*E ints; layout as lru_run writes it.
void lru_host_resolve(void *p, int layer, const int32_t *idx, int P, int prefetch_next, int32_t *io) {
    HostLru *h = static_cast<HostLru *>(p);
    const std::vector<uint32_t> req = request(h->t, idx, P);
    lru_run(h->t, layer, req.data(), 0, prefetch_next, io);
}

// An explicit prefetch of ids[n] (mode 1).
void lru_host_prefetch(void *p, int layer, const int32_t *ids, int n, int32_t *io) {
    HostLru *h = static_cast<HostLru *>(p);
    const std::vector<uint32_t> req = request(h->t, ids, n);
    lru_run(h->t, layer, req.data(), 1, 0, io);
}

// Eviction with the argument convention of expert_cache_evict.
void lru_host_evict(void *p, int layer, const int32_t *ids, int n) {
    HostLru *h = static_cast<HostLru *>(p);
    std::vector<int32_t> io(1 + std::max(n, 0));
    io[0] = (layer < 0 || n < 0) ? -1 : n;
    for (int i = 0; i < n; ++i) io[1 + i] = ids[i];
    lru_evict(h->t, layer, io.data());
}

int lru_host_slot_of(void *p, int layer, int e) {
    const HostLru *h = static_cast<HostLru *>(p);
    return h->slot_of[(size_t)layer * h->t.E + e];
}

void lru_host_counts(void *p, unsigned long long *hits_misses) {
    const HostLru *h = static_cast<HostLru *>(p);
    hits_misses[0] = h->counts[0];
    hits_misses[1] = h->counts[1];
}

}  // extern "C"
