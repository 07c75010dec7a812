// Host build of the expert cache's table functions (lru_table.cuh) for the CPU
// tests: the same code the cache runs on the device, driven one call at a time
// through a small C interface. Test infrastructure only.
#include <algorithm>
#include <vector>

#include "../expert_ffn_layer_top_b200/csrc/lru_table.cuh"

using namespace moe;

namespace {

struct HostLru {
    std::vector<int32_t> slot_of, owner, prev, next, ref, st, lastcnt;
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

// A table of S slots with room for Smax (>= S) after resizes.
void *lru_host_create(int S, int L, int E, int Smax) {
    HostLru *h = new HostLru();
    const int sw = (Smax + 31) / 32, lw = (E + 31) / 32;
    h->slot_of.assign((size_t)L * E, 0);
    h->lastcnt.assign((size_t)L * E, 0);
    h->owner.assign(Smax, 0);
    h->prev.assign(Smax, 0);
    h->next.assign(Smax, 0);
    h->ref.assign(Smax, 0);
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
    t.lastcnt = h->lastcnt.data();
    t.st = h->st.data();
    t.counts = h->counts;
    t.S = S;
    t.E = E;
    t.L = L;
    t.Smax = Smax;
    const int n = std::max(std::max(L * E, Smax), L * lw);
    for (int i = 0; i < n; ++i) lru_init_one(t, i);
    return h;
}

void lru_host_destroy(void *p) { delete static_cast<HostLru *>(p); }

// A layer's resolve from its routed expert ids idx[P] (mode 0 of the device kernel),
// followed by the prefetch of layer+1: pf_mode 0 none, 1 the first `depth` experts of
// its prediction (depth < 0: all), 2 the whole layer.
// io: at least 3 + 4*E ints; layout as lru_run writes it.
void lru_host_resolve(void *p, int layer, const int32_t *idx, int P, int pf_mode, int depth, int32_t *io) {
    HostLru *h = static_cast<HostLru *>(p);
    const std::vector<uint32_t> req = request(h->t, idx, P);
    std::vector<int32_t> cnt(h->t.E, 0);
    for (int i = 0; i < P; ++i)
        if (idx[i] >= 0 && idx[i] < h->t.E) ++cnt[idx[i]];
    std::vector<uint32_t> pf((h->t.E + 31) / 32, 0u);
    const bool pfn = pf_mode != 0 && layer + 1 < h->t.L;
    if (pfn) lru_predict(h->t, layer + 1, depth, pf_mode == 2, pf.data());
    lru_run(h->t, layer, req.data(), cnt.data(), 0, pfn ? pf.data() : nullptr, io);
}

// An explicit prefetch of ids[n] (mode 1).
void lru_host_prefetch(void *p, int layer, const int32_t *ids, int n, int32_t *io) {
    HostLru *h = static_cast<HostLru *>(p);
    const std::vector<uint32_t> req = request(h->t, ids, n);
    lru_run(h->t, layer, req.data(), nullptr, 1, nullptr, io);
}

// Resize to S_new slots; moves: room for 2 * S_new ints. Returns the move count or -1.
int lru_host_resize(void *p, int S_new, int32_t *moves) {
    HostLru *h = static_cast<HostLru *>(p);
    return lru_resize(h->t, S_new, moves);
}

// The prefetch plan of a cached call (lru_prefetch_plan): returns the depth; flags[0] =
// whole layer, flags[1] = none.
int lru_host_plan(int policy, int depth, int T, int k, int E, double bw, double t_comp, double expert_bytes,
                  int *flags) {
    bool full = false, none = false;
    const int d = lru_prefetch_plan(policy, depth, T, k, E, bw, t_comp, expert_bytes, &full, &none);
    flags[0] = full;
    flags[1] = none;
    return d;
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
