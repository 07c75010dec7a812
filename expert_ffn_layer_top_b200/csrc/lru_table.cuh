// The expert cache's table and its LRU policy, as plain functions over a set of
// arrays. The cache runs them on the device from a single thread (cache.cu). They
// also compile as ordinary host C++, which is how the tests run them against a CPU
// simulation of the same policy over long random traces.
//
// Source of the policy: winzheng.com page, section "FreeToken's Three-Layer
// Mechanism" (a global LRU expert cache reusing high-frequency experts);
// aimodeling.com English page, section "Three Engineering Cores". The rules
// below are this library's reading of "LRU":
//   - a call handles its expert ids once each, in ascending order;
//   - a hit moves the slot to the most-recent end;
//   - a miss takes the lowest free slot, else the least recently referenced slot
//     not referenced by this call or the previous one;
//   - a call that cannot fit fails before changing anything.
// Prefetch of the next layer (aimodeling.com English page, section "Three
// Engineering Cores": full-layer double-buffered streaming; winzheng.com page,
// section "FreeToken's Three-Layer Mechanism": the transfer adapts to the
// bandwidth it measures): the prediction for a layer is the set of experts its
// last resolve used, ranked by how many pairs each received (more first, ties
// to the lower id); a prefetch takes the first `depth` of them, or every
// expert of the layer when the whole layer is streamed.
// Resizing the slot pool (aimodeling.com, "Three Engineering Cores": elastic
// memory management without weight reloads): growing adds free slots;
// shrinking keeps the most recently referenced experts that fit, moves the
// ones above the new end into the lowest free slots (least recent first) and
// drops the rest, so no kept expert is fetched again.
#pragma once

#include <stdint.h>

#include "../../include/moe.h"

#ifdef __CUDACC__
#include "common.cuh"
#define LRU_HD __host__ __device__
#else
#define LRU_HD
#endif

namespace moe {

enum { ST_HEAD = 0, ST_TAIL, ST_CALLS, ST_FREE, ST_HINT, ST_LASTN, ST_N };
constexpr int kNone = -1;
constexpr int kNeverRef = -(1 << 30);

// slot_of[L*E]: slot of (layer, expert) or -1; owner[Smax]: key layer*E+e of a slot or -1;
// prev/next[Smax]: the intrusive recency list (head = least recent); ref[Smax]: index of
// the last call that referenced the slot; freeb[ceil(Smax/32)]: free-slot bitmap (bits
// of slots >= S stay clear); last[L][ceil(E/32)]: experts each layer used at its last
// resolve (the prefetch prediction); lastcnt[L][E]: pairs each of them received;
// st[ST_N]: head, tail, calls, free count, first bitmap word that may hold a free slot,
// slots referenced by the last call; counts: hits, misses. S slots are in use, and the
// arrays have room for Smax.
struct LruTable {
    int32_t *slot_of, *owner, *prev, *next, *ref;
    uint32_t *freeb, *last;
    int32_t *lastcnt;
    int32_t *st;
    unsigned long long *counts;
    int S, E, L, Smax;
};

// Largest pair count the prediction ranks by; counts above it rank as equal.
constexpr int kCntCap = (1 << 20) - 1;

// Ranking key of expert e with `cnt` pairs: larger first, unique per expert.
LRU_HD inline uint32_t lru_rank_key(int cnt, int e) {
    const uint32_t c = (uint32_t)(cnt < kCntCap ? cnt : kCntCap);
    return (c << 11) | (uint32_t)(2047 - e);
}

// 1-based index of the lowest set bit, 0 for none.
LRU_HD inline int lru_ffs(uint32_t v) {
#ifdef __CUDA_ARCH__
    return __ffs(v);
#else
    return __builtin_ffs((int)v);
#endif
}

// Records an inconsistency of the table in the library's device error word.
LRU_HD inline void lru_flag_error(int code) {
#ifdef __CUDA_ARCH__
    flag_error(code);
#else
    (void)code;
#endif
}

LRU_HD inline void lru_unlink(LruTable &t, int s) {
    const int p = t.prev[s], n = t.next[s];
    if (p != kNone) t.next[p] = n; else t.st[ST_HEAD] = n;
    if (n != kNone) t.prev[n] = p; else t.st[ST_TAIL] = p;
    t.prev[s] = t.next[s] = kNone;
}

LRU_HD inline void lru_append(LruTable &t, int s) {
    const int tl = t.st[ST_TAIL];
    t.prev[s] = tl;
    t.next[s] = kNone;
    if (tl != kNone) t.next[tl] = s; else t.st[ST_HEAD] = s;
    t.st[ST_TAIL] = s;
}

LRU_HD inline int lru_pop_free(LruTable &t) {
    const int words = (t.S + 31) / 32;
    for (int w = t.st[ST_HINT]; w < words; ++w) {
        const uint32_t v = t.freeb[w];
        if (v) {
            const int b = lru_ffs(v) - 1;
            t.freeb[w] = v & ~(1u << b);
            t.st[ST_HINT] = w;
            t.st[ST_FREE] -= 1;
            return w * 32 + b;
        }
    }
    return kNone;
}

// Table state of a fresh cache, element i of every array (i over max(L*E, Smax, L*ceil(E/32))).
LRU_HD inline void lru_init_one(LruTable &t, int i) {
    if (i < t.L * t.E) {
        t.slot_of[i] = kNone;
        t.lastcnt[i] = 0;
    }
    if (i < t.Smax) {
        t.owner[i] = kNone;
        t.prev[i] = t.next[i] = kNone;
        t.ref[i] = kNeverRef;
    }
    const int words = (t.Smax + 31) / 32;
    if (i < words) {
        const int rem = t.S - i * 32;
        t.freeb[i] = rem >= 32 ? 0xffffffffu : (rem > 0 ? ((1u << rem) - 1u) : 0u);
    }
    const int lw = (t.E + 31) / 32;
    if (i < t.L * lw) t.last[i] = 0;
    if (i == 0) {
        t.st[ST_HEAD] = t.st[ST_TAIL] = kNone;
        t.st[ST_CALLS] = 0;
        t.st[ST_FREE] = t.S;
        t.st[ST_HINT] = 0;
        t.st[ST_LASTN] = 0;
        t.counts[0] = t.counts[1] = 0;
    }
}

// One call (resolve or prefetch) of `layer` with the request bitmap `req`.
// Writes (e, slot) loads to out[0..2n). Returns the number of loads, or -1 (cache full).
LRU_HD inline int lru_call(LruTable &t, int layer, const uint32_t *req, bool counted, int32_t *out) {
    const int c = t.st[ST_CALLS];
    const int words = (t.E + 31) / 32;
    int misses = 0, newprot = 0;
    for (int w = 0; w < words; ++w)
        for (uint32_t v = req[w]; v; v &= v - 1) {
            const int e = w * 32 + lru_ffs(v) - 1;
            const int s = t.slot_of[layer * t.E + e];
            if (s < 0) ++misses;
            else if (t.ref[s] < c - 1) ++newprot;
        }
    const int occupied = t.S - t.st[ST_FREE];
    const int evictable = occupied - t.st[ST_LASTN] - newprot;
    if (misses > t.st[ST_FREE] + evictable) return -1;
    int nl = 0, nref = 0, hits = 0;
    for (int w = 0; w < words; ++w)
        for (uint32_t v = req[w]; v; v &= v - 1) {
            const int e = w * 32 + lru_ffs(v) - 1;
            const int key = layer * t.E + e;
            int s = t.slot_of[key];
            if (s >= 0) {
                ++hits;
                lru_unlink(t, s);
            } else {
                s = lru_pop_free(t);
                if (s == kNone) {
                    s = t.st[ST_HEAD];
                    while (s != kNone && t.ref[s] >= c - 1) s = t.next[s];
                    if (s == kNone) { lru_flag_error(2); return -1; }   // excluded by the count above
                    lru_unlink(t, s);
                    t.slot_of[t.owner[s]] = kNone;
                }
                t.owner[s] = key;
                t.slot_of[key] = s;
                out[2 * nl] = e;
                out[2 * nl + 1] = s;
                ++nl;
            }
            lru_append(t, s);
            t.ref[s] = c;
            ++nref;
        }
    t.st[ST_CALLS] = c + 1;
    t.st[ST_LASTN] = nref;
    if (counted) {
        t.counts[0] += hits;
        t.counts[1] += nl;
    }
    return nl;
}

// The prefetch request of `layer` (bitmap out[ceil(E/32)]): every expert when `full`,
// else the first `depth` of its prediction in rank order (depth < 0: all of it).
// Plain sequential code; the device kernel computes the same set with one warp.
LRU_HD inline void lru_predict(const LruTable &t, int layer, int depth, bool full, uint32_t *out) {
    const int words = (t.E + 31) / 32;
    for (int w = 0; w < words; ++w) {
        const int rem = t.E - w * 32;
        out[w] = full ? (rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u)) : 0u;
    }
    if (full) return;
    const uint32_t *pred = t.last + layer * words;
    if (depth < 0) {
        for (int w = 0; w < words; ++w) out[w] = pred[w];
        return;
    }
    uint32_t bound = 0xffffffffu;   // keys already taken are >= bound
    for (int j = 0; j < depth; ++j) {
        uint32_t best = 0u;
        int be = -1;
        for (int w = 0; w < words; ++w)
            for (uint32_t v = pred[w]; v; v &= v - 1) {
                const int e = w * 32 + lru_ffs(v) - 1;
                const uint32_t k = lru_rank_key(t.lastcnt[layer * t.E + e], e);
                if (k < bound && k > best) { best = k; be = e; }
            }
        if (be < 0) break;
        out[be >> 5] |= 1u << (be & 31);
        bound = best;
    }
}

// A table update given the request bitmap `req` of `layer`.
// mode 0: resolve (counted); cnt (nullable): pairs per expert of this call, kept as the
//         ranking of the layer's prediction; then, if pf_req is given, a prefetch of
//         layer+1 with that request (lru_predict of layer+1, computed before this call).
// mode 1: prefetch (not counted).
// Output in io: [0] status (0 ok, MOE_ERR_CACHE_FULL), [1] n resolve loads, [2] n prefetch
// loads (-1 = not run or did not fit), then the (expert, slot) pairs of both.
LRU_HD inline void lru_run(LruTable &t, int layer, const uint32_t *req, const int32_t *cnt, int mode,
                           const uint32_t *pf_req, int32_t *io) {
    const int words = (t.E + 31) / 32;
    int32_t *pairs = io + 3;
    const int na = lru_call(t, layer, req, mode == 0, pairs);
    if (na < 0) {
        io[0] = MOE_ERR_CACHE_FULL;
        io[1] = 0;
        io[2] = -1;
        return;
    }
    io[0] = 0;
    io[1] = na;
    io[2] = -1;
    if (mode == 0) {
        for (int w = 0; w < words; ++w) t.last[layer * words + w] = req[w];
        for (int e = 0; e < t.E; ++e) t.lastcnt[layer * t.E + e] = cnt ? cnt[e] : 0;
        if (pf_req && layer + 1 < t.L) {
            const int nb = lru_call(t, layer + 1, pf_req, false, pairs + 2 * na);
            io[2] = nb;   // -1 when the prediction does not fit: skipped, not an error
        }
    }
}

// Resize the pool to S_new slots (1 <= S_new <= Smax), between calls (no slot may be
// in use by the device). Writes the slot moves (from, to) to moves[0..2n) and returns
// n; moves holds room for S_new pairs. Returns -1 for an S_new outside 1..Smax.
LRU_HD inline int lru_resize(LruTable &t, int S_new, int32_t *moves) {
    if (S_new < 1 || S_new > t.Smax) return -1;
    const int S = t.S;
    if (S_new >= S) {   // grow: the new slots are free
        for (int s = S; s < S_new; ++s) {
            t.owner[s] = kNone;
            t.prev[s] = t.next[s] = kNone;
            t.ref[s] = kNeverRef;
            t.freeb[s >> 5] |= 1u << (s & 31);
        }
        t.st[ST_FREE] += S_new - S;
        if (S_new > S && (S >> 5) < t.st[ST_HINT]) t.st[ST_HINT] = S >> 5;
        t.S = S_new;
        return 0;
    }
    // shrink: keep the S_new most recent experts (walk from the most recent end)
    const int occupied = S - t.st[ST_FREE];
    int keep = occupied < S_new ? occupied : S_new;
    int s = t.st[ST_TAIL];
    for (int i = 0; i < keep; ++i) s = t.prev[s];
    // s is now the most recent slot to drop; drop it and everything less recent
    while (s != kNone) {
        const int p = t.prev[s];
        lru_unlink(t, s);
        t.slot_of[t.owner[s]] = kNone;
        t.owner[s] = kNone;
        t.ref[s] = kNeverRef;
        t.freeb[s >> 5] |= 1u << (s & 31);
        s = p;
    }
    // move the kept experts above the new end, least recent first, to the lowest free slots
    int n = 0, f = 0;
    for (s = t.st[ST_HEAD]; s != kNone;) {
        const int nx = t.next[s];
        if (s >= S_new) {
            while (!((t.freeb[f >> 5] >> (f & 31)) & 1u)) ++f;   // f < S_new: the kept fit below
            const int p = t.prev[s];
            t.freeb[f >> 5] &= ~(1u << (f & 31));
            t.owner[f] = t.owner[s];
            t.ref[f] = t.ref[s];
            t.slot_of[t.owner[f]] = f;
            t.prev[f] = p;
            t.next[f] = nx;
            if (p != kNone) t.next[p] = f; else t.st[ST_HEAD] = f;
            if (nx != kNone) t.prev[nx] = f; else t.st[ST_TAIL] = f;
            t.owner[s] = kNone;
            t.prev[s] = t.next[s] = kNone;
            t.ref[s] = kNeverRef;
            t.freeb[s >> 5] |= 1u << (s & 31);
            moves[2 * n] = s;
            moves[2 * n + 1] = f;
            ++n;
        }
        s = nx;
    }
    // slots from S_new on leave the pool
    for (int q = S_new; q < S; ++q) t.freeb[q >> 5] &= ~(1u << (q & 31));
    t.S = S_new;
    int nfree = 0, nref = 0;
    const int c = t.st[ST_CALLS];
    for (int q = 0; q < S_new; ++q) {
        nfree += (t.freeb[q >> 5] >> (q & 31)) & 1u;
        nref += t.ref[q] == c - 1;
    }
    t.st[ST_FREE] = nfree;
    t.st[ST_HINT] = 0;
    t.st[ST_LASTN] = nref;
    return n;
}

// Prefetch plan of one cached call (host code). Policies as moe_prefetch_policy in
// moe.h. For the adaptive policy: a call whose T tokens and k experts per token are
// expected to touch at least half of the E experts (uniform routing:
// E (1 - (1 - k/E)^T)) streams the whole next layer, since that layer's next call
// will need nearly all of it; otherwise the depth is the number of experts the
// measured host-to-device rate moves in the measured compute time of a layer,
// floor(bw * t_comp / expert_bytes), or the whole prediction before anything has
// been measured. Returns the depth (-1 = the whole prediction); *full is set when
// the whole layer is streamed, *none when nothing is prefetched.
inline int lru_prefetch_plan(int policy, int depth, int T, int k, int E, double bw_bytes_s, double t_comp_s,
                             double expert_bytes, bool *full, bool *none) {
    *full = false;
    *none = false;
    switch (policy) {
    case MOE_PREFETCH_NONE: *none = true; return 0;
    case MOE_PREFETCH_FULL_LAYER: *full = true; return E;
    case MOE_PREFETCH_ADAPTIVE: {
        double miss = 1.0;   // probability that a given expert receives none of the T k pairs
        const double q = 1.0 - (double)k / (double)E;
        for (int t = 0; t < T && miss > 1e-6; ++t) miss *= q;
        if ((1.0 - miss) * E >= 0.5 * E) { *full = true; return E; }
        if (!(bw_bytes_s > 0.0) || !(t_comp_s > 0.0) || !(expert_bytes > 0.0)) return -1;
        const double d = bw_bytes_s * t_comp_s / expert_bytes;
        return d >= (double)E ? E : (int)d;
    }
    default: return depth < 0 ? -1 : (depth > E ? E : depth);   // MOE_PREFETCH_PREDICTED
    }
}

// Free the slots matching (layer, ids): ids in io[1..io[0]]; io[0] = -1 or layer = -1 means
// every expert of the layer, or every slot.
LRU_HD inline void lru_evict(LruTable &t, int layer, const int32_t *io) {
    const int n = io[0];
    for (int s = 0; s < t.S; ++s) {
        const int key = t.owner[s];
        if (key < 0) continue;
        const int l = key / t.E, e = key % t.E;
        if (layer >= 0 && l != layer) continue;
        if (layer >= 0 && n >= 0) {
            bool m = false;
            for (int i = 0; i < n; ++i) m |= io[1 + i] == e;
            if (!m) continue;
        }
        lru_unlink(t, s);
        t.slot_of[key] = kNone;
        t.owner[s] = kNone;
        t.ref[s] = kNeverRef;
        t.freeb[s >> 5] |= 1u << (s & 31);
        t.st[ST_FREE] += 1;
        if ((s >> 5) < t.st[ST_HINT]) t.st[ST_HINT] = s >> 5;
    }
    int nref = 0;
    const int c = t.st[ST_CALLS];
    for (int s = 0; s < t.S; ++s) nref += t.ref[s] == c - 1;
    t.st[ST_LASTN] = nref;
}

}  // namespace moe
