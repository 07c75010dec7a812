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

// slot_of[L*E]: slot of (layer, expert) or -1; owner[S]: key layer*E+e of a slot or -1;
// prev/next[S]: the intrusive recency list (head = least recent); ref[S]: index of the
// last call that referenced the slot; freeb[ceil(S/32)]: free-slot bitmap;
// last[L][ceil(E/32)]: experts each layer used at its last resolve (the prefetch
// prediction); st[ST_N]: head, tail, calls, free count, first bitmap word that may
// hold a free slot, slots referenced by the last call; counts: hits, misses.
struct LruTable {
    int32_t *slot_of, *owner, *prev, *next, *ref;
    uint32_t *freeb, *last;
    int32_t *st;
    unsigned long long *counts;
    int S, E, L;
};

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

// Table state of a fresh cache, element i of every array (i over max(L*E, S, L*ceil(E/32))).
LRU_HD inline void lru_init_one(LruTable &t, int i) {
    if (i < t.L * t.E) t.slot_of[i] = kNone;
    if (i < t.S) {
        t.owner[i] = kNone;
        t.prev[i] = t.next[i] = kNone;
        t.ref[i] = kNeverRef;
    }
    const int words = (t.S + 31) / 32;
    if (i < words) {
        const int rem = t.S - i * 32;
        t.freeb[i] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
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

// A table update given the request bitmap `req` of `layer`.
// mode 0: resolve (counted); then, if prefetch_next, a prefetch of layer+1's prediction.
// mode 1: prefetch (not counted).
// Output in io: [0] status (0 ok, MOE_ERR_CACHE_FULL), [1] n resolve loads, [2] n prefetch
// loads (-1 = not run or did not fit), then the (expert, slot) pairs of both.
LRU_HD inline void lru_run(LruTable &t, int layer, const uint32_t *req, int mode, int prefetch_next, int32_t *io) {
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
        if (prefetch_next && layer + 1 < t.L) {
            const int nb = lru_call(t, layer + 1, t.last + (layer + 1) * words, false, pairs + 2 * na);
            io[2] = nb;   // -1 when the prediction does not fit: skipped, not an error
        }
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
