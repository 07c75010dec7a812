// Router logits, top-k selection and softmax gating.
//
// Each token activates k routed experts (winzheng.com page, section "Why Now of
// All Times"). The pages give no router formula; this library computes
//   l[t,e] = fp32( sum_h x[t,h] * Wr[h,e] ) + bias[e]
// with the products and the sum in fp64 (bf16*bf16 and bf16*fp32 products are
// exact in fp64) and one rounding to fp32, so the logits, and therefore the
// selected experts, do not depend on the summation order beyond fp64 rounding.
// Experts are ranked by logit (descending, ties to the lower index) and the
// gate weights are a softmax over the k selected logits.
//
// Up to 256 tokens: one launch of 8-CTA clusters that split H, reduce through
// distributed shared memory and finish with one warp per token (below).
// Larger batches: kernel 1 (partial) - fp64 tensor-core tiles of 64 tokens x
// 64 experts x one slice of H, fp64 partial sums to the workspace; kernel 2
// (finish) - one warp per token adds the partials in slice order, rounds, adds
// the bias, selects the top k and writes idx, w (and optionally the logits).
#include <cooperative_groups.h>

#include "common.cuh"
#include <algorithm>
#include <mutex>

#include "internal.h"
#include "permute_small.cuh"
#include "mx_codec.cuh"

namespace moe {

// Partial-sum kernel (fp64 tensor core): a block owns 64 tokens x 64 experts x
// one slice of H; the slice count is chosen so the grid fills the GPU a few
// times over. fp64 x and Wr tiles of 32 rows go through shared memory (double
// buffered); each warp accumulates a 32 x 32 (token, expert) tile with
// mma.sync.m8n8k4.f64, whose products of bf16 / fp32 inputs are exact and
// whose sums are fp64 in a fixed order.
constexpr int kDT = 64;          // tokens per block
constexpr int kDE = 64;          // experts per block
constexpr int kDK = 32;          // H rows per shared-memory stage
constexpr int kDThreads = 128;
constexpr int kXS = kDK + 4;     // x tile row stride (doubles): conflict-free A fragments
constexpr int kWS = kDE + 4;     // Wr tile row stride (doubles): conflict-free B fragments
constexpr int kTargetBlocks = 444;   // three blocks per SM of a 148-SM B200

static void router_split(int T, int H, int E, int *S, int *slice) {
    const int tiles = ((T + kDT - 1) / kDT) * ((E + kDE - 1) / kDE);
    // The split of H with the shortest estimated time, among splits up to about two waves of
    // blocks (at least 4; this bounds the fp64 partial sums): an SM runs 3 blocks at once at the
    // full fp64 tensor rate, 2 at about 80% of it, 1 at about half, so a block count just above
    // a multiple of 3 per SM leaves a slow tail (at prefill, 4 slices give 512 blocks: 68 SMs
    // run a 4th block alone).
    const int maxs = std::min(std::max(4, (2 * kTargetBlocks + tiles - 1) / tiles), (H + kDK - 1) / kDK);
    int s = 1;
    double best = 0.0;
    for (int c = 1; c <= maxs; ++c) {
        const int64_t blocks = (int64_t)tiles * c;
        const int64_t per_sm = (blocks + kTargetBlocks / 3 - 1) / (kTargetBlocks / 3);
        const double rounds = 3.0 * (double)(per_sm / 3) + (per_sm % 3 == 1 ? 2.0 : (per_sm % 3 == 2 ? 2.5 : 0.0));
        const double t = rounds / (double)blocks;   // in units of the whole router's work
        if (c == 1 || t < best - 1e-12) {
            best = t;
            s = c;
        }
    }
    int sl = (H + s - 1) / s;
    sl = (sl + kDK - 1) / kDK * kDK;
    *slice = sl;
    *S = (H + sl - 1) / sl;
}

size_t router_ws_bytes(int T, int H, int E) {
    if (T <= 0) return 0;
    int S, slice;
    router_split(T, H, E, &S, &slice);
    return align_up((size_t)S * T * E * sizeof(double), 256);
}

size_t router_ws_bound(int T, int H, int E) {
    // The split depends only on the tile count, so between tile boundaries the partials grow
    // with T; the largest over smaller batches sits at one of the boundaries below T.
    size_t m = router_ws_bytes(T, H, E);
    for (int t = kDT; t < T; t += kDT) m = std::max(m, router_ws_bytes(t, H, E));
    return m;
}

__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

// Exact widening to fp64 by moving the bit fields (the exponent is rebiased by
// 1023 - 127 = 896); zeros, subnormals, infinities and NaNs (exponent field 0
// or all ones) take the conversion instruction, which keeps Inf and NaN.
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) {
    const uint32_t ex = b & 0x7F80u;
    if (ex == 0 || ex == 0x7F80u) return (double)__uint_as_float(b << 16);
    const uint32_t hi = ((b & 0x8000u) << 16) | (((b & 0x7FFFu) << 13) + (896u << 20));
    return __hiloint2double((int)hi, 0);
}

__device__ __forceinline__ double f32_bits_to_f64(uint32_t f) {
    const uint32_t ex = f & 0x7F800000u;
    if (ex == 0 || ex == 0x7F800000u) return (double)__uint_as_float(f);
    const uint32_t hi = (f & 0x80000000u) | (((f & 0x7FFFFFFFu) >> 3) + (896u << 20));
    return __hiloint2double((int)hi, (int)(f << 29));
}

template <bool WR32>
__global__ void __launch_bounds__(kDThreads) router_dmma_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H,
                                                               const void *__restrict__ wr, int E, int slice,
                                                               int wvec, double *__restrict__ part) {
    extern __shared__ __align__(16) double dsm[];
    pdl_wait();
    pdl_release();
    double *xs = dsm;                        // [2][kDT * kXS]
    double *ws = dsm + 2 * kDT * kXS;        // [2][kDK * kWS]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * kDT, e0 = blockIdx.y * kDE, sl = blockIdx.z;
    const int hb = sl * slice, he = min(H, hb + slice);
    const int wt = warp >> 1, we = warp & 1;      // warp tile: tokens 32 wt.., experts 32 we..
    const int gq = lane >> 2, cq = lane & 3;      // fragment row / column of this lane

    // staging: thread -> x row (tid / 2), 16 consecutive h; Wr row (tid / 4), 16 consecutive experts
    const int xr = tid >> 1, xh = (tid & 1) * 16;
    const int wrow = tid >> 2, we16 = (tid & 3) * 16;
    double xv[16], wv[16];
    auto load = [&](int kc) {
        const int t = t0 + xr;
        const int h = kc + xh;
        if (t < T && h + 16 <= he) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)t * H + h);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint4 u = src[q];
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xv[q * 8 + 2 * i] = bf16_bits_to_f64(w4[i] & 0xFFFFu);
                    xv[q * 8 + 2 * i + 1] = bf16_bits_to_f64(w4[i] >> 16);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                xv[i] = (t < T && h + i < he)
                            ? bf16_bits_to_f64(reinterpret_cast<const uint16_t *>(x)[(int64_t)t * H + h + i])
                            : 0.0;
        }
        const int kr = kc + wrow;
        const int e = e0 + we16;
        if (wvec && kr < he && e + 16 <= E) {   // wvec: Wr rows are a multiple of 16 bytes
            if (WR32) {
                const uint4 *src = reinterpret_cast<const uint4 *>(reinterpret_cast<const float *>(wr) + (int64_t)kr * E + e);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 u = src[q];
                    wv[q * 4 + 0] = f32_bits_to_f64(u.x);
                    wv[q * 4 + 1] = f32_bits_to_f64(u.y);
                    wv[q * 4 + 2] = f32_bits_to_f64(u.z);
                    wv[q * 4 + 3] = f32_bits_to_f64(u.w);
                }
            } else {
                const uint4 *src =
                    reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(wr) + (int64_t)kr * E + e);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint4 u = src[q];
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        wv[q * 8 + 2 * i] = bf16_bits_to_f64(w4[i] & 0xFFFFu);
                        wv[q * 8 + 2 * i + 1] = bf16_bits_to_f64(w4[i] >> 16);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                double v = 0.0;
                if (kr < he && e + i < E)
                    v = WR32 ? f32_bits_to_f64(reinterpret_cast<const uint32_t *>(wr)[(int64_t)kr * E + e + i])
                             : bf16_bits_to_f64(reinterpret_cast<const uint16_t *>(wr)[(int64_t)kr * E + e + i]);
                wv[i] = v;
            }
        }
    };
    auto store = [&](int b) {
        double *xd = xs + b * kDT * kXS + xr * kXS + xh;
        double *wd = ws + b * kDK * kWS + wrow * kWS + we16;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            *reinterpret_cast<double2 *>(xd + i) = make_double2(xv[i], xv[i + 1]);
            *reinterpret_cast<double2 *>(wd + i) = make_double2(wv[i], wv[i + 1]);
        }
    };

    double acc[4][4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

    int b = 0;
    if (hb < he) {
        load(hb);
        store(0);
    }
    __syncthreads();
    for (int kc = hb; kc < he; kc += kDK) {
        const bool more = kc + kDK < he;
        if (more) load(kc + kDK);   // next stage in flight during the MMAs
        const double *xa = xs + b * kDT * kXS + (32 * wt + gq) * kXS + cq;
        const double *wb = ws + b * kDK * kWS + cq * kWS + 32 * we + gq;
#pragma unroll
        for (int ks = 0; ks < kDK; ks += 4) {
            double a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xa[i * 8 * kXS + ks];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = wb[ks * kWS + j * 8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[i][j], a[i], bb[j]);
        }
        if (more) {
            store(b ^ 1);
            b ^= 1;
        }
        __syncthreads();
    }
    // partial sums: lane holds rows gq, columns 2 cq, 2 cq + 1 of each 8 x 8 tile
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 32 * wt + 8 * i + gq;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + 32 * we + 8 * j + 2 * cq;
            double *dst = part + ((int64_t)sl * T + t) * E + e;
            if (e + 1 < E) {
                dst[0] = acc[i][j][0];
                dst[1] = acc[i][j][1];
            } else if (e < E) {
                dst[0] = acc[i][j][0];
            }
        }
    }
}

// Order-preserving 32-bit key of an fp32 logit (larger logit, larger key);
// -0 is folded into +0 so that equal logits always tie.
__device__ __forceinline__ uint32_t logit_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Warp-wide top-k of the logits held as v[i] for expert lane + 32 i (experts
// >= E excluded), descending, ties to the lower expert index, and the softmax
// over the k selected logits. Each round takes the largest key with one
// redux.sync and, among the lanes holding it, the lowest expert with a second;
// the selection stays in registers. Lanes j < k write idx_row[j], w_row[j].
__device__ __forceinline__ void topk_softmax_warp(float (&v)[kMaxRouterExperts / 32], int E, int k, int lane,
                                                  int32_t *idx_row, float *w_row) {
    constexpr int kPer = kMaxRouterExperts / 32;
    uint32_t key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) key[i] = lane + 32 * i < E ? logit_key(v[i]) : 0u;
    float selv[kMaxTopK];
    int seli[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        selv[j] = 0.0f;
        seli[j] = 0;
        if (j < k) {
            // this lane's best remaining expert (lowest index among equal keys)
            uint32_t bk = 0u;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (key[i] > bk) { bk = key[i]; bi = lane + 32 * i; }
            const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
            const int win = (int)__reduce_min_sync(0xffffffffu, bk == mk ? (uint32_t)bi : 0x7fffffffu);
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (lane + 32 * i == win) key[i] = 0u;   // taken
            selv[j] = key_logit(mk);
            seli[j] = win;
        }
    }
    // softmax over the selected logits, summed in selection order
    const float l0 = selv[0];
    float z = 0.0f, mine = 0.0f;
    int myidx = 0;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
            const float e = expf(selv[j] - l0);
            z += e;
            if (j == lane) { mine = e; myidx = seli[j]; }
        }
    }
    if (lane < k) {
        idx_row[lane] = myidx;
        w_row[lane] = mine / z;
    }
}

__global__ void __launch_bounds__(256) router_finish_kernel(const double *__restrict__ part, int S, int T, int E,
                                                           const float *__restrict__ bias, int k,
                                                           int32_t *__restrict__ idx, float *__restrict__ w,
                                                           float *__restrict__ logits) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    constexpr int kPer = kMaxRouterExperts / 32;
    // the partial sums of four slices for all of this lane's experts are loaded at once, then
    // added in slice order (the same fp64 order as one slice at a time)
    double sum[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) sum[i] = 0.0;
    for (int s0 = 0; s0 < S; s0 += 4) {
        double a[4][kPer];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int e = lane + 32 * i;
                a[j][i] = (s0 + j < S && e < E) ? __ldg(part + ((int64_t)(s0 + j) * T + t) * E + e) : 0.0;
            }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (s0 + j < S) {
#pragma unroll
                for (int i = 0; i < kPer; ++i) sum[i] += a[j][i];
            }
    }
    float v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        v[i] = 0.0f;
        if (e < E) {
            float l = (float)sum[i];
            if (bias) l = l + bias[e];
            v[i] = l;
            if (logits) logits[(int64_t)t * E + e] = l;
        }
    }
    topk_softmax_warp(v, E, k, lane, idx + (int64_t)t * k, w + (int64_t)t * k);
}

// Small batches (T <= 256): one kernel, clusters of 8 CTAs. The 8 CTAs of a
// cluster share a tile of TT tokens and split H into 8 contiguous slices; CTA r
// streams rows [r H/8, (r+1) H/8) of Wr into shared memory with bulk copies (a
// ring of chunks) and keeps fp64 sums for (token, expert) in registers: thread
// (g, e) owns expert e for every token of the tile over the g-th part of each
// chunk. The G parts are added in g order inside the CTA, then the 8 CTA sums in
// rank order through distributed shared memory, so the result is one fixed
// fp64 summation order. One warp per token rounds, biases and selects the top k.
//
// With fz.ticket set (the layer forward), the routing and the permutation run
// in this one kernel: every cluster publishes its tokens' top-k and takes a
// ticket, and the cluster that takes the last ticket sorts all T k pairs by
// expert (small_permute). No cluster waits on another.
constexpr int kRCl = 8;              // CTAs per cluster (H slices)
constexpr int kRClThreads = 256;
constexpr int kRClChunkMax = 24576;  // bytes of Wr per ring chunk
constexpr int kRClRing = 4;
constexpr int kTokenKernelMaxT = 256;

struct RouterClusterShape {
    int TT;      // tokens per cluster tile (1, 2, 4, 8 or 16)
    int EPP;     // threads per row group: E / 4 experts each, rounded up to a warp
    int G;       // row groups per chunk (kRClThreads / EPP)
    int hs;      // rows per CTA (H / 8)
    int RC;      // rows per chunk
    int nch;     // chunks per CTA
    size_t smem;
};

static bool router_cluster_shape(int T, int H, int E, int wr_is_fp32, RouterClusterShape *sh) {
    if (T > kTokenKernelMaxT || H % kRCl || E % 4) return false;
    const int eb = wr_is_fp32 ? 4 : 2;
    if ((E * eb) % 16) return false;
    sh->EPP = (E / 4 + 31) / 32 * 32;
    sh->G = kRClThreads / sh->EPP;
    sh->hs = H / kRCl;
    // Tokens per cluster: every cluster reads all of Wr, so the clusters are capped at 18 and at
    // 16 MB of Wr read in all (decode dims, 512 KB of Wr: 16 clusters at T = 64; Large, 2 MB:
    // 8 clusters at T = 32, measured 0.168 ms per layer against 0.176 with 16)
    const int64_t wr_bytes = (int64_t)H * E * eb;
    const int maxcl = (int)std::max<int64_t>(1, std::min<int64_t>(18, (16ll << 20) / wr_bytes));
    int TT = 1;
    while (TT < 16 && (T + TT - 1) / TT > maxcl) TT *= 2;
    sh->TT = TT;
    int rc = kRClChunkMax / (E * eb);
    if (rc > sh->hs) rc = sh->hs;
    int p = 1;
    while (p * 2 <= rc) p *= 2;
    while (p >= 4 * sh->G && (sh->hs % p || p % (4 * sh->G))) p /= 2;   // 4 rows per thread and step
    if (p < 4 * sh->G) return false;
    sh->RC = p;
    sh->nch = sh->hs / p;
    const size_t ring = (size_t)kRClRing * p * E * eb;
    const size_t red = (size_t)TT * sh->G * 4 * sh->EPP * sizeof(double);
    sh->smem = 64 + (ring > red ? ring : red) + (size_t)sh->hs * TT * sizeof(double);
    return sh->smem <= 200 * 1024;
}

// Ticket counters of the fused routing + permutation, one per stream (see
// route_ticket): zero when the module loads, and every fused launch leaves its
// counter at zero again (the last cluster resets it), so a launch counts from 0.
constexpr int kTicketSlots = 256;
__device__ unsigned int g_route_ticket[kTicketSlots];
// Per-expert row counts of the slot layout, one set per stream slot: zero when the module
// loads; the layer's combine clears them after the grouped FFN has read them.
__device__ int32_t g_slot_count[kTicketSlots * kMaxRouterExperts];

template <bool WR32, int TT>
__global__ void __cluster_dims__(kRCl, 1, 1) __launch_bounds__(kRClThreads)
    router_cluster_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H, const void *__restrict__ wr, int E,
                          int EPP, int G, int RC, int nch, const float *__restrict__ bias, int k,
                          int32_t *__restrict__ idx, float *__restrict__ w, float *__restrict__ logits,
                          RouterFuse fz) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int eb = WR32 ? 4 : 2;
    __shared__ int2 s_dest[16][kMaxTopK];   // slot layout: (tile, row) of each pair of the tile's tokens
    extern __shared__ __align__(128) uint8_t rsm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(rsm);            // [kRClRing]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(rsm + 48);
    const int hs = H / kRCl;
    const size_t chunk_bytes = (size_t)RC * E * eb;
    const size_t ring = (size_t)kRClRing * chunk_bytes;
    const int E2 = 4 * EPP;                                        // expert slots per row group
    const size_t red_bytes = (size_t)TT * G * E2 * sizeof(double);
    uint8_t *wring = rsm + 64;
    double *red = reinterpret_cast<double *>(rsm + 64);              // aliases the ring after the loop
    double *xs = reinterpret_cast<double *>(rsm + 64 + (ring > red_bytes ? ring : red_bytes));   // [hs][TT]
    // slot layout: the four-plane codes and plane scales of this CTA's slice of each token's row,
    // [TT][hs / 256 stages][4 planes] x (32 words, 8 scale bytes), after the x tile
    const int nls = hs / kMxStageK;
    uint32_t *pcode = reinterpret_cast<uint32_t *>(
        (reinterpret_cast<uintptr_t>(xs + (size_t)hs * TT) + 15) & ~uintptr_t(15));
    uint8_t *pscale = reinterpret_cast<uint8_t *>(pcode + (size_t)TT * nls * kMxPlanes * 32);

    const int tid = threadIdx.x;
    const int rank = (int)cluster.block_rank();
    const int t0 = blockIdx.y * TT;
    const int h0 = rank * hs;
    const uint8_t *wsrc = reinterpret_cast<const uint8_t *>(wr) + (size_t)h0 * E * eb;

    if (tid == 0) {
        for (int b = 0; b < kRClRing; ++b) mbar_init(&full[b], 1);
        *abort_flag = 0;
        fence_mbar_init();
        for (int c = 0; c < nch && c < kRClRing; ++c) {
            mbar_expect_tx(&full[c], (uint32_t)chunk_bytes);
            bulk_load(wring + c * chunk_bytes, wsrc + c * chunk_bytes, (uint32_t)chunk_bytes, &full[c]);
        }
    }
    // Wr is static and already on its way; x comes from the previous kernel
    pdl_wait();
    pdl_release();
    if (fz.sched_zero && blockIdx.x == 0 && blockIdx.y == 0 && tid < 2) fz.sched_zero[tid] = 0;
    // x tile -> shared, as fp64 (exact), layout [h][tt]; tokens past T are zero. Up to 8
    // loads per thread are in flight before the first conversion.
    for (int i0 = 0; i0 < hs * TT; i0 += 8 * kRClThreads) {
        uint16_t xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRClThreads + tid;
            const int tt = i / hs, h = i - tt * hs;
            xv[u] = (i < hs * TT && t0 + tt < T) ? reinterpret_cast<const uint16_t *>(x)[(int64_t)(t0 + tt) * H + h0 + h]
                                                  : (uint16_t)0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRClThreads + tid;
            const int tt = i / hs, h = i - tt * hs;
            if (i < hs * TT) xs[h * TT + tt] = bf16_bits_to_f64(xv[u]);
        }
    }
    __syncthreads();
    if (fz.cnt) {
        // The activation rows in the four-plane MXFP4 form do not depend on the routing: this CTA's
        // slice of them is made now, while the Wr slices stream in. One warp per (token, stage),
        // 8 elements per lane, 4 lanes per 32-block.
        const int wq = tid >> 5, lq = tid & 31;
        for (int item = wq; item < TT * nls; item += kRClThreads / 32) {
            const int tt2 = item / nls, ls = item - tt2 * nls;
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = (float)xs[(ls * kMxStageK + lq * 8 + i) * TT + tt2];
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const int s = mx_plane0_exp(amax);
            uint32_t pw[kMxPlanes];
            mx_planes8(v, s, pw);
#pragma unroll
            for (int pl = 0; pl < kMxPlanes; ++pl) {
                pcode[(item * kMxPlanes + pl) * 32 + lq] = pw[pl];
                if ((lq & 3) == 0) pscale[(item * kMxPlanes + pl) * 8 + (lq >> 2)] = (uint8_t)(s - 3 * pl);
            }
        }
    }

    // thread (g, ep) owns experts 4 ep .. 4 ep + 3 for every token of the tile over
    // rows [g rows_g, (g + 1) rows_g) of each chunk (a row group is whole warps, so
    // a warp reads one row of x at a time: a broadcast). Four rows' weights are
    // loaded before their FMAs; NA independent fp64 sums per (token, expert) keep
    // at least 8 chains in flight, added in order at the end.
    const int ep = tid % EPP, g = tid / EPP;
    const bool active = g < G && 4 * ep < E;
    const int rows_g = RC / G;   // a multiple of 4
    constexpr int NA = TT >= 2 ? 1 : 2;
    double acc[TT][4][NA];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
#pragma unroll
            for (int a = 0; a < NA; ++a) acc[tt][e4][a] = 0.0;
    for (int c = 0; c < nch; ++c) {
        const int b = c % kRClRing;
        mbar_wait(&full[b], (uint32_t)((c / kRClRing) & 1), abort_flag);
        if (active) {
            const uint8_t *wc = wring + b * chunk_bytes + (size_t)4 * ep * eb;
            const int rb = g * rows_g;
            for (int r0 = rb; r0 < rb + rows_g; r0 += 4) {
                double wv[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint8_t *src = wc + (size_t)(r0 + i) * E * eb;
                    if (WR32) {
                        const uint4 f = *reinterpret_cast<const uint4 *>(src);
                        wv[i][0] = f32_bits_to_f64(f.x);
                        wv[i][1] = f32_bits_to_f64(f.y);
                        wv[i][2] = f32_bits_to_f64(f.z);
                        wv[i][3] = f32_bits_to_f64(f.w);
                    } else {
                        const uint2 bb = *reinterpret_cast<const uint2 *>(src);
                        wv[i][0] = bf16_bits_to_f64(bb.x & 0xFFFFu);
                        wv[i][1] = bf16_bits_to_f64(bb.x >> 16);
                        wv[i][2] = bf16_bits_to_f64(bb.y & 0xFFFFu);
                        wv[i][3] = bf16_bits_to_f64(bb.y >> 16);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double *xr = xs + (size_t)(c * RC + r0 + i) * TT;
                    const int a = i % NA;
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt) {
                        const double xv = xr[tt];
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) acc[tt][e4][a] = fma(xv, wv[i][e4], acc[tt][e4][a]);
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0 && c + kRClRing < nch) {
            mbar_expect_tx(&full[b], (uint32_t)chunk_bytes);
            bulk_load(wring + b * chunk_bytes, wsrc + (size_t)(c + kRClRing) * chunk_bytes, (uint32_t)chunk_bytes,
                      &full[b]);
        }
    }
    // CTA sum over the row groups, in g order: red[tt][g][e]
    if (g < G) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
                double sum = acc[tt][e4][0];
#pragma unroll
                for (int a = 1; a < NA; ++a) sum += acc[tt][e4][a];
                red[((size_t)tt * G + g) * E2 + 4 * ep + e4] = sum;
            }
    }
    __syncthreads();
    if (tid < E) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            double sum = red[((size_t)tt * G) * E2 + tid];
            for (int gg = 1; gg < G; ++gg) sum += red[((size_t)tt * G + gg) * E2 + tid];
            red[((size_t)tt * G) * E2 + tid] = sum;
        }
    }
    // cluster sum in rank order; token tt of the tile is finished by CTA tt % 8, warp tt / 8
    constexpr int kPer = kMaxRouterExperts / 32;
    const int warp = tid >> 5, lane = tid & 31;
    const int tt = rank + kRCl * warp;
    const bool fin = tt < TT && t0 + tt < T;
    float bv[kPer];   // bias, loaded before the cluster barrier
#pragma unroll
    for (int i = 0; i < kPer; ++i) bv[i] = (fin && bias && lane + 32 * i < E) ? bias[lane + 32 * i] : 0.0f;
    cluster.sync();
    if (fin) {
        const int t = t0 + tt;
        const double *src[kRCl];
#pragma unroll
        for (int q = 0; q < kRCl; ++q) src[q] = cluster.map_shared_rank(red, q) + (size_t)tt * G * E2;
        float v[kPer];
#pragma unroll
        for (int i0 = 0; i0 < kPer; i0 += 4) {
            // all remote partial sums of four experts per lane in flight, then added in rank order
            double parts[4][kRCl];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < kRCl; ++q)
                    parts[i][q] = lane + 32 * (i0 + i) < E ? src[q][lane + 32 * (i0 + i)] : 0.0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ee = lane + 32 * (i0 + i);
                v[i0 + i] = 0.0f;
                if (ee < E) {
                    double sum = parts[i][0];
#pragma unroll
                    for (int q = 1; q < kRCl; ++q) sum += parts[i][q];
                    float l = (float)sum;
                    if (bias) l = l + bv[i0 + i];
                    v[i0 + i] = l;
                    if (logits) logits[(int64_t)t * E + ee] = l;
                }
            }
        }
        topk_softmax_warp(v, E, k, lane, idx + (int64_t)t * k, w + (int64_t)t * k);
        if (fz.ticket) __threadfence();   // the top-k is visible before this cluster's ticket
        if (fz.cnt) {
            // slot layout: each pair takes the next row of its expert's slot (the experts of a
            // token are distinct, so a slot never holds more than T rows); the tile and row it
            // lands in are left for the cluster's CTAs, which write the activation rows below
            if (lane < k) {
                const int e = idx[(int64_t)t * k + lane];   // written by this lane just above
                const int pos = atomicAdd(fz.cnt + e, 1);
                fz.pair_row[(int64_t)t * k + lane] = e * T + pos;
                s_dest[tt][lane] = make_int2(e * fz.mt + pos / fz.BN, pos % fz.BN);
            }
        }
    }
    cluster.sync();   // keep this CTA's shared memory alive until every peer has read it
    if (fz.cnt) {
        // Slot layout: every CTA copies its slice of each token's activation row (the codes made
        // above: whole 256-wide stages) into the tiles of the token's k rows; the destinations come
        // from the CTA that finished the token (rank tt % 8). Lane L moves 16-byte chunk L % 8 of
        // plane L / 8 and that 32-block's plane scale.
        const int st0 = h0 / kMxStageK, KST = H / kMxStageK;
        const int BB = bs_bblob_bytes(kBsMx, fz.BN), NROW = kMxPlanes * fz.BN;
        const int pl = lane >> 3, c = lane & 7;
        for (int item = warp; item < TT * nls; item += kRClThreads / 32) {
            const int tt2 = item / nls, ls = item - tt2 * nls;
            if (t0 + tt2 >= T) continue;   // warp-uniform
            const int2 *rd = cluster.map_shared_rank(&s_dest[0][0], tt2 % kRCl) + tt2 * kMaxTopK;
            const int2 dj = lane < k ? rd[lane] : make_int2(0, 0);
            const uint4 cw = *reinterpret_cast<const uint4 *>(pcode + (item * kMxPlanes + pl) * 32 + c * 4);
            const uint8_t sc = pscale[(item * kMxPlanes + pl) * 8 + c];
            const int st = st0 + ls;
            for (int j = 0; j < k; ++j) {
                const int tile = __shfl_sync(0xffffffffu, dj.x, j), n = __shfl_sync(0xffffffffu, dj.y, j);
                uint8_t *blob = fz.bslab + ((int64_t)tile * KST + st) * BB;
                const int Rw = pl * fz.BN + n;
                *reinterpret_cast<uint4 *>(blob + sw128_chunk(Rw, c)) = cw;
                blob[NROW * 128 + (c >> 2) * 512 + atom_offset(Rw, c & 3)] = sc;
            }
        }
        cluster.sync();   // every peer has read this CTA's destinations
    }
    if (fz.ticket && rank == 0) {
        __shared__ int s_last;
        if (tid == 0) {
            s_last = atomicAdd(fz.ticket, 1u) + 1u == gridDim.y;
            if (s_last) __threadfence();
        }
        __syncthreads();
        if (s_last) {   // the ring and the sums are no longer needed: their space is the scratch
            auto &ps = *reinterpret_cast<SmallPermuteSmem<kRClThreads> *>(rsm + 64);
            int32_t *sidx = reinterpret_cast<int32_t *>(rsm + 64 + sizeof(SmallPermuteSmem<kRClThreads>));
            small_permute<kRClThreads>(idx, T * k, E, fz.offsets, fz.sorted_pair, fz.pair_row, ps, sidx);
            if (tid == 0) atomicExch(fz.ticket, 0u);   // ready for the next launch on this counter
        }
    }
}

template <bool WR32, int TT>
static cudaError_t launch_router_cluster_t(const RouterClusterShape &sh, const void *x, int T, int H, const void *wr,
                                           int E, const float *bias, int k, int32_t *idx, float *w, float *logits,
                                           const RouterFuse &fz, cudaStream_t st) {
    auto kern = router_cluster_kernel<WR32, TT>;
    size_t smem = sh.smem;
    const size_t perm_smem = 64 + sizeof(SmallPermuteSmem<kRClThreads>) + (size_t)T * k * sizeof(int32_t);
    if (fz.ticket && smem < perm_smem) smem = perm_smem;
    // slot layout: the plane codes and scales after the x tile (16-byte aligned)
    if (fz.cnt) smem += 16 + (size_t)TT * (sh.hs / kMxStageK) * kMxPlanes * (32 * 4 + 8);
    if (smem > 48 * 1024) {
        cudaError_t e = ensure_max_smem<router_cluster_kernel<WR32, TT>>((int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(kRCl, (T + TT - 1) / TT);
    cudaError_t e = launch_pdl(kern, grid, dim3(kRClThreads), smem, st, reinterpret_cast<const __nv_bfloat16 *>(x),
                               T, H, wr, E, sh.EPP, sh.G, sh.RC, sh.nch, bias, k, idx, w, logits, fz);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

template <bool WR32>
static cudaError_t launch_router_cluster(const RouterClusterShape &sh, const void *x, int T, int H, const void *wr,
                                         int E, const float *bias, int k, int32_t *idx, float *w, float *logits,
                                         const RouterFuse &fz, cudaStream_t st) {
    switch (sh.TT) {
    case 1: return launch_router_cluster_t<WR32, 1>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
    case 2: return launch_router_cluster_t<WR32, 2>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
    case 4: return launch_router_cluster_t<WR32, 4>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
    case 8: return launch_router_cluster_t<WR32, 8>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
    default: return launch_router_cluster_t<WR32, 16>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
    }
}

// The ticket counter of (device, stream): launches on one stream run in order, so
// one counter per stream is never shared by two launches at once. Slots are
// handed out per (device, stream) on first use; a device holds kTicketSlots of
// them. Null once a device's slots are all taken (its later streams route and
// permute in two launches) or if the counters cannot be found.
static unsigned int *route_ticket(cudaStream_t st);

// The slot-layout row counts of stream st (kMaxRouterExperts of them), or null.
int32_t *route_slot_counts(cudaStream_t st) {
    static std::mutex mu;
    static int32_t *base[64] = {};
    static unsigned int *tbase[64] = {};
    unsigned int *tk = route_ticket(st);
    int dev = 0;
    if (!tk || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!base[dev]) {
        void *p = nullptr, *q = nullptr;
        if (cudaGetSymbolAddress(&p, g_slot_count) != cudaSuccess) return nullptr;
        if (cudaGetSymbolAddress(&q, g_route_ticket) != cudaSuccess) return nullptr;
        base[dev] = reinterpret_cast<int32_t *>(p);
        tbase[dev] = reinterpret_cast<unsigned int *>(q);
    }
    return base[dev] + (size_t)(tk - tbase[dev]) * kMaxRouterExperts;
}

bool router_cluster_ok(int T, int H, int E, int wr_is_fp32, const void *wr) {
    RouterClusterShape sh;
    return router_cluster_shape(T, H, E, wr_is_fp32, &sh) && (reinterpret_cast<uintptr_t>(wr) & 15) == 0;
}

static unsigned int *route_ticket(cudaStream_t st) {
    struct Slot { int dev; cudaStream_t st; int idx; };
    static std::mutex mu;
    static Slot slots[64 * kTicketSlots];
    static int nslots = 0, next_idx[64] = {};
    static unsigned int *base[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!base[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_ticket) != cudaSuccess) return nullptr;
        base[dev] = reinterpret_cast<unsigned int *>(p);
    }
    for (int i = 0; i < nslots; ++i)
        if (slots[i].dev == dev && slots[i].st == st) return base[dev] + slots[i].idx;
    // Every stream keeps its own counter: two streams sharing one could interleave
    // their tickets. Past kTicketSlots streams on a device, calls take the unfused
    // path (a separate permutation launch).
    if (next_idx[dev] >= kTicketSlots) return nullptr;
    const int idx = next_idx[dev]++;
    slots[nslots++] = Slot{dev, st, idx};
    return base[dev] + idx;
}

moe_status launch_router(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                         int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes, int nsm,
                         cudaStream_t st, const RouterFuse *fuse, int *fused) {
    if (fused) *fused = 0;
    if (T == 0) return MOE_OK;
    RouterClusterShape sh;
    if (router_cluster_shape(T, H, E, wr_is_fp32, &sh) && (reinterpret_cast<uintptr_t>(wr) & 15) == 0) {
        // the permutation joins this kernel when asked for and small enough for one block
        RouterFuse fz{};
        if (fuse && fuse->cnt) {   // slot layout: no permutation
            fz = *fuse;
            fz.ticket = nullptr;
        } else if (fuse && (int64_t)T * k <= kSmallP && E <= kSmallE) {
            fz = *fuse;
            fz.cnt = nullptr;
            fz.ticket = route_ticket(st);
        }
        cudaError_t e = wr_is_fp32
                            ? launch_router_cluster<true>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st)
                            : launch_router_cluster<false>(sh, x, T, H, wr, E, bias, k, idx, w, logits, fz, st);
        if (e != cudaSuccess) return set_cuda_error(e, "router_cluster launch");
        if (fused) *fused = fz.cnt ? 2 : (fz.ticket != nullptr);
        return MOE_OK;
    }
    int S, slice;
    router_split(T, H, E, &S, &slice);
    (void)nsm;
    const size_t need = (size_t)S * T * E * sizeof(double);
    if (ws_bytes < need) return set_error(MOE_ERR_OOM, "router workspace too small (%zu < %zu)", ws_bytes, need);
    double *part = reinterpret_cast<double *>(ws);
    dim3 grid((T + kDT - 1) / kDT, (E + kDE - 1) / kDE, S);
    const int smem = (int)((2 * kDT * kXS + 2 * kDK * kWS) * sizeof(double));
    auto kfn = wr_is_fp32 ? router_dmma_kernel<true> : router_dmma_kernel<false>;
    cudaError_t e = wr_is_fp32 ? ensure_max_smem<router_dmma_kernel<true>>(smem)
                               : ensure_max_smem<router_dmma_kernel<false>>(smem);
    if (e != cudaSuccess) return set_cuda_error(e, "router smem attribute");
    const int wvec = (E * (wr_is_fp32 ? 4 : 2)) % 16 == 0;
    e = launch_pdl(kfn, grid, dim3(kDThreads), smem, st, reinterpret_cast<const __nv_bfloat16 *>(x), T, H, wr, E, slice,
                   wvec, part);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_dmma launch");
    e = launch_pdl(router_finish_kernel, dim3((T + 7) / 8), dim3(256), 0, st, (const double *)part, S, T, E, bias, k,
                   idx, w, logits);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_finish launch");
    return MOE_OK;
}

}  // namespace moe
