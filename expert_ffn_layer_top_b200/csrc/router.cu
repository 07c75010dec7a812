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
// Larger batches: kernel 1 (partial) - a block owns 16 tokens x all experts x
// one slice of H, the slice count chosen so the grid fills the GPU, fp64 partial
// sums to the workspace; kernel 2 (finish) - one warp per token adds the
// partials in slice order, rounds, adds the bias, selects the top k with warp
// shuffles and writes idx, w (and optionally the logits).
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kTT = 16;   // tokens per block
constexpr int kHC = 16;   // H rows per shared-memory chunk
constexpr int kRThreads = 256;
constexpr int kMaxPairs = kTT * kMaxRouterExperts / kRThreads;   // (token, expert) pairs per thread

constexpr int kTargetBlocks = 296;   // two waves of a 148-SM B200

static void router_split(int T, int H, int *S, int *slice) {
    const int tb = (T + kTT - 1) / kTT;
    int s = (kTargetBlocks + tb - 1) / tb;
    const int maxs = H / kHC;
    if (s > maxs) s = maxs;
    if (s < 1) s = 1;
    int sl = (H + s - 1) / s;
    sl = (sl + kHC - 1) / kHC * kHC;
    *slice = sl;
    *S = (H + sl - 1) / sl;
}

size_t router_ws_bytes(int T, int H, int E) {
    if (T <= 0) return 0;
    int S, slice;
    router_split(T, H, &S, &slice);
    return align_up((size_t)S * T * E * sizeof(double), 256);
}

template <bool WR32>
__global__ void __launch_bounds__(kRThreads) router_partial_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H,
                                                                  const void *__restrict__ wr, int E, int slice,
                                                                  double *__restrict__ part) {
    __shared__ double xs[kTT][kHC];
    __shared__ double wsm[kHC][kMaxRouterExperts];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kTT;
    const int s = blockIdx.y;
    const int hb = s * slice;
    const int he = min(H, hb + slice);
    const int npairs = kTT * E;
    double acc[kMaxPairs];
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) acc[i] = 0.0;

    // per-thread share of one chunk: x (kTT*kHC = 256 values, one each) and Wr (kHC*E values)
    const int wper = (kHC * E + kRThreads - 1) / kRThreads;   // <= 16
    float xr;
    float wrr[kHC * kMaxRouterExperts / kRThreads];
    auto load_chunk = [&](int h0) {
        {
            const int tt = tid / kHC, hh = tid % kHC;
            const int t = t0 + tt, h = h0 + hh;
            xr = (t < T && h < he) ? __bfloat162float(x[(int64_t)t * H + h]) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kHC * kMaxRouterExperts / kRThreads; ++i) {
            if (i >= wper) break;
            const int li = tid + i * kRThreads;
            float v = 0.0f;
            if (li < kHC * E) {
                const int hh = li / E, e = li - hh * E;
                const int h = h0 + hh;
                if (h < he) {
                    v = WR32 ? reinterpret_cast<const float *>(wr)[(int64_t)h * E + e]
                             : __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(wr)[(int64_t)h * E + e]);
                }
            }
            wrr[i] = v;
        }
    };
    auto store_chunk = [&]() {
        xs[tid / kHC][tid % kHC] = (double)xr;
#pragma unroll
        for (int i = 0; i < kHC * kMaxRouterExperts / kRThreads; ++i) {
            if (i >= wper) break;
            const int li = tid + i * kRThreads;
            if (li < kHC * E) {
                const int hh = li / E, e = li - hh * E;
                wsm[hh][e] = (double)wrr[i];
            }
        }
    };

    if (hb < he) load_chunk(hb);
    for (int h0 = hb; h0 < he; h0 += kHC) {
        __syncthreads();
        store_chunk();
        __syncthreads();
        if (h0 + kHC < he) load_chunk(h0 + kHC);   // next chunk in flight during the math
#pragma unroll
        for (int i = 0; i < kMaxPairs; ++i) {
            const int q = tid + i * kRThreads;
            if (q < npairs) {
                const int tt = q / E, e = q - tt * E;
                double a = acc[i];
#pragma unroll
                for (int hh = 0; hh < kHC; ++hh) a = fma(xs[tt][hh], wsm[hh][e], a);
                acc[i] = a;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int q = tid + i * kRThreads;
        if (q < npairs) {
            const int tt = q / E, e = q - tt * E;
            const int t = t0 + tt;
            if (t < T) part[((int64_t)s * T + t) * E + e] = acc[i];
        }
    }
}

// Exact widening to fp64 by moving the bit fields (the exponent is rebiased by
// 1023 - 127 = 896); zeros and subnormals take the conversion instruction.
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) {
    if ((b & 0x7F80u) == 0) return (double)__uint_as_float(b << 16);
    const uint32_t hi = ((b & 0x8000u) << 16) | (((b & 0x7FFFu) << 13) + (896u << 20));
    return __hiloint2double((int)hi, 0);
}

__device__ __forceinline__ double f32_bits_to_f64(uint32_t f) {
    if ((f & 0x7F800000u) == 0) return (double)__uint_as_float(f);
    const uint32_t hi = (f & 0x80000000u) | (((f & 0x7FFFFFFFu) >> 3) + (896u << 20));
    return __hiloint2double((int)hi, (int)(f << 29));
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
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    constexpr int kPer = kMaxRouterExperts / 32;
    float v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        v[i] = 0.0f;
        if (e < E) {
            double sum = 0.0;
            for (int s = 0; s < S; ++s) sum += part[((int64_t)s * T + t) * E + e];
            float l = (float)sum;
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
constexpr int kRCl = 8;              // CTAs per cluster (H slices)
constexpr int kRClThreads = 256;
constexpr int kRClChunkMax = 24576;  // bytes of Wr per ring chunk
constexpr int kRClRing = 4;
constexpr int kTokenKernelMaxT = 256;

struct RouterClusterShape {
    int TT;      // tokens per cluster tile (1, 2, 4, 8 or 16)
    int EPP;     // expert pairs per row group, rounded up to a warp
    int G;       // row groups per chunk (kRClThreads / EPP)
    int hs;      // rows per CTA (H / 8)
    int RC;      // rows per chunk
    int nch;     // chunks per CTA
    size_t smem;
};

static bool router_cluster_shape(int T, int H, int E, int wr_is_fp32, RouterClusterShape *sh) {
    if (T > kTokenKernelMaxT || H % kRCl || E % 2) return false;
    const int eb = wr_is_fp32 ? 4 : 2;
    if ((E * eb) % 16) return false;
    sh->EPP = (E / 2 + 31) / 32 * 32;
    sh->G = kRClThreads / sh->EPP;
    sh->hs = H / kRCl;
    int TT = 1;
    while (TT < 16 && (T + TT - 1) / TT > 18) TT *= 2;
    sh->TT = TT;
    int rc = kRClChunkMax / (E * eb);
    if (rc > sh->hs) rc = sh->hs;
    int p = 1;
    while (p * 2 <= rc) p *= 2;
    while (p >= sh->G && (sh->hs % p || p % sh->G)) p /= 2;
    if (p < sh->G || p < 1) return false;
    sh->RC = p;
    sh->nch = sh->hs / p;
    const size_t ring = (size_t)kRClRing * p * E * eb;
    const size_t red = (size_t)TT * sh->G * 2 * sh->EPP * sizeof(double);
    sh->smem = 64 + (ring > red ? ring : red) + (size_t)sh->hs * TT * sizeof(double);
    return sh->smem <= 200 * 1024;
}

template <bool WR32, int TT>
__global__ void __cluster_dims__(kRCl, 1, 1) __launch_bounds__(kRClThreads)
    router_cluster_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H, const void *__restrict__ wr, int E,
                          int EPP, int G, int RC, int nch, const float *__restrict__ bias, int k,
                          int32_t *__restrict__ idx, float *__restrict__ w, float *__restrict__ logits) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int eb = WR32 ? 4 : 2;
    extern __shared__ __align__(128) uint8_t rsm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(rsm);            // [kRClRing]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(rsm + 48);
    const int hs = H / kRCl;
    const size_t chunk_bytes = (size_t)RC * E * eb;
    const size_t ring = (size_t)kRClRing * chunk_bytes;
    const int E2 = 2 * EPP;                                        // expert slots per row group
    const size_t red_bytes = (size_t)TT * G * E2 * sizeof(double);
    uint8_t *wring = rsm + 64;
    double *red = reinterpret_cast<double *>(rsm + 64);              // aliases the ring after the loop
    double *xs = reinterpret_cast<double *>(rsm + 64 + (ring > red_bytes ? ring : red_bytes));   // [hs][TT]

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
    // x tile -> shared, as fp64 (exact), layout [h][tt]; tokens past T are zero
    for (int i = tid; i < hs * TT; i += kRClThreads) {
        const int tt = i / hs, h = i - tt * hs;
        const int t = t0 + tt;
        xs[h * TT + tt] =
            t < T ? bf16_bits_to_f64(reinterpret_cast<const uint16_t *>(x)[(int64_t)t * H + h0 + h]) : 0.0;
    }
    __syncthreads();

    // thread (g, ep) owns experts 2 ep and 2 ep + 1 for every token of the tile over
    // rows [g rows_g, (g + 1) rows_g) of each chunk; NA independent fp64 sums per
    // (token, expert) keep at least 8 FMA chains in flight, added in order at the end
    const int ep = tid % EPP, g = tid / EPP;
    const bool active = g < G && 2 * ep < E;
    const int rows_g = RC / G;
    constexpr int NA = TT >= 4 ? 1 : 4 / TT;
    double acc[TT][2][NA];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int a = 0; a < NA; ++a) acc[tt][0][a] = acc[tt][1][a] = 0.0;
    for (int c = 0; c < nch; ++c) {
        const int b = c % kRClRing;
        mbar_wait(&full[b], (uint32_t)((c / kRClRing) & 1), abort_flag);
        if (active) {
            const uint8_t *wc = wring + b * chunk_bytes;
            const int rb = g * rows_g;
            for (int r0 = rb; r0 < rb + rows_g; r0 += NA) {
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    const int r = r0 + a;
                    if (r < rb + rows_g) {
                        double w0, w1;
                        if (WR32) {
                            const uint2 f = *reinterpret_cast<const uint2 *>(wc + ((size_t)r * E + 2 * ep) * 4);
                            w0 = f32_bits_to_f64(f.x);
                            w1 = f32_bits_to_f64(f.y);
                        } else {
                            const uint32_t bb = *reinterpret_cast<const uint32_t *>(wc + ((size_t)r * E + 2 * ep) * 2);
                            w0 = bf16_bits_to_f64(bb & 0xFFFFu);
                            w1 = bf16_bits_to_f64(bb >> 16);
                        }
                        const double *xr = xs + (size_t)(c * RC + r) * TT;
                        if constexpr (TT == 1) {
                            acc[0][0][a] = fma(xr[0], w0, acc[0][0][a]);
                            acc[0][1][a] = fma(xr[0], w1, acc[0][1][a]);
                        } else {
#pragma unroll
                            for (int tt = 0; tt < TT; tt += 2) {
                                const double2 xv = *reinterpret_cast<const double2 *>(xr + tt);
                                acc[tt][0][a] = fma(xv.x, w0, acc[tt][0][a]);
                                acc[tt][1][a] = fma(xv.x, w1, acc[tt][1][a]);
                                acc[tt + 1][0][a] = fma(xv.y, w0, acc[tt + 1][0][a]);
                                acc[tt + 1][1][a] = fma(xv.y, w1, acc[tt + 1][1][a]);
                            }
                        }
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
            for (int x2 = 0; x2 < 2; ++x2) {
                double sum = acc[tt][x2][0];
#pragma unroll
                for (int a = 1; a < NA; ++a) sum += acc[tt][x2][a];
                red[((size_t)tt * G + g) * E2 + 2 * ep + x2] = sum;
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
    }
    cluster.sync();   // keep this CTA's shared memory alive until every peer has read it
}

template <bool WR32, int TT>
static cudaError_t launch_router_cluster_t(const RouterClusterShape &sh, const void *x, int T, int H, const void *wr,
                                           int E, const float *bias, int k, int32_t *idx, float *w, float *logits,
                                           cudaStream_t st) {
    auto kern = router_cluster_kernel<WR32, TT>;
    if (sh.smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh.smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(kRCl, (T + TT - 1) / TT);
    count_launch();
    kern<<<grid, kRClThreads, sh.smem, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H, wr, E, sh.EPP, sh.G,
                                             sh.RC, sh.nch, bias, k, idx, w, logits);
    return cudaGetLastError();
}

template <bool WR32>
static cudaError_t launch_router_cluster(const RouterClusterShape &sh, const void *x, int T, int H, const void *wr,
                                         int E, const float *bias, int k, int32_t *idx, float *w, float *logits,
                                         cudaStream_t st) {
    switch (sh.TT) {
    case 1: return launch_router_cluster_t<WR32, 1>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
    case 2: return launch_router_cluster_t<WR32, 2>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
    case 4: return launch_router_cluster_t<WR32, 4>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
    case 8: return launch_router_cluster_t<WR32, 8>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
    default: return launch_router_cluster_t<WR32, 16>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
    }
}

moe_status launch_router(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                         int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes, int nsm,
                         cudaStream_t st) {
    if (T == 0) return MOE_OK;
    RouterClusterShape sh;
    if (router_cluster_shape(T, H, E, wr_is_fp32, &sh) && (reinterpret_cast<uintptr_t>(wr) & 15) == 0) {
        cudaError_t e = wr_is_fp32 ? launch_router_cluster<true>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st)
                                   : launch_router_cluster<false>(sh, x, T, H, wr, E, bias, k, idx, w, logits, st);
        return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "router_cluster launch");
    }
    int S, slice;
    router_split(T, H, &S, &slice);
    (void)nsm;
    const size_t need = (size_t)S * T * E * sizeof(double);
    if (ws_bytes < need) return set_error(MOE_ERR_OOM, "router workspace too small (%zu < %zu)", ws_bytes, need);
    double *part = reinterpret_cast<double *>(ws);
    dim3 grid((T + kTT - 1) / kTT, S);
    count_launch();
    if (wr_is_fp32)
        router_partial_kernel<true><<<grid, kRThreads, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H, wr,
                                                               E, slice, part);
    else
        router_partial_kernel<false><<<grid, kRThreads, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H,
                                                                wr, E, slice, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_partial launch");
    count_launch();
    router_finish_kernel<<<(T + 7) / 8, 256, 0, st>>>(part, S, T, E, bias, k, idx, w, logits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_finish launch");
    return MOE_OK;
}

}  // namespace moe
