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
// Kernel 1 (partial): a block owns 16 tokens x all experts x one slice of H;
// the slice count is chosen so small batches still fill the GPU. fp64 partial
// sums go to the workspace. Kernel 2 (finish): one warp per token adds the
// partials in slice order, rounds, adds the bias, selects the top k with warp
// shuffles and writes idx, w (and optionally the logits).
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

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
    return v1 > v2 || (v1 == v2 && i1 < i2);
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
    bool taken[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        taken[i] = true;
        v[i] = 0.0f;
        if (e < E) {
            double sum = 0.0;
            for (int s = 0; s < S; ++s) sum += part[((int64_t)s * T + t) * E + e];
            float l = (float)sum;
            if (bias) l = l + bias[e];
            v[i] = l;
            taken[i] = false;
            if (logits) logits[(int64_t)t * E + e] = l;
        }
    }
    float selv[kMaxTopK];
    int seli[kMaxTopK];
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (!taken[i] && better(v[i], e, bv, bi)) { bv = v[i]; bi = e; }
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, d);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, d);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        // owner marks it taken
#pragma unroll
        for (int i = 0; i < kPer; ++i)
            if (lane + 32 * i == bi) taken[i] = true;
        selv[j] = bv;
        seli[j] = bi;
    }
    if (lane == 0) {
        const float l0 = selv[0];
        float z = 0.0f;
        for (int j = 0; j < k; ++j) z += expf(selv[j] - l0);
        for (int j = 0; j < k; ++j) {
            idx[(int64_t)t * k + j] = seli[j];
            w[(int64_t)t * k + j] = expf(selv[j] - l0) / z;
        }
    }
}

moe_status launch_router(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                         int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes, int nsm,
                         cudaStream_t st) {
    if (T == 0) return MOE_OK;
    int S, slice;
    router_split(T, H, &S, &slice);
    (void)nsm;
    const size_t need = (size_t)S * T * E * sizeof(double);
    if (ws_bytes < need) return set_error(MOE_ERR_OOM, "router workspace too small (%zu < %zu)", ws_bytes, need);
    double *part = reinterpret_cast<double *>(ws);
    dim3 grid((T + kTT - 1) / kTT, S);
    if (wr_is_fp32)
        router_partial_kernel<true><<<grid, kRThreads, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H, wr,
                                                               E, slice, part);
    else
        router_partial_kernel<false><<<grid, kRThreads, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, H,
                                                                wr, E, slice, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_partial launch");
    router_finish_kernel<<<(T + 7) / 8, 256, 0, st>>>(part, S, T, E, bias, k, idx, w, logits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(e, "router_finish launch");
    return MOE_OK;
}

}  // namespace moe
