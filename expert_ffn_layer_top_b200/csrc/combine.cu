// Gate-weighted combine (un-permute): out[t] = sum_j w[t,j] * y_perm[pair_row[t*k+j]],
// accumulated in fp32 in order of j and rounded once to bf16. The pages give no
// combine formula; this is the standard weighted sum of the k expert outputs.
// One block per token, 8 channels (16-byte bf16 / 32-byte fp32 loads) per thread.
// early != 0: pair_row and w were complete before the previous kernel let this one
// start (the layer forward: they come from the routing, several kernels back, and every
// kernel of the library lets its successor start only after its own wait), so they
// are read before the wait for y_perm. Slot layout (cprefix non-null): pair_row holds
// e slab_T + pos and the row of y is cprefix[e] + pos (cprefix comes from the UP kernel,
// also several kernels back); block 0 then clears the layer's slot counts for the next call.
#include "common.cuh"
#include "internal.h"

namespace moe {

template <bool Y32>
__global__ void __launch_bounds__(256) combine_kernel(const void *__restrict__ y_perm,
                                                     const int32_t *__restrict__ pair_row,
                                                     const float *__restrict__ w, int k, int H,
                                                     __nv_bfloat16 *__restrict__ out, int early,
                                                     const int32_t *__restrict__ cprefix, int slab_T,
                                                     int32_t *__restrict__ cnt_zero, int E) {
    if (!early) pdl_wait();
    const int t = blockIdx.x;
    __shared__ int rows[kMaxTopK];
    __shared__ float ws[kMaxTopK];
    if (threadIdx.x < k) {
        int r = pair_row[(int64_t)t * k + threadIdx.x];
        if (cprefix) {
            const int e = r / slab_T;
            r = (r >= 0 && e < E) ? __ldcg(cprefix + e) + (r - e * slab_T) : -1;
        }
        // a row outside y_perm's T*k rows is reported, and row 0 read in its place
        if (r < 0 || (int64_t)r >= (int64_t)gridDim.x * k) {
            flag_error(2);
            r = 0;
        }
        rows[threadIdx.x] = r;
        ws[threadIdx.x] = w[(int64_t)t * k + threadIdx.x];
    }
    if (early) pdl_wait();
    pdl_release();
    if (cnt_zero && blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) cnt_zero[e] = 0;
    __syncthreads();
    for (int c = threadIdx.x * 8; c < H; c += blockDim.x * 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        // eight rows at a time: all loads issued first, then added in order of j
        for (int j0 = 0; j0 < k; j0 += 8) {
            if (Y32) {
                float4 a[8], b[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k) {
                        const float *src = reinterpret_cast<const float *>(y_perm) + (int64_t)rows[j0 + jj] * H + c;
                        a[jj] = *reinterpret_cast<const float4 *>(src);
                        b[jj] = *reinterpret_cast<const float4 *>(src + 4);
                    }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k) {
                        const float wj = ws[j0 + jj];
                        acc[0] += wj * a[jj].x; acc[1] += wj * a[jj].y; acc[2] += wj * a[jj].z; acc[3] += wj * a[jj].w;
                        acc[4] += wj * b[jj].x; acc[5] += wj * b[jj].y; acc[6] += wj * b[jj].z; acc[7] += wj * b[jj].w;
                    }
            } else {
                uint4 v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k)
                        v[jj] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(y_perm) +
                                                                (int64_t)rows[j0 + jj] * H + c);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k) {
                        const float wj = ws[j0 + jj];
                        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v[jj]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(p2[i]);
                            acc[2 * i] += wj * f.x;
                            acc[2 * i + 1] += wj * f.y;
                        }
                    }
            }
        }
        uint4 o;
        __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) o2[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        *reinterpret_cast<uint4 *>(out + (int64_t)t * H + c) = o;
    }
}

moe_status launch_combine(const void *y_perm, int y_is_fp32, const int32_t *pair_row, const float *w, int T, int k,
                          int H, void *out, cudaStream_t st, int early, const int32_t *cprefix, int slab_T,
                          int32_t *cnt_zero, int E) {
    if (T == 0) return MOE_OK;
    int threads = H / 8;
    if (threads > 256) threads = 256;
    threads = (threads + 31) / 32 * 32;
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(out);
    cudaError_t e = y_is_fp32
                        ? launch_pdl(combine_kernel<true>, dim3(T), dim3(threads), 0, st, y_perm, pair_row, w, k, H, o,
                                     early, cprefix, slab_T, cnt_zero, E)
                        : launch_pdl(combine_kernel<false>, dim3(T), dim3(threads), 0, st, y_perm, pair_row, w, k, H, o,
                                     early, cprefix, slab_T, cnt_zero, E);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "combine launch");
}

}  // namespace moe
