// Dense tensor-core throughput of this GPU for the MMA kinds the grouped FFN uses,
// measured with the library's own tcgen05 code: every SM's CTA issues a long chain of
// MMAs (M = 128, N = 256, four K steps per 128-byte swizzled row) on operands resident
// in its shared memory, accumulating into TMEM; nothing is read from or written to
// global memory. The rate of that chain is the roofline denominator for the FFN
// kernels of the same kind: bf16 (kind::f16), FP8 E4M3 (kind::f8f6f4), MXFP4
// (kind::mxf4, E8M0 scales per 32) and NVFP4 (kind::mxf4nvf4, E4M3 scales per 16).
// No counterpart in the pages: a measurement, not part of the layer.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kPeakM = 128, kPeakN = 256;

__device__ __forceinline__ void mma_ss_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// kind 0 bf16, 1 fp8 e4m3, 2 mxfp4, 3 nvfp4. Shared memory: A 128 x 128 B, B 256 x 128 B,
// eight zero scale atoms; TMEM: D at columns 0..255, A scales from 256, B scales from 384.
template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters) {
    extern __shared__ __align__(1024) uint8_t raw[];
    __shared__ uint64_t done;
    __shared__ uint32_t tbase;
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    constexpr int kA = kPeakM * 128, kB = kPeakN * 128, kSf = 8 * 512;
    for (int i = threadIdx.x; i < (kA + kB + kSf) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();   // the zeros are visible to the tensor core's reads
    if (threadIdx.x == 0) {
        mbar_init(&done, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t = tbase;
    if (threadIdx.x == 0) {
        const uint32_t s0 = smem_u32(sm);
        const uint64_t adesc = smem_desc_sw128(s0), bdesc = smem_desc_sw128(s0 + kA);
        const uint32_t sfa = t + 256, sfb = t + 384;
        if (KIND >= 2) {
            for (int a = 0; a < 4; ++a) {
                asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sfa + 4 * a),
                             "l"(((uint64_t)(((s0 + kA + kB + 512 * a) >> 4) & 0x3FFFu)) | ((uint64_t)8 << 16) |
                                 ((uint64_t)8 << 32) | (1ull << 46))
                             : "memory");
                asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sfb + 4 * a),
                             "l"(((uint64_t)(((s0 + kA + kB + 2048 + 512 * a) >> 4) & 0x3FFFu)) | ((uint64_t)8 << 16) |
                                 ((uint64_t)8 << 32) | (1ull << 46))
                             : "memory");
            }
        }
        constexpr uint32_t N8 = kPeakN >> 3, M16 = kPeakM >> 4;
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {   // 32 bytes further along the swizzled rows each step
                const uint32_t acc = (it | i) != 0;
                if constexpr (KIND == 0) {
                    mma_ss_f16(t, adesc + 2 * i, bdesc + 2 * i, (1u << 4) | (1u << 7) | (1u << 10) | (N8 << 17) | (M16 << 24),
                               acc);
                } else if constexpr (KIND == 1) {
                    mma_ss_f8(t, adesc + 2 * i, bdesc + 2 * i, (1u << 4) | (N8 << 17) | (M16 << 24), acc);
                } else if constexpr (KIND == 2) {
                    const uint32_t id = (uint32_t)(i & 1) * 2;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(t),
                        "l"(adesc + 2 * i), "l"(bdesc + 2 * i),
                        "r"((id << 4) | (1u << 7) | (1u << 10) | (N8 << 17) | (1u << 23) | (M16 << 24) | (id << 29)),
                        "r"(acc), "r"(sfa | (id << 30)), "r"(sfb | (id << 30))
                        : "memory");
                } else {
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(t),
                        "l"(adesc + 2 * i), "l"(bdesc + 2 * i), "r"((1u << 7) | (1u << 10) | (N8 << 17) | (M16 << 24)),
                        "r"(acc), "r"(sfa + 4 * i), "r"(sfb + 4 * i)
                        : "memory");
                }
            }
        }
        mma_commit(&done);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&done, 0)) {
            if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tmem_dealloc(t, 512);
}

template <int KIND>
static cudaError_t peak_launch(int grid, int iters, cudaStream_t st) {
    // at least 120 KB, so that one CTA runs per SM (each allocates all of TMEM)
    const int smem = 120 * 1024;
    static_assert(1024 + kPeakM * 128 + kPeakN * 128 + 8 * 512 <= 120 * 1024, "probe operands");
    cudaError_t e = ensure_max_smem<mma_peak_kernel<KIND>>(smem);
    if (e != cudaSuccess) return e;
    count_launch();
    mma_peak_kernel<KIND><<<grid, 128, smem, st>>>(iters);
    return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_tensor_peak(int kind, int iters, double *tflops) {
    if (kind < 0 || kind > 3 || iters < 1 || !tflops) return set_error(MOE_ERR_INVALID_ARG, "bad peak arguments");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error(e, "device");
    const int grid = num_sms(dev);
    auto run = [&](cudaStream_t st) {
        switch (kind) {
            case 0: return peak_launch<0>(grid, iters, st);
            case 1: return peak_launch<1>(grid, iters, st);
            case 2: return peak_launch<2>(grid, iters, st);
            default: return peak_launch<3>(grid, iters, st);
        }
    };
    cudaStream_t st = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    if ((e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking)) == cudaSuccess && (e = cudaEventCreate(&a)) == cudaSuccess &&
        (e = cudaEventCreate(&b)) == cudaSuccess && (e = run(st)) == cudaSuccess &&      // warm-up launch
        (e = cudaEventRecord(a, st)) == cudaSuccess) {
        for (int r = 0; r < 3 && e == cudaSuccess; ++r) e = run(st);
        if (e == cudaSuccess) e = cudaEventRecord(b, st);
        if (e == cudaSuccess) e = cudaEventSynchronize(b);
    }
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
    if (a) cudaEventDestroy(a);
    if (b) cudaEventDestroy(b);
    if (st) cudaStreamDestroy(st);
    if (e != cudaSuccess) return set_cuda_error(e, "tensor peak");
    const double kstep = kind == 0 ? 16.0 : kind == 1 ? 32.0 : 64.0;   // K per MMA
    const double flops = 3.0 * grid * (double)iters * 4.0 * 2.0 * kPeakM * kPeakN * kstep;
    *tflops = flops / (ms * 1e-3) / 1e12;
    return MOE_OK;
}
