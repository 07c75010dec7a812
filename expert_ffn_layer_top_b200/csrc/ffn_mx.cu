// Grouped SwiGLU expert FFN for FP4 experts on the block-scaled tensor core
// path, fp32 accumulation in TMEM, K = 64 per instruction:
//   MXFP4: tcgen05.mma kind::mxf4, one E8M0 scale per 32 K elements;
//   NVFP4: tcgen05.mma kind::mxf4nvf4 scale_vec::4X, one E4M3 scale per 16 K
//          elements, and the per-expert fp32 tensor scale in the epilogue.
// Both operands stay packed, two codes per byte, from HBM to the tensor core.
//
// Activations: a bf16 value x of a 32-block whose largest magnitude has binary
// exponent e is carried as four E2M1 planes, x ~ sum_p q_p 2^(s - 3p) with
// s = e - 1. Plane 0 rounds x 2^-s; each further plane rounds what is left at
// a unit 8 times finer. Every plane value lies in [-4, 4] (E2M1 reaches 6, so
// nothing saturates) and leaves a residual of at most half its unit, so the
// four planes are within 2^(e - 11), about 2^-11 of the block maximum, of x.
// The planes of a token are four rows of the B operand (plane p of token n is
// row p BN + n), each with its own scale; the epilogue adds the four columns.
// NVFP4 scales are E4M3, which hold the powers of two 2^-9..2^8 only: a token
// row with largest magnitude 2^E stores every plane scale multiplied by
// 2^(3p + C), C = 9 - E (so the largest block lands on 2^8), and the epilogue
// multiplies column (p, n) by 2^-(3p + C); blocks more than 2^17 below the row
// maximum keep the smallest scale and lose only digits below 2^-17 of it.
//
// Work item: an N tile of BN rows of one expert x one M tile of 128 weight rows
// (UP: 64 gate rows and the matching 64 up rows; DOWN: 128 rows). A stage is a
// 256-wide K slice and each operand of a stage arrives by one bulk copy:
//   weights, prepacked: 128 rows x 128 bytes, the 16-byte chunk c of row r at
//     r*128 + (c ^ (r % 8))*16 (the 128-byte swizzle of the MMA descriptor),
//     then the scale atoms of the stage (MXFP4: two, one per 128-wide half;
//     NVFP4: four, one per 64-wide quarter);
//   activations, written by the quantiser (MXFP4 DOWN: by the UP epilogue):
//     N = 4 BN rows in the same swizzled form, then their scale atoms.
// A scale atom is 512 bytes: byte (r % 32) * 16 + (r / 32) * 4 + j holds the
// scale of operand row r and scale block j of its K range; tcgen05.cp 32x128b.warpx4
// puts atom row l into TMEM lanes l, l+32, l+64, l+96 (4 columns), where the
// MMA reads the scale of row r: lane r, column r / 32, byte j.
//
// Activation format A4 (NVFP4 only): the activations are themselves in NVFP4
// form, one plane: x with the per-tensor scale s_g = amax|x| / (6 * 448), h with
// s_g = 1; E4M3 scales E4M3_RN_sat((amax_16 / 6) / s_g) per 16 K elements and
// E2M1 codes of v / (s_b s_g), ties to even. The B operand then has N = BN rows
// (one per token), and the epilogue multiplies by s_g and the weights' tensor
// scale. The UP epilogue writes h in this form for the down pass.
//
// Every wait is bounded; on timeout the CTA sets the device error word, drains
// its copies and MMAs and exits.
#include "common.cuh"
#include "internal.h"
#include "mx_codec.cuh"

namespace moe {

constexpr int kMxThreads = 544;   // 16 role warps + the item scheduler (warp 16)
constexpr int kMxSchedWarp = 16;
constexpr int kMxQ = 16;          // entries of the CTA's item queue
constexpr int kMxMaxStages = 12;
constexpr int kMxXch = 9;    // padded row of the gate/up exchange (8 values)
constexpr int kMxSmemCap = 227 * 1024;

// ------------------------------------------------------------------ device helpers

// 32 rows x 16 bytes of shared memory -> TMEM lanes (l, l+32, l+64, l+96), 4 columns.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, packed E2M1 operands, two E8M0 scales per
// row and instruction (bytes id, id + 1 of the scale column) read from TMEM.
__device__ __forceinline__ void mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// The same with kind::mxf4nvf4: four E4M3 scales per row and instruction
// (the whole 32-bit scale column).
__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
            "r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Shared-memory descriptor of a scale atom: no swizzle, K-major, core matrices
// of 8 rows x 16 bytes stacked 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
           (1ull << 46);
}

// Instruction descriptor, kind::mxf4 block-scaled: A and B E2M1 (format 1),
// E8M0 scales, both K-major, M = 128, K = 64; scale byte `id` (0 or 2) of each
// 32-bit scale column for both operands.
__host__ __device__ constexpr uint32_t idesc_mxf4(int N, uint32_t id) {
    return (id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) |
           (id << 29);
}

// Instruction descriptor, kind::mxf4nvf4 block-scaled: A and B E2M1, E4M3
// scales, both K-major, M = 128, K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (0u << 23) | ((128u >> 4) << 24);
}


// ------------------------------------------------------------------ activation quantiser

// Inverse of interleave8: operand order 0,4,1,5,2,6,3,7 back to natural order.
__device__ __forceinline__ uint4 deinterleave8(uint4 o) {
    uint4 v;
    v.x = __byte_perm(o.x, o.y, 0x5410);
    v.y = __byte_perm(o.z, o.w, 0x5410);
    v.z = __byte_perm(o.x, o.y, 0x7632);
    v.w = __byte_perm(o.z, o.w, 0x7632);
    return v;
}

// s_off[0..E] = offsets; s_tile[e] = sum over e' < e of ceil(n_e' / BN). 256 threads.
__device__ __forceinline__ void quant_tile_prefix(const int32_t *__restrict__ offsets, int E, int BN, int *s_off,
                                                  int *s_tile, int *s_wsum) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    int cnt[4], run = 0;   // 4 experts per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = tid * 4 + i;
        cnt[i] = e < E ? (s_off[e + 1] - s_off[e] + BN - 1) / BN : 0;
        run += cnt[i];
    }
    int incl = run;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int base = incl - run;
    for (int w = 0; w < warp; ++w) base += s_wsum[w];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = tid * 4 + i;
        if (e <= E) s_tile[e] = base;
        base += cnt[i];
    }
    __syncthreads();
}

// Expert e with s_off[e] <= r < s_off[e + 1].
__device__ __forceinline__ int expert_of_row(const int *s_off, int E, int r) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void bf16x8_to_float(uint4 u, float (&v)[8]) {
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[h]));
        v[2 * h] = f.x;
        v[2 * h + 1] = f.y;
    }
}

// MXFP4 activations. One warp per (permuted row r, 256-wide stage st),
// grid-stride; each lane takes 8 consecutive elements. The row is x_perm[r]
// (mode 0, operand order) or x[sorted_pair[r] / k] (mode 1, natural order).
// Its four planes go to rows p BN + n (n = (r - offsets[e]) % BN) of the
// activation blob (tile, st) of its N tile, tile = tile_start[e] + (r -
// offsets[e]) / BN; the plane scales go into that blob's scale atoms.
__global__ void __launch_bounds__(256) mx_quant_kernel(const uint4 *__restrict__ src, int mode,
                                                       const int32_t *__restrict__ sorted_pair, int k, int P, int K,
                                                       const int32_t *__restrict__ offsets, int E, int BN,
                                                       uint8_t *__restrict__ bblob, int *__restrict__ sched_zero) {
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_tile[kMaxExperts + 1];
    __shared__ int s_wsum[8];
    pdl_wait();
    pdl_release();
    if (sched_zero && blockIdx.x == 0 && threadIdx.x < 2) sched_zero[threadIdx.x] = 0;   // the FFN's claim counters
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K8 = K / 8, KST = K / kMxStageK, NROW = kMxPlanes * BN, BB = bs_bblob_bytes(kBsMx, BN);
    const int64_t units = (int64_t)P * KST;
    const int64_t nw = (int64_t)gridDim.x * 8;
    const int64_t u0 = (int64_t)blockIdx.x * 8 + warp;
    // the first unit's row goes out before the tile prefix, which it does not need
    uint4 uv0 = make_uint4(0, 0, 0, 0);
    if (u0 < units) {
        const int r = (int)(u0 / KST), st = (int)(u0 - (int64_t)r * KST);
        uv0 = src[(int64_t)(mode == 1 ? sorted_pair[r] / k : r) * K8 + st * 32 + lane];
    }
    quant_tile_prefix(offsets, E, BN, s_off, s_tile, s_wsum);
    for (int64_t u = u0; u < units; u += nw) {
        const int r = (int)(u / KST), st = (int)(u - (int64_t)r * KST);
        const int e = expert_of_row(s_off, E, r);
        const int rel = r - s_off[e];
        const int tile = s_tile[e] + rel / BN, n = rel % BN;
        uint4 uv = u == u0 ? uv0 : src[(int64_t)(mode == 1 ? sorted_pair[r] / k : r) * K8 + st * 32 + lane];
        if (mode == 0) uv = deinterleave8(uv);
        float v[8];
        bf16x8_to_float(uv, v);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        // 4 consecutive lanes hold one 32-block
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int s = mx_plane0_exp(amax);
        uint32_t pw[kMxPlanes];
        mx_planes8(v, s, pw);
        const int c16 = lane >> 2;   // 32-block within the stage
        uint8_t *blob = bblob + ((int64_t)tile * KST + st) * BB;
#pragma unroll
        for (int pl = 0; pl < kMxPlanes; ++pl) {
            const int R = pl * BN + n;
            *reinterpret_cast<uint32_t *>(blob + sw128_chunk(R, c16) + (lane & 3) * 4) = pw[pl];
            if ((lane & 3) == 0) blob[NROW * 128 + (c16 >> 2) * 512 + atom_offset(R, c16 & 3)] = (uint8_t)(s - 3 * pl);
        }
    }
}

// NVFP4 activations. One block per permuted row r (grid-stride), each thread
// 8 consecutive elements at a time: the row is x_perm[r] (mode 0),
// x[sorted_pair[r] / k] (mode 1) or src[r] (mode 2, natural order). A first
// pass finds the row maximum 2^E and the offset C = 9 - E (rowexp[r]); then
// every 16-block with maximum exponent e gets the E4M3 scale
// 2^min(8, max(-9, e - 1 + C)) for all four planes, plane p carrying the unit
// 2^(scale exponent - 3p - C). Rows and atoms as in mx_quant_kernel.
__global__ void __launch_bounds__(256) nv_quant_kernel(const uint4 *__restrict__ src, int mode,
                                                       const int32_t *__restrict__ sorted_pair, int k, int P, int K,
                                                       const int32_t *__restrict__ offsets, int E, int BN,
                                                       uint8_t *__restrict__ bblob, int32_t *__restrict__ rowexp,
                                                       int *__restrict__ sched_zero) {
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_tile[kMaxExperts + 1];
    __shared__ int s_wsum[8];
    __shared__ uint32_t s_max[8];
    pdl_wait();
    pdl_release();
    if (sched_zero && blockIdx.x == 0 && threadIdx.x < 2) sched_zero[threadIdx.x] = 0;   // the FFN's claim counters
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    quant_tile_prefix(offsets, E, BN, s_off, s_tile, s_wsum);
    const int K8 = K / 8, KST = K / kMxStageK, NROW = kMxPlanes * BN, BB = bs_bblob_bytes(kBsNv, BN);
    for (int r = blockIdx.x; r < P; r += gridDim.x) {
        const int e = expert_of_row(s_off, E, r);
        const int rel = r - s_off[e];
        const int tile = s_tile[e] + rel / BN, n = rel % BN;
        const uint4 *srow = src + (int64_t)(mode == 1 ? sorted_pair[r] / k : r) * K8;
        // pass 1: row maximum (order does not matter): warps, then the block
        float amax = 0.0f;
        for (int c = tid; c < K8; c += 256) {
            float v[8];
            bf16x8_to_float(__ldcg(srow + c), v);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
        if (lane == 0) s_max[warp] = wmax;
        __syncthreads();
        uint32_t bmax_bits = s_max[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) bmax_bits = max(bmax_bits, s_max[i]);
        __syncthreads();   // s_max is rewritten for the next row
        amax = __uint_as_float(bmax_bits);
        int Er = amax > 0.0f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 : 0;
        Er = Er < -90 ? -90 : Er;
        const int C = 9 - Er;
        if (tid == 0) rowexp[r] = C;
        // pass 2: planes, 8 elements per thread, 2 neighbouring lanes per 16-block
        for (int c = tid; c < K8; c += 256) {
            uint4 uv = __ldcg(srow + c);
            if (mode == 0) uv = deinterleave8(uv);
            float v[8];
            bf16x8_to_float(uv, v);
            float bmax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
            int ks = bmax > 0.0f ? (int)((__float_as_uint(bmax) >> 23) & 0xFF) - 128 + C : -9;
            ks = ks < -9 ? -9 : (ks > 8 ? 8 : ks);
            uint32_t pw[kMxPlanes];
            float rr[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) rr[i] = v[i];
#pragma unroll
            for (int pl = 0; pl < kMxPlanes; ++pl) {
                const int uexp = ks - 3 * pl - C;   // plane unit 2^uexp, |uexp| <= 126
                const float inv = exp2_neg_biased(uexp + 127), unit = exp2_biased(uexp + 127);
                float t[8], q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) t[i] = rr[i] * inv;
                pw[pl] = e2m1x8(t, q);
#pragma unroll
                for (int i = 0; i < 8; ++i) rr[i] = fmaf(-q[i], unit, rr[i]);
            }
            const int st = c >> 5, cc = c & 31, c16 = cc >> 2, b16 = cc >> 1;
            uint8_t *blob = bblob + ((int64_t)tile * KST + st) * BB;
            const uint8_t sb = e4m3_pow2(ks);
#pragma unroll
            for (int pl = 0; pl < kMxPlanes; ++pl) {
                const int R = pl * BN + n;
                *reinterpret_cast<uint32_t *>(blob + sw128_chunk(R, c16) + (cc & 3) * 4) = pw[pl];
                if ((cc & 1) == 0) blob[NROW * 128 + (b16 >> 2) * 512 + atom_offset(R, b16 & 3)] = sb;
            }
        }
    }
}

// ------------------------------------------------------------------ A4 activations

// Partial maxima of |src| (bf16, n8 groups of 8): part[b] = the maximum over block b's
// share (grid-stride). Maxima are exact, so the tensor scale does not depend on the split.
__global__ void __launch_bounds__(256) a4_amax_kernel(const uint4 *__restrict__ src, int64_t n8,
                                                      float *__restrict__ part, int *__restrict__ sched_zero) {
    __shared__ uint32_t s_max[8];
    pdl_wait();
    pdl_release();
    if (sched_zero && blockIdx.x == 0 && threadIdx.x < 2) sched_zero[threadIdx.x] = 0;   // the FFN's claim counters
    float amax = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (int64_t)gridDim.x * 256) {
        float v[8];
        bf16x8_to_float(__ldg(src + i), v);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
    // non-negative floats order like their bit patterns
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = wmax;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t m = s_max[0];
        for (int w = 1; w < 8; ++w) m = max(m, s_max[w]);
        part[blockIdx.x] = __uint_as_float(m);
    }
}

// A4 form of the activation rows into the blobs of the FFN's token tiles. The block
// first reduces the kA4Parts partial maxima to s_g = amax / (6 * 448) (1 for an all-zero
// x; block 0 stores it in *xscale for the UP epilogue). Then one warp per (row r,
// 256-wide stage), 8 consecutive elements per lane, two lanes per 16-block:
// s_b = E4M3(((amax_16 / 6) / s_g)), codes E2M1(v / (s_b s_g)) (0 when s_b s_g = 0),
// every step a correctly rounded binary32 operation. Rows: x[sorted_pair[r] / k]
// (mode 1) or src[r] (mode 2), natural order; placement as in mx_quant_kernel, one plane.
__global__ void __launch_bounds__(256) a4_quant_kernel(const uint4 *__restrict__ src, int mode,
                                                       const int32_t *__restrict__ sorted_pair, int k, int P, int K,
                                                       const int32_t *__restrict__ offsets, int E, int BN,
                                                       const float *__restrict__ part, float *__restrict__ xscale,
                                                       uint8_t *__restrict__ bblob) {
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_tile[kMaxExperts + 1];
    __shared__ int s_wsum[8];
    __shared__ float s_sg;
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    quant_tile_prefix(offsets, E, BN, s_off, s_tile, s_wsum);
    if (warp == 0) {
        uint32_t m = 0u;
        for (int i = lane; i < kA4Parts; i += 32) m = max(m, __float_as_uint(__ldcg(part + i)));
        m = __reduce_max_sync(0xffffffffu, m);
        const float amax = __uint_as_float(m);
        const float sg = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
        if (lane == 0) {
            s_sg = sg;
            if (blockIdx.x == 0) *xscale = sg;
        }
    }
    __syncthreads();
    const float sg = s_sg;
    const int K8 = K / 8, KST = K / kMxStageK, BB = bs_bblob_bytes(kBsNv, BN, 1);
    const int64_t units = (int64_t)P * KST;
    const int64_t nw = (int64_t)gridDim.x * 8;
    for (int64_t u = (int64_t)blockIdx.x * 8 + warp; u < units; u += nw) {
        const int r = (int)(u / KST), st = (int)(u - (int64_t)r * KST);
        const int e = expert_of_row(s_off, E, r);
        const int rel = r - s_off[e];
        const int tile = s_tile[e] + rel / BN, n = rel % BN;
        const uint4 uv = src[(int64_t)(mode == 1 ? sorted_pair[r] / k : r) * K8 + st * 32 + lane];
        float v[8];
        bf16x8_to_float(uv, v);
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));   // two lanes per 16-block
        const uint32_t sc = e4m3_code(__fdiv_rn(__fdiv_rn(bmax, 6.0f), sg));
        const float den = __fmul_rn(e4m3_value(sc), sg);
        float t[8], q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = den > 0.0f ? __fdiv_rn(v[i], den) : 0.0f;
        const uint32_t word = e2m1x8(t, q);
        uint8_t *blob = bblob + ((int64_t)tile * KST + st) * BB;
        *reinterpret_cast<uint32_t *>(blob + sw128_chunk(n, lane >> 2) + (lane & 3) * 4) = word;
        const int b16 = lane >> 1;   // 16-block within the stage
        if ((lane & 1) == 0) blob[BN * 128 + (b16 >> 2) * 512 + atom_offset(n, b16 & 3)] = (uint8_t)sc;
    }
}

// A4 form of the token rows straight into the activation blobs of the FFN's token tiles
// (the layer forward, where each token is in k pairs): the arithmetic of a4_quant_kernel,
// once per (token t, 256-wide stage), one warp each, then stored into the rows of the
// token's k pairs (row r = pair_row[t k + j] of its expert's tile, as in a4_quant_kernel).
// The next unit's x and pair_row loads are issued before this unit's arithmetic. Block 0 also stores s_g
// in *xscale.
__global__ void __launch_bounds__(256) a4_token_rows_kernel(const uint4 *__restrict__ x, int T, int K, int k,
                                                            const int32_t *__restrict__ pair_row,
                                                            const int32_t *__restrict__ offsets, int E, int BN,
                                                            const float *__restrict__ part, float *__restrict__ xscale,
                                                            uint8_t *__restrict__ bblob) {
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_tile[kMaxExperts + 1];
    __shared__ int s_wsum[8];
    __shared__ float s_sg;
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K8 = K / 8, KST = K / kMxStageK, BB = bs_bblob_bytes(kBsNv, BN, 1);
    const int64_t units = (int64_t)T * KST;
    const int64_t nw = (int64_t)gridDim.x * 8;
    int64_t u = (int64_t)blockIdx.x * 8 + warp;
    uint4 cur = u < units ? x[(u / KST) * K8 + (u % KST) * 32 + lane] : make_uint4(0, 0, 0, 0);
    int pr = (u < units && lane < k) ? pair_row[(u / KST) * k + lane] : 0;   // lane j < k: row of pair j
    quant_tile_prefix(offsets, E, BN, s_off, s_tile, s_wsum);
    if (warp == 0) {
        uint32_t m = 0u;
        for (int i = lane; i < kA4Parts; i += 32) m = max(m, __float_as_uint(__ldcg(part + i)));
        m = __reduce_max_sync(0xffffffffu, m);
        const float amax = __uint_as_float(m);
        const float sg = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
        if (lane == 0) {
            s_sg = sg;
            if (blockIdx.x == 0) *xscale = sg;
        }
    }
    __syncthreads();
    const float sg = s_sg;
    for (; u < units; u += nw) {
        const int t = (int)(u / KST), st = (int)(u - (int64_t)t * KST);
        const int64_t un = u + nw;
        const uint4 nxt = un < units ? x[(un / KST) * K8 + (un % KST) * 32 + lane] : cur;   // in flight
        const int prn = (un < units && lane < k) ? pair_row[(un / KST) * k + lane] : 0;
        // the token's pairs: lane j < k holds pair j's tile and row in it
        int tile_j = 0, n_j = 0;
        if (lane < k) {
            const int r = pr;
            const int e = expert_of_row(s_off, E, r);
            const int rel = r - s_off[e];
            tile_j = s_tile[e] + rel / BN;
            n_j = rel % BN;
        }
        float v[8];
        bf16x8_to_float(cur, v);
        cur = nxt;
        pr = prn;
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));   // two lanes per 16-block
        const uint32_t sc = e4m3_code(__fdiv_rn(__fdiv_rn(bmax, 6.0f), sg));
        const float den = __fmul_rn(e4m3_value(sc), sg);
        float tq[8], q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) tq[i] = den > 0.0f ? __fdiv_rn(v[i], den) : 0.0f;
        const uint32_t word = e2m1x8(tq, q);
        // the 4 scales of atom a (16-blocks 4a..4a+3, lanes 8a, 8a+2, 8a+4, 8a+6) as one word
        const uint32_t sw = sc | (__shfl_down_sync(0xffffffffu, sc, 2) << 8) |
                            (__shfl_down_sync(0xffffffffu, sc, 4) << 16) | (__shfl_down_sync(0xffffffffu, sc, 6) << 24);
        for (int j = 0; j < k; ++j) {
            const int tile = __shfl_sync(0xffffffffu, tile_j, j), n = __shfl_sync(0xffffffffu, n_j, j);
            uint8_t *blob = bblob + ((int64_t)tile * KST + st) * BB;
            *reinterpret_cast<uint32_t *>(blob + sw128_chunk(n, lane >> 2) + (lane & 3) * 4) = word;
            if ((lane & 7) == 0) *reinterpret_cast<uint32_t *>(blob + BN * 128 + (lane >> 3) * 512 + atom_offset(n, 0)) = sw;
        }
    }
}

// ------------------------------------------------------------------ grouped FFN kernel

struct MxSmem {
    uint64_t full[kMxMaxStages];
    uint64_t empty[kMxMaxStages];
    uint64_t accfull[8];      // stage-parallel: [buffer], every pipeline's MMA warp commits;
                              // item-parallel: [2 pipeline + buffer], that pipeline's MMA warp
    uint64_t accempty[8];     // the epilogue group that read the buffer (128 threads)
    uint64_t mmadone[4];
    uint64_t sfrdy[4];              // token-major mode: a scale group's copies landed (both helpers)
    uint64_t hdone[2];              // token-major mode: a helper's last copies landed
    uint64_t qfull[kMxQ];           // item queue: entry published (the scheduler)
    uint64_t qtake[kMxQ];           // the producers have started the entry's item
    uint64_t qempty[kMxQ];          // every reader of the entry has read it
    int qitem[kMxQ];                // the CTA's items in order; -1 ends the sequence
    uint64_t xfull[2], xempty[2];   // gate/up exchange, per epilogue group
    uint32_t tmem_base;
    int abort_flag;
    int total_items;
    // followed by int tile_start[E + 1], off[E + 1], slot[E]
};

struct MxItem {
    int e, rt, row0, nvalid, m, slot;
    int rtin;     // the tile of the phase's input blob (rt, or the expert's slot tile)
    int rt_out;   // the tile of the output blob (h for the down pass): the compact tile in expert order
};

// Head mode (p.slab_head): the experts whose first tile leads the item order, enough for
// every CTA's static first items.
__device__ __forceinline__ int mx_head_experts(const MxParams &p) {
    const int F = p.itempar ? p.pipes : 1;
    const int h = ((int)gridDim.x * F + p.m_tiles - 1) / p.m_tiles;
    return h < p.E ? h : p.E;
}

// tab = tile_start[E + 1], then off[E + 1] (a copy of offsets), then slot[E], then std_start[E + 1].
// tile_start: the prefix of each expert's tiles in item order (head mode: of the tiles after
// the head ones); std_start: the prefix of all its tiles (the compact order of the outputs).
__device__ __forceinline__ MxItem mx_item(const int *tab, const MxParams &p, int item, int BN) {
    const int *tile_start = tab, *off = tab + p.E + 1, *slot = tab + 2 * (p.E + 1);
    const int *std_start = tab + 3 * p.E + 2;
    MxItem it;
    it.rt = item / p.m_tiles;
    it.m = item - it.rt * p.m_tiles;
    const int SH = p.slab_head ? mx_head_experts(p) : 0;
    int lo = 0, t = 0;
    if (it.rt < SH) {
        lo = it.rt;   // the expert's first tile, possibly without rows
    } else {
        const int x = it.rt - SH;
        int hi = p.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_start[mid] <= x) lo = mid; else hi = mid - 1;
        }
        t = x - tile_start[lo] + (lo < SH ? 1 : 0);
    }
    it.rt_out = p.slab_head ? std_start[lo] + t : it.rt;
    it.e = lo;
    const int beg = off[lo];
    it.row0 = beg + t * BN;
    it.nvalid = min(BN, off[lo + 1] - beg - t * BN);
    it.slot = slot[lo];
    it.rtin = p.slab_mt ? lo * p.slab_mt + t : it.rt_out;
    return it;
}

// Entry j of the CTA's item queue: waits until the scheduler has published it and returns
// the item (-1: the sequence ended, or a wait gave up: then ok is cleared).
__device__ __forceinline__ int mx_q_get(MxSmem &sm, int j, volatile int *abort_flag, bool &ok) {
    if (!mbar_wait(&sm.qfull[j % kMxQ], (uint32_t)((j / kMxQ) & 1), abort_flag)) {
        ok = false;
        return -1;
    }
    return *reinterpret_cast<volatile int *>(&sm.qitem[j % kMxQ]);
}

// Warp roles (544 threads, one CTA per SM, persistent over items). NP
// independent pipelines: pipeline w is producer warp w, MMA warp 12 + w, its own
// ring of slots and its own double-buffered accumulators. It handles either
// stages w, w + NP, ... of every item (stage-parallel) or every stage of items
// w, w + NP, ... of the CTA (item-parallel, p.itempar), in order. One producer
// fills and one issuer drains each slot, both in order, so every parity wait on
// a slot barrier is exactly one phase after the previous one.
//   warps 0-3   producers: per stage one bulk copy of the weight blob and one
//               of the activation blob. Warp 2 also builds the tile prefix.
//   warps 12-15 MMA issuers (warp 12 owns TMEM): per stage one tcgen05.cp per
//               scale atom, four MMAs of K = 64, one commit.
//   warps 4-7   epilogue of the CTA's even items;
//   warps 8-11  epilogue of its odd items.
//   warp 16     item scheduler: publishes the CTA's items in order through a queue
//               in shared memory. The first (item-parallel: the first NP) are
//               static, blockIdx.x + j gridDim.x; the rest are claimed one by one
//               from a counter in global memory (zeroed by the kernel before this
//               one), each when the producers have started the item L entries
//               before it, so a CTA that streams faster takes more items and the
//               CTAs finish together. The epilogue adds the accumulators
//               of the pipelines that worked on the item (all NP, or the one
//               owner) and the four planes' columns.
// TMEM columns: accumulator (buffer a < NB, pipeline w) at (a NW + w) N; from NB NW N
// on, 16 NA scale columns per pipeline (two rotating groups of 8 NA: the NA
// weight atoms, then the NA activation atoms, 4 columns each).
template <int FMT, int PHASE, int BN, int PL>
__global__ void __launch_bounds__(kMxThreads, 1) ffn_mx_kernel(const __grid_constant__ MxParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    static_assert(PL == kMxPlanes || (PL == 1 && FMT == kBsNv), "A4 activations are NVFP4");
    // Token-major accumulators (A4 with tiles of 128 tokens): the MMA takes the 128 tokens as
    // its A operand (M) and the 128 weight rows as B (N), so a TMEM lane holds one token's
    // outputs. The UP epilogue then finds a channel's gate and up values in one thread, and
    // DOWN writes a token's 128 outputs as whole vectors. Smaller tiles keep the weights on M.
    constexpr bool TM = PL == 1 && BN == 128;
    constexpr int N = PL * BN;                              // MMA N: the planes' rows
    constexpr int NW = N <= 32 ? 4 : (N <= 64 ? 2 : 1);    // pipelines TMEM has room for
    constexpr int NA = bs_atoms(FMT);                       // scale atoms per operand and stage
    constexpr int ABLOB = bs_ablob_bytes(FMT);
    constexpr int BBLOB = bs_bblob_bytes(FMT, BN, PL);
    constexpr int STAGE = ABLOB + BBLOB;                    // a multiple of 1024
    static_assert(2 * NW * N + NW * 16 * NA <= 512, "TMEM columns");
    static_assert(!TM || 2 * NW * N + 4 * 8 * NA <= 512, "TMEM columns of the token-major mode");
    // accumulator buffers per pipeline: 2, or 3 where the plan found room (never in the
    // token-major or item-parallel modes); the scale columns follow them
    const int NB = p.nbuf;
    const uint32_t SFCOL = (uint32_t)(NB * NW * N);
    const int NP = p.pipes;                                 // <= NW; stage-parallel: divides the stages per item
    const int NSW = p.stages / NP;                          // slots per pipeline

    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *xch = reinterpret_cast<float *>(base + p.stages * STAGE);   // [2 groups][2 halves][64][kMxXch]
    MxSmem &sm = *reinterpret_cast<MxSmem *>(reinterpret_cast<uint8_t *>(xch) +
                                            (PHASE == kPhaseUp ? 2 * 128 * kMxXch * 4 : 0));
    int *tab = reinterpret_cast<int *>(&sm + 1);
    const int warp = warp_id(), lane = lane_id();
    volatile int *abort_flag = &sm.abort_flag;

    const int KST = p.K / kMxStageK;   // stages per item
    // Stage-parallel: pipeline w takes stages w, w + NP, ... of every item, and the
    // epilogue adds the pipelines' accumulators. Item-parallel (p.itempar): pipeline
    // w takes every stage of the CTA's items w, w + NP, ..., each in its own
    // accumulators, so its MMA warp meets an item boundary once per item.
    const bool IP = p.itempar != 0;
    const int j0 = IP ? (warp & 3) : 0, dj = IP ? NP : 1;   // the pipeline's items (w = warp & 3)
    const int st0 = IP ? 0 : (warp & 3), dst = IP ? 1 : NP;  // its stages of an item
    const int PER = IP ? KST : KST / NP;                     // stages per item and pipeline
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMxMaxStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < 8; ++a) {
            mbar_init(&sm.accfull[a], IP ? 1 : NP);
            mbar_init(&sm.accempty[a], 128);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sm.xfull[a], 128);
            mbar_init(&sm.xempty[a], 128);
        }
        for (int w = 0; w < 4; ++w) mbar_init(&sm.mmadone[w], 1);
        for (int g = 0; g < 4; ++g) mbar_init(&sm.sfrdy[g], 2);
        for (int h = 0; h < 2; ++h) mbar_init(&sm.hdone[h], 1);
        // readers of a queue entry: its producers and MMA warps (all NP, or the owner),
        // the token-major helpers, and the four warps of its epilogue group
        const uint32_t readers = (IP ? 2u : 2u * (uint32_t)p.pipes) + (TM ? 2u : 0u) + 4u;
        for (int e = 0; e < kMxQ; ++e) {
            mbar_init(&sm.qfull[e], 1);
            mbar_init(&sm.qtake[e], IP ? 1u : (uint32_t)p.pipes);
            mbar_init(&sm.qempty[e], readers);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    // Head mode: the static first item of each pipeline is an expert's first tile whatever the
    // routing (item = blockIdx.x + j0 gridDim.x, expert item / m_tiles), so its weights go out
    // now, while the routing kernel is still running and before the tile prefix waits on it.
    int pre_head = 0;
    if (p.slab_head) {
        __syncthreads();   // the barriers are initialised
        const int item = blockIdx.x + j0 * gridDim.x;
        if (warp < 4 && lane == 0 && warp < NP && item < mx_head_experts(p) * p.m_tiles) {
            const int e = item / p.m_tiles, m = item - e * p.m_tiles;
            const int slot = p.expert_map ? p.expert_map[e] : e;
            for (int st = st0; st < KST && pre_head < NSW; st += dst, ++pre_head) {
                const int s = warp * NSW + pre_head;
                mbar_expect_tx(&sm.full[s], (uint32_t)STAGE);
                bulk_load(base + s * STAGE, p.wbase + (int64_t)slot * p.w_estride + ((int64_t)m * KST + st) * ABLOB,
                          ABLOB, &sm.full[s]);
            }
        }
    }
    if (warp == 12) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        // Offsets come from the permutation, two launches back, so they are
        // complete before this kernel's predecessor could let it start. In the slot
        // layout the counts may come from the kernel just before (then: wait first).
        int *tile_start = tab, *off = tab + p.E + 1, *slot = tab + 2 * (p.E + 1), *std_start = tab + 3 * p.E + 2;
        if (p.slab_cnt && p.slab_wait) pdl_wait();
        const int SH = p.slab_head ? mx_head_experts(p) : 0;   // head mode: experts whose first tile leads
        int run = 0, rrun = 0, srun = 0;
        if (lane == 0) {
            tile_start[0] = 0;
            std_start[0] = 0;
            off[0] = p.slab_cnt ? 0 : p.offsets[0];
        }
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int nt = 0, nr = 0;
            if (e < p.E) {
                if (p.slab_cnt) {
                    nr = __ldcg(p.slab_cnt + e);
                } else {
                    nr = p.offsets[e + 1] - p.offsets[e];
                    off[e + 1] = p.offsets[e + 1];
                }
                slot[e] = p.expert_map ? p.expert_map[e] : e;
                nt = (nr + BN - 1) / BN;
            }
            // tiles in the item order after the head ones, rows, and all tiles (the compact order)
            int incl = e < SH ? (nt > 1 ? nt - 1 : 0) : nt, rincl = nr, sincl = nt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                const int vr = __shfl_up_sync(0xffffffffu, rincl, d);
                const int vs = __shfl_up_sync(0xffffffffu, sincl, d);
                if (lane >= d) {
                    incl += v;
                    rincl += vr;
                    sincl += vs;
                }
            }
            if (e < p.E) {
                tile_start[e + 1] = run + incl;
                std_start[e + 1] = srun + sincl;
                if (p.slab_cnt) {   // compact rows of h and y
                    off[e + 1] = rrun + rincl;
                    if (p.cprefix && blockIdx.x == 0) p.cprefix[e] = rrun + rincl - nr;
                }
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
            rrun += __shfl_sync(0xffffffffu, rincl, 31);
            srun += __shfl_sync(0xffffffffu, sincl, 31);
        }
        if (lane == 0) sm.total_items = (SH + run) * p.m_tiles;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = sm.tmem_base;
    const int total = sm.total_items;

    if (warp < 4) {
        // =================================================== producer of pipeline w
        const int w = warp;
        if (lane == 0 && w < NP) {
            // Weight half of a stage (codes + scale atoms): static data.
            auto issue_weights = [&](const MxItem &it, int st, int s) {
                uint64_t *fb = &sm.full[s];
                mbar_expect_tx(fb, (uint32_t)STAGE);
                bulk_load(base + s * STAGE,
                          p.wbase + (int64_t)it.slot * p.w_estride + ((int64_t)it.m * KST + st) * ABLOB, ABLOB,
                          fb);
            };
            // The slots start empty: the weights of this pipeline's first stages go out before
            // waiting for the kernel that writes the activations. Its first item is static
            // (queue entry j0), so they stay within that item. In head mode they went out
            // already, before the tile prefix.
            int pre = pre_head;
            if (!p.slab_head && blockIdx.x + j0 * gridDim.x < total) {
                const MxItem it = mx_item(tab, p, blockIdx.x + j0 * gridDim.x, BN);
                for (int st = st0; st < KST && pre < NSW; st += dst, ++pre) issue_weights(it, st, w * NSW + pre);
            }
            pdl_wait();
            if (w == 0) pdl_release();
            int loc = 0;   // stages this pipeline has issued
            bool ok = true;
            for (int jq = j0; ok; jq += dj) {   // this pipeline's queue entries
                const int item = mx_q_get(sm, jq, abort_flag, ok);
                if (item < 0) break;
                mbar_arrive(&sm.qtake[jq % kMxQ]);
                mbar_arrive(&sm.qempty[jq % kMxQ]);
                const MxItem it = mx_item(tab, p, item, BN);
                for (int st = st0; st < KST; st += dst, ++loc) {
                    const int s = w * NSW + loc % NSW;
                    const uint32_t round = (uint32_t)(loc / NSW);
                    if (loc >= pre) {
                        if (!mbar_wait(&sm.empty[s], (round & 1) ^ 1, abort_flag)) { ok = false; break; }
                        issue_weights(it, st, s);
                    }
                    bulk_load(base + s * STAGE + ABLOB, p.bblob + ((int64_t)it.rtin * KST + st) * BBLOB, BBLOB,
                              &sm.full[s]);
                }
            }
            // never leave while a copy into this CTA's shared memory is in flight
            for (int j = loc - 1; j >= 0 && j >= loc - NSW; --j) {
                const int s = w * NSW + j % NSW;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.full[s], (uint32_t)((j / NSW) & 1))) {
                    if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
                }
            }
        }
    } else if (TM && (warp == 13 || warp == 14) && lane == 0) {
        // =================================================== scale copies (token-major mode)
        // One thread issues the stage's scale-atom copies into TMEM at about 23 ns each, so the
        // MMA thread, left alone, would wait on them: warp 13 copies the weights' atoms and warp
        // 14 the activations', into one of G rotating column groups, and each commits to the
        // group's barrier, which the MMA warp waits on. A group is refilled only after the
        // MMAs of the stage G back (the slot's empty barrier) have completed.
        const int h = warp - 13;
        const int G = NSW - 1 < 4 ? NSW - 1 : 4;   // < NSW: empty barriers cannot alias
        const uint32_t base_u32 = smem_u32(base);
        int j = 0;
        bool ok = true;
        for (int jq = 0; ok; ++jq) {
            if (mx_q_get(sm, jq, abort_flag, ok) < 0) break;
            mbar_arrive(&sm.qempty[jq % kMxQ]);
            for (int k = 0; k < KST; ++k, ++j) {
                const int s = j % NSW;
                if (!mbar_wait(&sm.full[s], (uint32_t)((j / NSW) & 1), abort_flag)) { ok = false; break; }
                if (j >= G && !mbar_wait(&sm.empty[(j - G) % NSW], (uint32_t)(((j - G) / NSW) & 1), abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sp = base_u32 + s * STAGE;
                const uint32_t sfg = tmem + SFCOL + 32 * (j % G) + 16 * h;
#pragma unroll
                for (int a = 0; a < NA; ++a)
                    tmem_cp_atom(sfg + 4 * a, sf_atom_desc(h == 0 ? sp + kMxCodeBytes + 512 * a : sp + ABLOB + N * 128 + 512 * a));
                mma_commit(&sm.sfrdy[j % G]);
            }
        }
        mma_commit(&sm.hdone[h]);   // never leave with a copy into TMEM in flight
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&sm.hdone[h], 0)) {
            if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
        }
    } else if (warp == kMxSchedWarp) {
        // =================================================== item scheduler
        if (lane == 0) {
            const int F = IP ? p.pipes : 1;   // static items of each CTA
            const int L = IP ? p.pipes : 1;   // claim entry j once the producers took entry j - L
            int j = 0;
            bool ok = true;
            auto publish = [&](int item) {
                const int e = j % kMxQ;
                if (j >= kMxQ && !mbar_wait(&sm.qempty[e], (uint32_t)(((j / kMxQ) & 1) ^ 1), abort_flag)) {
                    ok = false;
                    return;
                }
                *reinterpret_cast<volatile int *>(&sm.qitem[e]) = item;
                mbar_arrive(&sm.qfull[e]);
                ++j;
            };
            for (int f = 0; f < F && ok; ++f) {
                const int item = blockIdx.x + f * gridDim.x;
                if (item >= total) break;
                publish(item);
            }
            if (p.sched) {
                pdl_wait();   // the counter was zeroed by the kernel before this one
                int next = F * gridDim.x;
                while (ok && next < total) {
                    if (j >= L && !mbar_wait(&sm.qtake[(j - L) % kMxQ], (uint32_t)(((j - L) / kMxQ) & 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    next = F * gridDim.x + (int)atomicAdd(reinterpret_cast<unsigned int *>(p.sched), 1u);
                    if (next < total) publish(next);
                }
            } else {   // no counter: the static order, blockIdx.x + j gridDim.x
                for (int item = blockIdx.x + F * gridDim.x; item < total && ok; item += gridDim.x) publish(item);
            }
            // end markers: a reader takes every entry (producers and MMA warps of the stage-parallel
            // modes), every NP-th (item-parallel) or every other one (epilogue groups), so each
            // residue meets one among max(2, NP) consecutive entries
            const int S = IP && p.pipes > 2 ? p.pipes : 2;
            for (int e = 0; e < S && ok; ++e) publish(-1);
        }
    } else if (warp >= 12) {
        // =================================================== MMA issuer of pipeline w
        const int w = warp - 12;
        if (TM && lane == 0 && w == 0) {
            // token-major mode: the scales come from the helper warps (above)
            const int G = NSW - 1 < 4 ? NSW - 1 : 4;
            int loc = 0, lt = 0;
            bool ok = true;
            const uint32_t base_u32 = smem_u32(base);
            for (int jq = 0; ok; ++jq, ++lt) {
                if (mx_q_get(sm, jq, abort_flag, ok) < 0) break;
                mbar_arrive(&sm.qempty[jq % kMxQ]);
                const int a = lt & 1;
                if (!mbar_wait(&sm.accempty[a], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(a * N);
                for (int k = 0; k < KST; ++k, ++loc) {
                    const int s = loc % NSW, g = loc % G;
                    if (!mbar_wait(&sm.full[s], (uint32_t)((loc / NSW) & 1), abort_flag) ||
                        !mbar_wait(&sm.sfrdy[g], (uint32_t)((loc / G) & 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sp = base_u32 + s * STAGE;
                    const uint32_t sfw = tmem + SFCOL + 32 * g, sfx = sfw + 16;
                    const uint64_t wdesc = smem_desc_sw128(sp), xdesc = smem_desc_sw128(sp + ABLOB);
#pragma unroll
                    for (int i = 0; i < 4; ++i)   // tokens as A, weights as B; K = 64 each
                        mma_nvf4(d, xdesc + (uint64_t)(2 * i), wdesc + (uint64_t)(2 * i), idesc_nvf4(N), sfx + 4 * i,
                                 sfw + 4 * i, (k | i) != 0);
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.accfull[a]);
            }
            mma_commit(&sm.mmadone[0]);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&sm.mmadone[0], 0)) {
                if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
            }
        } else if (!TM && lane == 0 && w < NP) {
            int loc = 0, lt = 0, sc = 0;
            bool ok = true;
            const uint32_t base_u32 = smem_u32(base);
            for (int jq = j0; ok; jq += dj, ++lt) {   // this pipeline's queue entries
                if (mx_q_get(sm, jq, abort_flag, ok) < 0) break;
                mbar_arrive(&sm.qempty[jq % kMxQ]);
                const int a = lt % NB, bi = IP ? 2 * w + a : a;   // lt: this pipeline's items so far
                if (!mbar_wait(&sm.accempty[bi], ((lt / NB) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)((a * NW + w) * N);
                for (int k = 0; k < PER; ++k, ++loc) {
                    const int s = w * NSW + loc % NSW;
                    if (!mbar_wait(&sm.full[s], (uint32_t)((loc / NSW) & 1), abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sp = base_u32 + s * STAGE;
                    const uint32_t sfa = tmem + SFCOL + 16 * NA * w + 8 * NA * sc;   // this stage's scales
                    const uint32_t sfb = sfa + 4 * NA;
#pragma unroll
                    for (int a = 0; a < NA; ++a) {
                        tmem_cp_atom(sfa + 4 * a, sf_atom_desc(sp + kMxCodeBytes + 512 * a));
                        tmem_cp_atom(sfb + 4 * a, sf_atom_desc(sp + ABLOB + N * 128 + 512 * a));
                    }
                    const uint64_t adesc = smem_desc_sw128(sp);
                    const uint64_t bdesc = smem_desc_sw128(sp + ABLOB);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {   // K = 64 each: 32 bytes further along the row
                        if constexpr (FMT == kBsMx) {   // two 32-blocks: bytes id, id + 1 of atom i / 2
                            const uint32_t id = (uint32_t)(i & 1) * 2, h = (uint32_t)(i >> 1) * 4;
                            mma_mxf4(d, adesc + (uint64_t)(2 * i), bdesc + (uint64_t)(2 * i), idesc_mxf4(N, id),
                                     (sfa + h) | (id << 30), (sfb + h) | (id << 30), (k | i) != 0);
                        } else {                        // four 16-blocks: the whole column of atom i
                            mma_nvf4(d, adesc + (uint64_t)(2 * i), bdesc + (uint64_t)(2 * i), idesc_nvf4(N),
                                     sfa + 4 * i, sfb + 4 * i, (k | i) != 0);
                        }
                    }
                    sc ^= 1;
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.accfull[bi]);
            }
            mma_commit(&sm.mmadone[w]);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&sm.mmadone[w], 0)) {
                if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
            }
        }
    } else {
        // =================================================== epilogue
        const int grp = (warp - 4) >> 2;   // 0: warps 4-7 (even items), 1: warps 8-11 (odd items)
        const int q = warp & 3;
        const int lrow = q * 32 + lane;    // TMEM lane == M-tile row
        float *xg = xch + grp * 128 * kMxXch;
        int lt = grp, xc = 0;
        bool ok = true;
        for (; ok; lt += 2) {   // queue entries grp, grp + 2, ...: lt is the item's place in the CTA
            int item = 0;
            if (lane == 0) item = mx_q_get(sm, lt, abort_flag, ok);
            item = __shfl_sync(0xffffffffu, item, 0);
            if (item < 0) break;   // the end, or lane 0 gave up (the abort flag is set)
            if (lane == 0) mbar_arrive(&sm.qempty[lt % kMxQ]);
            const MxItem it = mx_item(tab, p, item, BN);
            // NVFP4: the expert's tensor scale (static data), loaded once per item while the
            // accumulators are still being computed
            float iscale = 1.0f;
            if constexpr (FMT == kBsNv) iscale = p.tscale[it.e];
            // lt: the item's index in this CTA. Item-parallel: pipeline lt % NP, its item lt / NP.
            const int wi = IP ? lt % NP : 0, li = IP ? lt / NP : lt;
            const int a = li % NB, bi = IP ? 2 * wi + a : a;
            const int wlo = IP ? wi : 0, whi = IP ? wi + 1 : NP;   // accumulators to add
            if (!mbar_wait(&sm.accfull[bi], (li / NB) & 1, abort_flag)) break;
            tc_fence_after();
            // A4 UP: the tensor scale of x comes from the quantiser just before this kernel. It is
            // read only now: the accumulators hold its output, so the producer has passed the wait
            // on that kernel (these warps do not wait on it themselves).
            if constexpr (PL == 1 && PHASE == kPhaseUp) iscale *= __ldcg(p.xscale);
            const uint32_t acc0 = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * NW * N);
            if constexpr (TM) {
                // this thread's token is TMEM lane tok of the tile
                const int tok = q * 32 + lane;
                const bool valid = tok < it.nvalid;
                if constexpr (PHASE == kPhaseUp) {
                    // columns 0..63: gate of channels 64 m ..; 64..127: up of the same channels. h
                    // goes out in A4 form, 16 channels (one scale block) at a time.
                    uint8_t *blob = p.bblob_out + ((int64_t)it.rt_out * (p.I / kMxStageK) + ((it.m * 64) >> 8)) * BBLOB;
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        uint32_t G[16], U[16];
                        tmem_ld16(acc0 + blk * 16, G);
                        tmem_ld16(acc0 + 64 + blk * 16, U);
                        tmem_wait_ld();
                        float h[16], amax = 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float g = __uint_as_float(G[j]) * iscale, uu = __uint_as_float(U[j]) * iscale;
                            h[j] = __fdividef(g, 1.0f + __expf(-g)) * uu;
                            amax = fmaxf(amax, fabsf(h[j]));
                        }
                        const uint32_t sc = e4m3_code(__fdiv_rn(amax, 6.0f));
                        const float sb = e4m3_value(sc);
                        float t[8], qv[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) t[j] = sb > 0.0f ? __fdiv_rn(h[j], sb) : 0.0f;
                        const uint32_t w0 = e2m1x8(t, qv);
#pragma unroll
                        for (int j = 0; j < 8; ++j) t[j] = sb > 0.0f ? __fdiv_rn(h[8 + j], sb) : 0.0f;
                        const uint32_t w1 = e2m1x8(t, qv);
                        if (valid) {
                            const int c = (it.m * 64 + blk * 16) & 255;   // first channel within the stage
                            *reinterpret_cast<uint2 *>(blob + sw128_chunk(tok, c >> 5) + ((c & 31) >> 1)) =
                                make_uint2(w0, w1);
                            const int b16 = c >> 4;
                            blob[N * 128 + (b16 >> 2) * 512 + atom_offset(tok, b16 & 3)] = (uint8_t)sc;
                        }
                    }
                } else {
                    // the token's 128 outputs of this M tile, 32 at a time (two loads, one wait)
                    const int64_t o = (int64_t)(it.row0 + tok) * p.H + it.m * 128;
#pragma unroll 1
                    for (int b2 = 0; b2 < 8; b2 += 2) {
                        uint32_t V2[2][16];
                        tmem_ld16(acc0 + b2 * 16, V2[0]);
                        tmem_ld16(acc0 + b2 * 16 + 16, V2[1]);
                        tmem_wait_ld();
#pragma unroll
                        for (int hb = 0; hb < 2; ++hb) {
                        const int blk = b2 + hb;
                        const uint32_t (&V)[16] = V2[hb];
                        if (valid) {
                            float f[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(V[j]) * iscale;
                            if (p.out_fp32) {
                                float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + o + blk * 16);
#pragma unroll
                                for (int j = 0; j < 4; ++j) dst[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
                            } else {
                                uint32_t w[8];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(f[2 * j], f[2 * j + 1]);
                                    w[j] = *reinterpret_cast<const uint32_t *>(&b2);
                                }
                                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + o + blk * 16);
                                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                            }
                        }
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.accempty[bi]);
                continue;
            }
            constexpr int CH = BN < 16 ? BN : 16;   // tokens per chunk
            constexpr int HCH = CH / 2;             // UP: tokens per warp of a gate/up pair
            for (int c0 = 0; c0 < BN && ok; c0 += CH, ++xc) {
                // sum over the pipelines and the four planes for tokens c0..c0+CH-1; the
                // NVFP4 planes carry the extra factor 2^(3p) in their scales
                float val[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) val[j] = 0.0f;
                constexpr float kPw[kMxPlanes] = {1.0f, FMT == kBsNv ? 0.125f : 1.0f, FMT == kBsNv ? 0.015625f : 1.0f,
                                                  FMT == kBsNv ? 0.001953125f : 1.0f};
                if constexpr (BN <= 8 && PL == kMxPlanes) {
                    for (int w = wlo; w < whi; ++w) {   // all N <= 32 columns of pipeline w
                        uint32_t v0[16], v1[16];
                        tmem_ld16(acc0 + w * N, v0);
                        if constexpr (N > 16) tmem_ld16(acc0 + w * N + 16, v1);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < BN; ++j) {
#pragma unroll
                            for (int pl = 0; pl < kMxPlanes; ++pl) {
                                const int col = pl * BN + j;
                                val[j] = fmaf(__uint_as_float(col < 16 ? v0[col & 15] : v1[col & 15]), kPw[pl], val[j]);
                            }
                        }
                    }
                } else {
                    for (int w = wlo; w < whi; ++w) {
                        uint32_t v[PL][16];
#pragma unroll
                        for (int pl = 0; pl < PL; ++pl) tmem_ld16(acc0 + w * N + pl * BN + c0, v[pl]);
                        tmem_wait_ld();
#pragma unroll
                        for (int pl = 0; pl < PL; ++pl)
#pragma unroll
                            for (int j = 0; j < 16; ++j) val[j] = fmaf(__uint_as_float(v[pl][j]), kPw[pl], val[j]);
                    }
                }
                if constexpr (PL == 1) {   // A4: the tensor scales of the weights and (UP) of x; h has 1
#pragma unroll
                    for (int j = 0; j < CH; ++j) val[j] *= iscale;
                } else if constexpr (FMT == kBsNv) {   // 2^-C of each token row, times the expert's tensor scale
                    // one load per lane (token c0 + lane), handed to the other lanes
                    const int Cl = (lane < CH && c0 + lane < it.nvalid) ? __ldcg(p.rowexp + it.row0 + c0 + lane) : 0;
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        const int C = __shfl_sync(0xffffffffu, Cl, j);
                        val[j] *= exp2_neg_biased(C + 127) * iscale;
                    }
                }
                if (PHASE == kPhaseDown) {
                    const int ch = it.m * 128 + lrow;
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        if (c0 + j < it.nvalid) {
                            const int64_t o = (int64_t)(it.row0 + c0 + j) * p.H + ch;
                            if (p.out_fp32) reinterpret_cast<float *>(p.out)[o] = val[j];
                            else reinterpret_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(val[j]);
                        }
                    }
                } else {
                    // Warp q < 2 holds the gate rows of channels 32 q..32 q+31 of this M tile,
                    // warp q + 2 the up rows of the same channels. The gate warp finishes
                    // tokens 0..HCH-1 of the chunk and the up warp tokens HCH..CH-1; each
                    // hands the other the values of the other half through shared memory.
                    const bool gate = q < 2;
                    const int pr = q & 1;
                    if (!mbar_wait(&sm.xempty[grp], (xc & 1) ^ 1, abort_flag)) { ok = false; break; }
                    float *mine = xg + ((gate ? 0 : 64) + pr * 32 + lane) * kMxXch;
                    const float *theirs = xg + ((gate ? 64 : 0) + pr * 32 + lane) * kMxXch;
#pragma unroll
                    for (int j = 0; j < HCH; ++j) mine[j] = val[gate ? HCH + j : j];
                    mbar_arrive(&sm.xfull[grp]);
                    if (!mbar_wait(&sm.xfull[grp], xc & 1, abort_flag)) { ok = false; break; }
                    float other[8];
#pragma unroll
                    for (int j = 0; j < HCH; ++j) other[j] = theirs[j];
                    mbar_arrive(&sm.xempty[grp]);
                    const int t0 = gate ? 0 : HCH;   // first token of this warp's half
                    // channel ch = 64 m + 32 pr + lane: this warp holds one 32-block of h,
                    // which is one 16-byte chunk of a row of the down pass's activation blob
                    const int ch = it.m * 64 + pr * 32 + lane;
                    if constexpr (PL == 1) {
                        // A4: h in NVFP4 form with tensor scale 1. A 16-block of channels is 16 lanes:
                        // scale E4M3(amax / 6), codes E2M1(h / scale); lane pairs share a byte.
                        const int c16 = (ch >> 5) & 7, b16 = (ch & 255) >> 4;
                        uint8_t *blob = p.bblob_out + ((int64_t)it.rt_out * (p.I / kMxStageK) + (ch >> 8)) * BBLOB;
#pragma unroll
                        for (int j = 0; j < HCH; ++j) {
                            const float g = gate ? val[j] : other[j];
                            const float uu = gate ? other[j] : val[HCH + j];
                            const float hv = __fdividef(g, 1.0f + __expf(-g)) * uu;
                            float amax = fabsf(hv);
#pragma unroll
                            for (int d = 1; d < 16; d <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
                            const uint32_t sc = e4m3_code(__fdiv_rn(amax, 6.0f));
                            const float sb = e4m3_value(sc);
                            const float t = sb > 0.0f ? __fdiv_rn(hv, sb) : 0.0f;
                            const float to = __shfl_xor_sync(0xffffffffu, t, 1);
                            const bool odd = lane & 1;
                            uint32_t wv = e2m1x2_code(odd ? to : t, odd ? t : to) << (8 * ((lane >> 1) & 3));
                            wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
                            wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
                            const int tok = c0 + t0 + j;
                            if (tok < it.nvalid) {   // warp-uniform
                                if ((lane & 7) == 0)
                                    *reinterpret_cast<uint32_t *>(blob + sw128_chunk(tok, c16) + (lane >> 3) * 4) = wv;
                                if ((lane & 15) == 0) blob[N * 128 + (b16 >> 2) * 512 + atom_offset(tok, b16 & 3)] = (uint8_t)sc;
                            }
                        }
                        continue;
                    }
                    if constexpr (FMT == kBsNv) {   // h in bf16; the NVFP4 quantiser makes its planes
#pragma unroll
                        for (int j = 0; j < HCH; ++j) {
                            const float g = gate ? val[j] : other[j];
                            const float uu = gate ? other[j] : val[HCH + j];
                            const int tok = c0 + t0 + j;
                            if (tok < it.nvalid)
                                reinterpret_cast<__nv_bfloat16 *>(p.hout)[(int64_t)(it.row0 + tok) * p.I + ch] =
                                    __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * uu);
                        }
                        continue;
                    }
                    const int c16 = (ch >> 5) & 7;   // 32-block within the 256-wide stage
                    uint8_t *blob = p.bblob_out + ((int64_t)it.rt_out * (p.I / kMxStageK) + (ch >> 8)) * BBLOB;
#pragma unroll
                    for (int j = 0; j < HCH; ++j) {
                        const float g = gate ? val[j] : other[j];
                        const float uu = gate ? other[j] : val[HCH + j];
                        float r = __bfloat162float(__float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * uu));
                        // block maximum: non-negative floats order like their bit patterns
                        const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r))));
                        const int s = mx_plane0_exp(amax);
                        const int tok = c0 + t0 + j;
#pragma unroll
                        for (int pl = 0; pl < kMxPlanes; ++pl) {
                            // lanes 2i and 2i+1 round the same pair (channel 2i in the low
                            // nibble); each keeps its own rounded value
                            const int sp = s - 3 * pl;
                            const float t = r * exp2_neg_biased(sp);
                            const float to = __shfl_xor_sync(0xffffffffu, t, 1);
                            const bool odd = lane & 1;
                            float qlo, qhi;
                            uint32_t wv = e2m1x2(odd ? to : t, odd ? t : to, &qlo, &qhi) << (8 * ((lane >> 1) & 3));
                            r = fmaf(-(odd ? qhi : qlo), exp2_biased(sp), r);
                            wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
                            wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
                            if (tok < it.nvalid) {   // warp-uniform
                                const int R = pl * BN + tok;
                                if ((lane & 7) == 0)
                                    *reinterpret_cast<uint32_t *>(blob + sw128_chunk(R, c16) + (lane >> 3) * 4) = wv;
                                if (lane == 0) blob[N * 128 + (c16 >> 2) * 512 + atom_offset(R, c16 & 3)] = (uint8_t)sp;
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            tc_fence_before();
            mbar_arrive(&sm.accempty[bi]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 12) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

// Token tile of the block-scaled path from the mean rows per expert. The
// smallest tile is 8, not 4: with skewed routing a few experts take many rows,
// and every extra tile of an expert passes its weights through the SM again,
// while a half-empty tile of 8 costs only activation bytes.
int choose_bn_mx(int n_rows, int E) {
    const int avg = (n_rows + E - 1) / (E > 0 ? E : 1);
    if (avg <= 8) return 8;
    if (avg <= 16) return 16;
    return 32;
}

size_t mx_tiles_ub(int n_rows, int E) {
    const int BN = choose_bn_mx(n_rows, E);
    return (size_t)(n_rows + BN - 1) / BN + (size_t)E;
}

// Token tile of the A4 path (one plane, so up to 128 tokens fill N = 128): from the
// mean rows per expert, 32, 64 or 128.
int choose_bn_a4(int n_rows, int E) {
    const int avg = (n_rows + E - 1) / (E > 0 ? E : 1);
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    return 128;
}

size_t a4_blob_bytes(int n_rows, int K, int E) {
    const int BN = choose_bn_a4(n_rows, E);
    const size_t tiles = (size_t)(n_rows + BN - 1) / BN + (size_t)E;
    return align_up(tiles * (K / kMxStageK) * bs_bblob_bytes(kBsNv, BN, 1), 256);
}

// Activation blob bytes of n_rows rows and reduction K, sized for NVFP4 (the
// larger of the two formats' blobs).
size_t mx_blob_bytes(int n_rows, int K, int E) {
    return align_up(mx_tiles_ub(n_rows, E) * (K / kMxStageK) * bs_bblob_bytes(kBsNv, choose_bn_mx(n_rows, E)), 256);
}

// The largest blob over all row counts up to n_rows. Each size grows with the rows
// while the tile height stays put; it can drop where the height steps up (the mean
// rows per expert passing 8 and 16, or 32 and 64), so the last row count before each
// step is a candidate.
size_t mx_blob_bound(int n_rows, int K, int E) {
    size_t m = mx_blob_bytes(n_rows, K, E);
    for (int avg : {8, 16})
        if ((int64_t)avg * E < n_rows) m = std::max(m, mx_blob_bytes(avg * E, K, E));
    return m;
}

size_t a4_blob_bound(int n_rows, int K, int E) {
    size_t m = a4_blob_bytes(n_rows, K, E);
    for (int avg : {32, 64})
        if ((int64_t)avg * E < n_rows) m = std::max(m, a4_blob_bytes(avg * E, K, E));
    return m;
}

static size_t mx_smem_bytes(int fmt, int phase, int BN, int stages, int E, int planes) {
    const size_t stage = (size_t)bs_ablob_bytes(fmt) + bs_bblob_bytes(fmt, BN, planes);
    return 1024 + stages * stage + (phase == kPhaseUp ? 2 * 128 * kMxXch * 4 : 0) + sizeof(MxSmem) +
           (size_t)(4 * E + 3) * sizeof(int);
}

template <int FMT, int PHASE, int BN, int PL>
static cudaError_t mx_launch_one(const MxParams &p, int grid, size_t smem, cudaStream_t st) {
    auto kfn = ffn_mx_kernel<FMT, PHASE, BN, PL>;
    cudaError_t e = ensure_max_smem<ffn_mx_kernel<FMT, PHASE, BN, PL>>((int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kfn, dim3(grid), dim3(kMxThreads), smem, st, p);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

template <int FMT, int PHASE>
static cudaError_t mx_launch_bn(int BN, const MxParams &p, int grid, size_t smem, cudaStream_t st) {
    switch (BN) {
        case 8: return mx_launch_one<FMT, PHASE, 8, kMxPlanes>(p, grid, smem, st);
        case 16: return mx_launch_one<FMT, PHASE, 16, kMxPlanes>(p, grid, smem, st);
        default: return mx_launch_one<FMT, PHASE, 32, kMxPlanes>(p, grid, smem, st);
    }
}

template <int PHASE>
static cudaError_t a4_launch_bn(int BN, const MxParams &p, int grid, size_t smem, cudaStream_t st) {
    switch (BN) {
        case 32: return mx_launch_one<kBsNv, PHASE, 32, 1>(p, grid, smem, st);
        case 64: return mx_launch_one<kBsNv, PHASE, 64, 1>(p, grid, smem, st);
        default: return mx_launch_one<kBsNv, PHASE, 128, 1>(p, grid, smem, st);
    }
}

// Pipelines and ring depth of one phase: as many pipelines as divide the
// stages of an item and fit TMEM (4 for N <= 32, 2 for N = 64, else 1), with
// at least two slots each in the shared memory of one CTA. False if none fits.
// When that leaves one stage per item and pipeline, every stage would be an
// item boundary for its MMA warp: the pipelines take whole items instead.
bool mx_plan(int fmt, int phase, int BN, int K, int E, MxPlan *pl, int planes) {
    const int KST = K / kMxStageK;
    const int N = planes * BN;
    const int nw = N <= 32 ? 4 : (N <= 64 ? 2 : 1);
    int fit = kMxMaxStages;
    while (fit > 0 && mx_smem_bytes(fmt, phase, BN, fit, E, planes) > (size_t)kMxSmemCap) --fit;
    for (int np = nw < KST ? nw : KST; np >= 1; --np) {
        if (KST % np) continue;
        const int nsw = fit / np;
        if (nsw < 2) continue;
        pl->pipes = np;
        pl->stages = np * nsw;
        pl->itempar = np > 1 && KST / np == 1;
        // a third accumulator buffer lets the MMAs run up to two items ahead of the epilogue,
        // so a slow epilogue does not stop the weight stream (the ring holds about one item)
        const bool tm = planes == 1 && BN == 128;
        pl->nbuf = (!pl->itempar && !tm && 3 * nw * N + nw * 16 * bs_atoms(fmt) <= 512) ? 3 : 2;
        return true;
    }
    return false;
}

moe_status launch_mx_phase(int fmt, int phase, int BN, MxParams p, int num_sms, cudaStream_t st, int planes) {
    if (p.K % kMxStageK) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", p.K, kMxStageK);
    if (planes != kMxPlanes && (planes != 1 || fmt != kBsNv))
        return set_error(MOE_ERR_UNSUPPORTED, "A4 activations need NVFP4 experts");
    MxPlan pl;
    if (!mx_plan(fmt, phase, BN, p.K, p.E, &pl, planes))
        return set_error(MOE_ERR_UNSUPPORTED, "K=%d: no pipeline plan for the block-scaled FP4 path", p.K);
    p.pipes = pl.pipes;
    p.stages = pl.stages;
    p.itempar = pl.itempar;
    p.nbuf = pl.nbuf;
    size_t smem = mx_smem_bytes(fmt, phase, BN, pl.stages, p.E, planes);
    if (smem < 120 * 1024) smem = 120 * 1024;   // one CTA per SM: it allocates all 512 TMEM columns
    const int64_t items_ub = ((int64_t)p.n_rows / BN + p.E) * p.m_tiles;
    const int grid = (int)(items_ub < num_sms ? (items_ub > 0 ? items_ub : 1) : num_sms);
    cudaError_t e;
    if (planes == 1)
        e = phase == kPhaseUp ? a4_launch_bn<kPhaseUp>(BN, p, grid, smem, st) : a4_launch_bn<kPhaseDown>(BN, p, grid, smem, st);
    else if (fmt == kBsNv)
        e = phase == kPhaseUp ? mx_launch_bn<kBsNv, kPhaseUp>(BN, p, grid, smem, st)
                              : mx_launch_bn<kBsNv, kPhaseDown>(BN, p, grid, smem, st);
    else
        e = phase == kPhaseUp ? mx_launch_bn<kBsMx, kPhaseUp>(BN, p, grid, smem, st)
                              : mx_launch_bn<kBsMx, kPhaseDown>(BN, p, grid, smem, st);
    if (e != cudaSuccess) return set_cuda_error(e, "block-scaled ffn kernel launch");
    return MOE_OK;
}

moe_status launch_mx_quant(int fmt, const void *src, int mode, const int32_t *sorted_pair, int k, int P, int K,
                           const int32_t *offsets, int E, int BN, void *bblob, int32_t *rowexp, int num_sms,
                           cudaStream_t st, int *sched_zero) {
    if (P == 0) return MOE_OK;
    if (E > kMaxExperts) return set_error(MOE_ERR_UNSUPPORTED, "E=%d above %d", E, kMaxExperts);
    if (K % kMxStageK) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", K, kMxStageK);
    cudaError_t e;
    if (fmt == kBsNv) {   // one block per row
        const int blocks = P < num_sms * 8 ? P : num_sms * 8;
        e = launch_pdl(nv_quant_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4 *>(src), mode,
                       sorted_pair, k, P, K, offsets, E, BN, reinterpret_cast<uint8_t *>(bblob), rowexp, sched_zero);
    } else {              // one warp per (row, stage)
        if (mode == 2) return set_error(MOE_ERR_UNSUPPORTED, "MXFP4 quantiser mode 2");
        const int64_t units = (int64_t)P * (K / kMxStageK);
        const int blocks = (int)((units + 7) / 8 < (int64_t)num_sms * 8 ? (units + 7) / 8 : (int64_t)num_sms * 8);
        e = launch_pdl(mx_quant_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4 *>(src), mode,
                       sorted_pair, k, P, K, offsets, E, BN, reinterpret_cast<uint8_t *>(bblob), sched_zero);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "block-scaled quantiser launch");
}

}  // namespace moe

namespace moe {

moe_status launch_a4_amax(const void *src, int64_t n_elems, float *partials, int *sched_zero, cudaStream_t st) {
    const int64_t n8 = n_elems / 8;
    cudaError_t e = launch_pdl(a4_amax_kernel, dim3(kA4Parts), dim3(256), 0, st, reinterpret_cast<const uint4 *>(src),
                               n8, partials, sched_zero);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "A4 amax launch");
}

moe_status launch_a4_quant(const void *src, int mode, const int32_t *sorted_pair, int k, int P, int K,
                           const int32_t *offsets, int E, int BN, const float *partials, float *xscale, void *bblob,
                           int num_sms, cudaStream_t st) {
    if (P == 0) return MOE_OK;
    if (E > kMaxExperts) return set_error(MOE_ERR_UNSUPPORTED, "E=%d above %d", E, kMaxExperts);
    if (K % kMxStageK) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", K, kMxStageK);
    const int64_t units = (int64_t)P * (K / kMxStageK);
    const int blocks = (int)((units + 7) / 8 < (int64_t)num_sms * 8 ? (units + 7) / 8 : (int64_t)num_sms * 8);
    cudaError_t e = launch_pdl(a4_quant_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4 *>(src),
                               mode, sorted_pair, k, P, K, offsets, E, BN, partials, xscale,
                               reinterpret_cast<uint8_t *>(bblob));
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "A4 quantiser launch");
}

}  // namespace moe

namespace moe {

moe_status launch_a4_token_rows(const void *x, int T, int K, int k, const int32_t *pair_row, const int32_t *offsets,
                                int E, int BN, const float *partials, float *xscale, void *bblob, int num_sms,
                                cudaStream_t st) {
    if (T == 0) return MOE_OK;
    if (E > kMaxExperts) return set_error(MOE_ERR_UNSUPPORTED, "E=%d above %d", E, kMaxExperts);
    if (K % kMxStageK) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", K, kMxStageK);
    const int64_t units = (int64_t)T * (K / kMxStageK);
    const int blocks = (int)((units + 7) / 8 < (int64_t)num_sms * 8 ? (units + 7) / 8 : (int64_t)num_sms * 8);
    cudaError_t e = launch_pdl(a4_token_rows_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st,
                               reinterpret_cast<const uint4 *>(x), T, K, k, pair_row, offsets, E, BN, partials, xscale,
                               reinterpret_cast<uint8_t *>(bblob));
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "A4 token rows launch");
}

}  // namespace moe
