// Grouped SwiGLU expert FFN for MXFP4 experts on the block-scaled tensor core
// path: tcgen05.mma kind::mxf8f6f4.block_scale, E2M1 weights (A) times E4M3
// activations (B), one E8M0 scale per 32 K elements on both sides, fp32
// accumulation in TMEM. The weights are never decoded by the SM: the FP4
// codes go from HBM to shared memory by TMA, which spreads every 16 codes
// over 16 bytes (the operand layout this MMA kind reads), and their E8M0
// block scales go from shared memory to TMEM with tcgen05.cp.
//
// Activations keep bf16 precision: a bf16 value x in a block with E8M0
// exponent s is split as x = 2^s hi + 2^(s-4) lo with hi = rn_e4m3(x 2^-s) and
// lo = rn_e4m3(16 (x 2^-s - hi)). bf16 has 8 significant bits and E4M3 4, so
// the split is exact whenever lo is an E4M3 normal, i.e. for every element
// within 2^13 of its block maximum. hi rows and lo rows are stacked along N:
// one MMA with N = 2 BN yields both products (the lo rows carry scale s - 4),
// and the epilogue adds column j and column BN + j.
//
// Work item: an N tile of BN rows of one expert x one M tile of 128 weight rows
// (UP: 64 gate rows and the matching 64 up rows; DOWN: 128 rows). The warp
// roles are described at the kernel.
// A scale atom is 512 bytes: byte (r % 32) * 16 + (r / 32) * 4 + j holds the
// scale of operand row r and K block j of the stage; tcgen05.cp 32x128b.warpx4
// puts atom row l into TMEM lanes l, l+32, l+64, l+96 (4 columns), which is
// where the MMA reads the scale of row r: lane r, column r / 32, byte j.
//
// Every wait is bounded; on timeout the CTA sets the device error word, drains
// its copies and MMAs and exits.
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kMxThreads = 512;
constexpr int kMxBK = 128;                    // K elements per stage
constexpr int kMxCodeBytes = 128 * 64;        // packed FP4 codes of one (M tile, stage)
constexpr int kMxMaxStages = 12;
constexpr int kMxSfSlots = 4;                 // TMEM scale slots (8 columns each)
constexpr int kMxXch = 9;    // padded row of the gate/up exchange (8 values)

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(m), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// 32 rows x 16 bytes of shared memory -> TMEM lanes (l, l+32, l+64, l+96), 4 columns.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-32 E8M0 scales from TMEM.
__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Shared-memory descriptor of a scale atom: no swizzle, K-major, core matrices
// of 8 rows x 16 bytes stacked 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
           (1ull << 46);
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: A E2M1, B E4M3, E8M0
// scales, both K-major, M = 128; scale byte `id` of each 32-bit scale column.
__host__ __device__ constexpr uint32_t idesc_mx(int N, uint32_t id) {
    return (id << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) |
           (id << 29);
}

// Split 8 values of one 32-block (the caller gives the block's E8M0 exponent
// s, biased) into E4M3 hi and lo bytes.
__device__ __forceinline__ void mx_split8(const float (&v)[8], int sbiased, uint2 &hi, uint2 &lo) {
    const float inv = __uint_as_float((uint32_t)(254 - sbiased) << 23);   // 2^-(s - 127)
    uint32_t h[2] = {0, 0}, l[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float a = v[i] * inv, b = v[i + 1] * inv;
        const __nv_fp8x2_storage_t hp = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(hp, __NV_E4M3);
        const float2 hf = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
        const __nv_fp8x2_storage_t lp =
            __nv_cvt_float2_to_fp8x2(make_float2((a - hf.x) * 16.0f, (b - hf.y) * 16.0f), __NV_SATFINITE, __NV_E4M3);
        h[i >> 2] |= (uint32_t)hp << (8 * (i & 3));
        l[i >> 2] |= (uint32_t)lp << (8 * (i & 3));
    }
    hi = make_uint2(h[0], h[1]);
    lo = make_uint2(l[0], l[1]);
}

// Biased E8M0 exponent of the hi part of a block with maximum magnitude amax:
// the block maximum lands in [128, 256), inside E4M3's range; the lo part uses
// this minus 4. Kept in [4, 253] so both are valid E8M0 values and 2^-s is a
// normal float.
__device__ __forceinline__ int mx_block_exp(float amax) {
    if (!(amax > 0.0f)) return 127;
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;   // floor(log2) for normal amax
    int s = e - 7 + 127;
    return s < 4 ? 4 : (s > 253 ? 253 : s);
}

__device__ __forceinline__ uint32_t atom_offset(int row, int j) { return (row & 31) * 16 + (row >> 5) * 4 + j; }

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

// One warp per permuted row r (grid-stride). The row is x[sorted_pair[r] / k]
// (gather != 0, natural order) or x_perm[r] (operand order); it is written as
// E4M3 hi/lo planes q[0][r][K], q[1][r][K] in natural order, and its block
// scales go into the scale atoms of its N tile: tile = tile_start[e] + (r -
// offsets[e]) / BN, atom row n (hi) and n + BN (lo), n = (r - offsets[e]) % BN.
__global__ void __launch_bounds__(256) mx_quant_kernel(const uint4 *__restrict__ src, int gather,
                                                       const int32_t *__restrict__ sorted_pair, int k, int P, int K,
                                                       const int32_t *__restrict__ offsets, int E, int BN,
                                                       uint8_t *__restrict__ q, uint8_t *__restrict__ sfb) {
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_tile[kMaxExperts + 1];
    __shared__ int s_wsum[8];
    pdl_wait();
    pdl_release();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    // tile prefix: s_tile[e] = sum over e' < e of ceil(n_e' / BN), 256 threads x 4 experts
    {
        int cnt[4], run = 0;
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
    }
    __syncthreads();
    const int K8 = K / 8, KB = K / kMxBK;
    const int gw = blockIdx.x * 8 + warp, nw = gridDim.x * 8;
    for (int r = gw; r < P; r += nw) {
        int lo = 0, hi = E - 1;   // expert with s_off[e] <= r < s_off[e + 1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_off[mid] <= r) lo = mid; else hi = mid - 1;
        }
        const int rel = r - s_off[lo];
        const int tile = s_tile[lo] + rel / BN, n = rel % BN;
        const uint4 *srow = src + (int64_t)(gather ? sorted_pair[r] / k : r) * K8;
        uint8_t *atom0 = sfb + (int64_t)tile * KB * 512;
        // four 16-byte chunks per lane in flight, then each is split
        for (int c0 = lane; c0 < K8; c0 += 128) {
            uint4 uu[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (c0 + 32 * i < K8) uu[i] = srow[c0 + 32 * i];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = c0 + 32 * i;
                if (c >= K8) break;   // warp-uniform: K8 is a multiple of 32
                uint4 u = uu[i];
                if (!gather) u = deinterleave8(u);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
                float v[8];
                float amax = 0.0f;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[h]));
                    v[2 * h] = f.x;
                    v[2 * h + 1] = f.y;
                    amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                const int s = mx_block_exp(amax);
                uint2 h2, l2;
                mx_split8(v, s, h2, l2);
                *reinterpret_cast<uint2 *>(q + (int64_t)r * K + c * 8) = h2;
                *reinterpret_cast<uint2 *>(q + ((int64_t)P + r) * K + c * 8) = l2;
                if ((c & 3) == 0) {
                    const int b = c >> 2;   // 32-block along K
                    uint8_t *atom = atom0 + (b >> 2) * 512;
                    atom[atom_offset(n, b & 3)] = (uint8_t)s;
                    atom[atom_offset(n + BN, b & 3)] = (uint8_t)(s - 4);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ grouped FFN kernel

struct MxSmem {
    uint64_t full[kMxMaxStages];
    uint64_t empty[kMxMaxStages];
    uint64_t accfull[2];      // both MMA warps commit
    uint64_t accempty[2];     // the epilogue group of that buffer (128 threads)
    uint64_t mmadone[4];
    uint64_t xfull[2], xempty[2];   // gate/up exchange, per epilogue group
    uint32_t tmem_base;
    int abort_flag;
    int total_items;
    int tile_start[kMaxExperts + 1];
};

struct MxItem {
    int e, rt, row0, nvalid, m;
};

__device__ __forceinline__ MxItem mx_item(const MxSmem &sm, const MxParams &p, int item, int BN) {
    MxItem it;
    it.rt = item / p.m_tiles;
    it.m = item - it.rt * p.m_tiles;
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.tile_start[mid] <= it.rt) lo = mid; else hi = mid - 1;
    }
    it.e = lo;
    const int t = it.rt - sm.tile_start[lo];
    const int beg = p.offsets[lo];
    it.row0 = beg + t * BN;
    it.nvalid = min(BN, p.offsets[lo + 1] - beg - t * BN);
    return it;
}

// Warp roles (512 threads, one CTA per SM, persistent over items). The K
// stages of an item are dealt round-robin to NP independent pipelines: pipeline
// w (producer warp w, MMA warp 12 + w, its own ring of slots and its own
// accumulators) handles stages w, w + NP, ... of every item, in order. One
// producer fills and one issuer drains each slot, both in order, so every
// parity wait on a slot barrier is exactly one phase after the previous one.
//   warps 0-3   producers: per stage (SUB consecutive 128-wide K blocks) one
//               TMA box of FP4 codes, one bulk copy of their scale atoms, one
//               4D TMA box of the E4M3 hi/lo rows, one bulk copy of their scale
//               atoms. Warp 2 also builds the per-expert tile prefix first.
//   warps 12-15 MMA issuers (warp 12 owns TMEM).
//   warps 4-7   epilogue of even items (accumulator buffer 0);
//   warps 8-11  epilogue of odd items (buffer 1). The epilogue adds the NP
//               pipelines' accumulators.
// TMEM columns: accumulator (buffer a, pipeline w) at (a NW + w) N; four scale
// slots of 8 columns per pipeline from 2 NW N on.
template <int PHASE, int BN>
__global__ void __launch_bounds__(kMxThreads, 1)
ffn_mx_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap bmap, MxParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr int N = 2 * BN;                     // MMA N: hi rows then lo rows
    constexpr int NW = N <= 32 ? 4 : 2;           // pipelines TMEM has room for
    constexpr int A_BYTES = 128 * 128;            // FP4 codes of one K block, one byte each in shared memory
    constexpr int B_BYTES = N * 128;              // E4M3 rows of one K block
    const int SUB = p.sub;
    const int STAGE = SUB * (A_BYTES + B_BYTES + 1024);
    const uint32_t TX = (uint32_t)SUB * (A_BYTES / 2 + B_BYTES + 1024);   // FP4 boxes count packed bytes
    const uint32_t SFCOL = 2 * NW * N;                                   // first scale slot column
    const int NP = p.pipes;                       // pipelines (divides the stages per item, <= NW)
    const int NSW = p.stages / NP;                // slots per pipeline

    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int ns = p.stages;
    float *xch = reinterpret_cast<float *>(base + ns * STAGE);   // [2 groups][2 halves][64][kMxXch]
    MxSmem &sm = *reinterpret_cast<MxSmem *>(reinterpret_cast<uint8_t *>(xch) +
                                            (PHASE == kPhaseUp ? 2 * 128 * kMxXch * 4 : 0));
    const int warp = warp_id(), lane = lane_id();
    volatile int *abort_flag = &sm.abort_flag;

    const int KB = p.K / kMxBK;      // 128-wide K blocks
    const int NST = KB / SUB;        // stages per item
    const int PER = NST / NP;        // stages per item and pipeline
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMxMaxStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sm.accfull[a], NP);
            mbar_init(&sm.accempty[a], 128);
            mbar_init(&sm.xfull[a], 128);
            mbar_init(&sm.xempty[a], 128);
        }
        for (int w = 0; w < 4; ++w) mbar_init(&sm.mmadone[w], 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp < 4 && warp < NP && lane == 0) {
        tma_prefetch_desc(&wmap);
        tma_prefetch_desc(&bmap);
    }
    if (warp == 12) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        int run = 0;
        if (lane == 0) sm.tile_start[0] = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int nt = 0;
            if (e < p.E) nt = (p.offsets[e + 1] - p.offsets[e] + BN - 1) / BN;
            int incl = nt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            if (e < p.E) sm.tile_start[e + 1] = run + incl;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) sm.total_items = run * p.m_tiles;
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
            // Weight half of a stage (FP4 codes + their scale atoms): static data.
            auto issue_weights = [&](const MxItem &it, int st, int s) {
                const int slot = p.expert_map ? p.expert_map[it.e] : it.e;
                const uint8_t *wexp = p.wbase + (int64_t)slot * p.w_estride;
                const int blk = it.m * KB + st * SUB;
                uint64_t *fb = &sm.full[s];
                uint8_t *sp = base + s * STAGE;
                mbar_expect_tx(fb, TX);
                tma_load_4d(sp, &wmap, fb, 0, 0, blk, slot);
                bulk_load(sp + SUB * (A_BYTES + B_BYTES), wexp + (int64_t)p.m_tiles * KB * kMxCodeBytes + (int64_t)blk * 512,
                          SUB * 512, fb);
            };
            // The slots start empty: the weights of this pipeline's first NSW stages go out
            // before waiting for the kernel that writes the activations.
            int pre = 0;
            for (int item = blockIdx.x; item < total && pre < NSW; item += gridDim.x) {
                const MxItem it = mx_item(sm, p, item, BN);
                for (int st = w; st < NST && pre < NSW; st += NP, ++pre) issue_weights(it, st, w * NSW + pre);
            }
            pdl_wait();
            if (w == 0) pdl_release();
            int loc = 0;   // stages this pipeline has issued
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const MxItem it = mx_item(sm, p, item, BN);
                for (int st = w; st < NST; st += NP, ++loc) {
                    const int s = w * NSW + loc % NSW;
                    const uint32_t round = (uint32_t)(loc / NSW);
                    if (loc >= pre) {
                        if (!mbar_wait(&sm.empty[s], (round & 1) ^ 1, abort_flag)) { ok = false; break; }
                        issue_weights(it, st, s);
                    }
                    uint64_t *fb = &sm.full[s];
                    uint8_t *sp = base + s * STAGE;
                    const int kb = st * SUB;
                    tma_load_4d(sp + SUB * A_BYTES, &bmap, fb, 0, it.row0, 0, kb);
                    bulk_load(sp + SUB * (A_BYTES + B_BYTES) + SUB * 512, p.sfb + ((int64_t)it.rt * KB + kb) * 512,
                              SUB * 512, fb);
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
    } else if (warp >= 12) {
        // =================================================== MMA issuer of pipeline w
        const int w = warp - 12;
        if (lane == 0 && w < NP) {
            int loc = 0, lt = 0, sc = 0;
            bool ok = true;
            const uint32_t base_u32 = smem_u32(base);
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
                const int a = lt & 1;
                if (!mbar_wait(&sm.accempty[a], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)((a * NW + w) * N);
                for (int k = 0; k < PER; ++k, ++loc) {
                    const int s = w * NSW + loc % NSW;
                    if (!mbar_wait(&sm.full[s], (uint32_t)((loc / NSW) & 1), abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sp = base_u32 + s * STAGE;
                    const uint32_t sfa_s = sp + SUB * (A_BYTES + B_BYTES), sfb_s = sfa_s + SUB * 512;
                    for (int i = 0; i < SUB; ++i) {
                        const uint32_t sfa = tmem + SFCOL + 32 * w + sc * 8, sfb = sfa + 4;
                        tmem_cp_atom(sfa, sf_atom_desc(sfa_s + i * 512));
                        tmem_cp_atom(sfb, sf_atom_desc(sfb_s + i * 512));
                        const uint64_t adesc = smem_desc_sw128(sp + i * A_BYTES);
                        const uint64_t bdesc = smem_desc_sw128(sp + SUB * A_BYTES + i * B_BYTES);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_mx(d, adesc + (uint64_t)((j * 32) >> 4), bdesc + (uint64_t)((j * 32) >> 4),
                                   idesc_mx(N, (uint32_t)j), sfa | ((uint32_t)j << 30), sfb | ((uint32_t)j << 30),
                                   (k | i | j) != 0);
                        if (++sc == kMxSfSlots) sc = 0;
                    }
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.accfull[a]);
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
        for (int item = blockIdx.x + grp * gridDim.x; item < total && ok; item += 2 * gridDim.x, lt += 2) {
            const MxItem it = mx_item(sm, p, item, BN);
            const int a = grp;
            if (!mbar_wait(&sm.accfull[a], (lt >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t acc0 = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * NW * N);
            constexpr int CH = BN < 16 ? BN : 16;   // tokens per chunk
            constexpr int HCH = CH / 2;             // UP: tokens per warp of a gate/up pair
            for (int c0 = 0; c0 < BN && ok; c0 += CH, ++xc) {
                // hi + lo columns of the pipelines' accumulators for tokens c0..c0+CH-1
                float val[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) val[j] = 0.0f;
                if (BN < 16) {
                    uint32_t v[4][16];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if (w < NP) tmem_ld16(acc0 + w * N, v[w]);   // columns 0..BN-1 hi, BN..2BN-1 lo
                    tmem_wait_ld();
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if (w < NP) {
#pragma unroll
                            for (int j = 0; j < CH; ++j)
                                val[j] += __uint_as_float(v[w][j]) + __uint_as_float(v[w][(j + BN) & 15]);
                        }
                } else {
                    for (int w = 0; w < NP; ++w) {
                        uint32_t v[16], u[16];
                        tmem_ld16(acc0 + w * N + c0, v);
                        tmem_ld16(acc0 + w * N + BN + c0, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) val[j] += __uint_as_float(v[j]) + __uint_as_float(u[j]);
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
                    // channel ch = 64 m + 32 pr + lane: this warp holds one 32-block of h
                    const int ch = it.m * 64 + pr * 32 + lane;
                    const int blk = ch >> 5;                // 32-block along I
                    uint8_t *atom = p.sfb_out + ((int64_t)it.rt * (p.I / kMxBK) + (blk >> 2)) * 512;
#pragma unroll
                    for (int j = 0; j < HCH; ++j) {
                        const float g = gate ? val[j] : other[j];
                        const float uu = gate ? other[j] : val[HCH + j];
                        const float hv = __bfloat162float(__float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * uu));
                        // block maximum: non-negative floats order like their bit patterns
                        const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv))));
                        const int s = mx_block_exp(amax);
                        const float inv = __uint_as_float((uint32_t)(254 - s) << 23);
                        const float x = hv * inv;
                        const __nv_fp8_storage_t hb = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
                        const __half_raw hr = __nv_cvt_fp8_to_halfraw(hb, __NV_E4M3);
                        const float hf = __half2float(*reinterpret_cast<const __half *>(&hr));
                        const __nv_fp8_storage_t lb = __nv_cvt_float_to_fp8((x - hf) * 16.0f, __NV_SATFINITE, __NV_E4M3);
                        const int tok = c0 + t0 + j;
                        if (tok < it.nvalid) {
                            const int64_t row = it.row0 + tok;
                            p.q_out[row * p.I + ch] = hb;
                            p.q_out[((int64_t)p.n_rows + row) * p.I + ch] = lb;
                            if (lane == 0) {
                                atom[atom_offset(tok, blk & 3)] = (uint8_t)s;
                                atom[atom_offset(tok + BN, blk & 3)] = (uint8_t)(s - 4);
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            tc_fence_before();
            mbar_arrive(&sm.accempty[a]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 12) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

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

size_t mx_sf_bytes(int n_rows, int K, int E) { return align_up(mx_tiles_ub(n_rows, E) * (K / kMxBK) * 512, 256); }

static size_t mx_smem_bytes(int phase, int BN, int sub, int stages) {
    const size_t stage = (size_t)sub * (128 * 128 + (size_t)2 * BN * 128 + 1024);
    return 1024 + stages * stage + (phase == kPhaseUp ? 2 * 128 * kMxXch * 4 : 0) + sizeof(MxSmem);
}

template <int PHASE, int BN>
static cudaError_t mx_launch_one(const CUtensorMap &wmap, const CUtensorMap &bmap, const MxParams &p, int grid,
                                 size_t smem, cudaStream_t st) {
    auto kfn = ffn_mx_kernel<PHASE, BN>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kfn, dim3(grid), dim3(kMxThreads), smem, st, wmap, bmap, p);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

template <int PHASE>
static cudaError_t mx_launch_bn(int BN, const CUtensorMap &wmap, const CUtensorMap &bmap, const MxParams &p,
                                int grid, size_t smem, cudaStream_t st) {
    switch (BN) {
        case 8: return mx_launch_one<PHASE, 8>(wmap, bmap, p, grid, smem, st);
        case 16: return mx_launch_one<PHASE, 16>(wmap, bmap, p, grid, smem, st);
        default: return mx_launch_one<PHASE, 32>(wmap, bmap, p, grid, smem, st);
    }
}

// Stage size, pipelines and ring depth of one phase: one 128-wide K block per
// stage if possible (else two), as many pipelines as divide the stages of an
// item and fit TMEM (4 for N <= 32, else 2), and at least two slots per
// pipeline in at most 220 KiB of shared memory. Returns false if none fits.
bool mx_plan(int phase, int BN, int K, MxPlan *pl) {
    const int KB = K / kMxBK;
    const int nw = 2 * BN <= 32 ? 4 : 2;
    for (int sub = 1; sub <= 2; ++sub) {
        if (KB % sub) continue;
        const int nst = KB / sub;
        int fit = kMxMaxStages;
        while (fit > 0 && mx_smem_bytes(phase, BN, sub, fit) > 220 * 1024) --fit;
        for (int np = nw < nst ? nw : nst; np >= 1; --np) {
            if (nst % np) continue;
            int nsw = fit / np;
            if (nsw > 4) nsw = 4;
            if (nsw < 2) continue;
            pl->sub = sub;
            pl->pipes = np;
            pl->stages = np * nsw;
            return true;
        }
    }
    return false;
}

moe_status launch_mx_phase(int phase, int BN, const CUtensorMap &wmap, const CUtensorMap &bmap, MxParams p,
                           int num_sms, cudaStream_t st) {
    if (p.K % kMxBK) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", p.K, kMxBK);
    MxPlan pl;
    if (!mx_plan(phase, BN, p.K, &pl)) return set_error(MOE_ERR_UNSUPPORTED, "K=%d: no pipeline plan for MXFP4", p.K);
    p.sub = pl.sub;
    p.pipes = pl.pipes;
    p.stages = pl.stages;
    size_t smem = mx_smem_bytes(phase, BN, pl.sub, pl.stages);
    if (smem < 120 * 1024) smem = 120 * 1024;   // one CTA per SM: it allocates all 512 TMEM columns
    const int64_t items_ub = ((int64_t)p.n_rows / BN + p.E) * p.m_tiles;
    const int grid = (int)(items_ub < num_sms ? (items_ub > 0 ? items_ub : 1) : num_sms);
    cudaError_t e = phase == kPhaseUp ? mx_launch_bn<kPhaseUp>(BN, wmap, bmap, p, grid, smem, st)
                                      : mx_launch_bn<kPhaseDown>(BN, wmap, bmap, p, grid, smem, st);
    if (e != cudaSuccess) return set_cuda_error(e, "mx ffn kernel launch");
    return MOE_OK;
}

moe_status launch_mx_quant(const void *src, int gather, const int32_t *sorted_pair, int k, int P, int K,
                           const int32_t *offsets, int E, int BN, void *q, void *sfb, int num_sms, cudaStream_t st) {
    if (P == 0) return MOE_OK;
    if (E > kMaxExperts) return set_error(MOE_ERR_UNSUPPORTED, "E=%d above %d", E, kMaxExperts);
    int blocks = (P + 7) / 8;
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    cudaError_t e = launch_pdl(mx_quant_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4 *>(src),
                               gather, sorted_pair, k, P, K, offsets, E, BN, reinterpret_cast<uint8_t *>(q),
                               reinterpret_cast<uint8_t *>(sfb));
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "mx quant launch");
}

}  // namespace moe
