// Grouped SwiGLU expert FFN on the sm_100a tensor core (tcgen05, kind::f16).
//
// Computes, for every expert e and permuted row r of that expert,
//   UP:   h[r, c]  = silu(Wg_e[c] . x[r]) * (Wu_e[c] . x[r])   (bf16 out)
//   DOWN: y[r, j]  = W2_e[j] . h[r]                           (bf16 or fp32 out)
// with the expert weights stored as MXFP4, NVFP4, FP8 (E4M3, per-128 scales)
// or bf16 (formats named on the aimodeling.com page, section "Reported
// Numbers and Ecosystem Position"; the SwiGLU form is this library's reading).
//
// Design (swap-AB, weights on the MMA M side):
//   * M tile = 128 weight rows. UP: 64 gate rows + the 64 matching up rows, so
//     one MMA produces both halves of the SwiGLU for 64 channels. DOWN: 128 rows.
//   * N tile = BN permuted rows (tokens) of one expert, BN in {16,32,64,128}.
//   * K stage = 128 elements.
//   * Warp roles (512 threads, one CTA per SM, persistent over work items):
//       warp 0      TMA producer: raw weight tile (swizzled), activation tile
//                   (128-byte swizzle), and per tile the scale block (bulk copy).
//       warp 1      owns TMEM; one lane issues tcgen05.mma (A from TMEM,
//                   B from shared memory) and tcgen05.commit.
//       warps 4-7   epilogue: tcgen05.ld of the fp32 accumulator, SwiGLU (UP)
//                   or scaling (DOWN), stores.
//       warps 8-15  decoders: raw codes + scales -> exact bf16 (or bf16-rounded
//                   for FP8) weights, written straight into TMEM with
//                   tcgen05.st, so decoded weights never touch shared memory.
//   * K order inside every 8-element group is 0,4,1,5,2,6,3,7 in both
//     operands: one shift/multiply/mask then decodes an FP4 pair (k, k+4).
//   * Every wait is bounded; on timeout the CTA sets the device error word,
//     drains its in-flight copies and MMAs and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kThreads = 512;
constexpr int kBK = 128;            // K elements per stage
constexpr int kMaxStages = 4;
constexpr int kACol = 0;            // TMEM columns [0, 64*stages): A stages
constexpr int kAccCol = 256;        // TMEM columns [256, 256+2*BN): accumulators
constexpr int kXchStride = 17;      // padded row of the gate/up exchange buffer

template <int FMT>
struct RawFmt;
template <>
struct RawFmt<MOE_MXFP4> { static constexpr int kRowBytes = 64; };   // 128 e4m1 codes
template <>
struct RawFmt<MOE_NVFP4> { static constexpr int kRowBytes = 64; };
template <>
struct RawFmt<MOE_FP8_E4M3_K128> { static constexpr int kRowBytes = 128; };
template <>
struct RawFmt<MOE_BF16> { static constexpr int kRowBytes = 256; };

// bf16x2 multiply (exact for the power-of-two and short-significand factors used here).
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

// 8 E2M1 codes (one 32-bit word, K = 8g..8g+7) -> 4 bf16x2 words holding the
// pairs (k, k+4), k = 0..3, each equal to code value * 2^-126 (exponent field
// = E2M1 exponent bits, mantissa msb = E2M1 mantissa, so E2M1 subnormals map
// to bf16 subnormals); the caller multiplies by 2^126 * block scale.
__device__ __forceinline__ void e2m1x8_to_bf16_pattern(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t w2 = w >> 8;
    // (x & nibble pair) * (2^a + 2^b): two shifted copies with disjoint bits,
    // one puts the 3 magnitude bits at 8:6, the other the sign at 15.
    o[0] = ((w & 0x000F000Fu) * 4160u) & 0x81C081C0u;   // 2^6 + 2^12
    o[1] = ((w & 0x00F000F0u) * 260u) & 0x81C081C0u;    // 2^2 + 2^8
    o[2] = ((w2 & 0x000F000Fu) * 4160u) & 0x81C081C0u;
    o[3] = ((w2 & 0x00F000F0u) * 260u) & 0x81C081C0u;
}

// Two E4M3 bytes in bits 15:8 and 31:24 -> bf16x2 equal to value * 2^-120.
__device__ __forceinline__ uint32_t e4m3x2_hi_to_bf16_pattern(uint32_t x) {
    const uint32_t mag = (x >> 4) & 0x07F007F0u;
    return (x & 0x80008000u) | mag;
}

__device__ __forceinline__ uint32_t bf16x2_splat_bits(uint32_t b16) { return b16 | (b16 << 16); }

__device__ __forceinline__ float e4m3_to_f32(uint32_t v) {
    // value * 2^-120 as a binary32 pattern (exponent field = E4M3 exponent), then rescale exactly
    const uint32_t pat = ((v & 0x7Fu) << 20) | ((v & 0x80u) << 24);
    return __uint_as_float(pat) * 0x1p120f;
}

struct FfnSmem {
    uint64_t full[kMaxStages];
    uint64_t adec[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t accfull[2];
    uint64_t accempty[2];
    uint64_t scfull[2];
    uint64_t scempty[2];
    uint64_t mmadone;
    uint64_t xfull, xempty;   // gate/up exchange between epilogue warp pairs
    uint32_t tmem_base;
    int abort_flag;
    int total_items;
    int tile_start[kMaxExperts + 1];   // inclusive-prefix of row tiles per expert
};

struct ItemInfo {
    int e, row0, nvalid, m;
};

__device__ __forceinline__ ItemInfo decode_item(const FfnSmem &sm, const FfnParams &p, int item, int BN) {
    const int rt = item / p.m_tiles;
    ItemInfo it;
    it.m = item - rt * p.m_tiles;
    // expert with tile_start[e] <= rt < tile_start[e+1]
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.tile_start[mid] <= rt) lo = mid; else hi = mid - 1;
    }
    it.e = lo;
    const int t = rt - sm.tile_start[lo];
    const int beg = p.offsets[lo];
    const int n = p.offsets[lo + 1] - beg;
    it.row0 = beg + t * BN;
    it.nvalid = min(BN, n - t * BN);
    return it;
}

template <int FMT, int PHASE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap bmap, FfnParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr int RB = RawFmt<FMT>::kRowBytes;
    constexpr int RAWB = 128 * RB;              // raw weight bytes per stage
    constexpr int BSTAGE = BN * 256;            // activation bytes per stage (two 64-column atoms)

    // ---- shared memory carve-up (1024-aligned operand regions)
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nst = p.stages;
    uint8_t *bstage = base;
    uint8_t *rawst = bstage + nst * BSTAGE;
    uint8_t *scbuf = rawst + nst * RAWB;
    const int scb_bytes = 128 * p.s_rowbytes;   // per buffer (0 for bf16)
    float *xch = reinterpret_cast<float *>(scbuf + 2 * ((scb_bytes + 15) & ~15));
    FfnSmem &sm = *reinterpret_cast<FfnSmem *>(reinterpret_cast<uint8_t *>(xch) +
                                              (PHASE == kPhaseUp ? 64 * kXchStride * 4 : 0));

    const int warp = warp_id(), lane = lane_id();
    volatile int *abort_flag = &sm.abort_flag;

    // ---- set-up: barriers (thread 0), TMEM (warp 1), tile prefix (warp 2)
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.adec[s], 8);
            mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sm.accfull[a], 1);
            mbar_init(&sm.accempty[a], 128);
            mbar_init(&sm.scfull[a], 1);
            mbar_init(&sm.scempty[a], 8);
        }
        mbar_init(&sm.mmadone, 1);
        mbar_init(&sm.xfull, 64);
        mbar_init(&sm.xempty, 64);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&wmap);
        tma_prefetch_desc(&bmap);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        int run = 0;
        if (lane == 0) sm.tile_start[0] = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int nt = 0;
            if (e < p.E) {
                const int n = p.offsets[e + 1] - p.offsets[e];
                nt = (n + BN - 1) / BN;
            }
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
    const int KB = p.K / kBK;

    if (warp == 0) {
        // =================================================== TMA producer
        if (lane == 0) {
            int kc = 0, lt = 0;
            int issued_mask = 0;                 // stages with a load whose completion was not yet awaited here
            uint32_t issued_par[kMaxStages] = {0, 0, 0, 0};
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
                const ItemInfo it = decode_item(sm, p, item, BN);
                const int slot = p.expert_map ? p.expert_map[it.e] : it.e;
                int rowA, rowB;
                if (PHASE == kPhaseUp) { rowA = it.m * 64; rowB = p.I + it.m * 64; }
                else { rowA = it.m * 128; rowB = rowA + 64; }
                if (FMT != MOE_BF16) {
                    const int sb = lt & 1;
                    if (!mbar_wait(&sm.scempty[sb], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(&sm.scfull[sb], 128 * p.s_rowbytes);
                    const uint8_t *sbase = p.scale_base + (int64_t)slot * p.s_estride;
                    uint8_t *dst = scbuf + sb * ((scb_bytes + 15) & ~15);
                    bulk_load(dst, sbase + (int64_t)rowA * p.s_rowbytes, 64 * p.s_rowbytes, &sm.scfull[sb]);
                    bulk_load(dst + 64 * p.s_rowbytes, sbase + (int64_t)rowB * p.s_rowbytes, 64 * p.s_rowbytes,
                              &sm.scfull[sb]);
                }
                for (int kb = 0; kb < KB; ++kb, ++kc) {
                    const int s = kc % nst;
                    const uint32_t ph = (kc / nst) & 1;
                    if (!mbar_wait(&sm.empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
                    uint64_t *fb = &sm.full[s];
                    mbar_expect_tx(fb, RAWB + BSTAGE);
                    uint8_t *raw = rawst + s * RAWB;
                    if (FMT == MOE_BF16) {
                        // two 64-column boxes per 64-row half
                        tma_load_3d(raw + 0 * 8192, &wmap, fb, kb * kBK, rowA, slot);
                        tma_load_3d(raw + 1 * 8192, &wmap, fb, kb * kBK + 64, rowA, slot);
                        tma_load_3d(raw + 2 * 8192, &wmap, fb, kb * kBK, rowB, slot);
                        tma_load_3d(raw + 3 * 8192, &wmap, fb, kb * kBK + 64, rowB, slot);
                    } else {
                        const int kcoord = kb * RB;   // bytes along K
                        tma_load_3d(raw, &wmap, fb, kcoord, rowA, slot);
                        tma_load_3d(raw + RAWB / 2, &wmap, fb, kcoord, rowB, slot);
                    }
                    uint8_t *bs = bstage + s * BSTAGE;
                    tma_load_2d(bs, &bmap, fb, kb * kBK, it.row0);
                    tma_load_2d(bs + BN * 128, &bmap, fb, kb * kBK + 64, it.row0);
                    issued_mask |= 1 << s;
                    issued_par[s] = ph;
                }
            }
            // drain: never leave the CTA while a copy into its shared memory is in flight
            for (int s = 0; s < nst; ++s) {
                if (!(issued_mask & (1 << s))) continue;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.full[s], issued_par[s])) {
                    if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
                }
            }
        }
    } else if (warp == 1) {
        // =================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
            int kc = 0, lt = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
                const int a = lt & 1;
                if (!mbar_wait(&sm.accempty[a], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dcol = tmem + kAccCol + a * BN;
                for (int kb = 0; kb < KB; ++kb, ++kc) {
                    const int s = kc % nst;
                    const uint32_t ph = (kc / nst) & 1;
                    if (!mbar_wait(&sm.adec[s], ph, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&sm.full[s], ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t bsa = smem_u32(bstage + s * BSTAGE);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t atm = tmem + kACol + s * 64 + i * 8;
                        const uint32_t baddr = bsa + (i >> 2) * (BN * 128) + (i & 3) * 32;
                        mma_bf16_ts(dcol, atm, smem_desc_sw128(baddr), idesc, (kb | i) != 0);
                    }
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.accfull[a]);
            }
            // all MMAs of this CTA retire before TMEM is released
            mma_commit(&sm.mmadone);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&sm.mmadone, 0)) {
                if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // =================================================== epilogue
        const int q = warp & 3;
        const int lrow = q * 32 + lane;     // TMEM lane == M-tile row
        int lt = 0, xc = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
            const ItemInfo it = decode_item(sm, p, item, BN);
            const int a = lt & 1;
            if (!mbar_wait(&sm.accfull[a], (lt >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            float osc = 1.0f;
            if (FMT == MOE_NVFP4) osc = p.tscale[it.e] * 128.0f;   // decoded codes carry 2^-7
            const uint32_t acc = tmem + ((uint32_t)(q * 32) << 16) + kAccCol + a * BN;
            if (PHASE == kPhaseUp) {
                // rows 0-63: gate of channel c0+row; rows 64-127: up of the same channel
                const int ch = it.m * 64 + (lrow & 63);
                const int g8 = ch & ~7, j8 = ch & 7;
                const int pos = g8 + (j8 < 4 ? 2 * j8 : 2 * (j8 - 4) + 1);
                __nv_bfloat16 *hout = reinterpret_cast<__nv_bfloat16 *>(p.out);
                // up values cross from warps 6-7 to warps 4-5 through shared memory,
                // one 16-column chunk at a time, handed over with bounded mbarrier waits
                for (int c0 = 0; c0 < BN && ok; c0 += 16, ++xc) {
                    uint32_t v[16];
                    tmem_ld16(acc + c0, v);
                    tmem_wait_ld();
                    if (q >= 2) {
                        if (!mbar_wait(&sm.xempty, (xc & 1) ^ 1, abort_flag)) { ok = false; break; }
#pragma unroll
                        for (int j = 0; j < 16; ++j) xch[(lrow - 64) * kXchStride + j] = __uint_as_float(v[j]);
                        mbar_arrive(&sm.xfull);
                    } else {
                        if (!mbar_wait(&sm.xfull, xc & 1, abort_flag)) { ok = false; break; }
                        float u[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) u[j] = xch[lrow * kXchStride + j];
                        mbar_arrive(&sm.xempty);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (c0 + j < it.nvalid) {
                                const float g = __uint_as_float(v[j]) * osc;
                                const float uu = u[j] * osc;
                                const float hv = g / (1.0f + __expf(-g)) * uu;
                                hout[(int64_t)(it.row0 + c0 + j) * p.I + pos] = __float2bfloat16_rn(hv);
                            }
                        }
                    }
                }
                if (!ok) break;
            } else {
                const int ch = it.m * 128 + lrow;
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(acc + c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < it.nvalid) {
                            const float y = __uint_as_float(v[j]) * osc;
                            const int64_t o = (int64_t)(it.row0 + c0 + j) * p.H + ch;
                            if (p.out_fp32) reinterpret_cast<float *>(p.out)[o] = y;
                            else reinterpret_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(y);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.accempty[a]);
        }
    } else if (warp >= 8) {
        // =================================================== decoders
        const int dw = warp - 8;
        const int q = dw & 3;          // TMEM lane quarter (warp % 4)
        const int hf = dw >> 2;        // which 64-wide half of the K stage
        const int m = q * 32 + lane;   // M-tile row
        const int rh = m >> 6, rr = m & 63;
        int kc = 0, lt = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
            const int sb = lt & 1;
            const uint8_t *scrow = scbuf + sb * ((scb_bytes + 15) & ~15) + m * p.s_rowbytes;
            if (FMT != MOE_BF16) {
                if (!mbar_wait(&sm.scfull[sb], (lt >> 1) & 1, abort_flag)) { ok = false; break; }
            }
            for (int kb = 0; kb < KB; ++kb, ++kc) {
                const int s = kc % nst;
                const uint32_t ph = (kc / nst) & 1;
                if (!mbar_wait(&sm.full[s], ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint8_t *raw = rawst + s * RAWB;
                uint32_t o[32];
                if (FMT == MOE_MXFP4 || FMT == MOE_NVFP4) {
                    // row rr of half rh: 64 bytes, 16-byte chunks swizzled by ((rr >> 1) & 3)
                    const uint8_t *row = raw + rh * (RAWB / 2) + rr * 64;
                    bool big_any = false;
                    uint32_t f[4];   // bf16x2 factor per 16-element quarter of this thread's 64 elements
                    if (FMT == MOE_MXFP4) {
                        const uint32_t sc2 = *reinterpret_cast<const uint16_t *>(scrow + kb * 4 + hf * 2);
                        bool big = false;
#pragma unroll
                        for (int b = 0; b < 2; ++b) {
                            const uint32_t s8 = (sc2 >> (8 * b)) & 0xFF;
                            big |= s8 > 128;
                            // 2^126 * 2^(s-127) = 2^(s-1): bf16 exponent field s + 126
                            const uint32_t fb = (s8 <= 128 ? (s8 + 126) : 254u) << 7;
                            f[2 * b] = f[2 * b + 1] = bf16x2_splat_bits(fb);
                        }
                        big_any = __any_sync(0xffffffffu, big);
                        if (big_any) {
                            // rare: scales above 2^1 need a second exact multiply
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
                                const uint4 v = *reinterpret_cast<const uint4 *>(
                                    row + (((2 * hf + c) ^ ((rr >> 1) & 3)) << 4));
                                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int g = 0; g < 4; ++g) {
                                    uint32_t pr[4];
                                    e2m1x8_to_bf16_pattern(wv[g], pr);
                                    const int b = (c * 4 + g) >> 2;
                                    const uint32_t s8 = (sc2 >> (8 * b)) & 0xFF;
                                    const uint32_t f2 = bf16x2_splat_bits((s8 > 128 ? (s8 - 128 + 127) : 127u) << 7);
#pragma unroll
                                    for (int j = 0; j < 4; ++j) o[(c * 4 + g) * 4 + j] = bmul2(bmul2(pr[j], f[2 * b]), f2);
                                }
                            }
                        }
                    } else {
                        const uint32_t sc4 = *reinterpret_cast<const uint32_t *>(scrow + kb * 8 + hf * 4);
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            // 2^126 * e4m3 * 2^-7 (the 2^7 is restored in the epilogue with the tensor scale)
                            const float sv = e4m3_to_f32((sc4 >> (8 * b)) & 0xFF) * 0x1p119f;
                            const __nv_bfloat16 bs = __float2bfloat16_rn(sv);
                            f[b] = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
                        }
                    }
                    if (!(FMT == MOE_MXFP4 && big_any)) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(row + (((2 * hf + c) ^ ((rr >> 1) & 3)) << 4));
                        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint32_t pr[4];
                            e2m1x8_to_bf16_pattern(wv[g], pr);
                            const int gi = c * 4 + g;                      // 8-group index 0..7
                            const uint32_t fac = (FMT == MOE_MXFP4) ? f[(gi >> 2) * 2] : f[gi >> 1];
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[gi * 4 + j] = bmul2(pr[j], fac);
                        }
                    }
                    }
                } else if (FMT == MOE_FP8_E4M3_K128) {
                    const uint8_t *row = raw + rh * (RAWB / 2) + rr * 128;
                    const float sc = reinterpret_cast<const float *>(scrow)[kb];
                    // 2^120 * scale, rounded to bf16 (the one inexact step of this format)
                    const __nv_bfloat16 bs = __float2bfloat16_rn(sc * 0x1p120f);
                    const uint32_t fac = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(row + (((4 * hf + c) ^ (rr & 7)) << 4));
                        // v.x,v.y = K 16c..16c+7 ; v.z,v.w = 16c+8..16c+15
                        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int g = 0; g < 2; ++g) {
                            const uint32_t lo = wv[2 * g], hi = wv[2 * g + 1];   // K 0..3 and 4..7 of the group
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                // byte j of lo -> bits 15:8, byte j of hi -> bits 31:24
                                const uint32_t sel = ((4u + j) << 12) | (8u << 8) | ((uint32_t)j << 4) | 8u;
                                const uint32_t x = __byte_perm(lo, hi, sel) & 0xFF00FF00u;
                                o[(c * 2 + g) * 4 + j] = bmul2(e4m3x2_hi_to_bf16_pattern(x), fac);
                            }
                        }
                    }
                } else {
                    // bf16: box hf holds K 64*hf..64*hf+63 of this half's rows, 128-byte swizzle
                    const uint8_t *row = raw + (rh * 2 + hf) * 8192 + rr * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(row + ((c ^ (rr & 7)) << 4));
                        const uint4 iv = interleave8(v);
                        o[c * 4 + 0] = iv.x;
                        o[c * 4 + 1] = iv.y;
                        o[c * 4 + 2] = iv.z;
                        o[c * 4 + 3] = iv.w;
                    }
                }
                tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + kACol + s * 64 + hf * 32, o);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.adec[s]);
            }
            if (!ok) break;
            if (FMT != MOE_BF16) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.scempty[sb]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ dequantise

// One thread per 8-element group of one row: the same decode as the GEMM's
// decoder warps, written back in natural K order as bf16. NVFP4 applies the
// per-tensor scale in fp32 before the final rounding.
template <int FMT>
__global__ void dequant_kernel(const uint8_t *__restrict__ w, const uint8_t *__restrict__ scale, float tscale,
                               int rows, int K, __nv_bfloat16 *__restrict__ out) {
    const int64_t gidx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int groups = K / 8;
    if (gidx >= (int64_t)rows * groups) return;
    const int r = (int)(gidx / groups), g = (int)(gidx % groups);
    const int k0 = g * 8;
    uint32_t o[4];
    if (FMT == MOE_MXFP4 || FMT == MOE_NVFP4) {
        const uint32_t wv = *reinterpret_cast<const uint32_t *>(w + (int64_t)r * (K / 2) + k0 / 2);
        uint32_t pr[4];
        e2m1x8_to_bf16_pattern(wv, pr);
        if (FMT == MOE_MXFP4) {
            const uint32_t s8 = scale[(int64_t)r * (K / 32) + k0 / 32];
            const uint32_t f = bf16x2_splat_bits((s8 <= 128 ? s8 + 126 : 254u) << 7);
            const uint32_t f2 = bf16x2_splat_bits((s8 > 128 ? s8 - 128 + 127 : 127u) << 7);
            for (int j = 0; j < 4; ++j) o[j] = bmul2(bmul2(pr[j], f), f2);
        } else {
            const float sv = e4m3_to_f32(scale[(int64_t)r * (K / 16) + k0 / 16]) * 0x1p119f;
            const __nv_bfloat16 bs = __float2bfloat16_rn(sv);
            const uint32_t f = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
            for (int j = 0; j < 4; ++j) {
                const uint32_t d = bmul2(pr[j], f);   // value * 2^-7
                const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&d));
                const __nv_bfloat162 b = __floats2bfloat162_rn(v.x * 128.0f * tscale, v.y * 128.0f * tscale);
                o[j] = *reinterpret_cast<const uint32_t *>(&b);
            }
        }
    } else if (FMT == MOE_FP8_E4M3_K128) {
        const uint32_t lo = *reinterpret_cast<const uint32_t *>(w + (int64_t)r * K + k0);
        const uint32_t hi = *reinterpret_cast<const uint32_t *>(w + (int64_t)r * K + k0 + 4);
        const float sc = reinterpret_cast<const float *>(scale)[(int64_t)r * (K / 128) + k0 / 128];
        const __nv_bfloat16 bs = __float2bfloat16_rn(sc * 0x1p120f);
        const uint32_t fac = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
        for (int j = 0; j < 4; ++j) {
            const uint32_t sel = ((4u + j) << 12) | (8u << 8) | ((uint32_t)j << 4) | 8u;
            const uint32_t x = __byte_perm(lo, hi, sel) & 0xFF00FF00u;
            o[j] = bmul2(e4m3x2_hi_to_bf16_pattern(x), fac);
        }
    } else {
        const uint4 v = *reinterpret_cast<const uint4 *>(w + ((int64_t)r * K + k0) * 2);
        const uint4 iv = interleave8(v);
        o[0] = iv.x; o[1] = iv.y; o[2] = iv.z; o[3] = iv.w;
    }
    // o[j] holds (k0 + j, k0 + j + 4): write back in natural order
    uint16_t *dst = reinterpret_cast<uint16_t *>(out + (int64_t)r * K + k0);
    for (int j = 0; j < 4; ++j) {
        dst[j] = (uint16_t)(o[j] & 0xFFFF);
        dst[j + 4] = (uint16_t)(o[j] >> 16);
    }
}

moe_status launch_dequant(int fmt, const void *w, const void *scale, float tscale, int rows, int K, void *out,
                          cudaStream_t st) {
    const int64_t n = (int64_t)rows * (K / 8);
    if (n == 0) return MOE_OK;
    const int blocks = (int)((n + 255) / 256);
    const uint8_t *wp = reinterpret_cast<const uint8_t *>(w);
    const uint8_t *sp = reinterpret_cast<const uint8_t *>(scale);
    __nv_bfloat16 *op = reinterpret_cast<__nv_bfloat16 *>(out);
    switch (fmt) {
        case MOE_BF16: dequant_kernel<MOE_BF16><<<blocks, 256, 0, st>>>(wp, sp, tscale, rows, K, op); break;
        case MOE_FP8_E4M3_K128:
            dequant_kernel<MOE_FP8_E4M3_K128><<<blocks, 256, 0, st>>>(wp, sp, tscale, rows, K, op);
            break;
        case MOE_MXFP4: dequant_kernel<MOE_MXFP4><<<blocks, 256, 0, st>>>(wp, sp, tscale, rows, K, op); break;
        default: dequant_kernel<MOE_NVFP4><<<blocks, 256, 0, st>>>(wp, sp, tscale, rows, K, op); break;
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "dequant launch");
}

// ------------------------------------------------------------------ host side

static size_t ffn_smem_bytes(int fmt, int phase, int BN, int stages, int s_rowbytes) {
    const int rb = fmt == MOE_BF16 ? 256 : fmt == MOE_FP8_E4M3_K128 ? 128 : 64;
    size_t b = 1024;                                     // alignment slack
    b += (size_t)stages * BN * 256;
    b += (size_t)stages * 128 * rb;
    b += 2 * (size_t)((128 * s_rowbytes + 15) & ~15);
    if (phase == kPhaseUp) b += 64 * kXchStride * 4;
    b += sizeof(FfnSmem);
    return b;
}

template <int FMT, int PHASE, int BN>
static cudaError_t launch_one(const CUtensorMap &wmap, const CUtensorMap &bmap, const FfnParams &p, int grid,
                              size_t smem, cudaStream_t st) {
    auto kfn = ffn_tc_kernel<FMT, PHASE, BN>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, kThreads, smem, st>>>(wmap, bmap, p);
    return cudaGetLastError();
}

template <int FMT, int PHASE>
static cudaError_t launch_bn(int BN, const CUtensorMap &wmap, const CUtensorMap &bmap, const FfnParams &p, int grid,
                             size_t smem, cudaStream_t st) {
    switch (BN) {
        case 16: return launch_one<FMT, PHASE, 16>(wmap, bmap, p, grid, smem, st);
        case 32: return launch_one<FMT, PHASE, 32>(wmap, bmap, p, grid, smem, st);
        case 64: return launch_one<FMT, PHASE, 64>(wmap, bmap, p, grid, smem, st);
        default: return launch_one<FMT, PHASE, 128>(wmap, bmap, p, grid, smem, st);
    }
}

template <int PHASE>
static cudaError_t launch_fmt(int fmt, int BN, const CUtensorMap &wmap, const CUtensorMap &bmap, const FfnParams &p,
                              int grid, size_t smem, cudaStream_t st) {
    switch (fmt) {
        case MOE_BF16: return launch_bn<MOE_BF16, PHASE>(BN, wmap, bmap, p, grid, smem, st);
        case MOE_FP8_E4M3_K128: return launch_bn<MOE_FP8_E4M3_K128, PHASE>(BN, wmap, bmap, p, grid, smem, st);
        case MOE_MXFP4: return launch_bn<MOE_MXFP4, PHASE>(BN, wmap, bmap, p, grid, smem, st);
        default: return launch_bn<MOE_NVFP4, PHASE>(BN, wmap, bmap, p, grid, smem, st);
    }
}

int choose_bn(int n_rows, int E) {
    const int avg = (n_rows + E - 1) / (E > 0 ? E : 1);
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    return 128;
}

int scale_rowbytes(int fmt, int K) {
    switch (fmt) {
        case MOE_MXFP4: return K / 32;
        case MOE_NVFP4: return K / 16;
        case MOE_FP8_E4M3_K128: return (K / 128) * 4;
        default: return 0;
    }
}

// Launch one phase. The tensor maps are built by the caller (api.cu).
moe_status launch_ffn_phase(int phase, int fmt, int BN, const CUtensorMap &wmap, const CUtensorMap &bmap,
                            FfnParams p, int num_sms, cudaStream_t st) {
    int stages = kMaxStages;
    size_t smem = 0;
    for (; stages >= 2; --stages) {
        smem = ffn_smem_bytes(fmt, phase, BN, stages, p.s_rowbytes);
        if (smem <= 227 * 1024) break;
    }
    if (stages < 2) return set_error(MOE_ERR_UNSUPPORTED, "FFN tile does not fit in shared memory");
    // The CTA allocates all 512 TMEM columns: ask for enough shared memory that a
    // second CTA can never be co-resident on the SM (it would only block in alloc).
    if (smem < 120 * 1024) smem = 120 * 1024;
    p.stages = stages;
    // upper bound of work items; the kernel reads the exact count from the offsets
    const int64_t tiles_ub = (int64_t)p.n_rows / BN + p.E;
    const int64_t items_ub = tiles_ub * p.m_tiles;
    const int grid = (int)(items_ub < num_sms ? (items_ub > 0 ? items_ub : 1) : num_sms);
    cudaError_t e = phase == kPhaseUp ? launch_fmt<kPhaseUp>(fmt, BN, wmap, bmap, p, grid, smem, st)
                                      : launch_fmt<kPhaseDown>(fmt, BN, wmap, bmap, p, grid, smem, st);
    if (e != cudaSuccess) return set_cuda_error(e, "ffn kernel launch");
    return MOE_OK;
}

}  // namespace moe
