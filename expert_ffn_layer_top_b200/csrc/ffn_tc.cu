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
//   * K stage = 128 elements; stages are handled in groups of kG = 2 (16 MMAs).
//   * Warp roles (768 threads, one CTA per SM, persistent over work items):
//       warp 0      code producer: per stage one bulk copy of the prepacked
//                   weight blob (or TMA boxes + a per-tile scale copy for
//                   row-major weights) into a deep ring whose slots are freed
//                   as soon as the decoders have read them.
//       warp 2      activation producer: per group the TMA boxes of the
//                   activation tiles (128-byte swizzle), freed by the group's
//                   MMA completion.
//       warp 1      owns TMEM; one lane issues tcgen05.mma (A from TMEM,
//                   B from shared memory).
//       warps 4-7   epilogue: tcgen05.ld of the fp32 accumulator, SwiGLU (UP)
//                   or scaling (DOWN), stores.
//       warps 8-23  decoders: codes + scales -> exact bf16 (bf16-rounded for
//                   FP8) weights, written straight into TMEM with tcgen05.st,
//                   so decoded weights never touch shared memory.
//   * A tcgen05.mma of this shape costs ~52 cycles whatever N <= 64, and each
//     tcgen05.commit or wait-plus-fence in the issuing thread stalls the
//     tensor pipe for ~100+ cycles, so the issuing thread synchronises once
//     per group: it waits for the decoders of the group's last stage, issues
//     16 MMAs, and commits once to the group's barrier, which then frees both
//     the group's activation tiles and its TMEM slots.
//   * K order inside every 8-element group is 0,4,1,5,2,6,3,7 in both
//     operands: one shift/multiply/mask then decodes an FP4 pair (k, k+4).
//   * Every wait is bounded; on timeout the CTA sets the device error word,
//     drains its in-flight copies and MMAs and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kThreads = 768;
constexpr int kDecWarps = 16;       // warps 8..23
constexpr int kBK = 128;            // K elements per stage
constexpr int kG = 2;               // stages per MMA group (one commit, one wait)
constexpr int kMaxStages = 16;      // code ring (stages)
constexpr int kMaxBGroups = 8;      // activation ring (groups of kG stages)
constexpr int kMaxAStages = 6;      // TMEM ring of decoded weight tiles (64 columns each, multiple of kG)
constexpr int kXchStride = 17;      // padded row of the gate/up exchange buffer

// Per weight row and K stage (128 elements): code bytes and scale bytes.
template <int FMT>
struct RawFmt;
template <>
struct RawFmt<MOE_MXFP4> { static constexpr int kRowBytes = 64, kScaleBytes = 4; };   // 4 E8M0 (block 32)
template <>
struct RawFmt<MOE_NVFP4> { static constexpr int kRowBytes = 64, kScaleBytes = 8; };   // 8 E4M3 (block 16)
template <>
struct RawFmt<MOE_FP8_E4M3_K128> { static constexpr int kRowBytes = 128, kScaleBytes = 4; };   // 1 fp32
template <>
struct RawFmt<MOE_BF16> { static constexpr int kRowBytes = 256, kScaleBytes = 0; };

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

// bf16x2 factor 2^126 * 2^(s-127) for an E8M0 scale s <= 128; for s > 128 the
// factor saturates at 2^127 and a second factor 2^(s-128) completes it.
__device__ __forceinline__ uint32_t mx_factor(uint32_t s8) { return bf16x2_splat_bits((s8 <= 128 ? s8 + 126 : 254u) << 7); }
__device__ __forceinline__ uint32_t mx_factor2(uint32_t s8) { return bf16x2_splat_bits((s8 > 128 ? s8 - 1 : 127u) << 7); }

struct FfnSmem {
    uint64_t rfull[kMaxStages];                // code stage landed (producer expect_tx + copies)
    uint64_t rempty[kMaxStages];               // code stage read by all decoder warps
    uint64_t bfull[kMaxBGroups];               // activation tiles of a group landed
    uint64_t gdone[kMaxBGroups];               // group's MMAs complete (frees its activation tiles and TMEM slots)
    uint64_t adec[kMaxAStages];                // stage decoded into TMEM (one arrive per decoder warp)
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

// TILED: the weights were prepacked by moe_prepack into one contiguous blob per
// (M tile, K stage) - 128 rows of codes, 16-byte chunk-major, followed by the
// rows' scales for that stage - and each stage arrives with one bulk copy.
// Prepacked NVFP4 has the block-scaled path's blobs instead (one per 256-wide
// stage: 128-byte rows of codes in the 128-byte swizzle, then four scale
// atoms); a ring slot holds one such blob and serves two 128-wide stages.
// Otherwise the codes come from the row-major tensor through a 3D TMA box and
// the scales through one bulk copy per tile.
template <int FMT, int PHASE, int BN, bool TILED>
__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap bmap, FfnParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr int RB = RawFmt<FMT>::kRowBytes;
    constexpr int SBY = RawFmt<FMT>::kScaleBytes;
    constexpr int RAWB = 128 * RB;                          // code bytes per stage
    constexpr bool NVB = TILED && FMT == MOE_NVFP4;         // block-scaled blob layout
    constexpr int KPS = NVB ? 2 : 1;                        // 128-wide stages per ring slot
    constexpr int SB = KPS * (RAWB + (TILED ? 128 * SBY : 0));   // smem bytes per slot (codes [+ scales])
    constexpr int BSTAGE = BN * 256;            // activation bytes per stage (two 64-column atoms)
    constexpr int BGROUP = kG * BSTAGE;         // activation bytes per group

    // ---- shared memory carve-up (1024-aligned operand regions)
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nr = p.stages;                  // code ring depth (stages)
    const int nbg = p.bgroups;                // activation ring depth (groups)
    const int na = p.astages;                 // TMEM A stages, multiple of kG, na / kG <= nbg
    uint8_t *bstage = base;
    uint8_t *rawst = bstage + nbg * BGROUP;
    uint8_t *scbuf = rawst + nr * SB;
    const int scb_bytes = TILED ? 0 : 128 * p.s_rowbytes;   // per tile buffer (standard layout only)
    float *xch = reinterpret_cast<float *>(scbuf + 2 * ((scb_bytes + 15) & ~15));
    FfnSmem &sm = *reinterpret_cast<FfnSmem *>(reinterpret_cast<uint8_t *>(xch) +
                                              (PHASE == kPhaseUp ? 64 * kXchStride * 4 : 0));

    const int warp = warp_id(), lane = lane_id();
    volatile int *abort_flag = &sm.abort_flag;
    pdl_wait();   // offsets and activations come from the kernels before this one
    if (threadIdx.x == 0) pdl_release();

    // ---- set-up: barriers (thread 0), TMEM (warp 1), tile prefix (warp 3)
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&sm.rfull[s], 1);
            mbar_init(&sm.rempty[s], kDecWarps);
        }
        for (int g = 0; g < kMaxBGroups; ++g) {
            mbar_init(&sm.bfull[g], 1);
            mbar_init(&sm.gdone[g], 1);
        }
        for (int s = 0; s < kMaxAStages; ++s) mbar_init(&sm.adec[s], kDecWarps);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sm.accfull[a], 1);
            mbar_init(&sm.accempty[a], 128);
            mbar_init(&sm.scfull[a], 1);
            mbar_init(&sm.scempty[a], kDecWarps);
        }
        mbar_init(&sm.mmadone, 1);
        mbar_init(&sm.xfull, 64);
        mbar_init(&sm.xempty, 64);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0 && !TILED) tma_prefetch_desc(&wmap);
    if (warp == 2 && lane == 0) tma_prefetch_desc(&bmap);
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 3) {
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
    const uint32_t acc_col = (uint32_t)na * 64;   // accumulators follow the A ring
    const int total = sm.total_items;
    const int KB = p.K / kBK;                     // multiple of kG

    if (warp == 0) {
        // =================================================== code producer
        // Codes (and, tiled, their scales) stream through their own ring; a slot
        // is refilled as soon as the 16 decoder warps have read it.
        if (lane == 0) {
            int kc = 0, lt = 0, s = 0;           // kc: stages issued so far
            uint32_t ph = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
                const ItemInfo it = decode_item(sm, p, item, BN);
                const int slot = p.expert_map ? p.expert_map[it.e] : it.e;
                int rowA, rowB;
                if (PHASE == kPhaseUp) { rowA = it.m * 64; rowB = p.I + it.m * 64; }
                else { rowA = it.m * 128; rowB = rowA + 64; }
                if (FMT != MOE_BF16 && !TILED) {
                    const int sb = lt & 1;
                    if (!mbar_wait(&sm.scempty[sb], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(&sm.scfull[sb], 128 * p.s_rowbytes);
                    const uint8_t *sbase = p.scale_base + (int64_t)slot * p.s_estride;
                    uint8_t *dst = scbuf + sb * ((scb_bytes + 15) & ~15);
                    bulk_load(dst, sbase + (int64_t)rowA * p.s_rowbytes, 64 * p.s_rowbytes, &sm.scfull[sb]);
                    bulk_load(dst + 64 * p.s_rowbytes, sbase + (int64_t)rowB * p.s_rowbytes, 64 * p.s_rowbytes,
                              &sm.scfull[sb]);
                }
                for (int kb = 0; kb < KB; kb += KPS) {
                    if (!mbar_wait(&sm.rempty[s], ph ^ 1, abort_flag)) { ok = false; break; }
                    uint64_t *fb = &sm.rfull[s];
                    mbar_expect_tx(fb, SB);
                    uint8_t *raw = rawst + s * SB;
                    if (TILED) {
                        const uint8_t *src = p.wbase + (int64_t)slot * p.w_estride +
                                             ((int64_t)it.m * (KB / KPS) + kb / KPS) * SB;
                        bulk_load(raw, src, SB, fb);
                    } else if (FMT == MOE_BF16) {
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
                    ++kc;
                    if (++s == nr) { s = 0; ph ^= 1; }
                }
            }
            // drain: never leave the CTA while a copy into its shared memory is in
            // flight - wait for the completion of the last min(kc, nr) stages issued
            for (int j = kc - 1; j >= 0 && j >= kc - nr; --j) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.rfull[j % nr], (j / nr) & 1)) {
                    if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
                }
            }
        }
    } else if (warp == 2) {
        // =================================================== activation producer
        // One barrier per group of kG stages; a group's tiles are refilled once
        // the group's MMAs have completed.
        if (lane == 0) {
            int gc = 0, bg = 0;                  // gc: groups issued so far
            uint32_t bph = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const ItemInfo it = decode_item(sm, p, item, BN);
                for (int kb = 0; kb < KB; kb += kG) {
                    if (!mbar_wait(&sm.gdone[bg], bph ^ 1, abort_flag)) { ok = false; break; }
                    uint64_t *fb = &sm.bfull[bg];
                    mbar_expect_tx(fb, BGROUP);
                    uint8_t *bs = bstage + bg * BGROUP;
#pragma unroll
                    for (int g = 0; g < kG; ++g) {
                        tma_load_2d(bs + g * BSTAGE, &bmap, fb, (kb + g) * kBK, it.row0);
                        tma_load_2d(bs + g * BSTAGE + BN * 128, &bmap, fb, (kb + g) * kBK + 64, it.row0);
                    }
                    ++gc;
                    if (++bg == nbg) { bg = 0; bph ^= 1; }
                }
            }
            for (int j = gc - 1; j >= 0 && j >= gc - nbg; --j) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.bfull[j % nbg], (j / nbg) & 1)) {
                    if (globaltimer() - t0 > kWaitLimitNs) { flag_error(1); break; }
                }
            }
        }
    } else if (warp == 1) {
        // =================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
            const uint32_t desc_hi = (uint32_t)(smem_desc_sw128(0) >> 32);
            const uint32_t desc_lo0 = (uint32_t)smem_desc_sw128(smem_u32(bstage));
            int bg = 0, sa = 0, lt = 0;
            uint32_t bph = 0, pha = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
                const int a = lt & 1;
                if (!mbar_wait(&sm.accempty[a], ((lt >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dcol = tmem + acc_col + a * BN;
                for (int kb = 0; kb < KB; kb += kG) {
                    // decoders arrive stage by stage, so the group's last stage implies the rest
                    if (!mbar_wait(&sm.adec[sa + kG - 1], pha, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&sm.bfull[bg], bph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int g = 0; g < kG; ++g) {
                        const uint32_t lo = desc_lo0 + ((uint32_t)(bg * BGROUP + g * BSTAGE) >> 4);
                        const uint32_t atm = tmem + (sa + g) * 64;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            mma_bf16_ts_lohi(dcol, atm + i * 8,
                                             lo + (((i >> 2) * (BN * 128) + (i & 3) * 32) >> 4), desc_hi, idesc,
                                             (kb | g | i) != 0);
                    }
                    mma_commit(&sm.gdone[bg]);
                    if (++bg == nbg) { bg = 0; bph ^= 1; }
                    sa += kG;
                    if (sa == na) { sa = 0; pha ^= 1; }
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
            const uint32_t acc = tmem + ((uint32_t)(q * 32) << 16) + acc_col + a * BN;
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
        // 16 warps: warp (8 + dw) owns TMEM lane quarter q = dw % 4 (rows 32q..32q+31)
        // and the 32 K elements [32*sub, 32*sub + 32) of every stage, sub = dw / 4.
        const int dw = warp - 8;
        const int q = dw & 3;
        const int sub = dw >> 2;
        const int m = q * 32 + lane;   // M-tile row
        const int rh = m >> 6, rr = m & 63;
        int lt = 0, s = 0, sa = 0, gstart = 0;   // gstart: groups started
        uint32_t ph = 0;
        int lag_slot = 0;                        // group (gstart - na/kG) whose MMAs must have completed
        uint32_t lag_ph = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++lt) {
            const int sb = lt & 1;
            const uint8_t *scrow = scbuf + sb * ((scb_bytes + 15) & ~15) + m * p.s_rowbytes;
            if (FMT != MOE_BF16 && !TILED) {
                if (!mbar_wait(&sm.scfull[sb], (lt >> 1) & 1, abort_flag)) { ok = false; break; }
            }
            for (int kb = 0; kb < KB; ++kb) {
                if ((sa & (kG - 1)) == 0) {
                    // new group: its TMEM slots were last used by the group na/kG groups back
                    if (gstart >= na / kG) {
                        if (!mbar_wait(&sm.gdone[lag_slot], lag_ph, abort_flag)) { ok = false; break; }
                        if (++lag_slot == nbg) { lag_slot = 0; lag_ph ^= 1; }
                    }
                    ++gstart;
                }
                if (kb % KPS == 0 && !mbar_wait(&sm.rfull[s], ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint8_t *raw = rawst + s * SB;
                const int hk = kb & (KPS - 1);   // NVB: 128-wide half of the blob
                // 16-byte chunk c of this thread's row, and its scales for this stage
                auto chunk = [&](int c) -> uint4 {
                    const uint8_t *a;
                    if (NVB) a = raw + m * 128 + (((hk * 4 + c) ^ (m & 7)) << 4);
                    else if (TILED) a = raw + ((c * 128 + m) << 4);
                    else if (FMT == MOE_MXFP4 || FMT == MOE_NVFP4) a = raw + rh * (RAWB / 2) + rr * 64 + ((c ^ ((rr >> 1) & 3)) << 4);
                    else if (FMT == MOE_FP8_E4M3_K128) a = raw + rh * (RAWB / 2) + rr * 128 + ((c ^ (rr & 7)) << 4);
                    else a = raw + (rh * 2 + (c >> 3)) * 8192 + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
                    return *reinterpret_cast<const uint4 *>(a);
                };
                const uint8_t *scs = TILED ? raw + RAWB + m * SBY : scrow + kb * SBY;
                uint32_t o[16];
                if (FMT == MOE_MXFP4 || FMT == MOE_NVFP4) {
                    const uint4 v = chunk(sub);                 // 32 codes = 4 groups of 8
                    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
                    if (FMT == MOE_MXFP4) {
                        const uint32_t s8 = scs[sub];               // one E8M0 block of 32
                        const uint32_t f = mx_factor(s8);
                        const bool big = __any_sync(0xffffffffu, s8 > 128);
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint32_t pr[4];
                            e2m1x8_to_bf16_pattern(wv[g], pr);
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[g * 4 + j] = bmul2(pr[j], f);
                        }
                        if (big) {   // rare: scales above 2^1 need a second exact multiply
                            const uint32_t f2 = mx_factor2(s8);
#pragma unroll
                            for (int j = 0; j < 16; ++j) o[j] = bmul2(o[j], f2);
                        }
                    } else {
                        // two blocks of 16; NVB: blocks 2 sub, 2 sub + 1 of half hk sit in atom
                        // 2 hk + sub / 2 at scale positions 2 (sub % 2), + 1 of row m
                        const uint8_t *s2 = NVB ? raw + 128 * 128 + (2 * hk + (sub >> 1)) * 512 + (m & 31) * 16 +
                                                      (m >> 5) * 4 + 2 * (sub & 1)
                                                : scs + 2 * sub;
                        const uint32_t sc2 = *reinterpret_cast<const uint16_t *>(s2);
                        uint32_t f[2];
#pragma unroll
                        for (int b = 0; b < 2; ++b) {
                            // 2^126 * e4m3 * 2^-7 (the 2^7 is restored in the epilogue with the tensor scale)
                            const float sv = e4m3_to_f32((sc2 >> (8 * b)) & 0xFF) * 0x1p119f;
                            const __nv_bfloat16 bs = __float2bfloat16_rn(sv);
                            f[b] = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
                        }
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint32_t pr[4];
                            e2m1x8_to_bf16_pattern(wv[g], pr);
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[g * 4 + j] = bmul2(pr[j], f[g >> 1]);
                        }
                    }
                } else if (FMT == MOE_FP8_E4M3_K128) {
                    const float sc = *reinterpret_cast<const float *>(scs);
                    // 2^120 * scale, rounded to bf16 (the one inexact step of this format)
                    const __nv_bfloat16 bs = __float2bfloat16_rn(sc * 0x1p120f);
                    const uint32_t fac = bf16x2_splat_bits(*reinterpret_cast<const uint16_t *>(&bs));
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint4 v = chunk(2 * sub + c);
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
                    // bf16: K 32*sub..32*sub+31 are chunks 4*sub..4*sub+3
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 iv = interleave8(chunk(4 * sub + c));
                        o[c * 4 + 0] = iv.x;
                        o[c * 4 + 1] = iv.y;
                        o[c * 4 + 2] = iv.z;
                        o[c * 4 + 3] = iv.w;
                    }
                }
                tmem_st16(tmem + ((uint32_t)(q * 32) << 16) + sa * 64 + sub * 16, o);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sm.adec[sa]);
                    if (hk == KPS - 1) mbar_arrive(&sm.rempty[s]);   // codes read: the slot can be refilled
                }
                if (hk == KPS - 1 && ++s == nr) { s = 0; ph ^= 1; }
                if (++sa == na) sa = 0;
            }
            if (!ok) break;
            if (FMT != MOE_BF16 && !TILED) {
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
    count_launch();
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "dequant launch");
}

// ------------------------------------------------------------------ host side

int stage_scale_bytes(int fmt) {
    return fmt == MOE_MXFP4 ? 4 : fmt == MOE_NVFP4 ? 8 : fmt == MOE_FP8_E4M3_K128 ? 4 : 0;
}
int stage_code_bytes(int fmt) { return fmt == MOE_BF16 ? 256 : fmt == MOE_FP8_E4M3_K128 ? 128 : 64; }

static size_t ffn_smem_bytes(int fmt, int phase, int BN, int stages, int bgroups, int s_rowbytes, bool tiled) {
    const int rb = stage_code_bytes(fmt);
    size_t b = 1024;                                     // alignment slack
    b += (size_t)bgroups * kG * BN * 256;
    const int kps = tiled && fmt == MOE_NVFP4 ? 2 : 1;   // prepacked NVFP4: one 256-wide blob per slot
    b += (size_t)stages * kps * 128 * (rb + (tiled ? stage_scale_bytes(fmt) : 0));
    if (!tiled) b += 2 * (size_t)((128 * s_rowbytes + 15) & ~15);
    if (phase == kPhaseUp) b += 64 * kXchStride * 4;
    b += sizeof(FfnSmem);
    return b;
}

template <int FMT, int PHASE, int BN>
static cudaError_t launch_one(const CUtensorMap &wmap, const CUtensorMap &bmap, const FfnParams &p, int grid,
                              size_t smem, cudaStream_t st) {
    auto kfn = p.tiled ? ffn_tc_kernel<FMT, PHASE, BN, true> : ffn_tc_kernel<FMT, PHASE, BN, false>;
    cudaError_t e = p.tiled ? ensure_max_smem<ffn_tc_kernel<FMT, PHASE, BN, true>>((int)smem)
                            : ensure_max_smem<ffn_tc_kernel<FMT, PHASE, BN, false>>((int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kfn, dim3(grid), dim3(kThreads), smem, st, wmap, bmap, p);
    return e == cudaSuccess ? cudaGetLastError() : e;
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
    if (p.K % (kBK * kG)) return set_error(MOE_ERR_UNSUPPORTED, "K=%d is not a multiple of %d", p.K, kBK * kG);
    // TMEM: A ring of 64-column stages, then two accumulators of BN columns
    int na = (512 - 2 * BN) / 64;
    if (na > kMaxAStages) na = kMaxAStages;
    na -= na % kG;
    // Activation ring: one group more than the TMEM ring holds. The decoders
    // wait on the group barrier of the group na/kG back; with at least that many
    // activation groups no barrier can complete twice before that wait, so the
    // parity check cannot alias.
    int bgroups = na / kG + 1;
    if (bgroups > kMaxBGroups) bgroups = kMaxBGroups;
    int stages = kMaxStages;
    size_t smem = 0;
    for (;;) {
        for (stages = kMaxStages; stages >= 2; --stages) {
            smem = ffn_smem_bytes(fmt, phase, BN, stages, bgroups, p.s_rowbytes, p.tiled != 0);
            if (smem <= 227 * 1024) break;
        }
        if (stages >= 2) break;
        if (bgroups == 1) return set_error(MOE_ERR_UNSUPPORTED, "FFN tile does not fit in shared memory");
        --bgroups;
        if (na > bgroups * kG) na = bgroups * kG;
    }
    // The CTA allocates all 512 TMEM columns: ask for enough shared memory that a
    // second CTA can never be co-resident on the SM (it would only block in alloc).
    if (smem < 120 * 1024) smem = 120 * 1024;
    p.stages = stages;
    p.bgroups = bgroups;
    p.astages = na;
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
