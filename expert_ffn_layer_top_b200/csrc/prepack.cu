// Prepacking of expert weights into the tiled layout read by the grouped FFN.
//
// For every expert, M tile and 128-wide K stage the tiled layout holds one
// contiguous blob with the 128 weight rows of the tile (gate/up: 64 gate rows
// then the 64 matching up rows; down: 128 consecutive rows):
//   BF16, FP8: the codes as 16-byte chunks in chunk-major order (chunk c of
//     row r at (c*128 + r)*16), then each row's scales for that stage. The
//     decoding FFN moves a stage with one bulk copy and its decoder threads
//     read consecutive chunks without bank conflicts.
//   MXFP4, NVFP4 (stages 256 wide): one blob per (M tile, stage), in that
//     order. First the packed codes, 128 bytes per row in natural K order,
//     with the 16-byte chunk c of row r stored at r*128 + (c ^ (r % 8))*16:
//     the 128-byte swizzle the block-scaled MMA reads from shared memory, so
//     one bulk copy lands the operand ready to use. Then the 512-byte scale
//     atoms: the scale of row r and scale block j of the atom's K range at
//     byte (r % 32)*16 + (r / 32)*4 + j, the arrangement tcgen05.cp moves into
//     TMEM. MXFP4: two atoms (E8M0 per 32, one atom per 128-wide half), a
//     17 KiB blob; NVFP4: four atoms (E4M3 per 16, one per 64-wide quarter),
//     an 18 KiB blob.
// Values are untouched: this is a byte permutation.
#include "common.cuh"
#include "internal.h"

namespace moe {

// which = 0: w13 ([2I][H], tiles of 64 gate + 64 up rows); which = 1: w2 ([H][I], tiles of 128 rows)
static void tile_geometry(int fmt, int H, int I, int which, int *m_tiles, int *kb, int *K) {
    if (which == 0) {
        *m_tiles = I / 64;
        *K = H;
    } else {
        *m_tiles = H / 128;
        *K = I;
    }
    *kb = *K / 128;
    (void)fmt;
}

size_t prepacked_expert_bytes(int fmt, int H, int I, int which) {
    int mt, kb, K;
    tile_geometry(fmt, H, I, which, &mt, &kb, &K);
    const size_t sb = 128 * (size_t)(stage_code_bytes(fmt) + stage_scale_bytes(fmt));
    return (size_t)mt * kb * sb;
}

// One thread per (expert, M tile, K stage, tile row).
__global__ void prepack_kernel(const uint8_t *__restrict__ w, int64_t w_estride, const uint8_t *__restrict__ scale,
                               int64_t s_estride, int E, int I, int K, int which, int m_tiles, int KB, int RB,
                               int SBY, int row_bytes, int s_row_bytes, int mx, uint8_t *__restrict__ out,
                               int64_t out_estride) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)E * m_tiles * KB * 128;
    if (gid >= total) return;
    const int r = (int)(gid & 127);
    int64_t t = gid >> 7;
    const int kb = (int)(t % KB);
    t /= KB;
    const int m = (int)(t % m_tiles);
    const int e = (int)(t / m_tiles);
    const int row = which == 0 ? (r < 64 ? m * 64 + r : I + m * 64 + (r - 64)) : m * 128 + r;
    const int64_t SB = 128LL * (RB + SBY);
    uint8_t *blob = out + e * out_estride + ((int64_t)m * KB + kb) * SB;
    const uint8_t *src = w + e * w_estride + (int64_t)row * row_bytes + (int64_t)kb * RB;
    const uint8_t *ss = scale + e * s_estride + (int64_t)row * s_row_bytes + (int64_t)kb * SBY;
    if (mx) {   // FP4, RB = 64: this thread fills half `kb % 2` of row r of blob (m, kb / 2)
        const int half = kb & 1;
        const int blob = kMxCodeBytes + 2 * 128 * SBY;   // SBY = 4 (MXFP4) or 8 (NVFP4) scales per half
        uint8_t *mb = out + e * out_estride + ((int64_t)m * (KB / 2) + (kb >> 1)) * blob;
        for (int c = 0; c < 4; ++c) {
            const int cc = half * 4 + c;   // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4 *>(mb + r * 128 + ((cc ^ (r & 7)) << 4)) =
                *reinterpret_cast<const uint4 *>(src + c * 16);
        }
        for (int i = 0; i < SBY; ++i) {   // scale i of the half: atom half * SBY/4 + i/4, block i % 4
            uint8_t *atom = mb + kMxCodeBytes + (half * (SBY / 4) + i / 4) * 512;
            atom[(r & 31) * 16 + (r >> 5) * 4 + (i & 3)] = ss[i];
        }
        return;
    }
    for (int c = 0; c < RB / 16; ++c)
        *reinterpret_cast<uint4 *>(blob + ((c * 128 + r) << 4)) = *reinterpret_cast<const uint4 *>(src + c * 16);
    if (SBY) {
        for (int i = 0; i < SBY; ++i) blob[128 * RB + r * SBY + i] = ss[i];
    }
    (void)K;
}

moe_status launch_prepack(const moe_experts &in, int which, void *out, int64_t out_estride, cudaStream_t st) {
    int mt, KB, K;
    tile_geometry(in.fmt, in.H, in.I, which, &mt, &KB, &K);
    const int RB = stage_code_bytes(in.fmt), SBY = stage_scale_bytes(in.fmt);
    const int row_bytes = RB * KB;                 // bytes of one standard row (K elements)
    const int s_row_bytes = scale_rowbytes(in.fmt, K);
    const int64_t rows = which == 0 ? 2LL * in.I : in.H;
    const int64_t dense_w = rows * row_bytes, dense_s = rows * s_row_bytes;
    const int64_t w_es = which == 0 ? (in.w13_estride ? in.w13_estride : dense_w) : (in.w2_estride ? in.w2_estride : dense_w);
    const int64_t s_es =
        which == 0 ? (in.w13s_estride ? in.w13s_estride : dense_s) : (in.w2s_estride ? in.w2s_estride : dense_s);
    const uint8_t *w = reinterpret_cast<const uint8_t *>(which == 0 ? in.w13 : in.w2);
    const uint8_t *s = reinterpret_cast<const uint8_t *>(which == 0 ? in.w13_scale : in.w2_scale);
    const int64_t total = (int64_t)in.E * mt * KB * 128;
    const int blocks = (int)((total + 255) / 256);
    count_launch();
    prepack_kernel<<<blocks, 256, 0, st>>>(w, w_es, s, s_es, in.E, in.I, K, which, mt, KB, RB, SBY, row_bytes,
                                           s_row_bytes, in.fmt == MOE_MXFP4 || in.fmt == MOE_NVFP4, reinterpret_cast<uint8_t *>(out),
                                           out_estride);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "prepack launch");
}

}  // namespace moe
