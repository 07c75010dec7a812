// Internal declarations shared by the host-side translation units of libmoe.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 1024;   // grouped FFN / permutation limit
constexpr int kMaxRouterExperts = 256;
constexpr int kMaxTopK = 16;
constexpr int kPhaseUp = 0;
constexpr int kPhaseDown = 1;

struct FfnParams {
    const int32_t *offsets;     // [E+1]
    const int32_t *expert_map;  // nullable [E]
    int E, H, I;
    int K;                      // reduction dimension of this phase (H or I)
    int m_tiles;                // I/64 (up) or H/128 (down)
    int stages;                 // shared-memory ring depth, set by the launcher
    int astages;                // TMEM ring depth (decoded weight stages), set by the launcher
    int bgroups;                // activation ring depth (groups of stages), set by the launcher
    const uint8_t *scale_base;  // scale plane of this phase's tensor (nullable for bf16)
    int64_t s_estride;          // bytes between experts in the scale plane
    int s_rowbytes;             // scale bytes per weight row
    const float *tscale;        // nvfp4 per-expert tensor scale, else nullable
    void *out;                  // up: h bf16 [n_rows][I]; down: y [n_rows][H]
    int out_fp32;
    int n_rows;
    int tiled;                  // weights prepacked (moe_prepack): one blob per (M tile, K stage)
    const uint8_t *wbase;       // tiled: this phase's prepacked tensor
    int64_t w_estride;          // tiled: bytes between experts
};

// Block-scaled FP4 path (ffn_mx.cu) for MXFP4 (kind::mxf4, E8M0 scales per 32)
// and NVFP4 (kind::mxf4nvf4, E4M3 scales per 16) experts prepacked by
// moe_prepack; activations as four E2M1 planes with per-tile scale atoms.
constexpr int kBsMx = 0, kBsNv = 1;              // formats of the path
constexpr int kMxStageK = 256;                   // K elements per pipeline stage
constexpr int kMxCodeBytes = 128 * 128;          // packed codes of one (M tile, stage): 128 rows x 128 B
constexpr int kMxPlanes = 4;                     // E2M1 planes per activation value

// 512-byte scale atoms per operand and stage (each covers 4 scales per row).
__host__ __device__ constexpr int bs_atoms(int f) { return f == kBsNv ? 4 : 2; }
// Bytes of one weight blob (M tile, stage): codes, then the scale atoms.
__host__ __device__ constexpr int bs_ablob_bytes(int f) { return kMxCodeBytes + 512 * bs_atoms(f); }
// Bytes of one activation blob (N tile of BN rows, stage): `planes` BN rows of 128 B, then the
// scale atoms. Four planes carry bf16 activations (A16); one plane is the activation itself in
// NVFP4 form (A4).
__host__ __device__ constexpr int bs_bblob_bytes(int f, int BN, int planes = kMxPlanes) {
    return planes * BN * 128 + 512 * bs_atoms(f);
}
constexpr int kA4Parts = 592;   // partial maxima of |x| (A4 tensor scale), 4 per SM of a 148-SM part

struct MxParams {
    const int32_t *offsets;     // [E+1]
    const int32_t *expert_map;  // nullable [E]
    int E, H, I;
    int K;                      // reduction dimension of this phase (H or I)
    int m_tiles;                // I/64 (up) or H/128 (down)
    int stages;                 // shared-memory slots, set by the launcher
    int pipes;                  // independent producer/MMA pipelines, set by the launcher
    int itempar;                // pipelines take whole items (else stages of every item), set by the launcher
    int nbuf;                   // accumulator buffers per pipeline (2, or 3 where TMEM has room), set by the launcher
    int n_rows;
    const uint8_t *wbase;       // this phase's prepacked tensor: [m_tiles][K/256] weight blobs
    int64_t w_estride;          // bytes between experts (or cache slots)
    const uint8_t *bblob;       // activation blobs [tiles][K/256]
    const int32_t *rowexp;      // NVFP4: per-row exponent offset of the activation planes [n_rows]
    const float *tscale;        // NVFP4: per-expert tensor scale of this phase's weights [E]
    void *out;                  // down: y [n_rows][H] (bf16 or fp32)
    int out_fp32;
    uint8_t *bblob_out;         // MXFP4 and A4 up: blobs of h for the down pass [tiles][I/256]
    void *hout;                 // NVFP4 up: h bf16 [n_rows][I]
    const float *xscale;        // A4 up: device word with the per-tensor scale of x
    int *sched;                 // item claim counter of this phase (zero at launch), or null: static order
    // Slot layout of decode-sized batches (routing wrote the rows; no permutation ran):
    // expert e owns pair rows [e slab_T, (e + 1) slab_T), slab_cnt[e] of them used, and
    // its UP input tiles are e slab_mt ... (compact tiles otherwise). Rows of h and y stay
    // compact: expert e's start at the prefix of the counts, published in cprefix.
    const int32_t *slab_cnt;    // null: offsets describe the rows
    int slab_T, slab_mt;
    int32_t *cprefix;           // [E] written by the UP kernel in the slot layout
    int slab_wait;              // slab_cnt comes from the previous kernel: read it after the wait
    // Slot layout with most experts routed to: the first tile of each of the first experts
    // (enough for every CTA's static first items) leads the item order, present even when the
    // expert has no rows, so those items' weights go out before the tile prefix and the wait
    // on the router. Outputs (h, y rows) and input tiles read by index keep the compact order.
    int slab_head;
};

// error reporting (thread-local message), defined in api.cu
moe_status set_error(moe_status s, const char *fmt, ...);
moe_status set_cuda_error(cudaError_t e, const char *what);

int num_sms(int device);
int stage_scale_bytes(int fmt);
int stage_code_bytes(int fmt);
size_t prepacked_expert_bytes(int fmt, int H, int I, int which);
moe_status launch_prepack(const moe_experts &in, int which, void *out, int64_t out_estride, cudaStream_t st);
int choose_bn(int n_rows, int E);
int scale_rowbytes(int fmt, int K);

moe_status launch_ffn_phase(int phase, int fmt, int BN, const CUtensorMap &wmap, const CUtensorMap &bmap,
                            FfnParams p, int num_sms, cudaStream_t st);

int choose_bn_mx(int n_rows, int E);
struct MxPlan {
    int pipes, stages, itempar, nbuf;
};
bool mx_plan(int fmt, int phase, int BN, int K, int E, MxPlan *pl, int planes = kMxPlanes);
size_t mx_tiles_ub(int n_rows, int E);
size_t mx_blob_bytes(int n_rows, int K, int E);
size_t mx_blob_bound(int n_rows, int K, int E);   // max of mx_blob_bytes over row counts <= n_rows
// planes: kMxPlanes (A16 activations) or 1 (A4, NVFP4 only)
moe_status launch_mx_phase(int fmt, int phase, int BN, MxParams p, int num_sms, cudaStream_t st,
                           int planes = kMxPlanes);
// A4 (activations in NVFP4 form): token tile, workspace of the activation blobs, the
// partial maxima of |x| and the quantiser (src rows as launch_mx_quant modes 1 and 2).
int choose_bn_a4(int n_rows, int E);
size_t a4_blob_bytes(int n_rows, int K, int E);
size_t a4_blob_bound(int n_rows, int K, int E);   // max of a4_blob_bytes over row counts <= n_rows
moe_status launch_a4_amax(const void *src, int64_t n_elems, float *partials, int *sched_zero, cudaStream_t st);
moe_status launch_a4_token_rows(const void *x, int T, int K, int k, const int32_t *pair_row, const int32_t *offsets,
                                int E, int BN, const float *partials, float *xscale, void *bblob, int num_sms,
                                cudaStream_t st);
// Token-major A4 rows of x [T][K] (codes [T][K/2], scales [T][K/16]), then their scatter into
// the blobs of the pairs (the layer forward's path: each token quantised once, not k times).
moe_status launch_a4_quant(const void *src, int mode, const int32_t *sorted_pair, int k, int P, int K,
                           const int32_t *offsets, int E, int BN, const float *partials, float *xscale, void *bblob,
                           int num_sms, cudaStream_t st);
// src rows: mode 0 x_perm[r] (operand order), 1 x[sorted_pair[r] / k] (natural
// order), 2 src[r] (natural order; NVFP4 only). rowexp: NVFP4 only.
moe_status launch_mx_quant(int fmt, const void *src, int mode, const int32_t *sorted_pair, int k, int P, int K,
                           const int32_t *offsets, int E, int BN, void *bblob, int32_t *rowexp, int num_sms,
                           cudaStream_t st, int *sched_zero = nullptr);

moe_status launch_dequant(int fmt, const void *w, const void *scale, float tscale, int rows, int K, void *out,
                          cudaStream_t st);

// router (router.cu)
size_t router_ws_bytes(int T, int H, int E);
size_t router_ws_bound(int T, int H, int E);   // max of router_ws_bytes over batches <= T
// Outputs of the permutation for a router launch that also permutes (the
// layer forward); the launcher fills in the ticket counter.
struct RouterFuse {
    int32_t *offsets, *sorted_pair, *pair_row;
    unsigned int *ticket;
    // Slot layout (cnt non-null, MXFP4 FFN of a decode-sized batch): pair j of token t takes
    // row e T + atomicAdd(cnt + e, 1) of its expert e (pair_row), and the token's activation
    // row is written in the four-plane MXFP4 form into row pos % BN of tile e mt + pos / BN of
    // bslab. No permutation runs; cnt starts at zero (the layer's combine clears it again).
    int32_t *cnt;
    uint8_t *bslab;
    int BN, mt;
    int *sched_zero;   // the FFN's claim counters, zeroed here
};
// fuse may be null; *fused (if given): 1 the permutation was done, 2 the slot layout was
// written (fuse->cnt set; the cluster router must apply: router_cluster_ok).
int32_t *route_slot_counts(cudaStream_t st);
bool router_cluster_ok(int T, int H, int E, int wr_is_fp32, const void *wr);
moe_status launch_router(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                         int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes, int nsm,
                         cudaStream_t st, const RouterFuse *fuse = nullptr, int *fused = nullptr);

// permutation (permute.cu)
size_t permute_ws_bytes(int T, int k, int E);
size_t permute_scratch_bytes(int T, int k, int E);
// natural: x_perm rows in natural column order (A4 activations), else in the operand order
// 0,4,1,5,2,6,3,7 of every group of 8 (A16)
moe_status launch_permute(const int32_t *idx, int T, int k, int E, const void *x, int H, int32_t *offsets,
                          int32_t *sorted_pair, int32_t *pair_row, void *x_perm, void *ws, size_t ws_bytes,
                          cudaStream_t st, int natural = 0);

// combine (combine.cu)
moe_status launch_combine(const void *y_perm, int y_is_fp32, const int32_t *pair_row, const float *w, int T, int k,
                          int H, void *out, cudaStream_t st, int early = 0,
                          const int32_t *cprefix = nullptr, int slab_T = 1, int32_t *cnt_zero = nullptr,
                          int E = 0);

// tensor maps (api.cu)
moe_status make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                     const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle sw);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace moe
