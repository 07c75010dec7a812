/*
 * moe.h - C ABI of the B200 (sm_100a) MoE-layer library (libmoe.so).
 *
 * One hot path: the forward pass of a mixture-of-experts layer over
 * quantised experts, plus the device expert cache that lets an expert pool
 * larger than device memory stream from pinned host memory.
 *
 * Sources. The pages describing the serving engine this layer comes from give
 * the problem, not the kernels:
 *   [P3] winzheng.com, "FreeToken ... 753B local inference MoE":
 *        section "Why Now of All Times" - each token activates a few routed
 *        experts per layer (top-k routing); most experts can stay in host
 *        memory and be loaded on demand;
 *        section "FreeToken's Three-Layer Mechanism" - double-buffered
 *        streaming overlapping weight movement with compute, and a global
 *        LRU expert cache reusing high-frequency experts.
 *   [P4] aimodeling.com, "FreeToken: UC Berkeley Brings 753B GLM-5.2 MoE
 *        Inference to Consumer Hardware": section "Three Engineering Cores"
 *        (the same LRU cache and double-buffered streaming) and section
 *        "Reported Numbers and Ecosystem Position" (expert formats MXFP4,
 *        NVFP4, FP8 and BF16).
 * The pages give no router, gating, FFN or combine formula; this library
 * implements the standard top-k softmax SwiGLU MoE layer:
 *   logits = x.Wr (+ bias), rounded once to fp32 from an fp64 sum;
 *   idx = top-k logits (ties to the lower expert index);
 *   w = softmax over the k selected logits;
 *   y_p = W2_e . (silu(Wg_e . x_t) * (Wu_e . x_t)) for each pair p = (t, j);
 *   out_t = sum_j w[t,j] y_(t,j).
 *
 * Conventions for every call:
 *   - All pointers are device pointers unless marked "host".
 *   - The caller owns every buffer passed in. The library allocates nothing on
 *     the hot path; scratch comes from the caller's workspace `ws` of at least
 *     moe_workspace_size() bytes (256-byte aligned).
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream). The only host synchronisation is
 *     inside moe_layer_forward when a cache is given (the miss list is read
 *     back once per call).
 *   - Every call returns a moe_status; moe_last_error_string() gives a
 *     thread-local message for the last failure. There is no CPU fallback:
 *     unsupported shapes or formats return MOE_ERR_UNSUPPORTED.
 *   - Layouts are row-major. bf16 values are passed as raw 16-bit patterns.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* identical to cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned buffer */
    MOE_ERR_UNSUPPORTED = 2, /* shape or format outside the kernel set */
    MOE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    MOE_ERR_OOM = 4,         /* workspace too small, or a cache allocation failed */
    MOE_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired */
    MOE_ERR_CACHE_FULL = 6   /* the cache cannot hold one call's working set */
} moe_status;

/* Stored expert-weight formats ([P4] "Reported Numbers and Ecosystem Position").
 * For a tensor [R, K] (K = reduction dimension, contiguous):
 *   MOE_BF16          codes: bf16 [R][K]; no scales.
 *   MOE_FP8_E4M3_K128 codes: E4M3 bytes [R][K]; scale: fp32 [R][K/128].
 *   MOE_MXFP4         codes: E2M1, two per byte, low nibble = lower K index, [R][K/2];
 *                     scale: E8M0 bytes [R][K/32].
 *   MOE_NVFP4         codes: as MXFP4; scale: E4M3 bytes [R][K/16];
 *                     tscale: one fp32 per expert and tensor. */
typedef enum { MOE_BF16 = 0, MOE_FP8_E4M3_K128 = 1, MOE_MXFP4 = 2, MOE_NVFP4 = 3 } moe_wfmt;

/* Activation format inside the expert GEMMs. The pages name the weight formats
 * ([P4] "Reported Numbers and Ecosystem Position") but not the precision the
 * activations enter the GEMMs in; this library offers two, and the math of the
 * layer depends on the choice:
 *   MOE_ACT_A16  the activations as given: x in bf16, h rounded to bf16 before
 *                the down projection. The default.
 *   MOE_ACT_A4   the activations in NVFP4 form, so that both operands of every
 *                expert GEMM are FP4 (block-scaled FP4 tensor-core MMA): x with
 *                one per-tensor scale s_g = amax|x| / (6 * 448) over the whole
 *                [T][H] batch (1 if x is all zero), h with s_g = 1; per 16
 *                elements along K an E4M3 scale s_b = E4M3((amax_16 / 6) / s_g)
 *                and E2M1 codes of v / (s_b * s_g), both rounded to nearest,
 *                ties to even, saturating; the GEMM sees q * s_b * s_g.
 *                Prepacked NVFP4 experts only (MOE_ERR_UNSUPPORTED otherwise). */
typedef enum { MOE_ACT_A16 = 0, MOE_ACT_A4 = 1 } moe_actfmt;

/* Memory layout of the expert codes. STANDARD: row-major as described above.
 * TILED: produced by moe_prepack. The values are the same and so is the byte
 * count (codes plus scales); only the byte order differs. Weight rows form M
 * tiles of 128 (w13: 64 gate rows and the 64 matching up rows; w2: 128
 * consecutive rows), and every (M tile, K stage) is one contiguous blob, so
 * one bulk copy moves a stage. Blobs are ordered by M tile, then stage.
 *   BF16, FP8 (stages 128 wide): the codes as 16-byte chunks, chunk c of row r
 *     at (c*128 + r)*16, then each row's scales for the stage (FP8: one fp32).
 *   MXFP4, NVFP4 (stages 256 wide): 128 rows of packed codes, 128 bytes per
 *     row in natural K order, the 16-byte chunk c of row r at
 *     r*128 + (c XOR (r%8))*16; then 512-byte scale atoms, the scale of row r
 *     and block j of the atom's K range at byte (r%32)*16 + (r/32)*4 + j.
 *     MXFP4: two atoms (E8M0 per 32, one per 128-wide half), 17 KiB per blob.
 *     NVFP4: four atoms (E4M3 per 16, one per 64-wide quarter), 18 KiB.
 * Prepacked MXFP4 runs the block-scaled FP4 tensor-core path; prepacked NVFP4
 * runs it for up to 16 rows per expert on average, else the decoding path. */
typedef enum { MOE_LAYOUT_STANDARD = 0, MOE_LAYOUT_TILED = 1 } moe_layout;

/* The experts of one layer.
 *   w13: gate and up projections, per expert [2I][H] (gate rows 0..I-1, then up rows).
 *   w2:  down projection, per expert [H][I].
 *   *_scale: scale planes as above (NULL for MOE_BF16).
 *   *_tscale: [E] fp32 per-expert tensor scales (MOE_NVFP4 only, else NULL);
 *             always indexed by the logical expert id.
 *   *_estride: bytes from expert e to expert e+1 in each array; 0 = densely
 *             packed. Codes, scales and strides must be 16-byte aligned.
 *   expert_map: optional device [E] int32; when set, expert e's data is the
 *             expert_map[e]-th entry of the strided arrays (used by the cache).
 *   n_entries: number of entries in the strided arrays when expert_map is
 *             set (0 = E).
 *   layout:   MOE_LAYOUT_STANDARD (the arrays above) or MOE_LAYOUT_TILED
 *             (w13/w2 hold moe_prepack output, scales included; *_scale and
 *             the scale strides are ignored; *_estride 0 = densely packed). */
typedef struct {
    int fmt; /* moe_wfmt */
    int E, H, I;
    const void *w13;
    const void *w13_scale;
    const float *w13_tscale;
    const void *w2;
    const void *w2_scale;
    const float *w2_tscale;
    int64_t w13_estride, w13s_estride, w2_estride, w2s_estride;
    const int32_t *expert_map;
    int n_entries;
    int layout; /* moe_layout */
} moe_experts;

/* Router logits + top-k + softmax gating ([P3] "Why Now of All Times": a token
 * activates k routed experts).
 *   x: bf16 [T][H]; wr: [H][E], fp32 if wr_is_fp32 else bf16; bias: nullable fp32 [E].
 *   Logits are the fp64 sum of x*Wr rounded once to fp32, plus bias (one fp32 add).
 *   idx: int32 [T][k] in descending logit order, ties to the lower expert index.
 *   w: fp32 [T][k], softmax over the k selected logits. logits: nullable fp32 [T][E].
 *   ws: scratch of moe_workspace_size(T, H, ...) bytes (fp64 partial sums).
 *   Requires 1 <= k <= 16, k <= E <= 256, H % 8 == 0, x and wr 16-byte aligned.
 *   T == 0 is a no-op. Errors: INVALID_ARG for T < 0, H not a positive multiple
 *   of 8, NULL x, wr, idx, w or ws, x, wr or ws not 16-byte aligned, or idx, w,
 *   logits or bias not 4-byte aligned; UNSUPPORTED for k or E outside the
 *   limits; OOM when ws_bytes is below what the call needs. */
moe_status moe_route_topk(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                          int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Token-to-expert permutation (the dispatch implied by [P3] "Why Now of All
 * Times"): a counting sort of the T*k pairs p = t*k + j by expert, stable in p.
 *   offsets: int32 [E+1], exclusive scan of per-expert counts (offsets[E] = T*k).
 *   sorted_pair: int32 [T*k], the pairs in expert order; pair_row: its inverse.
 *   x_perm (nullable): bf16 [T*k][H], row r = x[sorted_pair[r] / k], laid out for
 *     moe_grouped_ffn with the same activation format `af`: MOE_ACT_A16 stores the
 *     columns of every aligned group of 8 in the order 0,4,1,5,2,6,3,7; MOE_ACT_A4
 *     stores them in natural order (the A4 FFN quantises the rows itself).
 *   Bit-exact and deterministic. Requires H % 8 == 0.
 *   Errors: INVALID_ARG for T < 0, k outside 1..16, E outside 1..1024, an unknown
 *   af, NULL offsets, NULL idx, sorted_pair, pair_row or ws when T > 0, x_perm
 *   without x, H not a positive multiple of 8 or x or x_perm not 16-byte aligned
 *   when x_perm is given, int32 arrays not 4-byte aligned, or ws not 16-byte
 *   aligned; OOM when ws_bytes is below what the call needs. */
moe_status moe_permute(const int32_t *idx, int T, int k, int E, const void *x, int H, int af, int32_t *offsets,
                       int32_t *sorted_pair, int32_t *pair_row, void *x_perm, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_permute (with af = MOE_ACT_A16) without a caller workspace: the same permutation, bit for bit,
 * with the scratch taken from a fixed device array inside the library instead
 * of `ws`. The pages have no counterpart; it exists for callers that cannot
 * hand over device memory (no allocation happens anywhere on this path).
 *   Scratch limit: MOE_PERMUTE_STATIC_SCRATCH_BYTES per device. Sizes whose
 *   scratch would exceed it (two arrays of ceil(T*k/1024)*E int32, each rounded
 *   up to 256 bytes; none when T*k <= 8192 and E <= 256) are rejected with
 *   MOE_ERR_UNSUPPORTED before anything is enqueued.
 *   No word of the scratch has to start at zero: every per-chunk counter and
 *   base is written before it is read within one call, so nothing is cleared.
 *   Set-up: the first call on a device looks the array's device address up
 *   (one runtime call, not a stream operation); make that first call before
 *   any stream capture on that device.
 *   Concurrency: every call on a device shares the one array, so calls whose
 *   kernels may overlap (different streams, or different host threads without
 *   ordering) race on it; serialise them on one stream.
 *   Arguments, layouts, ownership and the other errors are those of
 *   moe_permute. */
#define MOE_PERMUTE_STATIC_SCRATCH_BYTES (1u << 20)
moe_status moe_permute_static(const int32_t *idx, int T, int k, int E, const void *x, int H, int32_t *offsets,
                              int32_t *sorted_pair, int32_t *pair_row, void *x_perm, moe_stream_t stream);

/* Grouped SwiGLU expert FFN over the permuted rows ([P4] formats; the routed
 * experts of [P3] "Why Now of All Times"): for every expert e and row r in
 * [offsets[e], offsets[e+1]):
 *   h = silu(Wg_e . x_perm[r]) * (Wu_e . x_perm[r]), rounded to bf16 (A16) or
 *       put in NVFP4 form with tensor scale 1 (A4);
 *   y_perm[r] = W2_e . h   (bf16, or fp32 if y_is_fp32).
 *   x_perm: bf16 [n_rows][H] as moe_permute writes it for the same `af` (A16:
 *     interleaved columns; A4: natural order, quantised here with the tensor
 *     scale of the n_rows rows, which equals that of x when every token is
 *     among them).
 *   af: moe_actfmt; MOE_ACT_A4 needs prepacked NVFP4 experts (UNSUPPORTED else)
 *     and runs the block-scaled FP4 path with one plane per activation.
 *   offsets: int32 [E+1] as moe_permute writes them: offsets[0] = 0,
 *     non-decreasing, offsets[E] = n_rows. The kernels take them as given (they
 *     are read on the device only); other values make them read and write
 *     outside x_perm and y_perm.
 *   y_perm: [n_rows][H], natural column order.
 *   ws: scratch; moe_workspace_size(n_rows, H, I, E, 1, y_is_fp32) bytes
 *   always suffice. The decoding path (row-major experts, BF16, FP8, and
 *   prepacked NVFP4 with more than 16 rows per expert on average) keeps h there
 *   ([n_rows][I] bf16, operand column order). The block-scaled FP4 path
 *   (prepacked MXFP4; prepacked NVFP4 up to 16 rows per expert) keeps x_perm and
 *   h as four E2M1 planes each, within 2^-11 of each 32-block's (16-block's)
 *   maximum, with their scale atoms; for NVFP4 also h in bf16 [n_rows][I],
 *   natural column order, at the start of ws.
 *   Requires H % 256 == 0, I % 256 == 0, E <= 1024. n_rows == 0 is a no-op.
 *   Errors: UNSUPPORTED for an unknown format, E outside 1..1024, or H or I not
 *   positive multiples of 256; INVALID_ARG for NULL pointers, an unknown layout,
 *   missing scale planes or NVFP4 tensor scales, codes, scales, strides, x_perm,
 *   y_perm or ws not 16-byte aligned, tensor scales, expert_map or offsets not
 *   4-byte aligned, or n_rows < 0; OOM when ws_bytes is below what the call
 *   needs. */
moe_status moe_grouped_ffn(const void *x_perm, int n_rows, const int32_t *offsets, const moe_experts *experts,
                           int af, void *y_perm, int y_is_fp32, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Gate-weighted combine: out[t] = sum_{j<k} w[t,j] * y_perm[pair_row[t*k+j]],
 * accumulated in fp32 in order of j, rounded to bf16 (the outputs of a token's
 * k routed experts, [P3] "Why Now of All Times", weighted by its gates; the
 * pages give no formula, this is the standard top-k mixture).
 *   y_perm: [T*k][H] bf16 or fp32 (y_is_fp32); out: bf16 [T][H]. H % 8 == 0.
 *   T == 0 is a no-op. Errors: INVALID_ARG for T < 0, k outside 1..16, H not a
 *   positive multiple of 8, NULL pointers, y_perm or out not 16-byte aligned, or
 *   pair_row or w not 4-byte aligned. A pair_row entry outside 0..T*k-1 is found
 *   on the device: it sets the device error word to 2 (moe_device_error) and row
 *   0 is read in its place. */
moe_status moe_combine(const void *y_perm, int y_is_fp32, const int32_t *pair_row, const float *w, int T, int k,
                       int H, void *out, moe_stream_t stream);

/* Dequantise one expert tensor [rows][K] stored in `fmt` ([P4] formats) to bf16
 * [rows][K] (row-major, natural K order), with the same decode the grouped FFN
 * applies to its weight tiles. Exact for BF16 and MXFP4 (within bf16 range);
 * NVFP4 ((E2M1 * E4M3) * tscale) and FP8 (E4M3 * fp32 scale) are rounded to
 * bf16. w/scale as in moe_experts for a single expert; tscale: host value
 * (NVFP4 only). K must be a multiple of the format's block (128/32/16/8).
 * rows == 0 is a no-op. Errors: UNSUPPORTED for an unknown format; INVALID_ARG
 * for rows < 0, K not a positive multiple of the block, NULL pointers (scale
 * may be NULL for BF16), w or out not 16-byte aligned, or FP8 scales not
 * 4-byte aligned. */
moe_status moe_dequantize(int fmt, const void *w, const void *scale, float tscale, int rows, int K, void *out,
                          moe_stream_t stream);

/* Bytes of one expert's prepacked w13 (which = 0) or w2 (which = 1): equal to
 * its standard layout's code and scale bytes, since prepacking only reorders
 * bytes. Host-only; 0 for an unknown format, H or I not a positive multiple of
 * 256, or `which` other than 0 and 1. */
size_t moe_prepacked_expert_bytes(int fmt, int H, int I, int which);

/* Rewrite a layer's experts from MOE_LAYOUT_STANDARD into MOE_LAYOUT_TILED
 * (a device-side byte permutation, done once when weights are loaded).
 *   in: standard-layout experts (device pointers; expert_map must be NULL).
 *   out_w13, out_w2: device buffers of E * moe_prepacked_expert_bytes(...) bytes,
 *   16-byte aligned. The result is used through a moe_experts with
 *   layout = MOE_LAYOUT_TILED, w13 = out_w13, w2 = out_w2 (tscales unchanged).
 *   Errors: those of moe_grouped_ffn's expert checks; INVALID_ARG for a tiled
 *   input, an expert_map, or NULL or misaligned outputs. */
moe_status moe_prepack(const moe_experts *in, void *out_w13, void *out_w2, moe_stream_t stream);

struct expert_cache;

/* The whole layer: route -> permute -> grouped FFN -> combine (the MoE layer of
 * [P3] "Why Now of All Times": each token runs through its k routed experts;
 * with a cache, the experts come from the device cache fed by host streaming of
 * [P3] "FreeToken's Three-Layer Mechanism" and [P4] "Three Engineering Cores").
 *   af: moe_actfmt of the expert GEMMs (MOE_ACT_A4: prepacked NVFP4 experts;
 *     with a cache, a cache built on prepacked NVFP4 layers).
 *   cache: nullable. When set, `experts` gives the layer's shape and format
 *     only, the weights come from the cache's device slots for `layer`, and
 *     missing experts are streamed from the cache's pinned host pool first
 *     (one host synchronisation per call to read the miss list).
 *   idx_out, w_out: nullable copies of the routing.
 *   y_is_fp32: keep the expert outputs in fp32 before the combine.
 * Decode-sized MXFP4 batches (T <= 256, T k <= 8192, the activation tiles below
 * 64 MiB) skip the separate permutation and quantiser: the router gives each
 * pair a row in a per-expert slot of T rows by an atomic claim and writes the
 * token's four-plane activation rows straight into those rows' tiles. The order
 * of rows inside an expert then depends on timing, but every row's result does
 * not, so `out` is the same as on the other paths. The slots' row counts are
 * per stream and cleared by the call's last kernel.
 * T == 0 is a no-op. Errors: INVALID_ARG for NULL experts, x, wr, out or ws,
 * T < 0, an unknown af, k outside 1..min(16, E), x, wr or out not 16-byte
 * aligned, bias, idx_out or w_out not 4-byte aligned, or ws not 256-byte
 * aligned; UNSUPPORTED for a shape or format outside the kernels (as for
 * moe_grouped_ffn; the router takes E <= 256); OOM when ws_bytes is below
 * moe_workspace_size(); CACHE_FULL when the cache cannot hold the layer's
 * experts, with the table left unchanged. */
moe_status moe_layer_forward(const void *x, int T, const void *wr, int wr_is_fp32, const float *bias, int k,
                             const moe_experts *experts, int af, struct expert_cache *cache, int layer,
                             int y_is_fp32, void *out, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                             moe_stream_t stream);

/* Scratch bytes needed by moe_layer_forward / moe_route_topk / moe_permute /
 * moe_grouped_ffn for these sizes and activation format: an upper bound that
 * covers every path the sizes can take (the router's fp64 partial sums, the
 * routing, the permutation, x_perm, h or the FP4 activation blobs, y, and for
 * decode-sized batches the slot layout's tiles). The bound never decreases as T
 * grows, with the other sizes fixed, so a workspace sized for the largest batch
 * serves every smaller one. No counterpart in the pages: it is what lets every
 * call run without allocating. Host-only, no CUDA call; 0 for non-positive sizes
 * or an unknown af. */
size_t moe_workspace_size(int T, int H, int I, int E, int k, int y_is_fp32, int af);

/* ---------------------------------------------------------------- cache */
/* Device LRU expert cache with streaming from pinned host memory ([P3]
 * "FreeToken's Three-Layer Mechanism"; [P4] "Three Engineering Cores").
 * The slot pool is one device allocation of capacity_bytes / slot_bytes slots,
 * each holding one expert's w13, w2 and scales. The table (slot of each
 * (layer, expert), owner and recency of each slot) lives on the device and is
 * updated by a kernel; misses are copied host->device with cudaMemcpyAsync on
 * the cache's own copy stream, and the compute stream waits on an event.
 * Policy: ascending expert ids within a call; a miss takes the lowest free
 * slot, else evicts the least recently referenced slot not referenced by this
 * call or the previous one. */

/* host_layers: host array [n_layers] of layer descriptions whose code/scale
 * pointers are host pointers into page-locked (pinned) memory; all layers
 * share fmt, E, H, I. The library allocates the slot pool, the table, a copy
 * stream and events on `device`. The library keeps the pointers, not copies.
 * Errors: INVALID_ARG for NULL arguments, n_layers <= 0, or layers that differ
 * in format, shape or layout; UNSUPPORTED for a shape the grouped FFN rejects;
 * CACHE_FULL when capacity_bytes holds less than one expert; OOM or CUDA when
 * an allocation or copy fails. */
moe_status expert_cache_init(struct expert_cache **cache, size_t capacity_bytes, int n_layers,
                             const moe_experts *host_layers, int device);

/* Load the listed experts of `layer` (host array ids[n]) ahead of use, on the
 * copy stream, without counting hits or misses. Synchronises with `stream`
 * once to read back the loads the table update decided. n == 0 is a no-op.
 * Errors: INVALID_ARG for a bad layer, n outside 0..E or NULL ids; CACHE_FULL
 * when the experts do not fit, with the table left unchanged. */
moe_status expert_cache_prefetch(struct expert_cache *cache, int layer, const int32_t *ids, int n,
                                 moe_stream_t stream);

/* Free slots: layer -1 = every slot; n -1 = all experts of `layer`; else the
 * n listed experts (host array). Synchronous. Errors: INVALID_ARG for a layer
 * outside -1..n_layers-1, n > E, or NULL ids with n > 0. */
moe_status expert_cache_evict(struct expert_cache *cache, int layer, const int32_t *ids, int n);

/* Counters since init: hits and misses of layer-forward calls, bytes copied
 * host->device, and seconds the copy stream spent copying (event-timed). */
moe_status expert_cache_stats(struct expert_cache *cache, uint64_t *hits, uint64_t *misses, uint64_t *bytes_h2d,
                              double *copy_s);

/* Prefetch of the next layer, decided per cached layer call ([P4] "Three
 * Engineering Cores": full-layer double-buffered streaming; [P3] "FreeToken's
 * Three-Layer Mechanism": the transfer adapts to the bandwidth it measures).
 * After a call resolves layer l, experts of layer l+1 are loaded behind that
 * layer's own misses on the copy stream, so they arrive while layer l computes.
 * The prediction for layer l+1 is the set of experts its previous call used,
 * ranked by the pairs each received (more first, ties to the lower id).
 *   MOE_PREFETCH_NONE        nothing.
 *   MOE_PREFETCH_PREDICTED   the first `depth` experts of the prediction
 *                            (depth < 0: all of it). The default, depth -1.
 *   MOE_PREFETCH_FULL_LAYER  every expert of layer l+1 (prefill: the next call
 *                            touches nearly every expert).
 *   MOE_PREFETCH_ADAPTIVE    per call: the full layer when the call's T tokens
 *                            are expected to reach at least half of the E
 *                            experts (E (1 - (1 - k/E)^T) >= E/2); otherwise
 *                            the first floor(bw * t / expert_bytes) of the
 *                            prediction, bw being the measured host-to-device
 *                            rate and t the measured time of a cached layer's
 *                            FFN and combine (running averages); the whole
 *                            prediction until both have been measured.
 * A prefetch that does not fit in the free and evictable slots is skipped. */
typedef enum {
    MOE_PREFETCH_NONE = 0,
    MOE_PREFETCH_PREDICTED = 1,
    MOE_PREFETCH_FULL_LAYER = 2,
    MOE_PREFETCH_ADAPTIVE = 3
} moe_prefetch_policy;

/* Set the prefetch policy (host call, takes effect at the next layer call).
 * Errors: INVALID_ARG for a NULL cache or an unknown policy. */
moe_status expert_cache_set_prefetch(struct expert_cache *cache, int policy, int depth);

/* Resize the slot pool to floor(capacity_bytes / slot bytes) slots without
 * fetching any resident expert again ([P4] "Three Engineering Cores": elastic
 * memory management without weight reloads). The pool is a reserved virtual
 * address range backed by physical chunks: growing maps more chunks and adds
 * free slots; shrinking keeps the most recently used experts that fit, moves
 * those above the new end into the lowest free slots (least recent first, by
 * device-to-device copy on the cache's copy stream), drops the rest and unmaps
 * the chunks past the new end. Synchronous: it waits for the device, so no
 * layer call may be in flight on another thread. The table change follows the
 * rule of the cache's policy exactly.
 * Errors: INVALID_ARG for a NULL cache; CACHE_FULL for a capacity below one
 * expert; UNSUPPORTED when the pool could not be built on reserved addresses
 * (then only sizes within the first allocation are accepted) or the capacity
 * exceeds the reserved range (the device's memory); OOM or CUDA when mapping
 * fails, with the cache unchanged. */
moe_status expert_cache_resize(struct expert_cache *cache, size_t capacity_bytes);

/* What the cache measured since init. Seconds are summed over the cached layer
 * calls whose events have completed. */
typedef struct {
    double table_s;      /* device time of the table updates (event-timed) */
    double host_wait_s;  /* host time spent waiting for a table update to finish */
    double issue_s;      /* host time spent enqueueing copies */
    double copy_s;       /* time the copy stream spent copying (event-timed) */
    double compute_s;    /* caller-stream time of the cached calls' FFN and combine */
    double overlap_s;    /* copy time that fell inside those FFN-and-combine intervals */
    double h2d_gbs;      /* running average of the measured host-to-device rate, GB/s (0: none yet) */
    uint64_t calls;      /* cached layer calls */
    uint64_t prefetched; /* experts loaded by next-layer prefetches */
    uint64_t moved;      /* experts moved device-to-device by resizes */
    int n_slots;         /* slots in the pool now */
    int last_depth;      /* depth of the last call's prefetch (-1: whole prediction; E: whole layer) */
} moe_cache_report;

/* Fill *out (waits for the copy stream first). Errors: INVALID_ARG for NULL. */
moe_status expert_cache_report(struct expert_cache *cache, moe_cache_report *out);

/* Device slot of (layer, e), or -1 (synchronous read; for tests and tools). */
moe_status expert_cache_slot_of(struct expert_cache *cache, int layer, int e, int32_t *slot);

/* Waits for outstanding copies and frees everything the cache allocated. */
moe_status expert_cache_destroy(struct expert_cache *cache);

/* ---------------------------------------------------------------- misc */

/* Thread-local message describing the last failing call on this thread. */
const char *moe_last_error_string(void);

/* Reads and clears the device error word set by bounded waits and in-kernel
 * checks (0 = none; 1 = a wait timed out; 2 = bad argument seen on device).
 * Synchronises the device. */
moe_status moe_device_error(int *code);

/* Limit of the bounded device-side waits (the kernels' waits on barriers that
 * another role of the same CTA completes), in nanoseconds, on the current
 * device; 0 restores the default of 2 s. Waits that keep a CTA alive until its
 * own bulk copies and MMAs have landed keep the 2 s limit whatever is set. No
 * counterpart in the pages: a test hook for the failure path of the bounded
 * waits. Synchronous. Errors: CUDA. */
moe_status moe_set_wait_limit_ns(uint64_t ns);

/* Enqueue one small kernel that waits, through the same bounded-wait code as
 * the grouped FFN, on a barrier that nothing completes, with no copy or MMA in
 * flight. It gives up after the wait limit, sets the device error word to 1
 * and returns, leaving the context usable. No counterpart in the pages: the
 * test of the bounded waits. Errors: CUDA for a failed launch. */
moe_status moe_selftest_wait(moe_stream_t stream);

/* Dense tensor-core throughput of the current device for one MMA kind of the
 * grouped FFN (kind 0: bf16 kind::f16; 1: FP8 E4M3 kind::f8f6f4; 2: MXFP4
 * kind::mxf4; 3: NVFP4 kind::mxf4nvf4), measured by this library's own MMA loop:
 * one CTA per SM issues `iters` x 4 MMAs of M = 128, N = 256 on operands held in
 * shared memory (no memory traffic), a warm-up launch and three timed ones
 * (CUDA events). *tflops: the measured rate. No counterpart in the pages: the
 * roofline denominators of the FFN kernels. Synchronous; creates and destroys
 * its own stream and events. Errors: INVALID_ARG for an unknown kind, iters < 1
 * or NULL tflops; CUDA. */
moe_status moe_tensor_peak(int kind, int iters, double *tflops);

/* Library version, for logs. */
const char *moe_version(void);

/* Number of kernels this library has enqueued in this process, on every device
 * and stream, since it was loaded (a running count; the difference across a
 * region is the launch count of that region). No counterpart in the pages:
 * launch accounting for benchmarks. Never fails. */
uint64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
