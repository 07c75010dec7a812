// C-ABI entry points of libmoe (declared in include/moe.h): argument checks,
// workspace carving, TMA descriptor construction and kernel launches.
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

static thread_local char t_err[512] = "no error";

moe_status set_error(moe_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return s;
}

moe_status set_cuda_error(cudaError_t e, const char *what) {
    snprintf(t_err, sizeof(t_err), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
    return e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;
}

int num_sms(int device) {
    static int cache[64] = {0};
    if (device < 0 || device >= 64) return 148;
    if (!cache[device]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) v = 148;
        cache[device] = v;
    }
    return cache[device];
}

static int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return 0;
    return d;
}

// ------------------------------------------------------------------ fixed permutation scratch

// Scratch of moe_permute_static: a module-scope device array, so every device
// the library is loaded on has its own copy and nothing is allocated per call.
static __device__ __align__(256) uint8_t g_permute_scratch[MOE_PERMUTE_STATIC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
static void *g_permute_scratch_addr[kMaxScratchDevices];
static std::mutex g_permute_scratch_mu;

// Device address of the current device's scratch array, looked up on the first
// call on that device and kept.
static moe_status permute_scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxScratchDevices)
        return set_error(MOE_ERR_UNSUPPORTED, "device %d: fixed scratch covers devices 0..%d", dev,
                         kMaxScratchDevices - 1);
    std::lock_guard<std::mutex> lock(g_permute_scratch_mu);
    if (!g_permute_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress((void **)&p, g_permute_scratch);
        if (e != cudaSuccess) return set_cuda_error(e, "cudaGetSymbolAddress(permute scratch)");
        if (!p) return set_error(MOE_ERR_CUDA, "permute scratch has no device address");
        g_permute_scratch_addr[dev] = p;
    }
    *out = g_permute_scratch_addr[dev];
    return MOE_OK;
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

static PFN_encodeTiled_t encode_fn() {
    static PFN_encodeTiled_t fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled_t>(p);
    });
    return fn;
}

moe_status make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                     const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle sw) {
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return set_error(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (reinterpret_cast<uintptr_t>(base) & 15) return set_error(MOE_ERR_INVALID_ARG, "TMA base not 16-byte aligned");
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) {
            s[i] = strides_bytes[i];
            if (s[i] % 16) return set_error(MOE_ERR_INVALID_ARG, "TMA stride %llu not a multiple of 16",
                                            (unsigned long long)s[i]);
        }
    }
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(base), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(MOE_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

// ------------------------------------------------------------------ helpers

// True when p (possibly NULL) is not a multiple of `align` bytes.
static bool misaligned(const void *p, uintptr_t align) { return (reinterpret_cast<uintptr_t>(p) & (align - 1)) != 0; }

static int elem_bytes_x2(int fmt) {   // bytes per element, times 2
    return fmt == MOE_BF16 ? 4 : fmt == MOE_FP8_E4M3_K128 ? 2 : 1;
}

struct Strides {
    int64_t w13, w13s, w2, w2s;
};

static Strides default_strides(const moe_experts &x) {
    Strides s;
    if (x.layout == MOE_LAYOUT_TILED) {
        s.w13 = x.w13_estride ? x.w13_estride : (int64_t)prepacked_expert_bytes(x.fmt, x.H, x.I, 0);
        s.w2 = x.w2_estride ? x.w2_estride : (int64_t)prepacked_expert_bytes(x.fmt, x.H, x.I, 1);
        s.w13s = s.w2s = 0;
        return s;
    }
    const int64_t r13 = 2LL * x.I, r2 = x.H;
    s.w13 = x.w13_estride ? x.w13_estride : r13 * x.H * elem_bytes_x2(x.fmt) / 2;
    s.w13s = x.w13s_estride ? x.w13s_estride : r13 * scale_rowbytes(x.fmt, x.H);
    s.w2 = x.w2_estride ? x.w2_estride : r2 * x.I * elem_bytes_x2(x.fmt) / 2;
    s.w2s = x.w2s_estride ? x.w2s_estride : r2 * scale_rowbytes(x.fmt, x.I);
    return s;
}

static moe_status check_experts(const moe_experts *x) {
    if (!x) return set_error(MOE_ERR_INVALID_ARG, "experts is NULL");
    if (x->fmt < MOE_BF16 || x->fmt > MOE_NVFP4) return set_error(MOE_ERR_UNSUPPORTED, "unknown weight format %d", x->fmt);
    if (x->E <= 0 || x->E > kMaxExperts) return set_error(MOE_ERR_UNSUPPORTED, "E=%d outside 1..%d", x->E, kMaxExperts);
    if (x->H <= 0 || x->I <= 0 || x->H % 256 || x->I % 256)
        return set_error(MOE_ERR_UNSUPPORTED, "H=%d and I=%d must be positive multiples of 256", x->H, x->I);
    if (!x->w13 || !x->w2) return set_error(MOE_ERR_INVALID_ARG, "expert weights are NULL");
    if (x->layout != MOE_LAYOUT_STANDARD && x->layout != MOE_LAYOUT_TILED)
        return set_error(MOE_ERR_INVALID_ARG, "unknown layout %d", x->layout);
    if (x->layout == MOE_LAYOUT_STANDARD && x->fmt != MOE_BF16 && (!x->w13_scale || !x->w2_scale))
        return set_error(MOE_ERR_INVALID_ARG, "scale planes are NULL");
    if (x->fmt == MOE_NVFP4 && (!x->w13_tscale || !x->w2_tscale))
        return set_error(MOE_ERR_INVALID_ARG, "NVFP4 tensor scales are NULL");
    const Strides s = default_strides(*x);
    if ((s.w13 | s.w2 | s.w13s | s.w2s) & 15) return set_error(MOE_ERR_INVALID_ARG, "expert strides not 16-byte aligned");
    uintptr_t a = reinterpret_cast<uintptr_t>(x->w13) | reinterpret_cast<uintptr_t>(x->w2);
    if (x->layout == MOE_LAYOUT_STANDARD)
        a |= reinterpret_cast<uintptr_t>(x->w13_scale) | reinterpret_cast<uintptr_t>(x->w2_scale);
    if (a & 15) return set_error(MOE_ERR_INVALID_ARG, "expert arrays not 16-byte aligned");
    if (misaligned(x->w13_tscale, 4) || misaligned(x->w2_tscale, 4) || misaligned(x->expert_map, 4))
        return set_error(MOE_ERR_INVALID_ARG, "tensor scales and expert_map must be 4-byte aligned");
    return MOE_OK;
}

// Build the weight tensor map of one phase: 3D (K bytes|elements, rows, entries).
static moe_status weight_tmap(CUtensorMap *m, int fmt, const void *base, int rows, int K, int64_t estride,
                              int entries) {
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    CUtensorMapDataType dt;
    CUtensorMapSwizzle sw;
    if (fmt == MOE_BF16) {
        dt = CU_TENSOR_MAP_DATA_TYPE_UINT16;
        dims[0] = K;
        strides[0] = 2ULL * K;
        box[0] = 64;
        sw = CU_TENSOR_MAP_SWIZZLE_128B;
    } else if (fmt == MOE_FP8_E4M3_K128) {
        dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
        dims[0] = K;
        strides[0] = K;
        box[0] = 128;
        sw = CU_TENSOR_MAP_SWIZZLE_128B;
    } else {
        dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
        dims[0] = K / 2;
        strides[0] = K / 2;
        box[0] = 64;
        sw = CU_TENSOR_MAP_SWIZZLE_64B;
    }
    dims[1] = rows;
    dims[2] = entries;
    strides[1] = estride;
    box[1] = 64;
    box[2] = 1;
    return make_tmap(m, dt, 3, base, dims, strides, box, sw);
}

static moe_status act_tmap(CUtensorMap *m, const void *base, int rows, int K, int BN) {
    uint64_t dims[2] = {(uint64_t)K, (uint64_t)(rows > 0 ? rows : 1)};
    uint64_t strides[1] = {2ULL * K};
    uint32_t box[2] = {64, (uint32_t)BN};
    return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Scratch of the grouped FFN. Decoding path: h, bf16 [n][I] at offset 0.
// Block-scaled FP4 path: the activation blobs (four E2M1 planes and their scale
// atoms) of x and of h; NVFP4 also keeps h in bf16 at offset 0 and the per-row
// exponent offsets of x and h.
struct FfnWs {
    size_t h, re1, re2, a4, b1, b2, sched, total;
};

// h: bf16 [n][I] (the decoding paths' h buffer; NVFP4: h before its
// quantisation); re1, re2: NVFP4 per-row exponent offsets of x and h; a4: the A4
// tensor scale of x, then the partial maxima of |x|; b1, b2: activation blobs of
// x and h for the block-scaled FP4 path (four planes, or one in A4 form: the
// larger of the two sizes); sched: the block-scaled kernels' item claim counters (UP,
// DOWN), zeroed by the quantiser that runs first.
// bound: size the activation blobs for the largest need over all row counts up to n
// (the layout itself is always the one for n).
static FfnWs ffn_ws(int n, int H, int I, int E, bool bound = false) {
    FfnWs W;
    size_t o = 0;
    W.h = o; o += align_up((size_t)n * I * 2, 256);
    W.re1 = o; o += align_up((size_t)n * 4, 256);
    W.re2 = o; o += align_up((size_t)n * 4, 256);
    W.a4 = o; o += align_up((size_t)(1 + kA4Parts) * 4, 256);
    W.b1 = o; o += bound ? std::max(mx_blob_bound(n, H, E), a4_blob_bound(n, H, E))
                         : std::max(mx_blob_bytes(n, H, E), a4_blob_bytes(n, H, E));
    W.b2 = o; o += bound ? std::max(mx_blob_bound(n, I, E), a4_blob_bound(n, I, E))
                         : std::max(mx_blob_bytes(n, I, E), a4_blob_bytes(n, I, E));
    W.sched = o; o += 256;
    W.total = o;
    return W;
}

static size_t ffn_ws_bytes(int n_rows, int H, int I, int E) { return ffn_ws(n_rows, H, I, E).total; }

// Prepacked MXFP4 experts run the block-scaled FP4 path; prepacked NVFP4 runs it
// for token tiles of up to 16 rows (decode-sized batches) and the decoding
// bf16 tensor-core path, which reads the same blobs, for larger ones.
static bool use_bs(int fmt, int layout, int n_rows, int E) {
    if (layout != MOE_LAYOUT_TILED) return false;
    if (fmt == MOE_MXFP4) return true;
    return fmt == MOE_NVFP4 && choose_bn_mx(n_rows, E) <= 16;
}
static bool is_mx(const moe_experts &x, int n_rows) { return use_bs(x.fmt, x.layout, n_rows, x.E); }

// Activations already in the slot layout (the router wrote them; see RouterFuse).
struct SlotInput {
    const int32_t *cnt;
    uint8_t *blob;
    int T, mt;
    int32_t *cprefix;
};

// Block-scaled FP4 grouped FFN. The activations are quantised first: gathered
// from token rows x[sorted_pair[r] / k] (gather != 0) or read from x_perm; or
// they are in the slot layout already (slot non-null: MXFP4; no quantiser runs,
// and the router cleared the claim counters).
static moe_status mx_ffn_impl(const void *x_src, int gather, const int32_t *sorted_pair, int k, int n_rows,
                              const int32_t *offsets, const moe_experts *x, void *y_perm, int y_is_fp32, void *ws,
                              cudaStream_t st, const SlotInput *slot = nullptr) {
    if (n_rows == 0) return MOE_OK;
    const int E = x->E, H = x->H, I = x->I;
    const int fmt = x->fmt == MOE_NVFP4 ? kBsNv : kBsMx;
    const Strides s = default_strides(*x);
    const int BN = choose_bn_mx(n_rows, E);
    const int nsm = num_sms(current_device());
    const FfnWs W = ffn_ws(n_rows, H, I, E);
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    int32_t *re1 = reinterpret_cast<int32_t *>(b + W.re1), *re2 = reinterpret_cast<int32_t *>(b + W.re2);
    int *sched = reinterpret_cast<int *>(b + W.sched);
    moe_status r = MOE_OK;
    if (slot && fmt != kBsMx) return set_error(MOE_ERR_UNSUPPORTED, "the slot layout carries MXFP4 activations");
    if (!slot)
        r = launch_mx_quant(fmt, x_src, gather ? 1 : 0, sorted_pair, k, n_rows, H, offsets, E, BN, b + W.b1, re1, nsm,
                            st, sched);
    if (r != MOE_OK) return r;
    MxParams p;
    memset(&p, 0, sizeof(p));
    p.offsets = offsets;
    p.expert_map = x->expert_map;
    p.E = E;
    p.H = H;
    p.I = I;
    p.n_rows = n_rows;
    // ---- gate/up + SwiGLU; MXFP4 quantises h for the down pass in the epilogue
    p.K = H;
    p.m_tiles = I / 64;
    p.wbase = reinterpret_cast<const uint8_t *>(x->w13);
    p.w_estride = s.w13;
    p.bblob = b + W.b1;
    p.rowexp = re1;
    p.tscale = x->w13_tscale;
    p.bblob_out = b + W.b2;
    p.hout = b + W.h;
    p.sched = sched;
    if (slot) {
        p.bblob = slot->blob;
        p.slab_cnt = slot->cnt;
        p.slab_T = slot->T;
        p.slab_mt = slot->mt;
        p.cprefix = slot->cprefix;
        p.slab_wait = 1;   // the counts may come from the kernel just before
        // with at least 4 pairs per expert on average few experts are without rows (uniform
        // routing: under 2%), so an empty head tile rarely streams an unused expert's weights
        p.slab_head = n_rows >= 4 * E;
    }
    if ((r = launch_mx_phase(fmt, kPhaseUp, BN, p, nsm, st)) != MOE_OK) return r;
    if (fmt == kBsNv &&
        (r = launch_mx_quant(fmt, b + W.h, 2, nullptr, 1, n_rows, I, offsets, E, BN, b + W.b2, re2, nsm, st)) !=
            MOE_OK)
        return r;
    // ---- down projection
    p.K = I;
    p.m_tiles = H / 128;
    p.wbase = reinterpret_cast<const uint8_t *>(x->w2);
    p.w_estride = s.w2;
    p.bblob = b + W.b2;
    p.rowexp = re2;
    p.tscale = x->w2_tscale;
    p.bblob_out = nullptr;
    p.hout = nullptr;
    p.out = y_perm;
    p.out_fp32 = y_is_fp32;
    p.sched = sched + 1;
    p.slab_mt = 0;         // h is in compact tiles
    p.cprefix = nullptr;
    p.slab_wait = 0;       // the counts come from two kernels back
    // no head tiles: DOWN reads the counts before its wait, so its first weights go out early
    // anyway, and with three static items per CTA its head would span 28 experts (at decode
    // dims one of them often without rows, whose weights it would read for nothing)
    p.slab_head = 0;
    return launch_mx_phase(fmt, kPhaseDown, BN, p, nsm, st);
}

// A4 grouped FFN (activations in NVFP4 form; prepacked NVFP4 experts). The tensor
// scale of x comes from the rows the maxima are taken over: the token rows x [T][H]
// when gathering (every token appears k times among the pairs), else x_perm.
static moe_status a4_ffn_impl(const void *x_src, int gather, const void *amax_src, int64_t amax_elems,
                              const int32_t *sorted_pair, const int32_t *pair_row, int k, int n_rows,
                              const int32_t *offsets, const moe_experts *x, void *y_perm, int y_is_fp32, void *ws,
                              cudaStream_t st) {
    if (n_rows == 0) return MOE_OK;
    if (x->fmt != MOE_NVFP4 || x->layout != MOE_LAYOUT_TILED)
        return set_error(MOE_ERR_UNSUPPORTED, "A4 activations need prepacked NVFP4 experts");
    const int E = x->E, H = x->H, I = x->I;
    const Strides s = default_strides(*x);
    const int BN = choose_bn_a4(n_rows, E);
    const int nsm = num_sms(current_device());
    const FfnWs W = ffn_ws(n_rows, H, I, E);
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    float *xscale = reinterpret_cast<float *>(b + W.a4), *parts = xscale + 1;
    int *sched = reinterpret_cast<int *>(b + W.sched);
    moe_status r = launch_a4_amax(amax_src, amax_elems, parts, sched, st);
    if (r == MOE_OK && gather) {
        // token rows (amax_elems / H of them): each quantised once and placed in its k pairs' rows
        const int T = (int)(amax_elems / H);
        r = launch_a4_token_rows(x_src, T, H, k, pair_row, offsets, E, BN, parts, xscale, b + W.b1, nsm, st);
    } else if (r == MOE_OK) {
        r = launch_a4_quant(x_src, 2, sorted_pair, k, n_rows, H, offsets, E, BN, parts, xscale, b + W.b1, nsm, st);
    }
    if (r != MOE_OK) return r;
    MxParams p;
    memset(&p, 0, sizeof(p));
    p.offsets = offsets;
    p.expert_map = x->expert_map;
    p.E = E;
    p.H = H;
    p.I = I;
    p.n_rows = n_rows;
    // ---- gate/up + SwiGLU; the epilogue writes h in A4 form for the down pass
    p.K = H;
    p.m_tiles = I / 64;
    p.wbase = reinterpret_cast<const uint8_t *>(x->w13);
    p.w_estride = s.w13;
    p.bblob = b + W.b1;
    p.tscale = x->w13_tscale;
    p.bblob_out = b + W.b2;
    p.xscale = xscale;
    p.sched = sched;
    if ((r = launch_mx_phase(kBsNv, kPhaseUp, BN, p, nsm, st, 1)) != MOE_OK) return r;
    // ---- down projection
    p.K = I;
    p.m_tiles = H / 128;
    p.wbase = reinterpret_cast<const uint8_t *>(x->w2);
    p.w_estride = s.w2;
    p.bblob = b + W.b2;
    p.tscale = x->w2_tscale;
    p.bblob_out = nullptr;
    p.xscale = nullptr;
    p.out = y_perm;
    p.out_fp32 = y_is_fp32;
    p.sched = sched + 1;
    return launch_mx_phase(kBsNv, kPhaseDown, BN, p, nsm, st, 1);
}

// grouped FFN with explicit h buffer
static moe_status grouped_ffn_impl(const void *x_perm, int n_rows, const int32_t *offsets, const moe_experts *x,
                                   void *y_perm, int y_is_fp32, void *h, cudaStream_t st) {
    if (n_rows == 0) return MOE_OK;
    // prepacked MXFP4 has only the block-scaled path's blobs (use_bs always takes it)
    if (x->fmt == MOE_MXFP4 && x->layout == MOE_LAYOUT_TILED)
        return set_error(MOE_ERR_UNSUPPORTED, "prepacked MXFP4 runs on the block-scaled path only");
    const Strides s = default_strides(*x);
    const int nent = x->expert_map ? (int)(x->n_entries > 0 ? x->n_entries : x->E) : x->E;
    const int BN = choose_bn(n_rows, x->E);
    const int nsm = num_sms(current_device());
    CUtensorMap wmap, bmap;
    moe_status r;
    FfnParams p;
    memset(&p, 0, sizeof(p));
    p.offsets = offsets;
    p.expert_map = x->expert_map;
    p.E = x->E;
    p.H = x->H;
    p.I = x->I;
    p.n_rows = n_rows;
    const bool tiled = x->layout == MOE_LAYOUT_TILED;
    p.tiled = tiled;
    memset(&wmap, 0, sizeof(wmap));   // unused by the tiled kernels
    // ---- gate/up + SwiGLU
    if (tiled) {
        p.wbase = reinterpret_cast<const uint8_t *>(x->w13);
        p.w_estride = s.w13;
    } else if ((r = weight_tmap(&wmap, x->fmt, x->w13, 2 * x->I, x->H, s.w13, nent)) != MOE_OK) {
        return r;
    }
    if ((r = act_tmap(&bmap, x_perm, n_rows, x->H, BN)) != MOE_OK) return r;
    p.K = x->H;
    p.m_tiles = x->I / 64;
    p.scale_base = reinterpret_cast<const uint8_t *>(x->w13_scale);
    p.s_estride = s.w13s;
    p.s_rowbytes = scale_rowbytes(x->fmt, x->H);
    p.tscale = x->w13_tscale;
    p.out = h;
    p.out_fp32 = 0;
    if ((r = launch_ffn_phase(kPhaseUp, x->fmt, BN, wmap, bmap, p, nsm, st)) != MOE_OK) return r;
    // ---- down projection
    if (tiled) {
        p.wbase = reinterpret_cast<const uint8_t *>(x->w2);
        p.w_estride = s.w2;
    } else if ((r = weight_tmap(&wmap, x->fmt, x->w2, x->H, x->I, s.w2, nent)) != MOE_OK) {
        return r;
    }
    if ((r = act_tmap(&bmap, h, n_rows, x->I, BN)) != MOE_OK) return r;
    p.K = x->I;
    p.m_tiles = x->H / 128;
    p.scale_base = reinterpret_cast<const uint8_t *>(x->w2_scale);
    p.s_estride = s.w2s;
    p.s_rowbytes = scale_rowbytes(x->fmt, x->I);
    p.tscale = x->w2_tscale;
    p.out = y_perm;
    p.out_fp32 = y_is_fp32;
    return launch_ffn_phase(kPhaseDown, x->fmt, BN, wmap, bmap, p, nsm, st);
}

// workspace layout of moe_layer_forward
struct LayerWs {
    size_t router, idx, w, offsets, sorted, pair_row, perm, x_perm, h, y, slot, cprefix, total;
};

// Bytes of the slot layout's activation tiles (MXFP4, four planes) for a decode-sized
// batch: every expert gets room for T rows, ceil(T / BN) tiles. 0 where the layout is not
// used (large batches, or more than 64 MiB of tiles).
static size_t slot_blob_bytes(int T, int H, int E, int k) {
    // the router's 8 CTAs each write whole 256-wide stages of the rows: H % 2048 == 0
    if ((int64_t)T * k > 8192 || T > 256 || E > kMaxRouterExperts || H % (8 * kMxStageK)) return 0;
    const int BN = choose_bn_mx(T * k, E);
    const int64_t mt = (T + BN - 1) / BN;
    const int64_t bytes = (int64_t)E * mt * (H / kMxStageK) * bs_bblob_bytes(kBsMx, BN);
    return bytes <= (64ll << 20) ? align_up((size_t)bytes, 256) : 0;
}

// The largest slot region over all batches up to T (it depends on the tile height and
// stops above 256 tokens or 64 MiB).
static size_t slot_blob_bound(int T, int H, int E, int k) {
    size_t m = 0;
    for (int t = 1; t <= std::min(T, 256); ++t) m = std::max(m, slot_blob_bytes(t, H, E, k));
    return m;
}

// bound: every term that can shrink as T grows (the router's H split, the FP4
// activation blobs, the slot region) taken at its largest over all batches up to T,
// so the total never decreases with T. With bound set only the total is meaningful.
static LayerWs layer_ws(int T, int H, int I, int E, int k, int y32, bool bound = false) {
    LayerWs L;
    const size_t P = (size_t)T * k;
    size_t o = 0;
    L.router = o; o += align_up(bound ? router_ws_bound(T, H, E) : router_ws_bytes(T, H, E), 256);
    L.idx = o; o += align_up(P * 4, 256);
    L.w = o; o += align_up(P * 4, 256);
    L.offsets = o; o += align_up((size_t)(E + 1) * 4, 256);
    L.sorted = o; o += align_up(P * 4, 256);
    L.pair_row = o; o += align_up(P * 4, 256);
    L.perm = o; o += align_up(permute_ws_bytes(T, k, E), 256);
    L.x_perm = o; o += align_up(P * H * 2, 256);
    L.h = o; o += ffn_ws((int)P, H, I, E, bound).total;
    L.y = o; o += align_up(P * H * (y32 ? 4 : 2), 256);
    L.slot = o; o += bound ? slot_blob_bound(T, H, E, k) : slot_blob_bytes(T, H, E, k);
    L.cprefix = o; o += align_up((size_t)E * 4, 256);
    L.total = o;
    return L;
}

moe_status cache_resolve_and_map(struct expert_cache *c, int layer, const int32_t *idx, int T, int k,
                                 const moe_experts *shape, moe_experts *dev_view, cudaStream_t st);
void cache_compute_end(struct expert_cache *c, cudaStream_t st);
int cache_layout(const struct expert_cache *c);

// A kernel that waits, with the bounded wait of the FFN kernels, on an mbarrier that
// nothing completes; no copy or MMA is in flight. The wait gives up, flags error 1 and
// the kernel returns.
__global__ void __launch_bounds__(32) wait_selftest_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    mbar_wait(&bar, 0, &abort_flag);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_last_error_string(void) { return t_err; }

const char *moe_version(void) { return "libmoe 0.1 (sm_100a)"; }

uint64_t moe_kernel_launch_count(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

moe_status moe_device_error(int *code) {
    if (!code) return set_error(MOE_ERR_INVALID_ARG, "code is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return set_cuda_error(e, "device synchronize");
    int v = 0, z = 0;
    e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_dev_error, &z, sizeof(int));
    if (e != cudaSuccess) return set_cuda_error(e, "device error word");
    *code = v;
    return MOE_OK;
}

size_t moe_workspace_size(int T, int H, int I, int E, int k, int y_is_fp32, int af) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || (af != MOE_ACT_A16 && af != MOE_ACT_A4)) return 0;
    return layer_ws(T, H, I, E, k, y_is_fp32, true).total;
}

moe_status moe_route_topk(const void *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                          int k, int32_t *idx, float *w, float *logits, void *ws, size_t ws_bytes,
                          moe_stream_t stream) {
    if (T < 0 || H <= 0 || H % 8) return set_error(MOE_ERR_INVALID_ARG, "bad T=%d or H=%d", T, H);
    if (E < 1 || E > kMaxRouterExperts || k < 1 || k > kMaxTopK || k > E)
        return set_error(MOE_ERR_UNSUPPORTED, "router needs 1<=k<=%d, k<=E<=%d (E=%d k=%d)", kMaxTopK,
                         kMaxRouterExperts, E, k);
    if (T == 0) return MOE_OK;
    if (!x || !wr || !idx || !w || !ws) return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(wr)) & 15)
        return set_error(MOE_ERR_INVALID_ARG, "x and wr must be 16-byte aligned");
    if (misaligned(idx, 4) || misaligned(w, 4) || misaligned(logits, 4) || misaligned(bias, 4) || misaligned(ws, 16))
        return set_error(MOE_ERR_INVALID_ARG, "idx, w, logits and bias must be 4-byte aligned, ws 16-byte aligned");
    return launch_router(x, T, H, wr, wr_is_fp32, bias, E, k, idx, w, logits, ws, ws_bytes,
                         num_sms(current_device()), (cudaStream_t)stream);
}

moe_status moe_permute(const int32_t *idx, int T, int k, int E, const void *x, int H, int af, int32_t *offsets,
                       int32_t *sorted_pair, int32_t *pair_row, void *x_perm, void *ws, size_t ws_bytes,
                       moe_stream_t stream) {
    if (T < 0 || k < 1 || k > kMaxTopK || E < 1 || E > kMaxExperts)
        return set_error(MOE_ERR_INVALID_ARG, "bad T/k/E (%d %d %d)", T, k, E);
    if (af != MOE_ACT_A16 && af != MOE_ACT_A4) return set_error(MOE_ERR_INVALID_ARG, "unknown activation format %d", af);
    if (!offsets) return set_error(MOE_ERR_INVALID_ARG, "offsets is NULL");
    if (T > 0 && (!idx || !sorted_pair || !pair_row || (x_perm && !x) || !ws))
        return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (x_perm && (H <= 0 || H % 8)) return set_error(MOE_ERR_INVALID_ARG, "H must be a positive multiple of 8");
    if (x_perm && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_perm)) & 15))
        return set_error(MOE_ERR_INVALID_ARG, "x and x_perm must be 16-byte aligned");
    if (misaligned(idx, 4) || misaligned(offsets, 4) || misaligned(sorted_pair, 4) || misaligned(pair_row, 4) ||
        misaligned(ws, 16))
        return set_error(MOE_ERR_INVALID_ARG, "int32 arrays must be 4-byte aligned, ws 16-byte aligned");
    return launch_permute(idx, T, k, E, x, H, offsets, sorted_pair, pair_row, x_perm, ws, ws_bytes,
                          (cudaStream_t)stream, af == MOE_ACT_A4);
}

moe_status moe_permute_static(const int32_t *idx, int T, int k, int E, const void *x, int H, int32_t *offsets,
                              int32_t *sorted_pair, int32_t *pair_row, void *x_perm, moe_stream_t stream) {
    if (T < 0 || k < 1 || k > kMaxTopK || E < 1 || E > kMaxExperts)
        return set_error(MOE_ERR_INVALID_ARG, "bad T/k/E (%d %d %d)", T, k, E);
    const size_t need = permute_scratch_bytes(T, k, E);
    if (need > MOE_PERMUTE_STATIC_SCRATCH_BYTES)
        return set_error(MOE_ERR_UNSUPPORTED, "T=%d k=%d E=%d needs %zu scratch bytes; the fixed scratch holds %u", T,
                         k, E, need, (unsigned)MOE_PERMUTE_STATIC_SCRATCH_BYTES);
    void *scratch = nullptr;
    moe_status r = permute_scratch_address(&scratch);
    if (r != MOE_OK) return r;
    return moe_permute(idx, T, k, E, x, H, MOE_ACT_A16, offsets, sorted_pair, pair_row, x_perm, scratch,
                       MOE_PERMUTE_STATIC_SCRATCH_BYTES, stream);
}

moe_status moe_grouped_ffn(const void *x_perm, int n_rows, const int32_t *offsets, const moe_experts *experts,
                           int af, void *y_perm, int y_is_fp32, void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status r = check_experts(experts);
    if (r != MOE_OK) return r;
    if (af != MOE_ACT_A16 && af != MOE_ACT_A4) return set_error(MOE_ERR_INVALID_ARG, "unknown activation format %d", af);
    if (af == MOE_ACT_A4 && (experts->fmt != MOE_NVFP4 || experts->layout != MOE_LAYOUT_TILED))
        return set_error(MOE_ERR_UNSUPPORTED, "A4 activations need prepacked NVFP4 experts");
    if (n_rows < 0) return set_error(MOE_ERR_INVALID_ARG, "n_rows < 0");
    if (n_rows == 0) return MOE_OK;
    if (!x_perm || !offsets || !y_perm || !ws) return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    const size_t need = (af == MOE_ACT_A4 || is_mx(*experts, n_rows))
                            ? ffn_ws_bytes(n_rows, experts->H, experts->I, experts->E)
                            : align_up((size_t)n_rows * experts->I * 2, 256);
    if (ws_bytes < need) return set_error(MOE_ERR_OOM, "FFN workspace too small (%zu < %zu)", ws_bytes, need);
    if ((reinterpret_cast<uintptr_t>(x_perm) | reinterpret_cast<uintptr_t>(ws)) & 15)
        return set_error(MOE_ERR_INVALID_ARG, "x_perm and ws must be 16-byte aligned");
    if (misaligned(y_perm, 16) || misaligned(offsets, 4))
        return set_error(MOE_ERR_INVALID_ARG, "y_perm must be 16-byte aligned, offsets 4-byte aligned");
    if (af == MOE_ACT_A4)
        return a4_ffn_impl(x_perm, 0, x_perm, (int64_t)n_rows * experts->H, nullptr, nullptr, 1, n_rows, offsets, experts,
                           y_perm, y_is_fp32, ws, (cudaStream_t)stream);
    if (is_mx(*experts, n_rows))
        return mx_ffn_impl(x_perm, 0, nullptr, 1, n_rows, offsets, experts, y_perm, y_is_fp32, ws,
                           (cudaStream_t)stream);
    return grouped_ffn_impl(x_perm, n_rows, offsets, experts, y_perm, y_is_fp32, ws, (cudaStream_t)stream);
}

moe_status moe_dequantize(int fmt, const void *w, const void *scale, float tscale, int rows, int K, void *out,
                          moe_stream_t stream) {
    if (fmt < MOE_BF16 || fmt > MOE_NVFP4) return set_error(MOE_ERR_UNSUPPORTED, "unknown format %d", fmt);
    const int kq = fmt == MOE_FP8_E4M3_K128 ? 128 : fmt == MOE_MXFP4 ? 32 : fmt == MOE_NVFP4 ? 16 : 8;
    if (rows < 0 || K <= 0 || K % kq) return set_error(MOE_ERR_INVALID_ARG, "K=%d must be a multiple of %d", K, kq);
    if (rows == 0) return MOE_OK;
    if (!w || !out || (fmt != MOE_BF16 && !scale)) return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (fmt == MOE_FP8_E4M3_K128 && misaligned(scale, 4))
        return set_error(MOE_ERR_INVALID_ARG, "FP8 scales must be 4-byte aligned");
    if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(out)) & 15)
        return set_error(MOE_ERR_INVALID_ARG, "w and out must be 16-byte aligned");
    return launch_dequant(fmt, w, scale, tscale, rows, K, out, (cudaStream_t)stream);
}

size_t moe_prepacked_expert_bytes(int fmt, int H, int I, int which) {
    if (fmt < MOE_BF16 || fmt > MOE_NVFP4 || H <= 0 || I <= 0 || H % 256 || I % 256 || (which != 0 && which != 1))
        return 0;
    return prepacked_expert_bytes(fmt, H, I, which);
}

moe_status moe_prepack(const moe_experts *in, void *out_w13, void *out_w2, moe_stream_t stream) {
    moe_status r = check_experts(in);
    if (r != MOE_OK) return r;
    if (in->layout != MOE_LAYOUT_STANDARD || in->expert_map)
        return set_error(MOE_ERR_INVALID_ARG, "moe_prepack needs standard-layout experts without expert_map");
    if (!out_w13 || !out_w2 || ((reinterpret_cast<uintptr_t>(out_w13) | reinterpret_cast<uintptr_t>(out_w2)) & 15))
        return set_error(MOE_ERR_INVALID_ARG, "outputs must be non-NULL and 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    if ((r = launch_prepack(*in, 0, out_w13, (int64_t)prepacked_expert_bytes(in->fmt, in->H, in->I, 0), st)) != MOE_OK)
        return r;
    return launch_prepack(*in, 1, out_w2, (int64_t)prepacked_expert_bytes(in->fmt, in->H, in->I, 1), st);
}

moe_status moe_combine(const void *y_perm, int y_is_fp32, const int32_t *pair_row, const float *w, int T, int k,
                       int H, void *out, moe_stream_t stream) {
    if (T < 0 || k < 1 || k > kMaxTopK || H <= 0 || H % 8) return set_error(MOE_ERR_INVALID_ARG, "bad T/k/H");
    if (T == 0) return MOE_OK;
    if (!y_perm || !pair_row || !w || !out) return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(y_perm) | reinterpret_cast<uintptr_t>(out)) & 15)
        return set_error(MOE_ERR_INVALID_ARG, "y_perm and out must be 16-byte aligned");
    if (misaligned(pair_row, 4) || misaligned(w, 4))
        return set_error(MOE_ERR_INVALID_ARG, "pair_row and w must be 4-byte aligned");
    return launch_combine(y_perm, y_is_fp32, pair_row, w, T, k, H, out, (cudaStream_t)stream);
}

moe_status moe_layer_forward(const void *x, int T, const void *wr, int wr_is_fp32, const float *bias, int k,
                             const moe_experts *experts, int af, struct expert_cache *cache, int layer,
                             int y_is_fp32, void *out, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                             moe_stream_t stream) {
    if (!experts) return set_error(MOE_ERR_INVALID_ARG, "experts is NULL");
    const int E = experts->E, H = experts->H, I = experts->I;
    if (T < 0) return set_error(MOE_ERR_INVALID_ARG, "T < 0");
    if (af != MOE_ACT_A16 && af != MOE_ACT_A4) return set_error(MOE_ERR_INVALID_ARG, "unknown activation format %d", af);
    if (T == 0) return MOE_OK;
    if (k < 1 || k > kMaxTopK || k > E)
        return set_error(MOE_ERR_INVALID_ARG, "k=%d outside 1..min(%d, E=%d)", k, kMaxTopK, E);
    if (!cache) {
        moe_status r = check_experts(experts);
        if (r != MOE_OK) return r;
    } else if (experts->E <= 0 || H % 256 || I % 256) {
        return set_error(MOE_ERR_UNSUPPORTED, "bad layer shape");
    }
    if (!x || !wr || !out || !ws) return set_error(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (misaligned(bias, 4) || misaligned(idx_out, 4) || misaligned(w_out, 4) || misaligned(out, 16))
        return set_error(MOE_ERR_INVALID_ARG, "bias, idx_out and w_out must be 4-byte aligned, out 16-byte aligned");
    const LayerWs L = layer_ws(T, H, I, E, k, y_is_fp32);
    if (ws_bytes < L.total) return set_error(MOE_ERR_OOM, "workspace %zu < %zu bytes", ws_bytes, L.total);
    if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(MOE_ERR_INVALID_ARG, "ws must be 256-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(b + L.idx);
    float *w = w_out ? w_out : reinterpret_cast<float *>(b + L.w);
    int32_t *offsets = reinterpret_cast<int32_t *>(b + L.offsets);
    int32_t *sorted = reinterpret_cast<int32_t *>(b + L.sorted);
    int32_t *prow = reinterpret_cast<int32_t *>(b + L.pair_row);
    // The block-scaled FP4 path gathers the token rows itself while quantising them, so
    // it needs no x_perm, and for small batches the router kernel also permutes.
    const int layout = cache ? cache_layout(cache) : experts->layout;
    const bool a4 = af == MOE_ACT_A4;
    if (a4 && (experts->fmt != MOE_NVFP4 || layout != MOE_LAYOUT_TILED))
        return set_error(MOE_ERR_UNSUPPORTED, "A4 activations need prepacked NVFP4 experts");
    // both FP4-operand paths gather the token rows while quantising them (no x_perm)
    const bool mx = a4 || use_bs(experts->fmt, layout, T * k, E);
    moe_status r;
    int fused = 0;
    int32_t *slot_cnt = nullptr;   // the slot layout's row counts when the router wrote it
    if (mx) {
        if (H % 8 || E < 1 || E > kMaxRouterExperts || k < 1 || k > kMaxTopK || k > E)
            return set_error(MOE_ERR_UNSUPPORTED, "router needs 1<=k<=%d, k<=E<=%d (E=%d k=%d)", kMaxTopK,
                             kMaxRouterExperts, E, k);
        if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(wr)) & 15)
            return set_error(MOE_ERR_INVALID_ARG, "x and wr must be 16-byte aligned");
        RouterFuse fz{};
        fz.offsets = offsets;
        fz.sorted_pair = sorted;
        fz.pair_row = prow;
        // Decode-sized MXFP4 batches: the router writes the slot layout itself (pair rows by
        // atomic claims in per-expert slots, activation rows quantised straight into their
        // tiles), so neither the permutation nor the quantiser runs.
        if (!a4 && experts->fmt == MOE_MXFP4 && L.cprefix > L.slot && router_cluster_ok(T, H, E, wr_is_fp32, wr) &&
            (slot_cnt = route_slot_counts(st)) != nullptr) {
            const int BN = choose_bn_mx(T * k, E);
            fz.cnt = slot_cnt;
            fz.bslab = b + L.slot;
            fz.BN = BN;
            fz.mt = (T + BN - 1) / BN;
            fz.sched_zero = reinterpret_cast<int *>(b + L.h + ffn_ws(T * k, H, I, E).sched);
        }
        r = launch_router(x, T, H, wr, wr_is_fp32, bias, E, k, idx, w, nullptr, b + L.router, L.idx - L.router,
                          num_sms(current_device()), st, &fz, &fused);
        if (fused != 2) slot_cnt = nullptr;
    } else {
        r = moe_route_topk(x, T, H, wr, wr_is_fp32, bias, E, k, idx, w, nullptr, b + L.router, L.idx - L.router,
                           stream);
    }
    if (r != MOE_OK) return r;
    if (!fused) {
        r = moe_permute(idx, T, k, E, x, H, MOE_ACT_A16, offsets, sorted, prow, mx ? nullptr : b + L.x_perm,
                        b + L.perm, L.x_perm - L.perm, stream);
        if (r != MOE_OK) return r;
    }
    moe_experts view = *experts;
    if (cache) {
        r = cache_resolve_and_map(cache, layer, idx, T, k, experts, &view, st);
        if (r != MOE_OK) return r;
    }
    r = check_experts(&view);
    if (r == MOE_OK && !a4 && is_mx(view, T * k) != mx)
        r = set_error(MOE_ERR_INVALID_ARG, "cache layout differs from the layer's");
    const int BNs = choose_bn_mx(T * k, E);
    const SlotInput si{slot_cnt, b + L.slot, T, (T + BNs - 1) / BNs, reinterpret_cast<int32_t *>(b + L.cprefix)};
    if (r == MOE_OK) {
        if (a4)
            r = a4_ffn_impl(x, 1, x, (int64_t)T * H, sorted, prow, k, T * k, offsets, &view, b + L.y, y_is_fp32, b + L.h,
                            st);
        else if (mx)
            r = mx_ffn_impl(x, 1, sorted, k, T * k, offsets, &view, b + L.y, y_is_fp32, b + L.h, st,
                            slot_cnt ? &si : nullptr);
        else
            r = grouped_ffn_impl(b + L.x_perm, T * k, offsets, &view, b + L.y, y_is_fp32, b + L.h, st);
    }
    // the combine reads prow and w, written by the routing, before its wait for y; in the
    // slot layout it also maps the slot rows to y's rows and clears the counts
    if (r == MOE_OK)
        r = launch_combine(b + L.y, y_is_fp32, prow, w, T, k, H, out, st, 1, slot_cnt ? si.cprefix : nullptr, T,
                           slot_cnt, E);
    if (r != MOE_OK && slot_cnt) cudaMemsetAsync(slot_cnt, 0, sizeof(int32_t) * E, st);   // for the next call
    if (cache) cache_compute_end(cache, st);   // closes the call's timing record in every case
    return r;
}

moe_status moe_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns ? ns : kWaitLimitNs;
    cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "wait limit");
}

moe_status moe_selftest_wait(moe_stream_t stream) {
    count_launch();
    wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : set_cuda_error(e, "wait self-test launch");
}

}  // extern "C"
