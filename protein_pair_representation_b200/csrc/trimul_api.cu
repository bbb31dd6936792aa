// trimul_api.cu -- host side of the C ABI declared in include/trimul.h.
//
// Validates every call, owns the repacked layer weights, encodes the TMA tensor maps
// (driver entry point cuTensorMapEncodeTiled) and launches the three kernels of one
// update: K1 projection, K2 contraction, K3 output gate. There is no CPU or library
// fallback: anything outside the compiled set is reported as an error.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <new>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "kernels.h"
#include "sm100.cuh"
#include "trimul.h"

namespace trimul {
__device__ unsigned int g_device_error = 0;
}
// The offset of the stand-alone contraction, which has none.
static __device__ __align__(16) float g_zero_float[4] = {0.f, 0.f, 0.f, 0.f};

using namespace trimul;

struct trimul_layer {
    int c_z, c_h;
    float eps;
    bool has_bf16;               // tensor-core packing present
    void *mem;                   // single device allocation holding everything below
    // bf16 path
    uint16_t *k1_w;              // [4*c_h][c_z] packed, folded
    float4 *k1_vec;              // [2][c_h]
    uint16_t *k3_wo;             // [c_z][c_h] folded
    uint16_t *k3_wg;             // [c_z][c_z] folded
    float4 *k3_vec;              // [c_z]
    // K1's per-(batch, channel) sums of a and b and unmasked-pair counts, [65535 / c_h + 1][kAccStride]
    // (zero between forwards: the offsets kernel clears what it has read)
    unsigned long long *acc;
    // fp32 path
    F32Weights f32;
    // workspace
    void *ws;
    size_t ws_bytes;
    cudaEvent_t events[4];
    bool timing;
    bool skip_masked;            // find mask extents and leave out wholly masked tiles
    // valid lengths set by tri_mul_layer_set_valid_lengths: extents {L_b, L_b} on the device for
    // problems of vl_B x vl_N, and whether the rule chose to skip with them
    int *vl_ext;
    int64_t vl_B, vl_N;
    bool vl_skip;
};

// ------------------------------------------------------------------ error plumbing

static thread_local char g_last_error[512];

static trimul_status_t fail(trimul_status_t st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

namespace trimul {
// Lets other translation units of the library set the calling thread's error detail.
trimul_status_t set_last_error(trimul_status_t st, const char *msg) { return fail(st, "%s", msg); }
}  // namespace trimul

static trimul_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(TRIMUL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define TRY_CUDA(expr, what)                      \
    do {                                          \
        cudaError_t _e = (expr);                  \
        if (_e != cudaSuccess) return cuda_fail(_e, what); \
    } while (0)

// ------------------------------------------------------------------ device info

struct DeviceInfo {
    bool known;
    int major, minor, sms;
};
static DeviceInfo g_dev[64];
static std::mutex g_dev_mu;

static trimul_status_t device_info(DeviceInfo *out) {
    int dev = 0;
    TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(TRIMUL_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev[dev].known) {
        DeviceInfo d{};
        TRY_CUDA(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev), "attr major");
        TRY_CUDA(cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev), "attr minor");
        TRY_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev), "attr SMs");
        d.known = true;
        g_dev[dev] = d;
    }
    *out = g_dev[dev];
    return TRIMUL_OK;
}

static trimul_status_t require_sm100(DeviceInfo *d) {
    trimul_status_t st = device_info(d);
    if (st != TRIMUL_OK) return st;
    if (!(d->major == 10 && d->minor == 0))
        return fail(TRIMUL_ERR_UNSUPPORTED_DEVICE, "bf16 path needs compute capability 10.0, device is %d.%d", d->major,
                    d->minor);
    return TRIMUL_OK;
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// dims / box listed innermost first; strides are the byte strides of dims 1..rank-1.
static trimul_status_t make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *ptr,
                                const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                                CUtensorMapSwizzle sw, const char *what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(TRIMUL_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TRIMUL_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
    return TRIMUL_OK;
}

#define TRY(expr)                                 \
    do {                                          \
        trimul_status_t _s = (expr);              \
        if (_s != TRIMUL_OK) return _s;           \
    } while (0)

// Skipping by valid lengths is chosen when it leaves out at least this share of the dense work
// (measured on B200: the skipping instances and their tile tests cost a few percent; at B=1 N=512
// with 493 of 512 valid, 9% of the work, skipping did not pay; at B=4 N=256 with 162-237 valid,
// about 40%, it saved 8.5% of the time).
static constexpr double kSkipRule = 0.15;

// Batch elements the layer's channel sums have room for: B * c_h <= 65535 is enforced.
static int acc_batches(int c_h) { return 65535 / c_h + 1; }

// ------------------------------------------------------------------ validation helpers

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t dtype_size(trimul_dtype_t t) { return t == TRIMUL_F32 ? 4 : 2; }

static bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

static trimul_status_t check_pair(const trimul_pair_t *t, const char *name) {
    if (!t || !t->data) return fail(TRIMUL_ERR_INVALID_ARG, "%s: NULL tensor", name);
    if (t->dtype != TRIMUL_F32 && t->dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_INVALID_ARG, "%s: unknown dtype", name);
    if (t->B < 1 || t->N < 1 || t->C < 1) return fail(TRIMUL_ERR_INVALID_ARG, "%s: sizes must be positive", name);
    if (!aligned16(t->data)) return fail(TRIMUL_ERR_ALIGNMENT, "%s: pointer not 16-byte aligned", name);
    return TRIMUL_OK;
}

static size_t pair_bytes(const trimul_pair_t *t) {
    return (size_t)t->B * t->N * t->N * t->C * dtype_size(t->dtype);
}

// The size rules of z: they need no layer.
static trimul_status_t check_sizes(const trimul_pair_t *z) {
    TRY(check_pair(z, "z"));
    if (z->N < 8 || z->N % 8 != 0) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a positive multiple of 8", (long long)z->N);
    if (z->N > 16384) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld exceeds 16384", (long long)z->N);
    if (z->dtype == TRIMUL_BF16 && (long long)z->B * z->N * z->N / 128 > (1LL << 30))
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "problem too large: B * N^2 / 128 must not exceed 2^30");
    return TRIMUL_OK;
}

// The rules on out that need no layer: present, aligned, z's shape, fp32 on the fp32 path, apart from z.
static trimul_status_t check_out(const trimul_pair_t *z, const trimul_pair_t *out) {
    TRY(check_pair(out, "out"));
    if (out->B != z->B || out->N != z->N || out->C != z->C) return fail(TRIMUL_ERR_INVALID_ARG, "out shape differs from z");
    if (z->dtype == TRIMUL_F32 && out->dtype != TRIMUL_F32) return fail(TRIMUL_ERR_INVALID_ARG, "fp32 path writes fp32 out");
    if (overlap(out->data, pair_bytes(out), z->data, pair_bytes(z))) return fail(TRIMUL_ERR_INVALID_ARG, "out overlaps z");
    return TRIMUL_OK;
}

static trimul_status_t check_problem(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L) {
    TRY(check_sizes(z));
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    if (z->C != L->c_z) return fail(TRIMUL_ERR_INVALID_ARG, "z has %lld channels, layer expects c_z=%d", (long long)z->C, L->c_z);
    // the contraction's limit (B * c_h planes), checked here so that no stage has run when it fails
    if ((long long)z->B * L->c_h > 65535)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "B*c_h=%lld exceeds 65535", (long long)z->B * L->c_h);
    if (mask && !aligned16(mask)) return fail(TRIMUL_ERR_ALIGNMENT, "mask pointer not 16-byte aligned");
    if (z->dtype == TRIMUL_BF16 && !L->has_bf16)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "bf16 path supports (c_z, c_h) = (128,128) or (384,128); layer is (%d,%d)", L->c_z, L->c_h);
    return TRIMUL_OK;
}

// ------------------------------------------------------------------ layer

extern "C" trimul_status_t tri_mul_layer_create(const trimul_weights_desc_t *w, void *stream, trimul_layer_t **out) {
    if (!w || !out) return fail(TRIMUL_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    if (w->dtype != TRIMUL_F32 && w->dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_INVALID_ARG, "unknown weight dtype");
    if (w->c_z < 32 || w->c_h < 32 || w->c_z % 32 || w->c_h % 32 || w->c_z > 512 || w->c_h > 512)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "c_z and c_h must be multiples of 32 in [32, 512]");
    if (!(w->eps > 0.f)) return fail(TRIMUL_ERR_INVALID_ARG, "eps must be positive");
    if (!w->w_ag || !w->w_ap || !w->w_bg || !w->w_bp || !w->w_g || !w->w_o)
        return fail(TRIMUL_ERR_INVALID_ARG, "projection weights may not be NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int cz = w->c_z, ch = w->c_h;
    const int src_bf16 = w->dtype == TRIMUL_BF16;

    trimul_layer *L = new trimul_layer();
    memset(L, 0, sizeof(*L));
    L->c_z = cz;
    L->c_h = ch;
    L->eps = w->eps;
    L->has_bf16 = (ch == kHidden) && (cz == 128 || cz == 384);

    // carve one allocation
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = (off + bytes + 255) & ~size_t(255); return o; };
    size_t o_k1w = 0, o_k1v = 0, o_k3o = 0, o_k3g = 0, o_k3v = 0, o_acc = 0, acc_bytes = 0;
    if (L->has_bf16) {
        o_k1w = take((size_t)4 * ch * cz * 2);
        o_k1v = take((size_t)2 * ch * sizeof(float4));
        o_k3o = take((size_t)cz * ch * 2);
        o_k3g = take((size_t)cz * cz * 2);
        o_k3v = take((size_t)cz * sizeof(float4));
        acc_bytes = (size_t)acc_batches(ch) * kAccStride * sizeof(unsigned long long);
        o_acc = take(acc_bytes);
    }
    const size_t o_lig = take(cz * 4), o_lib = take(cz * 4);
    const size_t o_wag = take((size_t)ch * cz * 4), o_wap = take((size_t)ch * cz * 4);
    const size_t o_wbg = take((size_t)ch * cz * 4), o_wbp = take((size_t)ch * cz * 4);
    const size_t o_bag = take(ch * 4), o_bap = take(ch * 4), o_bbg = take(ch * 4), o_bbp = take(ch * 4);
    const size_t o_wgT = take((size_t)cz * cz * 4), o_bg = take(cz * 4);
    const size_t o_log = take(ch * 4), o_lob = take(ch * 4);
    const size_t o_woT = take((size_t)ch * cz * 4), o_bo = take(cz * 4);
    cudaError_t e = cudaMalloc(&L->mem, off);
    if (e != cudaSuccess) {
        delete L;
        return cuda_fail(e, "cudaMalloc(layer)");
    }
    uint8_t *m = reinterpret_cast<uint8_t *>(L->mem);

    auto conv = [&](const void *src, size_t o, int R, int K, int tr, const float **dst) -> cudaError_t {
        if (!src) { *dst = nullptr; return cudaSuccess; }
        *dst = reinterpret_cast<float *>(m + o);
        return to_f32_launch(src, src_bf16, reinterpret_cast<float *>(m + o), R, K, tr, st);
    };
    cudaError_t ce = cudaSuccess;
#define CONV(src, o, R, K, tr, dst) if (ce == cudaSuccess) ce = conv(src, o, R, K, tr, dst)
    CONV(w->ln_in_g, o_lig, 1, cz, 0, &L->f32.ln_in_g);
    CONV(w->ln_in_b, o_lib, 1, cz, 0, &L->f32.ln_in_b);
    CONV(w->w_ag, o_wag, ch, cz, 0, &L->f32.w_ag);
    CONV(w->w_ap, o_wap, ch, cz, 0, &L->f32.w_ap);
    CONV(w->w_bg, o_wbg, ch, cz, 0, &L->f32.w_bg);
    CONV(w->w_bp, o_wbp, ch, cz, 0, &L->f32.w_bp);
    CONV(w->b_ag, o_bag, 1, ch, 0, &L->f32.b_ag);
    CONV(w->b_ap, o_bap, 1, ch, 0, &L->f32.b_ap);
    CONV(w->b_bg, o_bbg, 1, ch, 0, &L->f32.b_bg);
    CONV(w->b_bp, o_bbp, 1, ch, 0, &L->f32.b_bp);
    CONV(w->w_g, o_wgT, cz, cz, 1, &L->f32.w_gT);
    CONV(w->b_g, o_bg, 1, cz, 0, &L->f32.b_g);
    CONV(w->ln_out_g, o_log, 1, ch, 0, &L->f32.ln_out_g);
    CONV(w->ln_out_b, o_lob, 1, ch, 0, &L->f32.ln_out_b);
    CONV(w->w_o, o_woT, cz, ch, 1, &L->f32.w_oT);
    CONV(w->b_o, o_bo, 1, cz, 0, &L->f32.b_o);
#undef CONV

    if (ce == cudaSuccess && L->has_bf16) {
        L->k1_w = reinterpret_cast<uint16_t *>(m + o_k1w);
        L->k1_vec = reinterpret_cast<float4 *>(m + o_k1v);
        L->k3_wo = reinterpret_cast<uint16_t *>(m + o_k3o);
        L->k3_wg = reinterpret_cast<uint16_t *>(m + o_k3g);
        L->k3_vec = reinterpret_cast<float4 *>(m + o_k3v);
        L->acc = reinterpret_cast<unsigned long long *>(m + o_acc);
        ce = cudaMemsetAsync(m + o_acc, 0, acc_bytes, st);
        const int ncol = k1_ncol(cz);
        const void *srcs[2][2] = {{w->w_ag, w->w_ap}, {w->w_bg, w->w_bp}};
        const void *biases[2][2] = {{w->b_ag, w->b_ap}, {w->b_bg, w->b_bp}};
        float *vecf = reinterpret_cast<float *>(L->k1_vec);
        for (int o = 0; o < 2 && ce == cudaSuccess; ++o)
            for (int kind = 0; kind < 2 && ce == cudaSuccess; ++kind) {
                FoldArgs fa{};
                fa.w = srcs[o][kind];
                fa.gamma = w->ln_in_g;
                fa.beta = w->ln_in_b;
                fa.bias = biases[o][kind];
                fa.src_bf16 = src_bf16;
                fa.R = ch;
                fa.K = cz;
                fa.dst = L->k1_w;
                fa.row_mode = k1_row_mode(cz);
                // both K1 kernels evaluate sigmoid(g) as 0.5 + 0.5 tanh(g / 2) and take the
                // gate rows pre-scaled by 1/2 (exact in bf16)
                fa.scale = kind == 0 ? 0.5f : 1.0f;
                fa.operand = o;
                fa.kind = kind;
                fa.ncol = ncol;
                fa.cpg = ncol / 2;
                fa.gpo = k1_groups(cz) / 2;
                fa.sum_out = vecf + (size_t)o * ch * 4 + kind * 2;
                fa.shift_out = vecf + (size_t)o * ch * 4 + kind * 2 + 1;
                fa.out_stride = 4;
                ce = fold_launch(fa, st);
            }
        float *v3 = reinterpret_cast<float *>(L->k3_vec);
        if (ce == cudaSuccess) {
            FoldArgs fa{};
            fa.w = w->w_o; fa.gamma = w->ln_out_g; fa.beta = w->ln_out_b; fa.bias = w->b_o;
            fa.src_bf16 = src_bf16; fa.R = cz; fa.K = ch; fa.dst = L->k3_wo; fa.dst_f16 = 1; fa.row_mode = 0;
            fa.sum_out = v3 + 0; fa.shift_out = v3 + 1; fa.out_stride = 4;
            ce = fold_launch(fa, st);
        }
        if (ce == cudaSuccess) {
            FoldArgs fa{};
            fa.w = w->w_g; fa.gamma = w->ln_in_g; fa.beta = w->ln_in_b; fa.bias = w->b_g;
            fa.src_bf16 = src_bf16; fa.R = cz; fa.K = cz; fa.dst = L->k3_wg; fa.row_mode = 0;
            fa.sum_out = v3 + 2; fa.shift_out = v3 + 3; fa.out_stride = 4;
            ce = fold_launch(fa, st);
        }
    }
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
    if (ce != cudaSuccess) {
        cudaFree(L->mem);
        delete L;
        return cuda_fail(ce, "layer packing");
    }
    *out = L;
    return TRIMUL_OK;
}

extern "C" void tri_mul_layer_destroy(trimul_layer_t *L) {
    if (!L) return;
    if (L->mem) cudaFree(L->mem);
    if (L->vl_ext) cudaFree(L->vl_ext);
    delete L;
}

static size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

static size_t ws_plane_bytes(int64_t B, int64_t N, int c_h, trimul_dtype_t dt) {
    return align256((size_t)B * c_h * N * N * dtype_size(dt));
}

// After the three planes: the mask extents {R_b, C_b} (int32), then the offset of the stored x
// (fp32, one value per batch element repeated over its c_h channel planes).
static size_t ws_ext_bytes(int64_t B) { return align256((size_t)B * 2 * sizeof(int)); }
static size_t ws_q_bytes(int64_t B, int c_h) { return align256((size_t)B * c_h * sizeof(float)); }

static size_t ws_total_bytes(const trimul_layer_t *L, int64_t B, int64_t N, trimul_dtype_t dt) {
    return 3 * ws_plane_bytes(B, N, L->c_h, dt) + ws_ext_bytes(B) + ws_q_bytes(B, L->c_h);
}

extern "C" size_t tri_mul_workspace_bytes(const trimul_layer_t *L, int64_t B, int64_t N, trimul_dtype_t dt) {
    if (!L || B < 1 || N < 1 || (dt != TRIMUL_F32 && dt != TRIMUL_BF16)) return 0;
    return ws_total_bytes(L, B, N, dt);
}

extern "C" trimul_status_t tri_mul_layer_bind_workspace(trimul_layer_t *L, void *ws, size_t bytes) {
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    if (ws && !aligned16(ws)) return fail(TRIMUL_ERR_ALIGNMENT, "workspace not 16-byte aligned");
    L->ws = ws;
    L->ws_bytes = ws ? bytes : 0;
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_layer_set_timing_events(trimul_layer_t *L, void *const *events) {
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    if (!events) {
        L->timing = false;
        return TRIMUL_OK;
    }
    for (int i = 0; i < 4; ++i) {
        if (!events[i]) return fail(TRIMUL_ERR_INVALID_ARG, "timing event %d is NULL", i);
        L->events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
    }
    L->timing = true;
    return TRIMUL_OK;
}

extern "C" int tri_mul_kernels_per_forward(void) { return 4; }

extern "C" trimul_status_t tri_mul_layer_set_mask_skipping(trimul_layer_t *L, int enable) {
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    L->skip_masked = enable != 0;
    return TRIMUL_OK;
}

// ------------------------------------------------------------------ kernel drivers

static int grid_for(int sms, long long work_units, int multiple) {
    long long g = work_units < sms ? work_units : sms;
    g = (g / multiple) * multiple;
    if (g < multiple) g = multiple;
    return (int)g;
}

// K1 on B x R x N pairs (R rows of N: the whole pair tensor, R = N, or one shard's rows).
static trimul_status_t run_project_bf16(const trimul_layer_t *L, const void *z, const void *mask, void *a, void *b,
                                        int B, int R, int N, cudaStream_t st, const int *ext, unsigned long long *acc) {
    DeviceInfo d;
    TRY(require_sm100(&d));
    const uint64_t NN = (uint64_t)R * N;
    const int cz = L->c_z, ch = L->c_h;
    K1Args p{};
    const int tp = k1_tile_pairs(cz);
    if (cz == 128) {
        // z [B][NN][128] viewed as {64 channels, NN pairs, 2 halves, B}: one copy brings both
        // 64-channel halves of one CTA's 64 pairs of a tile, laid out [half][pair][64]
        uint64_t dims[4] = {64, NN, 2, (uint64_t)B};
        uint64_t strides[3] = {(uint64_t)cz * 2, 128, NN * cz * 2};
        uint32_t box[4] = {64, 64, 2, 1};
        TRY(make_map(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, z, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K1 z"));
    } else {
        uint64_t dims[3] = {(uint64_t)cz, NN, (uint64_t)B};
        uint64_t strides[2] = {(uint64_t)cz * 2, NN * cz * 2};
        uint32_t box[3] = {64, (uint32_t)tp, 1};
        TRY(make_map(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, z, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K1 z"));
    }
    {
        uint64_t dims[2] = {(uint64_t)cz, (uint64_t)4 * ch};
        uint64_t strides[1] = {(uint64_t)cz * 2};
        uint32_t box[2] = {64, (uint32_t)k1_ncol(cz)};
        TRY(make_map(&p.tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L->k1_w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K1 w"));
    }
    {
        uint64_t dims[3] = {NN, (uint64_t)ch, (uint64_t)B};
        uint64_t strides[2] = {NN * 2, (uint64_t)ch * NN * 2};
        // c_z = 128: each warp of the channel-lane kernel stores a [32 channels][64 pairs] block
        // through a 128B swizzle; c_z = 384: pair-lane kernel stores [channels][128 pairs] rows
        // without swizzle
        const bool cm = k1_row_mode(cz) == 2;
        uint32_t box[3] = {cm ? 64u : 128u, cm ? 32u : (uint32_t)k1_channels_per_warpgroup(cz), 1};
        const CUtensorMapSwizzle sw = cm ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
        TRY(make_map(&p.tm_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, a, dims, strides, box, sw, "K1 a"));
        TRY(make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, b, dims, strides, box, sw, "K1 b"));
    }
    p.mask = reinterpret_cast<const uint16_t *>(mask);
    p.vec = L->k1_vec;
    p.B = B;
    p.N = N;
    p.NN = (long long)NN;
    p.tiles_per_batch = (int)((NN + tp - 1) / tp);
    p.eps = L->eps;
    p.ext = ext;
    p.rowdiv = host_rowdiv((uint64_t)N / 8);
    p.acc = acc;
    const int G = k1_groups(cz);
    const int grid = grid_for(d.sms, (long long)G * B * p.tiles_per_batch, G);
    TRY_CUDA(k1_launch(cz, p, grid, st), "K1 launch");
    return TRIMUL_OK;
}

static trimul_status_t run_contract_tc(const void *a, const void *b, void *x, int64_t BC, int N, bool incoming,
                                       bool f16, float x_scale, cudaStream_t st, const int *ext, int C,
                                       const float *xoff, int xoff_stride) {
    DeviceInfo d;
    TRY(require_sm100(&d));
    K2Args p{};
    const CUtensorMapDataType dt = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    uint64_t dims[3] = {(uint64_t)N, (uint64_t)N, (uint64_t)BC};
    uint64_t strides[2] = {(uint64_t)N * 2, (uint64_t)N * N * 2};
    if (!incoming) {
        uint32_t boxa[3] = {64, 128, 1}, boxb[3] = {64, 128, 1};   // one CTA's half of a pair tile each
        TRY(make_map(&p.tm_a, dt, 3, a, dims, strides, boxa, CU_TENSOR_MAP_SWIZZLE_128B, "K2 a"));
        TRY(make_map(&p.tm_b, dt, 3, b, dims, strides, boxb, CU_TENSOR_MAP_SWIZZLE_128B, "K2 b"));
    } else {
        uint32_t box[3] = {64, 64, 1};
        TRY(make_map(&p.tm_a, dt, 3, a, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K2 a"));
        TRY(make_map(&p.tm_b, dt, 3, b, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K2 b"));
    }
    {
        uint32_t box[3] = {64, 128, 1};
        TRY(make_map(&p.tm_x, dt, 3, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K2 x"));
    }
    p.f16 = f16;
    p.x_scale = x_scale;
    p.xoff = xoff;
    p.xoff_stride = xoff_stride;
    p.ext = ext;
    p.C = C;
    p.BC = (int)BC;
    p.N = N;
    p.m_tiles = (N + 255) / 256;        // 256-row tiles of a CTA pair
    p.n_tiles = (N + 255) / 256;
    p.k_chunks = (N + 63) / 64;
    p.incoming = incoming;
    TRY_CUDA(k2_launch(p, 0, st), "K2 launch");
    return TRIMUL_OK;
}

// K3 on B x R x N pairs (as run_project_bf16).
static trimul_status_t run_output_bf16(const trimul_layer_t *L, const void *z, const void *mask, const void *x,
                                       float x_scale, void *out, bool out_f32, bool residual, int B, int R, int N,
                                       cudaStream_t st, const int *ext) {
    DeviceInfo d;
    TRY(require_sm100(&d));
    const uint64_t NN = (uint64_t)R * N;
    const int cz = L->c_z, ch = L->c_h;
    K3Args p{};
    {
        // x [B][c_h][N*N] viewed as [B][N*N/64 blocks][c_h][64 pairs], so that one copy brings
        // the two 64-pair MN blocks of a 128-pair tile for 64 channels (N*N is a multiple of 64)
        uint64_t dims[4] = {64, (uint64_t)ch, NN / 64, (uint64_t)B};
        uint64_t strides[3] = {NN * 2, 128, (uint64_t)ch * NN * 2};
        uint32_t box[4] = {64, 64, 2, 1};
        TRY(make_map(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K3 x"));
    }
    {
        uint64_t dims[3] = {(uint64_t)cz, NN, (uint64_t)B};
        uint64_t strides[2] = {(uint64_t)cz * 2, NN * cz * 2};
        uint32_t box[3] = {64, 128, 1};
        TRY(make_map(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, z, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K3 z"));
    }
    {
        uint64_t dims[2] = {(uint64_t)ch, (uint64_t)cz};
        uint64_t strides[1] = {(uint64_t)ch * 2};
        uint32_t box[2] = {64, 128};
        TRY(make_map(&p.tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, L->k3_wo, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K3 wo"));
    }
    {
        uint64_t dims[2] = {(uint64_t)cz, (uint64_t)cz};
        uint64_t strides[1] = {(uint64_t)cz * 2};
        uint32_t box[2] = {64, 128};
        TRY(make_map(&p.tm_wg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L->k3_wg, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K3 wg"));
    }
    {
        const uint64_t es = out_f32 ? 4 : 2;
        uint64_t dims[3] = {(uint64_t)cz, NN, (uint64_t)B};
        uint64_t strides[2] = {(uint64_t)cz * es, NN * cz * es};
        uint32_t box[3] = {out_f32 ? 32u : 64u, 32, 1};   // one warp's 32 pair rows
        TRY(make_map(&p.tm_out, out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims,
                     strides, box, CU_TENSOR_MAP_SWIZZLE_128B, "K3 out"));
    }
    p.mask = reinterpret_cast<const uint16_t *>(mask);
    p.vec = L->k3_vec;
    p.B = B;
    p.N = N;
    p.NN = (long long)NN;
    p.tiles_per_batch = (int)((NN + 127) / 128);
    p.eps = L->eps;
    p.eps_x = L->eps * x_scale * x_scale;
    p.zres = residual ? reinterpret_cast<const uint16_t *>(z) : nullptr;
    p.ext = residual ? nullptr : ext;        // with a residual a masked pair copies z: nothing is skipped
    p.rowdiv = host_rowdiv((uint64_t)N / 8);
    const int G = k3_groups(cz);
    const int grid = grid_for(d.sms, (long long)G * B * p.tiles_per_batch, G);
    TRY_CUDA(k3_launch(cz, out_f32, p, grid, st), "K3 launch");
    return TRIMUL_OK;
}

// ------------------------------------------------------------------ public entry points

static trimul_status_t project_impl(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L, void *a_out,
                                    void *b_out, const int *ext, unsigned long long *acc, void *stream) {
    TRY(check_problem(z, mask, L));
    if (!a_out || !b_out) return fail(TRIMUL_ERR_INVALID_ARG, "a_out / b_out NULL");
    if (!aligned16(a_out) || !aligned16(b_out)) return fail(TRIMUL_ERR_ALIGNMENT, "a_out / b_out not 16-byte aligned");
    const size_t plane = (size_t)z->B * L->c_h * z->N * z->N * dtype_size(z->dtype);
    if (overlap(a_out, plane, b_out, plane) || overlap(a_out, plane, z->data, pair_bytes(z)) ||
        overlap(b_out, plane, z->data, pair_bytes(z)))
        return fail(TRIMUL_ERR_INVALID_ARG, "a_out, b_out and z overlap");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (z->dtype == TRIMUL_BF16)
        return run_project_bf16(L, z->data, mask, a_out, b_out, (int)z->B, (int)z->N, (int)z->N, st, ext, acc);
    TRY_CUDA(f32_project_launch(reinterpret_cast<const float *>(z->data), reinterpret_cast<const float *>(mask), L->f32,
                                L->c_z, L->c_h, (int)z->B, (int)z->N, L->eps, reinterpret_cast<float *>(a_out),
                                reinterpret_cast<float *>(b_out), st),
             "fp32 projection launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_project(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L, void *a_out,
                                           void *b_out, void *stream) {
    return project_impl(z, mask, L, a_out, b_out, nullptr, nullptr, stream);
}

extern "C" float tri_mul_contract_scale(int64_t N) {
    if (N < 1) return 0.f;
    int lg = 0;
    while ((int64_t(1) << lg) < N) ++lg;       // ceil(log2 N)
    return ldexpf(1.0f, -((lg + 1) / 2));       // 2^-ceil(log2(N) / 2)
}

// q: per (batch, channel) offsets subtracted from x_scale * x before rounding, or nullptr (none)
static trimul_status_t contract_impl(const void *a, const void *b, void *x, int64_t B, int64_t C, int64_t N,
                                     trimul_dtype_t dtype, trimul_direction_t dir, float x_scale, const int *ext,
                                     const float *q, void *stream) {
    if (!a || !b || !x) return fail(TRIMUL_ERR_INVALID_ARG, "NULL tensor");
    if (dtype != TRIMUL_F32 && dtype != TRIMUL_BF16 && dtype != TRIMUL_F16) return fail(TRIMUL_ERR_INVALID_ARG, "unknown dtype");
    if (!(x_scale > 0.f) || !(x_scale < 3.0e38f)) return fail(TRIMUL_ERR_INVALID_ARG, "x_scale must be positive and finite");
    if (dir != TRIMUL_OUTGOING && dir != TRIMUL_INCOMING) return fail(TRIMUL_ERR_INVALID_ARG, "unknown direction");
    if (B < 1 || C < 1) return fail(TRIMUL_ERR_INVALID_ARG, "B and C must be positive");
    if (N < 8 || N % 8 || N > 16384) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a multiple of 8 in [8, 16384]", (long long)N);
    if (B * C > 65535) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "B*C=%lld exceeds 65535", (long long)(B * C));
    if (!aligned16(a) || !aligned16(b) || !aligned16(x)) return fail(TRIMUL_ERR_ALIGNMENT, "pointer not 16-byte aligned");
    const size_t bytes = (size_t)B * C * N * N * dtype_size(dtype);
    if (overlap(x, bytes, a, bytes) || overlap(x, bytes, b, bytes)) return fail(TRIMUL_ERR_INVALID_ARG, "x overlaps a or b");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype != TRIMUL_F32) {
        static float *zero_dev[64];                 // one zero float per device for the offset-free call
        const float *xo = q;
        if (!xo) {
            int dev = 0;
            TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
            if (dev < 0 || dev >= 64) return fail(TRIMUL_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
            {
                std::lock_guard<std::mutex> lk(g_dev_mu);
                if (!zero_dev[dev]) {
                    void *pz = nullptr;
                    TRY_CUDA(cudaGetSymbolAddress(&pz, g_zero_float), "zero offset address");
                    zero_dev[dev] = reinterpret_cast<float *>(pz);
                }
                xo = zero_dev[dev];
            }
        }
        return run_contract_tc(a, b, x, B * C, (int)N, dir == TRIMUL_INCOMING, dtype == TRIMUL_F16, x_scale, st, ext,
                               (int)C, xo, q ? 1 : 0);
    }
    TRY_CUDA(f32_contract_launch(reinterpret_cast<const float *>(a), reinterpret_cast<const float *>(b),
                                 reinterpret_cast<float *>(x), (int)(B * C), (int)N, dir == TRIMUL_INCOMING, x_scale, st),
             "fp32 contraction launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_contract(const void *a, const void *b, void *x, int64_t B, int64_t C, int64_t N,
                                            trimul_dtype_t dtype, trimul_direction_t dir, float x_scale, void *stream) {
    return contract_impl(a, b, x, B, C, N, dtype, dir, x_scale, nullptr, nullptr, stream);
}

static trimul_status_t output_gate_impl(const trimul_pair_t *z, const void *mask, const void *x, float x_scale,
                                        const trimul_layer_t *L, trimul_pair_t *out, bool residual, const int *ext,
                                        void *stream) {
    TRY(check_sizes(z));
    TRY(check_out(z, out));
    TRY(check_problem(z, mask, L));
    if (!(x_scale > 0.f) || !(x_scale < 3.0e38f)) return fail(TRIMUL_ERR_INVALID_ARG, "x_scale must be positive and finite");
    if (!x) return fail(TRIMUL_ERR_INVALID_ARG, "x is NULL");
    if (!aligned16(x)) return fail(TRIMUL_ERR_ALIGNMENT, "x not 16-byte aligned");
    const size_t xbytes = (size_t)z->B * L->c_h * z->N * z->N * dtype_size(z->dtype);
    if (overlap(out->data, pair_bytes(out), x, xbytes)) return fail(TRIMUL_ERR_INVALID_ARG, "out overlaps x");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (z->dtype == TRIMUL_BF16)
        return run_output_bf16(L, z->data, mask, x, x_scale, out->data, out->dtype == TRIMUL_F32, residual, (int)z->B,
                               (int)z->N, (int)z->N, st, ext);
    TRY_CUDA(f32_output_launch(reinterpret_cast<const float *>(z->data), reinterpret_cast<const float *>(mask),
                               reinterpret_cast<const float *>(x), L->f32, L->c_z, L->c_h, (int)z->B, (int)z->N, L->eps,
                               L->eps * x_scale * x_scale, residual, reinterpret_cast<float *>(out->data), st),
             "fp32 output launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_output_gate(const trimul_pair_t *z, const void *mask, const void *x, float x_scale,
                                               const trimul_layer_t *L, trimul_pair_t *out, void *stream) {
    return output_gate_impl(z, mask, x, x_scale, L, out, false, nullptr, stream);
}

namespace trimul {
// One update with its intermediates in `ws` (ws_bytes long; the layer's bound workspace, or the
// no-allocation array). Every argument rule is checked before anything is launched: the sizes of
// z, then out, then the layer, then the buffer. timing: record the layer's timing events.
// check_only: run every check that does not need the buffer's address (ws_ptr is ignored) and
// return without touching the device.
trimul_status_t forward_buffers(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L,
                                trimul_direction_t dir, trimul_pair_t *out, bool residual, void *ws_ptr,
                                size_t ws_bytes, bool timing, void *stream, bool check_only, const int *given_ext) {
    TRY(check_sizes(z));
    TRY(check_out(z, out));
    if (dir != TRIMUL_OUTGOING && dir != TRIMUL_INCOMING) return fail(TRIMUL_ERR_INVALID_ARG, "unknown direction");
    TRY(check_problem(z, mask, L));
    const size_t plane = ws_plane_bytes(z->B, z->N, L->c_h, z->dtype);
    const size_t need = ws_total_bytes(L, z->B, z->N, z->dtype);
    if ((!check_only && !ws_ptr) || ws_bytes < need)
        return fail(TRIMUL_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu available", need,
                    (check_only || ws_ptr) ? ws_bytes : (size_t)0);
    if (check_only) return TRIMUL_OK;
    if (!aligned16(ws_ptr)) return fail(TRIMUL_ERR_ALIGNMENT, "workspace not 16-byte aligned");
    if (overlap(out->data, pair_bytes(out), ws_ptr, need) || overlap(z->data, pair_bytes(z), ws_ptr, need))
        return fail(TRIMUL_ERR_INVALID_ARG, "z or out overlaps the workspace");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(ws_ptr);
    void *a = ws, *b = ws + plane, *x = ws + 2 * plane;
    const bool tc = z->dtype == TRIMUL_BF16;
    uint8_t *aux = ws + 3 * plane;
    // tensor-core path with a mask: the mask's extents let the kernels leave out wholly masked
    // tiles. They come from the caller (given_ext), from the layer's valid lengths when they fit
    // this problem and the rule chose skipping, or, with mask skipping switched on, from a pass
    // over the mask into the workspace.
    const int *ext = nullptr;
    float *q = reinterpret_cast<float *>(aux + ws_ext_bytes(z->B));
    if (tc && mask) {
        if (given_ext) {
            ext = given_ext;
        } else if (L->vl_ext && L->vl_B == z->B && L->vl_N == z->N) {
            ext = L->vl_skip ? L->vl_ext : nullptr;
        } else if (L->skip_masked) {
            int *e = reinterpret_cast<int *>(aux);
            TRY_CUDA(mask_extents_launch(reinterpret_cast<const uint16_t *>(mask), (int)z->B, (int)z->N,
                                         host_rowdiv((uint64_t)z->N / 8), e, st),
                     "mask extents launch");
            ext = e;
        }
    }
    timing = timing && L->timing;
    if (timing) TRY_CUDA(cudaEventRecord(L->events[0], st), "event record");
    TRY(project_impl(z, mask, L, a, b, ext, tc ? L->acc : nullptr, stream));
    const float x_scale = tc ? tri_mul_contract_scale(z->N) : 1.0f;
    // the offset of the stored x from K1's channel sums (the fp32 path stores x as it is)
    if (tc) TRY_CUDA(xoffsets_launch(L->acc, (int)z->B, L->c_h, x_scale, q, st), "offsets launch");
    if (timing) TRY_CUDA(cudaEventRecord(L->events[1], st), "event record");
    TRY(contract_impl(a, b, x, z->B, L->c_h, z->N, tc ? TRIMUL_F16 : TRIMUL_F32, dir, x_scale, ext, tc ? q : nullptr, stream));
    if (timing) TRY_CUDA(cudaEventRecord(L->events[2], st), "event record");
    TRY(output_gate_impl(z, mask, x, x_scale, L, out, residual, ext, stream));
    if (timing) TRY_CUDA(cudaEventRecord(L->events[3], st), "event record");
    return TRIMUL_OK;
}

}  // namespace trimul

static trimul_status_t forward_impl(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L,
                                    trimul_direction_t dir, trimul_pair_t *out, bool residual, void *stream) {
    return forward_buffers(z, mask, L, dir, out, residual, L ? L->ws : nullptr, L ? L->ws_bytes : 0, true, stream, false,
                           nullptr);
}

extern "C" trimul_status_t tri_mul_forward(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L,
                                           trimul_direction_t dir, trimul_pair_t *out, void *stream) {
    return forward_impl(z, mask, L, dir, out, false, stream);
}

extern "C" trimul_status_t tri_mul_forward_residual(const trimul_pair_t *z, const void *mask, const trimul_layer_t *L,
                                                    trimul_direction_t dir, trimul_pair_t *out, void *stream) {
    return forward_impl(z, mask, L, dir, out, true, stream);
}

// ------------------------------------------------------------------ row-sharded update

// A slab of rows: rows [row0, row0 + R) of a [B, N, N, C] pair tensor, stored [B, R, N, C].
static trimul_status_t check_rows(const trimul_rows_t *t, const char *name) {
    if (!t || !t->data) return fail(TRIMUL_ERR_INVALID_ARG, "%s: NULL tensor", name);
    if (t->dtype != TRIMUL_BF16 && t->dtype != TRIMUL_F32) return fail(TRIMUL_ERR_INVALID_ARG, "%s: unknown dtype", name);
    if (t->B < 1 || t->R < 1 || t->N < 1 || t->C < 1) return fail(TRIMUL_ERR_INVALID_ARG, "%s: sizes must be positive", name);
    if (!aligned16(t->data)) return fail(TRIMUL_ERR_ALIGNMENT, "%s: pointer not 16-byte aligned", name);
    return TRIMUL_OK;
}

static size_t rows_bytes(const trimul_rows_t *t) { return (size_t)t->B * t->R * t->N * t->C * dtype_size(t->dtype); }

// The size rules of a shard (no layer needed): the tensor-core path, N a multiple of 128 in
// [128, 16384], the rows a multiple of 128 starting at a multiple of 128 inside [0, N).
static trimul_status_t check_shard_sizes(const trimul_rows_t *z) {
    TRY(check_rows(z, "z"));
    if (z->dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "a row-sharded update takes a bf16 z");
    if (z->N < 128 || z->N % 128 != 0 || z->N > 16384)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a multiple of 128 in [128, 16384]", (long long)z->N);
    if (z->R % 128 != 0 || z->row0 % 128 != 0 || z->row0 < 0 || z->row0 + z->R > z->N)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "shard rows [%lld, %lld) must be whole 128-row blocks inside [0, %lld)",
                    (long long)z->row0, (long long)(z->row0 + z->R), (long long)z->N);
    if ((long long)z->B * z->R * z->N / 128 > (1LL << 30))
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "problem too large: B * R * N / 128 must not exceed 2^30");
    return TRIMUL_OK;
}

static trimul_status_t check_shard_layer(const trimul_rows_t *z, const void *mask, const trimul_layer_t *L) {
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    if (z->C != L->c_z) return fail(TRIMUL_ERR_INVALID_ARG, "z has %lld channels, layer expects c_z=%d", (long long)z->C, L->c_z);
    if (!L->has_bf16)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "bf16 path supports (c_z, c_h) = (128,128) or (384,128); layer is (%d,%d)", L->c_z, L->c_h);
    if ((long long)z->B * L->c_h > 65535)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "B*c_h=%lld exceeds 65535", (long long)z->B * L->c_h);
    if (mask && !aligned16(mask)) return fail(TRIMUL_ERR_ALIGNMENT, "mask pointer not 16-byte aligned");
    return TRIMUL_OK;
}

static size_t shard_x_bytes(const trimul_layer_t *L, int64_t B, int64_t R, int64_t N) {
    return align256((size_t)B * L->c_h * R * N * 2);
}

static size_t shard_ws_bytes(const trimul_layer_t *L, int64_t B, int64_t R, int64_t N) {
    return shard_x_bytes(L, B, R, N) + ws_q_bytes(B, L->c_h);
}

extern "C" size_t tri_mul_shard_workspace_bytes(const trimul_layer_t *L, int64_t B, int64_t R, int64_t N) {
    if (!L || B < 1 || R < 1 || N < 1) return 0;
    return shard_ws_bytes(L, B, R, N);
}

static trimul_status_t check_shard_workspace(const trimul_rows_t *z, const trimul_layer_t *L) {
    const size_t need = shard_ws_bytes(L, z->B, z->R, z->N);
    if (!L->ws || L->ws_bytes < need)
        return fail(TRIMUL_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu bound", need, L->ws ? L->ws_bytes : (size_t)0);
    if (overlap(z->data, rows_bytes(z), L->ws, need)) return fail(TRIMUL_ERR_INVALID_ARG, "z overlaps the workspace");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_shard_project(const trimul_rows_t *z, const void *mask, const trimul_layer_t *L,
                                                 void *a_out, void *b_out, void *stream) {
    TRY(check_shard_sizes(z));
    TRY(check_shard_layer(z, mask, L));
    if (!a_out || !b_out) return fail(TRIMUL_ERR_INVALID_ARG, "a_out / b_out NULL");
    if (!aligned16(a_out) || !aligned16(b_out)) return fail(TRIMUL_ERR_ALIGNMENT, "a_out / b_out not 16-byte aligned");
    const size_t plane = (size_t)z->B * L->c_h * z->R * z->N * 2;
    if (overlap(a_out, plane, b_out, plane) || overlap(a_out, plane, z->data, rows_bytes(z)) ||
        overlap(b_out, plane, z->data, rows_bytes(z)))
        return fail(TRIMUL_ERR_INVALID_ARG, "a_out, b_out and z overlap");
    TRY(check_shard_workspace(z, L));
    const size_t need = shard_ws_bytes(L, z->B, z->R, z->N);
    if (overlap(a_out, plane, L->ws, need) || overlap(b_out, plane, L->ws, need))
        return fail(TRIMUL_ERR_INVALID_ARG, "a_out / b_out overlap the workspace");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *q = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(L->ws) + shard_x_bytes(L, z->B, z->R, z->N));
    TRY(run_project_bf16(L, z->data, mask, a_out, b_out, (int)z->B, (int)z->R, (int)z->N, st, nullptr, L->acc));
    // the offset of this shard's stored x, from its own rows' channel sums
    TRY_CUDA(xoffsets_launch(L->acc, (int)z->B, L->c_h, tri_mul_contract_scale(z->N), q, st), "offsets launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_shard_finish(const trimul_rows_t *z, const void *mask, const trimul_layer_t *L,
                                                trimul_direction_t dir, int G, const int64_t *shard_row0,
                                                const void *const *a_shards, const void *const *b_shards,
                                                trimul_rows_t *out, void *stream) {
    TRY(check_shard_sizes(z));
    TRY(check_rows(out, "out"));
    if (out->B != z->B || out->R != z->R || out->N != z->N || out->C != z->C || out->row0 != z->row0)
        return fail(TRIMUL_ERR_INVALID_ARG, "out rows differ from z's");
    if (overlap(out->data, rows_bytes(out), z->data, rows_bytes(z))) return fail(TRIMUL_ERR_INVALID_ARG, "out overlaps z");
    if (dir != TRIMUL_OUTGOING && dir != TRIMUL_INCOMING) return fail(TRIMUL_ERR_INVALID_ARG, "unknown direction");
    if (G < 1 || G > kMaxShards) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "G=%d shards: 1 to %d are supported", G, kMaxShards);
    if (!shard_row0 || !a_shards || !b_shards) return fail(TRIMUL_ERR_INVALID_ARG, "shard table is NULL");
    if (shard_row0[0] != 0 || shard_row0[G] != z->N)
        return fail(TRIMUL_ERR_INVALID_ARG, "shard rows must start at 0 and end at N");
    int self = -1;
    for (int g = 0; g < G; ++g) {
        if (shard_row0[g + 1] <= shard_row0[g] || shard_row0[g] % 128 != 0)
            return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "shard %d: rows must be ascending whole 128-row blocks", g);
        if (shard_row0[g] == z->row0 && shard_row0[g + 1] - shard_row0[g] == z->R) self = g;
        if (!b_shards[g] || !aligned16(b_shards[g]) || (dir == TRIMUL_INCOMING && (!a_shards[g] || !aligned16(a_shards[g]))))
            return fail(TRIMUL_ERR_INVALID_ARG, "shard %d: a / b missing or not 16-byte aligned", g);
    }
    if (self < 0) return fail(TRIMUL_ERR_INVALID_ARG, "z's rows are not one of the shards");
    if (!a_shards[self] || !aligned16(a_shards[self])) return fail(TRIMUL_ERR_INVALID_ARG, "this shard's a is missing or misaligned");
    TRY(check_shard_layer(z, mask, L));
    TRY(check_shard_workspace(z, L));
    if (overlap(out->data, rows_bytes(out), L->ws, shard_ws_bytes(L, z->B, z->R, z->N)))
        return fail(TRIMUL_ERR_INVALID_ARG, "out overlaps the workspace");
    DeviceInfo d;
    TRY(require_sm100(&d));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(L->ws);
    void *x = ws;
    const float *q = reinterpret_cast<const float *>(ws + shard_x_bytes(L, z->B, z->R, z->N));
    const int64_t BC = z->B * L->c_h;
    const bool incoming = dir == TRIMUL_INCOMING;
    K2ShardArgs sa{};
    K2Args &p = sa.base;
    const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    for (int g = 0; g < G; ++g) {
        const uint64_t Rg = (uint64_t)(shard_row0[g + 1] - shard_row0[g]);
        uint64_t dims[3] = {(uint64_t)z->N, Rg, (uint64_t)BC};
        uint64_t strides[2] = {(uint64_t)z->N * 2, Rg * z->N * 2};
        uint32_t boxb[3] = {64, incoming ? 64u : 128u, 1};
        TRY(make_map(&sa.tm_sb[g], dt, 3, b_shards[g], dims, strides, boxb, CU_TENSOR_MAP_SWIZZLE_128B, "K2 shard b"));
        if (incoming) {
            uint32_t boxa[3] = {64, 64, 1};
            TRY(make_map(&sa.tm_sa[g], dt, 3, a_shards[g], dims, strides, boxa, CU_TENSOR_MAP_SWIZZLE_128B, "K2 shard a"));
        }
        sa.row0[g] = (int)shard_row0[g];
    }
    sa.row0[G] = (int)z->N;
    sa.G = G;
    sa.i0 = (int)z->row0;
    {
        uint64_t dims[3] = {(uint64_t)z->N, (uint64_t)z->R, (uint64_t)BC};
        uint64_t strides[2] = {(uint64_t)z->N * 2, (uint64_t)z->R * z->N * 2};
        uint32_t boxa[3] = {64, 128, 1};
        TRY(make_map(&p.tm_a, dt, 3, a_shards[self], dims, strides, boxa, CU_TENSOR_MAP_SWIZZLE_128B, "K2 shard own a"));
        TRY(make_map(&p.tm_x, dt, 3, x, dims, strides, boxa, CU_TENSOR_MAP_SWIZZLE_128B, "K2 shard x"));
        p.tm_b = sa.tm_sb[0];
    }
    const float x_scale = tri_mul_contract_scale(z->N);
    p.f16 = true;
    p.x_scale = x_scale;
    p.xoff = q;
    p.xoff_stride = 1;
    p.ext = nullptr;
    p.C = L->c_h;
    p.BC = (int)BC;
    p.N = (int)z->N;
    p.m_tiles = (int)((z->R + 255) / 256);   // 256-row tiles of a CTA pair
    p.n_tiles = (int)((z->N + 255) / 256);
    p.k_chunks = (int)(z->N / 64);
    p.incoming = incoming;
    TRY_CUDA(k2_shard_launch(sa, 0, st), "K2 shard launch");
    return run_output_bf16(L, z->data, mask, x, x_scale, out->data, out->dtype == TRIMUL_F32, false, (int)z->B, (int)z->R,
                           (int)z->N, st, nullptr);
}

// ------------------------------------------------------------------ pair update and its graph

static trimul_status_t check_pair_update(const trimul_pair_t *z, const trimul_layer_t *Lo, const trimul_layer_t *Li,
                                         const trimul_pair_t *z_mid, const trimul_pair_t *out) {
    if (!Lo || !Li) return fail(TRIMUL_ERR_INVALID_ARG, "NULL layer");
    TRY(check_pair(z, "z"));
    TRY(check_pair(z_mid, "z_mid"));
    TRY(check_pair(out, "out"));
    if (z_mid->B != z->B || z_mid->N != z->N || z_mid->C != z->C || z_mid->dtype != z->dtype)
        return fail(TRIMUL_ERR_INVALID_ARG, "z_mid must have z's shape and dtype");
    if (overlap(z_mid->data, pair_bytes(z_mid), z->data, pair_bytes(z)) ||
        overlap(out->data, pair_bytes(out), z_mid->data, pair_bytes(z_mid)))
        return fail(TRIMUL_ERR_INVALID_ARG, "z, z_mid and out must not overlap");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_pair_update(const trimul_pair_t *z, const void *mask, const trimul_layer_t *Lo,
                                               const trimul_layer_t *Li, trimul_pair_t *z_mid, trimul_pair_t *out,
                                               void *stream) {
    TRY(check_pair_update(z, Lo, Li, z_mid, out));
    // with mask skipping on and no valid lengths set, one pass over the (shared) mask serves both
    // updates: its extents go to the first layer's workspace and both forwards read them there
    const int *ext = nullptr;
    const bool lengths = Lo->vl_ext && Lo->vl_B == z->B && Lo->vl_N == z->N;
    if (z->dtype == TRIMUL_BF16 && mask && Lo->skip_masked && !lengths) {
        TRY(forward_buffers(z, mask, Lo, TRIMUL_OUTGOING, z_mid, true, Lo->ws, Lo->ws_bytes, false, stream, true, nullptr));
        if (!aligned16(mask)) return fail(TRIMUL_ERR_ALIGNMENT, "mask pointer not 16-byte aligned");
        int *e = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(Lo->ws) + 3 * ws_plane_bytes(z->B, z->N, Lo->c_h, z->dtype));
        TRY_CUDA(mask_extents_launch(reinterpret_cast<const uint16_t *>(mask), (int)z->B, (int)z->N,
                                     host_rowdiv((uint64_t)z->N / 8), e, reinterpret_cast<cudaStream_t>(stream)),
                 "mask extents launch");
        ext = e;
    }
    TRY(forward_buffers(z, mask, Lo, TRIMUL_OUTGOING, z_mid, true, Lo->ws, Lo->ws_bytes, true, stream, false, ext));
    return forward_buffers(z_mid, mask, Li, TRIMUL_INCOMING, out, true, Li->ws, Li->ws_bytes, true, stream, false,
                           Li->skip_masked || Li == Lo ? ext : nullptr);
}

// ------------------------------------------------------------------ mask extents and valid lengths

extern "C" trimul_status_t tri_mul_mask_extents(const void *mask, int64_t B, int64_t N, trimul_dtype_t dtype,
                                                int32_t *extents, void *stream) {
    if (!mask || !extents) return fail(TRIMUL_ERR_INVALID_ARG, "mask / extents NULL");
    if (dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "extents are found for bf16 masks");
    if (B < 1 || B > 65535) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "B=%lld outside [1, 65535]", (long long)B);
    if (N < 8 || N % 8 || N > 16384) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a multiple of 8 in [8, 16384]", (long long)N);
    if (!aligned16(mask) || !aligned16(extents)) return fail(TRIMUL_ERR_ALIGNMENT, "mask / extents not 16-byte aligned");
    DeviceInfo d;
    TRY(require_sm100(&d));
    TRY_CUDA(mask_extents_launch(reinterpret_cast<const uint16_t *>(mask), (int)B, (int)N, host_rowdiv((uint64_t)N / 8),
                                 reinterpret_cast<int *>(extents), reinterpret_cast<cudaStream_t>(stream)),
             "mask extents launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_forward_extents(const trimul_pair_t *z, const void *mask, const int32_t *extents,
                                                   const trimul_layer_t *L, trimul_direction_t dir, trimul_pair_t *out,
                                                   void *stream) {
    if (!mask || !extents) return fail(TRIMUL_ERR_INVALID_ARG, "mask / extents NULL");
    if (!aligned16(extents)) return fail(TRIMUL_ERR_ALIGNMENT, "extents not 16-byte aligned");
    if (z && z->dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "extents are used on the bf16 path");
    return forward_buffers(z, mask, L, dir, out, false, L ? L->ws : nullptr, L ? L->ws_bytes : 0, true, stream, false,
                           reinterpret_cast<const int *>(extents));
}

// The share of one layer's dense work (its flops at N) that skipping by the valid lengths leaves
// out: K1 and K3 scale with the valid pairs (L_b^2), K2 with L_b^3.
extern "C" double tri_mul_skip_saving(const int64_t *lengths, int64_t B, int64_t N, int32_t c_z, int32_t c_h) {
    if (!lengths || B < 1 || N < 1 || c_z < 1 || c_h < 1) return 0.0;
    const double n = (double)N;
    const double dense_pairs = 2.0 * c_z * 4.0 * c_h + 2.0 * c_z * (c_z + c_h);   // K1 + K3 per pair
    double dense = 0.0, kept = 0.0;
    for (int64_t b = 0; b < B; ++b) {
        const double l = (double)(lengths[b] < 0 ? 0 : (lengths[b] > N ? N : lengths[b]));
        dense += n * n * dense_pairs + 2.0 * c_h * n * n * n;
        kept += l * l * dense_pairs + 2.0 * c_h * l * l * l;
    }
    return dense > 0.0 ? 1.0 - kept / dense : 0.0;
}

extern "C" trimul_status_t tri_mul_layer_set_valid_lengths(trimul_layer_t *L, const int64_t *lengths, int64_t B,
                                                           int64_t N, int32_t *skipping_out) {
    if (!L) return fail(TRIMUL_ERR_INVALID_ARG, "layer is NULL");
    if (skipping_out) *skipping_out = 0;
    if (!lengths) {                          // clear
        L->vl_B = L->vl_N = 0;
        L->vl_skip = false;
        return TRIMUL_OK;
    }
    if (B < 1 || N < 8 || N % 8 || N > 16384 || B * L->c_h > 65535)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "B=%lld N=%lld outside the supported sizes", (long long)B, (long long)N);
    for (int64_t b = 0; b < B; ++b)
        if (lengths[b] < 0 || lengths[b] > N) return fail(TRIMUL_ERR_INVALID_ARG, "length %lld of batch element %lld outside [0, N]",
                                                          (long long)lengths[b], (long long)b);
    if (L->vl_ext && L->vl_B < B) {
        cudaFree(L->vl_ext);
        L->vl_ext = nullptr;
    }
    if (!L->vl_ext) TRY_CUDA(cudaMalloc(&L->vl_ext, (size_t)B * 2 * sizeof(int)), "cudaMalloc(valid lengths)");
    int *host = new (std::nothrow) int[2 * B];
    if (!host) return fail(TRIMUL_ERR_INVALID_ARG, "out of host memory");
    for (int64_t b = 0; b < B; ++b) host[2 * b] = host[2 * b + 1] = (int)lengths[b];
    cudaError_t e = cudaMemcpy(L->vl_ext, host, (size_t)B * 2 * sizeof(int), cudaMemcpyHostToDevice);
    delete[] host;
    TRY_CUDA(e, "copy valid lengths");
    L->vl_B = B;
    L->vl_N = N;
    L->vl_skip = tri_mul_skip_saving(lengths, B, N, L->c_z, L->c_h) >= kSkipRule;
    if (skipping_out) *skipping_out = L->vl_skip ? 1 : 0;
    return TRIMUL_OK;
}

struct trimul_graph {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
};

extern "C" trimul_status_t tri_mul_pair_update_graph_create(const trimul_pair_t *z, const void *mask,
                                                            const trimul_layer_t *Lo, const trimul_layer_t *Li,
                                                            trimul_pair_t *z_mid, trimul_pair_t *out,
                                                            trimul_graph_t **graph_out) {
    if (!graph_out) return fail(TRIMUL_ERR_INVALID_ARG, "graph_out is NULL");
    *graph_out = nullptr;
    TRY(check_pair_update(z, Lo, Li, z_mid, out));
    if (Lo->timing || Li->timing) return fail(TRIMUL_ERR_INVALID_ARG, "switch the layers' timing events off before capture");
    cudaStream_t cs = nullptr;
    TRY_CUDA(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking), "capture stream");
    trimul_status_t st = TRIMUL_OK;
    cudaGraph_t g = nullptr;
    // relaxed: the first launch of a kernel may still set its shared-memory attribute while
    // the capture is open (no call made here synchronizes)
    cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed);
    if (e != cudaSuccess) {
        st = fail(TRIMUL_ERR_CUDA, "cudaStreamBeginCapture: %s", cudaGetErrorString(e));
    } else {
        st = tri_mul_pair_update(z, mask, Lo, Li, z_mid, out, cs);
        e = cudaStreamEndCapture(cs, &g);             // always end the capture, even after an error
        if (st == TRIMUL_OK && e != cudaSuccess) st = fail(TRIMUL_ERR_CUDA, "cudaStreamEndCapture: %s", cudaGetErrorString(e));
    }
    cudaGraphExec_t ex = nullptr;
    if (st == TRIMUL_OK) {
        e = cudaGraphInstantiateWithFlags(&ex, g, 0);
        if (e != cudaSuccess) st = fail(TRIMUL_ERR_CUDA, "cudaGraphInstantiate: %s", cudaGetErrorString(e));
    }
    cudaStreamDestroy(cs);
    if (st != TRIMUL_OK) {
        if (ex) cudaGraphExecDestroy(ex);
        if (g) cudaGraphDestroy(g);
        return st;
    }
    trimul_graph_t *h = new (std::nothrow) trimul_graph_t{g, ex};
    if (!h) {
        cudaGraphExecDestroy(ex);
        cudaGraphDestroy(g);
        return fail(TRIMUL_ERR_INVALID_ARG, "out of host memory");
    }
    *graph_out = h;
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_graph_launch(const trimul_graph_t *graph, void *stream) {
    if (!graph) return fail(TRIMUL_ERR_INVALID_ARG, "graph is NULL");
    TRY_CUDA(cudaGraphLaunch(graph->exec, reinterpret_cast<cudaStream_t>(stream)), "graph launch");
    return TRIMUL_OK;
}

extern "C" void tri_mul_graph_destroy(trimul_graph_t *graph) {
    if (!graph) return;
    cudaGraphExecDestroy(graph->exec);
    cudaGraphDestroy(graph->graph);
    delete graph;
}

// One CTA waits, with the kernels' bounded wait, on an mbarrier that nothing arrives at:
// the wait gives up after its limit (about one second), raises the abort flag and the device
// error word, and the kernel exits normally.
__global__ void selftest_bounded_wait_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, kErrTimeoutEpilogue);
    __syncthreads();
}

extern "C" trimul_status_t tri_mul_selftest_bounded_wait(void *stream) {
    DeviceInfo d;
    TRY(require_sm100(&d));
    selftest_bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    TRY_CUDA(cudaGetLastError(), "self-test launch");
    return TRIMUL_OK;
}

extern "C" trimul_status_t tri_mul_check_device_status(void) {
    TRY_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    unsigned int v = 0, zero = 0;
    TRY_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)), "read device error word");
    if (v) {
        TRY_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)), "clear device error word");
        if (v == (unsigned int)kErrRange)
            return fail(TRIMUL_ERR_RANGE, "a non-finite fp16 intermediate (x) was seen (code 0x%x)", v);
        return fail(TRIMUL_ERR_DEVICE_TIMEOUT, "a kernel gave up on a bounded wait (code 0x%x)", v);
    }
    return TRIMUL_OK;
}

// ------------------------------------------------------------------ pair transition

struct trimul_transition {
    int c, hidden;
    void *mem;                   // W1 [hidden][c] bf16, W2 [c][hidden] f16, b1 [hidden] f32, b2 [c] f32
    uint16_t *w1, *w2;
    float *b1, *b2;
    CUtensorMap tm_w1, tm_w2;
};

extern "C" trimul_status_t tri_mul_transition_create(int c, int hidden, trimul_dtype_t dtype, const void *w1,
                                                     const void *b1, const void *w2, const void *b2, void *stream,
                                                     trimul_transition_t **out) {
    if (!out) return fail(TRIMUL_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!w1 || !w2) return fail(TRIMUL_ERR_INVALID_ARG, "W1 and W2 are required");
    if (dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "the pair transition runs on bf16 weights");
    if (c != 128 || hidden != 256)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "pair transition supports c = 128, hidden = 256 (got %d, %d)", c, hidden);
    DeviceInfo d;
    TRY(require_sm100(&d));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    trimul_transition *T = new (std::nothrow) trimul_transition();
    if (!T) return fail(TRIMUL_ERR_INVALID_ARG, "out of host memory");
    T->c = c;
    T->hidden = hidden;
    const size_t wbytes = (size_t)c * hidden * 2;
    const size_t total = 2 * wbytes + (size_t)(hidden + c) * sizeof(float);
    if (cudaMalloc(&T->mem, total) != cudaSuccess) {
        delete T;
        return fail(TRIMUL_ERR_CUDA, "cudaMalloc of %zu bytes failed", total);
    }
    uint8_t *m = reinterpret_cast<uint8_t *>(T->mem);
    T->w1 = reinterpret_cast<uint16_t *>(m);
    T->w2 = reinterpret_cast<uint16_t *>(m + wbytes);
    T->b1 = reinterpret_cast<float *>(m + 2 * wbytes);
    T->b2 = T->b1 + hidden;
    trimul_status_t status = TRIMUL_OK;
    cudaError_t e = cudaMemcpyAsync(T->w1, w1, wbytes, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = bf16_to_f16_launch(w2, T->w2, (long long)c * hidden, st);   // GEMM2 runs in f16
    if (e == cudaSuccess) e = b1 ? to_f32_launch(b1, 1, T->b1, 1, hidden, 0, st) : cudaMemsetAsync(T->b1, 0, hidden * 4, st);
    if (e == cudaSuccess) e = b2 ? to_f32_launch(b2, 1, T->b2, 1, c, 0, st) : cudaMemsetAsync(T->b2, 0, c * 4, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) status = cuda_fail(e, "transition weights copy");
    if (status == TRIMUL_OK) {
        uint64_t dims1[2] = {(uint64_t)c, (uint64_t)hidden}, strides1[1] = {(uint64_t)c * 2};
        uint32_t box1[2] = {64, (uint32_t)hidden};
        status = make_map(&T->tm_w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T->w1, dims1, strides1, box1,
                          CU_TENSOR_MAP_SWIZZLE_128B, "transition W1");
    }
    if (status == TRIMUL_OK) {
        uint64_t dims2[2] = {(uint64_t)hidden, (uint64_t)c}, strides2[1] = {(uint64_t)hidden * 2};
        uint32_t box2[2] = {64, (uint32_t)c};
        status = make_map(&T->tm_w2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T->w2, dims2, strides2, box2,
                          CU_TENSOR_MAP_SWIZZLE_128B, "transition W2");
    }
    if (status != TRIMUL_OK) {
        cudaFree(T->mem);
        delete T;
        return status;
    }
    *out = T;
    return TRIMUL_OK;
}

extern "C" void tri_mul_transition_destroy(trimul_transition_t *T) {
    if (!T) return;
    if (T->mem) cudaFree(T->mem);
    delete T;
}

extern "C" trimul_status_t tri_mul_transition_forward(const trimul_pair_t *z, const void *mask,
                                                      const trimul_transition_t *T, trimul_pair_t *out, void *stream) {
    // shapes first (no handle needed), so that every size rule is checked before anything else
    TRY(check_pair(z, "z"));
    TRY(check_pair(out, "out"));
    if (z->dtype != TRIMUL_BF16) return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "the pair transition takes a bf16 z");
    if (z->N < 8 || z->N % 8 != 0 || z->N > 16384)
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a multiple of 8 in [8, 16384]", (long long)z->N);
    // the kernel walks B * N^2 / 64 tiles with int indices and int pair coordinates
    if ((long long)z->B * (z->N * z->N / 64) >= (1LL << 31))
        return fail(TRIMUL_ERR_UNSUPPORTED_SHAPE, "problem too large: B * N^2 / 64 must stay below 2^31");
    if (!T) return fail(TRIMUL_ERR_INVALID_ARG, "transition handle is NULL");
    if (z->C != T->c) return fail(TRIMUL_ERR_INVALID_ARG, "z has %lld channels, the transition %d", (long long)z->C, T->c);
    if (mask && !aligned16(mask)) return fail(TRIMUL_ERR_ALIGNMENT, "mask not 16-byte aligned");
    if (out->B != z->B || out->N != z->N || out->C != z->C) return fail(TRIMUL_ERR_INVALID_ARG, "out shape differs from z");
    if (overlap(out->data, pair_bytes(out), z->data, pair_bytes(z))) return fail(TRIMUL_ERR_INVALID_ARG, "out overlaps z");
    DeviceInfo d;
    TRY(require_sm100(&d));
    const uint64_t NN = (uint64_t)z->N * z->N;
    const uint64_t B = (uint64_t)z->B;
    PtArgs p{};
    {
        // z [B][NN][128] viewed as {64 channels, NN pairs, 2 halves, B}: one copy brings both
        // 64-channel halves of 64 pairs, laid out [half][pair][64]
        uint64_t dims[4] = {64, NN, 2, B};
        uint64_t strides[3] = {(uint64_t)T->c * 2, 128, NN * T->c * 2};
        uint32_t box[4] = {64, 64, 2, 1};
        TRY(make_map(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, z->data, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B, "transition z"));
    }
    {
        const bool f32 = out->dtype == TRIMUL_F32;
        const uint64_t es = f32 ? 4 : 2;
        uint64_t dims[3] = {(uint64_t)T->c, NN, B};
        uint64_t strides[2] = {(uint64_t)T->c * es, NN * T->c * es};
        uint32_t box[3] = {(uint32_t)T->c, 32, 1};
        TRY(make_map(&p.tm_out, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out->data,
                     dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE, "transition out"));
    }
    p.tm_w1 = T->tm_w1;
    p.tm_w2 = T->tm_w2;
    p.z = reinterpret_cast<const uint16_t *>(z->data);
    p.mask = reinterpret_cast<const uint16_t *>(mask);
    p.b1 = T->b1;
    p.b2 = T->b2;
    p.B = (int)z->B;
    p.NN = (long long)NN;
    p.tiles_per_batch = (int)(NN / 64);
    const int grid = grid_for(d.sms, (long long)B * p.tiles_per_batch, 1);
    TRY_CUDA(pt_launch(out->dtype == TRIMUL_F32, p, grid, reinterpret_cast<cudaStream_t>(stream)), "transition launch");
    return TRIMUL_OK;
}

extern "C" const char *tri_mul_status_string(trimul_status_t s) {
    switch (s) {
        case TRIMUL_OK: return "ok";
        case TRIMUL_ERR_INVALID_ARG: return "invalid argument";
        case TRIMUL_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case TRIMUL_ERR_UNSUPPORTED_DEVICE: return "unsupported device";
        case TRIMUL_ERR_WORKSPACE: return "workspace missing or too small";
        case TRIMUL_ERR_CUDA: return "CUDA error";
        case TRIMUL_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case TRIMUL_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case TRIMUL_ERR_RANGE: return "intermediate out of fp16 range";
    }
    return "unknown status";
}

extern "C" const char *tri_mul_last_error(void) { return g_last_error; }

extern "C" int tri_mul_abi_version(void) { return TRIMUL_ABI_VERSION; }
