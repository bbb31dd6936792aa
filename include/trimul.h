/*
 * trimul.h -- C ABI of the B200 (sm_100a) triangle multiplicative update.
 *
 * The operation (one "layer", one direction) on a pair tensor z [B, N, N, c_z]
 * with pair mask m [B, N, N]:
 *
 *   zhat_ij = LayerNorm_{c_z}(z_ij)
 *   a_ij    = m_ij * sigmoid(zhat_ij W_ag^T + b_ag) (.) (zhat_ij W_ap^T + b_ap)
 *   b_ij    = m_ij * sigmoid(zhat_ij W_bg^T + b_bg) (.) (zhat_ij W_bp^T + b_bp)
 *   outgoing: x_ij = sum_k a_ik (.) b_jk        incoming: x_ij = sum_k a_ki (.) b_kj
 *   out_ij  = m_ij * sigmoid(zhat_ij W_g^T + b_g) (.) (LayerNorm_{c_h}(x_ij) W_o^T + b_o)
 *
 * Sources: "RFProteina architecture" (BioNeMo Inference Runtime documentation),
 * section "Inside the velocity network" (a pair update applies outgoing, then
 * incoming triangle multiplication, each as a masked residual), section
 * "Triangle multiplication on SM90" (the three-kernel chain: K1 input projection
 * with the input LayerNorm folded into its weights, K2 the contraction compiled
 * per direction, K3 output gate and projection with both LayerNorms folded) and
 * section "Dual-GEMM gates" (the one-input gate sigma(x W_g^T + b_g) (.) (x W_p^T + b_p)
 * that also applies the pair mask and emits its output transposed for the
 * contraction, and the two-input gate sigma(x0 W_g^T + b_g) (.) (x1 W_p^T + b_p)
 * with x0 the normalized pair tensor and x1 the contracted hidden tensor).
 *
 * Conventions for every entry point:
 *   - All tensors are device pointers owned by the caller. Nothing here frees them.
 *   - Pair tensors are contiguous [B, N, N, C], channel fastest (channel-last).
 *   - Intermediate tensors a, b, x are contiguous [B, c_h, N, N] (channel-major:
 *     every channel is one N x N matrix), which is the layout the contraction reads.
 *     For a BF16 z they are stored as F16 (IEEE half: same 2 bytes and tensor-core
 *     rate as bf16, 3 more mantissa bits); x is stored pre-multiplied by the power of
 *     two tri_mul_contract_scale(N) (about 1/sqrt(N)) to stay far inside the F16
 *     range, and the output LayerNorm is evaluated with eps * scale^2, which is the
 *     same function of the unscaled x. For an F32 z they are F32 with scale 1.
 *   - Linear weights are row-major [out, in] with y = x W^T + bias. Bias and
 *     LayerNorm beta pointers may be NULL (= 0); LayerNorm gamma may be NULL (= 1).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Forward calls
 *     are asynchronous on it, allocate nothing and never synchronize.
 *   - There is no fallback: an unsupported shape, dtype or device is an error.
 *   - Errors are returned as trimul_status_t; tri_mul_last_error() gives a
 *     human-readable detail for the calling thread.
 */
#ifndef TRIMUL_H
#define TRIMUL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TRIMUL_OK = 0,
    TRIMUL_ERR_INVALID_ARG = 1,        /* NULL pointer, bad size, unknown enum, aliasing */
    TRIMUL_ERR_UNSUPPORTED_SHAPE = 2,  /* (c_z, c_h) or N outside the compiled set */
    TRIMUL_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not compute capability 10.0 */
    TRIMUL_ERR_WORKSPACE = 4,          /* no workspace bound, or bound one too small */
    TRIMUL_ERR_CUDA = 5,               /* a CUDA runtime / driver call failed */
    TRIMUL_ERR_DEVICE_TIMEOUT = 6,     /* a kernel gave up on a bounded wait (see below) */
    TRIMUL_ERR_ALIGNMENT = 7,          /* a tensor pointer is not 16-byte aligned */
    TRIMUL_ERR_RANGE = 8               /* a non-finite or out-of-range (|v| > 65504) fp16
                                          intermediate was seen (reported by
                                          tri_mul_check_device_status) */
} trimul_status_t;

typedef enum { TRIMUL_OUTGOING = 0, TRIMUL_INCOMING = 1 } trimul_direction_t;

/* F32: IEEE binary32. BF16: bfloat16. F16: IEEE binary16 (the intermediate type of
 * the tensor-core path). */
typedef enum { TRIMUL_F32 = 0, TRIMUL_BF16 = 1, TRIMUL_F16 = 2 } trimul_dtype_t;

/* A pair tensor [B, N, N, C], contiguous, channel-last. */
typedef struct {
    void *data;
    int64_t B, N, C;
    trimul_dtype_t dtype;
} trimul_pair_t;

/* Layer weights, all device pointers of storage type `dtype`, in this order:
 *   ln_in_g, ln_in_b [c_z]            input LayerNorm
 *   w_ag, w_ap, w_bg, w_bp [c_h, c_z]; b_ag, b_ap, b_bg, b_bp [c_h]
 *   w_g [c_z, c_z], b_g [c_z]         output gate
 *   ln_out_g, ln_out_b [c_h]          output LayerNorm
 *   w_o [c_z, c_h], b_o [c_z]         output projection
 * eps: LayerNorm epsilon for both norms (variance is the biased one, eps inside
 * the square root). */
typedef struct {
    int32_t c_z, c_h;
    trimul_dtype_t dtype;
    float eps;
    const void *ln_in_g, *ln_in_b;
    const void *w_ag, *b_ag, *w_ap, *b_ap;
    const void *w_bg, *b_bg, *w_bp, *b_bp;
    const void *w_g, *b_g;
    const void *ln_out_g, *ln_out_b;
    const void *w_o, *b_o;
} trimul_weights_desc_t;

/* Opaque layer handle: the weights repacked for both compute paths. */
typedef struct trimul_layer trimul_layer_t;

/* Build a layer handle from weights already on the current device.
 * The handle holds its own device copy: for the tensor-core path the input
 * LayerNorm gamma is folded into W_ag/W_ap/W_bg/W_bp/W_g (bf16, the type of z)
 * and the output LayerNorm gamma into W_o (F16, the type of x), all [out, in],
 * with per-row correction vectors sum_k W'[r, k] and sum_k beta[k] W[r, k] + bias[r]
 * in fp32 (the folding of "Triangle multiplication on SM90"); for the fp32 path it
 * keeps fp32 copies.
 * Runs on `stream` and synchronizes it before returning, so the caller may free
 * the source weights afterwards. Supported (c_z, c_h): any multiple of 32 up to
 * 512 for the fp32 path; (128, 128) and (384, 128) for the bf16 path (checked
 * at forward time). */
trimul_status_t tri_mul_layer_create(const trimul_weights_desc_t *weights, void *stream,
                                     trimul_layer_t **layer_out);

/* Free the handle and its device memory. NULL is ignored. */
void tri_mul_layer_destroy(trimul_layer_t *layer);

/* Bytes of workspace tri_mul_forward needs for B x N x N with z of type `dtype`:
 * a, b and x, each [B, c_h, N, N] of the intermediate type (F16 for a BF16 z,
 * F32 for an F32 z), 256-byte aligned, then, each 256-byte aligned, the mask extents
 * (2 int32 per batch element) and the offset of the stored x (c_h fp32 per batch
 * element). Returns 0 for an invalid layer or size. */
size_t tri_mul_workspace_bytes(const trimul_layer_t *layer, int64_t B, int64_t N,
                               trimul_dtype_t dtype);

/* Attach caller-owned device workspace to the handle (replaces any earlier one).
 * The handle does not own it. Two forwards that run concurrently on different
 * streams must use different handles: besides the workspace, the handle holds the
 * channel sums its projection step gathers during a forward. */
trimul_status_t tri_mul_layer_bind_workspace(trimul_layer_t *layer, void *workspace,
                                             size_t bytes);

/* One triangle multiplicative update (one direction). Returns the update only;
 * the residual add z += update is the caller's (or tri_mul_forward_residual's).
 * On the tensor-core path four kernels run: K1 (projection), a small pass that turns K1's
 * per-channel sums of a and b into one offset o per batch element, K2 (contraction, storing
 * x - o) and K3 (output gate). o = (1/c_h) sum_c Sa_c Sb_c / P^1.5 (Sa_c, Sb_c the channel sums
 * over the batch element, P its unmasked pairs) estimates the common mode of x that a large
 * mean of a and b produces; storing x - o keeps the F16 rounding of x small next to the
 * spread the output LayerNorm divides by, and the LayerNorm, which ignores a constant added
 * to every channel of a pair, needs no correction. The sums are integers (fixed point), so
 * results do not depend on the order tiles finish in.
 * With mask skipping switched on (tri_mul_layer_set_mask_skipping), on the tensor-core
 * path with a mask a first pass finds the mask's extents (the last row and column holding a
 * nonzero entry, per batch element) and the kernels leave out tiles that are masked in full
 * and the part of the contraction's k-range beyond them (the results are bitwise the same:
 * every product left out is an exact zero).
 *   z    : [B, N, N, c_z], dtype F32 (fp32 SIMT path) or BF16 (tensor-core path)
 *   mask : [B, N, N] in z's dtype with values 0 or 1, or NULL for all ones
 *   out  : [B, N, N, c_z]; F32 for the F32 path; F32 or BF16 for the BF16 path
 *          (must not overlap z or the workspace)
 * Requirements: N % 8 == 0 and 8 <= N <= 16384 (the pages pad token axes to
 * multiples of 8); B >= 1 and B * c_h <= 65535; on the BF16 path B * N^2 / 128
 * <= 2^30; every pointer 16-byte aligned; a workspace of at least
 * tri_mul_workspace_bytes() bound. The BF16 path needs an sm_100 device. The N and
 * tile rules are checked before the layer handle, B * c_h right after it; a violation
 * returns TRIMUL_ERR_UNSUPPORTED_SHAPE with nothing launched. */
trimul_status_t tri_mul_forward(const trimul_pair_t *z, const void *mask,
                                const trimul_layer_t *layer, trimul_direction_t direction,
                                trimul_pair_t *out, void *stream);

/* Step K1 alone ("x_x" input gate): a and b from z, written channel-major
 * [B, c_h, N, N] in the intermediate type (F16 for a BF16 z, F32 for an F32 z).
 * Same requirements as tri_mul_forward. */
trimul_status_t tri_mul_project(const trimul_pair_t *z, const void *mask,
                                const trimul_layer_t *layer, void *a_out, void *b_out,
                                void *stream);

/* Step K2 alone (the contraction): x from a and b, all [B, C, N, N] of `dtype`.
 *   outgoing: x[b,c,i,j] = x_scale * sum_k a[b,c,i,k] b[b,c,j,k]
 *   incoming: x[b,c,i,j] = x_scale * sum_k a[b,c,k,i] b[b,c,k,j]
 * F16 / BF16: tensor cores, fp32 accumulation, result rounded to `dtype` after the
 * scaling (sm_100 only). F32: fp32 FMA on CUDA cores. N % 8 == 0, 8 <= N <= 16384,
 * B * C <= 65535. x must not overlap a or b. Use a power of two for x_scale to keep
 * the scaling exact. */
trimul_status_t tri_mul_contract(const void *a, const void *b, void *x, int64_t B, int64_t C,
                                 int64_t N, trimul_dtype_t dtype, trimul_direction_t direction,
                                 float x_scale, void *stream);

/* The power of two tri_mul_forward multiplies x by on the tensor-core path:
 * 2^-ceil(log2(N) / 2). Returns 0 for N < 1. */
float tri_mul_contract_scale(int64_t N);

/* Step K3 alone ("x0_x1" output gate): out from z, the mask and x [B, c_h, N, N]
 * in the intermediate type, where x holds x_scale times the contraction (x_scale > 0;
 * the output LayerNorm then uses eps * x_scale^2). Same requirements as
 * tri_mul_forward. */
trimul_status_t tri_mul_output_gate(const trimul_pair_t *z, const void *mask, const void *x,
                                    float x_scale, const trimul_layer_t *layer,
                                    trimul_pair_t *out, void *stream);

/* tri_mul_forward for callers that cannot allocate device memory (for example a plug-in
 * inside a framework that owns the allocator and gives it no way to ask for memory, or
 * a path that must not risk an allocation failing or stalling mid-work). Same arguments,
 * checks, kernels and results as tri_mul_forward, but the intermediates (a, b, x and the
 * small per-batch vectors tri_mul_workspace_bytes() counts) live in a fixed array built
 * into the library (TRIMUL_NOALLOC_SCRATCH_BYTES of device memory on every GPU that loads
 * it, held until the process exits) instead of a bound workspace; the layer's workspace
 * and timing events are not used. It allocates nothing.
 *   - Every argument is checked before anything touches the device; a problem with
 *     tri_mul_workspace_bytes() > TRIMUL_NOALLOC_SCRATCH_BYTES (for a BF16 z with
 *     c_h = 128: B * N * N > 65536, e.g. N = 256 at B = 1 fits) is rejected with
 *     TRIMUL_ERR_WORKSPACE.
 *   - The first call in each device context looks up the array's device address (with
 *     that device current) and keeps it for that context; a reset device gets a new
 *     lookup. Make the first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (nothing in
 *     it needs to start at zero). Calls that overlap on the GPU (different streams
 *     without ordering between them, or concurrent host threads) race on it, and so do
 *     overlapping calls with one layer handle: order them.
 * This entry point is an engineering addition with no counterpart in the pages. */
#define TRIMUL_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u + 64u * 1024u)
trimul_status_t tri_mul_forward_noalloc(const trimul_pair_t *z, const void *mask,
                                        const trimul_layer_t *layer, trimul_direction_t direction,
                                        trimul_pair_t *out, void *stream);

/* The masked-residual form of tri_mul_forward: out = z + update, where update is what
 * tri_mul_forward would write ("RFProteina architecture", section "Two networks around one
 * state", subsection "Inside the velocity network": each triangle update is applied as a
 * masked residual; a masked pair keeps its z, its update being 0). The sum is formed in
 * fp32 from z's stored value and the fp32 update and rounded once to out's type. Same
 * arguments and requirements as tri_mul_forward. */
trimul_status_t tri_mul_forward_residual(const trimul_pair_t *z, const void *mask,
                                         const trimul_layer_t *layer, trimul_direction_t direction,
                                         trimul_pair_t *out, void *stream);

/* The two triangle updates of one pair update, in order on one stream (same page and
 * subsection: outgoing, then incoming triangle multiplication, each a masked residual):
 *   z_mid = z + U_outgoing(z)       with layer_out's weights, stored in z's dtype
 *   out   = z_mid + U_incoming(z_mid) with layer_in's weights
 * Each call uses its layer's bound workspace; the same handle may be passed for both (its
 * workspace is then reused in order). z_mid has z's shape and dtype; out has z's shape and
 * z's dtype, or F32 on the BF16 path. z, z_mid and out must not overlap one another or
 * either workspace. Other requirements as tri_mul_forward. */
trimul_status_t tri_mul_pair_update(const trimul_pair_t *z, const void *mask,
                                    const trimul_layer_t *layer_out, const trimul_layer_t *layer_in,
                                    trimul_pair_t *z_mid, trimul_pair_t *out, void *stream);

/* A CUDA graph of one tri_mul_pair_update on fixed buffers ("NVIDIA's BioNeMo Inference
 * Runtime", section "Three Layers of Acceleration", layer 2: a recorded sequence of GPU
 * work replayed with little host-side cost per launch). Creation captures the six kernel
 * launches (with their programmatic-launch edges) on an internal stream and instantiates
 * the graph; nothing runs. Each tri_mul_graph_launch replays it on `stream`, reading the
 * current contents of z and mask and writing z_mid and out. The buffers, both layers and
 * their bound workspaces must stay alive and unchanged in place (contents may change) for
 * the graph's lifetime; the layers' timing events are not recorded by the graph. */
typedef struct trimul_graph trimul_graph_t;
trimul_status_t tri_mul_pair_update_graph_create(const trimul_pair_t *z, const void *mask,
                                                 const trimul_layer_t *layer_out,
                                                 const trimul_layer_t *layer_in,
                                                 trimul_pair_t *z_mid, trimul_pair_t *out,
                                                 trimul_graph_t **graph_out);
trimul_status_t tri_mul_graph_launch(const trimul_graph_t *graph, void *stream);
/* Free the graph. NULL is ignored. */
void tri_mul_graph_destroy(trimul_graph_t *graph);

/* ---- Row-sharded update ("big mode") ----------------------------------------------------
 * One update split by rows over G shards (GPUs), as the commentary on the AI-refactored
 * structure-prediction code describes for complexes too large for one GPU: the pair tensor
 * is sharded across the GPUs of a node by rows, large intermediates chunked. Shard g owns
 * rows [row0[g], row0[g+1]) of z, of the mask and of the update, and of the a and b planes.
 *   outgoing: x_ij = sum_k a_ik b_jk needs this shard's a rows and b rows j from every shard;
 *   incoming: x_ij = sum_k a_ki b_kj needs a and b rows k from every shard (a's columns i of
 *             this shard's rows).
 * Phase 1 (tri_mul_shard_project) makes a and b of the shard's rows; between the phases the
 * caller makes every shard's a (incoming only) and b readable by the others (an all-gather
 * into local buffers, or peer mappings of the other GPUs' buffers: the contraction reads
 * them through TMA tensor maps, never with a multicast load); phase 2 (tri_mul_shard_finish)
 * contracts and gates the shard's rows. Both phases of one update use the same layer handle
 * and its bound workspace (tri_mul_shard_workspace_bytes: this shard's x and its offset),
 * in order on one stream; phase 1 computes the offset of the stored x from the shard's own
 * channel sums (see tri_mul_forward), so shards need not exchange anything else.
 * Tensor-core path only: bf16 z, (c_z, c_h) = (128, 128) or (384, 128); N a multiple of 128
 * in [128, 16384]; every shard a whole number of 128-row blocks; 1 <= G <= 8. Results equal
 * the unsharded update up to the offset's rounding (a per-shard offset instead of one per
 * batch element). */

/* Rows [row0, row0 + R) of a [B, N, N, C] pair tensor, stored contiguously as [B, R, N, C]. */
typedef struct {
    void *data;
    int64_t B, R, N, C, row0;
    trimul_dtype_t dtype;
} trimul_rows_t;

/* Workspace bytes one shard of R rows needs (bound with tri_mul_layer_bind_workspace):
 * x [B, c_h, R, N] F16 and the offset (c_h fp32 per batch element), each 256-byte aligned.
 * Returns 0 for an invalid layer or size. */
size_t tri_mul_shard_workspace_bytes(const trimul_layer_t *layer, int64_t B, int64_t R, int64_t N);

/* Phase 1: K1 on the shard's rows and the offsets pass. z and mask hold the shard's rows
 * (mask [B, R, N] in z's dtype, or NULL); a_out and b_out receive [B, c_h, R, N] F16 (caller
 * owned, not overlapping z, each other or the workspace). */
trimul_status_t tri_mul_shard_project(const trimul_rows_t *z, const void *mask, const trimul_layer_t *layer,
                                      void *a_out, void *b_out, void *stream);

/* Phase 2: the contraction for the shard's rows, then K3 on them, writing out (the shard's
 * rows of the update, F32 or BF16, z's shape, not overlapping z or the workspace).
 * shard_row0[0..G] are the shard boundaries (0 = shard_row0[0] < ... < shard_row0[G] = N, each a
 * multiple of 128); z's rows must be one of the shards. a_shards[g], b_shards[g]: shard g's
 * phase-1 a and b ([B, c_h, R_g, N] F16, device pointers readable from this GPU); a_shards is read
 * only for this shard (outgoing) or all shards (incoming). */
trimul_status_t tri_mul_shard_finish(const trimul_rows_t *z, const void *mask, const trimul_layer_t *layer,
                                     trimul_direction_t direction, int G, const int64_t *shard_row0,
                                     const void *const *a_shards, const void *const *b_shards,
                                     trimul_rows_t *out, void *stream);

/* Mask skipping ("RFProteina architecture", section "Kernel support": masks are left-aligned,
 * so per-row valid counts, computed once, bound the work of every pair update). With a mask's
 * extents {R_b, C_b} (1 + the last row / column of batch element b holding a nonzero mask
 * entry) the kernels leave out tiles that are masked in full (writing their zeros) and the
 * contraction's k-range beyond them; results are bitwise those without skipping. Extents come,
 * in this order, from a caller (tri_mul_forward_extents), from valid lengths set on the layer
 * (tri_mul_layer_set_valid_lengths, when they match the problem's B and N), or, with mask
 * skipping switched on (tri_mul_layer_set_mask_skipping, off by default), from a pass over the
 * mask (a memset and one small kernel) per forward, or once per tri_mul_pair_update. */
trimul_status_t tri_mul_layer_set_mask_skipping(trimul_layer_t *layer, int enable);

/* The extents of a bf16 mask [B, N, N] into extents[2B] (int32 on the device, 16-byte aligned):
 * a memset and one small kernel on `stream`. */
trimul_status_t tri_mul_mask_extents(const void *mask, int64_t B, int64_t N, trimul_dtype_t dtype,
                                     int32_t *extents, void *stream);

/* tri_mul_forward with the mask's extents given (device int32 [B][2], for instance from
 * tri_mul_mask_extents once per mask): skipping applies whatever the layer's settings. Every
 * nonzero mask entry of batch element b must lie in rows < R_b and columns < C_b. BF16 path. */
trimul_status_t tri_mul_forward_extents(const trimul_pair_t *z, const void *mask, const int32_t *extents,
                                        const trimul_layer_t *layer, trimul_direction_t direction,
                                        trimul_pair_t *out, void *stream);

/* The share of one layer's dense work (its flops at N) that skipping by left-aligned valid
 * lengths lengths[0..B) leaves out (K1 and K3 scale with L_b^2 pairs, K2 with L_b^3). */
double tri_mul_skip_saving(const int64_t *lengths, int64_t B, int64_t N, int32_t c_z, int32_t c_h);

/* Per-batch-element valid lengths of a left-aligned padding mask (host int64 [B]: mask entries
 * of batch element b are 0 at rows or columns >= lengths[b]), set once for all later forwards
 * of B x N problems on this handle: their extents {L_b, L_b} go to a device buffer the handle
 * allocates now (the call synchronizes), and skipping is used only when tri_mul_skip_saving
 * is at least 0.15 (it costs a few percent otherwise; *skipping_out, when not NULL, tells
 * which). NULL lengths clears them. */
trimul_status_t tri_mul_layer_set_valid_lengths(trimul_layer_t *layer, const int64_t *lengths, int64_t B, int64_t N,
                                                int32_t *skipping_out);

/* The fused pair transition, the step that follows the two triangle updates in a pair
 * update ("RFProteina architecture", section "Kernel support": one launch runs both linears,
 * the ReLU, the mask and the residual and keeps the hidden activation on chip):
 *   out_ij = z_ij + m_ij * (relu(z_ij . W1^T + b1) . W2^T + b2)
 * Weights [out, in] as for the triangle layer: W1 [hidden, c], b1 [hidden], W2 [c, hidden],
 * b2 [c]; biases may be NULL (0). Supported: bf16, c = 128, hidden = 256 (the pages' expansion
 * of 2); anything else returns TRIMUL_ERR_UNSUPPORTED_SHAPE. Creation copies the weights
 * into the handle (biases kept in fp32) and synchronizes `stream`. The forward takes z
 * [B, N, N, 128] bf16, a mask as tri_mul_forward, and writes out [B, N, N, 128] in F32 or
 * BF16 (not overlapping z); fp32 accumulation, the hidden activation rounded to f16 on
 * chip (W2 kept in f16 for that product); N a multiple of 8 in [8, 16384] and
 * B * N^2 / 64 < 2^31 (TRIMUL_ERR_UNSUPPORTED_SHAPE otherwise, checked before the handle);
 * sm_100 only. */
typedef struct trimul_transition trimul_transition_t;
trimul_status_t tri_mul_transition_create(int c, int hidden, trimul_dtype_t dtype, const void *w1,
                                          const void *b1, const void *w2, const void *b2,
                                          void *stream, trimul_transition_t **transition_out);
void tri_mul_transition_destroy(trimul_transition_t *transition);
trimul_status_t tri_mul_transition_forward(const trimul_pair_t *z, const void *mask,
                                           const trimul_transition_t *transition,
                                           trimul_pair_t *out, void *stream);

/* Optional per-kernel timing: when `events` is non-NULL, every later
 * tri_mul_forward on this handle records events[0] before K1 (after the mask-extents
 * pass), events[1] after K1 and the offsets pass, events[2] after K2 and events[3]
 * after K3 on its stream. The four values are cudaEvent_t created by the caller;
 * NULL switches recording off. Recording an event between two kernels ends the
 * overlap of one kernel's start with the previous one's end, so timed forwards run
 * a little slower than untimed ones. */
trimul_status_t tri_mul_layer_set_timing_events(trimul_layer_t *layer, void *const *events);

/* Number of kernels one tri_mul_forward launches on the tensor-core path: K1, the offsets
 * pass, K2 and K3 (one more, the mask-extents pass, with a mask and mask skipping switched
 * on). The fp32 path launches three (no offsets pass). */
int tri_mul_kernels_per_forward(void);

/* Synchronize the current device, then read and clear the library's device
 * error word. Every wait inside the tensor-core kernels is bounded (about one
 * second); a wait that runs out makes its kernel stop early, and this call reports
 * TRIMUL_ERR_DEVICE_TIMEOUT. K3 also flags a non-finite x (an F16 intermediate that
 * overflowed, or a non-finite input) as TRIMUL_ERR_RANGE. Outputs of such a launch
 * are undefined. */
trimul_status_t tri_mul_check_device_status(void);

/* Failure-path self-test: launches one kernel on `stream` that waits, with the same
 * bounded wait the tensor-core kernels use, on a barrier nothing will complete. The
 * wait gives up after about one second and records the timeout in the device error
 * word; a following tri_mul_check_device_status() must return
 * TRIMUL_ERR_DEVICE_TIMEOUT, and the device stays usable. No fault, trap or hang is
 * involved. sm_100 only. */
trimul_status_t tri_mul_selftest_bounded_wait(void *stream);

/* Static description of a status code. */
const char *tri_mul_status_string(trimul_status_t status);

/* Detail of the last error raised on the calling thread ("" if none). */
const char *tri_mul_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int tri_mul_abi_version(void);

#define TRIMUL_ABI_VERSION 103

#ifdef __cplusplus
}
#endif

#endif /* TRIMUL_H */
