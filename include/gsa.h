/*
 * gsa.h -- C ABI of the B200 (sm_100a) Global Sparse Attention (GSA) layer.
 *
 * The layer is the one described in "Speed3R: Sparse Feed-forward 3D
 * Reconstruction Models" (Paper-Notes, CVPR 2026), section "全局稀疏注意力
 * （GSA）核心设计" (GSA core design):
 *   - Q/K/V are split into special tokens and image tokens (equation for
 *     Q = [Q_spec; Q_img]);
 *   - special tokens attend densely to every token (equation for O_spec);
 *   - image tokens take two branches: a compression branch (s x s mean
 *     pooling, attention among the pooled tokens, guide scores
 *     S_guide = Q_comp K_comp^T, nearest upsampling) and a selection branch
 *     (top-k regions per compressed query, attention of the window's queries
 *     to the full-resolution tokens of those regions);
 *   - a gate g = sigmoid(W_g Q_img) mixes them: O_img = g*O_comp + (1-g)*O_sel.
 * The VGGT variant (section "Speed3R-VGGT 适配") adds a fixed global context
 * to the selection branch: every token of the reference frame and of frames
 * sampled every 100 frames.
 *
 * Everything here is plain C: pointers and sizes, no framework types.
 * Device pointers are CUDA device addresses owned by the caller; the context
 * owns its workspace (device memory allocated in gsa_create).
 * Streams are passed as void* holding a cudaStream_t (NULL = legacy default).
 * Every call returns an int status (GSA_OK = 0); nothing aborts the process
 * and no C++ exception crosses this boundary.
 */
#ifndef GSA_B200_H
#define GSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GSA_API __attribute__((visibility("default")))
#else
#define GSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define GSA_OK                 0
#define GSA_ERR_INVALID_ARG    1  /* NULL pointer, negative size, bad enum          */
#define GSA_ERR_SHAPE          2  /* grid not divisible by pool_s, head_dim != 64,
                                     topk outside [1, candidates], region with no
                                     valid token                                      */
#define GSA_ERR_UNSUPPORTED    3  /* valid but not implemented (e.g. topk > 128)      */
#define GSA_ERR_OOM            4  /* workspace allocation failed                      */
#define GSA_ERR_CUDA           5  /* a CUDA runtime call failed                       */
#define GSA_ERR_DEVICE_TIMEOUT 6  /* a bounded device-side wait ran out               */
#define GSA_ERR_DEVICE_BOUNDS  7  /* a device-side index check failed                 */

/* element type of every input and output of one context */
#define GSA_BF16 0
#define GSA_FP32 1

/* gate modes: LEARNED uses g = sigmoid(W_g q); the other two force g = 1
 * (compression branch only) or g = 0 (selection branch only).  They isolate
 * the branches for testing (section "门控聚合", gated aggregation).         */
#define GSA_GATE_LEARNED   0
#define GSA_GATE_COMP_ONLY 1
#define GSA_GATE_SEL_ONLY  2

/* maximum top-k and maximum number of fixed-context frames; top-k above 64
 * needs bf16 and pool_s = 4 (the notes' test-time top-128, section "测试时自适应") */
#define GSA_MAX_TOPK         128
#define GSA_MAX_FIXED_FRAMES 16

/* Layer variants of the notes' ablation study ("消融实验", rows (1) and (2)).
 * They change what is computed, not only the output:
 *   GSA_VARIANT_FULL           the layer as described: O_img = g O_comp + (1-g) O_sel
 *   GSA_VARIANT_NO_COMP_VALUE  "移除压缩分支 Value": the compressed branch keeps only
 *                              its guide (S_guide and the top-k; no V_comp, no P V),
 *                              O_img = O_sel (the gate has nothing to blend with)
 *   GSA_VARIANT_NO_SELECTION   "移除选择分支": no top-k and no selection branch,
 *                              O_img = Upsample(O'_comp); sel_idx_out must be NULL
 * gate_mode is ignored by the two ablation variants; special tokens are
 * computed as in the full layer.
 *   GSA_VARIANT_DESCRIPTOR     FlashVGGT's descriptor attention (a second method of
 *                              the same pages, "FlashVGGT ... 描述符注意力"): every frame's
 *                              valid K/V grid is resized bilinearly to
 *                              (grid_h / pool_s, grid_w / pool_s) descriptors, and
 *                              every image and special token attends to the
 *                              descriptors of all frames plus all special tokens.
 *                              topk, gate_mode and w_g are not used; sel_idx_out
 *                              must be NULL. */
#define GSA_VARIANT_FULL          0
#define GSA_VARIANT_NO_COMP_VALUE 1
#define GSA_VARIANT_NO_SELECTION  2
#define GSA_VARIANT_DESCRIPTOR    3

typedef struct gsa_ctx gsa_ctx;

typedef struct {
    int num_frames;        /* F >= 1                                              */
    int grid_h, grid_w;    /* valid patch grid per frame                          */
    int pad_h, pad_w;      /* stored grid, >= grid, divisible by pool_s; pad
                              tokens sit at the bottom rows / right cols          */
    int num_special;       /* special tokens per frame, >= 0 (0 = registers and
                              camera tokens removed, pi^3 adaptation)             */
    int num_heads;         /* H >= 1                                              */
    int head_dim;          /* must be 64                                          */
    int pool_s;            /* s in {1, 2, 4, 8}                                   */
    int topk;              /* regions per compressed query, 1..min(128, candidates);
                              above 64 only bf16 with pool_s = 4                  */
    int dtype;             /* GSA_BF16 or GSA_FP32                                */
    const int *fixed_frames; /* VGGT fixed global context frames (copied at
                              create); NULL with num_fixed_frames = 0 for pi^3   */
    int num_fixed_frames;
    int gate_mode;         /* GSA_GATE_*                                          */
    float softmax_scale;   /* 0 => 1/sqrt(head_dim)                               */
    int variant;           /* GSA_VARIANT_* (0 = the full layer)                  */
} gsa_config;

/* Validate `cfg` and create a context on the current CUDA device; allocates
 * the workspace (gsa_workspace_bytes).  On error *out is set to NULL. */
GSA_API int gsa_create(const gsa_config *cfg, gsa_ctx **out);

/* Bytes of device workspace a context with this config allocates (0 if the
 * config is invalid). */
GSA_API size_t gsa_workspace_bytes(const gsa_config *cfg);

/* One forward pass of the GSA layer, enqueued on `stream` (asynchronous: no
 * host synchronisation, no allocation).
 *   q_spec, k_spec, v_spec : [H][F][num_special][64]   (ignored if num_special=0)
 *   q_img,  k_img,  v_img  : [H][F][pad_h][pad_w][64]
 *   w_g                    : [H][64][64], row = output channel, no bias
 *   o_spec                 : [H][F][num_special][64]   output
 *   o_img                  : [H][F][pad_h][pad_w][64]  output; pad tokens get 0
 *   sel_idx_out            : optional [H][R][topk] int32 output, R =
 *                            F*(pad_h/s)*(pad_w/s); per row the selected regions
 *                            ordered by guide score descending, then index
 *                            ascending; NULL = not written
 * All tensors are contiguous, in the context's dtype, on the context's device.
 * One context serves one stream at a time.  Returns GSA_ERR_CUDA if a launch
 * fails; device-side errors surface at gsa_get_status. */
GSA_API int gsa_forward(gsa_ctx *ctx,
                const void *q_spec, const void *k_spec, const void *v_spec,
                const void *q_img, const void *k_img, const void *v_img,
                const void *w_g, void *o_spec, void *o_img, int32_t *sel_idx_out,
                void *stream);

/* Backward pass of gsa_forward ("Speed3R ... GSA": the notes train the layer
 * end to end; the region selection is a discrete choice and gets no gradient).
 * Call on the same context after gsa_forward with the same inputs: the
 * forward's pooled tensors, O'_comp, selection and softmax statistics are read
 * from the workspace.  o_spec is the forward's special-token output;
 * d_o_spec / d_o_img are the output gradients (context dtype, layouts of
 * o_spec / o_img).  Writes float32 gradients, the layouts of the inputs:
 * dq/dk/dv_img [H][F][pad_h][pad_w][64] (0 on pads), dq/dk/dv_spec
 * [H][F][num_special][64] (unused when num_special = 0), dw_g [H][64][64]
 * (0 when the gate is forced).  bf16 contexts of the full layer with
 * topk <= 64 only (GSA_ERR_UNSUPPORTED otherwise; every pool_s); allocates a scratch of
 * about 5 x H x R x 256 bytes plus one float per image-token channel on first
 * use (GSA_ERR_OOM if that fails), freed by gsa_destroy.  Asynchronous on
 * `stream`. */
GSA_API int gsa_backward(gsa_ctx *ctx,
                         const void *q_spec, const void *k_spec, const void *v_spec,
                         const void *q_img, const void *k_img, const void *v_img,
                         const void *w_g, const void *o_spec,
                         const void *d_o_spec, const void *d_o_img,
                         float *dq_spec, float *dk_spec, float *dv_spec,
                         float *dq_img, float *dk_img, float *dv_img, float *dw_g, void *stream);

/* gsa_forward with HOST buffers: the same arguments and layouts, every tensor
 * pointer (inputs, outputs, optional sel_idx_out) in host memory.  The heads
 * are processed in up to sixteen chunks: the host-to-device copies of chunk i+1
 * and the device-to-host copies of chunk i-1 overlap the layer on chunk i
 * (two extra streams of the context).  Asynchronous on `stream`: the outputs
 * are in host memory once `stream` has completed; the inputs may be reused
 * then too.  Overlap needs page-locked host memory (cudaHostAlloc or
 * cudaHostRegister); pageable memory still gives correct results, with the
 * copies serialised by the driver.  On first use the context allocates device
 * copies of one call's inputs and outputs (GSA_ERR_OOM if that fails); they
 * are freed by gsa_destroy.  The special-token split count is chosen per
 * chunk, so o_spec may differ from gsa_forward's in the last bits. */
GSA_API int gsa_forward_host(gsa_ctx *ctx,
                             const void *q_spec, const void *k_spec, const void *v_spec,
                             const void *q_img, const void *k_img, const void *v_img,
                             const void *w_g, void *o_spec, void *o_img,
                             int32_t *sel_idx_out, void *stream);

/* Dense global attention over every token of the same shape (the comparison
 * baseline, "Full Attn." in the notes' latency table):
 *   q, k, v, o : [H][F*(num_special + pad_h*pad_w)][64], per frame the special
 *                tokens then the padded image grid.  Pad tokens are never used
 *                as keys and their output rows are 0. */
GSA_API int gsa_dense_forward(gsa_ctx *ctx, const void *q, const void *k, const void *v,
                      void *o, void *stream);

/* Device pointer and size of an intermediate of the last gsa_forward, for
 * tests and profiling (valid until the next forward or gsa_destroy).
 * which: 0 Q_comp, 1 K_comp, 2 V_comp  (context dtype, [H][R][64])
 *        3 O'_comp (fp32, [H][R][64])
 *        4 selected regions (int32, [H][R][topk])
 *        5 O_sel (context dtype, [H][F][pad_h][pad_w][64]; written only with
 *          GSA_PROFILE_KEEP_OSEL or when selection and gate run as two kernels)
 *        6, 7 low parts of Q_comp, K_comp: bf16 contexts keep the pooled
 *          value x as bf16 hi = bf16(x) (items 0, 1) plus lo = bf16(x - hi)
 *          ([H][R][64] bf16), fp32 contexts return items 0, 1 again */
GSA_API int gsa_get_intermediate(gsa_ctx *ctx, int which, void **dev_ptr, size_t *bytes);

/* Profiling flags (bitwise or):
 *   GSA_PROFILE_TIMES      gsa_forward records CUDA events on its stream around
 *                          each kernel; gsa_get_kernel_times synchronises on the
 *                          last forward and writes up to `cap` durations in ms
 *                          (pool, compressed + top-k, with fixed frames in bf16
 *                          the fixed-context gather + attention, selection (with
 *                          the fused upsample/gate/blend, or followed by a
 *                          separate epilogue), special, special-merge) and their names
 *                          (static strings); it returns the number of entries
 *                          or a negative status.
 *   GSA_PROFILE_KEEP_OSEL  keep O_sel in the workspace (gsa_get_intermediate 5);
 *                          the fused selection kernel otherwise never writes it. */
#define GSA_PROFILE_TIMES     1
#define GSA_PROFILE_KEEP_OSEL 2
GSA_API int gsa_set_profiling(gsa_ctx *ctx, int flags);
GSA_API int gsa_get_kernel_times(gsa_ctx *ctx, float *ms, const char **names, int cap);

/* Synchronise the context's last stream and return (then clear) the device
 * error word: GSA_OK, GSA_ERR_DEVICE_BOUNDS or GSA_ERR_DEVICE_TIMEOUT. */
GSA_API int gsa_get_status(gsa_ctx *ctx);

/* Static text for a status code. */
GSA_API const char *gsa_strerror(int code);

/* Failure-detection self-test (the notes describe no counterpart).  Launches,
 * asynchronously on `stream`, one CTA that waits on an mbarrier nothing ever
 * completes, with the same bounded polling as the layer's kernels; the wait
 * gives up after limit_us microseconds of global time (1 .. 1,000,000) and
 * records GSA_ERR_DEVICE_TIMEOUT in the context's error word.  Nothing faults
 * or hangs, and the context stays usable: gsa_get_status then returns (and
 * clears) GSA_ERR_DEVICE_TIMEOUT, and later calls run normally.  With ctx NULL
 * the code goes to the status word of the allocation-free calls on the
 * current device instead (read with gsa_special_attention_noalloc_status).
 * Returns GSA_ERR_INVALID_ARG for a limit out of range (checked before any
 * CUDA call), GSA_ERR_CUDA if the launch fails. */
GSA_API int gsa_debug_expire_wait(gsa_ctx *ctx, unsigned int limit_us, void *stream);

/* Free the workspace and the context; NULL is accepted. */
GSA_API void gsa_destroy(gsa_ctx *ctx);

/* ---- allocation-free variant -------------------------------------------------
 * The notes describe no counterpart of this entry point; it serves callers that
 * cannot call cudaMalloc: a host program or serving engine that reserves all
 * device memory up front and hands the layer only its inputs and outputs, or a
 * latency-critical loop where an allocation's implicit synchronisation is not
 * acceptable.
 *
 * gsa_special_attention_noalloc computes the special-token output of
 * gsa_forward (every special token attends to every special token and every
 * valid image token, scale softmax_scale or 1/sqrt(64) when 0) for bf16
 * tensors with the layouts of gsa_forward:
 *   q_spec, k_spec, v_spec, o_spec : [H][F][num_special][64]
 *   k_img, v_img                   : [H][F][pad_h][pad_w][64]
 * It creates no context and allocates no memory: the per-split partial results
 * live in one static device array of GSA_NOALLOC_SCRATCH_BYTES per GPU, held
 * by every GPU that loads the library until the process exits.
 *   - The first call on a device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture.
 *   - All calls share the array and find the previous call's contents there;
 *     calls that overlap on the GPU race, so issue them on one stream (or
 *     otherwise serialise them).
 *   - Returns GSA_ERR_UNSUPPORTED, without launching anything, when the
 *     partials (256 + n_split * H * F * num_special * 264 bytes, n_split chosen
 *     as in gsa_forward) would exceed the array; GSA_ERR_INVALID_ARG for NULL
 *     pointers or bad sizes; GSA_ERR_CUDA if a launch fails.
 *   - Device-side errors (a bounded wait that ran out, a failed index check)
 *     are recorded in a status word inside the array, not returned here: read
 *     them with gsa_special_attention_noalloc_status.  The word stays set until
 *     read, and while it is set later calls stop early.
 *   - On a padded grid (pad_h > grid_h or pad_w > grid_w) the kernel derives
 *     the image keys' validity per key tile, because there is no workspace for
 *     the per-tile validity table that gsa_forward builds at create; such
 *     calls take longer than gsa_forward's special-token step (about 2x at 256
 *     frames of a 37x37 grid stored as 40x40). */
#define GSA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
GSA_API int gsa_special_attention_noalloc(const void *q_spec, const void *k_spec, const void *v_spec,
                                          const void *k_img, const void *v_img, void *o_spec,
                                          int num_heads, int num_frames, int num_special,
                                          int grid_h, int grid_w, int pad_h, int pad_w,
                                          float softmax_scale, void *stream);

/* Status of the allocation-free calls on the current device: synchronises
 * `stream`, returns the device status word (GSA_OK, GSA_ERR_DEVICE_TIMEOUT or
 * GSA_ERR_DEVICE_BOUNDS) and clears it.  Allocates nothing.  Returns
 * GSA_ERR_CUDA if a CUDA call fails. */
GSA_API int gsa_special_attention_noalloc_status(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* GSA_B200_H */
