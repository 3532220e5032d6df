/*
 * rf2.h - C ABI of the B200 (sm_100a) block-sparse attention library (librf2.so).
 *
 * The library computes the online block-sparse attention of RainFusion2.0
 * ("RainFusion2.0: Temporal-Spatial Awareness and Hardware-Efficient Block-wise Sparse
 * Attention"): a 3D-window token permutation of a [T, H, W] latent token grid, block-mean
 * representative tokens for Q and K, a pooled block-level score that selects, per
 * (batch, head, query block), the key blocks to keep at a target sparsity, a first-frame
 * sink that always keeps the key blocks of the first temporal window, attention over the
 * kept blocks only, and the inverse permutation.  Passages that define each step are
 * cited per entry point below (mlsanity index page, Abstract, the three key technical
 * insights (1)-(3); sciencestack page, TL;DR and Figures 1-3).  The pages give no formulas; the
 * readings used here are stated with each call.
 *
 * Conventions (every entry point):
 *  - Tensors are device pointers to contiguous row-major arrays.  Q/K/V/O in model order
 *    are [B, N, heads, D] bf16 with N = T*H*W tokens in raster (t, h, w) order.  Permuted
 *    tensors are [B, Npad, heads, D] bf16, Npad = Nb*blk, tokens in window order.
 *  - The caller owns every buffer.  No entry point allocates memory or synchronises
 *    the stream, except that RF2_CHECKED makes a call wait for its own work on `stream`
 *    and read the device status word back.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  All work
 *    is asynchronous on it.
 *  - Arguments are validated on the host before any launch; an invalid call returns an
 *    error and launches nothing.  Device pointers must be 16-byte aligned.
 *  - Supported: D in {64, 128}; blk = wt*wh*ww in {64, 128}; B, heads, T, H, W >= 1.
 *  - Return value: RF2_OK or an rf2_status error code.  A CUDA launch error maps to
 *    RF2_ERR_CUDA.
 */
#ifndef RF2_H
#define RF2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Geometry of one attention call.  The grid is padded at the high end of each axis to
 * window multiples: Tp = ceil(T/wt)*wt (same for H, W).  Blocks are windows numbered
 * row-major over (t/wt, h/wh, w/ww); Nb = (Tp/wt)*(Hp/wh)*(Wp/ww), blk = wt*wh*ww. */
typedef struct rf2_geom {
    int B, heads, T, H, W, D, wt, wh, ww;
} rf2_geom;

enum rf2_status {
    RF2_OK = 0,
    RF2_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, kmax too small ...   */
    RF2_ERR_UNSUPPORTED = 2,  /* D or block size outside the supported set              */
    RF2_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned                       */
    RF2_ERR_WORKSPACE = 4,    /* workspace missing or smaller than the size query says  */
    RF2_ERR_BAD_INDEX = 5,    /* a block index outside [0, Nb) (detected on device)      */
    RF2_ERR_TIMEOUT = 6,      /* a bounded device wait gave up (detected on device)      */
    RF2_ERR_CUDA = 7          /* a CUDA runtime error                                   */
};

enum rf2_flags {
    /* Sink outside the budget: kept = |S| + ceil((1-s)*(Nb-|S|) - 1e-6).  Default is the
     * in-budget reading: kept = max(ceil((1-s)*Nb - 1e-6) clamped to [1,Nb], |S|). */
    RF2_SINK_ADDITIVE = 1u,
    /* Wait for the call's work on `stream` and return the device status word. */
    RF2_CHECKED = 2u,
    /* rf2_predict_mask and rf2_sparse_attn: Q, K, V and O are in model order
     * [B, N, heads, D] (the tensors rf2_permute would take) instead of window order
     * [B, Npad, heads, D].  The kernels then gather each 3D window straight from model
     * order (pad tokens read as zeros) and write O rows to their tokens; the results are
     * those of the window-order call on rf2_permute'd inputs, bit for bit. */
    RF2_RASTER = 4u,
    /* The "without 3D permutation" ablation (sciencestack page, Figure 3 (b)): a block is
     * blk = wt*wh*ww consecutive tokens of model (raster) order instead of a 3D window.
     * Every entry point that takes flags then works on the flat geometry T' = H' = 1,
     * W' = N with window (1, 1, blk): Nb = ceil(N/blk), Npad = Nb*blk (the last block is
     * padded at its end), and "window order" is model order padded to Npad rows.  The
     * first-frame sink becomes the blocks that hold a token of frame 0, the first
     * ceil(H*W/blk) blocks.  rf2_permute and rf2_unpermute take no flags and keep
     * the 3D windows. */
    RF2_NO_PERMUTE = 8u,
    /* rf2_attention: quantise Q, K and V to e4m3 (rf2_quantize_fp8) after the mask
     * prediction and attend with rf2_sparse_attn_fp8.  D = 128 and 128-token blocks only. */
    RF2_FP8 = 16u
};

/* rf2_permute - 3D window permutation (mlsanity index page, Abstract, insight (2): tokens
 * are reordered so that each block is a spatio-temporal window; sciencestack page, TL;DR
 * and Figure 3).
 *   x  : [B, N, heads, D] bf16, raster order (read).
 *   xp : [B, Npad, heads, D] bf16 (written).  Token (t,h,w) goes to position
 *        block*blk + ((t%wt)*wh + h%wh)*ww + w%ww, block = ((t/wt)*(Hp/wh) + h/wh)*(Wp/ww)
 *        + w/ww.  Pad positions are written with zeros.
 * Errors: RF2_ERR_INVALID_ARG, RF2_ERR_UNSUPPORTED, RF2_ERR_ALIGNMENT, RF2_ERR_CUDA. */
int rf2_permute(const void* x, void* xp, const rf2_geom* g, void* stream);

/* rf2_unpermute - inverse of rf2_permute; pad positions are dropped.
 *   xp : [B, Npad, heads, D] bf16 (read).   x : [B, N, heads, D] bf16 (written). */
int rf2_unpermute(const void* xp, void* x, const rf2_geom* g, void* stream);

/* rf2_kept_count - number of key blocks every (b, head, query block) row keeps
 * (sciencestack page, TL;DR: target sparsity; mlsanity index page, insight (3): the
 * first-frame sink).  The sink S is the Hp/wh * Wp/ww blocks of temporal window 0 when
 * `sink` is non-zero (with RF2_NO_PERMUTE: the ceil(H*W/blk) blocks that hold frame 0).  Returns the count (>= 1) or -RF2_ERR_* on a bad argument.
 * This is the minimum `kmax` of rf2_predict_mask. */
int rf2_kept_count(const rf2_geom* g, double sparsity, int sink, unsigned flags);

/* rf2_workspace_size - bytes of device workspace that rf2_predict_mask (attention = 0)
 * or rf2_attention (attention = 1) needs for this geometry, sparsity and flags.  The
 * workspace holds a status word, the block means (three bf16 parts each), the pooled
 * scores and, for rf2_attention, the kept lists and counts.  Returns 0 on a bad
 * argument. */
size_t rf2_workspace_size(const rf2_geom* g, double sparsity, int sink, unsigned flags,
                          int attention);

/* rf2_predict_mask - online mask prediction on permuted Q and K (mlsanity index page,
 * Abstract, insight (1): block means stand in for the tokens when the mask is predicted;
 * insight (3): the first-frame sink).
 *   qp, kp : [B, Npad, heads, D] bf16, window order (read).  Pad positions are ignored.
 *            With RF2_RASTER: [B, N, heads, D], model order.
 *   Steps: qbar_i, kbar_j = fp32 mean over the real tokens of each block, per head;
 *   s_ij = qbar_i . kbar_j / sqrt(D) with fp32 accumulation (on the tensor cores, from
 *   each mean split into three bf16 parts; relative error about 1e-6); each row keeps
 *   the sink blocks plus the highest-scoring other blocks (ties to the lower id) up to
 *   rf2_kept_count.
 *   idx : [B, heads, Nb, kmax] int32 (written): ascending kept block ids, then -1.
 *   cnt : [B, heads, Nb] int32 (written): the kept count of each row.
 *   kmax >= rf2_kept_count(...) else RF2_ERR_INVALID_ARG.
 *   ws, ws_bytes : device scratch of at least rf2_workspace_size(..., 0) bytes.
 * Errors: RF2_ERR_INVALID_ARG, RF2_ERR_UNSUPPORTED, RF2_ERR_ALIGNMENT, RF2_ERR_WORKSPACE,
 *         RF2_ERR_CUDA. */
int rf2_predict_mask(const void* qp, const void* kp, const rf2_geom* g, double sparsity,
                     int sink, unsigned flags, int32_t* idx, int32_t* cnt, int kmax,
                     void* ws, size_t ws_bytes, void* stream);

/* Size of the fixed device scratch of rf2_predict_mask_noalloc (16 MiB). */
#define RF2_NOALLOC_SCRATCH_BYTES (16u << 20)

/* rf2_predict_mask_noalloc - rf2_predict_mask for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a deployment variant, not a step of
 * the method.  Some callers may not call cudaMalloc at all (code inside a framework that
 * owns every device allocation, or a plug-in that must not allocate after start-up), so
 * they cannot supply the `ws` scratch.  This call computes exactly what rf2_predict_mask
 * computes, with its scratch taken from a fixed file-scope device array of
 * RF2_NOALLOC_SCRATCH_BYTES instead; it allocates nothing.
 *   Arguments: as rf2_predict_mask, without ws/ws_bytes.  The caller still owns qp, kp,
 *   idx and cnt.
 *   Limit: the geometry's rf2_workspace_size(g, sparsity, sink, flags, 0) must not exceed
 *   RF2_NOALLOC_SCRATCH_BYTES, else the call returns RF2_ERR_WORKSPACE and launches
 *   nothing.  (The tiny, 480p and image-edit shapes fit; the 720p and long-video ones do
 *   not.)
 *   Set-up: the first call on a device looks up the array's device address with that
 *   device current (cudaGetSymbolAddress); make that first call before any stream
 *   capture.
 *   Sharing: the array exists on every GPU that loads the library until the process
 *   exits, and all calls on a device share it.  Each call clears its status word and
 *   writes all the other scratch it reads before reading it; calls that overlap on the
 *   GPU (other streams or host threads on the same device) race and must be serialised.
 * Errors: as rf2_predict_mask. */
int rf2_predict_mask_noalloc(const void* qp, const void* kp, const rf2_geom* g,
                             double sparsity, int sink, unsigned flags, int32_t* idx,
                             int32_t* cnt, int kmax, void* stream);

/* rf2_sparse_attn - block-sparse attention over the kept blocks (mlsanity index page,
 * title "block-wise sparse attention"; Abstract: skipping the computation of
 * insignificant tokens).  For each (b, head, query block i):
 *   O_i = softmax(Q_i K_S^T * scale + M) V_S over the tokens of the kept blocks
 *   S = idx[b, head, i, 0..cnt-1]; M = -inf on pad keys, 0 elsewhere.
 *   qp, kp, vp : [B, Npad, heads, D] bf16 (read).   op : [B, Npad, heads, D] bf16
 *   (written; pad query rows are written too, with values of no meaning).
 *   With RF2_RASTER: qp, kp, vp, op are [B, N, heads, D] in model order; every row of op
 *   is written.
 *   scale : softmax scale, > 0; 0 means 1/sqrt(D) (negative: RF2_ERR_INVALID_ARG).
 *   Softmax statistics and the accumulator
 *   are fp32; exp2 is taken in fp32 and P rounded to bf16 for the P.V product.
 *   status : optional device int32 (may be NULL); when given it must be zero on entry
 *   and receives RF2_ERR_BAD_INDEX / RF2_ERR_TIMEOUT if the kernel detects one
 *   (out-of-range ids are skipped, never dereferenced).  With RF2_CHECKED and a status
 *   word the call waits for the stream and returns that code.
 * Errors: RF2_ERR_INVALID_ARG, RF2_ERR_UNSUPPORTED, RF2_ERR_ALIGNMENT, RF2_ERR_CUDA,
 *         and (checked mode) RF2_ERR_BAD_INDEX, RF2_ERR_TIMEOUT. */
int rf2_sparse_attn(const void* qp, const void* kp, const void* vp, const int32_t* idx,
                    const int32_t* cnt, int kmax, const rf2_geom* g, float scale, void* op,
                    int32_t* status, unsigned flags, void* stream);

/* rf2_attention - the whole path (sciencestack page, Figure 1 "Workflow of
 * RainFusion2.0"): predict mask -> block-sparse attention, both on model-order tensors
 * (the 3D window permutation and its inverse are done by the kernels' window gathers
 * and row scatters, with no permuted copies).
 *   q, k, v : [B, N, heads, D] bf16 (read).   o : [B, N, heads, D] bf16 (written).
 *   idx_out : optional [B, heads, Nb, kept] int32 copy of the kept lists (may be NULL).
 *   ws, ws_bytes : device scratch of at least rf2_workspace_size(..., 1) bytes (with
 *   RF2_FP8 it also holds the e4m3 copies of Q, K, V and their scales).
 * Errors: as rf2_predict_mask and rf2_sparse_attn. */
int rf2_attention(const void* q, const void* k, const void* v, const rf2_geom* g,
                  double sparsity, int sink, float scale, void* o, int32_t* idx_out,
                  void* ws, size_t ws_bytes, unsigned flags, void* stream);

/* e4m3 variant of the attention.  The sciencestack page's TL;DR points to integrating
 * quantisation with the block-sparse attention for further speed; the FP8 form below is
 * this library's reading.  Every (batch, head,
 * block) of Q, K and V gets one scale: amax = max |x| over the block's real tokens and
 * the head's D channels, inv = 448 / amax, scale = amax / 448 (fp32, rounded to
 * nearest; amax = 0 gives 0 for both); code = e4m3(x * inv) with round to nearest even
 * and saturation to +-448.
 *
 * rf2_quantize_fp8 - q, k, v : [B, N, heads, D] bf16, model order (read).
 *   q8, k8, v8 : [B, N, heads, D] e4m3 codes, model order (written).
 *   scales : [3][B][heads][Nb] float (written): Q, K, V scales in that order.
 *   Every pointer 16-byte aligned.
 *   flags : RF2_NO_PERMUTE selects raster blocks.  Errors: RF2_ERR_INVALID_ARG,
 *   RF2_ERR_UNSUPPORTED, RF2_ERR_ALIGNMENT, RF2_ERR_CUDA. */
int rf2_quantize_fp8(const void* q, const void* k, const void* v, const rf2_geom* g, unsigned flags,
                     void* q8, void* k8, void* v8, float* scales, void* stream);

/* rf2_sparse_attn_fp8 - block-sparse attention over e4m3 operands (tcgen05 kind::f8f6f4):
 *   S = (Q8 K8_j^T) * sq * sk_j * scale with fp32 accumulation; P = exp2 of the scores
 *   minus the running max (fp32 row sums), multiplied by sv_j / max sv over the row's kept
 *   blocks and rounded to e4m3; O = (sum_j P_j V8_j) * max sv / l, written as bf16.
 *   q8, k8, v8 : [B, N, heads, 128] e4m3, model order; scales as rf2_quantize_fp8 writes
 *   them; idx, cnt, kmax, status as rf2_sparse_attn; o : [B, N, heads, 128] bf16.
 *   D = 128 and 128-token blocks only (else RF2_ERR_UNSUPPORTED).
 * Errors: as rf2_sparse_attn. */
int rf2_sparse_attn_fp8(const void* q8, const void* k8, const void* v8, const float* scales,
                        const int32_t* idx, const int32_t* cnt, int kmax, const rf2_geom* g, float scale,
                        void* o, int32_t* status, unsigned flags, void* stream);

/* Step schedule of the attention calls of one generation.  RainFusion v1 keeps the first
 * 10 % of the diffusion timesteps dense (pith.science review, "Free parameters": dense
 * timestep fraction); RainFusion2.0 predicts its mask online, on every step.  Reusing a
 * predicted mask for a few steps is a deployment option the pages do not describe. */
typedef struct rf2_schedule {
    int total_steps;        /* diffusion steps of one generation, >= 1                    */
    double dense_fraction;  /* leading fraction of steps run dense, in [0, 1] (pages: 0.1)  */
    int predict_interval;   /* a new mask every this many sparse steps, >= 1 (1: every step) */
} rf2_schedule;

enum rf2_step_action {
    RF2_STEP_DENSE = 0,    /* all blocks kept: rf2_attention with sparsity 0              */
    RF2_STEP_PREDICT = 1,  /* predict a new mask (rf2_predict_mask) and attend with it     */
    RF2_STEP_REUSE = 2     /* attend with the last predicted kept lists (rf2_sparse_attn)  */
};

/* rf2_schedule_action - the action of step `step` (0-based): the first
 * ceil(dense_fraction * total_steps - 1e-6) steps are dense; after them a new mask is
 * predicted on the first sparse step and every predict_interval-th one, and the steps in
 * between reuse it.  Host only (no device work).  Returns an rf2_step_action or
 * -RF2_ERR_INVALID_ARG on a bad schedule or a step outside [0, total_steps). */
int rf2_schedule_action(const rf2_schedule* schedule, int step);

/* RainFusion (v1) mask generators (pith.science review of "RainFusion: Adaptive Video
 * Generation Acceleration via Multi-Dimensional Visual Redundancy": "What carries the
 * argument", "Core claim", "Free parameters").  They emit kept lists for the same
 * block-sparse attention (rf2_sparse_attn with RF2_RASTER).  Blocks are the 3D windows of
 * rf2_geom; a block's coordinates are its temporal block tb and its window index
 * sw = hb * nbw + wb inside a temporal slab (nbw = Wp/ww, P = nbh * nbw windows per slab).
 * Head patterns, per (query block i, key block j):
 *   temporal, radius R: |sw_i - sw_j| <= R     spatial, radius R: |tb_i - tb_j| <= R
 *   textural, stride tau: (hb_j + wb_j) mod tau == 0 (a checkerboard of windows)
 * with R = floor(b * C + 1e-6) for bandwidth b, C = P (temporal) or Tp/wt (spatial).
 * ARM (adaptive recognition) recall of a band: mean over sampled query tokens of the
 * softmax mass (over the sampled keys, scale 1/sqrt(D)) whose key lies in the band, the
 * band judged on the windows of the two tokens.  Local sample: the H*W tokens of frame 0,
 * scored with the temporal band; global sample: raster tokens 0, omega, 2 omega, ...,
 * scored with the spatial band.  A head is temporal if its local recall at `bandwidth`
 * reaches alpha, else spatial if its global recall does, else textural.  With `dynamic`
 * (RainFusion+), a temporal or spatial head then takes the smallest bandwidth of 1/8,
 * 1/4, 1/2 whose recall reaches recall_target (else 1/2). */
typedef struct rf2_v1_params {
    double bandwidth;      /* band half-width as a fraction of the axis, (0, 1]; pages: 1/4  */
    int tau;               /* checkerboard stride of textural heads, >= 1; pages: 2          */
    double alpha;          /* recall threshold of the classification, [0, 1]; not given: 0.9 */
    int omega;             /* global sampling interval in tokens, >= 0; 0 means T            */
    int dynamic;           /* 1: RainFusion+ bandwidth per head                              */
    double recall_target;  /* RainFusion+ recall target, [0, 1]; pages: 0.9                  */
} rf2_v1_params;

/* Head classes written by rf2_v1_predict_mask. */
enum rf2_v1_class { RF2_V1_TEMPORAL = 0, RF2_V1_SPATIAL = 1, RF2_V1_TEXTURAL = 2 };

/* rf2_v1_kmax - the longest kept list any head class can produce for these parameters
 * (the minimum kmax of rf2_v1_predict_mask), or -RF2_ERR_* on a bad argument.  flags:
 * RF2_NO_PERMUTE is not supported (the patterns are defined on 3D windows). */
int rf2_v1_kmax(const rf2_geom* g, const rf2_v1_params* p, unsigned flags);

/* rf2_v1_workspace_size - device scratch of rf2_v1_predict_mask (status word, sample
 * coordinates, per-warp recall sums, head classes); 0 on a bad argument. */
size_t rf2_v1_workspace_size(const rf2_geom* g, const rf2_v1_params* p, unsigned flags);

/* rf2_v1_predict_mask - ARM classification of every (b, head) and its kept lists, all on
 * the device (no host synchronisation unless RF2_CHECKED).
 *   q, k : [B, N, heads, D] bf16, model order (read).
 *   idx  : [B, heads, Nb, kmax] int32 (written): ascending kept block ids, then -1.
 *   cnt  : [B, heads, Nb] int32 (written): kept count of each row (rows of one head differ
 *          at the band ends).
 *   head_class : optional [B, heads] int32 rf2_v1_class (may be NULL).
 *   recall     : optional [B, heads, 2, 4] float (may be NULL): local then global
 *          sample, levels (bandwidth, 1/8, 1/4, 1/2).
 *   kmax >= rf2_v1_kmax(...) else RF2_ERR_INVALID_ARG.
 *   ws, ws_bytes : device scratch of at least rf2_v1_workspace_size(...) bytes.
 * Errors: RF2_ERR_INVALID_ARG, RF2_ERR_UNSUPPORTED, RF2_ERR_ALIGNMENT, RF2_ERR_WORKSPACE,
 *         RF2_ERR_CUDA, and (checked mode) RF2_ERR_TIMEOUT. */
int rf2_v1_predict_mask(const void* q, const void* k, const rf2_geom* g, const rf2_v1_params* p,
                        unsigned flags, int32_t* idx, int32_t* cnt, int kmax, int32_t* head_class,
                        float* recall, void* ws, size_t ws_bytes, void* stream);

/* rf2_selftest_wait_timeout - diagnostic of the bounded device waits of every kernel.
 * Launches two one-warp CTAs on `stream` that each wait on an mbarrier that nothing
 * arrives at: the first gives up after short_s seconds and writes RF2_ERR_TIMEOUT to
 * *status (a device int32 the caller zeroes first); the second (limit long_s) gives up
 * as soon as it sees that value.  0 < short_s <= long_s <= 5.  Returns RF2_OK once
 * launched (the caller synchronises and reads *status), RF2_ERR_INVALID_ARG or
 * RF2_ERR_CUDA. */
int rf2_selftest_wait_timeout(int32_t* status, double short_s, double long_s, void* stream);

/* rf2_status_string - static, human-readable text of a status code. */
const char* rf2_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* RF2_H */
