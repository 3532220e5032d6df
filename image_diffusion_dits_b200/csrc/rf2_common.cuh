// Shared host/device definitions of the sm_100a block-sparse attention library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "rf2.h"

namespace rf2 {

// Derived geometry of one call (host-computed, passed to kernels by value).
// Blocks are (wt, wh, ww) windows of the grid padded at the high end of each axis,
// numbered row-major over (t/wt, h/wh, w/ww); tokens inside a window are row-major
// over (t%wt, h%wh, w%ww) ("3D window permutation", RainFusion2.0 TL;DR).
struct Geo {
  int B, heads, T, H, W, D, wt, wh, ww;
  int nbt, nbh, nbw;  // windows per axis
  int Nb, blk;        // blocks, tokens per block
  long long N, Npad;  // real tokens, padded tokens (per batch)
  int nsink;          // blocks that hold a token of frame 0 (the first-frame sink)
};

inline Geo make_geo(const rf2_geom& g) {
  Geo o;
  o.B = g.B; o.heads = g.heads; o.T = g.T; o.H = g.H; o.W = g.W; o.D = g.D;
  o.wt = g.wt; o.wh = g.wh; o.ww = g.ww;
  o.nbt = (g.T + g.wt - 1) / g.wt;
  o.nbh = (g.H + g.wh - 1) / g.wh;
  o.nbw = (g.W + g.ww - 1) / g.ww;
  o.Nb = o.nbt * o.nbh * o.nbw;
  o.blk = g.wt * g.wh * g.ww;
  o.N = (long long)g.T * g.H * g.W;
  o.Npad = (long long)o.Nb * o.blk;
  o.nsink = o.nbh * o.nbw;  // temporal window 0
  return o;
}

// Geometry of a call with `flags`.  RF2_NO_PERMUTE ("without 3D permutation" ablation,
// sciencestack page, Figure 3 (b)): blocks are blk consecutive raster tokens, i.e. the
// flat grid (1, 1, N) cut into (1, 1, blk) windows; the sink is the blocks holding a
// frame-0 token.  The caller checks that N fits an int (N < 2^31 follows from the
// coordinate limit of the kernels).
inline Geo make_call_geo(const rf2_geom& g, unsigned flags) {
  if (!(flags & RF2_NO_PERMUTE)) return make_geo(g);
  rf2_geom f = g;
  f.T = 1; f.H = 1; f.W = g.T * g.H * g.W;
  f.wt = 1; f.wh = 1; f.ww = g.wt * g.wh * g.ww;
  Geo o = make_geo(f);
  const long long frame = (long long)g.H * g.W;
  const long long ns = (frame + o.blk - 1) / o.blk;
  o.nsink = (int)(ns < o.Nb ? ns : o.Nb);
  return o;
}

// Raster token of permuted position p (within one batch), or -1 for a pad position.
__host__ __device__ __forceinline__ long long pos_to_token(const Geo& g, long long p) {
  int block = (int)(p / g.blk);
  int off = (int)(p - (long long)block * g.blk);
  int per_t = g.nbh * g.nbw;
  int tb = block / per_t;
  int rem = block - tb * per_t;
  int hb = rem / g.nbw;
  int wb = rem - hb * g.nbw;
  int whw = g.wh * g.ww;
  int dt = off / whw;
  int r2 = off - dt * whw;
  int dh = r2 / g.ww;
  int dw = r2 - dh * g.ww;
  int t = tb * g.wt + dt, h = hb * g.wh + dh, w = wb * g.ww + dw;
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return ((long long)t * g.H + h) * g.W + w;
}

// Permuted position of raster token n (within one batch).
__host__ __device__ __forceinline__ long long token_to_pos(const Geo& g, long long n) {
  int w = (int)(n % g.W);
  long long th = n / g.W;
  int h = (int)(th % g.H);
  int t = (int)(th / g.H);
  int block = ((t / g.wt) * g.nbh + h / g.wh) * g.nbw + w / g.ww;
  int off = ((t % g.wt) * g.wh + h % g.wh) * g.ww + w % g.ww;
  return (long long)block * g.blk + off;
}

// Real tokens of block j and, per axis, how many of the window's rows are real.
__host__ __device__ __forceinline__ void block_extent(const Geo& g, int j, int& nt, int& nh,
                                                      int& nw) {
  int per_t = g.nbh * g.nbw;
  int tb = j / per_t;
  int rem = j - tb * per_t;
  int hb = rem / g.nbw;
  int wb = rem - hb * g.nbw;
  nt = min(g.wt, g.T - tb * g.wt);
  nh = min(g.wh, g.H - hb * g.wh);
  nw = min(g.ww, g.W - wb * g.ww);
}

// Scratch of the mask prediction (after the call's status word): the bf16 parts of the
// block means of Q and K, then the pooled scores.  Shared by rf2_predict_mask and
// rf2_predict_mask_noalloc.
struct MaskScratch {
  __nv_bfloat16* q3;
  __nv_bfloat16* k3;
  float* scores;
  size_t bytes;
};

inline MaskScratch mask_scratch_layout(const Geo& g, unsigned char* base) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t parts = up((size_t)3 * g.B * g.heads * g.Nb * g.D * sizeof(__nv_bfloat16));
  MaskScratch m;
  m.q3 = reinterpret_cast<__nv_bfloat16*>(base);
  m.k3 = reinterpret_cast<__nv_bfloat16*>(base + parts);
  m.scores = reinterpret_cast<float*>(base + 2 * parts);
  m.bytes = 2 * parts + up((size_t)g.B * g.heads * g.Nb * g.Nb * sizeof(float));
  return m;
}

// Arguments of the RainFusion v1 generators (host-derived, passed by value).  Sample p = 0
// is the local sample (the H*W frame-0 tokens), p = 1 the global one (every omega-th
// raster token).  R[p][l] is the band radius of level l = (static bandwidth, 1/8, 1/4,
// 1/2) on that sample's axis (windows of a slab for p = 0, temporal blocks for p = 1).
struct Rf1Args {
  int S[2];           // sample slots (the local sample may hold pad slots, see wslots)
  int S_real[2];      // real samples (the mean's denominator)
  int coord_off[2];   // offsets of each sample's coordinates in the coordinate table
  int wslots;         // > 0: the local sample is ordered window by window, wslots = wh*ww
                      // slots per window (pad slots of partial windows included)
  int T;
  int tiles_max;      // max over p of ceil(S[p] / 128)
  int omega, HW, W, wh, ww, nbw, wt, heads;
  int R[2][4];
  int tau, dynamic;
  float alpha, target, scale_log2;
};

// Scratch of the v1 generators (after the call's status word).
struct Rf1Scratch {
  int* coords;       // [S0 + S1] window coordinate of every sampled token
  float* partial;    // [B*heads][2][tiles_max][4 warps][4 levels]
  int* clsparam;     // [B*heads][2]: class, radius or stride
  size_t bytes;
};

inline Rf1Scratch rf1_scratch_layout(const Geo& g, const Rf1Args& a, unsigned char* base) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  Rf1Scratch w;
  size_t off = 0;
  w.coords = reinterpret_cast<int*>(base + off);
  off += up((size_t)(a.S[0] + a.S[1]) * sizeof(int));
  w.partial = reinterpret_cast<float*>(base + off);
  off += up((size_t)g.B * g.heads * 2 * a.tiles_max * 16 * sizeof(float));
  w.clsparam = reinterpret_cast<int*>(base + off);
  off += up((size_t)g.B * g.heads * 2 * sizeof(int));
  w.bytes = off;
  return w;
}

// cuTensorMapEncodeTiled from the driver (looked up once), or null if unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Device status word values (match rf2_status).
constexpr int kStatusBadIndex = RF2_ERR_BAD_INDEX;
constexpr int kStatusTimeout = RF2_ERR_TIMEOUT;

// Launchers (defined in the kernel files, called by the C ABI layer).
cudaError_t launch_permute(const void* x, void* xp, const Geo& g, cudaStream_t s);
cudaError_t launch_unpermute(const void* xp, void* x, const Geo& g, cudaStream_t s);
// Block means of Q and K, each written as three bf16 parts hi + mid + lo (about 24
// significant bits together) in [3][B*heads*Nb][D] layout for the tensor-core scores.
// raster: Q and K in model order [B, N, heads, D], else window order [B, Npad, heads, D].
cudaError_t launch_pool(const void* qp, const void* kp, __nv_bfloat16* q3, __nv_bfloat16* k3, const Geo& g,
                        bool raster, cudaStream_t s);
// Pooled scores s = qbar . kbar * scale from the bf16 parts (tcgen05); status (may be
// null) receives RF2_ERR_TIMEOUT if a wait ran out.
cudaError_t launch_scores(const __nv_bfloat16* q3, const __nv_bfloat16* k3, float* scores, const Geo& g,
                          float scale, int nsink, int32_t* status, cudaStream_t s);
cudaError_t launch_topk(const float* scores, int32_t* idx, int32_t* cnt, int kmax, int kept,
                        int nsink, const Geo& g, cudaStream_t s);
// Returns cudaErrorNotSupported when the shape has no kernel instance.  raster: Q/K/V
// and O in model order [B, N, heads, D] (windows gathered and scattered in place), else
// window order [B, Npad, heads, D].
cudaError_t launch_sparse_attn(const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* cnt, int kmax, const Geo& g,
                               float scale, void* op, int32_t* status, bool raster, cudaStream_t s);

// e4m3 variant: per-(batch, head, block) quantisation of model-order Q, K, V into e4m3
// model-order tensors and scales [3][B][heads][Nb]; attention over them (D = 128,
// 128-token blocks, model order; cudaErrorNotSupported otherwise).
cudaError_t launch_quant_fp8(const void* q, const void* k, const void* v, uint8_t* q8, uint8_t* k8, uint8_t* v8,
                             float* scales, const Geo& g, cudaStream_t s);
cudaError_t launch_sparse_attn_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                   const int32_t* idx, const int32_t* cnt, int kmax, const Geo& g, float scale,
                                   void* op, int32_t* status, cudaStream_t s);

// RainFusion v1: ARM recall of the two samples, head classes, kept lists.  q, k in model
// order [B, N, heads, D].  cls_out [B*heads] and recall_out [B*heads][2][4] may be null.
cudaError_t launch_rf1(const void* q, const void* k, const Geo& g, const Rf1Args& a, const Rf1Scratch& w,
                       int32_t* cls_out, float* recall_out, int32_t* idx, int32_t* cnt, int kmax,
                       int32_t* status, cudaStream_t s);

}  // namespace rf2
