// C ABI of the block-sparse attention library: argument validation, workspace layout,
// and the launch sequence of each entry point.  Every compute step runs in the CUDA
// kernels of permute.cu, mask.cu and attn.cu.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include "rf2_common.cuh"

using rf2::Geo;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_geom(const rf2_geom* g, unsigned flags = 0) {
  if (g == nullptr) return RF2_ERR_INVALID_ARG;
  if (g->B < 1 || g->heads < 1 || g->T < 1 || g->H < 1 || g->W < 1 || g->wt < 1 || g->wh < 1 ||
      g->ww < 1 || g->D < 1)
    return RF2_ERR_INVALID_ARG;
  if (g->D != 64 && g->D != 128) return RF2_ERR_UNSUPPORTED;
  const long long blk = (long long)g->wt * g->wh * g->ww;
  if (blk != 64 && blk != 128) return RF2_ERR_UNSUPPORTED;
  const long long n = (long long)g->T * g->H * g->W;
  if ((long long)g->B * (n + blk) >= (1ll << 31)) return RF2_ERR_UNSUPPORTED;  // TMA coordinates
  Geo o = rf2::make_call_geo(*g, flags);
  if (o.Nb > 1024) return RF2_ERR_UNSUPPORTED;                  // kept lists live in smem
  if ((long long)o.B * o.Npad >= (1ll << 31)) return RF2_ERR_UNSUPPORTED;  // TMA coordinates
  return RF2_OK;
}

int nsink_of(const Geo& g, int sink) { return sink ? g.nsink : 0; }

// Kept blocks per row (both sides of the sink reading).  Every block holds at least one
// real token (padding is less than one window per axis), so all Nb blocks are valid.
int kept_of(const Geo& g, double sparsity, int sink, unsigned flags) {
  const int nv = g.Nb;
  const int ns = nsink_of(g, sink);
  if (flags & RF2_SINK_ADDITIVE) {
    long long extra = (long long)ceil((1.0 - sparsity) * (double)(nv - ns) - 1e-6);
    if (extra < 0) extra = 0;
    if (extra > nv - ns) extra = nv - ns;
    return ns + (int)extra;
  }
  long long k = (long long)ceil((1.0 - sparsity) * (double)nv - 1e-6);
  if (k < 1) k = 1;
  if (k > nv) k = nv;
  return (int)(k > ns ? k : ns);
}

struct MaskWs {
  int32_t* status;
  rf2::MaskScratch m;  // bf16 parts of the block means, pooled scores
  size_t bytes;
};

MaskWs mask_ws_layout(const Geo& g, uint8_t* base) {
  MaskWs w;
  w.status = reinterpret_cast<int32_t*>(base);
  w.m = rf2::mask_scratch_layout(g, base + kAlign);
  w.bytes = kAlign + align_up(w.m.bytes);
  return w;
}

struct AttnWs {
  MaskWs mask;
  int32_t *idx, *cnt;
  uint8_t *q8, *k8, *v8;  // RF2_FP8: e4m3 copies of Q, K, V
  float* scales;          // RF2_FP8: [3][B][heads][Nb]
  size_t bytes;
};

AttnWs attn_ws_layout(const Geo& g, int kept, uint8_t* base, unsigned flags = 0) {
  AttnWs w;
  w.mask = mask_ws_layout(g, base);
  size_t off = w.mask.bytes;
  w.idx = reinterpret_cast<int32_t*>(base + off);
  off += align_up((size_t)g.B * g.heads * g.Nb * kept * sizeof(int32_t));
  w.cnt = reinterpret_cast<int32_t*>(base + off);
  off += align_up((size_t)g.B * g.heads * g.Nb * sizeof(int32_t));
  w.q8 = w.k8 = w.v8 = nullptr;
  w.scales = nullptr;
  if (flags & RF2_FP8) {
    const size_t t8 = align_up((size_t)g.B * g.N * g.heads * g.D);
    w.q8 = base + off;
    w.k8 = base + off + t8;
    w.v8 = base + off + 2 * t8;
    off += 3 * t8;
    w.scales = reinterpret_cast<float*>(base + off);
    off += align_up((size_t)3 * g.B * g.heads * g.Nb * sizeof(float));
  }
  w.bytes = off;
  return w;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? RF2_OK : RF2_ERR_CUDA; }

bool log_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* s = getenv("RF2_LOG");
    v = (s != nullptr && s[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

void log_geo(const char* what, const Geo& g, int kept) {
  if (!log_enabled()) return;
  fprintf(stderr,
          "[rf2] %s B=%d heads=%d grid=%dx%dx%d D=%d window=%dx%dx%d Nb=%d blk=%d Npad=%lld "
          "kept=%d\n",
          what, g.B, g.heads, g.T, g.H, g.W, g.D, g.wt, g.wh, g.ww, g.Nb, g.blk, g.Npad, kept);
}

// In checked mode: wait for the stream and return the device status word.
int finish_checked(unsigned flags, const int32_t* status_dev, cudaStream_t s) {
  if (!(flags & RF2_CHECKED)) return RF2_OK;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  if (status_dev == nullptr) return RF2_OK;
  int32_t st = 0;
  e = cudaMemcpyAsync(&st, status_dev, sizeof(st), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  return st;
}

// RainFusion v1 generators: validated arguments, kernel arguments and kmax.
struct V1Call {
  Geo geo;
  rf2::Rf1Args a;
  int kmax;
};

int v1_radius(double bw, int C) { return (int)floor(bw * (double)C + 1e-6); }

int v1_prepare(const rf2_geom* g, const rf2_v1_params* p, unsigned flags, V1Call* c) {
  int st = check_geom(g, 0);
  if (st != RF2_OK) return st;
  if (flags & RF2_NO_PERMUTE) return RF2_ERR_UNSUPPORTED;
  if (p == nullptr || !(p->bandwidth > 0.0 && p->bandwidth <= 1.0) || p->tau < 1 ||
      !(p->alpha >= 0.0 && p->alpha <= 1.0) || !(p->recall_target >= 0.0 && p->recall_target <= 1.0) ||
      p->omega < 0 || (p->dynamic != 0 && p->dynamic != 1))
    return RF2_ERR_INVALID_ARG;
  Geo geo = rf2::make_geo(*g);
  if ((long long)geo.B * geo.heads > 65535) return RF2_ERR_UNSUPPORTED;  // grid z
  rf2::Rf1Args a;
  const long long omega = p->omega == 0 ? g->T : p->omega;
  // The local sample (frame 0) goes window by window when a tile holds whole windows,
  // so that 32 consecutive keys share a window; pad slots of partial windows are skipped.
  const int wslots = g->wh * g->ww;
  a.wslots = (wslots == 32 || wslots == 64 || wslots == 128) ? wslots : 0;
  a.S_real[0] = g->H * g->W;
  a.S[0] = a.wslots ? geo.nbh * geo.nbw * a.wslots : a.S_real[0];
  a.S[1] = a.S_real[1] = (int)((geo.N + omega - 1) / omega);
  a.T = g->T;
  a.coord_off[0] = 0;
  a.coord_off[1] = a.S[0];
  a.tiles_max = (max(a.S[0], a.S[1]) + 127) / 128;
  a.omega = (int)omega;
  a.HW = g->H * g->W;
  a.W = g->W; a.wh = g->wh; a.ww = g->ww; a.nbw = geo.nbw; a.wt = g->wt; a.heads = g->heads;
  const double levels[4] = {p->bandwidth, 0.125, 0.25, 0.5};
  const int P = geo.nbh * geo.nbw;
  for (int l = 0; l < 4; ++l) {
    a.R[0][l] = v1_radius(levels[l], P);
    a.R[1][l] = v1_radius(levels[l], geo.nbt);
  }
  a.tau = p->tau;
  a.dynamic = p->dynamic;
  a.alpha = (float)p->alpha;
  a.target = (float)p->recall_target;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g->D));
  // longest list: temporal nbt * min(P, 2R+1), spatial min(nbt, 2R+1) * P, textural
  // nbt * (windows of a slab on the checkerboard)
  int kmax = 0;
  for (int l = 0; l < (p->dynamic ? 4 : 1); ++l) {
    kmax = max(kmax, geo.nbt * min(P, 2 * a.R[0][l] + 1));
    kmax = max(kmax, min(geo.nbt, 2 * a.R[1][l] + 1) * P);
  }
  int tex = 0;
  for (int sw = 0; sw < P; ++sw) tex += ((sw / geo.nbw + sw % geo.nbw) % p->tau) == 0;
  kmax = max(kmax, geo.nbt * tex);
  c->geo = geo;
  c->a = a;
  c->kmax = kmax;
  return RF2_OK;
}

size_t v1_ws_bytes(const V1Call& c) {
  return kAlign + align_up(rf2::rf1_scratch_layout(c.geo, c.a, nullptr).bytes);
}

}  // namespace

extern "C" {

int rf2_quantize_fp8(const void* q, const void* k, const void* v, const rf2_geom* g, unsigned flags,
                     void* q8, void* k8, void* v8, float* scales, void* stream) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || q8 == nullptr || k8 == nullptr || v8 == nullptr ||
      scales == nullptr)
    return RF2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) || !aligned16(v8) ||
      ((uintptr_t)scales & 3u))
    return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_call_geo(*g, flags);
  log_geo("quantize_fp8", geo, 0);
  cudaError_t e = rf2::launch_quant_fp8(q, k, v, static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8),
                                        static_cast<uint8_t*>(v8), scales, geo, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RF2_ERR_UNSUPPORTED;
  return cuda_status(e);
}

int rf2_sparse_attn_fp8(const void* q8, const void* k8, const void* v8, const float* scales,
                        const int32_t* idx, const int32_t* cnt, int kmax, const rf2_geom* g, float scale,
                        void* o, int32_t* status, unsigned flags, void* stream) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return st;
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || scales == nullptr || idx == nullptr || cnt == nullptr ||
      o == nullptr || kmax < 1 || !isfinite(scale) || scale < 0.f)
    return RF2_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || ((uintptr_t)scales & 3u) ||
      ((uintptr_t)idx & 3u) || ((uintptr_t)cnt & 3u) || ((uintptr_t)status & 3u))
    return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_call_geo(*g, flags);
  const float sc = scale == 0.f ? (float)(1.0 / sqrt((double)geo.D)) : scale;
  log_geo("sparse_attn_fp8", geo, kmax);
  cudaError_t e = rf2::launch_sparse_attn_fp8(static_cast<const uint8_t*>(q8), static_cast<const uint8_t*>(k8),
                                              static_cast<const uint8_t*>(v8), scales, idx, cnt, kmax, geo, sc, o,
                                              status, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RF2_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  return finish_checked(flags, status, (cudaStream_t)stream);
}

int rf2_v1_kmax(const rf2_geom* g, const rf2_v1_params* p, unsigned flags) {
  V1Call c;
  int st = v1_prepare(g, p, flags, &c);
  return st != RF2_OK ? -st : c.kmax;
}

size_t rf2_v1_workspace_size(const rf2_geom* g, const rf2_v1_params* p, unsigned flags) {
  V1Call c;
  if (v1_prepare(g, p, flags, &c) != RF2_OK) return 0;
  return v1_ws_bytes(c);
}

int rf2_v1_predict_mask(const void* q, const void* k, const rf2_geom* g, const rf2_v1_params* p,
                        unsigned flags, int32_t* idx, int32_t* cnt, int kmax, int32_t* head_class,
                        float* recall, void* ws, size_t ws_bytes, void* stream) {
  V1Call c;
  int st = v1_prepare(g, p, flags, &c);
  if (st != RF2_OK) return st;
  if (q == nullptr || k == nullptr || idx == nullptr || cnt == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || ((uintptr_t)idx & 3u) || ((uintptr_t)cnt & 3u) ||
      ((uintptr_t)head_class & 3u) || ((uintptr_t)recall & 3u))
    return RF2_ERR_ALIGNMENT;
  if (kmax < c.kmax) return RF2_ERR_INVALID_ARG;
  if (ws == nullptr) return RF2_ERR_WORKSPACE;
  if (!aligned16(ws)) return RF2_ERR_ALIGNMENT;
  if (ws_bytes < v1_ws_bytes(c)) return RF2_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  const rf2::Rf1Scratch w = rf2::rf1_scratch_layout(c.geo, c.a, base + kAlign);
  cudaStream_t s = (cudaStream_t)stream;
  log_geo("v1_predict_mask", c.geo, c.kmax);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = rf2::launch_rf1(q, k, c.geo, c.a, w, head_class, recall, idx, cnt, kmax, status, s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  return finish_checked(flags, status, s);
}


const char* rf2_status_string(int status) {
  switch (status) {
    case RF2_OK: return "ok";
    case RF2_ERR_INVALID_ARG: return "invalid argument";
    case RF2_ERR_UNSUPPORTED: return "unsupported shape (D and block size must be 64 or 128, Nb <= 1024)";
    case RF2_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case RF2_ERR_WORKSPACE: return "workspace missing or too small";
    case RF2_ERR_BAD_INDEX: return "kept block index out of range";
    case RF2_ERR_TIMEOUT: return "device wait timed out";
    case RF2_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int rf2_schedule_action(const rf2_schedule* sc, int step) {
  if (sc == nullptr || sc->total_steps < 1 || sc->predict_interval < 1 ||
      !(sc->dense_fraction >= 0.0 && sc->dense_fraction <= 1.0))
    return -RF2_ERR_INVALID_ARG;
  if (step < 0 || step >= sc->total_steps) return -RF2_ERR_INVALID_ARG;
  long long n_dense = (long long)ceil(sc->dense_fraction * (double)sc->total_steps - 1e-6);
  if (n_dense < 0) n_dense = 0;
  if (n_dense > sc->total_steps) n_dense = sc->total_steps;
  if (step < n_dense) return RF2_STEP_DENSE;
  return ((step - n_dense) % sc->predict_interval == 0) ? RF2_STEP_PREDICT : RF2_STEP_REUSE;
}

int rf2_permute(const void* x, void* xp, const rf2_geom* g, void* stream) {
  int st = check_geom(g);
  if (st != RF2_OK) return st;
  if (x == nullptr || xp == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_geo(*g);
  log_geo("permute", geo, 0);
  return cuda_status(rf2::launch_permute(x, xp, geo, (cudaStream_t)stream));
}

int rf2_unpermute(const void* xp, void* x, const rf2_geom* g, void* stream) {
  int st = check_geom(g);
  if (st != RF2_OK) return st;
  if (x == nullptr || xp == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_geo(*g);
  log_geo("unpermute", geo, 0);
  return cuda_status(rf2::launch_unpermute(xp, x, geo, (cudaStream_t)stream));
}

int rf2_kept_count(const rf2_geom* g, double sparsity, int sink, unsigned flags) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return -st;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return -RF2_ERR_INVALID_ARG;
  return kept_of(rf2::make_call_geo(*g, flags), sparsity, sink, flags);
}

size_t rf2_workspace_size(const rf2_geom* g, double sparsity, int sink, unsigned flags,
                          int attention) {
  if (check_geom(g, flags) != RF2_OK) return 0;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return 0;
  Geo geo = rf2::make_call_geo(*g, flags);
  if (!attention) return mask_ws_layout(geo, nullptr).bytes;
  return attn_ws_layout(geo, kept_of(geo, sparsity, sink, flags), nullptr, flags).bytes;
}

static int predict_mask_impl(const void* qp, const void* kp, const Geo& geo, double sparsity,
                             int sink, unsigned flags, int32_t* idx, int32_t* cnt, int kmax,
                             const MaskWs& w, cudaStream_t s) {
  const int kept = kept_of(geo, sparsity, sink, flags);
  log_geo("predict_mask", geo, kept);
  cudaError_t e = rf2::launch_pool(qp, kp, w.m.q3, w.m.k3, geo, (flags & RF2_RASTER) != 0, s);
  if (e == cudaSuccess)
    e = rf2::launch_scores(w.m.q3, w.m.k3, w.m.scores, geo, (float)(1.0 / sqrt((double)geo.D)),
                           nsink_of(geo, sink), w.status, s);
  if (e == cudaSuccess)
    e = rf2::launch_topk(w.m.scores, idx, cnt, kmax, kept, nsink_of(geo, sink), geo, s);
  return cuda_status(e);
}

int rf2_predict_mask(const void* qp, const void* kp, const rf2_geom* g, double sparsity, int sink,
                     unsigned flags, int32_t* idx, int32_t* cnt, int kmax, void* ws,
                     size_t ws_bytes, void* stream) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return st;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return RF2_ERR_INVALID_ARG;
  if (qp == nullptr || kp == nullptr || idx == nullptr || cnt == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(idx) || !aligned16(cnt))
    return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_call_geo(*g, flags);
  if (kmax < kept_of(geo, sparsity, sink, flags)) return RF2_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned16(ws)) return ws == nullptr ? RF2_ERR_WORKSPACE : RF2_ERR_ALIGNMENT;
  MaskWs w = mask_ws_layout(geo, static_cast<uint8_t*>(ws));
  if (ws_bytes < w.bytes) return RF2_ERR_WORKSPACE;
  if (cudaMemsetAsync(w.status, 0, sizeof(int32_t), (cudaStream_t)stream) != cudaSuccess) return RF2_ERR_CUDA;
  st = predict_mask_impl(qp, kp, geo, sparsity, sink, flags, idx, cnt, kmax, w,
                         (cudaStream_t)stream);
  if (st != RF2_OK) return st;
  return finish_checked(flags, w.status, (cudaStream_t)stream);
}

int rf2_sparse_attn(const void* qp, const void* kp, const void* vp, const int32_t* idx,
                    const int32_t* cnt, int kmax, const rf2_geom* g, float scale, void* op,
                    int32_t* status, unsigned flags, void* stream) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return st;
  if (qp == nullptr || kp == nullptr || vp == nullptr || idx == nullptr || cnt == nullptr ||
      op == nullptr || kmax < 1 || !isfinite(scale) || scale < 0.f)
    return RF2_ERR_INVALID_ARG;
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(vp) || !aligned16(op) ||
      ((uintptr_t)idx & 3u) || ((uintptr_t)cnt & 3u) || ((uintptr_t)status & 3u))
    return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_call_geo(*g, flags);
  const float sc = scale == 0.f ? (float)(1.0 / sqrt((double)geo.D)) : scale;
  log_geo("sparse_attn", geo, kmax);
  cudaError_t e = rf2::launch_sparse_attn(qp, kp, vp, idx, cnt, kmax, geo, sc, op, status,
                                          (flags & RF2_RASTER) != 0, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return RF2_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  return finish_checked(flags, status, (cudaStream_t)stream);
}

int rf2_attention(const void* q, const void* k, const void* v, const rf2_geom* g, double sparsity,
                  int sink, float scale, void* o, int32_t* idx_out, void* ws, size_t ws_bytes,
                  unsigned flags, void* stream) {
  int st = check_geom(g, flags);
  if (st != RF2_OK) return st;
  if (!(sparsity >= 0.0 && sparsity <= 1.0) || !isfinite(scale) || scale < 0.f)
    return RF2_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      ((uintptr_t)idx_out & 3u))
    return RF2_ERR_ALIGNMENT;
  if (ws == nullptr) return RF2_ERR_WORKSPACE;
  if (!aligned16(ws)) return RF2_ERR_ALIGNMENT;
  Geo geo = rf2::make_call_geo(*g, flags);
  const int kept = kept_of(geo, sparsity, sink, flags);
  if ((flags & RF2_FP8) && (geo.D != 128 || geo.blk != 128)) return RF2_ERR_UNSUPPORTED;
  AttnWs w = attn_ws_layout(geo, kept, static_cast<uint8_t*>(ws), flags);
  if (ws_bytes < w.bytes) return RF2_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const float sc = scale == 0.f ? (float)(1.0 / sqrt((double)geo.D)) : scale;
  log_geo("attention", geo, kept);
  // Model-order tensors throughout: the kernels gather each window in place.
  cudaError_t e = cudaMemsetAsync(w.mask.status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  st = predict_mask_impl(q, k, geo, sparsity, sink, flags | RF2_RASTER, w.idx, w.cnt, kept, w.mask, s);
  if (st != RF2_OK) return st;
  if (flags & RF2_FP8) {
    e = rf2::launch_quant_fp8(q, k, v, w.q8, w.k8, w.v8, w.scales, geo, s);
    if (e == cudaSuccess)
      e = rf2::launch_sparse_attn_fp8(w.q8, w.k8, w.v8, w.scales, w.idx, w.cnt, kept, geo, sc, o, w.mask.status, s);
  } else {
    e = rf2::launch_sparse_attn(q, k, v, w.idx, w.cnt, kept, geo, sc, o, w.mask.status, true, s);
  }
  if (e == cudaErrorNotSupported) return RF2_ERR_UNSUPPORTED;
  if (e == cudaSuccess && idx_out != nullptr)
    e = cudaMemcpyAsync(idx_out, w.idx, (size_t)geo.B * geo.heads * geo.Nb * kept * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  return finish_checked(flags, w.mask.status, s);
}

}  // extern "C"
