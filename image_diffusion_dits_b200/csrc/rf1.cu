// RainFusion (v1) mask generators feeding the block-sparse attention kernel (pith.science
// review of "RainFusion: Adaptive Video Generation Acceleration via Multi-Dimensional
// Visual Redundancy": "What carries the argument", "Core claim", "Free parameters").
//
// Three head patterns, as masks over whole blocks (3D windows, coordinates tb = temporal
// block, sw = window index inside a temporal slab, (hb, wb) its row and column):
//   temporal, radius R : key block j kept iff |sw_i - sw_j| <= R  (same region, all frames)
//   spatial,  radius R : key block j kept iff |tb_i - tb_j| <= R  (all regions, nearby frames)
//   textural, stride t : key block j kept iff (hb_j + wb_j) mod t == 0 (a window checkerboard)
// ARM classifies each head from its recall: the mean, over sampled query tokens, of the
// softmax mass (over the sampled keys) that falls inside a band.  The local sample is the
// tokens of frame 0 and scores the temporal band on sw; the global sample is every
// omega-th raster token and scores the spatial band on tb.  Temporal if the local recall
// reaches alpha, else spatial if the global one does, else textural.  RainFusion+ then
// narrows a banded head to the smallest of the bandwidths 1/8, 1/4, 1/2 that keeps the
// recall target.
//
//   arm_recall_kernel : one CTA per (128 sampled queries, sample, b*heads).  TMA brings
//                       the query tile once and key tiles through a 2-stage ring; one
//                       thread issues the 128x128 products into a double-buffered TMEM
//                       accumulator; eight warps read the rows back (two per TMEM lane
//                       quarter, one per column half) and keep, per row, an online
//                       softmax with the total mass and the mass inside four band radii
//                       (the static bandwidth and the three RainFusion+ ones); a chunk of
//                       32 keys in one window takes one band test.  The halves are merged
//                       and each warp of the first half writes the sum over its rows of
//                       inside / total.  Key coordinates come from a table built by
//                       arm_coords_kernel.  The local sample is taken window by window
//                       (5-D boxes of frame 0, wh*ww slots per window, pad slots of
//                       partial windows marked and skipped), so its chunks share a
//                       window; the global sample is every omega-th token (4-D boxes).
//   arm_finalize_kernel: per (b, head) the recall (rows summed in a fixed order), the
//                       class and the band radius or stride.
//   rf1_lists_kernel   : one warp per (b, head, query block): ascending kept list by
//                       ballots over the key blocks, then -1 padding and the count.
#include <math.h>

#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace rf2 {
namespace {

constexpr int kATile = 128;           // sampled queries per CTA, keys per tile
constexpr int kAWarpsRows = 8;        // warps 0-7: rows (lane quarter w % 4, column half w / 4)
constexpr int kAThreads = 32 * kAWarpsRows + 32;  // + warp 8: TMA and MMA issue
constexpr int kATmemCols = 2 * kATile;
constexpr uint64_t kArmWaitNs = 500ull * 1000ull * 1000ull;

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x0,
                                            int x1, int x2, int x3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x0), "r"(x1), "r"(x2), "r"(x3)
      : "memory");
}

template <int D>
struct ArmCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kATile * 64 * 2;        // one 64-column slice of 128 rows
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kChunks * kTileBytes;        // 2 stages x kChunks slices
  static constexpr int kOffBar = kOffK + 2 * kChunks * kTileBytes;
  static constexpr int kUsed = kOffBar + 64 + kATile * 7 * 4 + 1024;  // + merge rows, alignment slack
  // at most two CTAs per SM, so that their TMEM (256 columns each) always fits
  static constexpr int kSmem = kUsed > 80 * 1024 ? kUsed : 80 * 1024;
};

// Window coordinate of every sample slot: sw for the local sample, tb for the global one
// (raster token m * omega); kPadSlot for a pad slot.  coords[a.coord_off[p] + m].  With
// a.wslots, local slot m is token (dh, dw) = divmod(m % wslots, ww) of frame-0 window
// sw = m / wslots; otherwise it is frame-0 token m.
constexpr int kPadSlot = -(1 << 30);

__global__ void arm_coords_kernel(Rf1Args a, int nbh, int* __restrict__ coords) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= a.S[0] + a.S[1]) return;
  if (t < a.S[0]) {
    int c;
    if (a.wslots) {
      const int sw = t / a.wslots, off = t - sw * a.wslots;
      const int hb = sw / a.nbw, wb = sw - hb * a.nbw;
      const int h = hb * a.wh + off / a.ww, w = wb * a.ww + off % a.ww;
      c = (hb < nbh && h < a.HW / a.W && w < a.W) ? sw : kPadSlot;
    } else {
      const int h = t / a.W, w = t - h * a.W;
      c = (h / a.wh) * a.nbw + w / a.ww;
    }
    coords[a.coord_off[0] + t] = c;
  } else {
    const long long n = (long long)(t - a.S[0]) * a.omega;
    coords[a.coord_off[1] + t - a.S[0]] = (int)(n / a.HW) / a.wt;
  }
}

template <int D>
__global__ void __launch_bounds__(kAThreads) arm_recall_kernel(const __grid_constant__ CUtensorMap tq0,
                                                               const __grid_constant__ CUtensorMap tk0,
                                                               const __grid_constant__ CUtensorMap tq1,
                                                               const __grid_constant__ CUtensorMap tk1,
                                                               Rf1Args a, const int* __restrict__ coords,
                                                               float* __restrict__ partial,
                                                               int* __restrict__ status) {
  using C = ArmCfg<D>;
  const int p = blockIdx.y;
  const int qt = blockIdx.x;
  const int S = a.S[p];
  const int nk = (S + kATile - 1) / kATile;
  if (qt * kATile >= S) return;  // this sample has fewer query tiles
  const int bh = blockIdx.z;
  const int b = bh / a.heads, head = bh - b * a.heads;
  const CUtensorMap* mq = p == 0 ? &tq0 : &tq1;
  const CUtensorMap* mk = p == 0 ? &tk0 : &tk1;
  // rows r0 .. r0+127 of sample p into a 128-row tile: one 4-D box (sample stride), or,
  // for the window-ordered local sample, 128 / wslots 5-D window boxes of frame 0
  const bool windowed = p == 0 && a.wslots > 0;
  auto load_rows = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, int kc, int r0) {
    if (windowed) {
      for (int u = 0; u < kATile / a.wslots; ++u) {
        const int sw = r0 / a.wslots + u;
        const int hb = sw / a.nbw, wb = sw - hb * a.nbw;
        ptx::tma_load_5d(dst + u * a.wslots * 128, map, bar, kc * 64, head, wb * a.ww, hb * a.wh, b * a.T);
      }
    } else {
      tma_load_4d(dst, map, bar, kc * 64, head, r0, b);
    }
  };

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_s;
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar_q = sbase + C::kOffBar;
  const uint32_t bar_kfull = bar_q + 8;    // [2]
  const uint32_t bar_acc = bar_q + 24;     // [2] products of a tile done
  const uint32_t bar_free = bar_q + 40;    // [2] rows read back from an accumulator
  const uint32_t bar_done = bar_q + 56;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(&tmem_slot), kATmemCols);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar_kfull + 8 * s, 1);
      ptx::mbar_init(bar_acc + 8 * s, 1);
      ptx::mbar_init(bar_free + 8 * s, kAWarpsRows);
    }
    ptx::mbar_init(bar_done, 1);
    abort_s = 0;
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_flag = &abort_s;

  if (warp == kAWarpsRows) {
    if (lane == 0) {
      ptx::prefetch_tmap(mq);
      ptx::prefetch_tmap(mk);
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(kATile, kATile, 0);
      ptx::mbar_arrive_expect_tx(bar_q, C::kChunks * C::kTileBytes);
      for (int kc = 0; kc < C::kChunks; ++kc)
        load_rows(sbase + C::kOffQ + kc * C::kTileBytes, mq, bar_q, kc, qt * kATile);
      int issued[2] = {0, 0}, waited[2] = {0, 0};
      auto load_k = [&](int kt) {
        const int st = kt & 1;
        ptx::mbar_arrive_expect_tx(bar_kfull + 8 * st, C::kChunks * C::kTileBytes);
        for (int kc = 0; kc < C::kChunks; ++kc)
          load_rows(sbase + C::kOffK + (st * C::kChunks + kc) * C::kTileBytes, mk, bar_kfull + 8 * st, kc,
                    kt * kATile);
        ++issued[st];
      };
      for (int kt = 0; kt < 2 && kt < nk; ++kt) load_k(kt);
      bool ok = ptx::mbar_wait(bar_q, 0, abort_flag, status, kArmWaitNs, kStatusTimeout);
      const bool q_landed = ok;
      for (int kt = 0; ok && kt < nk; ++kt) {
        const int st = kt & 1;
        const uint32_t ph = (uint32_t)(kt >> 1) & 1u;
        ok = ptx::mbar_wait(bar_kfull + 8 * st, ph, abort_flag, status, kArmWaitNs, kStatusTimeout);
        if (!ok) break;
        ++waited[st];
        if (kt >= 2) {
          ok = ptx::mbar_wait(bar_free + 8 * st, ph ^ 1u, abort_flag, status, kArmWaitNs, kStatusTimeout);
          if (!ok) break;
        }
        ptx::tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(st * kATile);
#pragma unroll
        for (int kc = 0; kc < C::kChunks; ++kc) {
          const uint64_t ad = ptx::smem_desc_sw128(sbase + C::kOffQ + kc * C::kTileBytes, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(sbase + C::kOffK + (st * C::kChunks + kc) * C::kTileBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_f16_ss(acc, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(bar_acc + 8 * st);
        if (kt + 2 < nk) {
          // the stage is free once these products have read it
          ok = ptx::mbar_wait(bar_acc + 8 * st, ph, abort_flag, status, kArmWaitNs, kStatusTimeout);
          if (!ok) break;
          load_k(kt + 2);
        }
      }
      // On an abort, let the copies in flight land before the CTA exits.
      if (!q_landed) ptx::mbar_wait(bar_q, 0, nullptr, nullptr, kArmWaitNs, 0);
      for (int st = 0; st < 2; ++st)
        for (; waited[st] < issued[st]; ++waited[st])
          ptx::mbar_wait(bar_kfull + 8 * st, (uint32_t)(waited[st] & 1), nullptr, nullptr, kArmWaitNs, 0);
      // Arrives once every product issued above has completed; no MMA is in flight when
      // the tensor memory is released.
      ptx::mma_commit(bar_done);
      ptx::mbar_wait(bar_done, 0, nullptr, nullptr, kArmWaitNs, 0);
    }
  } else {
    // rows: warp w reads TMEM lanes 32 (w % 4) .. + 31 (query qt * 128 + r) and keeps an
    // online softmax over the key columns of its half (w / 4) of every tile.  No CTA-wide
    // barrier inside the loop: a warp that gives up leaves without waiting for the others.
    const int lq = warp & 3, half = warp >> 2;
    const int r = lq * 32 + lane;
    const int qrow = qt * kATile + r;
    const int* cs = coords + a.coord_off[p];
    const int cq = qrow < S ? __ldg(cs + qrow) : kPadSlot;
    const bool row_valid = cq != kPadSlot;
    int R[4];
#pragma unroll
    for (int l = 0; l < 4; ++l) R[l] = a.R[p][l];
    float m = -INFINITY, tot = 0.f, in[4] = {0.f, 0.f, 0.f, 0.f};
    bool ok = true;
    for (int kt = 0; kt < nk; ++kt) {
      const int st = kt & 1;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc + 8 * st, (uint32_t)(kt >> 1) & 1u, abort_flag, status,
                                                  kArmWaitNs, kStatusTimeout));
      if (!ok) break;
      ptx::tc_fence_after();
      const int nvalid = min(kATile, S - kt * kATile);
#pragma unroll 1
      for (int c = half * 2; c < half * 2 + 2 && c * 32 < nvalid; ++c) {
        const int nv = min(32, nvalid - c * 32);
        // lane e holds the coordinate of key c * 32 + e; bit e of live: a real key
        const int ck = lane < nv ? __ldg(cs + kt * kATile + c * 32 + lane) : kPadSlot;
        const uint32_t live = __ballot_sync(0xffffffffu, ck != kPadSlot);
        const int ck0 = __shfl_sync(0xffffffffu, ck, 0);
        const bool uniform = live == 0xffffffffu && __all_sync(0xffffffffu, ck == ck0);
        uint32_t v[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(st * kATile + c * 32), v);
        float cm = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if ((live >> e) & 1u) cm = fmaxf(cm, __uint_as_float(v[e]));
        cm *= a.scale_log2;
        if (cm > m) {
          const float f = ptx::ex2(m - cm);
          tot *= f;
#pragma unroll
          for (int l = 0; l < 4; ++l) in[l] *= f;
          m = cm;
        }
        if (uniform) {
          // 32 real keys in one window: one band test for the chunk
          float csum = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) csum += ptx::ex2(fmaf(__uint_as_float(v[e]), a.scale_log2, -m));
          tot += csum;
          const int d = abs(cq - ck0);
#pragma unroll
          for (int l = 0; l < 4; ++l) in[l] += d <= R[l] ? csum : 0.f;
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int cke = __shfl_sync(0xffffffffu, ck, e);
            if ((live >> e) & 1u) {
              const float x = ptx::ex2(fmaf(__uint_as_float(v[e]), a.scale_log2, -m));
              tot += x;
              const int d = abs(cq - cke);
#pragma unroll
              for (int l = 0; l < 4; ++l) in[l] += d <= R[l] ? x : 0.f;
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_free + 8 * st);
    }
    // Merge the two column halves of each row (every row thread reaches this barrier
    // exactly once, whether or not its loop gave up), then per warp of the first half:
    // the sum of inside / total over its valid rows, in a fixed shuffle order.
    float* mrg = reinterpret_cast<float*>(smem + C::kOffBar + 64);  // [128 rows][7]
    if (half == 1) {
      float* o = mrg + r * 7;
      o[0] = m; o[1] = tot;
#pragma unroll
      for (int l = 0; l < 4; ++l) o[2 + l] = in[l];
      o[6] = ok ? 1.f : 0.f;
    }
    ptx::named_bar_sync(1, 32 * kAWarpsRows);
    if (half == 0) {
      const float* o = mrg + r * 7;
      const float m1 = o[0];
      const float mm = fmaxf(m, m1);
      const float f0 = ptx::ex2(m - mm), f1 = ptx::ex2(m1 - mm);
      tot = tot * f0 + o[1] * f1;
#pragma unroll
      for (int l = 0; l < 4; ++l) in[l] = in[l] * f0 + o[2 + l] * f1;
      ok = ok && o[6] != 0.f;
      float ratio[4];
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        ratio[l] = (ok && row_valid && tot > 0.f) ? in[l] / tot : 0.f;
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) ratio[l] += __shfl_xor_sync(0xffffffffu, ratio[l], sh);
      }
      if (lane < 4) {
        float v = ratio[0];
        if (lane == 1) v = ratio[1];
        if (lane == 2) v = ratio[2];
        if (lane == 3) v = ratio[3];
        partial[((((long long)bh * 2 + p) * a.tiles_max + qt) * 4 + lq) * 4 + lane] = v;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kATmemCols);
  }
}

// Per (b, head): recall, class, band radius or stride.  clsparam[bh] = {class, param}.
__global__ void arm_finalize_kernel(const float* __restrict__ partial, Rf1Args a, int BH,
                                    int* __restrict__ clsparam, int32_t* __restrict__ cls_out,
                                    float* __restrict__ recall_out) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= BH) return;
  float rec[2][4];
  for (int p = 0; p < 2; ++p) {
    const int tiles = (a.S[p] + kATile - 1) / kATile;
    for (int l = 0; l < 4; ++l) {
      float s = 0.f;
      for (int t = 0; t < tiles; ++t)
        for (int w = 0; w < 4; ++w) s += partial[((((long long)bh * 2 + p) * a.tiles_max + t) * 4 + w) * 4 + l];
      rec[p][l] = s / (float)a.S_real[p];
    }
  }
  int cls, prm;
  if (rec[0][0] >= a.alpha || rec[1][0] >= a.alpha) {
    const int p = rec[0][0] >= a.alpha ? 0 : 1;  // temporal first, then spatial
    cls = p == 0 ? 0 : 1;
    prm = a.R[p][0];
    if (a.dynamic) {
      prm = a.R[p][3];
      for (int l = 1; l <= 3; ++l)
        if (rec[p][l] >= a.target) {
          prm = a.R[p][l];
          break;
        }
    }
  } else {
    cls = 2;
    prm = a.tau;
  }
  clsparam[2 * bh] = cls;
  clsparam[2 * bh + 1] = prm;
  if (cls_out != nullptr) cls_out[bh] = cls;
  if (recall_out != nullptr)
    for (int p = 0; p < 2; ++p)
      for (int l = 0; l < 4; ++l) recall_out[(long long)bh * 8 + p * 4 + l] = rec[p][l];
}

constexpr int kListWarps = 8;

__global__ void __launch_bounds__(kListWarps * 32) rf1_lists_kernel(const int* __restrict__ clsparam, Geo g,
                                                                   long long rows, int32_t* __restrict__ idx,
                                                                   int32_t* __restrict__ cnt, int kmax) {
  const long long row = (long long)blockIdx.x * kListWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const long long bh = row / g.Nb;
  const int i = (int)(row - bh * g.Nb);
  const int cls = clsparam[2 * bh], prm = clsparam[2 * bh + 1];
  const int P = g.nbh * g.nbw;
  const int tbi = i / P, swi = i - tbi * P;
  int32_t* out = idx + row * kmax;
  int n = 0;
  for (int j0 = 0; j0 < g.Nb; j0 += 32) {
    const int j = j0 + lane;
    bool keep = false;
    if (j < g.Nb) {
      const int tbj = j / P, swj = j - tbj * P;
      if (cls == 0) keep = abs(swi - swj) <= prm;
      else if (cls == 1) keep = abs(tbi - tbj) <= prm;
      else {
        const int hb = swj / g.nbw, wb = swj - hb * g.nbw;
        keep = (hb + wb) % prm == 0;
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < kmax) out[pos] = j;
    n += __popc(bal);
  }
  const int kept = min(n, kmax);
  for (int pos = kept + lane; pos < kmax; pos += 32) out[pos] = -1;
  if (lane == 0) cnt[row] = kept;
}

// 4-D view (D, heads, samples, B) of model-order [B, N, heads, D]: sample m is token
// m * stride; box = 64 columns x 1 head x 128 samples, 128-byte swizzle, zero fill past
// the last sample.
bool make_sample_map(CUtensorMap* m, const void* base, const Geo& g, int samples, int stride) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)g.heads * g.D * 2;
  cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.heads, (cuuint64_t)samples, (cuuint64_t)g.B};
  cuuint64_t strides[3] = {(cuuint64_t)g.D * 2, row * (cuuint64_t)stride, row * (cuuint64_t)g.N};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)kATile, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D view (D, heads, W, H, T*B) of model-order [B, N, heads, D] (the frames of all
// batches in a row); box = 64 columns x 1 head x one (ww, wh) window of one frame,
// 128-byte swizzle, zero fill past the grid.
bool make_frame_window_map(CUtensorMap* m, const void* base, const Geo& g) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)g.heads * g.D * 2;
  cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.heads, (cuuint64_t)g.W, (cuuint64_t)g.H,
                        (cuuint64_t)g.T * g.B};
  cuuint64_t strides[4] = {(cuuint64_t)g.D * 2, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)g.ww, (cuuint32_t)g.wh, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_arm_d(const void* q, const void* k, const Geo& g, const Rf1Args& a, const int* coords,
                         float* partial, int32_t* status, cudaStream_t s) {
  using C = ArmCfg<D>;
  CUtensorMap tq0, tk0, tq1, tk1;
  const bool ok0 = a.wslots ? (make_frame_window_map(&tq0, q, g) && make_frame_window_map(&tk0, k, g))
                            : (make_sample_map(&tq0, q, g, a.S[0], 1) && make_sample_map(&tk0, k, g, a.S[0], 1));
  if (!ok0 || !make_sample_map(&tq1, q, g, a.S[1], a.omega) || !make_sample_map(&tk1, k, g, a.S[1], a.omega))
    return cudaErrorInvalidValue;
  static int configured_device = -1;  // one flag per instance (per D)
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(arm_recall_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid(a.tiles_max, 2, g.B * g.heads);
  arm_recall_kernel<D><<<grid, kAThreads, C::kSmem, s>>>(tq0, tk0, tq1, tk1, a, coords, partial, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rf1(const void* q, const void* k, const Geo& g, const Rf1Args& a, const Rf1Scratch& w,
                       int32_t* cls_out, float* recall_out, int32_t* idx, int32_t* cnt, int kmax,
                       int32_t* status, cudaStream_t s) {
  const int ns = a.S[0] + a.S[1];
  arm_coords_kernel<<<(ns + 255) / 256, 256, 0, s>>>(a, g.nbh, w.coords);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = g.D == 128 ? launch_arm_d<128>(q, k, g, a, w.coords, w.partial, status, s)
                 : launch_arm_d<64>(q, k, g, a, w.coords, w.partial, status, s);
  if (e != cudaSuccess) return e;
  const int BH = g.B * g.heads;
  arm_finalize_kernel<<<(BH + 127) / 128, 128, 0, s>>>(w.partial, a, BH, w.clsparam, cls_out, recall_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = (long long)BH * g.Nb;
  rf1_lists_kernel<<<(unsigned)((rows + kListWarps - 1) / kListWarps), kListWarps * 32, 0, s>>>(
      w.clsparam, g, rows, idx, cnt, kmax);
  return cudaGetLastError();
}

}  // namespace rf2
