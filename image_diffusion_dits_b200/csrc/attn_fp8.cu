// e4m3 variant of the block-sparse attention, sm_100a (tcgen05 kind::f8f6f4 + TMEM + TMA).
//
// The block-sparse attention of RainFusion2.0 (mlsanity index page: title, Abstract) with
// its operands quantised to FP8, following the sciencestack page's TL;DR, which points to
// integrating quantisation for further speed.  Q, K and V carry one e4m3 scale per
// (batch, head, block):
//   quant_fp8_kernel : per block, amax over its real tokens and the head's D channels,
//                      inv = 448 / amax and scale = amax / 448 (fp32, rounded), codes =
//                      e4m3(x * inv) (round to nearest even, saturating).  One CTA per
//                      (block, 128 channels of the heads*D row, tensor): the window's
//                      rows are read from HBM once into registers, reduced across the
//                      CTA, then converted and written as the e4m3 model-order tensor.
//   sparse_attn_fp8_kernel : the warp-specialised pipeline of the bf16 kernel with
//                      - S = Q K^T on e4m3 operands (kind::f8f6f4, K = 32 per MMA), the
//                        per-block scales sq * sk_j applied to the fp32 scores;
//                      - P = exp2(s - m) in packed f16, rounded to e4m3 after multiplying
//                        by sv_j / max_j sv_j (the V scale of block j folded into P, so
//                        that one accumulator serves blocks of different V scales),
//                        written to TMEM four codes per column over the S columns; the
//                        row sum adds the f16 values (f16x2 over 16 columns, then fp32);
//                      - O += P V with P from TMEM (kind::f8f6f4, V MN-major);
//                      - O = O_acc * max_j sv_j / l in the epilogue.
// Shared-memory tiles are half the bf16 size (128 rows x 128 bytes), so the K and V rings
// are five stages deep.  D = 128 and 128-token blocks, model order [B, N, heads, D].
#include <cuda.h>

#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace rf2 {
namespace {

// ------------------------------------------------------------------------------ helpers
// Two fp32 values to two e4m3 codes (nearest even, saturating): lo -> low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return (uint32_t)d;
}

// Packed f16 helpers for the probabilities.
__device__ __forceinline__ uint32_t f16x2_from(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t ex2_h2(uint32_t a) {
  uint32_t d;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// f16x2 (lo, hi) to two e4m3 codes (nearest even, saturating): lo -> low byte.
__device__ __forceinline__ uint32_t e4m3x2_h2(uint32_t a) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(d) : "r"(a));
  return (uint32_t)d;
}
__device__ __forceinline__ float h2_sum_f32(uint32_t a) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(a));
  return lo + hi;
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 8 columns of 32-bit from registers (thread i of the warp: lane base + i).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f8f6f4: A (M x K, e4m3) in TMEM, lane m holds
// row m and each 32-bit column four consecutive K elements (the lowest in the low byte).
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulator, e4m3 A and B (format 0), dense.
constexpr uint32_t idesc_e4m3_f32(int M, int N, int b_mn_major) {
  return (1u << 4) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------------------ quantise
constexpr int kQuantThreads = 256;
constexpr int kQuantCols = 16;                                 // 16-byte chunks per row and CTA (128 channels)
constexpr int kQuantItems = 128 * kQuantCols / kQuantThreads;  // chunks per thread (blk <= 128)

// CTA = (128 channels of the heads*D row = 128 / D heads, block j, b * 3 + tensor).  The
// window's real rows x 16 chunks are numbered r * 16 + c and thread t owns chunks t,
// t + 256, ...: its column c = t % 16 (so its head) is fixed, and each warp-wide copy
// covers two whole 256-byte row slices.  Every owned chunk is copied from HBM into shared
// memory with cp.async (no registers held while the copies are in flight, so six CTAs
// per SM keep ~190 KB of reads outstanding), the amax of each head is reduced over the
// lanes and then over the 8 warps, and each thread converts its own chunks from shared
// memory and stores the codes.  Q, K and V are read once; the window's row offsets come
// from a per-CTA table.
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quant_fp8_kernel(const int4* __restrict__ q, const int4* __restrict__ k,
                                                                 const int4* __restrict__ v, uint8_t* __restrict__ q8,
                                                                 uint8_t* __restrict__ k8, uint8_t* __restrict__ v8,
                                                                 float* __restrict__ scales, Geo g, int chunks) {
  constexpr int kPerHead = D / 8;                // chunks of one head's row
  constexpr int kHeads = kQuantCols / kPerHead;  // heads per CTA
  __shared__ __align__(16) int4 stage[kQuantItems * kQuantThreads];
  __shared__ int roff_s[128];
  __shared__ float red[kQuantThreads / 32][kHeads];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = tid & (kQuantCols - 1);
  const int hl = c / kPerHead;  // head within the CTA
  const int head0 = blockIdx.x * kHeads;
  const bool col_live = head0 + hl < g.heads;
  const int j = blockIdx.y;
  const int b = blockIdx.z / 3, t = blockIdx.z - b * 3;
  const int4* src = (t == 0 ? q : t == 1 ? k : v);
  uint8_t* dst = (t == 0 ? q8 : t == 1 ? k8 : v8);
  int nt, nh, nw;
  block_extent(g, j, nt, nh, nw);
  const int per_t = g.nbh * g.nbw;
  const int tb = j / per_t, hb = (j - tb * per_t) / g.nbw, wb = j - tb * per_t - hb * g.nbw;
  const long long row0 = (long long)b * g.N + ((long long)tb * g.wt * g.H + (long long)hb * g.wh) * g.W +
                         (long long)wb * g.ww;
  const int rows = nt * nh * nw;
  // token offset of each real row of the window from its first token (-1 past the real
  // rows), computed once per CTA: dividing per chunk costs more issue slots than the copy
  if (tid < 128) {
    int o = -1;
    if (tid < rows) {
      const int dw = tid % nw, rest = tid / nw;
      const int dh = rest % nh, dt = rest / nh;
      o = (int)(dt * (long long)g.H * g.W + dh * (long long)g.W + dw);
    }
    roff_s[tid] = o;
  }
  __syncthreads();
  // chunk index of the window's first token at this thread's column; a chunk is addressed
  // by its token offset from there (< B * N < 2^31)
  const long long base = row0 * chunks + (long long)head0 * kPerHead + c;
  const int rsub = tid / kQuantCols;
#pragma unroll
  for (int it = 0; it < kQuantItems; ++it) {
    const int ro = roff_s[rsub + it * (kQuantThreads / kQuantCols)];
    if (ro >= 0 && col_live) {
      const uint32_t sdst = ptx::smem_u32(&stage[it * kQuantThreads + tid]);
      const int4* gsrc = src + base + (long long)ro * chunks;
      asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(sdst), "l"(gsrc) : "memory");
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  float amax = 0.f;
#pragma unroll
  for (int it = 0; it < kQuantItems; ++it) {
    if (roff_s[rsub + it * (kQuantThreads / kQuantCols)] >= 0 && col_live) {
      const int4 x = stage[it * kQuantThreads + tid];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  // lanes l and l ^ 16 hold the same column; the kPerHead columns of a head are adjacent
#pragma unroll
  for (int o = 1; o < kPerHead; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
  if (lane < kQuantCols && (lane % kPerHead) == 0) red[warp][hl] = amax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red[w][hl]);
  if (!col_live) return;
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  if (tid < kQuantCols && c % kPerHead == 0)
    scales[(((long long)t * g.B + b) * g.heads + head0 + hl) * g.Nb + j] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
#pragma unroll
  for (int it = 0; it < kQuantItems; ++it) {
    const int ro = roff_s[rsub + it * (kQuantThreads / kQuantCols)];
    if (ro >= 0) {
      const int4 x = stage[it * kQuantThreads + tid];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&x);
      uint32_t w[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 f0 = __bfloat1622float2(h2[2 * e]), f1 = __bfloat1622float2(h2[2 * e + 1]);
        w[e] = e4m3x2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv)) |
               (e4m3x2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv)) << 16);
      }
      *reinterpret_cast<uint2*>(dst + (base + (long long)ro * chunks) * 8) = make_uint2(w[0], w[1]);
    }
  }
}

// ------------------------------------------------------------------------------ attention
constexpr int kBM = 128;
constexpr int kBLK = 128;
constexpr int kD = 128;
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kKStages = 5;
constexpr int kVStages = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
constexpr uint64_t kWaitLimitNs = 500ull * 1000ull * 1000ull;

constexpr int kTile = 128 * 128;                       // one e4m3 tile: 128 rows x 128 bytes
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;
constexpr int kOffV = kOffK + kKStages * kTile;
constexpr int kOffList = kOffV + kVStages * kTile;     // int32[1024]
constexpr int kOffExt = kOffList + 4096;               // int32[1024]
constexpr int kOffSc = kOffExt + 4096;                 // float[1024] sk_j * sq, float[1024] sv_j / vmax
constexpr int kOffXch = kOffSc + 8192;                 // float[2][2][128]
constexpr int kOffBar = kOffXch + 2048;
constexpr int kOffMisc = kOffBar + 256;
constexpr int kSmem = kOffMisc + 64 + 1024;

enum : int {
  BAR_Q = 0,
  BAR_KFULL = 1,                       // +stage
  BAR_KEMPTY = BAR_KFULL + kKStages,   // +stage
  BAR_VFULL = BAR_KEMPTY + kKStages,   // +stage
  BAR_VEMPTY = BAR_VFULL + kVStages,   // +stage
  BAR_SFULL = BAR_VEMPTY + kVStages,   // +stream
  BAR_PFULL = BAR_SFULL + 2,           // +stream
  BAR_DONE = BAR_PFULL + 2,
  BAR_XCH = BAR_DONE + 1,
  BAR_COUNT = BAR_XCH + 1
};
static_assert(BAR_COUNT * 8 <= 256, "barrier area");

struct Misc {
  uint32_t tmem_base;
  int n;
  int abort;
  float vmax;
};

__device__ __forceinline__ long long window_row_token(const Geo& g, int i, int r) {
  const int per_t = g.nbh * g.nbw;
  const int tb = i / per_t, hb = (i - tb * per_t) / g.nbw, wb = i - tb * per_t - hb * g.nbw;
  const int whw = g.wh * g.ww;
  const int dt = r / whw, dh = (r - dt * whw) / g.ww, dw = r - dt * whw - dh * g.ww;
  const int t = tb * g.wt + dt, h = hb * g.wh + dh, w = wb * g.ww + dw;
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return ((long long)t * g.H + h) * g.W + w;
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_fp8_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap tv, const float* __restrict__ scales,
                           const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int kmax,
                           __nv_bfloat16* __restrict__ op, Geo g, float scale_log2, int* __restrict__ status,
                           int b) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV;
  int* list_s = reinterpret_cast<int*>(smem + kOffList);
  int* ext_s = reinterpret_cast<int*>(smem + kOffExt);
  float* ksc_s = reinterpret_cast<float*>(smem + kOffSc);          // scale_log2 * sq * sk_j
  float* vsc_s = ksc_s + 1024;                                        // sv_j / vmax
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  Misc* misc = reinterpret_cast<Misc*>(smem + kOffMisc);
  volatile int* abort_flag = &misc->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qblk = blockIdx.x, head = blockIdx.y;
  const long long row = ((long long)b * g.heads + head) * g.Nb + qblk;
  const long long sc_bh = ((long long)b * g.heads + head) * g.Nb;      // scales of this (b, head)
  const long long sc_t = (long long)g.B * g.heads * g.Nb;              // per tensor
  auto load_block = [&](uint32_t dst, const CUtensorMap* map, uint32_t barrier, int j) {
    const int per_t = g.nbh * g.nbw;
    const int tb = j / per_t, hb = (j - tb * per_t) / g.nbw, wb = j - tb * per_t - hb * g.nbw;
    ptx::tma_load_5d(dst, map, barrier, 0, head, wb * g.ww, hb * g.wh, tb * g.wt);
  };

  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(&misc->tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < kKStages; ++s) {
      ptx::mbar_init(bar(BAR_KFULL + s), 1);
      ptx::mbar_init(bar(BAR_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      ptx::mbar_init(bar(BAR_VFULL + s), 1);
      ptx::mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(BAR_SFULL + s), 1);
      ptx::mbar_init(bar(BAR_PFULL + s), 4);
    }
    ptx::mbar_init(bar(BAR_DONE), 1);
    ptx::mbar_init(bar(BAR_XCH), kSoftmaxWarps);
    misc->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    // Compact the kept list (ids outside [0, Nb) dropped and reported), with each entry's
    // real extent and its K and V scales; vmax = the largest V scale of the row.
    int n_in = cnt[row];
    n_in = n_in < 0 ? 0 : (n_in > kmax ? kmax : n_in);
    n_in = n_in > 1024 ? 1024 : n_in;
    const int32_t* lst = idx + row * kmax;
    const float sq = scales[sc_bh + qblk];
    int n_out = 0;
    bool bad = false;
    float vmax = 0.f;
    for (int e0 = 0; e0 < n_in; e0 += 32) {
      const int e = e0 + lane;
      const int j = e < n_in ? lst[e] : -1;
      const bool ok = e < n_in && j >= 0 && j < g.Nb;
      bad |= (e < n_in) && !ok;
      const uint32_t m = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        int nt, nh, nw;
        block_extent(g, j, nt, nh, nw);
        const int pos = n_out + __popc(m & ((1u << lane) - 1u));
        list_s[pos] = j;
        ext_s[pos] = nt | (nh << 8) | (nw << 16);
        ksc_s[pos] = scale_log2 * sq * scales[sc_t + sc_bh + j];
        const float sv = scales[2 * sc_t + sc_bh + j];
        vsc_s[pos] = sv;
        vmax = fmaxf(vmax, sv);
      }
      n_out += __popc(m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    __syncwarp();
    const float rv = vmax > 0.f ? 1.0f / vmax : 0.f;
    for (int e = lane; e < n_out; e += 32) vsc_s[e] *= rv;
    if (__any_sync(0xffffffffu, bad) && lane == 0 && status != nullptr) atomicCAS(status, 0, kStatusBadIndex);
    if (lane == 0) {
      misc->n = n_out;
      misc->vmax = vmax;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int n = misc->n;

  if (n > 0) {
    if (warp == kProducerWarp && lane == 0) {
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tk);
      ptx::mbar_arrive_expect_tx(bar(BAR_Q), kTile);
      load_block(sQ, &tq, bar(BAR_Q), qblk);
      int issued[kKStages];
#pragma unroll
      for (int s = 0; s < kKStages; ++s) issued[s] = -1;
      for (int i = 0; i < n; ++i) {
        const int s = i % kKStages;
        if (i >= kKStages && !ptx::mbar_wait(bar(BAR_KEMPTY + s), ((i / kKStages) - 1) & 1, abort_flag, status,
                                             kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_KFULL + s), kTile);
        load_block(sK + s * kTile, &tk, bar(BAR_KFULL + s), list_s[i]);
        issued[s] = i;
      }
      if (*abort_flag) {
        ptx::mbar_wait(bar(BAR_Q), 0, nullptr, nullptr, kWaitLimitNs, 0);
        for (int s = 0; s < kKStages; ++s)
          if (issued[s] >= 0)
            ptx::mbar_wait(bar(BAR_KFULL + s), (issued[s] / kKStages) & 1, nullptr, nullptr, kWaitLimitNs, 0);
      }
    } else if (warp == kVProducerWarp && lane == 0) {
      ptx::prefetch_tmap(&tv);
      int issued[kVStages];
#pragma unroll
      for (int s = 0; s < kVStages; ++s) issued[s] = -1;
      for (int i = 0; i < n; ++i) {
        const int s = i % kVStages;
        if (i >= kVStages && !ptx::mbar_wait(bar(BAR_VEMPTY + s), ((i / kVStages) - 1) & 1, abort_flag, status,
                                             kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_VFULL + s), kTile);
        load_block(sV + s * kTile, &tv, bar(BAR_VFULL + s), list_s[i]);
        issued[s] = i;
      }
      if (*abort_flag) {
        for (int s = 0; s < kVStages; ++s)
          if (issued[s] >= 0)
            ptx::mbar_wait(bar(BAR_VFULL + s), (issued[s] / kVStages) & 1, nullptr, nullptr, kWaitLimitNs, 0);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      constexpr uint32_t idesc_s = idesc_e4m3_f32(kBM, kBLK, 0);
      constexpr uint32_t idesc_o = idesc_e4m3_f32(kBM, kD, 1);
      bool ok = ptx::mbar_wait(bar(BAR_Q), 0, abort_flag, status, kWaitLimitNs, kStatusTimeout);
      ptx::tc_fence_after();
      const uint64_t qdesc = ptx::smem_desc_sw128(sQ, 16, 1024);
      const uint64_t kdesc0 = ptx::smem_desc_sw128(sK, 16, 1024);
      const uint64_t vdesc0 = ptx::smem_desc_sw128(sV, kTile, 1024);
      auto wait_s = [&](int i) -> bool {
        return ptx::mbar_wait(bar(BAR_KFULL + i % kKStages), (i / kKStages) & 1, abort_flag, status, kWaitLimitNs,
                              kStatusTimeout);
      };
      // S_i = Q K_i^T into the S buffer of stream i%2: 4 MMAs of 32 e4m3 columns (32 bytes)
      auto issue_s = [&](int i) {
        const int ks = i % kKStages, st = i & 1;
        const uint64_t kdesc = kdesc0 + (uint64_t)((ks * kTile) >> 4);
        const uint32_t dS = tmem + (uint32_t)(128 * st);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ss(dS, qdesc + (uint64_t)(kk * 2), kdesc + (uint64_t)(kk * 2), idesc_s, kk > 0 ? 1u : 0u);
        ptx::mma_commit(bar(BAR_SFULL + st));
        ptx::mma_commit(bar(BAR_KEMPTY + ks));
      };
      auto wait_pv = [&](int i) -> bool {
        return ptx::mbar_wait(bar(BAR_PFULL + (i & 1)), (i >> 1) & 1, abort_flag, status, kWaitLimitNs,
                              kStatusTimeout) &&
               ptx::mbar_wait(bar(BAR_VFULL + i % kVStages), (i / kVStages) & 1, abort_flag, status, kWaitLimitNs,
                              kStatusTimeout);
      };
      // O_{i%2} += P_i V_i: A = P from TMEM (the first 32 columns of the stream's S buffer,
      // 4 e4m3 keys per column), B = V (MN-major: a key row of 128 bytes holds the D
      // columns); 32 keys = 8 columns per MMA.
      auto issue_pv = [&](int i) {
        const int vs = i % kVStages, st = i & 1;
        const uint64_t vdesc = vdesc0 + (uint64_t)((vs * kTile) >> 4);
        const uint32_t pt = tmem + (uint32_t)(128 * st);
        const uint32_t dO = tmem + kTmemO + (uint32_t)(128 * st);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ts(dO, pt + (uint32_t)(kk * 8), vdesc + (uint64_t)(kk * (32 * 128 / 16)), idesc_o,
                    (i >= 2 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(bar(BAR_VEMPTY + vs));
      };
      for (int i = 0; ok && i < n && i < 2; ++i) {
        ok = wait_s(i);
        if (ok) {
          ptx::tc_fence_after();
          issue_s(i);
        }
      }
      for (int i = 0; ok && i < n; ++i) {
        ok = wait_pv(i) && (i + 2 >= n || wait_s(i + 2));
        if (!ok) break;
        ptx::tc_fence_after();
        issue_pv(i);
        if (i + 2 < n) issue_s(i + 2);
      }
      ptx::mma_commit(bar(BAR_DONE));
      ptx::mbar_wait(bar(BAR_DONE), 0, nullptr, nullptr, kWaitLimitNs, 0);
    } else if (warp < kSoftmaxWarps) {
      const int st = warp >> 2;
      const int r = tid & (kBM - 1);
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t srow = tmem + lane_base + (uint32_t)(128 * st);
      const uint32_t orow_t = tmem + lane_base + kTmemO + (uint32_t)(128 * st);
      int cpk[kBLK / 32];
#pragma unroll
      for (int q = 0; q < kBLK / 32; ++q) {
        const int c = q * 32 + lane;
        const int whw = g.wh * g.ww;
        const int dt = c / whw, dh = (c - dt * whw) / g.ww, dw = c - dt * whw - dh * g.ww;
        cpk[q] = dt | (dh << 8) | (dw << 16);
      }
      const int full_ext = g.wt | (g.wh << 8) | (g.ww << 16);
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int i = st; i < n; i += 2) {
        const int t = i >> 1;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_SFULL + st), t & 1, abort_flag, status, kWaitLimitNs,
                                                     kStatusTimeout))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // scale of this block's scores (log2 units); kept positive so that a masked
        // -inf never meets a zero scale (a zero-scale block's raw scores are exactly 0)
        const float sc = fmaxf(ksc_s[i], 1e-30f);
        // Pad keys of a partial window are masked (-inf); validity is per column, the same
        // for every row, so each lane evaluates 1/32 of the columns and the warp shares bits.
        const int ext = ext_s[i];
        const bool partial = ext != full_ext;  // the same for the whole warp
        uint32_t vm[kBLK / 32];
        if (partial) {
          const int nt = ext & 255, nh = (ext >> 8) & 255, nw = ext >> 16;
#pragma unroll
          for (int q = 0; q < kBLK / 32; ++q)
            vm[q] = __ballot_sync(0xffffffffu,
                                  (cpk[q] & 255) < nt && ((cpk[q] >> 8) & 255) < nh && (cpk[q] >> 16) < nw);
        } else {
#pragma unroll
          for (int q = 0; q < kBLK / 32; ++q) vm[q] = 0xffffffffu;
        }
        // the whole S row in one TMEM load; the row max of the raw scores (the scale is
        // positive, so it commutes with max)
        float mx;
        uint32_t tt[kBLK];
        ptx::tmem_ld32x128(srow, tt);
        if (partial) {
#pragma unroll
          for (int c = 0; c < kBLK; ++c)
            if (!((vm[c >> 5] >> (c & 31)) & 1u)) tt[c] = __float_as_uint(-INFINITY);
        }
        {
          float mx8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(tt[e]);
#pragma unroll
          for (int c = 8; c + 8 < kBLK; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              mx8[e] = ptx::fmax3(mx8[e], __uint_as_float(tt[c + e]), __uint_as_float(tt[c + 8 + e]));
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], __uint_as_float(tt[kBLK - 8 + e]));
          mx = ptx::fmax3(ptx::fmax3(mx8[0], mx8[1], mx8[2]), ptx::fmax3(mx8[3], mx8[4], mx8[5]),
                          fmaxf(mx8[6], mx8[7]));
        }
        const float m_new = fmaxf(m_run, mx * sc);
        const bool grow = m_new > m_run + 8.0f;
        float alpha = 1.0f;
        if (grow) {
          alpha = ptx::ex2(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
        if (t >= 1 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t tt[32];
            ptx::tmem_ld32(orow_t + c * 32, tt);
#pragma unroll
            for (int e = 0; e < 32; ++e) tt[e] = __float_as_uint(__uint_as_float(tt[e]) * alpha);
            ptx::tmem_st32(orow_t + c * 32, tt);
          }
        }
        // 32 columns at a time: p = exp2(x * sc - m) in packed f16 (arguments from one packed
        // fp32 FMA per pair), P = e4m3(p * sv_j / vmax) from f16x2, four codes per word; the
        // row sum adds the f16 values of 16 columns in f16x2 and widens once.
        const uint64_t sc2 = ptx::f2(sc, sc), nm2 = ptx::f2(-m_run, -m_run);
        const uint32_t vs2 = f16x2_from(vsc_s[i], vsc_s[i]);
        float lsum = 0.f;
#pragma unroll
        for (int q = 0; q < kBLK / 32; ++q) {
          uint32_t pk[8];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t e2[8];
#pragma unroll
            for (int qd = 0; qd < 8; ++qd) {
              const int c = half * 16 + qd * 2;
              float a0, a1;
              const uint64_t xx = ptx::f2(__uint_as_float(tt[q * 32 + c]), __uint_as_float(tt[q * 32 + c + 1]));
              ptx::f2split(ptx::ffma2(xx, sc2, nm2), a0, a1);
              e2[qd] = ex2_h2(f16x2_from(a0, a1));
            }
#pragma unroll
            for (int qd = 0; qd < 4; ++qd)
              pk[half * 4 + qd] =
                  e4m3x2_h2(hmul2(e2[2 * qd], vs2)) | (e4m3x2_h2(hmul2(e2[2 * qd + 1], vs2)) << 16);
            lsum += h2_sum_f32(hadd2(hadd2(hadd2(e2[0], e2[1]), hadd2(e2[2], e2[3])),
                                     hadd2(hadd2(e2[4], e2[5]), hadd2(e2[6], e2[7]))));
          }
          // P columns 8q .. 8q+7 over S columns already loaded into registers
          tmem_st8(srow + q * 8, pk);
        }
        ptx::tmem_wait_st();
        l_run += lsum;
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(BAR_PFULL + st));
      }
      float* xch = reinterpret_cast<float*>(smem + kOffXch);
      xch[(st * 2 + 0) * 128 + r] = m_run;
      xch[(st * 2 + 1) * 128 + r] = l_run;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(BAR_XCH));
      ok = ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_XCH), 0, abort_flag, status, kWaitLimitNs,
                                                        kStatusTimeout));
      if (ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_DONE), 0, abort_flag, status, kWaitLimitNs,
                                                       kStatusTimeout))) {
        ptx::tc_fence_after();
        const float m0 = xch[0 * 128 + r], l0 = xch[1 * 128 + r];
        const float m1 = xch[2 * 128 + r], l1 = xch[3 * 128 + r];
        const float m = fmaxf(m0, m1);
        const float f0 = l0 > 0.f ? ptx::ex2(m0 - m) : 0.f;
        const float f1 = l1 > 0.f ? ptx::ex2(m1 - m) : 0.f;
        const float den = f0 * l0 + f1 * l1;
        const float inv = den > 0.f ? misc->vmax / den : 0.f;
        const float w0 = f0 * inv, w1 = f1 * inv;
        const bool use1 = n > 1;
        const long long n_tok = window_row_token(g, qblk, r);
        const long long orow_idx = n_tok < 0 ? -1 : (long long)b * g.N + n_tok;
        __nv_bfloat16* orow = op + (orow_idx * g.heads + head) * (long long)kD + st * (kD / 2);
#pragma unroll
        for (int c = 0; c < kD / 64; ++c) {
          const uint32_t col = (uint32_t)(st * (kD / 2) + c * 32);
          uint32_t a0[32], a1[32];
          ptx::tmem_ld32(tmem + lane_base + kTmemO + col, a0);
          if (use1) {
            ptx::tmem_ld32(tmem + lane_base + kTmemO + 128 + col, a1);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) a1[e] = 0u;
          }
          if (orow_idx >= 0) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                o[e] = __uint_as_float(a0[8 * v + e]) * w0 + (use1 ? __uint_as_float(a1[8 * v + e]) * w1 : 0.f);
              uint4 wv;
              wv.x = ptx::pack_bf16(o[0], o[1]);
              wv.y = ptx::pack_bf16(o[2], o[3]);
              wv.z = ptx::pack_bf16(o[4], o[5]);
              wv.w = ptx::pack_bf16(o[6], o[7]);
              reinterpret_cast<uint4*>(orow + c * 32)[v] = wv;
            }
          }
        }
      }
    }
  } else if (warp < 4) {
    const long long n_tok = window_row_token(g, qblk, tid);
    if (n_tok >= 0) {
      __nv_bfloat16* orow = op + (((long long)b * g.N + n_tok) * g.heads + head) * (long long)kD;
      for (int v = 0; v < kD / 8; ++v) reinterpret_cast<uint4*>(orow)[v] = make_uint4(0, 0, 0, 0);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// 5-D view of one batch of an e4m3 [B, N, heads, 128] tensor: dims (128 bytes, heads, W,
// H, T); box = one head's 128 bytes x one (ww, wh, wt) window, 128-byte swizzle.
bool make_window_map_e4m3(CUtensorMap* m, const void* base, const Geo& g) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)g.heads * kD;
  cuuint64_t dims[5] = {(cuuint64_t)kD, (cuuint64_t)g.heads, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
  cuuint64_t strides[4] = {(cuuint64_t)kD, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {(cuuint32_t)kD, 1, (cuuint32_t)g.ww, (cuuint32_t)g.wh, (cuuint32_t)g.wt};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_quant_fp8(const void* q, const void* k, const void* v, uint8_t* q8, uint8_t* k8, uint8_t* v8,
                             float* scales, const Geo& g, cudaStream_t s) {
  if (g.D != 128 && g.D != 64) return cudaErrorNotSupported;
  const int chunks = g.heads * g.D / 8;
  const int heads_per_cta = kQuantCols / (g.D / 8);
  dim3 grid((g.heads + heads_per_cta - 1) / heads_per_cta, g.Nb, g.B * 3);
  if (g.D == 128)
    quant_fp8_kernel<128><<<grid, kQuantThreads, 0, s>>>((const int4*)q, (const int4*)k, (const int4*)v, q8, k8, v8,
                                                          scales, g, chunks);
  else
    quant_fp8_kernel<64><<<grid, kQuantThreads, 0, s>>>((const int4*)q, (const int4*)k, (const int4*)v, q8, k8, v8,
                                                         scales, g, chunks);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* scales,
                                   const int32_t* idx, const int32_t* cnt, int kmax, const Geo& g, float scale,
                                   void* op, int32_t* status, cudaStream_t s) {
  if (g.D != kD || g.blk != kBLK) return cudaErrorNotSupported;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const float scale_log2 = scale * 1.4426950408889634f;
  const size_t bstride = (size_t)g.N * g.heads * kD;
  for (int b = 0; b < g.B; ++b) {
    CUtensorMap tq, tk, tv;
    if (!make_window_map_e4m3(&tq, q8 + b * bstride, g) || !make_window_map_e4m3(&tk, k8 + b * bstride, g) ||
        !make_window_map_e4m3(&tv, v8 + b * bstride, g))
      return cudaErrorInvalidValue;
    dim3 grid(g.Nb, g.heads, 1);
    sparse_attn_fp8_kernel<<<grid, kThreads, kSmem, s>>>(tq, tk, tv, scales, idx, cnt, kmax,
                                                         reinterpret_cast<__nv_bfloat16*>(op), g, scale_log2, status, b);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace rf2
