// Online mask prediction (RainFusion2.0, mlsanity index page, Abstract, insight (1)
// "block-wise mean values as representative tokens for sparse mask prediction" and
// insight (3) "first-frame sink"; sciencestack page, TL;DR "online adaptive").
//
//   pool   : qbar/kbar[b, head, j, :] = fp32 mean of the real tokens of block j.
//            HBM-bound streaming reduction over the permuted Q and K.
//   scores : s[b, head, i, j] = qbar_i . kbar_j * scale, an fp32 register-tiled product.
//   topk   : per row, the sink blocks plus the m best other blocks (ties to the lower
//            id) as an ascending list; one warp per row, exact bitwise search.
#include "rf2_common.cuh"

namespace rf2 {
namespace {

// ------------------------------------------------------------------------------- pool
// CTA = (16-byte chunk group of 128 chunks = 1024 channels, block j, b*2 + tensor).
// Each thread owns one 16-byte chunk (8 channels) of the heads*D row and sums it over
// the block's real rows, 8 rows in flight.
constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 8;

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const int4& v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 f = __bfloat1622float2(h[k]);
    a[2 * k] += f.x;
    a[2 * k + 1] += f.y;
  }
}

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const int4* __restrict__ qp,
                                                            const int4* __restrict__ kp,
                                                            float* __restrict__ qbar,
                                                            float* __restrict__ kbar, Geo g,
                                                            int chunks) {
  const int c = blockIdx.x * kPoolThreads + threadIdx.x;
  const int j = blockIdx.y;
  const int b = blockIdx.z >> 1;
  const int which = blockIdx.z & 1;
  if (c >= chunks) return;
  const int4* src = (which ? kp : qp) + ((long long)b * g.Npad + (long long)j * g.blk) * chunks + c;
  int nt, nh, nw;
  block_extent(g, j, nt, nh, nw);
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = 0.f;
  // Real rows of the window: (dt < nt, dh < nh, dw < nw); rows are row-major in the window.
  for (int dt = 0; dt < nt; ++dt) {
    for (int dh = 0; dh < nh; ++dh) {
      const int4* rowp = src + (long long)((dt * g.wh + dh) * g.ww) * chunks;
      int dw = 0;
      for (; dw + kPoolUnroll <= nw; dw += kPoolUnroll) {
        int4 v[kPoolUnroll];
#pragma unroll
        for (int u = 0; u < kPoolUnroll; ++u) v[u] = __ldcs(rowp + (long long)(dw + u) * chunks);
#pragma unroll
        for (int u = 0; u < kPoolUnroll; ++u) acc_bf16x8(a, v[u]);
      }
      for (; dw < nw; ++dw) acc_bf16x8(a, __ldcs(rowp + (long long)dw * chunks));
    }
  }
  const float inv = 1.0f / (float)(nt * nh * nw);
  const int ch = c * 8;           // channel within heads*D
  const int head = ch / g.D;
  const int d = ch - head * g.D;
  float* dst = (which ? kbar : qbar) + (((long long)b * g.heads + head) * g.Nb + j) * g.D + d;
  float4 o0 = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
  float4 o1 = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
  reinterpret_cast<float4*>(dst)[0] = o0;
  reinterpret_cast<float4*>(dst)[1] = o1;
}

// ------------------------------------------------------------------------------- scores
// CTA computes a 64 x 64 tile of s = qbar kbar^T * scale for one (b, head); 256 threads,
// each a 4 x 4 register tile.  Both 64 x D operand tiles are staged in shared memory in
// one pass (one exposed L2 latency per CTA), stored d-major with rows padded to 68
// floats so that a thread's 4 rows (and 4 columns) are one aligned float4 and the
// transposing stores hit distinct banks.  Every score is a sequential fmaf chain over d.
constexpr int kSTile = 64;
constexpr int kSPad = kSTile + 4;

template <int D>
__global__ void __launch_bounds__(256) scores_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     float* __restrict__ s, Geo g, float scale) {
  extern __shared__ __align__(16) float ssm[];
  float* qs = ssm;               // [D][kSPad]
  float* ks = ssm + D * kSPad;   // [D][kSPad]
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kSTile;
  const int j0 = blockIdx.x * kSTile;
  const float* qb = qbar + (long long)bh * g.Nb * D;
  const float* kb = kbar + (long long)bh * g.Nb * D;
  const int tid = threadIdx.x;
  const int ti = tid >> 4;   // rows 4*ti .. 4*ti+3
  const int tj = tid & 15;   // cols 4*tj .. 4*tj+3
  // fill: consecutive threads take consecutive rows of the same 4 d
#pragma unroll 4
  for (int f = tid; f < kSTile * D / 4; f += 256) {
    const int r = f % kSTile, d4 = f / kSTile;
    const int gi = i0 + r, gj = j0 + r;
    const float4 qv = gi < g.Nb ? __ldg(reinterpret_cast<const float4*>(qb + (long long)gi * D) + d4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 kv = gj < g.Nb ? __ldg(reinterpret_cast<const float4*>(kb + (long long)gj * D) + d4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    qs[(4 * d4 + 0) * kSPad + r] = qv.x;
    qs[(4 * d4 + 1) * kSPad + r] = qv.y;
    qs[(4 * d4 + 2) * kSPad + r] = qv.z;
    qs[(4 * d4 + 3) * kSPad + r] = qv.w;
    ks[(4 * d4 + 0) * kSPad + r] = kv.x;
    ks[(4 * d4 + 1) * kSPad + r] = kv.y;
    ks[(4 * d4 + 2) * kSPad + r] = kv.z;
    ks[(4 * d4 + 3) * kSPad + r] = kv.w;
  }
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 8
  for (int d = 0; d < D; ++d) {
    const float4 qv = reinterpret_cast<const float4*>(qs + d * kSPad)[ti];
    const float4 kv = reinterpret_cast<const float4*>(ks + d * kSPad)[tj];
    const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
    const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(qa[a], ka[c], acc[a][c]);
  }
  float* sb = s + (long long)bh * g.Nb * g.Nb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int gi = i0 + 4 * ti + a;
    if (gi >= g.Nb) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + 4 * tj + c;
      if (gj < g.Nb) sb[(long long)gi * g.Nb + gj] = acc[a][c] * scale;
    }
  }
}

// ------------------------------------------------------------------------------- top-k
// One warp per (b, head, i) row.  Scores map to order-preserving uint32 keys (every real
// key is > 0; 0 marks a non-candidate).  The m-th largest candidate key is found exactly
// by a 32-step bitwise search with warp-wide counts; candidates above it are kept, and
// equal ones in ascending block order until m are kept.  The output list (sink blocks and kept candidates) is
// emitted in ascending order with ballots.
constexpr int kTopkWarps = 8;
constexpr int kMaxPerLane = 32;  // Nb <= 1024

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int KPL>
__device__ __forceinline__ void topk_row(const float* __restrict__ sr, int32_t* __restrict__ out,
                                         int32_t* __restrict__ cnt_out, int Nb, int kmax, int kept,
                                         int nsink, int lane) {
  uint32_t key[KPL];
#pragma unroll
  for (int k = 0; k < KPL; ++k) {
    const int j = k * 32 + lane;
    key[k] = (j < Nb && j >= nsink) ? order_key(__ldg(sr + j)) : 0u;
  }
  const int m = kept - nsink;
  const int ncand = Nb - nsink;
  uint32_t thr = 0;   // the m-th largest candidate key
  int take_eq = 0;    // how many keys equal to thr are kept (lowest ids first)
  if (m > 0 && m < ncand) {
    // Bitwise search from the most significant bit: the largest t with
    // #{key >= t} >= m is the m-th largest key.
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t t = thr | (1u << bit);
      int c = 0;
#pragma unroll
      for (int k = 0; k < KPL; ++k) c += key[k] >= t;
      if ((int)__reduce_add_sync(0xffffffffu, (uint32_t)c) >= m) thr = t;
    }
    int above = 0;
#pragma unroll
    for (int k = 0; k < KPL; ++k) above += key[k] > thr;
    take_eq = m - (int)__reduce_add_sync(0xffffffffu, (uint32_t)above);
  } else if (m >= ncand) {
    thr = 1u;  // every candidate
  } else {
    thr = 0xffffffffu;  // m == 0: none
  }
  int pos = 0;
  int eq_taken = 0;
  const bool all = m >= ncand;
  const bool some = m > 0 && m < ncand;
#pragma unroll
  for (int k = 0; k < KPL; ++k) {
    if (k * 32 >= Nb) break;
    const int j = k * 32 + lane;
    const bool in_range = j < Nb;
    const bool is_sink = in_range && j < nsink;
    const bool above = in_range && !is_sink && (all ? key[k] != 0u : key[k] > thr);
    const bool eq = in_range && !is_sink && some && key[k] == thr;
    const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_taken + __popc(eqmask & ((1u << lane) - 1u));
    const bool take = is_sink || above || (eq && eq_rank < take_eq);
    eq_taken += __popc(eqmask);
    const uint32_t tmask = __ballot_sync(0xffffffffu, take);
    const int p = pos + __popc(tmask & ((1u << lane) - 1u));
    if (take && p < kmax) out[p] = j;
    pos += __popc(tmask);
  }
  for (int p = pos + lane; p < kmax; p += 32) out[p] = -1;
  if (lane == 0) *cnt_out = pos;
}

template <int KPL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ s,
                                                               int32_t* __restrict__ idx,
                                                               int32_t* __restrict__ cnt,
                                                               int Nb, long long rows, int kmax,
                                                               int kept, int nsink) {
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kTopkWarps + w;
  if (row >= rows) return;
  topk_row<KPL>(s + row * Nb, idx + row * kmax, cnt + row, Nb, kmax, kept, nsink, lane);
}

}  // namespace

cudaError_t launch_pool(const void* qp, const void* kp, float* qbar, float* kbar, const Geo& g,
                        cudaStream_t s) {
  int chunks = g.heads * g.D / 8;
  dim3 grid((chunks + kPoolThreads - 1) / kPoolThreads, g.Nb, g.B * 2);
  pool_kernel<<<grid, kPoolThreads, 0, s>>>((const int4*)qp, (const int4*)kp, qbar, kbar, g,
                                            chunks);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_scores_d(const float* qbar, const float* kbar, float* scores, const Geo& g,
                            float scale, cudaStream_t s) {
  const int smem = 2 * D * kSPad * (int)sizeof(float);
  static int configured_device = -1;  // one flag per instance (per D)
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid((g.Nb + kSTile - 1) / kSTile, (g.Nb + kSTile - 1) / kSTile, g.B * g.heads);
  scores_kernel<D><<<grid, 256, smem, s>>>(qbar, kbar, scores, g, scale);
  return cudaGetLastError();
}

cudaError_t launch_scores(const float* qbar, const float* kbar, float* scores, const Geo& g,
                          float scale, cudaStream_t s) {
  if (g.D == 128) return launch_scores_d<128>(qbar, kbar, scores, g, scale, s);
  return launch_scores_d<64>(qbar, kbar, scores, g, scale, s);
}

cudaError_t launch_topk(const float* scores, int32_t* idx, int32_t* cnt, int kmax, int kept,
                        int nsink, const Geo& g, cudaStream_t s) {
  if (g.Nb > kMaxPerLane * 32) return cudaErrorNotSupported;
  long long rows = (long long)g.B * g.heads * g.Nb;
  long long grid = (rows + kTopkWarps - 1) / kTopkWarps;
  // keys per lane: the smallest instance that covers Nb
  if (g.Nb <= 256)
    topk_kernel<8><<<(unsigned)grid, kTopkWarps * 32, 0, s>>>(scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (g.Nb <= 512)
    topk_kernel<16><<<(unsigned)grid, kTopkWarps * 32, 0, s>>>(scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (g.Nb <= 768)
    topk_kernel<24><<<(unsigned)grid, kTopkWarps * 32, 0, s>>>(scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else
    topk_kernel<32><<<(unsigned)grid, kTopkWarps * 32, 0, s>>>(scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  return cudaGetLastError();
}

}  // namespace rf2
