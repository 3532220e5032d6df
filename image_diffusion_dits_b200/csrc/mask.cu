// Online mask prediction (RainFusion2.0, mlsanity index page, Abstract, insight (1): the
// mean of each block stands in for its tokens when the mask is predicted; insight (3):
// the first-frame sink; sciencestack page, TL;DR: the mask is predicted online, per call).
//
//   pool   : qbar/kbar[b, head, j, :] = fp32 mean of the real tokens of block j.
//            HBM-bound streaming reduction over the permuted Q and K.
//   scores : s[b, head, i, j] = qbar_i . kbar_j * scale on the tensor cores: each mean is
//            split into three bf16 parts (hi + mid + lo, about 24 significant bits) and
//            the six products that matter at fp32 precision are accumulated in fp32.
//            Columns of sink blocks below a multiple of 32 are not computed.
//   topk   : per row, the sink blocks plus the m best other blocks (ties to the lower
//            id) as an ascending list; one warp per row, the exact m-th key found from a
//            value histogram of the row (a bracketed search where the histogram cannot
//            isolate it).
#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace rf2 {
namespace {

// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start while the kernel before it in the stream is finishing; grid_dep_wait blocks
// (in hardware) until that kernel has completed and its writes are visible.  It is a no-op
// for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

// RASTER: Q and K in model order [B, N, heads, D] (a window's rows are gathered line by
// line, (dt, dh) lines of nw consecutive tokens); else in window order [B, Npad, heads, D].
template <bool RASTER>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const int4* __restrict__ qp,
                                                            const int4* __restrict__ kp,
                                                            __nv_bfloat16* __restrict__ q3,
                                                            __nv_bfloat16* __restrict__ k3, Geo g,
                                                            int chunks) {
  const int c = blockIdx.x * kPoolThreads + threadIdx.x;
  const int j = blockIdx.y;
  const int b = blockIdx.z >> 1;
  const int which = blockIdx.z & 1;
  if (c >= chunks) return;
  int nt, nh, nw;
  block_extent(g, j, nt, nh, nw);
  const int4* base = (which ? kp : qp) + c;
  // first token of the window, and the row strides of its (dt, dh) lines
  long long row0, t_stride, h_stride;
  if (RASTER) {
    const int per_t = g.nbh * g.nbw;
    const int tb = j / per_t, hb = (j - tb * per_t) / g.nbw, wb = j - tb * per_t - hb * g.nbw;
    row0 = (long long)b * g.N + ((long long)tb * g.wt * g.H + (long long)hb * g.wh) * g.W + (long long)wb * g.ww;
    t_stride = (long long)g.H * g.W;
    h_stride = g.W;
  } else {
    row0 = (long long)b * g.Npad + (long long)j * g.blk;
    t_stride = (long long)g.wh * g.ww;
    h_stride = g.ww;
  }
  const int4* src = base + row0 * chunks;
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = 0.f;
  // Real rows of the window: (dt < nt, dh < nh, dw < nw); rows are row-major in the window.
  for (int dt = 0; dt < nt; ++dt) {
    for (int dh = 0; dh < nh; ++dh) {
      const int4* rowp = src + (dt * t_stride + dh * h_stride) * chunks;
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
  // the mean x in three bf16 parts: hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid);
  // both differences are exact in fp32
  const long long R = (long long)g.B * g.heads * g.Nb;
  __nv_bfloat16* dst = (which ? k3 : q3) + (((long long)b * g.heads + head) * g.Nb + j) * g.D + d;
  uint32_t part[3][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float x2[2] = {a[2 * e] * inv, a[2 * e + 1] * inv};
    uint16_t hb[3][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float r = x2[h];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const __nv_bfloat16 v = __float2bfloat16_rn(r);
        hb[q][h] = __bfloat16_as_ushort(v);
        r -= __bfloat162float(v);
      }
    }
#pragma unroll
    for (int q = 0; q < 3; ++q) part[q][e] = (uint32_t)hb[q][0] | ((uint32_t)hb[q][1] << 16);
  }
#pragma unroll
  for (int q = 0; q < 3; ++q)
    *reinterpret_cast<uint4*>(dst + q * R * g.D) = make_uint4(part[q][0], part[q][1], part[q][2], part[q][3]);
}

// ------------------------------------------------------------------------------- scores
// One CTA per 128 x 128 tile of s for one (b, head); the column tiles start at the sink
// boundary rounded down to 32 (the top-k reads no sink column).  D is taken 64 columns at a time:
// the three bf16 parts of 128 query means (A) and 128 key means (B) for those columns
// (96 KB) are loaded by TMA (128-byte swizzle, the same K-major layout as the attention
// kernel's Q and K tiles) and thread 0 issues, into one fp32 TMEM accumulator, the
// products lo.hi, hi.lo, mid.mid, mid.hi, hi.mid, hi.hi (smallest first); the dropped
// products are below 2^-24 of the score.  The staging is 96 KB (three parts of A and of
// B, 16 KB each), so two CTAs share an SM and one's loads overlap the other's products
// and stores.  The four warps then read their 32 rows from TMEM and store s * scale,
// turned around in the freed staging so that stores cover whole 128-byte row segments
// (when Nb is a multiple of 4; else element by element).  Rows or columns past Nb in a
// tile come from the next head's means (or TMA zero fill) and are not stored.
constexpr int kSTile = 128;
constexpr int kSThreads = 256;
constexpr uint64_t kScoresWaitNs = 500ull * 1000ull * 1000ull;

template <int D>
struct ScoresCfg {
  static constexpr int kChunks = D / 64;                         // 64-column slices of D
  static constexpr int kPartBytes = kSTile * 64 * 2;             // one part of one operand, one slice
  static constexpr int kOffA = 0;                                // 3 parts of A
  static constexpr int kOffB = 3 * kPartBytes;                   // 3 parts of B
  static constexpr int kOffBar = 6 * kPartBytes;                 // full + done barriers
  static constexpr int kSmem = kOffBar + 64 + 1024;              // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kSThreads) scores_kernel(const __grid_constant__ CUtensorMap ta,
                                                              const __grid_constant__ CUtensorMap tb,
                                                              float* __restrict__ s, Geo g, float scale,
                                                              int jbase, int* __restrict__ status) {
  using C = ScoresCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_s;
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar_full = sbase + C::kOffBar, bar_free = bar_full + 8, bar_done = bar_full + 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.z;
  const int i0 = blockIdx.y * kSTile, j0 = jbase + blockIdx.x * kSTile;
  const long long R = (long long)g.B * g.heads * g.Nb;  // rows of one part
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(&tmem_slot), kSTile);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    ptx::mbar_init(bar_full, 1);
    ptx::mbar_init(bar_free, 1);
    ptx::mbar_init(bar_done, 1);
    abort_s = 0;
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_flag = &abort_s;
  // the block means come from the pool kernel, which may still be finishing
  grid_dep_wait();
  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&ta);
    ptx::prefetch_tmap(&tb);
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(kSTile, kSTile, 0);
    constexpr int kPairs[6][2] = {{2, 0}, {0, 2}, {1, 1}, {1, 0}, {0, 1}, {0, 0}};  // (A part, B part)
    bool ok = true;
    int issued = 0;  // slices whose loads were issued
    for (int kc = 0; ok && kc < C::kChunks; ++kc) {
      // the staging buffers are free once the previous slice's products completed
      if (kc > 0) ok = ptx::mbar_wait(bar_free, (kc - 1) & 1, abort_flag, status, kScoresWaitNs, kStatusTimeout);
      if (!ok) break;
      ptx::mbar_arrive_expect_tx(bar_full, 6 * C::kPartBytes);
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        ptx::tma_load_2d(sbase + C::kOffA + q * C::kPartBytes, &ta, bar_full, kc * 64,
                         (int)(q * R + bh * g.Nb + i0));
        ptx::tma_load_2d(sbase + C::kOffB + q * C::kPartBytes, &tb, bar_full, kc * 64,
                         (int)(q * R + bh * g.Nb + j0));
      }
      issued = kc + 1;
      ok = ptx::mbar_wait(bar_full, kc & 1, abort_flag, status, kScoresWaitNs, kStatusTimeout);
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int pr = 0; pr < 6; ++pr) {
        const uint64_t ad = ptx::smem_desc_sw128(sbase + C::kOffA + kPairs[pr][0] * C::kPartBytes, 16, 1024);
        const uint64_t bd = ptx::smem_desc_sw128(sbase + C::kOffB + kPairs[pr][1] * C::kPartBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 columns = 32 bytes of the swizzled 128-byte rows
          ptx::mma_f16_ss(tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                          (kc > 0 || pr > 0 || kk > 0) ? 1u : 0u);
      }
      ptx::mma_commit(bar_free);
    }
    if (!ok && issued > 0)  // let the copies in flight land before the CTA exits
      ptx::mbar_wait(bar_full, (issued - 1) & 1, nullptr, nullptr, kScoresWaitNs, 0);
    // Arrives once every MMA issued above has completed (at once if none was issued);
    // this thread waits for it without the abort flag, so that no MMA is in flight when
    // the tensor memory is released.
    ptx::mma_commit(bar_done);
    ptx::mbar_wait(bar_done, 0, nullptr, nullptr, kScoresWaitNs, 0);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_done, 0, abort_flag, status, kScoresWaitNs,
                                                         kStatusTimeout)) &&
                  *abort_flag == 0;
  if (ok) {
    ptx::tc_fence_after();
    // warps w and w + 4 read TMEM lanes 32 (w % 4) .. + 31 (tile rows), each half of the
    // columns
    const int quad = warp & 3, c0 = (warp >> 2) * (kSTile / 64);
    const int r = quad * 32 + lane;  // tile row == TMEM lane
    const int gi = i0 + r;
    if ((g.Nb & 3) == 0) {
      // Every MMA has completed, so the operand staging is free: each warp turns its 32 x 32
      // chunk around in shared memory (rows padded to 33 words: no bank conflicts either
      // way) and eight lanes then store one whole 128-byte row segment, so no L2 sector is
      // left half written.
      float* tr = reinterpret_cast<float*>(smem) + warp * (32 * 33);
      const int rr0 = lane >> 3, cc = 4 * (lane & 7);
#pragma unroll 1
      for (int c = c0; c < c0 + kSTile / 64; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) tr[lane * 33 + e] = __uint_as_float(v[e]) * scale;
        __syncwarp();
        const int gj = j0 + c * 32 + cc;  // gj % 4 == 0 and Nb % 4 == 0: gj < Nb covers gj + 3
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + rr0;
          const int gr = i0 + quad * 32 + rr;
          if (gr < g.Nb && gj < g.Nb) {
            const float* t = tr + rr * 33 + cc;
            *reinterpret_cast<float4*>(s + (bh * g.Nb + gr) * (long long)g.Nb + gj) = make_float4(t[0], t[1], t[2], t[3]);
          }
        }
        __syncwarp();
      }
    } else {
      float* srow = s + (bh * g.Nb + gi) * (long long)g.Nb + j0;
#pragma unroll 1
      for (int c = c0; c < c0 + kSTile / 64; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c * 32, v);
        if (gi < g.Nb) {
          const int cb = c * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (j0 + cb + e < g.Nb) srow[cb + e] = __uint_as_float(v[e]) * scale;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kSTile);
  }
}

// ------------------------------------------------------------------------------- top-k
// One warp per (b, head, i) row.  Scores map to order-preserving uint32 keys (every real
// key is > 0; 0 marks a non-candidate).  The threshold thr, the m-th largest candidate
// key, is found exactly: from a 64-bin value histogram of the row (cut_by_histogram), or,
// where that cannot isolate it, by a bracketed search over the key range with warp-wide
// counts (interpolated and bisection steps in turn).  Candidates above thr are kept, and
// equal ones in ascending block order until m are kept.  The output list (sink blocks,
// then kept candidates) is emitted in ascending order with ballots.
constexpr int kTopkWarps = 8;
constexpr int kMaxPerLane = 32;  // Nb <= 1024

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int KPL>
__device__ __forceinline__ int count_ge(const uint32_t (&key)[KPL], uint32_t t) {
  int c = 0;
#pragma unroll
  for (int k = 0; k < KPL; ++k) c += key[k] >= t;
  return (int)__reduce_add_sync(0xffffffffu, (uint32_t)c);
}

// Score of an order key (the inverse of order_key).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Histogram bin of a key: fma(v, sc, off) clamped to [0, 63] and rounded to an integer by
// adding 1.5 * 2^23 (the sum's low mantissa bits are the rounded value).  Each step is
// monotone in v, so the bin never decreases as the key grows; equal keys share a bin.
__device__ __forceinline__ int bin_index(uint32_t k, float sc, float off) {
  return __float_as_int(__fadd_rn(__fmaf_rn(key_value(k), sc, off), 12582912.f)) & 63;
}

// Cut of a row from a 64-bin histogram of the candidate scores, linear in value between
// the row's smallest and largest score.  The bin of a key, min(63, max(0, trunc(fma(v,
// sc, off)))), never decreases as the key grows and equal keys share a bin, so the m-th
// largest key lies in the bin where the count of keys in it and above first reaches m;
// that bin's keys (at most 32, else this returns false and the caller searches) are
// gathered one per lane and ranked exactly.  On success thr is the m-th largest key,
// above = #{key > thr} and eqc = #{key == thr}.
template <int KPL>
__device__ __forceinline__ bool cut_by_histogram(const uint32_t (&key)[KPL], uint32_t lo_key, uint32_t hi_key,
                                                 int m, uint32_t* hist, uint32_t* list, int lane, uint32_t& thr,
                                                 int& above, int& eqc) {
  const float vmin = key_value(lo_key), vmax = key_value(hi_key);
  const float sc = 63.f / (vmax - vmin);
  const float off = -vmin * sc;
  // Equal ends (one bin), or an offset too large for fma(v, sc, off) to stay within 1/4 of
  // [0, 63] on [vmin, vmax] (its rounding errors are below 2 |off| 2^-24): then rounding
  // to the nearest integer gives a bin in 0 .. 63 without clamping.
  if (!(vmax > vmin) || !(fabsf(off) <= 1048576.f)) return false;
  reinterpret_cast<uint2*>(hist)[lane] = make_uint2(0u, 0u);
  __syncwarp();
  int bin[KPL];  // 64 for the pad and sink slots (key 0)
#pragma unroll
  for (int k = 0; k < KPL; ++k) {
    bin[k] = key[k] != 0u ? bin_index(key[k], sc, off) : 64;
    if (key[k] != 0u) atomicAdd(&hist[bin[k]], 1u);
  }
  __syncwarp();
  const uint2 cc = reinterpret_cast<const uint2*>(hist)[lane];  // bins 2 lane, 2 lane + 1
  uint32_t suf = cc.x + cc.y;                                    // keys in bins >= 2 lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += t;
  }
  const uint32_t suf_hi = suf - cc.x;                            // keys in bins >= 2 lane + 1
  // suf never grows with the lane; lane 0 holds every candidate (> m)
  const int L = 31 - __clz(__ballot_sync(0xffffffffu, suf >= (uint32_t)m));
  const bool upper = suf_hi >= (uint32_t)m;
  const int B_l = 2 * lane + (upper ? 1 : 0);
  const int nB_l = (int)(upper ? cc.y : cc.x);
  const int ab_l = (int)(upper ? suf_hi - cc.y : suf_hi);        // keys in bins above B
  const int B = __shfl_sync(0xffffffffu, B_l, L);
  const int nB = __shfl_sync(0xffffffffu, nB_l, L);
  const int ab = __shfl_sync(0xffffffffu, ab_l, L);
  if (nB > 32) return false;
  const int r = m - ab;  // rank of the cut inside bin B, 1 <= r <= nB
  int cnt = 0;
#pragma unroll
  for (int k = 0; k < KPL; ++k) {
    const bool in = bin[k] == B;
    const uint32_t bal = __ballot_sync(0xffffffffu, in);
    if (in) list[cnt + __popc(bal & ((1u << lane) - 1u))] = key[k];
    cnt += __popc(bal);
  }
  __syncwarp();
  const uint32_t x = lane < nB ? list[lane] : 0u;
  int gt = 0, ge = 0;
#pragma unroll 1
  for (int i = 0; i < nB; ++i) {
    const uint32_t y = __shfl_sync(0xffffffffu, x, i);
    gt += y > x;
    ge += y >= x;
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, lane < nB && gt < r && ge >= r);
  const int src = __ffs(hit) - 1;
  thr = __shfl_sync(0xffffffffu, x, src);
  const int g = __shfl_sync(0xffffffffu, gt, src), e = __shfl_sync(0xffffffffu, ge, src);
  above = ab + g;
  eqc = e - g;
  return true;
}

template <int KPL>
__device__ __forceinline__ void topk_row(const float* __restrict__ sr, int32_t* __restrict__ out,
                                         int32_t* __restrict__ cnt_out, int Nb, int kmax, int kept,
                                         int nsink, int lane, uint32_t* hist, uint32_t* list) {
  uint32_t key[KPL];
  uint32_t kmin1 = 0xffffffffu, kmax_key = 0u;  // kmin1: smallest key - 1 (key 0 wraps to the top)
#pragma unroll
  for (int k = 0; k < KPL; ++k) {
    const int j = k * 32 + lane;
    key[k] = (j < Nb && j >= nsink) ? order_key(__ldg(sr + j)) : 0u;
    kmin1 = min(kmin1, key[k] - 1u);
    kmax_key = max(kmax_key, key[k]);
  }
  const int m = kept - nsink;
  const int ncand = Nb - nsink;
  uint32_t thr;       // every candidate key >= thr is kept when take_eq covers all keys == thr
  int above = 0, eqc = 0;
  if (m <= 0) {
    thr = 0xffffffffu;  // none (no real key reaches the top value: keys are < 2^32 - 1 or
                        // equal to it only for NaN patterns, which the ordering puts last)
  } else if (m >= ncand) {
    thr = 1u;           // every candidate
  } else {
    const uint32_t lo_key = __reduce_min_sync(0xffffffffu, kmin1) + 1u;
    const uint32_t hi_key = __reduce_max_sync(0xffffffffu, kmax_key);
    if (!cut_by_histogram<KPL>(key, lo_key, hi_key, m, hist, list, lane, thr, above, eqc)) {
      // Bracket [lo, hi): #{key >= lo} = c_lo >= m > c_hi = #{key >= hi}.  Each step tries
      // a t inside the bracket, interpolated from the two counts on even steps and the
      // midpoint on odd steps, and stops when exactly m keys are >= t.  Otherwise the
      // bracket shrinks to one value: lo is then the m-th largest key.
      uint64_t lo = lo_key;
      uint64_t hi = (uint64_t)hi_key + 1u;
      int c_lo = ncand, c_hi = 0;
#pragma unroll 1
      for (int step = 0; hi - lo > 1; ++step) {
        const uint64_t w = hi - lo;
        uint64_t off;
        if (step & 1) {
          off = w >> 1;
        } else {
          const float frac = (float)(c_lo - m) / (float)(c_lo - c_hi);
          off = (uint64_t)((double)w * (double)frac);
        }
        off = off < 1 ? 1 : (off > w - 1 ? w - 1 : off);
        const uint32_t t = (uint32_t)(lo + off);
        const int c = count_ge<KPL>(key, t);
        if (c == m) {
          lo = t;
          break;
        }
        if (c > m) {
          lo = t;
          c_lo = c;
        } else {
          hi = t;
          c_hi = c;
        }
      }
      thr = (uint32_t)lo;
#pragma unroll
      for (int k = 0; k < KPL; ++k) {
        above += key[k] > thr;
        eqc += key[k] == thr;
      }
      above = (int)__reduce_add_sync(0xffffffffu, (uint32_t)above);
      eqc = (int)__reduce_add_sync(0xffffffffu, (uint32_t)eqc);
    }
  }
  // The sink blocks are ids 0 .. nsink - 1, the smallest, so the list starts with them.
  // Candidates (key != 0) above thr are kept; of those equal to thr, the take_eq lowest
  // ids (all of them when take_eq == eqc).  thr = 1 keeps every candidate.
  const int ns = min(nsink, kmax);
  for (int p = lane; p < ns; p += 32) out[p] = p;
  int pos = nsink;
  const int take_eq = (m > 0 && m < ncand) ? m - above : 0;
  if (m > 0 && (m >= ncand || take_eq == eqc)) {
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      if (k * 32 >= Nb) break;
      const bool take = key[k] >= thr;  // pad and sink slots hold key 0 < thr
      const uint32_t tmask = __ballot_sync(0xffffffffu, take);
      const int p = pos + __popc(tmask & ((1u << lane) - 1u));
      if (take && p < kmax) out[p] = k * 32 + lane;
      pos += __popc(tmask);
    }
  } else if (m > 0) {
    int eq_taken = 0;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      if (k * 32 >= Nb) break;
      const bool eq = key[k] == thr;
      const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
      const bool take = key[k] > thr || (eq && eq_taken + __popc(eqmask & ((1u << lane) - 1u)) < take_eq);
      eq_taken += __popc(eqmask);
      const uint32_t tmask = __ballot_sync(0xffffffffu, take);
      const int p = pos + __popc(tmask & ((1u << lane) - 1u));
      if (take && p < kmax) out[p] = k * 32 + lane;
      pos += __popc(tmask);
    }
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
  __shared__ __align__(8) uint32_t hist_s[kTopkWarps][64];
  __shared__ uint32_t list_s[kTopkWarps][32];
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kTopkWarps + w;
  grid_dep_wait();  // the scores come from the scores kernel, which may still be finishing
  if (row >= rows) return;
  topk_row<KPL>(s + row * Nb, idx + row * kmax, cnt + row, Nb, kmax, kept, nsink, lane, hist_s[w], list_s[w]);
}

// Launch with programmatic stream serialization (the kernel waits for its predecessor
// in the stream with grid_dep_wait before it reads that kernel's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

cudaError_t launch_pool(const void* qp, const void* kp, __nv_bfloat16* q3, __nv_bfloat16* k3, const Geo& g,
                        bool raster, cudaStream_t s) {
  int chunks = g.heads * g.D / 8;
  dim3 grid((chunks + kPoolThreads - 1) / kPoolThreads, g.Nb, g.B * 2);
  if (raster)
    pool_kernel<true><<<grid, kPoolThreads, 0, s>>>((const int4*)qp, (const int4*)kp, q3, k3, g, chunks);
  else
    pool_kernel<false><<<grid, kPoolThreads, 0, s>>>((const int4*)qp, (const int4*)kp, q3, k3, g, chunks);
  return cudaGetLastError();
}

// 2-D view [3 * B*heads*Nb rows, D] of the bf16 parts; box 64 columns x 128 rows, 128-byte
// swizzle (the K-major operand layout of the MMAs).
static bool make_parts_map(CUtensorMap* m, const void* base, const Geo& g) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)g.D, (cuuint64_t)3 * g.B * g.heads * g.Nb};
  cuuint64_t strides[1] = {(cuuint64_t)g.D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kSTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_scores_d(const __nv_bfloat16* q3, const __nv_bfloat16* k3, float* scores, const Geo& g,
                            float scale, int nsink, int32_t* status, cudaStream_t s) {
  using C = ScoresCfg<D>;
  // The top-k never reads a sink column's score (the sink is always kept): columns start
  // at the sink boundary rounded down to 32 (so that stores stay 128-byte aligned).
  const int jbase = nsink & ~31;
  if (jbase >= g.Nb) return cudaSuccess;  // every block is a sink block: no score is read
  CUtensorMap ta, tb;
  if (!make_parts_map(&ta, q3, g) || !make_parts_map(&tb, k3, g)) return cudaErrorInvalidValue;
  static int configured_device = -1;  // one flag per instance (per D)
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid((g.Nb - jbase + kSTile - 1) / kSTile, (g.Nb + kSTile - 1) / kSTile, g.B * g.heads);
  return launch_dependent(scores_kernel<D>, grid, dim3(kSThreads), C::kSmem, s, ta, tb, scores, g, scale, jbase,
                          status);
}

cudaError_t launch_scores(const __nv_bfloat16* q3, const __nv_bfloat16* k3, float* scores, const Geo& g,
                          float scale, int nsink, int32_t* status, cudaStream_t s) {
  if (g.D == 128) return launch_scores_d<128>(q3, k3, scores, g, scale, nsink, status, s);
  return launch_scores_d<64>(q3, k3, scores, g, scale, nsink, status, s);
}

cudaError_t launch_topk(const float* scores, int32_t* idx, int32_t* cnt, int kmax, int kept,
                        int nsink, const Geo& g, cudaStream_t s) {
  if (g.Nb > kMaxPerLane * 32) return cudaErrorNotSupported;
  long long rows = (long long)g.B * g.heads * g.Nb;
  long long grid = (rows + kTopkWarps - 1) / kTopkWarps;
  // keys per lane: the smallest instance that covers Nb (each unused slot costs
  // instructions in every pass over the keys)
  const int kpl = (g.Nb + 31) / 32;
  const unsigned blocks = (unsigned)grid, threads = kTopkWarps * 32;
  cudaError_t e;
  if (kpl <= 4)
    e = launch_dependent(topk_kernel<4>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 8)
    e = launch_dependent(topk_kernel<8>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 16)
    e = launch_dependent(topk_kernel<16>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 19)
    e = launch_dependent(topk_kernel<19>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 21)
    e = launch_dependent(topk_kernel<21>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 24)
    e = launch_dependent(topk_kernel<24>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else if (kpl <= 30)
    e = launch_dependent(topk_kernel<30>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  else
    e = launch_dependent(topk_kernel<32>, dim3(blocks), dim3(threads), 0, s, scores, idx, cnt, g.Nb, rows, kmax, kept, nsink);
  return e;
}

}  // namespace rf2
