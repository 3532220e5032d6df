// 3D-window permutation and its inverse (RainFusion2.0, mlsanity index page, Abstract,
// insight (2); sciencestack page, TL;DR "3D window permutation", Figure 3).
//
// Both are pure row gathers of [*, heads*D] bf16 rows: HBM-bound copies.  One CTA moves
// kRowsPerCta destination rows; each thread moves 16-byte chunks with 4 loads in flight
// before the matching stores, so every warp issues 512 contiguous bytes per access.
#include "rf2_common.cuh"

namespace rf2 {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerCta = 4;
constexpr int kUnroll = 4;

// Moves one row of `chunks` 16-byte chunks from src (or zeros when src == nullptr).
__device__ __forceinline__ void copy_row(const int4* __restrict__ src, int4* __restrict__ dst,
                                         int chunks) {
  for (int base = threadIdx.x; base < chunks; base += kThreads * kUnroll) {
    int4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int c = base + u * kThreads;
      if (src != nullptr && c < chunks) {
        v[u] = __ldcs(src + c);
      } else {
        v[u] = make_int4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int c = base + u * kThreads;
      if (c < chunks) __stcs(dst + c, v[u]);
    }
  }
}

__global__ void __launch_bounds__(kThreads) permute_kernel(const int4* __restrict__ x,
                                                           int4* __restrict__ xp, Geo g,
                                                           int chunks) {
  long long total = (long long)g.B * g.Npad;
  long long row0 = (long long)blockIdx.x * kRowsPerCta;
  for (int r = 0; r < kRowsPerCta; ++r) {
    long long row = row0 + r;
    if (row >= total) return;
    long long b = row / g.Npad;
    long long p = row - b * g.Npad;
    long long n = pos_to_token(g, p);
    const int4* src = n < 0 ? nullptr : x + (b * g.N + n) * chunks;
    copy_row(src, xp + row * chunks, chunks);
  }
}

__global__ void __launch_bounds__(kThreads) unpermute_kernel(const int4* __restrict__ xp,
                                                             int4* __restrict__ x, Geo g,
                                                             int chunks) {
  long long total = (long long)g.B * g.N;
  long long row0 = (long long)blockIdx.x * kRowsPerCta;
  for (int r = 0; r < kRowsPerCta; ++r) {
    long long row = row0 + r;
    if (row >= total) return;
    long long b = row / g.N;
    long long n = row - b * g.N;
    long long p = token_to_pos(g, n);
    copy_row(xp + (b * g.Npad + p) * chunks, x + row * chunks, chunks);
  }
}

}  // namespace

cudaError_t launch_permute(const void* x, void* xp, const Geo& g, cudaStream_t s) {
  int chunks = g.heads * g.D * 2 / 16;
  long long rows = (long long)g.B * g.Npad;
  long long grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
  permute_kernel<<<(unsigned)grid, kThreads, 0, s>>>((const int4*)x, (int4*)xp, g, chunks);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* xp, void* x, const Geo& g, cudaStream_t s) {
  int chunks = g.heads * g.D * 2 / 16;
  long long rows = (long long)g.B * g.N;
  long long grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
  unpermute_kernel<<<(unsigned)grid, kThreads, 0, s>>>((const int4*)xp, (int4*)x, g, chunks);
  return cudaGetLastError();
}

}  // namespace rf2
