// Block-sparse flash attention over the kept key blocks, sm_100a (tcgen05 + TMEM + TMA).
//
// RainFusion2.0 (mlsanity index page: title "block-wise sparse attention"; Abstract:
// skipping the computation of insignificant tokens).  For query block i of (b, head):
//   O_i = softmax(Q_i K_S^T * scale + M) V_S,   S = kept key blocks of the row,
//   M = -inf on pad keys (partial windows at the high end of an axis).
//
// One CTA per (query block, head, batch); query tile of 128 rows (a 64-token block uses
// the first 64).  Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Reads the S row from
//              TMEM in one load, online softmax in fp32 (exp2 domain), writes P (bf16
//              pairs) back into the same TMEM columns, rescales O in TMEM when the
//              running max grows by more than 2^8, and runs the epilogue.
//   warp 4     TMA producer: Q once, then K_j and V_j of each kept block j through two
//              independent 2-stage shared-memory rings.
//   warp 5     MMA issuer: S_i = Q K_i^T (both operands from shared memory, K-major) into
//              one of three TMEM S/P buffers, then O += P_{i-1} V_{i-1} with P read from
//              TMEM and V from shared memory (MN-major), one step behind, so the tensor
//              core computes S_{i+1} while the softmax works on S_i.
// TMEM: three 128-column S/P buffers and the 128-column O accumulator (512 columns).
// Every mbarrier wait is bounded in time; on expiry the CTA raises a timeout status,
// stops issuing work, drains what it issued and returns.
#include <cuda.h>

#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace rf2 {
namespace {

constexpr int kBM = 128;            // query rows per tile (TMEM lanes)
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kSBufs = 3;           // S/P buffers in TMEM
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 384;    // S/P buffer b at column 128*b
constexpr uint64_t kWaitLimitNs = 500ull * 1000ull * 1000ull;  // 0.5 s per wait

template <int D, int BLK>
struct Cfg {
  static constexpr int kAtomsD = D / 64;       // 128-byte column atoms of a [rows, D] tile
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = BLK * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffList = kOffV + 2 * kKVBytes;  // int32[1024] compacted kept list
  static constexpr int kOffBar = kOffList + 4096;        // mbarriers
  static constexpr int kOffMisc = kOffBar + 256;         // tmem slot, counts, flags
  static constexpr int kUsed = kOffMisc + 64;
  // Requested dynamic smem: 1 KB alignment slack; at least 116 KB so that at most one
  // CTA is resident per SM (each CTA allocates all 512 TMEM columns).
  static constexpr int kSmem = (kUsed + 1024) > 118784 ? (kUsed + 1024) : 118784;
};

// Barrier slots (8 bytes each) at kOffBar.
enum : int {
  BAR_Q = 0,
  BAR_KFULL = 1,    // +stage (2)
  BAR_KEMPTY = 3,   // +stage (2)
  BAR_VFULL = 5,    // +stage (2)
  BAR_VEMPTY = 7,   // +stage (2)
  BAR_SFULL = 9,    // +buffer (3): S_i computed
  BAR_PFULL = 12,   // +buffer (3): P_i written to TMEM
  BAR_SFREE = 15,   // +buffer (3): P_i V_i completed, buffer reusable
  BAR_ORDY = 18,    // every P_i V_i completed (O stable)
  BAR_DONE = 19,
  BAR_COUNT = 20
};

struct Misc {
  uint32_t tmem_base;
  int n;       // kept blocks after dropping out-of-range ids
  int abort;   // set by any role that gave up on a wait
  int pad;
};

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const int32_t* __restrict__ idx,
                       const int32_t* __restrict__ cnt, int kmax,
                       __nv_bfloat16* __restrict__ op, Geo g, float scale_log2,
                       int* __restrict__ status) {
  using C = Cfg<D, BLK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  int* list_s = reinterpret_cast<int*>(smem + C::kOffList);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kOffMisc);
  volatile int* abort_flag = &misc->abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qblk = blockIdx.x;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const long long row = ((long long)b * g.heads + head) * g.Nb + qblk;
  const long long brow0 = (long long)b * g.Npad;  // first row of batch b in the 3-D maps

  // ---------------------------------------------------------------- setup
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(&misc->tmem_base), kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(BAR_KFULL + s), 1);
      ptx::mbar_init(bar(BAR_KEMPTY + s), 1);
      ptx::mbar_init(bar(BAR_VFULL + s), 1);
      ptx::mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      ptx::mbar_init(bar(BAR_SFULL + s), 1);
      ptx::mbar_init(bar(BAR_PFULL + s), 4);
      ptx::mbar_init(bar(BAR_SFREE + s), 1);
    }
    ptx::mbar_init(bar(BAR_ORDY), 1);
    ptx::mbar_init(bar(BAR_DONE), 1);
    misc->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    // Compact the kept list into shared memory, dropping ids outside [0, Nb).
    int n_in = cnt[row];
    n_in = n_in < 0 ? 0 : (n_in > kmax ? kmax : n_in);
    n_in = n_in > 1024 ? 1024 : n_in;  // capacity of the shared-memory list
    const int32_t* lst = idx + row * kmax;
    int n_out = 0;
    bool bad = false;
    for (int e0 = 0; e0 < n_in; e0 += 32) {
      int e = e0 + lane;
      int j = e < n_in ? lst[e] : -1;
      bool ok = e < n_in && j >= 0 && j < g.Nb;
      bad |= (e < n_in) && !ok;
      uint32_t m = __ballot_sync(0xffffffffu, ok);
      if (ok) list_s[n_out + __popc(m & ((1u << lane) - 1u))] = j;
      n_out += __popc(m);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && status != nullptr)
      atomicCAS(status, 0, kStatusBadIndex);
    if (lane == 0) misc->n = n_out;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int n = misc->n;

  if (n > 0) {
    if (warp == kProducerWarp && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tk);
      ptx::prefetch_tmap(&tv);
      ptx::mbar_arrive_expect_tx(bar(BAR_Q), C::kQBytes);
#pragma unroll
      for (int a = 0; a < C::kAtomsD; ++a)
        ptx::tma_load_3d(sQ + a * (kBM * 128), &tq, bar(BAR_Q), a * 64, head,
                         (int)(brow0 + (long long)qblk * BLK));
      int issued_k[2] = {-1, -1}, issued_v[2] = {-1, -1};
      for (int i = 0; i < n; ++i) {
        const int s = i & 1;
        const int zrow = (int)(brow0 + (long long)list_s[i] * BLK);
        if (i >= 2 && !ptx::mbar_wait(bar(BAR_KEMPTY + s), ((i >> 1) & 1) ^ 1, abort_flag, status,
                                      kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_KFULL + s), C::kKVBytes);
#pragma unroll
        for (int a = 0; a < C::kAtomsD; ++a)
          ptx::tma_load_3d(sK + s * C::kKVBytes + a * (BLK * 128), &tk, bar(BAR_KFULL + s), a * 64,
                           head, zrow);
        issued_k[s] = i;
        if (i >= 2 && !ptx::mbar_wait(bar(BAR_VEMPTY + s), ((i >> 1) & 1) ^ 1, abort_flag, status,
                                      kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_VFULL + s), C::kKVBytes);
#pragma unroll
        for (int a = 0; a < C::kAtomsD; ++a)
          ptx::tma_load_3d(sV + s * C::kKVBytes + a * (BLK * 128), &tv, bar(BAR_VFULL + s), a * 64,
                           head, zrow);
        issued_v[s] = i;
      }
      if (*abort_flag) {
        // Let every copy this thread issued land before the CTA can exit.
        ptx::mbar_wait(bar(BAR_Q), 0, nullptr, nullptr, kWaitLimitNs, 0);
        for (int s = 0; s < 2; ++s) {
          if (issued_k[s] >= 0)
            ptx::mbar_wait(bar(BAR_KFULL + s), (issued_k[s] >> 1) & 1, nullptr, nullptr,
                           kWaitLimitNs, 0);
          if (issued_v[s] >= 0)
            ptx::mbar_wait(bar(BAR_VFULL + s), (issued_v[s] >> 1) & 1, nullptr, nullptr,
                           kWaitLimitNs, 0);
        }
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, BLK, 0);
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, D, 1);
      bool ok = ptx::mbar_wait(bar(BAR_Q), 0, abort_flag, status, kWaitLimitNs, kStatusTimeout);
      ptx::tc_fence_after();
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        const int pb = i % kSBufs;
        if (!ptx::mbar_wait(bar(BAR_PFULL + pb), (i / kSBufs) & 1, abort_flag, status,
                            kWaitLimitNs, kStatusTimeout))
          return false;
        if (!ptx::mbar_wait(bar(BAR_VFULL + s), (i >> 1) & 1, abort_flag, status, kWaitLimitNs,
                            kStatusTimeout))
          return false;
        ptx::tc_fence_after();
        const uint32_t vs = sV + s * C::kKVBytes;
        const uint32_t pt = tmem + (uint32_t)(128 * pb);
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          // A = P [128 x BLK] in TMEM: 16 keys = 8 columns of bf16 pairs.
          // B = V [BLK keys x D] read as N x K MN-major: 16 keys = 16 rows of 128 bytes;
          // the D atoms (64 columns each) are BLK*128 bytes apart.
          const uint64_t bd = ptx::smem_desc_sw128(vs + kk * (16 * 128), BLK * 128, 1024);
          ptx::mma_f16_ts(tmem + kTmemO, pt + kk * 8, bd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(bar(BAR_ORDY));
        ptx::mma_commit(bar(BAR_VEMPTY + s));
        ptx::mma_commit(bar(BAR_SFREE + pb));
        return true;
      };
      for (int i = 0; ok && i < n; ++i) {
        const int s = i & 1;
        const int sb = i % kSBufs;
        if (!ptx::mbar_wait(bar(BAR_KFULL + s), (i >> 1) & 1, abort_flag, status, kWaitLimitNs,
                            kStatusTimeout)) {
          ok = false;
          break;
        }
        // S/P buffer sb last held P_{i-3}: reusable once P_{i-3} V_{i-3} has completed.
        if (i >= kSBufs && !ptx::mbar_wait(bar(BAR_SFREE + sb), ((i / kSBufs) - 1) & 1, abort_flag,
                                           status, kWaitLimitNs, kStatusTimeout)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t ks = sK + s * C::kKVBytes;
        const uint32_t dS = tmem + (uint32_t)(128 * sb);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;  // 16 columns = 32 bytes inside an atom
          const uint64_t ad = ptx::smem_desc_sw128(sQ + (kk >> 2) * (kBM * 128) + koff, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(ks + (kk >> 2) * (BLK * 128) + koff, 16, 1024);
          ptx::mma_f16_ss(dS, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(BAR_SFULL + sb));
        ptx::mma_commit(bar(BAR_KEMPTY + s));
        if (i >= 1 && !issue_pv(i - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_pv(n - 1);
      // All MMAs this thread issued have completed once BAR_DONE fires.
      ptx::mma_commit(bar(BAR_DONE));
      ptx::mbar_wait(bar(BAR_DONE), 0, nullptr, nullptr, kWaitLimitNs, 0);
    } else if (warp < 4) {
      // ------------------------------------------------------------ softmax + epilogue
      const int r = tid;  // query row == TMEM lane
      const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
      float m_run = -INFINITY;
      float l_run = 0.f;
      bool ok = true;
      for (int i = 0; i < n; ++i) {
        const int sb = i % kSBufs;
        const int j = list_s[i];
        const uint32_t srow = tmem + lane_base + (uint32_t)(128 * sb);
        // Waits are per thread; giving up is decided for the whole warp so that the
        // warp-wide tcgen05 and shuffle operations below stay converged.
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_SFULL + sb), (i / kSBufs) & 1, abort_flag,
                                                     status, kWaitLimitNs, kStatusTimeout))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float x[BLK];
        {
          // the whole S row in one TMEM load (one round trip)
          uint32_t t[BLK];
          if constexpr (BLK == 128)
            ptx::tmem_ld32x128(srow, t);
          else
            ptx::tmem_ld32x64(srow, t);
#pragma unroll
          for (int c = 0; c < BLK; ++c) x[c] = __uint_as_float(t[c]);
        }
        // Pad keys of a partial window get -inf; validity is per column, the same for
        // every row, so each lane evaluates 1/32 of the columns and the warp shares bits.
        int nt, nh, nw;
        block_extent(g, j, nt, nh, nw);
        if (nt < g.wt || nh < g.wh || nw < g.ww) {
          uint32_t vm[BLK / 32];
          const int whw = g.wh * g.ww;
#pragma unroll
          for (int q = 0; q < BLK / 32; ++q) {
            const int c = q * 32 + lane;
            const int dt = c / whw;
            const int rem = c - dt * whw;
            const int dh = rem / g.ww;
            const int dw = rem - dh * g.ww;
            vm[q] = __ballot_sync(0xffffffffu, dt < nt && dh < nh && dw < nw);
          }
#pragma unroll
          for (int c = 0; c < BLK; ++c)
            if (!((vm[c >> 5] >> (c & 31)) & 1u)) x[c] = -INFINITY;
        }
        // Row max of the raw scores (scale > 0 commutes with max) over 8 independent
        // chains, so the reduction is not one long dependency chain.
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = x[e];
#pragma unroll
        for (int c = 8; c < BLK; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        // Running max in exp2 units: only moved when it grows by more than 8, so P <= 2^8
        // and O needs rescaling rarely; the final O / l is unchanged by this.
        const float m_new = fmaxf(m_run, mx * scale_log2);
        const bool grow = m_new > m_run + 8.0f;  // always true on the first block
        float alpha = 1.0f;
        if (grow) {
          alpha = ptx::ex2(m_run - m_new);  // 0 on the first block
          l_run *= alpha;
          m_run = m_new;
        }
        if (i >= 1 && __any_sync(0xffffffffu, grow)) {
          // O is stable once P_{i-1} V_{i-1} has completed.  S_i completing implies that
          // P_{i-2} V_{i-2} has (a commit covers every earlier MMA), and P_i V_i cannot
          // start before this warp publishes P_i, so BAR_ORDY is in phase i-1 or i here
          // and its parity wait is unambiguous.  tcgen05.ld/st are
          // warp-wide: the warp rescales its 32 rows of O together, rows that did not
          // grow with alpha = 1.
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_ORDY), (i - 1) & 1, abort_flag,
                                                       status, kWaitLimitNs, kStatusTimeout))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t t[32];
            ptx::tmem_ld32(tmem + lane_base + kTmemO + c * 32, t);
#pragma unroll
            for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
            ptx::tmem_st32(tmem + lane_base + kTmemO + c * 32, t);
          }
        }
        // P = exp2(s * scale_log2 - m_run): one FFMA and one ex2 per element, rounded to
        // bf16 pairs and written over the first BLK/2 columns of this S buffer (the A
        // operand of P V); the row sum uses 8 independent accumulators.
        const float neg_m = -m_run;
        float ls[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ls[e] = 0.f;
        uint32_t pk[BLK / 2];
#pragma unroll
        for (int c2 = 0; c2 < BLK / 2; ++c2) {
          const float p0 = ptx::ex2(fmaf(x[2 * c2], scale_log2, neg_m));
          const float p1 = ptx::ex2(fmaf(x[2 * c2 + 1], scale_log2, neg_m));
          ls[(2 * c2) & 7] += p0;
          ls[(2 * c2 + 1) & 7] += p1;
          pk[c2] = ptx::pack_bf16(p0, p1);
        }
        if constexpr (BLK == 128) {
          ptx::tmem_st32x64(srow, pk);
        } else {
          ptx::tmem_st32(srow, pk);
        }
        ptx::tmem_wait_st();
        l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(BAR_PFULL + sb));
      }
      // ---------------------------------------------------------- epilogue
      // BAR_DONE fires once every MMA of the CTA has completed (the softmax skips most
      // BAR_ORDY phases, so a parity wait there could alias an older phase).
      if (ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_DONE), 0, abort_flag, status,
                                                       kWaitLimitNs, kStatusTimeout))) {
        ptx::tc_fence_after();
        const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
        __nv_bfloat16* orow =
            op + ((brow0 + (long long)qblk * BLK + r) * g.heads + head) * (long long)D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t t[32];
          ptx::tmem_ld32(tmem + lane_base + kTmemO + c * 32, t);
          if (r < BLK) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = ptx::pack_bf16(__uint_as_float(t[8 * v + 0]) * inv, __uint_as_float(t[8 * v + 1]) * inv);
              w.y = ptx::pack_bf16(__uint_as_float(t[8 * v + 2]) * inv, __uint_as_float(t[8 * v + 3]) * inv);
              w.z = ptx::pack_bf16(__uint_as_float(t[8 * v + 4]) * inv, __uint_as_float(t[8 * v + 5]) * inv);
              w.w = ptx::pack_bf16(__uint_as_float(t[8 * v + 6]) * inv, __uint_as_float(t[8 * v + 7]) * inv);
              reinterpret_cast<uint4*>(orow + c * 32)[v] = w;
            }
          }
        }
      }
    }
  } else if (warp < 4 && tid < BLK) {
    // No kept block: the row attends to nothing; write zeros.
    __nv_bfloat16* orow = op + ((brow0 + (long long)qblk * BLK + tid) * g.heads + head) * (long long)D;
    for (int v = 0; v < D / 8; ++v) reinterpret_cast<uint4*>(orow)[v] = make_uint4(0, 0, 0, 0);
  }

  // ---------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace
}  // namespace rf2


namespace rf2 {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D view of a [B*Npad, heads, D] bf16 tensor; box = 64 columns x 1 head x `rows` tokens,
// 128-byte swizzle (one 128-byte row per token, 8-row swizzle atoms of 1024 bytes).
bool make_map(CUtensorMap* m, const void* base, const Geo& g, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.heads, (cuuint64_t)(g.B * g.Npad)};
  cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.heads * g.D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BLK>
cudaError_t launch_instance(const void* qp, const void* kp, const void* vp, const int32_t* idx,
                            const int32_t* cnt, int kmax, const Geo& g, float scale, void* op,
                            int32_t* status, cudaStream_t s) {
  using C = Cfg<D, BLK>;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, qp, g, kBM) || !make_map(&tk, kp, g, BLK) || !make_map(&tv, vp, g, BLK))
    return cudaErrorInvalidValue;
  auto kern = sparse_attn_kernel<D, BLK>;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid(g.Nb, g.heads, g.B);
  const float scale_log2 = scale * 1.4426950408889634f;  // log2(e)
  kern<<<grid, kThreads, C::kSmem, s>>>(tq, tk, tv, idx, cnt, kmax,
                                        reinterpret_cast<__nv_bfloat16*>(op), g, scale_log2,
                                        status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn(const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* cnt, int kmax, const Geo& g,
                               float scale, void* op, int32_t* status, cudaStream_t s) {
  if (g.D == 128 && g.blk == 128)
    return launch_instance<128, 128>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
  if (g.D == 64 && g.blk == 64)
    return launch_instance<64, 64>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
  if (g.D == 128 && g.blk == 64)
    return launch_instance<128, 64>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
  if (g.D == 64 && g.blk == 128)
    return launch_instance<64, 128>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
  return cudaErrorNotSupported;
}

}  // namespace rf2
