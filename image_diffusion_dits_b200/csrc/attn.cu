// Block-sparse flash attention over the kept key blocks, sm_100a (tcgen05 + TMEM + TMA).
//
// RainFusion2.0 (mlsanity index page: title "block-wise sparse attention"; Abstract:
// skipping the computation of insignificant tokens).  For query block i of (b, head):
//   O_i = softmax(Q_i K_S^T * scale + M) V_S,   S = kept key blocks of the row,
//   M = -inf on pad keys (partial windows at the high end of an axis).
//
// One CTA per (query block, head, batch); query tile of 128 rows (a 64-token block uses
// the first 64).  The kept blocks of the row are split into two streams, even and odd
// positions of the list; each stream has its own softmax warpgroup, running max, row
// sum, S/P buffer and O accumulator in TMEM, and the two partial results are merged in
// the epilogue (softmax over the union = the two partial softmaxes rescaled to a common
// max).  The streams run concurrently, so one warpgroup's TMEM round trips and
// exponentials overlap the other's, and the tensor core always has a tile of one
// stream to work on while the other stream's softmax runs.
// Warp roles (352 threads):
//   warps 0-3  softmax of stream 0, warps 4-7 softmax of stream 1: thread r owns query
//              row r = TMEM lane r.  Reads the S row in one TMEM load, online softmax in
//              the exp2 domain (fp32 max, sum, arguments and exp2), writes P (bf16 pairs)
//              over the S columns, rescales its O when its running max grows by more than
//              2^8.
//   warp 8     TMA producer of Q (once) and of K_j for each kept block j (3-stage ring).
//   warp 9     MMA issuer: S_i = Q K_i^T (SS, K-major) into the S/P buffer of stream i%2,
//              O_{i%2} += P_i V_i (P from TMEM, V MN-major from shared memory), then
//              S_{i+2} into the same buffer right behind it (MMAs execute in issue order).
//   warp 10    TMA producer of V_j (2-stage ring).
// TMEM: S/P buffers at columns 0 and 128, O accumulators at 256 and 384 (512 columns).
// Every mbarrier wait is bounded in time; on expiry the CTA raises a timeout status,
// stops issuing work, drains what it issued and returns.
#include <cuda.h>

#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace rf2 {
namespace {

constexpr int kBM = 128;            // query rows per tile (TMEM lanes)
constexpr int kSoftmaxWarps = 8;    // two warpgroups, one per stream
constexpr int kThreads = 352;       // 8 softmax warps + K producer + MMA + V producer
constexpr int kProducerWarp = 8;    // Q and K loads
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;  // V loads
constexpr int kKStages = 3;         // K ring depth
constexpr int kVStages = 2;         // V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;    // O of stream s at kTmemO + 128*s; S/P of stream s at 128*s
constexpr uint64_t kWaitLimitNs = 500ull * 1000ull * 1000ull;  // 0.5 s per wait

template <int D, int BLK>
struct Cfg {
  static constexpr int kAtomsD = D / 64;       // 128-byte column atoms of a [rows, D] tile
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = BLK * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffList = kOffV + kVStages * kKVBytes;  // int32[1024] kept list
  static constexpr int kOffExt = kOffList + 4096;        // int32[1024] real extent per entry
  static constexpr int kOffXch = kOffExt + 4096;         // float[2 stream][2 (m,l)][128]
  static constexpr int kOffBar = kOffXch + 2048;         // mbarriers
  static constexpr int kOffMisc = kOffBar + 256;         // tmem slot, counts, flags
  static constexpr int kUsed = kOffMisc + 64;
  // Requested dynamic smem: 1 KB alignment slack; at least 116 KB so that at most one
  // CTA is resident per SM (each CTA allocates all 512 TMEM columns).
  static constexpr int kSmem = (kUsed + 1024) > 118784 ? (kUsed + 1024) : 118784;
};

// Barrier slots (8 bytes each) at kOffBar.
enum : int {
  BAR_Q = 0,
  BAR_KFULL = 1,    // +stage (3)
  BAR_KEMPTY = 4,   // +stage (3)
  BAR_VFULL = 7,    // +stage (2)
  BAR_VEMPTY = 9,   // +stage (2)
  BAR_SFULL = 11,   // +stream (2): S_i of the stream computed
  BAR_PFULL = 13,   // +stream (2): P_i of the stream written to TMEM
  BAR_DONE = 15,    // every MMA of the CTA completed
  BAR_XCH = 16,     // both warpgroups posted their (max, sum)
  BAR_COUNT = 17
};

struct Misc {
  uint32_t tmem_base;
  int n;       // kept blocks after dropping out-of-range ids
  int abort;   // set by any role that gave up on a wait
  int pad;
};

// Row r of query block i as a model-order token of batch b (RASTER), or -1 for a pad row.
__device__ __forceinline__ long long window_row_token(const Geo& g, int i, int r) {
  const int per_t = g.nbh * g.nbw;
  const int tb = i / per_t, hb = (i - tb * per_t) / g.nbw, wb = i - tb * per_t - hb * g.nbw;
  const int whw = g.wh * g.ww;
  const int dt = r / whw, dh = (r - dt * whw) / g.ww, dw = r - dt * whw - dh * g.ww;
  const int t = tb * g.wt + dt, h = hb * g.wh + dh, w = wb * g.ww + dw;
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return ((long long)t * g.H + h) * g.W + w;
}

// RASTER: Q/K/V and O in model order [B, N, heads, D]: each window is one 5-D TMA box
// (64 columns x 1 head x ww x wh x wt tokens; tokens past the grid arrive as zeros, the
// same rows the window-order layout holds as zero pads) and O rows are written to their
// tokens.  Otherwise window order [B, Npad, heads, D] through 3-D boxes.  The shared-
// memory tiles are byte for byte the same in both layouts.
template <int D, int BLK, bool RASTER>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const int32_t* __restrict__ idx,
                       const int32_t* __restrict__ cnt, int kmax,
                       __nv_bfloat16* __restrict__ op, Geo g, float scale_log2,
                       int* __restrict__ status, int b_base) {
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
  const int b = b_base + (int)blockIdx.z;
  const long long row = ((long long)b * g.heads + head) * g.Nb + qblk;
  const long long brow0 = (long long)b * g.Npad;  // first row of batch b in the 3-D maps
  // TMA box of block j: window-order rows (3-D) or window coordinates (5-D, per batch)
  auto load_block = [&](uint32_t dst, const CUtensorMap* map, uint32_t barrier, int j, int rows) {
#pragma unroll
    for (int a = 0; a < D / 64; ++a) {
      if constexpr (RASTER) {
        const int per_t = g.nbh * g.nbw;
        const int tb = j / per_t, hb = (j - tb * per_t) / g.nbw, wb = j - tb * per_t - hb * g.nbw;
        ptx::tma_load_5d(dst + a * (rows * 128), map, barrier, a * 64, head, wb * g.ww, hb * g.wh, tb * g.wt);
      } else {
        ptx::tma_load_3d(dst + a * (rows * 128), map, barrier, a * 64, head, (int)(brow0 + (long long)j * BLK));
      }
    }
  };

  // ---------------------------------------------------------------- setup
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
  int* ext_s = reinterpret_cast<int*>(smem + C::kOffExt);
  if (warp == kProducerWarp) {
    // Compact the kept list into shared memory, dropping ids outside [0, Nb); with each
    // kept block store its real extent (nt | nh << 8 | nw << 16) for the pad-key mask.
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
      if (ok) {
        int nt, nh, nw;
        block_extent(g, j, nt, nh, nw);
        const int pos = n_out + __popc(m & ((1u << lane) - 1u));
        list_s[pos] = j;
        ext_s[pos] = nt | (nh << 8) | (nw << 16);
      }
      n_out += __popc(m);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && status != nullptr)
      atomicCAS(status, 0, kStatusBadIndex);
    if (lane == 0) misc->n = n_out;
  }
  if constexpr (RASTER && BLK < kBM) {
    // A window box fills BLK of the kBM Q rows; clear the rest once so that the unused
    // S rows are finite (their outputs are never written).
    for (int e = tid; e < C::kAtomsD * (kBM - BLK) * 8; e += kThreads) {
      const int a = e / ((kBM - BLK) * 8), rem = e - a * (kBM - BLK) * 8;
      reinterpret_cast<uint4*>(smem + C::kOffQ + a * (kBM * 128) + BLK * 128)[rem] = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int n = misc->n;

  if (n > 0) {
    if (warp == kProducerWarp && lane == 0) {
      // ------------------------------------------------------------ TMA producer: Q, K
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tk);
      // Q tile: kBM rows per atom in shared memory; a window-order box covers all kBM
      // rows (past a 64-token block: the next block's rows, never used), a window box BLK.
      ptx::mbar_arrive_expect_tx(bar(BAR_Q), RASTER ? C::kAtomsD * BLK * 128 : C::kQBytes);
      if constexpr (RASTER) {
        load_block(sQ, &tq, bar(BAR_Q), qblk, kBM);
      } else {
#pragma unroll
        for (int a = 0; a < C::kAtomsD; ++a)
          ptx::tma_load_3d(sQ + a * (kBM * 128), &tq, bar(BAR_Q), a * 64, head,
                           (int)(brow0 + (long long)qblk * BLK));
      }
      int issued[kKStages];
#pragma unroll
      for (int s = 0; s < kKStages; ++s) issued[s] = -1;
      for (int i = 0; i < n; ++i) {
        const int s = i % kKStages;
        if (i >= kKStages && !ptx::mbar_wait(bar(BAR_KEMPTY + s), ((i / kKStages) - 1) & 1, abort_flag,
                                             status, kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_KFULL + s), C::kKVBytes);
        load_block(sK + s * C::kKVBytes, &tk, bar(BAR_KFULL + s), list_s[i], BLK);
        issued[s] = i;
      }
      if (*abort_flag) {
        // Let every copy this thread issued land before the CTA can exit.
        ptx::mbar_wait(bar(BAR_Q), 0, nullptr, nullptr, kWaitLimitNs, 0);
        for (int s = 0; s < kKStages; ++s)
          if (issued[s] >= 0)
            ptx::mbar_wait(bar(BAR_KFULL + s), (issued[s] / kKStages) & 1, nullptr, nullptr,
                           kWaitLimitNs, 0);
      }
    } else if (warp == kVProducerWarp && lane == 0) {
      // ------------------------------------------------------------ TMA producer: V
      ptx::prefetch_tmap(&tv);
      int issued[kVStages];
#pragma unroll
      for (int s = 0; s < kVStages; ++s) issued[s] = -1;
      for (int i = 0; i < n; ++i) {
        const int s = i % kVStages;
        if (i >= kVStages && !ptx::mbar_wait(bar(BAR_VEMPTY + s), ((i / kVStages) - 1) & 1, abort_flag,
                                             status, kWaitLimitNs, kStatusTimeout))
          break;
        ptx::mbar_arrive_expect_tx(bar(BAR_VFULL + s), C::kKVBytes);
        load_block(sV + s * C::kKVBytes, &tv, bar(BAR_VFULL + s), list_s[i], BLK);
        issued[s] = i;
      }
      if (*abort_flag) {
        for (int s = 0; s < kVStages; ++s)
          if (issued[s] >= 0)
            ptx::mbar_wait(bar(BAR_VFULL + s), (issued[s] / kVStages) & 1, nullptr, nullptr,
                           kWaitLimitNs, 0);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, BLK, 0);
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, D, 1);
      bool ok = ptx::mbar_wait(bar(BAR_Q), 0, abort_flag, status, kWaitLimitNs, kStatusTimeout);
      ptx::tc_fence_after();
      // Shared-memory descriptors of the tile bases; every MMA step only adds a constant
      // to the start-address field (tiles stay inside the 14-bit address range).
      const uint64_t qdesc = ptx::smem_desc_sw128(sQ, 16, 1024);
      const uint64_t kdesc0 = ptx::smem_desc_sw128(sK, 16, 1024);
      const uint64_t vdesc0 = ptx::smem_desc_sw128(sV, BLK * 128, 1024);
      // S_i into the S/P buffer of stream i%2.  For i >= 2 that buffer holds P_{i-2}, which
      // P_{i-2} V_{i-2} reads; that MMA was issued before this one by this thread, and
      // tcgen05 MMAs issued by one thread execute in issue order, so S_i is issued
      // without waiting for it to complete (no drain of the tensor pipe per block).
      auto wait_s = [&](int i) -> bool {
        return ptx::mbar_wait(bar(BAR_KFULL + i % kKStages), (i / kKStages) & 1, abort_flag, status,
                              kWaitLimitNs, kStatusTimeout);
      };
      auto issue_s = [&](int i) {
        const int ks = i % kKStages;
        const int st = i & 1;
        const uint64_t kdesc = kdesc0 + (uint64_t)((ks * C::kKVBytes) >> 4);
        const uint32_t dS = tmem + (uint32_t)(128 * st);
        if constexpr (D == 128) {
          // step kk: atom kk/4, 16 columns = 32 bytes inside it (start address field >> 4)
          constexpr uint32_t QA = kBM * 128 / 16, KA = BLK * 128 / 16;
          ptx::mma8_ss<2, 4, 6, QA, QA + 2, QA + 4, QA + 6, 2, 4, 6, KA, KA + 2, KA + 4, KA + 6>(
              dS, qdesc, kdesc, idesc_s, 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = qdesc + (uint64_t)(((kk >> 2) * (kBM * 128) + (kk & 3) * 32) >> 4);
            const uint64_t bd = kdesc + (uint64_t)(((kk >> 2) * (BLK * 128) + (kk & 3) * 32) >> 4);
            ptx::mma_f16_ss(dS, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        ptx::mma_commit(bar(BAR_SFULL + st));
        ptx::mma_commit(bar(BAR_KEMPTY + ks));
      };
      // O_{i%2} += P_i V_i, P_i read from TMEM.
      auto wait_pv = [&](int i) -> bool {
        return ptx::mbar_wait(bar(BAR_PFULL + (i & 1)), (i >> 1) & 1, abort_flag, status,
                              kWaitLimitNs, kStatusTimeout) &&
               ptx::mbar_wait(bar(BAR_VFULL + i % kVStages), (i / kVStages) & 1, abort_flag, status,
                              kWaitLimitNs, kStatusTimeout);
      };
      auto issue_pv = [&](int i) {
        const int vs = i % kVStages;
        const int st = i & 1;
        const uint64_t vdesc = vdesc0 + (uint64_t)((vs * C::kKVBytes) >> 4);
        const uint32_t pt = tmem + (uint32_t)(128 * st);
        const uint32_t dO = tmem + kTmemO + (uint32_t)(128 * st);
        if constexpr (BLK == 128) {
          // A = P [128 x BLK] in TMEM: 16 keys = 8 columns of bf16 pairs.
          // B = V [BLK keys x D] read as N x K MN-major: 16 keys = 16 rows of 128 bytes;
          // the D atoms (64 columns each) are BLK*128 bytes apart.
          ptx::mma8_ts<8, 16, 24, 32, 40, 48, 56, 16 * 128 / 16>(dO, pt, vdesc, idesc_o,
                                                                  i >= 2 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk) {
            const uint64_t bd = vdesc + (uint64_t)((kk * (16 * 128)) >> 4);
            ptx::mma_f16_ts(dO, pt + kk * 8, bd, idesc_o, (i >= 2 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::mma_commit(bar(BAR_VEMPTY + vs));
      };
      for (int i = 0; ok && i < n && i < 2; ++i) {
        ok = wait_s(i);
        if (ok) {
          ptx::tc_fence_after();
          issue_s(i);
        }
      }
      // Streams alternate: P_i V_i, then S_{i+2}.  All three inputs are awaited before
      // either group is issued, so the two groups go to the tensor pipe back to back.
      // The waits suspend the thread (try_wait), so the MMA warp takes no issue slots
      // from the softmax warps that share its sub-partition while it waits.  (Two
      // issuing threads, one per stream, measured slower: the interleaved chains.)
      for (int i = 0; ok && i < n; ++i) {
        ok = wait_pv(i) && (i + 2 >= n || wait_s(i + 2));
        if (!ok) break;
        ptx::tc_fence_after();
        issue_pv(i);
        if (i + 2 < n) issue_s(i + 2);
      }
      // All MMAs this thread issued have completed once BAR_DONE fires.
      ptx::mma_commit(bar(BAR_DONE));
      ptx::mbar_wait(bar(BAR_DONE), 0, nullptr, nullptr, kWaitLimitNs, 0);
    } else if (warp < kSoftmaxWarps) {
      // ------------------------------------------------------------ softmax + epilogue
      const int st = warp >> 2;       // stream: kept-list positions st, st+2, st+4, ...
      const int r = tid & (kBM - 1);  // query row == TMEM lane
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t srow = tmem + lane_base + (uint32_t)(128 * st);
      const uint32_t orow_t = tmem + lane_base + kTmemO + (uint32_t)(128 * st);
      // (dt | dh << 8 | dw << 16) of the columns q*32 + lane this lane evaluates for the
      // pad-key masks
      int cpk[BLK / 32];
#pragma unroll
      for (int q = 0; q < BLK / 32; ++q) {
        const int c = q * 32 + lane;
        const int whw = g.wh * g.ww;
        const int dt = c / whw;
        const int dh = (c - dt * whw) / g.ww;
        const int dw = c - dt * whw - dh * g.ww;
        cpk[q] = dt | (dh << 8) | (dw << 16);
      }
      const int full_ext = g.wt | (g.wh << 8) | (g.ww << 16);
      float m_run = -INFINITY;
      float l_run = 0.f;
      bool ok = true;
      for (int i = st; i < n; i += 2) {
        const int t = i >> 1;  // position within the stream
        // Waits are per thread; giving up is decided for the whole warp so that the
        // warp-wide tcgen05 and shuffle operations below stay converged.
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_SFULL + st), t & 1, abort_flag, status,
                                                     kWaitLimitNs, kStatusTimeout))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float x[BLK];
        {
          // the whole S row in one TMEM load (one round trip)
          uint32_t tt[BLK];
          if constexpr (BLK == 128)
            ptx::tmem_ld32x128(srow, tt);
          else
            ptx::tmem_ld32x64(srow, tt);
#pragma unroll
          for (int c = 0; c < BLK; ++c) x[c] = __uint_as_float(tt[c]);
        }
        // Pad keys of a partial window get -inf; validity is per column, the same for
        // every row, so each lane evaluates 1/32 of the columns and the warp shares bits.
        const int ext = ext_s[i];
        if (ext != full_ext) {
          const int nt = ext & 255, nh = (ext >> 8) & 255, nw = ext >> 16;
          uint32_t vm[BLK / 32];
#pragma unroll
          for (int q = 0; q < BLK / 32; ++q)
            vm[q] = __ballot_sync(0xffffffffu, (cpk[q] & 255) < nt && ((cpk[q] >> 8) & 255) < nh &&
                                                   (cpk[q] >> 16) < nw);
#pragma unroll
          for (int c = 0; c < BLK; ++c)
            if (!((vm[c >> 5] >> (c & 31)) & 1u)) x[c] = -INFINITY;
        }
        // Row max of the raw scores (scale > 0 commutes with max): 8 independent chains
        // of three-input max instructions.
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = x[e];
#pragma unroll
        for (int c = 8; c + 8 < BLK; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = ptx::fmax3(mx8[e], x[c + e], x[c + 8 + e]);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[BLK - 8 + e]);
        const float mx = ptx::fmax3(ptx::fmax3(mx8[0], mx8[1], mx8[2]), ptx::fmax3(mx8[3], mx8[4], mx8[5]),
                                    fmaxf(mx8[6], mx8[7]));
        // Running max in exp2 units: only moved when it grows by more than 8, so P <= 2^8
        // and O needs rescaling rarely; the final O / l is unchanged by this.
        const float m_new = fmaxf(m_run, mx * scale_log2);
        const bool grow = m_new > m_run + 8.0f;  // always true on the stream's first block
        float alpha = 1.0f;
        if (grow) {
          alpha = ptx::ex2(m_run - m_new);  // 0 on the first block
          l_run *= alpha;
          m_run = m_new;
        }
        if (t >= 1 && __any_sync(0xffffffffu, grow)) {
          // This stream's O is stable: its previous P V was issued before S_i, and the
          // commit that signalled S_i covers every earlier MMA; its next P V needs P_i.
          // tcgen05.ld/st are warp-wide: the warp rescales its 32 rows together, rows
          // that did not grow with alpha = 1.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t tt[32];
            ptx::tmem_ld32(orow_t + c * 32, tt);
#pragma unroll
            for (int e = 0; e < 32; ++e) tt[e] = __float_as_uint(__uint_as_float(tt[e]) * alpha);
            ptx::tmem_st32(orow_t + c * 32, tt);
          }
        }
        // P = exp2(s * scale_log2 - m_run), rounded to bf16 pairs and written over the
        // first BLK/2 columns of this stream's S buffer (the A operand of P V); the row
        // sum uses four packed partial sums.
        const float neg_m = -m_run;
        const uint64_t sc2 = ptx::f2(scale_log2, scale_log2), nm2 = ptx::f2(neg_m, neg_m);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial row sums
        uint32_t pk[BLK / 2];
#pragma unroll
        for (int c2 = 0; c2 < BLK / 2; ++c2) {
          // arguments of a pair in one packed FFMA (fp32), then exp2 of each in fp32 on
          // the exp2 unit (measured: the packed f16 form costs the exp2 unit the same time
          // per element and needs three conversions per pair on top)
          float a0, a1;
          ptx::f2split(ptx::ffma2(ptx::f2(x[2 * c2], x[2 * c2 + 1]), sc2, nm2), a0, a1);
          const float p0 = ptx::ex2(a0), p1 = ptx::ex2(a1);
          ls2[c2 & 3] = ptx::fadd2(ls2[c2 & 3], ptx::f2(p0, p1));
          pk[c2] = ptx::pack_bf16(p0, p1);
        }
        if constexpr (BLK == 128)
          ptx::tmem_st32x64(srow, pk);
        else
          ptx::tmem_st32(srow, pk);
        ptx::tmem_wait_st();
        {
          float s0, s1;
          ptx::f2split(ptx::fadd2(ptx::fadd2(ls2[0], ls2[1]), ptx::fadd2(ls2[2], ls2[3])), s0, s1);
          l_run += s0 + s1;
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(BAR_PFULL + st));
      }
      // ---------------------------------------------------------- epilogue
      // Merge the two streams: m = max(m_0, m_1), f_s = 2^(m_s - m),
      // O = (f_0 O_0 + f_1 O_1) / (f_0 l_0 + f_1 l_1).  A stream with no block has
      // l_s = 0 and m_s = -inf (f_s = 0) and its O_s is never read.  Warpgroup s writes
      // output columns [s*D/2, (s+1)*D/2).
      float* xch = reinterpret_cast<float*>(smem + C::kOffXch);  // [stream][m, l][128]
      xch[(st * 2 + 0) * 128 + r] = m_run;
      xch[(st * 2 + 1) * 128 + r] = l_run;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(BAR_XCH));
      ok = ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_XCH), 0, abort_flag, status,
                                                        kWaitLimitNs, kStatusTimeout));
      // BAR_DONE fires once every MMA of the CTA has completed.
      if (ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(BAR_DONE), 0, abort_flag, status,
                                                       kWaitLimitNs, kStatusTimeout))) {
        ptx::tc_fence_after();
        const float m0 = xch[0 * 128 + r], l0 = xch[1 * 128 + r];
        const float m1 = xch[2 * 128 + r], l1 = xch[3 * 128 + r];
        const float m = fmaxf(m0, m1);
        const float f0 = l0 > 0.f ? ptx::ex2(m0 - m) : 0.f;
        const float f1 = l1 > 0.f ? ptx::ex2(m1 - m) : 0.f;
        const float den = f0 * l0 + f1 * l1;
        const float inv = den > 0.f ? 1.0f / den : 0.f;
        const float w0 = f0 * inv, w1 = f1 * inv;
        const bool use1 = n > 1;  // stream 1 holds at least one block
        long long orow_idx;  // output row of query row r (negative: a pad row, not written)
        if constexpr (RASTER) {
          const long long n_tok = r < BLK ? window_row_token(g, qblk, r) : -1;
          orow_idx = n_tok < 0 ? -1 : (long long)b * g.N + n_tok;
        } else {
          orow_idx = r < BLK ? brow0 + (long long)qblk * BLK + r : -1;
        }
        __nv_bfloat16* orow = op + (orow_idx * g.heads + head) * (long long)D + st * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t col = (uint32_t)(st * (D / 2) + c * 32);
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
  } else if (warp < 4 && tid < BLK) {
    // No kept block: the row attends to nothing; write zeros.
    long long orow_idx;
    if constexpr (RASTER) {
      const long long n_tok = window_row_token(g, qblk, tid);
      orow_idx = n_tok < 0 ? -1 : (long long)b * g.N + n_tok;
    } else {
      orow_idx = brow0 + (long long)qblk * BLK + tid;
    }
    if (orow_idx >= 0) {
      __nv_bfloat16* orow = op + (orow_idx * g.heads + head) * (long long)D;
      for (int v = 0; v < D / 8; ++v) reinterpret_cast<uint4*>(orow)[v] = make_uint4(0, 0, 0, 0);
    }
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

EncodeTiledFn tensor_map_encoder() {
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

namespace {

// 3-D view of a [B*Npad, heads, D] bf16 tensor; box = 64 columns x 1 head x `rows` tokens,
// 128-byte swizzle (one 128-byte row per token, 8-row swizzle atoms of 1024 bytes).
bool make_map(CUtensorMap* m, const void* base, const Geo& g, int rows) {
  EncodeTiledFn fn = tensor_map_encoder();
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

// 5-D view of one batch of a [B, N, heads, D] bf16 tensor in model order: dims (D, heads,
// W, H, T); box = 64 columns x 1 head x one (ww, wh, wt) window, 128-byte swizzle.  Box
// parts past W, H or T are zero filled.
bool make_window_map(CUtensorMap* m, const void* base, const Geo& g) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)g.heads * g.D * 2;  // bytes per token
  cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.heads, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
  cuuint64_t strides[4] = {(cuuint64_t)g.D * 2, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)g.ww, (cuuint32_t)g.wh, (cuuint32_t)g.wt};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BLK, bool RASTER>
cudaError_t launch_instance(const void* qp, const void* kp, const void* vp, const int32_t* idx,
                            const int32_t* cnt, int kmax, const Geo& g, float scale, void* op,
                            int32_t* status, cudaStream_t s) {
  using C = Cfg<D, BLK>;
  auto kern = sparse_attn_kernel<D, BLK, RASTER>;
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const float scale_log2 = scale * 1.4426950408889634f;  // log2(e)
  if constexpr (RASTER) {
    // one launch per batch: the 5-D maps address one batch's tokens
    const size_t bstride = (size_t)g.N * g.heads * g.D * 2;
    for (int b = 0; b < g.B; ++b) {
      CUtensorMap tq, tk, tv;
      if (!make_window_map(&tq, (const char*)qp + b * bstride, g) ||
          !make_window_map(&tk, (const char*)kp + b * bstride, g) ||
          !make_window_map(&tv, (const char*)vp + b * bstride, g))
        return cudaErrorInvalidValue;
      dim3 grid(g.Nb, g.heads, 1);
      kern<<<grid, kThreads, C::kSmem, s>>>(tq, tk, tv, idx, cnt, kmax, reinterpret_cast<__nv_bfloat16*>(op), g,
                                            scale_log2, status, b);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  } else {
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, qp, g, kBM) || !make_map(&tk, kp, g, BLK) || !make_map(&tv, vp, g, BLK))
      return cudaErrorInvalidValue;
    dim3 grid(g.Nb, g.heads, g.B);
    kern<<<grid, kThreads, C::kSmem, s>>>(tq, tk, tv, idx, cnt, kmax, reinterpret_cast<__nv_bfloat16*>(op), g,
                                          scale_log2, status, 0);
    return cudaGetLastError();
  }
}

template <int D, int BLK>
cudaError_t launch_layout(const void* qp, const void* kp, const void* vp, const int32_t* idx, const int32_t* cnt,
                          int kmax, const Geo& g, float scale, void* op, int32_t* status, bool raster,
                          cudaStream_t s) {
  if (raster) return launch_instance<D, BLK, true>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
  return launch_instance<D, BLK, false>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, s);
}

}  // namespace

cudaError_t launch_sparse_attn(const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* cnt, int kmax, const Geo& g,
                               float scale, void* op, int32_t* status, bool raster, cudaStream_t s) {
  if (g.D == 128 && g.blk == 128)
    return launch_layout<128, 128>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, raster, s);
  if (g.D == 64 && g.blk == 64)
    return launch_layout<64, 64>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, raster, s);
  if (g.D == 128 && g.blk == 64)
    return launch_layout<128, 64>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, raster, s);
  if (g.D == 64 && g.blk == 128)
    return launch_layout<64, 128>(qp, kp, vp, idx, cnt, kmax, g, scale, op, status, raster, s);
  return cudaErrorNotSupported;
}

}  // namespace rf2
