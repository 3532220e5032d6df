// rf2_predict_mask_noalloc: the mask prediction of rf2_predict_mask for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a framework that
// owns every device allocation (a caching allocator, an inference runtime with a fixed
// memory plan), or a plug-in loaded into a process that forbids allocation after its
// start-up phase.  They can still pass their inputs and outputs, but not the scratch
// that rf2_predict_mask takes as `ws`.  This entry point keeps that scratch in a
// file-scope device array of fixed size instead, so it allocates nothing per call.
//
// The array (kScratchBytes) exists on every GPU that loads this library, from module
// load until the process exits.  Every call on a device shares it and it keeps the last
// call's contents.  Each call first clears the one word that must start at zero (its
// status word) and writes every other byte it reads (the parts of the block means, then
// the pooled scores) before reading it.  Calls whose work
// overlaps on the GPU (on different streams, or different host threads, of the same
// device) race on the array and must be serialised by the caller.
#include <math.h>

#include <mutex>

#include "rf2_common.cuh"

namespace {

constexpr size_t kScratchBytes = RF2_NOALLOC_SCRATCH_BYTES;
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device.  In host code the name g_scratch is only a
// host-side stand-in; a kernel given it would fault, or read host memory where the GPU
// can reach it.  The address is looked up with the device current and kept together with
// the id of the context it belongs to: after a cudaDeviceReset the device gets a new
// primary context (with a new id) in which the module, and the array, are loaded anew,
// so the address is looked up again instead of reusing a stale one.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct ScratchSlot {
  unsigned long long ctx_id;  // 0: not looked up yet
  void* addr;
};
ScratchSlot g_scratch_slot[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Id of the calling thread's current context (never 0), or 0 if the driver cannot say.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id + 1;  // context ids may start at 0; 0 here means "unknown"
}

int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RF2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  // cudaFree(nullptr) is the runtime's documented way to make the device's primary
  // context current (it frees nothing), so that the id below is the context the kernels
  // of this call will run in.
  if (cudaFree(nullptr) != cudaSuccess) return RF2_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  ScratchSlot& slot = g_scratch_slot[dev];
  if (slot.addr == nullptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return RF2_ERR_CUDA;
    slot.addr = p;
    slot.ctx_id = ctx;
  }
  *out = slot.addr;
  return RF2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int rf2_predict_mask_noalloc(const void* qp, const void* kp, const rf2_geom* g,
                                        double sparsity, int sink, unsigned flags, int32_t* idx,
                                        int32_t* cnt, int kmax, void* stream) {
  // Same argument rules as rf2_predict_mask; its size query gives the scratch needed.
  const int kept = rf2_kept_count(g, sparsity, sink, flags);  // checks g and sparsity
  if (kept < 0) return -kept;
  const size_t need = rf2_workspace_size(g, sparsity, sink, flags, 0);
  if (need == 0) return RF2_ERR_INVALID_ARG;
  if (need > kScratchBytes) return RF2_ERR_WORKSPACE;  // geometry beyond the fixed maximum
  if (qp == nullptr || kp == nullptr || idx == nullptr || cnt == nullptr) return RF2_ERR_INVALID_ARG;
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(idx) || !aligned16(cnt)) return RF2_ERR_ALIGNMENT;
  if (kmax < kept) return RF2_ERR_INVALID_ARG;

  void* base = nullptr;
  int st = scratch_for_current_device(&base);
  if (st != RF2_OK) return st;
  const rf2::Geo geo = rf2::make_call_geo(*g, flags);
  // The same layout as the workspace of rf2_predict_mask: a status word, then the bf16
  // parts of the block means and the pooled scores.
  unsigned char* p = static_cast<unsigned char*>(base);
  int32_t* status = reinterpret_cast<int32_t*>(p);
  const rf2::MaskScratch m = rf2::mask_scratch_layout(geo, p + kAlign);

  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = rf2::launch_pool(qp, kp, m.q3, m.k3, geo, (flags & RF2_RASTER) != 0, s);
  if (e == cudaSuccess)
    e = rf2::launch_scores(m.q3, m.k3, m.scores, geo, (float)(1.0 / sqrt((double)geo.D)), sink ? geo.nsink : 0,
                           status, s);
  if (e == cudaSuccess)
    e = rf2::launch_topk(m.scores, idx, cnt, kmax, kept, sink ? geo.nsink : 0, geo, s);
  if (e != cudaSuccess) return RF2_ERR_CUDA;
  if (flags & RF2_CHECKED) {
    int32_t st_h = 0;
    if (cudaMemcpyAsync(&st_h, status, sizeof(st_h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return RF2_ERR_CUDA;
    return st_h;
  }
  return RF2_OK;
}
