// lwm_blockattn_fwd_noalloc: the forward pass with its scratch memory in a
// fixed array that the library owns, for callers that cannot allocate
// device memory at call time.
//
// Who needs it: code that must not call cudaMalloc once it is running,
// for example a latency-critical serving loop where an allocation can
// synchronise the device and stall other streams, or a plain C host that
// embeds this library without any device allocator of its own. Such a
// caller still owns q, k, v, out and lse; only the scratch moves here.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes.
// Every GPU that loads the library holds it until the process exits. In
// host code its name is only a stand-in for the device symbol, so each
// device's real address is looked up once with cudaGetSymbolAddress (with
// that device current) and cached; the first call on a device does this
// set-up, so make that first call before any stream capture begins.
//
// All calls share the array and it keeps whatever the last call left in
// it. The forward writes every scratch region it reads before reading it,
// so nothing needs clearing between calls. Calls whose execution overlaps
// on the GPU (different streams, or different host threads without
// ordering between them) race on the array: serialise them.
#include <mutex>

#include "api_checks.cuh"
#include "aux_kernels.cuh"

namespace lwm {
namespace {

constexpr size_t kNoAllocScratchBytes = LWM_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once
// per device). Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess)
      return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace lwm

extern "C" {

int lwm_blockattn_fwd_noalloc(const void* q, const void* k, const void* v,
                              const int32_t* segment_ids,
                              const int32_t* positions, double theta,
                              int block_q, int block_k, int max_pos, int B,
                              int N, int H, int D, int dtype,
                              int qk_precision, int rope_layout, void* out,
                              float* lse, void* stream) {
  // the forward's own checks first: an invalid or unsupported call reports
  // that, not the size of the scratch
  const int c = lwm::check_fwd_args(q, k, v, segment_ids, positions, theta,
                                    block_q, block_k, max_pos, B, N, H, D,
                                    dtype, qk_precision, rope_layout, out,
                                    lse);
  if (c == lwm::kFwdNothingToDo) return LWM_OK;
  if (c != LWM_OK) return c;
  const size_t need = lwm_blockattn_fwd_workspace_size(
      B, N, H, D, block_q, block_k, max_pos, dtype, qk_precision);
  if (need == 0) return LWM_ERR_INVALID_ARG;
  if (need > lwm::kNoAllocScratchBytes) return LWM_ERR_WORKSPACE;
  void* scratch = lwm::scratch_on_current_device();
  if (!scratch) return LWM_ERR_CUDA;
  return lwm_blockattn_fwd(q, k, v, segment_ids, positions, theta, block_q,
                           block_k, max_pos, B, N, H, D, dtype, qk_precision,
                           rope_layout, out, lse, scratch,
                           lwm::kNoAllocScratchBytes, stream);
}

}  // extern "C"
