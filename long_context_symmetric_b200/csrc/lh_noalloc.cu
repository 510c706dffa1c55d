// Allocation-free variant of lh_score_topk (no counterpart in the paper).
//
// Some callers cannot hand liblh a device workspace. Examples: code where a
// fixed arena owns every byte of device memory and may not grow, and code that
// may not call cudaMalloc at all on its hot path, because cudaMalloc can
// synchronise the device. For them lh_score_topk_noalloc keeps the top-K
// descent's scratch in a file-scope device array instead of a caller buffer.
// The caller still passes the inputs (sq) and the outputs (sel, map, slot).
#include "lh_common.cuh"

namespace lh {
namespace {

// Fixed scratch: 8 MiB per device that loads the library, held until the
// process exits. Enough for B*H*5*S int32 up to 2,097,152 (e.g. 16 heads at a
// 25,600-entry sub-sequence).
constexpr size_t kStaticScratchBytes = 8u << 20;
static __device__ __align__(256) int32_t g_select_scratch[kStaticScratchBytes / sizeof(int32_t)];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" lh_status lh_score_topk_noalloc(const lh_config* cfg, const double* sq, int32_t* sel,
                                           int32_t* map, int32_t* slot, void* stream) {
  lh_plan_t pl;
  lh_status st = lh_plan(cfg, &pl);
  if (st != LH_OK) return st;
  if (pl.ws_bytes > kStaticScratchBytes) return LH_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LH_ERR_CUDA;
  if (!g_scratch_addr[dev]) {
    // Set-up, once per device, on the first call with that device current. In
    // host code g_select_scratch names a host-side stand-in, not a device
    // address: the kernel needs the array's address on this device.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess) return LH_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  return lh_score_topk(cfg, sq, sel, map, slot, g_scratch_addr[dev], kStaticScratchBytes, stream);
}
