// moe_static_scratch.cu -- moe_dispatch_noalloc: the sender side of the dispatch for callers
// that cannot allocate device memory.
//
// moe_dispatch needs a caller-allocated workspace for the counters of its slot scan.
// Some callers have no way to allocate one: a plugin loaded into a host program that
// owns the whole device-memory budget, or code whose memory layout is frozen before
// the block's sizes are known.  This entry point keeps that scratch in a fixed array
// in the library's own device memory instead.  The array is file-scope, so every GPU
// that loads the library holds it (kStaticScratchInts int32 words, 8 MiB) until the
// process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace moe {
namespace {

// 2^21 int32 words = 8 MiB: enough for the slot scan of up to 2 million
// (chunk x (pool + expert)) counters, e.g. 65,536 tokens with 384 experts.
constexpr size_t kStaticScratchInts = size_t(1) << 21;

static __device__ __align__(256) int32_t g_dispatch_scratch[kStaticScratchInts];

// The device address of g_dispatch_scratch, per device.  In host code the array's
// name only stands in for the symbol; a kernel given it would read the wrong memory.
// The address is looked up once per device and kept for the life of the process: a
// cudaDeviceReset reloads the module and may move the array, so the library must not
// be used across a reset of a device it has already run on.
std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

moe_status_t scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index out of range for static scratch");
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(static dispatch scratch)");
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

size_t static_dispatch_scratch_ints() { return kStaticScratchInts; }

}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_dispatch_noalloc(moe_plan_t plan, const uint16_t* z, const int32_t* topk_idx,
                                             uint16_t* pools, int32_t* slot, void* stats, void* stream) {
  if (plan == nullptr) return fail(MOE_ERR_INVALID_ARG, "null plan");
  const Geo& g = plan_geo(plan);
  if (g.dropless)
    return fail(MOE_ERR_UNSUPPORTED, "moe_dispatch_noalloc: the dropless variant runs through moe_forward only");
  if (!pools || !stats) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (g.T > 0 && (!z || !topk_idx || !slot)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if ((reinterpret_cast<uintptr_t>(z) & 15) || (reinterpret_cast<uintptr_t>(pools) & 15))
    return fail(MOE_ERR_INVALID_ARG, "z and pools must be 16-byte aligned");
  const size_t need = scan_scratch_ints(g);
  if (need > kStaticScratchInts)
    return fail(MOE_ERR_UNSUPPORTED, "moe_dispatch_noalloc: this plan needs " + std::to_string(need) +
                                         " int32 words of scan scratch, the static array holds " +
                                         std::to_string(kStaticScratchInts) + "; use moe_dispatch");
  moe_status_t s = device_check();
  if (s != MOE_OK) return s;
  int32_t* scratch = nullptr;
  s = scratch_for_current_device(&scratch);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* stw = static_cast<int32_t*>(stats);
  // every scratch word the scan reads is written earlier in the same call, so the
  // array needs no clearing between calls
  s = launch_slot_scan(g, topk_idx, slot, stw, scratch, st);
  if (s != MOE_OK) return s;
  return launch_pack(g, z, topk_idx, slot, stw, pools, st);
}
