// mla_decode_noalloc: the decode step with its workspace in a static device array.
//
// Some callers cannot allocate device memory at decode time: a serving process whose
// memory pool is carved up once at start-up, a real-time loop that must not call the
// allocator (cudaMalloc can synchronise the device and take unbounded time), or a host
// program that drives this library through its C ABI alone and has no allocator of its
// own.  For them this entry point needs no workspace argument: it uses a fixed scratch
// array compiled into the library (kNoAllocScratchBytes on every GPU that loads the
// library, held until the process exits).  Everything else matches mla_decode.
#include <mutex>

#include "mla_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;   // 16 MiB
static_assert(kNoAllocScratchBytes == (size_t)MLA_NOALLOC_SCRATCH_BYTES, "header and library disagree");

// The scratch array.  In host code its name is only a stand-in symbol, never a device
// address: the device address is obtained per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch[kMaxDevices];   // device address of the array per device, once resolved

// The array's device address on `dev` (the current device), looked up the first time it
// succeeds and kept from then on.  A failed lookup is not remembered: the next call tries
// again, and the lookup's error is cleared so a later, unrelated status check does not
// pick it up.
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) == cudaSuccess) {
      g_scratch[dev] = p;
    } else {
      (void)cudaGetLastError();
    }
  }
  return g_scratch[dev];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" mla_status_t mla_decode_noalloc(const mla_plan_t* plan, const mla_cache_t* cache,
                                           const int32_t* seq_lens, const void* q, int32_t B, void* out,
                                           void* stream) {
  if (!plan || !cache || !seq_lens || !q || !out || B <= 0) return MLA_ERR_INVALID_ARG;
  const mla_config_t& cfg = plan->cfg;
  const mla_status_t st = mla_validate_cache(cfg, cache);   // the same checks as mla_decode
  if (st != MLA_OK) return st;
  if (B > cache->B) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || ((uintptr_t)seq_lens & 3)) return MLA_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev != plan->device) return MLA_ERR_INVALID_ARG;   // the plan's weights live on its device
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  void* scratch = scratch_address(dev);
  if (!scratch) return MLA_ERR_CUDA;

  int kernel = 1;
  const mla_status_t pk = mla_pick_decode_kernel(*plan, *cache, &kernel);
  if (pk != MLA_OK) return pk;
  const DecodeLayout L = mla_decode_layout(*plan, B, kernel);
  if (L.total > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  const cudaError_t e =
      mla_launch_decode(*plan, *cache, seq_lens, q, B, out, scratch, L, (cudaStream_t)stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
