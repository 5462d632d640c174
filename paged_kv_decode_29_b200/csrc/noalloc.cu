// noalloc.cu -- dec_attn_run_noalloc: split + combine with the workspace taken from a
// fixed device array owned by this library, for callers that cannot allocate device memory.
//
// Who needs it: a caller hosted inside an engine that owns all device memory through its own
// pool and gives plugins no way to allocate, or a deployment that pins its device memory
// budget up front and forbids allocation once decoding runs (an allocation can also stall the
// device at an unpredictable point of a decode step). Such a caller can still hand over its
// inputs, outputs and plan buffer, but not a workspace.
//
// How: the workspace lives in g_noalloc_scratch below, kDecattnNoallocBytes (64 MiB) per GPU.
// Host code cannot use the array's name as a device address, so the first call on each device
// (with that device current) looks the address up with cudaGetSymbolAddress and caches it;
// that first call also makes the CUDA runtime load the module holding the array, so it should
// come before any stream capture. The array stays allocated on every GPU where it was set up
// until the process exits. Nothing in it has to start at zero: the split kernel writes every
// partial the combine reads and zeroes the combine's per-row counters at the start of each run.
// All calls on a device share the one array, so calls whose work overlaps on the GPU (e.g. on
// two streams) race and corrupt each other's results; serialise them.
#include <mutex>

#include "common.cuh"
#include "host_errors.h"

namespace decattn {

constexpr size_t kDecattnNoallocBytes = size_t(64) << 20;  // keep equal to DECATTN_NOALLOC_SCRATCH_BYTES

static __device__ __align__(256) unsigned char g_noalloc_scratch[kDecattnNoallocBytes];

static_assert(kDecattnNoallocBytes == (size_t)DECATTN_NOALLOC_SCRATCH_BYTES, "scratch size mismatch");

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail("device ordinal beyond the scratch table", cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch); e != cudaSuccess || !ptr)
      return cuda_fail("scratch address (cudaGetSymbolAddress)", e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return DECATTN_OK;
}
}  // namespace

}  // namespace decattn

extern "C" int dec_attn_run_noalloc(const dec_attn_shape* shape, const void* q, const void* k_pages,
                                    const void* v_pages, const int32_t* page_table, const int32_t* seq_lens,
                                    const float* kv_scales, const dec_attn_plan_t* plan, float* out, float* lse,
                                    void* stream) {
  const size_t need = dec_attn_workspace_bytes(shape, plan);
  if (need == 0)  // invalid or unsupported arguments: dec_attn_run reports which, before any launch
    return dec_attn_run(shape, q, k_pages, v_pages, page_table, seq_lens, kv_scales, plan, nullptr, 0, out, lse,
                        stream);
  if (need > decattn::kDecattnNoallocBytes) return DECATTN_ESMALL;  // the fixed scratch cannot hold this plan
  void* scratch = nullptr;
  const int rc = decattn::noalloc_scratch(&scratch);
  if (rc != DECATTN_OK) return rc;
  return dec_attn_run(shape, q, k_pages, v_pages, page_table, seq_lens, kv_scales, plan, scratch,
                      decattn::kDecattnNoallocBytes, out, lse, stream);
}
