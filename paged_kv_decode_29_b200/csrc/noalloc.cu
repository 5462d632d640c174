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
// (with that device current) looks the address up with cudaGetSymbolAddress and caches it,
// together with the identity of the CUDA context it belongs to; that first call also makes the
// CUDA runtime load the module holding the array, so it should come before any stream capture.
// A cached address is only valid in its own context: after cudaDeviceReset the device gets a new
// primary context (and a new copy of the module), so a call that finds another context current
// looks the address up again instead of handing the kernels a dangling pointer. The array stays
// allocated on every GPU where it was set up until the process (or a device reset) ends it.
// Nothing in it has to start at zero: the split kernel writes every partial the combine reads
// and zeroes the combine's per-row counters at the start of each run.
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
struct ScratchEntry {
  void* ptr;             // device address of g_noalloc_scratch in context `ctx_id`
  unsigned long long ctx_id;
};
ScratchEntry g_noalloc[kMaxDevices] = {};

// Identity of the current CUDA context (cuCtxGetCurrent + cuCtxGetId, fetched through the
// runtime so that the library needs no libcuda link). 0 when the driver cannot say, in which
// case the address is looked up on every call.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool tried = false;
  if (!tried) {  // called with g_noalloc_mu held
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  }
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device, looked up once per (device,
// context) and again whenever the current context is not the one it was looked up in.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail("device ordinal beyond the scratch table", cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  const unsigned long long ctx = current_ctx_id();  // 0 also before the runtime's first call made one
  ScratchEntry& ent = g_noalloc[dev];
  if (!ent.ptr || ctx == 0 || ent.ctx_id != ctx) {
    void* ptr = nullptr;
    if (const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch); e != cudaSuccess || !ptr)
      return cuda_fail("scratch address (cudaGetSymbolAddress)", e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    ent.ptr = ptr;
    ent.ctx_id = current_ctx_id();  // the lookup has made the device's primary context current
  }
  *out = ent.ptr;
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
