// host_errors.h -- host-side record of the CUDA error behind a DECATTN_ECUDA result
// (dec_attn_last_error). Included by the host code of the C ABI entry points only.
#pragma once
#include <cuda_runtime.h>

namespace decattn {

// Records the failing step `what` and the CUDA error for dec_attn_last_error (per host thread) and
// returns DECATTN_ECUDA. e == cudaSuccess takes the runtime's last error (for a helper that returned
// false right after the failing call).
int cuda_fail(const char* what, cudaError_t e = cudaSuccess);  // api.cu

}  // namespace decattn
