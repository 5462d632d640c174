// combine.cu -- merges the split partials of every query row ("HPC-Ops: Tencent's CUDA
// Kernel Library for LLM Inference Hot Paths", "How the kernels are organized around
// specific workload shapes": a combine kernel merges the split-k results).
//
// Merge rule (log-sum-exp of normalised partials): for the n_b tiles of row (b, t, qh),
// M = max_i lse_i, w_i = e^{lse_i - M}, out = sum_i w_i o_i / sum_i w_i,
// lse = M + ln sum_i w_i. A tile that saw no key of the row has lse_i = -inf and weight
// 0; a row with no visible key at all gets out = 0, lse = -inf.
//
// One CTA per query row; each group of D/4 threads reads one partial row as float4s, the
// groups stride over the row's partials, and the CTA folds the group sums in shared
// memory. Rows of requests held in a single tile were written by the split kernel and
// are skipped here.
#include "common.cuh"

namespace decattn {


constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  constexpr int TPP = D / 4;                       // threads per partial row (float4 each)
  constexpr int PPB = kCombineThreads / TPP;       // partial rows in flight per pass
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
  if (hdr->magic != kPlanMagic || hdr->status != DECATTN_OK) return;  // the split kernel reports it
  const int row = blockIdx.x;
  const int b = row / (p.T * p.Hq), t = (row / p.Hq) % p.T, qh = row % p.Hq;
  const int L = p.seq_lens[b];
  const int nb = L > 0 ? (L + p.tl - 1) / p.tl : 0;
  if (nb == 1) return;
  float* orow = p.out + (int64_t)row * D;
  if (nb == 0) {
    for (int i = threadIdx.x; i < D; i += kCombineThreads) orow[i] = 0.f;
    if (threadIdx.x == 0) p.lse[row] = -INFINITY;
    return;
  }
  const int h = qh / p.G, r = t * p.G + (qh % p.G);
  const int32_t* pair_off = reinterpret_cast<const int32_t*>(p.plan + p.off_pair_off);
  const int64_t slot0 = pair_off[(int64_t)b * p.Hkv + h];
  __shared__ float red[kCombineThreads / 32];
  __shared__ float accs[PPB][D];
  __shared__ float ws[PPB];

  // pass 1: M = max lse_i
  float M = -INFINITY;
  for (int i = threadIdx.x; i < nb; i += kCombineThreads) M = fmaxf(M, p.part_lse[(slot0 + i) * p.GT + r]);
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = M;
  __syncthreads();
  M = red[0];
  #pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) M = fmaxf(M, red[w]);
  if (M == -INFINITY) {
    for (int i = threadIdx.x; i < D; i += kCombineThreads) orow[i] = 0.f;
    if (threadIdx.x == 0) p.lse[row] = -INFINITY;
    return;
  }

  // pass 2: weighted sum of the partial rows
  const int sub = threadIdx.x / TPP, q4 = threadIdx.x % TPP;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
  #pragma unroll 4
  for (int i = sub; i < nb; i += PPB) {
    const int64_t pr = (slot0 + i) * p.GT + r;
    const float li = p.part_lse[pr];
    const float4 v = reinterpret_cast<const float4*>(p.part_o + pr * D)[q4];
    const float w = li == -INFINITY ? 0.f : expf(li - M);
    acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
    W += w;
  }
  reinterpret_cast<float4*>(&accs[sub][0])[q4] = acc;
  if (q4 == 0) ws[sub] = W;
  __syncthreads();
  float Wt = 0.f;
  #pragma unroll
  for (int k = 0; k < PPB; ++k) Wt += ws[k];
  for (int i = threadIdx.x; i < D; i += kCombineThreads) {
    float s = 0.f;
    #pragma unroll
    for (int k = 0; k < PPB; ++k) s += accs[k][i];
    orow[i] = s / Wt;
  }
  if (threadIdx.x == 0) p.lse[row] = M + logf(Wt);
}

cudaError_t launch_combine(const CombineParams& p, int rows, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (p.D == 128) combine_kernel<128><<<rows, kCombineThreads, 0, st>>>(p);
  else if (p.D == 64) combine_kernel<64><<<rows, kCombineThreads, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace decattn
