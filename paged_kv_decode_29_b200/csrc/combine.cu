// combine.cu -- merges the split partials of every query row ("HPC-Ops: Tencent's CUDA
// Kernel Library for LLM Inference Hot Paths", "How the kernels are organized around
// specific workload shapes": a combine kernel merges the split-k results).
//
// Merge rule (log-sum-exp of normalised partials): for the n_b tiles of row (b, t, qh),
// M = max_i lse_i, w_i = e^{lse_i - M}, out = sum_i w_i o_i / sum_i w_i,
// lse = M + ln sum_i w_i. A tile that saw no key of the row has lse_i = -inf and weight
// 0; a row with no visible key at all gets out = 0, lse = -inf.
//
// Work decomposition (computed by the planner): each query row of request b is cut into
// cb_b chunks of up to kCombineChunk tiles; the items (b, row, chunk) are numbered request
// by request. The kernel is persistent: every warp takes items w, w + #warps, ...
//  * a warp loads the lse and the D floats of up to 16 partial rows at once (16 loads in
//    flight per lane) and folds them into (max, weight, weighted sum);
//  * a row made of one chunk is finished right there;
//  * otherwise the warp publishes its chunk state and bumps the row's counter; the warp
//    that brings the counter to cb_b merges the row's chunk states (8 at once, with an
//    online rescale between groups) and writes the row.
// Rows of requests held in a single tile were written by the split kernel (cb_b = 0).
#include <type_traits>

#include "common.cuh"

namespace decattn {

constexpr int kCombineThreads = 128;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineCtasPerSm = 4;
constexpr int kCombineSmemRequests = 4096;  // per-request arrays are copied to shared memory up to this batch
constexpr int kMergeGroup = 8;              // chunk states loaded at once by the merging warp

template <int D>
struct CombineVec {
  static constexpr int VEC = D / 32;  // floats per lane
  using T = typename std::conditional<VEC == 4, float4, float2>::type;
};

template <int D>
__device__ __forceinline__ void write_row(float* orow, float* lse_out, int lane, float M, float W,
                                          const float (&acc)[D / 32]) {
  constexpr int VEC = D / 32;
  using V = typename CombineVec<D>::T;
  V v;
  float* f = reinterpret_cast<float*>(&v);
  const bool empty = M == -INFINITY || !(W > 0.f);
  const float inv = empty ? 0.f : 1.f / W;
  #pragma unroll
  for (int e = 0; e < VEC; ++e) f[e] = acc[e] * inv;
  reinterpret_cast<V*>(orow)[lane] = v;
  if (lane == 0) *lse_out = empty ? -INFINITY : M + logf(W);
}

template <int D>
__global__ void __launch_bounds__(kCombineThreads, kCombineCtasPerSm) combine_kernel(const CombineParams p) {
  constexpr int VEC = D / 32;
  using V = typename CombineVec<D>::T;
  extern __shared__ int32_t req_sm[];  // [3][B + 1]: chunk prefix, tile prefix S, seq_lens
  // The plan is complete when this grid starts (the split kernel lets it launch only after its
  // own wait on the planner), so everything but the partials is read before waiting.
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
  if (hdr->magic != kPlanMagic || hdr->status != DECATTN_OK) return;  // the split kernel reports it
  const int32_t* cb_sm = plan_arr(p.plan, hdr->off_cb);
  const int32_t* S = plan_arr(p.plan, hdr->off_S);
  const int32_t* Ls = p.seq_lens;
  if (p.B <= kCombineSmemRequests) {
    int32_t* a = req_sm;
    int32_t* b = req_sm + (p.B + 1);
    int32_t* c = req_sm + 2 * (p.B + 1);
    for (int i = threadIdx.x; i <= p.B; i += kCombineThreads) {
      a[i] = cb_sm[i];
      b[i] = S[i];
      c[i] = i < p.B ? Ls[i] : 0;
    }
    __syncthreads();
    cb_sm = a; S = b; Ls = c;
  }
  griddep_wait();  // the split kernel's partials are complete and visible
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows_per_b = (int64_t)p.T * p.Hq;
  const int64_t total = rows_per_b * cb_sm[p.B];
  const int64_t nwarps = (int64_t)gridDim.x * kCombineWarps;

  for (int64_t w = (int64_t)blockIdx.x * kCombineWarps + warp; w < total; w += nwarps) {
    int lo = 0, hi = p.B - 1;  // request: last b with rows_per_b * cb[b] <= w
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (rows_per_b * cb_sm[mid] <= w) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int ncb = cb_sm[b + 1] - cb_sm[b];
    const int64_t local = w - rows_per_b * cb_sm[b];
    const int row_in_b = (int)(local / ncb), j = (int)(local - (int64_t)row_in_b * ncb);
    const int t = row_in_b / p.Hq, qh = row_in_b - t * p.Hq;
    const int64_t row = ((int64_t)b * p.T + t) * p.Hq + qh;
    float* orow = p.out + row * D;
    const int L = Ls[b];
    const int nb = L > 0 ? (L + p.tl - 1) / p.tl : 0;
    float acc[VEC];
    #pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    if (nb == 0) {  // no key at all
      write_row<D>(orow, p.lse + row, lane, -INFINITY, 0.f, acc);
      continue;
    }
    const int h = qh / p.G, r = t * p.G + (qh - h * p.G);
    const int nbs = S[b + 1] - S[b];  // == nb
    const int64_t slot0 = (int64_t)p.Hkv * S[b] + (int64_t)h * nbs + (int64_t)j * kCombineChunk;
    const int n = min(kCombineChunk, nb - j * kCombineChunk);
    // ---- fold up to kCombineChunk partial rows
    const float my_lse = lane < n ? p.part_lse[(slot0 + lane) * p.GT + r] : -INFINITY;
    V v[kCombineChunk];
    #pragma unroll
    for (int i = 0; i < kCombineChunk; ++i)
      if (i < n) v[i] = reinterpret_cast<const V*>(p.part_o + ((slot0 + i) * p.GT + r) * D)[lane];
    float M = my_lse;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float my_w = (lane < n && M != -INFINITY) ? expf(my_lse - M) : 0.f;
    float W = my_w;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
    #pragma unroll
    for (int i = 0; i < kCombineChunk; ++i) {
      const float wi = __shfl_sync(0xffffffffu, my_w, i);
      if (i < n) {
        const float* f = reinterpret_cast<const float*>(&v[i]);
        #pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += wi * f[e];
      }
    }
    if (ncb == 1) {
      write_row<D>(orow, p.lse + row, lane, M, W, acc);
      continue;
    }
    // ---- publish this chunk; the last chunk of the row merges them all
    float* cs = p.chunk_state + w * (D + 4);
    #pragma unroll
    for (int e = 0; e < VEC; ++e) cs[4 + lane * VEC + e] = acc[e];
    if (lane == 0) { cs[0] = M; cs[1] = W; }
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(&p.row_cnt[row], 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != ncb - 1) continue;
    __threadfence();
    // all chunk states of the row, in groups of kMergeGroup loaded at once (from L2: they were
    // written by other warps of this grid)
    const float* cs0 = p.chunk_state + (w - j) * (D + 4);
    float Mt = -INFINITY, Wt = 0.f;
    #pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    #pragma unroll 1
    for (int c0 = 0; c0 < ncb; c0 += kMergeGroup) {
      const int nc = min(kMergeGroup, ncb - c0);
      const float* g = cs0 + (int64_t)c0 * (D + 4);
      const float2 mw = lane < nc ? __ldcg(reinterpret_cast<const float2*>(g + (int64_t)lane * (D + 4)))
                                  : make_float2(-INFINITY, 0.f);
      const float mc = mw.x, wc = mw.y;
      V cv[kMergeGroup];
      #pragma unroll
      for (int i = 0; i < kMergeGroup; ++i)
        if (i < nc) cv[i] = __ldcg(reinterpret_cast<const V*>(g + (int64_t)i * (D + 4) + 4) + lane);
      float Mg = mc;
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) Mg = fmaxf(Mg, __shfl_xor_sync(0xffffffffu, Mg, o));
      const float Mn = fmaxf(Mt, Mg);
      if (Mn == -INFINITY) continue;  // no visible key in any chunk so far
      const float a = Mt == -INFINITY ? 0.f : expf(Mt - Mn);
      const float wl = mc == -INFINITY ? 0.f : expf(mc - Mn);
      float Wg = wl * wc;
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) Wg += __shfl_xor_sync(0xffffffffu, Wg, o);
      Wt = Wt * a + Wg;
      #pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] *= a;
      #pragma unroll
      for (int i = 0; i < kMergeGroup; ++i) {
        const float wi = __shfl_sync(0xffffffffu, wl, i);
        if (i < nc) {
          const float* f = reinterpret_cast<const float*>(&cv[i]);
          #pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += wi * f[e];
        }
      }
      Mt = Mn;
    }
    write_row<D>(orow, p.lse + row, lane, Mt, Wt, acc);
    if (lane == 0) p.row_cnt[row] = 0;  // ready for the next combine on this workspace
  }
}

cudaError_t launch_combine(const CombineParams& p, int device, cudaStream_t st) {
  if ((int64_t)p.B * p.T * p.Hq <= 0) return cudaSuccess;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return cudaErrorUnknown;
  const void* fn = p.D == 128 ? (const void*)combine_kernel<128> : (const void*)combine_kernel<64>;
  const int smem = p.B <= kCombineSmemRequests ? 12 * (p.B + 1) : 0;
  if (!ensure_smem_attr(fn, smem)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms * kCombineCtasPerSm);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // scheduled while the split kernel drains
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.D == 128) return cudaLaunchKernelEx(&cfg, combine_kernel<128>, p);
  if (p.D == 64) return cudaLaunchKernelEx(&cfg, combine_kernel<64>, p);
  return cudaErrorInvalidValue;
}

}  // namespace decattn
