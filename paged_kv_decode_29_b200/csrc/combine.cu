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
// by request (block-sparse plans: (request, KV head) pair by pair, since pairs keep their
// own tiles). The kernel is persistent: every warp takes items w, w + #warps, ...
//  * a warp loads the lse and the D floats of up to kCombineChunk (32) partial rows (8 loads in
//    flight per lane at a time) and folds them into (max, weight, weighted sum);
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
constexpr int kCombineGroup = 4;            // items a warp folds before one fence and its counter updates

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

// Items are numbered unit by unit: per request (dense plans: every KV head of a request has the
// same tiles) or per (request, KV head) pair (block-sparse plans); NU units of RPU query rows.
template <int D, bool SPARSE>
__global__ void __launch_bounds__(kCombineThreads, kCombineCtasPerSm) combine_kernel(const CombineParams p) {
  constexpr int VEC = D / 32;
  using V = typename CombineVec<D>::T;
  extern __shared__ int32_t req_sm[];  // chunk prefix [NU + 1], tile prefix [NU + 1], seq_lens [B + 1]
  // The plan is complete when this grid starts (the split kernel lets it launch only after its
  // own wait on the planner), so everything but the partials is read before waiting.
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
  if (hdr->magic != kPlanMagic || hdr->status != DECATTN_OK) return;  // the split kernel reports it
  const int NU = SPARSE ? p.B * p.Hkv : p.B;
  const int32_t* cb_sm = plan_arr(p.plan, hdr->off_cb);
  const int32_t* S = plan_arr(p.plan, hdr->off_S);
  const int32_t* Ls = p.seq_lens;
  if (NU <= kCombineSmemRequests) {
    int32_t* a = req_sm;
    int32_t* b = req_sm + (NU + 1);
    int32_t* c = req_sm + 2 * (NU + 1);
    for (int i = threadIdx.x; i <= NU; i += kCombineThreads) {
      a[i] = cb_sm[i];
      b[i] = S[i];
    }
    for (int i = threadIdx.x; i <= p.B; i += kCombineThreads) c[i] = i < p.B ? Ls[i] : 0;
    __syncthreads();
    cb_sm = a; S = b; Ls = c;
  }
  griddep_wait();  // the split kernel's partials are complete and visible
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item numbers fit 32 bits (checked on the host), so does every product below
  const int rows_per_b = SPARSE ? p.GT : p.T * p.Hq;  // query rows per unit
  const int total = rows_per_b * cb_sm[NU];
  const int nwarps = gridDim.x * kCombineWarps;

  // The warp's items w0, w0 + nwarps, ... are taken kCombineGroup at a time: each is folded; a
  // row made of one chunk is written at once, the others publish their chunk state. Then one
  // fence for the group and the row counters of its items bumped together (one lane each);
  // the warp merges the rows it completed.
  for (int w0 = blockIdx.x * kCombineWarps + warp; w0 < total; w0 += nwarps * kCombineGroup) {
    int64_t g_row = -1;  // lane k: row of the group's k-th item if that item published a chunk
    int g_first = 0;     // lane k: item number of chunk 0 of that row
    int g_ncb = 0;       // lane k: chunks of that row
    #pragma unroll 1
    for (int k = 0; k < kCombineGroup; ++k) {
      const int64_t wl = (int64_t)w0 + (int64_t)k * nwarps;
      if (wl >= total) break;
      const int w = (int)wl;
      int lo = 0, hi = NU - 1;  // unit: last u with rows_per_b * cb[u] <= w
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rows_per_b * cb_sm[mid] <= w) lo = mid; else hi = mid - 1;
      }
      const int u = lo;
      const int ncb = cb_sm[u + 1] - cb_sm[u];
      const int local = w - rows_per_b * cb_sm[u];
      const int row_in_u = local / ncb, j = local - row_in_u * ncb;
      int64_t row, slot_base;
      int r, nt;  // query row within the tile's partial block; tiles of the row's (request, head)
      if (SPARSE) {
        const int b = u / p.Hkv, h = u - b * p.Hkv;
        const int t = row_in_u / p.G, g = row_in_u - t * p.G;
        row = ((int64_t)b * p.T + t) * p.Hq + h * p.G + g;
        r = row_in_u;
        nt = S[u + 1] - S[u];  // kept tiles of the pair
        slot_base = S[u];
      } else {
        const int b = u;
        const int t = row_in_u / p.Hq, qh = row_in_u - t * p.Hq;
        row = ((int64_t)b * p.T + t) * p.Hq + qh;
        const int h = qh / p.G;
        r = t * p.G + (qh - h * p.G);
        const int L = Ls[b];
        nt = L > 0 ? (L + p.tl - 1) / p.tl : 0;  // == S[b + 1] - S[b]
        slot_base = (int64_t)p.Hkv * S[b] + (int64_t)h * nt;
      }
      float* orow = p.out + row * D;
      float acc[VEC];
      #pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
      if (nt == 0) {  // no key at all
        write_row<D>(orow, p.lse + row, lane, -INFINITY, 0.f, acc);
        continue;
      }
      const int64_t slot0 = slot_base + (int64_t)j * kCombineChunk;
      const int n = min(kCombineChunk, nt - j * kCombineChunk);
      // ---- fold up to kCombineChunk partial rows, kLoads loads in flight per lane at a time
      //      (with every warp loading, the fold runs at DRAM bandwidth; batches of kLoads keep the
      //      registers below the occupancy limit). Lane i holds the lse of row i of the chunk.
      static_assert(kCombineChunk <= 32 && kCombineChunk % 8 == 0, "one lse per lane, whole batches");
      const float my_lse = lane < n ? p.part_lse[(slot0 + lane) * p.GT + r] : -INFINITY;
      const V* src = reinterpret_cast<const V*>(p.part_o + (slot0 * p.GT + r) * D) + lane;
      const int64_t stride = (int64_t)p.GT * (D / VEC);  // V elements between consecutive tiles' rows
      constexpr int kLoads = 8;
      constexpr int kRounds = kCombineChunk / kLoads;
      V v[kLoads];
      #pragma unroll
      for (int i = 0; i < kLoads; ++i)
        if (i < n) v[i] = __ldcs(src + i * stride);
      float M = my_lse;
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float my_w = (lane < n && M != -INFINITY) ? expf(my_lse - M) : 0.f;
      float W = my_w;
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
      #pragma unroll
      for (int hf = 0; hf < kRounds; ++hf) {
        if (hf > 0) {
          if (n <= hf * kLoads) break;
          #pragma unroll
          for (int i = 0; i < kLoads; ++i)
            if (hf * kLoads + i < n) v[i] = __ldcs(src + (hf * kLoads + i) * stride);
        }
        #pragma unroll
        for (int i = 0; i < kLoads; ++i) {
          const float wi = __shfl_sync(0xffffffffu, my_w, hf * kLoads + i);
          if (hf * kLoads + i < n) {
            const float* f = reinterpret_cast<const float*>(&v[i]);
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] += wi * f[e];
          }
        }
      }
      if (ncb == 1) {
        write_row<D>(orow, p.lse + row, lane, M, W, acc);
        continue;
      }
      // ---- publish this chunk
      float* cs = p.chunk_state + (int64_t)w * (D + 4);
      V av;
      #pragma unroll
      for (int e = 0; e < VEC; ++e) reinterpret_cast<float*>(&av)[e] = acc[e];
      reinterpret_cast<V*>(cs + 4)[lane] = av;
      if (lane == 0) *reinterpret_cast<float2*>(cs) = make_float2(M, W);
      if (lane == k) { g_row = row; g_first = w - j; g_ncb = ncb; }
    }
    if (__ballot_sync(0xffffffffu, g_row >= 0) == 0u) continue;
    __threadfence();  // the group's chunk states are visible before its counters move
    int prev = -1;
    if (g_row >= 0) prev = atomicAdd(&p.row_cnt[g_row], 1);
    unsigned last = __ballot_sync(0xffffffffu, g_row >= 0 && prev == g_ncb - 1);
    if (last == 0u) continue;
    __threadfence();  // and the other chunks' states are read after the counter
    while (last != 0u) {
      const int k = __ffs(last) - 1;
      last &= last - 1u;
      const int64_t row = __shfl_sync(0xffffffffu, g_row, k);
      const int first = __shfl_sync(0xffffffffu, g_first, k);
      const int ncb = __shfl_sync(0xffffffffu, g_ncb, k);
      // ---- merge the row's chunk states, kMergeGroup loaded at once (from L2: they were written
      //      by other warps of this grid), with an online rescale between groups
      const float* cs0 = p.chunk_state + (int64_t)first * (D + 4);
      float acc[VEC];
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
      write_row<D>(p.out + row * D, p.lse + row, lane, Mt, Wt, acc);
      if (lane == 0) p.row_cnt[row] = 0;  // ready for the next combine on this workspace
    }
  }
}

cudaError_t launch_combine(const CombineParams& p, int device, cudaStream_t st) {
  if ((int64_t)p.B * p.T * p.Hq <= 0) return cudaSuccess;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return cudaErrorUnknown;
  if (p.D != 128 && p.D != 64) return cudaErrorInvalidValue;
  const void* fn = p.sparse ? (p.D == 128 ? (const void*)combine_kernel<128, true> : (const void*)combine_kernel<64, true>)
                            : (p.D == 128 ? (const void*)combine_kernel<128, false> : (const void*)combine_kernel<64, false>);
  const int64_t nu = p.sparse ? (int64_t)p.B * p.Hkv : p.B;
  const int smem = nu <= kCombineSmemRequests ? (int)(4 * (2 * (nu + 1) + p.B + 1)) : 0;
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
  void* args[] = {const_cast<CombineParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace decattn
