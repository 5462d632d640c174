// plan.cu -- the planner: uniform KV tiles greedily bin-packed onto the split kernel's
// CTAs, computed by one thread block so that it stays on the device (graph-capturable,
// no host round trip).
//
// Method: "HPC-Ops: Tencent's CUDA Kernel Library for LLM Inference Hot Paths", section
// "How the kernels are organized around specific workload shapes" -- requests are split
// into uniform KV tiles, the tiles are assigned before each decode step and balanced
// across CTAs with a greedy bin-packing strategy. Greedy rule used: largest tile first
// (stable), each to the least-loaded bin, lowest bin index on ties.
//
// How the block computes it without a sequential pass over every tile:
//  * full tiles all cost tile_len and come first in the sorted order, so the greedy pass
//    deals them round-robin: full tile f (in (b, h, i) order) goes to bin f mod N at
//    position f div N;
//  * after them, bins [F mod N, N) hold the least load; the next N - F mod N tiles (the
//    largest partial tiles) each find an untouched least-loaded bin, in index order;
//  * only the remaining partial tiles (at most one per (b, h)) need the sequential
//    least-loaded search, done by one warp with warp-wide min reductions.
#include "common.cuh"

namespace decattn {

constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxBins = 8192;

struct PlanScratch {
  int64_t* S;        // [B+1] exclusive prefix over requests of tiles per (b, h) pair
  int64_t* SF;       // [B+1] same for full tiles
  int32_t* SP;       // [B+1] same for "has a partial tile"
  int32_t* plist;    // [B]   requests with a partial tile, in b order
  int32_t* pcost;    // [B]   their partial-tile cost
  int32_t* sorted_b; // [B]   same requests sorted by cost desc, b asc
  int32_t* part_bin; // [B*Hkv] bin of the s-th partial tile in greedy order
  int32_t* part_pos; // [B*Hkv] its position among that bin's partial tiles
};

__host__ __device__ inline int64_t plan_scratch_bytes(int B, int Hkv) {
  return align_up(8 * (int64_t)(B + 1), 32) * 2 + align_up(4 * (int64_t)(B + 1), 32) +
         align_up(4 * (int64_t)B, 32) * 3 + align_up(4 * (int64_t)B * Hkv, 32) * 2;
}

__device__ inline PlanScratch carve_scratch(char* p, int B, int Hkv) {
  PlanScratch s;
  s.S = reinterpret_cast<int64_t*>(p); p += align_up(8 * (int64_t)(B + 1), 32);
  s.SF = reinterpret_cast<int64_t*>(p); p += align_up(8 * (int64_t)(B + 1), 32);
  s.SP = reinterpret_cast<int32_t*>(p); p += align_up(4 * (int64_t)(B + 1), 32);
  s.plist = reinterpret_cast<int32_t*>(p); p += align_up(4 * (int64_t)B, 32);
  s.pcost = reinterpret_cast<int32_t*>(p); p += align_up(4 * (int64_t)B, 32);
  s.sorted_b = reinterpret_cast<int32_t*>(p); p += align_up(4 * (int64_t)B, 32);
  s.part_bin = reinterpret_cast<int32_t*>(p); p += align_up(4 * (int64_t)B * Hkv, 32);
  s.part_pos = reinterpret_cast<int32_t*>(p);
  return s;
}

// Exclusive block-wide scan of (a, b, c) over kPlanThreads threads; returns the prefix and
// adds the block totals into tot.
struct Tri { long long a, b; int c; };

__device__ inline Tri block_exscan(Tri v, Tri& tot, Tri* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  Tri inc = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long a = __shfl_up_sync(0xffffffffu, inc.a, o);
    long long b = __shfl_up_sync(0xffffffffu, inc.b, o);
    int c = __shfl_up_sync(0xffffffffu, inc.c, o);
    if (lane >= o) { inc.a += a; inc.b += b; inc.c += c; }
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    Tri t = warp_tot[lane];
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long a = __shfl_up_sync(0xffffffffu, t.a, o);
      long long b = __shfl_up_sync(0xffffffffu, t.b, o);
      int c = __shfl_up_sync(0xffffffffu, t.c, o);
      if (lane >= o) { t.a += a; t.b += b; t.c += c; }
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  Tri base = w ? warp_tot[w - 1] : Tri{0, 0, 0};
  Tri all = warp_tot[31];
  __syncthreads();
  Tri ex{base.a + inc.a - v.a, base.b + inc.b - v.b, base.c + inc.c - v.c};
  tot.a += all.a; tot.b += all.b; tot.c += all.c;
  return ex;
}

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t* __restrict__ seq_lens, const PlanHeader init, char* __restrict__ plan) {
  const int B = init.batch, Hkv = init.n_kv_heads, tl = init.tile_len, N = init.n_bins;
  const int64_t max_units = init.max_units;
  extern __shared__ uint32_t sm_dyn[];
  uint32_t* load = sm_dyn;           // [N] bin load minus the common full-tile base
  int32_t* pcount = reinterpret_cast<int32_t*>(sm_dyn + N);  // [N] partial tiles per bin
  __shared__ Tri warp_tot[32];
  __shared__ int32_t sh_cost[kPlanThreads];
  __shared__ int32_t sh_status;

  PlanHeader* hdr = reinterpret_cast<PlanHeader*>(plan);
  int32_t* bin_off = reinterpret_cast<int32_t*>(plan + init.off_bin_off);
  int32_t* pair_off = reinterpret_cast<int32_t*>(plan + init.off_pair_off);
  Unit* units = reinterpret_cast<Unit*>(plan + init.off_units);
  PlanScratch sc = carve_scratch(plan + init.off_scratch, B, Hkv);
  const int tid = threadIdx.x;
  if (tid == 0) {
    sh_status = 0;
    PlanHeader h = init;
    h.magic = 0;  // published last, once the plan is complete
    *hdr = h;
  }

  // ---- 1. per-request tile counts and their prefix sums
  Tri carry{0, 0, 0};
  for (int base = 0; base < B; base += kPlanThreads) {
    const int b = base + tid;
    int64_t L = b < B ? seq_lens[b] : 0;
    if (L < 0) { atomicCAS(&sh_status, 0, DECATTN_EDEVICE); L = 0; }
    Tri v{(L + tl - 1) / tl, L / tl, (L % tl) != 0};
    Tri before = carry;
    Tri ex = block_exscan(v, carry, warp_tot);
    if (b < B) {
      sc.S[b] = before.a + ex.a;
      sc.SF[b] = before.b + ex.b;
      sc.SP[b] = before.c + ex.c;
      if (v.c) { sc.plist[before.c + ex.c] = b; sc.pcost[before.c + ex.c] = (int32_t)(L % tl); }
    }
  }
  if (tid == 0) { sc.S[B] = carry.a; sc.SF[B] = carry.b; sc.SP[B] = carry.c; }
  const int64_t U = (int64_t)Hkv * carry.a;
  const int64_t F = (int64_t)Hkv * carry.b;
  const int mB = carry.c;
  const int64_t m = (int64_t)Hkv * mB;
  __syncthreads();
  if (U > max_units) atomicCAS(&sh_status, 0, DECATTN_ECAPACITY);
  __syncthreads();
  if (sh_status != 0) {
    for (int k = tid; k <= N; k += kPlanThreads) bin_off[k] = 0;
    if (tid == 0) {
      hdr->n_units = 0;
      hdr->status = sh_status;
      __threadfence();
      hdr->magic = kPlanMagic;
    }
    return;
  }

  // ---- 2. pair offsets (first partial slot of each (b, h))
  for (int64_t p = tid; p < (int64_t)B * Hkv; p += kPlanThreads) {
    const int b = (int)(p / Hkv), h = (int)(p % Hkv);
    pair_off[p] = (int32_t)(Hkv * sc.S[b] + (int64_t)h * (sc.S[b + 1] - sc.S[b]));
  }
  if (tid == 0) pair_off[(int64_t)B * Hkv] = (int32_t)U;

  // ---- 3. requests with a partial tile, sorted by cost (desc), then b: rank by counting
  for (int jb = 0; jb < mB; jb += kPlanThreads) {
    const int j = jb + tid;
    const int cj = j < mB ? sc.pcost[j] : 0;
    int rank = 0;
    for (int cb = 0; cb < mB; cb += kPlanThreads) {
      __syncthreads();
      sh_cost[tid] = cb + tid < mB ? sc.pcost[cb + tid] : -1;
      __syncthreads();
      const int lim = min(kPlanThreads, mB - cb);
      for (int k = 0; k < lim; ++k) {
        const int c = sh_cost[k];
        rank += (c > cj) | ((c == cj) & (cb + k < j));
      }
    }
    if (j < mB) sc.sorted_b[rank] = sc.plist[j];
  }
  __syncthreads();

  // ---- 4. greedy placement of the partial tiles (s-th in sorted order: request
  //         sorted_b[s / Hkv], head s % Hkv)
  const int64_t qf = F / N;
  const int rf = (int)(F % N);
  const int64_t first = m < (int64_t)(N - rf) ? m : (int64_t)(N - rf);
  for (int k = tid; k < N; k += kPlanThreads) {
    uint32_t l = k < rf ? (uint32_t)tl : 0u;
    int32_t pc = 0;
    const int64_t s = k - rf;
    if (k >= rf && s < first) {
      l += (uint32_t)(seq_lens[sc.sorted_b[s / Hkv]] % tl);
      pc = 1;
      sc.part_bin[s] = k;
      sc.part_pos[s] = 0;
    }
    load[k] = l;
    pcount[k] = pc;
  }
  __syncthreads();
  if (tid < 32 && first < m) {
    const int lane = tid;
    // each lane watches bins lane, lane+32, ...; it caches the least (load, bin) among them
    uint32_t lmin = 0xffffffffu, lidx = 0xffffffffu;
    for (int k = lane; k < N; k += 32)
      if (load[k] < lmin) { lmin = load[k]; lidx = (uint32_t)k; }
    int32_t cost_next = 0;
    for (int64_t s0 = first; s0 < m; s0 += 32) {
      const int64_t s_l = s0 + lane;
      cost_next = s_l < m ? (int32_t)(seq_lens[sc.sorted_b[s_l / Hkv]] % tl) : 0;
      const int64_t n_here = m - s0 < 32 ? m - s0 : 32;
      for (int i = 0; i < n_here; ++i) {
        const uint32_t c = (uint32_t)__shfl_sync(0xffffffffu, cost_next, i);
        const uint32_t gmin = __reduce_min_sync(0xffffffffu, lmin);
        const uint32_t kbest = __reduce_min_sync(0xffffffffu, lmin == gmin ? lidx : 0xffffffffu);
        if (lane == (int)(kbest & 31)) {
          const int64_t s = s0 + i;
          sc.part_bin[s] = (int32_t)kbest;
          sc.part_pos[s] = pcount[kbest]++;
          load[kbest] += c;
          lmin = 0xffffffffu; lidx = 0xffffffffu;
          for (int k = lane; k < N; k += 32)
            if (load[k] < lmin) { lmin = load[k]; lidx = (uint32_t)k; }
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();

  // ---- 5. bin offsets (CSR): full tiles of bin k, then its partial tiles
  {
    Tri c2{0, 0, 0};
    for (int base = 0; base < N; base += kPlanThreads) {
      const int k = base + tid;
      const long long cnt = k < N ? (long long)(qf + (k < rf)) + pcount[k] : 0;
      Tri before = c2;
      Tri ex = block_exscan(Tri{cnt, 0, 0}, c2, warp_tot);
      if (k < N) bin_off[k] = (int32_t)(before.a + ex.a);
    }
    if (tid == 0) bin_off[N] = (int32_t)c2.a;
  }
  __syncthreads();

  // ---- 6. the tiles
  for (int64_t f = tid; f < F; f += kPlanThreads) {
    int lo = 0, hi = B - 1;  // last b with Hkv * SF[b] <= f
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)Hkv * sc.SF[mid] <= f) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int64_t fb = sc.SF[b + 1] - sc.SF[b];
    const int64_t r = f - (int64_t)Hkv * sc.SF[b];
    const int h = (int)(r / fb);
    const int64_t i = r % fb;
    const int64_t nb = sc.S[b + 1] - sc.S[b];
    const int32_t L = seq_lens[b];
    Unit u;
    u.b = b; u.h = h; u.tok_begin = (int32_t)(i * tl); u.tok_end = (int32_t)((i + 1) * tl); u.seq_len = L;
    u.slot = nb == 1 ? -1 : (int32_t)(Hkv * sc.S[b] + h * nb + i);
    u.tile = (int32_t)i; u.zero = 0;
    const int k = (int)(f % N);
    units[bin_off[k] + f / N] = u;
  }
  for (int64_t s = tid; s < m; s += kPlanThreads) {
    const int b = sc.sorted_b[s / Hkv], h = (int)(s % Hkv);
    const int64_t fb = sc.SF[b + 1] - sc.SF[b];
    const int64_t nb = sc.S[b + 1] - sc.S[b];
    const int32_t L = seq_lens[b];
    Unit u;
    u.b = b; u.h = h; u.tok_begin = (int32_t)(fb * tl); u.tok_end = L; u.seq_len = L;
    u.slot = nb == 1 ? -1 : (int32_t)(Hkv * sc.S[b] + h * nb + fb);
    u.tile = (int32_t)fb; u.zero = 0;
    const int k = sc.part_bin[s];
    units[bin_off[k] + (qf + (k < rf)) + sc.part_pos[s]] = u;
  }
  __syncthreads();
  if (tid == 0) {
    hdr->n_units = (int32_t)U;
    hdr->status = DECATTN_OK;
    __threadfence();
    hdr->magic = kPlanMagic;
  }
}

// ------------------------------------------------------------------ host side
struct PlanLayout {
  int64_t off_bin_off, off_pair_off, off_units, off_scratch, total;
};

static PlanLayout plan_layout(int B, int Hkv, int N, int64_t max_units) {
  PlanLayout L;
  int64_t o = sizeof(PlanHeader);
  L.off_bin_off = o; o = align_up(o + 4 * (int64_t)(N + 1), 32);
  L.off_pair_off = o; o = align_up(o + 4 * ((int64_t)B * Hkv + 1), 32);
  L.off_units = o; o = align_up(o + (int64_t)sizeof(Unit) * max_units, 32);
  L.off_scratch = o; o = align_up(o + plan_scratch_bytes(B, Hkv), 32);
  L.total = o;
  return L;
}

static int64_t plan_capacity(int B, int Hkv, int tl, int64_t max_total) {
  return (int64_t)Hkv * ((max_total + tl - 1) / tl + B);
}


static bool plan_args_ok(int B, int Hkv, int tl, int64_t max_total, int N) {
  if (B < 0 || Hkv <= 0 || tl <= 0 || (tl % 16) != 0 || max_total < 0 || N <= 0 || N > kPlanMaxBins) return false;
  const int64_t cap = plan_capacity(B, Hkv, tl, max_total);
  if (cap >= (1ll << 31) - 1 || max_total >= (1ll << 31)) return false;
  // keeps every relative bin load of the greedy pass below 2^32
  if ((double)B * Hkv * tl / N + 2.0 * tl >= 4294967295.0) return false;
  return true;
}

}  // namespace decattn

using namespace decattn;

extern "C" size_t dec_attn_plan_bytes(int batch, int n_kv_heads, int tile_len, int64_t max_total_kv_tokens,
                                       int n_bins) {
  if (n_bins == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    n_bins = default_bins(dev);
  }
  if (!plan_args_ok(batch, n_kv_heads, tile_len, max_total_kv_tokens, n_bins)) return 0;
  const int64_t cap = plan_capacity(batch, n_kv_heads, tile_len, max_total_kv_tokens);
  return (size_t)plan_layout(batch, n_kv_heads, n_bins, cap).total;
}

extern "C" int dec_attn_plan(const int32_t* seq_lens, int batch, int n_kv_heads, int tile_len,
                             int64_t max_total_kv_tokens, int n_bins, void* plan_buf, size_t plan_bytes,
                             dec_attn_plan_t* plan, void* stream) {
  if (!plan || !plan_buf || (batch > 0 && !seq_lens)) return DECATTN_EINVAL;
  if (n_bins == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DECATTN_ECUDA;
    n_bins = default_bins(dev);
    if (n_bins <= 0) return DECATTN_ECUDA;
  }
  if (batch < 0 || n_kv_heads <= 0 || tile_len <= 0 || max_total_kv_tokens < 0 || n_bins < 0) return DECATTN_EINVAL;
  if (!plan_args_ok(batch, n_kv_heads, tile_len, max_total_kv_tokens, n_bins)) return DECATTN_ENOTSUP;
  if ((reinterpret_cast<uintptr_t>(plan_buf) & 15) != 0) return DECATTN_EALIGN;
  const int64_t cap = plan_capacity(batch, n_kv_heads, tile_len, max_total_kv_tokens);
  const PlanLayout L = plan_layout(batch, n_kv_heads, n_bins, cap);
  if ((int64_t)plan_bytes < L.total) return DECATTN_ESMALL;

  PlanHeader h{};
  h.magic = 0;
  h.status = DECATTN_OK;
  h.n_bins = n_bins;
  h.batch = batch;
  h.n_kv_heads = n_kv_heads;
  h.tile_len = tile_len;
  h.n_units = 0;
  h.n_pairs = batch * n_kv_heads;
  h.max_units = cap;
  h.off_bin_off = (int32_t)L.off_bin_off;
  h.off_pair_off = (int32_t)L.off_pair_off;
  h.off_units = (int32_t)L.off_units;
  h.off_scratch = (int32_t)L.off_scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = (size_t)n_bins * 8;
  if (!ensure_smem_attr((const void*)plan_kernel, kPlanMaxBins * 8)) return DECATTN_ECUDA;
  plan_kernel<<<1, kPlanThreads, smem, st>>>(seq_lens, h, static_cast<char*>(plan_buf));
  if (cudaGetLastError() != cudaSuccess) return DECATTN_ECUDA;
  plan->buf = plan_buf;
  plan->buf_bytes = plan_bytes;
  plan->batch = batch;
  plan->n_kv_heads = n_kv_heads;
  plan->tile_len = tile_len;
  plan->n_bins = n_bins;
  plan->max_units = cap;
  return DECATTN_OK;
}
