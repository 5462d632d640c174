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
//    position f div N -- a closed form, so the plan stores only the prefix sums it is
//    decoded from (plan_unit() in common.cuh);
//  * after them, bins [F mod N, N) hold the least load; the next N - F mod N tiles (the
//    largest partial tiles) each find an untouched least-loaded bin, in index order;
//  * only the remaining partial tiles (at most one per (b, h)) need the sequential
//    least-loaded search, done by one warp with warp-wide min reductions.
// The plan's size is O(batch * n_kv_heads + n_bins), independent of the tile count.
#include "common.cuh"
#include "host_errors.h"

namespace decattn {

constexpr int kPlanThreads = 512;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPlanMaxBins = 8192;
constexpr int kPlanSmemRequests = 4096;  // per-request arrays sit in shared memory up to this batch
constexpr int kPlanMaxSmem = 200 * 1024;
constexpr int kPlanRegWords = 8;  // sparse planner: mask words of a pair held in registers

// Per-request arrays (index b): exclusive prefix sums over requests of the tiles of one
// (b, h) pair (S), of its full tiles (SF) and of "has a partial tile" (SP); the requests
// with a partial tile in b order (plist, with their partial-tile cost pcost) and sorted by
// that cost, largest first (sorted_b).
struct ReqArrays {
  int32_t *S, *SF, *SP, *plist, *pcost, *sorted_b;
};

__host__ __device__ inline int64_t req_stride(int B) { return align_up(4 * (int64_t)(B + 1), 16); }
__host__ __device__ inline int64_t req_arrays_bytes(int B) { return 6 * req_stride(B); }
__host__ __device__ inline int64_t plan_bins_smem(int N) { return align_up(12 * (int64_t)N + 4, 16); }

// Global scratch of the plan buffer: the per-request arrays when they do not fit in shared
// memory, then the bin and in-bin position of every partial tile in greedy order.
__host__ __device__ inline int64_t plan_scratch_bytes(int B, int Hkv) {
  return req_arrays_bytes(B) + 2 * align_up(4 * (int64_t)B * Hkv, 32);
}

__device__ inline ReqArrays carve_req(char* p, int B) {
  const int64_t st = req_stride(B);
  ReqArrays r;
  r.S = reinterpret_cast<int32_t*>(p);
  r.SF = reinterpret_cast<int32_t*>(p + st);
  r.SP = reinterpret_cast<int32_t*>(p + 2 * st);
  r.plist = reinterpret_cast<int32_t*>(p + 3 * st);
  r.pcost = reinterpret_cast<int32_t*>(p + 4 * st);
  r.sorted_b = reinterpret_cast<int32_t*>(p + 5 * st);
  return r;
}

// Exclusive block-wide scan of (a, b, c, d) over kPlanThreads threads; returns the prefix and
// adds the block totals into tot. warp_tot holds one entry per warp.
struct Tri { long long a, b; int c; long long d; };

__device__ inline Tri block_exscan(Tri v, Tri& tot, Tri* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  Tri inc = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long a = __shfl_up_sync(0xffffffffu, inc.a, o);
    long long b = __shfl_up_sync(0xffffffffu, inc.b, o);
    int c = __shfl_up_sync(0xffffffffu, inc.c, o);
    long long dd = __shfl_up_sync(0xffffffffu, inc.d, o);
    if (lane >= o) { inc.a += a; inc.b += b; inc.c += c; inc.d += dd; }
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    Tri t = lane < kPlanWarps ? warp_tot[lane] : Tri{0, 0, 0, 0};
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long a = __shfl_up_sync(0xffffffffu, t.a, o);
      long long b = __shfl_up_sync(0xffffffffu, t.b, o);
      int c = __shfl_up_sync(0xffffffffu, t.c, o);
      long long dd = __shfl_up_sync(0xffffffffu, t.d, o);
      if (lane >= o) { t.a += a; t.b += b; t.c += c; t.d += dd; }
    }
    if (lane < kPlanWarps) warp_tot[lane] = t;
  }
  __syncthreads();
  Tri base = w ? warp_tot[w - 1] : Tri{0, 0, 0, 0};
  Tri all = warp_tot[kPlanWarps - 1];
  __syncthreads();
  Tri ex{base.a + inc.a - v.a, base.b + inc.b - v.b, base.c + inc.c - v.c, base.d + inc.d - v.d};
  tot.a += all.a; tot.b += all.b; tot.c += all.c; tot.d += all.d;
  return ex;
}

// Greedy placement of the partial tiles s in [first, m) by one warp. Lane l owns the bins
// [l*K, (l+1)*K) and keeps their loads (relative to the common full-tile base) in
// registers; a warp-wide min over the packed key (load << 5 | lane) finds the least-loaded
// bin, the lowest bin index winning ties (lower lanes own lower bins, and each lane keeps
// its lowest-index minimum). Needs every relative load below 2^27 (checked on the host).
template <int KMAX>
__device__ void greedy_partials(int lane, int N, int first, int m, int Hkv, int tl,
                                const int32_t* __restrict__ seq_lens, const int32_t* sorted_b, uint32_t* load_sm,
                                int32_t* pcount_sm, int32_t* part_bin, int32_t* part_pos) {
  const int K = (N + 31) / 32;
  const int k0 = lane * K;
  uint32_t ld[KMAX];
  int32_t pc[KMAX];
  #pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const int k = k0 + j;
    const bool ok = j < K && k < N;
    ld[j] = ok ? load_sm[k] : 0x07ffffffu;  // above any real load
    pc[j] = ok ? pcount_sm[k] : 0;
  }
  uint32_t lmin = ld[0];
  int lj = 0;
  #pragma unroll
  for (int j = 1; j < KMAX; ++j)
    if (ld[j] < lmin) { lmin = ld[j]; lj = j; }
  for (int s0 = first; s0 < m; s0 += 32) {
    const int sl = s0 + lane;
    const uint32_t cl = sl < m ? (uint32_t)(seq_lens[sorted_b[sl / Hkv]] % tl) : 0u;
    const int n_here = min(32, m - s0);
    for (int i = 0; i < n_here; ++i) {
      const uint32_t c = __shfl_sync(0xffffffffu, cl, i);
      const uint32_t key = __reduce_min_sync(0xffffffffu, (lmin << 5) | (uint32_t)lane);
      if ((int)(key & 31u) == lane) {
        const int s = s0 + i;
        int pos = 0;
        #pragma unroll
        for (int j = 0; j < KMAX; ++j) {  // selects only: no store or branch per register
          const bool sel = j == lj;
          pos = sel ? pc[j] : pos;
          pc[j] += sel ? 1 : 0;
          ld[j] += sel ? c : 0u;
        }
        part_bin[s] = k0 + lj;
        part_pos[s] = pos;
        lmin = ld[0];
        lj = 0;
        #pragma unroll
        for (int j = 1; j < KMAX; ++j)
          if (ld[j] < lmin) { lmin = ld[j]; lj = j; }
      }
    }
  }
  #pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const int k = k0 + j;
    if (j < K && k < N) pcount_sm[k] = pc[j];
  }
}

// The same greedy pass over the partial tiles s in [first, m), batched across the block: the
// bins are kept sorted by key (load << 32 | bin) in shared memory, and each round tries the
// next up-to-kPlanThreads tiles (largest first) on the least-loaded bins in order. Tile t of
// the round goes to the t-th sorted bin exactly when that bin's key is below every key the
// round has made so far (a touched bin's key plus its tile), so the round assigns the longest
// prefix of such tiles (at least one), merges the touched bins back into the sorted list and
// repeats. Same assignment as one tile at a time, ties included (the bin index is the key's
// low word).
//
// Called only when the closed-form first batch left tiles over (first < m), so the first batch
// filled bins rf .. N-1 (rf = N - first), one tile each, with non-increasing loads, and bins
// 0 .. rf-1 hold one more full tile (load tl, above every partial tile's cost). The sorted list
// therefore starts without a sort: the first batch's bins by (load, bin), each placed with two
// binary searches, then bins 0 .. rf-1 in order. The merge of a round places every key by its
// rank: the round's new keys are sorted within each warp (32-key chunks), and a key's rank is
// its count of smaller keys in every chunk and in the untouched run.
// Called by every thread of the block. Shared area: two key lists [N], the round's new keys
// [kPlanThreads], warp minima [kPlanWarps], the round's prefix length, the costs of tiles
// [first, m).
__host__ __device__ inline int64_t greedy_batched_bytes(int N, int64_t max_partials) {
  return align_up(16 * (int64_t)N + 8 * (int64_t)(kPlanThreads + kPlanWarps) + 16 + 4 * max_partials, 16);
}

__device__ __forceinline__ int count_below32(const uint64_t* c, uint64_t k) {  // sorted c[0, 32)
  int pos = 0;
  #pragma unroll
  for (int step = 16; step > 0; step >>= 1)
    if (c[pos + step - 1] < k) pos += step;
  return pos + (c[pos] < k ? 1 : 0);  // pos = min(count, 31) here
}

__device__ __forceinline__ int count_below(const uint64_t* c, int n, uint64_t k) {  // sorted c[0, n)
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (c[mid] < k) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

__device__ void greedy_batched(int N, int first, int m, int Hkv, int tl, const int32_t* __restrict__ seq_lens,
                               const int32_t* sorted_b, const uint32_t* load_sm, int32_t* pcount_sm, uint8_t* area,
                               int32_t* part_bin, int32_t* part_pos) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* cur = reinterpret_cast<uint64_t*>(area);
  uint64_t* nxt = cur + N;
  uint64_t* Bn = nxt + N;
  uint64_t* wmin = Bn + kPlanThreads;
  int* sJ = reinterpret_cast<int*>(wmin + kPlanWarps);
  uint32_t* cost = reinterpret_cast<uint32_t*>(sJ + 4);
  const int rf = N - first;
  for (int s = first + tid; s < m; s += kPlanThreads) cost[s - first] = (uint32_t)(seq_lens[sorted_b[s / Hkv]] % tl);
  const uint32_t* c0 = load_sm + rf;  // the first batch's loads, non-increasing in s
  for (int s = tid; s < first; s += kPlanThreads) {
    const uint32_t c = c0[s];
    int lo = 0, hi = s;  // first index holding c
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (c0[mid] > c) lo = mid + 1;
      else hi = mid;
    }
    const int eq0 = lo;
    lo = s + 1;
    hi = first;  // first index below c
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (c0[mid] >= c) lo = mid + 1;
      else hi = mid;
    }
    cur[(first - lo) + (s - eq0)] = ((uint64_t)c << 32) | (uint32_t)(rf + s);
  }
  for (int k = tid; k < rf; k += kPlanThreads) cur[first + k] = ((uint64_t)load_sm[k] << 32) | (uint32_t)k;
  __syncthreads();
  for (int s = first; s < m;) {
    const int W = min(min(kPlanThreads, m - s), N);  // a round tries at most one tile per bin
    if (tid == 0) *sJ = W;
    const uint64_t a = tid < W ? cur[tid] : ~0ull;
    const uint64_t nw = tid < W ? a + ((uint64_t)cost[s - first + tid] << 32) : ~0ull;
    uint64_t x = nw;  // inclusive prefix minimum of the round's new keys
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x = min(x, y);
    }
    if (lane == 31) wmin[warp] = x;
    __syncthreads();
    uint64_t pm = ~0ull;
    for (int w = 0; w < warp; ++w) pm = min(pm, wmin[w]);
    const uint64_t up = __shfl_up_sync(0xffffffffu, x, 1);
    if (lane > 0) pm = min(pm, up);  // exclusive: the keys of tiles 0 .. tid-1
    if (tid < W && !(a < pm)) atomicMin(sJ, tid);
    __syncthreads();
    const int J = *sJ;  // >= 1: tile 0 always qualifies
    uint64_t key = ~0ull;
    if (tid < J) {
      const int bin = (int)(uint32_t)a;
      part_bin[s + tid] = bin;
      part_pos[s + tid] = pcount_sm[bin];
      pcount_sm[bin] += 1;  // the round's bins are distinct
      key = nw;
    }
    #pragma unroll
    for (int k = 2; k <= 32; k <<= 1)  // sort the warp's chunk, ascending (~0 pads last)
      #pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const uint64_t other = __shfl_xor_sync(0xffffffffu, key, j);
        key = (((lane & j) == 0) == ((lane & k) == 0)) ? min(key, other) : max(key, other);
      }
    Bn[tid] = key;
    __syncthreads();
    const int nc = (J + 31) >> 5;
    if (key != ~0ull) {
      int r = lane + count_below(cur + J, N - J, key);
      #pragma unroll
      for (int c = 0; c < kPlanWarps; ++c)
        if (c < nc && c != warp) r += count_below32(Bn + 32 * c, key);
      nxt[r] = key;
    }
    for (int i = J + tid; i < N; i += kPlanThreads) {
      const uint64_t xo = cur[i];
      int r = i - J;
      #pragma unroll
      for (int c = 0; c < kPlanWarps; ++c)
        if (c < nc) r += count_below32(Bn + 32 * c, xo);
      nxt[r] = xo;
    }
    __syncthreads();
    uint64_t* t = cur;
    cur = nxt;
    nxt = t;
    s += J;
  }
}

// Same rule with the loads in shared memory (more bins than the register version holds).
__device__ void greedy_partials_smem(int lane, int N, int first, int m, int Hkv, int tl,
                                     const int32_t* __restrict__ seq_lens, const int32_t* sorted_b, uint32_t* load_sm,
                                     int32_t* pcount_sm, int32_t* part_bin, int32_t* part_pos) {
  const int K = (N + 31) / 32;
  const int k0 = lane * K, k1 = min(N, k0 + K);
  uint32_t lmin = 0x07ffffffu;
  int lk = k0;
  for (int k = k0; k < k1; ++k)
    if (load_sm[k] < lmin) { lmin = load_sm[k]; lk = k; }
  for (int s0 = first; s0 < m; s0 += 32) {
    const int sl = s0 + lane;
    const uint32_t cl = sl < m ? (uint32_t)(seq_lens[sorted_b[sl / Hkv]] % tl) : 0u;
    const int n_here = min(32, m - s0);
    for (int i = 0; i < n_here; ++i) {
      const uint32_t c = __shfl_sync(0xffffffffu, cl, i);
      const uint32_t key = __reduce_min_sync(0xffffffffu, (lmin << 5) | (uint32_t)lane);
      if ((int)(key & 31u) == lane) {
        const int s = s0 + i;
        part_bin[s] = lk;
        part_pos[s] = pcount_sm[lk]++;
        load_sm[lk] += c;
        lmin = 0x07ffffffu;
        for (int k = k0; k < k1; ++k)
          if (load_sm[k] < lmin) { lmin = load_sm[k]; lk = k; }
      }
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t* __restrict__ seq_lens, const PlanHeader init, char* __restrict__ plan) {
  // Launched with programmatic serialisation: wait until the previous kernel of the stream has
  // finished (seq_lens, and the inputs the split kernel reads before its own wait, are final),
  // then let the split kernel start: it streams the full tiles, which need no plan, and waits
  // for this grid before reading the plan.
  griddep_wait();
  griddep_launch_dependents();
  const int B = init.batch, Hkv = init.n_kv_heads, tl = init.tile_len, N = init.n_bins;
  extern __shared__ __align__(16) uint8_t plan_smem[];
  uint32_t* load = reinterpret_cast<uint32_t*>(plan_smem);                   // [N] load above the full-tile base
  int32_t* pcount = reinterpret_cast<int32_t*>(plan_smem + 4 * (int64_t)N);  // [N] partial tiles per bin
  __shared__ Tri warp_tot[kPlanWarps];
  __shared__ int32_t sh_status;

  PlanHeader* hdr = reinterpret_cast<PlanHeader*>(plan);
  int32_t* gS = reinterpret_cast<int32_t*>(plan + init.off_S);
  int32_t* gSF = reinterpret_cast<int32_t*>(plan + init.off_SF);
  int32_t* gcb = reinterpret_cast<int32_t*>(plan + init.off_cb);
  int32_t* gsorted = reinterpret_cast<int32_t*>(plan + init.off_sorted);
  int32_t* gpbo = reinterpret_cast<int32_t*>(plan + init.off_pbin_off);
  int32_t* gplist = reinterpret_cast<int32_t*>(plan + init.off_plist);
  char* gscratch = plan + init.off_scratch;
  const bool req_in_smem = B <= kPlanSmemRequests;
  ReqArrays R = carve_req(req_in_smem ? reinterpret_cast<char*>(plan_smem + plan_bins_smem(N)) : gscratch, B);
  if (!req_in_smem) { R.S = gS; R.SF = gSF; R.sorted_b = gsorted; }
  int32_t* part_bin = reinterpret_cast<int32_t*>(gscratch + req_arrays_bytes(B));
  int32_t* part_pos = part_bin + align_up((int64_t)B * Hkv, 8);
  const int tid = threadIdx.x;
  if (tid == 0) {
    sh_status = 0;
    PlanHeader h = init;
    h.magic = 0;  // published last, once the plan is complete
    h.run_status = 0;
    *hdr = h;
  }

  // ---- 1. per-request tile counts and their prefix sums
  // (d: combine chunks per query row of the request, see combine_chunks())
  Tri carry{0, 0, 0, 0};
  for (int base = 0; base < B; base += kPlanThreads) {
    const int b = base + tid;
    int64_t L = b < B ? seq_lens[b] : 0;
    if (L < 0) { atomicCAS(&sh_status, 0, DECATTN_EDEVICE); L = 0; }
    const int64_t nb = (L + tl - 1) / tl;
    Tri v{nb, L / tl, (L % tl) != 0, b < B ? combine_chunks(nb) : 0};
    Tri before = carry;
    Tri ex = block_exscan(v, carry, warp_tot);
    if (b < B) {
      gcb[b] = (int32_t)(before.d + ex.d);
      R.S[b] = (int32_t)(before.a + ex.a);
      R.SF[b] = (int32_t)(before.b + ex.b);
      R.SP[b] = before.c + ex.c;
      if (v.c) { R.plist[before.c + ex.c] = b; R.pcost[before.c + ex.c] = (int32_t)(L % tl); }
    }
  }
  if (tid == 0) { R.S[B] = (int32_t)carry.a; R.SF[B] = (int32_t)carry.b; R.SP[B] = carry.c; gcb[B] = (int32_t)carry.d; }
  const int64_t U64 = (int64_t)Hkv * carry.a;
  __syncthreads();
  if (U64 > init.max_units) atomicCAS(&sh_status, 0, DECATTN_ECAPACITY);
  __syncthreads();
  if (sh_status != 0) {
    if (tid == 0) {
      hdr->n_units = 0;
      hdr->status = sh_status;
      __threadfence();
      hdr->magic = kPlanMagic;
    }
    return;
  }
  const int U = (int)U64;  // < 2^31 from here on: the capacity is checked against that on the host
  const int F = (int)((int64_t)Hkv * carry.b);
  const int mB = carry.c;
  const int m = Hkv * mB;

  // ---- 3. requests with a partial tile, sorted by cost (desc), then b: rank by counting
  for (int j = tid; j < mB; j += kPlanThreads) {
    const int cj = R.pcost[j];
    int rank = 0;
    for (int k = 0; k < mB; ++k) {
      const int c = R.pcost[k];
      rank += (c > cj) | ((c == cj) & (k < j));
    }
    R.sorted_b[rank] = R.plist[j];
  }
  __syncthreads();

  // ---- 4. greedy placement of the partial tiles (s-th in sorted order: request
  //         sorted_b[s / Hkv], head s % Hkv)
  const int qf = F / N;
  const int rf = F - qf * N;
  const int first = min(m, N - rf);
  for (int k = tid; k < N; k += kPlanThreads) {
    uint32_t l = k < rf ? (uint32_t)tl : 0u;
    int32_t pc = 0;
    const int s = k - rf;
    if (k >= rf && s < first) {
      l += (uint32_t)(seq_lens[R.sorted_b[s / Hkv]] % tl);
      pc = 1;
      part_bin[s] = k;
      part_pos[s] = 0;
    }
    load[k] = l;
    pcount[k] = pc;
  }
  __syncthreads();
  if (first < m && init.gsm_off > 0) {
    greedy_batched(N, first, m, Hkv, tl, seq_lens, R.sorted_b, load, pcount, plan_smem + init.gsm_off, part_bin,
                   part_pos);
  } else if (tid < 32 && first < m) {
    const int K = (N + 31) / 32;
#define DECATTN_GREEDY(KM) \
  greedy_partials<KM>(tid, N, first, m, Hkv, tl, seq_lens, R.sorted_b, load, pcount, part_bin, part_pos)
    if (K <= 4) DECATTN_GREEDY(4);
    else if (K <= 8) DECATTN_GREEDY(8);
    else if (K <= 12) DECATTN_GREEDY(12);
    else if (K <= 16) DECATTN_GREEDY(16);
    else if (K <= 20) DECATTN_GREEDY(20);
    else if (K <= 24) DECATTN_GREEDY(24);
    else if (K <= 32) DECATTN_GREEDY(32);
    else greedy_partials_smem(tid, N, first, m, Hkv, tl, seq_lens, R.sorted_b, load, pcount, part_bin, part_pos);
#undef DECATTN_GREEDY
  }
  __syncthreads();

  // ---- 5. per-bin CSR offsets of the partial tiles, and the partial tiles bin by bin
  {
    Tri c2{0, 0, 0, 0};
    for (int base = 0; base < N; base += kPlanThreads) {
      const int k = base + tid;
      Tri before = c2;
      Tri ex = block_exscan(Tri{k < N ? pcount[k] : 0, 0, 0, 0}, c2, warp_tot);
      if (k < N) gpbo[k] = (int32_t)(before.a + ex.a);
    }
    if (tid == 0) gpbo[N] = (int32_t)c2.a;
  }
  __syncthreads();
  for (int s = tid; s < m; s += kPlanThreads) gplist[gpbo[part_bin[s]] + part_pos[s]] = s;

  // ---- 6. publish the per-request arrays the decoder reads
  if (req_in_smem) {
    for (int b = tid; b <= B; b += kPlanThreads) { gS[b] = R.S[b]; gSF[b] = R.SF[b]; }
    for (int j = tid; j < mB; j += kPlanThreads) gsorted[j] = R.sorted_b[j];
  }
  __syncthreads();
  if (tid == 0) {
    hdr->n_units = U;
    hdr->n_full = F;
    hdr->n_partial = m;
    hdr->full_q = qf;
    hdr->full_r = rf;
    hdr->status = DECATTN_OK;
    __threadfence();
    hdr->magic = kPlanMagic;
  }
}

// ------------------------------------------------------------------ block-sparse planner
// "HPC-Ops ...", "How the kernels are organized around specific workload shapes": sparse
// attention takes a precomputed block mask and skips the masked-out KV tiles. The same greedy
// rule runs over the kept tiles only; each (request, KV head) pair p = b * Hkv + h keeps its
// own tiles (bit i % 32 of word i / 32 of mask row p keeps tile i; tiles past the row's
// mask_words words count as masked), so the plan's per-request arrays become per-pair ones
// (see plan_unit_sparse() in common.cuh).
__host__ __device__ inline int64_t plan_sparse_scratch_bytes(int B, int Hkv) {
  return 4 * align_up(4 * ((int64_t)B + 1), 32) + 3 * align_up(4 * ((int64_t)B * Hkv + 1), 32);
}

__device__ __forceinline__ uint32_t bits_below(int64_t n) {  // tiles [0, n) of a 32-tile word
  return n >= 32 ? 0xffffffffu : n <= 0 ? 0u : (1u << n) - 1u;
}

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_sparse_kernel(const int32_t* __restrict__ seq_lens, const uint32_t* __restrict__ mask, int W,
                   const PlanHeader init, char* __restrict__ plan) {
  griddep_wait();  // as the dense planner: inputs from the previous kernel are final
  griddep_launch_dependents();
  const int B = init.batch, Hkv = init.n_kv_heads, tl = init.tile_len, N = init.n_bins;
  const int P = B * Hkv;
  extern __shared__ __align__(16) uint8_t plan_smem[];
  uint32_t* load = reinterpret_cast<uint32_t*>(plan_smem);                   // [N] load above the full-tile base
  int32_t* pcount = reinterpret_cast<int32_t*>(plan_smem + 4 * (int64_t)N);  // [N] partial tiles per bin
  __shared__ Tri warp_tot[kPlanWarps];
  __shared__ int32_t sh_status;

  PlanHeader* hdr = reinterpret_cast<PlanHeader*>(plan);
  int32_t* PS = reinterpret_cast<int32_t*>(plan + init.off_S);
  int32_t* PF = reinterpret_cast<int32_t*>(plan + init.off_SF);
  int32_t* CBP = reinterpret_cast<int32_t*>(plan + init.off_cb);
  int32_t* spairs = reinterpret_cast<int32_t*>(plan + init.off_sorted);
  int32_t* gpbo = reinterpret_cast<int32_t*>(plan + init.off_pbin_off);
  int32_t* gplist = reinterpret_cast<int32_t*>(plan + init.off_plist);
  int32_t* KL = reinterpret_cast<int32_t*>(plan + init.off_kl);
  char* scr = plan + init.off_scratch;
  const int64_t rs = align_up(4 * ((int64_t)B + 1), 32), ps = align_up(4 * ((int64_t)P + 1), 32);
  int32_t* rq_list = reinterpret_cast<int32_t*>(scr);           // requests with a partial tile, b order
  int32_t* rq_cost = reinterpret_cast<int32_t*>(scr + rs);      // their partial-tile cost
  int32_t* rq_sorted = reinterpret_cast<int32_t*>(scr + 2 * rs);  // by cost (desc), then b
  int32_t* sb = reinterpret_cast<int32_t*>(scr + 4 * rs);       // [m] request of sorted partial pair s
  int32_t* part_bin = reinterpret_cast<int32_t*>(scr + 4 * rs + ps);
  int32_t* part_pos = reinterpret_cast<int32_t*>(scr + 4 * rs + 2 * ps);
  const int tid = threadIdx.x;
  if (tid == 0) {
    sh_status = 0;
    PlanHeader h = init;
    h.magic = 0;  // published last, once the plan is complete
    h.run_status = 0;
    *hdr = h;
  }

  // ---- 1. per pair: kept tiles (a), kept full tiles (b), kept partial tile (c), combine chunks (d);
  //         then the pair's kept-tile list KL[PS[p] + j] = index of its j-th kept tile. The
  //         first kPlanRegWords mask words stay in registers between the two (loads in flight
  //         together); a pair whose list would pass max_units is not listed (the plan fails).
  Tri carry{0, 0, 0, 0};
  for (int base = 0; base < P; base += kPlanThreads) {
    const int p = base + tid;
    Tri v{0, 0, 0, 0};
    uint32_t wr[kPlanRegWords];
    int64_t nb = 0, nw = 0;
    const uint32_t* row = mask + (int64_t)p * W;
    if (p < P) {
      int64_t L = seq_lens[p / Hkv];
      if (L < 0) { atomicCAS(&sh_status, 0, DECATTN_EDEVICE); L = 0; }
      nb = (L + tl - 1) / tl;
      const int64_t nf = L / tl;
      nw = min((nb + 31) / 32, (int64_t)W);
      #pragma unroll
      for (int w = 0; w < kPlanRegWords; ++w) wr[w] = w < nw ? __ldg(row + w) & bits_below(nb - 32 * w) : 0u;
      long long kept = 0, keptf = 0;
      #pragma unroll
      for (int w = 0; w < kPlanRegWords; ++w) {
        kept += __popc(wr[w]);
        keptf += __popc(wr[w] & bits_below(nf - 32 * w));
      }
      for (int64_t w = kPlanRegWords; w < nw; ++w) {
        const uint32_t word = __ldg(row + w);
        kept += __popc(word & bits_below(nb - 32 * w));
        keptf += __popc(word & bits_below(nf - 32 * w));
      }
      v = Tri{kept, keptf, (int)(kept - keptf), combine_chunks(kept)};  // the partial tile is the only non-full one
    }
    Tri before = carry;
    Tri ex = block_exscan(v, carry, warp_tot);
    if (p < P) {
      const long long o0 = before.a + ex.a;
      PS[p] = (int32_t)o0;
      PF[p] = (int32_t)(before.b + ex.b);
      CBP[p] = (int32_t)(before.d + ex.d);
      if (o0 + v.a <= init.max_units) {
        int o = (int)o0;
        #pragma unroll
        for (int w = 0; w < kPlanRegWords; ++w) {
          uint32_t word = wr[w];
          while (word) {
            KL[o++] = (int32_t)(32 * w + __ffs(word) - 1);
            word &= word - 1u;
          }
        }
        for (int64_t w = kPlanRegWords; w < nw; ++w) {
          uint32_t word = __ldg(row + w) & bits_below(nb - 32 * w);
          while (word) {
            KL[o++] = (int32_t)(32 * w + __ffs(word) - 1);
            word &= word - 1u;
          }
        }
      }
    }
  }
  if (tid == 0) { PS[P] = (int32_t)carry.a; PF[P] = (int32_t)carry.b; CBP[P] = (int32_t)carry.d; }
  const int64_t U64 = carry.a;
  __syncthreads();
  if (U64 > init.max_units) atomicCAS(&sh_status, 0, DECATTN_ECAPACITY);
  __syncthreads();
  if (sh_status != 0) {
    if (tid == 0) {
      hdr->n_units = 0;
      hdr->status = sh_status;
      __threadfence();
      hdr->magic = kPlanMagic;
    }
    return;
  }
  const int U = (int)U64;
  const int F = (int)carry.b;
  const int m = carry.c;

  // ---- 3. requests with a partial tile by cost (desc), then b; then, in that order, their
  //         pairs whose partial tile is kept (pair order within a request)
  Tri c2{0, 0, 0, 0};
  for (int base = 0; base < B; base += kPlanThreads) {
    const int b = base + tid;
    const int64_t L = b < B ? seq_lens[b] : 0;
    const int has = b < B && L > 0 && (L % tl) != 0;
    Tri before = c2;
    Tri ex = block_exscan(Tri{has, 0, 0, 0}, c2, warp_tot);
    if (has) {
      rq_list[before.a + ex.a] = b;
      rq_cost[before.a + ex.a] = (int32_t)(L % tl);
    }
  }
  const int mB = (int)c2.a;
  __syncthreads();
  for (int j = tid; j < mB; j += kPlanThreads) {
    const int cj = rq_cost[j];
    int rank = 0;
    for (int k = 0; k < mB; ++k) {
      const int c = rq_cost[k];
      rank += (c > cj) | ((c == cj) & (k < j));
    }
    rq_sorted[rank] = rq_list[j];
  }
  __syncthreads();
  Tri c3{0, 0, 0, 0};
  for (int base = 0; base < mB; base += kPlanThreads) {
    const int i = base + tid;
    int b = 0, last = 0;
    long long cnt = 0;
    if (i < mB) {
      b = rq_sorted[i];
      last = (int)((seq_lens[b] + tl - 1) / tl) - 1;  // the partial tile
      for (int h = 0; h < Hkv; ++h)
        if (last / 32 < W) cnt += (mask[((int64_t)b * Hkv + h) * W + last / 32] >> (last % 32)) & 1u;
    }
    Tri before = c3;
    Tri ex = block_exscan(Tri{cnt, 0, 0, 0}, c3, warp_tot);
    if (i < mB) {
      int o = (int)(before.a + ex.a);
      for (int h = 0; h < Hkv; ++h)
        if (last / 32 < W && ((mask[((int64_t)b * Hkv + h) * W + last / 32] >> (last % 32)) & 1u)) {
          spairs[o] = b * Hkv + h;
          sb[o] = b;
          ++o;
        }
    }
  }
  __syncthreads();

  // ---- 4. greedy placement of the kept partial tiles (s-th in sorted order: pair spairs[s])
  const int qf = F / N;
  const int rf = F - qf * N;
  const int first = min(m, N - rf);
  for (int k = tid; k < N; k += kPlanThreads) {
    uint32_t l = k < rf ? (uint32_t)tl : 0u;
    int32_t pc = 0;
    const int s = k - rf;
    if (k >= rf && s < first) {
      l += (uint32_t)(seq_lens[sb[s]] % tl);
      pc = 1;
      part_bin[s] = k;
      part_pos[s] = 0;
    }
    load[k] = l;
    pcount[k] = pc;
  }
  __syncthreads();
  if (first < m && init.gsm_off > 0) {
    greedy_batched(N, first, m, 1, tl, seq_lens, sb, load, pcount, plan_smem + init.gsm_off, part_bin, part_pos);
  } else if (tid < 32 && first < m) {
    const int K = (N + 31) / 32;
#define DECATTN_GREEDY(KM) greedy_partials<KM>(tid, N, first, m, 1, tl, seq_lens, sb, load, pcount, part_bin, part_pos)
    if (K <= 4) DECATTN_GREEDY(4);
    else if (K <= 8) DECATTN_GREEDY(8);
    else if (K <= 12) DECATTN_GREEDY(12);
    else if (K <= 16) DECATTN_GREEDY(16);
    else if (K <= 20) DECATTN_GREEDY(20);
    else if (K <= 24) DECATTN_GREEDY(24);
    else if (K <= 32) DECATTN_GREEDY(32);
    else greedy_partials_smem(tid, N, first, m, 1, tl, seq_lens, sb, load, pcount, part_bin, part_pos);
#undef DECATTN_GREEDY
  }
  __syncthreads();

  // ---- 5. per-bin CSR offsets of the partial tiles, and the partial tiles bin by bin
  {
    Tri c4{0, 0, 0, 0};
    for (int base = 0; base < N; base += kPlanThreads) {
      const int k = base + tid;
      Tri before = c4;
      Tri ex = block_exscan(Tri{k < N ? pcount[k] : 0, 0, 0, 0}, c4, warp_tot);
      if (k < N) gpbo[k] = (int32_t)(before.a + ex.a);
    }
    if (tid == 0) gpbo[N] = (int32_t)c4.a;
  }
  __syncthreads();
  for (int s = tid; s < m; s += kPlanThreads) gplist[gpbo[part_bin[s]] + part_pos[s]] = s;
  __syncthreads();
  if (tid == 0) {
    hdr->n_units = U;
    hdr->n_full = F;
    hdr->n_partial = m;
    hdr->full_q = qf;
    hdr->full_r = rf;
    hdr->status = DECATTN_OK;
    __threadfence();
    hdr->magic = kPlanMagic;
  }
}

// Writes the explicit work list of a finished plan: bin_off [N+1] and units [U] (CSR by
// bin), decoded with the same plan_unit() the split kernel uses. One block; for tests and
// diagnostics.
__global__ void __launch_bounds__(1024)
plan_export_kernel(const char* __restrict__ plan, const int32_t* __restrict__ seq_lens, int32_t* bin_off,
                   Unit* units, int64_t max_units, int32_t* n_out) {
  const PlanHeader h = *reinterpret_cast<const PlanHeader*>(plan);
  __shared__ long long carry;
  __shared__ long long part[1024];
  const bool ok = h.magic == kPlanMagic && h.status == DECATTN_OK && h.n_units <= max_units;
  if (threadIdx.x == 0) { carry = 0; *n_out = ok ? h.n_units : -1; }
  __syncthreads();
  if (!ok) return;
  for (int base = 0; base < h.n_bins; base += 1024) {
    const int k = base + threadIdx.x;
    part[threadIdx.x] = k < h.n_bins ? plan_bin_size(plan, h, k) : 0;
    __syncthreads();
    if (threadIdx.x == 0) {
      long long run = carry;
      for (int i = 0; i < 1024; ++i) { const long long v = part[i]; part[i] = run; run += v; }
      carry = run;
    }
    __syncthreads();
    if (k < h.n_bins) {
      bin_off[k] = (int32_t)part[threadIdx.x];
      const int n = plan_bin_size(plan, h, k);
      for (int j = 0; j < n; ++j)
        units[part[threadIdx.x] + j] = h.sparse ? plan_unit_sparse(plan, h, seq_lens, k, j)
                                                : plan_unit(plan, h, seq_lens, k, j);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) bin_off[h.n_bins] = (int32_t)carry;
}

// ------------------------------------------------------------------ host side
struct PlanLayout {
  int64_t off_S, off_SF, off_cb, off_sorted, off_pbin_off, off_plist, off_scratch, total;
};

static PlanLayout plan_layout(int B, int Hkv, int N) {
  PlanLayout L;
  int64_t o = sizeof(PlanHeader);
  L.off_S = o; o = align_up(o + 4 * ((int64_t)B + 1), 32);
  L.off_SF = o; o = align_up(o + 4 * ((int64_t)B + 1), 32);
  L.off_cb = o; o = align_up(o + 4 * ((int64_t)B + 1), 32);
  L.off_sorted = o; o = align_up(o + 4 * ((int64_t)B + 1), 32);
  L.off_pbin_off = o; o = align_up(o + 4 * ((int64_t)N + 1), 32);
  L.off_plist = o; o = align_up(o + 4 * ((int64_t)B * Hkv + 1), 32);
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
  if ((int64_t)B * Hkv >= (1ll << 28)) return false;
  if (plan_layout(B, Hkv, N).total >= (1ll << 31)) return false;
  // keeps every relative bin load of the greedy pass below 2^27 (its packed min key)
  if ((double)B * Hkv * tl / N + 2.0 * tl >= 134217727.0) return false;
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
  return (size_t)plan_layout(batch, n_kv_heads, n_bins).total;
}

extern "C" int dec_attn_plan(const int32_t* seq_lens, int batch, int n_kv_heads, int tile_len,
                             int64_t max_total_kv_tokens, int n_bins, void* plan_buf, size_t plan_bytes,
                             dec_attn_plan_t* plan, void* stream) {
  if (!plan || !plan_buf || (batch > 0 && !seq_lens)) return DECATTN_EINVAL;
  if (n_bins == 0) {
    int dev = 0;
    if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    n_bins = default_bins(dev);
    if (n_bins <= 0) return cuda_fail("SM count (cudaDeviceGetAttribute)");
  }
  if (batch < 0 || n_kv_heads <= 0 || tile_len <= 0 || max_total_kv_tokens < 0 || n_bins < 0) return DECATTN_EINVAL;
  if (!plan_args_ok(batch, n_kv_heads, tile_len, max_total_kv_tokens, n_bins)) return DECATTN_ENOTSUP;
  if ((reinterpret_cast<uintptr_t>(plan_buf) & 15) != 0) return DECATTN_EALIGN;
  const int64_t cap = plan_capacity(batch, n_kv_heads, tile_len, max_total_kv_tokens);
  const PlanLayout L = plan_layout(batch, n_kv_heads, n_bins);
  if ((int64_t)plan_bytes < L.total) return DECATTN_ESMALL;

  PlanHeader h{};
  h.n_bins = n_bins;
  h.batch = batch;
  h.n_kv_heads = n_kv_heads;
  h.tile_len = tile_len;
  h.max_units = cap;
  h.off_S = (int32_t)L.off_S;
  h.off_SF = (int32_t)L.off_SF;
  h.off_cb = (int32_t)L.off_cb;
  h.off_sorted = (int32_t)L.off_sorted;
  h.off_pbin_off = (int32_t)L.off_pbin_off;
  h.off_plist = (int32_t)L.off_plist;
  h.off_scratch = (int32_t)L.off_scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t smem =
      (size_t)plan_bins_smem(n_bins) + (batch <= kPlanSmemRequests ? (size_t)req_arrays_bytes(batch) : 0);
  smem = (size_t)align_up((int64_t)smem, 16);
  const int64_t gsm = greedy_batched_bytes(n_bins, (int64_t)batch * n_kv_heads);
  if ((int64_t)smem + gsm <= kPlanMaxSmem) {  // room for the batched greedy pass
    h.gsm_off = (int32_t)smem;
    smem += (size_t)gsm;
  }
  if (!ensure_smem_attr((const void*)plan_kernel, kPlanMaxSmem)) return cuda_fail("planner shared-memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // launched while the previous kernel drains
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (const cudaError_t e = cudaLaunchKernelEx(&cfg, plan_kernel, seq_lens, h, static_cast<char*>(plan_buf));
      e != cudaSuccess)
    return cuda_fail("planner launch", e);
  plan->buf = plan_buf;
  plan->buf_bytes = plan_bytes;
  plan->batch = batch;
  plan->n_kv_heads = n_kv_heads;
  plan->tile_len = tile_len;
  plan->n_bins = n_bins;
  plan->max_units = cap;
  plan->sparse = 0;
  return DECATTN_OK;
}

extern "C" int dec_attn_plan_export(const dec_attn_plan_t* plan, const int32_t* seq_lens, int32_t* bin_off,
                                    void* units, int64_t max_units, int32_t* n_units, void* stream) {
  if (!plan || !plan->buf || !bin_off || !units || !n_units || (plan->batch > 0 && !seq_lens) || max_units < 0)
    return DECATTN_EINVAL;
  plan_export_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const char*>(plan->buf), seq_lens, bin_off, static_cast<Unit*>(units), max_units, n_units);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DECATTN_OK : cuda_fail("plan export launch", e);
}

// ------------------------------------------------------------------ block-sparse plan (host)
namespace decattn {

struct SparseLayout {
  int64_t off_PS, off_PF, off_CBP, off_sp, off_pbo, off_pl, off_kl, off_scratch, total;
};

static SparseLayout plan_sparse_layout(int B, int Hkv, int N, int64_t cap) {
  const int64_t P = (int64_t)B * Hkv;
  SparseLayout L;
  int64_t o = sizeof(PlanHeader);
  L.off_PS = o; o = align_up(o + 4 * (P + 1), 32);
  L.off_PF = o; o = align_up(o + 4 * (P + 1), 32);
  L.off_CBP = o; o = align_up(o + 4 * (P + 1), 32);
  L.off_sp = o; o = align_up(o + 4 * (P + 1), 32);
  L.off_pbo = o; o = align_up(o + 4 * ((int64_t)N + 1), 32);
  L.off_pl = o; o = align_up(o + 4 * (P + 1), 32);
  L.off_kl = o; o = align_up(o + 4 * (cap + 1), 32);
  L.off_scratch = o; o = align_up(o + plan_sparse_scratch_bytes(B, Hkv), 32);
  L.total = o;
  return L;
}

}  // namespace decattn

extern "C" size_t dec_attn_plan_sparse_bytes(int batch, int n_kv_heads, int tile_len, int64_t max_total_kv_tokens,
                                              int n_bins) {
  if (n_bins == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    n_bins = default_bins(dev);
  }
  if (!plan_args_ok(batch, n_kv_heads, tile_len, max_total_kv_tokens, n_bins)) return 0;
  const SparseLayout L = plan_sparse_layout(batch, n_kv_heads, n_bins,
                                            plan_capacity(batch, n_kv_heads, tile_len, max_total_kv_tokens));
  return L.total >= (1ll << 31) ? 0 : (size_t)L.total;
}

extern "C" int dec_attn_plan_sparse(const int32_t* seq_lens, const uint32_t* tile_mask, int mask_words, int batch,
                                    int n_kv_heads, int tile_len, int64_t max_total_kv_tokens, int n_bins,
                                    void* plan_buf, size_t plan_bytes, dec_attn_plan_t* plan, void* stream) {
  if (!plan || !plan_buf || (batch > 0 && (!seq_lens || !tile_mask)) || mask_words <= 0) return DECATTN_EINVAL;
  if (n_bins == 0) {
    int dev = 0;
    if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    n_bins = default_bins(dev);
    if (n_bins <= 0) return cuda_fail("SM count (cudaDeviceGetAttribute)");
  }
  if (batch < 0 || n_kv_heads <= 0 || tile_len <= 0 || max_total_kv_tokens < 0 || n_bins < 0) return DECATTN_EINVAL;
  if (!plan_args_ok(batch, n_kv_heads, tile_len, max_total_kv_tokens, n_bins)) return DECATTN_ENOTSUP;
  if ((int64_t)batch * n_kv_heads * mask_words >= (1ll << 31)) return DECATTN_ENOTSUP;
  if ((reinterpret_cast<uintptr_t>(plan_buf) & 15) != 0 || (reinterpret_cast<uintptr_t>(tile_mask) & 3) != 0)
    return DECATTN_EALIGN;
  const int64_t cap = plan_capacity(batch, n_kv_heads, tile_len, max_total_kv_tokens);
  const SparseLayout L = plan_sparse_layout(batch, n_kv_heads, n_bins, cap);
  if (L.total >= (1ll << 31)) return DECATTN_ENOTSUP;
  if ((int64_t)plan_bytes < L.total) return DECATTN_ESMALL;

  PlanHeader h{};
  h.n_bins = n_bins;
  h.batch = batch;
  h.n_kv_heads = n_kv_heads;
  h.tile_len = tile_len;
  h.max_units = cap;
  h.off_S = (int32_t)L.off_PS;
  h.off_SF = (int32_t)L.off_PF;
  h.off_cb = (int32_t)L.off_CBP;
  h.off_sorted = (int32_t)L.off_sp;
  h.off_pbin_off = (int32_t)L.off_pbo;
  h.off_plist = (int32_t)L.off_pl;
  h.off_kl = (int32_t)L.off_kl;
  h.off_scratch = (int32_t)L.off_scratch;
  h.sparse = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t smem = (size_t)align_up(plan_bins_smem(n_bins), 16);
  const int64_t gsm = greedy_batched_bytes(n_bins, (int64_t)batch * n_kv_heads);
  if ((int64_t)smem + gsm <= kPlanMaxSmem) {  // room for the batched greedy pass
    h.gsm_off = (int32_t)smem;
    smem += (size_t)gsm;
  }
  if (!ensure_smem_attr((const void*)plan_sparse_kernel, kPlanMaxSmem)) return cuda_fail("sparse planner shared-memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // launched while the previous kernel drains
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (const cudaError_t e = cudaLaunchKernelEx(&cfg, plan_sparse_kernel, seq_lens, tile_mask, mask_words, h,
                                               static_cast<char*>(plan_buf));
      e != cudaSuccess)
    return cuda_fail("sparse planner launch", e);
  plan->buf = plan_buf;
  plan->buf_bytes = plan_bytes;
  plan->batch = batch;
  plan->n_kv_heads = n_kv_heads;
  plan->tile_len = tile_len;
  plan->n_bins = n_bins;
  plan->max_units = cap;
  plan->sparse = 1;
  return DECATTN_OK;
}
