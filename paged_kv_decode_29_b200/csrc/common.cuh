// common.cuh -- device helpers shared by the planner, split and combine kernels
// (sm_100a): mbarriers, TMA / bulk copies, ldmatrix, mma.sync, movmatrix,
// bounded waits and the plan-buffer layout.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/decattn.h"

namespace decattn {

// ------------------------------------------------------------------ plan layout
// The plan buffer starts with this header; the arrays follow at the byte offsets it
// records (multiples of 32). The work list is stored compactly:
//  * full tiles (cost tile_len) are dealt round-robin by the greedy rule, so bin k holds
//    full tiles f = k + n_bins * j for j < full_q + (k < full_r), with f counting the full
//    tiles in (b, h, i) order; (b, h, i) is recovered from the prefix array SF;
//  * after them, bin k holds the partial tiles plist[pbin_off[k] .. pbin_off[k + 1]) in
//    the order they were assigned; partial tile s is head s % Hkv of request
//    sorted[s / Hkv].
// plan_unit() decodes the j-th tile of bin k; it is the only reader of this encoding.
struct PlanHeader {
  int32_t magic;        // kPlanMagic once the planner kernel has written the plan
  int32_t status;       // DECATTN_OK or a negative device-detected status of the planner
  int32_t run_status;   // first device-detected error of a split kernel run on this plan (0 = none)
  int32_t n_bins;       // N: CTAs of the split kernel; bin k is run by CTA k
  int32_t batch;
  int32_t n_kv_heads;
  int32_t tile_len;
  int32_t n_units;      // U: tiles in the work list
  int32_t n_full;       // F: full tiles
  int32_t n_partial;    // m: partial tiles (at most one per (b, h))
  int32_t full_q;       // F / N
  int32_t full_r;       // F % N
  int64_t max_units;    // capacity (sizes the workspace's partial slots)
  int32_t off_S;        // int32 [batch + 1]: prefix over requests of n_b = ceil(L_b / tile_len)
  int32_t off_SF;       // int32 [batch + 1]: prefix over requests of full tiles floor(L_b / tile_len)
  int32_t off_cb;       // int32 [batch + 1]: prefix over requests of combine chunks per query row
  int32_t off_sorted;   // int32 [batch]: requests with a partial tile, by cost (desc), then b
  int32_t off_pbin_off; // int32 [n_bins + 1]: CSR offsets of each bin's partial tiles in plist
  int32_t off_plist;    // int32 [batch * n_kv_heads]: partial tiles, bin by bin
  int32_t off_scratch;  // planner scratch
  int32_t sparse;       // 1: block-sparse plan (per-pair arrays below, see plan_unit_sparse)
  int32_t off_kl;       // sparse: int32 [max_units]: tile index of kept tile j of pair p at PS[p] + j
  int32_t gsm_off;      // planner launch: offset of the batched greedy's shared-memory area (0: none)
  int32_t reserved[8];
};
static_assert(sizeof(PlanHeader) == 128, "plan header is 128 bytes");
constexpr int32_t kPlanMagic = 0x32504144;  // "DAP2"

// One tile of the work list.
struct Unit {
  int32_t b, h, tok_begin, tok_end, seq_len, slot, tile, zero;
};
static_assert(sizeof(Unit) == 32, "unit is 32 bytes");

__device__ __forceinline__ const int32_t* plan_arr(const char* plan, int32_t off) {
  return reinterpret_cast<const int32_t*>(plan + off);
}

// Number of tiles in bin k.
__device__ __forceinline__ int plan_bin_size(const char* plan, const PlanHeader& h, int k) {
  const int32_t* pbo = plan_arr(plan, h.off_pbin_off);
  return h.full_q + (k < h.full_r) + pbo[k + 1] - pbo[k];
}

// The j-th tile of bin k (j < plan_bin_size). A tile of a pair with several tiles writes
// partial slot S-prefix * Hkv + h * n_b + i; a pair held in one tile gets slot -1.
__device__ __forceinline__ Unit plan_unit(const char* plan, const PlanHeader& h, const int32_t* seq_lens, int k,
                                          int j) {
  const int32_t* S = plan_arr(plan, h.off_S);
  const int32_t* SF = plan_arr(plan, h.off_SF);
  const int N = h.n_bins, Hkv = h.n_kv_heads, tl = h.tile_len;
  const int fc = h.full_q + (k < h.full_r);
  int b, hh, i, end;
  if (j < fc) {
    const int f = k + N * j;
    int lo = 0, hi = h.batch - 1;  // last request b with Hkv * SF[b] <= f
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (Hkv * SF[mid] <= f) lo = mid; else hi = mid - 1;
    }
    b = lo;
    const int fb = SF[b + 1] - SF[b];
    const int r = f - Hkv * SF[b];
    hh = r / fb;
    i = r - hh * fb;
    end = (i + 1) * tl;
  } else {
    const int s = plan_arr(plan, h.off_plist)[plan_arr(plan, h.off_pbin_off)[k] + (j - fc)];
    b = plan_arr(plan, h.off_sorted)[s / Hkv];
    hh = s % Hkv;
    i = SF[b + 1] - SF[b];
    end = seq_lens[b];
  }
  const int nb = S[b + 1] - S[b];
  Unit u;
  u.b = b; u.h = hh; u.tok_begin = i * tl; u.tok_end = end; u.seq_len = seq_lens[b];
  u.slot = nb == 1 ? -1 : Hkv * S[b] + hh * nb + i;
  u.tile = i; u.zero = 0;
  return u;
}

// Block-sparse plans ("HPC-Ops ...", "How the kernels are organized around specific workload
// shapes": sparse attention skips the KV tiles a precomputed block mask masks out) index per
// (request, KV head) pair p = b * Hkv + h instead of per request, because each pair keeps its
// own tiles; the header offsets then mean:
//   off_S      PS  [P+1]: prefix over pairs of kept tiles (a pair's partial slots start at PS[p])
//   off_SF     PF  [P+1]: prefix over pairs of kept full tiles
//   off_cb     CBP [P+1]: prefix over pairs of combine chunks per query row
//   off_sorted      [P] : pairs whose partial tile is kept, by cost (desc), then pair index
//   off_kl     KL  [U]  : tile index of the pair's j-th kept tile at KL[PS[p] + j]
// Kept full tiles precede a pair's kept partial tile in tile order, so under the greedy rule
// kept full tile f (in (p, j) order) again sits in bin f mod N at position f div N.
__device__ __forceinline__ Unit plan_unit_sparse(const char* plan, const PlanHeader& h, const int32_t* seq_lens,
                                                 int k, int j) {
  const int32_t* PS = plan_arr(plan, h.off_S);
  const int32_t* PF = plan_arr(plan, h.off_SF);
  const int32_t* KL = plan_arr(plan, h.off_kl);
  const int N = h.n_bins, Hkv = h.n_kv_heads, tl = h.tile_len;
  const int fc = h.full_q + (k < h.full_r);
  int pr, kj;
  if (j < fc) {
    const int f = k + N * j;
    int lo = 0, hi = h.batch * Hkv - 1;  // last pair p with PF[p] <= f
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (PF[mid] <= f) lo = mid; else hi = mid - 1;
    }
    pr = lo;
    kj = f - PF[pr];
  } else {
    const int s = plan_arr(plan, h.off_plist)[plan_arr(plan, h.off_pbin_off)[k] + (j - fc)];
    pr = plan_arr(plan, h.off_sorted)[s];
    kj = PS[pr + 1] - PS[pr] - 1;  // the partial tile is the pair's last kept tile
  }
  const int b = pr / Hkv;
  const int m = PS[pr + 1] - PS[pr];
  const int i = KL[PS[pr] + kj];
  const int L = seq_lens[b];
  Unit u;
  u.b = b; u.h = pr - b * Hkv; u.tok_begin = i * tl; u.tok_end = min((i + 1) * tl, L); u.seq_len = L;
  u.slot = m == 1 ? -1 : PS[pr] + kj;
  u.tile = i; u.zero = 0;
  return u;
}

// Workspace: a status word, then partial outputs and their LSEs.
struct WorkspaceHeader {
  int32_t status;
  int32_t reserved[63];
};
static_assert(sizeof(WorkspaceHeader) == 256, "workspace header is 256 bytes");

// Arguments of the split kernel (one CTA per bin of the plan).
struct SplitParams {
  const uint16_t* q;        // bf16 [B][T][Hq][D]
  const int32_t* page_table;
  const int32_t* seq_lens;  // [B]
  const float* kv_scales;   // [2][num_pages][Hkv] or null
  const char* plan;
  float* out;               // [B][T][Hq][D]
  float* lse;               // [B][T][Hq]
  float* part_o;            // [max_units][GT][D]
  float* part_lse;          // [max_units][GT]
  int32_t* row_cnt;         // [B*T*Hq] combine counters, zeroed here for the combine that follows
  int32_t* status;          // run status word (plan header)
  int B, T, Hq, Hkv, G, GT, P, num_pages, mpps, n_bins;
  int tile_len;             // the plan's tile length
  int sparse;               // the plan is block-sparse (its tiles come from the plan only)
  int64_t max_units;        // the plan's capacity (partial slots of the workspace)
  float qk_scale_log2;      // sm_scale * log2(e)
  uint64_t wait_ns;         // a pipeline wait gives up after this long (kWaitLimitNs unless a test lowers it)
  int32_t skip_fill;        // tests only: CTA 0's producer leaves this ring fill out (-1: none)
};

// Arguments of the prefill kernel (prefill.cu). Query rows are packed: request b's Tb rows are
// rows qoff_b .. qoff_b + Tb - 1 of q [total_rows][Hq][D] (and of out / lse), with qoff_b = b T and
// Tb = T when cu_q is null (every request has T rows), else qoff_b = cu_q[b], Tb = cu_q[b+1] -
// cu_q[b] <= T (variable-length rows).
struct PrefillParams {
  const uint16_t* q;          // bf16 [total_rows][Hq][D]
  const int32_t* page_table;  // [B][mpps]
  const int32_t* seq_lens;    // [B]
  const int32_t* cu_q;        // [B + 1] row offsets, or null
  float* out;                 // [total_rows][Hq][D]
  float* lse;                 // [total_rows][Hq]
  int32_t* status;            // optional device word
  int B, T, Hq, Hkv, G, P, num_pages, mpps;
  int64_t total_rows;
  float qk_scale_log2;        // sm_scale * log2(e)
  uint64_t wait_ns;           // a pipeline wait gives up after this long
  int32_t skip_fill;          // tests only: CTA 0's producer leaves this K block out (-1: none)
};

// FP8 prefill: the E4M3 pages each request uses, widened to a bf16 scratch pool (prefill_fp8.cu).
struct WidenParams {
  const uint8_t* k_codes;     // E4M3 [num_pages][Hkv][P][D]
  const uint8_t* v_codes;
  const float* kv_scales;     // [2][num_pages][Hkv]: K, then V
  const int32_t* page_table;  // [B][mpps]
  const int32_t* seq_lens;    // [B]
  uint16_t* k_out;            // bf16 [B * mpps][Hkv][P][D]: page i of request b at b * mpps + i
  uint16_t* v_out;
  int32_t* pt_out;            // [B][mpps]: b * mpps + i
  int32_t* status;            // optional device word
  int B, Hkv, P, D, num_pages, mpps;
};

// Query rows of one KV head that a decode tile computes at once (G * T), and query tokens per
// request (T), that dec_attn_run supports.
constexpr int kMaxGT = 64;
constexpr int kMaxT = 8;

// The combine kernel folds the partials of one query row in chunks of this many tiles.
// A request with n_b tiles gives each of its rows cb_b = ceil(n_b / kCombineChunk) chunks
// (1 if n_b == 0: the row is zero-filled; 0 if n_b == 1: the split kernel wrote the row).
constexpr int kCombineChunk = 32;

__host__ __device__ inline int combine_chunks(int64_t n_b) {
  return n_b == 0 ? 1 : n_b == 1 ? 0 : (int)((n_b + kCombineChunk - 1) / kCombineChunk);
}

// Arguments of the combine kernel (persistent; warps walk the (row, chunk) items).
struct CombineParams {
  const char* plan;
  const int32_t* seq_lens;
  const float* part_o;
  const float* part_lse;
  float* out;
  float* lse;
  int32_t* row_cnt;         // [B*T*Hq] chunks of the row folded so far (zeroed by the split kernel)
  float* chunk_state;       // [items][D + 4]: max, weight, -, -, then the weighted sum
  int B, T, Hq, Hkv, G, GT, D, tl;
  int sparse;               // block-sparse plan: chunks are counted per (request, KV head) pair
};

__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ status
__device__ __forceinline__ void set_status(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// Programmatic dependent launch: let the next kernel of the stream start its prologue
// early / wait until the previous kernel has completed and its writes are visible.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// A pipeline wait gives up after this long; a healthy pipeline waits microseconds.
constexpr uint64_t kWaitLimitNs = 2000ull * 1000 * 1000;

// ------------------------------------------------------------------ shared-memory addresses
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Returns false (after setting
// DECATTN_ETIMEOUT) if it has not completed within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    #pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      set_status(status, DECATTN_ETIMEOUT);
      return false;
    }
  }
}

// Lane 0 waits and tells the rest of the warp (used where only lane 0 touches the staged
// data afterwards, e.g. the thread that issues the next copy into a freed stage).
__device__ __forceinline__ bool warp_wait_lane0(uint64_t* bar, uint32_t parity, int32_t* status,
                                                uint64_t limit_ns = kWaitLimitNs) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status, limit_ns) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ------------------------------------------------------------------ async copies
// 2-D tiled TMA load into shared memory, completion signalled on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Plain bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 4-byte asynchronous copy global -> shared (LDGSTS) ...
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// ... whose completion is folded into an mbarrier phase: the pending count is raised now
// and lowered when this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ warp-level matrix ops
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D (16x8 fp32) += A (16x16) * B (16x8); bf16 or f16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (16x8 fp32) += A (16x32 E4M3) * B (32x8 E4M3); each register holds 4 codes along k.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats -> two E4M3 codes (low byte from lo), round to nearest even, saturating at +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t v) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = v;
  return __half22float2(h);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two OCP E4M3 codes (low byte -> low half) -> f16x2 with the same values (every finite
// E4M3 value is exact in f16). CUDA's conversion, one hardware convert on sm_89 and later.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two fp32 lanes in one instruction (fma.rn.f32x2 / mul.rn.f32x2 / add.rn.f32x2, sm_100): (d0, d1) =
// (a0 b0 + c0, a1 b1 + c1), each rounded once as fmaf would; (a0 b0, a1 b1); and (a0 + b0, a1 + b1).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// ------------------------------------------------------------------ host-side launchers
// Wait limit and left-out fill for the next launches (api.cu; tests of the bounded waits).
void test_waits(uint64_t* wait_ns, int32_t* skip_fill);
int default_bins(int device);                                     // api.cu
bool ensure_smem_attr(const void* kernel, int bytes);             // api.cu
bool split_supported(int kv_dtype, int D, int GT);                // split.cu
cudaError_t launch_split(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int kv_dtype,
                         int D, cudaStream_t st);                 // split.cu
int split_ctas_per_sm();                                          // split.cu
bool split_tc_supported(int kv_dtype, int D, int GT);             // split_tc.cu
cudaError_t launch_split_tc(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int kv_dtype,
                            cudaStream_t st);                     // split_tc.cu
cudaError_t launch_combine(const CombineParams& p, int device, cudaStream_t st);  // combine.cu
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t st);  // prefill.cu
// bytes of the widened pool (K, then V at *off_v, then the page table at *off_pt)   prefill_fp8.cu
int64_t widen_scratch_bytes(int B, int mpps, int Hkv, int P, int D, int64_t* off_v, int64_t* off_pt);
cudaError_t launch_widen_kv(const WidenParams& p, cudaStream_t st);  // prefill_fp8.cu

}  // namespace decattn
