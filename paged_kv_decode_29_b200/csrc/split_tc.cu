// split_tc.cu -- the split kernel for FP8 E4M3 KV on the fifth-generation tensor cores
// (tcgen05, accumulators in tensor memory). Same method, plan, workspace and outputs as
// split.cu ("PaddlePaddle/HALOps" README, Highlights, GQA attention item: paged-KV decode with
// FP8 KV and speculative decoding; "HPC-Ops: Tencent's CUDA Kernel Library for LLM Inference
// Hot Paths", "How the kernels are organized around specific workload shapes": uniform tiles,
// greedy bins, a combine), for head_dim 128 and G*T <= 16.
//
// Both products run on E4M3 tensor cores (kind::f8f6f4) straight from the staged pages, so no
// element of K or V is ever converted. A tile is processed in chunks of 128 keys:
//  * S^T (128 keys x 16 query rows, fp32 in tensor memory) = K Q^T, A = the staged K codes as TMA
//    left them (K-major, 128-byte swizzle). B = q scaled by a power of two per row and split into
//    E4M3 parts written K-major by the softmax warps: hi and lo side by side (N = 32; their two
//    16-column halves are added when read), which carry a bf16 q exactly; Q8: hi only (N = 16).
//  * O^T (128 head dims x 16 query rows, fp32 in tensor memory) += V^T P^T, A = the staged V codes
//    (MN-major: head dims contiguous, 128-byte swizzle). B = P^T with P scaled by (V page scale) *
//    C (C a power of two per chunk that keeps P within E4M3's range) and split into three E4M3
//    parts x = hi + mid / 16 + lo / 256 side by side (N = 48; the epilogue adds the three 16-column
//    groups of O^T with those weights): about 12 significant bits, as close to P as an f16 P would
//    be, so the result meets the same tolerance as the bf16 path. Q8: one part (N = 16) and its own
//    tolerance.
// Thread j of the 128-thread softmax group owns key j of the chunk (tensor-memory lane j) and
// reads its scores with one tcgen05.ld, so the per-key work has no fragment shuffles.
//
// Online softmax with a reference maximum: P = 2^(s - m_ref) for every key of a tile, where
// m_ref is the exact maximum of the tile's first chunk and moves (to the running maximum) only
// when a later chunk holds a score above m_ref + kTcTau; then O^T and the running sums are
// rescaled in place. P is thus at most 2^kTcTau, and most chunks need only a one-flag-per-warp
// check instead of an exact maximum.
//
// CTA: 6 warps, 2 CTAs per SM, and one wave of CTAs: CTA i takes bins i, i + grid, ... .
//  * warps 0-3 (softmax group; warp w reads tensor-memory lanes 32w..32w+31): per chunk, scores ->
//    P and its E4M3 parts (while the previous chunk's P V runs), the O^T rescale when the
//    reference moves; per tile, the next tile's q (loaded from global memory during the last
//    chunk and published before the epilogue, so the MMA warp starts that tile meanwhile) and the
//    epilogue;
//  * warp 4 (producer): the bins' tiles (walk, then plan) and their K/V pages by TMA, 128-key
//    chunks in a three-stage ring, FP8 page scales by cp.async; the next tile's first page ids are
//    read while the current tile's first chunk is in flight;
//  * warp 5 (MMA): allocates tensor memory and issues every tcgen05.mma from one thread.
// Every wait is bounded; a wait that gives up sets DECATTN_ETIMEOUT and a CTA-wide abort flag,
// after which every role leaves its loop and the CTA frees its tensor memory and exits.
#include "common.cuh"
#include "tc.cuh"
#include "walk.cuh"

namespace decattn {

constexpr int kTcD = 128;          // head_dim
constexpr int kTcN = 16;           // query rows of the KV group (zero-padded): one 16-column group
constexpr int kTcChunk = 128;      // keys per chunk: the M of S^T and the contraction of O^T
constexpr int kTcBlk = kTcChunk / 16;  // 16-key blocks (one TMA box each) per chunk
constexpr int kTcThreads = 192;
constexpr int kTcTau = 6;          // P <= 2^kTcTau
constexpr int kTcStages = 3;       // chunk stages of the K/V ring

// Per mode: Q8 = one E4M3 part for q and for P (its own tolerance); otherwise two parts of q and
// three of P (the standard tolerance).
template <bool Q8>
struct TcMode {
  static constexpr int QP = Q8 ? 1 : 2;            // E4M3 parts of q
  static constexpr int PP = Q8 ? 1 : 3;            // E4M3 parts of P
  static constexpr int NS = QP * kTcN;             // S^T columns (per q part, 16 query rows)
  static constexpr int NO = PP * kTcN;             // O^T columns (per P part, 16 query rows)
  static constexpr int TMEM = Q8 ? 64 : 128;       // columns: S^T double buffer + O^T, a power of 2
  static_assert(2 * NS + NO <= TMEM, "tensor-memory columns");
};

// Shared-memory layout (offsets from a 1024-byte aligned base).
template <bool Q8>
struct TcSmem {
  using M = TcMode<Q8>;
  static constexpr int STAGES = kTcStages;
  static constexpr int KCH = kTcChunk * kTcD;                // bytes of one K (or V) chunk: 16 KB
  static constexpr int QB = M::QP * kTcN * kTcD;             // q parts [part][16][128], E4M3
  static constexpr int PPLANE = kTcChunk * kTcN;             // one E4M3 part of P^T: 2 KB
  static constexpr int PB = M::PP * PPLANE;                  // P^T of one chunk: [part][128 keys][16]
  // A chunk's P^T is written over its own K (MN-major interleaved, from the stage's start): the
  // softmax group writes it only after S^T of the chunk, the last reader of that K, is complete,
  // and the stage is refilled only after the chunk's P V.
  static constexpr int OFF_K = 0;                            // [stage][128 keys][128 B], 128-B swizzle
  static constexpr int OFF_V = OFF_K + STAGES * KCH;
  static constexpr int OFF_QB = OFF_V + STAGES * KCH;        // [tile parity] q parts, 128-B swizzle
  static constexpr int OFF_SC = OFF_QB + 2 * QB;             // per stage: 8 K scales, 8 V scales
  static constexpr int OFF_QCS = OFF_SC + STAGES * 2 * kTcBlk * 4;  // [tile parity][16]: 2^-E of q rows
  static constexpr int OFF_FLG = OFF_QCS + 2 * kTcN * 4;     // [2][8] per warp: "passes the reference" flag, then largest V scale
  static constexpr int OFF_RED = OFF_FLG + 2 * 8 * 4;        // [2][4][16] chunk maxima per warp
  static constexpr int OFF_ERED = OFF_RED + 2 * 4 * kTcN * 4;  // [2][4][16] row-sum partials (Q8: exact, rounded)
  static constexpr int OFF_UNIT = OFF_ERED + 2 * 4 * kTcN * 4;  // Unit x 2
  static constexpr int OFF_BAR = OFF_UNIT + 2 * (int)sizeof(Unit);
  static constexpr int NBAR = 18;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;        // tensor-memory base, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;                 // slack to align the base to 1024
  static_assert(OFF_QB % 1024 == 0 && QB % 1024 == 0, "swizzled q operands need 1024-byte bases");
  static_assert(OFF_BAR % 8 == 0, "mbarriers are 8-byte aligned");
  static_assert(PB <= KCH, "P^T fits in the K of its stage");
  static_assert(2 * (ALLOC + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Barrier slots. The P / P V hand-off has one barrier per chunk parity: chunk g (counted over all
// tiles of the CTA) signals kPReady + (g & 1) and its P V completes kPvDone + (g & 1), phase
// (g >> 1) & 1, so that the softmax group can compute and write chunk g + 1's P while chunk g's
// P V runs without ever running two phases ahead of a waiter (the MMA warp issues S^T of chunk
// g + 2 only after it has taken chunk g + 1's P).
// S^T has two tensor-memory buffers (chunk parity) and no "buffer read" barrier: S^T of chunk g + 2
// goes into chunk g's buffer, and the MMA warp issues it only after it has taken chunk g's P (and
// chunk g + 1's), which the softmax group signals after its last read of chunk g's S^T.
enum TcBar {
  kKvFull = 0,   // [stages] producer -> MMA, softmax: K, V and scales of a chunk landed
  kKvEmpty = 3,  // [stages] the stage may be refilled: the MMA commit after the chunk's P V
  kSFull = 6,    // [2] MMA commit -> softmax: S^T of a chunk is in tensor memory
  kPReady = 8,   // [chunk parity] 4 softmax warps -> MMA: P^T written, O^T rescaled
  kPvDone = 10,  // [chunk parity] MMA commit -> softmax: O^T += V^T P^T of a chunk complete
  kUFull = 12,   // [2] producer -> MMA, softmax: tile descriptor written
  kUEmpty = 14,  // [2] MMA + 4 softmax warps -> producer: tile descriptor read
  kQReady = 16,  // 4 softmax warps -> MMA: q hi / lo of the next tile written
  kFin = 17,     // MMA commit -> MMA: every tensor-core operation of the CTA complete
};
// The softmax group's own barrier: named barrier 1 over its 128 threads.
constexpr int kGroupBarrier = 1;

}  // namespace decattn

namespace decattn {

// q rows of a tile, bf16: thread (r = tid / 8, seg = tid % 8) loads elements 16 seg .. 16 seg + 15
// of query row r (rows >= G*T are zero).
__device__ __forceinline__ void tc_load_q(const SplitParams& p, const Unit& d, uint4 (&x)[2]) {
  const int r = threadIdx.x >> 3, seg = threadIdx.x & 7;
  x[0] = x[1] = make_uint4(0, 0, 0, 0);
  if (r < p.GT) {
    const int t = r / p.G, gg = r - t * p.G;
    const uint4* src = reinterpret_cast<const uint4*>(
        p.q + (((int64_t)d.b * p.T + t) * p.Hq + (int64_t)d.h * p.G + gg) * kTcD + 16 * seg);
    x[0] = __ldg(src);
    x[1] = __ldg(src + 1);
  }
}

// q parts of a tile into its operand buffer (E4M3, K-major, 128-byte swizzle) and the per-row
// factor 2^-E into qcs. q is scaled by a per-row power of two 2^E (largest |q| lands in
// [128, 256)) and rounded to E4M3: hi = E4M3(q 2^E); with two parts also lo = E4M3(q 2^E - hi)
// in the rows after hi's 16, which together carry the 8 significant bits of a bf16 q.
template <int QP>
__device__ __forceinline__ void tc_store_q(const uint4 (&x)[2], uint8_t* qb, float* qcs) {
  const int r = threadIdx.x >> 3, seg = threadIdx.x & 7;
  float v[16];
  #pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t w4[4] = {x[h].x, x[h].y, x[h].z, x[h].w};
    #pragma unroll
    for (int i = 0; i < 4; ++i) { v[8 * h + 2 * i] = bf16_lo(w4[i]); v[8 * h + 2 * i + 1] = bf16_hi(w4[i]); }
  }
  float amax = 0.f;
  #pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  // 2^E with E = 7 - floor(log2 amax): exponent-field arithmetic, exact
  const int ex = amax > 0.f ? ((__float_as_int(amax) >> 23) & 0xff) - 127 : 0;
  const int E = min(max(7 - ex, -100), 100);
  const float up = __int_as_float((127 + E) << 23);
  uint32_t hw[4], lw[4];
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t hh[2], ll[2];
    #pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float a0 = v[4 * i + 2 * k] * up, a1 = v[4 * i + 2 * k + 1] * up;
      hh[k] = f32x2_to_e4m3x2(a0, a1);
      if (QP == 2) {
        const float2 b = f16x2_to_float2(e4m3x2_to_f16x2(hh[k]));
        ll[k] = f32x2_to_e4m3x2(a0 - b.x, a1 - b.y);
      }
    }
    hw[i] = hh[0] | (hh[1] << 16);
    if (QP == 2) lw[i] = ll[0] | (ll[1] << 16);
  }
  const int off = r * kTcD + ((seg ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(qb + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  if (QP == 2) *reinterpret_cast<uint4*>(qb + kTcN * kTcD + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  if (seg == 0) qcs[r] = __int_as_float((127 - E) << 23);
}

template <bool Q8>
__global__ void __launch_bounds__(kTcThreads, 2)
split_tc_kernel(const SplitParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  using L = TcSmem<Q8>;
  using M = TcMode<Q8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  float* sc = reinterpret_cast<float*>(sm + L::OFF_SC);  // [stage][16]: K scales of the 8 blocks, then V scales
  Unit* umeta = reinterpret_cast<Unit*>(sm + L::OFF_UNIT);
  uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wl = p.wait_ns;  // every pipeline wait gives up after this long

  // The combine counters of this workspace start from zero on every run (as in split.cu).
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)p.B * p.T * p.Hq;
       i += (int64_t)gridDim.x * blockDim.x)
    p.row_cnt[i] = 0;
  // V is read in place by the MMA, including the rows of a tile's last chunk that no page fills:
  // they meet P = 0 and must be finite, so the ring starts zeroed (afterwards it only ever holds
  // codes from the pool). Ordered before the first TMA write and MMA read.
  for (int i = threadIdx.x; i < 2 * kTcStages * L::KCH / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(sm + L::OFF_K)[i] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&bar[kKvFull + s], 1);
      mbar_init(&bar[kKvEmpty + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[kSFull + s], 1);
      mbar_init(&bar[kUFull + s], 1);
      mbar_init(&bar[kUEmpty + s], 1 + 4);
      mbar_init(&bar[kPReady + s], 4);
      mbar_init(&bar[kPvDone + s], 1);
    }
    mbar_init(&bar[kQReady], 4);
    mbar_init(&bar[kFin], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {  // tensor memory: S^T (two buffers), O^T
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_sm)),
                 "n"(M::TMEM)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sm;

  if (warp == 4) {
    // ===================================================================== producer
    if (lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }
    const int P = p.P;
    int st = 0; uint32_t eph = 1;  // K/V ring stage and the parity of its "empty" wait
    int us = 0; uint32_t ueph = 1; // tile descriptor slot
    int64_t n_fill = 0;            // chunks issued
    bool ok = true;
    // Tiles of this CTA's bins (bin = blockIdx.x, blockIdx.x + gridDim.x, ...: the grid holds
    // only as many CTAs as are resident at once): each bin's full tiles from the walk, then
    // (after waiting for the planner, once) the rest from the plan, as in split.cu.
    int bin = blockIdx.x;
    FullTileWalk walk;
    walk_init(walk, p, lane, bin, p.n_bins);
    int jb = 0;              // next tile of the current bin
    int bin_units = -1;      // tiles of the current bin, once the plan is read
    bool plan_loaded = false, plan_good = false;
    int32_t pending = 0;
    PlanHeader hv = {};
    auto note = [&](int32_t code) {
      if (plan_loaded) set_status(p.status, code);
      else if (pending == 0) pending = code;
    };
    auto load_plan = [&]() {
      plan_loaded = true;
      griddep_wait();               // the plan kernel has finished and its writes are visible
      griddep_launch_dependents();  // the combine kernel may be scheduled now
      const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
      plan_good = hdr->magic == kPlanMagic && hdr->status == DECATTN_OK && hdr->n_bins == p.n_bins &&
                  hdr->batch == p.B && hdr->n_kv_heads == p.Hkv && hdr->tile_len == p.tile_len &&
                  hdr->sparse == p.sparse;
      if (plan_good) hv = *hdr;
      else if (lane == 0)
        set_status(p.status, hdr->magic != kPlanMagic ? DECATTN_EINVAL
                             : hdr->status != DECATTN_OK ? hdr->status : DECATTN_EINVAL);
      if (pending != 0) set_status(p.status, pending);
    };
    auto next_unit = [&](Unit& u) -> bool {
      while (bin < p.n_bins) {
        if (jb < walk.fc) { u = walk_unit(walk, p, lane, jb++, bin, p.n_bins); return true; }
        if (!plan_loaded) load_plan();
        if (plan_good && bin_units < 0) {
          if (walk.fc != 0 && hv.full_q + (bin < hv.full_r ? 1 : 0) != walk.fc) {  // walk and plan disagree
            if (lane == 0) set_status(p.status, DECATTN_EINVAL);
            plan_good = false;
          } else {
            bin_units = plan_bin_size(p.plan, hv, bin);
          }
        }
        if (plan_good && jb < bin_units) {
          u = hv.sparse ? plan_unit_sparse(p.plan, hv, p.seq_lens, bin, jb)
                        : plan_unit(p.plan, hv, p.seq_lens, bin, jb);
          ++jb;
          return true;
        }
        bin += gridDim.x;  // the next bin of this CTA
        jb = 0;
        bin_units = -1;
        walk_rebin(walk, bin, p.n_bins);
      }
      return false;
    };
    auto wait0 = [&](uint64_t* b, uint32_t par) -> bool {  // lane 0 waits, the warp follows
      int r = 1;
      if (lane == 0) r = tc_wait_suspend(b, par, p.status, abort, wl) ? 1 : 0;
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    // lane l: page id of page l of a tile's first window of 32 pages (0 past the tile's pages)
    auto first_window = [&](const Unit& u) -> int {
      const int pg0 = u.tok_begin / P, npg = (u.tok_end - u.tok_begin + P - 1) / P;
      return lane < npg ? p.page_table[(int64_t)u.b * p.mpps + min(pg0 + lane, p.mpps - 1)] : 0;
    };
    Unit dn;
    bool has_n = next_unit(dn);
    int pid_next = has_n ? first_window(dn) : 0;
    for (int u = 0; has_n && ok; ++u) {
      const Unit d = dn;
      if (!wait0(&bar[kUEmpty + us], ueph)) { ok = false; break; }
      if (lane == 0) {
        umeta[us] = d;
        mbar_arrive(&bar[kUFull + us]);
      }
      us ^= 1; if (us == 0) ueph ^= 1;
      const int pg0 = d.tok_begin / P;
      const int npg = (d.tok_end - d.tok_begin + P - 1) / P;
      if (lane == 0 && pg0 + npg > p.mpps) note(DECATTN_EDEVICE);  // row too short
      const int nblk = (d.tok_end - d.tok_begin + 15) / 16;
      int win = 0, pid_w = pid_next;  // page ids of pages [32 win, 32 win + 32) of the tile, one per lane
      bool checked = false;           // the window's ids have been range-checked
      bool looked = false;
      for (int b0 = 0; b0 < nblk && ok; b0 += kTcBlk) {
        const int nb = min(kTcBlk, nblk - b0);
        const int blk = b0 + lane;        // this lane's block (lane < nb)
        const int ip = (blk * 16) / P;    // its page, relative to the tile
        // a chunk starts page-aligned (tiles are multiples of the page size) and spans <= 8
        // pages, so all of its pages sit in one window of 32
        const int w_need = (b0 * 16) / P / 32;
        if (w_need != win) {
          win = w_need;
          const int pg = win * 32 + lane;
          pid_w = pg < npg ? p.page_table[(int64_t)d.b * p.mpps + min(pg0 + pg, p.mpps - 1)] : 0;
          checked = false;
        }
        if (!checked) {
          checked = true;
          const int pg = win * 32 + lane;
          if (pg < npg && (pid_w < 0 || pid_w >= p.num_pages)) {
            note(DECATTN_EDEVICE);
            pid_w = 0;  // keeps the copy inside the pool; the result is flagged invalid
          }
        }
        const int pid = __shfl_sync(0xffffffffu, pid_w, (ip - win * 32) & 31);
        if (!wait0(&bar[kKvEmpty + st], eph)) { ok = false; break; }
        // tests of the bounded waits leave one chunk of CTA 0 out: nothing completes that stage
        const bool fill = !(blockIdx.x == 0 && n_fill == p.skip_fill);
        if (fill && lane < nb) {  // FP8 page scales of the block (K, V), folded into the chunk's barrier
          const int64_t si = (int64_t)pid * p.Hkv + d.h;
          cp_async_4(&sc[st * 16 + lane], p.kv_scales + si);
          cp_async_4(&sc[st * 16 + 8 + lane], p.kv_scales + (int64_t)p.num_pages * p.Hkv + si);
          cp_async_mbar_arrive(&bar[kKvFull + st]);
        }
        __syncwarp();
        if (fill && lane == 0) mbar_arrive_expect_tx(&bar[kKvFull + st], (uint32_t)(nb * 2 * 16 * kTcD));
        __syncwarp();
        if (fill && lane < nb) {
          const int row = (pid * p.Hkv + d.h) * P + (blk * 16) % P;
          tma_load_2d(sm + L::OFF_K + st * L::KCH + lane * 16 * kTcD, &tmK, 0, row, &bar[kKvFull + st]);
          tma_load_2d(sm + L::OFF_V + st * L::KCH + lane * 16 * kTcD, &tmV, 0, row, &bar[kKvFull + st]);
        }
        ++n_fill;
        if (++st == kTcStages) { st = 0; eph ^= 1; }
        if (!looked) {  // the next tile's descriptor and first page ids, read while this tile's first copies fly
          looked = true;
          has_n = next_unit(dn);
          if (has_n) pid_next = first_window(dn);
        }
      }
      if (!looked && ok) {
        has_n = next_unit(dn);
        if (has_n) pid_next = first_window(dn);
      }
    }
    if (!plan_loaded) load_plan();
    if (ok) {
      // no more tiles: a descriptor with b = -1 tells the MMA warp and the softmax group to stop
      if (wait0(&bar[kUEmpty + us], ueph)) {
        if (lane == 0) {
          umeta[us].b = -1;
          mbar_arrive(&bar[kUFull + us]);
        }
      } else {
        ok = false;
      }
    }
    if (!ok && lane == 0) {
      *abort = 1;
      // let the copies already issued land before the CTA exits
      for (int64_t n = n_fill > kTcStages ? n_fill - kTcStages : 0; n < n_fill; ++n)
        mbar_wait(&bar[kKvFull + n % kTcStages], (uint32_t)((n / kTcStages) & 1), nullptr, wl);
    }
  } else if (warp == 5) {
    // ===================================================================== MMA issue
    if (lane == 0) {
      const uint32_t base = smem_u32(sm);
      // S^T: E4M3 x E4M3, both K-major, N = the q parts' columns; O^T: E4M3 x E4M3, both MN-major,
      // N = the P parts' columns
      constexpr uint32_t idS = umma_idesc(0, 0, 0, 0, kTcChunk, M::NS);
      constexpr uint32_t idO = umma_idesc(0, 0, 1, 1, kTcD, M::NO);
      int us = 0; uint32_t uph = 0;
      int64_t g = 0;  // chunks issued so far
      int ut = 0;     // tiles started so far
      bool ok = true;
      // descriptors, built once: the start address is the low 14 bits (16-byte units), so a
      // stage or a k-step adds to the base descriptor.
      //  K and q: K-major, 128-byte swizzle (8-row groups 1024 B apart; a 32-byte k-step); the q
      //    parts are consecutive 16-row blocks, so N = 32 spans hi then lo.
      //  V^T: the staged V (E4M3, MN-major: head dims contiguous, 128-byte swizzle; 8-key groups
      //    1024 B apart, a 32-key k-step is 4 KB).
      //  P^T: over the K of the chunk's stage, MN-major interleaved, key j of part q at
      //    q * 2 KB + 16 j: 8-key groups 128 B apart (leading offset), the next 16 columns (the
      //    next part) 2 KB on (stride offset).
      const uint64_t dK0 = umma_desc(base + L::OFF_K, 16, 1024, 2), dQ0 = umma_desc(base + L::OFF_QB, 16, 1024, 2);
      const uint64_t dV = umma_desc(base + L::OFF_V, 1024, 1024, 2);
      const uint64_t dP = umma_desc(base + L::OFF_K, 128, L::PPLANE, 0);
      const uint32_t tO = tmem + 2 * M::NS;
      // O^T (+)= V^T P^T over chunk gg's 128 keys. A tile's first chunk overwrites O^T: the
      // softmax group signals that chunk's P only after it has read the previous tile's O^T.
      auto pv = [&](int64_t gg, bool first_of_tile) -> bool {
        if (!tc_wait_suspend(&bar[kPReady + (gg & 1)], (uint32_t)((gg >> 1) & 1), p.status, abort, wl)) return false;
        tc_fence_after();
        const int sg = (int)(gg % kTcStages);
        const uint64_t a0 = dV + (uint64_t)((sg * L::KCH) >> 4);
        const uint64_t b0 = dP + (uint64_t)((sg * L::KCH) >> 4);
        #pragma unroll
        for (int k = 0; k < kTcChunk / 32; ++k)  // 32 keys per instruction: 4 KB of V, 512 B per P part
          umma_f8(tO, a0 + (uint64_t)(256 * k), b0 + (uint64_t)(32 * k), idO, (first_of_tile && k == 0) ? 0u : 1u);
        umma_commit(&bar[kPvDone + (gg & 1)]);
        umma_commit(&bar[kKvEmpty + sg]);  // K and V of the stage have both been read
        return true;
      };
      for (;;) {
        if (!tc_wait_suspend(&bar[kUFull + us], uph, p.status, abort, wl)) { ok = false; break; }
        const Unit d = umeta[us];
        mbar_arrive(&bar[kUEmpty + us]);
        us ^= 1; if (us == 0) uph ^= 1;
        if (d.b < 0) break;
        const int nc = (d.tok_end - d.tok_begin + kTcChunk - 1) / kTcChunk;
        if (!tc_wait_suspend(&bar[kQReady], (uint32_t)(ut & 1), p.status, abort, wl)) { ok = false; break; }
        const uint64_t dQ = dQ0 + (uint64_t)(((ut & 1) * L::QB) >> 4);
        for (int c = 0; c < nc; ++c, ++g) {
          const int st = (int)(g % kTcStages), sb = (int)(g & 1);
          if (!tc_wait_suspend(&bar[kKvFull + st], (uint32_t)((g / kTcStages) & 1), p.status, abort, wl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // S^T = K (q parts)^T: four 32-byte k-steps of the 128-byte swizzled rows
          const uint64_t dK = dK0 + (uint64_t)((st * L::KCH) >> 4);
          #pragma unroll
          for (int kk = 0; kk < kTcD / 32; ++kk)
            umma_f8(tmem + M::NS * sb, dK + (uint64_t)(2 * kk), dQ + (uint64_t)(2 * kk), idS, kk > 0 ? 1u : 0u);
          umma_commit(&bar[kSFull + sb]);
          if (c > 0 && !pv(g - 1, c == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!pv(g - 1, nc == 1)) { ok = false; break; }
        ++ut;
      }
      if (!ok) *abort = 1;
      // every tensor-core operation of the CTA completes before the memory is freed
      umma_commit(&bar[kFin]);
      mbar_wait(&bar[kFin], 0, nullptr);
    }
    __syncwarp();
  } else {
    // ===================================================================== softmax group
    const int key = threadIdx.x;  // key of the chunk / head dim of O^T = tensor-memory lane
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const float LN2 = 0.6931471805599453f;
    float* qcs_sm = reinterpret_cast<float*>(sm + L::OFF_QCS);   // [tile parity][16]
    int* red = reinterpret_cast<int*>(sm + L::OFF_RED);          // [2][4][16] chunk maxima (ordered ints)
    int* flg = reinterpret_cast<int*>(sm + L::OFF_FLG);          // [2][8]
    float* ered = reinterpret_cast<float*>(sm + L::OFF_ERED);    // [4][16] row-sum partials
    int us = 0; uint32_t uph = 0;
    int64_t g = 0;    // chunks processed so far
    int ut = 0;       // tiles processed so far
    // The group's barrier, with the AND of the four warps' states. A warp whose wait gave up
    // (which sets the abort flag) does not leave the loop on its own: it carries ok = false on
    // to the group's next barrier, which every warp reaches in the same order, and the barrier's
    // answer (the same in every thread) takes all four out together. The barrier thus always
    // completes: it needs no time limit.
    auto gsync = [&](bool mine) -> bool {
      const uint32_t in = (mine && *abort == 0) ? 1u : 0u;
      uint32_t all;
      asm volatile(
          "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
          "barrier.cta.red.and.aligned.pred po, %2, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
          : "=r"(all)
          : "r"(in), "n"(kGroupBarrier)
          : "memory");
      return all != 0u;
    };
    auto next_desc = [&](Unit& dd) -> bool {
      if (!tc_wait_warp(&bar[kUFull + us], uph, p.status, abort, wl)) return false;
      dd = umeta[us];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kUEmpty + us]);
      us ^= 1; if (us == 0) uph ^= 1;
      return true;
    };
    // q of a tile (if there is one) into operand buffer `par`; the MMA warp may start the tile
    // afterwards. The group's barrier is passed in either case.
    auto publish_q = [&](const uint4 (&x)[2], int par, bool have, bool mine) -> bool {
      if (have) {
        tc_store_q<M::QP>(x, sm + L::OFF_QB + par * L::QB, qcs_sm + kTcN * par);
        fence_async_smem();
      }
      if (!gsync(mine)) return false;
      if (have && lane == 0) mbar_arrive(&bar[kQReady]);
      return true;
    };
    // waits on a chunk's P V: chunk gg's completes kPvDone + (gg & 1), phase (gg >> 1) & 1
    auto wait_pv = [&](int64_t gg) -> bool {
      return tc_wait_warp(&bar[kPvDone + (gg & 1)], (uint32_t)((gg >> 1) & 1), p.status, abort, wl);
    };
    // this thread's row of O^T (its head dim): the P parts' 16-column groups, weighed 1, 1/16, 1/256
    auto o_sum = [&](uint32_t tO, float (&o)[kTcN]) {
      tmem_ld16(tO, o);
      #pragma unroll
      for (int q = 1; q < M::PP; ++q) {
        float t[kTcN];
        tmem_ld16(tO + kTcN * q, t);
        const float wq = q == 1 ? 0.0625f : 0.00390625f;
        #pragma unroll
        for (int n = 0; n < kTcN; ++n) o[n] += wq * t[n];
      }
    };
    Unit d;
    d.b = -1;
    bool ok = next_desc(d);
    {
      uint4 x[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      if (ok && d.b >= 0) tc_load_q(p, d, x);
      ok = publish_q(x, 0, ok && d.b >= 0, ok);
    }
    while (ok && d.b >= 0) {
      const int qp = ut & 1;
      const uint32_t tO = tmem + lane_off + 2 * M::NS;
      const float4* qcs4 = reinterpret_cast<const float4*>(qcs_sm + kTcN * qp);
      // lane n < G*T: the output row of query row n (final out, or the tile's partial slot)
      int64_t row_n = 0;
      if (lane < p.GT) {
        const int t = lane / p.G, gg = lane - (lane / p.G) * p.G;
        row_n = d.slot < 0 ? ((int64_t)d.b * p.T + t) * p.Hq + (int64_t)d.h * p.G + gg
                           : (int64_t)d.slot * p.GT + lane;
      }
      const int causal_base = d.seq_len - p.T;  // query row n sees key j iff j - base <= n / G
      // row sums of P: lacc (exact), and Q8: lrnd of the weights as rounded for P V
      float mref[kTcN], lacc[kTcN], lrnd[Q8 ? kTcN : 1];
      #pragma unroll
      for (int n = 0; n < kTcN; ++n) {
        mref[n] = -INFINITY;
        lacc[n] = 0.f;
        if constexpr (Q8) lrnd[n] = 0.f;
      }
      float c_ref = 1.f;  // the power of two that O^T carries (P scaled by (V page scale) * C)
      Unit dnext;
      dnext.b = -1;
      uint4 qx[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      const int nc = (d.tok_end - d.tok_begin + kTcChunk - 1) / kTcChunk;
      bool fail = false;  // a group barrier found a warp that gave up: the four leave together
      for (int c = 0; c < nc; ++c, ++g) {
        const int st = (int)(g % kTcStages), sb = (int)(g & 1);
        if (c == nc - 1) {  // the next tile: its descriptor now, its q rows in flight meanwhile
          if (!next_desc(dnext)) ok = false;
          else if (dnext.b >= 0) tc_load_q(p, dnext, qx);
        }
        // ---- the chunk's K, V and scales have landed; V stays in the stage as the E4M3 operand
        //      and the MMA warp frees the stage after the chunk's P V. (A wait that gives up
        //      leaves ok = false for the next group barrier; see gsync.)
        if (!tc_wait_warp(&bar[kKvFull + st], (uint32_t)((g / kTcStages) & 1), p.status, abort, wl)) ok = false;
        const int j = d.tok_begin + c * kTcChunk + key;
        const bool valid = j < d.tok_end;
        // this key's page scales
        const int blk = key >> 4;
        const float f = p.qk_scale_log2 * sc[st * 16 + blk];
        const float vsc = sc[st * 16 + 8 + blk];
        // P^T = P * (V page scale) * C with C a power of two such that the largest P (2^kTcTau)
        // times the chunk's largest V scale lands in (224, 448]; the same in every thread. The
        // largest scale of the keys in range (the producer filled their blocks; other slots hold
        // stale values) is reduced per warp here and over the warps at the group's next barrier.
        // V scales are >= 0, so their bit patterns order as the values.
        const uint32_t wsv = __reduce_max_sync(0xffffffffu, valid ? __float_as_uint(vsc) : 0u);
        auto chunk_c = [&]() -> float {
          const uint4 v4 = *reinterpret_cast<const uint4*>(flg + sb * 8 + 4);
          const float svmax = __uint_as_float(max(max(v4.x, v4.y), max(v4.z, v4.w)));
          const float r = 448.f / ((float)(1 << kTcTau) * svmax);
          // the largest power of two <= r (exponent field only); 1 when no scale is usable
          return (svmax > 0.f && r < 1e30f) ? __int_as_float(__float_as_int(r) & 0x7f800000) : 1.f;
        };
        if (!tc_wait_warp(&bar[kSFull + sb], (uint32_t)((g >> 1) & 1), p.status, abort, wl)) ok = false;
        tc_fence_after();
        // scores times the column factors f * 2^-E, in pairs
        float s[kTcN];
        if constexpr (M::QP == 2) {  // the q hi and lo halves of S^T, added
          float s2[2 * kTcN];
          tmem_ld32(tmem + lane_off + M::NS * sb, s2);
          #pragma unroll
          for (int q4 = 0; q4 < kTcN / 4; ++q4) {
            const float4 qc = qcs4[q4];
            const int n = 4 * q4;
            float f0, f1, f2, f3;
            fmul2(f0, f1, qc.x, qc.y, f, f);
            fmul2(f2, f3, qc.z, qc.w, f, f);
            fadd2(s[n], s[n + 1], s2[n], s2[n + 1], s2[kTcN + n], s2[kTcN + n + 1]);
            fadd2(s[n + 2], s[n + 3], s2[n + 2], s2[n + 3], s2[kTcN + n + 2], s2[kTcN + n + 3]);
            fmul2(s[n], s[n + 1], s[n], s[n + 1], f0, f1);
            fmul2(s[n + 2], s[n + 3], s[n + 2], s[n + 3], f2, f3);
          }
        } else {
          tmem_ld16(tmem + lane_off + M::NS * sb, s);
          #pragma unroll
          for (int q4 = 0; q4 < kTcN / 4; ++q4) {
            const float4 qc = qcs4[q4];
            const int n = 4 * q4;
            float f0, f1, f2, f3;
            fmul2(f0, f1, qc.x, qc.y, f, f);
            fmul2(f2, f3, qc.z, qc.w, f, f);
            fmul2(s[n], s[n + 1], s[n], s[n + 1], f0, f1);
            fmul2(s[n + 2], s[n + 3], s[n + 2], s[n + 3], f2, f3);
          }
        }

        // ---- mask; per-column maxima of the chunk
        int* rw = red + ((sb * 4 + warp) * kTcN);
        const int over = j - causal_base;  // > 0 only for the last T - 1 keys of the request
        if (!valid) {
          #pragma unroll
          for (int n = 0; n < kTcN; ++n) s[n] = -INFINITY;
        } else if (over > 0) {
          #pragma unroll
          for (int n = 0; n < kTcN; ++n)
            if (n < p.GT && over > n / p.G) s[n] = -INFINITY;
        }
        // does any score of the chunk pass the reference by more than kTcTau? (one flag per warp)
        // (a tile's first chunk goes straight to the exact maxima: its reference is unset)
        bool upd = c == 0;
        float c_chunk = 1.f;
        if (!upd) {
          bool over_ref = false;
          #pragma unroll
          for (int n = 0; n < kTcN; ++n) over_ref |= s[n] > mref[n] + (float)kTcTau;
          const int wflag = __any_sync(0xffffffffu, over_ref) ? 1 : 0;
          if (lane == 0) { flg[sb * 8 + warp] = wflag; flg[sb * 8 + 4 + warp] = (int)wsv; }
          if (!gsync(ok)) { fail = true; break; }
          const int4 f4 = *reinterpret_cast<const int4*>(flg + sb * 8);
          upd = (f4.x | f4.y | f4.z | f4.w) != 0;  // the same in every thread
          c_chunk = chunk_c();
        }
        float cm[kTcN];
        if (upd) {
          // exact maxima of the chunk: the reference moves to the running maximum
          #pragma unroll
          for (int n = 0; n < kTcN; ++n) {
            const int m = __reduce_max_sync(0xffffffffu, ordered_int(s[n]));
            if (lane == 0) rw[n] = m;
          }
          if (c == 0 && lane == 0) flg[sb * 8 + 4 + warp] = (int)wsv;
          if (!gsync(ok)) { fail = true; break; }
          if (c == 0) c_chunk = chunk_c();
          const int4* r4 = reinterpret_cast<const int4*>(red + sb * 4 * kTcN);
          #pragma unroll
          for (int q4 = 0; q4 < kTcN / 4; ++q4) {
            int4 m = r4[q4];
            #pragma unroll
            for (int w = 1; w < 4; ++w) {
              const int4 o = r4[w * (kTcN / 4) + q4];
              m.x = max(m.x, o.x); m.y = max(m.y, o.y); m.z = max(m.z, o.z); m.w = max(m.w, o.w);
            }
            cm[4 * q4] = ordered_float(m.x); cm[4 * q4 + 1] = ordered_float(m.y);
            cm[4 * q4 + 2] = ordered_float(m.z); cm[4 * q4 + 3] = ordered_float(m.w);
          }
        }
        // C may only shrink within a tile (the accumulated O^T carries the tile's C)
        float c_factor = 1.f;
        if (c == 0) {
          c_ref = c_chunk;
        } else if (c_chunk < c_ref) {
          c_factor = c_chunk / c_ref;  // a power of two: exact
          c_ref = c_chunk;
        }
        if (upd || c_factor != 1.f) {
          float alpha[kTcN];
          bool resc = c_factor != 1.f;
          #pragma unroll
          for (int n = 0; n < kTcN; ++n) {
            float a = 1.f;
            if (upd) {
              const float mn = fmaxf(mref[n], cm[n]);
              a = mn == -INFINITY ? 1.f : fast_exp2(mref[n] - mn);
              mref[n] = mn;
              lacc[n] *= a;
              if constexpr (Q8) lrnd[n] *= a;
            }
            alpha[n] = a * c_factor;
            resc |= alpha[n] != 1.f;
          }
          if (c > 0 && resc) {
            // O^T holds chunks 0 .. c-1 of this tile once the previous chunk's P V is done: rescale
            // every part's columns in place
            if (!wait_pv(g - 1)) ok = false;
            tc_fence_after();
            #pragma unroll
            for (int q = 0; q < M::PP; ++q) {
              float o[kTcN];
              tmem_ld16(tO + kTcN * q, o);
              #pragma unroll
              for (int n = 0; n < kTcN; ++n) o[n] *= alpha[n];
              tmem_st16(tO + kTcN * q, o);
            }
          }
        }
        // ---- P = 2^(s - m_ref) (at most 2^kTcTau); row sums in fp32
        float (&pr)[kTcN] = s;  // in place
        #pragma unroll
        for (int n = 0; n < kTcN; n += 2) {
          float d0, d1;
          fadd2(d0, d1, s[n], s[n + 1], mref[n] == -INFINITY ? 0.f : -mref[n], mref[n + 1] == -INFINITY ? 0.f : -mref[n + 1]);
          pr[n] = fast_exp2(d0);
          pr[n + 1] = fast_exp2(d1);
          fadd2(lacc[n], lacc[n + 1], lacc[n], lacc[n + 1], pr[n], pr[n + 1]);
        }
        // ---- P^T row of this key, 16 query rows: x = P * (V page scale) * C rounded to E4M3 parts,
        //      computed before the wait for the buffer. Q8: hi = E4M3(x) alone. Otherwise
        //      x = hi + mid / 16 + lo / 256: each rest (x minus the parts so far, exact in fp32) is
        //      scaled by 16 before it is rounded, so that the parts stay in E4M3's normal range for
        //      x >= 2^-6; the epilogue weighs the parts' O^T column groups by 1, 1/16, 1/256
        const float xs = vsc * c_ref;
        uint32_t w8[M::PP][4];
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          float x[4];
          fmul2(x[0], x[1], pr[4 * i], pr[4 * i + 1], xs, xs);
          fmul2(x[2], x[3], pr[4 * i + 2], pr[4 * i + 3], xs, xs);
          #pragma unroll
          for (int q = 0; q < M::PP; ++q) {
            const uint32_t lo = f32x2_to_e4m3x2(x[0], x[1]);
            const uint32_t hi = f32x2_to_e4m3x2(x[2], x[3]);
            w8[q][i] = valid ? (lo | (hi << 16)) : 0u;
            if (Q8 || q + 1 < M::PP) {
              const float2 a = f16x2_to_float2(e4m3x2_to_f16x2(lo)), b = f16x2_to_float2(e4m3x2_to_f16x2(hi));
              if constexpr (Q8) {
                // the output is normalised by the weights as rounded, so it stays a convex
                // combination of V rows (a single visible key reproduces its V row); lse keeps the
                // exact sums
                if (valid) {
                  const float rxs = 1.f / xs;
                  lrnd[4 * i] += a.x * rxs; lrnd[4 * i + 1] += a.y * rxs;
                  lrnd[4 * i + 2] += b.x * rxs; lrnd[4 * i + 3] += b.y * rxs;
                }
              } else {  // the rest times 16: 16 x - 16 part, one rounding of an exact result
                ffma2(x[0], x[1], x[0], x[1], 16.f, 16.f, -16.f * a.x, -16.f * a.y);
                ffma2(x[2], x[3], x[2], x[3], 16.f, 16.f, -16.f * b.x, -16.f * b.y);
              }
            }
          }
        }
        // P^T over the chunk's K: S^T of the chunk (complete, its barrier was waited on above) was
        // that K's last reader
        uint8_t* pbuf = sm + L::OFF_K + st * L::KCH;
        #pragma unroll
        for (int q = 0; q < M::PP; ++q)
          *reinterpret_cast<uint4*>(pbuf + q * L::PPLANE + key * kTcN) =
              make_uint4(w8[q][0], w8[q][1], w8[q][2], w8[q][3]);
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[kPReady + (g & 1)]);
      }
      if (fail) { ok = false; break; }
      // ---- the next tile's q: the MMA warp starts that tile while this one's epilogue runs
      if (!publish_q(qx, qp ^ 1, dnext.b >= 0, ok)) { ok = false; break; }

      // ---- epilogue: row sums over the tile, O^T / l, out or partial
      // row sums over the warp's 32 keys by a butterfly reduce-scatter (before the wait for the
      // tile's last P V): after the five levels, lanes 2c and 2c + 1 hold column c's sum (Q8: the
      // exact sums, then the rounded ones)
      auto warp_colsum = [&](const float (&in)[kTcN], float* dst) {
        float v[kTcN];
        #pragma unroll
        for (int n = 0; n < kTcN; ++n) v[n] = in[n];
        #pragma unroll
        for (int h = kTcN / 2, bit = 16; h >= 1; h >>= 1, bit >>= 1) {
          const bool up = (lane & bit) != 0;
          #pragma unroll
          for (int i = 0; i < h; ++i) {
            const float send = up ? v[i] : v[i + h];
            const float keep = up ? v[i + h] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        const int col = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
        if ((lane & 1) == 0) dst[warp * kTcN + col] = v[0];
      };
      warp_colsum(lacc, ered);
      if constexpr (Q8) warp_colsum(lrnd, ered + 4 * kTcN);
      if (!wait_pv(g - 1)) ok = false;
      tc_fence_after();
      float osum[kTcN];
      o_sum(tO, osum);
      tc_fence_before();
      if (!gsync(ok)) { ok = false; break; }
      // lane n: row n's sums, the reciprocal that normalises O^T and (one warp) its lse
      float l_n = 0.f, lr_n = 0.f;
      if (lane < kTcN) {
        l_n = ered[lane] + ered[kTcN + lane] + ered[2 * kTcN + lane] + ered[3 * kTcN + lane];
        const float* er = ered + (Q8 ? 4 * kTcN : 0);
        lr_n = er[lane] + er[kTcN + lane] + er[2 * kTcN + lane] + er[3 * kTcN + lane];
      }
      const float inv_n = lr_n > 0.f ? __fdividef(1.f, c_ref * lr_n) : 0.f;
      if (warp == 0 && lane < p.GT) {
        float mr = mref[0];
        #pragma unroll
        for (int n = 1; n < kTcN; ++n) mr = lane == n ? mref[n] : mr;
        float* dst_lse = (d.slot < 0 ? p.lse : p.part_lse) + row_n;
        *dst_lse = l_n > 0.f ? (mr + __log2f(l_n)) * LN2 : -INFINITY;
      }
      const int dd = key;  // head dim
      float* base_out = d.slot < 0 ? p.out : p.part_o;
      #pragma unroll
      for (int n = 0; n < kTcN; ++n) {
        if (n >= p.GT) break;
        const float o = osum[n];
        const int64_t row = __shfl_sync(0xffffffffu, row_n, n);
        const float inv = __shfl_sync(0xffffffffu, inv_n, n);
        base_out[row * kTcD + dd] = o * inv;
      }
      ++ut;
      d = dnext;
    }
    if (!ok) *abort = 1;
  }

  // ---- teardown: every role has left its loop; the MMA warp has seen its last MMA complete
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(M::TMEM) : "memory");
}

}  // namespace decattn

namespace decattn {

bool split_tc_supported(int kv_dtype, int D, int GT) {
  return (kv_dtype == DECATTN_KV_FP8E4M3 || kv_dtype == DECATTN_KV_FP8E4M3_MMA8) && D == kTcD && GT >= 1 &&
         GT <= kTcN;
}

template <bool Q8>
static cudaError_t launch_tc(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t st) {
  const int smem = TcSmem<Q8>::ALLOC;
  auto fn = split_tc_kernel<Q8>;
  if (!ensure_smem_attr((const void*)fn, smem)) return cudaErrorInvalidValue;
  // one wave: as many CTAs as are resident at once (2 per SM: the layout is sized for it),
  // each taking every grid-th bin
  static int sm_count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidValue;
  if (sm_count[dev] == 0 && cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(min(p.n_bins, 2 * sm_count[dev]));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps our prologue with the planner
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p, tmK, tmV);
}

cudaError_t launch_split_tc(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int kv_dtype,
                            cudaStream_t st) {
  return kv_dtype == DECATTN_KV_FP8E4M3_MMA8 ? launch_tc<true>(p, tmK, tmV, st) : launch_tc<false>(p, tmK, tmV, st);
}

}  // namespace decattn
