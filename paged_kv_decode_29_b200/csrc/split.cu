// split.cu -- the split kernel: one persistent CTA per bin of the plan; it walks its
// tiles, streams the page-table-indirected K/V rows of each tile through a shared-memory
// ring filled by TMA, and computes the tile's partial attention for the G*T query rows
// of its KV head.
//
// Method ("PaddlePaddle/HALOps" README, Highlights, GQA attention item: paged-KV decode,
// BF16/FP8 KV, GQA, speculative decoding, split-KV; "HPC-Ops: Tencent's CUDA Kernel
// Library for LLM Inference Hot Paths", "How the kernels are organized around specific
// workload shapes": uniform tiles balanced across CTAs, a combine merges the splits).
//
// CTA = 1 producer warp + NCW consumer warps.
//  * warp 0 (producer): reads the bin's tile list and page-table rows, and for every
//    16-key block issues two 2-D TMA copies (K rows, V rows) of one (page, KV head) into
//    the next ring stage; the tile's q rows go to a double-buffered q slot by bulk copy;
//    FP8 page scales ride along as 4-byte cp.async copies folded into the stage's
//    mbarrier. It waits only on "stage empty" barriers, so it runs ahead of the math.
//  * warps 1..NCW (consumers; with NCW = 2, 4 or 8 each takes one 8-row slice of the G*T
//    query rows, up to 64, and all read the same staged K/V): per 16-key block, S^T = K Q^T
//    on tensor cores with the keys on the MMA's M side ("SwapAB", as in the pages' Attention
//    SwapAB), so a G*T of 4..64 query rows fills N = 8 per warp instead of padding M to 16;
//    then an online softmax in
//    fp32 (log2 domain), then O^T += V^T P^T (again keys as the contraction, head_dim on
//    M). Probabilities go to the MMA as bf16 hi + bf16 lo (BF16 KV: two columns of the
//    same MMA when G*T <= 4, two N tiles otherwise), or as f16 hi + lo scaled by the page's V
//    scale (FP8 KV, two N tiles).
//  * FP8 KV: S^T runs on E4M3 MMAs straight from the staged codes (K is never widened);
//    V is widened to f16. With one consumer warp it is widened in registers; with several,
//    each widens its share of every V block into a shared f16 block (laid out like a bf16
//    stage, two buffers) and all read V^T from it with ldmatrix, so no element is
//    widened twice; the raw stage is released as soon as it is widened and used for S^T.
//  * occupancy: 4 CTAs per SM with one or two consumer warps (G*T <= 16); the wide variants
//    (G*T up to 32 / 64: 4 / 8 consumer warps) hold more registers and q rows per CTA and run
//    2 / 1 CTAs per SM, each with a deeper ring (80 / 144 KB) to keep as many bytes in flight.
//    The grid is one CTA per bin either way; with fewer CTAs resident than bins they run in
//    waves of equal load (the bins are balanced by the planner).
//  * the tile ends with either the final output (the tile covers its whole request) or
//    a normalised partial (o, lse) in the workspace for the combine kernel.
// FP8 KV with head_dim 128 and G*T <= 16 runs in split_tc.cu instead (tcgen05 tensor cores with
// tensor-memory accumulators); this kernel keeps the other FP8 shapes and all of BF16.
//
// Shared-memory staging uses the TMA 128-byte (or 64-byte) swizzle, so every ldmatrix
// below reads 8 distinct 16-byte bank groups.
#include "common.cuh"
#include "walk.cuh"

namespace decattn {


// FP8 KV: P is multiplied by (V page scale * kPScale) before its f16 rounding, so that small
// probabilities stay normal f16 numbers; the epilogue divides kPScale back out.
constexpr float kPScale = 256.f;
constexpr int kCtasPerSm = 4;  // CTAs per SM of the variants with up to 2 consumer warps (G*T <= 16)

// Resident CTAs per SM a variant is built for: 4 with one or two consumer warps; the wide
// variants (G*T > 16: 4 or 8 consumer warps, one 8-row slice of the query rows each) hold more
// registers and q rows per CTA and run 2 (4 warps) or 1 (8 warps) per SM with a deeper ring.
template <int NCW>
struct Occ {
  static constexpr int CPS = NCW <= 2 ? kCtasPerSm : NCW == 4 ? 2 : 1;
  static constexpr int RING = CPS == kCtasPerSm ? 40 * 1024 : CPS == 2 ? 80 * 1024 : 144 * 1024;
};

template <int KVT, int D>
struct Geo {
  static constexpr int ESZ = KVT == 0 ? 2 : 1;                  // bytes per KV element
  static constexpr int ROW = D * ESZ;                           // bytes of one key row
  static constexpr int RB = ROW >= 128 ? 128 : ROW;             // bytes of one TMA box row
  static constexpr int CPB = RB / 16;                           // 16-byte chunks per box row
  static constexpr int NBOX = ROW / RB;                         // boxes per 16-row block
  static constexpr int BOX_ELEMS = RB / ESZ;
  static constexpr int BOX_BYTES = 16 * RB;
  static constexpr int TILE = 16 * ROW;                         // K (or V) bytes per stage
  static_assert(RB == 128 || RB == 64, "box rows are 64 or 128 bytes");
  // byte offset of (row r, 16-byte chunk cg of the full row) in a stage buffer
  __device__ static __forceinline__ uint32_t off(int r, int cg) {
    const int box = cg / CPB, c = cg % CPB;
    const int sw = RB == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
    return (uint32_t)(box * BOX_BYTES + r * RB + (sw << 4));
  }
};

// VSH: the consumer warps share the widening of each FP8 V block (two f16 blocks in the layout
// of a bf16 stage, after the ring).
template <int KVT, int D, int NQ, bool VSH, int RING>
struct Smem {
  using G_ = Geo<KVT, D>;
  using G16 = Geo<0, D>;                                         // layout of a widened V block
  static constexpr int V16 = VSH ? 2 * G16::TILE : 0;
  static constexpr int STAGES = (RING - V16) / (2 * G_::TILE);
  static constexpr int QBYTES = 8 * NQ * D * 2;
  static constexpr int OFF_V16 = STAGES * 2 * G_::TILE;
  static constexpr int OFF_Q = OFF_V16 + V16;
  static constexpr int OFF_BAR = OFF_Q + 2 * QBYTES;
  static constexpr int NBAR = 2 * STAGES + 4 + (VSH ? 2 : 0);   // full, empty, qfull, qempty, vready
  static constexpr int OFF_META = OFF_BAR + 8 * NBAR;            // per stage: pad, K scale, V scale, pad
  static constexpr int OFF_QMETA = OFF_META + 16 * STAGES;       // Unit x 2
  static constexpr int BYTES = OFF_QMETA + 2 * (int)sizeof(Unit);
  static constexpr int ALLOC = BYTES + 1024;                     // slack to align the base to 1024
};

// Row of the staged q slot feeding MMA column n, or -1 for a zero column.
template <bool DUP>
__device__ __forceinline__ int qrow_of_col(int n, int GT) {
  if (DUP) {
    const int r = n & 3;  // columns 4..7 repeat rows 0..3 (they carry the low bf16 half of P)
    return r < GT ? r : -1;
  }
  return n < GT ? n : -1;
}

// KVT: 0 = bf16 KV, 1 = FP8 E4M3 KV.  NQ: 8-column tiles of S^T.  NPV: 8-column tiles of
// O^T.  DUP: bf16 with G*T <= 4 (hi in columns 0..3, lo in 4..7 of one tile).  NCW: consumer
// warps; consumer w owns S^T tiles [w*NQ/NCW, (w+1)*NQ/NCW) and the O^T tiles that go with them.
template <int KVT, int D, int NQ, int NPV, bool DUP, int NCW>
__global__ void __launch_bounds__(32 * (1 + NCW), Occ<NCW>::CPS)
split_kernel(const SplitParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  using G_ = Geo<KVT, D>;
  // FP8 with several consumer warps: they share the widening of every V block into a shared
  // f16 block, so that no element is widened twice
  constexpr bool VSH = KVT == 1 && NCW >= 2;
  using S_ = Smem<KVT, D, NQ, VSH, Occ<NCW>::RING>;
  using G16 = typename S_::G16;
  constexpr int STAGES = S_::STAGES;
  constexpr int NQW = NQ / NCW;    // S^T tiles per consumer warp
  constexpr int NPVW = NPV / NCW;  // O^T tiles per consumer warp
  static_assert(NQ % NCW == 0 && NPV % NCW == 0, "tiles split evenly over the consumer warps");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_::OFF_BAR);
  uint64_t* full = bar;
  uint64_t* empty = bar + STAGES;
  uint64_t* qfull = bar + 2 * STAGES;
  uint64_t* qempty = bar + 2 * STAGES + 2;
  uint64_t* vready = bar + 2 * STAGES + 4;  // VSH: both halves of widened V block b are written
  float* meta_sc = reinterpret_cast<float*>(sm + S_::OFF_META);      // [s*4 + 1] = K scale, [s*4 + 2] = V scale
  Unit* qmeta = reinterpret_cast<Unit*>(sm + S_::OFF_QMETA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wl = p.wait_ns;  // every pipeline wait gives up after this long
  // The combine counters of this workspace start from zero on every run. The combine of the
  // previous run has finished: the planner, which this grid may overlap, started after it.
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)p.B * p.T * p.Hq;
       i += (int64_t)gridDim.x * blockDim.x)
    p.row_cnt[i] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 32 * NCW); }
    for (int s = 0; s < 2; ++s) { mbar_init(&qfull[s], 1); mbar_init(&qempty[s], 32 * NCW); }
    if (VSH)
      for (int b = 0; b < 2; ++b) mbar_init(&vready[b], 32 * NCW);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ===================================================================== producer
    if (lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }
    const int P = p.P, kb_per_page = P / 16;
    int s = 0; uint32_t eph = 1;
    int qs = 0; uint32_t qeph = 1;
    bool ok = true;
    int64_t n_fill = 0, n_qfill = 0;  // copies issued so far (ring stages, q slots)
    // Tiles: the bin's full tiles from the walk, then (after waiting for the planner) the rest
    // from the plan. Errors found before the plan is complete are held back: the planner
    // clears the status word when it starts.
    FullTileWalk walk;
    walk_init(walk, p, lane, blockIdx.x, gridDim.x);
    bool waited = false;
    int n_units = walk.fc;
    int32_t pending = 0;
    PlanHeader hv = {};
    auto note = [&](int32_t code) {
      if (waited) set_status(p.status, code);
      else if (pending == 0) pending = code;
    };
    auto await_plan = [&]() {
      waited = true;
      griddep_wait();               // the plan kernel has finished and its writes are visible
      griddep_launch_dependents();  // the combine kernel may be scheduled now (it can read the
                                    // finished plan at once and waits for this grid before
                                    // reading partials)
      const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
      bool good = hdr->magic == kPlanMagic && hdr->status == DECATTN_OK && hdr->n_bins == (int)gridDim.x &&
                  hdr->batch == p.B && hdr->n_kv_heads == p.Hkv && hdr->tile_len == p.tile_len &&
                  hdr->sparse == p.sparse;
      if (good) {
        hv = *hdr;
        good = walk.fc == 0 || hv.full_q + ((int)blockIdx.x < hv.full_r ? 1 : 0) == walk.fc;
      }
      if (good) {
        n_units = plan_bin_size(p.plan, hv, blockIdx.x);
      } else if (lane == 0) {
        set_status(p.status, hdr->magic != kPlanMagic ? DECATTN_EINVAL
                             : hdr->status != DECATTN_OK ? hdr->status : DECATTN_EINVAL);
      }
      if (pending != 0) set_status(p.status, pending);
    };
    auto next_unit = [&](int j, Unit& u) -> bool {
      if (j < walk.fc) { u = walk_unit(walk, p, lane, j, blockIdx.x, gridDim.x); return true; }
      if (!waited) await_plan();
      if (j < n_units) {
        u = hv.sparse ? plan_unit_sparse(p.plan, hv, p.seq_lens, blockIdx.x, j)
                      : plan_unit(p.plan, hv, p.seq_lens, blockIdx.x, j);
        return true;
      }
      return false;
    };
    // The next tile's descriptor and first 32 page ids are fetched right after the current
    // tile's first stage is issued: they are ready long before its copies run out, and the
    // kernel's first copy waits on one tile decode only.
    Unit dn;
    bool has_n = next_unit(0, dn);
    int pid_next = 0;
    if (has_n) {
      const int pg0 = dn.tok_begin / P, npg = (dn.tok_end - dn.tok_begin + P - 1) / P;
      pid_next = lane < npg ? p.page_table[(int64_t)dn.b * p.mpps + min(pg0 + lane, p.mpps - 1)] : 0;
    }
    for (int u = 0; has_n && ok; ++u) {
      const Unit d = dn;
      int pid_l = pid_next;
      bool looked = false;  // every tile has at least one stage, so the look-ahead below runs
      // q rows of this tile: T bulk copies of G consecutive heads each
      if (!warp_wait_lane0(&qempty[qs], qeph, p.status, wl)) { ok = false; break; }
      if (lane == 0) {
        qmeta[qs] = d;
        const uint32_t bytes = (uint32_t)(p.G * D * 2);
        mbar_arrive_expect_tx(&qfull[qs], bytes * p.T);
        uint8_t* dst = sm + S_::OFF_Q + qs * S_::QBYTES;
        for (int t = 0; t < p.T; ++t)
          bulk_load(dst + t * bytes, p.q + (((int64_t)d.b * p.T + t) * p.Hq + (int64_t)d.h * p.G) * D, bytes,
                    &qfull[qs]);
      }
      ++n_qfill;
      qs ^= 1; if (qs == 0) qeph ^= 1;
      const int pg0 = d.tok_begin / P;
      const int npg = (d.tok_end - d.tok_begin + P - 1) / P;
      if (lane == 0 && pg0 + npg > p.mpps) note(DECATTN_EDEVICE);  // row too short
      for (int c0 = 0; c0 < npg && ok; c0 += 32) {
        if (c0 > 0)
          pid_l = c0 + lane < npg ? p.page_table[(int64_t)d.b * p.mpps + min(pg0 + c0 + lane, p.mpps - 1)] : 0;
        if (c0 + lane < npg && (pid_l < 0 || pid_l >= p.num_pages)) {
          note(DECATTN_EDEVICE);
          pid_l = 0;  // keeps the copy inside the pool; the result is flagged invalid
        }
        const int n_here = min(32, npg - c0);
        for (int i = 0; i < n_here && ok; ++i) {
          const int pid = __shfl_sync(0xffffffffu, pid_l, i);
          const int ip = c0 + i;
          for (int kb = 0; kb < kb_per_page; ++kb) {
            const int tok = d.tok_begin + ip * P + kb * 16;
            if (tok >= d.tok_end) break;
            if (!warp_wait_lane0(&empty[s], eph, p.status, wl)) { ok = false; break; }
            // tests of the bounded waits leave one fill of CTA 0 out: nothing completes that stage
            if (lane == 0 && !(blockIdx.x == 0 && n_fill == p.skip_fill)) {
              if (KVT == 1) {
                const int64_t si = (int64_t)pid * p.Hkv + d.h;
                cp_async_4(&meta_sc[s * 4 + 1], p.kv_scales + si);
                cp_async_4(&meta_sc[s * 4 + 2], p.kv_scales + (int64_t)p.num_pages * p.Hkv + si);
                cp_async_mbar_arrive(&full[s]);
              }
              mbar_arrive_expect_tx(&full[s], 2 * G_::TILE);
              const int row = (pid * p.Hkv + d.h) * P + kb * 16;
              uint8_t* ks = sm + s * 2 * G_::TILE;
              #pragma unroll
              for (int bx = 0; bx < G_::NBOX; ++bx) {
                tma_load_2d(ks + bx * G_::BOX_BYTES, &tmK, bx * G_::BOX_ELEMS, row, &full[s]);
                tma_load_2d(ks + G_::TILE + bx * G_::BOX_BYTES, &tmV, bx * G_::BOX_ELEMS, row, &full[s]);
              }
            }
            ++n_fill;
            if (++s == STAGES) { s = 0; eph ^= 1; }
            if (!looked) {
              looked = true;
              has_n = next_unit(u + 1, dn);
              if (has_n) {
                const int pg1 = dn.tok_begin / P, npg1 = (dn.tok_end - dn.tok_begin + P - 1) / P;
                pid_next = lane < npg1 ? p.page_table[(int64_t)dn.b * p.mpps + min(pg1 + lane, p.mpps - 1)] : 0;
              }
            }
          }
        }
      }
    }
    if (!waited) await_plan();
    if (ok) {
      // no more tiles: a unit with b = -1 tells the consumers to stop
      if (warp_wait_lane0(&qempty[qs], qeph, p.status, wl)) {
        if (lane == 0) {
          qmeta[qs].b = -1;
          mbar_arrive(&qfull[qs]);
        }
      } else {
        ok = false;
      }
    }
    if (!ok && lane == 0) {
      // a wait gave up: let the copies already issued land before the CTA exits. Fill n of
      // ring stage n % STAGES completes phase (n / STAGES) & 1 of its barrier.
      for (int64_t n = n_fill > STAGES ? n_fill - STAGES : 0; n < n_fill; ++n)
        mbar_wait(&full[n % STAGES], (uint32_t)((n / STAGES) & 1), nullptr, wl);
      for (int64_t n = n_qfill > 2 ? n_qfill - 2 : 0; n < n_qfill; ++n)
        mbar_wait(&qfull[n % 2], (uint32_t)((n / 2) & 1), nullptr, wl);
    }
    return;
  }

  // ======================================================================= consumer
  const int gid = lane >> 2, tig = lane & 3;
  const int nq0 = (warp - 1) * NQW;  // first S^T tile of this consumer warp
  int s = 0; uint32_t fph = 0;
  int qs = 0; uint32_t qfph = 0;
  int vblk = 0;       // VSH: V blocks widened so far (block vblk uses buffer vblk & 1)
  uint32_t vph = 0;   // VSH: bit b = phase of vready[b] to wait for next
  const float LN2 = 0.6931471805599453f;
  for (;;) {
    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[qs], qfph, p.status, wl))) return;
    const Unit d = qmeta[qs];
    if (d.b < 0) return;  // the producer has no more tiles
    // ---- q fragments (B operand of S^T = K Q^T): column n = query row
    // BF16 KV: bf16 pairs along k. FP8 KV: S^T = K Q^T runs on E4M3 MMAs (m16n8k32) straight
    // from the staged codes; q is scaled by a per-row power of two 2^E (largest |q| lands in
    // [128, 256)) and split into two E4M3 parts, hi = E4M3(q 2^E) and lo = E4M3(q 2^E - hi),
    // which together carry the 8 significant bits of a bf16 q. qcs = 2^-E undoes the scaling.
    constexpr int QK_STEPS = KVT == 0 ? D / 16 : D / 32;
    uint32_t qf[NQW][QK_STEPS][2];
    uint32_t ql[NQW][KVT == 1 ? QK_STEPS : 1][2];
    float qcs[NQW][2];
    {
      const uint8_t* qsm = sm + S_::OFF_Q + qs * S_::QBYTES;
      #pragma unroll
      for (int nw = 0; nw < NQW; ++nw) {
        const int r = qrow_of_col<DUP>(8 * (nq0 + nw) + gid, p.GT);
        const uint16_t* qr = reinterpret_cast<const uint16_t*>(qsm) + (r < 0 ? 0 : r) * D;
        if (KVT == 0) {
          #pragma unroll
          for (int kk = 0; kk < QK_STEPS; ++kk) {
            const uint32_t x0 = *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * tig);
            const uint32_t x1 = *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 8 + 2 * tig);
            qf[nw][kk][0] = r < 0 ? 0u : x0;
            qf[nw][kk][1] = r < 0 ? 0u : x1;
          }
        } else {
          // b0 holds k = 4tig..4tig+3, b1 holds k = 16+4tig..16+4tig+3 of each 32-wide k-step
          uint2 xv[QK_STEPS][2];
          float amax = 0.f;
          #pragma unroll
          for (int kk = 0; kk < QK_STEPS; ++kk)
            #pragma unroll
            for (int h = 0; h < 2; ++h) {
              xv[kk][h] = r < 0 ? make_uint2(0u, 0u)
                                : *reinterpret_cast<const uint2*>(qr + 32 * kk + 16 * h + 4 * tig);
              amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(xv[kk][h].x)), fabsf(bf16_hi(xv[kk][h].x))),
                                       fmaxf(fabsf(bf16_lo(xv[kk][h].y)), fabsf(bf16_hi(xv[kk][h].y)))));
            }
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          // 2^E with E = 7 - floor(log2 amax): exponent-field arithmetic, exact
          const int ex = amax > 0.f ? ((__float_as_int(amax) >> 23) & 0xff) - 127 : 0;
          const int E = min(max(7 - ex, -100), 100);
          const float up = __int_as_float((127 + E) << 23);
          const float down = __int_as_float((127 - E) << 23);
          #pragma unroll
          for (int kk = 0; kk < QK_STEPS; ++kk)
            #pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float v0 = bf16_lo(xv[kk][h].x) * up, v1 = bf16_hi(xv[kk][h].x) * up;
              const float v2 = bf16_lo(xv[kk][h].y) * up, v3 = bf16_hi(xv[kk][h].y) * up;
              const uint32_t h01 = f32x2_to_e4m3x2(v0, v1), h23 = f32x2_to_e4m3x2(v2, v3);
              const float2 b01 = f16x2_to_float2(e4m3x2_to_f16x2(h01));
              const float2 b23 = f16x2_to_float2(e4m3x2_to_f16x2(h23));
              const uint32_t l01 = f32x2_to_e4m3x2(v0 - b01.x, v1 - b01.y);
              const uint32_t l23 = f32x2_to_e4m3x2(v2 - b23.x, v3 - b23.y);
              qf[nw][kk][h] = h01 | (h23 << 16);
              ql[nw][kk][h] = l01 | (l23 << 16);
            }
          // this lane holds row gid's factor; the softmax needs columns 2tig and 2tig+1
          qcs[nw][0] = __shfl_sync(0xffffffffu, down, (2 * tig) * 4);
          qcs[nw][1] = __shfl_sync(0xffffffffu, down, (2 * tig + 1) * 4);
        }
      }
    }
    __syncwarp();
    mbar_arrive(&qempty[qs]);
    qs ^= 1; if (qs == 0) qfph ^= 1;

    // ---- per-column limits: key j is visible to query token t if j <= Lb - T + t
    int lim[NQW][2];
    #pragma unroll
    for (int nw = 0; nw < NQW; ++nw)
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = qrow_of_col<DUP>(8 * (nq0 + nw) + 2 * tig + e, p.GT);
        lim[nw][e] = r < 0 ? 0x7fffffff : d.seq_len - p.T + r / p.G;
      }
    int lim_min = 0x7fffffff;
    #pragma unroll
    for (int nw = 0; nw < NQW; ++nw) lim_min = min(lim_min, min(lim[nw][0], lim[nw][1]));
    lim_min = __reduce_min_sync(0xffffffffu, lim_min);
    const int safe_end = min(d.tok_end, lim_min + 1);  // keys below this need no mask

    float o[NPVW][D / 16][4];
    #pragma unroll
    for (int j = 0; j < NPVW; ++j)
      #pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) o[j][mt][0] = o[j][mt][1] = o[j][mt][2] = o[j][mt][3] = 0.f;
    float mrow[NQW][2], lrow[NQW][2];
    #pragma unroll
    for (int nw = 0; nw < NQW; ++nw) mrow[nw][0] = mrow[nw][1] = -INFINITY, lrow[nw][0] = lrow[nw][1] = 0.f;

    const int nkb = (d.tok_end - d.tok_begin + 15) / 16;
    for (int kbi = 0; kbi < nkb; ++kbi) {
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], fph, p.status, wl))) return;
      const int kbase = d.tok_begin + 16 * kbi;
      const uint32_t ks = smem_u32(sm + s * 2 * G_::TILE);
      const uint32_t vs = ks + G_::TILE;
      float sc2 = p.qk_scale_log2, vsc = 1.f;
      if (KVT == 1) {
        sc2 *= meta_sc[s * 4 + 1];
        vsc = meta_sc[s * 4 + 2] * kPScale;
      }
      const int vb = vblk & 1;
      if (VSH) {
        // ---- widen this warp's share of the V block to f16 in the layout of a bf16 stage: the
        //      block's 16 keys x D/16 raw 16-byte chunks (16 codes each) are dealt to the
        //      consumer warps' lanes, item i = (chunk i / 16, key i % 16)
        constexpr int ITEMS = 16 * (D / 16);
        constexpr int PER_LANE = (ITEMS + 32 * NCW - 1) / (32 * NCW);
        const uint8_t* vraw = sm + s * 2 * G_::TILE + G_::TILE;
        uint8_t* v16 = sm + S_::OFF_V16 + vb * G16::TILE;
        #pragma unroll
        for (int c = 0; c < PER_LANE; ++c) {
          const int item = (warp - 1) * 32 + lane + c * 32 * NCW;
          if (ITEMS % (32 * NCW) != 0 && item >= ITEMS) break;
          const int key = item & 15, cg = item >> 4;  // codes d = 16 cg .. 16 cg + 15 of this key
          const uint4 w = *reinterpret_cast<const uint4*>(vraw + G_::off(key, cg));
          uint4 lo, hi;
          lo.x = e4m3x2_to_f16x2(w.x & 0xffffu); lo.y = e4m3x2_to_f16x2(w.x >> 16);
          lo.z = e4m3x2_to_f16x2(w.y & 0xffffu); lo.w = e4m3x2_to_f16x2(w.y >> 16);
          hi.x = e4m3x2_to_f16x2(w.z & 0xffffu); hi.y = e4m3x2_to_f16x2(w.z >> 16);
          hi.z = e4m3x2_to_f16x2(w.w & 0xffffu); hi.w = e4m3x2_to_f16x2(w.w >> 16);
          *reinterpret_cast<uint4*>(v16 + G16::off(key, 2 * cg)) = lo;
          *reinterpret_cast<uint4*>(v16 + G16::off(key, 2 * cg + 1)) = hi;
        }
        mbar_arrive(&vready[vb]);
      }
      // ---- S^T = K Q^T  (rows: 16 keys; columns: query rows). Even and odd k-steps go to two
      //      accumulators so that two MMA chains are in flight.
      constexpr int NCH = KVT == 1 ? 4 : 2;  // independent accumulation chains
      float sacc[NCH][NQW][4];
      #pragma unroll
      for (int c = 0; c < NCH; ++c)
        #pragma unroll
        for (int nw = 0; nw < NQW; ++nw) sacc[c][nw][0] = sacc[c][nw][1] = sacc[c][nw][2] = sacc[c][nw][3] = 0.f;
      {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
        if (KVT == 0) {
          #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(ks + G_::off(r, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
            #pragma unroll
            for (int nw = 0; nw < NQW; ++nw) mma_bf16(sacc[kk & 1][nw], a, qf[nw][kk][0], qf[nw][kk][1]);
          }
        } else {
          // the staged codes are the A operand as they are: ldmatrix gives each lane 4 codes of
          // one key row per register, which is the m16n8k32 E4M3 A fragment
          #pragma unroll
          for (int kk = 0; kk < QK_STEPS; ++kk) {
            uint32_t a[4];
            ldsm_x4(ks + G_::off(r, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
            #pragma unroll
            for (int nw = 0; nw < NQW; ++nw) {
              mma_e4m3(sacc[2 * (kk & 1)][nw], a, qf[nw][kk][0], qf[nw][kk][1]);
              mma_e4m3(sacc[2 * (kk & 1) + 1][nw], a, ql[nw][kk][0], ql[nw][kk][1]);
            }
          }
        }
      }
      if (VSH) {
        // the raw stage is no longer read: K went into S^T, this warp's half of V into the f16 block
        __syncwarp();
        mbar_arrive(&empty[s]);
      }
      // ---- scale, mask, online softmax (log2 domain, fp32 state)
      const bool need_mask = kbase + 16 > safe_end;
      bool grew = false;
      float alpha[NQW][2];
      float pv[NQW][4];
      #pragma unroll
      for (int nw = 0; nw < NQW; ++nw) {
        float sv4[4];
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sum = KVT == 1 ? (sacc[0][nw][i] + sacc[1][nw][i]) + (sacc[NCH - 2][nw][i] + sacc[NCH - 1][nw][i])
                                     : sacc[0][nw][i] + sacc[1][nw][i];
          sv4[i] = sum * (KVT == 1 ? sc2 * qcs[nw][i & 1] : sc2);
          if (need_mask) {
            const int j = kbase + gid + (i >> 1) * 8;
            if (j >= d.tok_end || j > lim[nw][i & 1]) sv4[i] = -INFINITY;
          }
        }
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = fmaxf(sv4[e], sv4[e + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float mnew = fmaxf(mrow[nw][e], mx);
          grew |= mnew > mrow[nw][e];
          const float muse = mnew == -INFINITY ? 0.f : mnew;
          alpha[nw][e] = fast_exp2(mrow[nw][e] - muse);
          pv[nw][e] = fast_exp2(sv4[e] - muse);
          pv[nw][e + 2] = fast_exp2(sv4[e + 2] - muse);
          lrow[nw][e] = lrow[nw][e] * alpha[nw][e] + pv[nw][e] + pv[nw][e + 2];
          mrow[nw][e] = mnew;
        }
      }
      if (__any_sync(0xffffffffu, grew)) {
        #pragma unroll
        for (int j = 0; j < NPVW; ++j) {
          const int nw = DUP ? j : j / 2;
          #pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            o[j][mt][0] *= alpha[nw][0]; o[j][mt][1] *= alpha[nw][1];
            o[j][mt][2] *= alpha[nw][0]; o[j][mt][3] *= alpha[nw][1];
          }
        }
      }
      // ---- P^T as B fragments: C-fragment rows (keys) become the K index via movmatrix
      uint32_t bp[NPVW][2];
      #pragma unroll
      for (int nw = 0; nw < NQW; ++nw) {
        if (KVT == 1) {
          // f16 hi + lo of P * (V page scale) * kPScale: about 22 significant bits, so that P's
          // rounding stays far below the tolerance even for large |v| (f16 alone: 2^-11 |v|)
          const float x0 = pv[nw][0] * vsc, x1 = pv[nw][1] * vsc, x2 = pv[nw][2] * vsc, x3 = pv[nw][3] * vsc;
          const uint32_t h01 = pack_f16(x0, x1), h23 = pack_f16(x2, x3);
          const float2 f01 = f16x2_to_float2(h01), f23 = f16x2_to_float2(h23);
          bp[2 * nw][0] = movmatrix_t(h01);
          bp[2 * nw][1] = movmatrix_t(h23);
          bp[2 * nw + 1][0] = movmatrix_t(pack_f16(x0 - f01.x, x1 - f01.y));
          bp[2 * nw + 1][1] = movmatrix_t(pack_f16(x2 - f23.x, x3 - f23.y));
        } else {
          const uint32_t h01 = pack_bf16(pv[nw][0], pv[nw][1]);
          const uint32_t h23 = pack_bf16(pv[nw][2], pv[nw][3]);
          const uint32_t l01 = pack_bf16(pv[nw][0] - bf16_lo(h01), pv[nw][1] - bf16_hi(h01));
          const uint32_t l23 = pack_bf16(pv[nw][2] - bf16_lo(h23), pv[nw][3] - bf16_hi(h23));
          if (DUP) {
            const bool lo_lane = tig >= 2;  // columns 4..7 carry the low halves
            bp[0][0] = movmatrix_t(lo_lane ? l01 : h01);
            bp[0][1] = movmatrix_t(lo_lane ? l23 : h23);
          } else {
            bp[2 * nw][0] = movmatrix_t(h01);
            bp[2 * nw][1] = movmatrix_t(h23);
            bp[2 * nw + 1][0] = movmatrix_t(l01);
            bp[2 * nw + 1][1] = movmatrix_t(l23);
          }
        }
      }
      // ---- O^T += V^T P^T  (rows: head_dim; contraction: the 16 keys)
      if (KVT == 0) {
        const int q4 = lane >> 3;
        const int r = (lane & 7) + (q4 >> 1) * 8;
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(vs + G_::off(r, 2 * mt + (q4 & 1)), a[0], a[1], a[2], a[3]);
          #pragma unroll
          for (int j = 0; j < NPVW; ++j) mma_bf16(o[j][mt], a, bp[j][0], bp[j][1]);
        }
      } else if (VSH) {
        // both halves of the widened block are written: f16 V^T fragments as in the bf16 path
        if (!__all_sync(0xffffffffu, mbar_wait(&vready[vb], (vph >> vb) & 1u, p.status, wl))) return;
        vph ^= 1u << vb;
        const uint32_t v16 = smem_u32(sm + S_::OFF_V16 + vb * G16::TILE);
        const int q4 = lane >> 3;
        const int r = (lane & 7) + (q4 >> 1) * 8;
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(v16 + G16::off(r, 2 * mt + (q4 & 1)), a[0], a[1], a[2], a[3]);
          #pragma unroll
          for (int j = 0; j < NPVW; ++j) mma_f16(o[j][mt], a, bp[j][0], bp[j][1]);
        }
      } else {
        // thread (gid, tig) reads 4 codes at d = 32pp + 4gid .. +3 of keys 2tig, 2tig+1,
        // 2tig+8, 2tig+9 and pairs them by key: M-row gid of m-tile 2pp+sub is
        // d = 32pp + 4gid + 2sub, M-row gid+8 is d + 1.
        #pragma unroll
        for (int pp = 0; pp < D / 32; ++pp) {
          const int cg = 2 * pp + (gid >> 2), inb = (4 * gid) & 15;
          const uint8_t* vb = sm + s * 2 * G_::TILE + G_::TILE;
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vb + G_::off(2 * tig, cg) + inb);
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(vb + G_::off(2 * tig + 1, cg) + inb);
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(vb + G_::off(2 * tig + 8, cg) + inb);
          const uint32_t w3 = *reinterpret_cast<const uint32_t*>(vb + G_::off(2 * tig + 9, cg) + inb);
          #pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            // bytes 0,1 <- (key 2tig, key 2tig+1) at d offset 2sub, bytes 2,3 <- the same at 2sub+1
            const uint32_t sel = sub == 0 ? 0x5140u : 0x7362u;
            const uint32_t x01 = prmt(w0, w1, sel), x23 = prmt(w2, w3, sel);
            uint32_t a[4];
            a[0] = e4m3x2_to_f16x2(x01 & 0xffffu);
            a[1] = e4m3x2_to_f16x2(x01 >> 16);
            a[2] = e4m3x2_to_f16x2(x23 & 0xffffu);
            a[3] = e4m3x2_to_f16x2(x23 >> 16);
            #pragma unroll
            for (int j = 0; j < NPVW; ++j) mma_f16(o[j][2 * pp + sub], a, bp[j][0], bp[j][1]);
          }
        }
      }
      if (!VSH) {
        __syncwarp();
        mbar_arrive(&empty[s]);
      }
      ++vblk;
      if (++s == STAGES) { s = 0; fph ^= 1; }
    }

    // ---- epilogue: row sums, hi + lo, normalise, store
    #pragma unroll
    for (int nw = 0; nw < NQW; ++nw)
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lrow[nw][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        lrow[nw][e] = l;
      }
    if (DUP) {
      #pragma unroll
      for (int mt = 0; mt < D / 16; ++mt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) o[0][mt][i] += __shfl_xor_sync(0xffffffffu, o[0][mt][i], 2);
    } else {  // the products of P's hi and lo halves
      #pragma unroll
      for (int nw = 0; nw < NQW; ++nw)
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
          #pragma unroll
          for (int i = 0; i < 4; ++i) o[2 * nw][mt][i] += o[2 * nw + 1][mt][i];
    }
    #pragma unroll
    for (int nw = 0; nw < NQW; ++nw) {
      const int j = DUP ? nw : 2 * nw;
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = 8 * (nq0 + nw) + 2 * tig + e;
        if (DUP && n >= 4) continue;
        const int r = n < p.GT ? n : -1;
        if (r < 0) continue;
        const float l = lrow[nw][e];
        // FP8: P entered the MMA multiplied by kPScale (keeps it in f16's normal range)
        const float inv = l > 0.f ? (KVT == 1 ? 1.f / (kPScale * l) : 1.f / l) : 0.f;
        const float lse_v = l > 0.f ? (mrow[nw][e] + __log2f(l)) * LN2 : -INFINITY;
        const int t = r / p.G, g = r % p.G;
        float* dst;
        float* dst_lse;
        if (d.slot < 0) {
          const int64_t row = ((int64_t)d.b * p.T + t) * p.Hq + (int64_t)d.h * p.G + g;
          dst = p.out + row * D;
          dst_lse = p.lse + row;
        } else {
          const int64_t row = (int64_t)d.slot * p.GT + r;
          dst = p.part_o + row * D;
          dst_lse = p.part_lse + row;
        }
        if (KVT == 0 || VSH) {  // M-row gid of m-tile mt is d = 16 mt + gid
          #pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            dst[16 * mt + gid] = o[j][mt][e] * inv;
            dst[16 * mt + gid + 8] = o[j][mt][2 + e] * inv;
          }
        } else {  // register-widened FP8 V: M-row gid of m-tile 2pp+sub is d = 32pp + 4gid + 2sub
          #pragma unroll
          for (int pp = 0; pp < D / 32; ++pp) {
            float4 v;
            v.x = o[j][2 * pp][e] * inv;
            v.y = o[j][2 * pp][2 + e] * inv;
            v.z = o[j][2 * pp + 1][e] * inv;
            v.w = o[j][2 * pp + 1][2 + e] * inv;
            *reinterpret_cast<float4*>(dst + 32 * pp + 4 * gid) = v;
          }
        }
        if (gid == 0) *dst_lse = lse_v;
      }
    }
  }
}

// ------------------------------------------------------------------ host side
template <int KVT, int D, int NQ, int NPV, bool DUP, int NCW>
static cudaError_t launch_variant(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                  cudaStream_t st) {
  auto fn = split_kernel<KVT, D, NQ, NPV, DUP, NCW>;
  const int smem = Smem<KVT, D, NQ, KVT == 1 && NCW >= 2, Occ<NCW>::RING>::ALLOC;
  static_assert(Occ<NCW>::CPS * (Smem<KVT, D, NQ, KVT == 1 && NCW >= 2, Occ<NCW>::RING>::ALLOC + 1024) <=
                    228 * 1024, "the variant's CTAs fit an SM's shared memory");
  if (!ensure_smem_attr((const void*)fn, smem)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_bins);
  cfg.blockDim = dim3(32 * (1 + NCW));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps our prologue with the planner
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p, tmK, tmV);
}

template <int KVT, int D>
static cudaError_t launch_gt(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t st) {
  if constexpr (KVT == 0) {
    if (p.GT <= 4) return launch_variant<KVT, D, 1, 1, true, 1>(p, tmK, tmV, st);
    if (p.GT <= 8) return launch_variant<KVT, D, 1, 2, false, 1>(p, tmK, tmV, st);
    if (p.GT <= 16) return launch_variant<KVT, D, 2, 4, false, 2>(p, tmK, tmV, st);
    if (p.GT <= 32) return launch_variant<KVT, D, 4, 8, false, 4>(p, tmK, tmV, st);
    return launch_variant<KVT, D, 8, 16, false, 8>(p, tmK, tmV, st);
  } else {
    if (p.GT <= 8) return launch_variant<KVT, D, 1, 2, false, 1>(p, tmK, tmV, st);
    if (p.GT <= 16) return launch_variant<KVT, D, 2, 4, false, 2>(p, tmK, tmV, st);
    if (p.GT <= 32) return launch_variant<KVT, D, 4, 8, false, 4>(p, tmK, tmV, st);
    return launch_variant<KVT, D, 8, 16, false, 8>(p, tmK, tmV, st);
  }
}

bool split_supported(int kv_dtype, int D, int GT) {
  if (kv_dtype == DECATTN_KV_FP8E4M3_MMA8) return split_tc_supported(kv_dtype, D, GT);  // tcgen05 kernel only
  return GT >= 1 && GT <= kMaxGT && (D == 64 || D == 128) &&
         (kv_dtype == DECATTN_KV_BF16 || kv_dtype == DECATTN_KV_FP8E4M3);
}

cudaError_t launch_split(const SplitParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int kv_dtype, int D,
                         cudaStream_t st) {
  if (!split_supported(kv_dtype, D, p.GT)) return cudaErrorInvalidValue;
  if (kv_dtype == DECATTN_KV_BF16) return D == 128 ? launch_gt<0, 128>(p, tmK, tmV, st) : launch_gt<0, 64>(p, tmK, tmV, st);
  if (split_tc_supported(kv_dtype, D, p.GT)) return launch_split_tc(p, tmK, tmV, kv_dtype, st);  // tcgen05 path
  if (kv_dtype == DECATTN_KV_FP8E4M3_MMA8) return cudaErrorInvalidValue;  // the tcgen05 kernel only
  return D == 128 ? launch_gt<1, 128>(p, tmK, tmV, st) : launch_gt<1, 64>(p, tmK, tmV, st);
}

int split_ctas_per_sm() { return kCtasPerSm; }

}  // namespace decattn
