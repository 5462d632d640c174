// prefill.cu -- causal attention of many query rows per request over the paged KV cache: the
// prefill side of "PaddlePaddle/HALOps" README, Highlights, GQA attention item (variable-length
// prefill and paged-KV decode over a BF16 KV cache, GQA). The T query rows of request b are its
// last T positions: row t sees keys 0 .. Lb - T + t (the decode's bottom-right causal rule,
// with T large). A dense contraction, on the fifth-generation tensor cores:
//  * CTA = two tiles of 128 query rows that read the same keys: two q heads of one KV head with
//    the same rows when G is even, else two adjacent row blocks of one q head. Every K/V block
//    brought in by TMA serves both tiles. CTAs are numbered heaviest first.
//  * per block of 128 keys and tile u: S_u = Q_u K^T (128 x 128 fp32) in tensor memory on
//    kind::f16 (Q and K K-major, 128-byte swizzle); softmax warpgroup u (thread r owns query row
//    r = tensor-memory lane r) turns S_u into P_u, bf16 packed two to a column over S_u's first
//    64 columns; O_u += P_u V reads P_u from tensor memory and V as TMA staged it (head dims
//    contiguous: MN-major). O_0 and O_1 (128 x 128 fp32 each) stay in tensor memory.
//  * the MMA warp alternates the tiles: while warpgroup 0 works on S_0, the tensor core runs
//    tile 1's P V and next S, and the other way round.
//  * online softmax with a per-row reference maximum that moves only when a score passes it by
//    more than 2^kPfTau: P is computed in one pass against the current reference, and the pass
//    is redone (after rescaling the row of O) only in the rare block that moves it.
// CTA: 10 warps: 0-3 softmax of tile 0, 4-7 softmax of tile 1, 8 TMA producer (Q of both tiles
// first, then separate K and V rings of two 128-key stages), 9 MMA issue (one thread). The
// epilogue stages O through the Q area and writes it with TMA stores. Every wait is bounded
// (DECATTN_ETIMEOUT, then an orderly exit).
#include "common.cuh"
#include "tc.cuh"

namespace decattn {

constexpr int kPfD = 128;         // head_dim
constexpr int kPfM = 128;         // query rows per tile: the M of both products
constexpr int kPfN = 128;         // keys per block: the N of S and the contraction of P V
constexpr int kPfStages = 2;      // K stages and V stages
constexpr int kPfWarps = 10;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfTau = 8;         // P <= 2^kPfTau
constexpr int kPfTmemCols = 512;  // S_0, S_1, O_0, O_1: 128 columns each

// Shared-memory layout (offsets from a 1024-byte aligned base). A 128 x 128 bf16 tile is two
// "atoms" of 64 elements (128 bytes) per row: atom a holds elements 64a .. 64a + 63 of all 128
// rows, row r at 128 r, 16-byte chunk c at (c ^ (r % 8)) * 16 (the TMA 128-byte swizzle).
struct PfSmem {
  static constexpr int ATOM = 128 * 128;                  // 16 KB
  static constexpr int TILE = 2 * ATOM;                   // 32 KB
  static constexpr int OFF_Q = 0;                         // [tile]
  static constexpr int OFF_K = OFF_Q + 2 * TILE;          // [stage]
  static constexpr int OFF_V = OFF_K + kPfStages * TILE;  // [stage]
  static constexpr int OFF_BAR = OFF_V + kPfStages * TILE;
  static constexpr int NBAR = 16;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;     // tensor-memory base, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 227 * 1024, "one CTA per SM");
};

enum PfBar {
  kPfKFull = 0,    // [stage] producer -> MMA: K tile landed
  kPfKEmpty = 2,   // [stage] MMA commit after the block's last S -> producer
  kPfVFull = 4,    // [stage] producer -> MMA: V tile landed
  kPfVEmpty = 6,   // [stage] MMA commit after the block's last P V -> producer
  kPfSFull = 8,    // [tile] MMA commit -> softmax: S_u of the next block in tensor memory
  kPfPReady = 10,  // [tile] 4 softmax warps -> MMA: P_u written (and rows of O_u rescaled)
  kPfOFin = 12,    // [tile] MMA commit after tile u's last P V -> softmax epilogue
  kPfQFull = 14,   // producer -> MMA: Q of both tiles landed (TMA)
  kPfDrain = 15,   // MMA commit -> MMA: every tensor-core operation complete
};

// The two tiles of CTA `cta` (numbered heaviest first); the host sizes the grid the same way.
struct PfTile {
  int qh, t0, nkb;  // q head, first query row, key blocks its rows see
};

__host__ __device__ inline int pf_tiles_per_head(int T) { return (T + kPfM - 1) / kPfM; }
__host__ __device__ inline int pf_grid(int B, int T, int Hq, int G) {
  const int nqb = pf_tiles_per_head(T);
  return (G % 2 == 0) ? nqb * B * (Hq / 2) : ((nqb + 1) / 2) * B * Hq;
}

// All 128 columns of this warp's 32 lanes of S_u in one round trip (four loads, one wait).
__device__ __forceinline__ void pf_ld128(uint32_t taddr, float (&v)[128]) {
  uint32_t r[128];
  asm volatile(
      "{\n"
      " tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n"
      " tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n"
      " tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n"
      " tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n"
      " tcgen05.wait::ld.sync.aligned;\n}"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]),
        "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
        "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]),
        "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
      : "memory");
  #pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// P_u = 2^(s * scale - m) from the row's 128 scores, written as bf16 pairs (the lower key in
// the low half) over S_u's first 64 columns, chunk c of 32 keys on columns 16c .. 16c + 15.
// Returns the row sum of P in fp32.
__device__ __forceinline__ float pf_exp(uint32_t tS, const float (&v)[128], float sc, float m) {
  const float nmu = m == -INFINITY ? 0.f : -m;
  float la0 = 0.f, la1 = 0.f, lb0 = 0.f, lb1 = 0.f;
  #pragma unroll
  for (int c = 0; c < kPfN / 32; ++c) {
    uint32_t w[16];
    #pragma unroll
    for (int i = 32 * c; i < 32 * c + 32; i += 4) {
      float x0, x1, x2, x3;
      ffma2(x0, x1, v[i], v[i + 1], sc, sc, nmu, nmu);
      ffma2(x2, x3, v[i + 2], v[i + 3], sc, sc, nmu, nmu);
      const float p0 = fast_exp2(x0), p1 = fast_exp2(x1), p2 = fast_exp2(x2), p3 = fast_exp2(x3);
      fadd2(la0, la1, la0, la1, p0, p1);
      fadd2(lb0, lb1, lb0, lb1, p2, p3);
      w[(i - 32 * c) / 2] = pack_bf16(p0, p1);
      w[(i - 32 * c) / 2 + 1] = pack_bf16(p2, p3);
    }
    tmem_st16u(tS + 16 * c, w);
  }
  return (la0 + la1) + (lb0 + lb1);
}

// 3-D tiled TMA load into shared memory, completion signalled on an mbarrier.
__device__ __forceinline__ void pf_tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA store of a shared-memory box, tracked by this thread's bulk async-groups.
__device__ __forceinline__ void pf_tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void pf_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's bulk groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void pf_bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until every bulk group of this thread has completed (its global writes performed).
__device__ __forceinline__ void pf_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO) {
  using L = PfSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wl = p.wait_ns;  // every pipeline wait gives up after this long

  // ---- request, KV head and the two tiles of this CTA. The row-block step is the slowest
  //      index of the grid, counted down, so the CTAs with the most keys start first.
  const bool head_pair = (p.G % 2) == 0;
  const int ny = head_pair ? p.Hq / 2 : p.Hq;
  const int nsteps = head_pair ? pf_tiles_per_head(p.T) : (pf_tiles_per_head(p.T) + 1) / 2;
  const int step = nsteps - 1 - (int)blockIdx.x / (p.B * ny);
  const int rem = (int)blockIdx.x % (p.B * ny);
  const int b = rem / ny, y = rem % ny;
  const int Lb = p.seq_lens[b];
  // the request's query rows: Tb of them from packed row qoff on
  int Tb = p.T;
  int qoff = b * p.T;  // packed rows times Hq stay below 2^31 (checked on the host)
  if (p.cu_q) {
    const int c0 = p.cu_q[b], c1 = p.cu_q[b + 1];
    Tb = c1 - c0;
    qoff = c0;
    if (c0 < 0 || Tb < 0 || Tb > p.T || (int64_t)c1 > p.total_rows) {  // offsets outside the packed rows
      if (threadIdx.x == 0) set_status(p.status, DECATTN_EDEVICE);
      return;
    }
  }
  PfTile tl0, tl1;
  {
    tl0.qh = head_pair ? 2 * y : y;
    tl1.qh = head_pair ? 2 * y + 1 : y;
    tl0.t0 = head_pair ? step * kPfM : 2 * step * kPfM;
    tl1.t0 = head_pair ? step * kPfM : (2 * step + 1) * kPfM;
    // keys the tile's last row sees: [0, min(Lb, Lb - Tb + t_last + 1))
    const int tlast0 = min(tl0.t0 + kPfM, Tb) - 1, tlast1 = min(tl1.t0 + kPfM, Tb) - 1;
    const int kmax0 = (Lb < 0 || tl0.t0 >= Tb) ? 0 : max(0, min(Lb, Lb - Tb + tlast0 + 1));
    const int kmax1 = (Lb < 0 || tl1.t0 >= Tb) ? 0 : max(0, min(Lb, Lb - Tb + tlast1 + 1));
    tl0.nkb = (kmax0 + kPfN - 1) / kPfN;
    tl1.nkb = (kmax1 + kPfN - 1) / kPfN;
  }
  // a row block past the request's rows (variable-length rows, or T not a multiple of two
  // blocks): nothing to compute or write; the whole CTA leaves before it sets anything up
  if (tl0.t0 >= Tb && tl1.t0 >= Tb) {
    if (threadIdx.x == 0 && Lb < 0) set_status(p.status, DECATTN_EDEVICE);
    return;
  }
  const int h = tl0.qh / p.G;
  const int nkb_max = max(tl0.nkb, tl1.nkb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&bar[kPfKFull + s], 1);
      mbar_init(&bar[kPfKEmpty + s], 1);
      mbar_init(&bar[kPfVFull + s], 1);
      mbar_init(&bar[kPfVEmpty + s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bar[kPfSFull + u], 1);
      mbar_init(&bar[kPfPReady + u], 4);
      mbar_init(&bar[kPfOFin + u], 1);
    }
    mbar_init(&bar[kPfQFull], 1);
    mbar_init(&bar[kPfDrain], 1);
    *abort = 0;
    if (Lb < 0) set_status(p.status, DECATTN_EDEVICE);
    fence_mbar_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_sm)),
                 "n"(kPfTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sm;

  if (warp == 8) {
    // ===================================================================== producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      // Q of both tiles: per tile two boxes of 64 head dims x 128 packed rows, which land as the
      // two K-major 128-byte-swizzled atoms the MMA reads. Rows past the request's Tb belong to
      // the next request (or read as zeros past the last row): they are computed and never written.
      mbar_arrive_expect_tx(&bar[kPfQFull], 4u * (uint32_t)L::ATOM);
      #pragma unroll
      for (int a = 0; a < 2; ++a) {
        pf_tma_load_3d(sm + L::OFF_Q + a * L::ATOM, &tmQ, 64 * a, tl0.qh, qoff + tl0.t0, &bar[kPfQFull]);
        pf_tma_load_3d(sm + L::OFF_Q + L::TILE + a * L::ATOM, &tmQ, 64 * a, tl1.qh, qoff + tl1.t0,
                       &bar[kPfQFull]);
      }
    }
    int nk = 0, nv = 0;  // K / V blocks whose copies were issued
    for (int g = 0; g < nkb_max; ++g) {
      const int st = g % kPfStages;
      const uint32_t eph = (uint32_t)((g / kPfStages) & 1) ^ 1u;
      // lane i < 8: the 16-key group i of the block (its page id and row in the pool)
      const int key16 = g * kPfN + 16 * lane;
      const bool has = lane < kPfN / 16 && key16 < Lb;
      int row = 0;
      if (has) {
        const int pg = key16 / p.P;
        int pid = pg < p.mpps ? p.page_table[(int64_t)b * p.mpps + pg] : -1;
        if (pid < 0 || pid >= p.num_pages) {
          set_status(p.status, DECATTN_EDEVICE);
          pid = 0;  // keeps the copy inside the pool; the result is flagged invalid
        }
        row = (pid * p.Hkv + h) * p.P + key16 % p.P;
      }
      const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xffffffffu, has)) * 2u * 16u * 128u;
      int r = 1;
      if (lane == 0) r = tc_wait_suspend(&bar[kPfKEmpty + st], eph, p.status, abort, wl) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, r, 0)) break;
      // tests of the bounded waits leave one K block of CTA 0 out: nothing completes that stage
      const bool fill = !(blockIdx.x == 0 && g == p.skip_fill);
      if (fill && lane == 0) mbar_arrive_expect_tx(&bar[kPfKFull + st], bytes);
      __syncwarp();
      if (fill && has) {
        #pragma unroll
        for (int a = 0; a < 2; ++a)  // head dims 64a .. 64a + 63: one 128-byte swizzled atom
          tma_load_2d(sm + L::OFF_K + st * L::TILE + a * L::ATOM + lane * 16 * 128, &tmK, 64 * a, row,
                      &bar[kPfKFull + st]);
      }
      ++nk;
      if (lane == 0) r = tc_wait_suspend(&bar[kPfVEmpty + st], eph, p.status, abort, wl) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, r, 0)) break;
      if (lane < kPfN / 16 && !has) {
        // keys past the request's end: no copy; their P is 0, so their V rows must be finite
        uint8_t* vt = sm + L::OFF_V + st * L::TILE + lane * 16 * 128;
        #pragma unroll 4
        for (int i = 0; i < 2 * 16 * 128 / 16; ++i)
          reinterpret_cast<uint4*>(vt + (i >> 7) * L::ATOM)[i & 127] = make_uint4(0, 0, 0, 0);
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&bar[kPfVFull + st], bytes);
      __syncwarp();
      if (has) {
        #pragma unroll
        for (int a = 0; a < 2; ++a)
          tma_load_2d(sm + L::OFF_V + st * L::TILE + a * L::ATOM + lane * 16 * 128, &tmV, 64 * a, row,
                      &bar[kPfVFull + st]);
      }
      ++nv;
    }
    if (*abort && lane == 0) {
      // let the copies already issued land before the CTA exits
      for (int n = max(nk - kPfStages, 0); n < nk; ++n)
        mbar_wait(&bar[kPfKFull + n % kPfStages], (uint32_t)((n / kPfStages) & 1), nullptr, wl);
      for (int n = max(nv - kPfStages, 0); n < nv; ++n)
        mbar_wait(&bar[kPfVFull + n % kPfStages], (uint32_t)((n / kPfStages) & 1), nullptr, wl);
    }
  } else if (warp == 9) {
    // ===================================================================== MMA issue
    if (lane == 0) {
      const uint32_t base = smem_u32(sm);
      constexpr uint32_t idS = umma_idesc(1, 1, 0, 0, kPfM, kPfN);  // bf16 x bf16, both K-major
      constexpr uint32_t idO = umma_idesc(1, 1, 0, 1, kPfM, kPfD);  // bf16 x bf16, B (V) MN-major
      // descriptors (start address in 16-byte units in the low bits, so offsets add on):
      // Q and K K-major with 128-byte swizzle (8-row groups 1024 B apart; a 16-element k-step is
      // 32 bytes inside an atom, the next atom 16 KB on); V MN-major with 128-byte swizzle (the
      // two 64-element atoms of the head dims 16 KB apart, 8-key groups 1024 B apart).
      const uint64_t dQ0 = umma_desc(base + L::OFF_Q, 16, 1024, 2);
      const uint64_t dK0 = umma_desc(base + L::OFF_K, 16, 1024, 2);
      const uint64_t dV0 = umma_desc(base + L::OFF_V, L::ATOM, 1024, 2);
      const int nkb[2] = {tl0.nkb, tl1.nkb};
      auto kstep = [](int k) -> uint64_t {  // 16-element step k of a K-major 128-element operand
        return (uint64_t)(((k >> 2) * L::ATOM + (k & 3) * 32) >> 4);
      };
      auto issue_s = [&](int u, int g) {  // S_u = Q_u K(g)^T
        const uint64_t dQ = dQ0 + (uint64_t)((u * L::TILE) >> 4);
        const uint64_t dK = dK0 + (uint64_t)(((g % kPfStages) * L::TILE) >> 4);
        #pragma unroll
        for (int k = 0; k < kPfD / 16; ++k) umma_f16(tmem + kPfN * u, dQ + kstep(k), dK + kstep(k), idS, k > 0 ? 1u : 0u);
        umma_commit(&bar[kPfSFull + u]);
      };
      auto issue_pv = [&](int u, int g) {  // O_u += P_u V(g); P_u: 16 keys = 8 columns per step
        const uint64_t dV = dV0 + (uint64_t)(((g % kPfStages) * L::TILE) >> 4);
        const uint32_t tP = tmem + kPfN * u, tO = tmem + 2 * kPfN + kPfD * u;
        #pragma unroll
        for (int k = 0; k < kPfN / 16; ++k)  // V advances 16 keys = 2 KB
          umma_f16_tmem_a(tO, tP + 8 * k, dV + (uint64_t)((k * 2048) >> 4), idO, (g > 0 || k > 0) ? 1u : 0u);
      };
      bool ok = tc_wait_suspend(&bar[kPfQFull], 0, p.status, abort, wl);
      if (ok && nkb_max > 0) {
        ok = tc_wait_suspend(&bar[kPfKFull], 0, p.status, abort, wl);
        if (ok) {
          tc_fence_after();
          if (nkb[0] > 0) issue_s(0, 0);
          if (nkb[1] > 0) issue_s(1, 0);
          umma_commit(&bar[kPfKEmpty]);
        }
      }
      for (int g = 0; ok && g < nkb_max; ++g) {
        const int st = g % kPfStages;
        bool v_ready = false, k_ready = false;
        #pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (g >= nkb[u]) continue;
          if (!v_ready) {
            if (!tc_wait_suspend(&bar[kPfVFull + st], (uint32_t)((g / kPfStages) & 1), p.status, abort, wl)) { ok = false; break; }
            v_ready = true;
          }
          if (!tc_wait_suspend(&bar[kPfPReady + u], (uint32_t)(g & 1), p.status, abort, wl)) { ok = false; break; }
          tc_fence_after();
          issue_pv(u, g);
          if (u == 1 || g >= nkb[1]) umma_commit(&bar[kPfVEmpty + st]);  // the block's last P V
          if (g == nkb[u] - 1) umma_commit(&bar[kPfOFin + u]);
          if (g + 1 < nkb[u]) {
            const int sn = (g + 1) % kPfStages;
            if (!k_ready) {
              if (!tc_wait_suspend(&bar[kPfKFull + sn], (uint32_t)(((g + 1) / kPfStages) & 1), p.status, abort, wl)) {
                ok = false;
                break;
              }
              k_ready = true;
              tc_fence_after();
            }
            issue_s(u, g + 1);
            if (u == 1 || g + 1 >= nkb[1]) umma_commit(&bar[kPfKEmpty + sn]);  // the next block's last S
          }
        }
      }
      if (!ok) *abort = 1;
      umma_commit(&bar[kPfDrain]);
      mbar_wait(&bar[kPfDrain], 0, nullptr);
    }
    __syncwarp();
  } else {
    // ===================================================================== softmax warpgroups
    const int u = warp >> 2, wq = warp & 3;
    const int r = 32 * wq + lane;  // query row of the tile = tensor-memory lane
    const int qh = u ? tl1.qh : tl0.qh;
    const int t = (u ? tl1.t0 : tl0.t0) + r;
    const int nkb = u ? tl1.nkb : tl0.nkb;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const uint32_t tS = tmem + lane_off + kPfN * u;
    const uint32_t tO = tmem + lane_off + 2 * kPfN + kPfD * u;
    const int lim = t < Tb ? Lb - Tb + t : -1;  // the last key this row sees (< 0: none)
    const int lim_min = __reduce_min_sync(0xffffffffu, lim);
    const float sc = p.qk_scale_log2;
    float mref = -INFINITY, l = 0.f;  // reference maximum (log2 units) and row sum
    bool ok = true;
    for (int g = 0; g < nkb; ++g) {
      if (!tc_wait_suspend_warp(&bar[kPfSFull + u], (uint32_t)(g & 1), p.status, abort, wl)) { ok = false; break; }
      tc_fence_after();
      const int j0 = g * kPfN;
      const bool masked = j0 + kPfN - 1 > lim_min;  // warp-uniform: some row does not see every key
      const int nvis = lim - j0 + 1;                // keys j0 .. j0 + nvis - 1 are visible to the row
      // the row's 128 scores in registers; keys past the row's limit are invisible
      float v[128];
      pf_ld128(tS, v);
      if (masked) {
        #pragma unroll
        for (int i = 0; i < kPfN; ++i)
          if (i >= nvis) v[i] = -INFINITY;
      }
      // the row maximum (the scale is positive); the reference moves when it is passed by more
      // than 2^kPfTau
      float m0 = -INFINITY, m1 = -INFINITY;
      #pragma unroll
      for (int i = 0; i < kPfN; i += 4) {
        m0 = fmax3(m0, v[i], v[i + 1]);
        m1 = fmax3(m1, v[i + 2], v[i + 3]);
      }
      const float xmax = fmaxf(m0, m1) * sc;
      float alpha = 1.f;
      if (xmax > mref + (float)kPfTau) {  // false when the row sees nothing here (xmax = -inf)
        alpha = mref == -INFINITY ? 0.f : fast_exp2(mref - xmax);
        l *= alpha;
        mref = xmax;
      }
      l += pf_exp(tS, v, sc, mref);
      // O_u's rows hold every block before this one: S_u of this block was committed after the
      // previous P V, so that product is complete. Tensor-memory accesses are warp-wide: the warp
      // rescales when any of its rows moved (alpha = 1 for the others).
      if (g > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        #pragma unroll
        for (int q4 = 0; q4 < kPfD / 32; ++q4) {
          float o[32];
          tmem_ld32(tO + 32 * q4, o);
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + 32 * q4, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kPfPReady + u]);
    }
    // ---- epilogue: O / l and lse of row t
    if (ok && nkb > 0 && !tc_wait_suspend_warp(&bar[kPfOFin + u], 0, p.status, abort, wl)) ok = false;
    if (!ok) *abort = 1;
    if (ok) {  // warp-uniform: every lane takes part in the tensor-memory loads
      // O / l through shared memory: this warp's 32 rows, 32 columns at a time, into one of two
      // 4 KB boxes in its tile's Q area (no tensor-core operation reads Q_u any more: they all
      // completed before the tile's last P V), swizzled as the store's tensor map expects (row i
      // at 128 i, 16-byte chunk c at (c ^ (i % 8)) * 16), then a TMA store of the box to packed
      // rows qoff + t0w .. qoff + t0w + 31, head qh, head dims 32 q4 ... A warp whose 32 rows run
      // past the request's last row (the next rows are another request's) stores its valid rows
      // with plain stores instead.
      tc_fence_after();
      const int t0w = t - lane;  // the warp's first row
      const bool whole_box = t0w + 32 <= Tb;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint8_t* stage = sm + L::OFF_Q + warp * 8192;
      #pragma unroll
      for (int q4 = 0; q4 < kPfD / 32; ++q4) {
        float o[32];
        if (nkb > 0) {
          tmem_ld32(tO + 32 * q4, o);
        } else {
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (!whole_box) {
          if (t < Tb) {
            float4* dst = reinterpret_cast<float4*>(p.out + ((int64_t)(qoff + t) * p.Hq + qh) * kPfD + 32 * q4);
            #pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
          }
          continue;
        }
        uint8_t* box = stage + (q4 & 1) * 4096;
        if (q4 >= 2) {  // the store that read this box two chunks ago
          if (lane == 0) pf_bulk_wait_read<1>();
          __syncwarp();
        }
        #pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          pf_tma_store_3d(&tmO, box, 32 * q4, qh, qoff + t0w);
          pf_bulk_commit();
        }
      }
      if (lane == 0) pf_bulk_wait_all();
      __syncwarp();
      if (t < Tb) p.lse[(int64_t)(qoff + t) * p.Hq + qh] = l > 0.f ? (mref + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kPfTmemCols) : "memory");
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t st) {
  const int smem = PfSmem::ALLOC;
  if (!ensure_smem_attr((const void*)prefill_kernel, smem)) return cudaErrorInvalidValue;
  if (p.B == 0 || p.T == 0 || p.Hq == 0) return cudaSuccess;
  const int64_t grid = (int64_t)pf_grid(p.B, p.T, p.Hq, p.G);
  if (grid <= 0 || grid > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, prefill_kernel, p, tmQ, tmK, tmV, tmO);
}

}  // namespace decattn
