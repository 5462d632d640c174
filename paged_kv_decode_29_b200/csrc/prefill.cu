// prefill.cu -- causal attention of many query rows per request over the paged KV cache: the
// prefill side of "PaddlePaddle/HALOps" README, Highlights, GQA attention item (variable-length
// prefill and paged-KV decode over a BF16 KV cache, GQA). The T query rows of request b are its
// last T positions: row t sees keys 0 .. Lb - T + t (the decode's bottom-right causal rule,
// with T large). A dense contraction, on the fifth-generation tensor cores:
//  * CTA = (request, q head, block of 128 query rows), heaviest blocks first. Q (128 rows x 128
//    bf16) sits in shared memory as the A operand of S = Q K^T (K-major, 128-byte swizzle).
//  * per block of 128 keys: S (128 x 128 fp32) in tensor memory on kind::f16 (B = the K tile as
//    TMA staged it, K-major); thread r of the 128-thread softmax group owns query row r (tensor-
//    memory lane r), so a row's maximum and sum need no exchange between threads; P (bf16) goes to
//    shared memory as the A operand of O += P V, B = the V tile as staged (head dims contiguous:
//    MN-major); O (128 x 128 fp32) stays in tensor memory.
//  * online softmax with a per-row reference maximum that moves only when a score passes it by
//    more than 2^kPfTau (then the row of O is rescaled in place), so most blocks skip the rescale.
// CTA: 6 warps: warps 0-3 softmax group, warp 4 TMA producer (two K/V stages of 128 keys), warp 5
// MMA issue (one thread). Every wait is bounded (DECATTN_ETIMEOUT, then an orderly exit).
#include "common.cuh"
#include "tc.cuh"

namespace decattn {

constexpr int kPfD = 128;        // head_dim
constexpr int kPfM = 128;        // query rows per CTA: the M of both products
constexpr int kPfN = 128;        // keys per block: the N of S and the contraction of P V
constexpr int kPfStages = 2;     // K/V stages
constexpr int kPfThreads = 192;
constexpr int kPfTau = 8;        // P <= 2^kPfTau
constexpr int kPfTmemCols = 512; // S double buffer (2 x 128 columns), O (128)


// Shared-memory layout (offsets from a 1024-byte aligned base). A 128 x 128 bf16 tile is two
// "atoms" of 64 elements (128 bytes) per row: atom a holds elements 64a .. 64a + 63 of all 128
// rows, row r at 128 r, 16-byte chunk c at (c ^ (r % 8)) * 16 (the TMA 128-byte swizzle).
struct PfSmem {
  static constexpr int ATOM = 128 * 128;                 // 16 KB
  static constexpr int TILE = 2 * ATOM;                  // 32 KB
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = OFF_Q + TILE;         // [stage]: K tile, then V tile
  static constexpr int OFF_P = OFF_STAGE + kPfStages * 2 * TILE;
  static constexpr int OFF_BAR = OFF_P + TILE;
  static constexpr int NBAR = 12;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;    // tensor-memory base, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 227 * 1024, "one CTA per SM");
};

enum PfBar {
  kPfKvFull = 0,   // [2] producer -> MMA: K and V tiles of a key block landed
  kPfKvEmpty = 2,  // [2] MMA commit after the block's P V -> producer
  kPfSFull = 4,    // [2] MMA commit -> softmax: S of a key block in tensor memory
  kPfSFree = 6,    // [2] 4 softmax warps -> MMA: that S buffer has been read
  kPfPReady = 8,   // 4 softmax warps -> MMA: P written (and rows of O rescaled)
  kPfPvDone = 9,   // MMA commit -> softmax: O += P V of a block complete
  kPfQReady = 10,  // 4 softmax warps -> MMA: Q written
  kPfFin = 11,     // MMA commit -> MMA: every tensor-core operation complete
};

__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  using L = PfSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int qb = (int)gridDim.x - 1 - (int)blockIdx.x;  // the longest query blocks start first
  const int qh = blockIdx.y, b = blockIdx.z, h = qh / p.G;
  const int Lb = p.seq_lens[b];
  const int t0 = qb * kPfM;
  const int t_last = min(t0 + kPfM, p.T) - 1;
  // keys the block's last row sees: [0, min(Lb, Lb - T + t_last + 1))
  const int kmax = Lb < 0 ? 0 : max(0, min(Lb, Lb - p.T + t_last + 1));
  const int nkb = (kmax + kPfN - 1) / kPfN;

  // The K/V stages start zeroed: rows past a request's last page are never loaded, and their
  // contents meet P = 0 in the MMA, so they must be finite.
  for (int i = threadIdx.x; i < kPfStages * 2 * L::TILE / 16; i += kPfThreads)
    reinterpret_cast<uint4*>(sm + L::OFF_STAGE)[i] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&bar[kPfKvFull + s], 1);
      mbar_init(&bar[kPfKvEmpty + s], 1);
      mbar_init(&bar[kPfSFull + s], 1);
      mbar_init(&bar[kPfSFree + s], 4);
    }
    mbar_init(&bar[kPfPReady], 4);
    mbar_init(&bar[kPfPvDone], 1);
    mbar_init(&bar[kPfQReady], 4);
    mbar_init(&bar[kPfFin], 1);
    *abort = 0;
    if (Lb < 0) set_status(p.status, DECATTN_EDEVICE);
    fence_mbar_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_sm)),
                 "n"(kPfTmemCols)
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
    int st = 0; uint32_t eph = 1;
    int64_t n_fill = 0;
    for (int kb = 0; kb < nkb; ++kb) {
      int r = 1;
      if (lane == 0) r = tc_wait(&bar[kPfKvEmpty + st], eph, p.status, abort) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, r, 0)) break;
      // lane g < 8: the 16-key group g of the block (its page id and row in the pool)
      const int key16 = kb * kPfN + 16 * lane;
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
      const int ngroups = __popc(__ballot_sync(0xffffffffu, has));
      if (lane == 0) mbar_arrive_expect_tx(&bar[kPfKvFull + st], (uint32_t)(ngroups * 4 * 16 * 128));
      __syncwarp();
      if (has) {
        uint8_t* kt = sm + L::OFF_STAGE + st * 2 * L::TILE;
        uint8_t* vt = kt + L::TILE;
        #pragma unroll
        for (int a = 0; a < 2; ++a) {  // head dims 64a .. 64a + 63: one 128-byte swizzled atom
          tma_load_2d(kt + a * L::ATOM + lane * 16 * 128, &tmK, 64 * a, row, &bar[kPfKvFull + st]);
          tma_load_2d(vt + a * L::ATOM + lane * 16 * 128, &tmV, 64 * a, row, &bar[kPfKvFull + st]);
        }
      }
      ++n_fill;
      if (++st == kPfStages) { st = 0; eph ^= 1; }
    }
    if (*abort && lane == 0) {
      // let the copies already issued land before the CTA exits
      for (int64_t n = n_fill > kPfStages ? n_fill - kPfStages : 0; n < n_fill; ++n)
        mbar_wait(&bar[kPfKvFull + n % kPfStages], (uint32_t)((n / kPfStages) & 1), nullptr);
    }
  } else if (warp == 5) {
    // ===================================================================== MMA issue
    if (lane == 0) {
      const uint32_t base = smem_u32(sm);
      constexpr uint32_t idS = umma_idesc(1, 1, 0, 0, kPfM, kPfN);  // bf16 x bf16, both K-major
      constexpr uint32_t idO = umma_idesc(1, 1, 0, 1, kPfM, kPfD);  // bf16 x bf16, B (V) MN-major
      // descriptors (start address in 16-byte units in the low bits, so offsets add on):
      // Q, K, P K-major with 128-byte swizzle (8-row groups 1024 B apart; a 16-element k-step is
      // 32 bytes inside an atom, the next atom 16 KB on); V MN-major with 128-byte swizzle (the
      // two 64-element atoms of the head dims 16 KB apart, 8-key groups 1024 B apart).
      const uint64_t dQ = umma_desc(base + L::OFF_Q, 16, 1024, 2);
      const uint64_t dK0 = umma_desc(base + L::OFF_STAGE, 16, 1024, 2);
      const uint64_t dP = umma_desc(base + L::OFF_P, 16, 1024, 2);
      const uint64_t dV0 = umma_desc(base + L::OFF_STAGE + L::TILE, L::ATOM, 1024, 2);
      const uint32_t tO = tmem + 2 * kPfN;
      bool ok = tc_wait(&bar[kPfQReady], 0, p.status, abort);
      auto kstep = [](int k) -> uint64_t {  // 16-element step k of a K-major 128-element operand
        return (uint64_t)(((k >> 2) * L::ATOM + (k & 3) * 32) >> 4);
      };
      auto pv = [&](int g) -> bool {
        if (!tc_wait(&bar[kPfPReady], (uint32_t)(g & 1), p.status, abort)) return false;
        tc_fence_after();
        const int sg = g % kPfStages;
        const uint64_t dV = dV0 + (uint64_t)((sg * 2 * L::TILE) >> 4);
        #pragma unroll
        for (int k = 0; k < kPfN / 16; ++k)  // 16 keys per instruction: V advances 2 KB
          umma_f16(tO, dP + kstep(k), dV + (uint64_t)((k * 2048) >> 4), idO, (g > 0 || k > 0) ? 1u : 0u);
        umma_commit(&bar[kPfPvDone]);
        umma_commit(&bar[kPfKvEmpty + sg]);  // K and V of the stage have both been read
        return true;
      };
      for (int g = 0; ok && g < nkb; ++g) {
        const int st = g % kPfStages, sb = g & 1;
        if (!tc_wait(&bar[kPfKvFull + st], (uint32_t)((g / kPfStages) & 1), p.status, abort) ||
            !tc_wait(&bar[kPfSFree + sb], (uint32_t)(((g >> 1) & 1) ^ 1), p.status, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dK = dK0 + (uint64_t)((st * 2 * L::TILE) >> 4);
        #pragma unroll
        for (int k = 0; k < kPfD / 16; ++k)
          umma_f16(tmem + kPfN * sb, dQ + kstep(k), dK + kstep(k), idS, k > 0 ? 1u : 0u);
        umma_commit(&bar[kPfSFull + sb]);
        if (g > 0 && !pv(g - 1)) { ok = false; break; }
      }
      if (ok && nkb > 0 && !pv(nkb - 1)) ok = false;
      if (!ok) *abort = 1;
      umma_commit(&bar[kPfFin]);
      mbar_wait(&bar[kPfFin], 0, nullptr);
    }
    __syncwarp();
  } else {
    // ===================================================================== softmax group
    const int r = threadIdx.x;  // query row of the block = tensor-memory lane
    const int t = t0 + r;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const uint32_t tO = tmem + lane_off + 2 * kPfN;
    // ---- Q row t into its K-major swizzled place (zero past T)
    {
      uint4 x[16];
      const bool has = t < p.T;
      const uint4* src = reinterpret_cast<const uint4*>(p.q + (((int64_t)b * p.T + t) * p.Hq + qh) * kPfD);
      #pragma unroll
      for (int c = 0; c < 16; ++c) x[c] = has ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      #pragma unroll
      for (int c = 0; c < 16; ++c)  // chunk c: head dims 8c .. 8c + 7
        *reinterpret_cast<uint4*>(sm + L::OFF_Q + (c >> 3) * L::ATOM + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = x[c];
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[kPfQReady]);

    const int lim = t < p.T ? Lb - p.T + t : -1;  // the last key this row sees
    float mref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int g = 0; g < nkb; ++g) {
      const int sb = g & 1;
      if (!tc_wait_warp(&bar[kPfSFull + sb], (uint32_t)((g >> 1) & 1), p.status, abort)) { ok = false; break; }
      tc_fence_after();
      float s[kPfN];
      #pragma unroll
      for (int q4 = 0; q4 < kPfN / 32; ++q4) {
        float v[32];
        tmem_ld32(tmem + lane_off + kPfN * sb + 32 * q4, v);
        #pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * q4 + i] = v[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kPfSFree + sb]);
      // ---- scale, mask (keys past the row's limit or the request), block maximum
      const int j0 = g * kPfN;
      const int nvis = min(kPfN, min(lim, Lb - 1) - j0 + 1);  // keys j0 .. j0 + nvis - 1 are visible
      float bm = -INFINITY;
      #pragma unroll
      for (int i = 0; i < kPfN; ++i) {
        s[i] = i < nvis ? s[i] * p.qk_scale_log2 : -INFINITY;
        bm = fmaxf(bm, s[i]);
      }
      bool pv_waited = false;
      float alpha = 1.f;
      if (bm > mref + (float)kPfTau) {
        // the row's reference moves to this block's maximum; O's row is rescaled in place
        alpha = mref == -INFINITY ? 0.f : fast_exp2(mref - bm);
        l *= alpha;
        mref = bm;
      }
      // tensor-memory loads and stores are warp-wide: the warp rescales when any of its rows
      // needs it (alpha = 1 for the others)
      if (g > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!tc_wait_warp(&bar[kPfPvDone], (uint32_t)((g - 1) & 1), p.status, abort)) { ok = false; break; }
        pv_waited = true;
        tc_fence_after();
        #pragma unroll
        for (int q4 = 0; q4 < kPfD / 32; ++q4) {
          float o[32];
          tmem_ld32(tO + 32 * q4, o);
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + 32 * q4, o);
        }
      }
      // ---- P = 2^(s - m_ref) (at most 2^kPfTau), row sum, bf16 into the P tile (after the
      //      previous block's P V has read it)
      const float mu = mref == -INFINITY ? 0.f : mref;
      #pragma unroll
      for (int i = 0; i < kPfN; ++i) {
        s[i] = fast_exp2(s[i] - mu);
        l += s[i];
      }
      if (g > 0 && !pv_waited && !tc_wait_warp(&bar[kPfPvDone], (uint32_t)((g - 1) & 1), p.status, abort)) {
        ok = false;
        break;
      }
      #pragma unroll
      for (int c = 0; c < 16; ++c) {  // keys 8c .. 8c + 7
        const uint4 w = make_uint4(pack_bf16(s[8 * c], s[8 * c + 1]), pack_bf16(s[8 * c + 2], s[8 * c + 3]),
                                   pack_bf16(s[8 * c + 4], s[8 * c + 5]), pack_bf16(s[8 * c + 6], s[8 * c + 7]));
        *reinterpret_cast<uint4*>(sm + L::OFF_P + (c >> 3) * L::ATOM + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = w;
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kPfPReady]);
    }
    // ---- epilogue: O / l and lse of row t
    if (ok && nkb > 0 && !tc_wait_warp(&bar[kPfPvDone], (uint32_t)((nkb - 1) & 1), p.status, abort)) ok = false;
    if (!ok) *abort = 1;
    if (ok) {  // warp-uniform: every lane takes part in the tensor-memory loads
      tc_fence_after();
      const bool has = t < p.T;
      const int64_t row = ((int64_t)b * p.T + (has ? t : 0)) * p.Hq + qh;
      float4* dst = reinterpret_cast<float4*>(p.out + row * kPfD);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      #pragma unroll
      for (int q4 = 0; q4 < kPfD / 32; ++q4) {
        float o[32];
        if (nkb > 0) {
          tmem_ld32(tO + 32 * q4, o);
        } else {
          #pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (has) {
          #pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[8 * q4 + i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        }
      }
      if (has) p.lse[row] = l > 0.f ? (mref + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kPfTmemCols) : "memory");
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t st) {
  const int smem = PfSmem::ALLOC;
  if (!ensure_smem_attr((const void*)prefill_kernel, smem)) return cudaErrorInvalidValue;
  const int nqb = (p.T + kPfM - 1) / kPfM;
  if (p.B == 0 || nqb == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nqb, p.Hq, p.B);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, prefill_kernel, p, tmK, tmV);
}

}  // namespace decattn
