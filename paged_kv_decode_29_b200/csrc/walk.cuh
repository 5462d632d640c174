// walk.cuh -- the full tiles of a bin, listed from seq_lens without the plan. Used by the
// producer warps of both split kernels.
#pragma once
#include "common.cuh"

namespace decattn {

// ------------------------------------------------------------------ full tiles without the plan
// The greedy rule deals the full tiles round-robin: full tile f (counted in (b, h, i) order)
// lands in bin f mod N at position f div N, ahead of every partial tile. A CTA can therefore
// list its own full tiles from seq_lens alone and stream them while the planner is still
// running; only its partial tiles wait for the plan. The walk runs in the producer warp
// (every lane returns the same tile). It is used when the batch fits its 32 windows of 32
// requests and the planner's device-side checks are known to pass (no negative length, tile
// count within the capacity); otherwise every tile comes from the plan.
constexpr int kWalkMaxReq = 32 * 32;

struct FullTileWalk {
  int fc;             // full tiles of this bin listed by the walk (0: all come from the plan)
  int nwin;           // windows holding requests
  long long wsf, ws;  // lane l: full tiles / tiles of one KV head in the requests before window l
  int cur;            // window cached below (-1: none)
  int L;              // lane i: length of request 32 cur + i
  int nf_in, nb_in;   // lane i: inclusive prefix of full tiles / tiles over the cached window
  long long csf, cs;  // wsf, ws of the cached window
  uint32_t F;         // full tiles of all bins (valid when nwin > 0)
};

// bin: this CTA's bin of the nbins bins.
__device__ __forceinline__ void walk_init(FullTileWalk& w, const SplitParams& p, int lane, int bin, int nbins) {
  w.fc = 0; w.nwin = 0; w.wsf = 0; w.ws = 0; w.cur = -1;
  w.L = 0; w.nf_in = 0; w.nb_in = 0; w.csf = 0; w.cs = 0; w.F = 0;
  if (p.sparse || p.B > kWalkMaxReq || p.tile_len <= 0) return;  // a sparse plan lists every tile
  const uint32_t tl = (uint32_t)p.tile_len;  // 32-bit divisions: the 64-bit ones are software routines
  const int nwin = (p.B + 31) / 32;
  // window sums, one window per iteration (coalesced, the next window's load in flight); lane l
  // keeps window l. A request with more than 2^26 tiles turns the walk off, so that a window
  // sum fits 32 bits.
  uint32_t my_sf = 0, my_sb = 0;
  bool bad = false;
  int Lnext = lane < p.B ? __ldg(p.seq_lens + lane) : 0;
  #pragma unroll 1
  for (int w0 = 0; w0 < nwin; ++w0) {
    const int L = Lnext;
    const int bn = 32 * (w0 + 1) + lane;
    Lnext = bn < p.B ? __ldg(p.seq_lens + bn) : 0;
    const uint32_t Lu = L < 0 ? 0u : (uint32_t)L, nf = Lu / tl, nb = nf + (Lu != nf * tl ? 1u : 0u);
    bad |= L < 0 || nb > (1u << 26);
    const uint32_t sf = __reduce_add_sync(0xffffffffu, nf), sb = __reduce_add_sync(0xffffffffu, nb);
    if (lane == w0) { my_sf = sf; my_sb = sb; }
  }
  long long isf = my_sf, isb = my_sb;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long a = __shfl_up_sync(0xffffffffu, isf, o), c = __shfl_up_sync(0xffffffffu, isb, o);
    if (lane >= o) { isf += a; isb += c; }
  }
  const long long F = (long long)p.Hkv * __shfl_sync(0xffffffffu, isf, 31);
  const long long U = (long long)p.Hkv * __shfl_sync(0xffffffffu, isb, 31);
  // the planner reports a negative length or too many tiles; the tile and slot arithmetic
  // below is 32-bit
  if (__any_sync(0xffffffffu, bad) || U > p.max_units || U >= (1ll << 31)) return;
  w.wsf = isf - my_sf;
  w.ws = isb - my_sb;
  w.nwin = nwin;
  const uint32_t N = (uint32_t)nbins, Fu = (uint32_t)F;
  w.F = Fu;
  w.fc = (int)(Fu / N + ((uint32_t)bin < Fu % N ? 1u : 0u));
}

// The same walk for another bin (the window sums do not depend on the bin).
__device__ __forceinline__ void walk_rebin(FullTileWalk& w, int bin, int nbins) {
  if (w.nwin == 0) return;  // the walk is off: every tile comes from the plan
  const uint32_t N = (uint32_t)nbins;
  w.fc = (int)(w.F / N + ((uint32_t)bin < w.F % N ? 1u : 0u));
}

// The j-th full tile of this CTA's bin (j < fc); the same tile plan_unit() decodes.
__device__ __forceinline__ Unit walk_unit(FullTileWalk& w, const SplitParams& p, int lane, int j, int bin, int nbins) {
  const uint32_t tl = (uint32_t)p.tile_len;
  const int Hkv = p.Hkv;
  const long long f = (long long)bin + (long long)nbins * j;
  // window: the last one whose first full tile is <= f
  const int win = 31 - __clz(__ballot_sync(0xffffffffu, lane < w.nwin && (long long)Hkv * w.wsf <= f));
  if (win != w.cur) {
    const int b = 32 * win + lane;
    w.L = b < p.B ? __ldg(p.seq_lens + b) : 0;
    const uint32_t Lu = (uint32_t)w.L, q = Lu / tl;
    int nf = (int)q, nb = (int)(q + (Lu != q * tl ? 1u : 0u));
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, nf, o), c = __shfl_up_sync(0xffffffffu, nb, o);
      if (lane >= o) { nf += a; nb += c; }
    }
    w.nf_in = nf; w.nb_in = nb;
    w.csf = __shfl_sync(0xffffffffu, w.wsf, win);
    w.cs = __shfl_sync(0xffffffffu, w.ws, win);
    w.cur = win;
  }
  // request: the first one of the window whose full tiles reach past f
  const int i = __ffs(__ballot_sync(0xffffffffu, (long long)Hkv * (w.csf + w.nf_in) > f)) - 1;
  const int L = __shfl_sync(0xffffffffu, w.L, i);
  const int nfi = __shfl_sync(0xffffffffu, w.nf_in, i), nbi = __shfl_sync(0xffffffffu, w.nb_in, i);
  const uint32_t Lu = (uint32_t)L, fb = Lu / tl, nb = fb + (Lu != fb * tl ? 1u : 0u);
  const long long SFb = w.csf + nfi - (int)fb, Sb = w.cs + nbi - (int)nb;
  const uint32_t r = (uint32_t)(f - (long long)Hkv * SFb);
  const uint32_t hh = r / fb, it = r - hh * fb;
  Unit u;
  u.b = 32 * win + i; u.h = (int)hh; u.tok_begin = (int)(it * tl); u.tok_end = (int)((it + 1) * tl);
  u.seq_len = L;
  u.slot = nb == 1 ? -1 : (int)(Hkv * Sb + (long long)hh * nb + it);
  u.tile = (int)it; u.zero = 0;
  return u;
}

}  // namespace decattn
