// append.cu -- the fused pre-processing of a decode step: rotary position embedding of the
// step's new q and k rows, and the append of the new K/V rows into their pages, in one kernel
// ("PaddlePaddle/HALOps" README, Highlights, GQA attention item: fused pre/post-processing
// around paged-KV decode). The pages name the step without defining it; this kernel computes:
//  * rotate-half rotary embedding: for i < d/2, theta_i = base^(-2i/d); the pair
//    (x_i, x_{i+d/2}) at position pos becomes
//    (x_i cos(pos theta_i) - x_{i+d/2} sin(pos theta_i), x_{i+d/2} cos(pos theta_i) + x_i sin(pos theta_i));
//  * token t of request b sits at position Lb - T + t (seq_lens already counts the new tokens,
//    as the decode does);
//  * rotated q goes to q_out; rotated k and unchanged v go to page page_table[b][pos / P], slot
//    pos % P, of their KV head; a token with pos < 0 has no slot (its q is left unrotated).
//
// Block (token, g) takes rows 8g .. 8g+7 of the token's Hq + 2 Hkv rows (q heads, then k,
// then v), one warp per row, so that every row's load is in flight at once. The block first
// forms (cos, sin) of pos * theta_i in fp64 (theta_i comes from the host in fp64; pos * theta
// in fp32 would be off by up to ~0.016 rad at pos = 131072). Lane l holds elements
// [E l, E l + E) of both halves of its row, so each rotation pair sits in one lane; values are
// rotated in fp32 and rounded to bf16 (RNE).
#include <cmath>

#include "common.cuh"
#include "host_errors.h"

namespace decattn {

constexpr int kAppendWarps = 8;  // rows per block
constexpr int kAppendThreads = 32 * kAppendWarps;
constexpr int kAppendMaxHalf = 64;  // head_dim <= 128

struct AppendParams {
  const uint16_t* q_new;   // bf16 [B][T][Hq][D]
  const uint16_t* k_new;   // bf16 [B][T][Hkv][D]
  const uint16_t* v_new;   // bf16 [B][T][Hkv][D]
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint16_t* q_out;         // bf16 [B][T][Hq][D] (may be q_new)
  uint16_t* k_pages;       // bf16 [num_pages][Hkv][P][D]
  uint16_t* v_pages;
  int32_t* status;         // optional device word: DECATTN_EDEVICE for a bad page id
  int B, T, Hq, Hkv, P, num_pages, mpps;
  int rows;                       // rows per token this kernel writes: Hq + 2 Hkv (bf16 pages) or Hq (FP8)
  int groups;                     // row groups of kAppendWarps rows per token
  double theta[kAppendMaxHalf];   // base^(-2i/d), i < d/2
};

// The K / V side of the step for E4M3 pages (one fp32 scale per (page, KV head) and K or V): one
// block per (request, page touched by the new tokens, KV head, K or V), one thread per head dim.
struct AppendFp8Params {
  const uint16_t* k_new;   // bf16 [B][T][Hkv][D]
  const uint16_t* v_new;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint8_t* k_pages;        // E4M3 codes [num_pages][Hkv][P][D]
  uint8_t* v_pages;
  float* kv_scales;        // [2][num_pages][Hkv]
  int32_t* status;
  int B, T, Hkv, P, num_pages, mpps;
  int maxpg;                      // pages the T new tokens of a request can touch
  double theta[kAppendMaxHalf];
};

template <int E>
struct AppendVec;
template <>
struct AppendVec<1> { using T = uint16_t; };
template <>
struct AppendVec<2> { using T = uint32_t; };

template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_rope_kernel(const AppendParams p) {
  constexpr int HALF = D / 2;
  constexpr int E = D / 64;  // elements of each half per lane
  using V = typename AppendVec<E>::T;
  __shared__ float2 cs[HALF];  // (cos, sin) of pos * theta_i
  // the inputs are written by the previous kernel of the stream
  griddep_wait();
  const int bt = blockIdx.x / p.groups, grp = blockIdx.x - bt * p.groups;
  const int b = bt / p.T, t = bt - b * p.T;
  const int64_t pos = (int64_t)p.seq_lens[b] - p.T + t;
  const double rpos = pos < 0 ? 0.0 : (double)pos;
  // this warp's row (q heads, then k, then v): its loads go out before the shared work below
  const int lane = threadIdx.x & 31;
  const int r = grp * kAppendWarps + (threadIdx.x >> 5);
  const bool has_row = r < p.rows;
  const bool is_q = r < p.Hq, is_k = !is_q && r < p.Hq + p.Hkv;
  const int h = is_q ? 0 : is_k ? r - p.Hq : r - p.Hq - p.Hkv;
  const uint16_t* src = is_q ? p.q_new + ((int64_t)bt * p.Hq + r) * D
                             : (is_k ? p.k_new : p.v_new) + ((int64_t)bt * p.Hkv + h) * D;
  V lo = 0, hi = 0;
  if (has_row) {
    lo = reinterpret_cast<const V*>(src)[lane];
    hi = reinterpret_cast<const V*>(src + HALF)[lane];
  }
  for (int i = threadIdx.x; i < HALF; i += kAppendThreads) {
    double s, c;
    sincos(rpos * p.theta[i], &s, &c);
    cs[i] = make_float2((float)c, (float)s);
  }
  // the page slot of this token (none for pos < 0, or for a bad page id, which is reported)
  int64_t slot_row = -1;  // (page * Hkv) * P + slot, before adding the head
  if (pos >= 0) {
    const int64_t pg = pos / p.P;
    int pid = -1;
    if (pg < p.mpps) pid = p.page_table[(int64_t)b * p.mpps + pg];
    if (pid >= 0 && pid < p.num_pages) {
      slot_row = (int64_t)pid * p.Hkv * p.P + pos % p.P;
    } else if (threadIdx.x == 0 && grp == 0) {
      set_status(p.status, DECATTN_EDEVICE);
    }
  }
  __syncthreads();

  if (!has_row) return;
  uint16_t* dst;
  if (is_q) {
    dst = p.q_out + ((int64_t)bt * p.Hq + r) * D;
  } else {
    if (slot_row < 0) return;
    dst = (is_k ? p.k_pages : p.v_pages) + (slot_row + (int64_t)h * p.P) * D;
  }
  if (!is_q && !is_k) {
    reinterpret_cast<V*>(dst)[lane] = lo;
    reinterpret_cast<V*>(dst + HALF)[lane] = hi;
    return;
  }
  {
    float x1[E], x2[E];
    #pragma unroll
    for (int e = 0; e < E; ++e) {
      x1[e] = __uint_as_float((uint32_t)((lo >> (16 * e)) & 0xffffu) << 16);
      x2[e] = __uint_as_float((uint32_t)((hi >> (16 * e)) & 0xffffu) << 16);
    }
    V olo = 0, ohi = 0;
    #pragma unroll
    for (int e = 0; e < E; ++e) {
      const float2 c = cs[E * lane + e];
      const float y1 = x1[e] * c.x - x2[e] * c.y;
      const float y2 = x2[e] * c.x + x1[e] * c.y;
      olo |= (V)((V)__bfloat16_as_ushort(__float2bfloat16_rn(y1)) << (16 * e));
      ohi |= (V)((V)__bfloat16_as_ushort(__float2bfloat16_rn(y2)) << (16 * e));
    }
    reinterpret_cast<V*>(dst)[lane] = olo;
    reinterpret_cast<V*>(dst + HALF)[lane] = ohi;
  }
}

// E4M3 pages: the page's scale covers its valid rows (|value| <= 448 * scale). With x the new rows'
// values (k rotated as in append_rope_kernel, in fp32) and A = max |x| over the page's new rows, the
// scale becomes max(s, A / 448) if the page holds older rows (its slots before the first new one),
// else A / 448 (1 when A = 0); older codes are re-rounded, E4M3(value * (s / s')), only when the
// scale grows; new rows are E4M3(x / s'). Every rounding is fp32 then round-to-nearest-even
// (saturating) to E4M3.
template <int D>
__global__ void __launch_bounds__(D) append_fp8_kernel(const AppendFp8Params p) {
  constexpr int HALF = D / 2;
  __shared__ float wmax[D / 32];
  griddep_wait();  // the pages and scales were last touched by earlier kernels of the stream
  const int b = blockIdx.x / p.maxpg, pi = blockIdx.x - b * p.maxpg;
  const int h = blockIdx.y, which = blockIdx.z;  // 0: K, 1: V
  const int L = p.seq_lens[b];
  const int first = max(L - p.T, 0);  // the first new position with a slot
  if (L <= first) return;
  const int pg = first / p.P + pi;
  if (pg * p.P >= L) return;
  const int lo = max(first, pg * p.P), hi = min(L, pg * p.P + p.P);  // new positions in this page
  const int s_first = lo - pg * p.P;
  const int pid = pg < p.mpps ? p.page_table[(int64_t)b * p.mpps + pg] : -1;
  if (pid < 0 || pid >= p.num_pages) {
    if (threadIdx.x == 0) set_status(p.status, DECATTN_EDEVICE);
    return;
  }
  const int d = threadIdx.x;
  const uint16_t* src = which == 0 ? p.k_new : p.v_new;
  auto bf = [](uint16_t u) { return __uint_as_float((uint32_t)u << 16); };
  // element d of the new row at position pos (k: rotated)
  auto value = [&](int pos) -> float {
    const uint16_t* row = src + (((int64_t)b * p.T + (pos - (L - p.T))) * p.Hkv + h) * D;
    const float x = bf(row[d]);
    if (which == 1) return x;
    const int i = d < HALF ? d : d - HALF;
    const float xp = bf(row[d < HALF ? d + HALF : d - HALF]);
    double sn, cs;
    sincos((double)pos * p.theta[i], &sn, &cs);
    const float c = (float)cs, sf = (float)sn;
    return d < HALF ? x * c - xp * sf : x * c + xp * sf;
  };
  float amax = 0.f;
  for (int pos = lo; pos < hi; ++pos) amax = fmaxf(amax, fabsf(value(pos)));
  const int64_t si = ((int64_t)which * p.num_pages + pid) * p.Hkv + h;
  const float s_old = p.kv_scales[si];  // read by every thread before the barrier below
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((d & 31) == 0) wmax[d >> 5] = amax;
  __syncthreads();
  #pragma unroll
  for (int w = 0; w < D / 32; ++w) amax = fmaxf(amax, wmax[w]);
  const float s_new = s_first > 0 ? fmaxf(s_old, amax / 448.f) : (amax > 0.f ? amax / 448.f : 1.f);
  uint8_t* base = (which == 0 ? p.k_pages : p.v_pages) + ((int64_t)pid * p.Hkv + h) * p.P * D;
  if (s_first > 0 && s_new != s_old) {
    const float r = s_old / s_new;
    for (int sl = 0; sl < s_first; ++sl) {
      const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(base[sl * D + d]), __NV_E4M3);
      const float v = __half2float(__half(hr)) * r;
      base[sl * D + d] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
    }
  }
  for (int pos = lo; pos < hi; ++pos)
    base[(pos - pg * p.P) * D + d] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(value(pos) / s_new, __NV_SATFINITE, __NV_E4M3));
  if (d == 0) p.kv_scales[si] = s_new;
}

cudaError_t launch_append_fp8(const AppendFp8Params& p, int D, cudaStream_t st) {
  const int64_t blocks = (int64_t)p.B * p.maxpg;
  if (blocks <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, (unsigned)p.Hkv, 2);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, append_fp8_kernel<128>, p);
  if (D == 64) return cudaLaunchKernelEx(&cfg, append_fp8_kernel<64>, p);
  return cudaErrorInvalidValue;
}

cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t st) {
  const int64_t blocks = (int64_t)p.B * p.T * p.groups;
  if (blocks <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kAppendThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // launched while the previous kernel drains
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, append_rope_kernel<128>, p);
  if (D == 64) return cudaLaunchKernelEx(&cfg, append_rope_kernel<64>, p);
  return cudaErrorInvalidValue;
}

// Argument checks shared by both entry points; fills the row kernel's parameters.
static int append_setup(const dec_attn_shape* shape, const void* q_new, const void* k_new, const void* v_new,
                        const int32_t* page_table, const int32_t* seq_lens, float rope_base, void* q_out,
                        void* k_pages, void* v_pages, int32_t* status, bool fp8, AppendParams& p) {
  if (!shape) return DECATTN_EINVAL;
  const dec_attn_shape& s = *shape;
  if (s.batch < 0 || s.q_tokens <= 0 || s.n_q_heads <= 0 || s.n_kv_heads <= 0 || s.page_size <= 0 ||
      s.num_pages < 0 || s.max_pages_per_seq < 0 || s.n_q_heads % s.n_kv_heads != 0)
    return DECATTN_EINVAL;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return DECATTN_EINVAL;
  if (fp8 ? (s.kv_dtype != DECATTN_KV_FP8E4M3 && s.kv_dtype != DECATTN_KV_FP8E4M3_MMA8)
          : s.kv_dtype != DECATTN_KV_BF16)
    return DECATTN_ENOTSUP;
  if (s.head_dim != 64 && s.head_dim != 128) return DECATTN_ENOTSUP;
  if (s.batch == 0) return DECATTN_OK;
  if (!q_new || !k_new || !v_new || !page_table || !seq_lens || !q_out || !k_pages || !v_pages)
    return DECATTN_EINVAL;
  const uintptr_t need = s.head_dim == 128 ? 3 : 1;  // 4-byte (d = 128) or 2-byte lane accesses
  for (const void* ptr : {q_new, k_new, v_new, (const void*)q_out})
    if (reinterpret_cast<uintptr_t>(ptr) & need) return DECATTN_EALIGN;
  if (!fp8)
    for (const void* ptr : {(const void*)k_pages, (const void*)v_pages})
      if (reinterpret_cast<uintptr_t>(ptr) & need) return DECATTN_EALIGN;
  p.q_new = static_cast<const uint16_t*>(q_new);
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.q_out = static_cast<uint16_t*>(q_out);
  p.k_pages = fp8 ? nullptr : static_cast<uint16_t*>(k_pages);
  p.v_pages = fp8 ? nullptr : static_cast<uint16_t*>(v_pages);
  p.status = status;
  p.B = s.batch; p.T = s.q_tokens; p.Hq = s.n_q_heads; p.Hkv = s.n_kv_heads; p.P = s.page_size;
  p.num_pages = s.num_pages; p.mpps = s.max_pages_per_seq;
  p.rows = fp8 ? s.n_q_heads : s.n_q_heads + 2 * s.n_kv_heads;
  p.groups = (p.rows + kAppendWarps - 1) / kAppendWarps;
  for (int i = 0; i < s.head_dim / 2; ++i) p.theta[i] = std::pow((double)rope_base, -2.0 * i / s.head_dim);
  if ((int64_t)s.batch * s.q_tokens * p.groups > 0x7fffffff) return DECATTN_ENOTSUP;
  return 1;  // arguments good, work to launch
}

}  // namespace decattn

using namespace decattn;

extern "C" int dec_attn_append_rope(const dec_attn_shape* shape, const void* q_new, const void* k_new,
                                    const void* v_new, const int32_t* page_table, const int32_t* seq_lens,
                                    float rope_base, void* q_out, void* k_pages, void* v_pages, int32_t* status,
                                    void* stream) {
  AppendParams p;
  const int rc = append_setup(shape, q_new, k_new, v_new, page_table, seq_lens, rope_base, q_out, k_pages, v_pages,
                              status, false, p);
  if (rc <= 0) return rc;
  const cudaError_t e = launch_append(p, shape->head_dim, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DECATTN_OK : cuda_fail("append kernel launch", e);
}

extern "C" int dec_attn_append_rope_fp8(const dec_attn_shape* shape, const void* q_new, const void* k_new,
                                        const void* v_new, const int32_t* page_table, const int32_t* seq_lens,
                                        float rope_base, void* q_out, void* k_pages, void* v_pages, float* kv_scales,
                                        int32_t* status, void* stream) {
  AppendParams p;
  const int rc = append_setup(shape, q_new, k_new, v_new, page_table, seq_lens, rope_base, q_out, k_pages, v_pages,
                              status, true, p);
  if (rc <= 0) return rc;
  if (!kv_scales) return DECATTN_EINVAL;
  if ((reinterpret_cast<uintptr_t>(kv_scales) & 3) != 0) return DECATTN_EALIGN;
  const dec_attn_shape& s = *shape;
  AppendFp8Params f;
  f.k_new = p.k_new;
  f.v_new = p.v_new;
  f.page_table = page_table;
  f.seq_lens = seq_lens;
  f.k_pages = static_cast<uint8_t*>(k_pages);
  f.v_pages = static_cast<uint8_t*>(v_pages);
  f.kv_scales = kv_scales;
  f.status = status;
  f.B = s.batch; f.T = s.q_tokens; f.Hkv = s.n_kv_heads; f.P = s.page_size; f.num_pages = s.num_pages;
  f.mpps = s.max_pages_per_seq;
  f.maxpg = (s.q_tokens + s.page_size - 1) / s.page_size + 1;
  for (int i = 0; i < s.head_dim / 2; ++i) f.theta[i] = p.theta[i];
  if ((int64_t)s.batch * f.maxpg > 0x7fffffff || s.n_kv_heads > 65535) return DECATTN_ENOTSUP;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_append(p, s.head_dim, st);  // q rows
  if (e != cudaSuccess) return cuda_fail("append kernel launch", e);
  e = launch_append_fp8(f, s.head_dim, st);          // K / V pages and scales
  return e == cudaSuccess ? DECATTN_OK : cuda_fail("FP8 append kernel launch", e);
}
