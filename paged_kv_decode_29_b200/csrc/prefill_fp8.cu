// prefill_fp8.cu -- prefill over an FP8 (E4M3) KV cache ("PaddlePaddle/HALOps" README,
// Highlights, GQA attention item: prefill and paged-KV decode across BF16 / FP8 KV caches).
//
// Prefill is a dense contraction (tensor bound), and its bf16 kernel keeps two 128-row query
// tiles, a two-stage K ring and a two-stage V ring in shared memory, which leaves no room for an
// E4M3 staging ring beside them. So FP8 pages are widened first: one pass reads the E4M3 codes of
// the pages a request uses and writes code * (page scale) rounded to bf16 into a scratch pool
// laid out like a bf16 pool (scratch page b * max_pages_per_seq + i holds page i of request b),
// with its own page table; the bf16 prefill kernel then runs on it. The pass moves 3 bytes per
// element once (about 1 + 2 bytes; the prefill kernel reads K and V many times over from L2).
//
// Reading: the tensor cores see K and V as RN_bf16(RN_fp32(code * scale)) (relative error at most
// 2^-9 per element, plus one fp32 rounding of the product), where the oracle uses code * scale
// exactly; the tolerance of the result is derived from that bound.
#include "common.cuh"

namespace decattn {

constexpr int kWidenThreads = 128;

// CTA (w, y): scratch page w = b * mpps + i (page i of request b), y = kv * Hkv + h: K (kv = 0) or V
// of KV head h, one 16-code chunk per thread. Pages past the request's keys are never read by the
// prefill kernel and are left unwritten; a page id outside the pool is reported (DECATTN_EDEVICE)
// and its scratch page is zero.
__global__ void __launch_bounds__(kWidenThreads) widen_kv_kernel(const WidenParams p) {
  // 32-bit index arithmetic (the page index is below 2^31: the grid's x size): a 64-bit division
  // is a software routine, and every CTA converts only one slice
  const int w = (int)blockIdx.x;
  const int kv = (int)blockIdx.y / p.Hkv, h = (int)blockIdx.y - kv * p.Hkv;
  const int b = w / p.mpps;
  const int i = w - b * p.mpps;
  if (threadIdx.x == 0 && blockIdx.y == 0) p.pt_out[w] = (int32_t)w;
  const int Lb = p.seq_lens[b];
  if (Lb < 0) {
    if (threadIdx.x == 0 && i == 0 && blockIdx.y == 0) set_status(p.status, DECATTN_EDEVICE);
    return;
  }
  if ((int64_t)i * p.P >= Lb) return;
  const int pid = p.page_table[w];
  const bool good = pid >= 0 && pid < p.num_pages;
  if (!good && threadIdx.x == 0 && blockIdx.y == 0) set_status(p.status, DECATTN_EDEVICE);
  const float s = good ? p.kv_scales[(int64_t)kv * p.num_pages * p.Hkv + (int64_t)pid * p.Hkv + h] : 0.f;
  const uint8_t* src = (kv ? p.v_codes : p.k_codes) + ((int64_t)(good ? pid : 0) * p.Hkv + h) * p.P * p.D;
  uint16_t* dst = (kv ? p.v_out : p.k_out) + ((int64_t)w * p.Hkv + h) * p.P * p.D;
  const int per_slice = p.P * p.D / 16;  // 16-code chunks of the (page, KV head) slice
  for (int c = threadIdx.x; c < per_slice; c += kWidenThreads) {
    uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (good) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(src + 16 * c));
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      #pragma unroll
      for (int q = 0; q < 4; ++q) {
        #pragma unroll
        for (int half = 0; half < 2; ++half) {  // two codes at a time: exact in f16, then times s
          const float2 f = f16x2_to_float2(e4m3x2_to_f16x2(half ? (xw[q] >> 16) : (xw[q] & 0xffffu)));
          o[2 * q + half] = pack_bf16(f.x * s, f.y * s);
        }
      }
    }
    reinterpret_cast<uint4*>(dst + 16 * c)[0] = make_uint4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<uint4*>(dst + 16 * c)[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

int64_t widen_scratch_bytes(int B, int mpps, int Hkv, int P, int D, int64_t* off_v, int64_t* off_pt) {
  const int64_t kv = align_up((int64_t)B * mpps * Hkv * P * D * 2, 256);
  if (off_v) *off_v = kv;
  if (off_pt) *off_pt = 2 * kv;
  return 2 * kv + align_up((int64_t)B * mpps * 4, 256);
}

cudaError_t launch_widen_kv(const WidenParams& p, cudaStream_t st) {
  const int64_t grid = (int64_t)p.B * p.mpps;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffff || 2 * p.Hkv > 65535) return cudaErrorInvalidValue;
  widen_kv_kernel<<<dim3((unsigned)grid, (unsigned)(2 * p.Hkv)), kWidenThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace decattn
