// api.cu -- the C ABI front end: argument checks, workspace layout, TMA tensor maps and
// the launches of the split and combine kernels. See include/decattn.h for the contract.
#include <math.h>
#include <stddef.h>

#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "host_errors.h"

namespace decattn {

static std::mutex g_mu;

// The CUDA error behind the last DECATTN_ECUDA of this host thread (dec_attn_last_error).
static thread_local char g_last_error[256] = "";

int cuda_fail(const char* what, cudaError_t e) {
  if (e == cudaSuccess) e = cudaPeekAtLastError();
  snprintf(g_last_error, sizeof g_last_error, "%s: %s", what,
           e == cudaSuccess ? "failed without a CUDA runtime error (a driver-API call)" : cudaGetErrorString(e));
  return DECATTN_ECUDA;
}

// Wait limit and left-out fill of the next launches (dec_attn_test_set_waits): the library's
// default unless a test of the bounded waits lowers them.
static uint64_t g_test_wait_ns = kWaitLimitNs;
static int32_t g_test_skip_fill = -1;

void test_waits(uint64_t* wait_ns, int32_t* skip_fill) {
  std::lock_guard<std::mutex> lk(g_mu);
  *wait_ns = g_test_wait_ns;
  *skip_fill = g_test_skip_fill;
}

int default_bins(int device) {
  static std::map<int, int> cache;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = cache.find(device);
  if (it != cache.end()) return it->second;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) return -1;
  const int n = sms * split_ctas_per_sm();
  cache[device] = n;
  return n;
}

bool ensure_smem_attr(const void* kernel, int bytes) {
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(kernel, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done[key] = bytes;
  return true;
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// K or V pool viewed as a 2-D tensor: x = head_dim elements, y = (page * Hkv + h) * P + slot.
// A box is 16 rows of 128 (or 64) bytes, swizzled to match the kernel's ldmatrix reads.
static bool make_kv_map(CUtensorMap* map, const void* base, int kv_dtype, int D, int64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int esz = kv_dtype == DECATTN_KV_BF16 ? 2 : 1;
  const int row_bytes = D * esz;
  const int box_bytes = row_bytes >= 128 ? 128 : row_bytes;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(box_bytes / esz), 16};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      kv_dtype == DECATTN_KV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapSwizzle sw = box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Prefill queries as a 3-D bf16 tensor {head dim, q head, packed row} (q is [rows][Hq][D]); the
// kernel loads boxes of 64 head dims x 128 rows with 128-byte swizzle, the K-major layout of the
// MMA's A operand. Rows past the last one read as zeros.
static bool make_prefill_q_map(CUtensorMap* map, const void* q, int64_t rows, int Hq, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Prefill output as a 3-D fp32 tensor {head dim, q head, packed row} (out is [rows][Hq][D]); the
// kernel stores boxes of 32 rows x 32 head dims with 128-byte swizzle, only boxes whose rows all
// belong to one request (the ragged last box of a request is written with plain stores).
static bool make_prefill_out_map(CUtensorMap* map, float* out, int64_t rows, int Hq, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)Hq * D * 4};
  cuuint32_t box[3] = {32, 1, 32};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

struct WsLayout {
  int64_t off_part_lse, off_part_o, off_row_cnt, off_chunk, total;
  int64_t items;  // bound on the combine's (row, chunk) items
};

// Workspace: reserved header | partial lse [units][GT] | partial o [units][GT][D] |
// combine row counters [B*T*Hq] | combine chunk states [items][D + 4].
static WsLayout ws_layout(int64_t max_units, const dec_attn_shape& s) {
  const int GT = s.n_q_heads / s.n_kv_heads * s.q_tokens;
  const int D = s.head_dim;
  const int64_t rows = (int64_t)s.batch * s.q_tokens * s.n_q_heads;
  const int64_t items = (int64_t)GT * ((max_units + kCombineChunk - 1) / kCombineChunk) + rows;
  WsLayout w;
  int64_t o = sizeof(WorkspaceHeader);
  w.off_part_lse = o; o = align_up(o + 4 * max_units * GT, 256);
  w.off_part_o = o; o = align_up(o + 4 * max_units * GT * D, 256);
  w.off_row_cnt = o; o = align_up(o + 4 * rows, 256);
  w.off_chunk = o; o = align_up(o + 4 * items * (D + 4), 256);
  w.total = o;
  w.items = items;
  return w;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int check_shape(const dec_attn_shape* s, const dec_attn_plan_t* pl) {
  if (!s || !pl) return DECATTN_EINVAL;
  if (s->batch < 0 || s->n_q_heads <= 0 || s->n_kv_heads <= 0 || s->q_tokens <= 0 || s->page_size <= 0 ||
      s->num_pages < 0 || s->max_pages_per_seq < 0 || s->head_dim <= 0)
    return DECATTN_EINVAL;
  if (s->n_q_heads % s->n_kv_heads != 0) return DECATTN_EINVAL;
  if (pl->batch != s->batch || pl->n_kv_heads != s->n_kv_heads || pl->tile_len <= 0 || pl->n_bins <= 0 ||
      pl->max_units < 0 || !pl->buf)
    return DECATTN_EINVAL;
  const int G = s->n_q_heads / s->n_kv_heads;
  const int64_t GT = (int64_t)G * s->q_tokens;
  if (s->head_dim != 64 && s->head_dim != 128) return DECATTN_ENOTSUP;
  if (s->page_size % 16 != 0 || s->page_size > 256) return DECATTN_ENOTSUP;
  if (pl->tile_len % s->page_size != 0) return DECATTN_ENOTSUP;
  if (s->q_tokens > kMaxT || GT > kMaxGT || !split_supported(s->kv_dtype, s->head_dim, (int)GT))
    return DECATTN_ENOTSUP;
  if ((int64_t)s->num_pages * s->n_kv_heads * s->page_size >= (1ll << 31)) return DECATTN_ENOTSUP;
  if ((int64_t)s->batch * s->q_tokens * s->n_q_heads >= (1ll << 31)) return DECATTN_ENOTSUP;
  return DECATTN_OK;
}

// Checks the arguments and enqueues the requested stages (kStageSplit, kStageCombine).
enum { kStageSplit = 1, kStageCombine = 2 };

static int enqueue(int stages, const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                   const int32_t* page_table, const int32_t* seq_lens, const float* kv_scales,
                   const dec_attn_plan_t* plan, void* workspace, size_t workspace_bytes, float* out, float* lse,
                   void* stream) {
  int rc = check_shape(shape, plan);
  if (rc != DECATTN_OK) return rc;
  const dec_attn_shape& s = *shape;
  if (!workspace) return DECATTN_EINVAL;
  if (s.batch == 0) return DECATTN_OK;
  if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !out || !lse) return DECATTN_EINVAL;
  if (s.kv_dtype != DECATTN_KV_BF16 && !kv_scales) return DECATTN_EINVAL;
  if (s.num_pages <= 0 || s.max_pages_per_seq <= 0) return DECATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) || !aligned16(workspace) ||
      !aligned16(plan->buf))
    return DECATTN_EALIGN;
  if (((reinterpret_cast<uintptr_t>(page_table) | reinterpret_cast<uintptr_t>(seq_lens) |
        reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(kv_scales)) & 3) != 0)
    return DECATTN_EALIGN;
  const int G = s.n_q_heads / s.n_kv_heads;
  const int GT = G * s.q_tokens;
  const int D = s.head_dim;
  (void)GT;
  const WsLayout wl = ws_layout(plan->max_units, s);
  if ((int64_t)workspace_bytes < wl.total) return DECATTN_ESMALL;
  if (wl.items >= (1ll << 31)) return DECATTN_ENOTSUP;  // the combine numbers its items in 32 bits
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_fail("cudaGetDevice", e);

  char* ws = static_cast<char*>(workspace);
  int32_t* row_cnt = reinterpret_cast<int32_t*>(ws + wl.off_row_cnt);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part_o = reinterpret_cast<float*>(ws + wl.off_part_o);
  float* part_lse = reinterpret_cast<float*>(ws + wl.off_part_lse);

  if (stages & kStageSplit) {
    CUtensorMap tmK, tmV;
    const int64_t rows = (int64_t)s.num_pages * s.n_kv_heads * s.page_size;
    if (!make_kv_map(&tmK, k_pages, s.kv_dtype, D, rows) || !make_kv_map(&tmV, v_pages, s.kv_dtype, D, rows))
      return cuda_fail("K/V tensor map (cuTensorMapEncodeTiled)");
    const float scale = s.sm_scale > 0.f ? s.sm_scale : 1.0f / sqrtf((float)D);
    SplitParams sp;
    sp.q = static_cast<const uint16_t*>(q);
    sp.page_table = page_table;
    sp.seq_lens = seq_lens;
    sp.kv_scales = kv_scales;
    sp.plan = static_cast<const char*>(plan->buf);
    sp.out = out;
    sp.lse = lse;
    sp.part_o = part_o;
    sp.part_lse = part_lse;
    sp.row_cnt = row_cnt;
    sp.status = reinterpret_cast<int32_t*>(static_cast<char*>(plan->buf) + offsetof(PlanHeader, run_status));
    sp.B = s.batch; sp.T = s.q_tokens; sp.Hq = s.n_q_heads; sp.Hkv = s.n_kv_heads; sp.G = G; sp.GT = GT;
    sp.P = s.page_size; sp.num_pages = s.num_pages; sp.mpps = s.max_pages_per_seq; sp.n_bins = plan->n_bins;
    sp.tile_len = plan->tile_len; sp.max_units = plan->max_units; sp.sparse = plan->sparse;
    sp.qk_scale_log2 = scale * 1.4426950408889634f;
    test_waits(&sp.wait_ns, &sp.skip_fill);
    if (const cudaError_t e = launch_split(sp, tmK, tmV, s.kv_dtype, D, st); e != cudaSuccess)
      return cuda_fail("split kernel launch", e);
  }
  if (stages & kStageCombine) {
    CombineParams cp;
    cp.plan = static_cast<const char*>(plan->buf);
    cp.seq_lens = seq_lens;
    cp.part_o = part_o;
    cp.part_lse = part_lse;
    cp.out = out;
    cp.lse = lse;
    cp.row_cnt = row_cnt;
    cp.chunk_state = reinterpret_cast<float*>(ws + wl.off_chunk);
    cp.B = s.batch; cp.T = s.q_tokens; cp.Hq = s.n_q_heads; cp.Hkv = s.n_kv_heads; cp.G = G; cp.GT = GT; cp.D = D;
    cp.tl = plan->tile_len;
    cp.sparse = plan->sparse;
    if (const cudaError_t e = launch_combine(cp, dev, st); e != cudaSuccess) return cuda_fail("combine kernel launch", e);
  }
  return DECATTN_OK;
}

// Shared by dec_attn_prefill (cu_q null: T rows per request), dec_attn_prefill_varlen and the FP8
// prefill (on its widened pool). check_only: every check and tensor map, no launch.
static int prefill_enqueue(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                           const int32_t* page_table, const int32_t* seq_lens, const int32_t* cu_q,
                           int64_t total_rows, float* out, float* lse, int32_t* status, void* stream,
                           bool check_only = false) {
  if (!shape) return DECATTN_EINVAL;
  const dec_attn_shape& s = *shape;
  if (s.batch < 0 || s.q_tokens <= 0 || s.n_q_heads <= 0 || s.n_kv_heads <= 0 || s.page_size <= 0 ||
      s.num_pages < 0 || s.max_pages_per_seq < 0 || s.n_q_heads % s.n_kv_heads != 0 || total_rows < 0)
    return DECATTN_EINVAL;
  if (s.kv_dtype != DECATTN_KV_BF16 || s.head_dim != 128 || s.page_size % 16 != 0) return DECATTN_ENOTSUP;
  if (s.batch > 65535 || s.n_q_heads > 65535) return DECATTN_ENOTSUP;
  if (total_rows * s.n_q_heads >= (1ll << 31) || (int64_t)s.batch * s.q_tokens >= (1ll << 31) ||
      (int64_t)s.num_pages * s.n_kv_heads * s.page_size >= (1ll << 31))
    return DECATTN_ENOTSUP;
  if (s.batch == 0 || total_rows == 0) return DECATTN_OK;
  if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !out || !lse) return DECATTN_EINVAL;
  if (s.num_pages <= 0 || s.max_pages_per_seq <= 0) return DECATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out)) return DECATTN_EALIGN;
  if (((reinterpret_cast<uintptr_t>(page_table) | reinterpret_cast<uintptr_t>(seq_lens) |
        reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(status) | reinterpret_cast<uintptr_t>(cu_q)) &
       3) != 0)
    return DECATTN_EALIGN;
  CUtensorMap tmQ, tmK, tmV, tmO;
  const int64_t rows = (int64_t)s.num_pages * s.n_kv_heads * s.page_size;
  if (!make_prefill_q_map(&tmQ, q, total_rows, s.n_q_heads, s.head_dim) ||
      !make_kv_map(&tmK, k_pages, s.kv_dtype, s.head_dim, rows) ||
      !make_kv_map(&tmV, v_pages, s.kv_dtype, s.head_dim, rows) ||
      !make_prefill_out_map(&tmO, out, total_rows, s.n_q_heads, s.head_dim))
    return cuda_fail("prefill tensor maps (cuTensorMapEncodeTiled)");
  const float scale = s.sm_scale > 0.f ? s.sm_scale : 1.0f / sqrtf((float)s.head_dim);
  PrefillParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.cu_q = cu_q;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.B = s.batch; p.T = s.q_tokens; p.Hq = s.n_q_heads; p.Hkv = s.n_kv_heads; p.G = s.n_q_heads / s.n_kv_heads;
  p.P = s.page_size; p.num_pages = s.num_pages; p.mpps = s.max_pages_per_seq;
  p.total_rows = total_rows;
  p.qk_scale_log2 = scale * 1.4426950408889634f;
  test_waits(&p.wait_ns, &p.skip_fill);
  if (check_only) return DECATTN_OK;
  const cudaError_t e = launch_prefill(p, tmQ, tmK, tmV, tmO, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DECATTN_OK : cuda_fail("prefill kernel launch", e);
}

// FP8 prefill: widen the E4M3 pages each request uses into the workspace (bf16 pool with its own
// page table), then the bf16 prefill on it. Every check happens before the first launch.
static int prefill_fp8_enqueue(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                               const float* kv_scales, const int32_t* page_table, const int32_t* seq_lens,
                               const int32_t* cu_q, int64_t total_rows, void* workspace, int64_t workspace_bytes,
                               float* out, float* lse, int32_t* status, void* stream) {
  if (!shape) return DECATTN_EINVAL;
  const dec_attn_shape& s = *shape;
  if (s.batch < 0 || s.q_tokens <= 0 || s.n_kv_heads <= 0 || s.page_size <= 0 || s.num_pages < 0 ||
      s.max_pages_per_seq < 0 || total_rows < 0 || workspace_bytes < 0)
    return DECATTN_EINVAL;
  if (s.kv_dtype != DECATTN_KV_FP8E4M3 || s.head_dim != 128 || s.page_size % 16 != 0) return DECATTN_ENOTSUP;
  if ((int64_t)s.batch * s.max_pages_per_seq >= (1ll << 31)) return DECATTN_ENOTSUP;
  if (s.batch == 0 || total_rows == 0) return DECATTN_OK;
  if (!k_pages || !v_pages || !kv_scales || !page_table || !seq_lens || !workspace) return DECATTN_EINVAL;
  if (s.num_pages <= 0 || s.max_pages_per_seq <= 0) return DECATTN_EINVAL;
  if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(kv_scales) & 3) != 0)
    return DECATTN_EALIGN;
  int64_t off_v = 0, off_pt = 0;
  const int64_t need =
      widen_scratch_bytes(s.batch, s.max_pages_per_seq, s.n_kv_heads, s.page_size, s.head_dim, &off_v, &off_pt);
  if (workspace_bytes < need) return DECATTN_ESMALL;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  dec_attn_shape wide = s;  // the widened pool: bf16, page i of request b at b * max_pages_per_seq + i
  wide.kv_dtype = DECATTN_KV_BF16;
  wide.num_pages = s.batch * s.max_pages_per_seq;
  const int32_t* wide_pt = reinterpret_cast<const int32_t*>(ws + off_pt);
  int rc = prefill_enqueue(&wide, q, ws, ws + off_v, wide_pt, seq_lens, cu_q, total_rows, out, lse, status, stream,
                           /*check_only=*/true);
  if (rc != DECATTN_OK) return rc;
  WidenParams w;
  w.k_codes = static_cast<const uint8_t*>(k_pages);
  w.v_codes = static_cast<const uint8_t*>(v_pages);
  w.kv_scales = kv_scales;
  w.page_table = page_table;
  w.seq_lens = seq_lens;
  w.k_out = reinterpret_cast<uint16_t*>(ws);
  w.v_out = reinterpret_cast<uint16_t*>(ws + off_v);
  w.pt_out = reinterpret_cast<int32_t*>(ws + off_pt);
  w.status = status;
  w.B = s.batch; w.Hkv = s.n_kv_heads; w.P = s.page_size; w.D = s.head_dim;
  w.num_pages = s.num_pages; w.mpps = s.max_pages_per_seq;
  const cudaError_t e = launch_widen_kv(w, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("FP8 prefill widening launch", e);
  return prefill_enqueue(&wide, q, ws, ws + off_v, wide_pt, seq_lens, cu_q, total_rows, out, lse, status, stream);
}

}  // namespace decattn

using namespace decattn;

extern "C" int64_t dec_attn_prefill_fp8_workspace_bytes(const dec_attn_shape* shape) {
  if (!shape) return DECATTN_EINVAL;
  const dec_attn_shape& s = *shape;
  if (s.batch < 0 || s.n_kv_heads <= 0 || s.page_size <= 0 || s.max_pages_per_seq < 0 || s.head_dim <= 0)
    return DECATTN_EINVAL;
  return widen_scratch_bytes(s.batch, s.max_pages_per_seq, s.n_kv_heads, s.page_size, s.head_dim, nullptr, nullptr);
}

extern "C" int dec_attn_prefill_fp8(const dec_attn_shape* shape, const void* q, const void* k_pages,
                                    const void* v_pages, const float* kv_scales, const int32_t* page_table,
                                    const int32_t* seq_lens, const int32_t* cu_q_lens, int64_t total_q_rows,
                                    void* workspace, int64_t workspace_bytes, float* out, float* lse,
                                    int32_t* status, void* stream) {
  if (!shape) return DECATTN_EINVAL;
  if (!cu_q_lens && total_q_rows != (int64_t)shape->batch * shape->q_tokens) return DECATTN_EINVAL;
  return prefill_fp8_enqueue(shape, q, k_pages, v_pages, kv_scales, page_table, seq_lens, cu_q_lens, total_q_rows,
                             workspace, workspace_bytes, out, lse, status, stream);
}

extern "C" int dec_attn_prefill(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, const int32_t* seq_lens, float* out, float* lse,
                                int32_t* status, void* stream) {
  if (!shape) return DECATTN_EINVAL;
  if (shape->batch < 0 || shape->q_tokens <= 0) return DECATTN_EINVAL;
  return prefill_enqueue(shape, q, k_pages, v_pages, page_table, seq_lens, nullptr,
                         (int64_t)shape->batch * shape->q_tokens, out, lse, status, stream);
}

extern "C" int dec_attn_prefill_varlen(const dec_attn_shape* shape, const void* q, const void* k_pages,
                                       const void* v_pages, const int32_t* page_table, const int32_t* seq_lens,
                                       const int32_t* cu_q_lens, int64_t total_q_rows, float* out, float* lse,
                                       int32_t* status, void* stream) {
  if (!shape) return DECATTN_EINVAL;
  if (shape->batch > 0 && total_q_rows > 0 && !cu_q_lens) return DECATTN_EINVAL;
  return prefill_enqueue(shape, q, k_pages, v_pages, page_table, seq_lens, cu_q_lens, total_q_rows, out, lse, status,
                         stream);
}

extern "C" int dec_attn_default_bins(int device) { return default_bins(device); }

extern "C" int dec_attn_default_tile_len(int batch, int n_kv_heads, int64_t total_kv_tokens, int page_size,
                                         int head_dim, int rows_per_kv_head, int kv_dtype, int n_bins) {
  if (batch <= 0 || n_kv_heads <= 0 || total_kv_tokens < 0 || page_size <= 0 || page_size % 16 != 0 ||
      head_dim <= 0 || rows_per_kv_head <= 0 || n_bins <= 0)
    return DECATTN_EINVAL;
  const double elem = kv_dtype == DECATTN_KV_BF16 ? 2.0 : 1.0;
  const double N = (double)n_bins;
  const double W = (double)n_kv_heads * (double)total_kv_tokens;  // token-heads of the step
  const double tile_cost = 8192.0;  // fixed cost of a tile (q, epilogue, pipeline start) in KV-byte terms
  int best = 0;
  double best_est = 0.0;
  for (int tl = page_size; tl <= 8192; tl *= 2) {
    const double U = W / tl;  // tiles, as if every tile were full
    const double per_bin = U > 0 ? ceil(U / N) : 0.0;
    // the busiest bin's KV bytes and tile overheads, plus the partials every tile writes and the
    // combine reads back (fp32 o and lse per query row), spread over the bins
    const double est = per_bin * (tl * 2.0 * head_dim * elem + tile_cost) +
                       U * rows_per_kv_head * (head_dim + 1.0) * 8.0 / N;
    if (best == 0 || est < best_est) {  // the smaller estimate; on a tie the shorter tile
      best = tl;
      best_est = est;
    }
  }
  return best;
}

extern "C" size_t dec_attn_workspace_bytes(const dec_attn_shape* shape, const dec_attn_plan_t* plan) {
  if (check_shape(shape, plan) != DECATTN_OK) return 0;
  return (size_t)ws_layout(plan->max_units, *shape).total;
}

extern "C" int dec_attn_run(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                            const int32_t* page_table, const int32_t* seq_lens, const float* kv_scales,
                            const dec_attn_plan_t* plan, void* workspace, size_t workspace_bytes, float* out,
                            float* lse, void* stream) {
  return enqueue(kStageSplit | kStageCombine, shape, q, k_pages, v_pages, page_table,
                          seq_lens, kv_scales, plan, workspace, workspace_bytes, out, lse, stream);
}

extern "C" int dec_attn_split(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* page_table, const int32_t* seq_lens, const float* kv_scales,
                              const dec_attn_plan_t* plan, void* workspace, size_t workspace_bytes, float* out,
                              float* lse, void* stream) {
  return enqueue(kStageSplit, shape, q, k_pages, v_pages, page_table, seq_lens, kv_scales, plan,
                          workspace, workspace_bytes, out, lse, stream);
}

extern "C" int dec_attn_combine(const dec_attn_shape* shape, const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, const int32_t* seq_lens, const float* kv_scales,
                                const dec_attn_plan_t* plan, void* workspace, size_t workspace_bytes, float* out,
                                float* lse, void* stream) {
  return enqueue(kStageCombine, shape, q, k_pages, v_pages, page_table, seq_lens, kv_scales, plan,
                          workspace, workspace_bytes, out, lse, stream);
}

extern "C" int dec_attn_read_status(const dec_attn_plan_t* plan, const void* workspace, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (const cudaError_t e = cudaStreamSynchronize(st); e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
  (void)workspace;  // device errors of a run are recorded in the plan buffer's header
  if (plan && plan->buf) {
    PlanHeader h;
    if (const cudaError_t e = cudaMemcpy(&h, plan->buf, sizeof h, cudaMemcpyDeviceToHost); e != cudaSuccess)
      return cuda_fail("plan header copy", e);
    if (h.magic != kPlanMagic) return DECATTN_EINVAL;
    if (h.status != DECATTN_OK) return h.status;
    if (h.run_status != DECATTN_OK) return h.run_status;
  }
  return DECATTN_OK;
}

extern "C" int dec_attn_test_set_waits(uint64_t limit_ns, int32_t skip_fill) {
  if (limit_ns != 0 && (limit_ns < 100000ull || limit_ns > kWaitLimitNs)) return DECATTN_EINVAL;
  if (skip_fill < -1) return DECATTN_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  g_test_wait_ns = limit_ns == 0 ? kWaitLimitNs : limit_ns;
  g_test_skip_fill = skip_fill;
  return DECATTN_OK;
}

extern "C" size_t dec_attn_last_error(char* buf, size_t len) {
  const size_t n = strlen(g_last_error);
  if (buf && len > 0) {
    const size_t k = n < len - 1 ? n : len - 1;
    memcpy(buf, g_last_error, k);
    buf[k] = 0;
  }
  return n;
}

extern "C" const char* dec_attn_status_string(int status) {
  switch (status) {
    case DECATTN_OK: return "ok";
    case DECATTN_EINVAL: return "invalid argument";
    case DECATTN_ENOTSUP: return "unsupported shape or dtype";
    case DECATTN_ESMALL: return "buffer too small";
    case DECATTN_ECUDA: return "CUDA runtime error";
    case DECATTN_ETIMEOUT: return "device pipeline wait timed out";
    case DECATTN_EDEVICE: return "device detected invalid input (page id, seq_len)";
    case DECATTN_EALIGN: return "pointer not 16-byte aligned";
    case DECATTN_ECAPACITY: return "more tiles than the plan can hold";
    default: return "unknown status";
  }
}
