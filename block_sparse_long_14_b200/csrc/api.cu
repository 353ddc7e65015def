// libcosa C ABI: argument checks, workspace layout, TMA tensor maps, launches.
// The declarations and the contract of each entry point are in include/cosa.h.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "cosa_device.cuh"
#include "cosa_internal.h"

namespace cosa {
namespace {

constexpr size_t kStatusBytes = 256;
constexpr uint32_t kDefaultWaitLimit = 1u << 22;
std::atomic<uint32_t> g_wait_limit{kDefaultWaitLimit};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int ceil_div(long a, long b) { return static_cast<int>((a + b - 1) / b); }

int budget_bp(float budget) { return static_cast<int>(std::floor(static_cast<double>(budget) * 1e4 + 0.5)); }

int keep_count(long n, int bp) {
  const long k = (n * bp + 9999) / 10000;
  return static_cast<int>(k < 1 ? 1 : k);
}

int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Query heads handled together by one proxy CTA: the largest of 4, 2, 1 that divides G.
int proxy_group(const cosa_shape_t& s) {
  const int G = s.num_q_heads / s.num_kv_heads;
  return (G % 4 == 0) ? 4 : (G % 2 == 0) ? 2 : 1;
}

int check_shape(const cosa_shape_t* s) {
  if (s == nullptr) return COSA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1 || s->num_pages < 1 || s->total_tokens < 1 ||
      s->total_qblocks < 1 || s->max_seqlen < 1 || s->max_pages_per_seq < 1)
    return COSA_ERR_INVALID_ARG;
  if (s->cu_seqlens == nullptr || s->cu_qblocks == nullptr) return COSA_ERR_INVALID_ARG;
  if (s->page_layout != COSA_PAGES_HND && s->page_layout != COSA_PAGES_NHD) return COSA_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return COSA_ERR_INVALID_ARG;
  if (s->num_q_heads / s->num_kv_heads > 8) return COSA_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return COSA_ERR_UNSUPPORTED;
  if (s->block_size != 64 && s->block_size != 128) return COSA_ERR_UNSUPPORTED;
  if (s->page_size < 8 || s->page_size % 8 != 0 || s->block_size % s->page_size != 0) return COSA_ERR_UNSUPPORTED;
  if (s->max_pages_per_seq < ceil_div(s->max_seqlen, s->page_size)) return COSA_ERR_INVALID_ARG;
  if (s->kv_lens == nullptr && s->total_qblocks < ceil_div(s->max_seqlen, s->block_size)) return COSA_ERR_INVALID_ARG;
  if (s->kv_lens == nullptr) {
    if (s->max_seqlen > s->total_tokens) return COSA_ERR_INVALID_ARG;
  } else {
    // prefill after a cached prefix: keys counted apart from the queries
    if (s->cu_kblocks == nullptr || s->total_kblocks < 1) return COSA_ERR_INVALID_ARG;
    if (s->total_kblocks < ceil_div(s->max_seqlen, s->block_size)) return COSA_ERR_INVALID_ARG;
    if (s->total_kblocks < s->total_qblocks) return COSA_ERR_INVALID_ARG;
  }
  // TMA row coordinates of the page pool are int32
  if (static_cast<long>(s->num_pages) * s->num_kv_heads * s->page_size >= (1L << 31)) return COSA_ERR_UNSUPPORTED;
  const int npow2 = next_pow2(ceil_div(s->max_seqlen, s->block_size));
  if (score_smem_bytes(s->head_dim, proxy_group(*s), s->block_size / 16, npow2) > 200 * 1024)
    return COSA_ERR_UNSUPPORTED;
  return COSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Key blocks of the batch and their per-sequence offsets: the q-blocks'
// unless a cached prefix separates them.
int total_kblocks(const cosa_shape_t& s) { return s.kv_lens != nullptr ? s.total_kblocks : s.total_qblocks; }
const int32_t* cu_kblocks(const cosa_shape_t& s) { return s.kv_lens != nullptr ? s.cu_kblocks : s.cu_qblocks; }

// Workspace: status block, pooled int8 keys [Hkv, NKB, d], key scales
// [Hkv, NKB], pooled int8 query vectors [Hq, NQB, b/16 + 1, d], the q-block
// vectors' max-abs [Hq, NQB] (the Top-p cut's logit scale) and, at head_dim
// 128, the score rows, HRM blocks and selection retry list of the
// persistent proxy.
struct WsLayout {
  size_t kq_off, ks_off, qa_off, qm_off, cand_off, hrmj_off, retry_off, total;
  int cand_stride;   // candidates per row of the score rows (0: no score rows)
};

WsLayout ws_layout(const cosa_shape_t& s) {
  WsLayout w{};
  w.kq_off = kStatusBytes;
  const size_t kq_bytes = static_cast<size_t>(s.num_kv_heads) * total_kblocks(s) * s.head_dim;
  w.ks_off = align_up(w.kq_off + kq_bytes, 256);
  w.qa_off = align_up(w.ks_off + static_cast<size_t>(s.num_kv_heads) * total_kblocks(s) * 4, 256);
  const size_t qa_bytes =
      static_cast<size_t>(s.num_q_heads) * s.total_qblocks * (s.block_size / 16 + 1) * s.head_dim;
  w.qm_off = align_up(w.qa_off + qa_bytes, 256);
  w.cand_off = align_up(w.qm_off + static_cast<size_t>(s.num_q_heads) * s.total_qblocks * 4, 256);
  // head_dim 128: every row's candidate score bits [Hq, NQB, NKB_max] and HRM blocks [Hq, NQB, 8]
  w.cand_stride = s.head_dim == 128 ? ceil_div(s.max_seqlen, s.block_size) : 0;
  w.hrmj_off = align_up(w.cand_off + static_cast<size_t>(s.num_q_heads) * s.total_qblocks * w.cand_stride * 4, 256);
  w.retry_off = align_up(w.hrmj_off + (w.cand_stride > 0 ? static_cast<size_t>(s.num_q_heads) * s.total_qblocks * 32 : 0),
                         256);
  // the selection's retry list: a count, then up to one entry per row
  w.total = align_up(w.retry_off + (w.cand_stride > 0 ? 4 * (1 + static_cast<size_t>(s.num_q_heads) * s.total_qblocks) : 0),
                     256);
  return w;
}

// Radix-select scratch of the select kernel: histograms plus a buffer for the
// kept keys (rounded up to a power of two), shrunk if shared memory is short;
// rows whose keys do not fit fall back to a full in-place sort.
int select_scratch_bytes(const cosa_shape_t& s, int kmax, int GT, int npow2_max) {
  int kpow = 8;   // room for all HRM keys of a row (at most b / 16 <= 8) before the cut at k_i
  while (kpow < kmax) kpow <<= 1;
  if (kpow > npow2_max) kpow = npow2_max;
  int bytes = GT * 256 * 4 + GT * kpow * 8;
  while (kpow > 1 && (select_smem_bytes(s.head_dim, GT, npow2_max, bytes) > 200 * 1024 ||
                      select_tc_smem_bytes(GT, npow2_max, bytes) > 220 * 1024)) {
    kpow >>= 1;
    bytes = GT * 256 * 4 + GT * kpow * 8;
  }
  return bytes;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Tiled tensor map (bf16 and 128-byte swizzle with 128-byte inner boxes unless stated).
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint32_t elem[3] = {1, 1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims,
            strides_bytes, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace cosa

using namespace cosa;

extern "C" {

const char* cosa_error_string(int code) {
  switch (code) {
    case COSA_OK: return "ok";
    case COSA_ERR_INVALID_ARG: return "invalid argument";
    case COSA_ERR_UNSUPPORTED: return "unsupported shape";
    case COSA_ERR_WORKSPACE: return "workspace too small";
    case COSA_ERR_CUDA: return "CUDA error";
    case COSA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case COSA_ERR_DEVICE: return "device bounds check failed";
    default: return "unknown status";
  }
}

int cosa_version(void) { return 102; }

void cosa_debug_set_wait_limit(uint32_t spins) { g_wait_limit.store(spins == 0 ? kDefaultWaitLimit : spins); }

size_t cosa_workspace_size(const cosa_shape_t* shape, float budget, int32_t* kmax_out) {
  if (check_shape(shape) != COSA_OK) return 0;
  if (!(budget > 0.0f && budget <= 1.0f)) return 0;
  if (kmax_out != nullptr)
    *kmax_out = keep_count(ceil_div(shape->max_seqlen, shape->block_size), budget_bp(budget));
  return ws_layout(*shape).total;
}

int cosa_workspace_init(void* workspace, size_t ws_bytes, cosa_stream_t stream) {
  if (workspace == nullptr || ws_bytes < kStatusBytes) return COSA_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COSA_OK
             : COSA_ERR_CUDA;
}

}  // extern "C"

namespace {

// The shared body of cosa_proxy (top_p = 0: the budget cut bp) and
// cosa_proxy_top_p (bp = 10^4, the Top-p cut at top_p).
int proxy_impl(const cosa_shape_t* shape, const void* q, const void* k_pages, const int32_t* page_table, int bp,
               float top_p, int32_t kmax, int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags,
               void* workspace, size_t ws_bytes, cosa_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != COSA_OK) return rc;
  if (q == nullptr || k_pages == nullptr || page_table == nullptr || order == nullptr || count == nullptr ||
      n_hrm == nullptr || hrm_flags == nullptr || workspace == nullptr)
    return COSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return COSA_ERR_INVALID_ARG;
  if (kmax < keep_count(ceil_div(shape->max_seqlen, shape->block_size), bp)) return COSA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(*shape);
  if (ws_bytes < w.total) return COSA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  Status* status = reinterpret_cast<Status*>(ws);

  KPoolArgs ka{};
  ka.k_pages = static_cast<const __nv_bfloat16*>(k_pages);
  ka.page_table = page_table;
  ka.cu_seqlens = shape->cu_seqlens;
  ka.kv_lens = shape->kv_lens;
  ka.cu_kblocks = cu_kblocks(*shape);
  ka.kq = reinterpret_cast<int8_t*>(ws + w.kq_off);
  ka.ks = reinterpret_cast<float*>(ws + w.ks_off);
  ka.status = status;
  ka.batch = shape->batch;
  ka.num_kv_heads = shape->num_kv_heads;
  ka.head_dim = shape->head_dim;
  ka.block_size = shape->block_size;
  ka.page_size = shape->page_size;
  ka.max_pages_per_seq = shape->max_pages_per_seq;
  ka.num_pages = shape->num_pages;
  ka.nkb_total = total_kblocks(*shape);
  ka.nhd = shape->page_layout == COSA_PAGES_NHD ? 1 : 0;
  if (launch_kpool(ka, st) != cudaSuccess) return COSA_ERR_CUDA;

  ScoreArgs sa{};
  sa.q = static_cast<const __nv_bfloat16*>(q);
  sa.kq = ka.kq;
  sa.ks = ka.ks;
  sa.cu_seqlens = shape->cu_seqlens;
  sa.cu_qblocks = shape->cu_qblocks;
  sa.kv_lens = shape->kv_lens;
  sa.cu_kblocks = cu_kblocks(*shape);
  sa.order = order;
  sa.count = count;
  sa.n_hrm = n_hrm;
  sa.hrm = hrm_flags;
  sa.status = status;
  sa.batch = shape->batch;
  sa.num_q_heads = shape->num_q_heads;
  sa.num_kv_heads = shape->num_kv_heads;
  sa.head_dim = shape->head_dim;
  sa.block_size = shape->block_size;
  sa.nqb_total = shape->total_qblocks;
  sa.nkb_total = total_kblocks(*shape);
  sa.kmax = kmax;
  sa.bp = bp;
  sa.npow2_max = next_pow2(ceil_div(shape->max_seqlen, shape->block_size));
  sa.qa = reinterpret_cast<int8_t*>(ws + w.qa_off);
  sa.qm = reinterpret_cast<float*>(ws + w.qm_off);
  sa.top_p = top_p;
  const int GT = proxy_group(*shape);
  int q_stages = 0;
  // (the persistent kernel records each sub-row's best score tile in 8 bits: at most 256 score
  // tiles of 128 key blocks per row)
  if (shape->head_dim == 128 && top_p == 0.0f && w.cand_stride > 0 && sa.npow2_max <= 256 * 128 &&
      stream_fits(GT, shape->block_size / 16, sa.npow2_max, kmax, &q_stages) &&
      select_rows_smem_bytes(sa.npow2_max, kmax) <= 200 * 1024) {
    // the budget cut at head_dim 128: pooling, scores and HRM flags in one persistent kernel,
    // then the selection of every row, one warp each
    CUtensorMap q_map, kq_map;
    {
      // Q as (d, query head, token): a box is 16 rows of a tile's GT heads
      const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(shape->num_q_heads),
                                  static_cast<cuuint64_t>(shape->total_tokens)};
      const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(shape->num_q_heads) * 256};
      const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(GT), 16};
      if (!make_map(&q_map, q, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return COSA_ERR_CUDA;
    }
    {
      // int8 key vectors as a [Hkv * NKB, 128] byte matrix, 128 key blocks per score tile
      const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(shape->num_kv_heads) * total_kblocks(*shape)};
      const cuuint64_t strides[1] = {128};
      const cuuint32_t box[2] = {128, 128};
      if (!make_map(&kq_map, sa.kq, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return COSA_ERR_CUDA;
    }
    sa.cand = reinterpret_cast<uint32_t*>(ws + w.cand_off);
    sa.hrmj = reinterpret_cast<int32_t*>(ws + w.hrmj_off);
    sa.cand_stride = w.cand_stride;
    sa.retry = reinterpret_cast<int32_t*>(ws + w.retry_off);
    sa.wait_limit = g_wait_limit.load();
    const StreamLayout lay = stream_layout(GT, shape->block_size / 16, sa.npow2_max, kmax, q_stages);
    if (launch_stream(sa, GT, q_map, kq_map, lay, st) != cudaSuccess) return COSA_ERR_CUDA;
    return launch_select_rows(sa, st) == cudaSuccess ? COSA_OK : COSA_ERR_CUDA;
  }
  sa.scratch_bytes = select_scratch_bytes(*shape, kmax, GT, sa.npow2_max);
  if (launch_qpool(sa, GT, st) != cudaSuccess) return COSA_ERR_CUDA;
  if (shape->head_dim == 128) {
    // int8 key vectors as a [Hkv * NKB, 128] byte matrix for the tcgen05 score tiles
    CUtensorMap kq_map;
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(shape->num_kv_heads) * total_kblocks(*shape)};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, 64};   // 64 key blocks x 128 int8 dims per score tile
    if (!make_map(&kq_map, sa.kq, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return COSA_ERR_CUDA;
    if (launch_select_tc(sa, GT, kq_map, st) != cudaSuccess) return COSA_ERR_CUDA;
  } else {
    if (launch_select(sa, GT, st) != cudaSuccess) return COSA_ERR_CUDA;
  }
  return COSA_OK;
}

}  // namespace

extern "C" {

int cosa_proxy(const cosa_shape_t* shape, const void* q, const void* k_pages, const int32_t* page_table, float budget,
               int32_t kmax, int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags, void* workspace,
               size_t ws_bytes, cosa_stream_t stream) {
  if (!(budget > 0.0f && budget <= 1.0f)) return COSA_ERR_INVALID_ARG;
  return proxy_impl(shape, q, k_pages, page_table, budget_bp(budget), 0.0f, kmax, order, count, n_hrm, hrm_flags,
                    workspace, ws_bytes, stream);
}

int cosa_proxy_top_p(const cosa_shape_t* shape, const void* q, const void* k_pages, const int32_t* page_table,
                     float p, int32_t kmax, int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags,
                     void* workspace, size_t ws_bytes, cosa_stream_t stream) {
  if (!(p > 0.0f && p <= 1.0f)) return COSA_ERR_INVALID_ARG;
  return proxy_impl(shape, q, k_pages, page_table, 10000, p, kmax, order, count, n_hrm, hrm_flags, workspace,
                    ws_bytes, stream);
}

int cosa_remap(const cosa_shape_t* shape, const int32_t* page_table, const int32_t* order, const int32_t* count,
               int32_t kmax, int32_t* pages, cosa_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != COSA_OK) return rc;
  if (page_table == nullptr || order == nullptr || count == nullptr || pages == nullptr || kmax < 1)
    return COSA_ERR_INVALID_ARG;
  RemapArgs ra{};
  ra.page_table = page_table;
  ra.order = order;
  ra.count = count;
  ra.cu_seqlens = shape->cu_seqlens;
  ra.cu_qblocks = shape->cu_qblocks;
  ra.kv_lens = shape->kv_lens;
  ra.pages = pages;
  ra.status = nullptr;
  ra.batch = shape->batch;
  ra.num_q_heads = shape->num_q_heads;
  ra.block_size = shape->block_size;
  ra.page_size = shape->page_size;
  ra.max_pages_per_seq = shape->max_pages_per_seq;
  ra.num_pages = shape->num_pages;
  ra.nqb_total = shape->total_qblocks;
  ra.kmax = kmax;
  return launch_remap(ra, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COSA_OK : COSA_ERR_CUDA;
}

namespace {

// The shared body of cosa_attn and cosa_attn_delta: tau_per_seq selects
// between one threshold (log2_tau) and tau_s = delta / L_s (log2_delta).
int attn_impl(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
              const int32_t* page_table, const int32_t* order, const int32_t* count, int32_t kmax, float log2_tau,
              int tau_per_seq, float log2_delta, const uint8_t* keep, void* out, int32_t* visited, int32_t* skipped,
              uint8_t* skipbits, void* workspace, size_t ws_bytes, cosa_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != COSA_OK) return rc;
  if (q == nullptr || k_pages == nullptr || v_pages == nullptr || page_table == nullptr || order == nullptr ||
      count == nullptr || out == nullptr || visited == nullptr || skipped == nullptr || workspace == nullptr ||
      kmax < 1)
    return COSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return COSA_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return COSA_ERR_WORKSPACE;

  const int D = shape->head_dim;
  const int Hq = shape->num_q_heads;
  CUtensorMap qmap, kmap, vmap;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq),
                                static_cast<cuuint64_t>(shape->total_tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if (!make_map(&qmap, q, 3, dims, strides, box)) return COSA_ERR_CUDA;
  }
  if (shape->page_layout == COSA_PAGES_HND) {
    // rows of d elements, (page, kv head, token) major to minor
    const cuuint64_t rows = static_cast<cuuint64_t>(shape->num_pages) * shape->num_kv_heads * shape->page_size;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(shape->page_size)};
    if (!make_map(&kmap, k_pages, 2, dims, strides, box)) return COSA_ERR_CUDA;
    if (!make_map(&vmap, v_pages, 2, dims, strides, box)) return COSA_ERR_CUDA;
  } else {
    // (d, kv head, page * b_p + token): a box of one kv head's b_p tokens lands
    // in shared memory exactly like the HND box
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(shape->num_kv_heads),
                                static_cast<cuuint64_t>(shape->num_pages) * shape->page_size};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(shape->num_kv_heads) * D * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(shape->page_size)};
    if (!make_map(&kmap, k_pages, 3, dims, strides, box)) return COSA_ERR_CUDA;
    if (!make_map(&vmap, v_pages, 3, dims, strides, box)) return COSA_ERR_CUDA;
  }
  OskArgs oa{};
  oa.page_table = page_table;
  oa.order = order;
  oa.count = count;
  oa.cu_seqlens = shape->cu_seqlens;
  oa.cu_qblocks = shape->cu_qblocks;
  oa.kv_lens = shape->kv_lens;
  oa.k_pages = static_cast<const __nv_bfloat16*>(k_pages);
  oa.v_pages = static_cast<const __nv_bfloat16*>(v_pages);
  oa.out = static_cast<__nv_bfloat16*>(out);
  oa.visited = visited;
  oa.skipped = skipped;
  oa.skipbits = skipbits;
  oa.keep = keep;
  oa.nhd = shape->page_layout == COSA_PAGES_NHD ? 1 : 0;
  oa.status = reinterpret_cast<Status*>(workspace);
  oa.batch = shape->batch;
  oa.num_q_heads = Hq;
  oa.num_kv_heads = shape->num_kv_heads;
  oa.block_size = shape->block_size;
  oa.page_size = shape->page_size;
  oa.max_pages_per_seq = shape->max_pages_per_seq;
  oa.num_pages = shape->num_pages;
  oa.nqb_total = shape->total_qblocks;
  oa.kmax = kmax;
  oa.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  oa.log2_tau = log2_tau;
  oa.tau_per_seq = tau_per_seq;
  oa.log2_delta = log2_delta;
  oa.wait_limit = g_wait_limit.load();
  return launch_osk(oa, qmap, kmap, vmap, D, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COSA_OK
                                                                                                      : COSA_ERR_CUDA;
}

}  // namespace

int cosa_attn(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
              const int32_t* page_table, const int32_t* order, const int32_t* count, int32_t kmax, float tau,
              void* out, int32_t* visited, int32_t* skipped, uint8_t* skipbits, void* workspace, size_t ws_bytes,
              cosa_stream_t stream) {
  if (!(tau >= 0.0f && tau < 1.0f)) return COSA_ERR_INVALID_ARG;
  const float log2_tau = tau > 0.0f ? static_cast<float>(std::log2(static_cast<double>(tau))) : -INFINITY;
  return attn_impl(shape, q, k_pages, v_pages, page_table, order, count, kmax, log2_tau, 0, -INFINITY, nullptr, out,
                   visited, skipped, skipbits, workspace, ws_bytes, stream);
}

int cosa_attn_masked(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
                     const int32_t* page_table, const int32_t* order, const int32_t* count, int32_t kmax,
                     const uint8_t* keep, float tau, void* out, int32_t* visited, int32_t* skipped,
                     uint8_t* skipbits, void* workspace, size_t ws_bytes, cosa_stream_t stream) {
  if (keep == nullptr) return COSA_ERR_INVALID_ARG;
  if (!(tau >= 0.0f && tau < 1.0f)) return COSA_ERR_INVALID_ARG;
  const float log2_tau = tau > 0.0f ? static_cast<float>(std::log2(static_cast<double>(tau))) : -INFINITY;
  return attn_impl(shape, q, k_pages, v_pages, page_table, order, count, kmax, log2_tau, 0, -INFINITY, keep, out,
                   visited, skipped, skipbits, workspace, ws_bytes, stream);
}

int cosa_attn_delta(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* order, const int32_t* count, int32_t kmax, float delta,
                    void* out, int32_t* visited, int32_t* skipped, uint8_t* skipbits, void* workspace,
                    size_t ws_bytes, cosa_stream_t stream) {
  if (!(delta == -1.0f || (delta > 0.0f && std::isfinite(delta)))) return COSA_ERR_INVALID_ARG;
  const float log2_delta = delta > 0.0f ? static_cast<float>(std::log2(static_cast<double>(delta))) : -INFINITY;
  return attn_impl(shape, q, k_pages, v_pages, page_table, order, count, kmax, -INFINITY, 1, log2_delta, nullptr, out,
                   visited, skipped, skipbits, workspace, ws_bytes, stream);
}

int cosa_sync_status(void* workspace, cosa_stream_t stream) {
  if (workspace == nullptr) return COSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Status h{};
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return COSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return COSA_ERR_CUDA;
  if (h.bits == 0) return COSA_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(h), st) != cudaSuccess) return COSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return COSA_ERR_CUDA;
  return (h.bits & kErrTimeout) ? COSA_ERR_TIMEOUT : COSA_ERR_DEVICE;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// cosa_proxy_noalloc: the proxy with its pooled-key scratch in a static device
// array instead of a caller-provided workspace (contract in include/cosa.h).

static __device__ __align__(256) unsigned char g_noalloc_scratch[COSA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in for the symbol).
int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return COSA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return COSA_OK;
}
}  // namespace

extern "C" int cosa_proxy_noalloc(const cosa_shape_t* shape, const void* q, const void* k_pages,
                                  const int32_t* page_table, float budget, int32_t kmax, int32_t* order,
                                  int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags, cosa_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != COSA_OK) return rc;
  if (q == nullptr || k_pages == nullptr || page_table == nullptr || order == nullptr || count == nullptr ||
      n_hrm == nullptr || hrm_flags == nullptr)
    return COSA_ERR_INVALID_ARG;
  if (!(budget > 0.0f && budget <= 1.0f)) return COSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages)) return COSA_ERR_INVALID_ARG;
  const int bp = budget_bp(budget);
  if (kmax < keep_count(ceil_div(shape->max_seqlen, shape->block_size), bp)) return COSA_ERR_INVALID_ARG;
  // pooled keys [Hkv, NKB, d] int8, then scales [Hkv, NKB] fp32
  const size_t kq_bytes = align_up(static_cast<size_t>(shape->num_kv_heads) * total_kblocks(*shape) * shape->head_dim, 256);
  const size_t need = kq_bytes + static_cast<size_t>(shape->num_kv_heads) * total_kblocks(*shape) * 4;
  if (need > COSA_NOALLOC_SCRATCH_BYTES) return COSA_ERR_WORKSPACE;
  void* base = nullptr;
  rc = noalloc_scratch(&base);
  if (rc != COSA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* scratch = static_cast<unsigned char*>(base);

  KPoolArgs ka{};
  ka.k_pages = static_cast<const __nv_bfloat16*>(k_pages);
  ka.page_table = page_table;
  ka.cu_seqlens = shape->cu_seqlens;
  ka.kv_lens = shape->kv_lens;
  ka.cu_kblocks = cu_kblocks(*shape);
  ka.kq = reinterpret_cast<int8_t*>(scratch);
  ka.ks = reinterpret_cast<float*>(scratch + kq_bytes);
  ka.status = nullptr;
  ka.batch = shape->batch;
  ka.num_kv_heads = shape->num_kv_heads;
  ka.head_dim = shape->head_dim;
  ka.block_size = shape->block_size;
  ka.page_size = shape->page_size;
  ka.max_pages_per_seq = shape->max_pages_per_seq;
  ka.num_pages = shape->num_pages;
  ka.nkb_total = total_kblocks(*shape);
  ka.nhd = shape->page_layout == COSA_PAGES_NHD ? 1 : 0;
  if (launch_kpool(ka, st) != cudaSuccess) return COSA_ERR_CUDA;

  ScoreArgs sa{};
  sa.q = static_cast<const __nv_bfloat16*>(q);
  sa.kq = ka.kq;
  sa.ks = ka.ks;
  sa.cu_seqlens = shape->cu_seqlens;
  sa.cu_qblocks = shape->cu_qblocks;
  sa.kv_lens = shape->kv_lens;
  sa.cu_kblocks = cu_kblocks(*shape);
  sa.order = order;
  sa.count = count;
  sa.n_hrm = n_hrm;
  sa.hrm = hrm_flags;
  sa.status = nullptr;
  sa.batch = shape->batch;
  sa.num_q_heads = shape->num_q_heads;
  sa.num_kv_heads = shape->num_kv_heads;
  sa.head_dim = shape->head_dim;
  sa.block_size = shape->block_size;
  sa.nqb_total = shape->total_qblocks;
  sa.nkb_total = total_kblocks(*shape);
  sa.kmax = kmax;
  sa.bp = bp;
  sa.npow2_max = next_pow2(ceil_div(shape->max_seqlen, shape->block_size));
  if (launch_score(sa, proxy_group(*shape), st) != cudaSuccess) return COSA_ERR_CUDA;
  return COSA_OK;
}
