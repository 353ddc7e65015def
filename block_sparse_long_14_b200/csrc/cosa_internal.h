// Host-side argument blocks and launchers shared between libcosa's .cu files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "cosa.h"

namespace cosa {

struct Status;

struct KPoolArgs {
  const __nv_bfloat16* k_pages;
  const int32_t* page_table;
  const int32_t* cu_seqlens;
  const int32_t* kv_lens;      // nullable: key counts after a cached prefix (else the query counts)
  const int32_t* cu_kblocks;   // key-block offset of each sequence
  int8_t* kq;     // [Hkv, NKB, d]
  float* ks;      // [Hkv, NKB]
  Status* status;
  int batch, num_kv_heads, head_dim, block_size, page_size, max_pages_per_seq, num_pages, nkb_total;
  int nhd;             // pages are [P, b_p, Hkv, d] instead of [P, Hkv, b_p, d]
};

struct ScoreArgs {
  const __nv_bfloat16* q;
  const int8_t* kq;    // [Hkv, NKB, d]
  const float* ks;     // [Hkv, NKB]
  const int32_t* cu_seqlens;
  const int32_t* cu_qblocks;
  const int32_t* kv_lens;      // nullable, as in KPoolArgs
  const int32_t* cu_kblocks;
  int32_t* order;
  int32_t* count;
  int32_t* n_hrm;
  uint8_t* hrm;
  Status* status;
  int8_t* qa;          // pooled int8 query vectors [Hq, NQB, R + 1, d] (two-stage path only)
  int batch, num_q_heads, num_kv_heads, head_dim, block_size, nqb_total, kmax, bp, npow2_max;
  int nkb_total;       // key blocks of the batch (= nqb_total without a cached prefix)
  int scratch_bytes;   // radix-select scratch of the select kernel
  float* qm;           // [Hq, NQB] max-abs of each q-block sum vector (written by qpool; nullable)
  float top_p;         // 0: budget cut k_i from bp; in (0, 1]: Top-p cut (reads qm)
  uint32_t* cand;      // [Hq, NQB, cand_stride] score bits of each candidate (persistent proxy path)
  int32_t* hrmj;       // [Hq, NQB, 8] the HRM blocks of each row, -1 padded (persistent proxy path)
  int cand_stride;     // candidates per row the cand rows hold (the longest sequence's key blocks)
  int32_t* retry;      // [1 + Hq * NQB] rows the register selection leaves to select_rows_kernel
                       // (retry[0] = how many; nullable: every row by select_rows_kernel)
  uint32_t wait_limit; // polls per mbarrier wait of the persistent proxy kernel
};

struct RemapArgs {
  const int32_t* page_table;
  const int32_t* order;
  const int32_t* count;
  const int32_t* cu_seqlens;
  const int32_t* cu_qblocks;
  const int32_t* kv_lens;      // nullable, as in KPoolArgs
  int32_t* pages;
  Status* status;
  int batch, num_q_heads, block_size, page_size, max_pages_per_seq, num_pages, nqb_total, kmax;
};

struct OskArgs {
  const int32_t* page_table;
  const int32_t* order;
  const int32_t* count;
  const int32_t* cu_seqlens;
  const int32_t* cu_qblocks;
  const int32_t* kv_lens;      // nullable, as in KPoolArgs
  const __nv_bfloat16* k_pages;
  const __nv_bfloat16* v_pages;
  __nv_bfloat16* out;
  int32_t* visited;
  int32_t* skipped;
  uint8_t* skipbits;
  const uint8_t* keep;  // nullable: list entry t is computed only where keep[row, t] != 0
  int nhd;              // pages are [P, b_p, Hkv, d] instead of [P, Hkv, b_p, d]
  Status* status;
  int batch, num_q_heads, num_kv_heads, block_size, page_size, max_pages_per_seq, num_pages;
  int nqb_total, kmax;
  float scale_log2;  // log2(e) / sqrt(d)
  float log2_tau;    // log2(tau), -inf for tau = 0
  int tau_per_seq;   // 1: tau_s = delta / L_s per sequence (L_s its key count), log2(tau_s) = log2_delta - log2(L_s)
  float log2_delta;  // log2(delta), -inf when the skip is off
  uint32_t wait_limit;
};

size_t score_smem_bytes(int D, int GT, int R, int npow2_max);
size_t select_smem_bytes(int D, int GT, int npow2_max, int scratch_bytes);
cudaError_t launch_kpool(const KPoolArgs& a, cudaStream_t stream);
cudaError_t launch_score(const ScoreArgs& a, int GT, cudaStream_t stream);    // fused pool + select
cudaError_t launch_qpool(const ScoreArgs& a, int GT, cudaStream_t stream);    // pool -> a.qa
cudaError_t launch_select(const ScoreArgs& a, int GT, cudaStream_t stream);   // a.qa -> lists
// a.qa -> lists on tcgen05 int8 MMAs (head_dim 128); kq_map covers a.kq as [Hkv * NQB, 128] int8
cudaError_t launch_select_tc(const ScoreArgs& a, int GT, const CUtensorMap& kq_map, cudaStream_t stream);
size_t select_tc_smem_bytes(int GT, int npow2_max, int scratch_bytes);
// The persistent proxy kernel (head_dim 128, budget cut): pooling, scores and
// HRM flags of every tile in one launch, one CTA per SM, writing a.cand and
// a.hrmj.  Shared-memory layout (byte offsets from a 1024-aligned base: Q
// ring, key tiles, int8 query vectors, sub-row sums, tile table; ks and red
// are those of epilogue group 0, group 1's follow group_bytes later) and its
// limit:
struct StreamLayout {
  uint32_t q, k, a, sub, tiles, ks, red, group_bytes, bars, total;
  int q_stages;   // Q chunks in flight (16 rows each)
};
constexpr uint32_t kStreamSmemLimit = 227 * 1024;
StreamLayout stream_layout(int GT, int R, int npow2_max, int kmax, int q_stages);
// Deepest even Q ring (8, 6 or 4 stages) that fits (true), or false when 4 stages do not.
bool stream_fits(int GT, int R, int npow2_max, int kmax, int* q_stages);
// q_map: Q as (d, Hq, T) with boxes of (128, GT, 16), no swizzle; kq_map: the
// pooled keys as [Hkv * NKB, 128] int8 in boxes of 128 rows, 128B swizzle.
cudaError_t launch_stream(const ScoreArgs& a, int GT, const CUtensorMap& q_map, const CUtensorMap& kq_map,
                          const StreamLayout& lay, cudaStream_t stream);
// Selection of every row from a.cand / a.hrmj (one warp per (head, q-block) row): the ordered lists.
cudaError_t launch_select_rows(const ScoreArgs& a, cudaStream_t stream);
size_t select_rows_smem_bytes(int npow2_max, int kmax);
cudaError_t launch_remap(const RemapArgs& a, cudaStream_t stream);
cudaError_t launch_osk(const OskArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                       const CUtensorMap& vmap, int head_dim, cudaStream_t stream);
size_t osk_smem_bytes(int head_dim, int block_size);

}  // namespace cosa
