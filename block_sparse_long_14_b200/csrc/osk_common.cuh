// Parts of the ordered-skipping attention kernel (osk.cu): the hand copy of a
// ragged K/V block, and the softmax role of a 128-row tile.
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §4.3 "In-kernel logic skip" (one vote per 128-row query
// tile on the value side), §3.3 L1/L2.1/L2.2 (QK^T is paid for every visited
// block; the test uses the running max and is an AND over rows), Appendix
// C.2 (Algorithm A) and D.1.
//
// Eight warps serve one 128-row tile: two threads per query row (TMEM lane),
// each owning half of the block's key columns.  Per visited block they read S
// once (causal mask, half-row max, P = exp2(s log2e/sqrt(d) - tr) in bf16
// written back over the columns read, l summing that rounded P), vote on the
// skip against the exact running max at one named barrier of the eight
// warps, and, if kept, re-base P, l and O by exact powers of two when a row's
// reference rose.  The epilogue writes O / l in bf16.
#pragma once

#include <cstdint>
#include <cmath>

#include "cosa_device.cuh"
#include "cosa_internal.h"

namespace cosa {

constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kBQ = 128;              // query rows per tile (TMEM lanes)
constexpr float kRescaleLog2 = 8.0f;  // re-base a reference when a max exceeds it by more than 2^8

// Where a tile's softmax group meets the MMA issuer and itself (shared memory).
struct SoftmaxSync {
  uint64_t* s_full;      // S of the c-th computed block is in TMEM (phase c & 1)
  uint64_t* p_full;      // [2]: verdict (and P, if kept) of the c-th computed block, by c & 1; 8 arrivals
  uint64_t* o_done;      // [2]: P V of the k-th kept block has completed, by k & 1
  int* skip_flag;        // [2]: the verdict, by c & 1
  int* vote;             // [2][kSoftmaxWarps], by c & 1
  int* vote_end;         // [kSoftmaxWarps]
  float* half_max;       // [2][2][kBQ]: [c & 1][half][row] half-row maxima; the epilogue reuses
                         // the slot after the last computed block for the partial row sums
  float* half_ref;       // [2][2][kBQ]: [c & 1][half][row] the halves' P references
};

// One tile as its softmax group sees it.
struct SoftmaxTile {
  uint32_t tmem;          // the tile's S columns; O follows at tmem + BK
  int sw;                 // this warp's index in the group (0..7); the group starts at a warp multiple of 4
  int bar_id;             // the group's named barrier
  int i, b, rlo, rhi;     // q-block within its sequence, block size, present rows [rlo, rhi)
  long q_row0;            // packed row of the sequence's position 0
  int h;                  // query head
  long row_id;            // h * NQB + I: the list row
  int n;                  // list length
  const int32_t* ord;     // the ordered block list
  const uint8_t* keep_row;  // nullable: entry t is computed only where keep != 0
  float log2_tau;         // log2 of the skip threshold (-inf: no skip)
};

// Copy one key block (K or V) of `nvalid` tokens into a 128B-swizzled stage
// by hand, zero-filling rows past the sequence end or on a missing page.
template <int D, int BK>
__device__ __forceinline__ void manual_block_copy(unsigned char* stage, const __nv_bfloat16* pool, const int32_t* pt_row,
                                  int j, int nvalid, const OskArgs& a, int g, int lane) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  const int ppb = a.block_size / a.page_size;
  for (int idx = lane; idx < BK * CH; idx += 32) {
    const int row = idx / CH, ch = idx % CH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < nvalid) {
      const int page = __ldg(pt_row + j * ppb + row / a.page_size);
      if (page >= 0 && page < a.num_pages) {
        const long tok = a.nhd ? (static_cast<long>(page) * a.page_size + row % a.page_size) * a.num_kv_heads + g
                               : (static_cast<long>(page) * a.num_kv_heads + g) * a.page_size + row % a.page_size;
        const __nv_bfloat16* src = pool + tok * D + ch * 8;
        v = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        report(a.status, kErrBounds, 0x300);
      }
    }
    const int atom = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4*>(stage + atom * (BK * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
  }
  fence_proxy_async();
  __syncwarp();
}

template <int D, int BK>
__device__ void softmax_tile(const OskArgs& a, const SoftmaxTile& x, const SoftmaxSync& y, volatile int* abort) {
  constexpr int HALF = BK / 2;   // key columns per softmax thread
  const int lane = threadIdx.x & 31;
  const int b = x.b;
  const int quad = x.sw & 3, half = x.sw >> 2;
  const int r = quad * 32 + lane;                 // tile row = TMEM lane
  const int col0 = half * HALF;                   // first key column of this thread
  const bool row_valid = r >= x.rlo && r < x.rhi;
  const uint32_t lane_base = x.tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const float sl2 = a.scale_log2;
  float m = -INFINITY, mref = -INFINITY, l = 0.0f;
  int n_pv = 0, nskip = 0;
  bool aborted = false;
  int j_next = x.n > 0 ? __ldg(x.ord) : 0;
  int ncomp = 0;   // entries computed so far
  for (int t = 0; t < x.n; ++t) {
    const int j = j_next;
    if (t + 1 < x.n) j_next = __ldg(x.ord + t + 1);
    if (x.keep_row != nullptr && __ldg(x.keep_row + t) == 0) {
      if (x.sw == 0 && lane == 0 && a.skipbits != nullptr) a.skipbits[x.row_id * a.kmax + t] = 0;
      continue;
    }
    const int sb = ncomp & 1;
    ++ncomp;
    const uint32_t s_cols = lane_base + col0;
    bool ok = mbar_wait(y.s_full, sb, a.wait_limit, abort, a.status, 0x30);
    ok = __all_sync(0xffffffffu, ok) && !aborted;
    // One pass over this thread's S columns, 32 at a time: causal mask, half-row
    // max, and P = exp2(s * log2e/sqrt(d) - tr) in bf16 written back over the
    // columns already read, with the partial row sum of the bf16-rounded values
    // (the same P that P V reads, so a dominant key's rounding cancels in O / l).
    // tr is the thread's reference: the row's running reference mref, raised to
    // the next integer above a chunk's max when that max exceeds it by more than
    // 2^8 (the P already written for earlier chunks is then re-based).  References
    // are integers, so every re-basing multiplies by an exact power of two.
    float mx = -INFINITY;
    float tr = mref;
    float2 ls = make_float2(0.0f, 0.0f);
    if (ok) {
      tc_fence_after();
      const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) {
        float sc[32];
        tmem_ld32(s_cols + c * 32, sc);
        tc_wait_ld();
        // causal mask (only the diagonal block, or a block past it, can hide keys):
        // key k of block j is visible to row r iff j*b + k <= i*b + r
        if (j >= x.i) {
          const int lim = r - (j - x.i) * b - col0 - c * 32;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k > lim) sc[k] = -INFINITY;
        }
        float mx0 = sc[0], mx1 = sc[1], mx2 = sc[2], mx3 = sc[3];
#pragma unroll
        for (int k = 4; k < 32; k += 4) {
          mx0 = fmaxf(mx0, sc[k]);
          mx1 = fmaxf(mx1, sc[k + 1]);
          mx2 = fmaxf(mx2, sc[k + 2]);
          mx3 = fmaxf(mx3, sc[k + 3]);
        }
        const float cmx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        mx = fmaxf(mx, cmx);
        const float cm2 = cmx * sl2;   // -inf for a fully masked chunk
        const bool raise = cm2 > tr + kRescaleLog2;
        if (c > 0 && __any_sync(0xffffffffu, raise && tr != -INFINITY)) {
          // re-base the P of the earlier chunks (rare after a row's first kept block)
          const float f = raise ? pow2_int(tr - ceilf(cm2)) : 1.0f;
          tc_wait_st();
#pragma unroll 1
          for (int cc = 0; cc < c; ++cc) {
            uint32_t pk[16];
            tmem_ld16(s_cols + cc * 16, pk);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = scale_bf16x2(pk[e], f);
            tmem_st16(s_cols + cc * 16, pk);
          }
          ls.x *= f;
          ls.y *= f;
        }
        if (raise) tr = ceilf(cm2);
        const float nb = (tr == -INFINITY) ? 0.0f : -tr;
        const float2 nbx2 = make_float2(nb, nb);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // two logits per packed fp32 FMA, two sums per packed add
          const float2 x = fma_f32x2(make_float2(sc[2 * e], sc[2 * e + 1]), sl2x2, nbx2);
          pk[e] = pack_bf16x2(ex2_approx(x.x), ex2_approx(x.y));
          ls = add_f32x2(ls, unpack_bf16x2(pk[e]));
        }
        // P of chunk c goes to columns [16c, 16c + 16) of this thread's half, all already read
        tmem_st16(s_cols + c * 16, pk);
      }
    }
    // the skip vote takes the exact running max m; rows past the sequence end vote to skip
    const float m_half = (row_valid && mx != -INFINITY) ? mx * sl2 : -INFINITY;
    const float gap = (m_half == -INFINITY) ? -INFINITY : m_half - m;
    const bool votes_skip = !row_valid || gap < x.log2_tau;
    const bool wskip = __all_sync(0xffffffffu, votes_skip);
    if (lane == 0) y.vote[sb * kSoftmaxWarps + x.sw] = (ok ? 0 : 2) | (wskip ? 1 : 0);
    y.half_max[(sb * 2 + half) * kBQ + r] = m_half;
    y.half_ref[(sb * 2 + half) * kBQ + r] = tr;
    named_bar_sync(x.bar_id, kSoftmaxThreads);
    int vor = 0, vand = 1;
#pragma unroll
    for (int w = 0; w < kSoftmaxWarps; ++w) {
      const int v = y.vote[sb * kSoftmaxWarps + w];
      vor |= v;
      vand &= v;
    }
    if (vor & 2) { aborted = true; break; }
    if (vand & 1) {
      if (x.sw == 0 && lane == 0) {
        y.skip_flag[sb] = 1;
        ++nskip;
        if (a.skipbits != nullptr) a.skipbits[x.row_id * a.kmax + t] = 1;
      }
      // the dead P stores land before the S buffer is handed back
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&y.p_full[sb]);
      continue;
    }
    const float m_row = fmaxf(m_half, y.half_max[(sb * 2 + (half ^ 1)) * kBQ + r]);
    const float m_new = fmaxf(m, m_row);
    // the row's reference: the higher of its two halves' (identical in both threads of the row)
    const float ref_row = fmaxf(tr, y.half_ref[(sb * 2 + (half ^ 1)) * kBQ + r]);
    if (__any_sync(0xffffffffu, tr < ref_row)) {
      // this half's P is re-based to the row's reference (the other half raised it higher)
      const float f = (tr < ref_row) ? pow2_int(tr - ref_row) : 1.0f;
      tc_wait_st();
#pragma unroll 1
      for (int c = 0; c < HALF / 32; ++c) {
        uint32_t pk[16];
        tmem_ld16(s_cols + c * 16, pk);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = scale_bf16x2(pk[e], f);
        tmem_st16(s_cols + c * 16, pk);
      }
      ls.x *= f;
      ls.y *= f;
    }
    // O and l follow the row's reference (ref_row >= mref: tr starts at mref and only rises)
    float alpha = 1.0f;
    if (n_pv > 0 && __any_sync(0xffffffffu, ref_row > mref)) {
      // O must be complete up to the last kept block before it is re-based
      bool okw = mbar_wait(&y.o_done[(n_pv - 1) & 1], ((n_pv - 1) >> 1) & 1, a.wait_limit, abort, a.status,
                           0x31);
      if (!__all_sync(0xffffffffu, okw)) { aborted = true; continue; }
      tc_fence_after();
      alpha = pow2_int(mref - ref_row);   // 0 while mref is -inf
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        float ov[32];
        const uint32_t addr = lane_base + BK + half * (D / 2) + c * 32;
        tmem_ld32(addr, ov);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] *= alpha;
        tmem_st32(addr, ov);
      }
    }
    mref = ref_row;
    m = m_new;
    l = l * alpha + (ls.x + ls.y);
    tc_wait_st();
    tc_fence_before();
    if (x.sw == 0 && lane == 0) {
      y.skip_flag[sb] = 0;
      if (a.skipbits != nullptr) a.skipbits[x.row_id * a.kmax + t] = 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&y.p_full[sb]);
    ++n_pv;
  }
  // ---- epilogue: O / l -> bf16
  bool ok = !aborted && n_pv >= 1;
  if (ok) ok = mbar_wait(&y.o_done[(n_pv - 1) & 1], ((n_pv - 1) >> 1) & 1, a.wait_limit, abort, a.status, 0x32);
  ok = __all_sync(0xffffffffu, ok);
  float* half_l = y.half_max + (ncomp & 1) * 2 * kBQ;   // idle since the barrier of the last computed block
  half_l[half * kBQ + r] = l;
  if (lane == 0) y.vote_end[x.sw] = ok ? 1 : 0;
  named_bar_sync(x.bar_id, kSoftmaxThreads);
  int all_ok = 1;
#pragma unroll
  for (int w = 0; w < kSoftmaxWarps; ++w) all_ok &= y.vote_end[w];
  if (ncomp == 0) {
    // a keep mask that leaves nothing of the row: zero output, like an empty list
    if (row_valid) {
      uint4* dst = reinterpret_cast<uint4*>(a.out + ((x.q_row0 + x.i * b + r) * a.num_q_heads + x.h) * D +
                                            half * (D / 2));
      for (int q4 = 0; q4 < D / 16; ++q4) dst[q4] = make_uint4(0u, 0u, 0u, 0u);
    }
  } else if (all_ok) {
    tc_fence_after();
    const float lrow = half_l[r] + half_l[kBQ + r];
    const float inv_l = (row_valid && lrow > 0.0f) ? 1.0f / lrow : 0.0f;
    __nv_bfloat16* dst = a.out + ((x.q_row0 + x.i * b + r) * a.num_q_heads + x.h) * D + half * (D / 2);
#pragma unroll 1
    for (int c = 0; c < D / 64; ++c) {
      float ov[32];
      tmem_ld32(lane_base + BK + half * (D / 2) + c * 32, ov);
      tc_wait_ld();
      if (row_valid) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w4;
          w4.x = pack_bf16x2(ov[q4 * 8 + 0] * inv_l, ov[q4 * 8 + 1] * inv_l);
          w4.y = pack_bf16x2(ov[q4 * 8 + 2] * inv_l, ov[q4 * 8 + 3] * inv_l);
          w4.z = pack_bf16x2(ov[q4 * 8 + 4] * inv_l, ov[q4 * 8 + 5] * inv_l);
          w4.w = pack_bf16x2(ov[q4 * 8 + 6] * inv_l, ov[q4 * 8 + 7] * inv_l);
          *reinterpret_cast<uint4*>(dst + c * 32 + q4 * 8) = w4;
        }
      }
    }
  }
  if (x.sw == 0 && lane == 0) {
    a.visited[x.row_id] = ncomp;
    a.skipped[x.row_id] = nskip;
    if (a.skipbits != nullptr)
      for (int t = x.n; t < a.kmax; ++t) a.skipbits[x.row_id * a.kmax + t] = 0;
  }
}

}  // namespace cosa
