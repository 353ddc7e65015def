// Kernel-Aware Proxy (KAP) kernels.
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §4.2 (block ranking, flag-grouped sorting), §5.1 (the
// scoring and pooling run as a fused kernel), Appendix C.1 / Figure A (HRM
// and non-HRM groups sorted by score, HRM group first, leading entries kept
// under the stage-1 budget).
//
// Kernels (all tiles are one q-block x a group of up to 4 query heads that
// share a kv head):
//   kpool            one warp per (key block, kv head): fp32 token-by-token
//                    sum of the block's valid keys read through the page
//                    table, quantised to int8 with a per-block scale.
//   qpool            pools and quantises a tile's query vectors (16-row
//                    sub-rows and the block) and writes them to the
//                    workspace; a pure stream over Q.
//   kap_select_tc    (head_dim 128) exact integer scores of a tile's vectors
//                    against every causal key block with tcgen05 int8 MMAs
//                    (TMEM accumulators, TMA-fed key tiles), each sub-row's
//                    argmax (the HRM flags), the k_i smallest sort keys by
//                    radix select, written as the ordered lists.
//   kap_select       the same selection with int8 mma.sync scores (head_dim 64).
//   kap_score_select pooling and selection fused in one CTA; used where no
//                    workspace holds the pooled queries (the allocation-free
//                    entry point).
// Scores are exact integers, so the ordering is reproducible bit for bit.
// The stage-1 cut is the budget fraction k_i, or the pages' Top-p rule
// (top_p_emit), which keeps the shortest prefix of the full order holding
// a fraction p of the row's estimated attention mass.
#include <cfloat>
#include <cstdint>

#include "cosa_device.cuh"
#include "cosa_internal.h"
#include "kap_common.cuh"

namespace cosa {

// ============================================================================ kpool
template <int D, bool NHD>
__global__ void __launch_bounds__(256) kpool_kernel(KPoolArgs a) {
  constexpr int DPL = D / 32;  // dims per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long item = static_cast<long>(blockIdx.x) * 8 + warp;
  if (item >= static_cast<long>(a.nkb_total) * a.num_kv_heads) return;
  const int J = static_cast<int>(item / a.num_kv_heads);
  const int g = static_cast<int>(item % a.num_kv_heads);
  const int s = find_seq(a.cu_kblocks, a.batch, J);
  const int j = J - __ldg(a.cu_kblocks + s);
  const int L = seq_span(a.cu_seqlens, a.kv_lens, s, a.block_size).L;
  const int t0 = j * a.block_size;
  const int ntok = min(a.block_size, L - t0);
  if (ntok <= 0) {   // cu_kblocks disagrees with the key counts
    if (lane == 0) report(a.status, kErrBounds, 0x101);
    return;
  }

  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.0f;

  const int ppb = a.block_size / a.page_size;
  for (int u = 0; u < ppb; ++u) {
    const int tok = t0 + u * a.page_size;
    if (tok >= L) break;
    const int page = __ldg(a.page_table + static_cast<long>(s) * a.max_pages_per_seq + tok / a.page_size);
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) report(a.status, kErrBounds, 0x100);
      continue;
    }
    const int n_here = min(a.page_size, L - tok);
    // token t of the page: HND [P, Hkv, b_p, d] or NHD [P, b_p, Hkv, d]
    const __nv_bfloat16* base =
        a.k_pages + lane * DPL +
        (NHD ? static_cast<long>(page) * a.page_size * a.num_kv_heads * D + static_cast<long>(g) * D
             : (static_cast<long>(page) * a.num_kv_heads + g) * a.page_size * D);
    const long tstride = NHD ? static_cast<long>(a.num_kv_heads) * D : D;
#pragma unroll 8
    for (int t = 0; t < n_here; ++t) {
      if constexpr (DPL == 4) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(base + static_cast<long>(t) * tstride));
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        acc[0] = __fadd_rn(acc[0], __low2float(lo));
        acc[1] = __fadd_rn(acc[1], __high2float(lo));
        acc[2] = __fadd_rn(acc[2], __low2float(hi));
        acc[3] = __fadd_rn(acc[3], __high2float(hi));
      } else {
        const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(base + static_cast<long>(t) * tstride));
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&raw);
        acc[0] = __fadd_rn(acc[0], __low2float(v));
        acc[1] = __fadd_rn(acc[1], __high2float(v));
      }
    }
  }

  float M = 0.0f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) M = fmaxf(M, fabsf(acc[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const bool tiny = M < kTiny;
  const float inv = tiny ? 0.0f : __fdiv_rn(127.0f, M);
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    const int q = static_cast<int>(rintf(__fmul_rn(acc[e], inv)));
    packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * e);
  }
  int8_t* dst = a.kq + (static_cast<long>(g) * a.nkb_total + J) * D + lane * DPL;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint32_t*>(dst) = packed;
  } else {
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
  }
  if (lane == 0) {
    a.ks[static_cast<long>(g) * a.nkb_total + J] =
        tiny ? 0.0f : __fdiv_rn(__fdiv_rn(M, 127.0f), static_cast<float>(ntok));
  }
}

// ============================================================ kap_score_select
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ bool better(float s2, int j2, float s1, int j1) {
  return s2 > s1 || (s2 == s1 && j2 < j1);
}

// Ascending bitonic sort of `nseg` independent segments of `size` keys
// (a power of two), segment x at base + x * stride.  Whole-CTA (256 threads);
// index arithmetic by shifts and masks.
__device__ void bitonic_sort(uint64_t* base, int nseg, int size, int stride) {
  if (size < 2) return;
  int lg_n = 0;
  while ((1 << lg_n) < size) ++lg_n;
  const int pairs = nseg * size / 2;
  for (int k = 2, lg_k = 1; k <= size; k <<= 1, ++lg_k) {
    for (int jj = k >> 1, lg_j = lg_k - 1; jj > 0; jj >>= 1, --lg_j) {
      for (int idx = threadIdx.x; idx < pairs; idx += blockDim.x) {
        const int seg = idx >> (lg_n - 1);
        const int li = idx & ((size >> 1) - 1);
        const int x = ((li >> lg_j) << (lg_j + 1)) | (li & (jj - 1));
        uint64_t* p = base + seg * stride;
        const uint64_t va = p[x], vb = p[x + jj];
        const bool asc = (x & k) == 0;
        if ((va > vb) == asc) { p[x] = vb; p[x + jj] = va; }
      }
      __syncthreads();
    }
  }
}

template <int GT>
__device__ __forceinline__ Tile tile_of(const ScoreArgs& a) {
  return tile_at<GT>(a, static_cast<int>(blockIdx.x));
}

// Pooling of one tile (256 threads): the 16-row sub-row sums (token by token,
// fp32), the q-block sum (their fold), and the int8 quantisation of the
// (R + 1) vectors of each head into amat [GT][16][D] (rows 0..R; the rest 0).
template <int D, int GT, int R>
__device__ void pool_tile(const ScoreArgs& a, const Tile& tl, float* subsum, int8_t* amat, int* sub_valid,
                          float* qm_s) {
  constexpr int COLS = GT * D;
  constexpr int NCHUNK = COLS / 8;       // 16-byte chunks per token row of the head group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = a.block_size, i = tl.i, h0 = tl.h0, rlo = tl.rlo, rhi = tl.rhi;
  // sub-row sums 16-row sub-row sums, token by token, fp32
  for (int item = tid; item < R * NCHUNK; item += 256) {
    const int r = item / NCHUNK, ch = item % NCHUNK;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    const long row0 = tl.q_row0 + i * b + r * 16;   // rows outside [rlo, rhi) are never read
    const __nv_bfloat16* src = a.q + (row0 * a.num_q_heads + h0) * D + ch * 8;
    const long stride = static_cast<long>(a.num_q_heads) * D;
#pragma unroll
    for (int t0 = 0; t0 < 16; t0 += 8) {   // two batches of 8 independent loads, summed in row order
      uint4 raw[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int rr = r * 16 + t0 + t;
        if (rr >= rlo && rr < rhi) raw[t] = __ldg(reinterpret_cast<const uint4*>(src + (t0 + t) * stride));
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int rr = r * 16 + t0 + t;
        if (rr >= rlo && rr < rhi) {
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[t]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = __fadd_rn(acc[2 * e], __low2float(p2[e]));
            acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], __high2float(p2[e]));
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) subsum[r * COLS + ch * 8 + e] = acc[e];
  }
  for (int x = tid; x < GT * 16 * D / 4; x += 256) reinterpret_cast<uint32_t*>(amat)[x] = 0u;
  if (tid < R) sub_valid[tid] = sub_present(tl, tid) ? 1 : 0;
  __syncthreads();

  // block sum (fold of the sub-row sums) and int8 quantisation
  constexpr int DPL = D / 32;
  for (int vec = warp; vec < GT * (R + 1); vec += 8) {
    const int hh = vec / (R + 1), v = vec % (R + 1);
    float x[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      const int col = hh * D + lane * DPL + e;
      if (v == 0) {
        float acc = 0.0f;
        for (int r = 0; r < R; ++r) acc = __fadd_rn(acc, subsum[r * COLS + col]);
        x[e] = acc;
      } else {
        x[e] = subsum[(v - 1) * COLS + col];
      }
    }
    float M = 0.0f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) M = fmaxf(M, fabsf(x[e]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float inv = (M < kTiny) ? 0.0f : __fdiv_rn(127.0f, M);
#pragma unroll
    for (int e = 0; e < DPL; ++e)
      amat[(hh * 16 + v) * D + lane * DPL + e] = static_cast<int8_t>(rintf(__fmul_rn(x[e], inv)));
    if (qm_s != nullptr && v == 0 && lane == 0) qm_s[hh] = M;   // the q-block vector's scale
  }
  __syncthreads();

}

// Top-p stage-1 cut of one tile (256 threads; §5.1 "Hyperparameters" and
// Appendix D.1 give only p, so the mass is this library's reading).  Block
// j's share of the row's attention is estimated as
//   w_j = n_tok(j) exp((s_j - s_max) zscale),  zscale = (M_q / 127) / (n_rows sqrt(d)),
// zscale turning the pooled score s_j back into the mean logit between the
// q-block's rows and block j's keys (M_q: the q-block sum's max-abs, dropped
// from the ranking score).  Each head keeps the shortest prefix of its full
// flag-grouped order whose mass reaches p of the row's total (p = 1: all).
// One warp per head; fp32 masses summed in one fixed order (a contiguous
// chunk per lane, then the lanes in order), so the cut is deterministic.
template <int GT>
__device__ void top_p_emit(const ScoreArgs& a, const Tile& tl, uint64_t* keys) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = tl.n, b = a.block_size;
  bitonic_sort(keys, GT, tl.npow2, a.npow2_max);   // ascending keys = visit order; ends with a barrier
  if (warp >= GT) return;
  const int mt = warp;
  const uint64_t* kr = keys + mt * a.npow2_max;
  int nh = 0;   // HRM keys (bit 63 clear) form the prefix; every lane takes every ballot
  for (int base = 0; base < n; base += 32) {
    const int x = base + lane;
    nh += __popc(__ballot_sync(0xffffffffu, x < n && !(kr[x] >> 63)));
  }
  const float s_max = fmaxf(score_of_key(kr[0]), nh < n ? score_of_key(kr[nh]) : -FLT_MAX);
  const long row = static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I;
  const float qm = a.qm[row];
  const float zscale =
      __fdiv_rn(__fdiv_rn(qm, 127.0f), __fmul_rn(static_cast<float>(tl.rhi - tl.rlo), sqrtf(static_cast<float>(a.head_dim))));
  auto mass = [&](uint64_t key) {
    const int j = static_cast<int>(key & 0x7FFFFFFFu);
    const float ntok = static_cast<float>(min(b, tl.L - j * b));
    return __fmul_rn(ntok, expf(__fmul_rn(__fsub_rn(score_of_key(key), s_max), zscale)));
  };
  const int c = (n + 31) >> 5;
  const int lo = min(n, lane * c), hi = min(n, lo + c);
  float part = 0.0f;
  for (int x = lo; x < hi; ++x) part = __fadd_rn(part, mass(kr[x]));
  float inc = part;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc = __fadd_rn(inc, y);
  }
  const float total = __shfl_sync(0xffffffffu, inc, 31);
  float cum = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) cum = 0.0f;
  int first = n;   // entries kept: the first prefix whose mass reaches p * total (else all)
  if (a.top_p < 1.0f) {
    const float target = __fmul_rn(a.top_p, total);
    for (int x = lo; x < hi; ++x) {
      cum = __fadd_rn(cum, mass(kr[x]));
      if (cum >= target) { first = x + 1; break; }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, off));
  int k = max(1, first);
  if (k > a.kmax) {   // the host sizes kmax for every candidate; never taken
    if (lane == 0) report(a.status, kErrBounds, 0x205);
    k = a.kmax;
  }
  const long o = row * a.kmax;
  for (int t = lane; t < a.kmax; t += 32) {
    const uint64_t key = t < k ? kr[t] : 0ull;
    a.order[o + t] = t < k ? static_cast<int32_t>(key & 0x7FFFFFFFu) : -1;
    a.hrm[o + t] = (t < k && !(key >> 63)) ? 1 : 0;
  }
  if (lane == 0) {
    a.count[row] = k;
    a.n_hrm[row] = min(nh, k);
  }
}

// Selection and output of one tile (256 threads): each head's k_i smallest
// sort keys of keys [GT][npow2_max] (HRM flags already folded in), in
// ascending order, written as the visit lists.  `state` holds a few words
// of per-head radix-select state; `scratch` the histograms and buffers.
// kTopP = false compiles the Top-p cut out (kernels of entry points without it).
template <int GT, int R, bool kTopP = true>
__device__ void select_emit(const ScoreArgs& a, const Tile& tl, uint64_t* keys, float* state, unsigned char* scratch,
                            int scratch_bytes) {
  if constexpr (kTopP) {
    if (a.top_p > 0.0f) {
      top_p_emit<GT>(a, tl, keys);
      return;
    }
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = tl.n, npow2 = tl.npow2, h0 = tl.h0, I = tl.I;
  float* red_s = state;
  // ---- phase 4: each head's k_i smallest keys, in ascending order
  // The 64-bit keys are unique (they end in the block index), so a radix
  // select from the top byte down finds exactly the k_i smallest: at every
  // pass the bucket holding the k-th key is narrowed until all of it is
  // kept.  Only those keys are then sorted.  When every candidate is kept
  // (k_i = n), or the small buffers do not fit, all candidates are sorted.
  const int k_i = static_cast<int>(max(1LL, (static_cast<long long>(n) * a.bp + 9999) / 10000));
  int kpow = 1;
  while (kpow < k_i) kpow <<= 1;
  const bool select_path = (k_i < n) && (GT * 256 * 4 + GT * kpow * 8 <= scratch_bytes);
  const uint64_t* out_keys = keys;
  int out_stride = a.npow2_max;
  if (select_path) {
    int* hist = reinterpret_cast<int*>(scratch);                              // [GT][256]
    uint64_t* sel = reinterpret_cast<uint64_t*>(hist + GT * 256);             // [GT][kpow]
    unsigned long long* st_prefix = reinterpret_cast<unsigned long long*>(red_s);
    unsigned long long* st_mask = st_prefix + GT;
    unsigned long long* st_and = st_mask + GT;
    unsigned long long* st_or = st_and + GT;
    int* st_need = reinterpret_cast<int*>(st_or + GT);
    int* st_done = st_need + GT;
    int* st_cnt = st_done + GT;
    int* st_byte = st_cnt + GT;     // next key byte (from the top) each head's pass examines
    if (tid < GT) {
      st_need[tid] = k_i;
      st_done[tid] = 0;
      st_cnt[tid] = 0;
      st_and[tid] = ~0ull;
      st_or[tid] = 0ull;
    }
    __syncthreads();
    // The leading bytes every candidate of a head shares decide nothing: start
    // each head's radix passes at the first byte where its keys differ.
    for (int mt = 0; mt < GT; ++mt) {
      unsigned long long ka = ~0ull, ko = 0ull;
      for (int j = tid; j < n; j += 256) {
        const uint64_t key = keys[mt * a.npow2_max + j];
        ka &= key;
        ko |= key;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ka &= __shfl_xor_sync(0xffffffffu, ka, off);
        ko |= __shfl_xor_sync(0xffffffffu, ko, off);
      }
      if (lane == 0) {
        atomicAnd(&st_and[mt], ka);
        atomicOr(&st_or[mt], ko);
      }
    }
    __syncthreads();
    if (tid < GT) {
      const unsigned long long diff = st_and[tid] ^ st_or[tid];   // nonzero: n >= 2 distinct keys
      const int lead = __clzll(diff) >> 3;
      const unsigned long long m = lead == 0 ? 0ull : (~0ull << (64 - 8 * lead));
      st_mask[tid] = m;
      st_prefix[tid] = st_and[tid] & m;
      st_byte[tid] = lead;
    }
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
      for (int x = tid; x < GT * 256; x += 256) hist[x] = 0;
      __syncthreads();
      for (int mt = 0; mt < GT; ++mt) {
        if (st_done[mt]) continue;
        const unsigned long long pm = st_mask[mt], pv = st_prefix[mt];
        const int shift = 56 - 8 * st_byte[mt];
        // warp-aggregated increments: lanes landing in the same bin add once
        for (int base = warp * 32; base < n; base += 256) {
          const int j = base + lane;
          int bin = -1;
          if (j < n) {
            const uint64_t key = keys[mt * a.npow2_max + j];
            if ((key & pm) == pv) bin = static_cast<int>((key >> shift) & 255u);
          }
          const unsigned same = __match_any_sync(0xffffffffu, bin);
          if (bin >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[mt * 256 + bin], __popc(same));
        }
      }
      __syncthreads();
      if (warp < GT && !st_done[warp]) {
        int c[8];
        int sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[warp * 256 + 8 * lane + e];
          sum += c[e];
        }
        int inc = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += y;
        }
        const int need = st_need[warp];
        const int excl = inc - sum;
        if (excl < need && need <= inc) {   // this lane's bins hold the need-th key
          int below = excl, e = 0;
          while (below + c[e] < need) below += c[e++];
          const int rest = need - below;
          const int shift = 56 - 8 * st_byte[warp];
          st_need[warp] = rest;
          st_prefix[warp] |= static_cast<unsigned long long>(8 * lane + e) << shift;
          st_mask[warp] |= 255ull << shift;
          st_done[warp] = (c[e] == rest || st_byte[warp] == 7) ? 1 : 0;
          st_byte[warp] += 1;
        }
      }
      __syncthreads();
      int all = 1;
      for (int mt = 0; mt < GT; ++mt) all &= st_done[mt];
      if (all) break;
    }
    for (int x = tid; x < GT * kpow; x += 256) sel[x] = ~0ull;
    __syncthreads();
    for (int mt = 0; mt < GT; ++mt) {
      const unsigned long long pm = st_mask[mt], pv = st_prefix[mt];
      for (int j = tid; j < n; j += 256) {
        const uint64_t key = keys[mt * a.npow2_max + j];
        if ((key & pm) <= pv) {
          const int pos = atomicAdd(&st_cnt[mt], 1);
          if (pos < kpow) sel[mt * kpow + pos] = key;
          else report(a.status, kErrBounds, 0x201);
        }
      }
    }
    __syncthreads();
    if (kpow <= 64) {
      // At most 64 kept keys per head: one warp per head sorts them in
      // registers (lane holds positions lane and lane + 32) and writes the list.
      if (warp < GT) {
        const int mt = warp;
        uint64_t k0 = lane < k_i ? sel[mt * kpow + lane] : ~0ull;
        uint64_t k1 = lane + 32 < k_i ? sel[mt * kpow + lane + 32] : ~0ull;
#pragma unroll
        for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
          for (int jj = k >> 1; jj > 0; jj >>= 1) {
            const bool asc0 = (lane & k) == 0, asc1 = ((lane + 32) & k) == 0;
            if (jj == 32) {
              if ((k0 > k1) == asc0) { const uint64_t tmp = k0; k0 = k1; k1 = tmp; }
            } else {
              const uint64_t o0 = __shfl_xor_sync(0xffffffffu, k0, jj);
              const uint64_t o1 = __shfl_xor_sync(0xffffffffu, k1, jj);
              const bool lower = (lane & jj) == 0;
              k0 = (lower == asc0) ? (k0 < o0 ? k0 : o0) : (k0 < o0 ? o0 : k0);
              k1 = (lower == asc1) ? (k1 < o1 ? k1 : o1) : (k1 < o1 ? o1 : k1);
            }
          }
        }
        const long o = (static_cast<long>(h0 + mt) * a.nqb_total + I) * a.kmax;
        if (lane < a.kmax) {
          a.order[o + lane] = lane < k_i ? static_cast<int32_t>(k0 & 0x7FFFFFFFu) : -1;
          a.hrm[o + lane] = (lane < k_i && !(k0 >> 63)) ? 1 : 0;
        }
        if (lane + 32 < a.kmax) {
          a.order[o + lane + 32] = lane + 32 < k_i ? static_cast<int32_t>(k1 & 0x7FFFFFFFu) : -1;
          a.hrm[o + lane + 32] = (lane + 32 < k_i && !(k1 >> 63)) ? 1 : 0;
        }
        for (int t = lane + 64; t < a.kmax; t += 32) {
          a.order[o + t] = -1;
          a.hrm[o + t] = 0;
        }
        const int nh = __popc(__ballot_sync(0xffffffffu, lane < k_i && !(k0 >> 63))) +
                       __popc(__ballot_sync(0xffffffffu, lane + 32 < k_i && !(k1 >> 63)));
        if (lane == 0) {
          const long oc = static_cast<long>(h0 + mt) * a.nqb_total + I;
          a.count[oc] = k_i;
          a.n_hrm[oc] = nh;
        }
      }
      return;
    }
    bitonic_sort(sel, GT, kpow, kpow);
    out_keys = sel;
    out_stride = kpow;
  } else {
    bitonic_sort(keys, GT, npow2, a.npow2_max);
  }

  // ---- phase 5: emit the first k_i entries
  for (int x = tid; x < GT * a.kmax; x += 256) {
    const int mt = x / a.kmax, t = x % a.kmax;
    const long o = (static_cast<long>(h0 + mt) * a.nqb_total + I) * a.kmax + t;
    if (t < k_i) {
      const uint64_t key = out_keys[mt * out_stride + t];
      a.order[o] = static_cast<int32_t>(key & 0x7FFFFFFFu);
      a.hrm[o] = static_cast<uint8_t>((key >> 63) ? 0 : 1);
    } else {
      a.order[o] = -1;
      a.hrm[o] = 0;
    }
  }
  if (tid < GT) {
    int c = 0;
    while (c < k_i && !(out_keys[tid * out_stride + c] >> 63)) ++c;
    const long o = static_cast<long>(h0 + tid) * a.nqb_total + I;
    a.count[o] = k_i;
    a.n_hrm[o] = c;
  }
}

// Scoring and selection of one tile (256 threads) from its quantised vectors
// amat [GT][16][D]: exact integer scores on int8 tensor cores, each sub-row's
// argmax (the HRM flags), the k_i smallest sort keys, the output lists.
// `scratch` (scratch_bytes) holds the radix-select histograms and buffers.
template <int D, int GT, int R, bool kTopP = true>
__device__ void select_tile(const ScoreArgs& a, const Tile& tl, const int8_t* amat, const int* sub_valid,
                            float* red_s, int* red_j, uint64_t* keys, unsigned char* scratch, int scratch_bytes) {
  constexpr int QB = D / 4;              // bytes of a row each MMA quad-lane owns
  constexpr int QR = QB / 4;             // ... as 32-bit registers
  constexpr int KSTEPS = D / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = tl.n, npow2 = tl.npow2, kv = tl.kv, kb0 = tl.kb0;
  for (int x = tid; x < GT * npow2; x += 256) keys[(x / npow2) * a.npow2_max + (x % npow2)] = ~0ull;
  __syncthreads();

  // ---- phase 3: exact integer scores on int8 tensor cores, HRM argmax
  const int gq = lane >> 2, qd = lane & 3;
  uint32_t afr[GT][2][QR];  // rows gq and gq + 8, QB bytes each
#pragma unroll
  for (int mt = 0; mt < GT; ++mt) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(amat + (mt * 16 + gq + 8 * hr) * D + qd * QB);
#pragma unroll
      for (int x = 0; x < QR; ++x) afr[mt][hr][x] = src[x];
    }
  }
  float best_s[GT][2];
  int best_j[GT][2];
#pragma unroll
  for (int mt = 0; mt < GT; ++mt) {
    best_s[mt][0] = best_s[mt][1] = -FLT_MAX;
    best_j[mt][0] = best_j[mt][1] = 0x7FFFFFFF;
  }
  const int8_t* kq = a.kq + (static_cast<long>(kv) * a.nkb_total + kb0) * D;
  const float* ksp = a.ks + static_cast<long>(kv) * a.nkb_total + kb0;
  const int ntiles = (n + 7) >> 3;
  // key fragments and scales of a tile of 8 keys (zeros past n); fetched one tile ahead
  auto load_tile = [&](int tl, uint32_t (&bf)[QR], float& s0, float& s1) {
    const int key = tl * 8 + gq;
    if (tl < ntiles && key < n) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(kq + static_cast<long>(key) * D + qd * QB);
#pragma unroll
      for (int x = 0; x < QR; x += 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + x));
        bf[x] = v.x; bf[x + 1] = v.y; bf[x + 2] = v.z; bf[x + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int x = 0; x < QR; ++x) bf[x] = 0u;
    }
    const int k0 = tl * 8 + 2 * qd;
    s0 = (tl < ntiles && k0 < n) ? __ldg(ksp + k0) : 0.0f;
    s1 = (tl < ntiles && k0 + 1 < n) ? __ldg(ksp + k0 + 1) : 0.0f;
  };
  uint32_t bnext[QR];
  float ks0n, ks1n;
  load_tile(warp, bnext, ks0n, ks1n);
  for (int tile = warp; tile < ntiles; tile += 8) {
    uint32_t bfr[QR];
#pragma unroll
    for (int x = 0; x < QR; ++x) bfr[x] = bnext[x];
    const float ks0 = ks0n, ks1 = ks1n;
    load_tile(tile + 8, bnext, ks0n, ks1n);
    const int key0 = tile * 8 + 2 * qd;
#pragma unroll
    for (int mt = 0; mt < GT; ++mt) {
      int c[4] = {0, 0, 0, 0};
#pragma unroll
      for (int st = 0; st < KSTEPS; ++st)
        mma_s8(c, afr[mt][0][2 * st], afr[mt][1][2 * st], afr[mt][0][2 * st + 1], afr[mt][1][2 * st + 1],
               bfr[2 * st], bfr[2 * st + 1]);
      const float s00 = __fmul_rn(static_cast<float>(c[0]), ks0);
      const float s01 = __fmul_rn(static_cast<float>(c[1]), ks1);
      const float s10 = __fmul_rn(static_cast<float>(c[2]), ks0);
      const float s11 = __fmul_rn(static_cast<float>(c[3]), ks1);
      if (gq == 0) {  // matrix row 0: the q-block vector
        if (key0 < n) keys[mt * a.npow2_max + key0] = make_key(s00, key0);
        if (key0 + 1 < n) keys[mt * a.npow2_max + key0 + 1] = make_key(s01, key0 + 1);
      }
      if (gq >= 1 && gq <= R) {  // matrix rows 1..R: sub-rows
        if (key0 < n && s00 > best_s[mt][0]) { best_s[mt][0] = s00; best_j[mt][0] = key0; }
        if (key0 + 1 < n && s01 > best_s[mt][0]) { best_s[mt][0] = s01; best_j[mt][0] = key0 + 1; }
      }
      if (gq + 8 <= R) {
        if (key0 < n && s10 > best_s[mt][1]) { best_s[mt][1] = s10; best_j[mt][1] = key0; }
        if (key0 + 1 < n && s11 > best_s[mt][1]) { best_s[mt][1] = s11; best_j[mt][1] = key0 + 1; }
      }
    }
  }
  // argmax across the 4 lanes of each matrix row, then across warps
#pragma unroll
  for (int mt = 0; mt < GT; ++mt) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float sv = best_s[mt][hr];
      int jv = best_j[mt][hr];
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        const float s2 = __shfl_xor_sync(0xffffffffu, sv, off);
        const int j2 = __shfl_xor_sync(0xffffffffu, jv, off);
        if (better(s2, j2, sv, jv)) { sv = s2; jv = j2; }
      }
      if (qd == 0) {
        red_s[(warp * GT + mt) * 16 + gq + 8 * hr] = sv;
        red_j[(warp * GT + mt) * 16 + gq + 8 * hr] = jv;
      }
    }
  }
  __syncthreads();
  if (tid < GT * R) {
    const int mt = tid / R, v = tid % R;
    float sv = -FLT_MAX;
    int jv = 0x7FFFFFFF;
    for (int w = 0; w < 8; ++w) {
      const float s2 = red_s[(w * GT + mt) * 16 + v + 1];
      const int j2 = red_j[(w * GT + mt) * 16 + v + 1];
      if (better(s2, j2, sv, jv)) { sv = s2; jv = j2; }
    }
    if (sub_valid[v] && jv < n)
      atomicAnd(reinterpret_cast<unsigned long long*>(&keys[mt * a.npow2_max + jv]), ~(1ull << 63));
  }
  __syncthreads();

  select_emit<GT, R, kTopP>(a, tl, keys, red_s, scratch, scratch_bytes);
}

// ============================================================ tcgen05 scoring
// 16 TMEM lanes x 32 columns: thread t receives lane t/4 in registers
// 4c, 4c+1 and lane t/4 + 8 in registers 4c+2, 4c+3, at columns
// 8c + 2 (t % 4) + {0, 1}, c = 0..3.
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

constexpr int kTcN = 64;                  // candidate key blocks per score tile
constexpr int kTcRing = 2;                // key tiles in flight
constexpr int kTcTmemCols = 2 * kTcN;     // two accumulators: 3 CTAs per SM fit in TMEM
constexpr uint32_t kTcWaitLimit = 1u << 22;

size_t select_tc_smem_bytes(int GT, int npow2_max, int scratch_bytes) {
  return kTcRing * kTcN * 128 + 64 * 128 + static_cast<size_t>(GT) * npow2_max * 8 +
         static_cast<size_t>(scratch_bytes) + 2 * 2 * GT * 16 * 4 + 16 * GT * 4 + 64 +
         static_cast<size_t>(npow2_max) * 4;
}

// Proxy stage 2 on 5th-generation tensor cores (head_dim 128): scores of a
// tile's (R + 1) vectors per head against every causal key block.
// M = 64 rows: head mt's vectors occupy rows 16 mt .. 16 mt + R, which
// tcgen05 places in TMEM lanes 32 mt .. 32 mt + R of quadrant mt, so warp w
// (quadrant w % 4, key columns half w / 4) reads exactly its head's scores
// with the 16-lane TMEM load.  N = 64 key blocks per MMA, K = 128 dims in
// 4 steps of 32; the int8 key tiles arrive by TMA (128B swizzle), two tiles
// in flight, two TMEM accumulators (128 columns).  The small tiles keep the
// shared memory and TMEM of a CTA low enough for three CTAs per SM: the
// kernel is latency-bound, so resident CTAs are what hides the latency.
template <int GT, int R>
__global__ void __launch_bounds__(256, 3) kap_select_tc_kernel(const __grid_constant__ CUtensorMap kq_map, ScoreArgs a) {
  constexpr int D = 128;
  constexpr uint32_t IDESC = idesc_s8_s32(64, kTcN);
  extern __shared__ __align__(1024) unsigned char smem_tc[];
  // the key tiles need 1024-byte alignment for the 128B swizzle; dynamic shared
  // memory (no static shared memory here) starts right after the reserved 1 KiB
  if ((smem_u32(smem_tc) & 1023u) != 0) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x2FF);
    return;
  }
  unsigned char* sB = smem_tc;                                               // [kTcRing][128 keys][128 B]
  unsigned char* sA = smem_tc + kTcRing * kTcN * 128;                        // [64 rows][128 B]
  uint64_t* keys = reinterpret_cast<uint64_t*>(sA + 64 * 128);               // [GT][npow2_max]
  unsigned char* scratch = reinterpret_cast<unsigned char*>(keys + GT * a.npow2_max);
  float* red_s = reinterpret_cast<float*>(scratch + a.scratch_bytes);        // [2][GT][16]
  int* red_j = reinterpret_cast<int*>(red_s + 2 * GT * 16);                  // [2][GT][16]
  float* state = reinterpret_cast<float*>(red_j + 2 * GT * 16);              // select_emit state
  uint64_t* bars = reinterpret_cast<uint64_t*>(state + 16 * GT);             // b_full[ring], mma_done[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kTcRing + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* sKs = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(bars) + 64);   // [npow2_max] key scales

  const Tile tl = tile_of<GT>(a);
  if (tl.npow2 > a.npow2_max || tl.bad) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x203);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = tl.n, npow2 = tl.npow2;
  if (tid == 0) {
    for (int x = 0; x < kTcRing + 2; ++x) mbar_init(&bars[x], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  const int ntiles = (n + kTcN - 1) / kTcN;
  const int row0 = tl.kv * a.nkb_total + tl.kb0;   // Kq row of key block 0 of this sequence
  // key tiles cycle through a ring of kTcRing shared-memory slots (b_full[slot]);
  // accumulators alternate between two TMEM buffers (mma_done[t & 1])
  uint64_t* b_full = bars;
  uint64_t* mma_done = bars + kTcRing;
  auto issue_load = [&](int t) {
    const int slot = t % kTcRing;
    mbar_arrive_expect_tx(&b_full[slot], kTcN * 128);
    tma_load_2d(sB + slot * (kTcN * 128), &kq_map, &b_full[slot], 0, row0 + t * kTcN);
  };
  // the first key tiles are requested before the query vectors are staged
  if (tid == 0) {
    prefetch_tmap(&kq_map);
    for (int t = 0; t < kTcRing && t < ntiles; ++t) issue_load(t);
  }
  // A operand: rows 16 mt + v (v <= R) = head mt's vector v; other rows zero.  128B-swizzled K-major.
  for (int x = tid; x < 64 * 8; x += 256) {
    const int r = x >> 3, c = x & 7, mt = r >> 4, v = r & 15;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (mt < GT && v <= R)
      val = __ldg(reinterpret_cast<const uint4*>(
                      a.qa + ((static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I) * (R + 1) + v) * D) + c);
    *reinterpret_cast<uint4*>(sA + r * 128 + ((c ^ (r & 7)) << 4)) = val;
  }
  for (int x = tid; x < GT * npow2; x += 256) keys[(x / npow2) * a.npow2_max + (x % npow2)] = ~0ull;
  {
    const float* ks_row = a.ks + static_cast<long>(tl.kv) * a.nkb_total + tl.kb0;
    for (int x = tid; x < n; x += 256) sKs[x] = __ldg(ks_row + x);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
  auto issue_mma = [&](int t) {
    const int slot = t % kTcRing;
    if (!mbar_wait(&b_full[slot], (t / kTcRing) & 1, kTcWaitLimit, abort_flag, a.status, 0x210)) return;
    tc_fence_after();
#pragma unroll
    for (int ks = 0; ks < D / 32; ++ks) {
      const uint64_t ad = sw128_desc(a_base + ks * 32, 16, 1024);
      const uint64_t bd = sw128_desc(b_base + slot * (kTcN * 128) + ks * 32, 16, 1024);
      tc_mma_i8(tmem + (t & 1) * kTcN, ad, bd, IDESC, ks > 0 ? 1u : 0u);
    }
    tc_commit(&mma_done[t & 1]);
  };
  if (tid == 0) issue_mma(0);

  const int q = warp & 3, half = warp >> 2, v = lane >> 2;
  float best_s[2] = {-FLT_MAX, -FLT_MAX};
  int best_j[2] = {0x7FFFFFFF, 0x7FFFFFFF};
  for (int t = 0; t < ntiles; ++t) {
    if (tid == 0 && t + 1 < ntiles) issue_mma(t + 1);
    const bool ok = mbar_wait(&mma_done[t & 1], (t >> 1) & 1, kTcWaitLimit, abort_flag, a.status, 0x211);
    tc_fence_after();
    // the MMA of tile t has read its key slot: refill it right away
    if (tid == 0 && ok && t + kTcRing < ntiles) issue_load(t + kTcRing);
    if (q < GT && __all_sync(0xffffffffu, ok)) {
      uint32_t r[16];
      tmem_ld_16x256b_x4(tmem + (static_cast<uint32_t>(32 * q) << 16) + (t & 1) * kTcN + half * (kTcN / 2), r);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = t * kTcN + half * (kTcN / 2) + 8 * c + 2 * (lane & 3) + e;
          if (j < n) {
            const float ks = sKs[j];
            const float s_lo = __fmul_rn(static_cast<float>(static_cast<int>(r[4 * c + e])), ks);
            const float s_hi = __fmul_rn(static_cast<float>(static_cast<int>(r[4 * c + 2 + e])), ks);
            if (v == 0) keys[q * a.npow2_max + j] = make_key(s_lo, j);
            if (v >= 1 && v <= R && s_lo > best_s[0]) { best_s[0] = s_lo; best_j[0] = j; }
            if (v + 8 <= R && s_hi > best_s[1]) { best_s[1] = s_hi; best_j[1] = j; }
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();   // TMEM accumulator (t & 1) is free again
  }
  // each sub-row's argmax: the 4 lanes of a row, then the two column halves
  if (q < GT) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float sv = best_s[hr];
      int jv = best_j[hr];
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        const float s2 = __shfl_xor_sync(0xffffffffu, sv, off);
        const int j2 = __shfl_xor_sync(0xffffffffu, jv, off);
        if (better(s2, j2, sv, jv)) { sv = s2; jv = j2; }
      }
      if ((lane & 3) == 0) {
        red_s[(half * GT + q) * 16 + v + 8 * hr] = sv;
        red_j[(half * GT + q) * 16 + v + 8 * hr] = jv;
      }
    }
  }
  __syncthreads();
  if (tid < GT * R) {
    const int mt = tid / R, vv = tid % R;
    float sv = red_s[mt * 16 + vv + 1];
    int jv = red_j[mt * 16 + vv + 1];
    const float s2 = red_s[(GT + mt) * 16 + vv + 1];
    const int j2 = red_j[(GT + mt) * 16 + vv + 1];
    if (better(s2, j2, sv, jv)) { sv = s2; jv = j2; }
    if (sub_present(tl, vv) && jv < n)
      atomicAnd(reinterpret_cast<unsigned long long*>(&keys[mt * a.npow2_max + jv]), ~(1ull << 63));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTcTmemCols);
  select_emit<GT, R>(a, tl, keys, state, scratch, a.scratch_bytes);
}

// Fused proxy tile kernel: pooling and selection in one CTA, the pooled
// vectors never leaving shared memory.  Used where no workspace exists for
// them (cosa_proxy_noalloc).
template <int D, int GT, int R>
__global__ void __launch_bounds__(256, 2) kap_score_select_kernel(ScoreArgs a) {
  constexpr int COLS = GT * D;
  extern __shared__ __align__(16) unsigned char smem[];
  float* subsum = reinterpret_cast<float*>(smem);                       // [R][COLS]
  int8_t* amat = reinterpret_cast<int8_t*>(subsum + R * COLS);          // [GT][16][D]
  float* red_s = reinterpret_cast<float*>(amat + GT * 16 * D);          // [8][GT][16]
  int* red_j = reinterpret_cast<int*>(red_s + 8 * GT * 16);             // [8][GT][16]
  int* sub_valid = red_j + 8 * GT * 16;                                 // [R]
  uint64_t* keys = reinterpret_cast<uint64_t*>(sub_valid + 16);         // [GT][npow2_max]
  const Tile tl = tile_of<GT>(a);
  if (tl.npow2 > a.npow2_max || tl.bad) {  // host sizing guarantees npow2 fits
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x200);
    return;
  }
  pool_tile<D, GT, R>(a, tl, subsum, amat, sub_valid, nullptr);
  select_tile<D, GT, R, false>(a, tl, amat, sub_valid, red_s, red_j, keys, reinterpret_cast<unsigned char*>(subsum),
                        R * COLS * 4);
}

// Proxy stage 1 of the workspace path: pool and quantise a tile, write its
// (R + 1) int8 vectors per head to qa [Hq, NQB, R + 1, D].  Pure streaming of
// Q, many CTAs per SM.
template <int D, int GT, int R>
__global__ void __launch_bounds__(256, 3) qpool_kernel(ScoreArgs a) {
  constexpr int COLS = GT * D;
  extern __shared__ __align__(16) unsigned char smem[];
  float* subsum = reinterpret_cast<float*>(smem);                       // [R][COLS]
  int8_t* amat = reinterpret_cast<int8_t*>(subsum + R * COLS);          // [GT][16][D]
  int* sub_valid = reinterpret_cast<int*>(amat + GT * 16 * D);          // [R]
  float* qm_s = reinterpret_cast<float*>(sub_valid + 16);               // [GT]
  const Tile tl = tile_of<GT>(a);
  if (tl.bad) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x204);
    return;
  }
  pool_tile<D, GT, R>(a, tl, subsum, amat, sub_valid, qm_s);
  if (a.qm != nullptr && threadIdx.x < GT) a.qm[static_cast<long>(tl.h0 + threadIdx.x) * a.nqb_total + tl.I] = qm_s[threadIdx.x];
  constexpr int CH = (R + 1) * D / 16;   // 16-byte chunks per head
  for (int x = threadIdx.x; x < GT * CH; x += 256) {
    const int mt = x / CH, c = x % CH;
    int8_t* dst = a.qa + ((static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I) * (R + 1)) * D;
    reinterpret_cast<uint4*>(dst)[c] = reinterpret_cast<const uint4*>(amat + mt * 16 * D)[c];
  }
}

// Proxy stage 2 of the workspace path: scoring and selection of a tile from
// the vectors qpool wrote.
template <int D, int GT, int R>
__global__ void __launch_bounds__(256, 2) kap_select_kernel(ScoreArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int8_t* amat = reinterpret_cast<int8_t*>(smem);                       // [GT][16][D]
  float* red_s = reinterpret_cast<float*>(amat + GT * 16 * D);          // [8][GT][16]
  int* red_j = reinterpret_cast<int*>(red_s + 8 * GT * 16);             // [8][GT][16]
  int* sub_valid = red_j + 8 * GT * 16;                                 // [R]
  uint64_t* keys = reinterpret_cast<uint64_t*>(sub_valid + 16);         // [GT][npow2_max]
  unsigned char* scratch = reinterpret_cast<unsigned char*>(keys + GT * a.npow2_max);
  const Tile tl = tile_of<GT>(a);
  if (tl.npow2 > a.npow2_max || tl.bad) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x202);
    return;
  }
  constexpr int CH = D / 16;             // 16-byte chunks per row
  for (int x = threadIdx.x; x < GT * 16 * CH; x += 256) {
    const int mt = x / (16 * CH), row = (x / CH) % 16, c = x % CH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row <= R)
      v = __ldg(reinterpret_cast<const uint4*>(
                    a.qa + ((static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I) * (R + 1) + row) * D) + c);
    reinterpret_cast<uint4*>(amat + (mt * 16 + row) * D)[c] = v;
  }
  if (threadIdx.x < R) sub_valid[threadIdx.x] = sub_present(tl, static_cast<int>(threadIdx.x)) ? 1 : 0;
  __syncthreads();
  select_tile<D, GT, R>(a, tl, amat, sub_valid, red_s, red_j, keys, scratch, a.scratch_bytes);
}

// ============================================================ launchers
size_t score_smem_bytes(int D, int GT, int R, int npow2_max) {
  return static_cast<size_t>(R) * GT * D * 4 + static_cast<size_t>(GT) * 16 * D + 2 * 8 * GT * 16 * 4 + 16 * 4 +
         static_cast<size_t>(GT) * npow2_max * 8;
}

size_t qpool_smem_bytes(int D, int GT, int R) {
  return static_cast<size_t>(R) * GT * D * 4 + static_cast<size_t>(GT) * 16 * D + 16 * 4 + 4 * 4;
}

size_t select_smem_bytes(int D, int GT, int npow2_max, int scratch_bytes) {
  return static_cast<size_t>(GT) * 16 * D + 2 * 8 * GT * 16 * 4 + 16 * 4 + static_cast<size_t>(GT) * npow2_max * 8 +
         static_cast<size_t>(scratch_bytes);
}

enum class ProxyKernel { kFused, kPool, kSelect };

template <ProxyKernel K, int D, int GT, int R>
static cudaError_t launch_t(const ScoreArgs& a, cudaStream_t stream) {
  size_t smem;
  void (*kern)(ScoreArgs);
  if constexpr (K == ProxyKernel::kFused) {
    smem = score_smem_bytes(D, GT, R, a.npow2_max);
    kern = kap_score_select_kernel<D, GT, R>;
  } else if constexpr (K == ProxyKernel::kPool) {
    smem = qpool_smem_bytes(D, GT, R);
    kern = qpool_kernel<D, GT, R>;
  } else {
    smem = select_smem_bytes(D, GT, a.npow2_max, a.scratch_bytes);
    kern = kap_select_kernel<D, GT, R>;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.nqb_total) * (a.num_q_heads / GT);
  kern<<<grid, 256, smem, stream>>>(a);
  return cudaGetLastError();
}

template <ProxyKernel K, int D, int GT>
static cudaError_t launch_r(const ScoreArgs& a, cudaStream_t stream) {
  return a.block_size == 128 ? launch_t<K, D, GT, 8>(a, stream) : launch_t<K, D, GT, 4>(a, stream);
}

template <ProxyKernel K, int D>
static cudaError_t launch_g(const ScoreArgs& a, int GT, cudaStream_t stream) {
  switch (GT) {
    case 1: return launch_r<K, D, 1>(a, stream);
    case 2: return launch_r<K, D, 2>(a, stream);
    default: return launch_r<K, D, 4>(a, stream);
  }
}

template <ProxyKernel K>
static cudaError_t launch_proxy_kernel(const ScoreArgs& a, int GT, cudaStream_t stream) {
  return a.head_dim == 128 ? launch_g<K, 128>(a, GT, stream) : launch_g<K, 64>(a, GT, stream);
}

cudaError_t launch_kpool(const KPoolArgs& a, cudaStream_t stream) {
  const long items = static_cast<long>(a.nkb_total) * a.num_kv_heads;
  const unsigned grid = static_cast<unsigned>((items + 7) / 8);
  if (a.nhd) {
    if (a.head_dim == 128) kpool_kernel<128, true><<<grid, 256, 0, stream>>>(a);
    else kpool_kernel<64, true><<<grid, 256, 0, stream>>>(a);
  } else {
    if (a.head_dim == 128) kpool_kernel<128, false><<<grid, 256, 0, stream>>>(a);
    else kpool_kernel<64, false><<<grid, 256, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreArgs& a, int GT, cudaStream_t stream) {
  return launch_proxy_kernel<ProxyKernel::kFused>(a, GT, stream);
}

cudaError_t launch_qpool(const ScoreArgs& a, int GT, cudaStream_t stream) {
  return launch_proxy_kernel<ProxyKernel::kPool>(a, GT, stream);
}

cudaError_t launch_select(const ScoreArgs& a, int GT, cudaStream_t stream) {
  return launch_proxy_kernel<ProxyKernel::kSelect>(a, GT, stream);
}

template <int GT, int R>
static cudaError_t launch_select_tc_t(const ScoreArgs& a, const CUtensorMap& kq_map, cudaStream_t stream) {
  const size_t smem = select_tc_smem_bytes(GT, a.npow2_max, a.scratch_bytes);
  auto kern = kap_select_tc_kernel<GT, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.nqb_total) * (a.num_q_heads / GT);
  kern<<<grid, 256, smem, stream>>>(kq_map, a);
  return cudaGetLastError();
}

template <int GT>
static cudaError_t launch_select_tc_g(const ScoreArgs& a, const CUtensorMap& kq_map, cudaStream_t stream) {
  return a.block_size == 128 ? launch_select_tc_t<GT, 8>(a, kq_map, stream)
                             : launch_select_tc_t<GT, 4>(a, kq_map, stream);
}

cudaError_t launch_select_tc(const ScoreArgs& a, int GT, const CUtensorMap& kq_map, cudaStream_t stream) {
  switch (GT) {
    case 1: return launch_select_tc_g<1>(a, kq_map, stream);
    case 2: return launch_select_tc_g<2>(a, kq_map, stream);
    default: return launch_select_tc_g<4>(a, kq_map, stream);
  }
}

}  // namespace cosa
