// Kernel-Aware Proxy (KAP) kernels.
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §4.2 (block ranking, flag-grouped sorting), §5.1 (the
// scoring and pooling run as a fused kernel), Appendix C.1 / Figure A (HRM
// and non-HRM groups sorted by score, HRM group first, leading entries kept
// under the stage-1 budget).
//
// Two launches:
//   kpool            one warp per (key block, kv head): fp32 token-by-token
//                    sum of the block's valid keys read through the page
//                    table, quantised to int8 with a per-block scale.
//   kap_score_select one CTA per (q-block, group of up to 4 query heads that
//                    share a kv head): pools the q-block (16-row sub-rows and
//                    the block), quantises to int8, computes the exact
//                    integer scores against every causal key block with
//                    int8 tensor-core MMAs, takes each sub-row's argmax (the
//                    HRM flags), sorts the candidates by
//                    (HRM first, score descending, block ascending) and
//                    writes the first k_i.
// Both are bound by the HBM read of K and Q; the int8 MMAs keep the integer
// work off the critical path and make the scores exact, so the ordering is
// reproducible bit for bit.
#include <cfloat>
#include <cstdint>

#include "cosa_device.cuh"
#include "cosa_internal.h"

namespace cosa {

static constexpr float kTiny = 1.17549435e-38f;  // 2^-126: smallest normal fp32

// ============================================================================ kpool
template <int D>
__global__ void __launch_bounds__(256) kpool_kernel(KPoolArgs a) {
  constexpr int DPL = D / 32;  // dims per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long item = static_cast<long>(blockIdx.x) * 8 + warp;
  if (item >= static_cast<long>(a.nkb_total) * a.num_kv_heads) return;
  const int J = static_cast<int>(item / a.num_kv_heads);
  const int g = static_cast<int>(item % a.num_kv_heads);
  const int s = find_seq(a.cu_qblocks, a.batch, J);
  const int j = J - __ldg(a.cu_qblocks + s);
  const int L = __ldg(a.cu_seqlens + s + 1) - __ldg(a.cu_seqlens + s);
  const int t0 = j * a.block_size;
  const int ntok = min(a.block_size, L - t0);

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
    const __nv_bfloat16* base =
        a.k_pages + (static_cast<long>(page) * a.num_kv_heads + g) * a.page_size * D + lane * DPL;
#pragma unroll 8
    for (int t = 0; t < n_here; ++t) {
      if constexpr (DPL == 4) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(base + static_cast<long>(t) * D));
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        acc[0] = __fadd_rn(acc[0], __low2float(lo));
        acc[1] = __fadd_rn(acc[1], __high2float(lo));
        acc[2] = __fadd_rn(acc[2], __low2float(hi));
        acc[3] = __fadd_rn(acc[3], __high2float(hi));
      } else {
        const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(base + static_cast<long>(t) * D));
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

// Sort key: bit 63 = not HRM, bits 31..62 = score mapped to an unsigned
// order that is descending in the score, bits 0..30 = block index.
// Ascending keys give (HRM first, score descending, index ascending).
__device__ __forceinline__ uint64_t make_key(float sc, int j) {
  uint32_t u = __float_as_uint(sc);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;                         // -0 -> +0
  const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (1ull << 63) | (static_cast<uint64_t>(~asc) << 31) | static_cast<uint32_t>(j);
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

// Threads: 256.  GT = query heads per CTA (all sharing one kv head),
// R = sub-rows of 16 rows per q-block.
template <int D, int GT, int R>
__global__ void __launch_bounds__(256, 2) kap_score_select_kernel(ScoreArgs a) {
  constexpr int COLS = GT * D;
  constexpr int NCHUNK = COLS / 8;       // 16-byte chunks per token row of the head group
  constexpr int QB = D / 4;              // bytes of a row each MMA quad-lane owns
  constexpr int QR = QB / 4;             // ... as 32-bit registers
  constexpr int KSTEPS = D / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  float* subsum = reinterpret_cast<float*>(smem);                       // [R][COLS]
  int8_t* amat = reinterpret_cast<int8_t*>(subsum + R * COLS);          // [GT][16][D]
  float* red_s = reinterpret_cast<float*>(amat + GT * 16 * D);          // [8][GT][16]
  int* red_j = reinterpret_cast<int*>(red_s + 8 * GT * 16);             // [8][GT][16]
  int* sub_valid = red_j + 8 * GT * 16;                                 // [R]
  uint64_t* keys = reinterpret_cast<uint64_t*>(sub_valid + 16);         // [GT][npow2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ngroups = a.num_q_heads / GT;
  const int I = a.nqb_total - 1 - static_cast<int>(blockIdx.x) / ngroups;   // longest rows first
  const int hg = static_cast<int>(blockIdx.x) % ngroups;
  const int h0 = hg * GT;
  const int kv = h0 / (a.num_q_heads / a.num_kv_heads);
  const int s = find_seq(a.cu_qblocks, a.batch, I);
  const int qb0 = __ldg(a.cu_qblocks + s);
  const int i = I - qb0;
  const int tok0 = __ldg(a.cu_seqlens + s);
  const int L = __ldg(a.cu_seqlens + s + 1) - tok0;
  const int b = a.block_size;
  const int nrows = min(b, L - i * b);
  const int n = i + 1;
  int npow2 = 1;
  while (npow2 < n) npow2 <<= 1;
  if (npow2 > a.npow2_max) {  // host sizing guarantees this cannot happen
    if (tid == 0) report(a.status, kErrBounds, 0x200);
    return;
  }

  // ---- phase 1: 16-row sub-row sums, token by token, fp32
  for (int item = tid; item < R * NCHUNK; item += 256) {
    const int r = item / NCHUNK, ch = item % NCHUNK;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    const long row0 = static_cast<long>(tok0) + i * b + r * 16;
    const __nv_bfloat16* src = a.q + (row0 * a.num_q_heads + h0) * D + ch * 8;
    const long stride = static_cast<long>(a.num_q_heads) * D;
    uint4 raw[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (r * 16 + t < nrows) raw[t] = __ldg(reinterpret_cast<const uint4*>(src + t * stride));
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (r * 16 + t < nrows) {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[t]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] = __fadd_rn(acc[2 * e], __low2float(p2[e]));
          acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], __high2float(p2[e]));
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) subsum[r * COLS + ch * 8 + e] = acc[e];
  }
  for (int x = tid; x < GT * 16 * D / 4; x += 256) reinterpret_cast<uint32_t*>(amat)[x] = 0u;
  if (tid < R) sub_valid[tid] = (tid * 16 < nrows) ? 1 : 0;
  for (int x = tid; x < GT * npow2; x += 256) keys[(x / npow2) * a.npow2_max + (x % npow2)] = ~0ull;
  __syncthreads();

  // ---- phase 2: block sum (fold of the sub-row sums) and int8 quantisation
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
  }
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
  const int8_t* kq = a.kq + (static_cast<long>(kv) * a.nqb_total + qb0) * D;
  const float* ksp = a.ks + static_cast<long>(kv) * a.nqb_total + qb0;
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

  // ---- phase 4: each head's k_i smallest keys, in ascending order
  // The 64-bit keys are unique (they end in the block index), so a radix
  // select from the top byte down finds exactly the k_i smallest: at every
  // pass the bucket holding the k-th key is narrowed until all of it is
  // kept.  Only those keys are then sorted.  When every candidate is kept
  // (k_i = n), or the small buffers do not fit, all candidates are sorted.
  const int k_i = static_cast<int>(max(1LL, (static_cast<long long>(n) * a.bp + 9999) / 10000));
  int kpow = 1;
  while (kpow < k_i) kpow <<= 1;
  const bool select_path = (k_i < n) && (GT * 256 * 4 + GT * kpow * 8 <= R * COLS * 4);
  const uint64_t* out_keys = keys;
  int out_stride = a.npow2_max;
  if (select_path) {
    int* hist = reinterpret_cast<int*>(subsum);                               // [GT][256]
    uint64_t* sel = reinterpret_cast<uint64_t*>(hist + GT * 256);             // [GT][kpow]
    unsigned long long* st_prefix = reinterpret_cast<unsigned long long*>(red_s);
    unsigned long long* st_mask = st_prefix + GT;
    int* st_need = reinterpret_cast<int*>(st_mask + GT);
    int* st_done = st_need + GT;
    int* st_cnt = st_done + GT;
    if (tid < GT) {
      st_prefix[tid] = 0ull;
      st_mask[tid] = 0ull;
      st_need[tid] = k_i;
      st_done[tid] = 0;
      st_cnt[tid] = 0;
    }
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int x = tid; x < GT * 256; x += 256) hist[x] = 0;
      __syncthreads();
      for (int mt = 0; mt < GT; ++mt) {
        if (st_done[mt]) continue;
        const unsigned long long pm = st_mask[mt], pv = st_prefix[mt];
        for (int j = tid; j < n; j += 256) {
          const uint64_t key = keys[mt * a.npow2_max + j];
          if ((key & pm) == pv) atomicAdd(&hist[mt * 256 + static_cast<int>((key >> shift) & 255u)], 1);
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
          st_need[warp] = rest;
          st_prefix[warp] |= static_cast<unsigned long long>(8 * lane + e) << shift;
          st_mask[warp] |= 255ull << shift;
          st_done[warp] = (c[e] == rest) ? 1 : 0;
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

// ============================================================ launchers
size_t score_smem_bytes(int D, int GT, int R, int npow2_max) {
  return static_cast<size_t>(R) * GT * D * 4 + static_cast<size_t>(GT) * 16 * D + 2 * 8 * GT * 16 * 4 + 16 * 4 +
         static_cast<size_t>(GT) * npow2_max * 8;
}

template <int D, int GT, int R>
static cudaError_t launch_score_t(const ScoreArgs& a, cudaStream_t stream) {
  const size_t smem = score_smem_bytes(D, GT, R, a.npow2_max);
  auto kern = kap_score_select_kernel<D, GT, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.nqb_total) * (a.num_q_heads / GT);
  kern<<<grid, 256, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int GT>
static cudaError_t launch_score_r(const ScoreArgs& a, cudaStream_t stream) {
  return a.block_size == 128 ? launch_score_t<D, GT, 8>(a, stream) : launch_score_t<D, GT, 4>(a, stream);
}

template <int D>
static cudaError_t launch_score_d(const ScoreArgs& a, int GT, cudaStream_t stream) {
  switch (GT) {
    case 1: return launch_score_r<D, 1>(a, stream);
    case 2: return launch_score_r<D, 2>(a, stream);
    default: return launch_score_r<D, 4>(a, stream);
  }
}

cudaError_t launch_kpool(const KPoolArgs& a, cudaStream_t stream) {
  const long items = static_cast<long>(a.nkb_total) * a.num_kv_heads;
  const unsigned grid = static_cast<unsigned>((items + 7) / 8);
  if (a.head_dim == 128) kpool_kernel<128><<<grid, 256, 0, stream>>>(a);
  else kpool_kernel<64><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreArgs& a, int GT, cudaStream_t stream) {
  return a.head_dim == 128 ? launch_score_d<128>(a, GT, stream) : launch_score_d<64>(a, GT, stream);
}

}  // namespace cosa
