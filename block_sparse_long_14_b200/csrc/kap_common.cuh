// Device helpers shared by the Kernel-Aware Proxy kernels (kap.cu, kap_stream.cu).
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §4.2 (block ranking, flag-grouped sorting) and Appendix
// C.1 / Figure A (HRM group first, each group by score): the sort key that
// orders a row's candidates, the proxy tile's geometry, the int8 tcgen05 MMA
// and the warp radix select of a row's k_i smallest keys.
#pragma once

#include <cstdint>

#include "cosa_device.cuh"
#include "cosa_internal.h"

namespace cosa {

static constexpr float kTiny = 1.17549435e-38f;  // 2^-126: smallest normal fp32

// Sort key: bit 63 = not HRM, bits 31..62 = score mapped to an unsigned
// order that is descending in the score, bits 0..30 = block index.
// Ascending keys give (HRM first, score descending, index ascending).
// The score bits of a sort key: an unsigned order descending in the score.
__device__ __forceinline__ uint32_t score_bits(float sc) {
  uint32_t u = __float_as_uint(sc);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;                         // -0 -> +0
  const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~asc;
}

// The sort key of a non-HRM block j from its score bits.
__device__ __forceinline__ uint64_t key_of(uint32_t bits, int j) {
  return (1ull << 63) | (static_cast<uint64_t>(bits) << 31) | static_cast<uint32_t>(j);
}

__device__ __forceinline__ uint64_t make_key(float sc, int j) { return key_of(score_bits(sc), j); }

// The score a sort key was made from (make_key is a bijection on non-zero
// floats and maps both zeros to +0).
__device__ __forceinline__ float score_of_key(uint64_t key) {
  const uint32_t asc = ~static_cast<uint32_t>(key >> 31);
  return __uint_as_float((asc & 0x80000000u) ? (asc & 0x7FFFFFFFu) : ~asc);
}

// A sub-row candidate as one ordered word: the score's order-preserving bits
// above the complemented block index, so the larger word is the better
// candidate (higher score; the lower index on equal scores) and 0 is below
// every real one.
__device__ __forceinline__ uint64_t pack_best(float s, int j) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;                       // -0 -> +0
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(~j);
}

// Tile of the proxy: (q-block I, GT query heads h0.. sharing kv head kv).
// Its query rows are the tile rows [rlo, rhi) (absolute positions i*b + r);
// rlo > 0 only in the first q-block after a cached prefix.  Row r of the
// tile is packed q row q_row0 + i*b + r.  kb0: key block 0 of the sequence
// in the pooled-key arrays.  bad: the offsets disagree with the lengths.
struct Tile {
  int I, h0, kv, s, kb0, i, L, rlo, rhi, n, npow2;
  long q_row0;
  bool bad;
};

// Sub-row v (tile rows 16v .. 16v + 15) holds at least one query row.
__device__ __forceinline__ bool sub_present(const Tile& t, int v) { return v * 16 < t.rhi && v * 16 + 16 > t.rlo; }

// Tile number `tile` of the proxy grid: q-blocks from the last (the longest
// rows) to the first, each split into groups of GT query heads.
template <int GT>
__device__ __forceinline__ Tile tile_at(const ScoreArgs& a, int tile) {
  Tile t;
  const int ngroups = a.num_q_heads / GT;
  t.I = a.nqb_total - 1 - tile / ngroups;
  t.h0 = (tile % ngroups) * GT;
  t.kv = t.h0 / (a.num_q_heads / a.num_kv_heads);
  t.s = find_seq(a.cu_qblocks, a.batch, t.I);
  const SeqSpan sp = seq_span(a.cu_seqlens, a.kv_lens, t.s, a.block_size);
  t.kb0 = __ldg(a.cu_kblocks + t.s);
  t.i = t.I - __ldg(a.cu_qblocks + t.s) + sp.i0;
  t.L = sp.L;
  t.q_row0 = sp.q_row0;
  t.rlo = max(0, sp.off - t.i * a.block_size);
  t.rhi = min(a.block_size, t.L - t.i * a.block_size);
  t.bad = sp.off < 0 || t.rlo >= t.rhi;
  t.n = t.i + 1;
  t.npow2 = 1;
  while (t.npow2 < t.n) t.npow2 <<= 1;
  return t;
}

// Two fp32 round-to-nearest products in one packed instruction (each exactly __fmul_rn).
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// x with bits [pos, pos + 8) replaced by the low 8 bits of v.
__device__ __forceinline__ uint32_t bfi8(uint32_t v, uint32_t x, int pos) {
  uint32_t d;
  asm("bfi.b32 %0, %1, %2, %3, 8;" : "=r"(d) : "r"(v), "r"(x), "r"(pos));
  return d;
}

// Stage-1 count of a row with n causal candidates: k_i = max(1, ceil(n bp / 10^4)).
__device__ __forceinline__ int keep_count(int n, int bp) {
  return static_cast<int>(max(1LL, (static_cast<long long>(n) * bp + 9999) / 10000));
}

// D[tmem] (+)= A[smem] * B[smem]^T with tcgen05 kind::i8: s8 x s8 -> exact s32.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::i8: D format S32 (2) at bit 4, A and B
// signed 8-bit (1) at bits 7 and 10, K-major operands, N >> 3 at bit 17,
// M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// A row's k_i smallest sort keys by one warp, with no CTA-wide barrier.  The
// 64-bit keys are unique, so the k_i smallest are found exactly by a radix
// select over 8-bit digits, starting at the first digit where the row's keys
// differ: each pass histograms the keys that share the prefix found so far (a
// warp-private 256-bin histogram) and narrows the prefix to the bin holding
// the k_i-th smallest key, until that bin is kept whole.  The kept keys are
// compacted by ballot into sel[0, kpow) (padded with ~0) and sorted ascending
// by a warp bitonic network in shared memory.  Requires 1 <= k_i < n,
// kpow = the power of two >= k_i.  Returns the number kept (k_i unless the
// counts are inconsistent, which is reported).
static __device__ int warp_select_smallest(const uint64_t* kr, int n, int k_i, int kpow, int* hist, uint64_t* sel,
                                    Status* status) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  // the leading digits every key shares decide nothing
  unsigned long long ka = ~0ull, ko = 0ull;
  for (int x = lane; x < n; x += 32) {
    const uint64_t key = kr[x];
    ka &= key;
    ko |= key;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    ka &= __shfl_xor_sync(kFull, ka, off);
    ko |= __shfl_xor_sync(kFull, ko, off);
  }
  int byte = __clzll(ka ^ ko) >> 3;                 // first digit, from the top, where keys differ
  unsigned long long mask = byte == 0 ? 0ull : (~0ull << (64 - 8 * byte));
  unsigned long long prefix = ka & mask;
  int need = k_i;                                   // keys still to take from the current bucket
  for (;;) {
    const int shift = 56 - 8 * byte;
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0;
    __syncwarp();
    for (int base = 0; base < n; base += 32) {      // every lane takes every iteration
      const int x = base + lane;
      int bin = -1;
      if (x < n) {
        const uint64_t key = kr[x];
        if ((key & mask) == prefix) bin = static_cast<int>((key >> shift) & 255u);
      }
      const unsigned same = __match_any_sync(kFull, bin);
      if (bin >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
    }
    __syncwarp();
    int c[8];
    int sum = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = hist[lane * 8 + e];
      sum += c[e];
    }
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, inc, off);
      if (lane >= off) inc += y;
    }
    const int excl = inc - sum;
    const bool mine = excl < need && need <= inc;   // this lane's bins hold the need-th key
    const unsigned who = __ballot_sync(kFull, mine);
    if (who == 0) {                                 // counts inconsistent: cannot happen
      if (lane == 0) report(status, kErrBounds, 0x206);
      return 0;
    }
    int digit = 0, rest = 0, whole = 0;
    if (mine) {
      int below = excl, e = 0;
      while (below + c[e] < need) below += c[e++];
      digit = 8 * lane + e;
      rest = need - below;
      whole = c[e] == rest ? 1 : 0;
    }
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(kFull, digit, src);
    rest = __shfl_sync(kFull, rest, src);
    whole = __shfl_sync(kFull, whole, src);
    prefix |= static_cast<unsigned long long>(digit) << shift;
    mask |= 255ull << shift;
    need = rest;
    __syncwarp();                                   // histogram reads done before it is cleared again
    if (whole || byte == 7) break;                  // at the last digit a bucket is a single key
    ++byte;
  }
  // keep every key at or below the prefix: exactly the k_i smallest
  int cnt = 0;
  for (int base = 0; base < n; base += 32) {
    const int x = base + lane;
    const uint64_t key = x < n ? kr[x] : ~0ull;
    const bool keep = x < n && (key & mask) <= prefix;
    const unsigned bal = __ballot_sync(kFull, keep);
    const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
    if (keep) {
      if (pos < kpow) sel[pos] = key;
      else report(status, kErrBounds, 0x207);
    }
    cnt += __popc(bal);
  }
  if (cnt != k_i && lane == 0) report(status, kErrBounds, 0x208);
  for (int t = min(cnt, kpow) + lane; t < kpow; t += 32) sel[t] = ~0ull;
  __syncwarp();
  // ascending bitonic sort of sel[0, kpow)
  for (int k = 2; k <= kpow; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < (kpow >> 1); i += 32) {
        const int x = ((i & ~(j - 1)) << 1) | (i & (j - 1));   // lower element of pair i
        const uint64_t va = sel[x], vb = sel[x + j];
        if ((va > vb) == ((x & k) == 0)) {
          sel[x] = vb;
          sel[x + j] = va;
        }
      }
      __syncwarp();
    }
  }
  return min(cnt, k_i);
}

// Ascending bitonic sort of 32 V keys (32- or 64-bit) held V per lane by a
// warp (element e of the sequence is v[e % V] of lane e / V): the in-lane
// stages compare registers, the others exchange with lane ^ (j / V) by
// shuffles.
template <int V, typename T>
__device__ __forceinline__ void warp_sort_regs(T (&v)[V]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 2; kk <= 32 * V; kk <<= 1) {
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j < V) {
#pragma unroll
        for (int q = 0; q < V; ++q) {
          const int q2 = q ^ j;
          if (q2 > q) {
            const bool asc = ((V * lane + q) & kk) == 0;
            if ((v[q] > v[q2]) == asc) {
              const T t = v[q];
              v[q] = v[q2];
              v[q2] = t;
            }
          }
        }
      } else {
        const int pl = j / V;
        const bool keep_min = ((lane & pl) == 0) == (((V * lane) & kk) == 0);
#pragma unroll
        for (int q = 0; q < V; ++q) {
          const T p = __shfl_xor_sync(0xffffffffu, v[q], pl);
          v[q] = keep_min ? (v[q] < p ? v[q] : p) : (v[q] > p ? v[q] : p);
        }
      }
    }
  }
}

// The k smallest of n unique 64-bit keys kr[0..n) by one warp, for k small
// against n: 64 keys taken at evenly spaced positions are sorted in registers;
// a threshold T is the sample at a rank that puts about 2k keys at or below
// it; one pass compacts every key <= T into buf (ballot); if fewer than k
// were kept the rank is raised and the pass repeated (on the 128K layer at a
// 5% budget: 4% of the rows, and the kept set is 1.9 k at the median).  The
// kept set, padded with ~0, is sorted (in registers up to 128 keys, else in
// shared memory as a bitonic network over a power of two) and left in
// buf[0, cnt): its first k keys are exactly the k smallest.  Requires
// 1 <= k < n.  Returns the number of kept keys (>= k), or -1 when the kept set
// would exceed `cap` keys or no sample reaches k (the caller then uses
// warp_select_smallest).
static __device__ int warp_select_sampled(const uint64_t* kr, int n, int k, uint64_t* buf, int cap) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  // sample element e = 2 lane + q, taken at position (e n) / 64
  uint64_t smp[2] = {kr[(2 * lane * n) >> 6], kr[((2 * lane + 1) * n) >> 6]};
  warp_sort_regs<2>(smp);
  int r = min(63, (64 * k + n - 1) / n + 1);   // about 2k keys at or below the r-th sample (the sample
                                                // spacing is n / 64 ranks)
  int cnt = 0;
  for (int attempt = 0;; ++attempt) {
    const uint64_t t0 = __shfl_sync(kFull, smp[0], r >> 1), t1 = __shfl_sync(kFull, smp[1], r >> 1);
    const uint64_t T = (r & 1) ? t1 : t0;
    cnt = 0;
    for (int base = 0; base < n; base += 32) {   // every lane takes every iteration
      const int x = base + lane;
      const uint64_t key = x < n ? kr[x] : ~0ull;
      const bool keep = x < n && key <= T;
      const unsigned bal = __ballot_sync(kFull, keep);
      const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
      if (keep && pos < cap) buf[pos] = key;
      cnt += __popc(bal);
    }
    if (cnt >= k || r == 63 || attempt == 2) break;
    r = min(63, r + r / 2 + 2);
  }
  if (cnt < k || cnt > cap) return -1;
  __syncwarp();
  if (cnt <= 128) {
    uint64_t v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = 4 * lane + q < cnt ? buf[4 * lane + q] : ~0ull;
    warp_sort_regs<4>(v);
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (4 * lane + q < cnt) buf[4 * lane + q] = v[q];
    __syncwarp();
    return cnt;
  }
  int P = 1;
  while (P < cnt) P <<= 1;
  for (int t = cnt + lane; t < P; t += 32) buf[t] = ~0ull;
  __syncwarp();
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < (P >> 1); i += 32) {
        const int x = ((i & ~(j - 1)) << 1) | (i & (j - 1));   // lower element of pair i
        const uint64_t va = buf[x], vb = buf[x + j];
        if ((va > vb) == ((x & kk) == 0)) {
          buf[x] = vb;
          buf[x + j] = va;
        }
      }
      __syncwarp();
    }
  }
  return cnt;
}

}  // namespace cosa
