// The Kernel-Aware Proxy as one persistent kernel (head_dim 128, budget cut).
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §5.1 (scoring and pooling run as one fused kernel),
// §4.2 (block ranking, flag-grouped sorting) and Appendix C.1 / Figure A (HRM
// group first, then the rest, each by score, cut to the stage-1 budget).
//
// One CTA per SM walks its share of the tiles (q-block x group of GT query
// heads sharing a kv head, longest rows first), described once into shared
// memory.  The work of a tile moves through warp roles connected by
// mbarriers, so that consecutive tiles overlap: while an epilogue group ranks
// tile X, the pooling warps already sum the query rows of tile X+1, whose
// chunks stream in by TMA.
//   warp 0      Q producer: the tile's rows in chunks of 16 (one sub-row,
//               GT heads x 128 dims, 4 KiB per head) into an even ring of QS
//               slots (chunk c: slot c % QS, pooling warps of parity c % 2).
//   warp 1      key producer: the pooled int8 key blocks of the tile's kv head,
//               128 blocks (16 KiB, 128B swizzle) per score tile, 3 slots.
//   warps 2-9   pooling, two warps per query head taking the even and the odd
//               sub-rows: the fp32 sum of each 16-row sub-row token by token,
//               its int8 quantisation written as the MMA's B operand
//               (double-buffered across tiles); the even warp then folds the
//               head's sub-row sums in order into the q-block vector.
//   warp 10     MMA issuer: D[j][v] = Kq_j . q_v (s8 x s8 -> exact s32) with
//               tcgen05 kind::i8, 128 key blocks in M (one TMEM lane each) and
//               the tile's GT (R + 1) vectors in N, into one of the two TMEM
//               accumulators of the tile's epilogue group.
//   warps 11-18 epilogue, two groups of four warps (TMEM lane quadrants 3, 0,
//               1, 2 and 3, 0, 1, 2) taking alternate tiles: each lane turns
//               one key block's dots into its score bits per head (written to
//               the workspace row of that head) and keeps the sub-rows'
//               running argmax; the group then reduces the argmax to the HRM
//               blocks of each head (written next to the scores).
// The selection runs in its own kernels: select_fast_kernel, one warp per
// (head, q-block) row, many rows per SM, a sampled threshold and a register
// sort of the few keys below it; select_rows_kernel for the rows it leaves.
// Scores, flags and lists are bit-identical to the two-stage kernels: the same
// fp32 operations in the same order, and integer dots.  Every wait is bounded;
// on expiry the CTA records COSA_ERR_TIMEOUT, lets its own copies and MMAs
// land, frees TMEM and exits.
#include <cstdint>

#include "cosa_device.cuh"
#include "cosa_internal.h"
#include "kap_common.cuh"

namespace cosa {

namespace {

constexpr int kD = 128;
constexpr int kThreads = 608;
constexpr int kQWarp = 0, kKWarp = 1, kPoolWarp0 = 2, kMmaWarp = 10, kEpiWarp0 = 11;
constexpr int kEpiThreads = 128;     // one epilogue group
constexpr int kEpiBar0 = 2;          // named barriers 2 and 3: the two epilogue groups
constexpr int kHeadBar0 = 4;         // named barriers 4 to 7: the two pooling warps of a head
constexpr int kSelCap = 256;         // kept keys per row of the sampled selection
constexpr int kRowWarps = 8;         // rows per CTA of the selection kernel
constexpr int kKeys = 128;           // key blocks per score tile
constexpr int kKStages = 3;
constexpr int kAccBufs = 4;          // TMEM accumulators: two per epilogue group

__host__ __device__ constexpr int stream_np(int GT, int R) { return (GT * (R + 1) + 15) / 16 * 16; }

template <int GT, int R>
struct Shape {
  static constexpr int NV = GT * (R + 1);          // query vectors of a tile
  static constexpr int NP = stream_np(GT, R);      // MMA N (a multiple of 16)
  static constexpr int NS = GT * R;                // sub-rows of a tile
  static constexpr int ACC = NP <= 32 ? 32 : 64;   // TMEM columns per accumulator
  static constexpr int TMEM_COLS = kAccBufs * ACC;
  static constexpr int QSLOT = 16 * GT * kD * 2;   // one chunk: 16 rows x GT heads x d bf16
  static constexpr int KSLOT = kKeys * kD;         // one score tile of int8 key vectors
  static constexpr int ASLOT = NP * kD;            // the int8 query vectors (B operand)
  static constexpr uint32_t IDESC = idesc_s8_s32(kKeys, NP);
};

struct Bars {
  uint64_t q_full[8], q_empty[8];
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t a_full[2], a_empty[2];
  uint64_t acc_full[kAccBufs], acc_empty[kAccBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// The pooling warps' int8 vector of one lane (4 dims) into row `row` of the
// 128B-swizzled B operand.
__device__ __forceinline__ void store_vec(unsigned char* amat, int row, int lane, uint32_t packed) {
  *reinterpret_cast<uint32_t*>(amat + row * 128 + (((lane >> 2) ^ (row & 7)) << 4) + (lane & 3) * 4) = packed;
}

// int8 quantisation of a vector spread over a warp (4 dims per lane): M = max |x|,
// x -> rint(x * (127 / M)) with both operations rounded to nearest; M below the
// normal range gives zeros.  Returns the lane's 4 codes packed, and M.
__device__ __forceinline__ uint32_t quantize4(const float (&x)[4], float& M_out) {
  float M = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) M = fmaxf(M, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float inv = (M < kTiny) ? 0.0f : __fdiv_rn(127.0f, M);
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = __float2int_rn(__fmul_rn(x[e], inv));   // to nearest, ties to even (= rint)
    packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * e);
  }
  M_out = M;
  return packed;
}

// The CTA's first kTileCache tiles are described once, in the prologue, into
// shared memory; every role reads them from there (later tiles, if any, are
// described where they are met).
constexpr int kTileCache = 64;

template <int GT>
__device__ __forceinline__ Tile cached_tile(const ScoreArgs& a, const Tile* tiles, int tile) {
  const int it = (tile - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x);
  return it < kTileCache ? tiles[it] : tile_at<GT>(a, tile);
}

// The epilogue group eg: takes the CTA's tiles of parity eg.  Each lane turns
// one key block's dots into its score bits per head (written to the workspace
// row of that head) and updates the sub-rows' running argmax; the group then
// reduces the argmax to the HRM blocks of each head (written next to the
// scores).
template <int GT, int R>
__device__ __forceinline__ void stream_epilogue(const ScoreArgs& a, const StreamLayout& lay, Bars* bars,
                                                volatile int* abort, uint32_t tmem, unsigned char* smem,
                                                const Tile* tiles) {
  using S = Shape<GT, R>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int eg = (warp - kEpiWarp0) >> 2;
  const int et = threadIdx.x - (kEpiWarp0 + 4 * eg) * 32;   // 0..127
  const int ew = (warp - kEpiWarp0) & 3;
  const int bar = kEpiBar0 + eg;
  const int quad = warp & 3;                   // TMEM lane quadrant
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * quad) << 16);
  float* sKs = reinterpret_cast<float*>(smem + lay.ks + eg * lay.group_bytes);
  uint64_t* red = reinterpret_cast<uint64_t*>(smem + lay.red + eg * lay.group_bytes);
  const int ntiles = a.nqb_total * (a.num_q_heads / GT);
  int u = 0, kloc = 0;   // key tiles consumed by this group; this CTA's good tiles so far
  bool ok = true;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const Tile tl = cached_tile<GT>(a, tiles, tile);
    if (tl.bad || tl.npow2 > a.npow2_max) {
      if (et == 0 && eg == 0) report(a.status, kErrBounds, 0x237);
      continue;
    }
    if ((kloc++ & 1) != eg) continue;
    const int n = tl.n;
    const float* ks_row = a.ks + static_cast<long>(tl.kv) * a.nkb_total + tl.kb0;
    for (int x = et; x < n; x += kEpiThreads) sKs[x] = __ldg(ks_row + x);
    named_bar_sync(bar, kEpiThreads);
    uint32_t* cand_row = a.cand + (static_cast<long>(tl.h0) * a.nqb_total + tl.I) * a.cand_stride;
    const long cand_head = static_cast<long>(a.nqb_total) * a.cand_stride;   // one head further

    // Each sub-row's best over this lane's key blocks: its score and the score tile it came
    // from (8 bits each, four to a word).  The lane meets its blocks in ascending order, so a
    // strictly higher score is needed to replace the best: on equal scores the lowest block
    // stays, as in the packed order of pack_best.
    float bs[S::NS];
    uint32_t bk[(S::NS + 3) / 4];
#pragma unroll
    for (int x = 0; x < S::NS; ++x) bs[x] = -INFINITY;
#pragma unroll
    for (int x = 0; x < (S::NS + 3) / 4; ++x) bk[x] = 0u;
    const int ntk = (n + kKeys - 1) / kKeys;
    for (int kt = 0; kt < ntk; ++kt, ++u) {
      const int ab = 2 * eg + (u & 1);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->acc_full[ab], (u >> 1) & 1, a.wait_limit, abort,
                                                   a.status, 0x238));
      if (!ok) continue;
      tc_fence_after();
      const int j = kt * kKeys + 32 * quad + lane;         // this lane's key block
      const float ksj = j < n ? sKs[j] : 0.0f;
      // this lane's dots, 16 columns at a time: column mt (R + 1) is head mt's block
      // vector (its score bits), the next R its sub-rows (their running argmax)
#pragma unroll
      for (int c = 0; c < S::NP / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(lane_base + ab * S::ACC + c * 16, r);
        tc_wait_ld();
        if (c == S::NP / 16 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);   // the accumulator may be overwritten
        }
        if (j < n) {
          // the scores of the 16 columns, two round-to-nearest products per packed instruction
          float svs[16];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float2 p = mul_f32x2(make_float2(static_cast<float>(static_cast<int>(r[e])),
                                                   static_cast<float>(static_cast<int>(r[e + 1]))),
                                       make_float2(ksj, ksj));
            svs[e] = p.x;
            svs[e + 1] = p.y;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = c * 16 + e;
            if (col >= S::NV) continue;
            const int mt = col / (R + 1), v = col % (R + 1);
            const float sv = svs[e];
            if (v == 0) {
              cand_row[mt * cand_head + j] = score_bits(sv);
            } else {
              const int x = mt * R + v - 1;
              if (sv > bs[x]) {
                bs[x] = sv;
                bk[x / 4] = bfi8(static_cast<uint32_t>(kt), bk[x / 4], 8 * (x % 4));
              }
            }
          }
        }
      }
    }
    // each sub-row's best over the warp's 32 lanes by a butterfly that halves the entries a
    // lane carries at each step (lane x ends with entry x), then over the group's four warps
    uint64_t best[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      if (x < S::NS) {
        const int jx = 128 * static_cast<int>((bk[x / 4] >> (8 * (x % 4))) & 0xFFu) + 32 * quad + lane;
        best[x] = bs[x] == -INFINITY ? 0ull : pack_best(bs[x], jx);
      } else {
        best[x] = 0ull;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int x = 0; x < o; ++x) {
        const uint64_t send = upper ? best[x] : best[x + o];
        const uint64_t keep = upper ? best[x + o] : best[x];
        const uint64_t got = __shfl_xor_sync(0xffffffffu, send, o);
        best[x] = got > keep ? got : keep;
      }
    }
    if (lane < S::NS) red[ew * S::NS + lane] = best[0];
    named_bar_sync(bar, kEpiThreads);
    // the HRM blocks: each present sub-row's argmax (8 slots per head, -1 where none)
    if (et < GT * 8 && ok) {
      const int mt = et / 8, sr = et % 8;
      int jv = -1;
      if (sr < R) {
        uint64_t v = red[mt * R + sr];
#pragma unroll
        for (int w = 1; w < 4; ++w) v = red[w * S::NS + mt * R + sr] > v ? red[w * S::NS + mt * R + sr] : v;
        const int jj = static_cast<int>(~static_cast<uint32_t>(v));
        if (v != 0ull && sub_present(tl, sr) && jj >= 0 && jj < n) jv = jj;
      }
      a.hrmj[((static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I) << 3) + sr] = jv;
    }
    named_bar_sync(bar, kEpiThreads);   // key scales and maxima are free for the group's next tile
  }
}

}  // namespace

template <int GT, int R>
__global__ void __launch_bounds__(kThreads, 1)
    kap_stream_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap kq_map,
                      const ScoreArgs a, const StreamLayout lay) {
  using S = Shape<GT, R>;
  extern __shared__ __align__(1024) unsigned char smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x2F0);
    return;
  }
  unsigned char* sQ = smem + lay.q;
  unsigned char* sK = smem + lay.k;
  unsigned char* sA = smem + lay.a;
  float* sSub = reinterpret_cast<float*>(smem + lay.sub);
  Tile* tiles = reinterpret_cast<Tile*>(smem + lay.tiles);
  Bars* bars = reinterpret_cast<Bars*>(smem + lay.bars);
  volatile int* abort = &bars->abort;
  const int QS = lay.q_stages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = a.nqb_total * (a.num_q_heads / GT);
  const int b = a.block_size;

  if (tid == 0) {
    if (a.retry != nullptr && blockIdx.x == 0) a.retry[0] = 0;   // the selection's retry list starts empty
    for (int x = 0; x < QS; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->q_empty[x], 4);            // the four pooling warps of the chunk's parity
    }
    for (int x = 0; x < kKStages; ++x) {
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->a_full[x], 8);             // the eight pooling warps
      mbar_init(&bars->a_empty[x], 1);
    }
    for (int x = 0; x < kAccBufs; ++x) {
      mbar_init(&bars->acc_full[x], 1);
      mbar_init(&bars->acc_empty[x], 4);          // the four warps of the group
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < kTileCache; x += kThreads) {
    const int tile = blockIdx.x + x * gridDim.x;
    if (tile < ntiles) tiles[x] = tile_at<GT>(a, tile);
  }
  // the padding rows of both B-operand buffers stay zero
  for (int x = tid; x < 2 * (S::NP - S::NV) * 32; x += kThreads) {
    const int buf = x / ((S::NP - S::NV) * 32), rem = x % ((S::NP - S::NV) * 32);
    reinterpret_cast<uint32_t*>(sA + buf * S::ASLOT + S::NV * 128)[rem] = 0u;
  }
  fence_proxy_async();
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kQWarp) {
    // ======================================================== Q producer
    if (lane == 0) {
      prefetch_tmap(&q_map);
      int qc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const Tile tl = cached_tile<GT>(a, tiles, tile);
        if (tl.bad || tl.npow2 > a.npow2_max) continue;
        for (int v = 0; v < R && ok; ++v, ++qc) {
          const int slot = qc % QS, use = qc / QS;
          if (use >= 1) ok = mbar_wait(&bars->q_empty[slot], (use - 1) & 1, a.wait_limit, abort, a.status, 0x230);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->q_full[slot], S::QSLOT);
          // rows outside the tile's present rows (or the tensor) are loaded but never summed
          tma_load_3d(sQ + slot * S::QSLOT, &q_map, &bars->q_full[slot], 0, tl.h0,
                      static_cast<int>(tl.q_row0 + static_cast<long>(tl.i) * b + 16 * v));
        }
      }
      // every chunk requested has landed before the CTA exits
      for (int c = max(0, qc - QS); c < qc; ++c) mbar_drain(&bars->q_full[c % QS], (c / QS) & 1);
    }
  } else if (warp == kKWarp) {
    // ======================================================== key producer
    if (lane == 0) {
      prefetch_tmap(&kq_map);
      int kc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const Tile tl = cached_tile<GT>(a, tiles, tile);
        if (tl.bad || tl.npow2 > a.npow2_max) continue;
        const int ntk = (tl.n + kKeys - 1) / kKeys;
        const int row0 = tl.kv * a.nkb_total + tl.kb0;
        for (int kt = 0; kt < ntk && ok; ++kt, ++kc) {
          const int slot = kc % kKStages, use = kc / kKStages;
          if (use >= 1) ok = mbar_wait(&bars->k_empty[slot], (use - 1) & 1, a.wait_limit, abort, a.status, 0x231);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->k_full[slot], S::KSLOT);
          // key blocks past the row's candidates are loaded but never read
          tma_load_2d(sK + slot * S::KSLOT, &kq_map, &bars->k_full[slot], 0, row0 + kt * kKeys);
        }
      }
      for (int c = max(0, kc - kKStages); c < kc; ++c) mbar_drain(&bars->k_full[c % kKStages], (c / kKStages) & 1);
    }
  } else if (warp < kMmaWarp) {
    // ======================================================== pooling: two warps per query head,
    // the even and the odd sub-rows
    const int pw = warp - kPoolWarp0;
    const int mt = pw & 3, half = pw >> 2;
    const bool active = mt < GT;
    int qc = 0, tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const Tile tl = cached_tile<GT>(a, tiles, tile);
      if (tl.bad || tl.npow2 > a.npow2_max) continue;
      const int buf = tcount & 1;
      if (tcount >= 2)
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->a_empty[buf], ((tcount >> 1) - 1) & 1, a.wait_limit,
                                                     abort, a.status, 0x232));
      unsigned char* amat = sA + buf * S::ASLOT;
      // the sub-row sums of head mt go through shared memory (double-buffered across tiles)
      float* sums = sSub + (buf * GT + (active ? mt : 0)) * R * kD + lane * 4;
#pragma unroll 1
      for (int v = half; v < R; v += 2) {
        const int c = qc + v, slot = c % QS;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->q_full[slot], (c / QS) & 1, a.wait_limit, abort,
                                                     a.status, 0x233));
        if (ok && active) {
          // sub-row v: rows 16v .. 16v + 15 of the tile, summed token by token (present rows
          // only); all 16 rows are read first so the loads overlap
          const unsigned char* src = sQ + slot * S::QSLOT + mt * (kD * 2) + lane * 8;
          uint2 raw[16];
#pragma unroll
          for (int rr = 0; rr < 16; ++rr) raw[rr] = *reinterpret_cast<const uint2*>(src + rr * (GT * kD * 2));
          const int lo_row = tl.rlo - 16 * v, hi_row = tl.rhi - 16 * v;   // present rows [lo_row, hi_row)
          // two fp32 round-to-nearest adds per packed instruction, each dimension in token order
          float2 s01 = make_float2(0.0f, 0.0f), s23 = make_float2(0.0f, 0.0f);
          if (lo_row <= 0 && hi_row >= 16) {   // the whole sub-row is present
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
              s01 = add_f32x2(s01, make_float2(__uint_as_float(raw[rr].x << 16), __uint_as_float(raw[rr].x & 0xFFFF0000u)));
              s23 = add_f32x2(s23, make_float2(__uint_as_float(raw[rr].y << 16), __uint_as_float(raw[rr].y & 0xFFFF0000u)));
            }
          } else {
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
              if (rr >= lo_row && rr < hi_row) {
                s01 = add_f32x2(s01, make_float2(__uint_as_float(raw[rr].x << 16), __uint_as_float(raw[rr].x & 0xFFFF0000u)));
                s23 = add_f32x2(s23, make_float2(__uint_as_float(raw[rr].y << 16), __uint_as_float(raw[rr].y & 0xFFFF0000u)));
              }
            }
          }
          float sub[4] = {s01.x, s01.y, s23.x, s23.y};
          *reinterpret_cast<float4*>(sums + v * kD) = make_float4(sub[0], sub[1], sub[2], sub[3]);
          float M;
          const uint32_t packed = quantize4(sub, M);
          store_vec(amat, mt * (R + 1) + 1 + v, lane, packed);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_empty[slot]);
      }
      qc += R;
      // the q-block vector: the fold of the sub-row sums in order (their sum from zero), by the
      // even warp once the odd one has written its sums
      named_bar_sync(kHeadBar0 + mt, 64);
      if (ok && active && half == 0) {
        float2 b01 = make_float2(0.0f, 0.0f), b23 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int v = 0; v < R; ++v) {
          const float4 t = *reinterpret_cast<const float4*>(sums + v * kD);
          b01 = add_f32x2(b01, make_float2(t.x, t.y));
          b23 = add_f32x2(b23, make_float2(t.z, t.w));
        }
        float blk[4] = {b01.x, b01.y, b23.x, b23.y};
        float M;
        const uint32_t packed = quantize4(blk, M);
        store_vec(amat, mt * (R + 1), lane, packed);
        if (a.qm != nullptr && lane == 0) a.qm[static_cast<long>(tl.h0 + mt) * a.nqb_total + tl.I] = M;
      }
      fence_proxy_async();   // the generic-proxy stores reach the tensor core's view of shared memory
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full[buf]);
      ++tcount;
    }
  } else if (warp == kMmaWarp) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      int kc = 0, tcount = 0;
      int accg[2] = {0, 0};   // key tiles issued to each epilogue group
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const Tile tl = cached_tile<GT>(a, tiles, tile);
        if (tl.bad || tl.npow2 > a.npow2_max) continue;
        const int buf = tcount & 1, eg = tcount & 1;   // the tile's B-operand buffer and epilogue group
        ok = mbar_wait(&bars->a_full[buf], (tcount >> 1) & 1, a.wait_limit, abort, a.status, 0x234);
        if (!ok) break;
        const uint32_t a_base = smem_u32(sA + buf * S::ASLOT);
        const int ntk = (tl.n + kKeys - 1) / kKeys;
        for (int kt = 0; kt < ntk; ++kt, ++kc) {
          const int slot = kc % kKStages;
          const int u = accg[eg], ab = 2 * eg + (u & 1);
          ok = mbar_wait(&bars->k_full[slot], (kc / kKStages) & 1, a.wait_limit, abort, a.status, 0x235);
          if (ok && u >= 2)
            ok = mbar_wait(&bars->acc_empty[ab], ((u >> 1) - 1) & 1, a.wait_limit, abort, a.status, 0x236);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + slot * S::KSLOT);
#pragma unroll
          for (int ks = 0; ks < kD / 32; ++ks)
            tc_mma_i8(tmem + ab * S::ACC, sw128_desc(k_base + ks * 32, 16, 1024), sw128_desc(a_base + ks * 32, 16, 1024),
                      S::IDESC, ks > 0 ? 1u : 0u);
          tc_commit(&bars->k_empty[slot]);   // the key slot is free once these MMAs complete
          tc_commit(&bars->acc_full[ab]);
          ++accg[eg];
        }
        if (!ok) break;
        tc_commit(&bars->a_empty[buf]);      // the tile's vectors are read
        ++tcount;
      }
      // every MMA issued here completes before TMEM is freed
      tc_commit(&bars->drain);
      mbar_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ======================================================== epilogue: scores and HRM flags
    stream_epilogue<GT, R>(a, lay, bars, abort, tmem, smem, tiles);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, S::TMEM_COLS);
}

// ============================================================ selection of the rows
// One warp per (query head, q-block) row, longest rows first: the row's n sort
// keys rebuilt in shared memory from its score bits (block index in the low
// bits, the HRM blocks' top bit cleared), then its k_i smallest by a sampled
// threshold (warp_select_sampled; warp_select_smallest when the kept set does
// not fit), or all n sorted when k_i = n; written as the ordered list.  Each
// warp owns its shared memory: keys [npow2_max], kept keys [cap], histogram
// [256]; no CTA-wide synchronisation.
static __device__ void select_row(const ScoreArgs& a, int cap, long rr, uint64_t* keys, uint64_t* sel, int* hist) {
  const int lane = threadIdx.x & 31;
  const int I = a.nqb_total - 1 - static_cast<int>(rr / a.num_q_heads);
  const int h = static_cast<int>(rr % a.num_q_heads);
  const int s = find_seq(a.cu_qblocks, a.batch, I);
  const SeqSpan sp = seq_span(a.cu_seqlens, a.kv_lens, s, a.block_size);
  const int i = I - __ldg(a.cu_qblocks + s) + sp.i0;
  const int n = i + 1;
  if (sp.off < 0 || n > a.npow2_max || n > a.cand_stride) {
    if (lane == 0) report(a.status, kErrBounds, 0x240);
    return;
  }
  const long row = static_cast<long>(h) * a.nqb_total + I;
  const uint32_t* cr = a.cand + row * a.cand_stride;
  for (int x = lane; x < n; x += 32) keys[x] = key_of(__ldg(cr + x), x);
  __syncwarp();
  if (lane < 8) {
    const int j = __ldg(a.hrmj + row * 8 + lane);
    if (j >= 0 && j < n) atomicAnd(reinterpret_cast<unsigned long long*>(&keys[j]), ~(1ull << 63));
  }
  __syncwarp();
  const int k_i = keep_count(n, a.bp);
  const uint64_t* out = sel;
  if (k_i < n) {
    if (warp_select_sampled(keys, n, k_i, sel, min(cap, kSelCap)) < 0) {
      int kpow = 1;
      while (kpow < k_i) kpow <<= 1;
      if (kpow <= cap) warp_select_smallest(keys, n, k_i, kpow, hist, sel, a.status);
      else if (lane == 0) report(a.status, kErrBounds, 0x241);   // host sizing forbids it
    }
  } else {
    // every candidate kept: sort them all
    int P = 1;
    while (P < n) P <<= 1;
    for (int t = n + lane; t < P; t += 32) keys[t] = ~0ull;
    __syncwarp();
    for (int kk = 2; kk <= P; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int q = lane; q < (P >> 1); q += 32) {
          const int x = ((q & ~(j - 1)) << 1) | (q & (j - 1));
          const uint64_t va = keys[x], vb = keys[x + j];
          if ((va > vb) == ((x & kk) == 0)) {
            keys[x] = vb;
            keys[x + j] = va;
          }
        }
        __syncwarp();
      }
    }
    out = keys;
  }
  const long o = row * a.kmax;
  const int k_out = min(k_i, a.kmax);
  if (k_out < k_i && lane == 0) report(a.status, kErrBounds, 0x242);   // host sizing forbids it
  for (int t = lane; t < a.kmax; t += 32) {
    const uint64_t key = t < k_out ? out[t] : 0ull;
    a.order[o + t] = t < k_out ? static_cast<int32_t>(key & 0x7FFFFFFFu) : -1;
    a.hrm[o + t] = (t < k_out && !(key >> 63)) ? 1 : 0;
  }
  int nh = 0;
  for (int base = 0; base < k_out; base += 32) {
    const int t = base + lane;
    nh += __popc(__ballot_sync(0xffffffffu, t < k_out && !(out[t] >> 63)));
  }
  if (lane == 0) {
    a.count[row] = k_out;
    a.n_hrm[row] = nh;
  }
}

// Rows r = 0 .. rows - 1 (list == nullptr), else the rows list[1 .. list[0]].
__global__ void __launch_bounds__(kRowWarps * 32) select_rows_kernel(const ScoreArgs a, int cap, const int32_t* list) {
  extern __shared__ __align__(16) unsigned char smem_rows[];
  const int warp = threadIdx.x >> 5;
  const size_t per_warp = static_cast<size_t>(a.npow2_max + cap) * 8 + 256 * 4;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_rows + warp * per_warp);
  uint64_t* sel = keys + a.npow2_max;
  int* hist = reinterpret_cast<int*>(sel + cap);
  const long rows = static_cast<long>(a.num_q_heads) * a.nqb_total;
  const long first = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  const long stride = static_cast<long>(gridDim.x) * (blockDim.x >> 5);
  if (list == nullptr) {
    for (long t = first; t < rows; t += stride) select_row(a, cap, t, keys, sel, hist);
  } else {
    const long cnt = min(static_cast<long>(__ldg(list)), rows);
    for (long t = first; t < cnt; t += stride) {
      const long rr = __ldg(list + 1 + t);
      if (rr >= 0 && rr < rows) select_row(a, cap, rr, keys, sel, hist);
      else if ((threadIdx.x & 31) == 0) report(a.status, kErrBounds, 0x243);
    }
  }
}

// ============================================================ register selection of the rows
// One warp per row, longest rows first, with no per-row shared-memory copy of
// the keys: each key is rebuilt from the row's score bits (read from L2, where
// the score kernel left them) and the row's HRM blocks (held in every lane).
// Rows of at most 32 candidates (or whose budget keeps them all) are sorted
// whole in registers; longer rows take a sampled threshold (the upper 32 bits
// of 64 keys at evenly spaced positions, sorted in registers), one ballot pass
// that compacts the keys at or below it into a 256-key buffer, and a register
// sort of the kept set (32, 64, 128 or 256 keys wide).  A row whose kept set
// does not fit, or whose samples never reach k_i, goes to the retry list
// (list[0] = length, list[1..] = rows) that select_rows_kernel finishes.
constexpr int kFastWarps = 8;
constexpr int kFastCap = 256;

struct RowKeys {
  const uint32_t* cr;
  int hb[8];        // the row's HRM blocks (-1: none)
  uint64_t lmask;   // bit m: block 32 m + lane is an HRM block (m < 64)
  __device__ __forceinline__ void init(int lane) {
    lmask = 0ull;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (hb[q] >= 0 && (hb[q] & 31) == lane && hb[q] < 64 * 32) lmask |= 1ull << (hb[q] >> 5);
  }
  // the sort key of block x
  __device__ __forceinline__ uint64_t at(int x) const {
    const uint64_t key = key_of(__ldg(cr + x), x);
    bool f = false;
#pragma unroll
    for (int q = 0; q < 8; ++q) f |= hb[q] == x;
    return f ? key & ~(1ull << 63) : key;
  }
  // the same for a block of this lane (x = 32 m + lane)
  __device__ __forceinline__ uint64_t at_lane(int x) const {
    if (x >= 64 * 32) return at(x);
    const uint64_t key = key_of(__ldg(cr + x), x);
    return ((lmask >> (x >> 5)) & 1ull) ? key & ~(1ull << 63) : key;
  }
};

// The sorted keys v (element e = V lane + q) as the row's ordered list: the
// first k_out keys' blocks and HRM flags, -1 / 0 padding up to kmax.
template <int V>
__device__ __forceinline__ void emit_row(const ScoreArgs& a, long row, const uint64_t (&v)[V], int k_out) {
  const int lane = threadIdx.x & 31;
  const long o = row * a.kmax;
  int nh = 0;
#pragma unroll
  for (int q = 0; q < V; ++q) {
    const int e = V * lane + q;
    const bool in = e < k_out;
    if (e < a.kmax) {
      a.order[o + e] = in ? static_cast<int32_t>(v[q] & 0x7FFFFFFFu) : -1;
      a.hrm[o + e] = (in && !(v[q] >> 63)) ? 1 : 0;
    }
    nh += __popc(__ballot_sync(0xffffffffu, in && !(v[q] >> 63)));
  }
  for (int t = 32 * V + lane; t < a.kmax; t += 32) {
    a.order[o + t] = -1;
    a.hrm[o + t] = 0;
  }
  if (lane == 0) {
    a.count[row] = k_out;
    a.n_hrm[row] = nh;
  }
}

// Sort cnt <= 32 V keys (from buf, or from the row itself when buf is null)
// in registers and emit the first k_out.
template <int V>
__device__ __forceinline__ void sort_emit(const ScoreArgs& a, long row, const RowKeys& rk, const uint64_t* buf, int cnt,
                                          int k_out) {
  const int lane = threadIdx.x & 31;
  uint64_t v[V];
#pragma unroll
  for (int q = 0; q < V; ++q) {
    // any placement before the sort: the row's own blocks by lane, the buffer's in runs
    const int x = buf != nullptr ? V * lane + q : 32 * q + lane;
    v[q] = x < cnt ? (buf != nullptr ? buf[x] : rk.at_lane(x)) : ~0ull;
  }
  warp_sort_regs<V>(v);
  emit_row<V>(a, row, v, k_out);
}

__global__ void __launch_bounds__(kFastWarps * 32) select_fast_kernel(const ScoreArgs a) {
  constexpr unsigned kFull = 0xffffffffu;
  __shared__ uint64_t kept_all[kFastWarps][kFastCap];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* buf = kept_all[warp];
  const long rr = static_cast<long>(blockIdx.x) * kFastWarps + warp;
  if (rr >= static_cast<long>(a.num_q_heads) * a.nqb_total) return;
  const int I = a.nqb_total - 1 - static_cast<int>(rr / a.num_q_heads);
  const int h = static_cast<int>(rr % a.num_q_heads);
  const int s = find_seq(a.cu_qblocks, a.batch, I);
  const SeqSpan sp = seq_span(a.cu_seqlens, a.kv_lens, s, a.block_size);
  const int n = I - __ldg(a.cu_qblocks + s) + sp.i0 + 1;
  if (sp.off < 0 || n > a.cand_stride) {
    if (lane == 0) report(a.status, kErrBounds, 0x244);
    return;
  }
  const long row = static_cast<long>(h) * a.nqb_total + I;
  RowKeys rk;
  rk.cr = a.cand + row * a.cand_stride;
  const int hj = lane < 8 ? __ldg(a.hrmj + row * 8 + lane) : -1;
#pragma unroll
  for (int q = 0; q < 8; ++q) rk.hb[q] = __shfl_sync(kFull, hj, q);
  rk.init(lane);
  const int k_i = keep_count(n, a.bp);
  const int k_out = min(k_i, a.kmax);
  if (k_out < k_i && lane == 0) report(a.status, kErrBounds, 0x245);   // host sizing forbids it

  if (k_i == n || n <= 32) {
    // every candidate kept, or few: sort them all
    if (n <= 32) sort_emit<1>(a, row, rk, nullptr, n, k_out);
    else if (n <= 64) sort_emit<2>(a, row, rk, nullptr, n, k_out);
    else if (n <= 128) sort_emit<4>(a, row, rk, nullptr, n, k_out);
    else if (n <= 256) sort_emit<8>(a, row, rk, nullptr, n, k_out);
    else if (lane == 0) a.retry[1 + atomicAdd(a.retry, 1)] = static_cast<int32_t>(rr);
    return;
  }
  // The threshold compares the keys' upper 32 bits (flag and score bits but the lowest):
  // the keys kept form a down-set of the order, so once there are k_i of them they hold the
  // k_i smallest.  Sample element e = 2 lane + q, taken at position (e n) / 64.
  uint32_t smp[2] = {static_cast<uint32_t>(rk.at((2 * lane * n) >> 6) >> 32),
                     static_cast<uint32_t>(rk.at(((2 * lane + 1) * n) >> 6) >> 32)};
  warp_sort_regs<2>(smp);
  int r = min(63, (64 * k_i + n - 1) / n + 1);   // about 2 k_i keys at or below the r-th sample
  int cnt = 0;
  for (int attempt = 0; attempt < 3; ++attempt) {
    const uint32_t t0 = __shfl_sync(kFull, smp[0], r >> 1), t1 = __shfl_sync(kFull, smp[1], r >> 1);
    const uint32_t T = (r & 1) ? t1 : t0;
    cnt = 0;
    for (int base = 0; base < n; base += 128) {   // four loads in flight per lane
      uint64_t key[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int x = base + 32 * u + lane;
        key[u] = x < n ? rk.at_lane(x) : ~0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool keep = base + 32 * u + lane < n && static_cast<uint32_t>(key[u] >> 32) <= T;
        const unsigned bal = __ballot_sync(kFull, keep);
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        if (keep && pos < kFastCap) buf[pos] = key[u];
        cnt += __popc(bal);
      }
    }
    if (cnt >= k_i || r == 63) break;
    r = min(63, r + r / 2 + 2);
  }
  __syncwarp();
  if (cnt < k_i || cnt > kFastCap) {
    if (lane == 0) a.retry[1 + atomicAdd(a.retry, 1)] = static_cast<int32_t>(rr);
  } else if (cnt <= 32) {
    sort_emit<1>(a, row, rk, buf, cnt, k_out);
  } else if (cnt <= 64) {
    sort_emit<2>(a, row, rk, buf, cnt, k_out);
  } else if (cnt <= 128) {
    sort_emit<4>(a, row, rk, buf, cnt, k_out);
  } else {
    sort_emit<8>(a, row, rk, buf, cnt, k_out);
  }
}

// ============================================================ host side
StreamLayout stream_layout(int GT, int R, int npow2_max, int kmax, int q_stages) {
  (void)kmax;
  const int np = stream_np(GT, R);
  StreamLayout L{};
  L.q_stages = q_stages;
  uint32_t off = 0;
  L.q = off;
  off += static_cast<uint32_t>(q_stages) * 16 * GT * kD * 2;
  L.k = off;
  off += kKStages * kKeys * kD;
  L.a = off;
  off += 2 * np * kD;
  L.sub = off;
  off += 2 * GT * R * kD * 4;
  L.tiles = off;
  off += (kTileCache * sizeof(Tile) + 15) / 16 * 16;
  // one region per epilogue group: key scales, sub-row maxima
  uint32_t g = 0;
  L.ks = off + g;
  g += (static_cast<uint32_t>(npow2_max) * 4 + 15) / 16 * 16;
  L.red = off + g;
  g += 4 * GT * R * 8;
  L.group_bytes = (g + 15) / 16 * 16;
  off += 2 * L.group_bytes;
  L.bars = off;
  off += (sizeof(Bars) + 15) / 16 * 16;
  L.total = off;
  return L;
}

bool stream_fits(int GT, int R, int npow2_max, int kmax, int* q_stages) {
  // an even ring: chunk c goes to slot c % QS and to the pooling warps of parity c % 2, so
  // each slot serves one parity and its waits come in order (with an odd ring the
  // even-chunk warps could wait on a slot's next use before its current chunk landed,
  // where the phase parity cannot tell the two apart)
  for (int qs = 8; qs >= 4; qs -= 2) {
    if (stream_layout(GT, R, npow2_max, kmax, qs).total <= kStreamSmemLimit) {
      *q_stages = qs;
      return true;
    }
  }
  return false;
}

template <int GT, int R>
static cudaError_t launch_stream_t(const ScoreArgs& a, const CUtensorMap& q_map, const CUtensorMap& kq_map,
                                   const StreamLayout& lay, int grid, cudaStream_t stream) {
  auto kern = kap_stream_kernel<GT, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(lay.total));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, lay.total, stream>>>(q_map, kq_map, a, lay);
  return cudaGetLastError();
}

static int rows_cap(int npow2_max, int kmax) {
  int kpow = 1;
  while (kpow < kmax) kpow <<= 1;
  if (kpow > npow2_max) kpow = npow2_max;
  return kpow > kSelCap ? kpow : kSelCap;
}

size_t select_rows_smem_bytes(int npow2_max, int kmax) {
  return static_cast<size_t>(npow2_max + rows_cap(npow2_max, kmax)) * 8 + 256 * 4;   // one warp's share
}

cudaError_t launch_select_rows(const ScoreArgs& a, cudaStream_t stream) {
  const int cap = rows_cap(a.npow2_max, a.kmax);
  const size_t per_warp = select_rows_smem_bytes(a.npow2_max, a.kmax);
  int warps = kRowWarps;
  while (warps > 1 && per_warp * warps > 200 * 1024) warps >>= 1;
  if (per_warp * warps > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(per_warp * warps));
  if (e != cudaSuccess) return e;
  const long rows = static_cast<long>(a.num_q_heads) * a.nqb_total;
  long grid = (rows + warps - 1) / warps;
  if (a.retry != nullptr && a.kmax <= 128) {
    // the register selection (kept sets of about 2 k_i fit its 256-key buffer), then the
    // rows it leaves, on a grid of two CTAs per SM
    select_fast_kernel<<<static_cast<unsigned>((rows + kFastWarps - 1) / kFastWarps), kFastWarps * 32, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    grid = grid < 2L * sms ? grid : 2L * sms;
    select_rows_kernel<<<static_cast<unsigned>(grid), warps * 32, per_warp * warps, stream>>>(a, cap, a.retry);
  } else {
    select_rows_kernel<<<static_cast<unsigned>(grid), warps * 32, per_warp * warps, stream>>>(a, cap, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_stream(const ScoreArgs& a, int GT, const CUtensorMap& q_map, const CUtensorMap& kq_map,
                          const StreamLayout& lay, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int ntiles = a.nqb_total * (a.num_q_heads / GT);
  const int grid = ntiles < sms ? ntiles : sms;
  if (grid < 1) return cudaSuccess;
  const bool b128 = a.block_size == 128;
  switch (GT) {
    case 1: return b128 ? launch_stream_t<1, 8>(a, q_map, kq_map, lay, grid, stream)
                        : launch_stream_t<1, 4>(a, q_map, kq_map, lay, grid, stream);
    case 2: return b128 ? launch_stream_t<2, 8>(a, q_map, kq_map, lay, grid, stream)
                        : launch_stream_t<2, 4>(a, q_map, kq_map, lay, grid, stream);
    default: return b128 ? launch_stream_t<4, 8>(a, q_map, kq_map, lay, grid, stream)
                         : launch_stream_t<4, 4>(a, q_map, kq_map, lay, grid, stream);
  }
}

}  // namespace cosa
