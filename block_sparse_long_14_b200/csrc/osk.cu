// Ordered-Skipping Kernel (OSK) for sm_100a.
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention":
//   §4.3 "Physical jumping over pages" -- the inner loop runs only over the
//        retained blocks; dropped blocks cost no iteration, no mask test and
//        no synchronisation.
//   §4.3 "In-kernel logic skip" -- after S = Q K^T of a visited block, the
//        value side (exp, row sum, P V) is skipped when the block's row
//        maxima are negligible against the running max; one vote per
//        128-row query tile.
//   §4.3 "Any-order page visiting" -- blocks are visited in the order KAP
//        emitted (HRM first) through a page remap of the paged KV cache.
//   §3.3 L1 -- QK^T is paid for every visited block; L2.1/L2.2 -- the test
//        uses the running max and is an AND over the tile's rows.
//   Appendix C.2 (Algorithm A) and D.1 (b = 128 logical blocks, pages of any
//        size b_p resolving a block; the vote reuses the on-chip row maxima).
//
// One CTA per (query head, q-block) tile, 320 threads, two CTAs per SM,
// warp-specialised:
//   warps 0-7  softmax: two threads per query row (TMEM lane), each owning
//              half of the block's key columns, read 32 columns at a time.
//              First pass: causal mask on the diagonal block, half-row max,
//              the skip vote (a row votes to skip iff both of its halves lie
//              below the threshold, so no exchange is needed: warp
//              __all_sync + one 256-thread named barrier).  Second pass, if
//              kept: exp2 -> bf16 P written back over the already-read S
//              columns in TMEM, partial row sums; lazy rescaling of its half
//              of O in TMEM; the epilogue O / l.
//   warp 8     producer: page remap (order -> page_table) and TMA loads of the
//              Q tile and of each block's K and V pages into one K and one V
//              slot.  Block and page ids are loaded two blocks ahead of the
//              copies and lane u issues the boxes of page u; a block ending
//              past the sequence is copied by hand with zero fill so no stray
//              page slot reaches an MMA.
//   warp 9     MMA issuer: S = Q K^T (M=128, N=b, K=d; both operands in shared
//              memory) into the TMEM S buffer, then O += P V (M=128, N=d,
//              K=b) with P read from TMEM, unless the tile voted to skip;
//              completion is signalled with tcgen05.commit.
// Inside a CTA the chain is sequential (S, softmax, P V, next S); the second
// CTA on the SM (98 KiB of shared memory, 256 TMEM columns and at most 96
// registers per thread each) fills its gaps, prologue and epilogue included.
// The tensor pipe executes one thread's MMAs in issue order, so P V of block
// t has read its P before S of block t+1 overwrites the same columns.
// Every wait is bounded; on expiry the CTA records COSA_ERR_TIMEOUT, drains
// its own copies and MMAs, frees TMEM and exits.
#include <cstdint>
#include <cmath>

#include "cosa_device.cuh"
#include "cosa_internal.h"
#include "osk_common.cuh"

namespace cosa {

namespace {

constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kStages = 1;        // K and V slots per CTA (two CTAs share an SM)

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[1];   // S of the c-th computed block is in TMEM (phase c & 1)
  uint64_t p_full[2];   // softmax verdict (and P, if kept) for the c-th computed block, by c & 1
  uint64_t o_done[2];   // P V of the k-th kept block has completed, by k & 1
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
  int skip_flag[2];            // by c & 1, like p_full
  int vote[2][kSoftmaxWarps];  // by c & 1
  int vote_end[kSoftmaxWarps];
  float half_max[2][2][kBQ];   // [c & 1][half][row]: exchange of half-row maxima; the
                               // epilogue reuses the slot after the last computed block
                               // for the partial row sums
  float half_ref[2][2][kBQ];   // [c & 1][half][row]: exchange of the halves' P references
};

template <int D, int BK>
struct Cfg {
  static constexpr int Q_BYTES = kBQ * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + kStages * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + kStages * KV_BYTES;
  static constexpr int HALF = BK / 2;   // key columns per softmax thread
  static constexpr int KPH = HALF / 16; // K=16 MMA steps per half
  // one S buffer (P of block t overwrites it) and O: 256 columns for b = d = 128,
  // so two CTAs share an SM's TMEM
  static constexpr int TMEM_O = BK;
  static constexpr int TMEM_NEED = BK + D;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
  // Shared memory is padded so that the CTAs resident on one SM never ask
  // for more than the SM's 512 TMEM columns together (an allocation would
  // otherwise wait for another CTA to finish).
  static constexpr int SMEM_USED = OFF_BAR + static_cast<int>(sizeof(Bars));
  static constexpr int SMEM_MIN = TMEM_COLS == 512 ? 116 * 1024 : TMEM_COLS == 256 ? 78 * 1024 : 0;
  static constexpr int SMEM = SMEM_USED > SMEM_MIN ? SMEM_USED : SMEM_MIN;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(kBQ, BK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kBQ, D, false, true);
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(OFF_BAR + sizeof(Bars) <= static_cast<size_t>(SMEM), "barrier block inside the allocation");
  static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
};

}  // namespace

// Two CTAs of 10 warps put 5 warps on some SM sub-partitions, each with 16K
// registers, which caps a thread at 96 registers.
template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 2)
    osk_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const OskArgs a) {
  using C = Cfg<D, BK>;
  extern __shared__ __align__(1024) unsigned char smem[];
  // The operand tiles need 1024-byte alignment for the 128B swizzle; dynamic
  // shared memory starts right after the CTA's reserved 1 KiB, which gives it.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report(a.status, kErrBounds, 0x3FF);
    return;
  }
  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sK = smem + C::OFF_K;
  unsigned char* sV = smem + C::OFF_V;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  volatile int* abort = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- tile: kv-head-major, longest rows first within a kv head
  const int G = a.num_q_heads / a.num_kv_heads;
  const int per_kv = G * a.nqb_total;
  const int tile = blockIdx.x;
  const int g = tile / per_kv;
  const int rem = tile % per_kv;
  const int I = a.nqb_total - 1 - rem / G;
  const int h = g * G + rem % G;
  const int s = find_seq(a.cu_qblocks, a.batch, I);
  const int b = a.block_size;
  // rows of this tile: absolute positions i*b + r, present for r in [rlo, rhi)
  // (rlo > 0 only in the first q-block after a cached prefix); row r is
  // packed q/out row q_row0 + i*b + r
  const SeqSpan sp = seq_span(a.cu_seqlens, a.kv_lens, s, b);
  const int i = I - __ldg(a.cu_qblocks + s) + sp.i0;
  const long q_row0 = sp.q_row0;
  const int L = sp.L;
  const int rlo = max(0, sp.off - i * b);
  const int rhi = min(b, L - i * b);
  const int nkb = (L + b - 1) / b;
  if (sp.off < 0 || rlo >= rhi) {   // offsets disagree with the lengths: nothing is touched
    if (tid == 0) report(a.status, kErrBounds, 0x302);
    return;
  }
  // skip threshold of this sequence: one tau, or tau_s = delta / L_s
  const float log2_tau = a.tau_per_seq ? a.log2_delta - log2f(static_cast<float>(L)) : a.log2_tau;
  const long row_id = static_cast<long>(h) * a.nqb_total + I;
  int n = __ldg(a.count + row_id);
  if (n < 0 || n > a.kmax) {
    if (tid == 0) report(a.status, kErrBounds, 0x301);
    n = n < 0 ? 0 : a.kmax;
  }
  const int32_t* ord = a.order + row_id * a.kmax;
  // logical-mask execution: entry t of the list is computed only where keep != 0
  const uint8_t* keep_row = a.keep != nullptr ? a.keep + row_id * a.kmax : nullptr;
  const int32_t* pt_row = a.page_table + static_cast<long>(s) * a.max_pages_per_seq;

  if (tid == kProducerWarp * 32) {
    mbar_init(&bars->q_full, 1);
    for (int x = 0; x < kStages; ++x) {
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
      mbar_init(&bars->v_full[x], 1);
      mbar_init(&bars->v_empty[x], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->p_full[x], kSoftmaxWarps);   // one arrival per softmax warp
      mbar_init(&bars->o_done[x], 1);
    }
    mbar_init(&bars->mma_drain, 1);
    bars->abort = 0;
    mbar_fence_init();
    if (n > 0) {
      prefetch_tmap(&qmap);
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
#pragma unroll
      // a negative or past-the-end row coordinate reads zeros; those rows are not present
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sQ + c * (kBQ * 128), &qmap, &bars->q_full, c * 64, h, static_cast<int>(q_row0 + i * b));
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (n == 0) {
    // nothing listed: zero rows, zero counts
    if (tid >= rlo && tid < rhi) {
      uint4* dst = reinterpret_cast<uint4*>(a.out + ((q_row0 + i * b + tid) * a.num_q_heads + h) * D);
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid == 0) { a.visited[row_id] = 0; a.skipped[row_id] = 0; }
    if (a.skipbits != nullptr && tid < a.kmax) a.skipbits[row_id * a.kmax + tid] = 0;
  } else if (warp == kProducerWarp) {
    // =========================================================== producer
    int k_armed[kStages], v_armed[kStages];
    for (int x = 0; x < kStages; ++x) k_armed[x] = v_armed[x] = -1;
    bool ok = true;
    const int ppb = b / a.page_size;
    // Lane u < ppb holds page u of a block.  The loads run ahead of the
    // copies: the id of block t+2 and the page ids of block t+1 are already
    // in registers when block t is issued, so the order -> page table chain
    // of dependent loads never stalls a copy.
    auto block_id = [&](int t) { return t < n ? __ldg(ord + t) : -1; };
    auto page_of = [&](int jb) {
      return (lane < ppb && jb >= 0 && jb < nkb && jb * b + lane * a.page_size < L) ? __ldg(pt_row + jb * ppb + lane)
                                                                                     : -1;
    };
    int j_c = block_id(0);
    int pg_c = page_of(j_c);
    int j_n = block_id(1);
    int pg_n = page_of(j_n);
    int j_nn = block_id(2);
    int ncopy = 0;   // entries copied so far (all of them, unless a keep mask passes some over)
    for (int t = 0; t < n && ok; ++t) {
      if (keep_row != nullptr && __ldg(keep_row + t) == 0) {
        j_c = j_n;
        pg_c = pg_n;
        j_n = j_nn;
        pg_n = page_of(j_nn);
        j_nn = block_id(t + 3);
        continue;
      }
      const int slot = ncopy % kStages, use = ncopy / kStages;
      int j = j_c;
      const int page = pg_c;
      bool jvalid = (j >= 0 && j < nkb);
      if (!jvalid) {
        if (lane == 0) report(a.status, kErrBounds, 0x302);
        j = 0;
      }
      const int nvalid = jvalid ? min(b, L - j * b) : 0;
      // a bad page id sends the block down the checked path
      const bool pages_ok = __all_sync(0xffffffffu, lane >= ppb || (page >= 0 && page < a.num_pages));
      const bool via_tma = jvalid && nvalid == b && pages_ok;
      // lane u < ppb: first pool row of page u (HND), or its token row (NHD, with kv head g as y)
      const int row = a.nhd ? page * a.page_size : (page * a.num_kv_heads + g) * a.page_size;
      // look-ahead loads, consumed one and two blocks later
      const int pg_nn = page_of(j_nn);
      const int j_nnn = block_id(t + 3);
      for (int kvsel = 0; kvsel < 2 && ok; ++kvsel) {
        uint64_t* full = kvsel == 0 ? &bars->k_full[slot] : &bars->v_full[slot];
        uint64_t* empty = kvsel == 0 ? &bars->k_empty[slot] : &bars->v_empty[slot];
        unsigned char* stage = (kvsel == 0 ? sK : sV) + slot * C::KV_BYTES;
        const CUtensorMap* map = kvsel == 0 ? &kmap : &vmap;
        if (use >= 1) ok = mbar_wait(empty, (use - 1) & 1, a.wait_limit, abort, a.status, 0x10 + kvsel);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (via_tma) {
          if (lane == 0) mbar_arrive_expect_tx(full, C::KV_BYTES);
          __syncwarp();
          if (lane < ppb) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              unsigned char* dst = stage + c * (BK * 128) + lane * a.page_size * 128;
              if (a.nhd) tma_load_3d(dst, map, full, c * 64, g, row);
              else tma_load_2d(dst, map, full, c * 64, row);
            }
          }
          __syncwarp();
        } else {
          manual_block_copy<D, BK>(stage, kvsel == 0 ? a.k_pages : a.v_pages, pt_row, j, nvalid, a, g, lane);
          if (lane == 0) mbar_arrive(full);
        }
        if (kvsel == 0) k_armed[slot] = use; else v_armed[slot] = use;
      }
      ++ncopy;
      j_c = j_n;
      pg_c = pg_n;
      j_n = j_nn;
      pg_n = pg_nn;
      j_nn = j_nnn;
    }
    // drain: every load this warp started has landed before the CTA exits
    if (lane == 0) {
      mbar_drain(&bars->q_full, 0);
      for (int x = 0; x < kStages; ++x) {
        if (k_armed[x] >= 0) mbar_drain(&bars->k_full[x], k_armed[x] & 1);
        if (v_armed[x] >= 0) mbar_drain(&bars->v_full[x], v_armed[x] & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      bool ok = mbar_wait(&bars->q_full, 0, a.wait_limit, abort, a.status, 0x20);
      int kept = 0;
      // S = Q K^T of the u-th computed block into the S buffer (its commits follow separately)
      auto issue_s = [&](int u) -> bool {
        const int slot = u % kStages, use = u / kStages;
        if (!mbar_wait(&bars->k_full[slot], use & 1, a.wait_limit, abort, a.status, 0x21)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t ad = sw128_desc(q_base + (ks >> 2) * (kBQ * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(k_base + slot * C::KV_BYTES + (ks >> 2) * (BK * 128) + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem, ad, bd, C::IDESC_QK, ks > 0 ? 1u : 0u);
        }
        return true;
      };
      auto commit_s = [&](int u) {
        tc_commit(&bars->s_full[0]);
        tc_commit(&bars->k_empty[u % kStages]);
      };
      // the next list entry at or after x that is computed (every one, unless a keep mask passes some over)
      auto next_entry = [&](int x) {
        if (keep_row != nullptr)
          while (x < n && __ldg(keep_row + x) == 0) ++x;
        return x;
      };
      int t = next_entry(0);
      if (t < n && ok) {
        ok = issue_s(0);
        if (ok) commit_s(0);
      }
      for (int u = 0; t < n && ok; ++u) {
        const int vslot = u % kStages, vuse = u / kStages;
        ok = mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1, a.wait_limit, abort, a.status, 0x23);
        if (ok) ok = mbar_wait(&bars->v_full[vslot], vuse & 1, a.wait_limit, abort, a.status, 0x24);
        if (!ok) break;
        tc_fence_after();
        const int skip = *reinterpret_cast<volatile int*>(&bars->skip_flag[u & 1]);
        if (!skip) {
          const uint32_t p_tmem = tmem;
          const uint32_t d_o = tmem + C::TMEM_O;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // P of keys [16kk, 16kk+16): half kk / KPH wrote its P into the first
            // HALF/2 columns of its own S half
            const uint32_t a_t = p_tmem + (kk / C::KPH) * C::HALF + (kk % C::KPH) * 8;
            const uint64_t bd = sw128_desc(v_base + vslot * C::KV_BYTES + kk * 2048, BK * 128, 1024);
            tc_mma_ts(d_o, a_t, bd, C::IDESC_PV, (kept > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          mbar_arrive(&bars->v_empty[vslot]);   // no MMA reads this V
        }
        // S of the next computed block queues right behind P V (the tensor pipe keeps issue
        // order, so P V has read P before S overwrites it); the commits follow, and each
        // arrives once every MMA issued before it has completed
        const int tn = next_entry(t + 1);
        const bool has_next = tn < n;
        if (has_next) ok = issue_s(u + 1);
        if (!skip) {
          tc_commit(&bars->v_empty[vslot]);
          tc_commit(&bars->o_done[kept & 1]);
          ++kept;
        }
        if (has_next && ok) commit_s(u + 1);
        t = tn;
      }
      // drain: all MMAs issued by this thread complete before TMEM is freed
      tc_commit(&bars->mma_drain);
      mbar_drain(&bars->mma_drain, 0);
    }
    __syncwarp();
  } else {
    // =========================================================== softmax (warps 0-7)
    const SoftmaxTile x{tmem, warp, 1, i, b, rlo, rhi, q_row0, h, row_id, n, ord, keep_row, log2_tau};
    const SoftmaxSync y{&bars->s_full[0], bars->p_full, bars->o_done, bars->skip_flag, &bars->vote[0][0],
                        bars->vote_end, &bars->half_max[0][0][0], &bars->half_ref[0][0][0]};
    softmax_tile<D, BK>(a, x, y, abort);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int BK>
static cudaError_t launch_t(const OskArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                            const CUtensorMap& vmap, cudaStream_t stream) {
  using C = Cfg<D, BK>;
  auto kern = osk_kernel<D, BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.num_q_heads) * a.nqb_total;
  kern<<<grid, kThreads, C::SMEM, stream>>>(qmap, kmap, vmap, a);
  return cudaGetLastError();
}

size_t osk_smem_bytes(int head_dim, int block_size) {
  if (head_dim == 128) return block_size == 128 ? Cfg<128, 128>::SMEM : Cfg<128, 64>::SMEM;
  return block_size == 128 ? Cfg<64, 128>::SMEM : Cfg<64, 64>::SMEM;
}

cudaError_t launch_osk(const OskArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       int head_dim, cudaStream_t stream) {
  if (head_dim == 128)
    return a.block_size == 128 ? launch_t<128, 128>(a, qmap, kmap, vmap, stream)
                               : launch_t<128, 64>(a, qmap, kmap, vmap, stream);
  return a.block_size == 128 ? launch_t<64, 128>(a, qmap, kmap, vmap, stream)
                             : launch_t<64, 64>(a, qmap, kmap, vmap, stream);
}

}  // namespace cosa
