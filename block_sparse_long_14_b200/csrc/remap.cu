// Page remap: the KAP visit list -> physical KV pages.
//
// "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention", §4.3 "Any-order page visiting": OSK is fed the ordered
// activated block-ID list and remaps it at page granularity, so it composes
// with PagedAttention-style caches; Appendix D.1: a logical block resolves
// through b / b_p pages.  One thread per output entry.
#include "cosa_device.cuh"
#include "cosa_internal.h"

namespace cosa {

__global__ void __launch_bounds__(256) remap_kernel(RemapArgs a) {
  const int ppb = a.block_size / a.page_size;
  const long per_row = static_cast<long>(a.kmax) * ppb;
  const long total = static_cast<long>(a.num_q_heads) * a.nqb_total * per_row;
  for (long x = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<long>(gridDim.x) * blockDim.x) {
    const long row = x / per_row;
    const int e = static_cast<int>(x % per_row);
    const int t = e / ppb, u = e % ppb;
    const int I = static_cast<int>(row % a.nqb_total);
    int out = -1;
    if (t < __ldg(a.count + row)) {
      const int s = find_seq(a.cu_qblocks, a.batch, I);
      const int L = seq_span(a.cu_seqlens, a.kv_lens, s, a.block_size).L;   // key count
      const int nkb = (L + a.block_size - 1) / a.block_size;
      const int j = __ldg(a.order + row * a.kmax + t);
      if (j < 0 || j >= nkb) {
        report(a.status, kErrBounds, 0x400);
      } else if (j * a.block_size + u * a.page_size < L) {
        const int lp = j * ppb + u;
        if (lp < a.max_pages_per_seq) out = __ldg(a.page_table + static_cast<long>(s) * a.max_pages_per_seq + lp);
        else report(a.status, kErrBounds, 0x401);
      }
    }
    a.pages[x] = out;
  }
}

cudaError_t launch_remap(const RemapArgs& a, cudaStream_t stream) {
  const long total = static_cast<long>(a.num_q_heads) * a.nqb_total * a.kmax * (a.block_size / a.page_size);
  const long want = (total + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 148L * 16 ? (want < 1 ? 1 : want) : 148L * 16);
  remap_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace cosa
