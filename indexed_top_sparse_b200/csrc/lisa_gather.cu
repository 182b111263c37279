// Gather of the selected K/V rows into a contiguous buffer (sm_100a): the first half of the
// "gather, then attend" comparator the JSSA write-up argues against (section "Как JSSA сохраняет
// порядок токенов": the specialised kernel reads the selected rows in place because a gathered
// copy costs more than the attention itself).  Not on the decode path; it exists to measure that
// claim on this GPU beside the in-place attention.
//
// out[b][h][i] = (K row, V row) of position idx[b][h][i] for i < count[b][h], zeros after.
// One 16-byte chunk per thread-iteration, grid-strided: a plain bandwidth-bound copy.

#include "lisa_common.cuh"
#include "lisa_kernels.h"

namespace lisa {

namespace {

__global__ void __launch_bounds__(256) lisa_gather_kernel(GatherParams p) {
  pdl_wait();
  pdl_trigger();
  const int chunks = p.d * 2 / 16;  // 16-byte chunks of a K (or V) row
  const long long total = (long long)p.B * p.Hkv * p.M * 2 * chunks;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % chunks);
    const int part = (int)((e / chunks) % 2);  // 0: K, 1: V
    const long long row = e / (2 * chunks);    // (b, h, i)
    const int i = (int)(row % p.M);
    const long long bh = row / p.M;
    const int b = (int)(bh / p.Hkv), h = (int)(bh % p.Hkv);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    const int cnt = p.count[bh];
    const int n = min(max(p.seq_lens[b], 0), p.max_seq_len);
    if (i < cnt && cnt <= p.M) {
      const int t = p.idx[row];
      if (t >= 0 && t < n) {
        const int pg = p.page_table[(size_t)b * p.max_pages + (t >> p.log2ps)];
        if (pg >= 0 && pg < p.num_pages) {
          const size_t kv_row = ((size_t)pg * p.ps + (size_t)(t & (p.ps - 1))) * p.Hkv + h;
          const uint8_t* src = (part == 0 ? p.k_pool : p.v_pool) + kv_row * (size_t)p.kv_stride_bytes + c * 16;
          v = ldg_stream_16(src);
        } else if (c == 0 && part == 0) {
          flag_error(p.err, LISA_DEVERR_PAGE_ID);
        }
      } else if (c == 0 && part == 0) {
        flag_error(p.err, LISA_DEVERR_INDEX);
      }
    }
    reinterpret_cast<uint4*>(p.out)[e] = v;
  }
}

}  // namespace

cudaError_t launch_gather(const GatherParams& p, cudaStream_t stream) {
  return launch_pdl(lisa_gather_kernel, dim3(148 * 8), dim3(256), 0, stream, p);
}

}  // namespace lisa
