// Append step of indexed sparse decode (sm_100a): the producer side of the caches.
//
// What is computed (JSSA write-up, section "Как JSSA сохраняет порядок токенов": every cached
// position has a projected key in a low-rank subspace, stored as FP8 beside the full-size keys and
// values): the current token's key and value rows are copied into the paged K/V pools, and its
// projected key c = P_h k is stored in the projected-key pool, quantised to E4M3 with the head's
// scale.  The FP8 code is an integer decided by floating point, so the arithmetic is pinned down
// (fp32, sequential over d, each product and sum rounded separately) to make every code
// reproducible bit for bit on any implementation that follows the same steps.
//
// One CTA per (KV head, sequence): 16-byte copies of the K/V rows, and one thread per projected
// dimension for the dot product.  The work is a few hundred bytes per (b, h): latency bound.

#include <cuda_fp8.h>

#include "lisa_common.cuh"
#include "lisa_kernels.h"

namespace lisa {

namespace {

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads) lisa_append_kernel(AppendParams p) {
  __shared__ float kf[128];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const size_t bh = (size_t)b * p.Hkv + h;
  pdl_wait();  // k_new / v_new and the pools may come from the previous kernel
  pdl_trigger();
  int t = p.positions != nullptr ? p.positions[b] : p.seq_lens[b] - 1;
  if (t < 0 || t >= p.max_seq_len) {
    if (tid == 0) flag_error(p.err, LISA_DEVERR_INDEX);
    return;
  }
  const int pg = p.page_table[(size_t)b * p.max_pages + (t >> p.log2ps)];
  if (pg < 0 || pg >= p.num_pages) {
    if (tid == 0) flag_error(p.err, LISA_DEVERR_PAGE_ID);
    return;
  }
  const size_t slot = (size_t)pg * p.ps + (size_t)(t & (p.ps - 1));
  // K and V rows: d bf16 each, 16 bytes per thread.
  const size_t kv_row = slot * p.Hkv + h;
  const uint4* ksrc = reinterpret_cast<const uint4*>(p.k_new + bh * p.d);
  const uint4* vsrc = reinterpret_cast<const uint4*>(p.v_new + bh * p.d);
  uint4* kdst = reinterpret_cast<uint4*>(p.k_pool + kv_row * (size_t)p.kv_stride_bytes);
  uint4* vdst = reinterpret_cast<uint4*>(p.v_pool + kv_row * (size_t)p.kv_stride_bytes);
  const int chunks = p.d * 2 / 16;
  if (tid < chunks) kdst[tid] = ksrc[tid];
  else if (tid < 2 * chunks) vdst[tid - chunks] = vsrc[tid - chunks];
  // Projected key: c_i = sum_j P[h][i][j] * k[j], fp32, j ascending, no fused multiply-add.
  for (int j = tid; j < p.d; j += blockDim.x) kf[j] = __bfloat162float(p.k_new[bh * p.d + j]);
  __syncthreads();
  if (tid < p.r) {
    const float* Pr = p.P + ((size_t)h * p.r + tid) * p.d;
    float c = 0.f;
    for (int j = 0; j < p.d; ++j) c = __fadd_rn(c, __fmul_rn(Pr[j], kf[j]));
    const size_t crow = ((size_t)pg * p.Hkv + h) * p.ps + (size_t)(t & (p.ps - 1));
    if (p.kproj_fp8) {
      const float x = __fdiv_rn(c, p.kproj_scale[h]);
      const __nv_fp8_storage_t code = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
      reinterpret_cast<uint8_t*>(p.kproj)[crow * p.r + tid] = (uint8_t)code;
    } else {
      reinterpret_cast<float*>(p.kproj)[crow * p.r + tid] = c;
    }
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  return launch_pdl(lisa_append_kernel, dim3(p.Hkv, p.B), dim3(kAppendThreads), 0, stream, p);
}

}  // namespace lisa
