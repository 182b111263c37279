// Index stage of indexed sparse decode: indexer score and per-KV-head top-M selection (sm_100a).
//
// What is computed (JSSA write-up, section "Как JSSA сохраняет порядок токенов", decoding paragraph):
// the G queries of a KV head are averaged, projected with the head's r x d basis, and every cached
// position is scored against the FP8 (or fp32) projected-key cache; the M best positions are kept
// (a tie at the M-th score goes to the lower position) and reported in ascending order.
//
// Design on B200:
//  * Scoring streams the projected-key cache with 16-byte non-allocating vector loads, several per
//    thread in flight; a page block of one head (page_size * r bytes) is contiguous.  FP8 is decoded
//    with the hardware e4m3x2 -> f16x2 conversion and accumulated in fp32 on the CUDA cores (a single
//    query makes this a matrix-vector product: no tensor-core work to be had).
//  * Selection is fused with scoring.  A cluster of 8 CTAs owns one (b, KV head); each CTA scores a
//    contiguous, page-aligned eighth of the context into shared memory as order-preserving uint32
//    keys and builds a histogram of the top 11 key bits while the loads are in flight.  The eight
//    histograms are summed through distributed shared memory, the digit that holds the M-th key is
//    found, and two more passes (11 + 10 bits) pin the exact M-th key.  Each CTA then writes its
//    selected positions in ascending order at an offset derived from the other CTAs' counts.  No
//    fp32 score array ever goes to HBM on this path.

#include <cooperative_groups.h>

#include "lisa_common.cuh"
#include "lisa_kernels.h"

namespace cg = cooperative_groups;

namespace lisa {

namespace {

template <int R, bool FP8>
struct RowGeom {
  static constexpr int kElemBytes = FP8 ? 1 : 4;
  static constexpr int kRowBytes = R * kElemBytes;        // 16, 32, 64 or 128
  static constexpr int kLanesPerRow = kRowBytes / 16;     // 1, 2, 4, 8
  static constexpr int kRowsPerLoad = 32 / kLanesPerRow;  // rows one warp-wide 16-byte load covers
  static constexpr int kElemsPerLane = 16 / kElemBytes;   // elements in one 16-byte load
};

__device__ __forceinline__ int load_seq_len(const IndexParams& p, int b) {
  int n = p.seq_lens[b];
  if (n < 0 || n > p.max_seq_len) {
    flag_error(p.err, LISA_DEVERR_SEQ_LEN);
    n = n < 0 ? 0 : p.max_seq_len;
  }
  return n;
}

// qbar = mean of the G query rows of KV head h; u = P_h qbar.  Ends with a barrier.
__device__ void compute_projected_query(const IndexParams& p, int b, int h, float* qbar, float* u) {
  const int G = p.Hq / p.Hkv;
  for (int i = threadIdx.x; i < p.d; i += blockDim.x) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) acc += __bfloat162float(p.q[((size_t)b * p.Hq + (size_t)h * G + g) * p.d + i]);
    qbar[i] = acc / (float)G;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = warp; j < p.r; j += blockDim.x >> 5) {
    const float* Pr = p.P + ((size_t)h * p.r + j) * p.d;
    float acc = 0.f;
    for (int i = lane; i < p.d; i += 32) acc = fmaf(Pr[i], qbar[i], acc);
    acc = warp_sum(acc);
    if (lane == 0) u[j] = acc;
  }
  __syncthreads();
}

template <bool FP8>
__device__ __forceinline__ float dot16(const uint4& v, const float* uf) {
  if constexpr (FP8) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3);
      __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
      const float2 flo = __half22float2(*reinterpret_cast<__half2*>(&lo));
      const float2 fhi = __half22float2(*reinterpret_cast<__half2*>(&hi));
      a0 = fmaf(flo.x, uf[4 * i + 0], a0);
      a1 = fmaf(flo.y, uf[4 * i + 1], a1);
      a0 = fmaf(fhi.x, uf[4 * i + 2], a0);
      a1 = fmaf(fhi.y, uf[4 * i + 3], a1);
    }
    return a0 + a1;
  } else {
    float a = __uint_as_float(v.x) * uf[0];
    a = fmaf(__uint_as_float(v.y), uf[1], a);
    a = fmaf(__uint_as_float(v.z), uf[2], a);
    a = fmaf(__uint_as_float(v.w), uf[3], a);
    return a;
  }
}

// Score rows [t_begin, t_begin + nrows) of (b, h); t_begin is page aligned and pages[i] holds the
// (checked) page id of the i-th page of the range.  sink(local_row, score) runs on one lane per row.
template <int R, bool FP8, int U, class Sink>
__device__ __forceinline__ void stream_scores(const IndexParams& p, int h, int t_begin, int nrows,
                                              const int32_t* pages, const float* u, float scale, Sink sink) {
  using Geo = RowGeom<R, FP8>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int part = lane % Geo::kLanesPerRow, rsub = lane / Geo::kLanesPerRow;
  float uf[Geo::kElemsPerLane];
#pragma unroll
  for (int e = 0; e < Geo::kElemsPerLane; ++e) uf[e] = u[part * Geo::kElemsPerLane + e];
  const uint8_t* base = reinterpret_cast<const uint8_t*>(p.kproj);
  const int per_warp_iter = Geo::kRowsPerLoad * U;
  for (int r0 = warp * per_warp_iter; r0 < nrows; r0 += nwarps * per_warp_iter) {
    uint4 v[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int lr = r0 + k * Geo::kRowsPerLoad + rsub;
      if (lr < nrows) {
        const int t = t_begin + lr;
        const size_t row = (((size_t)pages[lr >> p.log2ps] * p.Hkv + h) << p.log2ps) + (t & (p.ps - 1));
        v[k] = ldg_stream_16(base + row * Geo::kRowBytes + part * 16);
      } else {
        v[k] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      float dot = dot16<FP8>(v[k], uf);
#pragma unroll
      for (int o = Geo::kLanesPerRow / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const int lr = r0 + k * Geo::kRowsPerLoad + rsub;
      if (part == 0 && lr < nrows) sink(lr, scale * dot);
    }
  }
}

// Checked page ids of pages [first_page, first_page + count) of sequence b.
__device__ __forceinline__ void load_pages(const IndexParams& p, int b, int first_page, int count, int32_t* pages) {
  for (int i = threadIdx.x; i < count; i += blockDim.x) {
    int pid = p.page_table[(size_t)b * p.max_pages + first_page + i];
    if (pid < 0 || pid >= p.num_pages) {
      flag_error(p.err, LISA_DEVERR_PAGE_ID);
      pid = 0;
    }
    pages[i] = pid;
  }
}

// Block-wide: among the nb bins of gh (counts of candidate keys per digit, high digit = high key),
// find the digit d holding the need-th largest candidate.  Writes d and the rank of that key within
// the digit (1-based) to out[0], out[1].  Ends with a barrier.
__device__ void find_digit(const uint32_t* gh, int nb, uint32_t need, uint32_t* warp_tot, uint32_t* out) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, nwarps = blockDim.x >> 5;
  const int per = nb / blockDim.x;
  uint32_t v = 0;
  for (int i = 0; i < per; ++i) v += gh[t * per + i];
  uint32_t x = v;  // inclusive suffix sum within the warp (lanes >= this lane)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) warp_tot[warp] = x;
  __syncthreads();
  uint32_t above = 0;
  for (int w = warp + 1; w < nwarps; ++w) above += warp_tot[w];
  const uint32_t incl = x + above, excl = incl - v;
  if (excl < need && need <= incl) {
    uint32_t acc = excl;
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t c = gh[t * per + i];
      if (acc + c >= need) {
        out[0] = (uint32_t)(t * per + i);
        out[1] = need - acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

struct SelectSmem {
  uint32_t hist[3][kBins];
  uint32_t ghist[kBins];
  float qbar[128];
  float u[32];
  uint32_t warp_tot[32];
  uint32_t digit[2];
  uint32_t cnt[2];     // this CTA's (#keys > K, #keys == K), read by the other CTAs of the cluster
  uint32_t wgt[32], weq[32];
};

}  // namespace

size_t select_smem_bytes(int chunk_max, int ps) {
  const int pages = (chunk_max + ps - 1) / ps;
  return sizeof(SelectSmem) + (size_t)chunk_max * 4 + (size_t)pages * 4;
}

// One cluster of kClusterSize CTAs per (b, KV head).  FROM_SCORES: keys come from p.scores
// (lisa_topm_select); otherwise the CTA computes them (lisa_index_topm / lisa_fused_decode).
template <int R, bool FP8, bool FROM_SCORES>
__global__ void __cluster_dims__(kClusterSize, 1, 1) __launch_bounds__(kIndexThreads, 2)
    lisa_index_select_kernel(IndexParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(SelectSmem));
  int32_t* pages = reinterpret_cast<int32_t*>(keys + p.chunk_max);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int n = load_seq_len(p, b);
  int32_t* idx_out = p.idx + ((size_t)b * p.Hkv + h) * p.M;

  if (n <= p.M) {  // every position is kept; the whole cluster takes this branch together
    for (int i = rank * blockDim.x + tid; i < p.M; i += kClusterSize * blockDim.x) idx_out[i] = i < n ? i : -1;
    if (rank == 0 && tid == 0) p.count[(size_t)b * p.Hkv + h] = n;
    return;
  }

  // This CTA's page-aligned slice of the context.
  const int chunk = ((((n + kClusterSize - 1) / kClusterSize) + p.ps - 1) >> p.log2ps) << p.log2ps;
  const int t_begin = rank * chunk;
  const int nrows = max(0, min(n, t_begin + chunk) - t_begin);

  for (int i = tid; i < 3 * kBins; i += blockDim.x) (&sm.hist[0][0])[i] = 0u;
  if constexpr (!FROM_SCORES) {
    load_pages(p, b, t_begin >> p.log2ps, (nrows + p.ps - 1) >> p.log2ps, pages);
    compute_projected_query(p, b, h, sm.qbar, sm.u);  // ends with a barrier
    const float scale = p.kproj_scale[h];
    stream_scores<R, FP8, 8>(p, h, t_begin, nrows, pages, sm.u, scale, [&](int lr, float s) {
      const uint32_t k = score_key(s);
      keys[lr] = k;
      atomicAdd(&sm.hist[0][k >> 21], 1u);
    });
  } else {
    __syncthreads();
    const float* src = p.scores + ((size_t)b * p.Hkv + h) * p.max_seq_len + t_begin;
    for (int lr = tid; lr < nrows; lr += blockDim.x) {
      const uint32_t k = score_key(src[lr]);
      keys[lr] = k;
      atomicAdd(&sm.hist[0][k >> 21], 1u);
    }
  }

  // Radix select of the M-th largest key over the cluster: digits of 11, 11 and 10 bits.
  const int shift[3] = {21, 10, 0};
  const int width[3] = {11, 11, 10};
  uint32_t prefix = 0, need = (uint32_t)p.M;
  for (int pass = 0; pass < 3; ++pass) {
    uint32_t* hp = sm.hist[pass];
    if (pass > 0) {
      const int hs = shift[pass - 1];
      const uint32_t mask = (1u << width[pass]) - 1u;
      for (int lr = tid; lr < nrows; lr += blockDim.x) {
        const uint32_t k = keys[lr];
        if ((k >> hs) == prefix) atomicAdd(&hp[(k >> shift[pass]) & mask], 1u);
      }
    }
    cluster.sync();  // every CTA's histogram of this pass is complete
    const int nb = 1 << width[pass];
    for (int i = tid; i < nb; i += blockDim.x) {
      uint32_t s = 0;
#pragma unroll
      for (int r = 0; r < kClusterSize; ++r) s += cluster.map_shared_rank(hp, r)[i];
      sm.ghist[i] = s;
    }
    __syncthreads();
    find_digit(sm.ghist, nb, need, sm.warp_tot, sm.digit);
    prefix = (prefix << width[pass]) | sm.digit[0];
    need = sm.digit[1];
  }
  const uint32_t K = prefix;      // the M-th largest key of (b, h)
  const uint32_t tie_take = need;  // keys equal to K to keep, lowest positions first

  // Count per warp over contiguous row ranges, then place this CTA's rows after the lower ranks'.
  const int wlen = (((nrows + nwarps - 1) / nwarps) + 31) & ~31;
  const int w0 = warp * wlen, w1 = min(nrows, w0 + wlen);
  uint32_t gt = 0, eq = 0;
  for (int lr = w0 + lane; lr < w1; lr += 32) {
    const uint32_t k = keys[lr];
    gt += (k > K);
    eq += (k == K);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    sm.wgt[warp] = gt;
    sm.weq[warp] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t a = 0, e = 0;
    for (int w = 0; w < nwarps; ++w) {
      a += sm.wgt[w];
      e += sm.weq[w];
    }
    sm.cnt[0] = a;
    sm.cnt[1] = e;
  }
  cluster.sync();
  uint32_t ties_before = 0, out_before = 0;
  for (int r = 0; r < rank; ++r) {
    const uint32_t* rc = cluster.map_shared_rank(sm.cnt, r);
    const uint32_t take = min(rc[1], tie_take > ties_before ? tie_take - ties_before : 0u);
    out_before += rc[0] + take;
    ties_before += rc[1];
  }
  for (int w = 0; w < warp; ++w) {
    const uint32_t take = min(sm.weq[w], tie_take > ties_before ? tie_take - ties_before : 0u);
    out_before += sm.wgt[w] + take;
    ties_before += sm.weq[w];
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = w0; base < w1; base += 32) {
    const int lr = base + lane;
    const bool valid = lr < w1;
    const uint32_t k = valid ? keys[lr] : 0u;
    const bool is_gt = valid && k > K;
    const bool is_eq = valid && k == K;
    const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t tie_rank = ties_before + __popc(beq & lt_mask);
    const bool take = is_gt || (is_eq && tie_rank < tie_take);
    const uint32_t bsel = __ballot_sync(0xffffffffu, take);
    const uint32_t slot = out_before + __popc(bsel & lt_mask);
    if (take && slot < (uint32_t)p.M) idx_out[slot] = t_begin + lr;
    ties_before += __popc(beq);
    out_before += __popc(bsel);
  }
  if (rank == 0 && tid == 0) p.count[(size_t)b * p.Hkv + h] = p.M;
  cluster.sync();  // no CTA leaves while another may still read its counters
}

// Scores only: one CTA per (kScoreChunk positions, KV head, sequence); writes fp32 scores.
template <int R, bool FP8>
__global__ void __launch_bounds__(kIndexThreads) lisa_score_kernel(IndexParams p) {
  __shared__ float qbar[128];
  __shared__ float u[32];
  __shared__ int32_t pages[kScoreChunk / 16];
  const int h = blockIdx.y, b = blockIdx.z;
  const int n = load_seq_len(p, b);
  const int t_begin = blockIdx.x * kScoreChunk;
  if (t_begin >= n) return;
  const int nrows = min(n - t_begin, kScoreChunk);
  load_pages(p, b, t_begin >> p.log2ps, (nrows + p.ps - 1) >> p.log2ps, pages);
  compute_projected_query(p, b, h, qbar, u);
  float* dst = p.scores + ((size_t)b * p.Hkv + h) * p.max_seq_len + t_begin;
  stream_scores<R, FP8, 8>(p, h, t_begin, nrows, pages, u, p.kproj_scale[h],
                           [&](int lr, float s) { dst[lr] = s; });
}

// ---------------------------------------------------------------------------------------------
// Host-side launchers (called from the C ABI layer after argument checks)
// ---------------------------------------------------------------------------------------------

template <typename K>
static cudaError_t set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int R, bool FP8>
static cudaError_t launch_select_t(const IndexParams& p, bool from_scores, cudaStream_t stream) {
  const size_t smem = select_smem_bytes(p.chunk_max, p.ps);
  dim3 grid(kClusterSize, p.Hkv, p.B);
  if (from_scores) {
    auto k = lisa_index_select_kernel<R, FP8, true>;
    cudaError_t e = set_smem(k, smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kIndexThreads, smem, stream>>>(p);
  } else {
    auto k = lisa_index_select_kernel<R, FP8, false>;
    cudaError_t e = set_smem(k, smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kIndexThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_index_select(const IndexParams& p, bool from_scores, cudaStream_t stream) {
  if (from_scores) return launch_select_t<32, true>(p, true, stream);  // geometry unused when reading scores
  if (p.kproj_fp8) {
    return p.r == 16 ? launch_select_t<16, true>(p, false, stream) : launch_select_t<32, true>(p, false, stream);
  }
  return p.r == 16 ? launch_select_t<16, false>(p, false, stream) : launch_select_t<32, false>(p, false, stream);
}

template <int R, bool FP8>
static cudaError_t launch_score_t(const IndexParams& p, cudaStream_t stream) {
  dim3 grid((p.max_seq_len + kScoreChunk - 1) / kScoreChunk, p.Hkv, p.B);
  lisa_score_kernel<R, FP8><<<grid, kIndexThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_index_score(const IndexParams& p, cudaStream_t stream) {
  if (p.kproj_fp8) return p.r == 16 ? launch_score_t<16, true>(p, stream) : launch_score_t<32, true>(p, stream);
  return p.r == 16 ? launch_score_t<16, false>(p, stream) : launch_score_t<32, false>(p, stream);
}

}  // namespace lisa
