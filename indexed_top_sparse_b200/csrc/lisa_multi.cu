// Multi-query indexer scores (lisa_index_score_multi), sm_100a.
//
// What is computed (JSSA write-up, section "Как JSSA сохраняет порядок токенов", decoding paragraph,
// applied to each of T query tokens of a sequence): token j of sequence b averages its G queries of
// KV head h, projects the mean with the head's r x d basis, and scores every position it may see,
// t <= n_b - T + j, against the FP8 projected-key cache:
//   s[b][j][h][t] = scale_h * < P_h qbar_{b,j,h}, c_t >.
//
// Design on B200: two kernels chained by programmatic dependent launch.
//  * lisa_multi_project_kernel forms the T projected queries of each (b, KV head) once, into the
//    workspace.
//  * lisa_score_multi_kernel streams the projected keys exactly like the single-query score stream:
//    each warp owns a contiguous quarter of a 4096-position chunk and moves it through a private
//    4-stage cp.async ring in shared memory, with no CTA-wide barrier in the loop.  Its first copies
//    are issued before it waits for the projected queries.  Every 16-row tile is one tensor-core
//    contraction [16 x r] . [r x 2T]: column pair (2j, 2j + 1) holds u_j as 2^E_j (u_hi + u_lo) in
//    f16, E4M3 -> f16 is exact and the products accumulate in fp32, so each score agrees with an
//    fp32 dot product to rounding.  Lane (g, t) of a warp receives the scores of query 4 nt + t for
//    rows g and g + 8 of the tile, so no column of the contraction is wasted.

#include "lisa_common.cuh"
#include "lisa_kernels.h"

namespace lisa {

namespace {

constexpr int kMultiChunk = 4096;       // positions per scoring CTA
constexpr int kMultiThreads = 128;      // 4 warps, 1024 positions each
constexpr int kMultiStageBytes = 2048;  // projected-key bytes per warp pipeline stage
constexpr int kMultiStages = 4;         // stages in each warp's shared-memory ring
constexpr int kMultiCtasPerSm = 6;
constexpr int kMultiTopmStage = 64;    // candidates a warp stages per query between flushes

// uq[b][j][h][0..r): the projected mean query of token j (fp32, 32 slots per row).
__global__ void __launch_bounds__(kMultiThreads) lisa_multi_project_kernel(MultiParams p) {
  __shared__ float qbar[kMultiMaxT][128];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = p.T, G = p.Hq / p.Hkv, d = p.d, R = p.r;
  pdl_wait();  // the queries may come from earlier work of the stream
  pdl_trigger();
  for (int e = tid; e < T * d; e += blockDim.x) {
    const int j = e / d, k = e % d;
    const __nv_bfloat16* qg = p.q + (((size_t)b * T + j) * p.Hq + (size_t)h * G) * d + k;
    float acc = 0.f;
    for (int gg = 0; gg < G; ++gg) acc += __bfloat162float(qg[(size_t)gg * d]);
    qbar[j][k] = acc / (float)G;
  }
  __syncthreads();
  // Warp w forms rows i = w, w + 4, ... of u_j = P_h qbar_j for every token: the rows of P are
  // read coalesced (lane k holds dimensions k, k + 32, ...), then one warp sum per (i, j).
  constexpr int kRowsPerWarp = 32 / (kMultiThreads / 32);
  constexpr int kPerLane = 128 / 32;
  float pr[kRowsPerWarp][kPerLane];
#pragma unroll
  for (int m = 0; m < kRowsPerWarp; ++m) {
    const int i = warp + 4 * m;
#pragma unroll
    for (int c = 0; c < kPerLane; ++c) {
      const int k = lane + 32 * c;
      pr[m][c] = (i < R && k < d) ? __ldg(p.P + ((size_t)h * R + i) * d + k) : 0.f;
    }
  }
#pragma unroll
  for (int m = 0; m < kRowsPerWarp; ++m) {
    const int i = warp + 4 * m;
    if (i >= R) break;
    for (int j = 0; j < T; ++j) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < kPerLane; ++c) {
        const int k = lane + 32 * c;
        if (k < d) a = fmaf(pr[m][c], qbar[j][k], a);
      }
      a = warp_sum(a);
      if (lane == 0) p.uq[(((size_t)b * T + j) * p.Hkv + h) * 32 + i] = a;
    }
  }
}

// TOPM = false: the scores of every visible (token, position) are written.  TOPM = true: nothing is
// written but the positions whose key reaches their token's sampled threshold, appended to that
// token's candidate buffer (staged per warp and token in shared memory, behind the ring).
template <int R, int NT, bool TOPM>
__global__ void __launch_bounds__(kMultiThreads, TOPM ? kMultiCtasPerSm - 1 : kMultiCtasPerSm) lisa_score_multi_kernel(MultiParams p) {
  extern __shared__ __align__(128) uint8_t ring[];   // [warp][kMultiStages][kMultiStageBytes], then the stage
  __shared__ const uint8_t* pbase[kMultiChunk / 16];  // global address of each page block of the chunk
  __shared__ float ush[kMultiMaxT][32];
  constexpr int RB = R;                        // FP8: one byte per dimension
  constexpr int CPR = RB / 16;                 // 16-byte chunks per row
  constexpr int RPS = kMultiStageBytes / RB;   // rows per stage
  constexpr int MT = RPS / 16;                 // 16-row tiles per stage
  constexpr int KS = R / 16;                   // k-steps of 16 dimensions
  constexpr int WROWS = kMultiChunk / (kMultiThreads / 32);
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int T = p.T;
  int n = p.seq_lens[b];
  if (n < 0 || n > p.max_seq_len) {
    if (tid == 0) flag_error(p.err, LISA_DEVERR_SEQ_LEN);
    n = n < 0 ? 0 : p.max_seq_len;
  }
  const int t_begin = blockIdx.x * kMultiChunk;
  // Every kernel of the launch waits for the projected queries, also CTAs with nothing to score.
  if (t_begin >= n) {
    pdl_wait();
    pdl_trigger();
    return;
  }
  const int nrows = min(n - t_begin, kMultiChunk);
  {
    const int npg = (nrows + p.ps - 1) >> p.log2ps;
    const uint8_t* base = reinterpret_cast<const uint8_t*>(p.kproj);
    for (int i = tid; i < npg; i += blockDim.x) {
      int pid = p.page_table[(size_t)b * p.max_pages + (t_begin >> p.log2ps) + i];
      if (pid < 0 || pid >= p.num_pages) {
        flag_error(p.err, LISA_DEVERR_PAGE_ID);
        pid = 0;
      }
      pbase[i] = base + ((((size_t)pid * p.Hkv + h) << p.log2ps) * RB);
    }
  }
  __syncthreads();

  uint8_t* wring = ring + warp * (kMultiStages * kMultiStageBytes);
  const int w0 = warp * WROWS;                        // first row of this warp (chunk-relative)
  const int wrows = max(0, min(nrows - w0, WROWS));   // rows this warp scores
  const int nstages = (wrows + RPS - 1) / RPS;
  // Rows are stored unswizzled: lane (g, t) reads bytes [t r/4, (t+1) r/4) of rows g and g + 8 of a
  // tile, which spreads a warp's reads over all banks.
  auto issue = [&](int stage) {
    if (stage >= nstages) return;
    uint8_t* dst = wring + (stage % kMultiStages) * kMultiStageBytes;
    if (p.ps >= RPS) {
      // the stage's rows are contiguous inside one page block: one base address
      const int lr0 = w0 + stage * RPS;
      const uint8_t* src = pbase[lr0 >> p.log2ps] + (lr0 & (p.ps - 1)) * RB;
      const int vbytes = min(RPS, wrows - stage * RPS) * RB;
#pragma unroll
      for (int k = 0; k < kMultiStageBytes / 512; ++k) {
        const int off = (lane + 32 * k) * 16;
        cp_async_16(smem_u32(dst + off), src + (off < vbytes ? off : 0), off < vbytes ? 16u : 0u);
      }
      return;
    }
#pragma unroll
    for (int k = 0; k < kMultiStageBytes / 512; ++k) {
      const int c = lane + 32 * k;  // 16-byte chunk of the stage
      const int r = c / CPR, part = c % CPR;
      const int lr = w0 + stage * RPS + r;
      const bool valid = lr < w0 + wrows;
      const int vr = valid ? lr : w0;
      const uint8_t* src = pbase[vr >> p.log2ps] + (vr & (p.ps - 1)) * RB + part * 16;
      cp_async_16(smem_u32(dst + c * 16), src, valid ? 16u : 0u);
    }
  };
#pragma unroll
  for (int st = 0; st < kMultiStages - 1; ++st) {
    issue(st);
    cp_async_commit();
  }
  // The projected keys are inputs of the call: their first stages are in flight before the
  // projected queries of the previous kernel are awaited.
  pdl_wait();
  pdl_trigger();
  for (int e = tid; e < T * R; e += blockDim.x) {
    const int j = e / R, i = e % R;
    ush[j][i] = p.uq[(((size_t)b * T + j) * p.Hkv + h) * 32 + i];
  }
  __syncthreads();
  // B fragments: lane (g, t) holds column g of each n-tile, i.e. part g & 1 of query (8 nt + g) / 2.
  uint32_t bf[NT][KS][2];
  float fac[NT];            // output scale of query 4 nt + t
  float* __restrict__ srow[NT];  // scores of that query from this warp's first row on
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int col = 8 * nt + g, j = col >> 1;
    float mx = 0.f;
    if (j < T)
      for (int i = 0; i < R; ++i) mx = fmaxf(mx, fabsf(ush[j][i]));
    const int E = mx > 0.f ? ilogbf(mx) - 13 : 0;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int e0 = (R / 4) * t4 + 4 * ks + 2 * jj;  // dimensions e0, e0 + 1
        __half v[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float x = j < T ? ldexpf(ush[j][e0 + q], -E) : 0.f;
          const __half hi = __float2half_rn(x);
          v[q] = (col & 1) ? __float2half_rn(x - __half2float(hi)) : hi;
        }
        bf[nt][ks][jj] = (uint32_t)__half_as_ushort(v[0]) | ((uint32_t)__half_as_ushort(v[1]) << 16);
      }
    }
    const int jo = 4 * nt + t4;
    float mo = 0.f;
    if (jo < T)
      for (int i = 0; i < R; ++i) mo = fmaxf(mo, fabsf(ush[jo][i]));
    const int Eo = mo > 0.f ? ilogbf(mo) - 13 : 0;
    fac[nt] = p.kproj_scale[h] * ldexpf(1.f, Eo);
    if constexpr (!TOPM)
      srow[nt] = p.scores + (((size_t)b * T + min(jo, T - 1)) * p.Hkv + h) * p.max_seq_len + t_begin + w0;
  }
  // lim[nt]: the last warp-relative row query 4 nt + t sees (negative: none).  A token whose context
  // is at most M positions long has its full set from the sample kernel and takes no candidates.
  int lim[NT];
  uint32_t tau[NT] = {};        // candidate threshold key of query 4 nt + t
  uint2* cdst[NT] = {};         // its candidate buffer
  uint32_t* ccnt[NT] = {};      // and count
  uint32_t wn[NT] = {};         // candidates of that query staged by this warp (same in its 8 lanes)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int jo = 4 * nt + t4;
    bool live = jo < T;
    if constexpr (TOPM) live = live && n - T + jo + 1 > p.M;
    lim[nt] = live ? min(n - T + jo - t_begin - w0, wrows - 1) : -1;
    if constexpr (TOPM) {
      const size_t pair = ((size_t)b * T + min(jo, T - 1)) * p.Hkv + h;
      tau[nt] = live ? p.tau[pair] : 0xffffffffu;
      cdst[nt] = reinterpret_cast<uint2*>(p.cand) + pair * (size_t)p.cap;
      ccnt[nt] = p.ccount + pair;
      wn[nt] = 0u;
    }
  }
  // Per-(warp, query) stages of kMultiTopmStage (key, position) entries, behind the ring.
  uint2* wstage = reinterpret_cast<uint2*>(ring + (kMultiThreads / 32) * kMultiStages * kMultiStageBytes) +
                  (size_t)warp * (4 * NT) * kMultiTopmStage;
  // Appends the staged candidates of the four queries of n-tile nt (lane group t of the warp owns
  // query 4 nt + t) to their buffers, one global atomic per query; entries past the capacity are
  // dropped and the count then sends that query to the exact path.
  auto flush = [&](int nt) {
    __syncwarp();
    const uint32_t cnt = wn[nt];
    uint32_t base = 0u;
    if (g == 0 && cnt > 0u) base = atomicAdd(ccnt[nt], cnt);
    base = __shfl_sync(0xffffffffu, base, t4);
    const uint2* st_q = wstage + (size_t)(4 * nt + t4) * kMultiTopmStage;
    for (uint32_t i = g; i < cnt; i += 8u) {
      const uint32_t slot = base + i;
      if (slot < (uint32_t)p.cap) cdst[nt][slot] = st_q[i];
    }
    wn[nt] = 0u;
    __syncwarp();
  };

  for (int st = 0; st < nstages; ++st) {
    issue(st + kMultiStages - 1);
    cp_async_commit();
    cp_async_wait<kMultiStages - 1>();
    __syncwarp();
    const uint8_t* src = wring + (st % kMultiStages) * kMultiStageBytes;
    // Tiles in groups of four (64 rows); with TOPM the group's candidates are staged after it.
#pragma unroll
    for (int mg = 0; mg < MT; mg += 4) {
    uint32_t keys[NT][8];
    uint32_t mask[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mask[nt] = 0u;
#pragma unroll
    for (int mt = mg; mt < mg + 4; ++mt) {
      const uint8_t* r0 = src + (mt * 16 + g) * RB + (R / 4) * t4;
      const uint8_t* r1 = r0 + 8 * RB;
      uint32_t x0[KS], x1[KS];
      if constexpr (R == 32) {
        const uint2 v0 = *reinterpret_cast<const uint2*>(r0);
        const uint2 v1 = *reinterpret_cast<const uint2*>(r1);
        x0[0] = v0.x;
        x0[1] = v0.y;
        x1[0] = v1.x;
        x1[1] = v1.y;
      } else {
        static_assert(R == 16, "FP8 projected keys have r = 16 or 32");
        x0[0] = *reinterpret_cast<const uint32_t*>(r0);
        x1[0] = *reinterpret_cast<const uint32_t*>(r1);
      }
      float dacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) dacc[nt][0] = dacc[nt][1] = dacc[nt][2] = dacc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_f16x2(x0[ks], a0, a2);
        e4m3x4_to_f16x2(x1[ks], a1, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16_16816(dacc[nt], a0, a1, a2, a3, bf[nt][ks][0], bf[nt][ks][1]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int rr = st * RPS + mt * 16 + g;
        const float s0 = fac[nt] * (dacc[nt][0] + dacc[nt][1]), s1 = fac[nt] * (dacc[nt][2] + dacc[nt][3]);
        if constexpr (TOPM) {
          const int k = 2 * (mt - mg);
          keys[nt][k] = score_key(s0);
          keys[nt][k + 1] = score_key(s1);
          if (rr <= lim[nt] && keys[nt][k] >= tau[nt]) mask[nt] |= 1u << k;
          if (rr + 8 <= lim[nt] && keys[nt][k + 1] >= tau[nt]) mask[nt] |= 2u << k;
        } else {
          if (rr <= lim[nt]) srow[nt][rr] = s0;
          if (rr + 8 <= lim[nt]) srow[nt][rr + 8] = s1;
        }
      }
    }
    if constexpr (TOPM) {
      // Slots from a prefix sum over the 8 lanes that hold the same query (lanes t, t + 4, ...).
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t c = (uint32_t)__popc(mask[nt]);
        uint32_t incl = c;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, incl, 28 + t4);
        if (__any_sync(0xffffffffu, wn[nt] + tot > (uint32_t)kMultiTopmStage)) flush(nt);
        uint32_t slot = wn[nt] + incl - c;
        uint2* st_q = wstage + (size_t)(4 * nt + t4) * kMultiTopmStage;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if ((mask[nt] >> k) & 1u) {
            const int row = st * RPS + (mg + (k >> 1)) * 16 + g + 8 * (k & 1);
            st_q[slot++] = make_uint2(keys[nt][k], (uint32_t)(t_begin + w0 + row));
          }
        }
        wn[nt] += tot;
      }
    }
    }
    __syncwarp();  // the slot is refilled by a later stage
  }
  cp_async_wait<0>();
  if constexpr (TOPM) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) flush(nt);
  }
}

template <int R, int NT, bool TOPM>
cudaError_t launch_score_multi_t(const MultiParams& p, cudaStream_t stream) {
  size_t smem = (size_t)(kMultiThreads / 32) * kMultiStages * kMultiStageBytes;
  if (TOPM) smem += (size_t)(kMultiThreads / 32) * (4 * NT) * kMultiTopmStage * sizeof(uint2);
  const dim3 grid((p.max_seq_len + kMultiChunk - 1) / kMultiChunk, p.Hkv, p.B);
  auto k = lisa_score_multi_kernel<R, NT, TOPM>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = prefer_max_smem(k);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, grid, dim3(kMultiThreads), smem, stream, p);
}

}  // namespace

cudaError_t launch_index_score_multi(const MultiParams& p, cudaStream_t stream) {
  cudaError_t e = launch_pdl(lisa_multi_project_kernel, dim3(p.Hkv, p.B), dim3(kMultiThreads), 0, stream, p);
  if (e != cudaSuccess) return e;
  const bool two = 2 * p.T > 8;  // 2T columns: one or two n-tiles of 8
  if (p.r == 16)
    return two ? launch_score_multi_t<16, 2, false>(p, stream) : launch_score_multi_t<16, 1, false>(p, stream);
  return two ? launch_score_multi_t<32, 2, false>(p, stream) : launch_score_multi_t<32, 1, false>(p, stream);
}

cudaError_t launch_index_topm_multi_stream(const MultiParams& p, cudaStream_t stream) {
  const bool two = 2 * p.T > 8;
  if (p.r == 16)
    return two ? launch_score_multi_t<16, 2, true>(p, stream) : launch_score_multi_t<16, 1, true>(p, stream);
  return two ? launch_score_multi_t<32, 2, true>(p, stream) : launch_score_multi_t<32, 1, true>(p, stream);
}

}  // namespace lisa
