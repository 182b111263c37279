// Basis calibration (sm_100a): the one-time step that produces the projection P of each KV head.
//
// What is computed (JSSA write-up, section "Как JSSA сохраняет порядок токенов": per head and layer
// the method accumulates query and key statistics once and takes the basis from eigenvectors of a
// matrix, the subspace being meant to preserve query-key scores).  Reading of the unnamed matrix:
// with Q = E[q q^T] over averaged group queries and K = E[k k^T] over keys, the expected product of
// the true score and the score through the projector P^T P is tr(P^T P K Q), maximised by the top-r
// eigenvectors of C = (Q K + K Q) / 2.  P's rows are those eigenvectors, largest eigenvalue first,
// each signed so that its entry of largest magnitude is positive.
//
// Kernels: second moments of the samples (fp32 accumulation, 64x64 output tiles), then one CTA per
// KV head that forms C in shared memory and diagonalises it with the parallel cyclic Jacobi method
// (round-robin pairing: d/2 disjoint rotations per round, d-1 rounds per sweep, at most kMaxSweeps
// sweeps; pairs already diagonal to fp32 resolution are skipped and a sweep without rotations ends
// it), then re-orthonormalises the r chosen eigenvectors (modified Gram-Schmidt).  Off the decode
// path.

#include "lisa_common.cuh"
#include "lisa_kernels.h"

namespace lisa {

namespace {

constexpr int kMomentTile = 64;
constexpr int kMomentThreads = 256;
constexpr int kJacobiThreads = 512;
constexpr int kMaxD = 128;
constexpr int kPitch = kMaxD + 1;  // shared-memory row pitch (floats), breaks bank conflicts
constexpr int kMaxSweeps = 16;

// M = X^T X / N for X = samples of one head ([N][d] bf16); blockIdx = (tile, head, which): which 0
// reads the queries into Q, 1 the keys into K.  Each thread owns a 4x4 block of a 64x64 tile.
__global__ void __launch_bounds__(kMomentThreads) lisa_moment_kernel(CalibParams p) {
  __shared__ float xi[32][kMomentTile + 1];
  __shared__ float xj[32][kMomentTile + 1];
  const int which = blockIdx.z, h = blockIdx.y;
  const int tiles = p.d / kMomentTile;
  const int ti = blockIdx.x / tiles, tj = blockIdx.x % tiles;
  const int N = which == 0 ? p.nq : p.nk;
  const __nv_bfloat16* X = (which == 0 ? p.q : p.k) + (size_t)h * N * p.d;
  float* out = (which == 0 ? p.Q : p.K) + (size_t)h * p.d * p.d;
  const int tid = threadIdx.x, ri = (tid / 16) * 4, rj = (tid % 16) * 4;
  float acc[4][4] = {};
  for (int n0 = 0; n0 < N; n0 += 32) {
    for (int e = tid; e < 32 * kMomentTile; e += blockDim.x) {
      const int s = e / kMomentTile, c = e % kMomentTile, n = n0 + s;
      xi[s][c] = n < N ? __bfloat162float(X[(size_t)n * p.d + ti * kMomentTile + c]) : 0.f;
      xj[s][c] = n < N ? __bfloat162float(X[(size_t)n * p.d + tj * kMomentTile + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int s = 0; s < 32; ++s) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(xi[s][ri + a], xj[s][rj + c], acc[a][c]);
    }
    __syncthreads();
  }
  const float inv = 1.f / (float)N;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      out[(size_t)(ti * kMomentTile + ri + a) * p.d + tj * kMomentTile + rj + c] = acc[a][c] * inv;
}

// One CTA per KV head: C = (Q K + K Q) / 2, Jacobi eigen-decomposition, top-r eigenvectors -> P.
__global__ void __launch_bounds__(kJacobiThreads) lisa_jacobi_kernel(CalibParams p) {
  extern __shared__ float jsm[];
  float* A = jsm;                  // [d][kPitch]
  float* V = jsm + kMaxD * kPitch;  // [d][kPitch], columns are eigenvectors
  __shared__ float rc[kMaxD / 2], rs[kMaxD / 2];
  __shared__ int rp[kMaxD / 2], rq[kMaxD / 2];
  __shared__ float evals[kMaxD];
  __shared__ int order[kMaxD];
  __shared__ int s_rot;
  const int h = blockIdx.x, tid = threadIdx.x, d = p.d, half = p.d / 2;
  const float* Q = p.Q + (size_t)h * d * d;
  const float* K = p.K + (size_t)h * d * d;
  for (int e = tid; e < d * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    float a = 0.f;
    for (int l = 0; l < d; ++l) a = fmaf(Q[i * d + l], K[l * d + j], fmaf(K[i * d + l], Q[l * d + j], a));
    A[i * kPitch + j] = 0.5f * a;
    V[i * kPitch + j] = i == j ? 1.f : 0.f;
  }
  __syncthreads();
  // symmetrise exactly (the two products are equal only up to rounding)
  for (int e = tid; e < d * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    if (i < j) {
      const float m = 0.5f * (A[i * kPitch + j] + A[j * kPitch + i]);
      A[i * kPitch + j] = m;
      A[j * kPitch + i] = m;
    }
  }
  __syncthreads();
  // Threshold Jacobi: a pair whose off-diagonal entry is below fp32 resolution of its diagonal pair
  // is not rotated (rotating it would only add rounding noise); a sweep without rotations ends it.
  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    if (tid == 0) s_rot = 0;
    __syncthreads();
    for (int round = 0; round < d - 1; ++round) {
      if (tid < half) {  // circle method: position 0 fixed, the others rotate by `round`
        auto player = [&](int k) { return k == 0 ? 0 : 1 + (k - 1 + round) % (d - 1); };
        int a = player(tid), b = player(d - 1 - tid);
        if (a > b) { const int t = a; a = b; b = t; }
        const float app = A[a * kPitch + a], aqq = A[b * kPitch + b], apq = A[a * kPitch + b];
        float c = 1.f, s = 0.f;
        if (fabsf(apq) > 1e-30f && fabsf(apq) > 1e-7f * sqrtf(fabsf(app * aqq))) {
          const float theta = (aqq - app) / (2.f * apq);
          const float t = copysignf(1.f, theta) / (fabsf(theta) + sqrtf(theta * theta + 1.f));
          c = rsqrtf(t * t + 1.f);
          s = t * c;
          atomicAdd(&s_rot, 1);
        }
        rp[tid] = a; rq[tid] = b; rc[tid] = c; rs[tid] = s;
      }
      __syncthreads();
      for (int e = tid; e < half * d; e += blockDim.x) {  // rows a, b of A
        const int pr = e / d, k = e % d, a = rp[pr], b = rq[pr];
        const float c = rc[pr], s = rs[pr], x = A[a * kPitch + k], y = A[b * kPitch + k];
        A[a * kPitch + k] = c * x - s * y;
        A[b * kPitch + k] = s * x + c * y;
      }
      __syncthreads();
      for (int e = tid; e < half * d; e += blockDim.x) {  // columns a, b of A and of V
        const int pr = e / d, k = e % d, a = rp[pr], b = rq[pr];
        const float c = rc[pr], s = rs[pr];
        const float x = A[k * kPitch + a], y = A[k * kPitch + b];
        A[k * kPitch + a] = c * x - s * y;
        A[k * kPitch + b] = s * x + c * y;
        const float u = V[k * kPitch + a], w = V[k * kPitch + b];
        V[k * kPitch + a] = c * u - s * w;
        V[k * kPitch + b] = s * u + c * w;
      }
      __syncthreads();
    }
    const int rotated = s_rot;
    __syncthreads();  // every thread has read the count before thread 0 clears it again
    if (rotated == 0) break;
  }
  // eigenvalues A[i][i]; order them (largest first, ties to the lower index)
  if (tid < d) evals[tid] = A[tid * kPitch + tid];
  __syncthreads();
  if (tid < d) {
    const float wi = evals[tid];
    int rank = 0;
    for (int j = 0; j < d; ++j) rank += (evals[j] > wi) || (evals[j] == wi && j < tid);
    order[rank] = tid;
  }
  __syncthreads();
  // the selected eigenvectors as rows (A's storage is free now), then modified Gram-Schmidt by one
  // warp to restore the orthonormality that fp32 rotations wear down
  for (int e = tid; e < p.r * d; e += blockDim.x) {
    const int i = e / d, k = e % d;
    A[i * kPitch + k] = V[k * kPitch + order[i]];
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    for (int i = 0; i < p.r; ++i) {
      float* xi = A + i * kPitch;
      for (int j = 0; j < i; ++j) {
        const float* xj = A + j * kPitch;
        float dot = 0.f;
        for (int k = lane; k < d; k += 32) dot = fmaf(xi[k], xj[k], dot);
        dot = warp_sum(dot);
        for (int k = lane; k < d; k += 32) xi[k] = fmaf(-dot, xj[k], xi[k]);
        __syncwarp();
      }
      float nn = 0.f;
      for (int k = lane; k < d; k += 32) nn = fmaf(xi[k], xi[k], nn);
      const float inv = rsqrtf(warp_sum(nn));
      for (int k = lane; k < d; k += 32) xi[k] *= inv;
      __syncwarp();
    }
  }
  __syncthreads();
  // row i of P, signed so that its largest-magnitude entry is positive
  for (int i = warp; i < p.r; i += blockDim.x >> 5) {
    const float* xi = A + i * kPitch;
    float best = -1.f;
    int arg = 0;
    for (int k = lane; k < d; k += 32) {
      const float v = fabsf(xi[k]);
      if (v > best) { best = v; arg = k; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (ob > best || (ob == best && oa < arg)) { best = ob; arg = oa; }
    }
    const float sign = xi[arg] < 0.f ? -1.f : 1.f;
    for (int k = lane; k < d; k += 32) p.P[((size_t)h * p.r + i) * d + k] = sign * xi[k];
    if (lane == 0 && p.eigvals != nullptr) p.eigvals[(size_t)h * p.r + i] = evals[order[i]];
  }
}

}  // namespace

size_t calib_jacobi_smem_bytes() { return (size_t)2 * kMaxD * kPitch * sizeof(float); }

cudaError_t launch_calibrate(const CalibParams& p, cudaStream_t stream) {
  const int tiles = p.d / kMomentTile;
  lisa_moment_kernel<<<dim3(tiles * tiles, p.Hkv, 2), kMomentThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = calib_jacobi_smem_bytes();
  e = cudaFuncSetAttribute(lisa_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  lisa_jacobi_kernel<<<p.Hkv, kJacobiThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace lisa
