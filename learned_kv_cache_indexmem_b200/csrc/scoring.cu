// scoring.cu -- indexer scores pooled per key by a running max over the
// causal queries, without materialising the score matrix.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.A Function (a dense query-to-key score matrix A, A[s,t] the
// importance of key t for query s) and Training (per-key importance pooled by
// a running maximum computed in a streaming, FlashAttention-like way to avoid
// the O(L^2) matrix); §2.A pre-eviction (queries arrive in ranges).
//
//   I[t] = max(I[t], max_{s in [max(t, q_begin), q_end)} qtilde_s . khat_t)
#include "common.cuh"
#include "internal.h"

namespace imem {
namespace {

constexpr int kKT = 64;   // keys per CTA
constexpr int kQT = 64;   // queries per step
constexpr int kSThreads = 256;

__global__ void __launch_bounds__(kSThreads)
scoring_kernel(const float* __restrict__ qt, const float* __restrict__ kh, int L, int dI,
               int q_begin, int q_end, float* __restrict__ running_max) {
  extern __shared__ float sm[];
  float* sK = sm;                    // [dI][kKT]
  float* sQ = sK + dI * kKT;         // [dI][kQT]
  float* sRed = sQ + dI * kQT;       // [16][kKT]
  const int bi = blockIdx.y;
  const int k0 = blockIdx.x * kKT;
  const int tid = threadIdx.x;
  const int tk = tid % 16, tq = tid / 16;

  for (int i = tid; i < kKT * dI; i += kSThreads) {
    const int kk = i / dI, j = i % dI;
    const int t = k0 + kk;
    sK[j * kKT + kk] = (t < q_end) ? kh[((size_t)bi * L + t) * dI + j] : 0.f;
  }
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  const int s_first = max(q_begin, k0);
  for (int s0 = s_first; s0 < q_end; s0 += kQT) {
    __syncthreads();
    for (int i = tid; i < kQT * dI; i += kSThreads) {
      const int qq = i / dI, j = i % dI;
      const int s = s0 + qq;
      sQ[j * kQT + qq] = (s < q_end) ? qt[((size_t)bi * L + s) * dI + j] : 0.f;
    }
    __syncthreads();
    float acc[4][4] = {};
    for (int j = 0; j < dI; ++j) {
      const float4 kv = *reinterpret_cast<const float4*>(&sK[j * kKT + tk * 4]);
      const float4 qv = *reinterpret_cast<const float4*>(&sQ[j * kQT + tq * 4]);
      const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
      const float qq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(kk[a], qq[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int t = k0 + tk * 4 + a;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int s = s0 + tq * 4 + b;
        if (s >= t && s < q_end) mx[a] = fmaxf(mx[a], acc[a][b]);
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int a = 0; a < 4; ++a) sRed[tq * kKT + tk * 4 + a] = mx[a];
  __syncthreads();
  if (tid < kKT) {
    const int t = k0 + tid;
    if (t < q_end) {
      float m = running_max[(size_t)bi * L + t];
      for (int i = 0; i < 16; ++i) m = fmaxf(m, sRed[i * kKT + tid]);
      running_max[(size_t)bi * L + t] = m;
    }
  }
}

}  // namespace

cudaError_t launch_scoring(const Ctx& c, int batch, int L, const float* qt, const float* kh,
                           float* running_max, int q_begin, int q_end, cudaStream_t st) {
  const int dI = c.cfg.idx_dim;
  const size_t smem = ((size_t)dI * kKT + dI * kQT + 16 * kKT) * sizeof(float);
  dim3 grid((q_end + kKT - 1) / kKT, batch);
  cudaError_t e = cudaFuncSetAttribute(scoring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  scoring_kernel<<<grid, kSThreads, smem, st>>>(qt, kh, L, dI, q_begin, q_end, running_max);
  return cudaGetLastError();
}

}  // namespace imem
