// memory.cu -- latent-memory update from the evicted tokens.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B Mechanism (fast weights): the evicted tokens update online a
// fixed-size state matrix M and a stabiliser vector b by an outer-product
// accumulation with decay. With phi(k) = W_phi k and decay lambda per evicted
// token, in ascending position order:
//   M <- lambda M + phi(k) v^T,   b <- lambda b + phi(k)
// Over n tokens this equals
//   M = lambda^n M0 + sum_i lambda^(n-1-i) phi(k_i) v_i^T   (same for b),
// so disjoint runs of evicted tokens can be accumulated independently with
// their absolute weights lambda^(n-1-i) and summed.
//
// Pass 1: grid (groups, Hkv, batch); a CTA accumulates the weighted sum of
// one run of evicted tokens for one (sequence, KV head) into fp32 partials.
// Pass 2: one CTA per (sequence, KV head) folds the partials in a fixed order
// into lambda^n M0 (deterministic).
#include "common.cuh"
#include "internal.h"

#include <math.h>

namespace imem {
namespace {

constexpr int kMemThreads = 256;
constexpr int kSub = 32;  // tokens per inner step

template <typename T, int D>
__global__ void __launch_bounds__(kMemThreads)
memory_partial_kernel(const T* __restrict__ K, const T* __restrict__ V,
                      const int32_t* __restrict__ idx_e, int n_e, int L, int Hkv,
                      const float* __restrict__ W_phi, int r, float lam, int tokens_per_group,
                      float* __restrict__ partials) {
  extern __shared__ float smem[];
  float* sW = smem;                 // [r][D]
  float* sK = sW + r * D;           // [kSub][D]
  float* sV = sK + kSub * D;        // [kSub][D]
  float* sP = sV + kSub * D;        // [kSub][r]  weighted phi
  const int g = blockIdx.x, kh = blockIdx.y, bi = blockIdx.z;
  const int G = gridDim.x;
  const int tid = threadIdx.x;
  const int j0 = g * tokens_per_group;
  const int j1 = min(n_e, j0 + tokens_per_group);

  for (int i = tid; i < r * D; i += kMemThreads) sW[i] = W_phi[i];

  // this thread's block of the r x D accumulator: RB rows x 8 columns
  const int cols8 = D / 8;                      // column blocks of 8
  const int nblk = (r * D) / 8;                 // blocks of 8 entries
  constexpr int kMaxBlk = 128 * 128 / 8 / kMemThreads;  // <= 8 blocks per thread
  float acc[kMaxBlk][8];
#pragma unroll
  for (int a = 0; a < kMaxBlk; ++a)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[a][e] = 0.f;
  float bacc = 0.f;  // threads < r accumulate b

  const size_t row_stride = (size_t)Hkv * D;
  const T* Kb = K + (size_t)bi * L * row_stride + (size_t)kh * D;
  const T* Vb = V + (size_t)bi * L * row_stride + (size_t)kh * D;
  const int32_t* E = idx_e + (size_t)bi * n_e;

  for (int s0 = j0; s0 < j1; s0 += kSub) {
    __syncthreads();
    // gather kSub evicted rows of this head (D/8 vectors per row)
    for (int i = tid; i < kSub * cols8; i += kMemThreads) {
      const int jj = i / cols8, cb = i % cols8;
      float kf[8], vf[8];
      if (s0 + jj < j1) {
        const int pos = E[s0 + jj];
        load8<T>(Kb + (size_t)pos * row_stride + cb * 8, kf);
        load8<T>(Vb + (size_t)pos * row_stride + cb * 8, vf);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) { kf[e] = 0.f; vf[e] = 0.f; }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) { sK[jj * D + cb * 8 + e] = kf[e]; sV[jj * D + cb * 8 + e] = vf[e]; }
    }
    __syncthreads();
    // weighted features: P[j][i] = lam^(n-1-j) * (W_phi k_j)[i]
    for (int i = tid; i < kSub * r; i += kMemThreads) {
      const int jj = i / r, ri = i % r;
      float a = 0.f;
      for (int c = 0; c < D; ++c) a = fmaf(sW[ri * D + c], sK[jj * D + c], a);
      const int j = s0 + jj;
      const float w = (j < j1) ? powf(lam, (float)(n_e - 1 - j)) : 0.f;
      sP[jj * r + ri] = a * w;
    }
    __syncthreads();
    // accumulate P^T V into this thread's blocks
#pragma unroll
    for (int a = 0; a < kMaxBlk; ++a) {
      const int blk = tid + a * kMemThreads;
      if (blk < nblk) {
        const int ri = blk / cols8, cb = blk % cols8;
        for (int jj = 0; jj < kSub; ++jj) {
          const float p = sP[jj * r + ri];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[a][e] = fmaf(p, sV[jj * D + cb * 8 + e], acc[a][e]);
        }
      }
    }
    if (tid < r)
      for (int jj = 0; jj < kSub; ++jj) bacc += sP[jj * r + tid];
  }

  float* out = partials + (((size_t)bi * Hkv + kh) * G + g) * (size_t)(r * D + r);
#pragma unroll
  for (int a = 0; a < kMaxBlk; ++a) {
    const int blk = tid + a * kMemThreads;
    if (blk < nblk) {
      const int ri = blk / cols8, cb = blk % cols8;
#pragma unroll
      for (int e = 0; e < 8; ++e) out[ri * D + cb * 8 + e] = acc[a][e];
    }
  }
  if (tid < r) out[r * D + tid] = bacc;
}

__global__ void memory_finalize_kernel(const float* __restrict__ partials, int G, int r, int D,
                                       float decay_n, float* __restrict__ M,
                                       float* __restrict__ bstab) {
  const int unit = blockIdx.x;
  const size_t psz = (size_t)r * D + r;
  const float* p = partials + (size_t)unit * G * psz;
  float* Mu = M + (size_t)unit * r * D;
  float* bu = bstab + (size_t)unit * r;
  for (int i = threadIdx.x; i < r * D + r; i += blockDim.x) {
    float a = (i < r * D) ? Mu[i] * decay_n : bu[i - r * D] * decay_n;
    for (int g = 0; g < G; ++g) a += p[g * psz + i];
    if (i < r * D) Mu[i] = a;
    else bu[i - r * D] = a;
  }
}

}  // namespace

int memory_groups(int batch, int n_kv_heads, int n_e, int chunk) {
  const int units = batch * n_kv_heads;
  const int chunks = (n_e + chunk - 1) / chunk;
  int G = (2 * 148 + units - 1) / units;
  if (G > chunks) G = chunks;
  if (G > kMemMaxGroups) G = kMemMaxGroups;
  if (G < 1) G = 1;
  return G;
}

cudaError_t launch_memory_update(const Ctx& c, int batch, int L, const void* K, const void* V,
                                 const int32_t* idx_e, int n_e, int chunk, float* M, float* bstab,
                                 float* partials, cudaStream_t st) {
  if (n_e == 0) return cudaSuccess;
  const int Hkv = c.cfg.n_kv_heads, D = c.cfg.head_dim, r = c.cfg.mem_r;
  const int G = memory_groups(batch, Hkv, n_e, chunk);
  const int chunks = (n_e + chunk - 1) / chunk;
  const int tokens_per_group = ((chunks + G - 1) / G) * chunk;
  dim3 grid(G, Hkv, batch);
  const size_t smem = ((size_t)r * D + 2 * kSub * D + kSub * r) * sizeof(float);
  cudaError_t e = cudaSuccess;
#define IMEM_MEM(TT, DD)                                                                       \
  do {                                                                                         \
    auto kfn = memory_partial_kernel<TT, DD>;                                                  \
    e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
    if (e != cudaSuccess) return e;                                                            \
    kfn<<<grid, kMemThreads, smem, st>>>((const TT*)K, (const TT*)V, idx_e, n_e, L, Hkv,       \
                                         c.W_phi, r, c.cfg.lambda, tokens_per_group, partials); \
  } while (0)
  if (c.cfg.dtype == IMEM_BF16) {
    if (D == 128) IMEM_MEM(__nv_bfloat16, 128); else IMEM_MEM(__nv_bfloat16, 64);
  } else {
    if (D == 128) IMEM_MEM(float, 128); else IMEM_MEM(float, 64);
  }
#undef IMEM_MEM
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float decay_n = (float)pow((double)c.cfg.lambda, (double)n_e);
  memory_finalize_kernel<<<batch * Hkv, 256, 0, st>>>(partials, G, r, D, decay_n, M, bstab);
  return cudaGetLastError();
}

}  // namespace imem
