// prologue.cu -- indexer features for a range of tokens.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.A Architecture: an MQA-style indexer that down-projects the
// multi-head queries to a low dimension, derives one shared key from the
// hidden state, applies QK-norm for stability and a learnable gate that
// modulates each head's contribution.
//
//   kI_t  = x_t W_ik              khat_t = kI_t / sqrt(mean(kI_t^2) + 1e-6)
//   qI_sh = q_sh W_iq[h]          qhat_sh = qI_sh / sqrt(mean(qI_sh^2) + 1e-6)
//   gamma_sh = sigmoid(x_s . w_ig[:, h])
//   qtilde_s = sum_h gamma_sh qhat_sh / sqrt(dI)
// Because no activation sits between the head products and the head sum,
// A[s,t] = sum_h gamma_sh (qhat_sh . khat_t)/sqrt(dI) = qtilde_s . khat_t exactly,
// so the scoring pass contracts over dI only.
//
// Also resets the running maximum of the tokens in the range to -inf (those
// keys get their first queries in this range).
#include "common.cuh"
#include "internal.h"

namespace imem {
namespace {

constexpr int kTok = 32;
constexpr int kPThreads = 256;
constexpr int kHChunk = 64;

template <typename T>
__global__ void __launch_bounds__(kPThreads)
prologue_kernel(const T* __restrict__ X, const T* __restrict__ Q, const T* __restrict__ W_iq,
                const T* __restrict__ W_ik, const T* __restrict__ w_ig, int L, int H, int Hq,
                int D, int dI, int q_begin, int q_end, __nv_bfloat16* __restrict__ qt,
                __nv_bfloat16* __restrict__ kh, float* __restrict__ running_max) {
  extern __shared__ float sm[];
  const int NC = dI + Hq;                 // key features + gate logits
  float* sX = sm;                         // [kTok][kHChunk]
  float* sWc = sX + kTok * kHChunk;       // [kHChunk][NC]
  float* sKG = sWc + kHChunk * NC;        // [kTok][NC] key features | gate logits
  float* sWq = sKG + kTok * NC;           // [D][dI]
  float* sQ = sWq + D * dI;               // [kTok][D]
  float* sQI = sQ + kTok * D;             // [kTok][dI]
  float* sRms = sQI + kTok * dI;          // [kTok]
  const int bi = blockIdx.y;
  const int t0 = q_begin + blockIdx.x * kTok;
  const int tid = threadIdx.x;

  // ---- key features and gate logits: [kTok, H] x [H, dI + Hq]
  const int n_out = kTok * NC;
  float acc[(kTok * 128) / kPThreads];    // NC <= 128
  for (int a = 0; a < (kTok * 128) / kPThreads; ++a) acc[a] = 0.f;
  for (int h0 = 0; h0 < H; h0 += kHChunk) {
    __syncthreads();
    for (int i = tid; i < kTok * kHChunk; i += kPThreads) {
      const int tt = i / kHChunk, c = i % kHChunk;
      const int t = t0 + tt;
      sX[i] = (t < q_end) ? Elem<T>::to_f(X[((size_t)bi * L + t) * H + h0 + c]) : 0.f;
    }
    for (int i = tid; i < kHChunk * NC; i += kPThreads) {
      const int c = i / NC, j = i % NC;
      sWc[i] = (j < dI) ? Elem<T>::to_f(W_ik[(size_t)(h0 + c) * dI + j])
                        : Elem<T>::to_f(w_ig[(size_t)(h0 + c) * Hq + (j - dI)]);
    }
    __syncthreads();
    for (int a = 0; a * kPThreads + tid < n_out; ++a) {
      const int o = a * kPThreads + tid, tt = o / NC, j = o % NC;
      float s = acc[a];
      for (int c = 0; c < kHChunk; ++c) s = fmaf(sX[tt * kHChunk + c], sWc[c * NC + j], s);
      acc[a] = s;
    }
  }
  for (int a = 0; a * kPThreads + tid < n_out; ++a) sKG[a * kPThreads + tid] = acc[a];
  __syncthreads();

  // ---- khat: RMS-normalised shared key (warp per token)
  const int lane = tid & 31, warp = tid >> 5;
  for (int tt = warp; tt < kTok; tt += kPThreads / 32) {
    const int t = t0 + tt;
    float ss = 0.f;
    for (int j = lane; j < dI; j += 32) ss += sKG[tt * NC + j] * sKG[tt * NC + j];
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / dI + 1e-6f);
    if (t < q_end)
      for (int j = lane; j < kIdxPad; j += 32)
        kh[((size_t)bi * L + t) * kIdxPad + j] = __float2bfloat16_rn(j < dI ? sKG[tt * NC + j] * inv : 0.f);
  }

  // ---- qtilde: per head projection, RMS norm, gate, sum
  const float inv_sqrt_dI = rsqrtf((float)dI);
  float qacc[(kTok * 64) / kPThreads];     // dI <= 64
  for (int a = 0; a < (kTok * 64) / kPThreads; ++a) qacc[a] = 0.f;
  const int n_q = kTok * dI;
  for (int h = 0; h < Hq; ++h) {
    __syncthreads();
    for (int i = tid; i < D * dI; i += kPThreads) sWq[i] = Elem<T>::to_f(W_iq[(size_t)h * D * dI + i]);
    for (int i = tid; i < kTok * D; i += kPThreads) {
      const int tt = i / D, c = i % D;
      const int t = t0 + tt;
      sQ[i] = (t < q_end) ? Elem<T>::to_f(Q[(((size_t)bi * L + t) * Hq + h) * D + c]) : 0.f;
    }
    __syncthreads();
    float qi[(kTok * 64) / kPThreads];
    for (int a = 0; a * kPThreads + tid < n_q; ++a) {
      const int o = a * kPThreads + tid, tt = o / dI, j = o % dI;
      float s = 0.f;
      for (int c = 0; c < D; ++c) s = fmaf(sQ[tt * D + c], sWq[c * dI + j], s);
      qi[a] = s;
      sQI[o] = s;
    }
    __syncthreads();
    for (int tt = warp; tt < kTok; tt += kPThreads / 32) {
      float ss = 0.f;
      for (int j = lane; j < dI; j += 32) ss += sQI[tt * dI + j] * sQI[tt * dI + j];
      ss = warp_sum(ss);
      if (lane == 0) {
        const float gamma = sigmoidf_(sKG[tt * NC + dI + h]);
        sRms[tt] = gamma * rsqrtf(ss / dI + 1e-6f) * inv_sqrt_dI;
      }
    }
    __syncthreads();
    for (int a = 0; a * kPThreads + tid < n_q; ++a) {
      const int o = a * kPThreads + tid, tt = o / dI;
      qacc[a] = fmaf(sRms[tt], qi[a], qacc[a]);
    }
  }
  for (int a = 0; a * kPThreads + tid < n_q; ++a) {
    const int o = a * kPThreads + tid, tt = o / dI, j = o % dI;
    const int t = t0 + tt;
    if (t < q_end) qt[((size_t)bi * L + t) * kIdxPad + j] = __float2bfloat16_rn(qacc[a]);
  }
  for (int i = tid; i < kTok * (kIdxPad - dI); i += kPThreads) {   // zero padding
    const int tt = i / (kIdxPad - dI), j = dI + i % (kIdxPad - dI);
    if (t0 + tt < q_end) qt[((size_t)bi * L + t0 + tt) * kIdxPad + j] = __float2bfloat16_rn(0.f);
  }
  if (tid < kTok && t0 + tid < q_end) running_max[(size_t)bi * L + t0 + tid] = -INFINITY;
}

}  // namespace

cudaError_t launch_prologue(const Ctx& c, int batch, int L, const void* X, const void* Q,
                            int q_begin, int q_end, __nv_bfloat16* qt, __nv_bfloat16* kh,
                            float* running_max, cudaStream_t st) {
  const int H = c.cfg.hidden, Hq = c.cfg.n_q_heads, D = c.cfg.head_dim, dI = c.cfg.idx_dim;
  const int NC = dI + Hq;
  const size_t smem = ((size_t)kTok * kHChunk + kHChunk * NC + kTok * NC + D * dI + kTok * D +
                       kTok * dI + kTok) * sizeof(float);
  dim3 grid((q_end - q_begin + kTok - 1) / kTok, batch);
  cudaError_t e;
  if (c.cfg.dtype == IMEM_BF16) {
    auto k = prologue_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kPThreads, smem, st>>>((const __nv_bfloat16*)X, (const __nv_bfloat16*)Q,
                                     (const __nv_bfloat16*)c.W_iq, (const __nv_bfloat16*)c.W_ik,
                                     (const __nv_bfloat16*)c.w_ig, L, H, Hq, D, dI, q_begin, q_end,
                                     qt, kh, running_max);
  } else {
    auto k = prologue_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kPThreads, smem, st>>>((const float*)X, (const float*)Q, (const float*)c.W_iq,
                                     (const float*)c.W_ik, (const float*)c.w_ig, L, H, Hq, D, dI,
                                     q_begin, q_end, qt, kh, running_max);
  }
  return cudaGetLastError();
}

}  // namespace imem
