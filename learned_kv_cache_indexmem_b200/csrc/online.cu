// online.cu -- decode-time online eviction at a fixed budget.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B (the memory is a fixed-size state updated online during
// inference from the tokens that leave the cache) and §2.A (the indexer's
// per-key importance is the running maximum of the gated scores over the
// queries that arrive).
//
// The cache holds B tokens in slots [0, B) in any order, each with its
// indexer key k^ (bf16), importance I and position. Per decode step, after
// the attention step (which appends the new token at slot B):
//   features  the new token's indexer query q~ = sum_h g_h q^_h / sqrt(dI)
//             and key k^ (per-head projections of the attention query, gate
//             logits and key from the hidden state, RMS norms): Hq + 8 CTAs
//             per sequence, one GEMV each, partials in the workspace;
//   score     I_t <- max(I_t, q~ . k^_t) for the cached tokens, the new
//             token's I = q~ . k^_new; the least important of the B + 1
//             (ties: the higher position) is found by a per-CTA minimum of a
//             packed (ordered importance, inverted position) key and a
//             last-CTA reduction;
//   evict     per KV head: phi = W_phi k_e, M <- lambda M + phi v_e^T,
//             b <- lambda b + phi; the new token's row moves into the freed
//             slot; cache_len returns to B.
// q~ and k^ are rounded to bf16 before their dot products, as in prefill.
#include "common.cuh"
#include "internal.h"

#include <math.h>

namespace imem {
namespace {

constexpr int kOnThreads = 256;
constexpr int kKSplit = 8;            // CTAs sharing the d_I key rows of a sequence

__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return Elem<T>::to_f(*p); }

// block-wide sum of one float per thread (kOnThreads threads); all threads
// receive the total
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kOnThreads / 32; ++w) t += red[w];
  return t;
}

// ---- initial state from the prefill ------------------------------------------
__global__ void __launch_bounds__(kOnThreads)
online_init_kernel(int L, int B, int cap, const float* __restrict__ running_max,
                   const int32_t* __restrict__ idx_r, const __nv_bfloat16* __restrict__ kh,
                   __nv_bfloat16* __restrict__ khat_ret, float* __restrict__ I_ret,
                   int32_t* __restrict__ pos_ret, int32_t* __restrict__ next_pos) {
  const int bi = blockIdx.y;
  const int j = blockIdx.x * (kOnThreads / 8) + threadIdx.x / 8, c = threadIdx.x % 8;
  if (j < B) {
    const int p = idx_r[(size_t)bi * B + j];
    reinterpret_cast<uint4*>(khat_ret + ((size_t)bi * cap + j) * kIdxPad)[c] =
        reinterpret_cast<const uint4*>(kh + ((size_t)bi * L + p) * kIdxPad)[c];
    if (c == 0) {
      I_ret[(size_t)bi * cap + j] = running_max[(size_t)bi * L + p];
      pos_ret[(size_t)bi * cap + j] = p;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) next_pos[bi] = L;
}

// ---- the new token's indexer features ----------------------------------------
// CTA h < Hq: qpart[h] = sigmoid(w_ig[:,h] . x) * rmsnorm(W_iq[h]^T q_h) / sqrt(dI)
// CTA Hq + s: kpart[rows of slice s] = W_ik^T x
template <typename T>
__global__ void __launch_bounds__(kOnThreads)
online_features_kernel(const T* __restrict__ x, const T* __restrict__ q, const T* __restrict__ WcT,
                       const T* __restrict__ WqT, int H, int Hq, int D, int dI,
                       float* __restrict__ qpart, float* __restrict__ kpart) {
  extern __shared__ float osm[];
  __shared__ float red[kOnThreads / 32];
  __shared__ float s_qi[64];
  const int bi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* xb = x + (size_t)bi * H;
  if ((int)blockIdx.x < Hq) {
    const int h = blockIdx.x;
    float* sq = osm;   // [D]
    for (int c = tid; c < D; c += kOnThreads) sq[c] = ldf(q + ((size_t)bi * Hq + h) * D + c);
    // gate logit over the hidden state (row dI + h of WcT is w_ig[:, h])
    const T* wg = WcT + (size_t)(dI + h) * H;
    float z = 0.f;
    for (int c = tid; c < H; c += kOnThreads) z = fmaf(ldf(wg + c), ldf(xb + c), z);
    z = block_sum(z, red);
    // qI_j = W_iq[h][:, j] . q_h (row h*dI + j of WqT), a warp per output
    for (int j = warp; j < dI; j += kOnThreads / 32) {
      const T* wr = WqT + ((size_t)h * dI + j) * D;
      float a = 0.f;
      for (int c = lane; c < D; c += 32) a = fmaf(ldf(wr + c), sq[c], a);
      a = warp_sum(a);
      if (lane == 0) s_qi[j] = a;
    }
    __syncthreads();
    float ss = 0.f;
    for (int j = tid; j < dI; j += kOnThreads) ss = fmaf(s_qi[j], s_qi[j], ss);
    ss = block_sum(ss, red);
    const float coef = sigmoidf_(z) * rsqrtf(ss / dI + 1e-6f) * rsqrtf((float)dI);
    for (int j = tid; j < dI; j += kOnThreads)
      qpart[((size_t)bi * Hq + h) * dI + j] = coef * s_qi[j];
  } else {
    const int s = blockIdx.x - Hq;
    const int per = (dI + kKSplit - 1) / kKSplit;
    for (int r = s * per + warp; r < min(dI, (s + 1) * per); r += kOnThreads / 32) {
      const T* wr = WcT + (size_t)r * H;
      float a = 0.f;
      for (int c = lane; c < H; c += 32) a = fmaf(ldf(wr + c), ldf(xb + c), a);
      a = warp_sum(a);
      if (lane == 0) kpart[(size_t)bi * dI + r] = a;
    }
  }
}

// ---- importances and the token to evict --------------------------------------
struct EvictCand {
  unsigned long long key;   // ordered importance << 32 | ~position (min wins)
  int slot;
  int pad;
};

__global__ void __launch_bounds__(kOnThreads)
online_score_kernel(int B, int cap, int Hq, int dI, int rows_per_cta,
                    const float* __restrict__ qpart, const float* __restrict__ kpart,
                    __nv_bfloat16* __restrict__ khat_ret, float* __restrict__ I_ret,
                    int32_t* __restrict__ pos_ret, const int32_t* __restrict__ next_pos,
                    EvictCand* __restrict__ cand, int* __restrict__ counter,
                    int* __restrict__ evict_slot, int32_t* __restrict__ evicted) {
  __shared__ float s_qt[64], s_kn[64];
  __shared__ float red[kOnThreads / 32];
  __shared__ unsigned long long s_key[kOnThreads / 32];
  __shared__ int s_slot[kOnThreads / 32];
  __shared__ int s_last;
  const int bi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nct = gridDim.x;
  // q~ (sum over heads) and the new key k^ (RMS norm), both rounded to bf16
  float kv = 0.f;
  if (tid < dI) {
    float a = 0.f;
    for (int h = 0; h < Hq; ++h) a += qpart[((size_t)bi * Hq + h) * dI + tid];
    s_qt[tid] = bf16_round(a);
    kv = kpart[(size_t)bi * dI + tid];
  }
  const float ss = block_sum(tid < dI ? kv * kv : 0.f, red);
  if (tid < dI) s_kn[tid] = bf16_round(kv * rsqrtf(ss / dI + 1e-6f));
  for (int j = tid + dI; j < 64; j += kOnThreads) { s_qt[j] = 0.f; s_kn[j] = 0.f; }
  __syncthreads();

  unsigned long long best = ~0ull;
  int best_slot = -1;
  const int t0 = blockIdx.x * rows_per_cta, t1 = min(B + 1, t0 + rows_per_cta);
  for (int t = t0 + tid; t < t1; t += kOnThreads) {
    float I;
    int pos;
    if (t < B) {
      const uint4* kr = reinterpret_cast<const uint4*>(khat_ret + ((size_t)bi * cap + t) * kIdxPad);
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < kIdxPad / 8; ++c) {
        float f[8];
        bf16x8_to_f32(kr[c], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(f[e], s_qt[8 * c + e], a);
      }
      I = fmaxf(I_ret[(size_t)bi * cap + t], a);
      I_ret[(size_t)bi * cap + t] = I;
      pos = pos_ret[(size_t)bi * cap + t];
    } else {   // slot B: the new token, scored by its own query
      float a = 0.f;
      for (int c = 0; c < 64; ++c) a = fmaf(s_kn[c], s_qt[c], a);
      I = a;
      pos = next_pos[bi];
      I_ret[(size_t)bi * cap + B] = I;
      pos_ret[(size_t)bi * cap + B] = pos;
      float f[8];
      for (int c = 0; c < kIdxPad / 8; ++c) {
        for (int e = 0; e < 8; ++e) f[e] = s_kn[8 * c + e];
        store8<__nv_bfloat16>(khat_ret + ((size_t)bi * cap + B) * kIdxPad + 8 * c, f);
      }
    }
    const unsigned long long key =
        ((unsigned long long)order_key(I) << 32) | (unsigned long long)(~(uint32_t)pos);
    if (key < best) { best = key; best_slot = t; }
  }
  // CTA minimum
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long k2 = __shfl_xor_sync(0xffffffffu, best, o);
    const int s2 = __shfl_xor_sync(0xffffffffu, best_slot, o);
    if (k2 < best) { best = k2; best_slot = s2; }
  }
  if (lane == 0) { s_key[warp] = best; s_slot[warp] = best_slot; }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < kOnThreads / 32; ++w)
      if (s_key[w] < best) { best = s_key[w]; best_slot = s_slot[w]; }
    cand[(size_t)bi * nct + blockIdx.x] = EvictCand{best, best_slot, 0};
    __threadfence();
    s_last = atomicAdd(&counter[bi], 1) == nct - 1;
  }
  __syncthreads();
  if (s_last && tid == 0) {
    // the last CTA of the sequence reduces the candidates
    __threadfence();
    unsigned long long k = ~0ull;
    int slot = -1;
    for (int i = 0; i < nct; ++i) {
      const EvictCand ci = cand[(size_t)bi * nct + i];
      if (ci.key < k) { k = ci.key; slot = ci.slot; }
    }
    evict_slot[bi] = slot;
    evicted[bi] = (int32_t)(~(uint32_t)(k & 0xffffffffull));
    counter[bi] = 0;
  }
}

// ---- memory update with the evicted token, slot refill ------------------------
template <typename T>
__global__ void __launch_bounds__(kOnThreads)
online_evict_kernel(int B, int cap, int Hkv, int D, int r, float lambda,
                    const int* __restrict__ evict_slot, const float* __restrict__ W_phi,
                    T* __restrict__ K_ret, T* __restrict__ V_ret,
                    __nv_bfloat16* __restrict__ khat_ret, float* __restrict__ I_ret,
                    int32_t* __restrict__ pos_ret, int32_t* __restrict__ next_pos,
                    int32_t* __restrict__ cache_len, float* __restrict__ M,
                    float* __restrict__ bstab) {
  extern __shared__ float osm[];
  float* sk = osm;          // [D]
  float* sv = sk + D;       // [D]
  float* sphi = sv + D;     // [r]
  const int kh = blockIdx.x, bi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = evict_slot[bi];
  const size_t rs = (size_t)Hkv * D;
  T* ke = K_ret + ((size_t)bi * cap + e) * rs + (size_t)kh * D;
  T* ve = V_ret + ((size_t)bi * cap + e) * rs + (size_t)kh * D;
  for (int c = tid; c < D; c += kOnThreads) { sk[c] = ldf(ke + c); sv[c] = ldf(ve + c); }
  __syncthreads();
  for (int j = warp; j < r; j += kOnThreads / 32) {
    float a = 0.f;
    for (int c = lane; c < D; c += 32) a = fmaf(W_phi[(size_t)j * D + c], sk[c], a);
    a = warp_sum(a);
    if (lane == 0) sphi[j] = a;
  }
  __syncthreads();
  float* Mu = M + ((size_t)bi * Hkv + kh) * r * D;
  for (int i = tid; i < r * D; i += kOnThreads) {
    const int j = i / D, c = i % D;
    Mu[i] = fmaf(lambda, Mu[i], sphi[j] * sv[c]);
  }
  for (int j = tid; j < r; j += kOnThreads) {
    float* bp = bstab + ((size_t)bi * Hkv + kh) * r + j;
    *bp = fmaf(lambda, *bp, sphi[j]);
  }
  if (e != B) {   // the new token (slot B) takes the freed slot
    const T* kn = K_ret + ((size_t)bi * cap + B) * rs + (size_t)kh * D;
    const T* vn = V_ret + ((size_t)bi * cap + B) * rs + (size_t)kh * D;
    for (int c = tid; c < D; c += kOnThreads) { ke[c] = kn[c]; ve[c] = vn[c]; }
  }
  if (kh == 0 && tid < kIdxPad / 8) {
    if (e != B) {
      reinterpret_cast<uint4*>(khat_ret + ((size_t)bi * cap + e) * kIdxPad)[tid] =
          reinterpret_cast<const uint4*>(khat_ret + ((size_t)bi * cap + B) * kIdxPad)[tid];
    }
    if (tid == 0) {
      if (e != B) {
        I_ret[(size_t)bi * cap + e] = I_ret[(size_t)bi * cap + B];
        pos_ret[(size_t)bi * cap + e] = pos_ret[(size_t)bi * cap + B];
      }
      cache_len[bi] = B;
      next_pos[bi] += 1;
    }
  }
}

}  // namespace

int online_score_ctas(int B) {
  int n = (B + 1 + kOnThreads - 1) / kOnThreads;
  return n > kOnlineMaxCtas ? kOnlineMaxCtas : n;
}

cudaError_t launch_online_init(const Ctx& c, int batch, int L, int B, int cap,
                               const float* running_max, const int32_t* idx_r,
                               const __nv_bfloat16* kh, __nv_bfloat16* khat_ret, float* I_ret,
                               int32_t* pos_ret, int32_t* next_pos, cudaStream_t st) {
  (void)c;
  dim3 g((B + kOnThreads / 8 - 1) / (kOnThreads / 8), batch);
  online_init_kernel<<<g, kOnThreads, 0, st>>>(L, B, cap, running_max, idx_r, kh, khat_ret, I_ret,
                                               pos_ret, next_pos);
  return cudaGetLastError();
}

cudaError_t launch_online_features(const Ctx& c, int batch, const void* x, const void* q,
                                   float* qpart, float* kpart, cudaStream_t st) {
  const int H = c.cfg.hidden, Hq = c.cfg.n_q_heads, D = c.cfg.head_dim, dI = c.cfg.idx_dim;
  dim3 g(Hq + kKSplit, batch);
  const size_t sm = (size_t)D * sizeof(float);
  if (c.cfg.dtype == IMEM_BF16)
    online_features_kernel<__nv_bfloat16><<<g, kOnThreads, sm, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)q, (const __nv_bfloat16*)c.WcT,
        (const __nv_bfloat16*)c.WqT, H, Hq, D, dI, qpart, kpart);
  else
    online_features_kernel<float><<<g, kOnThreads, sm, st>>>(
        (const float*)x, (const float*)q, (const float*)c.WcT, (const float*)c.WqT, H, Hq, D, dI,
        qpart, kpart);
  return cudaGetLastError();
}

cudaError_t launch_online_evict(const Ctx& c, int batch, int B, int cap, const float* qpart,
                                const float* kpart, void* khat_ret, float* I_ret, int32_t* pos_ret,
                                int32_t* next_pos, void* K_ret, void* V_ret, int32_t* cache_len,
                                float* M, float* bstab, int32_t* evicted, void* cand,
                                int* counter, int* evict_slot, cudaStream_t st) {
  const int nct = online_score_ctas(B);
  const int rows_per_cta = (B + 1 + nct - 1) / nct;
  online_score_kernel<<<dim3(nct, batch), kOnThreads, 0, st>>>(
      B, cap, c.cfg.n_q_heads, c.cfg.idx_dim, rows_per_cta, qpart, kpart,
      (__nv_bfloat16*)khat_ret, I_ret, pos_ret, next_pos, (EvictCand*)cand, counter, evict_slot,
      evicted);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int Hkv = c.cfg.n_kv_heads, D = c.cfg.head_dim, r = c.cfg.mem_r;
  const size_t sm = (size_t)(2 * D + r) * sizeof(float);
  dim3 g(Hkv, batch);
  if (c.cfg.dtype == IMEM_BF16)
    online_evict_kernel<__nv_bfloat16><<<g, kOnThreads, sm, st>>>(
        B, cap, Hkv, D, r, c.cfg.lambda, evict_slot, c.W_phi, (__nv_bfloat16*)K_ret,
        (__nv_bfloat16*)V_ret, (__nv_bfloat16*)khat_ret, I_ret, pos_ret, next_pos, cache_len, M,
        bstab);
  else
    online_evict_kernel<float><<<g, kOnThreads, sm, st>>>(
        B, cap, Hkv, D, r, c.cfg.lambda, evict_slot, c.W_phi, (float*)K_ret, (float*)V_ret,
        (__nv_bfloat16*)khat_ret, I_ret, pos_ret, next_pos, cache_len, M, bstab);
  return cudaGetLastError();
}

}  // namespace imem
