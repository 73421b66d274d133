// online.cu -- decode-time online eviction at a fixed budget.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B (the memory is a fixed-size state updated online during
// inference from the tokens that leave the cache) and §2.A (the indexer's
// per-key importance is the running maximum of the gated scores over the
// queries that arrive).
//
// The cache holds B tokens in slots [0, B) in any order, each with its
// indexer key k^ (bf16), importance I and position. Per decode step:
//   features     the new token's indexer query shares and key rows (per-head
//                projections of the attention query, gate logits and key
//                from the hidden state): Hq + 8 CTAs per sequence, one GEMV
//                each, partials in the workspace. It needs neither the cache
//                nor the memory, so the C ABI runs it on a second stream next
//                to the attention step (which appends the new token at slot B);
//   score+evict  (after both branches) one thread-block cluster per sequence,
//                a CTA per KV head: q~ and k^ from the partials (RMS norm),
//                I_t <- max(I_t, q~ . k^_t) for the cached tokens, the new
//                token's I = q~ . k^_new; the least important of the B + 1
//                (ties: the higher position) by per-CTA minima of a packed
//                (ordered importance, inverted position) key exchanged over
//                distributed shared memory; then per KV head phi = W_phi k_e,
//                M <- lambda M + phi v_e^T, b <- lambda b + phi; the new token
//                and the evicted one swap slots (row, indexer key,
//                importance, position), so slot B keeps the token that left
//                with the importance it was chosen by; cache_len returns to B
//                and the workspace's decode tag of the sequence is cleared
//                (rows of slot e and the memory changed after the attention).
// q~ and k^ are rounded to bf16 before their dot products, as in prefill.
#include "common.cuh"
#include "internal.h"

#include <cooperative_groups.h>
#include <math.h>

namespace imem {
namespace {

constexpr int kOnThreads = 256;
constexpr int kKSplit = 8;            // CTAs sharing the d_I key rows of a sequence (<= 8 rows each)

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

// Programmatic dependent launch: each online kernel may start while the
// previous kernel of the stream runs; it waits before reading anything that
// kernel may write, and lets its own dependents start early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

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
// Every load moves 8 elements (16 bytes of bf16); H and D are multiples of 64.
template <typename T>
__global__ void __launch_bounds__(kOnThreads)
online_features_kernel(const T* __restrict__ x, const T* __restrict__ q, const T* __restrict__ WcT,
                       const T* __restrict__ WqT, int H, int Hq, int D, int dI,
                       float* __restrict__ qpart, float* __restrict__ kpart) {
  __shared__ float red[kOnThreads / 32];
  __shared__ float s_red8[kOnThreads / 32][8];
  __shared__ float s_qi[64];
  const int bi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch();
  const T* xb = x + (size_t)bi * H;
  if ((int)blockIdx.x < Hq) {
    const int h = blockIdx.x;
    // gate logit over the hidden state (row dI + h of WcT is w_ig[:, h])
    const T* wg = WcT + (size_t)(dI + h) * H;
    float z = 0.f;
    for (int c = 8 * tid; c < H; c += 8 * kOnThreads) {
      float wf[8], xf[8];
      load8<T>(wg + c, wf);
      load8<T>(xb + c, xf);
#pragma unroll
      for (int e = 0; e < 8; ++e) z = fmaf(wf[e], xf[e], z);
    }
    z = block_sum(z, red);
    // qI_j = W_iq[h][:, j] . q_h (row h*dI + j of WqT): 4 threads per row,
    // each D/4 elements
    const T* qh = q + ((size_t)bi * Hq + h) * D;
    const int j = tid >> 2, part = tid & 3;
    float a = 0.f;
    if (j < dI) {
      const T* wr = WqT + ((size_t)h * dI + j) * D;
      for (int c = 8 * part; c < D; c += 32) {
        float wf[8], qf[8];
        load8<T>(wr + c, wf);
        load8<T>(qh + c, qf);
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(wf[e], qf[e], a);
      }
    }
    a += __shfl_xor_sync(0xffffffffu, a, 1);
    a += __shfl_xor_sync(0xffffffffu, a, 2);
    if (j < dI && part == 0) s_qi[j] = a;
    __syncthreads();
    const float ss = block_sum(tid < dI ? s_qi[tid] * s_qi[tid] : 0.f, red);
    const float coef = sigmoidf_(z) * rsqrtf(ss / dI + 1e-6f) * rsqrtf((float)dI);
    for (int jj = tid; jj < dI; jj += kOnThreads)
      qpart[((size_t)bi * Hq + h) * dI + jj] = coef * s_qi[jj];
  } else {
    // rows [r0, r0 + nr) of W_ik^T x: every thread takes 8 hidden elements
    // at a time for all rows of the slice
    const int s = blockIdx.x - Hq;
    const int per = (dI + kKSplit - 1) / kKSplit;
    const int r0 = s * per, nr = min(per, dI - r0);
    float acc[8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) acc[rr] = 0.f;
    for (int c = 8 * tid; c < H; c += 8 * kOnThreads) {
      float xf[8];
      load8<T>(xb + c, xf);
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        if (rr < nr) {
          float wf[8];
          load8<T>(WcT + (size_t)(r0 + rr) * H + c, wf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[rr] = fmaf(wf[e], xf[e], acc[rr]);
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const float v = warp_sum(acc[rr]);
      if (lane == 0) s_red8[warp][rr] = v;
    }
    __syncthreads();
    if (tid < nr) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kOnThreads / 32; ++w) t += s_red8[w][tid];
      kpart[(size_t)bi * dI + r0 + tid] = t;
    }
  }
}

// ---- importances, the token to evict, memory update and slot swap ------------
// After the attention step and the features (the join of the two streams):
// one thread-block cluster of Hkv CTAs per sequence.
// Phase 1 (every CTA): q~ (the sum of the heads' shares) and k^ (RMS norm),
// both rounded to bf16; for its block of the B + 1 candidate rows (slot B:
// the new token, scored by its own query) I_t <- max(I_t, q~ . k^_t), and the
// block's least important candidate as a packed key (ordered importance << 32
// | ~position: the minimum is the least important, ties to the higher
// position). Every CTA writes its candidate into every CTA's table
// (distributed shared memory); after a cluster barrier each takes the same
// minimum: the token e that leaves (the new token if no importance is
// ordered, e.g. NaN).
// Phase 2 (CTA = KV head kh): phi = W_phi k_e, M <- lambda M + phi v_e^T,
// b <- lambda b + phi, and the rows of slot e and slot B (the new token,
// appended by the attention step) swap for this head; CTA 0 also swaps the
// indexer keys, importances and positions (slot e takes the new token, slot
// B keeps the evicted one with the importance it was chosen by), writes the
// evicted position, returns cache_len to B, advances next_pos and clears the
// decode tag (slot e and the memory changed after the attention step).
__device__ __forceinline__ float order_key_inv(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

template <typename T>
__global__ void __launch_bounds__(kOnThreads)
online_score_evict_kernel(int B, int cap, int Hq, int Hkv, int D, int r, int dI, int rows_per_cta,
                          float lambda, const float* __restrict__ qpart,
                          const float* __restrict__ kpart, const float* __restrict__ W_phi,
                          T* __restrict__ K_ret, T* __restrict__ V_ret,
                          __nv_bfloat16* __restrict__ khat_ret, float* __restrict__ I_ret,
                          int32_t* __restrict__ pos_ret, int32_t* __restrict__ next_pos,
                          int32_t* __restrict__ cache_len, float* __restrict__ M,
                          float* __restrict__ bstab, int32_t* __restrict__ evicted,
                          int* __restrict__ dec_tag) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ float osm[];
  float* sk = osm;          // [D] the evicted token's key, this CTA's head
  float* sv = sk + D;       // [D] its value
  float* sphi = sv + D;     // [r]
  __shared__ float s_qt[64], s_kn[64];
  __shared__ float s_hsum[4][64];
  __shared__ float red[kOnThreads / 32];
  __shared__ unsigned long long s_key[kOnThreads / 32];
  __shared__ int s_slot[kOnThreads / 32];
  __shared__ unsigned long long s_ckey[kOnlineMaxCluster];   // one per CTA of the cluster
  __shared__ int s_cslot[kOnlineMaxCluster];
  __shared__ float s_Inew;
  __shared__ int s_e, s_epos;
  __shared__ float s_Ie;
  const int bi = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nct = gridDim.x, rank = blockIdx.x;
  // phase 0 of the cluster barrier: "this CTA is running" (its shared memory
  // may be written by the others only after every CTA has arrived)
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
  pdl_wait();
  pdl_launch();
  // q~ (sum over heads: 4 groups of heads per feature, loads in flight
  // together) and the new key k^ (RMS norm), both rounded to bf16
  {
    const int j = tid & 63, grp = tid >> 6;
    float a = 0.f;
    if (j < dI) {
      const int h0 = grp * ((Hq + 3) / 4), h1 = min(Hq, h0 + (Hq + 3) / 4);
#pragma unroll 8
      for (int h = h0; h < h1; ++h) a += qpart[((size_t)bi * Hq + h) * dI + j];
    }
    s_hsum[grp][j] = a;
  }
  const float kv = tid < dI ? kpart[(size_t)bi * dI + tid] : 0.f;
  __syncthreads();
  if (tid < dI) s_qt[tid] = bf16_round((s_hsum[0][tid] + s_hsum[1][tid]) + (s_hsum[2][tid] + s_hsum[3][tid]));
  const float ss = block_sum(kv * kv, red);
  if (tid < dI) s_kn[tid] = bf16_round(kv * rsqrtf(ss / dI + 1e-6f));
  for (int j = tid + dI; j < 64; j += kOnThreads) { s_qt[j] = 0.f; s_kn[j] = 0.f; }
  __syncthreads();
  if (warp == 0) {   // the new token's importance: its own score
    float a = fmaf(s_kn[lane], s_qt[lane], s_kn[lane + 32] * s_qt[lane + 32]);
    a = warp_sum(a);
    if (lane == 0) s_Inew = a;
  }
  __syncthreads();
  const int npos = next_pos[bi];

  unsigned long long best = ~0ull;
  int best_slot = -1;
  const int t0 = rank * rows_per_cta, t1 = min(B + 1, t0 + rows_per_cta);
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
      I = s_Inew;
      pos = npos;
    }
    const unsigned long long key =
        ((unsigned long long)order_key(I) << 32) | (unsigned long long)(~(uint32_t)pos);
    if (key < best) { best = key; best_slot = t; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long k2 = __shfl_xor_sync(0xffffffffu, best, o);
    const int s2 = __shfl_xor_sync(0xffffffffu, best_slot, o);
    if (k2 < best) { best = k2; best_slot = s2; }
  }
  if (lane == 0) { s_key[warp] = best; s_slot[warp] = best_slot; }
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");   // phase 0: all running
  if (tid == 0) {   // this CTA's candidate into slot `rank` of every CTA's table
    unsigned long long k = s_key[0];
    int sl = s_slot[0];
    for (int w = 1; w < kOnThreads / 32; ++w)
      if (s_key[w] < k) { k = s_key[w]; sl = s_slot[w]; }
    for (int d = 0; d < nct; ++d) {
      cluster.map_shared_rank(s_ckey, d)[rank] = k;
      cluster.map_shared_rank(s_cslot, d)[rank] = sl;
    }
  }
  cluster.sync();   // every candidate is in every table; every CTA's reads of
                    // the indexer keys and importances are done
  if (tid == 0) {
    unsigned long long k = ~0ull;
    int e = -1;
    for (int i = 0; i < nct; ++i)
      if (s_ckey[i] < k) { k = s_ckey[i]; e = s_cslot[i]; }
    if (e < 0) {   // no ordered candidate (NaN importances): the new token leaves
      s_e = B; s_epos = npos; s_Ie = s_Inew;
    } else {
      s_e = e;
      s_epos = (int32_t)(~(uint32_t)(k & 0xffffffffull));
      s_Ie = order_key_inv((uint32_t)(k >> 32));
    }
  }
  __syncthreads();
  const int e = s_e;
  // ---- phase 2: this CTA's KV head
  const int kh = rank;
  if (kh < Hkv) {
    const size_t rs = (size_t)Hkv * D;
    T* ke = K_ret + ((size_t)bi * cap + e) * rs + (size_t)kh * D;
    T* ve = V_ret + ((size_t)bi * cap + e) * rs + (size_t)kh * D;
    for (int c = tid; c < D; c += kOnThreads) { sk[c] = ldf(ke + c); sv[c] = ldf(ve + c); }
    __syncthreads();
    // phi = W_phi k: 4 threads per row, float4 loads
    for (int j0 = 0; j0 < r; j0 += kOnThreads / 4) {
      const int j = j0 + tid / 4, part = tid & 3;
      float a = 0.f;
      if (j < r) {
        const float4* wr = reinterpret_cast<const float4*>(W_phi + (size_t)j * D);
#pragma unroll 8
        for (int c4 = part; c4 < D / 4; c4 += 4) {
          const float4 w = __ldg(wr + c4);
          a = fmaf(w.x, sk[4 * c4], fmaf(w.y, sk[4 * c4 + 1], fmaf(w.z, sk[4 * c4 + 2], fmaf(w.w, sk[4 * c4 + 3], a))));
        }
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      if (j < r && part == 0) sphi[j] = a;
    }
    __syncthreads();
    float4* Mu = reinterpret_cast<float4*>(M + ((size_t)bi * Hkv + kh) * r * D);
#pragma unroll 4
    for (int i = tid; i < r * D / 4; i += kOnThreads) {
      const int j = (4 * i) / D, c = (4 * i) % D;
      float4 m = Mu[i];
      const float ph = sphi[j];
      m.x = fmaf(lambda, m.x, ph * sv[c]);
      m.y = fmaf(lambda, m.y, ph * sv[c + 1]);
      m.z = fmaf(lambda, m.z, ph * sv[c + 2]);
      m.w = fmaf(lambda, m.w, ph * sv[c + 3]);
      Mu[i] = m;
    }
    for (int j = tid; j < r; j += kOnThreads) {
      float* bp = bstab + ((size_t)bi * Hkv + kh) * r + j;
      *bp = fmaf(lambda, *bp, sphi[j]);
    }
    if (e != B) {   // the new token (slot B) and the evicted one swap rows
      T* kn = K_ret + ((size_t)bi * cap + B) * rs + (size_t)kh * D;
      T* vn = V_ret + ((size_t)bi * cap + B) * rs + (size_t)kh * D;
      for (int c = tid; c < D; c += kOnThreads) {
        const T k0 = ke[c], v0 = ve[c];
        ke[c] = kn[c]; ve[c] = vn[c];
        kn[c] = k0; vn[c] = v0;
      }
    }
  }
  if (rank == 0) {
    if (tid < kIdxPad / 8) {
      uint4* hb = reinterpret_cast<uint4*>(khat_ret + ((size_t)bi * cap + B) * kIdxPad) + tid;
      uint4* he = reinterpret_cast<uint4*>(khat_ret + ((size_t)bi * cap + e) * kIdxPad) + tid;
      float f[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) f[c] = s_kn[8 * tid + c];
      if (e != B) *hb = *he;
      store8<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(he), f);
    }
    if (tid == 0) {
      I_ret[(size_t)bi * cap + e] = s_Inew;
      pos_ret[(size_t)bi * cap + e] = npos;
      I_ret[(size_t)bi * cap + B] = s_Ie;
      pos_ret[(size_t)bi * cap + B] = s_epos;
      evicted[bi] = s_epos;
      cache_len[bi] = B;
      dec_tag[bi] = 0;
      next_pos[bi] = npos + 1;
    }
  }
}

}  // namespace

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

// launch with programmatic stream serialization (the kernels wait for their
// predecessor themselves)
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kOnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

cudaError_t launch_online_features(const Ctx& c, int batch, const void* x, const void* q,
                                   float* qpart, float* kpart, cudaStream_t st) {
  const int H = c.cfg.hidden, Hq = c.cfg.n_q_heads, D = c.cfg.head_dim, dI = c.cfg.idx_dim;
  dim3 g(Hq + kKSplit, batch);
  if (c.cfg.dtype == IMEM_BF16)
    return launch_pdl(online_features_kernel<__nv_bfloat16>, g, 0, st, x, q, c.WcT, c.WqT, H, Hq,
                      D, dI, qpart, kpart);
  return launch_pdl(online_features_kernel<float>, g, 0, st, x, q, c.WcT, c.WqT, H, Hq, D, dI,
                    qpart, kpart);
}

cudaError_t launch_online_score_evict(const Ctx& c, int batch, int B, int cap, const float* qpart,
                                      const float* kpart, void* khat_ret, float* I_ret,
                                      int32_t* pos_ret, int32_t* next_pos, void* K_ret, void* V_ret,
                                      int32_t* cache_len, float* M, float* bstab, int32_t* evicted,
                                      int* dec_tag, cudaStream_t st) {
  const int Hkv = c.cfg.n_kv_heads, D = c.cfg.head_dim, r = c.cfg.mem_r;
  const int nct = Hkv;   // one CTA per KV head
  if (nct > kOnlineMaxCluster) return cudaErrorInvalidValue;
  const int rows_per_cta = (B + 1 + nct - 1) / nct;
  const size_t sm = (size_t)(2 * D + r) * sizeof(float);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nct, batch, 1);
  cfg.blockDim = dim3(kOnThreads, 1, 1);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = nct;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (c.cfg.dtype == IMEM_BF16) {
    auto k = online_score_evict_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, k, B, cap, c.cfg.n_q_heads, Hkv, D, r, c.cfg.idx_dim,
                              rows_per_cta, c.cfg.lambda, qpart, kpart, (const float*)c.W_phi,
                              (__nv_bfloat16*)K_ret, (__nv_bfloat16*)V_ret,
                              (__nv_bfloat16*)khat_ret, I_ret, pos_ret, next_pos, cache_len, M,
                              bstab, evicted, dec_tag);
  }
  auto k = online_score_evict_kernel<float>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k, B, cap, c.cfg.n_q_heads, Hkv, D, r, c.cfg.idx_dim,
                            rows_per_cta, c.cfg.lambda, qpart, kpart, (const float*)c.W_phi,
                            (float*)K_ret, (float*)V_ret, (__nv_bfloat16*)khat_ret, I_ret, pos_ret,
                            next_pos, cache_len, M, bstab, evicted, dec_tag);
}

}  // namespace imem
