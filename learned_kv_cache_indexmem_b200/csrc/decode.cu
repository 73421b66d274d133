// decode.cu -- one decode step over the retained (compacted) KV cache with the
// gated latent-memory readout fused into the combine.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B Output: o = o_attn + g(q) * m(q), where o_attn is standard
// attention over the retained tokens and m(q) the readout of the memory M
// (with the stabiliser b); the readout weights are a projection phi and a gate
// g(q). The split-K combine uses the exact merge of softmax partial states
// (max, normaliser, unnormalised output) over disjoint key blocks, the
// online-softmax identity stated in "Context Memorization for Efficient Long
// Context Generation" (technical summary, Method).
//
// Grid (splits, Hkv, batch). Each CTA streams the rows of one split of one
// (sequence, KV head) and keeps a softmax state for every query head of the
// GQA group. The last CTA of a (sequence, KV head) -- found with a counter in
// the workspace, no waiting -- merges the partial states, adds the memory
// readout and writes the output; the last CTA of a sequence advances
// cache_len. Split 0 writes the new key/value row into the cache; the CTA that
// covers row cache_len reads it from k_new/v_new instead.
#include "common.cuh"
#include "internal.h"

#include <math.h>

namespace imem {
namespace {

constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int G>
struct Partial {  // one query head's softmax state in a split
  float m;        // running max of the log2-scaled logits
  float l;        // sum of 2^(s - m)
  float pad[2];
  float o[D];     // sum of 2^(s - m) v
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
              T* __restrict__ K_ret, T* __restrict__ V_ret, int32_t* __restrict__ cache_len,
              int cap, int Hkv, int rows_per_split, const float* __restrict__ M,
              const float* __restrict__ bstab, const float* __restrict__ W_phi,
              const float* __restrict__ w_gate, int r, float eps, float gate_override,
              int use_override, T* __restrict__ out, float* __restrict__ partials,
              int* __restrict__ counters, int* __restrict__ err) {
  constexpr int LPR = D / 8;          // lanes per row (8 elements per lane)
  constexpr int RPW = 32 / LPR;       // rows per warp iteration
  const int sp = blockIdx.x, kh = blockIdx.y, bi = blockIdx.z;
  const int S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = Hkv * G;

  __shared__ int s_flag;
  __shared__ float s_q[G][D];
  __shared__ Partial<D, G> s_part[4][G];   // per-warp states, then the merged state

  const int len = cache_len[bi];
  if (len >= cap) {  // full cache: the whole sequence is skipped by every CTA
    if (sp == 0 && kh == 0 && tid == 0) record_error(err, DEV_CACHE_FULL);
    return;
  }
  const int n = len + 1;  // rows including the new one
  const size_t row_stride = (size_t)Hkv * D;
  const T* Kb = K_ret + (size_t)bi * cap * row_stride + (size_t)kh * D;
  const T* Vb = V_ret + (size_t)bi * cap * row_stride + (size_t)kh * D;
  const T* kn = k_new + ((size_t)bi * Hkv + kh) * D;
  const T* vn = v_new + ((size_t)bi * Hkv + kh) * D;

  // query heads of the group, pre-scaled so that exp2 gives the softmax
  const float qscale = kLog2e * rsqrtf((float)D);
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    s_q[g][c] = Elem<T>::to_f(q[((size_t)bi * Hq + kh * G + g) * D + c]);
  }
  __syncthreads();

  // split 0 appends the new row to the cache
  if (sp == 0) {
    for (int c = tid; c < D; c += kThreads) {
      K_ret[((size_t)bi * cap + len) * row_stride + (size_t)kh * D + c] = kn[c];
      V_ret[((size_t)bi * cap + len) * row_stride + (size_t)kh * D + c] = vn[c];
    }
  }

  const int team = lane / LPR, tl = lane % LPR;
  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] = s_q[g][tl * 8 + e] * qscale;

  float m_run[G], l_run[G], o_acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o_acc[g][e] = 0.f;
  }

  const int r0 = sp * rows_per_split;
  const int r1 = min(n, r0 + rows_per_split);
  for (int base = r0 + warp * RPW; base < r1; base += 4 * RPW) {
    const int row = base + team;
    const bool valid = row < r1;
    float kf[8], vf[8];
    if (valid) {
      const T* kp = (row == len) ? kn : Kb + (size_t)row * row_stride;
      const T* vp = (row == len) ? vn : Vb + (size_t)row * row_stride;
      load8<T>(kp + tl * 8, kf);
      load8<T>(vp + tl * 8, vf);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) { kf[e] = 0.f; vf[e] = 0.f; }
    }
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(qf[g][e], kf[e], a);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      s[g] = a;
    }
    if (valid) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mn = fmaxf(m_run[g], s[g]);
        const float sc = exp2f(m_run[g] - mn);
        const float p = exp2f(s[g] - mn);
        l_run[g] = l_run[g] * sc + p;
#pragma unroll
        for (int e = 0; e < 8; ++e) o_acc[g][e] = fmaf(o_acc[g][e], sc, p * vf[e]);
        m_run[g] = mn;
      }
    }
  }

  // merge the row teams of the warp (lanes tl, tl+LPR, ...) into team 0
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, m_run[g], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l_run[g], off);
      const float mn = fmaxf(m_run[g], mo);
      const float sa = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - mn);
      const float sb = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
      l_run[g] = l_run[g] * sa + lo * sb;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o_acc[g][e], off);
        o_acc[g][e] = o_acc[g][e] * sa + oo * sb;
      }
      m_run[g] = mn;
    }
  }
  if (team == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (tl == 0) { s_part[warp][g].m = m_run[g]; s_part[warp][g].l = l_run[g]; }
#pragma unroll
      for (int e = 0; e < 8; ++e) s_part[warp][g].o[tl * 8 + e] = o_acc[g][e];
    }
  }
  __syncthreads();
  // merge the 4 warps into s_part[0]
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    float mx = -INFINITY;
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, s_part[w][g].m);
    float o = 0.f;
    for (int w = 0; w < 4; ++w)
      if (s_part[w][g].m != -INFINITY) o += s_part[w][g].o[c] * exp2f(s_part[w][g].m - mx);
    s_part[0][g].o[c] = o;  // each (g,c) read/written by one thread only
  }
  __syncthreads();
  if (tid < G) {
    const int g = tid;
    float mx = -INFINITY;
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, s_part[w][g].m);
    float l = 0.f;
    for (int w = 0; w < 4; ++w)
      if (s_part[w][g].m != -INFINITY) l += s_part[w][g].l * exp2f(s_part[w][g].m - mx);
    s_part[0][g].m = mx;
    s_part[0][g].l = l;
  }
  __syncthreads();

  const int unit = bi * Hkv + kh;
  if (S > 1) {
    // publish this split's state; the last CTA of the unit merges
    Partial<D, G>* gp = reinterpret_cast<Partial<D, G>*>(partials) + ((size_t)unit * S + sp) * G;
    for (int i = tid; i < G * D; i += kThreads) gp[i / D].o[i % D] = s_part[0][i / D].o[i % D];
    if (tid < G) { gp[tid].m = s_part[0][tid].m; gp[tid].l = s_part[0][tid].l; }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_flag = (atomicAdd(&counters[unit], 1) == S - 1);
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    if (tid == 0) counters[unit] = 0;
    // merge all splits (read through L2: written by other SMs)
    for (int i = tid; i < G * D; i += kThreads) {
      const int g = i / D, c = i % D;
      float mx = -INFINITY;
      for (int t = 0; t < S; ++t) mx = fmaxf(mx, __ldcg(&gp[(t - sp) * G + g].m));
      float o = 0.f;
      for (int t = 0; t < S; ++t) {
        const float mt = __ldcg(&gp[(t - sp) * G + g].m);
        if (mt != -INFINITY) o += __ldcg(&gp[(t - sp) * G + g].o[c]) * exp2f(mt - mx);
      }
      s_part[1][g].o[c] = o;
    }
    if (tid < G) {
      float mx = -INFINITY;
      for (int t = 0; t < S; ++t) mx = fmaxf(mx, __ldcg(&gp[(t - sp) * G + tid].m));
      float l = 0.f;
      for (int t = 0; t < S; ++t) {
        const float mt = __ldcg(&gp[(t - sp) * G + tid].m);
        if (mt != -INFINITY) l += __ldcg(&gp[(t - sp) * G + tid].l) * exp2f(mt - mx);
      }
      s_part[1][tid].l = l;
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += kThreads) s_part[0][i / D].o[i % D] = s_part[1][i / D].o[i % D];
    if (tid < G) s_part[0][tid].l = s_part[1][tid].l;
    __syncthreads();
  }

  // ---- memory readout: u = W_phi q, m = M^T u / (b . u + eps), g = sigmoid(w_gate . q)
  __shared__ float s_u[G][128];
  __shared__ float s_den[G], s_gate[G];
  const float* Mk = M + (size_t)unit * r * D;
  const float* bk = bstab + (size_t)unit * r;
  for (int i = tid; i < G * r; i += kThreads) {
    const int g = i / r, j = i % r;
    const float* wrow = W_phi + (size_t)j * D;
    float a = 0.f;
    for (int c = 0; c < D; ++c) a = fmaf(wrow[c], s_q[g][c], a);
    s_u[g][j] = a;
  }
  __syncthreads();
  if (warp < G) {
    const int g = warp;
    float a = 0.f;
    for (int j = lane; j < r; j += 32) a = fmaf(bk[j], s_u[g][j], a);
    a = warp_sum(a);
    float z = 0.f;
    const float* wg = w_gate + (size_t)(kh * G + g) * D;
    for (int c = lane; c < D; c += 32) z = fmaf(wg[c], s_q[g][c], z);
    z = warp_sum(z);
    if (lane == 0) {
      s_den[g] = a + eps;
      s_gate[g] = use_override ? gate_override : sigmoidf_(z);
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    float num = 0.f;
    for (int j = 0; j < r; ++j) num = fmaf(Mk[(size_t)j * D + c], s_u[g][j], num);
    const float oattn = s_part[0][g].o[c] / s_part[0][g].l;
    const float o = oattn + s_gate[g] * (num / s_den[g]);
    out[((size_t)bi * Hq + kh * G + g) * D + c] = Elem<T>::from_f(o);
  }

  // the last finished unit of the sequence advances cache_len
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    int* seq_cnt = counters + (size_t)gridDim.z * Hkv;
    if (atomicAdd(&seq_cnt[bi], 1) == Hkv - 1) {
      seq_cnt[bi] = 0;
      cache_len[bi] = len + 1;
    }
  }
}

template <typename T, int D>
cudaError_t launch_g(const Ctx& c, int G, dim3 grid, const void* q, const void* kn, const void* vn,
                     void* K_ret, void* V_ret, int32_t* cache_len, int cap, int rps,
                     const float* M, const float* bstab, void* out, float* partials,
                     int* counters, cudaStream_t st) {
  const int use_ov = !isnan(c.cfg.gate_override);
#define IMEM_DEC(GG)                                                                         \
  decode_kernel<T, D, GG><<<grid, kThreads, 0, st>>>(                                        \
      (const T*)q, (const T*)kn, (const T*)vn, (T*)K_ret, (T*)V_ret, cache_len, cap,         \
      c.cfg.n_kv_heads, rps, M, bstab, c.W_phi, c.w_gate, c.cfg.mem_r, c.cfg.eps,            \
      c.cfg.gate_override, use_ov, (T*)out, partials, counters, c.err)
  switch (G) {
    case 1: IMEM_DEC(1); break;
    case 2: IMEM_DEC(2); break;
    case 4: IMEM_DEC(4); break;
    case 8: IMEM_DEC(8); break;
    default: return cudaErrorInvalidValue;
  }
#undef IMEM_DEC
  return cudaGetLastError();
}

}  // namespace

int decode_splits(int batch, int n_kv_heads, int cap) {
  const int units = batch * n_kv_heads;
  int S = (2 * 148 + units - 1) / units;
  const int max_by_rows = (cap + 63) / 64;
  if (S > max_by_rows) S = max_by_rows;
  if (S > kDecodeMaxSplits) S = kDecodeMaxSplits;
  if (S < 1) S = 1;
  return S;
}

cudaError_t launch_decode(const Ctx& c, int batch, const void* q, const void* k_new,
                          const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                          int cap, const float* M, const float* bstab, void* out,
                          float* partials, int* counters, cudaStream_t st) {
  const int S = decode_splits(batch, c.cfg.n_kv_heads, cap);
  const int rps = (cap + S - 1) / S;
  dim3 grid(S, c.cfg.n_kv_heads, batch);
  const int D = c.cfg.head_dim;
  if (c.cfg.dtype == IMEM_BF16) {
    if (D == 128) return launch_g<__nv_bfloat16, 128>(c, c.group, grid, q, k_new, v_new, K_ret, V_ret, cache_len, cap, rps, M, bstab, out, partials, counters, st);
    if (D == 64) return launch_g<__nv_bfloat16, 64>(c, c.group, grid, q, k_new, v_new, K_ret, V_ret, cache_len, cap, rps, M, bstab, out, partials, counters, st);
  } else {
    if (D == 128) return launch_g<float, 128>(c, c.group, grid, q, k_new, v_new, K_ret, V_ret, cache_len, cap, rps, M, bstab, out, partials, counters, st);
    if (D == 64) return launch_g<float, 64>(c, c.group, grid, q, k_new, v_new, K_ret, V_ret, cache_len, cap, rps, M, bstab, out, partials, counters, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace imem
