// select.cu -- top-B retention and KV-cache compaction.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §1 (token eviction keeps the important tokens within a bounded
// budget and discards the rest) and §4 (experiments at 90% eviction); the
// retained set is one per (sequence, layer) because the indexer has a single
// shared key (§2.A).
//
// Selection: R = the B largest importances, ties to the lower position, with
// -0 and +0 equal. Each importance is mapped to an unsigned key that orders
// like the float; a 4-pass 8-bit radix select finds the B-th largest key T and
// how many keys equal to T are taken (the lowest positions), one CTA per
// sequence with eight loads in flight per thread. Then every warp
// counts the keys above and equal to T in its contiguous slice of positions,
// one scan over the warps gives each slice's offsets, and a second walk writes
// R and its complement E, both ascending.
//
// Compaction: K_ret[:, j] = K[:, R[j]] and V_ret likewise, all KV heads at
// once (one contiguous row of Hkv*d elements per token), 16-byte vectors.
//
// Pre-eviction during chunked prefill (§2.A: eviction before the whole
// prefix is processed): the same selection over the candidates of a query
// range (the retained tokens, then the range's tokens), then the retained
// candidates' indexer keys, importances and positions are compacted to the
// front of the candidate buffers and the evicted positions listed in order.
#include "common.cuh"
#include "internal.h"

#include <atomic>
#include <cooperative_groups.h>

namespace imem {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kUnroll = 8;   // keys loaded per thread before any is used

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float* __restrict__ I, int L, int stride, int B, int32_t* __restrict__ idx_r,
              int32_t* __restrict__ idx_e) {
  constexpr int kWarps = kSelThreads / 32;
  const int bi = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* Ib = I + (size_t)bi * stride;
  __shared__ int s_tot[256];            // digit histogram of the current pass
  __shared__ int s_cnt[2][kWarps];      // per warp: keys above T, keys equal to T
  __shared__ int s_base[2][kWarps];     // per warp: takes before it, equal keys before it
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_k;

  if (tid == 0) { s_prefix = 0; s_mask = 0; s_k = B; }
  // radix select of the B-th largest key, 8 bits a pass from the top
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) s_tot[tid] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    // kUnroll loads in flight per thread before any is used (one CTA streams
    // the whole row: latency, not bandwidth, is what limits it)
    for (int t0 = 0; t0 < L; t0 += kSelThreads * kUnroll) {
      float v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int t = t0 + u * kSelThreads + tid;
        v[u] = t < L ? Ib[t] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const uint32_t key = order_key(v[u]);
        if (t0 + u * kSelThreads + tid < L && (key & mask) == prefix)
          atomicAdd(&s_tot[(key >> shift) & 0xffu], 1);
      }
    }
    __syncthreads();
    if (tid < 32) {
      // find digit d (scanning from the top) where the running count reaches k
      const int k = s_k;
      // each lane sums 8 bins, top lanes first
      int local[8];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { local[i] = s_tot[255 - (tid * 8 + i)]; sum += local[i]; }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += n;
      }
      const int excl = incl - sum;
      if (excl < k && k <= incl) {  // exactly one lane
        int run = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run < k && k <= run + local[i]) {
            const uint32_t digit = 255u - (uint32_t)(tid * 8 + i);
            s_k = k - run;
            s_prefix = prefix | (digit << shift);
            s_mask = mask | (0xffu << shift);
          }
          run += local[i];
        }
      }
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;   // the B-th largest key
  const int take_eq = s_k;       // keys equal to T to retain (lowest positions)

  // ordered output: warp w owns the contiguous positions [w seg, (w+1) seg)
  const int seg = ((L + kWarps - 1) / kWarps + 31) & ~31;
  const int w0 = min(L, warp * seg), w1 = min(L, w0 + seg);
  int gt = 0, eq = 0;
  for (int t0 = w0; t0 < w1; t0 += 32 * kUnroll) {
    float v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = t0 + u * 32 + lane;
      v[u] = t < w1 ? Ib[t] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const bool in = t0 + u * 32 + lane < w1;
      const uint32_t key = order_key(v[u]);
      gt += __popc(__ballot_sync(0xffffffffu, in && key > T));
      eq += __popc(__ballot_sync(0xffffffffu, in && key == T));
    }
  }
  if (lane == 0) { s_cnt[0][warp] = gt; s_cnt[1][warp] = eq; }
  __syncthreads();
  if (warp == 0) {
    // equal keys before each warp, then each warp's takes and their prefix
    const int e = s_cnt[1][lane];
    int e_incl = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, e_incl, o);
      if (lane >= o) e_incl += n;
    }
    const int e_base = e_incl - e;
    const int takes = s_cnt[0][lane] + max(0, min(e, take_eq - e_base));
    int t_incl = takes;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t_incl, o);
      if (lane >= o) t_incl += n;
    }
    s_base[0][lane] = t_incl - takes;
    s_base[1][lane] = e_base;
  }
  __syncthreads();
  int before = s_base[0][warp], eq_seen = s_base[1][warp];
  const unsigned lt = (1u << lane) - 1u;
  for (int t0 = w0; t0 < w1; t0 += 32 * kUnroll) {
    float v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = t0 + u * 32 + lane;
      v[u] = t < w1 ? Ib[t] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = t0 + u * 32 + lane;
      const bool in = t < w1;
      const uint32_t key = order_key(v[u]);
      const bool is_eq = in && key == T;
      const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
      const bool take = in && (key > T || (is_eq && eq_seen + __popc(eqb & lt) < take_eq));
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      const int my = before + __popc(tb & lt);
      if (in) {
        if (take) idx_r[(size_t)bi * B + my] = t;
        else idx_e[(size_t)bi * (L - B) + (t - my)] = t;
      }
      before += __popc(tb);
      eq_seen += __popc(eqb);
    }
  }
}

// ---- the same selection over a thread-block cluster ---------------------------
// CTA `rank` of the cluster holds keys [rank * kpt * 1024, ...) in registers
// (warp w: the contiguous kpt * 32 positions from w * kpt * 32). Each radix
// pass builds a per-CTA histogram; after one cluster barrier every CTA sums
// all of them through distributed shared memory and picks the same digit
// (histograms double-buffered: a buffer is refilled two passes later, after
// every CTA's reads of it). Output: counts per warp and per CTA, one scan
// over the CTAs (shared memory of the others) and one over the warps.
constexpr int kCsMaxKpt = 16;
constexpr int kCsMaxCluster = 16;

__global__ void __launch_bounds__(kSelThreads, 1)
select_cluster_kernel(const float* __restrict__ I, int L, int stride, int B, int kpt,
                      int32_t* __restrict__ idx_r, int32_t* __restrict__ idx_e) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  constexpr int kWarps = kSelThreads / 32;
  const int CS = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int bi = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* Ib = I + (size_t)bi * stride;
  __shared__ int s_hist[2][256];
  __shared__ int s_tot[256];
  __shared__ int s_wcnt[2][kWarps];
  __shared__ int s_wbase[2][kWarps];
  __shared__ int s_cnt[2];                  // this CTA: keys above T, keys equal to T
  __shared__ int s_cbase[2];                // takes and equal keys before this CTA
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_k;

  const int w0 = rank * kpt * kSelThreads + warp * kpt * 32;   // this warp's first position
  uint32_t key[kCsMaxKpt];
  uint32_t valid = 0;
#pragma unroll
  for (int k = 0; k < kCsMaxKpt; ++k) {
    key[k] = 0u;
    const int t = w0 + k * 32 + lane;
    if (k < kpt && t < L) {
      key[k] = order_key(Ib[t]);
      valid |= 1u << k;
    }
  }
  if (tid == 0) { s_prefix = 0; s_mask = 0; s_k = B; }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass, buf = pass & 1;
    if (tid < 256) s_hist[buf][tid] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
#pragma unroll
    for (int k = 0; k < kCsMaxKpt; ++k)
      if ((valid >> k & 1u) && (key[k] & mask) == prefix)
        atomicAdd(&s_hist[buf][(key[k] >> shift) & 0xffu], 1);
    __syncthreads();
    cl.sync();   // every CTA's histogram of this pass is complete
    if (tid < 256) {
      int c = 0;
      for (int r = 0; r < CS; ++r) c += *cl.map_shared_rank(&s_hist[buf][tid], r);
      s_tot[tid] = c;
    }
    __syncthreads();
    if (tid < 32) {
      const int k = s_k;
      int local[8];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { local[i] = s_tot[255 - (tid * 8 + i)]; sum += local[i]; }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nn = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += nn;
      }
      const int excl = incl - sum;
      if (excl < k && k <= incl) {
        int run = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run < k && k <= run + local[i]) {
            const uint32_t digit = 255u - (uint32_t)(tid * 8 + i);
            s_k = k - run;
            s_prefix = prefix | (digit << shift);
            s_mask = mask | (0xffu << shift);
          }
          run += local[i];
        }
      }
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int take_eq = s_k;
  // counts of this warp's keys above and equal to T
  int gt = 0, eq = 0;
#pragma unroll
  for (int k = 0; k < kCsMaxKpt; ++k) {
    const bool in = valid >> k & 1u;
    gt += __popc(__ballot_sync(0xffffffffu, in && key[k] > T));
    eq += __popc(__ballot_sync(0xffffffffu, in && key[k] == T));
  }
  if (lane == 0) { s_wcnt[0][warp] = gt; s_wcnt[1][warp] = eq; }
  __syncthreads();
  if (warp == 0) {
    const int g = s_wcnt[0][lane], e = s_wcnt[1][lane];
    const int gs = __reduce_add_sync(0xffffffffu, g), es = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0) { s_cnt[0] = gs; s_cnt[1] = es; }
  }
  __syncthreads();
  cl.sync();   // every CTA's counts are visible
  if (warp == 0) {
    // equal keys and takes before this CTA, from the CTAs of lower rank
    const int r = lane;
    const int ge = r < CS ? *cl.map_shared_rank(&s_cnt[0], r) : 0;
    const int ee = r < CS ? *cl.map_shared_rank(&s_cnt[1], r) : 0;
    int e_incl = ee;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xffffffffu, e_incl, o);
      if (lane >= o) e_incl += nn;
    }
    const int e_base = e_incl - ee;
    const int takes = ge + max(0, min(ee, take_eq - e_base));
    int t_incl = takes;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xffffffffu, t_incl, o);
      if (lane >= o) t_incl += nn;
    }
    if (lane == rank) { s_cbase[0] = t_incl - takes; s_cbase[1] = e_base; }
  }
  __syncthreads();
  if (warp == 0) {
    // then the warps of this CTA, after the CTAs before it
    const int e = s_wcnt[1][lane];
    int e_incl = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xffffffffu, e_incl, o);
      if (lane >= o) e_incl += nn;
    }
    const int e_base = s_cbase[1] + e_incl - e;
    const int takes = s_wcnt[0][lane] + max(0, min(e, take_eq - e_base));
    int t_incl = takes;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xffffffffu, t_incl, o);
      if (lane >= o) t_incl += nn;
    }
    s_wbase[0][lane] = s_cbase[0] + t_incl - takes;
    s_wbase[1][lane] = e_base;
  }
  __syncthreads();
  int before = s_wbase[0][warp], eq_seen = s_wbase[1][warp];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kCsMaxKpt; ++k) {
    const int t = w0 + k * 32 + lane;
    const bool in = valid >> k & 1u;
    const bool is_eq = in && key[k] == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take = in && (key[k] > T || (is_eq && eq_seen + __popc(eqb & lt) < take_eq));
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int my = before + __popc(tb & lt);
    if (in) {
      if (take) idx_r[(size_t)bi * B + my] = t;
      else idx_e[(size_t)bi * (L - B) + (t - my)] = t;
    }
    before += __popc(tb);
    eq_seen += __popc(eqb);
  }
  cl.sync();   // no CTA leaves while another may read its shared memory
}

// One warp group per retained row: copies Hkv*d elements of K and V. Rows
// [0, n) of sequence bi come from positions idx_r[bi * idx_stride + j].
template <typename T>
__global__ void gather_kernel(const T* __restrict__ K, const T* __restrict__ V,
                              const int32_t* __restrict__ idx_r, T* __restrict__ K_ret,
                              T* __restrict__ V_ret, int L, int n, int idx_stride, int cap,
                              int row_elems, int rows_per_cta) {
  const int bi = blockIdx.y;
  const int vec = 16 / sizeof(T);
  const int nvec = row_elems / vec;
  for (int j = blockIdx.x * rows_per_cta; j < min(n, (blockIdx.x + 1) * rows_per_cta); ++j) {
    const int src = idx_r[(size_t)bi * idx_stride + j];
    const uint4* ks = reinterpret_cast<const uint4*>(K + ((size_t)bi * L + src) * row_elems);
    const uint4* vs = reinterpret_cast<const uint4*>(V + ((size_t)bi * L + src) * row_elems);
    uint4* kd = reinterpret_cast<uint4*>(K_ret + ((size_t)bi * cap + j) * row_elems);
    uint4* vd = reinterpret_cast<uint4*>(V_ret + ((size_t)bi * cap + j) * row_elems);
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
      kd[i] = __ldcs(ks + i);
      vd[i] = __ldcs(vs + i);
    }
  }
}

// ---- pre-eviction during chunked prefill ----------------------------------
// Candidate ci of a range is retained row ci (ci < n_R) or the range's token
// q0 + ci - n_R; candidate order is position order.
__device__ __forceinline__ int cand_pos(int ci, int n_R, int q0, const int32_t* ret_b) {
  return ci < n_R ? ret_b[ci] : q0 + ci - n_R;
}

constexpr int kRowsPerCompactCta = 32;   // 8 threads (16-byte chunks of a 128-byte key) per row

// Writes the selected candidates (idx_r), in position order, to rows [0, B)
// of the other candidate buffer and their positions to `retained`, and the
// evicted candidates' positions (idx_e, ascending) to `evicted`. It reads
// only the current buffer, so no row is overwritten before it is read.
__global__ void __launch_bounds__(256)
evict_compact_kernel(const int32_t* __restrict__ idx_r, const int32_t* __restrict__ idx_e, int B,
                     int n_ev, int n_R, int q0, int Lc, const int32_t* __restrict__ pos_c,
                     const __nv_bfloat16* __restrict__ kh_c, const float* __restrict__ I_c,
                     int32_t* __restrict__ pos_n, __nv_bfloat16* __restrict__ kh_n,
                     float* __restrict__ I_n, int32_t* __restrict__ retained,
                     int32_t* __restrict__ evicted) {
  const int bi = blockIdx.y;
  const int j = blockIdx.x * kRowsPerCompactCta + threadIdx.x / 8, c = threadIdx.x % 8;
  const int32_t* ret_b = pos_c + (size_t)bi * B;
  if (j < B) {
    const int ci = idx_r[(size_t)bi * B + j];
    const uint4* src = reinterpret_cast<const uint4*>(kh_c + ((size_t)bi * Lc + ci) * kIdxPad);
    reinterpret_cast<uint4*>(kh_n + ((size_t)bi * Lc + j) * kIdxPad)[c] = src[c];
    if (c == 0) {
      const int p = cand_pos(ci, n_R, q0, ret_b);
      pos_n[(size_t)bi * B + j] = p;
      retained[(size_t)bi * B + j] = p;
      I_n[(size_t)bi * Lc + j] = I_c[(size_t)bi * Lc + ci];
    }
  } else if (j < B + n_ev && c == 0) {
    const int e = j - B;
    evicted[(size_t)bi * n_ev + e] = cand_pos(idx_e[(size_t)bi * n_ev + e], n_R, q0, ret_b);
  }
}

__global__ void append_positions_kernel(int B, int n_R, int q0, int C, int32_t* __restrict__ retained,
                                        int32_t* __restrict__ pos) {
  const int bi = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < C) {
    retained[(size_t)bi * B + n_R + i] = q0 + i;
    pos[(size_t)bi * B + n_R + i] = q0 + i;
  }
}

// Selection of the B largest of L importances per sequence (stride between
// sequences): a cluster per sequence when the keys fit its registers, one
// CTA per sequence otherwise.
cudaError_t launch_select(int batch, const float* I, int L, int stride, int B, int32_t* idx_r,
                          int32_t* idx_e, cudaStream_t st) {
  int CS = (L + 4095) / 4096;
  if (CS < 1) CS = 1;
  if (CS > kCsMaxCluster) CS = kCsMaxCluster;
  const int kpt = (L + CS * kSelThreads - 1) / (CS * kSelThreads);
  if (kpt > kCsMaxKpt) {
    select_kernel<<<batch, kSelThreads, 0, st>>>(I, L, stride, B, idx_r, idx_e);
    return cudaGetLastError();
  }
  static std::atomic<uint64_t> attr_done{0};   // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    e = cudaFuncSetAttribute(select_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, batch, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_cluster_kernel, I, L, stride, B, kpt, idx_r, idx_e);
}

}  // namespace

cudaError_t launch_evict_chunk(const Ctx& c, int batch, int B, int Lc, int n_R, int q0, int C,
                               const EvictBuffers& w, int32_t* retained, int32_t* evicted,
                               cudaStream_t st) {
  (void)c;
  const int n = n_R + C, n_ev = n - B;
  if (n_ev <= 0) return cudaErrorInvalidValue;
  cudaError_t e = launch_select(batch, w.I_c, n, Lc, B, w.idx_r, w.idx_e, st);
  if (e != cudaSuccess) return e;
  dim3 g1((B + n_ev + kRowsPerCompactCta - 1) / kRowsPerCompactCta, batch);
  evict_compact_kernel<<<g1, 256, 0, st>>>(w.idx_r, w.idx_e, B, n_ev, n_R, q0, Lc, w.pos_c,
                                           w.kh_c, w.I_c, w.pos_n, w.kh_n, w.I_n, retained,
                                           evicted);
  return cudaGetLastError();
}

cudaError_t launch_append_positions(int batch, int B, int n_R, int q0, int C, int32_t* retained,
                                    int32_t* pos, cudaStream_t st) {
  if (C <= 0) return cudaSuccess;
  dim3 g((C + 255) / 256, batch);
  append_positions_kernel<<<g, 256, 0, st>>>(B, n_R, q0, C, retained, pos);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Ctx& c, int batch, int L, int n, const int32_t* idx,
                          int idx_stride, const void* K, const void* V, void* K_ret, void* V_ret,
                          int cap, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int row_elems = c.cfg.n_kv_heads * c.cfg.head_dim;
  const int rows_per_cta = 4;
  dim3 grid((n + rows_per_cta - 1) / rows_per_cta, batch);
  if (c.cfg.dtype == IMEM_BF16)
    gather_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
        (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx, (__nv_bfloat16*)K_ret,
        (__nv_bfloat16*)V_ret, L, n, idx_stride, cap, row_elems, rows_per_cta);
  else
    gather_kernel<float><<<grid, 128, 0, st>>>((const float*)K, (const float*)V, idx,
                                               (float*)K_ret, (float*)V_ret, L, n, idx_stride,
                                               cap, row_elems, rows_per_cta);
  return cudaGetLastError();
}

cudaError_t launch_select_compact(const Ctx& c, int batch, int L, int B, const float* running_max,
                                  const void* K, const void* V, int32_t* idx_r, int32_t* idx_e,
                                  void* K_ret, void* V_ret, int cap, void* /*scratch*/,
                                  cudaStream_t st) {
  cudaError_t e = launch_select(batch, running_max, L, L, B, idx_r, idx_e, st);
  if (e != cudaSuccess) return e;
  return launch_gather(c, batch, L, B, idx_r, B, K, V, K_ret, V_ret, cap, st);
}

}  // namespace imem
