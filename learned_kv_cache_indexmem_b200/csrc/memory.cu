// memory.cu -- latent-memory update from the evicted tokens.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B Mechanism (fast weights): the evicted tokens update online a
// fixed-size state matrix M and a stabiliser vector b by an outer-product
// accumulation with decay. With phi(k) = W_phi k and decay lambda per evicted
// token, in ascending position order:
//   M <- lambda M + phi(k) v^T,   b <- lambda b + phi(k)
// Over the n evicted tokens this equals
//   M = lambda^n M0 + W_phi S,  S = sum_i w_i k_i v_i^T,  w_i = lambda^(n-1-i)
//   b = lambda^n b0 + W_phi s,  s = sum_i w_i k_i
// (phi is linear), so disjoint runs of evicted tokens accumulate
// independently and W_phi is applied once at the end.
//
// Pass 1 (tensor cores): grid (groups, Hkv, batch); a CTA gathers the rows of
// one run [j0, j1) of evicted tokens for one (sequence, KV head) and
// accumulates
//   [S_g | s_g] (d x (d+1)) = K_c^T [w*V_c | w],  w_i = lambda^(j1-1-i)
// in tensor memory with tcgen05.mma over 64-token chunks. The weights are
// relative to the end of the run (the run's factor lambda^(n-j1) is applied
// in fp32 by pass 2), so they stay far from fp16's subnormal range for runs
// of moderate length. Operands are fp16 (bf16 keys convert exactly within
// fp16's range; w*v is rounded once to fp16) with fp32 accumulation; a key or
// weighted value beyond that range (|x| > 65504) is reported as DEV_RANGE.
// Both operands are MN-major in shared memory (a token is one 128-byte row per
// 64 features, so gathered rows are written as they arrive). Eight loader
// warps gather, convert and write the chunks; one thread issues the MMAs; a
// double-buffered mbarrier ring keeps them in step. An evicted index outside
// [0, L) reads no row and is reported as DEV_RANGE.
// Pass 2 (CUDA cores): per (sequence, KV head, 16 columns) sums the runs in a
// fixed order (deterministic), each scaled by its factor, and applies
// M = lambda^n M0 + W_phi S.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

#include <cuda_fp16.h>
#include <math.h>

namespace imem {
namespace {

constexpr int kLoaders = 256;            // 8 loader warps
constexpr int kMemThreads = kLoaders + 32;
constexpr int kChunk = 64;               // tokens per MMA chunk
constexpr int kStages = 2;

template <int D>
struct MemTile {
  static constexpr int A_ATOMS = 2;                    // M = 128 rows (d = 64 zero-padded)
  static constexpr int B_ATOMS = D / 64 + 1;           // d value columns + weight column
  static constexpr int N = D + 16;                     // MMA N
  static constexpr int A_BYTES = A_ATOMS * 8 * 1024;   // 8 K-groups of 8 tokens per atom column
  static constexpr int B_BYTES = B_ATOMS * 8 * 1024;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = kStages * STAGE + 1024 /*align*/ + 256 /*barriers*/;
};

// MN-major offset of (token jj in the chunk, 16-byte chunk cc of a feature row)
__device__ __forceinline__ uint32_t mn_off(int jj, int cc) {
  return (uint32_t)((cc >> 3) * 8192 + (jj >> 3) * 1024 + (jj & 7) * 128 +
                    ((((cc & 7) ^ (jj & 7))) << 4));
}

__device__ __forceinline__ uint4 to_half8(const float* f) {
  uint4 r;
  uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return r;
}

// Eight consecutive elements of a row, kept raw in registers until converted.
template <typename T> struct RawRow;
template <> struct RawRow<__nv_bfloat16> {
  using type = uint4;
  static __device__ __forceinline__ uint4 load(const __nv_bfloat16* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
  }
  static __device__ __forceinline__ uint4 zero() { return make_uint4(0, 0, 0, 0); }
  static __device__ __forceinline__ void to_f32(const uint4& v, float* f) { bf16x8_to_f32(v, f); }
};
struct F8 { float4 a, b; };
template <> struct RawRow<float> {
  using type = F8;
  static __device__ __forceinline__ F8 load(const float* p) {
    return F8{__ldcs(reinterpret_cast<const float4*>(p)), __ldcs(reinterpret_cast<const float4*>(p) + 1)};
  }
  static __device__ __forceinline__ F8 zero() {
    return F8{make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  }
  static __device__ __forceinline__ void to_f32(const F8& v, float* f) {
    f[0] = v.a.x; f[1] = v.a.y; f[2] = v.a.z; f[3] = v.a.w;
    f[4] = v.b.x; f[5] = v.b.y; f[6] = v.b.z; f[7] = v.b.w;
  }
};

template <typename T, int D, bool kSV>
__global__ void __launch_bounds__(kMemThreads, 2)
memory_tc_kernel(const T* __restrict__ K, const T* __restrict__ V, const int32_t* __restrict__ idx_e,
                 int n_e, int L, int Hkv, float log2lam, int tokens_per_group,
                 float* __restrict__ partials, float* __restrict__ sv_partials,
                 int* __restrict__ err) {
  using TL = MemTile<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * TL::STAGE);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_sv[8][16][8];   // per loader warp, per 16-byte column chunk: value sums

  const int g = blockIdx.x, kh = blockIdx.y, bi = blockIdx.z;
  const int G = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = g * tokens_per_group;
  const int j1 = min(n_e, j0 + tokens_per_group);
  const int nchunks = j1 > j0 ? (j1 - j0 + kChunk - 1) / kChunk : 0;
  const uint32_t sbase = tc::smem_addr(smem);
  const uint32_t full0 = tc::smem_addr(bars), empty0 = full0 + 8 * kStages,
                 done = full0 + 16 * kStages;

  // zero both stages once: padded rows of A and the unused weight columns stay 0
  for (int i = tid; i < kStages * TL::STAGE / 16; i += kMemThreads)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full0 + 8 * s, kLoaders);
      tc::mbar_init(empty0 + 8 * s, 1);
    }
    tc::mbar_init(done, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 8) {
    tc::tmem_alloc(tc::smem_addr(&s_tmem), 256);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = s_tmem;

  float* out = partials + (((size_t)bi * Hkv + kh) * G + g) * (size_t)D * (D + 1);

  if (warp < 8) {
    // ---------------- loaders: gather, convert, write MN-major fp16 rows
    constexpr int CH = D / 8;                       // 16-byte chunks per feature row
    constexpr int ITEMS = kChunk * CH / kLoaders;   // per thread per chunk
    const size_t row_stride = (size_t)Hkv * D;
    const T* Kb = K + (size_t)bi * L * row_stride + (size_t)kh * D;
    const T* Vb = V + (size_t)bi * L * row_stride + (size_t)kh * D;
    const int32_t* E = idx_e + (size_t)bi * n_e;
    // Software pipeline: the rows of chunk c+1 are in flight while chunk c is
    // converted and written; the evicted positions run one chunk further ahead.
    using Raw = RawRow<T>;
    typename Raw::type cur_k[ITEMS], cur_v[ITEMS], nxt_k[ITEMS], nxt_v[ITEMS];
    int pos_next[ITEMS];
    auto load_pos = [&](int c, int* pos) {
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int j = j0 + c * kChunk + (tid + it * kLoaders) / CH;
        int p = (c < nchunks && j < j1) ? __ldg(E + j) : -1;
        if (p >= L || (p < 0 && c < nchunks && j < j1)) {   // no row to read
          record_error(err, DEV_RANGE);
          p = -1;
        }
        pos[it] = p;
      }
    };
    auto load_rows = [&](const int* pos, typename Raw::type* kr, typename Raw::type* vr) {
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int cc = (tid + it * kLoaders) % CH;
        if (pos[it] >= 0) {
          kr[it] = Raw::load(Kb + (size_t)pos[it] * row_stride + cc * 8);
          vr[it] = Raw::load(Vb + (size_t)pos[it] * row_stride + cc * 8);
        } else {
          kr[it] = Raw::zero();
          vr[it] = Raw::zero();
        }
      }
    };
    // optional value sums sum_i w_i v_i: a thread's items all share the
    // column chunk tid % CH (kLoaders is a multiple of CH)
    static_assert(kLoaders % CH == 0, "fixed column chunk per loader thread");
    float svacc[kSV ? 8 : 1];
#pragma unroll
    for (int e = 0; e < (kSV ? 8 : 1); ++e) svacc[e] = 0.f;
    int pos_cur[ITEMS];
    load_pos(0, pos_cur);
    load_pos(1, pos_next);
    load_rows(pos_cur, cur_k, cur_v);
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % kStages;
      if (c + 1 < nchunks) {
        load_rows(pos_next, nxt_k, nxt_v);
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) pos_cur[it] = pos_next[it];
        load_pos(c + 2, pos_next);
      }
      if (c >= kStages && !tc::mbar_wait(empty0 + 8 * s, ((c / kStages) - 1) & 1)) {
        record_error(err, DEV_TIMEOUT);
        s_abort = 1;
        break;
      }
      unsigned char* a_p = smem + s * TL::STAGE;
      unsigned char* b_p = a_p + TL::A_BYTES;
      const int base = j0 + c * kChunk;
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int i = tid + it * kLoaders;
        const int jj = i / CH, cc = i % CH;
        const int j = base + jj;
        const float wv = (j < j1) ? exp2f((float)(j1 - 1 - j) * log2lam) : 0.f;
        float kf[8], vf[8];
        Raw::to_f32(cur_k[it], kf);
        Raw::to_f32(cur_v[it], vf);
        float big = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          vf[e] *= wv;
          big = fmaxf(big, fmaxf(fabsf(kf[e]), fabsf(vf[e])));
        }
        if (big > 65504.f) record_error(err, DEV_RANGE);   // beyond fp16's range
        if constexpr (kSV) {
#pragma unroll
          for (int e = 0; e < 8; ++e) svacc[e] += vf[e];
        }
        *reinterpret_cast<uint4*>(a_p + mn_off(jj, cc)) = to_half8(kf);
        *reinterpret_cast<uint4*>(b_p + mn_off(jj, cc)) = to_half8(vf);
        if (cc == 0)   // weight column: element 0 of the row in the last B atom
          *reinterpret_cast<__half*>(b_p + mn_off(jj, (D / 64) * 8)) = __float2half_rn(wv);
      }
      tc::fence_proxy_async();
      tc::mbar_arrive(full0 + 8 * s);
      if (c + 1 < nchunks) {
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) { cur_k[it] = nxt_k[it]; cur_v[it] = nxt_v[it]; }
      }
    }
    if constexpr (kSV) {
      // lanes with equal tid % CH hold the same columns: fold them, then the
      // 8 loader warps through shared memory (named barrier 1: loaders only)
#pragma unroll
      for (int off = CH; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) svacc[e] += __shfl_xor_sync(0xffffffffu, svacc[e], off);
      if (lane < CH) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s_sv[warp][lane][e] = svacc[e];
      }
      asm volatile("bar.sync 1, %0;\n" ::"n"(kLoaders) : "memory");
      if (tid < D) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) a += s_sv[w][tid / 8][tid % 8];
        sv_partials[(((size_t)bi * Hkv + kh) * G + g) * D + tid] = a;
      }
    }
  } else if (lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t IDESC = tc::idesc(tc::kFmtF16, 128, TL::N, true, true);
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % kStages;
      if (!tc::mbar_wait(full0 + 8 * s, (c / kStages) & 1)) {
        record_error(err, DEV_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc::fence_after();
      const uint32_t a_t = sbase + s * TL::STAGE, b_t = a_t + TL::A_BYTES;
#pragma unroll
      for (int k = 0; k < kChunk / 16; ++k) {   // 16 tokens = 2 K-groups per MMA
        const uint64_t ad = tc::sdesc_sw128(a_t + k * 2048, 8192, 1024);
        const uint64_t bd = tc::sdesc_sw128(b_t + k * 2048, 8192, 1024);
        tc::mma_f16(tmem, ad, bd, IDESC, (c > 0 || k > 0) ? 1u : 0u);
      }
      tc::mma_commit(empty0 + 8 * s);
    }
    tc::mma_commit(done);
  }

  // ---------------- epilogue: warps 0-3 read [S | s] rows from TMEM
  if (warp < 4) {
    const int row = warp * 32 + lane;   // feature index of k (TMEM lane)
    bool ok = true;
    if (nchunks > 0) ok = tc::mbar_wait(done, 0);
    if (!ok) record_error(err, DEV_TIMEOUT);
    tc::fence_after();
    if (nchunks > 0 && ok && !s_abort) {
      constexpr int NCOL = TL::N;   // multiple of 16
#pragma unroll 1
      for (int c0 = 0; c0 < NCOL; c0 += 16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
        if (row < D) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = c0 + e;
            if (col <= D) out[(size_t)row * (D + 1) + col] = v[e];
          }
        }
      }
    } else if (row < D) {
      for (int col = 0; col <= D; ++col) out[(size_t)row * (D + 1) + col] = 0.f;
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 8) tc::tmem_dealloc(tmem, 256);
}

// M[:, cols] = decay * M[:, cols] + W_phi * sum_g S_g[:, cols]; the extra
// column slice (blockIdx.x == D/16) does b from the s column.
// With sv_partials, slice D/16 + 1 does the value sums: s_v = decay * s_v +
// sum_g, and the sequence's count n_e += n_add (KV head 0 of the sequence).
// Run g covers evicted tokens [g*tpg, min(n, (g+1)*tpg)); its partial sums are
// weighted relative to its end, so it enters with the factor lambda^(n - end).
__device__ __forceinline__ float run_factor(int g, int tpg, int n, float log2lam) {
  const int end = min(n, (g + 1) * tpg);
  return exp2f((float)(n - end) * log2lam);
}

template <int D>
__global__ void __launch_bounds__(256)
memory_finalize_kernel(const float* __restrict__ partials, int G, int tpg, int n_tok,
                       float log2lam, const float* __restrict__ W_phi,
                       int r, float decay_n, float* __restrict__ M, float* __restrict__ bstab,
                       const float* __restrict__ sv_partials, float* __restrict__ s_v,
                       float* __restrict__ n_e, float n_add, int Hkv) {
  extern __shared__ float fsm[];
  __shared__ float s_fac[kMemMaxGroups];
  for (int gg = threadIdx.x; gg < G; gg += 256) s_fac[gg] = run_factor(gg, tpg, n_tok, log2lam);
  __syncthreads();
  if (blockIdx.x == D / 16 + 1) {   // value sums (only launched with sv_partials)
    const int unit = blockIdx.y;
    for (int c = threadIdx.x; c < D; c += 256) {
      float a = 0.f;
      for (int gg = 0; gg < G; ++gg)
        a = fmaf(s_fac[gg], __ldcg(&sv_partials[((size_t)unit * G + gg) * D + c]), a);
      float* sp = s_v + (size_t)unit * D + c;
      *sp = fmaf(*sp, decay_n, a);
    }
    if (threadIdx.x == 0 && unit % Hkv == 0) n_e[unit / Hkv] += n_add;
    return;
  }
  float* sW = fsm;                 // [r][D]
  float* sS = sW + r * D;          // [D][16]
  const int unit = blockIdx.y, sl = blockIdx.x;
  const int tid = threadIdx.x;
  const bool bcol = (sl == D / 16);
  const int ncols = bcol ? 1 : 16;
  const int col0 = bcol ? D : sl * 16;
  if (W_phi)   // null: the identity map (r == D)
    for (int i = tid; i < r * D / 4; i += 256)
      reinterpret_cast<float4*>(sW)[i] = __ldg(reinterpret_cast<const float4*>(W_phi) + i);
  const float* p = partials + (size_t)unit * G * D * (D + 1);
  for (int i = tid; i < D * ncols; i += 256) {
    const int dk = i / ncols, cc = i % ncols;
    float a = 0.f;
    for (int gg = 0; gg < G; ++gg)
      a = fmaf(s_fac[gg], __ldcg(&p[((size_t)gg * D + dk) * (D + 1) + col0 + cc]), a);
    sS[dk * 16 + cc] = a;
  }
  __syncthreads();
  for (int i = tid; i < r * ncols; i += 256) {
    const int ri = i / ncols, cc = i % ncols;
    float a = 0.f;
    if (W_phi) {
#pragma unroll 8
      for (int dk = 0; dk < D; ++dk) a = fmaf(sW[ri * D + dk], sS[dk * 16 + cc], a);
    } else {
      a = sS[ri * 16 + cc];
    }
    if (bcol) {
      float* bp = bstab + (size_t)unit * r + ri;
      *bp = fmaf(*bp, decay_n, a);
    } else {
      float* mp = M + ((size_t)unit * r + ri) * D + col0 + cc;
      *mp = fmaf(*mp, decay_n, a);
    }
  }
}

}  // namespace

// Number of runs the evicted tokens are split into per (sequence, KV head):
// about two CTAs per SM, each run a whole number of `chunk` tokens.
int memory_groups(int batch, int n_kv_heads, int n_e, int chunk) {
  const int units = batch * n_kv_heads;
  const int chunks = (n_e + chunk - 1) / chunk;
  int G = (2 * 148 + units / 2) / units;
  if (G > chunks) G = chunks;
  if (G > kMemMaxGroups) G = kMemMaxGroups;
  if (G < 1) G = 1;
  return G;
}

cudaError_t launch_memory_update(const Ctx& c, int batch, int L, const void* K, const void* V,
                                 const int32_t* idx_e, int n_e, int chunk, float* M, float* bstab,
                                 float* partials, float* sv_partials, float* s_v, float* n_count,
                                 cudaStream_t st) {
  if (n_e == 0) return cudaSuccess;
  const int Hkv = c.cfg.n_kv_heads, D = c.cfg.head_dim, r = c.cfg.mem_r;
  const int G = memory_groups(batch, Hkv, n_e, chunk);
  const int chunks = (n_e + chunk - 1) / chunk;
  const int tokens_per_group = ((chunks + G - 1) / G) * chunk;
  const int Gused = (n_e + tokens_per_group - 1) / tokens_per_group;   // no empty runs
  dim3 grid(Gused, Hkv, batch);
  const float log2lam = (float)log2((double)c.cfg.lambda);
  cudaError_t e = cudaSuccess;
#define IMEM_MEM(TT, DD)                                                                       \
  do {                                                                                         \
    auto kfn = sv_partials ? memory_tc_kernel<TT, DD, true> : memory_tc_kernel<TT, DD, false>; \
    e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,                 \
                             MemTile<DD>::SMEM);                                               \
    if (e != cudaSuccess) return e;                                                            \
    kfn<<<grid, kMemThreads, MemTile<DD>::SMEM, st>>>((const TT*)K, (const TT*)V, idx_e, n_e,  \
                                                      L, Hkv, log2lam, tokens_per_group,       \
                                                      partials, sv_partials, c.err);           \
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
  dim3 fgrid(D / 16 + 1 + (sv_partials ? 1 : 0), batch * Hkv);
  // moment statistics use the identity map: the finalize skips the product
  const float* phi = c.cfg.readout == IMEM_READOUT_MOMENT ? nullptr : c.W_phi;
  const size_t fsmem = ((size_t)r * D + (size_t)D * 16) * sizeof(float);
  if (D == 128) {
    e = cudaFuncSetAttribute(memory_finalize_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem);
    if (e != cudaSuccess) return e;
    memory_finalize_kernel<128><<<fgrid, 256, fsmem, st>>>(partials, Gused, tokens_per_group,
                                                           n_e, log2lam, phi, r, decay_n, M,
                                                           bstab, sv_partials, s_v, n_count,
                                                           (float)n_e, Hkv);
  } else {
    e = cudaFuncSetAttribute(memory_finalize_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem);
    if (e != cudaSuccess) return e;
    memory_finalize_kernel<64><<<fgrid, 256, fsmem, st>>>(partials, Gused, tokens_per_group,
                                                          n_e, log2lam, phi, r, decay_n, M,
                                                          bstab, sv_partials, s_v, n_count,
                                                          (float)n_e, Hkv);
  }
  return cudaGetLastError();
}

}  // namespace imem

// ---------------------------------------------------------------------------
// Memory update without any allocation.
//
// For callers that cannot allocate device memory at all -- for example code
// running where cudaMalloc is forbidden or would break the memory plan of a
// host framework (inside a pre-planned arena, or in a process whose device
// memory is owned by another allocator) -- imem_update_memory_static runs the
// same two kernels as imem_update_memory, but its scratch (the per-run partial
// sums [S | s]) lives in the fixed-size array below instead of a caller
// workspace, and it needs no context: the caller passes the dimensions, the
// decay and W_phi directly.
// ---------------------------------------------------------------------------
namespace imem {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)8 << 20;   // 8 MiB per device
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];
static __device__ int g_static_err;

// Device addresses of the scratch array and its error word in the context
// that is current now. Host code must not use the symbols themselves: they are
// host-side stand-ins, not device addresses. The lookup is repeated on every
// call (it allocates nothing): an address kept from an earlier call would be
// stale after cudaDeviceReset or in another context. The first lookup on a
// device loads the library's device code there if that has not happened yet,
// which is why the first call on a device belongs before any stream capture.
cudaError_t static_scratch(float** scratch, int** err) {
  void* p = nullptr;
  void* e = nullptr;
  cudaError_t r = cudaGetSymbolAddress(&p, g_static_scratch);
  if (r != cudaSuccess) return r;
  r = cudaGetSymbolAddress(&e, g_static_err);
  if (r != cudaSuccess) return r;
  *scratch = static_cast<float*>(p);
  *err = static_cast<int*>(e);
  return cudaSuccess;
}

template <typename T, int D>
cudaError_t launch_memory_static(int batch, int L, int Hkv, int r, float lambda, const void* K,
                                 const void* V, const int32_t* idx_e, int n_e, int chunk,
                                 const float* W_phi, float* M, float* bstab, float* scratch,
                                 int* err, cudaStream_t st) {
  const int units = batch * Hkv;
  const size_t psize = (size_t)D * (D + 1) * sizeof(float);
  int G = memory_groups(batch, Hkv, n_e, chunk);
  while (G > 1 && (size_t)units * G * psize > kStaticScratchBytes) --G;
  const int chunks = (n_e + chunk - 1) / chunk;
  const int tokens_per_group = ((chunks + G - 1) / G) * chunk;
  const int Gused = (n_e + tokens_per_group - 1) / tokens_per_group;
  const float log2lam = (float)log2((double)lambda);
  auto kfn = memory_tc_kernel<T, D, false>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       MemTile<D>::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<dim3(Gused, Hkv, batch), kMemThreads, MemTile<D>::SMEM, st>>>(
      (const T*)K, (const T*)V, idx_e, n_e, L, Hkv, log2lam, tokens_per_group, scratch, nullptr,
      err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float decay_n = (float)pow((double)lambda, (double)n_e);
  const size_t fsmem = ((size_t)r * D + (size_t)D * 16) * sizeof(float);
  e = cudaFuncSetAttribute(memory_finalize_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)fsmem);
  if (e != cudaSuccess) return e;
  memory_finalize_kernel<D><<<dim3(D / 16 + 1, units), 256, fsmem, st>>>(
      scratch, Gused, tokens_per_group, n_e, log2lam, W_phi, r, decay_n, M, bstab, nullptr,
      nullptr, nullptr, 0.f, Hkv);
  return cudaGetLastError();
}

}  // namespace
}  // namespace imem

extern "C" imem_status imem_update_memory_static(int batch, int L, int n_kv_heads, int head_dim,
                                                 int mem_r, float lambda, int dtype, const void* K,
                                                 const void* V, const int32_t* idx_evicted,
                                                 int n_evicted, int chunk, const float* W_phi,
                                                 float* M, float* bstab, void* stream) {
  using namespace imem;
  if (dtype != IMEM_FP32 && dtype != IMEM_BF16) return IMEM_ERR_INVALID_ARG;
  if (batch < 1 || L < 1 || n_kv_heads < 1) return IMEM_ERR_SHAPE;
  if (n_evicted < 0 || n_evicted > L) return IMEM_ERR_SHAPE;
  if (chunk < 64 || chunk % 64) return IMEM_ERR_SHAPE;
  if (!(lambda > 0.f && lambda <= 1.f)) return IMEM_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return IMEM_ERR_UNSUPPORTED;
  if (mem_r < 16 || mem_r % 16 || mem_r > 128) return IMEM_ERR_UNSUPPORTED;
  // the smallest split (one run per sequence and KV head) must fit the scratch
  if ((size_t)batch * n_kv_heads * head_dim * (head_dim + 1) * sizeof(float) > kStaticScratchBytes)
    return IMEM_ERR_UNSUPPORTED;
  const void* ptrs[] = {K, V, W_phi, M, bstab};
  for (const void* p : ptrs) {
    if (!p) return IMEM_ERR_INVALID_ARG;
    if ((uintptr_t)p & 15u) return IMEM_ERR_ALIGN;
  }
  if (n_evicted > 0) {
    if (!idx_evicted) return IMEM_ERR_INVALID_ARG;
    if ((uintptr_t)idx_evicted & 15u) return IMEM_ERR_ALIGN;
  }
  if (n_evicted == 0) return IMEM_OK;
  float* scratch = nullptr;
  int* err = nullptr;
  if (static_scratch(&scratch, &err) != cudaSuccess) return IMEM_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (dtype == IMEM_BF16)
    e = head_dim == 128 ? launch_memory_static<__nv_bfloat16, 128>(batch, L, n_kv_heads, mem_r, lambda, K, V, idx_evicted, n_evicted, chunk, W_phi, M, bstab, scratch, err, st)
                        : launch_memory_static<__nv_bfloat16, 64>(batch, L, n_kv_heads, mem_r, lambda, K, V, idx_evicted, n_evicted, chunk, W_phi, M, bstab, scratch, err, st);
  else
    e = head_dim == 128 ? launch_memory_static<float, 128>(batch, L, n_kv_heads, mem_r, lambda, K, V, idx_evicted, n_evicted, chunk, W_phi, M, bstab, scratch, err, st)
                        : launch_memory_static<float, 64>(batch, L, n_kv_heads, mem_r, lambda, K, V, idx_evicted, n_evicted, chunk, W_phi, M, bstab, scratch, err, st);
  return e == cudaSuccess ? IMEM_OK : IMEM_ERR_CUDA;
}

extern "C" imem_status imem_static_status(void* stream) {
  using namespace imem;
  float* scratch = nullptr;
  int* err = nullptr;
  if (static_scratch(&scratch, &err) != cudaSuccess) return IMEM_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return IMEM_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return IMEM_ERR_CUDA;
  }
  if (code == DEV_TIMEOUT) return IMEM_ERR_TIMEOUT;
  if (code == DEV_RANGE) return IMEM_ERR_RANGE;
  return IMEM_OK;
}
