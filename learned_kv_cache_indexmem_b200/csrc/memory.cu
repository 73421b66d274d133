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
// weighted value beyond that range (|x| >= 65520, which rounds to infinity)
// is reported as DEV_RANGE.
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

// Programmatic dependent launch: the finalize is launched while the
// tensor-core pass finishes; it stages W_phi, then waits for that pass.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

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

// Nonzero if one of the eight fp16 values is an infinity (a finite input that
// rounded beyond fp16's largest finite value, 65504).
__device__ __forceinline__ uint32_t half8_has_inf(const uint4& h) {
  const uint32_t w[4] = {h.x, h.y, h.z, h.w};
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) r |= __vcmpeq2(w[i] & 0x7fff7fffu, 0x7c007c00u);
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
__global__ void __maxnreg__(112)
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

  // head-major grid: the KV heads of one run are neighbours in launch order, so
  // they stream through the same token rows at about the same time
  const int kh = blockIdx.x, g = blockIdx.y, bi = blockIdx.z;
  const int G = gridDim.y;
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
    // bad: an evicted index outside [0, L) (its row is not read) or an
    // operand fp16 cannot hold was met; reported once after the loop
    uint32_t bad = 0;
    auto load_pos = [&](int c, int* pos) {
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int j = j0 + c * kChunk + (tid + it * kLoaders) / CH;
        int p = -1;
        if (c < nchunks && j < j1) {
          p = __ldg(E + j);
          if ((unsigned)p >= (unsigned)L) { bad = 1u; p = -1; }
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
#pragma unroll
        for (int e = 0; e < 8; ++e) vf[e] *= wv;
        if constexpr (kSV) {
#pragma unroll
          for (int e = 0; e < 8; ++e) svacc[e] += vf[e];
        }
        const uint4 hk = to_half8(kf), hv = to_half8(vf);
        bad |= half8_has_inf(hk) | half8_has_inf(hv);   // |x| >= 65520: beyond fp16
        *reinterpret_cast<uint4*>(a_p + mn_off(jj, cc)) = hk;
        *reinterpret_cast<uint4*>(b_p + mn_off(jj, cc)) = hv;
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
    if (bad) record_error(err, DEV_RANGE);
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

  // ---------------- epilogue: warps 0-3 read [S | s] rows from TMEM and store
  // them transposed (column c of the run's sum = D consecutive floats), so
  // that a warp's stores cover 128 contiguous bytes
  pdl_launch();   // the finalize may start staging W_phi (it waits for this grid)
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
            if (col <= D) out[(size_t)col * D + row] = v[e];
          }
        }
      }
    } else if (row < D) {
      for (int col = 0; col <= D; ++col) out[(size_t)col * D + row] = 0.f;
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 8) tc::tmem_dealloc(tmem, 256);
}

// M[:, cols] = decay * M[:, cols] + W_phi * sum_g S_g[:, cols] for 16
// columns a CTA; the extra column slice (blockIdx.x == D / 16) does b from
// the s column. With sv_partials, slice D / 16 + 1 does the value sums: s_v = decay * s_v +
// sum_g, and the sequence's count n_e += n_add (KV head 0 of the sequence).
// Run g covers evicted tokens [g*tpg, min(n, (g+1)*tpg)); its partial sums are
// weighted relative to its end, so it enters with the factor lambda^(n - end).
constexpr int kFinRuns = 12;   // runs' column slices a finalize CTA holds in shared memory at once

// dynamic shared memory of the finalize: S's padded columns and the run slices
inline size_t fin_smem(int D, int G) {
  return ((size_t)16 * (D + 16) + (size_t)(G < kFinRuns ? G : kFinRuns) * 16 * D) * sizeof(float);
}

__device__ __forceinline__ void fin_cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ float run_factor(int g, int tpg, int n, float log2lam) {
  const int end = min(n, (g + 1) * tpg);
  return exp2f((float)(n - end) * log2lam);
}

template <int D>
__global__ void __launch_bounds__(256, 2)
memory_finalize_kernel(const float* __restrict__ partials, int G, int tpg, int n_tok,
                       float log2lam, const float* __restrict__ W_phi,
                       int r, float decay_n, float* __restrict__ M, float* __restrict__ bstab,
                       const float* __restrict__ sv_partials, float* __restrict__ s_v,
                       float* __restrict__ n_e, float n_add, int Hkv, int* __restrict__ clear_tags,
                       int n_clear) {
  extern __shared__ float fsm[];
  __shared__ float s_fac[kMemMaxGroups];
  // the decode tags (no kernel of the update reads them; every earlier
  // reader has completed)
  if (clear_tags && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < n_clear; i += 256) clear_tags[i] = 0;
  for (int gg = threadIdx.x; gg < G; gg += 256) s_fac[gg] = run_factor(gg, tpg, n_tok, log2lam);
  __syncthreads();
  if (blockIdx.x == D / 16 + 1) {   // value sums (only launched with sv_partials)
    const int unit = blockIdx.y;
    pdl_wait();
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
  constexpr int BD = D / 4;        // a thread's block of d_k
  constexpr int SST = D + 16;      // padded column stride of sS: the four d_k blocks of a
                                   // column start in different banks
  float* sS = fsm;                 // [16][SST]: column c of S, d_k block b at b * (BD + 4)
  float* sP = fsm + 16 * SST;      // [kFinRuns][16 * D]: the runs' column slices as stored
  const int unit = blockIdx.y, sl = blockIdx.x;
  const int tid = threadIdx.x;
  const bool bcol = (sl == D / 16);
  const int ncols = bcol ? 1 : 16;
  const int col0 = bcol ? D : sl * 16;
  // product: thread (row rl of a pass of 64 rows, d_k block b) keeps its
  // W_phi block in registers; the four blocks of a row are neighbouring lanes
  // and meet by shuffles; lane b then writes columns 4b..4b+3 of the row
  const int b = tid & 3, rl = tid >> 2;
  float w[BD];
  float4 old = make_float4(0.f, 0.f, 0.f, 0.f);
  // the pass's W_phi blocks and old values (M and b are not written by the
  // tensor-core pass, and every earlier write to them has completed, so pass
  // 0 reads them before the wait)
  auto load_pass = [&](int pass) {
    const int ri = pass * 64 + rl;
    if (ri >= r) return;
    if (W_phi) {
#pragma unroll
      for (int j = 0; j < BD / 4; ++j) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(W_phi + (size_t)ri * D + b * BD) + j);
        w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
      }
    }
    if (bcol) old.x = bstab[(size_t)unit * r + ri];
    else old = *reinterpret_cast<const float4*>(M + ((size_t)unit * r + ri) * D + col0 + 4 * b);
  };
  load_pass(0);
  pdl_wait();
  // sum of the runs: up to kFinRuns runs' slices at once into shared memory
  // (cp.async: one round trip), then each item summed in run order
  const float* p = partials + (size_t)unit * G * D * (D + 1) + (size_t)col0 * D;
  const int pieces = ncols * D / 4;   // 16-byte pieces of a run's slice
  constexpr int IPT = 16 * D / 256;
  float acc[IPT];
#pragma unroll
  for (int k = 0; k < IPT; ++k) acc[k] = 0.f;
  for (int g0 = 0; g0 < G; g0 += kFinRuns) {
    const int nb = min(kFinRuns, G - g0);
    for (int k = tid; k < nb * pieces; k += 256) {
      const int u = k / pieces, pc = k % pieces;
      fin_cp_async16(tc::smem_addr(sP + (size_t)u * 16 * D + 4 * pc),
                     p + (size_t)(g0 + u) * D * (D + 1) + 4 * pc);
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    for (int u = 0; u < nb; ++u) {
      const float f = s_fac[g0 + u];
#pragma unroll
      for (int k = 0; k < IPT; ++k) {
        const int i = tid + k * 256;   // column i / D, row i % D
        if (i < ncols * D) acc[k] = fmaf(f, sP[(size_t)u * 16 * D + i], acc[k]);
      }
    }
    __syncthreads();   // the next batch rewrites sP
  }
#pragma unroll
  for (int k = 0; k < IPT; ++k) {
    const int i = tid + k * 256;
    if (i < ncols * D) {
      const int c = i / D, dk = i % D;
      sS[c * SST + dk + 4 * (dk / BD)] = acc[k];
    }
  }
  __syncthreads();
  const int npass = (r + 63) / 64;
  for (int pass = 0; pass < npass; ++pass) {
    if (pass > 0) load_pass(pass);
    const int ri = pass * 64 + rl;
    if (ri >= r) break;   // r is a multiple of 16: whole warps
    float a[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) a[c] = 0.f;
    if (W_phi) {
      const float* s0 = sS + b * (BD + 4);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        if (c < ncols) {
#pragma unroll
          for (int j = 0; j < BD / 4; ++j) {
            const float4 s4 = *reinterpret_cast<const float4*>(s0 + c * SST + 4 * j);
            a[c] = fmaf(w[4 * j], s4.x, a[c]);
            a[c] = fmaf(w[4 * j + 1], s4.y, a[c]);
            a[c] = fmaf(w[4 * j + 2], s4.z, a[c]);
            a[c] = fmaf(w[4 * j + 3], s4.w, a[c]);
          }
          a[c] += __shfl_xor_sync(0xffffffffu, a[c], 1);
          a[c] += __shfl_xor_sync(0xffffffffu, a[c], 2);
        }
      }
    } else {   // identity map: row ri of M takes row ri of S
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (c < ncols) a[c] = sS[c * SST + ri + 4 * (ri / BD)];
    }
    if (bcol) {
      if (b == 0) bstab[(size_t)unit * r + ri] = fmaf(old.x, decay_n, a[0]);
    } else {
      // columns 4b..4b+3 (selects keep a[] in registers)
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = b == 0 ? a[e] : b == 1 ? a[4 + e] : b == 2 ? a[8 + e] : a[12 + e];
      float4 v = old;
      v.x = fmaf(v.x, decay_n, o[0]); v.y = fmaf(v.y, decay_n, o[1]);
      v.z = fmaf(v.z, decay_n, o[2]); v.w = fmaf(v.w, decay_n, o[3]);
      *reinterpret_cast<float4*>(M + ((size_t)unit * r + ri) * D + col0 + 4 * b) = v;
    }
  }
}

// ---------------------------------------------------------------------------
// bf16 inputs: the same run sums [S_g | s_g] = (w K_c)^T [V_c | 1] with the
// rows gathered by cp.async straight into the operand layouts of the MMA, so
// that many chunks of rows are in flight per SM without registers:
//   A = (w k)^T, the decay weight applied to the key and split into two bf16
//       halves hi = bf16(w k), lo = bf16(w k - hi) (two MMAs into the same
//       accumulator; about 16 mantissa bits, fp32's range: no fp16 limit);
//       a key row lands in the A_hi buffer and is rewritten there in place;
//   B = [v | 1], the value row as loaded (bf16 is exact) and a column of
//       ones written once, which makes s = sum w k fall out of the same MMA.
// Chunks of 32 tokens; a ring of kBfStages stages; each loader thread keeps
// kBfAhead chunks in flight ahead of the one it converts, so that a stage is
// refilled kBfStages - kBfAhead chunks after its conversion (the MMAs of that
// chunk have long finished: the loaders rarely wait for them). Two CTAs per
// SM (each with its own ring and accumulator): at c2 shapes a 3-stage ring with
// one chunk ahead measured faster than a 7-stage ring with five ahead at one
// CTA per SM (75.9 vs 94.2 us for the stage). The run's evicted positions are
// read into shared memory once (runs of at most kRunMax tokens).
constexpr int kBfChunk = 32;
constexpr int kBfStages = 3;
constexpr int kBfAhead = 1;
constexpr int kBfLoaders = 256;   // loader threads (at most one 16-byte item each per chunk)
constexpr int kBfCtasPerSm = 2;
constexpr int kRunMax = 4096;

template <int D>
struct BfTile {
  static constexpr int KG = kBfChunk / 8;                // 8-token K groups per chunk
  static constexpr int ATOM_COL = KG * 1024;             // one 64-element MN block
  static constexpr int A_BYTES = 2 * ATOM_COL;           // M = 128 (d = 64 zero-padded)
  static constexpr int B_ATOMS = D / 64 + 1;             // value columns + the ones column
  static constexpr int B_BYTES = B_ATOMS * ATOM_COL;
  static constexpr int N = D + 16;
  static constexpr int STAGE = 2 * A_BYTES + B_BYTES;    // A_hi | A_lo | B
  static constexpr int SMEM = kBfStages * STAGE + kRunMax * 4 + 1024 + 256;
};

// loader threads and the block size (+ the MMA warp) of the bf16 kernel
template <int D> constexpr int bf_loaders() {
  return kBfChunk * (D / 8) < kBfLoaders ? kBfChunk * (D / 8) : kBfLoaders;
}
template <int D> constexpr int bf_threads() { return bf_loaders<D>() + 32; }

__device__ __forceinline__ uint32_t bf_off(int jj, int cc, int atom_col) {
  return (uint32_t)((cc >> 3) * atom_col + (jj >> 3) * 1024 + (jj & 7) * 128 +
                    (((cc & 7) ^ (jj & 7)) << 4));
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0: zero-fill the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(bf_threads<D>(), kBfCtasPerSm)
memory_bf16_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                   const int32_t* __restrict__ idx_e, int n_e, int L, int Hkv, float log2lam,
                   int tokens_per_run, float* __restrict__ partials, int* __restrict__ err) {
  using TL = BfTile<D>;
  constexpr int NL = bf_loaders<D>(), NT = NL + 32;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* s_pos = reinterpret_cast<int*>(smem + kBfStages * TL::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_pos + kRunMax);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  // head-major grid: the KV heads of one run are neighbours in launch order, so
  // they stream through the same token rows at about the same time
  const int kh = blockIdx.x, g = blockIdx.y, bi = blockIdx.z;
  const int G = gridDim.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = g * tokens_per_run;
  const int j1 = min(n_e, j0 + tokens_per_run);
  const int ntok = max(0, j1 - j0);
  const int nchunks = (ntok + kBfChunk - 1) / kBfChunk;
  const uint32_t sbase = tc::smem_addr(smem);
  const uint32_t full0 = tc::smem_addr(bars), empty0 = full0 + 8 * kBfStages,
                 done = full0 + 16 * kBfStages;

  // zero what no copy or conversion writes: the last atom column of B (the
  // ones column and the padding columns) and, for d = 64, the upper half of
  // A's rows in both key buffers; then the ones column of B (element 0 of the
  // first 16-byte chunk of that atom column)
  {
    constexpr int ATOM16 = TL::ATOM_COL / 16;             // 16-byte chunks per atom column
    constexpr int REGIONS = 1 + (D == 64 ? 2 : 0);
    for (int i = tid; i < kBfStages * REGIONS * ATOM16; i += NT) {
      const int st = i / (REGIONS * ATOM16), k = i % (REGIONS * ATOM16);
      const int region = k / ATOM16, o = k % ATOM16;
      const uint32_t off = region == 0 ? 2 * TL::A_BYTES + (TL::B_ATOMS - 1) * TL::ATOM_COL
                                       : (region - 1) * TL::A_BYTES + TL::ATOM_COL;
      reinterpret_cast<uint4*>(smem + st * TL::STAGE + off)[o] = make_uint4(0, 0, 0, 0);
    }
  }
  __syncthreads();
  for (int i = tid; i < kBfStages * kBfChunk; i += NT) {
    const int st = i / kBfChunk, jj = i % kBfChunk;
    *reinterpret_cast<__nv_bfloat16*>(smem + st * TL::STAGE + 2 * TL::A_BYTES +
                                      bf_off(jj, (D / 64) * 8, TL::ATOM_COL)) =
        __float2bfloat16_rn(1.f);
  }
  // the run's evicted positions (-1: no row: past the run, or out of range),
  // all of a thread's loads issued before its stores (one round trip)
  uint32_t bad = 0;
  const int32_t* E = idx_e + (size_t)bi * n_e + j0;
  {
    constexpr int PP = (kRunMax + NT - 1) / NT;
    int pv[PP];
#pragma unroll
    for (int k = 0; k < PP; ++k) {
      const int i = tid + k * NT;
      pv[k] = i < ntok ? __ldg(E + i) : -1;
    }
#pragma unroll
    for (int k = 0; k < PP; ++k) {
      const int i = tid + k * NT;
      if (i < nchunks * kBfChunk) {
        int p = pv[k];
        if (i < ntok && (unsigned)p >= (unsigned)L) { bad = 1u; p = -1; }
        s_pos[i] = p;
      }
    }
  }
  if (tid == 0) {
    for (int st = 0; st < kBfStages; ++st) {
      tc::mbar_init(full0 + 8 * st, NL);
      tc::mbar_init(empty0 + 8 * st, 1);
    }
    tc::mbar_init(done, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == NL / 32) {
    tc::tmem_alloc(tc::smem_addr(&s_tmem), 256);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = s_tmem;
  float* out = partials + (((size_t)bi * Hkv + kh) * G + g) * (size_t)D * (D + 1);

  if (warp < NL / 32) {
    // ---------------- loaders
    constexpr int CH = D / 8;                          // 16-byte chunks per row
    constexpr int ITEMS = kBfChunk * CH / NL;    // per thread per chunk (K and V each)
    static_assert(ITEMS >= 1 && kBfChunk * CH % NL == 0, "whole items per thread");
    const size_t row_stride = (size_t)Hkv * D;
    const __nv_bfloat16* Kb = K + (size_t)bi * L * row_stride + (size_t)kh * D;
    const __nv_bfloat16* Vb = V + (size_t)bi * L * row_stride + (size_t)kh * D;
    auto issue = [&](int c) {
      const uint32_t a = sbase + (uint32_t)((c % kBfStages) * TL::STAGE);
      const uint32_t b = a + 2 * TL::A_BYTES;
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int i = tid + it * NL, jj = i / CH, cc = i % CH;
        const int p = s_pos[c * kBfChunk + jj];
        const size_t off = (size_t)(p < 0 ? 0 : p) * row_stride + cc * 8;
        const uint32_t o = bf_off(jj, cc, TL::ATOM_COL);
        cp_async16_zfill(a + o, Kb + off, p >= 0);
        cp_async16_zfill(b + o, Vb + off, p >= 0);
      }
    };
    // exactly kBfAhead groups first (empty past the run's end), one per
    // iteration after: group k then holds chunk k, and waiting until at most
    // kBfAhead groups are pending at iteration c means chunk c has landed
    for (int c = 0; c < kBfAhead; ++c) {
      if (c < nchunks) issue(c);
      cp_async_commit_group();
    }
    for (int c = 0; c < nchunks; ++c) {
      const int cn = c + kBfAhead;
      if (cn < nchunks) {
        // its stage last held chunk cn - kBfStages: wait for that chunk's MMAs
        if (cn >= kBfStages &&
            !tc::mbar_wait(empty0 + 8 * (cn % kBfStages), ((cn / kBfStages) - 1) & 1)) {
          record_error(err, DEV_TIMEOUT);
          s_abort = 1;
          break;
        }
        issue(cn);
      }
      cp_async_commit_group();          // (possibly empty) keeps the group count uniform
      cp_async_wait_group<kBfAhead>();  // this thread's copies of chunk c have landed
      // A: the key rows this thread copied, scaled by the decay weight and
      // split into hi (in place) and lo
      unsigned char* a_p = smem + (c % kBfStages) * TL::STAGE;
#pragma unroll
      for (int it = 0; it < ITEMS; ++it) {
        const int i = tid + it * NL, jj = i / CH, cc = i % CH;
        const int j = j0 + c * kBfChunk + jj;
        const float w = j < j1 ? exp2f((float)(j1 - 1 - j) * log2lam) : 0.f;
        const uint32_t o = bf_off(jj, cc, TL::ATOM_COL);
        const uint4 raw = *reinterpret_cast<const uint4*>(a_p + o);
        float kf[8];
        bf16x8_to_f32(raw, kf);
        uint4 hi, lo;
        uint32_t* hw = reinterpret_cast<uint32_t*>(&hi);
        uint32_t* lw = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = w * kf[2 * e], x1 = w * kf[2 * e + 1];
          const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
          const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
          hw[e] = *reinterpret_cast<const uint32_t*>(&h);
          lw[e] = *reinterpret_cast<const uint32_t*>(&l);
        }
        *reinterpret_cast<uint4*>(a_p + o) = hi;
        *reinterpret_cast<uint4*>(a_p + TL::A_BYTES + o) = lo;
      }
      tc::fence_proxy_async();   // generic-proxy shared writes (and landed copies) -> MMA
      tc::mbar_arrive(full0 + 8 * (c % kBfStages));
    }
    cp_async_wait_group<0>();   // nothing of this thread in flight past here
    if (bad) record_error(err, DEV_RANGE);
  } else if (lane == 0) {
    // ---------------- MMA issuer: 2 x (16-token steps) x (hi, lo) per chunk
    constexpr uint32_t IDESC = tc::idesc(tc::kFmtBF16, 128, TL::N, true, true);
    for (int c = 0; c < nchunks; ++c) {
      const int st = c % kBfStages;
      if (!tc::mbar_wait(full0 + 8 * st, (c / kBfStages) & 1)) {
        record_error(err, DEV_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc::fence_after();
      const uint32_t a_t = sbase + st * TL::STAGE, b_t = a_t + 2 * TL::A_BYTES;
#pragma unroll
      for (int k = 0; k < kBfChunk / 16; ++k) {
        const uint64_t bd = tc::sdesc_sw128(b_t + k * 2048, TL::ATOM_COL, 1024);
        const uint64_t ah = tc::sdesc_sw128(a_t + k * 2048, TL::ATOM_COL, 1024);
        const uint64_t al = tc::sdesc_sw128(a_t + TL::A_BYTES + k * 2048, TL::ATOM_COL, 1024);
        tc::mma_f16(tmem, ah, bd, IDESC, (c > 0 || k > 0) ? 1u : 0u);
        tc::mma_f16(tmem, al, bd, IDESC, 1u);
      }
      tc::mma_commit(empty0 + 8 * st);
    }
    tc::mma_commit(done);
  }

  // ---------------- epilogue: warps 0-3 read [S | s] rows from TMEM and store
  // them transposed (column c of the run's sum = D consecutive floats), so
  // that a warp's stores cover 128 contiguous bytes
  pdl_launch();
  if (warp < 4) {
    const int row = warp * 32 + lane;   // feature index of k (TMEM lane)
    bool ok = true;
    if (nchunks > 0) ok = tc::mbar_wait(done, 0);
    if (!ok) record_error(err, DEV_TIMEOUT);
    tc::fence_after();
    if (nchunks > 0 && ok && !s_abort) {
#pragma unroll 1
      for (int c0 = 0; c0 < TL::N; c0 += 16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
        if (row < D) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = c0 + e;
            if (col <= D) out[(size_t)col * D + row] = v[e];
          }
        }
      }
    } else if (row < D) {
      for (int col = 0; col <= D; ++col) out[(size_t)col * D + row] = 0.f;
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == NL / 32) tc::tmem_dealloc(tmem, 256);
}

// Launches the finalize with programmatic stream serialization (it waits for
// the tensor-core pass itself, after staging W_phi).
template <int D>
cudaError_t launch_finalize(dim3 grid, size_t smem, cudaStream_t st, const float* partials, int G,
                            int tpg, int n_tok, float log2lam, const float* W_phi, int r,
                            float decay_n, float* M, float* bstab, const float* sv_partials,
                            float* s_v, float* n_count, float n_add, int Hkv,
                            int* clear_tags = nullptr, int n_clear = 0) {
  cudaError_t e = cudaFuncSetAttribute(memory_finalize_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, memory_finalize_kernel<D>, partials, G, tpg, n_tok, log2lam,
                            W_phi, r, decay_n, M, bstab, sv_partials, s_v, n_count, n_add, Hkv,
                            clear_tags, n_clear);
}

}  // namespace

// Split of the evicted tokens of every (sequence, KV head) into runs: a whole
// number of 64-token chunks per run, about two CTAs per SM in one wave
// (units * runs <= 2 * num_sms where the tokens allow). tokens_per_run is the
// run length; the last run of a unit may be shorter. The result does not
// depend on the split (the finalize applies each run's decay factor).
struct MemSplit { int runs, tokens_per_run; };
MemSplit memory_split(int batch, int n_kv_heads, int n_e, int num_sms, size_t max_runs_total) {
  const int units = batch * n_kv_heads;
  const int chunks = (n_e + kChunk - 1) / kChunk;
  int G = (2 * num_sms) / units;
  if (G > chunks) G = chunks;
  if (G > kMemMaxGroups) G = kMemMaxGroups;
  while (G > 1 && (size_t)units * G > max_runs_total) --G;
  if (G < 1) G = 1;
  const int tpr = ((chunks + G - 1) / G) * kChunk;
  return MemSplit{(n_e + tpr - 1) / tpr, tpr};
}

// Runs of the bf16 kernel (kBfCtasPerSm CTAs per SM): at least ceil(n / kRunMax) runs
// per unit (the run's positions sit in shared memory), a whole number of
// 32-token chunks each; among the run counts up to four waves, the one whose
// last wave is fullest (the fewest runs within 3% of the best), so that SMs do
// not idle in a partial wave.
MemSplit memory_split_bf16(int batch, int n_kv_heads, int n_e, int num_sms) {
  const int units = batch * n_kv_heads;
  const int chunks = (n_e + kBfChunk - 1) / kBfChunk;
  int lo = (n_e + kRunMax - 1) / kRunMax;
  if (lo < 1) lo = 1;
  const int slots = num_sms * kBfCtasPerSm;
  int hi = (4 * slots) / units;
  if (hi > chunks) hi = chunks;
  if (hi > kMemMaxGroups) hi = kMemMaxGroups;
  if (hi < lo) hi = lo;
  double best = -1.0;
  int G = lo;
  for (int g = lo; g <= hi; ++g) {
    const long ctas = (long)units * g;
    const long waves = (ctas + slots - 1) / slots;
    const double eff = (double)ctas / (double)(waves * slots);
    if (eff > best + 0.03) { best = eff; G = g; }
  }
  const int tpr = ((chunks + G - 1) / G) * kBfChunk;
  return MemSplit{(n_e + tpr - 1) / tpr, tpr};
}

// Upper bound of units * runs over both kernels for up to L evicted tokens
// per unit (sizes the partial sums in the workspace).
size_t memory_runs_bound(int units, int L, int num_sms) {
  return (size_t)units * ((L + kRunMax - 1) / kRunMax + 1) + 4 * (size_t)num_sms * kBfCtasPerSm +
         units;
}

cudaError_t launch_memory_update(const Ctx& c, int batch, int L, const void* K, const void* V,
                                 const int32_t* idx_e, int n_e, int chunk, float* M, float* bstab,
                                 float* partials, float* sv_partials, float* s_v, float* n_count,
                                 cudaStream_t st, int* clear_tags, int n_clear) {
  if (n_e == 0)
    return clear_tags ? cudaMemsetAsync(clear_tags, 0, (size_t)n_clear * sizeof(int), st)
                      : cudaSuccess;
  const int Hkv = c.cfg.n_kv_heads, D = c.cfg.head_dim, r = c.cfg.mem_r;
  (void)chunk;   // the split below does not change the result
  // bf16 gated memory: the cp.async-fed kernel, unless a run would exceed the
  // run count the finalize handles (n_e beyond kMemMaxGroups * kRunMax)
  const bool bf16_path = c.cfg.dtype == IMEM_BF16 && !sv_partials &&
                         (n_e + kRunMax - 1) / kRunMax <= kMemMaxGroups;
  const MemSplit sp = bf16_path ? memory_split_bf16(batch, Hkv, n_e, c.num_sms)
                                : memory_split(batch, Hkv, n_e, c.num_sms,
                                               (size_t)batch * Hkv + 2 * 148);
  const int tokens_per_group = sp.tokens_per_run;
  const int Gused = sp.runs;
  dim3 grid(Hkv, Gused, batch);
  const float log2lam = (float)log2((double)c.cfg.lambda);
  cudaError_t e = cudaSuccess;
#define IMEM_MEMBF(DD)                                                                        \
  do {                                                                                        \
    e = cudaFuncSetAttribute(memory_bf16_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             BfTile<DD>::SMEM);                                               \
    if (e != cudaSuccess) return e;                                                           \
    memory_bf16_kernel<DD><<<grid, bf_threads<DD>(), BfTile<DD>::SMEM, st>>>(                      \
        (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx_e, n_e, L, Hkv, log2lam,        \
        tokens_per_group, partials, c.err);                                                   \
  } while (0)
  if (bf16_path) {
    if (D == 128) IMEM_MEMBF(128); else IMEM_MEMBF(64);
  } else {
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
  }
#undef IMEM_MEM
#undef IMEM_MEMBF
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float decay_n = (float)pow((double)c.cfg.lambda, (double)n_e);
  dim3 fgrid(D / 16 + 1 + (sv_partials ? 1 : 0), batch * Hkv);
  // moment statistics use the identity map: the finalize skips the product
  const float* phi = c.cfg.readout == IMEM_READOUT_MOMENT ? nullptr : c.W_phi;
  const size_t fsmem = fin_smem(D, Gused);
  if (D == 128)
    e = launch_finalize<128>(fgrid, fsmem, st, partials, Gused, tokens_per_group, n_e, log2lam,
                             phi, r, decay_n, M, bstab, sv_partials, s_v, n_count, (float)n_e, Hkv,
                             clear_tags, n_clear);
  else
    e = launch_finalize<64>(fgrid, fsmem, st, partials, Gused, tokens_per_group, n_e, log2lam,
                            phi, r, decay_n, M, bstab, sv_partials, s_v, n_count, (float)n_e, Hkv,
                            clear_tags, n_clear);
  if (e != cudaSuccess) return e;
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
  (void)chunk;
  int num_sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  const MemSplit sp = memory_split(batch, Hkv, n_e, num_sms, kStaticScratchBytes / psize);
  const int tokens_per_group = sp.tokens_per_run;
  const int Gused = sp.runs;
  const float log2lam = (float)log2((double)lambda);
  auto kfn = memory_tc_kernel<T, D, false>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       MemTile<D>::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<dim3(Hkv, Gused, batch), kMemThreads, MemTile<D>::SMEM, st>>>(
      (const T*)K, (const T*)V, idx_e, n_e, L, Hkv, log2lam, tokens_per_group, scratch, nullptr,
      err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float decay_n = (float)pow((double)lambda, (double)n_e);
  const size_t fsmem = fin_smem(D, Gused);
  e = launch_finalize<D>(dim3(D / 16 + 1, units), fsmem, st, scratch, Gused, tokens_per_group, n_e,
                         log2lam, W_phi, r, decay_n, M, bstab, nullptr, nullptr, nullptr, 0.f, Hkv);
  if (e != cudaSuccess) return e;
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
