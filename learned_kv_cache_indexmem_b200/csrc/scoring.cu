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
//
// With the gated head sum folded into qtilde (exact, see prologue.cu) the
// contraction is over d_I = 64. Keys sit on the MMA M dimension (TMEM lanes)
// and queries on N, so each epilogue thread owns one key and the pooling is a
// register max over its TMEM row.
//
// Persistent kernel, one CTA per SM. Work item = (sequence, block of 256
// keys, tile of 256 queries); the causal items of all sequences are
// enumerated in closed form and split evenly over the CTAs. Per item the MMA
// thread issues, for each of the block's two 128-key tiles, 4 tcgen05.mma
// (M=128 keys, N=256 queries, K=16) from TMA-loaded, 128B-swizzled K-major
// tiles into that tile's 256-column TMEM accumulator. N=256 halves the
// shared-memory operand traffic per flop of an N=128 shape, and the two key
// tiles sharing one query tile halve the L2 traffic of one. Eight epilogue
// warps drain one accumulator while the other is being computed (tcgen05.ld,
// masked three-input maxima, a warp per 32 keys x 128 queries) and flush a
// key's maximum with an atomic float max when its key block ends (several
// CTAs may share a key block).
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

#include <atomic>

namespace imem {
namespace {

constexpr int kKB = 256;        // keys per key block (two M = 128 tiles)
constexpr int kQT = 256;        // queries per tile (N = 256)
constexpr int kBStages = 4;     // query-tile ring
constexpr int kEpiWarps = 8;
constexpr int kScThreads = 64 + kEpiWarps * 32;
constexpr int kABytes = kKB * 128;    // 256 rows x 128 B
constexpr int kBBytes = kQT * 128;    // 256 rows x 128 B
constexpr int kScSmem = 2 * kABytes + kBStages * kBBytes + 1024 + 256;

// Closed-form enumeration of the causal work items of one sequence: key
// block kb (keys [256 kb, 256 kb + 256)) takes the query tiles of 256 from
// qs = max(q_begin, 256 kb) to q_end; past q_begin that is Qc - kb tiles with
// Qc = ceil(q_end / 256), so the prefix sums are arithmetic series.
struct Sched {
  int q_begin, q_end, nkb, kb0, N0, Qc;
  long long per_seq;

  __host__ __device__ void init(int qb, int qe) {
    q_begin = qb; q_end = qe;
    nkb = (qe + kKB - 1) / kKB;
    kb0 = qb / kKB;
    N0 = (qe - qb + kQT - 1) / kQT;
    Qc = (qe + kQT - 1) / kQT;
    per_seq = prefix(nkb);
  }
  // query tiles of key block kb
  __host__ __device__ int nq(int kb) const { return kb <= kb0 ? N0 : Qc - kb; }
  // items of key blocks [0, kb)
  __host__ __device__ long long prefix(int kb) const {
    if (kb <= kb0 + 1) return (long long)kb * N0;
    const long long k1 = kb0 + 1, k2 = kb - 1, cnt = k2 - k1 + 1;
    return (long long)(kb0 + 1) * N0 + cnt * Qc - (k1 + k2) * cnt / 2;
  }
  __host__ __device__ int qstart(int kb) const { return kb * kKB > q_begin ? kb * kKB : q_begin; }
};

// Key blocks are visited in folded order 0, nkb-1, 1, nkb-2, ... so that every
// CTA's contiguous range of items mixes long blocks (few key-tile switches)
// and short ones (a switch and a diagonal tile every item or two).
__host__ __device__ inline int fold_kb(int p, int nkb) { return (p & 1) ? nkb - 1 - (p >> 1) : (p >> 1); }

constexpr int kMaxScCtas = 160;
// Where each CTA's range of items starts (computed on the host per launch).
struct ScStarts {
  int seq[kMaxScCtas], p[kMaxScCtas], j[kMaxScCtas], count[kMaxScCtas];
};

struct Cursor {
  int seq, p, kb, j;
  __device__ void init(const Sched& sc, int s0, int p0, int j0) {
    seq = s0; p = p0; j = j0; kb = fold_kb(p, sc.nkb);
  }
  __device__ void next(const Sched& sc) {
    if (++j == sc.nq(kb)) {
      j = 0;
      if (++p == sc.nkb) { p = 0; ++seq; }
      kb = fold_kb(p, sc.nkb);
    }
  }
};

__global__ void __launch_bounds__(kScThreads, 1)
scoring_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  int L, int q_begin, int q_end, const __grid_constant__ ScStarts starts,
                  float* __restrict__ running_max, int* __restrict__ err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = tc::smem_addr(smem);                 // 2 key blocks
  const uint32_t sB = sA + 2 * kABytes;                     // kBStages query tiles
  const uint32_t bar = sB + kBStages * kBBytes;
  const uint32_t a_full = bar, a_empty = bar + 16, b_full = bar + 32,
                 b_empty = b_full + 8 * kBStages, t_full = b_empty + 8 * kBStages,
                 t_empty = t_full + 16;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Sched sc;
  sc.init(q_begin, q_end);
  const long long i_begin = 0;
  const long long i_end = starts.count[blockIdx.x];

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(a_full + 8 * i, 1);
      tc::mbar_init(a_empty + 8 * i, 1);
      tc::mbar_init(t_full + 8 * i, 1);
      tc::mbar_init(t_empty + 8 * i, kEpiWarps);
    }
    for (int i = 0; i < kBStages; ++i) {
      tc::mbar_init(b_full + 8 * i, 1);
      tc::mbar_init(b_empty + 8 * i, 1);
    }
    tc::fence_mbar_init();
    tc::prefetch_tmap(&map_q);
    tc::prefetch_tmap(&map_k);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_addr(&s_tmem), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = s_tmem;

  if (i_begin < i_end) {
    if (warp == 0 && lane == 0) {
      // ---------------- TMA producer
      Cursor cu;
      cu.init(sc, starts.seq[blockIdx.x], starts.p[blockIdx.x], starts.j[blockIdx.x]);
      long long prev = -1;
      int kbi = -1;
      for (long long i = i_begin; i < i_end; ++i) {
        const long long kid = (long long)cu.seq * sc.nkb + cu.kb;
        if (kid != prev) {
          ++kbi;
          const int ab = kbi & 1;
          if (kbi >= 2 && !tc::mbar_wait(a_empty + 8 * ab, ((kbi >> 1) - 1) & 1)) {
            record_error(err, DEV_TIMEOUT);
            break;
          }
          tc::mbar_expect_tx(a_full + 8 * ab, kABytes);
          tc::tma_load_2d(sA + ab * kABytes, &map_k, a_full + 8 * ab, 0, cu.seq * L + cu.kb * kKB);
          prev = kid;
        }
        const int n = (int)(i - i_begin);
        const int st = n % kBStages;
        if (n >= kBStages && !tc::mbar_wait(b_empty + 8 * st, ((n / kBStages) - 1) & 1)) {
          record_error(err, DEV_TIMEOUT);
          break;
        }
        tc::mbar_expect_tx(b_full + 8 * st, kBBytes);
        tc::tma_load_2d(sB + st * kBBytes, &map_q, b_full + 8 * st, 0,
                        cu.seq * L + sc.qstart(cu.kb) + cu.j * kQT);
        cu.next(sc);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t IDESC = tc::idesc(tc::kFmtBF16, 128, kQT, false, false);
      Cursor cu;
      cu.init(sc, starts.seq[blockIdx.x], starts.p[blockIdx.x], starts.j[blockIdx.x]);
      long long prev = -1;
      int kbi = -1;
      for (long long i = i_begin; i < i_end; ++i) {
        const long long kid = (long long)cu.seq * sc.nkb + cu.kb;
        const int n = (int)(i - i_begin);
        if (kid != prev) {
          ++kbi;
          if (!tc::mbar_wait(a_full + 8 * (kbi & 1), (kbi >> 1) & 1)) { record_error(err, DEV_TIMEOUT); break; }
          prev = kid;
        }
        const int ab = kbi & 1;
        const int st = n % kBStages;
        if (!tc::mbar_wait(b_full + 8 * st, (n / kBStages) & 1)) { record_error(err, DEV_TIMEOUT); break; }
        bool ok = true;
#pragma unroll 1
        for (int kt = 0; kt < 2; ++kt) {   // the two key tiles share the query tile
          const int sub = 2 * n + kt, tb = sub & 1;
          if (sub >= 2 && !tc::mbar_wait(t_empty + 8 * tb, ((sub >> 1) - 1) & 1)) { ok = false; break; }
          tc::fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = tc::sdesc_sw128(sA + ab * kABytes + kt * (kABytes / 2) + k * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(sB + st * kBBytes + k * 32, 16, 1024);
            tc::mma_f16(tmem + tb * 256, ad, bd, IDESC, k > 0 ? 1u : 0u);
          }
          tc::mma_commit(t_full + 8 * tb);
        }
        if (!ok) { record_error(err, DEV_TIMEOUT); break; }
        tc::mma_commit(b_empty + 8 * st);
        cu.next(sc);
        const long long nkid = (long long)cu.seq * sc.nkb + cu.kb;
        if (i + 1 == i_end || nkid != kid) tc::mma_commit(a_empty + 8 * ab);
      }
    } else if (warp >= 2) {
      // ---------------- epilogue: masked row maxima, flushed per key block
      const int e = warp - 2;
      const int quarter = warp & 3;        // TMEM lanes this warp may read
      const int half = e >> 2;             // which 128 of the 256 query columns
      Cursor cu;
      cu.init(sc, starts.seq[blockIdx.x], starts.p[blockIdx.x], starts.j[blockIdx.x]);
      long long prev = -1;
      int pseq = 0, pkb = 0;
      float runmax[2] = {-INFINITY, -INFINITY};   // one key in each of the block's two tiles
      auto flush = [&](int seq, int kb) {
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
          const int t = kb * kKB + kt * 128 + quarter * 32 + lane;
          if (t < q_end && runmax[kt] != -INFINITY)
            atomic_max_float(&running_max[(size_t)seq * L + t], runmax[kt]);
        }
      };
      bool ok = true;
      for (long long i = i_begin; i < i_end && ok; ++i) {
        const long long kid = (long long)cu.seq * sc.nkb + cu.kb;
        if (kid != prev) {
          if (prev >= 0) flush(pseq, pkb);
          runmax[0] = runmax[1] = -INFINITY;
          prev = kid; pseq = cu.seq; pkb = cu.kb;
        }
        const int n = (int)(i - i_begin);
        const int s0 = sc.qstart(cu.kb) + cu.j * kQT + half * 128;   // first query of these columns
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
          if (!tc::mbar_wait(t_full + 8 * kt, n & 1)) { ok = false; break; }
          tc::fence_after();
          const int t = cu.kb * kKB + kt * 128 + quarter * 32 + lane;
          const bool full = (s0 >= t) && (s0 + 128 <= q_end);
          const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + kt * 256 + half * 128;
          // all four 32-column loads in flight, one wait
          uint32_t v0[32], v1[32], v2[32], v3[32];
          tc::tmem_ld32_async(base + 0, v0);
          tc::tmem_ld32_async(base + 32, v1);
          tc::tmem_ld32_async(base + 64, v2);
          tc::tmem_ld32_async(base + 96, v3);
          tc::tmem_wait_ld_dep<true>(v0);
          tc::tmem_wait_ld_dep<false>(v1);
          tc::tmem_wait_ld_dep<false>(v2);
          tc::tmem_wait_ld_dep<false>(v3);
          float m = runmax[kt];
          if (full) {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              m = tc::max3f(m, __uint_as_float(v0[x]), __uint_as_float(v0[x + 1]));
              m = tc::max3f(m, __uint_as_float(v1[x]), __uint_as_float(v1[x + 1]));
              m = tc::max3f(m, __uint_as_float(v2[x]), __uint_as_float(v2[x + 1]));
              m = tc::max3f(m, __uint_as_float(v3[x]), __uint_as_float(v3[x + 1]));
            }
          } else {
            // query s = s0 + column; valid when t <= s < q_end
            const int lo = t - s0, hi = q_end - s0;   // valid columns: [lo, hi)
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float a0 = (x >= lo && x < hi) ? __uint_as_float(v0[x]) : -INFINITY;
              const float a1 = (x + 32 >= lo && x + 32 < hi) ? __uint_as_float(v1[x]) : -INFINITY;
              const float a2 = (x + 64 >= lo && x + 64 < hi) ? __uint_as_float(v2[x]) : -INFINITY;
              const float a3 = (x + 96 >= lo && x + 96 < hi) ? __uint_as_float(v3[x]) : -INFINITY;
              m = tc::max3f(m, a0, a1);
              m = tc::max3f(m, a2, a3);
            }
          }
          runmax[kt] = m;
          tc::fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(t_empty + 8 * kt);
        }
        cu.next(sc);
      }
      if (!ok) record_error(err, DEV_TIMEOUT);
      if (prev >= 0) flush(pseq, pkb);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_scoring(const Ctx& c, int batch, int L, const __nv_bfloat16* qt,
                           const __nv_bfloat16* kh, float* running_max, int q_begin, int q_end,
                           cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_tmap_rows64(c, &mq, qt, (uint64_t)batch * L, kQT)) return cudaErrorInvalidValue;
  if (!make_tmap_rows64(c, &mk, kh, (uint64_t)batch * L, kKB)) return cudaErrorInvalidValue;
  Sched sc;
  sc.init(q_begin, q_end);
  const long long total = sc.per_seq * batch;
  int grid = c.num_sms < kMaxScCtas ? c.num_sms : kMaxScCtas;
  if (total < grid) grid = (int)total;
  // split the folded item sequence evenly; record each CTA's starting position
  ScStarts starts;
  {
    const long long per = (total + grid - 1) / grid;
    int seq = 0, p = 0, j = 0;
    long long done = 0;
    for (int b = 0; b < grid; ++b) {
      const long long cnt = (total - done) < per ? (total - done) : per;
      starts.seq[b] = seq; starts.p[b] = p; starts.j[b] = j; starts.count[b] = (int)cnt;
      long long left = cnt;   // advance by cnt items, a key block at a time
      while (left > 0) {
        const int kb = fold_kb(p, sc.nkb);
        const int rest = sc.nq(kb) - j;
        if (left < rest) { j += (int)left; left = 0; }
        else {
          left -= rest; j = 0;
          if (++p == sc.nkb) { p = 0; ++seq; }
        }
      }
      done += cnt;
    }
  }
  static std::atomic<uint64_t> attr_done{0};   // one bit per device
  const uint64_t bit = 1ull << (c.device & 63);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(scoring_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kScSmem);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  scoring_tc_kernel<<<grid, kScThreads, kScSmem, st>>>(mq, mk, L, q_begin, q_end, starts,
                                                       running_max, c.err);
  return cudaGetLastError();
}

}  // namespace imem
