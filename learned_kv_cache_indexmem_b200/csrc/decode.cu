// decode.cu -- one decode step over the retained (compacted) KV cache with the
// gated latent-memory readout.
//
// Source: "IndexMem: learned KV-cache eviction with latent memory" technical
// summary, §2.B Output: o = o_attn + g(q) * m(q), where o_attn is standard
// attention over the retained tokens and m(q) the readout of the memory M
// (normalised with the stabiliser b); the readout weights are a projection
// phi and a gate g(q). The split-K combine uses the exact merge of softmax
// partial states (max, normaliser, unnormalised output) over disjoint key
// blocks -- the online-softmax identity stated in "Context Memorization for
// Efficient Long Context Generation" (technical summary, Method).
//
// Grid (S + 1, Hkv, batch), one thread-block cluster of S + 1 CTAs per
// (sequence, KV head) -- a "unit". CTAs 0..S-1 each stream a contiguous block
// of cache rows and keep one softmax state per query head of the GQA group;
// CTA S computes the memory readout
//   u = W_phi q,  m = M^T u / (b . u + eps),  g = sigmoid(w_gate . q)
// meanwhile. Each attention CTA merges its warps' states straight into a slot
// of CTA S's shared memory (distributed shared memory), then arrives on the
// cluster barrier; CTA S merges the S states, adds g*m and writes the output.
// CTA 0 of the last unit of a sequence advances cache_len. CTA 0 appends the new
// key/value row to the cache; the CTA whose block covers row cache_len reads
// it from k_new/v_new.
//
// Latency: the kernel is launched with programmatic stream serialization, so
// its CTAs are resident before the previous kernel ends. CTA S stages W_phi
// (owned by the context) before the wait, and b and M too where M has a
// region of its own; an attention CTA reads a hint of cache_len before it and
// loads the rows of its block below the hint minus one (cp.async staging; TMA
// staging issues them right after the wait). After the wait a per-sequence
// tag in the workspace, 1 + the length that the last decode step left and
// cleared by every other call that writes the cache state, decides whether
// those early copies stand: they do when the tag matches the true length
// (the rows then predate the previous kernel, and b and M are unchanged);
// otherwise they are dropped and loaded again.
//
// bf16 attention: rows are staged in shared memory (a ring of two or three
// 64-row stages, XOR-swizzled 16-byte chunks) and contracted with warp-level
// tensor-core MMA (m16n8k16, fp32 accumulation) with the cache rows on M and
// the GQA heads on N: S = K q^T, then O^T += V^T P, V^T read with transposing
// shared-memory loads and P turned into the B operand by an in-register 8x8
// transpose. A warp's 16 rows cost 2 x D/16 MMAs. fp32 attention: CUDA cores.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

#include <cooperative_groups.h>
#include <math.h>

#include <atomic>
#include <mutex>
#include <type_traits>

namespace imem {
namespace {

constexpr int kThreads = 128;
constexpr int kStageRows = 64;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Partial {   // one query head's softmax state over a block of rows
  float m;         // max of the log2-scaled logits
  float l;         // sum of 2^(s - m)
  float pad[2];
  float o[D];      // sum of 2^(s - m) v (at byte 16)
};
static_assert(sizeof(Partial<128>) == 16 + 4 * 128, "o at byte 16");

// ---- warp-level tensor-core helpers (bf16) -----------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0: zero-fill the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }
// waits until at most n of this thread's cp.async groups are pending
__device__ __forceinline__ void cp_async_wait_dyn(int n) {
  if (n <= 0) cp_async_wait<0>();
  else if (n == 1) cp_async_wait<1>();
  else if (n == 2) cp_async_wait<2>();
  else cp_async_wait<3>();
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D = A(16x16) * B(16x8) + C with all four A registers
__device__ __forceinline__ void mma_bf16_a4(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// transpose of an 8x8 matrix of 16-bit pairs held one pair per lane
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stage buffers hold K then V, each as D/64 column halves of [64 rows][128 B]
// written by TMA with the 128-byte swizzle: 16-byte chunk cc of row rr of a
// half sits at rr * 128 + ((cc ^ (rr & 7)) << 4), which keeps ldmatrix
// conflict-free. tile_off gives the byte offset of chunk c (0..D/8) of a row.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int row, int c) {
  return (uint32_t)((c >> 3) * (kStageRows * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}
template <int D>
constexpr uint32_t kTileBytes = kStageRows * D * 2;   // one of K, V in a stage

// Ring of nst stage buffers, each with a transaction barrier. Global stage
// index gi uses buffer gi % nst in phase (gi / nst) & 1. Thread 0 issues the
// loads; last[b] (thread 0 only) is the last index issued into buffer b.
struct Ring {
  uint32_t buf0;   // shared address of buffer 0 (1024-byte aligned)
  uint32_t bar0;   // shared address of barrier 0 (barriers 8 bytes apart)
  int nst;
  int last[kDecodeMaxStages];
};

// Thread 0: loads the 64 cache rows starting at 2-D row y (of the [batch*cap,
// Hkv*D] view) into buffer gi % nst, columns x0..x0+D-1. A buffer is reused
// only once the load issued into it before has landed.
template <int D>
__device__ void ring_issue(Ring& rg, const CUtensorMap* tmK, const CUtensorMap* tmV, int gi,
                           int x0, int y, int* err) {
  const int b = gi % rg.nst;
  const uint32_t bar = rg.bar0 + 8u * b;
  if (rg.last[b] >= 0 && !tc::mbar_wait(bar, (uint32_t)(rg.last[b] / rg.nst) & 1u))
    record_error(err, DEV_TIMEOUT);
  rg.last[b] = gi;
  const uint32_t dst = rg.buf0 + (uint32_t)b * 2u * kTileBytes<D>;
  tc::mbar_expect_tx(bar, 2u * kTileBytes<D>);
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    tc::tma_load_2d(dst + h * (kStageRows * 128), tmK, bar, x0 + 64 * h, y);
    tc::tma_load_2d(dst + kTileBytes<D> + h * (kStageRows * 128), tmV, bar, x0 + 64 * h, y);
  }
}

// Thread 0: waits until the last load issued into every buffer has landed
// (before the buffers are reused for something else or the CTA exits).
template <int D>
__device__ void ring_drain(const Ring& rg, int* err) {
  for (int b = 0; b < rg.nst; ++b)
    if (rg.last[b] >= 0 && !tc::mbar_wait(rg.bar0 + 8u * b, (uint32_t)(rg.last[b] / rg.nst) & 1u))
      record_error(err, DEV_TIMEOUT);
}

// All threads: the cp.async form of ring_issue for rows [y_row, y_row + 64)
// of this unit's cache (Kb/Vb point at row 0, rows `row_stride` apart). Rows
// at or past `hi` are not loaded (zero-filled); one commit group per stage.
template <int D>
__device__ void ring_issue_lsu(const Ring& rg, const __nv_bfloat16* __restrict__ Kb,
                               const __nv_bfloat16* __restrict__ Vb, size_t row_stride, int gi,
                               int base, int hi) {
  constexpr int CH = D / 8;
  const uint32_t kdst = rg.buf0 + (uint32_t)(gi % rg.nst) * 2u * kTileBytes<D>;
  const uint32_t vdst = kdst + kTileBytes<D>;
  // thread -> (row rr = tid / CH + k * kThreads / CH, chunk c = tid % CH): the
  // chunk and the swizzle term (rr & 7) stay fixed over k
  const int c = threadIdx.x % CH, rr0 = threadIdx.x / CH;
  constexpr int RSTEP = kThreads / CH;
#pragma unroll
  for (int k = 0; k < kStageRows / RSTEP; ++k) {
    const int rr = rr0 + k * RSTEP, row = base + rr;
    const bool ok = row < hi;
    const size_t off = (size_t)(ok ? row : 0) * row_stride + c * 8;
    cp_async16(kdst + tile_off<D>(rr, c), Kb + off, ok);
    cp_async16(vdst + tile_off<D>(rr, c), Vb + off, ok);
  }
  cp_async_commit();
}

// All threads: cp.async loads of the rows in [lo, hi) of the stage that holds
// rows [base, base + 64) (ring index gi); the stage's other rows are left
// untouched and nothing is committed (the caller closes the group).
template <int D>
__device__ void ring_issue_rows(const Ring& rg, const __nv_bfloat16* __restrict__ Kb,
                                const __nv_bfloat16* __restrict__ Vb, size_t row_stride, int gi,
                                int base, int lo, int hi) {
  constexpr int CH = D / 8;
  const uint32_t kdst = rg.buf0 + (uint32_t)(gi % rg.nst) * 2u * kTileBytes<D>;
  const uint32_t vdst = kdst + kTileBytes<D>;
  const int c = threadIdx.x % CH, rr0 = threadIdx.x / CH;
  constexpr int RSTEP = kThreads / CH;
#pragma unroll
  for (int k = 0; k < kStageRows / RSTEP; ++k) {
    const int rr = rr0 + k * RSTEP, row = base + rr;
    if (row >= lo && row < hi) {
      const size_t off = (size_t)row * row_stride + c * 8;
      cp_async16(kdst + tile_off<D>(rr, c), Kb + off, true);
      cp_async16(vdst + tile_off<D>(rr, c), Vb + off, true);
    }
  }
}

// ---- attention over rows [r0, r1) for one unit, bf16 tensor-core path --------
// Stage st (rows r0 + 64 st ..) has global index g0 + st; stages below n_pre
// were issued before the row range was known. Rows past r1 in a stage are
// zeroed in shared memory, row len (the new token) is taken from kn/vn.
// Leaves the per-warp states in s_part[warp][g].
//
// kTma: stages are loaded by TMA (thread 0 issues, transaction barriers);
// otherwise by cp.async from every thread (rows below `hi` only). TMA frees
// the SM's issue slots and wins when CTAs stream in several waves; cp.async
// delivers the first rows sooner and wins when the grid is one wave.
template <int D, int G, bool kTma, int kXtra>
__device__ void attend_bf16(Ring& rg, const CUtensorMap* tmK, const CUtensorMap* tmV, int x0,
                            int y0, const __nv_bfloat16* __restrict__ Kb,
                            const __nv_bfloat16* __restrict__ Vb, size_t row_stride, int hi,
                            const __nv_bfloat16* kn, const __nv_bfloat16* vn, int len,
                            int r0, int r1, int g0, int n_pre, const float (*s_q)[D],
                            Partial<D> (*s_part)[G], int* err, const uint4* s_new) {
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const float sscale = kLog2e * rsqrtf((float)D);
  const int nst = rg.nst;

  // Cache rows on the MMA's M dimension, the GQA heads on N (8 columns,
  // heads >= G zero): S[row][head] = K q^T, then O^T[dim][head] += V^T P.
  // q as B fragments: b0 = dims 16s+2t.., b1 = +8, column g = head g
  uint32_t qb0[D / 16], qb1[D / 16];
#pragma unroll
  for (int s = 0; s < D / 16; ++s) {
    if (g < G) {
      qb0[s] = pack_bf16(s_q[g][16 * s + 2 * t], s_q[g][16 * s + 2 * t + 1]);
      qb1[s] = pack_bf16(s_q[g][16 * s + 8 + 2 * t], s_q[g][16 * s + 8 + 2 * t + 1]);
    } else {
      qb0[s] = 0u; qb1[s] = 0u;
    }
  }
  // O^T accumulators: o[mt] = dims 16mt+g (0, 1) and +8 (2, 3), heads 2t, 2t+1
  float o[D / 16][4];
#pragma unroll
  for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  // running max and this lane's share of the normaliser, heads 2t and 2t+1
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  const int n_stages = (r1 - r0 + kStageRows - 1) / kStageRows;
  int issued = max(n_pre, min(n_stages, nst));   // stages issued so far (cp.async groups)
  if constexpr (kTma) {
    if (tid == 0)
      for (int st = n_pre; st < n_stages && st < nst; ++st)
        ring_issue<D>(rg, tmK, tmV, g0 + st, x0, y0 + r0 + st * kStageRows, err);
  } else {
    for (int st = n_pre; st < n_stages && st < nst; ++st)
      ring_issue_lsu<D>(rg, Kb, Vb, row_stride, g0 + st, r0 + st * kStageRows, hi);
  }
  // stages beyond the ring (kXtra: launches whose blocks reach one more, 1,
  // or more, 2): after
  // the ring's stages, each warp streams its own 16 rows of every further
  // stage through its own rows of the ring's buffers (warp-local copies and
  // waits, no block barrier): the first further stage's K once the warp's
  // scores are done and its V once its first P V is done, the next ones (K
  // and V) once the slice they reuse has been consumed
  const bool extra = kXtra != 0 && !kTma && n_stages > nst && nst == kDecodeMaxStages &&
                     (kXtra == 2 || n_stages == nst + 1);
  if (!kTma && (n_stages <= nst || extra)) {
    // Every stage of this block is in the ring at once (one-wave grids): the
    // scores of all of a warp's row tiles first (independent MMA chains,
    // interleaved), one softmax over them, then all the P V products; the
    // stage-by-stage loop below would chain the tiles one after another.
    // this warp's rows of stage xs into its rows of the buffer at kt (K, V or
    // both: one cp.async group)
    int xg = 0;   // warp-local groups issued
    auto issue_slice = [&](uint32_t kt, int xs, bool k, bool v) {
      const int row0 = r0 + xs * kStageRows;
      for (int i = lane; i < 16 * CH; i += 32) {
        const int rr = warp * 16 + i / CH, c = i % CH, row = row0 + rr;
        const bool ok = row < hi;
        const size_t off = (size_t)(ok ? row : 0) * row_stride + c * 8;
        if (k) cp_async16(kt + tile_off<D>(rr, c), Kb + off, ok);
        if (v) cp_async16(kt + kTileBytes<D> + tile_off<D>(rr, c), Vb + off, ok);
      }
      cp_async_commit();
      ++xg;
    };
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll
    for (int st = 0; st < kDecodeMaxStages; ++st) {
      const int kb = r0 + st * kStageRows + warp * 16;
      if (st < n_stages && kb < r1 && (kb + 16 > r1 || (len >= kb && len < kb + 16))) {
        const uint32_t kt = rg.buf0 + (uint32_t)((g0 + st) % nst) * 2u * kTileBytes<D>;
        const uint32_t vt = kt + kTileBytes<D>;
        for (int i = lane; i < 16 * CH; i += 32) {
          const int rr = warp * 16 + i / CH, c = i % CH, row = kb + i / CH;
          if (row >= r1) {
            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(vt + tile_off<D>(rr, c)),
                         "r"(0u));
          } else if (row == len) {
            const uint4 kv = s_new[c];
            const uint4 vv = s_new[CH + c];
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(kt + tile_off<D>(rr, c)),
                         "r"(kv.x), "r"(kv.y), "r"(kv.z), "r"(kv.w));
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(vt + tile_off<D>(rr, c)),
                         "r"(vv.x), "r"(vv.y), "r"(vv.z), "r"(vv.w));
          }
        }
      }
    }
    __syncwarp();
    // scores: tiles past the block compute on whatever the buffer holds and
    // are masked by selection (never by arithmetic, so nothing there leaks)
    float sa[kDecodeMaxStages][4], sb[kDecodeMaxStages][4];
    uint32_t kts[kDecodeMaxStages];
#pragma unroll
    for (int st = 0; st < kDecodeMaxStages; ++st) {
      kts[st] = rg.buf0 + (uint32_t)((g0 + st) % nst) * 2u * kTileBytes<D>;
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[st][e] = sb[st][e] = 0.f;
    }
    {
      const int rr = warp * 16 + (lane & 15);
#pragma unroll
      for (int s2 = 0; s2 < D / 16; ++s2) {
#pragma unroll
        for (int st = 0; st < kDecodeMaxStages; ++st) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kts[st] + tile_off<D>(rr, 2 * s2 + (lane >> 4)), a0, a1, a2, a3);
          if (s2 & 1) mma_bf16_a4(sb[st], a0, a1, a2, a3, qb0[s2], qb1[s2]);
          else mma_bf16_a4(sa[st], a0, a1, a2, a3, qb0[s2], qb1[s2]);
        }
      }
    }
    if (extra) {   // this warp's K rows of the first stage are read: the next stage's K there
      __syncwarp();
      issue_slice(kts[0], nst, true, false);
    }
    float sc[kDecodeMaxStages][4];
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int st = 0; st < kDecodeMaxStages; ++st) {
      const int kb = r0 + st * kStageRows + warp * 16;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = kb + g + ((e >> 1) << 3);
        sc[st][e] = (st < n_stages && row < r1) ? (sa[st][e] + sb[st][e]) * sscale : -INFINITY;
      }
      mx[0] = fmaxf(mx[0], fmaxf(sc[st][0], sc[st][2]));
      mx[1] = fmaxf(mx[1], fmaxf(sc[st][1], sc[st][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], off));
      mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], off));
    }
    m_run[0] = mx[0];
    m_run[1] = mx[1];
#pragma unroll
    for (int st = 0; st < kDecodeMaxStages; ++st) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sc[st][e] = (sc[st][e] == -INFINITY) ? 0.f : exp2f(sc[st][e] - m_run[e & 1]);
      l_run[0] += sc[st][0] + sc[st][2];
      l_run[1] += sc[st][1] + sc[st][3];
    }
    const int rv = warp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
    for (int st = 0; st < kDecodeMaxStages; ++st) {
      const int kb = r0 + st * kStageRows + warp * 16;
      if (st < n_stages && kb < r1) {   // warp-uniform
        const uint32_t pb0 = movm_trans(pack_bf16(sc[st][0], sc[st][1]));
        const uint32_t pb1 = movm_trans(pack_bf16(sc[st][2], sc[st][3]));
        const uint32_t vt = kts[st] + kTileBytes<D>;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vt + tile_off<D>(rv, 2 * mt + ((lane >> 3) & 1)), a0, a1, a2, a3);
          mma_bf16_a4(o[mt], a0, a1, a2, a3, pb0, pb1);
        }
      }
      if (extra) {   // this warp's rows of stage st are consumed: refill them
        __syncwarp();
        if (st == 0) issue_slice(kts[0], nst, false, true);
        else if (kXtra == 2 && st + nst < n_stages) issue_slice(kts[st], st + nst, true, true);
      }
    }
    // the further stages, this warp's 16 rows each: patch, scores, running
    // max, P V, then the slice takes the stage nst further on
    for (int xs = nst; extra && xs < (kXtra == 1 ? nst + 1 : n_stages); ++xs) {
      // stage xs is group 2 + (xs - nst) of this warp's (K and V of stage nst
      // are groups 1 and 2): younger groups may stay pending
      if (kXtra == 1) cp_async_wait<0>();
      else cp_async_wait_dyn(xg - (2 + (xs - nst)));
      __syncwarp();
      const uint32_t kt = rg.buf0 + (uint32_t)((g0 + xs) % nst) * 2u * kTileBytes<D>;
      const uint32_t vt = kt + kTileBytes<D>;
      const int kb = r0 + xs * kStageRows + warp * 16;
      if (kb < r1) {
        if (kb + 16 > r1 || (len >= kb && len < kb + 16)) {
          for (int i = lane; i < 16 * CH; i += 32) {
            const int rr = warp * 16 + i / CH, c = i % CH, row = kb + i / CH;
            if (row >= r1) {
              asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(vt + tile_off<D>(rr, c)),
                           "r"(0u));
            } else if (row == len) {
              const uint4 kv = s_new[c];
              const uint4 vv = s_new[CH + c];
              asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(kt + tile_off<D>(rr, c)),
                           "r"(kv.x), "r"(kv.y), "r"(kv.z), "r"(kv.w));
              asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(vt + tile_off<D>(rr, c)),
                           "r"(vv.x), "r"(vv.y), "r"(vv.z), "r"(vv.w));
            }
          }
          __syncwarp();
        }
        float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int rr = warp * 16 + (lane & 15);
#pragma unroll
          for (int s2 = 0; s2 < D / 16; ++s2) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kt + tile_off<D>(rr, 2 * s2 + (lane >> 4)), a0, a1, a2, a3);
            if (s2 & 1) mma_bf16_a4(xb, a0, a1, a2, a3, qb0[s2], qb1[s2]);
            else mma_bf16_a4(xa, a0, a1, a2, a3, qb0[s2], qb1[s2]);
          }
        }
        float xs[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = kb + g + ((e >> 1) << 3);
          xs[e] = (row < r1) ? (xa[e] + xb[e]) * sscale : -INFINITY;
        }
        float xm[2] = {fmaxf(xs[0], xs[2]), fmaxf(xs[1], xs[3])};
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          xm[0] = fmaxf(xm[0], __shfl_xor_sync(0xffffffffu, xm[0], off));
          xm[1] = fmaxf(xm[1], __shfl_xor_sync(0xffffffffu, xm[1], off));
        }
        float corr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float m_new = fmaxf(m_run[h], xm[h]);
          corr[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - m_new);
          m_run[h] = m_new;
        }
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = (xs[e] == -INFINITY) ? 0.f : exp2f(xs[e] - m_run[e & 1]);
        l_run[0] = l_run[0] * corr[0] + (p[0] + p[2]);
        l_run[1] = l_run[1] * corr[1] + (p[1] + p[3]);
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          o[j][0] *= corr[0]; o[j][1] *= corr[1];
          o[j][2] *= corr[0]; o[j][3] *= corr[1];
        }
        const uint32_t pb0 = movm_trans(pack_bf16(p[0], p[1]));
        const uint32_t pb1 = movm_trans(pack_bf16(p[2], p[3]));
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vt + tile_off<D>(rv, 2 * mt + ((lane >> 3) & 1)), a0, a1, a2, a3);
          mma_bf16_a4(o[mt], a0, a1, a2, a3, pb0, pb1);
        }
      }
      if (kXtra == 2 && xs + nst < n_stages) {   // this warp's rows of the slice are consumed
        __syncwarp();
        issue_slice(kt, xs + nst, true, true);
      }
    }
  } else
  for (int st = 0; st < n_stages; ++st) {
    const int gi = g0 + st, b = gi % nst;
    if constexpr (kTma) {
      if (!tc::mbar_wait(rg.bar0 + 8u * b, (uint32_t)(gi / nst) & 1u) && lane == 0)
        record_error(err, DEV_TIMEOUT);
    } else {
      cp_async_wait_dyn(issued - (st + 1));   // groups younger than stage st may stay pending
      __syncthreads();
    }
    const uint32_t kt = rg.buf0 + (uint32_t)b * 2u * kTileBytes<D>;
    const uint32_t vt = kt + kTileBytes<D>;
    const int kb = r0 + st * kStageRows + warp * 16;   // this warp's 16 rows
    if (kb < r1) {
      // this warp's rows past r1 (V zeroed: 0 * garbage must not reach O) and
      // the new row, which CTA 0 is writing to the cache meanwhile
      if (kb + 16 > r1 || (len >= kb && len < kb + 16)) {
        for (int i = lane; i < 16 * CH; i += 32) {
          const int rr = warp * 16 + i / CH, c = i % CH, row = kb + i / CH;
          if (row >= r1) {
            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(vt + tile_off<D>(rr, c)),
                         "r"(0u));
          } else if (row == len) {
            const uint4 kv = s_new[c];
            const uint4 vv = s_new[CH + c];
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(kt + tile_off<D>(rr, c)),
                         "r"(kv.x), "r"(kv.y), "r"(kv.z), "r"(kv.w));
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(vt + tile_off<D>(rr, c)),
                         "r"(vv.x), "r"(vv.y), "r"(vv.z), "r"(vv.w));
          }
        }
        if constexpr (kTma) tc::fence_proxy_async();   // generic writes before the next TMA load
        __syncwarp();
      }
      // scores S[row][head] for rows kb..kb+15: one 16-row A tile per 16
      // dims (two accumulators, even and odd steps, for independent chains)
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int rr = warp * 16 + (lane & 15);
#pragma unroll
        for (int s2 = 0; s2 < D / 16; ++s2) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kt + tile_off<D>(rr, 2 * s2 + (lane >> 4)), a0, a1, a2, a3);
          if (s2 & 1) mma_bf16_a4(sb, a0, a1, a2, a3, qb0[s2], qb1[s2]);
          else mma_bf16_a4(sa, a0, a1, a2, a3, qb0[s2], qb1[s2]);
        }
      }
      // mask rows past r1, scale; sc[0..1]: row kb+g, sc[2..3]: row kb+g+8
      float sc[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = kb + g + ((e >> 1) << 3);
        sc[e] = (row < r1) ? (sa[e] + sb[e]) * sscale : -INFINITY;
      }
      // block max per head over the 16 rows (lanes of a head: same t)
      float mx[2] = {fmaxf(sc[0], sc[2]), fmaxf(sc[1], sc[3])};
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], off));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], off));
      }
      float corr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float m_new = fmaxf(m_run[h], mx[h]);
        corr[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - m_new);
        m_run[h] = m_new;
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = (sc[e] == -INFINITY) ? 0.f : exp2f(sc[e] - m_run[e & 1]);
      l_run[0] = l_run[0] * corr[0] + (p[0] + p[2]);
      l_run[1] = l_run[1] * corr[1] + (p[1] + p[3]);
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        o[j][0] *= corr[0]; o[j][1] *= corr[1];
        o[j][2] *= corr[0]; o[j][3] *= corr[1];
      }
      // P as the B operand (rows on K, heads on N): transpose the two 8x8
      // blocks of the score fragment (rows 0-7, rows 8-15)
      const uint32_t pb0 = movm_trans(pack_bf16(p[0], p[1]));
      const uint32_t pb1 = movm_trans(pack_bf16(p[2], p[3]));
      // O^T[dims][head] += V^T P: V^T as A tiles (16 dims x 16 rows) from the
      // row-major V stage with transposing loads
      const int rv = warp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vt + tile_off<D>(rv, 2 * mt + ((lane >> 3) & 1)), a0, a1, a2, a3);
        mma_bf16_a4(o[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncthreads();   // buffer b consumed by every warp
    if (st + nst < n_stages) {
      if constexpr (kTma) {
        if (tid == 0)
          ring_issue<D>(rg, tmK, tmV, g0 + st + nst, x0, y0 + r0 + (st + nst) * kStageRows, err);
      } else {
        ring_issue_lsu<D>(rg, Kb, Vb, row_stride, g0 + st + nst, r0 + (st + nst) * kStageRows, hi);
        ++issued;
      }
    }
  }
  // loads issued ahead that this block did not use must land before the
  // buffers are reused (s_part aliases them) or the CTA exits
  if constexpr (kTma) {
    if (tid == 0) ring_drain<D>(rg, err);
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();
  // per-lane shares of each head's normaliser -> the sum over its 8 lanes
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int head = 2 * t + h;
    if (head < G) {
      if (g == 0) { s_part[warp][head].m = m_run[h]; s_part[warp][head].l = l_run[h]; }
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        s_part[warp][head].o[16 * j + g] = o[j][h];
        s_part[warp][head].o[16 * j + g + 8] = o[j][2 + h];
      }
    }
  }
}

// ---- attention, fp32 CUDA-core path --------------------------------------------
template <int D, int G>
__device__ void attend_f32(const float* __restrict__ Kb, const float* __restrict__ Vb,
                           size_t row_stride, const float* kn, const float* vn, int len, int r0,
                           int r1, const float (*s_q)[D], Partial<D> (*s_part)[G]) {
  constexpr int LPR = D / 8;
  constexpr int RPW = 32 / LPR;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int team = lane / LPR, tl = lane % LPR;
  const float qscale = kLog2e * rsqrtf((float)D);
  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] = s_q[g][tl * 8 + e] * qscale;
  float m_run[G], l_run[G], o_acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY; l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o_acc[g][e] = 0.f;
  }
  for (int base = r0 + warp * RPW; base < r1; base += 4 * RPW) {
    const int row = base + team;
    const bool valid = row < r1;
    float kf[8], vf[8];
    if (valid) {
      const float* kp = (row == len) ? kn : Kb + (size_t)row * row_stride;
      const float* vp = (row == len) ? vn : Vb + (size_t)row * row_stride;
      load8<float>(kp + tl * 8, kf);
      load8<float>(vp + tl * 8, vf);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) { kf[e] = 0.f; vf[e] = 0.f; }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(qf[g][e], kf[e], a);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (valid) {
        const float mn = fmaxf(m_run[g], a);
        const float sc = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - mn);
        const float p = exp2f(a - mn);
        l_run[g] = l_run[g] * sc + p;
#pragma unroll
        for (int e = 0; e < 8; ++e) o_acc[g][e] = fmaf(o_acc[g][e], sc, p * vf[e]);
        m_run[g] = mn;
      }
    }
  }
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
}

// Merge the per-warp states w_part[0..3][g] into dst[g] (all threads of the
// block; ends with a barrier). dst may be another CTA's shared memory: each
// thread writes 4 consecutive columns with one 16-byte store.
template <int D, int G>
__device__ void merge_warps(const Partial<D> (*w_part)[G], uint32_t dst, uint32_t bar) {
  // dst, bar: this CTA's slots in the merge CTA and that CTA's push barrier
  // (shared::cluster addresses); every byte written counts on the barrier
  const int tid = threadIdx.x;
  __syncthreads();
  for (int i = tid; i < G * D / 4; i += kThreads) {
    const int g = (4 * i) / D, c = (4 * i) % D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, w_part[w][g].m);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      if (w_part[w][g].m != -INFINITY) {
        const float sc = exp2f(w_part[w][g].m - mx);
        const float4 v = *reinterpret_cast<const float4*>(&w_part[w][g].o[c]);
        o.x = fmaf(v.x, sc, o.x); o.y = fmaf(v.y, sc, o.y);
        o.z = fmaf(v.z, sc, o.z); o.w = fmaf(v.w, sc, o.w);
      }
    }
    tc::st_async_v4(dst + (uint32_t)(g * sizeof(Partial<D>) + 16 + 4 * c), o.x, o.y, o.z, o.w,
                    bar);
  }
  if (tid < G) {
    float mx = -INFINITY;
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, w_part[w][tid].m);
    float l = 0.f;
    for (int w = 0; w < 4; ++w)
      if (w_part[w][tid].m != -INFINITY) l += w_part[w][tid].l * exp2f(w_part[w][tid].m - mx);
    tc::st_async_v2(dst + (uint32_t)(tid * sizeof(Partial<D>)), mx, l, bar);
  }
}

// Bytes that one attention CTA pushes into the merge CTA (G heads: o, m, l).
template <int D, int G>
constexpr uint32_t push_bytes() { return (uint32_t)G * (4u * D + 8u); }

// Readout CTA: cp.async loads of b [r], s_v [D] (moment mode) and, if with_M,
// M [r][D] of one unit into shared memory, as one commit group.
template <int D>
__device__ void stage_readout_state(int unit, int r, const float* __restrict__ bstab,
                                    const float* __restrict__ s_v, const float* __restrict__ M,
                                    int moment, bool with_M, float* sb, float* ssv, float* sM) {
  const int tid = threadIdx.x;
  for (int i = tid; i < r / 4; i += kThreads)
    cp_async16(smem_u32(sb) + (uint32_t)i * 16u, bstab + (size_t)unit * r + 4 * i, true);
  if (moment)
    for (int i = tid; i < D / 4; i += kThreads)
      cp_async16(smem_u32(ssv) + (uint32_t)i * 16u, s_v + (size_t)unit * D + 4 * i, true);
  if (with_M) {
    const float* Mu = M + (size_t)unit * r * D;
    for (int i = tid; i < r * D / 4; i += kThreads)
      cp_async16(smem_u32(sM) + (uint32_t)i * 16u, Mu + 4 * i, true);
  }
  cp_async_commit();
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Cache rows per attention CTA for n rows over S CTAs: ceil(n / S) rounded up
// to 16 (one warp's rows of a stage), so that the split changes only every
// 16 S rows and a split chosen from a slightly stale length is usually right.
__device__ __forceinline__ int split_rows(int n, int S) { return ((n + S - 1) / S + 15) & ~15; }

__device__ __forceinline__ int ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Dynamic shared memory of one decode CTA (bytes). Attention CTAs use
// [0, att) for their row stages (then for the per-warp states); the readout
// CTA uses [0, readout) for its operands and result and receives the S
// attention states in [slot_off, slot_off + S * G * sizeof(Partial<D>)).
template <int D, int G>
struct DecSmem {
  static size_t att(bool bf16, int nst) {   // stage ring + slack for its 1024-byte alignment
    return bf16 ? (size_t)nst * 2 * kStageRows * D * 2 + 1024 : 0;
  }
  static constexpr size_t warps() { return (size_t)4 * G * sizeof(Partial<D>); }
  static_assert((kThreads / (D / 4)) * D == 4 * kThreads, "M^T u partials: RG * D = 4 * kThreads");
  // W_phi | b | u | den | gate | M^T u partials | g m | s_v | w_gate | M
  // (m_in_w: M shares the W_phi region)
  static size_t readout(int r, bool moment) {
    return ((size_t)r * D + r + (size_t)G * r + 2 * G + (size_t)4 * kThreads * G + (size_t)G * D +
            D + (size_t)G * D + (moment ? 0 : (size_t)r * D)) * sizeof(float);
  }
  static size_t slot_off(int r, bool moment) { return (readout(r, moment) + 127) / 128 * 128; }
  static size_t total(bool bf16, int nst, int r, int S, bool moment) {
    size_t w = att(bf16, nst);
    if (warps() > w) w = warps();
    const size_t rs = slot_off(r, moment) + (size_t)S * G * sizeof(Partial<D>);
    return rs > w ? rs : w;
  }
};

template <typename T, int D, int G, bool kTma, int NRO, int kXtra>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
              T* __restrict__ K_ret, T* __restrict__ V_ret, int32_t* __restrict__ cache_len,
              int cap, int Hkv, const float* __restrict__ M, const float* __restrict__ bstab,
              const float* __restrict__ s_v, const float* __restrict__ n_e, int moment,
              const float* __restrict__ W_phi, const float* __restrict__ w_gate, int r, float eps,
              float gate_override, int use_override, T* __restrict__ out,
              int* __restrict__ seq_counters, int* __restrict__ err, uint32_t slot_off, int nst,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(128) unsigned char dyn_smem[];
  cg::cluster_group cluster = cg::this_cluster();
  // Readout CTAs per cluster (NRO): two, each for half of the query heads of
  // the group, where the grid still fits one wave with the extra CTA (the
  // readout's products on 128 threads are then the critical path); CTA S
  // merges, CTA S + 1 pushes its readout to it.
  static_assert(NRO == 1 || (NRO == 2 && !kTma && G >= 2), "two readout CTAs: one-wave grids, G >= 2");
  constexpr int kNro = NRO;
  constexpr int HG = G / kNro;              // query heads per readout CTA
  const int S = gridDim.x - kNro;           // attention CTAs; CTA S = readout and merge
  const int rank = blockIdx.x;              // the cluster spans blockIdx.x
  const int kh = blockIdx.y, bi = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = Hkv * G;
  const int unit = bi * Hkv + kh;
  // per sequence: 1 + the length the last decode step left, 0 if another
  // call wrote the cache state since (see "Early loads")
  int* __restrict__ dec_tag = seq_counters + gridDim.z;

  __shared__ __align__(16) float s_q[G][D];
  __shared__ __align__(16) uint4 s_newrow[2 * D / 8];   // the new row: k_new | v_new (bf16)
  __shared__ float s_w[kDecodeMaxSplits][G];
  __shared__ float s_l[G];
  __shared__ int s_len_hint;
  __shared__ float s_wr[G], s_kq[G];   // moment readout: w_R and q.k_bar per head
  __shared__ __align__(8) uint64_t s_bar[kDecodeMaxStages];
  // the merge CTA's push barrier: completes when the attention CTAs' states
  // (and the second readout CTA's heads) have landed in its shared memory
  __shared__ __align__(8) uint64_t s_pushbar;
  Partial<D>* slots = reinterpret_cast<Partial<D>*>(dyn_smem + slot_off);   // readout CTA only
  if (rank == S && tid == 0) {   // before this CTA's arrival on the cluster barrier
    tc::mbar_init(smem_u32(&s_pushbar), 1);
    tc::fence_mbar_init();
  }

  // readout CTA's shared memory (see DecSmem::readout)
  constexpr int RG = kThreads / (D / 4);                    // row groups of the M^T u partials
  float* sW = reinterpret_cast<float*>(dyn_smem);          // [r][D] W_phi, 16-byte chunks XOR-swizzled
  float* sb = sW + (size_t)r * D;                           // [r]
  float* su = sb + r;                                       // [G][r]
  float* sden = su + G * r;                                 // [G]
  float* sgate = sden + G;                                  // [G]
  float* snum = sgate + G;                                  // [RG][G][D] partial M^T u
  float* ro = snum + RG * G * D;                            // [G][D] = g * m (moment: S q)
  float* ssv = ro + G * D;                                  // [D] moment: s_v of this unit
  float* sG = ssv + D;                                      // [G][D] w_gate rows of the group
  // [r][D] M of this unit: its own region in a one-wave grid (staged early,
  // latency), the W_phi region otherwise (staged after u, occupancy)
  float* sM = (moment || kTma) ? sW : sG + G * D;
  if (rank >= S && !moment) {
    // W_phi and w_gate belong to the context and are written only at
    // imem_init, so the readout CTA stages them before waiting for the
    // previous kernel (the moment readout uses neither: u = q, no gate)
    const uint32_t wdst = smem_u32(sW);
    for (int i = tid; i < r * D / 4; i += kThreads) {
      const int j = (4 * i) / D, cc = ((4 * i) % D) / 4;
      cp_async16(wdst + (uint32_t)(j * D + ((cc ^ (j & 7)) * 4)) * 4u, W_phi + 4 * i, true);
    }
    for (int i = tid; i < G * D / 4; i += kThreads)
      cp_async16(smem_u32(sG) + (uint32_t)i * 16u, w_gate + (size_t)kh * G * D + 4 * i, true);
    cp_async_commit();
  }
  // early b (and s_v) and M, where M has a region of its own: kept if the
  // check after the wait finds that no other kernel can have changed them
  const bool ro_early = moment || !kTma;
  if (rank >= S && ro_early) stage_readout_state<D>(unit, r, bstab, s_v, M, moment, true, sb, ssv, sM);
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  const size_t row_stride = (size_t)Hkv * D;
  const T* Kb = K_ret + (size_t)bi * cap * row_stride + (size_t)kh * D;
  const T* Vb = V_ret + (size_t)bi * cap * row_stride + (size_t)kh * D;
  Ring ring;
  ring.buf0 = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  ring.bar0 = smem_u32(s_bar);
  ring.nst = nst;
#pragma unroll
  for (int b = 0; b < kDecodeMaxStages; ++b) ring.last[b] = -1;
  // A hint of cache_len, read before the wait (relaxed: the previous kernel
  // may be advancing it). It picks this CTA's block under the split the hint
  // gives; the true length read after the wait decides.
  if (kBf16 && rank < S) {
    if (tid == 0) {
      if (kTma) {
        for (int b = 0; b < nst; ++b) tc::mbar_init(ring.bar0 + 8u * b, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
      }
      s_len_hint = max(0, min(ld_relaxed(cache_len + bi), cap - 1));
    }
    __syncthreads();
  }
  // Early loads. The first stages of the hinted block (n = hint + 1 or + 2)
  // are issued before the wait, as far as row hint - 2: the previous decode
  // step may still be appending row hint - 1 or hint. The remaining rows of
  // those stages are issued after the wait if the check there accepts them.
  int len_h = 0, per_h = 0, r0h = 0, blk_h = 0, pre_lim = 0, n_spec = 0, n_full = 0;
  if constexpr (kBf16) {
    if (rank < S) {
      len_h = s_len_hint;
      per_h = split_rows(len_h + 1, S);
      r0h = rank * per_h;
      blk_h = min(min(r0h + per_h, len_h + 2), cap);
      n_spec = blk_h > r0h ? min(nst, (blk_h - r0h + kStageRows - 1) / kStageRows) : 0;
      if constexpr (!kTma) {
        pre_lim = min(blk_h, max(r0h, len_h - 1));
        for (int st = 0; st < n_spec; ++st) {
          const int a = r0h + st * kStageRows, e = min(a + kStageRows, blk_h);
          if (a >= pre_lim) break;
          ring_issue_rows<D>(ring, Kb, Vb, row_stride, st, a, a, min(e, pre_lim));
          if (e > pre_lim) break;   // the stage holding row pre_lim stays an open group
          cp_async_commit();
          ++n_full;
        }
      }
    }
  }
  // The lines this step reads right after the wait, pulled into L2 while it
  // waits (a prefetch binds no value: a write by the kernel being waited for
  // still lands in L2 before the loads below read it).
  if (tid < G * D / 8) {
    const T* qp = q + ((size_t)bi * Hq + kh * G) * D + 8 * tid;
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(qp));
  }
  if (rank < S && tid < 2 * D / 8) {
    const T* np = (tid < D / 8 ? k_new : v_new) + ((size_t)bi * Hkv + kh) * D + 8 * (tid % (D / 8));
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(np));
  }
  // With programmatic dependent launch this kernel may start while the
  // previous kernel of the stream is still running: wait for it before
  // relying on anything another kernel may write (q, the cache, cache_len,
  // M, b).
  griddep_wait();
  // this step's own inputs first (q, cache_len), so that their loads do not
  // queue behind the row loads issued next
  static_assert(D % 8 == 0 && G * D / 8 <= kThreads, "q is read in groups of 8, one per thread");
  uint4 qraw[sizeof(T) / 2];   // 8 elements of q
  const bool qv = tid < G * D / 8;
  if (qv) {
    const uint4* qs = reinterpret_cast<const uint4*>(q + ((size_t)bi * Hq + kh * G) * D + 8 * tid);
#pragma unroll
    for (int e = 0; e < (int)(sizeof(T) / 2); ++e) qraw[e] = __ldcg(qs + e);
  }
  if (kBf16 && rank < S && tid < 2 * D / 8) {
    // the new row, read with q: the attention loop then patches it in from
    // shared memory instead of a round trip to L2 inside the loop
    const T* src = (tid < D / 8 ? k_new : v_new) + ((size_t)bi * Hkv + kh) * D;
    s_newrow[tid] = __ldcg(reinterpret_cast<const uint4*>(src) + (tid % (D / 8)));
  }
  const int len = __ldcg(cache_len + bi);
  const int tag = __ldcg(dec_tag + bi);
  if constexpr (kBf16 && kTma) {
    // TMA staging issues its early stages only now (one thread, few
    // instructions): the first stages of the hinted block
    if (rank < S && tid == 0)
      for (int st = 0; st < n_spec; ++st)
        ring_issue<D>(ring, &tmK, &tmV, st, kh * D, bi * cap + r0h + st * kStageRows, err);
  }
  if (qv) {
    float f[8];
    load8<T>(reinterpret_cast<const T*>(qraw), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) s_q[(8 * tid + e) / D][(8 * tid + e) % D] = f[e];
  }
  if (len >= cap) {   // full cache: the whole cluster (same sequence) skips it
    if (rank == 0 && kh == 0 && tid == 0) record_error(err, DEV_CACHE_FULL);
    if (kTma && tid == 0) ring_drain<D>(ring, err);
    cp_async_commit();   // closes an open group of early rows
    cp_async_wait<0>();
    return;
  }
  // phase 0 of the cluster barrier: "this CTA is running and has read
  // cache_len" (remote shared memory is written only after every CTA of the
  // cluster has arrived; cache_len is advanced only after every unit's CTAs
  // have arrived). Relaxed: a release arrive would also wait for this CTA's
  // loads in flight; every thread has branched on the length it loaded, so
  // that read has returned its value before the arrive.
  cluster_arrive_relaxed();
  griddep_launch();
  const int n = len + 1;
  // The early stages are this CTA's first stages if the true length gives the
  // same split. Rows loaded before the wait also need that no kernel which
  // may have been running then wrote them: tag == len + 1 says that the last
  // writer of this sequence's cache state was a decode step that left this
  // length (every other call of the library clears the tag), and the hint is
  // then len or len - 1, so those rows lie below the row that step appended.
  bool hit = split_rows(n, S) == per_h;
  if constexpr (!kTma) {
    hit = hit && tag == len + 1 && (len_h == len || len_h + 1 == len);
    if constexpr (kBf16) {
      if (rank < S && n_spec > 0) {
        if (hit) {
          // the rest of the early stages: from row pre_lim to the block's end
          for (int st = n_full; st < n_spec; ++st) {
            const int a = r0h + st * kStageRows, e = min(a + kStageRows, blk_h);
            ring_issue_rows<D>(ring, Kb, Vb, row_stride, st, a, max(a, pre_lim), e);
            cp_async_commit();
          }
        } else {
          cp_async_commit();   // closes an open group
          cp_async_wait<0>();  // drop them; the barrier below frees the buffers
          n_spec = 0;
        }
      }
    }
  }
  __syncthreads();

  if (rank < S) {
    const T* kn = k_new + ((size_t)bi * Hkv + kh) * D;
    const T* vn = v_new + ((size_t)bi * Hkv + kh) * D;
    if (rank == 0) {   // append the new row
      T* kd = K_ret + ((size_t)bi * cap + len) * row_stride + (size_t)kh * D;
      T* vd = V_ret + ((size_t)bi * cap + len) * row_stride + (size_t)kh * D;
      for (int c = tid; c < D; c += kThreads) { kd[c] = kn[c]; vd[c] = vn[c]; }
    }
    const int per = split_rows(n, S);
    const int r0 = min(n, rank * per), r1 = min(n, r0 + per);
    auto* w_part = reinterpret_cast<Partial<D>(*)[G]>(dyn_smem);   // aliases the stages
    if constexpr (kBf16) {
      // a miss leaves TMA stages 0..n_spec-1 spent: the block starts after them
      attend_bf16<D, G, kTma, kXtra>(ring, &tmK, &tmV, kh * D, bi * cap, Kb, Vb, row_stride, r1, kn, vn,
                              len, r0, r1, hit ? 0 : n_spec, hit ? n_spec : 0, s_q, w_part, err,
                              s_newrow);
    }
    else
      attend_f32<D, G>(Kb, Vb, row_stride, kn, vn, len, r0, r1, s_q, w_part);
    cluster_wait();   // phase 0 complete: every CTA of the cluster is running
    // CTA 0 counts the unit on its sequence's counter (every CTA of the unit
    // has read cache_len: each branched on the length it loaded before
    // arriving on the barrier just completed, so those loads have returned
    // their values); the last unit of the sequence advances cache_len. A
    // relaxed atomic whose result is used last, so that its round trip
    // overlaps the push (an acquire would stall the warp here).
    int arrived = 0;
    if (rank == 0 && tid == 0) arrived = atomicAdd(&seq_counters[bi], 1);
    // push this CTA's merged state into the readout CTA's slot (asynchronous
    // stores counted on its push barrier: nothing to wait for here)
    merge_warps<D, G>(w_part, tc::mapa(smem_u32(slots + (size_t)rank * G), S),
                      tc::mapa(smem_u32(&s_pushbar), S));
    if (rank == 0 && tid == 0 && arrived == Hkv - 1) {
      seq_counters[bi] = 0;
      cache_len[bi] = len + 1;
      dec_tag[bi] = len + 2;
    }
    return;
  }

  // ---- readout CTA: u = W_phi q, m = M^T u / (b.u + eps), g = sigmoid(w_gate . q)
  // for the heads [hg0, hg0 + HG) of this readout CTA
  const int hg0 = (rank - S) * HG;
  if (!ro_early || tag != len + 1) {
    // b (and s_v) and, where it has its own region, M: loaded now (the early
    // copies, if any, land first and are overwritten)
    if (ro_early) cp_async_wait<0>();
    stage_readout_state<D>(unit, r, bstab, s_v, M, moment, ro_early, sb, ssv, sM);
  }
  const float ne = moment ? __ldcg(n_e + bi) : 0.f;
  cp_async_wait<0>();
  __syncthreads();
  // gate: z = w_gate[h] . q (none in moment mode)
  for (int gg = warp; gg < HG && !moment; gg += kThreads / 32) {
    const int g = hg0 + gg;
    float z = 0.f;
    for (int c = lane; c < D; c += 32) z = fmaf(sG[g * D + c], s_q[g][c], z);
    z = warp_sum(z);
    if (lane == 0) sgate[g] = use_override ? gate_override : sigmoidf_(z);
  }
  if (moment) {
    for (int o = tid; o < HG * r; o += kThreads)   // u = q
      su[(hg0 + o / r) * r + o % r] = s_q[hg0 + o / r][o % r];
  } else {
    // u = W_phi q: a pair of threads per row of W_phi (one half each), all G
    // heads at once, so that each row is read once (q is a broadcast read)
    for (int o = tid; o < 2 * r; o += kThreads) {
      const int j = o >> 1, half = o & 1;
      const float4* wr = reinterpret_cast<const float4*>(sW + (size_t)j * D);
      float acc[HG];
#pragma unroll
      for (int gg = 0; gg < HG; ++gg) acc[gg] = 0.f;
#pragma unroll 4
      for (int cc = half * (D / 8); cc < (half + 1) * (D / 8); ++cc) {
        const float4 w = wr[cc ^ (j & 7)];
#pragma unroll
        for (int gg = 0; gg < HG; ++gg) {
          const float4 x = reinterpret_cast<const float4*>(&s_q[hg0 + gg][0])[cc];
          acc[gg] = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, acc[gg]))));
        }
      }
#pragma unroll
      for (int gg = 0; gg < HG; ++gg) {
        acc[gg] += __shfl_xor_sync(0xffffffffu, acc[gg], 1);
        if (half == 0) su[(hg0 + gg) * r + j] = acc[gg];
      }
    }
    if (kTma) {
      // M into the W_phi region, now that every thread is done with W_phi
      __syncthreads();
      const float* Mu = M + (size_t)unit * r * D;
      for (int i = tid; i < r * D / 4; i += kThreads)
        cp_async16(smem_u32(sM) + (uint32_t)i * 16u, Mu + 4 * i, true);
      cp_async_commit();
      cp_async_wait<0>();
    }
  }
  __syncthreads();
  for (int gg = warp; gg < HG; gg += kThreads / 32) {
    const int g = hg0 + gg;
    float a = 0.f;
    for (int j = lane; j < r; j += 32) a = fmaf(sb[j], su[g * r + j], a);
    a = warp_sum(a);
    if (lane == 0) sden[g] = moment ? a : a + eps;   // moment: s_k . q
  }
  {
    // partial M^T u over this thread's rows, for its 4 columns and every head
    const int cq = tid % (D / 4), rg = tid / (D / 4);       // D/4 column quads, RG row groups
    float4 acc[HG];
#pragma unroll
    for (int gg = 0; gg < HG; ++gg) acc[gg] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int j = rg; j < r; j += RG) {
      const float4 mv = reinterpret_cast<const float4*>(sM + (size_t)j * D)[cq];
#pragma unroll
      for (int gg = 0; gg < HG; ++gg) {
        const float uu = su[(hg0 + gg) * r + j];
        acc[gg].x = fmaf(mv.x, uu, acc[gg].x);
        acc[gg].y = fmaf(mv.y, uu, acc[gg].y);
        acc[gg].z = fmaf(mv.z, uu, acc[gg].z);
        acc[gg].w = fmaf(mv.w, uu, acc[gg].w);
      }
    }
#pragma unroll
    for (int gg = 0; gg < HG; ++gg)
      reinterpret_cast<float4*>(snum + ((size_t)rg * G + hg0 + gg) * D)[cq] = acc[gg];
  }
  __syncthreads();
  for (int i = hg0 * D + tid; i < (hg0 + HG) * D; i += kThreads) {
    const int g = i / D, c = i % D;
    float num = 0.f;
#pragma unroll
    for (int k = 0; k < RG; ++k) num += snum[((size_t)k * G + g) * D + c];
    ro[i] = moment ? num : sgate[g] * (num / sden[g]);
  }
  __syncthreads();
  if (kNro > 1 && rank > S) {
    // the second readout CTA: its heads' readout (and b . u, which the
    // moment readout's merge needs) into the merge CTA, then arrive
    cluster_wait();   // phase 0: the merge CTA is running (its push barrier is set up)
    const uint32_t bar = tc::mapa(smem_u32(&s_pushbar), S);
    for (int i = hg0 * D + tid; i < (hg0 + HG) * D; i += kThreads)
      tc::st_async_f32(tc::mapa(smem_u32(ro + i), S), ro[i], bar);
    if (tid < HG) tc::st_async_f32(tc::mapa(smem_u32(sden + hg0 + tid), S), sden[hg0 + tid], bar);
    return;
  }

  // ---- merge the S attention states that the other CTAs pushed into the slots
  cluster_wait();   // phase 0: every CTA of the cluster is running
  // every attention CTA's state (and the second readout CTA's heads): the
  // bytes they push, counted on this CTA's push barrier
  if (tid == 0)
    tc::mbar_expect_tx(smem_u32(&s_pushbar),
                       (uint32_t)S * push_bytes<D, G>() + (uint32_t)(kNro - 1) * HG * (4u * D + 4u));
  if (!tc::mbar_wait_cluster(smem_u32(&s_pushbar), 0)) record_error(err, DEV_TIMEOUT);
  // merge weights: a warp per head, a lane per slot (S <= 15 < 32)
  for (int g = warp; g < G; g += kThreads / 32) {
    const float mt = lane < S ? slots[lane * G + g].m : -INFINITY;
    const float mx = warp_max(mt);
    const float w = (mt == -INFINITY) ? 0.f : exp2f(mt - mx);
    const float l = warp_sum(lane < S ? w * slots[lane * G + g].l : 0.f);
    if (lane < S) s_w[lane][g] = w;
    if (lane == 0) {
      s_l[g] = l;
      if (moment) {
        // Jensen: log2 Z_E = log2 n_e + (q.k_bar) log2(e) / sqrt(d);
        // log2 Z_R = mx + log2 l (logits are kept in log2 units)
        float wr = 1.f, kq = 0.f;
        if (ne > 0.f) {
          kq = sden[g] / ne;
          const float lze = log2f(ne) + kq * (kLog2e * rsqrtf((float)D));
          wr = 1.f / (1.f + exp2f(lze - (mx + log2f(l))));
        }
        s_wr[g] = wr;
        s_kq[g] = kq;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D / 4; i += kThreads) {   // 4 consecutive columns per thread
    const int g = (4 * i) / D, c = (4 * i) % D;
    float4 vals[kDecodeMaxSplits];
#pragma unroll
    for (int t2 = 0; t2 < kDecodeMaxSplits; ++t2)
      vals[t2] = t2 < S ? *reinterpret_cast<const float4*>(&slots[t2 * G + g].o[c])
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t2 = 0; t2 < kDecodeMaxSplits; ++t2) {
      const float w = t2 < S ? s_w[t2][g] : 0.f;
      o.x = fmaf(w, vals[t2].x, o.x); o.y = fmaf(w, vals[t2].y, o.y);
      o.z = fmaf(w, vals[t2].z, o.z); o.w = fmaf(w, vals[t2].w, o.w);
    }
    const float inv_l = 1.f / s_l[g];
    float res[4] = {o.x * inv_l, o.y * inv_l, o.z * inv_l, o.w * inv_l};
    if (!moment) {
#pragma unroll
      for (int e = 0; e < 4; ++e) res[e] += ro[g * D + c + e];
    } else if (s_wr[g] < 1.f) {
      // f_E = v_bar + (S q - s_v (q.k_bar)) / (n_e sqrt(d)); mix with w_R
      const float wr = s_wr[g], kq = s_kq[g], inv_ne = 1.f / ne;
      const float scl = inv_ne * rsqrtf((float)D);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float sv = ssv[c + e];
        const float fe = sv * inv_ne + (ro[g * D + c + e] - sv * kq) * scl;
        res[e] = wr * res[e] + (1.f - wr) * fe;
      }
    }
    T* op = out + ((size_t)bi * Hq + kh * G + g) * D + c;
    if constexpr (kBf16) {
      const uint32_t lo = pack_bf16(res[0], res[1]), hi = pack_bf16(res[2], res[3]);
      *reinterpret_cast<uint2*>(op) = make_uint2(lo, hi);
    } else {
      *reinterpret_cast<float4*>(op) = make_float4(res[0], res[1], res[2], res[3]);
    }
  }
}

template <typename T, int D, int G, bool kTma, int NRO, int kXtra>
cudaError_t launch_tgs(const Ctx& c, int S, int nst, int batch, const void* q, const void* kn,
                      const void* vn, void* K_ret, void* V_ret, int32_t* cache_len, int cap,
                      const float* M, const float* bstab, const float* s_v, const float* n_e,
                      void* out, int* counters, cudaStream_t st) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  const int r = c.cfg.mem_r;
  // M shares the W_phi region in moment mode and in multi-wave (TMA) grids
  const bool m_in_w = c.cfg.readout == IMEM_READOUT_MOMENT || kTma;
  const size_t smem = DecSmem<D, G>::total(kBf16, nst, r, S, m_in_w);
  const uint32_t slot_off = (uint32_t)DecSmem<D, G>::slot_off(r, m_in_w);
  auto k = decode_kernel<T, D, G, kTma, NRO, kXtra>;
  // Per instantiation and device: the largest size set so far. Host threads
  // that launch at once read it lock-free; raising it takes the mutex, so
  // that a smaller size set late cannot undercut a larger one in use.
  static std::atomic<size_t> attr_smem[64];
  static std::mutex attr_mu;
  const int dv = c.device & 63;
  if (attr_smem[dv].load(std::memory_order_acquire) < smem) {
    std::lock_guard<std::mutex> lock(attr_mu);
    if (attr_smem[dv].load(std::memory_order_relaxed) < smem) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      attr_smem[dv].store(smem, std::memory_order_release);
    }
  }
  cudaLaunchConfig_t cfg = {};
  const int nro = NRO;   // readout CTAs per cluster
  cfg.gridDim = dim3(S + nro, c.cfg.n_kv_heads, batch);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S + nro;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int use_ov = !isnan(c.cfg.gate_override);
  // bf16: the retained cache as a [batch * cap, Hkv * D] matrix, 64-row boxes
  CUtensorMap mk, mv;
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  if (kTma) {
    const uint64_t width = (uint64_t)c.cfg.n_kv_heads * D, rows = (uint64_t)batch * cap;
    if (!make_tmap_bf16(c, &mk, K_ret, width, rows, kStageRows) ||
        !make_tmap_bf16(c, &mv, V_ret, width, rows, kStageRows))
      return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, k, (const T*)q, (const T*)kn, (const T*)vn, (T*)K_ret,
                            (T*)V_ret, cache_len, cap, c.cfg.n_kv_heads, M, bstab, s_v, n_e,
                            (int)(c.cfg.readout == IMEM_READOUT_MOMENT), (const float*)c.W_phi, (const float*)c.w_gate, r, c.cfg.eps,
                            c.cfg.gate_override, use_ov, (T*)out, counters, c.err, slot_off, nst,
                            mk, mv);
}

// TMA staging when the attention CTAs stream in more than one wave (two
// CTAs per SM), cp.async staging otherwise; fp32 has no staging.
template <typename T, int D, int G>
cudaError_t launch_tg(const Ctx& c, int S, int nst, int batch, const void* q, const void* kn,
                      const void* vn, void* K_ret, void* V_ret, int32_t* cache_len, int cap,
                      const float* M, const float* bstab, const float* s_v, const float* n_e,
                      void* out, int* counters, cudaStream_t st) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  const int units = batch * c.cfg.n_kv_heads;
  const bool tma = kBf16 && units * (S + 1) > 2 * c.num_sms;
  if (tma)
    return launch_tgs<T, D, G, kBf16, 1, 0>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap, M,
                                         bstab, s_v, n_e, out, counters, st);
  // a second readout CTA where the grid keeps about 1.5 CTAs per SM with it
  if constexpr (G >= 2) {
    if (S + 2 <= kDecodeMaxSplits && units * (S + 2) * 2 <= 3 * c.num_sms + 4)
      return launch_tgs<T, D, G, false, 2, 0>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap,
                                           M, bstab, s_v, n_e, out, counters, st);
  }
  // blocks longer than the ring (one-wave bf16 grids): the variant that
  // streams the further stages warp by warp
  const int per_max = ((cap + S - 1) / S + 15) / 16 * 16;
  const int st_max = (per_max + kStageRows - 1) / kStageRows;
  if (kBf16 && nst == kDecodeMaxStages && st_max == nst + 1)
    return launch_tgs<T, D, G, false, 1, 1>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap,
                                            M, bstab, s_v, n_e, out, counters, st);
  if (kBf16 && nst == kDecodeMaxStages && st_max > nst + 1)
    return launch_tgs<T, D, G, false, 1, 2>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap,
                                            M, bstab, s_v, n_e, out, counters, st);
  return launch_tgs<T, D, G, false, 1, 0>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap,
                                          M, bstab, s_v, n_e, out, counters, st);
}

template <typename T, int D>
cudaError_t launch_t(const Ctx& c, int S, int nst, int batch, const void* q, const void* kn,
                     const void* vn, void* K_ret, void* V_ret, int32_t* cache_len, int cap,
                     const float* M, const float* bstab, const float* s_v, const float* n_e,
                     void* out, int* counters, cudaStream_t st) {
  switch (c.group) {
    case 1: return launch_tg<T, D, 1>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
    case 2: return launch_tg<T, D, 2>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
    case 4: return launch_tg<T, D, 4>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
    case 8: return launch_tg<T, D, 8>(c, S, nst, batch, q, kn, vn, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Attention CTAs per (sequence, KV head) = the cluster size minus one: about
// 1.5 CTAs per SM in one wave, at most 160 cache rows per CTA while that keeps
// the wave, no CTA streaming more than 1024 rows, clusters of at most 16.
int decode_splits(int batch, int n_kv_heads, int cap) {
  const int units = batch * n_kv_heads;
  int S = (222 + units / 2) / units - 1;
  const int by_rows = (cap + 175) / 176;   // at least ~176 rows a CTA (c1: 4 splits measured 2% faster than 5)
  if (S > by_rows) S = by_rows;
  const int by_len = (cap + 1023) / 1024;
  if (S < by_len) S = by_len;
  if (S > kDecodeMaxSplits - 1) S = kDecodeMaxSplits - 1;
  if (S < 1) S = 1;
  return S;
}

// Stages of 64 rows in an attention CTA's ring. When the whole grid fits in
// one wave at two CTAs per SM, the ring holds every stage of a CTA's block
// (all row loads in flight at once, up to 3); otherwise two, which keeps three
// CTAs per SM resident for the streaming case.
int decode_stages(int batch, int n_kv_heads, int cap, int S) {
  const int ctas = batch * n_kv_heads * (S + 1);
  if (ctas > 2 * 148) return 2;
  const int per = (cap + S - 1) / S;
  int nst = (per + kStageRows - 1) / kStageRows;
  if (nst > kDecodeMaxStages) nst = kDecodeMaxStages;   // 3 x 32 KB keeps two CTAs per SM
  if (nst < 2) nst = 2;
  return nst;
}

cudaError_t launch_decode(const Ctx& c, int batch, const void* q, const void* k_new,
                          const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                          int cap, const float* M, const float* bstab, const float* s_v,
                          const float* n_e, void* out, int* counters, cudaStream_t st) {
  const int S = decode_splits(batch, c.cfg.n_kv_heads, cap);
  const int nst = decode_stages(batch, c.cfg.n_kv_heads, cap, S);
  const int D = c.cfg.head_dim;
  if (c.cfg.dtype == IMEM_BF16) {
    if (D == 128) return launch_t<__nv_bfloat16, 128>(c, S, nst, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
    if (D == 64) return launch_t<__nv_bfloat16, 64>(c, S, nst, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
  } else {
    if (D == 128) return launch_t<float, 128>(c, S, nst, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
    if (D == 64) return launch_t<float, 64>(c, S, nst, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, s_v, n_e, out, counters, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace imem
