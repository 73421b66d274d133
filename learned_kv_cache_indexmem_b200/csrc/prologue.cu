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
// Tensor-core kernel, persistent over 128-token tiles. Per tile:
//   GEMM1 (tcgen05, K = hidden): [kI | gate logits] = X_tile [W_ik | w_ig]
//   GEMM2 (tcgen05, K = d) per head h: qI_h = Q_tile[:, h] W_iq[h]
// X and Q tiles and the repacked K-major weights arrive by TMA through a
// 6-stage ring; GEMM1 accumulates in TMEM columns [0, 128), the per-head
// GEMM2 results cycle through a ring of TMEM buffers in [128, 512). Four
// epilogue warps (one token row per thread) normalise the key, then fold each
// head into qtilde in registers (RMS norm, gate, 1/sqrt(dI)) as soon as its
// buffer is ready, and write bf16 rows of kIdxPad features.
// bf16 inputs use kind::f16, fp32 inputs kind::tf32 (same 128-byte rows).
// Also resets the running maximum of the tokens in the range to -inf (those
// keys get their first queries in this range).
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

#include <atomic>
#include <type_traits>

namespace imem {
namespace {

constexpr int kTileM = 128;
constexpr int kStageA = 128 * 128;   // 128 rows x 128 bytes
constexpr int kStageB = 128 * 128;
constexpr int kPThreads = 192;       // producer, MMA, 4 epilogue warps
constexpr int kD1Cols = 128;         // TMEM columns reserved for GEMM1
// CTA pairs: the exchange slot (one row of partial sums per token, stride
// 4 mod 8 floats so that a warp's 16-byte stores spread over the banks) and
// the gates of a CTA's 16 heads
constexpr int kPairHeads = 16;
constexpr int kSlotStride = 84;

template <int SPLIT>
struct ProSmem {
  static constexpr int NST = SPLIT == 1 ? 6 : 5;                       // ring stages
  static constexpr int BARS = 512;
  static constexpr int SLOT = SPLIT == 1 ? 0 : kTileM * kSlotStride * 4;
  static constexpr int GAM = SPLIT == 1 ? 0 : kPairHeads * kTileM * 4;
  static constexpr int TOTAL = NST * (kStageA + kStageB) + BARS + SLOT + GAM + 1024;
};

__device__ __forceinline__ void add4(float* a, float4 v) {
  a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
}

__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\ntcgen05.wait::ld.sync.aligned;\n"
               : "=r"(r) : "r"(taddr) : "memory");
  return r;
}

// SPLIT = 1: one CTA per tile. SPLIT = 2: a cluster of two CTAs per tile
// (more CTAs for short ranges: an 8192-token range is 64 tiles); CTA r
// contracts half of the hidden dimension in GEMM1 and half of the heads in
// GEMM2, the pair exchanges partial sums over distributed shared memory:
// CTA 1 sends its kI partial and the gate-logit partials of CTA 0's heads,
// CTA 0 the gate-logit partials of CTA 1's heads; after the head fold CTA 1
// sends its q~ partial, and CTA 0 writes k^, q~ and the running maximum.
// (SPLIT = 2 needs 32 query heads: 16 per CTA.)
template <typename T, int SPLIT>
__global__ void __launch_bounds__(kPThreads, 1)
prologue_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_wc, const __grid_constant__ CUtensorMap map_wq,
                   int L, int H, int Hq, int D, int dI, int N1, int q_begin, int q_end, int batch,
                   __nv_bfloat16* __restrict__ qt, __nv_bfloat16* __restrict__ kh,
                   float* __restrict__ running_max, int out_stride, int out_shift,
                   int* __restrict__ err) {
  using SM = ProSmem<SPLIT>;
  constexpr int NST = SM::NST;
  constexpr int EPB = 128 / (int)sizeof(T);                  // elements per 128-byte row
  constexpr uint32_t FMT = std::is_same<T, float>::value ? tc::kFmtTF32 : tc::kFmtBF16;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = tc::smem_addr(smem);
  const uint32_t sB = sA + NST * kStageA;
  const uint32_t bar = sB + NST * kStageB;
  const uint32_t full0 = bar, empty0 = bar + 8 * NST, d1_full = bar + 16 * NST,
                 d1_empty = d1_full + 8, rx_full = d1_empty + 8, tx_free = rx_full + 8,
                 h_full0 = tx_free + 8;
  const int NB = (512 - kD1Cols) / dI;                        // head buffers in TMEM
  const uint32_t h_empty0 = h_full0 + 8 * NB;
  float* slot = reinterpret_cast<float*>(smem + NST * (kStageA + kStageB) + SM::BARS);
  float* gam = slot + kTileM * kSlotStride;                   // [kPairHeads][kTileM]
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = SPLIT == 1 ? 0 : (int)tc::cluster_ctarank();
  const int cid = blockIdx.x / SPLIT, ncl = gridDim.x / SPLIT;
  const int tiles_per_seq = (q_end - q_begin + kTileM - 1) / kTileM;
  const int n_tiles = tiles_per_seq * batch;
  const int nk1 = H / EPB, nk2 = D / EPB;
  // this CTA's share: GEMM1 k-blocks [k1b, k1b + nk1r), heads [hb, hb + nhr)
  const int k1b = rank * (nk1 / 2), nk1r = SPLIT == 1 ? nk1 : (rank == 0 ? nk1 / 2 : nk1 - nk1 / 2);
  const int hb = rank * kPairHeads, nhr = SPLIT == 1 ? Hq : kPairHeads;
  const int n_it = nk1r + nhr * nk2;
  const uint32_t tx1 = kStageA + N1 * 128, tx2 = kStageA + dI * 128;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      tc::mbar_init(full0 + 8 * i, 1);
      tc::mbar_init(empty0 + 8 * i, 1);
    }
    tc::mbar_init(d1_full, 1);
    tc::mbar_init(d1_empty, 4);
    tc::mbar_init(rx_full, 128);   // every epilogue thread of the other CTA arrives
    tc::mbar_init(tx_free, 128);
    for (int i = 0; i < NB; ++i) {
      tc::mbar_init(h_full0 + 8 * i, 1);
      tc::mbar_init(h_empty0 + 8 * i, 4);
    }
    tc::fence_mbar_init();
    tc::prefetch_tmap(&map_x);
    tc::prefetch_tmap(&map_q);
    tc::prefetch_tmap(&map_wc);
    tc::prefetch_tmap(&map_wq);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_addr(&s_tmem), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (SPLIT > 1) tc::cluster_sync_all();   // the other CTA's barriers exist before any remote arrive
  const uint32_t tmem = s_tmem;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int st = 0, ph = 0, used = 0;
    bool ok = true;
    for (int tile = cid; tile < n_tiles && ok; tile += ncl) {
      const int seq = tile / tiles_per_seq;
      const int row = seq * L + q_begin + (tile % tiles_per_seq) * kTileM;
      for (int it = 0; it < n_it && ok; ++it) {
        if (used >= NST && !tc::mbar_wait(empty0 + 8 * st, ph ^ 1)) { ok = false; break; }
        const uint32_t full = full0 + 8 * st;
        if (it < nk1r) {
          const int kx = k1b + it;
          tc::mbar_expect_tx(full, tx1);
          tc::tma_load_2d(sA + st * kStageA, &map_x, full, kx * EPB, row);
          tc::tma_load_2d(sB + st * kStageB, &map_wc, full, kx * EPB, 0);
        } else {
          const int h = hb + (it - nk1r) / nk2, kb = (it - nk1r) % nk2;
          tc::mbar_expect_tx(full, tx2);
          tc::tma_load_2d(sA + st * kStageA, &map_q, full, h * D + kb * EPB, row);
          tc::tma_load_2d(sB + st * kStageB, &map_wq, full, kb * EPB, h * dI);
        }
        ++used;
        if (++st == NST) { st = 0; ph ^= 1; }
      }
    }
    if (!ok) record_error(err, DEV_TIMEOUT);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t id1 = tc::idesc(FMT, 128, N1, false, false);
    const uint32_t id2 = tc::idesc(FMT, 128, dI, false, false);
    int st = 0, ph = 0, tcount = 0, hcount = 0;
    bool ok = true;
    for (int tile = cid; tile < n_tiles && ok; tile += ncl, ++tcount) {
      if (tcount >= 1 && !tc::mbar_wait(d1_empty, (tcount - 1) & 1)) { ok = false; break; }
      tc::fence_after();
      for (int it = 0; it < n_it && ok; ++it) {
        const bool g2 = it >= nk1r;
        const int kb = g2 ? (it - nk1r) % nk2 : it;
        int hbuf = 0;
        if (g2) {
          hbuf = hcount % NB;
          if (kb == 0 && hcount >= NB &&
              !tc::mbar_wait(h_empty0 + 8 * hbuf, ((hcount / NB) - 1) & 1)) {
            ok = false;
            break;
          }
        }
        if (!tc::mbar_wait(full0 + 8 * st, ph)) { ok = false; break; }
        tc::fence_after();
        const uint32_t d = g2 ? tmem + kD1Cols + hbuf * dI : tmem;
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // four 32-byte K steps per 128-byte row
          const uint64_t ad = tc::sdesc_sw128(sA + st * kStageA + k * 32, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(sB + st * kStageB + k * 32, 16, 1024);
          tc::mma_f16(d, ad, bd, g2 ? id2 : id1, (kb > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(empty0 + 8 * st);
        if (!g2 && it == nk1r - 1) tc::mma_commit(d1_full);
        if (g2 && kb == nk2 - 1) {
          tc::mma_commit(h_full0 + 8 * hbuf);
          ++hcount;
        }
        if (++st == NST) { st = 0; ph ^= 1; }
      }
    }
    if (!ok) record_error(err, DEV_TIMEOUT);
  } else if (warp >= 2) {
    // ---------------- epilogue: one token row per thread
    const int quarter = warp & 3;
    const int trow = quarter * 32 + lane;                     // token row in the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float inv_sqrt_dI = rsqrtf((float)dI);
    // pairs: this row of the own slot, the same row of the other CTA's slot,
    // and the other CTA's barriers
    const uint32_t peer = (uint32_t)(rank ^ 1);
    const uint32_t slot_own = tc::smem_addr(slot) + (uint32_t)(trow * kSlotStride * 4);
    const uint32_t slot_rem = SPLIT > 1 ? tc::mapa(slot_own, peer) : 0u;
    const uint32_t rx_rem = SPLIT > 1 ? tc::mapa(rx_full, peer) : 0u;
    const uint32_t tx_rem = SPLIT > 1 ? tc::mapa(tx_free, peer) : 0u;
    const float* srow = slot + trow * kSlotStride;
    int tcount = 0, hcount = 0, n_tx = 0, n_rx = 0;
    bool ok = true;
    for (int tile = cid; tile < n_tiles && ok; tile += ncl, ++tcount) {
      const int seq = tile / tiles_per_seq;
      const int t = q_begin + (tile % tiles_per_seq) * kTileM + trow;
      const bool valid = t < q_end;
      const size_t row = (size_t)seq * out_stride + t + out_shift;   // output row of token t
      if (!tc::mbar_wait(d1_full, tcount & 1)) { ok = false; break; }
      tc::fence_after();
      float acc[64];
      bool write_k = true;
      if constexpr (SPLIT > 1) {
        // 1. the partial sums the other CTA needs: CTA 0 -> 1 the gate logits
        //    of heads [16, 32); CTA 1 -> 0 kI and the gate logits of [0, 16)
        const int s0 = rank == 0 ? dI + kPairHeads : 0;
        const int s1 = rank == 0 ? dI + 2 * kPairHeads : dI + kPairHeads;
        if (n_tx > 0 && !tc::mbar_wait_cluster(tx_free, (n_tx - 1) & 1)) { ok = false; break; }
        for (int c = s0; c < s1; c += 16) {
          float v[16];
          tc::tmem_ld16(tmem + lane_base + c, v);
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            tc::st_cluster_v4(slot_rem + (uint32_t)((c - s0 + e) * 4), v[e], v[e + 1], v[e + 2],
                              v[e + 3]);
        }
        tc::mbar_arrive_remote(rx_rem);
        ++n_tx;
        // 2. the partial sums this CTA keeps: kI (CTA 0) and its heads' logits
        float lg[kPairHeads];
        if (rank == 0) {
#pragma unroll
          for (int c = 0; c < 64; c += 16)
            if (c < dI) tc::tmem_ld16(tmem + lane_base + c, acc + c);
        }
        tc::tmem_ld16(tmem + lane_base + dI + rank * kPairHeads, lg);
        // GEMM1's columns are read: the next tile's GEMM1 may start
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(d1_empty);
        // 3. the other CTA's partial sums
        if (!tc::mbar_wait_cluster(rx_full, n_rx & 1)) { ok = false; break; }
        // 16-byte reads: a row stride of 4 mod 8 floats keeps a quarter warp's
        // 16-byte accesses on distinct banks
        const float4* s4 = reinterpret_cast<const float4*>(srow);
        if (rank == 0) {
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            if (c < dI) add4(acc + c, s4[c / 4]);
#pragma unroll
          for (int h = 0; h < kPairHeads; h += 4) add4(lg + h, s4[(dI + h) / 4]);
        } else {
#pragma unroll
          for (int h = 0; h < kPairHeads; h += 4) add4(lg + h, s4[h / 4]);
        }
        tc::mbar_arrive_remote(tx_rem);
        ++n_rx;
#pragma unroll
        for (int h = 0; h < kPairHeads; ++h) gam[h * kTileM + trow] = sigmoidf_(lg[h]);
        write_k = rank == 0;
      } else {
#pragma unroll
        for (int c = 0; c < 64; c += 16)
          if (c < dI) tc::tmem_ld16(tmem + lane_base + c, acc + c);
      }
      // shared key: RMS-normalised kI
      if (write_k) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < dI) ss = fmaf(acc[c], acc[c], ss);
        const float kinv = rsqrtf(ss / dI + 1e-6f);
        if (valid) {
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (c + e < dI) ? acc[c + e] * kinv : 0.f;
            store8<__nv_bfloat16>(kh + row * kIdxPad + c, f);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] = 0.f;
      // heads: qtilde += gamma_h / (rms_h sqrt(dI)) * qI_h
      for (int hh = 0; hh < nhr; ++hh) {
        const float gamma = SPLIT > 1 ? gam[hh * kTileM + trow]
                                      : sigmoidf_(__uint_as_float(tmem_ld1(tmem + lane_base + dI + hh)));
        const int hbuf = hcount % NB;
        if (!tc::mbar_wait(h_full0 + 8 * hbuf, (hcount / NB) & 1)) { ok = false; break; }
        tc::fence_after();
        float v[64];
        float qs = 0.f;
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          if (c < dI) {
            tc::tmem_ld16(tmem + lane_base + kD1Cols + hbuf * dI + c, v + c);
#pragma unroll
            for (int e = 0; e < 16; ++e) qs = fmaf(v[c + e], v[c + e], qs);
          }
        }
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(h_empty0 + 8 * hbuf);
        ++hcount;
        const float coef = gamma * rsqrtf(qs / dI + 1e-6f) * inv_sqrt_dI;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < dI) acc[c] = fmaf(coef, v[c], acc[c]);
      }
      if (!ok) break;
      bool write_q = true;
      if constexpr (SPLIT > 1) {
        if (rank == 1) {
          // 4. this CTA's q~ partial to CTA 0
          if (!tc::mbar_wait_cluster(tx_free, (n_tx - 1) & 1)) { ok = false; break; }
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            if (c < dI) tc::st_cluster_v4(slot_rem + (uint32_t)(c * 4), acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
          tc::mbar_arrive_remote(rx_rem);
          ++n_tx;
          write_q = false;
        } else {
          if (!tc::mbar_wait_cluster(rx_full, n_rx & 1)) { ok = false; break; }
          const float4* s4 = reinterpret_cast<const float4*>(srow);
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            if (c < dI) add4(acc + c, s4[c / 4]);
          tc::mbar_arrive_remote(tx_rem);
          ++n_rx;
        }
      } else {
        // GEMM1's columns (gate logits) are no longer needed
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(d1_empty);
      }
      if (write_q && valid) {
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = (c + e < dI) ? acc[c + e] : 0.f;
          store8<__nv_bfloat16>(qt + row * kIdxPad + c, f);
        }
        running_max[row] = -INFINITY;
      }
    }
    if (!ok) record_error(err, DEV_TIMEOUT);
  }
  tc::fence_before();
  __syncthreads();
  // the other CTA may still arrive on this CTA's barriers until it is done
  if (SPLIT > 1) tc::cluster_sync_all();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// Weight repacking at init: WcT [N1][H] = [W_ik | w_ig]^T zero-padded to N1
// rows; WqT [Hq * dI][D] with row h*dI + j = W_iq[h][:, j].
template <typename T>
__global__ void pack_weights_kernel(const T* __restrict__ W_iq, const T* __restrict__ W_ik,
                                    const T* __restrict__ w_ig, int H, int Hq, int D, int dI,
                                    int N1, T* __restrict__ WcT, T* __restrict__ WqT) {
  const size_t nwc = (size_t)N1 * H, nwq = (size_t)Hq * dI * D;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nwc + nwq;
       i += (size_t)gridDim.x * blockDim.x) {
    if (i < nwc) {
      const int n = (int)(i / H), k = (int)(i % H);
      T v = Elem<T>::from_f(0.f);
      if (n < dI) v = W_ik[(size_t)k * dI + n];
      else if (n < dI + Hq) v = w_ig[(size_t)k * Hq + (n - dI)];
      WcT[i] = v;
    } else {
      const size_t j = i - nwc;
      const int rowi = (int)(j / D), c = (int)(j % D);
      const int h = rowi / dI, jj = rowi % dI;
      WqT[j] = W_iq[((size_t)h * D + c) * dI + jj];
    }
  }
}

template <typename T>
bool make_tmap(const Ctx& c, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_rows) {
  using Fn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                          const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                          CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                          CUtensorMapFloatOOBfill);
  if (!c.encode_tiled) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * sizeof(T)};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / sizeof(T)), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      std::is_same<T, float>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return ((Fn)c.encode_tiled)(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t launch_pro(const Ctx& c, int batch, int L, const void* X, const void* Q, int q_begin,
                       int q_end, __nv_bfloat16* qt, __nv_bfloat16* kh, float* running_max,
                       int out_stride, int out_shift, cudaStream_t st) {
  const int H = c.cfg.hidden, Hq = c.cfg.n_q_heads, D = c.cfg.head_dim, dI = c.cfg.idx_dim;
  CUtensorMap mx, mq, mwc, mwq;
  if (!make_tmap<T>(c, &mx, X, (uint64_t)batch * L, H, kTileM) ||
      !make_tmap<T>(c, &mq, Q, (uint64_t)batch * L, (uint64_t)Hq * D, kTileM) ||
      !make_tmap<T>(c, &mwc, c.WcT, c.N1, H, c.N1) ||
      !make_tmap<T>(c, &mwq, c.WqT, (uint64_t)Hq * dI, D, dI))
    return cudaErrorInvalidValue;
  const int tiles = ((q_end - q_begin + kTileM - 1) / kTileM) * batch;
  // CTA pairs for 32 query heads in bf16 (the pair's exchange slot holds
  // d_I + 16 partial sums per token): each tile on two SMs, so that short
  // ranges fill the GPU and long ones end in a fuller last wave
  const bool pair = Hq == 2 * kPairHeads && dI + kPairHeads <= kSlotStride - 4 &&
                    H / (128 / (int)sizeof(T)) >= 2;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) if (pair) {
    auto k = prologue_tc_kernel<T, 2>;
    static std::atomic<uint64_t> attr_done{0};
    const uint64_t bit = 1ull << (c.device & 63);
    if (!(attr_done.load() & bit)) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           ProSmem<2>::TOTAL);
      if (e != cudaSuccess) return e;
      attr_done.fetch_or(bit);
    }
    int clusters = c.num_sms / 2;
    if (tiles < clusters) clusters = tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = ProSmem<2>::TOTAL;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, mx, mq, mwc, mwq, L, H, Hq, D, dI, c.N1, q_begin, q_end,
                              batch, qt, kh, running_max, out_stride, out_shift, c.err);
  }
  int grid = c.num_sms;
  if (tiles < grid) grid = tiles;
  auto k = prologue_tc_kernel<T, 1>;
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t bit = 1ull << (c.device & 63);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ProSmem<1>::TOTAL);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  k<<<grid, kPThreads, ProSmem<1>::TOTAL, st>>>(mx, mq, mwc, mwq, L, H, Hq, D, dI, c.N1, q_begin,
                                                q_end, batch, qt, kh, running_max, out_stride,
                                                out_shift, c.err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t pack_indexer_weights(Ctx& c, const void* W_iq, const void* W_ik, const void* w_ig) {
  const int H = c.cfg.hidden, Hq = c.cfg.n_q_heads, D = c.cfg.head_dim, dI = c.cfg.idx_dim;
  c.N1 = (dI + Hq + 15) / 16 * 16;
  const size_t es = c.cfg.dtype == IMEM_BF16 ? 2 : 4;
  cudaError_t e = cudaMalloc(&c.WcT, (size_t)c.N1 * H * es);
  if (e == cudaSuccess) e = cudaMalloc(&c.WqT, (size_t)Hq * dI * D * es);
  if (e != cudaSuccess) return e;
  if (c.cfg.dtype == IMEM_BF16)
    pack_weights_kernel<__nv_bfloat16><<<256, 256>>>(
        (const __nv_bfloat16*)W_iq, (const __nv_bfloat16*)W_ik, (const __nv_bfloat16*)w_ig, H, Hq,
        D, dI, c.N1, (__nv_bfloat16*)c.WcT, (__nv_bfloat16*)c.WqT);
  else
    pack_weights_kernel<float><<<256, 256>>>((const float*)W_iq, (const float*)W_ik,
                                             (const float*)w_ig, H, Hq, D, dI, c.N1,
                                             (float*)c.WcT, (float*)c.WqT);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  return e;
}

cudaError_t launch_prologue(const Ctx& c, int batch, int L, const void* X, const void* Q,
                            int q_begin, int q_end, __nv_bfloat16* qt, __nv_bfloat16* kh,
                            float* running_max, cudaStream_t st, int out_stride, int out_shift) {
  if (out_stride <= 0) out_stride = L;
  if (c.cfg.dtype == IMEM_BF16)
    return launch_pro<__nv_bfloat16>(c, batch, L, X, Q, q_begin, q_end, qt, kh, running_max,
                                     out_stride, out_shift, st);
  return launch_pro<float>(c, batch, L, X, Q, q_begin, q_end, qt, kh, running_max, out_stride,
                           out_shift, st);
}

}  // namespace imem
