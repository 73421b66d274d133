// internal.h -- host-side declarations shared by the C-ABI layer and the
// kernel translation units. Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "indexmem.h"

namespace imem {

// Context of one layer: configuration, weights repacked for the kernels, and
// a device error word.
struct Ctx {
  imem_config cfg;
  int device;
  int group;            // Hq / Hkv
  // repacked weights (device, owned)
  void* WcT;            // [N1, H] model dtype: [W_ik | w_ig]^T, zero rows up to N1
  void* WqT;            // [Hq * dI, d] model dtype: W_iq[h]^T stacked by head
  int N1;               // dI + Hq rounded up to 16
  float* W_phi;         // [r, d]
  float* w_gate;        // [Hq, d]
  int* err;             // device error word
  int num_sms;          // streaming multiprocessors of the device
  void* encode_tiled;   // driver entry point cuTensorMapEncodeTiled
  // a second stream (created on first use): online eviction's new-token
  // features (forked from and joined back into the caller's stream by
  // events) and the pre-eviction's range work
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
  // pre-eviction: a range's selection, compaction and memory update run on
  // `side`, after ev_pe_fork of the caller's stream, beside the next range's
  // prologue (and the memory update beside its scoring too); ev_pe_compact
  // and ev_pe_done mark their ends. While pe_pending is set every call on the
  // context makes its stream wait for ev_pe_done before it enqueues work
  cudaEvent_t ev_pe_fork, ev_pe_compact, ev_pe_done;
  bool pe_pending;           // the last range's work on `side` may still run
  bool pe_compact_pending;   // ... and its selection and compaction too
  int pe_parity;             // candidate buffer of the next range (0 or 1)
};

// Indexer rows in the workspace: d_I features padded to 64 bf16 (128 bytes).
constexpr int kIdxPad = 64;

// 2-D TMA map over `rows` rows of 64 bf16 (128 bytes), box {64, box_rows},
// 128-byte swizzle, zero fill out of bounds. False if encoding fails.
bool make_tmap_rows64(const Ctx& c, CUtensorMap* map, const void* base, uint64_t rows,
                      uint32_t box_rows);

// 2-D TMA map over a row-major bf16 matrix [rows, width] (width * 2 bytes a
// multiple of 16), box {64, box_rows}, 128-byte swizzle, zero fill out of
// bounds. False if encoding fails.
bool make_tmap_bf16(const Ctx& c, CUtensorMap* map, const void* base, uint64_t width,
                    uint64_t rows, uint32_t box_rows);

// Layout of the caller's workspace for (batch, L).
constexpr int kOnlineMaxCluster = 16;  // KV heads (= CTAs of the online score-and-evict cluster), max

struct Workspace {
  size_t qt_off, kh_off;        // indexer q~ and k^ (bf16 [b, L, kIdxPad])
  size_t sel_off;               // selection scratch
  size_t dec_part_off;          // decode split partials
  size_t dec_cnt_off;           // decode counters (int), zero between calls
  size_t dec_tag_off;           // decode tags (int): right after the counters
  size_t on_qpart_off, on_kpart_off;   // online eviction: the new token's feature partials
  size_t mem_part_off;          // memory-update partials
  size_t sv_part_off;           // value-sum partials of the moment statistics
  size_t total;
};

constexpr int kDecodeMaxSplits = 16;          // CTAs per decode cluster (max)
constexpr int kDecodeMaxStages = 3;           // 64-row stages in a decode CTA's ring (max)
constexpr int kDecodeRowsPerSplit = 192;   // cache rows per decode CTA (target)
constexpr int kMemMaxGroups = 512;   // runs per (sequence, KV head) of the memory update (max)

Workspace workspace_layout(const Ctx& c, int batch, int L);

// Upper bound of (sequence, KV head) units x runs of the memory update for up
// to L evicted tokens per unit (the partial sums in the workspace).
size_t memory_runs_bound(int units, int L, int num_sms);

// Repacks the indexer weights K-major into c.WcT / c.WqT (allocates them).
cudaError_t pack_indexer_weights(Ctx& c, const void* W_iq, const void* W_ik, const void* w_ig);

// ---- launchers (return cudaGetLastError()) ----------------------------------

// Token t of sequence s (q_begin <= t < q_end) is written to output row
// s * out_stride + t + out_shift of qt, kh and running_max (out_stride 0: L).
cudaError_t launch_prologue(const Ctx& c, int batch, int L, const void* X, const void* Q,
                            int q_begin, int q_end, __nv_bfloat16* qt, __nv_bfloat16* kh,
                            float* running_max, cudaStream_t st, int out_stride = 0,
                            int out_shift = 0);

cudaError_t launch_scoring(const Ctx& c, int batch, int L, const __nv_bfloat16* qt,
                           const __nv_bfloat16* kh, float* running_max, int q_begin, int q_end,
                           cudaStream_t st);

cudaError_t launch_select_compact(const Ctx& c, int batch, int L, int B, const float* running_max,
                                  const void* K, const void* V, int32_t* idx_r, int32_t* idx_e,
                                  void* K_ret, void* V_ret, int cap, void* scratch,
                                  cudaStream_t st);

// Pre-eviction during chunked prefill: one query range [q0, q0 + C) over the
// candidates = n_R retained tokens + the range's C tokens, rows [0, n) of one
// of two candidate buffers (indexer keys [b, Lc, 64], importances [b, Lc], row
// stride Lc; positions of the retained rows [b, B]). Selects the B most
// important candidates and writes them, in position order, to rows [0, B) of
// the other buffer (keys, importances, positions) and their positions to
// `retained` [b, B]; the evicted positions, ascending, to `evicted`
// [b, n - B] (n = n_R + C > B). Reads nothing it writes.
struct EvictBuffers {
  __nv_bfloat16* kh_c;   // this range's candidates: keys [b, Lc, kIdxPad]
  float* I_c;            // importances [b, Lc]
  int32_t* pos_c;        // positions of the retained rows [b, B]
  __nv_bfloat16* kh_n;   // the other buffer: the rows retained after this range
  float* I_n;
  int32_t* pos_n;
  int32_t* idx_r;        // [b, B]
  int32_t* idx_e;        // [b, Lc]
};
cudaError_t launch_evict_chunk(const Ctx& c, int batch, int B, int Lc, int n_R, int q0, int C,
                               const EvictBuffers& w, int32_t* retained, int32_t* evicted,
                               cudaStream_t st);
// Appends positions q0..q0+C-1 at rows [n_R, n_R + C) of `retained` and of
// `pos` (both [b, B]).
cudaError_t launch_append_positions(int batch, int B, int n_R, int q0, int C, int32_t* retained,
                                    int32_t* pos, cudaStream_t st);
// Decode-time online eviction (online.cu).
cudaError_t launch_online_init(const Ctx& c, int batch, int L, int B, int cap,
                               const float* running_max, const int32_t* idx_r,
                               const __nv_bfloat16* kh, __nv_bfloat16* khat_ret, float* I_ret,
                               int32_t* pos_ret, int32_t* next_pos, cudaStream_t st);
cudaError_t launch_online_features(const Ctx& c, int batch, const void* x, const void* q,
                                   float* qpart, float* kpart, cudaStream_t st);
cudaError_t launch_online_score_evict(const Ctx& c, int batch, int B, int cap, const float* qpart,
                                      const float* kpart, void* khat_ret, float* I_ret,
                                      int32_t* pos_ret, int32_t* next_pos, void* K_ret, void* V_ret,
                                      int32_t* cache_len, float* M, float* bstab, int32_t* evicted,
                                      int* dec_tag, cudaStream_t st);

// A kernel whose bounded wait runs out after `limit` cycles (failure-path test).
cudaError_t launch_wait_selftest(const Ctx& c, long long limit, cudaStream_t st);

// K_ret/V_ret[:, :n] = K/V[idx[:, :n]] (idx stride `idx_stride`).
cudaError_t launch_gather(const Ctx& c, int batch, int L, int n, const int32_t* idx,
                          int idx_stride, const void* K, const void* V, void* K_ret, void* V_ret,
                          int cap, cudaStream_t st);

// sv_partials, s_v, n_count: value sums and evicted count (moment statistics);
// all three null for the plain memory update. clear_tags: n_clear ints set to
// zero on the stream before the update completes (the decode tags), or null.
cudaError_t launch_memory_update(const Ctx& c, int batch, int L, const void* K, const void* V,
                                 const int32_t* idx_e, int n_e, int chunk, float* M, float* bstab,
                                 float* partials, float* sv_partials, float* s_v, float* n_count,
                                 cudaStream_t st, int* clear_tags = nullptr, int n_clear = 0);

// s_v, n_e: the moment statistics' value sums and counts (moment readout);
// null for the gated readout.
cudaError_t launch_decode(const Ctx& c, int batch, const void* q, const void* k_new,
                          const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                          int cap, const float* M, const float* bstab, const float* s_v,
                          const float* n_e, void* out, int* counters, cudaStream_t st);

}  // namespace imem
