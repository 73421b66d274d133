// api.cu -- the C ABI (include/indexmem.h): host-side validation, context
// and workspace layout, and dispatch to the kernels. Nothing here computes
// part of the method; every step runs in a kernel.
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

#include <vector>

struct imem_ctx {
  imem::Ctx c;
};

namespace imem {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Workspace workspace_layout(const Ctx& c, int batch, int L) {
  // Regions that do not depend on L come first, so that decode (which is not
  // told L) finds them at the same offsets.
  Workspace w;
  size_t off = 0;
  const size_t units = (size_t)batch * c.cfg.n_kv_heads;
  w.dec_cnt_off = off;                        // one counter per sequence, then
  w.dec_tag_off = off + (size_t)batch * sizeof(int);   // the decode tags (one per sequence)
  off = align_up(off + (size_t)2 * batch * sizeof(int), 256);
  // online eviction: the new token's feature partials
  w.on_qpart_off = off;
  off = align_up(off + (size_t)batch * c.cfg.n_q_heads * c.cfg.idx_dim * sizeof(float), 256);
  w.on_kpart_off = off;
  off = align_up(off + (size_t)batch * c.cfg.idx_dim * sizeof(float), 256);
  w.dec_part_off = off;                       // (unused: decode merges in shared memory)
  // memory partials: one d x (d+1) sum [S | s] per run of evicted tokens
  const size_t runs = memory_runs_bound((int)units, L, c.num_sms);
  w.mem_part_off = off;
  off = align_up(off + runs * (size_t)c.cfg.head_dim * (c.cfg.head_dim + 1) * sizeof(float), 256);
  w.sv_part_off = off;                        // moment mode: one d-vector per run
  if (c.cfg.readout == IMEM_READOUT_MOMENT)
    off = align_up(off + runs * (size_t)c.cfg.head_dim * sizeof(float), 256);
  w.sel_off = off;
  off = align_up(off + 256, 256);
  w.qt_off = off;
  off = align_up(off + (size_t)batch * L * kIdxPad * 2, 1024);
  w.kh_off = off;
  off = align_up(off + (size_t)batch * L * kIdxPad * 2, 1024);
  w.total = off;
  return w;
}

// The decode tag of a sequence is 1 + the cache length its last decode step
// left (0: none, as in a zero-filled workspace); a decode step uses rows and
// memory it loaded before its launch-dependency wait only when the tag is
// 1 + the length it finds after the wait. Every call that writes a retained
// cache, its length or the memory state by other means clears the tags of
// the workspace it is given.
cudaError_t clear_decode_tags(const Ctx& c, int batch, void* workspace, cudaStream_t st) {
  const Workspace w = workspace_layout(c, batch, 1);
  return cudaMemsetAsync((char*)workspace + w.dec_tag_off, 0, (size_t)batch * sizeof(int), st);
}

// Pre-eviction workspace: the plain layout over Lc = B + chunk_max candidate
// rows (its q~ region holds the range's queries, its k^ region candidate
// buffer 0's keys), then buffer 1's keys, both buffers' importances and
// retained positions, and the selection's index lists.
struct EvictWorkspace {
  Workspace base;
  size_t kh1_off, I_off[2], pos_off[2], idx_r_off, idx_e_off, total;
};

EvictWorkspace evict_workspace_layout(const Ctx& c, int batch, int B, int chunk_max) {
  const size_t Lc = (size_t)B + chunk_max;
  EvictWorkspace w;
  w.base = workspace_layout(c, batch, (int)Lc);
  size_t off = w.base.total;
  w.kh1_off = off;     off = align_up(off + (size_t)batch * Lc * kIdxPad * 2, 1024);
  w.I_off[0] = off;    off = align_up(off + (size_t)batch * Lc * sizeof(float), 256);
  w.I_off[1] = off;    off = align_up(off + (size_t)batch * Lc * sizeof(float), 256);
  w.pos_off[0] = off;  off = align_up(off + (size_t)batch * B * sizeof(int32_t), 256);
  w.pos_off[1] = off;  off = align_up(off + (size_t)batch * B * sizeof(int32_t), 256);
  w.idx_r_off = off;   off = align_up(off + (size_t)batch * B * sizeof(int32_t), 256);
  w.idx_e_off = off;   off = align_up(off + (size_t)batch * Lc * sizeof(int32_t), 256);
  w.total = off;
  return w;
}

bool make_tmap_bf16(const Ctx& c, CUtensorMap* map, const void* base, uint64_t width,
                    uint64_t rows, uint32_t box_rows) {
  using Fn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                          const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                          CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                          CUtensorMapFloatOOBfill);
  if (!c.encode_tiled) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)width * 2};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = ((Fn)c.encode_tiled)(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                          const_cast<void*>(base), dims, strides, box, estr,
                                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_rows64(const Ctx& c, CUtensorMap* map, const void* base, uint64_t rows,
                      uint32_t box_rows) {
  return make_tmap_bf16(c, map, base, kIdxPad, rows, box_rows);
}

}  // namespace imem

using imem::Ctx;

namespace {

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

inline imem_status check_ptr(const void* p) {
  if (!p) return IMEM_ERR_INVALID_ARG;
  if (!aligned16(p)) return IMEM_ERR_ALIGN;
  return IMEM_OK;
}

#define IMEM_CHECK(expr)                 \
  do {                                   \
    imem_status s__ = (expr);            \
    if (s__ != IMEM_OK) return s__;      \
  } while (0)

inline imem_status cuda_status(cudaError_t e) {
  return e == cudaSuccess ? IMEM_OK : IMEM_ERR_CUDA;
}

imem_status check_device(const Ctx& c) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return IMEM_ERR_CUDA;
  return dev == c.device ? IMEM_OK : IMEM_ERR_INVALID_ARG;
}

// The second stream and the fork/join events of online eviction, created on
// first use (no device memory is allocated).
imem_status online_streams(Ctx& c) {
  if (c.side && c.ev_fork && c.ev_join) return IMEM_OK;
  if (!c.side && cudaStreamCreateWithFlags(&c.side, cudaStreamNonBlocking) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (!c.ev_fork && cudaEventCreateWithFlags(&c.ev_fork, cudaEventDisableTiming) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (!c.ev_join && cudaEventCreateWithFlags(&c.ev_join, cudaEventDisableTiming) != cudaSuccess)
    return IMEM_ERR_CUDA;
  return IMEM_OK;
}

// The pre-eviction's second stream and its events, created on first use.
imem_status prefill_streams(Ctx& c) {
  if (!c.side && cudaStreamCreateWithFlags(&c.side, cudaStreamNonBlocking) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (!c.ev_pe_fork &&
      cudaEventCreateWithFlags(&c.ev_pe_fork, cudaEventDisableTiming) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (!c.ev_pe_compact &&
      cudaEventCreateWithFlags(&c.ev_pe_compact, cudaEventDisableTiming) != cudaSuccess)
    return IMEM_ERR_CUDA;
  if (!c.ev_pe_done &&
      cudaEventCreateWithFlags(&c.ev_pe_done, cudaEventDisableTiming) != cudaSuccess)
    return IMEM_ERR_CUDA;
  return IMEM_OK;
}

// Makes `st` wait for pre-eviction work still running on the second stream
// (see imem_prefill_evict_chunk); every call that enqueues work does this
// first, so that work is complete before anything else of the library reads
// or writes the memory state, the retained or the evicted positions.
imem_status wait_pending(Ctx& c, cudaStream_t st) {
  if (!c.pe_pending) return IMEM_OK;
  if (cudaStreamWaitEvent(st, c.ev_pe_done, 0) != cudaSuccess) return IMEM_ERR_CUDA;
  c.pe_pending = false;
  c.pe_compact_pending = false;
  return IMEM_OK;
}
// The same for the last range's selection and compaction only.
imem_status wait_compact(Ctx& c, cudaStream_t st) {
  if (!c.pe_compact_pending) return IMEM_OK;
  if (cudaStreamWaitEvent(st, c.ev_pe_compact, 0) != cudaSuccess) return IMEM_ERR_CUDA;
  c.pe_compact_pending = false;
  return IMEM_OK;
}

}  // namespace

extern "C" {

const char* imem_status_string(imem_status s) {
  switch (s) {
    case IMEM_OK: return "IMEM_OK";
    case IMEM_ERR_INVALID_ARG: return "IMEM_ERR_INVALID_ARG";
    case IMEM_ERR_SHAPE: return "IMEM_ERR_SHAPE";
    case IMEM_ERR_ALIGN: return "IMEM_ERR_ALIGN";
    case IMEM_ERR_UNSUPPORTED: return "IMEM_ERR_UNSUPPORTED";
    case IMEM_ERR_CUDA: return "IMEM_ERR_CUDA";
    case IMEM_ERR_TIMEOUT: return "IMEM_ERR_TIMEOUT";
    case IMEM_ERR_RANGE: return "IMEM_ERR_RANGE";
  }
  return "IMEM_ERR_UNKNOWN";
}

imem_status imem_init(const imem_config* cfg, const imem_weights* w, imem_ctx** out) {
  if (!out) return IMEM_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !w) return IMEM_ERR_INVALID_ARG;
  const imem_config& k = *cfg;
  if (k.dtype != IMEM_FP32 && k.dtype != IMEM_BF16) return IMEM_ERR_INVALID_ARG;
  if (k.hidden <= 0 || k.n_q_heads <= 0 || k.n_kv_heads <= 0 || k.head_dim <= 0 ||
      k.idx_heads <= 0 || k.idx_dim <= 0 || k.mem_r <= 0)
    return IMEM_ERR_INVALID_ARG;
  if (!(k.lambda > 0.f && k.lambda <= 1.f) || !(k.eps >= 0.f) || isinf(k.eps))
    return IMEM_ERR_INVALID_ARG;
  if (k.idx_heads != k.n_q_heads) return IMEM_ERR_UNSUPPORTED;
  if (k.n_q_heads % k.n_kv_heads) return IMEM_ERR_SHAPE;
  const int group = k.n_q_heads / k.n_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return IMEM_ERR_UNSUPPORTED;
  if (k.head_dim != 64 && k.head_dim != 128) return IMEM_ERR_UNSUPPORTED;
  if (k.idx_dim != 32 && k.idx_dim != 64) return IMEM_ERR_UNSUPPORTED;
  if (k.hidden % 64) return IMEM_ERR_UNSUPPORTED;
  if (k.mem_r % 16 || k.mem_r > 128) return IMEM_ERR_UNSUPPORTED;
  if (k.idx_dim + k.n_q_heads > 128) return IMEM_ERR_UNSUPPORTED;
  if (k.readout != IMEM_READOUT_GATED && k.readout != IMEM_READOUT_MOMENT)
    return IMEM_ERR_INVALID_ARG;
  const bool moment = k.readout == IMEM_READOUT_MOMENT;
  if (moment && k.mem_r != k.head_dim) return IMEM_ERR_UNSUPPORTED;
  if (moment && k.lambda != 1.f) return IMEM_ERR_UNSUPPORTED;
  IMEM_CHECK(check_ptr(w->W_idx_q));
  IMEM_CHECK(check_ptr(w->W_idx_k));
  IMEM_CHECK(check_ptr(w->w_idx_g));
  if (!moment) {
    IMEM_CHECK(check_ptr(w->W_phi));
    IMEM_CHECK(check_ptr(w->w_gate));
  }

  imem_ctx* h = (imem_ctx*)calloc(1, sizeof(imem_ctx));
  if (!h) return IMEM_ERR_CUDA;
  Ctx& c = h->c;
  c.cfg = k;
  c.group = group;
  if (cudaGetDevice(&c.device) != cudaSuccess) { free(h); return IMEM_ERR_CUDA; }
  if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, c.device) != cudaSuccess) {
    free(h);
    return IMEM_ERR_CUDA;
  }
  {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &c.encode_tiled, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !c.encode_tiled) {
      free(h);
      return IMEM_ERR_CUDA;
    }
  }
  const size_t n_phi = (size_t)k.mem_r * k.head_dim;
  const size_t n_g = (size_t)k.n_q_heads * k.head_dim;
  cudaError_t e = imem::pack_indexer_weights(c, w->W_idx_q, w->W_idx_k, w->w_idx_g);
  if (e == cudaSuccess) e = cudaMalloc((void**)&c.W_phi, n_phi * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc((void**)&c.w_gate, n_g * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc((void**)&c.err, sizeof(int));
  if (moment) {
    // moment statistics: the identity map (S^T and s_k come out of the same
    // kernel as M and b) and no gate
    std::vector<float> eye(n_phi, 0.f);
    for (int i = 0; i < k.mem_r; ++i) eye[(size_t)i * k.head_dim + i] = 1.f;
    if (e == cudaSuccess)
      e = cudaMemcpy(c.W_phi, eye.data(), n_phi * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(c.w_gate, 0, n_g * sizeof(float));
  } else {
    if (e == cudaSuccess) e = cudaMemcpy(c.W_phi, w->W_phi, n_phi * sizeof(float), cudaMemcpyDeviceToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(c.w_gate, w->w_gate, n_g * sizeof(float), cudaMemcpyDeviceToDevice);
  }
  if (e == cudaSuccess) e = cudaMemset(c.err, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    imem_destroy(h);
    return IMEM_ERR_CUDA;
  }
  *out = h;
  return IMEM_OK;
}

void imem_destroy(imem_ctx* h) {
  if (!h) return;
  Ctx& c = h->c;
  cudaDeviceSynchronize();
  cudaFree(c.WcT);
  cudaFree(c.WqT);
  cudaFree(c.W_phi);
  cudaFree(c.w_gate);
  cudaFree(c.err);
  if (c.ev_fork) cudaEventDestroy(c.ev_fork);
  if (c.ev_join) cudaEventDestroy(c.ev_join);
  if (c.ev_pe_fork) cudaEventDestroy(c.ev_pe_fork);
  if (c.ev_pe_compact) cudaEventDestroy(c.ev_pe_compact);
  if (c.ev_pe_done) cudaEventDestroy(c.ev_pe_done);
  if (c.side) cudaStreamDestroy(c.side);
  free(h);
}

imem_status imem_workspace_size(imem_ctx* h, int batch, int L, int B, size_t* bytes) {
  if (!h || !bytes) return IMEM_ERR_INVALID_ARG;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (B < 1 || B > L) return IMEM_ERR_SHAPE;
  *bytes = imem::workspace_layout(h->c, batch, L).total;
  return IMEM_OK;
}

imem_status imem_score_and_evict(imem_ctx* h, int batch, int L, int B, const void* X,
                                 const void* Q, const void* K, const void* V, float* running_max,
                                 int q_begin, int q_end, int finalize, int32_t* idx_retained,
                                 int32_t* idx_evicted, void* K_ret, void* V_ret, int cap,
                                 void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (finalize != 0 && finalize != 1) return IMEM_ERR_INVALID_ARG;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (q_begin < 0 || q_end <= q_begin || q_end > L) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(X));
  IMEM_CHECK(check_ptr(Q));
  IMEM_CHECK(check_ptr(running_max));
  IMEM_CHECK(check_ptr(workspace));
  if (finalize) {
    if (q_end != L) return IMEM_ERR_SHAPE;
    if (B < 1 || B > L || cap < B) return IMEM_ERR_SHAPE;
    IMEM_CHECK(check_ptr(K));
    IMEM_CHECK(check_ptr(V));
    IMEM_CHECK(check_ptr(idx_retained));
    if (B < L) IMEM_CHECK(check_ptr(idx_evicted));
    IMEM_CHECK(check_ptr(K_ret));
    IMEM_CHECK(check_ptr(V_ret));
  }
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  cudaStream_t st = (cudaStream_t)stream;
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  char* wsb = (char*)workspace;
  IMEM_CHECK(cuda_status(imem::clear_decode_tags(c, batch, workspace, st)));
  __nv_bfloat16* qt = (__nv_bfloat16*)(wsb + ws.qt_off);
  __nv_bfloat16* kh = (__nv_bfloat16*)(wsb + ws.kh_off);
  IMEM_CHECK(cuda_status(imem::launch_prologue(c, batch, L, X, Q, q_begin, q_end, qt, kh,
                                               running_max, st)));
  IMEM_CHECK(cuda_status(imem::launch_scoring(c, batch, L, qt, kh, running_max, q_begin, q_end, st)));
  if (finalize)
    IMEM_CHECK(cuda_status(imem::launch_select_compact(c, batch, L, B, running_max, K, V,
                                                       idx_retained, idx_evicted, K_ret, V_ret,
                                                       cap, wsb + ws.sel_off, st)));
  return IMEM_OK;
}

imem_status imem_indexer_features(imem_ctx* h, int batch, int L, const void* X, const void* Q,
                                  float* running_max, int q_begin, int q_end, void* workspace,
                                  void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (q_begin < 0 || q_end <= q_begin || q_end > L) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(X));
  IMEM_CHECK(check_ptr(Q));
  IMEM_CHECK(check_ptr(running_max));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  char* wsb = (char*)workspace;
  return cuda_status(imem::launch_prologue(c, batch, L, X, Q, q_begin, q_end,
                                           (__nv_bfloat16*)(wsb + ws.qt_off),
                                           (__nv_bfloat16*)(wsb + ws.kh_off), running_max,
                                           (cudaStream_t)stream));
}

imem_status imem_indexer_score(imem_ctx* h, int batch, int L, float* running_max, int q_begin,
                               int q_end, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (q_begin < 0 || q_end <= q_begin || q_end > L) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(running_max));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  char* wsb = (char*)workspace;
  return cuda_status(imem::launch_scoring(c, batch, L, (const __nv_bfloat16*)(wsb + ws.qt_off),
                                          (const __nv_bfloat16*)(wsb + ws.kh_off), running_max,
                                          q_begin, q_end, (cudaStream_t)stream));
}

imem_status imem_select_compact(imem_ctx* h, int batch, int L, int B, const float* running_max,
                                const void* K, const void* V, int32_t* idx_retained,
                                int32_t* idx_evicted, void* K_ret, void* V_ret, int cap,
                                void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (B < 1 || B > L || cap < B) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(running_max));
  IMEM_CHECK(check_ptr(K));
  IMEM_CHECK(check_ptr(V));
  IMEM_CHECK(check_ptr(idx_retained));
  if (B < L) IMEM_CHECK(check_ptr(idx_evicted));
  IMEM_CHECK(check_ptr(K_ret));
  IMEM_CHECK(check_ptr(V_ret));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  cudaStream_t st = (cudaStream_t)stream;
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  IMEM_CHECK(cuda_status(imem::clear_decode_tags(c, batch, workspace, st)));
  return cuda_status(imem::launch_select_compact(c, batch, L, B, running_max, K, V, idx_retained,
                                                 idx_evicted, K_ret, V_ret, cap,
                                                 (char*)workspace + ws.sel_off, st));
}

imem_status imem_update_memory(imem_ctx* h, int batch, int L, const void* K, const void* V,
                               const int32_t* idx_evicted, int n_evicted, int chunk, float* M,
                               float* bstab, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.cfg.readout != IMEM_READOUT_GATED) return IMEM_ERR_UNSUPPORTED;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (n_evicted < 0 || n_evicted > L) return IMEM_ERR_SHAPE;
  if (chunk < 64 || chunk % 64) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(K));
  IMEM_CHECK(check_ptr(V));
  if (n_evicted > 0) IMEM_CHECK(check_ptr(idx_evicted));
  IMEM_CHECK(check_ptr(M));
  IMEM_CHECK(check_ptr(bstab));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  float* part = (float*)((char*)workspace + ws.mem_part_off);
  int* tags = (int*)((char*)workspace + imem::workspace_layout(c, batch, 1).dec_tag_off);
  return cuda_status(imem::launch_memory_update(c, batch, L, K, V, idx_evicted, n_evicted, chunk,
                                                M, bstab, part, nullptr, nullptr, nullptr,
                                                (cudaStream_t)stream, tags, batch));
}

imem_status imem_update_moments(imem_ctx* h, int batch, int L, const void* K, const void* V,
                                const int32_t* idx_evicted, int n_evicted, int chunk, float* S_T,
                                float* s_k, float* s_v, float* n_e, void* workspace,
                                void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.cfg.readout != IMEM_READOUT_MOMENT) return IMEM_ERR_UNSUPPORTED;
  if (batch < 1 || L < 1) return IMEM_ERR_SHAPE;
  if (n_evicted < 0 || n_evicted > L) return IMEM_ERR_SHAPE;
  if (chunk < 64 || chunk % 64) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(K));
  IMEM_CHECK(check_ptr(V));
  if (n_evicted > 0) IMEM_CHECK(check_ptr(idx_evicted));
  IMEM_CHECK(check_ptr(S_T));
  IMEM_CHECK(check_ptr(s_k));
  IMEM_CHECK(check_ptr(s_v));
  IMEM_CHECK(check_ptr(n_e));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  float* part = (float*)((char*)workspace + ws.mem_part_off);
  float* svp = (float*)((char*)workspace + ws.sv_part_off);
  int* tags = (int*)((char*)workspace + imem::workspace_layout(c, batch, 1).dec_tag_off);
  return cuda_status(imem::launch_memory_update(c, batch, L, K, V, idx_evicted, n_evicted, chunk,
                                                S_T, s_k, part, svp, s_v, n_e,
                                                (cudaStream_t)stream, tags, batch));
}

namespace {
imem_status decode_common(imem_ctx* h, int batch, const void* q, const void* k_new,
                          const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                          int cap, const float* M, const float* bstab, const float* s_v,
                          const float* n_e, void* out, void* workspace, void* stream) {
  const Ctx& c = h->c;
  const bool moment = c.cfg.readout == IMEM_READOUT_MOMENT;
  if (batch < 1 || cap < 1) return IMEM_ERR_SHAPE;
  if (moment) {
    IMEM_CHECK(check_ptr(s_v));
    IMEM_CHECK(check_ptr(n_e));
  }
  IMEM_CHECK(check_ptr(q));
  IMEM_CHECK(check_ptr(k_new));
  IMEM_CHECK(check_ptr(v_new));
  IMEM_CHECK(check_ptr(K_ret));
  IMEM_CHECK(check_ptr(V_ret));
  IMEM_CHECK(check_ptr(cache_len));
  IMEM_CHECK(check_ptr(M));
  IMEM_CHECK(check_ptr(bstab));
  IMEM_CHECK(check_ptr(out));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  // the decode regions of the workspace do not depend on L
  const imem::Workspace ws = imem::workspace_layout(c, batch, 1);
  char* wsb = (char*)workspace;
  return cuda_status(imem::launch_decode(c, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap,
                                         M, bstab, s_v, n_e, out, (int*)(wsb + ws.dec_cnt_off),
                                         (cudaStream_t)stream));
}
}  // namespace

imem_status imem_decode(imem_ctx* h, int batch, const void* q, const void* k_new,
                        const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len, int cap,
                        const float* M, const float* bstab, void* out, void* workspace,
                        void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  if (h->c.cfg.readout != IMEM_READOUT_GATED) return IMEM_ERR_UNSUPPORTED;
  return decode_common(h, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, nullptr,
                       nullptr, out, workspace, stream);
}

imem_status imem_decode_moment(imem_ctx* h, int batch, const void* q, const void* k_new,
                               const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                               int cap, const float* S_T, const float* s_k, const float* s_v,
                               const float* n_e, void* out, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  if (h->c.cfg.readout != IMEM_READOUT_MOMENT) return IMEM_ERR_UNSUPPORTED;
  return decode_common(h, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, S_T, s_k, s_v,
                       n_e, out, workspace, stream);
}

imem_status imem_decode_invalidate(imem_ctx* h, int batch, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  if (batch < 1) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_device(h->c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  return cuda_status(imem::clear_decode_tags(h->c, batch, workspace, (cudaStream_t)stream));
}

imem_status imem_workspace_size_evict(imem_ctx* h, int batch, int L, int B, int chunk_max,
                                     size_t* bytes) {
  if (!h || !bytes) return IMEM_ERR_INVALID_ARG;
  if (batch < 1 || L < 1 || B < 1 || chunk_max < 1) return IMEM_ERR_SHAPE;
  if ((size_t)B + chunk_max > (size_t)INT32_MAX / imem::kIdxPad) return IMEM_ERR_SHAPE;
  *bytes = imem::evict_workspace_layout(h->c, batch, B, chunk_max).total;
  return IMEM_OK;
}

imem_status imem_prefill_evict_chunk(imem_ctx* h, int batch, int L, int B, int chunk_max,
                                     const void* X, const void* Q, const void* K, const void* V,
                                     int q_begin, int q_end, int32_t* retained, int32_t* evicted,
                                     float* cand_importance, float* M, float* bstab,
                                     int mem_chunk, int finalize, void* K_ret, void* V_ret,
                                     int cap, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.cfg.readout != IMEM_READOUT_GATED) return IMEM_ERR_UNSUPPORTED;
  if (finalize != 0 && finalize != 1) return IMEM_ERR_INVALID_ARG;
  if (batch < 1 || L < 1 || B < 1 || chunk_max < 1) return IMEM_ERR_SHAPE;
  if (q_begin < 0 || q_end <= q_begin || q_end > L || q_end - q_begin > chunk_max)
    return IMEM_ERR_SHAPE;
  if (mem_chunk < 64 || mem_chunk % 64) return IMEM_ERR_SHAPE;
  const int n_R = B < q_begin ? B : q_begin;          // retained before this range
  const int C = q_end - q_begin, n = n_R + C, n_ev = n > B ? n - B : 0;
  IMEM_CHECK(check_ptr(X));
  IMEM_CHECK(check_ptr(Q));
  IMEM_CHECK(check_ptr(retained));
  IMEM_CHECK(check_ptr(workspace));
  if (cand_importance) IMEM_CHECK(check_ptr(cand_importance));
  if (n_ev > 0) {
    IMEM_CHECK(check_ptr(K));
    IMEM_CHECK(check_ptr(V));
    IMEM_CHECK(check_ptr(evicted));
    IMEM_CHECK(check_ptr(M));
    IMEM_CHECK(check_ptr(bstab));
  }
  if (finalize) {
    if (q_end != L) return IMEM_ERR_SHAPE;
    if (cap < (B < L ? B : L)) return IMEM_ERR_SHAPE;
    IMEM_CHECK(check_ptr(K));
    IMEM_CHECK(check_ptr(V));
    IMEM_CHECK(check_ptr(K_ret));
    IMEM_CHECK(check_ptr(V_ret));
  }
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(prefill_streams(h->c));
  Ctx& cm = h->c;
  cudaStream_t st = (cudaStream_t)stream;
  if (q_begin == 0) {
    // a new prefill: nothing of an earlier one may still run, buffer 0 first
    IMEM_CHECK(wait_pending(cm, st));
    cm.pe_parity = 0;
  }
  const int Lc = B + chunk_max;
  const imem::EvictWorkspace ws = imem::evict_workspace_layout(c, batch, B, chunk_max);
  char* wsb = (char*)workspace;
  IMEM_CHECK(cuda_status(imem::clear_decode_tags(c, batch, workspace, st)));
  // two candidate buffers: this range's candidates in buffer p, the rows it
  // retains compacted into buffer 1 - p (no row is overwritten before it is
  // read, and the next range's prologue writes its rows there while this
  // range's selection may still read buffer p)
  const int p = cm.pe_parity;
  __nv_bfloat16* khb[2] = {(__nv_bfloat16*)(wsb + ws.base.kh_off),
                           (__nv_bfloat16*)(wsb + ws.kh1_off)};
  imem::EvictBuffers eb;
  __nv_bfloat16* qt = (__nv_bfloat16*)(wsb + ws.base.qt_off);
  eb.kh_c = khb[p];
  eb.I_c = (float*)(wsb + ws.I_off[p]);
  eb.pos_c = (int32_t*)(wsb + ws.pos_off[p]);
  eb.kh_n = khb[1 - p];
  eb.I_n = (float*)(wsb + ws.I_off[1 - p]);
  eb.pos_n = (int32_t*)(wsb + ws.pos_off[1 - p]);
  eb.idx_r = (int32_t*)(wsb + ws.idx_r_off);
  eb.idx_e = (int32_t*)(wsb + ws.idx_e_off);
  // the range's indexer features go to candidate rows [n_R, n)
  IMEM_CHECK(cuda_status(imem::launch_prologue(c, batch, L, X, Q, q_begin, q_end, qt, eb.kh_c,
                                               eb.I_c, st, Lc, n_R - q_begin)));
  // rows [0, n_R) of buffer p come from the previous range's compaction
  IMEM_CHECK(wait_compact(cm, st));
  IMEM_CHECK(cuda_status(imem::launch_scoring(c, batch, Lc, qt, eb.kh_c, eb.I_c, n_R, n, st)));
  if (cand_importance)
    IMEM_CHECK(cuda_status(cudaMemcpyAsync(cand_importance, eb.I_c, (size_t)batch * Lc * sizeof(float),
                                           cudaMemcpyDeviceToDevice, st)));
  if (n_ev > 0) {
    // selection, compaction and the memory update on the second stream: they
    // run beside the next range's prologue (and the memory update beside its
    // scoring); the next call waits for the compaction before its scoring,
    // every other call for all of it first
    float* part = (float*)(wsb + ws.base.mem_part_off);
    IMEM_CHECK(cuda_status(cudaEventRecord(cm.ev_pe_fork, st)));
    IMEM_CHECK(cuda_status(cudaStreamWaitEvent(cm.side, cm.ev_pe_fork, 0)));
    cudaError_t se = imem::launch_evict_chunk(c, batch, B, Lc, n_R, q_begin, C, eb, retained,
                                              evicted, cm.side);
    // both events are recorded even after a failed launch, so that no later
    // wait refers to an event of an earlier range
    const cudaError_t e1 = cudaEventRecord(cm.ev_pe_compact, cm.side);
    if (se == cudaSuccess)
      se = imem::launch_memory_update(c, batch, L, K, V, evicted, n_ev, mem_chunk, M, bstab, part,
                                      nullptr, nullptr, nullptr, cm.side);
    const cudaError_t e2 = cudaEventRecord(cm.ev_pe_done, cm.side);
    cm.pe_pending = true;
    cm.pe_compact_pending = true;
    cm.pe_parity = 1 - p;
    IMEM_CHECK(cuda_status(se));
    IMEM_CHECK(cuda_status(e1));
    IMEM_CHECK(cuda_status(e2));
  } else {
    IMEM_CHECK(wait_pending(cm, st));
    IMEM_CHECK(cuda_status(imem::launch_append_positions(batch, B, n_R, q_begin, C, retained,
                                                         eb.pos_c, st)));
  }
  if (finalize) {
    IMEM_CHECK(wait_pending(cm, st));
    IMEM_CHECK(cuda_status(imem::launch_gather(c, batch, L, B < L ? B : L, retained, B, K, V,
                                               K_ret, V_ret, cap, st)));
  }
  return IMEM_OK;
}

imem_status imem_online_init(imem_ctx* h, int batch, int L, int B, const float* running_max,
                             const int32_t* idx_retained, const void* workspace, void* khat_ret,
                             float* I_ret, int32_t* pos_ret, int32_t* next_pos, int cap,
                             void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.cfg.readout != IMEM_READOUT_GATED) return IMEM_ERR_UNSUPPORTED;
  if (batch < 1 || L < 1 || B < 1 || B > L || cap < B + 1) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(running_max));
  IMEM_CHECK(check_ptr(idx_retained));
  IMEM_CHECK(check_ptr(workspace));
  IMEM_CHECK(check_ptr(khat_ret));
  IMEM_CHECK(check_ptr(I_ret));
  IMEM_CHECK(check_ptr(pos_ret));
  IMEM_CHECK(check_ptr(next_pos));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  const imem::Workspace ws = imem::workspace_layout(c, batch, L);
  const __nv_bfloat16* kh = (const __nv_bfloat16*)((const char*)workspace + ws.kh_off);
  return cuda_status(imem::launch_online_init(c, batch, L, B, cap, running_max, idx_retained, kh,
                                              (__nv_bfloat16*)khat_ret, I_ret, pos_ret, next_pos,
                                              (cudaStream_t)stream));
}

imem_status imem_decode_online(imem_ctx* h, int batch, int B, const void* x_new, const void* q,
                               const void* k_new, const void* v_new, void* K_ret, void* V_ret,
                               void* khat_ret, float* I_ret, int32_t* pos_ret, int32_t* next_pos,
                               int32_t* cache_len, int cap, float* M, float* bstab, void* out,
                               int32_t* evicted, void* workspace, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.cfg.readout != IMEM_READOUT_GATED) return IMEM_ERR_UNSUPPORTED;
  if (c.cfg.n_kv_heads > imem::kOnlineMaxCluster) return IMEM_ERR_UNSUPPORTED;
  if (batch < 1 || B < 1 || cap < B + 1) return IMEM_ERR_SHAPE;
  IMEM_CHECK(check_ptr(x_new));
  IMEM_CHECK(check_ptr(khat_ret));
  IMEM_CHECK(check_ptr(I_ret));
  IMEM_CHECK(check_ptr(pos_ret));
  IMEM_CHECK(check_ptr(next_pos));
  IMEM_CHECK(check_ptr(evicted));
  IMEM_CHECK(check_ptr(workspace));
  // the attention step's arguments too: nothing is enqueued unless all are valid
  IMEM_CHECK(check_ptr(q));
  IMEM_CHECK(check_ptr(k_new));
  IMEM_CHECK(check_ptr(v_new));
  IMEM_CHECK(check_ptr(K_ret));
  IMEM_CHECK(check_ptr(V_ret));
  IMEM_CHECK(check_ptr(cache_len));
  IMEM_CHECK(check_ptr(M));
  IMEM_CHECK(check_ptr(bstab));
  IMEM_CHECK(check_ptr(out));
  IMEM_CHECK(check_device(c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  IMEM_CHECK(online_streams(h->c));
  cudaStream_t st = (cudaStream_t)stream;
  const imem::Workspace ws = imem::workspace_layout(c, batch, 1);
  char* wsb = (char*)workspace;
  float* qpart = (float*)(wsb + ws.on_qpart_off);
  float* kpart = (float*)(wsb + ws.on_kpart_off);
  // the new token's indexer features need neither the cache nor the memory:
  // they run on the context's second stream beside the attention step
  IMEM_CHECK(cuda_status(cudaEventRecord(c.ev_fork, st)));
  IMEM_CHECK(cuda_status(cudaStreamWaitEvent(c.side, c.ev_fork, 0)));
  IMEM_CHECK(cuda_status(imem::launch_online_features(c, batch, x_new, q, qpart, kpart, c.side)));
  IMEM_CHECK(cuda_status(cudaEventRecord(c.ev_join, c.side)));
  // the attention step with the memory before this step's eviction (it
  // validates the remaining arguments and appends the new token at slot B)
  const imem_status ds = decode_common(h, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M,
                                       bstab, nullptr, nullptr, out, workspace, stream);
  // join first, so that the second stream's work is always waited for
  IMEM_CHECK(cuda_status(cudaStreamWaitEvent(st, c.ev_join, 0)));
  IMEM_CHECK(ds);
  // the importances, the token that leaves, the memory update and the slot
  // swap: one kernel after both branches
  return cuda_status(imem::launch_online_score_evict(c, batch, B, cap, qpart, kpart, khat_ret,
                                                     I_ret, pos_ret, next_pos, K_ret, V_ret,
                                                     cache_len, M, bstab, evicted,
                                                     (int*)(wsb + ws.dec_tag_off), st));
}

imem_status imem_selftest_wait(imem_ctx* h, long long limit_cycles, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  if (limit_cycles < 1 || limit_cycles > 2000000000LL) return IMEM_ERR_INVALID_ARG;
  IMEM_CHECK(check_device(h->c));
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  return cuda_status(imem::launch_wait_selftest(h->c, limit_cycles, (cudaStream_t)stream));
}

imem_status imem_join(imem_ctx* h, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  IMEM_CHECK(check_device(h->c));
  return wait_pending(h->c, (cudaStream_t)stream);
}

imem_status imem_sync(imem_ctx* h, void* stream) {
  if (!h) return IMEM_ERR_INVALID_ARG;
  IMEM_CHECK(wait_pending(h->c, (cudaStream_t)stream));
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return IMEM_ERR_CUDA;
  int code = 0;
  e = cudaMemcpy(&code, h->c.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return IMEM_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    cudaMemcpy(h->c.err, &zero, sizeof(int), cudaMemcpyHostToDevice);
  }
  if (code == imem::DEV_TIMEOUT) return IMEM_ERR_TIMEOUT;
  if (code == imem::DEV_CACHE_FULL) return IMEM_ERR_SHAPE;
  if (code == imem::DEV_RANGE) return IMEM_ERR_RANGE;
  return IMEM_OK;
}

}  // extern "C"
