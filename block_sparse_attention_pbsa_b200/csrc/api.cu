// extern "C" entry points of libpbsa: argument validation and dispatch to the kernels.
// Every check here runs on the host before anything is launched.
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

pbsa_status make_geo(const pbsa_geom* in, Geo* g) {
  if (in == nullptr) return PBSA_ERR_INVALID_ARG;
  if (in->heads <= 0 || in->head_dim <= 0 || in->frame_h <= 0 || in->frame_w <= 0 ||
      in->tile_h <= 0 || in->tile_w <= 0)
    return PBSA_ERR_INVALID_ARG;
  if (in->tile_h * in->tile_w != BT) return PBSA_ERR_INVALID_ARG;
  if (in->frame_h % in->tile_h != 0 || in->frame_w % in->tile_w != 0) return PBSA_ERR_INVALID_ARG;
  if (!(in->scale > 0.f) || !isfinite(in->scale)) return PBSA_ERR_INVALID_ARG;
  if (in->dtype != PBSA_F32 && in->dtype != PBSA_BF16) return PBSA_ERR_INVALID_ARG;
  if (in->head_dim != 32 && in->head_dim != 64 && in->head_dim != 128) return PBSA_ERR_UNSUPPORTED;
  if (in->dtype == PBSA_BF16 && in->head_dim == 32) return PBSA_ERR_UNSUPPORTED;
  if ((int64_t)in->frame_h * in->frame_w > (1 << 24) || in->heads > 4096) return PBSA_ERR_UNSUPPORTED;
  g->H = in->heads;
  g->d = in->head_dim;
  g->fh = in->frame_h;
  g->fw = in->frame_w;
  g->th = in->tile_h;
  g->tw = in->tile_w;
  g->tpr = in->frame_w / in->tile_w;
  g->bpf = (in->frame_h / in->tile_h) * g->tpr;
  g->tpf = in->frame_h * in->frame_w;
  g->scale = in->scale;
  g->dtype = in->dtype;
  g->esize = in->dtype == PBSA_BF16 ? 2 : 4;
  return PBSA_OK;
}

pbsa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return PBSA_OK;
  if (e == cudaErrorNotSupported) return PBSA_ERR_UNSUPPORTED;
  return PBSA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Pool rows (H * slots * 64) must be addressable with 32-bit TMA coordinates.
bool pool_ok(const Geo& g, int pool_slots) {
  return pool_slots > 0 && (int64_t)g.H * pool_slots * BT < ((int64_t)1 << 31);
}

// The bounded-wait path every kernel relies on, on its own: one thread waits on an mbarrier
// that nothing ever arrives on, gives up after limit_ns, records PBSA_ERR_TIMEOUT and returns.
__global__ void selftest_wait_kernel(void* ws, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait(&bar, 0, limit_ns)) record_error(ws, PBSA_ERR_TIMEOUT, 0, K_SELFTEST);
  }
}

}  // namespace

cudaError_t set_smem_once(const void* kernel, int bytes) {
  struct Entry { const void* k; int dev; int bytes; };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.k == kernel && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({kernel, dev, bytes});
  return e;
}

}  // namespace pbsa

using namespace pbsa;

extern "C" {

size_t pbsa_workspace_bytes(const pbsa_geom* gin, int max_q_blocks, int max_pool_entries) {
  Geo g;
  if (make_geo(gin, &g) != PBSA_OK || max_q_blocks < 0 || max_pool_entries < 0) return 0;
  const size_t mu = memory_update_ws_bytes(g, max_q_blocks > 0 ? max_q_blocks : 1,
                                           max_pool_entries > 0 ? max_pool_entries : 1);
  return mu > (size_t)WS_HEADER_BYTES ? mu : (size_t)WS_HEADER_BYTES;
}

pbsa_status pbsa_blockify(const pbsa_geom* gin, const void* x, int n_frames, float* reps,
                          int rep_slots, const int* dst_slot, void* pool, int pool_slots, void* ws,
                          void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (x == nullptr || reps == nullptr || n_frames <= 0 || rep_slots <= 0) return PBSA_ERR_INVALID_ARG;
  if (dst_slot == nullptr && rep_slots < n_frames * g.bpf) return PBSA_ERR_INVALID_ARG;
  if (pool != nullptr && (!pool_ok(g, pool_slots) || !aligned16(pool))) return PBSA_ERR_INVALID_ARG;
  if (pool != nullptr && dst_slot == nullptr && pool_slots < n_frames * g.bpf) return PBSA_ERR_INVALID_ARG;
  if (!aligned16(x) || (int64_t)n_frames * g.bpf * g.H > ((int64_t)1 << 30)) return PBSA_ERR_INVALID_ARG;
  return from_cuda(launch_blockify(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws,
                                   static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_blockify_kv(const pbsa_geom* gin, const void* k, const void* v, int n_frames, float* k_reps,
                             float* v_reps, int rep_slots, const int* dst_slot, void* k_pool, void* v_pool,
                             int pool_slots, int flags, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (k == nullptr || v == nullptr || k_reps == nullptr || k_pool == nullptr || v_pool == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (n_frames <= 0 || rep_slots <= 0 || !pool_ok(g, pool_slots)) return PBSA_ERR_INVALID_ARG;
  if (dst_slot == nullptr && (rep_slots < n_frames * g.bpf || pool_slots < n_frames * g.bpf))
    return PBSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_pool) || !aligned16(v_pool)) return PBSA_ERR_INVALID_ARG;
  if ((int64_t)n_frames * g.bpf * g.H > ((int64_t)1 << 30)) return PBSA_ERR_INVALID_ARG;
  if ((flags & ~PBSA_OVERLAP_PREVIOUS) != 0) return PBSA_ERR_INVALID_ARG;
  return from_cuda(launch_blockify_pair(g, k, v, n_frames, k_reps, v_reps, rep_slots, dst_slot, k_pool,
                                        v_pool, pool_slots, (flags & PBSA_OVERLAP_PREVIOUS) != 0, ws,
                                        static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_score_select(const pbsa_geom* gin, const float* q_reps, int nq, const float* k_reps,
                              int pool_slots, const int* cand_slot, const int* cand_gid, int ncand,
                              int k, const int* prefix_slot, const int* prefix_cnt, int prefix_ld,
                              int* out_slot, int* out_cnt, int out_ld, float* out_score, void* ws,
                              void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q_reps == nullptr || k_reps == nullptr || out_slot == nullptr || out_cnt == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (nq <= 0 || ncand < 0 || k < 0 || pool_slots <= 0 || prefix_ld < 0) return PBSA_ERR_INVALID_ARG;
  if (ncand > 0 && (cand_slot == nullptr || cand_gid == nullptr)) return PBSA_ERR_INVALID_ARG;
  if ((prefix_cnt == nullptr) != (prefix_slot == nullptr)) return PBSA_ERR_INVALID_ARG;
  if (prefix_slot == nullptr) prefix_ld = 0;
  if (out_ld < prefix_ld + k) return PBSA_ERR_INVALID_ARG;
  if (ncand > 1024) return PBSA_ERR_UNSUPPORTED;
  if (!aligned16(q_reps) || !aligned16(k_reps)) return PBSA_ERR_INVALID_ARG;
  return from_cuda(launch_score_select(g, q_reps, nq, k_reps, pool_slots, cand_slot, cand_gid, ncand,
                                       k, prefix_slot, prefix_cnt, prefix_ld, out_slot, out_cnt,
                                       out_ld, out_score, ws, static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_blockify_select_ex(const pbsa_geom* gin, const void* q, int q_frames, float* q_reps,
                                    const float* k_reps, int pool_slots, const int* cand_slot,
                                    const int* cand_gid, int ncand, int k, int top_frames,
                                    int n_recent_frames, const int* prefix_slot, const int* prefix_cnt,
                                    int prefix_ld, const int* suffix_slot, int suffix_n, int* out_slot,
                                    int* out_cnt, int out_ld, float* out_score, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q == nullptr || q_reps == nullptr || k_reps == nullptr || out_slot == nullptr ||
      out_cnt == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (q_frames <= 0 || ncand < 0 || k < 0 || pool_slots <= 0 || prefix_ld < 0 || suffix_n < 0)
    return PBSA_ERR_INVALID_ARG;
  if ((int64_t)q_frames * g.bpf > 65535 * 64) return PBSA_ERR_INVALID_ARG;
  if (ncand > 0 && (cand_slot == nullptr || cand_gid == nullptr)) return PBSA_ERR_INVALID_ARG;
  if ((prefix_cnt == nullptr) != (prefix_slot == nullptr)) return PBSA_ERR_INVALID_ARG;
  if (suffix_n > 0 && suffix_slot == nullptr) return PBSA_ERR_INVALID_ARG;
  if (top_frames >= 0 && (n_recent_frames < 0 || ncand % g.bpf != 0)) return PBSA_ERR_INVALID_ARG;
  if (prefix_slot == nullptr) prefix_ld = 0;
  if (out_ld < prefix_ld + k + suffix_n) return PBSA_ERR_INVALID_ARG;
  if (ncand > 1024 || (top_frames >= 0 && ncand / g.bpf > 256)) return PBSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(q_reps) || !aligned16(k_reps)) return PBSA_ERR_INVALID_ARG;
  return from_cuda(launch_blockify_select(g, q, q_frames, q_reps, k_reps, pool_slots, cand_slot,
                                          cand_gid, ncand, k, prefix_slot, prefix_cnt, prefix_ld,
                                          out_slot, out_cnt, out_ld, out_score,
                                          top_frames < 0 ? -1 : top_frames, n_recent_frames,
                                          suffix_slot, suffix_n, ws, static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_blockify_score_select(const pbsa_geom* gin, const void* q, int q_frames,
                                       float* q_reps, const float* k_reps, int pool_slots,
                                       const int* cand_slot, const int* cand_gid, int ncand, int k,
                                       const int* prefix_slot, const int* prefix_cnt, int prefix_ld,
                                       int* out_slot, int* out_cnt, int out_ld, float* out_score,
                                       void* ws, void* stream) {
  return pbsa_blockify_select_ex(gin, q, q_frames, q_reps, k_reps, pool_slots, cand_slot, cand_gid, ncand,
                                 k, -1, 0, prefix_slot, prefix_cnt, prefix_ld, nullptr, 0, out_slot,
                                 out_cnt, out_ld, out_score, ws, stream);
}

pbsa_status pbsa_blockify_hsa_select(const pbsa_geom* gin, const void* q, int q_frames, float* q_reps,
                                     const float* k_reps, int pool_slots, const int* cand_slot,
                                     const int* cand_gid, int ncand, int top_frames,
                                     int n_recent_frames, int k, const int* prefix_slot,
                                     const int* prefix_cnt, int prefix_ld, int* out_slot,
                                     int* out_cnt, int out_ld, float* out_score, void* ws,
                                     void* stream) {
  if (top_frames < 0 || n_recent_frames < 0) return PBSA_ERR_INVALID_ARG;
  return pbsa_blockify_select_ex(gin, q, q_frames, q_reps, k_reps, pool_slots, cand_slot, cand_gid, ncand,
                                 k, top_frames, n_recent_frames, prefix_slot, prefix_cnt, prefix_ld,
                                 nullptr, 0, out_slot, out_cnt, out_ld, out_score, ws, stream);
}

pbsa_status pbsa_blockify_train_select(const pbsa_geom* gin, const void* q, int q_frames, float* q_reps,
                                       const float* k_reps, int pool_slots, int seq_frames, int chunk_frames,
                                       int sink_frames, int k, int* out_slot, int* out_cnt, int out_ld,
                                       float* out_score, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q == nullptr || q_reps == nullptr || k_reps == nullptr || out_slot == nullptr || out_cnt == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (q_frames <= 0 || seq_frames <= 0 || chunk_frames <= 0 || k < 0 || q_frames % seq_frames != 0)
    return PBSA_ERR_INVALID_ARG;
  if (sink_frames < 0 || sink_frames > chunk_frames || sink_frames > seq_frames) return PBSA_ERR_INVALID_ARG;
  if ((int64_t)q_frames * g.bpf > 65535 * 64) return PBSA_ERR_INVALID_ARG;
  if (pool_slots < q_frames * g.bpf) return PBSA_ERR_INVALID_ARG;
  const int own = (chunk_frames < seq_frames ? chunk_frames : seq_frames) * g.bpf;
  if ((int64_t)out_ld < (int64_t)sink_frames * g.bpf + k + own) return PBSA_ERR_INVALID_ARG;
  const int n_chunks = (seq_frames + chunk_frames - 1) / chunk_frames;
  if (n_chunks > 1 && (int64_t)((n_chunks - 1) * chunk_frames - sink_frames) * g.bpf > 1024)
    return PBSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(q_reps) || !aligned16(k_reps)) return PBSA_ERR_INVALID_ARG;
  return from_cuda(launch_blockify_train_select(g, q, q_frames, q_reps, k_reps, pool_slots, seq_frames,
                                                chunk_frames, sink_frames, k, out_slot, out_cnt, out_ld,
                                                out_score, ws, static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_attend(const pbsa_geom* gin, const void* q, int q_frames, const void* k_pool,
                        const void* v_pool, int pool_slots, const int* kv_slot, const int* kv_cnt,
                        int kv_ld, void* o, float* lse, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q == nullptr || k_pool == nullptr || v_pool == nullptr || kv_slot == nullptr ||
      kv_cnt == nullptr || o == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (q_frames <= 0 || kv_ld <= 0 || !pool_ok(g, pool_slots)) return PBSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o))
    return PBSA_ERR_INVALID_ARG;
  const int64_t nq = (int64_t)q_frames * g.bpf;
  if (nq > 65535 * 2 || (int64_t)q_frames * g.tpf * g.H > ((int64_t)1 << 31)) return PBSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g.dtype == PBSA_BF16) {
    if (g.d != 128 || kv_ld > 512) return PBSA_ERR_UNSUPPORTED;
    return from_cuda(launch_attend_tc(g, q, q_frames, k_pool, v_pool, pool_slots, kv_slot, kv_cnt,
                                      kv_ld, o, lse, ws, st));
  }
  if (kv_ld > 4096) return PBSA_ERR_UNSUPPORTED;
  return from_cuda(launch_attend_f32(g, static_cast<const float*>(q), q_frames,
                                     static_cast<const float*>(k_pool), static_cast<const float*>(v_pool),
                                     pool_slots, kv_slot, kv_cnt, kv_ld, static_cast<float*>(o), lse,
                                     ws, st));
}

pbsa_status pbsa_memory_update(const pbsa_geom* gin, const float* q_reps, int nq, float* k_reps,
                               void* k_pool, void* v_pool, int pool_slots, int* slot_gid,
                               float* slot_ema, int capacity, int n_sink_gid, const int* cand_slot,
                               const int* cand_gid, int ncand, float gamma, int* p_list, int* p_cnt,
                               void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q_reps == nullptr || k_reps == nullptr || k_pool == nullptr || v_pool == nullptr ||
      slot_gid == nullptr || slot_ema == nullptr || ws == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (nq <= 0 || capacity <= 0 || ncand < 0 || n_sink_gid < 0) return PBSA_ERR_INVALID_ARG;
  if (ncand > 0 && (cand_slot == nullptr || cand_gid == nullptr)) return PBSA_ERR_INVALID_ARG;
  if (!(gamma >= 0.f && gamma <= 1.f)) return PBSA_ERR_INVALID_ARG;
  if (!pool_ok(g, pool_slots) || capacity > pool_slots) return PBSA_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_reps) || !aligned16(q_reps))
    return PBSA_ERR_INVALID_ARG;
  if (capacity + ncand > 2048 || nq > 65535) return PBSA_ERR_UNSUPPORTED;
  return from_cuda(launch_memory_update(g, q_reps, nq, k_reps, k_pool, v_pool, pool_slots, slot_gid,
                                        slot_ema, capacity, n_sink_gid, cand_slot, cand_gid, ncand,
                                        gamma, p_list, p_cnt, ws, static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_memory_update_plan(const pbsa_geom* gin, const float* q_reps, int nq, const float* k_reps,
                                    int pool_slots, int* slot_gid, float* slot_ema, int capacity, int n_sink_gid,
                                    const int* cand_slot, const int* cand_gid, int ncand, float gamma, int* p_list,
                                    int* p_cnt, int flags, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q_reps == nullptr || k_reps == nullptr || slot_gid == nullptr || slot_ema == nullptr || ws == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (nq <= 0 || capacity <= 0 || ncand < 0 || n_sink_gid < 0) return PBSA_ERR_INVALID_ARG;
  if (ncand > 0 && (cand_slot == nullptr || cand_gid == nullptr)) return PBSA_ERR_INVALID_ARG;
  if (!(gamma >= 0.f && gamma <= 1.f)) return PBSA_ERR_INVALID_ARG;
  if (!pool_ok(g, pool_slots) || capacity > pool_slots) return PBSA_ERR_INVALID_ARG;
  if (!aligned16(k_reps) || !aligned16(q_reps)) return PBSA_ERR_INVALID_ARG;
  if ((flags & ~PBSA_OVERLAP_PREVIOUS) != 0) return PBSA_ERR_INVALID_ARG;
  if (capacity + ncand > 2048 || nq > 65535) return PBSA_ERR_UNSUPPORTED;
  return from_cuda(launch_memory_update_plan(g, q_reps, nq, k_reps, pool_slots, slot_gid, slot_ema, capacity,
                                             n_sink_gid, cand_slot, cand_gid, ncand, gamma, p_list, p_cnt,
                                             (flags & PBSA_OVERLAP_PREVIOUS) != 0, ws,
                                             static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_memory_update_apply(const pbsa_geom* gin, float* k_reps, void* k_pool, void* v_pool,
                                     int pool_slots, int capacity, int ncand, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (k_reps == nullptr || k_pool == nullptr || v_pool == nullptr || ws == nullptr) return PBSA_ERR_INVALID_ARG;
  if (capacity <= 0 || ncand < 0 || !pool_ok(g, pool_slots) || capacity > pool_slots) return PBSA_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_reps)) return PBSA_ERR_INVALID_ARG;
  if (capacity + ncand > 2048) return PBSA_ERR_UNSUPPORTED;
  return from_cuda(launch_memory_update_apply(g, k_reps, k_pool, v_pool, pool_slots, capacity, ncand, ws,
                                              static_cast<cudaStream_t>(stream)));
}

size_t pbsa_bwd_workspace_bytes(const pbsa_geom* gin, int q_frames, int pool_slots, int kv_ld) {
  Geo g;
  if (make_geo(gin, &g) != PBSA_OK || q_frames <= 0 || pool_slots <= 0 || kv_ld <= 0) return 0;
  return attend_bwd_ws_bytes(g, q_frames, pool_slots, kv_ld);
}

pbsa_status pbsa_attend_bwd(const pbsa_geom* gin, const void* q, int q_frames, const void* k_pool,
                            const void* v_pool, int pool_slots, const int* kv_slot, const int* kv_cnt,
                            int kv_ld, const void* o, const void* d_o, const float* lse, void* dq,
                            void* dk_pool, void* dv_pool, void* ws, void* stream) {
  Geo g;
  pbsa_status s = make_geo(gin, &g);
  if (s != PBSA_OK) return s;
  if (q == nullptr || k_pool == nullptr || v_pool == nullptr || kv_slot == nullptr || kv_cnt == nullptr ||
      o == nullptr || d_o == nullptr || lse == nullptr || dq == nullptr || dk_pool == nullptr ||
      dv_pool == nullptr || ws == nullptr)
    return PBSA_ERR_INVALID_ARG;
  if (q_frames <= 0 || kv_ld <= 0 || !pool_ok(g, pool_slots)) return PBSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k_pool, v_pool, o, d_o, dq, dk_pool, dv_pool, ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return PBSA_ERR_INVALID_ARG;
  if (g.dtype != PBSA_BF16 || g.d != 128 || kv_ld > 512) return PBSA_ERR_UNSUPPORTED;
  const int64_t nq = (int64_t)q_frames * g.bpf;
  if (nq > 512 || (int64_t)q_frames * g.tpf * g.H > ((int64_t)1 << 31)) return PBSA_ERR_UNSUPPORTED;
  return from_cuda(launch_attend_bwd(g, q, q_frames, k_pool, v_pool, pool_slots, kv_slot, kv_cnt, kv_ld,
                                     o, d_o, lse, dq, dk_pool, dv_pool, ws, static_cast<cudaStream_t>(stream)));
}

pbsa_status pbsa_selftest_wait_timeout(void* ws, unsigned int limit_us, void* stream) {
  if (ws == nullptr || limit_us == 0 || limit_us > 1000000) return PBSA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ws, (unsigned long long)limit_us * 1000ull);
  return from_cuda(cudaGetLastError());
}

pbsa_status pbsa_get_device_error(void* ws, void* stream) {
  if (ws == nullptr) return PBSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PBSA_ERR_CUDA;
  DevErr e;
  if (cudaMemcpy(&e, ws, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return PBSA_ERR_CUDA;
  if (e.code != 0) {
    const DevErr zero = {0, 0, 0, 0};
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return PBSA_ERR_CUDA;
  }
  return static_cast<pbsa_status>(e.code);
}

const char* pbsa_status_string(pbsa_status s) {
  switch (s) {
    case PBSA_OK: return "ok";
    case PBSA_ERR_INVALID_ARG: return "invalid argument";
    case PBSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PBSA_ERR_CUDA: return "CUDA error";
    case PBSA_ERR_TIMEOUT: return "device wait timed out";
    case PBSA_ERR_DEVICE_INDEX: return "index out of range on the device";
  }
  return "unknown status";
}

}  // extern "C"
