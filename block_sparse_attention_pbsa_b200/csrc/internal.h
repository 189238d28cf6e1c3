// Host-side declarations shared by the translation units of libpbsa.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pbsa.h"

namespace pbsa {

// Validated, derived geometry.
struct Geo {
  int H, d;
  int fh, fw, th, tw;
  int tpr;   // tiles per row of a frame
  int bpf;   // blocks per frame
  int tpf;   // tokens per frame
  float scale;
  int dtype;
  int esize;  // bytes per token element
};

// Kernel ids recorded with device errors.
enum KernelId { K_BLOCKIFY = 1, K_SCORE = 2, K_ATTEND_F32 = 3, K_ATTEND_TC = 4, K_MU_SCORE = 5,
                K_MU_SELECT = 6, K_MU_COPY = 7, K_BWD_PREP = 8, K_BWD_KV = 9, K_BWD_Q = 10,
                K_SELFTEST = 11 };

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bound of every in-kernel wait

cudaError_t launch_blockify(const Geo& g, const void* x, int n_frames, float* reps, int rep_slots,
                            const int* dst_slot, void* pool, int pool_slots, void* ws,
                            cudaStream_t st);

// K and V (x1, reps1, pool1 nullable: one tensor only; reps0/reps1 nullable: no reps of that
// tensor) in one launch, with the same destination slots; overlap_previous: programmatic
// dependent launch after the previous kernel on the stream.
cudaError_t launch_blockify_pair(const Geo& g, const void* x0, const void* x1, int n_frames, float* reps0,
                                 float* reps1, int rep_slots, const int* dst_slot, void* pool0, void* pool1,
                                 int pool_slots, bool overlap_previous, void* ws, cudaStream_t st);

cudaError_t launch_score_select(const Geo& g, const float* q_reps, int nq, const float* k_reps,
                                int pool_slots, const int* cand_slot, const int* cand_gid,
                                int ncand, int k, const int* prefix_slot, const int* prefix_cnt,
                                int prefix_ld, int* out_slot, int* out_cnt, int out_ld,
                                float* out_score, void* ws, cudaStream_t st);

cudaError_t launch_blockify_select(const Geo& g, const void* x, int q_frames, float* q_reps,
                                   const float* k_reps, int pool_slots, const int* cand_slot,
                                   const int* cand_gid, int ncand, int k, const int* prefix_slot,
                                   const int* prefix_cnt, int prefix_ld, int* out_slot,
                                   int* out_cnt, int out_ld, float* out_score, int top_frames,
                                   int n_recent, const int* suffix_slot, int suffix_n, void* ws,
                                   cudaStream_t st);

// The trainable path's lists (chunk-causal, sequences folded into the frame axis, slot = block id).
cudaError_t launch_blockify_train_select(const Geo& g, const void* x, int q_frames, float* q_reps,
                                         const float* k_reps, int pool_slots, int seq_frames,
                                         int chunk_frames, int sink_frames, int k, int* out_slot,
                                         int* out_cnt, int out_ld, float* out_score, void* ws,
                                         cudaStream_t st);

cudaError_t launch_attend_f32(const Geo& g, const float* q, int q_frames, const float* k_pool,
                              const float* v_pool, int pool_slots, const int* kv_slot,
                              const int* kv_cnt, int kv_ld, float* o, float* lse, void* ws,
                              cudaStream_t st);

// Returns cudaErrorNotSupported when the tensor maps cannot be encoded.
cudaError_t launch_attend_tc(const Geo& g, const void* q, int q_frames, const void* k_pool,
                             const void* v_pool, int pool_slots, const int* kv_slot,
                             const int* kv_cnt, int kv_ld, void* o, float* lse, void* ws,
                             cudaStream_t st);

size_t memory_update_ws_bytes(const Geo& g, int max_q_blocks, int max_pool_entries);
cudaError_t launch_memory_update(const Geo& g, const float* q_reps, int nq, float* k_reps,
                                 void* k_pool, void* v_pool, int pool_slots, int* slot_gid,
                                 float* slot_ema, int C, int n_sink_gid, const int* cand_slot,
                                 const int* cand_gid, int ncand, float gamma, int* p_list,
                                 int* p_cnt, void* ws, cudaStream_t st);

// The update in two launches: plan (scores, ranking, slot table, copy list in ws; no pool
// access) and apply (the copies).  overlap_previous: programmatic dependent launch of the plan.
cudaError_t launch_memory_update_plan(const Geo& g, const float* q_reps, int nq, const float* k_reps,
                                      int pool_slots, int* slot_gid, float* slot_ema, int C, int n_sink_gid,
                                      const int* cand_slot, const int* cand_gid, int ncand, float gamma,
                                      int* p_list, int* p_cnt, bool overlap_previous, void* ws, cudaStream_t st);
cudaError_t launch_memory_update_apply(const Geo& g, float* k_reps, void* k_pool, void* v_pool, int pool_slots,
                                       int C, int ncand, void* ws, cudaStream_t st);

size_t attend_bwd_ws_bytes(const Geo& g, int q_frames, int pool_slots, int kv_ld);
cudaError_t launch_attend_bwd(const Geo& g, const void* q, int q_frames, const void* k_pool,
                              const void* v_pool, int pool_slots, const int* kv_slot,
                              const int* kv_cnt, int kv_ld, const void* o, const void* d_o,
                              const float* lse, void* dq, void* dk_pool, void* dv_pool, void* ws,
                              cudaStream_t st);

// cuTensorMapEncodeTiled, fetched from the driver at first use (no -lcuda link needed).
void* tensor_map_encoder();
// Encode a bf16 tensor map with 128-byte swizzle (dims/strides fastest first, strides in bytes).
bool encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device, size): later
// calls, including calls made while a stream is being captured, skip the driver call.
cudaError_t set_smem_once(const void* kernel, int bytes);

}  // namespace pbsa
