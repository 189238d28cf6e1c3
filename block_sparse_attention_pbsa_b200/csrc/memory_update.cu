// a4 -- persistent-memory update ("Top-C retention").
//
// Sparse Forcing (gist.science, English 2.C "Dynamic Update"; Chinese 2.2 "粗粒度评分与
// 更新"): as the local window slides, the blocks that leave it are coarse-scored together
// with the persistent set; the best are promoted into the persistent memory, low scorers
// are dropped, and the sink blocks are always kept.  The scoring rule is fixed as an EMA of
// each block's mean (over the chunk's query blocks) softmaxed coarse score.
//
// Three launches on the caller's stream:
//   1. mu_score_kernel  -- one CTA per (query block, head): scores over the pool and the
//      softmax row p_r, written to the workspace (deterministic, no atomics);
//   2. mu_select_kernel -- one CTA per head: a_b = mean_r p_{r,b}, the EMA, the rank of
//      every non-sink block, the new slot table and a copy list;
//   3. mu_copy_kernel   -- one CTA per (copy, head, K|V): promoted blocks are copied from
//      their window slots into the freed persistent slots (HBM-bound 16-byte copies).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int MU_THREADS = 256;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct MuLayout {
  size_t p_off, copy_off, ncopy_off, end;
};
__host__ __device__ inline MuLayout mu_layout(int H, int nq, int nb) {
  MuLayout L;
  L.p_off = WS_HEADER_BYTES;
  L.copy_off = L.p_off + align256((size_t)H * nq * nb * sizeof(float));
  L.ncopy_off = L.copy_off + align256((size_t)H * nb * 2 * sizeof(int));
  L.end = L.ncopy_off + align256((size_t)H * sizeof(int));
  return L;
}

// Entry j of head h's pool: j < C is persistent slot j (valid if its gid >= 0), j >= C is
// candidate j - C.  Returns the pool slot, or -2 when the entry is empty.
__device__ __forceinline__ int entry_slot(int j, int h, int C, const int* slot_gid,
                                          const int* cand_slot, const int* cand_gid, int ncand) {
  if (j < C) return slot_gid[(size_t)h * C + j] >= 0 ? j : -2;
  if (cand_gid[(size_t)h * ncand + (j - C)] < 0) return -2;
  return cand_slot[(size_t)h * ncand + (j - C)];
}

template <int D>
__global__ void __launch_bounds__(MU_THREADS) mu_score_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    const int* __restrict__ slot_gid, int C, const int* __restrict__ cand_slot,
    const int* __restrict__ cand_gid, int ncand, float scale, float* __restrict__ p_out, void* ws) {
  extern __shared__ float sc[];  // [nb]
  __shared__ float qs[D];
  __shared__ float red[MU_THREADS / 32];
  const int r = blockIdx.x, h = blockIdx.y, nb = C + ncand;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < D; e += MU_THREADS) qs[e] = q_reps[((size_t)h * nq + r) * D + e];
  __syncthreads();
  for (int j = warp; j < nb; j += MU_THREADS / 32) {
    const int s = entry_slot(j, h, C, slot_gid, cand_slot, cand_gid, ncand);
    const bool ok = s >= 0 && s < pool_slots;
    float acc = 0.f;
    if (ok) {
      const float* kr = k_reps + ((size_t)h * pool_slots + s) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) acc = fmaf(qs[lane + 32 * i], __ldg(kr + lane + 32 * i), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      // a candidate must live outside the persistent region, inside the pool
      const bool bad = j >= C && s != -2 && (s < C || s >= pool_slots);
      if (bad) record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_MU_SCORE);
      sc[j] = (ok && !bad) ? acc * scale : -INFINITY;
    }
  }
  __syncthreads();
  // softmax over the valid entries of this row (fixed-order block reductions)
  float m = -INFINITY;
  for (int j = threadIdx.x; j < nb; j += MU_THREADS) m = fmaxf(m, sc[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < MU_THREADS / 32; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < nb; j += MU_THREADS) {
    const float e = (sc[j] == -INFINITY) ? 0.f : expf(sc[j] - m);
    sc[j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < MU_THREADS / 32; ++w) sum += red[w];
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  float* prow = p_out + ((size_t)h * nq + r) * nb;
  for (int j = threadIdx.x; j < nb; j += MU_THREADS) prow[j] = sc[j] * inv;
}

__global__ void __launch_bounds__(MU_THREADS) mu_select_kernel(
    const float* __restrict__ p_in, int nq, int* __restrict__ slot_gid, float* __restrict__ slot_ema,
    int C, int n_sink_gid, const int* __restrict__ cand_slot, const int* __restrict__ cand_gid,
    int ncand, float gamma, int* __restrict__ copy_list, int* __restrict__ ncopy,
    int* __restrict__ p_list, int* __restrict__ p_cnt, void* ws) {
  extern __shared__ int sm[];
  const int h = blockIdx.x, nb = C + ncand;
  float* ema = reinterpret_cast<float*>(sm);   // [nb]
  int* gid = sm + nb;                          // [nb], -1 = empty entry
  int* rank = gid + nb;                        // [nb], -1 = not a ranked (non-sink) entry
  int* by_rank = rank + nb;                    // [nb]
  int* filled = by_rank + nb;                  // [nb], 1 = persistent slot refilled by a promotion
  __shared__ int n_sink_s;
  if (threadIdx.x == 0) n_sink_s = 0;
  __syncthreads();

  const float inv_nq = 1.0f / (float)nq;
  for (int j = threadIdx.x; j < nb; j += MU_THREADS) {
    int g;
    float prev = 0.f;
    if (j < C) {
      g = slot_gid[(size_t)h * C + j];
      prev = slot_ema[(size_t)h * C + j];
    } else {
      g = cand_gid[(size_t)h * ncand + (j - C)];
    }
    gid[j] = g;
    float a = 0.f;
    if (g >= 0) {
      const float* pc = p_in + (size_t)h * nq * nb + j;
      for (int r = 0; r < nq; ++r) a += pc[(size_t)r * nb];
      a *= inv_nq;
      if (g < n_sink_gid) atomicAdd(&n_sink_s, 1);
    }
    ema[j] = (g >= 0 && j < C) ? fmaf(gamma, prev, (1.0f - gamma) * a) : a;
    by_rank[j] = -1;
    filled[j] = 0;
  }
  __syncthreads();
  const int free_places = max(0, C - n_sink_s);
  for (int j = threadIdx.x; j < nb; j += MU_THREADS) {
    const int g = gid[j];
    int rk = -1;
    if (g >= n_sink_gid) {
      const float e = ema[j];
      rk = 0;
      for (int j2 = 0; j2 < nb; ++j2) {
        const int g2 = gid[j2];
        if (g2 < n_sink_gid) continue;  // empty entries and sinks are not ranked
        const float e2 = ema[j2];
        rk += (e2 > e) || (e2 == e && (g2 < g || (g2 == g && j2 < j)));
      }
      if (rk < free_places) by_rank[rk] = j;
    }
    rank[j] = rk;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Walk freed slots ascending and hand them to promoted candidates: sinks first (entry
    // order), then the kept non-sinks in rank order.  Serial: O(C + ncand).
    int next_free = 0, t = 0;
    auto take_free = [&](void) -> int {
      while (next_free < C) {
        const int j = next_free++;
        const bool stays = gid[j] >= 0 && (gid[j] < n_sink_gid || (rank[j] >= 0 && rank[j] < free_places));
        if (!stays) return j;
      }
      return -1;
    };
    auto promote = [&](int j) {
      const int dst = take_free();
      if (dst < 0) { record_error(ws, PBSA_ERR_INVALID_ARG, j, K_MU_SELECT); return; }
      copy_list[((size_t)h * nb + t) * 2 + 0] = cand_slot[(size_t)h * ncand + (j - C)];
      copy_list[((size_t)h * nb + t) * 2 + 1] = dst;
      ++t;
      filled[dst] = 1;
      slot_gid[(size_t)h * C + dst] = gid[j];
      slot_ema[(size_t)h * C + dst] = ema[j];
    };
    for (int j = C; j < nb; ++j)
      if (gid[j] >= 0 && gid[j] < n_sink_gid) promote(j);
    for (int q = 0; q < free_places && q < nb; ++q) {
      const int j = by_rank[q];
      if (j >= C) promote(j);
    }
    ncopy[h] = t;
  }
  __syncthreads();
  // Persistent entries: kept ones get their new EMA; dropped / empty ones are cleared unless
  // a promotion took the slot (thread 0 wrote those above, and they are not "stays").
  for (int j = threadIdx.x; j < C; j += MU_THREADS) {
    const int g = gid[j];
    const bool stays = g >= 0 && (g < n_sink_gid || (rank[j] >= 0 && rank[j] < free_places));
    if (stays) {
      slot_ema[(size_t)h * C + j] = ema[j];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Clear slots that are neither kept nor refilled; build the compacted persistent list.
    int n = 0;
    for (int j = 0; j < C; ++j) {
      const int g = gid[j];
      const bool stays = g >= 0 && (g < n_sink_gid || (rank[j] >= 0 && rank[j] < free_places));
      const bool refilled = filled[j] != 0;
      if (!stays && !refilled) {
        slot_gid[(size_t)h * C + j] = -1;
        slot_ema[(size_t)h * C + j] = 0.f;
      }
      if (stays || refilled) {
        if (p_list) p_list[(size_t)h * C + n] = j;
        ++n;
      }
    }
    if (p_cnt) p_cnt[h] = n;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(MU_THREADS) mu_copy_kernel(
    const int* __restrict__ copy_list, const int* __restrict__ ncopy, int nb, int C, float* k_reps,
    T* k_pool, T* v_pool, int pool_slots, void* ws) {
  const int t = blockIdx.x, h = blockIdx.y, which = blockIdx.z;
  if (t >= ncopy[h]) return;
  const int src = copy_list[((size_t)h * nb + t) * 2 + 0];
  const int dst = copy_list[((size_t)h * nb + t) * 2 + 1];
  if (src < C || src >= pool_slots || dst < 0 || dst >= C) {
    if (threadIdx.x == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, src, K_MU_COPY);
    return;
  }
  T* pool = which ? v_pool : k_pool;
  const uint4* s = reinterpret_cast<const uint4*>(pool + ((size_t)h * pool_slots + src) * BT * D);
  uint4* d = reinterpret_cast<uint4*>(pool + ((size_t)h * pool_slots + dst) * BT * D);
  constexpr int N16 = BT * D * (int)sizeof(T) / 16;
  uint4 buf[(N16 + MU_THREADS - 1) / MU_THREADS];
#pragma unroll
  for (int i = 0; i < (N16 + MU_THREADS - 1) / MU_THREADS; ++i) {
    const int e = threadIdx.x + i * MU_THREADS;
    if (e < N16) buf[i] = s[e];
  }
#pragma unroll
  for (int i = 0; i < (N16 + MU_THREADS - 1) / MU_THREADS; ++i) {
    const int e = threadIdx.x + i * MU_THREADS;
    if (e < N16) d[e] = buf[i];
  }
  if (which == 0)
    for (int e = threadIdx.x; e < D; e += MU_THREADS)
      k_reps[((size_t)h * pool_slots + dst) * D + e] = k_reps[((size_t)h * pool_slots + src) * D + e];
}

template <int D>
cudaError_t launch_mu(const Geo& g, const float* q_reps, int nq, float* k_reps, void* k_pool,
                      void* v_pool, int pool_slots, int* slot_gid, float* slot_ema, int C,
                      int n_sink_gid, const int* cand_slot, const int* cand_gid, int ncand,
                      float gamma, int* p_list, int* p_cnt, void* ws, cudaStream_t st) {
  const int nb = C + ncand;
  const MuLayout L = mu_layout(g.H, nq, nb);
  char* base = static_cast<char*>(ws);
  float* p = reinterpret_cast<float*>(base + L.p_off);
  int* copy_list = reinterpret_cast<int*>(base + L.copy_off);
  int* ncopy = reinterpret_cast<int*>(base + L.ncopy_off);
  cudaError_t e;

  const size_t smem1 = (size_t)nb * sizeof(float);
  if (smem1 > 48 * 1024) {
    e = cudaFuncSetAttribute(mu_score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
  }
  mu_score_kernel<D><<<dim3(nq, g.H), MU_THREADS, smem1, st>>>(
      q_reps, nq, k_reps, pool_slots, slot_gid, C, cand_slot, cand_gid, ncand, g.scale, p, ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const size_t smem2 = (size_t)nb * 5 * sizeof(int);
  if (smem2 > 48 * 1024) {
    e = cudaFuncSetAttribute(mu_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
  }
  mu_select_kernel<<<g.H, MU_THREADS, smem2, st>>>(p, nq, slot_gid, slot_ema, C, n_sink_gid,
                                                   cand_slot, cand_gid, ncand, gamma, copy_list,
                                                   ncopy, p_list, p_cnt, ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const int max_copies = C < nb ? C : nb;
  if (max_copies > 0) {
    dim3 grid(max_copies, g.H, 2);
    if (g.dtype == PBSA_BF16)
      mu_copy_kernel<__nv_bfloat16, D><<<grid, MU_THREADS, 0, st>>>(
          copy_list, ncopy, nb, C, k_reps, static_cast<__nv_bfloat16*>(k_pool),
          static_cast<__nv_bfloat16*>(v_pool), pool_slots, ws);
    else
      mu_copy_kernel<float, D><<<grid, MU_THREADS, 0, st>>>(copy_list, ncopy, nb, C, k_reps,
                                                            static_cast<float*>(k_pool),
                                                            static_cast<float*>(v_pool), pool_slots, ws);
  }
  return cudaGetLastError();
}

}  // namespace

size_t memory_update_ws_bytes(const Geo& g, int max_q_blocks, int max_pool_entries) {
  return mu_layout(g.H, max_q_blocks, max_pool_entries).end;
}

cudaError_t launch_memory_update(const Geo& g, const float* q_reps, int nq, float* k_reps,
                                 void* k_pool, void* v_pool, int pool_slots, int* slot_gid,
                                 float* slot_ema, int C, int n_sink_gid, const int* cand_slot,
                                 const int* cand_gid, int ncand, float gamma, int* p_list,
                                 int* p_cnt, void* ws, cudaStream_t st) {
#define PBSA_MU(DD)                                                                          \
  return launch_mu<DD>(g, q_reps, nq, k_reps, k_pool, v_pool, pool_slots, slot_gid, slot_ema, \
                       C, n_sink_gid, cand_slot, cand_gid, ncand, gamma, p_list, p_cnt, ws, st);
  if (g.d == 128) { PBSA_MU(128) }
  if (g.d == 64) { PBSA_MU(64) }
  if (g.d == 32) { PBSA_MU(32) }
#undef PBSA_MU
  return cudaErrorNotSupported;
}

}  // namespace pbsa
