// a4 -- persistent-memory update ("Top-C retention").
//
// Sparse Forcing (gist.science, English 2.C "Dynamic Update"; Chinese 2.2 "粗粒度评分与
// 更新"): as the local window slides, the blocks that leave it are coarse-scored together
// with the persistent set; the best are promoted into the persistent memory, low scorers
// are dropped, and the sink blocks are always kept.  The scoring rule is fixed as an EMA of
// each block's mean (over the chunk's query blocks) softmaxed coarse score.
//
// Three launches on the caller's stream:
//   1. mu_score_kernel  -- one CTA per (head, 8 query blocks): coarse scores against every
//      pool entry (representatives staged in shared memory) and the per-row softmax,
//      written to the workspace;
//   2. mu_select_kernel -- one CTA per head: a_b = mean_r p_{r,b} (coalesced, fixed-order
//      sums), the EMA, the rank of every non-sink block, the new slot table and a copy
//      list in the workspace;
//   3. mu_copy_kernel   -- one CTA per (copy, head, K|V): promoted blocks are copied from
//      their window slots into the freed persistent slots (HBM-bound 16-byte copies).
// All reductions run in a fixed order, so the update is deterministic.
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

constexpr int MU_RC = 8;       // query rows per score CTA
constexpr int MU_CH = 128;     // pool entries staged per pass
constexpr int MU_SEL_THREADS = 512;

// Pool entry j of head h: j < C is persistent slot j (empty when its gid < 0), j >= C is
// candidate j - C, which must live outside the persistent region.  Returns the gid (-1 for
// an empty or rejected entry) and the slot.
__device__ __forceinline__ int entry_of(int j, int h, int C, int ncand, int pool_slots,
                                        const int* slot_gid, const int* cand_slot,
                                        const int* cand_gid, int* slot_out, void* ws, bool report) {
  if (j < C) {
    *slot_out = j;
    return slot_gid[(size_t)h * C + j];
  }
  const int g = cand_gid[(size_t)h * ncand + (j - C)];
  const int s = cand_slot[(size_t)h * ncand + (j - C)];
  *slot_out = s;
  if (g >= 0 && (s < C || s >= pool_slots)) {
    if (report) record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_MU_SCORE);
    return -1;
  }
  return g;
}

template <int D>
__global__ void __launch_bounds__(MU_THREADS) mu_score_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    const int* __restrict__ slot_gid, int C, const int* __restrict__ cand_slot,
    const int* __restrict__ cand_gid, int ncand, float scale, float* __restrict__ p_out, void* ws) {
  constexpr int DP = D + 1;
  extern __shared__ float smem[];
  const int h = blockIdx.y, r0 = blockIdx.x * MU_RC, nb = C + ncand;
  const int nr = min(MU_RC, nq - r0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* ks = smem;                          // [MU_CH][DP]
  float* qs = ks + MU_CH * DP;               // [MU_RC][D]
  float* sc = qs + MU_RC * D;                // [MU_RC][nb]
  int* gid = reinterpret_cast<int*>(sc + MU_RC * nb);   // [nb]
  int* eslot = gid + nb;                                 // [nb]

  for (int j = tid; j < nb; j += MU_THREADS) {
    int sl;
    gid[j] = entry_of(j, h, C, ncand, pool_slots, slot_gid, cand_slot, cand_gid, &sl, ws, blockIdx.x == 0);
    eslot[j] = sl;
  }
  for (int i = tid; i < MU_RC * D; i += MU_THREADS) {
    const int r = i / D;
    qs[i] = r < nr ? q_reps[((size_t)h * nq + r0 + r) * D + (i - r * D)] : 0.f;
  }
  for (int base = 0; base < nb; base += MU_CH) {
    const int nc = min(MU_CH, nb - base);
    __syncthreads();   // metadata ready / previous pass done with ks
    stage_rows<D, DP, MU_THREADS>(ks, nc, [&](int c) -> const float* {
      return gid[base + c] >= 0 ? k_reps + ((size_t)h * pool_slots + eslot[base + c]) * D : nullptr;
    });
    __syncthreads();
    for (int p = tid; p < nc * (MU_RC / 4); p += MU_THREADS) {
      const int c = p % nc, rg = (p / nc) * 4;
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
      const float* kr = ks + c * DP;
#pragma unroll 8
      for (int e = 0; e < D; ++e) {
        const float kv = kr[e];
#pragma unroll
        for (int j = 0; j < 4; ++j) a4[j] = fmaf(qs[(rg + j) * D + e], kv, a4[j]);
      }
      const bool ok = gid[base + c] >= 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[(rg + j) * nb + base + c] = ok ? a4[j] * scale : -INFINITY;
    }
  }
  __syncthreads();
  // softmax of each row over the pool (one warp per row, fixed-order reductions)
  for (int r = warp; r < nr; r += MU_THREADS / 32) {
    const float* row = sc + r * nb;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) sum += row[j] == -INFINITY ? 0.f : expf(row[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.0f / sum : 0.f;
    float* prow = p_out + ((size_t)h * nq + r0 + r) * nb;
    for (int j = lane; j < nb; j += 32) prow[j] = row[j] == -INFINITY ? 0.f : expf(row[j] - m) * inv;
  }
}

__global__ void __launch_bounds__(MU_SEL_THREADS) mu_select_kernel(
    const float* __restrict__ p_in, int nq, int pool_slots, int* __restrict__ slot_gid,
    float* __restrict__ slot_ema, int C, int n_sink_gid, const int* __restrict__ cand_slot,
    const int* __restrict__ cand_gid, int ncand, float gamma, int* __restrict__ copy_list,
    int* __restrict__ ncopy, int* __restrict__ p_list, int* __restrict__ p_cnt, void* ws) {
  constexpr int NW = MU_SEL_THREADS / 32;
  extern __shared__ float smem[];
  const int h = blockIdx.x, nb = C + ncand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* part = smem;                        // [NW][nb] per-warp partial sums over rows
  float* ema = part + NW * nb;               // [nb]
  int* gid = reinterpret_cast<int*>(ema + nb);   // [nb]
  int* eslot = gid + nb;                         // [nb]
  int* rank = eslot + nb;                        // [nb]
  int* by_rank = rank + nb;                      // [nb]
  int* filled = by_rank + nb;                    // [nb]
  int* flist = filled + nb;                      // [nb] freed persistent slots, ascending
  int* plist2 = flist + nb;                      // [nb] promoted entries, in promotion order
  __shared__ int n_sink_s, n_free_s, n_promo_s;
  if (tid == 0) n_sink_s = 0;
  for (int j = tid; j < nb; j += MU_SEL_THREADS) {
    int sl;
    gid[j] = entry_of(j, h, C, ncand, pool_slots, slot_gid, cand_slot, cand_gid, &sl, ws, false);
    eslot[j] = sl;
    by_rank[j] = -1;
    filled[j] = 0;
  }
  // warp w sums rows w, w + NW, ...; lanes walk consecutive entries (coalesced)
  const float* pbase = p_in + (size_t)h * nq * nb;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    float a = 0.f;
    if (j < nb) {
#pragma unroll 4
      for (int r = warp; r < nq; r += NW) a += pbase[(size_t)r * nb + j];
      part[warp * nb + j] = a;
    }
  }
  __syncthreads();
  const float inv_nq = 1.0f / (float)nq;
  for (int j = tid; j < nb; j += MU_SEL_THREADS) {
    float a = 0.f;
    for (int w = 0; w < NW; ++w) a += part[w * nb + j];
    a *= inv_nq;
    const int g = gid[j];
    ema[j] = (g >= 0 && j < C) ? fmaf(gamma, slot_ema[(size_t)h * C + j], (1.0f - gamma) * a) : a;
    if (g >= 0 && g < n_sink_gid) atomicAdd(&n_sink_s, 1);
  }
  __syncthreads();
  const int free_places = max(0, C - n_sink_s);
  for (int j = tid; j < nb; j += MU_SEL_THREADS) {
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
  auto stays = [&](int j) {
    const int g = gid[j];
    return g >= 0 && (g < n_sink_gid || (rank[j] >= 0 && rank[j] < free_places));
  };
  // Hand the freed persistent slots (ascending) to the promoted candidates: sinks first
  // (entry order), then the kept non-sinks in rank order.  Warp 0 lists the freed slots,
  // warp 1 the promotion order (ballot prefix sums), then all threads apply it.
  if (warp == 0) {
    int n = 0;
    for (int base = 0; base < C; base += 32) {
      const int j = base + lane;
      const bool fr = j < C && !stays(j);
      const unsigned bal = __ballot_sync(0xffffffffu, fr);
      if (fr) flist[n + __popc(bal & ((1u << lane) - 1u))] = j;
      n += __popc(bal);
    }
    if (lane == 0) n_free_s = n;
  } else if (warp == 1) {
    int n = 0;
    for (int base = C; base < nb; base += 32) {         // sink candidates, entry order
      const int j = base + lane;
      const bool t = j < nb && gid[j] >= 0 && gid[j] < n_sink_gid;
      const unsigned bal = __ballot_sync(0xffffffffu, t);
      if (t) plist2[n + __popc(bal & ((1u << lane) - 1u))] = j;
      n += __popc(bal);
    }
    const int nq2 = min(free_places, nb);
    for (int base = 0; base < nq2; base += 32) {        // kept non-sink candidates, rank order
      const int q = base + lane;
      const int j = q < nq2 ? by_rank[q] : -1;
      const bool t = j >= C;
      const unsigned bal = __ballot_sync(0xffffffffu, t);
      if (t) plist2[n + __popc(bal & ((1u << lane) - 1u))] = j;
      n += __popc(bal);
    }
    if (lane == 0) n_promo_s = n;
  }
  __syncthreads();
  const int n_promo = n_promo_s, n_free = n_free_s;
  for (int t = tid; t < n_promo; t += MU_SEL_THREADS) {
    const int j = plist2[t];
    if (t >= n_free) {
      record_error(ws, PBSA_ERR_INVALID_ARG, j, K_MU_SELECT);
      continue;
    }
    const int dst = flist[t];
    copy_list[((size_t)h * nb + t) * 2 + 0] = eslot[j];
    copy_list[((size_t)h * nb + t) * 2 + 1] = dst;
    filled[dst] = 1;
    slot_gid[(size_t)h * C + dst] = gid[j];
    slot_ema[(size_t)h * C + dst] = ema[j];
  }
  if (tid == 0) ncopy[h] = min(n_promo, n_free);
  __syncthreads();
  // kept persistent entries take their new EMA; slots neither kept nor refilled are cleared
  for (int j = tid; j < C; j += MU_SEL_THREADS) {
    if (stays(j)) {
      slot_ema[(size_t)h * C + j] = ema[j];
    } else if (!filled[j]) {
      slot_gid[(size_t)h * C + j] = -1;
      slot_ema[(size_t)h * C + j] = 0.f;
    }
  }
  // compacted list of the valid persistent slots (ascending)
  if (warp == 0) {
    int n = 0;
    for (int base = 0; base < C; base += 32) {
      const int j = base + lane;
      const bool v = j < C && (stays(j) || filled[j]);
      const unsigned bal = __ballot_sync(0xffffffffu, v);
      if (v && p_list) p_list[(size_t)h * C + n + __popc(bal & ((1u << lane) - 1u))] = j;
      n += __popc(bal);
    }
    if (lane == 0 && p_cnt) p_cnt[h] = n;
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
  int* copy_list = reinterpret_cast<int*>(base + L.copy_off);
  int* ncopy = reinterpret_cast<int*>(base + L.ncopy_off);
  cudaError_t e;

  float* p = reinterpret_cast<float*>(base + L.p_off);
  const size_t smem1 = ((size_t)MU_CH * (D + 1) + (size_t)MU_RC * D + (size_t)MU_RC * nb) * 4 + (size_t)nb * 8;
  if ((e = set_smem_once((const void*)mu_score_kernel<D>, (int)smem1)) != cudaSuccess) return e;
  mu_score_kernel<D><<<dim3((nq + MU_RC - 1) / MU_RC, g.H), MU_THREADS, smem1, st>>>(
      q_reps, nq, k_reps, pool_slots, slot_gid, C, cand_slot, cand_gid, ncand, g.scale, p, ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem2 = ((size_t)(MU_SEL_THREADS / 32) * nb + nb) * 4 + (size_t)nb * 7 * sizeof(int);
  if ((e = set_smem_once((const void*)mu_select_kernel, (int)smem2)) != cudaSuccess) return e;
  mu_select_kernel<<<g.H, MU_SEL_THREADS, smem2, st>>>(p, nq, pool_slots, slot_gid, slot_ema, C, n_sink_gid,
                                                        cand_slot, cand_gid, ncand, gamma, copy_list, ncopy,
                                                        p_list, p_cnt, ws);
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
