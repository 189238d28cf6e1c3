// a4 -- persistent-memory update ("Top-C retention").
//
// Sparse Forcing (gist.science, English 2.C "Dynamic Update"; Chinese 2.2 "粗粒度评分与
// 更新"): as the local window slides, the blocks that leave it are coarse-scored together
// with the persistent set; the best are promoted into the persistent memory, low scorers
// are dropped, and the sink blocks are always kept.  The scoring rule is fixed as an EMA of
// each block's mean (over the chunk's query blocks) softmaxed coarse score.
//
// Pools of up to 256 entries with up to 128 query blocks take one launch, mu_cluster_kernel
// (described at the kernel).  Larger ones take two launches on the caller's stream:
//   1. mu_score_select_kernel -- one CTA per (head, 4 query blocks): coarse scores against
//      every pool entry (warp per entry, lanes over d), the per-row softmax, and the column
//      sums of its rows written to the workspace.  The last CTA of each head to finish
//      (an atomic count in the workspace, reset by that CTA) then sums the column partials
//      in a fixed order (a_b = mean_r p_{r,b}), applies the EMA, ranks every non-sink block,
//      and writes the new slot table, the persistent list and a copy list;
//   2. mu_copy_kernel -- one CTA per (copy, head, K|V): promoted blocks are copied from their
//      window slots into the freed persistent slots (HBM-bound 16-byte copies).
// All reductions run in a fixed order, so the update is deterministic.
#include <cooperative_groups.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int MU_THREADS = 256;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

constexpr int MU_RQ = 4;       // query rows per score CTA
constexpr int MU_BATCH = 12;   // pool entries per warp in flight

struct MuLayout {
  size_t part_off, copy_off, ncopy_off, count_off, end;
};
constexpr int MU_MAX_HEADS = 4096;   // the geometry's limit on heads
// count [MU_MAX_HEADS] finished score CTAs per head, at a fixed offset for every shape (zero
// between calls; no other data ever lands there, whatever shapes share the workspace); copy
// list [H][2][nb] (sources, then destinations); ncopy [H]; part [H][ceil(nq / MU_RQ)][nb] column
// partial sums.  The copy list's offset depends on H and nb only (the apply step finds it
// without nq).
__host__ __device__ inline MuLayout mu_layout(int H, int nq, int nb) {
  MuLayout L;
  const size_t nqb = (size_t)(nq + MU_RQ - 1) / MU_RQ;
  L.count_off = WS_HEADER_BYTES;
  L.copy_off = L.count_off + align256((size_t)MU_MAX_HEADS * sizeof(int));
  L.ncopy_off = L.copy_off + align256((size_t)H * nb * 2 * sizeof(int));
  L.part_off = L.ncopy_off + align256((size_t)H * sizeof(int));
  L.end = L.part_off + align256((size_t)H * nqb * nb * sizeof(float));
  return L;
}

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

template <int N> struct MuVec;
template <> struct MuVec<4> { using type = float4; };
template <> struct MuVec<2> { using type = float2; };
template <> struct MuVec<1> { using type = float; };
__device__ __forceinline__ void mu_vec_to(const float4& v, float* o) { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
__device__ __forceinline__ void mu_vec_to(const float2& v, float* o) { o[0] = v.x; o[1] = v.y; }
__device__ __forceinline__ void mu_vec_to(const float& v, float* o) { o[0] = v; }

// The selection of one head from its a_b (in ema[], overwritten by the EMA): ranks, slot
// assignment, slot table, copy list, persistent list.  Run by one CTA (all threads).
// prev_ema: the head's slot_ema before the update ([C]; global memory or a shared copy).
__device__ void mu_select_head(int h, int nb, int pool_slots, int* __restrict__ slot_gid,
                               float* __restrict__ slot_ema, const float* prev_ema, int C, int n_sink_gid, float gamma,
                               const int* gid, const int* eslot, float* ema, uint64_t* key, int* rank,
                               int* by_rank, int* filled, int* flist, int* plist2, int* copy_src, int* copy_dst,
                               int* ncopy_h, int* __restrict__ p_list, int* __restrict__ p_cnt, void* ws) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, NT = blockDim.x;
  __shared__ int n_sink_s, n_free_s, n_promo_s;
  if (tid == 0) n_sink_s = 0;
  __syncthreads();
  for (int j = tid; j < nb; j += NT) {
    const int g = gid[j];
    const float a = ema[j];
    const float e = (g >= 0 && j < C) ? fmaf(gamma, prev_ema[j], (1.0f - gamma) * a) : a;
    ema[j] = e;
    // ranking key of a non-sink block: larger EMA first, then the lower gid; empty entries
    // and sinks get 0, below every ranked key
    key[j] = g >= n_sink_gid ? rank_key(e, g) : 0ull;
    if (g >= 0 && g < n_sink_gid) atomicAdd(&n_sink_s, 1);
    by_rank[j] = -1;
    filled[j] = 0;
  }
  __syncthreads();
  const int free_places = max(0, C - n_sink_s);
  // rank = #ranked keys above this one, plus equal keys at a lower entry (branch-free)
  if (NT >= 2 * nb) {
    // two threads per entry (neighbouring lanes), each counting over half of the keys
    const int j = tid >> 1, half = tid & 1;
    const int lo = half ? (nb + 1) / 2 : 0, hi = half ? nb : (nb + 1) / 2;
    const uint64_t kj = j < nb ? key[j] : 0ull;
    int rk = 0;
    if (kj != 0ull) {
#pragma unroll 8
      for (int j2 = lo; j2 < hi; ++j2) {
        const uint64_t k2 = key[j2];
        rk += (int)(k2 > kj) | ((int)(k2 == kj) & (int)(j2 < j));
      }
    }
    rk += __shfl_xor_sync(0xffffffffu, rk, 1);
    if (half == 0 && j < nb) {
      if (kj != 0ull && rk < free_places) by_rank[rk] = j;
      rank[j] = kj != 0ull ? rk : -1;
    }
  } else {
    for (int j = tid; j < nb; j += NT) {
      const uint64_t kj = key[j];
      int rk = -1;
      if (kj != 0ull) {
        rk = 0;
#pragma unroll 8
        for (int j2 = 0; j2 < nb; ++j2) {
          const uint64_t k2 = key[j2];
          rk += (int)(k2 > kj) | ((int)(k2 == kj) & (int)(j2 < j));
        }
        if (rk < free_places) by_rank[rk] = j;
      }
      rank[j] = rk;
    }
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
  for (int t = tid; t < n_promo; t += NT) {
    const int j = plist2[t];
    if (t >= n_free) {
      record_error(ws, PBSA_ERR_INVALID_ARG, j, K_MU_SELECT);
      continue;
    }
    const int dst = flist[t];
    copy_src[t] = eslot[j];
    copy_dst[t] = dst;
    filled[dst] = 1;
    slot_gid[(size_t)h * C + dst] = gid[j];
    slot_ema[(size_t)h * C + dst] = ema[j];
  }
  if (tid == 0) *ncopy_h = min(n_promo, n_free);
  __syncthreads();
  // kept persistent entries take their new EMA; slots neither kept nor refilled are cleared
  for (int j = tid; j < C; j += NT) {
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

template <int D>
__global__ void __launch_bounds__(MU_THREADS) mu_score_select_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    int* __restrict__ slot_gid, float* __restrict__ slot_ema, int C, int n_sink_gid,
    const int* __restrict__ cand_slot, const int* __restrict__ cand_gid, int ncand, float gamma,
    float scale, float* __restrict__ part, int* __restrict__ copy_list, int* __restrict__ ncopy,
    int* __restrict__ count, int* __restrict__ p_list, int* __restrict__ p_cnt, void* ws) {
  constexpr int PL = D / 32;          // elements of a row per lane
  constexpr int NW = MU_THREADS / 32;
  using V = typename MuVec<PL>::type;
  extern __shared__ float smem[];
  const int h = blockIdx.y, r0 = blockIdx.x * MU_RQ, nb = C + ncand;
  const int nr = min(MU_RQ, nq - r0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* gid = reinterpret_cast<int*>(smem);          // [nb]
  int* eslot = gid + nb;                             // [nb]
  float* qs = reinterpret_cast<float*>(eslot + nb);  // [MU_RQ][D]
  float* sc = qs + MU_RQ * D;                        // [MU_RQ][nb] scores, then p
  __shared__ int last_s;

  for (int j = tid; j < nb; j += MU_THREADS) {
    int sl;
    gid[j] = entry_of(j, h, C, ncand, pool_slots, slot_gid, cand_slot, cand_gid, &sl, ws, blockIdx.x == 0);
    eslot[j] = sl;
  }
  for (int i = tid; i < MU_RQ * D; i += MU_THREADS) {
    const int r = i / D;
    qs[i] = r < nr ? q_reps[((size_t)h * nq + r0 + r) * D + (i - r * D)] : 0.f;
  }
  __syncthreads();

  // ---- scores: warp per pool entry, lanes over d, MU_BATCH entries in flight
  float ql[MU_RQ][PL];
#pragma unroll
  for (int r = 0; r < MU_RQ; ++r)
#pragma unroll
    for (int i = 0; i < PL; ++i) ql[r][i] = qs[r * D + lane * PL + i];
  for (int j0 = warp; j0 < nb; j0 += NW * MU_BATCH) {
    float kv[MU_BATCH][PL];
#pragma unroll
    for (int b = 0; b < MU_BATCH; ++b) {
      const int j = j0 + b * NW;
      if (j < nb && gid[j] >= 0) {
        const V w = __ldg(reinterpret_cast<const V*>(k_reps + ((size_t)h * pool_slots + eslot[j]) * D) + lane);
        mu_vec_to(w, kv[b]);
      } else {
#pragma unroll
        for (int i = 0; i < PL; ++i) kv[b][i] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < MU_BATCH; ++b) {
      const int j = j0 + b * NW;
      float a[MU_RQ];
#pragma unroll
      for (int r = 0; r < MU_RQ; ++r) {
        a[r] = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) a[r] = fmaf(ql[r][i], kv[b][i], a[r]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < MU_RQ; ++r) a[r] += __shfl_xor_sync(0xffffffffu, a[r], o);
      if (lane == 0 && j < nb) {
        const bool ok = gid[j] >= 0;
#pragma unroll
        for (int r = 0; r < MU_RQ; ++r) sc[r * nb + j] = ok ? a[r] * scale : -INFINITY;
      }
    }
  }
  __syncthreads();
  // ---- softmax of each row over the pool (one warp per row, fixed-order reductions)
  for (int r = warp; r < nr; r += NW) {
    float* row = sc + r * nb;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) sum += row[j] == -INFINITY ? 0.f : expf(row[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.0f / sum : 0.f;
    __syncwarp();
    for (int j = lane; j < nb; j += 32) row[j] = row[j] == -INFINITY ? 0.f : expf(row[j] - m) * inv;
  }
  __syncthreads();
  // ---- column sums of this CTA's rows (row order), then count this CTA as done
  float* my_part = part + ((size_t)h * gridDim.x + blockIdx.x) * nb;
  for (int j = tid; j < nb; j += MU_THREADS) {
    float a = 0.f;
    for (int r = 0; r < nr; ++r) a += sc[r * nb + j];
    my_part[j] = a;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last_s = atomicAdd(&count[h], 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  // ---- the last CTA of head h: a_b = mean over all rows, summed over the partials in order
  float* ema = sc;                                    // [nb]
  uint64_t* key = reinterpret_cast<uint64_t*>(sc + 2 * ((nb + 1) / 2) + 2);  // [nb], 8-byte aligned
  int* rank = reinterpret_cast<int*>(key + nb);       // [nb]
  int* by_rank = rank + nb;                           // [nb]
  int* filled = by_rank + nb;                         // [nb]
  int* flist = filled + nb;                           // [nb] freed persistent slots, ascending
  int* plist2 = flist + nb;                           // [nb] promoted entries, in promotion order
  const float* hpart = part + (size_t)h * gridDim.x * nb;
  const float inv_nq = 1.0f / (float)nq;
  const int nparts = (int)gridDim.x;
  for (int j = tid; j < nb; j += MU_THREADS) {
    float a = 0.f;
    for (int b0 = 0; b0 < nparts; b0 += 8) {   // eight loads in flight, summed in order
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = b0 + u < nparts ? __ldcg(hpart + (size_t)(b0 + u) * nb + j) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) a += v[u];
    }
    ema[j] = a * inv_nq;
  }
  mu_select_head(h, nb, pool_slots, slot_gid, slot_ema, slot_ema + (size_t)h * C, C, n_sink_gid, gamma, gid,
                 eslot, ema, key, rank, by_rank, filled, flist, plist2, copy_list + (size_t)h * nb * 2, copy_list + (size_t)h * nb * 2 + nb,
                 ncopy + h, p_list, p_cnt, ws);
  if (tid == 0) count[h] = 0;   // ready for the next call
}

template <typename T, int D>
__global__ void __launch_bounds__(MU_THREADS) mu_copy_kernel(
    const int* __restrict__ copy_list, const int* __restrict__ ncopy, int nb, int C, float* k_reps,
    T* k_pool, T* v_pool, int pool_slots, void* ws) {
  const int t = blockIdx.x, h = blockIdx.y, which = blockIdx.z;
  if (t >= ncopy[h]) return;
  const int src = copy_list[(size_t)h * nb * 2 + t];
  const int dst = copy_list[(size_t)h * nb * 2 + nb + t];
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

// ---------------------------------------------------------------------------- one-launch form
// Up to MF_MAX_NB pool entries and MF_NC * MF_MAX_R query blocks: one cluster of MF_NC CTAs
// per head does the whole update.
//  0. the K and V blocks of every candidate (each may be promoted) are prefetched into L2, so
//     their HBM reads overlap the scoring and ranking below;
//  1. CTA c copies the pool representatives into shared memory (cp.async, rows padded to
//     d + 4 floats) -- a persistent entry's slot is its index, so those rows are requested
//     before the candidate lists arrive -- and its query rows [c R, c R + R);
//  2. scores S = Q K^T for its rows (<= 16) and all entries on the tensor cores: m16n8k8
//     TF32 MMAs with each fp32 operand split into a TF32 high part and a TF32 residual
//     (hi*hi + hi*lo + lo*hi, fp32 accumulation: fp32-level accuracy);
//  3. softmax over the pool, one warp per row; thread j then sums p over the CTA's rows
//     (row order);
//  4. rank 0 adds the CTAs' column sums in rank order over distributed shared memory
//     (a_b = mean over all rows), applies the EMA, ranks and assigns slots (mu_select_head),
//     leaving the copy list in its shared memory;
//  5. every CTA takes copies t = c, c + MF_NC, ...: K and V blocks go through a ring of
//     shared-memory stages (one bulk load and one bulk store of a whole block each), the
//     k_reps row through plain loads and stores.
// The workspace holds only the error word.
constexpr int MF_NC = 8;
constexpr int MF_THREADS = 512;
constexpr int MF_MAX_NB = 256;     // pool entries
constexpr int MF_MAX_R = 16;       // query rows per CTA: one m16 tile
constexpr int MF_MAX_STAGES = 8;
constexpr int MF_MAX_MINE = MF_MAX_NB / MF_NC;   // copies per CTA (ncopy <= nb)
constexpr int MF_SCS = MF_MAX_NB + 8;            // score row stride (floats)

template <typename T, int D>
struct MfLayout {
  static constexpr int KS = D + 4;                        // padded representative row (floats)
  static constexpr int TILE = BT * D * (int)sizeof(T);    // one K or V block
  static constexpr int KB_BYTES = MF_MAX_NB * KS * 4;
  static constexpr int REGION = KB_BYTES > 4 * TILE ? KB_BYTES : 4 * TILE;   // reps, later copy stages
  static constexpr int STAGES = REGION / TILE < MF_MAX_STAGES ? REGION / TILE : MF_MAX_STAGES;
  static constexpr int OFF_Q = REGION;                             // float [MF_MAX_R][KS]
  static constexpr int OFF_S = OFF_Q + MF_MAX_R * KS * 4;           // float [MF_MAX_R][MF_SCS] scores, then p
  static constexpr int OFF_GID = OFF_S + MF_MAX_R * MF_SCS * 4;     // int [MF_MAX_NB]
  static constexpr int OFF_ESLOT = OFF_GID + MF_MAX_NB * 4;         // int [MF_MAX_NB]
  static constexpr int OFF_COL = OFF_ESLOT + MF_MAX_NB * 4;         // float [MF_MAX_NB] (read by rank 0)
  static constexpr int OFF_PREV = OFF_COL + MF_MAX_NB * 4;          // float [MF_MAX_NB] rank 0: old slot_ema
  static constexpr int OFF_SEL = OFF_PREV + MF_MAX_NB * 4;          // rank 0: ema, key (8 B), 5 int arrays
  static constexpr int OFF_CPY = OFF_SEL + MF_MAX_NB * (4 + 8 + 5 * 4);   // int src, dst [MF_MAX_NB], count
  static constexpr int OFF_MY = OFF_CPY + 2 * MF_MAX_NB * 4 + 16;         // int src, dst [MF_MAX_MINE], count
  static constexpr int OFF_BAR = OFF_MY + 2 * MF_MAX_MINE * 4 + 16;       // mbarriers [STAGES]
  static constexpr int BYTES = OFF_BAR + MF_MAX_STAGES * 8 + 128;         // + alignment slack
  static_assert(OFF_SEL % 16 == 0 && OFF_BAR % 8 == 0 && OFF_Q % 16 == 0, "layout alignment");
};

template <typename T, int D>
__global__ void __cluster_dims__(MF_NC, 1, 1) __launch_bounds__(MF_THREADS, 1) mu_cluster_kernel(
    const float* __restrict__ q_reps, int nq, float* k_reps, T* k_pool, T* v_pool, int pool_slots,
    int* __restrict__ slot_gid, float* __restrict__ slot_ema, int C, int n_sink_gid,
    const int* __restrict__ cand_slot, const int* __restrict__ cand_gid, int ncand, float gamma,
    float scale, int R, int* __restrict__ p_list, int* __restrict__ p_cnt, void* ws) {
  using L = MfLayout<T, D>;
  constexpr int KS = L::KS, CH = D / 4;   // 16-byte chunks per row
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t mf_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mf_raw) + 127) & ~(uintptr_t)127);
  float* kb = reinterpret_cast<float*>(sm);
  float* qs = reinterpret_cast<float*>(sm + L::OFF_Q);
  float* ss = reinterpret_cast<float*>(sm + L::OFF_S);
  int* gid = reinterpret_cast<int*>(sm + L::OFF_GID);
  int* eslot = reinterpret_cast<int*>(sm + L::OFF_ESLOT);
  float* col = reinterpret_cast<float*>(sm + L::OFF_COL);
  float* prev = reinterpret_cast<float*>(sm + L::OFF_PREV);
  int* my_src = reinterpret_cast<int*>(sm + L::OFF_MY);
  int* my_dst = my_src + MF_MAX_MINE;
  int* my_n = my_dst + MF_MAX_MINE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);

  const int c = (int)cluster.block_rank();
  const int h = blockIdx.y, nb = C + ncand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = c * R, nr = max(0, min(R, nq - r0));
  const float* krep_h = k_reps + (size_t)h * pool_slots * D;

  // ---- 0 + 1. prefetch candidates' blocks; entries, query rows and representatives
  for (int t = tid; t < ncand; t += MF_THREADS) {
    if (t % MF_NC != c) continue;    // CTA c prefetches candidates c, c + MF_NC, ...
    const int sl = cand_slot[(size_t)h * ncand + t];
    if (sl >= C && sl < pool_slots) {
      prefetch_l2(k_pool + ((size_t)h * pool_slots + sl) * BT * D, L::TILE);
      prefetch_l2(v_pool + ((size_t)h * pool_slots + sl) * BT * D, L::TILE);
    }
  }
  for (int i = tid; i < C * CH; i += MF_THREADS) {   // persistent rows: slot = entry index
    const int j = i / CH, e = i - j * CH;
    cp_async16(kb + j * KS + 4 * e, krep_h + (size_t)j * D + 4 * e);
  }
  for (int i = tid; i < MF_MAX_R * CH; i += MF_THREADS) {
    const int r = i / CH, e = i - r * CH;
    if (r < nr) cp_async16(qs + r * KS + 4 * e, q_reps + ((size_t)h * nq + r0 + r) * D + 4 * e);
    else reinterpret_cast<float4*>(qs + r * KS)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid < MF_MAX_NB) {
    int sl = 0;
    gid[tid] = tid < nb ? entry_of(tid, h, C, ncand, pool_slots, slot_gid, cand_slot, cand_gid, &sl, ws, c == 0) : -1;
    eslot[tid] = sl;
    if (c == 0 && tid < C) prev[tid] = slot_ema[(size_t)h * C + tid];
  }
  __syncthreads();
  for (int i = tid; i < ncand * CH; i += MF_THREADS) {   // candidate rows
    const int j = C + i / CH, e = i % CH;
    if (gid[j] >= 0) cp_async16(kb + j * KS + 4 * e, krep_h + (size_t)eslot[j] * D + 4 * e);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- 2. S = Q K^T (3xTF32 MMAs): warp w takes the 8-entry tiles w, w + 16, ...
  {
    const int g = lane >> 2, t4 = lane & 3;
    const int ntiles = (nb + 7) / 8;
    for (int nt = warp; nt < ntiles; nt += MF_THREADS / 32) {
      // six independent accumulation chains (the three products x even/odd k-steps), added
      // in a fixed order at the end
      float acc[6][4] = {};
      const float* brow = kb + (nt * 8 + g) * KS;   // entry nt*8 + g (rows past nb: unused results)
#pragma unroll
      for (int k0 = 0; k0 < D; k0 += 8) {
        const int par = (k0 >> 3) & 1;
        uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
        tf32_split(qs[g * KS + k0 + t4], ah[0], al[0]);
        tf32_split(qs[(g + 8) * KS + k0 + t4], ah[1], al[1]);
        tf32_split(qs[g * KS + k0 + t4 + 4], ah[2], al[2]);
        tf32_split(qs[(g + 8) * KS + k0 + t4 + 4], ah[3], al[3]);
        tf32_split(brow[k0 + t4], bh0, bl0);
        tf32_split(brow[k0 + t4 + 4], bh1, bl1);
        mma_tf32(acc[3 * par + 0], al, bh0, bh1);
        mma_tf32(acc[3 * par + 1], ah, bl0, bl1);
        mma_tf32(acc[3 * par + 2], ah, bh0, bh1);
      }
      float r4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        r4[e] = ((acc[0][e] + acc[3][e]) + (acc[1][e] + acc[4][e])) + (acc[2][e] + acc[5][e]);
      *reinterpret_cast<float2*>(ss + g * MF_SCS + nt * 8 + 2 * t4) = make_float2(r4[0], r4[1]);
      *reinterpret_cast<float2*>(ss + (g + 8) * MF_SCS + nt * 8 + 2 * t4) = make_float2(r4[2], r4[3]);
    }
  }
  __syncthreads();

  // ---- 3. softmax over the pool, warp r per row; then column sums in row order
  for (int r = warp; r < nr; r += MF_THREADS / 32) {
    float* row = ss + r * MF_SCS;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, gid[j] >= 0 ? row[j] * scale : -INFINITY);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) sum += gid[j] >= 0 ? expf(row[j] * scale - m) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.0f / sum : 0.f;
    for (int j = lane; j < nb; j += 32) row[j] = gid[j] >= 0 ? expf(row[j] * scale - m) * inv : 0.f;
  }
  __syncthreads();
  if (tid < MF_MAX_NB) {
    float a = 0.f;
    if (tid < nb)
      for (int r = 0; r < nr; ++r) a += ss[r * MF_SCS + tid];
    col[tid] = a;
  }
  cluster.sync();   // every CTA's column sums are in

  // ---- 4. rank 0: a_b over all rows (CTAs in rank order), EMA, ranking, slot assignment
  int* csrc = reinterpret_cast<int*>(sm + L::OFF_CPY);
  int* cdst = csrc + MF_MAX_NB;
  if (c == 0) {
    float* ema = reinterpret_cast<float*>(sm + L::OFF_SEL);
    uint64_t* key = reinterpret_cast<uint64_t*>(ema + MF_MAX_NB);
    int* rank = reinterpret_cast<int*>(key + MF_MAX_NB);
    int* by_rank = rank + MF_MAX_NB;
    int* filled = by_rank + MF_MAX_NB;
    int* flist = filled + MF_MAX_NB;
    int* plist2 = flist + MF_MAX_NB;
    if (tid < nb) {
      float part[MF_NC];
#pragma unroll
      for (int c2 = 0; c2 < MF_NC; ++c2) part[c2] = cluster.map_shared_rank(col, c2)[tid];
      float a = 0.f;
#pragma unroll
      for (int c2 = 0; c2 < MF_NC; ++c2) a += part[c2];
      ema[tid] = a * (1.0f / (float)nq);
    }
    __syncthreads();
    mu_select_head(h, nb, pool_slots, slot_gid, slot_ema, prev, C, n_sink_gid, gamma, gid, eslot, ema, key, rank,
                   by_rank, filled, flist, plist2, csrc, cdst, cdst + MF_MAX_NB, p_list, p_cnt, ws);
  }
  cluster.sync();   // the copy list is in rank 0's shared memory
  {
    const int* rsrc = cluster.map_shared_rank(csrc, 0);
    const int n_all = rsrc[2 * MF_MAX_NB];
    const int mine = n_all > c ? (n_all - 1 - c) / MF_NC + 1 : 0;
    if (tid < mine) {
      my_src[tid] = rsrc[c + tid * MF_NC];
      my_dst[tid] = rsrc[MF_MAX_NB + c + tid * MF_NC];
    }
    if (tid == 0) *my_n = mine;
  }
  cluster.sync();   // every CTA holds its share; no shared memory is read remotely after this

  // ---- 5. this CTA's copies: tile 2t = K block of copy t, 2t + 1 = its V block
  const int mine = *my_n;
  auto copy_ok = [&](int t) { return my_src[t] >= C && my_src[t] < pool_slots && my_dst[t] >= 0 && my_dst[t] < C; };
  if (tid == 0 && mine > 0) {
    const int ntiles = 2 * mine;
    for (int s2 = 0; s2 < L::STAGES; ++s2) mbar_init(&bars[s2], 1);
    fence_barrier_init();
    fence_proxy_async_smem();   // the stages held representatives written through the generic proxy
    auto tile_at = [&](int i, bool dst) -> T* {
      const int t = i >> 1;
      T* pool = (i & 1) ? v_pool : k_pool;
      return pool + ((size_t)h * pool_slots + (dst ? my_dst[t] : my_src[t])) * BT * D;
    };
    auto load = [&](int i) {
      uint64_t* bar = &bars[i % L::STAGES];
      if (copy_ok(i >> 1)) {
        mbar_arrive_expect_tx(bar, L::TILE);
        bulk_load(sm + (i % L::STAGES) * L::TILE, tile_at(i, false), L::TILE, bar);
      } else {
        mbar_arrive(bar);
      }
    };
    int issued = 0;
    for (; issued < ntiles && issued < L::STAGES; ++issued) load(issued);
    for (int i = 0; i < ntiles; ++i) {
      if (!mbar_wait(&bars[i % L::STAGES], (i / L::STAGES) & 1, kWaitLimitNs)) {
        record_error(ws, PBSA_ERR_TIMEOUT, i, K_MU_COPY);
        for (int j = i + 1; j < issued; ++j) mbar_wait(&bars[j % L::STAGES], (j / L::STAGES) & 1, kWaitLimitNs);
        break;
      }
      if (copy_ok(i >> 1)) bulk_store(tile_at(i, true), sm + (i % L::STAGES) * L::TILE, L::TILE);
      bulk_commit();
      // refill the stage of tile i - 1, whose store is the second newest bulk group
      if (i >= 1 && issued < ntiles) {
        bulk_wait_read<1>();
        load(issued++);
      }
    }
    bulk_wait_all();
  } else if (tid >= 32) {
    // k_reps rows of the promoted blocks (the other warps)
    for (int e = tid - 32; e < mine * CH; e += MF_THREADS - 32) {
      const int t = e / CH, i = e - t * CH;
      if (!copy_ok(t)) continue;
      reinterpret_cast<float4*>(k_reps + ((size_t)h * pool_slots + my_dst[t]) * D)[i] =
          reinterpret_cast<const float4*>(k_reps + ((size_t)h * pool_slots + my_src[t]) * D)[i];
    }
  }
  if (tid < mine && !copy_ok(tid)) record_error(ws, PBSA_ERR_DEVICE_INDEX, my_src[tid], K_MU_COPY);
}

// ---------------------------------------------------------------------------- plan / apply
// The update split in two: mu_plan_kernel scores, ranks and assigns (slot table, persistent
// list, copy list in the workspace) without touching the K/V pools, so it may run while the
// attention of the same chunk still reads them; mu_copy_kernel then applies the copy list.
// One CTA per head (up to MF_MAX_NB pool entries, any number of query blocks): the pool
// representatives are staged once; query rows go through the MMA tile 16 at a time (scores by
// split-TF32 MMAs, softmax per row by one warp, column sums in row order).  Launched as a
// programmatic dependent, the grid signals its own dependents at once and waits for the grid
// it overlaps before completing.
template <int D>
__global__ void __launch_bounds__(MF_THREADS, 1) mu_plan_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    int* __restrict__ slot_gid, float* __restrict__ slot_ema, int C, int n_sink_gid,
    const int* __restrict__ cand_slot, const int* __restrict__ cand_gid, int ncand, float gamma, float scale,
    int* __restrict__ copy_list, int* __restrict__ ncopy, int* __restrict__ p_list, int* __restrict__ p_cnt,
    void* ws) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using L = MfLayout<float, D>;
  constexpr int KS = L::KS, CH = D / 4;
  extern __shared__ uint8_t mp_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mp_raw) + 127) & ~(uintptr_t)127);
  float* kb = reinterpret_cast<float*>(sm);
  float* qs = reinterpret_cast<float*>(sm + L::OFF_Q);
  float* ss = reinterpret_cast<float*>(sm + L::OFF_S);
  int* gid = reinterpret_cast<int*>(sm + L::OFF_GID);
  int* eslot = reinterpret_cast<int*>(sm + L::OFF_ESLOT);
  float* col = reinterpret_cast<float*>(sm + L::OFF_COL);
  float* prev = reinterpret_cast<float*>(sm + L::OFF_PREV);
  const int h = blockIdx.x, nb = C + ncand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* krep_h = k_reps + (size_t)h * pool_slots * D;

  // ---- entries and representatives (a persistent entry's slot is its index)
  for (int i = tid; i < C * CH; i += MF_THREADS) {
    const int j = i / CH, e = i - j * CH;
    cp_async16(kb + j * KS + 4 * e, krep_h + (size_t)j * D + 4 * e);
  }
  if (tid < MF_MAX_NB) {
    int sl = 0;
    gid[tid] = tid < nb ? entry_of(tid, h, C, ncand, pool_slots, slot_gid, cand_slot, cand_gid, &sl, ws, true) : -1;
    eslot[tid] = sl;
    col[tid] = 0.f;
    if (tid < C) prev[tid] = slot_ema[(size_t)h * C + tid];
  }
  __syncthreads();
  for (int i = tid; i < ncand * CH; i += MF_THREADS) {
    const int j = C + i / CH, e = i % CH;
    if (gid[j] >= 0) cp_async16(kb + j * KS + 4 * e, krep_h + (size_t)eslot[j] * D + 4 * e);
  }

  // ---- query rows 16 at a time: scores, softmax, column sums (rows in order)
  const int gq = lane >> 2, t4 = lane & 3;
  const int ntiles = (nb + 7) / 8;
  for (int r0 = 0; r0 < nq; r0 += MF_MAX_R) {
    const int nr = min(MF_MAX_R, nq - r0);
    for (int i = tid; i < MF_MAX_R * CH; i += MF_THREADS) {
      const int r = i / CH, e = i - r * CH;
      if (r < nr) cp_async16(qs + r * KS + 4 * e, q_reps + ((size_t)h * nq + r0 + r) * D + 4 * e);
      else reinterpret_cast<float4*>(qs + r * KS)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int nt = warp; nt < ntiles; nt += MF_THREADS / 32) {
      float acc[6][4] = {};
      const float* brow = kb + (nt * 8 + gq) * KS;
#pragma unroll
      for (int k0 = 0; k0 < D; k0 += 8) {
        const int par = (k0 >> 3) & 1;
        uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
        tf32_split(qs[gq * KS + k0 + t4], ah[0], al[0]);
        tf32_split(qs[(gq + 8) * KS + k0 + t4], ah[1], al[1]);
        tf32_split(qs[gq * KS + k0 + t4 + 4], ah[2], al[2]);
        tf32_split(qs[(gq + 8) * KS + k0 + t4 + 4], ah[3], al[3]);
        tf32_split(brow[k0 + t4], bh0, bl0);
        tf32_split(brow[k0 + t4 + 4], bh1, bl1);
        mma_tf32(acc[3 * par + 0], al, bh0, bh1);
        mma_tf32(acc[3 * par + 1], ah, bl0, bl1);
        mma_tf32(acc[3 * par + 2], ah, bh0, bh1);
      }
      float r4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        r4[e] = ((acc[0][e] + acc[3][e]) + (acc[1][e] + acc[4][e])) + (acc[2][e] + acc[5][e]);
      *reinterpret_cast<float2*>(ss + gq * MF_SCS + nt * 8 + 2 * t4) = make_float2(r4[0], r4[1]);
      *reinterpret_cast<float2*>(ss + (gq + 8) * MF_SCS + nt * 8 + 2 * t4) = make_float2(r4[2], r4[3]);
    }
    __syncthreads();
    for (int r = warp; r < nr; r += MF_THREADS / 32) {
      float* row = ss + r * MF_SCS;
      float m = -INFINITY;
      for (int j = lane; j < nb; j += 32) m = fmaxf(m, gid[j] >= 0 ? row[j] * scale : -INFINITY);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int j = lane; j < nb; j += 32) sum += gid[j] >= 0 ? expf(row[j] * scale - m) : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = sum > 0.f ? 1.0f / sum : 0.f;
      for (int j = lane; j < nb; j += 32) row[j] = gid[j] >= 0 ? expf(row[j] * scale - m) * inv : 0.f;
    }
    __syncthreads();
    if (tid < nb) {
      float a = col[tid];
      for (int r = 0; r < nr; ++r) a += ss[r * MF_SCS + tid];
      col[tid] = a;
    }
    __syncthreads();   // qs and ss are rewritten by the next tile
  }

  // ---- a_b = mean over the rows, EMA, ranking, slot assignment
  {
    float* ema = reinterpret_cast<float*>(sm + L::OFF_SEL);
    uint64_t* key = reinterpret_cast<uint64_t*>(ema + MF_MAX_NB);
    int* rank = reinterpret_cast<int*>(key + MF_MAX_NB);
    int* by_rank = rank + MF_MAX_NB;
    int* filled = by_rank + MF_MAX_NB;
    int* flist = filled + MF_MAX_NB;
    int* plist2 = flist + MF_MAX_NB;
    if (tid < nb) ema[tid] = col[tid] * (1.0f / (float)nq);
    __syncthreads();
    mu_select_head(h, nb, pool_slots, slot_gid, slot_ema, prev, C, n_sink_gid, gamma, gid, eslot, ema, key, rank,
                   by_rank, filled, flist, plist2, copy_list + (size_t)h * nb * 2,
                   copy_list + (size_t)h * nb * 2 + nb, ncopy + h, p_list, p_cnt, ws);
  }
  // a programmatic dependent of another grid completes only after it (no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D>
cudaError_t launch_plan(const Geo& g, const float* q_reps, int nq, const float* k_reps, int pool_slots,
                        int* slot_gid, float* slot_ema, int C, int n_sink_gid, const int* cand_slot,
                        const int* cand_gid, int ncand, float gamma, int* p_list, int* p_cnt, bool overlap_previous,
                        void* ws, cudaStream_t st) {
  const int nb = C + ncand;
  const MuLayout L = mu_layout(g.H, nq, nb);
  char* base = static_cast<char*>(ws);
  int* copy_list = reinterpret_cast<int*>(base + L.copy_off);
  int* ncopy = reinterpret_cast<int*>(base + L.ncopy_off);
  cudaError_t e;
  if (nb <= MF_MAX_NB) {
    auto kern = mu_plan_kernel<D>;
    constexpr int smem = MfLayout<float, D>::BYTES;
    if ((e = set_smem_once((const void*)kern, smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.H);
    cfg.blockDim = dim3(MF_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap_previous ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, q_reps, nq, k_reps, pool_slots, slot_gid, slot_ema, C, n_sink_gid,
                              cand_slot, cand_gid, ncand, gamma, g.scale, copy_list, ncopy, p_list, p_cnt, ws);
  }
  // larger pools: the score kernel of the two-launch path (an ordinary launch: it does not
  // wait for a grid it would overlap)
  float* part = reinterpret_cast<float*>(base + L.part_off);
  int* count = reinterpret_cast<int*>(base + L.count_off);
  const size_t sel = (size_t)14 * nb * 4 + 16, sco = (size_t)MU_RQ * nb * 4;
  const size_t smem = (size_t)2 * nb * 4 + (size_t)MU_RQ * D * 4 + (sel > sco ? sel : sco);
  if ((e = set_smem_once((const void*)mu_score_select_kernel<D>, (int)smem)) != cudaSuccess) return e;
  mu_score_select_kernel<D><<<dim3((nq + MU_RQ - 1) / MU_RQ, g.H), MU_THREADS, smem, st>>>(
      const_cast<float*>(q_reps), nq, const_cast<float*>(k_reps), pool_slots, slot_gid, slot_ema, C, n_sink_gid,
      cand_slot, cand_gid, ncand, gamma, g.scale, part, copy_list, ncopy, count, p_list, p_cnt, ws);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_apply(const Geo& g, float* k_reps, void* k_pool, void* v_pool, int pool_slots, int C, int ncand,
                         void* ws, cudaStream_t st) {
  const int nb = C + ncand;
  const MuLayout L = mu_layout(g.H, 1, nb);
  char* base = static_cast<char*>(ws);
  const int* copy_list = reinterpret_cast<const int*>(base + L.copy_off);
  const int* ncopy = reinterpret_cast<const int*>(base + L.ncopy_off);
  const int max_copies = C < nb ? C : nb;
  if (max_copies <= 0) return cudaSuccess;
  dim3 grid(max_copies, g.H, 2);
  if (g.dtype == PBSA_BF16)
    mu_copy_kernel<__nv_bfloat16, D><<<grid, MU_THREADS, 0, st>>>(copy_list, ncopy, nb, C, k_reps,
                                                                  static_cast<__nv_bfloat16*>(k_pool),
                                                                  static_cast<__nv_bfloat16*>(v_pool), pool_slots, ws);
  else
    mu_copy_kernel<float, D><<<grid, MU_THREADS, 0, st>>>(copy_list, ncopy, nb, C, k_reps,
                                                          static_cast<float*>(k_pool), static_cast<float*>(v_pool),
                                                          pool_slots, ws);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_mu(const Geo& g, const float* q_reps, int nq, float* k_reps, void* k_pool,
                      void* v_pool, int pool_slots, int* slot_gid, float* slot_ema, int C,
                      int n_sink_gid, const int* cand_slot, const int* cand_gid, int ncand,
                      float gamma, int* p_list, int* p_cnt, void* ws, cudaStream_t st) {
  const int nb = C + ncand;
  const int R = (nq + MF_NC - 1) / MF_NC;
  if (nb <= MF_MAX_NB && R <= MF_MAX_R) {
    cudaError_t e;
#define PBSA_MF(TT)                                                                                        \
    {                                                                                                      \
      auto kern = mu_cluster_kernel<TT, D>;                                                                \
      if ((e = set_smem_once((const void*)kern, MfLayout<TT, D>::BYTES)) != cudaSuccess) return e;         \
      kern<<<dim3(MF_NC, g.H), MF_THREADS, MfLayout<TT, D>::BYTES, st>>>(                                  \
          q_reps, nq, k_reps, static_cast<TT*>(k_pool), static_cast<TT*>(v_pool), pool_slots, slot_gid,     \
          slot_ema, C, n_sink_gid, cand_slot, cand_gid, ncand, gamma, g.scale, R, p_list, p_cnt, ws);      \
    }
    if (g.dtype == PBSA_BF16) PBSA_MF(__nv_bfloat16) else PBSA_MF(float)
#undef PBSA_MF
    return cudaGetLastError();
  }
  const MuLayout L = mu_layout(g.H, nq, nb);
  char* base = static_cast<char*>(ws);
  float* part = reinterpret_cast<float*>(base + L.part_off);
  int* copy_list = reinterpret_cast<int*>(base + L.copy_off);
  int* ncopy = reinterpret_cast<int*>(base + L.ncopy_off);
  int* count = reinterpret_cast<int*>(base + L.count_off);
  cudaError_t e;

  // smem: gid, eslot [nb] + q rows [MU_RQ][D] + max(scores [MU_RQ][nb], select arrays: 6 x 4
  // bytes + 8-byte keys per entry, plus alignment)
  const size_t sel = (size_t)14 * nb * 4 + 16, sco = (size_t)MU_RQ * nb * 4;
  const size_t smem = (size_t)2 * nb * 4 + (size_t)MU_RQ * D * 4 + (sel > sco ? sel : sco);
  if ((e = set_smem_once((const void*)mu_score_select_kernel<D>, (int)smem)) != cudaSuccess) return e;
  mu_score_select_kernel<D><<<dim3((nq + MU_RQ - 1) / MU_RQ, g.H), MU_THREADS, smem, st>>>(
      q_reps, nq, k_reps, pool_slots, slot_gid, slot_ema, C, n_sink_gid, cand_slot, cand_gid, ncand,
      gamma, g.scale, part, copy_list, ncopy, count, p_list, p_cnt, ws);
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

namespace pbsa {

cudaError_t launch_memory_update_plan(const Geo& g, const float* q_reps, int nq, const float* k_reps,
                                      int pool_slots, int* slot_gid, float* slot_ema, int C, int n_sink_gid,
                                      const int* cand_slot, const int* cand_gid, int ncand, float gamma,
                                      int* p_list, int* p_cnt, bool overlap_previous, void* ws, cudaStream_t st) {
#define PBSA_MP(DD)                                                                                          \
  return launch_plan<DD>(g, q_reps, nq, k_reps, pool_slots, slot_gid, slot_ema, C, n_sink_gid, cand_slot,   \
                         cand_gid, ncand, gamma, p_list, p_cnt, overlap_previous, ws, st);
  if (g.d == 128) { PBSA_MP(128) }
  if (g.d == 64) { PBSA_MP(64) }
  if (g.d == 32) { PBSA_MP(32) }
#undef PBSA_MP
  return cudaErrorNotSupported;
}

cudaError_t launch_memory_update_apply(const Geo& g, float* k_reps, void* k_pool, void* v_pool, int pool_slots,
                                       int C, int ncand, void* ws, cudaStream_t st) {
  if (g.d == 128) return launch_apply<128>(g, k_reps, k_pool, v_pool, pool_slots, C, ncand, ws, st);
  if (g.d == 64) return launch_apply<64>(g, k_reps, k_pool, v_pool, pool_slots, C, ncand, ws, st);
  if (g.d == 32) return launch_apply<32>(g, k_reps, k_pool, v_pool, pool_slots, C, ncand, ws, st);
  return cudaErrorNotSupported;
}

}  // namespace pbsa
