// a2 -- coarse block scores + top-k local selection.
//
// Sparse Forcing (gist.science, English 2.C "Local Sparsity"): a lightweight coarse
// routing step scores each query block against the compressed representatives of the
// local-window blocks and keeps the top-K.  Here score = scale * <qbar, kbar> in fp32,
// and the k best are ranked by (score desc, block id asc, candidate position asc).
//
// One CTA per (head, 4 query blocks).  Each warp scores candidates against the 4 query
// representatives (one coalesced 512-byte read of kbar per candidate, butterfly
// reduction in a fixed order -> deterministic scores).  Selection is by rank counting:
// every (query, candidate) pair counts the candidates that beat it; ranks below k are
// written straight to their output position, so the output is sorted and exact.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int R = 4;  // query blocks per CTA

template <int D>
__global__ void __launch_bounds__(256) score_select_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    const int* __restrict__ cand_slot, const int* __restrict__ cand_gid, int ncand, int k,
    const int* __restrict__ prefix_slot, const int* __restrict__ prefix_cnt, int prefix_ld,
    int* __restrict__ out_slot, int* __restrict__ out_cnt, int out_ld, float* __restrict__ out_score,
    float scale, void* ws) {
  extern __shared__ float smem[];
  float* qs = smem;                    // [R][D]
  float* sc = qs + R * D;              // [R][ncand]
  int* gid = reinterpret_cast<int*>(sc + R * ncand);  // [ncand]
  int* slot = gid + ncand;                            // [ncand]

  const int h = blockIdx.y, r0 = blockIdx.x * R;
  const int nr = min(R, nq - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < R * D; i += 256) {
    const int r = i / D;
    qs[i] = r < nr ? q_reps[((size_t)h * nq + r0 + r) * D + (i - r * D)] : 0.f;
  }
  for (int c = threadIdx.x; c < ncand; c += 256) {
    gid[c] = cand_gid[(size_t)h * ncand + c];
    slot[c] = cand_slot[(size_t)h * ncand + c];
  }
  __syncthreads();

  for (int c = warp; c < ncand; c += 8) {
    const int s = slot[c];
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const bool ok = s >= 0 && s < pool_slots;
    if (ok) {
      const float* kr = k_reps + ((size_t)h * pool_slots + s) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const float kv = __ldg(kr + lane + 32 * i);
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = fmaf(qs[r * D + lane + 32 * i], kv, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
    }
    if (lane == 0) {
      if (!ok) record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_SCORE);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float v = acc[r] * scale;
        if (!ok || isnan(v)) v = -INFINITY;
        sc[r * ncand + c] = v;
      }
    }
  }

  int pc = prefix_cnt ? prefix_cnt[h] : 0;
  if (pc < 0 || pc > prefix_ld) {
    if (threadIdx.x == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, pc, K_SCORE);
    pc = pc < 0 ? 0 : prefix_ld;
  }
  for (int i = threadIdx.x; i < nr * pc; i += 256) {
    const int r = i / pc, j = i - r * pc;
    out_slot[((size_t)h * nq + r0 + r) * out_ld + j] = prefix_slot[(size_t)h * prefix_ld + j];
  }
  const int kk = min(k, ncand);
  if (threadIdx.x < nr) out_cnt[(size_t)h * nq + r0 + threadIdx.x] = pc + kk;
  __syncthreads();

  for (int i = threadIdx.x; i < nr * ncand; i += 256) {
    const int r = i / ncand, c = i - r * ncand;
    const float* row = sc + r * ncand;
    const float s = row[c];
    const int g = gid[c];
    int rank = 0;
    for (int c2 = 0; c2 < ncand; ++c2) {
      const float s2 = row[c2];
      const int g2 = gid[c2];
      rank += (s2 > s) || (s2 == s && (g2 < g || (g2 == g && c2 < c)));
    }
    if (rank < kk) {
      const size_t o = ((size_t)h * nq + r0 + r);
      out_slot[o * out_ld + pc + rank] = slot[c];
      if (out_score) out_score[o * k + rank] = s;
    }
  }
}

}  // namespace

cudaError_t launch_score_select(const Geo& g, const float* q_reps, int nq, const float* k_reps,
                                int pool_slots, const int* cand_slot, const int* cand_gid,
                                int ncand, int k, const int* prefix_slot, const int* prefix_cnt,
                                int prefix_ld, int* out_slot, int* out_cnt, int out_ld,
                                float* out_score, void* ws, cudaStream_t st) {
  const size_t smem = (size_t)R * g.d * 4 + (size_t)R * ncand * 4 + (size_t)ncand * 8;
  dim3 grid((nq + R - 1) / R, g.H);
#define PBSA_SS(DD)                                                                            \
  {                                                                                            \
    auto kern = score_select_kernel<DD>;                                                       \
    if (smem > 48 * 1024) {                                                                    \
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                           (int)smem);                                         \
      if (e != cudaSuccess) return e;                                                          \
    }                                                                                          \
    kern<<<grid, 256, smem, st>>>(q_reps, nq, k_reps, pool_slots, cand_slot, cand_gid, ncand,  \
                                  k, prefix_slot, prefix_cnt, prefix_ld, out_slot, out_cnt,     \
                                  out_ld, out_score, g.scale, ws);                              \
    return cudaGetLastError();                                                                 \
  }
  if (g.d == 128) PBSA_SS(128)
  if (g.d == 64) PBSA_SS(64)
  if (g.d == 32) PBSA_SS(32)
#undef PBSA_SS
  return cudaErrorNotSupported;
}

}  // namespace pbsa
