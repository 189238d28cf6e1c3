// a2 -- coarse block scores + top-k local selection.
//
// Sparse Forcing (gist.science, English 2.C "Local Sparsity"): a lightweight coarse
// routing step scores each query block against the compressed representatives of the
// local-window blocks and keeps the top-K.  Here score = scale * <qbar, kbar> in fp32,
// and the k best are ranked by (score desc, block id asc, candidate position asc).
//
// One CTA per (head, 8 query blocks), 256 threads.  The candidates' representatives are
// staged in shared memory, 128 at a time, with all threads' 16-byte loads in flight at
// once (the kernel is latency-bound: ~1 MB per call); every (query, candidate) dot
// product then runs from shared memory in a fixed order, so scores are deterministic.
// Selection is by rank counting: each (query, candidate) pair counts the candidates that
// beat it, and a rank below k is written straight to its output position.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int R = 8;        // query blocks per CTA
constexpr int CH = 128;     // candidates staged per pass
constexpr int THREADS = 256;

template <int D>
__global__ void __launch_bounds__(THREADS) score_select_kernel(
    const float* __restrict__ q_reps, int nq, const float* __restrict__ k_reps, int pool_slots,
    const int* __restrict__ cand_slot, const int* __restrict__ cand_gid, int ncand, int k,
    const int* __restrict__ prefix_slot, const int* __restrict__ prefix_cnt, int prefix_ld,
    int* __restrict__ out_slot, int* __restrict__ out_cnt, int out_ld, float* __restrict__ out_score,
    float scale, void* ws) {
  constexpr int DP = D + 1;   // padded row: conflict-free column reads
  extern __shared__ float smem[];
  float* ks = smem;                                            // [CH][DP]
  float* qs = ks + CH * DP;                                    // [R][D]
  uint64_t* key = reinterpret_cast<uint64_t*>(qs + R * D);     // [R][ncand] ranking keys
  float* sc = reinterpret_cast<float*>(key + R * ncand);       // [R][ncand] scores
  int* gid = reinterpret_cast<int*>(sc + R * ncand);           // [ncand]
  int* slot = gid + ncand;                                     // [ncand]

  const int h = blockIdx.y, r0 = blockIdx.x * R;
  const int nr = min(R, nq - r0);
  const int tid = threadIdx.x;

  for (int i = tid; i < R * D / 4; i += THREADS) {
    const int r = (i * 4) / D;
    const float4 v = r < nr ? reinterpret_cast<const float4*>(q_reps + ((size_t)h * nq + r0) * D)[i]
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(qs)[i] = v;
  }
  for (int c = tid; c < ncand; c += THREADS) {
    gid[c] = cand_gid[(size_t)h * ncand + c];
    slot[c] = cand_slot[(size_t)h * ncand + c];
  }
  __syncthreads();

  // ---- scores, CH candidates per pass: thread -> (candidate c, 4 query rows)
  for (int base = 0; base < ncand; base += CH) {
    const int nc = min(CH, ncand - base);
    stage_rows<D, DP, THREADS>(ks, nc, [&](int c) -> const float* {
      const int s = slot[base + c];
      return (s >= 0 && s < pool_slots) ? k_reps + ((size_t)h * pool_slots + s) * D : nullptr;
    });
    __syncthreads();
    for (int p = tid; p < nc * (R / 4); p += THREADS) {
      const int c = p % nc, rg = (p / nc) * 4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float* kr = ks + c * DP;
#pragma unroll 8
      for (int e = 0; e < D; ++e) {
        const float kv = kr[e];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(qs[(rg + j) * D + e], kv, acc[j]);
      }
      const int s = slot[base + c];
      const bool ok = s >= 0 && s < pool_slots;
      if (!ok && rg == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_SCORE);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = acc[j] * scale;
        if (!ok || isnan(v)) v = -INFINITY;
        sc[(rg + j) * ncand + base + c] = v;
        key[(rg + j) * ncand + base + c] = rank_key(v, gid[base + c]);
      }
    }
    __syncthreads();
  }

  // ---- prefix, counts, ranks
  int pc = prefix_cnt ? prefix_cnt[h] : 0;
  if (pc < 0 || pc > prefix_ld) {
    if (tid == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, pc, K_SCORE);
    pc = pc < 0 ? 0 : prefix_ld;
  }
  for (int i = tid; i < nr * pc; i += THREADS) {
    const int r = i / pc, j = i - r * pc;
    out_slot[((size_t)h * nq + r0 + r) * out_ld + j] = prefix_slot[(size_t)h * prefix_ld + j];
  }
  const int kk = min(k, ncand);
  if (tid < nr) out_cnt[(size_t)h * nq + r0 + tid] = pc + kk;

  // rank = #candidates with a larger key, plus equal keys at a lower position (branch-free)
  for (int i = tid; i < nr * ncand; i += THREADS) {
    const int r = i / ncand, c = i - r * ncand;
    const uint64_t* row = key + r * ncand;
    const uint64_t kc = row[c];
    int rank = 0;
#pragma unroll 8
    for (int c2 = 0; c2 < ncand; ++c2) {
      const uint64_t k2 = row[c2];
      rank += (int)(k2 > kc) | ((int)(k2 == kc) & (int)(c2 < c));
    }
    if (rank < kk) {
      const size_t o = ((size_t)h * nq + r0 + r);
      out_slot[o * out_ld + pc + rank] = slot[c];
      if (out_score) out_score[o * k + rank] = sc[r * ncand + c];
    }
  }
}

}  // namespace

cudaError_t launch_score_select(const Geo& g, const float* q_reps, int nq, const float* k_reps,
                                int pool_slots, const int* cand_slot, const int* cand_gid,
                                int ncand, int k, const int* prefix_slot, const int* prefix_cnt,
                                int prefix_ld, int* out_slot, int* out_cnt, int out_ld,
                                float* out_score, void* ws, cudaStream_t st) {
  const size_t smem = ((size_t)CH * (g.d + 1) + (size_t)R * g.d + (size_t)R * ncand) * 4 +
                      (size_t)R * ncand * 8 + (size_t)ncand * 8;
  dim3 grid((nq + R - 1) / R, g.H);
#define PBSA_SS(DD)                                                                            \
  {                                                                                            \
    auto kern = score_select_kernel<DD>;                                                       \
    cudaError_t e = set_smem_once((const void*)kern, (int)smem);                               \
    if (e != cudaSuccess) return e;                                                            \
    kern<<<grid, THREADS, smem, st>>>(q_reps, nq, k_reps, pool_slots, cand_slot, cand_gid,     \
                                      ncand, k, prefix_slot, prefix_cnt, prefix_ld, out_slot,  \
                                      out_cnt, out_ld, out_score, g.scale, ws);                \
    return cudaGetLastError();                                                                 \
  }
  if (g.d == 128) PBSA_SS(128)
  if (g.d == 64) PBSA_SS(64)
  if (g.d == 32) PBSA_SS(32)
#undef PBSA_SS
  return cudaErrorNotSupported;
}

}  // namespace pbsa
