// a3 (fp32) -- block-sparse fine attention in exact fp32 on the SIMT cores.
//
// Sparse Forcing (gist.science, English 2.C "Global Access" + "Local Sparsity"; Chinese
// 2.2 "掩码机制"): each query block attends, in one softmax, to the persistent blocks plus
// its selected local blocks.  This is the fp32 path (tensor cores have no exact fp32
// mode); the bf16 path runs on tcgen05 (attend_tc.cu).
//
// One CTA per (query block, head), 256 threads: thread (row, quarter) scores 16 keys of
// each 64-key block against its row, the row's 4 threads combine max/sum with shuffles
// (online softmax in fixed order), and then accumulate d/4 interleaved output columns.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

template <int D>
__global__ void __launch_bounds__(256) attend_f32_kernel(
    const float* __restrict__ q, Geo g, const float* __restrict__ k_pool,
    const float* __restrict__ v_pool, int pool_slots, const int* __restrict__ kv_slot,
    const int* __restrict__ kv_cnt, int kv_ld, int nq, float* __restrict__ o,
    float* __restrict__ lse, void* ws) {
  constexpr int DP = D + 1;  // padded row stride (bank-conflict free)
  extern __shared__ float sm[];
  float* Qs = sm;             // [64][DP]
  float* Ks = Qs + BT * DP;   // [64][DP]
  float* Vs = Ks + BT * DP;   // [64][DP]
  float* Ps = Vs + BT * DP;   // [64][65]

  const int r = blockIdx.x, h = blockIdx.y;
  const int row = threadIdx.x >> 2, quarter = threadIdx.x & 3;
  const int f = r / g.bpf, rem = r - f * g.bpf;
  const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
  auto token_of = [&](int rr) -> size_t {
    const int ly = rr / g.tw, lx = rr - ly * g.tw;
    return (size_t)f * g.tpf + (size_t)(ty * g.th + ly) * g.fw + tx * g.tw + lx;
  };
  for (int i = threadIdx.x; i < BT * D; i += 256) {
    const int rr = i / D, e = i - rr * D;
    Qs[rr * DP + e] = q[(token_of(rr) * g.H + h) * D + e];
  }

  float m = -INFINITY, l = 0.f;
  float acc[D / 4];
#pragma unroll
  for (int i = 0; i < D / 4; ++i) acc[i] = 0.f;

  int cnt = kv_cnt[(size_t)h * nq + r];
  if (cnt > kv_ld || cnt < 0) {
    if (threadIdx.x == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, cnt, K_ATTEND_F32);
    cnt = cnt < 0 ? 0 : kv_ld;
  }
  const int* list = kv_slot + ((size_t)h * nq + r) * kv_ld;
  for (int jb = 0; jb < cnt; ++jb) {
    const int slot = list[jb];
    if (slot < 0 || slot >= pool_slots) {
      if (threadIdx.x == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, slot, K_ATTEND_F32);
      continue;
    }
    __syncthreads();  // previous block's K/V/P fully consumed
    const float* kb = k_pool + ((size_t)h * pool_slots + slot) * BT * D;
    const float* vb = v_pool + ((size_t)h * pool_slots + slot) * BT * D;
    for (int i = threadIdx.x; i < BT * D / 4; i += 256) {
      const float4 kv = reinterpret_cast<const float4*>(kb)[i];
      const float4 vv = reinterpret_cast<const float4*>(vb)[i];
      const int rr = (i * 4) / D, e = (i * 4) - rr * D;
      float* kd = Ks + rr * DP + e;
      float* vd = Vs + rr * DP + e;
      kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
      vd[0] = vv.x; vd[1] = vv.y; vd[2] = vv.z; vd[3] = vv.w;
    }
    __syncthreads();
    float s[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = 0.f;
    for (int e = 0; e < D; ++e) {
      const float qv = Qs[row * DP + e];
#pragma unroll
      for (int i = 0; i < 16; ++i) s[i] = fmaf(qv, Ks[(quarter * 16 + i) * DP + e], s[i]);
    }
    float mb = -INFINITY;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      s[i] *= g.scale;
      mb = fmaxf(mb, s[i]);
    }
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const float mn = fmaxf(m, mb);
    const float corr = expf(m - mn);  // m = -inf on the first block -> 0
    float ps = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p = expf(s[i] - mn);
      Ps[row * 65 + quarter * 16 + i] = p;
      ps += p;
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l = l * corr + ps;
    m = mn;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < D / 4; ++i) acc[i] *= corr;
    for (int j = 0; j < BT; ++j) {
      const float p = Ps[row * 65 + j];
#pragma unroll
      for (int i = 0; i < D / 4; ++i) acc[i] = fmaf(p, Vs[j * DP + quarter + 4 * i], acc[i]);
    }
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const size_t t = token_of(row);
  float* od = o + (t * g.H + h) * D;
#pragma unroll
  for (int i = 0; i < D / 4; ++i) od[quarter + 4 * i] = acc[i] * inv;
  if (lse != nullptr && quarter == 0) {
    const size_t Tq = (size_t)nq / g.bpf * g.tpf;
    lse[(size_t)h * Tq + t] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attend_f32(const Geo& g, const float* q, int q_frames, const float* k_pool,
                              const float* v_pool, int pool_slots, const int* kv_slot,
                              const int* kv_cnt, int kv_ld, float* o, float* lse, void* ws,
                              cudaStream_t st) {
  const int nq = q_frames * g.bpf;
#define PBSA_AF(DD)                                                                             \
  {                                                                                             \
    const size_t smem = (size_t)(3 * BT * (DD + 1) + BT * 65) * sizeof(float);                  \
    cudaError_t e = set_smem_once((const void*)attend_f32_kernel<DD>, (int)smem);               \
    if (e != cudaSuccess) return e;                                                             \
    attend_f32_kernel<DD><<<dim3(nq, g.H), 256, smem, st>>>(q, g, k_pool, v_pool, pool_slots,   \
                                                            kv_slot, kv_cnt, kv_ld, nq, o, lse, ws); \
    return cudaGetLastError();                                                                  \
  }
  if (g.d == 128) PBSA_AF(128)
  if (g.d == 64) PBSA_AF(64)
  if (g.d == 32) PBSA_AF(32)
#undef PBSA_AF
  return cudaErrorNotSupported;
}

}  // namespace pbsa
