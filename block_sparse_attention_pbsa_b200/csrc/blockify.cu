// a1 -- blockify: mean-pooled block representatives + optional block-major copy.
//
// Sparse Forcing (gist.science, Chinese explainer 2.2 "blockified compression"; English
// 2.E): the latent token grid is cut into spatiotemporal blocks of 1 frame x 8x8 tokens,
// each summarised by one representative vector (the mean of its tokens), and stored
// block-contiguously so later reads are coalesced.
//
// One CTA per (block, head).  Each thread owns one 16-byte column chunk of the head's
// vector and a fixed set of the block's 64 rows; it issues all of its 16-byte loads up
// front (HBM-bound: bytes in flight matter), writes them straight to the pool slot, and
// sums its rows in fp32.  The row-group partial sums are added in a fixed order, so the
// representative is deterministic.
#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

template <typename T>
__device__ __forceinline__ void add_chunk(float* acc, const uint4& v);

template <>
__device__ __forceinline__ void add_chunk<float>(float* acc, const uint4& v) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

template <>
__device__ __forceinline__ void add_chunk<__nv_bfloat16>(float* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) blockify_kernel(const T* __restrict__ x, Geo g,
                                                      float* __restrict__ reps, int rep_slots,
                                                      const int* __restrict__ dst_slot,
                                                      T* __restrict__ pool, int pool_slots,
                                                      void* ws) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte chunk
  constexpr int CPR = D / VEC;         // chunks per row
  constexpr int RPP = 256 / CPR;       // rows per pass
  constexpr int PASSES = BT / RPP;
  __shared__ float part[RPP][D];

  const int b = blockIdx.x, h = blockIdx.y;
  const int slot = dst_slot ? __ldg(dst_slot + b) : b;
  if (slot < 0 || slot >= rep_slots || (pool != nullptr && slot >= pool_slots)) {
    if (threadIdx.x == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, slot, K_BLOCKIFY);
    return;
  }
  const int f = b / g.bpf, rem = b - f * g.bpf;
  const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
  const int c = threadIdx.x % CPR, rg = threadIdx.x / CPR;

  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int r = rg + p * RPP;
    const int ly = r / g.tw, lx = r - ly * g.tw;
    const size_t t = (size_t)f * g.tpf + (size_t)(ty * g.th + ly) * g.fw + tx * g.tw + lx;
    v[p] = __ldg(reinterpret_cast<const uint4*>(x + (t * g.H + h) * D) + c);
  }
  if (pool != nullptr) {
    T* dst = pool + ((size_t)h * pool_slots + slot) * BT * D;
#pragma unroll
    for (int p = 0; p < PASSES; ++p)
      reinterpret_cast<uint4*>(dst + (size_t)(rg + p * RPP) * D)[c] = v[p];
  }
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
#pragma unroll
  for (int p = 0; p < PASSES; ++p) add_chunk<T>(acc, v[p]);
#pragma unroll
  for (int i = 0; i < VEC; ++i) part[rg][c * VEC + i] = acc[i];
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += 256) {
    float s = 0.f;
#pragma unroll 4
    for (int q = 0; q < RPP; ++q) s += part[q][e];
    reps[((size_t)h * rep_slots + slot) * D + e] = s * (1.0f / BT);
  }
}

template <typename T, int D>
cudaError_t launch_t(const Geo& g, const void* x, int n_frames, float* reps, int rep_slots,
                     const int* dst_slot, void* pool, int pool_slots, void* ws, cudaStream_t st) {
  dim3 grid(n_frames * g.bpf, g.H);
  blockify_kernel<T, D><<<grid, 256, 0, st>>>(static_cast<const T*>(x), g, reps, rep_slots,
                                              dst_slot, static_cast<T*>(pool), pool_slots, ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_blockify(const Geo& g, const void* x, int n_frames, float* reps, int rep_slots,
                            const int* dst_slot, void* pool, int pool_slots, void* ws,
                            cudaStream_t st) {
  if (g.dtype == PBSA_BF16) {
    if (g.d == 128) return launch_t<__nv_bfloat16, 128>(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws, st);
    if (g.d == 64) return launch_t<__nv_bfloat16, 64>(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws, st);
  } else {
    if (g.d == 128) return launch_t<float, 128>(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws, st);
    if (g.d == 64) return launch_t<float, 64>(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws, st);
    if (g.d == 32) return launch_t<float, 32>(g, x, n_frames, reps, rep_slots, dst_slot, pool, pool_slots, ws, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace pbsa
