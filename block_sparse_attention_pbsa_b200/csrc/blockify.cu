// a1 -- blockify: mean-pooled block representatives + optional block-major copy.
//
// Sparse Forcing (gist.science, Chinese explainer 2.2 "blockified compression"; English
// 2.E): the latent token grid is cut into spatiotemporal blocks of 1 frame x 8x8 tokens,
// each summarised by one representative vector (the mean of its tokens), and stored
// block-contiguously so later reads are coalesced.
//
// A unit of work is one (tensor, block, head): a 64-token tile of one head, 16 KB in bf16
// at d = 128.  The kernel is persistent: a grid of a few CTAs per SM walks the units with a
// stride, and each CTA streams its units through a ring of shared-memory stages:
//  * one thread gathers a unit's 64 token rows (strided in the [T][H][d] raster) with a
//    single 5-D TMA box into a stage, NST units ahead of the consumers, so every SM keeps
//    NST x 16 KB of reads in flight;
//  * the same thread writes the stage to the unit's pool slot with one bulk copy (the pool
//    row block is contiguous), while all threads sum the tile's rows from shared memory;
//  * thread (c, rg) sums its 16-byte column chunk c over rows rg, rg + RPP, ... in that
//    order, and the RPP row-group partial sums are then added in row-group order: a fixed
//    order, so the representative is deterministic (and the same as the fused
//    blockify + select kernel's query representative);
//  * a stage is refilled one unit later, once its bulk copy has read it and every thread is
//    past it (NST - 1 loads stay in flight while a store drains).
// K and V of a chunk go through one launch (two tensor maps, units of both tensors).  On request
// the launch is a programmatic dependent of the previous kernel on the stream: it may start on
// SMs that kernel leaves idle and waits for it (griddepcontrol.wait) before completing.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int BY_THREADS = 256;
constexpr int BY_STAGES = 4;

struct BlockifyParams {
  int nz;          // tensors in this launch (1 or 2)
  int nblk, H;     // blocks of the frames given, heads
  int bpf, tpr, th, tw;
  int rep_slots, pool_slots;
  float* reps[2];  // nullable per tensor: representatives not wanted
  void* pool[2];   // nullable per tensor: no block-major copy
  const int* dst_slot;
  void* ws;
};

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
struct Tile {
  static constexpr int BYTES = BT * D * (int)sizeof(T);
  static constexpr int VEC = 16 / (int)sizeof(T);   // elements per 16-byte chunk
  static constexpr int CPR = D / VEC;               // chunks per row
  static constexpr int RPP = BY_THREADS / CPR;      // row groups
  static constexpr int PASSES = BT / RPP;           // rows per row group
  static constexpr int SMEM = BY_STAGES * BYTES + RPP * D * 4 + BY_STAGES * 8 + 16 + 128;
};

template <typename T, int D>
__global__ void __launch_bounds__(BY_THREADS) blockify_kernel(const __grid_constant__ CUtensorMap map0,
                                                              const __grid_constant__ CUtensorMap map1,
                                                              const BlockifyParams p) {
  using TL = Tile<T, D>;
  extern __shared__ uint8_t by_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(by_raw) + 127) & ~(uintptr_t)127);
  float* part = reinterpret_cast<float*>(sm + BY_STAGES * TL::BYTES);          // [RPP][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + TL::RPP * D);          // [BY_STAGES]

  const int tid = threadIdx.x;
  const int per_z = p.nblk * p.H;
  const int U = p.nz * per_z;
  const int first = blockIdx.x, stride = gridDim.x;
  const int mine = first < U ? (U - 1 - first) / stride + 1 : 0;
  const int c = tid % TL::CPR, rg = tid / TL::CPR;

  // unit u = (z, b, h), h fastest: neighbouring CTAs read neighbouring token rows
  auto issue = [&](int i) {
    const int u = first + i * stride;
    const int z = u / per_z, rem = u - z * per_z;
    const int b = rem / p.H, h = rem - b * p.H;
    const int f = b / p.bpf, t = b - f * p.bpf;
    const int ty = t / p.tpr, tx = t - ty * p.tpr;
    uint64_t* bar = &full[i % BY_STAGES];
    mbar_arrive_expect_tx(bar, TL::BYTES);
    tma_load_5d(sm + (i % BY_STAGES) * TL::BYTES, z ? &map1 : &map0, bar, 0, h, tx * p.tw, ty * p.th, f);
  };
  if (tid == 0) {
    for (int s = 0; s < BY_STAGES; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
    tma_prefetch_desc(&map0);
    if (p.nz > 1) tma_prefetch_desc(&map1);
    for (int i = 0; i < mine && i < BY_STAGES; ++i) issue(i);
  }
  __syncthreads();

  for (int i = 0; i < mine; ++i) {
    const int s = i % BY_STAGES;
    const int u = first + i * stride;
    const int z = u / per_z, rem = u - z * per_z;
    const int b = rem / p.H, h = rem - b * p.H;
    const int slot = p.dst_slot ? __ldg(p.dst_slot + b) : b;
    float* reps = z ? p.reps[1] : p.reps[0];   // selects, not a dynamic index (no local copy of p)
    T* pool = static_cast<T*>(z ? p.pool[1] : p.pool[0]);
    const bool ok = slot >= 0 && slot < p.rep_slots && (pool == nullptr || slot < p.pool_slots);
    const bool landed = mbar_wait(&full[s], (i / BY_STAGES) & 1, kWaitLimitNs);
    if (__syncthreads_or(!landed)) {
      // a copy never arrived: record it, wait (bounded) for this CTA's other copies in
      // flight, and leave
      if (tid == 0) {
        record_error(p.ws, PBSA_ERR_TIMEOUT, u, K_BLOCKIFY);
        const int issued = i == 0 ? min(mine, BY_STAGES) : min(mine, i - 1 + BY_STAGES);
        for (int j = i + 1; j < issued; ++j)
          mbar_wait(&full[j % BY_STAGES], (j / BY_STAGES) & 1, kWaitLimitNs);
        bulk_wait_all();
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      return;
    }
    const uint8_t* tile = sm + s * TL::BYTES;
    if (tid == 0) {   // one bulk group per unit (empty when nothing is stored)
      if (ok && pool != nullptr) bulk_store(pool + ((size_t)h * p.pool_slots + slot) * BT * D, tile, TL::BYTES);
      bulk_commit();
    }
    if (!ok) {
      if (tid == 0) record_error(p.ws, PBSA_ERR_DEVICE_INDEX, slot, K_BLOCKIFY);
    } else {
      if (reps != nullptr) {
        float acc[TL::VEC];
#pragma unroll
        for (int e = 0; e < TL::VEC; ++e) acc[e] = 0.f;
#pragma unroll
        for (int q = 0; q < TL::PASSES; ++q)
          add_chunk<T>(acc, reinterpret_cast<const uint4*>(tile + (size_t)(rg + q * TL::RPP) * D * sizeof(T))[c]);
        float4* pr = reinterpret_cast<float4*>(part + rg * D + c * TL::VEC);
#pragma unroll
        for (int e = 0; e < TL::VEC / 4; ++e) pr[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
      }
    }
    __syncthreads();   // every thread is past the stage (and the partial sums are in)
    // Refill the stage of unit i - 1 (its threads finished with it an iteration ago; its bulk
    // group is the second newest, so unit i's store may still be reading its own stage).
    if (tid == 0 && i >= 1 && i - 1 + BY_STAGES < mine) {
      bulk_wait_read<1>();
      issue(i - 1 + BY_STAGES);
    }
    if (ok && reps != nullptr) {
      for (int e = tid; e < D; e += BY_THREADS) {
        float sum = 0.f;
#pragma unroll 4
        for (int q = 0; q < TL::RPP; ++q) sum += part[q * D + e];
        reps[((size_t)h * p.rep_slots + slot) * D + e] = sum * (1.0f / BT);
      }
    }
    // the next iteration's barrier orders these reads of `part` before it is rewritten
  }
  if (tid == 0) bulk_wait_all();
  // Launched as a programmatic dependent, this grid must not complete before the grid it
  // overlaps: what follows on the stream then still runs after both.  (Returns at once for an
  // ordinary launch.)
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [n_frames][fh][fw][H][d] raster as a 5-D map (d, H, fw, fh, frames); one box = one block of
// one head, rows in (ly, lx) order -- the pool's row order.
bool encode_raster(CUtensorMap* m, const Geo& g, const void* x, int n_frames) {
  auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (enc == nullptr) return false;
  const cuuint64_t es = (cuuint64_t)g.esize;
  const cuuint64_t dims[5] = {(cuuint64_t)g.d, (cuuint64_t)g.H, (cuuint64_t)g.fw, (cuuint64_t)g.fh,
                              (cuuint64_t)n_frames};
  const cuuint64_t row = (cuuint64_t)g.d * es;
  const cuuint64_t strides[4] = {row, row * g.H, row * g.H * g.fw, row * g.H * g.fw * g.fh};
  const cuuint32_t box[5] = {(cuuint32_t)g.d, 1, (cuuint32_t)g.tw, (cuuint32_t)g.th, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, g.dtype == PBSA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5,
             const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Resident CTAs of `kernel` per SM times the SM count of the current device (cached).
int persistent_grid(const void* kernel, int smem) {
  struct Entry { const void* k; int dev, smem, grid; };
  static std::mutex mu;
  static Entry cache[64];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (cache[i].k == kernel && cache[i].dev == dev && cache[i].smem == smem) return cache[i].grid;
  int sms = 148, per_sm = 1;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, BY_THREADS, smem);
  const int grid = sms * (per_sm > 0 ? per_sm : 1);
  if (n < 64) cache[n++] = {kernel, dev, smem, grid};
  return grid;
}

template <typename T, int D>
cudaError_t launch_t(const Geo& g, const void* x0, const void* x1, int n_frames, const BlockifyParams& p,
                     bool overlap_previous, cudaStream_t st) {
  CUtensorMap m0, m1;
  if (!encode_raster(&m0, g, x0, n_frames)) return cudaErrorNotSupported;
  if (x1 != nullptr) {
    if (!encode_raster(&m1, g, x1, n_frames)) return cudaErrorNotSupported;
  } else {
    m1 = m0;
  }
  constexpr int smem = Tile<T, D>::SMEM;
  auto kern = blockify_kernel<T, D>;
  cudaError_t e = set_smem_once((const void*)kern, smem);
  if (e != cudaSuccess) return e;
  const long units = (long)p.nz * p.nblk * p.H;
  const int grid = (int)(units < persistent_grid((const void*)kern, smem) ? units : persistent_grid((const void*)kern, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(BY_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_previous ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, m0, m1, p);
}

}  // namespace

cudaError_t launch_blockify_pair(const Geo& g, const void* x0, const void* x1, int n_frames, float* reps0,
                                 float* reps1, int rep_slots, const int* dst_slot, void* pool0, void* pool1,
                                 int pool_slots, bool overlap_previous, void* ws, cudaStream_t st) {
  BlockifyParams p;
  p.nz = x1 != nullptr ? 2 : 1;
  p.nblk = n_frames * g.bpf;
  p.H = g.H;
  p.bpf = g.bpf;
  p.tpr = g.tpr;
  p.th = g.th;
  p.tw = g.tw;
  p.rep_slots = rep_slots;
  p.pool_slots = pool_slots;
  p.reps[0] = reps0;
  p.reps[1] = reps1;
  p.pool[0] = pool0;
  p.pool[1] = pool1;
  p.dst_slot = dst_slot;
  p.ws = ws;
  if (g.dtype == PBSA_BF16) {
    if (g.d == 128) return launch_t<__nv_bfloat16, 128>(g, x0, x1, n_frames, p, overlap_previous, st);
    if (g.d == 64) return launch_t<__nv_bfloat16, 64>(g, x0, x1, n_frames, p, overlap_previous, st);
  } else {
    if (g.d == 128) return launch_t<float, 128>(g, x0, x1, n_frames, p, overlap_previous, st);
    if (g.d == 64) return launch_t<float, 64>(g, x0, x1, n_frames, p, overlap_previous, st);
    if (g.d == 32) return launch_t<float, 32>(g, x0, x1, n_frames, p, overlap_previous, st);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_blockify(const Geo& g, const void* x, int n_frames, float* reps, int rep_slots,
                            const int* dst_slot, void* pool, int pool_slots, void* ws,
                            cudaStream_t st) {
  return launch_blockify_pair(g, x, nullptr, n_frames, reps, nullptr, rep_slots, dst_slot, pool, nullptr,
                              pool_slots, false, ws, st);
}

}  // namespace pbsa
