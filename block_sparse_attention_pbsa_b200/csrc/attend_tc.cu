// a3 (bf16) -- block-sparse fine attention on 5th-generation tensor cores (tcgen05).
//
// Sparse Forcing (gist.science, English 2.C "Global Access" + "Local Sparsity", 2.E "PBSA
// Kernel"; Chinese 2.2 "细粒度注意力" and "掩码机制"): every query block attends, in one
// softmax, to the persistent blocks (shared by all query blocks of a chunk) plus its own
// top-k local blocks.  Only the listed 64-token KV blocks are ever read.
//
// Design (sm_100a):
//  * One CTA per (head, pair of query blocks): the pair fills the 128 rows of one
//    M=128 tcgen05 MMA.  The two lists are merged in shared memory; each merged entry
//    carries a 2-bit mask (which query block of the pair attends it).  Persistent blocks
//    are shared by both halves, so most MMA rows are useful; rows of a half that does not
//    attend a block are masked in the softmax (p = 0) and cost no exponentials.
//  * Each step covers two KV blocks (N = 128 keys).  A producer warp gathers the blocks
//    with TMA (128-byte swizzle) into a 2-stage K ring and a 2-stage V ring; blocks that
//    do not exist (odd count) are loaded out of bounds, i.e. zero-filled.
//  * An MMA warp (one thread) issues S = Q K^T into one of two TMEM S buffers and
//    O += P V into a TMEM O accumulator, with tcgen05.commit -> mbarrier hand-offs.
//  * Four softmax warps (one TMEM lane = one query row per thread) read S with
//    tcgen05.ld, run the online softmax in the exp2 domain, write P (bf16, swizzled) to
//    shared memory for the PV MMA, and rescale O in TMEM only when the running max grows
//    by more than 2^8 (the final O / l is exact either way).
//  * Every wait is bounded; on expiry the kernel records PBSA_ERR_TIMEOUT in the
//    workspace, drains its own copies and MMAs, frees TMEM and returns.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int D = 128;
constexpr int MAXL = 1024;  // merged list capacity (two lists of <= 512)
constexpr int NTHREADS = 192;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;                 // 2 panels x [128 rows][128 B]
constexpr uint32_t SM_K = 32768;             // 2 stages x 2 panels x [128 keys][128 B]
constexpr uint32_t SM_V = SM_K + 2 * 32768;  // same
constexpr uint32_t SM_P = SM_V + 2 * 32768;  // 2 panels x [128 rows][128 B]
constexpr uint32_t SM_BAR = SM_P + 32768;    // mbarriers
constexpr uint32_t SM_MISC = SM_BAR + 256;
constexpr uint32_t SM_SLOT = SM_MISC + 64;   // int[MAXL] merged slots
constexpr uint32_t SM_FLAG = SM_SLOT + 4 * MAXL;   // uint8[MAXL] masks
constexpr uint32_t SM_LA = SM_FLAG + MAXL;         // int[512]
constexpr uint32_t SM_LB = SM_LA + 4 * 512;        // int[512]
constexpr uint32_t SM_ONLYB = SM_LB + 4 * 512;     // uint8[512]
constexpr uint32_t SM_TOTAL = SM_ONLYB + 512;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024;   // + alignment slack

enum { B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7, B_SFULL = 9,
       B_PFULL = 11, B_PVDONE = 12, B_MMADONE = 13, NUM_BARS = 14 };

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);

struct Params {
  int H, pool_slots, nq, kv_ld;
  int bpf, tpr, tpf, fw, th, tw;
  int kv_rows;  // H * pool_slots * 64 (first out-of-bounds row of the pool tensor map)
  float scale_log2;
  const int* kv_slot;
  const int* kv_cnt;
  __nv_bfloat16* o;
  float* lse;
  void* ws;
};

__device__ __forceinline__ void wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              void* ws, int where) {
  if (*abort_flag) return;
  if (!mbar_wait(bar, parity, kWaitLimitNs)) {
    record_error(ws, PBSA_ERR_TIMEOUT, where, K_ATTEND_TC);
    *abort_flag = 1;
  }
}


__global__ void __launch_bounds__(NTHREADS, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_MISC + 4);
  int* n_merged_s = reinterpret_cast<int*>(sm + SM_MISC + 8);
  int* mslot = reinterpret_cast<int*>(sm + SM_SLOT);
  uint8_t* mflag = sm + SM_FLAG;
  int* la = reinterpret_cast<int*>(sm + SM_LA);
  int* lb = reinterpret_cast<int*>(sm + SM_LB);
  uint8_t* onlyb = sm + SM_ONLYB;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int rA = 2 * blockIdx.x, rB = rA + 1;
  const bool hasB = rB < prm.nq;

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], 1);
    mbar_init(&bars[B_PFULL], 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // merge the two query blocks' lists; mask bit 0 = block A attends, bit 1 = block B
  int cA = prm.kv_cnt[(size_t)h * prm.nq + rA];
  int cB = hasB ? prm.kv_cnt[(size_t)h * prm.nq + rB] : 0;
  if (cA < 0 || cA > prm.kv_ld || cB < 0 || cB > prm.kv_ld) {
    if (tid == 0) record_error(prm.ws, PBSA_ERR_DEVICE_INDEX, cA < 0 || cA > prm.kv_ld ? cA : cB, K_ATTEND_TC);
    cA = min(max(cA, 0), prm.kv_ld);
    cB = min(max(cB, 0), prm.kv_ld);
  }
  const int* listA = prm.kv_slot + ((size_t)h * prm.nq + rA) * prm.kv_ld;
  const int* listB = prm.kv_slot + ((size_t)h * prm.nq + (hasB ? rB : rA)) * prm.kv_ld;
  for (int i = tid; i < cA; i += NTHREADS) la[i] = listA[i];
  for (int i = tid; i < cB; i += NTHREADS) lb[i] = listB[i];
  __syncthreads();
  for (int i = tid; i < cA; i += NTHREADS) {
    const int s = la[i];
    uint8_t f = 1;
    for (int j = 0; j < cB; ++j) f |= (lb[j] == s) ? 2 : 0;
    mslot[i] = s;
    mflag[i] = f;
  }
  for (int j = tid; j < cB; j += NTHREADS) {
    const int s = lb[j];
    bool in_a = false;
    for (int i = 0; i < cA; ++i) in_a |= (la[i] == s);
    onlyb[j] = in_a ? 0 : 1;
  }
  __syncthreads();
  if (tid == 0) {
    int pos = cA;
    for (int j = 0; j < cB; ++j)
      if (onlyb[j]) {
        mslot[pos] = lb[j];
        mflag[pos] = 2;
        ++pos;
      }
    *n_merged_s = pos;
  }
  __syncthreads();
  const int n = *n_merged_s;
  for (int i = tid; i < n; i += NTHREADS) {
    const int s = mslot[i];
    if (s < 0 || s >= prm.pool_slots) {
      record_error(prm.ws, PBSA_ERR_DEVICE_INDEX, s, K_ATTEND_TC);
      mslot[i] = -1;  // loaded out of bounds (zeros), and masked
      mflag[i] = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nsteps = (n + 1) >> 1;

  // ---------------------------------------------------------------- producer warp
  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(&bars[B_QFULL], 32768);
      for (int half = 0; half < 2; ++half) {
        const int r = (half == 1 && hasB) ? rB : rA;
        const int f = r / prm.bpf, rem = r - f * prm.bpf;
        const int ty = rem / prm.tpr, tx = rem - ty * prm.tpr;
        for (int p = 0; p < 2; ++p)
          tma_load_5d(sm + SM_Q + p * 16384 + half * 8192, &qmap, &bars[B_QFULL], p * 64, h,
                      tx * prm.tw, ty * prm.th, f);
      }
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        wait_or_abort(&bars[B_KEMPTY + s], ph ^ 1, abort_flag, prm.ws, 1);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&bars[B_KFULL + s], 32768);
        for (int b = 0; b < 2; ++b) {
          const int e = 2 * i + b;
          const int slot = e < n ? mslot[e] : -1;
          const int row0 = slot >= 0 ? (h * prm.pool_slots + slot) * 64 : prm.kv_rows;
          for (int p = 0; p < 2; ++p)
            tma_load_2d(sm + SM_K + s * 32768 + p * 16384 + b * 8192, &kmap, &bars[B_KFULL + s], p * 64, row0);
        }
        wait_or_abort(&bars[B_VEMPTY + s], ph ^ 1, abort_flag, prm.ws, 2);
        if (*abort_flag) {
          issued = 2 * i + 1;  // K of step i in flight, V not
          break;
        }
        mbar_arrive_expect_tx(&bars[B_VFULL + s], 32768);
        for (int b = 0; b < 2; ++b) {
          const int e = 2 * i + b;
          const int slot = e < n ? mslot[e] : -1;
          const int row0 = slot >= 0 ? (h * prm.pool_slots + slot) * 64 : prm.kv_rows;
          for (int p = 0; p < 2; ++p)
            tma_load_2d(sm + SM_V + s * 32768 + p * 16384 + b * 8192, &vmap, &bars[B_VFULL + s], p * 64, row0);
        }
        issued = 2 * i + 2;
      }
      if (*abort_flag) {
        // drain: wait (bounded) for every copy this warp issued before leaving
        mbar_wait(&bars[B_QFULL], 0, kWaitLimitNs);
        const int ksteps = (issued + 1) >> 1, vsteps = issued >> 1;
        for (int i = (ksteps > 2 ? ksteps - 2 : 0); i < ksteps; ++i)
          mbar_wait(&bars[B_KFULL + (i & 1)], (i >> 1) & 1, kWaitLimitNs);
        for (int i = (vsteps > 2 ? vsteps - 2 : 0); i < vsteps; ++i)
          mbar_wait(&bars[B_VFULL + (i & 1)], (i >> 1) & 1, kWaitLimitNs);
      }
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- MMA warp
  if (warp == 1) {
    if (lane == 0 && nsteps > 0) {
      const uint32_t q_base = smem_u32(sm + SM_Q), k_base = smem_u32(sm + SM_K);
      const uint32_t v_base = smem_u32(sm + SM_V), p_base = smem_u32(sm + SM_P);
      const uint32_t tS = tmem, tO = tmem + 256;
      auto issue_pv = [&](int j) {
        const int s = j & 1;
        wait_or_abort(&bars[B_PFULL], j & 1, abort_flag, prm.ws, 3);
        wait_or_abort(&bars[B_VFULL + s], (j >> 1) & 1, abort_flag, prm.ws, 4);
        if (*abort_flag) return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sw128_desc(p_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sw128_desc(v_base + s * 32768 + kk * 2048, 16384, 1024);
          mma_bf16_ss(tO, a, b, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[B_VEMPTY + s]);
        mma_commit(&bars[B_PVDONE]);
      };
      wait_or_abort(&bars[B_QFULL], 0, abort_flag, prm.ws, 5);
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i & 1;
        wait_or_abort(&bars[B_KFULL + s], (i >> 1) & 1, abort_flag, prm.ws, 6);
        if (*abort_flag) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sw128_desc(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sw128_desc(k_base + s * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tS + s * 128, a, b, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[B_SFULL + s]);
        mma_commit(&bars[B_KEMPTY + s]);
        if (i >= 1) issue_pv(i - 1);
      }
      if (!*abort_flag) issue_pv(nsteps - 1);
      // every MMA this thread issued has completed once this barrier flips
      mma_commit(&bars[B_MMADONE]);
      mbar_wait(&bars[B_MMADONE], 0, kWaitLimitNs);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- softmax warps
  if (warp >= 2) {
    const int wq = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;          // query row of the 128-row tile
    const int half = row >> 6;
    const bool row_valid = half == 0 || hasB;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float c = prm.scale_log2;
    uint8_t* prow = sm + SM_P + row * 128;
    const int sw = row & 7;
    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i & 1;
      const int fa = mflag[2 * i], fb = (2 * i + 1 < n) ? mflag[2 * i + 1] : 0;
      const bool va = row_valid && ((fa >> half) & 1), vb = row_valid && ((fb >> half) & 1);
      wait_or_abort(&bars[B_SFULL + s], (i >> 1) & 1, abort_flag, prm.ws, 7);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      tc_fence_after();
      uint32_t x[4][32];
      if (va) {
        tmem_ld32(tmem + lane_off + s * 128 + 0, x[0]);
        tmem_ld32(tmem + lane_off + s * 128 + 32, x[1]);
      }
      if (vb) {
        tmem_ld32(tmem + lane_off + s * 128 + 64, x[2]);
        tmem_ld32(tmem + lane_off + s * 128 + 96, x[3]);
      }
      tmem_wait_ld();
      float mb = -INFINITY;
      if (va) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e = 0; e < 32; ++e) mb = fmaxf(mb, __uint_as_float(x[q][e]));
      }
      if (vb) {
#pragma unroll
        for (int q = 2; q < 4; ++q)
#pragma unroll
          for (int e = 0; e < 32; ++e) mb = fmaxf(mb, __uint_as_float(x[q][e]));
      }
      mb *= c;
      float alpha = 1.f;
      bool rescale_o = false;
      if (mb > m + 8.0f) {  // also true on the first valid block (m = -inf)
        rescale_o = (m != -INFINITY) && i > 0;
        alpha = ex2_approx(m - mb);
        l *= alpha;
        m = mb;
      }
      // p = 2^(s*c - m), packed to bf16 pairs; masked halves give 0
      uint32_t pk[4][16];
      float ls = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool v = q < 2 ? va : vb;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0 = 0.f, p1 = 0.f;
          if (v) {
            p0 = ex2_approx(fmaf(__uint_as_float(x[q][2 * e]), c, -m));
            p1 = ex2_approx(fmaf(__uint_as_float(x[q][2 * e + 1]), c, -m));
          }
          ls += p0 + p1;
          pk[q][e] = pack_bf16(p0, p1);
        }
      }
      l += ls;
      // the P buffer and O are free once the previous PV has completed
      if (i >= 1) wait_or_abort(&bars[B_PVDONE], (i - 1) & 1, abort_flag, prm.ws, 8);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      // tcgen05.ld/st are warp-collective: the warp rescales if any of its rows must
      if (__any_sync(0xffffffffu, rescale_o)) {
        if (!rescale_o) alpha = 1.f;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + 256 + q * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tmem + lane_off + 256 + q * 32, ov);
        }
        tmem_wait_st();
      }
      // row of P: keys 0..63 -> panel 0, 64..127 -> panel 1; 16-byte chunks swizzled by row
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint8_t* panel = prow + (q >> 1) * 16384;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int chunk = (q & 1) * 4 + cc;
          *reinterpret_cast<uint4*>(panel + ((chunk ^ sw) << 4)) =
              make_uint4(pk[q][4 * cc], pk[q][4 * cc + 1], pk[q][4 * cc + 2], pk[q][4 * cc + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL]);
    }
    // epilogue: O / l -> bf16 raster rows, and the log-sum-exp
    if (nsteps > 0) wait_or_abort(&bars[B_PVDONE], (nsteps - 1) & 1, abort_flag, prm.ws, 9);
    if (row_valid && !__any_sync(0xffffffffu, *abort_flag != 0)) {
      const int r = half ? rB : rA;
      const int f = r / prm.bpf, rem = r - f * prm.bpf;
      const int ty = rem / prm.tpr, tx = rem - ty * prm.tpr;
      const int rr = row & 63, ly = rr / prm.tw, lx = rr - ly * prm.tw;
      const size_t t = (size_t)f * prm.tpf + (size_t)(ty * prm.th + ly) * prm.fw + tx * prm.tw + lx;
      uint4* dst = reinterpret_cast<uint4*>(prm.o + (t * prm.H + h) * D);
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t ov[32];
        if (nsteps > 0) {
          tmem_ld32(tmem + lane_off + 256 + q * 32, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16(__uint_as_float(ov[cc * 8 + 2 * e]) * inv, __uint_as_float(ov[cc * 8 + 2 * e + 1]) * inv);
          dst[q * 4 + cc] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (prm.lse != nullptr) {
        const size_t Tq = (size_t)prm.nq / prm.bpf * prm.tpf;
        prm.lse[(size_t)h * Tq + t] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

void* tensor_map_encoder() {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}

namespace {
// bf16 tensor map with 128-byte swizzle; dims/strides fastest first (strides in bytes, rank-1).
bool encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (enc == nullptr) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
             strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_attend_tc(const Geo& g, const void* q, int q_frames, const void* k_pool,
                             const void* v_pool, int pool_slots, const int* kv_slot,
                             const int* kv_cnt, int kv_ld, void* o, float* lse, void* ws,
                             cudaStream_t st) {
  if (g.d != D || g.dtype != PBSA_BF16) return cudaErrorNotSupported;
  const int nq = q_frames * g.bpf;
  CUtensorMap qmap, kmap, vmap;
  {
    const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)g.H, (cuuint64_t)g.fw, (cuuint64_t)g.fh,
                                (cuuint64_t)q_frames};
    const cuuint64_t row = (cuuint64_t)D * 2;
    const cuuint64_t strides[4] = {row, row * g.H, row * g.H * g.fw, row * g.H * g.fw * g.fh};
    const cuuint32_t box[5] = {64, 1, (cuuint32_t)g.tw, (cuuint32_t)g.th, 1};
    if (!encode_bf16(&qmap, q, 5, dims, strides, box)) return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)g.H * pool_slots * BT};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 64};
    if (!encode_bf16(&kmap, k_pool, 2, dims, strides, box)) return cudaErrorNotSupported;
    if (!encode_bf16(&vmap, v_pool, 2, dims, strides, box)) return cudaErrorNotSupported;
  }
  Params prm;
  prm.H = g.H;
  prm.pool_slots = pool_slots;
  prm.nq = nq;
  prm.kv_ld = kv_ld;
  prm.bpf = g.bpf;
  prm.tpr = g.tpr;
  prm.tpf = g.tpf;
  prm.fw = g.fw;
  prm.th = g.th;
  prm.tw = g.tw;
  prm.kv_rows = g.H * pool_slots * BT;
  prm.scale_log2 = g.scale * 1.4426950408889634f;
  prm.kv_slot = kv_slot;
  prm.kv_cnt = kv_cnt;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.ws = ws;
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((nq + 1) / 2, g.H);
  attend_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(qmap, kmap, vmap, prm);
  return cudaGetLastError();
}

}  // namespace pbsa
