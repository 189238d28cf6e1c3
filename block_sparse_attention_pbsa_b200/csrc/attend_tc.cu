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
//    with TMA (128-byte swizzle) into a 3-stage K ring and a 2-stage V ring; a block that
//    does not exist (odd count) is loaded out of bounds, i.e. zero-filled.
//  * An MMA warp (one thread) issues S = Q K^T into one of two TMEM S buffers.  Two
//    softmax warpgroups each own one of the step's two blocks and run an independent
//    online softmax (exp2 domain) over "their" half of the list, one TMEM lane = one
//    query row per thread.  Each writes its P (bf16) back into TMEM over the S columns it
//    consumed, and the MMA warp accumulates O_w += P_w V_w with the A operand read from
//    TMEM, into a per-warpgroup O accumulator (TMEM = S0 | S1 | O0 | O1 = 512 columns).
//    O_w is rescaled only when its running max grows by more than 2^8; the epilogue
//    merges the two streams exactly.
//  * Register split: the producer/MMA warpgroup runs on 56 registers, the softmax
//    warpgroups on 224 (setmaxnreg), so the softmax holds its row in registers.
//  * Every wait is bounded; on expiry the kernel records PBSA_ERR_TIMEOUT in the
//    workspace, drains its own copies and MMAs, frees TMEM and returns.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int D = 128;
constexpr int MAXL = 1024;           // merged list capacity (two lists of <= 512)
constexpr int NTHREADS = 384;        // warpgroup 0: producer + MMA; 1, 2: softmax
constexpr int KSTAGES = 3, VSTAGES = 2;
constexpr uint32_t REG_CTRL = 56, REG_SOFTMAX = 224;   // 128*56 + 256*224 = 384*168
static_assert(128 * REG_CTRL + 256 * REG_SOFTMAX <= NTHREADS * 168, "register split exceeds launch budget");

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;                          // 2 panels x [128 rows][128 B]
constexpr uint32_t SM_K = 32768;                      // KSTAGES x 2 panels x [128 keys][128 B]
constexpr uint32_t SM_V = SM_K + KSTAGES * 32768;     // VSTAGES x same
constexpr uint32_t SM_BAR = SM_V + VSTAGES * 32768;   // mbarriers
constexpr uint32_t SM_MISC = SM_BAR + 256;
constexpr uint32_t SM_SLOT = SM_MISC + 64;            // int[MAXL] merged slots
constexpr uint32_t SM_FLAG = SM_SLOT + 4 * MAXL;      // uint8[MAXL] masks
constexpr uint32_t SM_LA = SM_FLAG + MAXL;            // int[512]
constexpr uint32_t SM_LB = SM_LA + 4 * 512;           // int[512]
constexpr uint32_t SM_ONLYB = SM_LB + 4 * 512;        // uint8[512]
constexpr uint32_t SM_STAT = SM_ONLYB + 512;          // float2[2][128] epilogue (m, l) exchange
constexpr uint32_t SM_TOTAL = SM_STAT + 2 * 128 * 8;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024;      // + alignment slack

enum { B_QFULL = 0, B_KFULL = 1, B_KEMPTY = B_KFULL + KSTAGES, B_VFULL = B_KEMPTY + KSTAGES,
       B_VEMPTY = B_VFULL + VSTAGES, B_SFULL = B_VEMPTY + VSTAGES,
       B_PFULL = B_SFULL + 2,      // [warpgroup][step & 1]: a softmax warpgroup may run up to
                                   // two steps ahead of the MMA warp's wait, so P-full is a ring
       B_PVDONE = B_PFULL + 4, B_MMADONE = B_PVDONE + 2, NUM_BARS = B_MMADONE + 1 };
static_assert(NUM_BARS * 8 <= 256, "barrier area");

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
    for (int i = 0; i < 4; ++i) mbar_init(&bars[B_PFULL + i], 128);
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
  if (warp == 0) {
    // compact the B-only entries behind A's list, in order (warp ballot prefix sums)
    int pos = cA;
    for (int base = 0; base < cB; base += 32) {
      const int j = base + lane;
      const bool take = j < cB && onlyb[j];
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int at = pos + __popc(bal & ((1u << lane) - 1u));
        mslot[at] = lb[j];
        mflag[at] = 2;
      }
      pos += __popc(bal);
    }
    if (lane == 0) *n_merged_s = pos;
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

  // Each role's whole body sits inside the branch that sets its register budget.
  if (warp < 4) {
  setmaxnreg_dec<REG_CTRL>();
  // ---------------------------------------------------------------- producer warp
  // K of step i is issued one step ahead of V of step i-1, so K runs ahead of the PV MMAs.
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
      int kiss = 0, viss = 0;  // steps whose K / V loads were issued
      auto load_pair = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int i) {
        for (int b = 0; b < 2; ++b) {
          const int e = 2 * i + b;
          const int slot = e < n ? mslot[e] : -1;
          const int row0 = slot >= 0 ? (h * prm.pool_slots + slot) * 64 : prm.kv_rows;
          for (int p = 0; p < 2; ++p) tma_load_2d(dst + p * 16384 + b * 8192, map, bar, p * 64, row0);
        }
      };
      for (int i = 0; i <= nsteps; ++i) {
        if (i < nsteps) {
          const int s = i % KSTAGES;
          wait_or_abort(&bars[B_KEMPTY + s], ((i / KSTAGES) & 1) ^ 1, abort_flag, prm.ws, 1);
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&bars[B_KFULL + s], 32768);
          load_pair(&kmap, sm + SM_K + s * 32768, &bars[B_KFULL + s], i);
          kiss = i + 1;
        }
        if (i >= 1) {
          const int j = i - 1, s = j % VSTAGES;
          wait_or_abort(&bars[B_VEMPTY + s], ((j / VSTAGES) & 1) ^ 1, abort_flag, prm.ws, 2);
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&bars[B_VFULL + s], 32768);
          load_pair(&vmap, sm + SM_V + s * 32768, &bars[B_VFULL + s], j);
          viss = j + 1;
        }
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the last copy issued into every stage before leaving
        mbar_wait(&bars[B_QFULL], 0, kWaitLimitNs);
        for (int i = (kiss > KSTAGES ? kiss - KSTAGES : 0); i < kiss; ++i)
          mbar_wait(&bars[B_KFULL + i % KSTAGES], (i / KSTAGES) & 1, kWaitLimitNs);
        for (int i = (viss > VSTAGES ? viss - VSTAGES : 0); i < viss; ++i)
          mbar_wait(&bars[B_VFULL + i % VSTAGES], (i / VSTAGES) & 1, kWaitLimitNs);
      }
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- MMA warp
  // S_i -> TMEM columns [128 (i%2), +128); P_w(i) is written by softmax warpgroup w over the
  // first 32 columns of its block's S half; O_w accumulates in columns [256 + 128 w, +128).
  if (warp == 1) {
    if (lane == 0 && nsteps > 0) {
      const uint32_t q_base = smem_u32(sm + SM_Q), k_base = smem_u32(sm + SM_K);
      const uint32_t v_base = smem_u32(sm + SM_V);
      const uint32_t tO = tmem + 256;
      auto issue_pv = [&](int j) {
        const int sv = j % VSTAGES;
        wait_or_abort(&bars[B_VFULL + sv], (j / VSTAGES) & 1, abort_flag, prm.ws, 4);
        for (int w = 0; w < 2; ++w) {
          wait_or_abort(&bars[B_PFULL + 2 * w + (j & 1)], (j >> 1) & 1, abort_flag, prm.ws, 3);
          if (*abort_flag) return;
          tc_fence_after();
          const uint32_t a_tmem = tmem + (j & 1) * 128 + w * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t b = sw128_desc(v_base + sv * 32768 + w * 8192 + kk * 2048, 16384, 1024);
            mma_bf16_ts(tO + w * 128, a_tmem + kk * 8, b, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars[B_PVDONE + w]);
        }
        mma_commit(&bars[B_VEMPTY + sv]);
      };
      wait_or_abort(&bars[B_QFULL], 0, abort_flag, prm.ws, 5);
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int sk = i % KSTAGES;
        wait_or_abort(&bars[B_KFULL + sk], (i / KSTAGES) & 1, abort_flag, prm.ws, 6);
        if (*abort_flag) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sw128_desc(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sw128_desc(k_base + sk * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + (i & 1) * 128, a, b, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[B_SFULL + (i & 1)]);
        mma_commit(&bars[B_KEMPTY + sk]);
        if (i >= 1) issue_pv(i - 1);
      }
      if (!*abort_flag) issue_pv(nsteps - 1);
      // every MMA this thread issued has completed once this barrier flips
      mma_commit(&bars[B_MMADONE]);
      mbar_wait(&bars[B_MMADONE], 0, kWaitLimitNs);
    }
    __syncwarp();
  }

  } else {
  setmaxnreg_inc<REG_SOFTMAX>();
  // ---------------------------------------------------------------- softmax warpgroups
  {
    const int wg = (warp - 4) >> 2;          // 0: first block of each step, 1: second
    const int wq = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;          // query row of the 128-row tile
    const int half = row >> 6;
    const bool row_valid = half == 0 || hasB;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256 + wg * 128;
    const float c = prm.scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < nsteps; ++i) {
      const int e = 2 * i + wg;
      const bool v = row_valid && e < n && ((mflag[e] >> half) & 1);
      const uint32_t tS = tmem + lane_off + (i & 1) * 128 + wg * 64;
      wait_or_abort(&bars[B_SFULL + (i & 1)], (i >> 1) & 1, abort_flag, prm.ws, 7);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      tc_fence_after();
      uint32_t x[2][32];
      if (__any_sync(0xffffffffu, v)) {   // tcgen05.ld is warp-collective
        tmem_ld32(tS, x[0]);
        tmem_ld32(tS + 32, x[1]);
        tmem_wait_ld();
      }
      float mb = -INFINITY;
      if (v) {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) mx[e2 & 3] = fmaxf(mx[e2 & 3], __uint_as_float(x[q][e2]));
        mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
      }
      float alpha = 1.f;
      bool rescale_o = false;
      if (mb > m + 8.0f) {  // also true on the first valid block (m = -inf)
        rescale_o = (m != -INFINITY) && i > 0;
        alpha = ex2_approx(m - mb);
        l *= alpha;
        m = mb;
      }
      // p = 2^(s*c - m) packed to bf16 pairs; a masked block gives 0
      uint32_t pk[32];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float p0 = 0.f, p1 = 0.f;
          if (v) {
            p0 = ex2_approx(fmaf(__uint_as_float(x[q][2 * e2]), c, -m));
            p1 = ex2_approx(fmaf(__uint_as_float(x[q][2 * e2 + 1]), c, -m));
          }
          ls[e2 & 3] += p0 + p1;
          pk[q * 16 + e2] = pack_bf16(p0, p1);
        }
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // P over the S columns just read (the previous user of this buffer, PV(i-2), finished
      // before S_i was produced)
      tmem_st32(tS, pk);
      // O_w may only be rescaled once PV_w(i-1) has completed; tcgen05.ld/st are
      // warp-collective, so the warp rescales if any of its rows must
      if (__any_sync(0xffffffffu, rescale_o)) {
        wait_or_abort(&bars[B_PVDONE + wg], (i - 1) & 1, abort_flag, prm.ws, 8);
        if (!rescale_o) alpha = 1.f;
        tc_fence_after();
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t ov[32];
          tmem_ld32(tO + q * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) ov[e2] = __float_as_uint(__uint_as_float(ov[e2]) * alpha);
          tmem_st32(tO + q * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL + 2 * wg + (i & 1)]);
    }
    // epilogue: combine the two streams, O = (O_0 2^(m0-M) + O_1 2^(m1-M)) / L.  The
    // all-MMAs-done barrier has a single phase, so this wait cannot alias.
    if (nsteps > 0) wait_or_abort(&bars[B_MMADONE], 0, abort_flag, prm.ws, 9);
    float2* stat = reinterpret_cast<float2*>(sm + SM_STAT);
    stat[wg * 128 + row] = make_float2(m, l);
    asm volatile("bar.sync 1, 256;" ::: "memory");   // both softmax warpgroups, every path
    const float2 st0 = stat[row], st1 = stat[128 + row];
    const float M = fmaxf(st0.x, st1.x);
    const float f0 = st0.x == -INFINITY ? 0.f : ex2_approx(st0.x - M);
    const float f1 = st1.x == -INFINITY ? 0.f : ex2_approx(st1.x - M);
    const float Lsum = st0.y * f0 + st1.y * f1;
    if (row_valid && !__any_sync(0xffffffffu, *abort_flag != 0)) {
      const int r = half ? rB : rA;
      const int f = r / prm.bpf, rem = r - f * prm.bpf;
      const int ty = rem / prm.tpr, tx = rem - ty * prm.tpr;
      const int rr = row & 63, ly = rr / prm.tw, lx = rr - ly * prm.tw;
      const size_t t = (size_t)f * prm.tpf + (size_t)(ty * prm.th + ly) * prm.fw + tx * prm.tw + lx;
      uint4* dst = reinterpret_cast<uint4*>(prm.o + (t * prm.H + h) * D) + wg * 8;
      const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
      const float g0 = f0 * inv, g1 = f1 * inv;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t oa[32], ob[32];
        if (nsteps > 0) {
          tmem_ld32(tmem + lane_off + 256 + wg * 64 + q * 32, oa);
          tmem_ld32(tmem + lane_off + 384 + wg * 64 + q * 32, ob);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) oa[e2] = ob[e2] = 0u;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t wv[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int k0 = cc * 8 + 2 * e2;
            wv[e2] = pack_bf16(__uint_as_float(oa[k0]) * g0 + __uint_as_float(ob[k0]) * g1,
                               __uint_as_float(oa[k0 + 1]) * g0 + __uint_as_float(ob[k0 + 1]) * g1);
          }
          dst[q * 4 + cc] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      }
      if (prm.lse != nullptr && wg == 0) {
        const size_t Tq = (size_t)prm.nq / prm.bpf * prm.tpf;
        prm.lse[(size_t)h * Tq + t] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
      }
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
  cudaError_t e = set_smem_once((const void*)attend_tc_kernel, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((nq + 1) / 2, g.H);
  attend_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(qmap, kmap, vmap, prm);
  return cudaGetLastError();
}

}  // namespace pbsa
