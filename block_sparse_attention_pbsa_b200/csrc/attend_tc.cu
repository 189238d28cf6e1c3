// a3 (bf16) -- block-sparse fine attention on 5th-generation tensor cores (tcgen05).
//
// Sparse Forcing (gist.science, English 2.C "Global Access" + "Local Sparsity", 2.E "PBSA
// Kernel"; Chinese 2.2 "细粒度注意力" and "掩码机制"): every query block attends, in one
// softmax, to the persistent blocks (shared by all query blocks of a chunk) plus its own
// top-k local blocks.  Only the listed 64-token KV blocks are ever read.
//
// Design (sm_100a):
//  * One CTA per (head, pair of query blocks): the pair fills the 128 rows of one
//    M=128 tcgen05 MMA.  The two lists are merged in shared memory (bitmaps of the pool
//    slots); each merged entry carries a 2-bit mask (which query block of the pair attends
//    it).  Persistent blocks are shared by both halves, so most MMA rows are useful; rows of
//    a half that does not attend a block are masked in the softmax (p = 0).
//  * Each step covers two KV blocks (N = 128 keys).  Warp 0 gathers the K blocks, warp 2
//    the V blocks, with TMA (128-byte swizzle) into a 3-stage K ring and a 2-stage V ring;
//    a block that does not exist (odd count) is loaded out of bounds, i.e. zero-filled.
//    Q is loaded first, before the lists are read.
//  * TMEM holds three S/P buffers and one O accumulator (S0 | S1 | S2 | O = 512 columns);
//    step i uses S buffer i mod 3.  Two softmax warpgroups take alternate steps; one TMEM
//    lane = one query row per thread.  The online softmax works in the exp2 domain with
//    packed f32x2 arithmetic and writes P (bf16) back over the S columns it consumed.
//  * Warps 1 and 3 issue the MMAs of the even and the odd steps (one thread each; two
//    issuing threads keep the tensor pipe fuller than one).  Once P(i) is handed over, the
//    issuer of step i accumulates O += P(i) V(i) with the A operand read from TMEM, then
//    issues S(i+3) = Q K^T into the buffer P(i) occupied.  S(i+1) and S(i+2) already exist
//    by then, so a warpgroup never waits for its own PV before its next S: the loop is paced
//    by the exponentials and the tensor pipe, not by the chain S -> P -> PV -> next S.
//    PV(i) is issued once PV(i-1) has completed, so O accumulates in step order.
//  * The warpgroups take turns on the exponentials (the MUFU pipe is as busy as the tensor
//    pipe), so one warpgroup's exponentials overlap the other's MMAs.  That hand-off also
//    carries the row's reference maximum (shared memory): O has one reference per row, and
//    each warpgroup keeps its share of the row sum against the reference it last used.
//  * O is rescaled (in place, after PV(i-1) has completed) only when the reference grows by
//    more than 2^8; the epilogue adds the two warpgroups' row sums against the final
//    reference.
//  * Register split: the producer/issuer warpgroup runs on 64 registers, the softmax
//    warpgroups on 216 (setmaxnreg), so the softmax holds its row in registers.
//  * Each CTA signals programmatic dependents at its start (griddepcontrol.launch_dependents).
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
constexpr uint32_t REG_CTRL = 64, REG_SOFTMAX = 216;   // 128*64 + 256*216 = 384*165
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
constexpr uint32_t SM_MREF = SM_STAT + 2 * 128 * 8;   // float[128] running reference max per row
constexpr uint32_t SM_BITS = SM_MREF + 128 * 4;       // uint32[2][BITMAP_SLOTS / 32] list membership
constexpr int BITMAP_SLOTS = 8192;                    // pools up to this many slots merge in O(n)
constexpr uint32_t SM_TOTAL = SM_BITS + 2 * BITMAP_SLOTS / 8;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024;      // + alignment slack

constexpr int NSBUF = 3;             // S/P buffers in TMEM (O takes the fourth 128 columns)
enum { B_QFULL = 0, B_KFULL = 1, B_KEMPTY = B_KFULL + KSTAGES, B_VFULL = B_KEMPTY + KSTAGES,
       B_VEMPTY = B_VFULL + VSTAGES,
       B_SFULL = B_VEMPTY + VSTAGES,   // [S buffer]
       B_PFULL = B_SFULL + NSBUF,      // [S buffer], 128 arrivals (one per row)
       B_PVDONE = B_PFULL + NSBUF,     // [step parity]: PV of that step has completed
       B_MMADONE = B_PVDONE + 2,
       B_XDONE = B_MMADONE + 1,        // [warpgroup], 128 arrivals: its exponentials of a step are done
       NUM_BARS = B_XDONE + 2 };
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
  // The two lists are read first (at most 512 entries each: two per thread), before any set-up,
  // so their global loads are in flight while the barriers, Q's copy and TMEM are set up.
  static_assert(2 * NTHREADS >= 512, "two list entries per thread");
  const int* listA = prm.kv_slot + ((size_t)h * prm.nq + rA) * prm.kv_ld;
  const int* listB = prm.kv_slot + ((size_t)h * prm.nq + (hasB ? rB : rA)) * prm.kv_ld;
  int cA = prm.kv_cnt[(size_t)h * prm.nq + rA];
  int cB = hasB ? prm.kv_cnt[(size_t)h * prm.nq + rB] : 0;
  int la0 = 0, lb0 = 0, la1 = 0, lb1 = 0;
  if (tid < prm.kv_ld) { la0 = listA[tid]; lb0 = listB[tid]; }
  if (tid + NTHREADS < prm.kv_ld) { la1 = listA[tid + NTHREADS]; lb1 = listB[tid + NTHREADS]; }

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < NSBUF; ++i) mbar_init(&bars[B_PFULL + i], 128);
    for (int i = 0; i < 2; ++i) mbar_init(&bars[B_XDONE + i], 128);
    mbar_init(&bars[B_MMADONE], 2);
    *abort_flag = 0;
    fence_barrier_init();
    // Q (two 64-row blocks, strided raster rows): one 5-D box per 64 columns and block
    tma_prefetch_desc(&qmap);
    mbar_arrive_expect_tx(&bars[B_QFULL], 32768);
    for (int half = 0; half < 2; ++half) {
      const int r = (half == 1 && hasB) ? rB : rA;
      const int f = r / prm.bpf, rem = r - f * prm.bpf;
      const int ty = rem / prm.tpr, tx = rem - ty * prm.tpr;
      for (int p = 0; p < 2; ++p)
        tma_load_5d(sm + SM_Q + p * 16384 + half * 8192, &qmap, &bars[B_QFULL], p * 64, h,
                    tx * prm.tw, ty * prm.th, f);
    }
  }
  // A kernel launched after this one as a programmatic dependent (pbsa_blockify_kv with
  // PBSA_OVERLAP_PREVIOUS) may start once every CTA of this grid has started: it then only
  // takes SMs this grid leaves idle in its last wave.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // Merge the two query blocks' lists; mask bit 0 = block A attends, bit 1 = block B.  The
  // counts and the whole list rows are fetched together (one round trip); the Q load was
  // issued above, as it depends on nothing here.
  uint32_t* bitsA = reinterpret_cast<uint32_t*>(sm + SM_BITS);
  uint32_t* bitsB = bitsA + BITMAP_SLOTS / 32;
  const bool use_bits = prm.pool_slots <= BITMAP_SLOTS;
  if (use_bits)
    for (int i = tid; i < 2 * BITMAP_SLOTS / 32; i += NTHREADS) bitsA[i] = 0u;
  float* mref = reinterpret_cast<float*>(sm + SM_MREF);
  if (tid < 128) mref[tid] = -INFINITY;
  if (tid < prm.kv_ld) { la[tid] = la0; lb[tid] = lb0; }
  if (tid + NTHREADS < prm.kv_ld) { la[tid + NTHREADS] = la1; lb[tid + NTHREADS] = lb1; }
  if (cA < 0 || cA > prm.kv_ld || cB < 0 || cB > prm.kv_ld) {
    if (tid == 0) record_error(prm.ws, PBSA_ERR_DEVICE_INDEX, cA < 0 || cA > prm.kv_ld ? cA : cB, K_ATTEND_TC);
    cA = min(max(cA, 0), prm.kv_ld);
    cB = min(max(cB, 0), prm.kv_ld);
  }
  __syncthreads();
  auto in_range = [&](int s) { return s >= 0 && s < prm.pool_slots; };
  if (use_bits) {
    for (int i = tid; i < cA; i += NTHREADS)
      if (in_range(la[i])) atomicOr(&bitsA[la[i] >> 5], 1u << (la[i] & 31));
    for (int j = tid; j < cB; j += NTHREADS)
      if (in_range(lb[j])) atomicOr(&bitsB[lb[j] >> 5], 1u << (lb[j] & 31));
    __syncthreads();
    for (int i = tid; i < cA; i += NTHREADS) {
      const int s = la[i];
      mslot[i] = s;
      mflag[i] = (in_range(s) && ((bitsB[s >> 5] >> (s & 31)) & 1u)) ? 3 : 1;
    }
    for (int j = tid; j < cB; j += NTHREADS) {
      const int s = lb[j];
      onlyb[j] = (in_range(s) && ((bitsA[s >> 5] >> (s & 31)) & 1u)) ? 0 : 1;
    }
  } else {
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
  // ---------------------------------------------------------------- producer warps
  // Warp 0 loads Q and the K ring, warp 2 the V ring, so a V stage that is still in use
  // never holds back the prefetch of K.
  auto load_pair = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int i) {
    for (int b = 0; b < 2; ++b) {
      const int e = 2 * i + b;
      const int slot = e < n ? mslot[e] : -1;
      const int row0 = slot >= 0 ? (h * prm.pool_slots + slot) * 64 : prm.kv_rows;
      for (int p = 0; p < 2; ++p) tma_load_2d(dst + p * 16384 + b * 8192, map, bar, p * 64, row0);
    }
  };
  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_desc(&kmap);
      int kiss = 0;  // steps whose K loads were issued
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % KSTAGES;
        wait_or_abort(&bars[B_KEMPTY + s], ((i / KSTAGES) & 1) ^ 1, abort_flag, prm.ws, 1);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&bars[B_KFULL + s], 32768);
        load_pair(&kmap, sm + SM_K + s * 32768, &bars[B_KFULL + s], i);
        kiss = i + 1;
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the last copy issued into every stage before leaving
        for (int i = (kiss > KSTAGES ? kiss - KSTAGES : 0); i < kiss; ++i)
          mbar_wait(&bars[B_KFULL + i % KSTAGES], (i / KSTAGES) & 1, kWaitLimitNs);
      }
    }
    // Q was loaded at set-up; it must have landed before the CTA may exit, whether or not an
    // MMA consumed it (no steps, or an abort)
    if (lane == 0) mbar_wait(&bars[B_QFULL], 0, kWaitLimitNs);
    __syncwarp();
  }
  if (warp == 2) {
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_desc(&vmap);
      int viss = 0;  // steps whose V loads were issued
      for (int j = 0; j < nsteps; ++j) {
        const int s = j % VSTAGES;
        wait_or_abort(&bars[B_VEMPTY + s], ((j / VSTAGES) & 1) ^ 1, abort_flag, prm.ws, 2);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&bars[B_VFULL + s], 32768);
        load_pair(&vmap, sm + SM_V + s * 32768, &bars[B_VFULL + s], j);
        viss = j + 1;
      }
      if (*abort_flag) {
        for (int j = (viss > VSTAGES ? viss - VSTAGES : 0); j < viss; ++j)
          mbar_wait(&bars[B_VFULL + j % VSTAGES], (j / VSTAGES) & 1, kWaitLimitNs);
      }
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- MMA issuers
  // Step i uses S buffer i % 3 (TMEM columns [128 b, +128)); O is one accumulator in columns
  // [384, 512).  Warp 1 issues the tensor-core work of the even steps, warp 3 that of the
  // odd ones (one thread each: two issuing threads keep the tensor pipe fuller than one).
  // Once P(i) is handed over, the issuer of step i issues O += P(i) V(i) and then QK(i+3)
  // into the buffer P(i) occupied (same thread, so the tensor pipe runs them in that order);
  // S(i+1) and S(i+2) are computed by then, so no warpgroup's next S waits for its own PV.
  // PV(i) is issued only once PV(i-1) has completed, so O accumulates in step order (and
  // every earlier PV has completed when a softmax warpgroup rescales O).
  if (warp == 1 || warp == 3) {
    const int w = warp >> 1;
    if (lane == 0 && nsteps > 0) {
      const uint32_t tO = tmem + 384;
      // descriptors of the first 16-element K slice of each operand; a slice further on is
      // the same descriptor plus its byte offset / 16 (the start-address field)
      const uint64_t dq = sw128_desc(smem_u32(sm + SM_Q), 16, 1024);
      const uint64_t dk = sw128_desc(smem_u32(sm + SM_K), 16, 1024);
      const uint64_t dv = sw128_desc(smem_u32(sm + SM_V), 16384, 1024);
      auto issue_qk = [&](int i) {   // S_(i mod 3) = Q K_i^T, then free the K stage
        const int sk = i % KSTAGES, b = i % NSBUF;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_bf16_ss(tmem + b * 128, dq + off, dk + ((sk * 32768) >> 4) + off, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[B_SFULL + b]);
        mma_commit(&bars[B_KEMPTY + sk]);
      };
      wait_or_abort(&bars[B_QFULL], 0, abort_flag, prm.ws, 5);
      // the first three S: steps 0 and 2 from warp 1, step 1 from warp 3
      for (int j = w; j < NSBUF && j < nsteps; j += 2) {
        wait_or_abort(&bars[B_KFULL + j % KSTAGES], (j / KSTAGES) & 1, abort_flag, prm.ws, 6);
        if (*abort_flag) break;
        tc_fence_after();
        issue_qk(j);
      }
      for (int i = w; i < nsteps && !*abort_flag; i += 2) {
        const int sv = i % VSTAGES, b = i % NSBUF;
        // PV(i-1) complete first: it also orders the P-ready wait below after P(i-3)'s
        if (i >= 1) wait_or_abort(&bars[B_PVDONE + ((i - 1) & 1)], ((i - 1) >> 1) & 1, abort_flag, prm.ws, 12);
        wait_or_abort(&bars[B_VFULL + sv], (i / VSTAGES) & 1, abort_flag, prm.ws, 4);
        wait_or_abort(&bars[B_PFULL + b], (i / NSBUF) & 1, abort_flag, prm.ws, 3);
        if (*abort_flag) break;
        tc_fence_after();
        // O += P_i V_i: P_i (128 rows x 128 keys, bf16 pairs) sits over S_b in TMEM
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tO, tmem + b * 128 + kk * 8, dv + ((sv * 32768 + kk * 2048) >> 4), IDESC_PV,
                      (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[B_VEMPTY + sv]);
        mma_commit(&bars[B_PVDONE + (i & 1)]);
        if (i + NSBUF < nsteps) {
          wait_or_abort(&bars[B_KFULL + (i + NSBUF) % KSTAGES], ((i + NSBUF) / KSTAGES) & 1, abort_flag,
                        prm.ws, 6);
          if (*abort_flag) break;
          tc_fence_after();
          issue_qk(i + NSBUF);
        }
      }
      // every MMA of both issuers has completed once this barrier (count 2) flips
      mma_commit(&bars[B_MMADONE]);
      mbar_wait(&bars[B_MMADONE], 0, kWaitLimitNs);
    }
    __syncwarp();
  }

  } else {
  setmaxnreg_inc<REG_SOFTMAX>();
  // ---------------------------------------------------------------- softmax warpgroups
  {
    const int wg = (warp - 4) >> 2;          // this warpgroup takes the steps i = wg (mod 2)
    const int wq = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;          // query row of the 128-row tile
    const int half = row >> 6;
    const bool row_valid = half == 0 || hasB;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + 384;
    const float c = prm.scale_log2;
    // O has one reference maximum per row, mref[row], shared by both warpgroups: step i
    // reads it after the other warpgroup's step i-1 has published it.  l is this
    // warpgroup's share of the row sum, expressed against the reference m it last used.
    float m = -INFINITY, l = 0.f;
    for (int i = wg; i < nsteps; i += 2) {
      const int b = i % NSBUF;
      const uint32_t tS = tmem + lane_off + b * 128;
      const bool va = row_valid && ((mflag[2 * i] >> half) & 1);
      const bool vb = row_valid && 2 * i + 1 < n && ((mflag[2 * i + 1] >> half) & 1);
      wait_or_abort(&bars[B_SFULL + b], (i / NSBUF) & 1, abort_flag, prm.ws, 7);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      tc_fence_after();
      uint32_t x[4][32];
      // tcgen05.ld is warp-collective.  Every S column is finite (a block that does not exist
      // was loaded as zeros), so all four are read and masking is arithmetic.  The second
      // half is in flight while the first half's maximum is taken.
      tmem_ld32(tS + 0, x[0]);
      tmem_ld32(tS + 32, x[1]);
      tmem_wait_ld();
      tmem_ld32(tS + 64, x[2]);
      tmem_ld32(tS + 96, x[3]);
      float mx[2][2];
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        if (bb == 1) tmem_wait_ld();
        mx[bb][0] = mx[bb][1] = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2)
            mx[bb][e2 & 1] = fmax3(mx[bb][e2 & 1], __uint_as_float(x[2 * bb + q][2 * e2]),
                                   __uint_as_float(x[2 * bb + q][2 * e2 + 1]));
      }
      const float mba = va ? fmaxf(mx[0][0], mx[0][1]) : -INFINITY;
      const float mbb = vb ? fmaxf(mx[1][0], mx[1][1]) : -INFINITY;
      const float mb = fmaxf(mba, mbb) * c;
      // The two warpgroups take turns on the exponentials (the MUFU pipe is the scarce unit):
      // step i waits until the other warpgroup has finished those of step i-1, so one
      // warpgroup's exponentials overlap the other's MMAs instead of competing with them.
      // That wait also makes the reference maximum of step i-1 visible here.
      if (i >= 1) wait_or_abort(&bars[B_XDONE + (wg ^ 1)], ((i - 1) >> 1) & 1, abort_flag, prm.ws, 10);
      float alpha = 1.f;       // O's rescale factor for this row
      {
        const float mcur = mref[row];
        float mn = mcur;
        if (mb > mcur + 8.0f) {  // also true on the first valid block (mcur = -inf)
          if (mcur != -INFINITY) alpha = ex2_approx(mcur - mb);   // O holds earlier steps against mcur
          mn = mb;
        }
        mref[row] = mn;
        if (mn != m) {         // l in the new reference (l = 0 while m = -inf)
          l *= ex2_approx(m - mn);
          m = mn;
        }
      }
      // p = 2^(s*c - m) as bf16 pairs over the consumed S columns (32 keys per store).  A
      // masked block uses the factor 0 and the offset -inf, so it gives exact zeros without a
      // branch (x is finite).
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool v = q < 2 ? va : vb;
        const float cs = v ? c : 0.f, ms = v ? -m : -INFINITY;
        uint32_t pk[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float a0, a1, p0, p1;
          ffma2(__uint_as_float(x[q][2 * e2]), __uint_as_float(x[q][2 * e2 + 1]), cs, ms, a0, a1);
          p0 = ex2_approx(a0);
          p1 = ex2_approx(a1);
          if (e2 & 1) fadd2(ls[2], ls[3], p0, p1);
          else fadd2(ls[0], ls[1], p0, p1);
          pk[e2] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + q * 16, pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (i + 1 < nsteps) mbar_arrive(&bars[B_XDONE + wg]);
      // O holds PV(0..i-1) against the reference before this step.  Once PV(i-1) has
      // completed (PV(i) waits for this warpgroup's P), rows whose reference grew by more
      // than 2^8 are rescaled in place (alpha = 2^(old - new)).
      // tcgen05.ld/st are warp-collective, so the warp rescales if any of its rows must.
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        wait_or_abort(&bars[B_PVDONE + ((i - 1) & 1)], ((i - 1) >> 1) & 1, abort_flag, prm.ws, 11);
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
      mbar_arrive(&bars[B_PFULL + b]);
    }
    // epilogue: O is against the final reference M = mref[row]; L = l_0 2^(m_0-M) + l_1 2^(m_1-M).
    // The all-MMAs-done barrier has a single phase, so this wait cannot alias.
    if (nsteps > 0) wait_or_abort(&bars[B_MMADONE], 0, abort_flag, prm.ws, 9);
    float2* stat = reinterpret_cast<float2*>(sm + SM_STAT);
    stat[wg * 128 + row] = make_float2(m, l);
    asm volatile("bar.sync 1, 256;" ::: "memory");   // both softmax warpgroups, every path
    const float2 st0 = stat[row], st1 = stat[128 + row];
    const float M = mref[row];
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
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t oa[32];
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) oa[e2] = 0u;
        if (nsteps > 0) tmem_ld32(tO + wg * 64 + q * 32, oa);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t wv[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int k0 = cc * 8 + 2 * e2;
            wv[e2] = pack_bf16(__uint_as_float(oa[k0]) * inv, __uint_as_float(oa[k0 + 1]) * inv);
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
