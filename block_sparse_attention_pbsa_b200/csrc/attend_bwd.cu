// a5 -- backward of the block-sparse fine attention under the same block lists.
//
// Sparse Forcing (gist.science, English 2.D "Training Strategy"; Chinese 2.3): the model is
// trained with the same dynamic sparse cache as at inference, so the sparse attention
// needs its gradients.  With P recomputed from the forward's log-sum-exp:
//   P = exp(scale*Q K^T - LSE),  D_i = dO_i . O_i,  dP = dO V^T,  dS = P * (dP - D),
//   dV = P^T dO,  dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Deterministic design (no floating-point atomics), five launches; S and dP are computed
// once per (query block, KV block) pair, so the passes issue the five contractions S, dP, dV,
// dK, dQ:
//   1. bwd_prep_kernel  -- per query block: D and log2-domain LSE in block order, and the
//      number of query blocks attending each KV slot (integer atomics);
//   2. bwd_scan_kernel  -- per head: exclusive scan of those counts;
//   3. bwd_fill_kernel  -- per query block: the inverse lists (KV slot -> query block and the
//      slot's position in that block's list);
//   4. bwd_dkdv_kernel  -- one CTA per (head, pair of KV slots) over the query blocks that
//      attend them (sorted, merged with a per-half mask): S^T = K Q^T, dP^T = V dO^T,
//      dV += P^T dO and dK += dS^T Q with P^T, dS^T read from TMEM; each 64 x 64 dS^T tile
//      also goes to the workspace (one tile per list entry, 8 KB);
//   5. bwd_dqs_kernel   -- one CTA per (head, pair of query blocks): dQ += dS K over the
//      merged list, A = the stored dS^T tiles read query-contiguous (MN-major).
// The dS^T round trip through HBM (2 x 8 KB per pair) replaces the recomputation of S and dP
// that a dQ pass needs otherwise.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int D = 128;
constexpr float LOG2E = 1.4426950408889634f;

__host__ __device__ inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdLayout {
  size_t dvec, lvec, cnt, off, cur, inv, zero, ds, end;
};
__host__ __device__ inline BwdLayout bwd_layout(int H, int nq, int ps, int kv_ld) {
  BwdLayout L;
  L.dvec = WS_HEADER_BYTES;
  L.lvec = L.dvec + a256((size_t)H * nq * BT * 4);
  L.cnt = L.lvec + a256((size_t)H * nq * BT * 4);
  L.off = L.cnt + a256((size_t)H * ps * 4);
  L.cur = L.off + a256((size_t)H * ps * 4);
  L.inv = L.cur + a256((size_t)H * ps * 4);
  L.zero = L.inv + a256((size_t)H * nq * kv_ld * 4);
  L.ds = L.zero + BT * BT * 2;
  L.end = L.ds + (size_t)H * nq * kv_ld * BT * BT * 2;   // one 64 x 64 bf16 dS^T tile per list entry
  return L;
}

struct BwdGeo {
  int H, nq, kv_ld, pool_slots;
  int bpf, tpr, tpf, fw, th, tw;
};

__device__ __forceinline__ size_t token_of(const BwdGeo& g, int r, int row) {
  const int f = r / g.bpf, rem = r - f * g.bpf;
  const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
  const int ly = row / g.tw, lx = row - ly * g.tw;
  return (size_t)f * g.tpf + (size_t)(ty * g.th + ly) * g.fw + tx * g.tw + lx;
}

// ---------------------------------------------------------------------------- 1. prep
// D_i = sum_d dO_i * O_i (fp32 from the bf16 tensors), LSE in log2 units, both in block
// order; counts of query blocks per KV slot.
__global__ void __launch_bounds__(64) bwd_prep_kernel(
    BwdGeo g, const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
    const float* __restrict__ lse, const int* __restrict__ kv_slot, const int* __restrict__ kv_cnt,
    float* __restrict__ dvec, float* __restrict__ lvec, int* __restrict__ cnt, void* ws) {
  const int r = blockIdx.x, h = blockIdx.y, row = threadIdx.x;
  const size_t t = token_of(g, r, row);
  const uint4* op = reinterpret_cast<const uint4*>(o + (t * g.H + h) * D);
  const uint4* gp = reinterpret_cast<const uint4*>(d_o + (t * g.H + h) * D);
  uint4 a[16], b[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    a[i] = __ldg(op + i);
    b[i] = __ldg(gp + i);
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t x[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
    const uint32_t y[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[j] = fmaf(__uint_as_float(x[j] << 16), __uint_as_float(y[j] << 16), acc[j]);
      acc[j] = fmaf(__uint_as_float(x[j] & 0xFFFF0000u), __uint_as_float(y[j] & 0xFFFF0000u), acc[j]);
    }
  }
  const size_t Tq = (size_t)g.nq / g.bpf * g.tpf;
  const size_t bi = ((size_t)h * g.nq + r) * BT + row;
  dvec[bi] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  lvec[bi] = lse[(size_t)h * Tq + t] * LOG2E;
  int c = kv_cnt[(size_t)h * g.nq + r];
  c = min(max(c, 0), g.kv_ld);
  const int* list = kv_slot + ((size_t)h * g.nq + r) * g.kv_ld;
  for (int e = row; e < c; e += 64) {
    const int s = list[e];
    if (s < 0 || s >= g.pool_slots) {
      record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_BWD_PREP);
      continue;
    }
    atomicAdd(cnt + (size_t)h * g.pool_slots + s, 1);
  }
}

// ---------------------------------------------------------------------------- 2. scan
__global__ void __launch_bounds__(1024) bwd_scan_kernel(int ps, const int* __restrict__ cnt,
                                                       int* __restrict__ off, int* __restrict__ cur) {
  __shared__ int wsum[32];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (ps + 1023) / 1024;
  const int b0 = min(tid * per, ps), b1 = min(b0 + per, ps);
  const int* c = cnt + (size_t)h * ps;
  int local = 0;
  for (int i = b0; i < b1; ++i) local += c[i];
  int x = local;   // inclusive warp scan
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;
  }
  __syncthreads();
  int run = x - local + (warp > 0 ? wsum[warp - 1] : 0);   // exclusive prefix of this thread
  for (int i = b0; i < b1; ++i) {
    off[(size_t)h * ps + i] = run;
    cur[(size_t)h * ps + i] = 0;
    run += c[i];
  }
}

// ---------------------------------------------------------------------------- 3. fill
__global__ void __launch_bounds__(64) bwd_fill_kernel(BwdGeo g, const int* __restrict__ kv_slot,
                                                     const int* __restrict__ kv_cnt,
                                                     const int* __restrict__ off, int* __restrict__ cur,
                                                     int* __restrict__ inv) {
  const int r = blockIdx.x, h = blockIdx.y;
  int c = kv_cnt[(size_t)h * g.nq + r];
  c = min(max(c, 0), g.kv_ld);
  const int* list = kv_slot + ((size_t)h * g.nq + r) * g.kv_ld;
  for (int e = threadIdx.x; e < c; e += 64) {
    const int s = list[e];
    if (s < 0 || s >= g.pool_slots) continue;
    const size_t hs = (size_t)h * g.pool_slots + s;
    const int pos = off[hs] + atomicAdd(cur + hs, 1);
    inv[(size_t)h * g.nq * g.kv_ld + pos] = r * g.kv_ld + e;   // query block and list position
  }
}

__device__ __forceinline__ void wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              void* ws, int where, int kid) {
  if (*abort_flag) return;
  if (!mbar_wait(bar, parity, kWaitLimitNs)) {
    record_error(ws, PBSA_ERR_TIMEOUT, where, kid);
    *abort_flag = 1;
  }
}


// ---------------------------------------------------------------------------- shared pieces
constexpr int NT = 384;                                 // 12 warps
constexpr uint32_t REG_CTRL = 56, REG_WORK = 224;       // 128*56 + 256*224 = 384*168
constexpr uint32_t IDESC_BMN = idesc_bf16_f32(128, 128, 0, 1);    // B MN-major

// Merge two lists of keys (la[0..cA), lb[0..cB)): A's entries (mflag bit 0, plus bit 1 when
// also in B), then the B-only entries (bit 1), in order; mkey receives the keys.  pos_a /
// pos_b give each entry's position in its query block's list (nullptr: its index); mpa / mpb
// receive them per merged key (-1 where the key is absent from that list).  All NTH threads
// of the CTA call it; it ends with __syncthreads() and returns the merged count.
template <int NTH>
__device__ int merge_pair_pos(const int* la, const short* pos_a, int cA, const int* lb, const short* pos_b,
                              int cB, int* mkey, short* mpa, short* mpb, uint8_t* mflag, uint8_t* onlyb,
                              int* n_out) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < cA; i += NTH) {
    const int s = la[i];
    int pb = -1;
    for (int j = 0; j < cB; ++j)
      if (lb[j] == s) pb = pos_b ? pos_b[j] : j;
    mkey[i] = s;
    mpa[i] = (short)(pos_a ? pos_a[i] : i);
    mpb[i] = (short)pb;
    mflag[i] = pb >= 0 ? 3 : 1;
  }
  for (int j = tid; j < cB; j += NTH) {
    const int s = lb[j];
    bool in_a = false;
    for (int i = 0; i < cA; ++i) in_a |= (la[i] == s);
    onlyb[j] = in_a ? 0 : 1;
  }
  __syncthreads();
  if (warp == 0) {
    int pos = cA;
    for (int base = 0; base < cB; base += 32) {
      const int j = base + lane;
      const bool take = j < cB && onlyb[j];
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int at = pos + __popc(bal & ((1u << lane) - 1u));
        mkey[at] = lb[j];
        mpa[at] = -1;
        mpb[at] = (short)(pos_b ? pos_b[j] : j);
        mflag[at] = 2;
      }
      pos += __popc(bal);
    }
    if (lane == 0) *n_out = pos;
  }
  __syncthreads();
  return *n_out;
}

// ---------------------------------------------------------------------------- 4. dK, dV
// smem: K pair | V pair (2 panels x [128 keys][128 B] each) | KV_QST stages x (Q, dO tiles of one
// query block: 2 panels x [64 rows][128 B] each) | KV_QST x [log2-LSE | D] x 64 f32 | barriers |
// lists | per formation warp, a 4 KB buffer of dS^T rows on their way to the workspace
constexpr int KV_QST = 3;                                            // query-block stages
constexpr uint32_t KV_SM_K = 0, KV_SM_V = 32768, KV_SM_Q = 65536;    // Q stage s at +KV_STAGE*s
constexpr uint32_t KV_STAGE = 32768;                                 // Q (16 KB) + dO (16 KB)
constexpr uint32_t KV_SM_VEC = KV_SM_Q + KV_QST * KV_STAGE;          // [stage][lse2 | D][64] f32
constexpr uint32_t KV_SM_BAR = KV_SM_VEC + KV_QST * 512;
constexpr uint32_t KV_SM_MISC = KV_SM_BAR + 256;
constexpr uint32_t KV_SM_SLOT = KV_SM_MISC + 64;
constexpr uint32_t KV_SM_FLAG = KV_SM_SLOT + 4 * 1024;
constexpr uint32_t KV_SM_LA = KV_SM_FLAG + 1024;
constexpr uint32_t KV_SM_LB = KV_SM_LA + 4 * 512;
constexpr uint32_t KV_SM_ONLYB = KV_SM_LB + 4 * 512;
constexpr uint32_t KV_SM_TMP = KV_SM_ONLYB + 512;                    // int[512] sort scratch
constexpr uint32_t KV_SM_MPA = KV_SM_TMP + 4 * 512;                  // short[1024] positions in the
constexpr uint32_t KV_SM_MPB = KV_SM_MPA + 2 * 1024;                 //   query blocks' lists
constexpr uint32_t KV_SM_PLA = KV_SM_MPB + 2 * 1024;                 // short[512] each
constexpr uint32_t KV_SM_PLB = KV_SM_PLA + 2 * 512;
constexpr uint32_t KV_SM_STG = (KV_SM_PLB + 2 * 512 + 1023) & ~1023u;  // [8 warps][32 rows][128 B] dS^T
constexpr uint32_t KV_SMEM_BYTES = KV_SM_STG + 8 * 4096 + 1024;
static_assert(KV_SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
enum { KB_KVFULL = 0, KB_QFULL = 1, KB_QEMPTY = KB_QFULL + KV_QST, KB_SFULL = KB_QEMPTY + KV_QST /* [b] */,
       KB_PFULL = KB_SFULL + 2 /* [b], 128 arrivals */, KB_BFREE = KB_PFULL + 2 /* [b] */,
       KB_MMADONE = KB_BFREE + 2 /* 2 arrivals */, KB_NUM = KB_MMADONE + 1 };
constexpr uint32_t IDESC_N64 = idesc_bf16_f32(128, 64, 0, 0);   // S^T, dP^T of one query block

struct DkvParams {
  BwdGeo g;
  int kv_rows;
  int q_frames;
  float scale, scale_log2;
  const int* cnt;
  const int* off;
  const int* inv;
  const float* dvec;
  const float* lvec;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  __nv_bfloat16* ds;   // dS^T tiles, one per (head, query block, list position)
  void* ws;
};

// Sort src[0..n) ascending into dst by rank counting (n <= 512; entries distinct or not).
__device__ void sort_small(const int* src, int n, int* dst) {
  for (int i = threadIdx.x; i < n; i += NT) {
    const int x = src[i];
    int rk = 0;
    for (int j = 0; j < n; ++j) {
      const int y = src[j];
      rk += (y < x) | ((y == x) & (j < i));
    }
    dst[rk] = x;
  }
}

__global__ void __launch_bounds__(NT, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const DkvParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + KV_SM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + KV_SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + KV_SM_MISC + 4);
  int* n_merged_s = reinterpret_cast<int*>(sm + KV_SM_MISC + 8);
  int* mslot = reinterpret_cast<int*>(sm + KV_SM_SLOT);     // merged query blocks
  uint8_t* mflag = sm + KV_SM_FLAG;                         // bit k: attends KV slot 2p + k
  int* la = reinterpret_cast<int*>(sm + KV_SM_LA);
  int* lb = reinterpret_cast<int*>(sm + KV_SM_LB);
  int* tmp = reinterpret_cast<int*>(sm + KV_SM_TMP);
  const BwdGeo& g = prm.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, sA = 2 * blockIdx.x, sB = sA + 1;
  const bool hasB = sB < g.pool_slots;

  if (tid == 0) {
    for (int i = 0; i < KB_NUM; ++i) mbar_init(&bars[i], 1);
    mbar_init(&bars[KB_PFULL + 0], 128);
    mbar_init(&bars[KB_PFULL + 1], 128);
    mbar_init(&bars[KB_MMADONE], 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // the query blocks attending each of the two slots, sorted (the inverse lists are filled
  // with atomics, so their order is not reproducible until sorted)
  const size_t hb = (size_t)h * g.pool_slots;
  const int* invh = prm.inv + (size_t)h * g.nq * g.kv_ld;
  int cA = prm.cnt[hb + sA], cB = hasB ? prm.cnt[hb + sB] : 0;
  if (cA > 512 || cB > 512) {
    if (tid == 0) record_error(prm.ws, PBSA_ERR_UNSUPPORTED, max(cA, cB), K_BWD_KV);
    cA = min(cA, 512);
    cB = min(cB, 512);
  }
  for (int i = tid; i < cA; i += NT) tmp[i] = invh[prm.off[hb + sA] + i];
  __syncthreads();
  sort_small(tmp, cA, la);
  __syncthreads();
  if (hasB)
    for (int i = tid; i < cB; i += NT) tmp[i] = invh[prm.off[hb + sB] + i];
  __syncthreads();
  sort_small(tmp, cB, lb);
  __syncthreads();
  // split each entry into its query block and the slot's position in that block's list
  short* pla = reinterpret_cast<short*>(sm + KV_SM_PLA);
  short* plb = reinterpret_cast<short*>(sm + KV_SM_PLB);
  short* mpa = reinterpret_cast<short*>(sm + KV_SM_MPA);
  short* mpb = reinterpret_cast<short*>(sm + KV_SM_MPB);
  for (int i = tid; i < cA; i += NT) {
    const int v = la[i];
    la[i] = v / g.kv_ld;
    pla[i] = (short)(v - (v / g.kv_ld) * g.kv_ld);
  }
  for (int i = tid; i < cB; i += NT) {
    const int v = lb[i];
    lb[i] = v / g.kv_ld;
    plb[i] = (short)(v - (v / g.kv_ld) * g.kv_ld);
  }
  __syncthreads();
  const int n = merge_pair_pos<NT>(la, pla, cA, lb, plb, cB, mslot, mpa, mpb, mflag, sm + KV_SM_ONLYB,
                                   n_merged_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // one step per merged query block j; warpgroup (j & 1) forms P^T and dS^T of step j
  const int nsteps = n;
  float* vecs = reinterpret_cast<float*>(sm + KV_SM_VEC);  // [stage][lse2 | D][64]

  if (warp < 4) {
    setmaxnreg_dec<REG_CTRL>();
    if (warp == 0 && lane == 0 && nsteps > 0) {
      // ---- producer: the K, V pair once; then Q, dO, log2-LSE, D of one query block per step
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&domap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(&bars[KB_KVFULL], 65536);
      for (int b = 0; b < 2; ++b) {
        const int row0 = (b == 0 || hasB) ? (h * g.pool_slots + sA + b) * 64 : prm.kv_rows;
        for (int p = 0; p < 2; ++p) {
          tma_load_2d(sm + KV_SM_K + p * 16384 + b * 8192, &kmap, &bars[KB_KVFULL], p * 64, row0);
          tma_load_2d(sm + KV_SM_V + p * 16384 + b * 8192, &vmap, &bars[KB_KVFULL], p * 64, row0);
        }
      }
      int iss = 0;
      for (int j = 0; j < nsteps; ++j) {
        const int s = j % KV_QST;
        wait_or_abort(&bars[KB_QEMPTY + s], ((j / KV_QST) & 1) ^ 1, abort_flag, prm.ws, 1, K_BWD_KV);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&bars[KB_QFULL + s], KV_STAGE + 512);
        uint8_t* qdst = sm + KV_SM_Q + s * KV_STAGE;
        const int r = mslot[j];
        const int f = r / g.bpf, rem = r - f * g.bpf;
        const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
        for (int p = 0; p < 2; ++p) {
          tma_load_5d(qdst + p * 8192, &qmap, &bars[KB_QFULL + s], p * 64, h, tx * g.tw, ty * g.th, f);
          tma_load_5d(qdst + 16384 + p * 8192, &domap, &bars[KB_QFULL + s], p * 64, h, tx * g.tw, ty * g.th, f);
        }
        const size_t bi = ((size_t)h * g.nq + r) * BT;
        bulk_load(vecs + s * 128, prm.lvec + bi, 256, &bars[KB_QFULL + s]);
        bulk_load(vecs + s * 128 + 64, prm.dvec + bi, 256, &bars[KB_QFULL + s]);
        iss = j + 1;
      }
      if (*abort_flag) {
        mbar_wait(&bars[KB_KVFULL], 0, kWaitLimitNs);
        for (int j = (iss > KV_QST ? iss - KV_QST : 0); j < iss; ++j)
          mbar_wait(&bars[KB_QFULL + j % KV_QST], (j / KV_QST) & 1, kWaitLimitNs);
      }
    }
    // ---- MMA issuers.  TMEM: S^T[b] at 64 b, dP^T[b] at 128 + 64 b (keys on lanes, 64 queries
    // each), dV at 256, dK at 384; step j uses buffer b = j & 1.  Warp 1 issues S^T/dP^T(j)
    // as soon as buffer b is free (the dV/dK MMAs of step j-2 done); warp 3 issues the dV/dK
    // MMAs of every step in order, one thread, so dV and dK accumulate in a fixed order.
    if (warp == 1 && lane == 0 && nsteps > 0) {
      const uint64_t dk = sw128_desc(smem_u32(sm + KV_SM_K), 16, 1024);
      const uint64_t dv = sw128_desc(smem_u32(sm + KV_SM_V), 16, 1024);
      wait_or_abort(&bars[KB_KVFULL], 0, abort_flag, prm.ws, 2, K_BWD_KV);
      for (int j = 0; j < nsteps && !*abort_flag; ++j) {   // S^T = K Q_j^T, dP^T = V dO_j^T
        const int s = j % KV_QST, b = j & 1;
        if (j >= 2) wait_or_abort(&bars[KB_BFREE + b], ((j - 2) >> 1) & 1, abort_flag, prm.ws, 8, K_BWD_KV);
        wait_or_abort(&bars[KB_QFULL + s], (j / KV_QST) & 1, abort_flag, prm.ws, 3, K_BWD_KV);
        if (*abort_flag) break;
        tc_fence_after();
        const uint64_t dq_ = sw128_desc(smem_u32(sm + KV_SM_Q + s * KV_STAGE), 16, 1024);
        const uint64_t ddo = sw128_desc(smem_u32(sm + KV_SM_Q + s * KV_STAGE + 16384), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ka = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;   // K/V: 128-row panels
          const uint32_t kb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;    // Q/dO: 64-row panels
          mma_bf16_ss(tmem + b * 64, dk + ka, dq_ + kb, IDESC_N64, kk > 0 ? 1u : 0u);
          mma_bf16_ss(tmem + 128 + b * 64, dv + ka, ddo + kb, IDESC_N64, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[KB_SFULL + b]);
      }
      mma_commit(&bars[KB_MMADONE]);
      mbar_wait(&bars[KB_MMADONE], 0, kWaitLimitNs);
    }
    if (warp == 3 && lane == 0 && nsteps > 0) {
      for (int j = 0; j < nsteps && !*abort_flag; ++j) {
        const int s = j % KV_QST, b = j & 1;
        wait_or_abort(&bars[KB_PFULL + b], (j >> 1) & 1, abort_flag, prm.ws, 4, K_BWD_KV);
        if (*abort_flag) break;
        tc_fence_after();
        // dV += P^T dO_j, dK += dS^T Q_j: A from TMEM (bf16 pairs over S^T[b] / dP^T[b]), B =
        // the query block's 64 rows (d contiguous, two 64-column panels 8 KB apart).  S^T/dP^T(j)
        // completed before P(j) was formed, so these commits also cover them.
        const uint32_t q_base = smem_u32(sm + KV_SM_Q + s * KV_STAGE), do_base = q_base + 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_ts(tmem + 256, tmem + b * 64 + kk * 8, sw128_desc(do_base + kk * 2048, 8192, 1024), IDESC_BMN, acc);
          mma_bf16_ts(tmem + 384, tmem + 128 + b * 64 + kk * 8, sw128_desc(q_base + kk * 2048, 8192, 1024), IDESC_BMN, acc);
        }
        mma_commit(&bars[KB_QEMPTY + s]);
        mma_commit(&bars[KB_BFREE + b]);
      }
      mma_commit(&bars[KB_MMADONE]);
      mbar_wait(&bars[KB_MMADONE], 0, kWaitLimitNs);
    }
    __syncwarp();
  } else {
    setmaxnreg_inc<REG_WORK>();
    // ---- P^T and dS^T of the steps j = wg (mod 2); lanes are keys
    const int wg = (warp - 4) >> 2, wq = warp & 3;
    const int row = wq * 32 + lane, kh = row >> 6;   // key row, which slot of the pair
    const bool row_valid = kh == 0 || hasB;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float c = prm.scale_log2;
    const uint32_t tS = tmem + lane_off + wg * 64, tD = tmem + lane_off + 128 + wg * 64;
    for (int j = wg; j < nsteps; j += 2) {
      const bool v = row_valid && ((mflag[j] >> kh) & 1);
      const float* lse2 = vecs + (j % KV_QST) * 128;
      const float* dd = lse2 + 64;
      // the step's log2-LSE / D rows arrived with its Q-full barrier (TMA bulk copies)
      wait_or_abort(&bars[KB_QFULL + j % KV_QST], (j / KV_QST) & 1, abort_flag, prm.ws, 7, K_BWD_KV);
      wait_or_abort(&bars[KB_SFULL + wg], (j >> 1) & 1, abort_flag, prm.ws, 5, K_BWD_KV);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      tc_fence_after();
      // every column is finite (a missing block was loaded as zeros): read all, mask arithmetically
      uint32_t xs[2][32], xp[2][32];
      tmem_ld32(tS, xs[0]);
      tmem_ld32(tS + 32, xs[1]);
      tmem_ld32(tD, xp[0]);
      tmem_ld32(tD + 32, xp[1]);
      tmem_wait_ld();
      const float cs = v ? c : 0.f;
      uint32_t pp[32], pd[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const int c0 = q * 32 + 2 * e2;
          const float m0 = v ? -lse2[c0] : -INFINITY, m1 = v ? -lse2[c0 + 1] : -INFINITY;
          float a0, a1, t0, t1, d0, d1;
          a0 = fmaf(__uint_as_float(xs[q][2 * e2]), cs, m0);
          a1 = fmaf(__uint_as_float(xs[q][2 * e2 + 1]), cs, m1);
          const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
          t0 = __uint_as_float(xp[q][2 * e2]) - dd[c0];
          t1 = __uint_as_float(xp[q][2 * e2 + 1]) - dd[c0 + 1];
          fmul2(p0, p1, t0, t1, d0, d1);
          pp[q * 16 + e2] = pack_bf16(p0, p1);
          pd[q * 16 + e2] = pack_bf16(d0, d1);
        }
      }
      tmem_st32(tS, pp);
      tmem_st32(tD, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[KB_PFULL + wg]);
      // dS^T rows for the dQ pass, off the chain (this step's dV/dK MMAs run meanwhile): tile
      // (query block, position of this slot in its list), row = key, 64 query columns (128 B),
      // 16-byte chunk c of row k at ((c ^ (k & 7)) << 4) (the 128-byte swizzle, so that a plain
      // copy into aligned shared memory is an MMA operand).  The warp's 32 rows are staged in
      // shared memory and leave as one 4 KB bulk copy.  v is warp-uniform.
      if (v) {
        uint8_t* stg = sm + KV_SM_STG + (warp - 4) * 4096;
        if (lane == 0) bulk_wait_read<0>();   // this warp's previous copy has left the buffer
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((cc ^ (lane & 7)) << 4)) =
              make_uint4(pd[4 * cc], pd[4 * cc + 1], pd[4 * cc + 2], pd[4 * cc + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int pos = kh ? mpb[j] : mpa[j];
          bulk_store(prm.ds + ((((size_t)h * g.nq + mslot[j]) * g.kv_ld + pos) * BT + (wq & 1) * 32) * BT, stg, 4096);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();   // every dS^T copy of this warp has been written
    __syncwarp();
    // ---- epilogue: dV and dK = scale * (dS^T Q) rows of the pair's slots, warpgroup w
    // writes columns [64w, +64) of both
    if (nsteps > 0) wait_or_abort(&bars[KB_MMADONE], 0, abort_flag, prm.ws, 6, K_BWD_KV);
    if (row_valid && !__any_sync(0xffffffffu, *abort_flag != 0)) {
      const size_t base = (((size_t)h * g.pool_slots + sA + kh) * BT + (row & 63)) * D;
      uint4* dvd = reinterpret_cast<uint4*>(prm.dv + base) + wg * 8;
      uint4* dkd = reinterpret_cast<uint4*>(prm.dk + base) + wg * 8;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t a[32], b[32];
        if (nsteps > 0) {
          tmem_ld32(tmem + lane_off + 256 + wg * 64 + q * 32, a);
          tmem_ld32(tmem + lane_off + 384 + wg * 64 + q * 32, b);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) a[e2] = b[e2] = 0u;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t wa[4], wb[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int k0 = cc * 8 + 2 * e2;
            wa[e2] = pack_bf16(__uint_as_float(a[k0]), __uint_as_float(a[k0 + 1]));
            wb[e2] = pack_bf16(__uint_as_float(b[k0]) * prm.scale, __uint_as_float(b[k0 + 1]) * prm.scale);
          }
          dvd[q * 4 + cc] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          dkd[q * 4 + cc] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------- 5. dQ from dS
// dQ = scale * dS K with the dS^T tiles the dK/dV pass stored: one CTA per (head, pair of
// query blocks), 128 threads.  The two lists are merged; merged entry e brings the K block of
// its slot and the dS^T tiles of the two query blocks (a block that does not attend the slot
// gets a tile loaded out of bounds, i.e. zeros) into one stage; four MMAs (K = 16 keys each)
// accumulate dQ (128 query rows x 128 d) in TMEM, in the merged order (deterministic).
//   A = dS (M = the pair's 128 queries, K = keys): the two tiles, query-contiguous (MN-major),
//   B = K  (K = keys, N = d): d-contiguous (MN-major).
constexpr int DQ_NT = 128;
constexpr int DS_STAGES = 3;
constexpr uint32_t DS_STAGE = 32768;                            // K block (16 KB) + two dS^T tiles
constexpr uint32_t DS_SM_BAR = DS_STAGES * DS_STAGE;
constexpr uint32_t DS_SM_MISC = DS_SM_BAR + 128;
constexpr uint32_t DS_SM_SLOT = DS_SM_MISC + 64;                // int[1024] merged slots
constexpr uint32_t DS_SM_MPA = DS_SM_SLOT + 4 * 1024;           // short[1024] positions in list A
constexpr uint32_t DS_SM_MPB = DS_SM_MPA + 2 * 1024;            // short[1024] positions in list B
constexpr uint32_t DS_SM_FLAG = DS_SM_MPB + 2 * 1024;           // uint8[1024]
constexpr uint32_t DS_SM_LA = DS_SM_FLAG + 1024;                // int[512]
constexpr uint32_t DS_SM_LB = DS_SM_LA + 4 * 512;               // int[512]
constexpr uint32_t DS_SM_ONLYB = DS_SM_LB + 4 * 512;            // uint8[512]
constexpr uint32_t DS_SMEM_BYTES = DS_SM_ONLYB + 512 + 1024;
static_assert(2 * DS_SMEM_BYTES <= 228 * 1024, "two CTAs per SM");
enum { DB_FULL = 0, DB_EMPTY = DB_FULL + DS_STAGES, DB_DONE = DB_EMPTY + DS_STAGES, DB_NUM = DB_DONE + 1 };
static_assert(DB_NUM * 8 <= 128, "barrier area");
constexpr uint32_t IDESC_AMN_BMN = idesc_bf16_f32(128, 128, 1, 1);

struct DqsParams {
  BwdGeo g;
  int kv_rows;   // first out-of-bounds row of the K pool map
  float scale;
  const __nv_bfloat16* ds;     // dS^T tiles (128-byte swizzled rows)
  const __nv_bfloat16* zero;   // one all-zero tile, for a query block that does not attend
  const int* kv_slot;
  const int* kv_cnt;
  __nv_bfloat16* dq;
  void* ws;
};

__global__ void __launch_bounds__(DQ_NT, 2)
    bwd_dqs_kernel(const __grid_constant__ CUtensorMap kmap, const DqsParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + DS_SM_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + DS_SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + DS_SM_MISC + 4);
  int* n_merged_s = reinterpret_cast<int*>(sm + DS_SM_MISC + 8);
  int* mslot = reinterpret_cast<int*>(sm + DS_SM_SLOT);
  short* mpa = reinterpret_cast<short*>(sm + DS_SM_MPA);
  short* mpb = reinterpret_cast<short*>(sm + DS_SM_MPB);
  int* la = reinterpret_cast<int*>(sm + DS_SM_LA);
  int* lb = reinterpret_cast<int*>(sm + DS_SM_LB);
  const BwdGeo& g = prm.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, rA = 2 * blockIdx.x, rB = rA + 1;
  const bool hasB = rB < g.nq;

  if (tid == 0) {
    for (int i = 0; i < DB_NUM; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 128);
    tmem_relinquish();
  }
  int cA = prm.kv_cnt[(size_t)h * g.nq + rA];
  int cB = hasB ? prm.kv_cnt[(size_t)h * g.nq + rB] : 0;
  cA = min(max(cA, 0), min(g.kv_ld, 512));
  cB = min(max(cB, 0), min(g.kv_ld, 512));
  const int* listA = prm.kv_slot + ((size_t)h * g.nq + rA) * g.kv_ld;
  const int* listB = prm.kv_slot + ((size_t)h * g.nq + (hasB ? rB : rA)) * g.kv_ld;
  for (int i = tid; i < cA; i += DQ_NT) la[i] = listA[i];
  for (int i = tid; i < cB; i += DQ_NT) lb[i] = listB[i];
  __syncthreads();
  const int n = merge_pair_pos<DQ_NT>(la, nullptr, cA, lb, nullptr, cB, mslot, mpa, mpb, sm + DS_SM_FLAG,
                                      sm + DS_SM_ONLYB, n_merged_s);
  for (int i = tid; i < n; i += DQ_NT) {
    const int s = mslot[i];
    if (s < 0 || s >= g.pool_slots) {   // no dS was stored for it: zeros on both halves
      record_error(prm.ws, PBSA_ERR_DEVICE_INDEX, s, K_BWD_Q);
      mslot[i] = -1;
      mpa[i] = -1;
      mpb[i] = -1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0 && n > 0) {
    // ---- producer: per merged entry, K block + the two dS^T tiles into one stage
    tma_prefetch_desc(&kmap);
    int iss = 0;
    for (int e = 0; e < n; ++e) {
      const int st = e % DS_STAGES;
      wait_or_abort(&bars[DB_EMPTY + st], ((e / DS_STAGES) & 1) ^ 1, abort_flag, prm.ws, 1, K_BWD_Q);
      if (*abort_flag) break;
      mbar_arrive_expect_tx(&bars[DB_FULL + st], DS_STAGE);
      uint8_t* dst = sm + st * DS_STAGE;
      const int slot = mslot[e];
      const int krow = slot >= 0 ? (h * g.pool_slots + slot) * BT : prm.kv_rows;
      tma_load_2d(dst, &kmap, &bars[DB_FULL + st], 0, krow);
      tma_load_2d(dst + 8192, &kmap, &bars[DB_FULL + st], 64, krow);
      const int pa = mpa[e], pb = mpb[e];
      const __nv_bfloat16* ta = pa >= 0 ? prm.ds + (((size_t)h * g.nq + rA) * g.kv_ld + pa) * BT * BT : prm.zero;
      const __nv_bfloat16* tb = (pb >= 0 && hasB) ? prm.ds + (((size_t)h * g.nq + rB) * g.kv_ld + pb) * BT * BT : prm.zero;
      bulk_load(dst + 16384, ta, 8192, &bars[DB_FULL + st]);
      bulk_load(dst + 24576, tb, 8192, &bars[DB_FULL + st]);
      iss = e + 1;
    }
    if (*abort_flag)
      for (int e = (iss > DS_STAGES ? iss - DS_STAGES : 0); e < iss; ++e)
        mbar_wait(&bars[DB_FULL + e % DS_STAGES], (e / DS_STAGES) & 1, kWaitLimitNs);
  }
  if (warp == 1 && lane == 0 && n > 0) {
    // ---- MMA issuer: dQ += dS_e K_e, in merged order
    for (int e = 0; e < n && !*abort_flag; ++e) {
      const int st = e % DS_STAGES;
      wait_or_abort(&bars[DB_FULL + st], (e / DS_STAGES) & 1, abort_flag, prm.ws, 2, K_BWD_Q);
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t base = smem_u32(sm + st * DS_STAGE);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem, sw128_desc(base + 16384 + kk * 2048, 8192, 1024),
                    sw128_desc(base + kk * 2048, 8192, 1024), IDESC_AMN_BMN, (e > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars[DB_EMPTY + st]);
    }
    mma_commit(&bars[DB_DONE]);
  }
  __syncwarp();
  // ---- epilogue: every warp, its 32 TMEM lanes = query rows
  const int row = warp * 32 + lane, half = row >> 6;
  const bool row_valid = half == 0 || hasB;
  if (n > 0) wait_or_abort(&bars[DB_DONE], 0, abort_flag, prm.ws, 3, K_BWD_Q);
  tc_fence_after();
  if (row_valid && !__any_sync(0xffffffffu, *abort_flag != 0)) {
    const int r = half ? rB : rA;
    const size_t t = token_of(g, r, row & 63);
    uint4* dst = reinterpret_cast<uint4*>(prm.dq + (t * g.H + h) * D);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t ov[32];
      if (n > 0) {
        tmem_ld32(tmem + lane_off + q * 32, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) ov[e2] = 0u;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t wv[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)
          wv[e2] = pack_bf16(__uint_as_float(ov[cc * 8 + 2 * e2]) * prm.scale,
                             __uint_as_float(ov[cc * 8 + 2 * e2 + 1]) * prm.scale);
        dst[q * 4 + cc] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

size_t attend_bwd_ws_bytes(const Geo& g, int q_frames, int pool_slots, int kv_ld) {
  return bwd_layout(g.H, q_frames * g.bpf, pool_slots, kv_ld).end;
}

cudaError_t launch_attend_bwd(const Geo& gg, const void* q, int q_frames, const void* k_pool,
                              const void* v_pool, int pool_slots, const int* kv_slot,
                              const int* kv_cnt, int kv_ld, const void* o, const void* d_o,
                              const float* lse, void* dq, void* dk_pool, void* dv_pool, void* ws,
                              cudaStream_t st) {
  if (gg.d != D || gg.dtype != PBSA_BF16) return cudaErrorNotSupported;
  BwdGeo g;
  g.H = gg.H;
  g.nq = q_frames * gg.bpf;
  g.kv_ld = kv_ld;
  g.pool_slots = pool_slots;
  g.bpf = gg.bpf;
  g.tpr = gg.tpr;
  g.tpf = gg.tpf;
  g.fw = gg.fw;
  g.th = gg.th;
  g.tw = gg.tw;
  const BwdLayout L = bwd_layout(g.H, g.nq, pool_slots, kv_ld);
  char* base = static_cast<char*>(ws);
  float* dvec = reinterpret_cast<float*>(base + L.dvec);
  float* lvec = reinterpret_cast<float*>(base + L.lvec);
  int* cnt = reinterpret_cast<int*>(base + L.cnt);
  int* off = reinterpret_cast<int*>(base + L.off);
  int* cur = reinterpret_cast<int*>(base + L.cur);
  int* inv = reinterpret_cast<int*>(base + L.inv);
  __nv_bfloat16* ds = reinterpret_cast<__nv_bfloat16*>(base + L.ds);
  __nv_bfloat16* dzero = reinterpret_cast<__nv_bfloat16*>(base + L.zero);
  if (kv_ld > 32767) return cudaErrorNotSupported;
  cudaError_t e;
  if ((e = cudaMemsetAsync(dzero, 0, BT * BT * 2, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(cnt, 0, (size_t)g.H * pool_slots * 4, st)) != cudaSuccess) return e;

  CUtensorMap qmap, domap, kmap, vmap;
  {
    const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)g.H, (cuuint64_t)gg.fw, (cuuint64_t)gg.fh,
                                (cuuint64_t)q_frames};
    const cuuint64_t row = (cuuint64_t)D * 2;
    const cuuint64_t strides[4] = {row, row * g.H, row * g.H * gg.fw, row * g.H * gg.fw * gg.fh};
    const cuuint32_t box[5] = {64, 1, (cuuint32_t)gg.tw, (cuuint32_t)gg.th, 1};
    if (!encode_bf16(&qmap, q, 5, dims, strides, box)) return cudaErrorNotSupported;
    if (!encode_bf16(&domap, d_o, 5, dims, strides, box)) return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)g.H * pool_slots * BT};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 64};
    if (!encode_bf16(&kmap, k_pool, 2, dims, strides, box)) return cudaErrorNotSupported;
    if (!encode_bf16(&vmap, v_pool, 2, dims, strides, box)) return cudaErrorNotSupported;
  }
  const float scale = gg.scale;
  bwd_prep_kernel<<<dim3(g.nq, g.H), 64, 0, st>>>(g, static_cast<const __nv_bfloat16*>(o),
                                                   static_cast<const __nv_bfloat16*>(d_o), lse, kv_slot,
                                                   kv_cnt, dvec, lvec, cnt, ws);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_scan_kernel<<<g.H, 1024, 0, st>>>(pool_slots, cnt, off, cur);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_fill_kernel<<<dim3(g.nq, g.H), 64, 0, st>>>(g, kv_slot, kv_cnt, off, cur, inv);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  DkvParams kp;
  kp.g = g;
  kp.kv_rows = g.H * pool_slots * BT;
  kp.q_frames = q_frames;
  kp.scale = scale;
  kp.scale_log2 = scale * LOG2E;
  kp.cnt = cnt;
  kp.off = off;
  kp.inv = inv;
  kp.dvec = dvec;
  kp.lvec = lvec;
  kp.dk = static_cast<__nv_bfloat16*>(dk_pool);
  kp.dv = static_cast<__nv_bfloat16*>(dv_pool);
  kp.ds = ds;
  kp.ws = ws;
  if ((e = set_smem_once((const void*)bwd_dkdv_kernel, (int)KV_SMEM_BYTES)) != cudaSuccess) return e;
  bwd_dkdv_kernel<<<dim3((pool_slots + 1) / 2, g.H), NT, KV_SMEM_BYTES, st>>>(qmap, domap, kmap, vmap, kp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  DqsParams dp;
  dp.g = g;
  dp.kv_rows = g.H * pool_slots * BT;
  dp.ds = ds;
  dp.zero = dzero;
  dp.scale = scale;
  dp.kv_slot = kv_slot;
  dp.kv_cnt = kv_cnt;
  dp.dq = static_cast<__nv_bfloat16*>(dq);
  dp.ws = ws;
  if ((e = set_smem_once((const void*)bwd_dqs_kernel, (int)DS_SMEM_BYTES)) != cudaSuccess) return e;
  bwd_dqs_kernel<<<dim3((g.nq + 1) / 2, g.H), DQ_NT, DS_SMEM_BYTES, st>>>(kmap, dp);
  return cudaGetLastError();
}

}  // namespace pbsa
