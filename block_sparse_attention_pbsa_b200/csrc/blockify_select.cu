// a1 + a2 fused -- blockify of the query chunk, coarse scores and top-k in one pass.
//
// Sparse Forcing (gist.science, English 2.C "Local Sparsity" and 2.E "PBSA Kernel"; Chinese
// 2.2 "块化压缩"): each query block is summarised by the mean of its 64 tokens and routed
// to the top-k local blocks by the score scale * <qbar, kbar>.  Blockify and selection are
// the same two steps as pbsa_blockify + pbsa_score_select; here one CTA does both for one
// (query block, head), so Q is read from HBM once and qbar never makes a round trip.
//
// One CTA of 256 threads per (query block, head):
//  1. every thread issues its 16-byte loads of the block's tokens (same row/column split
//     and summation order as the blockify kernel, so qbar is bit-identical to it) together
//     with the candidate list;
//  2. qbar is reduced in shared memory in a fixed order and written to q_reps;
//  3. warp w scores candidates w, w+8, ...: each lane holds d/32 elements of qbar and of the
//     candidate's kbar row (coalesced row loads, several candidates in flight), and a
//     butterfly shuffle sums the lane partials (fixed order: deterministic);
//  4. ranks on (score desc, gid asc, position asc): lists of up to 256 candidates are sorted
//     by a bitonic network in shared memory (one element per thread), longer ones ranked by
//     counting; the first k are written behind the copied prefix, then an optional suffix
//     list shared by every row (e.g. the chunk's own blocks).
//
// Hierarchical variant (Light Forcing, papernotes.org notes, "方法详解" HSA, steps (1)-(3), as a
// selection policy over the local window): between 3 and 4, the candidates (whole frames,
// frame slot = position / bpf) get frame scores = the mean of their blocks' scores (the score
// of the frame's mean-pooled representative, by linearity), summed in block order; the
// n_recent latest frames are always chosen, plus the top_frames best others (score
// descending, the earlier frame on ties); blocks of the other frames leave the ranking.
//
// Chunk-causal variant (the trainable path: English 2.D "Training Strategy", the model is trained
// with the same dynamic sparse cache): sequences are folded into the frame axis and the pool holds
// their blocks in order (slot = global block id).  Query block r of sequence s, chunk c, attends
// its own chunk; for c >= 1 also the sequence's sink blocks and the top-k blocks, by the same
// coarse score, among the sequence's earlier non-sink blocks.  The lists come from r alone, so
// no candidate list is read; the selection is the flat top-k above.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr int BS_THREADS = 256;
constexpr int BS_BATCH = 9;   // candidates per warp in flight (144 candidates: two rounds)
constexpr int SORT_N = 256;   // candidate lists up to this long are ranked by a bitonic sort
constexpr int HSA_MAX_FRAMES = 256;

// Chunk-causal lists (seq_blocks = 0: the lists come from the call's arguments).
struct Causal {
  int seq_blocks;    // blocks per sequence
  int chunk_blocks;  // blocks per chunk
  int sink_blocks;   // leading blocks of a sequence that every later chunk attends
  int n_chunks;      // chunks per sequence (the last may be shorter)
  int groups;        // 8-query-block groups per chunk (the 8-block kernel's grid)
};

// Lists of query block r: candidates [cbase, cbase + ncand), prefix [pbase, pbase + pc),
// suffix [sbase, sbase + sn) -- all slots = global block ids.
struct CausalLists {
  int cbase, ncand, pbase, pc, sbase, sn;
};
__device__ __forceinline__ CausalLists causal_lists(const Causal& cz, int r) {
  const int sq0 = (r / cz.seq_blocks) * cz.seq_blocks;
  const int c = (r - sq0) / cz.chunk_blocks;
  const int cs = sq0 + c * cz.chunk_blocks;
  const int ce = min(cs + cz.chunk_blocks, sq0 + cz.seq_blocks);
  CausalLists l;
  l.cbase = sq0 + cz.sink_blocks;
  l.ncand = c == 0 ? 0 : cs - l.cbase;
  l.pbase = sq0;
  l.pc = c == 0 ? 0 : cz.sink_blocks;
  l.sbase = cs;
  l.sn = ce - cs;
  return l;
}

template <typename T>
__device__ __forceinline__ void add_chunk16(float* acc, const uint4& v);
template <>
__device__ __forceinline__ void add_chunk16<float>(float* acc, const uint4& v) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void add_chunk16<__nv_bfloat16>(float* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// d/32 consecutive fp32 values of a row, as one vector load
template <int N> struct Vec;
template <> struct Vec<4> { using type = float4; };
template <> struct Vec<2> { using type = float2; };
template <> struct Vec<1> { using type = float; };
__device__ __forceinline__ void vec_to(const float4& v, float* o) { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
__device__ __forceinline__ void vec_to(const float2& v, float* o) { o[0] = v.x; o[1] = v.y; }
__device__ __forceinline__ void vec_to(const float& v, float* o) { o[0] = v; }

template <typename T, int D, bool HSA, bool CAUSAL>
__global__ void __launch_bounds__(BS_THREADS) blockify_select_kernel(
    const T* __restrict__ x, Geo g, int nq, float* __restrict__ q_reps,
    const float* __restrict__ k_reps, int pool_slots, const int* __restrict__ cand_slot,
    const int* __restrict__ cand_gid, int ncap, int k, const int* __restrict__ prefix_slot,
    const int* __restrict__ prefix_cnt, int prefix_ld, int* __restrict__ out_slot,
    int* __restrict__ out_cnt, int out_ld, float* __restrict__ out_score, int top_frames,
    int n_recent, const int* __restrict__ suffix_slot, int suffix_n, Causal cz, void* ws) {
  constexpr int VEC = 16 / sizeof(T);   // token elements per 16-byte chunk
  constexpr int CPR = D / VEC;          // chunks per token row
  constexpr int RPP = BS_THREADS / CPR; // rows per pass
  constexpr int PASSES = BT / RPP;
  constexpr int PL = D / 32;            // qbar / kbar elements per lane
  using V = typename Vec<PL>::type;
  __shared__ float part[RPP][D];
  __shared__ float qb[D];
  extern __shared__ uint64_t dyn[];
  uint64_t* key = dyn;                                          // [ncap]
  float* sc = reinterpret_cast<float*>(key + ncap);             // [ncap]
  int* gid = reinterpret_cast<int*>(sc + ncap);                 // [ncap]
  int* slot = gid + ncap;                                       // [ncap]

  const int r = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  CausalLists cl = {0, ncap, 0, 0, 0, suffix_n};
  if (CAUSAL) cl = causal_lists(cz, r);
  const int ncand = cl.ncand;

  // ---- 1. loads: the block's tokens and the candidate list
  const int f = r / g.bpf, rem = r - f * g.bpf;
  const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
  const int c = tid % CPR, rg = tid / CPR;
  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int row = rg + p * RPP;
    const int ly = row / g.tw, lx = row - ly * g.tw;
    const size_t t = (size_t)f * g.tpf + (size_t)(ty * g.th + ly) * g.fw + tx * g.tw + lx;
    v[p] = __ldg(reinterpret_cast<const uint4*>(x + (t * g.H + h) * D) + c);
  }
  for (int j = tid; j < ncand; j += BS_THREADS) {
    gid[j] = CAUSAL ? cl.cbase + j : cand_gid[(size_t)h * ncap + j];
    slot[j] = CAUSAL ? cl.cbase + j : cand_slot[(size_t)h * ncap + j];
  }
  // ---- 2. qbar (fixed-order sums, as in the blockify kernel)
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
#pragma unroll
  for (int p = 0; p < PASSES; ++p) add_chunk16<T>(acc, v[p]);
#pragma unroll
  for (int i = 0; i < VEC; ++i) part[rg][c * VEC + i] = acc[i];
  __syncthreads();
  for (int e = tid; e < D; e += BS_THREADS) {
    float s = 0.f;
#pragma unroll 4
    for (int q = 0; q < RPP; ++q) s += part[q][e];
    s *= (1.0f / BT);
    qb[e] = s;
    q_reps[((size_t)h * nq + r) * D + e] = s;
  }
  __syncthreads();

  // ---- 3. scores: warp per candidate, lanes over d, BS_BATCH candidates in flight
  float ql[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) ql[i] = qb[lane * PL + i];
  constexpr int NW = BS_THREADS / 32;
  for (int c0 = warp; c0 < ncand; c0 += NW * BS_BATCH) {
    float kv[BS_BATCH][PL];
    bool ok[BS_BATCH];
#pragma unroll
    for (int b = 0; b < BS_BATCH; ++b) {
      const int cc = c0 + b * NW;
      const int s = cc < ncand ? slot[cc] : -1;
      ok[b] = cc < ncand && s >= 0 && s < pool_slots;
      if (ok[b]) {
        const V w = __ldg(reinterpret_cast<const V*>(k_reps + ((size_t)h * pool_slots + s) * D) + lane);
        vec_to(w, kv[b]);
      } else {
#pragma unroll
        for (int i = 0; i < PL; ++i) kv[b][i] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < BS_BATCH; ++b) {
      const int cc = c0 + b * NW;
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < PL; ++i) a = fmaf(ql[i], kv[b][i], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0 && cc < ncand) {
        float val = a * g.scale;
        if (!ok[b]) {
          if (r == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, slot[cc], K_SCORE);
          val = -INFINITY;
        }
        if (isnan(val)) val = -INFINITY;
        sc[cc] = val;
        key[cc] = rank_key(val, gid[cc]);
      }
    }
  }

  // ---- 4. prefix, count, ranks
  int pc = cl.pc;
  if (!CAUSAL) {
    pc = prefix_cnt ? prefix_cnt[h] : 0;
    if (pc < 0 || pc > prefix_ld) {
      if (tid == 0 && r == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, pc, K_SCORE);
      pc = pc < 0 ? 0 : prefix_ld;
    }
  }
  const int sn = cl.sn;
  const size_t o = (size_t)h * nq + r;
  for (int j = tid; j < pc; j += BS_THREADS)
    out_slot[o * out_ld + j] = CAUSAL ? cl.pbase + j : prefix_slot[(size_t)h * prefix_ld + j];
  int kk = min(k, ncand);
  __syncthreads();
  if (HSA) {
    // frame level: mean of each frame's block scores (block order), rank the non-recent
    // frames, drop the blocks of frames not chosen from the ranking (key 0 sorts last)
    __shared__ float fsc[HSA_MAX_FRAMES];
    __shared__ int fchosen[HSA_MAX_FRAMES], n_elig_s;
    const int bpf = g.bpf, nf = ncand / bpf, first_recent = max(0, nf - n_recent);
    for (int t = tid; t < nf; t += BS_THREADS) {
      float a = 0.f;
      for (int b = 0; b < bpf; ++b) a += sc[t * bpf + b];
      fsc[t] = a * (1.0f / (float)bpf);
    }
    __syncthreads();
    for (int t = tid; t < nf; t += BS_THREADS) {
      int rank = 0;
      if (t < first_recent)
        for (int t2 = 0; t2 < first_recent; ++t2)
          rank += (fsc[t2] > fsc[t]) | ((fsc[t2] == fsc[t]) & (t2 < t));
      fchosen[t] = t >= first_recent || rank < top_frames;
    }
    if (tid == 0) n_elig_s = 0;
    __syncthreads();
    for (int cc = tid; cc < ncand; cc += BS_THREADS) {
      if (fchosen[cc / bpf]) atomicAdd(&n_elig_s, 1);
      else key[cc] = 0ull;
    }
    __syncthreads();
    kk = min(k, n_elig_s);
  }
  if (tid == 0) out_cnt[o] = pc + kk + sn;
  for (int j = tid; j < sn; j += BS_THREADS)
    out_slot[o * out_ld + pc + kk + j] = CAUSAL ? cl.sbase + j : suffix_slot[j];
  if (ncand <= SORT_N) {
    // bitonic sort, descending on (key, -position); padding sorts last
    __shared__ uint64_t skey[SORT_N];
    __shared__ int spos[SORT_N];
    skey[tid] = tid < ncand ? key[tid] : 0ull;
    spos[tid] = tid < ncand ? tid : SORT_N + tid;
    __syncthreads();
    for (int kk2 = 2; kk2 <= SORT_N; kk2 <<= 1) {
      for (int j = kk2 >> 1; j > 0; j >>= 1) {
        const int ixj = tid ^ j;
        const uint64_t a = skey[tid], b = skey[ixj];
        const int pa = spos[tid], pb = spos[ixj];
        // does (b, pb) come before (a, pa) in the descending order?
        const bool b_first = b > a || (b == a && pb < pa);
        const bool lower = tid < ixj;
        const bool desc = (tid & kk2) == 0;   // this subsequence is sorted descending
        const bool take_b = (lower == desc) ? b_first : !b_first;
        __syncthreads();
        if (take_b) {
          skey[tid] = b;
          spos[tid] = pb;
        }
        __syncthreads();
      }
    }
    if (tid < kk) {
      const int cc = spos[tid];
      out_slot[o * out_ld + pc + tid] = slot[cc];
      if (out_score) out_score[o * k + tid] = sc[cc];
    }
  } else {
    for (int cc = tid; cc < ncand; cc += BS_THREADS) {
      const uint64_t kc = key[cc];
      int rank = 0;
#pragma unroll 8
      for (int c2 = 0; c2 < ncand; ++c2) {
        const uint64_t k2 = key[c2];
        rank += (int)(k2 > kc) | ((int)(k2 == kc) & (int)(c2 < cc));
      }
      if (rank < kk) {
        out_slot[o * out_ld + pc + rank] = slot[cc];
        if (out_score) out_score[o * k + rank] = sc[cc];
      }
    }
  }
}

// ---------------------------------------------------------------------------- 8-block form
// The flat policy with up to 256 candidates: one CTA of 512 threads per (head, 8 query blocks).
//  1. every thread issues the 16-byte token loads of its four (block, column chunk, row set)
//     shares -- blockify's split, so each block's mean is summed in blockify's order -- and
//     reads the candidate list; the candidates' representatives are then requested into
//     shared memory (cp.async, rows padded to d + 4 floats) while the token loads are still
//     in flight;
//  2. the 8 pooled queries (rows 0..7 of an m16 tile) times the candidates on the tensor
//     cores: m16n8k8 TF32 MMAs with each fp32 operand split into a TF32 high part and a TF32
//     residual (hi*hi + hi*lo + lo*hi, fp32 accumulation: fp32-level accuracy);
//  3. warp b selects query block b's k best: a radix search on the 64-bit ranking keys finds
//     the k-th largest key -- it stops as soon as exactly k keys lie at or above the
//     threshold -- and the chosen keys are put in order by a bitonic sort across the warp
//     (k <= 32) or by counting (larger k).
constexpr int S8_R = 8, S8_THREADS = 512;

template <typename T, int D>
struct S8Layout {
  static constexpr int VEC = 16 / (int)sizeof(T);
  static constexpr int CPR = D / VEC;             // chunks per token row
  static constexpr int RPP = BS_THREADS / CPR;    // rows per pass of a 256-thread blockify share
  static constexpr int KS = D + 4;                // padded representative row (floats)
  static __host__ __device__ size_t part_bytes() { return (size_t)S8_R * RPP * D * 4; }
  static __host__ __device__ int ncs(int ncand) { return ((ncand + 7) / 8) * 8 + 8; }   // score row stride
  // part | kb [ncand][KS] | qs [16][KS] | ss [S8_R][ncs] | slot, gid [ncand]
  static __host__ __device__ size_t bytes(int ncand) {
    return part_bytes() + (size_t)ncand * KS * 4 + (size_t)16 * KS * 4 + (size_t)S8_R * ncs(ncand) * 4 +
           (size_t)ncand * 8 + 16;
  }
};

template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(S8_THREADS) blockify_select8_kernel(
    const T* __restrict__ x, Geo g, int nq, float* __restrict__ q_reps,
    const float* __restrict__ k_reps, int pool_slots, const int* __restrict__ cand_slot,
    const int* __restrict__ cand_gid, int ncap, int k, const int* __restrict__ prefix_slot,
    const int* __restrict__ prefix_cnt, int prefix_ld, int* __restrict__ out_slot,
    int* __restrict__ out_cnt, int out_ld, float* __restrict__ out_score,
    const int* __restrict__ suffix_slot, int suffix_n, Causal cz, void* ws) {
  using L = S8Layout<T, D>;
  constexpr int VEC = L::VEC, CPR = L::CPR, RPP = L::RPP, KS = L::KS;
  constexpr int PASSES = BT / RPP;
  constexpr int NW = S8_THREADS / 32;
  constexpr int CH = D / 4;   // 16-byte chunks of a representative row
  extern __shared__ __align__(16) float sm8[];
  float* part = sm8;                                        // [S8_R][RPP][D]
  float* kb = part + L::part_bytes() / 4;                   // [ncap][KS]
  float* qs = kb + (size_t)ncap * KS;                       // [16][KS]
  float* ss = qs + 16 * KS;                                 // [S8_R][ncs]
  const int ncs = L::ncs(ncap);
  int* slot = reinterpret_cast<int*>(ss + S8_R * ncs);      // [ncap]
  int* gid = slot + ncap;                                   // [ncap]

  const int h = blockIdx.y;
  int r0 = blockIdx.x * S8_R, nr = min(S8_R, nq - r0);
  CausalLists cl = {0, ncap, 0, 0, 0, suffix_n};
  if (CAUSAL) {
    // CTA = (sequence, chunk, group of 8 query blocks inside the chunk): a group never spans
    // two chunks, so its 8 rows share one candidate list
    const int per_seq = cz.n_chunks * cz.groups;
    const int seq = blockIdx.x / per_seq, rest = blockIdx.x - seq * per_seq;
    const int c = rest / cz.groups;
    const int cs = seq * cz.seq_blocks + c * cz.chunk_blocks;
    r0 = cs + (rest - c * cz.groups) * S8_R;
    cl = causal_lists(cz, cs);
    nr = min(S8_R, cl.sbase + cl.sn - r0);
    if (nr <= 0) return;   // a group past the end of a shorter last chunk (whole CTA, no barrier yet)
  }
  const int ncand = cl.ncand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- 1. token loads: thread = (virtual blockify thread vt, block parity); blocks bp, bp+2, ..
  const int vt = tid % BS_THREADS, bp = tid / BS_THREADS;
  const int c = vt % CPR, rg = vt / CPR;
  uint4 v[S8_R / 2][PASSES];
#pragma unroll
  for (int u = 0; u < S8_R / 2; ++u) {
    const int b = bp + 2 * u;
    const int r = r0 + min(b, nr - 1);     // a missing block re-reads the last one (not stored)
    const int f = r / g.bpf, rem = r - f * g.bpf;
    const int ty = rem / g.tpr, tx = rem - ty * g.tpr;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int row = rg + p * RPP;
      const int ly = row / g.tw, lx = row - ly * g.tw;
      const size_t t = (size_t)f * g.tpf + (size_t)(ty * g.th + ly) * g.fw + tx * g.tw + lx;
      v[u][p] = __ldg(reinterpret_cast<const uint4*>(x + (t * g.H + h) * D) + c);
    }
  }
  for (int j = tid; j < ncand; j += S8_THREADS) {
    gid[j] = CAUSAL ? cl.cbase + j : cand_gid[(size_t)h * ncap + j];
    slot[j] = CAUSAL ? cl.cbase + j : cand_slot[(size_t)h * ncap + j];
  }
  for (int i = tid; i < 8 * CH; i += S8_THREADS)   // query rows 8..15 of the MMA tile are zero
    reinterpret_cast<float4*>(qs + (8 + i / CH) * KS)[i % CH] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  {
    const float* krep_h = k_reps + (size_t)h * pool_slots * D;
    for (int i = tid; i < ncand * CH; i += S8_THREADS) {
      const int j = i / CH, e = i - j * CH;
      const int s = slot[j];
      if (s >= 0 && s < pool_slots) cp_async16(kb + j * KS + 4 * e, krep_h + (size_t)s * D + 4 * e);
    }
  }
#pragma unroll
  for (int u = 0; u < S8_R / 2; ++u) {
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) add_chunk16<T>(acc, v[u][p]);
    float* pr = part + ((bp + 2 * u) * RPP + rg) * D + c * VEC;
#pragma unroll
    for (int i = 0; i < VEC; ++i) pr[i] = acc[i];
  }
  __syncthreads();
  // qbar (fixed-order sums, as in the blockify kernel) -> query rows of the MMA tile
  for (int i = tid; i < S8_R * D; i += S8_THREADS) {
    const int b = i / D, e = i - b * D;
    float s = 0.f;
#pragma unroll 4
    for (int q = 0; q < RPP; ++q) s += part[(b * RPP + q) * D + e];
    s *= (1.0f / BT);
    qs[b * KS + e] = s;
    if (b < nr) q_reps[((size_t)h * nq + r0 + b) * D + e] = s;
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- 2. scores on the tensor cores: warp w takes the 8-candidate tiles w, w + NW, ...
  {
    const int gq = lane >> 2, t4 = lane & 3;
    const int ntiles = (ncand + 7) / 8;
    for (int nt = warp; nt < ntiles; nt += NW) {
      float acc[6][4] = {};
      const float* brow = kb + (nt * 8 + gq) * KS;   // candidate nt*8 + gq (past ncand: unused)
      const uint32_t zero[1] = {0u};
#pragma unroll
      for (int k0 = 0; k0 < D; k0 += 8) {
        const int par = (k0 >> 3) & 1;
        uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
        tf32_split(qs[gq * KS + k0 + t4], ah[0], al[0]);
        tf32_split(qs[gq * KS + k0 + t4 + 4], ah[2], al[2]);
        ah[1] = ah[3] = al[1] = al[3] = zero[0];   // rows 8..15: zero queries
        tf32_split(brow[k0 + t4], bh0, bl0);
        tf32_split(brow[k0 + t4 + 4], bh1, bl1);
        mma_tf32(acc[3 * par + 0], al, bh0, bh1);
        mma_tf32(acc[3 * par + 1], ah, bl0, bl1);
        mma_tf32(acc[3 * par + 2], ah, bh0, bh1);
      }
      float r0v = ((acc[0][0] + acc[3][0]) + (acc[1][0] + acc[4][0])) + (acc[2][0] + acc[5][0]);
      float r1v = ((acc[0][1] + acc[3][1]) + (acc[1][1] + acc[4][1])) + (acc[2][1] + acc[5][1]);
      *reinterpret_cast<float2*>(ss + gq * ncs + nt * 8 + 2 * t4) = make_float2(r0v, r1v);
    }
  }
  int pc = cl.pc;
  if (!CAUSAL) {
    pc = prefix_cnt ? prefix_cnt[h] : 0;
    if (pc < 0 || pc > prefix_ld) {
      if (tid == 0 && r0 == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, pc, K_SCORE);
      pc = pc < 0 ? 0 : prefix_ld;
    }
  }
  const int sn = cl.sn;
  const int kk = min(k, ncand);
  for (int i = tid; i < nr * (pc + sn); i += S8_THREADS) {
    const int b = i / (pc + sn), j = i - b * (pc + sn);
    const size_t o = (size_t)h * nq + r0 + b;
    int val;
    if (CAUSAL) val = j < pc ? cl.pbase + j : cl.sbase + (j - pc);
    else val = j < pc ? prefix_slot[(size_t)h * prefix_ld + j] : suffix_slot[j - pc];
    out_slot[o * out_ld + (j < pc ? j : kk + j)] = val;
  }
  if (tid < nr) out_cnt[(size_t)h * nq + r0 + tid] = pc + kk + sn;
  __syncthreads();

  // ---- 3. warp b selects query block b's k best: element e = j*32 + lane (j < 8)
  if (warp < nr) {
    const int b = warp;
    auto score_of = [&](int e) {   // masked, scaled score of candidate e
      const int s = slot[e];
      float val = ss[b * ncs + e] * g.scale;
      if (s < 0 || s >= pool_slots) {
        if (b == 0 && r0 == 0) record_error(ws, PBSA_ERR_DEVICE_INDEX, s, K_SCORE);
        val = -INFINITY;
      }
      return isnan(val) ? -INFINITY : val;
    };
    uint64_t kv8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = j * 32 + lane;
      kv8[j] = e < ncand ? rank_key(score_of(e), gid[e]) : 0ull;
    }
    auto count_hi_ge = [&](uint32_t t) {
      int n = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) n += (uint32_t)(kv8[j] >> 32) >= t;
      return __reduce_add_sync(0xffffffffu, n);
    };
    // k-th largest high word (score order); stop early once exactly kk keys are at or above
    uint32_t th = 0;
    bool exact = false;
    if (kk > 0) {
#pragma unroll 1
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t t2 = th | (1u << bit);
        const int cnt = count_hi_ge(t2);
        if (cnt >= kk) {
          th = t2;
          if (cnt == kk) {
            exact = true;
            break;
          }
        }
      }
    }
    // the chosen set: exact -> every key whose high word is >= th; otherwise the keys above the
    // k-th key (high word, then the gid word), then keys equal to it in position order
    uint64_t tkey = 0;
    int n_above = 0;
    if (!exact && kk > 0) {
      int n_gt = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) n_gt += (uint32_t)(kv8[j] >> 32) > th;
      n_gt = __reduce_add_sync(0xffffffffu, n_gt);
      const int need = kk - n_gt;
      auto count_lo_ge = [&](uint32_t t) {
        int n = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) n += ((uint32_t)(kv8[j] >> 32) == th) && ((uint32_t)kv8[j] >= t);
        return __reduce_add_sync(0xffffffffu, n);
      };
      uint32_t tl = 0;
      if (need > 0 && count_lo_ge(0) > need) {
#pragma unroll 1
        for (int bit = 31; bit >= 0; --bit) {
          const uint32_t t2 = tl | (1u << bit);
          if (count_lo_ge(t2) >= need) tl = t2;
        }
      }
      tkey = ((uint64_t)th << 32) | tl;
#pragma unroll
      for (int j = 0; j < 8; ++j) n_above += kv8[j] > tkey;
      n_above = __reduce_add_sync(0xffffffffu, n_above);
    }
    int* chosen = reinterpret_cast<int*>(part) + b * 256;    // part is free after the pooling
    int eq_seen = 0, n_ch = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bool take;
      if (exact) {
        take = kv8[j] != 0ull && (uint32_t)(kv8[j] >> 32) >= th;
      } else {
        const bool eq = kk > 0 && kv8[j] == tkey;
        const unsigned eb = __ballot_sync(0xffffffffu, eq);
        const bool take_eq = eq && (eq_seen + __popc(eb & ((1u << lane) - 1u)) < kk - n_above);
        eq_seen += __popc(eb);
        take = (kk > 0 && kv8[j] > tkey) || take_eq;
      }
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      if (take) chosen[n_ch + __popc(tb & ((1u << lane) - 1u))] = j * 32 + lane;
      n_ch += __popc(tb);
    }
    __syncwarp();
    const size_t o = (size_t)h * nq + r0 + b;
    if (n_ch <= 32) {
      // order the chosen: larger key first, then the lower position (bitonic across lanes)
      int e = lane < n_ch ? chosen[lane] : 0x7FFFFFFF;
      float val = lane < n_ch ? score_of(e) : -INFINITY;
      uint64_t key = lane < n_ch ? rank_key(val, gid[e]) : 0ull;
#pragma unroll
      for (int k2 = 2; k2 <= 32; k2 <<= 1) {
#pragma unroll
        for (int j = k2 >> 1; j > 0; j >>= 1) {
          const uint64_t ok = __shfl_xor_sync(0xffffffffu, key, j);
          const int oe = __shfl_xor_sync(0xffffffffu, e, j);
          const float ov = __shfl_xor_sync(0xffffffffu, val, j);
          const bool other_first = ok > key || (ok == key && oe < e);
          const bool lower = (lane & j) == 0, desc = (lane & k2) == 0;
          if ((lower == desc) ? other_first : !other_first) {
            key = ok;
            e = oe;
            val = ov;
          }
        }
      }
      if (lane < n_ch) {
        out_slot[o * out_ld + pc + lane] = slot[e];
        if (out_score) out_score[o * k + lane] = val;
      }
    } else {
      // rank among the chosen: larger key first, then the lower position
      for (int t = lane; t < n_ch; t += 32) {
        const int e = chosen[t];
        const uint64_t ke = rank_key(score_of(e), gid[e]);
        int rank = 0;
        for (int u = 0; u < n_ch; ++u) {
          const int e2 = chosen[u];
          const uint64_t k2 = rank_key(score_of(e2), gid[e2]);
          rank += (k2 > ke) | ((k2 == ke) & (e2 < e));
        }
        out_slot[o * out_ld + pc + rank] = slot[e];
        if (out_score) out_score[o * k + rank] = score_of(e);
      }
    }
  }
}

// ncand: the candidate count (CAUSAL: the largest over the chunks, for the shared-memory layout).
template <typename T, int D, bool HSA, bool CAUSAL>
cudaError_t launch_t(const Geo& g, const void* x, int q_frames, float* q_reps, const float* k_reps,
                     int pool_slots, const int* cand_slot, const int* cand_gid, int ncand, int k,
                     const int* prefix_slot, const int* prefix_cnt, int prefix_ld, int* out_slot,
                     int* out_cnt, int out_ld, float* out_score, int top_frames, int n_recent,
                     const int* suffix_slot, int suffix_n, Causal cz, void* ws, cudaStream_t st) {
  const int nq = q_frames * g.bpf;
  if (!HSA && ncand <= 256) {
    const size_t smem8 = S8Layout<T, D>::bytes(ncand);
    auto kern8 = blockify_select8_kernel<T, D, CAUSAL>;
    cudaError_t e = set_smem_once((const void*)kern8, (int)smem8);
    if (e != cudaSuccess) return e;
    const int gx = CAUSAL ? (nq / cz.seq_blocks) * cz.n_chunks * cz.groups : (nq + S8_R - 1) / S8_R;
    kern8<<<dim3(gx, g.H), S8_THREADS, smem8, st>>>(
        static_cast<const T*>(x), g, nq, q_reps, k_reps, pool_slots, cand_slot, cand_gid, ncand, k,
        prefix_slot, prefix_cnt, prefix_ld, out_slot, out_cnt, out_ld, out_score, suffix_slot, suffix_n,
        cz, ws);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)ncand * (8 + 4 + 4 + 4);
  auto kern = blockify_select_kernel<T, D, HSA, CAUSAL>;
  cudaError_t e = set_smem_once((const void*)kern, (int)(smem > 0 ? smem : 8));
  if (e != cudaSuccess) return e;
  kern<<<dim3(nq, g.H), BS_THREADS, smem, st>>>(static_cast<const T*>(x), g, nq, q_reps, k_reps,
                                                 pool_slots, cand_slot, cand_gid, ncand, k,
                                                 prefix_slot, prefix_cnt, prefix_ld, out_slot,
                                                 out_cnt, out_ld, out_score, top_frames, n_recent,
                                                 suffix_slot, suffix_n, cz, ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_blockify_select(const Geo& g, const void* x, int q_frames, float* q_reps,
                                   const float* k_reps, int pool_slots, const int* cand_slot,
                                   const int* cand_gid, int ncand, int k, const int* prefix_slot,
                                   const int* prefix_cnt, int prefix_ld, int* out_slot,
                                   int* out_cnt, int out_ld, float* out_score, int top_frames,
                                   int n_recent, const int* suffix_slot, int suffix_n, void* ws,
                                   cudaStream_t st) {
  const bool hsa = top_frames >= 0;
  const Causal off = {0, 0, 0, 0, 0};
#define PBSA_BS(TT, DD)                                                                            \
  return hsa ? launch_t<TT, DD, true, false>(g, x, q_frames, q_reps, k_reps, pool_slots, cand_slot, \
                                             cand_gid, ncand, k, prefix_slot, prefix_cnt, prefix_ld, \
                                             out_slot, out_cnt, out_ld, out_score, top_frames,     \
                                             n_recent, suffix_slot, suffix_n, off, ws, st)         \
             : launch_t<TT, DD, false, false>(g, x, q_frames, q_reps, k_reps, pool_slots,         \
                                              cand_slot, cand_gid, ncand, k, prefix_slot,          \
                                              prefix_cnt, prefix_ld, out_slot, out_cnt, out_ld,    \
                                              out_score, 0, 0, suffix_slot, suffix_n, off, ws, st);
  if (g.dtype == PBSA_BF16) {
    if (g.d == 128) { PBSA_BS(__nv_bfloat16, 128) }
    if (g.d == 64) { PBSA_BS(__nv_bfloat16, 64) }
  } else {
    if (g.d == 128) { PBSA_BS(float, 128) }
    if (g.d == 64) { PBSA_BS(float, 64) }
    if (g.d == 32) { PBSA_BS(float, 32) }
  }
#undef PBSA_BS
  return cudaErrorNotSupported;
}

cudaError_t launch_blockify_train_select(const Geo& g, const void* x, int q_frames, float* q_reps,
                                         const float* k_reps, int pool_slots, int seq_frames,
                                         int chunk_frames, int sink_frames, int k, int* out_slot,
                                         int* out_cnt, int out_ld, float* out_score, void* ws,
                                         cudaStream_t st) {
  Causal cz;
  cz.seq_blocks = seq_frames * g.bpf;
  cz.chunk_blocks = chunk_frames * g.bpf;
  cz.sink_blocks = sink_frames * g.bpf;
  cz.n_chunks = (seq_frames + chunk_frames - 1) / chunk_frames;
  cz.groups = (cz.chunk_blocks + S8_R - 1) / S8_R;
  // the last chunk has the most candidates: every block of the earlier chunks but the sinks
  const int ncap = cz.n_chunks > 1 ? (cz.n_chunks - 1) * cz.chunk_blocks - cz.sink_blocks : 0;
  if (ncap > 1024) return cudaErrorNotSupported;
#define PBSA_TS(TT, DD)                                                                           \
  return launch_t<TT, DD, false, true>(g, x, q_frames, q_reps, k_reps, pool_slots, nullptr, nullptr, \
                                       ncap, k, nullptr, nullptr, 0, out_slot, out_cnt, out_ld,    \
                                       out_score, 0, 0, nullptr, 0, cz, ws, st);
  if (g.dtype == PBSA_BF16) {
    if (g.d == 128) { PBSA_TS(__nv_bfloat16, 128) }
    if (g.d == 64) { PBSA_TS(__nv_bfloat16, 64) }
  } else {
    if (g.d == 128) { PBSA_TS(float, 128) }
    if (g.d == 64) { PBSA_TS(float, 64) }
    if (g.d == 32) { PBSA_TS(float, 32) }
  }
#undef PBSA_TS
  return cudaErrorNotSupported;
}

}  // namespace pbsa
