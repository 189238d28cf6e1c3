/*
 * pbsa.h -- C ABI of the PBSA (Persistent Block-Sparse Attention) library, libpbsa.so.
 *
 * The method is the attention hot path of "Sparse Forcing: Native Trainable Sparse
 * Attention for Real-time Autoregressive Diffusion Video Generation" (gist.science,
 * English explainer, section 2 "Methodology": B "Structured Memory Decomposition",
 * C "Persistent Block-Sparse Attention (PBSA)", E "System Implementation: PBSA Kernel").
 * The KV cache of one attention layer is split into a persistent memory of capacity C
 * (sink blocks plus the best-scored older blocks) and a sliding local window.  Every
 * query block attends, in one softmax, to the persistent blocks plus its top-k local
 * blocks, chosen by coarse scores between mean-pooled block representatives; after a
 * chunk is finished the persistent memory is re-scored and updated in place.
 *
 * Conventions (all entry points)
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except the geometry
 *    struct, which is host memory read during the call.  The library never allocates
 *    device memory and keeps no pointer after a call returns.
 *  - All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and run on the current CUDA device.
 *  - Shape and scalar errors are detected on the host and returned synchronously as
 *    PBSA_ERR_INVALID_ARG (bad value) or PBSA_ERR_UNSUPPORTED (valid but not built);
 *    nothing is launched in that case.  A failed launch returns PBSA_ERR_CUDA.
 *  - Bad data found on the device (a slot id outside the pool) is skipped and recorded in
 *    the workspace's error word; pbsa_get_device_error() reports it.  A wait inside a
 *    kernel that exceeds its bound records PBSA_ERR_TIMEOUT the same way and the kernel
 *    returns.  No call traps, asserts or exits.
 *  - Token tensors are raster order [T][H][d] (T = frames * frame_h * frame_w, token
 *    t = frame*frame_h*frame_w + y*frame_w + x), in the geometry's dtype.
 *  - A block is 1 frame x (tile_h x tile_w) = 64 tokens.  Global block id of tile
 *    (ty, tx) of frame f is f*bpf + ty*(frame_w/tile_w) + tx, bpf = blocks per frame.
 *    Inside a block, token (ly, lx) is row ly*tile_w + lx.
 *  - A pool is the block-major KV cache of one layer: [H][pool_slots][64][d] in the
 *    geometry's dtype; k_reps is [H][pool_slots][d] fp32.  Slots 0..C-1 are the persistent
 *    memory; the caller places the local window and any staging area after them.
 */
#ifndef PBSA_H
#define PBSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PBSA_API __attribute__((visibility("default")))
#else
#define PBSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PBSA_OK = 0,
  PBSA_ERR_INVALID_ARG = 1,
  PBSA_ERR_UNSUPPORTED = 2,
  PBSA_ERR_CUDA = 3,
  PBSA_ERR_TIMEOUT = 4,
  PBSA_ERR_DEVICE_INDEX = 5
} pbsa_status;

typedef enum { PBSA_F32 = 0, PBSA_BF16 = 1 } pbsa_dtype;

/* Geometry of one attention layer.  tile_h*tile_w must be 64; frame_h, frame_w must be
 * multiples of tile_h, tile_w; head_dim a multiple of 32 and <= 128 (bf16 needs 128). */
typedef struct {
  int heads;      /* H */
  int head_dim;   /* d */
  int frame_h;    /* latent tokens per frame, vertically */
  int frame_w;    /* latent tokens per frame, horizontally */
  int tile_h;     /* block tile height (tokens) */
  int tile_w;     /* block tile width (tokens) */
  float scale;    /* softmax and coarse-score scale, normally 1/sqrt(d) */
  int dtype;      /* pbsa_dtype of token tensors and pools */
} pbsa_geom;

/* Bytes of device workspace needed by calls with at most `max_q_blocks` query blocks and
 * at most `max_pool_entries` (= C + candidates) entries in a memory update.  The first
 * 256 bytes hold the device error word; the caller zero-fills the workspace once before
 * first use.  One workspace must not be used by two calls that overlap in time. */
PBSA_API size_t pbsa_workspace_bytes(const pbsa_geom* g, int max_q_blocks, int max_pool_entries);

/* a1 -- blockify: mean-pooled representatives, and optionally a block-major copy.
 * (Chinese explainer 2.2 "blockified compression"; English 2.E "blockifying the latent
 * space, enabling coalesced reads".)
 *  x        [n_frames*frame_h*frame_w][H][d] raster, geometry dtype.
 *  reps     out [H][rep_slots][d] fp32: reps[h][slot(b)] = mean of block b's 64 tokens.
 *  dst_slot nullable [n_frames*bpf]: slot of local block b (b = f*bpf + tile); NULL means
 *           slot b.  Slots must be < rep_slots (and < pool_slots when pool is given).
 *  pool     nullable out [H][pool_slots][64][d]: block b's tokens are copied to slot(b).
 * Fully overwrites the destination rows; reads nothing else. */
PBSA_API pbsa_status pbsa_blockify(const pbsa_geom* g, const void* x, int n_frames,
                          float* reps, int rep_slots, const int* dst_slot,
                          void* pool, int pool_slots, void* ws, void* stream);

/* a1 for a committed chunk -- pbsa_blockify of K and of V in one launch, with the same
 * destination slots (the chunk's K and V blocks enter the cache together; English 2.E
 * "blockifying the latent space").  Equivalent to
 *   pbsa_blockify(k, n_frames, k_reps, rep_slots, dst_slot, k_pool, pool_slots) and
 *   pbsa_blockify(v, n_frames, v_reps, rep_slots, dst_slot, v_pool, pool_slots).
 *  k, v           [n_frames*frame_h*frame_w][H][d] raster, geometry dtype (16-byte aligned).
 *  k_reps         out [H][rep_slots][d] fp32 (required).
 *  v_reps         nullable out [H][rep_slots][d] fp32; NULL skips the V representatives
 *                 (the method only scores K).
 *  k_pool, v_pool out [H][pool_slots][64][d] (both required).
 *  dst_slot       nullable [n_frames*bpf], as for pbsa_blockify.
 *  flags          0, or PBSA_OVERLAP_PREVIOUS: launch as a programmatic dependent of the
 *                 previous kernel on `stream`.  The commit may then start on SMs that kernel
 *                 leaves idle (pbsa_attend signals this once all of its CTAs have started), and
 *                 it still completes only after that kernel, so later work on the stream sees
 *                 both.  Only valid when the previous kernel neither writes k or v nor reads
 *                 or writes the destination slots and k_reps rows (true of pbsa_attend before
 *                 the commit of the chunk it attended: its lists never name free ring slots).
 * Errors as for pbsa_blockify (an unknown flag bit is PBSA_ERR_INVALID_ARG). */
#define PBSA_OVERLAP_PREVIOUS 1
PBSA_API pbsa_status pbsa_blockify_kv(const pbsa_geom* g, const void* k, const void* v, int n_frames,
                          float* k_reps, float* v_reps, int rep_slots, const int* dst_slot,
                          void* k_pool, void* v_pool, int pool_slots, int flags, void* ws, void* stream);

/* a2 -- coarse score + top-k: for each head h and query block r,
 *   score(r, c) = scale * <q_reps[h][r], k_reps[h][cand_slot[h][c]]>  (fp32)
 * and the k best candidates (score descending, ties to the lower cand_gid, then the lower
 * position c).  (English 2.C "Local Sparsity": top-K local blocks from compressed block
 * representatives.)  The output row is the optional prefix followed by the selection:
 *   out_slot[h][r][0..pc)      = prefix_slot[h][0..pc),  pc = prefix_cnt ? prefix_cnt[h] : 0
 *   out_slot[h][r][pc + i]     = cand_slot of the i-th best candidate, i < min(k, ncand)
 *   out_cnt[h][r]              = pc + min(k, ncand)
 *   out_score[h][r][i]         = its score (nullable)
 *  q_reps [H][nq][d]; k_reps [H][pool_slots][d]; cand_slot, cand_gid [H][ncand];
 *  prefix_slot [H][prefix_ld]; out_slot [H][nq][out_ld] with out_ld >= prefix_ld + k.
 *  ncand <= 1024. */
PBSA_API pbsa_status pbsa_score_select(const pbsa_geom* g, const float* q_reps, int nq,
                              const float* k_reps, int pool_slots,
                              const int* cand_slot, const int* cand_gid, int ncand, int k,
                              const int* prefix_slot, const int* prefix_cnt, int prefix_ld,
                              int* out_slot, int* out_cnt, int out_ld, float* out_score,
                              void* ws, void* stream);

/* a1 + a2 fused -- blockify of a query chunk and top-k selection in one pass (the
 * "lightweight coarse routing" of English 2.C "Local Sparsity" over the blockified latent
 * space of 2.E; Chinese 2.2 "块化压缩").  Same results as pbsa_blockify(q, q_frames,
 * q_reps, nq, NULL, NULL, ...) followed by pbsa_score_select(q_reps, nq, ...) with the
 * same arguments, except that the scores are summed in a different (fixed) order, so
 * candidates whose scores differ only in the last bits may rank the other way:
 *   q_reps[h][r] = mean of query block r's 64 tokens (bit-identical to pbsa_blockify)
 *   out_slot / out_cnt / out_score as for pbsa_score_select.
 *  q      [q_frames*frame_h*frame_w][H][d] raster, geometry dtype (16-byte aligned);
 *         nq = q_frames*bpf query blocks.
 *  q_reps out [H][nq][d] fp32.
 *  Other arguments as for pbsa_score_select (ncand <= 1024). */
PBSA_API pbsa_status pbsa_blockify_score_select(const pbsa_geom* g, const void* q, int q_frames,
                                       float* q_reps, const float* k_reps, int pool_slots,
                                       const int* cand_slot, const int* cand_gid, int ncand, int k,
                                       const int* prefix_slot, const int* prefix_cnt, int prefix_ld,
                                       int* out_slot, int* out_cnt, int out_ld, float* out_score,
                                       void* ws, void* stream);

/* a1 + a2 fused, hierarchical selection -- as pbsa_blockify_score_select, but the candidates
 * are chosen in two levels, after the hierarchical sparse attention of the related Light
 * Forcing method (papernotes.org notes, "方法详解", HSA steps (1)-(3)):
 *   frame score(t)  = mean of the scores of frame t's blocks (= the score of its mean-pooled
 *                     representative), summed in block order;
 *   chosen frames   = the n_recent_frames latest frames + the top_frames best other frames
 *                     (score descending, the earlier frame on ties);
 *   selection       = the k best blocks of the chosen frames (score descending, then the lower
 *                     cand_gid, then the lower position).
 *  The candidates must come in whole frames in time order: ncand = nf * bpf, candidate c in
 *  frame slot c / bpf (nf <= 256).  out_cnt[h][r] = pc + min(k, blocks of the chosen frames).
 *  Other arguments, outputs and limits as for pbsa_blockify_score_select. */
PBSA_API pbsa_status pbsa_blockify_hsa_select(const pbsa_geom* g, const void* q, int q_frames,
                                     float* q_reps, const float* k_reps, int pool_slots,
                                     const int* cand_slot, const int* cand_gid, int ncand,
                                     int top_frames, int n_recent_frames, int k,
                                     const int* prefix_slot, const int* prefix_cnt, int prefix_ld,
                                     int* out_slot, int* out_cnt, int out_ld, float* out_score,
                                     void* ws, void* stream);

/* a1 + a2 fused, general form -- pbsa_blockify_score_select (top_frames < 0) or
 * pbsa_blockify_hsa_select (top_frames >= 0), with an optional suffix: after each row's
 * selection, suffix_slot[0..suffix_n) (device, shared by every head and query block) is
 * appended, and out_cnt[h][r] counts it.  The suffix serves lists that every query block
 * attends besides its selection, e.g. the current chunk's own blocks written into the pool at
 * the current noise level (the chunk-wise self-attention of the trainable path, English 2.D
 * "Training Strategy", applied at inference as a variant).  Requires out_ld >= prefix_ld + k +
 * suffix_n; other arguments, outputs and limits as for the two calls above. */
PBSA_API pbsa_status pbsa_blockify_select_ex(const pbsa_geom* g, const void* q, int q_frames,
                                    float* q_reps, const float* k_reps, int pool_slots,
                                    const int* cand_slot, const int* cand_gid, int ncand, int k,
                                    int top_frames, int n_recent_frames, const int* prefix_slot,
                                    const int* prefix_cnt, int prefix_ld, const int* suffix_slot,
                                    int suffix_n, int* out_slot, int* out_cnt, int out_ld,
                                    float* out_score, void* ws, void* stream);

/* a1 + a2 fused, the trainable path's lists -- the masks of chunk-wise training with the dynamic
 * sparse cache (English 2.D "Training Strategy": the model is trained with the same sparse cache
 * it uses at inference).  Sequences of seq_frames frames are folded into the frame axis
 * (q_frames = n_seq * seq_frames) and cut into chunks of chunk_frames frames (the last chunk of a
 * sequence may be shorter).  The pool holds every sequence's blocks in order: the slot of a block
 * is its global block id (pbsa_blockify / pbsa_blockify_kv with dst_slot = NULL), so k_reps are
 * the keys' representatives.  For query block r of sequence s (blocks [s0, s0 + seq_frames*bpf)),
 * chunk c (blocks [cs, ce)):
 *   c == 0:  out_slot[h][r] = cs .. ce-1                                (its own chunk)
 *   c >= 1:  out_slot[h][r] = s0 .. s0+S-1                              (the sinks, S = sink_frames*bpf)
 *                           + the k best of s0+S .. cs-1 by scale * <q_reps[h][r], k_reps[h][slot]>
 *                             (score descending, ties to the lower slot), best first
 *                           + cs .. ce-1                                (its own chunk)
 *   out_cnt[h][r] = the row's length; out_score[h][r][i] (nullable) = the i-th selected score.
 * q_reps[h][r] = mean of query block r's 64 tokens (bit-identical to pbsa_blockify).
 *  q       [q_frames*frame_h*frame_w][H][d] raster, geometry dtype (16-byte aligned).
 *  q_reps  out [H][q_frames*bpf][d] fp32;  k_reps [H][pool_slots][d] fp32, pool_slots >= q_frames*bpf.
 *  out_slot out [H][q_frames*bpf][out_ld], out_ld >= S + k + min(chunk_frames, seq_frames)*bpf;
 *  out_cnt  out [H][q_frames*bpf];  out_score nullable out [H][q_frames*bpf][k].
 *  0 <= sink_frames <= chunk_frames (the sinks lie in chunk 0); q_frames a multiple of seq_frames.
 *  At most 1024 candidates in a sequence's last chunk, else PBSA_ERR_UNSUPPORTED. */
PBSA_API pbsa_status pbsa_blockify_train_select(const pbsa_geom* g, const void* q, int q_frames,
                                       float* q_reps, const float* k_reps, int pool_slots,
                                       int seq_frames, int chunk_frames, int sink_frames, int k,
                                       int* out_slot, int* out_cnt, int out_ld, float* out_score,
                                       void* ws, void* stream);

/* a3 -- fine attention over the selected blocks (the hybrid mask of the Chinese
 * explainer 2.2 "掩码机制"; English 2.C "Global Access" + "Local Sparsity"):
 * for every token i of query block r of head h,
 *   o_i = sum_{j in A} softmax_j(scale * q_i . k_j) v_j,  lse_i = ln sum_{j in A} exp(scale * q_i . k_j)
 * where A = the 64 tokens of each pool slot kv_slot[h][r][0..kv_cnt[h][r]) -- one joint
 * softmax over the union.  Slots of one row must be distinct.  An empty row gives o = 0
 * and lse = -inf.
 *  q     [q_frames*frame_h*frame_w][H][d] raster; nq = q_frames*bpf query blocks.
 *  k_pool, v_pool [H][pool_slots][64][d];  kv_slot [H][nq][kv_ld];  kv_cnt [H][nq].
 *  o     out, same layout and dtype as q;  lse  nullable out [H][T_q] fp32 (raster t).
 * bf16: tcgen05 tensor cores, fp32 accumulation, d = 128, kv_ld <= 512.
 * fp32: exact fp32 SIMT path (d <= 128), kv_ld <= 4096. */
PBSA_API pbsa_status pbsa_attend(const pbsa_geom* g, const void* q, int q_frames,
                        const void* k_pool, const void* v_pool, int pool_slots,
                        const int* kv_slot, const int* kv_cnt, int kv_ld,
                        void* o, float* lse, void* ws, void* stream);

/* a5 -- backward of pbsa_attend under the same lists (English 2.D "Training Strategy": the
 * model is trained with the same dynamic sparse cache, so the sparse attention needs its
 * gradients):
 *   P = exp(scale * q_i . k_j - lse_i) over each row's listed blocks; D_i = dO_i . O_i;
 *   dV = P^T dO;  dP = dO V^T;  dS = P * (dP - D);  dQ = scale * dS K;  dK = scale * dS^T Q.
 *  q, o, d_o  [q_frames*frame_h*frame_w][H][d] raster bf16; lse [H][T_q] fp32 from pbsa_attend.
 *  k_pool, v_pool, kv_slot, kv_cnt, kv_ld as for pbsa_attend (slots of one row distinct).
 *  dq      out [T_q][H][d] raster bf16.
 *  dk_pool, dv_pool out [H][pool_slots][64][d] bf16: every slot is written (slots that no
 *          query block attends get zeros).
 *  bf16, d = 128, kv_ld <= 512, q_frames*bpf <= 512 query blocks.  Deterministic (no
 *  floating-point atomics).  S and dP are computed once per (query block, listed block) pair:
 *  the dK/dV pass stores each 64 x 64 dS tile (bf16) in the workspace and the dQ pass reads
 *  it back.
 *  ws: pbsa_bwd_workspace_bytes(g, q_frames, pool_slots, kv_ld) bytes of device memory whose
 *  first 256 bytes (the error word) are zero before first use.  It holds one 8 KB dS tile per
 *  (head, query block, list entry): H * q_frames*bpf * kv_ld * 8192 bytes, plus a few bytes
 *  per query row and per slot. */
PBSA_API size_t pbsa_bwd_workspace_bytes(const pbsa_geom* g, int q_frames, int pool_slots, int kv_ld);
PBSA_API pbsa_status pbsa_attend_bwd(const pbsa_geom* g, const void* q, int q_frames,
                                     const void* k_pool, const void* v_pool, int pool_slots,
                                     const int* kv_slot, const int* kv_cnt, int kv_ld,
                                     const void* o, const void* d_o, const float* lse,
                                     void* dq, void* dk_pool, void* dv_pool, void* ws, void* stream);

/* a4 -- persistent-memory update ("Top-C retention"; English 2.C "Dynamic Update",
 * Chinese 2.2 "粗粒度评分与更新"), per head h:
 *   pool    = valid persistent slots (slot_gid[h][j] >= 0, j < C) + the candidates
 *             (cand_slot/cand_gid [H][ncand]; e.g. the blocks leaving the local window)
 *   p_r     = softmax over the pool of scale * <q_reps[h][r], k_reps[h][slot]>
 *   a_b     = mean over the nq query blocks of p_{r,b}
 *   ema_b   = a_b for a candidate, gamma*slot_ema + (1-gamma)*a_b for a persistent block
 *   keep    = every sink (gid < n_sink_gid) + the top-(C - #sinks) others by ema_b
 *             (ties to the lower gid)
 * Kept persistent blocks stay in their slots; each kept candidate is copied (K, V blocks
 * and k_reps row) from its cand_slot into a freed persistent slot (ascending slot order,
 * candidates in rank order); slot_gid / slot_ema are rewritten (-1 / 0 for empty slots).
 * p_list (nullable out [H][C]) receives the valid persistent slots ascending and p_cnt
 * (nullable out [H]) their count -- the prefix for pbsa_score_select.
 *  Requires C + ncand <= 2048; cand slots must be >= C (outside the persistent region).
 *  Workspace: pbsa_workspace_bytes(g, nq, C + ncand). */
PBSA_API pbsa_status pbsa_memory_update(const pbsa_geom* g, const float* q_reps, int nq,
                               float* k_reps, void* k_pool, void* v_pool, int pool_slots,
                               int* slot_gid, float* slot_ema, int capacity, int n_sink_gid,
                               const int* cand_slot, const int* cand_gid, int ncand,
                               float gamma, int* p_list, int* p_cnt, void* ws, void* stream);

/* a4 in two launches, so that the scoring can overlap other work.  Together,
 *   pbsa_memory_update_plan(...) ; pbsa_memory_update_apply(...)
 * compute what pbsa_memory_update computes (the same rule; the column sums of the softmax may
 * be added in another order, so EMA values may differ in the last bits).
 * plan: everything but the block copies -- scores, softmax, EMA, ranking, the new slot_gid /
 *   slot_ema, p_list / p_cnt, and the copy list, which it leaves in `ws`.  It reads q_reps,
 *   k_reps, the slot table and the candidate lists; it never touches k_pool / v_pool.
 *   flags: 0, or PBSA_OVERLAP_PREVIOUS (pools of up to 256 entries): launch as a programmatic
 *   dependent of the previous kernel on `stream`, which may still be running (e.g. pbsa_attend
 *   of the same chunk, which reads the pools but nothing plan writes); plan completes only
 *   after that kernel.  Larger pools ignore the flag.
 * apply: copies the promoted blocks (K, V and k_reps rows) as listed in `ws`; `ws`, capacity
 *   and ncand must be those of the plan call, with nothing else using `ws` in between.
 * Arguments otherwise as for pbsa_memory_update; workspace pbsa_workspace_bytes(g, nq,
 * capacity + ncand). */
PBSA_API pbsa_status pbsa_memory_update_plan(const pbsa_geom* g, const float* q_reps, int nq,
                               const float* k_reps, int pool_slots, int* slot_gid, float* slot_ema,
                               int capacity, int n_sink_gid, const int* cand_slot, const int* cand_gid,
                               int ncand, float gamma, int* p_list, int* p_cnt, int flags, void* ws,
                               void* stream);
PBSA_API pbsa_status pbsa_memory_update_apply(const pbsa_geom* g, float* k_reps, void* k_pool,
                               void* v_pool, int pool_slots, int capacity, int ncand, void* ws,
                               void* stream);

/* pbsa_memory_update without a caller-provided workspace.  The paper has no counterpart;
 * this is a library convenience for callers that cannot allocate device memory (for
 * example a plug-in whose host application owns every device allocation, or a runtime
 * whose memory pools are frozen).  Arguments and results are those of
 * pbsa_memory_update, minus `ws`: the scratch is a fixed 4 MiB array inside the library,
 * one per GPU, held from the first call until the process exits.
 *  - Sizes: requires pbsa_workspace_bytes(g, nq, capacity + ncand) <= 4 MiB (about
 *    4*H*nq*(capacity + ncand) bytes); larger calls return PBSA_ERR_UNSUPPORTED and
 *    launch nothing.
 *  - Set-up: the first call on a device looks up that device's scratch address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - Sharing: every call uses the same scratch, which keeps the last call's contents;
 *    calls whose work overlaps on the GPU race.  Device-side index errors are recorded in
 *    the scratch's error word, which each call clears when it starts: read it with
 *    pbsa_memory_update_noalloc_error before the next call.
 *  - Allocates nothing (no cudaMalloc or allocating library call). */
PBSA_API pbsa_status pbsa_memory_update_noalloc(const pbsa_geom* g, const float* q_reps, int nq,
                                                float* k_reps, void* k_pool, void* v_pool,
                                                int pool_slots, int* slot_gid, float* slot_ema,
                                                int capacity, int n_sink_gid, const int* cand_slot,
                                                const int* cand_gid, int ncand, float gamma,
                                                int* p_list, int* p_cnt, void* stream);

/* Self-test of the bounded waits (the paper has no counterpart).  Every kernel that waits on an
 * mbarrier gives up after a time limit, records PBSA_ERR_TIMEOUT in the workspace's error word
 * and returns instead of hanging.  This launches one thread that waits, with that same code, on
 * an mbarrier nothing ever arrives on, for limit_us microseconds (1 .. 1000000): afterwards
 * pbsa_get_device_error(ws) reports PBSA_ERR_TIMEOUT and the context remains usable.
 *  ws: a workspace whose first 256 bytes are the error word. */
PBSA_API pbsa_status pbsa_selftest_wait_timeout(void* ws, unsigned int limit_us, void* stream);

/* The device error word of pbsa_memory_update_noalloc's built-in scratch, for its callers,
 * who hold no workspace to pass to pbsa_get_device_error (the paper has no counterpart).
 * Synchronises `stream`, reads and clears the word and returns it (PBSA_OK when clean):
 * PBSA_ERR_DEVICE_INDEX when the last update on this device met a candidate slot outside the
 * pool (that candidate was left out), PBSA_ERR_TIMEOUT when a bounded wait expired.  Runs on
 * the current device; the first use on a device looks up the scratch's address, like the
 * update's own first call. */
PBSA_API pbsa_status pbsa_memory_update_noalloc_error(void* stream);

/* Synchronises `stream`, reads and clears the workspace's device error word, and returns
 * it (PBSA_OK when clean). */
PBSA_API pbsa_status pbsa_get_device_error(void* ws, void* stream);

/* Static description of a status code. */
PBSA_API const char* pbsa_status_string(pbsa_status s);

#ifdef __cplusplus
}
#endif
#endif /* PBSA_H */
