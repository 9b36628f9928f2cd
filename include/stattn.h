/*
 * stattn.h -- C ABI of libstattn.so, the single-GPU (sm_100a) hot path of the
 * attention block of a spatial-temporal diffusion transformer.
 *
 * Sources of each operation (page title, then section):
 *   [SF]  "ScaleFusion: Scalable Inference of Spatial-Temporal Diffusion
 *         Transformers for High-Resolution Long Video Generation" (paper
 *         review), sections "三、技术架构" (layer table, distributed execution
 *         flow, core formulas of spatial-temporal independence) and
 *         "四、核心创新" (intra-layer schedule with N_T/N_S slices, inter-layer
 *         schedule with L_T/L_S partitions, pseudo-code).
 *   [SW]  "Technical Summary: SwiftFusion", Methodology 2 "Torus Attention"
 *         (all-to-all broken into chunks, partial attention per chunk).
 *   [xD]  "xDiT: an Inference Engine for Diffusion Transformers (DiTs) with
 *         Massive Parallelism", section 3 (image-DiT full attention over
 *         hundreds of thousands to millions of tokens).
 *   [CC]  "CoCoDiff: Optimizing Collective Communications for Distributed
 *         Diffusion Transformer Inference Under Ulysses Sequence
 *         Parallelism", sections on Ulysses all-to-all, "V-First" (RMSNorm on
 *         Q and K only) and "V-Major" (per-token L1 change of V, threshold,
 *         cached data for inactive tokens, full refresh every 10 steps).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates or frees device memory and never synchronises
 *     a stream (except st_check_device_status, which says so).
 *   - Every call is stream-ordered on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and returns before the work finishes.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns its status and launches nothing.  A launch error
 *     reported by the CUDA runtime returns ST_ERR_CUDA.  Waits inside the
 *     tensor-core attention kernel are bounded; a wait that runs out sets a
 *     device error word that st_check_device_status reports as
 *     ST_ERR_TIMEOUT.  No call aborts the process or traps the GPU.
 *   - bf16 is IEEE-style bfloat16 (1-8-7); reductions accumulate in fp32 and
 *     round to bf16 once, to nearest even.
 *   - Element strides are in ELEMENTS, not bytes.
 */
#ifndef STATTN_H
#define STATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *st_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  ST_OK = 0,
  ST_ERR_NULL = -1,         /* a required pointer is NULL                      */
  ST_ERR_SHAPE = -2,        /* a size is <= 0, out of range or inconsistent     */
  ST_ERR_DIVISIBILITY = -3, /* P, N_T, N_S or the head count does not divide    */
  ST_ERR_DTYPE = -4,        /* dtype / element size not supported by the call   */
  ST_ERR_ALIGN = -5,        /* pointer or row pitch not aligned as required     */
  ST_ERR_UNSUPPORTED = -6,  /* valid request this build has no kernel for       */
  ST_ERR_CUDA = -7,         /* the CUDA runtime reported an error               */
  ST_ERR_TIMEOUT = -8       /* a bounded device-side wait ran out               */
} st_status;

typedef enum { ST_F32 = 0, ST_BF16 = 1 } st_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char *st_status_string(st_status s);

/* ABI version of this header: 1. */
int st_abi_version(void);

/* ------------------------------------------------------------------------
 * Attention descriptor.
 *
 * Q, K, V and O are logical [B, T, S, H, D] tensors: B batches of T frames of
 * S tokens, each token a row of C = H*D channels with head h at channels
 * [h*D, (h+1)*D).  Element (b, t, s, h, d) lives at element offset
 *
 *   b*stride_b + (t / tb)*stride_tb + (t % tb)*stride_t
 *              + (s / sb)*stride_sb + (s % sb)*stride_s + h*D + d
 *
 * with tb = t_block (T when t_block == 0) and sb = s_block (S when 0).  The
 * two-level form addresses the sliced layouts [B,N_T,N_S,T/N_T,S/N_S/P,C] of
 * the ScaleFusion intra-layer schedule [SF "四、核心创新"] directly.  Zero
 * strides mean the dense layout [B, T, S, H*D].  Q, K, V and O share the
 * descriptor's strides.
 * ---------------------------------------------------------------------- */
typedef struct {
  int size;               /* sizeof(st_attn_desc), for ABI versioning          */
  int B, T, S, H, D;      /* sizes; D in {32, 64, 72, 80, 96, 128} for bf16      */
  st_dtype dtype;         /* dtype of Q, K, V (and of O unless o_fp32)          */
  float scale;            /* softmax scale; <= 0 means 1/sqrt(D)                */
  long long stride_b, stride_t, stride_s;   /* elements; 0 -> dense              */
  int t_block;            /* frames per frame block; 0 -> one level             */
  long long stride_tb;    /* elements between frame blocks                      */
  int s_block;            /* tokens per token block; 0 -> one level             */
  long long stride_sb;    /* elements between token blocks                      */
  int n_slices, slice;    /* compute slice `slice` of `n_slices` only (frames
                             for the spatial call, tokens for the temporal
                             call); slice < 0 or n_slices <= 1 -> everything   */
  int kv_begin, kv_end;   /* spatial call: keys [kv_begin, kv_end) of each
                             frame; 0,0 -> all S keys                           */
  int o_fp32;             /* nonzero: write O as fp32 (a normalised partial for
                             attn_chunk_merge) with the same element strides     */
} st_attn_desc;

/* Spatial attention [SF "三、技术架构" layer table; xD section 3]: for every
 * (b, t, h) in the selected frames,
 *     O[b,t,:,h,:] = softmax(Q[b,t,:,h,:] K[b,t,kv,h,:]^T * scale) V[b,t,kv,h,:]
 * over the keys kv of frame t.  T = 1, S = N is image-DiT full attention.  A
 * key range [kv_begin, kv_end) yields the partial result of one KV chunk of
 * ring / Torus attention [SW Methodology 2]; merge chunks with
 * attn_chunk_merge.
 *   lse: optional fp32 [B, T, H, S] dense, natural-log log-sum-exp of the
 *        scaled scores of each query row (-inf for an empty key range).
 *   bf16 runs on the tcgen05 tensor-core kernel (fp32 accumulation); fp32 runs
 *   on an fp32 FMA kernel.  Returns ST_ERR_ALIGN if a pointer or stride is not
 *   16-byte aligned, ST_ERR_UNSUPPORTED for a bf16 head dim outside the set
 *   above, ST_ERR_SHAPE for a bad key range. */
st_status st_attn_spatial(const st_attn_desc *desc, const void *q, const void *k,
                          const void *v, void *o, float *lse, st_stream_t stream);

/* Spatial attention over one KV chunk, merged into the accumulated result of
 * the chunks before it -- the per-chunk step of ring / Torus attention with
 * the log-sum-exp merge done in the same kernel [SW Methodology 2]:
 *     (O_c, lse_c) = the normalised partial and LSE of keys [kv_begin, kv_end)
 *     M = max(lse_a, lse_c),  w_a = exp(lse_a - M),  w_c = exp(lse_c - M)
 *     o = (w_a O_a + w_c O_c) / (w_a + w_c),  lse = M + ln(w_a + w_c)
 * which equals attn_chunk_merge of the two without writing O_c.
 *   o_acc: fp32 accumulated partial, same element strides as Q (read only).
 *   lse_acc: fp32 [B, T, H, S] dense LSE of o_acc (-inf: nothing accumulated).
 *   o: the merged result; fp32 when desc->o_fp32 (or for fp32 Q), and then it
 *      may be o_acc itself (in place), else Q's dtype (the final output,
 *      which must not overlap o_acc).
 *   lse: optional merged LSE, may be lse_acc.
 * Chain: chunk 0 with st_attn_spatial (o_fp32), chunks 1..R-2 in place with
 * o_fp32, the last chunk with o in Q's dtype.  Errors as st_attn_spatial;
 * ST_ERR_NULL for a missing accumulator, ST_ERR_SHAPE for a bf16 o equal to
 * o_acc.  The pages have no separate API for this fused form. */
st_status st_attn_spatial_merge(const st_attn_desc *desc, const void *q, const void *k,
                                const void *v, const float *o_acc, const float *lse_acc,
                                void *o, float *lse, st_stream_t stream);

/* Full attention over R KV ring chunks in one launch, the chunk-and-merge
 * scheme of ring / Torus attention [SW Methodology 2; SF "六" RingAttention]
 * with the merge carried inside the kernel:
 *   the S keys of each frame are cut into n_chunks chunks, chunk c holding keys
 *   [floor(c*S/R), floor((c+1)*S/R)).  A block of 256 query rows (one frame,
 *   one head) attends to its chunks in ring order, starting at the chunk that
 *   holds its first row -- the stationary chunk a ring rank owns -- and then
 *   c+1, c+2, ... modulo R, as the other chunks would arrive.  The running row
 *   max, row sum and unnormalised O are carried from one chunk into the next,
 *   which is the log-sum-exp merge of attn_chunk_merge applied chunk by chunk
 *   without writing a partial; the result equals the merge of the R
 *   per-chunk partials (and full attention over the S keys) up to rounding
 *   order.
 *   desc: as st_attn_spatial; kv_begin and kv_end must be 0 (the chunks
 *     partition the whole frame).  o_fp32 may be set.
 *   lse: optional fp32 [B, T, H, S], the merged natural-log LSE.
 *   n_chunks: 1..64, at most S, and S * n_chunks < 2^32.  ST_ERR_SHAPE
 *     otherwise.
 *   fp32 Q/K/V run the fp32 FMA kernel over the keys in natural order.
 *   Other errors as st_attn_spatial.  The pages give no API for this form. */
st_status st_attn_ring(const st_attn_desc *desc, const void *q, const void *k,
                       const void *v, void *o, float *lse, int n_chunks,
                       st_stream_t stream);

/* Temporal attention [SF "三、技术架构"]: for every (b, s, h) in the selected
 * tokens, attention over the T frames of token s.  T <= 64.
 *   lse: optional fp32 [B, S, H, T] dense.
 *   kv_begin/kv_end must be 0.  bf16 uses tensor-core mma tiles with fp32
 *   accumulation; fp32 uses fp32 FMA. */
st_status st_attn_temporal(const st_attn_desc *desc, const void *q, const void *k,
                           const void *v, void *o, float *lse, st_stream_t stream);

/* Log-sum-exp merge of KV-chunk partials [SW Methodology 2]:
 *     M = max_c lse_c,  lse = M + ln sum_c exp(lse_c - M),
 *     o = sum_c exp(lse_c - lse) * o_c
 *   o_parts, lse_parts: HOST arrays of n_chunks (1..16) DEVICE pointers;
 *     o_parts[c] is fp32 dense [n_units, S, H, D] (n_units = B*T frames),
 *     lse_parts[c] is fp32 dense [n_units, H, S].
 *   o_out: dense [n_units, S, H, D] in out_dtype.  lse_out: optional
 *   [n_units, H, S].  Rows whose every chunk has lse = -inf get o = 0.
 *   o_out and lse_out must not overlap each other or any part (ST_ERR_SHAPE):
 *   outputs are written while other threads still read the parts. */
st_status attn_chunk_merge(int n_chunks, const float *const *o_parts,
                           const float *const *lse_parts, long long n_units, int S,
                           int H, int D, void *o_out, st_dtype out_dtype,
                           float *lse_out, st_stream_t stream);

/* ------------------------------------------------------------------------
 * All-to-all relayout on a virtual partition [SF "三、技术架构" distributed
 * execution flow and "四、核心创新" pseudo-code; CC Ulysses section].
 *
 * The P shards of the distributed tensor are stacked as the outermost axis of
 * one buffer; the all-to-all is a permutation of rows inside HBM.
 *
 * ST_S2T / ST_T2S (T_or_N = T, S_or_H = S, C_or_D = C):
 *   x, shard p: [B, N_T, N_S, T/N_T, S/(N_S*P), C];  row (p,b,i,j,t1,s1) holds
 *      frame t = i*T/N_T + t1, token s = j*S/N_S + p*S/(N_S*P) + s1.
 *   y, shard q: [B, N_T, N_S, T/(N_T*P), S/N_S, C];  row (q,b,i,j,t2,s2) holds
 *      frame t = i*T/N_T + q*T/(N_T*P) + t2, token s = j*S/N_S + s2.
 *   S2T reads x and writes y; T2S reads y and writes x.  N_T = N_S = 1 gives
 *   the plain [B,T,S/P,C] <-> [B,T/P,S,C] exchange.  Only destination rows
 *   of blocks i0 <= i < i1, j0 <= j < j1 are written (one partition of the
 *   inter-layer schedule); (0, N_T, 0, N_S) writes everything.
 *   Requires N_T*P | T and N_S*P | S.
 * ST_SEQ2HEAD / ST_HEAD2SEQ (T_or_N = N tokens, S_or_H = H, C_or_D = D):
 *   in,  shard p: [B, N/P, H, D]; out, shard q: [B, H/P, N, D] (heads outer so
 *   each head's sequence is contiguous).  HEAD2SEQ is the inverse.  n_t, n_s
 *   must be 1 and the block range (0, 1, 0, 1).  Requires P | N and P | H.
 * rms_gamma (optional, fp32 device [rms_head_dim]): apply per-head RMSNorm
 *   y = x / sqrt(mean(x^2) + rms_eps) * gamma to every rms_head_dim-wide
 *   head segment while moving it [CC "V-First"]; elem_bytes must then be 2
 *   (bf16) or 4 (fp32) and rms_head_dim must divide C (ST) or equal D.
 * elem_bytes: 1, 2, 4 or 8; rows are moved with the widest vector (up to 16
 *   bytes) that the row pitch and both pointers allow.
 * in and out must not overlap.
 * ---------------------------------------------------------------------- */
typedef enum { ST_S2T = 0, ST_T2S = 1, ST_SEQ2HEAD = 2, ST_HEAD2SEQ = 3 } st_relayout_mode;

st_status ulysses_relayout(st_relayout_mode mode, const void *in, void *out,
                           int elem_bytes, int P, int B, int T_or_N, int S_or_H,
                           int C_or_D, int n_t, int n_s, int i0, int i1, int j0,
                           int j1, const float *rms_gamma, int rms_head_dim,
                           float rms_eps, st_stream_t stream);

/* ulysses_relayout restricted to the temporally sharded shards q0 <= q < q1
 * of y as well: S2T writes only y shards q0..q1-1 (every row of them inside
 * the block range), T2S writes only the x rows whose frames come from those
 * y shards.  Each y shard's frames are contiguous in y, so a shard range is a
 * contiguous set of frames for the attention, V-Major and merge calls that
 * follow -- the unit of an intra-GPU chunk-and-overlap schedule in which the
 * exchange of one shard range runs while another range is attended [SF "四、
 * 核心创新" intra-layer schedule].  Any partition of (0, P) into ranges gives
 * the same bytes as one call.  (q0, q1) = (0, P) is ulysses_relayout; the
 * sequence/head modes accept only that.  ST_ERR_SHAPE for an empty or
 * out-of-range shard range. */
st_status ulysses_relayout_range(st_relayout_mode mode, const void *in, void *out,
                                 int elem_bytes, int P, int B, int T_or_N, int S_or_H,
                                 int C_or_D, int n_t, int n_s, int i0, int i1, int j0,
                                 int j1, int q0, int q1, const float *rms_gamma,
                                 int rms_head_dim, float rms_eps, st_stream_t stream);

/* Rotary position embedding [CC "V-First": Q and K receive RMSNorm and
 * RoPE, V neither].  Reading (the pages give no formula): the D channels of a
 * head form D/2 interleaved pairs (x[2i], x[2i+1]); pair i of the token at
 * position m turns by a = m * theta^(-2i/D):
 *     (x0, x1) -> (x0 cos a - x1 sin a, x0 sin a + x1 cos a),
 * applied after the RMSNorm.  A token's position is its index in the
 * sequence the attention runs over: s inside its frame (S2T, the spatial
 * layer) or n (SEQ2HEAD, image attention).
 *
 * st_rope_table fills table (fp32 device, [n_pos][head_dim / 2][2], 16-byte
 * aligned) with (cos a, sin a) for every position m < n_pos and pair i,
 * computed in double precision.  head_dim even, theta > 0. */
st_status st_rope_table(int n_pos, int head_dim, float theta, float *table,
                        st_stream_t stream);

/* ulysses_relayout (S2T or SEQ2HEAD, every block and shard) with the fused
 * per-head RMSNorm (rms_gamma required) followed by the rotary embedding of
 * every moved head from rope_table (st_rope_table), which must hold at least
 * S (S2T) or N (SEQ2HEAD) positions: rope_positions.  ST_ERR_UNSUPPORTED for
 * the inverse modes, ST_ERR_SHAPE for an odd head dim or a short table,
 * ST_ERR_ALIGN unless rope_table is 16-byte aligned. */
st_status ulysses_relayout_rope(st_relayout_mode mode, const void *in, void *out,
                                int elem_bytes, int P, int B, int T_or_N, int S_or_H,
                                int C_or_D, int n_t, int n_s, const float *rms_gamma,
                                int rms_head_dim, float rms_eps, const float *rope_table,
                                int rope_positions, st_stream_t stream);

/* ------------------------------------------------------------------------
 * V-Major selective communication [CC "V-Major"].
 * ---------------------------------------------------------------------- */

/* Bytes of device workspace vmajor_mask_compact needs for n_tokens. */
size_t vmajor_workspace_bytes(long long n_tokens);

/* Per-token change mask and compaction:
 *     L1_n   = sum_c |v_cur[n,c] - v_prev[n,c]|   (fp32 accumulation)
 *     mask_n = (L1_n > tau) || force_all
 *     idx    = ascending list of active n,  *count = |idx|
 *   v_cur, v_prev: dense [n_tokens, C] of dtype.  mask: u8 [n_tokens];
 *   idx: int32 [n_tokens] (entries past *count are left untouched);
 *   count: ONE int32 in device memory, so later kernels read it without a
 *   host round trip.  l1_out: optional fp32 [n_tokens] copy of L1_n.
 *   workspace: caller-owned device memory of at least
 *   vmajor_workspace_bytes(n_tokens) bytes (no state is kept in it between
 *   calls).  force_all = 1 is the periodic full refresh.
 *   Requires C*elem size to be a multiple of 16 bytes and 16-byte aligned
 *   v_cur/v_prev. */
st_status vmajor_mask_compact(const void *v_cur, const void *v_prev,
                              long long n_tokens, int C, st_dtype dtype, float tau,
                              int force_all, unsigned char *mask, int *idx,
                              int *count, float *l1_out, void *workspace,
                              size_t workspace_bytes, st_stream_t stream);

/* vmajor_mask_compact without a workspace argument, for callers that may not
 * allocate device memory while they run (a serving loop bound to a fixed
 * memory pool, or code that must not risk cudaMalloc stalling or failing
 * mid-step).  The paper has no counterpart; this is a library convenience.
 * Same arguments, results and errors as vmajor_mask_compact, except that the
 * per-tile counts live in a file-scope device array of 512 KiB that every GPU
 * loading the library keeps until the process exits.
 *   n_tokens above 4,194,304 (1 << 22) returns ST_ERR_SHAPE.
 *   Makes no cudaMalloc/cudaFree and no allocating library call.  The first
 *   call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current.  Under CUDA's lazy
 *   module loading that lookup may be what loads the library's device code
 *   on the device, and loading the code allocates its device globals, this
 *   array among them: make the first call at start-up, before any stream
 *   capture, and later calls allocate nothing.
 *   The address is cached per device for the life of the process: do not
 *   call this entry point again after cudaDeviceReset (or any other teardown
 *   of the device's context) in the same process -- the cached address would
 *   no longer belong to the new context.
 *   All calls share the one array (it keeps the last call's contents, and
 *   nothing in it needs to start at zero): calls whose work overlaps on the GPU
 *   (two streams, or two host threads) race and must be serialised by the
 *   caller. */
st_status vmajor_mask_compact_noalloc(const void *v_cur, const void *v_prev,
                                      long long n_tokens, int C, st_dtype dtype,
                                      float tau, int force_all, unsigned char *mask,
                                      int *idx, int *count, float *l1_out,
                                      st_stream_t stream);

/* Cache update for the active tokens: for i < *count (read on the device),
 *     dst_cache[t][idx[i], :] = src[t][idx[i], :]        for t < n_tensors
 * and, when packed is not NULL, packed[t][i, :] = src[t][idx[i], :] (the
 * message of active rows a rank would send).  Rows are C elements of
 * elem_bytes each.  src, dst_cache, packed: HOST arrays of n_tensors (1..8)
 * DEVICE pointers to dense [n_tokens, C] ([n_tokens, C] capacity for packed).
 * Inactive tokens keep their cached rows. */
st_status vmajor_scatter_rows(const int *idx, const int *count, long long n_tokens,
                              int C, int elem_bytes, const void *const *src,
                              void *const *dst_cache, int n_tensors,
                              void *const *packed, st_stream_t stream);

/* Sender-side V-Major [CC "V-Major"]: the tokens whose V changed take part
 * in the all-to-all, the others keep their cached rows.  v_cur_x and v_prev_x
 * are V of this and of the previous step in the spatially sharded layout x of
 * ulysses_relayout (ST_S2T shapes P, B, T, S, C, n_t, n_s); the L1 change of
 * every token is measured there, and the row of every active token moves to
 * its place in the temporally sharded layout y of v_cache_y (the V cache the
 * spatial attention reads); rows of inactive tokens are not written.  mask,
 * l1_out (optional), idx and count are those of vmajor_mask_compact in y
 * numbering (row r of y = destination row r of the S2T exchange), with the
 * same threshold rule, precision and determinism; workspace as for
 * vmajor_mask_compact with n_tokens = B*T*S.  v_cache_y must not overlap the
 * inputs.  Errors as for ulysses_relayout and vmajor_mask_compact. */
st_status vmajor_relayout_mask(const void *v_cur_x, const void *v_prev_x, void *v_cache_y,
                               int P, int B, int T, int S, int C, int n_t, int n_s,
                               st_dtype dtype, float tau, int force_all,
                               unsigned char *mask, int *idx, int *count, float *l1_out,
                               void *workspace, size_t workspace_bytes, st_stream_t stream);

/* The S2T move of ulysses_relayout restricted to the destination rows
 * idx[0], ..., idx[*count - 1] (y numbering, as listed by vmajor_relayout_mask;
 * idx and count are device memory): e.g. K of the active tokens into the K
 * cache [CC "V-Major"].  rms_gamma (optional, fp32 device [rms_head_dim])
 * applies the per-head RMSNorm of ulysses_relayout on the way, with the same
 * arithmetic, so a written row holds the same bytes as in the full relayout;
 * with it a row may hold at most 32 heads (else ST_ERR_UNSUPPORTED).
 * rope_table (optional, needs rms_gamma; see st_rope_table) then turns each
 * moved head by the rotary angles of its token's index s in the frame, as
 * ulysses_relayout_rope does; it must hold rope_positions >= S rows and be
 * 16-byte aligned (else ST_ERR_SHAPE / ST_ERR_ALIGN).  Rows
 * not listed are neither read nor written.  in_x and out_y must not overlap. */
st_status vmajor_relayout_rows(const void *in_x, void *out_y, const int *idx, const int *count,
                               int P, int B, int T, int S, int C, int n_t, int n_s,
                               st_dtype dtype, const float *rms_gamma, int rms_head_dim,
                               float rms_eps, const float *rope_table, int rope_positions,
                               st_stream_t stream);

/* vmajor_mask_compact and vmajor_scatter_rows (without `packed`) in one call
 * [CC "V-Major" section]: the pass that decides a token is active also copies
 * its rows of every src tensor into dst_cache, so the cache update reads no
 * index list and the mask pass's rows are still in cache.  Arguments,
 * results and errors as the two calls (src[t] and dst_cache[t] are dense
 * [n_tokens, C] of dtype, 16-byte aligned; src may include v_cur).  Same
 * mask, idx, count and caches as the two calls, bit for bit. */
st_status vmajor_mask_compact_scatter(const void *v_cur, const void *v_prev,
                                      long long n_tokens, int C, st_dtype dtype, float tau,
                                      int force_all, unsigned char *mask, int *idx, int *count,
                                      float *l1_out, void *workspace, size_t workspace_bytes,
                                      const void *const *src, void *const *dst_cache,
                                      int n_tensors, st_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word that
 * bounded waits set.  Returns ST_ERR_TIMEOUT if a wait ran out since the last
 * call, ST_ERR_CUDA if the stream reports an error, else ST_OK. */
st_status st_check_device_status(st_stream_t stream);

/* SM budget of the calling host thread: the grids of the kernels it launches
 * afterwards are sized for at most `sms` SMs (persistent kernels start at
 * most one resident wave of that many SMs; 0 restores the whole device).
 * Used to share the GPU between two streams, e.g. attention on most SMs while
 * the memory-bound steps of the next shard range run on the rest; results do
 * not depend on it.  Host-side only (not stream-ordered); ST_ERR_SHAPE for a
 * negative count. */
st_status st_set_sm_budget(int sms);
int st_get_sm_budget(void);

/* Failure-detection self test: launches a one-thread kernel that waits, with
 * a 20 ms limit, on an mbarrier nothing ever arrives on, through the same
 * bounded-wait path the tensor-core attention kernel uses.  The wait runs
 * out, the kernel records it and returns; a following
 * st_check_device_status(stream) must report ST_ERR_TIMEOUT (and clears the
 * word).  Nothing faults, traps or hangs. */
st_status st_selftest_wait_timeout(st_stream_t stream);

/* Exponential self test: for each of the n fp32 values x[i] (device), writes
 * the two base-2 exponentials the attention kernel's softmax uses, evaluated
 * by the same device functions:
 *   y_poly[i]: 2^x on the FMA pipe -- range reduction x = j + f with j the
 *     nearest integer, 2^f from a degree-3 polynomial (coefficients from a
 *     Remez exchange on relative error over [-1/2, 1/2], maximum relative
 *     error 7.48e-5 before fp32 rounding), 2^j added into the exponent; x is
 *     clamped below at -125 and must be <= 8 (the softmax's arguments are
 *     scores minus a running max that trails the true max by at most 8);
 *   y_mufu[i]: ex2.approx.ftz.f32 on the special-function unit.
 * Device pointers, 4-byte aligned; n >= 0.  ST_ERR_NULL / ST_ERR_ALIGN /
 * ST_ERR_SHAPE on bad arguments.  Not part of the pages' method: it exists so
 * that the tests can bound the error of the kernel's exponentials. */
st_status st_selftest_ex2(const float *x, float *y_poly, float *y_mufu, int n,
                          st_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* STATTN_H */
