/*
 * lrkv.h - C ABI of the split-value-cache attention library (liblrkv.so).
 *
 * Several LoRA role adapters ("agents") attend over ONE shared base K/V cache.
 * The value projection of agent i splits exactly as
 *     V_i = X W0 + (X A_i) B_i
 * ("LRAgent: Efficient KV Cache Sharing for Multi-LoRA LLM Agents", Pith
 * review, "What carries the argument", Eq. 3), so the base cache X W0 is stored
 * once and each agent keeps only the rank-r cache U_i = X A_i.  Attention is
 * computed in the reordered form of Eq. 12 of the same page,
 *     O_h = P_h V_base,g + (P_h Umask_i) B_i,g,   P_h = softmax(q_h K_base,g^T * scale),
 * without ever forming an L x d_out adapter cache.  Keys carry no adapter term
 * (same page: key caches are shared, Fig. 7).  Umask_i is U_i with the rows
 * before the agent's aLoRA activation offset a_i removed ("RoleKV", Devpost,
 * "What it does": the adapter switches on only after the role header; the
 * offsets are passed explicitly, "Challenges we ran into").
 *
 * Notation: S sessions, N agents, Hq query heads, Hkv KV heads, G = Hq / Hkv,
 * d head_dim, r rank.  Query head h of agent i reads KV head g = h / G and the
 * column slice B_i[:, g*d : (g+1)*d].  U_i is one [rows, r] cache per
 * (session, agent) shared by every KV head.  Sharing modes (LRAgent page,
 * Fig. 2-3): LRKV_BASE_SHARED keeps one U_i per agent; LRKV_BASE_LR_SHARED
 * (one shared down-projection A) keeps ONE U for all agents, still masked by
 * each agent's own offset.
 *
 * Conventions of every entry point:
 *  - Ownership: the caller owns every buffer.  The library allocates and frees
 *    nothing, and never copies device memory to the host (the exceptions are
 *    the two status queries, which exist to do exactly that).
 *  - Pointers documented as "device" must be device (or managed) memory of the
 *    current device.  Tensors are bf16 unless stated.  Base addresses of q, K,
 *    V, U, B and out must be 16-byte aligned, and the token/head/session/page
 *    strides of K, V and U must be multiples of 8 elements (16 bytes): the
 *    tiles are moved by the Tensor Memory Accelerator.
 *  - Streams: every launch goes on the caller's stream (a cudaStream_t; 0 is
 *    the legacy default stream).  No call synchronises, except the status
 *    queries lrkv_query_device_status and lrkv_query_static_scratch_status.
 *  - Errors: every call returns an lrkv_status and never throws.  Host-side
 *    argument errors return before anything is launched.  Device-side checks
 *    (a seq_len beyond max_seq_len, a negative offset, a page id out of range,
 *    a bounded wait that gave up) never fault: they record a flag in the
 *    workspace and are read back with lrkv_query_device_status (the
 *    static-scratch decode: lrkv_query_static_scratch_status).  After a
 *    timeout, reset the workspace (lrkv_workspace_reset) before reusing it:
 *    the abandoned launch may have left its merge tickets counting.
 *    lrkv_last_error_detail() gives a thread-local text for the last failure.
 *    A pointer argument not documented as optional ("or NULL") must not be
 *    NULL: LRKV_ERR_INVALID_ARGUMENT.
 *  - Supported: an sm_100 GPU (B200) as the current device; head_dim in
 *    {64, 128}; rank in {8, 16, 32}; Hq a multiple of Hkv; page_size 64; at
 *    most 16 agents per call.  Anything else returns LRKV_ERR_UNSUPPORTED.
 */
#ifndef LRKV_H
#define LRKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* lrkv_stream_t;

typedef enum {
  LRKV_OK = 0,
  LRKV_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad size, inconsistent view        */
  LRKV_ERR_UNSUPPORTED = 2,        /* head_dim / rank / page size / GPU not supported  */
  LRKV_ERR_MISALIGNED = 3,         /* base address or stride not 16-byte aligned       */
  LRKV_ERR_WORKSPACE_TOO_SMALL = 4,
  LRKV_ERR_CUDA = 5,               /* a CUDA runtime or driver call failed             */
  LRKV_ERR_DEVICE_FAULT = 6,       /* a device-side check flagged bad data             */
  LRKV_ERR_TIMEOUT = 7             /* a bounded wait inside a kernel gave up           */
} lrkv_status;

typedef enum { LRKV_BASE_SHARED = 0, LRKV_BASE_LR_SHARED = 1 } lrkv_mode;
typedef enum { LRKV_BF16 = 0, LRKV_F32 = 1 } lrkv_dtype;

/* Problem shape shared by the attention calls. */
typedef struct {
  int32_t num_sessions;   /* S  (decode: sessions in the batch; prefill: sessions the views index) */
  int32_t num_agents;     /* N                                                                     */
  int32_t num_q_heads;    /* Hq                                                                    */
  int32_t num_kv_heads;   /* Hkv, Hq % Hkv == 0                                                    */
  int32_t head_dim;       /* d in {64, 128}                                                        */
  int32_t rank;           /* r in {8, 16, 32}                                                      */
  int32_t mode;           /* lrkv_mode                                                             */
  float softmax_scale;    /* 0 => 1/sqrt(head_dim); LoRA's alpha/r is folded into B by the caller  */
} lrkv_problem;

/*
 * The shared base K/V cache (bf16, head_dim contiguous).  K and V use the same
 * layout and strides (in elements).
 *  Dense  (page_table == NULL): element (s, g, t, e) at s*stride_session +
 *         g*stride_head + t*stride_token + e.  Each (s, g) holds at least the
 *         call's max_seq_len (decode) or ctx_len+T (prefill) token rows.
 *  Paged  (page_table != NULL): physical page p holds page_size tokens of every
 *         KV head: element (p, g, j, e) at p*stride_page + g*stride_head +
 *         j*stride_token + e.  Logical token t of session s lives in page
 *         page_table[s*page_table_stride + t/page_size], slot t % page_size
 *         (a paged cache is the route to physical sharing named in "Shared-Prefix
 *         KV Reuse Across Standard LoRA Adapters", section 3.2).  page_table is
 *         device int32; num_pages bounds every id (an id outside [0, num_pages)
 *         is skipped and flagged on the device).
 */
typedef struct {
  const void* k;
  const void* v;
  int64_t stride_session;
  int64_t stride_head;
  int64_t stride_token;
  const int32_t* page_table;
  int64_t page_table_stride;
  int64_t stride_page;
  int32_t page_size;
  int32_t num_pages;
} lrkv_kv_view;

/*
 * Low-rank caches U (bf16, rank contiguous).  Row t of agent slot i of
 * session s at u + s*stride_session + i*stride_agent + t*stride_token.
 * Agent slots: N in BaseShared, 1 in BaseLRShared.  num_rows is the row
 * capacity of each (session, agent) cache.  Rows before an agent's offset and
 * rows at or past seq_len are never read into the result (they may hold
 * anything, NaN included).
 */
typedef struct {
  void* u;
  int64_t stride_session;
  int64_t stride_agent;
  int64_t stride_token;
  int32_t num_rows;
} lrkv_u_view;

/* ---------------------------------------------------------------------- */
/* Low-rank cache append.                                                  */
/* ---------------------------------------------------------------------- */

/*
 * U_i[start_row + t, :] = X[t, :] A_i  for t in [0, T) and every agent slot
 * i in [0, n_a), in session `session` of u_dst (LRAgent page, Eq. 3: the
 * rank-r cache X A_i; Fig. 3: it is computed for the tokens the agent has not
 * processed yet).  In BaseLRShared pass the one shared A with n_a = 1.
 *   x   device bf16 [T, Dm], row-major (one X shared by all agents)
 *   a   device bf16 [n_a, Dm, r], row-major
 * Numerics, a fixed contract: acc = +0.0f; for k = 0 .. Dm-1 in order,
 * acc = fmaf(x[t,k], a[k,j], acc); then round to nearest even bf16.  The
 * bf16 x bf16 product is exact in fp32, so the result is bit-determined.
 * Errors: start_row < 0, start_row + T > u_dst->num_rows, n_a < 1, T < 0,
 * Dm < 1 return LRKV_ERR_INVALID_ARGUMENT.  T == 0 is a no-op.
 */
lrkv_status lrkv_append_lr_cache(const void* x, const void* a, int32_t n_a, int32_t T,
                                 int32_t Dm, int32_t r, const lrkv_u_view* u_dst,
                                 int32_t session, int32_t start_row, lrkv_stream_t stream);

/*
 * Catch-up append over per-agent ranges: for every agent slot i in [0, n_a),
 * U_i[t, :] = X[t, :] A_i for t in [row_begin[i], row_end[i]) of session
 * `session` of u_dst (LRAgent page, Fig. 3(a): in BaseShared every agent
 * computes its own rank-r cache for the context tokens it has not processed
 * yet, so the ranges differ per agent; Fig. 3(b): in BaseLRShared the one
 * shared U is appended once: n_a = 1).  X row t is the hidden state of
 * absolute position t.
 *   x          device bf16 [x_rows, Dm], row-major
 *   a          device bf16 [n_a, Dm, r], row-major
 *   row_begin, row_end   HOST int32 [n_a] (the caller's scheduler knows them)
 * Same fixed-order numerics as lrkv_append_lr_cache (bit-determined).  Rows
 * outside each agent's range are not written.  Empty ranges are no-ops.
 * Errors: a range with row_begin < 0, row_begin > row_end, row_end > x_rows or
 * row_end > u_dst->num_rows, n_a < 1, Dm < 1 return LRKV_ERR_INVALID_ARGUMENT;
 * r not in {8, 16, 32} returns LRKV_ERR_UNSUPPORTED.
 */
lrkv_status lrkv_append_lr_cache_ranges(const void* x, int32_t x_rows, const void* a, int32_t n_a, int32_t Dm,
                                        int32_t r, const int32_t* row_begin, const int32_t* row_end,
                                        const lrkv_u_view* u_dst, int32_t session, lrkv_stream_t stream);

/* ---------------------------------------------------------------------- */
/* Decode: one query token per (session, agent) over the shared cache.     */
/* ---------------------------------------------------------------------- */

/*
 * Bytes of workspace lrkv_attn_decode needs for this shape and host-side
 * bound max_seq_len on the current device; 0 if the shape is invalid.
 */
size_t lrkv_decode_workspace_bytes(const lrkv_problem* p, int32_t max_seq_len);

/*
 * out[s, i, h, :] = sum_{t < seq_lens[s]} P[t] (V_base,g[t] + [t >= a_{s,i}] U_i[t] B_i,g)
 * with P = softmax(q[s,i,h] . K_base,g[t] * scale) over t < seq_lens[s].
 * Computed as P V_base + (P Umask_i) B_i: the rank-r accumulator is kept
 * per query row and B_i is applied once per row in the epilogue.
 *   q              device bf16 [S, N, Hq, d] contiguous
 *   kv             the shared base cache (dense or paged)
 *   seq_lens       device int32 [S]; each in [0, max_seq_len]
 *   max_seq_len    host-side bound on seq_lens (sizes the split of the work)
 *   u              low-rank caches; u->num_rows >= max_seq_len
 *   b              device bf16 [N, r, Hkv*d] contiguous
 *   alora_offsets  device int32 [S, N] (a_{s,i}), or NULL for all zero
 *   out            device [S, N, Hq, d] contiguous, bf16 or fp32 (out_dtype)
 *   workspace      device, >= lrkv_decode_workspace_bytes(p, max_seq_len),
 *                  16-byte aligned, zero-filled once before its first use
 *                  (lrkv_workspace_reset); every call leaves it reusable.
 *                  Calls that share a workspace must be ordered (same stream).
 * A session with seq_len 0 gets a zero output.
 */
lrkv_status lrkv_attn_decode(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv,
                             const int32_t* seq_lens, int32_t max_seq_len,
                             const lrkv_u_view* u, const void* b,
                             const int32_t* alora_offsets, void* out, int32_t out_dtype,
                             void* workspace, size_t workspace_bytes, lrkv_stream_t stream);

/*
 * Decode over a contiguous range of KV heads: the query heads h with
 * h / G in [kv_head_begin, kv_head_begin + kv_head_count), same result for
 * them as lrkv_attn_decode.  Every KV head's rows read only its own K/V slice
 * and its own column slice of B_i (Eq. 12 of the LRAgent page holds per head),
 * so the heads of a model can be split over GPUs with no exchange: each GPU
 * holds the K/V of its heads (the paged long-context case is 30 GB of base K/V
 * in 28 layers; the LRAgent page, Fig. 5, shows how such caches outgrow one
 * device), its own copy of q, U and B, and writes its heads of out.
 *   p            the whole problem (num_kv_heads = the model's Hkv)
 *   kv           the shard: its head 0 is KV head kv_head_begin; K and V hold
 *                kv_head_count heads (dense or paged, layout as above)
 *   q, b, out    the whole problem's tensors ([S, N, Hq, d], [N, r, Hkv*d],
 *                [S, N, Hq, d]); out rows of other heads are not written
 *   workspace    >= lrkv_decode_kv_heads_workspace_bytes(p, kv_head_count, ...)
 * Other arguments as lrkv_attn_decode.  A range outside [0, Hkv) or an empty
 * one returns LRKV_ERR_INVALID_ARGUMENT.  The split of the keys between CTAs
 * depends on the number of heads in the launch, so a shard's output may differ
 * from the same heads of a whole-problem call by fp32 rounding (both are within
 * the stated tolerance of the exact result).
 */
size_t lrkv_decode_kv_heads_workspace_bytes(const lrkv_problem* p, int32_t kv_head_count, int32_t max_seq_len);
lrkv_status lrkv_attn_decode_kv_heads(const lrkv_problem* p, int32_t kv_head_begin, int32_t kv_head_count,
                                      const void* q, const lrkv_kv_view* kv, const int32_t* seq_lens,
                                      int32_t max_seq_len, const lrkv_u_view* u, const void* b,
                                      const int32_t* alora_offsets, void* out, int32_t out_dtype,
                                      void* workspace, size_t workspace_bytes, lrkv_stream_t stream);

/*
 * Decode with the library's own scratch, for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a convenience of the
 * library, not part of the method.
 *
 * Who needs it: code whose device memory belongs to someone else's allocator
 * (a serving engine that hands its plug-ins only tensors), and code for which a
 * cudaMalloc is not acceptable at call time - cudaMalloc synchronises the whole
 * device, and on a long-running server with a fragmented heap it can fail even
 * when enough memory is free in total.
 *
 * Same arguments and result as lrkv_attn_decode, minus the workspace.  The
 * scratch is one file-scope device array of LRKV_STATIC_SCRATCH_BYTES that
 * every GPU which loads the library keeps until the process exits.  The call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *  - Shapes whose lrkv_decode_workspace_bytes() exceeds the scratch size return
 *    LRKV_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *  - The first call on a device looks up the scratch's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call clears the scratch's flag and ticket words on `stream`, then
 *    runs the same kernel as lrkv_attn_decode.  All calls share the one array
 *    and it keeps the last call's contents, so calls that can overlap on the GPU
 *    (different streams, or different host threads on one device) race and
 *    give wrong results: order them.  The device-side flags of the most recent
 *    call (a bad seq_len, offset or page id, a bounded wait that gave up) stay
 *    in the scratch until the next call clears them: read them with
 *    lrkv_query_static_scratch_status.
 */
#define LRKV_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
lrkv_status lrkv_attn_decode_static_scratch(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv,
                                            const int32_t* seq_lens, int32_t max_seq_len,
                                            const lrkv_u_view* u, const void* b,
                                            const int32_t* alora_offsets, void* out, int32_t out_dtype,
                                            lrkv_stream_t stream);

/*
 * The device-side flags of the most recent lrkv_attn_decode_static_scratch call
 * on the current device: synchronise `stream`, read them and, when `clear` is
 * non-zero, reset them.  Same results as lrkv_query_device_status (LRKV_OK,
 * LRKV_ERR_DEVICE_FAULT, LRKV_ERR_TIMEOUT; *flags_out gets the raw bits).
 * Like the scratch itself this has no counterpart on the pages.
 */
lrkv_status lrkv_query_static_scratch_status(int32_t clear, uint32_t* flags_out, lrkv_stream_t stream);

/* ---------------------------------------------------------------------- */
/* Prefill chunk: T new rows per agent, causal, over one session.          */
/* ---------------------------------------------------------------------- */

/* Bytes of workspace lrkv_attn_prefill_chunk needs; 0 if the call would refuse
 * the shape.  It holds the status header, one ticket per 128-row tile and the
 * partial (m, l, O, Z) rows of tiles whose key blocks are split between CTAs
 * (the blocks of all tiles are divided evenly over one CTA per SM). */
size_t lrkv_prefill_workspace_bytes(const lrkv_problem* p, int32_t ctx_len, int32_t T);

/*
 * Row j of agent i sits at absolute position ctx_len + j and attends to keys
 * t <= ctx_len + j of session `session` (bottom-right causal alignment):
 * out[i, j, h, :] = sum_t P[t] (V_base,g[t] + [t >= a_i] U_i[t] B_i,g).
 * The chunk's own base K/V must already be in the cache at rows
 * [ctx_len, ctx_len + T), and its U rows appended (lrkv_append_lr_cache).
 * A role switch ("RoleKV", "What it does") is such a chunk: the new role's
 * header rows over the shared context, its adapter active from its offset.
 * Supported set: the global one (any G = Hq / Hkv up to 128; every rank).
 * Numerics: bf16 Q K^T and P [V | U] on the tensor cores with fp32
 * accumulation; the rank-r accumulator Z = P Umask_i enters Z B_i,g as two
 * bf16 terms (Z = Z_hi + Z_lo), about 2^-17 of |Z| from the fp32 value.
 *   q              device bf16 [N, T, Hq, d] contiguous
 *   kv, u          views as above (u->num_rows >= ctx_len + T)
 *   b              device bf16 [N, r, Hkv*d]
 *   alora_offsets  device int32 [N], or NULL for all zero
 *   out            device [N, T, Hq, d] contiguous, bf16 or fp32
 *   workspace      device, >= lrkv_prefill_workspace_bytes, zero-filled once
 *                  (the tickets return to zero by the end of every call; calls
 *                  sharing a workspace must be ordered on one stream)
 */
lrkv_status lrkv_attn_prefill_chunk(const lrkv_problem* p, const void* q, const lrkv_kv_view* kv,
                                    int32_t session, int32_t ctx_len, int32_t T,
                                    const lrkv_u_view* u, const void* b,
                                    const int32_t* alora_offsets, void* out, int32_t out_dtype,
                                    void* workspace, size_t workspace_bytes,
                                    lrkv_stream_t stream);

/* ---------------------------------------------------------------------- */
/* Workspace and status.                                                   */
/* ---------------------------------------------------------------------- */
/* Value projection into the split caches.                                 */
/* ---------------------------------------------------------------------- */

/*
 * [V_base | U_1 ... U_n] = X [W0_v | A_1 ... A_n] for T new tokens, written
 * into the caches: base value rows start_row .. start_row+T-1 of session
 * `session` for every KV head (kv->v; kv->k is not touched), and the same rows
 * of every low-rank slot of u_dst (LRAgent page, Eq. 3: agent i's value
 * projection splits as X W0 + (X A_i) B_i, so one product with the weights side
 * by side gives the shared base values and all U_i rows).
 *   x        device bf16 [T, Dm] row-major, Dm % 8 == 0
 *   w        device bf16 [Dm, Hkv*d + n_u*r] row-major: W0_v (KV head g in
 *            columns [g d, (g+1) d)), then A_1 .. A_{n_u} (r columns each);
 *            n_u = N in BaseShared, 1 in BaseLRShared
 *   kv       dense: kv_rows is the row capacity of each (session, head);
 *            paged: rows map through the session's page-table row
 *   workspace  device, >= 256 bytes, zero-filled once: status flags
 * Numerics: bf16 inputs, fp32 accumulation on the tensor cores in an
 * unspecified order, round to nearest even bf16.  The U rows are therefore not
 * bit-identical to lrkv_append_lr_cache's fixed-order ones.
 * Errors: invalid shapes or rows past the caches return
 * LRKV_ERR_INVALID_ARGUMENT, unaligned pointers or strides LRKV_ERR_MISALIGNED;
 * an out-of-range page id sets a device flag (lrkv_query_device_status) and
 * that row's values are not written.  T == 0 is a no-op.
 */
lrkv_status lrkv_value_projection(const lrkv_problem* p, const void* x, int32_t T, int32_t Dm, const void* w,
                                  const lrkv_kv_view* kv, int32_t kv_rows, const lrkv_u_view* u_dst,
                                  int32_t session, int32_t start_row, void* workspace, size_t workspace_bytes,
                                  lrkv_stream_t stream);

/* ---------------------------------------------------------------------- */

/* Zero-fill a workspace on `stream` (asynchronous). */
lrkv_status lrkv_workspace_reset(void* workspace, size_t workspace_bytes, lrkv_stream_t stream);

/*
 * Synchronise `stream`, read the device-side flags of `workspace` and, when
 * `clear` is non-zero, reset them.  Returns LRKV_OK, LRKV_ERR_DEVICE_FAULT
 * (bad seq_len, offset or page id seen) or LRKV_ERR_TIMEOUT (a bounded wait
 * gave up).  *flags_out (if not NULL) receives the raw flag bits.
 */
lrkv_status lrkv_query_device_status(const void* workspace, int32_t clear, uint32_t* flags_out,
                                     lrkv_stream_t stream);

/*
 * Failure-detection test hook (no counterpart on the pages: it tests the
 * library's own error path).  Arms the next lrkv_attn_decode,
 * lrkv_attn_decode_static_scratch or lrkv_attn_prefill_chunk call made from
 * this host thread: in that launch the copy-issuing warps issue nothing and
 * every bounded wait gives up after `spin_cap` failed attempts, so the waits
 * run out the way they would if a copy never arrived.  The launch records
 * LRKV_DEVFLAG_TIMEOUT (lrkv_query_device_status then returns
 * LRKV_ERR_TIMEOUT), leaves its output undefined, and returns with no copy or
 * tensor-core operation in flight, so the context stays usable; reset the
 * workspace before reusing it.  spin_cap 0 disarms.  Never faults, traps or
 * hangs the GPU: every wait stays bounded.
 */
lrkv_status lrkv_debug_stall_next_launch(uint32_t spin_cap);

const char* lrkv_status_string(lrkv_status s);
const char* lrkv_last_error_detail(void);
/* Library version as major*10000 + minor*100 + patch. */
int32_t lrkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LRKV_H */
