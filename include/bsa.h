/*
 * bsa.h -- C ABI of the B200 (sm_100a) block-sparse causal attention
 * forward, its gradients, selected-page decode and BSBR's between-chunk
 * retrieval term.
 *
 * What the library computes ("Block-Sparse Attention", ai-model-reference,
 * sections "How It Works" and "Math Or Compute Schema"): the sequence of n
 * tokens is cut into blocks of B tokens; query block i attends densely only
 * to the key blocks its block mask M_B keeps; every dropped pair gets -inf
 * before the softmax (scale 1/sqrt(d) in every shipped workload); inside the
 * diagonal block the token-level causal mask applies (key u <= query t), as
 * in "bsbr" ("Solution", the within-chunk causal mask M_in) and in BF1
 * (section 3.1, the self block is read causally).  Block masks are compiled on
 * the host into CSR form ("Block Sparse Attention in LLMs", section 6: the
 * allowed_blocks list per query block).
 *
 * Conventions shared by every call:
 *   - Every function returns a bsa_status (0 = BSA_OK); nothing throws or
 *     aborts.  bsa_last_error() gives a message for the calling thread.
 *   - Tensors are caller-owned device pointers: q is [heads][n][d] bf16,
 *     k and v are [kv_heads][n][d] bf16, o is [heads][n][d] bf16 and lse is
 *     [heads][n] float32, all contiguous.  A batch of b sequences with H
 *     query heads and Hk key/value heads is passed folded: heads = b*H,
 *     kv_heads = b*Hk.  Query slice f reads key/value slice
 *     f / (heads / kv_heads) (contiguous grouped-query sharing) and layout
 *     head f % layout_heads.
 *   - Streams are caller-owned cudaStream_t values passed as void* (NULL is
 *     the legacy default stream).  bsa_forward is asynchronous on that stream
 *     and allocates nothing.
 *   - A bsa_layout is library-owned: created only by bsa_build_layout (so it
 *     is always valid and causal) and released only by bsa_free.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad scale, wrong device ...  */
  BSA_ERR_SHAPE = 2,          /* sizes inconsistent with each other or with the layout */
  BSA_ERR_UNSUPPORTED = 3,    /* a size the kernels are not built for (B, d)           */
  BSA_ERR_NONCAUSAL = 4,      /* an explicit block mask keeps a block j > i            */
  BSA_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed                     */
  BSA_ERR_OOM = 6,            /* host or device allocation failed                      */
  BSA_ERR_DEVICE_TIMEOUT = 7  /* a kernel wait ran out; the kernel returned early      */
} bsa_status;

/* Block-layout families.
 *  BAND_GLOBAL: kept(i) = {max(0, i-window) .. i}, plus block 0 when
 *      global_first != 0.  window = 0, global_first = 0 is BSBR's
 *      within-chunk (block-diagonal) term ("bsbr", "Solution"); window >= 1
 *      with block 0 is the local band plus global anchor block ("Block-Sparse
 *      Attention", "How It Works"; "Block Sparse Attention in LLMs", 5B).
 *  DYADIC: BAND_GLOBAL(window, global_first) plus i - 2^k for every
 *      k >= dyadic_kmin with i - 2^k >= 0 (BF1, Method and section 3.1:
 *      self, two local predecessors, the first block and dyadic predecessors;
 *      window = 2, global_first = 1, dyadic_kmin = 2).  Sets, so overlaps
 *      count once.
 *  RANDOM: static random mask (BF1's "static-random graph" control, whose
 *      generator is unpublished; this library's reading): the diagonal and
 *      block 0 are always kept; row i keeps
 *      min(i+1, max(mandatory, floor((ppm*(i+1) + 500000) / 1000000)))
 *      blocks, ppm = round(density * 1e6); the others are drawn uniformly
 *      without replacement from {1 .. i-1} by a partial Fisher-Yates shuffle
 *      (draw t swaps candidate t with candidate t + x mod (i-1-t)), x being
 *      successive SplitMix64 outputs from state seed + (h+1)*0x9E3779B97F4A7C15
 *      for layout head h, rows taken in order.
 *  EXPLICIT: the caller's block mask M_B ("Block-Sparse Attention", "Math Or
 *      Compute Schema"): mask[h][i][j] != 0 keeps key block j for query
 *      block i of layout head h.  Any kept j > i gives BSA_ERR_NONCAUSAL.
 *      Rows may be empty (their output is o = 0, lse = -inf). */
typedef enum bsa_pattern_kind {
  BSA_PATTERN_BAND_GLOBAL = 0,
  BSA_PATTERN_DYADIC = 1,
  BSA_PATTERN_RANDOM = 2,
  BSA_PATTERN_EXPLICIT = 3
} bsa_pattern_kind;

typedef struct bsa_pattern {
  int32_t kind;          /* bsa_pattern_kind                                        */
  int32_t window;        /* BAND_GLOBAL/DYADIC: local predecessors kept (>= 0)      */
  int32_t global_first;  /* BAND_GLOBAL/DYADIC: nonzero keeps block 0               */
  int32_t dyadic_kmin;   /* DYADIC: smallest exponent k of the offsets 2^k (>= 0)   */
  double density;        /* RANDOM: target fraction of causal blocks, in [0, 1]     */
  uint64_t seed;         /* RANDOM: generator seed                                  */
  const uint8_t* mask;   /* EXPLICIT: host array [layout_heads][nb][nb], row-major,
                            read only during bsa_build_layout; else ignored         */
} bsa_pattern;

typedef struct bsa_layout bsa_layout;   /* opaque */

/* Compile a pattern into a block layout for sequences of n tokens in blocks of
 * B tokens (nb = ceil(n / B); a shorter last block is allowed).
 * layout_heads >= 1 separate layouts are built (the RANDOM family draws each
 * from its own stream; the other families repeat the same rows).
 * Produces, on the host: row_ptr[layout_heads*nb + 1] and col_idx[nnz]
 * (rows in order head-major, columns strictly ascending, all <= the row's
 * block index), and the longest-row-first order of each layout head's rows
 * (ties broken by ascending row).  When device >= 0 the three arrays and a
 * device status word are uploaded to that device synchronously; device = -1
 * builds a host-only layout (inspection and tests; bsa_forward rejects it).
 * On success *out owns everything; release it with bsa_free. */
int bsa_build_layout(const bsa_pattern* spec, int n, int B, int layout_heads,
                     int device, bsa_layout** out);

/* Read-only host view of a layout's CSR arrays; valid until bsa_free.
 * rows = layout_heads * nb. */
int bsa_layout_csr(const bsa_layout* layout, const int32_t** row_ptr,
                   const int32_t** col_idx, int* rows, int* nnz);

/* Read-only host view of the longest-row-first order: order[h*nb + r] is the
 * query block processed at rank r for layout head h.  count = layout_heads*nb. */
int bsa_layout_order(const bsa_layout* layout, const int32_t** order, int* count);

/* Read-only host view of the forward's work table: for layout head h and rank
 * r in the longest-row-first order, work[4*(h*nb + r) .. +3] = (query block
 * order[h*nb + r], its first entry in col_idx, its kept-block count, 1 if its
 * last kept block is the diagonal one else 0): one work item of bsa_forward
 * decodes from one such entry.  count = layout_heads*nb entries (4 words
 * each); uploaded with the layout and staged by bsa_forward_noalloc. */
int bsa_layout_work(const bsa_layout* layout, const int32_t** work, int* count);

/* Read-only host view of the transposed layout: for layout head h and key
 * block j, row_idx[col_ptr[h*nb + j] .. col_ptr[h*nb + j + 1]) lists, in
 * ascending order, the query blocks whose rows keep j (the key/value side of
 * the gradients reads the layout this way).  cols = layout_heads * nb. */
int bsa_layout_csc(const bsa_layout* layout, const int32_t** col_ptr,
                   const int32_t** row_idx, int* cols, int* nnz);

/* Block-sparse causal attention forward on the caller's stream.
 * For every folded query head f and token t (block i = t / B):
 *   s_tu = scale * <q[f][t], k[g][u]>,  g = f / (heads / kv_heads),
 *   over the keys u allowed by layout head f % layout_heads (block j of u kept
 *   by block i, and j < i or u <= t);
 *   lse[f][t] = ln sum_u exp(s_tu),  o[f][t] = sum_u exp(s_tu - lse) v[g][u].
 * Rows with no allowed key get o = 0 and lse = -inf.
 * Requirements (checked before anything is launched; violations return an
 * error and launch nothing): layout built for this n and B on the current
 * device; B in {64, 128}; d in {64, 128}; heads and kv_heads >= 1,
 * heads % kv_heads == 0, heads % layout_heads == 0; scale finite and > 0;
 * q, k, v, o non-null and 16-byte aligned; lse non-null and 4-byte aligned.
 * o and lse must not overlap the inputs.  Enqueues one kernel and returns.
 * Work counters: each call takes the next of 64 work counters held in the
 * layout's device block (the kernel leaves it at zero when it ends), so
 * forwards and backwards with the same layout may run at the same time on
 * different streams.  A call that comes back to a counter makes its stream
 * wait for the previous call on that counter (an event the library records
 * after each call), so any number of calls may be in flight: beyond 64 the
 * calls are ordered, never mixed.  A call made while `stream` is capturing a
 * CUDA graph gets one of 192 further counters of its own for good (the
 * captured launch replays on it; replays of one graph run one after another)
 * and BSA_ERR_UNSUPPORTED once those are used up.  The layout is locked
 * while a call enqueues its work, so calls from several host threads are
 * safe.  A device-side wait that runs out (never expected) makes the kernel
 * return early and is reported by bsa_get_status. */
int bsa_forward(const void* q, const void* k, const void* v,
                const bsa_layout* layout, int B, int n, int heads, int kv_heads,
                int d, float scale, void* o, float* lse, void* stream);

/* Synchronise `stream`, then read and clear the layout's device status word:
 * BSA_OK, or BSA_ERR_DEVICE_TIMEOUT if any forward on this layout since the
 * last call had a wait run out.  For a host-only layout (device = -1) the
 * word read is the status of the most recent bsa_forward_noalloc call on the
 * current device. */
int bsa_get_status(const bsa_layout* layout, void* stream);

/* Diagnostics: launch the forward kernel of this layout's shape in a mode
 * where every thread waits on a barrier that nothing completes, with the
 * given wait limit in nanoseconds (at most 10^9), so that the bounded-wait
 * path runs: the kernel records BSA_ERR_DEVICE_TIMEOUT in the status word and
 * returns; nothing is read or written besides the status word. */
int bsa_debug_timeout_probe(const bsa_layout* layout, int d, uint64_t timeout_ns,
                            void* stream);

/* The forward from and to host memory (the end-to-end form of bsa_forward):
 * q, k, v are copied from q_host, k_host, v_host into the caller's device
 * buffers q, k, v, the forward runs, and o, lse are copied back into o_host,
 * lse_host.  The work is cut into `groups` runs of whole key/value heads (at
 * most kv_heads; fewer when layout heads require coarser runs, since every
 * run must start at a query head of layout head 0), and run i + 1's
 * host-to-device copies, run i's forward and run i - 1's device-to-host
 * copies proceed at the same time: two copy streams of the library (created
 * once per device, ordered against `stream` with events) carry the copies,
 * `stream` the forwards.  Everything is enqueued after the work already on
 * `stream`, and `stream` completes only after the last copy back, so
 * synchronising `stream` makes o_host and lse_host valid.  Layouts and
 * requirements as for bsa_forward, plus host pointers non-null (page-locked
 * host memory lets the copies overlap; pageable memory works but serialises
 * them) and groups >= 1; these are checked before anything is enqueued.  A
 * CUDA error while enqueueing (not expected) returns BSA_ERR_CUDA with the
 * runs before it already enqueued; synchronise the device before reusing the
 * buffers then.  No device allocation. */
int bsa_forward_host(const void* q_host, const void* k_host, const void* v_host,
                     const bsa_layout* layout, int B, int n, int heads, int kv_heads,
                     int d, float scale, void* q, void* k, void* v, void* o, float* lse,
                     void* o_host, float* lse_host, int groups, void* stream);

/* Forward pass for callers that cannot allocate device memory.  This call has
 * no counterpart on the pages that define the method; it exists for processes
 * whose device memory belongs to someone else (a serving framework that
 * reserved the GPU's memory in its own pool, a host application that lends the
 * library only the buffers it passes in) and for code that must not allocate
 * while running, since cudaMalloc/cudaFree can synchronise the whole device.
 * Same arguments, checks and result as bsa_forward, except that `layout` may
 * be host-only (built with device = -1) and nothing is allocated: on the
 * caller's stream the call copies what the kernel reads of the layout (its
 * work table, four words per query block row, and col_idx) into a block of
 * device memory that the library declares statically (4 MiB of layout words
 * plus a status word; every GPU that loads the library holds it until the
 * process exits), clears the status word and launches the same kernel.  A
 * layout needing more than 1,048,576 32-bit words (4 * rows + nnz) is rejected
 * with BSA_ERR_SHAPE.  The first call on a
 * device looks up that block's device address (cudaGetSymbolAddress) and keeps
 * it for the process, so make the first call on each device before any stream
 * capture, and do not use this entry point on a device after a
 * cudaDeviceReset of it.  The layout arrays are copied from host memory at
 * every call, so a call on a stream that is capturing a CUDA graph is refused
 * with BSA_ERR_UNSUPPORTED and enqueues nothing.  All calls share the block
 * and each overwrites what the last one left: calls that overlap on the GPU
 * race.  A device wait that runs out is recorded in the block's status word,
 * which bsa_get_status reads when given the host-only layout. */
int bsa_forward_noalloc(const void* q, const void* k, const void* v,
                        const bsa_layout* layout, int B, int n, int heads, int kv_heads,
                        int d, float scale, void* o, float* lse, void* stream);

/* Selected-page decode ("BF1: A Causal Dyadic Sparse-Attention Retrofit for
 * Efficient Long-Context Transformers", section 5: one new query token per
 * sequence reads the same block route as prefill, over a cache of keys and
 * values; the route is planned once, in the layout, and reused every step).
 * For sequence b (0 <= b < batch) whose new token is at position
 * t = positions[b] (block i = t / B, B the layout's block size), query row
 * f = b*H + h (H = heads / batch) attends to the cached keys u <= t of the key
 * blocks that block row i of layout head f % layout_heads keeps, reading
 * key/value head h / (H / Hkv) of the sequence (Hkv = kv_heads / batch):
 *   s_u = scale * <q[f], k_u>,  lse[f] = ln sum_u exp(s_u),
 *   o[f] = sum_u exp(s_u - lse[f]) v_u;
 * a row with no allowed key gets o = 0 and lse = -inf.  Layouts (device
 * memory, caller-owned): q, o [heads][d] bf16; k_cache, v_cache
 * [num_pages][Hkv][B][d] bf16, page p holding the B consecutive tokens of one
 * logical block for every key/value head of a sequence (rows past a
 * sequence's end are never read); page_table [batch][max_blocks] int32, the
 * page of logical block j of sequence b; positions [batch] int32; lse [heads]
 * fp32.  The new token's own key and value must already be in the cache.
 * Requirements (checked before launch; errors launch nothing): layout on the
 * current device; B in {64, 128}; d in {64, 128}; batch, heads, kv_heads >= 1;
 * heads and kv_heads multiples of batch; H a multiple of Hkv and of
 * layout_heads; max_blocks >= the layout's blocks; num_pages >= 1; scale
 * finite and > 0; pointers non-null, q, caches and o 16-byte aligned, the rest
 * 4-byte aligned; num_pages must be the number of pages the caches hold.  A
 * position outside [0, n) or a page outside [0, num_pages) read on the device
 * is not dereferenced: the rows it concerns get o = 0, lse = -inf and
 * bsa_get_status then reports BSA_ERR_SHAPE.  Launches one kernel (a
 * thread-block cluster launch: the CTAs of a cluster split a row's kept pages
 * and merge their partial softmax states on chip) and returns after
 * enqueueing it; no allocation, no workspace, no synchronisation. */
int bsa_decode(const void* q, const void* k_cache, const void* v_cache,
               const int32_t* page_table, int max_blocks, int num_pages,
               const int32_t* positions, const bsa_layout* layout, int batch,
               int heads, int kv_heads, int d, float scale, void* o, float* lse,
               void* stream);

/* Gradients of the forward ("BF1: A Causal Dyadic Sparse-Attention Retrofit
 * for Efficient Long-Context Transformers", section 4: the operator is gated
 * on its gradients and adaptation trains through the route).  Given the
 * forward's inputs, its outputs o and lse, and dout = dL/do, for the same
 * allowed pairs (t, u) and P_tu = exp(s_tu - lse_t):
 *   D_t = <dout_t, o_t>,  dS_tu = P_tu (<dout_t, v_u> - D_t),
 *   dq_t = scale sum_u dS_tu k_u,  dk_u = scale sum_t dS_tu q_t,
 *   dv_u = sum_t P_tu dout_t,
 * dk and dv summing over the query heads of the key/value head's group.
 * Layouts: q, o, dout [heads][n][d] bf16; k, v [kv_heads][n][d] bf16; lse
 * [heads][n] fp32 (the forward's, natural log); dq [heads][n][d] fp32; dk,
 * dv [kv_heads][n][d] fp32; workspace [heads][n] fp32 (receives D).  All
 * device memory, caller-owned, not overlapping.  Requirements as for
 * bsa_forward (checked before launch; errors launch nothing), plus dout, dq,
 * dk, dv 16-byte aligned and workspace 4-byte aligned.  Enqueues the clear
 * of dk and dv (two memsets, or a kernel clearing only the rows that several
 * CTAs add into) and three kernels (D, dq, dk/dv) on the stream, and
 * returns.  The dq and dk/dv kernels share one work counter, taken as for
 * bsa_forward (the same rotation, ordering and capture rules), so forwards
 * and backwards on one layout may be in flight at once in any number.  The
 * dk/dv kernel adds its partial sums in fp32, so their
 * summation order (and last bits) may differ from run to run.  A wait that
 * runs out is reported by bsa_get_status as for the forward. */
int bsa_backward(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dout, const bsa_layout* layout,
                 int B, int n, int heads, int kv_heads, int d, float scale,
                 float* dq, float* dk, float* dv, float* workspace, void* stream);

/* Bytes of device workspace bsa_bsbr_retrieval needs: the chunk states
 * (kv_heads x chunks x d x d fp32) and meta keys (kv_heads x chunks x d fp32),
 * chunks = ceil(n / B).  0 for sizes < 1. */
size_t bsa_bsbr_workspace_bytes(int n, int B, int kv_heads, int d);

/* BSBR's between-chunk retrieval term ("bsbr", jvboid.dev/projects/bsbr,
 * section "Solution"), added to o in place.  Chunks are the layout's blocks of
 * B tokens.  With R_c, H_c the means of q[f] and k[g] over chunk c (g = f /
 * (heads / kv_heads)) and F_c = sum over the chunk's tokens of k_u^T v_u:
 *   A_cc' = softmax over c' < c of scale <R_c, H_c'>,   S_c = sum_{c' < c} A_cc' F_c',
 *   o[f][t] += q[f][t] S_c   for every token t of chunk c >= 1
 * (chunk 0 retrieves nothing).  Called after bsa_forward with a
 * block-diagonal layout (BAND_GLOBAL, window 0, no global block), o becomes
 * the whole BSBR attention output; lse stays the within-chunk term's.
 * Layouts: q, o [heads][n][d] bf16; k, v [kv_heads][n][d] bf16; workspace
 * device memory of at least bsa_bsbr_workspace_bytes.  The layout supplies
 * the device, B, n and the status word (its kept blocks are not read).
 * Requirements (checked before launch): layout on the current device and
 * built for this n and B; B in {64, 128}; d in {64, 128}; heads a multiple of
 * kv_heads; scale finite and > 0; q, k, v, o, workspace 16-byte aligned and
 * workspace_bytes large enough.  Enqueues two kernels (none for a single
 * chunk) and returns; no allocation.  The retrieval costs O(chunks^2 d^2)
 * per head (each chunk sums the states of all earlier chunks). */
int bsa_bsbr_retrieval(const void* q, const void* k, const void* v,
                       const bsa_layout* layout, int B, int n, int heads,
                       int kv_heads, int d, float scale, void* o,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Read-only host view of the key/value-gradient work list: for layout head
 * h, segments seg_ptr[h] .. seg_ptr[h+1] - 1, segment s being the triple
 * segs[3s .. 3s+2] = (key block j, first index into the transposed layout's
 * row_idx, entry count <= 16), longest first.  Every column of the
 * transposed layout is cut into runs of at most 16 query blocks. */
int bsa_layout_segments(const bsa_layout* layout, const int32_t** seg_ptr,
                        const int32_t** segs, int* layout_heads, int* count);

/* Release a layout and its device arrays (NULL is a no-op).  The caller must
 * make sure no forward that uses it is still running. */
void bsa_free(bsa_layout* layout);

/* Message describing the last error returned on the calling thread. */
const char* bsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
