/*
 * gad_attn.h - C ABI of the paged FP8 gated attention decode library
 * (libgad_attn.so, hand-written CUDA for sm_100a).
 *
 * One call runs one decode step (q_len 1) or one causal verify block
 * (q_len <= 8) of gated grouped-query attention over a paged FP8 E4M3 KV
 * cache, as defined on the task page "Gated attention decode
 * (muse_attention_decode)", section "What to compute":
 *
 *   q, k, v, gate = split(qkv[t])
 *   q = rmsnorm(q) * 5.473 ; k = rmsnorm(k)           per 64-wide head
 *   q, k = rope(q, p), rope(k, p)                      when use_rope != 0
 *   cache[cache_loc[t]] = fp8(k), fp8(v)               E4M3, scaled
 *   a = softmax(q . K^T / 8) . V                       keys up to p (window or all)
 *   out = rmsnorm(a) * sigmoid(gate)                   bf16
 *
 * Model shape (section "Shapes"): 16 query heads, 2 KV heads, head dim 64;
 * query head h reads KV head h / 8.  The page's tests also run "heads dp",
 * read here as every head of the layer on one GPU (128 query, 16 KV heads);
 * gad_attn_decode_heads takes such head counts.  Readings of points the page leaves open:
 * rmsnorm eps 1e-6 with unit weights; RoPE is the NeoX half-split rotation of
 * dims (i, i+32) by p * 10000^(-2i/64); a sliding window W attends keys i with
 * p - W < i <= p; stored code = E4M3(x / scale) with round-to-nearest-even and
 * saturation to +-448, dequantised value = code * scale.
 *
 * All pointers are DEVICE pointers unless stated.  All buffers belong to the
 * caller; the library keeps no state between calls except per-device launch
 * settings and the scratch pointer registered for the descriptor form
 * (gad_attn_set_workspace).  Calls are asynchronous on `stream`, never
 * synchronise the host, never read device values on the host and never
 * allocate, so they can be captured in a CUDA graph.
 */
#ifndef GAD_ATTN_H
#define GAD_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The page's per-GPU shape ("heads tp8"); gad_attn_decode_heads takes
 * multiples of it. */
#define GAD_HQ 16          /* query heads per GPU            */
#define GAD_HKV 2          /* key/value heads per GPU        */
#define GAD_HEAD_DIM 64
#define GAD_QKV_COLS 2304  /* q 16x64 | k 2x64 | v 2x64 | gate 16x64 */
#define GAD_OUT_COLS 1024  /* 16 heads x 64                  */
#define GAD_ROW_BYTES 128  /* one cache row: 2 KV heads x 64 E4M3 codes */
#define GAD_MAX_L 8        /* longest verify block           */
#define GAD_MAX_B 4096     /* most requests in one call; also the most
                              work items (request, token chunk, heads)    */
#define GAD_MAX_PREFILL_L 65536 /* longest block of gad_attn_prefill */
#define GAD_HIDDEN 8192    /* decoder hidden size: rows of the o-projection weight */
#define GAD_MAX_OPROJ_T 262144 /* most tokens in one projection call */
#define GAD_NOALLOC_SCRATCH_BYTES (16u << 20) /* built-in scratch of gad_attn_decode_noalloc */

/* Return codes (0 = success). */
typedef enum {
    GAD_OK = 0,
    GAD_ERR_NULL = -1,        /* a required pointer is NULL                     */
    GAD_ERR_SHAPE = -2,       /* B, L, max_pages or num_rows out of range       */
    GAD_ERR_ALIGN = -3,       /* a pointer is not aligned as documented         */
    GAD_ERR_UNSUPPORTED = -4, /* page_size not 1 or 64, window < 0, or head
                                 counts other than hq = 8 hkv, hkv = 2, 4, 6 .. */
    GAD_ERR_WORKSPACE = -5,   /* workspace NULL or smaller than required        */
    GAD_ERR_CUDA = -6,        /* a CUDA call or kernel launch failed            */
    GAD_ERR_DEVICE = -7,      /* current device is not compute capability 10.x  */
    GAD_ERR_DTYPE = -8,       /* a tensor descriptor has the wrong element type */
    GAD_ERR_STRIDE = -9       /* a tensor descriptor is not densely packed,
                                 row-major                                      */
} gad_status;

/* Bits of a step's status word (gad_attn_step_status, gad_oproj_status).
 * Every wait inside the kernels is bounded: a kernel whose pipeline stalls
 * (a wait that does not end within 2 s) gives up, lets the work it has in
 * flight finish, frees its tensor memory and sets its bit, instead of hanging
 * the GPU.  The step's outputs are then not valid. */
#define GAD_STATUS_ATTN_WAIT 1   /* an attention kernel gave up a wait */
#define GAD_STATUS_OPROJ_WAIT 2  /* the output projection gave up a wait */

/*
 * Bytes of device workspace that gad_attn_decode needs for B requests of L
 * tokens on the CURRENT device (it depends on the device's SM count).
 * Returns 0 and sets gad_last_error() when B or L is out of range or no CUDA
 * device is present.  Host-only; launches nothing.
 */
size_t gad_attn_workspace_bytes(int B, int L);

/*
 * Workspace bytes of gad_attn_decode_heads for B requests of L tokens with
 * hq query and hkv KV heads, on the CURRENT device.  Returns 0 and sets
 * gad_last_error() on the same conditions as gad_attn_workspace_bytes and on
 * unsupported head counts.  gad_attn_workspace_bytes(B, L) equals
 * gad_attn_workspace_bytes_heads(B, L, 16, 2).  Host-only.
 */
size_t gad_attn_workspace_bytes_heads(int B, int L, int hq, int hkv);

/*
 * One step.  T = B * L tokens; token t = b * L + j is token j of request b.
 *
 *   qkv         bf16 [T, 2304], row-major, 16-byte aligned.  Columns:
 *               q heads [0,1024), k heads [1024,1152), v heads [1152,1280),
 *               gate [1280,2304); each head 64 contiguous values.
 *   positions   int64 [T]: position p of each token, 0 <= p < 2^31.  Token t
 *               attends the cache keys i with lo <= i <= p, lo = 0 (window == 0)
 *               or max(0, p - window + 1).  Contract: p = seq_lens[b] + j.
 *   seq_lens    int32 [B]: keys cached before this step (the serving stack's
 *               lengths).  Accepted for interface compatibility; the ranges
 *               come from `positions`.  May be NULL.
 *   page_table  int32 [B, max_pages], row-major: cache row of key i of request
 *               b is page_table[b][i / page_size] * page_size + i % page_size.
 *   cache_loc   int64 [T]: the cache row receiving token t's k and v.
 *               Contract: cache_loc[t] is the row of key positions[t], and no
 *               request reads a row that another token of this step writes
 *               (except its own block's new keys).
 *   k_cache,    uint8 [num_rows, 2, 64] E4M3 codes, 16-byte aligned, with
 *   v_cache     num_rows = num_pages * page_size < 2^31.  Rows cache_loc[t] are
 *               overwritten; no other byte is written.
 *   k_scale,    float32 [1] each (device): the caches' dequantisation scales.
 *   v_scale
 *   page_size   1 or 64.
 *   window      > 0: sliding window of that many keys; 0: full attention.
 *   use_rope    nonzero: rotate q and k by their position.
 *   out         bf16 [T, 1024], row-major, 16-byte aligned.
 *   workspace   device scratch of at least gad_attn_workspace_bytes(B, L)
 *               bytes, 256-byte aligned, owned by the caller; its contents on
 *               entry do not matter.  Calls that overlap on the GPU must use
 *               different workspaces.
 *   stream      a cudaStream_t (NULL = legacy default stream).
 *
 * Errors: argument checks run on the host before any launch; on failure the
 * call launches nothing and returns a negative gad_status.  Device VALUES
 * (positions, page_table, cache_loc) are not checked against the contract:
 * keys whose page index falls outside the page-table row, and rows outside
 * [0, num_rows), are read as zeros and never written, so a contract
 * violation gives wrong numbers but no out-of-bounds access.
 */
int gad_attn_decode(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                    const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                    uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                    int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                    void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gad_attn_decode for other head counts: hq query heads over hkv KV heads,
 * with hkv a positive multiple of 2 and hq = 8 hkv (query head h reads KV
 * head h / 8), e.g. hq = 128, hkv = 16 for the page's "heads dp" tests
 * (section "Shapes" and its list of tests).  gad_attn_decode is this call
 * with hq = 16, hkv = 2.  The layouts widen with the head counts:
 *
 *   qkv         bf16 [T, 64 (2 hq + 2 hkv)]: q heads [0, 64 hq), k heads
 *               [64 hq, 64 (hq + hkv)), v heads [.., 64 (hq + 2 hkv)), gate
 *               [.., 64 (2 hq + 2 hkv)); each head 64 contiguous values.
 *   k_cache,    uint8 [num_rows, hkv, 64] E4M3 codes (64 hkv bytes per row).
 *   v_cache
 *   out         bf16 [T, 64 hq].
 *   workspace   at least gad_attn_workspace_bytes_heads(B, L, hq, hkv) bytes.
 *
 * B * hkv / 2 may not exceed GAD_MAX_B (GAD_ERR_SHAPE).  Other head counts
 * return GAD_ERR_UNSUPPORTED.  Every other argument, the error behaviour and
 * the contract are those of gad_attn_decode.
 */
int gad_attn_decode_heads(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                          int L, int hq, int hkv, int max_pages, int64_t num_rows, int page_size,
                          int window, int use_rope, void* out, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * Profiling variant of gad_attn_decode: same arguments and semantics, plus
 * `events`, an array of four cudaEvent_t created by the caller.  It records
 * events[0] before the prep kernel, events[1] between prep and decode,
 * events[2] between decode and combine and events[3] after combine, all on
 * `stream`, so cudaEventElapsedTime gives each kernel's device time.  Because
 * an event sits between the kernels, they run strictly one after another
 * (no programmatic dependent launch overlap); use gad_attn_decode in
 * production.  Returns GAD_ERR_NULL if events or any of its entries is NULL.
 */
int gad_attn_decode_timed(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                          int L, int max_pages, int64_t num_rows, int page_size, int window,
                          int use_rope, void* out, void* workspace, size_t workspace_bytes,
                          void* stream, void* const* events);

/*
 * Profiling variant of gad_attn_decode_heads: its arguments plus the four
 * events of gad_attn_decode_timed, recorded the same way.
 */
int gad_attn_decode_heads_timed(const void* qkv, const int64_t* positions,
                                const int32_t* seq_lens, const int32_t* page_table,
                                const int64_t* cache_loc, uint8_t* k_cache, uint8_t* v_cache,
                                const float* k_scale, const float* v_scale, int B, int L, int hq,
                                int hkv, int max_pages, int64_t num_rows, int page_size,
                                int window, int use_rope, void* out, void* workspace,
                                size_t workspace_bytes, void* stream, void* const* events);

/*
 * Prefill: the same step for a block of L new tokens per request, causal
 * within the block, 1 <= L <= GAD_MAX_PREFILL_L.  The page "Prefill layer
 * (muse_prefill_layer)" runs this attention (its "What to compute": QK-norm,
 * RoPE, write fp8(k), fp8(v), rmsnorm(attention(q)) * sigmoid(g)) at q_len
 * 753 on an 80,000-token context and at q_len 16,384.  Arguments, layouts
 * and error behaviour are those of gad_attn_decode with L tokens per request
 * (token t = b * L + j at position positions[t], contract positions[t] =
 * seq_lens[b] + j); the workspace comes from gad_attn_prefill_workspace_bytes.
 * For L > GAD_MAX_L each request's tokens are split into chunks of 32, one
 * work item per (chunk, KV head), and 2 B ceil(L / 32) may not exceed
 * GAD_MAX_B (GAD_ERR_SHAPE), e.g. L = 16,384 admits B <= 4; L <= GAD_MAX_L
 * runs as gad_attn_decode.
 */
int gad_attn_prefill(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                     const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                     uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                     int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                     void* out, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of gad_attn_prefill on the CURRENT device (0 on bad
 * arguments, with gad_last_error() set).  Host-only. */
size_t gad_attn_prefill_workspace_bytes(int B, int L);

/* Profiling variant of gad_attn_prefill, with the four events of
 * gad_attn_decode_timed. */
int gad_attn_prefill_timed(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                           const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                           uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                           int L, int max_pages, int64_t num_rows, int page_size, int window,
                           int use_rope, void* out, void* workspace, size_t workspace_bytes,
                           void* stream, void* const* events);

/*
 * Output projection that follows the attention in the decoder layer (the
 * pages "Decode layer (muse_decode_layer)" and "Prefill layer
 * (muse_prefill_layer)", section "What to compute":
 * a = (rmsnorm(attention(q)) * sigmoid(g)) @ o.T, its all-reduce being the
 * identity on one GPU):
 *
 *   a[t][n] = sum_k out[t][k] * o_weight[n][k]     fp32 accumulation, bf16 a
 *
 *   out       bf16 [T, K] row-major (the attention step's output: K = 1024)
 *   o_weight  bf16 [N, K] row-major (N = GAD_HIDDEN for the decoder layer)
 *   a         bf16 [T, N] row-major, written
 *   K a positive multiple of 64, N a positive multiple of 128, 1 <= T <=
 *   GAD_MAX_OPROJ_T; all three pointers 16-byte aligned (GAD_ERR_SHAPE,
 *   GAD_ERR_ALIGN, GAD_ERR_NULL otherwise, checked before any launch).
 * One hand-written tcgen05 kernel (TMA-staged operands, accumulator in tensor
 * memory); asynchronous on `stream`, allocates nothing, graph-capturable.
 */
int gad_oproj(const void* out, const void* o_weight, void* a, int T, int K, int N, void* stream);

/*
 * The attention step followed by its output projection in one call:
 * gad_attn_decode's step (or gad_attn_prefill's for L > GAD_MAX_L; any
 * 1 <= L <= GAD_MAX_PREFILL_L), writing `out` as they do, then
 * a = out @ o_weight^T as in gad_oproj with K = 1024 and N = hidden.  The
 * projection kernel is chained to the step's last kernel by programmatic
 * dependent launch: its first weight tiles load while the step finishes.
 * workspace: gad_attn_prefill_workspace_bytes(B, L) bytes (which equals
 * gad_attn_workspace_bytes(B, L) for L <= GAD_MAX_L).  Arguments and errors
 * as gad_attn_decode and gad_oproj.
 */
int gad_attn_decode_oproj(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                          int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                          void* out, void* workspace, size_t workspace_bytes, const void* o_weight,
                          int hidden, void* a, void* stream);

/*
 * Allocation-free variant of gad_attn_decode.  The page has no counterpart:
 * this is a library convenience for callers that cannot provide device
 * scratch memory, e.g. code inside a framework whose memory pool owns every
 * device allocation, plugins that must not call cudaMalloc (it can
 * synchronise the device and is refused while a graph capture is running),
 * or plain C hosts with no device allocator.
 *
 * Same arguments and results as gad_attn_decode, minus the workspace: the
 * step's scratch is a fixed device array of GAD_NOALLOC_SCRATCH_BYTES
 * (16 MiB) inside the library, which every GPU that loads the library holds
 * until the process exits.  The caller still passes all inputs and outputs.
 *   - Sizes whose scratch (gad_attn_workspace_bytes(B, L)) exceeds 16 MiB are
 *     rejected with GAD_ERR_WORKSPACE before anything is launched; on a
 *     148-SM B200 that admits L = 1 steps up to B = 621 and L = 8 steps up to
 *     B = 135 (use gad_attn_decode beyond that).
 *   - It never allocates (no cudaMalloc, cudaFree or allocating library
 *     call).  The first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and caches it;
 *     make that first call before any stream capture on that device.
 *   - Every call on a device shares the one array.  Nothing in it needs to
 *     start at zero (each call writes every scratch byte it later reads), but
 *     calls that overlap on the GPU (different streams, or graphs replayed
 *     concurrently) race on it and give wrong results: serialise them.
 */
int gad_attn_decode_noalloc(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                            const int32_t* page_table, const int64_t* cache_loc,
                            uint8_t* k_cache, uint8_t* v_cache, const float* k_scale,
                            const float* v_scale, int B, int L, int max_pages, int64_t num_rows,
                            int page_size, int window, int use_rope, void* out, void* stream);

/*
 * Status of the last step that ran with `workspace` (a step of gad_attn_decode,
 * gad_attn_decode_heads, gad_attn_prefill, gad_attn_decode_oproj or
 * gad_attn_decode_t): a cudaMemcpyAsync on `stream` of the step's status word
 * (GAD_STATUS_* bits, 0 when every wait ended in time) into the HOST int
 * *status.  Read *status only after `stream` has synchronised.  The word sits at
 * offset 0 of the workspace; each step's first kernel clears it, so it reports
 * the latest step only.  workspace == NULL reads the word of the built-in
 * scratch of gad_attn_decode_noalloc on the current device.  Returns GAD_OK,
 * GAD_ERR_NULL (status NULL), GAD_ERR_ALIGN or GAD_ERR_CUDA.
 */
int gad_attn_step_status(const void* workspace, int* status, void* stream);

/*
 * Status of the standalone projection (gad_oproj): a cudaMemcpyAsync on
 * `stream` of its device status word into the HOST int *status, then a clear of
 * the word, both ordered on `stream`.  The word is one per device, shared by
 * every gad_oproj call on it, and keeps its bits until this call reads them.
 * Projections chained to a step (gad_attn_decode_oproj) report into the
 * step's word instead.  Returns GAD_OK, GAD_ERR_NULL or GAD_ERR_CUDA.
 */
int gad_oproj_status(int* status, void* stream);

/* ------------------------------------------------------------------------- */
/* Tensor-descriptor form                                                     */
/* ------------------------------------------------------------------------- */

/* Element types of gad_tensor. */
typedef enum {
    GAD_DTYPE_BF16 = 1,
    GAD_DTYPE_E4M3 = 2,  /* FP8 E4M3 codes, one byte each */
    GAD_DTYPE_U8 = 3,    /* bytes; accepted for the caches as E4M3 codes */
    GAD_DTYPE_I32 = 4,
    GAD_DTYPE_I64 = 5,
    GAD_DTYPE_F32 = 6
} gad_dtype;

/* A device tensor: data pointer, element type (gad_dtype), rank 1..4, extents
 * and strides in elements.  The descriptor is read during the call only; the
 * memory stays the caller's. */
typedef struct {
    void* data;
    int32_t dtype;
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
} gad_tensor;

/*
 * Registers caller-owned device scratch for gad_attn_decode_t on the CURRENT
 * device (256-byte aligned; NULL unregisters).  The library keeps the pointer
 * and size, never the memory.  Register it before the steps that use it and
 * outside any stream capture; steps on one device that overlap on the GPU
 * share this scratch and race, so run them on one stream (or use
 * gad_attn_decode with a workspace per stream).  Returns GAD_OK,
 * GAD_ERR_ALIGN, GAD_ERR_CUDA or GAD_ERR_DEVICE.  Host-only.
 */
int gad_attn_set_workspace(void* workspace, size_t bytes);

/*
 * Bytes of scratch gad_attn_decode_t needs for B requests of L tokens with
 * `max_pages` page-table entries per request, page size `page_size` and
 * sliding window `window` (0: full), on the CURRENT device; 0 with
 * gad_last_error() set on bad arguments.  (On this design the size depends on
 * B, L and the device's SM count only; the other arguments are checked.)
 */
size_t gad_attn_workspace_bytes_t(int B, int L, int max_pages, int page_size, int window);

/*
 * The step with every array passed as a tensor descriptor: exactly the
 * arguments of the page's attention call ("What to compute" and the inputs
 * listed in "Shapes"), with the sizes read from the descriptors and
 * cross-checked:
 *
 *   out         bf16 [B, L, 64 hq]      gives B, L (1..GAD_MAX_PREFILL_L) and hq
 *   qkv         bf16 [B L, 64 (2 hq + 2 hkv)]   gives hkv
 *   positions   i64 [B L]
 *   seq_lens    i32 [B], or NULL (checked, not read: ranges come from positions)
 *   page_table  i32 [B, max_pages]
 *   cache_loc   i64 [B L]
 *   k_cache,    e4m3 (or u8) [num_pages, page_size, hkv, 64]
 *   v_cache
 *   k_scale,    f32 [1]
 *   v_scale
 *
 * Every descriptor must be densely packed and row-major.  A wrong element type
 * returns GAD_ERR_DTYPE, a wrong rank or extent GAD_ERR_SHAPE, a wrong stride
 * GAD_ERR_STRIDE, a NULL descriptor or data pointer GAD_ERR_NULL, and no
 * registered scratch GAD_ERR_WORKSPACE, all before any launch; then the call
 * runs gad_attn_decode_heads (or gad_attn_prefill for L > GAD_MAX_L) on the
 * registered scratch, with their checks, semantics and errors.
 */
int gad_attn_decode_t(const gad_tensor* qkv, const gad_tensor* positions, const gad_tensor* seq_lens,
                      const gad_tensor* page_table, const gad_tensor* cache_loc,
                      const gad_tensor* k_cache, const gad_tensor* v_cache,
                      const gad_tensor* k_scale, const gad_tensor* v_scale, int page_size,
                      int window, int use_rope, const gad_tensor* out, void* stream);

/* Message for the last nonzero status returned on this host thread. */
const char* gad_last_error(void);

/* Static name of a gad_status value. */
const char* gad_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GAD_ATTN_H */
