/*
 * b200attn — causal scaled-dot-product attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libb200attn.so.  Plain pointers and sizes only.
 *
 * The operation (both entry points):
 *   O = softmax(Q K^T * scale + mask) V, per batch b and query head h, where
 *   query head h reads key/value head h / (H / Hkv) — multi-head (Hkv = H),
 *   grouped-query (H / Hkv > 1) and multi-query (Hkv = 1) layouts.
 *   Sources: "Hesper.Layers.Attention" (Mathematical Definition, Multi-Head
 *   Attention, Causal Masking); "Grouped-Query Attention" §5.1 (one K/V head
 *   serves group_size query heads, repeat_interleave order) and §5.2 (scores,
 *   causal bias, softmax, weighted sum); "Causal Multi-Head Self-Attention",
 *   The causal mask (masked positions get probability exactly zero; every row
 *   sums to one); "Multi-query attention, annotated" §2.4 and §3 (incremental
 *   attention against a cache; one shared K/V head).
 *
 * Mask: query row i sits at absolute position p_i = start_pos + i (start_pos
 * = 0 for prefill) and, when causal, sees key j iff j <= p_i; masked keys get
 * weight exactly 0.  This is the convention of the makarna cached-attention
 * loop ("attention_cached.go", CausalAttentionCached: new tokens start at
 * startPos and see every key up to their own position).
 *
 * Layouts (all row-major, contiguous, device memory unless stated):
 *   Q, O : [B, H, Tq, d]
 *   K, V : [B, Hkv, S_cap, d]   (prefill: S_cap = S = T)
 *   lse  : [B, H, Tq] float32, optional; lse = max_j s_j + ln sum_j e^{s_j - max}
 *          over the visible scaled scores s_j (natural log).
 * Element type: ATTN_F32 (float), ATTN_BF16, ATTN_F16 for Q, K, V and O alike;
 * accumulation is always float32.  Output is rounded to nearest-even.
 *
 * Ownership: the caller owns every buffer it passes.  No call allocates or
 * frees device memory or synchronises (attn_device_status excepted); kernels
 * are enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 * Two pieces of device state persist between calls, both in the library's
 * own statically sized module memory on every device that loads it: the
 * device status word that bounded waits and page-table checks write (read and
 * cleared by attn_device_status), and the fixed scratch array of
 * attn_cached_noalloc, which keeps the last such call's split partials.  The
 * host keeps per-device kernel attributes and the scratch array's address.
 *
 * Errors: every argument is checked before anything is enqueued; on any error
 * nothing is launched and O is left untouched.  Nothing aborts the process.
 *   ATTN_ERR_INVALID_ARG  null pointer with a non-empty problem, negative size,
 *                         Hkv = 0, H % Hkv != 0, S > S_cap, start_pos < 0,
 *                         start_pos + Tnew > S, non-finite scale, a pointer not
 *                         aligned to 16 bytes, or d <= 0;
 *   ATTN_ERR_UNSUPPORTED  d > 256;
 *   ATTN_ERR_WORKSPACE    workspace smaller than attn_cached_workspace_size();
 *   ATTN_ERR_CUDA         a CUDA runtime error while encoding or launching;
 *   ATTN_ERR_DEVICE_TIMEOUT reported by attn_device_status() when a kernel gave
 *                         up a bounded wait (it then exits cleanly);
 *   ATTN_ERR_DEVICE_INDEX reported by attn_device_status() when a paged call met
 *                         a page table or length entry out of range (it clamps
 *                         it and never reads outside the pools; that output is
 *                         then meaningless).
 * A problem with B * H * Tq = 0 returns ATTN_OK and launches nothing.
 */
#ifndef B200ATTN_H
#define B200ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,
    ATTN_ERR_UNSUPPORTED = 2,
    ATTN_ERR_WORKSPACE = 3,
    ATTN_ERR_CUDA = 4,
    ATTN_ERR_DEVICE_TIMEOUT = 5,
    ATTN_ERR_DEVICE_INDEX = 6
} attn_status_t;

typedef enum { ATTN_F32 = 0, ATTN_BF16 = 1, ATTN_F16 = 2 } attn_dtype_t;

/* Which kernel family a call uses (see attn_prefill_plan / attn_cached_plan). */
typedef enum {
    ATTN_KERNEL_NONE = 0,        /* empty problem: nothing launched            */
    ATTN_KERNEL_SIMT = 1,        /* float32 CUDA-core kernel (any d <= 256)    */
    ATTN_KERNEL_TCGEN05 = 2,     /* TMA + tcgen05/TMEM fused prefill kernel    *
                                  * (+ the merge of a cached call's key-range  *
                                  * pieces, when its last pass is cut)         */
    ATTN_KERNEL_SPLITKV = 3      /* split-KV decode kernel + LSE combine       */
} attn_kernel_t;

/*
 * Full-sequence attention ("Hesper.Layers.Attention", forward, steps 4-6;
 * "Causal Multi-Head Self-Attention", Dataflow and shapes).
 *   q [B,H,T,d], k/v [B,Hkv,T,d], o [B,H,T,d]; lse nullable [B,H,T].
 *   causal != 0: row i sees keys 0..i; causal = 0: every key.
 * Equivalent to attn_cached with Tnew = S = S_cap = T and start_pos = 0.
 */
ATTN_API attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                           attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                           int64_t d, float scale, int causal, void* stream);

/*
 * KV-cached attention ("Multi-query attention, annotated" §2.4: new queries
 * against the cached keys and values; "attention_cached.go",
 * CausalAttentionCached).  The history already holds the new tokens' keys and
 * values at positions start_pos .. start_pos + Tnew - 1.
 *   q [B,H,Tnew,d]; k_hist/v_hist [B,Hkv,S_cap,d], first S rows valid;
 *   o [B,H,Tnew,d]; lse nullable [B,H,Tnew].  Always causal.
 *   workspace: device buffer of at least attn_cached_workspace_size() bytes,
 *   16-byte aligned (may be NULL when that size is 0); its contents on entry
 *   do not matter and are clobbered.  It holds fp32 partial results: the
 *   split-KV decode's per-split rows, or, for a chunked prefill on the
 *   tensor-core kernel whose last pass of work units would leave most SMs
 *   idle, those units' rows computed in 2-4 pieces of the key range (merged
 *   by a second kernel on the same stream).
 */
ATTN_API attn_status_t attn_cached(const void* q, const void* k_hist, const void* v_hist, void* o,
                          float* lse, attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                          int64_t Tnew, int64_t S, int64_t S_cap, int64_t d, int64_t start_pos,
                          float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_cached without a workspace argument, for callers that may not allocate
 * device memory themselves: plugins that receive only their input and output
 * buffers from a host framework owning the allocator, and serving loops that
 * forbid allocation (and the synchronisation it can bring) once warm.  The
 * pages have no counterpart to this call; it exists for such callers only.
 *
 * Same operation, arguments, layouts and errors as attn_cached minus
 * `workspace` / `workspace_bytes`.  The partials go to one library-owned
 * device array of ATTN_NOALLOC_SCRATCH_BYTES (16 MiB), present on every GPU
 * that loads the library until the process exits.  A chunked prefill cuts
 * fewer pieces (or none) rather than need more than the array; a split-KV
 * decode whose attn_cached_workspace_size() exceeds it returns
 * ATTN_ERR_WORKSPACE and launches nothing.  The call allocates nothing: the
 * first call on each device looks up the array's device address (with that
 * device current), so make that first call before any stream capture; the
 * lookup is keyed on the device's context, so after a device reset the next
 * call (again outside any capture) looks the new address up.  All
 * calls on a device share the one array and it keeps the last call's data;
 * calls that can overlap on the GPU (different streams, no ordering between
 * them) race on it and must be serialised by the caller.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
ATTN_API attn_status_t attn_cached_noalloc(const void* q, const void* k_hist, const void* v_hist,
                                           void* o, float* lse, attn_dtype_t dtype, int64_t B,
                                           int64_t H, int64_t Hkv, int64_t Tnew, int64_t S,
                                           int64_t S_cap, int64_t d, int64_t start_pos,
                                           float scale, void* stream);

/*
 * Append new tokens' keys and values to a KV cache, rotating the keys with
 * rotary position embedding on the way ("Hesper.Layers.Attention", the fused
 * RoPE-K and cache-write kernels and the no-RoPE batched write;
 * "Grouped-Query Attention" §5.1, apply_rope at offset start_pos before the
 * cache append).  For new token t at position p = start_pos + t and
 * i < d/2, with angle a = p * rope_base^(-2i/d) (NeoX pairing: dimension i
 * turns together with i + d/2):
 *   K_cache[p][i]       = K[t][i] cos a - K[t][i + d/2] sin a
 *   K_cache[p][i + d/2] = K[t][i + d/2] cos a + K[t][i] sin a
 *   V_cache[p]          = V[t]
 * rope_base <= 0 writes K unrotated.  The angle is reduced in double
 * precision, then rotated in fp32; results are rounded to nearest-even.
 *   k_new, v_new: [B, Hkv, Tnew, d]; k_cache, v_cache: [B, Hkv, S_cap, d];
 *   rows start_pos .. start_pos + Tnew - 1 of every (b, kv head) are written,
 *   nothing else is touched.
 * Errors (nothing launched): ATTN_ERR_INVALID_ARG for a null or unaligned
 * (16-byte) pointer, negative size, start_pos + Tnew > S_cap, non-finite
 * rope_base, or d not a multiple of 8 (4 for ATTN_F32); ATTN_ERR_UNSUPPORTED
 * for d > 256, Hkv > 65536 or B * Tnew > 2^31.  An empty append (B, Hkv or Tnew = 0) returns ATTN_OK.
 */
ATTN_API attn_status_t attn_kv_append_rope(const void* k_new, const void* v_new, void* k_cache,
                                           void* v_cache, attn_dtype_t dtype, int64_t B,
                                           int64_t Hkv, int64_t Tnew, int64_t S_cap, int64_t d,
                                           int64_t start_pos, float rope_base, void* stream);

/*
 * Local (sliding-window) attention: the query at absolute position p sees
 * only keys p - window < j <= p, the current position and the previous
 * window - 1 ("Multi-query attention, annotated" §4.1: local decoder
 * self-attention over the current position and the previous 31).  Otherwise
 * identical to attn_prefill (causal) and attn_cached; window = 0 is plain
 * causal attention.  Key tiles wholly outside every row's window are never
 * loaded.  Errors as for those calls, plus ATTN_ERR_INVALID_ARG for window < 0.
 * attn_cached_local needs attn_cached_local_workspace_size() bytes of
 * workspace (the split plan covers only the keys inside the window).
 */
ATTN_API attn_status_t attn_prefill_local(const void* q, const void* k, const void* v, void* o,
                                          float* lse, attn_dtype_t dtype, int64_t B, int64_t H,
                                          int64_t Hkv, int64_t T, int64_t d, float scale,
                                          int64_t window, void* stream);
ATTN_API attn_status_t attn_cached_local(const void* q, const void* k_hist, const void* v_hist,
                                         void* o, float* lse, attn_dtype_t dtype, int64_t B,
                                         int64_t H, int64_t Hkv, int64_t Tnew, int64_t S,
                                         int64_t S_cap, int64_t d, int64_t start_pos, float scale,
                                         int64_t window, void* workspace, size_t workspace_bytes,
                                         void* stream);
ATTN_API size_t attn_cached_local_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H,
                                                 int64_t Hkv, int64_t Tnew, int64_t S, int64_t d,
                                                 int64_t start_pos, int64_t window);

/*
 * KV-cached attention over a paged cache: a logical-to-physical page table
 * ("Causal Multi-Head Self-Attention", Algorithm and cache boundaries: paged
 * decode reads a K/V page table; attention_cached.go, CausalAttentionPackedBlocks:
 * head-major blocks [kv head][token within block][d]).  Same result as
 * attn_cached on the gathered history, each sequence with its own length.
 *   q [B,H,Tnew,d]; o [B,H,Tnew,d]; lse nullable [B,H,Tnew].  Always causal.
 *   k_pages, v_pages [num_pages, Hkv, page_size, d]: page p holds, for every
 *     K/V head, page_size consecutive tokens.
 *   page_table (device, int32) [B, max_pages]: token j of sequence b lives in
 *     physical page page_table[b][j / page_size], row j % page_size.
 *   kv_lens (device, int32) [B]: L_b, the tokens of sequence b in the cache,
 *     new ones included; its Tnew new tokens sit at positions L_b - Tnew ..
 *     L_b - 1 and see keys 0 .. their own position.
 *   max_kv_len (host): a bound on every L_b, used to plan the split; at most
 *     max_pages * page_size.
 *   page_size: a power of two, 8 .. 2^20.
 *   workspace: at least attn_cached_paged_workspace_size() bytes, 16-byte
 *     aligned; may be NULL when that size is 0 (partials as for attn_cached).
 * The device arrays are read, never written; entries out of range are
 * reported through attn_device_status() as ATTN_ERR_DEVICE_INDEX.
 * Kernels: bf16 / fp16 with d a multiple of 16 in [64, 128] and
 * H / Hkv * Tnew <= 16, or d = 256 and H / Hkv * Tnew <= 8, run the split-KV
 * decode kernels; other
 * bf16 / fp16 shapes with d a multiple of 16 in [64, 128] (chunked prefill)
 * run the tensor-core prefill kernel, which copies whole pages and zeroes the
 * rows past L_b in shared memory.  Rows of a page past L_b may hold anything
 * (NaN and inf included): no result depends on them.  Everything
 * else returns ATTN_ERR_UNSUPPORTED (float32 included).  ATTN_ERR_INVALID_ARG as for
 * attn_cached, plus: page_size not a power of two in range, max_kv_len < Tnew
 * or > max_pages * page_size, num_pages = 0, null or unaligned (4-byte) table
 * or lengths.
 */
ATTN_API attn_status_t attn_cached_paged(const void* q, const void* k_pages, const void* v_pages,
                                         void* o, float* lse, attn_dtype_t dtype, int64_t B,
                                         int64_t H, int64_t Hkv, int64_t Tnew, int64_t d,
                                         const int32_t* page_table, int64_t max_pages,
                                         int64_t num_pages, int64_t page_size,
                                         const int32_t* kv_lens, int64_t max_kv_len, float scale,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_cached_paged needs (0 if none or unsupported). */
ATTN_API size_t attn_cached_paged_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H,
                                                 int64_t Hkv, int64_t Tnew, int64_t d,
                                                 int64_t max_kv_len);

/*
 * Backward pass of full-sequence attention ("Causal Multi-Head Self-Attention",
 * Two exact full-sequence algorithms: the memory-linear path keeps only each
 * row's statistics from the forward and rebuilds every probability from Q, K
 * and them; a context upstream yields query, key and value gradients through
 * the exact softmax vector-Jacobian product; Causal mask: a masked score
 * carries exactly zero gradient).
 *   q [B,H,T,d], k/v [B,Hkv,T,d]: the forward's inputs; o [B,H,T,d]: its
 *   output; lse [B,H,T] float32: the row statistic (natural log) that
 *   attn_prefill wrote for the same q, k, v, scale and causal; dout
 *   [B,H,T,d]: the gradient of the loss with respect to o.
 *   dq [B,H,T,d], dk/dv [B,Hkv,T,d]: overwritten with the gradients; dk and dv
 *   hold the sums over the G = H/Hkv query heads that share each K/V head.
 *   Every tensor row-major and contiguous, 16-byte aligned, one dtype (f32,
 *   bf16 or f16) for all but lse.
 *   workspace: at least attn_prefill_backward_workspace_size() bytes, 16-byte
 *   aligned; contents on entry irrelevant, scratch afterwards.
 * Kernels: bf16/f16 with d a multiple of 16 in [64, 128] on the tensor cores;
 * float32, and 16-bit head widths outside that set, on CUDA cores in float32
 * (any d <= 256; larger d returns ATTN_ERR_UNSUPPORTED).
 * Errors as for attn_prefill plus ATTN_ERR_WORKSPACE; checks precede every
 * launch.  An empty problem launches nothing (with H = 0 but B*Hkv*T > 0,
 * dk and dv are set to zero).  Three kernels on `stream`, no allocation, no
 * synchronisation.
 */
ATTN_API size_t attn_prefill_backward_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H,
                                                     int64_t Hkv, int64_t T, int64_t d);
ATTN_API attn_status_t attn_prefill_backward(const void* q, const void* k, const void* v,
                                             const void* o, const float* lse, const void* dout,
                                             void* dq, void* dk, void* dv, attn_dtype_t dtype,
                                             int64_t B, int64_t H, int64_t Hkv, int64_t T,
                                             int64_t d, float scale, int causal, void* workspace,
                                             size_t workspace_bytes, void* stream);
/* The backward pass of local attention (attn_prefill_local's forward): row i
 * reads keys i - window < j <= i, so gradients flow only through those scores
 * ("Multi-query attention, annotated" §4.1; "Causal Multi-Head
 * Self-Attention", Causal mask: a masked score carries zero gradient).
 * Arguments, kernels, workspace and errors as for attn_prefill_backward
 * (always causal); window = 0, or a window of at least T, is plain causal
 * attention; window < 0 returns ATTN_ERR_INVALID_ARG. */
ATTN_API attn_status_t attn_prefill_backward_local(const void* q, const void* k, const void* v,
                                                   const void* o, const float* lse, const void* dout,
                                                   void* dq, void* dk, void* dv, attn_dtype_t dtype,
                                                   int64_t B, int64_t H, int64_t Hkv, int64_t T,
                                                   int64_t d, float scale, int64_t window,
                                                   void* workspace, size_t workspace_bytes,
                                                   void* stream);

/* Bytes of workspace attn_cached needs for this problem (0 if none).  Pure
 * host arithmetic; valid without a GPU.  Returns 0 for arguments that
 * attn_cached would reject. */
ATTN_API size_t attn_cached_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                  int64_t Tnew, int64_t S, int64_t d, int64_t start_pos);

/* Kernel family the call with these arguments would use; host-only, no GPU
 * needed.  Returns ATTN_KERNEL_NONE for an empty problem and -1 cast to
 * attn_kernel_t for arguments the entry point would reject. */
ATTN_API attn_kernel_t attn_prefill_plan(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                                int64_t d, int causal);
ATTN_API attn_kernel_t attn_cached_plan(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                               int64_t Tnew, int64_t S, int64_t S_cap, int64_t d,
                               int64_t start_pos);

/* Human-readable name of a status code (static string, never NULL). */
ATTN_API const char* attn_status_string(attn_status_t status);

/*
 * Device-side status.  Every wait inside the kernels is bounded; a wait that
 * runs out records ATTN_ERR_DEVICE_TIMEOUT in a per-device status word and
 * the kernel exits cleanly, leaving the context usable.  This call
 * synchronises `stream`, returns the recorded status (ATTN_OK if none) and,
 * if `reset` != 0, clears it.  Unlike the compute calls it blocks the host.
 */
ATTN_API attn_status_t attn_device_status(void* stream, int reset);

/* Bound for every device-side wait, in nanoseconds (default 2e9).  Tests
 * shorten it; 0 restores the default.  Host-side setting read at launch. */
ATTN_API void attn_set_wait_timeout_ns(uint64_t ns);

/* Test hook for the device timeout path (no counterpart in the pages):
 * flags & 1 makes the TMA producers of the tensor-core prefill, backward and
 * split-KV decode kernels issue no copies, so every bounded wait on them runs
 * out, the kernel
 * records ATTN_ERR_DEVICE_TIMEOUT and exits cleanly (its output is then
 * undefined).  0 restores normal operation.  Read at launch; not for
 * production use. */
ATTN_API void attn_test_set_flags(uint32_t flags);

/* Library version, as major * 10000 + minor * 100 + patch. */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* B200ATTN_H */
