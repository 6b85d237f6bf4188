/*
 * attn.h -- C ABI of the B200 (sm_100a) exact scaled-dot-product attention
 * forward library (libattn_b200.so).
 *
 * The operation ("Attention mechanisms: from alignment to efficient long
 * context", sections 3, 5, 9 and 19; "Transformer Architecture Breakdown ...",
 * section 1.2):
 *
 *     O = softmax(Q K^T * scale + M) V,    lse = log(sum(exp(Q K^T * scale + M)))
 *
 * computed tile by tile with the online-softmax recurrence (running max m,
 * running sum l, rescale factor alpha; "Coding interview (14): attention from
 * scratch", section 3.7; "Transformer Architecture Deconstructed ...", online
 * softmax), so the Nq x Nk score matrix never reaches device memory.
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE memory, row-major and contiguous:
 *       q   bf16 [B, Hq,  Nq, d]      k, v  bf16 [B, Hkv, Nk, d]
 *       o   bf16 [B, Hq,  Nq, d]      lse   fp32 [B, Hq, Nq]   (natural log)
 *     Query head h reads kv head h / (Hq / Hkv) (MHA: Hkv = Hq, MQA: Hkv = 1;
 *     "Attention mechanisms ...", sections 8 and 9).
 *   - The mask M is never materialised.  Key j is visible to query row i of
 *     batch b iff j < key_lens[b] and, when causal, j <= i + (Nk - Nq)
 *     (lower-triangular for Nq == Nk; bottom-right aligned otherwise, as in
 *     the multi-token decode mask of "Coding interview (14)", self-test 5).
 *     Masked entries get exactly zero weight (-inf).  A row with no visible
 *     key gets O = 0 and lse = -inf.
 *   - key_lens: DEVICE int32 [B] or NULL (= Nk for every batch).  Values are
 *     clamped to [0, Nk] by the kernels; keys at or beyond key_lens[b] must
 *     hold finite values (they are read by whole tiles, then masked).
 *   - stream: a cudaStream_t passed as void*.  Calls only enqueue work on it
 *     and never synchronise; results are valid once the stream reaches them.
 *   - Pointers must be 16-byte aligned.  No call retains or frees a caller
 *     pointer.
 *   - Return value: an attn_status.  Argument checks happen on the host
 *     before any launch; nothing is printed and nothing throws.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

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
  ATTN_EINVAL = 1,        /* null required pointer, bad size, Hq % Hkv != 0, bad scale */
  ATTN_EUNSUPPORTED = 2,  /* a shape this library does not implement (e.g. d not 64/128) */
  ATTN_EALIGN = 3,        /* a pointer not 16-byte aligned */
  ATTN_EWORKSPACE = 4,    /* workspace missing or smaller than attn_workspace_size() */
  ATTN_ECUDA = 5,         /* a CUDA runtime / driver call failed (launch, attribute) */
  ATTN_ETIMEOUT = 6,      /* a kernel gave up waiting on a barrier (device status) */
  ATTN_ERANGE = 7         /* a kernel met an out-of-range block-table entry (device status) */
} attn_status;

/* Exact attention forward.  Dispatch: calls with at most 64 query rows per kv
 * head ((Hq / Hkv) * Nq <= 64: single-token decode, multi-token decode) and
 * B <= 2048 run the split-KV decode kernel followed by the log-sum-exp
 * combine pass; all
 * others run the tiled prefill kernel (TMA + tcgen05/TMEM, persistent, one
 * CTA per SM).
 *   d: 64 or 128.  scale: finite and > 0 (usually 1/sqrt(d); "Transformer
 *   Architecture Breakdown ...", section 1.2).  causal: 0 or 1 (ignored in
 *   effect for Nq == 1, where j <= Nk - 1 always holds).
 *   lse may be NULL.  Both paths need scratch device memory (decode: its
 *   partial results; prefill: the work-item counter of its scheduler, zeroed
 *   in-stream before each launch): this entry point uses a workspace owned by
 *   the library, or the caller's buffer registered for the current device
 *   with attn_set_workspace.  The library's own is allocated with cudaMalloc
 *   on the first call per device and again whenever a call needs more; an
 *   outgrown buffer is kept (not freed, so no device-wide synchronisation is
 *   needed and work still queued on it is safe) until process exit.  The
 *   host side is thread-safe, but every call on a device shares the one
 *   buffer on the GPU: calls that overlap on the GPU (other streams, other
 *   host threads) must not run concurrently -- use attn_fwd_ws, with a
 *   workspace per stream, for that.
 * Errors: ATTN_EINVAL / EUNSUPPORTED / EALIGN before any launch; ATTN_ECUDA
 * if a launch or the workspace allocation fails; ATTN_EWORKSPACE if a
 * registered workspace is smaller than attn_workspace_size(...). */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
             float scale, const int32_t* key_lens, void* stream);

/* attn_fwd with a caller-owned device workspace of at least
 * attn_workspace_size(...) bytes (256-byte aligned; its contents need no
 * initialisation).  The workspace must stay untouched until the stream has
 * passed this call.  Returns ATTN_EWORKSPACE when it is missing or too small. */
ATTN_API int attn_fwd_ws(const void* q, const void* k, const void* v, void* o,
                float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                int causal, float scale, const int32_t* key_lens,
                void* workspace, size_t workspace_bytes, void* stream);

/* Query alignment (the `align` argument of attn_fwd_ex). */
#define ATTN_ALIGN_NK 0      /* row i at key position p = i + (Nk - Nq) */
#define ATTN_ALIGN_KEYLEN 1  /* row i at p = i + (L - Nq), L = clamp(key_lens[b], 0, Nk) */

/* The general entry point: attn_fwd_ws plus a sliding window and a choice of
 * query positions.
 *   Query row i of batch b sits at key position p (align, above).  Key j is
 *   visible iff j < L, and (causal) j <= p, and (window > 0) |p - j| < window
 *   ("Attention mechanisms ...", section 11).  window = 0: no window;
 *   window < 0, or align not 0/1: ATTN_EINVAL.  With causal = 1 a row sees
 *   the last `window` positions up to and including its own; with causal = 0
 *   it also sees window - 1 positions after it.
 *   ATTN_ALIGN_KEYLEN is multi-token decode over ragged caches ("Coding
 *   interview (14)", self-test 5): the Nq rows are the newest Nq tokens of
 *   each sequence, whose cache plus those tokens fill keys [0, L); with
 *   causal = 1, row i sees the L - Nq cached keys and new tokens 0..i.  With
 *   L = Nk for every sequence both alignments agree.  The ABI's other entry
 *   points use ATTN_ALIGN_NK.
 *   The prefill kernel scores only the KV tiles that hold visible keys
 *   (attn_fwd_tile_plan_ex gives them, attn_fwd_trace observes them); the
 *   decode kernels read each
 *   sequence's keys from the first one its first row sees up to L.
 *   Workspace: attn_workspace_size(...) bytes, as for attn_fwd_ws.
 * Errors: as attn_fwd_ws. */
ATTN_API int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                         int window, int align, float scale, const int32_t* key_lens,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Decode over a paged KV cache ("Attention mechanisms ...", section 20;
 * "Transformer internals", PagedAttention): logical key j of kv head h of
 * sequence b lives in physical block p = block_table[b * max_pages +
 * j / page_size], row j % page_size:
 *     k_cache, v_cache  bf16 [num_pages, Hkv, page_size, d]   (DEVICE)
 *     block_table       int32 [B, max_pages]                  (DEVICE)
 *     key_lens          int32 [B], required (DEVICE): sequence lengths
 *   q/o bf16 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq] or NULL.  The Nq query rows
 *   of a sequence are its newest Nq tokens (ATTN_ALIGN_KEYLEN of attn_fwd_ex);
 *   causal and window as there, with Nk = max_pages * page_size.
 *   Runs the split-KV decode kernels: (Hq / Hkv) * Nq <= 64, B <= 2048.  page_size: a
 *   multiple of 8 dividing 128 (d = 128) or 64 (d = 64) -- 8, 16, 32, 64
 *   (and 128 for d = 128).  Only entries j / page_size < ceil(key_lens[b] /
 *   page_size) of a sequence's table row are read; rows of its last page at
 *   or beyond key_lens[b] must hold finite values.  The kernels check every
 *   table entry they read: an entry outside [0, num_pages) is never used as
 *   an address -- that page's keys and values read as zeros -- and the device
 *   status word records ATTN_ERANGE (attn_device_status returns it after the
 *   stream passes the call).  No entry makes a kernel read outside k_cache /
 *   v_cache.
 *   Workspace: attn_workspace_size(B, Hq, Hkv, Nq, Nk, d) bytes.
 * Errors: ATTN_EINVAL (null table or key_lens, bad sizes), ATTN_EUNSUPPORTED
 * (page_size, more than 64 query rows per kv head or 2048 sequences, d), then
 * as attn_fwd_ws. */
ATTN_API int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_table, int max_pages, int page_size,
                            int num_pages, void* o, float* lse, int B, int Hq, int Hkv,
                            int Nq, int d, int causal, int window, float scale,
                            const int32_t* key_lens, void* workspace,
                            size_t workspace_bytes, void* stream);

/* attn_fwd_ex with align = ATTN_ALIGN_NK: sliding-window attention. */
ATTN_API int attn_fwd_window(const void* q, const void* k, const void* v, void* o,
                             float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             int causal, int window, float scale,
                             const int32_t* key_lens, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_fwd_ws needs for these sizes on the current device
 * (0 for invalid sizes). */
ATTN_API size_t attn_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/* Registers a caller-owned DEVICE buffer as attn_fwd's workspace on the
 * current device, in place of the library's own; ptr = NULL with bytes = 0
 * returns to the library's own.  (The pages define no library interface;
 * this is the allocation side of the boundary, for callers that manage device
 * memory themselves.)
 *   ptr: 256-byte aligned, bytes > 0; the library never frees it, never grows
 *   it and never allocates in its place: an attn_fwd call that needs more
 *   than `bytes` (attn_workspace_size) returns ATTN_EWORKSPACE before any
 *   launch.  The caller keeps the buffer alive, and untouched by other work,
 *   until every attn_fwd call that used it has completed on its stream and it
 *   has been unregistered or replaced.  Registration is per device and
 *   process-wide (all threads); it does not affect attn_fwd_ws and the other
 *   entry points that take their workspace as an argument.
 * Errors: ATTN_EINVAL if exactly one of ptr / bytes is zero, ATTN_EALIGN for
 * a misaligned ptr (both before any CUDA call), ATTN_ECUDA if no device is
 * current. */
ATTN_API int attn_set_workspace(void* ptr, size_t bytes);

/* RoPE prologue ("Transformer Architecture Breakdown ...", section 3.1;
 * "Coding interview (14)", section 3.5): for each row x of x_in at position
 * t = pos_offset + row index along N, and i = 0..d/2-1,
 *     theta_i = base^(-2i/d),  (a, b) -> (a cos t*theta_i - b sin t*theta_i,
 *                                         a sin t*theta_i + b cos t*theta_i)
 * pairing 0: (a, b) = (x_i, x_{i+d/2});  pairing 1: (a, b) = (x_{2i}, x_{2i+1}).
 *   x_in, x_out: DEVICE bf16 [B, H, N, d]; x_out == x_in (in place) allowed,
 *   partial overlap is not.  d even, 2 <= d <= 256.  base > 0, finite.
 *   The angle is formed and reduced in fp64; the rotation runs in fp32; the
 *   result is rounded to bf16 (nearest even). */
ATTN_API int rope_apply(const void* x_in, void* x_out, int B, int H, int N, int d,
               float base, int pos_offset, int pairing, void* stream);

/* Attention with the RoPE prologue of q fused in: as attn_fwd_ws, but q holds
 * UN-rotated queries; row i of q is rotated at position q_pos_offset + i with
 * rope_apply's frequencies, pairing and arithmetic (bit for bit the values
 * rope_apply would store), then attends.  k must hold keys already rotated
 * (rope_apply at their positions; a KV cache stores them that way).
 *   Prefill shapes rotate each Q tile in shared memory after its TMA load
 *   (each thread of the tile's softmax warpgroup rotates its own row), with a
 *   (cos, sin) table of the Nq positions built in the workspace; decode
 *   shapes ((Hq/Hkv) * Nq <= 64)
 *   rotate q into the workspace and run the decode kernels.
 *   rope_base > 0, rope_pairing 0 (i, i + d/2) or 1 (2i, 2i + 1),
 *   q_pos_offset >= 0.  Positions: row i of EVERY sequence is rotated at
 *   q_pos_offset + i, matching the ATTN_ALIGN_NK query positions this entry
 *   point attends with (q_pos_offset = Nk - Nq puts the rows at the end of
 *   the keys).  Ragged caches whose newest tokens sit at key_lens[b] - Nq + i
 *   need per-sequence positions: rotate q with rope_apply per sequence and
 *   call attn_fwd_ex with ATTN_ALIGN_KEYLEN instead.
 *   Workspace: attn_rope_workspace_size(...) bytes (256-byte aligned,
 *   contents need no initialisation).
 * Errors: as attn_fwd_ws. */
ATTN_API int attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                           float scale, const int32_t* key_lens, float rope_base,
                           int rope_pairing, int q_pos_offset, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_fwd_rope needs (0 for invalid sizes). */
ATTN_API size_t attn_rope_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/* Tile shape (query rows Br, keys Bc) the prefill kernel uses for head
 * dimension d.  Returns ATTN_EUNSUPPORTED for other d. */
ATTN_API int attn_prefill_tile_shape(int d, int* Br, int* Bc);

/* The closed-form KV-tile range of every (b, query tile): the tiles that
 * hold a key visible to one of the tile's rows (the causal, key-length,
 * window and alignment rules of attn_fwd_ex).  Writes first[b * nqt + qt]
 * and count[b * nqt + qt] (nqt = ceil(Nq / Br); first = -1, count = 0 when
 * the tile sees no key).  Evaluates the device function the prefill kernel's
 * scheduler uses; what the kernel itself computes is observed by
 * attn_fwd_trace.  first/count: DEVICE int32 [B * nqt]. */
ATTN_API int attn_fwd_tile_plan(int B, int Nq, int Nk, int d, int causal,
                       const int32_t* key_lens, int32_t* first,
                       int32_t* count, void* stream);

/* attn_fwd_tile_plan under a sliding window of `window` keys (0 = none) and
 * a query alignment (as attn_fwd_ex): first = the first KV tile holding a
 * key visible to one of the tile's rows, count = how many in a row (the
 * range covers every visible key of the tile's rows and no tile without
 * one).  The prefill kernel scores exactly these tiles (attn_fwd_trace). */
ATTN_API int attn_fwd_tile_plan_ex(int B, int Nq, int Nk, int d, int causal,
                                   int window, int align, const int32_t* key_lens,
                                   int32_t* first, int32_t* count, void* stream);

/* attn_fwd_ex on the prefill kernel with a trace of the work it does (a
 * test hook; the pages define no such interface): for every query tile
 * (b, h, qt) of Br rows, the MMA-issuing thread records the first and last
 * KV tile whose scores it computed for that tile and how many, as it issues
 * them: trace[((b * Hq + h) * nqt + qt) * 3 + {0, 1, 2}] = {first, last,
 * count}, nqt = ceil(Nq / Br).  Entries of query tiles that score no KV tile
 * are not written (initialise them, e.g. to {-1, -1, 0}).  Output as
 * attn_fwd_ex.
 *   trace: DEVICE int32 [B * Hq * nqt * 3].  Shapes the decode kernels take
 *   ((Hq / Hkv) * Nq <= 64, B <= 2048) return ATTN_EUNSUPPORTED.
 *   Workspace as attn_fwd_ws (attn_workspace_size bytes).
 * Errors: ATTN_EINVAL for a null trace, else as attn_fwd_ex. */
ATTN_API int attn_fwd_trace(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                            int window, int align, float scale, const int32_t* key_lens,
                            void* workspace, size_t workspace_bytes, int32_t* trace,
                            void* stream);

/* attn_fwd_tile_plan_ex with align = ATTN_ALIGN_NK. */
ATTN_API int attn_fwd_tile_plan_window(int B, int Nq, int Nk, int d, int causal,
                                       int window, const int32_t* key_lens,
                                       int32_t* first, int32_t* count, void* stream);

/* Decode (Nq == 1) that allocates nothing.  The pages have no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc -- code
 * running under a fixed, preallocated memory budget, inside an allocator
 * hook or another runtime's callback, or on latency-critical paths where
 * cudaMalloc's implicit device synchronisation is not acceptable.
 *   Arguments, layouts and result are those of attn_fwd with Nq = 1:
 *   q/o bf16 [B, Hq, 1, d], k/v bf16 [B, Hkv, Nk, d], lse fp32 [B, Hq, 1] or
 *   NULL, key_lens device int32 [B] or NULL, d 64 or 128.
 *   The split-KV partial results live in a device array built into the
 *   library (attn_decode_static_max_bytes() = 8 MiB), held on every GPU that
 *   loads the library until the process exits.  Sizes whose partials do not
 *   fit return ATTN_EWORKSPACE before any launch.
 *   All calls share that array and it keeps the last call's contents: calls
 *   that overlap on the GPU (other streams or threads) race and must be
 *   serialised.  No part of it needs to start at zero.
 *   The first call on a device looks up the array's device address with
 *   that device current and caches it; make that first call before any
 *   stream capture.
 * Errors: as attn_fwd, plus ATTN_EWORKSPACE for sizes beyond the array. */
ATTN_API int attn_fwd_decode_static(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int Hq, int Hkv, int Nk, int d,
                                    float scale, const int32_t* key_lens, void* stream);

/* Size in bytes of the device array attn_fwd_decode_static works in. */
ATTN_API size_t attn_decode_static_max_bytes(void);

/* Synchronises `stream`, then returns the device status word of the current
 * device: ATTN_ETIMEOUT if a kernel of this library gave up on a barrier
 * wait, ATTN_ERANGE if a paged decode met an out-of-range block-table entry
 * (the last such event since the last reset), else ATTN_OK (ATTN_ECUDA if
 * the synchronisation failed).  reset != 0 clears the word. */
ATTN_API int attn_device_status(void* stream, int reset);

/* attn_device_status(stream, 1): the status since the last read, then
 * cleared (read-and-clear, like cudaGetLastError). */
ATTN_API int attn_last_device_status(void* stream);

/* Failure-detection test hook: launches one tiny kernel whose single thread
 * waits on a barrier that nothing ever completes, giving up after limit_ns
 * (1 ns .. 1 s).  The wait's limit expires, the kernel records ATTN_ETIMEOUT
 * in the device status word (read it with attn_device_status) and returns;
 * nothing faults or hangs and the context stays usable.  Every barrier wait in
 * the attention kernels takes the same path, with a 2 s limit. */
ATTN_API int attn_debug_timeout_probe(unsigned long long limit_ns, void* stream);

/* Human-readable name of a status code (static string). */
ATTN_API const char* attn_strerror(int status);

/* ABI version of this header (incremented on incompatible changes). */
ATTN_API int attn_abi_version(void);

#define ATTN_ABI_VERSION 1

#ifdef __cplusplus
}
#endif
#endif
