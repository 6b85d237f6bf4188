/*
 * oracle.h -- plain, slow, fp64 CPU oracle for exact scaled dot-product
 * attention forward.  TEST INFRASTRUCTURE ONLY: only tests/, the package's
 * smoke() entry and bench.py's cpu_baseline / reference leg may load it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Every function takes bf16 inputs as raw 16-bit patterns (exactly widened to
 * double) and computes in double precision.  Sources (page title, section):
 *
 *   [CIA] "Coding interview (14): attention from scratch" (arganzheng.life),
 *         sections 3.1 softmax, 3.2 sdpa, 3.4 GQA, 3.5 RoPE, 3.6 KV cache,
 *         3.7 online softmax; self-test 5 (new tokens after a cache).
 *   [TAB] "Transformer Architecture Breakdown: Self-Attention, MHA/GQA/MQA,
 *         RoPE & FlashAttention 1/2/3" (airsota.com), sections 1.2, 3.1, 4.2.
 *   [AME] "Attention mechanisms: from alignment to efficient long context"
 *         (fahimfaisal.info), sections 3, 5, 9, 11 sliding window, 19,
 *         20 PagedAttention.
 *   [TIN] "Transformer Internals" (vanos001.github.io), Paged Attention.
 *   [TAD] "Transformer Architecture Deconstructed: Attention, Geometric
 *         Scaling, and Memory IO" (byronfinn.github.io), "Online Softmax and
 *         Blocked Incremental Computation".
 *
 * Parity status: every function here is pinned by tests/test_oracle.py
 * (closed forms, invariants, library special cases, printed worked values).
 */
#ifndef ATTN_ORACLE_H
#define ATTN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Stable softmax of x[0..n) into out ([CIA] 3.1: subtract the max, then
 * exponentiate and normalise).  n >= 1. */
void oracle_softmax(const double* x, int64_t n, double* out);

/* log(sum(exp(x))) computed as max + log(sum(exp(x - max))) ([CIA] 3.1).
 * Returns -inf for n == 0. */
double oracle_logsumexp(const double* x, int64_t n);

/* RoPE: out[b,h,t,:] = R(pos_offset + t) * x[b,h,t,:] in fp64 ([TAB] 3.1,
 * [CIA] 3.5).  theta_i = base^(-2i/d), i = 0..d/2-1.  pairing 0 rotates
 * (x_i, x_{i+d/2}); pairing 1 rotates (x_{2i}, x_{2i+1}).  Each pair (a, b)
 * becomes (a cos - b sin, a sin + b cos) with angle t * theta_i. */
void oracle_rope(const uint16_t* x, double* out, int64_t B, int64_t H,
                 int64_t N, int64_t d, double base, int64_t pos_offset,
                 int pairing);

/* Number of keys visible to query row i: keys j in [0, result) are visible.
 * L = key_len clamped to [0, Nk]; causal adds j <= i + (Nk - Nq)
 * (bottom-right alignment, [CIA] self-test 5).  Result may be 0. */
int64_t oracle_visible_prefix(int64_t i, int64_t Nq, int64_t Nk, int causal,
                              int64_t key_len);

/* Key position p of query row i.  align 0: p = i + (Nk - Nq) (the Nq rows
 * end at key Nk - 1).  align 1: p = i + (L - Nq), L = key_len clamped to
 * [0, Nk] (the rows are the newest Nq tokens of each sequence, [CIA]
 * self-test 5). */
int64_t oracle_query_position(int64_t i, int64_t Nq, int64_t Nk,
                              int64_t key_len, int align);

/* Visible keys of query row i as a range [lo, hi) (hi == lo: none):
 * j < L; causal adds j <= p; a sliding window w > 0 adds |p - j| < w
 * ([AME] 11); p from oracle_query_position. */
void oracle_visible_range_ex(int64_t i, int64_t Nq, int64_t Nk, int causal,
                             int64_t key_len, int64_t window, int align,
                             int64_t* lo, int64_t* hi);

/* oracle_visible_range_ex with align 0. */
void oracle_visible_range(int64_t i, int64_t Nq, int64_t Nk, int causal,
                          int64_t key_len, int64_t window, int64_t* lo,
                          int64_t* hi);

/* Definition of the result ([AME] 3, 5, 9; [CIA] 3.2, 3.4):
 *   g = h / (Hq / Hkv);  s_j = scale * <q_i, k_j> for visible j (the range
 *   of oracle_visible_range_ex; window <= 0 means no window, align picks
 *   the query positions);
 *   m = max s; p_j = exp(s_j - m); l = sum p; O_i = sum p_j v_j / l;
 *   lse_i = m + log(l).  No visible key: O_i = 0, lse_i = -inf.
 * Layout: q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] row-major bf16 bits.
 * rows: flat row ids r = (b*Hq + h)*Nq + i, or NULL for every row in order.
 * o: [nrows, d] doubles; lse: [nrows] (may be NULL).
 * rope != 0 rotates q at position q_pos_offset + i and k at k_pos_offset + j
 * in fp64 before the dot product; rope_round != 0 then rounds the rotated
 * rows to bf16 (nearest even), which models a RoPE pass that stores bf16
 * before the attention reads it.
 * key_lens: int32[B] or NULL (= Nk).  nthreads >= 1.
 * Returns 0, or -1 on invalid arguments. */
int oracle_attn_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                     int64_t Nk, int64_t d, int causal, int64_t window,
                     int align, double scale, const int32_t* key_lens, int rope,
                     double rope_base,
                     int rope_pairing, int rope_round, int64_t q_pos_offset,
                     int64_t k_pos_offset, const int64_t* rows, int64_t nrows,
                     double* o, double* lse, int nthreads);

/* Same result through the one-query-at-a-time online recurrence ([CIA] 3.7,
 * [AME] 19, [TAD] online softmax): keys visited in blocks of `block`, with a
 * running max m, running sum l and unnormalised accumulator rescaled by
 * exp(m_old - m_new) whenever the max grows.  No RoPE. */
int oracle_attn_online_rows(const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, int64_t B, int64_t Hq,
                            int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
                            int causal, int64_t window, int align,
                            double scale, const int32_t* key_lens,
                            int64_t block, const int64_t* rows, int64_t nrows,
                            double* o, double* lse, int nthreads);

/* Which KV tiles a query tile touches, by brute force over the visibility
 * predicate: tile jt (keys [jt*Bc, min((jt+1)*Bc, Nk))) is touched by query
 * tile qt (rows [qt*Br, min((qt+1)*Br, Nq))) iff some row of the query tile
 * sees some key of the KV tile.  Writes the first and last touched tile and
 * the count (first = last = -1, count = 0 when none). */
void oracle_kv_tiles(int64_t Nq, int64_t Nk, int causal, int64_t key_len,
                     int64_t Br, int64_t Bc, int64_t qt, int64_t* first,
                     int64_t* last, int64_t* count);

/* Same with a sliding window (window <= 0: none). */
void oracle_kv_tiles_window(int64_t Nq, int64_t Nk, int causal,
                            int64_t key_len, int64_t window, int64_t Br,
                            int64_t Bc, int64_t qt, int64_t* first,
                            int64_t* last, int64_t* count);

/* Same with a sliding window and a query alignment (see
 * oracle_query_position). */
void oracle_kv_tiles_ex(int64_t Nq, int64_t Nk, int causal, int64_t key_len,
                        int64_t window, int align, int64_t Br, int64_t Bc,
                        int64_t qt, int64_t* first, int64_t* last,
                        int64_t* count);

/* Paged KV cache ([TIN] PagedAttention; [AME] 20): key j of kv head h of
 * sequence b is row j % page_size of head h in physical block
 * block_table[b * max_pages + j / page_size]; cache [num_pages, Hkv,
 * page_size, d].  Gathers keys [0, key_lens[b]) into out [B, Hkv, Nk, d]
 * (zeros beyond key_lens[b]); attention over a paged cache is attention
 * over this gathered cache.  Returns 0, or -1 for a table entry outside
 * [0, num_pages) or max_pages * page_size < Nk. */
int oracle_gather_paged(const uint16_t* cache, int64_t num_pages, int64_t Hkv,
                        int64_t page_size, int64_t d,
                        const int32_t* block_table, int64_t max_pages,
                        const int32_t* key_lens, int64_t B, int64_t Nk,
                        uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
