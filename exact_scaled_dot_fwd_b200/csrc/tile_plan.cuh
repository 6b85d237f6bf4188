// tile_plan.cuh -- which keys a query row sees, which KV tiles a query tile
// visits, and which of them need element-wise masking.  Used by the prefill
// and decode kernels and by the tile-plan debug entry point, so all report
// the same set.
//
// Query row i sits at key position p = i + off, where off = Nk - Nq (the
// rows end at key Nk - 1) or off = L - Nq (align 1: the rows are the newest
// Nq tokens of a sequence of L keys; "Coding interview (14)", self-test 5).
// Key j is visible iff j < L (L = clamp(key_len, 0, Nk)), and, when causal,
// j <= p, and, with a sliding window w > 0 ("Attention mechanisms ...",
// section 11), |p - j| < w.  The visible keys of a row form a range
// [lo, hi) whose ends never decrease with i, and the rows that see any key
// form one contiguous block, so a query tile's KV tiles are a contiguous
// range computable in closed form.
#pragma once

namespace attn {

__host__ __device__ __forceinline__ int clamp_len(int key_len, int Nk) {
  return key_len < 0 ? 0 : (key_len > Nk ? Nk : key_len);
}

// p - i for the rows of a sequence with L keys (align 0: Nk - Nq, 1: L - Nq).
__host__ __device__ __forceinline__ int query_offset(int Nq, int Nk, int L, int align) {
  return (align ? L : Nk) - Nq;
}

// Number of visible keys (the prefix length) of query row i without a window.
__host__ __device__ __forceinline__ int visible_prefix(int i, int off, int causal, int L) {
  int n = L;
  if (causal) {
    const long long c = (long long)i + off + 1;
    if (c < n) n = c < 0 ? 0 : (int)c;
  }
  return n;
}

// Visible keys [lo, hi) of query row i (hi <= lo: none).
__host__ __device__ __forceinline__ void visible_range(int i, int off, int causal, int L,
                                                       int window, int* lo, int* hi) {
  int h = visible_prefix(i, off, causal, L);
  int l = 0;
  if (window > 0) {
    const long long p = (long long)i + off;
    if (p - window + 1 > l) l = (int)(p - window + 1);
    if (p + window < h) h = p + window < 0 ? 0 : (int)(p + window);
  }
  *lo = l;
  *hi = h > l ? h : l;
}

struct KvRange {
  int begin;       // first KV tile visited
  int count;       // tiles begin .. begin+count-1 are visited
  int um_begin;    // tiles in [um_begin, um_end) need no element mask
  int um_end;
};

// KV tiles of query tile qt (rows [qt*Br, min(qt*Br + Br, Nq))).
__host__ __device__ __forceinline__ KvRange kv_tile_range(int qt, int Br, int Bc, int Nq, int off,
                                                          int causal, int L, int window) {
  KvRange r;
  r.begin = 0;
  r.count = 0;
  r.um_begin = 0;
  r.um_end = 0;
  const int i0 = qt * Br;
  int i1 = i0 + Br;
  if (i1 > Nq) i1 = Nq;
  if (window <= 0) {
    // prefix ranges: tiles 0 .. ceil(n_max / Bc) - 1, unmasked below n_min / Bc
    const int nmax = visible_prefix(i1 - 1, off, causal, L);
    const int nmin = visible_prefix(i0, off, causal, L);
    r.count = (nmax + Bc - 1) / Bc;
    r.um_end = nmin / Bc;
    return r;
  }
  if (i1 <= i0 || L <= 0) return r;
  // rows that see at least one key: positions p in [p_min, p_max]
  const long long p_min = causal ? 0 : 1 - (long long)window;
  const long long p_max = (long long)L + window - 2;
  long long pa = (long long)i0 + off, pb = (long long)i1 - 1 + off;
  if (pa < p_min) pa = p_min;
  if (pb > p_max) pb = p_max;
  if (pa > pb) return r;
  int lo_a, hi_a, lo_b, hi_b;
  visible_range((int)(pa - off), off, causal, L, window, &lo_a, &hi_a);
  visible_range((int)(pb - off), off, causal, L, window, &lo_b, &hi_b);
  const int S = lo_a, E = hi_b;   // union of the rows' ranges
  if (E <= S) return r;
  r.begin = S / Bc;
  r.count = (E + Bc - 1) / Bc - r.begin;
  // element masks are needed unless a tile lies inside every row's range
  int lo_first, hi_first, lo_last, hi_last;
  visible_range(i0, off, causal, L, window, &lo_first, &hi_first);
  visible_range(i1 - 1, off, causal, L, window, &lo_last, &hi_last);
  const int um_b = (lo_last + Bc - 1) / Bc;   // first tile at or after every row's lo
  const int um_e = hi_first / Bc;             // tiles ending at or before every row's hi
  if (hi_first > lo_last && um_e > um_b) {
    r.um_begin = um_b;
    r.um_end = um_e;
  }
  return r;
}

// Decode (a few query rows per sequence, all read against one key range):
// keys [*lo, L) cover every row's visible range.  The last row's range ends
// at L (its position is at least L - 1) and row 0's starts first (range
// ends never decrease with the row); rows whose ranges start later or end
// earlier are masked element-wise.  Returns L - *lo (>= 0).
__host__ __device__ __forceinline__ int decode_key_range(int L, int off, int window, int* lo) {
  int l = 0;
  if (window > 0 && (long long)off - window + 1 > 0) l = off - window + 1;   // row 0's first key
  if (l > L) l = L;
  *lo = l;
  return L - l;
}

// Decode work split: the units' keys are laid end to end and split evenly
// over the CTAs, with `seg` virtual keys in front of every non-empty unit --
// the cost of starting a segment (its Q, the first tile's pipeline, the
// partial result) in keys, so a CTA whose range holds a unit start gets
// fewer real keys.
__host__ __device__ __forceinline__ int virtual_len(int len, int seg) {
  return len > 0 ? len + seg : 0;
}

}  // namespace attn
