// tile_plan.cuh -- which KV tiles a query tile visits, and which of them need
// element-wise masking.  Used by the prefill kernel and by the tile-plan debug
// entry point, so both report the same set.
//
// Key j is visible to query row i iff j < L and (not causal or
// j <= i + (Nk - Nq)), L = clamp(key_len, 0, Nk).  The visible keys of a row
// form a prefix whose length grows with i, so a query tile with rows
// [i0, i1) visits KV tiles 0 .. ceil(n(i1 - 1) / Bc) - 1 (n = prefix length)
// and every tile at or beyond floor(n(i0) / Bc) holds a masked element for
// some row.  Tiles wholly past every row's prefix are skipped.
#pragma once

namespace attn {

__host__ __device__ __forceinline__ int clamp_len(int key_len, int Nk) {
  return key_len < 0 ? 0 : (key_len > Nk ? Nk : key_len);
}

// Number of visible keys (the prefix length) of query row i.
__host__ __device__ __forceinline__ int visible_prefix(int i, int Nq, int Nk, int causal, int L) {
  int n = L;
  if (causal) {
    const long long c = (long long)i + (Nk - Nq) + 1;
    if (c < n) n = c < 0 ? 0 : (int)c;
  }
  return n;
}

struct KvRange {
  int count;        // tiles 0 .. count-1 are visited
  int first_masked; // tiles >= first_masked need the element mask
};

__host__ __device__ __forceinline__ KvRange kv_tile_range(int qt, int Br, int Bc, int Nq, int Nk,
                                                          int causal, int L) {
  const int i0 = qt * Br;
  int i1 = i0 + Br;
  if (i1 > Nq) i1 = Nq;
  KvRange r;
  const int nmax = visible_prefix(i1 - 1, Nq, Nk, causal, L);
  const int nmin = visible_prefix(i0, Nq, Nk, causal, L);
  r.count = (nmax + Bc - 1) / Bc;
  r.first_masked = nmin / Bc;
  return r;
}

}  // namespace attn
