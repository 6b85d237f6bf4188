// prefill.cu -- tiled exact attention forward (Nq > 1) on the sm_100a
// tensor cores: TMA -> shared memory, tcgen05.mma with accumulators in tensor
// memory (TMEM), online softmax in registers, TMA store of the output.
//
// Method ("Attention mechanisms ...", section 19; "Transformer Architecture
// Breakdown ...", section 4.2; "Coding interview (14)", section 3.7): stream
// K/V tiles past a block of queries, keep per row the running max m, running
// sum l and the unnormalised output O; when m grows, rescale O and l by
// 2^(m_old - m_new); divide by l at the end.  The score tile lives only in
// TMEM and registers.
//
// Work item = two query tiles of 128 rows that share one kv head (rows 2p,
// 2p+1 of one head, or -- when a kv head serves an even number of query heads
// -- the same rows of two query heads).  The kernel is persistent: one CTA
// per SM takes items one at a time from a global counter over a list sorted
// by cost (causal: most KV tiles first) -- greedy longest-first scheduling --
// and the next item's loads and first MMAs overlap the current item's tail.
// The K/V producer claims the item and hands its index to the other roles
// through a small ring in shared memory.  Warp roles:
//   warps 0-3  softmax for query tile 0 (one row per thread = one TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    tcgen05.mma issuer (one thread) and TMEM allocator
//   warp  9    K/V TMA producer and item scheduler (one thread)
//   warp 10    Q TMA producer (one thread)
// TMEM (512 columns): S0 | S1 | O0 | O1; P (bf16) is written over the first
// 64 columns of its S buffer and read by the MMA straight from TMEM.
// The MMA issue order per KV tile j is PV0(j), S0(j+1), PV1(j), S1(j+1):
// while one softmax group turns S into P, the tensor core works on the other
// query tile.  tcgen05 MMAs of one thread execute in issue order, so S(j+1)
// overwrites P(j) only after PV(j) has read it, and the commit after S(j+1)
// also covers PV(j) -- the softmax may rescale O as soon as S(j+1) is ready.
//
// Barrier phases run on across items; every role sees the same item
// sequence and derives the same tile counts, so the counters stay in step.
//
// Lazy rescale: O and l are rescaled only when a row's max grows by more
// than 8 (log2 units); otherwise the stale max is kept (P <= 2^8, exact in
// the final O / l because O and l share the same reference).
//
// Fused RoPE of Q (kRope instantiation, one more warp): after a Q tile
// lands, warps 10-11 rotate it in shared memory, two rows per thread (row i
// at position q_pos_offset + i, cos/sin from a table built for the call, the
// arithmetic of rope_math.cuh), and release it to the MMA issuer on Q_READY;
// the softmax warps never wait for it.  K is expected rotated (a KV cache
// stores keys rotated once); rotating K here would redo the work for every
// query tile that reads the K tile.
//
// Sliding window ("Attention mechanisms ...", section 11): a query tile
// visits the contiguous KV-tile range that covers its rows' windows.  When
// the two tiles of an item start at different KV tiles, the item's K/V
// stream covers the union of their ranges and each slot joins it at its own
// first tile and leaves after its own last: no scores are computed for a
// tile outside a query tile's range.

//
// Trace (FwdArgs::trace, a test hook): the MMA issuer records for every
// query tile the first and last KV tile whose scores it computed and how
// many, as it issues them.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "rope_math.cuh"
#include "tcgen05.cuh"
#include "tile_plan.cuh"

namespace attn {

namespace pf {

constexpr int kM = 128;        // query rows per tile (= TMEM lanes)
constexpr int kN = 128;        // keys per KV tile
constexpr int kMaxSortB = 64;  // batches up to this size are ordered by key length
// K/V ring stages: d = 128 fits three K and two V tiles beside the two Q
// tiles (224 KB); d = 64 fits three of each.
template <int D> struct Stages { static constexpr int K = 3, V = D == 128 ? 2 : 3; };
// 11 warps; the fused-RoPE instantiation adds a 12th, so that warps 10-11
// rotate the Q tiles (below)
constexpr int threads(bool rope) { return rope ? 384 : 352; }
constexpr int kItemSlots = 4;   // depth of the shared-memory ring of work items
// arrivals that free an item slot: MMA warp, the Q warp (fused RoPE: both Q
// warps, every thread), 256 softmax threads (every softmax thread arrives:
// measured faster than one elected arrival per warp after a warp barrier)
constexpr int item_readers(bool rope) { return rope ? 1 + 64 + 256 : 2 + 256; }
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Smem {
  static constexpr int kBox = 128 * 128;          // one 64-column box of a 128-row tile
  static constexpr int kTile = 128 * D * 2;       // Q, K or V tile
  static constexpr int kQ = 0;                    // Q[2]
  static constexpr int kKS = Stages<D>::K, kVS = Stages<D>::V;
  static constexpr int kK = kQ + 2 * kTile;       // K[kKS]
  static constexpr int kV = kK + kKS * kTile;     // V[kVS]
  static constexpr int kBar = kV + kVS * kTile;
  enum {
    Q_FULL = 0,                 // [2]
    Q_EMPTY = 2,                // [2] committed after the last S MMA of a tile
    K_FULL = 4,
    K_EMPTY = K_FULL + kKS,
    V_FULL = K_EMPTY + kKS,
    V_EMPTY = V_FULL + kVS,
    S_FULL = V_EMPTY + kVS,
    P_FULL = S_FULL + 2,
    O_FULL = P_FULL + 2,
    MMA_DONE = O_FULL + 2,
    ITEM_FULL = MMA_DONE + 1,            // [kItemSlots]
    ITEM_EMPTY = ITEM_FULL + kItemSlots, // [kItemSlots]
    Q_READY = ITEM_EMPTY + kItemSlots,   // [2] rotated Q tile in place (fused RoPE)
    NUM_BARS = Q_READY + 2
  };
  static constexpr int kItems = kBar + NUM_BARS * 8;      // int [kItemSlots]
  static constexpr int kTmemSlot = kItems + kItemSlots * 4;
  static constexpr int kAbort = kTmemSlot + 16;
  static constexpr int kPerm = kAbort + 16;              // int [kMaxSortB]
  static constexpr int kTotal = kPerm + kMaxSortB * 4 + 1024;   // + alignment slack
  static_assert(kTotal <= 232448, "shared memory over the 227 KB per-CTA limit");
};

struct Tile {
  int row_tile, head, count;
  int first;              // step of the item's KV stream at which this tile joins it
  int um_begin, um_end;   // KV tiles (absolute index) that need no element mask
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

}  // namespace pf

struct FwdArgs {
  unsigned int* sched;   // item counter, zero at launch
  __nv_bfloat16* o;
  float* lse;
  const int32_t* key_lens;
  int B, Hq, Hkv, Nq, Nk, causal;
  int window;       // sliding window in keys, 0 = none
  int align;        // query positions: 0 end at key Nk - 1, 1 at key key_lens[b] - 1
  const float2* rope_tab;   // fused RoPE of Q: (cos, sin) [Nq][d/2] (kRope)
  int rope_pairing;         // 0: (i, i + d/2), 1: (2i, 2i + 1)
  int head_pairs;   // 1: tiles are heads (2p, 2p+1) at one row tile; 0: row tiles 2p, 2p+1
  int ntq;          // ceil(Nq / 128)
  int units;        // items per cost rank (head_pairs: B*Hq/2, else B*Hq)
  int ranks;        // cost ranks (row tiles, or row-tile pairs)
  int band;         // ranks per band (item order: band, unit, rank in band)
  int sort_b;       // 1: sequences in the order of their key lengths, longest first
  int total;        // number of items
  float scale_log2;
  int32_t* trace;   // test hook: per query tile {first, last, count} of the KV tiles scored, or null
};

namespace pf {

struct Item {
  Tile tl[2];       // tl[0] has the fewer KV tiles
  int b, n, L;      // n: steps of the item's KV stream
  int off;          // key position of query row i is i + off
  int kv_begin;     // KV tile of stream step 0
  int kv_row0;      // cache row of KV tile kv_begin
};

// Item `idx` of the ordered list (window: the sliding window, 0 = none;
// callers pass a compile-time 0 when the launch has no window).  Ranks walk the row tiles (row pairs)
// from the most KV tiles to the fewest when causal; bands of `band` ranks
// keep one unit's (head's) items next to each other so the CTAs that run at
// the same time share its K/V in L2 (band = 1: plain rank-major order; a
// non-causal launch, whose ranks all cost the same, takes one band: unit-
// major order).  With sort_b the units' sequences come longest first
// (perm: the sequences by decreasing key length), so the list runs from the
// most expensive items to the cheapest and the dynamic claim is greedy
// longest-first across ragged batches too.
__device__ __forceinline__ Item make_item(const FwdArgs& a, int idx, int window, const int* perm) {
  Item it;
  const int per_band = a.units * a.band;
  const int full = a.ranks / a.band;
  int rank, unit;
  if (idx < full * per_band) {
    const int bi = idx / per_band, rem = idx - bi * per_band;
    unit = rem / a.band;
    rank = bi * a.band + (rem - unit * a.band);
  } else {
    const int lb = a.ranks - full * a.band, rem = idx - full * per_band;
    unit = rem / lb;
    rank = full * a.band + (rem - unit * lb);
  }
  if (a.head_pairs) {
    const int rt = a.causal ? (a.ntq - 1 - rank) : rank;
    const int hp2 = a.Hq >> 1;
    const int bs = unit / hp2;
    const int hp = unit - bs * hp2;
    it.b = (perm != nullptr && a.sort_b) ? perm[bs] : bs;
    it.tl[0].row_tile = it.tl[1].row_tile = rt;
    it.tl[0].head = 2 * hp;
    it.tl[1].head = 2 * hp + 1;
  } else {
    const int np = (a.ntq + 1) >> 1;
    const int p = a.causal ? (np - 1 - rank) : rank;
    const int bs = unit / a.Hq;
    const int h = unit - bs * a.Hq;
    it.b = (perm != nullptr && a.sort_b) ? perm[bs] : bs;
    it.tl[0].row_tile = 2 * p;
    it.tl[1].row_tile = 2 * p + 1;
    it.tl[0].head = it.tl[1].head = h;
  }
  it.L = clamp_len(a.key_lens ? a.key_lens[it.b] : a.Nk, a.Nk);
  it.off = query_offset(a.Nq, a.Nk, it.L, a.align);
  int begin[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    KvRange r;
    r.begin = r.count = r.um_begin = r.um_end = 0;
    if (it.tl[t].row_tile < a.ntq)
      r = kv_tile_range(it.tl[t].row_tile, kM, kN, a.Nq, it.off, a.causal, it.L, window);
    begin[t] = r.begin;
    it.tl[t].count = r.count;
    it.tl[t].um_begin = r.um_begin;
    it.tl[t].um_end = r.um_end;
  }
  // the stream starts at the earlier first tile (only a window makes the two
  // differ); each tile joins it at its own offset
  if (it.tl[0].count > 0 && it.tl[1].count > 0)
    it.kv_begin = begin[0] < begin[1] ? begin[0] : begin[1];
  else
    it.kv_begin = it.tl[0].count > 0 ? begin[0] : begin[1];
  it.n = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    it.tl[t].first = it.tl[t].count > 0 ? begin[t] - it.kv_begin : 0;
    const int e = it.tl[t].first + it.tl[t].count;
    if (e > it.n) it.n = e;
  }
  if (it.tl[0].count > it.tl[1].count) {
    const Tile x = it.tl[0];
    it.tl[0] = it.tl[1];
    it.tl[1] = x;
  }
  const int hk = it.tl[1].head / (a.Hq / a.Hkv);
  it.kv_row0 = (it.b * a.Hkv + hk) * a.Nk + it.kv_begin * kN;
  return it;
}

}  // namespace pf

// Rotate row r of the Q tile at `qs` (two or one 64-column boxes, 128-byte
// swizzle) in place; `pos_row` indexes the (cos, sin) table.  Two 16-byte
// chunks per step keep their table loads in flight together.
template <int D>
__device__ __forceinline__ void rope_q_row(uint8_t* qs, int r, int pos_row, const FwdArgs& a) {
  constexpr int kBox = 128 * 128;
  constexpr int kHalf = D / 2;
  auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
  auto hi = [](uint32_t w) { return __uint_as_float(w & 0xffff0000u); };
  const float4* tab = reinterpret_cast<const float4*>(a.rope_tab + (size_t)pos_row * kHalf);
  if (a.rope_pairing == 0) {
    // half pairs (i, i + D/2): chunk c of the first half with chunk c of the
    // second (D = 128: the same swizzled offset in the other box; D = 64:
    // chunk c + 4 of the same row)
#pragma unroll
    for (int c0 = 0; c0 < D / 16; c0 += 2) {
      uint4 va[2], vb[2];
      float4 cs[2][4];   // (cos, sin) of pairs 8c .. 8c+7
      uint8_t* pa[2];
      uint8_t* pb[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = c0 + u;
        pa[u] = qs + sw128_offset(r, c);
        pb[u] = D == 128 ? pa[u] + kBox : qs + sw128_offset(r, c + 4);
        va[u] = *reinterpret_cast<const uint4*>(pa[u]);
        vb[u] = *reinterpret_cast<const uint4*>(pb[u]);
#pragma unroll
        for (int q = 0; q < 4; ++q) cs[u][q] = tab[4 * c + q];
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
        const uint32_t wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float ra0, rb0, ra1, rb1;
          rope_rotate(lo(wa[k]), lo(wb[k]), make_float2(cs[u][k].x, cs[u][k].y), ra0, rb0);
          rope_rotate(hi(wa[k]), hi(wb[k]), make_float2(cs[u][k].z, cs[u][k].w), ra1, rb1);
          oa[k] = pack_bf16x2(ra0, ra1);
          ob[k] = pack_bf16x2(rb0, rb1);
        }
        *reinterpret_cast<uint4*>(pa[u]) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        *reinterpret_cast<uint4*>(pb[u]) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
      }
    }
  } else {
    // adjacent pairs (2i, 2i + 1): 4 pairs per 16-byte chunk
#pragma unroll
    for (int c0 = 0; c0 < D / 8; c0 += 2) {
      uint4 v[2];
      float4 cs[2][2];   // (cos, sin) of pairs 4c .. 4c+3
      uint8_t* p[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = c0 + u;
        p[u] = qs + (c >> 3) * kBox + sw128_offset(r, c & 7);
        v[u] = *reinterpret_cast<const uint4*>(p[u]);
        cs[u][0] = tab[2 * c];
        cs[u][1] = tab[2 * c + 1];
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 cc = cs[u][k >> 1];
          const float2 c2 = (k & 1) ? make_float2(cc.z, cc.w) : make_float2(cc.x, cc.y);
          float r0, r1;
          rope_rotate(lo(w[k]), hi(w[k]), c2, r0, r1);
          o[k] = pack_bf16x2(r0, r1);
        }
        *reinterpret_cast<uint4*>(p[u]) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

template <int D, bool kWindow, bool kRope>
__global__ void __launch_bounds__(pf::threads(kRope), 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, FwdArgs a) {
  using namespace pf;
  using L = Smem<D>;
  constexpr int kBoxes = D / 64;
  const int window = kWindow ? a.window : 0;
  constexpr int kKS = L::kKS, kVS = L::kVS;
  // TMEM columns: S of tile t at 128 t, O of tile t at 256 + D t
  constexpr uint32_t kIdescS = tc::idesc_bf16(kM, kN, false, false);
  constexpr uint32_t kIdescPV = tc::idesc_bf16(kM, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  // (the fused-RoPE instantiation keeps the plain order: the lookup pushed
  // its register allocation into spills, 1.8% slower)
  const int* perm = kRope ? nullptr : reinterpret_cast<int*>(smem + L::kPerm);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* items = reinterpret_cast<volatile int*>(smem + L::kItems);
  // next item index from the ring (every reader calls it once per item);
  // -1 ends the stream.  One thread, one arrival.
  auto next_item = [&](int& k) -> int {
    const int slot = k % kItemSlots;
    if (!mbar_wait(&bars[L::ITEM_FULL + slot], (k / kItemSlots) & 1, abort_flag)) return -1;
    const int idx = items[slot];
    mbar_arrive(&bars[L::ITEM_EMPTY + slot]);
    ++k;
    return idx;
  };


  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i) {
      uint32_t cnt = 1;
      if (i == L::P_FULL || i == L::P_FULL + 1) cnt = 128;
      if (i >= L::ITEM_EMPTY && i < L::ITEM_EMPTY + kItemSlots) cnt = item_readers(kRope);
      if (i == L::Q_READY || i == L::Q_READY + 1) cnt = 64;    // the two Q warps
      mbar_init(&bars[i], cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (!kRope && a.sort_b && threadIdx.x < a.B) {   // perm[rank] = sequence, longest first, ties by index
    const int i = threadIdx.x;
    const int li = clamp_len(a.key_lens[i], a.Nk);
    int rank = 0;
    for (int j = 0; j < a.B; ++j) {
      const int lj = clamp_len(a.key_lens[j], a.Nk);
      rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    reinterpret_cast<int*>(smem + L::kPerm)[rank] = i;
  }
  if (warp == 8) {
    tc::alloc(tmem_slot, 512);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------- K/V producer + scheduler
    if (lane == 0) {
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      int g = 0, k = 0;
      int gk = 0;   // K tiles whose barrier was armed (one more than g if a V wait gave up)
      bool ok = true;
      int idx = (int)atomicAdd(a.sched, 1u);
      while (ok) {
        if (idx >= a.total) idx = -1;
        const int slot = k % kItemSlots;
        if (!mbar_wait(&bars[L::ITEM_EMPTY + slot], ((k / kItemSlots) & 1) ^ 1, abort_flag)) break;
        items[slot] = idx;
        mbar_arrive(&bars[L::ITEM_FULL + slot]);
        ++k;
        if (idx < 0) break;
        const Item it = make_item(a, idx, window, perm);
        // claim the next item only while issuing this item's last tile, so
        // no CTA sits on a claimed item (greedy longest-first stays greedy);
        // the atomic's latency hides behind the last loads
        int nxt = -1;
        if (it.n == 0) nxt = (int)atomicAdd(a.sched, 1u);
        for (int j = 0; ok && j < it.n; ++j, ++g) {
          if (j == it.n - 1) nxt = (int)atomicAdd(a.sched, 1u);
          const int ks = g % kKS;
          if (!mbar_wait(&bars[L::K_EMPTY + ks], ((g / kKS) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars[L::K_FULL + ks], L::kTile);
          ++gk;
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d(smem + L::kK + ks * L::kTile + bx * L::kBox, &tk, bx * 64,
                        it.kv_row0 + j * kN, &bars[L::K_FULL + ks]);
          const int vs = g % kVS;
          if (!mbar_wait(&bars[L::V_EMPTY + vs], ((g / kVS) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars[L::V_FULL + vs], L::kTile);
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d(smem + L::kV + vs * L::kTile + bx * L::kBox, &tv, bx * 64,
                        it.kv_row0 + j * kN, &bars[L::V_FULL + vs]);
        }
        idx = nxt;
      }
      // every issued load must land before the CTA may exit (normally they
      // have all been consumed already, and these waits return at once);
      // counted per ring: a K tile whose V slot never freed was still loaded
      for (int j = gk - kKS > 0 ? gk - kKS : 0; j < gk; ++j)
        mbar_wait(&bars[L::K_FULL + j % kKS], (j / kKS) & 1, nullptr);
      for (int j = g - kVS > 0 ? g - kVS : 0; j < g; ++j)
        mbar_wait(&bars[L::V_FULL + j % kVS], (j / kVS) & 1, nullptr);
    }
  } else if (kRope && warp >= 10) {
    // ------------------------------------------------- Q producer + RoPE of Q
    // Lane 0 of warp 10 loads each Q tile; once it lands, the 64 threads of
    // warps 10-11 rotate it in place (rows q and q + 64 each, row i at
    // position q_pos_offset + i, cos/sin from the call's table, the
    // arithmetic of rope_math.cuh) and release it to the MMA issuer on
    // Q_READY.  The rotation runs while the softmax warps finish the
    // previous item, off their critical path.
    const int q = (warp - 10) * 32 + lane;
    if (warp == 10 && lane == 0) tma_prefetch_desc(&tq);
    int qn[2] = {0, 0}, k = 0;
    bool ok = true;
    for (int idx; ok && (idx = next_item(k)) >= 0;) {
      const Item it = make_item(a, idx, window, perm);
      if (it.n == 0) continue;
      for (int t = 0; t < 2 && ok; ++t) {
        if (it.tl[t].count == 0) continue;
        if (q == 0) {
          if (qn[t] > 0 && !mbar_wait(&bars[L::Q_EMPTY + t], (qn[t] - 1) & 1, abort_flag)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(&bars[L::Q_FULL + t], L::kTile);
            for (int bx = 0; bx < kBoxes; ++bx)
              tma_load_3d(smem + L::kQ + t * L::kTile + bx * L::kBox, &tq, bx * 64,
                          it.tl[t].row_tile * kM, it.b * a.Hq + it.tl[t].head,
                          &bars[L::Q_FULL + t]);
          }
        }
        if (!mbar_wait(&bars[L::Q_FULL + t], qn[t] & 1, abort_flag)) { ok = false; break; }
        ++qn[t];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = q + 64 * h, row = it.tl[t].row_tile * kM + r;
          if (row < a.Nq) rope_q_row<D>(smem + L::kQ + t * L::kTile, r, row, a);
        }
        fence_proxy_async_smem();   // the tensor core reads what this thread wrote
        mbar_arrive(&bars[L::Q_READY + t]);
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ Q producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      int qn[2] = {0, 0}, k = 0;
      bool ok = true;
      for (int idx; ok && (idx = next_item(k)) >= 0;) {
        const Item it = make_item(a, idx, window, perm);
        if (it.n == 0) continue;
        for (int t = 0; t < 2 && ok; ++t) {
          if (it.tl[t].count == 0) continue;
          if (qn[t] > 0 && !mbar_wait(&bars[L::Q_EMPTY + t], (qn[t] - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          ++qn[t];
          mbar_arrive_expect_tx(&bars[L::Q_FULL + t], L::kTile);
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_3d(smem + L::kQ + t * L::kTile + bx * L::kBox, &tq, bx * 64,
                        it.tl[t].row_tile * kM, it.b * a.Hq + it.tl[t].head, &bars[L::Q_FULL + t]);
        }
      }
      for (int t = 0; t < 2; ++t)   // the last Q load of each slot must land before exit
        if (qn[t] > 0) mbar_wait(&bars[L::Q_FULL + t], (qn[t] - 1) & 1, nullptr);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop -- waits, item bookkeeping and the
    // MMA descriptors are warp-uniform -- and one elected lane issues each
    // group of tcgen05 instructions.  (A loop run by a single lane made
    // every MMA issue cost about 100 cycles, which capped the tensor core
    // below the rate its 64-cycle 128x128x16 MMAs allow.)
    {
      const uint32_t q_base = smem_u32(smem + L::kQ);
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      // Descriptors are built once per call; a k-step only moves the start
      // address field (bits 0-13 hold address >> 4, and shared memory stays
      // below 256 KB, so the add never carries out of it).
      auto issue_s = [&](int t, int ks) {
        const uint64_t da = tc::smem_desc_sw128(q_base + t * L::kTile, 16, 1024);
        const uint64_t db = tc::smem_desc_sw128(k_base + ks * L::kTile, 16, 1024);
        const uint32_t dt = tmem + 128u * t;
        if (elect_one()) {
          tc::mma_ss(dt, da, db, kIdescS, 0u);
#pragma unroll
          for (int kk = 1; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * L::kBox + (kk & 3) * 32) >> 4);
            tc::mma_ss(dt, da + off, db + off, kIdescS, 1u);
          }
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int vs, bool acc) {
        const uint64_t dv = tc::smem_desc_sw128(v_base + vs * L::kTile, L::kBox, 1024);
        const uint32_t dt = tmem + 256u + D * t, pa = tmem + 128u * t;
        if (elect_one()) {
          tc::mma_ts(dt, pa, dv, kIdescPV, acc ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kN / 16; ++kk)
            tc::mma_ts(dt, pa + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV, 1u);
        }
        __syncwarp();
      };
      auto commit = [&](int bar) {
        if (elect_one()) tc::commit(&bars[bar]);
        __syncwarp();
      };
      // next item index, read by lane 0 and handed to the warp (one arrival)
      auto next_item_w = [&](int& k) -> int {
        int idx = -1;
        if (lane == 0) idx = next_item(k);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        k = __shfl_sync(0xffffffffu, k, 0);
        return idx;
      };
      // Each slot's work is one stream of KV tiles across items: in the step
      // that finishes item i, the S MMA of item i+1's first tile is issued
      // for every slot that starts item i+1 on its first stream step, so a
      // slot with fewer tiles moves on while the other one finishes.  Slot t
      // takes part in stream steps [f[t], f[t] + c[t]) of an item.
      int qf[2] = {0, 0}, pw[2] = {0, 0}, g = 0, k = 0;
      int tr_first[2] = {0, 0}, tr_cnt[2] = {0, 0};
      bool ok = true;
      struct Counts { int c[2], f[2], n, kv_begin, qid[2]; };   // all the issuer needs of an item
      auto fetch = [&](Counts& it) -> bool {   // next item that has KV tiles
        for (int idx; (idx = next_item_w(k)) >= 0;) {
          const Item full = make_item(a, idx, window, perm);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            it.c[t] = full.tl[t].count;
            it.f[t] = full.tl[t].first;
            it.qid[t] = (full.b * a.Hq + full.tl[t].head) * a.ntq + full.tl[t].row_tile;
          }
          it.n = full.n;
          it.kv_begin = full.kv_begin;
          if (it.n > 0) return true;
        }
        return false;
      };
      // trace hook: the KV tile of stream step `step` was scored for slot t
      auto trace_s = [&](const Counts& it, int t, int step) {
        if (a.trace == nullptr) return;
        const int kt = it.kv_begin + step;
        if (tr_cnt[t] == 0) tr_first[t] = kt;
        ++tr_cnt[t];
        if (step == it.f[t] + it.c[t] - 1) {
          if (lane == 0) {
            int32_t* r = a.trace + 3 * (size_t)it.qid[t];
            r[0] = tr_first[t];
            r[1] = kt;
            r[2] = tr_cnt[t];
          }
          tr_cnt[t] = 0;
        }
      };
      auto issue_first_s = [&](const Counts& it, int t, int ks) -> bool {
        if (!mbar_wait_warp(&bars[(kRope ? L::Q_READY : L::Q_FULL) + t], qf[t] & 1, abort_flag))
          return false;
        ++qf[t];
        tc::fence_after();
        issue_s(t, ks);
        commit(L::S_FULL + t);
        if (it.c[t] == 1) commit(L::Q_EMPTY + t);
        trace_s(it, t, it.f[t]);
        return true;
      };
      Counts cur, nxt;
      if (fetch(cur)) {
        ok = mbar_wait_warp(&bars[L::K_FULL + 0], 0, abort_flag);
        for (int t = 0; t < 2 && ok; ++t)
          if (cur.c[t] > 0 && cur.f[t] == 0) ok = issue_first_s(cur, t, 0);
        if (ok) commit(L::K_EMPTY + 0);
        int j = 0;
        while (ok) {
          const int vs = g % kVS, ksn = (g + 1) % kKS;
          const bool last = j == cur.n - 1;
          const bool more = last ? fetch(nxt) : true;
          if (!mbar_wait_warp(&bars[L::V_FULL + vs], (g / kVS) & 1, abort_flag)) { ok = false; break; }
          bool k_next = false;
          auto need_k = [&]() -> bool {
            if (k_next) return true;
            if (!mbar_wait_warp(&bars[L::K_FULL + ksn], ((g + 1) / kKS) & 1, abort_flag)) return false;
            tc::fence_after();
            k_next = true;
            return true;
          };
          for (int t = 0; t < 2 && ok; ++t) {
            const int f = cur.f[t], e = f + cur.c[t];
            if (j >= f && j < e) {
              if (!mbar_wait_warp(&bars[L::P_FULL + t], pw[t] & 1, abort_flag)) { ok = false; break; }
              ++pw[t];
              tc::fence_after();
              issue_pv(t, vs, j > f);
              if (j == e - 1) commit(L::O_FULL + t);
            }
            if (j + 1 >= f && j + 1 < e) {                    // same item, next tile
              if (!need_k()) { ok = false; break; }
              if (j + 1 == f) {                               // this slot joins the stream
                if (!issue_first_s(cur, t, ksn)) { ok = false; break; }
              } else {
                issue_s(t, ksn);
                commit(L::S_FULL + t);
                if (j + 2 == e) commit(L::Q_EMPTY + t);
                trace_s(cur, t, j + 1);
              }
            } else if (last && more && nxt.c[t] > 0 && nxt.f[t] == 0) {   // next item, first tile
              if (!need_k() || !issue_first_s(nxt, t, ksn)) { ok = false; break; }
            }
          }
          if (!ok) break;
          // every K tile the producer loads is released once, even one that
          // no slot scored (the ranges of an item's tiles leave no gap, so
          // this does not happen; it keeps the ring in step regardless)
          if (!k_next && (!last || more) && !need_k()) { ok = false; break; }
          commit(L::V_EMPTY + vs);
          if (k_next) commit(L::K_EMPTY + ksn);
          ++g;
          if (!last) {
            ++j;
          } else {
            if (!more) break;
            cur = nxt;
            j = 0;
          }
        }
      }
      // every MMA of this CTA must be complete before TMEM is released
      commit(L::MMA_DONE);
      mbar_wait_warp(&bars[L::MMA_DONE], 0, nullptr);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;                 // query tile slot of this warpgroup
    const int r = (warp & 3) * 32 + lane;    // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t scol = 128u * t, ocol = 256u + D * t;
    const float sl2 = a.scale_log2;
    // (not in the fused-RoPE instantiation: the extra store path made it
    // spill and measured 1.7% slower there)
    const bool o_32B = !kRope && (reinterpret_cast<uintptr_t>(a.o) & 31) == 0;
    int sw = 0, ow = 0, k = 0;
    bool ok = true;
    int idx = next_item(k);
    while (ok && idx >= 0) {
      const Item it = make_item(a, idx, window, perm);
      const Tile T = t == 0 ? it.tl[0] : it.tl[1];
      const bool mine = T.row_tile < a.ntq;
      const int row = T.row_tile * kM + r;
      int vlo, vhi;   // this row's visible keys [vlo, vhi)
      visible_range(row, it.off, a.causal, it.L, window, &vlo, &vhi);
      float m_run = -INFINITY, l_run = 0.f;

      for (int j = 0; mine && j < T.count; ++j) {
        if (!mbar_wait(&bars[L::S_FULL + t], sw & 1, abort_flag)) { ok = false; break; }
        ++sw;
        tc::fence_after();
        const int kt = it.kv_begin + T.first + j;   // KV tile index
        const bool masked = kWindow ? (kt < T.um_begin || kt >= T.um_end) : kt >= T.um_end;
        const int lim = vhi - kt * kN;    // keys [base, lim) of this tile are visible
        const int base = vlo - kt * kN;
        // Unmasked tiles after a row's first: the running max usually stands
        // (the lazy rescale keeps it unless a score passes it by more than 8
        // in log2 units), so P is computed with it from a single read of S,
        // the tile's max taken on the way, and P is written only if no row of
        // the warp needs a rescale.  Otherwise S is still intact in TMEM and
        // the two-pass path below runs.  When P is written it is bit for bit
        // what the two-pass path writes.  (Not in the window instantiation:
        // there the extra registers spilled and it measured 6% slower.)
        if (!kWindow && !masked && j > 0) {
          const float2 c_sl2 = make_float2(sl2, sl2), c_m = make_float2(-m_run, -m_run);
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          uint32_t pk[64];
          float rsum = 0.f;
#pragma unroll
          for (int c8 = 0; c8 < kN / 64; ++c8) {
            float sv[64];
            tc::ld32f(tmem + lane_off + scol + 64 * c8, sv);
            tc::ld32f(tmem + lane_off + scol + 64 * c8 + 32, sv + 32);
            tc::wait_ld();
            float2 rs2 = make_float2(0.f, 0.f), rs3 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              m4[e & 3] = max3(m4[e & 3], sv[2 * e], sv[2 * e + 1]);
              const float2 x = __ffma2_rn(make_float2(sv[2 * e], sv[2 * e + 1]), c_sl2, c_m);
              const float2 p = make_float2(exp2_approx(x.x), exp2_approx(x.y));
              if (e & 1) rs3 = __fadd2_rn(rs3, p); else rs2 = __fadd2_rn(rs2, p);
              pk[32 * c8 + e] = pack_bf16x2(p.x, p.y);
            }
            rs2 = __fadd2_rn(rs2, rs3);
            rsum += rs2.x + rs2.y;
          }
          const float m_tile = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
          const bool keep = m_run != -INFINITY && !(m_tile > m_run + kRescaleLog2);
          if (__all_sync(0xffffffffu, keep)) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::st16(tmem + lane_off + scol + 16 * c, pk + 16 * c);
            l_run += rsum;
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&bars[L::P_FULL + t]);
            continue;
          }
        }
        // A masked tile is taken in 32-key chunks, each classified for the
        // whole warp from the range of its rows' bounds: a chunk no row sees
        // any key of is skipped (P = 0 without reading S), a chunk every row
        // sees in full takes no mask, and only the rest is masked per key.
        // (A causal diagonal tile is one skipped, partial or full chunk per
        // warp and chunk; a window's edge tile likewise.)
        int lmin = 0, lmax = 0, bmin = 0, bmax = 0;
        if (masked) {
          lmin = __reduce_min_sync(0xffffffffu, lim);
          lmax = __reduce_max_sync(0xffffffffu, lim);
          if (kWindow) {
            bmin = __reduce_min_sync(0xffffffffu, base);
            bmax = __reduce_max_sync(0xffffffffu, base);
          }
        }
        auto chunk_dead = [&](int c0) { return c0 >= lmax || (kWindow && c0 + 32 <= bmin); };
        auto chunk_full = [&](int c0) { return c0 + 32 <= lmin && (!kWindow || c0 >= bmax); };
        // pass 1: row max of the (masked) scores
        float mx = -INFINITY;
        if (!masked) {
          // four independent max chains: the reduction's latency is a quarter
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c8 = 0; c8 < kN / 64; ++c8) {
            float sv[64];
            tc::ld32f(tmem + lane_off + scol + 64 * c8, sv);
            tc::ld32f(tmem + lane_off + scol + 64 * c8 + 32, sv + 32);
            tc::wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) m4[e & 3] = max3(m4[e & 3], sv[2 * e], sv[2 * e + 1]);
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        } else {
#pragma unroll 1
          for (int c4 = 0; c4 < kN / 32; ++c4) {
            const int c0 = 32 * c4;
            if (chunk_dead(c0)) continue;
            float sv[32];
            tc::ld32f(tmem + lane_off + scol + c0, sv);
            tc::wait_ld();
            if (chunk_full(c0)) {
              float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int e = 0; e < 16; ++e) m4[e & 3] = max3(m4[e & 3], sv[2 * e], sv[2 * e + 1]);
              mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int c = c0 + e;
                mx = fmaxf(mx, (c >= lim || (kWindow && c < base)) ? -INFINITY : sv[e]);
              }
            }
          }
        }
        const float m_tile = mx * sl2;
        const bool need = m_tile > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? fmaxf(m_run, m_tile) : m_run;
          if (j > 0) {
            const float f = (need && m_run != -INFINITY) ? exp2_approx(m_run - m_new) : 1.f;
            l_run *= f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float o[32];
              tc::ld32f(tmem + lane_off + ocol + 32 * c, o);
              tc::wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= f;
              tc::st32f(tmem + lane_off + ocol + 32 * c, o);
            }
          }
          m_run = m_new;
        }
        // pass 2: P = 2^(s * scale * log2e - m) as bf16 pairs over the first
        // 64 columns of S (chunk c reads S columns [64 c, 64 c + 64) and
        // writes P columns [32 c, 32 c + 32), which were already read)
        // Unmasked tiles scale, shift and sum on packed f32x2 pairs (one
        // instruction per two scores; the row sum keeps two partial sums).
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        float rs = 0.f;
        if (!masked) {
          const float2 c_sl2 = make_float2(sl2, sl2), c_m = make_float2(-m_use, -m_use);
#pragma unroll
          for (int c8 = 0; c8 < kN / 64; ++c8) {
            float sv[64];
            tc::ld32f(tmem + lane_off + scol + 64 * c8, sv);
            tc::ld32f(tmem + lane_off + scol + 64 * c8 + 32, sv + 32);
            tc::wait_ld();
            uint32_t pk[32];
            float2 rs2 = make_float2(0.f, 0.f), rs3 = make_float2(0.f, 0.f);   // two sum chains
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float2 x = __ffma2_rn(make_float2(sv[2 * e], sv[2 * e + 1]), c_sl2, c_m);
              const float2 p = make_float2(exp2_approx(x.x), exp2_approx(x.y));
              if (e & 1) rs3 = __fadd2_rn(rs3, p); else rs2 = __fadd2_rn(rs2, p);
              pk[e] = pack_bf16x2(p.x, p.y);
            }
            rs2 = __fadd2_rn(rs2, rs3);
            rs += rs2.x + rs2.y;
            tc::st16(tmem + lane_off + scol + 32 * c8, pk);
            tc::st16(tmem + lane_off + scol + 32 * c8 + 16, pk + 16);
          }
        } else {
#pragma unroll 1
          for (int c4 = 0; c4 < kN / 32; ++c4) {
            const int c0 = 32 * c4;
            uint32_t pk[16];
            if (chunk_dead(c0)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) pk[e] = 0u;
            } else {
              float sv[32];
              tc::ld32f(tmem + lane_off + scol + c0, sv);
              tc::wait_ld();
              if (chunk_full(c0)) {
                const float2 c_sl2 = make_float2(sl2, sl2), c_m = make_float2(-m_use, -m_use);
                float2 rs2 = make_float2(0.f, 0.f), rs3 = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const float2 x = __ffma2_rn(make_float2(sv[2 * e], sv[2 * e + 1]), c_sl2, c_m);
                  const float2 p = make_float2(exp2_approx(x.x), exp2_approx(x.y));
                  if (e & 1) rs3 = __fadd2_rn(rs3, p); else rs2 = __fadd2_rn(rs2, p);
                  pk[e] = pack_bf16x2(p.x, p.y);
                }
                rs2 = __fadd2_rn(rs2, rs3);
                rs += rs2.x + rs2.y;
              } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const int c = c0 + 2 * e;
                  const float x0 = (c >= lim || (kWindow && c < base)) ? -INFINITY : sv[2 * e];
                  const float x1 = (c + 1 >= lim || (kWindow && c + 1 < base)) ? -INFINITY : sv[2 * e + 1];
                  const float p0 = exp2_approx(fmaf(x0, sl2, -m_use));
                  const float p1 = exp2_approx(fmaf(x1, sl2, -m_use));
                  rs += p0 + p1;
                  pk[e] = pack_bf16x2(p0, p1);
                }
              }
            }
            tc::st16(tmem + lane_off + scol + 16 * c4, pk);
          }
        }
        l_run += rs;
        tc::wait_st();
        tc::fence_before();
        mbar_arrive(&bars[L::P_FULL + t]);
      }
      if (!ok) break;
      const int nidx = next_item(k);
      if (!mine) {
        idx = nidx;
        continue;
      }

      // ---- epilogue: O / l -> bf16 straight to global; lse
      const bool have = T.count > 0;
      if (have) {
        if (!mbar_wait(&bars[L::O_FULL + t], ow & 1, abort_flag)) { ok = false; break; }
        ++ow;
        tc::fence_after();
      }
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = a.o + (((size_t)it.b * a.Hq + T.head) * a.Nq + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (have) {
          tc::ld32f(tmem + lane_off + ocol + 32 * c, o);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
        if (row < a.Nq) {
          uint4 v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            v[q].x = pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
            v[q].y = pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
            v[q].z = pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
            v[q].w = pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
          }
          // a row is D * 2 bytes, so its 32-column chunks are 32-byte
          // aligned whenever o is: one full sector per store
          if (o_32B) {
            st_global_32B(orow + 32 * c, v[0], v[1]);
            st_global_32B(orow + 32 * c + 16, v[2], v[3]);
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q) = v[q];
          }
        }
      }
      tc::fence_before();
      if (a.lse && row < a.Nq)
        a.lse[((size_t)it.b * a.Hq + T.head) * a.Nq + row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      idx = nidx;
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 8) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side

bool prefill_supported(int d) { return d == 64 || d == 128; }

size_t prefill_workspace_bytes() { return 256; }

void prefill_tile_shape(int d, int* Br, int* Bc) {
  (void)d;
  *Br = pf::kM;
  *Bc = pf::kN;
}

int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, int causal, int window, int align,
                   float scale, const int32_t* key_lens, const float2* rope_tab,
                   int rope_pairing, void* workspace, int num_sms, cudaStream_t st,
                   int32_t* trace) {
  CUtensorMap tq, tk, tv;
  if (make_tmap_3d_bf16(&tq, q, d, Nq, (uint64_t)B * Hq, 64, pf::kM) != ATTN_OK) return ATTN_ECUDA;
  if (make_tmap_2d_bf16(&tk, k, d, (uint64_t)B * Hkv * Nk, 64, pf::kN) != ATTN_OK) return ATTN_ECUDA;
  if (make_tmap_2d_bf16(&tv, v, d, (uint64_t)B * Hkv * Nk, 64, pf::kN) != ATTN_OK) return ATTN_ECUDA;
  FwdArgs a;
  a.sched = static_cast<unsigned int*>(workspace);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.key_lens = key_lens;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.causal = causal;
  a.window = window;
  a.align = align;
  a.rope_tab = rope_tab;
  a.rope_pairing = rope_pairing;
  a.trace = trace;
  a.ntq = (Nq + pf::kM - 1) / pf::kM;
  a.head_pairs = ((Hq / Hkv) % 2 == 0) ? 1 : 0;
  a.scale_log2 = scale * kLog2e;
  a.units = a.head_pairs ? B * (Hq / 2) : B * Hq;
  a.ranks = a.head_pairs ? a.ntq : (a.ntq + 1) / 2;
  const long long total = (long long)a.units * a.ranks;
  if (total >= (1ll << 31)) return ATTN_EUNSUPPORTED;
  a.total = (int)total;
  const int grid = a.total < num_sms ? a.total : num_sms;
  // Band size: plain rank order while all of K/V fits comfortably in L2;
  // otherwise enough ranks per band that the heads in flight (about
  // grid / band) keep their K/V within ~64 MB of L2.
  const double kv_head = 4.0 * (double)Nk * d;   // K + V bytes of one kv head
  const double kv_all = kv_head * B * Hkv;
  int band = 1;
  if (!causal) {
    band = a.ranks;
  } else if (kv_all > 64.0 * (1 << 20)) {
    band = (int)ceil(grid * kv_head / (64.0 * (1 << 20)));
    if (band > a.ranks) band = a.ranks;
    if (band < 1) band = 1;
  }
  a.band = band;
  a.sort_b = (key_lens != nullptr && B > 1 && B <= pf::kMaxSortB) ? 1 : 0;
  // the item counter starts every launch at zero (stream-ordered)
  if (cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st) != cudaSuccess) return ATTN_ECUDA;
  // a window shifts each tile's first visible key: a separate instantiation
  // keeps that arithmetic out of the unwindowed kernel
  const bool win = window > 0, rope = rope_tab != nullptr;
  using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, FwdArgs);
  Kern kern;
  if (d == 128)
    kern = rope ? (win ? prefill_tc_kernel<128, true, true> : prefill_tc_kernel<128, false, true>)
                : (win ? prefill_tc_kernel<128, true, false> : prefill_tc_kernel<128, false, false>);
  else
    kern = rope ? (win ? prefill_tc_kernel<64, true, true> : prefill_tc_kernel<64, false, true>)
                : (win ? prefill_tc_kernel<64, true, false> : prefill_tc_kernel<64, false, false>);
  const int smem = d == 128 ? pf::Smem<128>::kTotal : pf::Smem<64>::kTotal;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ECUDA;
  kern<<<grid, pf::threads(rope), smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

__global__ void tile_plan_kernel(const int32_t* key_lens, int B, int Nq, int Nk, int causal,
                                 int window, int align, int Br, int Bc, int nqt, int32_t* first,
                                 int32_t* count) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * nqt) return;
  const int b = idx / nqt, qt = idx - b * nqt;
  const int L_b = clamp_len(key_lens ? key_lens[b] : Nk, Nk);
  const KvRange r =
      kv_tile_range(qt, Br, Bc, Nq, query_offset(Nq, Nk, L_b, align), causal, L_b, window);
  first[idx] = r.count > 0 ? r.begin : -1;
  count[idx] = r.count;
}

int launch_tile_plan(int B, int Nq, int Nk, int d, int causal, int window, int align,
                     const int32_t* key_lens, int32_t* first, int32_t* count, cudaStream_t st) {
  int Br, Bc;
  prefill_tile_shape(d, &Br, &Bc);
  const int nqt = (Nq + Br - 1) / Br;
  const int n = B * nqt;
  if (n == 0) return ATTN_OK;
  tile_plan_kernel<<<(n + 255) / 256, 256, 0, st>>>(key_lens, B, Nq, Nk, causal, window, align,
                                                    Br, Bc, nqt, first, count);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace attn
