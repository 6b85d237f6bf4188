// decode_tc.cu -- split-KV decode (one or a few query rows per sequence,
// d == 128) on the tcgen05 tensor cores.
//
// Same work split and partial-result format as the mma.sync decode kernel in
// decode.cu (balanced global key ranges per CTA, one partial per (CTA, unit)
// segment, merged by the log-sum-exp combine pass), but the two products run
// as tcgen05 MMAs with the roles of the operands swapped so that the 128-row
// MMA dimension is the keys:
//   S^T [128 keys x N heads]  = K_tile [128 x d] . Q^T      (TMEM, fp32)
//   O^T [d x N heads]        += V_tile^T [d x 128] . P^T   (TMEM, fp32)
// N = the unit's query rows rounded up to 16: its G = Hq / Hkv query heads
// times the Nq query rows of each (multi-token decode: Nq new tokens verified
// at once; "Coding interview (14)", self-test 5), R = G * Nq <= 64; these rows
// are contiguous in q, o and lse.  One softmax thread owns one
// key (one TMEM lane of S^T) and, for O^T, one dimension of d.  The per-head
// maximum over the tile's keys is one warp-wide redux.sync max per head plus
// a four-entry exchange (one per warp) in shared memory; per-head running
// sums stay per thread until the segment ends, where a butterfly
// transpose-reduce across the warp sums them.  P^T goes to shared memory (bf16,
// the B operand of the PV MMA).  S^T is double-buffered in TMEM, so the S MMA
// of tile j+2 and the loads run while the softmax works on tile j.
//
// Warp roles: warps 0-3 softmax (TMEM lane quarters 0-3), warp 4 MMA issuer
// (the whole warp runs its loop; one elected lane issues the tcgen05
// instructions) and TMEM allocator, warp 5 TMA producer.
//
// Ring depths are chosen per launch: 3 K and 3 V tiles when they fit beside
// the per-sequence arrays of the batch (most batches), else 2 + 3, else 2 + 2
// (measured on the MQA decode workload: 2 + 3 with a single-lane MMA loop
// 4736 GB/s, 3 + 3 4774, 3 + 3 with the warp-wide MMA loop 4834).
//
// Paged KV cache ("Attention mechanisms ...", section 20; "Transformer
// internals", PagedAttention): key j of a sequence lives in physical block
// block_table[b][j / page_size] at offset j % page_size (cache [num_pages,
// Hkv, page_size, d]).  A 128-key tile starts on a page boundary and arrives
// as 128 / page_size TMA boxes of page_size rows, one per page, into the same
// swizzled tile layout; pages past the segment's end are loaded from a row
// past the cache (the TMA fills zeros), so unused table entries are never
// read, and an entry outside [0, num_pages) is replaced by that row and
// reported (ATTN_ERANGE in the device status word).  Keys of the tile
// outside the segment are masked.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tile_plan.cuh"

namespace attn {
namespace dtc {

constexpr int kTile = 128;   // keys per tile
constexpr int kD = 128;
constexpr int kMaxB = 2048;
constexpr float kRescaleLog2 = 8.0f;

// 4D tiled load (no multicast): coordinates (x inner, y, z, w); the paged
// cache's grouped boxes.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, int x, int y,
                                            int z, int w, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}

template <int N, int KS_, int VS_>
struct Smem {
  // Ring depths.  A K slot frees as soon as its S MMA has run, a V slot only
  // after the softmax of its tile and the PV MMA, so V needs at least as deep
  // a ring as K to keep enough loads in flight.  The launch picks the
  // deepest pair that fits beside the per-sequence arrays of its batch.
  static constexpr int KS = KS_;                  // K ring stages
  static constexpr int VS = VS_;                  // V ring stages
  static constexpr int kKV = kTile * kD * 2;   // one K or V tile (32 KB)
  // A K/V tile of a contiguous cache lands as two 64-column halves of 128
  // keys (kBox apart); one of a paged cache as 16 groups of 8 keys, each
  // [half 0 | half 1] of 1 KB, so that a page is one TMA box.  In both, each
  // half is a column of 1 KB 128-byte-swizzled atoms at a uniform stride.
  static constexpr int kBox = kTile * 128;     // 64-column box of a K/V tile
  static constexpr uint32_t half_step(bool paged) { return paged ? 1024u : (uint32_t)kBox; }
  static constexpr uint32_t group_stride(bool paged) { return paged ? 2048u : 1024u; }
  static constexpr int kQBox = N * 128;        // 64-column box of Q (N rows)
  static constexpr int kPBox = N * 128;        // 64-key box of P^T (N rows)
  static constexpr int kK = 0;
  static constexpr int kV = kK + KS * kKV;
  static constexpr int kQ = kV + VS * kKV;
  static constexpr int kP = kQ + 2 * kQBox;    // P^T [2 buffers][2 boxes]
  static constexpr int kRed = kP + 4 * kPBox;      // float [4][64]
  static constexpr int kMs = kRed + 4 * 64 * 4;    // float [64] running max (log2 units)
  static constexpr int kAs = kMs + 64 * 4;         // float [64] this tile's rescale factor
  static constexpr int kLs = kAs + 64 * 4;         // float [64] segment row sums
  static constexpr int kBar = kLs + 64 * 4;
  enum {
    K_FULL = 0,
    K_EMPTY = K_FULL + KS,
    V_FULL = K_EMPTY + KS,
    V_EMPTY = V_FULL + VS,
    Q_FULL = V_EMPTY + VS,
    Q_EMPTY = Q_FULL + 1,
    S_FULL = Q_EMPTY + 1,    // [2]
    P_FULL = S_FULL + 2,     // [2], 128 arrivals
    PV_DONE = P_FULL + 2,    // [2]
    MMA_DONE = PV_DONE + 2,
    NUM_BARS = MMA_DONE + 1
  };
  static constexpr int kTmemSlot = kBar + NUM_BARS * 8;
  static constexpr int kAbort = kTmemSlot + 16;
  // per-sequence arrays, sized by the launch's B: int [B + 1] key prefix over
  // b, int [B] keys per unit, int [B] first key
  static constexpr int kScan = kAbort + 16;
  static constexpr int scan_bytes(int B) { return (3 * B + 2) * 4; }
  static constexpr int total(int B) { return kScan + scan_bytes(B) + 1024; }   // + alignment slack
  static constexpr bool fits(int B) { return total(B) <= 232448; }
};

struct Seg {
  int u, lo, hi;      // unit and its keys [lo, hi), relative to the unit's first key
  int start, end;     // the same keys as absolute key indices of the sequence
  int base, n;        // first key of tile 0 (page-aligned when paged), tiles
};

// (B * Hkv * Nk < 2^31 is checked on the host, so every prefix fits an int.)
__device__ __forceinline__ long long unit_prefix(const int* pb, const int* lens, int u,
                                                 int Hkv, int seg) {
  const int b = u / Hkv, h = u - b * Hkv;
  return (long long)Hkv * pb[b] + (long long)h * virtual_len(lens[b], seg);
}

// One butterfly step across lanes `OFF` apart: each lane keeps the half of
// its HALF*2 values selected by its lane bit and combines it with the
// partner's other half.
template <int HALF, int OFF, bool SUM, int NV>
__device__ __forceinline__ void bfly_step(float (&v)[NV], int lane) {
  const bool up = (lane & OFF) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = up ? v[i] : v[i + HALF];
    const float keep = up ? v[i + HALF] : v[i];
    const float got = __shfl_xor_sync(0xffffffffu, send, OFF);
    v[i] = SUM ? keep + got : fmaxf(keep, got);
  }
}

// Reduce N per-lane values (one per head) over the 32 lanes of the warp.
// Afterwards v[0 .. R) hold the results for heads lane*R + i (N >= 32,
// R = N / 32) or head lane & 15 (N == 16, R = 1).
template <int N, bool SUM>
__device__ __forceinline__ void bfly_reduce(float (&v)[N], int lane) {
  if constexpr (N == 64) {
    bfly_step<32, 16, SUM>(v, lane);
    bfly_step<16, 8, SUM>(v, lane);
    bfly_step<8, 4, SUM>(v, lane);
    bfly_step<4, 2, SUM>(v, lane);
    bfly_step<2, 1, SUM>(v, lane);
  } else if constexpr (N == 32) {
    bfly_step<16, 16, SUM>(v, lane);
    bfly_step<8, 8, SUM>(v, lane);
    bfly_step<4, 4, SUM>(v, lane);
    bfly_step<2, 2, SUM>(v, lane);
    bfly_step<1, 1, SUM>(v, lane);
  } else {
    bfly_step<8, 8, SUM>(v, lane);
    bfly_step<4, 4, SUM>(v, lane);
    bfly_step<2, 2, SUM>(v, lane);
    bfly_step<1, 1, SUM>(v, lane);
    const float o = __shfl_xor_sync(0xffffffffu, v[0], 16);
    v[0] = SUM ? v[0] + o : fmaxf(v[0], o);
  }
}

// Per-head maximum over the warp's 32 keys into red[warp][head]: one
// warp-wide f32 max reduction (redux.sync) per head; lane h & 31 keeps the
// result of head h and stores it.
template <int N>
__device__ __forceinline__ void col_max_to_red(float* red, int warp, int lane,
                                               const float (&v)[N]) {
  float mine[N > 32 ? 2 : 1];
#pragma unroll
  for (int i = 0; i < (N > 32 ? 2 : 1); ++i) mine[i] = -INFINITY;
#pragma unroll
  for (int h = 0; h < N; ++h) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v[h]));
    if ((h & 31) == lane) mine[h >> 5] = r;
  }
  if (N >= 32 || lane < N) red[warp * 64 + lane] = mine[0];
  if (N > 32) red[warp * 64 + 32 + lane] = mine[N > 32 ? 1 : 0];
}

// Store this warp's reduced values into red[warp][head].
template <int N>
__device__ __forceinline__ void put_red(float* red, int warp, int lane, const float (&v)[N]) {
  if constexpr (N >= 32) {
    constexpr int R = N / 32;
#pragma unroll
    for (int i = 0; i < R; ++i) red[warp * 64 + lane * R + i] = v[i];
  } else {
    if (lane < 16) red[warp * 64 + lane] = v[0];
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[N]) {
  if constexpr (N == 16) {
    tc::ld16f(taddr, v);
  } else {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) tc::ld32f(taddr + 32 * c, v + 32 * c);
  }
}

template <int N>
__device__ __forceinline__ void tmem_st_row(uint32_t taddr, const float (&v)[N]) {
  if constexpr (N == 16) {
    tc::st16f(taddr, v);
  } else {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) tc::st32f(taddr + 32 * c, v + 32 * c);
  }
}


}  // namespace dtc

struct DecodeTcArgs {
  const int32_t* key_lens;
  float* part_o;
  float* part_lse;
  int B, Hq, Hkv, Nk, G, grid;
  int Nq, R;                 // query rows per sequence, rows per unit (G * Nq)
  int causal, window, align;
  int seg_cost;              // virtual keys in front of every non-empty unit
  float scale_log2;
  // paged cache (kernel instantiation with kPaged): Nk = max_pages * page_size
  const int32_t* block_table;
  int max_pages, page_size, num_pages, oob_row;   // oob_row: first row past the cache
};

template <int N, bool kPaged, int KS_, int VS_>
__global__ void __launch_bounds__(192, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, DecodeTcArgs a) {
  using namespace dtc;
  using L = Smem<N, KS_, VS_>;
  constexpr int KS = L::KS, VS = L::VS;
  constexpr uint32_t kIdescS = tc::idesc_bf16(kTile, N, false, false);
  // P^T, the PV MMA's B operand: K-major up to 32 rows (each head's keys
  // contiguous, two boxes of 64 keys; a thread stores its key's P head by
  // head); MN-major at N = 64, where a key's 64 heads are one 128-byte row
  // and a thread stores them as eight 16-byte chunks.
  constexpr bool kPMn = N == 64;
  constexpr uint32_t kIdescPV = tc::idesc_bf16(kD, N, true, kPMn);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  int* pb = reinterpret_cast<int*>(smem + L::kScan);   // [B + 1]
  int* lens_s = pb + a.B + 2;                          // [B]
  int* lo_s = lens_s + a.B;                            // [B]
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* m_s = reinterpret_cast<float*>(smem + L::kMs);
  float* a_s = reinterpret_cast<float*>(smem + L::kAs);
  float* l_s = reinterpret_cast<float*>(smem + L::kLs);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  // the combine pass may launch now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.B, Hkv = a.Hkv, U = B * Hkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i)
      mbar_init(&bars[i], (i == L::P_FULL || i == L::P_FULL + 1) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tc::alloc(tmem_slot, 256);
    tc::relinquish();
  }
  // Launched as a programmatic dependent of the previous kernel in the
  // stream: the set-up above may overlap its tail (the previous decode
  // call's combine pass releases its dependents early); nothing is read
  // from or written to global memory before the previous grid has
  // completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // key lengths (clamped) and their exclusive prefix over b, by warp 5
  if (warp == 5) {
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int len = 0;
      if (b < B) {
        const int Lb = clamp_len(a.key_lens ? a.key_lens[b] : a.Nk, a.Nk);
        int lo;
        len = decode_key_range(Lb, query_offset(a.Nq, a.Nk, Lb, a.align), a.window, &lo);
        lens_s[b] = len;   // keys [lo, L) of every unit of sequence b
        lo_s[b] = lo;
      }
      const int vlen = virtual_len(len, a.seg_cost);
      int x = vlen;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < B) pb[b] = carry + x - vlen;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pb[B] = carry;
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long T = (long long)Hkv * pb[B];
  const long long start = T * blockIdx.x / a.grid;
  const long long end = T * (blockIdx.x + 1) / a.grid;
  int u0 = 0;
  if (start < end) {
    int lo = 0, hi = U - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (unit_prefix(pb, lens_s, mid, Hkv, a.seg_cost) <= start) lo = mid; else hi = mid - 1;
    }
    u0 = lo;
  }
  auto next_seg = [&](int& u, Seg& s) -> bool {
    while (u < U) {
      const long long p0 = unit_prefix(pb, lens_s, u, Hkv, a.seg_cost);
      if (p0 >= end) return false;
      const int len = lens_s[u / Hkv];
      const long long r0 = p0 + (len > 0 ? a.seg_cost : 0);   // the unit's first real key
      const long long p1 = r0 + len;
      const long long lo = start > r0 ? start : r0, hi = end < p1 ? end : p1;
      const int cur = u++;
      if (hi > lo) {
        s.u = cur; s.lo = (int)(lo - r0); s.hi = (int)(hi - r0);
        const int kl = lo_s[cur / Hkv];
        s.start = kl + s.lo;
        s.end = kl + s.hi;
        s.base = kPaged ? s.start - s.start % a.page_size : s.start;
        s.n = (s.end - s.base + kTile - 1) / kTile;
        return true;
      }
    }
    return false;
  };

  if (warp == 5) {
    // ------------------------------------------------------------ producer
    // Lane 0 waits on the rings and arms the barriers.  The K/V loads of a
    // tile are issued by lane 0 (contiguous cache) or by lane p for page p of
    // the tile (paged: each lane reads its own block-table entry one tile
    // ahead, so the reads overlap and the code stays small).
    if (start < end) {
      if (lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
      }
      int u = u0, g = 0, qn = 0;
      int gk = 0, gv = 0;   // K and V tiles whose barriers were armed (for the drain)
      Seg s;
      bool ok = true;
      const int npg = kPaged ? kTile / a.page_size : 1;
      const bool issuer = kPaged ? lane < npg : lane == 0;
      while (ok && next_seg(u, s)) {
        const int b = s.u / Hkv, h = s.u - b * Hkv;
        const int n = s.n;
        bool w = true;
        if (lane == 0) {
          w = qn == 0 || mbar_wait(&bars[L::Q_EMPTY], (qn - 1) & 1, abort_flag);
          if (w) {
            mbar_arrive_expect_tx(&bars[L::Q_FULL], 2 * L::kQBox);
            for (int bx = 0; bx < 2; ++bx)
              tma_load_2d(smem + L::kQ + bx * L::kQBox, &tmap_q, bx * 64,
                          (b * a.Hq + h * a.G) * a.Nq, &bars[L::Q_FULL]);
          }
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) break;
        ++qn;
        const int row0 = s.u * a.Nk + s.base;   // contiguous cache
        const int32_t* table = kPaged ? a.block_table + (size_t)b * a.max_pages : nullptr;
        // paged: the cache row of this lane's page of tile j (or a row past
        // the cache, which the TMA fills with zeros)
        auto page_row = [&](int j) -> int {
          const int pg = (s.base + j * kTile) / a.page_size + lane;
          return (lane < npg && pg * a.page_size < s.end)
                     ? paged_cache_row(table[pg], a.num_pages, Hkv, h, a.page_size, a.oob_row)
                     : a.oob_row;
        };
        int prow = kPaged ? page_row(0) : 0;
        const uint32_t so = kPaged ? (uint32_t)(lane * a.page_size * 256) : 0u;   // page's groups
        for (int j = 0; j < n; ++j, ++g) {
          const int ks = g % KS, vs = g % VS;
          const int pnext = (kPaged && j + 1 < n) ? page_row(j + 1) : 0;
          const int r = kPaged ? prow : row0 + j * kTile;
          if (lane == 0) {
            w = mbar_wait(&bars[L::K_EMPTY + ks], ((g / KS) & 1) ^ 1, abort_flag);
            if (w) mbar_arrive_expect_tx(&bars[L::K_FULL + ks], L::kKV);
          }
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
          ++gk;
          if (issuer) {
            if constexpr (kPaged) {
              tma_load_4d(smem + L::kK + ks * L::kKV + so, &tmap_k, 0, 0, 0, r >> 3,
                          &bars[L::K_FULL + ks]);
            } else {
              for (int bx = 0; bx < 2; ++bx)
                tma_load_2d(smem + L::kK + ks * L::kKV + bx * L::kBox, &tmap_k, bx * 64, r,
                            &bars[L::K_FULL + ks]);
            }
          }
          if (lane == 0) {
            w = mbar_wait(&bars[L::V_EMPTY + vs], ((g / VS) & 1) ^ 1, abort_flag);
            if (w) mbar_arrive_expect_tx(&bars[L::V_FULL + vs], L::kKV);
          }
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
          ++gv;
          if (issuer) {
            if constexpr (kPaged) {
              tma_load_4d(smem + L::kV + vs * L::kKV + so, &tmap_v, 0, 0, 0, r >> 3,
                          &bars[L::V_FULL + vs]);
            } else {
              for (int bx = 0; bx < 2; ++bx)
                tma_load_2d(smem + L::kV + vs * L::kKV + bx * L::kBox, &tmap_v, bx * 64, r,
                            &bars[L::V_FULL + vs]);
            }
          }
          prow = pnext;
        }
      }
      // every issued load must land before the CTA may exit (counted per
      // ring: a K tile whose V slot never freed was still armed and loaded)
      if (lane == 0) {
        for (int j = gk - KS > 0 ? gk - KS : 0; j < gk; ++j)
          mbar_wait(&bars[L::K_FULL + j % KS], (j / KS) & 1, nullptr);
        for (int j = gv - VS > 0 ? gv - VS : 0; j < gv; ++j)
          mbar_wait(&bars[L::V_FULL + j % VS], (j / VS) & 1, nullptr);
        if (qn > 0) mbar_wait(&bars[L::Q_FULL], (qn - 1) & 1, nullptr);
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs the loop (warp-uniform waits and descriptors); one
    // elected lane issues each group of tcgen05 instructions
    if (start < end) {
      const uint32_t k_base = smem_u32(smem + L::kK), v_base = smem_u32(smem + L::kV);
      const uint32_t q_base = smem_u32(smem + L::kQ), p_base = smem_u32(smem + L::kP);
      // descriptors built once per call; a k-step only moves the start
      // address field (address >> 4 in bits 0-13, no carry below 256 KB)
      // a k-step of 16 keys is two 8-key groups; one of 64 columns a half
      constexpr uint32_t kHalf = L::half_step(kPaged), kGroup = L::group_stride(kPaged);
      auto issue_s = [&](int g) {
        const uint64_t dk = tc::smem_desc_sw128(k_base + (g % KS) * L::kKV, 16, kGroup);
        const uint64_t dq = tc::smem_desc_sw128(q_base, 16, 1024);
        const uint32_t dt = tmem + (uint32_t)((g & 1) * N);
        if (elect_one()) {
          tc::mma_ss(dt, dk, dq, kIdescS, 0u);
#pragma unroll
          for (int kk = 1; kk < kD / 16; ++kk)
            tc::mma_ss(dt, dk + (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4),
                       dq + (uint64_t)(((kk >> 2) * L::kQBox + (kk & 3) * 32) >> 4), kIdescS, 1u);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int g, bool acc) {
        const uint64_t dv = tc::smem_desc_sw128(v_base + (g % VS) * L::kKV, kHalf, kGroup);
        // MN-major P^T: one 64-head atom across, 8-key groups 1 KB apart
        const uint64_t dp = tc::smem_desc_sw128(p_base + (g & 1) * 2 * L::kPBox,
                                                kPMn ? 2u * L::kPBox : 16u, 1024);
        if (elect_one()) {
          tc::mma_ss(tmem + 2u * N, dv, dp, kIdescPV, acc ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kTile / 16; ++kk) {
            const uint32_t pk = kPMn ? (uint32_t)(kk * 2048)
                                     : (uint32_t)((kk >> 2) * L::kPBox + (kk & 3) * 32);
            tc::mma_ss(tmem + 2u * N, dv + (uint64_t)((kk * 2 * kGroup) >> 4),
                       dp + (uint64_t)(pk >> 4), kIdescPV, 1u);
          }
        }
        __syncwarp();
      };
      auto commit = [&](int bar) {
        if (elect_one()) tc::commit(&bars[bar]);
        __syncwarp();
      };
      int u = u0, g = 0, qf = 0;
      Seg s;
      bool ok = true;
      while (ok && next_seg(u, s)) {
        const int n = s.n;
        if (!mbar_wait_warp(&bars[L::Q_FULL], qf & 1, abort_flag)) break;
        ++qf;
        for (int t = 0; t < 2 && t < n && ok; ++t) {
          const int gt = g + t;
          if (!mbar_wait_warp(&bars[L::K_FULL + gt % KS], (gt / KS) & 1, abort_flag)) { ok = false; break; }
          tc::fence_after();
          issue_s(gt);
          commit(L::S_FULL + (gt & 1));
          commit(L::K_EMPTY + gt % KS);
        }
        if (ok && n <= 2) commit(L::Q_EMPTY);
        for (int j = 0; ok && j < n; ++j, ++g) {
          if (!mbar_wait_warp(&bars[L::P_FULL + (g & 1)], (g >> 1) & 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait_warp(&bars[L::V_FULL + g % VS], (g / VS) & 1, abort_flag)) { ok = false; break; }
          tc::fence_after();
          issue_pv(g, j > 0);
          commit(L::PV_DONE + (g & 1));
          commit(L::V_EMPTY + g % VS);
          if (j + 2 < n) {
            const int g2 = g + 2;
            if (!mbar_wait_warp(&bars[L::K_FULL + g2 % KS], (g2 / KS) & 1, abort_flag)) { ok = false; break; }
            tc::fence_after();
            issue_s(g2);
            commit(L::S_FULL + (g2 & 1));
            commit(L::K_EMPTY + g2 % KS);
            if (j + 2 == n - 1) commit(L::Q_EMPTY);
          }
        }
      }
      commit(L::MMA_DONE);
      mbar_wait_warp(&bars[L::MMA_DONE], 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int Lr = warp * 32 + lane;                 // key row of S^T, dimension of O^T
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    // Above 32 rows a thread cannot keep its whole row of S^T in registers
    // beside its N running sums: it reads S^T from TMEM in 32-column parts,
    // once for the maxima and again for P.
    constexpr bool kReload = N > 32;
    constexpr int NC = kReload ? 32 : N;
    uint8_t* p_smem = smem + L::kP;
    int u = u0, g = 0;
    Seg s;
    bool ok = start < end;
    while (ok && next_seg(u, s)) {
      const int n = s.n;
      // the rows' position offset
      const int sb = s.u / a.Hkv;
      const int Lb = clamp_len(a.key_lens ? a.key_lens[sb] : a.Nk, a.Nk);
      const int off = query_offset(a.Nq, a.Nk, Lb, a.align);
      asm volatile("bar.sync 1, 128;" ::: "memory");   // previous segment done with m_s / l_s
      if (Lr < 64) m_s[Lr] = -INFINITY;
      float lp[N];
#pragma unroll
      for (int h = 0; h < N; ++h) lp[h] = 0.f;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      for (int j = 0; j < n; ++j, ++g) {
        const int buf = g & 1;
        // A wait that gives up only clears ok: the thread carries on to the
        // next barrier, where all four warps vote (bar_or) and leave
        // together -- one that left alone would strand the others at it.
        if (!mbar_wait(&bars[L::S_FULL + buf], (g >> 1) & 1, abort_flag)) ok = false;
        tc::fence_after();
        const int kfirst = s.base + j * kTile;   // absolute key of this tile's row 0
        const bool valid = kfirst + Lr < s.end && (!kPaged || kfirst + Lr >= s.start);
        // rows (tokens) that do not see every key of this tile: causal keys
        // past row 0's position, window keys before the last row's window
        const int klast = kfirst + kTile - 1;
        const bool tile_mask =
            (a.causal && klast > off) ||
            (a.window > 0 && ((long long)kfirst < (long long)off + a.Nq - a.window ||
                              (!a.causal && (long long)klast >= (long long)off + a.window)));
        // this key is visible to the rows whose token index t satisfies
        // t >= key - off (causal) and |off + t - key| < window
        int tlo = -(1 << 30), thi = 1 << 30;
        if (tile_mask) {
          const int key = kfirst + Lr;
          if (a.causal) tlo = key - off;
          if (a.window > 0) {
            const int wlo = key - off - a.window + 1;
            tlo = tlo > wlo ? tlo : wlo;
            thi = key - off + a.window - 1;
          }
        }
        // S^T columns h0 .. h0 + NC of buffer `buf`, masked
        float sv[NC];
        auto load_s = [&](int h0) {
          tmem_ld_row<NC>(tmem + lane_off + (uint32_t)(buf * N + h0), sv);
          tc::wait_ld();
          if (!valid) {
#pragma unroll
            for (int h = 0; h < NC; ++h) sv[h] = -INFINITY;
          }
          if (tile_mask) {
            int t = h0 % a.Nq;
#pragma unroll
            for (int h = 0; h < NC; ++h) {
              if (t < tlo || t > thi) sv[h] = -INFINITY;
              t = t + 1 == a.Nq ? 0 : t + 1;
            }
          }
        };
        // per-head max over the tile's keys
#pragma unroll
        for (int h0 = 0; h0 < N; h0 += NC) {
          load_s(h0);
          col_max_to_red<NC>(red + h0, warp, lane, sv);
        }
        if (bar_vote_or(1, 128, !ok || *abort_flag != 0)) {   // (also orders the red[] writes)
          ok = false;
          break;
        }
        bool need = false;
        if (Lr < N) {
          const float mt = fmaxf(fmaxf(red[Lr], red[64 + Lr]), fmaxf(red[128 + Lr], red[192 + Lr])) * sl2;
          const float mo = m_s[Lr];
          need = mt > mo + kRescaleLog2;
          const float mn = need ? fmaxf(mo, mt) : mo;
          a_s[Lr] = (need && mo != -INFINITY) ? exp2_approx(mo - mn) : 1.f;
          m_s[Lr] = mn;
        }
        const bool any = bar_vote_or(1, 128, need);
        float mu[NC];
        auto load_mu = [&](int h0) {
#pragma unroll
          for (int h = 0; h < NC; ++h) {
            const float m = m_s[h0 + h];
            mu[h] = m == -INFINITY ? 0.f : m;
          }
        };
        if (!kReload) load_mu(0);
        if (any) {
          float al[N];
#pragma unroll
          for (int h = 0; h < N; ++h) {
            al[h] = a_s[h];
            lp[h] *= al[h];
          }
          if (j > 0) {   // O^T holds tiles < j: wait for PV of tile j-1, then rescale
            if (mbar_wait(&bars[L::PV_DONE + ((g - 1) & 1)], ((g - 1) >> 1) & 1, abort_flag)) {
              tc::fence_after();
#pragma unroll
              for (int h0 = 0; h0 < N; h0 += NC) {
                float o[NC];
                tmem_ld_row<NC>(tmem + lane_off + 2u * N + h0, o);
                tc::wait_ld();
#pragma unroll
                for (int h = 0; h < NC; ++h) o[h] *= al[h0 + h];
                tmem_st_row<NC>(tmem + lane_off + 2u * N + h0, o);
              }
              tc::wait_st();
            } else {
              ok = false;
            }
          }
        }
        // P^T buffer `buf` was read by PV of tile g-2
        if (g >= 2 && !mbar_wait(&bars[L::PV_DONE + buf], ((g - 2) >> 1) & 1, abort_flag)) ok = false;
        uint8_t* pb_ = p_smem + buf * 2 * L::kPBox + (Lr >> 6) * L::kPBox;
        const int kc = (Lr & 63) >> 3, kb = (Lr & 7) * 2;
#pragma unroll
        for (int h0 = 0; h0 < N; h0 += NC) {
          if (kReload) {   // S^T is still in TMEM: its buffer is reused after P_FULL
            load_s(h0);
            load_mu(h0);   // before this part's P stores
          }
          if constexpr (kPMn) {
            // this key's row of P^T: heads h0 .. h0 + 32 are 16-byte chunks
            // h0 / 8 .. h0 / 8 + 3, swizzled with the key's row in its atom
            uint8_t* prow = p_smem + buf * 2 * L::kPBox + Lr * 128;
#pragma unroll
            for (int c = 0; c < NC / 8; ++c) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int h = 8 * c + 2 * i;
                const float p0 = exp2_approx(fmaf(sv[h], sl2, -mu[h]));
                const float p1 = exp2_approx(fmaf(sv[h + 1], sl2, -mu[h + 1]));
                lp[h0 + h] += p0;
                lp[h0 + h + 1] += p1;
                w[i] = pack_bf16x2(p0, p1);
              }
              const int cc = h0 / 8 + c;
              *reinterpret_cast<uint4*>(prow + ((cc ^ (Lr & 7)) << 4)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int h = 0; h < NC; ++h) {
              const float p = exp2_approx(fmaf(sv[h], sl2, -mu[h]));
              lp[h0 + h] += p;
              const int hh = h0 + h;
              const uint32_t off = (uint32_t)hh * 128u + (uint32_t)((kc ^ (hh & 7)) << 4) + kb;
              *reinterpret_cast<__nv_bfloat16*>(pb_ + off) = __float2bfloat16_rn(p);
            }
          }
        }
        fence_proxy_async_smem();
        tc::fence_before();
        mbar_arrive(&bars[L::P_FULL + buf]);
      }
      if (bar_vote_or(1, 128, !ok)) {
        ok = false;
        break;
      }

      // ---- segment end: per-head sums, O^T / l, partial results
      const int glast = g - 1;
      if (!mbar_wait(&bars[L::PV_DONE + (glast & 1)], (glast >> 1) & 1, abort_flag)) ok = false;
      tc::fence_after();
      float o[N];
      tmem_ld_row<N>(tmem + lane_off + 2u * N, o);
      tc::wait_ld();
      bfly_reduce<N, true>(lp, lane);
      put_red<N>(red, warp, lane, lp);
      if (bar_vote_or(1, 128, !ok)) {
        ok = false;
        break;
      }
      if (Lr < N) l_s[Lr] = (red[Lr] + red[64 + Lr]) + (red[128 + Lr] + red[192 + Lr]);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const size_t slot = (size_t)blockIdx.x + s.u;
#pragma unroll
      for (int h = 0; h < N; ++h) {
        if (h < a.R) {
          const float l = l_s[h];
          a.part_o[(slot * a.R + h) * kD + Lr] = l > 0.f ? o[h] / l : 0.f;
        }
      }
      if (Lr < a.R && Lr < N) {
        const float l = l_s[Lr];
        a.part_lse[slot * a.R + Lr] = l > 0.f ? m_s[Lr] + __log2f(l) : -INFINITY;
      }
      tc::fence_before();
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 4) {
    tc::fence_after();
    tc::dealloc(tmem, 256);
  }
}

namespace {
template <int N, bool kPaged, int KS, int VS>
int launch_tc_t(int grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const DecodeTcArgs& a, cudaStream_t st) {
  auto kern = decode_tc_kernel<N, kPaged, KS, VS>;
  const int smem = dtc::Smem<N, KS, VS>::total(a.B);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ECUDA;
  return launch_programmatic(kern, dim3(grid), dim3(192), smem, st, tq, tk, tv, a);
}

// The deepest rings that fit with the batch's per-sequence arrays:
// 3 K + 3 V tiles, else 2 + 3, else 2 + 2.
template <int N, bool kPaged>
int launch_tc_rings(int grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const DecodeTcArgs& a, cudaStream_t st) {
  if (dtc::Smem<N, 3, 3>::fits(a.B)) return launch_tc_t<N, kPaged, 3, 3>(grid, tq, tk, tv, a, st);
  if (dtc::Smem<N, 2, 3>::fits(a.B)) return launch_tc_t<N, kPaged, 2, 3>(grid, tq, tk, tv, a, st);
  return launch_tc_t<N, kPaged, 2, 2>(grid, tq, tk, tv, a, st);
}
}  // namespace

bool decode_tc_supported(int B, int Hq, int Hkv, int Nq, int d) {
  return d == 128 && (Hq / Hkv) * Nq <= 64 && B <= dtc::kMaxB;
}

int launch_decode_split_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                           int Nq, int Nk, const DecodeMask& mk, const PagedKv* pg, float scale,
                           const int32_t* key_lens, float* part_o, float* part_lse, int grid,
                           cudaStream_t st) {
  const int G = Hq / Hkv, R = G * Nq;
  const int N = R <= 16 ? 16 : (R <= 32 ? 32 : 64);
  CUtensorMap tq, tk, tv;
  // contiguous: [B * Hkv * Nk, d] in 128-row, 64-column boxes; paged:
  // [num_pages * Hkv * page_size, d] in 8-row groups, one page per box
  const uint64_t rows = pg ? (uint64_t)pg->num_pages * Hkv * pg->page_size
                           : (uint64_t)B * Hkv * Nk;
  if (make_tmap_2d_bf16(&tq, q, dtc::kD, (uint64_t)B * Hq * Nq, 64, (uint32_t)N) != ATTN_OK)
    return ATTN_ECUDA;
  if (pg) {
    const uint32_t groups = (uint32_t)pg->page_size / 8;
    if (make_tmap_grouped_bf16(&tk, k, rows, groups) != ATTN_OK) return ATTN_ECUDA;
    if (make_tmap_grouped_bf16(&tv, v, rows, groups) != ATTN_OK) return ATTN_ECUDA;
  } else {
    if (make_tmap_2d_bf16(&tk, k, dtc::kD, rows, 64, dtc::kTile) != ATTN_OK) return ATTN_ECUDA;
    if (make_tmap_2d_bf16(&tv, v, dtc::kD, rows, 64, dtc::kTile) != ATTN_OK) return ATTN_ECUDA;
  }
  DecodeTcArgs a;
  a.block_table = pg ? pg->block_table : nullptr;
  a.max_pages = pg ? pg->max_pages : 0;
  a.page_size = pg ? pg->page_size : 0;
  a.num_pages = pg ? pg->num_pages : 0;
  a.oob_row = (int)rows;
  a.key_lens = key_lens;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nk = Nk; a.G = G; a.grid = grid;
  a.Nq = Nq; a.R = R;
  a.causal = mk.causal; a.window = mk.window; a.align = mk.align;
  a.seg_cost = mk.seg_cost;
  a.scale_log2 = scale * kLog2e;
  if (pg) {
    if (N == 16) return launch_tc_rings<16, true>(grid, tq, tk, tv, a, st);
    if (N == 32) return launch_tc_rings<32, true>(grid, tq, tk, tv, a, st);
    return launch_tc_rings<64, true>(grid, tq, tk, tv, a, st);
  }
  if (N == 16) return launch_tc_rings<16, false>(grid, tq, tk, tv, a, st);
  if (N == 32) return launch_tc_rings<32, false>(grid, tq, tk, tv, a, st);
  return launch_tc_rings<64, false>(grid, tq, tk, tv, a, st);
}

}  // namespace attn
