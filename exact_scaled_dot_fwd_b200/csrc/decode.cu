// decode.cu -- split-KV decode (one or a few query rows per sequence) and its
// log-sum-exp combine pass.
//
// One new query token per sequence reads the whole KV cache of its sequence
// ("Coding interview (14): attention from scratch", section 3.6: the newest
// token needs no causal mask, only the cache length; "Transformer
// Architecture Deconstructed ...", KV cache section: decode is a
// bandwidth-bound matrix-vector product).  All Hq/Hkv query heads that share
// a kv head are processed together, so every K/V byte is read from HBM once.
// Multi-token decode (Nq new tokens per sequence, e.g. verifying a draft;
// "Coding interview (14)", self-test 5) processes the R = (Hq/Hkv) * Nq rows
// of a kv head together the same way; the causal mask among the new tokens
// (and a sliding window, if any) is applied per (key, row).
//
// Work split.  Unit u = (b, kv head h) owns len_u = clamp(key_lens[b], 0, Nk)
// keys.  The units' keys are laid end to end (T keys in total) and CTA c of a
// one-wave grid of `grid` CTAs takes the global key range
// [c*T/grid, (c+1)*T/grid), which may cover
// the tail of one unit and the head of the next.  Every non-empty unit is
// laid out with seg_cost virtual keys in front of its real ones (about the
// cost of starting a segment, in keys), so a CTA whose range spans many short
// units gets fewer real keys.  Each (CTA, unit) piece is a
// segment: the CTA runs the online-softmax recurrence over it and writes a
// partial (O_s / l_s, log2 l_s + m_s) into slot c + u (unique: a later CTA
// never touches an earlier unit).  The combine pass merges the slots of each
// unit with the two-block merge rule of the online softmax ("Transformer
// Architecture Breakdown ...", section 4.2), generalised to n blocks.
//
// Head dimension 128 runs the tcgen05 split kernel of decode_tc.cu (same
// work split and partial format); the mma.sync split kernel below serves
// d = 64.  Both read either a contiguous cache or a paged one ("Attention
// mechanisms ...", section 20: key j in block block_table[b][j / page_size]
// at offset j % page_size); a paged tile starts on a page boundary and
// arrives as one TMA box per page, pages past the segment's end coming from
// a row past the cache (zero fill).
//
// Data movement.  K and V tiles of 64 keys arrive by TMA (2D tensor map over
// the [B*Hkv*Nk, d] cache, 128-byte swizzle) into a 4-stage shared-memory ring
// filled by a dedicated producer warp.  Consumer warps own 16 query heads
// (one m16 tile) and a quarter (16 keys) of every tile; they use
// ldmatrix + mma.sync.m16n8k16 (bf16 in, fp32 accumulate) for S = Q K^T and
// O += P V.  At 32 heads per kv head the path needs ~32 FLOP per byte, well
// inside what the tensor pipe sustains, so the kernel stays HBM-bound.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tile_plan.cuh"

namespace attn {

namespace {

constexpr int kTileKeys = 64;
constexpr int kStages = 4;
constexpr int kMaxScanB = 2048;

template <int D>
struct DecodeSmem {
  static constexpr int kTileBytes = kTileKeys * D * 2;   // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  // layout (from a 1024-byte aligned base)
  static constexpr int kRing = 0;
  static constexpr int kBars = kRing + kStages * kStageBytes;   // full[S], empty[S]
  static constexpr int kScan = kBars + 2 * kStages * 8;          // int64 [kMaxScanB + 1]
  static constexpr int kLens = kScan + (kMaxScanB + 1) * 8;      // int [kMaxScanB]
  static constexpr int kLo = kLens + kMaxScanB * 4;               // int [kMaxScanB]
  static constexpr int kMbuf = kLo + kMaxScanB * 4;               // float [4 kq][4 mt][16]
  static constexpr int kLbuf = kMbuf + 4 * 4 * 16 * 4;           // float [4 mt][16]
  static constexpr int kObuf = kLbuf + 4 * 16 * 4;               // float [4 mt][16][D]
  static constexpr int kAbort = kObuf + 4 * 16 * D * 4;
  static constexpr int kTotal = kAbort + 16 + 1024;              // + alignment slack
};

struct Seg {
  int u, lo, hi;
};

// Prefix of unit u: keys of all units before u (units are b-major, h-minor).
__device__ __forceinline__ long long unit_prefix(const long long* pb, const int* lens, int u,
                                                 int Hkv, int seg) {
  const int b = u / Hkv, h = u - b * Hkv;
  return (long long)Hkv * pb[b] + (long long)h * virtual_len(lens[b], seg);
}

}  // namespace

struct DecodeArgs {
  const __nv_bfloat16* q;
  const int32_t* key_lens;
  float* part_o;
  float* part_lse;
  int B, Hq, Hkv, Nk, G, grid;
  int Nq, R;                 // query rows per sequence, rows per unit (G * Nq)
  int causal, window, align;
  int seg_cost;              // virtual keys in front of every non-empty unit
  float scale_log2;
  // paged cache (kPaged): Nk = max_pages * page_size
  const int32_t* block_table;
  int max_pages, page_size, num_pages, oob_row;   // oob_row: first row past the cache
};

template <int D, int MT, bool kPaged>
__global__ void __launch_bounds__((MT * 4 + 1) * 32, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, DecodeArgs a) {
  using L = DecodeSmem<D>;
  constexpr int kConsumerWarps = MT * 4;
  constexpr int kConsumerThreads = kConsumerWarps * 32;
  constexpr int kBoxes = D / 64;             // 128-byte swizzle boxes per row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + kStages;
  long long* pb = reinterpret_cast<long long*>(smem + L::kScan);
  float* mbuf = reinterpret_cast<float*>(smem + L::kMbuf);
  float* lbuf = reinterpret_cast<float*>(smem + L::kLbuf);
  float* obuf = reinterpret_cast<float*>(smem + L::kObuf);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  int* lens_s = reinterpret_cast<int*>(smem + L::kLens);
  int* lo_s = reinterpret_cast<int*>(smem + L::kLo);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.B, Hkv = a.Hkv, U = B * Hkv;

  // the combine pass may launch now; it waits for this grid's results
  asm volatile("griddepcontrol.launch_dependents;");
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // a programmatic dependent of the previous kernel in the stream (as the
  // tcgen05 split kernel): global memory only after the previous grid
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // key lengths (clamped) and their exclusive prefix over b, by warp 0
  if (warp == 0) {
    long long carry = 0;
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
      long long x = vlen;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < B) pb[b] = carry + x - vlen;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pb[B] = carry;
  }
  __syncthreads();

  const long long T = (long long)Hkv * pb[B];
  const long long start = T * blockIdx.x / a.grid;
  const long long end = T * (blockIdx.x + 1) / a.grid;
  // first unit whose key range contains `start`
  int u0 = 0;
  if (start < end) {
    int lo = 0, hi = U - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (unit_prefix(pb, lens_s, mid, Hkv, a.seg_cost) <= start) lo = mid; else hi = mid - 1;
    }
    u0 = lo;
  }
  // first tile of a segment (relative to the unit's first key kl): its
  // first key, or the start of the page holding it when the cache is paged
  auto first_tile = [&](const Seg& s, int kl) -> int {
    return kPaged ? s.lo - (kl + s.lo) % a.page_size : s.lo;
  };
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
        return true;
      }
    }
    return false;
  };

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    // Lane 0 waits on the ring and arms the stage's barrier; the loads are
    // issued by lane 0 (contiguous cache) or by lane p for page p of the
    // tile (paged: each lane reads its block-table entry one tile ahead).
    if (start < end) {
      if (lane == 0) {
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
      }
      int u = u0, it = 0;
      Seg s;
      bool ok = true;
      const int npg = kPaged ? kTileKeys / a.page_size : 1;
      const bool issuer = kPaged ? lane < npg : lane == 0;
      while (ok && next_seg(u, s)) {
        const int b = s.u / Hkv, h = s.u - b * Hkv, kl = lo_s[b];
        const int32_t* table = kPaged ? a.block_table + (size_t)b * a.max_pages : nullptr;
        // paged: the cache row of this lane's page of the tile at t (or a row
        // past the cache, which the TMA fills with zeros)
        auto page_row = [&](int t) -> int {
          const int pg = (kl + t) / a.page_size + lane;
          return (lane < npg && pg * a.page_size < kl + s.hi)
                     ? paged_cache_row(table[pg], a.num_pages, Hkv, h, a.page_size, a.oob_row)
                     : a.oob_row;
        };
        const int t0 = first_tile(s, kl);
        int prow = kPaged ? page_row(t0) : 0;
        const int so = kPaged ? lane * a.page_size * 128 : 0;
        for (int t = t0; t < s.hi; t += kTileKeys, ++it) {
          const int st = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const int pnext = (kPaged && t + kTileKeys < s.hi) ? page_row(t + kTileKeys) : 0;
          const int r = kPaged ? prow : s.u * a.Nk + kl + t;
          bool w = true;
          if (lane == 0) {
            w = mbar_wait(&empty[st], ph ^ 1, abort_flag);
            if (w) mbar_arrive_expect_tx(&full[st], L::kStageBytes);
          }
          if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
          uint8_t* kt = smem + L::kRing + st * L::kStageBytes;
          uint8_t* vt = kt + L::kTileBytes;
          if (issuer) {
#pragma unroll
            for (int bx = 0; bx < kBoxes; ++bx) {
              tma_load_2d(kt + bx * (kTileKeys * 128) + so, &tmap_k, bx * 64, r, &full[st]);
              tma_load_2d(vt + bx * (kTileKeys * 128) + so, &tmap_v, bx * 64, r, &full[st]);
            }
          }
          prow = pnext;
        }
      }
      // drain: every armed stage must land before the CTA may exit
      if (lane == 0)
        for (int j = it - kStages > 0 ? it - kStages : 0; j < it; ++j)
          mbar_wait(&full[j % kStages], (j / kStages) & 1, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int mt = warp % MT, kq = warp / MT;
  const int g = lane >> 2, t4 = lane & 3;
  int u = u0, it = 0;
  Seg s;
  bool alive = start < end;
  while (alive && next_seg(u, s)) {
    const int b = s.u / Hkv, h = s.u - b * Hkv;
    // Q fragments for rows mt*16 .. mt*16+15 of this unit (row r = head
    // (r / Nq) of the group, token r % Nq; the unit's rows are contiguous)
    uint32_t qa[D / 16][4];
    const int r0 = mt * 16 + g, r1 = r0 + 8;
    {
      const size_t qrow = ((size_t)b * a.Hq + (size_t)h * a.G) * a.Nq;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + (qrow + r0) * D);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + (qrow + r1) * D);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qa[ks][0] = r0 < a.R ? q0[ks * 8 + t4] : 0u;
        qa[ks][1] = r1 < a.R ? q1[ks * 8 + t4] : 0u;
        qa[ks][2] = r0 < a.R ? q0[ks * 8 + 4 + t4] : 0u;
        qa[ks][3] = r1 < a.R ? q1[ks * 8 + 4 + t4] : 0u;
      }
    }
    // positions of this thread's two rows; key index of segment position 0
    const int Lb = clamp_len(a.key_lens ? a.key_lens[b] : a.Nk, a.Nk);
    const int off = query_offset(a.Nq, a.Nk, Lb, a.align);
    const int pos0 = off + r0 % a.Nq, pos1 = off + r1 % a.Nq;
    const int key_base = lo_s[b];
    const bool row_masks = a.Nq > 1 || a.window > 0;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float acc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

    for (int t = first_tile(s, key_base); t < s.hi; t += kTileKeys, ++it) {
      const int st = it % kStages;
      if (!mbar_wait(&full[st], (it / kStages) & 1, abort_flag)) { alive = false; break; }
      const uint32_t kbase = smem_u32(smem + L::kRing + st * L::kStageBytes);
      const uint32_t vbase = kbase + L::kTileBytes;
      // ---- S = Q K^T for keys kq*16 .. kq*16+15 of the tile
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        // matrices: (keys +0..7, d chunk 2ks), (keys +0..7, chunk 2ks+1),
        //           (keys +8..15, chunk 2ks), (keys +8..15, chunk 2ks+1)
        const int mi = lane >> 3, r = lane & 7;
        const uint32_t key = kq * 16 + (mi >> 1) * 8 + r;
        const uint32_t chunk = 2 * ks + (mi & 1);
        const uint32_t addr = kbase + (chunk >> 3) * (kTileKeys * 128) + sw128_offset(key, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_bf16_16816(sc[0], qa[ks], b0, b1);
        mma_bf16_16816(sc[1], qa[ks], b2, b3);
      }
      // ---- mask, scale (log2 domain), online softmax
      const int kfirst = t + kq * 16;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kfirst + n * 8 + 2 * t4 + (e & 1);
          bool vis = key < s.hi && (!kPaged || key >= s.lo);
          if (row_masks) {   // causal among the new tokens, sliding window
            const int dlt = (e >> 1 ? pos1 : pos0) - (key_base + key);
            vis = vis && (!a.causal || dlt >= 0) &&
                  (a.window <= 0 || (dlt < a.window && dlt > -a.window));
          }
          const float v = vis ? sc[n][e] * a.scale_log2 : -INFINITY;
          sc[n][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      float alpha[2], mu[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float mn = fmaxf(m[r], mx[r]);
        mu[r] = mn == -INFINITY ? 0.f : mn;
        alpha[r] = exp2_approx(m[r] - mu[r]);
        m[r] = mn;
      }
      uint32_t pa[4];
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const float p0 = exp2_approx(sc[n][0] - mu[0]);
        const float p1 = exp2_approx(sc[n][1] - mu[0]);
        const float p2 = exp2_approx(sc[n][2] - mu[1]);
        const float p3 = exp2_approx(sc[n][3] - mu[1]);
        rs[0] += p0 + p1;
        rs[1] += p2 + p3;
        pa[2 * n + 0] = pack_bf16x2(p0, p1);
        pa[2 * n + 1] = pack_bf16x2(p2, p3);
      }
      l[0] = l[0] * alpha[0] + rs[0];
      l[1] = l[1] * alpha[1] + rs[1];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        acc[n][0] *= alpha[0]; acc[n][1] *= alpha[0];
        acc[n][2] *= alpha[1]; acc[n][3] *= alpha[1];
      }
      // ---- O += P V over keys kq*16 .. +15 (V rows), d in steps of 16
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        // matrices: (keys +0..7, chunk 2dn), (keys +8..15, chunk 2dn),
        //           (keys +0..7, chunk 2dn+1), (keys +8..15, chunk 2dn+1)
        const int mi = lane >> 3, r = lane & 7;
        const uint32_t key = kq * 16 + (mi & 1) * 8 + r;
        const uint32_t chunk = 2 * dn + (mi >> 1);
        const uint32_t addr = vbase + (chunk >> 3) * (kTileKeys * 128) + sw128_offset(key, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * dn], pa, b0, b1);
        mma_bf16_16816(acc[2 * dn + 1], pa, b2, b3);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- merge the four key quarters of each head tile
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
      l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
    if (t4 == 0) {
      mbuf[(kq * 4 + mt) * 16 + g] = m[0];
      mbuf[(kq * 4 + mt) * 16 + g + 8] = m[1];
    }
    // A wait that gave up ends the tile loop of its warp only; the consumer
    // warps leave together here, on a vote at the barrier (one that left
    // alone would strand the others at it).
    if (bar_vote_or(1, kConsumerThreads, !alive)) {
      alive = false;
      break;
    }
    float f[2], M[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mm = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) mm = fmaxf(mm, mbuf[(q * 4 + mt) * 16 + g + 8 * r]);
      M[r] = mm;
      f[r] = mm == -INFINITY ? 0.f : exp2_approx(m[r] - mm);
    }
    float* ob = obuf + mt * 16 * D;
    for (int q = 0; q < 4; ++q) {
      if (kq == q) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const int c = n * 8 + 2 * t4;
          float* o0 = ob + g * D + c;
          float* o1 = ob + (g + 8) * D + c;
          if (q == 0) {
            o0[0] = acc[n][0] * f[0]; o0[1] = acc[n][1] * f[0];
            o1[0] = acc[n][2] * f[1]; o1[1] = acc[n][3] * f[1];
          } else {
            o0[0] += acc[n][0] * f[0]; o0[1] += acc[n][1] * f[0];
            o1[0] += acc[n][2] * f[1]; o1[1] += acc[n][3] * f[1];
          }
        }
        if (t4 == 0) {
          if (q == 0) { lbuf[mt * 16 + g] = l[0] * f[0]; lbuf[mt * 16 + g + 8] = l[1] * f[1]; }
          else { lbuf[mt * 16 + g] += l[0] * f[0]; lbuf[mt * 16 + g + 8] += l[1] * f[1]; }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads));
    }
    // ---- write the partial of slot (blockIdx.x + unit)
    const size_t slot = (size_t)blockIdx.x + s.u;
    for (int idx = threadIdx.x; idx < MT * 16 * D; idx += kConsumerThreads) {
      const int row = idx / D, c = idx - row * D;   // row = mt*16 + r
      if (row < a.R) {
        const float lv = lbuf[row];
        a.part_o[(slot * a.R + row) * D + c] = lv > 0.f ? obuf[idx] / lv : 0.f;
      }
    }
    if (kq == 0 && t4 == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = mt * 16 + g + 8 * r;
        if (row < a.R) {
          const float lv = lbuf[row];
          a.part_lse[slot * a.R + row] = lv > 0.f ? M[r] + __log2f(lv) : -INFINITY;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads));   // obuf/mbuf reused next segment
  }
}

// Combine: one CTA per (unit, kCombineThreads / D rows), one thread per
// output element, which merges the unit's slots for its (row, d) with the
// running-max recurrence of the online softmax over the slots: lse =
// log2 sum_s 2^lse_s, O = sum_s 2^(lse_s - lse) O_s.  A row no slot saw a key
// for (masked everywhere) gets O = 0, lse = -inf.
struct CombineArgs {
  const int32_t* key_lens;
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Nk, G, grid;
  int Nq, R;
  int window, align;
  int seg_cost;
};

constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(CombineArgs a) {
  // the next decode call's split kernel may start its set-up now (it waits
  // for this grid before it touches global memory)
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ float cs[];          // int flags [ns]: slots written by this launch
  __shared__ long long s_red[2][kCombineThreads / 32];
  __shared__ long long s_pb[2];
  __shared__ int s_len;
  const int u = blockIdx.x, b = u / a.Hkv, h = u - b * a.Hkv;
  const int G = a.R;                                 // rows of a unit
  constexpr int HB = kCombineThreads / D;            // rows of this block
  const int g0 = blockIdx.y * HB;
  const int gn = (G - g0) < HB ? (G - g0) : HB;
  // unit start and total key count: block-wide sums over the key lengths
  long long before = 0, total = 0;
  for (int bb = threadIdx.x; bb < a.B; bb += blockDim.x) {
    const int Lb = clamp_len(a.key_lens ? a.key_lens[bb] : a.Nk, a.Nk);
    int lo;
    const int len = decode_key_range(Lb, query_offset(a.Nq, a.Nk, Lb, a.align), a.window, &lo);
    const int vlen = virtual_len(len, a.seg_cost);
    total += vlen;
    if (bb < b) before += vlen;
    if (bb == b) s_len = len;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if ((threadIdx.x & 31) == 0) {
    s_red[0][threadIdx.x >> 5] = before;
    s_red[1][threadIdx.x >> 5] = total;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long pb = 0, tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { pb += s_red[0][w]; tot += s_red[1][w]; }
    s_pb[0] = (long long)a.Hkv * pb + (long long)h * virtual_len(s_len, a.seg_cost) +
              (s_len > 0 ? a.seg_cost : 0);                   // the unit's first real key
    s_pb[1] = (long long)a.Hkv * tot;                         // T
  }
  __syncthreads();
  const long long p0 = s_pb[0], T = s_pb[1];
  const int len = s_len;
  // the unit's rows are contiguous in o and lse
  const size_t row0 = ((size_t)b * a.Hq + (size_t)h * a.G) * a.Nq + g0;
  __nv_bfloat16* orow = a.o + row0 * D;
  if (len == 0) {
    // o / lse may be read by earlier work in the stream only through the split
    // kernel's inputs, so writing before the dependency wait is safe
    for (int idx = threadIdx.x; idx < gn * D; idx += blockDim.x) orow[idx] = __float2bfloat16(0.f);
    if (a.lse && threadIdx.x < gn) a.lse[row0 + threadIdx.x] = -INFINITY;
    return;
  }
  // CTAs whose ranges intersect [p0, p0 + len); empty ranges wrote no slot
  auto cta_of = [&](long long x) -> int {
    long long c = (x * a.grid) / T;
    while (c + 1 < a.grid && T * (c + 1) / a.grid <= x) ++c;
    while (c > 0 && T * c / a.grid > x) --c;
    return (int)c;
  };
  const int c0 = cta_of(p0), c1 = cta_of(p0 + len - 1);
  const int ns = c1 - c0 + 1;
  auto nonempty = [&](int c) -> bool { return T * c / a.grid < T * (c + 1) / a.grid; };
  // launched as a programmatic dependent of the split kernel: everything
  // above reads only inputs; the partials are ready after this wait
  // which of the unit's slots this launch wrote (CTAs with empty key ranges
  // write none; their slots hold stale data), settled before the wait
  int* written = reinterpret_cast<int*>(cs);   // [ns]
  for (int k = threadIdx.x; k < ns; k += blockDim.x) written[k] = nonempty(c0 + k) ? 1 : 0;
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // one thread per output: the slots' log-sum-exps and partials are loaded
  // together and merged with the running-max recurrence over the slots
  for (int idx = threadIdx.x; idx < gn * D; idx += blockDim.x) {
    const int g = idx / D, c = idx - g * D;
    const float* lsrc = a.part_lse + ((size_t)c0 + u) * G + g0 + g;
    const float* osrc = a.part_o + (((size_t)c0 + u) * G + g0 + g) * D + c;
    const size_t ls = (size_t)G, os = (size_t)G * D;   // next slot
    float m = -INFINITY, acc = 0.f, sum = 0.f;
    int k = 0;
    auto merge = [&](float lk, float xk) {
      if (lk == -INFINITY) return;   // no visible key of this row in the slot
      if (lk > m) {
        const float f = m == -INFINITY ? 0.f : exp2_approx(m - lk);
        acc *= f;
        sum *= f;
        m = lk;
      }
      const float w = exp2_approx(lk - m);
      acc = fmaf(w, xk, acc);
      sum += w;
    };
    for (; k + 4 <= ns; k += 4) {
      float lk[4], xk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool wr = written[k + e] != 0;
        lk[e] = wr ? lsrc[(k + e) * ls] : -INFINITY;
        xk[e] = wr ? osrc[(k + e) * os] : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) merge(lk[e], xk[e]);
    }
    for (; k < ns; ++k)
      if (written[k]) merge(lsrc[k * ls], osrc[k * os]);
    orow[idx] = __float2bfloat16(sum > 0.f ? acc / sum : 0.f);
    if (c == 0 && a.lse) a.lse[row0 + g] = sum > 0.f ? (m + __log2f(sum)) * kLn2 : -INFINITY;
  }
}

// ------------------------------------------------------------------ host side

namespace {
template <int D, int MT, bool kPaged>
int launch_decode_t(const DecodePlan& p, const CUtensorMap& tk, const CUtensorMap& tv,
                    const DecodeArgs& a, cudaStream_t st) {
  auto kern = decode_split_kernel<D, MT, kPaged>;
  const int smem = DecodeSmem<D>::kTotal;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ATTN_ECUDA;
  return launch_programmatic(kern, dim3(p.grid), dim3((MT * 4 + 1) * 32), smem, st, tk, tv, a);
}
}  // namespace

DecodePlan decode_plan(int B, int Hq, int Hkv, int Nq, int d, int num_sms) {
  DecodePlan p;
  p.grid = num_sms;   // one CTA per SM (the ring takes most of shared memory)
  p.G = Hq / Hkv;
  p.R = p.G * Nq;
  p.slots = (size_t)p.grid + (size_t)B * Hkv;
  p.part_o_bytes = ((p.slots * p.R * d * sizeof(float)) + 255) & ~size_t(255);
  p.part_lse_bytes = ((p.slots * p.R * sizeof(float)) + 255) & ~size_t(255);
  p.workspace_bytes = p.part_o_bytes + p.part_lse_bytes;
  return p;
}

bool decode_supported(int B, int Hq, int Hkv, int Nq, int d) {
  const long long R = (long long)(Hq / Hkv) * Nq;
  return (d == 64 || d == 128) && Nq >= 1 && R >= 1 && R <= 64 && B <= kMaxScanB;
}

// Virtual keys charged to every non-empty unit in the work split: about the
// cost of starting a segment, in keys (see virtual_len in tile_plan.cuh).
constexpr int kSegCost = 320;

int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int d, const DecodeMask& mk_in, const PagedKv* pg,
                  float scale, const int32_t* key_lens, void* workspace, const DecodePlan& p,
                  cudaStream_t st) {
  DecodeMask mk = mk_in;
  // the split's key prefix is an int: keep the virtual total below 2^31
  mk.seg_cost = (long long)B * Hkv * ((long long)Nk + kSegCost) < (1ll << 31) ? kSegCost : 0;
  int rc;
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.key_lens = key_lens;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + p.part_o_bytes);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nk = Nk; a.G = p.G; a.grid = p.grid;
  a.Nq = Nq; a.R = p.R;
  a.causal = mk.causal; a.window = mk.window; a.align = mk.align;
  a.seg_cost = mk.seg_cost;
  a.scale_log2 = scale * kLog2e;
  if (d == 128) {   // decode_supported ensures the tcgen05 kernel takes it
    if (!decode_tc_supported(B, Hq, Hkv, Nq, d)) return ATTN_EUNSUPPORTED;
    rc = launch_decode_split_tc(q, k, v, B, Hq, Hkv, Nq, Nk, mk, pg, scale, key_lens, a.part_o,
                                a.part_lse, p.grid, st);
  } else {
    // contiguous: [B * Hkv * Nk, d] in 64-row boxes; paged: [num_pages * Hkv *
    // page_size, d] in page_size-row boxes
    CUtensorMap tk, tv;
    const uint64_t rows = pg ? (uint64_t)pg->num_pages * Hkv * pg->page_size
                             : (uint64_t)B * Hkv * Nk;
    const uint32_t box = pg ? (uint32_t)pg->page_size : (uint32_t)kTileKeys;
    if (make_tmap_2d_bf16(&tk, k, d, rows, 64, box) != ATTN_OK) return ATTN_ECUDA;
    if (make_tmap_2d_bf16(&tv, v, d, rows, 64, box) != ATTN_OK) return ATTN_ECUDA;
    a.block_table = pg ? pg->block_table : nullptr;
    a.max_pages = pg ? pg->max_pages : 0;
    a.page_size = pg ? pg->page_size : 0;
    a.num_pages = pg ? pg->num_pages : 0;
    a.oob_row = (int)rows;
    const int MT = (p.R + 15) / 16;
    if (pg) {
      rc = MT == 1 ? launch_decode_t<64, 1, true>(p, tk, tv, a, st)
         : MT == 2 ? launch_decode_t<64, 2, true>(p, tk, tv, a, st)
                   : launch_decode_t<64, 4, true>(p, tk, tv, a, st);
    } else {
      rc = MT == 1 ? launch_decode_t<64, 1, false>(p, tk, tv, a, st)
         : MT == 2 ? launch_decode_t<64, 2, false>(p, tk, tv, a, st)
                   : launch_decode_t<64, 4, false>(p, tk, tv, a, st);
    }
  }
  if (rc != ATTN_OK) return rc;
  CombineArgs c;
  c.key_lens = key_lens;
  c.part_o = a.part_o;
  c.part_lse = a.part_lse;
  c.o = static_cast<__nv_bfloat16*>(o);
  c.lse = lse;
  c.B = B; c.Hq = Hq; c.Hkv = Hkv; c.Nk = Nk; c.G = p.G; c.grid = p.grid;
  c.Nq = Nq; c.R = p.R;
  c.window = mk.window; c.align = mk.align;
  c.seg_cost = mk.seg_cost;
  // shared memory: the unit's slot lse's ([slots][heads of the block], at most
  // grid + 1 slots) + [heads of the block]
  const int hb = kCombineThreads / d;
  const size_t csmem = ((size_t)(p.grid + 2) * hb) * sizeof(float);
  const dim3 cgrid(B * Hkv, (p.R + hb - 1) / hb);
  // programmatic dependent launch: the combine grid may start while the
  // split kernel drains; it waits for the split's results in the kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = cgrid;
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = csmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (d == 128) {
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<128>, c) != cudaSuccess) return ATTN_ECUDA;
  } else {
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<64>, c) != cudaSuccess) return ATTN_ECUDA;
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace attn
