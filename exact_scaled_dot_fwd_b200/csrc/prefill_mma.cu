// prefill_mma.cu -- tiled exact attention forward (Nq > 1) on the mma.sync
// tensor path.  Correctness baseline for the tcgen05/TMEM kernel.
//
// FlashAttention-style tiling ("Attention mechanisms ...", section 19;
// "Transformer Architecture Breakdown ...", section 4.2): a CTA owns Br = 64
// query rows of one (b, h); K/V tiles of Bc = 64 keys stream through a
// TMA-filled shared-memory ring; each of 4 consumer warps owns 16 rows and
// keeps its running max m, running sum l and unnormalised O in registers; the
// score tile never leaves the SM.  Causal / padded tiles past every row's
// visible prefix are skipped (tile_plan.cuh); only boundary tiles are masked.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tile_plan.cuh"

namespace attn {

namespace {
constexpr int kBr = 64, kBc = 64, kStages = 3;

template <int D>
struct PrefillSmem {
  static constexpr int kQBytes = kBr * D * 2;
  static constexpr int kTileBytes = kBc * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQ = 0;
  static constexpr int kRing = kQ + kQBytes;
  static constexpr int kBars = kRing + kStages * kStageBytes;  // qbar, full[S], empty[S]
  static constexpr int kAbort = kBars + (1 + 2 * kStages) * 8;
  static constexpr int kTotal = kAbort + 16 + 1024;
};
}  // namespace

struct PrefillArgs {
  __nv_bfloat16* o;
  float* lse;
  const int32_t* key_lens;
  int B, Hq, Hkv, Nq, Nk, causal, nqt;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(160, 1)
    prefill_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, PrefillArgs a) {
  using L = PrefillSmem<D>;
  constexpr int kBoxes = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* full = qbar + 1;
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  // heaviest query tiles first (causal work grows with the tile index)
  const int qt = a.causal ? (a.nqt - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv, hk = h / G;
  const int L_b = clamp_len(a.key_lens ? a.key_lens[b] : a.Nk, a.Nk);
  const KvRange kr = kv_tile_range(qt, kBr, kBc, a.Nq, a.Nk, a.causal, L_b);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qbar, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int qrow = (b * a.Hq + h) * a.Nq + qt * kBr;
      const int krow = (b * a.Hkv + hk) * a.Nk;
      mbar_arrive_expect_tx(qbar, L::kQBytes);
      for (int bx = 0; bx < kBoxes; ++bx)
        tma_load_2d(smem + L::kQ + bx * kBr * 128, &tq, bx * 64, qrow, qbar);
      int it = 0;
      for (; it < kr.count; ++it) {
        const int st = it % kStages;
        if (!mbar_wait(&empty[st], ((it / kStages) & 1) ^ 1, abort_flag)) break;
        uint8_t* kt = smem + L::kRing + st * L::kStageBytes;
        uint8_t* vt = kt + L::kTileBytes;
        mbar_arrive_expect_tx(&full[st], L::kStageBytes);
        for (int bx = 0; bx < kBoxes; ++bx) {
          tma_load_2d(kt + bx * kBc * 128, &tk, bx * 64, krow + it * kBc, &full[st]);
          tma_load_2d(vt + bx * kBc * 128, &tv, bx * 64, krow + it * kBc, &full[st]);
        }
      }
      mbar_wait(qbar, 0, nullptr);
      for (int j = it - kStages > 0 ? it - kStages : 0; j < it; ++j)
        mbar_wait(&full[j % kStages], (j / kStages) & 1, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, t4 = lane & 3;
  const int r0 = qt * kBr + warp * 16 + g, r1 = r0 + 8;
  const int n0 = visible_prefix(r0, a.Nq, a.Nk, a.causal, L_b);
  const int n1 = visible_prefix(r1, a.Nq, a.Nk, a.causal, L_b);

  if (!mbar_wait(qbar, 0, abort_flag)) return;
  uint32_t qa[D / 16][4];
  {
    const uint32_t qbase = smem_u32(smem + L::kQ);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      // A 16x16: (rows +0..7, chunk 2ks), (rows +8..15, 2ks), (rows +0..7, 2ks+1), (rows +8..15, 2ks+1)
      const int mi = lane >> 3, r = lane & 7;
      const uint32_t row = warp * 16 + (mi & 1) * 8 + r;
      const uint32_t chunk = 2 * ks + (mi >> 1);
      ldsm_x4(qbase + (chunk >> 3) * (kBr * 128) + sw128_offset(row, chunk & 7), qa[ks][0], qa[ks][1],
              qa[ks][2], qa[ks][3]);
    }
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  for (int it = 0; it < kr.count; ++it) {
    const int st = it % kStages;
    if (!mbar_wait(&full[st], (it / kStages) & 1, abort_flag)) break;
    const uint32_t kbase = smem_u32(smem + L::kRing + st * L::kStageBytes);
    const uint32_t vbase = kbase + L::kTileBytes;
    float sc[kBc / 8][4];
#pragma unroll
    for (int n = 0; n < kBc / 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < kBc / 16; ++np) {
        const int mi = lane >> 3, r = lane & 7;
        const uint32_t key = np * 16 + (mi >> 1) * 8 + r;
        const uint32_t chunk = 2 * ks + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + (chunk >> 3) * (kBc * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
        mma_bf16_16816(sc[2 * np], qa[ks], b0, b1);
        mma_bf16_16816(sc[2 * np + 1], qa[ks], b2, b3);
      }
    }
    float mx[2] = {-INFINITY, -INFINITY};
    const bool masked = it >= kr.first_masked;
#pragma unroll
    for (int n = 0; n < kBc / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = sc[n][e] * a.scale_log2;
        if (masked) {
          const int key = it * kBc + n * 8 + 2 * t4 + (e & 1);
          if (key >= ((e >> 1) ? n1 : n0)) v = -INFINITY;
        }
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
    float rs[2] = {0.f, 0.f};
    uint32_t pa[kBc / 16][4];
#pragma unroll
    for (int n = 0; n < kBc / 8; ++n) {
      const float p0 = exp2_approx(sc[n][0] - mu[0]);
      const float p1 = exp2_approx(sc[n][1] - mu[0]);
      const float p2 = exp2_approx(sc[n][2] - mu[1]);
      const float p3 = exp2_approx(sc[n][3] - mu[1]);
      rs[0] += p0 + p1;
      rs[1] += p2 + p3;
      pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l[0] = l[0] * alpha[0] + rs[0];
    l[1] = l[1] * alpha[1] + rs[1];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= alpha[0]; acc[n][1] *= alpha[0];
      acc[n][2] *= alpha[1]; acc[n][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < kBc / 16; ++kk) {
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        const int mi = lane >> 3, r = lane & 7;
        const uint32_t key = kk * 16 + (mi & 1) * 8 + r;
        const uint32_t chunk = 2 * dn + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + (chunk >> 3) * (kBc * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * dn], pa[kk], b0, b1);
        mma_bf16_16816(acc[2 * dn + 1], pa[kk], b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- epilogue: O = acc / l (bf16), lse = (m + log2 l) * ln 2
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
  const float inv0 = l[0] > 0.f ? 1.f / l[0] : 0.f;
  const float inv1 = l[1] > 0.f ? 1.f / l[1] : 0.f;
  const size_t obase = ((size_t)b * a.Hq + h) * a.Nq;
  if (r0 < a.Nq) {
    uint32_t* o0 = reinterpret_cast<uint32_t*>(a.o + (obase + r0) * D);
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o0[n * 4 + t4] = pack_bf16x2(acc[n][0] * inv0, acc[n][1] * inv0);
    if (a.lse && t4 == 0) a.lse[obase + r0] = l[0] > 0.f ? (m[0] + __log2f(l[0])) * kLn2 : -INFINITY;
  }
  if (r1 < a.Nq) {
    uint32_t* o1 = reinterpret_cast<uint32_t*>(a.o + (obase + r1) * D);
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o1[n * 4 + t4] = pack_bf16x2(acc[n][2] * inv1, acc[n][3] * inv1);
    if (a.lse && t4 == 0) a.lse[obase + r1] = l[1] > 0.f ? (m[1] + __log2f(l[1])) * kLn2 : -INFINITY;
  }
}

__global__ void tile_plan_kernel(const int32_t* key_lens, int B, int Nq, int Nk, int causal, int Br,
                                 int Bc, int nqt, int32_t* first, int32_t* count) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * nqt) return;
  const int b = idx / nqt, qt = idx - b * nqt;
  const int L_b = clamp_len(key_lens ? key_lens[b] : Nk, Nk);
  const KvRange r = kv_tile_range(qt, Br, Bc, Nq, Nk, causal, L_b);
  first[idx] = r.count > 0 ? 0 : -1;
  count[idx] = r.count;
}

bool prefill_supported(int d) { return d == 64 || d == 128; }

void prefill_tile_shape(int d, int* Br, int* Bc) {
  (void)d;
  *Br = kBr;
  *Bc = kBc;
}

int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, int causal, float scale,
                   const int32_t* key_lens, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (make_tmap_2d_bf16(&tq, q, d, (uint64_t)B * Hq * Nq, 64, kBr) != ATTN_OK) return ATTN_ECUDA;
  if (make_tmap_2d_bf16(&tk, k, d, (uint64_t)B * Hkv * Nk, 64, kBc) != ATTN_OK) return ATTN_ECUDA;
  if (make_tmap_2d_bf16(&tv, v, d, (uint64_t)B * Hkv * Nk, 64, kBc) != ATTN_OK) return ATTN_ECUDA;
  PrefillArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.key_lens = key_lens;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.causal = causal;
  a.nqt = (Nq + kBr - 1) / kBr;
  a.scale_log2 = scale * kLog2e;
  dim3 grid(a.nqt, Hq, B);
  if (d == 128) {
    auto kern = prefill_mma_kernel<128>;
    const int smem = PrefillSmem<128>::kTotal;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ATTN_ECUDA;
    kern<<<grid, 160, smem, st>>>(tq, tk, tv, a);
  } else {
    auto kern = prefill_mma_kernel<64>;
    const int smem = PrefillSmem<64>::kTotal;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ATTN_ECUDA;
    kern<<<grid, 160, smem, st>>>(tq, tk, tv, a);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

int launch_tile_plan(int B, int Nq, int Nk, int d, int causal, const int32_t* key_lens,
                     int32_t* first, int32_t* count, cudaStream_t st) {
  int Br, Bc;
  prefill_tile_shape(d, &Br, &Bc);
  const int nqt = (Nq + Br - 1) / Br;
  const int n = B * nqt;
  if (n == 0) return ATTN_OK;
  tile_plan_kernel<<<(n + 255) / 256, 256, 0, st>>>(key_lens, B, Nq, Nk, causal, Br, Bc, nqt, first,
                                                    count);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace attn
