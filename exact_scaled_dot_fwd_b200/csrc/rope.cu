// rope.cu -- RoPE prologue kernel.
//
// Rotates every pair of a row at position t by the angle t * theta_i,
// theta_i = base^(-2i/d) ("Transformer Architecture Breakdown ...", section
// 3.1: 2x2 rotation blocks, counter-clockwise; "Coding interview (14)",
// section 3.5: frequencies and the two pairing conventions).
//
// Memory-bound elementwise pass.  A CTA owns kPos consecutive positions for a
// slab of (b, h) rows: it first builds the cos/sin of those positions in
// shared memory (angle formed and reduced in fp64, stored fp32), then streams
// the rows with 16-byte vector loads and stores.  The angle table is built
// once per CTA and reused by every head of the slab, so the fp64 work is
// negligible against the row traffic.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "rope_math.cuh"

namespace attn {

namespace {
constexpr int kPos = 32;        // positions per CTA
constexpr int kHeads = 16;      // (b, h) rows per CTA slab
constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
}  // namespace

struct RopeArgs {
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  int BH, N, d, pos_offset, pairing;
  double base;
};

// Vector path: d % 16 == 0.  Each work item is one 16-byte chunk of a row
// (adjacent pairing: 4 pairs) or two chunks (half pairing: chunk c of the
// first half and chunk c of the second half, 8 pairs).
__global__ void __launch_bounds__(kThreads) rope_kernel(RopeArgs a) {
  extern __shared__ float tab[];   // [kPos][d/2] cos, then [kPos][d/2] sin
  const int half = a.d / 2;
  const int t0 = blockIdx.x * kPos;
  const int npos = (a.N - t0) < kPos ? (a.N - t0) : kPos;
  float* cs = tab;
  float* sn = tab + kPos * half;
  for (int idx = threadIdx.x; idx < npos * half; idx += blockDim.x) {
    const int p = idx / half, i = idx - p * half;
    const float2 c = rope_cos_sin((long long)a.pos_offset + t0 + p, i, a.d, a.base);
    cs[idx] = c.x;
    sn[idx] = c.y;
  }
  __syncthreads();

  const int bh0 = blockIdx.y * kHeads;
  const int nbh = (a.BH - bh0) < kHeads ? (a.BH - bh0) : kHeads;
  const int chunks = a.pairing ? a.d / 8 : a.d / 16;   // work items per row
  const int items = nbh * npos * chunks;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int c = it % chunks;
    const int p = (it / chunks) % npos;
    const int r = it / (chunks * npos);
    const size_t row = ((size_t)(bh0 + r) * a.N + t0 + p) * a.d;
    const float* cp = cs + p * half;
    const float* sp = sn + p * half;
    if (a.pairing) {
      // adjacent pairs (2i, 2i+1), i = 4c .. 4c+3
      const uint4 v = *reinterpret_cast<const uint4*>(a.x + row + 8 * c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 4 * c + k;
        const float x0 = bf16_lo(w[k]), x1 = bf16_hi(w[k]);
        float r0, r1;
        rope_rotate(x0, x1, make_float2(cp[i], sp[i]), r0, r1);
        o[k] = pack_bf16x2(r0, r1);
      }
      *reinterpret_cast<uint4*>(a.y + row + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      // half-split pairs (i, i + d/2), i = 8c .. 8c+7
      const uint4 va = *reinterpret_cast<const uint4*>(a.x + row + 8 * c);
      const uint4 vb = *reinterpret_cast<const uint4*>(a.x + row + half + 8 * c);
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
      const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 8 * c + 2 * k;
        const float a0 = bf16_lo(wa[k]), a1 = bf16_hi(wa[k]);
        const float b0 = bf16_lo(wb[k]), b1 = bf16_hi(wb[k]);
        float ra0, rb0, ra1, rb1;
        rope_rotate(a0, b0, make_float2(cp[i], sp[i]), ra0, rb0);
        rope_rotate(a1, b1, make_float2(cp[i + 1], sp[i + 1]), ra1, rb1);
        oa[k] = pack_bf16x2(ra0, ra1);
        ob[k] = pack_bf16x2(rb0, rb1);
      }
      *reinterpret_cast<uint4*>(a.y + row + 8 * c) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
      *reinterpret_cast<uint4*>(a.y + row + half + 8 * c) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
  }
}

// Scalar path for any even d (d % 16 != 0): one pair per work item.
__global__ void __launch_bounds__(kThreads) rope_kernel_scalar(RopeArgs a) {
  extern __shared__ float tab[];
  const int half = a.d / 2;
  const int t0 = blockIdx.x * kPos;
  const int npos = (a.N - t0) < kPos ? (a.N - t0) : kPos;
  float* cs = tab;
  float* sn = tab + kPos * half;
  for (int idx = threadIdx.x; idx < npos * half; idx += blockDim.x) {
    const int p = idx / half, i = idx - p * half;
    const float2 c = rope_cos_sin((long long)a.pos_offset + t0 + p, i, a.d, a.base);
    cs[idx] = c.x;
    sn[idx] = c.y;
  }
  __syncthreads();
  const int bh0 = blockIdx.y * kHeads;
  const int nbh = (a.BH - bh0) < kHeads ? (a.BH - bh0) : kHeads;
  const int items = nbh * npos * half;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int i = it % half;
    const int p = (it / half) % npos;
    const int r = it / (half * npos);
    const size_t row = ((size_t)(bh0 + r) * a.N + t0 + p) * a.d;
    const int ia = a.pairing ? 2 * i : i;
    const int ib = a.pairing ? 2 * i + 1 : i + half;
    const float x0 = __bfloat162float(a.x[row + ia]);
    const float x1 = __bfloat162float(a.x[row + ib]);
    float r0, r1;
    rope_rotate(x0, x1, make_float2(cs[p * half + i], sn[p * half + i]), r0, r1);
    a.y[row + ia] = __float2bfloat16_rn(r0);
    a.y[row + ib] = __float2bfloat16_rn(r1);
  }
}

// (cos, sin) table for positions pos_offset .. pos_offset + N - 1: tab[t * d/2 + i].
__global__ void rope_table_kernel(float2* tab, int N, int d, double base, int pos_offset) {
  const int half = d / 2;
  const long long n = (long long)N * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(idx / half), i = (int)(idx - (long long)t * half);
    tab[idx] = rope_cos_sin((long long)pos_offset + t, i, d, base);
  }
}

int launch_rope_table(float2* tab, int N, int d, float base, int pos_offset, cudaStream_t st) {
  const long long n = (long long)N * (d / 2);
  if (n == 0) return ATTN_OK;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  rope_table_kernel<<<blocks, 256, 0, st>>>(tab, N, d, (double)base, pos_offset);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

int launch_rope(const void* x_in, void* x_out, int B, int H, int N, int d, float base,
                int pos_offset, int pairing, cudaStream_t st) {
  if (B * (long long)H * N == 0) return ATTN_OK;
  RopeArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x_in);
  a.y = static_cast<__nv_bfloat16*>(x_out);
  a.BH = B * H; a.N = N; a.d = d; a.pos_offset = pos_offset; a.pairing = pairing;
  a.base = (double)base;
  dim3 grid((N + kPos - 1) / kPos, (a.BH + kHeads - 1) / kHeads);
  const size_t smem = 2 * kPos * (d / 2) * sizeof(float);
  if (d % 16 == 0) rope_kernel<<<grid, kThreads, smem, st>>>(a);
  else rope_kernel_scalar<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace attn
