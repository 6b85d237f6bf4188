// kernels.h -- host-side interface between the C ABI (api.cu) and the
// kernel files.  Internal to libattn_b200.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "attn.h"

namespace attn {

// 2D bf16 tensor map over a row-major [rows, cols] matrix with a box of
// box_cols x box_rows and 128-byte swizzling (box_cols * 2 must be 128).
int make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows);

// 3D bf16 tensor map over [mats, rows, cols] (row-major) with a box of
// box_cols x box_rows x 1 and 128-byte swizzling; loads and stores clip at
// the end of each matrix.
int make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint64_t mats, uint32_t box_cols, uint32_t box_rows);

// ---- decode (Nq == 1)
struct DecodePlan {
  int grid = 0;          // CTAs of the split kernel (one wave)
  int G = 0;             // query heads per kv head
  size_t slots = 0;      // partial-result slots (grid + B*Hkv)
  size_t part_o_bytes = 0, part_lse_bytes = 0, workspace_bytes = 0;
};
DecodePlan decode_plan(int B, int Hq, int Hkv, int d, int num_sms);
bool decode_supported(int B, int Hq, int Hkv, int d);
// tcgen05 split kernel (d == 128, up to 64 query heads per kv head); writes
// the same partial-result format as the mma.sync split kernel.
bool decode_tc_supported(int B, int Hq, int Hkv, int d);
int launch_decode_split_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                           int Nk, int kv_lo, float scale, const int32_t* key_lens,
                           float* part_o, float* part_lse, int grid, cudaStream_t st);
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nk, int d, int kv_lo, float scale, const int32_t* key_lens,
                  void* workspace, const DecodePlan& p, cudaStream_t st);
// Decode reads keys [kv_lo, min(key_lens[b], Nk)) of every sequence; kv_lo is
// Nk - window (at least 0) under a sliding window of `window` keys, else 0.

// ---- prefill (Nq > 1)
bool prefill_supported(int d);
size_t prefill_workspace_bytes();   // scheduler counter
void prefill_tile_shape(int d, int* Br, int* Bc);
int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, int causal, int window, float scale,
                   const int32_t* key_lens, void* workspace, int num_sms, cudaStream_t st);
int launch_tile_plan(int B, int Nq, int Nk, int d, int causal, int window,
                     const int32_t* key_lens, int32_t* first, int32_t* count, cudaStream_t st);

// ---- RoPE
int launch_rope(const void* x_in, void* x_out, int B, int H, int N, int d, float base,
                int pos_offset, int pairing, cudaStream_t st);

}  // namespace attn
