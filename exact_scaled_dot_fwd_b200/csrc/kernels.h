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

// 4D bf16 tensor map over a row-major [rows, 128] matrix (rows % 8 == 0)
// seen as groups of 8 rows: a box of box_groups groups lands in shared memory
// group after group, each as [64-column half 0 | half 1] of 8 rows x 128 B,
// 128-byte swizzled.  One box thus covers whole rows (both halves) while each
// half keeps a uniform 2 KB stride between its 8-row groups.
int make_tmap_grouped_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                           uint32_t box_groups);

// Launch `kern` as a programmatic dependent of the previous kernel in the
// stream (cudaLaunchAttributeProgrammaticStreamSerialization): it may start
// once that kernel has called griddepcontrol.launch_dependents (or ended) and
// must execute griddepcontrol.wait before it touches global memory.
template <typename... P, typename... A>
int launch_programmatic(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<A&&>(args)...) != cudaSuccess) return ATTN_ECUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

// ---- decode (R = (Hq / Hkv) * Nq <= 64 query rows per kv head)
struct DecodePlan {
  int grid = 0;          // CTAs of the split kernel (one wave)
  int G = 0;             // query heads per kv head
  int R = 0;             // query rows per kv head (G * Nq)
  size_t slots = 0;      // partial-result slots (grid + B*Hkv)
  size_t part_o_bytes = 0, part_lse_bytes = 0, workspace_bytes = 0;
};
// Mask of a decode call: causal among the Nq rows, sliding window, query
// alignment (0: rows end at key Nk - 1; 1: at key key_lens[b] - 1).
struct DecodeMask {
  int causal = 0, window = 0, align = 0;
  // virtual keys charged to every non-empty unit in the work split (see
  // virtual_len in tile_plan.cuh); set by launch_decode
  int seg_cost = 0;
};
// Paged KV cache: cache [num_pages, Hkv, page_size, d]; key j of sequence b
// is row j % page_size of block block_table[b * max_pages + j / page_size].
struct PagedKv {
  const int32_t* block_table = nullptr;
  int max_pages = 0, page_size = 0, num_pages = 0;
};
DecodePlan decode_plan(int B, int Hq, int Hkv, int Nq, int d, int num_sms);
bool decode_supported(int B, int Hq, int Hkv, int Nq, int d);
// tcgen05 split kernel (d == 128, up to 64 query rows per kv head); writes
// the same partial-result format as the mma.sync split kernel.
bool decode_tc_supported(int B, int Hq, int Hkv, int Nq, int d);
int launch_decode_split_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                           int Nq, int Nk, const DecodeMask& mk, const PagedKv* pg, float scale,
                           const int32_t* key_lens, float* part_o, float* part_lse, int grid,
                           cudaStream_t st);
// Each sequence's units read keys [lo, L) (decode_key_range in tile_plan.cuh).
// pg == nullptr: contiguous k/v [B, Hkv, Nk, d]; else a paged cache with
// Nk = max_pages * page_size.
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int d, const DecodeMask& mk, const PagedKv* pg,
                  float scale, const int32_t* key_lens, void* workspace, const DecodePlan& p,
                  cudaStream_t st);

// ---- prefill (Nq > 1)
bool prefill_supported(int d);
size_t prefill_workspace_bytes();   // scheduler counter
void prefill_tile_shape(int d, int* Br, int* Bc);
// trace (test hook, may be null): int32 [B * Hq * ceil(Nq / 128)][3], per query
// tile {first, last, count} of the KV tiles whose scores the kernel computes;
// tiles it computes none for are left as they are.
int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, int causal, int window, int align,
                   float scale, const int32_t* key_lens, const float2* rope_tab,
                   int rope_pairing, void* workspace, int num_sms, cudaStream_t st,
                   int32_t* trace = nullptr);
int launch_tile_plan(int B, int Nq, int Nk, int d, int causal, int window, int align,
                     const int32_t* key_lens, int32_t* first, int32_t* count, cudaStream_t st);

// ---- RoPE
int launch_rope(const void* x_in, void* x_out, int B, int H, int N, int d, float base,
                int pos_offset, int pairing, cudaStream_t st);
// (cos, sin) of positions pos_offset .. pos_offset + N - 1: tab[t * d/2 + i]
int launch_rope_table(float2* tab, int N, int d, float base, int pos_offset, cudaStream_t st);

}  // namespace attn
