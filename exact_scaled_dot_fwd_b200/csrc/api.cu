// api.cu -- the C ABI of libattn_b200.so: argument checks, dispatch, the
// library-owned decode workspace, TMA descriptor encoding and the device
// status word.  Declarations and contracts are in include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>

#include "attn.h"
#include "common.cuh"
#include "kernels.h"

namespace attn {

__device__ int g_device_status = 0;

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// attn_fwd's workspace, one per device: the library's own (grown on demand)
// unless the caller registered a buffer of its own with attn_set_workspace.
// A buffer that is outgrown is retired, not freed: work already queued on
// some stream (or launched by another host thread that read the old pointer)
// may still use it, and freeing it would need a device-wide synchronisation.
// Retired buffers are released at process exit with the current one.
struct OwnedWorkspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  void* user = nullptr;     // caller-owned, never freed here
  size_t user_bytes = 0;
};
constexpr int kMaxDevices = 64;
OwnedWorkspace g_ws[kMaxDevices];
std::vector<void*> g_retired;
std::mutex g_ws_mu;

struct WorkspaceReaper {
  ~WorkspaceReaper() {
    // process exit: the CUDA driver may already be tearing down; ignore errors
    for (auto& w : g_ws)
      if (w.ptr) cudaFree(w.ptr);
    for (void* p : g_retired) cudaFree(p);
  }
} g_reaper;

int check_common(const void* q, const void* k, const void* v, const void* o, int B, int Hq, int Hkv,
                 int Nq, int Nk, int d, int causal, float scale) {
  if (!q || !k || !v || !o) return ATTN_EINVAL;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return ATTN_EINVAL;
  if (Hq % Hkv != 0) return ATTN_EINVAL;
  if (causal != 0 && causal != 1) return ATTN_EINVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_EINVAL;
  if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
  if ((long long)B * Hq * Nq >= (1ll << 31) || (long long)B * Hkv * Nk >= (1ll << 31))
    return ATTN_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_EALIGN;
  return ATTN_OK;
}

}  // namespace

int make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ATTN_ECUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ECUDA;
}

int make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                      uint64_t mats, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ATTN_ECUDA;
  cuuint64_t dims[3] = {cols, rows, mats};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ECUDA;
}

int make_tmap_grouped_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                           uint32_t box_groups) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows % 8 != 0) return ATTN_ECUDA;
  // (64 columns, 8 rows, 2 halves, rows / 8 groups); a row is 256 bytes
  cuuint64_t dims[4] = {64, 8, 2, rows / 8};
  cuuint64_t strides[3] = {256, 128, 2048};
  cuuint32_t box[4] = {64, 8, 2, box_groups};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ECUDA;
}

// Failure-detection hook: one thread waits on an mbarrier that nothing ever
// arrives on, with a short limit; the wait gives up, records ATTN_ETIMEOUT and
// the kernel returns.  No fault, no hang.
__global__ void timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_for(&bar, 0, nullptr, limit_ns);
  }
}

}  // namespace attn

using namespace attn;

extern "C" {

int attn_abi_version(void) { return ATTN_ABI_VERSION; }

const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_EINVAL: return "ATTN_EINVAL: invalid argument";
    case ATTN_EUNSUPPORTED: return "ATTN_EUNSUPPORTED: shape not supported by this library";
    case ATTN_EALIGN: return "ATTN_EALIGN: pointer not 16-byte aligned";
    case ATTN_EWORKSPACE: return "ATTN_EWORKSPACE: workspace missing or too small";
    case ATTN_ECUDA: return "ATTN_ECUDA: CUDA call failed";
    case ATTN_ETIMEOUT: return "ATTN_ETIMEOUT: a kernel gave up waiting on a barrier";
    case ATTN_ERANGE: return "ATTN_ERANGE: a kernel met an out-of-range block-table entry";
    default: return "unknown attn status";
  }
}

size_t attn_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  (void)Nk;
  if (Nq <= 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return 0;
  // the decode kernels take every call with at most 64 query rows per kv head
  if (!decode_supported(B, Hq, Hkv, Nq, d)) return prefill_workspace_bytes();
  const int sms = current_sms();
  if (sms <= 0) return 0;
  return decode_plan(B, Hq, Hkv, Nq, d, sms).workspace_bytes;
}

int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int d, int causal, int window, int align, float scale,
                const int32_t* key_lens, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(q, k, v, o, B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != ATTN_OK) return rc;
  if (window < 0 || (align != 0 && align != 1)) return ATTN_EINVAL;
  if (lse && !aligned16(lse)) return ATTN_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (decode_supported(B, Hq, Hkv, Nq, d)) {
    const int sms = current_sms();
    if (sms <= 0) return ATTN_ECUDA;
    const DecodePlan p = decode_plan(B, Hq, Hkv, Nq, d, sms);
    if (!workspace || workspace_bytes < p.workspace_bytes) return ATTN_EWORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_EALIGN;
    DecodeMask mk;
    mk.causal = causal;
    mk.window = window;
    mk.align = align;
    return launch_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, mk, nullptr, scale, key_lens,
                         workspace, p, st);
  }
  if (!prefill_supported(d)) return ATTN_EUNSUPPORTED;
  if (!workspace || workspace_bytes < prefill_workspace_bytes()) return ATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_EALIGN;
  const int sms = current_sms();
  if (sms <= 0) return ATTN_ECUDA;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, window, align, scale,
                        key_lens, nullptr, 0, workspace, sms, st);
}

int attn_fwd_trace(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int Hq, int Hkv, int Nq, int Nk, int d, int causal, int window, int align,
                   float scale, const int32_t* key_lens, void* workspace, size_t workspace_bytes,
                   int32_t* trace, void* stream) {
  if (!trace) return ATTN_EINVAL;
  int rc = check_common(q, k, v, o, B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != ATTN_OK) return rc;
  if (window < 0 || (align != 0 && align != 1)) return ATTN_EINVAL;
  if (decode_supported(B, Hq, Hkv, Nq, d)) return ATTN_EUNSUPPORTED;   // prefill kernel only
  if (lse && !aligned16(lse)) return ATTN_EALIGN;
  if (!workspace || workspace_bytes < prefill_workspace_bytes()) return ATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_EALIGN;
  const int sms = current_sms();
  if (sms <= 0) return ATTN_ECUDA;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, window, align, scale,
                        key_lens, nullptr, 0, workspace, sms, static_cast<cudaStream_t>(stream),
                        trace);
}

size_t attn_rope_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  const size_t base = attn_workspace_size(B, Hq, Hkv, Nq, Nk, d);
  if (base == 0 || d <= 0) return 0;
  // decode shapes: the rotated q; prefill: the (cos, sin) table of the rows
  const size_t extra = decode_supported(B, Hq, Hkv, Nq, d)
                           ? (size_t)B * Hq * Nq * d * 2
                           : (size_t)Nq * (d / 2) * sizeof(float2);
  return ((base + 255) & ~size_t(255)) + ((extra + 255) & ~size_t(255));
}

int attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                  const int32_t* key_lens, float rope_base, int rope_pairing, int q_pos_offset,
                  void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(q, k, v, o, B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != ATTN_OK) return rc;
  if (!std::isfinite(rope_base) || !(rope_base > 0.f)) return ATTN_EINVAL;
  if (rope_pairing != 0 && rope_pairing != 1) return ATTN_EINVAL;
  if (q_pos_offset < 0 || (long long)q_pos_offset + Nq > (1ll << 31) - 1) return ATTN_EINVAL;
  if (lse && !aligned16(lse)) return ATTN_EALIGN;
  const size_t need = attn_rope_workspace_size(B, Hq, Hkv, Nq, Nk, d);
  if (need == 0) return ATTN_ECUDA;
  if (!workspace || workspace_bytes < need) return ATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_EALIGN;
  const size_t base = (attn_workspace_size(B, Hq, Hkv, Nq, Nk, d) + 255) & ~size_t(255);
  void* extra = static_cast<uint8_t*>(workspace) + base;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (decode_supported(B, Hq, Hkv, Nq, d)) {
    // decode shapes: rotate q into the workspace, then the decode kernels
    rc = launch_rope(q, extra, B, Hq, Nq, d, rope_base, q_pos_offset, rope_pairing, st);
    if (rc != ATTN_OK) return rc;
    return attn_fwd_ws(extra, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, key_lens,
                       workspace, base, stream);
  }
  if (!prefill_supported(d)) return ATTN_EUNSUPPORTED;
  const int sms = current_sms();
  if (sms <= 0) return ATTN_ECUDA;
  float2* tab = static_cast<float2*>(extra);
  rc = launch_rope_table(tab, Nq, d, rope_base, q_pos_offset, st);
  if (rc != ATTN_OK) return rc;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, 0, 0, scale, key_lens,
                        tab, rope_pairing, workspace, sms, st);
}

int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, int max_pages, int page_size, int num_pages,
                   void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d, int causal,
                   int window, float scale, const int32_t* key_lens, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!block_table || !key_lens) return ATTN_EINVAL;
  if (max_pages <= 0 || num_pages <= 0 || page_size <= 0) return ATTN_EINVAL;
  if ((long long)max_pages * page_size >= (1ll << 31)) return ATTN_EUNSUPPORTED;
  const int Nk = max_pages * page_size;   // logical capacity of a sequence
  int rc = check_common(q, k_cache, v_cache, o, B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != ATTN_OK) return rc;
  if (window < 0) return ATTN_EINVAL;
  // whole pages per tile (128 keys for d = 128, 64 for d = 64), 1 KB-aligned boxes
  const int tile = d == 128 ? 128 : 64;
  if (page_size % 8 != 0 || tile % page_size != 0) return ATTN_EUNSUPPORTED;
  if ((long long)num_pages * Hkv * page_size >= (1ll << 31)) return ATTN_EUNSUPPORTED;
  if (!decode_supported(B, Hq, Hkv, Nq, d)) return ATTN_EUNSUPPORTED;
  if (lse && !aligned16(lse)) return ATTN_EALIGN;
  const int sms = current_sms();
  if (sms <= 0) return ATTN_ECUDA;
  const DecodePlan p = decode_plan(B, Hq, Hkv, Nq, d, sms);
  if (!workspace || workspace_bytes < p.workspace_bytes) return ATTN_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_EALIGN;
  DecodeMask mk;
  mk.causal = causal;
  mk.window = window;
  mk.align = 1;   // each sequence's query rows are its newest tokens
  PagedKv pg;
  pg.block_table = block_table;
  pg.max_pages = max_pages;
  pg.page_size = page_size;
  pg.num_pages = num_pages;
  return launch_decode(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nq, Nk, d, mk, &pg, scale,
                       key_lens, workspace, p, static_cast<cudaStream_t>(stream));
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, int causal, int window, float scale,
                    const int32_t* key_lens, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, window, 0, scale, key_lens,
                     workspace, workspace_bytes, stream);
}

int attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int d, int causal, float scale, const int32_t* key_lens,
                void* workspace, size_t workspace_bytes, void* stream) {
  return attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, 0, 0, scale, key_lens,
                     workspace, workspace_bytes, stream);
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, int causal, float scale, const int32_t* key_lens,
             void* stream) {
  int rc = check_common(q, k, v, o, B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != ATTN_OK) return rc;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  {
    if (!prefill_supported(d)) return ATTN_EUNSUPPORTED;
    const size_t need = attn_workspace_size(B, Hq, Hkv, Nq, Nk, d);
    if (need == 0) return ATTN_ECUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ECUDA;
    std::lock_guard<std::mutex> lock(g_ws_mu);
    OwnedWorkspace& w = g_ws[dev];
    if (w.user) {
      // a registered buffer is never replaced behind the caller's back
      if (w.user_bytes < need) return ATTN_EWORKSPACE;
      ws = w.user;
      ws_bytes = w.user_bytes;
    } else if (w.bytes < need) {
      void* p = nullptr;
      if (cudaMalloc(&p, need) != cudaSuccess) return ATTN_ECUDA;
      if (w.ptr) g_retired.push_back(w.ptr);
      w.ptr = p;
      w.bytes = need;
    }
    if (!w.user) {
      ws = w.ptr;
      ws_bytes = w.bytes;
    }
  }
  return attn_fwd_ws(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, key_lens, ws, ws_bytes,
                     stream);
}

int rope_apply(const void* x_in, void* x_out, int B, int H, int N, int d, float base,
               int pos_offset, int pairing, void* stream) {
  if (!x_in || !x_out) return ATTN_EINVAL;
  if (B <= 0 || H <= 0 || N <= 0 || d < 2 || d % 2 != 0) return ATTN_EINVAL;
  if (!std::isfinite(base) || !(base > 0.f)) return ATTN_EINVAL;
  if (pairing != 0 && pairing != 1) return ATTN_EINVAL;
  if (pos_offset < 0) return ATTN_EINVAL;
  if (d > 256) return ATTN_EUNSUPPORTED;
  if ((long long)pos_offset + N > (1ll << 31) - 1) return ATTN_EINVAL;
  if ((long long)B * H > 65535ll * 16) return ATTN_EUNSUPPORTED;
  if (!aligned16(x_in) || !aligned16(x_out)) return ATTN_EALIGN;
  const size_t bytes = (size_t)B * H * N * d * 2;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(x_in), b0 = reinterpret_cast<uintptr_t>(x_out);
  if (a0 != b0 && a0 < b0 + bytes && b0 < a0 + bytes) return ATTN_EINVAL;   // partial overlap
  return launch_rope(x_in, x_out, B, H, N, d, base, pos_offset, pairing,
                     static_cast<cudaStream_t>(stream));
}

int attn_prefill_tile_shape(int d, int* Br, int* Bc) {
  if (!Br || !Bc) return ATTN_EINVAL;
  if (!prefill_supported(d)) return ATTN_EUNSUPPORTED;
  prefill_tile_shape(d, Br, Bc);
  return ATTN_OK;
}

int attn_fwd_tile_plan_ex(int B, int Nq, int Nk, int d, int causal, int window, int align,
                          const int32_t* key_lens, int32_t* first, int32_t* count,
                          void* stream) {
  if (!first || !count) return ATTN_EINVAL;
  if (B <= 0 || Nq <= 0 || Nk <= 0 || (causal != 0 && causal != 1) || window < 0 ||
      (align != 0 && align != 1))
    return ATTN_EINVAL;
  if (!prefill_supported(d)) return ATTN_EUNSUPPORTED;
  return launch_tile_plan(B, Nq, Nk, d, causal, window, align, key_lens, first, count,
                          static_cast<cudaStream_t>(stream));
}

int attn_fwd_tile_plan_window(int B, int Nq, int Nk, int d, int causal, int window,
                              const int32_t* key_lens, int32_t* first, int32_t* count,
                              void* stream) {
  return attn_fwd_tile_plan_ex(B, Nq, Nk, d, causal, window, 0, key_lens, first, count, stream);
}

int attn_fwd_tile_plan(int B, int Nq, int Nk, int d, int causal, const int32_t* key_lens,
                       int32_t* first, int32_t* count, void* stream) {
  return attn_fwd_tile_plan_window(B, Nq, Nk, d, causal, 0, key_lens, first, count, stream);
}

int attn_debug_timeout_probe(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return ATTN_EINVAL;
  timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

int attn_last_device_status(void* stream) { return attn_device_status(stream, 1); }

int attn_set_workspace(void* ptr, size_t bytes) {
  if ((ptr == nullptr) != (bytes == 0)) return ATTN_EINVAL;
  if ((reinterpret_cast<uintptr_t>(ptr) & 255u) != 0) return ATTN_EALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ECUDA;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  g_ws[dev].user = ptr;
  g_ws[dev].user_bytes = bytes;
  return ATTN_OK;
}

int attn_device_status(void* stream, int reset) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return ATTN_ECUDA;
  if (reset) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_device_status, &z, sizeof z) != cudaSuccess) return ATTN_ECUDA;
  }
  return v == 0 ? ATTN_OK : v;
}

}  // extern "C"
