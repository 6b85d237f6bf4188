// decode_static.cu -- decode (Nq == 1) that allocates nothing.
//
// Some callers cannot call cudaMalloc: code that runs under a fixed,
// preallocated memory budget (a serving loop that owns all device memory up
// front), code running inside an allocator hook or another runtime's
// callback, or latency-critical paths where cudaMalloc's implicit device
// synchronisation is not acceptable.  attn_fwd_decode_static gives them the
// split-KV decode with its scratch (the per-split partial outputs and their
// log-sum-exps) taken from a file-scope device array instead of a workspace:
//   - the array is kDecodeStaticScratchBytes (8 MiB), allocated when the
//     library is loaded and held on every GPU that loads it until exit;
//   - sizes whose partials do not fit are rejected with ATTN_EWORKSPACE;
//   - every call shares the array and keeps the last call's contents, so
//     calls that overlap on the GPU (different streams, different threads)
//     race: serialise them;
//   - nothing in it has to start at zero: every partial the combine pass
//     reads is written by the same call first.
// The first call on a device looks up the array's device address
// (cudaGetSymbolAddress with that device current) and caches it; make that
// first call before any stream capture.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace attn {
namespace {

constexpr size_t kDecodeStaticScratchBytes = 8u << 20;   // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeStaticScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ECUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace attn

extern "C" {

size_t attn_decode_static_max_bytes(void) { return attn::kDecodeStaticScratchBytes; }

int attn_fwd_decode_static(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Nk, int d, float scale,
                           const int32_t* key_lens, void* stream) {
  using namespace attn;
  if (!q || !k || !v || !o) return ATTN_EINVAL;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nk <= 0 || d <= 0 || Hq % Hkv != 0) return ATTN_EINVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_EINVAL;
  if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
  if ((long long)B * Hq >= (1ll << 31) || (long long)B * Hkv * Nk >= (1ll << 31))
    return ATTN_EUNSUPPORTED;
  if (!decode_supported(B, Hq, Hkv, 1, d)) return ATTN_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_EALIGN;
  if (lse && !aligned16(lse)) return ATTN_EALIGN;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ECUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return ATTN_ECUDA;
  const DecodePlan p = decode_plan(B, Hq, Hkv, 1, d, sms);
  if (p.workspace_bytes > kDecodeStaticScratchBytes) return ATTN_EWORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != ATTN_OK) return rc;
  return launch_decode(q, k, v, o, lse, B, Hq, Hkv, 1, Nk, d, DecodeMask(), nullptr, scale, key_lens,
                       scratch, p, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
