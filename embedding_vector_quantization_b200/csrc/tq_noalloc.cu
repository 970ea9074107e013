// Allocation-free variant of the decode attention entry point.
//
// Some callers cannot allocate device memory when they call us: a plugin or
// custom op inside an inference engine that is handed only its input and
// output buffers, a real-time serving loop whose allocator is frozen after
// start-up, or a host program with no device allocator of its own. For them,
// tq_attn_decode_noalloc runs the same kernels as tq_attn_decode but takes its
// split-K scratch (rotated queries and per-chunk partial sums) from a fixed
// array that lives inside libtq.so. Every GPU that loads the library holds
// this array until the process exits.
//
// The array's address is a device address that host code cannot name
// directly; it is looked up once per device with cudaGetSymbolAddress while
// that device is current, on the first call made on that device. The address
// belongs to the device's context: after cudaDeviceReset (or anything else that
// destroys and re-creates the primary context) it is stale, as are all handles
// created before; the library must not be used again in that process.

#include <cuda_runtime.h>

#include <mutex>

#include "tq.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

}  // namespace

extern "C" int tq_attn_decode_noalloc(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype,
                                      int B, int Hq, int Hkv, const tq_cache* k, const tq_cache* v,
                                      const int32_t* len, float scale, float* out, void* stream) {
  if (!hk || !hv) return tq_internal_fail(TQ_EINVAL, "tq_attn_decode_noalloc: handle is NULL");
  if (B < 0 || Hq < 1 || Hkv < 1) return tq_internal_fail(TQ_EINVAL, "tq_attn_decode_noalloc: bad B/Hq/Hkv");
  // nothing to attend: tq_attn_decode checks the rest and returns without touching any buffer
  if (B == 0) return tq_attn_decode(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, len, scale, out, nullptr, 0, stream);
  if (!k) return tq_internal_fail(TQ_EINVAL, "tq_attn_decode_noalloc: key cache is NULL");
  const size_t need = tq_internal_attn_workspace_min_bytes(hk, hv, B, Hq, Hkv, k->L_cap);
  if (need == 0) return tq_internal_fail(TQ_EINVAL, "tq_attn_decode_noalloc: invalid shape");
  if (need > kNoAllocScratchBytes)
    return tq_internal_fail(TQ_EINVAL,
                            "tq_attn_decode_noalloc: this shape needs %zu bytes of scratch, more than the "
                            "library's fixed %zu-byte array; use tq_attn_decode with a caller workspace",
                            need, kNoAllocScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq_internal_fail(TQ_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tq_internal_fail(TQ_EUNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // with device `dev` current
      if (e != cudaSuccess)
        return tq_internal_fail(TQ_ECUDA, "cudaGetSymbolAddress(no-alloc scratch): %s", cudaGetErrorString(e));
      g_noalloc_addr[dev] = p;
    }
    scratch = g_noalloc_addr[dev];
  }
  return tq_attn_decode(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, len, scale, out, scratch, kNoAllocScratchBytes,
                        stream);
}
