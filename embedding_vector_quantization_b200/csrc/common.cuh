// Device helpers shared by the kernels of libtq: element loads, the packed
// bit-row reader, error-word reporting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "tq.h"

namespace tqk {

constexpr float kQjlScale = 1.2533141373155002512f;  // sqrt(pi / 2)

// Error bits OR-ed into a handle's device error word (decoded by the host).
constexpr int kErrCapacity = 1;
constexpr int kErrTimeout = 2;
constexpr int kErrInternal = 4;   // a kernel found its own launch state unusable (e.g. shared memory alignment)
constexpr int kErrBounds = 8;     // TQ_CHECK=1: a device-resident argument (a length) was out of range

__device__ __forceinline__ void report_error(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i);
template <>
__device__ __forceinline__ float load_elem<TQ_F32>(const void* p, int64_t i) {
  return static_cast<const float*>(p)[i];
}
template <>
__device__ __forceinline__ float load_elem<TQ_F16>(const void* p, int64_t i) {
  return __half2float(static_cast<const __half*>(p)[i]);
}
template <>
__device__ __forceinline__ float load_elem<TQ_BF16>(const void* p, int64_t i) {
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ float load_any(const void* p, int dtype, int64_t i) {
  if (dtype == TQ_F32) return load_elem<TQ_F32>(p, i);
  if (dtype == TQ_F16) return load_elem<TQ_F16>(p, i);
  return load_elem<TQ_BF16>(p, i);
}

// Stored per-vector norm (fp32 or fp16) as float.
__device__ __forceinline__ float load_norm(const void* p, int norm_dtype, int64_t i) {
  return norm_dtype == TQ_F16 ? __half2float(static_cast<const __half*>(p)[i])
                              : static_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_norm(void* p, int norm_dtype, int64_t i, double v) {
  if (norm_dtype == TQ_F16)
    static_cast<__half*>(p)[i] = __double2half(v);
  else
    static_cast<float*>(p)[i] = static_cast<float>(v);
}

// Index j of a packed row (LSB-first contiguous, b bits per index). `row` is
// 4-byte aligned; a field may straddle two 32-bit words.
__device__ __forceinline__ uint32_t packed_field(const uint32_t* row, int j, int b) {
  const int bit = j * b;
  const int w = bit >> 5, off = bit & 31;
  uint32_t v = row[w] >> off;
  if (off + b > 32) v |= row[w + 1] << (32 - off);
  return v & ((1u << b) - 1u);
}

// Bit j of a sign row.
__device__ __forceinline__ uint32_t sign_bit(const uint32_t* row, int j) {
  return (row[j >> 5] >> (j & 31)) & 1u;
}

// ---- programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream still runs; it must
// wait (grid_dep_wait) before touching that kernel's outputs. Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- asynchronous 16-byte copies (global -> shared): every thread issues all of its
// copies, then waits once, so a staging loop costs one memory latency, not one per element.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// ---- TMA bulk copies (global -> shared) completed on an mbarrier

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// Bounded wait (the thread sleeps between polls); false if the limit was reached.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, int limit = 1 << 16) {
  const uint32_t addr = smem_addr(bar);
  for (int it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(20000)
        : "memory");
    if (done) return true;
  }
  return false;
}

// One contiguous copy; dst, src 16-byte aligned and bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Copies `bytes` (<= 2^20 per call chunk) in pieces the bulk engine accepts.
__device__ __forceinline__ void bulk_g2s_large(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  const uint32_t piece = 1u << 16;
  for (uint32_t off = 0; off < bytes; off += piece)
    bulk_g2s(static_cast<unsigned char*>(dst) + off, static_cast<const unsigned char*>(src) + off,
             min(piece, bytes - off), bar);
}

}  // namespace tqk
