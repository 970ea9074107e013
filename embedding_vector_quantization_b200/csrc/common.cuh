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

}  // namespace tqk
