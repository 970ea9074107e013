// Encode of a few vectors at a time (streaming append, small batches), d <= 512.
//
// Same computation as encode_simt_kernel ("Google TurboQuant: 6x KV-cache
// compression", sections "Stage 1" and "Stage 2": norm, y = Pi x / ||x||,
// Lloyd-Max cell, bit-pack; prod: signs of (S Pi^T)(y - c[idx]) and ||x|| ||y - c||),
// organised for latency instead of throughput: one CTA owns up to kRowsMax rows
// and every thread owns one output coordinate of a subset of the rows, reading
// Pi^T (and (S Pi^T)^T) with coalesced loads from L2.
//
// Append mode: the CTA owns the Hkv rows of one sequence b, writes them at slot
// len[b] of each head and, once all heads are written, advances len[b] itself
// ("Fractal KV-cache archive" (gist.science), "Problem statement": O(1) append
// to a growing cache). A full sequence is skipped and reported.
#pragma once

#include "common.cuh"
#include "encode_simt.cuh"

namespace tqk {

constexpr int kRowsMax = 16;
constexpr int kRowsThreads = 256;
constexpr int kRowsMaxD = 512;

// Pi^T (and (S Pi^T)^T) are staged in shared memory when they fit (d * (d + m) <= kStageFloats).
constexpr int kStageFloats = 128 * 256;

__host__ __device__ inline bool encode_rows_staged(int d, int m) { return d * (d + m) <= kStageFloats; }

__host__ __device__ inline size_t encode_rows_smem_bytes(int d, int m) {
  size_t b = (size_t)kRowsMax * d * 4 * 2 + (size_t)kRowsMax * (8 + 4 + 4) + 32 * 4 + 16;
  if (encode_rows_staged(d, m)) b += (size_t)d * (d + m) * 4;
  return b;
}

// rows handled by CTA c: plain mode rows [c*kRowsMax, ...); append mode the Hkv rows of sequence c.
__global__ void __launch_bounds__(kRowsThreads) encode_rows_kernel(EncodeArgs a, int advance) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = a.d, m = a.m, bits = a.bits, L = 1 << bits;
  const bool append = a.len != nullptr;
  const int R = append ? a.Hkv : (int)min((int64_t)kRowsMax, a.rows - (int64_t)blockIdx.x * kRowsMax);
  const int64_t r0 = append ? (int64_t)blockIdx.x * a.Hkv : (int64_t)blockIdx.x * kRowsMax;
  float* xs = reinterpret_cast<float*>(smem_raw);      // [kRowsMax][d]  input, then e = y - c[idx]
  float* ys = xs + kRowsMax * d;                       // [kRowsMax][d]  rotated unit coordinates
  double* nrm = reinterpret_cast<double*>(ys + kRowsMax * d);  // [kRowsMax]
  float* inv = reinterpret_cast<float*>(nrm + kRowsMax);       // [kRowsMax]
  float* esq = inv + kRowsMax;                                 // [kRowsMax]
  float* bnd = esq + kRowsMax;                                 // [16]
  float* cen = bnd + 16;                                       // [16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(cen + 16);      // [2] (16 bytes)
  float* mats = reinterpret_cast<float*>(bar + 2);             // [d][d] Pi^T then [d][m] (S Pi^T)^T, if staged
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool staged = encode_rows_staged(d, m);

  // output slot (same for every head of the sequence in append mode)
  int64_t slot = 0;
  bool skip = false;
  if (append) {
    const int32_t pos = a.len[blockIdx.x];
    skip = pos < 0 || pos >= a.L_cap;
    slot = pos;
  }
  if (skip) {
    if (tid == 0) report_error(a.err, kErrCapacity);
    return;
  }
  auto out_row = [&](int r) -> int64_t { return append ? (r0 + r) * a.L_cap + slot : r0 + r; };

  if (tid < L - 1) bnd[tid] = a.bnd[tid];
  if (tid < L) cen[tid] = a.cent[tid];
  if (tid < kRowsMax) esq[tid] = 0.f;
  for (int i = tid; i < R * d; i += blockDim.x) xs[i] = load_any(a.x, a.x_dtype, r0 * d + i);
  if (staged && tid == 0) {  // one bulk copy per matrix: a single memory round trip
    bar_init(bar, 1);
    const uint32_t b1 = (uint32_t)d * d * 4, b2 = (uint32_t)d * m * 4;
    bar_expect_tx(bar, b1 + b2);
    bulk_g2s_large(mats, a.PiT, b1, bar);
    if (m > 0) bulk_g2s_large(mats + d * d, a.MT, b2, bar);
  }
  const float* PiT = staged ? mats : a.PiT;
  const float* MT = staged ? mats + d * d : a.MT;
  __syncthreads();
  const bool arrived = !staged || bar_wait(bar, 0);
  if (__syncthreads_or(!arrived)) {   // the decision is the same for every thread of the CTA
    if (tid == 0) {
      report_error(a.err, kErrTimeout);
      (void)bar_wait(bar, 0);         // one more bounded wait for the copy still in flight
    }
    return;
  }

  // norms in fp64, one warp per row
  for (int r = warp; r < R; r += blockDim.x / 32) {
    double s = 0.0;
    for (int k = lane; k < d; k += 32) s += (double)xs[r * d + k] * (double)xs[r * d + k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      const double nn = sqrt(s);
      nrm[r] = nn;
      inv[r] = nn > 0.0 ? (float)(1.0 / nn) : 0.f;
      store_norm(a.norms, a.norm_dtype, out_row(r), nn);
    }
  }
  __syncthreads();

  // y = Pi x / ||x||: thread -> coordinate j and rows rg, rg + groups, ... (at most kRowsMax / groups of them)
  const int groups = max(1, (int)blockDim.x / d);
  for (int base = tid; base < d * groups; base += blockDim.x) {
    const int j = base % d, rg = base / d;
    const int nr = (R - rg + groups - 1) / groups;   // rows of this thread
    float acc[kRowsMax];
#pragma unroll
    for (int i = 0; i < kRowsMax; ++i) acc[i] = 0.f;
    const float* xr = xs + rg * d;
    const int rstride = groups * d;
    for (int k = 0; k < d; ++k) {
      const float p = PiT[(size_t)k * d + j];
#pragma unroll
      for (int i = 0; i < kRowsMax; ++i)
        if (i < nr) acc[i] = fmaf(p, xr[i * rstride + k], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < kRowsMax; ++i)
      if (i < nr) ys[(rg + i * groups) * d + j] = acc[i] * inv[rg + i * groups];
  }
  __syncthreads();

  // bucketize + pack: thread -> (row, 32-coordinate group); prod keeps e = y - c[idx]
  const int ngroups = d / 32;
  for (int w = tid; w < R * ngroups; w += blockDim.x) {
    const int r = w / ngroups, grp = w % ngroups;
    // QJL-only rows (0 MSE bits): no codes; idx stays 0 (centroid 0) and nothing is written
    uint32_t* dst = bits ? reinterpret_cast<uint32_t*>(a.codes + out_row(r) * (int64_t)a.codes_B) + grp * bits : nullptr;
    uint64_t win = 0;
    int nb = 0, wout = 0;
    float e2 = 0.f;
    for (int tt = 0; tt < 32; ++tt) {
      const int j = grp * 32 + tt;
      const float y = ys[r * d + j];
      uint32_t idx = 0;
      for (int i = 0; i < L - 1; ++i) idx += (y > bnd[i]) ? 1u : 0u;
      win |= (uint64_t)idx << nb;
      nb += bits;
      if (nb >= 32) { dst[wout++] = (uint32_t)win; win >>= 32; nb -= 32; }
      if (m > 0) {
        const float e = y - cen[idx];
        xs[r * d + j] = e;
        e2 += e * e;
      }
    }
    if (m > 0) atomicAdd(&esq[r], e2);
  }
  __syncthreads();
  if (m > 0) {
    // rnorm = ||x|| * ||e||; z = (S Pi^T) e, one thread per projection i and a stride of rows
    if (tid < R && a.rnorms)   // QJL-only rows keep the norm alone
      a.rnorms[out_row(tid)] = __double2half(nrm[tid] > 0.0 ? nrm[tid] * sqrt((double)esq[tid]) : 0.0);
    const int pgroups = max(1, (int)blockDim.x / m);
    for (int base = tid; base < m * pgroups; base += blockDim.x) {
      const int i = base % m, rg = base / m;
      const int nr = (R - rg + pgroups - 1) / pgroups;
      float acc[kRowsMax];
#pragma unroll
      for (int u = 0; u < kRowsMax; ++u) acc[u] = 0.f;
      const float* er = xs + rg * d;
      const int rstride = pgroups * d;
      for (int k = 0; k < d; ++k) {
        const float p = MT[(size_t)k * m + i];
#pragma unroll
        for (int u = 0; u < kRowsMax; ++u)
          if (u < nr) acc[u] = fmaf(p, er[u * rstride + k], acc[u]);
      }
      // lanes of a warp hold 32 consecutive projections of the same rows: one ballot per row
#pragma unroll
      for (int u = 0; u < kRowsMax; ++u) {
        if (u >= nr) break;
        const int r = rg + u * pgroups;
        const bool pos = nrm[r] == 0.0 || acc[u] >= 0.f;
        const uint32_t word = __ballot_sync(0xffffffffu, pos);
        if ((i & 31) == 0)
          reinterpret_cast<uint32_t*>(a.signs + out_row(r) * (int64_t)a.signs_B)[i >> 5] = word;
      }
    }
  }
  if (append && advance) {
    __syncthreads();
    if (tid == 0) a.len[blockIdx.x] = (int32_t)(slot + 1);
  }
}

}  // namespace tqk
