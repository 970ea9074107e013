// Latency-oriented kernels of the decode step for head dimensions up to 128:
// streaming append, query rotation and the split-K combine. Each stages the
// small constant matrices it needs (Pi^T, (S Pi^T)^T, S^T, Pi_V, S_V) and its
// other inputs with one TMA bulk copy -- a single memory round trip -- and then
// works from shared memory, one thread per output coordinate.
//
//  * append_cluster_kernel: one CTA per (sequence, KV head) vector, the Hkv CTAs
//    of a sequence form a thread-block cluster. Encode as in "Google TurboQuant:
//    6x KV-cache compression" (ebisuda.net), "Stage 1" / "Stage 2"; every CTA
//    reads len[b] before a cluster barrier, after which rank 0 advances len[b]
//    ("Fractal KV-cache archive" (gist.science), "Problem statement": O(1)
//    append to a growing cache).
//  * qprep_staged_kernel: q' = Pi q and q_s = S q for a group of query rows.
//  * combine_staged_kernel: log-sum-exp merge of one query head's chunk partials
//    and the map back from the rotated domain,
//    o = (Pi_V^T acc + sqrt(pi/2)/m S_V^T acc_s) / sum p.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "encode_simt.cuh"

namespace tqk {

constexpr int kSmallMaxD = 128;
constexpr int kSmallThreads = 256;

// ---------------------------------------------------------------- append

__host__ __device__ inline size_t append_cluster_smem_bytes(int d, int m) {
  return (size_t)d * (d + m) * 4 + (size_t)3 * d * 4 + 64 + 4 * 16 + 64;
}

__global__ void __launch_bounds__(kSmallThreads) append_cluster_kernel(EncodeArgs a, int advance) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = a.d, m = a.m, bits = a.bits, L = 1 << bits;
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t r = (int64_t)b * a.Hkv + h;   // input row
  float* mat = reinterpret_cast<float*>(smem_raw);          // [d][d] Pi^T, then [d][m] (S Pi^T)^T
  float* xs = mat + (size_t)d * (d + m);                    // [d] input, then e
  float* ys = xs + d;                                       // [d]
  float* zs = ys + d;                                       // [d] (unused slot)
  uint32_t* words = reinterpret_cast<uint32_t*>(zs + d);    // [16] packed code words
  uint64_t* bar = reinterpret_cast<uint64_t*>(words + 16);  // [2]
  float* red = reinterpret_cast<float*>(bar + 2);           // [16]
  double* nrm = reinterpret_cast<double*>(red + 16);        // [2]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int32_t pos = a.len[b];
  const bool full = pos < 0 || pos >= a.L_cap;
  if (tid == 0 && !full) {
    bar_init(bar, 1);
    const uint32_t b1 = (uint32_t)d * d * 4, b2 = (uint32_t)d * m * 4;
    bar_expect_tx(bar, b1 + b2);
    bulk_g2s_large(mat, a.PiT, b1, bar);
    if (m > 0) bulk_g2s_large(mat + (size_t)d * d, a.MT, b2, bar);
  }
  if (tid < 16) words[tid] = 0u;
  if (tid < d) xs[tid] = load_any(a.x, a.x_dtype, r * d + tid);
  __syncthreads();
  if (full) {
    if (tid == 0 && h == 0) report_error(a.err, kErrCapacity);
  } else {
    const int64_t orow = r * a.L_cap + pos;
    if (warp == 0) {
      double s = 0.0;
      for (int k = lane; k < d; k += 32) s += (double)xs[k] * (double)xs[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        nrm[0] = sqrt(s);
        store_norm(a.norms, a.norm_dtype, orow, nrm[0]);
      }
    }
    const bool arrived = bar_wait(bar, 0);
    if (__syncthreads_or(!arrived)) {
      if (tid == 0) {
        report_error(a.err, kErrTimeout);
        (void)bar_wait(bar, 0);
      }
    } else {
      const double nn = nrm[0];
      const float inv = nn > 0.0 ? (float)(1.0 / nn) : 0.f;
      float e = 0.f;
      if (tid < d) {
        float acc = 0.f;
#pragma unroll 8
        for (int k = 0; k < d; ++k) acc = fmaf(mat[k * d + tid], xs[k], acc);
        const float y = acc * inv;
        uint32_t idx = 0;
        for (int i = 0; i < L - 1; ++i) idx += (y > a.bnd[i]) ? 1u : 0u;
        const int bit = tid * bits;
        atomicOr(&words[bit >> 5], idx << (bit & 31));
        if ((bit & 31) + bits > 32) atomicOr(&words[(bit >> 5) + 1], idx >> (32 - (bit & 31)));
        e = y - a.cent[idx];
      }
      __syncthreads();   // all reads of xs are done: it now holds e
      if (tid < d) xs[tid] = e;
      if (tid < d * bits / 32) reinterpret_cast<uint32_t*>(a.codes + orow * (int64_t)a.codes_B)[tid] = words[tid];
      if (m > 0) {
        float e2 = e * e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) e2 += __shfl_xor_sync(0xffffffffu, e2, o);
        if (lane == 0) red[warp] = e2;
        __syncthreads();
        if (tid == 0) {
          float t = 0.f;
          for (int w = 0; w < kSmallThreads / 32; ++w) t += red[w];
          a.rnorms[orow] = __double2half(nn > 0.0 ? nn * sqrt((double)t) : 0.0);
        }
        const float* mt = mat + (size_t)d * d;
        float z = 0.f;
        if (tid < m) {
#pragma unroll 8
          for (int k = 0; k < d; ++k) z = fmaf(mt[k * m + tid], xs[k], z);
        }
        const uint32_t wsig = __ballot_sync(0xffffffffu, nn == 0.0 || z >= 0.f);
        if (tid < m && lane == 0) reinterpret_cast<uint32_t*>(a.signs + orow * (int64_t)a.signs_B)[warp] = wsig;
      }
    }
  }
  if (advance) {
    // every CTA of the sequence has read len[b]; then rank 0 moves it on
    cg::this_cluster().sync();
    if (!full && h == 0 && tid == 0) a.len[b] = pos + 1;
  }
}

// ---------------------------------------------------------------- query rotation

constexpr int kQRows = 8;

__host__ __device__ inline size_t qprep_staged_smem_bytes(int d, int m) {
  return (size_t)d * (d + m) * 4 + (size_t)kQRows * d * 4 + 16;
}

// mats = [Pi^T | S^T] as two row-major blocks [d][d] and [d][m].
__global__ void __launch_bounds__(kSmallThreads) qprep_staged_kernel(const void* q, int q_dtype, int rows, int d,
                                                                     const float* PiT, const float* ST, int m,
                                                                     float* out_r, float* out_s, int* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* mat = reinterpret_cast<float*>(smem_raw);
  float* qsh = mat + (size_t)d * (d + m);
  uint64_t* bar = reinterpret_cast<uint64_t*>(qsh + kQRows * d);
  const int row0 = blockIdx.x * kQRows, nr = min(kQRows, rows - row0);
  const int tid = threadIdx.x;
  if (tid == 0) {
    bar_init(bar, 1);
    const uint32_t b1 = (uint32_t)d * d * 4, b2 = (uint32_t)d * m * 4;
    bar_expect_tx(bar, b1 + b2);
    bulk_g2s_large(mat, PiT, b1, bar);
    if (m > 0) bulk_g2s_large(mat + (size_t)d * d, ST, b2, bar);
  }
  for (int i = tid; i < nr * d; i += blockDim.x) qsh[i] = load_any(q, q_dtype, (int64_t)row0 * d + i);
  __syncthreads();
  const bool arrived = bar_wait(bar, 0);
  if (__syncthreads_or(!arrived)) {
    if (tid == 0) { report_error(err, kErrTimeout); (void)bar_wait(bar, 0); }
    return;
  }
  for (int o = tid; o < d + m; o += blockDim.x) {
    const bool rot = o < d;
    const float* col = rot ? mat + o : mat + (size_t)d * d + (o - d);
    const int ld = rot ? d : m;
    float acc[kQRows];
#pragma unroll
    for (int r = 0; r < kQRows; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int k = 0; k < d; ++k) {
      const float v = col[(size_t)k * ld];
#pragma unroll
      for (int r = 0; r < kQRows; ++r) acc[r] = fmaf(v, qsh[r * d + k], acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kQRows; ++r) {
      if (r >= nr) break;
      if (rot)
        out_r[(size_t)(row0 + r) * d + o] = acc[r];
      else
        out_s[(size_t)(row0 + r) * m + (o - d)] = acc[r];
    }
  }
}

// ---------------------------------------------------------------- combine

// Partial results: [B*Hq][nsplit][stride] floats, stride = pad4(d + mv + 2):
// rotated-domain value sum (d), QJL sum (mv), chunk max, chunk sum of p.
__host__ __device__ inline int partial_stride(int d, int mv) { return (d + mv + 2 + 3) / 4 * 4; }

__host__ __device__ inline size_t combine_staged_smem_bytes(int nsplit, int d, int mv) {
  return 16 + (size_t)nsplit * partial_stride(d, mv) * 4 + (size_t)d * (d + mv) * 4 + (size_t)nsplit * 4 +
         (size_t)(d + mv) * 4 + 64;
}

struct CombineStagedArgs {
  const float* part;
  int nsplit, d, mv;
  const float* PiV;   // [d][d]
  const float* SV;    // [mv][d]
  float* out;         // [B*Hq][d]
  int* err;
};

__global__ void __launch_bounds__(kSmallThreads) combine_staged_kernel(CombineStagedArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = a.d, mv = a.mv, dm = d + mv, stride = partial_stride(d, mv), ns = a.nsplit;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw);  // [2] (16 bytes, keeps the copies 16-byte aligned)
  float* P = reinterpret_cast<float*>(smem_raw + 16);     // [ns][stride]
  float* mats = P + (size_t)ns * stride;                  // [d][d] Pi_V then [mv][d] S_V
  float* w = mats + (size_t)d * dm;                       // [ns]
  float* acc = w + ns;                                    // [d + mv]
  float* misc = acc + dm;                                 // [16]
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    bar_init(bar, 1);
    const uint32_t bp = (uint32_t)ns * stride * 4, b1 = (uint32_t)d * d * 4, b2 = (uint32_t)mv * d * 4;
    bar_expect_tx(bar, bp + b1 + b2);
    bulk_g2s_large(P, a.part + (size_t)row * ns * stride, bp, bar);
    bulk_g2s_large(mats, a.PiV, b1, bar);
    if (mv > 0) bulk_g2s_large(mats + (size_t)d * d, a.SV, b2, bar);
  }
  __syncthreads();
  const bool arrived = bar_wait(bar, 0);
  if (__syncthreads_or(!arrived)) {
    if (tid == 0) { report_error(a.err, kErrTimeout); (void)bar_wait(bar, 0); }
    return;
  }
  if (warp == 0) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, P[s * stride + dm]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = P[s * stride + dm];
      const float ws = (ms == -INFINITY) ? 0.f : __expf(ms - M);
      w[s] = ws;
      Ls += ws * P[s * stride + dm + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (lane == 0) misc[0] = Ls;
  }
  __syncthreads();
  for (int j = tid; j < dm; j += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < ns; ++s) v = fmaf(w[s], P[s * stride + j], v);
    acc[j] = v;
  }
  __syncthreads();
  const float qscale = (mv > 0) ? kQjlScale / (float)mv : 0.f;
  for (int j = tid; j < d; j += blockDim.x) {
    float o = 0.f, os = 0.f;
#pragma unroll 8
    for (int k = 0; k < d; ++k) o = fmaf(mats[k * d + j], acc[k], o);
    for (int k = 0; k < mv; ++k) os = fmaf(mats[(size_t)(d + k) * d + j], acc[d + k], os);
    o = fmaf(qscale, os, o);
    const float Ls = misc[0];
    a.out[(size_t)row * d + j] = (Ls > 0.f) ? o / Ls : 0.f;
  }
}

}  // namespace tqk
