// Latency-oriented kernels of the decode step: streaming append, query rotation
// and the split-K combine.
//
//  * append_cluster_kernel: one CTA per (sequence, KV head) vector, the Hkv CTAs
//    of a sequence form a thread-block cluster. Encode as in "Google TurboQuant:
//    6x KV-cache compression" (ebisuda.net), "Stage 1" / "Stage 2", with Pi^T and
//    (S Pi^T)^T staged by one TMA bulk copy; every CTA reads len[b] before a
//    cluster barrier, after which rank 0 advances len[b] ("Fractal KV-cache
//    archive" (gist.science), "Problem statement": O(1) append to a growing cache).
//  * qprep_wide_kernel: q' = Pi q and q_s = S q; each CTA owns 32 output columns of
//    a group of query rows and stages only those columns of Pi^T / S^T.
//  * combine_wide_kernel: log-sum-exp merge of one query head's chunk partials and
//    the map back from the rotated domain, o = (Pi_V^T acc + sqrt(pi/2)/m S_V^T acc_s)
//    / sum p; each CTA owns 32 output coordinates.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "encode_simt.cuh"

namespace tqk {

constexpr int kSmallMaxD = 128;
constexpr int kSmallThreads = 256;

// ---------------------------------------------------------------- append

__host__ __device__ inline size_t append_cluster_smem_bytes(int d, int m) {
  return (size_t)d * (d + m) * 4 + (size_t)3 * d * 4 + 64 + 4 * 16 + 64 + 32 * 4;
}

// Encodes input row b * Hkv + h into slot len[b] of KV head h (len itself is not changed);
// a full sequence is skipped and flagged once (by head 0). Returns the slot, or -1 if skipped.
__device__ __forceinline__ int32_t append_vector(const EncodeArgs& a, int b, int h, unsigned char* smem_raw) {
  const int d = a.d, m = a.m, bits = a.bits, L = 1 << bits;
  const int64_t r = (int64_t)b * a.Hkv + h;   // input row
  float* mat = reinterpret_cast<float*>(smem_raw);          // [d][d] Pi^T, then [d][m] (S Pi^T)^T
  float* xs = mat + (size_t)d * (d + m);                    // [d] input, then e
  float* ys = xs + d;                                       // [d]
  float* zs = ys + d;                                       // [d] (unused slot)
  uint32_t* words = reinterpret_cast<uint32_t*>(zs + d);    // [16] packed code words
  uint64_t* bar = reinterpret_cast<uint64_t*>(words + 16);  // [2]
  float* red = reinterpret_cast<float*>(bar + 2);           // [16]
  double* nrm = reinterpret_cast<double*>(red + 16);        // [2]
  float* tbnd = reinterpret_cast<float*>(nrm + 2);          // [16] boundaries, then [16] centroids
  float* tcent = tbnd + 16;
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
  if (tid < L - 1) tbnd[tid] = a.bnd[tid];
  if (tid < L) tcent[tid] = a.cent[tid];
  grid_dep_launch();   // a dependent kernel may start once this CTA's loads are in flight
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
        for (int i = 0; i < L - 1; ++i) idx += (y > tbnd[i]) ? 1u : 0u;
        const int bit = tid * bits;
        atomicOr(&words[bit >> 5], idx << (bit & 31));
        if ((bit & 31) + bits > 32) atomicOr(&words[(bit >> 5) + 1], idx >> (32 - (bit & 31)));
        e = y - tcent[idx];
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
        if (tid == 0 && a.rnorms) {   // QJL-only rows keep the norm alone
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
  return full ? -1 : pos;
}

__global__ void __launch_bounds__(kSmallThreads) append_cluster_kernel(EncodeArgs a, int advance) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int32_t pos = append_vector(a, b, h, smem_raw);
  if (advance) {
    // every CTA of the sequence has read len[b]; then rank 0 moves it on
    cg::this_cluster().sync();
    if (pos >= 0 && h == 0 && threadIdx.x == 0) a.len[b] = pos + 1;
  }
}

// ---------------------------------------------------------------- query rotation

constexpr int kQRows = 8;      // query rows per CTA (small batches)
constexpr int kQRowsBig = 64;  // query rows per CTA from 512 rows on: the column slice is staged once per 64 rows

// q' = Pi q and q_s = S q for d <= kWideMaxD: CTA (row group, column block) computes 32 of the d + m
// outputs (q' = Pi q for o < d, q_s = S q after) of up to kQRows query rows. It stages
// only its 32 columns of Pi^T (or S^T), d x 32 floats, with every thread's vector loads in
// flight at once, then forms the dot products from shared memory.
constexpr int kWideMaxD = 512;
constexpr int kWideCols = 32;

__host__ __device__ inline size_t qprep_wide_smem_bytes(int d, int rpc) {
  return (size_t)d * kWideCols * 4 + (size_t)rpc * d * 4;
}

__device__ __forceinline__ void qprep_tile(const void* q, int q_dtype, int rows, int d, const float* PiT,
                                           const float* ST, int m, float* out_r, float* out_s, int rg, int cb,
                                           int rpc, unsigned char* smem_raw) {
  float* sub = reinterpret_cast<float*>(smem_raw);   // [d][32]
  float* qsh = sub + (size_t)d * kWideCols;           // [rpc][d]
  const int row0 = rg * rpc, nr = min(rpc, rows - row0);
  const int o0 = cb * kWideCols;
  const bool rot = o0 < d;
  const float* src = rot ? PiT + o0 : ST + (o0 - d);
  const int ld = rot ? d : m;
  const int tid = threadIdx.x;
  for (int i = tid; i < d * (kWideCols / 4); i += blockDim.x) {
    const int k = i / (kWideCols / 4), c4 = i % (kWideCols / 4);
    cp_async16(reinterpret_cast<float4*>(sub) + i, src + (size_t)k * ld + 4 * c4);
  }
  if (q_dtype == TQ_F32 && (d % 4) == 0 && (reinterpret_cast<uintptr_t>(q) & 15) == 0) {
    const float* qf = static_cast<const float*>(q) + (size_t)row0 * d;
    for (int i = tid; i < nr * d / 4; i += blockDim.x) cp_async16(reinterpret_cast<float4*>(qsh) + i, qf + 4 * i);
  } else {
#pragma unroll 4
    for (int i = tid; i < nr * d; i += blockDim.x) qsh[i] = load_any(q, q_dtype, (int64_t)row0 * d + i);
  }
  grid_dep_launch();   // a dependent kernel may start once this CTA's loads are in flight
  cp_async_wait_all();
  __syncthreads();
  const int c = tid % kWideCols;
  for (int r = tid / kWideCols; r < nr; r += blockDim.x / kWideCols) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int k = 0; k < d; ++k) acc[k & 3] = fmaf(sub[k * kWideCols + c], qsh[r * d + k], acc[k & 3]);
    const float v = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    if (rot)
      out_r[(size_t)(row0 + r) * d + o0 + c] = v;
    else
      out_s[(size_t)(row0 + r) * m + (o0 - d) + c] = v;
  }
}

__global__ void __launch_bounds__(kSmallThreads) qprep_wide_kernel(const void* q, int q_dtype, int rows, int d,
                                                                   const float* PiT, const float* ST, int m,
                                                                   float* out_r, float* out_s, int rpc) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  grid_dep_launch();
  qprep_tile(q, q_dtype, rows, d, PiT, ST, m, out_r, out_s, blockIdx.x, blockIdx.y, rpc, smem_raw);
}

// ---------------------------------------------------------------- batched query rotation

// C = X B for a batch of fp32 query rows (X [rows][K] row-major, B [K][N] row-major: Pi^T or
// S^T), C [rows][N]: 128 x 128 output tiles per CTA, 8 x 8 per thread, K in steps of 16 through
// shared memory (X transposed on the way in). For the large query batches of the search, where
// the per-row kernels above re-read B once per row group. K % 16 == 0 and N % 4 == 0; rows and
// N need not be multiples of the tile.
constexpr int kRotBM = 128, kRotBN = 128, kRotBK = 16;
__global__ void __launch_bounds__(256) rotate_tiled_kernel(const float* __restrict__ X, int rows, int K,
                                                           const float* __restrict__ B, int N,
                                                           float* __restrict__ C) {
  __shared__ __align__(16) float As[kRotBK][kRotBM];
  __shared__ __align__(16) float Bs[kRotBK][kRotBN];
  grid_dep_launch();
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kRotBM, n0 = blockIdx.x * kRotBN;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kRotBK) {
    // X tile: 128 rows x 16 k, two float4 per thread, stored transposed
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = tid + 256 * r, row = e >> 2, kq = (e & 3) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + row < rows) v = *reinterpret_cast<const float4*>(X + (size_t)(m0 + row) * K + k0 + kq);
      As[kq][row] = v.x;
      As[kq + 1][row] = v.y;
      As[kq + 2][row] = v.z;
      As[kq + 3][row] = v.w;
    }
    // B tile: 16 k x 128 columns, two float4 per thread
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = tid + 256 * r, kk = e >> 5, c = (e & 31) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n0 + c < N) v = *reinterpret_cast<const float4*>(B + (size_t)(k0 + kk) * N + n0 + c);
      *reinterpret_cast<float4*>(&Bs[kk][c]) = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRotBK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = m0 + ty * 8 + i;
    if (row >= rows) continue;
#pragma unroll
    for (int j = 0; j < 8; j += 4) {
      const int col = n0 + tx * 8 + j;
      if (col < N)
        *reinterpret_cast<float4*>(C + (size_t)row * N + col) =
            make_float4(acc[i][j], acc[i][j + 1], acc[i][j + 2], acc[i][j + 3]);
    }
  }
}

// ---------------------------------------------------------------- decode-step prologue

// One launch for the independent first half of a decode step: CTAs [0, nvec) append the
// new keys, [nvec, 2 nvec) the new values (slot len[b], len unchanged: the combine that
// ends the step advances it), and the rest rotate the queries (qprep_tile).
struct PrologueArgs {
  EncodeArgs k, v;
  int nvec;          // B * Hkv
  const void* q;
  int q_dtype, rows, d, m, qcols;
  const float* PiT;
  const float* ST;
  float* qr;
  float* qs;
  const void* pf[2];       // prefetched into L2 for a later kernel of the step (may be NULL)
  uint32_t pf_bytes[2];    // multiples of 16
};

__global__ void __launch_bounds__(kSmallThreads) decode_prologue_kernel(PrologueArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // each role signals the attention kernel (launched as this one's dependent) once its own
  // loads are in flight, so that they queue ahead of the attention's streaming reads
  const int bid = blockIdx.x;
  if (bid == 0 && threadIdx.x < 2 && p.pf[threadIdx.x] && p.pf_bytes[threadIdx.x])
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p.pf[threadIdx.x]), "r"(p.pf_bytes[threadIdx.x])
                 : "memory");
  if (bid < 2 * p.nvec) {
    const int v = bid % p.nvec;
    const EncodeArgs& a = bid < p.nvec ? p.k : p.v;
    (void)append_vector(a, v / a.Hkv, v % a.Hkv, smem_raw);
  } else {
    const int t = bid - 2 * p.nvec;
    qprep_tile(p.q, p.q_dtype, p.rows, p.d, p.PiT, p.ST, p.m, p.qr, p.qs, t / p.qcols, t % p.qcols, kQRows,
               smem_raw);
  }
}

// ---------------------------------------------------------------- combine

// Partial results: [B*Hq][nsplit][stride] floats, stride = pad4(d + mv + 2):
// rotated-domain value sum (d), QJL sum (mv), chunk max, chunk sum of p.
__host__ __device__ inline int partial_stride(int d, int mv) { return (d + mv + 2 + 3) / 4 * 4; }

struct CombineWideArgs {
  int32_t* len_advance;   // decode step: len[b] += 1 (below L_cap) once the step is done, else NULL
  int Hq;
  int64_t L_cap;
  const float* part;
  int nsplit, d, mv;
  const float* PiV;   // [d][d]
  const float* SV;    // [mv][d]
  float* out;         // [B*Hq][d]
  int* err;
};

// Wide combine for d <= kWideMaxD: CTA (query row, 32-coordinate block) merges all chunk
// partials of its row by log-sum-exp (w_s = exp(max_s - M), L = sum_s w_s l_s), forms the
// rotated-domain sums acc = sum_s w_s part_s, and applies its 32 columns of the inverse map:
// o_j = (sum_k Pi_V[k][j] acc[k] + sqrt(pi/2)/m sum_k S_V[k][j] acc_s[k]) / L.
__host__ __device__ inline size_t combine_wide_smem_bytes(int nsplit, int d, int mv) {
  return (size_t)(d + mv) * kWideCols * 4 + (size_t)nsplit * 4 + (size_t)(d + mv) * 4 + 64 +
         (size_t)nsplit * partial_stride(d, mv) * 4;
}

__global__ void __launch_bounds__(kSmallThreads) combine_wide_kernel(CombineWideArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = a.d, mv = a.mv, dm = d + mv, stride = partial_stride(d, mv), ns = a.nsplit;
  float* P = reinterpret_cast<float*>(smem_raw);      // [ns][stride]: this row's partials (stride % 4 == 0)
  float* cols = P + (size_t)ns * stride;               // [d + mv][32]: Pi_V rows k, then S_V rows k
  float* w = cols + (size_t)dm * kWideCols;            // [ns]
  float* acc = w + ns;                                 // [d + mv]
  float* misc = acc + dm;                              // [16]
  const int row = blockIdx.x, j0 = blockIdx.y * kWideCols;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < dm * (kWideCols / 4); i += blockDim.x) {
    const int k = i / (kWideCols / 4), c4 = i % (kWideCols / 4);
    const float* src = (k < d) ? a.PiV + (size_t)k * d : a.SV + (size_t)(k - d) * d;
    cp_async16(reinterpret_cast<float4*>(cols) + i, src + j0 + 4 * c4);
  }
  grid_dep_wait();   // the partials (and, in a decode step, len) come from the attention kernel
  {  // all of the row's partials (stride is a multiple of 4 floats)
    const float* src = a.part + (size_t)row * ns * stride;
    for (int i = tid; i < ns * stride / 4; i += blockDim.x) cp_async16(reinterpret_cast<float4*>(P) + i, src + 4 * i);
  }
  cp_async_wait_all();
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, P[(size_t)s * stride + dm]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = P[(size_t)s * stride + dm];
      const float ws = (ms == -INFINITY) ? 0.f : __expf(ms - M);
      w[s] = ws;
      Ls += ws * P[(size_t)s * stride + dm + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (lane == 0) misc[0] = Ls;
  }
  __syncthreads();
  for (int j = tid; j < dm; j += blockDim.x) {
    float v0 = 0.f, v1 = 0.f;
    int s = 0;
    for (; s + 1 < ns; s += 2) {
      v0 = fmaf(w[s], P[(size_t)s * stride + j], v0);
      v1 = fmaf(w[s + 1], P[(size_t)(s + 1) * stride + j], v1);
    }
    if (s < ns) v0 = fmaf(w[s], P[(size_t)s * stride + j], v0);
    acc[j] = v0 + v1;
  }
  __syncthreads();
  // thread (c, slice): partial dot over k = slice, slice + 8, ... for column c, then a shuffle-free
  // reduction through shared memory (the 8 slices of a column are 8 warps)
  const float qscale = (mv > 0) ? kQjlScale / (float)mv : 0.f;
  const int c = tid % kWideCols, sl = tid / kWideCols, nsl = blockDim.x / kWideCols;
  float o = 0.f, os = 0.f;
  for (int k = sl; k < d; k += nsl) o = fmaf(cols[k * kWideCols + c], acc[k], o);
  for (int k = sl; k < mv; k += nsl) os = fmaf(cols[(d + k) * kWideCols + c], acc[d + k], os);
  __syncthreads();
  float* red = cols;   // reuse: [nsl][32]
  red[sl * kWideCols + c] = fmaf(qscale, os, o);
  __syncthreads();
  if (tid < kWideCols) {
    float t = 0.f;
    for (int i = 0; i < nsl; ++i) t += red[i * kWideCols + tid];
    const float Ls = misc[0];
    a.out[(size_t)row * d + j0 + tid] = (Ls > 0.f) ? t / Ls : 0.f;
  }
  if (a.len_advance && blockIdx.y == 0 && row % a.Hq == 0 && tid == 0) {
    const int b = row / a.Hq;
    const int32_t cur = a.len_advance[b];
    if (cur >= 0 && cur < a.L_cap) a.len_advance[b] = cur + 1;
  }
}

}  // namespace tqk
