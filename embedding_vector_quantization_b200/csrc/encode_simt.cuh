// Encode and append, SIMT version (any d % 32 == 0, any bits, fp32 CUDA cores).
//
// "Google TurboQuant: 6x KV-cache compression" (ebisuda.net), section
// "Stage 1: PolarQuant": store the norm, rotate y = Pi x / ||x||, map every
// coordinate to its Lloyd-Max cell, no per-block scale; section "Stage 2:
// QJL residual correction": one sign bit per random projection of the
// residual plus its norm. "TurboQuant / PolarQuant / QJL technical deep dive"
// (gemilab.net), section "GPU kernel optimisation": transform all tokens in
// parallel, compute the projection as a matrix product, pack for locality.
//
// One CTA encodes a tile of kBM vectors x kBN output coordinates: a tiled
// fp32 GEMM (x tile and Pi^T tile staged in shared memory) accumulates Pi x
// while the same x tile feeds an fp64 sum of squares (the norm); the epilogue
// scales by 1/||x||, bucketizes against the boundaries and packs each
// 32-coordinate group into `bits` words. Prod handles (d <= kBN, one column
// block) keep e = y - c[idx] in shared memory and run a second GEMM
// z = (S Pi^T) e, whose signs are the QJL bits (sign(0) = +1); ||r|| = ||x|| ||e||.
#pragma once

#include "common.cuh"

namespace tqk {

constexpr int kEncBM = 64;
constexpr int kEncBN = 128;
constexpr int kEncBK = 32;
constexpr int kEncThreads = 256;

struct EncodeArgs {
  const void* x;       // [rows][d], x_dtype
  int x_dtype;
  int64_t rows;
  int d, bits, m, norm_dtype;
  const float* PiT;    // [d][d], PiT[k][j] = Pi[j][k]
  const float* MT;     // [d][m], MT[k][i] = (S Pi^T)[i][k]  (prod)
  const float* cent;   // [2^bits]
  const float* bnd;    // [2^bits - 1]
  uint8_t* codes;
  int codes_B;
  uint8_t* signs;
  int signs_B;
  void* norms;
  __half* rnorms;
  // append mode (len != nullptr): input row r = b * Hkv + h goes to cache row
  // r * L_cap + len[b]; a full sequence is skipped and flagged.
  int32_t* len;
  int Hkv;
  int64_t L_cap;
  int* err;
};

__host__ __device__ inline size_t encode_smem_bytes(int m) {
  size_t f = (size_t)kEncBK * kEncBM + (size_t)kEncBK * kEncBN + (size_t)kEncBM * (kEncBN + 1);
  size_t bytes = f * 4;                       // As, Bs, Ys
  bytes += kEncBM * 8;                        // fp64 squared norms
  bytes += kEncBM * 4 * 2;                    // 1/n, ||e||^2
  bytes += 32 * 4;                            // boundaries (<= 15) + centroids (<= 16)
  bytes += (size_t)kEncBM * ((m + 31) / 32) * 4;  // sign words
  return bytes;
}

__device__ __forceinline__ int64_t encode_out_row(const EncodeArgs& a, int64_t r) {
  if (a.len == nullptr) return r;
  const int64_t b = r / a.Hkv;
  const int32_t pos = a.len[b];
  if (pos < 0 || pos >= a.L_cap) return -1;
  return r * a.L_cap + pos;
}

__global__ void __launch_bounds__(kEncThreads) encode_simt_kernel(EncodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* As = reinterpret_cast<float*>(smem_raw);  // [BK][BM]
  float* Bs = As + kEncBK * kEncBM;                // [BK][BN]
  float* Ys = Bs + kEncBK * kEncBN;                // [BM][BN+1]
  double* nsq = reinterpret_cast<double*>(Ys + kEncBM * (kEncBN + 1));  // [BM]
  float* inv = reinterpret_cast<float*>(nsq + kEncBM);                  // [BM]
  float* esq = inv + kEncBM;                                            // [BM]
  float* bnd = esq + kEncBM;                                            // [16]
  float* cen = bnd + 16;                                                // [16]
  uint32_t* sgn = reinterpret_cast<uint32_t*>(cen + 16);                // [BM][m/32]

  const int tid = threadIdx.x;
  const int64_t v0 = (int64_t)blockIdx.x * kEncBM;
  const int j0 = blockIdx.y * kEncBN;
  const int d = a.d;
  const int L = 1 << a.bits;
  const bool prod = a.m > 0;
  const int mw = (a.m + 31) / 32;

  if (tid < L - 1) bnd[tid] = a.bnd[tid];
  if (tid < L) cen[tid] = a.cent[tid];
  if (tid < kEncBM) { nsq[tid] = 0.0; esq[tid] = 0.f; }
  if (prod)
    for (int i = tid; i < kEncBM * mw; i += kEncThreads) sgn[i] = 0u;

  const int tr = tid >> 4;  // vectors tr*4 .. +3
  const int tc = tid & 15;  // coordinates tc*8 .. +7
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int lv = tid >> 2, lk = (tid & 3) * 8;  // A loader: vector lv, k = lk .. lk+7
  const int bk = tid >> 3, bc = (tid & 7) * 16;  // B loader: row bk, cols bc .. bc+15
  double my_sq = 0.0;
  __syncthreads();

  for (int k0 = 0; k0 < d; k0 += kEncBK) {
    const int64_t v = v0 + lv;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float val = 0.f;
      if (v < a.rows) val = load_any(a.x, a.x_dtype, v * d + k0 + lk + e);
      As[(lk + e) * kEncBM + lv] = val;
      my_sq += (double)val * (double)val;
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int j = j0 + bc + e;
      Bs[bk * kEncBN + bc + e] = (j < d) ? a.PiT[(size_t)(k0 + bk) * d + j] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kEncBK; ++kk) {
      float av[4], bv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk * kEncBM + tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) bv[j] = Bs[kk * kEncBN + tc * 8 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  atomicAdd(&nsq[lv], my_sq);
  __syncthreads();
  if (tid < kEncBM) {
    const double nn = sqrt(nsq[tid]);
    nsq[tid] = nn;
    inv[tid] = nn > 0.0 ? (float)(1.0 / nn) : 0.f;
    const int64_t r = v0 + tid;
    if (blockIdx.y == 0 && r < a.rows) {
      const int64_t orow = encode_out_row(a, r);
      if (orow >= 0)
        store_norm(a.norms, a.norm_dtype, orow, nn);
      else
        report_error(a.err, kErrCapacity);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
      Ys[(tr * 4 + i) * (kEncBN + 1) + tc * 8 + j] = acc[i][j] * inv[tr * 4 + i];
  __syncthreads();

  // Bucketize + pack: thread -> (vector pv, 32-coordinate group g of this tile).
  {
    const int pv = tid >> 2, g = tid & 3;
    const int64_t r = v0 + pv;
    const int jg = j0 + g * 32;
    const int64_t orow = (r < a.rows) ? encode_out_row(a, r) : -1;
    float e2 = 0.f;
    if (orow >= 0 && jg < d) {
      // QJL-only rows (0 MSE bits) have no codes: idx stays 0 (centroid 0) and nothing is written
      uint32_t* dst = a.bits ? reinterpret_cast<uint32_t*>(a.codes + orow * (int64_t)a.codes_B) + (jg >> 5) * a.bits
                             : nullptr;
      uint64_t win = 0;
      int nb = 0, wout = 0;
      for (int t = 0; t < 32; ++t) {
        float* yp = &Ys[pv * (kEncBN + 1) + g * 32 + t];
        const float y = *yp;
        uint32_t idx = 0;
        for (int i = 0; i < L - 1; ++i) idx += (y > bnd[i]) ? 1u : 0u;  // #{bnd < y}; ties go low
        win |= (uint64_t)idx << nb;
        nb += a.bits;
        if (nb >= 32) { dst[wout++] = (uint32_t)win; win >>= 32; nb -= 32; }
        if (prod) {
          const float e = y - cen[idx];
          *yp = e;
          e2 += e * e;
        }
      }
    }
    if (prod) {
      e2 += __shfl_xor_sync(0xffffffffu, e2, 1);
      e2 += __shfl_xor_sync(0xffffffffu, e2, 2);
      if (g == 0) esq[pv] = e2;
    }
  }
  if (!prod) return;
  __syncthreads();

  // QJL stage (prod handles; gridDim.y == 1 so Ys holds every coordinate).
  if (tid < kEncBM) {
    const int64_t r = v0 + tid;
    if (r < a.rows) {
      const int64_t orow = encode_out_row(a, r);
      if (orow >= 0 && a.rnorms) {   // QJL-only rows keep the norm alone
        const double nn = nsq[tid];
        a.rnorms[orow] = __double2half(nn > 0.0 ? nn * sqrt((double)esq[tid]) : 0.0);
      }
    }
  }
  for (int i0 = 0; i0 < a.m; i0 += kEncBN) {
    float z[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) z[i][j] = 0.f;
    for (int k0 = 0; k0 < d; k0 += kEncBK) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int col = i0 + bc + e;
        Bs[bk * kEncBN + bc + e] = (col < a.m) ? a.MT[(size_t)(k0 + bk) * a.m + col] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kEncBK; ++kk) {
        float av[4], bv[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = Ys[(tr * 4 + i) * (kEncBN + 1) + k0 + kk];
#pragma unroll
        for (int j = 0; j < 8; ++j) bv[j] = Bs[kk * kEncBN + tc * 8 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) z[i][j] = fmaf(av[i], bv[j], z[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int vv = tr * 4 + i;
      const bool zero_vec = nsq[vv] == 0.0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = i0 + tc * 8 + j;
        if (col < a.m && (zero_vec || z[i][j] >= 0.f))
          atomicOr(&sgn[vv * mw + (col >> 5)], 1u << (col & 31));
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < kEncBM * mw; i += kEncThreads) {
    const int vv = i / mw, w = i % mw;
    const int64_t r = v0 + vv;
    if (r >= a.rows) continue;
    const int64_t orow = encode_out_row(a, r);
    if (orow < 0) continue;
    reinterpret_cast<uint32_t*>(a.signs + orow * (int64_t)a.signs_B)[w] = sgn[i];
  }
}

// len[b] += 1 for every sequence that was not full (after an append).
__global__ void advance_len_kernel(int32_t* len, int B, int64_t L_cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && len[b] < L_cap) len[b] += 1;
}

// Test hook: pack byte indices [rows][d] into the code layout.
__global__ void pack_indices_kernel(const uint8_t* idx, int64_t rows, int d, int bits,
                                    uint8_t* codes, int codes_B) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int groups = d / 32;
  if (t >= rows * groups) return;
  const int64_t r = t / groups;
  const int g = (int)(t % groups);
  const uint8_t* src = idx + r * d + g * 32;
  uint32_t* dst = reinterpret_cast<uint32_t*>(codes + r * codes_B) + g * bits;
  uint64_t win = 0;
  int nb = 0, wout = 0;
  for (int i = 0; i < 32; ++i) {
    win |= (uint64_t)(src[i] & ((1u << bits) - 1u)) << nb;
    nb += bits;
    if (nb >= 32) { dst[wout++] = (uint32_t)win; win >>= 32; nb -= 32; }
  }
}

}  // namespace tqk
