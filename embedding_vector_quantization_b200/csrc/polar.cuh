// PolarQuant's recursive polar transform: encode and inner-product scores.
//
// "PolarQuant explainer" (aibr.jp), sections 1 and 3, and "TurboQuant: redefining AI
// efficiency" (hakusoku.com), section "PolarQuant": after a random preconditioning the
// vector is turned into polar coordinates by a recursive algorithm -- pairs of coordinates
// become a radius and an angle, pairs of radii again a radius and an angle, down to one
// radius -- and the angles, whose laws are known in closed form, are quantized with
// codebooks built for those laws; no per-block scale is stored.
//
// Encode (one CTA per 64 vectors): y = Pi x / ||x|| by an fp32 SIMT GEMM into shared memory
// (norm in fp64 from the staged input), then level 1 pairs (y_2i, y_2i+1) into
// (hypot, atan2 in (-pi, pi]) and every further level pairs the radii (angle in [0, pi/2]);
// each angle is bucketized against its level's boundaries and the indices are packed
// level after level, LSB-first, into a 16-byte-aligned row.
//
// Scores (one CTA per (sequence, KV head, chunk), one key per thread): with q' = Pi q, the
// score is ||x|| times the root of the transform tree folded bottom-up -- a pair of level 1
// contributes q'_2i cos(theta) + q'_2i+1 sin(theta), read from a per-query table of
// 2^b1 entries per pair, and each further level folds two partial scores as
// S_left cos(psi) + S_right sin(psi) with psi's cosine and sine from the level's table.
// The tree is walked depth first (a binary counter over the level-1 pairs), so a key needs
// log2(d) partial scores per query head in registers.
#pragma once

#include "common.cuh"
#include "encode_simt.cuh"

namespace tqk {
namespace polar {

constexpr int kMaxLevels = 8;   // d <= 256
constexpr int kMaxG = 8;        // query heads per KV head
constexpr int kBM = 64;         // vectors per encode CTA
constexpr int kThreads = 256;   // encode
constexpr int kSThreads = 128;  // score: keys per round

// Per handle on the device: per level, the boundaries (2^b - 1 of 16 slots) and the cosine
// and sine of the centroids.
struct Table {
  float bnd[kMaxLevels][16];
  float cs[kMaxLevels][16];
  float sn[kMaxLevels][16];
};

struct Layout {
  int d, nlev;
  int bits[kMaxLevels];   // index width of each level (level 1 first)
  int off[kMaxLevels];    // bit offset of each level's field in the row
};

struct EncodeArgs {
  const void* x;
  int x_dtype;
  int64_t rows;
  Layout lay;
  int norm_dtype;
  const float* PiT;   // [d][d], PiT[k][j] = Pi[j][k]
  const Table* tab;
  uint8_t* codes;
  int codes_B;
  void* norms;
  // append mode (len != nullptr): input row r = b * Hkv + h goes to cache row r * L_cap + len[b]
  int32_t* len;
  int Hkv;
  int64_t L_cap;
  int* err;
};

__host__ __device__ inline size_t encode_smem_bytes(int d) {
  return sizeof(Table) + (size_t)kBM * 8 + (size_t)kBM * 4            // table, fp64 norms, 1/n
         + (size_t)kEncBK * kBM * 4 + (size_t)kEncBK * kEncBN * 4       // GEMM tiles
         + (size_t)kBM * (d + 1) * 4 + (size_t)kBM * (d / 2 + 1) * 4    // y (then even-level radii), odd-level radii
         + (size_t)kBM * d;                                             // indices
}

__device__ __forceinline__ int64_t polar_out_row(const EncodeArgs& a, int64_t r) {
  if (a.len == nullptr) return r;
  const int32_t pos = a.len[r / a.Hkv];
  if (pos < 0 || pos >= a.L_cap) return -1;
  return r * a.L_cap + pos;
}

// #{i : bnd[i] < v}: an angle on a boundary goes to the lower cell
__device__ __forceinline__ uint32_t bucket(const float* bnd, int nb, float v) {
  uint32_t idx = 0;
  for (int i = 0; i < nb; ++i) idx += (v > bnd[i]) ? 1u : 0u;
  return idx;
}

__global__ void __launch_bounds__(kThreads) polar_encode_kernel(EncodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = a.lay.d, P = d / 2;
  Table* tab = reinterpret_cast<Table*>(smem_raw);
  double* nsq = reinterpret_cast<double*>(tab + 1);               // [kBM]
  float* inv = reinterpret_cast<float*>(nsq + kBM);               // [kBM]
  float* As = inv + kBM;                                          // [BK][BM]
  float* Bs = As + kEncBK * kBM;                                  // [BK][BN]
  float* Y = Bs + kEncBK * kEncBN;                                // [BM][d + 1]
  float* R = Y + kBM * (d + 1);                                   // [BM][d / 2 + 1]
  uint8_t* I = reinterpret_cast<uint8_t*>(R + kBM * (P + 1));     // [BM][d]: level fields, index per angle
  const int tid = threadIdx.x;
  const int64_t v0 = (int64_t)blockIdx.x * kBM;
  const int nv = (int)min((int64_t)kBM, a.rows - v0);

  for (int i = tid; i < (int)(sizeof(Table) / 4); i += kThreads)
    reinterpret_cast<float*>(tab)[i] = reinterpret_cast<const float*>(a.tab)[i];
  if (tid < kBM) nsq[tid] = 0.0;
  __syncthreads();
  // norms in fp64 from the input as loaded (warp w: vectors w, w + 8, ...)
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int v = warp; v < nv; v += kThreads / 32) {
      double s = 0.0;
      for (int k = lane; k < d; k += 32) {
        const double e = (double)load_any(a.x, a.x_dtype, (v0 + v) * d + k);
        s += e * e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) nsq[v] = sqrt(s);
    }
  }
  __syncthreads();
  if (tid < kBM) {
    const double nn = nsq[tid];
    inv[tid] = nn > 0.0 ? (float)(1.0 / nn) : 0.f;
    if (tid < nv) {
      const int64_t orow = polar_out_row(a, v0 + tid);
      if (orow >= 0)
        store_norm(a.norms, a.norm_dtype, orow, nn);
      else
        report_error(a.err, kErrCapacity);
    }
  }
  __syncthreads();

  // y = Pi x / ||x||, 128 output coordinates at a time (the encode_simt GEMM tiling)
  const int tr = tid >> 4, tc = tid & 15;
  const int lv = tid >> 2, lk = (tid & 3) * 8;
  const int bk = tid >> 3, bc = (tid & 7) * 16;
  for (int j0 = 0; j0 < d; j0 += kEncBN) {
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < d; k0 += kEncBK) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        As[(lk + e) * kBM + lv] = (lv < nv) ? load_any(a.x, a.x_dtype, (v0 + lv) * d + k0 + lk + e) : 0.f;
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
        for (int i = 0; i < 4; ++i) av[i] = As[kk * kBM + tr * 4 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) bv[j] = Bs[kk * kEncBN + tc * 8 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = j0 + tc * 8 + j;
        if (col < d) Y[(tr * 4 + i) * (d + 1) + col] = acc[i][j] * inv[tr * 4 + i];
      }
  }
  __syncthreads();

  // the recursion: level 1 reads y and writes radii to R; each further level reads the previous
  // level's radii (R or the front of Y) and writes its own to the other buffer
  int idx_base = 0;
  for (int l = 0; l < a.lay.nlev; ++l) {
    const int pairs = d >> (l + 1);
    const float* src = (l == 0) ? Y : ((l & 1) ? R : Y);
    const int sstride = (l == 0) ? d + 1 : ((l & 1) ? P + 1 : d + 1);
    float* dst = (l & 1) ? Y : R;
    const int dstride = (l & 1) ? d + 1 : P + 1;
    const int nb = (1 << a.lay.bits[l]) - 1;
    for (int it = tid; it < kBM * pairs; it += kThreads) {
      const int v = it / pairs, i = it % pairs;
      const float u0 = src[v * sstride + 2 * i], u1 = src[v * sstride + 2 * i + 1];
      const float ang = atan2f(u1, u0);
      I[v * d + idx_base + i] = (uint8_t)bucket(tab->bnd[l], nb, ang);
      dst[v * dstride + i] = hypotf(u0, u1);
    }
    idx_base += pairs;
    __syncthreads();
  }

  // pack: one thread per vector, the level fields one after the other, LSB-first
  if (tid < nv) {
    const int64_t orow = polar_out_row(a, v0 + tid);
    if (orow >= 0) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + orow * (int64_t)a.codes_B);
      uint64_t win = 0;
      int nb = 0, wout = 0, k = 0;
      for (int l = 0; l < a.lay.nlev; ++l) {
        const int pairs = d >> (l + 1), b = a.lay.bits[l];
        for (int i = 0; i < pairs; ++i, ++k) {
          win |= (uint64_t)I[tid * d + k] << nb;
          nb += b;
          if (nb >= 32) { dst[wout++] = (uint32_t)win; win >>= 32; nb -= 32; }
        }
      }
      if (nb > 0) dst[wout++] = (uint32_t)win;
      for (; wout < a.codes_B / 4; ++wout) dst[wout] = 0u;   // pad bits are zero
    }
  }
}

// ---------------------------------------------------------------- scores

struct ScoreArgs {
  const float* qr;   // [B*Hq][d] Pi q
  int B, Hq, Hkv;
  Layout lay;
  const uint8_t* codes;
  int codes_B;
  const void* norms;
  int norm_dtype;
  const Table* tab;
  int64_t L_cap, chunk;
  const int32_t* len;
  float* logits;     // [B][Hq][L_cap]
};

__host__ __device__ inline size_t score_smem_bytes(int d, int bits1, int G, int codes_B) {
  return sizeof(Table) + (size_t)(d / 2) * (1 << bits1) * G * 4 + (size_t)kSThreads * (codes_B / 4 + 1) * 4;
}

// Field of width b at bit offset o of a row of 32-bit words (LSB-first).
__device__ __forceinline__ uint32_t field(const uint32_t* row, int o, int b) {
  const int w = o >> 5, s = o & 31;
  uint32_t v = row[w] >> s;
  if (s + b > 32) v |= row[w + 1] << (32 - s);
  return v & ((1u << b) - 1u);
}

template <int D>
__global__ void __launch_bounds__(kSThreads) polar_score_kernel(ScoreArgs a) {
  constexpr int NL = (D >= 256) ? 8 : (D >= 128) ? 7 : (D >= 64) ? 6 : 5;   // log2(D)
  constexpr int P1 = D / 2;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = a.Hq / a.Hkv;
  const int b1 = a.lay.bits[0], L1 = 1 << b1;
  Table* tab = reinterpret_cast<Table*>(smem_raw);
  float* T1 = reinterpret_cast<float*>(tab + 1);                   // [P1][L1][G]
  uint32_t* rows = reinterpret_cast<uint32_t*>(T1 + P1 * L1 * G);  // [kSThreads][codes_B / 4 + 1]
  const int rstride = a.codes_B / 4 + 1;
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, b = bh / a.Hkv, hk = bh % a.Hkv, h0 = hk * G;

  for (int i = tid; i < (int)(sizeof(Table) / 4); i += kSThreads)
    reinterpret_cast<float*>(tab)[i] = reinterpret_cast<const float*>(a.tab)[i];
  __syncthreads();
  // level-1 table of the group's queries: T1[p][k][g] = q'_2p cos(theta_k) + q'_2p+1 sin(theta_k)
  for (int i = tid; i < P1 * L1 * G; i += kSThreads) {
    const int g = i % G, k = (i / G) % L1, p = i / (G * L1);
    const float* q = a.qr + ((size_t)b * a.Hq + h0 + g) * D;
    T1[i] = q[2 * p] * tab->cs[0][k] + q[2 * p + 1] * tab->sn[0][k];
  }
  __syncthreads();

  const int64_t L = min((int64_t)max(a.len[b], 0), a.L_cap);
  const int64_t start = (int64_t)blockIdx.y * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  uint32_t* my = rows + tid * rstride;
  for (int64_t base = start; base < end; base += kSThreads) {
    const int64_t i = base + tid;
    if (i < end) {
      const int64_t row = (int64_t)bh * a.L_cap + i;
      const uint4* src = reinterpret_cast<const uint4*>(a.codes + row * (int64_t)a.codes_B);
      for (int w = 0; w < a.codes_B / 16; ++w) {
        const uint4 u = src[w];
        my[4 * w] = u.x;
        my[4 * w + 1] = u.y;
        my[4 * w + 2] = u.z;
        my[4 * w + 3] = u.w;
      }
      float stk[NL][kMaxG];   // left partial score waiting at each level
      float cur[kMaxG];
#pragma unroll
      for (int p = 0; p < P1; ++p) {
        const float* t1 = T1 + (p * L1 + (int)field(my, p * b1, b1)) * G;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) cur[g] = (g < G) ? t1[g] : 0.f;
#pragma unroll
        for (int k = 1; k < NL; ++k) {
          if (((p >> (k - 1)) & 1) == 0) {   // a left child: wait for its sibling
#pragma unroll
            for (int g = 0; g < kMaxG; ++g) stk[k][g] = cur[g];
            break;
          }
          const int bk = a.lay.bits[k];
          const uint32_t ai = field(my, a.lay.off[k] + (p >> k) * bk, bk);
          const float c = tab->cs[k][ai], s = tab->sn[k][ai];
#pragma unroll
          for (int g = 0; g < kMaxG; ++g) cur[g] = fmaf(stk[k][g], c, cur[g] * s);
        }
      }
      const float n = load_norm(a.norms, a.norm_dtype, row);
      for (int g = 0; g < G; ++g) a.logits[((int64_t)b * a.Hq + h0 + g) * a.L_cap + i] = n * cur[g];
    }
  }
}

}  // namespace polar
}  // namespace tqk
