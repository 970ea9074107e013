// Top-k inner-product search over packed database vectors, SIMT version.
//
// "TurboQuant: redefining AI efficiency" (hakusoku.com), section "Impact on
// high-dimensional vector search": nearest-neighbour search runs directly on
// the compressed vectors. Scores are s = ||x|| <Pi q, c[idx]> (queries rotated
// once); ranking: score descending, equal scores by lower index.
//
// One CTA owns a query tile (kSQ queries) and a contiguous chunk of the
// database. For each kSK-key tile it dequantizes the centroid values into
// shared memory one 32-coordinate slice at a time, accumulates the kSQ x kSK
// score tile with an fp32 register-blocked product, and folds the tile into a
// per-query running top-k kept in shared memory. The full score matrix is
// never written; a merge kernel reduces the per-chunk lists.
#pragma once

#include "common.cuh"

namespace tqk {

constexpr int kSQ = 64;
constexpr int kSK = 64;
constexpr int kSearchThreads = 256;
constexpr int kMaxTopK = 64;

struct SearchArgs {
  const float* qr;     // [nq][d] rotated queries
  int nq, d, bits, norm_dtype, codes_B, k;
  const uint8_t* codes;
  const void* norms;
  int64_t n, chunk;
  const float* cent;
  float* cand_s;       // [nchunks][nq][k]
  int64_t* cand_i;     // [nchunks][nq][k]
};

__host__ __device__ inline size_t search_smem_bytes(int k) {
  return (size_t)(32 * kSQ + 32 * kSK + kSQ * (kSK + 1) + 16) * 4 + (size_t)kSQ * k * (4 + 8) + 64;
}

// (s, i) ranks before (t, j): higher score, or equal score and lower index.
__device__ __forceinline__ bool ranks_before(float s, int64_t i, float t, int64_t j) {
  return s > t || (s == t && i < j);
}

__global__ void __launch_bounds__(kSearchThreads) search_simt_kernel(SearchArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Qs = reinterpret_cast<float*>(smem_raw);  // [32][kSQ]
  float* Ks = Qs + 32 * kSQ;                       // [32][kSK]
  float* Ss = Ks + 32 * kSK;                       // [kSQ][kSK+1]
  float* cen = Ss + kSQ * (kSK + 1);               // [16]
  int64_t* topi = reinterpret_cast<int64_t*>(cen + 16);  // [kSQ][k]  (8-byte aligned: offsets are multiples of 8)
  float* tops = reinterpret_cast<float*>(topi + (size_t)kSQ * a.k);  // [kSQ][k]

  const int tid = threadIdx.x;
  const int q0 = blockIdx.y * kSQ;
  const int64_t c0 = (int64_t)blockIdx.x * a.chunk;
  const int64_t c1 = min(a.n, c0 + a.chunk);
  const int d = a.d, K = a.k;
  if (tid < (1 << a.bits)) cen[tid] = a.cent[tid];
  for (int i = tid; i < kSQ * K; i += kSearchThreads) { tops[i] = -INFINITY; topi[i] = -1; }
  __syncthreads();

  const int tr = tid >> 4;  // queries tr*4 .. +3
  const int tc = tid & 15;  // keys tc*4 .. +3
  const int lk = tid >> 2, lc = (tid & 3) * 8;  // loaders: row (query/key) lk, coords lc .. lc+7

  for (int64_t kb = c0; kb < c1; kb += kSK) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    const int64_t key = kb + lk;
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(a.codes + min(key, a.n - 1) * (int64_t)a.codes_B);
    for (int j0 = 0; j0 < d; j0 += 32) {
      const int q = q0 + lk;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        Qs[(lc + e) * kSQ + lk] = (q < a.nq) ? a.qr[(size_t)q * d + j0 + lc + e] : 0.f;
        Ks[(lc + e) * kSK + lk] = (key < c1) ? cen[packed_field(kw, j0 + lc + e, a.bits)] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < 32; ++kk) {
        float qv[4], kv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qv[i] = Qs[kk * kSQ + tr * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) kv[j] = Ks[kk * kSK + tc * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t kk = kb + tc * 4 + j;
      const float nrm = (kk < c1) ? load_norm(a.norms, a.norm_dtype, kk) : 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        Ss[(tr * 4 + i) * (kSK + 1) + tc * 4 + j] = (kk < c1) ? acc[i][j] * nrm : -INFINITY;
    }
    __syncthreads();
    if (tid < kSQ && q0 + tid < a.nq) {
      float* ts = tops + tid * K;
      int64_t* ti = topi + tid * K;
      const int nk = (int)min((int64_t)kSK, c1 - kb);
      for (int j = 0; j < nk; ++j) {
        const float s = Ss[tid * (kSK + 1) + j];
        const int64_t idx = kb + j;
        if (!ranks_before(s, idx, ts[K - 1], ti[K - 1]) && ti[K - 1] >= 0) continue;
        int pos = K - 1;
        while (pos > 0 && (ti[pos - 1] < 0 || ranks_before(s, idx, ts[pos - 1], ti[pos - 1]))) {
          ts[pos] = ts[pos - 1];
          ti[pos] = ti[pos - 1];
          --pos;
        }
        ts[pos] = s;
        ti[pos] = idx;
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < kSQ * K; i += kSearchThreads) {
    const int q = q0 + i / K;
    if (q >= a.nq) continue;
    const size_t o = ((size_t)blockIdx.x * a.nq + q) * K + (i % K);
    a.cand_s[o] = tops[i];
    a.cand_i[o] = topi[i];
  }
}

// Merge the per-chunk lists of one query: one warp per query, a k-way merge of the sorted lists
// (best first; an entry with index < 0 ends a list). Lane l owns lists l, l + 32, ...; their
// read positions live in shared memory and each lane keeps the best current head of its lists.
// Every round the warp picks the best head over the lanes ((score, index): higher score, then
// lower index), writes it, and only the owning lane advances that list and rescans its own.
__global__ void topk_merge_kernel(const float* cand_s, const int64_t* cand_i, int nchunks, int nq, int K,
                                  float* out_s, int64_t* out_i) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int* pos = reinterpret_cast<int*>(smem_raw);   // [nchunks]
  const int q = blockIdx.x, lane = threadIdx.x;
  for (int c = lane; c < nchunks; c += 32) pos[c] = 0;
  __syncwarp();
  auto entry = [&](int c, int r) { return ((size_t)c * nq + q) * K + r; };
  float bs = -INFINITY;
  int64_t bi = -1;
  int bc = -1;
  auto rescan = [&]() {
    bs = -INFINITY, bi = -1, bc = -1;
    for (int c = lane; c < nchunks; c += 32) {
      const int r = pos[c];
      if (r >= K) continue;
      const int64_t i = cand_i[entry(c, r)];
      if (i < 0) continue;
      const float sv = cand_s[entry(c, r)];
      if (bc < 0 || ranks_before(sv, i, bs, bi)) bs = sv, bi = i, bc = c;
    }
  };
  rescan();
  for (int r = 0; r < K; ++r) {
    float ws = bs;
    int64_t wi = bi;
    int wl = bc >= 0 ? lane : 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, ws, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
      const int ol = __shfl_xor_sync(0xffffffffu, wl, o);
      const bool take = ol < 32 && (wl == 32 || ranks_before(os, oi, ws, wi) || (os == ws && oi == wi && ol < wl));
      if (take) ws = os, wi = oi, wl = ol;
    }
    if (lane == 0) {
      out_s[(size_t)q * K + r] = wl < 32 ? ws : -INFINITY;
      out_i[(size_t)q * K + r] = wl < 32 ? wi : -1;
    }
    if (wl == lane) {
      ++pos[bc];
      rescan();
    }
    __syncwarp();
  }
}

}  // namespace tqk
