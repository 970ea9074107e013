// Query preparation, inner-product scores and split-K decode attention over
// packed codes, SIMT version (any bits, any prod/MSE mix, d <= 256).
//
// Scores: s = ||x|| <Pi q, c[idx]> (+ rnorm sqrt(pi/2)/m <S q, 2 sigma - 1> for
// prod) -- "TurboQuant: redefining AI efficiency" (hakusoku.com), section
// "QJL": full-precision query against low-precision data; "Google TurboQuant:
// 6x KV-cache compression" (ebisuda.net), section "Stage 2". The query is
// rotated once (q' = Pi q, q_s = S q), so no key is ever dequantized to the
// original basis.
//
// Attention: softmax(scale * s) V per query head, grouped-query mapping
// h -> h / (Hq / Hkv) ("TurboQuant / PolarQuant / QJL technical deep dive"
// (gemilab.net), section "Scaled dot-product attention"). One CTA handles one
// (sequence, KV head, context chunk) for all query heads of the group: an
// online softmax over 128-key blocks, the value sum kept in the rotated domain
// (acc = sum p ||v|| c[vidx], acc_s = sum p rnorm (2 sigma - 1)); a combine
// kernel merges the chunks by log-sum-exp and maps back once:
// o = (Pi_V^T acc + sqrt(pi/2)/m S_V^T acc_s) / sum p.
#pragma once

#include "common.cuh"
#include "small_kernels.cuh"

namespace tqk {

constexpr int kMaxGroup = 8;      // query heads per KV head
constexpr int kAttnThreads = 128; // keys per block = threads
constexpr int kMaxHeadDim = 256;

// ---------------------------------------------------------------- query prep

// out_r[row][j] = sum_k Pi[j][k] q[row][k];  out_s[row][i] = sum_k S[i][k] q[row][k].
// One CTA per group of up to kQprepRows query rows and 64 output rows of
// [Pi; S]; four threads share an output row, each loading its quarter of the
// matrix row at once (16-byte loads, all in flight), then two shuffles combine
// the quarters. Each loaded element serves every query row of the group.
constexpr int kQprepRows = 8;
__global__ void __launch_bounds__(256) qprep_kernel(const void* q, int q_dtype, int rows, int d, const float* Pi,
                                                    const float* S, int m, float* out_r, float* out_s) {
  extern __shared__ float qsh[];   // [kQprepRows][d]
  const int row0 = blockIdx.x * kQprepRows;
  const int nr = min(kQprepRows, rows - row0);
  const int o = blockIdx.y * 64 + (threadIdx.x >> 2), part = threadIdx.x & 3;
  const int q4 = d / 16;           // float4s per quarter row (d % 32 == 0)
  constexpr int kMaxQ4 = 64;       // d <= 4096
  float4 mv[kMaxQ4 / 8];
  const bool active = o < d + m;
  const float4* mrow = nullptr;
  if (active) {
    mrow = reinterpret_cast<const float4*>((o < d) ? (Pi + (size_t)o * d) : (S + (size_t)(o - d) * d)) + part * q4;
  }
  for (int i = threadIdx.x; i < nr * d; i += blockDim.x) qsh[i] = load_any(q, q_dtype, (int64_t)row0 * d + i);
  __syncthreads();
  float acc[kQprepRows];
#pragma unroll
  for (int r = 0; r < kQprepRows; ++r) acc[r] = 0.f;
  for (int c0 = 0; c0 < q4; c0 += kMaxQ4 / 8) {
    const int nc = min(kMaxQ4 / 8, q4 - c0);
#pragma unroll
    for (int u = 0; u < kMaxQ4 / 8; ++u)
      mv[u] = (active && u < nc) ? mrow[c0 + u] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kMaxQ4 / 8; ++u) {
      if (u >= nc) break;
      const int k = 4 * (part * q4 + c0 + u);
#pragma unroll
      for (int r = 0; r < kQprepRows; ++r) {
        if (r < nr) {
          const float* qq = qsh + r * d + k;
          acc[r] = fmaf(mv[u].x, qq[0], fmaf(mv[u].y, qq[1], fmaf(mv[u].z, qq[2], fmaf(mv[u].w, qq[3], acc[r]))));
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kQprepRows; ++r) {
    acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
    acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 2);
  }
  if (active && part == 0) {
#pragma unroll
    for (int r = 0; r < kQprepRows; ++r) {
      if (r >= nr) break;
      if (o < d)
        out_r[(size_t)(row0 + r) * d + o] = acc[r];
      else
        out_s[(size_t)(row0 + r) * m + (o - d)] = acc[r];
    }
  }
}

// ---------------------------------------------------------------- cache view

struct CacheView {
  const uint8_t* codes;   // NULL for QJL-only rows (bits == 0)
  const uint8_t* signs;
  const void* norms;
  const __half* rnorms;   // NULL for QJL-only rows: the norm weighs the signs
  int bits, m, norm_dtype, codes_B, signs_B;
  const float* cent;
};

// Weight of a row's sign sum: the residual norm (prod), or the norm itself (QJL-only rows,
// whose sketch is of the whole vector: "TurboQuant: redefining AI efficiency", "QJL").
__device__ __forceinline__ float qjl_norm(const CacheView& c, int64_t row) {
  return c.rnorms ? __half2float(c.rnorms[row]) : load_norm(c.norms, c.norm_dtype, row);
}

// MSE and QJL parts of G query scores for one key row (thread-serial over d).
__device__ __forceinline__ void key_scores(const CacheView& c, int64_t row, int d, int G,
                                           const float* qr_s, const float* qs_s, const float* cen,
                                           float* out) {
  float am[kMaxGroup];
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) am[g] = 0.f;
  const uint32_t* cw = c.bits ? reinterpret_cast<const uint32_t*>(c.codes + row * (int64_t)c.codes_B) : nullptr;
  for (int j = 0; c.bits && j < d; ++j) {
    const float cv = cen[packed_field(cw, j, c.bits)];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
      if (g < G) am[g] = fmaf(qr_s[g * d + j], cv, am[g]);
  }
  const float n = load_norm(c.norms, c.norm_dtype, row);
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) out[g] = n * am[g];
  if (c.m > 0) {
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(c.signs + row * (int64_t)c.signs_B);
    float as[kMaxGroup];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) as[g] = 0.f;
    for (int j = 0; j < c.m; ++j) {
      const float pm = sign_bit(sw, j) ? 1.f : -1.f;
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g)
        if (g < G) as[g] = fmaf(qs_s[g * c.m + j], pm, as[g]);
    }
    const float w = qjl_norm(c, row) * (kQjlScale / (float)c.m);
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) out[g] = fmaf(w, as[g], out[g]);
  }
}

// ---------------------------------------------------------------- score

struct ScoreArgs {
  const float* qr;  // [B*Hq][d]
  const float* qs;  // [B*Hq][m]
  int B, Hq, Hkv, d;
  CacheView k;
  int64_t L_cap, chunk;
  const int32_t* len;
  float* logits;    // [B][Hq][L_cap]
};

__global__ void __launch_bounds__(kAttnThreads) score_simt_kernel(ScoreArgs a) {
  extern __shared__ float sm[];
  const int G = a.Hq / a.Hkv;
  const int bh = blockIdx.x;  // b * Hkv + hk
  const int b = bh / a.Hkv, hk = bh % a.Hkv;
  float* qr_s = sm;
  float* qs_s = qr_s + G * a.d;
  float* cen = qs_s + G * a.k.m;
  const int h0 = hk * G;
  for (int i = threadIdx.x; i < G * a.d; i += blockDim.x)
    qr_s[i] = a.qr[((size_t)b * a.Hq + h0) * a.d + i];
  for (int i = threadIdx.x; i < G * a.k.m; i += blockDim.x)
    qs_s[i] = a.qs[((size_t)b * a.Hq + h0) * a.k.m + i];
  if (threadIdx.x < (1 << a.k.bits)) cen[threadIdx.x] = a.k.cent[threadIdx.x];
  __syncthreads();
  const int64_t L = min((int64_t)max(a.len[b], 0), a.L_cap);  // never read past the cache
  const int64_t start = (int64_t)blockIdx.y * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  for (int64_t i = start + threadIdx.x; i < end; i += blockDim.x) {
    float s[kMaxGroup];
    key_scores(a.k, (int64_t)bh * a.L_cap + i, a.d, G, qr_s, qs_s, cen, s);
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
      if (g < G) a.logits[((int64_t)b * a.Hq + h0 + g) * a.L_cap + i] = s[g];
  }
}

// ---------------------------------------------------------------- attention

struct AttnArgs {
  const float* qr;  // K-side rotated queries [B*Hq][d]
  const float* qs;  // K-side S q [B*Hq][mk]
  int B, Hq, Hkv, d;
  CacheView k, v;
  int64_t L_cap, chunk;
  int nsplit;
  const int32_t* len;
  int len_extra;    // 1 inside a decode step: the token appended at slot len[b] counts
  float scale;
  float* part;      // [B*Hq][nsplit][partial_stride(d, mv)]
};

__global__ void __launch_bounds__(kAttnThreads) attn_split_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  grid_dep_launch();
  grid_dep_wait();
  const int G = a.Hq / a.Hkv;
  const int d = a.d, mk = a.k.m, mv = a.v.m;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / a.Hkv, hk = bh % a.Hkv, h0 = hk * G;
  const int tid = threadIdx.x;

  float* qr_s = sm;                       // [G][d]
  float* qs_s = qr_s + G * d;             // [G][mk]
  float* kcen = qs_s + G * mk;            // [16]
  float* vcen = kcen + 16;                // [16]
  float* p_s = vcen + 16;                 // [G][128]
  float* wv_s = p_s + G * kAttnThreads;   // [128] value norms
  float* wr_s = wv_s + kAttnThreads;      // [128] value rnorms
  float* st_s = wr_s + kAttnThreads;      // [G][4]: running max, sum, rescale

  for (int i = tid; i < G * d; i += blockDim.x) qr_s[i] = a.qr[((size_t)b * a.Hq + h0) * d + i];
  for (int i = tid; i < G * mk; i += blockDim.x) qs_s[i] = a.qs[((size_t)b * a.Hq + h0) * mk + i];
  if (tid < (1 << a.k.bits)) kcen[tid] = a.k.cent[tid];
  if (tid < (1 << a.v.bits)) vcen[tid] = a.v.cent[tid];
  if (tid < G) { st_s[tid * 4 + 0] = -INFINITY; st_s[tid * 4 + 1] = 0.f; st_s[tid * 4 + 2] = 1.f; }
  __syncthreads();

  // thread tid owns value coordinates j = tid and tid + 128 (and QJL coords likewise)
  float acc[kMaxGroup][2], accs[kMaxGroup][2];
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) { acc[g][0] = acc[g][1] = 0.f; accs[g][0] = accs[g][1] = 0.f; }

  const int64_t L = min((int64_t)max(a.len[b], 0) + a.len_extra, a.L_cap);  // never read past the cache
  const int64_t start = (int64_t)split * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  const int64_t base = (int64_t)bh * a.L_cap;
  const int warp = tid >> 5, lane = tid & 31;

  for (int64_t sb = start; sb < end; sb += kAttnThreads) {
    const int64_t i = sb + tid;
    float s[kMaxGroup];
    if (i < end) {
      key_scores(a.k, base + i, d, G, qr_s, qs_s, kcen, s);
      wv_s[tid] = load_norm(a.v.norms, a.v.norm_dtype, base + i);
      wr_s[tid] = (mv > 0) ? qjl_norm(a.v, base + i) : 0.f;  // sqrt(pi/2)/m applied in combine
    } else {
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) s[g] = -INFINITY;
      wv_s[tid] = 0.f;
      wr_s[tid] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
      if (g < G) p_s[g * kAttnThreads + tid] = (i < end) ? s[g] * a.scale : -INFINITY;
    __syncthreads();
    // softmax statistics: warp w handles query heads g = w, w + 4, ...
    for (int g = warp; g < G; g += kAttnThreads / 32) {
      float* pg = p_s + g * kAttnThreads;
      float mx = -INFINITY;
      for (int t = lane; t < kAttnThreads; t += 32) mx = fmaxf(mx, pg[t]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mold = st_s[g * 4 + 0];
      const float mnew = fmaxf(mold, mx);
      float sum = 0.f;
      for (int t = lane; t < kAttnThreads; t += 32) {
        const float p = (pg[t] == -INFINITY) ? 0.f : __expf(pg[t] - mnew);
        pg[t] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float alpha = (mold == -INFINITY) ? 0.f : __expf(mold - mnew);
        st_s[g * 4 + 0] = mnew;
        st_s[g * 4 + 1] = st_s[g * 4 + 1] * alpha + sum;
        st_s[g * 4 + 2] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
      if (g < G) {
        const float alpha = st_s[g * 4 + 2];
        acc[g][0] *= alpha; acc[g][1] *= alpha; accs[g][0] *= alpha; accs[g][1] *= alpha;
      }
    }
    const int nk = (int)min((int64_t)kAttnThreads, end - sb);
    for (int t = 0; t < nk; ++t) {
      const int64_t row = base + sb + t;
      const uint32_t* vw = a.v.bits ? reinterpret_cast<const uint32_t*>(a.v.codes + row * (int64_t)a.v.codes_B) : nullptr;
      const float wn = wv_s[t];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int j = tid + r * kAttnThreads;
        if (j < d && a.v.bits) {   // QJL-only values have no MSE part
          const float cv = vcen[packed_field(vw, j, a.v.bits)] * wn;
#pragma unroll
          for (int g = 0; g < kMaxGroup; ++g)
            if (g < G) acc[g][r] = fmaf(p_s[g * kAttnThreads + t], cv, acc[g][r]);
        }
      }
      if (mv > 0) {
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.v.signs + row * (int64_t)a.v.signs_B);
        const float wr = wr_s[t];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int j = tid + r * kAttnThreads;
          if (j < mv) {
            const float pm = sign_bit(sw, j) ? wr : -wr;
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g)
              if (g < G) accs[g][r] = fmaf(p_s[g * kAttnThreads + t], pm, accs[g][r]);
          }
        }
      }
    }
    __syncthreads();
  }

  const int stride = partial_stride(d, mv);
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) {
    if (g >= G) break;
    float* out = a.part + (((size_t)b * a.Hq + h0 + g) * a.nsplit + split) * stride;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = tid + r * kAttnThreads;
      if (j < d) out[j] = acc[g][r];
      if (j < mv) out[d + j] = accs[g][r];
    }
    if (tid == 0) { out[d + mv] = st_s[g * 4 + 0]; out[d + mv + 1] = st_s[g * 4 + 1]; }
  }
}

struct CombineArgs {
  const float* part;  // [B*Hq][nsplit][partial_stride(d, mv)]
  int Hq, Hkv, nsplit, d, mv;
  const float* PiV;   // [d][d] row-major
  const float* SV;    // [mv][d] row-major
  float* out;         // [B*Hq][d]
};

constexpr int kCombineThreads = 1024;

// One CTA per (sequence, query head). Thread (j, part) first issues its loads
// of an eighth of column j of [Pi_V; sqrt(pi/2)/m S_V] (so they travel while the
// chunk weights are merged), then:
// 1) log-sum-exp weights of the chunks (warp 0);
// 2) merged rotated-domain sums acc (d) and QJL sums (mv), two threads per entry;
// 3) o_j = (sum_k Pi_V[k][j] acc_k + sqrt(pi/2)/m sum_k S_V[k][j] acc_s_k) / sum p.
__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(CombineArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, mv = a.mv, stride = partial_stride(d, mv), dm = d + mv;
  const int row = blockIdx.x;                   // b * Hq + h
  float* w = sm;                                // [nsplit]
  float* acc = w + a.nsplit;                    // [2][d + mv] (two halves of the splits)
  float* part_o = acc + 2 * dm;                 // [8][d]
  float* Ls = part_o + 8 * d;                   // [1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float qscale = (mv > 0) ? kQjlScale / (float)mv : 0.f;
  constexpr int kMaxRows = 32;                  // per part: (d + mv) / 8 <= 32 (d + mv <= 256)
  const int quarter = tid >> 7, j = tid & 127;  // quarter = part 0..7
  const int kq = (dm + 7) / 8, k0 = quarter * kq, k1 = min(dm, k0 + kq);
  float mcol[kMaxRows];
#pragma unroll
  for (int u = 0; u < kMaxRows; ++u) {
    const int k = k0 + u;
    float v = 0.f;
    if (j < d && k < k1) v = (k < d) ? a.PiV[(size_t)k * d + j] : qscale * a.SV[(size_t)(k - d) * d + j];
    mcol[u] = v;
  }
  const float* p = a.part + (size_t)row * a.nsplit * stride;
  if (warp == 0) {
    float M = -INFINITY;
    for (int s = lane; s < a.nsplit; s += 32) M = fmaxf(M, p[(size_t)s * stride + dm]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    for (int s = lane; s < a.nsplit; s += 32) {
      const float ms = p[(size_t)s * stride + dm];
      const float ws = (ms == -INFINITY) ? 0.f : __expf(ms - M);
      w[s] = ws;
      Lsum += ws * p[(size_t)s * stride + dm + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if (lane == 0) Ls[0] = Lsum;
  }
  __syncthreads();
  for (int i = tid; i < 2 * dm; i += blockDim.x) {
    const int half = i / dm, jj = i % dm;
    const int s0 = half * ((a.nsplit + 1) / 2), s1 = half ? a.nsplit : (a.nsplit + 1) / 2;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int s = s0;
    for (; s + 8 <= s1; s += 8) {   // 8 independent loads in flight
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = p[(size_t)(s + u) * stride + jj];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = fmaf(w[s + u], x[u], v[u]);
    }
    for (; s < s1; ++s) v[0] = fmaf(w[s], p[(size_t)s * stride + jj], v[0]);
    acc[i] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
  }
  __syncthreads();
  if (j < d) {
    float o = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxRows; ++u) {
      const int k = k0 + u;
      if (k < k1) o = fmaf(mcol[u], acc[k] + acc[dm + k], o);
    }
    part_o[quarter * d + j] = o;
  }
  __syncthreads();
  for (int i = tid; i < d; i += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) v += part_o[q * d + i];
    const float L = Ls[0];
    a.out[(size_t)row * d + i] = (L > 0.f) ? v / L : 0.f;
  }
}

}  // namespace tqk
