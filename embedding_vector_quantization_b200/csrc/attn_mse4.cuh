// Decode attention over 4-bit MSE K and V caches at d = 128 with 4 query heads per KV
// head, on int8 tensor-core MMAs (mma.sync m16n8k32) fed by TMA bulk copies.
//
// Computes tq_attn_decode's definition ("TurboQuant / PolarQuant / QJL technical deep
// dive" (gemilab.net), "Scaled dot-product attention"; "Google TurboQuant: 6x KV-cache
// compression" (ebisuda.net), "Stage 1"): s = n_k <q', c[idx]>, softmax over the chunk,
// rotated-domain value sums sum_i p_i n_v,i c[vidx_i]. Only the arithmetic is rearranged:
//
//  * A symmetric 16-level codebook written in the +-1 variables s_i = 2 b_i - 1 of its four
//    index bits has only odd-degree Walsh terms, so c[idx] = c[0] + sum_S w_S beta_S(idx)
//    over eight 0/1 planes: the four bits b_i and the four three-bit parities
//    b_i ^ b_j ^ b_k. A packed 4-bit word gives every plane of its 8 coordinates with
//    shifts and one 3-input XOR; (plane >> 0) & 0x01010101 holds the low-nibble
//    coordinates of 4 bytes, & 0x10101010 the high-nibble ones (value 16).
//  * Keys (MMA rows): sum_S w_S <q', beta_S> with w_S q' rounded to 22-bit integers
//    against one step per head and split into int8 pieces hi * 2^14 + mid * 2^7 + lo
//    (n tile 0: hi and mid of the 4 heads; n tile 1: lo at columns 2h), so all planes
//    accumulate exactly into int32 sums per piece.
//  * Values (bit rows of the codes as MMA rows, tokens as the reduction): per-plane
//    integer sums of the softmax weights p n_v rounded to 16 bits against the chunk
//    maximum (unsigned 8-bit hi/lo pieces, u8 x u8 MMAs), combined with w_S once per chunk.
//  * Two passes per chunk as in attn_mma.cuh: all key blocks (exact chunk maximum), then
//    all value blocks with one weight scale.
//
// Partials use the split kernel's layout ([B*Hq][nsplit][partial_stride(128, 0)]:
// rotated-domain value sum, max, sum of weights) and are merged by the combine kernel.
#pragma once

#include "attn_mma.cuh"

namespace tqk {
namespace am4 {

using amma::exp2_approx;
using amma::ldsm_t8_x2;
using amma::ldsm_x4;
using amma::mbar_expect_tx;
using amma::mbar_init;
using amma::mbar_wait;
using amma::mma_s8;
using amma::mma_u8;
using amma::smem_u32;
using amma::tma_bulk_g2s;

constexpr int kD = 128;
constexpr int kG = 4;
constexpr int kBlk = 256;
constexpr int kStages = 4;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCodesB = 64;
constexpr int kStageCodes = kBlk * kCodesB;              // 16384
constexpr int kStageBytes = kStageCodes + 2 * kBlk * 2;  // + key norms + value norms: 17408
constexpr int kMaxChunk = 1024;
constexpr int kPlanes = 8;   // {0}, {1}, {2}, {3}, {0,1,2}, {0,1,3}, {0,2,3}, {1,2,3}

struct Args {
  const float* qr;  // [B*Hq][128] Pi_K q
  int B, Hq, Hkv;
  const uint8_t* kcodes;
  const __half* knorm;
  const uint8_t* vcodes;
  const __half* vnorm;
  int64_t L_cap, chunk;
  int nsplit;
  const int32_t* len;
  int len_extra;           // 1 inside a decode step: the token appended at slot len[b] counts
  float kc0, kw[kPlanes];  // K codebook: c[idx] = kc0 + sum_S kw[S] beta_S(idx)
  float vc0, vw[kPlanes];  // V codebook
  float scale;
  float* part;             // [B*Hq][nsplit][partial_stride(128, 0)]
  int* err;
};

struct __align__(16) Smem {
  unsigned char stage[kStages][kStageBytes];
  float logits[kG][kMaxChunk];     // key pass output: scaled logits in log2 units [head][token]
  uint32_t qfrag[2][32][4][8][2];  // key-side B fragments [n tile][k-step][quad index t][column g][register]
  uint8_t pw[2][8][kBlk];          // integer weights of a value block, double buffered [buf][col][token]
  float acc[kG][kD];               // value sums by coordinate (rotated domain), before the scale
  float qconst[kG][2];             // c0 sum(q'), integer step of the query pieces
  float red_f[kWarps][kG];
  float hmax[kG];
  float dv[kG];                    // weight step per head: max_t p_t ||v_t|| / 65535
  float red_w[kWarps][kG];         // per warp: max_t (logit + log2 ||v_t||)
  int red_i[kWarps][kG];
  __half vnorm[kMaxChunk];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort_flag;
};

// Plane S of every nibble of a packed word, at bit 0 (low nibble) and bit 4 (high nibble).
template <int S>
__device__ __forceinline__ uint32_t plane(uint32_t x) {
  const uint32_t x1 = x >> 1, x2 = x >> 2, x3 = x >> 3;
  if (S == 0) return x;
  if (S == 1) return x1;
  if (S == 2) return x2;
  if (S == 3) return x3;
  if (S == 4) return x ^ x1 ^ x2;
  if (S == 5) return x ^ x1 ^ x3;
  if (S == 6) return x ^ x2 ^ x3;
  return x1 ^ x2 ^ x3;
}

// Where the query value of coordinate c, plane S sits in the B fragments: k-step
// (2 S + nibble) * 2 + half, k index = byte within the half (c = 2 byte + nibble).
__device__ __forceinline__ int qfrag_offset(int S, int c) {
  const int byte = c >> 1, nu = c & 1, h = byte >> 5, kb = byte & 31;
  const int kk = (S * 2 + nu) * 2 + h, slot = kb >> 4, t = (kb & 15) >> 2, e = kb & 3;
  return (((kk * 4 + t) * 8) * 2 + slot) * 4 + e;   // byte offset for column g = 0
}

// Query pieces of heads h0 .. h0 + 3 (warps 0..3, one head each): w_S q'_c rounded to
// 22-bit integers against max |w_S q'_c| and split into int8 pieces hi * 2^14 + mid * 2^7 + lo
// in B-fragment order (n tile 0: column 2h = hi, 2h + 1 = mid; n tile 1: column 2h = lo).
__device__ __forceinline__ void prepare_query4(const float* qr_rows, const float* kw, float kc0,
                                               uint32_t (&qfrag)[2][32][4][8][2], float (&qconst)[kG][2]) {
  const int lane = threadIdx.x & 31, h = threadIdx.x >> 5;
  if (h >= kG) return;
  const float* qr = qr_rows + (size_t)h * kD;
  float q[4], sq = 0.f, mq = 0.f, mw = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[i] = qr[lane + 32 * i];
    sq += q[i];
    mq = fmaxf(mq, fabsf(q[i]));
  }
#pragma unroll
  for (int S = 0; S < kPlanes; ++S) mw = fmaxf(mw, fabsf(kw[S]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
  }
  const float mx = mq * mw;
  const float dq = mx > 0.f ? mx / amma::kQMax : 1.f;
  int8_t* qf0 = reinterpret_cast<int8_t*>(&qfrag[0][0][0][0][0]);
  int8_t* qf1 = reinterpret_cast<int8_t*>(&qfrag[1][0][0][0][0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = lane + 32 * i;
#pragma unroll
    for (int S = 0; S < kPlanes; ++S) {
      const int xi = __float2int_rn(kw[S] * q[i] / dq);                      // |xi| <= 127 * 2^14
      const int hi = (xi >= 0) ? (xi + 8192) >> 14 : -((-xi + 8192) >> 14);  // |hi| <= 127
      const int r = xi - hi * 16384;                                         // |r| <= 2^13
      const int mid = (r >= 0) ? (r + 64) >> 7 : -((-r + 64) >> 7);         // |mid| <= 64
      const int off = qfrag_offset(S, c);
      qf0[off + (2 * h) * 8] = (int8_t)hi;
      qf0[off + (2 * h + 1) * 8] = (int8_t)mid;
      qf1[off + (2 * h) * 8] = (int8_t)(r - 128 * mid);                      // |lo| <= 64
      qf1[off + (2 * h + 1) * 8] = 0;
    }
  }
  if (lane == 0) {
    qconst[h][0] = kc0 * sq;
    qconst[h][1] = dq;
  }
}

// Raw scores n_k <q', c[idx]> of keys kbase + g, kbase + g + 8 (m-tile 0) and kbase + 128 + g,
// kbase + 136 + g (m-tile 1) of a staged key block, for query head t = lane % 4.
template <int S>
__device__ __forceinline__ void key_plane(const uint32_t (&cw)[2][8], const uint32_t (&qfrag)[2][32][4][8][2],
                                          int (&a1)[2][4], int (&a16)[2][4], int (&l1)[2][4], int (&l16)[2][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t p[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) p[mt][i] = plane<S>(cw[mt][4 * h + i]);
#pragma unroll
    for (int nu = 0; nu < 2; ++nu) {
      const int kk = (S * 2 + nu) * 2 + h;
      const uint2 b = *reinterpret_cast<const uint2*>(&qfrag[0][kk][t][g][0]);
      const uint2 bl = *reinterpret_cast<const uint2*>(&qfrag[1][kk][t][g][0]);
      const uint32_t m = nu ? 0x10101010u : 0x01010101u;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        // words: p[0] = key g word t, p[1] = key g word 4+t, p[2] = key g+8 word t, p[3] = key g+8 word 4+t
        int(&acc)[4] = nu ? a16[mt] : a1[mt];
        int(&accl)[4] = nu ? l16[mt] : l1[mt];
        const uint32_t x0 = p[mt][0] & m, x1 = p[mt][2] & m, x2 = p[mt][1] & m, x3 = p[mt][3] & m;
        mma_s8(acc, x0, x1, x2, x3, b.x, b.y);
        mma_s8(accl, x0, x1, x2, x3, bl.x, bl.y);
      }
    }
  }
}

__device__ __forceinline__ void key_scores4(const unsigned char* st, const __half* nrm, int kbase,
                                            const uint32_t (&qfrag)[2][32][4][8][2], float c0h, float dqh,
                                            float (&sc)[2][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2;
  uint32_t cw[2][8];
  {
    const int mat = lane >> 3, r = lane & 7;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int key = kbase + 128 * mt + r + 8 * (mat >> 1);
      uint32_t w4[4];
      ldsm_x4(w4, st + key * kCodesB + 16 * (mat & 1));
      cw[mt][0] = w4[0]; cw[mt][1] = w4[1]; cw[mt][2] = w4[2]; cw[mt][3] = w4[3];
      ldsm_x4(w4, st + key * kCodesB + 32 + 16 * (mat & 1));
      cw[mt][4] = w4[0]; cw[mt][5] = w4[1]; cw[mt][6] = w4[2]; cw[mt][7] = w4[3];
    }
  }
  // per m-tile: the x1 and the x16 families of n tile 0 (hi, mid) and n tile 1 (lo)
  int a1[2][4] = {}, a16[2][4] = {}, l1[2][4] = {}, l16[2][4] = {};
  key_plane<0>(cw, qfrag, a1, a16, l1, l16);
  key_plane<1>(cw, qfrag, a1, a16, l1, l16);
  key_plane<2>(cw, qfrag, a1, a16, l1, l16);
  key_plane<3>(cw, qfrag, a1, a16, l1, l16);
  key_plane<4>(cw, qfrag, a1, a16, l1, l16);
  key_plane<5>(cw, qfrag, a1, a16, l1, l16);
  key_plane<6>(cw, qfrag, a1, a16, l1, l16);
  key_plane<7>(cw, qfrag, a1, a16, l1, l16);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {  // r = 0: key g, r = 1: key g + 8
      const int key = kbase + 128 * mt + g + 8 * r;
      const int hi = 2 * r, md = 2 * r + 1;
      // the hi sum times 2^14 is formed in float (exact: |sum| < 2^17); the rest is exact in int32
      const int phi = a1[mt][hi] + (a16[mt][hi] >> 4);
      const int rest = 128 * (a1[mt][md] + (a16[mt][md] >> 4)) + l1[mt][hi] + (l16[mt][hi] >> 4);
      const float dot = 16384.f * (float)phi + (float)rest;
      sc[mt][r] = __half2float(nrm[key]) * (c0h + dqh * dot);
    }
}

// Value side: this warp's integer weight sums per (plane, nibble) over the 32 tokens
// tk .. tk + 31 for bytes 16 bg + g and 16 bg + g + 8 of the code rows.
template <int S>
__device__ __forceinline__ void value_plane(const uint32_t (&r)[4], uint32_t b0, uint32_t b1, int (&vacc)[kPlanes][2][4]) {
  const uint32_t p0 = plane<S>(r[0]), p1 = plane<S>(r[1]), p2 = plane<S>(r[2]), p3 = plane<S>(r[3]);
  mma_u8(vacc[S][0], p0 & 0x01010101u, p1 & 0x01010101u, p2 & 0x01010101u, p3 & 0x01010101u, b0, b1);
  mma_u8(vacc[S][1], p0 & 0x10101010u, p1 & 0x10101010u, p2 & 0x10101010u, p3 & 0x10101010u, b0, b1);
}

__global__ void __launch_bounds__(kThreads, 2) attn_mse4_kernel(Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / a.Hkv, hk = bh % a.Hkv, h0 = hk * kG;

  const int64_t L = min((int64_t)max(a.len[b], 0) + a.len_extra, a.L_cap);
  const int64_t start = (int64_t)split * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  const int ntok = (int)max((int64_t)0, end - start);
  const int nblk = (ntok + kBlk - 1) / kBlk;
  const int64_t row0 = (int64_t)bh * a.L_cap + start;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  for (int i = tid; i < kG * kD; i += kThreads) (&sm.acc[0][0])[i] = 0.f;
  if (tid < kG) sm.dv[tid] = 1.f;   // an empty chunk keeps unit steps (its sums are 0)
  __syncthreads();

  auto issue = [&](int j) {  // job j: key block j (j < nblk) or value block j - nblk
    const bool kside = j < nblk;
    const int jj = kside ? j : j - nblk;
    const int64_t tok0 = (int64_t)jj * kBlk;
    const int ncopy = (int)min((int64_t)kBlk, a.L_cap - (start + tok0));   // multiple of 8 (L_cap % 8 == 0)
    const int64_t r = row0 + tok0;
    unsigned char* st = sm.stage[j % kStages];
    uint64_t* bar = &sm.full[j % kStages];
    mbar_expect_tx(bar, (uint32_t)ncopy * (kCodesB + (kside ? 4 : 0)));
    tma_bulk_g2s(st, (kside ? a.kcodes : a.vcodes) + r * kCodesB, ncopy * kCodesB, bar);
    if (kside) {
      tma_bulk_g2s(st + kStageCodes, a.knorm + r, ncopy * 2, bar);
      tma_bulk_g2s(st + kStageCodes + 2 * kBlk, a.vnorm + r, ncopy * 2, bar);
    }
  };
  const int njobs = 2 * nblk;
  constexpr int kAhead = kStages - 2;
  grid_dep_launch();
  // in a decode step the kernel before this one writes only slot len[b] and the queries
  const int64_t slot = (int64_t)max(a.len[b], 0);
  const bool holds_new = a.len_extra && slot >= start && slot < start + a.chunk;
  if (holds_new) grid_dep_wait();
  if (tid == 0)
    for (int j = 0; j < min(kAhead, njobs); ++j) issue(j);
  if (!holds_new) grid_dep_wait();

  prepare_query4(a.qr + ((size_t)b * a.Hq + h0) * kD, a.kw, a.kc0, sm.qfrag, sm.qconst);
  __syncthreads();
  const float c0h = sm.qconst[t][0], dqh = sm.qconst[t][1];
  const float scale2 = a.scale * 1.4426950408889634f;
  float run_max = -INFINITY, wv_max = -INFINITY;   // wv_max: log2 of the largest p ||v|| of head t
  float lsum = 0.f;
  int wsum = 0;
  const int bg = warp & 3, half = warp >> 2;   // value side: 16-byte group of the code rows, token half
  int issued = min(kAhead, njobs);
  // start of job j: refill the stage of job j - 2 once every warp has released it, then wait
  // for job j's copy (no warp ever leaves early: a wait that runs out sets abort_flag, after
  // which nothing is issued or waited for and every warp still meets the same barriers)
  auto begin_job = [&](int j) {
    const bool aborted = *(volatile int*)&sm.abort_flag != 0;
    if (tid == 0 && !aborted && j + kAhead < njobs) {
      const int jo = j + kAhead - kStages;
      if (jo >= 0 && !mbar_wait(&sm.empty[jo % kStages], (jo / kStages) & 1)) {
        sm.abort_flag = 1;
      } else {
        issue(j + kAhead);
        issued = j + kAhead + 1;
      }
    }
    if (!aborted && !mbar_wait(&sm.full[j % kStages], (j / kStages) & 1)) sm.abort_flag = 1;
  };
  auto end_job = [&](int j) {
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&sm.empty[j % kStages])) : "memory");
  };

  // ---------------- key pass: warp w scores keys 16w .. 16w+15 and 128+16w .. of every block
  for (int j = 0; j < nblk; ++j) {
    begin_job(j);
    const unsigned char* st = sm.stage[j % kStages];
    const int tok_base = j * kBlk;
    const int nvalid = min(kBlk, ntok - tok_base);
    const __half* nrm = reinterpret_cast<const __half*>(st + kStageCodes);
    float sc[2][2];
    key_scores4(st, nrm, 16 * warp, sm.qfrag, c0h, dqh, sc);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int key = 128 * mt + 16 * warp + g + 8 * r;
        const float v = (key < nvalid) ? sc[mt][r] * scale2 : -INFINITY;   // log2 units
        sm.logits[t][tok_base + key] = v;
        run_max = fmaxf(run_max, v);
        wv_max = fmaxf(wv_max, v + __log2f(__half2float(nrm[kBlk + key])));   // its weight exp2(v - max) ||v||
      }
    // value norms of these tokens came with the key block: keep them for the value pass
    if (tid < kBlk) sm.vnorm[tok_base + tid] = nrm[kBlk + tid];
    end_job(j);
  }

  // ---------------- between the passes: chunk maxima and the value weight scale
  if (nblk > 0) {
    __syncthreads();
    float m = run_max;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (g == 0) sm.red_f[warp][t] = m;
    float wv = wv_max;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) wv = fmaxf(wv, __shfl_xor_sync(0xffffffffu, wv, o));
    if (g == 0) sm.red_w[warp][t] = wv;
    __syncthreads();
    if (tid < kG) {
      float mm = -INFINITY, mv = -INFINITY;
      for (int w = 0; w < kWarps; ++w) {
        mm = fmaxf(mm, sm.red_f[w][tid]);
        mv = fmaxf(mv, sm.red_w[w][tid]);
      }
      sm.hmax[tid] = mm;
      // 16-bit weights per head against the head's largest weight (a hair above it, so that the
      // approximate exp2 / log2 cannot push the largest weight past 65535)
      const float s1 = exp2_approx(mv - mm) * (1.f + 1.f / 4096.f) / 65535.f;
      sm.dv[tid] = (s1 > 0.f && s1 < INFINITY) ? s1 : 1.f;
    }
    __syncthreads();
  }

  // ---------------- value pass: integer weights of each block (all threads), then MMAs
  int vacc[kPlanes][2][4];
#pragma unroll
  for (int S = 0; S < kPlanes; ++S)
#pragma unroll
    for (int nu = 0; nu < 2; ++nu) vacc[S][nu][0] = vacc[S][nu][1] = vacc[S][nu][2] = vacc[S][nu][3] = 0;
  for (int j = nblk; j < njobs; ++j) {
    begin_job(j);
    const int jj = j - nblk;
    const unsigned char* st = sm.stage[j % kStages];
    const int tok_base = jj * kBlk;
    const int nvalid = min(kBlk, ntok - tok_base);
    {
      {
        const int h = tid & 3, q4 = (tid >> 2) * 4;
        const float hm = sm.hmax[h], inv1 = 1.f / sm.dv[h];
        const float4 l4 = *reinterpret_cast<const float4*>(&sm.logits[h][tok_base + q4]);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
        uint32_t w1h = 0, w1l = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q4 + q < nvalid) {
            const float p = exp2_approx(lv[q] - hm);
            const int w1 = min(__float2int_rn(p * __half2float(sm.vnorm[tok_base + q4 + q]) * inv1), 65535);
            w1h |= (uint32_t)(w1 >> 8) << (8 * q);
            w1l |= (uint32_t)(w1 & 255) << (8 * q);
            lsum += p;
            wsum += w1;
          }
        }
        uint8_t* blk = &sm.pw[jj & 1][0][0];
        *reinterpret_cast<uint32_t*>(blk + (2 * h) * kBlk + q4) = w1h;
        *reinterpret_cast<uint32_t*>(blk + (2 * h + 1) * kBlk + q4) = w1l;
      }
      __syncthreads();
      const uint8_t* pw = &sm.pw[jj & 1][0][0];
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const int tk = 128 * half + 32 * kq;   // first token of this 32-token k-step
        uint32_t r[4];
        const int tok = tk + (lane & 15) + 16 * (lane >> 4);
        ldsm_t8_x2(r, st + tok * kCodesB + 16 * bg);
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(pw + g * kBlk + tk + 4 * t);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(pw + g * kBlk + tk + 16 + 4 * t);
        value_plane<0>(r, b0, b1, vacc);
        value_plane<1>(r, b0, b1, vacc);
        value_plane<2>(r, b0, b1, vacc);
        value_plane<3>(r, b0, b1, vacc);
        value_plane<4>(r, b0, b1, vacc);
        value_plane<5>(r, b0, b1, vacc);
        value_plane<6>(r, b0, b1, vacc);
        value_plane<7>(r, b0, b1, vacc);
      }
    }
    end_job(j);
  }

  __syncthreads();
  if (sm.abort_flag) {
    if (tid == 0) {
      report_error(a.err, kErrTimeout);
      for (int jx = max(0, issued - kStages); jx < issued; ++jx)
        (void)mbar_wait(&sm.full[jx % kStages], (jx / kStages) & 1);
    }
    __syncthreads();
    return;
  }
  {  // sums of p and of the integer weights per head (threads with lane % 4 == head)
    float l = lsum;
    int w1 = wsum;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      w1 += __shfl_xor_sync(0xffffffffu, w1, o);
    }
    if (lane < kG) {
      sm.red_f[warp][lane] = l;
      sm.red_i[warp][lane] = w1;
    }
  }
  // value sums: plane sums of bytes 16 bg + g (+ 8), head t, combined with w_S; the two
  // token halves add into the shared per-coordinate sums (coordinate = 2 byte + nibble)
  {
    float cs[2][2] = {{0.f, 0.f}, {0.f, 0.f}};   // [row g / g+8][nibble]
#pragma unroll
    for (int S = 0; S < kPlanes; ++S)
#pragma unroll
      for (int nu = 0; nu < 2; ++nu) {
        const int f = nu ? 4 : 0;
        const float v0 = 256.f * (float)(vacc[S][nu][0] >> f) + (float)(vacc[S][nu][1] >> f);
        const float v1 = 256.f * (float)(vacc[S][nu][2] >> f) + (float)(vacc[S][nu][3] >> f);
        cs[0][nu] = fmaf(a.vw[S], v0, cs[0][nu]);
        cs[1][nu] = fmaf(a.vw[S], v1, cs[1][nu]);
      }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int nu = 0; nu < 2; ++nu) atomicAdd(&sm.acc[t][2 * (16 * bg + g + 8 * r) + nu], cs[r][nu]);
  }
  __syncthreads();
  const int stride = partial_stride(kD, 0);
  for (int i = tid; i < kG * kD; i += kThreads) {
    const int h = i / kD, c = i % kD;
    int W = 0;
    for (int w = 0; w < kWarps; ++w) W += sm.red_i[w][h];
    a.part[(((size_t)b * a.Hq + h0 + h) * a.nsplit + split) * stride + c] = sm.dv[h] * (a.vc0 * (float)W + sm.acc[h][c]);
  }
  if (tid < kG) {
    float l = 0.f;
    for (int w = 0; w < kWarps; ++w) l += sm.red_f[w][tid];
    float* o = a.part + (((size_t)b * a.Hq + h0 + tid) * a.nsplit + split) * stride;
    o[kD] = (ntok > 0) ? sm.hmax[tid] * 0.6931471805599453f : -INFINITY;   // natural-log units
    o[kD + 1] = (ntok > 0) ? l : 0.f;
  }
}

}  // namespace am4
}  // namespace tqk
