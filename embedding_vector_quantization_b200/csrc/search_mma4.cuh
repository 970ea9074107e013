// Top-k inner-product search over 4-bit MSE codes on int8 tensor-core MMAs.
//
// "TurboQuant: redefining AI efficiency" (hakusoku.com), "Impact on high-dimensional
// vector search": scores s = ||x|| <Pi q, c[idx]>, ranked by score (equal scores: lower
// index first). A symmetric 16-level codebook written in the +-1 variables of its four index
// bits has only odd-degree Walsh terms, c[idx] = c[0] + sum_S w_S beta_S(idx) over eight 0/1
// planes (the four bits and the four three-bit parities; attn_mse4.cuh forms them the same
// way), so
//   <q', c[idx]> = c[0] sum(q') + sum_S <w_S q', beta_S>,
// eight 0/1 bit-plane dot products. Database vectors are the MMA rows, queries the columns:
// each coordinate's eight plane values w_S q'_c are rounded to 15-bit integers against one
// step per query and split into int8 hi/lo pieces, so every dot product accumulates exactly
// in int32 (one accumulator for the low-nibble coordinates, one for the high-nibble ones,
// whose mask leaves the bit at value 16).
//
// One CTA owns 4 queries (one MMA column tile of 4 queries x hi/lo; their fragments take
// 16 d bytes of shared memory, 24 KB per query at d = 1536, in lane order) and a contiguous
// chunk of the database in blocks of 256 vectors, which arrive as d / 256 column slices of 128
// bytes per row (2-D TMA tiles with the 128-byte swizzle, one slice per stage of a 3-stage
// ring). Warp w scores vectors 32w .. 32w+31 of a block (two MMA row tiles); warps 0..3 keep
// the running top-k (k <= 32) of one query each, one list entry per lane. topk_merge_kernel
// reduces the per-chunk lists.
#pragma once

#include <cuda.h>

#include "attn_mse4.cuh"
#include "search_mma.cuh"

namespace tqk {
namespace sm4 {

using amma::ldsm_x4;
using amma::mbar_expect_tx;
using amma::mbar_init;
using amma::mbar_wait;
using amma::mma_s8;
using amma::smem_u32;
using am4::plane;
using sm2::before;
using sm2::list_insert;

constexpr int kQT = 4;           // queries per CTA (one MMA column tile of 4 queries x hi/lo)
constexpr int kVB = 256;         // vectors per block (two 16-row MMA tiles per warp)
constexpr int kStages = 3;       // slice stages
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxD = 1536;      // codes_B = d / 2 <= 768
constexpr int kMaxCodesB = kMaxD / 2;
constexpr int kMaxK = 32;        // one list entry per lane
constexpr int kPlanes = 8;
constexpr int kMaxSteps = kMaxCodesB / 32 * kPlanes * 2;   // k-steps: 32-byte chunks x planes x nibbles
constexpr int kSlice = 128;                                // bytes of a code row per TMA slice
constexpr int kSliceBytes = kVB * kSlice;                  // 32 KB

struct Args {
  const float* qr;       // [nq][d] rotated queries
  int nq, d, codes_B, k, norm_dtype;
  const void* norms;     // [n]
  int64_t n, chunk;
  float c0, w[kPlanes];  // c[idx] = c0 + sum_S w[S] beta_S(idx)
  float* cand_s;         // [nchunks][nq][k]
  int64_t* cand_i;       // [nchunks][nq][k]
  int* err;
};

struct __align__(1024) Smem {
  unsigned char stage[kStages][kSliceBytes];   // 128-byte column slices of a block's code rows, swizzled
  uint32_t qfrag[kMaxSteps][8][4][2];          // [k-step][column g][quad t][register]
  float sc[kQT][kVB + 8];                      // a block's scores [query][vector]
  float qc0[kQT], qstep[kQT];                  // c0 sum(q'), integer step of the query pieces
  uint64_t full[kStages];
  uint64_t empty[kStages];   // one arrival per warp when it is done with the slice
  int abort_flag;
};

// Dynamic shared memory to request: the Smem block plus room to align it to 1024 bytes.
__host__ __device__ inline size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Where the value of coordinate c, plane S sits: byte c / 2 of the code row (chunk byte / 32,
// k index byte % 32), nibble c % 2 -> k-step (chunk * 8 + S) * 2 + nibble. Byte offset for
// column g = 0 (column g adds 32 g).
__device__ __forceinline__ int q_offset(int c, int S) {
  const int byte = c >> 1, nu = c & 1, kk = ((byte >> 5) * kPlanes + S) * 2 + nu;
  const int kb = byte & 31, slot = kb >> 4, t = (kb & 15) >> 2, e = kb & 3;
  return ((((kk * 8) * 4 + t) * 2 + slot) * 4) + e;
}

// The 16 MMAs of plane S of one 32-byte chunk: both row tiles, both nibble families.
template <int S>
__device__ __forceinline__ void chunk_plane(const uint32_t (&cw)[2][4], const Smem& sm, int kk0, int g, int t,
                                            int (&acc)[2][2][4]) {
  uint32_t p[2][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) p[m][i] = plane<S>(cw[m][i]);
#pragma unroll
  for (int nu = 0; nu < 2; ++nu) {
    const uint32_t mk = nu ? 0x10101010u : 0x01010101u;
    const uint2 b = *reinterpret_cast<const uint2*>(&sm.qfrag[kk0 + S * 2 + nu][g][t][0]);
#pragma unroll
    for (int m = 0; m < 2; ++m) mma_s8(acc[m][nu], p[m][0] & mk, p[m][2] & mk, p[m][1] & mk, p[m][3] & mk, b.x, b.y);
  }
}

// cmap: the codes as a 2-D uint8 tensor {codes_B, n}, box {128, 256}, 128-byte swizzle.
__global__ void __launch_bounds__(kThreads, 1) search_mma4_kernel(const __grid_constant__ CUtensorMap cmap, Args a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int q0 = blockIdx.y * kQT;
  const int64_t c0 = (int64_t)blockIdx.x * a.chunk, c1 = min(a.n, c0 + a.chunk);
  const int nblk = (int)((max(c1 - c0, (int64_t)0) + kVB - 1) / kVB);
  const int nch = a.codes_B / 32;   // 32-byte chunks of a code row
  const int nsteps = nch * kPlanes * 2;
  const int nsl = (a.codes_B + kSlice - 1) / kSlice;
  const int njobs = nblk * nsl;     // job J: slice J % nsl of block J / nsl

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], kWarps);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  for (int i = tid; i < nsteps * 8 * 4 * 2; i += kThreads) (&sm.qfrag[0][0][0][0])[i] = 0u;
  __syncthreads();
  int issued = 0;
  auto issue = [&](int J) {   // whole boxes arrive (rows past n and bytes past codes_B as zeros)
    const int64_t v0 = c0 + (int64_t)(J / nsl) * kVB;
    uint64_t* bar = &sm.full[J % kStages];
    mbar_expect_tx(bar, (uint32_t)kSliceBytes);
    sm2::tma_tile_2d(sm.stage[J % kStages], &cmap, (J % nsl) * kSlice, (int)v0, bar);
    issued = J + 1;
  };
  if (tid == 0)
    for (int J = 0; J < min(kStages, njobs); ++J) issue(J);
  grid_dep_wait();   // the rotated queries come from the kernel before this one

  // query pieces: warp w < 4 prepares query w of the tile
  if (warp < kQT) {
    const int q = q0 + warp;
    const float* qv = a.qr + (size_t)q * a.d;
    float wmax = 0.f;
#pragma unroll
    for (int S = 0; S < kPlanes; ++S) wmax = fmaxf(wmax, fabsf(a.w[S]));
    float sq = 0.f, mq = 0.f;
    if (q < a.nq)
      for (int c = lane; c < a.d; c += 32) {
        const float v = qv[c];
        sq += v;
        mq = fmaxf(mq, fabsf(v));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
    }
    const float mx = mq * wmax;
    const float step = mx > 0.f ? mx / 16256.f : 1.f;
    if (q < a.nq) {
      int8_t* qf = reinterpret_cast<int8_t*>(&sm.qfrag[0][0][0][0]);
      const int col = 2 * warp;
      for (int c = lane; c < a.d; c += 32) {
        const float v = qv[c];
#pragma unroll
        for (int S = 0; S < kPlanes; ++S) {
          const int xi = __float2int_rn(a.w[S] * v / step);
          const int hi = (xi >= 0) ? (xi + 64) >> 7 : -((-xi + 64) >> 7);
          const int off = q_offset(c, S);
          qf[off + col * 32] = (int8_t)hi;                     // column 2 q: hi piece
          qf[off + (col + 1) * 32] = (int8_t)(xi - 128 * hi);  // column 2 q + 1: lo piece
        }
      }
    }
    if (lane == 0) {
      sm.qc0[warp] = a.c0 * sq;
      sm.qstep[warp] = step;
    }
  }
  __syncthreads();

  // this lane's rows of ldmatrix: row tile 0 at vr0, row tile 1 at vr0 + 16 (same row mod 8)
  const int mat = lane >> 3, vr0 = 32 * warp + (lane & 7) + 8 * (mat >> 1);
  float ls = -INFINITY;   // warps 0..3: running top-k of query `warp`, lane j holds entry j
  int64_t li = -1;
  for (int j = 0; j < nblk; ++j) {
    const int64_t v0 = c0 + (int64_t)j * kVB;
    const int nv = (int)min((int64_t)kVB, c1 - v0);
    int acc[2][2][4] = {};   // [row tile][nibble family]
    for (int sl = 0; sl < nsl; ++sl) {
      const int J = j * nsl + sl;
      // warp-uniform (the guarded code is warp-collective)
      const bool aborted = __any_sync(0xffffffffu, *(volatile int*)&sm.abort_flag != 0);
      if (tid == 0 && !aborted && J >= 1 && J - 1 + kStages < njobs) {
        // refill the stage of job J - 1 with job J - 1 + kStages once every warp has released it
        if (!mbar_wait(&sm.empty[(J - 1) % kStages], ((J - 1) / kStages) & 1)) sm.abort_flag = 1;
        else issue(J - 1 + kStages);
      }
      if (!aborted && !mbar_wait(&sm.full[J % kStages], (J / kStages) & 1)) sm.abort_flag = 1;
      if (!aborted) {
        const unsigned char* st = sm.stage[J % kStages];
        const int nc4 = min(4, nch - 4 * sl);   // 32-byte chunks in this slice
        for (int c4 = 0; c4 < nc4; ++c4) {
          // cw[m][0] = vector g word t, [1] = vector g word 4+t, [2] = vector g+8 word t, [3] = g+8 word 4+t
          // (16-byte unit u of a slice row sits at unit u ^ (row % 8))
          const int unit = ((c4 << 1) | (mat & 1)) ^ (vr0 & 7);
          uint32_t cw[2][4];
          ldsm_x4(cw[0], st + vr0 * kSlice + 16 * unit);
          ldsm_x4(cw[1], st + (vr0 + 16) * kSlice + 16 * unit);
          const int kk0 = (4 * sl + c4) * kPlanes * 2;
          chunk_plane<0>(cw, sm, kk0, g, t, acc);
          chunk_plane<1>(cw, sm, kk0, g, t, acc);
          chunk_plane<2>(cw, sm, kk0, g, t, acc);
          chunk_plane<3>(cw, sm, kk0, g, t, acc);
          chunk_plane<4>(cw, sm, kk0, g, t, acc);
          chunk_plane<5>(cw, sm, kk0, g, t, acc);
          chunk_plane<6>(cw, sm, kk0, g, t, acc);
          chunk_plane<7>(cw, sm, kk0, g, t, acc);
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&sm.empty[J % kStages])) : "memory");
    }
    const bool aborted = __any_sync(0xffffffffu, *(volatile int*)&sm.abort_flag != 0);
    __syncthreads();   // the previous block's top-k pass is done with sm.sc
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int r = 0; r < 2; ++r) {   // columns 2t, 2t + 1: query t, hi and lo pieces
        const int hi = 2 * r, lo = 2 * r + 1;
        const int dot = 128 * (acc[m][0][hi] + (acc[m][1][hi] >> 4)) + (acc[m][0][lo] + (acc[m][1][lo] >> 4));
        const int vi = 32 * warp + 16 * m + g + 8 * r;
        const float nrm = vi < nv ? load_norm(a.norms, a.norm_dtype, v0 + vi) : 0.f;
        sm.sc[t][vi] = nrm * (sm.qc0[t] + sm.qstep[t] * (float)dot);
      }
    __syncthreads();
    if (!aborted && warp < kQT && q0 + warp < a.nq) {
#pragma unroll 2
      for (int i = 0; i < kVB / 32; ++i) {
        const int vi = lane + 32 * i;
        const bool valid = vi < nv;
        const float s = valid ? sm.sc[warp][vi] : -INFINITY;
        const int64_t idx = v0 + vi;
        float ts = __shfl_sync(0xffffffffu, ls, a.k - 1);
        int64_t ti = __shfl_sync(0xffffffffu, li, a.k - 1);
        uint32_t mk = __ballot_sync(0xffffffffu, valid && before(s, idx, ts, ti));
        while (mk) {
          const int src = __ffs(mk) - 1;
          const float cs = __shfl_sync(0xffffffffu, s, src);
          const int64_t ci = __shfl_sync(0xffffffffu, idx, src);
          list_insert(ls, li, a.k, cs, ci);
          ts = __shfl_sync(0xffffffffu, ls, a.k - 1);
          ti = __shfl_sync(0xffffffffu, li, a.k - 1);
          mk &= ~(1u << src);
          mk &= __ballot_sync(0xffffffffu, valid && before(s, idx, ts, ti));
        }
      }
    }
  }

  __syncthreads();
  if (sm.abort_flag) {
    if (tid == 0) {
      report_error(a.err, kErrTimeout);
      for (int jx = max(0, issued - kStages); jx < issued; ++jx)
        (void)mbar_wait(&sm.full[jx % kStages], (jx / kStages) & 1);
    }
    return;
  }
  const int q = q0 + warp;
  if (warp < kQT && q < a.nq && lane < a.k) {
    const size_t o = ((size_t)blockIdx.x * a.nq + q) * a.k + lane;
    a.cand_s[o] = ls;
    a.cand_i[o] = li;
  }
}

}  // namespace sm4
}  // namespace tqk
