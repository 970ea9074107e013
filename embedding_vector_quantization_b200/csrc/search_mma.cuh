// Top-k inner-product search over 2-bit MSE codes on int8 tensor-core MMAs.
//
// "TurboQuant: redefining AI efficiency" (hakusoku.com), "Impact on high-dimensional
// vector search": scores s = ||x|| <Pi q, c[idx]> on the compressed vectors, ranked by
// score (equal scores: lower index first). A symmetric 2-bit codebook is affine in its
// index bits, c[idx] = c0 + (c1 - c0) b0 + (c2 - c0) b1, so
//   <q', c[idx]> = c0 sum(q') + <(c1 - c0) q', b0> + <(c2 - c0) q', b1>,
// two 0/1 bit-plane dot products. Database vectors are the MMA rows (their packed code
// words, shifted and masked into 0/1 bytes), queries the columns: the scaled query values
// are rounded to 15-bit integers against one step per query and split into int8 hi/lo
// pieces, so every dot product accumulates exactly in int32.
//
// One CTA owns 16 queries (their B fragments stay in shared memory: 64 d bytes, stored in
// lane order so that a warp's fragment load covers all 32 banks) and a contiguous chunk of
// the database, in blocks of 256 vectors. A block arrives as d / 512 column slices of
// 128 bytes per row (2-D TMA tiles with the 128-byte swizzle, one slice per stage of a
// 3-stage ring): the rows of a slice are 128 bytes apart and the swizzle spreads the 8 rows
// an ldmatrix reads over all banks (unswizzled code rows of d / 4 bytes would put them in
// one bank). Warp w scores vectors 32w .. 32w+31 of a block (two MMA row tiles, so each
// query fragment loaded from shared memory feeds two MMAs) against the 16 queries;
// the block's scores go through shared memory to the warps that own the queries (two each),
// which keep a running top-k (k <= 32) with one list entry per lane. At the end each query's
// list goes to the per-chunk candidate arrays, which topk_merge_kernel reduces.
#pragma once

#include <cuda.h>

#include "attn_mma.cuh"
#include "search_simt.cuh"

namespace tqk {
namespace sm2 {

using amma::ldsm_x4;
using amma::mbar_expect_tx;
using amma::mbar_init;
using amma::mbar_wait;
using amma::mma_s8;
using amma::smem_u32;
using amma::tma_bulk_g2s;

constexpr int kQT = 16;          // queries per CTA (4 MMA column tiles of 4 queries x hi/lo)
constexpr int kRT = 3;           // 16-row MMA tiles per warp
constexpr int kVB = 8 * 16 * kRT;  // vectors per block (384)
constexpr int kBoxRows = 128;    // rows per TMA box (a box dimension is at most 256)
constexpr int kStages = 2;       // slice stages
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxD = 1536;      // codes_B = d / 4 <= 384
constexpr int kMaxCodesB = kMaxD / 4;
constexpr int kMaxK = 32;        // one list entry per lane
constexpr int kMaxSteps = kMaxCodesB / 32 * 8;   // k-steps: 32-byte chunks x (4 shifts x 2 masks)
constexpr int kSlice = 128;                       // bytes of a code row per TMA slice (the swizzle span)
constexpr int kMaxSlices = kMaxCodesB / kSlice;
constexpr int kSliceBytes = kVB * kSlice;         // 48 KB

struct Args {
  const float* qr;       // [nq][d] rotated queries
  int nq, d, codes_B, k, norm_dtype;
  const uint8_t* codes;  // [n][codes_B]
  const void* norms;     // [n]
  int64_t n, chunk;
  float c0, w0, w1;      // c[idx] = c0 + w0 b0 + w1 b1
  float* cand_s;         // [nchunks][nq][k]
  int64_t* cand_i;       // [nchunks][nq][k]
  int* err;
};

struct __align__(1024) Smem {
  unsigned char stage[kStages][kSliceBytes];         // 128-byte column slices of a block's code rows, swizzled
  uint32_t qfrag[kMaxSteps][4][8][4][2];             // [k-step][column tile][column g][quad t][register]
  float sc[kQT][kVB + 8];                            // a block's scores [query][vector] (rows 8 banks apart)
  float qc0[kQT], qstep[kQT];                 // c0 sum(q'), integer step of the query pieces
  uint64_t full[kStages];
  uint64_t empty[kStages];   // one arrival per warp when it is done with the slice
  int abort_flag;
};

// Where the query value of coordinate c, plane p sits: byte c / 4 of the code row (chunk
// byte / 32, k index byte % 32), bit 2 (c % 4) + p -> shift s = bit % 4, mask family bit / 4.
__device__ __forceinline__ int q_offset(int c, int p, int nt) {
  const int byte = c >> 2, bit = 2 * (c & 3) + p;
  const int kk = (byte >> 5) * 8 + (bit >> 2) * 4 + (bit & 3);
  const int kb = byte & 31, slot = kb >> 4, t = (kb & 15) >> 2, e = kb & 3;
  return ((((kk * 4 + nt) * 8) * 4 + t) * 2 + slot) * 4 + e;   // byte offset for column g = 0 (g adds 32 g)
}

// Dynamic shared memory to request: the Smem block plus room to align it to 1024 bytes.
__host__ __device__ inline size_t smem_bytes() { return sizeof(Smem) + 1024; }

__device__ __forceinline__ void tma_tile_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// (s, i) ranks before (t, j): higher score, or equal score and lower index.
__device__ __forceinline__ bool before(float s, int64_t i, float t, int64_t j) { return s > t || (s == t && i < j); }

// Offers candidate (s, i) to a warp-held sorted list (lane j < k holds entry j, best first).
__device__ __forceinline__ void list_insert(float& ls, int64_t& li, int k, float s, int64_t i) {
  const int lane = threadIdx.x & 31;
  const bool b = lane < k && before(s, i, ls, li);
  const uint32_t m = __ballot_sync(0xffffffffu, b);
  if (m == 0) return;
  const int pos = __ffs(m) - 1;
  const float ps = __shfl_up_sync(0xffffffffu, ls, 1);
  const int64_t pi = __shfl_up_sync(0xffffffffu, li, 1);
  if (lane > pos && lane < k) { ls = ps; li = pi; }
  if (lane == pos) { ls = s; li = i; }
}

// cmap: the codes as a 2-D uint8 tensor {codes_B, n}, box {128, 128}, 128-byte swizzle.
__global__ void __launch_bounds__(kThreads, 1) search_mma2_kernel(const __grid_constant__ CUtensorMap cmap, Args a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int q0 = blockIdx.y * kQT;
  const int64_t c0 = (int64_t)blockIdx.x * a.chunk, c1 = min(a.n, c0 + a.chunk);
  const int nblk = (int)((max(c1 - c0, (int64_t)0) + kVB - 1) / kVB);
  const int nch = a.codes_B / 32;   // 32-byte chunks of a code row
  const int nsteps = nch * 8;
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
  for (int i = tid; i < nsteps * 4 * 4 * 8 * 2; i += kThreads) (&sm.qfrag[0][0][0][0][0])[i] = 0u;
  __syncthreads();
  int issued = 0;
  auto issue = [&](int J) {   // whole boxes arrive (rows past n and bytes past codes_B as zeros)
    const int64_t v0 = c0 + (int64_t)(J / nsl) * kVB;
    const int sl = J % nsl;
    uint64_t* bar = &sm.full[J % kStages];
    mbar_expect_tx(bar, (uint32_t)kSliceBytes);
    for (int bx = 0; bx < kVB / kBoxRows; ++bx)   // boxes of {128 bytes, 128 rows}
      tma_tile_2d(sm.stage[J % kStages] + bx * kBoxRows * kSlice, &cmap, sl * kSlice, (int)v0 + bx * kBoxRows, bar);
    issued = J + 1;
  };
  if (tid == 0)
    for (int J = 0; J < min(kStages, njobs); ++J) issue(J);
  grid_dep_wait();   // the rotated queries come from the kernel before this one

  // query pieces: warp w prepares queries 2w and 2w + 1 of the tile
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int ql = 2 * warp + qq, q = q0 + ql;
    const float* qv = a.qr + (size_t)q * a.d;
    float sq = 0.f, mx = 0.f;
    if (q < a.nq)
      for (int c = lane; c < a.d; c += 32) {
        const float v = qv[c];
        sq += v;
        mx = fmaxf(mx, fmaxf(fabsf(a.w0 * v), fabsf(a.w1 * v)));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const float step = mx > 0.f ? mx / 16256.f : 1.f;
    if (q < a.nq) {
      int8_t* qf = reinterpret_cast<int8_t*>(&sm.qfrag[0][0][0][0][0]);
      const int nt = ql >> 2, col = 2 * (ql & 3);
      for (int c = lane; c < a.d; c += 32) {
        const float v = qv[c];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const int xi = __float2int_rn((p ? a.w1 : a.w0) * v / step);
          const int hi = (xi >= 0) ? (xi + 64) >> 7 : -((-xi + 64) >> 7);
          const int off = q_offset(c, p, nt);
          qf[off + col * 32] = (int8_t)hi;                     // column 2 (q % 4): hi piece
          qf[off + (col + 1) * 32] = (int8_t)(xi - 128 * hi);  // column 2 (q % 4) + 1: lo piece
        }
      }
    }
    if (lane == 0) {
      sm.qc0[ql] = a.c0 * sq;
      sm.qstep[ql] = step;
    }
  }
  __syncthreads();

  // this lane's rows of ldmatrix: row tile r at vr0 + 16 r (the same row mod 8)
  const int mat = lane >> 3, vr0 = 16 * kRT * warp + (lane & 7) + 8 * (mat >> 1);
  float ls[2] = {-INFINITY, -INFINITY};   // running top-k of queries 2w, 2w+1: lane j holds entry j
  int64_t li[2] = {-1, -1};
  for (int j = 0; j < nblk; ++j) {
    const int64_t v0 = c0 + (int64_t)j * kVB;
    const int nv = (int)min((int64_t)kVB, c1 - v0);
    int acc1[kRT][4][4] = {}, acc16[kRT][4][4] = {};   // [row tile][column tile]
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
          uint32_t cw[kRT][4];
#pragma unroll
          for (int m = 0; m < kRT; ++m) ldsm_x4(cw[m], st + (vr0 + 16 * m) * kSlice + 16 * unit);
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            uint32_t x[kRT][4];
#pragma unroll
            for (int m = 0; m < kRT; ++m)
#pragma unroll
              for (int i = 0; i < 4; ++i) x[m][i] = cw[m][i] >> s;
#pragma unroll
            for (int fam = 0; fam < 2; ++fam) {
              const uint32_t mk = fam ? 0x10101010u : 0x01010101u;
              const int kk = (4 * sl + c4) * 8 + fam * 4 + s;
#pragma unroll
              for (int nt = 0; nt < 4; ++nt) {
                const uint2 b = *reinterpret_cast<const uint2*>(&sm.qfrag[kk][nt][g][t][0]);
#pragma unroll
                for (int m = 0; m < kRT; ++m) {
                  int(&acc)[4] = fam ? acc16[m][nt] : acc1[m][nt];
                  mma_s8(acc, x[m][0] & mk, x[m][2] & mk, x[m][1] & mk, x[m][3] & mk, b.x, b.y);
                }
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&sm.empty[J % kStages])) : "memory");
    }
    const bool aborted = __any_sync(0xffffffffu, *(volatile int*)&sm.abort_flag != 0);
    __syncthreads();   // the previous block's top-k pass is done with sm.sc
#pragma unroll
    for (int m = 0; m < kRT; ++m)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int ql = 4 * nt + t;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int hi = 2 * r, lo = 2 * r + 1;
          const int dot = 128 * (acc1[m][nt][hi] + (acc16[m][nt][hi] >> 4)) + (acc1[m][nt][lo] + (acc16[m][nt][lo] >> 4));
          const int vi = 16 * kRT * warp + 16 * m + g + 8 * r;
          const float nrm = vi < nv ? load_norm(a.norms, a.norm_dtype, v0 + vi) : 0.f;
          sm.sc[ql][vi] = nrm * (sm.qc0[ql] + sm.qstep[ql] * (float)dot);
        }
      }
    __syncthreads();
    if (!aborted) {
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int ql = 2 * warp + qq;
        if (q0 + ql >= a.nq) continue;   // the same for the whole warp
#pragma unroll 2
        for (int i = 0; i < kVB / 32; ++i) {
          const int vi = lane + 32 * i;
          const bool valid = vi < nv;
          const float s = valid ? sm.sc[ql][vi] : -INFINITY;
          const int64_t idx = v0 + vi;
          float ts = __shfl_sync(0xffffffffu, ls[qq], a.k - 1);
          int64_t ti = __shfl_sync(0xffffffffu, li[qq], a.k - 1);
          uint32_t mk = __ballot_sync(0xffffffffu, valid && before(s, idx, ts, ti));
          while (mk) {
            const int src = __ffs(mk) - 1;
            const float cs = __shfl_sync(0xffffffffu, s, src);
            const int64_t ci = __shfl_sync(0xffffffffu, idx, src);
            list_insert(ls[qq], li[qq], a.k, cs, ci);
            ts = __shfl_sync(0xffffffffu, ls[qq], a.k - 1);
            ti = __shfl_sync(0xffffffffu, li[qq], a.k - 1);
            mk &= ~(1u << src);
            mk &= __ballot_sync(0xffffffffu, valid && before(s, idx, ts, ti));
          }
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
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int q = q0 + 2 * warp + qq;
    if (q < a.nq && lane < a.k) {
      const size_t o = ((size_t)blockIdx.x * a.nq + q) * a.k + lane;
      a.cand_s[o] = ls[qq];
      a.cand_i[o] = li[qq];
    }
  }
}

}  // namespace sm2
}  // namespace tqk
