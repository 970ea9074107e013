// Top-k inner-product search over MSE codes of 1 to 4 bits on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory, query operand staged by TMA).
//
// "TurboQuant: redefining AI efficiency" (hakusoku.com), "Impact on high-dimensional vector
// search": s = ||x|| <Pi q, c[idx]> over the compressed database, ranked by score (equal scores:
// lower index first).
//
// Fixed point. The centroids and each rotated query are rounded to integers against one step
// each, c_i ~ step_c C_i and q'_j ~ step_q Q_j with |C|, |Q| <= 16319, and split into int8 pieces
// C = 128 C_h + C_l, Q = 128 Q_h + Q_l (C_l, Q_l in [-64, 63], C_h, Q_h in [-127, 127]). Then
//   <Q, C[idx]> = 16384 <Q_h, C_h[idx]> + 128 (<Q_l, C_h[idx]> + <Q_h, C_l[idx]>) + <Q_l, C_l[idx]>;
// the kernel forms the first two terms exactly in int32 (two accumulators, three int8
// contractions of depth d) and drops the last, at most 64 * 64 per coordinate: 1.6e-5 of
// max|c| max|q'|, below the 15-bit rounding of c and q' themselves.
// Any codebook works (no symmetry or affine structure is assumed): a coordinate's two operand
// bytes C_h[idx], C_l[idx] come from 16-entry tables by byte permutes.
//
// d is a multiple of 64 (at least 128): a last K-chunk of 64 coordinates reads the query pieces
// past d as zeros (the TMA box's out-of-bounds fill), so whatever the expansion writes there adds
// nothing.
//
// Tiles. Queries are the MMA rows (M = 128 per CTA, one per tensor-memory lane), database vectors
// the columns (N = 256 per tile). A CTA holds one query tile and walks a contiguous chunk of the
// database, 256 vectors per tile; a tile is a loop over K-chunks of 128 coordinates (one 128-byte
// swizzle atom of int8):
//   warp 0, lane 0   TMA: Q_h and Q_l of the K-chunk (two 16 KB boxes, 128-byte swizzle), 3 stages
//   warp 1           tensor-memory allocation (512 columns: acc_hi, acc_mid); lane 0 issues
//                    4 K-steps x 3 MMAs per K-chunk, then commits the stages and the accumulator
//   warps 2-9        expansion: thread p owns vector row p of the tile, keeps its packed codes of
//                    the next K-chunk in flight in registers, and writes C_h and C_l of all 128
//                    coordinates into the swizzled B tiles of a 2-stage ring
//   warps 10-17      epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 and columns of
//                    half (w - 10) / 4 of the tile, so thread t owns query 32 (w % 4) + lane on those
//                    128 vectors: it turns the accumulators into scores and keeps the query's running
//                    top-k (k <= 16 or <= 32) over its half as a sorted list in registers.
// Per query, chunk and half the list goes to the candidate arrays ([chunk][half] counts as one
// chunk), which topk_merge_kernel reduces. Every list's k-th best score is a lower bound of the
// query's final k-th best, so each list publishes it (atomicMax into gbound) once full, and every
// list reads the query's bound once per tile: a vector scoring below it cannot be in the final
// top-k and is not considered (equal scores still are: the lower index may win them).
// Every wait is bounded; a wait that runs out sets an abort flag (checked by every loop) and the
// error word's kErrTimeout bit; the kernel then waits (bounded) for its own copies and MMAs and
// frees its tensor memory.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "encode_tc.cuh"

namespace tqk {
namespace stc {

using etc::bar_arrive;
using etc::expect_tx;
using etc::mma_commit;
using etc::sts128;
using etc::sw128_desc;
using etc::tc_fence_after;
using etc::tc_fence_before;
using etc::tma_load_2d;
using etc::wait_bar;

constexpr int kQ = 128;          // queries per CTA (MMA M, tensor-memory lanes)
constexpr int kV = 256;          // vectors per tile (MMA N)
constexpr int kKC = 128;         // coordinates per K-chunk
constexpr int kQS = 3;           // query-operand stages
constexpr int kVS = 2;           // vector-operand stages
constexpr int kMaxK = 32;        // list entries per query
constexpr int kMaxBits = 4;
constexpr int kCMax = 16319;     // |C|, |Q| bound: 128 * 127 + 63
constexpr int kExpandWarp0 = 2, kEpiWarp0 = 10;   // eight expansion warps, then the epilogue warps
constexpr int kEpiWarps = 8;     // two per tensor-memory lane quarter: one per half of the tile's columns
constexpr int kHalves = kEpiWarps / 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);   // 18 warps
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kQStage = 2u * kQ * kKC;              // 32 KB: Q_h box, then Q_l box
constexpr uint32_t kVStage = 2u * kV * kKC;              // 64 KB: C_h tile, then C_l tile
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffV = kOffQ + kQS * kQStage;         // 96 KB
constexpr uint32_t kOffNorm = kOffV + kVS * kVStage;      // 224 KB: float [2][kV]
constexpr uint32_t kOffBars = kOffNorm + 2 * kV * 4;
// q_full[kQS], q_empty[kQS], v_full[kVS], v_empty[kVS], acc_full, acc_empty
constexpr int kNumBars = 2 * kQS + 2 * kVS + 2;
constexpr uint32_t kOffTmemSlot = kOffBars + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4;
static_assert(kSmemBytes <= 232448, "search_tc layout exceeds the shared memory of one CTA");

struct Args {
  int nq, nq_pad, d, k, norm_dtype, codes_B;
  const uint8_t* codes;    // [n][codes_B]
  const void* norms;       // [n]
  const float* qscale;     // [nq]: step_q * step_c
  int64_t n, chunk;        // database rows, rows per CTA chunk (a multiple of kV)
  uint32_t th[4], tl[4];   // C_h[idx], C_l[idx] as bytes, idx = 0 .. 15
  float* cand_s;           // [nchunks][kHalves][nq][k]
  int64_t* cand_i;
  int* gbound;             // [nq]: the largest k-th best score any list has reached, as an ordered int
  int* err;
};

// Order-preserving map between floats and ints (its own inverse), for atomicMax on scores.
__device__ __forceinline__ int float_ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord_float(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

// 16-entry table lookup of four 4-bit indices (nibbles 0..3 of x) -> four bytes: two 8-entry
// permutes, then a permute that takes byte j from the second when bit 3 of nibble j is set.
__device__ __forceinline__ uint32_t lut16(uint32_t x, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  const uint32_t sel = x & 0x7777u;
  const uint32_t lo = __byte_perm(t0, t1, sel), hi = __byte_perm(t2, t3, sel);
  return __byte_perm(lo, hi, 0x3210u | ((x >> 1) & 0x4444u));
}

// Four fields of BITS bits (bits 0 .. 4 BITS - 1 of x) -> selector nibbles 0..3 (BITS = 1, 3).
template <int BITS>
__device__ __forceinline__ uint32_t nibbles4(uint32_t x) {
  constexpr uint32_t m = (1u << BITS) - 1;
  return (x & m) | ((x >> BITS & m) << 4) | ((x >> (2 * BITS) & m) << 8) | ((x >> (3 * BITS) & m) << 12);
}

// Eight 2-bit fields (bits 0..15 of x) -> nibbles 0..7.
__device__ __forceinline__ uint32_t nibbles8_2bit(uint32_t x) {
  uint32_t t = x & 0xFFFFu;
  t = (t | (t << 8)) & 0x00FF00FFu;
  t = (t | (t << 4)) & 0x0F0F0F0Fu;
  t = (t | (t << 2)) & 0x33333333u;
  return t;
}

// Operand bytes of 16 coordinates (unit u of a 128-coordinate code chunk w[]) -> h[4], l[4].
template <int BITS>
__device__ __forceinline__ void expand_unit(const uint32_t (&w)[4 * BITS], int u, const uint32_t (&th)[4],
                                            const uint32_t (&tl)[4], uint32_t (&h)[4], uint32_t (&l)[4]) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t x = w[2 * u + half];
      h[2 * half] = lut16(x, th[0], th[1], th[2], th[3]);
      l[2 * half] = lut16(x, tl[0], tl[1], tl[2], tl[3]);
      h[2 * half + 1] = lut16(x >> 16, th[0], th[1], th[2], th[3]);
      l[2 * half + 1] = lut16(x >> 16, tl[0], tl[1], tl[2], tl[3]);
    }
  } else if constexpr (BITS == 2) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t t = nibbles8_2bit(w[u] >> (16 * half));
      h[2 * half] = __byte_perm(th[0], 0u, t);
      l[2 * half] = __byte_perm(tl[0], 0u, t);
      h[2 * half + 1] = __byte_perm(th[0], 0u, t >> 16);
      l[2 * half + 1] = __byte_perm(tl[0], 0u, t >> 16);
    }
  } else if constexpr (BITS == 1) {
    const uint32_t x = w[u >> 1] >> (16 * (u & 1));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t s = nibbles4<1>(x >> (4 * j));
      h[j] = __byte_perm(th[0], th[1], s);
      l[j] = __byte_perm(tl[0], tl[1], s);
    }
  } else {   // BITS == 3: unit u is the 48 bits at bit 48 u of the chunk
    const int wi = (3 * u) >> 1, sh = 16 * (u & 1);
    const uint32_t w0 = w[wi], w1 = w[wi + 1], w2 = (wi + 2 < 12) ? w[wi + 2 < 12 ? wi + 2 : 0] : 0u;
    const uint64_t win = (uint64_t)__funnelshift_r(w0, w1, sh) | ((uint64_t)(__funnelshift_r(w1, w2, sh) & 0xFFFFu) << 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t s = nibbles4<3>((uint32_t)(win >> (12 * j)));
      h[j] = __byte_perm(th[0], th[1], s);
      l[j] = __byte_perm(tl[0], tl[1], s);
    }
  }
}

// Packed codes of one row's K-chunk: 16 BITS bytes = 4 BITS words, of which the first `nbytes`
// (a multiple of 8) are read and the rest are zero. Rows are 16-byte aligned when d % 128 == 0
// (a16), else 8-byte aligned (d % 64 == 0).
template <int BITS>
__device__ __forceinline__ void load_chunk(const uint8_t* row, bool ok, int nbytes, bool a16, uint32_t (&w)[4 * BITS]) {
#pragma unroll
  for (int i = 0; i < 4 * BITS; ++i) w[i] = 0u;
  if (!ok) return;
  if (a16 && nbytes == 16 * BITS) {
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(row) + i);
      w[4 * i] = x.x;
      w[4 * i + 1] = x.y;
      w[4 * i + 2] = x.z;
      w[4 * i + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2 * BITS; ++i)
      if (8 * i < nbytes) {
        const uint2 x = __ldg(reinterpret_cast<const uint2*>(row) + i);
        w[2 * i] = x.x;
        w[2 * i + 1] = x.y;
      }
  }
}

// Named barrier over n threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Instruction descriptor, kind::i8: int32 accumulate, A and B signed 8-bit, both K-major, M = 128, N = kV.
__host__ __device__ constexpr uint32_t idesc_i8() {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kV >> 3) << 17) | ((uint32_t)(kQ >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld1x2(uint32_t ta, uint32_t tb, uint32_t& x, uint32_t& y) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n" : "=r"(x) : "r"(ta));
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n" : "=r"(y) : "r"(tb));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" : "+r"(x), "+r"(y) : : "memory");
}

// Waits for this thread's tensor-memory loads; the loaded registers are operands, so that no use
// of them is scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld8x2(uint32_t (&x)[8], uint32_t (&y)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7]),
                 "+r"(y[0]), "+r"(y[1]), "+r"(y[2]), "+r"(y[3]), "+r"(y[4]), "+r"(y[5]), "+r"(y[6]), "+r"(y[7])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld2(uint32_t (&x)[16], uint32_t (&y)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7]),
                 "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]), "+r"(x[14]), "+r"(x[15]),
                 "+r"(y[0]), "+r"(y[1]), "+r"(y[2]), "+r"(y[3]), "+r"(y[4]), "+r"(y[5]), "+r"(y[6]), "+r"(y[7]),
                 "+r"(y[8]), "+r"(y[9]), "+r"(y[10]), "+r"(y[11]), "+r"(y[12]), "+r"(y[13]), "+r"(y[14]), "+r"(y[15])
               :
               : "memory");
}

// qmap: the query pieces as a 2-D int8 tensor {d, 2 nq_pad} (Q_h rows, then Q_l rows), box
// {128, 128}, 128-byte swizzle. Grid: (chunks, query tiles of 128).
template <int BITS, int KMAX>
__global__ void __launch_bounds__(kThreads, 1) search_tc_kernel(const __grid_constant__ CUtensorMap qmap, Args a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = smem_addr(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q0 = blockIdx.y * kQ;
  const int64_t c0 = (int64_t)blockIdx.x * a.chunk, c1 = min(a.n, c0 + a.chunk);
  const int ntiles = (int)((max(c1 - c0, (int64_t)0) + kV - 1) / kV);
  const int nkc = (a.d + kKC - 1) / kKC;   // the last K-chunk may hold 64 coordinates
  const int total = ntiles * nkc;   // K-chunks of this CTA

  const uint32_t bars = base + kOffBars;
  auto q_full = [&](int s) { return bars + 8u * s; };
  auto q_empty = [&](int s) { return bars + 8u * (kQS + s); };
  auto v_full = [&](int s) { return bars + 8u * (2 * kQS + s); };
  auto v_empty = [&](int s) { return bars + 8u * (2 * kQS + kVS + s); };
  const uint32_t acc_full = bars + 8u * (2 * kQS + 2 * kVS), acc_empty = acc_full + 8u;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  float* nrm_s = reinterpret_cast<float*>(smem + kOffNorm);

  if ((base & 1023u) != 0) {   // the swizzled operand layout needs 1024-byte alignment
    if (tid == 0) report_error(a.err, kErrInternal);
    return;
  }
  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kQS; ++s) {
      bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + s, 1);
      bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + kQS + s, 1);
    }
    for (int s = 0; s < kVS; ++s) {
      bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + 2 * kQS + s, kEpiWarp0 - kExpandWarp0);   // expansion warps
      bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + 2 * kQS + kVS + s, 1);
    }
    bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + 2 * kQS + 2 * kVS, 1);       // acc_full: commit
    bar_init(reinterpret_cast<uint64_t*>(smem + kOffBars) + 2 * kQS + 2 * kVS + 1, kEpiWarps);   // acc_empty
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(base + kOffTmemSlot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemSlot);
  int* const err = a.err;
  auto fail_wait = [&]() {
    *abort_flag = 1;
    report_error(err, kErrTimeout);
  };
  grid_dep_wait();   // the query pieces come from the kernel before this one

  if (warp == 0) {
    // ---------------- TMA: query pieces of every K-chunk
    if (lane == 0) {
      int issued = 0;
      for (; issued < total; ++issued) {
        const int s = issued % kQS, kc = issued % nkc;
        if (issued >= kQS && !*abort_flag && !wait_bar(q_empty(s), ((issued / kQS) - 1) & 1)) fail_wait();
        if (*abort_flag) break;
        expect_tx(q_full(s), kQStage);
        tma_load_2d(base + kOffQ + s * kQStage, &qmap, kc * kKC, q0, q_full(s));
        tma_load_2d(base + kOffQ + s * kQStage + kQStage / 2, &qmap, kc * kKC, a.nq_pad + q0, q_full(s));
      }
      // never leave with a copy still landing in this CTA's shared memory
      for (int i = (issued > kQS ? issued - kQS : 0); i < issued; ++i) (void)wait_bar(q_full(i % kQS), (i / kQS) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8();
      const uint32_t acc_hi = tmem, acc_mid = tmem + (uint32_t)kV;
      int it = 0, committed_tiles = 0;
      for (int t = 0; t < ntiles && !*abort_flag; ++t) {
        if (t >= 1 && !wait_bar(acc_empty, (t - 1) & 1)) { fail_wait(); break; }
        tc_fence_after();
        for (int kc = 0; kc < nkc; ++kc, ++it) {
          const int sq = it % kQS, sv = it % kVS;
          if (!wait_bar(q_full(sq), (it / kQS) & 1) || !wait_bar(v_full(sv), (it / kVS) & 1)) { fail_wait(); break; }
          tc_fence_after();
          const uint32_t qa = base + kOffQ + sq * kQStage, vb = base + kOffV + sv * kVStage;
#pragma unroll
          for (int kk = 0; kk < kKC / 32; ++kk) {
            const uint32_t off = kk * 32;
            const uint64_t ah = sw128_desc(qa + off), al = sw128_desc(qa + kQStage / 2 + off);
            const uint64_t bh = sw128_desc(vb + off), bl = sw128_desc(vb + kVStage / 2 + off);
            const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
            mma_i8(acc_hi, ah, bh, idesc, acc);
            mma_i8(acc_mid, al, bh, idesc, acc);
            mma_i8(acc_mid, ah, bl, idesc, 1u);
          }
          mma_commit(q_empty(sq));
          mma_commit(v_empty(sv));
        }
        if (*abort_flag) break;
        mma_commit(acc_full);
        committed_tiles = t + 1;
      }
      // tensor memory is released below: make sure no MMA still writes it
      if (committed_tiles > 0) (void)wait_bar(acc_full, (committed_tiles - 1) & 1);
    }
  } else if (warp < kEpiWarp0) {
    // ---------------- expansion: codes -> C_h / C_l operand tiles
    const int p = tid - 32 * kExpandWarp0;   // 0 .. 255: row p
    constexpr int W = 4 * BITS;
    const int cbytes = kKC * BITS / 8;       // code bytes of a row's K-chunk
    const int last_bytes = (a.d - (nkc - 1) * kKC) * BITS / 8;   // ... of its last K-chunk
    const bool a16 = (a.codes_B & 15) == 0;
    const uint8_t* codes = a.codes;
    const int64_t codes_B = a.codes_B;
    uint32_t th[4], tl[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      th[i] = a.th[i];
      tl[i] = a.tl[i];
    }
    uint32_t cur[W], nxt[W];
    auto fetch = [&](int itx, uint32_t(&w)[W]) {
      const int t = itx / nkc, kc = itx % nkc;
      const int64_t v = c0 + (int64_t)t * kV + p;
      const bool ok = itx < total && v < c1;
      load_chunk<BITS>(codes + (ok ? v : 0) * codes_B + (int64_t)kc * cbytes, ok, kc == nkc - 1 ? last_bytes : cbytes,
                       a16, w);
    };
    fetch(0, cur);
    for (int it = 0; it < total; ++it) {
      fetch(it + 1, nxt);
      const int s = it % kVS;
      bool ok = !*abort_flag;
      if (ok && it >= kVS && !wait_bar(v_empty(s), ((it / kVS) - 1) & 1)) { fail_wait(); ok = false; }
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint32_t vb = base + kOffV + s * kVStage;
      const uint32_t rh = vb + p * 128, rl = rh + kVStage / 2;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t h[4], l[4];
        expand_unit<BITS>(cur, u, th, tl, h, l);
        const uint32_t o = (uint32_t)((u ^ (p & 7)) << 4);
        sts128(rh + o, h[0], h[1], h[2], h[3]);
        sts128(rl + o, l[0], l[1], l[2], l[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) bar_arrive(v_full(s));
#pragma unroll
      for (int i = 0; i < W; ++i) cur[i] = nxt[i];
    }
  } else {
    // ---------------- epilogue: scores and running top-k, one query per thread
    const int quarter = warp & 3, ql = 32 * quarter + lane, q = q0 + ql;
    const int e = tid - 32 * kEpiWarp0;   // 0 .. 32 kEpiWarps - 1
    const int half = (warp - kEpiWarp0) >> 2;
    constexpr int kStepsPerHalf = kV / 8 / kHalves;
    const bool qok = q < a.nq;
    const float qscale128 = qok ? 128.f * a.qscale[q] : 0.f;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16);
    // the list, descending: entries KMAX - k .. KMAX - 1 are the running top-k (empty: -inf),
    // the ones before them +inf sentinels that no score displaces, so the k-th best is always
    // the last entry and an insertion bubbles through fixed register positions
    const int k = a.k;   // <= KMAX
    float ls[KMAX];
    int li[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ls[j] = j < KMAX - k ? INFINITY : -INFINITY;
      li[j] = -1;
    }
    float thr = -INFINITY;
    // every position from the old list at once: x keeps its entry if that is >= s, takes s if
    // entry x - 1 is >= s, else takes entry x - 1 (the last entry falls off)
    auto insert = [&](float sj, int ci) {
      bool prev_ge = true;
      float lp = 0.f;
      int ip = -1;
#pragma unroll
      for (int x = 0; x < KMAX; ++x) {
        const bool ge = ls[x] >= sj;
        const float lx = ls[x];
        const int ix = li[x];
        ls[x] = ge ? lx : (prev_ge ? sj : lp);
        li[x] = ge ? ix : (prev_ge ? ci : ip);
        lp = lx;
        ip = ix;
        prev_ge = ge;
      }
      thr = ls[KMAX - 1];
    };
    float gb = -INFINITY;   // the query's shared lower bound, read once per tile
    for (int t = 0; t < ntiles; ++t) {
      const int64_t v0 = c0 + (int64_t)t * kV;
      const int nv = (int)min((int64_t)kV, c1 - v0);
      float* nb = nrm_s + (t & 1) * kV;
      if (qok) gb = fmaxf(gb, ord_float(*reinterpret_cast<volatile int*>(a.gbound + q)));
      for (int j = e; j < kV; j += 32 * kEpiWarps) nb[j] = j < nv ? load_norm(a.norms, a.norm_dtype, v0 + j) : 0.f;
      bool ok = !*abort_flag;
      if (ok && !wait_bar(acc_full, t & 1)) { fail_wait(); ok = false; }
      // one decision for all epilogue warps (this barrier also publishes the norms): tcgen05.ld
      // is warp-collective and every epilogue warp must reach the same barriers
      if (bar_red_or(1, 32 * kEpiWarps, !ok)) break;
      tc_fence_after();
      // 8 columns per step; the next step's accumulators load while this step is scored
      // (tcgen05.wait::ld waits for every load of the thread, so the loaded registers are copied
      // out before the next loads are issued into them)
      // this warp's steps: [st0, st1) of the tile's (nv + 7) / 8 (the same for the whole warp).
      // Pass 1 scores every column against the threshold and bound as they stood at the start of
      // the tile and keeps one bit per candidate; pass 2 (rare: a candidate in any lane) reloads
      // those columns, in index order, and inserts what still qualifies.
      const int st0 = half * kStepsPerHalf, st1 = min((nv + 7) / 8, st0 + kStepsPerHalf);
      uint64_t cbits[kStepsPerHalf / 8];
      uint32_t hA[8], mA[8];
      if (st0 < st1) {
        tmem_ld8(lane_addr + 8 * st0, hA);
        tmem_ld8(lane_addr + kV + 8 * st0, mA);
      }
#pragma unroll
      for (int gr = 0; gr < kStepsPerHalf / 8; ++gr) {
        uint64_t bits = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int st = st0 + 8 * gr + i;
          if (st < st1) {   // the same for the whole warp
            tmem_wait_ld8x2(hA, mA);
            uint32_t h[8], mm[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = hA[j], mm[j] = mA[j];
            if (st + 1 < st1) {
              tmem_ld8(lane_addr + 8 * (st + 1), hA);
              tmem_ld8(lane_addr + kV + 8 * (st + 1), mA);
            }
            const int c = 8 * st;
            const float4 n0 = *reinterpret_cast<const float4*>(nb + c);
            const float4 n1 = *reinterpret_cast<const float4*>(nb + c + 4);
            const float nr[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
            uint32_t cand = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              // 16384 acc_hi + 128 acc_mid = 128 (128 acc_hi + acc_mid)
              const float sj = fmaf(128.f, (float)(int)h[j], (float)(int)mm[j]) * (qscale128 * nr[j]);
              cand |= (sj > thr && sj >= gb) ? (1u << j) : 0u;
            }
            if (nv - c < 8) cand &= (1u << max(nv - c, 0)) - 1u;
            bits |= (uint64_t)cand << (8 * i);
          }
        }
        cbits[gr] = qok ? bits : 0ull;
      }
#pragma unroll
      for (int gr = 0; gr < kStepsPerHalf / 8; ++gr) {
        const uint32_t lo = __reduce_or_sync(0xffffffffu, (uint32_t)cbits[gr]);
        const uint32_t hi = __reduce_or_sync(0xffffffffu, (uint32_t)(cbits[gr] >> 32));
        uint64_t any = ((uint64_t)hi << 32) | lo;
        while (any) {   // the same for the whole warp
          const int bit = __ffsll((long long)any) - 1;
          any &= any - 1;
          const int col = 8 * st0 + 64 * gr + bit;
          uint32_t x, y;
          tmem_ld1x2(lane_addr + col, lane_addr + kV + col, x, y);
          if (cbits[gr] >> bit & 1ull) {
            const float sj = fmaf(128.f, (float)(int)x, (float)(int)y) * (qscale128 * nb[col]);
            if (sj > thr && sj >= gb) insert(sj, (int)(v0 + col));   // an equal score ranks after
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(acc_empty);
      if (qok && thr > -INFINITY) atomicMax(a.gbound + q, float_ord(thr));
    }
    if (qok && !*abort_flag) {
      const size_t o = (((size_t)blockIdx.x * kHalves + half) * a.nq + q) * k - (KMAX - k);
#pragma unroll
      for (int x = 0; x < KMAX; ++x)
        if (x >= KMAX - k) {
          a.cand_s[o + x] = ls[x];
          a.cand_i[o + x] = li[x];
        }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Query pieces: row q of qr (rotated queries, fp32) -> Q_h (row q) and Q_l (row nq_pad + q) of
// `pieces`, Q = rint(q' / step_q) with step_q = max_j |q'_j| / 16319; qscale[q] = step_q * step_c;
// gbound[q] starts at -inf. Rows nq .. nq_pad - 1 are zero. One warp per row.
__global__ void search_tc_qprep_kernel(const float* qr, int nq, int nq_pad, int d, float step_c, int8_t* pieces,
                                       float* qscale, int* gbound) {
  grid_dep_launch();
  grid_dep_wait();   // qr comes from the rotation kernel before this one
  const int lane = threadIdx.x & 31;
  const int q = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (q >= nq_pad) return;
  int8_t* ph = pieces + (size_t)q * d;
  int8_t* pl = pieces + (size_t)(nq_pad + q) * d;
  if (q >= nq) {
    for (int j = lane; j < d; j += 32) ph[j] = pl[j] = 0;
    return;
  }
  const float* row = qr + (size_t)q * d;
  float mx = 0.f;
  for (int j = lane; j < d; j += 32) mx = fmaxf(mx, fabsf(row[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float inv = mx > 0.f ? (float)kCMax / mx : 0.f;
  for (int j = lane; j < d; j += 32) {
    const int x = max(-kCMax, min(kCMax, __float2int_rn(row[j] * inv)));
    const int h = (x + 64) >> 7;   // floor: x - 128 h in [-64, 63]
    ph[j] = (int8_t)h;
    pl[j] = (int8_t)(x - 128 * h);
  }
  if (lane == 0) {
    qscale[q] = mx > 0.f ? (mx / (float)kCMax) * step_c : 0.f;
    gbound[q] = float_ord(-INFINITY);
  }
}

// The bound pass's result: gbound[q] = the k-th best score of the sample (when it has k vectors).
__global__ void search_tc_bound_kernel(const float* ts, const int64_t* ti, int nq, int k, int* gbound) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q < nq && ti[(size_t)q * k + k - 1] >= 0) atomicMax(gbound + q, float_ord(ts[(size_t)q * k + k - 1]));
}

}  // namespace stc
}  // namespace tqk
