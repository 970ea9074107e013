// MSE encode of large vectors (d a multiple of 256, 256 <= d <= 4096) on the 5th-generation
// tensor cores: y = Pi x / ||x||, idx_j = #{i : beta_i < y_j}, LSB-first bit-pack ("Google
// TurboQuant: 6x KV-cache compression" (ebisuda.net), "Stage 1"; the same arithmetic as
// encode_simt_kernel).
//
// The rotation is a dense GEMM, Y = X Pi^T, run as tcgen05 kind::f16 contractions with bf16
// operands and fp32 accumulators in tensor memory. Pi is split once per handle into a bf16
// pair, Pi = Pi_h + Pi_l (to ~2^-17); each row of x is split on the fly, x = x_h + x_l (exact for
// bf16 input, where x_l = 0 and its contraction is skipped). The accumulator takes
// x_h Pi_h^T + x_h Pi_l^T + x_l Pi_h^T (the x_l Pi_l term, ~2^-18, is dropped), so y is accurate to
// ~1e-6 of the unit scale, inside the 1e-5 band around a decision boundary where an index may
// differ from fp64.
//
// Tiles: a CTA owns 128 rows (tensor-memory lanes) at a time and walks the output coordinates in
// passes of 256 (MMA N), each pass a loop over K-chunks of 64 coordinates (one 128-byte swizzle
// atom of bf16); the two accumulators alternate between passes, so a pass's epilogue overlaps the
// next pass's MMAs.
//   warp 0, lane 0   TMA: Pi_h and Pi_l rows of the pass (two {64, 256} boxes), 2 stages
//   warp 1           tensor-memory allocation (512 columns); lane 0 issues the MMAs
//   warps 2-9        conversion: thread t owns half t / 128 of row t % 128's 64 inputs of the
//                    K-chunk (their loads for the next K-chunk in flight), and writes x_h, x_l into
//                    the swizzled A tiles (2 stages); in the first pass of a tile it also sums
//                    ||x||^2 in fp64, and the tile's norms go to smem and to the output
//   warps 10-13      epilogue: thread r reads row r of the pass's accumulator, scales by 1/||x||,
//                    bucketizes and packs the pass's 256 indices into the code row.
// The input is re-read (from L2) once per pass. Every wait is bounded; a wait that runs out sets
// an abort flag and the error word's kErrTimeout bit.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "encode_tc.cuh"
#include "search_tc.cuh"

namespace tqk {
namespace ebig {

using etc::bar_arrive;
using etc::expect_tx;
using etc::mma_commit;
using etc::mma_f16;
using etc::sts128;
using etc::sw128_desc;
using etc::tc_fence_after;
using etc::tc_fence_before;
using etc::tma_load_2d;
using etc::wait_bar;
using stc::bar_red_or;
using stc::tmem_ld16;

constexpr int kM = 128;          // rows per tile (tensor-memory lanes)
constexpr int kN = 256;          // output coordinates per pass (MMA N)
constexpr int kKC = 64;          // K-chunk: 64 bf16 = one 128-byte swizzle atom
constexpr int kStages = 2;
constexpr int kConvWarps = 8;    // two per row: each converts 32 of the K-chunk's 64 inputs
constexpr int kConvWarp0 = 2, kEpiWarp0 = kConvWarp0 + kConvWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);   // 14 warps
constexpr int kMinD = 256, kMaxD = 4096;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kAStage = 2u * kM * kKC * 2;   // 32 KB: x_h tile, then x_l tile
constexpr uint32_t kBStage = 2u * kN * kKC * 2;   // 64 KB: Pi_h rows, then Pi_l rows
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kAStage;     // 64 KB
constexpr uint32_t kOffNorm = kOffB + kStages * kBStage;  // 192 KB: float [2][kM] 1 / ||x|| (by tile parity)
constexpr uint32_t kOffSq = kOffNorm + 2 * kM * 4;        // double [2][kM] partial sums of x^2
constexpr uint32_t kOffTab = kOffSq + 2 * kM * 8;         // float [16] boundaries
constexpr uint32_t kOffBars = kOffTab + 64;
// a_full[S], a_empty[S], b_full[S], b_empty[S], acc_full[2], acc_empty[2], norm_ready
constexpr int kNumBars = 4 * kStages + 5;
constexpr uint32_t kOffTmemSlot = kOffBars + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4;
static_assert(kSmemBytes <= 232448, "encode_big layout exceeds the shared memory of one CTA");

struct Args {
  const void* x;       // [rows][d], x_dtype
  int x_dtype;
  int64_t rows;
  int d, bits, norm_dtype, codes_B;
  const float* bnd;    // [2^bits - 1]
  uint8_t* codes;      // [rows][codes_B]
  void* norms;         // [rows]
  int* err;
};

// Instruction descriptor, kind::f16: fp32 accumulate, A and B bf16, both K-major, M = 128, N = kN.
__host__ __device__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

// Waits for this thread's tensor-memory loads, with the loaded registers as operands.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

__device__ __forceinline__ uint32_t bf16_bits2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


// Half a row's 32 inputs of a K-chunk (element offset off of the row) as fp32 values.
template <int IN>
__device__ __forceinline__ void load_half(const void* x, int64_t elem, bool ok, float (&v)[32]) {
  if (!ok) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
    return;
  }
  if constexpr (IN == TQ_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + elem);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = __ldg(p + i);
      v[4 * i] = f.x, v[4 * i + 1] = f.y, v[4 * i + 2] = f.z, v[4 * i + 3] = f.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + elem);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldg(p + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if constexpr (IN == TQ_BF16) {
          v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
          v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        } else {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
          v[8 * i + 2 * j] = f.x, v[8 * i + 2 * j + 1] = f.y;
        }
      }
    }
  }
}

// pmap: Pi_h rows then Pi_l rows as a 2-D bf16 tensor {d, 2 d}, box {64, 256}, 128-byte swizzle.
// Grid: persistent CTAs over the 128-row tiles.
template <int IN>
__global__ void __launch_bounds__(kThreads, 1) encode_big_tc_kernel(const __grid_constant__ CUtensorMap pmap, Args a) {
  constexpr bool kLo = IN != TQ_BF16;   // x_l is zero for bf16 input
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = smem_addr(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = a.d, npass = d / kN, nkc = d / kKC;
  const int64_t ntiles = (a.rows + kM - 1) / kM;
  const int my_tiles = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  const int total = my_tiles * npass * nkc;   // K-chunks of this CTA

  const uint32_t bars = base + kOffBars;
  auto a_full = [&](int s) { return bars + 8u * s; };
  auto a_empty = [&](int s) { return bars + 8u * (kStages + s); };
  auto b_full = [&](int s) { return bars + 8u * (2 * kStages + s); };
  auto b_empty = [&](int s) { return bars + 8u * (3 * kStages + s); };
  auto acc_full = [&](int i) { return bars + 8u * (4 * kStages + i); };
  auto acc_empty = [&](int i) { return bars + 8u * (4 * kStages + 2 + i); };
  const uint32_t norm_ready = bars + 8u * (4 * kStages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  float* inv_s = reinterpret_cast<float*>(smem + kOffNorm);
  double* sq_s = reinterpret_cast<double*>(smem + kOffSq);
  float* bnd_s = reinterpret_cast<float*>(smem + kOffTab);

  if ((base & 1023u) != 0) {   // the swizzled operand layout needs 1024-byte alignment
    if (tid == 0) report_error(a.err, kErrInternal);
    return;
  }
  if (tid < 15) bnd_s[tid] = tid < (1 << a.bits) - 1 ? a.bnd[tid] : INFINITY;
  if (tid == 0) {
    *abort_flag = 0;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + kOffBars);
    for (int s = 0; s < kStages; ++s) {
      bar_init(b + s, kConvWarps);              // a_full: the conversion warps
      bar_init(b + kStages + s, 1);             // a_empty: MMA commit
      bar_init(b + 2 * kStages + s, 1);         // b_full: TMA
      bar_init(b + 3 * kStages + s, 1);         // b_empty: MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      bar_init(b + 4 * kStages + i, 1);         // acc_full: MMA commit
      bar_init(b + 4 * kStages + 2 + i, 4);     // acc_empty: the epilogue warps
    }
    bar_init(b + 4 * kStages + 4, kConvWarps / 2);   // norm_ready: the warps of the rows' first halves
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

  if (warp == 0) {
    // ---------------- TMA: Pi_h and Pi_l rows [256 p, 256 p + 256) of every K-chunk
    if (lane == 0) {
      int issued = 0;
      for (; issued < total; ++issued) {
        const int s = issued % kStages, kc = issued % nkc, pass = (issued / nkc) % npass;
        if (issued >= kStages && !*abort_flag && !wait_bar(b_empty(s), ((issued / kStages) - 1) & 1)) fail_wait();
        if (*abort_flag) break;
        expect_tx(b_full(s), kBStage);
        tma_load_2d(base + kOffB + s * kBStage, &pmap, kc * kKC, pass * kN, b_full(s));
        tma_load_2d(base + kOffB + s * kBStage + kBStage / 2, &pmap, kc * kKC, d + pass * kN, b_full(s));
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        (void)wait_bar(b_full(i % kStages), (i / kStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue: acc[pass % 2] += x_h Pi_h^T + x_h Pi_l^T (+ x_l Pi_h^T)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16();
      int it = 0, np = 0;   // K-chunks and passes issued
      for (int pt = 0; pt < my_tiles * npass && !*abort_flag; ++pt, ++np) {
        const int ai = pt & 1;
        if (pt >= 2 && !wait_bar(acc_empty(ai), ((pt >> 1) - 1) & 1)) { fail_wait(); break; }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(ai * kN);
        for (int kc = 0; kc < nkc; ++kc, ++it) {
          const int s = it % kStages;
          if (!wait_bar(a_full(s), (it / kStages) & 1) || !wait_bar(b_full(s), (it / kStages) & 1)) {
            fail_wait();
            break;
          }
          tc_fence_after();
          const uint32_t ab = base + kOffA + s * kAStage, bb = base + kOffB + s * kBStage;
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk) {
            const uint32_t off = kk * 32;
            const uint64_t ah = sw128_desc(ab + off), al = sw128_desc(ab + kAStage / 2 + off);
            const uint64_t bh = sw128_desc(bb + off), bl = sw128_desc(bb + kBStage / 2 + off);
            mma_f16(acc, ah, bh, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
            mma_f16(acc, ah, bl, idesc, 1u);
            if (kLo) mma_f16(acc, al, bh, idesc, 1u);
          }
          mma_commit(a_empty(s));
          mma_commit(b_empty(s));
        }
        if (*abort_flag) break;
        mma_commit(acc_full(ai));
      }
      // tensor memory is released below: make sure no MMA still writes it
      if (np > 0) (void)wait_bar(acc_full((np - 1) & 1), ((np - 1) >> 1) & 1);
    }
  } else if (warp < kEpiWarp0) {
    // ---------------- conversion: x -> x_h, x_l operand tiles; the tile's norms
    const int t = tid - 32 * kConvWarp0;      // 0 .. 255
    const int r = t & (kM - 1), h = t >> 7;   // row of the tile, half of the K-chunk
    float cur[32], nxt[32];
    auto fetch = [&](int itx, float(&v)[32]) {
      const int tl = itx / (npass * nkc), kc = itx % nkc;
      const int64_t row = ((int64_t)blockIdx.x + (int64_t)tl * gridDim.x) * kM + r;
      const bool ok = itx < total && row < a.rows;
      load_half<IN>(a.x, (ok ? row : 0) * d + kc * kKC + h * 32, ok, v);
    };
    fetch(0, cur);
    double sq = 0.0;
    for (int it = 0; it < total; ++it) {
      fetch(it + 1, nxt);
      const int s = it % kStages, kc = it % nkc, pass = (it / nkc) % npass, tl = it / (npass * nkc);
      bool ok = !*abort_flag;
      if (ok && it >= kStages && !wait_bar(a_empty(s), ((it / kStages) - 1) & 1)) { fail_wait(); ok = false; }
      // one decision for all conversion warps (they meet at a named barrier once per tile)
      if (bar_red_or(2, 32 * kConvWarps, !ok)) break;
      if (pass == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sq += (double)cur[i] * (double)cur[i];
      }
      const uint32_t ah = base + kOffA + s * kAStage + r * 128, al = ah + kAStage / 2;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {   // 8 inputs per 16-byte chunk
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float x0 = cur[8 * c4 + 2 * k], x1 = cur[8 * c4 + 2 * k + 1];
          hw[k] = bf16_bits2(x0, x1);
          lw[k] = kLo ? bf16_bits2(x0 - __uint_as_float(hw[k] << 16), x1 - __uint_as_float(hw[k] & 0xFFFF0000u)) : 0u;
        }
        const uint32_t o = (uint32_t)(((h * 4 + c4) ^ (r & 7)) << 4);
        sts128(ah + o, hw[0], hw[1], hw[2], hw[3]);
        if (kLo) sts128(al + o, lw[0], lw[1], lw[2], lw[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) bar_arrive(a_full(s));
      if (pass == 0 && kc == nkc - 1) {   // the tile's norms, from both halves' sums
        sq_s[h * kM + r] = sq;
        sq = 0.0;
        bar_red_or(2, 32 * kConvWarps, false);
        if (h == 0) {
          const int64_t row = ((int64_t)blockIdx.x + (int64_t)tl * gridDim.x) * kM + r;
          const double nn = sqrt(sq_s[r] + sq_s[kM + r]);
          inv_s[(tl & 1) * kM + r] = nn > 0.0 ? (float)(1.0 / nn) : 0.f;
          if (row < a.rows) store_norm(a.norms, a.norm_dtype, row, nn);
          __syncwarp();
          if (lane == 0) bar_arrive(norm_ready);
        }
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) cur[i] = nxt[i];
    }
  } else {
    // ---------------- epilogue: y = acc / ||x||, bucketize, pack 256 indices per pass
    const int quarter = warp & 3, r = 32 * quarter + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16);
    const int bits = a.bits, pbytes = kN * bits / 8;
    for (int pt = 0; pt < my_tiles * npass; ++pt) {
      const int tl = pt / npass, pass = pt % npass, ai = pt & 1;
      const int64_t row = ((int64_t)blockIdx.x + (int64_t)tl * gridDim.x) * kM + r;
      bool ok = !*abort_flag;
      if (ok && pass == 0 && !wait_bar(norm_ready, tl & 1)) { fail_wait(); ok = false; }
      if (ok && !wait_bar(acc_full(ai), (pt >> 1) & 1)) { fail_wait(); ok = false; }
      if (!__all_sync(0xffffffffu, ok)) break;   // tcgen05.ld is warp-collective
      tc_fence_after();
      const float inv = inv_s[(tl & 1) * kM + r];
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + (row < a.rows ? row : 0) * a.codes_B + pass * pbytes);
      uint64_t win = 0;
      int nb = 0, nw = 0;
#pragma unroll 1
      for (int cb = 0; cb < kN / 16; ++cb) {
        uint32_t v[16];
        tmem_ld16(lane_addr + ai * kN + 16 * cb, v);
        tmem_wait_ld16(v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float y = __uint_as_float(v[j]) * inv;
          // #{i : beta_i < y} over the sorted boundaries (padded with +inf to 15) by bisection
          int idx = (y > bnd_s[7]) ? 8 : 0;
          idx += (y > bnd_s[idx + 3]) ? 4 : 0;
          idx += (y > bnd_s[idx + 1]) ? 2 : 0;
          idx += (y > bnd_s[idx]) ? 1 : 0;
          win |= (uint64_t)idx << nb;
          nb += bits;
          if (nb >= 32) {
            if (row < a.rows) dst[nw] = (uint32_t)win;
            ++nw;
            win >>= 32;
            nb -= 32;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(acc_empty(ai));
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

}  // namespace ebig
}  // namespace tqk
