// Encode of 16-bit vectors at d = 128 on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// Computes exactly what encode_simt_kernel computes ("Google TurboQuant: 6x
// KV-cache compression" (ebisuda.net), "Stage 1" and "Stage 2"; "TurboQuant /
// PolarQuant / QJL technical deep dive" (gemilab.net), "PolarQuant"):
//   n = ||x|| (fp64), y = Pi x / n, idx_j = #{i : beta_i < y_j}, LSB-first bit-pack;
//   prod: e = y - c[idx], sigma_i = [ (M e)_i >= 0 ] with M = S Pi^T, rnorm = n ||e||.
//
// Both contractions are dense 128 x 128 x 128 tiles (128 vectors per tile):
//   D1 = X Pi^T      A = X (bf16 or f16, exact), B = Pi as a hi + lo pair of the same
//                    16-bit type (Pi = hi + lo to ~2^-17): two MMA passes;
//   D2 = E M^T       A = E as a bf16 hi + lo pair, B = M as a bf16 hi + lo pair:
//                    three passes (the lo x lo term, ~2^-18, is dropped).
// The rotated coordinates are then accurate to ~1e-6 of the unit scale, well inside the
// 1e-5 band around decision boundaries where an index or sign may differ from fp64.
//
// Shared-memory operands use the 128-byte-swizzled K-major layout: a 128 x 128 16-bit
// matrix is two 16 KB atoms (K 0..63, 64..127); row r of an atom occupies bytes
// [128 r, 128 r + 128) with its 16-byte chunk c stored at chunk position c ^ (r % 8).
// Pi and M arrive pre-swizzled from the handle; X tiles come by 2D TMA with the same
// swizzle; E is written by the epilogue threads in that layout.
//
// Roles (persistent CTAs, one per SM, over the CTA's tiles i = 0, 1, ...):
//   epilogue groups g = 0 .. G-1 of four warps (G = 4 MSE, 2 prod): group g owns the tiles
//     i = g (mod G) and its own accumulators in tensor memory; warp 4g + q reads TMEM lanes
//     32q .. 32q + 31, so every thread owns one vector (row) of the tile, all 128 columns;
//   warp 4G lane 0      producer: operand copies, then one X tile per stage;
//   warp 4G + 1         tensor-memory allocation; lane 0 issues each contraction as soon as
//                       its operands are staged and its accumulator has been read out.
// The norm: with fp16 storage it is ||D1 row|| = ||(Pi_hi + Pi_lo) x||, equal to ||x|| to
// ~1e-6 relative (far below an fp16 ulp); with fp32 storage it is summed in fp64 from the
// staged x. Up to 2 bits the compares run on the unnormalised row (acc > n beta_i) and the
// residual is kept as n e, whose signs under M and whose norm n ||e|| are what is stored.
// prod: the residual is parked in the row's own D1 columns (tcgen05.st) while the indices
// are packed, so the shared E tile is held only while it is copied out and contracted.
// Every wait is bounded; a wait that runs out sets an abort flag, after which no thread
// waits again and the error word records kErrTimeout.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace tqk {
namespace etc {

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr uint32_t kAtom = 16384;        // [128 rows][64 16-bit elements], 128-byte swizzled
constexpr uint32_t kMat = 2 * kAtom;     // a 128 x 128 16-bit operand
constexpr uint32_t kTmemCols = 512;      // MSE: D1 of groups 0..3; prod: D1 of groups 0, 1, then their D2

// Pre-swizzled operand block of a handle (d = 128): offsets of its 32 KB matrices.
constexpr uint32_t kOpPiBf16Hi = 0, kOpPiBf16Lo = 1, kOpMHi = 2, kOpMLo = 3, kOpPiF16Hi = 4, kOpPiF16Lo = 5;
constexpr uint32_t kOpCount = 6;

template <bool PROD>
struct Layout {
  static constexpr int kGroups = PROD ? 2 : 4;
  static constexpr int kStages = PROD ? 1 : 4;
  static constexpr int kThreads = (4 * kGroups + 2) * 32;
  static constexpr int kProducerWarp = 4 * kGroups, kMmaWarp = 4 * kGroups + 1;
  static constexpr uint32_t kPiHi = 0, kPiLo = kMat;
  static constexpr uint32_t kMHi = 2 * kMat, kMLo = 3 * kMat;            // prod only
  static constexpr uint32_t kX = PROD ? 4 * kMat : 2 * kMat;
  static constexpr uint32_t kEHi = kX + kStages * kMat, kELo = kEHi + kMat;  // prod only
  static constexpr uint32_t kOps = PROD ? kELo + kMat : kX + kStages * kMat;
  static constexpr uint32_t kTab = kOps;            // float[16] boundaries, float[16] centroids
  static constexpr uint32_t kBars = kTab + 128;
  // b_full, x_full[S], x_empty[S], d1_full[G], d1_empty[G], e_full, e_empty, d2_full[G], d2_empty[G]
  static constexpr int kNumBars = 1 + 2 * kStages + 4 * kGroups + 2;
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kXSeen = kAbort + 4;
  static constexpr uint32_t kBytes = kXSeen + 4;
  __host__ __device__ static constexpr uint32_t d1_col(int g) { return 128u * g; }
  __host__ __device__ static constexpr uint32_t d2_col(int g) { return 256u + 128u * g; }
};
static_assert(Layout<true>::kBytes <= 232448, "prod layout exceeds the shared memory of one CTA");

struct Args {
  int64_t rows;
  int norm_dtype;
  const uint8_t* ops;    // kOpCount pre-swizzled 32 KB matrices
  const float* cent;     // [2^bits]
  const float* bnd;      // [2^bits - 1]
  uint8_t* codes;
  int codes_B;
  uint8_t* signs;
  int signs_B;
  void* norms;
  __half* rnorms;
  int* err;
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
  for (int it = 0; it < (1 << 16); ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(20000)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// Shared-memory matrix descriptor: 128-byte swizzle, K-major, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;                // leading-dimension offset (unused with this swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;      // stride-dimension offset: next 8-row group
  d |= (uint64_t)1 << 46;                // descriptor version
  d |= (uint64_t)2 << 61;                // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulate, A and B of one 16-bit type
// (0 = f16, 1 = bf16), both K-major, M = 128, N = 128.
__host__ __device__ constexpr uint32_t mma_idesc(uint32_t ab_type) {
  return (1u << 4) | (ab_type << 7) | (ab_type << 10) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32], int o) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr + (uint32_t)o));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// Waits for this thread's tensor-memory loads with the 32 loaded registers as operands, so
// that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]),
                 "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]),
                 "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                 "+r"(v[30]), "+r"(v[31])
               :
               : "memory");
}

// Streams the 128 columns of this thread's row at tensor-memory address `col` through
// f(chunk, regs) in four 32-column chunks (the chunk loop is kept rolled: the epilogue
// groups run different parts of the kernel at once, and a compact body stays in the
// instruction cache).
template <typename F>
__device__ __forceinline__ void for_row_chunks(uint32_t col, bool ok, F&& f) {
#pragma unroll 1
  for (int c4 = 0; c4 < 4; ++c4) {
    uint32_t v[32];
    if (ok) {
      tmem_ld32(col, v, 32 * c4);
      tmem_wait_ld(v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0u;
    }
    f(c4, v);
  }
}

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

template <bool F16IN>
__device__ __forceinline__ float2 pair_to_float2(uint32_t w) {
  if (F16IN) return __half22float2(*reinterpret_cast<__half2*>(&w));
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Non-blocking probe of a barrier phase.
__device__ __forceinline__ bool test_bar(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t x) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n" ::"r"(taddr), "r"(x) : "memory");
}
__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t x, uint32_t y) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};\n" ::"r"(taddr), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&v)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}

// ---------------------------------------------------------------- kernel

template <int BITS, bool PROD, bool NORM32>
__global__ void __launch_bounds__(Layout<PROD>::kThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap xmap, Args a, int f16in) {
  using L = Layout<PROD>;
  constexpr int S = L::kStages, G = L::kGroups;
  constexpr int NB = (1 << BITS) - 1;
  constexpr bool kUnit = BITS > 2;   // 3 and 4 bits: normalise, then search the unit table
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = smem_addr(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t ntiles = (a.rows + kTile - 1) / kTile;
  const int my_tiles = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

  const uint32_t bars = base + L::kBars;
  const uint32_t b_full = bars;
  auto x_full = [&](int s) { return bars + 8u * (1 + s); };
  auto x_empty = [&](int s) { return bars + 8u * (1 + S + s); };
  auto d1_full = [&](int g) { return bars + 8u * (1 + 2 * S + g); };
  auto d1_empty = [&](int g) { return bars + 8u * (1 + 2 * S + G + g); };
  const uint32_t e_full = bars + 8u * (1 + 2 * S + 2 * G), e_empty = e_full + 8;
  auto d2_full = [&](int g) { return bars + 8u * (3 + 2 * S + 2 * G + g); };
  auto d2_empty = [&](int g) { return bars + 8u * (3 + 2 * S + 3 * G + g); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  volatile int* x_seen = reinterpret_cast<volatile int*>(smem + L::kXSeen);   // tiles whose copy has landed

  if ((base & 1023u) != 0) {   // the swizzled operand layout needs 1024-byte alignment
    if (tid == 0) report_error(a.err, kErrInternal);
    return;
  }
  float* bnd_s = reinterpret_cast<float*>(smem + L::kTab);
  float* cent_s = bnd_s + 16;
  if (tid < NB) bnd_s[tid] = a.bnd[tid];
  if (tid < (1 << BITS)) cent_s[tid] = a.cent[tid];
  if (tid == 0) {
    *abort_flag = 0;
    *x_seen = 0;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::kBars);
    bar_init(b, 1);
    for (int s = 0; s < S; ++s) {
      bar_init(b + 1 + s, 1);
      // freed by the first contraction's commit, and (fp32 norms) by the owning group reading x
      bar_init(b + 1 + S + s, NORM32 ? 1 + 4 : 1);
    }
    for (int g = 0; g < G; ++g) {
      bar_init(b + 1 + 2 * S + g, 1);          // d1_full[g]: MMA commit
      bar_init(b + 1 + 2 * S + G + g, 4);      // d1_empty[g]: the group's four warps
      bar_init(b + 3 + 2 * S + 2 * G + g, 1);  // d2_full[g]: MMA commit
      bar_init(b + 3 + 2 * S + 3 * G + g, 4);  // d2_empty[g]
    }
    bar_init(b + 1 + 2 * S + 2 * G, 4);        // e_full: the writing group's four warps
    bar_init(b + 2 + 2 * S + 2 * G, 1);        // e_empty: MMA commit
  }
  if (warp == L::kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(base + L::kTmemSlot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  auto fail_wait = [&]() {
    *abort_flag = 1;
    report_error(a.err, kErrTimeout);
  };

  if (warp == L::kProducerWarp) {
    if (lane == 0) {
      const uint32_t pi_hi = f16in ? kOpPiF16Hi : kOpPiBf16Hi, pi_lo = f16in ? kOpPiF16Lo : kOpPiBf16Lo;
      expect_tx(b_full, (PROD ? 4 : 2) * kMat);
      bulk_load(base + L::kPiHi, a.ops + pi_hi * kMat, kMat, b_full);
      bulk_load(base + L::kPiLo, a.ops + pi_lo * kMat, kMat, b_full);
      if (PROD) {
        bulk_load(base + L::kMHi, a.ops + kOpMHi * kMat, kMat, b_full);
        bulk_load(base + L::kMLo, a.ops + kOpMLo * kMat, kMat, b_full);
      }
      int issued = 0;
      for (; issued < my_tiles; ++issued) {
        const int64_t tile = blockIdx.x + (int64_t)issued * gridDim.x;
        const int s = issued % S;
        if (issued >= S && !*abort_flag && !wait_bar(x_empty(s), ((issued / S) - 1) & 1)) fail_wait();
        if (*abort_flag) break;
        expect_tx(x_full(s), kMat);
        tma_load_2d(base + L::kX + s * kMat, &xmap, 0, (int)(tile * kTile), x_full(s));
        tma_load_2d(base + L::kX + s * kMat + kAtom, &xmap, 64, (int)(tile * kTile), x_full(s));
      }
      // never leave with a copy still landing in this CTA's shared memory
      (void)wait_bar(b_full, 0);
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i) (void)wait_bar(x_full(i % S), (i / S) & 1);
    }
  } else if (warp == L::kMmaWarp) {
    if (lane == 0) {
      const uint32_t id_in = mma_idesc(f16in ? 0u : 1u), id_bf = mma_idesc(1u);
      uint32_t last_bar = 0, last_parity = 0;
      if (!wait_bar(b_full, 0)) fail_wait();
      // n1 / n2: this CTA's tiles whose first / second contraction has been issued
      int n1 = 0, n2 = 0;
      const int want2 = PROD ? my_tiles : 0;
      uint32_t idle = 0;
      while ((n1 < my_tiles || n2 < want2) && !*abort_flag) {
        bool progressed = false;
        if (n1 < my_tiles) {
          const int s = n1 % S, g = n1 % G;
          if (test_bar(x_full(s), (n1 / S) & 1) && (n1 < G || test_bar(d1_empty(g), ((n1 / G) - 1) & 1))) {
            tc_fence_after();
            const uint32_t d1 = tmem + L::d1_col(g);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
              const uint64_t ad = sw128_desc(base + L::kX + s * kMat + off);
              mma_f16(d1, ad, sw128_desc(base + L::kPiHi + off), id_in, kk > 0 ? 1u : 0u);
              mma_f16(d1, ad, sw128_desc(base + L::kPiLo + off), id_in, 1u);
            }
            mma_commit(d1_full(g));
            mma_commit(x_empty(s));
            last_bar = d1_full(g);
            last_parity = (n1 / G) & 1;
            ++n1;
            progressed = true;
          }
        }
        if (PROD && n2 < n1) {
          const int g = n2 % G;
          if (test_bar(e_full, n2 & 1) && (n2 < G || test_bar(d2_empty(g), ((n2 / G) - 1) & 1))) {
            tc_fence_after();
            const uint32_t d2 = tmem + L::d2_col(g);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
              const uint64_t eh = sw128_desc(base + L::kEHi + off), el = sw128_desc(base + L::kELo + off);
              const uint64_t mh = sw128_desc(base + L::kMHi + off), ml = sw128_desc(base + L::kMLo + off);
              mma_f16(d2, eh, mh, id_bf, kk > 0 ? 1u : 0u);
              mma_f16(d2, eh, ml, id_bf, 1u);
              mma_f16(d2, el, mh, id_bf, 1u);
            }
            mma_commit(d2_full(g));
            mma_commit(e_empty);
            last_bar = d2_full(g);
            last_parity = (n2 / G) & 1;
            ++n2;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else {
          if (++idle > (1u << 22)) { fail_wait(); break; }
          __nanosleep(32);
        }
      }
      // tensor memory is released below: make sure no MMA still writes it
      if (n1 > 0) (void)wait_bar(last_bar, last_parity);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (one row per thread)
    const int g = warp >> 2, q = warp & 3, r = 32 * q + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t d1 = lane_addr + L::d1_col(g), d2 = lane_addr + L::d2_col(g);
    float bnd[kUnit ? 1 : NB], cent[kUnit ? 1 : (1 << BITS)];
#pragma unroll
    for (int i = 0; i < (kUnit ? 0 : NB); ++i) bnd[i] = a.bnd[i];
#pragma unroll
    for (int i = 0; i < (kUnit ? 0 : (1 << BITS)); ++i) cent[i] = a.cent[i];
    for (int it = g; it < my_tiles; it += G) {
      const int use = it / G;   // how many tiles this group has taken before
      const int64_t tile = blockIdx.x + (int64_t)it * gridDim.x;
      const int s = it % S;
      const int64_t row = tile * kTile + r;
      const bool valid = row < a.rows;
      bool ok = !*abort_flag;

      // ---- ||x||^2
      double nn = 0.0;
      if (NORM32) {   // fp64 over the staged tile
        // With fewer stages than groups the stage is shared in tile order: wait until the
        // previous tile's copy has been seen to land, so that the barrier is in this tile's
        // phase (it cannot be further on: the next copy needs this group's release below)
        // and its parity cannot match an older, completed phase.
        if (S < G && ok) {
          uint32_t spins = 0;
          while (*x_seen < it && !*abort_flag) {
            if (++spins > (1u << 22)) { fail_wait(); ok = false; break; }
            __nanosleep(64);
          }
        }
        if (ok && !wait_bar(x_full(s), (it / S) & 1)) { fail_wait(); ok = false; }
        if (S < G && ok && lane == 0) atomicMax(const_cast<int*>(x_seen), it + 1);
        if (ok) {
          double p[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint4 w4 = lds128(base + L::kX + s * kMat + (c >> 3) * kAtom + r * 128 + (((c & 7) ^ (r & 7)) << 4));
            const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = f16in ? pair_to_float2<true>(w[k]) : pair_to_float2<false>(w[k]);
              p[k] = fma((double)f.x, (double)f.x, p[k]);
              p[k] = fma((double)f.y, (double)f.y, p[k]);
            }
          }
          nn = (p[0] + p[1]) + (p[2] + p[3]);
        }
        __syncwarp();
        if (lane == 0) bar_arrive(x_empty(s));
      }
      if (ok && !*abort_flag && !wait_bar(d1_full(g), use & 1)) { fail_wait(); ok = false; }
      ok = __all_sync(0xFFFFFFFFu, ok && !*abort_flag);   // tcgen05.ld / st are warp-collective
      if (ok) tc_fence_after();
      if (!NORM32 && ok) {   // ||D1 row||^2 in fp32, four chains
        float f[4] = {0.f, 0.f, 0.f, 0.f};
        for_row_chunks(d1, ok, [&](int, uint32_t(&c)[32]) {
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j & 3] = fmaf(__uint_as_float(c[j]), __uint_as_float(c[j]), f[j & 3]);
        });
        nn = ((double)f[0] + (double)f[1]) + ((double)f[2] + (double)f[3]);
      }
      const double n = sqrt(nn);
      const float nf = (float)n, inv = n > 0.0 ? (float)(1.0 / n) : 0.f;
      float thr[kUnit ? 1 : NB], nc[kUnit ? 1 : (1 << BITS)];
#pragma unroll
      for (int i = 0; i < (kUnit ? 0 : NB); ++i) thr[i] = n > 0.0 ? nf * bnd[i] : bnd[i];
#pragma unroll
      for (int i = 0; i < (kUnit ? 0 : (1 << BITS)); ++i) nc[i] = nf * cent[i];

      // ---- indices and packed words (32 coordinates -> BITS words per chunk); prod: residual
      //      back into the row's D1 columns
      if (valid && ok) store_norm(a.norms, a.norm_dtype, row, n);
      float esq[2] = {0.f, 0.f};
      for_row_chunks(d1, ok, [&](int c4, uint32_t(&v)[32]) {
        uint32_t words[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i) words[i] = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          uint32_t idx = 0;
          float e;
          if (!kUnit) {
            const float y = __uint_as_float(v[j]);
            float c = nc[0];
#pragma unroll
            for (int i = 0; i < (kUnit ? 0 : NB); ++i) {
              const bool gt = y > thr[i];
              idx += gt ? 1u : 0u;
              c = gt ? nc[i + 1] : c;
            }
            e = y - c;
          } else {
            const float y = __uint_as_float(v[j]) * inv;
#pragma unroll
            for (int step = 1 << (BITS - 1); step >= 1; step >>= 1) idx += (y > bnd_s[idx + step - 1]) ? step : 0u;
            e = PROD ? y - cent_s[idx] : 0.f;
          }
          const int bit = j * BITS;
          words[bit >> 5] |= idx << (bit & 31);
          if ((bit & 31) + BITS > 32) words[(bit >> 5) + 1] |= idx >> (32 - (bit & 31));
          if (PROD) {
            esq[j & 1] = fmaf(e, e, esq[j & 1]);
            v[j] = __float_as_uint(e);
          }
        }
        if (valid && ok) {
          uint8_t* dst = a.codes + row * (int64_t)a.codes_B + 4 * BITS * c4;
          if (BITS == 4) {
            *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1 % BITS], words[2 % BITS], words[3 % BITS]);
          } else if (BITS == 2) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1 % BITS]);
          } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) reinterpret_cast<uint32_t*>(dst)[i] = words[i];
          }
        }
        if (PROD && ok) {
          asm volatile(
              "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
              "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(d1 + 32 * c4),
              "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
              "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
              "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
              "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
              : "memory");
        }
      });
      if (!PROD) {
        if (ok) tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(d1_empty(g));
      } else {
        // ---- residual -> shared E tile (bf16 hi + lo, swizzled A layout), once the previous
        //      tile's second contraction has finished reading it
        if (ok) tmem_wait_st();
        if (ok && it > 0 && !*abort_flag && !wait_bar(e_empty, (it - 1) & 1)) { fail_wait(); ok = false; }
        ok = __all_sync(0xFFFFFFFFu, ok && !*abort_flag);
        for_row_chunks(d1, ok, [&](int c4, uint32_t(&v)[32]) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float e0 = __uint_as_float(v[8 * cc + 2 * k]), e1 = __uint_as_float(v[8 * cc + 2 * k + 1]);
              hi[k] = bf16x2_bits(e0, e1);
              lo[k] = bf16x2_bits(e0 - __uint_as_float(hi[k] << 16), e1 - __uint_as_float(hi[k] & 0xFFFF0000u));
            }
            if (ok) {
              const int c = 4 * (c4 & 1) + cc;   // chunk within the 64-column atom c4 / 2
              const uint32_t off = (c4 >> 1) * kAtom + r * 128 + (uint32_t)((c ^ (r & 7)) << 4);
              sts128(base + L::kEHi + off, hi[0], hi[1], hi[2], hi[3]);
              sts128(base + L::kELo + off, lo[0], lo[1], lo[2], lo[3]);
            }
          }
        });
        if (ok) tc_fence_before();
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          bar_arrive(d1_empty(g));
          bar_arrive(e_full);
        }
        // rnorm = n ||e||: the residual is n e below 3 bits, e from 3 bits on
        const double es = (double)esq[0] + (double)esq[1];
        if (valid && ok) a.rnorms[row] = __double2half(n > 0.0 ? (kUnit ? n * sqrt(es) : sqrt(es)) : 0.0);

        // ---- signs of z = D2: sigma = [z >= 0], all ones for a zero vector
        if (ok && !*abort_flag && !wait_bar(d2_full(g), use & 1)) { fail_wait(); ok = false; }
        ok = __all_sync(0xFFFFFFFFu, ok && !*abort_flag);
        if (ok) tc_fence_after();
        uint32_t* srow = reinterpret_cast<uint32_t*>(a.signs + row * (int64_t)a.signs_B);
        for_row_chunks(d2, ok, [&](int c4, uint32_t(&v)[32]) {
          uint32_t w = 0u;
#pragma unroll
          for (int j = 0; j < 32; ++j) w |= (__uint_as_float(v[j]) >= 0.f) ? (1u << j) : 0u;
          if (valid && ok) srow[c4] = (n == 0.0) ? 0xFFFFFFFFu : w;
        });
        if (ok) tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(d2_empty(g));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == L::kMmaWarp) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace etc
}  // namespace tqk
