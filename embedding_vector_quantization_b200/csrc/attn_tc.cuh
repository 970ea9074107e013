// Decode attention over 3-bit prod caches (2-bit Lloyd-Max codes + 1-bit QJL signs,
// m = 128) at d = 128 with 4 query heads per KV head, on the tcgen05 tensor cores.
//
// What is computed is tq_attn_decode's definition ("TurboQuant / PolarQuant / QJL
// technical deep dive" (gemilab.net), "Scaled dot-product attention"; "Google
// TurboQuant: 6x KV-cache compression" (ebisuda.net), "Stage 1" and "Stage 2"), with
// the same integer arithmetic as the mma.sync kernel in attn_mma.cuh (22-bit code-side
// queries, 15-bit QJL-side queries, 16-bit softmax weights against the chunk's largest
// p ||v|| and p rnorm, int32 sums); the weight steps come from per-head maxima of
// l + log2 ||v|| (and l + log2 rnorm) kept while the keys are scored, so the two
// kernels' weights can differ by one unit in the last place.
//
// Operand form. Bit s (0..7) of every packed byte gives a 0/1 byte plane; with the
// LSB-first packing, bit s of code byte cb is bit s % 2 of the index of coordinate
// 4 cb + s / 2, and bit s of sign byte sb is the sign of projection 8 sb + s. One
// token's operand row is its 8 code planes of 32 bytes followed by its 8 sign planes of
// 16 bytes: 384 bytes, word u = 8 s + k (code word k, u < 64), 64 + 4 s + k (sign word k).
//   * Keys: row = key (tensor-memory lane), K = the 384 row bytes (12 K-steps of 32): the
//     planes are written straight into tensor memory (tcgen05.st) and are the A operand
//     of `tcgen05.mma.kind::i8` with A in tensor memory; B holds the query pieces for
//     each (plane, byte): N = 32 columns, 3 h + {hi, mid, lo} of (c1 - c0) q' or
//     (c2 - c0) q' on the code K-steps, 12 + 2 h + {hi, lo} of S q on the sign K-steps.
//   * Values: the same rows in shared memory (128-byte swizzle, three 128-byte regions
//     per token) are the A operand read MN-major: row = one of 128 (plane, byte)
//     positions of a region, K = tokens; B = the integer weights of 32 tokens,
//     N = 16 columns (2 h + {hi, lo} of w1 = p ||v||, 8 + 2 h + {hi, lo} of w2 = p rnorm).
//     The accumulators hold sum_t w_t bit_t for every (coordinate, bit) and projection.
//
// Schedule. A persistent CTA per SM walks its items (sequence, KV head, chunk of at
// most 2048 tokens). Warp 0 streams 128-token tiles of codes and signs (keys of an item,
// then its values) through an 8-stage bulk-copy ring, and with each key tile the four
// norm rows of its tokens (||k||, rnorm_k, ||v||, rnorm_v) through an 8-stage norm ring;
// two groups of four warps (4-7, 8-11; alternate tiles) turn each tile into operand rows
// (thread = token); warp 1 issues the MMAs; warps 12-15 (thread = key)
// turn key accumulators into logits, then write each value tile's integer weights,
// and at the end of the item read the value sums and store the item's partial results
// ([B*Hq][nsplit][d + m + 2]: rotated-domain value sum, QJL sum, max, sum of weights,
// merged by the combine kernel). The copies of an item's tiles are issued while earlier
// work is still being scored, so the cold read of the cache stays in flight.
//
// Decode step: the kernel before this one (append + query rotation) writes only slot
// len[b] and the rotated queries. The copies never wait for it; the threads that read
// the new token (its codes and signs when expanding, its norms when scoring) do so from
// global memory after griddepcontrol.wait.
#pragma once

#include "common.cuh"
#include "encode_tc.cuh"
#include "attn_mma.cuh"

namespace tqk {
namespace atc {

using amma::Args;
using etc::bar_arrive;
using etc::bulk_load;
using etc::expect_tx;
using etc::mma_commit;
using etc::sw128_desc;
using etc::tc_fence_after;
using etc::tc_fence_before;
using etc::wait_bar;

constexpr int kD = 128, kM = 128, kG = 4;
constexpr int kT = 128;                    // tokens per tile
constexpr int kMaxChunk = 2048;            // tokens per item
constexpr int kRawStages = 8;
constexpr int kNS = 8;                     // norm stages (key tiles: ||k||, rnorm_k, ||v||, rnorm_v)
constexpr uint32_t kNormStage = 4 * kT * 2;
constexpr uint32_t kRawStage = kT * 48;    // codes (32 B per token), then signs (16 B)
constexpr int kAB = 2;                     // key operand buffers in tensor memory (96 columns each)
constexpr int kAcc = 2;                    // key accumulator sets (4 x 32 columns each: K-steps j % 4)
constexpr int kVP = 2;                     // value operand stages in shared memory
constexpr int kWS = 2;                     // weight operand stages
constexpr int kMmaWarp = 1, kExpWarp0 = 4, kEpiWarp0 = 12;   // two groups of four expansion warps
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColA = 0, kColV = 96 * kAB, kColAcc = 256;   // 0, 192 (3 x 16), 256 (2 x 128)

constexpr uint32_t kVPStage = 3 * kT * 128;                          // 48 KB: three regions of 128 rows
constexpr uint32_t kQBytes = 3 * 32 * 128;                           // 12 KB: 3 K-blocks x 32 rows
constexpr uint32_t kWStage = 16 * 128;                               // 2 KB: 16 rows x 128 tokens
constexpr uint32_t kOffVP = 0;
constexpr uint32_t kOffQ = kOffVP + kVP * kVPStage;                  //  98304
constexpr uint32_t kOffW = kOffQ + kQBytes;                          // 110592
constexpr uint32_t kOffRaw = kOffW + kWS * kWStage;                  // 114688
constexpr uint32_t kOffNrm = kOffRaw + kRawStages * kRawStage;       // 163840: half [kNS][4][kT]
constexpr uint32_t kOffLog = kOffNrm + kNS * kNormStage;              // 172032: float [4][kMaxChunk]
constexpr uint32_t kOffVN = kOffLog + kG * kMaxChunk * 4;            // 204800: half2 [kMaxChunk] (||v||, rnorm)
constexpr uint32_t kOffMisc = kOffVN + kMaxChunk * 4;                // 212992
// misc: red[4 warps][16] floats (256 B), hc[8][4] per-head constants (128 B), ired[4][8] ints (128 B)
constexpr uint32_t kOffRed = kOffMisc, kOffHc = kOffMisc + 256, kOffIred = kOffMisc + 384;
constexpr uint32_t kOffBars = kOffMisc + 512;
// barriers: raw_full[8], raw_empty[8], nrm_full[8], nrm_empty[8], a_full[4], a_empty[4], acc_full[2], acc_empty[2],
// vp_full[2], vp_empty[2], w_full[2], w_empty[2], q_full, vacc_full, vacc_empty, done
constexpr int kBRawF = 0, kBRawE = kBRawF + kRawStages, kBNF = kBRawE + kRawStages, kBNE = kBNF + kNS;
constexpr int kBAF = kBNE + kNS, kBAE = kBAF + kAB;
constexpr int kBAccF = kBAE + kAB, kBAccE = kBAccF + kAcc, kBVPF = kBAccE + kAcc, kBVPE = kBVPF + kVP;
constexpr int kBWF = kBVPE + kVP, kBWE = kBWF + kWS, kBQF = kBWE + kWS, kBVAF = kBQF + 1, kBVAE = kBVAF + 1;
constexpr int kBDone = kBVAE + 1, kNumBars = kBDone + 1;
constexpr uint32_t kOffTmemSlot = kOffBars + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4;
static_assert(kSmemBytes <= 232448, "attention layout exceeds the shared memory of one CTA");
static_assert(kColV + 48 <= kColAcc && kColAcc + 128 * kAcc <= kTmemCols, "tensor-memory columns");

// Instruction descriptors, kind::i8, int32 accumulate, M = 128.
// Keys: A (tensor memory) and B signed 8-bit, K-major, N = 32.
// Values: A and B unsigned 8-bit, A MN-major (transposed), B K-major, N = 16.
__host__ __device__ constexpr uint32_t idesc_key() {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(32 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_val() {
  return (2u << 4) | (0u << 7) | (0u << 10) | (1u << 15) | ((uint32_t)(16 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: 128 M rows of
// one byte per K index are one swizzle row; 8 K indices make a 1024-byte atom, and the
// atoms of consecutive K groups follow each other (1024 bytes apart). Both offset fields
// hold 1024: one is the K-group stride, the other the stride between atoms along M, of
// which there is only one.
__device__ __forceinline__ uint64_t mn_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(1024 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// MMA with A in tensor memory (lane = row, 8 columns per 32 K bytes).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&v)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr));
}
template <int N>
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; i += 4)
    asm volatile("" : "+r"(v[i]), "+r"(v[i + 1]), "+r"(v[i + 2]), "+r"(v[i + 3]));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ void sts8(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;\n" ::"r"(a), "r"(v) : "memory");
}
// Asks the L2 to fetch [p, p + bytes) (16-byte aligned, bytes a multiple of 16); no completion.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool bar_red_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Byte offset of (row n, K byte col) in a K-major tile of 128-byte rows with the 128-byte
// swizzle (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t swz(int n, int col) {
  return (uint32_t)((n >> 3) * 1024 + (n & 7) * 128 + ((((col >> 4) ^ (n & 7)) & 7) << 4) + (col & 15));
}

// One work item: (sequence, KV head, chunk).
struct Item {
  int b, bh, split, ntok, nk;
  int64_t start, row0;
  int s_loc;   // the new token's position in the chunk (decode step), else -1
};

__device__ __forceinline__ Item item_of(const Args& a, int it) {
  Item x;
  x.bh = it / a.nsplit;
  x.split = it - x.bh * a.nsplit;
  x.b = x.bh / a.Hkv;
  const int64_t L = min((int64_t)max(a.len[x.b], 0) + a.len_extra, a.L_cap);
  x.start = (int64_t)x.split * a.chunk;
  const int64_t end = min(L, x.start + a.chunk);
  x.ntok = (int)max((int64_t)0, end - x.start);
  x.nk = (x.ntok + kT - 1) / kT;
  x.row0 = (int64_t)x.bh * a.L_cap + x.start;
  const int64_t slot = (int64_t)max(a.len[x.b], 0);
  x.s_loc = (a.len_extra && slot >= x.start && slot < end) ? (int)(slot - x.start) : -1;
  return x;
}

// The 32 operand words of block blk (0: code planes 0-3, 1: code planes 4-7, 2: sign
// planes) of a token with code words cw and sign words sw.
__device__ __forceinline__ void plane_block(const uint32_t (&cw)[8], const uint32_t (&sw)[4], int blk,
                                            uint32_t (&o)[32]) {
  if (blk < 2) {
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
      for (int k = 0; k < 8; ++k) o[8 * s4 + k] = (cw[k] >> (4 * blk + s4)) & 0x01010101u;
  } else {
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
      for (int k = 0; k < 4; ++k) o[4 * s + k] = (sw[k] >> s) & 0x01010101u;
  }
}

// Grid: min(items, SMs) persistent CTAs; CTA c takes items c, c + grid, ...
__global__ void __launch_bounds__(kThreads, 1) attn_prod2_tc_kernel(Args a, int nitems) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = smem_addr(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t bars = base + kOffBars;
  auto bar = [=](int i) { return bars + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  int* const err = a.err;
  if ((base & 1023u) != 0) {   // the swizzled operand tiles need 1024-byte alignment
    if (tid == 0) report_error(err, kErrInternal);
    return;
  }
  if (tid == 0) {
    *abort_flag = 0;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + kOffBars);
    for (int s = 0; s < kRawStages; ++s) {
      bar_init(b + kBRawF + s, 1);
      bar_init(b + kBRawE + s, 4);   // the four expansion warps
    }
    for (int s = 0; s < kNS; ++s) {
      bar_init(b + kBNF + s, 1);
      bar_init(b + kBNE + s, 4);     // the four epilogue warps
    }
    for (int s = 0; s < kAB; ++s) {
      bar_init(b + kBAF + s, 4);
      bar_init(b + kBAE + s, 1);     // MMA commit
    }
    for (int s = 0; s < kAcc; ++s) {
      bar_init(b + kBAccF + s, 1);
      bar_init(b + kBAccE + s, 4);   // the four epilogue warps
    }
    for (int s = 0; s < kVP; ++s) {
      bar_init(b + kBVPF + s, 4);
      bar_init(b + kBVPE + s, 1);
    }
    for (int s = 0; s < kWS; ++s) {
      bar_init(b + kBWF + s, 4);
      bar_init(b + kBWE + s, 1);
    }
    bar_init(b + kBQF, 4);
    bar_init(b + kBVAF, 1);
    bar_init(b + kBVAE, 4);
    bar_init(b + kBDone, 1);
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(base + kOffTmemSlot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemSlot);
  grid_dep_launch();
  auto fail = [=]() {
    *abort_flag = 1;
    report_error(err, kErrTimeout);
  };

  if (warp == 0) {
    // ---------------- bulk copies: code and sign rows of every tile (keys of an item, then values)
    if (lane == 0) {
      // Every row of an item is requested into L2 one item ahead (the first item at launch), so
      // the cold read streams at full rate whatever the depth of the copy ring; the ring's copies
      // then come from L2.
      auto prefetch_item = [&](int it) {
        if (it >= nitems) return;
        const Item y = item_of(a, it);
        if (y.ntok == 0) return;
        const uint32_t n = (uint32_t)y.ntok, n8 = (n + 7u) & ~7u;
        prefetch_l2(a.kcodes + y.row0 * 32, n * 32u);
        prefetch_l2(a.ksigns + y.row0 * 16, n * 16u);
        prefetch_l2(a.knorm + y.row0, n8 * 2u);
        prefetch_l2(a.krn + y.row0, n8 * 2u);
        prefetch_l2(a.vnorm + y.row0, n8 * 2u);
        prefetch_l2(a.vrn + y.row0, n8 * 2u);
        prefetch_l2(a.vcodes + y.row0 * 32, n * 32u);
        prefetch_l2(a.vsigns + y.row0 * 16, n * 16u);
      };
      prefetch_item(blockIdx.x);
      int rit = 0, nit = 0;
      bool stop = false;
      for (int it = blockIdx.x; it < nitems && !stop; it += gridDim.x) {
        const Item x = item_of(a, it);
        prefetch_item(it + gridDim.x);
        for (int kind = 0; kind < 2 && !stop; ++kind) {
          const uint8_t* cg = kind ? a.vcodes : a.kcodes;
          const uint8_t* sg = kind ? a.vsigns : a.ksigns;
          for (int t = 0; t < x.nk; ++t, ++rit) {
            const int s = rit % kRawStages;
            if (*abort_flag) { stop = true; break; }
            if (rit >= kRawStages && !wait_bar(bar(kBRawE + s), ((rit / kRawStages) - 1) & 1)) {
              fail();
              stop = true;
              break;
            }
            const uint32_t n = (uint32_t)min(kT, x.ntok - t * kT);
            const int64_t r = x.row0 + (int64_t)t * kT;
            const uint32_t st = base + kOffRaw + (uint32_t)s * kRawStage;
            if (kind == 0) {
              // the key tile's norms and the values' norms (whole 8-token groups: L_cap % 8 == 0 and
              // chunks start on 128-token boundaries, so the rounded rows stay inside the sequence)
              const int ns = nit % kNS;
              if (nit >= kNS && !wait_bar(bar(kBNE + ns), ((nit / kNS) - 1) & 1)) {
                fail();
                stop = true;
                break;
              }
              const uint32_t n8 = (n + 7u) & ~7u;
              const uint32_t nst = base + kOffNrm + (uint32_t)ns * kNormStage;
              expect_tx(bar(kBNF + ns), n8 * 8u);
              bulk_load(nst, a.knorm + r, n8 * 2u, bar(kBNF + ns));
              bulk_load(nst + kT * 2, a.krn + r, n8 * 2u, bar(kBNF + ns));
              bulk_load(nst + kT * 4, a.vnorm + r, n8 * 2u, bar(kBNF + ns));
              bulk_load(nst + kT * 6, a.vrn + r, n8 * 2u, bar(kBNF + ns));
              ++nit;
            }
            expect_tx(bar(kBRawF + s), n * 48u);
            bulk_load(st, cg + r * 32, n * 32u, bar(kBRawF + s));
            bulk_load(st + kT * 32, sg + r * 16, n * 16u, bar(kBRawF + s));
          }
        }
      }
      // never leave with a copy still landing in this CTA's shared memory
      for (int i = max(rit - kRawStages, 0); i < rit; ++i)
        (void)wait_bar(bar(kBRawF + i % kRawStages), (uint32_t)(i / kRawStages) & 1u);
      for (int i = max(nit - kNS, 0); i < nit; ++i)
        (void)wait_bar(bar(kBNF + i % kNS), (uint32_t)(i / kNS) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (one thread)
    if (lane == 0) {
      int ait = 0, cit = 0, vit = 0, ai = 0;
      bool stop = false;
      for (int it = blockIdx.x; it < nitems && !stop; it += gridDim.x) {
        const Item x = item_of(a, it);
        if (x.nk == 0) continue;
        if (*abort_flag) break;
        if (!wait_bar(bar(kBQF), ai & 1)) { fail(); break; }
        tc_fence_after();
        // key tiles: 12 K-steps of the 384 operand bytes into one 32-column accumulator
        for (int t = 0; t < x.nk; ++t, ++ait, ++cit) {
          const int ab = ait % kAB, cb = cit % kAcc;
          if (*abort_flag) { stop = true; break; }
          if (!wait_bar(bar(kBAF + ab), (ait / kAB) & 1) ||
              (cit >= kAcc && !wait_bar(bar(kBAccE + cb), ((cit / kAcc) - 1) & 1))) {
            fail();
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t acol = tmem + kColA + 96u * ab, dcol = tmem + kColAcc + 128u * cb;
          // K-step j accumulates into sub-accumulator j % 4: four independent chains of three MMAs
          // (one chain of twelve small MMAs would run at the tensor pipe's latency, not its rate)
#pragma unroll
          for (int j = 0; j < 12; ++j) {
            const uint64_t bd = sw128_desc(base + kOffQ + (uint32_t)(j >> 2) * 4096u + (uint32_t)(j & 3) * 32u);
            mma_ts(dcol + 32u * (j & 3), acol + 8u * j, bd, idesc_key(), j >= 4 ? 1u : 0u);
          }
          mma_commit(bar(kBAE + ab));
          mma_commit(bar(kBAccF + cb));
        }
        if (stop) break;
        // value tiles: three regions x 4 K-steps of 32 tokens, accumulated over the item
        for (int t = 0; t < x.nk; ++t, ++vit) {
          const int vb = vit % kVP, wb = vit % kWS;
          if (*abort_flag) { stop = true; break; }
          if (!wait_bar(bar(kBVPF + vb), (vit / kVP) & 1) || !wait_bar(bar(kBWF + wb), (vit / kWS) & 1) ||
              (t == 0 && ai >= 1 && !wait_bar(bar(kBVAE), (ai - 1) & 1))) {
            fail();
            stop = true;
            break;
          }
          tc_fence_after();
          // the three regions' chains interleaved
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int g = 0; g < 3; ++g) {
              const uint64_t ad = mn_desc(base + kOffVP + (uint32_t)vb * kVPStage + g * 16384u + j * 4096u);
              const uint64_t bd = sw128_desc(base + kOffW + (uint32_t)wb * kWStage + j * 32u);
              mma_ss(tmem + kColV + 16u * g, ad, bd, idesc_val(), (t > 0 || j > 0) ? 1u : 0u);
            }
          mma_commit(bar(kBVPE + vb));
          mma_commit(bar(kBWE + wb));
        }
        if (stop) break;
        mma_commit(bar(kBVAF));
        ++ai;
      }
      // tensor memory is released below: no MMA may still be running
      mma_commit(bar(kBDone));
      (void)wait_bar(bar(kBDone), 0);
    }
  } else if (warp >= kExpWarp0 && warp < kEpiWarp0) {
    // ---------------- expansion: thread = token row of the tile (and tensor-memory lane)
    // group g (warps 4 + 4g .. 7 + 4g) takes the tiles whose sequence number has parity g
    const int grp = (warp - kExpWarp0) >> 2, q4 = warp & 3, r = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    int rit = 0, ait = 0, vit = 0;
    bool waited = false, stop = false;
    for (int it = blockIdx.x; it < nitems && !stop; it += gridDim.x) {
      const Item x = item_of(a, it);
      for (int kind = 0; kind < 2 && !stop; ++kind) {
        for (int t = 0; t < x.nk; ++t, ++rit) {
          if ((rit & 1) != grp) {   // the other group's tile
            if (kind == 0) ++ait;
            else ++vit;
            continue;
          }
          const int s = rit % kRawStages;
          bool ok = !*abort_flag;
          if (ok && !wait_bar(bar(kBRawF + s), (rit / kRawStages) & 1)) { fail(); ok = false; }
          if (!__all_sync(0xffffffffu, ok)) { stop = true; break; }
          const int tok = t * kT + r;
          uint32_t cw[8], sw[4];
#pragma unroll
          for (int i = 0; i < 8; ++i) cw[i] = 0u;
#pragma unroll
          for (int i = 0; i < 4; ++i) sw[i] = 0u;
          if (tok < x.ntok) {
            if (tok == x.s_loc) {
              // the token the previous kernel appended: its rows as that kernel wrote them
              if (!waited) {
                grid_dep_wait();
                waited = true;
              }
              const int64_t row = x.row0 + tok;
              const uint4* cp = reinterpret_cast<const uint4*>((kind ? a.vcodes : a.kcodes) + row * 32);
              const uint4 c0 = __ldcg(cp), c1 = __ldcg(cp + 1);
              const uint4 s0 = __ldcg(reinterpret_cast<const uint4*>((kind ? a.vsigns : a.ksigns) + row * 16));
              cw[0] = c0.x, cw[1] = c0.y, cw[2] = c0.z, cw[3] = c0.w, cw[4] = c1.x, cw[5] = c1.y, cw[6] = c1.z,
              cw[7] = c1.w;
              sw[0] = s0.x, sw[1] = s0.y, sw[2] = s0.z, sw[3] = s0.w;
            } else {
              const uint4* cp = reinterpret_cast<const uint4*>(smem + kOffRaw + s * kRawStage + r * 32);
              const uint4 c0 = cp[0], c1 = cp[1];
              const uint4 s0 = *reinterpret_cast<const uint4*>(smem + kOffRaw + s * kRawStage + kT * 32 + r * 16);
              cw[0] = c0.x, cw[1] = c0.y, cw[2] = c0.z, cw[3] = c0.w, cw[4] = c1.x, cw[5] = c1.y, cw[6] = c1.z,
              cw[7] = c1.w;
              sw[0] = s0.x, sw[1] = s0.y, sw[2] = s0.z, sw[3] = s0.w;
            }
          }
          __syncwarp();
          if (lane == 0) bar_arrive(bar(kBRawE + s));   // the stage's rows are in registers
          if (kind == 0) {
            const int ab = ait % kAB;
            ok = true;
            if (ait >= kAB && !wait_bar(bar(kBAE + ab), ((ait / kAB) - 1) & 1)) { fail(); ok = false; }
            if (!__all_sync(0xffffffffu, ok)) { stop = true; break; }
            tc_fence_after();
#pragma unroll
            for (int blk = 0; blk < 3; ++blk) {
              uint32_t o[32];
              plane_block(cw, sw, blk, o);
              tmem_st32(lane_base + kColA + 96u * ab + 32u * blk, o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) bar_arrive(bar(kBAF + ab));
            ++ait;
          } else {
            const int vb = vit % kVP;
            ok = true;
            if (vit >= kVP && !wait_bar(bar(kBVPE + vb), ((vit / kVP) - 1) & 1)) { fail(); ok = false; }
            if (!__all_sync(0xffffffffu, ok)) { stop = true; break; }
            const uint32_t rowa = base + kOffVP + (uint32_t)vb * kVPStage + (uint32_t)r * 128u;
#pragma unroll
            for (int blk = 0; blk < 3; ++blk) {
              uint32_t o[32];
              plane_block(cw, sw, blk, o);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                sts128(rowa + blk * 16384u + (uint32_t)((c ^ (r & 7)) << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2],
                       o[4 * c + 3]);
            }
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) bar_arrive(bar(kBVPF + vb));
            ++vit;
          }
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------- epilogue: thread = key / token row of the tile (and tensor-memory lane)
    const int q4 = warp - kEpiWarp0, r = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    float* logit = reinterpret_cast<float*>(smem + kOffLog);   // [head][kMaxChunk], log2 units
    __half2* vnr = reinterpret_cast<__half2*>(smem + kOffVN);  // (||v||, rnorm) of the chunk's tokens
    float* red = reinterpret_cast<float*>(smem + kOffRed);     // [warp][16]
    float* hc = reinterpret_cast<float*>(smem + kOffHc);       // [head][4]: c0 sum(q'), code step, sign step, sum(S q)
    int* ired = reinterpret_cast<int*>(smem + kOffIred);       // [warp][8]
    const float scale2 = a.scale * 1.4426950408889634f;
    const float kqjl = kQjlScale / (float)kM;
    const int stride = partial_stride(kD, kM);
    const uint32_t qtile = base + kOffQ;
    // the query operand's bytes that no item writes (rows 12-19 of the code K-blocks, 0-11 of the
    // sign K-block, 20-31 of all) stay zero; every item rewrites all the others
    for (int i = r; i < (int)(kQBytes / 16); i += 128) sts128(qtile + 16u * i, 0u, 0u, 0u, 0u);
    named_bar(1, 128);
    grid_dep_wait();   // the rotated queries (and the new token's norms) come from the kernel before this one
    int cit = 0, wit = 0, ai = 0, nit = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
      const Item x = item_of(a, it);
      const size_t hq0 = (size_t)x.b * a.Hq + (size_t)(x.bh % a.Hkv) * kG;   // the item's first query head
      if (x.nk == 0) {   // an empty chunk: zero sums and max -inf
        for (int i = r; i < kG * stride; i += 128) {
          const int h = i / stride, j = i - h * stride;
          a.part[((hq0 + h) * a.nsplit + x.split) * stride + j] = (j == kD + kM) ? -INFINITY : 0.f;
        }
        continue;
      }
      if (bar_red_or(1, 128, *abort_flag != 0)) break;

      // ---- query operand of the item: each warp scatters one head's pieces
      {
        const int h = q4;
        const float* qr = a.qr + (hq0 + h) * kD;
        const float* qs = a.qs + (hq0 + h) * kM;
        float x0[4], x1[4], xs[4], sq = 0.f, ss = 0.f, mx = 0.f, ms = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float q = qr[lane + 32 * i], sv = qs[lane + 32 * i];
          x0[i] = a.kb0 * q;
          x1[i] = a.kb1 * q;
          xs[i] = sv;
          sq += q;
          ss += sv;
          mx = fmaxf(mx, fmaxf(fabsf(x0[i]), fabsf(x1[i])));
          ms = fmaxf(ms, fabsf(sv));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sq += __shfl_xor_sync(0xffffffffu, sq, o);
          ss += __shfl_xor_sync(0xffffffffu, ss, o);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
        }
        const float dm = mx > 0.f ? mx / amma::kQMax : 1.f;
        const float ds = ms > 0.f ? ms / amma::kSMax : 1.f;
        const float idm = 1.f / dm, ids = 1.f / ds;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = lane + 32 * i;
#pragma unroll
          for (int beta = 0; beta < 2; ++beta) {
            // 22-bit integer hi * 2^14 + mid * 2^7 + lo of (c_{1+beta} - c0) q'_c / step
            const int xi = __float2int_rn((beta ? x1[i] : x0[i]) * idm);
            const int hi = (xi >= 0) ? (xi + 8192) >> 14 : -((-xi + 8192) >> 14);
            const int rr = xi - hi * 16384;
            const int mid = (rr >= 0) ? (rr + 64) >> 7 : -((-rr + 64) >> 7);
            const int j = 2 * (c & 3) + beta, col = 32 * (j & 3) + (c >> 2);   // K-step = plane, byte = c / 4
            const uint32_t kb = qtile + (uint32_t)(j >> 2) * 4096u;
            sts8(kb + swz(3 * h, col), (uint32_t)(hi & 255));
            sts8(kb + swz(3 * h + 1, col), (uint32_t)(mid & 255));
            sts8(kb + swz(3 * h + 2, col), (uint32_t)((rr - mid * 128) & 255));
          }
          {
            // 15-bit integer hi * 2^7 + lo of (S q)_p / step, p = c: sign byte p / 8, plane p % 8
            const int xi = __float2int_rn(xs[i] * ids);
            const int hi = (xi >= 0) ? (xi + 64) >> 7 : -((-xi + 64) >> 7);
            const int sb = c >> 3, sp = c & 7;
            const int col = 32 * (sp >> 1) + 16 * (sp & 1) + sb;   // K-step 8 + sp / 2
            const uint32_t kb = qtile + 2u * 4096u;
            sts8(kb + swz(12 + 2 * h, col), (uint32_t)(hi & 255));
            sts8(kb + swz(13 + 2 * h, col), (uint32_t)((xi - 128 * hi) & 255));
          }
        }
        if (lane == 0) {
          hc[4 * h + 0] = a.kc0 * sq;
          hc[4 * h + 1] = dm;
          hc[4 * h + 2] = ds;
          hc[4 * h + 3] = ss;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      named_bar(1, 128);
      if (lane == 0) bar_arrive(bar(kBQF));
      float c0h[kG], dmh[kG], dsh[kG], ssh[kG];
#pragma unroll
      for (int h = 0; h < kG; ++h) c0h[h] = hc[4 * h], dmh[h] = hc[4 * h + 1], dsh[h] = hc[4 * h + 2], ssh[h] = hc[4 * h + 3];

      // ---- key tiles: logits (log2 units) and, per head, the maxima of l, l + log2 ||v||, l + log2 rnorm
      float hm[kG], a1[kG], a2[kG];
#pragma unroll
      for (int h = 0; h < kG; ++h) hm[h] = a1[h] = a2[h] = -INFINITY;
      // A failed wait makes this warp skip the rest of its waits and tensor-memory accesses; the
      // warps agree at the next CTA-wide point (bar.red) and leave together.
      bool bad = false;
      for (int t = 0; t < x.nk; ++t, ++cit, ++nit) {
        const int cb = cit % kAcc, ns = nit % kNS;
        const int tok = t * kT + r;
        const bool valid = tok < x.ntok;
        bool ok = !bad && !*abort_flag;
        if (ok && !wait_bar(bar(kBNF + ns), (nit / kNS) & 1)) { fail(); ok = false; }
        bad = !__all_sync(0xffffffffu, ok);
        if (bad) break;
        float kn = 0.f, krn = 0.f;
        __half2 vv = __floats2half2_rn(0.f, 0.f);
        if (valid) {
          if (tok == x.s_loc) {   // the appended token: its norms as the previous kernel wrote them
            const int64_t row = x.row0 + tok;
            kn = __half2float(__ldcg(a.knorm + row));
            krn = __half2float(__ldcg(a.krn + row));
            vv = __halves2half2(__ldcg(a.vnorm + row), __ldcg(a.vrn + row));
          } else {
            const __half* nst = reinterpret_cast<const __half*>(smem + kOffNrm + ns * kNormStage);
            kn = __half2float(nst[r]);
            krn = __half2float(nst[kT + r]);
            vv = __halves2half2(nst[2 * kT + r], nst[3 * kT + r]);
          }
        }
        __syncwarp();
        if (lane == 0) bar_arrive(bar(kBNE + ns));
        ok = !*abort_flag;
        if (ok && !wait_bar(bar(kBAccF + cb), (cit / kAcc) & 1)) { fail(); ok = false; }
        bad = !__all_sync(0xffffffffu, ok);
        if (bad) break;
        tc_fence_after();
        int acc[20];
#pragma unroll
        for (int c = 0; c < 20; ++c) acc[c] = 0;
#pragma unroll
        for (int u2 = 0; u2 < 4; u2 += 2) {   // the four sub-accumulators, two at a time
          uint32_t v[2][16], w4[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            tmem_ld16(lane_base + kColAcc + 128u * cb + 32u * (u2 + u), v[u]);
            tmem_ld4(lane_base + kColAcc + 128u * cb + 32u * (u2 + u) + 16u, w4[u]);
          }
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            tmem_wait_ld_regs(v[u]);
            tmem_wait_ld_regs(w4[u]);
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] += (int)v[u][c];
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[16 + c] += (int)w4[u][c];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(bar(kBAccE + cb));
        if (valid) {
          const float2 nv = __half22float2(vv);
          const float lv = __log2f(nv.x), lr = __log2f(nv.y);
#pragma unroll
          for (int h = 0; h < kG; ++h) {
            // exact in int32: 256 (plane, byte) positions of |piece| <= 127, times 2^14
            const int mse = acc[3 * h] * 16384 + acc[3 * h + 1] * 128 + acc[3 * h + 2];
            const int qjl = acc[12 + 2 * h] * 128 + acc[13 + 2 * h];
            const float sc = kn * (c0h[h] + dmh[h] * (float)mse) + krn * kqjl * (2.f * dsh[h] * (float)qjl - ssh[h]);
            const float l = sc * scale2;
            logit[h * kMaxChunk + tok] = l;
            hm[h] = fmaxf(hm[h], l);
            a1[h] = fmaxf(a1[h], l + lv);
            a2[h] = fmaxf(a2[h], l + lr);
          }
          vnr[tok] = vv;
        }
      }
      if (bar_red_or(1, 128, bad)) break;
#pragma unroll
      for (int h = 0; h < kG; ++h)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          hm[h] = fmaxf(hm[h], __shfl_xor_sync(0xffffffffu, hm[h], o));
          a1[h] = fmaxf(a1[h], __shfl_xor_sync(0xffffffffu, a1[h], o));
          a2[h] = fmaxf(a2[h], __shfl_xor_sync(0xffffffffu, a2[h], o));
        }
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < kG; ++h) red[16 * q4 + h] = hm[h], red[16 * q4 + 4 + h] = a1[h], red[16 * q4 + 8 + h] = a2[h];
      named_bar(1, 128);
      // weights: w1 = p ||v|| / st1, w2 = p rnorm / st2, the steps being each head's largest p ||v||
      // and p rnorm of the chunk over 65535 (16-bit weights, split into 8-bit pieces hi * 256 + lo)
      float M[kG], st1[kG], st2[kG], inv1[kG], inv2[kG];
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        float m = -INFINITY, x1m = -INFINITY, x2m = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          m = fmaxf(m, red[16 * w + h]);
          x1m = fmaxf(x1m, red[16 * w + 4 + h]);
          x2m = fmaxf(x2m, red[16 * w + 8 + h]);
        }
        M[h] = m;
        const float s1 = exp2f(x1m - m) / 65535.f, s2 = exp2f(x2m - m) / 65535.f;
        st1[h] = s1 > 0.f ? s1 : 1.f;
        inv1[h] = s1 > 0.f ? 1.f / s1 : 0.f;
        st2[h] = s2 > 0.f ? s2 : 1.f;
        inv2[h] = s2 > 0.f ? 1.f / s2 : 0.f;
      }
      named_bar(1, 128);   // red is rewritten below
      // round to nearest through the float adder (0 <= x < 2^22)
      auto to_int = [](float xx) { return __float_as_int(xx + 12582912.f) - 0x4B400000; };
      float lsum[kG] = {0.f, 0.f, 0.f, 0.f};
      int W1[kG] = {0, 0, 0, 0}, W2[kG] = {0, 0, 0, 0};
      for (int t = 0; t < x.nk; ++t, ++wit) {
        const int wb = wit % kWS;
        bool ok = !*abort_flag;
        if (ok && wit >= kWS && !wait_bar(bar(kBWE + wb), ((wit / kWS) - 1) & 1)) { fail(); ok = false; }
        bad = !__all_sync(0xffffffffu, ok);
        if (bad) break;
        const int tok = t * kT + r;
        uint32_t by[16];
#pragma unroll
        for (int n = 0; n < 16; ++n) by[n] = 0u;
        if (tok < x.ntok) {
          const float2 nv = __half22float2(vnr[tok]);
#pragma unroll
          for (int h = 0; h < kG; ++h) {
            const float p = amma::exp2_approx(logit[h * kMaxChunk + tok] - M[h]);
            lsum[h] += p;
            const int w1 = min(to_int(p * nv.x * inv1[h]), 65535), w2 = min(to_int(p * nv.y * inv2[h]), 65535);
            W1[h] += w1;
            W2[h] += w2;
            by[2 * h] = (uint32_t)(w1 >> 8);
            by[2 * h + 1] = (uint32_t)(w1 & 255);
            by[8 + 2 * h] = (uint32_t)(w2 >> 8);
            by[9 + 2 * h] = (uint32_t)(w2 & 255);
          }
        }
        const uint32_t wt = base + kOffW + (uint32_t)wb * kWStage;
#pragma unroll
        for (int n = 0; n < 16; ++n) sts8(wt + swz(n, r), by[n]);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(bar(kBWF + wb));
      }
#pragma unroll
      for (int h = 0; h < kG; ++h)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
          W1[h] += __shfl_xor_sync(0xffffffffu, W1[h], o);
          W2[h] += __shfl_xor_sync(0xffffffffu, W2[h], o);
        }
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < kG; ++h) red[16 * q4 + h] = lsum[h], ired[8 * q4 + h] = W1[h], ired[8 * q4 + 4 + h] = W2[h];

      // ---- value sums of the item -> shared (the logits are dead: every weight tile is written)
      {
        bool ok = !*abort_flag;
        if (ok && !bad && !wait_bar(bar(kBVAF), ai & 1)) { fail(); ok = false; }
        if (bar_red_or(1, 128, !ok || bad)) break;   // (also publishes red / ired)
      }
      tc_fence_after();
      uint32_t va0[16], va1[16], va2[16];
      tmem_ld16(lane_base + kColV, va0);
      tmem_ld16(lane_base + kColV + 16u, va1);
      tmem_ld16(lane_base + kColV + 32u, va2);
      tmem_wait_ld();
      tmem_wait_ld_regs(va0);
      tmem_wait_ld_regs(va1);
      tmem_wait_ld_regs(va2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(bar(kBVAE));
      // row r of region g is operand byte 128 g + r: word u = 32 g + r / 4, byte r % 4
      float* S = logit;   // [head][384]: bit 0 of coordinate c, bit 1 of c, projection p
      {
        const int w = r >> 2, bb = r & 3;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t* vg = g ? va1 : va0;
          const int s_pl = 4 * g + (w >> 3), cbyte = 4 * (w & 7) + bb;
          const int c = 4 * cbyte + (s_pl >> 1), beta = s_pl & 1;
#pragma unroll
          for (int h = 0; h < kG; ++h)
            S[h * 384 + beta * 128 + c] = (float)(256 * (int)vg[2 * h] + (int)vg[2 * h + 1]);
        }
        const int s_pl = w >> 2, sb = 4 * (w & 3) + bb, p = 8 * sb + s_pl;
#pragma unroll
        for (int h = 0; h < kG; ++h) S[h * 384 + 256 + p] = (float)(256 * (int)va2[8 + 2 * h] + (int)va2[9 + 2 * h]);
      }
      named_bar(1, 128);
      // ---- partial results: rotated-domain value sum, QJL sum, max (natural-log units), sum of p
      {
        float Wf1[kG], Wf2[kG], L[kG];
#pragma unroll
        for (int h = 0; h < kG; ++h) {
          int i1 = 0, i2 = 0;
          float l = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) i1 += ired[8 * w + h], i2 += ired[8 * w + 4 + h], l += red[16 * w + h];
          Wf1[h] = (float)i1;
          Wf2[h] = (float)i2;
          L[h] = l;
        }
        for (int o = r; o < kG * (kD + kM); o += 128) {
          const int h = o / (kD + kM), j = o - h * (kD + kM);
          float v;
          if (j < kD) v = st1[h] * (a.vc0 * Wf1[h] + a.vb0 * S[h * 384 + j] + a.vb1 * S[h * 384 + 128 + j]);
          else v = st2[h] * (2.f * S[h * 384 + 256 + (j - kD)] - Wf2[h]);
          a.part[((hq0 + h) * a.nsplit + x.split) * stride + j] = v;
        }
#pragma unroll
        for (int h = 0; h < kG; ++h)
          if (r == h) {
            float* o = a.part + ((hq0 + h) * a.nsplit + x.split) * stride;
            o[kD + kM] = M[h] * 0.6931471805599453f;
            o[kD + kM + 1] = L[h];
          }
      }
      named_bar(1, 128);   // shared scratch is reused by the next item
      ++ai;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace atc
}  // namespace tqk
