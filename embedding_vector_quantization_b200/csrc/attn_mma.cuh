// Decode attention over 3-bit prod caches (2-bit Lloyd-Max codes + 1-bit QJL
// signs, m = 128) at d = 128 with 4 query heads per KV head, on int8 tensor-core
// MMAs (mma.sync m16n8k32) fed by TMA bulk copies.
//
// What is computed is exactly tq_attn_decode's definition ("TurboQuant / PolarQuant
// / QJL technical deep dive" (gemilab.net), "Scaled dot-product attention";
// "Google TurboQuant: 6x KV-cache compression" (ebisuda.net), "Stage 1" and
// "Stage 2"); only the arithmetic is rearranged so that the packed bits feed the
// tensor cores directly:
//
//  * A symmetric 2-bit codebook is affine in the two index bits:
//    c[idx] = c0 + (c1 - c0) b0 + (c2 - c0) b1  (the b0*b1 coefficient
//    c3 - c2 - c1 + c0 vanishes by symmetry). So <q', c[idx]> is c0*sum(q') plus
//    two 0/1 dot products, and sum_i w_i c[idx_ij] is c0*sum(w) plus two 0/1
//    weighted sums. Sign bits give <qs, 2 sigma - 1> = 2 <qs, sigma> - sum(qs).
//  * 0/1 bit planes become int8 MMA operands with one AND per 4 elements:
//    (word >> s) & 0x01010101 (value 1) or (word >> s) & 0x10101010 (value 16);
//    every MMA uses one of the two mask families, so its accumulator is exact
//    after a final division by 16 (kept in separate accumulators for keys).
//  * Query side (keys as the MMA rows): queries are rotated once, scaled by the
//    codebook slopes, rounded to 22-bit integers and split into three int8 pieces
//    (hi * 2^14 + mid * 2^7 + lo): one n8 tile holds the hi and mid pieces of the
//    4 heads, a second n8 tile the lo pieces (columns 2h; the odd columns are 0).
//    The QJL projections S q (weighed by the small residual norms) are rounded to
//    15-bit integers, two pieces hi * 2^7 + lo in the first tile only.
//  * Value side (bit rows of the value codes as the MMA rows, tokens as the
//    reduction): softmax weights p * ||v|| (and p * rnorm for the QJL part) are
//    rounded to 16-bit integers against the chunk maximum and split into two
//    unsigned 8-bit pieces (hi * 256 + lo; u8 x u8 MMAs, since bits and weights
//    are non-negative); ldmatrix .trans.b8 gathers "byte j of 4 consecutive
//    tokens" into one register.
//  * Precision: a query piece is off by at most half a step of max|q| / 2^21, a
//    weight by half a step of max ||v|| / 65535; on keys and values with 10x
//    outlier channels this keeps the attention output within a few 1e-4 of the
//    exact result (the 15-bit queries and 14-bit weights used before reached 1.3e-3).
//  * Two passes per context chunk: all key scores first (kept in shared memory,
//    giving the exact chunk maximum), then all values with one fixed weight
//    scale, so the value sums accumulate in int32 across the whole chunk.
//  * The whole chunk (at most 896 tokens: 93 KB of keys and values) is staged in
//    shared memory: every TMA copy of the chunk is issued at launch, one mbarrier
//    per 256-token block of keys and of values, so the cold read of the cache has
//    all of its bytes requested at once and the key pass starts on the first block
//    while the rest arrive.
//
// Partial results use the layout of the split kernel in score_attn_simt.cuh
// ([B*Hq][nsplit][d + m + 2]: rotated-domain value sum, QJL sum, max, sum of
// weights) and are merged by the combine kernel.
#pragma once

#include "common.cuh"
#include "small_kernels.cuh"

namespace tqk {
namespace amma {

constexpr int kD = 128;
constexpr int kM = 128;
constexpr int kG = 4;
constexpr int kBlk = 256;                     // tokens per block (one mbarrier each)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCodesB = 32, kSignsB = 16;
constexpr int kStageCodes = kBlk * kCodesB;   // 8192
constexpr int kStageSigns = kBlk * kSignsB;   // 4096
constexpr int kMaxChunk = 896;                // the chunk's keys and values fit shared memory twice per SM
constexpr int kMaxBlk = (kMaxChunk + kBlk - 1) / kBlk;   // 4
// padded row strides against shared-memory bank conflicts: the 4 heads' logit rows start 8 banks
// apart, and the rows of a weight block 4 banks apart
constexpr int kLogitStride = kMaxChunk + 8;
constexpr int kPwRow = kBlk + 16;

struct Args {
  const float* qr;  // [B*Hq][128] Pi_K q
  const float* qs;  // [B*Hq][128] S_K q
  int B, Hq, Hkv;
  const uint8_t* kcodes;
  const uint8_t* ksigns;
  const __half* knorm;
  const __half* krn;
  const uint8_t* vcodes;
  const uint8_t* vsigns;
  const __half* vnorm;
  const __half* vrn;
  int64_t L_cap, chunk;
  int nsplit;
  const int32_t* len;
  int len_extra;        // 1 inside a decode step: the token appended at slot len[b] counts
  float kc0, kb0, kb1;  // K codebook: c[idx] = kc0 + kb0*b0 + kb1*b1
  float vc0, vb0, vb1;  // V codebook
  float scale;          // softmax scale
  float* part;          // [B*Hq][nsplit][d + m + 2]
  int* err;
};

// Key-pass data of the chunk; after the key pass its codes and signs are dead and hold the
// value pass's integer weights and sums instead.
struct __align__(16) KeyArea {
  union {
    unsigned char codes[kMaxChunk * kCodesB];
    uint8_t pw[kMaxBlk][2][8][kPwRow];  // integer softmax weights of the chunk's value blocks:
                                        // [block][0: value weights, 1: QJL weights][col = head*2+piece][token]
  };
  union {
    unsigned char signs[kMaxChunk * kSignsB];
    float vacc[3][kG][128];     // value-side sums of the two token halves (rows of each byte group)
  };
  __half kn[kMaxChunk];         // key norms, residual norms, and the value norms and residual norms
  __half krn[kMaxChunk];        // (these arrive with the keys: the weight steps need them)
  __half vn[kMaxChunk];
  __half vrn[kMaxChunk];
};

struct __align__(16) Smem {
  KeyArea k;
  unsigned char vcodes[kMaxChunk * kCodesB];
  unsigned char vsigns[kMaxChunk * kSignsB];
  float logits[kG][kLogitStride];  // key pass output: scaled logits in log2 units [head][token]
  uint32_t qfrag[2][12][2][4][8];  // key-side B fragments: [n tile][k-step][register][quad index t][column g]
  float qconst[kG][4];        // c0*sum(q'), delta_mse, delta_qjl, sum(qs)
  float red_f[kWarps][kG];
  float hmax[kG];
  float dv[2][kG];            // weight steps per head: max_t p_t ||v_t|| / 65535 (0: values, 1: QJL)
  float inv[2][kG];
  float red_w[kWarps][2][kG]; // per warp and head: the largest p ||v|| and p rnorm
  int red_i[kWarps][2 * kG];
  uint64_t kfull[kMaxBlk];    // key block j has arrived
  uint64_t vfull[kMaxBlk];    // value block j has arrived
  int W[2][kG];               // chunk sums of the integer value / QJL weights per head
  int abort_flag;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) { return bar_wait(bar, parity); }

__device__ __forceinline__ void tma_bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};\n"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Unsigned variant (0/1 bit planes times non-negative weight pieces).
__device__ __forceinline__ void mma_u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};\n"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}

__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}

// Two 16x16 byte tiles, transposed: r[0], r[1] = tile 0 columns g, g+8 of rows
// 4t..4t+3; r[2], r[3] = the same for tile 1 (g = lane/4, t = lane%4).
__device__ __forceinline__ void ldsm_t8_x2(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}

// 2^x by the hardware's approximate base-2 exponential (flushes subnormal results to 0);
// the weights it feeds are rounded to 14 bits right after.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack4(int8_t a, int8_t b, int8_t c, int8_t d) {
  return (uint32_t)(uint8_t)a | ((uint32_t)(uint8_t)b << 8) | ((uint32_t)(uint8_t)c << 16) |
         ((uint32_t)(uint8_t)d << 24);
}

// Where a query-side element sits in the key-side B fragments (inverse of the
// A-operand construction in the key pass): returns the byte offset within
// qfrag for column g = 0. Code plane p of code c: k-step 2(c%4)+p, register
// c/64, quad index (c/16)%4, byte (c%16)/4. Sign bit i: word t = i/32, byte
// e = (i%32)/8, bit u = i%8 -> k-step 8+u (u<2), 8+u-2 (u=2,3), 10+u-4
// (u=4,5), 10+u-6 (u=6,7); register 0 for u in {0,1,4,5}, 1 otherwise.
__device__ __forceinline__ int qfrag_code_offset(int plane, int c) {
  const int kk = 2 * (c & 3) + plane, slot = c >> 6, t = (c >> 4) & 3, e = (c & 15) >> 2;
  return (((kk * 2 + slot) * 4 + t) * 8) * 4 + e;
}
__device__ __forceinline__ int qfrag_sign_offset(int i) {
  const int t = i >> 5, e = (i & 31) >> 3, u = i & 7;
  const int grp = (u < 4) ? 8 : 10, w = u & 3, slot = w >> 1, s = w & 1;
  const int kk = grp + s;
  return (((kk * 2 + slot) * 4 + t) * 8) * 4 + e;
}

// Query side of the key MMAs for the kG heads h0 .. h0 + 3 of sequence b (one warp per
// head, warps 0..3): rotated queries scaled by the codebook slopes, rounded to 22-bit
// integers against their maximum and split into int8 pieces hi * 2^14 + mid * 2^7 + lo in
// B-fragment order (n tile 0: column 2h = hi, 2h + 1 = mid; n tile 1: column 2h = lo); S q
// rounded to 15-bit integers, hi * 2^7 + lo in n tile 0 (columns 2h, 2h + 1).
// qconst[h] = {c0 sum(q'), step of the code pieces, step of the sign pieces, sum(S q)}.
constexpr float kQMax = 2080768.f;   // 127 * 2^14: the largest |integer| a query value maps to
constexpr float kSMax = 16256.f;     // 127 * 2^7: the same for the QJL projections
__device__ __forceinline__ void prepare_query(const float* qr_rows, const float* qs_rows, float kb0, float kb1,
                                              float kc0, uint32_t (&qfrag)[2][12][2][4][8],
                                              float (&qconst)[kG][4]) {
  const int lane = threadIdx.x & 31, h = threadIdx.x >> 5;
  if (h >= kG) return;
  const float* qr = qr_rows + (size_t)h * kD;
  const float* qsv = qs_rows + (size_t)h * kM;
  float x0[4], x1[4], xs[4], sq = 0.f, ss = 0.f, mx = 0.f, ms = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float q = qr[lane + 32 * i];
    const float s = qsv[lane + 32 * i];
    x0[i] = kb0 * q;
    x1[i] = kb1 * q;
    xs[i] = s;
    sq += q;
    ss += s;
    mx = fmaxf(mx, fmaxf(fabsf(x0[i]), fabsf(x1[i])));
    ms = fmaxf(ms, fabsf(s));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
  }
  const float dm = mx > 0.f ? mx / kQMax : 1.f;
  const float ds = ms > 0.f ? ms / kSMax : 1.f;
  int8_t* qf0 = reinterpret_cast<int8_t*>(&qfrag[0][0][0][0][0]);
  int8_t* qf1 = reinterpret_cast<int8_t*>(&qfrag[1][0][0][0][0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = lane + 32 * i;
    const float v[3] = {x0[i] / dm, x1[i] / dm, xs[i] / ds};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int xi = __float2int_rn(v[c]);                                   // |xi| <= 127 * 2^14
      const int hi = (xi >= 0) ? (xi + 8192) >> 14 : -((-xi + 8192) >> 14);  // |hi| <= 127
      const int r = xi - hi * 16384;                                         // |r| <= 2^13
      const int mid = (r >= 0) ? (r + 64) >> 7 : -((-r + 64) >> 7);         // |mid| <= 64
      const int off = qfrag_code_offset(c, j);
      qf0[off + (2 * h) * 4] = (int8_t)hi;
      qf0[off + (2 * h + 1) * 4] = (int8_t)mid;
      qf1[off + (2 * h) * 4] = (int8_t)(r - mid * 128);                      // |lo| <= 64
      qf1[off + (2 * h + 1) * 4] = 0;
    }
    {
      const int xi = __float2int_rn(v[2]);                                   // |xi| <= 127 * 2^7
      const int hi = (xi >= 0) ? (xi + 64) >> 7 : -((-xi + 64) >> 7);        // |hi| <= 127
      const int off = qfrag_sign_offset(j);
      qf0[off + (2 * h) * 4] = (int8_t)hi;
      qf0[off + (2 * h + 1) * 4] = (int8_t)(xi - 128 * hi);                  // |lo| <= 64
    }
  }
  if (lane == 0) {
    qconst[h][0] = kc0 * sq;
    qconst[h][1] = dm;
    qconst[h][2] = ds;
    qconst[h][3] = ss;
  }
}

// Raw scores (tq_score's formula) of keys kbase[i] + g and kbase[i] + g + 8 of a staged key
// block (NT m-tiles of 16 keys, their MMAs interleaved for independent accumulator chains) for
// query head t = lane % 4: the code bit planes against the query pieces of n tile 0 (hi and mid,
// fragments qb held in registers) and n tile 1 (lo: lo(k-step, register) returns this thread's
// fragment word, from registers or shared memory), the sign bit planes against the two pieces of
// S q in n tile 0.
// LO: the code side uses all three query pieces (22-bit queries, what the attention needs so that
// softmax does not amplify the rounding); without it the lo piece is skipped and the code-side
// query is the 15-bit hi/mid value, which raw scores are accurate enough with (about 3e-5 relative).
template <int NT, bool LO, typename LoFn>
__device__ __forceinline__ void mtile_scores(const unsigned char* codes, const unsigned char* signs, const __half* nrm,
                                             const __half* rnm, const int (&kbase)[NT], const uint32_t (&qb)[12][2],
                                             LoFn lo, float c0h, float dmh, float dsh, float ssh, float (&sc)[NT][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2;
  uint32_t cw[NT][4], sw[NT][2];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const int mat = lane >> 3, r = lane & 7;
    const int key = kbase[i] + r + 8 * (mat >> 1);
    ldsm_x4(cw[i], codes + key * kCodesB + 16 * (mat & 1));
    const int skey = kbase[i] + r + 8 * (mat & 1);
    ldsm_x2(sw[i], signs + skey * kSignsB);
  }
  // per m-tile: codes (x1 and x16 families, n tiles 0 and 1) and signs (n tile 0)
  int dm1[NT][4] = {}, dm16[NT][4] = {}, lm1[NT][4] = {}, lm16[NT][4] = {}, ds1[NT][4] = {}, ds16[NT][4] = {};
  // code words: cw[0] = key g word t, cw[1] = key g word 4+t, cw[2] = key g+8 word t, cw[3] = key g+8 word 4+t
#pragma unroll
  for (int s = 0; s < 4; ++s) {
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint32_t x0 = cw[i][0] >> s, x1 = cw[i][1] >> s, x2 = cw[i][2] >> s, x3 = cw[i][3] >> s;
      const uint32_t a0 = x0 & 0x01010101u, a1 = x2 & 0x01010101u, a2 = x1 & 0x01010101u, a3 = x3 & 0x01010101u;
      const uint32_t b0 = x0 & 0x10101010u, b1 = x2 & 0x10101010u, b2 = x1 & 0x10101010u, b3 = x3 & 0x10101010u;
      mma_s8(dm1[i], a0, a1, a2, a3, qb[s][0], qb[s][1]);
      mma_s8(dm16[i], b0, b1, b2, b3, qb[4 + s][0], qb[4 + s][1]);
      if (LO) {
        mma_s8(lm1[i], a0, a1, a2, a3, lo(s, 0), lo(s, 1));
        mma_s8(lm16[i], b0, b1, b2, b3, lo(4 + s, 0), lo(4 + s, 1));
      }
    }
  }
  // sign words: sw[0] = key g word t, sw[1] = key g+8 word t
#pragma unroll
  for (int s = 0; s < 2; ++s) {
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint32_t y0 = sw[i][0] >> s, y1 = sw[i][1] >> s, z0 = sw[i][0] >> (s + 2), z1 = sw[i][1] >> (s + 2);
      const uint32_t a0 = y0 & 0x01010101u, a1 = y1 & 0x01010101u, a2 = z0 & 0x01010101u, a3 = z1 & 0x01010101u;
      const uint32_t b0 = y0 & 0x10101010u, b1 = y1 & 0x10101010u, b2 = z0 & 0x10101010u, b3 = z1 & 0x10101010u;
      mma_s8(ds1[i], a0, a1, a2, a3, qb[8 + s][0], qb[8 + s][1]);
      mma_s8(ds16[i], b0, b1, b2, b3, qb[10 + s][0], qb[10 + s][1]);
    }
  }
  const float kqjl = kQjlScale / (float)kM;
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int r = 0; r < 2; ++r) {  // r = 0: key g, r = 1: key g + 8
      const int key = kbase[i] + g + 8 * r;
      const int hi = 2 * r, md = 2 * r + 1;   // tile 0: columns 2t (hi) and 2t + 1 (mid); tile 1: column 2t (lo)
      // exact in int32: at most 256 code positions of |piece| <= 127 each, times 2^14
      const int mse = (dm1[i][hi] + (dm16[i][hi] >> 4)) * 16384 + (dm1[i][md] + (dm16[i][md] >> 4)) * 128 +
                      (LO ? lm1[i][hi] + (lm16[i][hi] >> 4) : 0);
      // column 2t + 1 holds the lo piece of S q here
      const int qjl = (ds1[i][hi] + (ds16[i][hi] >> 4)) * 128 + ds1[i][md] + (ds16[i][md] >> 4);
      const float n = __half2float(nrm[key]), rn = __half2float(rnm[key]);
      sc[i][r] = n * (c0h + dmh * (float)mse) + rn * kqjl * (2.f * dsh * (float)qjl - ssh);
    }
}

__global__ void __launch_bounds__(kThreads, 2) attn_prod2_kernel(Args a) {
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
  const int nblk = (ntok + kBlk - 1) / kBlk;           // <= kMaxBlk (chunk <= kMaxChunk)
  const int64_t row0 = (int64_t)bh * a.L_cap + start;  // cache row of the chunk's first token

  // ---------------- setup: barriers
  if (tid == 0) {
    for (int j = 0; j < kMaxBlk; ++j) {
      mbar_init(&sm.kfull[j], 1);
      mbar_init(&sm.vfull[j], 1);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid < 2 * kG) (&sm.dv[0][0])[tid] = 1.f;   // an empty chunk keeps unit steps (its sums are 0)
  __syncthreads();

  // Every copy of the chunk, issued at once by warp 0: key blocks first (codes, signs, the key
  // norms and residual norms and the value norms and residual norms), then value blocks
  // (codes, signs). Rows up to L_cap are copied (whole 8-token groups, L_cap % 8 == 0), at
  // most the chunk's kMaxChunk slots.
  auto issue_all = [&]() {
    if (warp != 0) return;
    auto ncopy_of = [&](int j) {
      return (int)min(min((int64_t)kBlk, a.L_cap - (start + (int64_t)j * kBlk)), (int64_t)(kMaxChunk - j * kBlk));
    };
    if (lane < nblk) {
      const uint32_t nc = (uint32_t)ncopy_of(lane);
      mbar_expect_tx(&sm.kfull[lane], nc * (kCodesB + kSignsB + 8));
      mbar_expect_tx(&sm.vfull[lane], nc * (kCodesB + kSignsB));
    }
    __syncwarp();
    // copy c of block j: lane c handles copy c of every block (8 copies per block pair)
    if (lane < 8) {
      for (int j = 0; j < nblk; ++j) {
        const int nc = ncopy_of(j);
        const int64_t r = row0 + (int64_t)j * kBlk;
        const int tk = j * kBlk;
        switch (lane) {
          case 0: tma_bulk_g2s(sm.k.codes + tk * kCodesB, a.kcodes + r * kCodesB, nc * kCodesB, &sm.kfull[j]); break;
          case 1: tma_bulk_g2s(sm.k.signs + tk * kSignsB, a.ksigns + r * kSignsB, nc * kSignsB, &sm.kfull[j]); break;
          case 2: tma_bulk_g2s(sm.k.kn + tk, a.knorm + r, nc * 2, &sm.kfull[j]); break;
          case 3: tma_bulk_g2s(sm.k.krn + tk, a.krn + r, nc * 2, &sm.kfull[j]); break;
          case 4: tma_bulk_g2s(sm.k.vn + tk, a.vnorm + r, nc * 2, &sm.kfull[j]); break;
          case 5: tma_bulk_g2s(sm.k.vrn + tk, a.vrn + r, nc * 2, &sm.kfull[j]); break;
          default: break;
        }
      }
      for (int j = 0; j < nblk; ++j) {
        const int nc = ncopy_of(j);
        const int64_t r = row0 + (int64_t)j * kBlk;
        const int tk = j * kBlk;
        if (lane == 6) tma_bulk_g2s(sm.vcodes + tk * kCodesB, a.vcodes + r * kCodesB, nc * kCodesB, &sm.vfull[j]);
        if (lane == 7) tma_bulk_g2s(sm.vsigns + tk * kSignsB, a.vsigns + r * kSignsB, nc * kSignsB, &sm.vfull[j]);
      }
    }
  };
  grid_dep_launch();
  // The kernel before this one in a decode step (append + query rotation) writes only the
  // slot len[b] and the rotated queries, so every CTA streams its chunk before waiting for it;
  // the one chunk per sequence that holds the slot copies that token's rows again after the
  // wait (patch_slot), once the block that holds it has arrived.
  const int64_t slot = (int64_t)max(a.len[b], 0);
  const bool holds_new = a.len_extra && slot >= start && slot < end;
  const int s_loc = holds_new ? (int)(slot - start) : -1, s_blk = holds_new ? s_loc / kBlk : -1;
  issue_all();
  grid_dep_wait();
  // this token's rows as the previous kernel wrote them (key side: codes, signs, the four norms;
  // value side: codes, signs); called with the block's data resident, followed by a CTA barrier
  auto patch_slot = [&](bool key_side) {
    const int64_t r = row0 + s_loc;
    if (key_side) {
      if (tid < 8) reinterpret_cast<uint32_t*>(sm.k.codes + s_loc * kCodesB)[tid] =
          reinterpret_cast<const uint32_t*>(a.kcodes + r * kCodesB)[tid];
      else if (tid < 12) reinterpret_cast<uint32_t*>(sm.k.signs + s_loc * kSignsB)[tid - 8] =
          reinterpret_cast<const uint32_t*>(a.ksigns + r * kSignsB)[tid - 8];
      else if (tid == 12) sm.k.kn[s_loc] = a.knorm[r];
      else if (tid == 13) sm.k.krn[s_loc] = a.krn[r];
      else if (tid == 14) sm.k.vn[s_loc] = a.vnorm[r];
      else if (tid == 15) sm.k.vrn[s_loc] = a.vrn[r];
    } else {
      if (tid < 8) reinterpret_cast<uint32_t*>(sm.vcodes + s_loc * kCodesB)[tid] =
          reinterpret_cast<const uint32_t*>(a.vcodes + r * kCodesB)[tid];
      else if (tid < 12) reinterpret_cast<uint32_t*>(sm.vsigns + s_loc * kSignsB)[tid - 8] =
          reinterpret_cast<const uint32_t*>(a.vsigns + r * kSignsB)[tid - 8];
    }
  };

  // query constants and int8 pieces (one warp per head)
  prepare_query(a.qr + ((size_t)b * a.Hq + h0) * kD, a.qs + ((size_t)b * a.Hq + h0) * kM, a.kb0, a.kb1, a.kc0,
                sm.qfrag, sm.qconst);
  __syncthreads();

  // B fragments of the key-side MMAs, n tile 0 (constant for the CTA): 12 k-steps x 2 registers
  uint32_t qb[12][2], ql[8][2];   // n tile 0 (all k-steps) and n tile 1 (lo pieces: the code k-steps)
#pragma unroll
  for (int kk = 0; kk < 12; ++kk)
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      qb[kk][sl] = sm.qfrag[0][kk][sl][t][g];
      if (kk < 8) ql[kk][sl] = sm.qfrag[1][kk][sl][t][g];
    }
  auto lo_reg = [&](int kk, int sl) { return ql[kk][sl]; };

  const float scale2 = a.scale * 1.4426950408889634f;
  const float c0h = sm.qconst[t][0], dmh = sm.qconst[t][1], dsh = sm.qconst[t][2], ssh = sm.qconst[t][3];
  float run_max = -INFINITY;   // this thread's max logit of head t

  // No warp ever leaves early: a wait that runs out sets abort_flag, after which no further
  // waits happen, so every warp still meets the same CTA barriers; the results are discarded.
  auto wait_full = [&](uint64_t* bar) {
    if (*(volatile int*)&sm.abort_flag) return;
    if (!mbar_wait(bar, 0)) sm.abort_flag = 1;
  };

  // ---------------- key pass: warp w scores keys 16w .. 16w+15 and 128+16w .. of every block
  for (int j = 0; j < nblk; ++j) {
    wait_full(&sm.kfull[j]);
    if (j == s_blk) {   // uniform in the CTA
      patch_slot(true);
      __syncthreads();
    }
    const int tok_base = j * kBlk;
    const int nvalid = min(kBlk, ntok - tok_base);
    const unsigned char* kc = sm.k.codes + tok_base * kCodesB;
    const unsigned char* ks = sm.k.signs + tok_base * kSignsB;
    const __half* nrm = sm.k.kn + tok_base;
    const __half* rnm = sm.k.krn + tok_base;
    // warp w: keys 16w .. 16w+15 and 128+16w .. 128+16w+15 (both m-tiles at once, or the first
    // alone when the block's valid keys end before the second; warp-uniform)
    float sc[2][2];
    if (16 * warp + 128 < nvalid) {
      const int kb2[2] = {16 * warp, 128 + 16 * warp};
      mtile_scores<2, true>(kc, ks, nrm, rnm, kb2, qb, lo_reg, c0h, dmh, dsh, ssh, sc);
    } else if (16 * warp < nvalid) {
      const int kb1[1] = {16 * warp};
      float sc1[1][2];
      mtile_scores<1, true>(kc, ks, nrm, rnm, kb1, qb, lo_reg, c0h, dmh, dsh, ssh, sc1);
      sc[0][0] = sc1[0][0], sc[0][1] = sc1[0][1], sc[1][0] = sc[1][1] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int kbase = 128 * mt + 16 * warp;
#pragma unroll
      for (int r = 0; r < 2; ++r) {  // r = 0: key g, r = 1: key g + 8
        const int key = kbase + g + 8 * r;
        // softmax scale * log2(e): the weights are exp2(logit - max)
        // (the last block of a chunk may be partial: nothing past its valid keys is stored, the
        // logits rows hold kMaxChunk tokens)
        if (key < nvalid) {
          const float v = sc[mt][r] * scale2;
          sm.logits[t][tok_base + key] = v;
          run_max = fmaxf(run_max, v);
        }
      }
    }
  }

  // Integer softmax weights of the chunk, all value blocks at once (all threads): thread ->
  // (head h = tid & 3, 4 consecutive tokens q4 .. q4 + 3 of every block). With
  // p = exp2(logit - max): w1 = round(p ||v|| / dv[0][h]), w2 = round(p rnorm / dv[1][h]), the
  // steps being each head's largest p ||v|| and p rnorm of the chunk over 65535 (16-bit
  // weights), split into 8-bit pieces (hi * 256 + lo). Also the sums of p and of the weights.
  float lsum = 0.f;
  int wsum[2] = {0, 0};
  if (nblk > 0) {
    __syncthreads();   // the key area's codes and signs are dead from here on
    if (lane == 0) {
      for (int h = 0; h < kG; ++h) sm.red_f[warp][h] = -INFINITY;
    }
    __syncwarp();
    float m = run_max;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (g == 0) sm.red_f[warp][t] = m;
    __syncthreads();
    if (tid < kG) {
      float mm = -INFINITY;
      for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, sm.red_f[w][tid]);
      sm.hmax[tid] = mm;
    }
    __syncthreads();
    const int h = tid & 3, q4 = (tid >> 2) * 4;
    const float hm = sm.hmax[h];
    float pv[kMaxBlk][4], pr[kMaxBlk][4];   // p ||v|| and p rnorm of this thread's tokens
    float mv = 0.f, mr = 0.f;
#pragma unroll
    for (int jj = 0; jj < kMaxBlk; ++jj) {
      const int tb = jj * kBlk, nval = min(kBlk, ntok - tb);
      const float4 l4 = (q4 < nval) ? *reinterpret_cast<const float4*>(&sm.logits[h][tb + q4])
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
      const __half2 n01 = *reinterpret_cast<const __half2*>(&sm.k.vn[tb + q4]);
      const __half2 n23 = *reinterpret_cast<const __half2*>(&sm.k.vn[tb + q4 + 2]);
      const __half2 r01 = *reinterpret_cast<const __half2*>(&sm.k.vrn[tb + q4]);
      const __half2 r23 = *reinterpret_cast<const __half2*>(&sm.k.vrn[tb + q4 + 2]);
      const float2 fn01 = __half22float2(n01), fn23 = __half22float2(n23);
      const float2 fr01 = __half22float2(r01), fr23 = __half22float2(r23);
      const float vn[4] = {fn01.x, fn01.y, fn23.x, fn23.y}, vr[4] = {fr01.x, fr01.y, fr23.x, fr23.y};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool ok = q4 + q < nval;   // tokens past the chunk's end get zero weight
        const float pp = ok ? exp2_approx(lv[q] - hm) : 0.f;
        lsum += pp;
        pv[jj][q] = ok ? pp * vn[q] : 0.f;   // (norm slots past the copied rows hold stale data)
        pr[jj][q] = ok ? pp * vr[q] : 0.f;
        mv = fmaxf(mv, pv[jj][q]);
        mr = fmaxf(mr, pr[jj][q]);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
      mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
    }
    if (g == 0) sm.red_w[warp][0][t] = mv, sm.red_w[warp][1][t] = mr;
    __syncthreads();
    if (tid < 2 * kG) {
      float mx = 0.f;
      for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, sm.red_w[w][tid / kG][tid % kG]);
      const float st = mx / 65535.f;
      sm.dv[tid / kG][tid % kG] = st > 0.f ? st : 1.f;
      sm.inv[tid / kG][tid % kG] = st > 0.f ? 1.f / st : 0.f;
    }
    __syncthreads();
    const float inv1 = sm.inv[0][h], inv2 = sm.inv[1][h];
    // round to nearest (even) through the float adder: x + 1.5 * 2^23 leaves the integer in the low
    // mantissa bits for 0 <= x < 2^22 (here x <= 65535 * (1 + 2^-23))
    auto to_int = [](float x) { return __float_as_int(x + 12582912.f) - 0x4B400000; };
#pragma unroll
    for (int jj = 0; jj < kMaxBlk; ++jj) {
      if (jj >= nblk) break;
      uint32_t w1h = 0, w1l = 0, w2h = 0, w2l = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int w1 = min(to_int(pv[jj][q] * inv1), 65535), w2 = min(to_int(pr[jj][q] * inv2), 65535);
        w1h |= (uint32_t)(w1 >> 8) << (8 * q);
        w1l |= (uint32_t)(w1 & 255) << (8 * q);
        w2h |= (uint32_t)(w2 >> 8) << (8 * q);
        w2l |= (uint32_t)(w2 & 255) << (8 * q);
        wsum[0] += w1;
        wsum[1] += w2;
      }
      uint8_t* blk = &sm.k.pw[jj][0][0][0];
      *reinterpret_cast<uint32_t*>(blk + (2 * h) * kPwRow + q4) = w1h;
      *reinterpret_cast<uint32_t*>(blk + (2 * h + 1) * kPwRow + q4) = w1l;
      *reinterpret_cast<uint32_t*>(blk + (8 + 2 * h) * kPwRow + q4) = w2h;
      *reinterpret_cast<uint32_t*>(blk + (8 + 2 * h + 1) * kPwRow + q4) = w2l;
    }
    __syncthreads();
  }

  // ---------------- value pass (warps 0..5: byte group bg, token half)
  // value-side accumulators: 8 m-tiles (bit rows 0..7 of bytes g, g+8 of this warp's byte group)
  int vacc[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u) vacc[u][0] = vacc[u][1] = vacc[u][2] = vacc[u][3] = 0;
  const int bg = warp % 3, half = warp / 3;
  for (int jj = 0; jj < nblk; ++jj) {
    wait_full(&sm.vfull[jj]);
    if (jj == s_blk) {   // uniform in the CTA
      patch_slot(false);
      __syncthreads();
    }
    if (warp < 6) {
      const uint8_t* pw = &sm.k.pw[jj][bg == 2 ? 1 : 0][0][0];
      const unsigned char* vc = sm.vcodes + jj * kStageCodes;
      const unsigned char* vs = sm.vsigns + jj * kStageSigns;
      const int nvalv = min(kBlk, ntok - jj * kBlk);
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const int tk = 128 * half + 32 * kq;  // first token of this 32-token k-step
        if (tk >= nvalv) break;               // past the chunk's end (weights 0; warp-uniform)
        uint32_t r[4];
        const int tok = tk + (lane & 15) + 16 * (lane >> 4);
        const unsigned char* rowp = (bg < 2) ? vc + tok * kCodesB + 16 * bg : vs + tok * kSignsB;
        ldsm_t8_x2(r, rowp);
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(pw + g * kPwRow + tk + 4 * t);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(pw + g * kPwRow + tk + 16 + 4 * t);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t x0 = r[0] >> s, x1 = r[1] >> s, x2 = r[2] >> s, x3 = r[3] >> s;
          mma_u8(vacc[s], x0 & 0x01010101u, x1 & 0x01010101u, x2 & 0x01010101u, x3 & 0x01010101u, b0, b1);
          mma_u8(vacc[4 + s], x0 & 0x10101010u, x1 & 0x10101010u, x2 & 0x10101010u, x3 & 0x10101010u, b0, b1);
        }
      }
    }
  }

  __syncthreads();
  if (sm.abort_flag) {
    // a copy never completed: record it, then wait (bounded) for the copies that may still be in
    // flight into this CTA's shared memory before leaving
    if (tid == 0) {
      report_error(a.err, kErrTimeout);
      for (int j = 0; j < nblk; ++j) {
        (void)mbar_wait(&sm.kfull[j], 0);
        (void)mbar_wait(&sm.vfull[j], 0);
      }
    }
    __syncthreads();
    return;
  }

  // ---------------- sums of p and integer weights per head (held by threads with lane & 3 == head)
  {
    float l = lsum;
    int w1 = wsum[0], w2 = wsum[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      w1 += __shfl_xor_sync(0xffffffffu, w1, o);
      w2 += __shfl_xor_sync(0xffffffffu, w2, o);
    }
    if (lane < kG) {
      sm.red_f[warp][lane] = l;
      sm.red_i[warp][lane] = w1;
      sm.red_i[warp][kG + lane] = w2;
    }
  }
  // value sums of the two token halves -> shared (half 1 writes, half 0 adds); rows are
  // (byte g, bit u) -> [g * 8 + u] and (byte g + 8, bit u) -> [64 + g * 8 + u]; columns head t (hi, lo)
  if (warp >= 3 && warp < 6) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = (u < 4) ? 0 : 4;
      const float v0 = 256.f * (float)(vacc[u][0] >> f) + (float)(vacc[u][1] >> f);
      const float v1 = 256.f * (float)(vacc[u][2] >> f) + (float)(vacc[u][3] >> f);
      sm.k.vacc[bg][t][g * 8 + u] = v0;          // byte g, bit u
      sm.k.vacc[bg][t][64 + g * 8 + u] = v1;     // byte g + 8, bit u
    }
  }
  __syncthreads();
  if (warp < 3) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = (u < 4) ? 0 : 4;
      const float v0 = 256.f * (float)(vacc[u][0] >> f) + (float)(vacc[u][1] >> f);
      const float v1 = 256.f * (float)(vacc[u][2] >> f) + (float)(vacc[u][3] >> f);
      sm.k.vacc[bg][t][g * 8 + u] += v0;
      sm.k.vacc[bg][t][64 + g * 8 + u] += v1;
    }
  }
  __syncthreads();

  // ---------------- partial outputs: rotated-domain value sum, QJL sum, max, sum of p
  const int stride = partial_stride(kD, kM);
  if (tid < 2 * kG) {
    int W = 0;
    for (int w = 0; w < kWarps; ++w) W += sm.red_i[w][tid];
    sm.W[tid / kG][tid % kG] = W;
  }
  __syncthreads();
  for (int i = tid; i < kG * (kD + kM); i += kThreads) {
    const int h = i / (kD + kM), j = i % (kD + kM);
    const int W1 = sm.W[0][h], W2 = sm.W[1][h];
    float v;
    if (j < kD) {
      // code c = j: byte c / 4 (group c / 64), bits 2(c % 4) (plane 0) and 2(c % 4) + 1 (plane 1)
      const int byte = j >> 2, grp = byte >> 4, bl = byte & 15, u0 = 2 * (j & 3);
      const int idx = (bl < 8) ? bl * 8 : 64 + (bl - 8) * 8;
      const float d0 = sm.k.vacc[grp][h][idx + u0], d1 = sm.k.vacc[grp][h][idx + u0 + 1];
      v = sm.dv[0][h] * (a.vc0 * (float)W1 + a.vb0 * d0 + a.vb1 * d1);
    } else {
      const int p = j - kD, byte = p >> 3, u = p & 7;
      const int idx = (byte < 8) ? byte * 8 + u : 64 + (byte - 8) * 8 + u;
      v = sm.dv[1][h] * (2.f * sm.k.vacc[2][h][idx] - (float)W2);
    }
    a.part[(((size_t)b * a.Hq + h0 + h) * a.nsplit + split) * stride + j] = v;
  }
  if (tid < kG) {
    float l = 0.f;
    for (int w = 0; w < kWarps; ++w) l += sm.red_f[w][tid];
    float* o = a.part + (((size_t)b * a.Hq + h0 + tid) * a.nsplit + split) * stride;
    o[kD + kM] = (ntok > 0) ? sm.hmax[tid] * 0.6931471805599453f : -INFINITY;   // back to natural-log units
    o[kD + kM + 1] = (ntok > 0) ? l : 0.f;
  }
}

// ================================================================ scores (tq_score)
//
// The key pass above on its own: raw scores s = ||k|| <q', c[idx]> + rnorm sqrt(pi/2)/m
// <S q, 2 sigma - 1> of every key of the chunk for the 4 query heads of a KV head,
// written to logits [B][Hq][L_cap] ("TurboQuant: redefining AI efficiency", "QJL";
// "Google TurboQuant", "Stage 2"). Key blocks of 256 stream through a 5-stage TMA ring;
// every thread stores its scores directly: per store instruction a warp writes 8
// consecutive keys of each of the 4 heads, i.e. whole 32-byte sectors. tq_score runs it with
// 15-bit code-side queries; the two-kernel attention below with the fused kernel's 22-bit ones.

constexpr int kSStages = 5;   // 5 x 13 KB: three CTAs still fit an SM, three blocks in flight per CTA
constexpr int kSStageBytes = kStageCodes + kStageSigns + 2 * kBlk * 2;  // codes, signs, norms, rnorms: 13312

struct ScoreArgs {
  const float* qr;  // [B*Hq][128] Pi q
  const float* qs;  // [B*Hq][128] S q
  int B, Hq, Hkv;
  const uint8_t* kcodes;
  const uint8_t* ksigns;
  const __half* knorm;
  const __half* krn;
  int64_t L_cap, chunk;
  const int32_t* len;
  int len_extra;    // 1 inside a decode step: the key appended at slot len[b] by the kernel before counts
  float kc0, kb0, kb1;
  float* logits;    // [B][Hq][L_cap]
  int* err;
};

struct __align__(16) ScoreSmem {
  unsigned char stage[kSStages][kSStageBytes];
  uint32_t qfrag[2][12][2][4][8];
  float qconst[kG][4];
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  int abort_flag;
};

// LO: 22-bit code-side queries and the decode-step slot handling (the two-kernel attention's
// scores), else 15-bit queries (tq_score's raw scores).
template <bool LO>
__global__ void __launch_bounds__(kThreads, 3) score_prod2_kernel(ScoreArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / a.Hkv, hk = bh % a.Hkv, h0 = hk * kG;
  const int64_t L = min((int64_t)max(a.len[b], 0) + (LO ? a.len_extra : 0), a.L_cap);
  const int64_t start = (int64_t)split * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  const int ntok = (int)max((int64_t)0, end - start);
  const int nblk = (ntok + kBlk - 1) / kBlk;
  const int64_t row0 = (int64_t)bh * a.L_cap + start;
  if (nblk == 0) return;
  // inside a decode step the kernel before this one writes slot len[b]; copies issued before the
  // wait below may hold that key's old rows, so the one warp that scores it reads them again
  const int64_t slot = (int64_t)max(a.len[b], 0);
  const int s_loc = (LO && a.len_extra && slot >= start && slot < end) ? (int)(slot - start) : -1;

  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int j) {
    const int64_t tok0 = (int64_t)j * kBlk;
    const int ncopy = (int)min((int64_t)kBlk, a.L_cap - (start + tok0));   // multiple of 8 (L_cap % 8 == 0)
    const int64_t r = row0 + tok0;
    unsigned char* st = sm.stage[j % kSStages];
    uint64_t* bar = &sm.full[j % kSStages];
    mbar_expect_tx(bar, (uint32_t)ncopy * (kCodesB + kSignsB + 4));
    tma_bulk_g2s(st, a.kcodes + r * kCodesB, ncopy * kCodesB, bar);
    tma_bulk_g2s(st + kStageCodes, a.ksigns + r * kSignsB, ncopy * kSignsB, bar);
    tma_bulk_g2s(st + kStageCodes + kStageSigns, a.knorm + r, ncopy * 2, bar);
    tma_bulk_g2s(st + kStageCodes + kStageSigns + 2 * kBlk, a.krn + r, ncopy * 2, bar);
  };
  constexpr int kAhead = kSStages - 2;
  if (tid == 0)
    for (int j = 0; j < min(kAhead, nblk); ++j) issue(j);
  int issued = min(kAhead, nblk);
  grid_dep_wait();   // the rotated queries come from the kernel before this one

  prepare_query(a.qr + ((size_t)b * a.Hq + h0) * kD, a.qs + ((size_t)b * a.Hq + h0) * kM, a.kb0, a.kb1, a.kc0,
                sm.qfrag, sm.qconst);
  __syncthreads();
  uint32_t qb[12][2];
#pragma unroll
  for (int kk = 0; kk < 12; ++kk)
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) qb[kk][slot] = sm.qfrag[0][kk][slot][t][g];
  // lo-piece fragments stay in shared memory here (three CTAs per SM leave no room in registers)
  const uint32_t* qlo = &sm.qfrag[1][0][0][t][g];
  auto lo_smem = [&](int kk, int sl) { return qlo[(kk * 2 + sl) * 32]; };
  const float c0h = sm.qconst[t][0], dmh = sm.qconst[t][1], dsh = sm.qconst[t][2], ssh = sm.qconst[t][3];
  float* lrow = a.logits + ((size_t)b * a.Hq + h0 + t) * a.L_cap + start;   // head t's scores of the chunk

  // No thread leaves this loop early (see attn_prod2_kernel): a wait that runs out stops
  // new copies and further waits, and the remaining blocks are skipped uniformly.
  for (int j = 0; j < nblk; ++j) {
    // warp-uniform (the guarded code is warp-collective)
    const bool aborted = __any_sync(0xffffffffu, *(volatile int*)&sm.abort_flag != 0);
    if (tid == 0 && !aborted && j + kAhead < nblk) {
      const int jo = j + kAhead - kSStages;   // the stage's previous block (j - 2)
      if (jo >= 0 && !mbar_wait(&sm.empty[jo % kSStages], (jo / kSStages) & 1)) {
        sm.abort_flag = 1;
      } else {
        issue(j + kAhead);
        issued = j + kAhead + 1;
      }
    }
    if (!aborted && !mbar_wait(&sm.full[j % kSStages], (j / kSStages) & 1)) sm.abort_flag = 1;
    const unsigned char* st = sm.stage[j % kSStages];
    if (LO && !aborted && s_loc >= 0 && s_loc / kBlk == j && warp == ((s_loc % kBlk) % 128) / 16) {
      // the warp whose m-tiles hold the appended key (rows 16w.. and 128 + 16w..) patches its rows
      const int kk = s_loc & (kBlk - 1);
      const int64_t r = row0 + s_loc;
      unsigned char* sw = sm.stage[j % kSStages];
      if (lane < 8)
        reinterpret_cast<uint32_t*>(sw + kk * kCodesB)[lane] = __ldcg(reinterpret_cast<const uint32_t*>(a.kcodes + r * kCodesB) + lane);
      else if (lane < 12)
        reinterpret_cast<uint32_t*>(sw + kStageCodes + kk * kSignsB)[lane - 8] =
            __ldcg(reinterpret_cast<const uint32_t*>(a.ksigns + r * kSignsB) + lane - 8);
      else if (lane == 12)
        reinterpret_cast<__half*>(sw + kStageCodes + kStageSigns)[kk] = __ldcg(a.knorm + r);
      else if (lane == 13)
        reinterpret_cast<__half*>(sw + kStageCodes + kStageSigns)[kBlk + kk] = __ldcg(a.krn + r);
      __syncwarp();
    }
    const __half* nrm = reinterpret_cast<const __half*>(st + kStageCodes + kStageSigns);
    const __half* rnm = nrm + kBlk;
    const int tb = j * kBlk, nvalid = min(kBlk, ntok - tb);
    float sc[2][2];
    if (!aborted) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int kb1[1] = {128 * mt + 16 * warp};
        float sc1[1][2];
        mtile_scores<1, LO>(st, st + kStageCodes, nrm, rnm, kb1, qb, lo_smem, c0h, dmh, dsh, ssh, sc1);
        sc[mt][0] = sc1[0][0], sc[mt][1] = sc1[0][1];
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&sm.empty[j % kSStages])) : "memory");
    if (!aborted) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int key = 128 * mt + 16 * warp + g + 8 * r;
          if (key < nvalid) lrow[tb + key] = sc[mt][r];
        }
    }
  }
  __syncthreads();
  if (sm.abort_flag && tid == 0) {
    report_error(a.err, kErrTimeout);
    for (int jx = max(0, issued - kSStages); jx < issued; ++jx) (void)mbar_wait(&sm.full[jx % kSStages], (jx / kSStages) & 1);
  }
}


// ================================================================ value pass over stored scores
//
// The second half of a two-kernel form of attn_prod2_kernel for caches much larger than L2: the
// score kernel above (22-bit queries, the same logits as the fused kernel's key pass) writes every
// key's raw score, and this kernel turns a chunk's scores into the same 16-bit integer weights
// (against each head's largest p ||v|| and p rnorm in the chunk) and runs the same value pass over
// value blocks streamed through a TMA ring, writing the same partial results. Both halves stream
// through small rings with three CTAs per SM, which keeps more of the cold read in flight than the
// fused kernel's whole-chunk staging (two CTAs per SM).
struct VArgs {
  const float* logits;  // [B][Hq][L_cap] raw scores (score_prod2_kernel<true>)
  int B, Hq, Hkv;
  const uint8_t* vcodes;
  const uint8_t* vsigns;
  const __half* vnorm;
  const __half* vrn;
  int64_t L_cap, chunk;
  int nsplit;
  const int32_t* len;
  int len_extra;
  float vc0, vb0, vb1;  // V codebook
  float scale;
  float* part;          // [B*Hq][nsplit][d + m + 2]
  int* err;
};

constexpr int kVStages = 4;
constexpr int kVStageBytes = kStageCodes + kStageSigns;   // 12288
constexpr int kVAhead = kVStages - 2;

struct __align__(16) VSmem {
  unsigned char stage[kVStages][kVStageBytes];
  uint8_t pw[2][2][8][kPwRow];   // [buffer][0: value weights, 1: QJL weights][col = head*2+piece][token]
  float vacc[3][kG][128];
  float red[kWarps][3][kG];
  int red_i[kWarps][2 * kG];
  float hmax[kG];
  float dv[2][kG];
  float inv[2][kG];
  int W[2][kG];
  uint64_t full[kVStages];
  uint64_t empty[kVStages];
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 3) value_prod2_kernel(VArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  VSmem& sm = *reinterpret_cast<VSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / a.Hkv, hk = bh % a.Hkv, h0 = hk * kG;
  // the scores and, in a decode step, the appended value come from the kernels before this one
  // (which this one starts after: the score kernel triggers nothing early)
  grid_dep_wait();
  const int64_t L = min((int64_t)max(a.len[b], 0) + a.len_extra, a.L_cap);
  const int64_t start = (int64_t)split * a.chunk;
  const int64_t end = min(L, start + a.chunk);
  const int ntok = (int)max((int64_t)0, end - start);
  const int nblk = (ntok + kBlk - 1) / kBlk;
  const int64_t row0 = (int64_t)bh * a.L_cap + start;
  const int stride = partial_stride(kD, kM);
  if (ntok == 0) {   // an empty chunk: zero sums, max -inf
    for (int i = tid; i < kG * stride; i += kThreads) {
      const int h = i / stride, j = i - h * stride;
      a.part[(((size_t)b * a.Hq + h0 + h) * a.nsplit + split) * stride + j] = (j == kD + kM) ? -INFINITY : 0.f;
    }
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int j) {
    const int64_t tok0 = (int64_t)j * kBlk;
    const int ncopy = (int)min((int64_t)kBlk, a.L_cap - (start + tok0));   // multiple of 8 (L_cap % 8 == 0)
    const int64_t r = row0 + tok0;
    unsigned char* st = sm.stage[j % kVStages];
    uint64_t* bar = &sm.full[j % kVStages];
    mbar_expect_tx(bar, (uint32_t)ncopy * (kCodesB + kSignsB));
    tma_bulk_g2s(st, a.vcodes + r * kCodesB, ncopy * kCodesB, bar);
    tma_bulk_g2s(st + kStageCodes, a.vsigns + r * kSignsB, ncopy * kSignsB, bar);
  };
  if (tid == 0)
    for (int j = 0; j < min(kVAhead, nblk); ++j) issue(j);
  int issued = min(kVAhead, nblk);

  // ---- per head over the chunk: the largest l, l + log2 ||v|| and l + log2 rnorm (l = the score
  // in log2 units), so that the weight steps max p ||v|| / 65535 and max p rnorm / 65535 are known
  // before the first value block
  const float scale2 = a.scale * 1.4426950408889634f;
  const float* lg = a.logits + ((size_t)b * a.Hq + h0) * a.L_cap + start;   // head h: lg + h * L_cap
  {
    const int h = t;
    float m = -INFINITY, m1 = -INFINITY, m2 = -INFINITY;
    for (int tok = tid >> 2; tok < ntok; tok += kThreads / 4) {
      const float l = lg[(size_t)h * a.L_cap + tok] * scale2;
      const float vn = __half2float(a.vnorm[row0 + tok]), vr = __half2float(a.vrn[row0 + tok]);
      m = fmaxf(m, l);
      m1 = fmaxf(m1, l + __log2f(vn));
      m2 = fmaxf(m2, l + __log2f(vr));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    }
    if (g == 0) sm.red[warp][0][h] = m, sm.red[warp][1][h] = m1, sm.red[warp][2][h] = m2;
  }
  __syncthreads();
  if (tid < kG) {
    float m = -INFINITY, m1 = -INFINITY, m2 = -INFINITY;
    for (int w = 0; w < kWarps; ++w) {
      m = fmaxf(m, sm.red[w][0][tid]);
      m1 = fmaxf(m1, sm.red[w][1][tid]);
      m2 = fmaxf(m2, sm.red[w][2][tid]);
    }
    sm.hmax[tid] = m;
    const float s1 = exp2f(m1 - m) / 65535.f, s2 = exp2f(m2 - m) / 65535.f;
    sm.dv[0][tid] = s1 > 0.f ? s1 : 1.f;
    sm.inv[0][tid] = s1 > 0.f ? 1.f / s1 : 0.f;
    sm.dv[1][tid] = s2 > 0.f ? s2 : 1.f;
    sm.inv[1][tid] = s2 > 0.f ? 1.f / s2 : 0.f;
  }
  __syncthreads();
  // ---- value blocks: weights of the block (all threads) into one of two weight buffers, then
  // the value MMAs (warps 0..5: three byte groups x two token halves), exactly as in the fused kernel
  const int h = tid & 3, q4 = (tid >> 2) * 4;
  const float hm = sm.hmax[h], inv1 = sm.inv[0][h], inv2 = sm.inv[1][h];
  // round to nearest (even) through the float adder (0 <= x < 2^22)
  auto to_int = [](float x) { return __float_as_int(x + 12582912.f) - 0x4B400000; };
  float lsum = 0.f;
  int wsum[2] = {0, 0};
  int vacc[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u) vacc[u][0] = vacc[u][1] = vacc[u][2] = vacc[u][3] = 0;
  const int bg = warp % 3, half = warp / 3;
  for (int jj = 0; jj < nblk; ++jj) {
    const bool aborted = __syncthreads_or(*(volatile int*)&sm.abort_flag != 0);   // uniform decision
    if (aborted) break;
    if (tid == 0 && jj + kVAhead < nblk) {
      const int jo = jj + kVAhead - kVStages;   // the stage's previous block
      if (jo >= 0 && !mbar_wait(&sm.empty[jo % kVStages], (jo / kVStages) & 1)) {
        sm.abort_flag = 1;
      } else {
        issue(jj + kVAhead);
        issued = jj + kVAhead + 1;
      }
    }
    {
      const int tb = jj * kBlk, nval = min(kBlk, ntok - tb);
      uint32_t w1h = 0, w1l = 0, w2h = 0, w2l = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int tok = tb + q4 + q;
        if (q4 + q < nval) {   // tokens past the chunk's end get zero weight
          const float l = lg[(size_t)h * a.L_cap + tok] * scale2;
          const float pp = exp2_approx(l - hm);
          lsum += pp;
          const float vn = __half2float(a.vnorm[row0 + tok]), vr = __half2float(a.vrn[row0 + tok]);
          const int w1 = min(to_int(pp * vn * inv1), 65535), w2 = min(to_int(pp * vr * inv2), 65535);
          w1h |= (uint32_t)(w1 >> 8) << (8 * q);
          w1l |= (uint32_t)(w1 & 255) << (8 * q);
          w2h |= (uint32_t)(w2 >> 8) << (8 * q);
          w2l |= (uint32_t)(w2 & 255) << (8 * q);
          wsum[0] += w1;
          wsum[1] += w2;
        }
      }
      uint8_t* blk = &sm.pw[jj & 1][0][0][0];
      *reinterpret_cast<uint32_t*>(blk + (2 * h) * kPwRow + q4) = w1h;
      *reinterpret_cast<uint32_t*>(blk + (2 * h + 1) * kPwRow + q4) = w1l;
      *reinterpret_cast<uint32_t*>(blk + (8 + 2 * h) * kPwRow + q4) = w2h;
      *reinterpret_cast<uint32_t*>(blk + (8 + 2 * h + 1) * kPwRow + q4) = w2l;
    }
    bool ok = true;
    if (warp < 6 && !mbar_wait(&sm.full[jj % kVStages], (jj / kVStages) & 1)) ok = false;
    if (!ok && lane == 0) sm.abort_flag = 1;
    __syncthreads();   // the block's weights are written (and the previous block's MMAs are done)
    if (warp < 6 && __all_sync(0xffffffffu, ok)) {
      const uint8_t* pw = &sm.pw[jj & 1][bg == 2 ? 1 : 0][0][0];
      const unsigned char* vc = sm.stage[jj % kVStages];
      const unsigned char* vs = vc + kStageCodes;
      const int nvalv = min(kBlk, ntok - jj * kBlk);
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const int tk = 128 * half + 32 * kq;  // first token of this 32-token k-step
        if (tk >= nvalv) break;               // past the chunk's end (weights 0; warp-uniform)
        uint32_t r[4];
        const int tok = tk + (lane & 15) + 16 * (lane >> 4);
        const unsigned char* rowp = (bg < 2) ? vc + tok * kCodesB + 16 * bg : vs + tok * kSignsB;
        ldsm_t8_x2(r, rowp);
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(pw + g * kPwRow + tk + 4 * t);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(pw + g * kPwRow + tk + 16 + 4 * t);
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const uint32_t x0 = r[0] >> s4, x1 = r[1] >> s4, x2 = r[2] >> s4, x3 = r[3] >> s4;
          mma_u8(vacc[s4], x0 & 0x01010101u, x1 & 0x01010101u, x2 & 0x01010101u, x3 & 0x01010101u, b0, b1);
          mma_u8(vacc[4 + s4], x0 & 0x10101010u, x1 & 0x10101010u, x2 & 0x10101010u, x3 & 0x10101010u, b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&sm.empty[jj % kVStages])) : "memory");
  }

  __syncthreads();
  if (sm.abort_flag) {
    // a copy never completed: record it, then wait (bounded) for the copies that may still be in
    // flight into this CTA's shared memory before leaving
    if (tid == 0) {
      report_error(a.err, kErrTimeout);
      for (int jx = max(0, issued - kVStages); jx < issued; ++jx)
        (void)mbar_wait(&sm.full[jx % kVStages], (jx / kVStages) & 1);
    }
    __syncthreads();
    return;
  }

  // ---- sums of p and integer weights per head, value sums of the two token halves
  {
    float l = lsum;
    int w1 = wsum[0], w2 = wsum[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      w1 += __shfl_xor_sync(0xffffffffu, w1, o);
      w2 += __shfl_xor_sync(0xffffffffu, w2, o);
    }
    if (lane < kG) {
      sm.red[warp][0][lane] = l;
      sm.red_i[warp][lane] = w1;
      sm.red_i[warp][kG + lane] = w2;
    }
  }
  if (warp >= 3 && warp < 6) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = (u < 4) ? 0 : 4;
      const float v0 = 256.f * (float)(vacc[u][0] >> f) + (float)(vacc[u][1] >> f);
      const float v1 = 256.f * (float)(vacc[u][2] >> f) + (float)(vacc[u][3] >> f);
      sm.vacc[bg][t][g * 8 + u] = v0;          // byte g, bit u
      sm.vacc[bg][t][64 + g * 8 + u] = v1;     // byte g + 8, bit u
    }
  }
  __syncthreads();
  if (warp < 3) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = (u < 4) ? 0 : 4;
      const float v0 = 256.f * (float)(vacc[u][0] >> f) + (float)(vacc[u][1] >> f);
      const float v1 = 256.f * (float)(vacc[u][2] >> f) + (float)(vacc[u][3] >> f);
      sm.vacc[bg][t][g * 8 + u] += v0;
      sm.vacc[bg][t][64 + g * 8 + u] += v1;
    }
  }
  if (tid < 2 * kG) {
    int W = 0;
    for (int w = 0; w < kWarps; ++w) W += sm.red_i[w][tid];
    sm.W[tid / kG][tid % kG] = W;
  }
  __syncthreads();

  // ---- partial outputs: rotated-domain value sum, QJL sum, max (natural-log units), sum of p
  for (int i = tid; i < kG * (kD + kM); i += kThreads) {
    const int hh = i / (kD + kM), j = i % (kD + kM);
    const int W1 = sm.W[0][hh], W2 = sm.W[1][hh];
    float v;
    if (j < kD) {
      // code c = j: byte c / 4 (group c / 64), bits 2(c % 4) (plane 0) and 2(c % 4) + 1 (plane 1)
      const int byte = j >> 2, grp = byte >> 4, bl = byte & 15, u0 = 2 * (j & 3);
      const int idx = (bl < 8) ? bl * 8 : 64 + (bl - 8) * 8;
      const float d0 = sm.vacc[grp][hh][idx + u0], d1 = sm.vacc[grp][hh][idx + u0 + 1];
      v = sm.dv[0][hh] * (a.vc0 * (float)W1 + a.vb0 * d0 + a.vb1 * d1);
    } else {
      const int p = j - kD, byte = p >> 3, u = p & 7;
      const int idx = (byte < 8) ? byte * 8 + u : 64 + (byte - 8) * 8 + u;
      v = sm.dv[1][hh] * (2.f * sm.vacc[2][hh][idx] - (float)W2);
    }
    a.part[(((size_t)b * a.Hq + h0 + hh) * a.nsplit + split) * stride + j] = v;
  }
  if (tid < kG) {
    float l = 0.f;
    for (int w = 0; w < kWarps; ++w) l += sm.red[w][0][tid];
    float* o = a.part + (((size_t)b * a.Hq + h0 + tid) * a.nsplit + split) * stride;
    o[kD + kM] = sm.hmax[tid] * 0.6931471805599453f;   // back to natural-log units
    o[kD + kM + 1] = l;
  }
}

}  // namespace amma
}  // namespace tqk
