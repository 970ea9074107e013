// C ABI of libtq.so (declared in include/tq.h): handle lifetime, argument
// validation, workspace layout and kernel launches. Every entry point returns
// a status and records a message for tq_last_error(); nothing throws.
//
// Fault injection for tests (host side only; no GPU fault is ever caused):
//   TQ_FAULT=alloc   -> tq_create* fails with TQ_ENOMEM before allocating
//   TQ_FAULT=launch  -> hot calls fail with TQ_ECUDA before launching
//   TQ_FAULT=timeout -> hot calls record a wait timeout in the handle's error word (no wait
//                       happens), as a kernel does when a copy never arrives
// Checks: TQ_CHECK=1 makes the hot calls that read device lengths first validate every
// len[b] against 0 .. L_cap on the device, recording an out-of-range length in the handle's
// error word (tq_last_status: TQ_EINVAL) instead of clamping it silently.
// Tracing: every hot call is an NVTX range named after the entry point.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "tq.h"
#include "host_math.h"
#include "internal.h"
#include "common.cuh"
#include "encode_simt.cuh"
#include "encode_rows.cuh"
#include "score_attn_simt.cuh"
#include "search_simt.cuh"
#include "attn_mma.cuh"
#include "attn_tc.cuh"
#include "small_kernels.cuh"
#include "encode_tc.cuh"
#include "attn_mse4.cuh"
#include "search_tc.cuh"
#include "encode_big_tc.cuh"
#include "polar.cuh"

struct tq_handle {
  int d = 0, bits = 0, m = 0, norm_dtype = TQ_F32;
  uint64_t seed = 0;
  int codes_B = 0, signs_B = 0;
  int device = 0;
  std::vector<double> Pi, S, cent, bnd;  // host fp64
  float* dPi = nullptr;   // [d][d]   y = Pi u
  float* dPiT = nullptr;  // [d][d]   transpose
  float* dS = nullptr;    // [m][d]
  float* dST = nullptr;   // [d][m]   S^T
  float* dMT = nullptr;   // [d][m]   (S Pi^T)^T
  float* dcent = nullptr; // [2^bits]
  float* dbnd = nullptr;  // [2^bits - 1]
  int* derr = nullptr;    // device error word
  uint8_t* dOps = nullptr; // d = 128: pre-swizzled 16-bit hi/lo operands of the tensor-core encode
  uint16_t* dPiB = nullptr; // MSE, d % 256 = 0, 256 <= d <= 4096: Pi as a bf16 pair, [2][d][d] (hi rows, lo rows)
  // recursive polar transform handles (tq_create_polar): per-level angle codebooks
  int polar = 0;
  tqk::polar::Layout play{};
  std::vector<std::vector<double>> pcent, pbnd;
  tqk::polar::Table* dTab = nullptr;
};

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return TQ_OK;
}

bool fault_is(const char* what) {
  const char* f = std::getenv("TQ_FAULT");
  return f && std::strcmp(f, what) == 0;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(TQ_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define TQ_CUDA(call)                                   \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// One NVTX range per hot call (free when no profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

bool check_mode() {
  const char* c = std::getenv("TQ_CHECK");
  return c && std::strcmp(c, "1") == 0;
}

int launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return ok();
}

// True the first time (kernel slot, device) is seen: per-device one-time kernel attributes.
bool once_per_device(int slot, int device) {
  static std::atomic<uint64_t> seen[32];
  if (slot < 0 || slot >= 32 || device < 0 || device >= 64) return true;
  const uint64_t bit = 1ull << device;
  return (seen[slot].fetch_or(bit) & bit) == 0;
}

// ---- kernel timer: events recorded around launches while enabled
struct TimedLaunch {
  std::string name;
  cudaEvent_t start, stop;
};
std::mutex g_timer_mu;
std::atomic<bool> g_timer_on{false};
std::vector<TimedLaunch> g_timer_pending;
std::vector<cudaEvent_t> g_timer_pool;

cudaEvent_t timer_event() {
  if (!g_timer_pool.empty()) {
    cudaEvent_t e = g_timer_pool.back();
    g_timer_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one kernel launch with events when the timer is on. Inside a stream
// capture the records become real event-record nodes of the graph
// (cudaEventRecordExternal), re-recorded by every replay.
struct KernelScope {
  const char* name;
  cudaStream_t stream;
  cudaEvent_t start = nullptr, stop = nullptr;
  unsigned flags = cudaEventRecordDefault;
  KernelScope(const char* n, cudaStream_t s) : name(n), stream(s) {
    if (!g_timer_on.load(std::memory_order_relaxed)) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      flags = cudaEventRecordExternal;
    std::lock_guard<std::mutex> lk(g_timer_mu);
    start = timer_event();
    stop = timer_event();
    cudaEventRecordWithFlags(start, stream, flags);
  }
  ~KernelScope() {
    if (!start) return;
    cudaEventRecordWithFlags(stop, stream, flags);
    std::lock_guard<std::mutex> lk(g_timer_mu);
    g_timer_pending.push_back({name, start, stop});
  }
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_dtype(int dt) { return dt == TQ_F32 || dt == TQ_F16 || dt == TQ_BF16; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

void free_device(tq_handle* h) {
  cudaFree(h->dPi);
  cudaFree(h->dPiT);
  cudaFree(h->dS);
  cudaFree(h->dST);
  cudaFree(h->dMT);
  cudaFree(h->dcent);
  cudaFree(h->dbnd);
  cudaFree(h->derr);
  cudaFree(h->dOps);
  cudaFree(h->dPiB);
  h->dPiB = nullptr;
  cudaFree(h->dTab);
  h->dPi = h->dPiT = h->dS = h->dST = h->dMT = h->dcent = h->dbnd = nullptr;
  h->derr = nullptr;
  h->dOps = nullptr;
  h->dTab = nullptr;
}

template <typename T>
int upload(T** dst, const std::vector<T>& src, const char* what) {
  if (src.empty()) return TQ_OK;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), src.size() * sizeof(T));
  if (e != cudaSuccess) return fail(TQ_ENOMEM, "cudaMalloc(%s): %s", what, cudaGetErrorString(e));
  e = cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return TQ_OK;
}

// One [128][128] matrix of 16-bit values (row n, reduction index k) in the 128-byte-swizzled
// K-major layout the tensor-core encode reads: two atoms of K 0..63 and 64..127, row n at
// byte 128 n of its atom, 16-byte chunk c at chunk position c ^ (n % 8).
void swizzle_k128(const std::vector<uint16_t>& src, uint8_t* dst) {
  for (int n = 0; n < 128; ++n)
    for (int k = 0; k < 128; ++k) {
      const int atom = k >> 6, chunk = (k & 63) >> 3, e = k & 7;
      const size_t off = (size_t)atom * tqk::etc::kAtom + (size_t)n * 128 + (size_t)((chunk ^ (n & 7)) << 4) + e * 2;
      std::memcpy(dst + off, &src[(size_t)n * 128 + k], 2);
    }
}

// Tensor-core operands of a d = 128 handle: Pi (bf16 and f16 hi/lo pairs) and, for prod
// with m = 128, M = S Pi^T (bf16 hi/lo): value = hi + lo with lo the rounded remainder.
std::vector<uint8_t> tc_operands(const std::vector<double>& Pi, const std::vector<double>& M) {
  const size_t mat = tqk::etc::kMat;
  std::vector<uint8_t> ops(mat * tqk::etc::kOpCount, 0);
  std::vector<uint16_t> hi(128 * 128), lo(128 * 128);
  auto split_bf16 = [&](const std::vector<double>& A) {
    for (size_t i = 0; i < A.size(); ++i) {
      const __nv_bfloat16 h = __float2bfloat16((float)A[i]);
      hi[i] = __bfloat16_as_ushort(h);
      lo[i] = __bfloat16_as_ushort(__float2bfloat16((float)(A[i] - (double)__bfloat162float(h))));
    }
  };
  auto split_f16 = [&](const std::vector<double>& A) {
    for (size_t i = 0; i < A.size(); ++i) {
      const __half h = __float2half((float)A[i]);
      hi[i] = __half_as_ushort(h);
      lo[i] = __half_as_ushort(__float2half((float)(A[i] - (double)__half2float(h))));
    }
  };
  split_bf16(Pi);
  swizzle_k128(hi, ops.data() + tqk::etc::kOpPiBf16Hi * mat);
  swizzle_k128(lo, ops.data() + tqk::etc::kOpPiBf16Lo * mat);
  split_f16(Pi);
  swizzle_k128(hi, ops.data() + tqk::etc::kOpPiF16Hi * mat);
  swizzle_k128(lo, ops.data() + tqk::etc::kOpPiF16Lo * mat);
  if (!M.empty()) {
    split_bf16(M);
    swizzle_k128(hi, ops.data() + tqk::etc::kOpMHi * mat);
    swizzle_k128(lo, ops.data() + tqk::etc::kOpMLo * mat);
  }
  return ops;
}

int create_common(int d, int bits_mse, int m, uint64_t seed, int norm_dtype, tq_handle** out) {
  if (!out) return fail(TQ_EINVAL, "out is NULL");
  *out = nullptr;
  if (d < 32 || d > 4096) return fail(TQ_EUNSUPPORTED, "d=%d outside 32..4096", d);
  if (d % 32 != 0) return fail(TQ_EUNSUPPORTED, "d=%d is not a multiple of 32", d);
  if (bits_mse < (m > 0 ? 0 : 1) || bits_mse > 4) return fail(TQ_EUNSUPPORTED, "MSE bits=%d outside 1..4", bits_mse);
  if (m < 0 || m % 32 != 0 || m > 1024) return fail(TQ_EUNSUPPORTED, "qjl_m=%d (needs m %% 32 == 0, m <= 1024)", m);
  if (m > 0 && d > tqk::kEncBN) return fail(TQ_EUNSUPPORTED, "prod handles need d <= %d", tqk::kEncBN);
  if (fault_is("alloc")) return fail(TQ_ENOMEM, "injected allocation failure (TQ_FAULT=alloc)");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");

  tq_handle* h = new tq_handle();
  h->d = d;
  h->bits = bits_mse;
  h->m = m;
  h->seed = seed;
  h->norm_dtype = norm_dtype;
  h->device = dev;
  h->codes_B = d * bits_mse / 8;
  h->signs_B = m / 8;
  const int L = 1 << bits_mse;
  h->Pi.resize((size_t)d * d);
  h->S.resize((size_t)m * d);
  h->cent.resize(L);
  h->bnd.resize(L - 1);
  tqhost::rotation(d, m, seed, h->Pi.data(), m ? h->S.data() : nullptr);
  if (bits_mse == 0) {
    // QJL-only rows: no MSE stage; its one-cell codebook is the coordinate law's mean, 0
    h->cent[0] = 0.0;
  } else if (tqhost::codebook(d, bits_mse, h->cent.data(), h->bnd.data()) != 0) {
    delete h;
    return fail(TQ_EINVAL, "codebook(d=%d, bits=%d) failed", d, bits_mse);
  }
  std::vector<float> Pi(h->Pi.begin(), h->Pi.end()), PiT((size_t)d * d), S(h->S.begin(), h->S.end()),
      ST((size_t)d * m), MT((size_t)d * m), cent(h->cent.begin(), h->cent.end()), bnd(h->bnd.begin(), h->bnd.end());
  for (int i = 0; i < m; ++i)
    for (int k = 0; k < d; ++k) ST[(size_t)k * m + i] = (float)h->S[(size_t)i * d + k];
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) PiT[(size_t)j * d + i] = (float)h->Pi[(size_t)i * d + j];
  // M = S Pi^T (m x d): M[i][k] = sum_j S[i][j] Pi[k][j]; stored transposed MT[k][i].
  std::vector<double> M((size_t)m * d);
  for (int i = 0; i < m; ++i)
    for (int k = 0; k < d; ++k) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += h->S[(size_t)i * d + j] * h->Pi[(size_t)k * d + j];
      M[(size_t)i * d + k] = acc;
      MT[(size_t)k * m + i] = (float)acc;
    }
  std::vector<uint8_t> ops;
  if (d == tqk::etc::kD && (m == 0 || m == tqk::etc::kD)) ops = tc_operands(h->Pi, M);
  // Pi = Pi_h + Pi_l as bf16 (round to nearest even), for the tensor-core encode of large d
  std::vector<uint16_t> pib;
  if (m == 0 && bits_mse > 0 && d % tqk::ebig::kN == 0 && d >= tqk::ebig::kMinD && d <= tqk::ebig::kMaxD) {
    pib.resize((size_t)2 * d * d);
    auto bf16 = [](float f) {
      uint32_t u;
      std::memcpy(&u, &f, 4);
      u += 0x7FFFu + ((u >> 16) & 1u);
      return (uint16_t)(u >> 16);
    };
    for (size_t i = 0; i < (size_t)d * d; ++i) {
      const float v = (float)h->Pi[i];
      const uint16_t hi = bf16(v);
      const uint32_t hb = (uint32_t)hi << 16;
      float hf;
      std::memcpy(&hf, &hb, 4);
      pib[i] = hi;
      pib[(size_t)d * d + i] = bf16((float)(h->Pi[i] - (double)hf));
    }
  }
  int st = TQ_OK;
  if ((st = upload(&h->dPi, Pi, "Pi")) || (st = upload(&h->dPiT, PiT, "PiT")) ||
      (st = upload(&h->dS, S, "S")) || (st = upload(&h->dST, ST, "ST")) || (st = upload(&h->dMT, MT, "MT")) ||
      (st = upload(&h->dcent, cent, "centroids")) || (st = upload(&h->dbnd, bnd, "bounds")) ||
      (st = upload(&h->dOps, ops, "tensor-core operands")) || (st = upload(&h->dPiB, pib, "bf16 rotation pair"))) {
    free_device(h);
    delete h;
    return st;
  }
  e = cudaMalloc(&h->derr, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(h->derr, 0, sizeof(int));
  if (e != cudaSuccess) {
    free_device(h);
    delete h;
    return fail(TQ_ENOMEM, "cudaMalloc(error word): %s", cudaGetErrorString(e));
  }
  *out = h;
  return ok();
}

// Recursive polar transform handle: d a power of two (32 .. 256), log2 d levels, bits1 at
// level 1 and bits_up at every further level (each 1..4); Pi as for the MSE path (seed).
int create_polar(int d, int bits1, int bits_up, uint64_t seed, tq_handle** out) {
  if (!out) return fail(TQ_EINVAL, "out is NULL");
  *out = nullptr;
  if (d < 32 || d > 256 || (d & (d - 1)) != 0)
    return fail(TQ_EUNSUPPORTED, "polar handles need d a power of two in 32..256 (d=%d)", d);
  if (bits1 < 1 || bits1 > 4 || bits_up < 1 || bits_up > 4)
    return fail(TQ_EUNSUPPORTED, "polar level bits %d/%d outside 1..4", bits1, bits_up);
  if (fault_is("alloc")) return fail(TQ_ENOMEM, "injected allocation failure (TQ_FAULT=alloc)");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  tq_handle* h = new tq_handle();
  h->d = d;
  h->bits = 0;
  h->m = 0;
  h->seed = seed;
  h->norm_dtype = TQ_F32;
  h->device = dev;
  h->polar = 1;
  int nlev = 0;
  while ((1 << nlev) < d) ++nlev;
  h->play.d = d;
  h->play.nlev = nlev;
  int off = 0;
  tqk::polar::Table tab{};
  h->pcent.resize(nlev);
  h->pbnd.resize(nlev);
  for (int l = 0; l < nlev; ++l) {
    const int b = l == 0 ? bits1 : bits_up, L = 1 << b;
    h->play.bits[l] = b;
    h->play.off[l] = off;
    off += (d >> (l + 1)) * b;
    h->pcent[l].resize(L);
    h->pbnd[l].resize(L - 1);
    if (tqhost::polar_codebook(l + 1, b, h->pcent[l].data(), h->pbnd[l].data()) != 0) {
      delete h;
      return fail(TQ_EINVAL, "polar codebook (level %d, %d bits) failed", l + 1, b);
    }
    for (int i = 0; i < 16; ++i) tab.bnd[l][i] = i < L - 1 ? (float)h->pbnd[l][i] : INFINITY;
    for (int i = 0; i < L; ++i) {
      tab.cs[l][i] = (float)std::cos(h->pcent[l][i]);
      tab.sn[l][i] = (float)std::sin(h->pcent[l][i]);
    }
  }
  h->codes_B = 16 * ((off + 127) / 128);
  h->signs_B = 0;
  h->Pi.resize((size_t)d * d);
  tqhost::rotation(d, 0, seed, h->Pi.data(), nullptr);
  std::vector<float> Pi(h->Pi.begin(), h->Pi.end()), PiT((size_t)d * d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) PiT[(size_t)j * d + i] = (float)h->Pi[(size_t)i * d + j];
  std::vector<uint8_t> tb(sizeof(tab));
  std::memcpy(tb.data(), &tab, sizeof(tab));
  int st = TQ_OK;
  if ((st = upload(&h->dPi, Pi, "Pi")) || (st = upload(&h->dPiT, PiT, "PiT")) ||
      (st = upload(reinterpret_cast<uint8_t**>(&h->dTab), tb, "polar tables"))) {
    free_device(h);
    delete h;
    return st;
  }
  e = cudaMalloc(&h->derr, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(h->derr, 0, sizeof(int));
  if (e != cudaSuccess) {
    free_device(h);
    delete h;
    return fail(TQ_ENOMEM, "cudaMalloc(error word): %s", cudaGetErrorString(e));
  }
  *out = h;
  return ok();
}

int polar_encode_launch(const tq_handle* h, const void* x, int x_dtype, int64_t n, uint8_t* codes, void* norms,
                        int32_t* len, int Hkv, int64_t L_cap, cudaStream_t s) {
  tqk::polar::EncodeArgs a{};
  a.x = x; a.x_dtype = x_dtype; a.rows = n; a.lay = h->play; a.norm_dtype = h->norm_dtype; a.PiT = h->dPiT;
  a.tab = h->dTab; a.codes = codes; a.codes_B = h->codes_B; a.norms = norms; a.len = len; a.Hkv = Hkv;
  a.L_cap = L_cap; a.err = h->derr;
  const size_t smem = tqk::polar::encode_smem_bytes(h->d);
  if (once_per_device(14, h->device))
    cudaFuncSetAttribute(tqk::polar::polar_encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  KernelScope ks(len ? "append" : "encode", s);
  tqk::polar::polar_encode_kernel<<<(unsigned)((n + tqk::polar::kBM - 1) / tqk::polar::kBM), tqk::polar::kThreads,
                                    smem, s>>>(a);
  return launch_check("polar_encode_kernel");
}

template <int D>
int polar_score_launch_d(const tq_handle* h, const tqk::polar::ScoreArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t bit = 1ull << (h->device & 63);
  if ((attr_done.fetch_or(bit) & bit) == 0)
    cudaFuncSetAttribute(tqk::polar::polar_score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  KernelScope ks("score", s);
  tqk::polar::polar_score_kernel<D><<<grid, tqk::polar::kSThreads, smem, s>>>(a);
  return launch_check("polar_score_kernel");
}

// QJL-only handles (prod with no MSE bits) store signs and the norm only: no codes, no rnorms.
bool qjl_only(const tq_handle* h) { return h->m > 0 && h->bits == 0; }

tqk::CacheView view_of(const tq_handle* h, const tq_cache* c) {
  tqk::CacheView v;
  v.codes = c->codes;
  v.signs = c->signs;
  v.norms = c->norms;
  v.rnorms = qjl_only(h) ? nullptr : static_cast<const __half*>(c->rnorms);
  v.bits = h->bits;
  v.m = h->m;
  v.norm_dtype = h->norm_dtype;
  v.codes_B = h->codes_B;
  v.signs_B = h->signs_B;
  v.cent = h->dcent;
  return v;
}

int check_cache(const tq_handle* h, const tq_cache* c, const char* name) {
  if (!c) return fail(TQ_EINVAL, "%s cache is NULL", name);
  if ((!c->codes && h->codes_B > 0) || !c->norms) return fail(TQ_EINVAL, "%s cache: codes/norms NULL", name);
  if (h->m > 0 && !c->signs) return fail(TQ_EINVAL, "%s cache: prod handle needs signs", name);
  if (h->m > 0 && !qjl_only(h) && !c->rnorms) return fail(TQ_EINVAL, "%s cache: prod handle needs rnorms", name);
  if (c->L_cap < 1) return fail(TQ_EINVAL, "%s cache: L_cap=%lld", name, (long long)c->L_cap);
  if ((c->codes && !aligned(c->codes, 16)) || (c->signs && !aligned(c->signs, 16)) || !aligned(c->norms, 4) ||
      (c->rnorms && !aligned(c->rnorms, 2)))
    return fail(TQ_EINVAL, "%s cache: misaligned pointer", name);
  return TQ_OK;
}

// TQ_SPLITK=<n> (tests and tuning): forces the context chunk of the split kernels to n
// tokens (attention, scores) or vectors (search), rounded up to the kernel's block and
// clamped to its limits; 0 or unset keeps the built-in policy. The workspace size
// functions see the same value, so set it before sizing a workspace.
int64_t splitk_override() {
  const char* e = std::getenv("TQ_SPLITK");
  if (!e || !*e) return 0;
  const long long v = std::atoll(e);
  return v > 0 ? (int64_t)v : 0;
}

int64_t round_chunk(int64_t v, int64_t blk, int64_t lo, int64_t hi) {
  v = (v + blk - 1) / blk * blk;
  return std::min<int64_t>(hi, std::max<int64_t>(lo, v));
}

// Attention split policy (shared by every attention kernel): about two CTAs per
// SM, chunks a multiple of 128 tokens and at most 896 tokens long (the 3-bit kernel
// stages a whole chunk of keys and values in shared memory).
void attn_split(int B, int Hkv, int64_t L_cap, int* nsplit, int64_t* chunk) {
  const int64_t units = std::max<int64_t>(1, (int64_t)B * Hkv);
  const int64_t ns = std::max<int64_t>(1, (2 * 148 + units - 1) / units);
  int64_t ch = (L_cap + ns - 1) / ns;
  ch = std::min<int64_t>(tqk::amma::kMaxChunk, std::max<int64_t>(128, (ch + 127) / 128 * 128));
  if (const int64_t f = splitk_override()) ch = round_chunk(f, 128, 128, tqk::amma::kMaxChunk);
  *chunk = ch;
  *nsplit = (int)((L_cap + ch - 1) / ch);
}

// Split of the tcgen05 3-bit attention (one persistent CTA per SM): about one item
// (sequence, KV head, chunk) per SM when the batch has fewer KV heads than SMs, chunks a
// multiple of 128 tokens and at most 2048 tokens long (the logits of a chunk stay in
// shared memory).
void attn_tc_split(int B, int Hkv, int64_t L_cap, int sms, int* nsplit, int64_t* chunk) {
  constexpr int64_t kMax = tqk::atc::kMaxChunk;
  const int64_t units = std::max<int64_t>(1, (int64_t)B * Hkv);
  const int64_t per = std::max<int64_t>(1, sms / units);
  const int64_t ns = std::max<int64_t>(per, (L_cap + kMax - 1) / kMax);
  int64_t ch = (L_cap + ns - 1) / ns;
  ch = std::min<int64_t>(kMax, std::max<int64_t>(128, (ch + 127) / 128 * 128));
  if (const int64_t f = splitk_override()) ch = round_chunk(f, 128, 128, kMax);
  *chunk = ch;
  *nsplit = (int)((L_cap + ch - 1) / ch);
}

// The two-kernel 3-bit attention (score kernel, then value kernel) for caches much larger than
// L2: prod 2+1 handles of the fast path's format, at least 256 MB of packed K and V
// (TQ_ATTN_2K=1 forces it for any such shape, TQ_ATTN_2K=0 disables it). It needs a scores
// buffer in the workspace, so it runs only when the caller's workspace holds one.
bool attn_2k_wanted(const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv, int64_t L_cap) {
  auto fmt = [](const tq_handle* h) {
    return h->d == 128 && h->m == 128 && h->bits == 2 && h->norm_dtype == TQ_F16 &&
           std::fabs(h->cent[3] - h->cent[2] - h->cent[1] + h->cent[0]) < 1e-12;
  };
  if (Hkv < 1 || Hq != 4 * Hkv || !fmt(hk) || !fmt(hv)) return false;
  const char* e = std::getenv("TQ_ATTN_2K");
  if (e && *e) return *e != '0';
  return (double)B * Hkv * (double)L_cap * 104.0 >= 256e6;
}

// Split of its value kernel (three CTAs per SM): about four waves, chunks whole 256-token blocks.
void attn_2k_split(int B, int Hkv, int64_t L_cap, int sms, int* nsplit, int64_t* chunk) {
  const int64_t units = std::max<int64_t>(1, (int64_t)B * Hkv);
  const int64_t ns = std::max<int64_t>(1, (4 * 3 * (int64_t)sms + units - 1) / units);
  int64_t ch = (L_cap + ns - 1) / ns;
  ch = std::max<int64_t>(256, (ch + 255) / 256 * 256);
  if (const int64_t f = splitk_override()) ch = round_chunk(f, 256, 256, (L_cap + 255) / 256 * 256);
  *chunk = ch;
  *nsplit = (int)((L_cap + ch - 1) / ch);
}

void search_split(int nq, int64_t n, int* nchunks, int64_t* chunk) {
  const int64_t qt = (nq + tqk::kSQ - 1) / tqk::kSQ;
  int64_t nc = (2 * 148 + qt - 1) / qt;
  nc = std::max<int64_t>(1, std::min<int64_t>(nc, (n + tqk::kSK - 1) / tqk::kSK));
  int64_t ch = (n + nc - 1) / nc;
  ch = (ch + tqk::kSK - 1) / tqk::kSK * tqk::kSK;
  if (const int64_t f = splitk_override()) ch = round_chunk(f, tqk::kSK, tqk::kSK, (n + tqk::kSK - 1) / tqk::kSK * tqk::kSK);
  *chunk = ch;
  *nchunks = (int)((n + ch - 1) / ch);
}

int sm_count(int device) {
  static std::atomic<int> counts[64];
  if (device < 0 || device >= 64) return 148;
  int c = counts[device].load();
  if (c == 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || c <= 0) c = 148;
    counts[device].store(c);
  }
  return c;
}

// Split of the tcgen05 search (one CTA per SM, 128 queries per CTA): chunks x query tiles is
// the smallest whole number of waves, chunks a multiple of 256 vectors.
void search_tc_split(int nq, int64_t n, int sms, int* nchunks, int64_t* chunk) {
  const int64_t vb = tqk::stc::kV;
  const int64_t qt = (nq + tqk::stc::kQ - 1) / tqk::stc::kQ;
  int64_t a = sms, bq = qt;
  while (bq) { const int64_t r = a % bq; a = bq; bq = r; }
  int64_t nc = sms / a;
  nc = std::max<int64_t>(1, std::min<int64_t>(nc, (n + vb - 1) / vb));
  int64_t ch = (n + nc - 1) / nc;
  ch = (ch + vb - 1) / vb * vb;
  if (const int64_t f = splitk_override()) ch = round_chunk(f, vb, vb, (n + vb - 1) / vb * vb);
  *chunk = ch;
  *nchunks = (int)((n + ch - 1) / ch);
}

// The tcgen05 search covers MSE codes of 1 to 4 bits with d a multiple of 64 (at least 128) and
// k <= 32; TQ_SIMT=1 forces the SIMT kernel.
bool search_tc_ok(const tq_handle* h, int64_t n, int k) {
  if (std::getenv("TQ_SIMT")) return false;
  return h->bits >= 1 && h->bits <= tqk::stc::kMaxBits && h->d % 64 == 0 && h->d >= tqk::stc::kKC &&
         k <= tqk::stc::kMaxK && n < ((int64_t)1 << 31);
}

// Centroids as 15-bit integers against one step, split into int8 pieces C = 128 C_h + C_l
// (C_l in [-64, 63]); the pieces go to the kernel as little-endian byte tables.
void centroid_pieces(const std::vector<double>& c, float* step_c, uint32_t th[4], uint32_t tl[4]) {
  double cmax = 0.0;
  for (double v : c) cmax = std::max(cmax, std::fabs(v));
  const double step = cmax > 0.0 ? cmax / tqk::stc::kCMax : 1.0;
  for (int w = 0; w < 4; ++w) th[w] = tl[w] = 0u;
  for (size_t i = 0; i < c.size() && i < 16; ++i) {
    long x = std::lround(c[i] / step);
    x = std::max<long>(-tqk::stc::kCMax, std::min<long>(tqk::stc::kCMax, x));
    const long hi = (long)std::floor((x + 64) / 128.0), lo = x - 128 * hi;
    th[i / 4] |= (uint32_t)(uint8_t)(int8_t)hi << (8 * (i % 4));
    tl[i / 4] |= (uint32_t)(uint8_t)(int8_t)lo << (8 * (i % 4));
  }
  *step_c = (float)step;
}

// The int8 tensor-core attention kernel covers 3-bit prod K and V caches (2-bit
// codes + 128 QJL signs, fp16 norms) at d = 128 with 4 query heads per KV head.
// TQ_SIMT=1 forces the SIMT kernels (used by tests to cross-check both paths).
bool attn_prod2_fast_path(const tq_handle* hk, const tq_handle* hv, int G, const tq_cache* k, const tq_cache* v) {
  if (std::getenv("TQ_SIMT")) return false;
  auto ok_handle = [](const tq_handle* h) {
    return h->d == 128 && h->m == 128 && h->bits == 2 && h->norm_dtype == TQ_F16 &&
           std::fabs(h->cent[3] - h->cent[2] - h->cent[1] + h->cent[0]) < 1e-12;
  };
  auto ok_cache = [](const tq_cache* c) {
    return aligned(c->codes, 16) && aligned(c->signs, 16) && aligned(c->norms, 16) && aligned(c->rnorms, 16);
  };
  return G == 4 && ok_handle(hk) && ok_handle(hv) && k->L_cap % 8 == 0 && ok_cache(k) && ok_cache(v);
}

// tq_score on the int8 tensor cores: the same key formats as the attention fast path.
bool score_prod2_fast_path(const tq_handle* hk, int G, const tq_cache* k) {
  if (std::getenv("TQ_SIMT")) return false;
  const bool fmt = hk->d == 128 && hk->m == 128 && hk->bits == 2 && hk->norm_dtype == TQ_F16 &&
                   std::fabs(hk->cent[3] - hk->cent[2] - hk->cent[1] + hk->cent[0]) < 1e-12;
  return G == 4 && fmt && k->L_cap % 8 == 0 && aligned(k->codes, 16) && aligned(k->signs, 16) &&
         aligned(k->norms, 16) && aligned(k->rnorms, 16);
}

// Walsh-plane form of a symmetric 16-level codebook (the int8 tensor-core 4-bit
// attention): c[idx] = c[0] + sum_S w[S] beta_S(idx) over the planes {0}, {1}, {2}, {3},
// {0,1,2}, {0,1,3}, {0,2,3}, {1,2,3} (beta = bit, or parity of three bits). In the +-1
// variables s_i = 2 b_i - 1 the coefficients are a_T = mean_idx c[idx] prod_{i in T} s_i;
// w[S] = 2 a_S. False if an even-degree coefficient does not vanish (no symmetry).
bool plane_coeffs4(const std::vector<double>& c, float* c0, float* w) {
  if (c.size() != 16) return false;
  static const int kMasks[8] = {1, 2, 4, 8, 7, 11, 13, 14};
  double cmax = 0.0;
  for (double v : c) cmax = std::max(cmax, std::fabs(v));
  double a[16];
  for (int T = 0; T < 16; ++T) {
    double acc = 0.0;
    for (int idx = 0; idx < 16; ++idx) {
      double prod = 1.0;
      for (int i = 0; i < 4; ++i)
        if (T >> i & 1) prod *= ((idx >> i) & 1) ? 1.0 : -1.0;
      acc += c[idx] * prod;
    }
    a[T] = acc / 16.0;
    if (__builtin_popcount(T) % 2 == 0 && std::fabs(a[T]) > 1e-12 * cmax) return false;
  }
  for (int p = 0; p < 8; ++p) w[p] = (float)(2.0 * a[kMasks[p]]);
  *c0 = (float)c[0];
  return true;
}

// The int8 tensor-core kernel for 4-bit MSE K and V caches (fp16 norms) at d = 128 with
// 4 query heads per KV head.
bool attn_mse4_fast_path(const tq_handle* hk, const tq_handle* hv, int G, const tq_cache* k, const tq_cache* v) {
  if (std::getenv("TQ_SIMT")) return false;
  float c0, w[8];
  auto ok_handle = [&](const tq_handle* h) {
    return h->d == 128 && h->m == 0 && h->bits == 4 && h->norm_dtype == TQ_F16 && plane_coeffs4(h->cent, &c0, w);
  };
  auto ok_cache = [](const tq_cache* c) { return aligned(c->codes, 16) && aligned(c->norms, 16); };
  return G == 4 && ok_handle(hk) && ok_handle(hv) && k->L_cap % 8 == 0 && ok_cache(k) && ok_cache(v);
}

struct ScoreWs { float* qr; float* qs; };
size_t score_ws_layout(const tq_handle* h, int rows, char* base, ScoreWs* w) {
  size_t off = 0;
  const size_t qr = round_up((size_t)rows * h->d * 4, 256);
  const size_t qs = round_up((size_t)rows * std::max(h->m, 1) * 4, 256);
  if (w) { w->qr = reinterpret_cast<float*>(base + off); w->qs = reinterpret_cast<float*>(base + off + qr); }
  off += qr + qs;
  return off;
}

// with_2k: room for the two-kernel attention too (its partials and the [B*Hq][L_cap] scores).
size_t attn_ws_layout(const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv, int64_t L_cap,
                      char* base, ScoreWs* w, float** part, int* nsplit, int64_t* chunk, bool with_2k = false,
                      float** logits = nullptr) {
  size_t off = score_ws_layout(hk, B * Hq, base, w);
  int ns, ns_tc;
  int64_t ch, ch_tc;
  attn_split(B, Hkv, L_cap, &ns, &ch);
  if (nsplit) *nsplit = ns;
  if (chunk) *chunk = ch;
  if (part) *part = reinterpret_cast<float*>(base + off);
  // room for the partials of every split (the tcgen05 3-bit kernel and the two-kernel form have their own)
  attn_tc_split(B, Hkv, L_cap, sm_count(hk->device), &ns_tc, &ch_tc);
  int ns_max = std::max(ns, ns_tc);
  if (with_2k) {
    int ns_2k;
    int64_t ch_2k;
    attn_2k_split(B, Hkv, L_cap, sm_count(hk->device), &ns_2k, &ch_2k);
    ns_max = std::max(ns_max, ns_2k);
  }
  off += round_up((size_t)B * Hq * ns_max * tqk::partial_stride(hv->d, hv->m) * 4, 256);
  if (with_2k) {
    if (logits) *logits = reinterpret_cast<float*>(base + off);
    off += round_up((size_t)B * Hq * (size_t)L_cap * 4, 256);
  }
  return off;
}

// mma: 0 for the SIMT kernel, else the queries per CTA of the tensor-core kernel.
// The bound pass of the tcgen05 search: the first kSearchSample vectors are searched first, and
// their exact k-th best score per query (a lower bound of the whole database's) seeds the score
// bound of the full pass, which then sets aside far fewer candidates. Only for n >= 4 samples.
constexpr int64_t kSearchSample = 32768;
struct SampleWs {
  int nchunks = 0;
  int64_t chunk = 0;
  float* cs = nullptr;     // [nchunks][halves][nq][k]
  int64_t* ci = nullptr;
  float* ts = nullptr;     // [nq][k]: the sample's top-k
  int64_t* ti = nullptr;
};

// tc: the tcgen05 search, which also takes the int8 query pieces [2][nq_pad][d], their scales
// [nq_pad], the per-query score bounds [nq_pad] and the bound pass's arrays (pieces / qscale /
// gbound / sample, else unused); otherwise the SIMT search.
size_t search_ws_layout(const tq_handle* h, int nq, int64_t n, int k, char* base, float** qr, float** cs,
                        int64_t** ci, int* nchunks, int64_t* chunk, bool tc, int8_t** pieces = nullptr,
                        float** qscale = nullptr, int** gbound = nullptr, SampleWs* sample = nullptr) {
  int nc;
  int64_t ch;
  if (tc)
    search_tc_split(nq, n, sm_count(h->device), &nc, &ch);
  else
    search_split(nq, n, &nc, &ch);
  if (nchunks) *nchunks = nc;
  if (chunk) *chunk = ch;
  if (tc) nc *= tqk::stc::kHalves;   // one candidate list per chunk and column half
  size_t off = 0;
  if (qr) *qr = reinterpret_cast<float*>(base + off);
  off += round_up((size_t)nq * h->d * 4, 256);
  if (tc) {
    const size_t nq_pad = (size_t)(nq + tqk::stc::kQ - 1) / tqk::stc::kQ * tqk::stc::kQ;
    if (pieces) *pieces = reinterpret_cast<int8_t*>(base + off);
    off += round_up(2 * nq_pad * h->d, 256);
    if (qscale) *qscale = reinterpret_cast<float*>(base + off);
    off += round_up(nq_pad * 4, 256);
    if (gbound) *gbound = reinterpret_cast<int*>(base + off);
    off += round_up(nq_pad * 4, 256);
    if (n >= 4 * kSearchSample) {
      SampleWs sw;
      search_tc_split(nq, kSearchSample, sm_count(h->device), &sw.nchunks, &sw.chunk);
      const size_t lists = (size_t)sw.nchunks * tqk::stc::kHalves * nq * k;
      sw.cs = reinterpret_cast<float*>(base + off);
      off += round_up(lists * 4, 256);
      sw.ci = reinterpret_cast<int64_t*>(base + off);
      off += round_up(lists * 8, 256);
      sw.ts = reinterpret_cast<float*>(base + off);
      off += round_up((size_t)nq * k * 4, 256);
      sw.ti = reinterpret_cast<int64_t*>(base + off);
      off += round_up((size_t)nq * k * 8, 256);
      if (sample) *sample = sw;
    }
  }
  if (cs) *cs = reinterpret_cast<float*>(base + off);
  off += round_up((size_t)nc * nq * k * 4, 256);
  if (ci) *ci = reinterpret_cast<int64_t*>(base + off);
  off += round_up((size_t)nc * nq * k * 8, 256);
  return off;
}

int launch_qprep(const tq_handle* h, const void* q, int q_dtype, int rows, float* qr, float* qs, cudaStream_t s) {
  if (rows == 0) return TQ_OK;
  // large fp32 batches (the search's queries): the tiled kernel
  if (rows >= 256 && q_dtype == TQ_F32 && aligned(q, 16) && h->d % tqk::kRotBK == 0 && h->d % 4 == 0 &&
      h->m % 4 == 0) {
    KernelScope ks("qprep", s);
    const float* X = static_cast<const float*>(q);
    const dim3 gr((unsigned)((h->d + tqk::kRotBN - 1) / tqk::kRotBN), (unsigned)((rows + tqk::kRotBM - 1) / tqk::kRotBM));
    tqk::rotate_tiled_kernel<<<gr, 256, 0, s>>>(X, rows, h->d, h->dPiT, h->d, qr);
    if (qs && h->m > 0) {
      const dim3 gs((unsigned)((h->m + tqk::kRotBN - 1) / tqk::kRotBN), gr.y);
      tqk::rotate_tiled_kernel<<<gs, 256, 0, s>>>(X, rows, h->d, h->dST, h->m, qs);
    }
    return launch_check("rotate_tiled_kernel");
  }
  if (h->d <= tqk::kWideMaxD && h->m <= tqk::kWideMaxD) {
    if (once_per_device(6, h->device))
      cudaFuncSetAttribute(tqk::qprep_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    const int rpc = rows >= 512 ? tqk::kQRowsBig : tqk::kQRows;   // query rows per CTA
    dim3 grid((unsigned)((rows + rpc - 1) / rpc), (unsigned)((h->d + h->m) / tqk::kWideCols));
    KernelScope ks("qprep", s);
    tqk::qprep_wide_kernel<<<grid, tqk::kSmallThreads, tqk::qprep_wide_smem_bytes(h->d, rpc), s>>>(
        q, q_dtype, rows, h->d, h->dPiT, h->dST, h->m, qr, qs, rpc);
    return launch_check("qprep_wide_kernel");
  }
  const int groups = (rows + tqk::kQprepRows - 1) / tqk::kQprepRows;
  dim3 grid(groups, (h->d + h->m + 63) / 64);
  if (once_per_device(5, h->device))
    cudaFuncSetAttribute(tqk::qprep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  KernelScope ks("qprep", s);
  tqk::qprep_kernel<<<grid, 256, (size_t)tqk::kQprepRows * h->d * sizeof(float), s>>>(q, q_dtype, rows, h->d, h->dPi, h->dS, h->m, qr, qs);
  return launch_check("qprep_kernel");
}

// Small batches (and every append) go to the latency-oriented kernel: one CTA per
// <= 16 rows (or per sequence), every thread one output coordinate.
bool rows_kernel_ok(const tq_handle* h, int64_t rows_per_cta) {
  return h->d <= tqk::kRowsMaxD && rows_per_cta <= tqk::kRowsMax;
}

int encode_rows_launch(const tq_handle* h, tqk::EncodeArgs& a, unsigned grid, int advance, cudaStream_t s) {
  const size_t smem = tqk::encode_rows_smem_bytes(h->d, h->m);
  if (once_per_device(4, h->device))
    cudaFuncSetAttribute(tqk::encode_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  KernelScope ks(a.len ? "append" : "encode", s);
  tqk::encode_rows_kernel<<<grid, tqk::kRowsThreads, smem, s>>>(a, advance);
  return launch_check("encode_rows_kernel");
}

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel of the stream finishes, and waits (griddepcontrol.wait) before reading its outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- tensor-core encode (d = 128, bf16 / f16 input)

PFN_cuTensorMapEncodeTiled tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  });
  return fn;
}

// Code rows as a 2-D byte tensor {row_bytes, rows} for tile loads of box_rows rows and
// box_bytes (128) bytes with the 128-byte swizzle; bytes and rows past the tensor load as zeros.
int codes_map_2d(const uint8_t* codes, int64_t rows, int row_bytes, int box_bytes, int box_rows, CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return TQ_OK;
}

bool tc_encode_ok(const tq_handle* h, const tqk::EncodeArgs& a) {
  if (std::getenv("TQ_SIMT")) return false;
  return h->dOps && h->bits > 0 && a.len == nullptr && (a.x_dtype == TQ_BF16 || a.x_dtype == TQ_F16) && a.rows >= 1024 &&
         a.rows < (int64_t)1 << 31;
}

template <int BITS, bool PROD, bool NORM32>
int tc_launch_one(const tq_handle* h, const CUtensorMap& map, const tqk::etc::Args& ea, int f16in, unsigned grid,
                  cudaStream_t s) {
  auto kern = tqk::etc::encode_tc_kernel<BITS, PROD, NORM32>;
  const size_t smem = tqk::etc::Layout<PROD>::kBytes;
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t bit = 1ull << (h->device & 63);
  if ((attr_done.fetch_or(bit) & bit) == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(encode_tc_kernel)");
  }
  KernelScope ks("encode", s);
  kern<<<grid, tqk::etc::Layout<PROD>::kThreads, smem, s>>>(map, ea, f16in);
  return launch_check("encode_tc_kernel");
}

template <bool PROD, bool NORM32>
int tc_launch_bits(const tq_handle* h, const CUtensorMap& map, const tqk::etc::Args& ea, int f16in, unsigned grid,
                   cudaStream_t s) {
  switch (h->bits) {
    case 1: return tc_launch_one<1, PROD, NORM32>(h, map, ea, f16in, grid, s);
    case 2: return tc_launch_one<2, PROD, NORM32>(h, map, ea, f16in, grid, s);
    case 3: return tc_launch_one<3, PROD, NORM32>(h, map, ea, f16in, grid, s);
    default: return tc_launch_one<4, PROD, NORM32>(h, map, ea, f16in, grid, s);
  }
}

int encode_tc_launch(const tq_handle* h, const tqk::EncodeArgs& a, cudaStream_t s) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)h->d, (cuuint64_t)a.rows};
  const cuuint64_t strides[1] = {(cuuint64_t)h->d * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, a.x_dtype == TQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(a.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  tqk::etc::Args ea{};
  ea.rows = a.rows; ea.norm_dtype = a.norm_dtype; ea.ops = h->dOps; ea.cent = a.cent; ea.bnd = a.bnd;
  ea.codes = a.codes; ea.codes_B = a.codes_B; ea.signs = a.signs; ea.signs_B = a.signs_B;
  ea.norms = a.norms; ea.rnorms = a.rnorms; ea.err = a.err;
  const int64_t tiles = (a.rows + tqk::etc::kTile - 1) / tqk::etc::kTile;
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, sm_count(h->device));
  const int f16 = a.x_dtype == TQ_F16 ? 1 : 0;
  const bool n32 = a.norm_dtype == TQ_F32;
  if (h->m > 0)
    return n32 ? tc_launch_bits<true, true>(h, map, ea, f16, grid, s) : tc_launch_bits<true, false>(h, map, ea, f16, grid, s);
  return n32 ? tc_launch_bits<false, true>(h, map, ea, f16, grid, s) : tc_launch_bits<false, false>(h, map, ea, f16, grid, s);
}

// The tensor-core encode of large vectors: MSE handles with d % 256 == 0 (256 .. 4096), at least
// 256 rows, not an append.
bool big_tc_ok(const tq_handle* h, const tqk::EncodeArgs& a) {
  return !std::getenv("TQ_SIMT") && h->dPiB && a.len == nullptr && a.rows >= 256 && a.rows < ((int64_t)1 << 31);
}

int encode_big_tc_launch(const tq_handle* h, const tqk::EncodeArgs& a, cudaStream_t s) {
  PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int d = h->d;
  CUtensorMap pmap;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)2 * d};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {(cuuint32_t)tqk::ebig::kKC, (cuuint32_t)tqk::ebig::kN};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(&pmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->dPiB, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  tqk::ebig::Args ea{};
  ea.x = a.x; ea.x_dtype = a.x_dtype; ea.rows = a.rows; ea.d = d; ea.bits = h->bits; ea.norm_dtype = a.norm_dtype;
  ea.codes_B = h->codes_B; ea.bnd = h->dbnd; ea.codes = a.codes; ea.norms = a.norms; ea.err = h->derr;
  auto kern = a.x_dtype == TQ_F32 ? tqk::ebig::encode_big_tc_kernel<TQ_F32>
            : a.x_dtype == TQ_BF16 ? tqk::ebig::encode_big_tc_kernel<TQ_BF16>
                                   : tqk::ebig::encode_big_tc_kernel<TQ_F16>;
  if (once_per_device(25 + a.x_dtype, h->device))
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tqk::ebig::kSmemBytes);
  const int64_t ntiles = (a.rows + tqk::ebig::kM - 1) / tqk::ebig::kM;
  const unsigned grid = (unsigned)std::min<int64_t>(ntiles, sm_count(h->device));
  KernelScope ks("encode", s);
  kern<<<grid, tqk::ebig::kThreads, tqk::ebig::kSmemBytes, s>>>(pmap, ea);
  return launch_check("encode_big_tc_kernel");
}

int encode_launch(const tq_handle* h, tqk::EncodeArgs& a, cudaStream_t s) {
  if (tc_encode_ok(h, a)) return encode_tc_launch(h, a, s);
  if (big_tc_ok(h, a)) return encode_big_tc_launch(h, a, s);
  if (a.len == nullptr && a.rows <= 256 && rows_kernel_ok(h, 1))
    return encode_rows_launch(h, a, (unsigned)((a.rows + tqk::kRowsMax - 1) / tqk::kRowsMax), 0, s);
  const size_t smem = tqk::encode_smem_bytes(h->m);
  if (once_per_device(0, h->device))
    cudaFuncSetAttribute(tqk::encode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  dim3 grid((unsigned)((a.rows + tqk::kEncBM - 1) / tqk::kEncBM), (h->d + tqk::kEncBN - 1) / tqk::kEncBN);
  KernelScope ks(a.len ? "append" : "encode", s);
  tqk::encode_simt_kernel<<<grid, tqk::kEncThreads, smem, s>>>(a);
  return launch_check("encode_simt_kernel");
}

}  // namespace

// Error reporting for the library's other translation units.
int tq_internal_fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

namespace tqk {
// TQ_CHECK=1: every len[b] must lie in 0 .. L_cap.
__global__ void check_lens_kernel(const int32_t* len, int B, int64_t L_cap, int* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && (len[b] < 0 || (int64_t)len[b] > L_cap)) report_error(err, kErrBounds);
}

// TQ_FAULT=timeout: the error a timed-out wait records, without any wait.
__global__ void inject_error_kernel(int* err, int bit) {
  if (threadIdx.x == 0) report_error(err, bit);
}

// The failure path of every bounded wait, on its own: thread 0 waits for phase 0 of a
// barrier that expects one arrival and never gets it, gives up after `limit` polls and
// records kErrTimeout, as a kernel does when a copy or a release never completes.
__global__ void selftest_wait_kernel(int* err, int limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    bar_init(&bar, 1);
    if (!bar_wait(&bar, 0, limit)) report_error(err, kErrTimeout);
  }
}
}  // namespace tqk

namespace {
// TQ_CHECK and TQ_FAULT=timeout work that precedes a hot call's kernels (len may be NULL).
int pre_launch(const tq_handle* h, const int32_t* len, int B, int64_t L_cap, cudaStream_t s) {
  if (len && B > 0 && check_mode()) {
    tqk::check_lens_kernel<<<(B + 255) / 256, 256, 0, s>>>(len, B, L_cap, h->derr);
    if (int st = launch_check("check_lens_kernel")) return st;
  }
  if (fault_is("timeout")) {
    tqk::inject_error_kernel<<<1, 32, 0, s>>>(h->derr, tqk::kErrTimeout);
    return launch_check("inject_error_kernel");
  }
  return TQ_OK;
}

}  // namespace

// ============================================================================
extern "C" {

int tq_codebook_host(int d, int bits, double* centroids, double* bounds) {
  if (!centroids || !bounds) return fail(TQ_EINVAL, "NULL output");
  if (d < 3 || d > 65536 || bits < 1 || bits > 8) return fail(TQ_EINVAL, "d=%d bits=%d out of range", d, bits);
  if (tqhost::codebook(d, bits, centroids, bounds) != 0) return fail(TQ_EINVAL, "codebook failed");
  return ok();
}

int tq_rotation_host(int d, int m, uint64_t seed, double* Pi, double* S) {
  if (!Pi) return fail(TQ_EINVAL, "Pi is NULL");
  if (d < 1 || d > 8192 || m < 0 || m > 8192) return fail(TQ_EINVAL, "d=%d m=%d out of range", d, m);
  if (m > 0 && !S) return fail(TQ_EINVAL, "S is NULL with m > 0");
  tqhost::rotation(d, m, seed, Pi, S);
  return ok();
}

int tq_create(int d, int bits, uint64_t seed, tq_handle** out) {
  return create_common(d, bits, 0, seed, TQ_F32, out);
}

int tq_create_prod(int d, int bits, int qjl_m, uint64_t seed, tq_handle** out) {
  if (bits < 1 || bits > 5) return fail(TQ_EUNSUPPORTED, "prod bits=%d outside 1..5", bits);
  if (qjl_m < 32) return fail(TQ_EUNSUPPORTED, "qjl_m=%d < 32", qjl_m);
  return create_common(d, bits - 1, qjl_m, seed, TQ_F16, out);
}

int tq_create_polar(int d, int bits_level1, int bits_upper, uint64_t seed, tq_handle** out) {
  return create_polar(d, bits_level1, bits_upper, seed, out);
}

int tq_polar_info(const tq_handle* h, int* nlevels, int* bits_level1, int* bits_upper) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (!h->polar) return fail(TQ_EINVAL, "not a polar handle");
  if (nlevels) *nlevels = h->play.nlev;
  if (bits_level1) *bits_level1 = h->play.bits[0];
  if (bits_upper) *bits_upper = h->play.bits[1];
  return ok();
}

int tq_get_polar_codebook(const tq_handle* h, int level, double* centroids, double* bounds) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (!h->polar) return fail(TQ_EINVAL, "not a polar handle");
  if (level < 1 || level > h->play.nlev) return fail(TQ_EINVAL, "level %d outside 1..%d", level, h->play.nlev);
  if (centroids) std::memcpy(centroids, h->pcent[level - 1].data(), h->pcent[level - 1].size() * sizeof(double));
  if (bounds) std::memcpy(bounds, h->pbnd[level - 1].data(), h->pbnd[level - 1].size() * sizeof(double));
  return ok();
}

int tq_polar_codebook_host(int level, int bits, double* centroids, double* bounds) {
  if (!centroids || !bounds) return fail(TQ_EINVAL, "NULL output");
  if (level < 1 || level > 16 || bits < 1 || bits > 8) return fail(TQ_EINVAL, "level=%d bits=%d out of range", level, bits);
  if (tqhost::polar_codebook(level, bits, centroids, bounds) != 0) return fail(TQ_EINVAL, "polar codebook failed");
  return ok();
}

int tq_set_norm_dtype(tq_handle* h, int dtype) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (dtype != TQ_F32 && dtype != TQ_F16) return fail(TQ_EINVAL, "norm dtype %d (TQ_F32 or TQ_F16)", dtype);
  h->norm_dtype = dtype;
  return ok();
}

void tq_destroy(tq_handle* h) {
  if (!h) return;
  free_device(h);
  delete h;
}

int tq_get_info(const tq_handle* h, int* d, int* bits_mse, int* qjl_m, int* norm_dtype) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (d) *d = h->d;
  if (bits_mse) *bits_mse = h->bits;
  if (qjl_m) *qjl_m = h->m;
  if (norm_dtype) *norm_dtype = h->norm_dtype;
  return ok();
}

int tq_code_bytes(const tq_handle* h, int* codes_B, int* signs_B) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (codes_B) *codes_B = h->codes_B;
  if (signs_B) *signs_B = h->signs_B;
  return ok();
}

int tq_get_codebook(const tq_handle* h, double* centroids, double* bounds) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (h->polar) return fail(TQ_EINVAL, "polar handles have one codebook per level (tq_get_polar_codebook)");
  if (centroids) std::memcpy(centroids, h->cent.data(), h->cent.size() * sizeof(double));
  if (bounds) std::memcpy(bounds, h->bnd.data(), h->bnd.size() * sizeof(double));
  return ok();
}

int tq_get_rotation(const tq_handle* h, double* Pi, double* S) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (Pi) std::memcpy(Pi, h->Pi.data(), h->Pi.size() * sizeof(double));
  if (S && h->m > 0) std::memcpy(S, h->S.data(), h->S.size() * sizeof(double));
  return ok();
}

int tq_encode(const tq_handle* h, const void* x, int x_dtype, int64_t n, uint8_t* codes, uint8_t* signs,
              void* norms, void* rnorms, void* stream) {
  NvtxRange nvtx("tq_encode");
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (n < 0) return fail(TQ_EINVAL, "n=%lld", (long long)n);
  if (!valid_dtype(x_dtype)) return fail(TQ_EINVAL, "x dtype %d", x_dtype);
  if (n == 0) return ok();
  if (!x || (!codes && h->codes_B > 0) || !norms) return fail(TQ_EINVAL, "x/codes/norms NULL");
  if (h->m > 0 && (!signs || (!rnorms && !qjl_only(h)))) return fail(TQ_EINVAL, "prod handle needs signs and rnorms");
  if (qjl_only(h)) codes = nullptr, rnorms = nullptr;   // QJL-only rows: signs and the norm
  if (!aligned(x, 16) || (codes && !aligned(codes, 16)) || (signs && !aligned(signs, 16)) || !aligned(norms, 4))
    return fail(TQ_EINVAL, "misaligned pointer");
  if (fault_is("launch")) return fail(TQ_ECUDA, "injected launch failure (TQ_FAULT=launch)");
  if (int st = pre_launch(h, nullptr, 0, 0, static_cast<cudaStream_t>(stream))) return st;
  if (h->polar) return polar_encode_launch(h, x, x_dtype, n, codes, norms, nullptr, 0, 0, static_cast<cudaStream_t>(stream));
  tqk::EncodeArgs a{};
  a.x = x; a.x_dtype = x_dtype; a.rows = n; a.d = h->d; a.bits = h->bits; a.m = h->m;
  a.norm_dtype = h->norm_dtype; a.PiT = h->dPiT; a.MT = h->dMT; a.cent = h->dcent; a.bnd = h->dbnd;
  a.codes = codes; a.codes_B = h->codes_B; a.signs = signs; a.signs_B = h->signs_B;
  a.norms = norms; a.rnorms = static_cast<__half*>(rnorms); a.len = nullptr; a.err = h->derr;
  return encode_launch(h, a, static_cast<cudaStream_t>(stream));
}

int tq_pack_indices(const tq_handle* h, const uint8_t* idx, int64_t n, uint8_t* codes, void* stream) {
  NvtxRange nvtx("tq_pack_indices");
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (n < 0) return fail(TQ_EINVAL, "n=%lld", (long long)n);
  if (n == 0) return ok();
  if (h->bits == 0) return fail(TQ_EINVAL, "QJL-only and polar handles have no MSE codes to pack");
  if (!idx || !codes) return fail(TQ_EINVAL, "NULL pointer");
  if (!aligned(codes, 4)) return fail(TQ_EINVAL, "codes misaligned");
  const int64_t work = n * (h->d / 32);
  KernelScope ks("pack", static_cast<cudaStream_t>(stream));
  tqk::pack_indices_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      idx, n, h->d, h->bits, codes, h->codes_B);
  return launch_check("pack_indices_kernel");
}

int tq_append(const tq_handle* h, const void* x_new, int x_dtype, int B, int Hkv, const tq_cache* cache,
              int32_t* len, int advance, void* stream) {
  NvtxRange nvtx("tq_append");
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (B < 0 || Hkv < 1) return fail(TQ_EINVAL, "B=%d Hkv=%d", B, Hkv);
  if (!valid_dtype(x_dtype)) return fail(TQ_EINVAL, "x dtype %d", x_dtype);
  if (B == 0) return ok();
  int st = check_cache(h, cache, "append");
  if (st) return st;
  if (!x_new || !len) return fail(TQ_EINVAL, "x_new/len NULL");
  if (!aligned(x_new, 16)) return fail(TQ_EINVAL, "x_new misaligned");
  if (fault_is("launch")) return fail(TQ_ECUDA, "injected launch failure (TQ_FAULT=launch)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = pre_launch(h, len, B, cache->L_cap, s))) return st;
  if (h->polar) {
    if ((st = polar_encode_launch(h, x_new, x_dtype, (int64_t)B * Hkv, cache->codes, cache->norms, len, Hkv,
                                  cache->L_cap, s)))
      return st;
    if (!advance) return ok();
    KernelScope ks("advance_len", s);
    tqk::advance_len_kernel<<<(B + 255) / 256, 256, 0, s>>>(len, B, cache->L_cap);
    return launch_check("advance_len_kernel");
  }
  tqk::EncodeArgs a{};
  a.x = x_new; a.x_dtype = x_dtype; a.rows = (int64_t)B * Hkv; a.d = h->d; a.bits = h->bits; a.m = h->m;
  a.norm_dtype = h->norm_dtype; a.PiT = h->dPiT; a.MT = h->dMT; a.cent = h->dcent; a.bnd = h->dbnd;
  a.codes = cache->codes; a.codes_B = h->codes_B; a.signs = cache->signs; a.signs_B = h->signs_B;
  a.norms = cache->norms; a.rnorms = qjl_only(h) ? nullptr : static_cast<__half*>(cache->rnorms);
  a.len = len; a.Hkv = Hkv; a.L_cap = cache->L_cap; a.err = h->derr;
  if (qjl_only(h)) a.codes = nullptr;
  if (h->d <= tqk::kSmallMaxD && h->m <= tqk::kSmallMaxD && Hkv <= 8) {
    // one CTA per (sequence, head); the Hkv CTAs of a sequence form a cluster
    const size_t smem = tqk::append_cluster_smem_bytes(h->d, h->m);
    if (once_per_device(8, h->device))
      cudaFuncSetAttribute(tqk::append_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)Hkv, (unsigned)B, 1);
    cfg.blockDim = dim3(tqk::kSmallThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)Hkv;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int adv = advance ? 1 : 0;
    KernelScope ks("append", s);
    cudaError_t e = cudaLaunchKernelEx(&cfg, tqk::append_cluster_kernel, a, adv);
    if (e != cudaSuccess) return cuda_fail(e, "append_cluster_kernel");
    return launch_check("append_cluster_kernel");
  }
  if (rows_kernel_ok(h, Hkv)) return encode_rows_launch(h, a, (unsigned)B, advance ? 1 : 0, s);
  st = encode_launch(h, a, s);
  if (st) return st;
  if (advance) {
    KernelScope ks("advance_len", s);
    tqk::advance_len_kernel<<<(B + 255) / 256, 256, 0, s>>>(len, B, cache->L_cap);
    return launch_check("advance_len_kernel");
  }
  return ok();
}

size_t tq_score_workspace_bytes(const tq_handle* hk, int B, int Hq) {
  if (!hk || B < 0 || Hq < 0) return 0;
  return score_ws_layout(hk, B * Hq, nullptr, nullptr);
}

size_t tq_attn_workspace_bytes(const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv, int64_t L_cap) {
  if (!hk || !hv || B < 0 || Hq < 1 || Hkv < 1 || L_cap < 1) return 0;
  return attn_ws_layout(hk, hv, B, Hq, Hkv, L_cap, nullptr, nullptr, nullptr, nullptr, nullptr,
                        attn_2k_wanted(hk, hv, B, Hq, Hkv, L_cap));
}

size_t tq_internal_attn_workspace_min_bytes(const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv,
                                            int64_t L_cap) {
  if (!hk || !hv || B < 0 || Hq < 1 || Hkv < 1 || L_cap < 1) return 0;
  return attn_ws_layout(hk, hv, B, Hq, Hkv, L_cap, nullptr, nullptr, nullptr, nullptr, nullptr, false);
}

size_t tq_search_workspace_bytes(const tq_handle* h, int nq, int64_t n, int k) {
  if (!h || nq < 0 || n < 1 || k < 1) return 0;
  size_t b = 0;
  for (bool tc : {false, true})
    b = std::max(b, search_ws_layout(h, nq, n, k, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, tc));
  return b;
}

int tq_score(const tq_handle* hk, const float* q, int B, int Hq, int Hkv, const tq_cache* k, const int32_t* len,
             float* logits, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("tq_score");
  if (!hk) return fail(TQ_EINVAL, "handle is NULL");
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return fail(TQ_EINVAL, "B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  if (Hq / Hkv > tqk::kMaxGroup) return fail(TQ_EUNSUPPORTED, "group Hq/Hkv=%d > %d", Hq / Hkv, tqk::kMaxGroup);
  if (hk->d > tqk::kMaxHeadDim) return fail(TQ_EUNSUPPORTED, "score needs d <= %d", tqk::kMaxHeadDim);
  if (B == 0) return ok();
  int st = check_cache(hk, k, "key");
  if (st) return st;
  if (!q || !len || !logits || !workspace) return fail(TQ_EINVAL, "NULL pointer");
  const size_t need = tq_score_workspace_bytes(hk, B, Hq);
  if (ws_bytes < need) return fail(TQ_EINVAL, "workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(workspace, 16)) return fail(TQ_EINVAL, "workspace misaligned");
  if (fault_is("launch")) return fail(TQ_ECUDA, "injected launch failure (TQ_FAULT=launch)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = pre_launch(hk, len, B, k->L_cap, s))) return st;
  ScoreWs w;
  score_ws_layout(hk, B * Hq, static_cast<char*>(workspace), &w);
  st = launch_qprep(hk, q, TQ_F32, B * Hq, w.qr, w.qs, s);
  if (st) return st;
  const int64_t units = (int64_t)B * Hkv;
  if (hk->polar) {
    if (Hq / Hkv > tqk::polar::kMaxG) return fail(TQ_EUNSUPPORTED, "polar scores need Hq/Hkv <= %d", tqk::polar::kMaxG);
    tqk::polar::ScoreArgs pa{};
    pa.qr = w.qr; pa.B = B; pa.Hq = Hq; pa.Hkv = Hkv; pa.lay = hk->play; pa.codes = k->codes; pa.codes_B = hk->codes_B;
    pa.norms = k->norms; pa.norm_dtype = hk->norm_dtype; pa.tab = hk->dTab; pa.L_cap = k->L_cap; pa.len = len;
    pa.logits = logits;
    int64_t ns = std::max<int64_t>(1, std::min<int64_t>((8 * 148 + units - 1) / units, (k->L_cap + 127) / 128));
    pa.chunk = ((k->L_cap + ns - 1) / ns + 127) / 128 * 128;
    if (const int64_t f = splitk_override()) pa.chunk = round_chunk(f, 128, 128, (k->L_cap + 127) / 128 * 128);
    ns = (k->L_cap + pa.chunk - 1) / pa.chunk;
    const dim3 grid((unsigned)units, (unsigned)ns);
    const size_t smem = tqk::polar::score_smem_bytes(hk->d, hk->play.bits[0], Hq / Hkv, hk->codes_B);
    switch (hk->d) {
      case 32: return polar_score_launch_d<32>(hk, pa, grid, smem, s);
      case 64: return polar_score_launch_d<64>(hk, pa, grid, smem, s);
      case 128: return polar_score_launch_d<128>(hk, pa, grid, smem, s);
      default: return polar_score_launch_d<256>(hk, pa, grid, smem, s);
    }
  }
  if (score_prod2_fast_path(hk, Hq / Hkv, k)) {
    // about eight waves of 3 CTAs per SM; chunks are whole 256-key blocks
    const int64_t target = 8 * 3 * (int64_t)sm_count(hk->device);
    int64_t chunk = ((units * k->L_cap + target - 1) / target + 255) / 256 * 256;
    chunk = std::max<int64_t>(256, std::min<int64_t>(chunk, (k->L_cap + 255) / 256 * 256));
    if (const int64_t f = splitk_override()) chunk = round_chunk(f, 256, 256, (k->L_cap + 255) / 256 * 256);
    const int64_t nsp = (k->L_cap + chunk - 1) / chunk;
    tqk::amma::ScoreArgs m{};
    m.qr = w.qr; m.qs = w.qs; m.B = B; m.Hq = Hq; m.Hkv = Hkv;
    m.kcodes = k->codes; m.ksigns = k->signs; m.knorm = static_cast<const __half*>(k->norms);
    m.krn = static_cast<const __half*>(k->rnorms);
    m.L_cap = k->L_cap; m.chunk = chunk; m.len = len;
    m.kc0 = (float)hk->cent[0]; m.kb0 = (float)(hk->cent[1] - hk->cent[0]); m.kb1 = (float)(hk->cent[2] - hk->cent[0]);
    m.logits = logits; m.err = hk->derr;
    const size_t msmem = sizeof(tqk::amma::ScoreSmem);
    if (once_per_device(10, hk->device)) {
      cudaFuncSetAttribute(tqk::amma::score_prod2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
      cudaFuncSetAttribute(tqk::amma::score_prod2_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
    KernelScope ks("score", s);
    const cudaError_t e = launch_pdl(tqk::amma::score_prod2_kernel<false>, dim3((unsigned)units, (unsigned)nsp),
                                     dim3(tqk::amma::kThreads), msmem, s, m);
    if (e != cudaSuccess) return cuda_fail(e, "score_prod2_kernel");
    return launch_check("score_prod2_kernel");
  }
  tqk::ScoreArgs a{};
  a.qr = w.qr; a.qs = w.qs; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = hk->d; a.k = view_of(hk, k);
  a.L_cap = k->L_cap; a.len = len; a.logits = logits;
  int64_t ns = std::max<int64_t>(1, std::min<int64_t>((8 * 148 + units - 1) / units, (k->L_cap + 127) / 128));
  a.chunk = ((k->L_cap + ns - 1) / ns + 127) / 128 * 128;
  if (const int64_t f = splitk_override()) a.chunk = round_chunk(f, 128, 128, (k->L_cap + 127) / 128 * 128);
  ns = (k->L_cap + a.chunk - 1) / a.chunk;
  const int G = Hq / Hkv;
  const size_t smem = ((size_t)G * (hk->d + hk->m) + 16) * 4;
  KernelScope ks("score", s);
  tqk::score_simt_kernel<<<dim3((unsigned)units, (unsigned)ns), tqk::kAttnThreads, smem, s>>>(a);
  return launch_check("score_simt_kernel");
}

}  // extern "C"

namespace {

// Argument checks shared by tq_attn_decode and tq_decode_step (TQ_OK also for B == 0).
int attn_check(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
               const tq_cache* k, const tq_cache* v, const int32_t* len, float scale, float* out, void* workspace,
               size_t ws_bytes) {
  if (!hk || !hv) return fail(TQ_EINVAL, "handle is NULL");
  if (hk->polar || hv->polar) return fail(TQ_EUNSUPPORTED, "decode attention takes MSE, prod or QJL-only handles");
  if (hk->d != hv->d) return fail(TQ_EINVAL, "K and V handles differ in d (%d vs %d)", hk->d, hv->d);
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return fail(TQ_EINVAL, "B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  if (Hq / Hkv > tqk::kMaxGroup) return fail(TQ_EUNSUPPORTED, "group Hq/Hkv=%d > %d", Hq / Hkv, tqk::kMaxGroup);
  if (hk->d > tqk::kMaxHeadDim || hv->m > tqk::kMaxHeadDim || hv->d + hv->m > 256)
    return fail(TQ_EUNSUPPORTED, "attention needs d <= %d and d + m_V <= 256", tqk::kMaxHeadDim);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_EINVAL, "q dtype %d", q_dtype);
  if (B == 0) return ok();
  int st = check_cache(hk, k, "key");
  if (st) return st;
  if ((st = check_cache(hv, v, "value"))) return st;
  if (k->L_cap != v->L_cap) return fail(TQ_EINVAL, "K and V caches differ in L_cap");
  if (!q || !len || !out || !workspace) return fail(TQ_EINVAL, "NULL pointer");
  // the minimum (without the two-kernel attention's scores buffer, which is used when present)
  const size_t need = tq_internal_attn_workspace_min_bytes(hk, hv, B, Hq, Hkv, k->L_cap);
  if (ws_bytes < need) return fail(TQ_EINVAL, "workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned(workspace, 16)) return fail(TQ_EINVAL, "workspace misaligned");
  if (!std::isfinite(scale)) return fail(TQ_EINVAL, "scale is not finite");
  if (fault_is("launch")) return fail(TQ_ECUDA, "injected launch failure (TQ_FAULT=launch)");
  return ok();
}

// Query rotation (unless a decode-step prologue did it), split attention and combine.
// fused: the token appended at slot len[b] by the prologue counts, and the combine
// advances len[b] once everything that reads it is done.
int attn_impl(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
              const tq_cache* k, const tq_cache* v, int32_t* len, float scale, float* out, void* workspace,
              size_t ws_bytes, cudaStream_t s, bool fused) {
  ScoreWs w;
  float* part;
  int nsplit;
  int64_t chunk;
  attn_ws_layout(hk, hv, B, Hq, Hkv, k->L_cap, static_cast<char*>(workspace), &w, &part, &nsplit, &chunk);
  int st = TQ_OK;
  if (!fused && (st = launch_qprep(hk, q, q_dtype, B * Hq, w.qr, w.qs, s))) return st;
  tqk::AttnArgs a{};
  a.qr = w.qr; a.qs = w.qs; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = hk->d;
  a.k = view_of(hk, k); a.v = view_of(hv, v); a.L_cap = k->L_cap; a.chunk = chunk; a.nsplit = nsplit;
  a.len = len; a.len_extra = fused ? 1 : 0; a.scale = scale; a.part = part;
  const int G = Hq / Hkv;
  const char* tce0 = std::getenv("TQ_ATTN_TC");
  const bool tc0 = tce0 && *tce0 && *tce0 != '0';
  if (!tc0 && attn_prod2_fast_path(hk, hv, G, k, v) && attn_2k_wanted(hk, hv, B, Hq, Hkv, k->L_cap) &&
      ws_bytes >= attn_ws_layout(hk, hv, B, Hq, Hkv, k->L_cap, nullptr, nullptr, nullptr, nullptr, nullptr, true)) {
    // two kernels: every key's score (22-bit queries) into the workspace, then the value pass
    // (timed together as the split attention)
    float* logits = nullptr;
    attn_ws_layout(hk, hv, B, Hq, Hkv, k->L_cap, static_cast<char*>(workspace), nullptr, nullptr, nullptr, nullptr,
                   true, &logits);
    const int sms = sm_count(hk->device);
    const int64_t units = (int64_t)B * Hkv;
    const int64_t target = 8 * 3 * (int64_t)sms;   // scores: about eight waves of 3 CTAs per SM
    int64_t sch = ((units * k->L_cap + target - 1) / target + 255) / 256 * 256;
    sch = std::max<int64_t>(256, std::min<int64_t>(sch, (k->L_cap + 255) / 256 * 256));
    const int64_t nsp = (k->L_cap + sch - 1) / sch;
    tqk::amma::ScoreArgs ms{};
    ms.qr = w.qr; ms.qs = w.qs; ms.B = B; ms.Hq = Hq; ms.Hkv = Hkv;
    ms.kcodes = k->codes; ms.ksigns = k->signs; ms.knorm = static_cast<const __half*>(k->norms);
    ms.krn = static_cast<const __half*>(k->rnorms);
    ms.L_cap = k->L_cap; ms.chunk = sch; ms.len = len; ms.len_extra = fused ? 1 : 0;
    ms.kc0 = (float)hk->cent[0]; ms.kb0 = (float)(hk->cent[1] - hk->cent[0]); ms.kb1 = (float)(hk->cent[2] - hk->cent[0]);
    ms.logits = logits; ms.err = hk->derr;
    int64_t vch;
    attn_2k_split(B, Hkv, k->L_cap, sms, &nsplit, &vch);
    tqk::amma::VArgs mv{};
    mv.logits = logits; mv.B = B; mv.Hq = Hq; mv.Hkv = Hkv;
    mv.vcodes = v->codes; mv.vsigns = v->signs; mv.vnorm = static_cast<const __half*>(v->norms);
    mv.vrn = static_cast<const __half*>(v->rnorms);
    mv.L_cap = k->L_cap; mv.chunk = vch; mv.nsplit = nsplit; mv.len = len; mv.len_extra = fused ? 1 : 0;
    mv.vc0 = (float)hv->cent[0]; mv.vb0 = (float)(hv->cent[1] - hv->cent[0]); mv.vb1 = (float)(hv->cent[2] - hv->cent[0]);
    mv.scale = scale; mv.part = part; mv.err = hk->derr;
    const size_t ssmem = sizeof(tqk::amma::ScoreSmem), vsmem = sizeof(tqk::amma::VSmem);
    if (once_per_device(13, hk->device)) {
      cudaFuncSetAttribute(tqk::amma::score_prod2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
      cudaFuncSetAttribute(tqk::amma::score_prod2_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      cudaFuncSetAttribute(tqk::amma::value_prod2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)vsmem);
      cudaFuncSetAttribute(tqk::amma::value_prod2_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
    {
      KernelScope ks("attn_split", s);
      cudaError_t e = launch_pdl(tqk::amma::score_prod2_kernel<true>, dim3((unsigned)units, (unsigned)nsp),
                                 dim3(tqk::amma::kThreads), ssmem, s, ms);
      if (e != cudaSuccess) return cuda_fail(e, "score_prod2_kernel");
      e = launch_pdl(tqk::amma::value_prod2_kernel, dim3((unsigned)units, (unsigned)nsplit), dim3(tqk::amma::kThreads),
                     vsmem, s, mv);
      if (e != cudaSuccess) return cuda_fail(e, "value_prod2_kernel");
    }
    if ((st = launch_check("value_prod2_kernel"))) return st;
  } else if (attn_prod2_fast_path(hk, hv, G, k, v)) {
    tqk::amma::Args m{};
    // TQ_ATTN_TC=1: the tcgen05 kernel (attn_tc.cuh), measured slower than this mma.sync one at
    // these shapes (each of its small MMAs costs the tensor pipe about as much as a full-width one)
    const char* tce = std::getenv("TQ_ATTN_TC");
    const bool tc = tce && *tce && *tce != '0';
    if (tc) {
      const int sms = sm_count(hk->device);
      attn_tc_split(B, Hkv, k->L_cap, sms, &nsplit, &chunk);
    }
    m.qr = w.qr; m.qs = w.qs; m.B = B; m.Hq = Hq; m.Hkv = Hkv;
    m.kcodes = k->codes; m.ksigns = k->signs; m.knorm = static_cast<const __half*>(k->norms);
    m.krn = static_cast<const __half*>(k->rnorms);
    m.vcodes = v->codes; m.vsigns = v->signs; m.vnorm = static_cast<const __half*>(v->norms);
    m.vrn = static_cast<const __half*>(v->rnorms);
    m.L_cap = k->L_cap; m.chunk = chunk; m.nsplit = nsplit; m.len = len; m.len_extra = fused ? 1 : 0;
    m.kc0 = (float)hk->cent[0]; m.kb0 = (float)(hk->cent[1] - hk->cent[0]); m.kb1 = (float)(hk->cent[2] - hk->cent[0]);
    m.vc0 = (float)hv->cent[0]; m.vb0 = (float)(hv->cent[1] - hv->cent[0]); m.vb1 = (float)(hv->cent[2] - hv->cent[0]);
    m.scale = scale; m.part = part; m.err = hk->derr;
    if (tc) {
      const int nitems = B * Hkv * nsplit;
      const int grid = std::max(1, std::min(nitems, sm_count(hk->device)));
      if (once_per_device(12, hk->device))
        cudaFuncSetAttribute(tqk::atc::attn_prod2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tqk::atc::kSmemBytes);
      {
        KernelScope ks("attn_split", s);
        const cudaError_t e = launch_pdl(tqk::atc::attn_prod2_tc_kernel, dim3((unsigned)grid),
                                         dim3(tqk::atc::kThreads), (size_t)tqk::atc::kSmemBytes, s, m, nitems);
        if (e != cudaSuccess) return cuda_fail(e, "attn_prod2_tc_kernel");
      }
      if ((st = launch_check("attn_prod2_tc_kernel"))) return st;
    } else {
    const size_t msmem = sizeof(tqk::amma::Smem);
    if (once_per_device(2, hk->device)) {
      cudaFuncSetAttribute(tqk::amma::attn_prod2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
      cudaFuncSetAttribute(tqk::amma::attn_prod2_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
    {
      KernelScope ks("attn_split", s);
      const cudaError_t e = launch_pdl(tqk::amma::attn_prod2_kernel, dim3((unsigned)(B * Hkv), (unsigned)nsplit),
                                       dim3(tqk::amma::kThreads), msmem, s, m);
      if (e != cudaSuccess) return cuda_fail(e, "attn_prod2_kernel");
    }
    if ((st = launch_check("attn_prod2_kernel"))) return st;
    }
  } else if (attn_mse4_fast_path(hk, hv, G, k, v)) {
    tqk::am4::Args m4{};
    m4.qr = w.qr; m4.B = B; m4.Hq = Hq; m4.Hkv = Hkv;
    m4.kcodes = k->codes; m4.knorm = static_cast<const __half*>(k->norms);
    m4.vcodes = v->codes; m4.vnorm = static_cast<const __half*>(v->norms);
    m4.L_cap = k->L_cap; m4.chunk = chunk; m4.nsplit = nsplit; m4.len = len; m4.len_extra = fused ? 1 : 0;
    plane_coeffs4(hk->cent, &m4.kc0, m4.kw);
    plane_coeffs4(hv->cent, &m4.vc0, m4.vw);
    m4.scale = scale; m4.part = part; m4.err = hk->derr;
    const size_t msmem = sizeof(tqk::am4::Smem);
    if (once_per_device(11, hk->device)) {
      cudaFuncSetAttribute(tqk::am4::attn_mse4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
      cudaFuncSetAttribute(tqk::am4::attn_mse4_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
    {
      KernelScope ks("attn_split", s);
      const cudaError_t e = launch_pdl(tqk::am4::attn_mse4_kernel, dim3((unsigned)(B * Hkv), (unsigned)nsplit),
                                       dim3(tqk::am4::kThreads), msmem, s, m4);
      if (e != cudaSuccess) return cuda_fail(e, "attn_mse4_kernel");
    }
    if ((st = launch_check("attn_mse4_kernel"))) return st;
  } else {
    const size_t smem = ((size_t)G * (hk->d + hk->m) + 32 + (size_t)G * tqk::kAttnThreads +
                         2 * tqk::kAttnThreads + 4 * (size_t)G) * 4;
    {
      KernelScope ks("attn_split", s);
      const cudaError_t e = launch_pdl(tqk::attn_split_simt_kernel, dim3((unsigned)(B * Hkv), (unsigned)nsplit),
                                       dim3(tqk::kAttnThreads), smem, s, a);
      if (e != cudaSuccess) return cuda_fail(e, "attn_split_simt_kernel");
    }
    if ((st = launch_check("attn_split_simt_kernel"))) return st;
  }
  if (hv->d <= tqk::kWideMaxD && hv->m <= tqk::kWideMaxD &&
      tqk::combine_wide_smem_bytes(nsplit, hv->d, hv->m) <= 200 * 1024) {
    tqk::CombineWideArgs cs{};
    cs.part = part; cs.nsplit = nsplit; cs.d = hv->d; cs.mv = hv->m; cs.PiV = hv->dPi; cs.SV = hv->dS;
    cs.out = out; cs.err = hv->derr;
    cs.len_advance = fused ? len : nullptr; cs.Hq = Hq; cs.L_cap = k->L_cap;
    if (once_per_device(7, hv->device))
      cudaFuncSetAttribute(tqk::combine_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    KernelScope ks("attn_combine", s);
    const cudaError_t e = launch_pdl(tqk::combine_wide_kernel, dim3((unsigned)(B * Hq), (unsigned)(hv->d / tqk::kWideCols)),
                                     dim3(tqk::kSmallThreads), tqk::combine_wide_smem_bytes(nsplit, hv->d, hv->m), s, cs);
    if (e != cudaSuccess) return cuda_fail(e, "combine_wide_kernel");
    return launch_check("combine_wide_kernel");
  }
  tqk::CombineArgs c{};
  c.part = part; c.Hq = Hq; c.Hkv = Hkv; c.nsplit = nsplit; c.d = hv->d; c.mv = hv->m; c.PiV = hv->dPi;
  c.SV = hv->dS; c.out = out;
  const size_t csmem = ((size_t)nsplit + 2 * (size_t)(hv->d + hv->m) + 8 * (size_t)hv->d + 4) * 4;
  if (once_per_device(3, hv->device))
    cudaFuncSetAttribute(tqk::attn_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  {
    KernelScope ks("attn_combine", s);
    tqk::attn_combine_kernel<<<B * Hq, tqk::kCombineThreads, csmem, s>>>(c);
  }
  if ((st = launch_check("attn_combine_kernel"))) return st;
  if (fused) {
    KernelScope ks("advance_len", s);
    tqk::advance_len_kernel<<<(B + 255) / 256, 256, 0, s>>>(len, B, k->L_cap);
    return launch_check("advance_len_kernel");
  }
  return TQ_OK;
}

}  // namespace

extern "C" {

int tq_attn_decode(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                   const tq_cache* k, const tq_cache* v, const int32_t* len, float scale, float* out,
                   void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("tq_attn_decode");
  int st = attn_check(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, len, scale, out, workspace, ws_bytes);
  if (st || B == 0) return st;
  if ((st = pre_launch(hk, len, B, k->L_cap, static_cast<cudaStream_t>(stream)))) return st;
  return attn_impl(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, const_cast<int32_t*>(len), scale, out, workspace,
                   ws_bytes, static_cast<cudaStream_t>(stream), false);
}

int tq_decode_step(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype, const void* k_new,
                   const void* v_new, int x_dtype, int B, int Hq, int Hkv, const tq_cache* k, const tq_cache* v,
                   int32_t* len, float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("tq_decode_step");
  int st = attn_check(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, len, scale, out, workspace, ws_bytes);
  if (st || B == 0) return st;
  if (!valid_dtype(x_dtype)) return fail(TQ_EINVAL, "x dtype %d", x_dtype);
  if (!k_new || !v_new) return fail(TQ_EINVAL, "k_new/v_new NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return fail(TQ_EINVAL, "k_new/v_new misaligned");
  if (hk->d > tqk::kSmallMaxD || hk->m > tqk::kSmallMaxD || hv->m > tqk::kSmallMaxD || hk->d > tqk::kWideMaxD)
    return fail(TQ_EUNSUPPORTED, "tq_decode_step needs d <= %d and m <= %d", tqk::kSmallMaxD, tqk::kSmallMaxD);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = pre_launch(hk, len, B, k->L_cap, s))) return st;
  ScoreWs w;
  float* part;
  int nsplit;
  int64_t chunk;
  attn_ws_layout(hk, hv, B, Hq, Hkv, k->L_cap, static_cast<char*>(workspace), &w, &part, &nsplit, &chunk);
  auto enc = [&](const tq_handle* h, const void* x, const tq_cache* c) {
    tqk::EncodeArgs a{};
    a.x = x; a.x_dtype = x_dtype; a.rows = (int64_t)B * Hkv; a.d = h->d; a.bits = h->bits; a.m = h->m;
    a.norm_dtype = h->norm_dtype; a.PiT = h->dPiT; a.MT = h->dMT; a.cent = h->dcent; a.bnd = h->dbnd;
    a.codes = c->codes; a.codes_B = h->codes_B; a.signs = c->signs; a.signs_B = h->signs_B;
    a.norms = c->norms; a.rnorms = qjl_only(h) ? nullptr : static_cast<__half*>(c->rnorms);
    a.len = len; a.Hkv = Hkv; a.L_cap = c->L_cap; a.err = h->derr;
    if (qjl_only(h)) a.codes = nullptr;
    return a;
  };
  tqk::PrologueArgs p{};
  p.k = enc(hk, k_new, k);
  p.v = enc(hv, v_new, v);
  p.nvec = B * Hkv;
  p.q = q; p.q_dtype = q_dtype; p.rows = B * Hq; p.d = hk->d; p.m = hk->m; p.qcols = (hk->d + hk->m) / tqk::kWideCols;
  p.PiT = hk->dPiT; p.ST = hk->dST; p.qr = w.qr; p.qs = w.qs;
  p.pf[0] = hv->dPi; p.pf[1] = hv->dS;   // the combine's matrices: into L2 while the step runs
  p.pf_bytes[0] = (uint32_t)((size_t)hv->d * hv->d * 4);
  p.pf_bytes[1] = (uint32_t)((size_t)hv->m * hv->d * 4);
  const size_t smem = std::max({tqk::append_cluster_smem_bytes(hk->d, hk->m), tqk::append_cluster_smem_bytes(hv->d, hv->m),
                                tqk::qprep_wide_smem_bytes(hk->d, tqk::kQRows)});
  if (once_per_device(9, hk->device))
    cudaFuncSetAttribute(tqk::decode_prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  const unsigned grid = (unsigned)(2 * p.nvec + ((B * Hq + tqk::kQRows - 1) / tqk::kQRows) * p.qcols);
  {
    KernelScope ks("prologue", s);
    tqk::decode_prologue_kernel<<<grid, tqk::kSmallThreads, smem, s>>>(p);
  }
  if ((st = launch_check("decode_prologue_kernel"))) return st;
  return attn_impl(hk, hv, q, q_dtype, B, Hq, Hkv, k, v, len, scale, out, workspace, ws_bytes, s, true);
}


int tq_search_topk(const tq_handle* h, const float* q, int nq, const uint8_t* codes, const void* norms, int64_t n,
                   int k, int64_t* idx, float* score, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("tq_search_topk");
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (h->m > 0 || h->polar) return fail(TQ_EUNSUPPORTED, "search takes MSE handles");
  if (nq < 0 || n < 1 || k < 1 || k > tqk::kMaxTopK || k > n)
    return fail(TQ_EINVAL, "nq=%d n=%lld k=%d", nq, (long long)n, k);
  if (nq == 0) return ok();
  if (!q || !codes || !norms || !idx || !score || !workspace) return fail(TQ_EINVAL, "NULL pointer");
  if (!aligned(codes, 16) || !aligned(norms, 4) || !aligned(workspace, 16)) return fail(TQ_EINVAL, "misaligned pointer");
  const size_t need = tq_search_workspace_bytes(h, nq, n, k);
  if (ws_bytes < need) return fail(TQ_EINVAL, "workspace %zu < %zu bytes", ws_bytes, need);
  if (fault_is("launch")) return fail(TQ_ECUDA, "injected launch failure (TQ_FAULT=launch)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (int st0 = pre_launch(h, nullptr, 0, 0, s)) return st0;
  float *qr, *cs;
  int64_t* ci;
  int nchunks;
  int64_t chunk;
  if (search_tc_ok(h, n, k)) {
    int8_t* pieces;
    float* qscale;
    int* gbound;
    SampleWs sw;
    search_ws_layout(h, nq, n, k, static_cast<char*>(workspace), &qr, &cs, &ci, &nchunks, &chunk, true, &pieces,
                     &qscale, &gbound, &sw);
    const int nq_pad = (nq + tqk::stc::kQ - 1) / tqk::stc::kQ * tqk::stc::kQ;
    tqk::stc::Args m{};
    m.nq = nq; m.nq_pad = nq_pad; m.d = h->d; m.k = k; m.norm_dtype = h->norm_dtype; m.codes_B = h->codes_B;
    m.codes = codes; m.norms = norms; m.qscale = qscale; m.n = n; m.chunk = chunk;
    m.cand_s = cs; m.cand_i = ci; m.gbound = gbound; m.err = h->derr;
    float step_c;
    centroid_pieces(h->cent, &step_c, m.th, m.tl);
    CUtensorMap qmap;
    int st = codes_map_2d(reinterpret_cast<const uint8_t*>(pieces), 2 * (int64_t)nq_pad, h->d, tqk::stc::kKC,
                          tqk::stc::kQ, &qmap);
    if (st) return st;
    if ((st = launch_qprep(h, q, TQ_F32, nq, qr, nullptr, s))) return st;
    {
      KernelScope ks("search_qprep", s);
      const cudaError_t e = launch_pdl(tqk::stc::search_tc_qprep_kernel, dim3((unsigned)(nq_pad / 8)), dim3(256), 0,
                                       s, (const float*)qr, nq, nq_pad, h->d, step_c, pieces, qscale, gbound);
      if (e != cudaSuccess) return cuda_fail(e, "search_tc_qprep_kernel");
    }
    if ((st = launch_check("search_tc_qprep_kernel"))) return st;
    // the running lists hold 16 entries for k <= 16, else 32
    using Kern = void (*)(const CUtensorMap, tqk::stc::Args);
    static const Kern kerns[2][4] = {
        {tqk::stc::search_tc_kernel<1, 16>, tqk::stc::search_tc_kernel<2, 16>, tqk::stc::search_tc_kernel<3, 16>,
         tqk::stc::search_tc_kernel<4, 16>},
        {tqk::stc::search_tc_kernel<1, 32>, tqk::stc::search_tc_kernel<2, 32>, tqk::stc::search_tc_kernel<3, 32>,
         tqk::stc::search_tc_kernel<4, 32>}};
    const int big = k > 16 ? 1 : 0;
    auto kern = kerns[big][h->bits - 1];
    if (once_per_device(16 + 4 * big + h->bits, h->device))
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tqk::stc::kSmemBytes);
    const char* sample_env = std::getenv("TQ_SEARCH_SAMPLE");   // "0": no bound pass (tests compare both)
    if (sample_env && std::strcmp(sample_env, "0") == 0) sw.nchunks = 0;
    if (sw.nchunks > 0) {   // bound pass over the first kSearchSample vectors
      tqk::stc::Args ms = m;
      ms.n = kSearchSample; ms.chunk = sw.chunk; ms.cand_s = sw.cs; ms.cand_i = sw.ci;
      {
        KernelScope ks("search_sample", s);
        const cudaError_t e = launch_pdl(kern, dim3((unsigned)sw.nchunks, (unsigned)(nq_pad / tqk::stc::kQ)),
                                         dim3(tqk::stc::kThreads), (size_t)tqk::stc::kSmemBytes, s, qmap, ms);
        if (e != cudaSuccess) return cuda_fail(e, "search_tc_kernel");
      }
      if ((st = launch_check("search_tc_kernel"))) return st;
      {
        KernelScope ks("search_sample", s);
        const int nl = sw.nchunks * tqk::stc::kHalves;
        tqk::topk_merge_kernel<<<nq, 32, (size_t)nl * 4 + 16, s>>>(sw.cs, sw.ci, nl, nq, k, sw.ts, sw.ti);
        tqk::stc::search_tc_bound_kernel<<<(nq + 255) / 256, 256, 0, s>>>(sw.ts, sw.ti, nq, k, gbound);
      }
      if ((st = launch_check("search_tc_bound_kernel"))) return st;
    }
    {
      KernelScope ks("search", s);
      const cudaError_t e = launch_pdl(kern, dim3((unsigned)nchunks, (unsigned)(nq_pad / tqk::stc::kQ)),
                                       dim3(tqk::stc::kThreads), (size_t)tqk::stc::kSmemBytes, s, qmap, m);
      if (e != cudaSuccess) return cuda_fail(e, "search_tc_kernel");
    }
    if ((st = launch_check("search_tc_kernel"))) return st;
    KernelScope ks("topk_merge", s);
    const int nl = nchunks * tqk::stc::kHalves;
    tqk::topk_merge_kernel<<<nq, 32, (size_t)nl * 4 + 16, s>>>(cs, ci, nl, nq, k, score, idx);
    return launch_check("topk_merge_kernel");
  }
  search_ws_layout(h, nq, n, k, static_cast<char*>(workspace), &qr, &cs, &ci, &nchunks, &chunk, false);
  int st = launch_qprep(h, q, TQ_F32, nq, qr, nullptr, s);
  if (st) return st;
  tqk::SearchArgs a{};
  a.qr = qr; a.nq = nq; a.d = h->d; a.bits = h->bits; a.norm_dtype = h->norm_dtype; a.codes_B = h->codes_B;
  a.k = k; a.codes = codes; a.norms = norms; a.n = n; a.chunk = chunk; a.cent = h->dcent; a.cand_s = cs; a.cand_i = ci;
  const size_t smem = tqk::search_smem_bytes(k);
  if (once_per_device(1, h->device))
    cudaFuncSetAttribute(tqk::search_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  dim3 grid((unsigned)nchunks, (unsigned)((nq + tqk::kSQ - 1) / tqk::kSQ));
  {
    KernelScope ks("search", s);
    tqk::search_simt_kernel<<<grid, tqk::kSearchThreads, smem, s>>>(a);
  }
  if ((st = launch_check("search_simt_kernel"))) return st;
  KernelScope ks("topk_merge", s);
  tqk::topk_merge_kernel<<<nq, 32, (size_t)nchunks * 4 + 16, s>>>(cs, ci, nchunks, nq, k, score, idx);
  return launch_check("topk_merge_kernel");
}

int tq_timer_enable(int on) {
  if (on) {  // pre-create events so that a stream capture never has to create one
    std::lock_guard<std::mutex> lk(g_timer_mu);
    while (g_timer_pool.size() < 64) {
      cudaEvent_t e = nullptr;
      cudaError_t err = cudaEventCreate(&e);
      if (err != cudaSuccess) return cuda_fail(err, "cudaEventCreate");
      g_timer_pool.push_back(e);
    }
  }
  g_timer_on.store(on != 0);
  return ok();
}

int tq_timer_read(const char* name, double* ms, int* launches, int forget) {
  std::lock_guard<std::mutex> lk(g_timer_mu);
  double total = 0.0;
  int count = 0;
  std::vector<TimedLaunch> keep;
  for (auto& t : g_timer_pending) {
    if (name && t.name != name) {
      keep.push_back(t);
      continue;
    }
    cudaError_t e = cudaEventSynchronize(t.stop);
    float el = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&el, t.start, t.stop);
    if (e != cudaSuccess) {
      g_timer_pending.clear();
      return cuda_fail(e, "tq_timer_read");
    }
    total += el;
    ++count;
    if (forget) {
      g_timer_pool.push_back(t.start);
      g_timer_pool.push_back(t.stop);
    } else {
      keep.push_back(t);
    }
  }
  g_timer_pending.swap(keep);
  if (ms) *ms += total;
  if (launches) *launches += count;
  return ok();
}

int tq_selftest_wait_timeout(const tq_handle* h, int limit, void* stream) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  if (limit < 1 || limit > (1 << 16)) return fail(TQ_EINVAL, "limit=%d outside 1..65536", limit);
  tqk::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->derr, limit);
  return launch_check("selftest_wait_kernel");
}

int tq_last_status(const tq_handle* h, void* stream) {
  if (!h) return fail(TQ_EINVAL, "handle is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word = 0;
  e = cudaMemcpy(&word, h->derr, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word) {
    e = cudaMemset(h->derr, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  }
  if (word & tqk::kErrInternal) return fail(TQ_ECUDA, "a kernel found its shared memory misaligned");
  if (word & tqk::kErrBounds) return fail(TQ_EINVAL, "a length len[b] outside 0 .. L_cap (found by TQ_CHECK=1)");
  if (word & tqk::kErrTimeout) return fail(TQ_ETIMEOUT, "a bounded device wait timed out");
  if (word & tqk::kErrCapacity) return fail(TQ_ECAPACITY, "append skipped a full sequence (len == L_cap)");
  return ok();
}

const char* tq_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
