// C ABI of the GPT block library: argument checks, workspace layout and the
// launch sequence of one block / one stack training step.  All compute runs
// in the kernels included below (single translation unit).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/gptblock.h"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "elementwise.cuh"
#include "rows.cuh"
#include "gemm.cuh"

using namespace gptb;

namespace {

// ------------------------------------------------------------ accounting --
std::atomic<long long> g_launches{0};
std::mutex g_timing_mu;
bool g_timing = false;
struct TimedLaunch {
  cudaEvent_t a, b;
  double flops;
  bool fp8;  // e4m3 operands
};
std::vector<TimedLaunch> g_timed;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

#define LAUNCHED() g_launches.fetch_add(1, std::memory_order_relaxed)
#define CK(x)                                   \
  do {                                          \
    if ((x) != cudaSuccess) return GPTB_ERR_CUDA; \
  } while (0)
#define CKL()                                                  \
  do {                                                         \
    LAUNCHED();                                                \
    if (cudaPeekAtLastError() != cudaSuccess) {                \
      cudaGetLastError();                                      \
      return GPTB_ERR_CUDA;                                    \
    }                                                          \
  } while (0)
#define TRY(x)                     \
  do {                             \
    int _r = (x);                  \
    if (_r != GPTB_OK) return _r;  \
  } while (0)

// ------------------------------------------------------------ device info --
struct DevInfo {
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
};
DevInfo dev_info() {
  static DevInfo cache[64];
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  DevInfo& d = cache[dev & 63];
  if (d.sms == 0) {
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
  }
  return d;
}

// ------------------------------------------------------------ side stream --
// A second stream (per host thread and device) for the backward's weight-
// gradient GEMMs, which nothing on the block's input-gradient chain consumes:
// forked as soon as their inputs are written, they fill the SMs that the
// chain's kernels leave idle (a GEMM's last wave, a row kernel's spare
// resources).
// Fork and join by events; created once, never released.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t ev[5] = {};
  bool ok = false;
  bool tried = false;
};
SideStream& side_stream() {
  thread_local SideStream cache[16];
  int dev = 0;
  cudaGetDevice(&dev);
  SideStream& ss = cache[dev & 15];
  if (!ss.tried) {
    ss.tried = true;
    bool good = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; i < 5 && good; ++i) good = cudaEventCreateWithFlags(&ss.ev[i], cudaEventDisableTiming) == cudaSuccess;
    ss.ok = good;
    if (!good) cudaGetLastError();
  }
  return ss;
}

// ------------------------------------------------------------ tensor maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor map with 128-byte swizzle: inner extent `inner`, `outer` rows of
// `ld` elements; box = box_inner x box_outer.  Out-of-range reads fill zeros.
bool make_tmap(CUtensorMap* m, const void* ptr, bool fp8, uint64_t inner, uint64_t outer, uint64_t ld,
               uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * esz};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// GEMM operand maps: [batch][outer][inner] (row stride ld, batch stride bs
// elements; batch 1 is the plain matrix), 128-byte swizzle
bool make_tmap_gemm(CUtensorMap* m, const void* ptr, int esz, uint64_t inner, uint64_t outer, uint64_t ld,
                    uint32_t box_inner, uint32_t box_outer, int batch, long long bs) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (batch > 1 && (bs <= 0 || (bs * esz) % 16)) return false;
  const uint64_t bstride = (batch > 1 ? (uint64_t)bs : ld * outer) * (uint64_t)esz;
  cuuint64_t dims[3] = {inner, outer, (cuuint64_t)batch};
  cuuint64_t strides[2] = {ld * (uint64_t)esz, bstride};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 or bf16 [outer2][outer1][inner] view (row stride ld, plane stride
// ld*outer1), 128-byte swizzle; a store box that runs past outer1 is clipped
// there (the sequence end)
bool make_tmap_3d(CUtensorMap* m, const void* ptr, bool f32, uint64_t inner, uint64_t outer1, uint64_t outer2,
                  uint64_t ld, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = f32 ? 4 : 2;
  cuuint64_t dims[3] = {inner, outer1, outer2};
  cuuint64_t strides[2] = {ld * esz, ld * esz * outer1};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// --------------------------------------------------------------- GEMM ----
struct Op {
  const void* p;
  long long ld;  // row stride (elements) of the stored matrix
  bool mn;       // false: stored [rows, K] (K-major); true: stored [K, rows]
};

// split count for weight-gradient GEMMs: minimise waves * (k blocks per split
// + a fixed per-unit epilogue cost)
int plan_splits(int tiles, int kb_total, int sms) {
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= 16 && s <= kb_total; ++s) {
    const long long units = (long long)tiles * s;
    const long long waves = (units + sms - 1) / sms;
    const long long cost = waves * ((kb_total + s - 1) / s + 8);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// Largest number of two-CTA clusters of a pair-form GEMM kernel that fit on
// the device at once (one CTA per SM); a persistent grid larger than this
// would leave clusters waiting for others to finish.
template <class K>
int max_pair_clusters(K kern, int smem) {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  int& c = cache[dev & 63];
  if (c == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (dev_info().sms / 2));
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = dev_info().sms / 2;
    }
    c = std::min(n, dev_info().sms / 2);
  }
  return c;
}

template <bool AM, bool BM, bool F8, bool PAIR>
int launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to, const CUtensorMap& to2,
              const CUtensorMap& tx, int M, int N, int K, int splits, int nbatch, const EpiParams& ep,
              cudaStream_t st) {
  auto kern = gemm_tc_kernel<AM, BM, F8, PAIR>;
  const int smem = TcShape<PAIR>::SMEM;
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const long long units = (long long)((M + TcShape<PAIR>::TILE_M - 1) / TcShape<PAIR>::TILE_M) *
                          ((N + TC_BN - 1) / TC_BN) * splits * nbatch;
  if (!PAIR) {
    const int grid = (int)std::min<long long>(units, dev_info().sms);
    kern<<<grid, TC_THREADS, smem, st>>>(ta, tb, to, to2, tx, M, N, K, splits, nbatch, ep);
  } else {
    const int clusters = (int)std::min<long long>(units, max_pair_clusters(kern, smem));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, to, to2, tx, M, N, K, splits, nbatch, ep) != cudaSuccess) {
      cudaGetLastError();
      LAUNCHED();
      return GPTB_ERR_CUDA;
    }
  }
  CKL();
  return GPTB_OK;
}

// GEMMs with at least this many rows run in the pair form (two CTAs, M = 256
// per tile); smaller ones in the single-CTA form.
constexpr int GEMM_PAIR_MIN_M = 256;

// C[b] = A[b] op B[b] for b < batch: operand b starts bs* elements after
// operand 0 (tensor-core path only; the epilogue kinds with per-row side
// outputs take batch 1)
int gemm_batched(int dtype, Op A, Op B, int M, int N, int K, EpiParams ep, int batch, long long bsA, long long bsB,
                 long long bsO, long long bsX, cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch == 0) return GPTB_OK;
  if (batch < 0) return GPTB_ERR_INVALID_ARG;
  if (batch > 1 && (dtype == GPTB_F32 || ep.kind == EPI_XENT || ep.kind == EPI_QKV || ep.kind == EPI_DOT ||
                    ep.amax_out))
    return GPTB_ERR_UNSUPPORTED;
  if (K <= 0) return ep.kind == EPI_ACCUM_F32 ? GPTB_OK : GPTB_ERR_INVALID_ARG;
  cudaEvent_t ea = nullptr, eb = nullptr;
  bool timed = false;
  {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    if (g_timing) {
      ea = take_event();
      eb = take_event();
      timed = ea && eb;
    }
  }
  if (timed) cudaEventRecord(ea, st);
  int rc = GPTB_OK;
  if (dtype == GPTB_F32) {
    if (ep.kind == EPI_XENT || ep.kind == EPI_QKV || ep.kind == EPI_DOT) return GPTB_ERR_UNSUPPORTED;
    dim3 grid((N + 63) / 64, (M + 63) / 64);
    const float* a = static_cast<const float*>(A.p);
    const float* b = static_cast<const float*>(B.p);
    if (!A.mn && !B.mn) gemm_simt_f32_kernel<false, false><<<grid, 256, 0, st>>>(a, A.ld, b, B.ld, M, N, K, ep);
    else if (!A.mn && B.mn) gemm_simt_f32_kernel<false, true><<<grid, 256, 0, st>>>(a, A.ld, b, B.ld, M, N, K, ep);
    else if (A.mn && B.mn) gemm_simt_f32_kernel<true, true><<<grid, 256, 0, st>>>(a, A.ld, b, B.ld, M, N, K, ep);
    else gemm_simt_f32_kernel<true, false><<<grid, 256, 0, st>>>(a, A.ld, b, B.ld, M, N, K, ep);
    LAUNCHED();
    if (cudaPeekAtLastError() != cudaSuccess) {
      cudaGetLastError();
      rc = GPTB_ERR_CUDA;
    }
  } else {
    // tcgen05 path: bf16 operands, or e4m3 operands when dtype == GPTB_FP8_E4M3
    const DevInfo di = dev_info();
    if (di.cc_major != 10) return GPTB_ERR_UNSUPPORTED;
    const bool f8 = dtype == GPTB_FP8_E4M3;
    const int align = f8 ? 16 : 8;  // row strides must be multiples of 16 bytes
    const uint32_t bk = f8 ? 128 : 64;
    const bool acc32 = ep.kind == EPI_ACCUM_F32;
    const bool has_aux = ep.kind == EPI_RESID || ep.kind == EPI_DRELU2 || ep.kind == EPI_DOT;
    if (ep.out_f32 && !acc32) return GPTB_ERR_UNSUPPORTED;
    // a row's groups of 128 columns must lie inside one N tile
    if (ep.kind == EPI_DOT && (N % 128 || !ep.rowdot || ep.T <= 0 || M % ep.T)) return GPTB_ERR_INVALID_ARG;  // tensor-core outputs are bf16 or fp32 accumulations
    if (ep.kind == EPI_XENT && (!ep.xent_part || !ep.targets || !ep.xent_zy || ep.xent_nt < (N + TC_BN - 1) / TC_BN))
      return GPTB_ERR_INVALID_ARG;
    if (!aligned16(A.p) || !aligned16(B.p) || !aligned16(ep.out) || (A.ld % align) || (B.ld % align) ||
        (ep.ldo % (acc32 ? 4 : 8)) || (N % 8))
      return GPTB_ERR_INVALID_ARG;
    if (has_aux && (!aligned16(ep.aux) || ep.ld_aux % 8)) return GPTB_ERR_INVALID_ARG;
    const bool pair = M >= GEMM_PAIR_MIN_M;
    const int b_rows = pair ? TcShape<true>::B_ROWS : TcShape<false>::B_ROWS;  // rows of B one CTA stages
    CUtensorMap ta, tb, to, to2, tx;
    const int oe = f8 ? 1 : 2;  // operand element size
    bool ok = A.mn ? make_tmap_gemm(&ta, A.p, oe, M, K, A.ld, bk, bk, batch, bsA)
                   : make_tmap_gemm(&ta, A.p, oe, K, M, A.ld, bk, TC_BM, batch, bsA);
    ok = ok && (B.mn ? make_tmap_gemm(&tb, B.p, oe, N, K, B.ld, bk, bk, batch, bsB)
                     : make_tmap_gemm(&tb, B.p, oe, K, N, B.ld, bk, b_rows, batch, bsB));
    // epilogue maps: 32-row boxes of 64 bf16 / 32 fp32 columns, 128-byte swizzle
    ok = ok && (acc32 ? make_tmap_gemm(&to, ep.out, 4, N, M, ep.ldo, 32, 32, batch, bsO)
                      : make_tmap_gemm(&to, ep.out, 2, N, M, ep.ldo, 64, 32, batch, bsO));
    to2 = to;
    tx = to;
    if (ok && has_aux) ok = make_tmap_gemm(&tx, ep.aux, 2, N, M, ep.ld_aux, 64, 32, batch, bsX);
    if (!ok) return GPTB_ERR_CUDA;
    int splits = 1;
    if (ep.kind == EPI_ACCUM_F32) {
      const int tile_m = pair ? TcShape<true>::TILE_M : TcShape<false>::TILE_M;
      const int tiles = ((M + tile_m - 1) / tile_m) * ((N + TC_BN - 1) / TC_BN);
      splits = plan_splits(tiles, (K + (int)bk - 1) / (int)bk, pair ? di.sms / 2 : di.sms);
    }
    const int sel = (A.mn ? 1 : 0) | (B.mn ? 2 : 0) | (f8 ? 4 : 0) | (pair ? 8 : 0);
    switch (sel) {
      case 0: rc = launch_tc<false, false, false, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 1: rc = launch_tc<true, false, false, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 2: rc = launch_tc<false, true, false, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 3: rc = launch_tc<true, true, false, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 4: rc = launch_tc<false, false, true, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 6: rc = launch_tc<false, true, true, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 7: rc = launch_tc<true, true, true, false>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 8: rc = launch_tc<false, false, false, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 9: rc = launch_tc<true, false, false, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 10: rc = launch_tc<false, true, false, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 11: rc = launch_tc<true, true, false, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 12: rc = launch_tc<false, false, true, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 14: rc = launch_tc<false, true, true, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      case 15: rc = launch_tc<true, true, true, true>(ta, tb, to, to2, tx, M, N, K, splits, batch, ep, st); break;
      default: rc = GPTB_ERR_UNSUPPORTED;  // e4m3 with A M-major and B K-major: not used
    }
  }
  if (timed) {
    cudaEventRecord(eb, st);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timed.push_back({ea, eb, 2.0 * M * (double)N * K * batch, dtype == GPTB_FP8_E4M3});
  }
  return rc;
}

int gemm(int dtype, Op A, Op B, int M, int N, int K, EpiParams ep, cudaStream_t st) {
  return gemm_batched(dtype, A, B, M, N, K, ep, 1, 0, 0, 0, 0, st);
}

EpiParams epi(int kind, int dtype, void* out, long long ldo, const void* aux = nullptr, long long ld_aux = 0,
              void* out2 = nullptr, long long ldo2 = 0) {
  EpiParams e;
  e.kind = kind;
  e.out_f32 = (kind == EPI_ACCUM_F32 || dtype == GPTB_F32) ? 1 : 0;  // FP8 configs store bf16
  e.out = out;
  e.ldo = ldo;
  e.aux = aux;
  e.ld_aux = ld_aux;
  e.out2 = out2;
  e.ldo2 = ldo2;
  e.alpha = nullptr;
  e.beta = nullptr;
  e.amax_a = nullptr;
  e.amax_b = nullptr;
  e.a_e5m2 = 0;
  e.rope = nullptr;
  e.rstd_qk = nullptr;
  e.ve_table = nullptr;
  e.idx = nullptr;
  e.sg = nullptr;
  e.T = e.H = e.Hkv = 0;
  e.eps = 0.f;
  e.rowdot = nullptr;
  e.xent_part = nullptr;
  e.xent_nt = 0;
  e.targets = nullptr;
  e.xent_zy = nullptr;
  e.amax_out = nullptr;
  return e;
}
EpiParams epi8(EpiParams e, const float* amax_a, const float* amax_b, bool a_e5m2 = false) {
  e.amax_a = amax_a;
  e.amax_b = amax_b;
  e.a_e5m2 = a_e5m2 ? 1 : 0;
  return e;
}

// ---------------------------------------------------------- workspace -----
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

struct Dims {
  long long N;
  int B, T, d, H, Hkv, hd, F, V, L, Wq, NH, esz;
  bool fp8;
  bool grad_e5m2;  // FP8: gradient operands in e5m2
  bool fp8_lm;     // FP8: the lm_head GEMMs in FP8 as well
};
Dims dims_of(const gptb_config& c) {
  Dims m;
  m.B = c.B;
  m.T = c.T;
  m.N = (long long)c.B * c.T;
  m.d = c.d;
  m.H = c.n_head;
  m.Hkv = c.n_kv_head;
  m.hd = c.head_dim;
  m.F = c.mlp_hidden;
  m.V = c.vocab;
  m.L = c.n_layer;
  m.Wq = (c.n_head + 2 * c.n_kv_head) * c.head_dim;
  m.NH = c.n_head + c.n_kv_head;
  m.esz = c.dtype == GPTB_F32 ? 4 : 2;
  m.fp8 = c.dtype == GPTB_FP8_E4M3;
  m.grad_e5m2 = m.fp8 && (c.fp8_flags & GPTB_FP8_GRAD_E5M2);
  m.fp8_lm = m.fp8 && (c.fp8_flags & GPTB_FP8_LM_HEAD);
  return m;
}

struct Saved {
  void *h, *qkv, *o, *h2, *act;
  float *rstd1, *sg, *rstd_qk, *lse, *rstd2;
  // FP8 only: e4m3 copies of the four weights (reused by the input-gradient
  // GEMMs) and of the four GEMM activations (reused by the weight-gradient
  // GEMMs), and the amax of each
  uint8_t *wqkv8, *wo8, *wfc8, *wproj8;
  uint8_t *h8, *o8, *h2_8, *act8;
  float* amax;  // [h, o, h2, act, wqkv, wo, wfc, wproj]
};
Saved carve_saved(Carve& cv, const Dims& m) {
  Saved s;
  const size_t e = m.esz;
  s.h = cv.take(m.N * m.d * e);
  s.rstd1 = (float*)cv.take(m.N * 4);
  s.sg = (float*)cv.take(m.N * m.Hkv * 4);
  s.qkv = cv.take(m.N * m.Wq * e);
  s.rstd_qk = (float*)cv.take(m.N * m.NH * 4);
  s.o = cv.take(m.N * (long long)m.H * m.hd * e);
  s.lse = (float*)cv.take((size_t)m.B * m.H * m.T * 4);
  s.h2 = cv.take(m.N * m.d * e);
  s.rstd2 = (float*)cv.take(m.N * 4);
  s.act = cv.take(m.N * m.F * e);
  s.wqkv8 = s.wo8 = s.wfc8 = s.wproj8 = nullptr;
  s.h8 = s.o8 = s.h2_8 = s.act8 = nullptr;
  s.amax = nullptr;
  if (m.fp8) {
    const long long Ho = (long long)m.H * m.hd;
    s.wqkv8 = (uint8_t*)cv.take((size_t)m.Wq * m.d);
    s.wo8 = (uint8_t*)cv.take((size_t)m.d * Ho);
    s.wfc8 = (uint8_t*)cv.take((size_t)m.F * m.d);
    s.wproj8 = (uint8_t*)cv.take((size_t)m.d * m.F);
    s.h8 = (uint8_t*)cv.take((size_t)(m.N * m.d));
    s.o8 = (uint8_t*)cv.take((size_t)(m.N * Ho));
    s.h2_8 = (uint8_t*)cv.take((size_t)(m.N * m.d));
    s.act8 = (uint8_t*)cv.take((size_t)(m.N * m.F));
    s.amax = (float*)cv.take(8 * 4);
  }
  return s;
}

struct Scratch {
  float2* rope;
  // forward
  void *xm, *x1;
  // backward
  void *du, *dh2, *dx1, *dO, *dqkv, *dh;
  float *D, *dq, *dk, *dv, *dz;
  uint8_t* g8[4];  // FP8: e4m3 copies of the gradients feeding a GEMM pair [dx_out, du, dx1, dqkv]
  float* gamax;  // FP8: amax of the gradients [dx_out, du, dx1, dqkv]
};
Scratch carve_scratch(Carve& cv, const Dims& m) {
  Scratch s;
  const size_t e = m.esz;
  s.rope = (float2*)cv.take((size_t)m.T * (m.hd / 2) * sizeof(float2));
  const size_t start = cv.off;
  s.xm = cv.take(m.N * m.d * e);
  s.x1 = cv.take(m.N * m.d * e);
  const size_t fwd_end = cv.off;
  cv.off = start;  // backward temporaries reuse the forward's space
  s.du = cv.take(m.N * m.F * e);
  s.dh2 = cv.take(m.N * m.d * e);
  s.dx1 = cv.take(m.N * m.d * e);
  s.dO = cv.take(m.N * (long long)m.H * m.hd * e);
  s.dqkv = cv.take(m.N * m.Wq * e);
  s.dh = cv.take(m.N * m.d * e);
  s.D = (float*)cv.take((size_t)m.B * m.H * m.T * 4);
  s.dq = (float*)cv.take(m.N * (long long)m.H * m.hd * 4);
  s.dk = (float*)cv.take(m.N * (long long)m.Hkv * m.hd * 4);
  s.dv = (float*)cv.take(m.N * (long long)m.Hkv * m.hd * 4);
  s.dz = (float*)cv.take(m.N * m.Hkv * 4);
  for (auto& q : s.g8) q = nullptr;
  s.gamax = nullptr;
  if (m.fp8) {  // one copy per gradient: the weight-gradient GEMM on the side stream may still read one
    s.g8[0] = (uint8_t*)cv.take(m.N * m.d);
    s.g8[1] = (uint8_t*)cv.take(m.N * m.F);
    s.g8[2] = (uint8_t*)cv.take(m.N * m.d);
    s.g8[3] = (uint8_t*)cv.take(m.N * m.Wq);
    s.gamax = (float*)cv.take(4 * 4);  // [block input gradient, du, dx1, dqkv]
  }
  cv.off = std::max(cv.off, fwd_end);
  return s;
}

// lm_head temporaries: one row chunk of logits (overwritten by their
// gradient), the chunk's per-(row, 256-column tile) softmax statistics from
// the logits GEMM, z at the target and the log-sum-exp of each row, and the
// loss of every row.
struct LmWs {
  void* logits;
  float2* part;
  float* zy;
  float* lse;
  float* row_loss;
  int chunk;
  // FP8 lm_head: e4m3 copies of hf [N, d] and W_lm [V, d], the chunk's FP8
  // logits gradient, and the amax slots [hf, W_lm, bound of dz]
  uint8_t *h8, *w8, *dz8;
  float* amx;
};
int lm_tiles(int V) { return (V + TC_BN - 1) / TC_BN; }
LmWs carve_lm(Carve& cv, const Dims& m) {
  LmWs l;
  l.chunk = (int)std::min<long long>(m.N, 8192);
  l.logits = cv.take((size_t)l.chunk * m.V * m.esz);
  l.part = (float2*)cv.take((size_t)l.chunk * lm_tiles(m.V) * sizeof(float2));
  l.zy = (float*)cv.take((size_t)l.chunk * 4);
  l.lse = (float*)cv.take((size_t)l.chunk * 4);
  l.row_loss = (float*)cv.take(m.N * 4);
  l.h8 = l.w8 = l.dz8 = nullptr;
  l.amx = nullptr;
  if (m.fp8_lm) {
    l.h8 = (uint8_t*)cv.take((size_t)(m.N * m.d));
    l.w8 = (uint8_t*)cv.take((size_t)m.V * m.d);
    l.dz8 = (uint8_t*)cv.take((size_t)l.chunk * m.V);
    l.amx = (float*)cv.take(4 * 4);
  }
  return l;
}

struct StackWs {
  std::vector<void*> x_in;
  std::vector<Saved> saved;
  void *xL, *hf, *dhf, *dxA, *dxB, *dx_bo;
  float *rstd_f, *dx0;
  Scratch scr;
  LmWs lm;
};
StackWs carve_stack(Carve& cv, const Dims& m) {
  StackWs s;
  const size_t row = m.N * m.d * m.esz;
  for (int i = 0; i < m.L; ++i) s.x_in.push_back(cv.take(row));
  for (int i = 0; i < m.L; ++i) s.saved.push_back(carve_saved(cv, m));
  s.xL = cv.take(row);
  s.hf = cv.take(row);
  s.rstd_f = (float*)cv.take(m.N * 4);
  s.dhf = cv.take(row);
  s.dxA = cv.take(row);
  s.dxB = cv.take(row);
  s.dx_bo = cv.take(row);
  s.dx0 = (float*)cv.take(m.N * m.d * 4);
  s.scr = carve_scratch(cv, m);
  s.lm = carve_lm(cv, m);
  return s;
}

// ------------------------------------------------------------ checks ------
int check_config(const gptb_config* c) {
  if (!c) return GPTB_ERR_INVALID_ARG;
  if (c->dtype != GPTB_F32 && c->dtype != GPTB_BF16 && c->dtype != GPTB_FP8_E4M3) return GPTB_ERR_UNSUPPORTED;
  if (c->fp8_flags & ~(GPTB_FP8_GRAD_E5M2 | GPTB_FP8_LM_HEAD)) return GPTB_ERR_INVALID_ARG;
  if (c->fp8_flags && c->dtype != GPTB_FP8_E4M3) return GPTB_ERR_INVALID_ARG;
  if ((c->fp8_flags & GPTB_FP8_LM_HEAD) && (c->d % 16 || c->vocab % 16)) return GPTB_ERR_INVALID_ARG;
  if (c->B < 1 || c->T < 1 || c->d < 8 || c->d % 8 || c->d > 8 * 32 * BR_MAX_WARPS) return GPTB_ERR_INVALID_ARG;
  if (c->n_head < 1 || c->n_kv_head < 1 || c->n_head % c->n_kv_head) return GPTB_ERR_INVALID_ARG;
  if (c->mlp_hidden < 8 || c->mlp_hidden % 8 || c->vocab < 8 || c->vocab % 8) return GPTB_ERR_INVALID_ARG;
  if (c->n_layer < 1 || c->n_layer > GPTB_MAX_LAYERS) return GPTB_ERR_INVALID_ARG;
  if (c->backout_layer < -1 || c->backout_layer >= c->n_layer) return GPTB_ERR_INVALID_ARG;
  if (c->smear_ch < 0 || c->smear_ch > 256 || c->smear_ch > c->d) return GPTB_ERR_INVALID_ARG;
  if (!(c->norm_eps >= 0.f) || !(c->rope_base > 0.f)) return GPTB_ERR_INVALID_ARG;
  for (int i = 0; i < c->n_layer; ++i) {
    if (c->window[i] < -1) return GPTB_ERR_INVALID_ARG;
    if (c->has_ve[i] && (c->ve_gate_ch < 1 || c->ve_gate_ch > 256 || c->ve_gate_ch > c->d)) return GPTB_ERR_INVALID_ARG;
  }
  if (c->dtype == GPTB_F32) {
    if (c->head_dim < 2 || c->head_dim % 2 || c->head_dim > 128 || c->T > 1024) return GPTB_ERR_UNSUPPORTED;
  } else {
    if (c->head_dim != 128) return GPTB_ERR_UNSUPPORTED;
    if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  }
  if (((long long)c->B * c->T) > (1ll << 31) / 4) return GPTB_ERR_INVALID_ARG;
  return GPTB_OK;
}

// one CTA per token row: ceil(d/8) threads rounded up to whole warps
int br_threads(int d) { return ((d / 8 + 31) / 32) * 32; }
// grid of the warp-per-row kernels (8 rows per 256-thread block in flight, grid-stride beyond)
int warp_rows_grid(long long rows) {
  return (int)std::max<long long>(1, std::min<long long>((rows + 7) / 8, (long long)dev_info().sms * 8));
}
int br_grid(long long rows, int threads) {
  const long long cap = (long long)dev_info().sms * (2048 / threads) * 2;
  return (int)std::max<long long>(1, std::min(rows, cap));
}

int grid_rows(long long rows) {
  const long long wpb = EW_THREADS / 32;
  const long long need = (rows + wpb - 1) / wpb;
  const long long cap = (long long)dev_info().sms * 8;
  return (int)std::max<long long>(1, std::min(need, cap));
}

template <class T>
int rope_init(const gptb_config& c, float2* tab, cudaStream_t st) {
  const long long n = (long long)c.T * (c.head_dim / 2);
  rope_table_kernel<<<(int)std::min<long long>((n + 255) / 256, 4096), 256, 0, st>>>(tab, c.T, c.head_dim / 2,
                                                                                     (double)c.rope_base);
  CKL();
  return GPTB_OK;
}


// per-tensor FP8 quantisation: amax (fp32 bits, atomicMax) then codes, e4m3
// (scale 448/amax) or e5m2 (57344/amax)
// (amax_ready: the producer of x already published its amax into *amax)
template <class T>
int quant(const T* x, long long n, uint8_t* out, float* amax, bool e5m2, cudaStream_t st, bool amax_ready = false) {
  const long long n8 = n / 8;
  const int grid = (int)std::max<long long>(1, std::min<long long>((n8 + 255) / 256, (long long)dev_info().sms * 8));
  if (!amax_ready) {
    CK(cudaMemsetAsync(amax, 0, sizeof(float), st));
    amax_kernel<T><<<grid, 256, 0, st>>>(x, n8, reinterpret_cast<unsigned int*>(amax));
    CKL();
  }
  quantize_fp8_kernel<T><<<grid, 256, 0, st>>>(x, n8, amax, e5m2 ? 1 : 0, out);
  CKL();
  return GPTB_OK;
}

// One GEMM operand: the storage-dtype matrix and, for FP8 configs, its e4m3
// copy and amax slot (quant = produce the copy now; false = already produced).
struct Operand {
  const void* p;
  long long ld;
  bool mn;
  long long elems;
  uint8_t* q;
  float* amax;
  bool quant;
  bool e5m2;        // FP8 copy in e5m2 (gradient operands of the e5m2 variant)
  bool amax_ready;  // FP8: the producer of p already wrote its amax (no amax pass)
};

// A projection GEMM of the block in the config's arithmetic: f32 (SIMT) or
// bf16 (tcgen05) operands as stored, or per-tensor e4m3 operands (FP8: every
// product of the four block GEMMs -- forward, input gradient and weight
// gradient -- takes the e4m3 copies of its two bf16 operands).
template <class T>
int proj(const gptb_config& c, const Operand& A, const Operand& B, int M, int N, int K, const EpiParams& e,
         cudaStream_t st) {
  if (c.dtype != GPTB_FP8_E4M3) return gemm(c.dtype, {A.p, A.ld, A.mn}, {B.p, B.ld, B.mn}, M, N, K, e, st);
  if (!A.q || !B.q || !A.amax || !B.amax || B.e5m2) return GPTB_ERR_INVALID_ARG;
  if (A.quant) TRY(quant<T>((const T*)A.p, A.elems, A.q, A.amax, A.e5m2, st, A.amax_ready));
  if (B.quant) TRY(quant<T>((const T*)B.p, B.elems, B.q, B.amax, false, st, B.amax_ready));
  return gemm(GPTB_FP8_E4M3, {A.q, A.ld, A.mn}, {B.q, B.ld, B.mn}, M, N, K, epi8(e, A.amax, B.amax, A.e5m2), st);
}

// ------------------------------------------------------ block forward -----
template <class T>
int block_fwd_impl(const gptb_config& c, int layer, const gptb_block_weights& w, const T* x, const T* x0,
                   const int32_t* idx, T* x_out, const Saved& S, const Scratch& X, cudaStream_t st) {
  const Dims m = dims_of(c);
  const int brt = br_threads(m.d);
  const int brg = br_grid(m.N, brt);
  const bool ve = c.has_ve[layer] != 0;
  if (!w.w_qkv || !w.w_o || !w.w_fc || !w.w_proj || !w.lambdas || (ve && (!w.w_ve_gate || !w.ve_table)))
    return GPTB_ERR_INVALID_ARG;
  // FP8: the producers of the four GEMM activations publish their amax into S.amax[0..3]
  unsigned int* am = m.fp8 ? reinterpret_cast<unsigned int*>(S.amax) : nullptr;
  if (m.fp8) CK(cudaMemsetAsync(S.amax, 0, 4 * sizeof(float), st));
  br_mix_norm_kernel<T><<<brg, brt, 0, st>>>(x, x0, w.lambdas, (T*)X.xm, (T*)S.h, S.rstd1, m.N, m.d, c.norm_eps,
                                                ve ? (const T*)w.w_ve_gate : nullptr, S.sg, m.Hkv, c.ve_gate_ch,
                                                am ? am + 0 : nullptr);
  CKL();
  const long long Ho = (long long)m.H * m.hd;
  if (c.dtype == GPTB_F32) {
    TRY(gemm(c.dtype, {S.h, m.d, false}, {w.w_qkv, m.d, false}, (int)m.N, m.Wq, m.d,
             epi(EPI_STORE, c.dtype, S.qkv, m.Wq), st));
    qkv_post_kernel<T><<<grid_rows(m.N * (m.NH + (ve ? m.Hkv : 0))), EW_THREADS, 0, st>>>(
        (T*)S.qkv, m.Wq, S.rstd_qk, X.rope, m.T, m.N, m.H, m.Hkv, m.hd, c.norm_eps,
        ve ? (const T*)w.ve_table : nullptr, idx, S.sg);
    CKL();
  } else {
    // tensor-core QKV projection with QK RMSNorm + RoPE + value embedding fused into its epilogue
    EpiParams e = epi(EPI_QKV, c.dtype, S.qkv, m.Wq);
    e.rope = X.rope;
    e.rstd_qk = S.rstd_qk;
    e.ve_table = ve ? (const bf16*)w.ve_table : nullptr;
    e.idx = idx;
    e.sg = S.sg;
    e.T = m.T;
    e.H = m.H;
    e.Hkv = m.Hkv;
    e.eps = c.norm_eps;
    TRY(proj<T>(c, {S.h, m.d, false, m.N * m.d, S.h8, S.amax + 0, true, false, true},
                {w.w_qkv, m.d, false, (long long)m.Wq * m.d, S.wqkv8, S.amax + 4, true}, (int)m.N, m.Wq, m.d, e, st));
  }
  const int W = c.window[layer];
  if (c.dtype == GPTB_F32) {
    attn_fwd_simt_kernel<T><<<dim3(m.T, m.H, m.B), 128, 0, st>>>((const T*)S.qkv, m.Wq, (T*)S.o,
                                                                 (long long)m.H * m.hd, S.lse, m.T, m.H, m.Hkv, m.hd, W);
    CKL();
  } else {
    // tcgen05 flash attention: one tensor map (64-column boxes of 128 rows)
    // over the packed qkv buffer serves the Q, K and V tiles
    CUtensorMap tq, to;
    if (!make_tmap(&tq, S.qkv, false, (uint64_t)m.Wq, (uint64_t)m.N, (uint64_t)m.Wq, 64, 128)) return GPTB_ERR_CUDA;
    // o as [B][T][H*hd]: 64-column x 32-row store boxes that clip at each sequence end
    if (!make_tmap_3d(&to, S.o, false, (uint64_t)Ho, (uint64_t)m.T, (uint64_t)m.B, (uint64_t)Ho, 64, 32))
      return GPTB_ERR_CUDA;
    CK(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM));
    attn_fwd_tc_kernel<<<(unsigned)(((m.T + FA_QB - 1) / FA_QB) * m.H * m.B), FA_THREADS, FA_SMEM, st>>>(
        tq, to, S.lse, m.T, m.H, m.Hkv, W, am ? am + 1 : nullptr);
    CKL();
  }
  TRY(proj<T>(c, {S.o, Ho, false, m.N * Ho, S.o8, S.amax + 1, true, false, true},
              {w.w_o, Ho, false, m.d * Ho, S.wo8, S.amax + 5, true}, (int)m.N, m.d, (int)Ho,
              epi(EPI_RESID, c.dtype, X.x1, m.d, X.xm, m.d), st));
  br_norm_warp_kernel<T><<<warp_rows_grid(m.N), 256, 0, st>>>((const T*)X.x1, nullptr, nullptr, (T*)S.h2, S.rstd2, m.N, m.d,
                                            c.norm_eps, am ? am + 2 : nullptr);
  CKL();
  EpiParams erelu = epi(EPI_RELU2, c.dtype, S.act, m.F);
  erelu.amax_out = am ? am + 3 : nullptr;
  TRY(proj<T>(c, {S.h2, m.d, false, m.N * m.d, S.h2_8, S.amax + 2, true, false, true},
              {w.w_fc, m.d, false, (long long)m.F * m.d, S.wfc8, S.amax + 6, true}, (int)m.N, m.F, m.d, erelu, st));
  TRY(proj<T>(c, {S.act, m.F, false, m.N * m.F, S.act8, S.amax + 3, true, false, true},
              {w.w_proj, m.F, false, (long long)m.d * m.F, S.wproj8, S.amax + 7, true}, (int)m.N, m.d, m.F,
              epi(EPI_RESID, c.dtype, x_out, m.d, X.x1, m.d), st));
  return GPTB_OK;
}

// ----------------------------------------------------- block backward -----
template <class T>
int block_bwd_impl(const gptb_config& c, int layer, const gptb_block_weights& w, const T* x, const T* x0,
                   const int32_t* idx, const Saved& S, const T* dx2, const T* dx_extra, T* dx, float* dx0_acc,
                   const gptb_block_grads& g, const Scratch& X, cudaStream_t st) {
  const Dims m = dims_of(c);
  const int brt = br_threads(m.d);
  const int brg = br_grid(m.N, brt);
  const bool ve = c.has_ve[layer] != 0;
  if (!g.w_qkv || !g.w_o || !g.w_fc || !g.w_proj || !g.lambdas || (ve && (!g.w_ve_gate || !g.ve_table)))
    return GPTB_ERR_INVALID_ARG;
  const int dt = c.dtype;
  const int N = (int)m.N;
  const long long Ho = (long long)m.H * m.hd, Kv = (long long)m.Hkv * m.hd;
  // MLP
  // (FP8: the weight-gradient GEMM quantises the gradient, whose e4m3 copy the
  // input-gradient GEMM then reuses with the forward's e4m3 weight; the other
  // weight-gradient operand is the forward's saved e4m3 activation)
  const long long Nd = m.N * m.d;
  // FP8: amax slots of the four gradients [block input, du, dx1, dqkv]; the
  // producers of the last three publish theirs (no separate amax pass)
  float* ga[4] = {nullptr, nullptr, nullptr, nullptr};
  unsigned int* gam[4] = {nullptr, nullptr, nullptr, nullptr};
  if (m.fp8) {
    for (int i = 0; i < 4; ++i) {
      ga[i] = X.gamax + i;
      gam[i] = reinterpret_cast<unsigned int*>(X.gamax + i);
    }
    CK(cudaMemsetAsync(X.gamax + 1, 0, 3 * sizeof(float), st));
  }
  const bool e5 = m.grad_e5m2;
  // The weight-gradient GEMMs go to the side stream, each forked as soon as
  // its inputs are written and issued after the input-gradient GEMM beside it
  // (measured: 2 % off the d24 step, 4 % of its clock cycles; forking them
  // next to the memory-bound kernels instead was slower).  FP8: the gradient's
  // e4m3 copy, which both GEMMs of a pair read, is made on the main stream
  // before the fork (on one stream the weight-gradient GEMM makes it).
  SideStream* ss = nullptr;
  if (dt != GPTB_F32) {
    SideStream& s2 = side_stream();
    if (s2.ok) ss = &s2;
  }
  const bool q_first = ss && m.fp8;
  auto qgrad = [&](int i, const void* p, long long elems, bool amax_ready) -> int {
    return q_first ? quant<T>((const T*)p, elems, X.g8[i], ga[i], e5, st, amax_ready) : GPTB_OK;
  };
  cudaStream_t sw = ss ? ss->s : st;  // stream of the weight-gradient GEMMs
  auto fork = [&](int e) -> int {
    if (ss) {
      CK(cudaEventRecord(ss->ev[e], st));
      CK(cudaStreamWaitEvent(ss->s, ss->ev[e], 0));
    }
    return GPTB_OK;
  };
  auto wgrad_proj = [&]() {
    return proj<T>(c, {dx2, m.d, true, Nd, X.g8[0], ga[0], !q_first, e5}, {S.act, m.F, true, 0, S.act8, S.amax + 3, false},
                   m.d, m.F, N, epi(EPI_ACCUM_F32, dt, g.w_proj, m.F), sw);
  };
  auto wgrad_fc = [&]() {
    return proj<T>(c, {X.du, m.F, true, m.N * m.F, X.g8[1], ga[1], !q_first, e5, true},
                   {S.h2, m.d, true, 0, S.h2_8, S.amax + 2, false}, m.F, m.d, N, epi(EPI_ACCUM_F32, dt, g.w_fc, m.d),
                   sw);
  };
  EpiParams edr = epi(EPI_DRELU2, dt, X.du, m.F, S.act, m.F);
  edr.amax_out = gam[1];
  if (ss) {
    TRY(qgrad(0, dx2, Nd, false));
    TRY(fork(0));  // dx2 (and its e4m3 copy) and the saved activations are ready
    TRY(proj<T>(c, {dx2, m.d, false, Nd, X.g8[0], ga[0], false, e5},
                {w.w_proj, m.F, true, 0, S.wproj8, S.amax + 7, false}, N, m.F, m.d, edr, st));
    TRY(wgrad_proj());
    TRY(qgrad(1, X.du, m.N * m.F, true));
    TRY(fork(1));  // du
    TRY(proj<T>(c, {X.du, m.F, false, m.N * m.F, X.g8[1], ga[1], false, e5},
                {w.w_fc, m.d, true, 0, S.wfc8, S.amax + 6, false}, N, m.d, m.F, epi(EPI_STORE, dt, X.dh2, m.d), st));
    TRY(wgrad_fc());
  } else {
    TRY(wgrad_proj());
    TRY(proj<T>(c, {dx2, m.d, false, Nd, X.g8[0], ga[0], false, e5},
                {w.w_proj, m.F, true, 0, S.wproj8, S.amax + 7, false}, N, m.F, m.d, edr, st));
    TRY(wgrad_fc());
    TRY(proj<T>(c, {X.du, m.F, false, m.N * m.F, X.g8[1], ga[1], false, e5},
                {w.w_fc, m.d, true, 0, S.wfc8, S.amax + 6, false}, N, m.d, m.F, epi(EPI_STORE, dt, X.dh2, m.d), st));
  }
  br_norm_bwd_kernel<T><<<brg, brt, 0, st>>>(dx2, (const T*)X.dh2, (const T*)S.h2, S.rstd2, (T*)X.dx1, m.N, m.d,
                                                gam[2]);
  CKL();
  // attention output projection
  auto wgrad_o = [&]() {
    return proj<T>(c, {X.dx1, m.d, true, Nd, X.g8[2], ga[2], !q_first, e5, true}, {S.o, Ho, true, 0, S.o8, S.amax + 1, false},
                   m.d, (int)Ho, N, epi(EPI_ACCUM_F32, dt, g.w_o, Ho), sw);
  };
  if (ss) {
    TRY(qgrad(2, X.dx1, Nd, true));
    TRY(fork(2));  // dx1
  } else {
    TRY(wgrad_o());
  }
  // dO = dx1 Wo, and the attention backward's D = rowsum(dO * o) per head
  if constexpr (std::is_same<T, bf16>::value) {
    // bf16 / FP8 configurations: D comes out of the dO GEMM's epilogue (o read by TMA)
    EpiParams ed = epi(EPI_DOT, dt, X.dO, Ho, S.o, Ho);
    ed.rowdot = X.D;
    ed.T = m.T;
    ed.H = m.H;
    TRY(proj<T>(c, {X.dx1, m.d, false, Nd, X.g8[2], ga[2], false, e5}, {w.w_o, Ho, true, 0, S.wo8, S.amax + 5, false}, N,
                (int)Ho, m.d, ed, st));
    if (ss) TRY(wgrad_o());
  } else {
    TRY(proj<T>(c, {X.dx1, m.d, false, Nd, X.g8[2], ga[2], true, e5}, {w.w_o, Ho, true, 0, S.wo8, S.amax + 5, false}, N,
                (int)Ho, m.d, epi(EPI_STORE, dt, X.dO, Ho), st));
    attn_bwd_pre_kernel<T><<<grid_rows(m.N * m.H), EW_THREADS, 0, st>>>((const T*)S.o, Ho, (const T*)X.dO, Ho, X.D,
                                                                       m.B, m.T, m.H, m.hd);
    CKL();
  }
  CK(cudaMemsetAsync(X.dq, 0, m.N * Ho * 4, st));
  const int W = c.window[layer];
  if (dt == GPTB_F32) {
    CK(cudaMemsetAsync(X.dk, 0, m.N * Kv * 4, st));
    CK(cudaMemsetAsync(X.dv, 0, m.N * Kv * 4, st));
    attn_bwd_simt_kernel<T><<<dim3(m.T, m.H, m.B), 128, 0, st>>>((const T*)S.qkv, m.Wq, (const T*)X.dO, Ho, S.lse,
                                                                 X.D, X.dq, Ho, X.dk, X.dv, Kv, m.T, m.H, m.Hkv, m.hd,
                                                                 W);
    CKL();
  } else {
    // tcgen05 flash backward: K/V tiles (128 rows) and Q/dO tiles (64 rows) by
    // TMA, dQ accumulated with fp32 reductions at L2 into the zeroed buffer,
    // dK / dV (bf16) written whole by TMA stores (every key row of every tile)
    CUtensorMap tkv, tq, tdo, tdk, tdv;
    bool okm = make_tmap(&tkv, S.qkv, false, (uint64_t)m.Wq, (uint64_t)m.N, (uint64_t)m.Wq, 64, 128);
    okm = okm && make_tmap(&tq, S.qkv, false, (uint64_t)m.Wq, (uint64_t)m.N, (uint64_t)m.Wq, 64, 64);
    okm = okm && make_tmap(&tdo, X.dO, false, (uint64_t)Ho, (uint64_t)m.N, (uint64_t)Ho, 64, 64);
    okm = okm && make_tmap_3d(&tdk, X.dk, false, (uint64_t)Kv, (uint64_t)m.T, (uint64_t)m.B, (uint64_t)Kv, 64, 32);
    okm = okm && make_tmap_3d(&tdv, X.dv, false, (uint64_t)Kv, (uint64_t)m.T, (uint64_t)m.B, (uint64_t)Kv, 64, 32);
    if (!okm) return GPTB_ERR_CUDA;
    CK(cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AB2_SMEM));
    const int nkb = (m.T + AB2_BK - 1) / AB2_BK;
    attn_bwd_tc_kernel<<<nkb * m.Hkv * m.B, AB2_THREADS, AB2_SMEM, st>>>(tkv, tq, tdo, tdk, tdv, S.lse, X.D, X.dq, Ho,
                                                                       m.T, m.H, m.Hkv, m.B, W);
    CKL();
  }
  if constexpr (std::is_same<T, bf16>::value) {
    qkv_post_bwd_h128_kernel<<<grid_rows(m.N), EW_THREADS, 0, st>>>(
        (const bf16*)S.qkv, m.Wq, S.rstd_qk, X.rope, X.dq, Ho, (const bf16*)X.dk, (const bf16*)X.dv, Kv,
        (bf16*)X.dqkv, m.T, m.N, m.H, m.Hkv, ve ? (const bf16*)w.ve_table : nullptr, idx, S.sg,
        ve ? g.ve_table : nullptr, X.dz, gam[3]);
  } else {
    qkv_post_bwd_kernel<T><<<grid_rows(m.N * (m.H + 2 * m.Hkv)), EW_THREADS, 0, st>>>(
        (const T*)S.qkv, m.Wq, S.rstd_qk, X.rope, X.dq, Ho, X.dk, X.dv, Kv, (T*)X.dqkv, m.T, m.N, m.H, m.Hkv, m.hd,
        ve ? (const T*)w.ve_table : nullptr, idx, S.sg, ve ? g.ve_table : nullptr, X.dz);
  }
  CKL();
  // QKV projection
  auto wgrad_qkv = [&]() -> int {
    TRY(proj<T>(c, {X.dqkv, m.Wq, true, m.N * m.Wq, X.g8[3], ga[3], !q_first, e5, true},
                {S.h, m.d, true, 0, S.h8, S.amax + 0, false}, m.Wq, m.d, N, epi(EPI_ACCUM_F32, dt, g.w_qkv, m.d), sw));
    if (ve) {
      const int nthreads = ((m.Hkv * c.ve_gate_ch + 31) / 32) * 32;
      if (nthreads > 1024) return GPTB_ERR_UNSUPPORTED;
      ve_gate_wgrad_kernel<T><<<dev_info().sms * 4, nthreads, 0, sw>>>(X.dz, (const T*)S.h, m.N, m.d, m.Hkv,
                                                                       c.ve_gate_ch, g.w_ve_gate);
      CKL();
    }
    return GPTB_OK;
  };
  if (ss) {
    TRY(qgrad(3, X.dqkv, m.N * m.Wq, true));
    TRY(fork(3));  // dqkv, dz
  } else {
    TRY(wgrad_qkv());
  }
  TRY(proj<T>(c, {X.dqkv, m.Wq, false, m.N * m.Wq, X.g8[3], ga[3], false, e5},
              {w.w_qkv, m.d, true, 0, S.wqkv8, S.amax + 4, false}, N, m.d, m.Wq, epi(EPI_STORE, dt, X.dh, m.d), st));
  if (ss) TRY(wgrad_qkv());
  br_mix_norm_bwd_warp_kernel<T><<<warp_rows_grid(m.N), 256, 0, st>>>((const T*)X.dh, ve ? X.dz : nullptr,
                                                         ve ? (const T*)w.w_ve_gate : nullptr, m.Hkv, c.ve_gate_ch,
                                                         (const T*)S.h, S.rstd1, (const T*)X.dx1, x, x0, w.lambdas,
                                                         dx_extra, dx, dx0_acc, g.lambdas, m.N, m.d);
  CKL();
  if (ss) {  // join: the layer's weight gradients are complete at this point of the stream
    CK(cudaEventRecord(ss->ev[4], ss->s));
    CK(cudaStreamWaitEvent(st, ss->ev[4], 0));
  }
  return GPTB_OK;
}

// -------------------------------------------------------------- lm head ---
template <class T>
int lm_head_impl(const gptb_config& c, const T* h, const T* w_lm, const int32_t* targets, float* loss_out, T* dh,
                 float* dw_lm, const LmWs& lw, cudaStream_t st) {
  const Dims m = dims_of(c);
  const int brt = br_threads(m.d);
  const int brg = br_grid(m.N, brt);
  const int dt = c.dtype == GPTB_FP8_E4M3 ? GPTB_BF16 : c.dtype;  // lm_head bf16 unless GPTB_FP8_LM_HEAD
  if constexpr (std::is_same<T, bf16>::value) {
    if (m.fp8_lm) {
      // FP8 lm_head: e4m3 copies of the whole hf and of W_lm (per-tensor scales)
      if (!lw.h8 || !lw.w8 || !lw.dz8 || !lw.amx) return GPTB_ERR_UNSUPPORTED;
      TRY(quant<bf16>(h, m.N * m.d, lw.h8, lw.amx + 0, false, st));
      TRY(quant<bf16>(w_lm, (long long)m.V * m.d, lw.w8, lw.amx + 1, false, st));
    }
  }
  for (long long c0 = 0; c0 < m.N; c0 += lw.chunk) {
    const int rows = (int)std::min<long long>(lw.chunk, m.N - c0);
    const T* hc = h + c0 * m.d;
    if constexpr (std::is_same<T, bf16>::value) {
      // logits GEMM whose epilogue also emits the per-tile softmax statistics
      // and z at the target; then the row log-sum-exp and the logits gradient
      EpiParams e = epi(EPI_XENT, dt, lw.logits, m.V);
      e.xent_part = lw.part;
      e.xent_nt = lm_tiles(m.V);
      e.targets = targets + c0;
      e.xent_zy = lw.zy;
      if (m.fp8_lm)
        TRY(gemm(GPTB_FP8_E4M3, {lw.h8 + c0 * m.d, m.d, false}, {lw.w8, m.d, false}, rows, m.V, m.d,
                 epi8(e, lw.amx + 0, lw.amx + 1), st));
      else
        TRY(gemm(dt, {hc, m.d, false}, {w_lm, m.d, false}, rows, m.V, m.d, e, st));
      xent_lse_kernel<<<grid_rows(rows), EW_THREADS, 0, st>>>(lw.part, lm_tiles(m.V), lw.zy, targets + c0, m.V,
                                                               lw.lse, lw.row_loss + c0, rows);
      CKL();
      if (m.fp8_lm) {
        // the logits gradient as FP8 codes with the scale its bound 1/N fixes,
        // then the two gradient GEMMs on FP8 operands
        xent_grad_fp8_kernel<<<rows, XENT_GRAD_THREADS, 0, st>>>((const bf16*)lw.logits, m.V, m.V, targets + c0,
                                                                  lw.lse, 1.f / (float)m.N, m.grad_e5m2 ? 1 : 0,
                                                                  lw.dz8, m.V, lw.amx + 2, rows);
        CKL();
        TRY(gemm(GPTB_FP8_E4M3, {lw.dz8, m.V, false}, {lw.w8, m.d, true}, rows, m.d, m.V,
                 epi8(epi(EPI_STORE, dt, dh + c0 * m.d, m.d), lw.amx + 2, lw.amx + 1, m.grad_e5m2), st));
        TRY(gemm(GPTB_FP8_E4M3, {lw.dz8, m.V, true}, {lw.h8 + c0 * m.d, m.d, true}, m.V, m.d, rows,
                 epi8(epi(EPI_ACCUM_F32, dt, dw_lm, m.d), lw.amx + 2, lw.amx + 0, m.grad_e5m2), st));
        continue;
      }
      xent_grad_kernel<<<rows, XENT_GRAD_THREADS, 0, st>>>((bf16*)lw.logits, m.V, m.V, targets + c0, lw.lse,
                                                            1.f / (float)m.N, rows);
    } else {
      TRY(gemm(dt, {hc, m.d, false}, {w_lm, m.d, false}, rows, m.V, m.d, epi(EPI_STORE, dt, lw.logits, m.V), st));
      xent_rows_kernel<T><<<rows, 512, 0, st>>>((T*)lw.logits, m.V, m.V, targets + c0, lw.row_loss + c0,
                                                1.f / (float)m.N, rows);
    }
    CKL();
    TRY(gemm(dt, {lw.logits, m.V, false}, {w_lm, m.d, true}, rows, m.d, m.V, epi(EPI_STORE, dt, dh + c0 * m.d, m.d),
             st));
    TRY(gemm(dt, {lw.logits, m.V, true}, {hc, m.d, true}, m.V, m.d, rows, epi(EPI_ACCUM_F32, dt, dw_lm, m.d), st));
  }
  mean_kernel<<<1, 1024, 0, st>>>(lw.row_loss, m.N, loss_out);
  CKL();
  return GPTB_OK;
}

// --------------------------------------------------------------- stack ----
template <class T>
int stack_impl(const gptb_config& c, const gptb_model_weights& w, const int32_t* idx, const int32_t* targets,
               float* loss_out, const gptb_model_grads& g, const StackWs& S, cudaStream_t st,
               gptb_grads_ready_fn ready = nullptr, void* user = nullptr) {
  const Dims m = dims_of(c);
  const int brt = br_threads(m.d);
  const int brg = br_grid(m.N, brt);
  if (!w.wte || !w.w_lm || !g.wte || !g.w_lm) return GPTB_ERR_INVALID_ARG;
  if (c.smear_ch > 0 && (!w.w_smear_gate || !w.smear_lambda || !g.w_smear_gate || !g.smear_lambda))
    return GPTB_ERR_INVALID_ARG;
  if (c.backout_layer >= 0 && (!w.backout_lambda || !g.backout_lambda)) return GPTB_ERR_INVALID_ARG;
  TRY(rope_init<T>(c, S.scr.rope, st));
  br_embed_smear_kernel<T><<<brg, brt, 0, st>>>(idx, (const T*)w.wte, (const T*)w.w_smear_gate, w.smear_lambda,
                                                   (T*)S.x_in[0], m.B, m.T, m.d, c.smear_ch);
  CKL();
  const T* x0 = (const T*)S.x_in[0];
  for (int i = 0; i < m.L; ++i) {
    T* xo = (T*)(i + 1 < m.L ? S.x_in[i + 1] : S.xL);
    TRY(block_fwd_impl<T>(c, i, w.layers[i], (const T*)S.x_in[i], x0, idx, xo, S.saved[i], S.scr, st));
  }
  const T* x_bo = c.backout_layer >= 0 ? (const T*)S.x_in[c.backout_layer] : nullptr;
  br_norm_warp_kernel<T><<<warp_rows_grid(m.N), 256, 0, st>>>((const T*)S.xL, x_bo, w.backout_lambda, (T*)S.hf, S.rstd_f, m.N, m.d,
                                            c.norm_eps, nullptr);
  CKL();
  TRY(lm_head_impl<T>(c, (const T*)S.hf, (const T*)w.w_lm, targets, loss_out, (T*)S.dhf, g.w_lm, S.lm, st));
  br_final_norm_bwd_kernel<T><<<brg, brt, 0, st>>>((const T*)S.dhf, (const T*)S.hf, S.rstd_f, x_bo,
                                                      w.backout_lambda, (T*)S.dxA, (T*)S.dx_bo, g.backout_lambda,
                                                      m.N, m.d);
  CKL();
  CK(cudaMemsetAsync(S.dx0, 0, m.N * m.d * 4, st));
  T* cur = (T*)S.dxA;
  T* nxt = (T*)S.dxB;
  for (int i = m.L - 1; i >= 0; --i) {
    const T* extra = (i == c.backout_layer) ? (const T*)S.dx_bo : nullptr;
    TRY(block_bwd_impl<T>(c, i, w.layers[i], (const T*)S.x_in[i], x0, idx, S.saved[i], cur, extra, nxt, S.dx0,
                          g.layers[i], S.scr, st));
    if (ready) ready(i, user);  // layer i's weight gradients are complete once this point of the stream is
    std::swap(cur, nxt);
  }
  br_smear_embed_bwd_kernel<T><<<brg, brt, 0, st>>>(cur, S.dx0, idx, (const T*)w.wte, (const T*)w.w_smear_gate,
                                                       w.smear_lambda, g.wte, g.w_smear_gate, g.smear_lambda, m.B, m.T,
                                                       m.d, c.smear_ch);
  CKL();
  if (ready) ready(-1, user);  // the embedding, lm_head, smear and backout gradients
  return GPTB_OK;
}

}  // namespace

// ------------------------------------------------------ wait self-test ----
// One CTA waits on an mbarrier that nothing arrives on.  The bounded wait
// must expire, record ERRW_TIMEOUT_PROBE and let the kernel return.
__device__ int g_probe_result = -1;
__global__ void wait_probe_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_warp(&bar, 0, &abort_flag, ERRW_TIMEOUT_PROBE);
  if (threadIdx.x == 0) g_probe_result = ok ? 1 : 0;
}

// ================================================================ C ABI ====
extern "C" {

size_t gptb_workspace_bytes(const gptb_config* cfg, int kind) {
  if (!cfg || cfg->B < 1 || cfg->T < 1 || cfg->n_layer < 1 || cfg->n_layer > GPTB_MAX_LAYERS) return 0;
  const Dims m = dims_of(*cfg);
  Carve cv(nullptr);
  switch (kind) {
    case GPTB_WS_BLOCK_SAVED: carve_saved(cv, m); break;
    case GPTB_WS_BLOCK_SCRATCH: carve_scratch(cv, m); break;
    case GPTB_WS_LM_HEAD: carve_lm(cv, m); break;
    case GPTB_WS_STACK: carve_stack(cv, m); break;
    default: return 0;
  }
  return (cv.off + 255) & ~size_t(255);
}

int gpt_block_forward(const gptb_config* cfg, int layer, const gptb_block_weights* w, const void* x, const void* x0,
                      const int32_t* idx, void* x_out, void* saved, void* scratch, gptb_stream_t stream) {
  TRY(check_config(cfg));
  if (!w || !x || !x0 || !idx || !x_out || !saved || !scratch || layer < 0 || layer >= cfg->n_layer)
    return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  Carve cs(saved), cx(scratch);
  const Saved S = carve_saved(cs, m);
  const Scratch X = carve_scratch(cx, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32) {
    TRY(rope_init<float>(*cfg, X.rope, st));
    return block_fwd_impl<float>(*cfg, layer, *w, (const float*)x, (const float*)x0, idx, (float*)x_out, S, X, st);
  }
  TRY(rope_init<bf16>(*cfg, X.rope, st));
  return block_fwd_impl<bf16>(*cfg, layer, *w, (const bf16*)x, (const bf16*)x0, idx, (bf16*)x_out, S, X, st);
}

int gpt_block_backward(const gptb_config* cfg, int layer, const gptb_block_weights* w, const void* x, const void* x0,
                       const int32_t* idx, const void* saved, const void* dx_out, const void* dx_extra, void* dx,
                       float* dx0_accum, gptb_block_grads* g, void* scratch, gptb_stream_t stream) {
  TRY(check_config(cfg));
  if (!w || !x || !x0 || !idx || !saved || !dx_out || !dx || !dx0_accum || !g || !scratch || layer < 0 ||
      layer >= cfg->n_layer)
    return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  Carve cs(const_cast<void*>(saved)), cx(scratch);
  const Saved S = carve_saved(cs, m);
  const Scratch X = carve_scratch(cx, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32) {
    TRY(rope_init<float>(*cfg, X.rope, st));
    return block_bwd_impl<float>(*cfg, layer, *w, (const float*)x, (const float*)x0, idx, S, (const float*)dx_out,
                                 (const float*)dx_extra, (float*)dx, dx0_accum, *g, X, st);
  }
  TRY(rope_init<bf16>(*cfg, X.rope, st));
  return block_bwd_impl<bf16>(*cfg, layer, *w, (const bf16*)x, (const bf16*)x0, idx, S, (const bf16*)dx_out,
                              (const bf16*)dx_extra, (bf16*)dx, dx0_accum, *g, X, st);
}

int lm_head_xent(const gptb_config* cfg, const void* h, const void* w_lm, const int32_t* targets, float* loss_out,
                 void* dh, float* dw_lm, void* ws, gptb_stream_t stream) {
  TRY(check_config(cfg));
  if (!h || !w_lm || !targets || !loss_out || !dh || !dw_lm || !ws) return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  Carve cv(ws);
  const LmWs lw = carve_lm(cv, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32)
    return lm_head_impl<float>(*cfg, (const float*)h, (const float*)w_lm, targets, loss_out, (float*)dh, dw_lm, lw, st);
  return lm_head_impl<bf16>(*cfg, (const bf16*)h, (const bf16*)w_lm, targets, loss_out, (bf16*)dh, dw_lm, lw, st);
}

int gpt_stack_step(const gptb_config* cfg, const gptb_model_weights* w, const int32_t* idx, const int32_t* targets,
                   float* loss_out, gptb_model_grads* g, void* ws, gptb_stream_t stream) {
  TRY(check_config(cfg));
  if (!w || !idx || !targets || !loss_out || !g || !ws) return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  Carve cv(ws);
  const StackWs S = carve_stack(cv, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32) return stack_impl<float>(*cfg, *w, idx, targets, loss_out, *g, S, st);
  return stack_impl<bf16>(*cfg, *w, idx, targets, loss_out, *g, S, st);
}

int gpt_stack_step_hooked(const gptb_config* cfg, const gptb_model_weights* w, const int32_t* idx,
                          const int32_t* targets, float* loss_out, gptb_model_grads* g, void* ws, gptb_stream_t stream,
                          gptb_grads_ready_fn ready, void* user) {
  TRY(check_config(cfg));
  if (!w || !idx || !targets || !loss_out || !g || !ws || !ready) return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  Carve cv(ws);
  const StackWs S = carve_stack(cv, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32) return stack_impl<float>(*cfg, *w, idx, targets, loss_out, *g, S, st, ready, user);
  return stack_impl<bf16>(*cfg, *w, idx, targets, loss_out, *g, S, st, ready, user);
}

int gptb_gemm_bf16(const void* A, int a_mn, long long lda, const void* B, int b_mn, long long ldb, void* C, int c_f32,
                   long long ldc, int M, int N, int K, gptb_stream_t stream) {
  if (!A || !B || !C || M < 0 || N < 0 || K < 0) return GPTB_ERR_INVALID_ARG;
  if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  EpiParams e = epi(c_f32 ? EPI_ACCUM_F32 : EPI_STORE, GPTB_BF16, C, ldc);
  return gemm(GPTB_BF16, {A, lda, a_mn != 0}, {B, ldb, b_mn != 0}, M, N, K, e, reinterpret_cast<cudaStream_t>(stream));
}

int gptb_gemm_bf16_batched(const void* A, int a_mn, long long lda, long long stride_a, const void* B, int b_mn,
                           long long ldb, long long stride_b, void* C, int c_f32, long long ldc, long long stride_c,
                           int M, int N, int K, int batch, gptb_stream_t stream) {
  if (!A || !B || !C || M < 0 || N < 0 || K < 0 || batch < 1) return GPTB_ERR_INVALID_ARG;
  if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  EpiParams e = epi(c_f32 ? EPI_ACCUM_F32 : EPI_STORE, GPTB_BF16, C, ldc);
  return gemm_batched(GPTB_BF16, {A, lda, a_mn != 0}, {B, ldb, b_mn != 0}, M, N, K, e, batch, stride_a, stride_b,
                      stride_c, 0, reinterpret_cast<cudaStream_t>(stream));
}

size_t gptb_gemm_fp8_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return ((size_t)M * K + 255) / 256 * 256 + ((size_t)N * K + 255) / 256 * 256 + 256;
}

int gptb_gemm_fp8(const void* A, int a_mn, long long lda, const void* B, int b_mn, long long ldb, float* C,
                  long long ldc, int M, int N, int K, int a_e5m2, void* workspace, size_t workspace_bytes,
                  gptb_stream_t stream) {
  if (!A || !B || !C || !workspace || M <= 0 || N <= 0 || K <= 0) return GPTB_ERR_INVALID_ARG;
  if (a_mn && !b_mn) return GPTB_ERR_UNSUPPORTED;  // the one layout the block never uses
  if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  if (workspace_bytes < gptb_gemm_fp8_workspace_bytes(M, N, K) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GPTB_ERR_WORKSPACE;
  // the stored matrices must be dense (row stride = the inner extent) for the per-tensor cast
  if (lda != (a_mn ? M : K) || ldb != (b_mn ? N : K)) return GPTB_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint8_t* a8 = w;
  uint8_t* b8 = w + ((size_t)M * K + 255) / 256 * 256;
  float* amax = reinterpret_cast<float*>(b8 + ((size_t)N * K + 255) / 256 * 256);
  if (((long long)M * K) % 8 || ((long long)N * K) % 8) return GPTB_ERR_INVALID_ARG;
  TRY(quant<bf16>(static_cast<const bf16*>(A), (long long)M * K, a8, amax + 0, a_e5m2 != 0, st));
  TRY(quant<bf16>(static_cast<const bf16*>(B), (long long)N * K, b8, amax + 1, false, st));
  return gemm(GPTB_FP8_E4M3, {a8, lda, a_mn != 0}, {b8, ldb, b_mn != 0}, M, N, K,
              epi8(epi(EPI_ACCUM_F32, GPTB_FP8_E4M3, C, ldc), amax + 0, amax + 1, a_e5m2 != 0), st);
}

// ------------------------------------------------------ optimizer step --

int gptb_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, long long n, float lr, float beta1,
                    float beta2, float eps, float weight_decay, int step, gptb_stream_t stream) {
  if (!p || !g || !m || !v || n < 0 || step < 1) return GPTB_ERR_INVALID_ARG;
  if (n == 0) return GPTB_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const double bc1 = 1.0 - std::pow((double)beta1, step), bc2 = 1.0 - std::pow((double)beta2, step);
  if (!(bc1 > 0.0) || !(bc2 > 0.0)) return GPTB_ERR_INVALID_ARG;  // beta1 or beta2 outside [0, 1)
  const bool vec4 = (n % 4 == 0) && aligned16(p) && aligned16(g) && aligned16(m) && aligned16(v) &&
                    (p_bf16 == nullptr || (reinterpret_cast<uintptr_t>(p_bf16) & 7u) == 0);
  const long long items = vec4 ? n / 4 : n;
  const int threads = 256;
  const long long cap = (long long)dev_info().sms * 8;
  const int grid = (int)std::max<long long>(1, std::min((items + threads - 1) / threads, cap));
  adamw_kernel<<<grid, threads, 0, st>>>(p, g, m, v, reinterpret_cast<bf16*>(p_bf16), n, lr, beta1, beta2, eps,
                                         1.f - lr * weight_decay, (float)(1.0 / bc1), (float)(1.0 / std::sqrt(bc2)),
                                         vec4 ? 1 : 0);
  CKL();
  return GPTB_OK;
}

namespace {
constexpr size_t PE_HEADER = 1024;  // sum of squares (4 B) at 0, coefficients (<= 64 x 3 floats) at 256
size_t pe_align(size_t b) { return (b + 255) & ~size_t(255); }
}  // namespace

// Polar Express workspace for `count` matrices of m x n: header (per-matrix
// sums of squares at 0, coefficients at 256), two count x m x n iterates,
// and count Gram matrices A and B of the smaller side
constexpr int PE_MAX_BATCH = 64;
size_t pe_bytes(int count, int m, int n, int steps) {
  if (count <= 0 || count > PE_MAX_BATCH || m <= 0 || n <= 0 || steps < 1 || steps > 64) return 0;
  const size_t s = (size_t)std::min(m, n);
  return PE_HEADER + 2 * pe_align((size_t)count * m * n * 2) + 2 * pe_align((size_t)count * s * s * 2);
}

size_t gptb_polar_express_workspace_bytes(int m, int n, int steps) { return pe_bytes(1, m, n, steps); }

}  // extern "C"

namespace {
// The Polar Express loop on a bf16 [m, n] matrix into out (workspace laid out
// as gptb_polar_express_workspace_bytes describes; arguments already checked).
int polar_express_impl(const void* G, void* out, int m, int n, int count, const float* coeffs, int steps, uint8_t* w,
                       cudaStream_t st) {
  const size_t ne = (size_t)m * n;
  float* sumsq = reinterpret_cast<float*>(w);  // [count]
  float* cf = reinterpret_cast<float*>(w + 256);
  bf16* X[2];
  X[0] = reinterpret_cast<bf16*>(w + PE_HEADER);
  X[1] = reinterpret_cast<bf16*>(w + PE_HEADER + pe_align(count * ne * 2));
  const bool wide = m < n;
  const int s = wide ? m : n;  // side of the Gram matrix
  const size_t ss = (size_t)s * s;
  bf16* A = reinterpret_cast<bf16*>(w + PE_HEADER + 2 * pe_align(count * ne * 2));
  bf16* Bm = reinterpret_cast<bf16*>(w + PE_HEADER + 2 * pe_align(count * ne * 2) + pe_align(count * ss * 2));
  // the coefficients travel in the launch parameters (the host array is read here)
  HostFloats192 hc;
  std::memcpy(hc.v, coeffs, sizeof(float) * 3 * steps);
  store_floats_kernel<<<1, 64, 0, st>>>(hc, 3 * steps, cf, sumsq, count);
  CKL();
  const int grid = (int)std::max<long long>(1, std::min<long long>(((long long)ne + 255) / 256, dev_info().sms * 8LL / count + 1));
  sumsq_bf16_kernel<<<dim3(grid, count), 256, 0, st>>>(static_cast<const bf16*>(G), (long long)ne, sumsq, (long long)ne);
  CKL();
  scale_by_norm_bf16_kernel<<<dim3(grid, count), 256, 0, st>>>(static_cast<const bf16*>(G), X[0], (long long)ne, sumsq,
                                                               1e-7f, (long long)ne);
  CKL();
  // every product runs once over the whole batch (one launch, count slices)
  const long long bne = (long long)ne, bss = (long long)ss;
  bf16* cur = X[0];
  for (int t = 0; t < steps; ++t) {
    const float* a = cf + 3 * t;
    bf16* nxt = (t == steps - 1) ? static_cast<bf16*>(out) : X[(t + 1) & 1];
    // A = Gram matrix of the smaller side (X^T X for a tall X, X X^T for a wide one)
    if (!wide)
      TRY(gemm_batched(GPTB_BF16, {cur, n, true}, {cur, n, true}, n, n, m, epi(EPI_STORE, GPTB_BF16, A, n), count, bne,
                       bne, bss, 0, st));
    else
      TRY(gemm_batched(GPTB_BF16, {cur, n, false}, {cur, n, false}, m, m, n, epi(EPI_STORE, GPTB_BF16, A, m), count,
                       bne, bne, bss, 0, st));
    // B = b A + c A A   (A symmetric, so A A = A A^T)
    EpiParams eb = epi(EPI_RESID, GPTB_BF16, Bm, s, A, s);
    eb.alpha = a + 2;
    eb.beta = a + 1;
    TRY(gemm_batched(GPTB_BF16, {A, s, false}, {A, s, false}, s, s, s, eb, count, bss, bss, bss, bss, st));
    // X = a X + X B   (B symmetric); for a wide X the same update of X^T reads X = a X + B X
    EpiParams ex = epi(EPI_RESID, GPTB_BF16, nxt, n, cur, n);
    ex.beta = a;
    if (!wide)
      TRY(gemm_batched(GPTB_BF16, {cur, n, false}, {Bm, s, false}, m, n, n, ex, count, bne, bss, bne, bne, st));
    else
      TRY(gemm_batched(GPTB_BF16, {Bm, s, false}, {cur, n, true}, m, n, m, ex, count, bss, bne, bne, bne, st));
    cur = nxt;
  }
  return GPTB_OK;
}
}  // namespace

extern "C" {

int gptb_polar_express(const void* G, void* out, int m, int n, const float* coeffs, int steps, void* workspace,
                       size_t workspace_bytes, gptb_stream_t stream) {
  if (!G || !out || !coeffs || !workspace || m <= 0 || n <= 0 || m % 8 || n % 8 || steps < 1 || steps > 64)
    return GPTB_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GPTB_ERR_INVALID_ARG;
  const size_t ne = (size_t)m * n;
  {
    const uintptr_t a = reinterpret_cast<uintptr_t>(G), b = reinterpret_cast<uintptr_t>(out);
    if (a < b + ne * 2 && b < a + ne * 2) return GPTB_ERR_INVALID_ARG;  // out overlaps G
  }
  if (workspace_bytes < gptb_polar_express_workspace_bytes(m, n, steps)) return GPTB_ERR_WORKSPACE;
  if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  return polar_express_impl(G, out, m, n, 1, coeffs, steps, static_cast<uint8_t*>(workspace),
                            reinterpret_cast<cudaStream_t>(stream));
}

// Muon workspace for `count` matrices: the batched Polar Express workspace,
// the bf16 inputs u and outputs o, per-row step sizes, two sums per matrix
size_t muon_bytes(int count, int m, int n, int steps) {
  const size_t pe = pe_bytes(count, m, n, steps);
  if (pe == 0) return 0;
  return pe + 2 * pe_align((size_t)count * m * n * 2) + pe_align((size_t)count * m * 4) + pe_align((size_t)count * 8);
}

size_t gptb_muon_workspace_bytes(int m, int n, int steps) { return muon_bytes(1, m, n, steps); }
size_t gptb_muon_batched_workspace_bytes(int count, int m, int n, int steps) { return muon_bytes(count, m, n, steps); }

// One Muon step on `count` matrices of m x n (pointer arrays on the host)
int muon_impl(int count, float* const* w, void* const* w_bf16, const float* const* g, float* const* buf,
              float* const* v, int m, int n, const float* coeffs, int steps, float lr, float mu, float beta2,
              float weight_decay, void* workspace, size_t workspace_bytes, cudaStream_t st) {
  if (count <= 0 || count > PE_MAX_BATCH || !w || !g || !buf || !v || !coeffs || !workspace || m <= 0 || n <= 0 ||
      m % 8 || n % 8 || steps < 1 || steps > 64)
    return GPTB_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!w[i] || !g[i] || !buf[i] || !v[i]) return GPTB_ERR_INVALID_ARG;
    if (!aligned16(w[i]) || !aligned16(g[i]) || !aligned16(buf[i]) ||
        (w_bf16 && w_bf16[i] && (reinterpret_cast<uintptr_t>(w_bf16[i]) & 7u)))
      return GPTB_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GPTB_ERR_INVALID_ARG;
  if (workspace_bytes < muon_bytes(count, m, n, steps)) return GPTB_ERR_WORKSPACE;
  if (dev_info().cc_major != 10) return GPTB_ERR_UNSUPPORTED;
  const size_t ne = (size_t)m * n;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t pe = pe_bytes(count, m, n, steps);
  bf16* u = reinterpret_cast<bf16*>(ws + pe);
  bf16* o = reinterpret_cast<bf16*>(ws + pe + pe_align(count * ne * 2));
  float* step = reinterpret_cast<float*>(ws + pe + 2 * pe_align(count * ne * 2));
  float* sums = reinterpret_cast<float*>(ws + pe + 2 * pe_align(count * ne * 2) + pe_align((size_t)count * m * 4));
  const long long n4 = (long long)ne / 4;  // m, n multiples of 8
  const int grid = (int)std::max<long long>(1, std::min<long long>((n4 + 255) / 256, dev_info().sms * 8LL));
  // momentum (Nesterov): buf = mu buf + g, u = g + mu buf (bf16), into the batch's slices
  for (int i = 0; i < count; ++i) {
    muon_momentum_kernel<<<grid, 256, 0, st>>>(g[i], buf[i], u + i * ne, n4, mu, sums + 2 * i);
    CKL();
  }
  TRY(polar_express_impl(u, o, m, n, count, coeffs, steps, ws, st));
  // NorMuon: per-row second moment and step size, then the norm-keeping scale and the update
  for (int i = 0; i < count; ++i) {
    normuon_rows_kernel<<<grid_rows(m), EW_THREADS, 0, st>>>(o + i * ne, m, n, v[i], beta2, step + (size_t)i * m,
                                                             sums + 2 * i);
    CKL();
    muon_apply_kernel<<<grid, 256, 0, st>>>(w[i], static_cast<bf16*>(w_bf16 ? w_bf16[i] : nullptr), o + i * ne,
                                            step + (size_t)i * m, sums + 2 * i, m, n, lr, weight_decay);
    CKL();
  }
  return GPTB_OK;
}

int gptb_muon_step(float* w, void* w_bf16, const float* g, float* buf, float* v, int m, int n, const float* coeffs,
                   int steps, float lr, float mu, float beta2, float weight_decay, void* workspace,
                   size_t workspace_bytes, gptb_stream_t stream) {
  void* wb[1] = {w_bf16};
  return muon_impl(1, &w, w_bf16 ? wb : nullptr, &g, &buf, &v, m, n, coeffs, steps, lr, mu, beta2, weight_decay,
                   workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int gptb_muon_step_batched(int count, float* const* w, void* const* w_bf16, const float* const* g, float* const* buf,
                           float* const* v, int m, int n, const float* coeffs, int steps, float lr, float mu,
                           float beta2, float weight_decay, void* workspace, size_t workspace_bytes,
                           gptb_stream_t stream) {
  return muon_impl(count, w, w_bf16, g, buf, v, m, n, coeffs, steps, lr, mu, beta2, weight_decay, workspace,
                   workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

// --------------------------------------------------------------- decode --

size_t gptb_decode_workspace_bytes(int B, int H, int T_max) {
  if (B < 0 || H <= 0 || T_max <= 0) return 0;
  return (size_t)B * H * decode_pieces(T_max) * DEC_PART * sizeof(float) + 256;
}

int gptb_decode_attention(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, void* o,
                          float* lse, int B, int H, int Hkv, int T_max, int window, void* workspace,
                          size_t workspace_bytes, gptb_stream_t stream) {
  if (!q || !k_cache || !v_cache || !lens || !o || B < 0 || H <= 0 || Hkv <= 0 || H % Hkv || T_max <= 0)
    return GPTB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return GPTB_ERR_INVALID_ARG;
  if (B == 0) return GPTB_OK;
  if (H / Hkv > DEC_MAX_G) return GPTB_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace)) return GPTB_ERR_INVALID_ARG;
  if (workspace_bytes < gptb_decode_workspace_bytes(B, H, T_max)) return GPTB_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(workspace);
  // the K and V caches as [B*T_max, Hkv*128] bf16 matrices: K in two 64-column
  // boxes of DEC_SPLIT rows with a 128-byte swizzle, V in one unswizzled box of
  // DEC_SPLIT rows x 128 columns
  CUtensorMap tk, tv;
  {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GPTB_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)Hkv * DEC_HD, (cuuint64_t)B * T_max};
    cuuint64_t strides[1] = {(cuuint64_t)Hkv * DEC_HD * 2};
    cuuint32_t boxk[2] = {64, DEC_SPLIT};
    cuuint32_t boxv[2] = {DEC_HD, DEC_SPLIT};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k_cache), dims, strides, boxk, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTB_ERR_CUDA;
    if (fn(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(v_cache), dims, strides, boxv, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTB_ERR_CUDA;
  }
  const long long items = (long long)B * Hkv * decode_pieces(T_max);
  if (items > INT_MAX) return GPTB_ERR_UNSUPPORTED;
  const int grid = (int)std::min<long long>(items, std::max(1, dev_info().sms));  // persistent
  CK(cudaFuncSetAttribute(decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DEC_SMEM));
  decode_split_kernel<<<grid, DEC_THREADS, DEC_SMEM, st>>>(tk, tv, static_cast<const bf16*>(q), lens, part, H, Hkv,
                                                            T_max, window, (int)items);
  CKL();
  decode_combine_kernel<<<B * H, DEC_HD, 0, st>>>(part, lens, static_cast<bf16*>(o), lse, H, T_max);
  CKL();
  return GPTB_OK;
}

int gptb_cast_f32_bf16(const float* x, void* y, long long n, float scale, gptb_stream_t stream) {
  if (!x || !y || n < 0) return GPTB_ERR_INVALID_ARG;
  if (n == 0) return GPTB_OK;
  const int grid = (int)std::max<long long>(1, std::min<long long>((n + 255) / 256, dev_info().sms * 8LL));
  cast_f32_bf16_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, static_cast<bf16*>(y), n, scale);
  CKL();
  return GPTB_OK;
}

int gptb_cast_bf16_f32(const void* x, float* y, long long n, float scale, gptb_stream_t stream) {
  if (!x || !y || n < 0) return GPTB_ERR_INVALID_ARG;
  if (n == 0) return GPTB_OK;
  const int grid = (int)std::max<long long>(1, std::min<long long>((n + 255) / 256, dev_info().sms * 8LL));
  cast_bf16_f32_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<const bf16*>(x), y, n,
                                                                                  scale);
  CKL();
  return GPTB_OK;
}

int gptb_device_error(gptb_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GPTB_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return GPTB_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return GPTB_ERR_CUDA;
    return (v & 0xf00) == 0x200 ? GPTB_ERR_BAD_INPUT : GPTB_ERR_TIMEOUT;
  }
  return GPTB_OK;
}

int gptb_probe_bounded_wait(unsigned long long limit_ns, gptb_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned long long prev = 0;
  if (cudaMemcpyFromSymbol(&prev, g_wait_limit_ns, sizeof(prev)) != cudaSuccess) return GPTB_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_wait_limit_ns, &limit_ns, sizeof(limit_ns)) != cudaSuccess) return GPTB_ERR_CUDA;
  wait_probe_kernel<<<1, 32, 0, st>>>();
  LAUNCHED();
  const bool launched = cudaPeekAtLastError() == cudaSuccess;
  const int rc = launched ? gptb_device_error(stream) : GPTB_ERR_CUDA;
  cudaMemcpyToSymbol(g_wait_limit_ns, &prev, sizeof(prev));
  int res = -1;
  cudaMemcpyFromSymbol(&res, g_probe_result, sizeof(res));
  if (rc == GPTB_ERR_TIMEOUT && res != 0) return GPTB_ERR_CUDA;  // the kernel must have seen the expiry
  return rc;
}

int gptb_set_wait_limit_ns(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns)) == cudaSuccess ? GPTB_OK : GPTB_ERR_CUDA;
}

void gptb_reset_counters(void) {
  g_launches.store(0);
  std::lock_guard<std::mutex> lk(g_timing_mu);
  for (auto& t : g_timed) {
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_timed.clear();
}

long long gptb_launch_count(void) { return g_launches.load(); }

int gptb_set_gemm_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  g_timing = enable != 0;
  return GPTB_OK;
}

int gptb_gemm_timing(double* ms, double* flops, double* ms_fp8, double* flops_fp8, long long* launches) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  double tf = 0, tf8 = 0;
  // every launch as [start, end] on one time base (the first launch's start
  // event); the device time of the GEMMs is the union of these intervals: the
  // sum of the durations when no two overlap, each instant counted once when
  // launches on two streams (the bf16 backward's weight gradients) run together
  std::vector<std::pair<double, double>> iv, iv8;
  iv.reserve(g_timed.size());
  for (auto& t : g_timed) {
    if (cudaEventSynchronize(t.b) != cudaSuccess) return GPTB_ERR_CUDA;
    float e0 = 0.f, e1 = 0.f;
    if (cudaEventElapsedTime(&e0, g_timed[0].a, t.a) != cudaSuccess) return GPTB_ERR_CUDA;
    if (cudaEventElapsedTime(&e1, g_timed[0].a, t.b) != cudaSuccess) return GPTB_ERR_CUDA;
    iv.push_back({e0, e1});
    tf += t.flops;
    if (t.fp8) {
      iv8.push_back({e0, e1});
      tf8 += t.flops;
    }
  }
  auto covered = [](std::vector<std::pair<double, double>>& v) {
    std::sort(v.begin(), v.end());
    double total = 0, lo = 0, hi = 0;
    bool open = false;
    for (const auto& p : v) {
      if (!open || p.first > hi) {
        if (open) total += hi - lo;
        lo = p.first;
        hi = p.second;
        open = true;
      } else {
        hi = std::max(hi, p.second);
      }
    }
    if (open) total += hi - lo;
    return total;
  };
  const double tms = covered(iv), tms8 = covered(iv8);
  if (ms) *ms = tms;
  if (flops) *flops = tf;
  if (ms_fp8) *ms_fp8 = tms8;
  if (flops_fp8) *flops_fp8 = tf8;
  if (launches) *launches = (long long)g_timed.size();
  return GPTB_OK;
}

const char* gptb_error_string(int code) {
  switch (code) {
    case GPTB_OK: return "ok";
    case GPTB_ERR_INVALID_ARG: return "invalid argument";
    case GPTB_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case GPTB_ERR_CUDA: return "CUDA error";
    case GPTB_ERR_TIMEOUT: return "bounded device wait expired";
    case GPTB_ERR_WORKSPACE: return "workspace too small";
    case GPTB_ERR_BAD_INPUT: return "invalid input data found on the device (a target outside [0, vocab))";
    default: return "unknown error";
  }
}

}  // extern "C"

// ======================================================= no-alloc lm_head ==
// lm_head_xent for callers that cannot allocate device memory: its scratch
// (one chunk of logits, the chunk's softmax statistics, and the per-row
// losses) lives in this file-scope device array instead of a caller-provided
// workspace.  Every GPU that loads the library holds the array until the
// process exits.
namespace {

constexpr size_t NOALLOC_LOGITS_BYTES = size_t(8) << 20;  // logits of one row chunk
constexpr size_t NOALLOC_PART_BYTES = size_t(1) << 20;    // per-(row, tile) statistics of the chunk
constexpr long long NOALLOC_MAX_ROWS = 65536;             // B*T limit (row losses; z at the target and
                                                          // the log-sum-exp of a chunk's rows)
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[NOALLOC_LOGITS_BYTES + NOALLOC_PART_BYTES + 3 * NOALLOC_MAX_ROWS * 4];

// Device address of g_noalloc_scratch on the current device (host code only
// sees a host-side stand-in under the name).  Looked up on every call, so a
// module reloaded at another address after a context teardown is still found.
int noalloc_scratch(unsigned char** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
    cudaGetLastError();
    return GPTB_ERR_CUDA;
  }
  *out = static_cast<unsigned char*>(p);
  return GPTB_OK;
}

}  // namespace

extern "C" int lm_head_xent_noalloc(const gptb_config* cfg, const void* h, const void* w_lm, const int32_t* targets,
                                    float* loss_out, void* dh, float* dw_lm, gptb_stream_t stream) {
  TRY(check_config(cfg));
  if (!h || !w_lm || !targets || !loss_out || !dh || !dw_lm) return GPTB_ERR_INVALID_ARG;
  const Dims m = dims_of(*cfg);
  if (m.fp8_lm) return GPTB_ERR_UNSUPPORTED;  // its FP8 copies of hf and W_lm need a workspace
  if (m.N > NOALLOC_MAX_ROWS) return GPTB_ERR_WORKSPACE;
  long long rows = (long long)(NOALLOC_LOGITS_BYTES / ((size_t)m.V * m.esz));
  rows = std::min<long long>(rows, (long long)(NOALLOC_PART_BYTES / (lm_tiles(m.V) * sizeof(float2))));
  if (rows < 1) return GPTB_ERR_WORKSPACE;
  unsigned char* base = nullptr;
  TRY(noalloc_scratch(&base));
  LmWs lw;
  lw.logits = base;
  lw.part = reinterpret_cast<float2*>(base + NOALLOC_LOGITS_BYTES);
  lw.row_loss = reinterpret_cast<float*>(base + NOALLOC_LOGITS_BYTES + NOALLOC_PART_BYTES);
  lw.zy = lw.row_loss + NOALLOC_MAX_ROWS;
  lw.lse = lw.zy + NOALLOC_MAX_ROWS;
  lw.chunk = (int)std::min<long long>(rows, m.N);
  lw.h8 = lw.w8 = lw.dz8 = nullptr;
  lw.amx = nullptr;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == GPTB_F32)
    return lm_head_impl<float>(*cfg, (const float*)h, (const float*)w_lm, targets, loss_out, (float*)dh, dw_lm, lw, st);
  return lm_head_impl<bf16>(*cfg, (const bf16*)h, (const bf16*)w_lm, targets, loss_out, (bf16*)dh, dw_lm, lw, st);
}
