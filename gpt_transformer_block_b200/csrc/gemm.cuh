// GEMMs of the block: C = A * B^T with A [M,K], B [N,K] and a fused epilogue.
//
// Every projection of the block is an nn.Linear (y = x W^T with W [out,in]),
// so the three products of training map onto one kernel with per-operand
// majorness:
//   forward   y  = x  W^T : A = x  (K-major),  B = W  (K-major)
//   dgrad     dx = dy W   : A = dy (K-major),  B = W  (N-major, W is [K,N])
//   wgrad     dW = dy^T x : A = dy (M-major),  B = x  (N-major)
//
// bf16 / e4m3 path (tcgen05): persistent, warp-specialised kernel.
//   warp 0   TMA producer (128-byte swizzled tiles, 4-stage mbarrier ring)
//   warp 1   TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-5 epilogue: tcgen05.ld 32 lanes x 64 columns per step, fused
//             elementwise op into a swizzled per-warp smem tile, written by
//             TMA bulk stores (bf16) or TMA bulk reduce-add (fp32 weight
//             gradients); residual / saved-u inputs arrive by TMA loads
//   Tile 128 x 256 per CTA, two TMEM accumulators (2 x 256 columns) so the
//   epilogue of tile i overlaps the MMAs of tile i+1.  Pair form: a cluster
//   of two CTAs runs M = 256 tcgen05.mma (cta_group::2) on a 256 x 256 tile,
//   each CTA staging half of A and half of B (loads without multicast; the
//   odd CTA's loads complete on the even CTA's barriers), so each SM reads a
//   third less operand data per FLOP.  Split-K over the K blocks is used for
//   weight gradients (long K, few tiles); partial sums meet in the fp32
//   gradient through TMA reduce-adds.
// fp32 path (SIMT, FFMA): a plain tiled kernel with the same epilogues, for
//   the fp32 configuration whose 1e-5 tolerance tensor-core fp32 (tf32)
//   inputs cannot meet.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace gptb {

enum EpiKind : int {
  EPI_STORE = 0,      // out = alpha*acc
  EPI_RESID = 1,      // out = beta*aux + alpha*acc           (residual add)
  EPI_RELU2 = 2,      // out = relu(alpha*acc)^2              (MLP activation)
  EPI_DRELU2 = 3,     // out = alpha*acc * 2*sqrt(aux)          (aux = saved relu(u)^2:
                      //   d relu(u)^2 / du = 2 relu(u) = 2 sqrt(relu(u)^2), so u
                      //   itself need not be kept)
  EPI_ACCUM_F32 = 4,  // out(f32) += alpha*acc, atomic          (weight grads)
  EPI_QKV = 5,        // q,k heads: rope(rmsnorm(acc)) + saved rstd; v heads:
                      // acc + 3*sigmoid(z) * VE[idx] (value-embedding layers)
  EPI_DOT = 6,        // out = alpha*acc (bf16) and, per row and 128-column
                      // group h, rowdot[b, h, t] = sum(out * aux) (aux = the
                      // attention output o, out = dO: the backward's D term)
  EPI_XENT = 7,       // out = z = alpha*acc (bf16 logits) and, per row and
                      // 256-column tile n, the softmax statistics of the
                      // tile: xent_part[row, n] = (max z, sum exp(z - max));
                      // xent_zy[row] = z[row, targets[row]] (fp32)
};

struct EpiParams {
  int kind;
  int out_f32;  // element type of out/out2/aux: 1 = float, 0 = bf16
  void* out;
  long long ldo;
  const void* aux;
  long long ld_aux;
  void* out2;
  long long ldo2;
  const float* alpha;  // device scalar or nullptr (= 1)
  const float* beta;   // EPI_RESID: device scale of aux, or nullptr (= 1)
  // e4m3 operands: per-tensor amax of A and B; the product is rescaled by
  // (amax_a / 448) * (amax_b / 448), the inverse of the two quantisation scales
  const float* amax_a;
  const float* amax_b;
  int a_e5m2;  // A operand in e5m2 (its scale 57344/amax; B is always e4m3, 448/amax)
  // EPI_QKV: per-head QK RMSNorm + RoPE and the value-embedding add
  const float2* rope;     // [T, 64] (cos, sin)
  float* rstd_qk;         // [M, H + Hkv]
  const bf16* ve_table;   // [V, Hkv*128] or nullptr
  const int32_t* idx;     // [M] token ids
  const float* sg;        // [M, Hkv] sigmoid of the gate logits
  int T, H, Hkv;
  float eps;
  float* rowdot;          // EPI_DOT: [B, H, T] fp32
  // EPI_XENT: per-(row, 256-column tile) statistics, row stride xent_nt
  float2* xent_part;
  int xent_nt;
  const int32_t* targets;  // [M] class ids; ids outside [0, N) match no column
  float* xent_zy;          // [M]
  // EPI_RELU2 / EPI_DRELU2: max |out| of the stored values (FP8 amax), or nullptr
  unsigned int* amax_out;
};

__device__ __forceinline__ float epi_beta(const EpiParams& ep) { return ep.beta ? *ep.beta : 1.f; }
__device__ __forceinline__ float epi_alpha(const EpiParams& ep) {
  float a = ep.alpha ? *ep.alpha : 1.f;
  if (ep.amax_a)
    a *= (fmaxf(*ep.amax_a, 1e-12f) / (ep.a_e5m2 ? 57344.f : 448.f)) * (fmaxf(*ep.amax_b, 1e-12f) / 448.f);
  return a;
}

// ---------------------------------------------------------------- epilogue
template <class T>
__device__ __forceinline__ void epi_store8_t(const EpiParams& ep, long long r, int c, float (&v)[8]) {
  T* o = reinterpret_cast<T*>(ep.out) + r * ep.ldo + c;
  switch (ep.kind) {
    case EPI_RESID: {
      float a[8];
      load8(reinterpret_cast<const T*>(ep.aux) + r * ep.ld_aux + c, a);
      const float beta = epi_beta(ep);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = fmaf(beta, a[i], v[i]);
      store8(o, v);
    } break;
    case EPI_RELU2: {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = fmaxf(v[i], 0.f);
        v[i] = t * t;
      }
      store8(o, v);
    } break;
    case EPI_DRELU2: {
      float a[8];
      load8(reinterpret_cast<const T*>(ep.aux) + r * ep.ld_aux + c, a);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= 2.f * sqrtf(fmaxf(a[i], 0.f));
      store8(o, v);
    } break;
    default:
      store8(o, v);
  }
}

__device__ __forceinline__ void epi_apply8(const EpiParams& ep, long long r, int c, float (&v)[8]) {
  if (ep.kind == EPI_ACCUM_F32) {
    float* o = reinterpret_cast<float*>(ep.out) + r * ep.ldo + c;
    atomicAdd(reinterpret_cast<float4*>(o), make_float4(v[0], v[1], v[2], v[3]));
    atomicAdd(reinterpret_cast<float4*>(o + 4), make_float4(v[4], v[5], v[6], v[7]));
  } else if (ep.out_f32) {
    epi_store8_t<float>(ep, r, c, v);
  } else {
    epi_store8_t<bf16>(ep, r, c, v);
  }
}

template <class T>
__device__ __forceinline__ void epi_scalar_t(const EpiParams& ep, long long r, int c, float v) {
  T* o = reinterpret_cast<T*>(ep.out) + r * ep.ldo + c;
  switch (ep.kind) {
    case EPI_RESID: *o = from_f<T>(fmaf(epi_beta(ep), to_f(reinterpret_cast<const T*>(ep.aux)[r * ep.ld_aux + c]), v)); break;
    case EPI_RELU2: {
      const float t = fmaxf(v, 0.f);
      *o = from_f<T>(t * t);
    } break;
    case EPI_DRELU2:
      *o = from_f<T>(v * 2.f * sqrtf(fmaxf(to_f(reinterpret_cast<const T*>(ep.aux)[r * ep.ld_aux + c]), 0.f)));
      break;
    default: *o = from_f<T>(v);
  }
}
__device__ __forceinline__ void epi_apply1(const EpiParams& ep, long long r, int c, float v) {
  if (ep.kind == EPI_ACCUM_F32) atomicAdd(reinterpret_cast<float*>(ep.out) + r * ep.ldo + c, v);
  else if (ep.out_f32) epi_scalar_t<float>(ep, r, c, v);
  else epi_scalar_t<bf16>(ep, r, c, v);
}

// ------------------------------------------------------ tcgen05 kernel ----
constexpr int TC_BM = 128;   // rows of A (and TMEM lanes of D) per CTA
constexpr int TC_BN = 256;   // columns of D per CTA (one TMEM accumulator)
constexpr int TC_THREADS = 192;
constexpr int TC_GROUP_M = 8;

// per epilogue warp: four 32-row x 128-byte staging tiles (two output tiles
// written alternately, so a chunk's store overlaps the next chunk, and two
// input tiles of the residual / saved activation, loaded one chunk ahead)
constexpr int TC_EPI_TILE = 4096;
constexpr int TC_EPI_BYTES = 4 * 4 * TC_EPI_TILE;

// Tile shape of the two kernel forms.
//   single: one CTA computes a 128 x 256 tile (A 128 rows, B 256 rows per stage)
//   pair:   a cluster of two CTAs computes a 256 x 256 tile with M = 256
//           tcgen05.mma issued by the even CTA; each CTA stages its own 128
//           rows of A and 128 rows of B (so each SM reads 32 KB of operands
//           per 64-deep K block instead of 48 KB) and holds its 128 rows of D
template <bool PAIR> struct TcShape {
  static constexpr int TILE_M = PAIR ? 256 : 128;
  static constexpr int B_ROWS = PAIR ? 128 : 256;
  static constexpr int STAGES = PAIR ? 5 : 3;
  static constexpr int A_BYTES = TC_BM * 128;
  static constexpr int B_BYTES = B_ROWS * 128;
  // stages * (A + B) + epilogue staging + barriers + 1 KB alignment slack
  static constexpr int SMEM = STAGES * (A_BYTES + B_BYTES) + TC_EPI_BYTES + 256 + 1024;
  static_assert(SMEM <= 232448, "GEMM shared memory above the per-CTA limit");
};

// unit u -> (split-K part, batch entry, tile row, tile column); the tiles of
// one (split, batch entry) are walked in groups of TC_GROUP_M tile rows
__device__ __forceinline__ void tc_unit_coords(int u, int tiles_m, int tiles_n, int nbatch, int& tm, int& tn,
                                               int& split, int& bz) {
  const int tiles = tiles_m * tiles_n;
  const int sb = u / tiles;
  split = sb / nbatch;
  bz = sb - split * nbatch;
  const int t = u - sb * tiles;
  const int per_group = TC_GROUP_M * tiles_n;
  const int g = t / per_group;
  const int first_m = g * TC_GROUP_M;
  const int gsize = min(tiles_m - first_m, TC_GROUP_M);
  const int r = t - g * per_group;
  tm = first_m + r % gsize;
  tn = r / gsize;
}

// EPI_QKV for one 128-column head of the tile (one TMEM lane quarter = 32
// rows, thread = row): q/k heads get the per-head RMSNorm (rstd saved) and the
// rotation of the pairs (j, j+64) by the row's position; v heads get
// + 3*sigmoid(z)*VE[idx] on value-embedding layers.  Columns 0..63 go to
// staging tile stg0, 64..127 to stg1 (32 rows x 128 bytes, 128-byte swizzle).
__device__ __forceinline__ void epi_qkv_head(const EpiParams& ep, uint32_t ta, uint8_t* stg0, uint8_t* stg1, int lane,
                                             float alpha, int head, int grow, bool rv) {
  const int swz = lane & 7;
  uint8_t* p0 = stg0 + lane * 128;
  uint8_t* p1 = stg1 + lane * 128;
  if (head < ep.H + ep.Hkv) {
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(ta + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(v[i]) * alpha;
        ss = fmaf(x, x, ss);
      }
    }
    const float rr = rsqrtf(ss * (1.f / 128.f) + ep.eps);
    const float sc = alpha * rr;
    const float2* cs = ep.rope + (long long)(rv ? grow % ep.T : 0) * 64;
#pragma unroll
    for (int j0 = 0; j0 < 64; j0 += 32) {
      uint32_t a1[32], a2[32];
      tmem_ld_32x32b_x32(ta + j0, a1);
      tmem_ld_32x32b_x32(ta + 64 + j0, a2);
      tmem_ld_wait();
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float y1[8], y2[8];
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const float4 c2 = *reinterpret_cast<const float4*>(cs + j0 + g * 8 + k);  // (cos, sin) of two pairs
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float c = h ? c2.z : c2.x, sn = h ? c2.w : c2.y;
            const float x1 = __uint_as_float(a1[g * 8 + k + h]) * sc, x2 = __uint_as_float(a2[g * 8 + k + h]) * sc;
            y1[k + h] = x1 * c - x2 * sn;
            y2[k + h] = x1 * sn + x2 * c;
          }
        }
        const int chunk = (j0 >> 3) + g;
        store8(reinterpret_cast<bf16*>(p0 + ((chunk ^ swz) << 4)), y1);
        store8(reinterpret_cast<bf16*>(p1 + ((chunk ^ swz) << 4)), y2);
      }
    }
    if (rv) ep.rstd_qk[(long long)grow * (ep.H + ep.Hkv) + head] = rr;
  } else {
    const int kv = head - ep.H - ep.Hkv;
    const bool ve = ep.ve_table != nullptr && rv;
    const float gate = ve ? 3.f * ep.sg[(long long)grow * ep.Hkv + kv] : 0.f;
    const bf16* e = ve ? ep.ve_table + (long long)ep.idx[grow] * ep.Hkv * 128 + kv * 128 : nullptr;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(ta + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(v[g * 8 + i]) * alpha;
        if (ve) {
          float ev[8];
          load8(e + c * 32 + g * 8, ev);
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] = fmaf(gate, ev[i], y[i]);
        }
        const int chunk = (c & 1) * 4 + g;
        store8(reinterpret_cast<bf16*>((c < 2 ? p0 : p1) + ((chunk ^ swz) << 4)), y);
      }
    }
  }
}

// The epilogue warps' role for one epilogue kind (the kind is a template
// parameter, so each kind's per-chunk loop is compact straight-line code).
template <int KIND, bool PAIR>
__device__ __forceinline__ void tc_epilogue(const EpiParams& ep, const CUtensorMap* tmO_, const CUtensorMap* tmX_,
                                            uint32_t tmem_base, uint8_t* sEpi, uint64_t* aux_bar, uint64_t* tfull,
                                            uint64_t* tempty, volatile int* abort_flag, int M, int N, int unit0,
                                            int ustep, int units, int tiles_m, int tiles_n, int nbatch, int warp,
                                            int lane, uint32_t rank) {
  using SH = TcShape<PAIR>;
  const CUtensorMap& tmO = *tmO_;
  const CUtensorMap& tmX = *tmX_;
  const int q = warp & 3;  // TMEM lane quarter this warp may access
  uint8_t* ebuf = sEpi + (warp - 2) * (4 * TC_EPI_TILE);  // this warp's four staging tiles
  uint64_t* abar = &aux_bar[(warp - 2) * 2];
  constexpr bool has_aux = (KIND == EPI_RESID || KIND == EPI_DRELU2 || KIND == EPI_DOT);
  constexpr bool acc32 = (KIND == EPI_ACCUM_F32);
  const int swz = (lane & 7);  // 16-byte chunk swizzle of this lane's 128-byte staging row
  // Staging tiles: bf16 output chunks alternate between tiles 0 and 1, and
  // the input chunks (residual, saved activation, O) between tiles 2 and 3;
  // fp32 chunks and the q/k/v heads take two tiles each, alternating
  // between tiles 0-1 and 2-3.  Every chunk commits one bulk group, so
  // waiting until at most one group is still reading frees the tile(s) of
  // the chunk before last.
  uint32_t ns = 0;          // bulk groups committed by this warp
  uint32_t na = 0, nw = 0;  // input-tile loads issued / consumed by this warp
  auto chunks_of = [&](int tn_) { return min(TC_BN / 64, (N - tn_ * TC_BN + 63) / 64); };
  // load the input chunk cc_ of unit u_ into the next input tile (lane 0; the count advances on every lane)
  auto issue_aux = [&](int u_, int cc_) {
    if (lane == 0) {
      int tm_, tn_, sp_, bz_;
      tc_unit_coords(u_, tiles_m, tiles_n, nbatch, tm_, tn_, sp_, bz_);
      uint64_t* bar = &abar[na & 1u];
      mbar_arrive_expect_tx(bar, TC_EPI_TILE);
      tma_load_3d(ebuf + (2 + (na & 1u)) * TC_EPI_TILE, &tmX, bar, tn_ * TC_BN + cc_ * 64,
                  tm_ * SH::TILE_M + (int)rank * TC_BM + q * 32, bz_);
    }
    ++na;
  };
  if (has_aux && unit0 < units) issue_aux(unit0, 0);
  int acc = 0;
  uint32_t acc_phase = 0;
  const float alpha = epi_alpha(ep);
  const float beta = epi_beta(ep);
  float oam = 0.f;  // max |out| stored by this thread (FP8 amax of EPI_RELU2 / EPI_DRELU2 outputs)
  bool ok = true;
  for (int u = unit0; u < units && ok; u += ustep) {
    int tm, tn, split, bz;
    tc_unit_coords(u, tiles_m, tiles_n, nbatch, tm, tn, split, bz);
    if (!mbar_wait_warp(&tfull[acc], acc_phase, abort_flag, ERRW_TIMEOUT_EPILOGUE)) break;
    tc_fence_after();
    const int row0 = tm * SH::TILE_M + (int)rank * TC_BM + q * 32;
    if constexpr (KIND == EPI_QKV) {
#pragma unroll 1
      for (int hb = 0; hb < TC_BN / 128; ++hb) {
        const int col0 = tn * TC_BN + hb * 128;
        if (col0 >= N) break;  // warp-uniform
        uint8_t* st0 = ebuf + (ns & 1u) * 2 * TC_EPI_TILE;
        if (lane == 0) bulk_wait_read1();
        __syncwarp();
        const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TC_BN + hb * 128);
        epi_qkv_head(ep, ta, st0, st0 + TC_EPI_TILE, lane, alpha, col0 / 128, row0 + lane, row0 + lane < M);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmO, st0, col0, row0, bz);
          tma_store_3d(&tmO, st0 + TC_EPI_TILE, col0 + 64, row0, bz);
          bulk_commit_group();
        }
        ++ns;
      }
    }
    float dsum = 0.f;  // EPI_DOT: this row's running sum over the current 128-column group
    // EPI_XENT: this row's running max and sum of exp2((z - max) * log2 e) over the tile
    float xm = -INFINITY, xs = 0.f;
    const int xy = (KIND == EPI_XENT && row0 + lane < M) ? ep.targets[row0 + lane] : -1;
    const int nch = (KIND == EPI_QKV) ? 0 : chunks_of(tn);
#pragma unroll 1
    for (int cc = 0; cc < nch; ++cc) {
      const int col0 = tn * TC_BN + cc * 64;
      const bool tail = col0 + 64 > N;  // warp-uniform: the last chunk of a ragged N
      uint32_t r0[32], r1[32];
      const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TC_BN + cc * 64);
      tmem_ld_32x32b_x32(ta, r0);
      tmem_ld_32x32b_x32(ta + 32, r1);
      if constexpr (has_aux) {
        // the next input chunk (of this tile, else of the next unit) goes
        // into the other input tile, read by the chunk before this one
        if (cc + 1 < nch) issue_aux(u, cc + 1);
        else if (u + ustep < units) issue_aux(u + ustep, 0);
      }
      // this chunk's output tile(s) are free once the bulk group of the chunk before last has read them
      if (lane == 0) bulk_wait_read1();
      __syncwarp();
      tmem_ld_wait();
      uint8_t* cur_in = ebuf + (2 + (nw & 1u)) * TC_EPI_TILE;
      if constexpr (has_aux) {
        if (!mbar_wait_warp(&abar[nw & 1u], (nw >> 1) & 1u, abort_flag, ERRW_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
        ++nw;
      }
      uint8_t* p0 = ebuf + (acc32 ? (ns & 1u) * 2 * TC_EPI_TILE : (ns & 1u) * TC_EPI_TILE) + lane * 128;
      uint8_t* p1 = acc32 ? p0 + TC_EPI_TILE : cur_in + lane * 128;
      float xml2 = 0.f;  // EPI_XENT: running max * log2 e after this chunk
      if constexpr (KIND == EPI_XENT) {
        // the chunk's max as eight independent chains (columns past N left out)
        float cm8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) cm8[j] = xm;
        if (!tail) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            cm8[i & 7] = fmaxf(cm8[i & 7], __uint_as_float(i < 32 ? r0[i] : r1[i - 32]) * alpha);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (col0 + i < N) cm8[i & 7] = fmaxf(cm8[i & 7], __uint_as_float(i < 32 ? r0[i] : r1[i - 32]) * alpha);
        }
#pragma unroll
        for (int j = 1; j < 8; ++j) cm8[0] = fmaxf(cm8[0], cm8[j]);
        const float cm = cm8[0];
        if (cm > xm) {  // rescale the sum to the new max (0 while the max was -inf)
          xs = (xm == -INFINITY) ? 0.f : xs * fast_exp2((xm - cm) * LOG2E);
          xm = cm;
        }
        xml2 = xm * LOG2E;
      }
      if constexpr (acc32) {
        // fp32: columns 0..31 -> tile 0, 32..63 -> tile 1 (32 x 128-byte rows each)
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          *reinterpret_cast<float4*>(p0 + ((g ^ swz) << 4)) =
              make_float4(__uint_as_float(r0[4 * g]) * alpha, __uint_as_float(r0[4 * g + 1]) * alpha,
                          __uint_as_float(r0[4 * g + 2]) * alpha, __uint_as_float(r0[4 * g + 3]) * alpha);
          *reinterpret_cast<float4*>(p1 + ((g ^ swz) << 4)) =
              make_float4(__uint_as_float(r1[4 * g]) * alpha, __uint_as_float(r1[4 * g + 1]) * alpha,
                          __uint_as_float(r1[4 * g + 2]) * alpha, __uint_as_float(r1[4 * g + 3]) * alpha);
        }
      } else {
        // bf16: 8 chunks of 8 columns; the input chunk (if any) has the same swizzle
        float xsum[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(g < 4 ? r0[g * 8 + i] : r1[(g - 4) * 8 + i]) * alpha;
          uint8_t* cp0 = p0 + ((g ^ swz) << 4);
          if constexpr (has_aux) {
            float a[8];
            load8(reinterpret_cast<const bf16*>(p1 + ((g ^ swz) << 4)), a);
            if constexpr (KIND == EPI_RESID) {
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = fmaf(beta, a[i], v[i]);
            } else if constexpr (KIND == EPI_DRELU2) {
              // 2 relu(u) = 2 sqrt(a) as a * rsqrt(a); a below the smallest
              // normal float (where the flushing rsqrt gives inf) counts as 0
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] *= (a[i] >= 1.17549435e-38f) ? 2.f * a[i] * fast_rsqrt(a[i]) : 0.f;
            } else {
              // the dot takes the values as stored (rounded to bf16)
#pragma unroll
              for (int i = 0; i < 8; ++i) dsum = fmaf(__bfloat162float(__float2bfloat16_rn(v[i])), a[i], dsum);
            }
          }
          if constexpr (KIND == EPI_XENT) {
            const int c8 = col0 + g * 8;
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) e[i] = fast_exp2(fmaf(v[i], LOG2E, -xml2));
            if (tail) {  // columns past N (the last tile's tail) do not take part
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (c8 + i >= N) e[i] = 0.f;
            }
            xsum[g] = ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
            if (xy >= c8 && xy < c8 + 8) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (xy == c8 + i) ep.xent_zy[row0 + lane] = v[i];
            }
          }
          if constexpr (KIND == EPI_RELU2) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float t = fmaxf(v[i], 0.f);
              v[i] = t * t;
            }
          }
          if ((KIND == EPI_RELU2 || KIND == EPI_DRELU2) && ep.amax_out && row0 + lane < M) {
            const int c8 = col0 + g * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (c8 + i < N) oam = fmaxf(oam, fabsf(v[i]));
          }
          store8(reinterpret_cast<bf16*>(cp0), v);
        }
        if constexpr (KIND == EPI_XENT)
          xs += ((xsum[0] + xsum[1]) + (xsum[2] + xsum[3])) + ((xsum[4] + xsum[5]) + (xsum[6] + xsum[7]));
      }
      if (KIND == EPI_DOT && (cc & 1)) {  // a 128-column group (one head) is complete
        const int row = row0 + lane;
        if (row < M) {
          const int bb = row / ep.T, t = row - bb * ep.T;
          ep.rowdot[((long long)bb * ep.H + col0 / 128) * ep.T + t] = dsum;
        }
        dsum = 0.f;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        uint8_t* t0 = p0 - lane * 128;
        if constexpr (acc32) {
          tma_reduce_add_3d(&tmO, t0, col0, row0, bz);
          tma_reduce_add_3d(&tmO, t0 + TC_EPI_TILE, col0 + 32, row0, bz);
        } else {
          tma_store_3d(&tmO, t0, col0, row0, bz);
        }
        bulk_commit_group();
      }
      ++ns;
    }
    // (a tile cut short by the N tail still covers at least one chunk)
    if (KIND == EPI_XENT && ok && row0 + lane < M)
      ep.xent_part[(long long)(row0 + lane) * ep.xent_nt + tn] = make_float2(xm, xs);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (PAIR) mbar_arrive_cluster(map_shared_rank(&tempty[acc], 0));
      else mbar_arrive(&tempty[acc]);
    }
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1u;
  }
  // input-tile loads still in flight (issued ahead of an abort) land before the CTA exits
  while (nw < na) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(&abar[nw & 1u], (nw >> 1) & 1u)) {
      if (globaltimer_ns() - t0 > 100000000ull) {
        record_error(ERRW_TIMEOUT_DRAIN);
        break;
      }
    }
    ++nw;
  }
  if (lane == 0) bulk_wait0();
  if ((KIND == EPI_RELU2 || KIND == EPI_DRELU2) && ep.amax_out) {
    oam = warp_max(oam);
    if (lane == 0) atomicMax(ep.amax_out, __float_as_uint(stored_abs_max_bf16(oam)));
  }
}

template <bool A_MN, bool B_MN, bool FP8, bool PAIR>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                   const __grid_constant__ CUtensorMap tmX, int M, int N, int K, int splits, int nbatch,
                   EpiParams ep) {
  using SH = TcShape<PAIR>;
  constexpr int STAGES = SH::STAGES;
  constexpr int ELEM = FP8 ? 1 : 2;
  constexpr int BK = 128 / ELEM;      // one 128-byte swizzle row of K (64 bf16 / 128 e4m3)
  constexpr int MMA_K = 32 / ELEM;    // K per tcgen05.mma (16 bf16 / 32 e4m3)
  constexpr int ATOM = BK;            // MN extent of one swizzle atom for MN-major operands
  constexpr int A_BYTES = SH::A_BYTES;
  constexpr int B_BYTES = SH::B_BYTES;
  constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;             // bytes landing in one CTA per stage
  constexpr uint32_t FULL_TX = PAIR ? 2 * STAGE_TX : STAGE_TX;  // bytes a stage's full barrier waits for
  constexpr uint32_t IDESC0 = make_idesc(SH::TILE_M, TC_BN, A_MN, B_MN, FP8);
  // kind::f8f6f4 A format (bits 7-9): 0 = e4m3, 1 = e5m2
  const uint32_t IDESC = IDESC0 | ((FP8 && ep.a_e5m2) ? (1u << 7) : 0u);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sEpi = sB + STAGES * B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + TC_EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* aux_bar = drain + 1;  // [8] two per epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux_bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pair: both CTAs of a cluster walk the same units; the even CTA (rank 0)
  // issues the MMAs and owns the stage and accumulator-drain barriers
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int ustep = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
  const int tiles_m = (M + SH::TILE_M - 1) / SH::TILE_M, tiles_n = (N + TC_BN - 1) / TC_BN;
  const int units = tiles_m * tiles_n * splits * nbatch;
  const int kb_total = (K + BK - 1) / BK;
  const int kb_per = (kb_total + splits - 1) / splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], PAIR ? 8 : 4);  // the epilogue warps of both CTAs drain an accumulator
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&aux_bar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if (PAIR) tmem_alloc_pair(tmem_slot, 512);
    else tmem_alloc(tmem_slot, 512);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with a load in flight, and the phase they complete
      bool ok = true;
      for (int u = unit0; u < units && ok; u += ustep) {
        int tm, tn, split, bz;
        tc_unit_coords(u, tiles_m, tiles_n, nbatch, tm, tn, split, bz);
        const int kb0 = split * kb_per, kb1 = min(kb_total, kb0 + kb_per);
        const int arow = tm * SH::TILE_M + (int)rank * TC_BM;      // this CTA's rows of A
        const int brow = tn * TC_BN + (int)rank * SH::B_ROWS;      // this CTA's rows of B
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, ERRW_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          // the even CTA arms its stage barrier for both CTAs' bytes; the odd
          // CTA's loads count down the same barrier (a count that goes below
          // zero before the arming is allowed: the phase needs the arrival)
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], FULL_TX);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          uint8_t* a = sA + stage * A_BYTES;
          uint8_t* b = sB + stage * B_BYTES;
          const int k0 = kb * BK;
          auto load = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
            if (PAIR) tma_load_3d_pair(dst, m, map_shared_rank(&full[stage], 0), c0, c1, bz);
            else tma_load_3d(dst, m, &full[stage], c0, c1, bz);
          };
          if (!A_MN) {
            load(a, &tmA, k0, arow);
          } else {
#pragma unroll
            for (int i = 0; i < TC_BM / ATOM; ++i) load(a + i * BK * 128, &tmA, arow + i * ATOM, k0);
          }
          if (!B_MN) {
            load(b, &tmB, k0, brow);
          } else {
#pragma unroll
            for (int i = 0; i < SH::B_ROWS / ATOM; ++i) load(b + i * BK * 128, &tmB, brow + i * ATOM, k0);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // after an abort, wait (bounded) for the loads this thread issued to land
      // before the CTA exits; a consumed stage's phase has already completed.
      // The odd CTA of a pair cannot wait on the even CTA's barriers: it gives
      // its loads a fixed 1 ms.
      if (!ok) {
        if (PAIR && rank != 0) {
          const unsigned long long t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 1000000ull) {
          }
        } else {
          for (int s2 = 0; s2 < STAGES; ++s2) {
            if (!(armed & (1u << s2))) continue;
            const uint32_t par = (armed_par >> s2) & 1u;
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[s2], par)) {
              if (globaltimer_ns() - t0 > 100000000ull) {
                record_error(ERRW_TIMEOUT_DRAIN);
                break;
              }
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += ustep) {
        int tm, tn, split, bz;
        tc_unit_coords(u, tiles_m, tiles_n, nbatch, tm, tn, split, bz);
        const int kb0 = split * kb_per, kb1 = min(kb_total, kb0 + kb_per);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, ERRW_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TC_BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, ERRW_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / MMA_K; ++k) {
            // K-major: advance 32 bytes along the swizzled row; MN-major: MMA_K rows of 128 bytes
            const uint64_t ad = A_MN ? smem_desc_sw128(a_addr + k * MMA_K * 128, BK * 128, 1024)
                                     : smem_desc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(b_addr + k * MMA_K * 128, BK * 128, 1024)
                                     : smem_desc_sw128(b_addr + k * 32, 16, 1024);
            const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
            if (PAIR) {
              if (FP8) mma_f8_ss_pair(d_tmem, ad, bd, IDESC, accum);
              else mma_bf16_ss_pair(d_tmem, ad, bd, IDESC, accum);
            } else {
              if (FP8) mma_f8_ss(d_tmem, ad, bd, IDESC, accum);
              else mma_bf16_ss(d_tmem, ad, bd, IDESC, accum);
            }
          }
          // the stage is free again in both CTAs once these MMAs have read it
          if (PAIR) mma_commit_pair_both(&empty[stage]);
          else mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR) mma_commit_pair_both(&tfull[acc]);
        else mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (*abort_flag) {
        // let every MMA this thread issued finish before TMEM is released
        if (PAIR) mma_commit_pair_local(drain);
        else mma_commit(drain);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0)) {
          if (globaltimer_ns() - t0 > 100000000ull) {
            record_error(ERRW_TIMEOUT_DRAIN);
            break;
          }
        }
      }
    }
  } else {
    // one code path per epilogue kind
    auto run = [&](auto kind) {
      tc_epilogue<decltype(kind)::value, PAIR>(ep, &tmO, &tmX, tmem_base, sEpi, aux_bar, tfull, tempty, abort_flag, M, N,
                                               unit0, ustep, units, tiles_m, tiles_n, nbatch, warp, lane, rank);
    };
    switch (ep.kind) {
      case EPI_STORE: run(std::integral_constant<int, EPI_STORE>{}); break;
      case EPI_RESID: run(std::integral_constant<int, EPI_RESID>{}); break;
      case EPI_RELU2: run(std::integral_constant<int, EPI_RELU2>{}); break;
      case EPI_DRELU2: run(std::integral_constant<int, EPI_DRELU2>{}); break;
      case EPI_ACCUM_F32: run(std::integral_constant<int, EPI_ACCUM_F32>{}); break;
      case EPI_QKV: run(std::integral_constant<int, EPI_QKV>{}); break;
      case EPI_DOT: run(std::integral_constant<int, EPI_DOT>{}); break;
      case EPI_XENT: run(std::integral_constant<int, EPI_XENT>{}); break;
      default: break;
    }
  }
  tc_fence_before();
  __syncthreads();
  // pair: neither CTA leaves (or frees its tensor memory) while the other may
  // still arrive on its barriers
  if (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------- SIMT kernel ---
// fp32 FFMA GEMM, 64x64 tile, 256 threads with 4x4 outputs each.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(256) gemm_simt_f32_kernel(const float* __restrict__ A, long long lda,
                                                            const float* __restrict__ B, long long ldb, int M, int N,
                                                            int K, EpiParams ep) {
  __shared__ float sa[16][64 + 4];
  __shared__ float sb[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i / 64, mm = i % 64;
      const int gm = m0 + mm, gk = k0 + kk, gn = n0 + mm;
      sa[kk][mm] = (gm < M && gk < K) ? (A_MN ? A[(long long)gk * lda + gm] : A[(long long)gm * lda + gk]) : 0.f;
      sb[kk][mm] = (gn < N && gk < K) ? (B_MN ? B[(long long)gk * ldb + gn] : B[(long long)gn * ldb + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sa[kk][ty + 16 * i];
        b[i] = sb[kk][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float alpha = epi_alpha(ep);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = m0 + ty + 16 * i, c = n0 + tx + 16 * j;
      if (r < M && c < N) epi_apply1(ep, r, c, acc[i][j] * alpha);
    }
}

}  // namespace gptb
