// Causal grouped-query attention with an optional sliding window.
//
//   o[t,h] = sum_{j in vis(t)} softmax_j(q[t,h].k[j,kv] / sqrt(hd)) v[j,kv]
//   kv = h / (H/Hkv), vis(t) = { j : j <= t and (W < 0 or t - j <= W) }
// (the feature list of the nanochat GPT model: GQA, sliding window; the
// flash_attn_func(q, k, v, causal=True, window_size=...) call of its
// attention module).
//
// bf16, hd = 128: flash-style kernels on mma.sync.m16n8k16 (fp32 accumulate).
//   forward  : CTA = 128 queries of one head, 8 warps x 16 rows, 64-key tiles
//              double-buffered with cp.async into XOR-swizzled smem; online
//              softmax in base 2; only key tiles that intersect the window
//              [t-W, t] are visited (sliding-window tile skipping).  Writes o
//              (bf16) and the row log-sum-exp (fp32).
//   backward : CTA = 64 keys of one kv head, 4 warps x 16 keys; loops over the
//              G query heads of the group and over 32-query tiles that can
//              see its keys; recomputes P from the saved LSE; dK, dV stay in
//              registers (summed over the group), dQ is accumulated in fp32
//              with vector atomics.
// fp32 (any hd <= 128, T <= 1024): plain SIMT kernels, used by the fp32
// configuration.
#pragma once
#include "common.cuh"

namespace gptb {

// ------------------------------------------------------------ mma.sync ----
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill rows past the end
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// smem tile of R rows x 128 bf16 (256 B per row); 16-byte chunk c of row r
// lives at chunk c ^ (r & 7) so that ldmatrix row groups hit distinct banks
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int chunk) {
  return base + (uint32_t)(r * 256 + ((chunk ^ (r & 7)) << 4));
}

// load R rows (starting at global row g0) of a [rows, ld] bf16 matrix at
// column offset col0 (128 wide) into a swizzled tile; rows >= nrows are zero
template <int R, int NT>
__device__ __forceinline__ void load_tile128(uint32_t sbase, const bf16* g, long long ld, int g0, int nrows) {
  for (int i = threadIdx.x; i < R * 16; i += NT) {
    const int r = i >> 4, c = i & 15;
    const bool ok = (g0 + r) < nrows;
    const bf16* src = g + (long long)(ok ? (g0 + r) : 0) * ld + c * 8;
    cp_async16(swz(sbase, r, c), src, ok);
  }
}


// ------------------------------------------------------ forward (bf16) ----
constexpr int AF_BR = 128, AF_BC = 64, AF_THREADS = 256;
constexpr int AF_SMEM = (AF_BR + 4 * AF_BC) * 256;  // Q + 2x(K,V)

__global__ void __launch_bounds__(AF_THREADS, 1)
    attn_fwd_bf16_kernel(const bf16* __restrict__ qkv, long long ldqkv, bf16* __restrict__ o, long long ldo,
                         float* __restrict__ lse, int T, int H, int Hkv, int window) {
  extern __shared__ __align__(128) uint8_t smem_att[];
  const int nqb = (T + AF_BR - 1) / AF_BR;
  const int qb = nqb - 1 - blockIdx.x;  // heavy (late) query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = H / Hkv, kvh = h / G;
  const int q0 = qb * AF_BR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;

  const uint32_t sQ = smem_u32(smem_att);
  const uint32_t sK0 = sQ + AF_BR * 256;
  const uint32_t sV0 = sK0 + 2 * AF_BC * 256;
  const bf16* base = qkv + (long long)b * T * ldqkv;
  const bf16* gq = base + h * 128;
  const bf16* gk = base + (H + kvh) * 128;
  const bf16* gv = base + (H + Hkv + kvh) * 128;

  const int kb_lo = (window >= 0) ? max(0, q0 - window) / AF_BC : 0;
  const int kb_hi = min(T - 1, q0 + AF_BR - 1) / AF_BC;

  load_tile128<AF_BR, AF_THREADS>(sQ, gq, ldqkv, q0, T);
  load_tile128<AF_BC, AF_THREADS>(sK0, gk, ldqkv, kb_lo * AF_BC, T);
  load_tile128<AF_BC, AF_THREADS>(sV0, gv, ldqkv, kb_lo * AF_BC, T);
  cp_async_commit();

  float oacc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[8][4];
  const float sl2 = LOG2E / sqrtf(128.f);
  const int row0 = q0 + warp * 16 + g;  // rows row0 and row0 + 8

  for (int kb = kb_lo; kb <= kb_hi; ++kb) {
    const int st = (kb - kb_lo) & 1;
    if (kb < kb_hi) {
      const int ns = st ^ 1;
      load_tile128<AF_BC, AF_THREADS>(sK0 + ns * AF_BC * 256, gk, ldqkv, (kb + 1) * AF_BC, T);
      load_tile128<AF_BC, AF_THREADS>(sV0 + ns * AF_BC * 256, gv, ldqkv, (kb + 1) * AF_BC, T);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kb == kb_lo) {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = kc * 2 + (lane >> 4);
        ldsm_x4(swz(sQ, r, ch), qf[kc][0], qf[kc][1], qf[kc][2], qf[kc][3]);
      }
    }
    const uint32_t sK = sK0 + st * AF_BC * 256, sV = sV0 + st * AF_BC * 256;
    // S = Q K^T  (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int ch = kc * 2 + ((lane >> 3) & 1);
        ldsm_x4(swz(sK, r, ch), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kc], b0, b1);
        mma16816(s[2 * np + 1], qf[kc], b2, b3);
      }
    }
    // mask + online softmax (base 2)
    const int k0 = kb * AF_BC;
    const bool need_mask = (k0 + AF_BC - 1 > q0) || (k0 + AF_BC > T) ||
                           (window >= 0 && q0 + AF_BR - 1 - k0 > window);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int t = row0 + hr * 8;
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = s[nt][hr * 2 + e] * sl2;
          if (need_mask) {
            const int j = k0 + nt * 8 + t4 * 2 + e;
            const bool vis = (j <= t) && (j < T) && (window < 0 || t - j <= window);
            v = vis ? v : -INFINITY;
          }
          s[nt][hr * 2 + e] = v;
          mx = fmaxf(mx, v);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[hr], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = exp2f(m_r[hr] - m_use);
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float p = exp2f(s[nt][hr * 2 + e] - m_use);
          s[nt][hr * 2 + e] = p;
          sum += p;
        }
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      l_r[hr] = l_r[hr] * corr + sum;
      m_r[hr] = m_new;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        oacc[i][hr * 2] *= corr;
        oacc[i][hr * 2 + 1] *= corr;
      }
    }
    // O += P V
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = kc * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = np * 2 + (lane >> 4);
        ldsm_x4_t(swz(sV, r, ch), b0, b1, b2, b3);
        mma16816(oacc[2 * np], pa, b0, b1);
        mma16816(oacc[2 * np + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }
  // finalize
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int t = row0 + hr * 8;
    if (t >= T) continue;
    const float inv = l_r[hr] > 0.f ? 1.f / l_r[hr] : 0.f;
    bf16* orow = o + ((long long)b * T + t) * ldo + h * 128;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int c = nt * 8 + t4 * 2;
      *reinterpret_cast<__nv_bfloat162*>(orow + c) =
          __floats2bfloat162_rn(oacc[nt][hr * 2] * inv, oacc[nt][hr * 2 + 1] * inv);
    }
    if (t4 == 0) lse[((long long)b * H + h) * T + t] = (m_r[hr] + log2f(l_r[hr])) * LN2;
  }
}

// --------------------------------------------- backward preprocess -------
// D[b,h,t] = sum_c do[t,h,c] * o[t,h,c]   (one warp per (token, head))
template <class T>
__global__ void attn_bwd_pre_kernel(const T* __restrict__ o, long long ldo, const T* __restrict__ dO, long long lddo,
                                    float* __restrict__ D, int B, int Tn, int H, int hd) {
  const long long nw = (long long)B * Tn * H;
  const int lane = threadIdx.x & 31;
  for (long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; w < nw;
       w += ((long long)gridDim.x * blockDim.x) >> 5) {
    const long long n = w / H;
    const int h = (int)(w - n * H);
    float acc = 0.f;
    for (int c = lane; c < hd; c += 32) acc += to_f(o[n * ldo + h * hd + c]) * to_f(dO[n * lddo + h * hd + c]);
    acc = warp_sum(acc);
    if (lane == 0) {
      const long long b = n / Tn, t = n - b * Tn;
      D[(b * H + h) * Tn + t] = acc;
    }
  }
}

// ----------------------------------------------------- backward (bf16) ----
constexpr int AB_BC = 64, AB_BR = 32, AB_THREADS = 128;
constexpr int AB_DS_LD = AB_BC + 8;  // padded dS rows (144 B) keep ldmatrix conflict-free
constexpr int AB_SMEM = 2 * AB_BC * 256 + 4 * AB_BR * 256 + AB_BR * AB_DS_LD * 2 + 4 * AB_BR * 4;

__global__ void __launch_bounds__(AB_THREADS)
    attn_bwd_bf16_kernel(const bf16* __restrict__ qkv, long long ldqkv, const bf16* __restrict__ dO, long long lddo,
                         const float* __restrict__ lse, const float* __restrict__ Dd, float* __restrict__ dq_acc,
                         long long lddq, float* __restrict__ dk_out, float* __restrict__ dv_out, long long lddkv,
                         int T, int H, int Hkv, int window) {
  extern __shared__ __align__(128) uint8_t smem_att[];
  const int kb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int G = H / Hkv;
  const int k0 = kb * AB_BC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;

  const uint32_t sK = smem_u32(smem_att);
  const uint32_t sV = sK + AB_BC * 256;
  const uint32_t sQ0 = sV + AB_BC * 256;      // 2 stages x 32 rows
  const uint32_t sO0 = sQ0 + 2 * AB_BR * 256;  // dO, 2 stages
  bf16* sdS = reinterpret_cast<bf16*>(smem_att + 2 * AB_BC * 256 + 4 * AB_BR * 256);  // [32 q][64 keys]
  float* sL = reinterpret_cast<float*>(smem_att + 2 * AB_BC * 256 + 4 * AB_BR * 256 + AB_BR * AB_DS_LD * 2);
  // sL: [2 stages][lse 32 | D 32]

  const bf16* base = qkv + (long long)b * T * ldqkv;
  const bf16* gk = base + (H + kvh) * 128;
  const bf16* gv = base + (H + Hkv + kvh) * 128;
  load_tile128<AB_BC, AB_THREADS>(sK, gk, ldqkv, k0, T);
  load_tile128<AB_BC, AB_THREADS>(sV, gv, ldqkv, k0, T);
  cp_async_commit();

  // query tiles that can see keys [k0, k0+63]: t >= k0 and t <= k0 + 63 + W
  const int qt_lo = k0 / AB_BR;
  const int q_hi = (window >= 0) ? min(T - 1, k0 + AB_BC - 1 + window) : T - 1;
  const int qt_hi = q_hi / AB_BR;
  const int nq = qt_hi - qt_lo + 1;
  const int steps = G * nq;

  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  const float scale = 1.f / sqrtf(128.f);
  const float sl2 = LOG2E * scale;

  auto issue = [&](int step, int stg) {
    const int hh = kvh * G + step / nq;
    const int qt = qt_lo + step % nq;
    const bf16* gq = base + hh * 128;
    const bf16* gdo = dO + (long long)b * T * lddo + hh * 128;
    load_tile128<AB_BR, AB_THREADS>(sQ0 + stg * AB_BR * 256, gq, ldqkv, qt * AB_BR, T);
    load_tile128<AB_BR, AB_THREADS>(sO0 + stg * AB_BR * 256, gdo, lddo, qt * AB_BR, T);
    if (threadIdx.x < AB_BR) {
      const int t = qt * AB_BR + threadIdx.x;
      const long long li = ((long long)b * H + hh) * T + t;
      sL[stg * 64 + threadIdx.x] = (t < T) ? lse[li] * LOG2E : 0.f;
      sL[stg * 64 + 32 + threadIdx.x] = (t < T) ? Dd[li] : 0.f;
    }
  };
  if (steps > 0) issue(0, 0);
  cp_async_commit();

  const int key_r0 = k0 + warp * 16 + g;  // this thread's key rows key_r0, key_r0 + 8
  for (int step = 0; step < steps; ++step) {
    const int stg = step & 1;
    const int hh = kvh * G + step / nq;
    const int qt = qt_lo + step % nq;
    const int qbase = qt * AB_BR;
    if (step + 1 < steps) {
      issue(step + 1, stg ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sQ = sQ0 + stg * AB_BR * 256, sO = sO0 + stg * AB_BR * 256;
    const float* l2 = sL + stg * 64;
    const float* Dv = l2 + 32;

    // S^T = K Q^T (16 keys x 32 queries per warp);  dP^T = V dO^T
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) st[i][0] = st[i][1] = st[i][2] = st[i][3] = dpt[i][0] = dpt[i][1] = dpt[i][2] = dpt[i][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t ka[4], va[4];
      const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int ch = kc * 2 + (lane >> 4);
      ldsm_x4(swz(sK, r, ch), ka[0], ka[1], ka[2], ka[3]);
      ldsm_x4(swz(sV, r, ch), va[0], va[1], va[2], va[3]);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int rq = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int chq = kc * 2 + ((lane >> 3) & 1);
        ldsm_x4(swz(sQ, rq, chq), b0, b1, b2, b3);
        mma16816(st[2 * np], ka, b0, b1);
        mma16816(st[2 * np + 1], ka, b2, b3);
        ldsm_x4(swz(sO, rq, chq), b0, b1, b2, b3);
        mma16816(dpt[2 * np], va, b0, b1);
        mma16816(dpt[2 * np + 1], va, b2, b3);
      }
    }
    // P^T and dS^T (scaled by 1/sqrt(hd))
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key_r0 + (e >> 1) * 8;
        const int ql = nt * 8 + t4 * 2 + (e & 1);
        const int t = qbase + ql;
        const bool vis = (key <= t) && (t < T) && (key < T) && (window < 0 || t - key <= window);
        const float p = vis ? exp2f(st[nt][e] * sl2 - l2[ql]) : 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - Dv[ql]) * scale;
      }
    }
    // dV += P^T dO ;  dK += dS^T Q   (k = 32 queries: 2 chunks of 16)
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
      uint32_t pa[4], da[4];
      pa[0] = pack_bf16(st[2 * kc][0], st[2 * kc][1]);
      pa[1] = pack_bf16(st[2 * kc][2], st[2 * kc][3]);
      pa[2] = pack_bf16(st[2 * kc + 1][0], st[2 * kc + 1][1]);
      pa[3] = pack_bf16(st[2 * kc + 1][2], st[2 * kc + 1][3]);
      da[0] = pack_bf16(dpt[2 * kc][0], dpt[2 * kc][1]);
      da[1] = pack_bf16(dpt[2 * kc][2], dpt[2 * kc][3]);
      da[2] = pack_bf16(dpt[2 * kc + 1][0], dpt[2 * kc + 1][1]);
      da[3] = pack_bf16(dpt[2 * kc + 1][2], dpt[2 * kc + 1][3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = kc * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = np * 2 + (lane >> 4);
        ldsm_x4_t(swz(sO, r, ch), b0, b1, b2, b3);
        mma16816(dv[2 * np], pa, b0, b1);
        mma16816(dv[2 * np + 1], pa, b2, b3);
        ldsm_x4_t(swz(sQ, r, ch), b0, b1, b2, b3);
        mma16816(dk[2 * np], da, b0, b1);
        mma16816(dk[2 * np + 1], da, b2, b3);
      }
    }
    // dS (bf16) to smem as [query][key]
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = warp * 16 + g + (e >> 1) * 8;
        const int ql = nt * 8 + t4 * 2 + (e & 1);
        sdS[ql * AB_DS_LD + kl] = __float2bfloat16_rn(dpt[nt][e]);
      }
    }
    __syncthreads();
    // dQ[32 x 128] += dS[32 x 64] K[64 x 128]; warp -> 16 queries x 64 columns
    {
      const int mt = warp & 1, nh = warp >> 1;
      float dqa[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
      const uint32_t sdsb = smem_u32(sdS);
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        uint32_t a[4];
        {
          const int r = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int c = kc * 16 + (lane >> 4) * 8;
          ldsm_x4(sdsb + (uint32_t)((r * AB_DS_LD + c) * 2), a[0], a[1], a[2], a[3]);
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          const int r = kc * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int ch = nh * 8 + np * 2 + (lane >> 4);
          ldsm_x4_t(swz(sK, r, ch), b0, b1, b2, b3);
          mma16816(dqa[2 * np], a, b0, b1);
          mma16816(dqa[2 * np + 1], a, b2, b3);
        }
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int t = qbase + mt * 16 + g + hr * 8;
        if (t < T) {
          float* dst = dq_acc + ((long long)b * T + t) * lddq + hh * 128 + nh * 64;
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
            atomicAdd(reinterpret_cast<float2*>(dst + nt * 8 + t4 * 2), make_float2(dqa[nt][hr * 2], dqa[nt][hr * 2 + 1]));
        }
      }
    }
    __syncthreads();
  }
  // write dK, dV (fp32) for this CTA's keys
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int key = key_r0 + hr * 8;
    if (key >= T) continue;
    float* dkr = dk_out + ((long long)b * T + key) * lddkv + kvh * 128;
    float* dvr = dv_out + ((long long)b * T + key) * lddkv + kvh * 128;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int c = nt * 8 + t4 * 2;
      *reinterpret_cast<float2*>(dkr + c) = make_float2(dk[nt][hr * 2], dk[nt][hr * 2 + 1]);
      *reinterpret_cast<float2*>(dvr + c) = make_float2(dv[nt][hr * 2], dv[nt][hr * 2 + 1]);
    }
  }
}

// -------------------------------------------------------- SIMT (fp32) -----
// one CTA per (query t, head h, batch b); T <= 1024, hd <= 128
template <class T>
__global__ void __launch_bounds__(128)
    attn_fwd_simt_kernel(const T* __restrict__ qkv, long long ldqkv, T* __restrict__ o, long long ldo,
                         float* __restrict__ lse, int Tn, int H, int Hkv, int hd, int window) {
  __shared__ float sq[128];
  __shared__ float sp[1024];
  __shared__ float red[32];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (H / Hkv);
  const T* base = qkv + (long long)b * Tn * ldqkv;
  for (int c = threadIdx.x; c < hd; c += blockDim.x) sq[c] = to_f(base[(long long)t * ldqkv + h * hd + c]);
  __syncthreads();
  const int lo = (window >= 0) ? max(0, t - window) : 0;
  const float scale = 1.f / sqrtf((float)hd);
  float mx = -INFINITY;
  for (int j = lo + threadIdx.x; j <= t; j += blockDim.x) {
    const T* kr = base + (long long)j * ldqkv + (H + kvh) * hd;
    float s = 0.f;
    for (int c = 0; c < hd; ++c) s = fmaf(sq[c], to_f(kr[c]), s);
    s *= scale;
    sp[j - lo] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = lo + threadIdx.x; j <= t; j += blockDim.x) {
    const float p = expf(sp[j - lo] - mx);
    sp[j - lo] = p;
    sum += p;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w];
  const float inv = 1.f / sum;
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float acc = 0.f;
    for (int j = lo; j <= t; ++j) acc = fmaf(sp[j - lo], to_f(base[(long long)j * ldqkv + (H + Hkv + kvh) * hd + c]), acc);
    o[((long long)b * Tn + t) * ldo + h * hd + c] = from_f<T>(acc * inv);
  }
  if (threadIdx.x == 0) lse[((long long)b * H + h) * Tn + t] = mx + logf(sum);
}

// dq (plain store, this CTA owns row t of head h), dk/dv via fp32 atomics
template <class T>
__global__ void __launch_bounds__(128)
    attn_bwd_simt_kernel(const T* __restrict__ qkv, long long ldqkv, const T* __restrict__ dO, long long lddo,
                         const float* __restrict__ lse, const float* __restrict__ Dd, float* __restrict__ dq,
                         long long lddq, float* __restrict__ dk, float* __restrict__ dv, long long lddkv, int Tn,
                         int H, int Hkv, int hd, int window) {
  __shared__ float sq[128], sdo[128];
  __shared__ float sp[1024], sds[1024];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (H / Hkv);
  const T* base = qkv + (long long)b * Tn * ldqkv;
  const long long n = (long long)b * Tn + t;
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    sq[c] = to_f(base[(long long)t * ldqkv + h * hd + c]);
    sdo[c] = to_f(dO[n * lddo + h * hd + c]);
  }
  __syncthreads();
  const int lo = (window >= 0) ? max(0, t - window) : 0;
  const float scale = 1.f / sqrtf((float)hd);
  const float L = lse[((long long)b * H + h) * Tn + t];
  const float Dt = Dd[((long long)b * H + h) * Tn + t];
  for (int j = lo + threadIdx.x; j <= t; j += blockDim.x) {
    const T* kr = base + (long long)j * ldqkv + (H + kvh) * hd;
    const T* vr = base + (long long)j * ldqkv + (H + Hkv + kvh) * hd;
    float s = 0.f, dp = 0.f;
    for (int c = 0; c < hd; ++c) {
      s = fmaf(sq[c], to_f(kr[c]), s);
      dp = fmaf(sdo[c], to_f(vr[c]), dp);
    }
    const float p = expf(s * scale - L);
    sp[j - lo] = p;
    sds[j - lo] = p * (dp - Dt) * scale;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float acc = 0.f;
    for (int j = lo; j <= t; ++j) acc = fmaf(sds[j - lo], to_f(base[(long long)j * ldqkv + (H + kvh) * hd + c]), acc);
    dq[n * lddq + h * hd + c] = acc;
  }
  for (int i = threadIdx.x; i < (t - lo + 1) * hd; i += blockDim.x) {
    const int jj = i / hd, c = i - jj * hd;
    const long long m = (long long)b * Tn + lo + jj;
    atomicAdd(dk + m * lddkv + kvh * hd + c, sds[jj] * sq[c]);
    atomicAdd(dv + m * lddkv + kvh * hd + c, sp[jj] * sdo[c]);
  }
}

}  // namespace gptb
