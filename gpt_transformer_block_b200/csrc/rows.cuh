// Row-wise fused kernels of the block and the stack: one CTA per token row.
//
// The row of d elements is spread over ceil(d/8) threads (rounded up to whole
// warps), 8 contiguous elements (one 16-byte bf16 vector) per thread.  Every
// input of the row is loaded at the top, so a thread has all of its row's
// memory requests in flight at once; reductions over the row (RMSNorm, dot
// products) go through warp shuffles and a small shared-memory array.  Grids
// loop over rows; many small CTAs per SM keep enough bytes in flight to run
// these HBM-bound kernels near copy bandwidth.  Scalar-parameter gradients
// (lambdas, gate weights) are accumulated per thread over the CTA's rows and
// added to the fp32 gradient with one atomic per CTA.
//
// Readings (the pages give snippets only): parameter-free RMSNorm with eps
// inside the rsqrt; lambda mix x = resid_lambda*x + x0_lambda*x0 at the start
// of each block; value-embedding gate 3*sigmoid(h[:, :C] Wg^T) per kv head;
// smear x[t] += smear_lambda*sigmoid(x[t,:C].w)*x[t-1]; backout
// x -= backout_lambda * x_backout.
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int BR_MAX_WARPS = 8;  // rows up to 2048 elements

struct BRow {
  int tid, lane, warp, nwarps, c0;  // c0 = first of this thread's 8 elements
  bool act;                          // c0 < d
  __device__ BRow(int d) {
    tid = threadIdx.x;
    lane = tid & 31;
    warp = tid >> 5;
    nwarps = blockDim.x >> 5;
    c0 = tid * 8;
    act = c0 < d;
  }
};

// sum over the CTA; every thread gets the result (two __syncthreads)
__device__ __forceinline__ float br_sum(float v, float* sh, const BRow& r) {
  v = warp_sum(v);
  if (r.lane == 0) sh[r.warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < r.nwarps; ++w) s += sh[w];
  __syncthreads();
  return s;
}
// two sums at once
__device__ __forceinline__ void br_sum2(float& a, float& b, float* sh, const BRow& r) {
  a = warp_sum(a);
  b = warp_sum(b);
  if (r.lane == 0) {
    sh[r.warp] = a;
    sh[BR_MAX_WARPS + r.warp] = b;
  }
  __syncthreads();
  float sa = 0.f, sb = 0.f;
  for (int w = 0; w < r.nwarps; ++w) {
    sa += sh[w];
    sb += sh[BR_MAX_WARPS + w];
  }
  __syncthreads();
  a = sa;
  b = sb;
}
// dot of the row's first C channels with w (threads whose c0 < C), result on every thread
template <class W>
__device__ __forceinline__ float br_head_dot(const float (&v)[8], const W* w, int C, float* sh, const BRow& r) {
  float s = 0.f;
  if (r.c0 < C) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (r.c0 + e < C) s = fmaf(v[e], to_f(w[r.c0 + e]), s);
  }
  return br_sum(s, sh, r);
}
__device__ __forceinline__ void br_add_global(float* gdst, float v, float* sh, const BRow& r) {
  const float s = br_sum(v, sh, r);
  if (r.tid == 0) atomicAdd(gdst, s);
}

// Register cache of a warp-per-row kernel: lane l holds the 8-element chunks at
// columns 8l + 256j (j < BR_CHUNKS) of its row as loaded (16 bytes of bf16, or
// 32 of fp32), so the row crosses HBM once.  Worth it only with few cached
// arrays: two (the forward norm) keep ~128 registers; four plus the backward's
// other streams cost occupancy and measured slower than reading the row twice.
constexpr int BR_CHUNKS = BR_MAX_WARPS;  // the same 2048-element row limit
template <class T> struct Raw8;
template <> struct Raw8<bf16> { uint4 u; };
template <> struct Raw8<float> { float4 a, b; };
__device__ __forceinline__ void raw_load(const bf16* p, Raw8<bf16>& r) { r.u = *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void raw_load(const float* p, Raw8<float>& r) {
  r.a = *reinterpret_cast<const float4*>(p);
  r.b = *reinterpret_cast<const float4*>(p + 4);
}
__device__ __forceinline__ void raw_unpack(const Raw8<bf16>& r, float (&v)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void raw_unpack(const Raw8<float>& r, float (&v)[8]) {
  v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
  v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}

// ---------------------------------------------------------------- forward

// x_s[n] = wte[idx[n]] (+ smear from the previous token of the same row)
template <class T>
__global__ void __launch_bounds__(256)
    br_embed_smear_kernel(const int32_t* __restrict__ idx, const T* __restrict__ wte, const T* __restrict__ w_smear,
                          const float* __restrict__ smear_lambda, T* __restrict__ xs, int B, int Tn, int d, int C) {
  __shared__ float sh[2 * BR_MAX_WARPS];
  const BRow r(d);
  const float lam = C > 0 ? *smear_lambda : 0.f;
  const long long N = (long long)B * Tn;
  for (long long n = blockIdx.x; n < N; n += gridDim.x) {
    const int t = (int)(n % Tn);
    float e[8] = {}, p[8] = {};
    if (r.act) {
      load8(wte + (long long)idx[n] * d + r.c0, e);
      if (C > 0 && t > 0) load8(wte + (long long)idx[n - 1] * d + r.c0, p);
    }
    if (C > 0 && t > 0) {
      const float g = lam * sigmoidf_(br_head_dot(e, w_smear, C, sh, r));
#pragma unroll
      for (int k = 0; k < 8; ++k) e[k] = fmaf(g, p[k], e[k]);
    }
    if (r.act) store8(xs + n * d + r.c0, e);
  }
}

// xm = a*x + b*x0; h = rmsnorm(xm); optional VE gate sigmoid(h[:, :Cg] Wg^T)
template <class T>
__global__ void __launch_bounds__(256)
    br_mix_norm_kernel(const T* __restrict__ x, const T* __restrict__ x0, const float* __restrict__ lam,
                       T* __restrict__ xm_out, T* __restrict__ h_out, float* __restrict__ rstd_out, long long N, int d,
                       float eps, const T* __restrict__ w_gate, float* __restrict__ sg_out, int Hkv, int Cg,
                       unsigned int* __restrict__ amax_h) {
  __shared__ float sh[2 * BR_MAX_WARPS];
  __shared__ float hg[256];  // the gate's input channels of the current row
  __shared__ float sa[32];
  const BRow r(d);
  const float a = lam[0], b = lam[1];
  float am = 0.f;  // max |h| stored by this thread (FP8 amax)
  for (long long n = blockIdx.x; n < N; n += gridDim.x) {
    float v[8] = {}, v0[8] = {};
    if (r.act) {
      load8(x + n * d + r.c0, v);
      load8(x0 + n * d + r.c0, v0);
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = a * v[k] + b * v0[k];
      ss = fmaf(v[k], v[k], ss);
    }
    if (r.act) store8(xm_out + n * d + r.c0, v);
    const float rstd = rsqrtf(br_sum(ss, sh, r) / d + eps);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] *= rstd;
      am = fmaxf(am, fabsf(v[k]));
    }
    if (r.act) store8(h_out + n * d + r.c0, v);
    if (r.tid == 0) rstd_out[n] = rstd;
    if (w_gate != nullptr && r.warp == 0) {
      // the first Cg (<= 256) channels live in warp 0: gather them in shared
      // memory, then lane k computes gate k on its own (no serial reductions)
      if (r.c0 < Cg) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (r.c0 + e < Cg) hg[r.c0 + e] = v[e];
      }
      __syncwarp();
      for (int k = r.lane; k < Hkv; k += 32) {
        const T* wk = w_gate + (long long)k * Cg;
        float z = 0.f;
        for (int c = 0; c < Cg; ++c) z = fmaf(hg[c], to_f(wk[c]), z);
        sg_out[n * Hkv + k] = sigmoidf_(z);
      }
      __syncwarp();  // hg is rewritten for the next row
    }
  }
  if (amax_h) block_amax_publish(am, amax_h, sa);
}

// h = rmsnorm(x - lam_bo * x_bo)   (backout + final norm when x_bo != null).
// One warp per row, the row kept in registers between the sum of squares (a
// warp reduction, no block barrier) and the scaling.
template <class T>
__global__ void __launch_bounds__(256)
    br_norm_warp_kernel(const T* __restrict__ x, const T* __restrict__ x_bo, const float* __restrict__ lam_bo,
                        T* __restrict__ h_out, float* __restrict__ rstd_out, long long N, int d, float eps,
                        unsigned int* __restrict__ amax_h) {
  __shared__ float sa[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float lb = x_bo ? *lam_bo : 0.f;
  float am = 0.f;
  for (long long n = (long long)blockIdx.x * 8 + warp; n < N; n += (long long)gridDim.x * 8) {
    const long long ro = n * d;
    Raw8<T> xr[BR_CHUNKS], br[BR_CHUNKS];
#pragma unroll
    for (int j = 0; j < BR_CHUNKS; ++j) {
      const int c = lane * 8 + j * 256;
      if (c < d) {
        raw_load(x + ro + c, xr[j]);
        if (x_bo) raw_load(x_bo + ro + c, br[j]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < BR_CHUNKS; ++j) {
      const int c = lane * 8 + j * 256;
      if (c < d) {
        float v[8], w[8] = {};
        raw_unpack(xr[j], v);
        if (x_bo) raw_unpack(br[j], w);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          v[k] -= lb * w[k];
          ss = fmaf(v[k], v[k], ss);
        }
      }
    }
    const float rstd = rsqrtf(warp_sum(ss) / d + eps);
#pragma unroll
    for (int j = 0; j < BR_CHUNKS; ++j) {
      const int c = lane * 8 + j * 256;
      if (c < d) {
        float v[8], w[8] = {};
        raw_unpack(xr[j], v);
        if (x_bo) raw_unpack(br[j], w);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          v[k] = (v[k] - lb * w[k]) * rstd;
          am = fmaxf(am, fabsf(v[k]));
        }
        store8(h_out + ro + c, v);
      }
    }
    if (lane == 0) rstd_out[n] = rstd;
  }
  if (amax_h) block_amax_publish(am, amax_h, sa);
}

}  // namespace gptb

namespace gptb {

// --------------------------------------------------------------- backward

// out = dres + rstd * (dh - h * mean(dh * h))      (RMSNorm backward + residual)
template <class T>
__global__ void __launch_bounds__(256)
    br_norm_bwd_kernel(const T* __restrict__ dres, const T* __restrict__ dh, const T* __restrict__ h,
                       const float* __restrict__ rstd, T* __restrict__ out, long long N, int d,
                       unsigned int* __restrict__ amax_out) {
  __shared__ float sh[2 * BR_MAX_WARPS];
  __shared__ float sa[32];
  const BRow r(d);
  float am = 0.f;
  for (long long n = blockIdx.x; n < N; n += gridDim.x) {
    float g[8] = {}, y[8] = {}, o[8] = {};
    if (r.act) {
      load8(dh + n * d + r.c0, g);
      load8(h + n * d + r.c0, y);
      load8(dres + n * d + r.c0, o);
    }
    const float rs = rstd[n];
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) dot = fmaf(g[k], y[k], dot);
    const float m = br_sum(dot, sh, r) / d;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      o[k] += rs * (g[k] - y[k] * m);
      am = fmaxf(am, fabsf(o[k]));
    }
    if (r.act) store8(out + n * d + r.c0, o);
  }
  if (amax_out) block_amax_publish(am, amax_out, sa);
}

// Block-input backward: dh (+ dz Wg on the first Cg channels) through the
// first RMSNorm, plus the residual path dx1; then the lambda mix:
//   dxm = dx1 + rstd*(dh - h*mean(dh*h));  dx = a*dxm (+ dx_extra);
//   dx0_acc += b*dxm;  dlam += (sum dxm*x, sum dxm*x0)
// One warp per row: a first pass over the row forms mean(dh*h) (a warp
// reduction, no block barrier), a second reads the row again (from L1 / L2)
// with the other inputs and writes the outputs.  With no barrier per row and
// few registers an SM keeps tens of rows in flight (a block per row kept
// three).
template <class T>
__global__ void __launch_bounds__(256)
    br_mix_norm_bwd_warp_kernel(const T* __restrict__ dh, const float* __restrict__ dz, const T* __restrict__ w_gate,
                                int Hkv, int Cg, const T* __restrict__ h, const float* __restrict__ rstd,
                                const T* __restrict__ dx1, const T* __restrict__ x, const T* __restrict__ x0,
                                const float* __restrict__ lam, const T* __restrict__ dx_extra, T* __restrict__ dx_out,
                                float* __restrict__ dx0_acc, float* __restrict__ dlam, long long N, int d) {
  __shared__ float sred[16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float a = lam[0], b = lam[1];
  float pa = 0.f, pb = 0.f;
  for (long long n = (long long)blockIdx.x * 8 + warp; n < N; n += (long long)gridDim.x * 8) {
    const long long ro = n * d;
    // dh of 8 columns from c, plus the value-embedding gate term on the first Cg columns
    auto grad8 = [&](int c, float (&g)[8]) {
      load8(dh + ro + c, g);
      if (dz != nullptr && c < Cg) {
        for (int k = 0; k < Hkv; ++k) {
          const float z = dz[n * Hkv + k];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (c + e < Cg) g[e] = fmaf(z, to_f(w_gate[(long long)k * Cg + c + e]), g[e]);
        }
      }
    };
    float dot = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      float g[8], y[8];
      grad8(c, g);
      load8(h + ro + c, y);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(g[e], y[e], dot);
    }
    const float m = warp_sum(dot) / d;
    const float rs = rstd[n];
    for (int c = lane * 8; c < d; c += 256) {
      float g[8], y[8], o[8], xv[8], x0v[8], acc[8], ex[8] = {};
      grad8(c, g);
      load8(h + ro + c, y);
      load8(dx1 + ro + c, o);
      load8(x + ro + c, xv);
      load8(x0 + ro + c, x0v);
      load8(dx0_acc + ro + c, acc);
      if (dx_extra) load8(dx_extra + ro + c, ex);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dxm = o[e] + rs * (g[e] - y[e] * m);
        pa = fmaf(dxm, xv[e], pa);
        pb = fmaf(dxm, x0v[e], pb);
        acc[e] = fmaf(b, dxm, acc[e]);
        o[e] = fmaf(a, dxm, ex[e]);
      }
      store8(dx0_acc + ro + c, acc);
      store8(dx_out + ro + c, o);
    }
  }
  pa = warp_sum(pa);
  pb = warp_sum(pb);
  if (lane == 0) {
    sred[warp] = pa;
    sred[8 + warp] = pb;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sa = 0.f, sb = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      sa += sred[w];
      sb += sred[8 + w];
    }
    atomicAdd(dlam, sa);
    atomicAdd(dlam + 1, sb);
  }
}

// Final norm + backout backward:
//   dxf = rstd*(dhf - hf*mean(dhf*hf)); dxL = dxf; dx_bo = -lam*dxf;
//   dlam_bo += -sum dxf*x_bo
template <class T>
__global__ void __launch_bounds__(256)
    br_final_norm_bwd_kernel(const T* __restrict__ dhf, const T* __restrict__ hf, const float* __restrict__ rstd,
                             const T* __restrict__ x_bo, const float* __restrict__ lam_bo, T* __restrict__ dxL,
                             T* __restrict__ dx_bo, float* __restrict__ dlam_bo, long long N, int d) {
  __shared__ float sh[2 * BR_MAX_WARPS];
  const BRow r(d);
  const float lb = x_bo ? *lam_bo : 0.f;
  float part = 0.f;
  for (long long n = blockIdx.x; n < N; n += gridDim.x) {
    float g[8] = {}, y[8] = {}, xb[8] = {};
    if (r.act) {
      load8(dhf + n * d + r.c0, g);
      load8(hf + n * d + r.c0, y);
      if (x_bo) load8(x_bo + n * d + r.c0, xb);
    }
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) dot = fmaf(g[k], y[k], dot);
    const float m = br_sum(dot, sh, r) / d;
    const float rs = rstd[n];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      g[k] = rs * (g[k] - y[k] * m);
      part = fmaf(-g[k], xb[k], part);
    }
    if (r.act) store8(dxL + n * d + r.c0, g);
    if (x_bo) {
#pragma unroll
      for (int k = 0; k < 8; ++k) g[k] *= -lb;
      if (r.act) store8(dx_bo + n * d + r.c0, g);
    }
  }
  if (x_bo) br_add_global(dlam_bo, part, sh, r);
}

// Smear + embedding backward for row n = (b, t):
//   dxs = dx + dx0_acc (the smeared embedding feeds layer 0 as x and as x0)
//   demb[t] = dxs[t] + lam*g[t+1]*dxs[t+1] + [t>=1] dz_t * w (first C channels)
//   dz_t = lam * (dxs[t].emb[t-1]) * g_t (1 - g_t),  g_t = sigmoid(emb[t,:C].w)
//   dlam += g_t (dxs[t].emb[t-1]);  dw += dz_t emb[t,:C];  dwte[idx[t]] += demb[t]
template <class T>
__global__ void __launch_bounds__(256)
    br_smear_embed_bwd_kernel(const T* __restrict__ dx, const float* __restrict__ dx0_acc,
                              const int32_t* __restrict__ idx, const T* __restrict__ wte,
                              const T* __restrict__ w_smear, const float* __restrict__ smear_lambda,
                              float* __restrict__ dwte, float* __restrict__ dw_smear, float* __restrict__ dlam, int B,
                              int Tn, int d, int C) {
  __shared__ float sh[2 * BR_MAX_WARPS];
  const BRow r(d);
  const float lam = C > 0 ? *smear_lambda : 0.f;
  float plam = 0.f, pw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const long long N = (long long)B * Tn;
  for (long long n = blockIdx.x; n < N; n += gridDim.x) {
    const int t = (int)(n % Tn);
    float g[8] = {}, tmp[8] = {}, e0[8] = {}, ep[8] = {}, e1[8] = {}, d1[8] = {}, a1[8] = {};
    const bool prev = C > 0 && t >= 1, next = C > 0 && t + 1 < Tn;
    if (r.act) {
      load8(dx + n * d + r.c0, g);
      load8(dx0_acc + n * d + r.c0, tmp);
      if (C > 0) load8(wte + (long long)idx[n] * d + r.c0, e0);
      if (prev) load8(wte + (long long)idx[n - 1] * d + r.c0, ep);
      if (next) {
        load8(wte + (long long)idx[n + 1] * d + r.c0, e1);
        load8(dx + (n + 1) * d + r.c0, d1);
        load8(dx0_acc + (n + 1) * d + r.c0, a1);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) g[k] += tmp[k];  // g = dxs[t]
    if (C > 0) {
      float s = 0.f, z0 = 0.f, z1 = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) s = fmaf(g[k], ep[k], s);
      if (r.c0 < C) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (r.c0 + k < C) {
            const float wk = to_f(w_smear[r.c0 + k]);
            z0 = fmaf(e0[k], wk, z0);
            z1 = fmaf(e1[k], wk, z1);
          }
      }
      br_sum2(s, z0, sh, r);
      z1 = br_sum(z1, sh, r);
      float dzt = 0.f;
      if (prev) {
        const float gt = sigmoidf_(z0);
        plam += (r.tid == 0) ? gt * s : 0.f;
        dzt = lam * s * gt * (1.f - gt);
        if (r.c0 < C) {
#pragma unroll
          for (int k = 0; k < 8; ++k) pw[k] = fmaf(dzt, e0[k], pw[k]);
        }
      }
      if (next) {
        const float g1 = lam * sigmoidf_(z1);
#pragma unroll
        for (int k = 0; k < 8; ++k) g[k] = fmaf(g1, d1[k] + a1[k], g[k]);
      }
      if (r.c0 < C) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (r.c0 + k < C) g[k] = fmaf(dzt, to_f(w_smear[r.c0 + k]), g[k]);
      }
    }
    if (r.act) {
      float* dst = dwte + (long long)idx[n] * d + r.c0;
      red_add_v4_f32(dst, g[0], g[1], g[2], g[3]);
      red_add_v4_f32(dst + 4, g[4], g[5], g[6], g[7]);
    }
  }
  if (C > 0) {
    br_add_global(dlam, plam, sh, r);
    // channel c0+k of the threads that hold the first C channels
    if (r.c0 < C) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (r.c0 + k < C) atomicAdd(dw_smear + r.c0 + k, pw[k]);
    }
  }
}

}  // namespace gptb
