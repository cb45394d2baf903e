// Row-wise fused kernels of the block and the stack (HBM-bound).
//
// One warp owns one token row; each lane moves 16-byte vectors (8 elements)
// and the row stays in registers between the reduction and the write, so
// every row is read once and written once.  Grids are sized to a multiple of
// the SM count and loop over rows.  Scalar-parameter gradients (lambdas, gate
// weights) are reduced per warp in registers, per block in shared memory and
// then added to the fp32 gradient with one atomic per block.
//
// Readings (the pages give snippets only): parameter-free RMSNorm with eps
// inside the rsqrt; lambda mix x = resid_lambda*x + x0_lambda*x0 at the start
// of each block; value-embedding gate 3*sigmoid(h[:, :C] Wg^T) per kv head;
// smear x[t] += smear_lambda*sigmoid(x[t,:C].w)*x[t-1]; backout
// x -= backout_lambda * x_backout.
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int EW_THREADS = 256;
constexpr int EW_MAXC = 8;  // up to 8 chunks x 8 elements x 32 lanes: rows up to 2048 wide
// Row kernels are instantiated per NC = ceil(d / 256) so a row costs exactly
// NC*8 registers per array.

struct RowLoop {
  long long row, nrows, stride;
  __device__ RowLoop(long long n) : nrows(n) {
    const long long wpb = blockDim.x >> 5;
    row = blockIdx.x * wpb + (threadIdx.x >> 5);
    stride = gridDim.x * wpb;
  }
};

template <class T, int NC>
__device__ __forceinline__ void load_row(const T* p, int d, float (&v)[NC][8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = (i * 32 + lane) * 8;
    if (c < d) load8(p + c, v[i]);
  }
}
template <class T, int NC>
__device__ __forceinline__ void store_row(T* p, int d, const float (&v)[NC][8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = (i * 32 + lane) * 8;
    if (c < d) store8(p + c, v[i]);
  }
}
template <int NC>
__device__ __forceinline__ float row_dot(const float (&a)[NC][8], const float (&b)[NC][8], int d) {
  const int lane = threadIdx.x & 31;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = (i * 32 + lane) * 8;
    if (c < d) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(a[i][e], b[i][e], s);
    }
  }
  return warp_sum(s);
}
// dot of the first C channels of a row with a length-C weight vector
template <class W, int NC>
__device__ __forceinline__ float head_dot(const float (&a)[NC][8], const W* w, int C) {
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  const int c0 = lane * 8;  // chunk 0 holds channels lane*8 .. lane*8+7
  if (c0 < C) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (c0 + e < C) s = fmaf(a[0][e], to_f(w[c0 + e]), s);
  }
  return warp_sum(s);
}

// block-level reduction of per-thread partials into a global fp32 accumulator
__device__ __forceinline__ void block_add(float* gdst, float v, float* sred) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += sred[w];
    atomicAdd(gdst, s);
  }
}

// ---------------------------------------------------------------- forward

// x_s[n] = wte[idx[n]] (+ smear from the previous token of the same row)
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    embed_smear_kernel(const int32_t* __restrict__ idx, const T* __restrict__ wte, const T* __restrict__ w_smear,
                       const float* __restrict__ smear_lambda, T* __restrict__ xs, int B, int Tn, int d, int C) {
  const float lam = C > 0 ? *smear_lambda : 0.f;
  for (RowLoop it(B * (long long)Tn); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    const int t = (int)(n % Tn);
    float e[NC][8];
    load_row(wte + (long long)idx[n] * d, d, e);
    if (C > 0 && t > 0) {
      const float gte = lam * sigmoidf_(head_dot(e, w_smear, C));
      float p[NC][8];
      load_row(wte + (long long)idx[n - 1] * d, d, p);
#pragma unroll
      for (int i = 0; i < NC; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) e[i][k] = fmaf(gte, p[i][k], e[i][k]);
    }
    store_row(xs + n * d, d, e);
  }
}

// xm = a*x + b*x0; h = rmsnorm(xm); optional VE gate sigmoid(h[:, :Cg] Wg^T)
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    mix_norm_kernel(const T* __restrict__ x, const T* __restrict__ x0, const float* __restrict__ lam,
                    T* __restrict__ xm_out, T* __restrict__ h_out, float* __restrict__ rstd_out, long long N, int d,
                    float eps, const T* __restrict__ w_gate, float* __restrict__ sg_out, int Hkv, int Cg) {
  const float a = lam[0], b = lam[1];
  const int lane = threadIdx.x & 31;
  for (RowLoop it(N); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    float v[NC][8], v0[NC][8];
    load_row(x + n * d, d, v);
    load_row(x0 + n * d, d, v0);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) v[i][k] = a * v[i][k] + b * v0[i][k];
    store_row(xm_out + n * d, d, v);
    const float rstd = rsqrtf(row_dot(v, v, d) / d + eps);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) v[i][k] *= rstd;
    store_row(h_out + n * d, d, v);
    if (lane == 0) rstd_out[n] = rstd;
    if (w_gate != nullptr) {
      for (int k = 0; k < Hkv; ++k) {
        const float z = head_dot(v, w_gate + (long long)k * Cg, Cg);
        if (lane == 0) sg_out[n * Hkv + k] = sigmoidf_(z);
      }
    }
  }
}

// h = rmsnorm(x - lam_bo * x_bo)   (backout + final norm when x_bo != null)
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    norm_kernel(const T* __restrict__ x, const T* __restrict__ x_bo, const float* __restrict__ lam_bo,
                T* __restrict__ h_out, float* __restrict__ rstd_out, long long N, int d, float eps) {
  const float lb = x_bo ? *lam_bo : 0.f;
  for (RowLoop it(N); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    float v[NC][8];
    load_row(x + n * d, d, v);
    if (x_bo) {
      float w[NC][8];
      load_row(x_bo + n * d, d, w);
#pragma unroll
      for (int i = 0; i < NC; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) v[i][k] -= lb * w[i][k];
    }
    const float rstd = rsqrtf(row_dot(v, v, d) / d + eps);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) v[i][k] *= rstd;
    store_row(h_out + n * d, d, v);
    if ((threadIdx.x & 31) == 0) rstd_out[n] = rstd;
  }
}

// rope table: (cos, sin) of t * base^(-2j/hd), computed in double
__global__ void rope_table_kernel(float2* __restrict__ tab, int Tn, int half, double base) {
  const long long n = (long long)Tn * half;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / half), j = (int)(i % half);
    const double ang = (double)t * pow(base, -2.0 * j / (2.0 * half));
    tab[i] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// per (token, head): q,k <- rope(rmsnorm(q,k)) in place, rstd saved;
// v += 3*sigmoid(z) * VE[idx] on value-embedding layers
template <class T>
__global__ void __launch_bounds__(EW_THREADS)
    qkv_post_kernel(T* __restrict__ qkv, long long ld, float* __restrict__ rstd_qk, const float2* __restrict__ rope,
                    int Tn, long long N, int H, int Hkv, int hd, float eps, const T* __restrict__ ve_table,
                    const int32_t* __restrict__ idx, const float* __restrict__ sg) {
  const int lane = threadIdx.x & 31;
  const int nh_norm = H + Hkv;
  const int nh = nh_norm + (ve_table ? Hkv : 0);
  const int half = hd / 2;
  for (RowLoop it(N * nh); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row / nh;
    const int hh = (int)(it.row - n * nh);
    T* p = qkv + n * ld + (long long)hh * hd;
    if (hh < nh_norm) {
      const int t = (int)(n % Tn);
      float ss = 0.f;
      for (int j = lane; j < hd; j += 32) {
        const float v = to_f(p[j]);
        ss = fmaf(v, v, ss);
      }
      const float r = rsqrtf(warp_sum(ss) / hd + eps);
      for (int j = lane; j < half; j += 32) {
        const float x1 = to_f(p[j]) * r, x2 = to_f(p[j + half]) * r;
        const float2 cs = rope[(long long)t * half + j];
        p[j] = from_f<T>(x1 * cs.x - x2 * cs.y);
        p[j + half] = from_f<T>(x1 * cs.y + x2 * cs.x);
      }
      if (lane == 0) rstd_qk[n * nh_norm + hh] = r;
    } else {
      const int kv = hh - nh_norm;
      T* v = p;  // v head kv sits right after the H+Hkv normed heads
      const float gate = 3.f * sg[n * Hkv + kv];
      const T* e = ve_table + (long long)idx[n] * Hkv * hd + (long long)kv * hd;
      for (int j = lane; j < hd; j += 32) v[j] = from_f<T>(to_f(v[j]) + gate * to_f(e[j]));
    }
  }
}

// --------------------------------------------------------------- backward

// out = dres + rstd * (dh - h * mean(dh * h))      (RMSNorm backward + residual)
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    norm_bwd_kernel(const T* __restrict__ dres, const T* __restrict__ dh, const T* __restrict__ h,
                    const float* __restrict__ rstd, T* __restrict__ out, long long N, int d) {
  for (RowLoop it(N); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    float g[NC][8], y[NC][8], r[NC][8];
    load_row(dh + n * d, d, g);
    load_row(h + n * d, d, y);
    load_row(dres + n * d, d, r);
    const float m = row_dot(g, y, d) / d;
    const float rs = rstd[n];
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) r[i][k] += rs * (g[i][k] - y[i][k] * m);
    store_row(out + n * d, d, r);
  }
}

// backward of q,k <- rope(rmsnorm(.)) and of the VE term, per (token, head).
// dq (fp32 [N, H*hd]), dk/dv (fp32 [N, Hkv*hd]) -> dqkv (T [N, ld]);
// dVE[idx] += gate * dv (fp32 atomics); dz = (dv . ve) * 3 sig (1 - sig)
template <class T>
__global__ void __launch_bounds__(EW_THREADS)
    qkv_post_bwd_kernel(const T* __restrict__ qkv, long long ld, const float* __restrict__ rstd_qk,
                        const float2* __restrict__ rope, const float* __restrict__ dq, long long lddq,
                        const float* __restrict__ dk, const float* __restrict__ dv, long long lddkv,
                        T* __restrict__ dqkv, int Tn, long long N, int H, int Hkv, int hd,
                        const T* __restrict__ ve_table, const int32_t* __restrict__ idx, const float* __restrict__ sg,
                        float* __restrict__ dve_table, float* __restrict__ dz) {
  const int lane = threadIdx.x & 31;
  const int nh = H + 2 * Hkv;
  const int half = hd / 2;
  for (RowLoop it(N * nh); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row / nh;
    const int hh = (int)(it.row - n * nh);
    T* out = dqkv + n * ld + (long long)hh * hd;
    if (hh < H + Hkv) {
      const int t = (int)(n % Tn);
      const float* g = (hh < H) ? dq + n * lddq + (long long)hh * hd : dk + n * lddkv + (long long)(hh - H) * hd;
      const T* y = qkv + n * ld + (long long)hh * hd;  // rope(q_normed)
      // undo the rotation on both the gradient and the stored output
      float dot = 0.f;
      for (int j = lane; j < half; j += 32) {
        const float2 cs = rope[(long long)t * half + j];
        const float g1 = g[j] * cs.x + g[j + half] * cs.y, g2 = -g[j] * cs.y + g[j + half] * cs.x;
        const float y1 = to_f(y[j]) * cs.x + to_f(y[j + half]) * cs.y;
        const float y2 = -to_f(y[j]) * cs.y + to_f(y[j + half]) * cs.x;
        dot += g1 * y1 + g2 * y2;
      }
      const float m = warp_sum(dot) / hd;
      const float r = rstd_qk[n * (H + Hkv) + hh];
      for (int j = lane; j < half; j += 32) {
        const float2 cs = rope[(long long)t * half + j];
        const float g1 = g[j] * cs.x + g[j + half] * cs.y, g2 = -g[j] * cs.y + g[j + half] * cs.x;
        const float y1 = to_f(y[j]) * cs.x + to_f(y[j + half]) * cs.y;
        const float y2 = -to_f(y[j]) * cs.y + to_f(y[j + half]) * cs.x;
        out[j] = from_f<T>(r * (g1 - y1 * m));
        out[j + half] = from_f<T>(r * (g2 - y2 * m));
      }
    } else {
      const int kv = hh - H - Hkv;
      const float* g = dv + n * lddkv + (long long)kv * hd;
      float dgate = 0.f;
      if (ve_table) {
        const long long row = (long long)idx[n] * Hkv * hd + (long long)kv * hd;
        const float gate = 3.f * sg[n * Hkv + kv];
        for (int j = lane; j < hd; j += 32) {
          dgate = fmaf(g[j], to_f(ve_table[row + j]), dgate);
          atomicAdd(dve_table + row + j, gate * g[j]);
        }
        dgate = warp_sum(dgate);
        if (lane == 0) {
          const float s = sg[n * Hkv + kv];
          dz[n * Hkv + kv] = dgate * 3.f * s * (1.f - s);
        }
      }
      for (int j = lane; j < hd; j += 32) out[j] = from_f<T>(g[j]);
    }
  }
}

// Block-input backward: dh (+ dz Wg on the first Cg channels) through the
// first RMSNorm, plus the residual path dx1; then the lambda mix:
//   dxm = dx1 + rstd*(dh - h*mean(dh*h));  dx = a*dxm (+ dx_extra);
//   dx0_acc += b*dxm;  dlam += (sum dxm*x, sum dxm*x0)
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    mix_norm_bwd_kernel(const T* __restrict__ dh, const float* __restrict__ dz, const T* __restrict__ w_gate, int Hkv,
                        int Cg, const T* __restrict__ h, const float* __restrict__ rstd, const T* __restrict__ dx1,
                        const T* __restrict__ x, const T* __restrict__ x0, const float* __restrict__ lam,
                        const T* __restrict__ dx_extra, T* __restrict__ dx_out, float* __restrict__ dx0_acc,
                        float* __restrict__ dlam, long long N, int d) {
  __shared__ float sred[EW_THREADS / 32];
  const float a = lam[0], b = lam[1];
  const int lane = threadIdx.x & 31;
  float pa = 0.f, pb = 0.f;
  for (RowLoop it(N); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    float g[NC][8], y[NC][8];
    load_row(dh + n * d, d, g);
    load_row(h + n * d, d, y);
    if (dz != nullptr) {
      const int c0 = lane * 8;
      if (c0 < Cg) {
        for (int k = 0; k < Hkv; ++k) {
          const float z = dz[n * Hkv + k];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (c0 + e < Cg) g[0][e] = fmaf(z, to_f(w_gate[(long long)k * Cg + c0 + e]), g[0][e]);
        }
      }
    }
    const float m = row_dot(g, y, d) / d;
    const float rs = rstd[n];
    float r[NC][8];
    load_row(dx1 + n * d, d, r);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) r[i][k] += rs * (g[i][k] - y[i][k] * m);  // r = dxm
    // lambda grads
    load_row(x + n * d, d, g);
    load_row(x0 + n * d, d, y);
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = (i * 32 + lane) * 8;
      if (c < d) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          pa = fmaf(r[i][k], g[i][k], pa);
          pb = fmaf(r[i][k], y[i][k], pb);
        }
      }
    }
    // dx0 accumulation (fp32)
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = (i * 32 + lane) * 8;
      if (c < d) {
        float acc[8];
        load8(dx0_acc + n * d + c, acc);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = fmaf(b, r[i][k], acc[k]);
        store8(dx0_acc + n * d + c, acc);
      }
    }
    if (dx_extra) load_row(dx_extra + n * d, d, g);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) r[i][k] = a * r[i][k] + (dx_extra ? g[i][k] : 0.f);
    store_row(dx_out + n * d, d, r);
  }
  block_add(dlam, pa, sred);
  block_add(dlam + 1, pb, sred);
}

// dWg[k][c] += sum_n dz[n,k] * h[n,c]   (c < Cg), one thread per (k,c) pair
template <class T>
__global__ void ve_gate_wgrad_kernel(const float* __restrict__ dz, const T* __restrict__ h, long long N, int d,
                                     int Hkv, int Cg, float* __restrict__ dwg) {
  const int k = threadIdx.x / Cg, c = threadIdx.x % Cg;
  if (k >= Hkv) return;
  const long long per = (N + gridDim.x - 1) / gridDim.x;
  const long long n0 = blockIdx.x * per, n1 = min(N, n0 + per);
  float acc = 0.f;
  for (long long n = n0; n < n1; ++n) acc = fmaf(dz[n * Hkv + k], to_f(h[n * d + c]), acc);
  atomicAdd(dwg + k * Cg + c, acc);
}

// Final norm + backout backward:
//   dxf = rstd*(dhf - hf*mean(dhf*hf)); dxL = dxf; dx_bo = -lam*dxf;
//   dlam_bo += -sum dxf*x_bo
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    final_norm_bwd_kernel(const T* __restrict__ dhf, const T* __restrict__ hf, const float* __restrict__ rstd,
                          const T* __restrict__ x_bo, const float* __restrict__ lam_bo, T* __restrict__ dxL,
                          T* __restrict__ dx_bo, float* __restrict__ dlam_bo, long long N, int d) {
  __shared__ float sred[EW_THREADS / 32];
  const float lb = x_bo ? *lam_bo : 0.f;
  const int lane = threadIdx.x & 31;
  float part = 0.f;
  for (RowLoop it(N); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    float g[NC][8], y[NC][8];
    load_row(dhf + n * d, d, g);
    load_row(hf + n * d, d, y);
    const float m = row_dot(g, y, d) / d;
    const float rs = rstd[n];
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) g[i][k] = rs * (g[i][k] - y[i][k] * m);
    store_row(dxL + n * d, d, g);
    if (x_bo) {
      load_row(x_bo + n * d, d, y);
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const int c = (i * 32 + lane) * 8;
        if (c < d) {
#pragma unroll
          for (int k = 0; k < 8; ++k) part = fmaf(-g[i][k], y[i][k], part);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) g[i][k] *= -lb;
      }
      store_row(dx_bo + n * d, d, g);
    }
  }
  if (x_bo) block_add(dlam_bo, part, sred);
}

// Smear + embedding backward for row n = (b, t):
//   dxs = dx + dx0_acc (the smeared embedding feeds layer 0 as x and as x0)
//   demb[t] = dxs[t] + lam*g[t+1]*dxs[t+1] + [t>=1] dz_t * w (first C channels)
//   dz_t = lam * (dxs[t].emb[t-1]) * g_t (1 - g_t),  g_t = sigmoid(emb[t,:C].w)
//   dlam += g_t (dxs[t].emb[t-1]);  dw += dz_t emb[t,:C];  dwte[idx[t]] += demb[t]
template <class T, int NC>
__global__ void __launch_bounds__(EW_THREADS)
    smear_embed_bwd_kernel(const T* __restrict__ dx, const float* __restrict__ dx0_acc, const int32_t* __restrict__ idx,
                           const T* __restrict__ wte, const T* __restrict__ w_smear,
                           const float* __restrict__ smear_lambda, float* __restrict__ dwte,
                           float* __restrict__ dw_smear, float* __restrict__ dlam, int B, int Tn, int d, int C) {
  __shared__ float sred[EW_THREADS / 32];
  __shared__ float sw[EW_THREADS];
  const int lane = threadIdx.x & 31;
  const float lam = C > 0 ? *smear_lambda : 0.f;
  float plam = 0.f, pw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (RowLoop it(B * (long long)Tn); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row;
    const int t = (int)(n % Tn);
    float g[NC][8], tmp[NC][8];
    load_row(dx + n * d, d, g);
    load_row(dx0_acc + n * d, d, tmp);
#pragma unroll
    for (int i = 0; i < NC; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) g[i][k] += tmp[i][k];  // g = dxs[t]
    if (C > 0) {
      // first channels of emb[t] (chunk 0 of this lane)
      float e0[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (lane * 8 < C) load8(wte + (long long)idx[n] * d + lane * 8, e0);
      float dzt = 0.f;
      if (t >= 1) {
        load_row(wte + (long long)idx[n - 1] * d, d, tmp);
        const float s = row_dot(g, tmp, d);
        float z = 0.f;
        if (lane * 8 < C) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (lane * 8 + k < C) z = fmaf(e0[k], to_f(w_smear[lane * 8 + k]), z);
        }
        const float gt = sigmoidf_(warp_sum(z));
        plam += (lane == 0) ? gt * s : 0.f;
        dzt = lam * s * gt * (1.f - gt);
#pragma unroll
        for (int k = 0; k < 8; ++k) pw[k] = fmaf(dzt, e0[k], pw[k]);
      }
      if (t + 1 < Tn) {
        float z = 0.f;
        if (lane * 8 < C) {
          float e1[8];
          load8(wte + (long long)idx[n + 1] * d + lane * 8, e1);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (lane * 8 + k < C) z = fmaf(e1[k], to_f(w_smear[lane * 8 + k]), z);
        }
        const float g1 = lam * sigmoidf_(warp_sum(z));
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          const int c = (i * 32 + lane) * 8;
          if (c < d) {
            float a[8], b[8];
            load8(dx + (n + 1) * d + c, a);
            load8(dx0_acc + (n + 1) * d + c, b);
#pragma unroll
            for (int k = 0; k < 8; ++k) g[i][k] = fmaf(g1, a[k] + b[k], g[i][k]);
          }
        }
      }
      if (lane * 8 < C) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (lane * 8 + k < C) g[0][k] = fmaf(dzt, to_f(w_smear[lane * 8 + k]), g[0][k]);
      }
    }
    float* dst = dwte + (long long)idx[n] * d;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int c = (i * 32 + lane) * 8;
      if (c < d) {
        atomicAdd(reinterpret_cast<float4*>(dst + c), make_float4(g[i][0], g[i][1], g[i][2], g[i][3]));
        atomicAdd(reinterpret_cast<float4*>(dst + c + 4), make_float4(g[i][4], g[i][5], g[i][6], g[i][7]));
      }
    }
  }
  if (C > 0) {
    block_add(dlam, plam, sred);
    // per channel c = lane*8 + k: sum the lanes' partials over the block's warps
    for (int k = 0; k < 8; ++k) {
      __syncthreads();
      sw[threadIdx.x] = pw[k];
      __syncthreads();
      if (threadIdx.x < 32 && lane * 8 + k < C) {
        float s = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += sw[w * 32 + lane];
        atomicAdd(dw_smear + lane * 8 + k, s);
      }
    }
  }
}

// ------------------------------------------------------ cross-entropy ----
// One CTA per logits row (bf16, V wide): lse, row loss, and the gradient
// (softmax - onehot) * inv_n written back over the logits in bf16.
__device__ __forceinline__ void lse_combine(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float mn = fmaxf(m, m2);
  s = s * expf(m - mn) + s2 * expf(m2 - mn);
  m = mn;
}

template <class T>
__global__ void __launch_bounds__(512)
    xent_rows_kernel(T* __restrict__ logits, long long ld, int V, const int32_t* __restrict__ targets,
                     float* __restrict__ row_loss, float inv_n, int nrows) {
  __shared__ float sm[16], ss[16];
  const long long r = blockIdx.x;
  if (r >= nrows) return;
  T* z = logits + r * ld;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  float m = -INFINITY, s = 0.f;
  for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
    float v[8];
    load8(z + c, v);
    float mx = v[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) mx = fmaxf(mx, v[k]);
    const float mn = fmaxf(m, mx);
    float acc = (m == -INFINITY) ? 0.f : s * expf(m - mn);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc += expf(v[k] - mn);
    m = mn;
    s = acc;
  }
  // combine (m, s) across the warp, then across warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_combine(m, s, m2, s2);
  }
  if (lane == 0) {
    sm[warp] = m;
    ss[warp] = s;
  }
  __syncthreads();
  float M = sm[0], S = ss[0];
  for (int w = 1; w < nw; ++w) lse_combine(M, S, sm[w], ss[w]);
  const float lse = M + logf(S);
  const int y = targets[r];
  const float zy = to_f(z[y]);
  __syncthreads();
  for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
    float v[8];
    load8(z + c, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (expf(v[k] - lse) - (c + k == y ? 1.f : 0.f)) * inv_n;
    store8(z + c, v);
  }
  if (threadIdx.x == 0) row_loss[r] = lse - zy;
}

// loss = mean of the row losses (single CTA, fixed order)
__global__ void __launch_bounds__(1024) mean_kernel(const float* __restrict__ x, long long n, float* __restrict__ out) {
  __shared__ float sred[32];
  float s = 0.f;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) s += x[i];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sred[w];
    *out = t / (float)n;
  }
}

}  // namespace gptb

namespace gptb {

// ------------------------------------------------- FP8 (e4m3) per tensor --
// Per-tensor dynamic scaling: s = 448 / max|x|; codes = RNE-satfinite(x * s).
// amax is kept as float bits so that atomicMax on the unsigned pattern orders
// non-negative floats correctly.
template <class T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, long long n8, unsigned int* __restrict__ amax) {
  __shared__ float sred[8];
  float m = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    load8(x + i * 8, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, sred[w]);
    atomicMax(amax, __float_as_uint(m));
  }
}

__device__ __forceinline__ float fp8_inv_scale(const float* amax) { return fmaxf(*amax, 1e-12f) / 448.f; }

template <class T>
__global__ void __launch_bounds__(256)
    quantize_e4m3_kernel(const T* __restrict__ x, long long n8, const float* __restrict__ amax, uint8_t* __restrict__ out) {
  const float s = 448.f / fmaxf(*amax, 1e-12f);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    load8(x + i * 8, v);
    uint2 o;
    __nv_fp8x2_storage_t p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      p[k] = __nv_cvt_float2_to_fp8x2(make_float2(v[2 * k] * s, v[2 * k + 1] * s), __NV_SATFINITE, __NV_E4M3);
    o.x = (uint32_t)p[0] | ((uint32_t)p[1] << 16);
    o.y = (uint32_t)p[2] | ((uint32_t)p[3] << 16);
    *reinterpret_cast<uint2*>(out + i * 8) = o;
  }
}

}  // namespace gptb

namespace gptb {

// ------------------------------------------- vectorised hd = 128 variants --
// One warp per (token, head).  Lane l holds elements 4l..4l+3 of the head:
// lanes 0-15 the first half (rotation partner j), lanes 16-31 the second half
// (j + 64); the partner value is one shuffle (lane ^ 16) away.

__device__ __forceinline__ void ld4(const bf16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void st4(bf16* p, const float (&v)[4]) {
  uint2 u;
  u.x = pack_bf16(v[0], v[1]);
  u.y = pack_bf16(v[2], v[3]);
  *reinterpret_cast<uint2*>(p) = u;
}

__global__ void __launch_bounds__(EW_THREADS)
    qkv_post_h128_kernel(bf16* __restrict__ qkv, long long ld, float* __restrict__ rstd_qk,
                         const float2* __restrict__ rope, int Tn, long long N, int H, int Hkv, float eps,
                         const bf16* __restrict__ ve_table, const int32_t* __restrict__ idx,
                         const float* __restrict__ sg) {
  const int lane = threadIdx.x & 31;
  const int nh_norm = H + Hkv;
  const int nh = nh_norm + (ve_table ? Hkv : 0);
  const bool hi = lane >= 16;
  const int j0 = (lane & 15) * 4;
  for (RowLoop it(N * nh); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row / nh;
    const int hh = (int)(it.row - n * nh);
    bf16* p = qkv + n * ld + (long long)hh * 128 + lane * 4;
    float x[4];
    ld4(p, x);
    if (hh < nh_norm) {
      float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
      const float r = rsqrtf(warp_sum(ss) * (1.f / 128.f) + eps);
      const int t = (int)(n % Tn);
      const float4 c01 = *reinterpret_cast<const float4*>(rope + (long long)t * 64 + j0);
      const float4 c23 = *reinterpret_cast<const float4*>(rope + (long long)t * 64 + j0 + 2);
      const float cs[4][2] = {{c01.x, c01.y}, {c01.z, c01.w}, {c23.x, c23.y}, {c23.z, c23.w}};
      float y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mine = x[e] * r;
        const float other = __shfl_xor_sync(0xffffffffu, x[e], 16) * r;
        // first half: x1 c - x2 s ; second half: x1 s + x2 c  (x1 = first-half value)
        y[e] = hi ? (other * cs[e][1] + mine * cs[e][0]) : (mine * cs[e][0] - other * cs[e][1]);
      }
      st4(p, y);
      if (lane == 0) rstd_qk[n * nh_norm + hh] = r;
    } else {
      const int kv = hh - nh_norm;
      const float gate = 3.f * sg[n * Hkv + kv];
      float e[4];
      ld4(ve_table + (long long)idx[n] * Hkv * 128 + (long long)kv * 128 + lane * 4, e);
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = fmaf(gate, e[i], x[i]);
      st4(p, x);
    }
  }
}

__global__ void __launch_bounds__(EW_THREADS)
    qkv_post_bwd_h128_kernel(const bf16* __restrict__ qkv, long long ld, const float* __restrict__ rstd_qk,
                             const float2* __restrict__ rope, const float* __restrict__ dq, long long lddq,
                             const float* __restrict__ dk, const float* __restrict__ dv, long long lddkv,
                             bf16* __restrict__ dqkv, int Tn, long long N, int H, int Hkv,
                             const bf16* __restrict__ ve_table, const int32_t* __restrict__ idx,
                             const float* __restrict__ sg, float* __restrict__ dve_table, float* __restrict__ dz) {
  const int lane = threadIdx.x & 31;
  const int nh = H + 2 * Hkv;
  const bool hi = lane >= 16;
  const int j0 = (lane & 15) * 4;
  for (RowLoop it(N * nh); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row / nh;
    const int hh = (int)(it.row - n * nh);
    bf16* out = dqkv + n * ld + (long long)hh * 128 + lane * 4;
    if (hh < H + Hkv) {
      const float* gp = (hh < H) ? dq + n * lddq + (long long)hh * 128 : dk + n * lddkv + (long long)(hh - H) * 128;
      const float4 g4 = *reinterpret_cast<const float4*>(gp + lane * 4);
      const float g[4] = {g4.x, g4.y, g4.z, g4.w};
      float y[4];
      ld4(qkv + n * ld + (long long)hh * 128 + lane * 4, y);
      const int t = (int)(n % Tn);
      const float4 c01 = *reinterpret_cast<const float4*>(rope + (long long)t * 64 + j0);
      const float4 c23 = *reinterpret_cast<const float4*>(rope + (long long)t * 64 + j0 + 2);
      const float cs[4][2] = {{c01.x, c01.y}, {c01.z, c01.w}, {c23.x, c23.y}, {c23.z, c23.w}};
      // undo the rotation on the gradient and on the stored (rotated) output:
      // first half: a1 c + a2 s ; second half: -a1 s + a2 c  (a1 = first-half value)
      float gu[4], yu[4], dot = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float go = __shfl_xor_sync(0xffffffffu, g[e], 16);
        const float yo = __shfl_xor_sync(0xffffffffu, y[e], 16);
        gu[e] = hi ? (g[e] * cs[e][0] - go * cs[e][1]) : (g[e] * cs[e][0] + go * cs[e][1]);
        yu[e] = hi ? (y[e] * cs[e][0] - yo * cs[e][1]) : (y[e] * cs[e][0] + yo * cs[e][1]);
        dot = fmaf(gu[e], yu[e], dot);
      }
      const float m = warp_sum(dot) * (1.f / 128.f);
      const float r = rstd_qk[n * (H + Hkv) + hh];
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = r * (gu[e] - yu[e] * m);
      st4(out, o);
    } else {
      const int kv = hh - H - Hkv;
      const float4 g4 = *reinterpret_cast<const float4*>(dv + n * lddkv + (long long)kv * 128 + lane * 4);
      float g[4] = {g4.x, g4.y, g4.z, g4.w};
      if (ve_table) {
        const long long row = (long long)idx[n] * Hkv * 128 + (long long)kv * 128 + lane * 4;
        const float s = sg[n * Hkv + kv];
        const float gate = 3.f * s;
        float e[4];
        ld4(ve_table + row, e);
        const float dg = warp_sum(g[0] * e[0] + g[1] * e[1] + g[2] * e[2] + g[3] * e[3]);
        atomicAdd(reinterpret_cast<float4*>(dve_table + row), make_float4(gate * g[0], gate * g[1], gate * g[2], gate * g[3]));
        if (lane == 0) dz[n * Hkv + kv] = dg * 3.f * s * (1.f - s);
      }
      st4(out, g);
    }
  }
}

}  // namespace gptb

namespace gptb {

// D[b,h,t] = sum_c dO[t,h,c] * o[t,h,c] for hd = 128: one warp per (token, head),
// 8-byte loads per lane
__global__ void __launch_bounds__(EW_THREADS)
    attn_bwd_pre_h128_kernel(const bf16* __restrict__ o, long long ldo, const bf16* __restrict__ dO, long long lddo,
                             float* __restrict__ D, int Tn, long long N, int H) {
  const int lane = threadIdx.x & 31;
  for (RowLoop it(N * H); it.row < it.nrows; it.row += it.stride) {
    const long long n = it.row / H;
    const int h = (int)(it.row - n * H);
    float a[4], g[4];
    ld4(o + n * ldo + (long long)h * 128 + lane * 4, a);
    ld4(dO + n * lddo + (long long)h * 128 + lane * 4, g);
    const float s = warp_sum(a[0] * g[0] + a[1] * g[1] + a[2] * g[2] + a[3] * g[3]);
    if (lane == 0) {
      const long long b = n / Tn, t = n - b * Tn;
      D[(b * H + h) * Tn + t] = s;
    }
  }
}

}  // namespace gptb
