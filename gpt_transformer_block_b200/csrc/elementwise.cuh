// Per-(token, head) and per-tensor kernels of the block (HBM-bound):
//   - QK RMSNorm + RoPE and the value-embedding add: backward (one warp per
//     token, vectorised for hd = 128) and a generic forward and backward for
//     the fp32 configuration (bf16/fp8 fuse the forward into the QKV GEMM
//     epilogue);
//   - the value-embedding gate weight gradient;
//   - cross-entropy: the row log-sum-exp from the logits GEMM's per-tile
//     statistics and the logits gradient (bf16), a two-pass row kernel (fp32),
//     and the loss mean;
//   - FP8 (e4m3) per-tensor amax and quantisation.
// (The attention-backward term D = rowsum(dO o o) comes out of the dO GEMM's
// epilogue for bf16/fp8, and out of attn_bwd_pre_kernel in attention.cuh for
// the fp32 configuration.)
// The per-token-row kernels (norms, lambda mix, smear, backout) are in rows.cuh.
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int EW_THREADS = 256;

constexpr float E4M3_MAXF = 448.f, E5M2_MAXF = 57344.f;

// 8 floats times s -> 8 FP8 codes (RNE, saturating), e4m3 or e5m2
__device__ __forceinline__ uint2 to_fp8x8(const float (&v)[8], float s, bool e5m2) {
  __nv_fp8x2_storage_t p[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    p[k] = __nv_cvt_float2_to_fp8x2(make_float2(v[2 * k] * s, v[2 * k + 1] * s), __NV_SATFINITE,
                                    e5m2 ? __NV_E5M2 : __NV_E4M3);
  return make_uint2((uint32_t)p[0] | ((uint32_t)p[1] << 16), (uint32_t)p[2] | ((uint32_t)p[3] << 16));
}


struct RowLoop {
  long long row, nrows, stride;
  __device__ RowLoop(long long n) : nrows(n) {
    const long long wpb = blockDim.x >> 5;
    row = blockIdx.x * wpb + (threadIdx.x >> 5);
    stride = gridDim.x * wpb;
  }
};

// ---------------------------------------------------------------- forward

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

// ------------------------------------------------------ cross-entropy ----
// fp32 logits (SIMT path): one CTA per logits row computes the lse (online
// max / sum over the row), the row loss, and the gradient
// (softmax - onehot) * inv_n written back over the logits.
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
  const bool y_ok = y >= 0 && y < V;  // an out-of-range target is reported, never read
  const float zy = y_ok ? to_f(z[y]) : 0.f;
  __syncthreads();
  for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
    float v[8];
    load8(z + c, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (expf(v[k] - lse) - (c + k == y ? 1.f : 0.f)) * inv_n;
    store8(z + c, v);
  }
  if (threadIdx.x == 0) {
    if (!y_ok) record_error(ERRW_BAD_TARGET);
    row_loss[r] = y_ok ? lse - zy : 0.f;
  }
}

// bf16 logits (tensor-core path): the row statistics come out of the logits
// GEMM's epilogue (EPI_XENT: per 256-column tile the max and the sum of
// exp(z - max), and z at the target), so no kernel reduces over a stored row.
// xent_lse_kernel: one warp per row combines the row's tile statistics into
// the log-sum-exp and the row loss lse - z[y].
__global__ void __launch_bounds__(256)
    xent_lse_kernel(const float2* __restrict__ part, int nt, const float* __restrict__ zy,
                    const int32_t* __restrict__ targets, int V, float* __restrict__ lse_l2,
                    float* __restrict__ row_loss, int rows) {
  const int lane = threadIdx.x & 31;
  const long long wpb = blockDim.x >> 5;
  for (long long r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    float m = -INFINITY, sm = 0.f;
    for (int t = lane; t < nt; t += 32) {
      const float2 p = part[r * nt + t];
      lse_combine(m, sm, p.x, p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sm, o);
      lse_combine(m, sm, m2, s2);
    }
    if (lane == 0) {
      const float lse = m + logf(sm);
      lse_l2[r] = lse * LOG2E;
      const int y = targets[r];
      if (y < 0 || y >= V) {
        record_error(ERRW_BAD_TARGET);  // no z[y]: the row adds nothing to the loss
        row_loss[r] = 0.f;
      } else {
        row_loss[r] = lse - zy[r];
      }
    }
  }
}

// The gradient of the mean loss with respect to the logits, (softmax - onehot)
// / n, written in bf16 over the logits: one CTA per row, a pure stream (each
// thread issues XENT_GRAD_VEC 16-byte loads before using any of them).  An
// out-of-range target drops the one-hot term (and was reported above).
constexpr int XENT_GRAD_THREADS = 256, XENT_GRAD_VEC = 8;
__global__ void __launch_bounds__(XENT_GRAD_THREADS)
    xent_grad_kernel(bf16* __restrict__ z, long long ld, int V, const int32_t* __restrict__ targets,
                     const float* __restrict__ lse_l2, float inv_n, int rows) {
  const int r = blockIdx.x;
  if (r >= rows) return;
  bf16* zr = z + (long long)r * ld;
  const float l2 = lse_l2[r];
  const int y = targets[r];
  const int nvec = V / 8;
  for (int v0 = threadIdx.x; v0 < nvec; v0 += XENT_GRAD_THREADS * XENT_GRAD_VEC) {
    uint4 u[XENT_GRAD_VEC];
#pragma unroll
    for (int j = 0; j < XENT_GRAD_VEC; ++j) {
      const int vi = v0 + j * XENT_GRAD_THREADS;
      if (vi < nvec) u[j] = *reinterpret_cast<const uint4*>(zr + (long long)vi * 8);
    }
#pragma unroll
    for (int j = 0; j < XENT_GRAD_VEC; ++j) {
      const int vi = v0 + j * XENT_GRAD_THREADS;
      if (vi < nvec) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
        float v[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          v[2 * k] = f.x;
          v[2 * k + 1] = f.y;
        }
        const int c = vi * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (fast_exp2(fmaf(v[k], LOG2E, -l2)) - (c + k == y ? 1.f : 0.f)) * inv_n;
        store8(zr + c, v);
      }
    }
  }
}

// The FP8 lm_head variant: the same gradient (softmax - onehot)/n, rounded to
// bf16 (the tensor the FP8 cast applies to) and written as FP8 codes with the
// fixed scale qmax * n that |dz| <= 1/n allows, into a separate [rows, V]
// byte buffer; block 0 also stores the bound 1/n, the dequantisation amax.
__global__ void __launch_bounds__(XENT_GRAD_THREADS)
    xent_grad_fp8_kernel(const bf16* __restrict__ z, long long ld, int V, const int32_t* __restrict__ targets,
                         const float* __restrict__ lse_l2, float inv_n, int e5m2, uint8_t* __restrict__ out,
                         long long ldo, float* __restrict__ bound, int rows) {
  const int r = blockIdx.x;
  if (r == 0 && threadIdx.x == 0) *bound = inv_n;
  if (r >= rows) return;
  const bf16* zr = z + (long long)r * ld;
  uint8_t* orow = out + (long long)r * ldo;
  const float l2 = lse_l2[r];
  const int y = targets[r];
  const float s = (e5m2 ? E5M2_MAXF : E4M3_MAXF) / inv_n;
  const int nvec = V / 8;
  for (int v0 = threadIdx.x; v0 < nvec; v0 += XENT_GRAD_THREADS * XENT_GRAD_VEC) {
    uint4 u[XENT_GRAD_VEC];
#pragma unroll
    for (int j = 0; j < XENT_GRAD_VEC; ++j) {
      const int vi = v0 + j * XENT_GRAD_THREADS;
      if (vi < nvec) u[j] = *reinterpret_cast<const uint4*>(zr + (long long)vi * 8);
    }
#pragma unroll
    for (int j = 0; j < XENT_GRAD_VEC; ++j) {
      const int vi = v0 + j * XENT_GRAD_THREADS;
      if (vi < nvec) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
        float v[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          v[2 * k] = f.x;
          v[2 * k + 1] = f.y;
        }
        const int c = vi * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = __bfloat162float(__float2bfloat16_rn((fast_exp2(fmaf(v[k], LOG2E, -l2)) - (c + k == y ? 1.f : 0.f)) * inv_n));
        *reinterpret_cast<uint2*>(orow + c) = to_fp8x8(v, s, e5m2 != 0);
      }
    }
  }
}

// ------------------------------------------------------ optimizer step --
// AdamW over n fp32 parameters (decoupled weight decay, bias-corrected
// moments; inv_bc1 = 1/(1-b1^t), inv_sqrt_bc2 = 1/sqrt(1-b2^t)), with an
// optional bf16 copy of the new parameters.  vec4: all arrays hold whole
// 16-byte groups (n % 4 == 0, aligned), else one element per thread.
__device__ __forceinline__ void adamw_one(float& p, float g, float& m, float& v, float lr, float b1, float b2,
                                          float eps, float decay, float inv_bc1, float inv_sqrt_bc2) {
  m = fmaf(b1, m, (1.f - b1) * g);
  v = fmaf(b2, v, (1.f - b2) * g * g);
  p = p * decay - lr * (m * inv_bc1) / (sqrtf(v) * inv_sqrt_bc2 + eps);
}
__global__ void adamw_kernel(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                             float* __restrict__ v, bf16* __restrict__ pb, long long n, float lr, float b1, float b2,
                             float eps, float decay, float inv_bc1, float inv_sqrt_bc2, int vec4) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (vec4) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n / 4; i += stride) {
      float4 pp = reinterpret_cast<float4*>(p)[i], mm = reinterpret_cast<float4*>(m)[i],
             vv = reinterpret_cast<float4*>(v)[i];
      const float4 gg = reinterpret_cast<const float4*>(g)[i];
      adamw_one(pp.x, gg.x, mm.x, vv.x, lr, b1, b2, eps, decay, inv_bc1, inv_sqrt_bc2);
      adamw_one(pp.y, gg.y, mm.y, vv.y, lr, b1, b2, eps, decay, inv_bc1, inv_sqrt_bc2);
      adamw_one(pp.z, gg.z, mm.z, vv.z, lr, b1, b2, eps, decay, inv_bc1, inv_sqrt_bc2);
      adamw_one(pp.w, gg.w, mm.w, vv.w, lr, b1, b2, eps, decay, inv_bc1, inv_sqrt_bc2);
      reinterpret_cast<float4*>(p)[i] = pp;
      reinterpret_cast<float4*>(m)[i] = mm;
      reinterpret_cast<float4*>(v)[i] = vv;
      if (pb) reinterpret_cast<uint2*>(pb)[i] = make_uint2(pack_bf16(pp.x, pp.y), pack_bf16(pp.z, pp.w));
    }
  } else {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) {
      float pp = p[i], mm = m[i], vv = v[i];
      adamw_one(pp, g[i], mm, vv, lr, b1, b2, eps, decay, inv_bc1, inv_sqrt_bc2);
      p[i] = pp;
      m[i] = mm;
      v[i] = vv;
      if (pb) pb[i] = __float2bfloat16_rn(pp);
    }
  }
}

// small host arrays (Polar Express coefficients) reach the device through the
// launch parameters: no pageable host copy, nothing that waits on the host
struct HostFloats192 {
  float v[192];
};
__global__ void store_floats_kernel(HostFloats192 src, int n, float* __restrict__ dst, float* __restrict__ zero,
                                    int nzero) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src.v[i];
  if (zero)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0.f;
}

// sum of squares of a bf16 array into *out (fp32, zeroed by the caller);
// blockIdx.y selects one of several arrays `stride` elements apart (and out[y])
__global__ void __launch_bounds__(256)
    sumsq_bf16_kernel(const bf16* __restrict__ x, long long n, float* __restrict__ out, long long stride) {
  __shared__ float sred[8];
  x += blockIdx.y * stride;
  out += blockIdx.y;
  float s = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float t = __bfloat162float(x[i]);
    s = fmaf(t, t, s);
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sred[w];
    atomicAdd(out, t);
  }
}

// y = x / (sqrt(*sumsq) + eps), rounded to bf16; blockIdx.y selects one of
// several arrays `stride` elements apart (and sumsq[y])
__global__ void scale_by_norm_bf16_kernel(const bf16* __restrict__ x, bf16* __restrict__ y, long long n,
                                          const float* __restrict__ sumsq, float eps, long long stride) {
  x += blockIdx.y * stride;
  y += blockIdx.y * stride;
  const float inv = 1.f / (sqrtf(sumsq[blockIdx.y]) + eps);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16_rn(__bfloat162float(x[i]) * inv);
}

// Muon momentum (Nesterov form): buf = mu buf + g; u = g + mu buf in bf16,
// the input of the orthogonalisation.  Four elements per thread step.  Also
// zeroes the two NorMuon sums used later in the step.
__global__ void muon_momentum_kernel(const float* __restrict__ g, float* __restrict__ buf, bf16* __restrict__ u,
                                     long long n4, float mu, float* __restrict__ sums) {
  if (blockIdx.x == 0 && threadIdx.x < 2) sums[threadIdx.x] = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 gg = reinterpret_cast<const float4*>(g)[i];
    float4 b = reinterpret_cast<float4*>(buf)[i];
    b.x = fmaf(mu, b.x, gg.x);
    b.y = fmaf(mu, b.y, gg.y);
    b.z = fmaf(mu, b.z, gg.z);
    b.w = fmaf(mu, b.w, gg.w);
    reinterpret_cast<float4*>(buf)[i] = b;
    reinterpret_cast<uint2*>(u)[i] =
        make_uint2(pack_bf16(fmaf(mu, b.x, gg.x), fmaf(mu, b.y, gg.y)), pack_bf16(fmaf(mu, b.z, gg.z), fmaf(mu, b.w, gg.w)));
  }
}

// NorMuon statistics, one warp per row (neuron) of the orthogonalised update
// o [m, n]: v_mean = mean(o^2) over the row, v = beta2 v + (1-beta2) v_mean,
// step = 1/sqrt(max(v, 1e-10)); sums[0] += v_mean, sums[1] += v_mean step^2.
__global__ void __launch_bounds__(256)
    normuon_rows_kernel(const bf16* __restrict__ o, int m, int n, float* __restrict__ v, float beta2,
                        float* __restrict__ step, float* __restrict__ sums) {
  const int lane = threadIdx.x & 31;
  const long long wpb = blockDim.x >> 5;
  float s1 = 0.f, s2 = 0.f;  // this warp's share of the two sums (lane 0)
  for (long long r = blockIdx.x * wpb + (threadIdx.x >> 5); r < m; r += gridDim.x * wpb) {
    const bf16* row = o + r * n;
    float ss = 0.f;
    for (int c = lane * 8; c < n; c += 256) {
      float x[8];
      load8(row + c, x);
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(x[k], x[k], ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) {
      const float vm = ss / (float)n;
      const float vv = fmaf(beta2, v[r], (1.f - beta2) * vm);
      v[r] = vv;
      const float st = rsqrtf(fmaxf(vv, 1e-10f));
      step[r] = st;
      s1 += vm;
      s2 += vm * st * st;
    }
  }
  if (lane == 0) {
    atomicAdd(&sums[0], s1);
    atomicAdd(&sums[1], s2);
  }
}

// w = w (1 - lr wd) - lr o step[row] sqrt(sums[0]) / max(sqrt(sums[1]), 1e-10),
// and the bf16 working copy (if any).  Four elements per thread step.
__global__ void muon_apply_kernel(float* __restrict__ w, bf16* __restrict__ wb, const bf16* __restrict__ o,
                                  const float* __restrict__ step, const float* __restrict__ sums, int m, int n,
                                  float lr, float wd) {
  const float ratio = sqrtf(sums[0]) / fmaxf(sqrtf(sums[1]), 1e-10f);
  const float decay = 1.f - lr * wd;
  const long long n4 = (long long)m * n / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const long long r = (i * 4) / n;
    const float sc = lr * step[r] * ratio;
    const uint2 ou = reinterpret_cast<const uint2*>(o)[i];
    const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ou.x));
    const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ou.y));
    float4 ww = reinterpret_cast<float4*>(w)[i];
    ww.x = fmaf(ww.x, decay, -sc * o01.x);
    ww.y = fmaf(ww.y, decay, -sc * o01.y);
    ww.z = fmaf(ww.z, decay, -sc * o23.x);
    ww.w = fmaf(ww.w, decay, -sc * o23.y);
    reinterpret_cast<float4*>(w)[i] = ww;
    if (wb) reinterpret_cast<uint2*>(wb)[i] = make_uint2(pack_bf16(ww.x, ww.y), pack_bf16(ww.z, ww.w));
  }
}

// y = bf16(x * scale) and x = float(y) * scale over n elements: gradient
// buckets travel between ranks in bf16 (half the bytes of the fp32 gradients)
__global__ void cast_f32_bf16_kernel(const float* __restrict__ x, bf16* __restrict__ y, long long n, float scale) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i] * scale);
}
__global__ void cast_bf16_f32_kernel(const bf16* __restrict__ x, float* __restrict__ y, long long n, float scale) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    y[i] = __bfloat162float(x[i]) * scale;
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

// codes = RNE-satfinite(x * qmax / amax), qmax = 448 (e4m3) or 57344 (e5m2)
template <class T>
__global__ void __launch_bounds__(256)
    quantize_fp8_kernel(const T* __restrict__ x, long long n8, const float* __restrict__ amax, int e5m2,
                        uint8_t* __restrict__ out) {
  const float s = (e5m2 ? E5M2_MAXF : E4M3_MAXF) / fmaxf(*amax, 1e-12f);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    load8(x + i * 8, v);
    *reinterpret_cast<uint2*>(out + i * 8) = to_fp8x8(v, s, e5m2 != 0);
  }
}

}  // namespace gptb

namespace gptb {

// ------------------------------------------- vectorised hd = 128 variants --

__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
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

// backward of q,k <- rope(rmsnorm(.)) and of the VE term for hd = 128: one
// warp per token.  For q and k heads lane l holds the rotation pairs
// (2l, 2l+64) and (2l+1, 2l+65), so undoing the rotation needs no shuffle;
// the (cos, sin) of the lane's two frequencies are loaded once per token.  Heads are taken QB at a time
// with all of their loads issued before any compute, so each warp keeps
// several kilobytes in flight.
// Two heads at a time with four blocks per SM (64 registers) measured fastest:
// more heads per warp (at 2 or 3 blocks per SM) or more blocks (with spills)
// were slower.
constexpr int QKV_BWD_HEADS = 2;
__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
}
__global__ void __launch_bounds__(EW_THREADS, 4)
    qkv_post_bwd_h128_kernel(const bf16* __restrict__ qkv, long long ld, const float* __restrict__ rstd_qk,
                             const float2* __restrict__ rope, const float* __restrict__ dq, long long lddq,
                             const bf16* __restrict__ dk, const bf16* __restrict__ dv, long long lddkv,
                             bf16* __restrict__ dqkv, int Tn, long long N, int H, int Hkv,
                             const bf16* __restrict__ ve_table, const int32_t* __restrict__ idx,
                             const float* __restrict__ sg, float* __restrict__ dve_table, float* __restrict__ dz,
                             unsigned int* __restrict__ amax_out) {
  constexpr int QB = QKV_BWD_HEADS;
  __shared__ float sa[32];
  float am = 0.f;  // max |dqkv| this lane stores (FP8 amax)
  const int lane = threadIdx.x & 31;
  const int nqk = H + Hkv;
  const long long wpb = blockDim.x >> 5;
  for (long long n = blockIdx.x * wpb + (threadIdx.x >> 5); n < N; n += gridDim.x * wpb) {
    const int t = (int)(n % Tn);
    // (cos, sin) of frequencies 2l and 2l+1
    const float4 cs = *reinterpret_cast<const float4*>(rope + (long long)t * 64 + lane * 2);
    const bf16* yrow = qkv + n * ld + lane * 2;
    bf16* orow = dqkv + n * ld + lane * 2;
    // q and k heads: undo the rotation on the gradient and on the stored
    // (rotated, normalised) output, then the RMSNorm backward
    for (int h0 = 0; h0 < nqk; h0 += QB) {
      float2 g1[QB], g2[QB];      // gradient, first / second half
      uint32_t y1[QB], y2[QB];    // stored output, 2 bf16 each
      float r[QB];
#pragma unroll
      for (int b = 0; b < QB; ++b) {
        const int hh = h0 + b;
        if (hh < nqk) {
          if (hh < H) {  // dq: fp32 (summed over key tiles by reductions); dk: bf16
            const float* gp = dq + n * lddq + (long long)hh * 128 + lane * 2;
            g1[b] = *reinterpret_cast<const float2*>(gp);
            g2[b] = *reinterpret_cast<const float2*>(gp + 64);
          } else {
            const bf16* gp = dk + n * lddkv + (long long)(hh - H) * 128 + lane * 2;
            g1[b] = bf2_to_f2(*reinterpret_cast<const uint32_t*>(gp));
            g2[b] = bf2_to_f2(*reinterpret_cast<const uint32_t*>(gp + 64));
          }
          y1[b] = *reinterpret_cast<const uint32_t*>(yrow + (long long)hh * 128);
          y2[b] = *reinterpret_cast<const uint32_t*>(yrow + (long long)hh * 128 + 64);
          r[b] = rstd_qk[n * nqk + hh];
        }
      }
#pragma unroll
      for (int b = 0; b < QB; ++b) {
        const int hh = h0 + b;
        if (hh < nqk) {  // warp-uniform
          const float2 ya = bf2_to_f2(y1[b]), yb = bf2_to_f2(y2[b]);
          // inverse rotation: first half a1 c + a2 s, second half -a1 s + a2 c
          const float gu[4] = {g1[b].x * cs.x + g2[b].x * cs.y, g1[b].y * cs.z + g2[b].y * cs.w,
                               g2[b].x * cs.x - g1[b].x * cs.y, g2[b].y * cs.z - g1[b].y * cs.w};
          const float yu[4] = {ya.x * cs.x + yb.x * cs.y, ya.y * cs.z + yb.y * cs.w, yb.x * cs.x - ya.x * cs.y,
                               yb.y * cs.z - ya.y * cs.w};
          float dot = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) dot = fmaf(gu[e], yu[e], dot);
          const float m = warp_sum(dot) * (1.f / 128.f);
          float o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o[e] = r[b] * (gu[e] - yu[e] * m);
            am = fmaxf(am, fabsf(o[e]));
          }
          *reinterpret_cast<uint32_t*>(orow + (long long)hh * 128) = pack_bf16(o[0], o[1]);
          *reinterpret_cast<uint32_t*>(orow + (long long)hh * 128 + 64) = pack_bf16(o[2], o[3]);
        }
      }
    }
    bf16* vout = dqkv + n * ld + lane * 4;  // v heads: lane l holds elements 4l..4l+3
    // v heads: the gradient passes through; with value embeddings also the
    // VE-table gradient (3*sigmoid(z) * dv, scattered by token id) and dz
    const long long ve_row = ve_table ? (long long)idx[n] * Hkv * 128 + lane * 4 : 0;
    for (int k0 = 0; k0 < Hkv; k0 += QB) {
      float4 g4[QB];
      uint2 eb[QB];
      float sv[QB];
#pragma unroll
      for (int b = 0; b < QB; ++b) {
        const int kv = k0 + b;
        if (kv < Hkv) {
          float t4[4];
          load4(dv + n * lddkv + (long long)kv * 128 + lane * 4, t4);
          g4[b] = make_float4(t4[0], t4[1], t4[2], t4[3]);
          if (ve_table) {
            eb[b] = *reinterpret_cast<const uint2*>(ve_table + ve_row + (long long)kv * 128);
            sv[b] = sg[n * Hkv + kv];
          }
        }
      }
#pragma unroll
      for (int b = 0; b < QB; ++b) {
        const int kv = k0 + b;
        if (kv < Hkv) {  // warp-uniform
        const float g[4] = {g4[b].x, g4[b].y, g4[b].z, g4[b].w};
        if (ve_table) {
          const float2 e01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&eb[b].x));
          const float2 e23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&eb[b].y));
          const float gate = 3.f * sv[b];
          const float dg = warp_sum(g[0] * e01.x + g[1] * e01.y + g[2] * e23.x + g[3] * e23.y);
          red_add_v4_f32(dve_table + ve_row + (long long)kv * 128, gate * g[0], gate * g[1], gate * g[2], gate * g[3]);
          if (lane == 0) dz[n * Hkv + kv] = dg * 3.f * sv[b] * (1.f - sv[b]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(g[e]));
        st4(vout + (long long)(nqk + kv) * 128, g);
        }
      }
    }
  }
  if (amax_out) block_amax_publish(am, amax_out, sa);
}

}  // namespace gptb

