// Causal grouped-query attention with an optional sliding window.
//
//   o[t,h] = sum_{j in vis(t)} softmax_j(q[t,h].k[j,kv] / sqrt(hd)) v[j,kv]
//   kv = h / (H/Hkv), vis(t) = { j : j <= t and (W < 0 or t - j <= W) }
// (the feature list of the nanochat GPT model: GQA, sliding window; the
// flash_attn_func(q, k, v, causal=True, window_size=...) call of its
// attention module).
//
// bf16, hd = 128: the tcgen05/TMEM flash kernels of attention_tc.cuh.
// This file: the backward preprocess D = rowsum(dO o o) and plain SIMT
// kernels (any hd <= 128, T <= 1024) used by the fp32 configuration.
#pragma once
#include "common.cuh"

namespace gptb {

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
