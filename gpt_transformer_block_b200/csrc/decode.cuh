// One decode step of attention over a KV cache (the inference engine's
// generation loop: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour
// 50€ ?", § "Comment nanochat fonctionne" › 6 "Moteur d'inférence" — a KV
// cache filled at prefill, one new token per sequence per step — with the
// training attention's causal window and grouped-query heads).
//
// bf16 cache, hd = 128, fp32 arithmetic.  One CTA per (sequence, kv head)
// serves the G query heads of the group, so each cached K / V row is read
// from HBM once per step (decode is bound by reading the cache):
//   pass 1  thread per visible key: s[g][j] = q_g . k_j / sqrt(128) for all
//           G heads (q in shared memory, the key row in 16-byte loads);
//   pass 2  per head: max and sum of exp over the scores (block reductions),
//           scores replaced by exp(s - max);
//   pass 3  thread per (key parity, output column): o_g = sum_j p_j v_j / l,
//           coalesced 256-byte V rows, the two parities added in shared memory.
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int DEC_THREADS = 256;
constexpr int DEC_HD = 128;

// dynamic shared memory of decode_attn_kernel for G heads per kv head and a cache of Tmax rows
inline size_t decode_smem_bytes(int G, int Tmax) {
  return sizeof(float) * ((size_t)G * DEC_HD + (size_t)G * Tmax + 2 * DEC_HD + 64);
}

__device__ __forceinline__ float dec_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < DEC_THREADS / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}
__device__ __forceinline__ float dec_block_sum(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < DEC_THREADS / 32; ++w) r += red[w];
  return r;
}

__global__ void __launch_bounds__(DEC_THREADS)
    decode_attn_kernel(const bf16* __restrict__ q, const bf16* __restrict__ kc, const bf16* __restrict__ vc,
                       const int32_t* __restrict__ lens, bf16* __restrict__ o, float* __restrict__ lse, int H, int Hkv,
                       int Tmax, int window) {
  extern __shared__ float dsm[];
  const int G = H / Hkv;
  const int b = blockIdx.x / Hkv, kvh = blockIdx.x - (blockIdx.x / Hkv) * Hkv;
  float* sq = dsm;                      // [G][128] queries, pre-scaled
  float* ss = sq + G * DEC_HD;          // [G][Tmax] scores, then exp(s - max)
  float* so = ss + (size_t)G * Tmax;    // [2][128] pass-3 partial sums
  float* red = so + 2 * DEC_HD;         // [8] block reductions, [8..] per-head max / sum
  const int tid = threadIdx.x;
  const int len = lens[b];
  const bool valid = len >= 1 && len <= Tmax;
  const int t = len - 1;
  const int lo = valid ? ((window >= 0) ? max(0, t - window) : 0) : 0;
  const int nvis = valid ? t - lo + 1 : 0;
  const long long rs = (long long)Hkv * DEC_HD;  // cache row stride
  const bf16* kb = kc + (long long)b * Tmax * rs + (long long)kvh * DEC_HD;
  const bf16* vb = vc + (long long)b * Tmax * rs + (long long)kvh * DEC_HD;
  const float scale = rsqrtf((float)DEC_HD);
  for (int i = tid; i < G * DEC_HD; i += DEC_THREADS)
    sq[i] = __bfloat162float(q[((long long)b * H + kvh * G) * DEC_HD + i]) * scale;
  __syncthreads();
  // pass 1: scores of every visible key for the G heads
  for (int j = tid; j < nvis; j += DEC_THREADS) {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + (long long)(lo + j) * rs);
    for (int g = 0; g < G; ++g) {
      const float* qg = sq + g * DEC_HD;
      float acc = 0.f;
#pragma unroll 4
      for (int c = 0; c < DEC_HD / 8; ++c) {
        float kv8[8];
        load8(reinterpret_cast<const bf16*>(kr + c), kv8);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qg[c * 8 + e], kv8[e], acc);
      }
      ss[(size_t)g * Tmax + j] = acc;
    }
  }
  __syncthreads();
  // pass 2: per head max and sum of exp
  for (int g = 0; g < G; ++g) {
    float* sg = ss + (size_t)g * Tmax;
    float m = -INFINITY;
    for (int j = tid; j < nvis; j += DEC_THREADS) m = fmaxf(m, sg[j]);
    m = dec_block_max(m, red);
    float l = 0.f;
    for (int j = tid; j < nvis; j += DEC_THREADS) {
      const float e = expf(sg[j] - m);
      sg[j] = e;
      l += e;
    }
    l = dec_block_sum(l, red);
    if (tid == 0) {
      red[8 + 2 * g] = m;
      red[9 + 2 * g] = l;
    }
  }
  __syncthreads();
  // pass 3: o_g = sum_j p_j v_j / l_g   (thread = column d, key parity half)
  const int d = tid & (DEC_HD - 1), half = tid >> 7;
  for (int g = 0; g < G; ++g) {
    const float* pg = ss + (size_t)g * Tmax;
    float acc = 0.f;
    for (int j = half; j < nvis; j += 2) acc = fmaf(pg[j], __bfloat162float(vb[(long long)(lo + j) * rs + d]), acc);
    so[half * DEC_HD + d] = acc;
    __syncthreads();
    if (half == 0) {
      const float l = red[9 + 2 * g];
      const float val = valid ? (so[d] + so[DEC_HD + d]) / l : 0.f;
      o[((long long)b * H + kvh * G + g) * DEC_HD + d] = __float2bfloat16_rn(val);
      if (d == 0 && lse) lse[(long long)b * H + kvh * G + g] = valid ? red[8 + 2 * g] + logf(l) : -INFINITY;
    }
    __syncthreads();
  }
}

}  // namespace gptb
