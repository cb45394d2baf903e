// One decode step of attention over a KV cache (the inference engine's
// generation loop: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour
// 50€ ?", § "Comment nanochat fonctionne" › 6 "Moteur d'inférence" — a KV
// cache filled at prefill, one new token per sequence per step — with the
// training attention's causal window and grouped-query heads).
//
// bf16 cache, hd = 128, fp32 arithmetic.  Decode reads every visible cached
// K / V row once, so it is bound by HBM; the keys of each (sequence, kv head)
// are split into pieces of DEC_SPLIT rows handled by separate CTAs (enough
// CTAs in flight to keep the memory system busy), each serving the G query
// heads of its group:
//   decode_split_kernel   per piece: scores of its keys for the G heads
//                         (thread per key, 16-byte loads of the key row),
//                         the piece's max and sum of exp per head, and the
//                         unnormalised sum of p_j v_j (a warp per key, each
//                         lane 4 columns, so a V row is one 256-byte access);
//                         writes (max, sum, o[128]) per (head, piece)
//   decode_combine_kernel per (sequence, head): rescales the pieces to the
//                         common max, o = sum o_p e^(m_p - m) / sum l_p e^(m_p - m)
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int DEC_THREADS = 256;
constexpr int DEC_HD = 128;
constexpr int DEC_SPLIT = 256;      // keys per piece (one per thread in the score pass)
constexpr int DEC_MAX_G = 16;       // query heads per kv head

__host__ __device__ inline int decode_pieces(int Tmax) { return (Tmax + DEC_SPLIT - 1) / DEC_SPLIT; }
// workspace floats per (sequence, head, piece): max, sum, o[128]
constexpr int DEC_PART = 2 + DEC_HD;

__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const bf16* __restrict__ q, const bf16* __restrict__ kc, const bf16* __restrict__ vc,
                        const int32_t* __restrict__ lens, float* __restrict__ part, int H, int Hkv, int Tmax,
                        int window) {
  __shared__ __align__(16) float sq[DEC_MAX_G * DEC_HD];     // queries, pre-scaled
  __shared__ __align__(16) float ss[DEC_MAX_G * DEC_SPLIT];  // scores, then exp(s - max)
  __shared__ __align__(16) float sred[8 * DEC_HD];           // per-warp partial outputs
  __shared__ float sml[2 * DEC_MAX_G];                       // per-head max, sum
  const int G = H / Hkv;
  const int P = decode_pieces(Tmax);
  const int piece = blockIdx.x % P;
  const int bk = blockIdx.x / P;
  const int b = bk / Hkv, kvh = bk - (bk / Hkv) * Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = lens[b];
  const bool valid = len >= 1 && len <= Tmax;
  const int t = len - 1;
  const int lo = valid ? ((window >= 0) ? max(0, t - window) : 0) : 0;
  const int nvis = valid ? t - lo + 1 : 0;
  const int j0 = piece * DEC_SPLIT;                    // first visible key (offset from lo) of this piece
  const int nk = max(0, min(DEC_SPLIT, nvis - j0));    // keys of this piece
  const long long rs = (long long)Hkv * DEC_HD;        // cache row stride
  const bf16* kb = kc + (long long)b * Tmax * rs + (long long)kvh * DEC_HD;
  const bf16* vb = vc + (long long)b * Tmax * rs + (long long)kvh * DEC_HD;
  float* out = part + ((long long)b * H + kvh * G) * P * DEC_PART;  // [G][P][DEC_PART]
  if (nk == 0) {  // nothing visible here: an empty piece (max -inf, sum 0)
    for (int g = tid; g < G; g += DEC_THREADS) {
      out[((long long)g * P + piece) * DEC_PART] = -INFINITY;
      out[((long long)g * P + piece) * DEC_PART + 1] = 0.f;
    }
    return;
  }
  const float scale = rsqrtf((float)DEC_HD);
  for (int i = tid; i < G * DEC_HD; i += DEC_THREADS)
    sq[i] = __bfloat162float(q[((long long)b * H + kvh * G) * DEC_HD + i]) * scale;
  __syncthreads();
  // scores: thread per key, the whole key row in registers
  if (tid < nk) {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + (long long)(lo + j0 + tid) * rs);
    uint4 u[DEC_HD / 8];
#pragma unroll
    for (int c = 0; c < DEC_HD / 8; ++c) u[c] = kr[c];
    for (int g = 0; g < G; ++g) {
      const float* qg = sq + g * DEC_HD;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < DEC_HD / 8; ++c) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          acc = fmaf(qg[c * 8 + 2 * e], f.x, acc);
          acc = fmaf(qg[c * 8 + 2 * e + 1], f.y, acc);
        }
      }
      ss[g * DEC_SPLIT + tid] = acc;
    }
  }
  __syncthreads();
  // per head: max and sum of exp over the piece (warp g handles head g, ... )
  for (int g = warp; g < G; g += DEC_THREADS / 32) {
    float* sg = ss + g * DEC_SPLIT;
    float m = -INFINITY;
    for (int j = lane; j < nk; j += 32) m = fmaxf(m, sg[j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float e = fast_exp2((sg[j] - m) * LOG2E);
      sg[j] = e;
      l += e;
    }
    l = warp_sum(l);
    if (lane == 0) {
      sml[2 * g] = m;
      sml[2 * g + 1] = l;
    }
  }
  __syncthreads();
  // sum of p_j v_j: warp w takes keys w, w+8, ...; lane = columns 4 lane .. 4 lane + 3
  for (int g = 0; g < G; ++g) {
    const float* pg = ss + g * DEC_SPLIT;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j = warp; j < nk; j += DEC_THREADS / 32) {
      const uint2 vv = *reinterpret_cast<const uint2*>(vb + (long long)(lo + j0 + j) * rs + lane * 4);
      const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.x));
      const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.y));
      const float p = pg[j];
      a0 = fmaf(p, v01.x, a0);
      a1 = fmaf(p, v01.y, a1);
      a2 = fmaf(p, v23.x, a2);
      a3 = fmaf(p, v23.y, a3);
    }
    *reinterpret_cast<float4*>(sred + warp * DEC_HD + lane * 4) = make_float4(a0, a1, a2, a3);
    __syncthreads();
    float* og = out + ((long long)g * P + piece) * DEC_PART;
    if (tid < DEC_HD) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < DEC_THREADS / 32; ++w) s += sred[w * DEC_HD + tid];
      og[2 + tid] = s;
    }
    if (tid == 0) {
      og[0] = sml[2 * g];
      og[1] = sml[2 * g + 1];
    }
    __syncthreads();
  }
}

// one CTA of DEC_HD threads per (sequence, query head): combine the pieces
__global__ void __launch_bounds__(DEC_HD)
    decode_combine_kernel(const float* __restrict__ part, const int32_t* __restrict__ lens, bf16* __restrict__ o,
                          float* __restrict__ lse, int H, int Tmax) {
  const int P = decode_pieces(Tmax);
  const int bh = blockIdx.x, b = bh / H;
  const int d = threadIdx.x;
  const float* pp = part + (long long)bh * P * DEC_PART;
  const int len = lens[b];
  const bool valid = len >= 1 && len <= Tmax;
  float m = -INFINITY;
  for (int p = 0; p < P; ++p) m = fmaxf(m, pp[(long long)p * DEC_PART]);
  float l = 0.f, acc = 0.f;
  if (valid && m > -INFINITY) {
    for (int p = 0; p < P; ++p) {
      const float mp = pp[(long long)p * DEC_PART];
      if (mp == -INFINITY) continue;
      const float w = expf(mp - m);
      l = fmaf(pp[(long long)p * DEC_PART + 1], w, l);
      acc = fmaf(pp[(long long)p * DEC_PART + 2 + d], w, acc);
    }
  }
  o[(long long)bh * DEC_HD + d] = __float2bfloat16_rn(l > 0.f ? acc / l : 0.f);
  if (d == 0 && lse) lse[bh] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

}  // namespace gptb
