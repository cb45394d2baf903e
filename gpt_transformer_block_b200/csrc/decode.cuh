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
//   decode_split_kernel   per piece: one TMA load of the piece's V rows
//                         (DEC_SPLIT x 128, bf16) into shared memory, issued
//                         first so it overlaps the score pass; scores of its
//                         keys for the G heads (thread per key, the key row as
//                         16-byte loads); the piece's max and sum of exp per
//                         head; the unnormalised sum of p_j v_j read from the
//                         staged tile (thread = output column and half of the
//                         keys); writes (max, sum, o[128]) per (head, piece)
//   decode_combine_kernel per (sequence, head): rescales the pieces to the
//                         common max, o = sum o_p e^(m_p - m) / sum l_p e^(m_p - m)
#pragma once
#include "common.cuh"

namespace gptb {

#ifndef GPTB_DEC_SPLIT
#define GPTB_DEC_SPLIT 256
#endif
constexpr int DEC_HD = 128;
constexpr int DEC_SPLIT = GPTB_DEC_SPLIT;  // keys per piece (one per thread in the score pass)
constexpr int DEC_THREADS = DEC_SPLIT;
static_assert(DEC_SPLIT == 128 || DEC_SPLIT == 256, "a piece is one or two key halves of 128 threads");
constexpr int DEC_MAX_G = 16;       // query heads per kv head

__host__ __device__ inline int decode_pieces(int Tmax) { return (Tmax + DEC_SPLIT - 1) / DEC_SPLIT; }
// workspace floats per (sequence, head, piece): max, sum, o[128]
constexpr int DEC_PART = 2 + DEC_HD;

constexpr int DEC_V_BYTES = DEC_SPLIT * DEC_HD * 2;  // the staged V tile (dynamic shared memory)

__global__ void __launch_bounds__(DEC_THREADS, 512 / DEC_THREADS)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_v, const bf16* __restrict__ q,
                        const bf16* __restrict__ kc, const int32_t* __restrict__ lens, float* __restrict__ part,
                        int H, int Hkv, int Tmax, int window) {
  extern __shared__ __align__(128) uint8_t dec_smem[];   // [DEC_SPLIT][DEC_HD] bf16 V rows
  __shared__ __align__(16) float sq[DEC_MAX_G * DEC_HD];     // queries, pre-scaled
  __shared__ __align__(16) float ss[DEC_MAX_G * DEC_SPLIT];  // scores, then exp(s - max)
  __shared__ __align__(16) float sred[DEC_HD];               // the second key half's partial outputs
  __shared__ float sml[2 * DEC_MAX_G];                       // per-head max, sum
  __shared__ __align__(8) uint64_t vbar;
  const bf16* sv = reinterpret_cast<const bf16*>(dec_smem);
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
  float* out = part + ((long long)b * H + kvh * G) * P * DEC_PART;  // [G][P][DEC_PART]
  if (nk == 0) {  // nothing visible here: an empty piece (max -inf, sum 0)
    for (int g = tid; g < G; g += DEC_THREADS) {
      out[((long long)g * P + piece) * DEC_PART] = -INFINITY;
      out[((long long)g * P + piece) * DEC_PART + 1] = 0.f;
    }
    return;
  }
  // the V rows of the piece: one TMA box of DEC_SPLIT rows (rows past the
  // piece or past the cache are read or zero-filled and never used)
  if (tid == 0) {
    mbar_init(&vbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&vbar, DEC_V_BYTES);
    tma_load_2d(dec_smem, &tm_v, &vbar, kvh * DEC_HD, b * Tmax + lo + j0);
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
  // the staged V tile (a bounded wait: on expiry the error is recorded, the
  // copy gets a further bounded wait before the CTA leaves, and nothing is written)
  volatile int no_abort = 0;
  bool ok = mbar_wait(&vbar, 0, &no_abort, ERRW_TIMEOUT_EPILOGUE);
  ok = __syncthreads_and(ok);
  if (!ok) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(&vbar, 0))
      if (globaltimer_ns() - t0 > 100000000ull) break;
    return;
  }
  // sum of p_j v_j: thread = column c and one of the DEC_THREADS / 128 parts of the keys
  const int c = tid & (DEC_HD - 1), kh = tid >> 7;
  const int jh = (DEC_THREADS == 256) ? (nk + 1) / 2 : nk;
  const int ja = kh ? jh : 0, jb = kh ? nk : jh;
  for (int g = 0; g < G; ++g) {
    const float* pg = ss + g * DEC_SPLIT;
    float a0 = 0.f, a1 = 0.f;  // two chains
    int j = ja;
    for (; j + 1 < jb; j += 2) {
      a0 = fmaf(pg[j], __bfloat162float(sv[j * DEC_HD + c]), a0);
      a1 = fmaf(pg[j + 1], __bfloat162float(sv[(j + 1) * DEC_HD + c]), a1);
    }
    if (j < jb) a0 = fmaf(pg[j], __bfloat162float(sv[j * DEC_HD + c]), a0);
    if (kh) sred[c] = a0 + a1;
    __syncthreads();
    float* og = out + ((long long)g * P + piece) * DEC_PART;
    if (!kh) og[2 + c] = (DEC_THREADS == 256) ? (a0 + a1) + sred[c] : a0 + a1;
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
