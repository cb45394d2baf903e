// One decode step of attention over a KV cache (the inference engine's
// generation loop: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour
// 50€ ?", § "Comment nanochat fonctionne" › 6 "Moteur d'inférence" — a KV
// cache filled at prefill, one new token per sequence per step — with the
// training attention's causal window and grouped-query heads).
//
// bf16 cache, hd = 128, fp32 arithmetic.  Decode reads every visible cached
// K / V row once, so it is bound by HBM.  The keys of each (sequence, kv head)
// are split into pieces of DEC_SPLIT rows; each piece serves the G query heads
// of its group and yields a partial softmax (max, sum, o) that a second kernel
// combines:
//   decode_split_kernel   persistent, one CTA per SM over the pieces: a
//                         producer warp loads each piece by TMA into a ring of
//                         DEC_STAGES shared-memory stages -- its K rows (two
//                         64-column boxes, 128-byte swizzle, so that a thread
//                         reading a whole key row hits no bank twice per
//                         wavefront) and V rows (one unswizzled box) -- and two
//                         groups of four warps take alternate pieces, so one
//                         group's arithmetic overlaps the other's and the loads
//                         of the pieces ahead.  Per piece: scores (thread per
//                         key), per-head max and sum of exp (a warp per head),
//                         the unnormalised sum of p_j v_j (thread per pair of
//                         output columns and half of the keys); writes
//                         (max, sum, o[128]) per (head, piece)
//   decode_combine_kernel per (sequence, head): rescales the pieces to the
//                         common max, o = sum o_p e^(m_p - m) / sum l_p e^(m_p - m)
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int DEC_HD = 128;
constexpr int DEC_SPLIT = 128;   // keys per piece (one per thread of a group in the score pass)
constexpr int DEC_GROUP = 128;   // threads of a consumer group
constexpr int DEC_THREADS = 2 * DEC_GROUP + 32;  // two consumer groups and the producer warp
constexpr int DEC_STAGES = 3;
constexpr int DEC_MAX_G = 8;     // query heads per kv head

__host__ __device__ inline int decode_pieces(int Tmax) { return (Tmax + DEC_SPLIT - 1) / DEC_SPLIT; }
// workspace floats per (sequence, head, piece): max, sum, o[128]
constexpr int DEC_PART = 2 + DEC_HD;

constexpr int DEC_K_BYTES = DEC_SPLIT * DEC_HD * 2;  // two 64-column swizzled halves of 16 KB
constexpr int DEC_STAGE_BYTES = 2 * DEC_K_BYTES;     // K rows, then V rows
constexpr int DEC_SMEM = 1024 + DEC_STAGES * DEC_STAGE_BYTES;

__device__ __forceinline__ float2 bf2_to_f2_dec(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
}

// keys of piece `piece` of sequence b: rows lo + j0 .. lo + j0 + nk - 1 of the cache
struct DecPiece {
  int b, kvh, piece, lo, nk;
};
__device__ __forceinline__ DecPiece dec_piece(int w, int P, int Hkv, int Tmax, int window,
                                              const int32_t* __restrict__ lens) {
  DecPiece d;
  d.piece = w % P;
  const int bk = w / P;
  d.b = bk / Hkv;
  d.kvh = bk - d.b * Hkv;
  const int len = lens[d.b];
  const bool valid = len >= 1 && len <= Tmax;
  const int t = len - 1;
  d.lo = valid ? ((window >= 0) ? max(0, t - window) : 0) : 0;
  const int nvis = valid ? t - d.lo + 1 : 0;
  d.nk = max(0, min(DEC_SPLIT, nvis - d.piece * DEC_SPLIT));
  return d;
}

__global__ void __launch_bounds__(DEC_THREADS, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const bf16* __restrict__ q, const int32_t* __restrict__ lens, float* __restrict__ part,
                        int H, int Hkv, int Tmax, int window, int items) {
  extern __shared__ uint8_t dec_smem_raw[];
  uint8_t* stages =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float sq_all[2][DEC_MAX_G * DEC_HD];     // queries, pre-scaled, per group
  __shared__ __align__(16) float ss_all[2][DEC_MAX_G * DEC_SPLIT];  // scores, then exp(s - max)
  __shared__ __align__(16) float sred_all[2][DEC_HD];               // the second key half's partial outputs
  __shared__ float sml_all[2][2 * DEC_MAX_G];                       // per-head max, sum
  __shared__ __align__(8) uint64_t full[DEC_STAGES], empty[DEC_STAGES];
  __shared__ int abort_flag;      // a bounded wait expired somewhere in the CTA
  __shared__ int group_stop[2];   // ... in this consumer group (decided together at a group barrier)
  __shared__ int n_issued;        // pieces the producer has loaded
  const int G = H / Hkv;
  const int P = decode_pieces(Tmax);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, nctas = gridDim.x;
  if (tid == 0) {
    for (int s = 0; s < DEC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DEC_GROUP / 32);  // one arrival per warp of the consuming group
    }
    abort_flag = 0;
    group_stop[0] = group_stop[1] = 0;
    n_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 2 * DEC_GROUP / 32) {
    // ---------------------------------------------------------- producer
    // every piece is loaded, an empty one too, so that stage k % DEC_STAGES
    // holds the CTA's k-th piece; rows past the cache are zero-filled and rows
    // past a piece's keys are never used
    if (lane == 0) {
      for (int k = 0;; ++k) {
        const int w = cta + k * nctas;
        if (w >= items) break;
        const int s = k % DEC_STAGES;
        if (k >= DEC_STAGES &&
            !mbar_wait(&empty[s], ((k / DEC_STAGES) - 1) & 1, &abort_flag, ERRW_TIMEOUT_PRODUCER))
          break;
        const DecPiece d = dec_piece(w, P, Hkv, Tmax, window, lens);
        uint8_t* st = stages + s * DEC_STAGE_BYTES;
        const int row = d.b * Tmax + d.lo + d.piece * DEC_SPLIT;
        mbar_arrive_expect_tx(&full[s], DEC_STAGE_BYTES);
        tma_load_2d(st, &tm_k, &full[s], d.kvh * DEC_HD, row);
        tma_load_2d(st + DEC_K_BYTES / 2, &tm_k, &full[s], d.kvh * DEC_HD + 64, row);
        tma_load_2d(st + DEC_K_BYTES, &tm_v, &full[s], d.kvh * DEC_HD, row);
        n_issued = k + 1;
      }
    }
  } else {
    // ---------------------------------------------- consumer group gi: pieces k with k % 2 == gi
    const int gi = tid / DEC_GROUP, t = tid % DEC_GROUP, gw = t >> 5;
    float* sq = sq_all[gi];
    float* ss = ss_all[gi];
    float* sred = sred_all[gi];
    float* sml = sml_all[gi];
    auto group_sync = [&]() { named_bar_sync(1 + gi, DEC_GROUP); };
    const float scale = rsqrtf((float)DEC_HD);
    for (int k = gi;; k += 2) {
      const int w = cta + k * nctas;
      if (w >= items) break;
      const int s = k % DEC_STAGES;
      const DecPiece d = dec_piece(w, P, Hkv, Tmax, window, lens);
      for (int i = t; i < G * DEC_HD; i += DEC_GROUP)
        sq[i] = __bfloat162float(q[((long long)d.b * H + d.kvh * G) * DEC_HD + i]) * scale;
      // this piece's rows (bounded: on expiry the error is recorded, the group
      // stops together -- every warp decides after the same group barrier --
      // and the CTA drains its loads below)
      const bool ok = mbar_wait_warp(&full[s], (k / DEC_STAGES) & 1, &abort_flag, ERRW_TIMEOUT_EPILOGUE);
      if (!ok && lane == 0) group_stop[gi] = 1;
      group_sync();  // (also makes sq visible)
      if (group_stop[gi]) break;
      const uint8_t* sk = stages + s * DEC_STAGE_BYTES;
      const uint32_t* sv2 = reinterpret_cast<const uint32_t*>(sk + DEC_K_BYTES);  // V rows as bf16 pairs
      float* out = part + ((long long)d.b * H + d.kvh * G) * P * DEC_PART;     // [G][P][DEC_PART]
      // scores: thread per key, its key row from the swizzled K tile
      if (t < d.nk) {
        uint4 u[DEC_HD / 8];
#pragma unroll
        for (int c = 0; c < DEC_HD / 8; ++c)
          u[c] = *reinterpret_cast<const uint4*>(sk + (c >> 3) * (DEC_K_BYTES / 2) + t * 128 +
                                                 (((c & 7) ^ (t & 7)) << 4));
        for (int g = 0; g < G; ++g) {
          const float4* qg = reinterpret_cast<const float4*>(sq + g * DEC_HD);
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int c = 0; c < DEC_HD / 8; ++c) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[c]);
            const float4 qa = qg[2 * c], qb = qg[2 * c + 1];
            const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
            const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
            acc0 = fmaf(qa.x, f0.x, acc0);
            acc1 = fmaf(qa.y, f0.y, acc1);
            acc0 = fmaf(qa.z, f1.x, acc0);
            acc1 = fmaf(qa.w, f1.y, acc1);
            acc0 = fmaf(qb.x, f2.x, acc0);
            acc1 = fmaf(qb.y, f2.y, acc1);
            acc0 = fmaf(qb.z, f3.x, acc0);
            acc1 = fmaf(qb.w, f3.y, acc1);
          }
          ss[g * DEC_SPLIT + t] = acc0 + acc1;
        }
      }
      group_sync();
      // per head: max and sum of exp over the piece (warp gw handles heads gw, gw+4, ...)
      for (int g = gw; g < G; g += DEC_GROUP / 32) {
        float* sg = ss + g * DEC_SPLIT;
        float m = -INFINITY;
        for (int j = lane; j < d.nk; j += 32) m = fmaxf(m, sg[j]);
        m = warp_max(m);
        float l = 0.f;
        for (int j = lane; j < d.nk; j += 32) {
          const float e = fast_exp2((sg[j] - m) * LOG2E);
          sg[j] = e;
          l += e;
        }
        l = warp_sum(l);
        if (lane == 0) {
          sml[2 * g] = d.nk > 0 ? m : -INFINITY;  // an empty piece: max -inf, sum 0
          sml[2 * g + 1] = l;
        }
      }
      group_sync();
      // sum of p_j v_j: thread = output columns 2cp, 2cp+1 and one half of the keys
      const int cp = t & 63, kh = t >> 6;
      const int jh = (d.nk + 1) / 2;
      const int ja = kh ? jh : 0, jb = kh ? d.nk : jh;
      for (int g = 0; g < G; ++g) {
        const float* pg = ss + g * DEC_SPLIT;
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;  // two chains per column
        int j = ja;
        for (; j + 1 < jb; j += 2) {
          const float p0 = pg[j], p1 = pg[j + 1];
          const float2 v0 = bf2_to_f2_dec(sv2[j * (DEC_HD / 2) + cp]);
          const float2 v1 = bf2_to_f2_dec(sv2[(j + 1) * (DEC_HD / 2) + cp]);
          a0 = fmaf(p0, v0.x, a0);
          a1 = fmaf(p0, v0.y, a1);
          b0 = fmaf(p1, v1.x, b0);
          b1 = fmaf(p1, v1.y, b1);
        }
        if (j < jb) {
          const float2 v0 = bf2_to_f2_dec(sv2[j * (DEC_HD / 2) + cp]);
          a0 = fmaf(pg[j], v0.x, a0);
          a1 = fmaf(pg[j], v0.y, a1);
        }
        a0 += b0;
        a1 += b1;
        if (kh) {
          sred[2 * cp] = a0;
          sred[2 * cp + 1] = a1;
        }
        group_sync();
        float* og = out + ((long long)g * P + d.piece) * DEC_PART;
        if (!kh) {
          og[2 + 2 * cp] = a0 + sred[2 * cp];
          og[3 + 2 * cp] = a1 + sred[2 * cp + 1];
        }
        if (t == 0) {
          og[0] = sml[2 * g];
          og[1] = sml[2 * g + 1];
        }
        group_sync();
      }
      // the stage is free for the producer (sq, ss, sml, sred belong to this group)
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  // on an expired wait, the loads still in flight complete (bounded) before
  // the CTA leaves: each stage's last fill (piece k of the stage, fill k / DEC_STAGES)
  __syncthreads();
  if (tid == 0 && abort_flag) {
    for (int k = max(0, n_issued - DEC_STAGES); k < n_issued; ++k) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&full[k % DEC_STAGES], (k / DEC_STAGES) & 1))
        if (globaltimer_ns() - t0 > 100000000ull) break;
    }
  }
}

// one CTA of DEC_HD threads per (sequence, query head): combine the pieces in
// one pass (running max; the sums so far are rescaled when it grows), four
// pieces' loads in flight at a time
__global__ void __launch_bounds__(DEC_HD)
    decode_combine_kernel(const float* __restrict__ part, const int32_t* __restrict__ lens, bf16* __restrict__ o,
                          float* __restrict__ lse, int H, int Tmax) {
  const int P = decode_pieces(Tmax);
  const int bh = blockIdx.x, b = bh / H;
  const int d = threadIdx.x;
  const float* pp = part + (long long)bh * P * DEC_PART;
  const int len = lens[b];
  const bool valid = len >= 1 && len <= Tmax;
  float m = -INFINITY, l = 0.f, acc = 0.f;
  if (valid) {
    for (int p0 = 0; p0 < P; p0 += 4) {
      float mp[4], lp[4], op[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = p0 + u < P;
        const float* q = pp + (long long)(in ? p0 + u : 0) * DEC_PART;
        mp[u] = in ? q[0] : -INFINITY;
        lp[u] = in ? q[1] : 0.f;
        op[u] = in ? q[2 + d] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (mp[u] == -INFINITY) continue;  // an empty piece
        if (mp[u] > m) {
          const float r = expf(m - mp[u]);  // 0 while m is -inf
          l *= r;
          acc *= r;
          m = mp[u];
        }
        const float w = expf(mp[u] - m);
        l = fmaf(lp[u], w, l);
        acc = fmaf(op[u], w, acc);
      }
    }
  }
  o[(long long)bh * DEC_HD + d] = __float2bfloat16_rn(l > 0.f ? acc / l : 0.f);
  if (d == 0 && lse) lse[bh] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

}  // namespace gptb
