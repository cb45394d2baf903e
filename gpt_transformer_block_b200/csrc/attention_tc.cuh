// Attention forward on the 5th-generation tensor cores (tcgen05 + TMEM), bf16,
// hd = 128.  Same math as attention.cuh (causal GQA, sliding window, LSE).
//
// CTA = two tiles of 128 queries (256 consecutive queries) of one head; 10 warps:
//   warp 0    TMA producer: both query tiles once, then K and V tiles of 128
//             keys into two 2-stage rings (64-column boxes of the packed qkv
//             buffer, 128-byte swizzle).  A K slot is refilled once every
//             score product that reads it is done, a V slot once every PV
//             product is.
//   warp 1    TMEM owner + single-thread MMA issuer.  For query tile t and key tile j:
//               S_t  = Q_t K_j^T  (M=128, N=128, K=128) into TMEM columns 128t .. 128t+127
//               O_t += P_t V_j    (M=128, N=128, K=128; P_t read from TMEM, V an
//                                 MN-major smem operand) into columns 256+128t ..
//             P_t (bf16 pairs) overwrites the first 64 columns of S_t: the
//             products of one thread run in issue order, so the next S_t,
//             issued after the PV product that reads P_t, cannot overwrite it
//             early.  Issue order S_0 S_1 | PV_0 S_0' | PV_1 S_1' | ...: the
//             tensor core works on one tile's products while the other
//             tile's softmax runs.
//   warps 2-5 softmax of query tile 0, warps 6-9 of query tile 1: thread =
//             one query row (its TMEM lane) over all 128 keys of the key tile,
//             so the row max needs no exchange between threads.  Masks
//             (causal / window / sequence end), keeps a running max in base 2
//             and rescales O_t in TMEM only when the max grows by more than 8
//             (a factor 256; P stays below 256 in bf16 and the final
//             normalisation uses the same max, so the result is exact), writes
//             P_t, and at the end normalises O_t and writes the LSE, and o
//             through the then idle Q_t tile with TMA stores.
// Only key tiles that intersect a query tile's visible range are visited.
// The grid is one-dimensional and ordered longest-first (see the CTA index
// mapping).
#pragma once
#include "common.cuh"

namespace gptb {

constexpr int FA_BM = 128, FA_BN = 128;
constexpr int FA_TILE = 128 * 128 * 2;  // one 128x128 bf16 tile: 32 KB (two 64-column swizzled halves)
constexpr int FA_QB = 2 * FA_BM;        // queries per CTA
constexpr int FA_THREADS = 320;
constexpr int FA_SMEM = 1024 /*align*/ + 2 * FA_TILE /*Q tiles*/ + 4 * FA_TILE /*K,V x2*/ + 256 /*barriers*/;

// K-major SW128 descriptor of a 128-row tile, k-th 16-element K step
__device__ __forceinline__ uint64_t fa_desc_k(uint32_t tile, int k) {
  return smem_desc_sw128(tile + (uint32_t)((k >> 2) * 16384 + (k & 3) * 32), 16, 1024);
}
// MN-major SW128 descriptor (two 64-wide MN halves 16 KB apart), k-th 16-row K step
__device__ __forceinline__ uint64_t fa_desc_mn(uint32_t tile, int k) {
  return smem_desc_sw128(tile + (uint32_t)(k * 2048), 16384, 1024);
}

__global__ void __launch_bounds__(FA_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_o,
                       float* __restrict__ lse, int T, int H, int Hkv, int window, unsigned int* __restrict__ amax_o) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fa_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                // 2 query tiles
  uint8_t* sK = sQ + 2 * FA_TILE;    // 2 stages
  uint8_t* sV = sK + 2 * FA_TILE;    // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * FA_TILE);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2 slots]
  uint64_t* k_empty = bars + 3;   // [2 slots]
  uint64_t* v_full = bars + 5;    // [2 slots]
  uint64_t* v_empty = bars + 7;   // [2 slots]
  uint64_t* s_full = bars + 9;    // [2 query tiles] S_t of the next key tile computed
  uint64_t* p_full = bars + 11;   // [2 query tiles] P_t written (one arrival per softmax warp)
  uint64_t* o_done = bars + 13;   // [2 query tiles] O_t += P_t V_j done
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // one CTA per (256-query block, head, sequence), heaviest work first: every
  // (head, sequence)'s last query block (the most key tiles under a causal
  // mask), then every second-to-last one, ..., so that the CTAs still running
  // at the end of the grid are the short ones
  const int nqb = (T + FA_QB - 1) / FA_QB;
  const int nhb = (int)gridDim.x / nqb;  // heads x sequences
  const int qb = nqb - 1 - (int)blockIdx.x / nhb;
  const int h = ((int)blockIdx.x % nhb) % H, b = ((int)blockIdx.x % nhb) / H;
  const int kvh = h / (H / Hkv);
  const int q0 = qb * FA_QB;
  // key tiles that intersect the visible keys of query tile t (empty past T)
  int lo[2], hi[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = q0 + t * FA_BM;
    lo[t] = (window >= 0) ? max(0, qt - window) / FA_BN : 0;
    hi[t] = (qt < T) ? min(qt + FA_BM - 1, T - 1) / FA_BN : lo[t] - 1;
  }
  // the ranges are monotone in t and overlap or touch, so their union is one range
  const int jlo = lo[0];
  const int jhi = max(hi[0], hi[1]);
  const int row_base = b * T;  // row of token (b, 0) in the packed [B*T, Wq] buffer
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const int nq = (hi[1] >= lo[1]) ? 2 : 1;
      mbar_arrive_expect_tx(q_full, nq * FA_TILE);
      for (int t = 0; t < nq; ++t) {
        tma_load_2d(sQ + t * FA_TILE, &tm_qkv, q_full, h * 128, row_base + q0 + t * FA_BM);
        tma_load_2d(sQ + t * FA_TILE + 16384, &tm_qkv, q_full, h * 128 + 64, row_base + q0 + t * FA_BM);
      }
      for (int j = jlo; j <= jhi; ++j) {
        const int i = j - jlo, st = i & 1;
        const uint32_t par = ((i >> 1) & 1) ^ 1u;
        const int kr = row_base + j * FA_BN;
        if (!mbar_wait(&k_empty[st], par, abort_flag, ERRW_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(&k_full[st], FA_TILE);
        uint8_t* k = sK + st * FA_TILE;
        tma_load_2d(k, &tm_qkv, &k_full[st], (H + kvh) * 128, kr);
        tma_load_2d(k + 16384, &tm_qkv, &k_full[st], (H + kvh) * 128 + 64, kr);
        if (!mbar_wait(&v_empty[st], par, abort_flag, ERRW_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(&v_full[st], FA_TILE);
        uint8_t* v = sV + st * FA_TILE;
        tma_load_2d(v, &tm_qkv, &v_full[st], (H + Hkv + kvh) * 128, kr);
        tma_load_2d(v + 16384, &tm_qkv, &v_full[st], (H + Hkv + kvh) * 128 + 64, kr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = make_idesc(128, 128, false, false, false);
      constexpr uint32_t IDESC_O = make_idesc(128, 128, false, true, false);
      bool ok = mbar_wait(q_full, 0, abort_flag, ERRW_TIMEOUT_MMA);
      auto in = [&](int t, int j) { return j >= lo[t] && j <= hi[t]; };
      // S_t for key tile j; the K slot is released after its last score product
      auto issue_s = [&](int t, int j) -> bool {
        const int i = j - jlo, st = i & 1;
        if (!mbar_wait(&k_full[st], (i >> 1) & 1, abort_flag, ERRW_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + t * FA_TILE), aK = smem_u32(sK + st * FA_TILE);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ss(tmem + t * 128, fa_desc_k(aQ, k), fa_desc_k(aK, k), IDESC_S, k > 0 ? 1u : 0u);
        mma_commit(&s_full[t]);
        if (t == 1 || !in(1, j)) mma_commit(&k_empty[st]);
        return true;
      };
      // O_t += P_t V_j once the softmax has written P_t; the V slot is released after its last PV product
      auto issue_pv = [&](int t, int j) -> bool {
        const int i = j - jlo, st = i & 1;
        const int c = j - lo[t];
        if (!mbar_wait(&v_full[st], (i >> 1) & 1, abort_flag, ERRW_TIMEOUT_MMA)) return false;
        if (!mbar_wait(&p_full[t], c & 1, abort_flag, ERRW_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(sV + st * FA_TILE);
        // A = P_t from TMEM (lane = query row, 8 columns per 16 keys)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + k * 8, fa_desc_mn(aV, k), IDESC_O,
                      (c > 0 || k > 0) ? 1u : 0u);
        mma_commit(&o_done[t]);
        if (t == 1 || !in(1, j)) mma_commit(&v_empty[st]);
        return true;
      };
      if (ok && in(0, jlo)) ok = issue_s(0, jlo);
      if (ok && hi[1] >= lo[1]) ok = issue_s(1, lo[1]);
      for (int j = jlo; ok && j <= jhi; ++j) {
        if (in(0, j)) {
          ok = issue_pv(0, j) && (j + 1 > hi[0] || issue_s(0, j + 1));
          if (!ok) break;
        }
        if (in(1, j)) ok = issue_pv(1, j) && (j + 1 > hi[1] || issue_s(1, j + 1));
      }
      if (*abort_flag) {
        mma_commit(drain);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0))
          if (globaltimer_ns() - t0 > 100000000ull) { record_error(ERRW_TIMEOUT_DRAIN); break; }
      }
    }
  } else {
    // softmax of query tile tt: TMEM lane quarter qw = warp % 4 -> rows 32*qw .. 32*qw+31
    const int tt = (warp - 2) >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;        // row within the query tile
    const int tq = q0 + tt * FA_BM + r;  // query position
    const uint32_t lane_addr = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_col = (uint32_t)(tt * 128), o_col = (uint32_t)(256 + tt * 128);
    const float sl2 = LOG2E / sqrtf(128.f);
    const int qt0 = q0 + tt * FA_BM;  // first query of the tile
    // keys visible from query tq: [tq - W, tq] (or [0, tq]) clipped to the sequence
    const int kv_lo = (window >= 0) ? tq - window : 0;
    const int kv_hi = min(tq, T - 1);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int lo_t = tt ? lo[1] : lo[0];
    const int n = (tt ? hi[1] : hi[0]) - lo_t + 1;  // key tiles of this query tile (0 past T)
    for (int c = 0; c < n && ok; ++c) {
      const int k0 = (lo_t + c) * FA_BN;
      ok = mbar_wait_warp(&s_full[tt], c & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tmem_ld_32x32b_x32(lane_addr + s_col + k * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[k * 32]));
      tmem_ld_wait();
      const bool need_mask =
          (k0 + FA_BN - 1 > qt0) || (k0 + FA_BN > T) || (window >= 0 && qt0 + FA_BM - 1 - k0 > window);
      // masked scores become -inf; visible keys of row tq: kv_lo..kv_hi
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const int jk = k0 + i;
          v[i] = (jk >= kv_lo && jk <= kv_hi) ? v[i] : __float_as_uint(-INFINITY);
        }
      }
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = __uint_as_float(v[i]);
#pragma unroll
      for (int i = 8; i < 128; ++i) mp[i & 7] = fmaxf(mp[i & 7], __uint_as_float(v[i]));
      const float mx =
          fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * sl2;
      // the running max moves only when it grows by more than 8 (base 2)
      const bool grow = mx > m_used + 8.f;
      const float corr = grow ? fast_exp2(m_used - mx) : 1.f;  // 0 when m_used is -inf
      if (grow) {
        l *= corr;
        m_used = mx;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      // P = exp2(s*scale - m) as bf16 pairs (key 2c in the low half) over the
      // first 64 columns of S_t
      float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hq = 0; hq < 4; ++hq) {  // 32 keys (16 columns of P) at a time
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = hq * 32 + 2 * e;
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[i]), sl2, -mu));  // exp2(-inf) = 0 for masked keys
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[i + 1]), sl2, -mu));
          lp[(2 * e) & 3] += p0;
          lp[(2 * e + 1) & 3] += p1;
          pk[e] = pack_bf16(p0, p1);
        }
        tmem_st_32x32b_x16(lane_addr + s_col + hq * 16, pk);
      }
      l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
      // O_t to the new max (the TMEM accesses are warp-collective: the whole
      // warp enters, rows that keep their max use 1).  O_t holds every PV
      // product up to key tile c-1 (the commit of S_t above follows them);
      // the wait states it.
      if (c > 0 && __any_sync(0xffffffffu, grow)) {
        ok = mbar_wait_warp(&o_done[tt], (c - 1) & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          uint32_t w[32];
          tmem_ld_32x32b_x32(lane_addr + o_col + k * 32, w);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * corr);
          tmem_st_32x32b_x32(lane_addr + o_col + k * 32, w);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[tt]);
    }
    float oam = 0.f;  // max |o| this thread stores (FP8 amax)
    if (n > 0 && __all_sync(0xffffffffu, ok) &&
        mbar_wait_warp(&o_done[tt], (n - 1) & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // O_t (bf16) leaves through the Q_t tile, free once every S_t product
      // has completed (they precede the last PV_t that o_done follows): two
      // 64-column halves of 128 rows x 128 bytes, 128-byte swizzle; each warp
      // stores its 32 rows with two TMA boxes that clip at the sequence end
      uint8_t* stg = sQ + tt * FA_TILE;
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // columns 32k .. 32k+31
        uint32_t w[32];
        tmem_ld_32x32b_x32(lane_addr + o_col + k * 32, w);
        tmem_ld_wait();
        if (amax_o && tq < T) {
#pragma unroll
          for (int i = 0; i < 32; ++i) oam = fmaxf(oam, fabsf(__uint_as_float(w[i]) * inv));
        }
        uint8_t* row = stg + (k >> 1) * 16384 + r * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 u;
          u.x = pack_bf16(__uint_as_float(w[g * 8 + 0]) * inv, __uint_as_float(w[g * 8 + 1]) * inv);
          u.y = pack_bf16(__uint_as_float(w[g * 8 + 2]) * inv, __uint_as_float(w[g * 8 + 3]) * inv);
          u.z = pack_bf16(__uint_as_float(w[g * 8 + 4]) * inv, __uint_as_float(w[g * 8 + 5]) * inv);
          u.w = pack_bf16(__uint_as_float(w[g * 8 + 6]) * inv, __uint_as_float(w[g * 8 + 7]) * inv);
          const int cg = (k & 1) * 4 + g;  // 16-byte chunk within the 128-byte half row
          *reinterpret_cast<uint4*>(row + ((cg ^ (r & 7)) << 4)) = u;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int row0 = q0 + tt * FA_BM + qw * 32;  // first query of this warp's rows
      if (lane == 0 && row0 < T) {                 // (a box wholly past the sequence end is not issued)
        tma_store_3d(&tm_o, stg + qw * 4096, h * 128, row0, b);
        tma_store_3d(&tm_o, stg + 16384 + qw * 4096, h * 128 + 64, row0, b);
        bulk_commit_group();
        bulk_wait_read0();  // the tile's shared memory is read before the CTA ends
      }
      __syncwarp();
      if (tq < T) lse[((long long)b * H + h) * T + tq] = (m_used + log2f(l)) * LN2;
    }
    if (amax_o) {  // the warp's max |o| (FP8 amax)
      oam = warp_max(oam);
      if (lane == 0 && oam > 0.f) atomicMax(amax_o, __float_as_uint(stored_abs_max_bf16(oam)));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gptb

namespace gptb {

// ---------------------------------------------- backward (bf16, tcgen05) ---
// CTA = 128 keys of one kv head; loops over the G query heads of the group
// and over the 64-query tiles that can see its keys (causal + window).
// Per step (one query head, one 64-query tile), on the tensor core:
//   S^T  = K Q^T      (M=128 keys, N=64, K=128)      -> TMEM cols 256..319
//   dP^T = V dO^T     (M=128 keys, N=64, K=128)      -> TMEM cols 320..383
//   dV  += P^T dO     (M=128, N=128, K=64 queries)   -> TMEM cols 128..255
//   dK  += dS^T Q     (M=128, N=128, K=64)           -> TMEM cols   0..127
//   dQ^T = K^T dS^T   (M=128 hd, N=64, K=128 keys)   -> TMEM cols 384..447
// Shared-memory bandwidth, not the tensor core, bounds this loop (the
// N=64 products read 6 KB of operands per 32 MMA cycles), so operands that
// can stay off shared memory do: P^T and dS^T go to TMEM as bf16 (cols
// 448..479 and 480..511) and are the A operands of dV / dK, read from TMEM;
// only dS^T is also written to smem, as the B operand of dQ^T; dQ leaves
// TMEM straight to L2 as fp32 reductions, without a staging tile.
// Warps: 0 TMA producer (K, V once; Q, dO, LSE, D per step in a 4-stage
// ring), 1 MMA issuer, 2-9 softmax backward (thread = key row, 32 of the 64
// queries): P^T = exp2(S^T*scale*log2e - LSE*log2e), dS^T = P^T (dP^T - D)/sqrt(hd);
// 10-17 dQ epilogue (thread = hd lane of dQ^T, 32 of the 64 queries; two
// warps per TMEM lane quarter, as the reductions are bound by how many
// requests each warp keeps in flight).  At the end the softmax warps
// write dK, dV (bf16) through swizzled staging tiles in the then idle Q/dO
// ring and TMA stores that clip at the sequence end.
// CTA order: groups of AB2_GROUP (kv head, sequence) pairs, key-tile-major
// inside a group, so the tiles with the most query tiles (the first ones
// under a causal mask) start first while the CTAs in flight reduce into the
// dQ rows of one or two groups only (a few MB that stay in L2, where a
// whole-batch order would send every reduction to DRAM and back).
constexpr int AB2_BK = 128, AB2_BQ = 64;
constexpr int AB2_GROUP = 16;
constexpr int AB2_THREADS = 576;
constexpr int AB2_KV_TILE = 128 * 128 * 2;  // 32 KB
constexpr int AB2_Q_TILE = 64 * 128 * 2;    // 16 KB
constexpr int AB2_PS_TILE = 128 * 64 * 2;   // 16 KB
constexpr int AB2_STAGES = 4;              // Q / dO / LSE / D ring
constexpr int AB2_SMEM = 1024 + 2 * AB2_KV_TILE + 2 * AB2_STAGES * AB2_Q_TILE + AB2_PS_TILE + 256 +
                         AB2_STAGES * 2 * 64 * 4;
// the dK / dV staging (8 warps x 2 tiles of 32 rows x 128 bytes) fits in the Q / dO ring
static_assert(8 * 2 * 4096 <= 2 * AB2_STAGES * AB2_Q_TILE, "dK/dV staging does not fit the ring");

__global__ void __launch_bounds__(AB2_THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dk,
                       const __grid_constant__ CUtensorMap tm_dv, const float* __restrict__ lse,
                       const float* __restrict__ Dd, float* __restrict__ dq, long long lddq, int T, int H, int Hkv,
                       int Bsz, int window) {
  extern __shared__ uint8_t ab_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ab_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + AB2_KV_TILE;
  uint8_t* sQ = sV + AB2_KV_TILE;                  // AB2_STAGES stages
  uint8_t* sDO = sQ + AB2_STAGES * AB2_Q_TILE;     // AB2_STAGES stages
  uint8_t* sDS = sDO + AB2_STAGES * AB2_Q_TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + AB2_PS_TILE);
  uint64_t* kv_full = bars + 0;
  uint64_t* qdo_full = bars + 1;                 // [AB2_STAGES] TMA bytes + one arrival after LSE / D are stored
  uint64_t* qdo_empty = bars + 1 + AB2_STAGES;   // [AB2_STAGES]
  uint64_t* s_full = bars + 1 + 2 * AB2_STAGES;
  uint64_t* s_empty = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* ds_free = s_full + 3;
  uint64_t* dq_full = s_full + 4;
  uint64_t* dq_free = s_full + 5;
  uint64_t* acc_done = s_full + 6;
  uint64_t* drain = s_full + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sLD = reinterpret_cast<float*>(bars + 32);  // [AB2_STAGES][lse*log2e 64 | D 64]

  const int nkb = (T + AB2_BK - 1) / AB2_BK;
  const int npairs = Hkv * Bsz;
  const int grp = blockIdx.x / (AB2_GROUP * nkb);
  const int gsize = min(AB2_GROUP, npairs - grp * AB2_GROUP);  // the last group may be smaller
  const int wg = blockIdx.x - grp * AB2_GROUP * nkb;
  const int kb = wg / gsize;
  const int pair = grp * AB2_GROUP + wg % gsize;
  const int kvh = pair % Hkv, b = pair / Hkv;
  const int G = H / Hkv;
  const int k0 = kb * AB2_BK;
  const int row_base = b * T;
  const int qt_lo = k0 / AB2_BQ;
  const int q_hi = (window >= 0) ? min(T - 1, k0 + AB2_BK - 1 + window) : T - 1;
  const int nq = q_hi / AB2_BQ - qt_lo + 1;
  const int steps = G * nq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < AB2_STAGES; ++i) {
      mbar_init(&qdo_full[i], 2);
      mbar_init(&qdo_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 8);
    mbar_init(p_full, 8);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 8);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_kv);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dk);
    tma_prefetch_desc(&tm_dv);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * AB2_KV_TILE);
      tma_load_2d(sK, &tm_kv, kv_full, (H + kvh) * 128, row_base + k0);
      tma_load_2d(sK + 16384, &tm_kv, kv_full, (H + kvh) * 128 + 64, row_base + k0);
      tma_load_2d(sV, &tm_kv, kv_full, (H + Hkv + kvh) * 128, row_base + k0);
      tma_load_2d(sV + 16384, &tm_kv, kv_full, (H + Hkv + kvh) * 128 + 64, row_base + k0);
    }
    bool ok = true;
    for (int i = 0; i < steps && ok; ++i) {
      const int st = i % AB2_STAGES;
      const int hh = kvh * G + i / nq;
      const int q0 = (qt_lo + i % nq) * AB2_BQ;
      ok = mbar_wait_warp(&qdo_empty[st], ((i / AB2_STAGES) & 1) ^ 1u, abort_flag, ERRW_TIMEOUT_PRODUCER);
      if (!ok) break;
      // the tile loads go out first; LSE and D (plain loads, guarded at the
      // sequence end) overlap them and complete the stage with a second arrival
      if (lane == 0) {
        mbar_arrive_expect_tx(&qdo_full[st], 2 * AB2_Q_TILE);
        uint8_t* q = sQ + st * AB2_Q_TILE;
        uint8_t* d = sDO + st * AB2_Q_TILE;
        tma_load_2d(q, &tm_q, &qdo_full[st], hh * 128, row_base + q0);
        tma_load_2d(q + 8192, &tm_q, &qdo_full[st], hh * 128 + 64, row_base + q0);
        tma_load_2d(d, &tm_do, &qdo_full[st], hh * 128, row_base + q0);
        tma_load_2d(d + 8192, &tm_do, &qdo_full[st], hh * 128 + 64, row_base + q0);
      }
      float* ld = sLD + st * 128;
      for (int e = lane; e < 64; e += 32) {
        const int t = q0 + e;
        const long long li = ((long long)b * H + hh) * T + t;
        ld[e] = (t < T) ? lse[li] * LOG2E : 0.f;
        ld[64 + e] = (t < T) ? Dd[li] : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qdo_full[st]);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = make_idesc(128, 64, false, false, false);   // S^T, dP^T
      constexpr uint32_t ID_G = make_idesc(128, 128, false, true, false);   // dV, dK (A from TMEM)
      constexpr uint32_t ID_Q = make_idesc(128, 64, true, true, false);     // dQ^T
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aDS = smem_u32(sDS);
      bool ok = mbar_wait(kv_full, 0, abort_flag, ERRW_TIMEOUT_MMA);
      auto grads = [&](int i) -> bool {
        const int st = i % AB2_STAGES;
        if (!mbar_wait(p_full, i & 1, abort_flag, ERRW_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + st * AB2_Q_TILE), aDO = smem_u32(sDO + st * AB2_Q_TILE);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          // A: P^T / dS^T in TMEM (lane = key, 8 columns per 16 queries)
          // B: dO / Q as MN-major (hd halves 8 KB apart), K step = 16 query rows
          mma_bf16_ts(tmem + 128, tmem + 448 + k * 8, smem_desc_sw128(aDO + k * 2048, 8192, 1024), ID_G, acc);
          mma_bf16_ts(tmem + 0, tmem + 480 + k * 8, smem_desc_sw128(aQ + k * 2048, 8192, 1024), ID_G, acc);
        }
        if (!mbar_wait(dq_free, (i & 1) ^ 1u, abort_flag, ERRW_TIMEOUT_MMA)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          // A = K^T (MN-major over hd, halves 16 KB apart), B = dS (MN-major over queries), K step = 16 keys
          mma_bf16_ss(tmem + 384, smem_desc_sw128(aK + k * 2048, 16384, 1024),
                      smem_desc_sw128(aDS + k * 2048, 8192, 1024), ID_Q, k > 0 ? 1u : 0u);
        }
        mma_commit(ds_free);
        mma_commit(&qdo_empty[st]);
        mma_commit(dq_full);
        return true;
      };
      for (int i = 0; ok && i < steps; ++i) {
        const int st = i % AB2_STAGES;
        if (!mbar_wait(&qdo_full[st], (i / AB2_STAGES) & 1, abort_flag, ERRW_TIMEOUT_MMA)) { ok = false; break; }
        if (!mbar_wait(s_empty, (i & 1) ^ 1u, abort_flag, ERRW_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + st * AB2_Q_TILE), aDO = smem_u32(sDO + st * AB2_Q_TILE);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          // K-major over hd: A rows = keys (halves 16 KB apart), B rows = queries (halves 8 KB apart)
          const uint32_t ka = (uint32_t)((k >> 2) * 16384 + (k & 3) * 32), kq = (uint32_t)((k >> 2) * 8192 + (k & 3) * 32);
          mma_bf16_ss(tmem + 256, smem_desc_sw128(aK + ka, 16, 1024), smem_desc_sw128(aQ + kq, 16, 1024), ID_S, k > 0);
          mma_bf16_ss(tmem + 320, smem_desc_sw128(aV + ka, 16, 1024), smem_desc_sw128(aDO + kq, 16, 1024), ID_S, k > 0);
        }
        mma_commit(s_full);
        if (i > 0 && !grads(i - 1)) { ok = false; break; }
      }
      if (ok && steps > 0) ok = grads(steps - 1);
      mma_commit(acc_done);
      if (*abort_flag) {
        mma_commit(drain);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0))
          if (globaltimer_ns() - t0 > 100000000ull) { record_error(ERRW_TIMEOUT_DRAIN); break; }
      }
    }
  } else if (warp < 10) {
    // ---------------------------------------------------- softmax backward
    const int qw = warp & 3;
    const int cb = (warp - 2) >> 2;          // queries cb*32 .. cb*32+31 of the tile
    const int r = qw * 32 + lane;            // key row within the tile
    const int key = k0 + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(qw * 32) << 16);
    const float scale = rsqrtf(128.f);
    const float sl2 = LOG2E * scale;
    // queries that see this key: [key, key + W] (or [key, T)) inside the sequence
    const int q_vis_lo = key;
    const int q_vis_hi = (key < T) ? ((window >= 0) ? min(T - 1, key + window) : T - 1) : -1;
    bool ok = true;
    for (int i = 0; i < steps && ok; ++i) {
      const int st = i % AB2_STAGES;
      const int q0 = (qt_lo + i % nq) * AB2_BQ;
      ok = mbar_wait_warp(s_full, i & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE);
      if (!ok) break;
      tc_fence_after();
      const int tq = q0 + cb * 32;  // first query of this warp's columns
      const bool need_mask = (key > tq) || (k0 + AB2_BK - 1 > tq) || (tq + 32 > T) || (k0 + AB2_BK > T) ||
                             (window >= 0 && tq + 31 - k0 > window);
      const float4* l2v = reinterpret_cast<const float4*>(sLD + st * 128 + cb * 32);
      const float4* ddv = reinterpret_cast<const float4*>(sLD + st * 128 + 64 + cb * 32);
      // P^T and dS^T for this warp's 32 queries, packed to bf16 pairs (query
      // 2j in the low half); S^T and dP^T come in with one TMEM round trip
      uint32_t pu[16], du[16];
      {
        uint32_t sv[32], dv[32];
        tmem_ld_32x32b_x32(lane_addr + 256 + cb * 32, sv);
        tmem_ld_32x32b_x32(lane_addr + 320 + cb * 32, dv);
        tmem_ld_wait();
        // S^T / dP^T are in registers: the next step's products may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 a = l2v[g], d = ddv[g];
          const float l2[4] = {a.x, a.y, a.z, a.w}, dd[4] = {d.x, d.y, d.z, d.w};
          float pe[4], de[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = tq + g * 4 + e;
            const bool vis = !need_mask || (t >= q_vis_lo && t <= q_vis_hi);
            pe[e] = vis ? fast_exp2(fmaf(__uint_as_float(sv[g * 4 + e]), sl2, -l2[e])) : 0.f;
            de[e] = pe[e] * (__uint_as_float(dv[g * 4 + e]) - dd[e]) * scale;
          }
          pu[g * 2] = pack_bf16(pe[0], pe[1]);
          pu[g * 2 + 1] = pack_bf16(pe[2], pe[3]);
          du[g * 2] = pack_bf16(de[0], de[1]);
          du[g * 2 + 1] = pack_bf16(de[2], de[3]);
        }
      }
      // the previous step's dV/dK/dQ MMAs must be done reading P^T / dS^T
      if (i > 0) {
        ok = mbar_wait_warp(ds_free, (i - 1) & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE);
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_32x32b_x16(lane_addr + 448 + cb * 16, pu);
      tmem_st_32x32b_x16(lane_addr + 480 + cb * 16, du);
      uint8_t* drow = sDS + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int cc = cb * 4 + c;  // 16-byte chunk (8 queries) within the 128-byte row
        *reinterpret_cast<uint4*>(drow + ((cc ^ (r & 7)) << 4)) =
            make_uint4(du[c * 4], du[c * 4 + 1], du[c * 4 + 2], du[c * 4 + 3]);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // dK, dV rows (bf16) for this CTA's keys, columns cb*64 .. cb*64+63, through
    // two 32-row x 128-byte swizzled staging tiles per warp in the (now idle) Q/dO ring
    if (__all_sync(0xffffffffu, ok) && mbar_wait_warp(acc_done, 0, abort_flag, ERRW_TIMEOUT_EPILOGUE)) {
      tc_fence_after();
      uint8_t* stg = sQ + (warp - 2) * 2 * 4096;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(lane_addr + which * 128 + cb * 64, v0);
        tmem_ld_32x32b_x32(lane_addr + which * 128 + cb * 64 + 32, v1);
        tmem_ld_wait();
        uint8_t* prow = stg + which * 4096 + lane * 128;
#pragma unroll
        for (int g = 0; g < 8; ++g) {  // 16-byte chunk g: columns 8g .. 8g+7
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c0 = g * 8 + 2 * j;
            const float lo = __uint_as_float(c0 < 32 ? v0[c0] : v1[c0 - 32]);
            const float hi = __uint_as_float(c0 + 1 < 32 ? v0[c0 + 1] : v1[c0 + 1 - 32]);
            w[j] = pack_bf16(lo, hi);
          }
          *reinterpret_cast<uint4*>(prow + ((g ^ (lane & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && k0 + qw * 32 < T) {  // (a box wholly past the sequence end is not issued)
        tma_store_3d(&tm_dk, stg, kvh * 128 + cb * 64, k0 + qw * 32, b);
        tma_store_3d(&tm_dv, stg + 4096, kvh * 128 + cb * 64, k0 + qw * 32, b);
        bulk_commit_group();
        bulk_wait_read0();  // the staging tiles are read before the CTA ends
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------- dQ epilogue
    // TMEM gives each thread one hd column of dQ^T (64 queries).  A 4x4
    // transpose among each group of 4 lanes (two butterfly stages of
    // shuffles) turns that into 4 consecutive hd values of one query, so one
    // 16-byte fp32 reduction per thread covers 4 rows x 128 bytes per warp:
    // a quarter of the reduction instructions of one-float-per-lane.
    const int qw = warp & 3;
    const int qh = (warp - 10) >> 2;  // queries qh*32 .. qh*32+31 of the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(qw * 32) << 16);
    bool ok = true;
    for (int i = 0; i < steps; ++i) {
      const int hh = kvh * G + i / nq;
      const int q0 = (qt_lo + i % nq) * AB2_BQ;
      ok = ok && mbar_wait_warp(dq_full, i & 1, abort_flag, ERRW_TIMEOUT_EPILOGUE);
      uint32_t v0[32];
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(lane_addr + 384 + qh * 32, v0);
        tmem_ld_wait();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
      if (ok) {
        const int m4 = lane & 3;
        const bool b1 = (m4 & 2) != 0, b0 = (m4 & 1) != 0;
        const int nv = T - q0 - qh * 32;  // query rows of this half inside the sequence
        float* dst = dq + (long long)(row_base + q0 + qh * 32 + m4) * lddq + hh * 128 + qw * 32 + (lane & ~3);
#pragma unroll
        for (int qb = 0; qb < 8; ++qb) {
          // a[j]: query 4qb+j at this lane's hd  ->  a[j]: query 4qb+m4 at hd (lane&~3)+j
          float a[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) a[j] = __uint_as_float(v0[qb * 4 + j]);
#pragma unroll
          for (int t = 0; t < 2; ++t) {  // swap the off-diagonal 2x2 blocks (lane bit 1)
            const float y = __shfl_xor_sync(0xffffffffu, b1 ? a[t] : a[2 + t], 2);
            if (b1) a[t] = y; else a[2 + t] = y;
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {  // transpose inside each 2x2 block (lane bit 0)
            const float y = __shfl_xor_sync(0xffffffffu, b0 ? a[2 * t] : a[2 * t + 1], 1);
            if (b0) a[2 * t] = y; else a[2 * t + 1] = y;
          }
          if (4 * qb + m4 < nv) red_add_v4_f32(dst + (long long)(4 * qb) * lddq, a[0], a[1], a[2], a[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gptb
