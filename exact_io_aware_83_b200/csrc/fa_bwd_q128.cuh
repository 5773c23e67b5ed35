// fa_bwd_q128.cuh - backward main kernel for dense d = 128 attention (full or causal)
// with 128-query steps.
//
// The work is that of fa_bwd_main_kernel (FlashAttention-2 page, "Algorithm" and the
// next-generation page, "Recomputation": recompute S^T = K Q^T and P^T from the saved
// logsumexp, then dV += P^T dO, dP^T = V dO^T, dS = P o (dP - Delta), dK += dS^T Q and
// dQ += dS K), one CTA per 128-key block, but each step covers 128 query rows.  Every
// product of a step is then an M = 128, N = 128 tcgen05 MMA: S^T, dP^T and dQ^T are
// [128 x 128] where 64-query steps make them [128 x 64], and on B200 an N = 64 product
// costs about as much tensor-core time as an N = 128 one.
//
// Tensor memory holds dV, dK, S^T and dP^T at 128 fp32 columns each, all 512 columns, so
// dQ^T is accumulated into the dP^T columns once the elementwise warps have read dP^T
// (their dS^T arrival orders the read before the MMA), and the next step's dP^T is issued
// only after the dQ drain has read dQ^T back.  Shared memory (226.6 KB) holds K and V, two
// Q stages with their LSE rows, one dO stage with its Delta row, dS^T and a 32 KB staging
// buffer for the drain's fp32 TMA reduce-adds of dQ.  The loader writes the next step's
// Delta only after the elementwise warps have finished this step's dS^T.
//
// Roles: warps 0-7 P^T and dS^T (two warpgroups, 64 query columns each; thread = key
// row), 8-11 the dQ drain (thread = d column), 12 the MMA issuer, 13 the loader.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct Q128Layout {
  static constexpr int kBQ = 128;
  static constexpr int kChunk = 128 * 128;          // [128 rows x 64] bf16 box, 16 KB
  static constexpr int kTile = 2 * kChunk;          // [128 x 128] bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;       // Q ring: two stages
  static constexpr int kOffDO = kOffQ + 2 * kTile;  // one dO stage
  static constexpr int kOffDS = kOffDO + kTile;     // dS^T: two [128 keys x 64 queries] chunks
  static constexpr int kOffDQ = kOffDS + kTile;     // dQ staging: [kDQRows queries x 128] fp32
  static constexpr int kDQRows = 64;
  static constexpr int kOffLse = kOffDQ + kDQRows * 128 * 4;  // [Q stage][128] fp32 (log2 units)
  static constexpr int kOffDelta = kOffLse + 2 * kBQ * 4;     // [128] fp32, with the dO stage
  static constexpr int kOffBar = kOffDelta + kBQ * 4;
  enum {
    kBarKV,
    kBarQFull,
    kBarQEmpty = kBarQFull + 2,
    kBarDOFull = kBarQEmpty + 2,
    kBarDOEmpty,
    kBarS,
    kBarDP,
    kBarP,
    kBarDS,
    kBarDSEmpty,
    kBarDQ,
    kBarDQEmpty,
    kBarFinal,
    kBarDrain,
    kNumBars
  };
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // tensor memory: dV | dK | S^T | dP^T (dQ^T shares the dP^T columns)
  static constexpr uint32_t kTmDV = 0, kTmDK = 128, kTmS = 256, kTmDP = 384;
  // Query columns per elementwise warpgroup.  A warpgroup packs its bf16 P^T into the
  // first 32 of its own 64 S^T columns, so K-step kk (16 queries) sits at pcol(kk).
  static constexpr int kHC = 64;
  __host__ __device__ static constexpr uint32_t pcol(int kk) {
    return static_cast<uint32_t>((kk / 4) * kHC + (kk % 4) * 8);
  }
  static_assert(kSmemBytes <= 232448, "shared-memory budget");
};

template <int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_q128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using L = Q128Layout;
  constexpr int BQ = L::kBQ;
  constexpr int HC = L::kHC;
  constexpr uint32_t kSite = 7;  // kernel id in the device status word
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  float *lse_s = reinterpret_cast<float *>(smem + L::kOffLse);
  float *delta_s = reinterpret_cast<float *>(smem + L::kOffDelta);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };
  const uint32_t sK = base + L::kOffK, sV = base + L::kOffV;
  const uint32_t sQ = base + L::kOffQ, sDO = base + L::kOffDO;
  const uint32_t sDS = base + L::kOffDS, sDQ = base + L::kOffDQ;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- unit: (b, kv head, key block) in the order unit_order gives
  int head, kb;
  unit_order(static_cast<int>(blockIdx.x), p.B * p.Hkv, p.nkb, p.tsz, p.tail, head, kb);
  const int kvh = head % p.Hkv;
  const int b = head / p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int kv0 = kb * 128;
  // 128-row query blocks; under the causal mask only those from the diagonal on see a key
  // of this block.  kb < ceil(N / 128), so every CTA has at least one step per head.
  const int q_first = MODE == kAttnCausal ? kb : 0;
  const int nq = (p.N + BQ - 1) / BQ - q_first;
  const int T = g * nq;  // steps: (query head of the group, query block)
  const int kv_c2 = b * p.Hkv + kvh;
  auto step_head = [&](int i) { return kvh * g + i / nq; };
  auto step_q0 = [&](int i) { return (q_first + i % nq) * BQ; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == L::kBarP || i == L::kBarDS) cnt = 8;  // one arrival per elementwise warp
      if (i == L::kBarDQEmpty) cnt = 4;              // one per dQ-drain warp
      // Q and dO stages: the TMA expect-tx arrival plus the arrival after the LSE (Delta)
      // stores.
      if (i == L::kBarQFull || i == L::kBarQFull + 1 || i == L::kBarDOFull) cnt = 2;
      mbar_init(bar(i), cnt);
    }
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];

  if (warp == 13) {
    // ================================================================ loader
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar(L::kBarKV), 2 * L::kTile);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_3d(sK + c * L::kChunk, &tm_k, bar(L::kBarKV), c * 64, kv0, kv_c2);
        tma_load_3d(sV + c * L::kChunk, &tm_v, bar(L::kBarKV), c * 64, kv0, kv_c2);
      }
    }
    // A step's LSE and Delta values (4 of each a lane) are read from global memory one
    // iteration early, so that their latency overlaps this iteration's waits instead of
    // delaying the next Q load.  Query rows past N get LSE = +inf, so their probabilities
    // (and dS) are exactly 0.
    auto fetch = [&](int k, float (&lv)[4], float (&dv)[4]) {
      const int qk = step_q0(k);
      const size_t rk = static_cast<size_t>(b * p.Hq + step_head(k)) * p.N;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = qk + lane + 32 * u;
        lv[u] = q < p.N ? p.lse[rk + q] * 1.4426950408889634f : INFINITY;
        dv[u] = q < p.N ? p.delta[rk + q] : 0.f;
      }
    };
    float lse_c[4], dl_c[4];
    fetch(0, lse_c, dl_c);
    int issued_q = 0, issued_do = 0;
    for (int i = 0; ok && i < T; ++i) {
      const int st = i & 1;
      const int h = step_head(i), q0 = step_q0(i);
      const int c2 = b * p.Hq + h;
      float lse_n[4], dl_n[4];
      if (i + 1 < T) fetch(i + 1, lse_n, dl_n);
      ok = warp_wait_bounded(bar(L::kBarQEmpty + st), ((i >> 1) & 1) ^ 1, abort_flag,
                             wait_site(kSite, L::kBarQEmpty + st, i));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(L::kBarQFull + st), L::kTile);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sQ + st * L::kTile + c * L::kChunk, &tm_q, bar(L::kBarQFull + st), c * 64, q0, c2);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) lse_s[st * BQ + lane + 32 * u] = lse_c[u];
      // The stores above are ordered before lane 0's arrival by the warp barrier; the
      // phase completes only when that arrival and the TMA bytes are both in.
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarQFull + st));
      ++issued_q;
      // dO_i once dV and dP^T have read dO_{i-1}; Delta_i once dS^T_{i-1}, the last reader
      // of Delta_{i-1}, is done.
      ok = warp_wait_bounded(bar(L::kBarDOEmpty), (i & 1) ^ 1, abort_flag, wait_site(kSite, L::kBarDOEmpty, i));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(L::kBarDOFull), L::kTile);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sDO + c * L::kChunk, &tm_do, bar(L::kBarDOFull), c * 64, q0, c2);
      }
      ++issued_do;
      const bool ds_ok =
          i == 0 || warp_wait_bounded(bar(L::kBarDS), (i - 1) & 1, abort_flag, wait_site(kSite, L::kBarDS, i - 1));
      if (ds_ok) {
#pragma unroll
        for (int u = 0; u < 4; ++u) delta_s[lane + 32 * u] = dl_c[u];
      }
      // Arrive even after an abort, so that the phase completes once the bytes are in.
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarDOFull));
      if (!(ok = ds_ok)) break;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        lse_c[u] = lse_n[u];
        dl_c[u] = dl_n[u];
      }
    }
    // Loads still in flight after an abort land before the CTA exits: the last two Q
    // stages and the last dO load (each earlier one was consumed before the next issued).
    if (lane == 0) {
      for (int i = issued_q > 2 ? issued_q - 2 : 0; i < issued_q; ++i)
        wait_drain(bar(L::kBarQFull + (i & 1)), (i >> 1) & 1, 100000000ull);
      if (issued_do > 0) wait_drain(bar(L::kBarDOFull), (issued_do - 1) & 1, 100000000ull);
      wait_drain(bar(L::kBarKV), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 12) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_st = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T: both K-major
      constexpr uint32_t id_kv = idesc_bf16_f32(128, 128, 0, 1);  // dV, dK: B (dO / Q) MN-major
      constexpr uint32_t id_dq = idesc_bf16_f32(128, 128, 1, 1);  // dQ^T = K^T dS^T: both MN-major
      // S^T (or dP^T) = A B^T over d: A = K (or V) [128 x 128], B = Q_i (or dO_i) [128 x 128].
      auto issue_st = [&](uint32_t dst, uint32_t a0, uint32_t b0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk / 4) * L::kChunk + (kk % 4) * 32;
          mma_ss(tmem + dst, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024), id_st, kk > 0);
        }
      };
      // dV += P^T dO_j : M = 128 keys, N = 128 d, K = 128 queries; P^T (bf16) in TMEM.
      auto issue_dv = [&](int j) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + L::kTmDV, tmem + L::kTmS + L::pcol(kk), sdesc_sw128(sDO + kk * 2048, L::kChunk, 1024),
                 id_kv, (j > 0 || kk > 0));
      };
      auto wt = [&](int b_, uint32_t parity, int j) {
        return wait_bounded(bar(b_), parity, abort_flag, wait_site(kSite, b_, j));
      };
      // Issue order, which fills the wait for the dQ drain with the next step's dV:
      //   prologue  S^T_0, dP^T_0, dV_0, S^T_1
      //   step i    dK_i, dQ^T_i, dV_{i+1}, dP^T_{i+1} (once dQ^T_i is drained), S^T_{i+2}
      // S^T_j overwrites P^T_{j-1} after dV_{j-1} has read it (issue order); dO_j is
      // released after dV_j and dP^T_j, its two readers.
      bool ok = wt(L::kBarKV, 0, 0) && wt(L::kBarQFull, 0, 0) && wt(L::kBarDOFull, 0, 0);
      if (ok) {
        tc_fence_after_sync();
        issue_st(L::kTmS, sK, sQ);
        tc_commit(bar(L::kBarS));
        issue_st(L::kTmDP, sV, sDO);
        tc_commit(bar(L::kBarDP));
        ok = wt(L::kBarP, 0, 0);
      }
      if (ok) {
        tc_fence_after_sync();
        issue_dv(0);
        tc_commit(bar(L::kBarDOEmpty));
        if (T > 1 && (ok = wt(L::kBarQFull + 1, 0, 1))) {
          tc_fence_after_sync();
          issue_st(L::kTmS, sK, sQ + L::kTile);
          tc_commit(bar(L::kBarS));
        }
      }
      for (int i = 0; ok && i < T; ++i) {
        const int st = i & 1;
        const uint32_t q_t = sQ + st * L::kTile;
        // dK += dS^T Q_i : M = 128 keys, N = 128 d, K = 128 queries; dS^T K-major in two chunks.
        if (!(ok = wt(L::kBarDS, i & 1, i))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::kTmDK, sdesc_sw128(sDS + (kk / 4) * L::kChunk + (kk % 4) * 32, 16, 1024),
                 sdesc_sw128(q_t + kk * 2048, L::kChunk, 1024), id_kv, (i > 0 || kk > 0));
        tc_commit(bar(L::kBarQEmpty + st));
        // dQ_i^T = K^T dS^T : M = 128 d, N = 128 queries, K = 128 keys, into the dP^T
        // columns, which the elementwise warps read before their dS^T arrival.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::kTmDP, sdesc_sw128(sK + kk * 2048, L::kChunk, 1024),
                 sdesc_sw128(sDS + kk * 2048, L::kChunk, 1024), id_dq, kk > 0);
        tc_commit(bar(L::kBarDQ));
        tc_commit(bar(L::kBarDSEmpty));
        if (i + 1 < T) {
          const int j = i + 1;
          if (!(ok = wt(L::kBarP, j & 1, j) && wt(L::kBarDOFull, j & 1, j))) break;
          tc_fence_after_sync();
          issue_dv(j);
          // dP^T_j overwrites dQ^T_i once the drain has read it.
          if (!(ok = wt(L::kBarDQEmpty, i & 1, i))) break;
          tc_fence_after_sync();
          issue_st(L::kTmDP, sV, sDO);
          tc_commit(bar(L::kBarDP));
          tc_commit(bar(L::kBarDOEmpty));
          if (j + 1 < T) {
            if (!(ok = wt(L::kBarQFull + ((j + 1) & 1), ((j + 1) >> 1) & 1, j + 1))) break;
            tc_fence_after_sync();
            issue_st(L::kTmS, sK, sQ + ((j + 1) & 1) * L::kTile);
            tc_commit(bar(L::kBarS));
          }
        }
      }
      if (ok) tc_commit(bar(L::kBarFinal));
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ================================================================ P^T / dS^T
    // Thread = one key row (TMEM lane); warpgroup wg owns query columns [wg*HC, wg*HC+HC).
    const int wg = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int kv = kv0 + r;
    const int c0 = wg * HC;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + L::kTmS + lane_off + c0;
    const uint32_t tDP = tmem + L::kTmDP + lane_off + c0;
    const bool row_live = kv < p.N;
    const float sl2 = p.sl2;
    const uint32_t rowp = sDS + wg * L::kChunk + r * 128;  // this row of this warpgroup's dS^T chunk
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
      const int st = i & 1;
      const int q0 = step_q0(i) + c0;  // first query column of this warpgroup
      if (!(ok = warp_wait_bounded(bar(L::kBarQFull + st), (i >> 1) & 1, abort_flag,
                                   wait_site(kSite, L::kBarQFull + st, i))))
        break;
      if (!(ok = warp_wait_bounded(bar(L::kBarS), i & 1, abort_flag, wait_site(kSite, L::kBarS, i)))) break;
      tc_fence_after_sync();
      const float4 *lse4 = reinterpret_cast<const float4 *>(lse_s + st * BQ + c0);
      const float4 *dl4 = reinterpret_cast<const float4 *>(delta_s + c0);
      // P^T over the warpgroup's 64 columns from one TMEM load: exponentials, masks (key
      // rows past N and, causal, queries before this key; query rows past N already have
      // P = 0), then the bf16 pairs into the first 32 of its S^T columns.  The packed pairs
      // are also P for this step's dS: 64 fp32 values would leave too few of a thread's 128
      // registers to load dP^T in one piece.
      uint32_t pk[HC / 2];
      {
        uint32_t rr[HC];
        tmem_ld_x64(tS, rr);
        const bool diag = MODE == kAttnCausal && q0 < kv;
#pragma unroll
        for (int c4 = 0; c4 < HC / 4; ++c4) {
          const float4 l = lse4[c4];
          float e[4];
          e[0] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 0]), sl2, -l.x));
          e[1] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 1]), sl2, -l.y));
          e[2] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 2]), sl2, -l.z));
          e[3] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 3]), sl2, -l.w));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (!row_live || (diag && q0 + 4 * c4 + j < kv)) e[j] = 0.f;
          pk[2 * c4] = pack_bf16x2(e[0], e[1]);
          pk[2 * c4 + 1] = pack_bf16x2(e[2], e[3]);
        }
        tmem_st_x32(tS, pk);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarP));

      // dS^T = P^T o (dP^T - Delta) into this row of shared memory (128-byte swizzled), once
      // the previous step's dK and dQ^T have read dS^T.
      if (!(ok = warp_wait_bounded(bar(L::kBarDSEmpty), (i & 1) ^ 1, abort_flag,
                                   wait_site(kSite, L::kBarDSEmpty, i))))
        break;
      // Delta_i is in once dO_i's barrier phase is complete (the MMA waited for it too).
      if (!(ok = warp_wait_bounded(bar(L::kBarDOFull), i & 1, abort_flag, wait_site(kSite, L::kBarDOFull, i))))
        break;
      if (!(ok = warp_wait_bounded(bar(L::kBarDP), i & 1, abort_flag, wait_site(kSite, L::kBarDP, i)))) break;
      tc_fence_after_sync();
      {
        uint32_t rr[HC];
        tmem_ld_x64(tDP, rr);
#pragma unroll
        for (int uu = 0; uu < HC / 8; ++uu) {  // 16-byte unit uu: columns 8uu .. 8uu + 7
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * uu + e;  // pair j: columns 2j (low half) and 2j + 1
            const float4 dd = dl4[j / 2];
            const float d0 = (j & 1) ? dd.z : dd.x, d1 = (j & 1) ? dd.w : dd.y;
            const float p0 = __uint_as_float(pk[j] << 16), p1 = __uint_as_float(pk[j] & 0xFFFF0000u);
            w[e] = pack_bf16x2(p0 * (__uint_as_float(rr[2 * j]) - d0), p1 * (__uint_as_float(rr[2 * j + 1]) - d1));
          }
          st_shared_v4(rowp + ((uu ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      // dQ^T is accumulated into the dP^T columns after this arrival.
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarDS));
    }

    // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK, as bf16 into the
    // V / K tiles' shared memory (no longer read), then one thread TMA-stores both.
    bool okw = ok && warp_wait_bounded(bar(L::kBarFinal), 0, abort_flag, wait_site(kSite, L::kBarFinal, 0));
    okw = named_bar_and(1, 256, okw && *abort_flag == 0);
    if (okw) {
      tc_fence_after_sync();
      const uint32_t tacc = tmem + (wg ? L::kTmDK : L::kTmDV) + lane_off;
      const float mul = wg ? p.scale : 1.f;
      const uint32_t stage = wg ? sK : sV;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld_x32(tacc + cc * 32, o);
        const uint32_t rowbase = stage + (cc / 2) * L::kChunk + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = (cc % 2) * 4 + uu;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * mul, __uint_as_float(o[8 * uu + 2 * e + 1]) * mul);
          st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 256);
      if (threadIdx.x == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_store_3d(&tm_dv, sV + c * L::kChunk, c * 64, kv0, kv_c2);
          tma_store_3d(&tm_dk, sK + c * L::kChunk, c * 64, kv0, kv_c2);
        }
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    }
  } else {
    // ================================================================ dQ^T drain (warps 8-11)
    // Thread = one d column (TMEM lane).  Per step: read query columns 0-63 of dQ^T, stage
    // them as [64 x 128] fp32 rows and reduce-add them into dQacc; read columns 64-127 and
    // release the dP^T columns to the MMA issuer; then stage and reduce those once the first
    // reduce has read the staging buffer.  (128 registers a thread do not hold all 128
    // columns at once.)
    const int wq = warp - 8;
    const int dl = wq * 32 + lane;  // d column (TMEM lane)
    const uint32_t tDQ = tmem + L::kTmDP + (static_cast<uint32_t>(wq * 32) << 16);
    float *stage = reinterpret_cast<float *>(smem + L::kOffDQ);
    const int tid = threadIdx.x - 256;
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
      // The warpgroup leaves the loop together: the named barriers below need all four warps.
      ok = warp_wait_bounded(bar(L::kBarDQ), i & 1, abort_flag, wait_site(kSite, L::kBarDQ, i));
      if (!(ok = named_bar_and(2, 128, ok))) break;
      tc_fence_after_sync();
      const int h = step_head(i), q0 = step_q0(i);
      const int c2 = b * p.Hq + h;
      uint32_t acc[64];
      tmem_ld_x64(tDQ, acc);
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        if (hp == 1) {
          tmem_ld_x64(tDQ + 64, acc);
          // The dP^T columns are free for the next step once all four warps have read them.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::kBarDQEmpty));
          // Rows from q0 + 64 on add nothing when they start past N (uniform).
          if (q0 + 64 >= p.N) break;
        }
        // The previous reduce must have finished reading the staging buffer.
        if (tid == 0) bulk_wait_group_read0();
        named_bar_sync(2, 128);
#pragma unroll
        for (int c = 0; c < 64; ++c) stage[c * 128 + dl] = __uint_as_float(acc[c]);
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (tid == 0) {
          tma_reduce_add_3d(&tm_dqacc, sDQ, 0, q0 + hp * 64, c2);
          bulk_commit_group();
        }
      }
    }
    if (tid == 0) bulk_wait_group0();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

template <int MODE>
inline bool bwd_launch_q128(EncodeTiledFnBwd enc, const void *q, const void *k, const void *v, const void *dout,
                            void *dk, void *dv, float *dqacc, int B, int Hq, int Hkv, int N, const BwdParams &p,
                            cudaStream_t s) {
  using L = Q128Layout;
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  const long long hq = static_cast<long long>(B) * Hq, hkv = static_cast<long long>(B) * Hkv;
  if (!bwd_map(enc, &tq, q, false, 128, N, hq, 64, L::kBQ) || !bwd_map(enc, &tdo, dout, false, 128, N, hq, 64, L::kBQ) ||
      !bwd_map(enc, &tk, k, false, 128, N, hkv, 64, 128) || !bwd_map(enc, &tv, v, false, 128, N, hkv, 64, 128) ||
      !bwd_map(enc, &tdk, dk, false, 128, N, hkv, 64, 128) || !bwd_map(enc, &tdv, dv, false, 128, N, hkv, 64, 128) ||
      !bwd_map(enc, &tdq, dqacc, true, 128, N, hq, 128, L::kDQRows))
    return false;
  const unsigned grid = static_cast<unsigned>(B) * Hkv * p.nkb;
  if (grid == 0) return true;
  fa_bwd_q128_kernel<MODE><<<grid, kBwdThreads, L::kSmemBytes, s>>>(tq, tk, tv, tdo, tdk, tdv, tdq, p);
  return cudaGetLastError() == cudaSuccess;
}

}  // namespace fa
