// fa_bwd_pair.cuh - backward main kernel for d = 256 (dense full or causal attention) as
// a cluster of two CTAs on two SMs that split the work by role and exchange bf16 tiles
// through distributed shared memory.
//
// The gradient is the one fa_bwd.cuh states (recompute P from Q, K and the LSE; dP = dO V^T;
// dS = P (dP - Delta); dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K).  At d = 256 one
// SM cannot hold dK and dV of a 128-key block in tensor memory next to the score tiles
// (2 x 256 fp32 columns is the whole of it), so two CTAs share each key block.  Splitting
// the d columns (the single-CTA layout) makes both CTAs recompute S^T and dP^T over all
// 256 columns, and its 32-row query steps run the tensor core at N = 32.  This kernel
// splits by role instead, with 64-row query steps:
//   rank 0 (S role):  S^T = K Q^T (K, Q in full), P = exp2(S^T scale log2e - LSE2) ->
//                     P^T as bf16 into rank 1's shared memory;
//                     dK[:, 0:128] += dS^T Q[:, 0:128];  dQ^T = K^T dS^T (all 256 columns,
//                     two 128-row halves) -> fp32 TMA reduce-add into the dQ accumulator.
//   rank 1 (dP role): dP^T = V dO^T (V, dO in full), dS^T = P^T (dP^T - Delta) -> bf16, its
//                     own copy and one into rank 0's shared memory;
//                     dV += P^T dO (all 256 columns, N = 256);  dK[:, 128:256] += dS^T
//                     Q[:, 128:256].
// Each rank issues 24 (rank 1) to 36 (rank 0) tcgen05 MMAs per 64 query rows, against 88
// for the d-split layout.  The tiles cross between the SMs once each way per step (16 KB
// of P^T, 16 KB of dS^T): the elementwise warps write the tile into a local send buffer,
// and one thread copies it with a shared::cta -> shared::cluster bulk copy whose bytes
// complete on the receiver's "full" mbarrier (after a remote arrive.expect_tx), so no warp
// waits for the remote stores.  Send and receive buffers are double-buffered; a receive
// buffer's "free" barrier lives in the sender's CTA (arrivals from the receiver's
// elementwise warps and from a multicast tcgen05.commit of the receiver's MMAs), and its
// completion also tells the sender that the copy out of its send buffer has finished.
// No TMA load uses cluster multicast.
//
// Roles inside each CTA: warps 0-7 elementwise (two warpgroups, one key row per thread,
// 32 of the 64 query columns per warpgroup); warps 8-11 drain dQ^T (rank 0; idle on rank
// 1); warp 12 issues the MMAs; warp 13 loads.  Every wait is bounded (fa_common.cuh); both
// CTAs always reach the closing cluster barrier.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct PairLayout {
  static constexpr int kD = 256, kBQ = 64;
  static constexpr int kKChunk = 128 * 128;         // [128 rows x 64 cols] bf16 box
  static constexpr int kKTile = 4 * kKChunk;        // K (rank 0) or V (rank 1), 64 KB
  static constexpr int kQChunk = kBQ * 128;         // [64 rows x 64 cols] bf16 box
  static constexpr int kQTile = 4 * kQChunk;        // Q or dO, 32 KB
  static constexpr int kXBytes = 128 * 128;         // P^T / dS^T tile [128 keys x 64 q] bf16
  static constexpr int kStages = 2;                 // ring stages (both ranks)
  // rank 0 ring stage: Q; rank 1 ring stage: dO and Q[:, 128:256]
  static constexpr int kStage0Bytes = kQTile;
  static constexpr int kStage1Bytes = kQTile + 2 * kQChunk;
  static constexpr int kDQStage = kBQ * 64 * 4;     // [64 queries x 64 d] fp32 dQ staging
  static constexpr int kOffKV = 0;
  static constexpr int kOffRing = kKTile;
  static constexpr int kRingBytes = kStages * kStage1Bytes;              // 96 KB
  // rank 0 keeps its two dQ staging tiles after its (smaller) ring
  static constexpr int kOffDQ = kOffRing + kStages * kStage0Bytes;
  static constexpr int kOffX = kOffRing + kRingBytes;                    // 2 receive buffers
  static constexpr int kOffY = kOffX + 2 * kXBytes;                      // 2 send buffers
  static constexpr int kOffVec = kOffY + 2 * kXBytes;                    // [stage][64] fp32
  static constexpr int kOffBar = kOffVec + kStages * kBQ * 4;
  // mbarriers (the same offsets in both CTAs: multicast commits and remote arrivals
  // address the peer's barrier by the local offset)
  static constexpr int kBarRingFull = 0;                 // [2]
  static constexpr int kBarRingEmpty = 2;                // [2]
  static constexpr int kBarScore = 4;                    // [2] S^T (rank 0) / dP^T (rank 1) ready
  static constexpr int kBarSFree = 6;                    // [2] rank 0: S^T read by the warps
  static constexpr int kBarXFull = 8;                    // [2] my receive buffer holds its tile
  static constexpr int kBarXFree = 10;                   // [2] the peer's receive buffer is free
  static constexpr int kBarDS = 12;                      // [2] rank 1: own dS^T written
  static constexpr int kBarDSEmpty = 14;                 // [2] rank 1: own dS^T read by dK1
  static constexpr int kBarDQFull = 16;                  // [2] rank 0
  static constexpr int kBarDQEmpty = 18;                 // [2] rank 0
  static constexpr int kBarKV = 20;
  static constexpr int kBarFinal = 21;
  static constexpr int kBarDrain = 22;
  static constexpr int kNumBars = 23;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // tensor memory (512 columns)
  static constexpr uint32_t kTmDK0 = 0, kTmS = 128, kTmDQ = 256;          // rank 0
  static constexpr uint32_t kTmDV = 0, kTmDK1 = 256, kTmDP = 384;         // rank 1
  static_assert(kOffDQ + 2 * kDQStage <= kOffX, "rank 0 dQ staging inside the ring region");
  static_assert(kSmemBytes <= 232448, "shared-memory budget");
};

template <int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using L = PairLayout;
  constexpr int BQ = L::kBQ;
  static_assert(MODE == kAttnFull || MODE == kAttnCausal, "dense variants only");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  float *vec = reinterpret_cast<float *>(smem + L::kOffVec);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };
  const uint32_t sKV = base + L::kOffKV, sRing = base + L::kOffRing, sX = base + L::kOffX, sY = base + L::kOffY;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  // ---- unit: (b, kv head, key block), the same for both CTAs of the cluster
  int head, kb;
  unit_order(static_cast<int>(blockIdx.x) / 2, p.B * p.Hkv, p.nkb, p.tsz, p.tail, head, kb);
  const int kvh = head % p.Hkv;
  const int b = head / p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int kv0 = kb * 128;
  const int q_first = MODE == kAttnCausal ? kv0 / BQ : 0;
  const int nq = (p.N + BQ - 1) / BQ - q_first;
  const int T = g * nq;  // steps: (query head of the group, 64-row query block)
  auto step_head = [&](int i) { return kvh * g + i / nq; };
  auto step_q0 = [&](int i) { return (q_first + i % nq) * BQ; };
  auto vec_row = [&](int hh, int q) -> size_t { return static_cast<size_t>(b * p.Hq + hh) * p.N + q; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      const int j = i & ~1;  // first barrier of a pair
      if (j == L::kBarRingFull) cnt = 2;                        // expect-tx + vector stores
      if (j == L::kBarSFree || j == L::kBarDS) cnt = 8;         // one per elementwise warp
      if (j == L::kBarXFree) cnt = rank == 0 ? 9 : 1;           // peer: 8 warps + MMA | MMA
      if (j == L::kBarDQEmpty) cnt = 4;                         // one per drain warp
      // kBarXFull: the peer's arrive.expect_tx plus the bulk copy's bytes (count 1)
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
  // Both CTAs' barriers are initialised before either signals the other.
  cluster_sync_all();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];

  // Bounded wait on a local barrier that the peer CTA arrives on.
  auto wait_peer = [&](uint32_t bar_addr, uint32_t parity, uint32_t site) -> bool {
    if (mbar_try_wait_cluster(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      if (mbar_try_wait_cluster(bar_addr, parity)) return true;
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        if (atomicCAS(&g_fa_status, FA_OK, FA_ERR_DEVICE_TIMEOUT) == FA_OK)
          atomicExch(&g_fa_status_site,
                     static_cast<unsigned long long>(site) | (static_cast<unsigned long long>(blockIdx.x) << 32));
        return false;
      }
    }
  };

  const int kv_c1 = kv0, kv_c2 = b * p.Hkv + kvh;
  constexpr int S = L::kStages;
  auto stage_addr = [&](int st) -> uint32_t {
    return sRing + static_cast<uint32_t>(st) * (rank == 0 ? L::kStage0Bytes : L::kStage1Bytes);
  };

  if (warp == 13) {
    // ================================================================ loader
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(rank == 0 ? &tm_k : &tm_v);
      if (rank == 1) tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar(L::kBarKV), L::kKTile);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tma_load_3d(sKV + c * L::kKChunk, rank == 0 ? &tm_k : &tm_v, bar(L::kBarKV), c * 64, kv_c1, kv_c2);
    }
    int issued = 0;
    for (int i = 0; ok && i < T; ++i) {
      const int st = i % S, use = i / S;
      ok = warp_wait_bounded(bar(L::kBarRingEmpty + st), (use & 1) ^ 1, abort_flag,
                             wait_site(6, L::kBarRingEmpty + st, i));
      if (!ok) break;
      const int h = step_head(i), q0 = step_q0(i);
      if (lane == 0) {
        const int c2 = b * p.Hq + h;
        const uint32_t dst = stage_addr(st);
        if (rank == 0) {
          mbar_arrive_expect_tx(bar(L::kBarRingFull + st), L::kStage0Bytes);
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * L::kQChunk, &tm_q, bar(L::kBarRingFull + st), c * 64, q0, c2);
        } else {
          mbar_arrive_expect_tx(bar(L::kBarRingFull + st), L::kStage1Bytes);
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * L::kQChunk, &tm_do, bar(L::kBarRingFull + st), c * 64, q0, c2);
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d(dst + L::kQTile + c * L::kQChunk, &tm_q, bar(L::kBarRingFull + st), 128 + c * 64, q0, c2);
        }
      }
      // rank 0: LSE * log2(e) (+inf past the sequence, so P = 0 there); rank 1: Delta.
      float *v = vec + st * BQ;
      for (int c = lane; c < BQ; c += 32) {
        const int q = q0 + c;
        const bool live = q < p.N;
        v[c] = rank == 0 ? (live ? p.lse[vec_row(h, q)] * 1.4426950408889634f : INFINITY)
                         : (live ? p.delta[vec_row(h, q)] : 0.f);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarRingFull + st));
      ++issued;
    }
    if (lane == 0) {
      for (int i = issued > S ? issued - S : 0; i < issued; ++i)
        wait_drain(bar(L::kBarRingFull + i % S), (i / S) & 1, 100000000ull);
      wait_drain(bar(L::kBarKV), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 12) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint16_t peer_mask = static_cast<uint16_t>(1u << peer);
      bool ok = wait_bounded(bar(L::kBarKV), 0, abort_flag, wait_site(6, L::kBarKV, 0));
      if (rank == 0) {
        constexpr uint32_t id_s = idesc_bf16_f32(128, BQ, 0, 0);    // S^T = K Q^T, K-major both
        constexpr uint32_t id_dk = idesc_bf16_f32(128, 128, 0, 1);  // dK0 = dS^T Q[:, 0:128]
        constexpr uint32_t id_dq = idesc_bf16_f32(128, BQ, 1, 1);   // dQ^T_h = K[:, h]^T dS^T
        auto issue_s = [&](int i) {  // S^T(i) into score buffer i % 2
          const uint32_t qt = stage_addr(i % S);
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint32_t oa = (kk / 4) * L::kKChunk + (kk % 4) * 32;
            const uint32_t ob = (kk / 4) * L::kQChunk + (kk % 4) * 32;
            mma_ss(tmem + L::kTmS + 64 * (i % 2), sdesc_sw128(sKV + oa, 16, 1024), sdesc_sw128(qt + ob, 16, 1024),
                   id_s, kk > 0);
          }
          tc_commit(bar(L::kBarScore + i % 2));
        };
        for (int s = 0; ok && s < 2 && s < T; ++s) {
          ok = wait_bounded(bar(L::kBarRingFull + s), 0, abort_flag, wait_site(6, L::kBarRingFull + s, s));
          if (ok) {
            tc_fence_after_sync();
            issue_s(s);
          }
        }
        for (int i = 0; ok && i < T; ++i) {
          const int xb = i % 2, st = i % S;
          const uint32_t qt = stage_addr(st), xt = sX + xb * L::kXBytes;
          // dK0 += dS^T Q[:, 0:128] (dS^T from the peer, K-major; Q MN-major, N = 128)
          if (!(ok = wait_peer(bar(L::kBarXFull + xb), (i / 2) & 1, wait_site(6, L::kBarXFull + xb, i)))) break;
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ss(tmem + L::kTmDK0, sdesc_sw128(xt + kk * 32, 16, 1024),
                   sdesc_sw128(qt + kk * 2048, L::kQChunk, 1024), id_dk, (i > 0 || kk > 0));
          tc_commit(bar(L::kBarRingEmpty + st));  // Q(i): S^T(i) and dK0(i) were its readers
          // dQ^T(i), both 128-column halves, into dQ buffer i % 2
          if (!(ok = wait_bounded(bar(L::kBarDQEmpty + xb), ((i / 2) & 1) ^ 1, abort_flag,
                                  wait_site(6, L::kBarDQEmpty + xb, i))))
            break;
          tc_fence_after_sync();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + L::kTmDQ + 128 * xb + 64 * h,
                     sdesc_sw128(sKV + (2 * h) * L::kKChunk + kk * 2048, L::kKChunk, 1024),
                     sdesc_sw128(xt + kk * 2048, 128 * 128, 1024), id_dq, kk > 0);
          }
          tc_commit(bar(L::kBarDQFull + xb));
          tc_commit_mc(bar(L::kBarXFree + xb), peer_mask);  // the peer may send into buffer xb again
          // S^T(i + 2) into the buffer S^T(i) used, once the warps have read it and Q(i + 2)
          // has arrived in the stage Q(i) left
          if (i + 2 < T) {
            if (!(ok = wait_bounded(bar(L::kBarSFree + xb), (i / 2) & 1, abort_flag,
                                    wait_site(6, L::kBarSFree + xb, i))))
              break;
            if (!(ok = wait_bounded(bar(L::kBarRingFull + st), ((i + 2) / S) & 1, abort_flag,
                                    wait_site(6, L::kBarRingFull + st, i + 2))))
              break;
            tc_fence_after_sync();
            issue_s(i + 2);
          }
        }
      } else {
        constexpr uint32_t id_dp = idesc_bf16_f32(128, BQ, 0, 0);   // dP^T = V dO^T
        constexpr uint32_t id_dv = idesc_bf16_f32(128, 256, 0, 1);  // dV = P^T dO, N = 256
        constexpr uint32_t id_dk = idesc_bf16_f32(128, 128, 0, 1);  // dK1 = dS^T Q[:, 128:256]
        auto issue_dp = [&](int i) {  // dP^T(i) into score buffer i % 2
          const uint32_t dt = stage_addr(i % S);
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint32_t oa = (kk / 4) * L::kKChunk + (kk % 4) * 32;
            const uint32_t ob = (kk / 4) * L::kQChunk + (kk % 4) * 32;
            mma_ss(tmem + L::kTmDP + 64 * (i % 2), sdesc_sw128(sKV + oa, 16, 1024), sdesc_sw128(dt + ob, 16, 1024),
                   id_dp, kk > 0);
          }
          tc_commit(bar(L::kBarScore + i % 2));
        };
        if (ok && T > 0) {
          ok = wait_bounded(bar(L::kBarRingFull), 0, abort_flag, wait_site(6, L::kBarRingFull, 0));
          if (ok) {
            tc_fence_after_sync();
            issue_dp(0);
          }
        }
        for (int i = 0; ok && i < T; ++i) {
          const int xb = i % 2, st = i % S;
          const uint32_t dt = stage_addr(st), xt = sX + xb * L::kXBytes, yt = sY + xb * L::kXBytes;
          // dV += P^T dO (P^T from the peer, K-major; dO MN-major, N = 256)
          if (!(ok = wait_peer(bar(L::kBarXFull + xb), (i / 2) & 1, wait_site(6, L::kBarXFull + xb, i)))) break;
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ss(tmem + L::kTmDV, sdesc_sw128(xt + kk * 32, 16, 1024), sdesc_sw128(dt + kk * 2048, L::kQChunk, 1024),
                   id_dv, (i > 0 || kk > 0));
          tc_commit_mc(bar(L::kBarXFree + xb), peer_mask);  // P^T(i)'s buffer read by the MMA
          // dK1 += dS^T Q[:, 128:256] (own dS^T, send buffer xb)
          if (!(ok = wait_bounded(bar(L::kBarDS + xb), (i / 2) & 1, abort_flag, wait_site(6, L::kBarDS + xb, i)))) break;
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ss(tmem + L::kTmDK1, sdesc_sw128(yt + kk * 32, 16, 1024),
                   sdesc_sw128(dt + L::kQTile + kk * 2048, L::kQChunk, 1024), id_dk, (i > 0 || kk > 0));
          tc_commit(bar(L::kBarDSEmpty + xb));
          tc_commit(bar(L::kBarRingEmpty + st));
          // dP^T(i + 1): its buffer held dP^T(i - 1), read before dS^T(i - 1) was written
          if (i + 1 < T) {
            const int st1 = (i + 1) % S;
            if (!(ok = wait_bounded(bar(L::kBarRingFull + st1), ((i + 1) / S) & 1, abort_flag,
                                    wait_site(6, L::kBarRingFull + st1, i + 1))))
              break;
            tc_fence_after_sync();
            issue_dp(i + 1);
          }
        }
      }
      if (ok) tc_commit(bar(L::kBarFinal));
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ================================================================ elementwise
    const int wg = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;  // key row within the block (TMEM lane)
    const int kv = kv0 + r;
    const int c0 = wg * 32;        // this warpgroup's query columns
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const bool row_live = kv < p.N;
    bool ok = true;
    int sent = 0;  // tiles copied to the peer (by thread 0)
    // Every warp reaches the warpgroups' AND-barrier once per step, whatever its waits did,
    // so a wait that gives up makes all eight warps leave the loop together.
    for (int i = 0; i < T; ++i) {
      const int st = i % S, xb = i % 2;
      const int q0 = step_q0(i) + c0;
      const uint32_t yt = sY + xb * L::kXBytes;
      bool good = warp_wait_bounded(bar(L::kBarRingFull + st), (i / S) & 1, abort_flag,
                                    wait_site(6, L::kBarRingFull + st, i)) &&
                  warp_wait_bounded(bar(L::kBarScore + xb), (i / 2) & 1, abort_flag, wait_site(6, L::kBarScore + xb, i));
      uint32_t w[16];
      if (good) {
        tc_fence_after_sync();
        uint32_t rr[32];
        tmem_ld_x32(tmem + (rank == 0 ? L::kTmS : L::kTmDP) + 64 * xb + lane_off + c0, rr);
        const float4 *v4 = reinterpret_cast<const float4 *>(vec + st * BQ + c0);
        if (rank == 0) {
          // P^T = exp2(S^T scale log2e - LSE2) with the masks, as bf16
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::kBarSFree + xb));
          float pr[32];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 l = v4[c4];
            pr[4 * c4 + 0] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 0]), p.sl2, -l.x));
            pr[4 * c4 + 1] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 1]), p.sl2, -l.y));
            pr[4 * c4 + 2] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 2]), p.sl2, -l.z));
            pr[4 * c4 + 3] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 3]), p.sl2, -l.w));
          }
          if (!row_live) {
#pragma unroll
            for (int c = 0; c < 32; ++c) pr[c] = 0.f;
          } else if (MODE == kAttnCausal && q0 < kv) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (q0 + c < kv) pr[c] = 0.f;
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) w[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
        } else {
          // dS^T = P^T (dP^T - Delta) with P^T from the peer
          good = __all_sync(0xffffffffu, wait_peer(bar(L::kBarXFull + xb), (i / 2) & 1,
                                                   wait_site(6, L::kBarXFull + xb, i)));
          if (good) {
            uint32_t pw[16];
            const uint32_t rowp = sX + xb * L::kXBytes + r * 128;
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const int unit = c0 / 8 + uu;
              ld_shared_v4(rowp + ((unit ^ (r & 7)) * 16), pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
            }
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              const float4 dd = v4[c4];
              const float p0 = __uint_as_float(pw[2 * c4] << 16), p1 = __uint_as_float(pw[2 * c4] & 0xFFFF0000u);
              const float p2 = __uint_as_float(pw[2 * c4 + 1] << 16), p3 = __uint_as_float(pw[2 * c4 + 1] & 0xFFFF0000u);
              w[2 * c4] =
                  pack_bf16x2(p0 * (__uint_as_float(rr[4 * c4 + 0]) - dd.x), p1 * (__uint_as_float(rr[4 * c4 + 1]) - dd.y));
              w[2 * c4 + 1] =
                  pack_bf16x2(p2 * (__uint_as_float(rr[4 * c4 + 2]) - dd.z), p3 * (__uint_as_float(rr[4 * c4 + 3]) - dd.w));
            }
            // P^T(i) read (the values above are in registers): one of the buffer's 9 arrivals
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(bar(L::kBarXFree + xb), peer));
            // send buffer xb is also dK1's A operand: dK1(i - 2) must have read it
            good = warp_wait_bounded(bar(L::kBarDSEmpty + xb), ((i / 2) & 1) ^ 1, abort_flag,
                                     wait_site(6, L::kBarDSEmpty + xb, i));
          }
        }
      }
      // Send buffer xb was last copied out for step i - 2; that copy has finished once the
      // peer released its receive buffer xb (the copy's bytes complete before the peer can).
      good = good && __all_sync(0xffffffffu, wait_peer(bar(L::kBarXFree + xb), ((i / 2) & 1) ^ 1,
                                                        wait_site(6, L::kBarXFree + xb, i)));
      if (good) {
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = c0 / 8 + uu;
          st_shared_v4(yt + r * 128 + ((unit ^ (r & 7)) * 16), w[4 * uu], w[4 * uu + 1], w[4 * uu + 2], w[4 * uu + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (rank == 1 && lane == 0) mbar_arrive(bar(L::kBarDS + xb));
      }
      // all 8 warps' rows are in: one thread sends the tile
      if (!named_bar_and(3, 256, good)) {
        ok = false;
        break;
      }
      if (threadIdx.x == 0) {
        const uint32_t pbar = mapa_shared(bar(L::kBarXFull + xb), peer);
        mbar_arrive_expect_tx_cluster(pbar, L::kXBytes);
        bulk_copy_to_cluster(mapa_shared(sX + xb * L::kXBytes, peer), yt, L::kXBytes, pbar);
      }
      ++sent;
    }
    // Before the closing cluster barrier, with or without an abort: every tile this CTA
    // sent has been released by the peer (rank 0: the peer read P^T; rank 1: the peer's MMAs
    // read dS^T), so no copy into the peer's shared memory and no arrival on this CTA's
    // barriers is still in flight.  After an abort the wait ends at its limit, long after
    // any 16 KB copy has landed.
    if (lane == 0) {
      for (int xb = 0; xb < 2 && xb < sent; ++xb) {
        const int uses = (sent - xb + 1) / 2;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_cluster(bar(L::kBarXFree + xb), (uses - 1) & 1))
          if (globaltimer_ns() - t0 > 100000000ull) break;
      }
    }
    __syncwarp();

    // ---- epilogue: bf16 tiles into shared memory that is no longer read, then TMA stores.
    // rank 0: dK[:, 0:128] (scale) into the K tile.  rank 1: dV (256 columns) into the V
    // tile and dK[:, 128:256] into the ring.
    bool okw = ok && warp_wait_bounded(bar(L::kBarFinal), 0, abort_flag, wait_site(6, L::kBarFinal, 0));
    okw = named_bar_and(1, 256, okw && *abort_flag == 0);
    if (okw) {
      tc_fence_after_sync();
      // 32-column chunks: rank 0 has 4 (dK0); rank 1 has 8 of dV then 4 of dK1.
      const int nch = rank == 0 ? 4 : 12;
      const int lo = rank == 0 ? wg * 2 : wg * 6, hi = rank == 0 ? lo + 2 : lo + 6;
      for (int cc = lo; cc < hi && cc < nch; ++cc) {
        const bool is_dv = rank == 1 && cc < 8;
        const int col = is_dv ? cc * 32 : (rank == 0 ? cc * 32 : (cc - 8) * 32);  // column in its tensor
        const uint32_t tsrc = tmem + lane_off +
                              (rank == 0 ? L::kTmDK0 : (is_dv ? L::kTmDV : L::kTmDK1)) + static_cast<uint32_t>(col);
        const float mul = is_dv ? 1.f : p.scale;
        const uint32_t stage = (rank == 1 && !is_dv) ? sRing : sKV;
        uint32_t o[32];
        tmem_ld_x32(tsrc, o);
        const uint32_t rowbase = stage + (col / 64) * L::kKChunk + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = ((col % 64) / 32) * 4 + uu;
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wv[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * mul, __uint_as_float(o[8 * uu + 2 * e + 1]) * mul);
          st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), wv[0], wv[1], wv[2], wv[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 256);
      if (threadIdx.x == 0) {
        if (rank == 0) {
#pragma unroll
          for (int c = 0; c < 2; ++c) tma_store_3d(&tm_dk, sKV + c * L::kKChunk, c * 64, kv_c1, kv_c2);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_store_3d(&tm_dv, sKV + c * L::kKChunk, c * 64, kv_c1, kv_c2);
#pragma unroll
          for (int c = 0; c < 2; ++c) tma_store_3d(&tm_dk, sRing + c * L::kKChunk, 128 + c * 64, kv_c1, kv_c2);
        }
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    }
  } else if (rank == 0) {
    // ================================================================ dQ^T drain (rank 0, warps 8-11)
    // Thread = TMEM lane = d row within a 128-column half.  Per step four passes of a
    // [64 queries x 64 d] fp32 staging tile (half h, rows 64 sub ..), each reduce-added into
    // the accumulator by TMA, through two staging tiles so that one fills while the other's
    // reduce reads it; the two warps whose lanes a pass covers fill it.
    const int wq = warp - 8;
    const int dl = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int tid = threadIdx.x - 256;
    bool ok = true;
    int npass = 0;
    for (int i = 0; ok && i < T; ++i) {
      const int xb = i % 2;
      ok = warp_wait_bounded(bar(L::kBarDQFull + xb), (i / 2) & 1, abort_flag, wait_site(6, L::kBarDQFull + xb, i));
      if (!(ok = named_bar_and(2, 128, ok))) break;
      tc_fence_after_sync();
      const int h_row = step_head(i), q0 = step_q0(i);
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass, ++npass) {
        const int h = pass / 2, sub = pass % 2;
        const bool mine = (wq / 2) == sub;
        const uint32_t stg = base + L::kOffDQ + static_cast<uint32_t>(npass % 2) * L::kDQStage;
        float *stage = reinterpret_cast<float *>(smem + L::kOffDQ + (npass % 2) * L::kDQStage);
        if (tid == 0) bulk_wait_group_read1();  // the reduce from this tile two passes ago
        named_bar_sync(2, 128);
        if (mine) {
          uint32_t acc[64];
          tmem_ld_x64(tmem + L::kTmDQ + 128 * xb + 64 * h + lane_off, acc);
          if (h == 1) {  // this warp's last read of dQ^T(i)
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarDQEmpty + xb));
          }
          const int cl = dl - 64 * sub;
#pragma unroll
          for (int c = 0; c < 64; ++c) stage[c * 64 + cl] = __uint_as_float(acc[c]);
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (tid == 0) {
          tma_reduce_add_3d(&tm_dqacc, stg, 128 * h + 64 * sub, q0, b * p.Hq + h_row);
          bulk_commit_group();
        }
      }
    }
    if (tid == 0) bulk_wait_group0();
  }

  tc_fence_before_sync();
  __syncthreads();
  // No CTA leaves while its peer may still write to its shared memory.
  cluster_sync_all();
  if (warp == 12) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// Host: dense d = 256 backward through the pair kernel (maps over Q / dO with 64-row boxes,
// a [64 x 64] fp32 box for the dQ reduce).  The caller has run fa_bwd_pre_kernel.
template <int MODE>
inline bool bwd_launch_pair(EncodeTiledFnBwd enc, const void *q, const void *k, const void *v, const void *dout,
                            void *dk, void *dv, float *dqacc, int B, int Hq, int Hkv, int N,
                            const BwdParams &p, cudaStream_t s) {
  using L = PairLayout;
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  const long long hq = static_cast<long long>(B) * Hq, hkv = static_cast<long long>(B) * Hkv;
  if (!bwd_map(enc, &tq, q, false, 256, N, hq, 64, L::kBQ) || !bwd_map(enc, &tdo, dout, false, 256, N, hq, 64, L::kBQ) ||
      !bwd_map(enc, &tk, k, false, 256, N, hkv, 64, 128) || !bwd_map(enc, &tv, v, false, 256, N, hkv, 64, 128) ||
      !bwd_map(enc, &tdk, dk, false, 256, N, hkv, 64, 128) || !bwd_map(enc, &tdv, dv, false, 256, N, hkv, 64, 128) ||
      !bwd_map(enc, &tdq, dqacc, true, 256, N, hq, 64, L::kBQ))
    return false;
  const unsigned grid = 2u * static_cast<unsigned>(B) * Hkv * p.nkb;
  if (grid == 0) return true;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = L::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fa_bwd_pair_kernel<MODE>, tq, tk, tv, tdo, tdk, tdv, tdq, p) == cudaSuccess;
}

}  // namespace fa
