// fa_fwd_persist.cuh - persistent forward kernel for dense full and causal attention
// (head dimensions 64 and 128) on sm_100a.
//
// Same computation, roles and pipeline as fa_fwd_kernel (fa_fwd.cuh): two 128-row query
// tiles per work unit sharing every K/V block, the online-softmax recurrence of the
// "FlashAttention1" Q&A page (question on computing the softmax, items 1-3), S and P in
// tensor memory, K/V through a TMA ring.  What differs is the lifetime of a CTA, the
// tile scheduler of the FlashAttention-2 page ("Better Parallelism": work units over
// batch x heads x query blocks) made persistent ("careful scheduling", the Q&A page's key
// innovations, item 6): one CTA per SM walks work units until none is left, so one unit's
// tail (its last P V products and softmax steps, the O epilogue) overlaps the next unit's
// Q load and first Q K^T instead of leaving the SM to a CTA that starts from nothing.
//
//  * Unit assignment is dynamic: CTA c starts with unit c; the TMA warp takes every later
//    unit from a global atomic counter (units numbered heaviest first by unit_order), so
//    an SM that finishes early takes the next heaviest unit, as the hardware does when it
//    starts a new CTA.  The unit index reaches the other roles through a two-slot ring in
//    shared memory.  The counter belongs to one of kUnitSlots slots chosen per launch by
//    the host; the last CTA to finish resets it to zero for the slot's next launch.
//  * The Q slot of a tile is reloaded for the next unit as soon as the tile's last Q K^T
//    of the current unit has completed ("Q free"); the next unit's first Q K^T can then
//    run while the tile's softmax warpgroup is still in the epilogue.
//  * O leaves through one staging tile in shared memory (shared by both query tiles, in
//    epilogue order) and a TMA store; rows past N are clipped by the tensor map.
//  * The next unit's first P V overwrites a tile's O accumulator only after the softmax
//    warpgroup has read it out: the warpgroup reads O (tcgen05.wait::ld) before it signals
//    P of the next unit's first block, and that P V waits for the signal.
//  * Every barrier's phase is counted across units by the roles that wait on it.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

// Launch slots of the unit counters (one slot per launch in flight on the device).
constexpr int kUnitSlots = 64;
__device__ unsigned int g_fa_unit_next[kUnitSlots];  // next unit to hand out, minus gridDim.x
__device__ unsigned int g_fa_unit_done[kUnitSlots];  // CTAs finished

template <int D>
struct FwdPLayout {
  using Base = FwdLayout<D>;
  static constexpr int kChunks = Base::kChunks;
  static constexpr int kChunkBytes = Base::kChunkBytes;
  static constexpr int kTileBytes = Base::kTileBytes;
  static constexpr int kStages = Base::kStages;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffStage = kOffKV + kStages * kTileBytes;  // O staging tile
  static constexpr int kOffBar = kOffStage + kTileBytes;
  static constexpr int kBarQ = 0;                       // [2] Q tile landed
  static constexpr int kBarQFree = 2;                   // [2] last Q K^T of the tile's unit done
  static constexpr int kBarKVFull = 4;                  // [S]
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarS = kBarKVEmpty + kStages;   // [2]
  static constexpr int kBarP = kBarS + 2;               // [2] one arrival per softmax warp
  static constexpr int kBarO = kBarP + 2;               // [2]
  static constexpr int kBarUnitFull = kBarO + 2;        // [2] unit index written
  static constexpr int kBarUnitEmpty = kBarUnitFull + 2;  // [2] read by the 9 consumer warps
  static constexpr int kBarStage = kBarUnitEmpty + 2;   // staging tile free again
  static constexpr int kBarDrain = kBarStage + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // [0] TMEM base, [1] abort, [2..3] unit ring
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kUnitConsumers = 9;         // MMA warp + 8 softmax warps
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return Base::tm_s(t); }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return Base::tm_o(t); }
  static_assert(kSmemBytes <= 232448, "shared-memory budget");
};

// Registers of the persistent kernel's warpgroups: the MMA and TMA warps carry unit state
// across units, so the producer warpgroup keeps 104; 2 * 128 * 200 + 128 * 104 = 64512 <=
// 384 * 168, and per SM sub-partition 200 + 200 + 104 <= 3 * 168.
constexpr uint32_t kFwdPRegsSoftmax = 200;
constexpr uint32_t kFwdPRegsProducer = 104;
static_assert(2 * 128 * kFwdPRegsSoftmax + 128 * kFwdPRegsProducer <= kFwdThreads * kFwdRegsLaunch,
              "register split");

// One work unit of the dense kernel: two query tiles (two query blocks of one head, or
// the same query block of two heads of one K/V group) and their key-block counts.
struct FwdUnit {
  int b, h[2], qb[2], nblk[2], nu;
};

__device__ __forceinline__ void fwd_unit(const FwdParams &p, int u, bool causal, FwdUnit &x) {
  int head, level;
  bool v1 = true;
  if (p.pair_heads) {
    const int hp_count = p.Hq / 2;
    unit_order(u, p.B * hp_count, p.nqb, p.tsz, p.tail, head, level);
    const int hp = head % hp_count;
    x.b = head / hp_count;
    x.h[0] = 2 * hp;
    x.h[1] = 2 * hp + 1;
    x.qb[0] = x.qb[1] = p.nqb - 1 - level;
  } else {
    const int npairs = (p.nqb + 1) / 2;
    unit_order(u, p.B * p.Hq, npairs, p.tsz, p.tail, head, level);
    const int pi = npairs - 1 - level;
    x.h[0] = x.h[1] = head % p.Hq;
    x.b = head / p.Hq;
    x.qb[0] = 2 * pi;
    x.qb[1] = 2 * pi + 1;
    v1 = x.qb[1] < p.nqb;
  }
  x.nblk[0] = causal ? x.qb[0] + 1 : p.nqb;
  x.nblk[1] = !v1 ? 0 : (causal ? x.qb[1] + 1 : p.nqb);
  x.nu = x.nblk[0] > x.nblk[1] ? x.nblk[0] : x.nblk[1];
}

template <int D, int MODE, bool DROP = false>  // MODE: kAttnFull or kAttnCausal
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                          const FwdParams p, int units, int slot) {
  static_assert(MODE == kAttnFull || MODE == kAttnCausal, "dense variants only");
  using L = FwdPLayout<D>;
  constexpr int S = L::kStages;
  constexpr bool CAUSAL = MODE == kAttnCausal;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const uint32_t sQ = base + L::kOffQ;
  const uint32_t sKV = base + L::kOffKV;
  const uint32_t sStage = base + L::kOffStage;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  volatile int *unit_ring = reinterpret_cast<volatile int *>(misc + 2);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int g = p.Hq / p.Hkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == L::kBarP || i == L::kBarP + 1) cnt = 4;
      if (i == L::kBarUnitEmpty || i == L::kBarUnitEmpty + 1) cnt = L::kUnitConsumers;
      mbar_init(bar(i), cnt);
    }
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), L::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];

  // Consumers: the it-th unit index from the ring (-1 ends the walk); false on abort.
  auto take_unit = [&](int it, int &u) -> bool {
    const int sl = it & 1;
    if (!warp_wait_bounded(bar(L::kBarUnitFull + sl), (it >> 1) & 1, abort_flag,
                           wait_site(5, L::kBarUnitFull + sl, it)))
      return false;
    u = unit_ring[sl];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kBarUnitEmpty + sl));
    return true;
  };

  if (warp >= 8) {
  // ================================================================ producer warpgroup
  setmaxnreg_dec<kFwdPRegsProducer>();
  if (warp == 9) {
    // ================================================================ TMA producer + scheduler
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      int qn[2] = {0, 0};  // Q loads per tile so far
      int seq = 0;         // K/V ring items issued so far
      bool ok = true;
      for (int it = 0; ok; ++it) {
        // Next unit: this CTA's own first, then the shared counter (heaviest first).
        const int u = it == 0 ? static_cast<int>(blockIdx.x)
                              : static_cast<int>(gridDim.x + atomicAdd(&g_fa_unit_next[slot], 1u));
        const int sl = it & 1;
        if (!wait_bounded(bar(L::kBarUnitEmpty + sl), ((it >> 1) & 1) ^ 1, abort_flag,
                          wait_site(5, L::kBarUnitEmpty + sl, it))) {
          ok = false;
          break;
        }
        unit_ring[sl] = u < units ? u : -1;
        mbar_arrive(bar(L::kBarUnitFull + sl));  // release: orders the ring write before it
        if (u >= units) break;
        FwdUnit x;
        fwd_unit(p, u, CAUSAL, x);
        const int kvh = x.h[0] / g;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || x.nblk[t] == 0) continue;
          if (qn[t] > 0 && !wait_bounded(bar(L::kBarQFree + t), (qn[t] - 1) & 1, abort_flag,
                                         wait_site(5, L::kBarQFree + t, it))) {
            ok = false;
            continue;
          }
          mbar_arrive_expect_tx(bar(L::kBarQ + t), L::kTileBytes);
#pragma unroll
          for (int cc = 0; cc < L::kChunks; ++cc)
            tma_load_3d(sQ + t * L::kTileBytes + cc * L::kChunkBytes, &tm_q, bar(L::kBarQ + t), cc * 64,
                        x.qb[t] * 128, x.b * p.Hq + x.h[t]);
          ++qn[t];
        }
        for (int j = 0; ok && j < x.nu; ++j) {
#pragma unroll
          for (int kind = 0; kind < 2; ++kind) {
            const int s2 = seq % S, use = seq / S;
            if (!wait_bounded(bar(L::kBarKVEmpty + s2), (use & 1) ^ 1, abort_flag,
                              wait_site(5, L::kBarKVEmpty + s2, j))) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::kBarKVFull + s2), L::kTileBytes);
            const CUtensorMap *m = kind ? &tm_v : &tm_k;
#pragma unroll
            for (int cc = 0; cc < L::kChunks; ++cc)
              tma_load_3d(sKV + s2 * L::kTileBytes + cc * L::kChunkBytes, m, bar(L::kBarKVFull + s2),
                          cc * 64, j * 128, x.b * p.Hkv + kvh);
            ++seq;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // No copy may still be landing in shared memory when the CTA exits.
      for (int s2 = seq > S ? seq - S : 0; s2 < seq; ++s2)
        wait_drain(bar(L::kBarKVFull + s2 % S), (s2 / S) & 1, 100000000ull);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (qn[t] > 0) wait_drain(bar(L::kBarQ + t), (qn[t] - 1) & 1, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 8) {
    // ================================================================ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    // Ring position of the K (V) block of global step j: the producer loads K_j, V_j as
    // items 2j, 2j + 1.
    auto kslot = [](int j) { return (2 * j) % S; };
    auto kpar = [](int j) { return static_cast<uint32_t>(((2 * j) / S) & 1); };
    auto vslot = [](int j) { return (2 * j + 1) % S; };
    auto vpar = [](int j) { return static_cast<uint32_t>(((2 * j + 1) / S) & 1); };
    auto issue_qk = [&](int t, int j) {
      const uint32_t a0 = sQ + t * L::kTileBytes;
      const uint32_t b0 = sKV + kslot(j) * L::kTileBytes;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * L::kChunkBytes + (kk % 4) * 32;
        mma_ss(tmem + L::tm_s(t), sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024), idesc_qk,
               kk > 0);
      }
    };
    auto issue_pv = [&](int t, int j, bool first) {
      const uint32_t b0 = sKV + vslot(j) * L::kTileBytes;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + L::tm_o(t), tmem + L::tm_s(t) + kk * 8, sdesc_sw128(b0 + kk * 2048, L::kChunkBytes, 1024),
               idesc_pv, (!first || kk > 0));
    };
    int qn[2] = {0, 0}, pn[2] = {0, 0};  // Q loads consumed and P phases per tile
    int G0 = 0;                          // global K/V step of the unit's block 0
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int u;
      if (!(ok = take_unit(it, u)) || u < 0) break;
      if (lane == 0) {
        FwdUnit x;
        fwd_unit(p, u, CAUSAL, x);
        const int last[2] = {x.nblk[0] - 1, x.nblk[1] - 1};
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || x.nblk[t] == 0) continue;
          ok = wait_bounded(bar(L::kBarQ + t), qn[t] & 1, abort_flag, wait_site(5, L::kBarQ + t, it));
          ++qn[t];
        }
        if (ok)
          ok = wait_bounded(bar(L::kBarKVFull + kslot(G0)), kpar(G0), abort_flag,
                            wait_site(5, L::kBarKVFull + kslot(G0), 0));
        if (ok) {
          tc_fence_after_sync();
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (x.nblk[t] == 0) continue;
            issue_qk(t, G0);
            tc_commit(bar(L::kBarS + t));
            if (last[t] == 0) tc_commit(bar(L::kBarQFree + t));  // the tile's only Q K^T
          }
          tc_commit(bar(L::kBarKVEmpty + kslot(G0)));
        }
        for (int j = 0; ok && j < x.nu; ++j) {
          const int gj = G0 + j;
          if (!wait_bounded(bar(L::kBarKVFull + vslot(gj)), vpar(gj), abort_flag,
                            wait_site(5, L::kBarKVFull + vslot(gj), j))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          bool knext = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || j > last[t]) continue;
            if (!wait_bounded(bar(L::kBarP + t), pn[t] & 1, abort_flag, wait_site(5, L::kBarP + t, j))) {
              ok = false;
              continue;
            }
            ++pn[t];
            tc_fence_after_sync();
            issue_pv(t, gj, j == 0);
            if (j < last[t]) {
              if (!knext) {
                if (!wait_bounded(bar(L::kBarKVFull + kslot(gj + 1)), kpar(gj + 1), abort_flag,
                                  wait_site(5, L::kBarKVFull + kslot(gj + 1), j + 1))) {
                  ok = false;
                  continue;
                }
                tc_fence_after_sync();
                knext = true;
              }
              issue_qk(t, gj + 1);
              tc_commit(bar(L::kBarS + t));
              if (j + 1 == last[t]) tc_commit(bar(L::kBarQFree + t));  // the tile's last Q K^T
            } else {
              tc_commit(bar(L::kBarO + t));
            }
          }
          if (!ok) break;
          tc_commit(bar(L::kBarKVEmpty + vslot(gj)));
          if (knext) tc_commit(bar(L::kBarKVEmpty + kslot(gj + 1)));
        }
        G0 += x.nu;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (!ok) *abort_flag = 1;
    // Nothing issued by this thread may still run when tensor memory is released.
    if (lane == 0) {
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
    }
    __syncwarp();
  }
  } else {
    // ================================================================ softmax warpgroups
    setmaxnreg_inc<kFwdPRegsSoftmax>();
    const int t = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + L::tm_s(t) + lane_off;
    const uint32_t tO = tmem + L::tm_o(t) + lane_off;
    const float sl2 = p.sl2;
    int sn = 0, on = 0;  // S phases and O phases of this tile so far
    int epi = 0;         // epilogues before this one (both tiles, in order)
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int u = -1;
      // Every decision that leads to a named barrier is made by the whole warpgroup: a warp
      // that gave up waiting (abort) takes the others out of the walk with it.
      ok = named_bar_and(1 + t, 128, take_unit(it, u));
      if (!ok || u < 0) break;
      FwdUnit x;
      fwd_unit(p, u, CAUSAL, x);
      // The staging tile is used by tile 0 and then tile 1 of every unit.
      const int my_epi = epi + ((t == 1 && x.nblk[0] > 0) ? 1 : 0);
      epi += (x.nblk[0] > 0 ? 1 : 0) + (x.nblk[1] > 0 ? 1 : 0);
      const int my_n = t ? x.nblk[1] : x.nblk[0];
      if (my_n == 0) continue;  // tile past the last query block: no rows
      const int my_qb = t ? x.qb[1] : x.qb[0];
      const int my_h = t ? x.h[1] : x.h[0];
      const int qrow = my_qb * 128 + r;
      float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
      for (int j = 0; ok && j < my_n; ++j) {
        if (!warp_wait_bounded(bar(L::kBarS + t), sn & 1, abort_flag, wait_site(5, L::kBarS + t, j))) {
          ok = false;
          break;
        }
        ++sn;
        tc_fence_after_sync();
        uint32_t s[128];
        {
          uint32_t (&s0)[64] = *reinterpret_cast<uint32_t(*)[64]>(&s[0]);
          uint32_t (&s1)[64] = *reinterpret_cast<uint32_t(*)[64]>(&s[64]);
          tmem_ld_x64_nowait(tS, s0);
          tmem_ld_x64_nowait(tS + 64, s1);
          tmem_wait_ld_2x64(s0, s1);
        }
        const int kv0 = j * 128;
        const bool masked = (CAUSAL && j == my_qb) || kv0 + 128 > p.N;
        if (masked) {
          const int lim = CAUSAL ? min(qrow + 1, p.N) : p.N;  // keys kv < lim are visible
#pragma unroll
          for (int cc = 0; cc < 128; ++cc)
            if (kv0 + cc >= lim) s[cc] = __float_as_uint(-INFINITY);
        }
        const float smax = row_max128(s);
        const float m_cand = smax * sl2;
        const float m_new = (m_cand > m_run + kRescaleThreshold) ? m_cand : m_run;
        const float alpha = ex2_approx(m_run - m_new);
        float lsum, ppmax;
        if (masked)
          exp_block<128, false, DROP>(s, sl2, m_new, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow, x.b * p.Hq + my_h);
        else
          exp_block<128, true, DROP>(s, sl2, m_new, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow, x.b * p.Hq + my_h);
        l_run = l_run * alpha + lsum;
        r_run = r_run * alpha + (lsum + pmax_rounding(smax, sl2, m_new, ppmax));
        m_run = m_new;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O was last written by P V of block j-1, which completed before S_j was ready.
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld_x32(tO + cc * 32, o);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float x0, x1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2), x0, x1);
              o[i] = __float_as_uint(x0);
              o[i + 1] = __float_as_uint(x1);
            }
            tmem_st_x32(tO + cc * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kBarP + t));  // one arrival per warp
      }

      // ---- epilogue: O / r -> bf16 -> staging tile -> TMA store; LSE straight to memory.
      // O is read out before this warpgroup signals P of the next unit's first block,
      // which the P V that overwrites O waits for.
      if (ok) ok = warp_wait_bounded(bar(L::kBarO + t), on & 1, abort_flag, wait_site(5, L::kBarO + t, it));
      ++on;
      // The staging tile is free once the previous epilogue's store has read it.
      if (ok && my_epi > 0)
        ok = warp_wait_bounded(bar(L::kBarStage), (my_epi - 1) & 1, abort_flag, wait_site(5, L::kBarStage, it));
      if (!named_bar_and(1 + t, 128, ok && *abort_flag == 0)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const float inv_l = (DROP ? p.drop.inv_keep : 1.f) / r_run;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld_x32(tO + cc * 32, o);
        const uint32_t rowbase = sStage + (cc / 2) * L::kChunkBytes + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = (cc % 2) * 4 + uu;  // 16-byte unit within the 128-byte row
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * inv_l,
                               __uint_as_float(o[8 * uu + 2 * e + 1]) * inv_l);
          st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before_sync();
      fence_proxy_async_smem();
      named_bar_sync(1 + t, 128);
      if (r == 0) {
#pragma unroll
        for (int cc = 0; cc < L::kChunks; ++cc)
          tma_store_3d(&tm_o, sStage + cc * L::kChunkBytes, cc * 64, my_qb * 128, x.b * p.Hq + my_h);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(bar(L::kBarStage));
      }
      if (qrow < p.N) p.lse[static_cast<size_t>(x.b * p.Hq + my_h) * p.N + qrow] = (m_run + log2f(l_run)) * kLn2;
    }
    if (!ok) *abort_flag = 1;
    // Stores issued by this warpgroup's thread must be complete before the CTA exits.
    if (r == 0) bulk_wait_group0();
  }

  // ---- teardown: every role has drained; release tensor memory; the last CTA resets the
  // launch slot's counters for the slot's next use.
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&g_fa_unit_done[slot], 1u) == gridDim.x - 1) {
      atomicExch(&g_fa_unit_next[slot], 0u);
      atomicExch(&g_fa_unit_done[slot], 0u);
    }
  }
}

}  // namespace fa
