// fa_common.cuh - device status word and bounded pipeline waits shared by the kernels.
//
// Every wait on an mbarrier in the attention kernels is bounded in time.  When a wait
// gives up, the kernel records FA_ERR_DEVICE_TIMEOUT (plus a site code) in the device
// status word, raises a per-CTA abort flag in shared memory so that every other role
// stops waiting too, and all roles drain to the common exit, where tensor memory is
// released.  The host reads and clears the word with fa_device_status().
#pragma once

#include <climits>
#include <cuda_bf16.h>

#include "fa.h"
#include "sm100_ptx.cuh"

namespace fa {

// A single pipeline wait never legitimately takes more than microseconds; two seconds
// only trips on a broken pipeline.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Device status word (FA_OK or FA_ERR_DEVICE_TIMEOUT) and the site of the first failure:
// bits 0..15 iteration, 16..23 barrier id, 24..31 kernel id, 32..63 blockIdx.x.
__device__ int g_fa_status;
__device__ unsigned long long g_fa_status_site;

__device__ __forceinline__ uint32_t wait_site(uint32_t kernel, uint32_t barrier, uint32_t iter) {
  return (kernel << 24) | ((barrier & 0xFFu) << 16) | (iter & 0xFFFFu);
}

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                       uint32_t site, uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      if (atomicCAS(&g_fa_status, FA_OK, FA_ERR_DEVICE_TIMEOUT) == FA_OK)
        atomicExch(&g_fa_status_site,
                   static_cast<unsigned long long>(site) |
                       (static_cast<unsigned long long>(blockIdx.x) << 32));
      return false;
    }
  }
}

// Wait for the phase of `bar` with parity `parity`; false if the wait gave up (or another
// role of this CTA already did).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int *abort_flag, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, site);
}

// The same for all 32 lanes of a warp: every lane waits, and the warp proceeds only if
// every lane saw the phase complete, so warp-collective tcgen05 instructions that follow
// are never reached by part of a warp.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int *abort_flag, uint32_t site) {
  const bool ok = wait_bounded(bar, parity, abort_flag, site);
  return __all_sync(0xffffffffu, ok);
}

// Best-effort wait used while draining after an abort: time-bounded, ignores the flag.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

// Counter-based generator Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011), written from its published definition: ten
// rounds of two 32 x 32 -> 64-bit products mixed with the key, the key advanced by a Weyl
// sequence between rounds.  Used for the attention-dropout keep mask.
__device__ __forceinline__ void philox4x32_10(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, uint32_t k0,
                                              uint32_t k1, uint32_t (&out)[4]) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, x0), lo0 = 0xD2511F53u * x0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, x2), lo1 = 0xCD9E8D57u * x2;
    const uint32_t y0 = hi1 ^ x1 ^ k0, y2 = hi0 ^ x3 ^ k1;
    x0 = y0;
    x1 = lo1;
    x2 = y2;
    x3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

// Dropout keep mask: probability (row i, key j) of query head bh is kept iff the 16-bit
// value j % 8 of Philox4x32-10(counter = (j / 8, i, bh, 0), key = (k0, k1)) - the low (even
// j) or high (odd j) half of output word (j % 8) / 2 - is >= thr = min(floor(p 2^16),
// 2^16 - 1).  Kept values are scaled by inv_keep = 2^16 / (2^16 - thr), the inverse of the
// exact keep probability.  thr2 holds thr in both halves, for packed halfword compares.
struct DropCfg {
  uint32_t k0, k1, thr, thr2;
  float inv_keep;
};

// Kernel variants: dense attention over every key, dense causal attention, and the general
// form (packed variable-length sequences and/or a key band), whose extra bookkeeping the
// two common dense cases do not pay for.
// kAttnSparse: dense layout with a 0/1 mask over 128 x 128 blocks (and optionally the
// causal mask); only enabled blocks are visited.
constexpr int kAttnFull = 0, kAttnCausal = 1, kAttnGeneral = 2, kAttnSparse = 3;

// Order of the work units of a grid: `heads` rows of `levels` units each, level 0 the
// heaviest (the most key blocks under a causal mask).  Levels are cut into tiers of `tsz`
// levels; the tiers run heaviest first, and inside a tier one head's units are consecutive,
// so the CTAs that run together share that head's K/V (or Q/dO) in L2.  tsz = levels is
// head-major order, tsz = 1 pure heaviest-first.  The hardware starts CTAs in index order,
// so heavy units never start last and leave a long tail.  With tail > 0 the last `tail`
// heads come after all the others, level by level (heaviest first): only the end of the
// grid gives up head locality, and it ends on the lightest units.
__host__ __device__ __forceinline__ void unit_order(int u, int heads, int levels, int tsz, int tail,
                                                    int &head, int &level) {
  const int front = (heads - tail) * levels;
  if (u >= front) {
    const int v = u - front;
    level = v / tail;
    head = heads - tail + v % tail;
    return;
  }
  const int per_tier = (heads - tail) * tsz;
  const int t = u / per_tier;
  const int v = u - t * per_tier;
  const int cnt = min(tsz, levels - t * tsz);
  head = v / cnt;
  level = t * tsz + v % cnt;
}

// The sequence a CTA works on.  Dense: Lq = Lk = N.  Packed: the lengths of sequence b and
// its first rows in the packed tensors.  The keys are aligned to the END of the queries:
// query i sits at key position c = i + dlt, dlt = Lk - Lq (0 for self-attention), and sees
// the keys j with c - left <= j <= c + right, 0 <= j < Lk.
struct SeqGeom {
  int Lq, Lk, dlt, q_base, k_base;
};

// Records FA_ERR_SEQLENS when packed offsets are inconsistent (decreasing, past the packed
// rows, or a sequence longer than the launch was sized for).
__device__ __forceinline__ void report_bad_seqlens() {
  if (atomicCAS(&g_fa_status, FA_OK, FA_ERR_SEQLENS) == FA_OK)
    atomicExch(&g_fa_status_site, static_cast<unsigned long long>(blockIdx.x) << 32);
}

// Geometry of batch entry b; false (after reporting) when the offsets are inconsistent.
__device__ __forceinline__ bool seq_geom(const int *cu_q, const int *cu_k, int N, int total_q,
                                         int total_k, int max_lq, int max_lk, int b, SeqGeom &g) {
  if (!cu_q) {
    g = SeqGeom{N, N, 0, 0, 0};
    return true;
  }
  const int q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_k[b], k1 = cu_k[b + 1];
  if (q0 < 0 || q1 < q0 || q1 > total_q || k0 < 0 || k1 < k0 || k1 > total_k || q1 - q0 > max_lq ||
      k1 - k0 > max_lk) {
    report_bad_seqlens();
    return false;
  }
  g = SeqGeom{q1 - q0, k1 - k0, (k1 - k0) - (q1 - q0), q0, k0};
  return true;
}

// Self-test of the watchdog path: one thread waits, with a short limit, on an mbarrier
// that nothing ever arrives at.  The wait must give up, record FA_ERR_DEVICE_TIMEOUT in
// the status word, and return; no fault, trap or hang is involved.
__global__ void fa_watchdog_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  abort_flag = 0;
  mbar_init(b, 1);
  fence_mbar_init();
  wait_slow(b, 0, &abort_flag, wait_site(15, 0, 0), limit_ns);
}

}  // namespace fa
