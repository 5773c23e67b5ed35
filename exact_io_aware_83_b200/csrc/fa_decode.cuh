// fa_decode.cuh - attention of a few new query rows against a long key/value cache on
// sm_100a, split over the cache, and the merge of partial results.
//
// What it computes: for batch b, query head h and new token t < Nq, with len the number
// of valid cached keys of batch b,
//   O = sum_j softmax_j(scale q . k_j) v_j and LSE = ln sum_j exp(scale q . k_j)
// over the keys j < len (causal: j <= len - Nq + t, the new tokens being the last Nq
// positions).  This is the incremental, streaming case named on the "FlashAttention1"
// Q&A page (question on scaling to long sequences, item 8).  Splitting the keys into
// ranges whose partial results are combined afterwards is the "efficient reduction" of
// the same page (question on the key algorithmic innovations, item 3):
//   LSE = ln sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s.
//
// B200 design:
//  * Decode is bound by reading the cache from HBM (about 4 d flop per 4 d bytes of K and
//    V for each query row), so the kernel keeps TMA loads of K/V blocks in flight on
//    every SM.  A CTA owns (b, K/V head, key range); the grid holds B * Hkv * splits CTAs,
//    with enough splits to cover the SMs.
//  * The g = Hq / Hkv query heads that share a K/V head and their Nq tokens form R = g Nq
//    rows, contiguous in [B, Hq, Nq, d]; they are processed together, so each cache block
//    is read once for all of them.
//  * Scores are computed transposed, S^T = K Q^T (M = 128 keys on the TMEM lanes, N = R
//    rounded up to 16..128): each of the 128 softmax threads owns one key, so the
//    exponentials are spread over all four SM sub-partitions however few the query rows.
//    The softmax max over keys is a max across lanes (redux.sync in each warp, then a
//    four-warp exchange through shared memory).
//  * P^T goes to shared memory as bf16 (the B operand) and O^T = V^T P^T accumulates in
//    TMEM (M = 128 head-dimension lanes).  A third MMA with an all-ones A operand sums the
//    bf16 probabilities of every query row into TMEM; O is normalised by that sum (the
//    weights the P V product used), the LSE by the fp32 sum the threads keep.
//  * S^T is double-buffered in TMEM, so the tensor core computes block j+1's scores while
//    the softmax of block j runs; K and V blocks stream through a ring of shared-memory
//    slots filled by TMA in the order K_0, V_0, K_1, V_1, ...
//  * The running max is moved only when a column's max rises by more than 2^8 (log2
//    units); the rare rescale of O^T waits for the previous block's P V.
#pragma once

#include "fa_common.cuh"
#include "fa_fwd.cuh"

namespace fa {

struct DecodeParams {
  const int *lens;       // [B] valid keys per batch (nullptr: all Nk), clamped to [0, Nk]
  __nv_bfloat16 *o;      // [B, Hq, Nq, D]               (splits == 1)
  float *lse;            // [B, Hq, Nq]                  (splits == 1)
  float *o_part;         // [splits, B * Hq * Nq, D] fp32 (splits > 1)
  float *lse_part;       // [splits, B * Hq * Nq]
  int B, Hkv, Nq, Nk;
  int R;                 // query rows per K/V head: (Hq / Hkv) * Nq
  int splits, chunk;     // split s covers keys [s * chunk, (s + 1) * chunk), chunk % 128 == 0
  int causal;
  float sl2;             // scale * log2(e)
};

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

// D: head dimension; RP: query rows padded to the MMA's N (16, 32, 64 or 128).
template <int D, int RP>
struct DecodeLayout {
  static constexpr int kKeys = 128;                  // keys per block = TMEM lanes of S^T
  static constexpr int kChunks = D / 64;             // 128-byte swizzle chunks per row
  static constexpr int kNH = D >= 128 ? D / 128 : 1; // 128-lane slices of O^T
  static constexpr int kKVChunk = kKeys * 128;       // [128 keys x 64] bf16 TMA box
  static constexpr int kKVTile = kChunks * kKVChunk;
  static constexpr int kQChunk = RP * 128;           // [RP rows x 64] bf16 TMA box
  static constexpr int kQBytes = kChunks * kQChunk;
  static constexpr int kPChunk = RP * 128;           // P^T: RP rows x 64 keys
  static constexpr int kPBytes = 2 * kPChunk;        // 128 keys
  static constexpr int kOnesBytes = 1024;            // one 8 x 64 swizzle atom of 1.0
  // For D = 64 the V^T operand (M = 128) also reads a second 64-column chunk: that half
  // of O^T is unused, and this pad keeps the read inside shared memory.
  static constexpr int kPad = (D == 64) ? kKVChunk : 0;
  static constexpr int kVecBytes = 6 * RP * 4;       // red[4][RP] | mu[RP] | al[RP]
  static constexpr int kNumBarsMax = 8 + 2 * 8;
  static constexpr int kFixed = kQBytes + 2 * kPBytes + kOnesBytes + kPad + kVecBytes + kNumBarsMax * 8 + 16;
  // Up to 16 query rows and d = 64, two CTAs share an SM (each with half the shared
  // memory): the softmax of one block is a serial chain (load, max exchange,
  // exponentials, P store), and a second CTA's chain hides it when a block carries few
  // bytes (d = 64).
  static constexpr int kCtasPerSM = (RP == 16 && D == 64) ? 2 : 1;
  static constexpr int kSmemBudget = (kCtasPerSM == 2) ? 232448 / 2 - 1024 : 232448;
  static constexpr int kSlotsFit = (kSmemBudget - 1024 - kFixed) / kKVTile;
  static constexpr int kSlots = kSlotsFit > 8 ? 8 : kSlotsFit;
  static constexpr int kOffKV = 0;
  static constexpr int kOffPad = kOffKV + kSlots * kKVTile;
  static constexpr int kOffQ = kOffPad + kPad;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffOnes = kOffP + 2 * kPBytes;
  static constexpr int kOffVec = kOffOnes + kOnesBytes;
  static constexpr int kOffBar = kOffVec + kVecBytes;
  // mbarriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done, o_final, drain
  static constexpr int kBarQ = 0;
  static constexpr int kBarKVFull = 1;
  static constexpr int kBarKVEmpty = kBarKVFull + kSlots;
  static constexpr int kBarS = kBarKVEmpty + kSlots;
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarODone = kBarP + 2;
  static constexpr int kBarOFinal = kBarODone + 1;
  static constexpr int kBarDrain = kBarOFinal + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // tensor memory: S^T_0 | S^T_1 | O^T (kNH slices) | ones sum
  __host__ __device__ static constexpr uint32_t tm_s(int buf) { return static_cast<uint32_t>(buf * RP); }
  __host__ __device__ static constexpr uint32_t tm_o(int h) { return static_cast<uint32_t>((2 + h) * RP); }
  static constexpr uint32_t kTmR = static_cast<uint32_t>((2 + kNH) * RP);
  static constexpr uint32_t kTmemCols = static_cast<uint32_t>(pow2_at_least((3 + kNH) * RP));
  static_assert(RP == 16 || RP == 32 || RP == 64 || RP == 128, "padded query rows");
  static_assert((3 + kNH) * RP <= 512, "tensor-memory budget");
  static_assert(kSlots >= 2, "K/V ring");
  static_assert(kNumBars <= kNumBarsMax, "barrier budget");
  static_assert(kSmemBytes <= kSmemBudget, "shared-memory budget");
};

// Warp 0: TMA loads; warp 1: TMEM allocation and MMA issue; warps 2-5: softmax (one key
// per thread; warp w owns TMEM lane quadrant w % 4).
constexpr int kDecodeThreads = 192;

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

template <int D, int RP>
__global__ void __launch_bounds__(kDecodeThreads, DecodeLayout<D, RP>::kCtasPerSM)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using L = DecodeLayout<D, RP>;
  constexpr int S = L::kSlots;
  constexpr int CW = RP < 32 ? RP : 32;  // score columns per TMEM load
  constexpr int NCH = RP / CW;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- unit: (b, K/V head, key range)
  int u = blockIdx.x;
  const int split = u % p.splits;
  u /= p.splits;
  const int kvh = u % p.Hkv;
  const int b = u / p.Hkv;
  int len = p.lens ? p.lens[b] : p.Nk;
  len = len < 0 ? 0 : (len > p.Nk ? p.Nk : len);
  const int k_begin = split * p.chunk;
  const int k_end = min(k_begin + p.chunk, len);
  const int nblk = k_end > k_begin ? (k_end - k_begin + 127) / 128 : 0;
  const long long rows_total = static_cast<long long>(p.B) * p.Hkv * p.R;
  const long long row0 = static_cast<long long>(b * p.Hkv + kvh) * p.R;  // first query row
  const long long part0 = static_cast<long long>(split) * rows_total + row0;

  if (nblk == 0) {
    // No key of this range is visible: O = 0 and LSE = -inf for every row.
    for (int i = threadIdx.x; i < p.R * D; i += blockDim.x) {
      if (p.splits == 1)
        p.o[row0 * D + i] = __float2bfloat16_rn(0.f);
      else
        p.o_part[part0 * D + i] = 0.f;
    }
    for (int c = threadIdx.x; c < p.R; c += blockDim.x) {
      if (p.splits == 1)
        p.lse[row0 + c] = -INFINITY;
      else
        p.lse_part[part0 + c] = -INFINITY;
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const uint32_t sKV = base + L::kOffKV;
  const uint32_t sQ = base + L::kOffQ;
  const uint32_t sP = base + L::kOffP;
  const uint32_t sOnes = base + L::kOffOnes;
  float *vec = reinterpret_cast<float *>(smem + L::kOffVec);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(bar(i), (i == L::kBarP || i == L::kBarP + 1) ? 4u : 1u);
    misc[1] = 0;
    fence_mbar_init();
  }
  // The all-ones A operand (bf16 1.0 = 0x3F80), read by the tensor core (async proxy).
  {
    uint32_t *ones = reinterpret_cast<uint32_t *>(smem + L::kOffOnes);
    for (int i = threadIdx.x; i < L::kOnesBytes / 4; i += blockDim.x) ones[i] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), L::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar(L::kBarQ), L::kQBytes);
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(sQ + c * L::kQChunk, &tm_q, bar(L::kBarQ), c * 64, 0, b * p.Hkv + kvh);
      int issued = 0;
      for (int i = 0; i < 2 * nblk; ++i) {
        const int slot = i % S, use = i / S;
        if (!wait_bounded(bar(L::kBarKVEmpty + slot), (use & 1) ^ 1, abort_flag,
                          wait_site(4, L::kBarKVEmpty + slot, i)))
          break;
        mbar_arrive_expect_tx(bar(L::kBarKVFull + slot), L::kKVTile);
        const CUtensorMap *m = (i & 1) ? &tm_v : &tm_k;
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sKV + slot * L::kKVTile + c * L::kKVChunk, m, bar(L::kBarKVFull + slot), c * 64,
                      k_begin + (i >> 1) * 128, b * p.Hkv + kvh);
        ++issued;
      }
      // No copy may still be landing in shared memory when the CTA exits.
      for (int i = issued > S ? issued - S : 0; i < issued; ++i)
        wait_drain(bar(L::kBarKVFull + i % S), (i / S) & 1, 100000000ull);
      wait_drain(bar(L::kBarQ), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kq = idesc_bf16_f32(128, RP, 0, 0);  // S^T = K Q^T; sums = 1 P^T
      constexpr uint32_t id_vp = idesc_bf16_f32(128, RP, 1, 0);  // O^T += V^T P^T (V^T MN-major)
      bool ok = wait_bounded(bar(L::kBarQ), 0, abort_flag, wait_site(4, L::kBarQ, 0));
      auto ring_wait = [&](int i) -> int {
        const int slot = i % S;
        if (ok && !wait_bounded(bar(L::kBarKVFull + slot), (i / S) & 1, abort_flag,
                                wait_site(4, L::kBarKVFull + slot, i)))
          ok = false;
        return slot;
      };
      // S^T_j = K_j Q^T : M = 128 keys, N = RP query rows, K = D (16 per instruction).
      auto issue_qk = [&](int j) {
        const int slot = ring_wait(2 * j);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t a0 = sKV + slot * L::kKVTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + L::tm_s(j & 1),
                 sdesc_sw128(a0 + (kk / 4) * L::kKVChunk + (kk % 4) * 32, 16, 1024),
                 sdesc_sw128(sQ + (kk / 4) * L::kQChunk + (kk % 4) * 32, 16, 1024), id_kq, kk > 0);
        tc_commit(bar(L::kBarS + (j & 1)));
        tc_commit(bar(L::kBarKVEmpty + slot));
      };
      if (ok) issue_qk(0);
      if (ok && nblk > 1) issue_qk(1);
      for (int j = 0; ok && j < nblk; ++j) {
        if (!wait_bounded(bar(L::kBarP + (j & 1)), (j >> 1) & 1, abort_flag,
                          wait_site(4, L::kBarP + (j & 1), j))) {
          ok = false;
          break;
        }
        const int vslot = ring_wait(2 * j + 1);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t v0 = sKV + vslot * L::kKVTile;
        const uint32_t p0 = sP + (j & 1) * L::kPBytes;
        // O^T_h += V^T P^T : M = 128 head-dimension columns, N = RP, K = 128 keys.
#pragma unroll
        for (int h = 0; h < L::kNH; ++h)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + L::tm_o(h),
                   sdesc_sw128(v0 + (2 * h) * L::kKVChunk + kk * 2048, L::kKVChunk, 1024),
                   sdesc_sw128(p0 + (kk / 4) * L::kPChunk + (kk % 4) * 32, 16, 1024), id_vp,
                   (j > 0 || kk > 0));
        // Row sums of the bf16 P: every row of the ones operand is the same 8-row atom
        // (row-group stride 0).
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::kTmR, sdesc_sw128(sOnes + (kk % 4) * 32, 16, 0),
                 sdesc_sw128(p0 + (kk / 4) * L::kPChunk + (kk % 4) * 32, 16, 1024), id_kq,
                 (j > 0 || kk > 0));
        tc_commit(bar(L::kBarODone));
        tc_commit(bar(L::kBarKVEmpty + vslot));
        // S^T_{j+2} reuses block j's score buffer, which the softmax has finished reading
        // (its P_j arrival came after its last load).
        if (j + 2 < nblk) issue_qk(j + 2);
      }
      if (ok) tc_commit(bar(L::kBarOFinal));
      // Nothing issued by this thread may still run when tensor memory is released.
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax warpgroup
    const int q = warp & 3;                       // TMEM lane quadrant
    const int lk = q * 32 + lane;                 // key of the block = O^T lane = d index
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float *red = vec;                             // [4][RP] per-warp column maxima / sums
    float *mu = vec + 4 * RP;                     // exponent offset per column
    float *al = vec + 5 * RP;                     // rescale factor per column
    const float sl2 = p.sl2;
    const int pos0 = len - p.Nq;                  // position of the first new token
    float l_part[RP];                             // this key's share of each row's sum
#pragma unroll
    for (int c = 0; c < RP; ++c) l_part[c] = 0.f;
    float m_run = -INFINITY;                      // running offset of column lk (lk < RP)

    // Scores of columns [ch * CW, ch * CW + CW) for this thread's key, hidden keys -inf.
    auto load_scores = [&](uint32_t tS, int ch, int kv, uint32_t (&sc)[CW]) {
      if constexpr (CW == 16)
        tmem_ld_x16(tS + ch * CW, sc);
      else
        tmem_ld_x32(tS + ch * CW, sc);
      if (kv >= k_end) {
#pragma unroll
        for (int c = 0; c < CW; ++c) sc[c] = __float_as_uint(-INFINITY);
      } else if (p.causal && kv > pos0) {
        // column c is token t = c mod Nq, which sees keys up to pos0 + t
        int t = (ch * CW) % p.Nq;
        const int hide_below = kv - pos0;         // tokens t < hide_below cannot see kv
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          if (t < hide_below) sc[c] = __float_as_uint(-INFINITY);
          t = (t + 1 == p.Nq) ? 0 : t + 1;
        }
      }
    };

    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const uint32_t tS = tmem + L::tm_s(j & 1) + lane_off;
      const int kv = k_begin + j * 128 + lk;
      bool okw = ok && warp_wait_bounded(bar(L::kBarS + (j & 1)), (j >> 1) & 1, abort_flag,
                                         wait_site(4, L::kBarS + (j & 1), j));
      if (okw) {
        tc_fence_after_sync();
        // Pass 1: per-warp maximum of every column.
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          uint32_t sc[CW];
          load_scores(tS, ch, kv, sc);
#pragma unroll
          for (int c = 0; c < CW; ++c) {
            const float m = warp_max_f32(__uint_as_float(sc[c]));
            if (lane == ((ch * CW + c) & 31)) red[q * RP + ch * CW + c] = m;
          }
        }
      }
      ok = named_bar_and(1, 128, okw);
      if (!ok) break;
      if (lk < RP) {
        // Column owner: block max over the four warps, stale-offset update.
        const float mc = fmaxf(fmaxf(red[lk], red[RP + lk]), fmaxf(red[2 * RP + lk], red[3 * RP + lk])) * sl2;
        const float mn = (mc > m_run + kRescaleThreshold) ? mc : m_run;
        al[lk] = (mn == m_run) ? 1.f : ex2_approx(m_run - mn);  // 0 at a column's first key
        mu[lk] = (mn == -INFINITY) ? 0.f : mn;                    // no inf - inf below
        m_run = mn;
      }
      named_bar_sync(1, 128);
      bool resc = false;
#pragma unroll
      for (int c = 0; c < RP; c += 4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(al + c);
        resc |= (a4.x != 1.f) | (a4.y != 1.f) | (a4.z != 1.f) | (a4.w != 1.f);
        l_part[c] *= a4.x;
        l_part[c + 1] *= a4.y;
        l_part[c + 2] *= a4.z;
        l_part[c + 3] *= a4.w;
      }
      if (resc && j > 0) {
        // O^T and the sums were last written by P V of block j - 1.
        if (warp_wait_bounded(bar(L::kBarODone), (j - 1) & 1, abort_flag, wait_site(4, L::kBarODone, j))) {
          tc_fence_after_sync();
#pragma unroll
          for (int h = 0; h <= L::kNH; ++h) {   // the O^T slices, then the sums
            const uint32_t t0 = tmem + (h < L::kNH ? L::tm_o(h) : L::kTmR) + lane_off;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
              uint32_t o[CW];
              if constexpr (CW == 16) tmem_ld_x16(t0 + ch * CW, o); else tmem_ld_x32(t0 + ch * CW, o);
#pragma unroll
              for (int c = 0; c < CW; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * al[ch * CW + c]);
              if constexpr (CW == 16) tmem_st_x16(t0 + ch * CW, o); else tmem_st_x32(t0 + ch * CW, o);
            }
          }
          tmem_wait_st();
        } else {
          ok = false;  // the abort flag is up; the next barrier ends every warp's loop
        }
      }
      // Pass 2: P = 2^(s scale log2e - offset), this key's sums, and P^T (bf16) into the
      // swizzled K-major B operand: row = query column, 64 keys per 128-byte row.
      const uint32_t pbuf = sP + (j & 1) * L::kPBytes + (lk / 64) * L::kPChunk;
      const uint32_t unit = static_cast<uint32_t>((lk % 64) / 8), byte = static_cast<uint32_t>((lk % 8) * 2);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        uint32_t sc[CW];
        load_scores(tS, ch, kv, sc);
#pragma unroll
        for (int c4 = 0; c4 < CW; c4 += 4) {
          const float4 m4 = *reinterpret_cast<const float4 *>(mu + ch * CW + c4);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = ch * CW + c4 + e;
            const float pr = ex2_approx(fmaf(__uint_as_float(sc[c4 + e]), sl2, -mm[e]));
            l_part[c] += pr;
            const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
            st_shared_u16(pbuf + c * 128 + ((unit ^ static_cast<uint32_t>(c & 7)) * 16) + byte,
                          __bfloat16_as_ushort(pb));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarP + (j & 1)));  // one arrival per warp
    }

    // ---- epilogue: LSE from the fp32 sums, O^T / (bf16 sums) -> global memory
    bool okf = ok && warp_wait_bounded(bar(L::kBarOFinal), 0, abort_flag, wait_site(4, L::kBarOFinal, 0));
    okf = named_bar_and(1, 128, okf && *abort_flag == 0);
    if (okf) {
      tc_fence_after_sync();
#pragma unroll
      for (int c = 0; c < RP; ++c) {
        float v = l_part[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == (c & 31)) red[q * RP + c] = v;
      }
      named_bar_sync(1, 128);
      if (lk < p.R && lk < RP) {
        const float l = (red[lk] + red[RP + lk]) + (red[2 * RP + lk] + red[3 * RP + lk]);
        const float lse = l > 0.f ? (m_run + log2f(l)) * kLn2 : -INFINITY;
        if (p.splits == 1)
          p.lse[row0 + lk] = lse;
        else
          p.lse_part[part0 + lk] = lse;
      }
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        uint32_t rs[CW];
        if constexpr (CW == 16) tmem_ld_x16(tmem + L::kTmR + lane_off + ch * CW, rs);
        else tmem_ld_x32(tmem + L::kTmR + lane_off + ch * CW, rs);
#pragma unroll
        for (int h = 0; h < L::kNH; ++h) {
          const int dcol = h * 128 + lk;
          uint32_t o[CW];
          if constexpr (CW == 16) tmem_ld_x16(tmem + L::tm_o(h) + lane_off + ch * CW, o);
          else tmem_ld_x32(tmem + L::tm_o(h) + lane_off + ch * CW, o);
          if (dcol < D) {
#pragma unroll
            for (int c = 0; c < CW; ++c) {
              const int row = ch * CW + c;
              if (row >= p.R) break;
              const float r = __uint_as_float(rs[c]);
              const float val = r > 0.f ? __uint_as_float(o[c]) / r : 0.f;
              if (p.splits == 1)
                p.o[(row0 + row) * D + dcol] = __float2bfloat16_rn(val);
              else
                p.o_part[(part0 + row) * D + dcol] = val;
            }
          }
        }
      }
    }
  }

  // ---- teardown: every role has drained; release tensor memory
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Merge of partial results (one warp per query row):
//   LSE = ln sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s
// o_part [S, rows, D] fp32 (each part normalised), lse_part [S, rows]; parts with
// LSE_s = -inf carry no weight, and a row whose parts are all -inf gets O = 0, LSE = -inf.
template <int D>
__global__ void __launch_bounds__(256)
    fa_merge_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
                    __nv_bfloat16 *__restrict__ o, float *__restrict__ lse, int S, long long rows) {
  constexpr int kPer = D / 32;  // elements per lane
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  constexpr float kLog2e = 1.4426950408889634f;
  float m = -INFINITY;
  for (int s = 0; s < S; ++s) m = fmaxf(m, lse_part[static_cast<long long>(s) * rows + row]);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float out_lse = -INFINITY;
  if (m != -INFINITY) {
    float l = 0.f;
    for (int s = 0; s < S; ++s) l += ex2_approx((lse_part[static_cast<long long>(s) * rows + row] - m) * kLog2e);
    out_lse = m + log2f(l) * kLn2;
    for (int s = 0; s < S; ++s) {
      const float w = ex2_approx((lse_part[static_cast<long long>(s) * rows + row] - out_lse) * kLog2e);
      if (w == 0.f) continue;
      const float *src = o_part + (static_cast<long long>(s) * rows + row) * D + lane * kPer;
#pragma unroll
      for (int e = 0; e < kPer; e += 2) {
        const float2 x = *reinterpret_cast<const float2 *>(src + e);
        acc[e] = fmaf(w, x.x, acc[e]);
        acc[e + 1] = fmaf(w, x.y, acc[e + 1]);
      }
    }
  }
  uint32_t *dst = reinterpret_cast<uint32_t *>(o + row * D + lane * kPer);
#pragma unroll
  for (int e = 0; e < kPer; e += 2) dst[e / 2] = pack_bf16x2(acc[e], acc[e + 1]);
  if (lane == 0) lse[row] = out_lse;
}

}  // namespace fa
