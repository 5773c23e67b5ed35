// fa_fwd_d256.cuh - forward attention kernel for head dimension 256 on sm_100a.
//
// Same computation and recurrence as fa_fwd.cuh (online softmax over key blocks with a
// rescale of the partial output when the running max moves; the "FlashAttention1" Q&A
// page's softmax question, items 1-3), shaped for d = 256, which the FlashAttention-2
// page lists as the largest supported head dimension:
//  * a CTA owns ONE 128-row query tile: two d = 256 fp32 output accumulators would need
//    512 tensor-memory columns on their own;
//  * key blocks are 64 rows, so Q (64 KB) plus a 4-slot K/V ring of 32 KB tiles fits in
//    shared memory;
//  * tensor memory holds O (256 columns) and TWO score buffers S_a | S_b (64 columns
//    each): the tensor core computes S_{j+1} while the softmax warps work on S_j, and
//    P_j (bf16) is written over S_j for the P V product;
//  * the tensor core consumes K/V in the order K_0, K_1, V_0, K_2, V_1, K_3, ..., which
//    is also the order the TMA warp loads them;
//  * a rescale of O for block j must wait until P V of block j-1 has finished (with two
//    score buffers, S_j being ready does not imply it); the softmax warps wait on a
//    per-block completion barrier only in the rare blocks that move the max.
#pragma once

#include "fa_common.cuh"
#include "fa_fwd.cuh"

namespace fa {

struct FwdD256Layout {
  static constexpr int D = 256;
  static constexpr int kQRows = 128;
  static constexpr int kKRows = 64;
  static constexpr int kChunks = 4;                       // 64-column swizzle chunks per row
  static constexpr int kQChunkBytes = kQRows * 128;       // 16 KB
  static constexpr int kKChunkBytes = kKRows * 128;       // 8 KB
  static constexpr int kQBytes = kChunks * kQChunkBytes;  // 64 KB
  static constexpr int kKVBytes = kChunks * kKChunkBytes; // 32 KB
  static constexpr int kStages = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kQBytes;
  static constexpr int kOffBar = kOffKV + kStages * kKVBytes;
  // mbarriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done, o_full, drain
  static constexpr int kBarQ = 0;
  static constexpr int kBarKVFull = 1;
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarS = kBarKVEmpty + kStages;
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarPV = kBarP + 2;
  static constexpr int kBarO = kBarPV + 1;
  static constexpr int kBarDrain = kBarO + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // Block-sparse variant only: after misc, a 16-byte header {blocks} and the list of the
  // 64-key blocks to visit (uint16), two per enabled 128-key mask block.
  static constexpr int kOffList = kOffMisc + 16;
  static constexpr int kSmemBytesSparse = kOffList + 16 + 2 * (2 * kMaxSparseBlocks) + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmS0 = 0;     // S_a: columns 0..63, S_b: 64..127
  static constexpr uint32_t kTmO = 128;    // O: columns 128..383
  static_assert(kSmemBytesSparse <= 232448, "shared-memory budget");
};

constexpr int kFwdD256Threads = 192;  // warps 0-3 softmax, 4 MMA, 5 TMA

template <int MODE, bool DROP = false>  // MODE: kAttnFull, kAttnCausal, kAttnGeneral or kAttnSparse
__global__ void __launch_bounds__(kFwdD256Threads, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const FwdParams p) {
  using L = FwdD256Layout;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const uint32_t sQ = base + L::kOffQ;
  const uint32_t sKV = base + L::kOffKV;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- unit = (b, h, query block), ordered by unit_order (last query blocks, the longest
  // under a causal mask, are level 0)
  int head, level;
  unit_order(blockIdx.x, p.B * p.Hq, p.nqb, p.tsz, p.tail, head, level);
  const int qb = p.nqb - 1 - level;
  const int h = head % p.Hq;
  const int b = head / p.Hq;
  const int kvh = h / (p.Hq / p.Hkv);
  constexpr bool GEN = MODE == kAttnGeneral;
  constexpr bool SPARSE = MODE == kAttnSparse;
  constexpr bool GENLIKE = GEN || SPARSE;  // rows may see no key at all
  const bool packed = GEN && p.cu_q != nullptr;
  // Block-sparse: the 64-key blocks of the enabled 128-key mask blocks of this query block
  // (up to the diagonal when causal), in order; written to shared memory by the TMA warp
  // before the roles start.
  const uint16_t *blist = reinterpret_cast<const uint16_t *>(smem + L::kOffList + 16);
  SeqGeom sg{p.N, p.N, 0, 0, 0};
  // 64-key blocks [jlo, jlo + nblk) that some row of the query block can see; the loop
  // index j below counts from jlo.  nblk = 0: no row sees a key (O = 0, LSE = -inf).
  int jlo = 0, nblk;
  if constexpr (GEN) {
    if (!seq_geom(p.cu_q, p.cu_k, p.N, p.total_q, p.total_k, p.nqb * 128, INT_MAX, b, sg)) return;
    if (qb * 128 >= sg.Lq) return;  // packed: the block starts past the sequence's end
    int jhi = -1;
    key_block_range<64>(p.left, p.right, sg, qb * 128, jlo, jhi);
    nblk = jhi - jlo + 1;
  } else if constexpr (!SPARSE) {
    const int nkb_all = (p.N + 63) / 64;
    nblk = MODE == kAttnCausal ? min(2 * qb + 2, nkb_all) : nkb_all;
  }
  // TMA coordinates (dimensions 1 and 2): dense maps are [B*H][N][d], packed [total][H][d].
  const int q_c1 = packed ? h : qb * 128, q_c2 = packed ? sg.q_base + qb * 128 : b * p.Hq + h;
  auto kv_coords = [&](int row, int &c1, int &c2) {
    c1 = packed ? kvh : row;
    c2 = packed ? sg.k_base + row : b * p.Hkv + kvh;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(bar(i), (i == L::kBarP || i == L::kBarP + 1) ? 4u : 1u);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(misc), L::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  if constexpr (SPARSE) {
    if (warp == 5) {
      const uint8_t *row = p.bmask + (static_cast<size_t>(b * p.Hq + h) * p.nqb + qb) * p.nqb;
      const int hi = p.right == 0 ? qb : p.nqb - 1;
      const int nkb64 = (p.N + 63) / 64;
      uint16_t *list = reinterpret_cast<uint16_t *>(smem + L::kOffList + 16);
      int n = 0;
      for (int base0 = 0; base0 <= hi; base0 += 32) {
        const int kb = base0 + lane;
        const bool m = kb <= hi && row[kb] != 0;
        const bool two = m && 2 * kb + 1 < nkb64;  // the second half exists
        const uint32_t u1 = __ballot_sync(0xffffffffu, m), u2 = __ballot_sync(0xffffffffu, two);
        const uint32_t below = (1u << lane) - 1u;
        const int at = n + __popc(u1 & below) + __popc(u2 & below);
        if (m) list[at] = static_cast<uint16_t>(2 * kb);
        if (two) list[at + 1] = static_cast<uint16_t>(2 * kb + 1);
        n += __popc(u1) + __popc(u2);
      }
      if (lane == 0) *reinterpret_cast<int *>(smem + L::kOffList) = n;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];
  if constexpr (SPARSE) nblk = *reinterpret_cast<const int *>(smem + L::kOffList);

  // Load/consume order of the K/V ring: K_0, K_1, then V_j followed by K_{j+2}.
  // Item index -> (is_v, block).  Both the TMA warp and the MMA warp walk this order.
  if (warp == 5) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      if (nblk > 0) {
        mbar_arrive_expect_tx(bar(L::kBarQ), L::kQBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sQ + c * L::kQChunkBytes, &tm_q, bar(L::kBarQ), c * 64, q_c1, q_c2);
      }
      int seq = 0;
      bool ok = nblk > 0;
      auto produce = [&](bool is_v, int j) {
        const int slot = seq % S, use = seq / S;
        if (!wait_bounded(bar(L::kBarKVEmpty + slot), (use & 1) ^ 1, abort_flag,
                          wait_site(2, L::kBarKVEmpty + slot, j))) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(bar(L::kBarKVFull + slot), L::kKVBytes);
        const CUtensorMap *m = is_v ? &tm_v : &tm_k;
        int c1, c2;
        kv_coords((SPARSE ? blist[j] : jlo + j) * 64, c1, c2);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sKV + slot * L::kKVBytes + c * L::kKChunkBytes, m, bar(L::kBarKVFull + slot), c * 64,
                      c1, c2);
        ++seq;
      };
      if (ok) produce(false, 0);
      if (ok && nblk > 1) produce(false, 1);
      for (int j = 0; ok && j < nblk; ++j) {
        produce(true, j);
        if (ok && j + 2 < nblk) produce(false, j + 2);
      }
      for (int s2 = seq > S ? seq - S : 0; s2 < seq; ++s2)
        wait_drain(bar(L::kBarKVFull + s2 % S), (s2 / S) & 1, 100000000ull);
      if (nblk > 0) wait_drain(bar(L::kBarQ), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 4) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      int seq = 0;
      bool ok = nblk > 0 && wait_bounded(bar(L::kBarQ), 0, abort_flag, wait_site(2, L::kBarQ, 0));
      // Take the next ring item: wait until it has landed; returns its slot.
      auto consume = [&](int j) -> int {
        const int slot = seq % S, use = seq / S;
        if (!wait_bounded(bar(L::kBarKVFull + slot), use & 1, abort_flag,
                          wait_site(2, L::kBarKVFull + slot, j)))
          ok = false;
        ++seq;
        return slot;
      };
      // S_buf = Q K_j^T : M = 128, N = 64 keys, K = 256.
      auto issue_qk = [&](int j) {
        const int slot = consume(j);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t buf = L::kTmS0 + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint32_t ka = (kk / 4) * L::kQChunkBytes + (kk % 4) * 32;
          const uint32_t kb = (kk / 4) * L::kKChunkBytes + (kk % 4) * 32;
          mma_ss(tmem + buf, sdesc_sw128(sQ + ka, 16, 1024),
                 sdesc_sw128(sKV + slot * L::kKVBytes + kb, 16, 1024), idesc_qk, kk > 0);
        }
        tc_commit(bar(L::kBarS + (j & 1)));
        tc_commit(bar(L::kBarKVEmpty + slot));
      };
      if (ok) issue_qk(0);
      if (ok && nblk > 1) issue_qk(1);
      for (int j = 0; ok && j < nblk; ++j) {
        const int vslot = consume(j);
        if (!ok) break;
        if (!wait_bounded(bar(L::kBarP + (j & 1)), (j >> 1) & 1, abort_flag,
                          wait_site(2, L::kBarP + (j & 1), j))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        // O += P_j V_j : M = 128, N = 256, K = 64 keys (4 instructions of 16 keys).
        const uint32_t pbuf = L::kTmS0 + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + L::kTmO, tmem + pbuf + kk * 8,
                 sdesc_sw128(sKV + vslot * L::kKVBytes + kk * 2048, L::kKChunkBytes, 1024), idesc_pv,
                 (j > 0 || kk > 0));
        tc_commit(bar(L::kBarPV));
        tc_commit(bar(L::kBarKVEmpty + vslot));
        if (j + 2 < nblk) issue_qk(j + 2);
      }
      if (ok) tc_commit(bar(L::kBarO));
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax warpgroup
    const int r = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tO = tmem + L::kTmO + lane_off;
    const int qrow = qb * 128 + r;
    bool ok = true;
    // l_run: sum of the fp32 probabilities (for the LSE); r_run: the same with each
    // block's largest probability counted as rounded to bf16 (see pmax_rounding).
    float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
    const float sl2 = p.sl2;
    for (int j = 0; ok && j < nblk; ++j) {
      const uint32_t tS = tmem + L::kTmS0 + (j & 1) * 64 + lane_off;
      if (!warp_wait_bounded(bar(L::kBarS + (j & 1)), (j >> 1) & 1, abort_flag,
                             wait_site(2, L::kBarS + (j & 1), j))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t s[64];
      tmem_ld_x64(tS, s);
      const int kv0 = (SPARSE ? blist[j] : jlo + j) * 64;
      bool masked;
      if constexpr (GEN) {
        masked = block_needs_mask<64>(p.left, p.right, sg.Lk, qb * 128 + sg.dlt, kv0);
        if (masked) mask_scores<64>(s, p.left, p.right, sg.Lk, qrow + sg.dlt, kv0);
      } else {
        // (block-sparse: a row's first block always holds a visible key, the diagonal
        // block's first half coming before its second)
        const bool causal = MODE == kAttnCausal || (SPARSE && p.right == 0);
        masked = (causal && kv0 + 63 > qb * 128) || kv0 + 64 > p.N;
        if (masked) {
          const int lim = causal ? min(qrow + 1, p.N) : p.N;  // keys kv < lim are visible
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (kv0 + c >= lim) s[c] = __float_as_uint(-INFINITY);
        }
      }
      const float smax = row_max<64>(s);
      const float m_cand = smax * sl2;
      const float m_new = (m_cand > m_run + kRescaleThreshold) ? m_cand : m_run;
      // A band can hide a whole block from a row: while its max is still -inf the offset
      // stays 0 and alpha 1.
      const float alpha = (GEN && m_new == m_run) ? 1.f : ex2_approx(m_run - m_new);
      const float m_use = (GEN && m_new == -INFINITY) ? 0.f : m_new;
      float lsum, ppmax;
      if (masked)
        exp_block<64, false, DROP>(s, sl2, m_use, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow, b * p.Hq + h);
      else
        exp_block<64, true, DROP>(s, sl2, m_new, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow, b * p.Hq + h);
      l_run = l_run * alpha + lsum;
      r_run = r_run * alpha + (lsum + pmax_rounding(smax, sl2, m_use, ppmax));
      m_run = m_new;
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // P V of block j-1 must have finished before O is rescaled.
        if (!warp_wait_bounded(bar(L::kBarPV), (j - 1) & 1, abort_flag, wait_site(2, L::kBarPV, j))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
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
      if (lane == 0) mbar_arrive(bar(L::kBarP + (j & 1)));  // one arrival per warp
    }

    bool okw = ok && ((GENLIKE && nblk == 0) || warp_wait_bounded(bar(L::kBarO), 0, abort_flag, wait_site(2, L::kBarO, 0)));
    okw = named_bar_and(1, 128, okw && *abort_flag == 0);
    if (okw) {
      tc_fence_after_sync();
      // rows without keys: O = 0; dropout scales the kept probabilities by 1 / (1 - p)
      const float inv_l = (!GENLIKE || r_run > 0.f) ? (DROP ? p.drop.inv_keep : 1.f) / r_run : 0.f;
      // A packed block that ends past its sequence stores its rows directly.
      const bool direct = packed && qb * 128 + 128 > sg.Lq;
      const bool row_ok = qrow < sg.Lq;
      __nv_bfloat16 *orow = packed ? p.o + (static_cast<size_t>(sg.q_base + qrow) * p.Hq + h) * 256 : nullptr;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t o[32];
        if (!GENLIKE || nblk > 0) {
          tmem_ld_x32(tO + cc * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        const uint32_t rowbase = sQ + (cc / 2) * L::kQChunkBytes + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = (cc % 2) * 4 + uu;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * inv_l,
                               __uint_as_float(o[8 * uu + 2 * e + 1]) * inv_l);
          if (!direct)
            st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
          else if (row_ok)
            *reinterpret_cast<uint4 *>(orow + cc * 32 + uu * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (!direct) {
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (r == 0) {
#pragma unroll
          for (int c = 0; c < L::kChunks; ++c) tma_store_3d(&tm_o, sQ + c * L::kQChunkBytes, c * 64, q_c1, q_c2);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      }
      if (row_ok) {
        const float lse = (!GENLIKE || l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        if (packed)
          p.lse[static_cast<size_t>(sg.q_base + qrow) * p.Hq + h] = lse;
        else
          p.lse[static_cast<size_t>(b * p.Hq + h) * p.N + qrow] = lse;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
