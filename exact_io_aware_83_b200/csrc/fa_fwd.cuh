// fa_fwd.cuh - forward attention kernel for head dimensions 64 and 128 on sm_100a.
//
// What it computes (per query row i of head h, keys j in J(i)):
//   O_i = sum_j softmax_j(scale * q_i . k_j) v_j,  LSE_i = ln sum_j exp(scale * q_i . k_j)
// where J(i) is every key, or the local window i - left <= j <= i + right (causal
// attention is left unlimited, right = 0; the "FlashAttention1" Q&A's scaling question,
// item 4, pairs the method with local attention), or the keys of the enabled 128 x 128
// blocks of a block mask (block-sparse attention, named in the deep-dive page's closing
// paragraph).  Key blocks no row of a tile can see are skipped, not masked.  The score
// matrix is processed one 128 x 128 tile at a time with the online-softmax
// recurrence of the "FlashAttention1" Q&A page (question on computing the softmax,
// items 1-3): a running row maximum m, a running sum l, and a rescale of the partial
// output by exp(m_old - m_new) when a new key block raises the maximum (the deep-dive
// page's "Intuition" for merging blocks).  Nothing N x N is written to memory (the
// "Tiling" bullet of the FlashAttention-2 page).
//
// B200 design (not the pages' A100 one):
//  * One CTA owns two 128-row query tiles that share every K/V block: either two query
//    blocks of one head, or - for grouped-query attention with an even group - the same
//    query block of two heads that share a K/V head, so each K/V tile is loaded once for
//    both.  Work units are ordered by unit_order (fa_common.cuh), heavy units first
//    where that shortens the tail.
//  * Warp roles: warps 0-3 and 4-7 are the softmax warpgroups of tile 0 and tile 1
//    (one query row per thread, the row's TMEM lane); warp 8 allocates tensor memory and
//    issues every tcgen05.mma from one lane; warp 9 issues the TMA loads from one lane;
//    registers are moved from the producer warpgroup to the softmax warpgroups.
//  * Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1.  S = Q K^T lands in TMEM as
//    fp32; the softmax warps read it, write P as bf16 over the first half of the same
//    columns, and the MMA warp computes O += P V with P taken straight from TMEM.
//  * K and V blocks stream through a ring of shared-memory slots filled by TMA in the
//    order K_0, V_0, K_1, V_1, ...; 128-byte swizzled tiles feed the tensor core directly.
//  * The two tiles ping-pong: while the softmax warps of one tile work, the tensor core
//    runs the other tile's P V and next Q K^T.  (Block-sparse: the two tiles' masks differ,
//    so the two S buffers are shared and a tile can also run a block ahead on its own.)
//  * exp is evaluated as exp2 with scale*log2(e) folded into one FMA.  The running max
//    used as the exponent offset is only moved when a row's max rises by more than 2^8
//    (the recurrence is exact for any offset; keeping it avoids rescaling O for most
//    blocks).
#pragma once

#include "fa_common.cuh"

namespace fa {

struct FwdParams {
  float *lse;             // dense: [B, Hq, N]; packed sequences: [total_q, Hq]
  __nv_bfloat16 *o;       // packed sequences: O, for the rows of tiles that end past a sequence
  const int *cu_q, *cu_k; // packed sequences: [B + 1] row offsets (nullptr: dense [B, H, N, d])
  int B, Hq, Hkv, N;      // dense: N = sequence length
  int total_q, total_k;   // packed sequences: rows of the packed Q and K
  int nqb;                // 128-row query blocks per sequence (packed: of the longest)
  int pair_heads;         // 1: a unit is (2 heads, 1 query block); 0: (1 head, 2 query blocks)
  int left, right;        // key band around the diagonal: [c - left, c + right]; -1 = unlimited
  float sl2;              // scale * log2(e)
  DropCfg drop;           // dropout (kernels instantiated with DROP only)
  const uint8_t *bmask;   // block-sparse: [B, Hq, nqb, nqb] 0/1 over 128 x 128 blocks
  int tsz;                // unit order: levels per tier (see unit_order)
  int tail;               // unit order: heads taken level by level at the end
};

// Blocks of KB keys [lo, hi] that some row q0 .. min(q0 + 127, Lq - 1) of a query tile can
// see; false when no row sees any key.
template <int KB>
__device__ __forceinline__ bool key_block_range(int left, int right, const SeqGeom &g, int q0, int &lo,
                                                int &hi) {
  const int c0 = q0 + g.dlt, c1 = min(q0 + 127, g.Lq - 1) + g.dlt;
  const int first = (left < 0) ? 0 : max(0, c0 - left);
  const int last = (right < 0) ? g.Lk - 1 : min(g.Lk - 1, c1 + right);
  if (last < first) return false;
  lo = first / KB;
  hi = last / KB;
  return true;
}

// True when some key of the block [kv0, kv0 + KB) is hidden from some row of the
// 128-row query tile whose first row sits at key position c0 (band edge or end of keys).
template <int KB>
__device__ __forceinline__ bool block_needs_mask(int left, int right, int Lk, int c0, int kv0) {
  return kv0 + KB > Lk || (left >= 0 && c0 + 127 - kv0 > left) || (right >= 0 && kv0 + KB - 1 - c0 > right);
}

// Hides with -inf the scores of keys kv0 + c outside the band of the row at key position
// c_row, and keys past Lk.
template <int NC>
__device__ __forceinline__ void mask_scores(uint32_t (&s)[NC], int left, int right, int Lk, int c_row,
                                            int kv0) {
  // key kv0 + c is visible iff c_lo <= c < c_hi
  const int rel = c_row - kv0;
  const int c_hi = min(Lk - kv0, right < 0 ? INT_MAX : rel + right + 1);
  if (left < 0) {  // causal and right-bounded bands: one comparison per key
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (c >= c_hi) s[c] = __float_as_uint(-INFINITY);
  } else {
    const int c_lo = rel - left;
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (c < c_lo || c >= c_hi) s[c] = __float_as_uint(-INFINITY);
  }
}

constexpr float kLn2 = 0.693147180559945309f;
// Longest block-sparse sequence, in 128-key blocks (the per-CTA block list lives in shared
// memory).
constexpr int kMaxSparseBlocks = 4096;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct FwdLayout {
  static constexpr int kRows = 128;                // query rows per tile = keys per block
  static constexpr int kChunks = D / 64;           // 128-byte swizzle chunks per row
  static constexpr int kChunkBytes = kRows * 128;  // one [128 x 64] bf16 TMA box
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 64) ? 6 : 4;  // K/V ring slots
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  // mbarriers: q_full[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] drain
  static constexpr int kBarQ = 0;
  static constexpr int kBarKVFull = 2;
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarS = kBarKVEmpty + kStages;
  static constexpr int kBarP = kBarS + 2;
  static constexpr int kBarO = kBarP + 2;
  static constexpr int kBarPV = kBarO + 2;    // block-sparse: P V of tile t completed
  static constexpr int kBarSX = kBarPV + 2;   // block-sparse: S buffer b holds a tile-1 block
  static constexpr int kBarDrain = kBarSX + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-B alignment
  // Block-sparse variant only: after misc, a 16-byte header {steps, blocks of tile 0, blocks
  // of tile 1} and the CTA's key-block list (uint16: block | tile-0 bit 14 | tile-1 bit 15).
  static constexpr int kOffList = kOffMisc + 16;
  static constexpr int kSmemBytesSparse = kOffList + 16 + 2 * kMaxSparseBlocks + 1024;
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return static_cast<uint32_t>(t) * 128u; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return 256u + static_cast<uint32_t>(t * D); }
  static_assert(256 + 2 * D <= 512, "tensor-memory budget");
  static_assert(kSmemBytesSparse <= 232448, "shared-memory budget");
};

// Warps 0-7: softmax warpgroups of the two tiles; warp 8: MMA; warp 9: TMA; warps 10-11
// idle.  The kernel launches with 168 registers per thread (65536 / 384, rounded down to
// a multiple of 8); the producer warpgroup (warps 8-11) then gives registers back and the
// softmax warpgroups take them: 2 * 128 * 216 + 128 * 72 = 64512 <= 384 * 168 = 64512,
// and per SM sub-partition (one warp of each warpgroup) 216 + 216 + 72 <= 3 * 168.  The
// host checks the launch register count before launching.
constexpr int kFwdThreads = 384;
constexpr uint32_t kFwdRegsLaunch = 168;
constexpr uint32_t kFwdRegsSoftmax = 216;
constexpr uint32_t kFwdRegsProducer = 72;
static_assert(2 * 128 * kFwdRegsSoftmax + 128 * kFwdRegsProducer <= kFwdThreads * kFwdRegsLaunch,
              "register split");

// Row maximum of N raw scores (fp32 bits): four independent chains of 3-input max.
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&s)[N]) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < N; c += 8) {
    m0 = fmax3(m0, __uint_as_float(s[c + 0]), __uint_as_float(s[c + 1]));
    m1 = fmax3(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
    m2 = fmax3(m2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
    m3 = fmax3(m3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) { return row_max<128>(s); }

// P = 2^(s * sl2 - m) for N scores, packed to bf16 pairs and stored to TMEM at tP (32
// packed columns at a time, so few packed words are live at once), and the fp32 sum
// lsum.  With POLY, every sixteenth pair is evaluated on the FMA pipe (f2_exp2_poly)
// instead of the MUFU unit, to balance the two pipes (measured: 1/16 beats 0, 1/8, 1/4,
// 3/8 and 1/2 now that the row sums are cheap); blocks containing masked
// keys use the MUFU path only so masked keys give exact zeros.  The caller waits for the
// stores (tcgen05.wait::st) before signalling the MMA warp.
//
// O is normalised by the sum of the probabilities as the P V product saw them, i.e. after
// rounding to bf16.  That sum differs from lsum mostly through the rounding of each
// block's largest probability (in nearly one-hot rows it is the whole sum), so the
// caller adds that one rounding error, bf16(p_max) - p_max, to lsum instead of summing
// every rounded value (which would cost two more adds per pair).
// With DROP, P = 0 for keys the dropout mask drops (the sums keep every key: they
// normalise the softmax, dropout only reweights it); (dkey8, drow, dbh) = (first key / 8,
// row, query head) are the mask's counter words for this row.
// ppmax: the largest probability evaluated on the FMA pipe (0 without POLY), so the
// caller can tell which evaluation produced the block's largest probability.
template <int N, bool POLY, bool DROP = false>
__device__ __forceinline__ void exp_block(const uint32_t (&s)[N], float sl2, float m, uint32_t tP, float &lsum,
                                          float &ppmax, const DropCfg &dc = DropCfg{}, uint32_t dkey8 = 0,
                                          uint32_t drow = 0, uint32_t dbh = 0) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t l0 = 0, l1 = 0;  // packed (0.f, 0.f)
  float pm = 0.f;
#pragma unroll
  for (int h = 0; h < N / 64; ++h) {
    uint32_t pk[32];
    uint32_t dw[4];  // mask values of the current group of eight keys (two per word)
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int pp = h * 32 + q;
      if constexpr (DROP) {
        if ((q & 3) == 0) philox4x32_10(dkey8 + static_cast<uint32_t>(pp / 4), drow, dbh, 0u, dc.k0, dc.k1, dw);
      }
      const uint64_t x =
          f2_fma(f2_pack(__uint_as_float(s[2 * pp]), __uint_as_float(s[2 * pp + 1])), sl2x2, negm2);
      uint64_t pr;
      if (POLY && (pp & 15) == 15) {
        pr = f2_exp2_poly(x);
        float a0, a1;
        f2_unpack(pr, a0, a1);
        pm = fmax3(pm, a0, a1);
      } else {
        float x0, x1;
        f2_unpack(x, x0, x1);
        pr = f2_pack(ex2_approx(x0), ex2_approx(x1));
      }
      float p0, p1;
      f2_unpack(pr, p0, p1);
      pk[q] = pack_bf16x2(p0, p1);
      if (pp & 1)
        l1 = f2_add(l1, pr);
      else
        l0 = f2_add(l0, pr);
      if constexpr (DROP) pk[q] &= __vcmpgeu2(dw[q & 3], dc.thr2);  // keys 2pp, 2pp+1 = low, high half
    }
    tmem_st_x32(tP + h * 32, pk);
  }
  float a, b;
  f2_unpack(f2_add(l0, l1), a, b);
  lsum = a + b;
  ppmax = pm;
}

// bf16 rounding error of the probability of a block's largest score (raw maximum smax,
// offset m).  The largest probability was evaluated either on the MUFU path, which this
// repeats bit for bit, or on the FMA pipe, in which case it is (within the polynomial's
// ~1e-4 relative error) ppmax, the largest of those values.
__device__ __forceinline__ float pmax_rounding(float smax, float sl2, float m, float ppmax) {
  const float pmufu = ex2_approx(fmaf(smax, sl2, -m));
  const float pmax = ppmax >= pmufu * 0.9990234375f ? ppmax : pmufu;  // 1 - 2^-10
  return __bfloat162float(__float2bfloat16_rn(pmax)) - pmax;
}

// Epilogue of the uncommon tiles: O / sum (0 for rows without keys, or all 0 when the tile
// saw no key) either into the tile's swizzled staging rows (`direct` false, for a TMA
// store) or straight to this thread's row of O in global memory (`row_ok` rows only).
template <int D>
__device__ __noinline__ void fwd_epilogue_rows(uint32_t tO, bool has_keys, float r_run, bool row_ok,
                                               bool direct, uint32_t stage, int r, __nv_bfloat16 *orow) {
  using L = FwdLayout<D>;
  const float inv_l = r_run > 0.f ? 1.f / r_run : 0.f;
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    if (has_keys) {
      tmem_ld_x32(tO + cc * 32, o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0u;
    }
    const uint32_t rowbase = stage + (cc / 2) * L::kChunkBytes + r * 128;
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
      const int unit = (cc % 2) * 4 + uu;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * inv_l, __uint_as_float(o[8 * uu + 2 * e + 1]) * inv_l);
      if (!direct)
        st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
      else if (row_ok)
        *reinterpret_cast<uint4 *>(orow + cc * 32 + uu * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int D, int MODE, bool DROP = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams p) {
  using L = FwdLayout<D>;
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

  // ---- which two query tiles this CTA owns
  const int g = p.Hq / p.Hkv;
  int b, h[2], qb[2];
  bool valid[2];
  {
    const int u = blockIdx.x;
    int head, level;
    if (p.pair_heads) {
      const int hp_count = p.Hq / 2;
      unit_order(u, p.B * hp_count, p.nqb, p.tsz, p.tail, head, level);
      const int q = p.nqb - 1 - level;
      const int hp = head % hp_count;
      b = head / hp_count;
      h[0] = 2 * hp;
      h[1] = 2 * hp + 1;
      qb[0] = qb[1] = q;
      valid[0] = valid[1] = true;
    } else {
      const int npairs = (p.nqb + 1) / 2;
      unit_order(u, p.B * p.Hq, npairs, p.tsz, p.tail, head, level);
      const int pi = npairs - 1 - level;
      h[0] = h[1] = head % p.Hq;
      b = head / p.Hq;
      qb[0] = 2 * pi;
      qb[1] = 2 * pi + 1;
      valid[0] = true;
      valid[1] = qb[1] < p.nqb;
    }
  }
  const int kvh = h[0] / g;
  constexpr bool GEN = MODE == kAttnGeneral;
  constexpr bool SPARSE = MODE == kAttnSparse;
  constexpr bool GENLIKE = GEN || SPARSE;  // rows may see no key at all
  const bool packed = GEN && p.cu_q != nullptr;
  SeqGeom sg{p.N, p.N, 0, 0, 0};
  // Key blocks: the CTA walks the union [ulo, ulo + nu) of its tiles' ranges (contiguous:
  // the tiles are the same rows or adjacent rows, and each range is an interval around
  // its rows' key positions); tile t takes part in the local blocks [a[t], a[t] + nblk[t]).
  // A tile whose rows see no key at all has nblk = 0 and only writes O = 0, LSE = -inf.
  int a[2] = {0, 0}, nblk[2], ulo = 0, nu;
  if constexpr (GEN) {
    if (!seq_geom(p.cu_q, p.cu_k, p.N, p.total_q, p.total_k, p.nqb * 128, INT_MAX, b, sg)) return;
    // Packed sequences: tiles that start past the sequence's end have no rows.
    valid[0] = valid[0] && qb[0] * 128 < sg.Lq;
    valid[1] = valid[1] && qb[1] * 128 < sg.Lq;
    if (!valid[0]) return;  // then tile 1 (same or later block) is past the end too
    int lo0 = 0, hi0 = -1, lo1 = 0, hi1 = -1;
    const bool has0 = key_block_range<128>(p.left, p.right, sg, qb[0] * 128, lo0, hi0);
    const bool has1 = valid[1] && key_block_range<128>(p.left, p.right, sg, qb[1] * 128, lo1, hi1);
    ulo = has0 ? (has1 ? min(lo0, lo1) : lo0) : lo1;
    const int uhi = has0 ? (has1 ? max(hi0, hi1) : hi0) : hi1;
    nu = (has0 || has1) ? uhi - ulo + 1 : 0;
    a[0] = has0 ? lo0 - ulo : 0;
    nblk[0] = has0 ? hi0 - lo0 + 1 : 0;
    a[1] = has1 ? lo1 - ulo : 0;
    nblk[1] = has1 ? hi1 - lo1 + 1 : 0;
  } else if constexpr (!SPARSE) {
#pragma unroll
    for (int t = 0; t < 2; ++t) nblk[t] = !valid[t] ? 0 : (MODE == kAttnCausal ? qb[t] + 1 : p.nqb);
    nu = nblk[0] > nblk[1] ? nblk[0] : nblk[1];
  }
  // Block-sparse: tile t visits the enabled key blocks of its mask row (those up to the
  // diagonal when causal), in order; the CTA walks the union of the two tiles' lists, which
  // an idle warp writes to shared memory before the roles start.
  const uint16_t *blist = reinterpret_cast<const uint16_t *>(smem + L::kOffList + 16);
  // TMA coordinates (dimensions 1 and 2) of a 128-row tile: dense maps are [B*H][N][d],
  // packed maps [total][H][d].
  auto q_coords = [&](int hh, int row, int &c1, int &c2) {
    c1 = packed ? hh : row;
    c2 = packed ? sg.q_base + row : b * p.Hq + hh;
  };
  auto kv_coords = [&](int row, int &c1, int &c2) {
    c1 = packed ? kvh : row;
    c2 = packed ? sg.k_base + row : b * p.Hkv + kvh;
  };

  // ---- barriers and tensor memory
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(bar(i), (i == L::kBarP || i == L::kBarP + 1) ? 4u : 1u);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), L::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  if constexpr (SPARSE) {
    if (warp == 10) {
      const bool causal = p.right == 0;
      const uint8_t *row[2];
      int hi[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        row[t] = p.bmask + (static_cast<size_t>(b * p.Hq + h[t]) * p.nqb + qb[t]) * p.nqb;
        hi[t] = !valid[t] ? -1 : (causal ? qb[t] : p.nqb - 1);
      }
      uint16_t *list = reinterpret_cast<uint16_t *>(smem + L::kOffList + 16);
      int n = 0, c0 = 0, c1 = 0;
      const int hmax = hi[0] > hi[1] ? hi[0] : hi[1];
      for (int base0 = 0; base0 <= hmax; base0 += 32) {
        const int kb = base0 + lane;
        const bool m0 = kb <= hi[0] && row[0][kb] != 0;
        const bool m1 = kb <= hi[1] && row[1][kb] != 0;
        const uint32_t u = __ballot_sync(0xffffffffu, m0 || m1);
        if (m0 || m1)
          list[n + __popc(u & ((1u << lane) - 1u))] =
              static_cast<uint16_t>(kb | (m0 ? 1 << 14 : 0) | (m1 ? 1 << 15 : 0));
        n += __popc(u);
        c0 += __popc(__ballot_sync(0xffffffffu, m0));
        c1 += __popc(__ballot_sync(0xffffffffu, m1));
      }
      if (lane == 0) {
        int *hdr = reinterpret_cast<int *>(smem + L::kOffList);
        hdr[0] = n;
        hdr[1] = c0;
        hdr[2] = c1;
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];
  if constexpr (SPARSE) {
    const int *hdr = reinterpret_cast<const int *>(smem + L::kOffList);
    nu = hdr[0];
    nblk[0] = hdr[1];
    nblk[1] = hdr[2];
  }

  if (warp >= 8) {
  // ================================================================ producer warpgroup
  setmaxnreg_dec<kFwdRegsProducer>();
  if (warp >= 10) {
    // idle warps of the producer warpgroup
  } else if (warp == 9) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (nblk[t] == 0) continue;
        int c1, c2;
        q_coords(h[t], qb[t] * 128, c1, c2);
        mbar_arrive_expect_tx(bar(L::kBarQ + t), L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sQ + t * L::kTileBytes + c * L::kChunkBytes, &tm_q, bar(L::kBarQ + t), c * 64, c1, c2);
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; ok && j < nu; ++j) {
#pragma unroll
        for (int kind = 0; kind < 2; ++kind) {
          const int seq = 2 * j + kind, slot = seq % S, use = seq / S;
          if (!wait_bounded(bar(L::kBarKVEmpty + slot), (use & 1) ^ 1, abort_flag,
                            wait_site(1, L::kBarKVEmpty + slot, j))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::kBarKVFull + slot), L::kTileBytes);
          const CUtensorMap *m = kind ? &tm_v : &tm_k;
          int c1, c2;
          kv_coords((SPARSE ? (blist[j] & 0x3FFF) : ulo + j) * 128, c1, c2);
#pragma unroll
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_3d(sKV + slot * L::kTileBytes + c * L::kChunkBytes, m, bar(L::kBarKVFull + slot),
                        c * 64, c1, c2);
          ++issued;
        }
      }
      // No copy may still be landing in shared memory when the CTA exits.
      for (int seq = issued > S ? issued - S : 0; seq < issued; ++seq)
        wait_drain(bar(L::kBarKVFull + seq % S), (seq / S) & 1, 100000000ull);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (nblk[t] > 0) wait_drain(bar(L::kBarQ + t), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 8) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      auto kslot = [](int j) { return (2 * j) % S; };
      auto kpar = [](int j) { return static_cast<uint32_t>(((2 * j) / S) & 1); };
      auto vslot = [](int j) { return (2 * j + 1) % S; };
      auto vpar = [](int j) { return static_cast<uint32_t>(((2 * j + 1) / S) & 1); };
      // S_t = Q_t K_j^T : M = 128 query rows, N = 128 keys, K = D (16 per instruction).
      // (buf: the S buffer; the dense variants use buffer t for tile t)
      auto issue_qk = [&](int t, int j, int buf) {
        const uint32_t a0 = sQ + t * L::kTileBytes;
        const uint32_t b0 = sKV + kslot(j) * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::kChunkBytes + (kk % 4) * 32;
          mma_ss(tmem + L::tm_s(buf), sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024),
                 idesc_qk, kk > 0);
        }
      };
      // O_t += P_t V_j : M = 128 query rows, N = D, K = 128 keys; P (bf16) in TMEM,
      // V MN-major in shared memory (16 key rows = 2048 bytes per instruction).
      auto issue_pv = [&](int t, int j, bool first, int buf) {
        const uint32_t b0 = sKV + vslot(j) * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + L::tm_o(t), tmem + L::tm_s(buf) + kk * 8,
                 sdesc_sw128(b0 + kk * 2048, L::kChunkBytes, 1024), idesc_pv, (!first || kk > 0));
      };

      if constexpr (SPARSE) {
        // Union step j loads key block blist[j]; tile t takes part in the steps whose entry
        // carries its bit.  Score tiles are numbered n = 0, 1, ... in list order (tile 0
        // before tile 1 within a step) and use the two S buffers alternately (n & 1), so a
        // tile whose blocks come in a run can have its next Q K^T computed while its
        // softmax works on the current one.  Score tile n + 2 is issued right after P V of
        // score tile n, which frees its buffer.  Every barrier has one waiter that takes
        // its phases in order and can never fall two phases behind or ahead: "S ready" per
        // (buffer, tile) (kBarS + b for tile 0, kBarSX + b for tile 1), "P written" per
        // buffer (the MMA consumes score tiles in order, and a buffer's next occupant is
        // issued only after its P was consumed), "P V done" per tile for the softmax's rare
        // rescale of O.
        const int total = nblk[0] + nblk[1];
        auto first_pos = [&](int &j, int &t) {
          j = 0;
          t = (blist[0] & (1u << 14)) ? 0 : 1;
        };
        auto advance = [&](int &j, int &t) {
          if (t == 0 && (blist[j] & (1u << 15))) {
            t = 1;
            return;
          }
          ++j;
          if (j < nu) t = (blist[j] & (1u << 14)) ? 0 : 1;
        };
        auto last_of_step = [&](int j, int t) { return t == 1 || !(blist[j] & (1u << 15)); };
        bool ok = nu > 0;
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (ok && nblk[t] > 0) ok = wait_bounded(bar(L::kBarQ + t), 0, abort_flag, wait_site(1, L::kBarQ + t, 0));
        int qj = 0, qt = 0, nq = 0, k_ready = -1;
        auto issue_next_qk = [&]() {
          if (qj != k_ready) {
            if (!wait_bounded(bar(L::kBarKVFull + kslot(qj)), kpar(qj), abort_flag,
                              wait_site(1, L::kBarKVFull + kslot(qj), qj))) {
              ok = false;
              return;
            }
            tc_fence_after_sync();
            k_ready = qj;
          }
          issue_qk(qt, qj, nq & 1);
          tc_commit(bar((qt ? L::kBarSX : L::kBarS) + (nq & 1)));
          if (last_of_step(qj, qt)) tc_commit(bar(L::kBarKVEmpty + kslot(qj)));
          ++nq;
          advance(qj, qt);
        };
        if (ok) {
          first_pos(qj, qt);
          issue_next_qk();
          if (ok && total > 1) issue_next_qk();
        }
        int cnt[2] = {0, 0};  // P V products issued per tile
        int pj = 0, pt = 0, v_ready = -1;
        if (ok) first_pos(pj, pt);
        for (int n = 0; ok && n < total; ++n) {
          if (pj != v_ready) {
            if (!wait_bounded(bar(L::kBarKVFull + vslot(pj)), vpar(pj), abort_flag,
                              wait_site(1, L::kBarKVFull + vslot(pj), pj))) {
              ok = false;
              break;
            }
            v_ready = pj;
          }
          if (!wait_bounded(bar(L::kBarP + (n & 1)), (n >> 1) & 1, abort_flag,
                            wait_site(1, L::kBarP + (n & 1), n))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          issue_pv(pt, pj, cnt[pt] == 0, n & 1);
          ++cnt[pt];
          tc_commit(bar(L::kBarPV + pt));
          if (cnt[pt] == nblk[pt]) tc_commit(bar(L::kBarO + pt));  // the tile's last block
          if (last_of_step(pj, pt)) tc_commit(bar(L::kBarKVEmpty + vslot(pj)));
          if (n + 2 < total) issue_next_qk();
          advance(pj, pt);
        }
        tc_commit(bar(L::kBarDrain));
        wait_drain(bar(L::kBarDrain), 0, 100000000ull);
      } else {
      // Local block range of each tile (an empty tile gets an empty range; in the dense
      // variants every tile starts at block 0).
      const int first[2] = {!GEN ? 0 : (nblk[0] > 0 ? a[0] : 1 << 30), !GEN ? 0 : (nblk[1] > 0 ? a[1] : 1 << 30)};
      const int last[2] = {a[0] + nblk[0] - 1, a[1] + nblk[1] - 1};
      bool ok = nu > 0;
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (ok && nblk[t] > 0) ok = wait_bounded(bar(L::kBarQ + t), 0, abort_flag, wait_site(1, L::kBarQ + t, 0));
      if (ok) ok = wait_bounded(bar(L::kBarKVFull + kslot(0)), kpar(0), abort_flag,
                                wait_site(1, L::kBarKVFull + kslot(0), 0));
      if (ok) {
        tc_fence_after_sync();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (nblk[t] == 0 || a[t] != 0) continue;
          issue_qk(t, 0, t);
          tc_commit(bar(L::kBarS + t));
        }
        tc_commit(bar(L::kBarKVEmpty + kslot(0)));
      }
      for (int j = 0; ok && j < nu; ++j) {
        if (!wait_bounded(bar(L::kBarKVFull + vslot(j)), vpar(j), abort_flag,
                          wait_site(1, L::kBarKVFull + vslot(j), j))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        bool knext = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          // Tile t takes part in blocks first[t] .. last[t]; at j = first[t] - 1 only its
          // first S = Q K^T is due.
          if (!ok || j + 1 < first[t] || j > last[t]) continue;
          if (j >= first[t]) {
            if (!wait_bounded(bar(L::kBarP + t), (j - first[t]) & 1, abort_flag, wait_site(1, L::kBarP + t, j))) {
              ok = false;
              continue;
            }
            tc_fence_after_sync();
            issue_pv(t, j, j == first[t], t);
          }
          if (j < last[t]) {
            if (!knext) {
              if (!wait_bounded(bar(L::kBarKVFull + kslot(j + 1)), kpar(j + 1), abort_flag,
                                wait_site(1, L::kBarKVFull + kslot(j + 1), j + 1))) {
                ok = false;
                continue;
              }
              tc_fence_after_sync();
              knext = true;
            }
            issue_qk(t, j + 1, t);
            tc_commit(bar(L::kBarS + t));
          } else {
            tc_commit(bar(L::kBarO + t));  // jt is this tile's last block
          }
        }
        if (!ok) break;
        tc_commit(bar(L::kBarKVEmpty + vslot(j)));
        if (knext) tc_commit(bar(L::kBarKVEmpty + kslot(j + 1)));
      }
      // Nothing issued by this thread may still run when tensor memory is released.
      tc_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0, 100000000ull);
      }
    }
    __syncwarp();
  }
  } else {
    // ================================================================ softmax warpgroups
    setmaxnreg_inc<kFwdRegsSoftmax>();
    const int t = warp / 4;
    const int wq = warp % 4;          // TMEM lane quadrant of this warp
    const int r = wq * 32 + lane;     // row of the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t tS = tmem + L::tm_s(t) + lane_off;  // block-sparse: the block's S buffer
    const uint32_t tO = tmem + L::tm_o(t) + lane_off;
    // This warpgroup's tile (selects instead of runtime-indexed arrays keep them in registers).
    const int my_qb = t ? qb[1] : qb[0];
    const int my_h = t ? h[1] : h[0];
    const int my_n = t ? nblk[1] : nblk[0];
    const int my_j0 = ulo + (t ? a[1] : a[0]);  // first key block of this tile
    const bool my_valid = t ? valid[1] : valid[0];
    const int qrow = my_qb * 128 + r;
    bool ok = my_valid;
    // l_run: sum of the fp32 probabilities (for the LSE); r_run: the same with each
    // block's largest probability counted as rounded to bf16, i.e. (to within the other,
    // much smaller rounding errors) the weights the P V product actually used, so that
    // O / r_run is a properly normalised average.
    float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
    const float sl2 = p.sl2;
    // Block-sparse: this tile's current entry of the block list, and the number of score
    // tiles (both tiles) listed before it, which gives the block's S buffer and phase.
    int cur = -1, nbase = 0, prev_bits = 0, uses0 = 0, uses1 = 0;  // uses: own blocks per buffer
    for (int j = 0; ok && j < my_n; ++j) {
      int sb = L::kBarS + t, sp = j & 1, pb = L::kBarP + t;
      if constexpr (SPARSE) {
        do {
          nbase += prev_bits;
          ++cur;
          prev_bits = __popc(static_cast<uint32_t>(blist[cur]) >> 14);
        } while (cur < nu - 1 && !(blist[cur] & (1u << (14 + t))));
        const int n = nbase + ((t == 1 && (blist[cur] & (1u << 14))) ? 1 : 0);
        const int bsel = n & 1;
        sb = (t ? L::kBarSX : L::kBarS) + bsel;
        sp = (bsel ? uses1 : uses0) & 1;
        if (bsel) ++uses1; else ++uses0;
        pb = L::kBarP + bsel;
        tS = tmem + L::tm_s(bsel) + lane_off;
      }
      if (!warp_wait_bounded(bar(sb), sp, abort_flag, wait_site(1, sb, j))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t s[128];
      {
        // Two 64-column loads and one wait (a single 128-register load cannot be
        // allocated once the warpgroup's register budget is set with setmaxnreg).
        uint32_t (&s0)[64] = *reinterpret_cast<uint32_t(*)[64]>(&s[0]);
        uint32_t (&s1)[64] = *reinterpret_cast<uint32_t(*)[64]>(&s[64]);
        tmem_ld_x64_nowait(tS, s0);
        tmem_ld_x64_nowait(tS + 64, s1);
        tmem_wait_ld_2x64(s0, s1);
      }
      const int kv0 = (SPARSE ? (blist[cur] & 0x3FFF) : my_j0 + j) * 128;
      bool masked;
      if constexpr (GEN) {
        masked = block_needs_mask<128>(p.left, p.right, sg.Lk, my_qb * 128 + sg.dlt, kv0);
        if (masked) mask_scores<128>(s, p.left, p.right, sg.Lk, qrow + sg.dlt, kv0);
      } else {
        const bool causal = MODE == kAttnCausal || (SPARSE && p.right == 0);
        masked = (causal && kv0 == my_qb * 128) || kv0 + 128 > p.N;
        if (masked) {
          const int lim = causal ? min(qrow + 1, p.N) : p.N;  // keys kv < lim are visible
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (kv0 + c >= lim) s[c] = __float_as_uint(-INFINITY);
        }
      }
      const float smax = row_max128(s);
      const float m_cand = smax * sl2;
      const float m_new = (m_cand > m_run + kRescaleThreshold) ? m_cand : m_run;
      // 0 on a row's first visible block, else <= 1.  A band can hide a whole block from
      // a row; while its max is still -inf the offset stays 0 and alpha 1 (no inf - inf).
      const float alpha = (GEN && m_new == m_run) ? 1.f : ex2_approx(m_run - m_new);
      const float m_use = (GEN && m_new == -INFINITY) ? 0.f : m_new;
      float lsum, ppmax;
      if (masked)
        exp_block<128, false, DROP>(s, sl2, m_use, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow,
                                    b * p.Hq + my_h);   // exact zeros for masked keys
      else
        exp_block<128, true, DROP>(s, sl2, m_new, tS, lsum, ppmax, p.drop, kv0 >> 3, qrow, b * p.Hq + my_h);
      l_run = l_run * alpha + lsum;
      r_run = r_run * alpha + (lsum + pmax_rounding(smax, sl2, m_use, ppmax));
      m_run = m_new;
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O was last written by P V of block j-1.  Dense: it completed before S_j was
        // ready.  Block-sparse: S_j may have been computed ahead of it, so wait for it.
        if constexpr (SPARSE) {
          if (!warp_wait_bounded(bar(L::kBarPV + t), (j - 1) & 1, abort_flag, wait_site(1, L::kBarPV + t, j))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
        }
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
      if (lane == 0) mbar_arrive(bar(pb));  // one arrival per warp
    }

    // ---- epilogue: O / l -> bf16 -> shared memory (this tile's Q slot) -> TMA store.  Two
    // cases take a separate path: a packed tile that ends past its sequence stores its
    // rows directly, and a tile that sees no key writes O = 0 (no MMA touched it).
    if (my_valid) {
      bool okw = ok && ((GENLIKE && my_n == 0) ||
                        warp_wait_bounded(bar(L::kBarO + t), 0, abort_flag, wait_site(1, L::kBarO + t, 0)));
      okw = named_bar_and(1 + t, 128, okw && *abort_flag == 0);
      const bool direct = packed && my_qb * 128 + 128 > sg.Lq;
      if (okw && (!GENLIKE || (!direct && my_n > 0))) {
        tc_fence_after_sync();
        // rows without keys: O = 0; dropout scales the kept probabilities by 1 / (1 - p)
        const float inv_l = (!GEN || r_run > 0.f) ? (DROP ? p.drop.inv_keep : 1.f) / r_run : 0.f;
        const uint32_t stage = sQ + t * L::kTileBytes;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld_x32(tO + cc * 32, o);
          const uint32_t rowbase = stage + (cc / 2) * L::kChunkBytes + r * 128;
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const int unit = (cc % 2) * 4 + uu;   // 16-byte unit within the 128-byte row
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * inv_l,
                                 __uint_as_float(o[8 * uu + 2 * e + 1]) * inv_l);
            st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + t, 128);
        if (r == 0) {
          int c1, c2;
          q_coords(my_h, my_qb * 128, c1, c2);
#pragma unroll
          for (int c = 0; c < L::kChunks; ++c) tma_store_3d(&tm_o, stage + c * L::kChunkBytes, c * 64, c1, c2);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      } else if (GENLIKE && okw) {
        fwd_epilogue_rows<D>(tO, my_n > 0, r_run, qrow < sg.Lq, direct, sQ + t * L::kTileBytes, r,
                             p.o + (static_cast<size_t>(sg.q_base + qrow) * p.Hq + my_h) * D);
        if (!direct) {
          fence_proxy_async_smem();
          named_bar_sync(1 + t, 128);
          if (r == 0) {
            int c1, c2;
            q_coords(my_h, my_qb * 128, c1, c2);
#pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
              tma_store_3d(&tm_o, sQ + t * L::kTileBytes + c * L::kChunkBytes, c * 64, c1, c2);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
        }
      }
      if (okw && qrow < sg.Lq) {
        const float lse = (!GENLIKE || l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        if (packed)
          p.lse[static_cast<size_t>(sg.q_base + qrow) * p.Hq + my_h] = lse;
        else
          p.lse[static_cast<size_t>(b * p.Hq + my_h) * p.N + qrow] = lse;
      }
    }
  }

  // ---- teardown: every role has drained; release tensor memory
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
