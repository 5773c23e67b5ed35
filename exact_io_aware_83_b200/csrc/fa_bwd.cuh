// fa_bwd.cuh - backward attention kernels for sm_100a.
//
// The pages require only that the backward pass recompute the attention tiles on chip
// instead of storing them ("The Future of AI ..." page, bullet "Recomputation"; the
// "FlashAttention1" Q&A, question on integration, item 6).  The gradient itself is the
// plain calculus of L = <O, dO> for O = softmax(scale Q K^T) V:
//   P_ij   = exp(scale q_i.k_j - LSE_i)             (recomputed from Q, K and the LSE)
//   dP_ij  = do_i . v_j
//   Delta_i = sum_j P_ij dP_ij = do_i . o_i
//   dS_ij  = P_ij (dP_ij - Delta_i)
//   dV_j   = sum_i P_ij do_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
// (dK, dV summed over the query heads that share a K/V head), with P_ij = 0 for keys
// outside query i's window i - left <= j <= i + right (causal: left unlimited, right 0)
// or, block-sparse, outside the enabled 128 x 128 blocks of the query head's mask.
//
// Three kernels on one stream:
//  1. fa_bwd_pre:  Delta_i = <dO_i, O_i> (fp32) and a zeroed fp32 dQ accumulator.
//  2. fa_bwd_main: one CTA per (b, K/V head, 128-key block).  It keeps K_j and V_j in
//     shared memory and dK_j, dV_j in tensor memory, and walks every (query head of the
//     group, 64-row query block) that can see the key block (a window or a block mask
//     skips the others):
//        S^T  = K Q_i^T        (tcgen05, TMEM)      P^T = exp2(S^T scale log2e - LSE2_i)
//        dP^T = V dO_i^T       (tcgen05, TMEM)      dS^T = P^T (dP^T - Delta_i)
//        dV  += P^T dO_i       (P^T read from TMEM as the A operand)
//        dK  += dS^T Q_i       (dS^T from swizzled shared memory, K-major)
//        dQ_i^T = K^T dS^T     (same dS^T tile read MN-major) -> fp32 TMA reduce-add
//     Warps 0-7 are two elementwise warpgroups: each thread owns one key row (its TMEM
//     lane) and each warpgroup half of the query columns (P^T, dS^T, then the dV / dK
//     epilogue); warps 8-11 drain dQ^T from TMEM into the fp32 accumulator; warp 12
//     issues the MMAs; warp 13 loads (TMA for K, V, Q_i, dO_i; plain loads for LSE_i and
//     Delta_i).
//  3. fa_bwd_post: dQ = bf16(scale * dQacc).
// For d = 256 the two K/V accumulators would need all 512 TMEM columns, so two CTAs
// share each key block, each owning one 128-column half of dK, dV and dQ (both
// recompute S^T and dP^T over the full d), with 32-row query blocks so the tiles fit.
#pragma once

#include "fa_common.cuh"

namespace fa {

// ============================================================================ pre / post

template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_pre_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout,
                      float *__restrict__ delta, float *__restrict__ dqacc, long long rows) {
  constexpr int kPer = D / 32;  // bf16 elements per lane
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const __nv_bfloat16 *orow = o + row * D + lane * kPer;
  const __nv_bfloat16 *drow = dout + row * D + lane * kPer;
  float acc = 0.f;
  if constexpr (kPer == 2) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(orow);
    const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162 *>(drow);
    acc = __bfloat162float(a.x) * __bfloat162float(c.x) + __bfloat162float(a.y) * __bfloat162float(c.y);
  } else {
    constexpr int kVec = kPer / 4;  // 8-byte vectors
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      const uint2 a = reinterpret_cast<const uint2 *>(orow)[v];
      const uint2 c = reinterpret_cast<const uint2 *>(drow)[v];
      const __nv_bfloat162 *a2 = reinterpret_cast<const __nv_bfloat162 *>(&a);
      const __nv_bfloat162 *c2 = reinterpret_cast<const __nv_bfloat162 *>(&c);
#pragma unroll
      for (int e = 0; e < 2; ++e)
        acc += __bfloat162float(a2[e].x) * __bfloat162float(c2[e].x) +
               __bfloat162float(a2[e].y) * __bfloat162float(c2[e].y);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
  float *qrow = dqacc + row * D;
#pragma unroll
  for (int c = lane * 4; c < D; c += 128)
    *reinterpret_cast<float4 *>(qrow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(256)
    fa_bwd_post_kernel(const float *__restrict__ dqacc, __nv_bfloat16 *__restrict__ dq, float scale,
                       long long n8) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4 *>(dqacc)[2 * i];
  const float4 c = reinterpret_cast<const float4 *>(dqacc)[2 * i + 1];
  uint4 w;
  w.x = pack_bf16x2(a.x * scale, a.y * scale);
  w.y = pack_bf16x2(a.z * scale, a.w * scale);
  w.z = pack_bf16x2(c.x * scale, c.y * scale);
  w.w = pack_bf16x2(c.z * scale, c.w * scale);
  reinterpret_cast<uint4 *>(dq)[i] = w;
}

// ============================================================================ main kernel

struct BwdParams {
  const float *lse;       // dense: [B, Hq, N]; packed sequences: [total_q, Hq]
  const float *delta;     // same layout as lse
  __nv_bfloat16 *dk, *dv; // packed sequences: for the rows of key blocks that end past a sequence
  const int *cu_q, *cu_k; // packed sequences: [B + 1] row offsets (nullptr: dense [B, H, N, d])
  int B, Hq, Hkv, N;
  int total_q, total_k;
  int nkb;                // key blocks of 128 per sequence (packed: of the longest)
  int left, right;        // key band around the diagonal (see SeqGeom); -1 = unlimited
  float sl2;              // scale * log2(e)
  float scale;
  DropCfg drop;           // dropout (kernels instantiated with DROP only)
  const uint8_t *bmask;   // block-sparse: [B, Hq, nkb, nkb] 0/1 over 128 x 128 blocks
  int tsz;                // unit order: key-block levels per tier (see unit_order)
  int tail;               // unit order: heads taken level by level at the end
};

// D: head dimension (contraction of S^T and dP^T); DH: output columns owned by a CTA
// (D, or 128 when D = 256); BQ: query rows per step.
template <int D, int DH, int BQ>
struct BwdLayout {
  static constexpr int kKRows = 128;
  static constexpr int kChunks = D / 64;
  static constexpr int kKChunk = kKRows * 128;      // [128 x 64] bf16 box
  static constexpr int kKTile = kChunks * kKChunk;
  static constexpr int kQChunk = BQ * 128;          // [BQ x 64] bf16 box
  static constexpr int kQTile = kChunks * kQChunk;
  static constexpr int kQStages = (D == 256) ? 2 : 3;
  static constexpr int kDSRowBytes = 128;           // dS^T rows padded to one 128-B swizzle row
  static constexpr int kDSBytes = kKRows * kDSRowBytes;
  static constexpr int kDQHalves = (BQ * DH * 4 > 32768) ? 2 : 1;  // dQ staging passes
  static constexpr int kDQCols = DH / kDQHalves;    // d columns staged per pass
  static constexpr int kDQBytes = BQ * kDQCols * 4;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKTile;
  static constexpr int kOffQ = kOffV + kKTile;                // Q ring
  static constexpr int kOffDO = kOffQ + kQStages * kQTile;    // dO ring
  static constexpr int kOffDS = kOffDO + kQStages * kQTile;
  static constexpr int kOffDQ = kOffDS + kDSBytes;
  static constexpr int kOffVec = kOffDQ + kDQBytes;           // [stage][lse2 | delta][BQ] fp32
  static constexpr int kVecBytes = kQStages * 2 * BQ * 4;
  static constexpr int kOffBar = kOffVec + kVecBytes;
  // mbarriers
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;
  static constexpr int kBarQEmpty = kBarQFull + kQStages;
  static constexpr int kBarS = kBarQEmpty + kQStages;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarP = kBarDP + 1;
  static constexpr int kBarDS = kBarP + 1;
  static constexpr int kBarDSEmpty = kBarDS + 1;
  static constexpr int kBarDQ = kBarDSEmpty + 1;
  static constexpr int kBarDQEmpty = kBarDQ + 1;
  static constexpr int kBarFinal = kBarDQEmpty + 1;
  static constexpr int kBarDrain = kBarFinal + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // Block-sparse variant only: after misc, a 16-byte header (steps counted by each of the
  // four warps that build it) and a bitmap per query head of the group: bit qb of head hh
  // is set when 128-row query block qb of that head sees this key block.
  static constexpr int kOffList = kOffMisc + 16;
  static constexpr int kSparseBitmapBytes =
      (232448 - (kOffList + 16 + 1024)) / 4 * 4 < 8192 ? (232448 - (kOffList + 16 + 1024)) / 4 * 4 : 8192;
  static constexpr int kSmemBytesSparse = kOffList + 16 + kSparseBitmapBytes + 1024;
  // tensor memory: dV | dK | S^T | dP^T | dQ^T
  static constexpr uint32_t kTmDV = 0;
  static constexpr uint32_t kTmDK = DH;
  static constexpr uint32_t kTmS = 2 * DH;
  static constexpr uint32_t kTmDP = 2 * DH + BQ;
  static constexpr uint32_t kTmDQ = 2 * DH + 2 * BQ;
  static constexpr uint32_t kTmemCols = 512;
  // Elementwise work is split between two warpgroups by query column: each owns HC of
  // the BQ columns of every key row.  Its bf16 P^T half is packed into the first HC/2
  // columns of its OWN S^T half, so neither warpgroup overwrites scores the other has
  // not read yet.  K-step kk (16 queries) of P^T therefore sits at column pcol(kk).
  static constexpr int kHC = BQ / 2;
  static constexpr int kKStepsPerHalf = kHC / 16;
  __host__ __device__ static constexpr uint32_t pcol(int kk) {
    return static_cast<uint32_t>((kk / kKStepsPerHalf) * kHC + (kk % kKStepsPerHalf) * 8);
  }
  static_assert(kTmDQ + BQ <= 512, "tensor-memory budget");
  static_assert(kSmemBytesSparse <= 232448 && kSparseBitmapBytes >= 256, "shared-memory budget");
  static_assert(BQ == 32 || BQ == 64, "query block");
};

// Warps 0-7: two elementwise warpgroups; 8-11: dQ drain; 12: MMA; 13: loader.
constexpr int kBwdThreads = 448;

// Block-sparse backward: the steps of a key-block CTA are (query head hh of the group,
// BQ-row query block) for every 128-row query block whose bit is set in head hh's bitmap,
// heads in order, blocks in order, the 128 / BQ sub-blocks of each block in order (the last
// block of the sequence has only those that start before N).  Each role walks the same
// sequence with its own cursor.
struct SparseSteps {
  const uint32_t *bits;  // [g][W] words
  int W, g, nqb, nsub, nsub_last;
  int hh, qb, sub;
  __device__ __forceinline__ void init(const uint32_t *bits_, int W_, int g_, int nqb_, int nsub_, int nsub_last_) {
    bits = bits_;
    W = W_;
    g = g_;
    nqb = nqb_;
    nsub = nsub_;
    nsub_last = nsub_last_;
    hh = 0;
    qb = -1;
    sub = 0;
  }
  // First set bit >= from in head hh's bitmap, or -1.
  __device__ __forceinline__ int find(int from) const {
    for (int w = from >> 5; w < W; ++w) {
      uint32_t u = bits[hh * W + w];
      if (w == (from >> 5)) u &= ~0u << (from & 31);
      if (u) return w * 32 + __ffs(u) - 1;
    }
    return -1;
  }
  // Moves to the next step (the first one on the first call); bounded by the bitmap.
  __device__ __forceinline__ void next() {
    if (qb >= 0 && ++sub < (qb == nqb - 1 ? nsub_last : nsub)) return;
    sub = 0;
    while (hh < g) {
      qb = find(qb + 1);
      if (qb >= 0) return;
      ++hh;
      qb = -1;
    }
  }
  template <int BQ>
  __device__ __forceinline__ int q0() const { return qb * 128 + sub * BQ; }
};

// Kernel variants (kAttnFull, kAttnCausal, kAttnGeneral, kAttnSparse, see fa_common.cuh):
// dense full and dense causal attention, the general form (packed sequences and/or a key
// band), and a 0/1 mask over 128 x 128 blocks (optionally with the causal mask).
template <int D, int DH, int BQ, int MODE, bool DROP = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using L = BwdLayout<D, DH, BQ>;
  constexpr int QS = L::kQStages;
  constexpr int HC = L::kHC;
  constexpr int kHalves = D / DH;  // CTAs per key block
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  float *vec = reinterpret_cast<float *>(smem + L::kOffVec);
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBar + 8u * static_cast<uint32_t>(i); };
  const uint32_t sK = base + L::kOffK, sV = base + L::kOffV;
  const uint32_t sQ = base + L::kOffQ, sDO = base + L::kOffDO;
  const uint32_t sDS = base + L::kOffDS, sDQ = base + L::kOffDQ;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- unit: (b, kv head, key block, d half); first key blocks (heaviest under a causal
  // mask) first
  const int half = static_cast<int>(blockIdx.x) % kHalves;
  int head, kb;
  unit_order(static_cast<int>(blockIdx.x) / kHalves, p.B * p.Hkv, p.nkb, p.tsz, p.tail, head, kb);
  const int kvh = head % p.Hkv;
  const int b = head / p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int kv0 = kb * 128;
  constexpr bool GEN = MODE == kAttnGeneral;
  const bool packed = GEN && p.cu_q != nullptr;
  SeqGeom sg{p.N, p.N, 0, 0, 0};
  int q_first, nq;
  if constexpr (GEN) {
    if (!seq_geom(p.cu_q, p.cu_k, p.N, p.total_q, p.total_k, INT_MAX, p.nkb * 128, b, sg)) return;
    if (kv0 >= sg.Lk) return;  // packed: the block starts past the sequence's keys
    // Query blocks that can see some key of this block: query i sits at key position
    // i + dlt and sees key j iff j - right <= i + dlt <= j + left.
    const int kv1 = min(kv0 + 127, sg.Lk - 1);
    const int first_i = p.right < 0 ? 0 : max(0, kv0 - p.right - sg.dlt);
    const int last_i = p.left < 0 ? sg.Lq - 1 : min(sg.Lq - 1, kv1 + p.left - sg.dlt);
    q_first = first_i / BQ;
    nq = last_i >= first_i ? last_i / BQ - q_first + 1 : 0;  // 0: dK = dV = 0
  } else {
    q_first = MODE == kAttnCausal ? kv0 / BQ : 0;
    nq = (p.N + BQ - 1) / BQ - q_first;
  }
  constexpr bool SPARSE = MODE == kAttnSparse;
  constexpr bool GENLIKE = GEN || SPARSE;  // a key block may see no query at all
  int T = g * nq;  // steps: (query head of the group, query block); block-sparse: counted below
  const int spW = (p.nkb + 31) / 32;
  constexpr int kSub = 128 / BQ;
  const int spSubLast = (p.N - (p.nkb - 1) * 128 + BQ - 1) / BQ;
  uint32_t *spbits = reinterpret_cast<uint32_t *>(smem + L::kOffList + 16);
  const int dcol0 = half * DH;  // first output column owned by this CTA
  // TMA coordinates (dimensions 1 and 2): dense maps are [B*H][N][cols], packed [total][H][cols].
  auto q_coords = [&](int hh, int row, int &c1, int &c2) {
    c1 = packed ? hh : row;
    c2 = packed ? sg.q_base + row : b * p.Hq + hh;
  };
  const int kv_c1 = packed ? kvh : kv0, kv_c2 = packed ? sg.k_base + kv0 : b * p.Hkv + kvh;
  // Row of query q of head hh in the LSE / Delta vectors.
  auto vec_row = [&](int hh, int q) -> size_t {
    return packed ? static_cast<size_t>(sg.q_base + q) * p.Hq + hh : static_cast<size_t>(b * p.Hq + hh) * p.N + q;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == L::kBarP || i == L::kBarDS) cnt = 8;   // one arrival per elementwise warp
      if (i == L::kBarDQEmpty) cnt = 4;               // one per dQ-drain warp
      // Q/dO stages: the TMA expect-tx arrival plus the arrival after the LSE / Delta stores.
      if (i >= L::kBarQFull && i < L::kBarQFull + QS) cnt = 2;
      mbar_init(bar(i), cnt);
    }
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_u32(misc), L::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  if constexpr (SPARSE) {
    // Warps 8-11 (idle until the first dQ) read this key block's column of the mask for
    // every head of the group, sixteen independent loads per lane in flight, and write the
    // bitmaps and their step counts.
    if (warp >= 8 && warp < 12) {
      const int wq = warp - 8, nw = g * spW;
      const int qlo = p.right == 0 ? kb : 0;  // causal: query blocks at or after the diagonal
      const size_t col0 = static_cast<size_t>(b * p.Hq + kvh * g) * p.nkb * p.nkb + kb;
      int steps = 0;
      for (int f0 = wq; f0 < nw; f0 += 4 * 16) {
        bool v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int fw = f0 + 4 * k;
          const int hh = fw / spW, qb = (fw - hh * spW) * 32 + lane;
          v[k] = fw < nw && qb >= qlo && qb < p.nkb &&
                 p.bmask[col0 + (static_cast<size_t>(hh) * p.nkb + qb) * p.nkb] != 0;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int fw = f0 + 4 * k;
          const uint32_t u = __ballot_sync(0xffffffffu, v[k]);
          if (fw < nw && lane == 0) {
            spbits[fw] = u;
            steps += __popc(u) * kSub;
            // the sequence's last query block has only the sub-blocks that start before N
            if (fw % spW == spW - 1 && ((u >> ((p.nkb - 1) & 31)) & 1u)) steps -= kSub - spSubLast;
          }
        }
      }
      if (lane == 0) reinterpret_cast<int *>(smem + L::kOffList)[wq] = steps;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = misc[0];
  if constexpr (SPARSE) {
    const int *hdr = reinterpret_cast<const int *>(smem + L::kOffList);
    T = hdr[0] + hdr[1] + hdr[2] + hdr[3];
  }

  auto step_head = [&](int i) { return kvh * g + i / nq; };
  auto step_q0 = [&](int i) { return (q_first + i % nq) * BQ; };
  // Block-sparse: each role's cursor, moved once per step before (h, q0) are used.
  SparseSteps cur;
  if constexpr (SPARSE) cur.init(spbits, spW, g, p.nkb, kSub, spSubLast);

  if (warp == 13) {
    // ================================================================ loader
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar(L::kBarKV), 2 * L::kKTile);
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c) {
        tma_load_3d(sK + c * L::kKChunk, &tm_k, bar(L::kBarKV), c * 64, kv_c1, kv_c2);
        tma_load_3d(sV + c * L::kKChunk, &tm_v, bar(L::kBarKV), c * 64, kv_c1, kv_c2);
      }
    }
    int issued = 0;
    for (int i = 0; ok && i < T; ++i) {
      const int st = i % QS, use = i / QS;
      ok = warp_wait_bounded(bar(L::kBarQEmpty + st), (use & 1) ^ 1, abort_flag,
                             wait_site(3, L::kBarQEmpty + st, i));
      if (!ok) break;
      if constexpr (SPARSE) cur.next();
      const int h = SPARSE ? kvh * g + cur.hh : step_head(i), q0 = SPARSE ? cur.q0<BQ>() : step_q0(i);
      if (lane == 0) {
        int c1, c2;
        q_coords(h, q0, c1, c2);
        mbar_arrive_expect_tx(bar(L::kBarQFull + st), 2 * L::kQTile);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_3d(sQ + st * L::kQTile + c * L::kQChunk, &tm_q, bar(L::kBarQFull + st), c * 64, c1, c2);
          tma_load_3d(sDO + st * L::kQTile + c * L::kQChunk, &tm_do, bar(L::kBarQFull + st), c * 64, c1, c2);
        }
      }
      float *lse2 = vec + (st * 2) * BQ;
      float *dl = vec + (st * 2 + 1) * BQ;
      for (int c = lane; c < BQ; c += 32) {
        const int q = q0 + c;
        // Query rows past the sequence get LSE = +inf, so their probabilities are exactly 0
        // (and so are their dS and their dQ contributions).  A row that sees no key has
        // LSE = -inf but is never inside this block's band.
        const bool live = q < sg.Lq;
        lse2[c] = live ? p.lse[vec_row(h, q)] * 1.4426950408889634f : INFINITY;
        dl[c] = live ? p.delta[vec_row(h, q)] : 0.f;
      }
      // The stores above are ordered before lane 0's arrival by the warp barrier; the
      // barrier phase completes only when that arrival and the TMA bytes are both in.
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarQFull + st));
      ++issued;
    }
    if (lane == 0) {
      for (int i = issued > QS ? issued - QS : 0; i < issued; ++i)
        wait_drain(bar(L::kBarQFull + i % QS), (i / QS) & 1, 100000000ull);
      wait_drain(bar(L::kBarKV), 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 12) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_st = idesc_bf16_f32(128, BQ, 0, 0);   // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16_f32(128, DH, 0, 1);   // dV, dK (B = dO / Q, MN-major)
      constexpr uint32_t id_dq = idesc_bf16_f32(128, BQ, 1, 1);   // dQ^T = K^T dS^T
      // S^T (or dP^T) = A B^T over d: A = K (or V) [128 x D], B = Q_i (or dO_i) [BQ x D].
      auto issue_st = [&](uint32_t dst, uint32_t a0, uint32_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * L::kKChunk + (kk % 4) * 32;
          const uint32_t ob = (kk / 4) * L::kQChunk + (kk % 4) * 32;
          mma_ss(tmem + dst, sdesc_sw128(a0 + oa, 16, 1024), sdesc_sw128(b0 + ob, 16, 1024), id_st, kk > 0);
        }
      };
      bool ok = wait_bounded(bar(L::kBarKV), 0, abort_flag, wait_site(3, L::kBarKV, 0));
      if (ok && (!GENLIKE || T > 0)) ok = wait_bounded(bar(L::kBarQFull), 0, abort_flag, wait_site(3, L::kBarQFull, 0));
      if (ok && (!GENLIKE || T > 0)) {
        tc_fence_after_sync();
        issue_st(L::kTmS, sK, sQ);
        tc_commit(bar(L::kBarS));
        issue_st(L::kTmDP, sV, sDO);
        tc_commit(bar(L::kBarDP));
      }
      for (int i = 0; ok && i < T; ++i) {
        const int st = i % QS;
        const uint32_t q_t = sQ + st * L::kQTile, do_t = sDO + st * L::kQTile;
        // dV += P^T dO_i : M = 128 keys, N = DH, K = BQ queries; P^T (bf16) in TMEM.
        if (!(ok = wait_bounded(bar(L::kBarP), i & 1, abort_flag, wait_site(3, L::kBarP, i)))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_ts(tmem + L::kTmDV, tmem + L::kTmS + L::pcol(kk),
                 sdesc_sw128(do_t + (dcol0 / 64) * L::kQChunk + kk * 2048, L::kQChunk, 1024), id_kv,
                 (i > 0 || kk > 0));
        // Next step's S^T can start as soon as P^T has been consumed (issue order).
        if (i + 1 < T) {
          const int st1 = (i + 1) % QS;
          if (!(ok = wait_bounded(bar(L::kBarQFull + st1), ((i + 1) / QS) & 1, abort_flag,
                                  wait_site(3, L::kBarQFull + st1, i + 1))))
            break;
          tc_fence_after_sync();
          issue_st(L::kTmS, sK, sQ + st1 * L::kQTile);
          tc_commit(bar(L::kBarS));
        }
        // dK += dS^T Q_i : M = 128 keys, N = DH, K = BQ; dS^T K-major in shared memory.
        if (!(ok = wait_bounded(bar(L::kBarDS), i & 1, abort_flag, wait_site(3, L::kBarDS, i)))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_ss(tmem + L::kTmDK, sdesc_sw128(sDS + kk * 32, 16, 1024),
                 sdesc_sw128(q_t + (dcol0 / 64) * L::kQChunk + kk * 2048, L::kQChunk, 1024), id_kv,
                 (i > 0 || kk > 0));
        // dQ_i^T = K^T dS^T : M = 128 d columns, N = BQ, K = 128 keys; both MN-major.
        if (!(ok = wait_bounded(bar(L::kBarDQEmpty), (i & 1) ^ 1, abort_flag,
                                wait_site(3, L::kBarDQEmpty, i))))
          break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::kTmDQ, sdesc_sw128(sK + (dcol0 / 64) * L::kKChunk + kk * 2048, L::kKChunk, 1024),
                 sdesc_sw128(sDS + kk * 2048, 128 * 128, 1024), id_dq, kk > 0);
        tc_commit(bar(L::kBarDQ));
        tc_commit(bar(L::kBarDSEmpty));
        tc_commit(bar(L::kBarQEmpty + st));
        if (i + 1 < T) {
          issue_st(L::kTmDP, sV, sDO + ((i + 1) % QS) * L::kQTile);
          tc_commit(bar(L::kBarDP));
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
    const bool row_live = kv < sg.Lk;
    const float sl2 = p.sl2;
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
      const int st = i % QS;
      if constexpr (SPARSE) cur.next();
      const int q0 = (SPARSE ? cur.q0<BQ>() : step_q0(i)) + c0;  // first query column of this warpgroup
      if (!(ok = warp_wait_bounded(bar(L::kBarQFull + st), (i / QS) & 1, abort_flag,
                                   wait_site(3, L::kBarQFull + st, i))))
        break;
      if (!(ok = warp_wait_bounded(bar(L::kBarS), i & 1, abort_flag, wait_site(3, L::kBarS, i)))) break;
      tc_fence_after_sync();
      const float4 *lse4 = reinterpret_cast<const float4 *>(vec + (st * 2) * BQ + c0);
      const float4 *dl4 = reinterpret_cast<const float4 *>(vec + (st * 2 + 1) * BQ + c0);
      float pr[HC];
      {
        uint32_t rr[HC];
        if constexpr (HC == 32) tmem_ld_x32(tS, rr); else tmem_ld_x16(tS, rr);
#pragma unroll
        for (int c4 = 0; c4 < HC / 4; ++c4) {
          const float4 l = lse4[c4];
          pr[4 * c4 + 0] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 0]), sl2, -l.x));
          pr[4 * c4 + 1] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 1]), sl2, -l.y));
          pr[4 * c4 + 2] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 2]), sl2, -l.z));
          pr[4 * c4 + 3] = ex2_approx(fmaf(__uint_as_float(rr[4 * c4 + 3]), sl2, -l.w));
        }
      }
      // Masks: key rows past N, and queries q0 + c whose window misses this key
      // (visible iff c_lo <= c <= c_hi).  Query rows past N already have P = 0.
      if (!row_live) {
#pragma unroll
        for (int c = 0; c < HC; ++c) pr[c] = 0.f;
      } else if (GEN && (p.left >= 0 || p.right >= 0)) {
        const int c_lo = p.right < 0 ? INT_MIN : kv - p.right - sg.dlt - q0;
        const int c_hi = p.left < 0 ? INT_MAX : kv + p.left - sg.dlt - q0;
        if (c_lo > 0 || c_hi < HC - 1) {
#pragma unroll
          for (int c = 0; c < HC; ++c)
            if (c < c_lo || c > c_hi) pr[c] = 0.f;
        }
      } else if ((MODE == kAttnCausal || (SPARSE && p.right == 0)) && q0 < kv) {
#pragma unroll
        for (int c = 0; c < HC; ++c)
          if (q0 + c < kv) pr[c] = 0.f;
      }
      // Dropout: bit c of `keep` is set when (query q0 + c, this key) is kept.  One Philox
      // call gives the mask values of eight consecutive keys for one query; the eight
      // lanes of a key group each call it for a different query and swap values in eight
      // shuffles.
      uint32_t keep = 0xFFFFFFFFu;
      if constexpr (DROP) {
        keep = 0u;
        const int m = lane & 7;  // == kv & 7
        const uint32_t bh = static_cast<uint32_t>(b * p.Hq + (SPARSE ? kvh * g + cur.hh : step_head(i)));
#pragma unroll
        for (int t = 0; t < HC / 8; ++t) {
          uint32_t w[4];
          philox4x32_10(static_cast<uint32_t>(kv) >> 3, static_cast<uint32_t>(q0 + 8 * t + m), bh, 0u, p.drop.k0,
                        p.drop.k1, w);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int si = (m + kk) & 7;  // value this lane sends: the key of lane (m + kk) & 7
            const uint32_t sw = (si >> 1) == 0 ? w[0] : (si >> 1) == 1 ? w[1] : (si >> 1) == 2 ? w[2] : w[3];
            const uint32_t sv = (si & 1) ? (sw >> 16) : (sw & 0xFFFFu);
            const int from = (m - kk) & 7;  // that lane drew for query q0 + 8t + from
            const uint32_t rv = __shfl_sync(0xffffffffu, sv, (lane & ~7) | from);
            keep |= (rv >= p.drop.thr ? 1u : 0u) << (8 * t + from);
          }
        }
      }
      {
        // P^T as the A operand of dV += P^T dO: dropped entries are 0 (the 1 / (1 - p)
        // factor is applied to dV in the epilogue).
        uint32_t pk[HC / 2];
#pragma unroll
        for (int c = 0; c < HC / 2; ++c)
          pk[c] = pack_bf16x2(((keep >> (2 * c)) & 1u) ? pr[2 * c] : 0.f, ((keep >> (2 * c + 1)) & 1u) ? pr[2 * c + 1] : 0.f);
        if constexpr (HC == 32) tmem_st_x16(tS, pk); else tmem_st_x8(tS, pk);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarP));

      if (!(ok = warp_wait_bounded(bar(L::kBarDP), i & 1, abort_flag, wait_site(3, L::kBarDP, i)))) break;
      tc_fence_after_sync();
      uint32_t dsk[HC / 2];
      {
        uint32_t rr[HC];
        if constexpr (HC == 32) tmem_ld_x32(tDP, rr); else tmem_ld_x16(tDP, rr);
        if constexpr (DROP) {
          // dS = P (Z dP / (1 - p) - Delta) with the dropout mask Z.
#pragma unroll
          for (int c = 0; c < HC; ++c)
            rr[c] = __float_as_uint(((keep >> c) & 1u) ? __uint_as_float(rr[c]) * p.drop.inv_keep : 0.f);
        }
#pragma unroll
        for (int c4 = 0; c4 < HC / 4; ++c4) {
          const float4 dd = dl4[c4];
          dsk[2 * c4] = pack_bf16x2(pr[4 * c4 + 0] * (__uint_as_float(rr[4 * c4 + 0]) - dd.x),
                                    pr[4 * c4 + 1] * (__uint_as_float(rr[4 * c4 + 1]) - dd.y));
          dsk[2 * c4 + 1] = pack_bf16x2(pr[4 * c4 + 2] * (__uint_as_float(rr[4 * c4 + 2]) - dd.z),
                                        pr[4 * c4 + 3] * (__uint_as_float(rr[4 * c4 + 3]) - dd.w));
        }
      }
      // dS^T row r, this warpgroup's 16-byte units -> shared memory (128-byte swizzled row).
      if (!(ok = warp_wait_bounded(bar(L::kBarDSEmpty), (i & 1) ^ 1, abort_flag,
                                   wait_site(3, L::kBarDSEmpty, i))))
        break;
      const uint32_t rowp = sDS + r * 128;
#pragma unroll
      for (int uu = 0; uu < HC / 8; ++uu) {
        const int unit = c0 / 8 + uu;
        st_shared_v4(rowp + ((unit ^ (r & 7)) * 16), dsk[4 * uu], dsk[4 * uu + 1], dsk[4 * uu + 2],
                     dsk[4 * uu + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarDS));
    }

    // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK, as bf16 into the
    // V / K tiles' shared memory (no longer read), then one thread TMA-stores both.
    bool okw = ok && warp_wait_bounded(bar(L::kBarFinal), 0, abort_flag, wait_site(3, L::kBarFinal, 0));
    okw = named_bar_and(1, 256, okw && *abort_flag == 0);
    if (okw) {
      tc_fence_after_sync();
      const uint32_t tacc = tmem + (wg ? L::kTmDK : L::kTmDV) + lane_off;
      const float mul = wg ? p.scale : (DROP ? p.drop.inv_keep : 1.f);
      const uint32_t stage = wg ? sK : sV;
      // A packed key block that ends past its sequence stores its rows directly.
      const bool direct = packed && kv0 + 128 > sg.Lk;
      __nv_bfloat16 *drow = packed ? (wg ? p.dk : p.dv) + (static_cast<size_t>(sg.k_base + kv) * p.Hkv + kvh) * D + dcol0
                                   : nullptr;
#pragma unroll
      for (int cc = 0; cc < DH / 32; ++cc) {
        uint32_t o[32];
        if (!GENLIKE || T > 0) {
          tmem_ld_x32(tacc + cc * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;  // no query sees this block
        }
        const uint32_t rowbase = stage + (cc / 2) * L::kKChunk + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = (cc % 2) * 4 + uu;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[8 * uu + 2 * e]) * mul,
                               __uint_as_float(o[8 * uu + 2 * e + 1]) * mul);
          if (!direct)
            st_shared_v4(rowbase + ((unit ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
          else if (row_live)
            *reinterpret_cast<uint4 *>(drow + cc * 32 + uu * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (!direct) {
        fence_proxy_async_smem();
        named_bar_sync(1, 256);
        if (threadIdx.x == 0) {
#pragma unroll
          for (int c = 0; c < DH / 64; ++c) {
            tma_store_3d(&tm_dv, sV + c * L::kKChunk, dcol0 + c * 64, kv_c1, kv_c2);
            tma_store_3d(&tm_dk, sK + c * L::kKChunk, dcol0 + c * 64, kv_c1, kv_c2);
          }
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      }
    }
  } else {
    // ================================================================ dQ^T drain (warps 8-11)
    const int wq = warp - 8;
    const int dl = wq * 32 + lane;  // d column (TMEM lane) within this CTA's half
    const uint32_t tDQ = tmem + L::kTmDQ + (static_cast<uint32_t>(wq * 32) << 16);
    const bool lane_live = dl < DH;  // d = 64 pads M to 128; upper lanes are junk
    float *stage = reinterpret_cast<float *>(smem + L::kOffDQ);
    const int tid = threadIdx.x - 256;
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
      // The warpgroup leaves the loop together: the named barriers below need all four warps.
      ok = warp_wait_bounded(bar(L::kBarDQ), i & 1, abort_flag, wait_site(3, L::kBarDQ, i));
      if (!(ok = named_bar_and(2, 128, ok))) break;
      tc_fence_after_sync();
      float acc[BQ];
      if (wq * 32 < DH) {
#pragma unroll
        for (int c0 = 0; c0 < BQ; c0 += 32) {
          uint32_t rr[32];
          tmem_ld_x32(tDQ + c0, rr);
#pragma unroll
          for (int c = 0; c < 32; ++c) acc[c0 + c] = __uint_as_float(rr[c]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarDQEmpty));
      if constexpr (SPARSE) cur.next();
      const int h = SPARSE ? kvh * g + cur.hh : step_head(i), q0 = SPARSE ? cur.q0<BQ>() : step_q0(i);
#pragma unroll
      for (int hp = 0; hp < L::kDQHalves; ++hp) {
        // The previous reduce must have finished reading the staging buffer.
        if (tid == 0) bulk_wait_group_read0();
        named_bar_sync(2, 128);
        const int cl = dl - hp * L::kDQCols;  // column within this pass
        if (lane_live && cl >= 0 && cl < L::kDQCols) {
#pragma unroll
          for (int c = 0; c < BQ; ++c) stage[c * L::kDQCols + cl] = acc[c];
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (tid == 0) {
          int c1, c2;
          q_coords(h, q0, c1, c2);
          tma_reduce_add_3d(&tm_dqacc, sDQ, dcol0 + hp * L::kDQCols, c1, c2);
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
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ============================================================================ host side

inline size_t pad256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline size_t bwd_workspace_bytes(int B, int Hq, int N, int d) {
  const size_t rows = static_cast<size_t>(B) * Hq * N;
  return pad256(rows * 4) + pad256(rows * static_cast<size_t>(d) * 4);
}

typedef CUresult (*EncodeTiledFnBwd)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline bool bwd_map(EncodeTiledFnBwd enc, CUtensorMap *m, const void *ptr, bool f32, int d, int N,
                    long long heads, int box_cols, int box_rows) {
  const cuuint64_t esz = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esz,
                                 static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same over packed rows [total][H][d]: a box is box_rows consecutive rows of one head.
inline bool bwd_map_packed(EncodeTiledFnBwd enc, CUtensorMap *m, const void *ptr, bool f32, int d, int H,
                           int total, int box_cols, int box_rows) {
  const cuuint64_t esz = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total > 0 ? total : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esz,
                                 static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed variable-length sequences ([total, H, d] rows, [B + 1] offsets on the device).
struct PackedSeqs {
  const int *cu_q, *cu_k;
  int total_q, total_k, max_q, max_k;
};

template <int D, int DH, int BQ, int MODE, bool DROP = false>
inline void bwd_launch_main(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const CUtensorMap &tdo, const CUtensorMap &tdk, const CUtensorMap &tdv,
                            const CUtensorMap &tdq, const BwdParams &p, unsigned grid, cudaStream_t s) {
  using L = BwdLayout<D, DH, BQ>;
  fa_bwd_main_kernel<D, DH, BQ, MODE, DROP>
      <<<grid, kBwdThreads, MODE == kAttnSparse ? L::kSmemBytesSparse : L::kSmemBytes, s>>>(tq, tk, tv, tdo, tdk,
                                                                                           tdv, tdq, p);
}

typedef int (*TimerStartFn)(int, cudaStream_t);
typedef void (*TimerStopFn)(int, int, cudaStream_t);

// Unit order of a backward launch: tiers of key-block levels (1: head-major) and the
// number of (b, kv head) rows taken level by level at the end of the grid.
struct BwdOrder {
  int tiers, tail;
};

// Dense d = 256 backward main kernel as a two-CTA cluster (fa_bwd_pair.cuh).
template <int MODE>
bool bwd_launch_pair(EncodeTiledFnBwd enc, const void *q, const void *k, const void *v, const void *dout, void *dk,
                     void *dv, float *dqacc, int B, int Hq, int Hkv, int N, const BwdParams &p, cudaStream_t s);

// Dense d = 128 backward main kernel with 128-query steps (fa_bwd_q128.cuh), taken from
// this sequence length on.
constexpr int kQ128MinN = 4096;
template <int MODE>
bool bwd_launch_q128(EncodeTiledFnBwd enc, const void *q, const void *k, const void *v, const void *dout, void *dk,
                     void *dv, float *dqacc, int B, int Hq, int Hkv, int N, const BwdParams &p, cudaStream_t s);

template <int D, int DH, int BQ>
inline int bwd_launch_d(const void *q, const void *k, const void *v, const void *o, const float *lse,
                        const void *dout, void *dq, void *dk, void *dv, void *workspace, int B, int Hq,
                        int Hkv, int N, int left, int right, float scale, cudaStream_t s, EncodeTiledFnBwd enc,
                        TimerStartFn tstart, TimerStopFn tstop, const PackedSeqs *pk, const DropCfg *drop,
                        const uint8_t *bmask, BwdOrder order) {
  const long long rows = pk ? static_cast<long long>(pk->total_q) * Hq : static_cast<long long>(B) * Hq * N;
  float *delta = static_cast<float *>(workspace);
  float *dqacc = reinterpret_cast<float *>(static_cast<char *>(workspace) + pad256(static_cast<size_t>(rows) * 4));
  using L = BwdLayout<D, DH, BQ>;
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  if (pk) {
    if (!bwd_map_packed(enc, &tq, q, false, D, Hq, pk->total_q, 64, BQ) ||
        !bwd_map_packed(enc, &tdo, dout, false, D, Hq, pk->total_q, 64, BQ) ||
        !bwd_map_packed(enc, &tk, k, false, D, Hkv, pk->total_k, 64, 128) ||
        !bwd_map_packed(enc, &tv, v, false, D, Hkv, pk->total_k, 64, 128) ||
        !bwd_map_packed(enc, &tdk, dk, false, D, Hkv, pk->total_k, 64, 128) ||
        !bwd_map_packed(enc, &tdv, dv, false, D, Hkv, pk->total_k, 64, 128) ||
        !bwd_map_packed(enc, &tdq, dqacc, true, D, Hq, pk->total_q, L::kDQCols, BQ))
      return FA_ERR_CUDA;
  } else {
    const long long hq = static_cast<long long>(B) * Hq, hkv = static_cast<long long>(B) * Hkv;
    if (!bwd_map(enc, &tq, q, false, D, N, hq, 64, BQ) || !bwd_map(enc, &tdo, dout, false, D, N, hq, 64, BQ) ||
        !bwd_map(enc, &tk, k, false, D, N, hkv, 64, 128) || !bwd_map(enc, &tv, v, false, D, N, hkv, 64, 128) ||
        !bwd_map(enc, &tdk, dk, false, D, N, hkv, 64, 128) || !bwd_map(enc, &tdv, dv, false, D, N, hkv, 64, 128) ||
        !bwd_map(enc, &tdq, dqacc, true, D, N, hq, L::kDQCols, BQ))
      return FA_ERR_CUDA;
  }

  fa_bwd_pre_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
      static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), delta, dqacc, rows);

  BwdParams p;
  p.lse = lse;
  p.delta = delta;
  p.dk = static_cast<__nv_bfloat16 *>(dk);
  p.dv = static_cast<__nv_bfloat16 *>(dv);
  p.cu_q = pk ? pk->cu_q : nullptr;
  p.cu_k = pk ? pk->cu_k : nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = pk ? 0 : N;
  p.total_q = pk ? pk->total_q : 0;
  p.total_k = pk ? pk->total_k : 0;
  p.nkb = pk ? (pk->max_k + 127) / 128 : (N + 127) / 128;
  p.left = left;
  p.right = right;
  p.scale = scale;
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.drop = drop ? *drop : DropCfg{};
  p.bmask = bmask;
  // Unit order (unit_order): `order.tiers` tiers of key-block levels (1: head-major), the
  // last `order.tail` (b, kv head) rows level by level.
  const int tiers = order.tiers < 1 ? 1 : order.tiers;
  p.tsz = (p.nkb + tiers - 1) / tiers;
  const int heads = B * Hkv;
  p.tail = order.tail < 0 ? 0 : (order.tail < heads ? order.tail : heads - 1);
  const unsigned grid = static_cast<unsigned>(B) * Hkv * p.nkb * (D / DH);
  const int tslot = tstart(1, s);
  // Dense full and causal attention run as CTA pairs that split the work by role at
  // d = 256, and with 128-query steps at d = 128 from N = 4096 on.  Below that a CTA has
  // too few steps to repay the longer pipeline start of 128-query steps (measured on B200:
  // 128-query steps +4% at N = 8192, +2% at N = 4096, -5% at N = 2048).
  const bool dense = !pk && !drop && !bmask && left < 0 && right <= 0;
  if (dense && (D == 256 || (D == 128 && N >= kQ128MinN)) && grid > 0) {
    bool launched;
    if (D == 256)
      launched = right == 0 ? bwd_launch_pair<kAttnCausal>(enc, q, k, v, dout, dk, dv, dqacc, B, Hq, Hkv, N, p, s)
                            : bwd_launch_pair<kAttnFull>(enc, q, k, v, dout, dk, dv, dqacc, B, Hq, Hkv, N, p, s);
    else
      launched = right == 0 ? bwd_launch_q128<kAttnCausal>(enc, q, k, v, dout, dk, dv, dqacc, B, Hq, Hkv, N, p, s)
                            : bwd_launch_q128<kAttnFull>(enc, q, k, v, dout, dk, dv, dqacc, B, Hq, Hkv, N, p, s);
    if (!launched) {
      tstop(1, tslot, s);
      return FA_ERR_CUDA;
    }
  } else if (grid > 0) {
    // Dense full and causal attention have their own variants; packed sequences and other
    // bands take the general one.
    if (bmask)  // block-sparse: dense layout, causal or not (right = 0 or -1)
      bwd_launch_main<D, DH, BQ, kAttnSparse>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
    else if (drop && right == 0)  // dropout: dense attention only (the host checks)
      bwd_launch_main<D, DH, BQ, kAttnCausal, true>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
    else if (drop)
      bwd_launch_main<D, DH, BQ, kAttnFull, true>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
    else if (pk || (left >= 0 || (right >= 0 && right != 0)))
      bwd_launch_main<D, DH, BQ, kAttnGeneral>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
    else if (right == 0)
      bwd_launch_main<D, DH, BQ, kAttnCausal>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
    else
      bwd_launch_main<D, DH, BQ, kAttnFull>(tq, tk, tv, tdo, tdk, tdv, tdq, p, grid, s);
  }
  tstop(1, tslot, s);

  const long long n8 = rows * D / 8;
  fa_bwd_post_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, s>>>(
      dqacc, static_cast<__nv_bfloat16 *>(dq), scale, n8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <typename Enc>
inline int bwd_launch(const void *q, const void *k, const void *v, const void *o, const float *lse,
                      const void *dout, void *dq, void *dk, void *dv, void *workspace, int B, int Hq,
                      int Hkv, int N, int d, int left, int right, float scale, cudaStream_t s, Enc enc,
                      TimerStartFn tstart, TimerStopFn tstop, const PackedSeqs *pk = nullptr,
                      const DropCfg *drop = nullptr, const uint8_t *bmask = nullptr, BwdOrder order = {1, 0}) {
  const EncodeTiledFnBwd e = reinterpret_cast<EncodeTiledFnBwd>(enc);
  if (d == 64)
    return bwd_launch_d<64, 64, 64>(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, left, right,
                                    scale, s, e, tstart, tstop, pk, drop, bmask, order);
  if (d == 128)
    return bwd_launch_d<128, 128, 64>(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, left, right,
                                      scale, s, e, tstart, tstop, pk, drop, bmask, order);
  return bwd_launch_d<256, 128, 32>(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, left, right,
                                    scale, s, e, tstart, tstop, pk, drop, bmask, order);
}

}  // namespace fa
