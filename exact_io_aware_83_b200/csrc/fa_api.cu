// fa_api.cu - host side of libfa_sm100.so: argument checks, TMA tensor maps, launches.
//
// The C entry points are declared (with their contracts) in include/fa.h.  This file is
// the only translation unit of the library; the kernels are included from the .cuh
// files beside it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "fa.h"
#include "fa_common.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_d256.cuh"
#include "fa_fwd_persist.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd_pair.cuh"
#include "fa_bwd_q128.cuh"
#include "fa_decode.cuh"

namespace {

using fa::FwdParams;

constexpr int kMaxDevices = 64;

// FA_DEBUG=1 in the environment prints the CUDA call that made an entry point return
// FA_ERR_CUDA (to stderr).
bool debug_enabled() {
  static const bool on = [] {
    const char *e = std::getenv("FA_DEBUG");
    return e && e[0] == '1';
  }();
  return on;
}

bool cuda_ok(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return true;
  if (debug_enabled()) std::fprintf(stderr, "[fa] %s: %s\n", what, cudaGetErrorString(e));
  return false;
}

// cuTensorMapEncodeTiled, fetched once through the runtime so the library does not link
// the driver library directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cuda_ok(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q),
                "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)") &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device capability check (sm_100) and one-time kernel attribute setup.
struct DeviceState {
  std::once_flag once;
  bool ok = false;
  int sms = 148;  // multiprocessors: the persistent kernels launch one CTA per SM
};
DeviceState g_dev[kMaxDevices];

// A kernel that rebalances registers with setmaxnreg must have been compiled for the
// launch register count its split assumes; otherwise setmaxnreg.inc could never be
// satisfied.  Refuse to use such a kernel rather than launch it.
template <typename K>
bool regs_at_least(K kernel, int regs) {
  cudaFuncAttributes attr;
  if (!cuda_ok(cudaFuncGetAttributes(&attr, kernel), "cudaFuncGetAttributes")) return false;
  if (attr.numRegs >= regs) return true;
  if (debug_enabled())
    std::fprintf(stderr, "[fa] kernel compiled for %d registers per thread, split needs %d\n", attr.numRegs, regs);
  return false;
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  const bool ok = cuda_ok(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                          "cudaFuncSetAttribute(max dynamic shared memory)");
  if (!ok && debug_enabled()) std::fprintf(stderr, "[fa]   requested %d bytes\n", bytes);
  return ok;
}

int current_sms() {
  int dev = 0;
  return (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) ? g_dev[dev].sms : 148;
}

bool device_ready() {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice") || dev < 0 || dev >= kMaxDevices) return false;
  DeviceState &st = g_dev[dev];
  std::call_once(st.once, [&] {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return;
    if (major != 10 || minor != 0) {  // sm_100a code only
      if (debug_enabled()) std::fprintf(stderr, "[fa] device is sm_%d%d, not sm_100\n", major, minor);
      return;
    }
    bool ok = encode_fn() != nullptr;
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnFull>, fa::FwdLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnCausal>, fa::FwdLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnGeneral>, fa::FwdLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnFull>, fa::FwdLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnCausal>, fa::FwdLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnGeneral>, fa::FwdLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnSparse>, fa::FwdLayout<64>::kSmemBytesSparse);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnSparse>, fa::FwdLayout<128>::kSmemBytesSparse);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnSparse>, fa::FwdD256Layout::kSmemBytesSparse);
    ok = ok && set_smem(fa::fa_bwd_main_kernel<64, 64, 64, fa::kAttnSparse>,
                        fa::BwdLayout<64, 64, 64>::kSmemBytesSparse);
    ok = ok && set_smem(fa::fa_bwd_main_kernel<128, 128, 64, fa::kAttnSparse>,
                        fa::BwdLayout<128, 128, 64>::kSmemBytesSparse);
    ok = ok && set_smem(fa::fa_bwd_main_kernel<256, 128, 32, fa::kAttnSparse>,
                        fa::BwdLayout<256, 128, 32>::kSmemBytesSparse);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<64, fa::kAttnFull>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<64, fa::kAttnCausal>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<64, fa::kAttnGeneral>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<128, fa::kAttnFull>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<128, fa::kAttnCausal>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<128, fa::kAttnGeneral>, fa::kFwdRegsLaunch);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnFull, true>, fa::FwdLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<64, fa::kAttnCausal, true>, fa::FwdLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnFull, true>, fa::FwdLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_kernel<128, fa::kAttnCausal, true>, fa::FwdLayout<128>::kSmemBytes);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<64, fa::kAttnFull, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<64, fa::kAttnCausal, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<128, fa::kAttnFull, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_kernel<128, fa::kAttnCausal, true>, fa::kFwdRegsLaunch);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnFull, true>, fa::FwdD256Layout::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnCausal, true>, fa::FwdD256Layout::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnFull>, fa::FwdD256Layout::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnCausal>, fa::FwdD256Layout::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_d256_kernel<fa::kAttnGeneral>, fa::FwdD256Layout::kSmemBytes);
    using fa::BwdLayout;
    using fa::fa_bwd_main_kernel;
    ok = ok && set_smem(fa_bwd_main_kernel<64, 64, 64, fa::kAttnFull>, BwdLayout<64, 64, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<64, 64, 64, fa::kAttnCausal>, BwdLayout<64, 64, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<64, 64, 64, fa::kAttnGeneral>, BwdLayout<64, 64, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<128, 128, 64, fa::kAttnFull>, BwdLayout<128, 128, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<128, 128, 64, fa::kAttnCausal>, BwdLayout<128, 128, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<128, 128, 64, fa::kAttnGeneral>, BwdLayout<128, 128, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<256, 128, 32, fa::kAttnFull>, BwdLayout<256, 128, 32>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<256, 128, 32, fa::kAttnCausal>, BwdLayout<256, 128, 32>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<256, 128, 32, fa::kAttnGeneral>, BwdLayout<256, 128, 32>::kSmemBytes);
    ok = ok && set_smem(fa::fa_bwd_pair_kernel<fa::kAttnFull>, fa::PairLayout::kSmemBytes);
    ok = ok && set_smem(fa::fa_bwd_pair_kernel<fa::kAttnCausal>, fa::PairLayout::kSmemBytes);
    ok = ok && set_smem(fa::fa_bwd_q128_kernel<fa::kAttnFull>, fa::Q128Layout::kSmemBytes);
    ok = ok && set_smem(fa::fa_bwd_q128_kernel<fa::kAttnCausal>, fa::Q128Layout::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<64, 64, 64, fa::kAttnFull, true>, BwdLayout<64, 64, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<64, 64, 64, fa::kAttnCausal, true>, BwdLayout<64, 64, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<128, 128, 64, fa::kAttnFull, true>, BwdLayout<128, 128, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<128, 128, 64, fa::kAttnCausal, true>, BwdLayout<128, 128, 64>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<256, 128, 32, fa::kAttnFull, true>, BwdLayout<256, 128, 32>::kSmemBytes);
    ok = ok && set_smem(fa_bwd_main_kernel<256, 128, 32, fa::kAttnCausal, true>, BwdLayout<256, 128, 32>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<64, 16>, fa::DecodeLayout<64, 16>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<64, 32>, fa::DecodeLayout<64, 32>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<64, 64>, fa::DecodeLayout<64, 64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<64, 128>, fa::DecodeLayout<64, 128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<128, 16>, fa::DecodeLayout<128, 16>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<128, 32>, fa::DecodeLayout<128, 32>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<128, 64>, fa::DecodeLayout<128, 64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<128, 128>, fa::DecodeLayout<128, 128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<256, 16>, fa::DecodeLayout<256, 16>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<256, 32>, fa::DecodeLayout<256, 32>::kSmemBytes);
    ok = ok && set_smem(fa::fa_decode_kernel<256, 64>, fa::DecodeLayout<256, 64>::kSmemBytes);
    using fa::FwdPLayout;
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<64, fa::kAttnFull>, FwdPLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<64, fa::kAttnCausal>, FwdPLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<128, fa::kAttnFull>, FwdPLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<128, fa::kAttnCausal>, FwdPLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<64, fa::kAttnFull, true>, FwdPLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<64, fa::kAttnCausal, true>, FwdPLayout<64>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<128, fa::kAttnFull, true>, FwdPLayout<128>::kSmemBytes);
    ok = ok && set_smem(fa::fa_fwd_persist_kernel<128, fa::kAttnCausal, true>, FwdPLayout<128>::kSmemBytes);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<64, fa::kAttnFull>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<64, fa::kAttnCausal>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<128, fa::kAttnFull>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<128, fa::kAttnCausal>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<64, fa::kAttnFull, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<64, fa::kAttnCausal, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<128, fa::kAttnFull, true>, fa::kFwdRegsLaunch);
    ok = ok && regs_at_least(fa::fa_fwd_persist_kernel<128, fa::kAttnCausal, true>, fa::kFwdRegsLaunch);
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0) st.sms = sms;
    if (!ok && debug_enabled()) std::fprintf(stderr, "[fa] device setup failed\n");
    st.ok = ok;
  });
  return st.ok;
}

// 3-D bf16 tensor map over [heads][N][d] with [rows x 64] boxes and 128-byte swizzle.
bool make_map_bf16(CUtensorMap *m, const void *ptr, int d, int N, long long heads, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over packed rows [total][H][d] (a tile = box_rows consecutive
// rows of one head: box {64, 1, box_rows}), 128-byte swizzle.  The shared-memory image of
// a box is the same [box_rows x 64] tile as that of make_map_bf16.
bool make_map_packed(CUtensorMap *m, const void *ptr, int d, int H, int total, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total > 0 ? total : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- optional event pairs around the main kernels (fa_kernel_timing)
constexpr int kMaxTimed = 4096;
struct KernelTimer {
  cudaEvent_t ev[3][kMaxTimed][2] = {};
  int count[3] = {0, 0, 0};
  bool enabled = false;
};
KernelTimer g_timer;

cudaEvent_t timer_event(int which, int i, int edge) {
  cudaEvent_t &e = g_timer.ev[which][i][edge];
  if (!e && cudaEventCreate(&e) != cudaSuccess) e = nullptr;
  return e;
}

// Returns the slot index to close with timer_stop, or -1 when not recording.
int timer_start(int which, cudaStream_t s) {
  if (!g_timer.enabled || g_timer.count[which] >= kMaxTimed) return -1;
  const int i = g_timer.count[which];
  cudaEvent_t a = timer_event(which, i, 0), b = timer_event(which, i, 1);
  if (!a || !b || cudaEventRecord(a, s) != cudaSuccess) return -1;
  return i;
}

void timer_stop(int which, int slot, cudaStream_t s) {
  if (slot < 0) return;
  if (cudaEventRecord(g_timer.ev[which][slot][1], s) == cudaSuccess) g_timer.count[which] = slot + 1;
}

int check_sizes(int B, int Hq, int Hkv, int N, int d, float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_GQA;
  // Row indices (b*H + h)*N + i must fit in int32 for the kernels' index arithmetic, and
  // the grid size in int32.
  // N <= 2^30 keeps window arithmetic (row +- window, both below N) inside int32.
  const long long rows = static_cast<long long>(B) * Hq * N;
  if (N > (1 << 30) || rows >= (1ll << 31) ||
      static_cast<long long>(B) * Hq * ((N + 127) / 128) >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Window bound as the kernels take it: -1 (unlimited) or a value below N - 1.  A bound
// of N - 1 or more hides nothing and is unlimited too.  Bounds below -1 are rejected.
bool normalise_window(int w, int N, int *out) {
  if (w < -1) return false;
  *out = (w < 0 || w >= N - 1) ? -1 : w;
  return true;
}

// ---- static scratch for fa_bwd_noalloc (callers that cannot allocate device memory)
//
// One buffer per GPU that loads the library, alive until the process exits.  Host code
// must not use `g_noalloc_scratch` itself as a device address (on the host it names a
// shadow variable); the address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

struct NoallocState {
  std::mutex mu;
  void *ptr = nullptr;  // set only once a lookup has succeeded
};
NoallocState g_noalloc[kMaxDevices];

// Device address of the static scratch on the current device (nullptr on failure).
// Looked up on the first fa_bwd_noalloc call made with the device current; a failed
// lookup (for instance one attempted inside a stream capture) is not remembered, so a
// later call retries it, and its error is cleared from the runtime so that it cannot
// surface as the status of a later, unrelated launch.
void *noalloc_scratch() {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice") || dev < 0 || dev >= kMaxDevices) return nullptr;
  NoallocState &st = g_noalloc[dev];
  std::lock_guard<std::mutex> lock(st.mu);
  if (!st.ptr) {
    void *p = nullptr;
    if (cuda_ok(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(no-alloc scratch)"))
      st.ptr = p;
    else
      (void)cudaGetLastError();
  }
  return st.ptr;
}

// ---- decode (a few new query rows against a long cache) and the merge of partials

constexpr int kMaxDecodeSplits = 1024;

// Query rows handled by one decode CTA, padded to the MMA width the kernel is built for.
int decode_rows_padded(int R) { return R <= 16 ? 16 : R <= 32 ? 32 : R <= 64 ? 64 : 128; }

int check_decode_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_GQA;
  const long long R = static_cast<long long>(Hq / Hkv) * Nq;
  if (R > (d == 256 ? 64 : 128)) return FA_ERR_UNSUPPORTED;
  if (Nk > (1 << 30) || static_cast<long long>(B) * Hq * Nq >= (1ll << 31) ||
      static_cast<long long>(B) * Hkv * Nk >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t decode_workspace(int B, int Hq, int Nq, int d, int splits) {
  if (splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(B) * Hq * Nq;
  return fa::pad256(static_cast<size_t>(splits) * rows * d * 4) + fa::pad256(static_cast<size_t>(splits) * rows * 4);
}

template <int D, int RP>
void launch_decode(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                   const fa::DecodeParams &p, unsigned grid, cudaStream_t s) {
  fa::fa_decode_kernel<D, RP><<<grid, fa::kDecodeThreads, fa::DecodeLayout<D, RP>::kSmemBytes, s>>>(tq, tk, tv, p);
}

template <int D>
void launch_decode_d(int RP, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const fa::DecodeParams &p, unsigned grid, cudaStream_t s) {
  if (RP == 16) launch_decode<D, 16>(tq, tk, tv, p, grid, s);
  else if (RP == 32) launch_decode<D, 32>(tq, tk, tv, p, grid, s);
  else if (RP == 64) launch_decode<D, 64>(tq, tk, tv, p, grid, s);
  else if constexpr (D != 256) launch_decode<D, 128>(tq, tk, tv, p, grid, s);
}

void launch_merge(const float *o_part, const float *lse_part, void *o, float *lse, int S, long long rows,
                  int d, cudaStream_t s) {
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
  if (d == 64) fa::fa_merge_kernel<64><<<grid, 256, 0, s>>>(o_part, lse_part, ob, lse, S, rows);
  else if (d == 128) fa::fa_merge_kernel<128><<<grid, 256, 0, s>>>(o_part, lse_part, ob, lse, S, rows);
  else fa::fa_merge_kernel<256><<<grid, 256, 0, s>>>(o_part, lse_part, ob, lse, S, rows);
}

// Launches the forward kernel for d (maps and parameters prepared by the caller).
template <int D, int MODE, bool DROP>
void launch_fwd_d(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &to,
                  const FwdParams &p, unsigned units, cudaStream_t s) {
  constexpr bool sparse = MODE == fa::kAttnSparse;
  if constexpr (D == 256)
    fa::fa_fwd_d256_kernel<MODE, DROP><<<units, fa::kFwdD256Threads,
                                         sparse ? fa::FwdD256Layout::kSmemBytesSparse : fa::FwdD256Layout::kSmemBytes,
                                         s>>>(tq, tk, tv, to, p);
  else
    fa::fa_fwd_kernel<D, MODE, DROP><<<units, fa::kFwdThreads,
                                       sparse ? fa::FwdLayout<D>::kSmemBytesSparse : fa::FwdLayout<D>::kSmemBytes,
                                       s>>>(tq, tk, tv, to, p);
}

// Forward scheduler for dense full and causal attention (d = 64, 128): the persistent
// kernel (one CTA per SM walking the units) or one CTA per unit.  fa_set_fwd_scheduler.
std::atomic<int> g_fwd_persistent{[] {
  const char *e = std::getenv("FA_FWD_PERSISTENT");  // "0": start with one CTA per unit
  return (e && e[0] == '0') ? 0 : 1;
}()};
std::atomic<unsigned> g_unit_slot{0};

template <int D, int MODE, bool DROP>
void launch_fwd_persist(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &to,
                        const FwdParams &p, unsigned units, cudaStream_t s) {
  const unsigned sms = static_cast<unsigned>(current_sms());
  const unsigned grid = units < sms ? units : sms;
  const int slot = static_cast<int>(g_unit_slot.fetch_add(1u) % fa::kUnitSlots);
  fa::fa_fwd_persist_kernel<D, MODE, DROP><<<grid, fa::kFwdThreads, fa::FwdPLayout<D>::kSmemBytes, s>>>(
      tq, tk, tv, to, p, static_cast<int>(units), slot);
}

template <int D>
void launch_fwd_mode(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &to,
                     const FwdParams &p, unsigned units, int mode, bool drop, cudaStream_t s) {
  if constexpr (D != 256) {
    if (g_fwd_persistent.load() && (mode == fa::kAttnFull || mode == fa::kAttnCausal)) {
      if (drop && mode == fa::kAttnCausal) launch_fwd_persist<D, fa::kAttnCausal, true>(tq, tk, tv, to, p, units, s);
      else if (drop) launch_fwd_persist<D, fa::kAttnFull, true>(tq, tk, tv, to, p, units, s);
      else if (mode == fa::kAttnCausal) launch_fwd_persist<D, fa::kAttnCausal, false>(tq, tk, tv, to, p, units, s);
      else launch_fwd_persist<D, fa::kAttnFull, false>(tq, tk, tv, to, p, units, s);
      return;
    }
  }
  if (drop && mode == fa::kAttnCausal) launch_fwd_d<D, fa::kAttnCausal, true>(tq, tk, tv, to, p, units, s);
  else if (drop) launch_fwd_d<D, fa::kAttnFull, true>(tq, tk, tv, to, p, units, s);
  else if (mode == fa::kAttnGeneral) launch_fwd_d<D, fa::kAttnGeneral, false>(tq, tk, tv, to, p, units, s);
  else if (mode == fa::kAttnSparse) launch_fwd_d<D, fa::kAttnSparse, false>(tq, tk, tv, to, p, units, s);
  else if (mode == fa::kAttnCausal) launch_fwd_d<D, fa::kAttnCausal, false>(tq, tk, tv, to, p, units, s);
  else launch_fwd_d<D, fa::kAttnFull, false>(tq, tk, tv, to, p, units, s);
}

// Launches the forward kernel for d (maps and parameters prepared by the caller).  With
// `drop`, mode must be kAttnFull or kAttnCausal.
int launch_fwd(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &to,
               FwdParams &p, int d, int mode, cudaStream_t s, const fa::DropCfg *drop = nullptr) {
  const int g = p.Hq / p.Hkv;
  p.drop = drop ? *drop : fa::DropCfg{};
  if (mode != fa::kAttnSparse) p.bmask = nullptr;
  const int tslot = timer_start(0, s);
  // Unit order (unit_order), chosen from B200 measurements (forward TFLOP/s): dense causal
  // attention runs its heavy units first up to 16 query blocks, every level alone (gpt_2k
  // 660 -> 724; 826 against 777 for the head-major order below, persistent kernel); beyond,
  // head-major with half of the head pairs level by level at the end (persistent kernel, 8k
  // causal: two tiers of levels 1066, a tail of an eighth 1090-1095, a quarter 1098, 3/8
  // 1115, a half 1124-1141, 5/8 1134-1136, 3/4 1132; GQA 4k: an eighth 1072, a quarter to 5/8
  // 1086-1102, 3/4 1094); a band or a block mask goes level by level (window_8k_1k 578 ->
  // 611, blocksparse_8k 560 -> 614); full attention and packed sequences stay head-major
  // (packed: 680 head-major, 669-679 tiered).  The d = 256 forward keeps an eighth
  // (causal d = 256 was not measured).
  auto order = [&](int levels) {
    if (mode == fa::kAttnCausal) return p.nqb <= 16 ? 1 : levels;
    if (mode == fa::kAttnSparse || (mode == fa::kAttnGeneral && p.cu_q == nullptr)) return 1;
    return levels;
  };
  p.tail = 0;
  if (d == 256) {
    p.pair_heads = 0;
    p.tsz = order(p.nqb);
    if (mode == fa::kAttnCausal && p.nqb > 16) p.tail = p.B * p.Hq / 8;
    const unsigned units = static_cast<unsigned>(p.B) * p.Hq * p.nqb;
    launch_fwd_mode<256>(tq, tk, tv, to, p, units, mode, drop != nullptr, s);
  } else {
    p.pair_heads = (g % 2 == 0) ? 1 : 0;
    p.tsz = order(p.pair_heads ? p.nqb : (p.nqb + 1) / 2);
    if (mode == fa::kAttnCausal && p.nqb > 16) p.tail = (p.pair_heads ? p.B * (p.Hq / 2) : p.B * p.Hq) / 2;
    const unsigned units = p.pair_heads ? static_cast<unsigned>(p.B) * (p.Hq / 2) * p.nqb
                                        : static_cast<unsigned>(p.B) * p.Hq * ((p.nqb + 1) / 2);
    if (d == 64)
      launch_fwd_mode<64>(tq, tk, tv, to, p, units, mode, drop != nullptr, s);
    else
      launch_fwd_mode<128>(tq, tk, tv, to, p, units, mode, drop != nullptr, s);
  }
  const bool launched = cuda_ok(cudaGetLastError(), "fa_fwd launch");
  timer_stop(0, tslot, s);
  return launched ? FA_OK : FA_ERR_CUDA;
}

// Dropout configuration: keep iff the 16-bit Philox value >= floor(p 2^16) (capped at
// 2^16 - 1); kept values are scaled by the inverse of the exact keep probability.
bool make_drop(float p, unsigned long long seed, fa::DropCfg *out) {
  if (!(p >= 0.f) || !(p < 1.f)) return false;
  const double t = std::floor(static_cast<double>(p) * 65536.0);
  out->thr = t >= 65535.0 ? 65535u : static_cast<uint32_t>(t);
  out->thr2 = out->thr | (out->thr << 16);
  out->k0 = static_cast<uint32_t>(seed);
  out->k1 = static_cast<uint32_t>(seed >> 32);
  out->inv_keep = static_cast<float>(65536.0 / (65536.0 - static_cast<double>(out->thr)));
  return true;
}

// Packed-sequence sizes: totals up to 2^29 rows keep every band computation in int32.
int check_varlen_sizes(int B, int Hq, int Hkv, int total_q, int total_k, int max_q, int max_k, int d,
                       float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0)
    return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_GQA;
  if (total_q > (1 << 29) || total_k > (1 << 29) || max_q > (1 << 29) || max_k > (1 << 29) ||
      static_cast<long long>(total_q) * Hq >= (1ll << 31) ||
      static_cast<long long>(B) * Hq * ((max_q + 127) / 128) >= (1ll << 31) ||
      static_cast<long long>(B) * Hkv * ((max_k + 127) / 128) * 2 >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Window bound for packed sequences: a bound of max_q + max_k or more hides nothing.
bool normalise_window_varlen(int w, int max_q, int max_k, int *out) {
  if (w < -1) return false;
  *out = (w < 0 || static_cast<long long>(w) >= static_cast<long long>(max_q) + max_k) ? -1 : w;
  return true;
}

// Backward unit order (unit_order), from B200 measurements.  Dense causal attention runs
// head-major - one (b, kv head) row's key blocks heaviest first, its CTAs together in L2 -
// except for the last heads, which go level by level so that the grid ends on the lightest
// units: a quarter of the heads up to 16 key blocks, 3/8 beyond (main kernel TFLOP/s:
// gpt_2k 678 -> 694 and DRAM 977 -> 629 MB per launch against three tiers of levels over
// all heads, which stream every head's Q / dO / dQ rows once per tier - half of the heads
// in the tail ran as fast with 955 MB; 8k causal against head-major 800, with 4 of its 32
// heads in the tail 831, 6 843, 8 851, 12 853-855, 16 853, 20 847, 24 830).  A band goes
// level by level (window_8k_1k backward call 518 -> 541); full attention and (in the
// callers) block masks and packed sequences stay head-major.
fa::BwdOrder bwd_order(int B, int Hkv, int N, int left, int right) {
  if (left < 0 && right < 0) return {1, 0};
  if (left < 0 && right == 0) {
    const int heads = B * Hkv;
    return {1, (N + 127) / 128 <= 16 ? heads / 4 : heads * 3 / 8};
  }
  return {1 << 20, 0};
}

// Block-sparse limits: the forward keeps each CTA's key-block list in shared memory (at most
// 4096 blocks of 128 keys), the backward a bitmap of g x ceil(nb / 32) words.
int check_blocksparse(const unsigned char *mask, int Hq, int Hkv, int N, int d, int causal) {
  if (!mask || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  const long long nb = (N + 127) / 128;
  if (nb > fa::kMaxSparseBlocks) return FA_ERR_UNSUPPORTED;
  const long long words = static_cast<long long>(Hq / Hkv) * ((nb + 31) / 32);
  const int cap = d == 64 ? fa::BwdLayout<64, 64, 64>::kSparseBitmapBytes
                  : d == 128 ? fa::BwdLayout<128, 128, 64>::kSparseBitmapBytes
                             : fa::BwdLayout<256, 128, 32>::kSparseBitmapBytes;
  if (words * 4 > cap) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 102; }

const char *fa_status_string(int code) {
  switch (code) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported size (d must be 64, 128 or 256)";
    case FA_ERR_GQA: return "Hq must be a multiple of Hkv";
    case FA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error (no sm_100 device or launch failure)";
    case FA_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case FA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the static no-alloc buffer holds";
    case FA_ERR_SEQLENS: return "packed-sequence offsets inconsistent with the sizes given";
    default: return "unknown status";
  }
}

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
           int N, int d, int causal, float scale, void *stream) {
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  return fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, d, -1, causal ? 0 : -1, scale, stream);
}

int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                  int Hkv, int N, int d, int window_left, int window_right, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  int left = -1, right = -1;
  if (!normalise_window(window_left, N, &left) || !normalise_window(window_right, N, &right))
    return FA_ERR_INVALID_ARG;
  const bool window = left >= 0 || right >= 0;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;

  // Q and O move in 128-row tiles; K and V in 128-row blocks (64-row for d = 256).
  const int kv_rows = d == 256 ? 64 : 128;
  CUtensorMap tq, tk, tv, to;
  if (!make_map_bf16(&tq, q, d, N, static_cast<long long>(B) * Hq, 128) ||
      !make_map_bf16(&tk, k, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&tv, v, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&to, o, d, N, static_cast<long long>(B) * Hq, 128)) {
    if (debug_enabled()) std::fprintf(stderr, "[fa] cuTensorMapEncodeTiled failed (fa_fwd)\n");
    return FA_ERR_CUDA;
  }

  FwdParams p;
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.total_q = p.total_k = 0;
  p.nqb = (N + 127) / 128;
  p.left = left;
  p.right = right;
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  // Dense full and causal attention have their own kernel variants; other bands the general one.
  const int mode = !window ? fa::kAttnFull : (left < 0 && right == 0 ? fa::kAttnCausal : fa::kAttnGeneral);
  return launch_fwd(tq, tk, tv, to, p, d, mode, static_cast<cudaStream_t>(stream));
}

int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse, const int *cu_seqlens_q,
                  const int *cu_seqlens_k, int B, int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q,
                  int max_seqlen_k, int d, int window_left, int window_right, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
  int rc = check_varlen_sizes(B, Hq, Hkv, total_q, total_k, max_seqlen_q, max_seqlen_k, d, scale);
  if (rc != FA_OK) return rc;
  int left = -1, right = -1;
  if (!normalise_window_varlen(window_left, max_seqlen_q, max_seqlen_k, &left) ||
      !normalise_window_varlen(window_right, max_seqlen_q, max_seqlen_k, &right))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  if (total_q == 0 || max_seqlen_q == 0) return FA_OK;  // no query rows

  const int kv_rows = d == 256 ? 64 : 128;
  CUtensorMap tq, tk, tv, to;
  if (!make_map_packed(&tq, q, d, Hq, total_q, 128) || !make_map_packed(&tk, k, d, Hkv, total_k, kv_rows) ||
      !make_map_packed(&tv, v, d, Hkv, total_k, kv_rows) || !make_map_packed(&to, o, d, Hq, total_q, 128)) {
    if (debug_enabled()) std::fprintf(stderr, "[fa] cuTensorMapEncodeTiled failed (fa_fwd_varlen)\n");
    return FA_ERR_CUDA;
  }
  FwdParams p;
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = 0;
  p.total_q = total_q;
  p.total_k = total_k;
  p.nqb = (max_seqlen_q + 127) / 128;
  p.left = left;
  p.right = right;
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  return launch_fwd(tq, tk, tv, to, p, d, fa::kAttnGeneral, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  if (check_sizes(B, Hq, Hkv, N, d, 1.0f) != FA_OK) return 0;
  return fa::bwd_workspace_bytes(B, Hq, N, d);
}

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
           int B, int Hq, int Hkv, int N, int d, int causal, float scale, void *stream) {
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  return fa_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d,
                       -1, causal ? 0 : -1, scale, stream);
}

int fa_bwd_window(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                  int B, int Hq, int Hkv, int N, int d, int window_left, int window_right, float scale,
                  void *stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  int left = -1, right = -1;
  if (!normalise_window(window_left, N, &left) || !normalise_window(window_right, N, &right))
    return FA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < fa::bwd_workspace_bytes(B, Hq, N, d)) return FA_ERR_WORKSPACE;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  return fa::bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, d, left, right,
                        scale, static_cast<cudaStream_t>(stream), encode_fn(), &timer_start,
                        &timer_stop, nullptr, nullptr, nullptr, bwd_order(B, Hkv, N, left, right));
}

size_t fa_bwd_varlen_workspace_bytes(int Hq, int total_q, int d) {
  if (Hq < 1 || total_q < 0 || total_q > (1 << 29) || (d != 64 && d != 128 && d != 256) ||
      static_cast<long long>(total_q) * Hq >= (1ll << 31))
    return 0;
  return fa::bwd_workspace_bytes(1, Hq, total_q, d);
}

int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
                  void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes, const int *cu_seqlens_q,
                  const int *cu_seqlens_k, int B, int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q,
                  int max_seqlen_k, int d, int window_left, int window_right, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !cu_seqlens_q || !cu_seqlens_k)
    return FA_ERR_INVALID_ARG;
  int rc = check_varlen_sizes(B, Hq, Hkv, total_q, total_k, max_seqlen_q, max_seqlen_k, d, scale);
  if (rc != FA_OK) return rc;
  int left = -1, right = -1;
  if (!normalise_window_varlen(window_left, max_seqlen_q, max_seqlen_k, &left) ||
      !normalise_window_varlen(window_right, max_seqlen_q, max_seqlen_k, &right))
    return FA_ERR_INVALID_ARG;
  const size_t need = fa::bwd_workspace_bytes(1, Hq, total_q, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (total_k > 0 && (total_q == 0 || max_seqlen_q == 0 || max_seqlen_k == 0)) {
    // No query row sees a key: dK = dV = 0 (and there is no dQ row to write).
    if (!cuda_ok(cudaMemsetAsync(dk, 0, static_cast<size_t>(total_k) * Hkv * d * 2, s), "cudaMemsetAsync(dK)") ||
        !cuda_ok(cudaMemsetAsync(dv, 0, static_cast<size_t>(total_k) * Hkv * d * 2, s), "cudaMemsetAsync(dV)"))
      return FA_ERR_CUDA;
  }
  if (total_q == 0 || max_seqlen_q == 0 || max_seqlen_k == 0) {
    if (total_q > 0 &&
        !cuda_ok(cudaMemsetAsync(dq, 0, static_cast<size_t>(total_q) * Hq * d * 2, s), "cudaMemsetAsync(dQ)"))
      return FA_ERR_CUDA;
    return FA_OK;
  }
  const fa::PackedSeqs pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k};
  return fa::bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, 0, d, left, right, scale, s,
                        encode_fn(), &timer_start, &timer_stop, &pk);
}

int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                   int N, int d, int causal, float dropout_p, unsigned long long seed, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  fa::DropCfg drop;
  if (!make_drop(dropout_p, seed, &drop)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f) return fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  const int kv_rows = d == 256 ? 64 : 128;
  CUtensorMap tq, tk, tv, to;
  if (!make_map_bf16(&tq, q, d, N, static_cast<long long>(B) * Hq, 128) ||
      !make_map_bf16(&tk, k, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&tv, v, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&to, o, d, N, static_cast<long long>(B) * Hq, 128))
    return FA_ERR_CUDA;
  FwdParams p;
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.cu_q = p.cu_k = nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.total_q = p.total_k = 0;
  p.nqb = (N + 127) / 128;
  p.left = -1;
  p.right = causal ? 0 : -1;
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  return launch_fwd(tq, tk, tv, to, p, d, causal ? fa::kAttnCausal : fa::kAttnFull, static_cast<cudaStream_t>(stream),
                    &drop);
}

int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
                   void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                   int N, int d, int causal, float dropout_p, unsigned long long seed, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  fa::DropCfg drop;
  if (!make_drop(dropout_p, seed, &drop)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f)
    return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d, causal, scale,
                  stream);
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  if (!workspace || workspace_bytes < fa::bwd_workspace_bytes(B, Hq, N, d)) return FA_ERR_WORKSPACE;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  // N = 1 with causal is full attention (normalise_window's rule); the mask is the same.
  return fa::bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, d, -1, causal ? 0 : -1, scale,
                        static_cast<cudaStream_t>(stream), encode_fn(), &timer_start, &timer_stop, nullptr, &drop,
                        nullptr, bwd_order(B, Hkv, N, -1, causal ? 0 : -1));
}

int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                       const unsigned char *block_mask, int B, int Hq, int Hkv, int N, int d, int causal,
                       float scale, void *stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  rc = check_blocksparse(block_mask, Hq, Hkv, N, d, causal);
  if (rc != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  const int kv_rows = d == 256 ? 64 : 128;
  CUtensorMap tq, tk, tv, to;
  if (!make_map_bf16(&tq, q, d, N, static_cast<long long>(B) * Hq, 128) ||
      !make_map_bf16(&tk, k, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&tv, v, d, N, static_cast<long long>(B) * Hkv, kv_rows) ||
      !make_map_bf16(&to, o, d, N, static_cast<long long>(B) * Hq, 128))
    return FA_ERR_CUDA;
  FwdParams p;
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.cu_q = p.cu_k = nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.total_q = p.total_k = 0;
  p.nqb = (N + 127) / 128;
  p.left = -1;
  p.right = causal ? 0 : -1;  // the kernel reads causality from right == 0
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.bmask = block_mask;
  return launch_fwd(tq, tk, tv, to, p, d, fa::kAttnSparse, static_cast<cudaStream_t>(stream));
}

int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o, const float *lse,
                       const void *dout, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                       const unsigned char *block_mask, int B, int Hq, int Hkv, int N, int d, int causal,
                       float scale, void *stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  rc = check_blocksparse(block_mask, Hq, Hkv, N, d, causal);
  if (rc != FA_OK) return rc;
  if (!workspace || workspace_bytes < fa::bwd_workspace_bytes(B, Hq, N, d)) return FA_ERR_WORKSPACE;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  return fa::bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, d, -1, causal ? 0 : -1, scale,
                        static_cast<cudaStream_t>(stream), encode_fn(), &timer_start, &timer_stop, nullptr, nullptr,
                        block_mask);
}

int fa_set_fwd_scheduler(int persistent) {
  if (persistent != 0 && persistent != 1) return FA_ERR_INVALID_ARG;
  return g_fwd_persistent.exchange(persistent);
}

int fa_get_fwd_scheduler(void) { return g_fwd_persistent.load(); }

int fa_kernel_timing(int enable) {
  if (enable != 0 && enable != 1) return FA_ERR_INVALID_ARG;
  g_timer.enabled = enable != 0;
  if (enable) g_timer.count[0] = g_timer.count[1] = g_timer.count[2] = 0;
  return FA_OK;
}

int fa_kernel_time_ms(int which, float *ms, int *launches) {
  if (which < 0 || which > 2 || !ms || !launches) return FA_ERR_INVALID_ARG;
  float total = 0.f;
  for (int i = 0; i < g_timer.count[which]; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_timer.ev[which][i][1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_timer.ev[which][i][0], g_timer.ev[which][i][1]) != cudaSuccess)
      return FA_ERR_CUDA;
    total += t;
  }
  *ms = total;
  *launches = g_timer.count[which];
  return FA_OK;
}

int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N,
                   int d, int causal, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  const size_t need = fa::bwd_workspace_bytes(B, Hq, N, d);
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  void *scratch = noalloc_scratch();
  if (!scratch) return FA_ERR_CUDA;
  return fa::bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, scratch, B, Hq, Hkv, N, d, -1, causal ? 0 : -1, scale,
                        static_cast<cudaStream_t>(stream), encode_fn(), &timer_start, &timer_stop, nullptr,
                        nullptr, nullptr, bwd_order(B, Hkv, N, -1, causal ? 0 : -1));
}

int fa_watchdog_selftest(int limit_us, void *stream) {
  if (limit_us < 1 || limit_us > 10000000) return FA_ERR_INVALID_ARG;
  if (!device_ready()) return FA_ERR_CUDA;
  fa::fa_watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
  return cuda_ok(cudaGetLastError(), "fa_watchdog_selftest launch") ? FA_OK : FA_ERR_CUDA;
}

int fa_decode_num_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  if (check_decode_sizes(B, Hq, Hkv, Nq, Nk, d, 1.0f) != FA_OK) return 0;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    (void)cudaGetLastError();
    sms = 148;
  }
  // As many splits as fit into one wave of (b, K/V head) units - one CTA per SM, or two
  // for the variants with up to 16 query rows per K/V head and d = 64 - but at least two 128-key
  // blocks per split so each CTA streams a few blocks.
  const int slots = sms * (decode_rows_padded((Hq / Hkv) * Nq) == 16 && d == 64 ? 2 : 1);
  const long long units = static_cast<long long>(B) * Hkv;
  long long s = units >= slots ? 1 : slots / units;
  const long long blocks = (Nk + 127) / 128;
  const long long max_by_len = blocks / 2 > 1 ? blocks / 2 : 1;
  if (s > max_by_len) s = max_by_len;
  if (s > kMaxDecodeSplits) s = kMaxDecodeSplits;
  return static_cast<int>(s < 1 ? 1 : s);
}

size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits) {
  if (check_decode_sizes(B, Hq, Hkv, Nq, Nk, d, 1.0f) != FA_OK) return 0;
  if (num_splits < 1 || num_splits > kMaxDecodeSplits) return 0;
  return decode_workspace(B, Hq, Nq, d, num_splits);
}

int fa_decode(const void *q, const void *k, const void *v, void *o, float *lse, const int *seqlens_k,
              void *workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Nq, int Nk, int d,
              int causal, int num_splits, float scale, void *stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > kMaxDecodeSplits) return FA_ERR_INVALID_ARG;
  int rc = check_decode_sizes(B, Hq, Hkv, Nq, Nk, d, scale);
  if (rc != FA_OK) return rc;
  if (static_cast<long long>(B) * Hkv * num_splits >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace(B, Hq, Nq, d, num_splits);
  if (need > 0 && (!workspace || workspace_bytes < need)) return FA_ERR_WORKSPACE;
  const void *ptrs[] = {q, k, v, o, lse};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if ((need > 0 && !aligned16(workspace)) || (reinterpret_cast<uintptr_t>(seqlens_k) & 3u)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;

  const int g = Hq / Hkv, R = g * Nq, RP = decode_rows_padded(R);
  CUtensorMap tq, tk, tv;
  // Q viewed as [B * Hkv][R][d]: the rows of the query heads that share a K/V head.
  if (!make_map_bf16(&tq, q, d, R, static_cast<long long>(B) * Hkv, RP) ||
      !make_map_bf16(&tk, k, d, Nk, static_cast<long long>(B) * Hkv, 128) ||
      !make_map_bf16(&tv, v, d, Nk, static_cast<long long>(B) * Hkv, 128)) {
    if (debug_enabled()) std::fprintf(stderr, "[fa] cuTensorMapEncodeTiled failed (fa_decode)\n");
    return FA_ERR_CUDA;
  }
  const size_t rows = static_cast<size_t>(B) * Hq * Nq;
  fa::DecodeParams p;
  p.lens = seqlens_k;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.lse = lse;
  p.o_part = num_splits > 1 ? static_cast<float *>(workspace) : nullptr;
  p.lse_part = num_splits > 1
                   ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                               fa::pad256(static_cast<size_t>(num_splits) * rows * d * 4))
                   : nullptr;
  p.B = B;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.R = R;
  p.splits = num_splits;
  const int per = (Nk + num_splits - 1) / num_splits;
  p.chunk = (per + 127) / 128 * 128;
  p.causal = causal;
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(B) * Hkv * num_splits;
  const int tslot = timer_start(2, s);
  if (d == 64) launch_decode_d<64>(RP, tq, tk, tv, p, grid, s);
  else if (d == 128) launch_decode_d<128>(RP, tq, tk, tv, p, grid, s);
  else launch_decode_d<256>(RP, tq, tk, tv, p, grid, s);
  timer_stop(2, tslot, s);
  if (num_splits > 1) launch_merge(p.o_part, p.lse_part, o, lse, num_splits, static_cast<long long>(rows), d, s);
  return cuda_ok(cudaGetLastError(), "fa_decode launch") ? FA_OK : FA_ERR_CUDA;
}

int fa_merge(const float *o_parts, const float *lse_parts, void *o, float *lse, int num_parts, int rows,
             int d, void *stream) {
  if (!o_parts || !lse_parts || !o || !lse || num_parts < 1 || rows < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_parts) * rows * d >= (1ll << 40)) return FA_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (!device_ready()) return FA_ERR_CUDA;
  launch_merge(o_parts, lse_parts, o, lse, num_parts, rows, d, static_cast<cudaStream_t>(stream));
  return cuda_ok(cudaGetLastError(), "fa_merge launch") ? FA_OK : FA_ERR_CUDA;
}

int fa_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int status = 0;
  if (cudaMemcpyFromSymbol(&status, fa::g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (status != FA_OK) {
    const int zero = 0;
    const unsigned long long zero64 = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(fa::g_fa_status_site, &zero64, sizeof(zero64)) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return status;
}

}  // extern "C"
