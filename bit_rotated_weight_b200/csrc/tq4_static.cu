// tq4_1s_linear_static: the small-m quantized linear layer for callers that
// cannot allocate device memory.
//
// Some hosts of this layer hand it only its input and output buffers: plugin
// runtimes and serving engines that plan every device allocation at start-up
// and forbid new ones afterwards (cudaMalloc can synchronize the device, fail
// under memory pressure mid-request, or break a fixed memory budget).  Such a
// caller cannot supply the workspace tq4_1s_linear asks for.  This entry point
// runs the same two kernels as tq4_1s_linear's small-m path (activation
// rotation, then the stream-K dequant-GEMM) but keeps their scratch -- the
// rotated activations and their row scales, the stream-K partial sums and the
// tile counters -- in one file-scope device array of fixed size.  The array is
// reserved on a GPU when the library's device code is loaded there: with
// CUDA's default lazy module loading that is the first call of the library
// on that GPU that needs it (the first call of this entry point looks up the
// array's address, which loads the module), after which it is held until the
// process exits.
#include <mutex>

#include "tq4_internal.h"

#define TQ_STATIC_API extern "C" __attribute__((visibility("default")))

namespace tq4 {
namespace {

// Limits of the static scratch: m <= 32 rows, k <= 8192, n <= 32768, and at
// most 148 CTAs in the stream-K grid.
constexpr int64_t kStaticMaxM = 32;
constexpr int64_t kStaticMaxK = 8192;
constexpr int64_t kStaticMaxN = 32768;
constexpr int kStaticMaxGrid = 148;
constexpr size_t kStaticXBytes = static_cast<size_t>(kStaticMaxM * kStaticMaxK) * 2;   // x' (fp16)
constexpr size_t kStaticPartialBytes = static_cast<size_t>(kStaticMaxGrid) * 2 * 128 * kSegRows * 4;
constexpr size_t kStaticScaleBytes = 256;                                              // x' row scales
constexpr size_t kStaticCounterBytes = static_cast<size_t>(kStaticMaxN / 128) * 8;
constexpr size_t kStaticScratchBytes =
    kStaticXBytes + kStaticScaleBytes + kStaticPartialBytes + kStaticCounterBytes;   // ~5.2 MiB

// The scratch itself.  In host code this name is only a stand-in for the
// device symbol: its device address must be fetched with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_linear_scratch[kStaticScratchBytes];

// Device address of g_linear_scratch on the current device, looked up once
// per device (with that device current) and cached.
int scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return TQ_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return TQ_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return TQ_OK;
}

}  // namespace
}  // namespace tq4

using namespace tq4;

TQ_STATIC_API int tq4_1s_linear_static(const uint16_t* x, int64_t m, const tq4_1s_weight* w, uint16_t* y,
                                       tq4_stream_t stream) {
  if (!w) return TQ_ERR_INVALID_ARG;
  if (w->n <= 0 || w->k <= 0 || (w->k % 32) != 0 || w->num_experts != 1 || (w->flags & ~TQ_WEIGHT_STATIC) != 0 || m < 0)
    return TQ_ERR_INVALID_ARG;
  if (!w->codes || !w->scales) return TQ_ERR_INVALID_ARG;
  if (m > kStaticMaxM || w->k > kStaticMaxK || w->n > kStaticMaxN) return TQ_ERR_SCRATCH_LIMIT;
  if (m == 0) return TQ_OK;
  if (!x || !y) return TQ_ERR_INVALID_ARG;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(x) || !a16(y) || !a16(w->codes) || !a16(w->scales)) return TQ_ERR_ALIGNMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc) return rc;
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;

  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint16_t* xr = reinterpret_cast<uint16_t*>(base);
  float* xscale = reinterpret_cast<float*>(base + kStaticXBytes);
  float* partials = reinterpret_cast<float*>(base + kStaticXBytes + kStaticScaleBytes);
  unsigned long long* counters =
      reinterpret_cast<unsigned long long*>(base + kStaticXBytes + kStaticScaleBytes + kStaticPartialBytes);
  const int64_t row_tiles = (w->n + 127) / 128, k_iters = (w->k + 127) / 128;
  const int64_t tiles = row_tiles;   // m <= 32: one segment
  const int64_t T = tiles * k_iters;
  int grid = sms < kStaticMaxGrid ? sms : kStaticMaxGrid;
  if (T < grid) grid = static_cast<int>(T);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t mask = 0;
  tq4_1s_sign_mask(w->seed, &mask);

  // m <= 32 is one segment: the stream-K kernel rotates x itself when no CTA
  // runs more iterations than it has stages; otherwise the rotation kernel
  // writes x' into the scratch first.  The tile counters carry each launch's
  // epoch, so what a previous call left in them does no harm.
  const int split = choose_cluster_split(tiles, k_iters, sms < kStaticMaxGrid ? sms : kStaticMaxGrid);
  if (split > 1) grid = static_cast<int>(tiles * split);
  const bool fused = split > 1 || (T + grid - 1) / grid <= kFusedMaxIters;
  if (!fused && launch_rotate_scaled(x, w->k, nullptr, 1, nullptr, m, m, xr, xscale, mask, st) != cudaSuccess)
    return TQ_ERR_CUDA;
  // the cached tensor maps of tq4_1s_linear: codes [1][n][k/2] (64 B x 128
  // rows), x' (TMA-fed mode) or x (fused mode) [m][k] (64 x 16), and in the
  // cluster split-K mode x as one 3-D box per CTA
  alignas(64) CUtensorMap tc, tx, tx3;
  if (!map_codes(&tc, w) || !map_bf16(&tx, fused ? static_cast<const void*>(x) : xr, m, w->k, 16)) return TQ_ERR_CUDA;
  const bool box3 = split > 1 && (w->k % 64) == 0;
  if (box3 && !map_x3(&tx3, x, m, w->k)) return TQ_ERR_CUDA;
  StreamKArgs a{};
  a.n = static_cast<int32_t>(w->n);
  a.k = static_cast<int32_t>(w->k);
  a.row_tiles = static_cast<int32_t>(row_tiles);
  a.k_iters = static_cast<int32_t>(k_iters);
  a.nseg_host = 1;
  a.m_host = static_cast<int32_t>(m);
  a.nb_max = m > 16 ? 2 : 1;
  a.scales = w->scales;
  a.codes = w->codes;
  a.xr = fused ? nullptr : xr;
  a.row_scale = xscale;
  if (fused) {
    a.x_raw = x;
    sign_xor_words(mask, a.x_sign);
  }
  a.epoch = next_epoch();
  a.cluster_s = split;
  a.x_box3 = box3 ? 1 : 0;
  a.mode = EPI_DENSE;
  a.out_a = y;
  a.partials = partials;
  a.counters = counters;
  a.max_tiles = static_cast<int32_t>(tiles);
  return launch_streamk(&tc, &tx, box3 ? &tx3 : nullptr, a, grid, st) == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
