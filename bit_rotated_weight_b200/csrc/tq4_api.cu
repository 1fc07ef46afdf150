// Host side of libtq4_1s.so: the extern "C" entry points declared in
// include/tq4_1s.h -- argument validation, the codebook, the RHT sign mask,
// TMA tensor-map construction and the launch sequences of each call.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "tq4_internal.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace tq4 {

// ------------------------------------------------------------------ codebook
// 16-level Lloyd-Max quantizer of N(0,1) ("16-level Lloyd-Max", model card
// section "What Config-I means").  The quantizer of a symmetric density is
// odd-symmetric, so only the 8 positive levels m_0 < ... < m_7 are iterated,
// with interval edges b_0 = 0, b_j = (m_{j-1} + m_j) / 2, b_8 = +inf and the
// centroid update m_j = E[X | b_j < X < b_{j+1}].
static CodebookF32 compute_codebook() {
  const double inv_sqrt2 = 0.70710678118654752440;
  const double inv_sqrt2pi = 0.39894228040143267794;
  auto pdf = [&](double x) { return std::isinf(x) ? 0.0 : inv_sqrt2pi * std::exp(-0.5 * x * x); };
  auto upper_tail = [&](double x) { return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x * inv_sqrt2); };  // P(X > x)
  double mlev[8];
  for (int j = 0; j < 8; ++j) mlev[j] = 0.35 * (j + 0.5);
  for (int iter = 0; iter < 100000; ++iter) {
    double edge[9];
    edge[0] = 0.0;
    for (int j = 1; j < 8; ++j) edge[j] = 0.5 * (mlev[j - 1] + mlev[j]);
    edge[8] = INFINITY;
    double change = 0.0;
    for (int j = 0; j < 8; ++j) {
      const double mass = upper_tail(edge[j]) - upper_tail(edge[j + 1]);
      const double next = (pdf(edge[j]) - pdf(edge[j + 1])) / mass;
      change = std::fmax(change, std::fabs(next - mlev[j]));
      mlev[j] = next;
    }
    if (change < 1e-14) break;
  }
  CodebookF32 cb{};
  for (int j = 0; j < 8; ++j) {
    cb.levels[8 + j] = static_cast<float>(mlev[j]);
    cb.levels[7 - j] = -static_cast<float>(mlev[j]);
  }
  cb.thresholds[7] = 0.0f;
  for (int j = 1; j < 8; ++j) {
    const float tj = static_cast<float>(0.5 * (mlev[j - 1] + mlev[j]));
    cb.thresholds[7 + j] = tj;
    cb.thresholds[7 - j] = -tj;
  }
  cb.thresholds[15] = INFINITY;
  return cb;
}

const CodebookF32& codebook() {
  static const CodebookF32 cb = compute_codebook();
  return cb;
}

static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

static std::atomic<int64_t> g_fail_next{0};
static std::atomic<int> g_withhold{0};
bool take_injected_failure() {
  int64_t v = g_fail_next.load(std::memory_order_relaxed);
  while (v > 0)
    if (g_fail_next.compare_exchange_weak(v, v - 1, std::memory_order_relaxed)) return true;
  return false;
}
bool withhold_arrival_hook() { return g_withhold.load(std::memory_order_relaxed) != 0; }

// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): first output from `state`.
static uint32_t sign_mask_of(uint64_t state) {
  uint64_t z = state + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return static_cast<uint32_t>(z);
}

// ------------------------------------------------------------------ helpers
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  int ok = -1;   // -1 unknown, 0 unsupported, 1 sm_100
  int sms = 0;
};

int check_device(int* sms_out) {
  static std::mutex mu;
  static DeviceInfo info[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return TQ_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> g(mu);
  if (info[dev].ok < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return TQ_ERR_UNSUPPORTED_DEVICE;
    }
    info[dev].ok = (major == 10 && minor == 0) ? 1 : 0;
    info[dev].sms = sms;
  }
  if (info[dev].ok != 1) return TQ_ERR_UNSUPPORTED_DEVICE;
  if (sms_out) *sms_out = info[dev].sms;
  return TQ_OK;
}

static int weight_ok(const tq4_1s_weight* w, bool need_ptrs) {
  if (!w) return TQ_ERR_INVALID_ARG;
  if (w->n <= 0 || w->k <= 0 || (w->k % 32) != 0 || w->num_experts <= 0 || (w->flags & ~TQ_WEIGHT_STATIC) != 0)
    return TQ_ERR_INVALID_ARG;
  if (w->n > (1ll << 30) || w->k > (1ll << 30) || w->num_experts > (1 << 20)) return TQ_ERR_INVALID_ARG;
  if (need_ptrs) {
    if (!w->codes || !w->scales) return TQ_ERR_INVALID_ARG;
    if (!aligned16(w->codes) || !aligned16(w->scales)) return TQ_ERR_ALIGNMENT;
  }
  return TQ_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor maps depend only on the address, shape and box they describe, so
// encoded ones are kept: a weight, or an activation buffer, used call after
// call is encoded once.  The cache is 4-way set associative (512 sets, the
// set chosen by a hash of the key, round-robin replacement in a set), so a
// model's few hundred weights and buffers all stay resident and a lookup
// costs four compares.
struct MapKey {
  int kind;
  const void* ptr;
  int64_t d0, d1, d2;
  bool operator==(const MapKey& o) const {
    return kind == o.kind && ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && d2 == o.d2;
  }
  uint64_t hash() const {
    uint64_t h = reinterpret_cast<uintptr_t>(ptr) ^ (static_cast<uint64_t>(kind) << 56);
    for (const int64_t v : {d0, d1, d2}) h = (h ^ static_cast<uint64_t>(v)) * 0x9E3779B97F4A7C15ull;
    return h ^ (h >> 29);
  }
};

template <typename Encode>
static bool cached_map(CUtensorMap* m, const MapKey& key, Encode encode) {
  struct Entry {
    MapKey key;
    bool valid;
    CUtensorMap map;
  };
  constexpr int kSets = 512, kWays = 4;
  static std::mutex mu;
  static Entry cache[kSets][kWays];
  static uint8_t next[kSets];
  const int set = static_cast<int>(key.hash() & (kSets - 1));
  {
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < kWays; ++i)
      if (cache[set][i].valid && cache[set][i].key == key) {
        *m = cache[set][i].map;
        return true;
      }
  }
  if (!encode(m)) return false;
  std::lock_guard<std::mutex> g(mu);
  Entry& e = cache[set][next[set]];
  next[set] = static_cast<uint8_t>((next[set] + 1) % kWays);
  e.key = key;
  e.map = *m;
  e.valid = true;
  return true;
}

// Codes plane [E][n][k/2] bytes, box 64 B x 128 rows, 64-byte swizzle.
bool map_codes(CUtensorMap* m, const tq4_1s_weight* w) {
  return cached_map(m, MapKey{0, w->codes, w->n, w->k, w->num_experts}, [&](CUtensorMap* out) {
    const uint64_t dims[3] = {static_cast<uint64_t>(w->k / 2), static_cast<uint64_t>(w->n),
                              static_cast<uint64_t>(w->num_experts)};
    const uint64_t strides[2] = {static_cast<uint64_t>(w->k / 2), static_cast<uint64_t>(w->n * (w->k / 2))};
    const uint32_t box[3] = {64, 128, 1};
    return make_map(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w->codes, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
  });
}

// x [rows][cols] (cols % 64 == 0) viewed as [cols/64][rows][64] 16-bit,
// box 64 x 32 x 2*kFusedMaxIters, 128-byte swizzle: one copy fills the B
// tiles of all stages of a fused CTA.
bool map_x3(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  return cached_map(m, MapKey{1, base, rows, cols, 0}, [&](CUtensorMap* out) {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / 64)};
    const uint64_t strides[2] = {static_cast<uint64_t>(cols * 2), 128};
    const uint32_t box[3] = {64, static_cast<uint32_t>(kSegRows), static_cast<uint32_t>(2 * kFusedMaxIters)};
    return make_map(out, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  });
}

bool map_x3d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows, uint32_t box_chunks) {
  return cached_map(m, MapKey{4, base, rows, cols, static_cast<int64_t>(box_rows) * 1024 + box_chunks},
                    [&](CUtensorMap* out) {
                      const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(cols / 64)};
                      const uint64_t strides[2] = {static_cast<uint64_t>(cols * 2), 128};
                      const uint32_t box[3] = {64, box_rows, box_chunks};
                      return make_map(out, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, base, dims, strides, box,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
                    });
}

// 16-bit matrix [rows][cols] row-major (bf16 or fp16), box 64 x box_rows,
// 128-byte swizzle.
bool map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  return cached_map(m, MapKey{2, base, rows, cols, box_rows}, [&](CUtensorMap* out) {
    const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(cols * 2)};
    const uint32_t box[2] = {64, box_rows};
    return make_map(out, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  });
}

// fp8 cache codes [n][k] bytes, box 128 B x 128 rows, 128-byte swizzle.
static bool map_fp8(CUtensorMap* m, const uint8_t* q, int64_t n, int64_t k) {
  return cached_map(m, MapKey{3, q, n, k, 1}, [&](CUtensorMap* out) {
    const uint64_t dims[3] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n), 1};
    const uint64_t strides[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n * k)};
    const uint32_t box[3] = {128, 128, 1};
    return make_map(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  });
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Small-m path threshold: up to this many rows, the stream-K kernel streams
// the packed weight once per 32-row segment; above it, dequantize + GEMM.
constexpr int64_t kSmallM = 128;

struct SmallLayout {
  size_t xr, xscale, partials, counters, total;
  int grid;
  int64_t tiles;
};

// Small-m workspace: the rotated activations (fp16, per-row scales; unused
// when the kernel rotates x itself), the stream-K fp32
// partials and the tile counters.  Counters carry the launch's epoch and the
// last arriver of each split tile resets its counter, so the workspace needs
// no initialisation and a captured call can be replayed.
static SmallLayout small_layout(int64_t m, const tq4_1s_weight* w, int sms) {
  SmallLayout L{};
  const int64_t nseg = (m + kSegRows - 1) / kSegRows;
  const int64_t rt = (w->n + 127) / 128, ki = (w->k + 127) / 128;
  L.tiles = nseg * rt;
  const int64_t T = L.tiles * ki;
  L.grid = static_cast<int>(T < sms ? T : sms);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.xr = take(static_cast<size_t>(m * w->k) * 2);
  L.xscale = take(static_cast<size_t>(m) * 4);
  L.partials = take(static_cast<size_t>(sms) * 2 * 128 * kSegRows * 4);
  L.counters = take(static_cast<size_t>(L.tiles) * 8);
  L.total = off;
  return L;
}

// The dense kernel rotates x itself when it is one segment and no CTA runs
// more iterations than it has stages.
static bool small_fused(int64_t m, int64_t tiles_times_ki, int grid) {
  return m <= kSegRows && (tiles_times_ki + grid - 1) / grid <= kFusedMaxIters;
}

struct MoeLayout {
  size_t offsets, pairs, segs, nseg, npv, ids, wts, xr, xscale, h, hr, hscale, zw, partials, cnt_up, cnt_dn, total;
  int64_t P, maxseg, rt_up, rt_dn;
  int nb_max, chunk;
};

static MoeLayout moe_layout(int64_t m, int32_t topk, const tq4_1s_weight* up, const tq4_1s_weight* dn, int sms) {
  MoeLayout L{};
  const int64_t E = up->num_experts;
  const int64_t H = up->k, I = up->n;
  L.P = m * topk;
  // Token columns per segment: the accumulators are sized for 16 * nb_max
  // columns, so no segment may hold more rows.  With distinct expert ids per
  // token an expert takes at most m rows, so up to 16 tokens one 16-column
  // block suffices; a token that names an expert twice adds a row, and the
  // 16-row segments keep that case correct too.
  L.nb_max = m > 16 ? 2 : 1;
  L.chunk = 16 * L.nb_max;
  L.maxseg = (L.P + L.chunk - 1) / L.chunk + (E < L.P ? E : L.P) + 1;
  L.rt_up = (I + 127) / 128;
  L.rt_dn = (dn->n + 127) / 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.offsets = take((E + 1) * 4);
  L.pairs = take(L.P * 4);
  L.segs = take(L.maxseg * 16);
  L.nseg = take(4);
  L.npv = take(4);
  L.ids = take(L.P * 4);   // router output (tq4_1s_moe_logits)
  L.wts = take(L.P * 4);
  L.xr = take(L.P * H * 2);
  L.xscale = take(L.P * 4);
  L.h = take(L.P * I * 2);
  L.hr = take(L.P * I * 2);
  L.hscale = take(L.P * 4);
  L.zw = take(L.P * H * 4);
  L.partials = take(static_cast<size_t>(sms) * 2 * 128 * kSegRows * 4);
  L.cnt_up = take(L.maxseg * L.rt_up * 8);
  L.cnt_dn = take(L.maxseg * L.rt_dn * 8);
  L.total = off;
  return L;
}

static int cuda_rc(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

}  // namespace tq4

using namespace tq4;

// ==================================================================== ABI
TQ_API int tq4_1s_version(void) { return 102; }

TQ_API const char* tq4_1s_error_string(int code) {
  switch (code) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case TQ_ERR_UNSUPPORTED_DEVICE: return "current device is not an sm_100 (B200) GPU";
    case TQ_ERR_WORKSPACE: return "workspace missing or too small";
    case TQ_ERR_CUDA: return "CUDA call failed";
    case TQ_ERR_TIMEOUT: return "a bounded device wait timed out";
    case TQ_ERR_BAD_ROUTING: return "routing expert id out of range";
    case TQ_ERR_NONFINITE: return "non-finite value in quantize input";
    case TQ_ERR_SCRATCH_LIMIT: return "shape exceeds the fixed scratch of tq4_1s_linear_static (m<=32, k<=8192, n<=32768)";
    default: return "unknown error code";
  }
}

TQ_API int tq4_1s_packed_bytes(int64_t n, int64_t k, int32_t num_experts, size_t* codes_bytes,
                               size_t* scales_bytes) {
  if (n <= 0 || k <= 0 || k % 32 != 0 || num_experts <= 0 || !codes_bytes || !scales_bytes) return TQ_ERR_INVALID_ARG;
  *codes_bytes = static_cast<size_t>(num_experts) * static_cast<size_t>(n) * static_cast<size_t>(k / 2);
  *scales_bytes = static_cast<size_t>(num_experts) * static_cast<size_t>(n) * static_cast<size_t>(k / 16) * 2;
  return TQ_OK;
}

TQ_API int tq4_1s_sign_mask(uint64_t seed, uint32_t* mask) {
  if (!mask) return TQ_ERR_INVALID_ARG;
  *mask = sign_mask_of(seed);
  return TQ_OK;
}

TQ_API int tq4_1s_codebook(float* levels, float* thresholds) {
  const CodebookF32& cb = codebook();
  if (levels) std::memcpy(levels, cb.levels, sizeof(float) * 16);
  if (thresholds) std::memcpy(thresholds, cb.thresholds, sizeof(float) * 15);
  return TQ_OK;
}

TQ_API int tq4_1s_quantize(const void* W, int dtype, const tq4_1s_weight* out, tq4_stream_t stream) {
  int rc = weight_ok(out, true);
  if (rc) return rc;
  if (!W || (dtype != TQ_DTYPE_F32 && dtype != TQ_DTYPE_BF16)) return TQ_ERR_INVALID_ARG;
  if (!aligned16(W)) return TQ_ERR_ALIGNMENT;
  if ((rc = check_device(nullptr))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  const int64_t rows = out->n * out->num_experts;
  return cuda_rc(launch_quantize(W, dtype, out->codes, out->scales, rows, out->k, sign_mask_of(out->seed),
                                 codebook(), reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API int tq4_1s_quantize_batched(const void* const* W, int dtype, const tq4_1s_weight* outs, int32_t count,
                                   tq4_stream_t stream) {
  if (count < 0 || (count > 0 && (!W || !outs))) return TQ_ERR_INVALID_ARG;
  if (dtype != TQ_DTYPE_F32 && dtype != TQ_DTYPE_BF16) return TQ_ERR_INVALID_ARG;
  if (count == 0) return TQ_OK;
  for (int32_t i = 0; i < count; ++i) {
    int rc = weight_ok(&outs[i], true);
    if (rc) return rc;
    if (!W[i]) return TQ_ERR_INVALID_ARG;
    if (!aligned16(W[i])) return TQ_ERR_ALIGNMENT;
  }
  int rc = check_device(nullptr);
  if (rc) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  std::vector<QuantItem> items(static_cast<size_t>(count));
  for (int32_t i = 0; i < count; ++i)
    items[i] = QuantItem{W[i], outs[i].codes, outs[i].scales, outs[i].n * outs[i].num_experts, outs[i].k,
                         sign_mask_of(outs[i].seed)};
  return cuda_rc(launch_quantize_batch(items.data(), count, dtype, codebook(), reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API int tq4_1s_dequantize(const tq4_1s_weight* w, float* W_out, tq4_stream_t stream) {
  int rc = weight_ok(w, true);
  if (rc) return rc;
  if (!W_out) return TQ_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return TQ_ERR_ALIGNMENT;
  if ((rc = check_device(nullptr))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  return cuda_rc(launch_dequantize_f32(w->codes, w->scales, W_out, w->n * w->num_experts, w->k,
                                       sign_mask_of(w->seed), codebook(), reinterpret_cast<cudaStream_t>(stream)));
}

static int sms_or_default() {
  int sms = 148;
  if (check_device(&sms) != TQ_OK) sms = 148;
  return sms;
}

TQ_API size_t tq4_1s_linear_workspace(int64_t m, const tq4_1s_weight* w) {
  if (m < 0 || weight_ok(w, false) != TQ_OK || w->num_experts != 1) return 0;
  if (m == 0) return 0;
  if (m <= kSmallM) return small_layout(m, w, sms_or_default()).total;
  return align256(static_cast<size_t>(w->n) * static_cast<size_t>(w->k) * 2);
}

TQ_API int tq4_1s_linear(const uint16_t* x, int64_t m, const tq4_1s_weight* w, uint16_t* y, void* ws,
                         size_t ws_bytes, tq4_stream_t stream) {
  int rc = weight_ok(w, true);
  if (rc) return rc;
  if (w->num_experts != 1 || m < 0 || m > (1ll << 24)) return TQ_ERR_INVALID_ARG;
  if (m == 0) return TQ_OK;
  if (!x || !y) return TQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TQ_ERR_ALIGNMENT;
  int sms = 0;
  if ((rc = check_device(&sms))) return rc;
  const bool small = m <= kSmallM;
  const SmallLayout L = small ? small_layout(m, w, sms) : SmallLayout{};
  const size_t need = small ? L.total : align256(static_cast<size_t>(w->n) * static_cast<size_t>(w->k) * 2);
  if (!ws || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const uint32_t mask = sign_mask_of(w->seed);

  if (small && m <= kSegRows) {
    // the decode-block kernel: one launch, activation-dependent work only
    // after the dependency wait (see tq4_decode.cu)
    const int nb = m > 16 ? 2 : 1;
    const int64_t KI = (w->k + 127) / 128;
    const int split = choose_decode_split(L.tiles, KI, sms, nb);
    if (split > 0) {
      alignas(64) CUtensorMap tc, tx, ts;
      const bool sc_tma = (w->k % 128) == 0;
      const bool box3 = (w->k % 64) == 0;
      if (!map_codes(&tc, w) ||
          !(box3 ? map_x3d(&tx, x, m, w->k, static_cast<uint32_t>(16 * nb), 2 * kFusedMaxIters)
                 : map_bf16(&tx, x, m, w->k, static_cast<uint32_t>(16 * nb))) ||
          (sc_tma && !map_bf16(&ts, w->scales, w->n, w->k / 16, 128)))
        return TQ_ERR_CUDA;
      DecodeArgs d{};
      d.n = static_cast<int32_t>(w->n);
      d.k = static_cast<int32_t>(w->k);
      d.m = static_cast<int32_t>(m);
      d.nb = nb;
      d.row_tiles = static_cast<int32_t>(L.tiles);
      d.k_iters = static_cast<int32_t>(KI);
      d.split = split;
      d.static_w = (w->flags & TQ_WEIGHT_STATIC) ? 1 : 0;
      d.test_withhold = withhold_arrival_hook() ? 1 : 0;
      d.x = x;
      d.scales = w->scales;
      d.scales_tma = sc_tma ? 1 : 0;
      d.x_box3 = box3 ? 1 : 0;
      d.y = y;
      sign_xor_words(mask, d.x_sign);
      d.sign_bits = mask;
      return cuda_rc(launch_decode(&tc, &tx, &ts, d, st));
    }
  }
  if (small) {
    const int64_t T = L.tiles * ((w->k + 127) / 128);
    if (T > INT32_MAX) return TQ_ERR_INVALID_ARG;   // 32-bit iteration space
    // m <= 32 (one segment): cluster split-K when it fits in one wave, else
    // stream-K (the kernel rotates x itself when every CTA has a stage per
    // iteration, else the rotation kernel feeds x' through memory)
    const int64_t KI = (w->k + 127) / 128;
    const int split = m <= kSegRows ? choose_cluster_split(L.tiles, KI, sms) : 1;
    const int grid = split > 1 ? static_cast<int>(L.tiles * split) : L.grid;
    const bool fused = split > 1 || small_fused(m, T, L.grid);
    uint16_t* xr = reinterpret_cast<uint16_t*>(base + L.xr);
    float* xscale = reinterpret_cast<float*>(base + L.xscale);
    // TMA-fed mode: x' = R x (fp16, per-row scale) by the rotation kernel
    if (!fused && launch_rotate_scaled(x, w->k, nullptr, 1, nullptr, m, m, xr, xscale, mask, st) != cudaSuccess)
      return TQ_ERR_CUDA;
    alignas(64) CUtensorMap tc, tx, tx3;
    // the producer stages x' (TMA-fed mode) or the raw x (fused mode)
    if (!map_codes(&tc, w) || !map_bf16(&tx, fused ? static_cast<const void*>(x) : xr, m, w->k, 16))
      return TQ_ERR_CUDA;
    const bool box3 = split > 1 && (w->k % 64) == 0;
    if (box3 && !map_x3(&tx3, x, m, w->k)) return TQ_ERR_CUDA;
    StreamKArgs a{};
    a.n = static_cast<int32_t>(w->n);
    a.k = static_cast<int32_t>(w->k);
    a.row_tiles = static_cast<int32_t>((w->n + 127) / 128);
    a.k_iters = static_cast<int32_t>((w->k + 127) / 128);
    a.nseg_host = static_cast<int32_t>((m + kSegRows - 1) / kSegRows);
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
    a.partials = reinterpret_cast<float*>(base + L.partials);
    a.counters = reinterpret_cast<unsigned long long*>(base + L.counters);
    a.max_tiles = static_cast<int32_t>(L.tiles);
    return cuda_rc(launch_streamk(&tc, &tx, box3 ? &tx3 : nullptr, a, grid, st));
  }
  // large m: W_hat in bf16, then the tensor-core GEMM
  uint16_t* wh = reinterpret_cast<uint16_t*>(base);
  cudaError_t e = launch_dequantize_bf16(w->codes, w->scales, wh, w->n, w->k, mask, codebook(), st);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  alignas(64) CUtensorMap tx, tw;
  if (!map_bf16(&tx, x, m, w->k, 128) || !map_bf16(&tw, wh, w->n, w->k, 256)) return TQ_ERR_CUDA;
  const int64_t tiles = ((m + 127) / 128) * ((w->n + 255) / 256);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  return cuda_rc(launch_gemm_bf16(&tx, &tw, y, static_cast<int32_t>(m), static_cast<int32_t>(w->n),
                                  static_cast<int32_t>(w->k), grid, st));
}

// ------------------------------------------------------------------ fp8 cache
TQ_API int tq4_1s_to_fp8(const tq4_1s_weight* w, uint8_t* q, float* wscale, tq4_stream_t stream) {
  int rc = weight_ok(w, true);
  if (rc) return rc;
  if (!q || !wscale) return TQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(wscale)) return TQ_ERR_ALIGNMENT;
  if ((rc = check_device(nullptr))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  return cuda_rc(launch_to_fp8(w->codes, w->scales, q, wscale, w->n * w->num_experts, w->k, sign_mask_of(w->seed),
                               codebook(), reinterpret_cast<cudaStream_t>(stream)));
}

static int fp8_check(int64_t m, int64_t n, int64_t k) {
  if (m < 0 || m > (1ll << 24) || n <= 0 || k <= 0 || k % 32 != 0 || n > (1ll << 30) || k > (1ll << 30))
    return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

TQ_API size_t tq4_1s_linear_fp8_workspace(int64_t m, int64_t n, int64_t k) {
  if (fp8_check(m, n, k) != TQ_OK || m == 0) return 0;
  return align256(static_cast<size_t>(n) * static_cast<size_t>(k) * 2);   // the bf16 weight of the large-m path
}

TQ_API int tq4_1s_linear_fp8(const uint16_t* x, int64_t m, const uint8_t* q, const float* wscale, int64_t n,
                             int64_t k, int32_t flags, uint16_t* y, void* ws, size_t ws_bytes, tq4_stream_t stream) {
  int rc = fp8_check(m, n, k);
  if (rc) return rc;
  if ((flags & ~TQ_WEIGHT_STATIC) != 0) return TQ_ERR_INVALID_ARG;
  if (m == 0) return TQ_OK;
  if (!x || !q || !wscale || !y) return TQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(wscale) || !aligned16(y)) return TQ_ERR_ALIGNMENT;
  int sms = 0;
  if ((rc = check_device(&sms))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t tiles = (n + 127) / 128, KI = (k + 127) / 128;
  if (m <= kSegRows) {
    const int nb = m > 16 ? 2 : 1;
    const int split = choose_decode_split(tiles, KI, sms, nb, true);
    if (split > 0) {
      if (take_injected_failure()) return TQ_ERR_CUDA;
      alignas(64) CUtensorMap tc, tx;
      const bool box3 = (k % 64) == 0;
      if (!map_fp8(&tc, q, n, k) ||
          !(box3 ? map_x3d(&tx, x, m, k, static_cast<uint32_t>(16 * nb), 2 * kFusedMaxIters)
                 : map_bf16(&tx, x, m, k, static_cast<uint32_t>(16 * nb))))
        return TQ_ERR_CUDA;
      DecodeArgs d{};
      d.n = static_cast<int32_t>(n);
      d.k = static_cast<int32_t>(k);
      d.m = static_cast<int32_t>(m);
      d.nb = nb;
      d.row_tiles = static_cast<int32_t>(tiles);
      d.k_iters = static_cast<int32_t>(KI);
      d.split = split;
      d.static_w = (flags & TQ_WEIGHT_STATIC) ? 1 : 0;
      d.test_withhold = withhold_arrival_hook() ? 1 : 0;
      d.fp8 = 1;
      d.x_box3 = box3 ? 1 : 0;
      d.wscale = wscale;
      d.x = x;
      d.y = y;
      return cuda_rc(launch_decode(&tc, &tx, &tc, d, st));
    }
  }
  // large m (or a shape the decode kernel does not take): the bf16 weight in
  // the workspace, then the tensor-core GEMM
  const size_t need = align256(static_cast<size_t>(n) * static_cast<size_t>(k) * 2);
  if (!ws || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  uint16_t* wh = static_cast<uint16_t*>(ws);
  if (launch_fp8_to_bf16(q, wscale, wh, n, k, st) != cudaSuccess) return TQ_ERR_CUDA;
  alignas(64) CUtensorMap tx, tw;
  if (!map_bf16(&tx, x, m, k, 128) || !map_bf16(&tw, wh, n, k, 256)) return TQ_ERR_CUDA;
  const int64_t gt = ((m + 127) / 128) * ((n + 255) / 256);
  const int grid = static_cast<int>(gt < sms ? gt : sms);
  return cuda_rc(launch_gemm_bf16(&tx, &tw, y, static_cast<int32_t>(m), static_cast<int32_t>(n),
                                  static_cast<int32_t>(k), grid, st));
}

// ------------------------------------------------------------------ affine format
static int affine_ok(const tq4_1s_affine_weight* w, bool need_ptrs) {
  if (!w) return TQ_ERR_INVALID_ARG;
  if (w->n <= 0 || w->k <= 0 || (w->k % 64) != 0 || w->reserved != 0) return TQ_ERR_INVALID_ARG;
  if (w->bits != 4 && w->bits != 6 && w->bits != 8) return TQ_ERR_INVALID_ARG;
  if (w->n > (1ll << 30) || w->k > (1ll << 30)) return TQ_ERR_INVALID_ARG;
  if (need_ptrs) {
    if (!w->codes || !w->scales || !w->biases) return TQ_ERR_INVALID_ARG;
    if (!aligned16(w->codes) || !aligned16(w->scales) || !aligned16(w->biases)) return TQ_ERR_ALIGNMENT;
  }
  return TQ_OK;
}

TQ_API int tq4_1s_affine_quantize(const float* W, const tq4_1s_affine_weight* out, tq4_stream_t stream) {
  int rc = affine_ok(out, true);
  if (rc) return rc;
  if (!W) return TQ_ERR_INVALID_ARG;
  if (!aligned16(W)) return TQ_ERR_ALIGNMENT;
  if ((rc = check_device(nullptr))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  return cuda_rc(launch_affine_quantize(W, out->codes, out->scales, out->biases, out->n, out->k, out->bits,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API int tq4_1s_affine_dequantize(const tq4_1s_affine_weight* w, float* W_out, tq4_stream_t stream) {
  int rc = affine_ok(w, true);
  if (rc) return rc;
  if (!W_out) return TQ_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return TQ_ERR_ALIGNMENT;
  if ((rc = check_device(nullptr))) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  return cuda_rc(launch_affine_dequantize(w->codes, w->scales, w->biases, W_out, false, w->n, w->k, w->bits,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API size_t tq4_1s_affine_linear_workspace(int64_t m, const tq4_1s_affine_weight* w) {
  if (m <= 0 || m > (1ll << 24) || affine_ok(w, false) != TQ_OK) return 0;
  return align256(static_cast<size_t>(w->n) * static_cast<size_t>(w->k) * 2);
}

TQ_API int tq4_1s_affine_linear(const uint16_t* x, int64_t m, const tq4_1s_affine_weight* w, uint16_t* y, void* ws,
                                size_t ws_bytes, tq4_stream_t stream) {
  int rc = affine_ok(w, true);
  if (rc) return rc;
  if (m < 0 || m > (1ll << 24)) return TQ_ERR_INVALID_ARG;
  if (m == 0) return TQ_OK;
  if (!x || !y) return TQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TQ_ERR_ALIGNMENT;
  int sms = 0;
  if ((rc = check_device(&sms))) return rc;
  const size_t need = align256(static_cast<size_t>(w->n) * static_cast<size_t>(w->k) * 2);
  if (!ws || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* wh = static_cast<uint16_t*>(ws);
  if (launch_affine_dequantize(w->codes, w->scales, w->biases, wh, true, w->n, w->k, w->bits, st) != cudaSuccess)
    return TQ_ERR_CUDA;
  alignas(64) CUtensorMap tx, tw;
  if (!map_bf16(&tx, x, m, w->k, 128) || !map_bf16(&tw, wh, w->n, w->k, 256)) return TQ_ERR_CUDA;
  const int64_t gt = ((m + 127) / 128) * ((w->n + 255) / 256);
  const int grid = static_cast<int>(gt < sms ? gt : sms);
  return cuda_rc(launch_gemm_bf16(&tx, &tw, y, static_cast<int32_t>(m), static_cast<int32_t>(w->n),
                                  static_cast<int32_t>(w->k), grid, st));
}

static int64_t H_of(const tq4_1s_weight* up) { return up->k; }

static int moe_check(int64_t m, int32_t topk, const tq4_1s_weight* up, const tq4_1s_weight* down, bool ptrs) {
  int rc = weight_ok(up, ptrs);
  if (rc) return rc;
  if ((rc = weight_ok(down, ptrs))) return rc;
  if (m < 0 || topk <= 0 || topk > 64 || m * topk > (1ll << 26)) return TQ_ERR_INVALID_ARG;
  if (up->num_experts != down->num_experts || up->k != down->n || up->n != down->k) return TQ_ERR_INVALID_ARG;
  if (up->num_experts > 4096) return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

TQ_API size_t tq4_1s_moe_workspace(int64_t m, int32_t topk, const tq4_1s_weight* up, const tq4_1s_weight* down) {
  if (moe_check(m, topk, up, down, false) != TQ_OK) return 0;
  if (m == 0) return 0;
  return moe_layout(m, topk, up, down, sms_or_default()).total;
}

// The MoE launch sequence shared by tq4_1s_moe (caller's routing) and
// tq4_1s_moe_logits (router on the device: `logits` non-null, ids and weights
// produced into the workspace).
static int moe_impl(const uint16_t* x, int64_t m, const int32_t* topk_ids, const float* topk_w, const float* logits,
                    int32_t topk, const tq4_1s_weight* up, const tq4_1s_weight* down, uint16_t* y, void* ws,
                    size_t ws_bytes, tq4_stream_t stream) {
  int rc = moe_check(m, topk, up, down, true);
  if (rc) return rc;
  if (m == 0) return TQ_OK;
  if (!x || !y || (logits ? false : (!topk_ids || !topk_w))) return TQ_ERR_INVALID_ARG;
  if (logits && (up->num_experts > 1024 || topk > 32 || topk > up->num_experts))
    return TQ_ERR_INVALID_ARG;   // router limits
  if (!aligned16(x) || !aligned16(y)) return TQ_ERR_ALIGNMENT;
  if (logits ? !aligned16(logits) : (!aligned16(topk_ids) || !aligned16(topk_w))) return TQ_ERR_ALIGNMENT;
  int sms = 0;
  if ((rc = check_device(&sms))) return rc;
  const MoeLayout L = moe_layout(m, topk, up, down, sms);
  if (L.maxseg * L.rt_up * ((H_of(up) + 127) / 128) > INT32_MAX ||
      L.maxseg * L.rt_dn * ((up->n + 127) / 128) > INT32_MAX)
    return TQ_ERR_INVALID_ARG;   // 32-bit iteration space
  if (!ws || ws_bytes < L.total) return TQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return TQ_ERR_ALIGNMENT;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int64_t E = up->num_experts, H = up->k, I = up->n;
  int32_t* offsets = reinterpret_cast<int32_t*>(base + L.offsets);
  int32_t* pairs = reinterpret_cast<int32_t*>(base + L.pairs);
  int4* segs = reinterpret_cast<int4*>(base + L.segs);
  int32_t* nseg = reinterpret_cast<int32_t*>(base + L.nseg);
  int32_t* npv = reinterpret_cast<int32_t*>(base + L.npv);
  uint16_t* xr = reinterpret_cast<uint16_t*>(base + L.xr);
  uint16_t* hr = reinterpret_cast<uint16_t*>(base + L.hr);
  float* zw = reinterpret_cast<float*>(base + L.zw);
  if (logits) {
    topk_ids = reinterpret_cast<const int32_t*>(base + L.ids);
    topk_w = reinterpret_cast<const float*>(base + L.wts);
  }
  cudaError_t e = launch_moe_route(topk_ids, L.P, static_cast<int32_t>(E), offsets, pairs, segs, nseg, L.chunk,
                                   npv, st, logits, topk, reinterpret_cast<int32_t*>(base + L.ids),
                                   reinterpret_cast<float*>(base + L.wts));
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  float* xscale = reinterpret_cast<float*>(base + L.xscale);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + L.h);
  float* hscale = reinterpret_cast<float*>(base + L.hscale);
  // x' of each sorted pair row (x row pairs[r] / topk), rotated by the up
  // projection's signs
  e = launch_rotate_scaled(x, H, pairs, topk, npv, 0, L.P, xr, xscale, sign_mask_of(up->seed), st);
  if (e != cudaSuccess) return TQ_ERR_CUDA;

  alignas(64) CUtensorMap tcu, txr, tcd, thr;
  if (!map_codes(&tcu, up) || !map_bf16(&txr, xr, L.P, H, 16) || !map_codes(&tcd, down) ||
      !map_bf16(&thr, hr, L.P, I, 16))
    return TQ_ERR_CUDA;
  StreamKArgs a{};
  a.n = static_cast<int32_t>(I);
  a.k = static_cast<int32_t>(H);
  a.row_tiles = static_cast<int32_t>(L.rt_up);
  a.k_iters = static_cast<int32_t>((H + 127) / 128);
  a.segs = segs;
  a.nseg_dev = nseg;
  a.nb_max = L.nb_max;   // segments hold at most 16 * nb_max rows (the route's chunk)
  a.scales = up->scales;
  a.codes = up->codes;
  a.xr = xr;
  a.row_scale = xscale;
  a.epoch = next_epoch();
  a.cluster_s = 1;
  a.x_resident = (L.nb_max == 1 && H <= kResidentMaxK) ? 1 : 0;
  a.mode = EPI_UP;
  a.out_a = h;
  a.partials = reinterpret_cast<float*>(base + L.partials);
  a.counters = reinterpret_cast<unsigned long long*>(base + L.cnt_up);
  a.max_tiles = static_cast<int32_t>(L.maxseg * L.rt_up);
  if ((e = launch_streamk(&tcu, &txr, nullptr, a, sms, st)) != cudaSuccess) return TQ_ERR_CUDA;

  // h' = R_down h per sorted pair row
  e = launch_rotate_scaled(h, I, nullptr, 1, npv, 0, L.P, hr, hscale, sign_mask_of(down->seed), st);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  StreamKArgs b = a;
  b.n = static_cast<int32_t>(H);
  b.k = static_cast<int32_t>(I);
  b.row_tiles = static_cast<int32_t>(L.rt_dn);
  b.k_iters = static_cast<int32_t>((I + 127) / 128);
  b.scales = down->scales;
  b.codes = down->codes;
  b.xr = hr;
  b.row_scale = hscale;
  b.x_resident = (L.nb_max == 1 && I <= kResidentMaxK) ? 1 : 0;
  b.epoch = next_epoch();
  b.mode = EPI_DOWN;
  b.out_a = nullptr;
  b.out_f = zw;
  b.pairs = pairs;
  b.topk_w = topk_w;
  b.counters = reinterpret_cast<unsigned long long*>(base + L.cnt_dn);
  b.max_tiles = static_cast<int32_t>(L.maxseg * L.rt_dn);
  if ((e = launch_streamk(&tcd, &thr, nullptr, b, sms, st)) != cudaSuccess) return TQ_ERR_CUDA;
  return cuda_rc(launch_moe_combine(zw, topk_ids, m, topk, H, static_cast<int32_t>(E), y, st));
}

TQ_API int tq4_1s_moe(const uint16_t* x, int64_t m, const int32_t* topk_ids, const float* topk_w, int32_t topk,
                      const tq4_1s_weight* up, const tq4_1s_weight* down, uint16_t* y, void* ws, size_t ws_bytes,
                      tq4_stream_t stream) {
  if (!topk_ids || !topk_w) {
    const int rc = moe_check(m, topk, up, down, true);
    return rc ? rc : (m == 0 ? TQ_OK : TQ_ERR_INVALID_ARG);
  }
  return moe_impl(x, m, topk_ids, topk_w, nullptr, topk, up, down, y, ws, ws_bytes, stream);
}

TQ_API int tq4_1s_moe_logits(const uint16_t* x, int64_t m, const float* logits, int32_t topk,
                             const tq4_1s_weight* up, const tq4_1s_weight* down, uint16_t* y, void* ws,
                             size_t ws_bytes, tq4_stream_t stream) {
  if (!logits) {
    const int rc = moe_check(m, topk, up, down, true);
    return rc ? rc : (m == 0 ? TQ_OK : TQ_ERR_INVALID_ARG);
  }
  return moe_impl(x, m, nullptr, nullptr, logits, topk, up, down, y, ws, ws_bytes, stream);
}

TQ_API int tq4_1s_router_topk(const float* logits, int64_t m, int32_t num_experts, int32_t topk, int32_t* ids,
                              float* weights, tq4_stream_t stream) {
  if (m < 0 || num_experts <= 0 || num_experts > 1024 || topk <= 0 || topk > 32 || topk > num_experts ||
      m * num_experts > (1ll << 40))
    return TQ_ERR_INVALID_ARG;
  if (m == 0) return TQ_OK;
  if (!logits || !ids || !weights) return TQ_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc) return rc;
  if (take_injected_failure()) return TQ_ERR_CUDA;
  return cuda_rc(launch_router(logits, m, num_experts, topk, ids, weights, reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API int tq4_1s_moe_route(const int32_t* topk_ids, int64_t m, int32_t topk, int32_t num_experts, int32_t* offsets,
                            int32_t* pairs, tq4_stream_t stream) {
  if (m < 0 || topk <= 0 || num_experts <= 0 || num_experts > 4096 || m * topk > (1ll << 26))
    return TQ_ERR_INVALID_ARG;
  if (!topk_ids || !offsets || !pairs) return TQ_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc) return rc;
  return cuda_rc(launch_moe_route(topk_ids, m * topk, num_experts, offsets, pairs, nullptr, nullptr, kSegRows,
                                  nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

TQ_API int tq4_1s_debug_hook(int what, int64_t value) {
  switch (what) {
    case TQ_HOOK_FAIL_NEXT_CALLS:
      if (value < 0) return TQ_ERR_INVALID_ARG;
      g_fail_next.store(value, std::memory_order_relaxed);
      return TQ_OK;
    case TQ_HOOK_WAIT_NS: {
      if (value < 0) return TQ_ERR_INVALID_ARG;
      const int rc = check_device(nullptr);
      if (rc) return rc;
      const unsigned long long ns = value == 0 ? TQ_WAIT_NS_DEFAULT : static_cast<unsigned long long>(value);
      return cudaMemcpyToSymbol(g_wait_ns, &ns, sizeof(ns)) == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
    }
    case TQ_HOOK_WITHHOLD_ARRIVAL:
      if (value != 0 && value != 1) return TQ_ERR_INVALID_ARG;
      g_withhold.store(static_cast<int>(value), std::memory_order_relaxed);
      return TQ_OK;
    default:
      return TQ_ERR_INVALID_ARG;
  }
}

TQ_API uint64_t tq4_1s_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

TQ_API int tq4_1s_get_status(tq4_stream_t stream, int32_t* status) {
  if (!status) return TQ_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return TQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  *status = v;
  return TQ_OK;
}
