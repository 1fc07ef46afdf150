// Internal declarations shared by the library's translation units.
#pragma once
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "tq4_common.cuh"

namespace tq4 {

// Kernel attributes (dynamic shared-memory size, carveout) belong to each
// device's context: `set` runs once per device, and again after a failure.
// Two threads that race on the first call both run it (it is idempotent).
template <typename Set>
cudaError_t once_per_device(std::atomic<uint64_t>& done, Set set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = uint64_t(1) << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = set();
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// The fp32 codebook handed to kernels by value (kernel parameter space).
struct CodebookF32 {
  float levels[16];       // ascending, levels[15 - j] == -levels[j]
  float thresholds[16];   // 15 used: midpoints of adjacent levels
};

// Count of kernel launches issued by the library (tq4_1s_launch_count).
void note_launches(int n);

// Test hooks (tq4_1s_debug_hook): a pending injected failure makes the next
// launching call return TQ_ERR_CUDA before it launches anything; the
// withhold flag is copied into decode launches.
bool take_injected_failure();
bool withhold_arrival_hook();

// Host-side codebook computation (Lloyd iteration), run once per process.
const CodebookF32& codebook();

// Host helpers of the entry points (tq4_api.cu): the current device's check
// (compute capability 10.0; SM count cached per device) and cached TMA tensor
// maps -- the codes plane [E][n][k/2] (box 64 B x 128 rows, 64-byte swizzle),
// a 16-bit [rows][cols] matrix (box 64 x box_rows, 128-byte swizzle) and
// the same viewed as [cols/64][rows][64] (box 64 x 32 x 2 kFusedMaxIters).
int check_device(int* sms_out);
bool map_codes(CUtensorMap* m, const tq4_1s_weight* w);
bool map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows);
bool map_x3(CUtensorMap* m, const void* base, int64_t rows, int64_t cols);
// x [rows][cols] (cols % 64 == 0) viewed as [cols/64][rows][64] 16-bit, box 64 x
// box_rows x box_chunks, 128-byte swizzle.
bool map_x3d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows, uint32_t box_chunks);

// One segment of rows of the rotated activations multiplied by one expert:
// x = expert, y = first row, z = row count (<= 16 * nb_max <= kSegRows),
// w unused.
constexpr int kSegRows = 32;

// One tensor of a batched quantize launch: rows x k (k % 32 == 0), its sign
// mask, input W (fp32 or bf16, the batch's dtype) and output planes.
struct QuantItem {
  const void* W;
  uint8_t* codes;
  uint16_t* scales;
  int64_t rows, k;
  uint32_t mask;
};
cudaError_t launch_quantize_batch(const QuantItem* items, int count, int dtype, const CodebookF32& cb,
                                  cudaStream_t st);
cudaError_t launch_quantize(const void* W, int dtype, uint8_t* codes, uint16_t* scales, int64_t rows, int64_t k,
                            uint32_t mask, const CodebookF32& cb, cudaStream_t st);
cudaError_t launch_dequantize_f32(const uint8_t* codes, const uint16_t* scales, float* out, int64_t rows, int64_t k,
                                  uint32_t mask, const CodebookF32& cb, cudaStream_t st);
cudaError_t launch_dequantize_bf16(const uint8_t* codes, const uint16_t* scales, uint16_t* out, int64_t rows,
                                   int64_t k, uint32_t mask, const CodebookF32& cb, cudaStream_t st);
// The fp8-resident cache: TQ4_1S rows -> E4M3 codes [rows][k] + fp32 row
// scales, and the cache -> bf16 weight (large-m path of the fp8 linear).
cudaError_t launch_to_fp8(const uint8_t* codes, const uint16_t* scales, uint8_t* q, float* wscale, int64_t rows,
                          int64_t k, uint32_t mask, const CodebookF32& cb, cudaStream_t st);
cudaError_t launch_fp8_to_bf16(const uint8_t* q, const float* wscale, uint16_t* out, int64_t rows, int64_t k,
                               cudaStream_t st);
// The MLX-style affine format: fp32 rows -> bit-stream codes + bf16
// scales/biases per group of 64, and back (fp32 or bf16 out).
cudaError_t launch_affine_quantize(const float* W, uint8_t* codes, uint16_t* scales, uint16_t* biases, int64_t rows,
                                   int64_t k, int bits, cudaStream_t st);
cudaError_t launch_affine_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, void* out,
                                     bool bf16_out, int64_t rows, int64_t k, int bits, cudaStream_t st);
// Activation rotation for the stream-K GEMM: x' = r H diag(s) x per 32-slice
// of each row, scaled by a per-row power of two 2^-e and rounded to fp16
// [rows][k]; row_scale[row] = 2^e.  Row r reads x row
// gather[r] / topk when a gather list is given, else row r.  Rows at or past
// the valid count (rows_valid_dev when non-null, else rows_valid_host) are
// not written.
cudaError_t launch_rotate_scaled(const uint16_t* x, int64_t k, const int32_t* gather, int32_t topk,
                                 const int32_t* rows_valid_dev, int64_t rows_valid_host, int64_t rows_alloc,
                                 uint16_t* xr, float* row_scale, uint32_t mask, cudaStream_t st);
// Routing: offsets, stably bucketed pairs, segment list and counts.  With
// `logits` (fp32 [m][num_experts], m = npairs / topk) the router runs first in
// the same kernel and writes ids_out / w_out ([m][topk]), which the routing
// then reads; otherwise `ids` is the caller's.
cudaError_t launch_moe_route(const int32_t* ids, int64_t npairs, int32_t num_experts, int32_t* offsets,
                             int32_t* pairs, int4* segs, int32_t* nseg, int32_t chunk, int32_t* npairs_valid,
                             cudaStream_t st, const float* logits = nullptr, int32_t topk = 1,
                             int32_t* ids_out = nullptr, float* w_out = nullptr);
// The router alone: ids/w [m][topk] from fp32 logits [m][num_experts]
// (num_experts <= 1024, topk <= 32).
cudaError_t launch_router(const float* logits, int64_t m, int32_t num_experts, int32_t topk, int32_t* ids, float* w,
                          cudaStream_t st);
cudaError_t launch_moe_combine(const float* zw, const int32_t* ids, int64_t m, int32_t topk, int64_t h,
                               int32_t num_experts, uint16_t* y, cudaStream_t st);

// ---------------------------------------------------------------- stream-K
enum EpilogueMode : int32_t { EPI_DENSE = 0, EPI_UP = 1, EPI_DOWN = 2 };

struct StreamKArgs {
  int32_t n, k;              // rows / columns of one expert's weight
  int32_t row_tiles;         // ceil(n / 128)
  int32_t k_iters;           // ceil(k / 128)
  int32_t nseg_host;         // segment count when segs == nullptr (dense): ceil(m / kSegRows)
  int32_t m_host;            // dense row count
  int32_t nb_max;            // max 16-row blocks per segment (1 or 2): accumulator layout
  const int4* segs;          // device segment list (MoE) or nullptr
  const int32_t* nseg_dev;   // device segment count (MoE) or nullptr
  const uint16_t* scales;    // [E][n][k/16]
  const uint8_t* codes;      // [E][n][k/2] (read by the exact fallback of the epilogue only)
  const uint16_t* xr;        // x' fp16 [rows][k] in memory (TMA-fed and grouped modes); nullptr in fused mode
  const float* row_scale;    // x' row r holds x'_r * 2^-e_r; row_scale[r] = 2^e_r (TMA-fed mode)
  const uint16_t* x_raw;     // fused mode (dense, m <= kSegRows, <= kFusedMaxIters iterations per CTA):
                             // raw bf16 x [m][k], rotated by the kernel itself; nullptr otherwise
  uint32_t x_sign[16];       // fused mode: the weight's sign mask as XOR words on bf16 pairs --
                             // word i flips bit 15 / bit 31 where sign i*2 / i*2+1 is negative
  uint32_t epoch;            // tag of this launch in the tile counters (never 0)
  int32_t cluster_s;         // >= 2: fused split-K mode -- grid = tiles * cluster_s, one cluster per
                             // tile, partials reduced through distributed shared memory; else 1
  int32_t x_box3;            // cluster mode with k % 64 == 0: x arrives as one 3-D box (tm_x3)
  int32_t x_resident;        // grouped mode, segments of <= 16 rows, k <= kResidentMaxK: a segment's
                             // x' for all of k is loaded once into shared memory (no per-iteration x')
  int32_t mode;              // EpilogueMode
  uint16_t* out_a;           // dense: y [m][n]; up: h = relu(u)^2 [P][n] (bf16)
  float* out_f;              // down: z*w [m*topk][n]
  const int32_t* pairs;      // MoE: flat slot index of each sorted row
  const float* topk_w;       // MoE: router weights (flat)
  float* partials;           // [grid][2][128][kSegRows]
  unsigned long long* counters;   // [tiles]: (epoch << 32) | arrivals
  int32_t max_tiles;         // capacity of counters
};

// Iterations per CTA up to which the dense kernel can rotate x in its
// prologue (one pipeline stage per iteration, no stage reuse).
constexpr int kFusedMaxIters = 8;

// Largest k whose 16-row x' (fp16) fits the stream-K kernel's B tiles at once.
constexpr int kResidentMaxK = 3072;

// A fresh counter tag for each stream-K launch.
uint32_t next_epoch();

// The sign mask as XOR words over bf16 pairs (StreamKArgs::x_sign).
inline void sign_xor_words(uint32_t mask, uint32_t (&w)[16]) {
  for (int i = 0; i < 16; ++i)
    w[i] = (((mask >> (2 * i)) & 1u) << 15) | (((mask >> (2 * i + 1)) & 1u) << 31);
}

// Bytes of dynamic shared memory the stream-K kernel uses.
size_t streamk_smem_bytes();
// How many clusters of s stream-K CTAs can be resident at once (0 on error).
int streamk_max_clusters(int s);
// Cluster split-K factor for a fused dense launch of `tiles` row tiles and
// k_iters k iterations: the largest s in [2, 8] with s <= k_iters, at most
// kFusedMaxIters iterations per CTA, tiles * s <= sms and all clusters
// resident at once; 1 if none fits.
int choose_cluster_split(int64_t tiles, int64_t k_iters, int sms);

// tm_x: the x' (TMA-fed) or x (fused) tiles, box 64 x 16; tm_x3 (cluster
// split-K mode, else may be null): x viewed as [k/64][m][64], box 64 x 32 x
// 2*kFusedMaxIters.
cudaError_t launch_streamk(const void* tm_codes, const void* tm_x, const void* tm_x3, const StreamKArgs& a, int grid,
                           cudaStream_t st);

// ---------------------------------------------------------------- decode
// The decode-block kernel: m <= 32 tokens, one CTA per (128-row tile, k
// range of at most kFusedMaxIters iterations), `split` CTAs per tile in a
// cluster.  tm_codes: the codes plane (map_codes).
struct DecodeArgs {
  int32_t n, k, m, nb;          // rows, columns, tokens, 16-token blocks (1 or 2)
  int32_t row_tiles, k_iters;   // ceil(n / 128), ceil(k / 128)
  int32_t split;                // CTAs per row tile (>= 1, <= k_iters)
  int32_t static_w;             // the weight may be read before the dependency wait
  int32_t test_withhold;        // test hook: rotation warp 7 never reports (its bounded waiters run out)
  int32_t fp8;                  // the weight is the fp8 cache (codes = E4M3 [n][k], wscale [n]), else TQ4_1S
  int32_t scales_tma;           // TQ4_1S with k % 128 == 0: the scales come by TMA (tm_scales), else by loads
  int32_t x_box3;               // k % 64 == 0: tm_x views x as [k/64][m][64] (one 3-D box per CTA), else 2-D
  const float* wscale;          // fp8 cache: one fp32 scale per row
  const uint16_t* x;            // bf16 [m][k]
  const uint16_t* scales;       // [n][k/16] fp16 bits
  uint16_t* y;                  // bf16 [m][n]
  uint32_t x_sign[16];          // sign mask as XOR words on bf16 pairs
  uint32_t sign_bits;           // the same mask, bit i = sign of element i of a 32-slice
};
// tm_codes: the codes plane (or the fp8 cache); tm_x: x [m][k] bf16, box 64 x 16 nb,
// 128-byte swizzle (a.x_box3: the map_x3d view, box 64 x 16 nb x 16); tm_scales: the scales [n][k/16], box 64 x 128, 128-byte
// swizzle (read only when a.scales_tma).
cudaError_t launch_decode(const void* tm_codes, const void* tm_x, const void* tm_scales, const DecodeArgs& a,
                          cudaStream_t st);
// The split for a decode launch of `tiles` row tiles (0: the kernel does not fit).
int choose_decode_split(int64_t tiles, int64_t k_iters, int sms, int nb, bool f8 = false);
size_t decode_smem_bytes(int nb, bool f8);

// ---------------------------------------------------------------- GEMM
// y[m][n] = bf16( x[m][k] * w[n][k]^T ), bf16 operands via TMA tensor maps.
cudaError_t launch_gemm_bf16(const void* tm_x, const void* tm_w, uint16_t* y, int32_t m, int32_t n, int32_t k,
                             int grid, cudaStream_t st);
size_t gemm_smem_bytes();

}  // namespace tq4
