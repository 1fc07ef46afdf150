// Stream-K dequant-GEMM for small m (decode blocks of 16 tokens, MoE expert
// groups) on sm_100a.
//
// Computes D[n][j] = sum_k w_n[n][k] * x'[j][k] for 128-row tiles of one
// expert's weight, where w_n = c[code] * d are the rotated-domain levels
// ("What Config-I means": 16-level Lloyd-Max codes, two half-block scales)
// and x' = R x is the activation rotated per 32-slice (route B: rotating the
// activations instead of inverse-rotating the weights, which is equivalent
// because R is orthogonal).  x' is fp16, each row scaled by a power of two
// 2^-e that puts its largest possible value in [2^13, 2^14); the levels are
// fp16(c[code] * 256 * d).  Both operands fp16 (relative rounding 2^-11,
// well inside the layer's tolerance), fp32 accumulation; the epilogue
// multiplies by 2^e / 256, which is exact.
//
// x' comes from one of two places.  TMA-fed mode: the rotation kernel wrote
// it to global memory (row_scale = 2^e per row) and the producer stages it
// with TMA.  Fused mode (a dense layer of at most kSegRows rows whose CTAs
// run at most kFusedMaxIters iterations each, so every iteration has a stage
// of its own): the producer stages the raw bf16 x tiles into the B regions
// first, then the codes; the dequant and epilogue warps take each row's
// maximum over the k range this CTA covers and rotate the tiles in place
// while the codes are in flight -- no second launch, no x' round trip
// through memory.
//
// Per 128-row x 128-k iteration of a tile:
//   warp 0      TMA: codes tile [128 x 64 B] (64-byte swizzle) and, in
//               TMA-fed mode, the x' tiles [rows x 128 k] (128-byte swizzle)
//               into a stage;
//   warps 2-17  four dequant warpgroups (round-robin iterations), thread =
//               weight row: 16 B of codes + 8 scales -> 128 levels.  Each
//               code byte (two nibbles) indexes a shared-memory table of
//               fp16 level pairs {256 c[lo], 256 c[hi]}, one copy per lane so
//               a warp's 32 lookups hit 32 banks, and one packed fp16 multiply
//               by {d, d} scales the pair.  The levels go to tensor memory
//               with tcgen05.st (the MMA A operand), as two 64-k halves
//               signalled separately;
//   warps 1, 22-24  lane 0: one MMA issuer per dequant group: 4 tcgen05.mma
//               per half (M=128, N=16*nb, K=16, A from tensor memory, B from
//               shared memory) into the group's own accumulator --
//               single-thread issue costs ~66-98 cycles per small-N
//               instruction, so the four groups issue in parallel;
//   warps 18-21 epilogue, thread = row: tcgen05.ld of the accumulators, the
//               groups summed, scaled back, the mode's store.
// The flattened (segment, row tile, k iteration) space is split evenly over
// the CTAs (stream-K).  A tile split between CTAs is finished by whichever
// contributor arrives last on the tile's counter: it sums all contributors'
// fp32 partials in CTA order (deterministic) and runs the epilogue, so no
// CTA ever waits on another.  Cluster split-K mode (fused mode with a grid of
// tiles x s CTAs, s per tile): the even split gives each CTA 1/s of one
// tile's k range; the s CTAs of a tile form a thread-block cluster, each
// owns 1/s of the tile's rows: every CTA stores each row of its partial into
// the owner's shared memory (distributed shared memory), and after one
// cluster barrier each owner sums its rows over the s partials in rank order
// -- deterministic, no partials or counters in global memory.
#include <atomic>
#include <chrono>
#include <mutex>
#include <random>

#include "tq4_internal.h"

namespace tq4 {
namespace {

constexpr int kDequantGroups = 4;
constexpr int kFirstDequantWarp = 2;
constexpr int kFirstEpilogueWarp = kFirstDequantWarp + 4 * kDequantGroups;
// MMA-issuing threads: lane 0 of warp 1 serves dequant group 0, lane 0 of
// warps 22, 23, 24 groups 1, 2, 3 (the four land on four different SMSPs).
constexpr int kFirstIssuerWarp = kFirstEpilogueWarp + 4;
constexpr int kThreads = (kFirstIssuerWarp + kDequantGroups - 1) * 32;
__device__ __forceinline__ int issuer_group(int warp) { return warp == 1 ? 0 : warp - kFirstIssuerWarp + 1; }
// fused mode: the dequant and epilogue warps rotate x before their own work
constexpr int kPrologueThreads = (kFirstEpilogueWarp + 4 - kFirstDequantWarp) * 32;
constexpr int kStages = 12;
constexpr int kCodesBytes = 128 * 64;    // 128 rows x 128 k codes
constexpr int kXHalfBytes = kSegRows * 128;   // up to 32 token rows x 64 k of fp16 x' (128-B swizzle span)
constexpr int kXBytes = 2 * kXHalfBytes; // two k-halves
constexpr int kStageBytes = kCodesBytes + kXBytes;
// Shared memory: the codes of the stages [kStages][kCodesBytes], then the B
// tiles [kStages][kXBytes] (contiguous, so one TMA box can fill several),
// then the level-pair table.
constexpr int kBOff = kStages * kCodesBytes;
// Cluster split-K: each CTA receives the partial rows it reduces into the
// codes of stages kFusedMaxIters.. (never loaded in fused mode):
// [source rank][32 tokens][rows per CTA] floats.
constexpr int kRedOff = kFusedMaxIters * kCodesBytes;
constexpr int kLutBytes = 256 * 32 * 4;  // fp16 level-pair table, one copy per lane
constexpr int kTmemCols = 512;
// Tensor memory: columns [0, 256) hold the accumulators, [256, 512) the four
// A stages (one per dequant group, 64 columns = 128 k of fp16 levels).  With
// 16 nb columns per group accumulator (nb = 16-token blocks per segment),
// so 64 nb columns per set of four, and 256 / (64 nb) sets (4 or 2)
// rotate between tile portions.
constexpr int kAccRegion = 256;
constexpr int kACol0 = kAccRegion;
constexpr int kAColsPerStage = 64;
static_assert(kACol0 + kDequantGroups * kAColsPerStage <= kTmemCols, "tensor memory budget");
static_assert(kFusedMaxIters <= kStages, "fused mode gives each iteration its own stage");
// fp16 levels carry a factor 256 (2^8): with it, half-block scales d from
// ~2e-6 up to 65504 / fp16(256 * max level) ~ 93.6 give normal, finite fp16
// levels.  A larger scale overflows its levels, which makes the row's sums
// non-finite; the epilogue then recomputes that row's portion exactly
// (exact_row_portion).
constexpr float kLevelScale = 256.0f;

struct SharedState {
  uint64_t full[kStages];      // the stage's codes and x' tiles landed
  uint64_t done[kStages];      // the stage may be refilled: the MMAs of the iteration that used it completed
                               // (x' in the stage), or its four dequant warps read its codes (resident x')
  uint64_t afull[kDequantGroups][2];   // a half A stage (64 k) holds fresh levels (128 arrivals)
  uint64_t afree[kDequantGroups][2];   // the MMAs reading a half A stage completed
  uint64_t dfull[4];           // all four groups finished a portion (4 arrivals), per set
  uint64_t dempty[4];          // the epilogue drained an accumulator set (128 arrivals)
  uint64_t issuer_done[kDequantGroups];
  uint64_t xready;             // fused mode: every stage's x' tile is written (one arrival per prologue warp)
  uint64_t xland[kFusedMaxIters];   // fused mode: the raw x tiles of a stage landed (TMA)
  uint64_t rland;              // resident mode: the current segment's x' (all of k) landed
  uint64_t rfree;              // resident mode: the MMAs reading the previous segment's x' completed (4 commits)
  float row_scale[kSegRows];   // fused mode: 2^e of each row
  unsigned row_max[kSegRows];  // fused mode: max |x| of each row over this CTA's k range (float bits)
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int epi_ok[2];
  int x_ok;                    // fused mode: the epilogue saw xready complete
};

struct Seg {
  int e, row0, count;
};

__device__ __forceinline__ Seg get_seg(const StreamKArgs& a, int s) {
  if (a.segs) {
    const int4 v = __ldcg(a.segs + s);
    return {v.x, v.y, v.z};
  }
  const int r0 = s * kSegRows;
  return {0, r0, min(kSegRows, a.m_host - r0)};
}

// floor(a / b) for 0 <= a < 2^62, 0 < b < 2^31: an fp64 estimate, then an
// exact integer correction (the estimate is off by at most one) -- far
// cheaper than a 64-bit integer division.
__device__ __forceinline__ int floordiv(long long a, int b) {
  long long q = static_cast<long long>(static_cast<double>(a) * (1.0 / static_cast<double>(b)));
  if (q * b > a) --q;
  else if ((q + 1) * b <= a) ++q;
  return static_cast<int>(q);
}
// First iteration of CTA c when T iterations are split over G CTAs:
// floor(c T / G) = c q + floor(c r / G) with q = T / G, r = T % G; c r < G^2
// fits 32 bits for any grid below 2^16 CTAs.
__device__ __forceinline__ int range_begin(int c, int T, int G) {
  const unsigned q = static_cast<unsigned>(T) / static_cast<unsigned>(G);
  const unsigned r = static_cast<unsigned>(T) - q * static_cast<unsigned>(G);
  return static_cast<int>(static_cast<unsigned>(c) * q +
                          static_cast<unsigned>(c) * r / static_cast<unsigned>(G));
}
// The CTA whose range holds iteration i: ceil((i + 1) G / T) - 1.
__device__ __forceinline__ int owner_of(int i, int T, int G) {
  return floordiv(static_cast<long long>(i + 1) * G + T - 1, T) - 1;
}

// Position of an iteration in the (segment, row tile, k iteration) space,
// advanced incrementally so the loops do no integer division.
struct Cursor {
  int tile, kit, sgi, rt;
  __device__ __forceinline__ void init(int it, int KI, int RT) {
    tile = it / KI;
    kit = it - tile * KI;
    sgi = tile / RT;
    rt = tile - sgi * RT;
  }
  __device__ __forceinline__ void advance(int n, int KI, int RT) {
    kit += n;
    while (kit >= KI) {
      kit -= KI;
      ++tile;
      if (++rt == RT) {
        rt = 0;
        ++sgi;
      }
    }
  }
};

// Bounded wait that ignores the abort flag (used while winding down).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(addr, parity)) {
    if (global_timer() - t0 > TQ_WAIT_NS) {
      raise_status(TQ_DEV_TIMEOUT);
      return;
    }
  }
}

// Lane 0 waits (bounded); the outcome is broadcast so the whole warp takes
// the same branch before any .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abortp) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abortp) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Dequantize one half-block: 16 codes in q0 (elements 0..7) and q1 (8..15),
// one nibble each, low nibble first; dd = {d, d} in fp16.  Each code byte
// indexes the lane's copy of the level-pair table (`lut_lane` = byte address
// of the copy's entry 0; entries are 128 bytes apart); out[i] = fp16 pair
// {element 2i, element 2i+1} = fp16(256 c[code] * d) each.
__device__ __forceinline__ void dequant_half(uint32_t q0, uint32_t q1, uint32_t dd, uint32_t lut_lane,
                                             uint32_t* out) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const uint32_t q = w ? q1 : q0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t idx = prmt(q, 0u, 0x4440u + static_cast<uint32_t>(b));   // byte b, zero-extended
      uint32_t v;   // (the table is written once, before the kernel's first barrier)
      asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(lut_lane + idx * 128u));
      uint32_t r;
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(dd));
      out[4 * w + b] = r;
    }
  }
}

// 32-point Sylvester butterfly on a register array (stages h = 1..16).
__device__ __forceinline__ void fwht32_regs_sk(float (&a)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (!(j & h)) {
        const float x = a[j], y = a[j + h];
        a[j] = __fadd_rn(x, y);
        a[j + h] = __fsub_rn(x, y);
      }
    }
  }
}

__device__ __forceinline__ float relu2_bf16(float v) {
  const float r = fmaxf(v, 0.0f);
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(r, r)));
}

// The per-mode store of 16 tokens [j0, j0 + 16) of one finished tile row
// (thread = weight row `row`).
__device__ __forceinline__ void epilogue_store(const StreamKArgs& a, const float (&v)[16], int j0, int row,
                                               const Seg& sg) {
  const int cnt = sg.count - j0;
  if (row >= a.n) return;
  if (a.mode == EPI_DENSE) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cnt)
        a.out_a[static_cast<int64_t>(sg.row0 + j0 + j) * a.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
  } else if (a.mode == EPI_UP) {
    // h = bf16(relu(u)^2) per sorted pair row: the down projection's input
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cnt)
        a.out_a[static_cast<int64_t>(sg.row0 + j0 + j) * a.n + row] =
            __bfloat16_as_ushort(__float2bfloat16_rn(relu2_bf16(v[j])));
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < cnt) {
        const int p = __ldcg(a.pairs + sg.row0 + j0 + j);
        a.out_f[static_cast<int64_t>(p) * a.n + row] = __fmul_rn(__ldcg(a.topk_w + p), v[j]);
      }
    }
  }
}

struct LevelTable {
  uint32_t h[16];    // fp16 bits of 256 * levels[0..15]
};

// The exact path for one weight row of one tile portion, taken when the
// row's sums came out non-finite: a level fp16(256 c) * d overflows fp16
// for a half-block scale d above ~93.6.  Recomputes the sums of tokens
// j0 .. j0 + ntok - 1 (ntok <= 16) over the portion's columns [kc0, kc1) on
// the CUDA cores with fp32 levels 256 c d, in the accumulator's domain:
// out[j] = sum_k 256 c[code_k] d_k x'[j0 + j][k].  x' comes from memory
// (xg: row j at xg + j * k_row) or, in fused mode (xg == nullptr), from the
// CTA's B tiles (xs: local iteration li's tile at xs + li * kXBytes, as the
// prologue left it: row j at 128 j in each 64-k half, chunk c at c ^ (j & 7)),
// with column kc0 in local iteration li0.  Tokens past ntok are zero.
__device__ __noinline__ void exact_row_portion(const uint8_t* crow, const uint16_t* srow, int kc0, int kc1,
                                               const uint16_t* xg, int k_row, const uint8_t* xs, int li0, int j0,
                                               int ntok, const uint32_t* lvl, float* out) {
  for (int j = 0; j < 16; ++j) out[j] = 0.0f;
  for (int kk = kc0; kk < kc1; ++kk) {
    const uint32_t b = crow[kk >> 1];
    const uint32_t code = (kk & 1) ? (b >> 4) : (b & 15u);
    const float w = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(lvl[code]))),
                              __half2float(__ushort_as_half(srow[kk >> 4])));
    const int li = li0 + (kk >> 7) - (kc0 >> 7), e = kk & 127, e64 = e & 63;
    for (int j = 0; j < ntok; ++j) {
      const int jj = j0 + j;
      const uint16_t xb =
          xg ? xg[static_cast<int64_t>(jj) * k_row + kk]
             : *reinterpret_cast<const uint16_t*>(xs + li * kXBytes + (e >> 6) * kXHalfBytes + jj * 128 +
                                                  ((((e64 >> 3) ^ (jj & 7))) << 4) + (e64 & 7) * 2);
      out[j] = __fmaf_rn(w, __half2float(__ushort_as_half(xb)), out[j]);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    streamk_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_x3, const StreamKArgs a,
                   const __grid_constant__ LevelTable lt) {
  __shared__ SharedState sh;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* lut = smem + kStages * kStageBytes;
  auto codes_of = [&](int st) { return smem + st * kCodesBytes; };
  auto btile_of = [&](int st) { return smem + kBOff + st * kXBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Grouped (MoE) mode reads the routing kernel's segment list right away;
  // the dense mode defers the dependency wait to the roles that need it.
  if (a.segs) pdl_wait();
  const int nseg = a.segs ? __ldcg(a.nseg_dev) : a.nseg_host;
  const int KI = a.k_iters;
  if (a.segs && nseg * a.row_tiles > a.max_tiles) {
    // more segments than the counters were sized for: the routing step is
    // inconsistent; nothing is computed
    if (threadIdx.x == 0) raise_status(TQ_DEV_BAD_ROUTING);
    return;
  }
  const int T = nseg * a.row_tiles * KI;   // < 2^31 (checked by the host)
  const int G = gridDim.x;
  const int it_begin = range_begin(blockIdx.x, T, G);
  const int it_end = range_begin(blockIdx.x + 1, T, G);
  const int cnt = it_end - it_begin;
  if (cnt <= 0) {
    // (the host never gives a cluster-mode CTA an empty range; if one had
    // one, it would still meet its cluster's barrier)
    if (a.cluster_s > 1) cluster_sync_all();
    return;
  }
  const bool fused = a.x_raw != nullptr;
  // accumulator layout (see kAccRegion): width per group, number of sets
  const int acc_w = 16 * a.nb_max;
  const int nsets = kAccRegion / (kDequantGroups * acc_w);
  const int tile_begin = it_begin / KI, tile_last = (it_end - 1) / KI;
  const int nportions = tile_last - tile_begin + 1;

  if (warp == 0) {
    // the barriers, spread over the lanes of warp 0
    constexpr int kBars = 2 * kStages + 4 * kDequantGroups + 12 + 1 + kFusedMaxIters + 2;
    for (int i = lane; i < kBars; i += 32) {
      if (i < kStages) mbar_init(&sh.full[i], 1);
      else if (i < 2 * kStages) mbar_init(&sh.done[i - kStages], a.x_resident ? 4 : 1);
      else if (i < 2 * kStages + 2 * kDequantGroups) {
        const int g = i - 2 * kStages;
        mbar_init(&sh.afull[g >> 1][g & 1], 128);
      } else if (i < 2 * kStages + 4 * kDequantGroups) {
        const int g = i - 2 * kStages - 2 * kDequantGroups;
        mbar_init(&sh.afree[g >> 1][g & 1], 1);
      } else if (i < 2 * kStages + 4 * kDequantGroups + 4) {
        mbar_init(&sh.dfull[i - 2 * kStages - 4 * kDequantGroups], kDequantGroups);
      } else if (i < 2 * kStages + 4 * kDequantGroups + 8) {
        mbar_init(&sh.dempty[i - 2 * kStages - 4 * kDequantGroups - 4], 128);
      } else if (i < 2 * kStages + 4 * kDequantGroups + 12) {
        mbar_init(&sh.issuer_done[i - 2 * kStages - 4 * kDequantGroups - 8], 1);
      } else if (i == 2 * kStages + 4 * kDequantGroups + 12) {
        mbar_init(&sh.xready, kPrologueThreads / 32);
      } else if (i < 2 * kStages + 4 * kDequantGroups + 13 + kFusedMaxIters) {
        mbar_init(&sh.xland[i - 2 * kStages - 4 * kDequantGroups - 13], 1);
      } else if (i == 2 * kStages + 4 * kDequantGroups + 13 + kFusedMaxIters) {
        mbar_init(&sh.rland, 1);
      } else {
        mbar_init(&sh.rfree, kDequantGroups);
      }
    }
    static_assert(kSegRows == 32, "one row maximum per lane");
    sh.row_max[lane] = 0u;
    if (lane == 0) {
      sh.abort_flag = 0;
      sh.last_flag = 0;
    }
    fence_mbar_init();
  }
  {
    // table entry b (a code byte) of lane l's copy, at byte 128 b + 4 l:
    // {256 c[b & 15], 256 c[b >> 4]}
    uint32_t* lw = reinterpret_cast<uint32_t*>(lut);
    for (int i = threadIdx.x - 64; warp >= 2 && i < 256 * 32; i += kThreads - 64) {
      const int b = i >> 5;
      lw[i] = lt.h[b & 15] | (lt.h[b >> 4] << 16);
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    if (!fused) {
      tma_prefetch_desc(&tm_x);
    }
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  volatile int* abortp = &sh.abort_flag;

  // In fused mode the kernel before this one may have written anything, the
  // weight included: the prologue warps wait for it before any global read
  // (the producer does the same).
  if (fused && warp >= kFirstDequantWarp && warp < kFirstEpilogueWarp + 4) pdl_wait();
  // The dequant warps' first scale loads go out before the prologue, so their
  // latency overlaps it; in fused mode a group has at most two iterations and
  // loads the scales of both, before the weight stream starts.
  uint32_t first_raw[4] = {0u, 0u, 0u, 0u}, second_raw[4] = {0u, 0u, 0u, 0u};
  if (warp >= kFirstDequantWarp && warp < kFirstEpilogueWarp) {
    const int wg = (warp - kFirstDequantWarp) >> 2;
    const int t = (warp & 3) * 32 + lane;
    const int kh16 = a.k / 16;
    auto load_scales = [&](int li, uint32_t (&raw)[4]) {
      Cursor c0;
      c0.init(it_begin + li, KI, a.row_tiles);
      const int row = c0.rt * 128 + t;
      if (row < a.n) {
        const uint32_t* sp = reinterpret_cast<const uint32_t*>(
            a.scales + (static_cast<int64_t>(get_seg(a, c0.sgi).e) * a.n + row) * kh16 + c0.kit * 8);
        if ((kh16 & 7) == 0) {   // 16-byte aligned rows: one load
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(sp));
          raw[0] = v.x;
          raw[1] = v.y;
          raw[2] = v.z;
          raw[3] = v.w;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) raw[j] = (c0.kit * 8 + 2 * j < kh16) ? __ldg(sp + j) : 0u;
        }
      }
    };
    if (wg < cnt) load_scales(wg, first_raw);
    if (fused && wg + kDequantGroups < cnt) load_scales(wg + kDequantGroups, second_raw);
  }

  if (fused && warp >= kFirstDequantWarp && warp < kFirstEpilogueWarp + 4) {
    // ------------------------------------------------------------ fused prologue
    // Stage li's B region holds the bf16 x tile of its k range, as the TMA
    // wrote it: row j at 128 j within each 64-k half, 16-byte chunk c at
    // chunk c ^ (j & 7) (128-byte swizzle); rows past m and k past the end
    // are zero.  Unit u = (iteration li, slice sl, row j), j fastest: the 32
    // values of row j at k = 128 kit(li) + 32 sl, chunks (sl & 1) * 4 + q of
    // half sl >> 1.  Pass 1 takes each row's max |x| over the units; pass 2
    // applies the signs, the butterfly and r 2^-e, rounds to fp16 and writes
    // the slice back in place.  The exponent e puts sqrt(32) max|x|, the
    // bound on |x'|, in [2^13, 2^14).
    const int ptid = threadIdx.x - kFirstDequantWarp * 32;
    const int m = a.m_host;
    const int units = cnt * 4 * m;
    bool xok = true;
    for (int li = 0; li < (a.x_box3 ? 1 : cnt); ++li) xok = xok && warp_wait(&sh.xland[li], 0, abortp);
    // a unit's row base in shared memory and the XOR giving its 4 chunks
    auto unit_row = [&](int u, int& cx) -> uint8_t* {
      const int j = u % m, rest = u / m, sl = rest & 3, li = rest >> 2;
      cx = ((sl & 1) * 4) ^ (j & 7);   // chunk q sits at chunk q ^ cx
      return btile_of(li) + (sl >> 1) * kXHalfBytes + j * 128;
    };
    for (int u = ptid; xok && u < units; u += kPrologueThreads) {
      float mx = 0.0f;
      int cx;
      const uint8_t* rowp = unit_row(u, cx);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((q ^ cx) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mx = fmaxf(mx, fabsf(__uint_as_float(ww[e] << 16)));
          mx = fmaxf(mx, fabsf(__uint_as_float(ww[e] & 0xFFFF0000u)));
        }
      }
      atomicMax(&sh.row_max[u % m], __float_as_uint(mx));   // non-negative floats order as integers
    }
    named_bar_sync(2, kPrologueThreads);
    const float r = __uint_as_float(0x3E3504F3u);
    for (int u = ptid; xok && u < units; u += kPrologueThreads) {
      const int j = u % m, rest = u / m, sl = rest & 3, li = rest >> 2;
      int cx;
      uint8_t* rowp = unit_row(u, cx);
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((q ^ cx) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t sw = ww[e] ^ a.x_sign[4 * q + e];   // the signs s_i, on the bf16 sign bits
          v[8 * q + 2 * e] = __uint_as_float(sw << 16);
          v[8 * q + 2 * e + 1] = __uint_as_float(sw & 0xFFFF0000u);
        }
      }
      fwht32_regs_sk(v);
      const float mx = __uint_as_float(sh.row_max[j]);
      int e = 0;
      if (mx > 0.0f && isfinite(mx)) {
        int ex;
        frexpf(__fmul_rn(mx, 5.65685415f), &ex);   // the bound lies in [2^(ex-1), 2^ex)
        e = ex - 14;
        e = e < -100 ? -100 : (e > 100 ? 100 : e);
      }
      if (li == 0 && sl == 0) sh.row_scale[j] = ldexpf(1.0f, e);
      const float rd = __fmul_rn(r, ldexpf(1.0f, -e));   // exact: r times a power of two
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hw[4];
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          const __half2 h = __floats2half2_rn(__fmul_rn(v[8 * q + 2 * c2], rd), __fmul_rn(v[8 * q + 2 * c2 + 1], rd));
          hw[c2] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(rowp + ((q ^ cx) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
    }
    fence_proxy_async_smem();   // the generic-proxy writes, before the tensor core reads them
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.xready);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int armed[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed[i] = -1;
      auto load_x = [&](int st, int kit, const Seg& sg, int nb, uint64_t* bar) {
        for (int b = 0; b < nb; ++b) {
#pragma unroll
          for (int kh = 0; kh < 2; ++kh)
            tma_load_2d(btile_of(st) + kh * kXHalfBytes + (16 * b) * 128, &tm_x, bar, kit * 128 + 64 * kh,
                        sg.row0 + 16 * b);
        }
      };
      // TMA-fed mode: the codes of the first stages go out before the
      // dependency wait -- the kernel before this one (the activation
      // rotation) lets it start only once everything earlier has finished,
      // and does not write the weight.  Fused mode: any kernel may come
      // before, so wait first.
      const int npre = cnt < kStages ? cnt : kStages;
      // per 16-row block: two k-halves of 16 x 128 B of x' per iteration (none
      // in fused mode; none in resident mode, where a segment's x' for all of
      // k is loaded once when the CTA reaches the segment)
      const bool resident = a.x_resident != 0;
      const uint32_t xbytes = (fused || resident) ? 0u : 2u * 2048u;
      int rseg = -1, rcount = 0;   // resident mode: segment whose x' is loaded, loads so far
      auto load_resident = [&](int sgi, const Seg& sg) -> bool {
        // every MMA of the previous segment has read its x' (the issuers'
        // commits), then all 2 KI 64-k halves of this one, 16 rows each
        if (rcount > 0 && !mbar_wait(&sh.rfree, (rcount - 1) & 1, abortp)) return false;
        mbar_arrive_expect_tx(&sh.rland, static_cast<uint32_t>(2 * KI) * 2048u);
        for (int kh = 0; kh < 2 * KI; ++kh) tma_load_2d(smem + kBOff + kh * 2048, &tm_x, &sh.rland, 64 * kh, sg.row0);
        rseg = sgi;
        ++rcount;
        return true;
      };
      Cursor cur;
      cur.init(it_begin, KI, a.row_tiles);
      const Cursor first = cur;
      if (fused) {
        pdl_wait();
        // the raw x tiles first (small; the prologue needs them), then the
        // weight stream behind them (one segment of m <= kSegRows rows)
        const Seg sx = get_seg(a, 0);
        const int nbx = (sx.count + 15) >> 4;
        if (a.x_box3) {
          // one box: the 2 * kFusedMaxIters 64-k chunks from this CTA's first
          // k, 32 rows each, straight into the contiguous B tiles (chunks past
          // this CTA's range land in B tiles it does not use)
          mbar_arrive_expect_tx(&sh.xland[0], 2u * kFusedMaxIters * kXHalfBytes);
          tma_load_3d(btile_of(0), &tm_x3, &sh.xland[0], 0, 0, 2 * first.kit);
        } else {
          Cursor cx = first;
          for (int li = 0; li < cnt; ++li, cx.advance(1, KI, a.row_tiles)) {
            mbar_arrive_expect_tx(&sh.xland[li], static_cast<uint32_t>(nbx) * 2u * 2048u);
            load_x(li, cx.kit, sx, nbx, &sh.xland[li]);
          }
        }
      }
      Seg sg = get_seg(a, cur.sgi);
      int seg_of = cur.sgi;
      bool rok = true;
      for (int li = 0; li < npre; ++li, cur.advance(1, KI, a.row_tiles)) {
        if (cur.sgi != seg_of) {
          seg_of = cur.sgi;
          sg = get_seg(a, seg_of);
        }
        if (resident && cur.sgi != rseg && !(rok = load_resident(cur.sgi, sg))) break;
        const int nb = (sg.count + 15) >> 4;
        mbar_arrive_expect_tx(&sh.full[li], kCodesBytes + nb * xbytes);
        armed[li] = 0;
        tma_load_3d(codes_of(li), &tm_codes, &sh.full[li], cur.kit * 64, cur.rt * 128, sg.e);
      }
      if (!fused && !resident) {
        pdl_wait();   // x' and its row scales are the rotation kernel's output
        Cursor c2 = first;
        Seg sg2 = get_seg(a, c2.sgi);
        int seg2 = c2.sgi;
        for (int li = 0; li < npre; ++li, c2.advance(1, KI, a.row_tiles)) {
          if (c2.sgi != seg2) {
            seg2 = c2.sgi;
            sg2 = get_seg(a, seg2);
          }
          load_x(li, c2.kit, sg2, (sg2.count + 15) >> 4, &sh.full[li]);
        }
      }
      // (fused mode: cnt <= kStages, so the loop below does not run)
      for (int li = npre; rok && li < cnt; ++li, cur.advance(1, KI, a.row_tiles)) {
        const int s = li % kStages;
        const uint32_t ph = (li / kStages) & 1;
        if (!mbar_wait(&sh.done[s], ph ^ 1u, abortp)) break;
        if (cur.sgi != seg_of) {
          seg_of = cur.sgi;
          sg = get_seg(a, seg_of);
        }
        if (resident && cur.sgi != rseg && !(rok = load_resident(cur.sgi, sg))) break;
        const int nb = (sg.count + 15) >> 4;
        mbar_arrive_expect_tx(&sh.full[s], kCodesBytes + nb * xbytes);
        armed[s] = static_cast<int>(ph);
        tma_load_3d(codes_of(s), &tm_codes, &sh.full[s], cur.kit * 64, cur.rt * 128, sg.e);
        if (!resident) load_x(s, cur.kit, sg, nb, &sh.full[s]);
      }
      if (*abortp) {
        // wind down: let every armed copy land before the CTA exits
        for (int i = 0; i < kStages; ++i)
          if (armed[i] >= 0) drain_wait(&sh.full[i], static_cast<uint32_t>(armed[i]));
        if (fused)
          for (int i = 0; i < (a.x_box3 ? 1 : cnt); ++i) drain_wait(&sh.xland[i], 0);
        if (resident && rcount > 0) drain_wait(&sh.rland, (rcount - 1) & 1);
      }
    }
  } else if (warp >= kFirstDequantWarp && warp < kFirstEpilogueWarp) {
    // ------------------------------------------------------------ dequant
    // Group wg takes the iterations li = wg (mod 4).  Per iteration: the 8
    // scales of the row (fetched one iteration ahead), 16 B of codes per row
    // from the stage, and 128 levels per row written with tcgen05.st into the
    // group's A stage -- as two 64-k halves, each signalled separately, so the
    // tensor core reads one half while the group fills the other.
    const int wg = (warp - kFirstDequantWarp) >> 2;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int t = q * 32 + lane;            // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t a_stage = tmem + kACol0 + wg * kAColsPerStage;
    const uint32_t lut_lane = smem_u32(lut) + 4u * static_cast<uint32_t>(lane);
    const int kh16 = a.k / 16;
    int seg_cached = -1, e_cached = 0;   // expert of the segment whose scales were last fetched
    auto fetch_scales = [&](const Cursor& c, uint32_t (&raw)[4]) {
      if (c.sgi != seg_cached) {
        seg_cached = c.sgi;
        e_cached = get_seg(a, c.sgi).e;
      }
      const int row = c.rt * 128 + t;
      const bool rv = row < a.n;
      const uint32_t* sp = reinterpret_cast<const uint32_t*>(
          a.scales + (static_cast<int64_t>(e_cached) * a.n + (rv ? row : 0)) * kh16 + c.kit * 8);
      if ((kh16 & 7) == 0) {   // 16-byte aligned rows: one load
        const uint4 v = rv ? __ldg(reinterpret_cast<const uint4*>(sp)) : make_uint4(0u, 0u, 0u, 0u);
        raw[0] = v.x;
        raw[1] = v.y;
        raw[2] = v.z;
        raw[3] = v.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = (rv && c.kit * 8 + 2 * j < kh16) ? __ldg(sp + j) : 0u;
      }
    };
    uint32_t next_raw[4] = {first_raw[0], first_raw[1], first_raw[2], first_raw[3]};
    Cursor ahead;         // the iteration whose scales are in flight
    ahead.init(it_begin + wg, KI, a.row_tiles);
    int use = 0;    // how many times this group has filled its A stage
    for (int li = wg; li < cnt; li += kDequantGroups, ++use) {
      uint32_t sraw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) sraw[j] = next_raw[j];
      if (li + kDequantGroups < cnt) {
        if (fused) {
#pragma unroll
          for (int j = 0; j < 4; ++j) next_raw[j] = second_raw[j];
        } else {
          ahead.advance(kDequantGroups, KI, a.row_tiles);
          fetch_scales(ahead, next_raw);
        }
      }
      const int s = li % kStages;
      if (!warp_wait(&sh.full[s], (li / kStages) & 1, abortp)) break;
      const uint8_t* cb = codes_of(s) + t * 64;
      bool ok = true;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // this half was last read by the MMAs of the group's previous use
        if (use > 0 && !warp_wait(&sh.afree[wg][h], (use - 1) & 1, abortp)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kb2 = 0; kb2 < 2; ++kb2) {
          const int kb = 2 * h + kb2;
          const uint4 c = *reinterpret_cast<const uint4*>(cb + 16 * (kb ^ ((t >> 1) & 3)));
          uint32_t o[16];
          const uint32_t sp = sraw[kb];   // scales of the block's two halves
          dequant_half(c.x, c.y, prmt(sp, 0u, 0x1010u), lut_lane, o);
          dequant_half(c.z, c.w, prmt(sp, 0u, 0x3232u), lut_lane, o + 8);
          tmem_st16(a_stage + lane_base + 16 * kb, o);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.afull[wg][h]);
      }
      if (!ok) break;
      // resident x': the MMAs read only tensor memory and the resident x', so
      // the codes stage is free as soon as this warp has read it (the refill
      // gets the MMAs' latency as extra lead)
      if (a.x_resident) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.done[s]);
      }
    }
  } else if ((warp == 1 || warp >= kFirstIssuerWarp) && lane == 0) {
    // ------------------------------------------------------------ MMA issue
    // Issuer of group w: the iterations li = w (mod 4), in order.  Per half A
    // stage: wait until the group filled it, issue 4 MMAs (K = 16) into the
    // group's accumulator, commit to the half's `afree`; after the second
    // half commit to the stage's `done`; at the end of a portion commit (or,
    // with no iteration in it, arrive) on `dfull`.
    const int w = issuer_group(warp);
    int use = 0;   // fills of the group's A stage consumed so far
    bool ok = !fused || mbar_wait(&sh.xready, 0, abortp);   // fused mode: the B tiles are written
    const bool resident = a.x_resident != 0;
    int iseg = -1, rn = 0;   // resident mode: segment whose x' the MMAs read, loads waited for
    for (int pi = 0; pi < nportions && ok; ++pi) {
      const int tile = tile_begin + pi;
      const int pf = (tile * KI > it_begin ? tile * KI : it_begin) - it_begin;
      const int pe = ((tile + 1) * KI < it_end ? (tile + 1) * KI : it_end) - it_begin;
      const int db = pi % nsets;
      const uint32_t dpar = static_cast<uint32_t>((pi / nsets) & 1);
      // the accumulator set must be free before any MMA or arrival of this portion
      if (!mbar_wait(&sh.dempty[db], dpar ^ 1u, abortp)) {
        ok = false;
        break;
      }
      const Seg sg = get_seg(a, tile / a.row_tiles);
      const int nb = (sg.count + 15) >> 4;
      const uint32_t idesc = idesc_f16(128, 16 * nb);
      if (resident && tile / a.row_tiles != iseg) {
        // a new segment: release the previous one's x' once these MMAs are
        // done, then wait for this one's
        if (iseg >= 0) mma_commit(&sh.rfree);
        if (!mbar_wait(&sh.rland, rn & 1, abortp)) {
          ok = false;
          break;
        }
        ++rn;
        iseg = tile / a.row_tiles;
      }
      const uint32_t acc = tmem + db * (kAccRegion / nsets) + w * acc_w;
      const uint32_t a_stage = tmem + kACol0 + w * kAColsPerStage;
      bool started = false;
      // first local iteration of this portion that belongs to group w
      for (int li = pf + ((w - pf) % kDequantGroups + kDequantGroups) % kDequantGroups; li < pe && ok;
           li += kDequantGroups) {
        const int s = li % kStages;
        // resident mode: the iteration's k slice of the segment's x'; else the stage's B tile
        const int kit_li = it_begin + li - tile * KI;
        const uint32_t xb = resident ? smem_u32(smem + kBOff + kit_li * 2 * 2048) : smem_u32(btile_of(s));
        // the B tile (x') of this stage must have landed too (resident x':
        // the stage holds only codes, which the dequant warps waited for --
        // and may already be refilled, so its barrier is not waited on here)
        if (!resident && !mbar_wait(&sh.full[s], (li / kStages) & 1, abortp)) {
          ok = false;
          break;
        }
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(&sh.afull[w][h], use & 1, abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // half h of the stage's B tile is k-half h of x'; the descriptor's
          // start address (16-byte units) advances by 2 per 16-k step
          const uint64_t bdesc0 = sdesc_k128(xb + h * (resident ? 2048 : kXHalfBytes));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(acc, a_stage + 32 * h + 8 * kk, bdesc0 + static_cast<uint64_t>(2 * kk), idesc,
                   (!started && h == 0 && kk == 0) ? 0u : 1u);
          mma_commit(&sh.afree[w][h]);
        }
        if (!ok) break;
        if (!resident) mma_commit(&sh.done[s]);
        started = true;
        ++use;
      }
      if (!ok) break;
      if (started) mma_commit(&sh.dfull[db]);
      else mbar_arrive(&sh.dfull[db]);
    }
    mma_commit(&sh.issuer_done[w]);
    drain_wait(&sh.issuer_done[w], 0);
  } else if (warp >= kFirstEpilogueWarp && warp < kFirstEpilogueWarp + 4) {
    // ------------------------------------------------------------ epilogue
    pdl_wait();   // y, the partials and the counters may still be in use upstream
    const int q = warp & 3;
    const int t = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // fused mode: the row scales come from the prologue
    if (fused) {
      if (t == 0) sh.x_ok = mbar_wait(&sh.xready, 0, abortp) ? 1 : 0;
      named_bar_sync(1, 128);
    }
    int sgi = tile_begin / a.row_tiles;
    int rt = tile_begin - sgi * a.row_tiles;
    for (int pi = 0; pi < nportions && (!fused || sh.x_ok); ++pi) {
      const int tile = tile_begin + pi;
      if (pi > 0 && ++rt == a.row_tiles) {
        rt = 0;
        ++sgi;
      }
      const int tile_first = tile * KI;
      const int portion_first = it_begin > tile_first ? it_begin : tile_first;
      const int portion_end = (tile + 1) * KI < it_end ? (tile + 1) * KI : it_end;
      const int db = pi % nsets;
      // one thread waits; the decision is published before the group barrier
      // so all four epilogue warps leave together on a timeout
      if (t == 0) sh.epi_ok[pi & 1] = mbar_wait(&sh.dfull[db], (pi / nsets) & 1, abortp) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!sh.epi_ok[pi & 1]) break;
      tc_fence_after();
      const Seg sg = get_seg(a, sgi);
      const int nb = (sg.count + 15) >> 4;
      const int row = rt * 128 + t;
      // group w wrote an accumulator iff one of the portion's local
      // iterations is congruent to w mod 4
      const int lpf = portion_first - it_begin, plen = portion_end - portion_first;
      const uint32_t dbase = tmem + lane_base + db * (kAccRegion / nsets);
      const bool whole = (portion_first == tile_first) && (portion_end == tile_first + KI);
      const int slot = (pi == 0) ? 0 : 1;
      float* pbase = a.partials + ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * 128 + t) * kSegRows;
      for (int c = 0; c < nb; ++c) {
        // columns [16c, 16c+16) of each group's accumulator
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
        for (int w = 0; w < kDequantGroups; ++w) {
          const int off = ((w - lpf) % kDequantGroups + kDequantGroups) % kDequantGroups;
          if (off >= plen) continue;
          uint32_t rr[16];
          tmem_ld16(dbase + w * acc_w + 16 * c, rr);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __fadd_rn(v[j], __uint_as_float(rr[j]));
        }
        {
          // a non-finite sum: some level overflowed fp16 (a half-block scale
          // above ~93.6), or the inputs hold an Inf or NaN; the row's portion
          // is recomputed exactly (the latter stays non-finite, as it should).
          // v * 0 is 0 for a finite v and NaN otherwise, so one test covers the
          // 16 columns (a padding column only costs a needless recompute).
          const int ntok = sg.count - 16 * c < 16 ? sg.count - 16 * c : 16;
          float z = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) z = __fmaf_rn(v[j], 0.0f, z);
          const bool bad = z != z;
          if (bad && row < a.n) {
            const int kc0 = (portion_first - tile_first) * 128;
            const int kc1 = min((portion_end - tile_first) * 128, a.k);
            const int64_t wrow = static_cast<int64_t>(sg.e) * a.n + row;
            float ex[16];   // (its own array: v stays in registers)
            exact_row_portion(a.codes + wrow * (a.k / 2), a.scales + wrow * (a.k / 16), kc0, kc1,
                              a.xr ? a.xr + static_cast<int64_t>(sg.row0) * a.k : nullptr, a.k,
                              smem + kBOff, lpf, 16 * c, ntok, lt.h, ex);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = ex[j];
          }
        }
        // back from the scaled domain: times 2^e / 256 per token (exact), with
        // 2^e from the prologue in fused mode (it may differ between the CTAs
        // of a split tile, so it is applied before the partials are published)
        // or else the rotation kernel's row_scale
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int jj = 16 * c + j;
          if (jj < sg.count) {
            const float s = fused ? sh.row_scale[jj] : __ldcg(a.row_scale + sg.row0 + jj);
            v[j] = __fmul_rn(v[j], __fmul_rn(s, 1.0f / kLevelScale));
          }
        }
        if (c == nb - 1) {
          tc_fence_before();
          mbar_arrive(&sh.dempty[db]);
        }
        if (a.cluster_s > 1) {
          // cluster split-K: row t goes to the CTA that owns it, slot of this
          // CTA's rank: [rank][token][row - first row of the owner]
          const int s_n = a.cluster_s;
          const int q = (t * s_n) >> 7;                       // owner: floor(t s / 128)
          const int rpc = (128 + s_n - 1) / s_n;              // rows per CTA (at most)
          const int tl = t - (q * 128 + s_n - 1) / s_n;       // row within the owner's range
          const uint32_t dst0 = smem_u32(smem + kRedOff) +
                                static_cast<uint32_t>(((static_cast<int>(cluster_ctarank()) * 32 + 16 * c) * rpc + tl) * 4);
#pragma unroll
          for (int j = 0; j < 16; ++j) st_dsmem_f32(dst0 + static_cast<uint32_t>(j * rpc * 4), static_cast<uint32_t>(q), v[j]);
        } else if (whole) {
          epilogue_store(a, v, 16 * c, row, sg);
        } else {
          float4* pp = reinterpret_cast<float4*>(pbase + 16 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j) pp[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      if (whole || a.cluster_s > 1) continue;
      // split tile: publish the partial, the last contributor finishes it.
      // The group barrier orders the 128 threads' partial stores before thread
      // 0's release (acq_rel, gpu scope) on the tile counter; the last
      // arriver's acquire orders its reads of the others' partials after it.
      // A counter holds (epoch << 32) | arrivals: a value left by another
      // launch (another epoch) counts as zero arrivals, so the counters never
      // need clearing; the last arriver resets its counter to zero, which
      // covers a later launch with the same epoch (a graph replay).
      named_bar_sync(1, 128);
      const int c_first = owner_of(tile_first, T, G);
      const int c_last = owner_of(tile_first + KI - 1, T, G);
      if (t == 0) {
        unsigned ncontrib = 0;
        for (int c = c_first; c <= c_last; ++c)
          if (range_begin(c + 1, T, G) > range_begin(c, T, G)) ++ncontrib;
        unsigned long long* ctr = a.counters + tile;
        const unsigned long long tag = static_cast<unsigned long long>(a.epoch) << 32;
        unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(ctr), want = 0;
        bool done = false;
        for (int attempt = 0; attempt < (1 << 20) && !done; ++attempt) {
          want = ((cur >> 32) == a.epoch) ? cur + 1 : (tag | 1ull);
          unsigned long long prev;
          asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;"
                       : "=l"(prev) : "l"(ctr), "l"(cur), "l"(want) : "memory");
          done = (prev == cur);
          cur = prev;
        }
        if (!done) raise_status(TQ_DEV_TIMEOUT);
        const bool last = done && (want & 0xFFFFFFFFull) == ncontrib;
        // After the last arrival no CTA of this launch touches the counter
        // again, so it is reset: a launch that reuses this epoch (a CUDA graph
        // replays its kernels with the arguments they were captured with)
        // then counts from zero.  The next launch reads the counter only after
        // this grid has completed (stream order, or its dependent-launch wait).
        if (last) *reinterpret_cast<volatile unsigned long long*>(ctr) = 0ull;
        sh.last_flag = last ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (sh.last_flag) {
        for (int ch = 0; ch < nb; ++ch) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
          for (int c = c_first; c <= c_last; ++c) {
            const int cb0 = range_begin(c, T, G);
            if (range_begin(c + 1, T, G) <= cb0) continue;
            const int cslot = (cb0 / KI == tile) ? 0 : 1;
            const float4* src = reinterpret_cast<const float4*>(
                a.partials + ((static_cast<int64_t>(c) * 2 + cslot) * 128 + t) * kSegRows + 16 * ch);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 f = __ldcg(src + j);
              acc[4 * j] = __fadd_rn(acc[4 * j], f.x);
              acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], f.y);
              acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], f.z);
              acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], f.w);
            }
          }
          epilogue_store(a, acc, 16 * ch, row, sg);
        }
      }
      named_bar_sync(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.cluster_s > 1) {
    // Cluster split-K reduction.  Every thread of every CTA of the cluster
    // reaches the barrier (on a timeout too: the roles above always run to
    // their end), so it cannot hang; it orders every CTA's stores into the
    // owners' buffers before the owners read them.  Nothing reads another
    // CTA's shared memory after it, so no second barrier is needed.
    cluster_sync_all();
    if (!sh.abort_flag) {
      const int s_n = a.cluster_s;
      const int rank = static_cast<int>(cluster_ctarank());
      const int tile = tile_begin;   // one tile per CTA in this mode
      const int rt = tile % a.row_tiles;
      const Seg sg = get_seg(a, tile / a.row_tiles);
      const int rpc = (128 + s_n - 1) / s_n;
      const int r0 = (rank * 128 + s_n - 1) / s_n, r1 = ((rank + 1) * 128 + s_n - 1) / s_n;
      const int nrow = r1 - r0;
      const float* red = reinterpret_cast<const float*>(smem + kRedOff);
      for (int idx = threadIdx.x; idx < nrow * sg.count; idx += kThreads) {
        const int j = idx / nrow, tl = idx - j * nrow;
        const int row = rt * 128 + r0 + tl;
        if (row >= a.n) continue;
        float acc = 0.0f;
        for (int q = 0; q < s_n; ++q) acc = __fadd_rn(acc, red[(q * 32 + j) * rpc + tl]);
        a.out_a[static_cast<int64_t>(sg.row0 + j) * a.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
      }
    }
  }
  // Dependents may launch once every CTA is done: a kernel that waits on this
  // one gains nothing from taking an SM early, and its CTAs would only delay
  // this kernel's CTAs that have not started yet.
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Epochs of one process start at a random value, not at 1: a workspace that
// was never initialised may hold structured data (small integers, indices)
// where a counter sits, and a counter whose upper word happened to equal the
// current epoch would be miscounted.  Successive epochs still differ, and 0
// is never used.
static uint32_t first_epoch() {
  uint32_t seed = 0x9E3779B9u;
  try {
    std::random_device rd;
    seed ^= rd();
  } catch (...) {
  }
  seed ^= static_cast<uint32_t>(std::chrono::steady_clock::now().time_since_epoch().count());
  return seed | 0x40000000u;   // away from the small values structured data is full of
}

uint32_t next_epoch() {
  static std::atomic<uint32_t> epoch{first_epoch()};
  uint32_t e = epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  if (e == 0) e = epoch.fetch_add(1, std::memory_order_relaxed) + 1;   // 0 marks never-used counters
  return e;
}

int choose_cluster_split(int64_t tiles, int64_t k_iters, int sms) {
  static std::mutex mu;
  static int cap[64][9];   // per device, per s: resident clusters (+1; 0 = not queried yet)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 1;
  }
  for (int s = 8; s >= 2; --s) {
    if (s > k_iters || (k_iters + s - 1) / s > kFusedMaxIters || tiles * s > sms) continue;
    int c;
    {
      std::lock_guard<std::mutex> g(mu);
      if (cap[dev][s] == 0) cap[dev][s] = streamk_max_clusters(s) + 1;
      c = cap[dev][s] - 1;
    }
    if (tiles <= c) return s;
  }
  return 1;
}

int streamk_max_clusters(int s) {
  // clusters of s CTAs (one per SM) that can be resident at once
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(s));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = streamk_smem_bytes();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(s);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaFuncSetAttribute(streamk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(streamk_smem_bytes())) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, streamk_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

size_t streamk_smem_bytes() { return static_cast<size_t>(kStages) * kStageBytes + kLutBytes + 1024; }

cudaError_t launch_streamk(const void* tm_codes, const void* tm_x, const void* tm_x3, const StreamKArgs& a,
                           int grid, cudaStream_t st) {
  static bool attr_set = false;
  const size_t smem = streamk_smem_bytes();
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(streamk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(streamk_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  static const LevelTable lt = [] {
    LevelTable t;
    const CodebookF32& cb = codebook();
    for (int i = 0; i < 16; ++i)
      t.h[i] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(cb.levels[i] * kLevelScale)));
    return t;
  }();
  const CUtensorMap& m0 = *static_cast<const CUtensorMap*>(tm_codes);
  const CUtensorMap& m1 = *static_cast<const CUtensorMap*>(tm_x);
  const CUtensorMap& m3 = *static_cast<const CUtensorMap*>(tm_x3 ? tm_x3 : tm_x);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.cluster_s > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(a.cluster_s);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, streamk_kernel, m0, m1, m3, a, lt);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace tq4
