// Stream-K dequant-GEMM for small m (decode blocks of 16 tokens, MoE expert
// groups) on sm_100a.
//
// Computes D[n][j] = sum_k w_n[n][k] * x'[j][k] for 128-row tiles of one
// expert's weight, where w_n = c[code] * d are the rotated-domain levels
// ("What Config-I means": 16-level Lloyd-Max codes, two half-block scales)
// and x' = R x is the activation rotated per 32-slice, split into bf16 hi and
// lo rows (route B: rotating the activations instead of inverse-rotating the
// weights, which is equivalent because R is orthogonal).  Per 128-k
// iteration of a 128-row tile:
//   warp 0      TMA: packed codes tile [128 x 64 B] (64-byte swizzle) and the
//               x' hi/lo tiles [rows x 128 k] (128-byte swizzle) into a
//               shared-memory stage, completing on an mbarrier;
//   warps 4-19  four dequant warpgroups (round-robin iterations), thread = row:
//               16 B of codes + 8 fp16 scales -> 128 bf16 levels through a
//               per-half-block scaled table looked up with byte permutes,
//               written to tensor memory with tcgen05.st (the MMA A operand);
//               one thread of the group then issues 8 tcgen05.mma (M=128,
//               N=32*nb, K=16, A from tensor memory, B from shared memory)
//               into the group's own accumulator -- four concurrent issuers;
//   warps 2-3   (dense bf16 mode) rotate x per 32-slice in registers and
//               write the x' hi/lo B tiles into the stage, 128-byte swizzled;
//   warp 1      allocates / frees tensor memory;
//   warps 20-23 epilogue, thread = row: tcgen05.ld of the accumulator in
//               16-token chunks, hi + lo columns summed, then the mode's store.
// The flattened (segment, row tile, k iteration) space is split evenly over
// the CTAs (stream-K).  A tile split between CTAs is finished by whichever
// contributor arrives last on the tile's counter: it sums all contributors'
// fp32 partials in CTA order (deterministic) and runs the epilogue, so no
// CTA ever waits on another.
#include "tq4_internal.h"

namespace tq4 {
namespace {

constexpr int kThreads = 800;
constexpr int kDequantGroups = 4;
constexpr int kFirstDequantWarp = 4;
constexpr int kFirstEpilogueWarp = kFirstDequantWarp + 4 * kDequantGroups;
// Two MMA-issuing threads: lane 0 of warp 1 serves dequant groups 0 and 1,
// lane 0 of the last warp (24) groups 2 and 3.
constexpr int kIssuerWarpB = kFirstEpilogueWarp + 4;
static_assert((kIssuerWarpB + 1) * 32 == kThreads, "warp roles cover the block");
constexpr int kStages = 8;
constexpr int kAStages = 4;
constexpr int kCodesBytes = 128 * 64;    // 128 rows x 128 k codes
constexpr int kXHalfBytes = 64 * 128;    // 64 rows x 64 k bf16 (one 128-B swizzle span)
constexpr int kXBytes = 2 * kXHalfBytes; // two k-halves
constexpr int kStageBytes = kCodesBytes + kXBytes;
constexpr int kTmemCols = 512;
// Tensor memory: columns [0, 256) hold the accumulators, [256, 512) the four
// A stages (one per dequant warpgroup, 64 columns = 128 k of bf16 levels).
// Each warpgroup issues the MMAs of its own iterations into its own
// accumulator (N = 32 * nb columns): single-thread tcgen05.mma issue costs
// ~66-98 cycles per instruction at small N, so four concurrent issuers are
// needed to keep pace with the weight stream.  With nb = 1 (<= 16 tokens per
// segment) the four accumulators take 128 columns and two accumulator sets
// alternate between tile portions; with nb = 2 one set of 256 columns.
constexpr int kAccRegion = 256;
constexpr int kACol0 = kAccRegion;
constexpr int kAColsPerStage = 64;
static_assert(kACol0 + kAStages * kAColsPerStage <= kTmemCols, "tensor memory budget");
static_assert(kAStages == kDequantGroups, "one A stage per dequant warpgroup");

struct SharedState {
  uint64_t full[kStages];      // TMA landed (codes, x') and rotated x' written
  uint64_t done[kStages];      // the MMAs of the iteration that used this stage completed
  uint64_t afull[kDequantGroups][2];   // a half A stage (64 k) holds fresh levels (128 arrivals)
  uint64_t afree[kDequantGroups][2];   // the MMAs reading a half A stage completed
  uint64_t dfull[2];           // all four warpgroups finished a portion (4 arrivals)
  uint64_t dempty[2];          // the epilogue drained an accumulator set (128 arrivals)
  uint64_t issuer_done[2];
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
  int epi_ok[2];
};

struct Seg {
  int e, row0, count;
};

__device__ __forceinline__ Seg get_seg(const StreamKArgs& a, int s) {
  if (a.segs) {
    const int4 v = a.segs[s];
    return {v.x, v.y, v.z};
  }
  const int r0 = s * kSegRows;
  return {0, r0, min(kSegRows, a.m_host - r0)};
}

// First iteration of CTA c when T iterations are split over G CTAs.
__device__ __forceinline__ int64_t range_begin(int64_t c, int64_t T, int64_t G) { return c * T / G; }
// The CTA whose range holds iteration i.
__device__ __forceinline__ int64_t owner_of(int64_t i, int64_t T, int64_t G) { return ((i + 1) * G + T - 1) / T - 1; }

// Position of an iteration in the (segment, row tile, k iteration) space,
// advanced incrementally so the loops do no integer division.
struct Cursor {
  int tile, kit, sgi, rt;
  __device__ __forceinline__ void init(int64_t it, int KI, int RT) {
    tile = static_cast<int>(it / KI);
    kit = static_cast<int>(it - static_cast<int64_t>(tile) * KI);
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

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
template <bool kF16>
__device__ __forceinline__ uint32_t x2_from_f32x2(uint64_t v) {
  const float lo = __uint_as_float(static_cast<uint32_t>(v)), hi = __uint_as_float(static_cast<uint32_t>(v >> 32));
  if constexpr (kF16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    return pack_bf16x2(lo, hi);
  }
}

// Dequantize one half-block (16 codes in q0 = elements 0..7, q1 = 8..15, one
// nibble each, low nibble first) with scale d into 8 registers of bf16 pairs
// {element 2i, element 2i+1}, value bf16(c[code] * d) (or fp16 when kF16)
// with one rounding of the fp32 product.
//
// The codebook is odd-symmetric (c[15-j] = -c[j]), so a code j maps to a
// magnitude index m = j-8 (j >= 8) or 7-j (j < 8) and a sign (j < 8).  The 8
// scaled magnitudes are built per half-block as bf16 and split into a
// low-byte plane and a high-byte plane (two registers each); prmt then looks
// up four codes at a time by byte index, the sign is OR-ed into the high
// bytes, and a last prmt interleaves low/high bytes into bf16 pairs.
template <bool kF16>
__device__ __forceinline__ void dequant_half(uint32_t q0, uint32_t q1, float d, const uint64_t (&cm2)[4],
                                             uint32_t* out) {
  const uint64_t dd = pack_f32x2(d, d);
  const uint32_t p01 = x2_from_f32x2<kF16>(fmul2(cm2[0], dd));
  const uint32_t p23 = x2_from_f32x2<kF16>(fmul2(cm2[1], dd));
  const uint32_t p45 = x2_from_f32x2<kF16>(fmul2(cm2[2], dd));
  const uint32_t p67 = x2_from_f32x2<kF16>(fmul2(cm2[3], dd));
  const uint32_t lo0 = prmt(p01, p23, 0x6420u), lo1 = prmt(p45, p67, 0x6420u);
  const uint32_t hi0 = prmt(p01, p23, 0x7531u), hi1 = prmt(p45, p67, 0x7531u);
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const uint32_t q = w ? q1 : q0;
    const uint32_t pos = (q >> 3) & 0x11111111u;            // 1 where code >= 8
    const uint32_t m = (q ^ (0x77777777u - pos * 7u)) & 0x77777777u;  // magnitude index per nibble
    const uint32_t qs = q << 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t sel = h ? (m >> 16) : m;
      const uint32_t l4 = prmt(lo0, lo1, sel);
      uint32_t h4 = prmt(hi0, hi1, sel);
      // 0xFF per byte where the code is >= 8 (sign bit of nibble replicated)
      const uint32_t posmask = prmt(qs, q, h ? 0xFBEAu : 0xD9C8u);
      h4 |= ~posmask & 0x80808080u;
      out[4 * w + 2 * h + 0] = prmt(l4, h4, 0x5140u);
      out[4 * w + 2 * h + 1] = prmt(l4, h4, 0x7362u);
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

__device__ __forceinline__ float warp_fwht32_epi(float a, int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const float p = __shfl_xor_sync(0xFFFFFFFFu, a, h);
    a = (lane & h) ? __fsub_rn(p, a) : __fadd_rn(a, p);
  }
  return a;
}

// The per-mode store of 16 tokens [j0, j0 + 16) of one finished tile row
// (thread = weight row `row`).
__device__ __forceinline__ void epilogue_store(const StreamKArgs& a, float (&v)[16], int j0, int row, int lane,
                                               const Seg& sg) {
  const int cnt = sg.count - j0;
  if (a.row_scale) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cnt) v[j] = __fmul_rn(v[j], a.row_scale[sg.row0 + j0 + j]);
  }
  if (a.mode == EPI_DENSE) {
    if (row < a.n) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < cnt)
          a.out_a[static_cast<int64_t>(sg.row0 + j0 + j) * a.n + row] =
              __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
    }
  } else if (a.mode == EPI_UP) {
    // h = bf16(relu(u)^2), then rotate the 32-slice held by this warp with the
    // down projection's signs and split into hi/lo rows for the next stage.
    const int slice0 = row - lane;
    if (slice0 < a.n) {
      const bool neg = (a.next_mask >> lane) & 1u;
      const float r = __uint_as_float(0x3E3504F3u);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < cnt) {
          const float hv = relu2_bf16(v[j]);
          const float t = __fmul_rn(warp_fwht32_epi(neg ? -hv : hv, lane), r);
          const __nv_bfloat16 hi = __float2bfloat16_rn(t);
          const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(t, __bfloat162float(hi)));
          const int64_t off = static_cast<int64_t>(sg.row0 + j0 + j) * a.n + row;
          a.out_a[off] = __bfloat16_as_ushort(hi);
          a.out_b[off] = __bfloat16_as_ushort(lo);
        }
      }
    }
  } else {
    if (row < a.n) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < cnt) {
          const int p = a.pairs[sg.row0 + j0 + j];
          a.out_f[static_cast<int64_t>(p) * a.n + row] = __fmul_rn(a.topk_w[p], v[j]);
        }
      }
    }
  }
}

struct Codemag {
  float v[8];   // levels[8..15]: the positive magnitudes, ascending
};

template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
    streamk_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_xhi,
                   const __grid_constant__ CUtensorMap tm_xlo, const StreamKArgs a, const Codemag cmag) {
  __shared__ SharedState sh;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Grouped (MoE) mode reads the routing kernel's segment list right away;
  // the dense mode defers the dependency wait to the roles that need it.
  if (a.segs) pdl_wait();
  const int nseg = a.segs ? *a.nseg_dev : a.nseg_host;
  const int KI = a.k_iters;
  const int64_t T = static_cast<int64_t>(nseg) * a.row_tiles * KI;
  const int64_t G = gridDim.x;
  const int64_t it_begin = range_begin(blockIdx.x, T, G);
  const int64_t it_end = range_begin(blockIdx.x + 1, T, G);
  const int cnt = static_cast<int>(it_end - it_begin);
  if (cnt <= 0) return;
  // accumulator layout (see kAccRegion): width per warpgroup, number of sets
  const int acc_w = 32 * a.nb_max;
  const int nsets = (a.nb_max == 1) ? 2 : 1;
  const int64_t tile_begin = it_begin / KI, tile_last = (it_end - 1) / KI;
  const int nportions = static_cast<int>(tile_last - tile_begin + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], a.x_raw ? 3 : 1);   // producer (+ the two rotation warps)
      mbar_init(&sh.done[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.dfull[i], kDequantGroups);
      mbar_init(&sh.dempty[i], 128);
    }
    for (int i = 0; i < kDequantGroups; ++i)
      for (int h = 0; h < 2; ++h) {
        mbar_init(&sh.afull[i][h], 128);
        mbar_init(&sh.afree[i][h], 1);
      }
    for (int i = 0; i < 2; ++i) mbar_init(&sh.issuer_done[i], 1);
    sh.abort_flag = 0;
    sh.last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_xhi);
    tma_prefetch_desc(&tm_xlo);
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
  if (threadIdx.x == 0) pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (!a.x_raw) pdl_wait();   // x' tiles are the previous kernel's output
      int armed[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed[i] = -1;
      Cursor cur;
      cur.init(it_begin, KI, a.row_tiles);
      Seg sg = get_seg(a, cur.sgi);
      int seg_of = cur.sgi;
      for (int li = 0; li < cnt; ++li, cur.advance(1, KI, a.row_tiles)) {
        const int s = li % kStages;
        const uint32_t ph = (li / kStages) & 1;
        if (!mbar_wait(&sh.done[s], ph ^ 1u, abortp)) break;
        if (cur.sgi != seg_of) {
          seg_of = cur.sgi;
          sg = get_seg(a, seg_of);
        }
        const int kit = cur.kit, rt = cur.rt;
        const int nb = (sg.count + 15) >> 4;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&sh.full[s], kCodesBytes + (a.x_raw ? 0 : nb * 4 * 2048));
        armed[s] = static_cast<int>(ph);
        tma_load_3d(st, &tm_codes, &sh.full[s], kit * 64, rt * 128, sg.e);
        for (int b = 0; b < nb && !a.x_raw; ++b) {
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            uint8_t* xb = st + kCodesBytes + kh * kXHalfBytes;
            tma_load_2d(xb + (16 * b) * 128, &tm_xhi, &sh.full[s], kit * 128 + 64 * kh, sg.row0 + 16 * b);
            tma_load_2d(xb + (16 * nb + 16 * b) * 128, &tm_xlo, &sh.full[s], kit * 128 + 64 * kh,
                        sg.row0 + 16 * b);
          }
        }
      }
      if (*abortp) {
        // wind down: let every armed copy land before the CTA exits
        for (int i = 0; i < kStages; ++i)
          if (armed[i] >= 0) drain_wait(&sh.full[i], static_cast<uint32_t>(armed[i]));
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ rotation
    // Dense bf16 mode: x' = r H diag(s) x per 32-slice, split into bf16 hi and
    // lo, written straight into the stage's B tile.  Unit u = (token j, slice
    // sl) of the iteration's 128 k; the 64 threads take units u and u + 64.
    if (a.x_raw) {
      pdl_wait();   // x may be the previous kernel's output
      const int tid = (warp - 2) * 32 + lane;
      const float r = __uint_as_float(0x3E3504F3u);
      Cursor cur;
      cur.init(it_begin, KI, a.row_tiles);
      for (int li = 0; li < cnt; ++li, cur.advance(1, KI, a.row_tiles)) {
        const int s = li % kStages;
        if (!warp_wait(&sh.done[s], ((li / kStages) & 1) ^ 1u, abortp)) break;
        const Seg sg = get_seg(a, cur.sgi);
        const int nb = (sg.count + 15) >> 4;
        uint8_t* xb = smem + s * kStageBytes + kCodesBytes;
        for (int u = tid; u < 64 * nb; u += 64) {
          const int j = u >> 2, sl = u & 3;
          const int k0 = cur.kit * 128 + 32 * sl;
          float v[32];
          if (j < sg.count && k0 < a.k) {
            const uint4* src =
                reinterpret_cast<const uint4*>(a.x_raw + static_cast<int64_t>(sg.row0 + j) * a.k + k0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 w = __ldg(src + q);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                v[8 * q + 2 * e] = __uint_as_float(ww[e] << 16);
                v[8 * q + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if ((a.x_mask >> i) & 1u) v[i] = -v[i];
            fwht32_regs_sk(v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.0f;
          }
          // hi row j, lo row 16nb + j; slice sl covers bytes [(sl&1)*64, +64)
          // of the 128-byte row in k-half (sl >> 1); 16-byte chunk c of row
          // `row` sits at chunk c ^ (row & 7) (128-byte swizzle)
          uint8_t* half = xb + (sl >> 1) * kXHalfBytes;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float f0 = __fmul_rn(v[8 * q + 2 * e], r), f1 = __fmul_rn(v[8 * q + 2 * e + 1], r);
              const __nv_bfloat16 h0 = __float2bfloat16_rn(f0), h1 = __float2bfloat16_rn(f1);
              const __nv_bfloat16 l0 = __float2bfloat16_rn(__fsub_rn(f0, __bfloat162float(h0)));
              const __nv_bfloat16 l1 = __float2bfloat16_rn(__fsub_rn(f1, __bfloat162float(h1)));
              hw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
              lw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
            }
            const int c = (sl & 1) * 4 + q;
            const int rh = j, rl = 16 * nb + j;
            *reinterpret_cast<uint4*>(half + rh * 128 + ((c ^ (rh & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(half + rl * 128 + ((c ^ (rl & 7)) << 4)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.full[s]);
      }
    }
  } else if (warp >= kFirstDequantWarp && warp < kFirstEpilogueWarp) {
    // ------------------------------------------------------------ dequant
    // Warpgroup wg takes the iterations li = wg (mod 4).  Per iteration: the
    // 8 fp16 scales (fetched one iteration ahead), 16 B of codes per row from
    // the stage, and 128 levels per row written with tcgen05.st into the
    // group's A stage -- as two 64-k halves, each signalled separately, so the
    // tensor core reads one half while the group fills the other.
    const int wg = (warp - kFirstDequantWarp) >> 2;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int t = q * 32 + lane;            // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t a_stage = tmem + kACol0 + wg * kAColsPerStage;
    uint64_t cm2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cm2[i] = pack_f32x2(cmag.v[2 * i], cmag.v[2 * i + 1]);
    const int kh16 = a.k / 16;
    auto fetch_scales = [&](const Cursor& c, uint32_t (&raw)[4]) {
      const int kit = c.kit, rt = c.rt;
      const int e = get_seg(a, c.sgi).e;
      const int row = rt * 128 + t;
      const bool rv = row < a.n;
      const uint32_t* sp = reinterpret_cast<const uint32_t*>(
          a.scales + (static_cast<int64_t>(e) * a.n + (rv ? row : 0)) * kh16 + kit * 8);
#pragma unroll
      for (int j = 0; j < 4; ++j) raw[j] = (rv && kit * 8 + 2 * j < kh16) ? __ldg(sp + j) : 0u;
    };
    uint32_t next_raw[4] = {0u, 0u, 0u, 0u};
    Cursor ahead;   // the iteration whose scales are in flight
    ahead.init(it_begin + wg, KI, a.row_tiles);
    if (wg < cnt) fetch_scales(ahead, next_raw);
    int use = 0;    // how many times this group has filled its A stage
    for (int li = wg; li < cnt; li += kDequantGroups, ++use) {
      float dsc[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h2 = *reinterpret_cast<const __half2*>(&next_raw[j]);
        const float2 f2 = __half22float2(h2);
        dsc[2 * j] = f2.x;
        dsc[2 * j + 1] = f2.y;
      }
      if (li + kDequantGroups < cnt) {
        ahead.advance(kDequantGroups, KI, a.row_tiles);
        fetch_scales(ahead, next_raw);
      }
      const int s = li % kStages;
      if (!warp_wait(&sh.full[s], (li / kStages) & 1, abortp)) break;
      const uint8_t* cb = smem + s * kStageBytes + t * 64;
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
          dequant_half<kF16>(c.x, c.y, dsc[2 * kb], cm2, o);
          dequant_half<kF16>(c.z, c.w, dsc[2 * kb + 1], cm2, o + 8);
          tmem_st16(a_stage + lane_base + 16 * kb, o);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.afull[wg][h]);
      }
      if (!ok) break;
    }
  } else if ((warp == 1 || warp == kIssuerWarpB) && lane == 0) {
    // ------------------------------------------------------------ MMA issue
    // Issuer A (warp 1) serves groups 0-1, issuer B groups 2-3: the
    // iterations li with li % 4 in {gb, gb + 1}, in order.  Per half A stage:
    // wait until the group filled it, issue 4 MMAs (K = 16) into the group's
    // accumulator, commit to the half's `afree`; after the second half commit
    // to the stage's `done`; at the end of a portion commit to `dfull`.
    const int gb = (warp == 1) ? 0 : 2;
    const int ib = (warp == 1) ? 0 : 1;
    int use0 = 0, use1 = 0;   // fills of group gb / gb + 1 consumed so far
    bool ok = true;
    for (int pi = 0; pi < nportions && ok; ++pi) {
      const int64_t tile = tile_begin + pi;
      const int pf = static_cast<int>((tile * KI > it_begin ? tile * KI : it_begin) - it_begin);
      const int pe = static_cast<int>(((tile + 1) * KI < it_end ? (tile + 1) * KI : it_end) - it_begin);
      const int db = pi % nsets;
      const uint32_t dpar = static_cast<uint32_t>((pi / nsets) & 1);
      // the accumulator set must be free before any MMA or arrival of this portion
      if (!mbar_wait(&sh.dempty[db], dpar ^ 1u, abortp)) {
        ok = false;
        break;
      }
      const Seg sg = get_seg(a, static_cast<int>(tile / a.row_tiles));
      const int nb = (sg.count + 15) >> 4;
      const uint32_t idesc = kF16 ? idesc_f16(128, 32 * nb) : idesc_bf16(128, 32 * nb);
      bool started0 = false, started1 = false;
      for (int li = pf; li < pe && ok; ++li) {
        const int w = li % kDequantGroups;
        if (w != gb && w != gb + 1) continue;
        const bool second = (w != gb);
        const int use = second ? use1 : use0;
        const bool started = second ? started1 : started0;
        const int s = li % kStages;
        const uint32_t acc = tmem + db * (kAccRegion / nsets) + w * acc_w;
        const uint32_t a_stage = tmem + kACol0 + w * kAColsPerStage;
        const uint32_t xb = smem_u32(smem + s * kStageBytes + kCodesBytes);
        // the B tile (x') of this stage must have landed too
        if (!mbar_wait(&sh.full[s], (li / kStages) & 1, abortp)) {
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
          const uint64_t bdesc0 = sdesc_k128(xb + h * kXHalfBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(acc, a_stage + 32 * h + 8 * kk, bdesc0 + static_cast<uint64_t>(2 * kk), idesc,
                   (!started && h == 0 && kk == 0) ? 0u : 1u);
          mma_commit(&sh.afree[w][h]);
        }
        if (!ok) break;
        mma_commit(&sh.done[s]);
        if (second) {
          started1 = true;
          ++use1;
        } else {
          started0 = true;
          ++use0;
        }
      }
      if (!ok) break;
      if (started0) mma_commit(&sh.dfull[db]);
      else mbar_arrive(&sh.dfull[db]);
      if (started1) mma_commit(&sh.dfull[db]);
      else mbar_arrive(&sh.dfull[db]);
    }
    mma_commit(&sh.issuer_done[ib]);
    drain_wait(&sh.issuer_done[ib], 0);
  } else if (warp >= kFirstEpilogueWarp && warp < kFirstEpilogueWarp + 4) {
    // ------------------------------------------------------------ epilogue
    pdl_wait();   // y, the partials and the counters may still be in use upstream
    const int q = warp & 3;
    const int t = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int sgi = static_cast<int>(tile_begin / a.row_tiles);
    int rt = static_cast<int>(tile_begin - static_cast<int64_t>(sgi) * a.row_tiles);
    for (int pi = 0; pi < nportions; ++pi) {
      const int64_t tile = tile_begin + pi;
      if (pi > 0 && ++rt == a.row_tiles) {
        rt = 0;
        ++sgi;
      }
      const int64_t tile_first = tile * KI;
      const int64_t portion_first = it_begin > tile_first ? it_begin : tile_first;
      const int64_t portion_end = (tile + 1) * KI < it_end ? (tile + 1) * KI : it_end;
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
      // warpgroup w wrote an accumulator iff one of the portion's local
      // iterations is congruent to w mod 4
      const int lpf = static_cast<int>(portion_first - it_begin), plen = static_cast<int>(portion_end - portion_first);
      const uint32_t dbase = tmem + lane_base + db * (kAccRegion / nsets);
      const bool whole = (portion_first == tile_first) && (portion_end == tile_first + KI);
      const int slot = (pi == 0) ? 0 : 1;
      float* pbase = a.partials + ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * 128 + t) * kSegRows;
      for (int c = 0; c < nb; ++c) {
        // hi columns [16c, 16c+16), lo columns [16nb + 16c, +16) of each accumulator
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
        for (int w = 0; w < kDequantGroups; ++w) {
          const int off = ((w - lpf) % kDequantGroups + kDequantGroups) % kDequantGroups;
          if (off >= plen) continue;
          for (int part = 0; part < 2; ++part) {   // hi columns, then lo columns
            uint32_t rr[16];
            tmem_ld16(dbase + w * acc_w + 16 * nb * part + 16 * c, rr);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __fadd_rn(v[j], __uint_as_float(rr[j]));
          }
        }
        if (c == nb - 1) {
          tc_fence_before();
          mbar_arrive(&sh.dempty[db]);
        }
        if (whole) {
          epilogue_store(a, v, 16 * c, row, lane, sg);
        } else {
          float4* pp = reinterpret_cast<float4*>(pbase + 16 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j) pp[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      if (whole) continue;
      // split tile: publish the partial, the last contributor finishes it.
      // The group barrier orders the 128 threads' partial stores before thread
      // 0's release (acq_rel, gpu scope) on the tile counter; the last
      // arriver's acquire orders its reads of the others' partials after it.
      named_bar_sync(1, 128);
      const int64_t c_first = owner_of(tile_first, T, G);
      const int64_t c_last = owner_of(tile_first + KI - 1, T, G);
      if (t == 0) {
        int ncontrib = 0;
        for (int64_t c = c_first; c <= c_last; ++c)
          if (range_begin(c + 1, T, G) > range_begin(c, T, G)) ++ncontrib;
        int old;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(&a.counters[tile]) : "memory");
        sh.last_flag = (old == ncontrib - 1) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (sh.last_flag) {
        for (int ch = 0; ch < nb; ++ch) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
          for (int64_t c = c_first; c <= c_last; ++c) {
            const int64_t cb0 = range_begin(c, T, G);
            if (range_begin(c + 1, T, G) <= cb0) continue;
            const int cslot = (cb0 / KI == tile) ? 0 : 1;
            const float4* src =
                reinterpret_cast<const float4*>(a.partials + ((c * 2 + cslot) * 128 + t) * kSegRows + 16 * ch);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 f = __ldcg(src + j);
              acc[4 * j] = __fadd_rn(acc[4 * j], f.x);
              acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], f.y);
              acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], f.z);
              acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], f.w);
            }
          }
          epilogue_store(a, acc, 16 * ch, row, lane, sg);
        }
        if (t == 0) a.counters[tile] = 0;
      }
      named_bar_sync(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t streamk_smem_bytes() { return static_cast<size_t>(kStages) * kStageBytes + 1024; }

cudaError_t launch_streamk(const void* tm_codes, const void* tm_xhi, const void* tm_xlo, const StreamKArgs& a,
                           int grid, cudaStream_t st) {
  static bool attr_set = false;
  const size_t smem = streamk_smem_bytes();
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(streamk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(streamk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  Codemag cm;
  const CodebookF32& cb = codebook();
  for (int i = 0; i < 8; ++i) cm.v[i] = cb.levels[8 + i];
  const CUtensorMap& m0 = *static_cast<const CUtensorMap*>(tm_codes);
  const CUtensorMap& m1 = *static_cast<const CUtensorMap*>(tm_xhi);
  const CUtensorMap& m2 = *static_cast<const CUtensorMap*>(tm_xlo);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = a.f16 ? cudaLaunchKernelEx(&cfg, streamk_kernel<true>, m0, m1, m2, a, cm)
                        : cudaLaunchKernelEx(&cfg, streamk_kernel<false>, m0, m1, m2, a, cm);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace tq4
