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
//   warps 4-11  two dequant warpgroups (alternate iterations), thread = row:
//               16 B of codes + 8 fp16 scales -> 128 bf16 levels through a
//               per-half-block scaled table looked up with byte permutes,
//               written to tensor memory with tcgen05.st (the MMA A operand);
//   warp 1      one thread issues 8 tcgen05.mma (M=128, N=32*nb, K=16,
//               A from tensor memory, B from shared memory) into a TMEM
//               accumulator and commits to the stage / A-stage barriers;
//   warps 12-15 epilogue, thread = row: tcgen05.ld of the accumulator,
//               hi + lo columns summed, then the mode's store.
// The flattened (segment, row tile, k iteration) space is split evenly over
// the CTAs (stream-K).  A tile split between CTAs is finished by whichever
// contributor arrives last on the tile's counter: it sums all contributors'
// fp32 partials in CTA order (deterministic) and runs the epilogue, so no
// CTA ever waits on another.
#include "tq4_internal.h"

namespace tq4 {
namespace {

constexpr int kThreads = 512;
constexpr int kStages = 8;
constexpr int kAStages = 6;
constexpr int kCodesBytes = 128 * 64;    // 128 rows x 128 k codes
constexpr int kXHalfBytes = 64 * 128;    // 64 rows x 64 k bf16 (one 128-B swizzle span)
constexpr int kXBytes = 2 * kXHalfBytes; // two k-halves
constexpr int kStageBytes = kCodesBytes + kXBytes;
constexpr int kTmemCols = 512;
constexpr int kDCols = 64;
constexpr int kACol0 = 2 * kDCols;
constexpr int kAColsPerStage = 64;
static_assert(kACol0 + kAStages * kAColsPerStage <= kTmemCols, "tensor memory budget");
static_assert(kStages % 2 == 0 && kAStages % 2 == 0, "two dequant warpgroups alternate");

struct SharedState {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t afull[kAStages];
  uint64_t aempty[kAStages];
  uint64_t dfull[2];
  uint64_t dempty[2];
  uint64_t mma_done;
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

// The per-mode store of one finished tile row (thread = weight row `row`).
__device__ __forceinline__ void epilogue_store(const StreamKArgs& a, float (&v)[kSegRows], int row, int lane,
                                               const Seg& sg) {
  if (a.row_scale) {
#pragma unroll
    for (int j = 0; j < kSegRows; ++j)
      if (j < sg.count) v[j] = __fmul_rn(v[j], a.row_scale[sg.row0 + j]);
  }
  if (a.mode == EPI_DENSE) {
    if (row < a.n) {
#pragma unroll
      for (int j = 0; j < kSegRows; ++j)
        if (j < sg.count)
          a.out_a[static_cast<int64_t>(sg.row0 + j) * a.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
    }
  } else if (a.mode == EPI_UP) {
    // h = bf16(relu(u)^2), then rotate the 32-slice held by this warp with the
    // down projection's signs and split into hi/lo rows for the next stage.
    const int slice0 = row - lane;
    if (slice0 < a.n) {
      const bool neg = (a.next_mask >> lane) & 1u;
      const float r = __uint_as_float(0x3E3504F3u);
#pragma unroll
      for (int j = 0; j < kSegRows; ++j) {
        if (j < sg.count) {
          const float hv = relu2_bf16(v[j]);
          const float t = __fmul_rn(warp_fwht32_epi(neg ? -hv : hv, lane), r);
          const __nv_bfloat16 hi = __float2bfloat16_rn(t);
          const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(t, __bfloat162float(hi)));
          const int64_t off = static_cast<int64_t>(sg.row0 + j) * a.n + row;
          a.out_a[off] = __bfloat16_as_ushort(hi);
          a.out_b[off] = __bfloat16_as_ushort(lo);
        }
      }
    }
  } else {
    if (row < a.n) {
#pragma unroll
      for (int j = 0; j < kSegRows; ++j) {
        if (j < sg.count) {
          const int p = a.pairs[sg.row0 + j];
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
  const int nseg = a.segs ? *a.nseg_dev : a.nseg_host;
  const int64_t KI = a.k_iters;
  const int64_t T = static_cast<int64_t>(nseg) * a.row_tiles * KI;
  const int64_t G = gridDim.x;
  const int64_t it_begin = range_begin(blockIdx.x, T, G);
  const int64_t it_end = range_begin(blockIdx.x + 1, T, G);
  const int cnt = static_cast<int>(it_end - it_begin);
  if (cnt <= 0) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&sh.afull[i], 128);
      mbar_init(&sh.aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.dfull[i], 1);
      mbar_init(&sh.dempty[i], 128);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0;
    sh.last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_xhi);
    tma_prefetch_desc(&tm_xlo);
  }
  if (warp == 2) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  volatile int* abortp = &sh.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int armed[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed[i] = -1;
      for (int li = 0; li < cnt; ++li) {
        const int s = li % kStages;
        const uint32_t ph = (li / kStages) & 1;
        if (!mbar_wait(&sh.empty[s], ph ^ 1u, abortp)) break;
        const int64_t it = it_begin + li;
        const int64_t tile = it / KI;
        const int kit = static_cast<int>(it - tile * KI);
        const int sgi = static_cast<int>(tile / a.row_tiles);
        const int rt = static_cast<int>(tile - static_cast<int64_t>(sgi) * a.row_tiles);
        const Seg sg = get_seg(a, sgi);
        const int nb = (sg.count + 15) >> 4;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&sh.full[s], kCodesBytes + nb * 4 * 2048);
        armed[s] = static_cast<int>(ph);
        tma_load_3d(st, &tm_codes, &sh.full[s], kit * 64, rt * 128, sg.e);
        for (int b = 0; b < nb; ++b) {
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int pi = -1;
      for (int li = 0; li < cnt; ++li) {
        const int64_t it = it_begin + li;
        const int64_t tile = it / KI;
        const int kit = static_cast<int>(it - tile * KI);
        const bool first = (li == 0) || (kit == 0);
        const bool last = (li == cnt - 1) || (kit == KI - 1);
        if (first) {
          ++pi;
          if (!mbar_wait(&sh.dempty[pi & 1], ((pi >> 1) & 1) ^ 1u, abortp)) break;
        }
        const int s = li % kStages;
        if (!mbar_wait(&sh.full[s], (li / kStages) & 1, abortp)) break;
        const int as = li % kAStages;
        if (!mbar_wait(&sh.afull[as], (li / kAStages) & 1, abortp)) break;
        tc_fence_after();
        const int sgi = static_cast<int>(tile / a.row_tiles);
        const Seg sg = get_seg(a, sgi);
        const int nb = (sg.count + 15) >> 4;
        const uint32_t idesc = kF16 ? idesc_f16(128, 32 * nb) : idesc_bf16(128, 32 * nb);
        const uint32_t d_addr = tmem + (pi & 1) * kDCols;
        const uint32_t a_addr = tmem + kACol0 + as * kAColsPerStage;
        const uint32_t xb = smem_u32(smem + s * kStageBytes + kCodesBytes);
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint64_t bdesc = sdesc_k128(xb + (k16 >> 2) * kXHalfBytes + (k16 & 3) * 32);
          mma_ts(d_addr, a_addr + 8 * k16, bdesc, idesc, (k16 > 0 || !first) ? 1u : 0u);
        }
        mma_commit(&sh.empty[s]);
        mma_commit(&sh.aempty[as]);
        if (last) mma_commit(&sh.dfull[pi & 1]);
      }
      mma_commit(&sh.mma_done);
      drain_wait(&sh.mma_done, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ dequant
    const int wg = (warp - 4) >> 2;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int t = q * 32 + lane;            // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint64_t cm2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cm2[i] = pack_f32x2(cmag.v[2 * i], cmag.v[2 * i + 1]);
    const int kh16 = a.k / 16;
    for (int li = wg; li < cnt; li += 2) {
      const int64_t it = it_begin + li;
      const int64_t tile = it / KI;
      const int kit = static_cast<int>(it - tile * KI);
      const int sgi = static_cast<int>(tile / a.row_tiles);
      const int rt = static_cast<int>(tile - static_cast<int64_t>(sgi) * a.row_tiles);
      const Seg sg = get_seg(a, sgi);
      const int row = rt * 128 + t;
      float dsc[8];
      {
        const bool rv = row < a.n;
        const uint16_t* sp = a.scales + (static_cast<int64_t>(sg.e) * a.n + (rv ? row : 0)) * kh16 + kit * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool ok = rv && (kit * 8 + j < kh16);
          dsc[j] = ok ? __half2float(__ushort_as_half(__ldg(sp + j))) : 0.0f;
        }
      }
      const int s = li % kStages;
      if (!warp_wait(&sh.full[s], (li / kStages) & 1, abortp)) break;
      const int as = li % kAStages;
      if (!warp_wait(&sh.aempty[as], ((li / kAStages) & 1) ^ 1u, abortp)) break;
      tc_fence_after();
      const uint8_t* cb = smem + s * kStageBytes + t * 64;
      const uint32_t tbase = tmem + lane_base + kACol0 + as * kAColsPerStage;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        const uint4 c = *reinterpret_cast<const uint4*>(cb + 16 * (kb ^ ((t >> 1) & 3)));
        uint32_t o[16];
        dequant_half<kF16>(c.x, c.y, dsc[2 * kb], cm2, o);
        dequant_half<kF16>(c.z, c.w, dsc[2 * kb + 1], cm2, o + 8);
        tmem_st16(tbase + 16 * kb, o);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.afull[as]);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int t = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int pi = -1;
    for (int li = 0; li < cnt; ++li) {
      const int64_t it = it_begin + li;
      const int64_t tile = it / KI;
      const int kit = static_cast<int>(it - tile * KI);
      if (!((li == cnt - 1) || (kit == KI - 1))) continue;
      ++pi;
      const int db = pi & 1;
      // one thread waits; the decision is published before the group barrier
      // so all four epilogue warps leave together on a timeout
      if (t == 0) sh.epi_ok[db] = mbar_wait(&sh.dfull[db], (pi >> 1) & 1, abortp) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!sh.epi_ok[db]) break;
      tc_fence_after();
      const int sgi = static_cast<int>(tile / a.row_tiles);
      const int rt = static_cast<int>(tile - static_cast<int64_t>(sgi) * a.row_tiles);
      const Seg sg = get_seg(a, sgi);
      const int nb = (sg.count + 15) >> 4;
      float v[kSegRows];
      {
        uint32_t r0[16], r1[16];
        const uint32_t dbase = tmem + lane_base + db * kDCols;
        if (nb == 1) {
          tmem_ld16(dbase, r0);
          tmem_ld16(dbase + 16, r1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = __fadd_rn(__uint_as_float(r0[j]), __uint_as_float(r1[j]));
            v[16 + j] = 0.0f;
          }
        } else {
          uint32_t r2[16], r3[16];
          tmem_ld16(dbase, r0);
          tmem_ld16(dbase + 16, r1);
          tmem_ld16(dbase + 32, r2);
          tmem_ld16(dbase + 48, r3);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = __fadd_rn(__uint_as_float(r0[j]), __uint_as_float(r2[j]));
            v[16 + j] = __fadd_rn(__uint_as_float(r1[j]), __uint_as_float(r3[j]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.dempty[db]);

      const int64_t tile_first = tile * KI;
      const int64_t portion_first = it_begin > tile_first ? it_begin : tile_first;
      const bool whole = (portion_first == tile_first) && (kit == KI - 1);
      const int row = rt * 128 + t;
      if (whole) {
        epilogue_store(a, v, row, lane, sg);
        continue;
      }
      // split tile: publish the partial, the last contributor finishes it
      const int slot = (pi == 0) ? 0 : 1;
      float4* pp = reinterpret_cast<float4*>(a.partials +
                                             ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * 128 + t) * kSegRows);
#pragma unroll
      for (int j = 0; j < kSegRows / 4; ++j) pp[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      __threadfence();
      named_bar_sync(1, 128);
      const int64_t c_first = owner_of(tile_first, T, G);
      const int64_t c_last = owner_of(tile_first + KI - 1, T, G);
      if (t == 0) {
        int ncontrib = 0;
        for (int64_t c = c_first; c <= c_last; ++c)
          if (range_begin(c + 1, T, G) > range_begin(c, T, G)) ++ncontrib;
        const int old = atomicAdd(&a.counters[tile], 1);
        sh.last_flag = (old == ncontrib - 1) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (sh.last_flag) {
        __threadfence();
        float acc[kSegRows];
#pragma unroll
        for (int j = 0; j < kSegRows; ++j) acc[j] = 0.0f;
        for (int64_t c = c_first; c <= c_last; ++c) {
          const int64_t cb0 = range_begin(c, T, G);
          if (range_begin(c + 1, T, G) <= cb0) continue;
          const int cslot = (cb0 / KI == tile) ? 0 : 1;
          const float4* src = reinterpret_cast<const float4*>(
              a.partials + ((c * 2 + cslot) * 128 + t) * kSegRows);
#pragma unroll
          for (int j = 0; j < kSegRows / 4; ++j) {
            const float4 f = __ldcg(src + j);
            acc[4 * j] = __fadd_rn(acc[4 * j], f.x);
            acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], f.y);
            acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], f.z);
            acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], f.w);
          }
        }
        epilogue_store(a, acc, row, lane, sg);
        if (t == 0) a.counters[tile] = 0;
      }
      named_bar_sync(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, kTmemCols);
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
  if (a.f16)
    streamk_kernel<true><<<grid, kThreads, smem, st>>>(m0, m1, m2, a, cm);
  else
    streamk_kernel<false><<<grid, kThreads, smem, st>>>(m0, m1, m2, a, cm);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace tq4
