// Decode-block dequant-GEMM for sm_100a: y[m][n] = bf16(x W_hat^T) for
// m <= 32 tokens (a 16-token denoise block), one launch per call.
//
// Route B (as in the stream-K kernel): the activations are rotated instead of
// inverse-rotating the weight, x' = R x per 32-slice with R = r H diag(s)
// ("What Config-I means": per-32-block randomized Walsh-Hadamard rotation;
// R is orthogonal, so x W_hat^T = x' (c[code] d)^T), and the weight side is a
// table lookup and a multiply per weight pair: the rotated-domain levels
// fp16(256 c[code]) * d go to tensor memory as the A operand of tcgen05.mma
// (M = 128 weight rows, N = 16 tokens per block, K = 16), x' (fp16, scaled by
// a power of two per token) is the B operand in shared memory, fp32
// accumulation, exact scaling back in the epilogue.
//
// One CTA = one 128-row tile of W and one k range of at most 8 iterations of
// 128 k; the `split` CTAs of a tile form a thread-block cluster and reduce
// their fp32 partial tiles through distributed shared memory in rank order
// (deterministic).  What this kernel is built around is the chain of calls a
// layer stack makes -- each call's input is the previous call's output --
// where per-call latency, not bandwidth, is the limit, so it moves as much
// work as it can in front of the wait for the previous kernel:
//   * it lets the next kernel launch as soon as all its CTAs are running: the
//     next call's CTAs take SMs as this call's CTAs leave (and the SMs this
//     grid does not use) and do their own set-up meanwhile;
//   * every codes tile of the CTA and its scales tile are requested at entry
//     (one shared-memory stage per iteration; no ring whose refills would
//     queue behind other traffic), before the wait when the weight is
//     flagged static;
//   * the dequant warps then turn as many tiles as tensor memory holds (6 of
//     8 at 16 tokens) into A operands, whether or not the wait has ended;
//   * only the activation-dependent work follows the wait: x comes by TMA
//     straight into the swizzled B tiles; at 16 tokens of TQ4_1S the tensor
//     core multiplies it by the block-diagonal sign-folded Hadamard matrix
//     (elsewhere eight warps butterfly each 32-slice in registers), x' is
//     written back in place as fp16 with a power-of-two scale per token
//     (1 for any activation of ordinary range); then the MMAs, the
//     remaining tiles and the epilogue.
//
// Warps (640 threads, one CTA per SM):
//   4      lane 0: producer of the scales and codes tiles (in that order)
//          and of every barrier but xland (its warp takes no part in the
//          set-up stores);
//   16     lane 0: producer of the x tiles -- its own barrier, the wait and
//          the copy at entry, so that x lands during the set-up (its warp
//          takes no part in the set-up stores either) -- and of a weight not
//          flagged static after the set-up; 16 and 17 lane 0 issue the
//          rotation MMAs;
//   1-3, 17-19  lane 0: MMA issuers, one per (dequant group, 64-k half);
//   0-3    epilogue (thread = tile row) once the MMAs are done, then the
//          cluster reduction of the rows this CTA owns (all warps);
//   4-15   three dequant groups of four warps (thread = tile row): per
//          iteration 16 B of codes + 8 scales -> 128 fp16 levels -> tensor
//          memory, as two 64-k halves signalled separately;
//   0-3, 16-19  the x rotation after the wait.
#include <mutex>
#include <type_traits>

#include "tq4_internal.h"

namespace tq4 {
namespace {

constexpr int kGroups = 3;                 // dequant groups
constexpr int kFirstDqWarp = 4;            // warps 4-15: dequant
constexpr int kHiWarp = kFirstDqWarp + 4 * kGroups;             // warps 16-19: rotation (17-19 also issue)
constexpr int kFirstHiIssuerWarp = kHiWarp + 1;                 // warps 17-19: issuers of the second halves
constexpr int kProducerWarp = kFirstDqWarp;                     // warp 4, lane 0: TMA producer (issue only)
constexpr int kRotWarps = 8;                                    // warps 0-3 and 16-19 rotate x
constexpr int kIssuers = 2 * kGroups;                           // one per (group, 64-k half)
constexpr int kThreads = (kHiWarp + 4) * 32;                    // 640
constexpr int kMaxIters = kFusedMaxIters;  // iterations (128 k) per CTA
constexpr int kStagesD = kMaxIters;        // one codes stage per iteration
constexpr int kCodesTile = 128 * 64;       // codes of one iteration: 128 rows x 64 B
constexpr int kLutBytesD = 256 * 32 * 4;   // fp16 level-pair table, one copy per lane
constexpr int kAColsD = 64;                // tensor-memory columns of one A stage (128 k of fp16)
constexpr int kTmemColsD = 512;
constexpr float kLevelScaleD = 256.0f;
// A stages: the tensor memory beside the accumulators (16 nb columns per group)
__host__ __device__ constexpr int a_stages(int nb) { return (kTmemColsD - kIssuers * 16 * nb) / kAColsD; }

struct DecodeShared {
  uint64_t full[kStagesD];           // codes tile landed (TMA bytes)
  uint64_t afull[kMaxIters][2];      // A stage s, half h holds fresh levels (4 warp arrivals)
  uint64_t afree[kMaxIters][2];      // the MMAs reading A stage s, half h completed
  uint64_t xready;                   // every token's x' is in the B tiles (8 warp arrivals)
  uint64_t dfull;                    // every issuer's MMAs completed (kIssuers arrivals)
  uint64_t idone[kIssuers];          // an issuer's own MMAs completed (teardown)
  uint64_t eready;                   // every dequant thread wrote its row exponent (12 warp arrivals)
  uint64_t xland;                    // the x tiles landed (TMA bytes)
  uint64_t sfull;                    // the scales tile landed (TMA bytes)
  uint64_t rdone;                    // the rotation MMAs completed (tensor-core rotation; one commit per block)
  uint64_t redfull;                  // cluster reduction: every CTA's partial rows of this CTA landed (bytes)
  int8_t rexp[kGroups][128];         // row exponent of each group's levels (see the dequant)
  float row_scale[kSegRows];         // 2^e of each token
  uint32_t tok_max[kSegRows];        // max |x| of each token over the CTA's k range (fp32 bits)
  int own[3];                        // cluster reduction: rows per CTA, first and count of this CTA's rows
  uint32_t tmem_base;
  int abort_flag;
};

// Dynamic shared memory: codes stages | B tiles [iters][2 halves][16 nb rows x 128 B] |
// level table and scales tile [128 rows][64 scales] (TQ4_1S only) | the
// rotation's B operand (16 tokens of TQ4_1S) | cluster reduction buffer
// [split][rows per CTA][16 nb] fp32.  The fp8 cache (f8)
// streams 128 B of codes per row and iteration and needs neither.
__host__ __device__ constexpr int tile_bytes(bool f8) { return f8 ? 2 * kCodesTile : kCodesTile; }
__host__ __device__ constexpr int b_half_bytes(int nb) { return 16 * nb * 128; }
__host__ __device__ constexpr int off_b(bool f8) { return kStagesD * tile_bytes(f8); }
__host__ __device__ constexpr int off_lut(int nb, bool f8) { return off_b(f8) + kMaxIters * 2 * b_half_bytes(nb); }
__host__ __device__ constexpr int off_sc(int nb, bool f8) { return off_lut(nb, f8) + (f8 ? 0 : kLutBytesD); }
constexpr int kScTileBytes = 128 * 128;   // 128 rows x 64 fp16 scales (8 iterations)
// The rotation runs on the tensor core at 16 tokens of TQ4_1S (tc_rotation):
// the B operand is the 64 x 64 block-diagonal matrix diag(H S, H S) in bf16.
__host__ __device__ constexpr bool tc_rotation(int nb, bool f8) { return nb == 1 && !f8; }
constexpr int kRotBBytes = 64 * 128;
__host__ __device__ constexpr int off_rb(int nb, bool f8) { return off_sc(nb, f8) + (f8 ? 0 : kScTileBytes); }
__host__ __device__ constexpr int off_red(int nb, bool f8) { return off_rb(nb, f8) + (tc_rotation(nb, f8) ? kRotBBytes : 0); }
// (the reduction buffer holds split * ceil(128 / split) <= 135 rows)
__host__ __device__ constexpr int smem_total(int nb, bool f8) { return off_red(nb, f8) + 136 * 16 * nb * 4 + 1024; }

// 2^e for an integer e in [-126, 127], from its exponent bits (the library
// call costs tens of instructions on paths where every cycle counts).
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

struct LevelTableD {
  uint32_t h[16];   // fp16 bits of 256 * levels[0..15]
  float max_level;
};

// Dequantize one half-block (16 codes in q0, q1; dd = {d, d} fp16) through
// the lane's copy of the level-pair table: out[i] = {level(2i) d, level(2i+1) d}.
__device__ __forceinline__ void dq_half(uint32_t q0, uint32_t q1, uint32_t dd, uint32_t lut_lane, uint32_t* out) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const uint32_t q = w ? q1 : q0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t idx = prmt(q, 0u, 0x4440u + static_cast<uint32_t>(b));
      uint32_t v;
      asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(lut_lane + idx * 128u));
      uint32_t r;
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(dd));
      out[4 * w + b] = r;
    }
  }
}

__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, volatile int* abortp) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abortp) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(addr, parity)) {
    if (global_timer() - t0 > TQ_WAIT_NS) {
      raise_status(TQ_DEV_TIMEOUT);
      return;
    }
  }
}

// Position of 4-token group gi of local row tl in the reduction buffer's row:
// the groups are XOR-swizzled so that eight consecutive rows' float4 at the
// same gi fall in eight different 16-byte bank groups.
template <int NB>
__device__ __forceinline__ int red_pos(int tl, int gi) {
  return NB == 1 ? (gi ^ ((tl >> 1) & 3)) : (gi ^ (tl & 7));
}

// Asynchronous 16-byte store into CTA `rank` of the cluster; its completion
// counts the bytes on that CTA's mbarrier at the same offset as local_bar.
__device__ __forceinline__ void st_async_v4(uint32_t local_addr, uint32_t local_bar, uint32_t rank, float a, float b,
                                            float c, float d) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(local_bar), "r"(rank));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(ra),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(rb)
               : "memory");
}

// F8: the weight is the fp8-resident cache (E4M3 codes [n][k], one fp32
// scale per row; "Help wanted": dequantize once, keep fp8 resident) instead of
// TQ4_1S: no rotation (the cache is in the weight's own domain), levels are
// the E4M3 values converted to fp16 (exact), and the row scale multiplies the
// accumulator in the epilogue.
template <int NB, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_sc, const DecodeArgs a, const __grid_constant__ LevelTableD lt) {
  __shared__ DecodeShared sh;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  constexpr int kTile = tile_bytes(F8);
  uint8_t* btiles = smem + off_b(F8);
  uint8_t* lut = smem + off_lut(NB, F8);
  uint8_t* red = smem + off_red(NB, F8);
  const uint8_t* sctile = smem + off_sc(NB, F8);
  constexpr int kHalf = b_half_bytes(NB);
  constexpr int kAccW = 16 * NB;           // columns of one accumulator
  constexpr int kACol0 = 0;                // A stages first, then an accumulator per (group, half)
  constexpr int kAccCol0 = a_stages(NB) * kAColsD;
  constexpr bool kTcRot = tc_rotation(NB, F8);
  constexpr int kNA = a_stages(NB);        // A stages in tensor memory (6 at NB == 1, 5 at NB == 2)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = a.split;
  const int tile = blockIdx.x / split;
  const int rank = blockIdx.x - tile * split;
  const int KI = a.k_iters;
  const int it0 = rank * KI / split, it1 = (rank + 1) * KI / split;
  const int cnt = it1 - it0;   // >= 1 (split <= KI), <= kMaxIters (host)
  const int row0 = tile * 128;
  const bool stat = a.static_w != 0;
  volatile int* abortp = &sh.abort_flag;

  // The codes tiles and the scales tile are requested first of all: the
  // producer initialises their barriers and issues the copies before the
  // rest of the set-up, so HBM latency overlaps it.  A weight flagged static
  // is not written by any kernel still in flight, so it may be read before
  // the wait for the previous kernel; otherwise the tiles are only pulled
  // into L2 now and loaded after the wait (by the x producer, below).
  const bool sc_tma = !F8 && a.scales_tma != 0;
  auto issue_weight = [&]() {
    // the scales tile first: every dequant thread needs it before its first
    // iteration, and copies land in about the order they are issued
    if (sc_tma) {
      mbar_arrive_expect_tx(&sh.sfull, kScTileBytes);
      tma_load_2d(const_cast<uint8_t*>(sctile), &tm_sc, &sh.sfull, it0 * 8, row0);
    }
    for (int li = 0; li < cnt; ++li) {
      mbar_arrive_expect_tx(&sh.full[li], kTile);
      tma_load_3d(smem + li * kTile, &tm_codes, &sh.full[li], (it0 + li) * (F8 ? 128 : 64), row0, 0);
    }
  };
  if (warp == kProducerWarp && lane == 0) {
    for (int li = 0; li < cnt; ++li) mbar_init(&sh.full[li], 1);
    mbar_init(&sh.sfull, 1);
    fence_mbar_init();
    if (stat) {
      issue_weight();
    } else {
      for (int li = 0; li < cnt; ++li) tma_prefetch_l2_3d(&tm_codes, (it0 + li) * (F8 ? 128 : 64), row0, 0);
      if (sc_tma) tma_prefetch_l2_2d(&tm_sc, it0 * 8, row0);
    }
    // then the other barriers, first used after the set-up barrier (the
    // producer's warp takes no part in the set-up stores below, so this
    // serial work runs beside them)
    for (int i = 0; i < kMaxIters; ++i) {
      mbar_init(&sh.afull[i][0], 4);
      mbar_init(&sh.afull[i][1], 4);
      mbar_init(&sh.afree[i][0], 1);
      mbar_init(&sh.afree[i][1], 1);
    }
    mbar_init(&sh.xready, kRotWarps);
    mbar_init(&sh.dfull, kIssuers);
    for (int i = 0; i < kIssuers; ++i) mbar_init(&sh.idone[i], 1);
    mbar_init(&sh.eready, 4 * kGroups);
    mbar_init(&sh.rdone, 2);
    mbar_init(&sh.redfull, 1);
    // the bytes this CTA receives in the cluster reduction: its rows from
    // every CTA of the cluster, itself included
    if (split > 1)
      mbar_arrive_expect_tx(&sh.redfull, static_cast<uint32_t>(split * (((rank + 1) * 128 + split - 1) / split -
                                                                         (rank * 128 + split - 1) / split) *
                                                               16 * NB * 4));
    fence_mbar_init();
  }
  // The x producer (lane 0 of warp 16; its warp takes no part in the set-up
  // stores): its own barrier, the wait for the previous kernel (x is its
  // output), and the x tiles at once, so that they land while the set-up
  // runs.  (The B tiles are written by nothing else before the rotation.)
  if (warp == kHiWarp && lane == 0) {
    mbar_init(&sh.xland, 1);
    fence_mbar_init();
    pdl_wait();
    if (a.x_box3) {
      // one 3-D box: all 2 kMaxIters half tiles from this CTA's first k
      // (those past its range land in B tiles it does not use)
      mbar_arrive_expect_tx(&sh.xland, static_cast<uint32_t>(2 * kMaxIters * kHalf));
      tma_load_3d(btiles, &tm_x, &sh.xland, 0, 0, 2 * it0);
    } else {
      mbar_arrive_expect_tx(&sh.xland, static_cast<uint32_t>(2 * cnt * kHalf));
      for (int u = 0; u < 2 * cnt; ++u) tma_load_2d(btiles + u * kHalf, &tm_x, &sh.xland, (2 * it0 + u) * 64, 0);
    }
  }
  const int dq_group = (warp >= kFirstDqWarp && warp < kHiWarp) ? (warp - kFirstDqWarp) >> 2 : -1;
  const int trow = (warp & 3) * 32 + lane;   // tile row of this thread (dequant and epilogue)
  // dequant threads: the scales of their (up to 3) iterations, 16 B each
  uint32_t sraw[3][4];
  auto load_scales = [&]() {
    if (sc_tma) {
      // the tile [128 rows][64 scales] (128-byte swizzle: chunk c of row t at
      // c ^ (t & 7)); iteration li's 8 scales are chunk li of the row
      const bool ok = wwait(&sh.sfull, 0, abortp);
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int li = dq_group + kGroups * u;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (ok && li < cnt) v = *reinterpret_cast<const uint4*>(sctile + trow * 128 + ((li ^ (trow & 7)) << 4));
        sraw[u][0] = v.x;
        sraw[u][1] = v.y;
        sraw[u][2] = v.z;
        sraw[u][3] = v.w;
      }
      return;
    }
    const int row = row0 + trow;
    const int kh16 = a.k / 16;
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int li = dq_group + kGroups * u;
#pragma unroll
      for (int j = 0; j < 4; ++j) sraw[u][j] = 0u;
      if (!F8 && li < cnt && row < a.n) {
        const int kit = it0 + li;
        const uint32_t* sp = reinterpret_cast<const uint32_t*>(a.scales + static_cast<int64_t>(row) * kh16 + kit * 8);
        if ((kh16 & 7) == 0) {
          const uint4 v = __ldcg(reinterpret_cast<const uint4*>(sp));
          sraw[u][0] = v.x;
          sraw[u][1] = v.y;
          sraw[u][2] = v.z;
          sraw[u][3] = v.w;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) sraw[u][j] = (kit * 8 + 2 * j < kh16) ? __ldcg(sp + j) : 0u;
        }
      }
    }
  };
  // the set-up stores below are shared by the warps other than the two
  // producers' (4 and 16)
  constexpr int kSetupWarps = kThreads / 32 - 2;
  const int setup_warp = warp < kProducerWarp ? warp : (warp < kHiWarp ? warp - 1 : warp - 2);
  const bool setup_role = warp != kProducerWarp && warp != kHiWarp;
  if (warp == 0) {
    if (lane == 0) sh.abort_flag = 0;
    sh.tok_max[lane] = 0u;
  } else if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemColsD);
    tmem_relinquish();
  }
  if (!F8) {
    // level-pair table: entry b (a code byte) of lane l's copy at byte
    // 128 b + 4 l holds {256 c[b & 15], 256 c[b >> 4]} (fp16 pair).  Lane j
    // of each warp holds level j; one 16-byte store per lane writes four
    // entries per warp (lane l: entry 4 s + (l >> 3), copies 4 (l & 7) + 0..3),
    // taking the two levels by shuffles.
    const uint32_t hl = lt.h[lane & 15];
    uint4* lw4 = reinterpret_cast<uint4*>(lut);
#pragma unroll
    for (int it = 0; it < (64 + kSetupWarps - 1) / kSetupWarps; ++it) {
      const int s4 = setup_warp + kSetupWarps * it;   // warp-uniform
      if (setup_role && s4 < 64) {
        const int b = 4 * s4 + (lane >> 3);
        const uint32_t lo = __shfl_sync(0xFFFFFFFFu, hl, b & 15), hi = __shfl_sync(0xFFFFFFFFu, hl, b >> 4);
        const uint32_t v = lo | (hi << 16);
        lw4[b * 8 + (lane & 7)] = make_uint4(v, v, v, v);
      }
    }
  }
  if (kTcRot) {
    // The rotation's B operand: row n (output k of a 64-k half tile), column
    // i (input k) holds H[n % 32][i % 32] s[i % 32] when n and i lie in the
    // same 32-slice, else 0 -- H the Walsh-Hadamard matrix in natural order
    // ((-1)^popcount(n & i)), s the signs.  bf16 +-1 and 0 are exact.  K-major,
    // 128-byte swizzle: 8 entries (16 B) per store, chunk c of row n at c ^ (n & 7).
    uint8_t* rb = smem + off_rb(NB, F8);
    for (int t = setup_warp * 32 + lane; setup_role && t < 64 * 8; t += kSetupWarps * 32) {
      const int n = t >> 3, c = t & 7;   // chunk c: inputs 8 c .. 8 c + 7
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if ((n >> 5) == (c >> 2)) {
        // bit i of hb: parity of popcount((n % 32) & i), the sign of H[n][i]
        const int nn = n & 31;
        uint32_t hb = 0u;
        if (nn & 1) hb ^= 0xAAAAAAAAu;
        if (nn & 2) hb ^= 0xCCCCCCCCu;
        if (nn & 4) hb ^= 0xF0F0F0F0u;
        if (nn & 8) hb ^= 0xFF00FF00u;
        if (nn & 16) hb ^= 0xFFFF0000u;
        const uint32_t bits = ((hb ^ a.sign_bits) >> (8 * (c & 3))) & 0xFFu;
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)
          w[e2] = 0x3F803F80u | (((bits >> (2 * e2)) & 1u) << 15) | (((bits >> (2 * e2 + 1)) & 1u) << 31);
      }
      *reinterpret_cast<uint4*>(rb + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
  }
  // All CTAs of this grid are resident once every one of them is here: the
  // next kernel may launch now.  Its CTAs take the SMs this grid leaves free
  // and those its CTAs release, and set up meanwhile; anything of theirs that
  // reads this kernel's output waits in griddepcontrol.wait.  (Before the
  // set-up barrier, which the x producer reaches only after its wait.)
  if (threadIdx.x == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every CTA of the cluster has initialised its barriers once all have
  // arrived here; the epilogue waits for that before its first remote store.
  if (split > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const uint32_t tmem = sh.tmem_base;

  // ------------------------------------------------------------ dequant
  // Group g dequantizes iterations g, g + 3, g + 6 of the CTA into A stage
  // li % kNA; an iteration past the first kNA reuses a stage once the MMAs of
  // the iteration kNA before it have read it.  Before the wait (static
  // weight) a group does the iterations that need no stage back; the rest
  // after the rotation.  (A stages in shared memory, tried for the last two
  // iterations, were slower: their 16-byte stores double the dequant's
  // shared-memory traffic, which already bounds its rate.)
  uint32_t ff = 0u;   // {2^-e, 2^-e}: this thread's row exponent (see below)
  int dq_done = 0;    // iterations of this group dequantized so far
  auto dq_exponent = [&]() {
    // Row exponent of this group's levels: the scales of the group's
    // iterations are multiplied by 2^-e (exact) so that the largest lies in
    // [32, 64) -- levels fp16(256 c) * d 2^-e then stay normal and finite for
    // every finite fp16 scale -- and the epilogue multiplies the group's
    // accumulator by 2^e (exact).
    uint32_t dmax = 0u;
#pragma unroll
    for (int u = 0; u < 3; ++u)
#pragma unroll
      for (int j = 0; j < 4; ++j) asm("max.f16x2 %0, %1, %2;" : "=r"(dmax) : "r"(dmax), "r"(sraw[u][j]));
    const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dmax));
    const float mx = fmaxf(dm.x, dm.y);
    int e = 0;
    if (mx > 0.0f && isfinite(mx)) {
      int ex;
      frexpf(mx, &ex);   // mx in [2^(ex-1), 2^ex)
      e = ex - 6;
      e = e < -15 ? -15 : (e > 14 ? 14 : e);
    }
    sh.rexp[dq_group][trow] = static_cast<int8_t>(e);
    ff = static_cast<uint32_t>(15 - e) * 0x04000400u;   // {2^-e, 2^-e} in fp16 (normal for e in [-15, 14])
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.eready);
  };
  // Dequantize this group's iterations up to (excluding) `li_end`; false on abort.
  auto dq_run = [&](int li_end) -> bool {
    const int g = dq_group;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t lut_lane = smem_u32(lut) + 4u * static_cast<uint32_t>(lane);
    for (;;) {
      const int li = g + kGroups * dq_done;
      if (li >= li_end || li >= cnt) return true;
      const int sa = li % kNA;
      const uint32_t a_stage = tmem + kACol0 + sa * kAColsD;
      if (!wwait(&sh.full[li], 0, abortp)) return false;
      const uint8_t* cb = smem + li * kTile + trow * (F8 ? 128 : 64);
      uint32_t sr[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sr[j] = (dq_done == 0) ? sraw[0][j] : (dq_done == 1 ? sraw[1][j] : sraw[2][j]);
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(sr[j]) : "r"(sr[j]), "r"(ff));
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (li >= kNA && !wwait(&sh.afree[sa][h], ((li / kNA) - 1) & 1, abortp)) return false;
        tc_fence_after();
#pragma unroll
        for (int kb2 = 0; kb2 < 2; ++kb2) {
          const int kb = 2 * h + kb2;
          uint32_t o[16];
          if (F8) {
            // fp8 cache: 128 B of E4M3 codes per row (128-byte swizzle: 16-byte
            // chunk c of row t at chunk c ^ (t & 7)); each byte pair converts to
            // an fp16 pair exactly
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const uint4 c = *reinterpret_cast<const uint4*>(cb + 16 * ((2 * kb + ch) ^ (trow & 7)));
              const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
              for (int j = 0; j < 4; ++j)
                asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                    "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
                    : "=r"(o[8 * ch + 2 * j]), "=r"(o[8 * ch + 2 * j + 1])
                    : "r"(cw[j]));
            }
          } else {
            // TQ4_1S: 16 B of codes (64-byte swizzle: chunk kb of row t at
            // kb ^ ((t >> 1) & 3)), each byte a pair of codes looked up in the
            // lane's table, times the pair of scaled half-block scales
            const uint4 c = *reinterpret_cast<const uint4*>(cb + 16 * (kb ^ ((trow >> 1) & 3)));
            dq_half(c.x, c.y, prmt(sr[kb], 0u, 0x1010u), lut_lane, o);
            dq_half(c.z, c.w, prmt(sr[kb], 0u, 0x3232u), lut_lane, o + 8);
          }
          tmem_st16(a_stage + lane_base + 16 * kb, o);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.afull[sa][h]);
      }
      ++dq_done;
    }
  };
  // The dequant warps read the weight only through the tiles the producers
  // copy -- after the wait for the previous kernel when it is not flagged
  // static -- except for the scales when they come by plain loads: only then
  // do they wait for the previous kernel themselves.  (One call site of the
  // dequant loop keeps the kernel's code compact.)
  if (dq_group >= 0) {
    if (!stat && !sc_tma) {
      if (!F8 && row0 + trow < a.n) {
        // the scales this thread will load after the wait, pulled into L2 now
        const uint16_t* sp0 = a.scales + static_cast<int64_t>(row0 + trow) * (a.k / 16);
        for (int u = 0; u < 3; ++u) {
          const int li = dq_group + kGroups * u;
          if (li < cnt) asm volatile("prefetch.global.L2 [%0];" ::"l"(sp0 + (it0 + li) * 8));
        }
      }
      pdl_wait();
    }
    load_scales();
    dq_exponent();
    dq_run(kMaxIters);
  } else {
    pdl_wait();
  }
  // A weight not flagged static is copied after the wait too, by the x
  // producer (its barriers come from the set-up).
  if (warp == kHiWarp && lane == 0 && !stat) issue_weight();

  // ------------------------------------------------------------ x rotation
  // x came by TMA straight into the B tiles: half tile u = 2 li + h holds the
  // 16 nb tokens' 64 k of iteration li, half h, as bf16 in the layout the MMA
  // reads (K-major rows of 128 B, 8-row groups 1024 B apart, 16-byte chunks
  // XOR-swizzled by row; tokens past m and k past the end are zero).  A
  // 32-slice of a token is four chunks of one row, so it is rotated in place:
  // bf16 in, fp16 x' 2^-e out, the same bytes.  The eight warps that do not
  // dequantize (0-3 and 16-19) take the half tiles round-robin; lane l takes
  // the slice at chunks 4 (l >> 4) + 0..3 of token l & 15 (and of token
  // 16 + (l & 15) at nb = 2), so the eight lanes of a quarter warp touch
  // eight different chunk positions: no bank conflicts.  The scale 2^e of a
  // token is common to its whole k range in the CTA (one accumulator).  On
  // the tensor-core path x' is converted at e = 0 while its exact max |x'|
  // per token is taken, and only tokens whose max falls outside [2^-4, 2^15)
  // are converted again (see there).  On the register path a first pass
  // takes max |x| per token (shared-memory atomic max, then a barrier of the
  // rotation warps), and e puts 5.66 max |x| >= sqrt(32) max |x| -- a bound
  // on |x'|, each x' being r = 1/sqrt(32) times a sum of 32 signed x -- in
  // [2^13, 2^14), so fp16 cannot overflow.  Signs flip bf16 sign bits; the
  // butterfly runs in registers in the fixed stage order.
  const int rot = warp < 4 ? warp : ((warp >= kHiWarp && warp < kHiWarp + 4) ? warp - kHiWarp + 4 : -1);
  if (rot >= 0 && kTcRot) {
    // Tensor-core rotation (16 tokens of TQ4_1S): the x tiles as A (bf16,
    // 128 rows = 8 half tiles x 16 tokens per block, K = 64 k) times the
    // block-diagonal sign-folded Hadamard matrix as B give x' / r in tensor
    // memory (the accumulators' columns, free until the main MMAs).  Rotation
    // warp (w & 3, block w >= 16) reads row 32 (w & 3) + lane of its block:
    // half tile 8 block + row / 16, token row % 16.
    const bool xok = wwait(&sh.xland, 0, abortp);
    if ((warp == kHiWarp || warp == kHiWarp + 1) && lane == 0) {
      // lane 0 of warp 16 issues block 0, of warp 17 block 1 (when the CTA
      // has more than 4 iterations), each committing once to rdone
      const int b = warp - kHiWarp;
      if (xok && (b == 0 || cnt > 4)) {
        tc_fence_after();
        const uint64_t rbd = sdesc_k128(smem_u32(smem + off_rb(NB, F8)));
        const uint32_t idr = idesc_bf16(128, 64);
        const uint64_t ad = sdesc_k128(smem_u32(btiles + b * 8 * kHalf));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kAccCol0 + 64 * b, ad + static_cast<uint64_t>(2 * kk), rbd + static_cast<uint64_t>(2 * kk), idr,
                 kk > 0 ? 1u : 0u);
        mma_commit(&sh.rdone);
      } else {
        mbar_arrive(&sh.rdone);
      }
    }
    __syncwarp();
    const int trw = (warp & 3) * 32 + lane;      // row of the block (tensor-memory lane)
    const int blk = warp >= kHiWarp ? 1 : 0;
    const int u = 8 * blk + (trw >> 4), t = trw & 15;
    const bool live = xok && u < 2 * cnt;
    uint8_t* rowp = btiles + u * kHalf + (t >> 3) * 1024 + (t & 7) * 128;
    const bool rok = wwait(&sh.rdone, 0, abortp);
    tc_fence_after();
    const uint32_t taddr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kAccCol0 + 64 * blk;
    // x R2 = x' / r from tensor memory to fp16, in place (the factor r joins
    // the token scale of the epilogue).  A token's scale 2^-e is common to
    // its whole k range in the CTA, and every value of it must come out
    // finite and, to keep full precision, not too small: the first pass
    // converts with e = 0 and takes the token's exact max |x R2| (a
    // shared-memory atomic max over the rows of the token; non-negative
    // floats order as their bits; a NaN is left out of the max and shows in
    // the output).  Tokens whose max lies in [2^-4, 2^15) -- about any
    // activation -- keep it; the others are converted again with the e that
    // puts the max in [2^13, 2^14) (e = 0 for an infinite max, which then
    // shows in the output as it should).
    auto convert = [&](auto scaled, float rd) -> float {
      float mx = 0.0f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t rv[32];
        tmem_ld32(taddr + 32 * hh, rv);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t hw[4];
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
              float v0 = __uint_as_float(rv[8 * j + 2 * c2]), v1 = __uint_as_float(rv[8 * j + 2 * c2 + 1]);
              if constexpr (decltype(scaled)::value) {
                v0 = __fmul_rn(v0, rd);
                v1 = __fmul_rn(v1, rd);
              } else {
                mx = fmaxf(mx, fmaxf(fabsf(v0), fabsf(v1)));
              }
              const __half2 hh2 = __floats2half2_rn(v0, v1);
              hw[c2] = *reinterpret_cast<const uint32_t*>(&hh2);
            }
            *reinterpret_cast<uint4*>(rowp + (((4 * hh + j) ^ (t & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
      }
      return mx;
    };
    if (xok && rok) {
      uint32_t mb = __float_as_uint(convert(std::false_type{}, 1.0f));   // max |x R2| of this row, e = 0
      // the token's two rows of this warp combined, then over the warps
      const uint32_t ob = __shfl_xor_sync(0xFFFFFFFFu, mb, 16);
      mb = mb > ob ? mb : ob;
      if (lane < 16 && mb != 0u) atomicMax(&sh.tok_max[t], mb);
    }
    named_bar_sync(1, kRotWarps * 32);
    if (xok && rok) {
      const uint32_t tb = sh.tok_max[t];
      int e = 0;
      const bool keep = tb == 0u || (tb >= 0x3D800000u && tb < 0x47000000u);   // 0, or [2^-4, 2^15)
      if (!keep && tb < 0x7F800000u) {
        int ex;
        frexpf(__uint_as_float(tb), &ex);   // max in [2^(ex-1), 2^ex)
        e = ex - 14;
        e = e < -100 ? -100 : (e > 100 ? 100 : e);
      }
      if (blk == 0 && trw < 16) sh.row_scale[t] = exp2i(e);
      // (warp-uniform: tcgen05.ld is warp-collective)
      if (__any_sync(0xFFFFFFFFu, !keep && e != 0)) convert(std::true_type{}, exp2i(-e));
    }
    tc_fence_before();          // the tensor-memory reads, before the main MMAs reuse the columns
    fence_proxy_async_smem();   // generic-proxy writes, before the tensor core reads them
    __syncwarp();
    if (lane == 0 && !(a.test_withhold && rot == 7)) mbar_arrive(&sh.xready);
    if (warp == kHiWarp && lane == 0 && *abortp) {
      for (int li = 0; li < cnt; ++li) drain(&sh.full[li], 0);
      if (sc_tma) drain(&sh.sfull, 0);
      drain(&sh.xland, 0);
      drain(&sh.rdone, 0);
    }
  } else if (rot >= 0) {
    const bool xok = wwait(&sh.xland, 0, abortp);
    const int nunits = 2 * cnt;
    const int tl = lane & 15, c0 = (lane >> 4) * 4;
    if (xok) {
      uint32_t m16[NB];
#pragma unroll
      for (int rr = 0; rr < NB; ++rr) m16[rr] = 0u;
      for (int u = rot; u < nunits; u += kRotWarps) {
#pragma unroll
        for (int rr = 0; rr < NB; ++rr) {
          const int t = tl + 16 * rr;
          const uint8_t* rowp = btiles + u * kHalf + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(rowp + (((c0 + q) ^ (t & 7)) << 4));
            m16[rr] = __vmaxu2(m16[rr], w4.x & 0x7FFF7FFFu);
            m16[rr] = __vmaxu2(m16[rr], w4.y & 0x7FFF7FFFu);
            m16[rr] = __vmaxu2(m16[rr], w4.z & 0x7FFF7FFFu);
            m16[rr] = __vmaxu2(m16[rr], w4.w & 0x7FFF7FFFu);
          }
        }
      }
#pragma unroll
      for (int rr = 0; rr < NB; ++rr) {
        uint32_t mb = m16[rr] >> 16 > (m16[rr] & 0xFFFFu) ? m16[rr] >> 16 : (m16[rr] & 0xFFFFu);
        const uint32_t ob = __shfl_xor_sync(0xFFFFFFFFu, mb, 16);   // the token's other slice position
        mb = mb > ob ? mb : ob;
        if (lane < 16 && mb != 0u) atomicMax(&sh.tok_max[tl + 16 * rr], mb << 16);
      }
    }
    named_bar_sync(1, kRotWarps * 32);
    if (xok) {
      const float r = __uint_as_float(0x3E3504F3u);
#pragma unroll 1
      for (int u = rot; u < nunits; u += kRotWarps) {
#pragma unroll 1
        for (int rr = 0; rr < NB; ++rr) {
          const int t = tl + 16 * rr;
          const float tmx = __uint_as_float(sh.tok_max[t]);   // max |x| (NaN, Inf: bits above Inf)
          const float bound = F8 ? tmx : __fmul_rn(tmx, 5.66f);
          int e = 0;
          if (bound > 0.0f && isfinite(bound)) {
            int ex;
            frexpf(bound, &ex);   // bound in [2^(ex-1), 2^ex)
            e = ex - 14;
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
          }
          if (rot == 0 && u == 0 && lane < 16) sh.row_scale[t] = exp2i(e);
          const float rd = F8 ? exp2i(-e) : __fmul_rn(r, exp2i(-e));   // exact
          uint8_t* rowp = btiles + u * kHalf + (t >> 3) * 1024 + (t & 7) * 128;
          float v[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(rowp + (((c0 + q) ^ (t & 7)) << 4));
            const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const uint32_t sw = F8 ? ww[e2] : (ww[e2] ^ a.x_sign[4 * q + e2]);
              v[8 * q + 2 * e2] = __uint_as_float(sw << 16);
              v[8 * q + 2 * e2 + 1] = __uint_as_float(sw & 0xFFFF0000u);
            }
          }
          if (!F8) {
#pragma unroll
            for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (!(j & h)) {
                  const float p = v[j], q = v[j + h];
                  v[j] = __fadd_rn(p, q);
                  v[j + h] = __fsub_rn(p, q);
                }
              }
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t hw[4];
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
              const __half2 hh = __floats2half2_rn(__fmul_rn(v[8 * q + 2 * c2], rd), __fmul_rn(v[8 * q + 2 * c2 + 1], rd));
              hw[c2] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(rowp + (((c0 + q) ^ (t & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
      }
    }
    fence_proxy_async_smem();   // generic-proxy writes, before the tensor core reads them
    __syncwarp();
    if (lane == 0 && !(a.test_withhold && rot == 7)) mbar_arrive(&sh.xready);
    // the x producer: on an abort, every copy it or the weight producer issued lands before exit
    if (warp == kHiWarp && lane == 0 && *abortp) {
      for (int li = 0; li < cnt; ++li) drain(&sh.full[li], 0);
      if (sc_tma) drain(&sh.sfull, 0);
      drain(&sh.xland, 0);
    }
  }

  if (((warp >= 1 && warp <= kGroups) || warp >= kFirstHiIssuerWarp) && lane == 0) {
    // ------------------------------------------------------------ MMA issue
    // Issuer (g, h): the 4 MMAs of half h of each of group g's iterations,
    // into its own accumulator (single-thread issue costs ~65 cycles per
    // instruction at this N, so six threads issue in parallel).
    const int g = warp >= kFirstHiIssuerWarp ? warp - kFirstHiIssuerWarp : warp - 1;
    const int h = warp >= kFirstHiIssuerWarp ? 1 : 0;
    const int ii = 2 * g + h;
    const uint32_t acc = tmem + kAccCol0 + ii * kAccW;
    const uint32_t idesc = idesc_f16(128, 16 * NB);
    bool ok = mbar_wait(&sh.xready, 0, abortp);
    int use = 0;
    for (int li = g; ok && li < cnt; li += kGroups, ++use) {
      const int sa = li % kNA;
      const uint32_t a_stage = tmem + kACol0 + sa * kAColsD;
      if (!mbar_wait(&sh.afull[sa][h], (li / kNA) & 1, abortp)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t bdesc = sdesc_k128(smem_u32(btiles + (li * 2 + h) * kHalf));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(acc, a_stage + 32 * h + 8 * kk, bdesc + static_cast<uint64_t>(2 * kk), idesc,
               (use == 0 && kk == 0) ? 0u : 1u);
      mma_commit(&sh.afree[sa][h]);
    }
    if (use > 0) mma_commit(&sh.dfull);
    else mbar_arrive(&sh.dfull);
    // its MMAs complete before the CTA can release tensor memory
    mma_commit(&sh.idone[ii]);
    drain(&sh.idone[ii], 0);
  }
  if (warp < 4) {
    __syncwarp();
    // ------------------------------------------------------------ epilogue
    // thread = tile row trow; the groups' accumulators summed in group order,
    // each scaled back by its row exponent, then by the token's 2^e and the
    // level factor (TQ4_1S) or the row's scale (fp8 cache) -- all exact but
    // the last.  (xready also orders the token scales the rotation wrote.)
    // (the owner and local row of this thread's row, and the rows this CTA
    // owns, before the waits)
    const int q_own = (trow * split) >> 7;
    const int rpc = (128 + split - 1) / split;
    const int tl_own = trow - (q_own * 128 + split - 1) / split;
    if (threadIdx.x == 0) {
      const int r0 = (rank * 128 + split - 1) / split;
      sh.own[0] = rpc;
      sh.own[1] = r0;
      sh.own[2] = ((rank + 1) * 128 + split - 1) / split - r0;
    }
    int ok = 0;
    if (lane == 0)
      ok = (mbar_wait(&sh.xready, 0, abortp) && mbar_wait(&sh.eready, 0, abortp) && mbar_wait(&sh.dfull, 0, abortp))
               ? 1
               : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0) && !*abortp;   // (a timed-out role: no output)
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int ngroups = cnt < kGroups ? cnt : kGroups;   // groups (and their two accumulators) with work
    // (the tensor-core rotation leaves the factor r = 1/sqrt(32) of x' to here)
    const float wsc = F8 ? ((row0 + trow < a.n) ? __ldcg(a.wscale + row0 + trow) : 0.0f)
                         : (kTcRot ? __uint_as_float(0x3E3504F3u) / kLevelScaleD : 1.0f / kLevelScaleD);
    if (split > 1) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    // the cluster reduction counts bytes: every CTA sends all its rows, zeros
    // when a role timed out
    if (ok || split > 1) {
#pragma unroll
      for (int c = 0; c < NB; ++c) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
        for (int g = 0; ok && g < ngroups; ++g) {
          // the group's two accumulators (its 64-k halves), one wait for both
          uint32_t r0[16], r1[16];
          tmem_ld16(tmem + lane_base + kAccCol0 + (2 * g) * kAccW + 16 * c, r0);
          tmem_ld16(tmem + lane_base + kAccCol0 + (2 * g + 1) * kAccW + 16 * c, r1);
          tmem_wait_ld();
          // 2^e from its exponent bits (e in [-15, 14]); r * 2^e is exact, so
          // the fused multiply-add rounds as the separate add would
          const float rs = exp2i(sh.rexp[g][trow]);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __fmaf_rn(__uint_as_float(r0[j]), rs, v[j]);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __fmaf_rn(__uint_as_float(r1[j]), rs, v[j]);
        }
        if (ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], __fmul_rn(sh.row_scale[16 * c + j], wsc));
        }
        if (split > 1) {
          // row trow goes to the CTA that owns it: [source rank][row - owner's
          // first row][16 nb tokens], its 4-token groups swizzled (red_pos)
          const uint32_t dst = smem_u32(red) + static_cast<uint32_t>((rank * rpc + tl_own) * 16 * NB * 4);
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            st_async_v4(dst + 16u * static_cast<uint32_t>(red_pos<NB>(tl_own, 4 * c + j / 4)), smem_u32(&sh.redfull),
                        static_cast<uint32_t>(q_own), v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else {
          const int row = row0 + trow;
          if (row < a.n) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (16 * c + j < a.m)
                a.y[static_cast<int64_t>(16 * c + j) * a.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (split > 1) {
    // The other warps' half of the cluster barrier (the epilogue warps passed
    // it before their stores).  Then this CTA's rows from every CTA of the
    // cluster: the byte count completes even when a role timed out (zeros
    // are sent), so once it has, no other CTA writes here and this CTA may
    // leave whenever it is done.
    if (warp >= 4) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    // (a bounded wait that does not give up on this CTA's abort flag: the
    // other CTAs' stores must land before this CTA may exit)
    int rok = 1;
    if (lane == 0) {
      const uint32_t addr = smem_u32(&sh.redfull);
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(addr, 0)) {
        if (global_timer() - t0 > TQ_WAIT_NS) {
          raise_status(TQ_DEV_TIMEOUT);
          *abortp = 1;
          rok = 0;
          break;
        }
      }
    }
    rok = __shfl_sync(0xFFFFFFFFu, rok, 0);
    if (rok && !sh.abort_flag) {
      // thread -> (local row tl, 4-token group gi), lanes along rows: the
      // float4 reads are free of bank conflicts and the stores of one token
      // are coalesced; partials summed in source-rank order
      constexpr int kG = 4 * NB;   // 4-token groups per row
      const int rpc_own = sh.own[0], r0_own = sh.own[1], nrow_own = sh.own[2];
      const int idx = threadIdx.x;
      const int tl = (idx & 31) + 32 * ((idx >> 5) / kG), gi = (idx >> 5) % kG;
      if (tl < nrow_own && 4 * gi < a.m) {
        const int row = row0 + r0_own + tl;
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        const float* rb = reinterpret_cast<const float*>(red) + 4 * red_pos<NB>(tl, gi);
        for (int q = 0; q < split; ++q) {
          const float4 p = *reinterpret_cast<const float4*>(rb + (q * rpc_own + tl) * 16 * NB);
          acc.x = __fadd_rn(acc.x, p.x);
          acc.y = __fadd_rn(acc.y, p.y);
          acc.z = __fadd_rn(acc.z, p.z);
          acc.w = __fadd_rn(acc.w, p.w);
        }
        if (row < a.n) {
          const float av[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * gi + u < a.m)
              a.y[static_cast<int64_t>(4 * gi + u) * a.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(av[u]));
        }
      }
    }
  }
  if (warp == 1) tmem_dealloc(tmem, kTmemColsD);
}

template <int NB, bool F8>
cudaError_t launch_decode_nb(const void* tm_codes, const void* tm_x, const void* tm_scales, const DecodeArgs& a,
                             cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  const int smem = smem_total(NB, F8);
  cudaError_t e0 = once_per_device(attr_done, [&] {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<NB, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<NB, F8>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
  });
  if (e0 != cudaSuccess) return e0;
  static const LevelTableD lt = [] {
    LevelTableD t;
    const CodebookF32& cb = codebook();
    for (int i = 0; i < 16; ++i)
      t.h[i] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(cb.levels[i] * kLevelScaleD)));
    t.max_level = __half2float(__float2half_rn(cb.levels[15] * kLevelScaleD));
    return t;
  }();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.row_tiles * a.split));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.split > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(a.split);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  const CUtensorMap& m0 = *static_cast<const CUtensorMap*>(tm_codes);
  const CUtensorMap& m1 = *static_cast<const CUtensorMap*>(tm_x);
  // (no scales map: any valid map stands in; the kernel does not read it)
  const CUtensorMap& m2 = *static_cast<const CUtensorMap*>(a.scales_tma ? tm_scales : tm_codes);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<NB, F8>, m0, m1, m2, a, lt);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

template <int NB, bool F8>
int decode_max_clusters_nb(int s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(s));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_total(NB, F8));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(s);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaFuncSetAttribute(decode_kernel<NB, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_total(NB, F8)) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<NB, F8>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

size_t decode_smem_bytes(int nb, bool f8) {
  return static_cast<size_t>(nb == 1 ? (f8 ? smem_total(1, true) : smem_total(1, false))
                                     : (f8 ? smem_total(2, true) : smem_total(2, false)));
}

cudaError_t launch_decode(const void* tm_codes, const void* tm_x, const void* tm_scales, const DecodeArgs& a,
                          cudaStream_t st) {
  if (a.fp8)
    return a.nb == 1 ? launch_decode_nb<1, true>(tm_codes, tm_x, tm_scales, a, st)
                     : launch_decode_nb<2, true>(tm_codes, tm_x, tm_scales, a, st);
  return a.nb == 1 ? launch_decode_nb<1, false>(tm_codes, tm_x, tm_scales, a, st)
                   : launch_decode_nb<2, false>(tm_codes, tm_x, tm_scales, a, st);
}

int choose_decode_split(int64_t tiles, int64_t k_iters, int sms, int nb, bool f8) {
  // the largest s in [1, 8] with s <= k_iters, at most kMaxIters iterations
  // per CTA, one CTA per SM (tiles * s <= sms) and all clusters resident at
  // once; 0 if none fits.  Cluster capacities are queried once per device.
  static std::mutex mu;
  static int cap[64][4][9];   // per (nb, format): resident clusters + 1 (0 = not queried yet)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  for (int s = 8; s >= 1; --s) {
    if (s > k_iters || (k_iters + s - 1) / s > kMaxIters || tiles * s > sms) continue;
    if (s == 1) return 1;
    int c;
    {
      std::lock_guard<std::mutex> g(mu);
      int& slot = cap[dev][(nb == 1 ? 0 : 1) + (f8 ? 2 : 0)][s];
      if (slot == 0)
        slot = (f8 ? (nb == 1 ? decode_max_clusters_nb<1, true>(s) : decode_max_clusters_nb<2, true>(s))
                   : (nb == 1 ? decode_max_clusters_nb<1, false>(s) : decode_max_clusters_nb<2, false>(s))) +
               1;
      c = slot - 1;
    }
    if (tiles <= c) return s;
  }
  return 0;
}

}  // namespace tq4
