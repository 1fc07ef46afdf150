// Tensor-core GEMM for large m on sm_100a: y[m][n] = bf16(x[m][k] * W[n][k]^T)
// with bf16 operands and fp32 accumulation in tensor memory.
//
// This is the large-m half of the quantized linear layer (the model card's
// "bf16 tensor-core dequant", section "Performance"): the packed weight is
// first dequantized to bf16 W_hat by a streaming pre-pass, then multiplied
// here.  Persistent CTAs (one per SM) walk 128 x 256 output tiles, m fastest
// so that concurrently running CTAs share weight tiles in L2.
//   warp 0     TMA producer: 128x64 x tile and 256x64 W tile per stage,
//              128-byte swizzle, 4-stage mbarrier ring;
//   warp 1     one thread issues tcgen05.mma M=128 N=256 K=16 (4 per stage)
//              into one of two TMEM accumulators (512 columns in all);
//   warp 2     allocates / frees tensor memory;
//   warps 4-7  epilogue, thread = output row: tcgen05.ld, bf16, 16-B stores;
//              the second accumulator lets the next tile's MMAs overlap.
#include "tq4_internal.h"

namespace tq4 {
namespace {

constexpr int kThreads = 256;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;

struct GemmShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t dfull[2];
  uint64_t dempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok[2];
};

__device__ __forceinline__ void drain_wait_g(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(addr, parity)) {
    if (global_timer() - t0 > TQ_WAIT_NS) {
      raise_status(TQ_DEV_TIMEOUT);
      return;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     uint16_t* __restrict__ y, int32_t m, int32_t n, int32_t k) {
  __shared__ GemmShared sh;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (m + kBM - 1) / kBM;
  const int tiles_n = (n + kBN - 1) / kBN;
  const int tiles = tiles_m * tiles_n;
  const int kiters = (k + kBK - 1) / kBK;
  if (static_cast<int>(blockIdx.x) >= tiles) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.dfull[i], 1);
      mbar_init(&sh.dempty[i], 128);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
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
    if (lane == 0) {
      int armed[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) armed[i] = -1;
      int li = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int mt = tile % tiles_m, nt = tile / tiles_m;
        for (int kk = 0; kk < kiters; ++kk, ++li) {
          const int s = li % kStages;
          const uint32_t ph = (li / kStages) & 1;
          if (!mbar_wait(&sh.empty[s], ph ^ 1u, abortp)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&sh.full[s], kStageBytes);
          armed[s] = static_cast<int>(ph);
          tma_load_2d(st, &tm_x, &sh.full[s], kk * kBK, mt * kBM);
          tma_load_2d(st + kABytes, &tm_w, &sh.full[s], kk * kBK, nt * kBN);
        }
      }
      if (*abortp)
        for (int i = 0; i < kStages; ++i)
          if (armed[i] >= 0) drain_wait_g(&sh.full[i], static_cast<uint32_t>(armed[i]));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, kBN);
      int li = 0, ti = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++ti) {
        const int db = ti & 1;
        if (!mbar_wait(&sh.dempty[db], ((ti >> 1) & 1) ^ 1u, abortp)) break;
        tc_fence_after();
        const uint32_t d_addr = tmem + db * kBN;
        for (int kk = 0; kk < kiters; ++kk, ++li) {
          const int s = li % kStages;
          if (!mbar_wait(&sh.full[s], (li / kStages) & 1, abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16)
            mma_ss(d_addr, sdesc_k128(a0 + k16 * 32), sdesc_k128(b0 + k16 * 32), idesc, (kk | k16) ? 1u : 0u);
          mma_commit(&sh.empty[s]);
        }
        if (ok) mma_commit(&sh.dfull[db]);
      }
      mma_commit(&sh.mma_done);
      drain_wait_g(&sh.mma_done, 0);
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    const int t = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const bool vec_ok = (n % 8) == 0;
    int ti = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++ti) {
      const int db = ti & 1;
      if (t == 0) sh.epi_ok[db] = mbar_wait(&sh.dfull[db], (ti >> 1) & 1, abortp) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!sh.epi_ok[db]) break;
      tc_fence_after();
      const int mt = tile % tiles_m, nt = tile / tiles_m;
      const int row = mt * kBM + t;
      uint16_t* yrow = y + static_cast<int64_t>(row) * n;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r0[16], r1[16];
        const uint32_t taddr = tmem + lane_base + db * kBN + 32 * c;
        tmem_ld16(taddr, r0);
        tmem_ld16(taddr + 16, r1);
        tmem_wait_ld();
        if (row < m) {
          const int col0 = nt * kBN + 32 * c;
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            pk[j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
            pk[8 + j] = pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
          }
          if (vec_ok && col0 + 32 <= n) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          } else {
            for (int j = 0; j < 32; ++j)
              if (col0 + j < n) yrow[col0 + j] = static_cast<uint16_t>((pk[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.dempty[db]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t gemm_smem_bytes() { return static_cast<size_t>(kStages) * kStageBytes + 1024; }

cudaError_t launch_gemm_bf16(const void* tm_x, const void* tm_w, uint16_t* y, int32_t m, int32_t n, int32_t k,
                             int grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = gemm_smem_bytes();
  const cudaError_t e = once_per_device(attr_done, [&] {
    return cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
  });
  if (e != cudaSuccess) return e;
  gemm_bf16_kernel<<<grid, kThreads, smem, st>>>(*static_cast<const CUtensorMap*>(tm_x),
                                                 *static_cast<const CUtensorMap*>(tm_w), y, m, n, k);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace tq4
