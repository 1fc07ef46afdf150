// TQ4_1S streaming kernels for sm_100a: quantize, dequantize, activation
// rotation, and the MoE routing and combine steps.
//
// Format and arithmetic follow the Nemotron-TheHobbit-30B-A3B model card,
// section "What Config-I means" (per-32-block RHT rotation, 16-level
// Lloyd-Max codes, two half-block scales).  The weight kernels give one
// thread one 32-element block, its 32-point butterfly in registers (stage h
// pairs elements j and j+h); the activation kernel spreads a slice over a
// warp and runs the same butterfly through lane shuffles.
#include "tq4_internal.h"

namespace tq4 {

__device__ int g_status = 0;

// r = fp32(1/sqrt(32))
__device__ __forceinline__ float rsqrt32() { return __uint_as_float(0x3E3504F3u); }

// fp32 -> fp16 bits, round to nearest even, saturating at 65504, NaN -> 0x7E00.
__device__ __forceinline__ uint16_t f16_sat_bits(float x) {
  if (x != x) return 0x7E00u;
  const float ax = fabsf(x);
  if (ax >= 65520.0f) return (x < 0.0f) ? 0xFBFFu : 0x7BFFu;
  return __half_as_ushort(__float2half_rn(x));
}

// ------------------------------------------------------------------ quantize
template <typename T>
__device__ __forceinline__ float load_w(const T* p);
template <>
__device__ __forceinline__ float load_w<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_w<uint16_t>(const uint16_t* p) { return bf16_bits_to_f32(__ldg(p)); }

// One thread per 32-element block: the whole butterfly runs in registers in
// the fixed order (stage h pairs elements j and j+h for j with bit h clear),
// so the result is bit-identical to the warp-shuffle form and to the oracle.
__device__ __forceinline__ void fwht32_regs(float (&a)[32]) {
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

template <typename T>
__device__ __forceinline__ void load_block(const T* p, float (&w)[32]);
template <>
__device__ __forceinline__ void load_block<float>(const float* p, float (&w)[32]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = __ldg(q + i);
    w[4 * i] = f.x;
    w[4 * i + 1] = f.y;
    w[4 * i + 2] = f.z;
    w[4 * i + 3] = f.w;
  }
}
template <>
__device__ __forceinline__ void load_block<uint16_t>(const uint16_t* p, float (&w)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(q + i);
    const uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[8 * i + 2 * j] = __uint_as_float(v[j] << 16);
      w[8 * i + 2 * j + 1] = __uint_as_float(v[j] & 0xFFFF0000u);
    }
  }
}

// Quantize: one thread per 32-block (sign flip, butterfly, x r, per-half RMS
// by the pairwise tree, fp16 scale, nearest level by the thresholds, nibble
// packing).  Consecutive threads take consecutive blocks of a row.
template <typename T>
__global__ void __launch_bounds__(256) quantize_kernel(const T* __restrict__ W, uint8_t* __restrict__ codes,
                                                       uint16_t* __restrict__ scales, int64_t rows, int64_t k,
                                                       uint32_t mask, CodebookF32 cb) {
  __shared__ float s_t[16];
  if (threadIdx.x < 16) s_t[threadIdx.x] = cb.thresholds[threadIdx.x];
  __syncthreads();
  const int64_t kb_per_row = k / 32;
  const int64_t nblocks = rows * kb_per_row;
  const float r = rsqrt32();
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = b / kb_per_row, kb = b - row * kb_per_row;
    float a[32];
    load_block<T>(W + row * k + kb * 32, a);
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      finite = finite && isfinite(a[i]);
      if ((mask >> i) & 1u) a[i] = -a[i];
    }
    if (!finite) raise_status(TQ_DEV_NONFINITE);
    fwht32_regs(a);
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] = __fmul_rn(a[i], r);
    uint32_t words[4] = {0u, 0u, 0u, 0u};
    uint32_t dpair = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) p[i] = __fmul_rn(a[16 * h + i], a[16 * h + i]);
#pragma unroll
      for (int st = 8; st >= 1; st >>= 1)
#pragma unroll
        for (int i = 0; i < st; ++i) p[i] = __fadd_rn(p[i], p[i + st]);
      const float rms = __fsqrt_rn(__fmul_rn(p[0], 0.0625f));
      const uint16_t dbits = f16_sat_bits(rms);
      dpair |= static_cast<uint32_t>(dbits) << (16 * h);
      const float d = __half2float(__ushort_as_half(dbits));
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        uint32_t code;
        if (d == 0.0f) {
          code = 7u;
        } else {
          const float u = __fdiv_rn(a[16 * h + i], d);
          // number of thresholds strictly below u (binary search, sorted t)
          code = (u > s_t[7]) ? 8u : 0u;
          code += (u > s_t[code + 3]) ? 4u : 0u;
          code += (u > s_t[code + 1]) ? 2u : 0u;
          code += (u > s_t[code]) ? 1u : 0u;
        }
        const int e = 16 * h + i;   // element index; nibble e of the 16-byte block
        words[e >> 3] |= code << (4 * (e & 7));
      }
    }
    *reinterpret_cast<uint4*>(codes + row * (k / 2) + kb * 16) = make_uint4(words[0], words[1], words[2], words[3]);
    *reinterpret_cast<uint32_t*>(scales + row * (k / 16) + kb * 2) = dpair;
  }
}

// ------------------------------------------------------------------ dequantize
// W_hat = diag(s) * r * H * (c[code] * d), fp32 or bf16 output; one thread per
// 32-block, butterfly in registers.
template <typename TO>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                         const uint16_t* __restrict__ scales, TO* __restrict__ out,
                                                         int64_t rows, int64_t k, uint32_t mask, CodebookF32 cb) {
  __shared__ float s_c[16];
  if (threadIdx.x < 16) s_c[threadIdx.x] = cb.levels[threadIdx.x];
  __syncthreads();
  const int64_t kb_per_row = k / 32;
  const int64_t nblocks = rows * kb_per_row;
  const float r = rsqrt32();
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = b / kb_per_row, kb = b - row * kb_per_row;
    const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes + row * (k / 2) + kb * 16));
    const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(scales + row * (k / 16) + kb * 2));
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    const float d0 = __half2float(__ushort_as_half(static_cast<uint16_t>(sw & 0xFFFFu)));
    const float d1 = __half2float(__ushort_as_half(static_cast<uint16_t>(sw >> 16)));
    float a[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const uint32_t code = (words[e >> 3] >> (4 * (e & 7))) & 0xFu;
      a[e] = __fmul_rn(s_c[code], e < 16 ? d0 : d1);
    }
    fwht32_regs(a);
    TO* o = out + row * k + kb * 32;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float x = __fmul_rn(a[e], r);
      a[e] = ((mask >> e) & 1u) ? -x : x;
    }
    if constexpr (sizeof(TO) == 4) {
      float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
      for (int i = 0; i < 8; ++i) o4[i] = make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
    } else {
      uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o4[i] = make_uint4(pack_bf16x2(a[8 * i], a[8 * i + 1]), pack_bf16x2(a[8 * i + 2], a[8 * i + 3]),
                           pack_bf16x2(a[8 * i + 4], a[8 * i + 5]), pack_bf16x2(a[8 * i + 6], a[8 * i + 7]));
    }
  }
}

// ------------------------------------------------------------------ activations
// The activation side of route B: x' = r H diag(s) x per 32-slice of each row
// (rotating x by the weight's RHT instead of inverse-rotating the weight;
// equivalent because R is orthogonal).  Each row is scaled by 2^-e, where e
// puts the largest value x' can take, sqrt(32) * max|x| (each x'_i is r times
// a signed sum of 32 entries), in [2^13, 2^14): the row then uses the full
// fp16 precision and cannot overflow; the result is rounded to fp16, and
// row_scale[row] = 2^e (exact) undoes the scaling in the GEMM epilogue.
//
// One CTA of four warps per row; lane i of a warp holds element i of a
// slice, and the 32-point butterfly runs across the warp through shfl_xor
// (stage h exchanges lanes i and i^h: the lane with bit h clear keeps
// a + partner, the other partner - a), the same order as the one-thread form.
// First pass: the row maximum; second pass (L1 hits): rotate, scale, round.
// The CTA is small (128 threads, at most 48 registers each, no shared
// arrays) so that it fits on an SM beside a running stream-K CTA.
constexpr int kRotThreads = 128;

__device__ __forceinline__ float warp_fwht32(float a, int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const float p = __shfl_xor_sync(0xFFFFFFFFu, a, h);
    a = (lane & h) ? __fsub_rn(p, a) : __fadd_rn(a, p);
  }
  return a;
}

__global__ void __launch_bounds__(kRotThreads, 10)
    rotate_scaled_kernel(const uint16_t* __restrict__ x, int64_t k, const int32_t* __restrict__ gather,
                         int32_t topk, const int32_t* __restrict__ rows_valid_dev, int64_t rows_valid_host,
                         uint16_t* __restrict__ xr_out, float* __restrict__ row_scale, uint32_t mask) {
  __shared__ float s_max[kRotThreads / 32];
  // x, the gather list and the valid count may be the previous kernel's
  // output.  Dependents may start once every CTA is past this wait: nothing
  // before this kernel is still running then, and the stream-K kernel that
  // follows reads only the weight before its own wait.
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int64_t row = blockIdx.x;
  const int64_t rows_valid = rows_valid_dev ? static_cast<int64_t>(*rows_valid_dev) : rows_valid_host;
  if (row >= rows_valid) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kRotThreads / 32;
  const int64_t src = gather ? static_cast<int64_t>(__ldcg(gather + row) / topk) : row;
  const uint16_t* xr = x + src * k + lane;
  const int64_t nsl = k / 32;
  float mx = 0.0f;
  {
    // 16 loads in flight per lane: a 4096-wide row is one round trip
    int64_t sl = warp;
    for (; sl + 15 * kWarps < nsl; sl += 16 * kWarps) {
      uint16_t v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = __ldg(xr + (sl + u * kWarps) * 32);
#pragma unroll
      for (int u = 0; u < 16; ++u) mx = fmaxf(mx, fabsf(bf16_bits_to_f32(v[u])));
    }
    for (; sl < nsl; sl += kWarps) mx = fmaxf(mx, fabsf(bf16_bits_to_f32(__ldg(xr + sl * 32))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (lane == 0) s_max[warp] = mx;
  __syncthreads();
  mx = s_max[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, s_max[w]);
  int e = 0;
  if (mx > 0.0f && isfinite(mx)) {
    int ex;
    frexpf(__fmul_rn(mx, 5.65685415f), &ex);   // the bound lies in [2^(ex-1), 2^ex)
    e = ex - 14;
    e = e < -100 ? -100 : (e > 100 ? 100 : e);
  }
  if (threadIdx.x == 0) row_scale[row] = ldexpf(1.0f, e);
  const float rd = __fmul_rn(rsqrt32(), ldexpf(1.0f, -e));   // exact: r times a power of two
  const bool neg = (mask >> lane) & 1u;
  uint16_t* oh = xr_out + row * k + lane;
  auto emit = [&](int64_t sl, uint16_t raw) {
    const float xv = bf16_bits_to_f32(raw);
    const float v = __fmul_rn(warp_fwht32(neg ? -xv : xv, lane), rd);
    oh[sl * 32] = __half_as_ushort(__float2half_rn(v));
  };
  int64_t sl = warp;
  for (; sl + 3 * kWarps < nsl; sl += 4 * kWarps) {
    uint16_t v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(xr + (sl + u * kWarps) * 32);
#pragma unroll
    for (int u = 0; u < 4; ++u) emit(sl + u * kWarps, v[u]);
  }
  for (; sl < nsl; sl += kWarps) emit(sl, __ldg(xr + sl * 32));
}

// ------------------------------------------------------------------ MoE routing
// One CTA: per-expert counts, exclusive prefix (offsets), and a stable
// bucketing of flat slot indices p = t*topk + j by expert.  Stability comes
// from assigning positions in p order: each thread handles a contiguous run
// of p, and runs are ranked by a second pass over the per-thread counts.
// Also writes (when the pointers are non-null) the segment list used by the
// grouped stream-K launches -- chunks of at most `chunk` consecutive rows of
// one expert -- and the segment and valid-pair counts.
__global__ void __launch_bounds__(1024) moe_route_kernel(const int32_t* __restrict__ ids, int64_t npairs,
                                                         int32_t num_experts, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ pairs, int4* __restrict__ segs,
                                                         int32_t* __restrict__ nseg_out, int32_t chunk,
                                                         int32_t* __restrict__ npairs_valid) {
  extern __shared__ int32_t sh[];
  int32_t* cnt = sh;                       // [num_experts]
  int32_t* base = sh + num_experts;        // [num_experts]
  __shared__ int32_t s_bad;
  const int tid = threadIdx.x;
  for (int e = tid; e < num_experts; e += blockDim.x) cnt[e] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int64_t p = tid; p < npairs; p += blockDim.x) {
    const int e = ids[p];
    if (e >= 0 && e < num_experts) atomicAdd(&cnt[e], 1);
    else atomicAdd(&s_bad, 1);
  }
  __syncthreads();
  // Exclusive scans over experts of (count, segment count), one expert per
  // thread per pass of the block, carried across passes.
  __shared__ int32_t s_wsum[2][32];
  __shared__ int32_t s_carry[2];
  if (tid == 0) {
    s_carry[0] = 0;
    s_carry[1] = 0;
  }
  __syncthreads();
  const int lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  for (int e0 = 0; e0 < num_experts; e0 += blockDim.x) {
    const int e = e0 + tid;
    const int32_t c = (e < num_experts) ? cnt[e] : 0;
    const int32_t ns = (c + chunk - 1) / chunk;
    int32_t ic = c, is = ns;   // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t yc = __shfl_up_sync(0xFFFFFFFFu, ic, o), ys = __shfl_up_sync(0xFFFFFFFFu, is, o);
      if (lane >= o) {
        ic += yc;
        is += ys;
      }
    }
    if (lane == 31) {
      s_wsum[0][wid] = ic;
      s_wsum[1][wid] = is;
    }
    __syncthreads();
    int32_t pc = s_carry[0], ps = s_carry[1];
    for (int w = 0; w < wid; ++w) {
      pc += s_wsum[0][w];
      ps += s_wsum[1][w];
    }
    const int32_t off = pc + ic - c, soff = ps + is - ns;
    if (e < num_experts) {
      offsets[e] = off;
      base[e] = off;
      if (segs)
        for (int32_t k = 0; k < ns; ++k) segs[soff + k] = make_int4(e, off + k * chunk, min(chunk, c - k * chunk), 0);
    }
    __syncthreads();
    if (tid == blockDim.x - 1) {
      s_carry[0] = pc + ic;
      s_carry[1] = ps + is;
    }
    __syncthreads();
    (void)nw;
  }
  if (tid == 0) {
    offsets[num_experts] = s_carry[0];
    if (npairs_valid) *npairs_valid = s_carry[0];
    if (nseg_out) *nseg_out = s_carry[1];
    if (s_bad) raise_status(TQ_DEV_BAD_ROUTING);
  }
  __syncthreads();
  // Stable scatter by warp 0, 32 slots at a time in p order: lanes holding
  // the same expert take consecutive positions in lane order.
  if (tid < 32) {
    const unsigned lt_mask = (1u << tid) - 1u;
    for (int64_t p0 = 0; p0 < npairs; p0 += 32) {
      const int64_t p = p0 + tid;
      const int e = (p < npairs) ? ids[p] : -1;
      const bool ok = e >= 0 && e < num_experts;
      const int key = ok ? e : -1 - tid;   // invalid slots group with nobody
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
      const int rank = __popc(peers & lt_mask);
      if (ok) pairs[base[e] + rank] = static_cast<int32_t>(p);
      __syncwarp();
      if (ok && rank == 0) base[e] += __popc(peers);
      __syncwarp();
    }
  }
}

// y[t][n] = bf16( sum_j zw[t*topk + j][n] ) over slots with a valid expert id.
__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ zw, const int32_t* __restrict__ ids,
                                                          int64_t m, int32_t topk, int64_t h, int32_t num_experts,
                                                          uint16_t* __restrict__ y) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= m * h) return;
  const int64_t t = i / h, n = i - t * h;
  float s = 0.0f;
  for (int j = 0; j < topk; ++j) {
    const int64_t p = t * topk + j;
    const int e = ids[p];
    if (e >= 0 && e < num_experts) s = __fadd_rn(s, zw[p * h + n]);
  }
  y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
}

// ------------------------------------------------------------------ launchers
static int grid_threads(int64_t threads_needed, int threads) {
  int64_t blocks = (threads_needed + threads - 1) / threads;
  const int64_t cap = 148LL * (2048 / threads);
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<int>(blocks);
}

cudaError_t launch_quantize(const void* W, int dtype, uint8_t* codes, uint16_t* scales, int64_t rows, int64_t k,
                            uint32_t mask, const CodebookF32& cb, cudaStream_t st) {
  const int g = grid_threads(rows * (k / 32), 256);
  if (dtype == TQ_DTYPE_F32)
    quantize_kernel<float><<<g, 256, 0, st>>>(static_cast<const float*>(W), codes, scales, rows, k, mask, cb);
  else
    quantize_kernel<uint16_t><<<g, 256, 0, st>>>(static_cast<const uint16_t*>(W), codes, scales, rows, k, mask, cb);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_f32(const uint8_t* codes, const uint16_t* scales, float* out, int64_t rows, int64_t k,
                                  uint32_t mask, const CodebookF32& cb, cudaStream_t st) {
  dequantize_kernel<float><<<grid_threads(rows * (k / 32), 256), 256, 0, st>>>(codes, scales, out, rows, k, mask,
                                                                                cb);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_bf16(const uint8_t* codes, const uint16_t* scales, uint16_t* out, int64_t rows,
                                   int64_t k, uint32_t mask, const CodebookF32& cb, cudaStream_t st) {
  dequantize_kernel<uint16_t><<<grid_threads(rows * (k / 32), 256), 256, 0, st>>>(codes, scales, out, rows, k,
                                                                                   mask, cb);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_rotate_scaled(const uint16_t* x, int64_t k, const int32_t* gather, int32_t topk,
                                 const int32_t* rows_valid_dev, int64_t rows_valid_host, int64_t rows_alloc,
                                 uint16_t* xr, float* row_scale, uint32_t mask, cudaStream_t st) {
  if (rows_alloc <= 0) return cudaSuccess;
  static bool attr_set = false;
  if (!attr_set) {
    // the stream-K kernel runs with the largest shared-memory carveout; an SM
    // hosts CTAs of two kernels at once only if their carveouts agree
    const cudaError_t e =
        cudaFuncSetAttribute(rotate_scaled_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows_alloc));
  cfg.blockDim = dim3(kRotThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, rotate_scaled_kernel, x, k, gather, topk, rows_valid_dev,
                                           rows_valid_host, xr, row_scale, mask);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_moe_route(const int32_t* ids, int64_t npairs, int32_t num_experts, int32_t* offsets,
                             int32_t* pairs, int4* segs, int32_t* nseg, int32_t chunk, int32_t* npairs_valid,
                             cudaStream_t st) {
  const size_t sh = sizeof(int32_t) * 2 * static_cast<size_t>(num_experts);
  moe_route_kernel<<<1, 1024, sh, st>>>(ids, npairs, num_experts, offsets, pairs, segs, nseg, chunk, npairs_valid);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_moe_combine(const float* zw, const int32_t* ids, int64_t m, int32_t topk, int64_t h,
                               int32_t num_experts, uint16_t* y, cudaStream_t st) {
  const int64_t n = m * h;
  const int g = static_cast<int>((n + 255) / 256);
  moe_combine_kernel<<<g, 256, 0, st>>>(zw, ids, m, topk, h, num_experts, y);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace tq4
