// TQ4_1S streaming kernels for sm_100a: quantize, dequantize, activation
// rotation, and the MoE routing and combine steps.
//
// Format and arithmetic follow the Nemotron-TheHobbit-30B-A3B model card,
// section "What Config-I means" (per-32-block RHT rotation, 16-level
// Lloyd-Max codes, two half-block scales).  The weight kernels give one
// thread one 32-element block, its 32-point butterfly in registers (stage h
// pairs elements j and j+h); the activation kernel spreads a slice over a
// warp and runs the same butterfly through lane shuffles.
#include <climits>

#include <cuda_fp8.h>

#include "tq4_internal.h"

namespace tq4 {

__device__ int g_status = 0;
__device__ unsigned long long g_wait_ns = TQ_WAIT_NS_DEFAULT;

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

// Thresholds of the quantizer in shared memory: t[0..14] (sorted, t[15]
// unused), and a bucket table over |u| for a symmetric codebook
// (t[14 - k] == -t[k], so t[7] == 0), whose positive thresholds are
// p[j] = t[8 + j], j < 7.  Bucket i >= 1 holds the floats whose bits >> 19
// (exponent and top 4 mantissa bits) equal kQBucket0 + i - 1, i.e.
// [2^-5, 2^3) in 128 buckets; bucket 0 is below 2^-5, the last one 2^3 and
// above.  Entry i: x = the bits of the p[j] inside the bucket (those of
// +inf if none), y = the number of p[j] below the bucket.  Non-negative
// floats order as their bits, so |u| > p[j] is bits(|u|) > x and
// |u| >= p[j] is bits(|u|) + 1 > x.  fast: the codebook is symmetric and no
// bucket holds two thresholds (else the full search runs).
constexpr int kQBucket0 = 122 << 4;   // bits of 2^-5, >> 19
constexpr int kQBuckets = 130;
struct QuantThresholds {
  float t[16];
  uint2 bucket[kQBuckets];
  int fast;
};

// Quantize one 32-element block held in registers (sign flip, butterfly, x r,
// per-half RMS by the pairwise tree, fp16 scale, nearest level by the
// thresholds, nibble packing) -- the fixed fp32 operation order that the
// packing's bit-exactness rests on.  words = the 16 code bytes, dpair = the
// two fp16 scales (half 0 in the low 16 bits).  Returns false when a half
// block's sum of squares is not finite: an input was Inf or NaN (which makes
// every output of the butterfly non-finite), or a finite input was above
// ~2^63; the caller then checks the inputs themselves.
__device__ __forceinline__ bool quantize_block(float (&a)[32], uint32_t mask, const QuantThresholds& th,
                                               uint32_t (&words)[4], uint32_t& dpair) {
  const float r = rsqrt32();
  bool sums_finite = true;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if ((mask >> i) & 1u) a[i] = -a[i];
  fwht32_regs(a);
#pragma unroll
  for (int i = 0; i < 32; ++i) a[i] = __fmul_rn(a[i], r);
#pragma unroll
  for (int i = 0; i < 4; ++i) words[i] = 0u;
  dpair = 0u;
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
    // u = fl(a / d), correctly rounded, and its code: the number of
    // thresholds strictly below u.
    const bool fin = isfinite(p[0]);
    sums_finite = sums_finite && fin;
    if (fin && d != 0.0f) {
      // With y = RN(1/d) once per half block, q = RN(a y), the exact
      // residual r = a - q d (one fma) and RN(q + r y) give the correctly
      // rounded quotient whenever nothing overflows (Markstein's theorem;
      // checked against the division on every positive fp16 d): a finite sum
      // of squares bounds |a| by 2^63, and |a / d| then stays near 4 or below.
      const float y = __frcp_rn(d);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float q = __fmul_rn(a[16 * h + i], y);
        const float u = __fmaf_rn(__fmaf_rn(-q, d, a[16 * h + i]), y, q);
        uint32_t code;
        if (th.fast) {
          // symmetric thresholds: u > 0 has 8 + #{p[j] < u} below it, u <= 0
          // has #{t[k] < u, k < 7} = #{p[j] > |u|} = 7 - #{p[j] <= |u|}; both
          // counts from |u|'s bucket: the thresholds below it, plus the one
          // inside it if |u| passes it (> for u > 0, >= for u <= 0)
          const bool pos = u > 0.0f;
          const uint32_t ab = __float_as_uint(u) & 0x7FFFFFFFu;
          int q = static_cast<int>(ab >> 19) - (kQBucket0 - 1);
          q = q < 0 ? 0 : (q > kQBuckets - 1 ? kQBuckets - 1 : q);
          const uint2 e = th.bucket[q];
          const uint32_t c = e.y + ((ab + (pos ? 0u : 1u) > e.x) ? 1u : 0u);
          code = pos ? 8u + c : 7u - c;
        } else {
          code = (u > th.t[7]) ? 8u : 0u;
          code += (u > th.t[code + 3]) ? 4u : 0u;
          code += (u > th.t[code + 1]) ? 2u : 0u;
          code += (u > th.t[code]) ? 1u : 0u;
        }
        const int e = 16 * h + i;   // element index; nibble e of the 16-byte block
        words[e >> 3] |= code << (4 * (e & 7));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        uint32_t code = 7u;   // d == 0: the zero level's code
        if (d != 0.0f) {
          const float u = __fdiv_rn(a[16 * h + i], d);
          code = (u > th.t[7]) ? 8u : 0u;
          code += (u > th.t[code + 3]) ? 4u : 0u;
          code += (u > th.t[code + 1]) ? 2u : 0u;
          code += (u > th.t[code]) ? 1u : 0u;
        }
        const int e = 16 * h + i;
        words[e >> 3] |= code << (4 * (e & 7));
      }
    }
  }
  return sums_finite;
}

// The tensors of one quantize launch.  A tensor of B blocks (B = rows * k / 32,
// blocks consecutive in its flat row-major order) owns the warp chunks
// [chunk0, chunk0 + ceil(B / 32)) of the launch; a chunk is 32 consecutive
// blocks.  Passed by value (kernel parameter space).
constexpr int kQuantBatch = 48;
struct QuantTensor {
  const void* W;
  uint8_t* codes;
  uint16_t* scales;
  int64_t nblocks;
  int64_t chunk0;
  uint32_t mask;
};
struct QuantBatch {
  int32_t count;
  int64_t nchunks;
  QuantTensor t[kQuantBatch];
};

// Quantize.  A warp takes 32 consecutive blocks at a time: it reads them
// with coalesced 16-byte loads (lane l, load i: bytes 16 l + 512 i of the
// chunk), writes them to its shared-memory tile, and each lane then quantizes
// one block from the tile in registers and stores its 16 code bytes and two
// scales (coalesced too).  Tile rows are one block each, their 16-byte
// pieces XOR-swizzled so that neither the writes nor the per-lane row reads
// conflict on banks.  The arithmetic per block is long (a correctly rounded
// division per element), so latency is hidden by occupancy: few registers,
// four CTAs per SM.
template <typename T>
__global__ void __launch_bounds__(256, 4) quantize_kernel(const __grid_constant__ QuantBatch qb, CodebookF32 cb) {
  constexpr int kRowBytes = 32 * static_cast<int>(sizeof(T));   // one block: 128 B (fp32) or 64 B (bf16)
  constexpr int kPieces = kRowBytes / 16;                        // 16-byte pieces per block
  constexpr int kLoads = kPieces;                                // 16-byte loads per lane per chunk
  __shared__ QuantThresholds th;
  __shared__ __align__(16) uint8_t tile[8][32 * kRowBytes];
  if (threadIdx.x < 16) th.t[threadIdx.x] = cb.thresholds[threadIdx.x];
  auto bucket_of = [](float x) {   // x >= 0
    const int q = static_cast<int>(__float_as_uint(x) >> 19) - (kQBucket0 - 1);
    return q < 0 ? 0 : (q > kQBuckets - 1 ? kQBuckets - 1 : q);
  };
  for (int i = threadIdx.x; i < kQBuckets; i += blockDim.x) {
    const float lo = i == 0 ? 0.0f : __uint_as_float(static_cast<uint32_t>(kQBucket0 + i - 1) << 19);
    const float hi = i == kQBuckets - 1 ? INFINITY : __uint_as_float(static_cast<uint32_t>(kQBucket0 + i) << 19);
    uint32_t below = 0u, inside = 0x7F800000u;   // (+inf)
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      const float pj = cb.thresholds[8 + j];
      if (pj < lo) {
        ++below;
      } else if (pj < hi) {
        inside = __float_as_uint(pj);
      }
    }
    th.bucket[i] = make_uint2(inside, below);
  }
  if (threadIdx.x == 0) {
    // symmetric, positive, and no two (sorted) thresholds in one bucket
    bool fast = cb.thresholds[7] == 0.0f;
#pragma unroll
    for (int k = 0; k < 7; ++k) fast = fast && cb.thresholds[14 - k] == -cb.thresholds[k] && cb.thresholds[8 + k] > 0.0f;
#pragma unroll
    for (int j = 0; j + 1 < 7; ++j) fast = fast && bucket_of(cb.thresholds[8 + j]) != bucket_of(cb.thresholds[9 + j]);
    th.fast = fast ? 1 : 0;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* my = tile[warp];
  // swizzled byte offset of piece c of block (row) b
  auto tpos = [](int b, int c) {
    const int sw = (kPieces == 8) ? (b & 7) : ((b >> 1) & 3);
    return b * kRowBytes + 16 * (c ^ sw);
  };
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  int tix = 0;   // tensor of the current chunk (chunks are visited in increasing order)
  for (int64_t ch = static_cast<int64_t>(blockIdx.x) * 8 + warp; ch < qb.nchunks; ch += nwarps) {
    while (tix + 1 < qb.count && ch >= qb.t[tix + 1].chunk0) ++tix;
    const QuantTensor& q = qb.t[tix];
    const int64_t b0 = (ch - q.chunk0) * 32;
    {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(q.W) + b0 * 32);
      uint4 buf[kLoads];
#pragma unroll
      for (int i = 0; i < kLoads; ++i) {
        const int piece = lane + 32 * i;   // 16-byte piece of the chunk
        buf[i] = (b0 + piece / kPieces < q.nblocks) ? __ldg(src + piece) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < kLoads; ++i) {
        const int piece = lane + 32 * i;
        *reinterpret_cast<uint4*>(my + tpos(piece / kPieces, piece % kPieces)) = buf[i];
      }
    }
    __syncwarp();
    float a[32];
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int c = 0; c < kPieces; ++c) {
        const float4 f = *reinterpret_cast<const float4*>(my + tpos(lane, c));
        a[4 * c] = f.x;
        a[4 * c + 1] = f.y;
        a[4 * c + 2] = f.z;
        a[4 * c + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < kPieces; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(my + tpos(lane, c));
        const uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a[8 * c + 2 * j] = __uint_as_float(v[j] << 16);
          a[8 * c + 2 * j + 1] = __uint_as_float(v[j] & 0xFFFF0000u);
        }
      }
    }
    __syncwarp();   // the tile is rewritten with the next chunk after this
    const int64_t b = b0 + lane;
    if (b < q.nblocks) {
      uint32_t words[4], dpair;
      if (!quantize_block(a, q.mask, th, words, dpair)) {
        // a sum of squares was not finite: flag an input that is Inf or NaN
        bool finite = true;
#pragma unroll
        for (int c = 0; c < kPieces; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(my + tpos(lane, c));
          const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if constexpr (sizeof(T) == 4) {
              finite = finite && isfinite(__uint_as_float(v[j]));
            } else {
              finite = finite && isfinite(__uint_as_float(v[j] << 16)) && isfinite(__uint_as_float(v[j] & 0xFFFF0000u));
            }
          }
        }
        if (!finite) raise_status(TQ_DEV_NONFINITE);
      }
      *reinterpret_cast<uint4*>(q.codes + b * 16) = make_uint4(words[0], words[1], words[2], words[3]);
      *reinterpret_cast<uint32_t*>(q.scales + b * 2) = dpair;
    }
    __syncwarp();   // every lane is done with the tile (the check above reads it)
  }
}

// ------------------------------------------------------------------ dequantize
// W_hat of one 32-block in fp32: levels c[code] * d, the butterfly, x r, the
// signs -- one rounding per operation in this fixed order.
__device__ __forceinline__ void dequant_block_f32(const uint4 cw, uint32_t sw, uint32_t mask, const float* s_c,
                                                  float (&a)[32]) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
  const float d0 = __half2float(__ushort_as_half(static_cast<uint16_t>(sw & 0xFFFFu)));
  const float d1 = __half2float(__ushort_as_half(static_cast<uint16_t>(sw >> 16)));
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const uint32_t code = (words[e >> 3] >> (4 * (e & 7))) & 0xFu;
    a[e] = __fmul_rn(s_c[code], e < 16 ? d0 : d1);
  }
  fwht32_regs(a);
  const float r = rsqrt32();
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float x = __fmul_rn(a[e], r);
    a[e] = ((mask >> e) & 1u) ? -x : x;
  }
}

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
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = b / kb_per_row, kb = b - row * kb_per_row;
    const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes + row * (k / 2) + kb * 16));
    const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(scales + row * (k / 16) + kb * 2));
    float a[32];
    dequant_block_f32(cw, sw, mask, s_c, a);
    TO* o = out + row * k + kb * 32;
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

// ------------------------------------------------------------------ fp8 cache
// TQ4_1S -> the fp8-resident cache of the model card's "Help wanted" (dequantize
// once, keep the weight resident in fp8): per row n, s_n = fp32(amax_n / 448)
// over the row's W_hat, codes = E4M3(fp32(W_hat / s_n)) rounded to nearest
// even and saturating; a zero row gets s_n = 0 and zero codes.  One CTA per
// row: a first pass takes the row maximum, a second dequantizes again and
// converts (W_hat is not kept).
__global__ void __launch_bounds__(256) to_fp8_kernel(const uint8_t* __restrict__ codes,
                                                     const uint16_t* __restrict__ scales, uint8_t* __restrict__ q,
                                                     float* __restrict__ wscale, int64_t rows, int64_t k,
                                                     uint32_t mask, CodebookF32 cb) {
  __shared__ float s_c[16];
  __shared__ float s_max[8];
  if (threadIdx.x < 16) s_c[threadIdx.x] = cb.levels[threadIdx.x];
  __syncthreads();
  const int64_t nkb = k / 32;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint8_t* cr = codes + row * (k / 2);
    const uint16_t* sr = scales + row * (k / 16);
    float mx = 0.0f;
    for (int64_t kb = threadIdx.x; kb < nkb; kb += blockDim.x) {
      float a[32];
      dequant_block_f32(__ldg(reinterpret_cast<const uint4*>(cr + kb * 16)),
                        __ldg(reinterpret_cast<const uint32_t*>(sr + kb * 2)), mask, s_c, a);
#pragma unroll
      for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(a[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = s_max[0];
    for (int w = 1; w < 8; ++w) mx = fmaxf(mx, s_max[w]);
    __syncthreads();   // s_max is rewritten for the next row
    const float sc = __fdiv_rn(mx, 448.0f);
    if (threadIdx.x == 0) wscale[row] = sc;
    for (int64_t kb = threadIdx.x; kb < nkb; kb += blockDim.x) {
      float a[32];
      dequant_block_f32(__ldg(reinterpret_cast<const uint4*>(cr + kb * 16)),
                        __ldg(reinterpret_cast<const uint32_t*>(sr + kb * 2)), mask, s_c, a);
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t word = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float v = (sc == 0.0f) ? 0.0f : __fdiv_rn(a[4 * i + j], sc);
          const uint32_t b = static_cast<uint32_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
          word |= b << (8 * j);
        }
        w[i] = word;
      }
      uint4* dst = reinterpret_cast<uint4*>(q + row * k + kb * 32);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

// fp8 cache -> bf16 weight: out[n][k] = bf16(s_n * e4m3(q[n][k])) (the large-m
// path of the fp8 linear); a thread converts 16 codes.
__global__ void __launch_bounds__(256) fp8_to_bf16_kernel(const uint8_t* __restrict__ q,
                                                          const float* __restrict__ wscale,
                                                          uint16_t* __restrict__ out, int64_t rows, int64_t k) {
  const int64_t per_row = k / 16, total = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / per_row, c = i - row * per_row;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + row * k + c * 16));
    const float sc = __ldg(wscale + row);
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(vw[j] >> (16 * h)),
                                                          __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        o[2 * j + h] = pack_bf16x2(__fmul_rn(f.x, sc), __fmul_rn(f.y, sc));
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + row * k + c * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ------------------------------------------------------------------ affine format
// MLX-style affine group quantization (the MLX port's README, "Quantization
// (6-bit, scheme mixed_v1)"; 4/6/8-bit family): groups of 64 weights of a
// row, scale = (max - min) / (2^b - 1) and bias = min in fp32, stored as bf16;
// q = clamp(rint(fp32(fp32(w - bias) / scale)), 0, 2^b - 1) against the stored
// values (zero scale: q = 0); codes as one little-endian bit stream per row.
// One thread per group; a group's codes are 8 b bytes, byte-aligned.
constexpr int kAffGroup = 64;

__global__ void __launch_bounds__(256) affine_quantize_kernel(const float* __restrict__ W, uint8_t* __restrict__ codes,
                                                              uint16_t* __restrict__ scales,
                                                              uint16_t* __restrict__ biases, int64_t groups,
                                                              int bits) {
  const float qmax = static_cast<float>((1 << bits) - 1);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4* w4 = reinterpret_cast<const float4*>(W + g * kAffGroup);
    float lo = INFINITY, hi = -INFINITY;
    for (int i = 0; i < kAffGroup / 4; ++i) {
      const float4 f = __ldg(w4 + i);
      lo = fminf(fminf(lo, f.x), fminf(f.y, fminf(f.z, f.w)));
      hi = fmaxf(fmaxf(hi, f.x), fmaxf(f.y, fmaxf(f.z, f.w)));
    }
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
    const __nv_bfloat16 bb = __float2bfloat16_rn(lo);
    scales[g] = __bfloat16_as_ushort(sb);
    biases[g] = __bfloat16_as_ushort(bb);
    const float sc = __bfloat162float(sb), bi = __bfloat162float(bb);
    // pack into 32-bit words through a 64-bit accumulator
    uint32_t* out = reinterpret_cast<uint32_t*>(codes + g * (8 * bits));
    unsigned long long accb = 0ull;
    int nacc = 0, nw = 0;
    for (int i = 0; i < kAffGroup / 4; ++i) {
      const float4 f = __ldg(w4 + i);
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float q = 0.0f;
        if (sc != 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(fv[j], bi), sc)), 0.0f), qmax);
        accb |= static_cast<unsigned long long>(static_cast<uint32_t>(q)) << nacc;
        nacc += bits;
        if (nacc >= 32) {
          out[nw++] = static_cast<uint32_t>(accb);
          accb >>= 32;
          nacc -= 32;
        }
      }
    }
  }
}

template <typename TO>
__global__ void __launch_bounds__(256) affine_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                                const uint16_t* __restrict__ scales,
                                                                const uint16_t* __restrict__ biases,
                                                                TO* __restrict__ out, int64_t groups, int bits) {
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t* in = reinterpret_cast<const uint32_t*>(codes + g * (8 * bits));
    const float sc = bf16_bits_to_f32(__ldg(scales + g)), bi = bf16_bits_to_f32(__ldg(biases + g));
    TO* o = out + g * kAffGroup;
    unsigned long long accb = 0ull;
    int nacc = 0, nr = 0;
    for (int i = 0; i < kAffGroup; ++i) {
      if (nacc < bits) {
        accb |= static_cast<unsigned long long>(__ldg(in + nr++)) << nacc;
        nacc += 32;
      }
      const uint32_t q = static_cast<uint32_t>(accb) & mask;
      accb >>= bits;
      nacc -= bits;
      const float v = __fadd_rn(__fmul_rn(sc, static_cast<float>(q)), bi);
      if constexpr (sizeof(TO) == 4) o[i] = v;
      else o[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
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
//
// The router (model card, "The model underneath": 6 of 128 experts per token;
// "Performance": no host syncs in the MoE) runs first when logits are given:
// softmax over all experts, the topk largest taken (equal logits: lower id
// first), their probabilities renormalised.  One warp per token; lane l holds
// the logits of experts l, l + 32, ...; each round the lanes propose their
// best untaken expert and a shuffle reduction picks the warp's (largest
// logit, then lowest id).  The selected j-th logit stays with lane j; the
// weights are exp(z_j - z_max) / sum over the selected, in fp64 (the full
// softmax's denominator cancels).  A NaN logit is never chosen and sets
// TQ_DEV_NONFINITE.
__device__ void router_rows(const float* __restrict__ z, int64_t m, int32_t num_experts, int32_t topk,
                            int32_t* __restrict__ ids, float* __restrict__ w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int per_lane = (num_experts + 31) / 32;   // <= 32 (num_experts <= 1024)
  for (int64_t t = warp; t < m; t += nwarps) {
    const float* zt = z + t * num_experts;
    uint32_t taken = 0u;   // bit i: expert lane + 32 i already chosen
    bool nan_seen = false;
    float myz = 0.0f;
    int mye = 0;
    for (int j = 0; j < topk; ++j) {
      float bz = -INFINITY;
      int be = INT_MAX;
      for (int i = 0; i < per_lane; ++i) {
        const int e = i * 32 + lane;
        if (e >= num_experts || ((taken >> i) & 1u)) continue;
        const float v = __ldg(zt + e);
        if (v != v) {
          nan_seen = true;
          continue;
        }
        if (v > bz || (v == bz && e < be)) {
          bz = v;
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oz = __shfl_xor_sync(0xFFFFFFFFu, bz, o);
        const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
        if (oz > bz || (oz == bz && oe < be)) {
          bz = oz;
          be = oe;
        }
      }
      if (be != INT_MAX && (be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == j) {
        myz = bz;
        mye = be;
      }
    }
    if (__any_sync(0xFFFFFFFFu, nan_seen) && lane == 0) raise_status(TQ_DEV_NONFINITE);
    const float zmax = __shfl_sync(0xFFFFFFFFu, myz, 0);
    const double ex = (lane < topk && mye != INT_MAX) ? exp(static_cast<double>(myz) - static_cast<double>(zmax)) : 0.0;
    double sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane < topk) {
      ids[t * topk + lane] = (mye == INT_MAX) ? -1 : mye;
      w[t * topk + lane] = static_cast<float>(ex / sum);
    }
  }
}

__global__ void __launch_bounds__(1024) moe_route_kernel(const int32_t* __restrict__ ids_in, int64_t npairs,
                                                         int32_t num_experts, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ pairs, int4* __restrict__ segs,
                                                         int32_t* __restrict__ nseg_out, int32_t chunk,
                                                         int32_t* __restrict__ npairs_valid,
                                                         const float* __restrict__ logits, int32_t topk,
                                                         int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
  extern __shared__ int32_t sh[];
  if (logits) {
    router_rows(logits, npairs / topk, num_experts, topk, ids_out, w_out);
    __syncthreads();   // the ids written above are read by the whole block below
  }
  const int32_t* ids = logits ? ids_out : ids_in;
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

cudaError_t launch_affine_quantize(const float* W, uint8_t* codes, uint16_t* scales, uint16_t* biases, int64_t rows,
                                   int64_t k, int bits, cudaStream_t st) {
  const int64_t groups = rows * (k / kAffGroup);
  affine_quantize_kernel<<<grid_threads(groups, 256), 256, 0, st>>>(W, codes, scales, biases, groups, bits);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_affine_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, void* out,
                                     bool bf16_out, int64_t rows, int64_t k, int bits, cudaStream_t st) {
  const int64_t groups = rows * (k / kAffGroup);
  if (bf16_out)
    affine_dequantize_kernel<uint16_t><<<grid_threads(groups, 256), 256, 0, st>>>(
        codes, scales, biases, static_cast<uint16_t*>(out), groups, bits);
  else
    affine_dequantize_kernel<float><<<grid_threads(groups, 256), 256, 0, st>>>(codes, scales, biases,
                                                                               static_cast<float*>(out), groups, bits);
  note_launches(1);
  return cudaGetLastError();
}


cudaError_t launch_quantize_batch(const QuantItem* items, int count, int dtype, const CodebookF32& cb,
                                  cudaStream_t st) {
  for (int i0 = 0; i0 < count; i0 += kQuantBatch) {
    QuantBatch qb{};
    qb.count = count - i0 < kQuantBatch ? count - i0 : kQuantBatch;
    int64_t chunks = 0;
    for (int i = 0; i < qb.count; ++i) {
      const QuantItem& it = items[i0 + i];
      QuantTensor& q = qb.t[i];
      q.W = it.W;
      q.codes = it.codes;
      q.scales = it.scales;
      q.nblocks = it.rows * (it.k / 32);
      q.chunk0 = chunks;
      q.mask = it.mask;
      chunks += (q.nblocks + 31) / 32;
    }
    qb.nchunks = chunks;
    if (chunks == 0) continue;
    int64_t blocks = (chunks + 7) / 8;
    const int64_t cap = 148LL * 4 * 4;
    if (blocks > cap) blocks = cap;
    if (dtype == TQ_DTYPE_F32)
      quantize_kernel<float><<<static_cast<int>(blocks), 256, 0, st>>>(qb, cb);
    else
      quantize_kernel<uint16_t><<<static_cast<int>(blocks), 256, 0, st>>>(qb, cb);
    note_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_quantize(const void* W, int dtype, uint8_t* codes, uint16_t* scales, int64_t rows, int64_t k,
                            uint32_t mask, const CodebookF32& cb, cudaStream_t st) {
  const QuantItem it{W, codes, scales, rows, k, mask};
  return launch_quantize_batch(&it, 1, dtype, cb, st);
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

cudaError_t launch_to_fp8(const uint8_t* codes, const uint16_t* scales, uint8_t* q, float* wscale, int64_t rows,
                          int64_t k, uint32_t mask, const CodebookF32& cb, cudaStream_t st) {
  const int64_t g = rows < 148LL * 8 ? rows : 148LL * 8;
  to_fp8_kernel<<<static_cast<unsigned>(g), 256, 0, st>>>(codes, scales, q, wscale, rows, k, mask, cb);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fp8_to_bf16(const uint8_t* q, const float* wscale, uint16_t* out, int64_t rows, int64_t k,
                               cudaStream_t st) {
  fp8_to_bf16_kernel<<<grid_threads(rows * (k / 16), 256), 256, 0, st>>>(q, wscale, out, rows, k);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_rotate_scaled(const uint16_t* x, int64_t k, const int32_t* gather, int32_t topk,
                                 const int32_t* rows_valid_dev, int64_t rows_valid_host, int64_t rows_alloc,
                                 uint16_t* xr, float* row_scale, uint32_t mask, cudaStream_t st) {
  if (rows_alloc <= 0) return cudaSuccess;
  // the stream-K kernel runs with the largest shared-memory carveout; an SM
  // hosts CTAs of two kernels at once only if their carveouts agree
  static std::atomic<uint64_t> attr_done{0};
  const cudaError_t ea = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(rotate_scaled_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (ea != cudaSuccess) return ea;
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
                             cudaStream_t st, const float* logits, int32_t topk, int32_t* ids_out, float* w_out) {
  const size_t sh = sizeof(int32_t) * 2 * static_cast<size_t>(num_experts);
  moe_route_kernel<<<1, 1024, sh, st>>>(ids, npairs, num_experts, offsets, pairs, segs, nseg, chunk, npairs_valid,
                                        logits, topk, ids_out, w_out);
  note_launches(1);
  return cudaGetLastError();
}

// The router alone (parity hook): one CTA of 32 warps per 32 tokens.
__global__ void __launch_bounds__(1024) router_kernel(const float* __restrict__ logits, int64_t m, int32_t num_experts,
                                                      int32_t topk, int32_t* __restrict__ ids, float* __restrict__ w) {
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t rows = m - t0 < 32 ? m - t0 : 32;
  router_rows(logits + t0 * num_experts, rows, num_experts, topk, ids + t0 * topk, w + t0 * topk);
}

cudaError_t launch_router(const float* logits, int64_t m, int32_t num_experts, int32_t topk, int32_t* ids, float* w,
                          cudaStream_t st) {
  router_kernel<<<static_cast<unsigned>((m + 31) / 32), 1024, 0, st>>>(logits, m, num_experts, topk, ids, w);
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
