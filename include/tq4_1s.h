/*
 * tq4_1s.h -- C ABI of libtq4_1s.so, the B200 (sm_100a) TQ4_1S layer.
 *
 * TQ4_1S ("Config-I") is the weight format of the Nemotron-TheHobbit-30B-A3B
 * model card, section "What Config-I means": each 32-element block of a
 * weight row (along K) is rotated by a randomized Walsh-Hadamard transform,
 * then coded with 4-bit indices into a fixed 16-level Lloyd-Max codebook of
 * N(0,1), with two half-block scales -- about 5 bits per weight.  Section
 * "Running it" swaps quantized Linears for an on-the-fly dequant layer;
 * section "Performance" adds a sync-free MoE and bf16 tensor-core matmuls;
 * section "The model underneath" gives the 128-expert, top-6 MoE.
 *
 * Format (readings of what the card leaves open):
 *   - signs: s_i = -1 where bit i of sign_mask is set, one 32-sign vector per
 *     tensor (per expert stack), sign_mask = low 32 bits of the first
 *     SplitMix64 output for the tensor's seed;
 *   - rotation R = r * H * diag(s), H the natural-order 32-point Sylvester
 *     Hadamard matrix, r = fp32(1/sqrt(32));
 *   - per 16-element half h of a rotated block v: d_h = fp16(rms(v_h))
 *     (round to nearest even, saturating at 65504);
 *     code_i = #{ j : v_i / d_h > t_j } over the 15 fp32 midpoints of the
 *     codebook (all codes 7 when d_h == 0);
 *   - codes plane  uint8 [E][n][k/2]: element 2i of a row in the low nibble
 *     of byte i, 2i+1 in the high nibble;
 *     scales plane uint16 [E][n][k/16]: fp16 bits, scale of half (k/16).
 *   - dequantized weight: W_hat = diag(s) * r * H * (c[code] * d) per block.
 *
 * Conventions for every entry point:
 *   - All pointers named as device pointers must point to device memory of
 *     the current CUDA device; host pointers are noted as such.  The caller
 *     owns every buffer; the library allocates nothing on these paths.
 *   - Calls are asynchronous on the given stream (a cudaStream_t; NULL is
 *     the legacy default stream) and do not synchronize, except
 *     tq4_1s_get_status().
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns its error code and launches nothing.
 *   - Conditions found on the device (a routing id out of range, a bounded
 *     wait that timed out, a non-finite input to quantize) set bits of a
 *     per-device status word, read and cleared by tq4_1s_get_status().
 */
#ifndef TQ4_1S_H_
#define TQ4_1S_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, without requiring the CUDA headers. */
typedef struct CUstream_st* tq4_stream_t;

/* Return codes. */
enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,         /* null pointer, bad size, k % 32 != 0, m < 0, ... */
  TQ_ERR_ALIGNMENT = 2,           /* a device pointer not 16-byte aligned */
  TQ_ERR_UNSUPPORTED_DEVICE = 3,  /* current device is not compute capability 10.0 */
  TQ_ERR_WORKSPACE = 4,           /* workspace null or smaller than the query says */
  TQ_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
  TQ_ERR_TIMEOUT = 6,             /* status: a bounded device wait gave up */
  TQ_ERR_BAD_ROUTING = 7,         /* status: a routing expert id was out of range */
  TQ_ERR_NONFINITE = 8,           /* status: quantize saw a NaN or infinity */
  TQ_ERR_SCRATCH_LIMIT = 9        /* tq4_1s_linear_static: shape beyond its fixed scratch */
};

/* Bits of the device status word (tq4_1s_get_status). */
enum {
  TQ_DEV_TIMEOUT = 1,
  TQ_DEV_BAD_ROUTING = 2,
  TQ_DEV_NONFINITE = 4,
  TQ_DEV_SCALE_RANGE = 8   /* reserved: set by no kernel since ABI 1.02 (every finite scale is handled) */
};

/* Input dtypes of tq4_1s_quantize. */
enum { TQ_DTYPE_F32 = 0, TQ_DTYPE_BF16 = 1 };

/* Bits of tq4_1s_weight.flags.
 *   TQ_WEIGHT_STATIC: the caller guarantees that no kernel that may still be
 *   running when a call reading this weight is enqueued writes its codes or
 *   scales -- every write to them (tq4_1s_quantize included) has completed,
 *   e.g. the stream or device was synchronized after it, as when weights are
 *   quantized or loaded once at start-up.  The decode-block kernel of
 *   tq4_1s_linear may then start streaming the weight before the previous
 *   kernel on the stream has finished (its own input still waits).  Without
 *   the bit every read of the weight waits for the previous kernel.  Setting
 *   it for a weight that an unfinished kernel writes gives undefined results.
 * Other bits must be 0. */
enum { TQ_WEIGHT_STATIC = 1 };

/* A packed TQ4_1S tensor or stack of num_experts tensors of shape [n][k]. */
typedef struct {
  int64_t n;            /* rows (output features), > 0                          */
  int64_t k;            /* columns (input features), > 0, multiple of 32        */
  int32_t num_experts;  /* 1 for a dense layer                                  */
  int32_t flags;        /* TQ_WEIGHT_* bits; 0 by default                      */
  uint64_t seed;        /* RHT seed; the sign mask is derived from it           */
  uint8_t* codes;       /* device, [num_experts][n][k/2], 16-byte aligned       */
  uint16_t* scales;     /* device, [num_experts][n][k/16], 16-byte aligned      */
} tq4_1s_weight;

/* ABI version of this header (major * 100 + minor). */
int tq4_1s_version(void);

/* Human-readable text for a return code or status bit.  Never NULL. */
const char* tq4_1s_error_string(int code);

/* Host, pure.  Bytes of the codes and scales planes of an [e][n][k] stack
 * (n*k/2*e and n*(k/16)*2*e: exactly 5 bits per weight, per the ~5 bits per
 * weight of "What Config-I means").  INVALID_ARG for bad sizes. */
int tq4_1s_packed_bytes(int64_t n, int64_t k, int32_t num_experts, size_t* codes_bytes, size_t* scales_bytes);

/* Host, pure.  The RHT sign mask of a seed: low 32 bits of the first output
 * of SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) from state `seed`.
 * Reading of the randomized rotation of "What Config-I means", whose signs
 * the card does not specify. */
int tq4_1s_sign_mask(uint64_t seed, uint32_t* mask);

/* Host, pure.  The fp32 codebook the kernels use: levels[16], the 16-level
 * Lloyd-Max quantizer of N(0,1) ("16-level Lloyd-Max", What Config-I means),
 * ascending; thresholds[15], the fp32 midpoints.  Either pointer may be NULL. */
int tq4_1s_codebook(float* levels, float* thresholds);

/* Quantize W (device, [num_experts][n][k], dtype F32 or BF16, row-major,
 * 16-byte aligned) into out->codes / out->scales (device buffers sized by
 * tq4_1s_packed_bytes) with the RHT seed out->seed.  Steps: sign flip,
 * 32-point butterfly, x r, half-block RMS, fp16 scale, nearest level by the
 * 15 midpoints, nibble packing ("What Config-I means").  A block holding a
 * NaN or infinity sets TQ_DEV_NONFINITE; its output follows the same
 * arithmetic (NaN scales are stored as 0x7E00, NaN codes as 0). */
int tq4_1s_quantize(const void* W, int dtype, const tq4_1s_weight* out, tq4_stream_t stream);

/* tq4_1s_quantize for `count` tensors in as few launches as possible (up to
 * 48 tensors per launch), as when a whole checkpoint is converted
 * ("Reproduction": the quantizer runs on the GPU).  W is a HOST array of
 * `count` device pointers, outs a HOST array of `count` weight descriptors;
 * tensor i is quantized from W[i] into outs[i] exactly as tq4_1s_quantize
 * would (same bits), all inputs of one dtype.  Every descriptor and pointer
 * is validated before anything is launched; count == 0 is a no-op. */
int tq4_1s_quantize_batched(const void* const* W, int dtype, const tq4_1s_weight* outs, int32_t count,
                            tq4_stream_t stream);

/* Dequantize a packed tensor stack to fp32 W_out (device, [E][n][k]):
 * W_hat = diag(s) * r * H * (c[code] * d) per block.  Test/debug path. */
int tq4_1s_dequantize(const tq4_1s_weight* w, float* W_out, tq4_stream_t stream);

/* Bytes of workspace tq4_1s_linear needs for m rows with weight w (dense,
 * num_experts == 1).  0 on invalid arguments.
 * Small m (<= 128): the workspace holds the rotated activations, the
 * stream-K partial sums and the tile counters; large m: the bf16 dequantized
 * weight.  No initialisation is needed: the tile counters carry each launch's
 * epoch and the launch that finishes a split tile resets its counter, so a
 * call may also be captured into a CUDA graph and replayed.  Calls that
 * share a workspace must not overlap on the GPU. */
size_t tq4_1s_linear_workspace(int64_t m, const tq4_1s_weight* w);

/* The quantized linear layer of "Running it": y[m][n] = bf16(x * W_hat^T),
 * fp32 accumulation on the tensor cores, no bias.
 *   x  device bf16 bits [m][k], row-major, 16-byte aligned;
 *   y  device bf16 bits [m][n], row-major, 16-byte aligned;
 *   ws device workspace of at least tq4_1s_linear_workspace(m, w) bytes,
 *      16-byte aligned, owned by the caller.
 * Small m (<= 128) rotates each 32-slice of x by the weight's own RHT
 * (x' = R x; R's orthogonality makes this equivalent to inverse-rotating W),
 * scales each row by a power of two that keeps it inside the fp16 range,
 * rounds it to fp16, and multiplies the rotated-domain levels
 * fp16(256 c[code]) * d (fp16 product) by x' on the tensor cores, streaming
 * the packed weight once and scaling back exactly.  For m <= 32 with a short
 * k range per CTA this is one kernel launch (the kernel rotates x itself;
 * the CTAs sharing a row tile form a cluster and reduce their partial sums
 * on chip); there a power of two per row and dequant group, taken from the
 * row's largest half-block scale, keeps the levels normal and finite for
 * every finite scale.  Otherwise a stream-K kernel splits the weight stream
 * evenly over the SMs (x' from a rotation kernel through the workspace, or
 * rotated in the kernel); its levels are finite for half-block scales up to
 * 65504 / fp16(256 c_max) (about 93.6), and where a larger scale makes a
 * row's sums non-finite the kernel recomputes that row's part exactly on
 * the CUDA cores (slower, same result).  Large m dequantizes W_hat to bf16
 * in the workspace and runs a tensor-core GEMM.
 * m == 0 is a no-op. */
int tq4_1s_linear(const uint16_t* x, int64_t m, const tq4_1s_weight* w, uint16_t* y, void* ws, size_t ws_bytes,
                  tq4_stream_t stream);

/* The fp8-resident weight cache of the model card's "Help wanted" section:
 * dequantize the TQ4_1S weight once and keep it resident in fp8 (about 8
 * bits per weight instead of 5), so no forward pass dequantizes TQ4_1S.
 * Format (reading; the card names only "fp8"): OCP E4M3 codes q [rows][k]
 * (row-major bytes, rows = n * num_experts) and one fp32 scale per row,
 *   s_n = fp32(amax_n / 448),  q[n][k] = E4M3(fp32(W_hat[n][k] / s_n))
 * with W_hat the dequantized weight (as tq4_1s_dequantize computes it),
 * amax_n the largest |W_hat| of row n, rounding to nearest even, saturating
 * at +-448; a zero row has s_n = 0 and zero codes.  The cached weight is
 * s_n * q[n][k].
 *   q      device uint8 [rows][k], 16-byte aligned, written;
 *   wscale device float [rows], 16-byte aligned, written. */
int tq4_1s_to_fp8(const tq4_1s_weight* w, uint8_t* q, float* wscale, tq4_stream_t stream);

/* Workspace bytes of tq4_1s_linear_fp8 (the bf16 weight of its large-m
 * path); 0 on invalid arguments or m == 0. */
size_t tq4_1s_linear_fp8_workspace(int64_t m, int64_t n, int64_t k);

/* y[m][n] = bf16(x * (s q)^T) with the fp8 cache (q [n][k], wscale [n]) of
 * tq4_1s_to_fp8; fp32 accumulation on the tensor cores.  For m <= 32 this is
 * the decode-block kernel of tq4_1s_linear streaming 1 byte per weight (the
 * E4M3 values convert to fp16 exactly; x is scaled per row by a power of two
 * and rounded to fp16; no workspace is used and ws may be NULL); otherwise
 * the cache is expanded to a bf16 weight in the workspace and multiplied by
 * the tensor-core GEMM.  flags: TQ_WEIGHT_STATIC or 0, as for tq4_1s_weight.
 * k % 32 == 0; m == 0 is a no-op. */
int tq4_1s_linear_fp8(const uint16_t* x, int64_t m, const uint8_t* q, const float* wscale, int64_t n, int64_t k,
                      int32_t flags, uint16_t* y, void* ws, size_t ws_bytes, tq4_stream_t stream);

/* A second weight format, for a bytes-versus-accuracy comparison with
 * TQ4_1S: the MLX port's affine group quantization ("Nemotron-Labs-TwoTower-
 * 30B-A3B -- MLX 6-bit", section "Quantization (6-bit, scheme mixed_v1)":
 * the bulk of the weights at 6 bits, embeddings and heads at >= 8 bits; the
 * family also at 4 bits).  Reading of what the README leaves open: groups
 * of 64 consecutive weights of a row; per group scale = (max - min) /
 * (2^bits - 1) and bias = min, computed in fp32 and stored as bf16;
 * q = clamp(rint(fp32(fp32(w - bias) / scale)), 0, 2^bits - 1) against the
 * stored values (a zero scale gives q = 0); the codes of a row are one
 * little-endian bit stream (element i in bits [bits i, bits i + bits)).
 * Dequantized weight: fp32(fp32(scale * q) + bias).  bits + 0.5 bits per
 * weight (4.5, 6.5, 8.5). */
typedef struct {
  int64_t n;          /* rows, > 0                                             */
  int64_t k;          /* columns, > 0, multiple of 64                          */
  int32_t bits;       /* 4, 6 or 8                                             */
  int32_t reserved;   /* must be 0                                             */
  uint8_t* codes;     /* device, [n][k * bits / 8], 16-byte aligned            */
  uint16_t* scales;   /* device, bf16 bits [n][k / 64], 16-byte aligned        */
  uint16_t* biases;   /* device, bf16 bits [n][k / 64], 16-byte aligned        */
} tq4_1s_affine_weight;

/* Quantize W (device fp32 [n][k], 16-byte aligned) into out's planes. */
int tq4_1s_affine_quantize(const float* W, const tq4_1s_affine_weight* out, tq4_stream_t stream);

/* Dequantize to fp32 W_out (device [n][k]). */
int tq4_1s_affine_dequantize(const tq4_1s_affine_weight* w, float* W_out, tq4_stream_t stream);

/* Workspace bytes of tq4_1s_affine_linear (the bf16 weight); 0 on invalid
 * arguments. */
size_t tq4_1s_affine_linear_workspace(int64_t m, const tq4_1s_affine_weight* w);

/* y[m][n] = bf16(x * W_hat^T) for the affine format: the weight dequantized
 * to bf16 in the workspace, then the tensor-core GEMM (the comparison path;
 * the TQ4_1S decode kernel is the streaming one).  m == 0 is a no-op. */
int tq4_1s_affine_linear(const uint16_t* x, int64_t m, const tq4_1s_affine_weight* w, uint16_t* y, void* ws,
                         size_t ws_bytes, tq4_stream_t stream);

/* tq4_1s_linear for callers that cannot allocate device memory.  (The model
 * card has no counterpart: this is a deployment variant of the layer above.)
 * Plugin hosts and serving runtimes that fix every device allocation at
 * start-up and forbid new ones later cannot hand tq4_1s_linear a workspace;
 * this entry point takes only x, w and y and keeps its scratch (rotated
 * activations, stream-K partial sums, tile counters) in a fixed device array
 * inside the library: about 5.2 MiB per GPU, reserved when the library's
 * device code is loaded on that GPU -- under CUDA's default lazy module
 * loading, at the first call there (this entry point's first call loads it)
 * -- and held until the process exits.  A caller with a fixed memory budget
 * makes one warm-up call at start-up, outside any stream capture, so that
 * the reservation happens then.
 *   Limits: m <= 32, w->k <= 8192, w->n <= 32768, dense weight; larger
 *   shapes return TQ_ERR_SCRATCH_LIMIT and launch nothing.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call outside any stream capture.
 *   All calls share the one array, so calls that overlap on the GPU (on
 *   different streams, or from different host threads) race and corrupt each
 *   other's results; serialize them.  Each launch tags the tile counters
 *   it uses with its own epoch and resets those it finishes, so a previous
 *   call's leftovers do no harm, also across replays of a CUDA graph.
 * Same arguments, result and numerics as tq4_1s_linear's small-m path; no
 * allocation of any kind. */
int tq4_1s_linear_static(const uint16_t* x, int64_t m, const tq4_1s_weight* w, uint16_t* y, tq4_stream_t stream);

/* Bytes of workspace tq4_1s_moe needs.  0 on invalid arguments. */
size_t tq4_1s_moe_workspace(int64_t m, int32_t topk, const tq4_1s_weight* up, const tq4_1s_weight* down);

/* The sync-free MoE layer ("Performance"; 128 experts top-6 in "The model
 * underneath"):  for each token t and slot j < topk with expert
 * e = topk_ids[t][j] and weight w = topk_w[t][j]:
 *     u = x_t * W_up[e]^T,  h = bf16(relu(u)^2),  z = h * W_down[e]^T,
 *     y_t = bf16(sum_j w_tj * z_tj)      (slots in order)
 *   x        device bf16 bits [m][H]            (H = up->k = down->n)
 *   topk_ids device int32 [m][topk]; ids outside [0, E) are skipped and set
 *            TQ_DEV_BAD_ROUTING
 *   topk_w   device float [m][topk]
 *   up       stack of E experts [I][H]; down stack of E experts [H][I]
 *   y        device bf16 bits [m][H]
 *   ws       device workspace of tq4_1s_moe_workspace() bytes.
 * Routing, gathering, both projections and the combine all run on the
 * device; nothing synchronizes with the host, and the call can be captured
 * into a CUDA graph and replayed (same workspace rules as tq4_1s_linear). */
int tq4_1s_moe(const uint16_t* x, int64_t m, const int32_t* topk_ids, const float* topk_w, int32_t topk,
               const tq4_1s_weight* up, const tq4_1s_weight* down, uint16_t* y, void* ws, size_t ws_bytes,
               tq4_stream_t stream);

/* tq4_1s_moe with the router on the device (model card, "Performance": the
 * MoE made sync-free; "The model underneath": top-6 of 128 experts): the
 * routing decisions come from the router's logits instead of the caller.
 *   logits device float [m][E] (E = up->num_experts <= 1024), 16-byte
 *          aligned; topk <= 32 and <= E.
 * Per token: softmax over all E experts, the topk of largest probability
 * chosen (equal logits: the lower expert id first), their probabilities
 * renormalised to sum to 1 -- as tq4_1s_router_topk -- then the layer of
 * tq4_1s_moe with those ids and weights.  The router runs inside the routing
 * kernel, so the call is the same number of launches as tq4_1s_moe, needs no
 * host sync, and captures into a CUDA graph.  Workspace: tq4_1s_moe_workspace
 * (it includes room for the router's output).  A NaN logit is never chosen
 * and sets TQ_DEV_NONFINITE. */
int tq4_1s_moe_logits(const uint16_t* x, int64_t m, const float* logits, int32_t topk, const tq4_1s_weight* up,
                      const tq4_1s_weight* down, uint16_t* y, void* ws, size_t ws_bytes, tq4_stream_t stream);

/* The MoE router on its own (parity hook and standalone use):
 *   logits  device float [m][num_experts] (num_experts <= 1024);
 *   ids     device int32 [m][topk] (topk <= 32, <= num_experts): the chosen
 *           experts in descending logit order, equal logits lower id first;
 *   weights device float [m][topk]: exp(z_j - z_max) / sum over the chosen,
 *           i.e. the full softmax restricted to the chosen and renormalised
 *           (computed in fp64, rounded to fp32).
 * m == 0 is a no-op. */
int tq4_1s_router_topk(const float* logits, int64_t m, int32_t num_experts, int32_t topk, int32_t* ids,
                       float* weights, tq4_stream_t stream);

/* The routing step of tq4_1s_moe on its own (exposed for parity tests):
 * offsets (device int32 [num_experts + 1]) = exclusive prefix of per-expert
 * counts; pairs (device int32 [m*topk]) = flat slot indices t*topk + j
 * grouped by expert, ascending within an expert.  Entries past
 * offsets[num_experts] are left unspecified. */
int tq4_1s_moe_route(const int32_t* topk_ids, int64_t m, int32_t topk, int32_t num_experts, int32_t* offsets,
                     int32_t* pairs, tq4_stream_t stream);

/* Host, pure.  Number of kernel launches this process has issued through
 * the library so far (all devices); a launch captured into a CUDA graph
 * counts once, at capture. */
uint64_t tq4_1s_launch_count(void);

/* Test hooks -- fault injection for the library's failure-handling tests;
 * not for production use.  (The model card has no counterpart.)
 *   TQ_HOOK_FAIL_NEXT_CALLS, value n >= 0: the next n calls that would
 *     launch kernels fail with TQ_ERR_CUDA after validating their arguments
 *     and before launching anything (a host-side stand-in for a failed
 *     launch); 0 cancels.  Host only.
 *   TQ_HOOK_WAIT_NS, value ns >= 0: the limit of every bounded device wait
 *     on the current device (0 restores the default of 2 s).
 *   TQ_HOOK_WITHHOLD_ARRIVAL, value 0 or 1: while 1, the decode-block kernel
 *     of tq4_1s_linear runs with one rotation warp that never reports its
 *     activations ready, so the waits on them run out: the kernel sets
 *     TQ_DEV_TIMEOUT, lets its copies and MMAs finish, frees its tensor
 *     memory and returns (the output is then unspecified).
 * Returns TQ_OK, or TQ_ERR_INVALID_ARG for an unknown hook or value. */
enum { TQ_HOOK_FAIL_NEXT_CALLS = 1, TQ_HOOK_WAIT_NS = 2, TQ_HOOK_WITHHOLD_ARRIVAL = 3 };
int tq4_1s_debug_hook(int what, int64_t value);

/* Synchronize `stream`, then read and clear the current device's status
 * word (a mask of TQ_DEV_* bits) into *status (host). */
int tq4_1s_get_status(tq4_stream_t stream, int32_t* status);

#ifdef __cplusplus
}
#endif

#endif /* TQ4_1S_H_ */
