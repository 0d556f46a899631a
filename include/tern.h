/*
 * tern.h -- C ABI of the packed ternary-weight GEMV library (libtern.so).
 *
 * The library computes, for a weight matrix W of N rows (outputs) by K
 * columns (inputs) stored as packed trit planes t in {-1, 0, +1},
 *
 *     y[m][n] = sum_p sum_groups s[p][n][grp] * sum_{k in grp} t[p][n][k] * x[m][k]
 *
 * in three weight formats:
 *   TERN_FMT_BITNET  one plane, 2 bits per weight, 4 weights per byte, one
 *                    per-tensor scale applied once at the end ("Ternary GEMV
 *                    (No Multiplication)", QORA-LLM-2B model page);
 *   TERN_FMT_TQ      K additive trit planes ("TQ{K}P"), one fp16 scale per
 *                    plane per group of g weights along the input dimension
 *                    (sasori README, "K and g - the quality dials" and
 *                    "How it works");
 *   TERN_FMT_BT3     balanced ternary of depth d (3^d levels): weight =
 *                    cb[idx] * sum_j 3^j t_j (d = 3: 9 t2 + 3 t1 + t0, 27
 *                    levels), trits base-3 packed five per byte, group 16,
 *                    27-entry log-spaced scale codebook with the index stored
 *                    as three trits (Entrit Llama-3.1-8B-trit-uniform-d3
 *                    card, "Quantization details", d = 3; depths 2 and 4 by
 *                    the same rule: the card's positional weights, one trit
 *                    fewer or more per weight).
 *
 * Conventions for every call:
 *   - All pointers named d_* are device pointers; the others are host
 *     pointers. The caller owns every buffer; the library allocates no memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device work is enqueued asynchronously on it.
 *   - Argument errors are detected on the host and returned before anything
 *     is enqueued. A launch failure returns TERN_ECUDA.
 *   - Device-side failures (a bounded wait that expired inside a kernel) are
 *     recorded in a device error word; tern_device_error() reads and clears it.
 *   - Activations and outputs are row-major [M][K] and [M][N]. bf16 values
 *     are passed as their 16-bit patterns.
 *
 * The packed buffer layout is fixed by tern_pack(); it is documented in the
 * repository's design notes and decoded independently by the test oracle.
 */
#ifndef TERN_H_
#define TERN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TERN_ABI_VERSION 1

typedef enum {
  TERN_OK = 0,
  TERN_EINVAL = 1,       /* bad argument: NULL pointer, size, unsupported value */
  TERN_EFORMAT = 2,      /* bad data: a trit outside {-1,0,1}, an index above 26,
                            a non-finite scale, or a packed header that does not
                            match the descriptor */
  TERN_EALIGN = 3,       /* a device pointer is not 16-byte aligned */
  TERN_ENOSPACE = 4,     /* output buffer or workspace smaller than required */
  TERN_EUNSUPPORTED = 5, /* valid request this build has no kernel for */
  TERN_ECUDA = 6,        /* a CUDA runtime call failed */
  TERN_ETIMEOUT = 7      /* a bounded wait inside a kernel expired */
} tern_status;

typedef enum { TERN_FMT_BITNET = 1, TERN_FMT_TQ = 2, TERN_FMT_BT3 = 3 } tern_format;

/* TERN_ACT_INT8: x is int8 [M][K] with one fp32 scale per token (x = xq * sx);
 *   the sums are exact integers and y is fp32, bit-identical to the oracle.
 * TERN_ACT_BF16: x is bf16 [M][K]; y is accurate to fp32 accumulation (each
 *   group's sum is exact for every activation within 2^15 of the group's
 *   largest, then rounded once to fp32 and accumulated in fp32).
 * TERN_ACT_BF16_Q8: x is bf16 [M][K]; each token is quantised to int8 inside
 *   the GEMV by the rule of tern_quantize_act, then the int8 path runs; the
 *   result is bit-identical to tern_quantize_act followed by TERN_ACT_INT8
 *   (d_xscale is ignored). BITNET and TQ only. */
typedef enum { TERN_ACT_INT8 = 1, TERN_ACT_BF16 = 2, TERN_ACT_BF16_Q8 = 3 } tern_act;
typedef enum { TERN_OUT_F32 = 1, TERN_OUT_BF16 = 2 } tern_out;

/* Descriptor flags. */
#define TERN_F_PDL 1u /* launch with programmatic dependent launch: the kernel may
                         read the packed weights before the preceding kernel on
                         the stream has finished (it still waits for that kernel
                         before it reads x or writes y or the workspace). Set it
                         only when no preceding kernel writes the packed buffer. */

typedef struct tern_desc {
  int32_t fmt;          /* tern_format */
  int32_t n;            /* output rows N >= 1 */
  int32_t k;            /* input columns K >= 1 */
  int32_t planes;       /* BITNET: 1; TQ: 1..4; BT3: the depth d, 2..4 */
  int32_t group;        /* BITNET: ignored (whole row); TQ: g, a multiple of 16
                           in {16,32,64,128,256} dividing K; BT3: 16 */
  float tensor_scale;   /* BITNET: the per-tensor scale s_w; else ignored */
  uint32_t flags;       /* TERN_F_* */
} tern_desc;

/* Human-readable name of a status code (static string). */
const char* tern_status_string(tern_status s);

/* Size in bytes of the packed buffer for `desc` (256-byte header + streams).
 * Follows the pages' bits-per-weight accounting: sasori README, "K and g -
 * the quality dials" (K (2 + 16/g) bits per weight for TQ{K}P); Entrit card,
 * "Quantization details" (about 5 bits per weight at d = 3, group 16); the
 * physical size adds whole 32-row tiles and 64- or 80-weight columns. */
tern_status tern_packed_size(const tern_desc* desc, size_t* bytes);

/*
 * Pack logical weights into the library's layout (host only, no device work).
 * The pages' "convert once, then run" step: sasori README, "Quickstart -
 * quantize" (the quantiser writes a packed GGUF) and QORA-LLM-2B, "Converting
 * from Safetensors" (bf16 weights to a 2-bit ternary binary); the byte layout
 * is this library's own (the pages' formats are not given in full).
 *   trits       int8 [planes][N][K], values -1, 0, +1 (TERN_EFORMAT otherwise).
 *               BT3: plane p holds t_p, the trit of weight 3^p (p < d).
 *   scales_fp16 TQ: fp16 bit patterns [planes][N][K/group], finite; else NULL.
 *   scale_idx   BT3: uint8 [N][K/16], values 0..26 (codebook index); else NULL.
 *   codebook    BT3: float [27], finite; stored in the header; else NULL.
 *   out         host buffer of out_cap bytes (TERN_ENOSPACE if too small);
 *               *out_used receives the packed size.
 * TQ scales are also checked against the exactness bound of the int8 path
 * (the exact group-scaled sum must fit in 62 bits; TERN_EFORMAT otherwise).
 */
tern_status tern_pack(const tern_desc* desc, const int8_t* trits, const uint16_t* scales_fp16,
                      const uint8_t* scale_idx, const float* codebook, void* out, size_t out_cap,
                      size_t* out_used);

/*
 * Workspace needed by tern_gemv / tern_gemm_batched for `m` tokens. No page
 * defines it: it is this library's scratch for split reductions and the
 * tensor-core path.
 *   m < 16: 0 for most layers (K-splits normally reduce inside a thread-block
 *     cluster; only a very long K needs more splits than a cluster holds).
 *   m >= 16 (2-bit formats, TERN_ACT_INT8 or TERN_ACT_BF16_Q8): the tensor-
 *     core path needs arrival counters and exact int64 partial sums for the
 *     row tiles that several CTAs share (sized for 256 tokens), the
 *     activations in MMA order and, for bf16 input, their int8 quantisation.
 * The workspace must be 256-byte aligned and zero-filled before its first
 * use; every call leaves its counters and partial sums at zero again, so the
 * workspace can be reused by later calls (with any m up to the m it was sized
 * for) without clearing. Calls that may run at the same time need separate
 * workspaces.
 */
tern_status tern_workspace_size(const tern_desc* desc, int32_t m, size_t* bytes);

/*
 * Per-token absmax int8 quantisation of bf16 activations (a reading of the
 * single-GEMV workload's "per-token absmax"; the pages give no rounding rule):
 *   a = max |x|, inv = fl32(127 / a), xq = clamp(rint(fl32(x * inv)), -127, 127)
 *   (round half to even), sx = fl32(a / 127); an all-zero token gives xq = 0, sx = 0.
 *   A token whose a is below 127 / FLT_MAX (about 3.7e-37) has inv = +inf: its
 *   non-zero values give +-127 and its zeros 0. Activations must be finite.
 *   d_x_bf16 [m][k] bf16 bits; d_xq int8 [m][k]; d_xscale float [m].
 */
tern_status tern_quantize_act(const uint16_t* d_x_bf16, int32_t m, int32_t k, int8_t* d_xq,
                              float* d_xscale, void* stream);

/*
 * y = W x for one token (M = 1); same as tern_gemm_batched with m = 1.
 * The decode GEMV of the pages: QORA-LLM-2B, "Ternary GEMV (No
 * Multiplication)" (add/sub of activations, one scalar multiply at the end);
 * sasori README, "How it works" (per-group scaled trit planes, additions
 * instead of weight multiplies); Entrit card, "Quantization details".
 *   d_packed  the bytes produced by tern_pack, copied to the device,
 *             16-byte aligned.
 *   act       TERN_ACT_INT8: d_x int8 [K], d_xscale float [1];
 *             TERN_ACT_BF16: d_x bf16 [K], d_xscale NULL;
 *             TERN_ACT_BF16_Q8: d_x bf16 [K], quantised inside the GEMV
 *             (d_xscale ignored). BT3 takes TERN_ACT_BF16 only.
 *   out       TERN_OUT_F32 (float [N]) or TERN_OUT_BF16 (bf16 bits [N]).
 *   d_ws      workspace of ws_bytes (see tern_workspace_size); may be NULL when
 *             tern_workspace_size reports 0, otherwise TERN_ENOSPACE.
 */
tern_status tern_gemv(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                      const float* d_xscale, tern_out out, void* d_y, void* d_ws, size_t ws_bytes,
                      void* stream);

/*
 * Y = X W^T for m tokens (m >= 1), the weights read once for all tokens.
 * The same product as tern_gemv for a batch of tokens (sasori README, "g
 * (group-size)": fine groups cost decode speed; the several-token and prefill
 * forms are this library's, the pages run one token at a time).
 *   d_x [m][K] (int8 or bf16 bits), d_xscale float [m] for TERN_ACT_INT8,
 *   d_y [m][N]. For TERN_ACT_INT8 the result is bit-identical to the oracle.
 *   TERN_ACT_BF16 (TQ and BT3) runs on the CUDA cores for any m: balanced
 *   ternary reads the weights once per pass of up to eight tokens, the TQ
 *   planes once per token.
 * For m >= 16 with the 2-bit formats and int8 (or in-kernel quantised bf16)
 * activations the product runs on the tensor cores (tcgen05 int8 MMA, up to
 * 256 tokens per launch); the fp16 group scales are split into small integer
 * digits folded into the int8 weight operand, so the result stays exact.
 * That path needs the workspace tern_workspace_size(desc, m) reports
 * (TERN_ENOSPACE without it); from m = 9 it is taken whenever that workspace
 * is given, and from m = 5 when the activations of a CUDA-core pass would
 * crowd shared memory (long K). Otherwise, with 2..15 tokens, the weights are
 * read once per pass of up to eight tokens on the CUDA cores; those kernels
 * cover BitNet, TQ{1..4}P with g = 256, TQ2P with g = 32 and TQ3P with g = 64;
 * other plane and group combinations take the tensor path with a workspace
 * (TERN_EUNSUPPORTED without one). One token: every TQ{1..4}P with
 * g = 32, 64, 128, 256.
 */
tern_status tern_gemm_batched(const tern_desc* desc, const void* d_packed, int32_t m, tern_act act,
                              const void* d_x, const float* d_xscale, tern_out out, void* d_y,
                              void* d_ws, size_t ws_bytes, void* stream);

/*
 * Several independent single-token GEMVs in one launch (for example the q, k
 * and v projections of a decode step, or gate and up). The pages state one
 * GEMV per projection (QORA-LLM-2B, "SubLN Pattern"); running independent
 * ones together is a launch-level choice of this library.
 *   count       1..256 problems; descs[i] must share fmt, planes, group and
 *               flags (n and k may differ; a launch with several k balances
 *               its work by columns, and smaller launches run one kernel per
 *               run of equal k).
 *   d_packed[i], d_x[i] ([K]), d_xscale[i] (TERN_ACT_INT8, else ignored and may
 *               be NULL), d_y[i] ([n_i]): as tern_gemv, one per problem.
 * Needs no workspace. Returns TERN_EUNSUPPORTED if K is too large to split
 * within one thread-block cluster.
 */
tern_status tern_gemv_grouped(int32_t count, const tern_desc* descs, const void* const* d_packed, tern_act act,
                              const void* const* d_x, const float* const* d_xscale, tern_out out, void* const* d_y,
                              void* stream);

/*
 * tern_gemv without a caller-provided workspace, for callers that cannot
 * allocate device memory (code running where cudaMalloc is not permitted, or
 * inside a framework that owns every device allocation). The pages have no
 * counterpart; this is a deployment convenience of this library.
 *   Arguments as tern_gemv (one token), minus d_ws / ws_bytes.
 *   Scratch: a fixed 1 MiB array in device memory owned by the library; every
 *   GPU that loads the library holds it until the process exits. A layer whose
 *   workspace (tern_workspace_size with m = 1: the largest over all
 *   activation modes, whatever `act` is) exceeds 1 MiB is rejected with
 *   TERN_ENOSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture. The address is kept for the life of the process: after
 *   cudaDeviceReset (or any teardown of the device's primary context) this
 *   call must not be used again in that process. Each call clears the part of
 *   the scratch it uses on `stream`
 *   (cudaMemsetAsync) and never allocates or frees memory.
 *   All calls on a device share the same scratch: calls that may overlap on
 *   the GPU (different streams without ordering between them) race.
 */
tern_status tern_gemv_noalloc(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                              const float* d_xscale, tern_out out, void* d_y, void* stream);

/*
 * Read-ceiling measurement: stream `bytes` of d_src once, folding them into a
 * checksum, with one of the access shapes the GEMV kernels can use (the pages
 * have no counterpart; the bandwidth it reaches is the roofline the GEMV
 * kernels are reported against).
 *   mode 0: 16-byte loads per thread, `depth` (1, 2, 4 or 8) in flight;
 *   mode 1: bulk async copies of `chunk` bytes into a per-warp ring of `depth`
 *           shared-memory stages; mode 2: one such ring per CTA.
 *   ctas_per_sm x SM-count CTAs of 32*warps threads; d_sink: one unsigned
 *   (left unchanged unless a checksum hits a fixed value). d_src 16-byte aligned.
 */
tern_status tern_stream_read(const void* d_src, size_t bytes, int32_t mode, int32_t chunk, int32_t depth,
                             int32_t ctas_per_sm, int32_t warps, unsigned* d_sink, void* stream);

/*
 * Read and clear the device error word (synchronises `stream`).
 * Returns TERN_OK if no kernel reported a failure, TERN_ETIMEOUT if a bounded
 * wait expired, TERN_EFORMAT if a kernel met packed data it cannot use (the
 * tensor path: a header scale-digit count outside 1..6), TERN_ECUDA if the
 * read failed.
 */
tern_status tern_device_error(void* stream);

/*
 * Dense -> ternary fit of a weight matrix on the GPU, producing the inputs of
 * tern_pack (the pages' "quantize" step: sasori README, "How it works & paper"
 * -- each matrix fit on its own into K per-group-scaled trit planes, weight
 * only, no calibration -- and "K and g"). Greedy residual planes: per row and
 * group of g, and plane p, gamma = mean |R_p|; t = sign(R_p) where |R_p| >
 * gamma / 2, else 0; s = fp16_rn(mean of |R_p| over the non-zero trits) (0 if
 * none); R_{p+1} = R_p - s t; R_0 = W. fp64 arithmetic, group sums in index
 * order.
 *   d_w       fp32 [n][k], device.
 *   d_trits   int8 [planes][n][k] out; d_scales fp16 bits [planes][n][k/group] out.
 *   planes 1..4; group a power of two in 16..256 dividing k.
 */
tern_status tern_fit_tq(const float* d_w, int32_t n, int32_t k, int32_t planes, int32_t group, int8_t* d_trits,
                        uint16_t* d_scales, void* stream);

/*
 * Dense -> balanced ternary fit of depth d (Entrit card, "Quantization
 * details": uniform PTQ, depth 3, group 16, 27-entry log-spaced codebook):
 * per row and group of 16, for each codebook entry c the levels L =
 * clamp(rint(w / c), -(3^d-1)/2, (3^d-1)/2); the entry with the least sum of
 * squared errors (lowest index on a tie); trits = balanced-ternary digits of L
 * (L = sum_j 3^j t_j). fp64 arithmetic, sums in index order.
 *   d_w        fp32 [n][k], k a multiple of 16; d_codebook fp32 [27], device.
 *   d_trits    int8 [depth][n][k] out; d_idx uint8 [n][k/16] out. depth 2..4.
 */
tern_status tern_fit_bt(const float* d_w, int32_t n, int32_t k, int32_t depth, const float* d_codebook,
                        int8_t* d_trits, uint8_t* d_idx, void* stream);

/*
 * Decode step of a BitNet b1.58 transformer at batch 1 (QORA-LLM-2B page,
 * "Architecture" and "SubLN Pattern (4 norms per layer)"). Per layer:
 *   x = RMSNorm(h) -> q, k, v (ternary linears) -> RoPE (rotate_half) on q, k
 *   -> k, v appended to the bf16 cache at `pos` -> GQA attention over
 *   positions 0..pos -> RMSNorm -> o_proj -> h += o -> RMSNorm -> gate, up ->
 *   RMSNorm(relu(gate)^2 * up) -> down_proj -> h += d.
 * Every ternary linear quantises its input per token to int8 (the rule of
 * tern_quantize_act on fp32 values) and is exact as in tern_gemv. RMSNorm:
 * y_i = fl(fl(x_i * r) * g_i), r = 1/sqrt(mean(x^2) + eps) rounded once to
 * fp32. RoPE products and sums rounded in fp32; relu^2 * up and the residual
 * adds in fp32; attention (scores scaled by 1/sqrt(128), softmax, weighted
 * values) in fp32.
 */
typedef struct tern_decode_model {
  int32_t layers;        /* 1..64 */
  int32_t hidden;        /* D, a multiple of 64 */
  int32_t inter;         /* F (FFN width), a multiple of 64 */
  int32_t heads;         /* H query heads of 128; H * 128 a multiple of 64 */
  int32_t kv_heads;      /* KVH, H / KVH in 1..4, KVH <= 16 */
  int32_t head_dim;      /* 128 */
  int32_t max_pos;       /* cache capacity in positions */
  float eps;             /* RMSNorm epsilon */
  /* host array [layers * 7] of device pointers to tern_pack'ed BitNet buffers
     (16-byte aligned), per layer in the order q [H*128][D], k [KVH*128][D],
     v [KVH*128][D], o [D][H*128], gate [F][D], up [F][D], down [D][F] */
  const void* const* packed;
  const float* d_gains;  /* fp32 [layers][2D + H*128 + F]: input_layernorm (D),
                            attn_sub_norm (H*128), post_attention_layernorm (D),
                            ffn_sub_norm (F) */
  uint16_t* d_kcache;    /* bf16 [layers][KVH][max_pos][128] keys (after RoPE) */
  uint16_t* d_vcache;    /* bf16 [layers][KVH][max_pos][128] values */
  const float* d_rope;   /* fp32 [max_pos][64][2] cos, sin (tern_decode_rope_table) */
} tern_decode_model;

/* cos and sin of p * theta^(-2i/head_dim), p < max_pos, i < head_dim/2, each
 * computed in double precision and rounded to fp32, into the host buffer out
 * [max_pos][head_dim/2][2] (RoPE, "rotate_half, theta=500,000" on the
 * QORA-LLM-2B page). */
tern_status tern_decode_rope_table(int32_t max_pos, int32_t head_dim, double theta, float* out);

/* Workspace of tern_decode_step (256-byte aligned, zero-filled before its
 * first use; a completed step leaves it ready for the next). No page defines
 * it: barrier counters, the GEMVs' partial row sums, the attention's partial
 * softmax states and output. */
tern_status tern_decode_workspace_size(const tern_decode_model* model, size_t* bytes);

/*
 * Run stages first..last (inclusive) of the decode step of the token at
 * position `pos` (0 <= pos < max_pos). Stage index = 5 * layer + s with
 * s = 0 q/k/v, 1 attention, 2 o_proj, 3 gate/up, 4 down_proj; a run may
 * start at s = 0, 2 or 3 (TERN_EINVAL otherwise). The whole step is
 * first = 0, last = 5 * layers - 1.
 *   d_h_in   fp32 [D]: the residual stream where the run starts.
 *   d_h_out  fp32 [D]: the residual stream after the run's last residual add.
 *   d_attn_in  fp32 [H*128]: the attention output when the run starts at an
 *              o_proj stage, else ignored (may be NULL).
 *   d_trace  optional fp32 [layers][2*H*128 + 2*KVH*128]: per layer q after
 *            RoPE [H*128], k after RoPE [KVH*128], v [KVH*128], attention
 *            output [H*128] (written for the layers whose stages run).
 * The cache positions 0..pos-1 must hold the earlier tokens' keys and values;
 * the step writes position pos of every layer it runs attention for. One
 * cooperative launch with one CTA per SM; all waits are bounded (1 s), and a
 * step that gave up reports TERN_ETIMEOUT through tern_device_error, after
 * which the workspace must be zero-filled again.
 */
tern_status tern_decode_step(const tern_decode_model* model, int32_t pos, const float* d_h_in, float* d_h_out,
                             int32_t first, int32_t last, const float* d_attn_in, float* d_trace, void* d_ws,
                             size_t ws_bytes, void* stream);

/*
 * Failure-detection self-test (the pages have no counterpart). Enqueues one
 * small kernel whose bounded wait cannot succeed: it waits on a shared-memory
 * barrier that nothing arrives at, gives up after about limit_ns nanoseconds
 * (the GEMV kernels use the same wait with a 1 s limit), records a timeout in
 * the device error word and returns. A later tern_device_error() reports
 * TERN_ETIMEOUT once; the CUDA context stays usable.
 *   limit_ns  1,000 .. 1,000,000,000 (TERN_EINVAL otherwise).
 */
tern_status tern_selftest_wait(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TERN_H_ */
