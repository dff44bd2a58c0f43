/*
 * dit.h — C ABI of the B200 (sm_100a) Flux-style DiT block forward.
 *
 * Sources of the operations (web pages, cited by title and section):
 *   [CG]  "compile_graph" write-up on ChituDiffusion / Flux.1-dev (chenyy20.com):
 *         §1.1 the memory-bound tail fused around each GEMM/attention
 *         (LayerNorm, GELU, adaLN modulation (1+scale)*x+shift);
 *         §2 the traced single-stream block (S=4608, dim 3072, 24 x 128, bf16)
 *         and the 57-block model; §3.1 RoPE as complex arithmetic from position
 *         ids, the double-stream and single-stream block lists; §6.3 attention
 *         operands (B, S, H, D); §1.2 and §4 CUDA-graph capture with static
 *         buffers, fixed shapes and addresses, no host sync, no allocation.
 *   [WAN] Wan2.1 local-acceleration page (mhpq.cn), §1.1: video DiT blocks over
 *         long (t, h, w) token sequences, dominated by self-attention.
 *   [SDXL] SDXL inference-optimisation guide (javey-q.github.io), §3.3:
 *         classifier-free guidance and its late-step cut-off.
 *
 * Conventions shared by every call
 *   - dit_bf16 is the raw bit pattern of a bfloat16 value.
 *   - Every pointer named as a device buffer must point to memory of the
 *     current CUDA device.  The caller owns all memory; the library keeps no
 *     pointer after a call returns, except the graph object, which keeps the
 *     pointers it was created with until it is destroyed.
 *   - Matrices are row-major; a leading dimension (ld*) is the distance between
 *     rows in elements.  Unless a call says otherwise, every device pointer and
 *     every ld * sizeof(element) must be a multiple of 16 bytes (TMA rule).
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Calls enqueue
 *     work on it and return; they neither allocate device memory nor
 *     synchronise, so they can be captured into a CUDA graph.  Exceptions are
 *     named: dit_get_device_error synchronises, dit_forward_graph_create
 *     captures on a private stream.
 *   - The block-path kernels (LN-modulate, adaLN, the GEMMs, attention, the
 *     merge) are launched with programmatic stream serialization: a kernel may
 *     begin its prologue (barrier setup, TMEM allocation) while the previous
 *     kernel of the stream drains, and it touches no global memory before
 *     that kernel has completed, so stream order holds for every buffer.
 *     DIT_DISABLE_PDL=1 in the environment launches them the plain way.
 *   - No call aborts or traps.  Argument errors return a status before any work
 *     is enqueued.  A kernel that waits longer than the wait limit (default 2 s)
 *     on an internal barrier records DIT_ERR_TIMEOUT in the device error word,
 *     releases its resources and exits; dit_get_device_error reports it.
 *   - Per-device state is set up by the first call on each device and kept
 *     until the process exits: kernel attributes, the driver's tensor-map
 *     encoder, the host-buffer pipeline's streams and events, and the address
 *     of the allocation-free call's scratch array.  A device reset
 *     (cudaDeviceReset) while the library is loaded invalidates that state and
 *     is not supported.
 */
#ifndef DIT_H_
#define DIT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library is built with hidden visibility; everything declared here is
 * exported. */
#if defined(DIT_BUILD) && defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef uint16_t dit_bf16;

typedef enum {
  DIT_OK = 0,
  DIT_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
  DIT_ERR_SHAPE = 2,         /* size outside what the kernel supports */
  DIT_ERR_ALIGNMENT = 3,     /* pointer or stride not 16-byte aligned */
  DIT_ERR_UNSUPPORTED = 4,   /* e.g. head_dim != 128, no sm_100 device */
  DIT_ERR_CUDA = 5,          /* a CUDA runtime call failed */
  DIT_ERR_NOT_CAPTURABLE = 6,/* the call cannot run while the stream captures */
  DIT_ERR_TIMEOUT = 7,       /* a device-side wait ran out (device error word) */
  DIT_ERR_WORKSPACE = 8      /* workspace pointer null or too small */
} dit_status;

const char* dit_status_string(dit_status s);

/* Library version as major*10000 + minor*100 + patch. */
int dit_version(void);

/* Text of the last CUDA runtime error that made a call on this host thread
 * return DIT_ERR_CUDA ("no error" if none).  Static storage; do not free. */
const char* dit_last_cuda_error(void);

/* ------------------------------------------------------------------------
 * Device error word and wait limit
 * ------------------------------------------------------------------------ */

/* Synchronises `stream`, then reads the device error word of the current
 * device into *code (0 = no error; otherwise DIT_ERR_TIMEOUT in the low byte
 * and the waiting site in the upper bytes).  Returns DIT_ERR_TIMEOUT when the
 * word is set, DIT_OK otherwise.  Not capturable. */
dit_status dit_get_device_error(void* stream, uint32_t* code);

/* Clears the device error word of the current device (enqueued on stream). */
dit_status dit_clear_device_error(void* stream);

/* Upper bound, in nanoseconds, on any single wait inside a kernel (default
 * 2e9).  Applies to kernels launched after the call. */
dit_status dit_set_wait_limit_ns(uint64_t limit_ns);

/* Opt-in L2 residency for the weight of the output GEMMs (the projections
 * whose activation operand is larger than their weight, e.g. the single-stream
 * block's [attn | mlp] x W2, 94 MB at the Flux width).  Those GEMMs visit
 * their tiles N-fastest, so every wave of tiles re-reads the whole weight; with
 * this set, the weight's loads take the L2 evict-last policy, and at the end of
 * the GEMM each CTA returns its share of the weight to normal priority.
 * bytes: size of the persisting L2 set-aside, clipped to the device maximum
 * (cudaDevAttrMaxPersistingL2CacheSize); 0 turns it off.  This sets
 * cudaLimitPersistingL2CacheSize, a limit of the calling process's context on
 * the current device that every kernel of the process shares, until it is set
 * again or the context ends.  Affects GEMMs launched after the call. */
dit_status dit_set_weight_l2_persist(size_t bytes);

/* Failure-detection self test: launches one CTA that waits on a barrier that
 * nothing ever arrives on, with the given limit.  The kernel must give up,
 * record DIT_ERR_TIMEOUT in the device error word and exit.  Enqueued on
 * stream; read the result with dit_get_device_error. */
dit_status dit_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Self test of the 2^x approximation the attention softmax evaluates on the
 * FMA pipe for a part of its exponentials (Cody-Waite split plus a fitted
 * cubic; stated maximum relative error 7.5e-5; inputs below -126 are clamped
 * to -126).  y[i] = that approximation of 2^x[i]; x, y device float [n]. */
dit_status dit_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* ------------------------------------------------------------------------
 * RoPE table ([CG] §3.1: positions from ids, rotation as complex product)
 * ------------------------------------------------------------------------ */

/* rope[t][p] = (cos phi, sin phi) as two floats, phi = ids[t][a] * theta^(-2j/2P_a)
 * for pair p = (sum of P_b for b < a) + j, where P_a = axes_pairs[a] and the
 * pairs sum to head_dim/2 (Flux: 8, 28, 28; video: 22, 21, 21).
 *   ids   device int32 [S][n_axes] (n_axes <= 3; each row t holds (t, h, w)).
 *   rope  device float [S][sum P][2].  Computed in double, stored as float.
 * Alignment: 4 bytes suffices. */
dit_status dit_rope_table(const int32_t* ids, int S, int n_axes, const int* axes_pairs,
                          double theta, float* rope, void* stream);

/* ------------------------------------------------------------------------
 * adaLN modulation vector ([CG] §1.1: the modulation that feeds (1+scale)*x+shift)
 * ------------------------------------------------------------------------ */

/* out[b][n] = sum_k W[n][k] * silu(vec[b][k]) + bias[n]  in fp32.
 *   vec   device bf16 [B][ldv], W device bf16 [N][ldw] (nn.Linear layout),
 *   bias  device bf16 [N] or NULL (= 0), out device float [B][ldo].
 * The single block uses N = 3D chunks (shift, scale, gate); the double block
 * and video block N = 6D (shift1, scale1, gate1, shift2, scale2, gate2).
 * Requires K % 8 == 0, 1 <= B <= 8, K <= 8192, B * K <= 51200.  HBM-bound on
 * the weight read. */
dit_status dit_adaln_modulation(const dit_bf16* vec, int64_t ldv, const dit_bf16* W, int64_t ldw,
                                const dit_bf16* bias, float* out, int64_t ldo,
                                int B, int N, int K, void* stream);

/* Same contraction with the input map and the output type chosen by flags:
 *   DIT_VEC_SILU_IN   apply silu to the input before the product
 *   DIT_VEC_OUT_BF16  write bf16 (round-to-nearest-even) instead of fp32 */
enum { DIT_VEC_SILU_IN = 1, DIT_VEC_OUT_BF16 = 2 };
dit_status dit_vec_linear(const dit_bf16* x, int64_t ldx, const dit_bf16* W, int64_t ldw,
                          const dit_bf16* bias, void* out, int64_t ldo,
                          int B, int N, int K, int flags, void* stream);

/* ------------------------------------------------------------------------
 * LayerNorm + adaLN modulate ([CG] §1.1)
 * ------------------------------------------------------------------------ */

/* y[r] = (1 + scale[b]) * (x[r] - mean) / sqrt(var + eps) + shift[b]
 * per row r of D elements, b = r / S (rows of batch b are contiguous), biased
 * variance, no LayerNorm affine.  shift/scale: device float, row b at
 * shift + b * mod_stride; pass shift = scale = NULL for a plain LayerNorm.
 * Mean and variance are taken in fp32 over the row shifted by its first
 * element (relative error of the variance below about D * 2^-24 for any
 * row; a row of equal values normalises to exactly 0).
 *   x, y device bf16 [B*S][ld].  y must not alias x.  D % 8 == 0, D <= 8192. */
dit_status dit_modulate_norm(const dit_bf16* x, int64_t ldx, const float* shift, const float* scale,
                             int64_t mod_stride, dit_bf16* y, int64_t ldy,
                             int B, int S, int D, float eps, void* stream);

/* ------------------------------------------------------------------------
 * QK RMSNorm + 3-axis RoPE ([CG] §3.1)
 * ------------------------------------------------------------------------ */

/* For every token t (of B*S rows) and head h, for q and for k:
 *   u = x / sqrt(mean(x^2) + eps) * s          (x = head vector of head_dim 128)
 *   (u[2p], u[2p+1]) <- (u0 cos - u1 sin, u0 sin + u1 cos), (cos, sin) = rope[t mod S][p]
 *   q, k       device bf16, head h of token r at q + r*ld_in + h*128 (same for k)
 *   q_scale, k_scale device bf16 [128] or NULL (= 1)
 *   rope       device float [S][64][2] from dit_rope_table, or NULL (no rotation)
 *   q_out, k_out device bf16 with row stride ld_out; may equal q, k (in place).
 * head_dim must be 128. */
dit_status dit_qk_norm_rope(const dit_bf16* q, const dit_bf16* k, int64_t ld_in,
                            const dit_bf16* q_scale, const dit_bf16* k_scale, const float* rope,
                            dit_bf16* q_out, dit_bf16* k_out, int64_t ld_out,
                            int B, int S, int H, int head_dim, float eps, void* stream);

/* ------------------------------------------------------------------------
 * Attention ([CG] §2 joint full attention, 24 x 128; §6.3 operands (B, S, H, D))
 * ------------------------------------------------------------------------ */

/* o[b, i, h, :] = sum_j softmax_j(scale * q[b,i,h,:] . k[b,j,h,:]) v[b,j,h,:]
 * No mask.  Token i of batch b, head h lives at q + (b*Sq + i)*ldq + h*128 (same
 * for k, v with Skv and o with Sq).  lse: NULL or device float [B][H][Sq] that
 * receives the natural-log sum-exp of the scaled logits per query.
 * head_dim must be 128; Sq, Skv >= 1 (any value: ragged tails are masked).
 * Tensor cores (tcgen05, TMEM accumulators), online softmax.  o must not
 * alias q, k or v. */
dit_status dit_attention(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v,
                         int64_t ldq, int64_t ldk, int64_t ldv, dit_bf16* o, int64_t ldo,
                         float* lse, int B, int Sq, int Skv, int H, int head_dim,
                         float softmax_scale, void* stream);

/* Attention of q against one more key set, merged into a running result
 * ([CG] §5: a ring hop adds the attention over the shard in hand to the
 * result over the shards seen so far, by log-sum-exp).  On entry o (same
 * layout as dit_attention's output) and lse (required, fp32 [B][H][Sq],
 * natural log) hold the running result over earlier keys; on return they
 * hold the result over the union:
 *   lse' = log(exp(lse) + exp(lse_cur)),
 *   o'   = exp(lse - lse') o + exp(lse_cur - lse') o_cur,
 * where (o_cur, lse_cur) is dit_attention over k, v.  A row whose running
 * lse is -inf (nothing accumulated yet) gets o_cur exactly as dit_attention
 * would write it (o is then only read, with weight 0, and must be finite).
 * One launch, no extra buffer: the merge runs in the epilogue, each thread
 * reading its row of o before writing it.  Arguments and errors as
 * dit_attention; lse == NULL is DIT_ERR_INVALID_ARG. */
dit_status dit_attention_accumulate(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v,
                                    int64_t ldq, int64_t ldk, int64_t ldv, dit_bf16* o, int64_t ldo,
                                    float* lse, int B, int Sq, int Skv, int H, int head_dim,
                                    float softmax_scale, void* stream);

/* Attention with the keys split across CTAs, for query sets too short to fill
 * the GPU (one rank of a sequence-parallel ring: [CG] §5, 576 queries per GPU
 * at CP = 8).  The key range is cut into n_split contiguous parts of whole
 * 128-key tiles (fewer when Skv has fewer tiles); one launch computes the
 * attention of every query tile over every part, each part's result (bf16)
 * and lse (fp32) going to the workspace, and the log-sum-exp merge
 * (dit_attention_merge) combines the parts into o and lse.  accumulate = 0:
 * the result is dit_attention's over k, v, with one more bf16 rounding of
 * each part; lse may be NULL.  accumulate = 1: o and lse (required) hold a
 * running result on entry, as for dit_attention_accumulate, and the merge
 * includes it.  n_split: 1..4 (1 behaves as dit_attention or
 * dit_attention_accumulate and needs no workspace).  workspace: device, 256-byte
 * aligned, at least dit_attention_split_workspace(B, Sq, H, n_split) bytes,
 * owned by the caller and reusable once the stream has passed this call.
 * Other arguments and errors as dit_attention; DIT_ERR_WORKSPACE when the
 * workspace is missing or too small.  Two launches, no synchronisation,
 * capturable. */
dit_status dit_attention_split(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v,
                               int64_t ldq, int64_t ldk, int64_t ldv, dit_bf16* o, int64_t ldo,
                               float* lse, int B, int Sq, int Skv, int H, int head_dim,
                               float softmax_scale, int n_split, int accumulate, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Bytes of workspace dit_attention_split needs (0 for invalid sizes). */
size_t dit_attention_split_workspace(int B, int Sq, int H, int n_split);

/* Merge of attention results over disjoint key sets ([CG] §5: sequence-
 * parallel ring attention merges each hop's partial result by its
 * log-sum-exp):
 *   lse[b,h,i] = log sum_j exp(lse_j[b,h,i])
 *   o[b,i,h,:] = sum_j exp(lse_j[b,h,i] - lse[b,h,i]) o_j[b,i,h,:]
 * n: 1..8 parts.  o_parts, lse_parts: host arrays of n device pointers; part
 * j is bf16 [B][Sq][ld_in] (head h at column h*128, as dit_attention writes
 * it) with its fp32 lse [B][H][Sq] from dit_attention.  o: bf16 [B][Sq][ld_out];
 * lse_out: NULL or fp32 [B][H][Sq].  o may equal any o_parts[j] and lse_out
 * any lse_parts[j] (so a ring can merge into its running result).  Weights
 * and sums in fp32; o rounded to bf16 once.  1 <= B, H <= 65535.
 * A part over an empty key set has lse = -inf and weight 0 (its o values must
 * be finite: they are multiplied by that zero weight).  A row whose every
 * part is empty gets o = 0 and lse = -inf. */
dit_status dit_attention_merge(int n, const dit_bf16* const* o_parts, const float* const* lse_parts,
                               int64_t ld_in, dit_bf16* o, float* lse_out, int64_t ld_out,
                               int B, int Sq, int H, void* stream);

/* ------------------------------------------------------------------------
 * GEMM with fused epilogue ([CG] §1.1 tail fused into the producing kernel;
 * the block's linears: QKV|MLP-in and the output projection)
 * ------------------------------------------------------------------------ */

typedef enum {
  DIT_EPI_NONE = 0,            /* C = A W^T */
  DIT_EPI_BIAS = 1,            /* C = A W^T + bias */
  DIT_EPI_BIAS_GELU_COLS = 2,  /* C = A W^T + bias; gelu_tanh on columns >= gelu_col_begin */
  DIT_EPI_BIAS_GATED_RESIDUAL = 3 /* C = resid + gate[b] * (A W^T + bias) */
} dit_epilogue;

typedef struct {
  const dit_bf16* A; int64_t lda;   /* device [M][lda], K used columns */
  const dit_bf16* W; int64_t ldw;   /* device [N][ldw] (nn.Linear weight) */
  const dit_bf16* bias;             /* device [N] or NULL (= 0) */
  dit_bf16* C; int64_t ldc;         /* output of columns [0, split_col) */
  dit_bf16* C2; int64_t ldc2;       /* output of columns [split_col, N), column n at
                                       C2 + (n - split_col); NULL = every column to C */
  int split_col;                    /* multiple of 32 when C2 != NULL */
  int M, N, K;                      /* N % 32 == 0, K % 8 == 0 */
  dit_epilogue epi;
  int gelu_col_begin;               /* multiple of 32 */
  const float* gate;                /* device fp32, row b at gate + b*gate_stride */
  int64_t gate_stride;
  const dit_bf16* resid; int64_t ldr; /* device [M][ldr]; may equal C (in place) */
  int rows_per_batch;               /* row m belongs to batch m / rows_per_batch */
  /* Optional QK RMSNorm + RoPE fused into the epilogue ([CG] §3.1), the same
   * operation as dit_qk_norm_rope applied to output columns [0, qk_cols):
   * columns [0, qk_cols/2) are q heads and [qk_cols/2, qk_cols) k heads, 128
   * columns per head.  qk_cols = 0 disables it; otherwise qk_cols % 256 == 0,
   * epi is DIT_EPI_NONE/BIAS/BIAS_GELU_COLS and those columns go to C. */
  int qk_cols;
  int qk_norm;                      /* 1: RMSNorm each head (eps qk_eps) then scale */
  float qk_eps;
  const dit_bf16* q_scale;          /* device [128] or NULL (= 1) */
  const dit_bf16* k_scale;
  const float* rope;                /* device [rope_rows][64][2] or NULL (no rotation) */
  int rope_rows;                    /* output row m uses rope row m % rope_rows */
} dit_gemm_args;

/* bf16 x bf16 -> fp32 accumulate on tcgen05 (256 x 256 tiles over SM pairs
 * when M > 128, else 128 x 256 on one SM; TMA-fed, TMEM accumulators,
 * persistent CTAs); epilogue rounds to bf16 (nearest-even). */
dit_status dit_gemm_epilogue(const dit_gemm_args* args, void* stream);

/* Two independent GEMMs with the same epilogue kind and the same K in one
 * persistent launch ([CG] §3.1: the double-stream block runs the same layer
 * on the text and the image stream with separate weights).  The tiles of b
 * follow those of a in one schedule, so a GEMM with few tiles (512 text rows)
 * fills the SMs the other leaves idle.  Each result is the one
 * dit_gemm_epilogue gives for its arguments, bit for bit.  a and b are
 * validated as for dit_gemm_epilogue; a->epi != b->epi or a->K != b->K is
 * DIT_ERR_INVALID_ARG.  With M <= 128 in either, the two run as two launches.
 * The outputs must not overlap each other or the other GEMM's inputs. */
dit_status dit_gemm_epilogue_grouped(const dit_gemm_args* a, const dit_gemm_args* b, void* stream);

/* ------------------------------------------------------------------------
 * Blocks ([CG] §2 single-stream block; §3.1 double-stream blocks; [WAN] §1.1)
 * ------------------------------------------------------------------------ */

typedef struct {
  int B;          /* batch */
  int S;          /* tokens per sample (text + image) */
  int n_txt;      /* text tokens (double block: the first n_txt tokens of the
                     joint sequence; image tokens = S - n_txt) */
  int D;          /* model dim = H * head_dim */
  int H;          /* heads */
  int head_dim;   /* 128 */
  int M;          /* MLP hidden */
  float eps;      /* LayerNorm and RMSNorm epsilon (1e-6) */
} dit_block_cfg;

typedef struct {
  const dit_bf16 *W_mod, *b_mod;     /* [3D][D], [3D]   (shift, scale, gate) */
  const dit_bf16 *W1, *b1;           /* [3D+M][D], [3D+M]  rows: q | k | v | mlp */
  const dit_bf16 *q_scale, *k_scale; /* [head_dim] */
  const dit_bf16 *W2, *b2;           /* [D][D+M], [D]   input: attn | gelu(mlp) */
} dit_single_weights;

typedef struct {
  const dit_bf16 *W_mod, *b_mod;     /* [6D][D] (shift1, scale1, gate1, shift2, scale2, gate2) */
  const dit_bf16 *W_qkv, *b_qkv;     /* [3D][D] */
  const dit_bf16 *q_scale, *k_scale; /* [head_dim] */
  const dit_bf16 *W_proj, *b_proj;   /* [D][D] */
  const dit_bf16 *W_mlp1, *b_mlp1;   /* [M][D] */
  const dit_bf16 *W_mlp2, *b_mlp2;   /* [D][M] */
} dit_stream_weights;

typedef struct {
  dit_stream_weights txt, img;
} dit_double_weights;

typedef struct {
  const dit_bf16 *W_mod, *b_mod;     /* [6D][D] */
  const dit_bf16 *W_qkv, *b_qkv;     /* [3D][D] self-attention q | k | v */
  const dit_bf16 *W_o, *b_o;         /* [D][D] */
  const dit_bf16 *W_cq, *b_cq;       /* [D][D] cross-attention query */
  const dit_bf16 *W_ckv, *b_ckv;     /* [2D][D] cross-attention key | value (from ctx) */
  const dit_bf16 *W_co, *b_co;       /* [D][D] */
  const dit_bf16 *W_f1, *b_f1;       /* [M][D] */
  const dit_bf16 *W_f2, *b_f2;       /* [D][M] */
} dit_video_weights;

/* Workspace sizes in bytes (256-byte aligned pointer required). */
size_t dit_single_block_workspace(const dit_block_cfg* cfg);
size_t dit_double_block_workspace(const dit_block_cfg* cfg);
size_t dit_video_block_workspace(const dit_block_cfg* cfg, int n_ctx);

/* Flux single-stream block:
 *   (shift, scale, gate) = W_mod silu(vec) + b_mod
 *   h = ((1+scale) LN(x) + shift) W1^T + b1 = [q | k | v | mlp]
 *   o = attention(rope(rms(q)), rope(rms(k)), v); a = gelu_tanh(mlp)
 *   out = x + gate * ([o | a] W2^T + b2)
 * x, out: device bf16 [B*S][D] (out may equal x); vec: device bf16 [B][D];
 * rope: device float [S][64][2] from dit_rope_table.  Five kernels: the QK
 * RMSNorm + RoPE runs inside the GEMM1 epilogue. */
dit_status dit_single_block_fwd(const dit_block_cfg* cfg, const dit_single_weights* w,
                                const dit_bf16* x, const dit_bf16* vec, const float* rope,
                                dit_bf16* out, void* ws, size_t ws_bytes, void* stream);

/* Same call that additionally records events[i] (cudaEvent_t, may not be NULL)
 * on the stream before kernel i and events[5] after the last of its five
 * kernels (adaLN, LN-modulate, GEMM1 with fused QK-norm+RoPE, attention,
 * GEMM2), so a caller can time every kernel.  n_events must be >= 6.  Its
 * kernels start only when the previous one has finished (the plain call lets
 * each kernel's prologue overlap the end of the one before). */
dit_status dit_single_block_fwd_profiled(const dit_block_cfg* cfg, const dit_single_weights* w,
                                         const dit_bf16* x, const dit_bf16* vec, const float* rope,
                                         dit_bf16* out, void* ws, size_t ws_bytes,
                                         void* const* events, int n_events, void* stream);

/* Allocation-free variant of dit_single_block_fwd.  (The pages have no
 * counterpart to this call; it exists for deployment.)  For callers that may
 * not allocate device memory: plug-ins whose host framework owns all device
 * memory through its own pool, and serving loops that must not call
 * cudaMalloc/cudaFree once running (those calls can synchronise the device).
 * Same inputs and outputs as dit_single_block_fwd, but the intermediates live
 * in a 16 MiB array inside the library that each device keeps until exit.
 *   - A configuration that dit_single_block_fwd rejects gets the same status
 *     here.  Valid configurations whose workspace (dit_single_block_workspace)
 *     exceeds 16 MiB are rejected with DIT_ERR_WORKSPACE (e.g. S=256, D=384
 *     fits; S=4608, D=3072 does not).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call
 *     before capturing any stream into a graph.
 *   - All calls share the one array: calls that may overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the caller.
 *     Nothing in the array needs clearing between calls.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
dit_status dit_single_block_fwd_noalloc(const dit_block_cfg* cfg, const dit_single_weights* w,
                                        const dit_bf16* x, const dit_bf16* vec, const float* rope,
                                        dit_bf16* out, void* stream);

/* Host-buffer pipeline of independent single-stream block forwards, e.g. a
 * server's queue of requests.  (The pages have no counterpart to this call;
 * the block itself is the one of dit_single_block_fwd, five kernels.)
 *   Request i reads x_host[i] (bf16 [B*S][D]) and vec_host[i] (bf16 [B][D])
 *   from host memory and writes out_host[i] (bf16 [B*S][D]) back to host
 *   memory; out_host[i] may equal x_host[i].
 *   Request i+1's host-to-device copy and request i-1's device-to-host copy
 *   run on two streams internal to the library while request i computes on
 *   `stream`.  The device staging is double-buffered inside the workspace and
 *   ordered by events.  One cudaMemcpyAsync per copy.
 *   Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for
 *   the copies to overlap the compute; pageable buffers give the same results.
 *   The call returns once everything is enqueued.  `stream` waits for the
 *   last copy, so the outputs are in host memory once `stream` completes.
 *   The internal streams and events are created on a device's first call and
 *   kept; enqueues from several host threads are serialised inside the call.
 *   Calls that share a workspace must not overlap.  Not for stream capture.
 * rope: device float [S][64][2].  ws: device, 256-byte aligned, at least
 * dit_single_block_host_workspace(cfg) bytes.  n >= 1; every pointer non-NULL. */
size_t dit_single_block_host_workspace(const dit_block_cfg* cfg);
dit_status dit_single_block_fwd_host(const dit_block_cfg* cfg, const dit_single_weights* w, int n,
                                     const dit_bf16* const* x_host, const dit_bf16* const* vec_host,
                                     dit_bf16* const* out_host, const float* rope, void* ws,
                                     size_t ws_bytes, void* stream);

/* Flux double-stream block: per stream s in (txt, img) its own adaLN (6
 * chunks), LN-modulate, QKV, QK RMSNorm; RoPE + joint attention over the
 * sequence txt | img (rope rows in that order); then
 *   x_s += gate1 (o_s W_proj^T + b_proj);  x_s += gate2 MLP((1+scale2) LN(x_s) + shift2)
 * img: [B][S-n_txt][D], txt: [B][n_txt][D] device bf16; outputs may equal
 * the inputs. */
dit_status dit_double_block_fwd(const dit_block_cfg* cfg, const dit_double_weights* w,
                                const dit_bf16* img, const dit_bf16* txt, const dit_bf16* vec,
                                const float* rope, dit_bf16* img_out, dit_bf16* txt_out,
                                void* ws, size_t ws_bytes, void* stream);

/* Wan-style video block ([WAN] §1.1):
 *   x += gate1 * SelfAttn(RoPE q, RoPE k, v) W_o^T       on (1+scale1) LN(x) + shift1
 *   x += CrossAttn(LN(x) W_cq^T, ctx W_ckv^T) W_co^T      (no RoPE, no gate)
 *   x += gate2 * W_f2 gelu(W_f1 ((1+scale2) LN(x) + shift2))
 * x, out: device bf16 [B*S][D]; ctx: device bf16 [B*n_ctx][D]; no QK norm. */
dit_status dit_video_block_fwd(const dit_block_cfg* cfg, const dit_video_weights* w,
                               const dit_bf16* x, const dit_bf16* ctx, int n_ctx,
                               const dit_bf16* vec, const float* rope, dit_bf16* out,
                               void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Whole denoising loop in one CUDA graph ([CG] §1.2, §4, §7: capture once with
 * static buffers and replay; flowmatch-euler steps)
 * ------------------------------------------------------------------------ */

typedef struct {
  int D, H, head_dim, M;             /* block dims */
  int channels;                      /* latent channels (16); patch 2x2 */
  int txt_dim;                       /* raw text feature dim (4096) */
  int t_dim;                         /* timestep embedding dim (256) */
  int n_double, n_single;
  const dit_double_weights* double_blocks;   /* host array [n_double] */
  const dit_single_weights* single_blocks;   /* host array [n_single] */
  const dit_bf16 *W_img_in, *b_img_in;       /* [D][4*channels] */
  const dit_bf16 *W_txt_in, *b_txt_in;       /* [D][txt_dim] */
  const dit_bf16 *W_t1, *b_t1;               /* [D][t_dim] */
  const dit_bf16 *W_t2, *b_t2;               /* [D][D] */
  const dit_bf16 *W_fmod, *b_fmod;           /* [2D][D] final (shift, scale) */
  const dit_bf16 *W_out, *b_out;             /* [4*channels][D] */
  float eps;
} dit_model;

typedef struct {
  int n_txt, grid_h, grid_w;         /* text tokens; image grid (latent / 2) */
  int steps;                         /* Euler steps over t_i = 1 - i/steps */
  const dit_bf16* latent_in;         /* device bf16 [channels][2 grid_h][2 grid_w] */
  const dit_bf16* txt;               /* device bf16 [n_txt][txt_dim] */
  const int32_t* ids;                /* device int32 [n_txt + grid_h grid_w][3] */
  float* latent_out;                 /* device float [channels][2 grid_h][2 grid_w] */
  /* Model-level step cache ([CG] §7: the loop decides per step whether to
   * run the forward; skipped steps predict the velocity from history by a
   * finite difference along t).  fresh: host array [steps], 1 = run the
   * model at step i, 0 = predict; NULL = every step fresh.  Step 0 must be
   * fresh.  cache_order 0 reuses the last model velocity; 1 extrapolates
   * linearly from the last two, v(t) = v_a + (t - t_a)(v_a - v_b)/(t_a - t_b)
   * (the last one alone until two exist).  Read at graph creation. */
  const uint8_t* fresh;
  int cache_order;
  /* Classifier-free guidance ([SDXL] §3.3: v = v_u + g (v_c - v_u), read for
   * the flow-matching velocity).  txt_uncond: NULL = no guidance; otherwise a
   * device bf16 [n_txt][txt_dim] unconditional text.  A guided step runs the
   * model once with txt and once with txt_uncond (same timestep embedding and
   * modulation) and combines the two velocities in fp32.  cfg_steps: guidance
   * on steps < cfg_steps only (the guide's late-step cut-off); < 0 = every
   * step.  Cached steps predict from the guided velocities. */
  const dit_bf16* txt_uncond;
  float guidance;
  int cfg_steps;
} dit_loop_io;

/* Size in bytes of each struct of this header as the library was compiled,
 * for a binding to check its own layout: which = 0 dit_gemm_args,
 * 1 dit_block_cfg, 2 dit_single_weights, 3 dit_stream_weights,
 * 4 dit_double_weights, 5 dit_video_weights, 6 dit_model, 7 dit_loop_io;
 * 0 for any other value.  Host only: needs no GPU. */
size_t dit_abi_struct_size(int which);

/* Host-side plan of the model-level step cache for `steps` Euler steps (the
 * bookkeeping dit_forward_* follows, exposed so a caller can inspect it and so
 * it can be checked without a GPU).  Per step i, arrays of length steps:
 *   keep_slot[i] >= 0: the model runs and its velocity is kept in history
 *     slot keep_slot[i] (0 or 1); -1 on a predicted step, and on every step
 *     when fresh == NULL (no cache).
 *   on a predicted step (fresh[i] == 0) the velocity is
 *     ca[i] * v[slot_a[i]] + cb[i] * v[slot_b[i]]  (slot_b[i] = -1: one term);
 *     ca, cb follow v = v_a + (t_i - t_a)(v_a - v_b)/(t_a - t_b) for order 1
 *     with the two newest fresh steps a, b, and v = v_a otherwise.
 *     slot_a, slot_b, ca, cb are -1, -1, 0, 0 on steps that run the model.
 * Same validation as dit_forward_*: fresh[0] must be 1, cache_order 0 or 1.
 * Host only: needs no GPU. */
dit_status dit_step_cache_plan(int steps, const uint8_t* fresh, int cache_order, int* keep_slot, int* slot_a,
                               int* slot_b, float* ca, float* cb);

typedef struct dit_graph dit_graph;

size_t dit_forward_workspace(const dit_model* m, const dit_loop_io* io);

/* Runs the loop eagerly (kernel by kernel) on stream. */
dit_status dit_forward_eager(const dit_model* m, const dit_loop_io* io, void* ws, size_t ws_bytes,
                             void* stream);

/* Captures the same kernel sequence into one CUDA graph (on a private
 * stream) and instantiates it.  All pointers are baked in: refill io's input
 * buffers in place between launches.  *out receives the handle. */
dit_status dit_forward_graph_create(const dit_model* m, const dit_loop_io* io, void* ws,
                                    size_t ws_bytes, dit_graph** out);
dit_status dit_forward_graph_launch(dit_graph* g, void* stream);
/* Number of kernel nodes in the graph (*n). */
dit_status dit_forward_graph_nodes(const dit_graph* g, size_t* n);
dit_status dit_forward_graph_destroy(dit_graph* g);

#if defined(DIT_BUILD) && defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* DIT_H_ */
