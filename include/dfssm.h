/*
 * dfssm.h -- C ABI of libdfssm.so, the B200 (sm_100a) DF-SSM decode step.
 *
 * Method: "Density Field State Space Models" (C. Shinde).  Every projection of a
 * Mamba-2 layer is a frozen 1-bit sign scaffold plus an int8 low-rank correction
 * (Section 3.2, Eq. 3; int8 per-channel scales, Section 3.3; 1-bit packed
 * storage, Table 1).  The scaffold feeds the causal depthwise conv1d step (a
 * stateful shift register) and the selective-SSM recurrence over preallocated
 * persistent state (Section 4.1), with the corrected Mamba-2 forms of Appendix B
 * (Table 12): h = A h + (x * dt) (outer) B, and gate before norm,
 * norm(y * silu(z)).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller (the library
 *     never allocates, frees, creates streams or synchronises).  `stream` is a
 *     cudaStream_t passed as void*; all work is enqueued on it, so every call
 *     may be captured into a CUDA graph.
 *   - fp16 values travel as uint16_t bit patterns (IEEE binary16).
 *   - Return value: 0 on success, a negative DFSSM_ERR_* code otherwise; argument
 *     errors are detected on the host before anything is enqueued.  The message
 *     of the calling thread's last failure is available from dfssm_last_error().
 *   - Alignment: every pointer must be 16-byte aligned (DFSSM_ERR_MISALIGNED).
 */
#ifndef DFSSM_H
#define DFSSM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DFSSM_API __attribute__((visibility("default")))
#else
#define DFSSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DFSSM_OK = 0,
  DFSSM_ERR_INVALID_ARG = -1,        /* null pointer, non-positive size, bad enum */
  DFSSM_ERR_UNSUPPORTED_SHAPE = -2,  /* e.g. cols % 256 != 0, d_inner != nheads*headdim, ngroups != 1 */
  DFSSM_ERR_MISALIGNED = -3,         /* a pointer is not 16-byte aligned */
  DFSSM_ERR_WORKSPACE_TOO_SMALL = -4,
  DFSSM_ERR_CUDA = -5,               /* a CUDA runtime call or launch failed */
  DFSSM_ERR_DEVICE = -6,             /* no usable sm_100 device */
  DFSSM_ERR_NOT_BUILT = -7           /* a facility this build of the library leaves out */
};

enum { DFSSM_DTYPE_F16 = 0, DFSSM_DTYPE_F32 = 1 };

/* Sign-word layouts.  ROWMAJOR: uint32 [rows][cols/32], bit j of word k holds
 * column 32k+j, bit = 1 encodes +1 and bit = 0 encodes -1.  TILED: the same bits
 * permuted into 16-row x 256-column tiles of 128 words (rows padded up to a
 * multiple of 16 with clear bits).  For weight (row, col) with r16 = row % 16,
 * c = col % 256, m = c / 64, p = c % 64, t = p / 16, e = (p % 16) / 8,
 * h = (p % 8) / 4, i = p % 4:
 *   lane = (r16 % 8) * 4 + t,  q = r16 / 8 + 2 * h,  s = 2 * m + e,
 *   bit = s + 8 * i,
 *   word = ((row / 16) * (cols / 256) + col / 256) * 128 + lane * 4 + q.
 * Each warp lane reads one 16-byte vector (words q = 0..3) per tile; for each of
 * the tile's eight 32-column m16n8k32 tensor-core products s, (word_q >> s) &
 * 0x01010101 is the lane's int8 A-fragment register q with bytes 0/1 for -1/+1
 * (fragment column 4t+i, +16 for q >= 2, is tile column 64m + 16t + 8e + i, +4).
 * Products 2m and 2m+1 together cover tile columns 64m .. 64m+63, lane t's
 * B-fragment bytes of both being the 16 consecutive columns 64m + 16t ...  The
 * projection kernels consume TILED words only. */
enum { DFSSM_LAYOUT_ROWMAJOR = 0, DFSSM_LAYOUT_TILED = 1 };

/* Shape of one layer.  in_proj: d_model -> 2*d_inner + 2*ngroups*d_state + nheads
 * ([z | x | B | C | dt]); conv over the conv_dim = d_inner + 2*ngroups*d_state
 * channels [x | B | C]; out_proj: d_inner -> d_model.  Supported: ngroups == 1,
 * d_conv == 4, d_inner == nheads*headdim, d_model and d_inner multiples of 256,
 * headdim a multiple of 16 (<= 128), d_state a multiple of 4 (<= 256),
 * 0 <= rank <= 128 and a multiple of 4. */
typedef struct dfssm_dims {
  int32_t batch, d_model, d_inner, nheads, headdim, d_state, ngroups, d_conv, rank;
  /* SSM state storage: 0 fp32; 1 fp16 (each step's fp64 update rounded once to
   * fp16; halves the state stream).  fp16 state runs the multi-launch path at
   * every batch size: the batch-1 token kernel holds fp32 state. */
  int32_t ssm_state_dtype;
  /* Prompt pass only: 1 passes the SSM state carried from each 64-token chunk of the
   * scan to the next through the density-field codec (DF-SSD; "Density Field State
   * Space Models", Section 3.4 and Appendix D; see dfssm_df_encode); 0 (the default)
   * carries it exactly.  The state after the last chunk is stored as computed.
   * Decode steps ignore it. */
  int32_t df_chunk_codec;
} dfssm_dims;

/* One DF-SSM projection (Eq. 3 with a per-row scaffold scale):
 *   y[o] = alpha[o] * sum_k s[o,k] x[k] + sB[o] * sum_j B[o,j] u[j],
 *   u[j] = acc[j] * sA[j] * sx,  acc[j] = sum_k A[j,k] xq[k]  (int8 x int8 -> int32),
 *   xq = clamp(rint(x / sx), -127, 127), sx = max|x| / 127 (fp32; sx = 1, xq = 0 for x == 0).
 * bits : TILED sign words, dfssm_packed_words(rows, cols, DFSSM_LAYOUT_TILED) words
 * alpha: fp16 [rows]            A : int8 [rank][cols]      sA: fp16 [rank]
 * B    : int8 [rows][rank]      sB: fp16 [rows]
 * A, sA, B, sB may be NULL only when the rank in use is 0. */
typedef struct dfssm_proj {
  int32_t rows, cols;
  const uint32_t* bits;
  const uint16_t* alpha;
  const int8_t* A;
  const uint16_t* sA;
  const int8_t* B;
  const uint16_t* sB;
} dfssm_proj;

/* Weights of one layer.  prenorm_w fp16 [d_model]; conv_w fp16 [conv_dim][d_conv]
 * (tap d_conv-1 multiplies the newest input); conv_b fp16 [conv_dim]; dt_bias,
 * A_log, D fp32 [nheads]; gnorm_w fp16 [d_inner]. */
typedef struct dfssm_layer_weights {
  const uint16_t* prenorm_w;
  dfssm_proj in;
  const uint16_t* conv_w;
  const uint16_t* conv_b;
  const float* dt_bias;
  const float* A_log;
  const float* D;
  const uint16_t* gnorm_w;
  dfssm_proj out;
} dfssm_layer_weights;

/* Persistent per-layer state, updated in place each step (caller-owned).
 * conv_state fp32 [batch][d_conv-1][conv_dim], index 0 the oldest input;
 * ssm_state [batch][nheads][headdim][d_state], fp32 or fp16 per dims->ssm_state_dtype. */
typedef struct dfssm_layer_state {
  float* conv_state;
  void* ssm_state;
} dfssm_layer_state;

/* Byte offsets of the intermediates a step leaves in its workspace (valid after
 * the stream has reached the end of the call).  For dfssm_model_decode they hold
 * the LAST layer's values.  ~0 marks a region the call does not have.
 * Digit planes: an fp16 activation x is the integer X = x * 2^24 (|X| < 2^40),
 * written as 6 balanced base-256 digits D_d in [-128, 127] with X = sum D_d 256^d;
 * the scaffold product is computed exactly from these planes. */
typedef struct dfssm_ws_layout {
  size_t total_bytes;
  size_t status;     /* uint32 status word, 0 = ok.  Value 1: the batch-1 token kernel found
                        the abort flag of an earlier failed call set and did nothing (zero
                        the workspace).  Value 2: a token id was out of range
                        (clamped).  Values 4 .. 16384: a bounded wait of the batch-1 token
                        kernel gave up (each wait has its own value) and the call's outputs
                        are invalid.  Value 32768: a streamed SSM-state copy did not land
                        in time (multi-launch path); outputs invalid.  Bits are or-ed in and
                        never cleared by the library. */
  size_t x_in;       /* fp16  [batch][d_model]    pre-norm output (in_proj activation) */
  size_t xq_in;      /* int8  [batch][d_model]    its int8 LoRA codes */
  size_t sx_in;      /* fp32  [batch]             their scales */
  size_t acc_in;     /* int32 [batch][rank]       in_proj A.xq partials */
  size_t u_in;       /* fp64  [batch][rank]       acc * sA * sx */
  size_t xd_in;      /* int8  [batch][6][d_model] digit planes of x_in */
  size_t xdsum_in;   /* int32 [batch][6]          digit-plane sums */
  size_t zxbcdt;     /* fp64  [batch][in_rows]    in_proj output [z|x|B|C|dt] */
  size_t xc;         /* fp64  [batch][conv_dim]   conv output after SiLU */
  size_t g;          /* fp32  [batch][d_inner]    y * silu(z) */
  size_t x_out;      /* fp16  [batch][d_inner]    gated-norm output (out_proj activation) */
  size_t xq_out;     /* int8  [batch][d_inner] */
  size_t sx_out;     /* fp32  [batch] */
  size_t acc_out;    /* int32 [batch][rank] */
  size_t u_out;      /* fp64  [batch][rank] */
  size_t xd_out;     /* int8  [batch][6][d_inner] */
  size_t xdsum_out;  /* int32 [batch][6] */
  size_t res;        /* fp32  [batch][d_model]    residual stream (model decode only) */
  size_t scratch;    /* internal */
  size_t control;    /* uint32 [4] control words of the batch-1 token kernel: [0] launch epoch,
                        [1] abort flag (both zero in a fresh workspace, kept by the library);
                        [2], [3] test hooks, zero in normal use: [2] = c + 1 makes CTA c
                        withhold its layer-0 residual words and [3] = n bounds every wait at
                        n polls, so that a test can make a bounded wait run out without any
                        GPU fault (the call then returns with a status value in 4 .. 16384). */
} dfssm_ws_layout;

/* ---- weight packing (not on the timed path) ------------------------------ */

/* Number of uint32 words of a packed [rows x cols] sign matrix in `layout`. */
DFSSM_API size_t dfssm_packed_words(int rows, int cols, int layout);

/* Pack a dense row-major matrix w ([rows][cols], fp16 or fp32 per `dtype`) into
 * sign words: bit = 1 where w >= 0 (so -0.0 packs to +1), 0 otherwise (NaN too).
 * cols % 32 == 0 (ROWMAJOR) or cols % 256 == 0 (TILED).  `bits` receives
 * dfssm_packed_words(rows, cols, layout) words.  Table 1 ("1-bit packed"). */
DFSSM_API int dfssm_pack_weights(const void* w, int dtype, int rows, int cols, int layout,
                       uint32_t* bits, void* stream);

/* Permute ROWMAJOR sign words into the TILED layout (exact bit permutation). */
DFSSM_API int dfssm_repack_bits(const uint32_t* rowmajor, int rows, int cols, uint32_t* tiled,
                      void* stream);

/* ---- one projection (Eq. 3) --------------------------------------------- */

DFSSM_API size_t dfssm_proj_workspace_bytes(int rows, int cols, int rank, int batch);

/* Eq. 3 (Section 3.2), one scaffold + int8 LoRA projection, Section 4.1's "bits
 * expanded on the fly" done in registers (the packed words are never expanded in
 * memory).
 * y [batch][rows] fp32 = projection of x [batch][cols] fp16 (finite values).  The
 * scaffold sum is exact (integer arithmetic on the activation's digit planes), the
 * LoRA stage 2 and scaling are fp64, y is rounded once to fp32.  The workspace
 * receives xq_in, sx_in, acc_in, u_in, xd_in and xdsum_in (see dfssm_ws_layout)
 * at the offsets dfssm_proj_workspace_layout reports. */
DFSSM_API int dfssm_proj_forward(const dfssm_proj* p, int rank, int batch, const uint16_t* x, float* y,
                       void* ws, size_t ws_bytes, void* stream);
/* Same projection as dfssm_proj_forward, for callers that cannot call cudaMalloc
 * (no allocator is available to them, or they must not risk the device-wide
 * synchronisation an allocation can cause).  The paper has no counterpart; this
 * is a convenience of this library.  The scratch is a fixed 4 MiB array inside
 * the library that every GPU which loads the library holds until exit; a call
 * whose dfssm_proj_workspace_bytes exceeds 4 MiB returns
 * DFSSM_ERR_WORKSPACE_TOO_SMALL without enqueueing anything.  The first call on
 * a device looks up that device's address of the array, so make it before any
 * stream capture.  That address is kept for the life of the process: after a
 * cudaDeviceReset (or any other reset of the device's primary context) do not call
 * this entry point on that device again.  All calls on a device share the one array, which keeps the
 * last call's contents: calls whose kernels may overlap on the GPU (different
 * streams without ordering) race on it.  Nothing in it needs to start at zero. */
DFSSM_API int dfssm_proj_forward_noalloc(const dfssm_proj* p, int rank, int batch, const uint16_t* x,
                                         float* y, void* stream);

DFSSM_API int dfssm_proj_workspace_layout(int rows, int cols, int rank, int batch, dfssm_ws_layout* out);

/* ---- decode step -------------------------------------------------------- */

/* Workspace for dfssm_layer_step (n_layer == 0, vocab == 0) or for
 * dfssm_model_decode (n_layer >= 1, vocab >= 1).  Section 4.1 preallocates all
 * decode buffers once so that the token step can be a graph replay; this is that
 * preallocation, owned by the caller.  The workspace must be zero-filled once
 * before its first use; the library leaves its control words consistent after
 * every call whose status word (dfssm_ws_layout.status) stays 0.  After a call that
 * left a nonzero status in values 4 .. 16384 (a bounded wait gave up), every later
 * call on the same workspace returns at once with status value 1 or-ed in, until
 * the caller zero-fills the workspace again. */
DFSSM_API size_t dfssm_workspace_bytes(const dfssm_dims* d, int n_layer, int vocab);
DFSSM_API int dfssm_workspace_layout(const dfssm_dims* d, int n_layer, int vocab, dfssm_ws_layout* out);

/* One decode token through one layer, residual add included ("Density Field State
 * Space Models", Section 4.1: the decode step runs the conv1d step as a stateful
 * shift register and the SSM step as a stateful recurrence over preallocated
 * persistent state, the whole step replayed as a CUDA graph; Appendix B, Table 12:
 * h = A h + (x * dt) (outer) B and the gate before the norm, norm(y * silu(z));
 * Section 3.2, Eq. 3 and Table 1 for the two projections):
 *   x = fp16(rmsnorm(residual) * prenorm_w); [z|xBC|dt] = in_proj(x);
 *   xc = silu(conv1d_step(xBC)); SSM update of ssm_state; g = y * silu(z);
 *   xo = fp16(rmsnorm(g) * gnorm_w); residual += out_proj(xo).
 * residual fp32 [batch][d_model] in/out; state updated in place.  RMSNorm eps 1e-5. */
DFSSM_API int dfssm_layer_step(const dfssm_dims* d, const dfssm_layer_weights* w, const dfssm_layer_state* s,
                     float* residual, void* ws, size_t ws_bytes, void* stream);

/* One greedy decode token for all batch rows through the whole model ("Density
 * Field State Space Models", Section 4.1: the batch-1 decode path, one graph per
 * token; Section 4.3 and Table 2: batch-1 and batched decode throughput; Section 3.3
 * and Table 1: tied embedding / LM head; Appendix B, Table 12 for each layer):
 *   residual = embed[tok_in]; n_layer layer steps; xf = rmsnorm(residual) * normf_w;
 *   logits = embed . xf (tied LM head, fp32 accumulation); tok_out = argmax
 *   (lowest token id wins ties).
 * embed fp16 [vocab][d_model]; layers/states HOST arrays of n_layer entries, read at
 * call time (under stream capture their pointers are baked into the graph);
 * tok_in/tok_out int32 [batch] device (may alias); logits fp32 [batch][vocab] or NULL.
 * n_layer <= 64. */
DFSSM_API int dfssm_model_decode(const dfssm_dims* d, int n_layer, int vocab, const uint16_t* embed,
                       const dfssm_layer_weights* layers, const dfssm_layer_state* states,
                       const uint16_t* normf_w, const int32_t* tok_in, int32_t* tok_out,
                       float* logits, void* ws, size_t ws_bytes, void* stream);

/* dfssm_model_decode with the int8 per-row embedding / tied LM head ("Density Field
 * State Space Models", Section 3.3: the embedding is quantised to int8 per row;
 * Table 1: embedding + LM head int8).  embed_q int8 [vocab][d_model] and embed_scale
 * fp32 [vocab] (device, 16-byte aligned; from dfssm_quantize_rows_int8 or any
 * per-row quantiser).  The gathered row is embed_scale[t] * embed_q[t] (an fp32
 * product); logit v = embed_scale[v] * (embed_q[v] . xf), fp32 accumulation.
 * Everything else as dfssm_model_decode, same workspace. */
DFSSM_API int dfssm_model_decode_q8(const dfssm_dims* d, int n_layer, int vocab, const int8_t* embed_q,
                                    const float* embed_scale, const dfssm_layer_weights* layers,
                                    const dfssm_layer_state* states, const uint16_t* normf_w,
                                    const int32_t* tok_in, int32_t* tok_out, float* logits, void* ws,
                                    size_t ws_bytes, void* stream);

/* Per-row int8 quantisation of a dense fp16 matrix w [rows][cols] (device):
 * scale[r] = max_k |w[r][k]| / 127 (an fp32 divide; 1 for an all-zero row) and
 * q[r][k] = round-half-even(w[r][k] / scale[r]) clamped to [-127, 127], the
 * decision taken in fp32.  q int8 [rows][cols], scale fp32 [rows], caller-owned,
 * 16-byte aligned.  Not on the timed path (done once when a model is loaded). */
DFSSM_API int dfssm_quantize_rows_int8(const uint16_t* w, int rows, int cols, int8_t* q, float* scale,
                                       void* stream);

/* ---- prompt pass (prefill) ---------------------------------------------- */

/* The step before decode: a prompt of T tokens per batch row goes through a layer
 * (or the model) in one pass ("Density Field State Space Models", Section 2: the
 * chunked state space duality (SSD) form of the Mamba-2 scan; Appendix B: chunks of
 * block_len 64).  Every token row gets the same per-token arithmetic as the decode
 * step (pre-norm, both projections with their exact scaffold, LoRA, gate, gated
 * norm); the conv runs along the sequence from the stored conv state, and the SSM
 * runs as the chunked scan from the stored SSM state, carried in fp64 through the
 * prompt and stored once at the end.  On return the states are those after the
 * last prompt token, ready for dfssm_model_decode.  Limits: T >= 1, batch * T <=
 * 65535, headdim * d_state <= 8192 (the scan keeps a head's state in shared memory).
 *
 * Workspace: dfssm_prefill_workspace_bytes(d, T, 0, 0) for a layer,
 * (d, T, n_layer, vocab) for the model; no zero-fill needed.  Its layout (the
 * dfssm_ws_layout regions for batch * T token rows, token-major: row b * T + t)
 * holds the last layer's intermediates of every prompt token. */
DFSSM_API size_t dfssm_prefill_workspace_bytes(const dfssm_dims* d, int T, int n_layer, int vocab);
DFSSM_API int dfssm_prefill_workspace_layout(const dfssm_dims* d, int T, int n_layer, int vocab,
                                             dfssm_ws_layout* out);

/* One layer over the prompt: residual fp32 [batch][T][d_model] in/out (every token's
 * residual after the layer), state updated in place. */
DFSSM_API int dfssm_layer_prefill(const dfssm_dims* d, int T, const dfssm_layer_weights* w,
                                  const dfssm_layer_state* s, float* residual, void* ws, size_t ws_bytes,
                                  void* stream);

/* The model over the prompt: tokens int32 [batch][T] (device); every layer's state
 * updated in place; logits fp32 [batch][vocab] (or NULL) and tok_out int32 [batch]
 * (greedy, lowest id on ties) of the LAST prompt token, so that tok_out is the first
 * decode input.  fp16 tied embedding / LM head. */
DFSSM_API int dfssm_model_prefill(const dfssm_dims* d, int n_layer, int vocab, const uint16_t* embed,
                                  const dfssm_layer_weights* layers, const dfssm_layer_state* states,
                                  const uint16_t* normf_w, int T, const int32_t* tokens, int32_t* tok_out,
                                  float* logits, void* ws, size_t ws_bytes, void* stream);

/* Number of kernel launches one dfssm_model_decode call enqueues for these
 * arguments (0 if they are invalid). */
DFSSM_API int dfssm_model_decode_launches(const dfssm_dims* d, int n_layer, int vocab);

/* Per-phase cycle counters of the batch-1 token kernel (a measurement facility,
 * not part of the method; the paper reports a per-layer time breakdown in Table 13
 * and this is the same kind of breakdown for the fused kernel).  Only a library
 * built with -DDFSSM_PHASE_TIMERS records them; the default build returns
 * DFSSM_ERR_NOT_BUILT.  Entry [cta * 32 + slot] is the sum over the calls since the
 * last reset of the clock64 cycles thread 0 of that CTA spent in phase `slot`
 * (slots 0..18 in the kernel's phase order; slot 31 counts calls).  Copies
 * min(max_entries, 256 * 32) entries to the host buffer `out` (synchronous), then
 * zeroes the counters if `reset` is nonzero.  Returns the number of entries copied. */
DFSSM_API int dfssm_phase_timers(uint64_t* out, int max_entries, int reset);

/* Message describing the calling thread's last nonzero return ("" if none). */
DFSSM_API const char* dfssm_last_error(void);

/* ABI version (major * 100 + minor). */
DFSSM_API int dfssm_version(void);

/* ---- density-field state codec ("Density Field State Space Models", Section 3.4;
 * Appendix D: K = 23 at d_state 128) ----------------------------------------------
 * A state row of n = d_state values is held as a K x K binary field, K the least
 * integer with K^2 >= 4 n: four cells per value (raster order; spare cells 0).  The
 * row's mean mu and population standard deviation sigma (fp64, summed left to right)
 * give lo = mu - 3 sigma and span = 6 sigma, kept as fp32; value i's 8-bit code is
 * q = rint(255 clip((h - lo) / span, 0, 1)) (128 if span == 0); a first-order
 * sigma-delta with a signed 8-bit error e (0 at the row's first cell, carried along
 * the row) sets cell = [e + q >= 128], e <- e + q - 255 cell; the readout is
 * lo + span * (ones among the value's four cells) / 4, rounded to fp32.
 *
 * dfssm_df_field_words: 32-bit words of one row's field (cell c is bit c % 32 of word
 * c / 32), or a negative code for d_state < 1. */
DFSSM_API int dfssm_df_field_words(int d_state);

/* rows: fp32 [n_rows][d_state] (device).  cells: [n_rows][dfssm_df_field_words]
 * words; lo, span: fp32 [n_rows] (device, written).  rows_out: fp32 [n_rows][d_state]
 * readout (may be NULL, may equal rows).  Enqueued on `stream`; 16-byte alignment is
 * not required.  Errors: DFSSM_ERR_INVALID_ARG (null pointer, n_rows < 0,
 * d_state < 1), DFSSM_ERR_CUDA. */
DFSSM_API int dfssm_df_encode(const float* rows, int n_rows, int d_state, uint32_t* cells, float* lo,
                              float* span, float* rows_out, void* stream);

/* Readout of fields written by dfssm_df_encode into rows: fp32 [n_rows][d_state]. */
DFSSM_API int dfssm_df_decode(const uint32_t* cells, const float* lo, const float* span, int n_rows,
                              int d_state, float* rows, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DFSSM_H */
