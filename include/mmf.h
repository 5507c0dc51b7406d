/*
 * mmf.h — C ABI of the B200 (sm_100a) FusedBitLinear library (libmmf.so).
 *
 * FusedBitLinear is the projection used for every i/f/g/o and gate/down projection of the
 * HGRNBit (MatMul-free) language model.  Sources (page title, section):
 *   [P1] "matmulfreellm 評価: 行列積を消した HGRNBit を Transformers 互換で読む",
 *        section "HGRNBit という層構成を読む" — FusedBitLinear holds an RMSNorm(eps=1e-08)
 *        inside the projection; gate_proj is 2048 -> 11264, down_proj 5632 -> 2048, SiLU.
 *   [P3] "MatMul-Free LM: Ternary-Gewichte statt Matrixmultiplikation im Transformer",
 *        section "HGRNBit: was in einem Block tatsächlich passiert" — bias=False; the norm is
 *        fused with the ternary projection.
 *   [P4] "MatMul-freie LLMs: Zentrale Konzepte erklärt", sections "MatMul durch ternäre
 *        Operationen ersetzen" (absmean quantisation of W to {-1,0,1}; products become adds
 *        and subtracts) and "Kernkomponenten: MLGRU und GLU" (figure items 4 and 5; the GLU
 *        paragraph).
 *
 * What one forward call computes, for x [T x K], norm weight g [K], packed weight codes c
 * [N x K] with scale beta:
 *   r_t     = sqrt(mean_k x_tk^2 + eps)                      (mean of squares in double,
 *                                                              rounded once to float)
 *   xhat_tk = (x_tk * (1/r_t)) * g_k                          (float)
 *   gamma_t = max(max_k |xhat_tk|, 1e-5)
 *   q_tk    = clamp(round_half_even(xhat_tk * (127/gamma_t)), -128, 127)      (int8)
 *   acc_tn  = sum_{c_nk=+1} q_tk - sum_{c_nk=-1} q_tk                         (int32, exact)
 *   y_tn    = acc_tn * (gamma_t/127) * beta                   (float, stored as f16 or f32)
 * and the GLU form (gate_proj, N2 = 2I outputs) writes
 *   h_ti    = silu(y_ti) * y_t,I+i,  silu(z) = z / (1 + exp(-z)),  i < I       (f16 or f32)
 *
 * Weight quantisation (once per weight matrix):
 *   beta    = max( float( double(exact sum_{n,k} |W_nk|) / (N*K) ), 1e-5 )
 *   c_nk    = clamp(round_half_even(W_nk / beta), -1, 1)      (division in float)
 *
 * Packed weight layout ("Wp", N x K/4 bytes, row-major, the library's own format — the pages
 * fix none): the 16 codes k = 16G + 4i + j (i, j in 0..3) of group G of a row live in the
 * little-endian 32-bit word at bytes 4G..4G+3 of that row, at bits 8j+2i and 8j+2i+1, as
 * e = c + 1 (0, 1 or 2; the value 3 never occurs).  Equivalently byte j of a word holds the
 * codes of k = j, j+4, j+8, j+12 of its group at bit pairs 0, 2, 4, 6.
 *
 * Conventions for every entry point:
 *   - Memory: every pointer except those marked "host" is device memory owned by the caller.
 *     The library allocates nothing per call.  Scratch comes from the caller's workspace.
 *   - Alignment: every device pointer must be 16-byte aligned; workspaces 256-byte aligned.
 *   - Shapes: row-major, contiguous.  K % 128 == 0 with 128 <= K <= 8192; N % 128 == 0;
 *     1 <= T <= 16777216.
 *   - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream and never synchronise the host, except
 *     mmf_get_device_status.
 *   - Errors: argument checks run on the host before any launch and return a status without
 *     touching the device.  A failed launch returns MMF_ERR_CUDA.  A device-side wait that
 *     runs past its time limit latches MMF_ERR_TIMEOUT in a device status word that
 *     mmf_get_device_status reads; the kernel then returns instead of hanging.
 *   - Threads: calls on distinct streams may run concurrently from distinct host threads as
 *     long as they use distinct workspaces.
 */
#ifndef MMF_H_
#define MMF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MMF_OK = 0,
  MMF_ERR_INVALID_ARG = 1,        /* null pointer, bad dtype, non-positive eps, ... */
  MMF_ERR_UNSUPPORTED_SHAPE = 2,  /* a dimension outside the limits above */
  MMF_ERR_ALIGNMENT = 3,          /* a pointer not aligned as required */
  MMF_ERR_CUDA = 4,               /* a CUDA runtime or driver call failed */
  MMF_ERR_TIMEOUT = 5,            /* a device-side wait ran past its limit */
  MMF_ERR_WORKSPACE = 6,          /* workspace missing or smaller than required */
  MMF_ERR_RESOURCES = 7,          /* the device cannot hold every CTA of a program at once */
  MMF_ERR_PLAN = 8                /* a program run found no valid plan in its workspace */
} mmf_status;

typedef enum { MMF_F32 = 0, MMF_F16 = 1 } mmf_dtype;

/* ---- weight quantisation ([P4] "MatMul durch ternäre Operationen ersetzen") ------------- */

/* Workspace bytes mmf_quantize_weights needs for an N x K matrix (a fixed 4 KiB). */
size_t mmf_quantize_weights_workspace_bytes(int64_t N, int64_t K);

/* W [N x K] (wdt: f32 or f16, finite values) -> Wp [N x K/4] packed codes and beta (one
 * float, device).  Runs three kernels: an exact sum of |W|, a one-thread finalisation of
 * beta, and the encode+pack pass.  ws must hold mmf_quantize_weights_workspace_bytes. */
mmf_status mmf_quantize_weights(const void* W, mmf_dtype wdt, int64_t N, int64_t K,
                                uint8_t* Wp, float* beta, void* ws, size_t ws_bytes,
                                void* stream);

/* Encode+pack pass alone, with beta given (device float): the codes of W under that beta.
 * Lets callers (and the parity tests) fix beta and compare codes bit for bit. */
mmf_status mmf_ternary_encode(const void* W, mmf_dtype wdt, int64_t N, int64_t K,
                              const float* beta, uint8_t* Wp, void* stream);

/* ---- forward ([P1], [P3]; [P4] figure items 4 and 5) ------------------------------------ */

/* Workspace bytes one forward call with T tokens, K inputs and N weight rows needs: the int8
 * activation codes [T x K], gamma [T] and the code row sums [T], each 256-byte aligned, and
 * for T > 128 (the prefill contraction) the weight codes expanded to int8 [N x K]. */
size_t mmf_forward_workspace_bytes(int64_t T, int64_t K, int64_t N);

/* y [T x N] = FusedBitLinear(x [T x K]).  xdt: f32 or f16.  norm_w: K floats or NULL
 * (all ones).  eps > 0 (the model uses 1e-8).  Wp/beta from mmf_quantize_weights.
 * ydt: f32 or f16.  Two launches on `stream`: RMSNorm + activation quantisation, then the
 * tensor-core ternary contraction with the dequantisation epilogue. */
mmf_status mmf_bitlinear_forward(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                 const float* norm_w, float eps, const uint8_t* Wp,
                                 const float* beta, int64_t N, void* y, mmf_dtype ydt,
                                 void* ws, size_t ws_bytes, void* stream);

/* gate_proj with the fused SiLU-GLU epilogue ([P4] GLU paragraph; [P1] 2I -> I).
 * Wp holds the whole 2I x K gate_proj (N2 = 2I rows, one beta); h [T x I] receives
 * silu(first half) * second half.  N2 % 128 == 0. */
mmf_status mmf_bitlinear_glu_forward(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                     const float* norm_w, float eps, const uint8_t* Wp,
                                     const float* beta, int64_t N2, void* h, mmf_dtype hdt,
                                     void* ws, size_t ws_bytes, void* stream);

/* ---- the two halves of the forward, exported for bit-exact checks ------------------------ */

/* RMSNorm + activation quantisation alone: A [T x K] int8, gamma [T], rowsum [T] (the plain
 * sum of each row of A; may be NULL). */
mmf_status mmf_quantize_activations(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                    const float* norm_w, float eps, int8_t* A, float* gamma,
                                    int32_t* rowsum, void* stream);

/* Workspace bytes mmf_bitlinear_forward_quantized needs for the prefill contraction: the weight
 * codes expanded to int8 [N x K] when T > 128, else 0. */
size_t mmf_quantized_workspace_bytes(int64_t T, int64_t K, int64_t N);

/* Second half of the forward: contraction + dequantisation (+ SiLU-GLU when glu != 0, then
 * N is 2I and y is T x I) from activation codes already produced by mmf_quantize_activations
 * (A [T x K], gamma [T], rowsum [T]).  Lets callers reuse one quantised input for several
 * projections whose norm weights are equal.  ws: NULL with ws_bytes 0 (the contraction that
 * needs no workspace), or mmf_quantized_workspace_bytes(T, K, N) bytes, 256-byte aligned;
 * for T > 128 and N % 256 == 0 the latter selects the faster prefill contraction, which first
 * expands the packed codes into ws.  Same results either way. */
mmf_status mmf_bitlinear_forward_quantized(const int8_t* A, const float* gamma,
                                           const int32_t* rowsum, int64_t T, int64_t K,
                                           const uint8_t* Wp, const float* beta, int64_t N,
                                           int glu, void* y, mmf_dtype ydt, void* ws,
                                           size_t ws_bytes, void* stream);

/* acc [T x N] int32 = ternary accumulation of given codes A [T x K] against Wp.  Exact.
 * ws must hold mmf_forward_workspace_bytes(T, K, N). */
mmf_status mmf_ternary_accumulate_i32(const int8_t* A, int64_t T, int64_t K, const uint8_t* Wp,
                                      int64_t N, int32_t* acc, void* ws, size_t ws_bytes,
                                      void* stream);

/* ---- a whole decode step in one launch ---------------------------------------------------- */

/* One FusedBitLinear of a program.  Projections are grouped into dependency levels: the input
 * of a level-L projection may be the output of any projection of a lower level (for example
 * down_proj reading gate_proj's GLU output), never of the same or a higher level. */
typedef struct {
  const void* x;          /* input [T x K] (device), f16 or f32 */
  mmf_dtype xdt;
  const float* norm_w;    /* K floats or NULL (all ones) */
  const uint8_t* Wp;      /* packed weights [N x K/4] from mmf_quantize_weights */
  const float* beta;      /* device float */
  int64_t K;              /* in_features: K % 128 == 0, K <= 8192 (f16) or 4096 (f32) */
  int64_t N;              /* weight rows: N % 128 == 0 (2I for the GLU form) */
  int32_t glu;            /* 1: SiLU-GLU epilogue, output is T x N/2 */
  int32_t level;          /* 0-based dependency level */
  void* y;                /* output (device), T x N (or T x N/2) */
  mmf_dtype ydt;
} mmf_projection;

/* Workspace bytes a program of n projections at T tokens needs: the plan, the quantised
 * inputs, split-K accumulators and counters, and a re-tiled copy of every projection's packed
 * weights (N*K/4 bytes each, rounded up to whole 512-wide k-stages).  0 if the program is not
 * supported (T > 64, more than 1024 projections or 128 levels, or a shape outside the limits). */
size_t mmf_program_workspace_bytes(const mmf_projection* p, int n, int64_t T);

/* Plans a program into `ws` ([P1], [P3]; [P4] figure items 4 and 5, for every projection):
 * groups projections that share an input into one quantisation, splits every level's
 * k-blocks over the SMs and zeroes the counters.  It also re-tiles every projection's packed
 * weights (Wp, canonical layout L1) into the workspace, in blocks that one contiguous copy
 * brings on chip: runs read that copy, so Wp may be freed once the init has executed (the
 * program then holds one copy of the weights, not two), and a change of the weights needs a
 * new init.  The other pointers in `p` are baked into the plan: every later mmf_program_run
 * reads and writes those same buffers.  All device work is stream-ordered on `stream`; the
 * init copies from pageable host memory, so it must not be captured into a CUDA graph.
 * 1 <= T <= 64.  Returns MMF_ERR_RESOURCES if the device cannot hold one CTA on every SM at
 * once (the runs' grid-wide waits need every CTA resident). */
mmf_status mmf_program_init(const mmf_projection* p, int n, int64_t T, float eps, void* ws,
                            size_t ws_bytes, void* stream);

/* Runs a planned program: one persistent launch, one CTA per SM.  Level by level, every CTA
 * quantises a share of the level's input rows (RMSNorm + int8), then streams its share of the
 * packed weights through the tcgen05 contraction (weights are prefetched across levels), and
 * the level ends when every output is written.
 * Co-residency: the CTAs wait for one another at every level, so the launch is made
 * cooperative where the driver accepts that (it then places the whole grid at once, or fails
 * with MMF_ERR_RESOURCES); where it does not, a run needs the whole GPU to itself.  Either way
 * every grid-wide wait is bounded: a CTA that is never placed makes the others record
 * MMF_ERR_TIMEOUT (mmf_get_device_status) and return instead of hanging; call
 * mmf_program_init again before the next run in that case.
 * The launch checks the plan in `ws` (a magic number, the init's generation, the token tile
 * and the grid size): a workspace that no longer holds the plan it was initialised with is
 * refused without any other read or write, and mmf_get_device_status then returns
 * MMF_ERR_PLAN.  `ws` not passed to a successful mmf_program_init: MMF_ERR_INVALID_ARG.
 * Calls on one workspace must not overlap. */
mmf_status mmf_program_run(void* ws, void* stream);

/* ---- MLGRU recurrence + FusedRMSNormSwishGate ----------------------------------------------
 * [P4] "MatMul-freie LLMs: Zentrale Konzepte erklärt", section "Kernkomponenten: MLGRU und GLU",
 * the MLGRU paragraph: token by token, element-wise gates with values between 0 and 1 weigh
 * the previous hidden state against the current token.  [P1] section "HGRNBit という層構成を読む":
 * the attention side gates through FusedRMSNormSwishGate ahead of o_proj.  The pages give no
 * formula; the library computes, for the i/f/g projection outputs I, F, G [T x H] and j < H:
 *   f_tj = sigmoid(F_tj),  c_tj = silu(I_tj),  h_tj = f_tj * h_(t-1)j + (1 - f_tj) * c_tj
 *   o_tj = h_tj / sqrt(mean_j h_tj^2 + eps) * w_j * silu(G_tj)
 * with h before the first token = h0 (zero when NULL), in float (exp and reciprocals through
 * the fast intrinsics: relative error a few 1e-6 before the output's own rounding).  Tokens are
 * scanned in chunks of 32; chunk boundaries change only the rounding order of h.
 *
 * Shapes: 1 <= T <= 16777216; H a multiple of 256, 256 <= H <= 4096.  I, F, G, o: row-major,
 * 16-byte aligned, all of dtype xdt (I/F/G) and odt (o).  h0, hT, norm_w: [H] fp32 (may be
 * NULL), 16-byte aligned.  ws: mmf_mlgru_workspace_bytes(T, H) bytes, 256-byte aligned (NULL
 * with ws_bytes 0 when that is 0, i.e. T <= 32).  Errors as for the forward; a workspace that
 * is missing or too small: MMF_ERR_WORKSPACE.  Asynchronous on `stream`. */
size_t mmf_mlgru_workspace_bytes(int64_t T, int64_t H);

mmf_status mmf_mlgru_forward(const void* I, const void* F, const void* G, mmf_dtype xdt,
                             int64_t T, int64_t H, const float* h0, const float* norm_w,
                             float eps, void* o, mmf_dtype odt, float* hT, void* ws,
                             size_t ws_bytes, void* stream);

/* The same recurrence and gate, fused with o_proj's activation pre-pass: instead of o it
 * writes what mmf_quantize_activations(o16, MMF_F16, T, H, oproj_norm_w, oproj_eps, A, gamma,
 * rowsum) would write for o16 = o rounded to fp16 (A [T x H] int8 row-major, gamma [T],
 * rowsum [T] or NULL), ready for mmf_bitlinear_forward_quantized with K = H.  The sum of
 * squares of a row is added in another order, so in rare rows its last bit, and with it a
 * code, can differ from the separate pre-pass. */
mmf_status mmf_mlgru_forward_quantized(const void* I, const void* F, const void* G,
                                       mmf_dtype xdt, int64_t T, int64_t H, const float* h0,
                                       const float* norm_w, float eps,
                                       const float* oproj_norm_w, float oproj_eps, int8_t* A,
                                       float* gamma, int32_t* rowsum, float* hT, void* ws,
                                       size_t ws_bytes, void* stream);

/* ---- backward (straight-through) ------------------------------------------------------------
 * The pages print no backward pass.  [P4] "MatMul durch ternäre Operationen ersetzen": the
 * weights are trained in full precision and quantised to {-1,0,1} during training, i.e. both
 * quantisers sit inside the training forward pass.  The library takes the straight-through
 * reading: rounding and clamping pass the gradient unchanged, so the gradient is that of the
 * bilinear map of the dequantised operands (xq_tk = q_tk * gamma_t/127, wq_nk = c_nk * beta)
 * after the RMSNorm (xhat = x / r * g, r as in the forward), with the latent weight taking
 * wq's gradient.  For the loss gradient dy [T x N] of the forward's y:
 *   dW_nk  = sum_t dy_tn * xq_tk                                        (fp32 [N x K])
 *   dxh_tk = beta * sum_n dy_tn * c_nk
 *   dx_tk  = g_k dxh_tk / r_t - x_tk (sum_j g_j dxh_tj x_tj) / (K r_t^3)   (dxdt [T x K])
 *   dg_k   = sum_t dxh_tk * x_tk / r_t                                  (fp32 [K])
 * Both sums over n and t run on the tensor cores with fp16 operands and fp32 accumulation:
 * dy and the codes are exact in fp16, dy_tn * gamma_t/127 is rounded once to fp16 (relative
 * error at most 2^-11 per term of dW).  r_t and the norm step are float.
 *
 * x, xdt, T, K, norm_w, eps, Wp, beta, N: as passed to the forward.  A [T x K] int8 and gamma
 * [T]: the forward's activation codes and scales (from mmf_quantize_activations), or both NULL
 * to have the call recompute them from x.  dy: fp16 [T x N], row-major.  dx (dxdt f32 or f16),
 * dW and dnorm_w: outputs, each may be NULL to skip it (at least one must be given); they are
 * overwritten, not accumulated into.  ws: mmf_backward_workspace_bytes(T, K, N) bytes, 256-byte
 * aligned.  Errors as for the forward.  Asynchronous on `stream` (up to eleven launches). */
size_t mmf_backward_workspace_bytes(int64_t T, int64_t K, int64_t N);

mmf_status mmf_bitlinear_backward(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                  const float* norm_w, float eps, const int8_t* A,
                                  const float* gamma, const uint8_t* Wp, const float* beta,
                                  int64_t N, const void* dy, void* dx, mmf_dtype dxdt,
                                  float* dW, float* dnorm_w, void* ws, size_t ws_bytes,
                                  void* stream);

/* ---- forward without any allocation ------------------------------------------------------ */

/* The pages have no counterpart to this entry point; it serves callers that cannot call
 * cudaMalloc (a plugin inside an application that owns all device memory, a real-time decode
 * loop that must not allocate, C code without a device allocator).  Same arguments and
 * result as mmf_bitlinear_forward, without the workspace: the scratch (int8 codes [T x K],
 * gamma [T], code sums [T], each rounded up to 256 bytes) lives in a fixed 4 MiB device
 * array that every GPU loading the library holds until the process exits.  Calls whose
 * scratch would exceed 4 MiB are rejected with MMF_ERR_WORKSPACE before any launch (for
 * example T = 64 with K = 8192 fits; T = 512 with K = 8192 does not).  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, device current); make
 * that first call before any stream capture.  All calls share the array: nothing in it needs
 * to start at zero, but calls whose work overlaps on the GPU race on it, so order them on one
 * stream (or with events). */
mmf_status mmf_bitlinear_forward_noalloc(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                         const float* norm_w, float eps, const uint8_t* Wp,
                                         const float* beta, int64_t N, void* y, mmf_dtype ydt,
                                         void* stream);

/* ---- status ------------------------------------------------------------------------------ */

/* Reads and clears the device status word of the current device (synchronises the device).
 * Returns MMF_OK, MMF_ERR_TIMEOUT if a kernel gave up on a wait since the last read,
 * MMF_ERR_PLAN if a program run refused its workspace (and nothing timed out), or
 * MMF_ERR_CUDA if the read itself failed. */
mmf_status mmf_get_device_status(void);

/* Launches one block whose single wait can never be satisfied and must give up after
 * `limit_ns` nanoseconds (1e3 <= limit_ns <= 1e9); the next mmf_get_device_status then
 * returns MMF_ERR_TIMEOUT.  Exercises the same bounded-wait routine the pipelined kernels
 * use, without any copy or tensor-core work in flight. */
mmf_status mmf_debug_wait_timeout_probe(uint64_t limit_ns, void* stream);

/* Human-readable name of a status. */
const char* mmf_status_string(mmf_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
int mmf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MMF_H_ */
