/*
 * had.h -- C ABI of the B200 (sm_100a) library for binarized-QK top-N
 * attention, as defined by "Hamming Attention Distillation: Binarizing Keys
 * and Queries for Efficient Long-Context Transformers" (HAD) and
 * "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 * Transformers" (BinaryAttention).
 *
 * Operation (per batch b, head h, valid length L = seqlens[b] or n):
 *   mu_X[c]  = mean_{i<L} X[i,c]                 X in {Q, K}   (BinaryAttention §2.2, scaled binarization)
 *   X~[i,c]  = sign(X[i,c] - mu_X[c]) in {-1,+1}, packed to bits (bit 1 = -1)   (§2.2; HAD abstract)
 *   s_ij     = d - 2 * popcount(q~_i XOR k~_j)                 (§2.1 distance view, §2.2 XNOR + popcount)
 *   l_ij     = fmaf(s_ij, c, b_ij),  c = fp32(alpha_q[h] * alpha_k[h] / sqrt(d))   (§2.3 eq.)
 *   kept_i   = the min(N, L) keys j < L with the largest l_ij, ties to the lower j;
 *              N == 0 or N >= L keeps all L keys   (HAD method: top-N per query)
 *   p_ij     = softmax over kept_i of l_ij   (§2.3 eq.)
 *   O_i      = sum_j p_ij V_j                                   (HAD_MODE_FLOAT)
 *   O_i[c]   = (sum_j A_ij Vq_jc) * sv_c / 255,  A_ij = floor(255 p_ij + 0.5) in uint8,
 *              sv_c = absmax_{j<L} |V_jc| / 127, Vq = clamp(rint(V / sv_c), -127, 127)   (HAD_MODE_U8I8, §2.4)
 *   O_i[c]   = the same with sv_c = absmax_{j<L} |V_jc| / 7, Vq = clamp(rint(V / sv_c), -7, 7)   (HAD_MODE_U8I4:
 *              BinaryAttention's conclusion names lower-bit V without defining it; this is the §2.4
 *              scheme at 4 bits)
 * Rows i >= L of O are written as 0.  Padding tokens never enter a mean, a
 * scale, a score or a softmax.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller (for example
 *     torch tensors' data_ptr()), except in had_attention_host, which takes
 *     host arrays.  Q, K, V, O are contiguous [B][H][n][d].
 *     Device pointers must be 16-byte aligned.
 *   - The library never allocates, frees or synchronizes in these calls: work
 *     is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and the call returns.  Scratch memory is the caller's
 *     `workspace` of at least the size the matching *_workspace_size() returns.
 *   - Host-side validation happens before any launch: on an error status
 *     nothing was enqueued and no output was touched.
 *   - Errors detected on the device (a seqlens entry outside [1, n]) set a
 *     sticky device status word and zero the affected batch's outputs; read
 *     it with had_get_device_status().
 *   - Head dims d = 64 and 128 (d = 32 too in had_binarize_pack,
 *     had_binarize_pack_noalloc, had_quantize_v and had_quantize_v4; had_scores_int is d = 64
 *     only); HAD_ERR_UNSUPPORTED otherwise.  n <= 16384, H <= 256, B*H <= 65535.
 */
#ifndef HAD_H_
#define HAD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HAD_OK = 0,
  HAD_ERR_INVALID = 1,      /* null/misaligned pointer, bad size, alpha <= 0, workspace too small */
  HAD_ERR_UNSUPPORTED = 2,  /* d not 64 or 128, n > 16384, H > 256, unsupported dtype/mode combination */
  HAD_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed; see had_last_cuda_error() */
  HAD_ERR_DEVICE = 4,       /* device-detected error (bad seqlens); from had_get_device_status() */
  HAD_ERR_TIMEOUT = 5       /* a bounded device-side wait expired; from had_get_device_status() */
} had_status;

typedef enum { HAD_F32 = 0, HAD_BF16 = 1 } had_dtype;

typedef enum {
  HAD_MODE_FLOAT = 0,  /* float softmax and float A.V (bf16 P x bf16 V, fp32 accumulate; fp32 V exact to ~1e-5) */
  HAD_MODE_U8I8 = 1,   /* uint8 A (scale 1/255) x per-channel int8 V, int32 accumulate (BinaryAttention §2.4) */
  HAD_MODE_U8I4 = 2    /* uint8 A x per-channel 4-bit V (codes in [-7, 7], stored two per byte), int32 accumulate;
                          had_attention, had_attention_prepare/_prepared and had_attention_host only */
} had_mode;

typedef struct {
  int B, H, n, d;           /* batch, heads, tokens per sequence (padded length), head dim */
  had_dtype in_dtype;       /* dtype of Q, K, V (and of X in had_binarize_pack) */
  const int32_t* seqlens;   /* DEVICE [B] valid lengths in [1, n], or NULL for all n */
} had_shape;

/* Learnable attention bias B of BinaryAttention §2.3.
 * dense == 0: the relative-position bias ("position-sensitive bias", the option
 *   its experiments use).  Token t >= prefix is patch (y, x) =
 *   divmod(t - prefix, gw) of a gh x gw grid; then
 *   b_ij = table[h][(y_i - y_j) + gh - 1][(x_i - x_j) + gw - 1], and b_ij = 0
 *   when i < prefix or j < prefix (class tokens).  Requires gh*gw + prefix == n.
 * dense == 1: the dense learnable matrix (one bias per query-key pair):
 *   b_ij = table[h][i][j], table [H][n][n]; gh, gw and prefix are ignored.  Its
 *   extended tables take 2 * H * n * (n + 2) floats of workspace, so n is
 *   limited to 4096 (HAD_ERR_UNSUPPORTED above).
 * A bias that is a sum of functions of the relative offset (y_i - y_j,
 * x_i - x_j), such as a spatial plus a directional term, is a
 * relative-position table: pass its (2gh-1) x (2gw-1) values with dense == 0. */
typedef struct {
  const float* table;  /* DEVICE fp32 (HOST in had_attention_host); NULL means no bias */
  int gh, gw;
  int prefix;
  int dense;           /* 0: relative-position table; 1: dense [H][n][n] matrix */
} had_relpos_bias;

/* ---- binarize and pack (BinaryAttention §2.2; HAD abstract) --------------
 * X: [B][H][n][d] in s->in_dtype.  bits: DEVICE uint32 [B][H][n][d/32]; bit j
 * of word w is 1 iff X[b,h,i,32w+j] < mu[b,h,32w+j] (sign -1); tokens i >= L
 * get all-zero words.  mu_in: DEVICE fp32 [B][H][d] to use as the means, or
 * NULL to compute them (fp64 sum over the valid tokens, / L, rounded once to
 * fp32).  mu_out: DEVICE fp32 [B][H][d] receives the means used, or NULL.
 * workspace: needed only when mu_in is NULL. */
size_t had_binarize_pack_workspace_size(const had_shape* s);
had_status had_binarize_pack(const void* X, const had_shape* s, const float* mu_in, float* mu_out, uint32_t* bits,
                             void* workspace, size_t ws_bytes, void* stream);

/* had_binarize_pack_noalloc: the same computed-means pack as had_binarize_pack
 * (mu_in == NULL), for callers that cannot allocate device memory at the point
 * of call -- for example a plugin run inside a host framework that owns every
 * device allocation, or a latency-critical loop that must not call cudaMalloc
 * (which can synchronize the device) -- and so cannot supply a workspace.  The
 * paper has no counterpart: this is a library convenience.
 * Its scratch is a fixed 4 MiB device array inside the library, which every
 * GPU that loads the library holds until the process exits; shapes with
 * B*H*ceil(n/64) > 8192 are rejected with HAD_ERR_UNSUPPORTED (message in
 * had_last_cuda_error()).  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current), so make
 * that first call before any stream capture.  All calls on a device share the
 * one array: calls that overlap on the GPU (other streams, other host
 * threads) race and corrupt each other's means; serialize them.  Nothing in
 * the array needs clearing: each call overwrites every entry it reads.
 * Allocates and frees nothing. */
had_status had_binarize_pack_noalloc(const void* X, const had_shape* s, float* mu_out, uint32_t* bits, void* stream);

/* ---- the hot path (HAD + BinaryAttention, formulas above) ----------------
 * bias: HOST pointer to a had_relpos_bias (its table is device memory), or
 * NULL.  alpha_q, alpha_k: HOST fp32 [H] positive per-head scales of the
 * binarized Q and K (BinaryAttention §2.2), or NULL for 1.  N: top-N per
 * query; 0 (or >= L) = dense.  O: DEVICE [B][H][n][d] in o_dtype. */
size_t had_attention_workspace_size(const had_shape* s, int N, had_mode mode, const had_relpos_bias* bias);
had_status had_attention(const void* Q, const void* K, const void* V, const had_shape* s,
                         const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                         had_mode mode, void* O, had_dtype o_dtype, void* workspace, size_t ws_bytes, void* stream);

/* The same operation in two stages, for callers that time or reuse them:
 * had_attention_prepare runs the per-head statistics and the sign/pack of Q
 * and K (and the int8 or 4-bit V of the uint8 modes, and the bias range of top-N with a
 * bias) into `workspace`; had_attention_prepared then runs the fused
 * score/top-N/softmax/A.V kernel over that workspace.  Both must get the same
 * s, bias, N and mode; had_attention_prepared reads V only in HAD_MODE_FLOAT.
 * had_attention == prepare + prepared on one stream. */
had_status had_attention_prepare(const void* Q, const void* K, const void* V, const had_shape* s,
                                 const had_relpos_bias* bias, int N, had_mode mode, void* workspace, size_t ws_bytes,
                                 void* stream);
had_status had_attention_prepared(const void* V, const had_shape* s, const had_relpos_bias* bias,
                                  const float* alpha_q, const float* alpha_k, int N, had_mode mode, void* O,
                                  had_dtype o_dtype, void* workspace, size_t ws_bytes, void* stream);

/* ---- the projection before the path, fused with the binarization ---------
 * had_qkv_prepare takes the step that produces the attention's inputs, the QKV
 * projection Q|K|V = X Wqkv^T, and binarizes Q and K in its epilogue instead of
 * in a separate quantization pass (BinaryAttention §2.2 scaled binarization; its
 * Table 8 counts that pass against the kernel):
 *   mu_Q[b][h][c] = mean over the valid tokens of X[b] Wq^T, computed as
 *                   xbar_b . Wq[h*64 + c] with xbar_b the mean of X[b]'s valid tokens
 *                   (the same value in exact arithmetic; fp64, one rounding to fp32);
 *   Q bits        = (X Wq^T < mu_Q) per token and channel, from the fp32 tensor-core
 *                   projection; likewise K (as the +-1 rows the score MMA reads);
 *   V_out         = X Wv^T, rounded to bf16.
 * It fills `workspace` as had_attention_prepare does (including the bias tables
 * and, in the uint8 modes, the quantized V), so that had_attention_prepared(V_out,
 * s, bias, alpha_q, alpha_k, N, mode, O, ...) on the same stream and workspace
 * completes the path.
 *   X:     DEVICE bf16 [B][n][Dm] tokens; Dm > 0, a multiple of 64, <= 16384.
 *   Wqkv:  DEVICE bf16 [3*H*64][Dm], a linear layer's weight layout: row h*64 + c
 *          is Q's channel c of head h, row H*64 + h*64 + c K's, row 2*H*64 + h*64 + c V's.
 *   s:     B, H, n, d = 64, in_dtype HAD_BF16 (HAD_ERR_UNSUPPORTED otherwise), seqlens.
 *   V_out: DEVICE bf16 [B][H][n][64] (written for every token < n).
 *   workspace: at least had_qkv_workspace_size(s, Dm, N, mode, bias) bytes.
 * Errors as had_attention (host validation first; device errors in the status word). */
size_t had_qkv_workspace_size(const had_shape* s, int Dm, int N, had_mode mode, const had_relpos_bias* bias);
had_status had_qkv_prepare(const void* X, const void* Wqkv, const had_shape* s, int Dm, const had_relpos_bias* bias,
                           int N, had_mode mode, void* V_out, void* workspace, size_t ws_bytes, void* stream);

/* ---- host arrays in, host array out --------------------------------------
 * had_attention_host: had_attention on HOST memory, with the copies inside the
 * call.  Q, K, V: HOST [B][H][n][d] in s->in_dtype; O: HOST [B][H][n][d] in
 * o_dtype; s->seqlens: HOST int32 [B] (each in [1, n], checked on the host) or
 * NULL; bias->table: HOST fp32 (as the bias struct describes) or bias NULL; alpha_q,
 * alpha_k as in had_attention.  The batch is cut into chunks of chunk_b
 * sequences (0: the library picks about 8 MiB of inputs per chunk, and when one
 * sequence holds more, cuts each sequence into equal groups of heads of at most
 * 16 MiB).  Chunk k's Q, K, V are copied in on one side stream while chunks k-1
 * and k-2 are computed, alternately on `stream` and on a side compute stream,
 * and chunk k-3's O is copied out on another side stream.  The chunks cycle
 * through four device slots in `workspace`, which needs at least
 * had_attention_host_workspace_size(s, N, mode, bias, chunk_b) bytes.  Every
 * (b, h) is computed by the same kernels as in had_attention, so O is
 * bit-identical to it for any chunk_b.
 * Copies overlap one another and the kernels only from page-locked host memory
 * (cudaHostAlloc / cudaHostRegister); pageable memory works, serialized.  The
 * call enqueues all of it behind the work already on `stream` and returns: O
 * is complete once `stream` has reached that point.  The host arrays must stay
 * valid and unchanged until then.  Each call creates up to three streams and
 * some events and releases them (CUDA frees them once their work is done);
 * it allocates no memory. */
size_t had_attention_host_workspace_size(const had_shape* s, int N, had_mode mode, const had_relpos_bias* bias,
                                         int chunk_b);
had_status had_attention_host(const void* Q, const void* K, const void* V, const had_shape* s,
                              const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                              had_mode mode, void* O, had_dtype o_dtype, int chunk_b, void* workspace,
                              size_t ws_bytes, void* stream);

/* ---- in-library dense comparison mode ------------------------------------
 * Standard attention on the unbinarized inputs (the full-precision attention the
 * pages compare against): l = (q . k)/sqrt(d) + b_ij with bf16 q, k on the
 * tcgen05 tensor cores (fp32 accumulate in tensor memory), fp32 softmax with an
 * online row maximum, bf16 P x V.  Requires in_dtype == HAD_BF16 and N == 0 or
 * N >= n (dense); otherwise HAD_ERR_UNSUPPORTED.  The workspace holds the bias
 * tables: had_dense_reference_workspace_size(s, bias) bytes (0 without a bias,
 * when workspace may be NULL). */
size_t had_dense_reference_workspace_size(const had_shape* s, const had_relpos_bias* bias);
had_status had_dense_reference_mode(const void* Q, const void* K, const void* V, const had_shape* s,
                                    const had_relpos_bias* bias, int N, void* O, had_dtype o_dtype,
                                    void* workspace, size_t ws_bytes, void* stream);

/* ---- parity / debug exports (small shapes; not part of the timed path) ---
 * had_scores_int: S DEVICE int32 [B][H][n][n], S = d - 2*popcount(q XOR k) for
 * i, j < L and 0 elsewhere, from packed bits as had_binarize_pack writes them. */
had_status had_scores_int(const uint32_t* qbits, const uint32_t* kbits, const had_shape* s, int32_t* S,
                          void* stream);

/* had_attention_scores: the integer scores s_ij = d - 2*popcount(q~_i XOR k~_j)
 * (BinaryAttention §2.1-§2.2) exactly as the fused kernel forms them -- the
 * +-1 int8 tensor-core product of the binarized Q and K in tensor memory --
 * written out as DEVICE int32 S [B][H][n][n] (0 where i >= L or j >= L).
 * Q, K as in had_attention; workspace as had_attention_workspace_size(s, 0,
 * HAD_MODE_FLOAT, NULL).  For parity checks on small shapes. */
had_status had_attention_scores(const void* Q, const void* K, const had_shape* s, int32_t* S, void* workspace,
                                size_t ws_bytes, void* stream);

/* had_topn_indices: the kept set of every query row, as DEVICE int32
 * [B][H][n][N] in ascending key order, padded with -1 (rows i >= L are all
 * -1).  Same arguments and workspace as had_attention with N >= 1. */
had_status had_topn_indices(const void* Q, const void* K, const had_shape* s, const had_relpos_bias* bias,
                            const float* alpha_q, const float* alpha_k, int N, int32_t* idx, void* workspace,
                            size_t ws_bytes, void* stream);

/* had_attention_codes_u8: the uint8 attention codes A_ij = floor(255 p_ij + 0.5)
 * (0 off the kept set and for j >= L) of query rows [row_begin, row_end) of
 * every (b, h), as DEVICE uint8 [B][H][row_end-row_begin][n].  Same
 * arguments and workspace as had_attention in HAD_MODE_U8I8. */
had_status had_attention_codes_u8(const void* Q, const void* K, const void* V, const had_shape* s,
                                  const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                                  int row_begin, int row_end, uint8_t* A, void* workspace, size_t ws_bytes,
                                  void* stream);

/* had_quantize_v: the per-channel int8 V of HAD_MODE_U8I8 (BinaryAttention
 * §2.4): Vq DEVICE int8 [B][H][n][d] (0 for tokens i >= L) and vscale DEVICE
 * fp32 [B][H][d].  Needs had_attention_workspace_size(s, 0, HAD_MODE_U8I8, NULL). */
had_status had_quantize_v(const void* V, const had_shape* s, int8_t* Vq, float* vscale, void* workspace,
                          size_t ws_bytes, void* stream);

/* had_quantize_v4: the per-channel 4-bit V of HAD_MODE_U8I4, one code in
 * [-7, 7] per int8 of Vq DEVICE [B][H][n][d] (0 for tokens i >= L; the attention
 * kernel stores them two per byte), vscale DEVICE fp32 [B][H][d] = absmax / 7
 * (1 where the absmax is 0).  Needs had_attention_workspace_size(s, 0,
 * HAD_MODE_U8I4, NULL); errors as had_quantize_v. */
had_status had_quantize_v4(const void* V, const had_shape* s, int8_t* Vq, float* vscale, void* workspace,
                           size_t ws_bytes, void* stream);

/* ---- tensor-pipe probe (a measurement aid; the pages have no counterpart) --
 * had_probe_mma_rate: the rate this GPU's tensor cores sustain on the two MMA
 * kinds the hot path issues -- kind 0: tcgen05.mma kind::i8 (the +-1 score
 * contraction of BinaryAttention §2.2, and the uint8 A x int8 V of §2.4);
 * kind 1: kind::f16 with bf16 operands (the float A.V).  One CTA per SM issues
 * `iters` (2 .. 2^22) back-to-back M=128 N=256 MMAs (K = 32 int8 or 16 bf16
 * elements each) from operands resident in shared memory into one tensor-memory
 * accumulator.  *tops receives 2*M*N*K*iters*SMs / elapsed in 10^12 ops/s, and
 * *ms (if not NULL) the elapsed milliseconds.  Runs on the legacy default
 * stream of the current device and waits for it (not for use in a hot loop);
 * allocates no device memory. */
had_status had_probe_mma_rate(int kind, int iters, double* tops, double* ms);

/* ---- the timeout path (a test hook; the pages have no counterpart) --------
 * had_debug_bounded_wait: every pipeline wait of the fused kernel (TMA loads,
 * tensor-core MMAs, the softmax warps' hand-offs) gives up after max_cycles SM
 * clocks (0 = the default, about one second; else at least 10000), sets the
 * HAD_ERR_TIMEOUT bit of the device status word, skips the rest of its work,
 * writes zero output, waits (with a bound of its own) for its loads and MMAs in
 * flight, and frees its tensor memory.  force_expiry != 0 makes one thread of
 * every CTA of the following launches first wait on a barrier that nothing
 * completes, so that this path runs; force_expiry = 0 restores normal runs.
 * The setting is library-wide and read at each launch (not thread-safe). */
had_status had_debug_bounded_wait(long long max_cycles, int force_expiry);

/* ---- status ---------------------------------------------------------------
 * had_get_device_status: synchronizes the current device, reads the sticky
 * device status word of the current device, clears it, and returns HAD_OK,
 * HAD_ERR_DEVICE or HAD_ERR_TIMEOUT. */
had_status had_get_device_status(void);
const char* had_status_string(had_status st);
/* The last CUDA error string recorded by a call that returned HAD_ERR_CUDA (thread-local). */
const char* had_last_cuda_error(void);
/* Library version as an integer (major*10000 + minor*100 + patch). */
int had_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HAD_H_ */
