/*
 * fa.h — C ABI of the B200 (sm_100a) exact attention library (libfa_b200.so).
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(Q Kᵀ · scale [+ causal mask]) V
 * tile by tile with an online softmax, so the N×N score and probability
 * matrices never reach device memory, and the training backward that
 * recomputes the probabilities per tile from Q, K, V, O and the saved row
 * log-sum-exp.
 *
 * Where each operation is defined (page title and section):
 *   scores S = QKᵀ/√d ............ "FlashAttention 详解（零基础入门）" §2.3
 *   safe softmax, row max ........ same page, §2.4
 *   O = PV ....................... same page, §2.5
 *   tiling, running m and ℓ ...... same page, §5.2, §5.4 and the §6.2 pseudocode
 *   causal mask (key j ≤ query i)  "Flash Attention 优化", nanoGPT manual fallback
 *   varlen packing ............... "FlashAttention 与算子融合", 工程实践 (varlen / packing)
 *   backward recomputation ....... "FlashAttention 短片讲解稿", segment "第三招 · 反向重计算"
 *   FLOP convention 4·B·h·s²·d ... "FlashAttention 与算子融合", 标准 Attention 浪费在哪
 *
 * Common conventions for every entry point
 * ----------------------------------------
 * Layout.  q, k, v, o, dO, dq, dk, dv are row-major [T, H, d] arrays (token,
 *   head, feature) with d contiguous, a token stride of H·d elements, all in
 *   one 16-bit dtype (FA_BF16 or FA_FP16).  lse is fp32 [T, H].  Self-attention
 *   only: queries and keys come from the same T tokens.
 * Sequences.  cu_seqlens == NULL: the T = B·N tokens form B sequences of N
 *   tokens (total_tokens must equal B·N).  cu_seqlens != NULL: a DEVICE int32
 *   array of B+1 non-decreasing prefix offsets with cu_seqlens[0] = 0 and
 *   cu_seqlens[B] ≤ total_tokens; N is then an upper bound on every sequence
 *   length (it sizes the launch grid).  A sequence of length 0 produces no rows.
 *   Offsets are not read on the host; a kernel that finds them inconsistent
 *   (decreasing, above total_tokens, a length above N) skips its work and
 *   records FA_ERR_INVALID_ARG in the device status word.
 * Causal.  causal = 1 hides key j from query i when j > i, with positions
 *   counted from the start of each sequence.
 * Numerics.  Products accumulate in fp32 on the tensor cores; the softmax runs
 *   in fp32 with base-2 exponentials (scale·log2(e) folded in, an exact
 *   reformulation); P is rounded to the input dtype before P·V; outputs are
 *   rounded to nearest-even.  Results equal the mathematical definition up to
 *   rounding, not bit for bit.
 * lse.  Natural-log log-sum-exp of the scaled, masked scores of each row.
 * Pointers.  Device pointers, 16-byte aligned, owned by the caller.  The
 *   library never allocates, frees or synchronises (except
 *   fa_check_device_status, which synchronises the given stream).
 * Streams.  Every launch goes on `stream` (a cudaStream_t; 0 = legacy default).
 * Sizes.  d ∈ {64, 128}; B, H, N ≥ 1; total_tokens ≥ 1; H·d·2 bytes and T·H·d
 *   elements must fit the tensor-map limits (checked: FA_ERR_UNSUPPORTED).
 * Errors.  Argument errors are returned synchronously before anything is
 *   launched.  Launch failures map to FA_ERR_CUDA.  Every wait inside the
 *   kernels is bounded by a watchdog; when one expires the kernel records
 *   FA_ERR_TIMEOUT in the device status word and returns, leaving the context
 *   usable.  Read that word with fa_check_device_status.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Opaque stream handle: pass a cudaStream_t. */
typedef void* fa_stream_t;

/*
 * Forward pass ("FlashAttention 详解" §6.2; the tiled loop with running m, ℓ).
 *   q, k, v      in   [T, H, d] dtype
 *   o            out  [T, H, d] dtype   O = softmax(QKᵀ·scale + mask) V
 *   lse          out  [T, H] fp32       row log-sum-exp (natural log)
 *   B, H, N, d   batch (number of sequences), heads, sequence length (max
 *                length when cu_seqlens != NULL), head dimension (64 or 128)
 *   scale        finite, > 0 (usually 1/√d)
 *   causal       0 or 1
 *   cu_seqlens   NULL or device int32 [B+1]
 *   total_tokens T, the number of token rows in every [T, …] array
 *   dtype        FA_BF16 or FA_FP16
 * Rows of o/lse that belong to no sequence are left untouched.
 * Returns FA_OK or an error code; see the conventions above.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, float scale, int causal,
           const int32_t* cu_seqlens, int total_tokens, int dtype, fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: an fp32 dQ accumulator [T, H, d]
 * and the fp32 row terms D_i = Σ_c dO_ic·O_ic [T, H], each 256-byte aligned.
 * Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int total_tokens, int H, int d);

/*
 * Backward pass: gradients of ⟨O, dO⟩ with respect to q, k, v, recomputing P
 * tile by tile from q, k and lse ("FlashAttention 短片讲解稿", segment
 * "第三招 · 反向重计算").  The gradient equations are the chain rule of the
 * forward definition: dV = Pᵀ dO, dP = dO Vᵀ, D_i = Σ_c dO_ic O_ic,
 * dS = P ∘ (dP − D), dQ = scale·dS K, dK = scale·dSᵀ Q.
 *   q, k, v, o   in   [T, H, d] dtype (o from fa_fwd with the same arguments)
 *   lse          in   [T, H] fp32 (from fa_fwd)
 *   dO           in   [T, H, d] dtype
 *   dq, dk, dv   out  [T, H, d] dtype; rows that belong to no sequence are left
 *                untouched
 *   workspace    device buffer of at least fa_bwd_workspace_bytes(T, H, d)
 *                bytes, 256-byte aligned, owned by the caller; its contents on
 *                entry do not matter and on return are unspecified
 * Other arguments as for fa_fwd.  Launches three kernels on `stream`:
 * fa_bwd_preprocess, fa_bwd_main and fa_bwd_postprocess, in that order.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv,
           int B, int H, int N, int d, float scale, int causal,
           const int32_t* cu_seqlens, int total_tokens, int dtype,
           void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * The three stages of fa_bwd, callable one at a time (same arguments and
 * rules as fa_bwd; each returns after launching its kernel).  Calling
 * preprocess, main and postprocess in order on one stream is fa_bwd.
 *   preprocess  D_i = Σ_c dO_ic·O_ic (fp32) and a zeroed fp32 dQ accumulator
 *   main        per key tile: recompute Sᵀ and Pᵀ, accumulate dV, dK in tensor
 *               memory and write them; add dQ partial sums into the accumulator
 *   postprocess dq = scale · accumulator, rounded to the dtype
 */
int fa_bwd_preprocess(const void* o, const void* dO, int B, int H, int N, int d,
                      const int32_t* cu_seqlens, int total_tokens, int dtype,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream);
int fa_bwd_main(const void* q, const void* k, const void* v, const float* lse,
                const void* dO, void* dk, void* dv,
                int B, int H, int N, int d, float scale, int causal,
                const int32_t* cu_seqlens, int total_tokens, int dtype,
                void* workspace, size_t workspace_bytes, fa_stream_t stream);
int fa_bwd_postprocess(void* dq, int B, int H, int N, int d, float scale,
                       const int32_t* cu_seqlens, int total_tokens, int dtype,
                       void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Size in bytes of the library's static device scratch used by fa_bwd_noalloc
 * (32 MiB, held by every GPU that loads the library until the process exits).
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * fa_bwd without a caller-provided workspace.  The method's pages have no
 * counterpart: this exists for callers that cannot allocate device memory —
 * a plugin whose host engine owns all of the GPU's memory and passes it only
 * input and output buffers, or code that must not call cudaMalloc (it can
 * synchronise the device and can fail under a fixed memory budget).
 * Arguments and results as for fa_bwd, minus workspace and workspace_bytes;
 * the dQ accumulator and D live in a static device array of
 * FA_NOALLOC_SCRATCH_BYTES inside the library.  Nothing is allocated or freed.
 *   - Returns FA_ERR_UNSUPPORTED, launching nothing, when the problem needs more
 *     scratch than that.  The rule is exactly fa_bwd_workspace_bytes(total_tokens,
 *     H, d) <= FA_NOALLOC_SCRATCH_BYTES, which holds up to total_tokens·H =
 *     floor(FA_NOALLOC_SCRATCH_BYTES / (4·d + 4)) token-heads: 65,027 at
 *     d = 128 and 129,055 at d = 64.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents (the first kernel of every call zeroes what must start at zero).
 *     Calls whose kernels overlap on the GPU — e.g. on two streams with no
 *     ordering between them — race on the array and give wrong results.
 *   - Every call looks up the array's device address in the CUDA context that
 *     is current on the calling thread (a __device__ array has one copy per
 *     context), so callers on a non-primary context, or after cudaDeviceReset,
 *     get their own context's array.  The first lookup in a context may load
 *     the library's device code into it; make that first call before any
 *     stream capture.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal,
                   const int32_t* cu_seqlens, int total_tokens, int dtype, fa_stream_t stream);

/*
 * Dropout on the attention probabilities (the dropout_p of the SDPA
 * interface, "Flash Attention 优化", SDPA signature): the forward uses
 * O = (M ∘ P / (1 − p̂)) V with a keep mask M drawn inside the kernels, and
 * the backward draws the same mask again instead of storing it.  LSE is that
 * of the undropped softmax.  Otherwise as fa_fwd / fa_bwd.
 *   dropout_p  in [0, 1); the decisions compare one random byte with
 *              t = round(256·dropout_p) (clamped to 255): an element is kept
 *              when the byte ≥ t, so p̂ = t/256 and kept probabilities are
 *              scaled by 256/(256 − t).  t = 0 gives exactly fa_fwd / fa_bwd.
 *   seed       64-bit key of the generator; offset  its fourth counter word
 *              (advance it between calls that must draw different masks).
 * Mask of element (query i, key j), positions counted from the start of the
 * sequence, of sequence b and head h: byte (j mod 4) of output word (i mod 4)
 * of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011) with counter
 * (j/4, i/4, b·H + h, offset) and key (seed low 32 bits, seed high 32 bits).
 * fa_bwd_dropout needs the same dropout_p, seed and offset as the forward.
 * Errors as for fa_fwd / fa_bwd; dropout_p outside [0, 1) or NaN returns
 * FA_ERR_INVALID_ARG.
 */
int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal,
                   const int32_t* cu_seqlens, int total_tokens, int dtype,
                   float dropout_p, uint64_t seed, uint32_t offset, fa_stream_t stream);
int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal,
                   const int32_t* cu_seqlens, int total_tokens, int dtype,
                   float dropout_p, uint64_t seed, uint32_t offset,
                   void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Forward with 8-bit floating-point inputs (the FP8 path the pages credit to
 * FlashAttention-3, "Flash Attention 优化", 工程实践 "精度"): q, k, v are
 * e4m3 (OCP FP8 E4M3: 1 sign, 4 exponent, 3 mantissa bits, bias 7, no
 * infinities, ±448 largest), one byte per element, in the [T, H, d] layout
 * of fa_fwd; the real value of an element is its e4m3 value × the tensor's
 * descale.  Computes what fa_fwd computes for the real values: the descales
 * of q and k are folded into the softmax scale, v's multiplies O at the end.
 * The probabilities P are rounded to e4m3 before the P·V product (rows whose
 * keys fit in one 128-key tile carry P as the sum of two e4m3 parts), the
 * scores, the softmax statistics and O accumulate in fp32.
 *   o     bf16 [T, H, d] (written); lse  fp32 [T, H] as for fa_fwd.
 *   q_descale, k_descale, v_descale  finite and > 0.
 * d must be 128 (FA_ERR_UNSUPPORTED otherwise).  Other errors as fa_fwd; a
 * descale that is not finite and positive, or a scale·q_descale·k_descale
 * that is not, returns FA_ERR_INVALID_ARG.  No backward: the e4m3 path is
 * for inference.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int H, int N, int d, float scale, int causal,
               const int32_t* cu_seqlens, int total_tokens,
               float q_descale, float k_descale, float v_descale, fa_stream_t stream);

/*
 * fa_fwd_fp8 with one descale per (sequence, head) instead of per tensor:
 * q_descale, k_descale, v_descale are fp32 device arrays [B·H] (index b·H + h,
 * b the sequence), 4-byte aligned, read by the kernel (values are not
 * checked on the host: each must be finite and > 0, else the output is
 * undefined).  The descales of (b, h) are folded into that unit's softmax
 * constant and output factor, exactly as the per-tensor ones are.  Errors as
 * fa_fwd_fp8 (a null or misaligned descale array: FA_ERR_INVALID_ARG).
 */
int fa_fwd_fp8_per_head(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int N, int d, float scale, int causal,
                        const int32_t* cu_seqlens, int total_tokens,
                        const float* q_descale, const float* k_descale, const float* v_descale,
                        fa_stream_t stream);

/*
 * fa_fwd_fp8 with one descale per (128-token block, head): the blocks of a
 * sequence are its tokens [128i, 128i + 128) (the last one ragged), numbered
 * sequence after sequence, so block i of sequence b is number
 * n_b + i with n_b = Σ_{b' < b} ceil(L_b' / 128) (dense: b·ceil(N/128) + i).
 * q_descale, k_descale, v_descale are fp32 device arrays [num_blocks·H],
 * index (n_b + i)·H + h, 4-byte aligned, read by the kernel (values are not
 * checked on the host: each must be finite and > 0, else the output is
 * undefined).  The real value of element (token, h, c) is its e4m3 value ×
 * the descale of its block and head.
 * A query tile is one block, so q's descale is folded into its softmax
 * constant; k's is folded into the constant of each key tile; v's enters the
 * exponent of each key tile's P as log2(v descale), so the rounded P already
 * carries it, and the softmax sum takes each tile's P divided by it (the row
 * maximum tracked is that of scale·s + log2 v descale, which keeps every P
 * ≤ 256 and leaves O = Σ P V / Σ P unchanged).
 *   num_blocks  the arrays' length / H: ≥ B·ceil(N/128) for a dense batch
 *               (FA_ERR_INVALID_ARG otherwise); with cu_seqlens each
 *               sequence is checked on the device, and one whose blocks
 *               would lie past num_blocks is skipped and reported as
 *               inconsistent offsets are (fa_check_device_status).
 * Other errors as fa_fwd_fp8_per_head.
 */
int fa_fwd_fp8_per_block(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int N, int d, float scale, int causal,
                         const int32_t* cu_seqlens, int total_tokens,
                         const float* q_descale, const float* k_descale, const float* v_descale,
                         int num_blocks, fa_stream_t stream);

/*
 * Merge of normalised partial attention results: the same queries attended
 * to disjoint key sets (the blocks a ring of ranks visits in ring /
 * context-parallel attention, "FlashAttention 与算子融合", 工程实践 "与 CP
 * 配合"), combined one part at a time by the block-merge rule of the same
 * page ("FlashAttention 的两个关键", online softmax) written for normalised
 * parts:  LSE' = ln(e^LSE_acc + e^LSE_b),
 *         O'   = e^(LSE_acc − LSE')·O_acc + e^(LSE_b − LSE')·O_b.
 * A part with LSE = −∞ (no key) changes nothing.
 *   acc_o     fp32 [T, H, d], the running O (read unless first; written
 *             unless out is given).
 *   acc_lse   fp32 [T, H], the running LSE (read unless first; always
 *             written with the merged LSE).
 *   part_o    dtype [T, H, d] and part_lse fp32 [T, H]: the part, as fa_fwd
 *             writes them.
 *   out       NULL, or dtype [T, H, d]: the merged O is written here (rounded
 *             to nearest even) instead of into acc_o — for the last part.
 *   first     1: the running result is just this part (acc_o, acc_lse are
 *             not read).
 * acc_o, part_o, out 16-byte aligned, the LSE arrays 4-byte aligned; d ∈
 * {64, 128}; errors as fa_fwd (FA_ERR_INVALID_ARG for bad arguments,
 * FA_ERR_CUDA for a failed launch).  Asynchronous on `stream`.
 */
int fa_attn_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, void* out,
                  int T, int H, int d, int dtype, int first, fa_stream_t stream);

/*
 * Accumulation of gradient partials (the ring backward: the dK and dV
 * contributions of each rank to a key/value shard add up in fp32 as the
 * shard travels): over n elements,
 *   v = (first ? 0 : acc[i]) + (part ? part[i] : 0);
 *   out ? out[i] = dtype(v) (nearest even) : acc[i] = v.
 *   acc   fp32 [n], 16-byte aligned; part, out  dtype [n] or NULL, 16-byte
 *   aligned; n a positive multiple of 8.
 * FA_ERR_INVALID_ARG for bad arguments, FA_ERR_CUDA for a failed launch.
 * Asynchronous on `stream`.
 */
int fa_accumulate(float* acc, const void* part, void* out, long long n, int dtype, int first,
                  fa_stream_t stream);

/*
 * Decode: one new query token per sequence attends to every key of its
 * sequence in a K/V cache (token-by-token generation, the workload
 * "FlashAttention 短片讲解稿", segment "适用范围与关键结论", sets apart from
 * training and prefill).  No mask: every cached key precedes or is the
 * current token.
 *   q, o       [B, H, d], one row per sequence (same dtype as k and v).
 *   k, v       [total_keys, H, d]: sequence b's keys are rows
 *              [cu_seqlens_k[b], cu_seqlens_k[b+1]) of a device int32
 *              cu_seqlens_k (B+1 entries), or rows [b·Nk, (b+1)·Nk) when
 *              cu_seqlens_k == NULL (total_keys must then equal B·Nk).  Nk
 *              bounds every sequence's key count.
 *   lse        fp32 [B, H], natural-log log-sum-exp of the scaled scores; a
 *              sequence with no key gets o = 0 and lse = −inf.
 * The keys of each (sequence, head) are split into chunks of 512 that are
 * reduced in parallel to partial (max, sum, output) triples in `workspace`
 * (device memory the caller owns, 256-byte aligned, at least
 * fa_decode_workspace_bytes(B, H, Nk, d) bytes); a second kernel merges them
 * with the block-merge rule of "FlashAttention 与算子融合" ("FlashAttention 的两个
 * 关键": max of the maxima, sums and partial outputs rescaled to it).
 * Arithmetic in fp32 on the CUDA cores (the single query makes this a stream
 * over the cache, bound by memory bandwidth).  Errors as for fa_fwd; B and H
 * above 65535 return FA_ERR_UNSUPPORTED.  The two kernels are enqueued on
 * `stream`; nothing is allocated or synchronised.
 */
size_t fa_decode_workspace_bytes(int B, int H, int Nk, int d);
int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse,
              int B, int H, int Nk, int d, float scale, const int32_t* cu_seqlens_k,
              int total_keys, int dtype, void* workspace, size_t workspace_bytes,
              fa_stream_t stream);

/*
 * Synchronises `stream`, returns the device status word (FA_OK, or the first
 * FA_ERR_TIMEOUT / FA_ERR_INVALID_ARG a kernel recorded since the last call)
 * and clears it.  Returns FA_ERR_CUDA if the synchronisation itself failed.
 */
int fa_check_device_status(fa_stream_t stream);

/* Sets the watchdog limit of every later launch, in nanoseconds of device
 * time one wait may take (default 4e9).  Values below 1e6 are raised to 1e6. */
void fa_set_watchdog_ns(uint64_t ns);

/*
 * Self-test of the watchdog: launches one block that waits on a barrier no
 * thread ever completes, under a limit of `timeout_ns`.  The wait gives up,
 * the kernel records FA_ERR_TIMEOUT and returns.  Returns the status read
 * back by fa_check_device_status (FA_ERR_TIMEOUT when the watchdog works).
 */
int fa_watchdog_selftest(uint64_t timeout_ns, fa_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* fa_status_string(int status);

/* Library version string (static). */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
