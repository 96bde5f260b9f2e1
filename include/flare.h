/*
 * flare.h -- C ABI of the FLARE / FLARE++ token-mixing library for B200
 * (sm_100a).
 *
 * The operator (per batch b and head h, scale s, softmax in fp32):
 *   encode  Z = softmax_N(s Q K^T) V      -- "Flare Fast Low Rank Attention"
 *           skill page, section 2 "Implement Encode Stage" and section 4
 *           (latents are the queries, the sequence gives keys and values);
 *   decode  Y = softmax_M(s K Q^T) Z      -- FLARE arXiv 2508.12594 abstract:
 *           the second of two SDPA calls, giving an input-input mixing matrix
 *           W = softmax(s K Q^T) softmax(s Q K^T) of rank at most M;
 *   FLARE++ Q_dyn = Q + encode(Q, K, V), then encode and decode with Q_dyn
 *           -- FLARE++ arXiv 2608.11519 abstract (input-conditioned queries
 *           that correct the learned ones);
 *   backward: gradients of sum(Y * dY) with respect to Q, K, V.  The pages
 *           give none; it is the chain rule through both softmax stages,
 *           with the logits recomputed.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer to contiguous row-major data
 *     (token tensors may instead be strided: the *_ex calls), 16-byte
 *     aligned.  Shapes:
 *       Q        [H,M,D] when q_batch_stride == 0 (learned latents shared by
 *                the batch) or [B,H,M,D] when q_batch_stride == H*M*D;
 *       K, V, Y, dY, dK, dV   [B,H,N,D];
 *       Z_save   [B,H,M,D] float32;   lse_save  [B,H,M] float32 (natural log
 *                of the encode softmax denominators, max included);
 *       Q_dyn_out [B,H,M,D] in the input dtype.
 *   - dtype: FLARE_F32 or FLARE_BF16 for Q, K, V, Y, dY, dQ, dK, dV.  All
 *     arithmetic accumulates in float32; bf16 operands feed the tensor cores.
 *   - Supported sizes: B, H >= 1; N >= 1; D in {16, 32}; M a multiple of 16
 *     in [16, 256]; B*H*N*D < 2^40; B*H <= 65535 (one grid row per head;
 *     larger products return FLARE_ERR_UNSUPPORTED).  scale must be finite
 *     and > 0.
 *   - The caller owns every buffer.  The library never allocates or frees
 *     memory and never synchronises the device (flare_device_status is the
 *     one exception and says so; flare_fwd_host creates and releases CUDA
 *     events to order its two streams).  Work is enqueued on `stream` (a
 *     cudaStream_t; NULL = legacy default stream).
 *   - `workspace` is caller-allocated device memory of at least
 *     flare_workspace_size(op, ...) bytes, 256-byte aligned.  Its contents
 *     need no initialisation and are scratch between calls, except that
 *     flare_encode -> flare_combine -> flare_decode pass their intermediate
 *     results through it.  Two calls that run concurrently must not share a
 *     workspace.
 *   - Errors are returned, never thrown.  All arguments are validated
 *     before anything is enqueued, so a call that returns an error other
 *     than FLARE_ERR_CUDA has no side effect.  FLARE_ERR_CUDA means a launch
 *     failed; the CUDA error is left for cudaGetLastError.
 *   - Every wait inside a kernel is bounded.  A wait that runs out sets an
 *     error word in the workspace header instead of hanging; read it with
 *     flare_device_status after the stream has been synchronised.
 *   - The library is thread-safe and holds no mutable global state, with
 *     one exception: flare_fwd_noalloc's fixed device scratch array (one per
 *     device) and the cache of its per-device address, described with that
 *     call below.
 */
#ifndef FLARE_H_
#define FLARE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLARE_API __attribute__((visibility("default")))
#else
#define FLARE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FLARE_F32 = 0, FLARE_BF16 = 1 } flare_dtype_t;

typedef enum {
  FLARE_OK = 0,
  FLARE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or scale */
  FLARE_ERR_UNSUPPORTED = 2,   /* valid but unsupported D, M or stride      */
  FLARE_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
  FLARE_ERR_CUDA = 4,          /* a kernel launch failed                    */
  FLARE_ERR_DEVICE_TIMEOUT = 5 /* a kernel's bounded wait ran out           */
} flare_status_t;

typedef enum {
  FLARE_OP_FWD = 0,
  FLARE_OP_PP_FWD = 1,
  FLARE_OP_BWD = 2,
  FLARE_OP_PP_BWD = 3
} flare_op_t;

/*
 * Layout of one token tensor (K, V, Y, dY, dK or dV) of logical shape
 * [B,H,N,D] whose head dimension D is contiguous: element (b, h, n, d) sits
 * at element offset b*b_stride + h*h_stride + n*n_stride + d from the base
 * pointer.  Contiguous [B,H,N,D] is {H*N*D, N*D, D}; the layout of a fused
 * projection's output [B,N,H,D] is {N*H*D, D, H*D}.  Used by the *_ex entry
 * points.  Every stride must be >= 1, a multiple of 16 bytes and
 * below 2^40 bytes (else FLARE_ERR_INVALID_ARG, or FLARE_ERR_UNSUPPORTED for
 * a stride that is not a multiple of 16 bytes).  The rows of an output
 * tensor must not overlap (checked: in order of stride, each dimension with
 * more than one index must step over all rows of the dimensions inside it;
 * else FLARE_ERR_INVALID_ARG); inputs may share or overlap rows.
 */
typedef struct {
  int64_t b_stride, h_stride, n_stride;
} flare_strides_t;

/* Library ABI version (major*10000 + minor*100 + patch). */
FLARE_API int flare_version(void);

/*
 * Description of the last FLARE_ERR_CUDA returned on the calling host thread
 * (the failing call and the CUDA error name), or of a size rejection by
 * flare_fwd_noalloc, or "" if none.  Thread-local
 * storage, valid until the next FLARE call on this thread.
 */
FLARE_API const char* flare_last_error_detail(void);

/* Human-readable text for a status code (static storage, never NULL). */
FLARE_API const char* flare_status_string(flare_status_t status);

/*
 * Bytes of workspace needed by `op` for these sizes on the current device,
 * or 0 when the sizes are invalid or unsupported.  The stage calls
 * flare_encode / flare_combine / flare_decode use FLARE_OP_FWD's size.
 */
FLARE_API size_t flare_workspace_size(flare_op_t op, int64_t B, int64_t H, int64_t N, int64_t M,
                            int64_t D, flare_dtype_t dtype);

/*
 * FLARE forward from and to HOST memory: Q, K, V are copied in and Y is
 * copied out by the library, overlapped with the compute.  The heads go in
 * about 16 chunks (each inside one batch element): a chunk's K and V are
 * copied in on `copy_stream` while `stream` runs the previous chunk's
 * forward and copies its Y out, so the call takes about as long as its
 * host-to-device copies.  Q_host / K_host / V_host / Y_host: host memory
 * (page-locked for the copies to overlap), laid out as flare_fwd's device
 * tensors; Q_dev, K_dev, V_dev, Y_dev: caller-owned device buffers of the
 * same sizes, overwritten.  workspace: flare_fwd_host_workspace_size bytes.
 * Everything is ordered after the work already on `stream`, and the call's
 * results (Y_host) are complete once `stream` is: synchronise `stream`
 * before reading Y_host.  copy_stream may equal stream (no overlap).
 * Returns the codes of flare_fwd; the device error word is read with
 * flare_device_status on the workspace.
 */
FLARE_API flare_status_t flare_fwd_host(const void* Q_host, int64_t q_batch_stride,
                                        const void* K_host, const void* V_host, void* Y_host,
                                        void* Q_dev, void* K_dev, void* V_dev, void* Y_dev,
                                        int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                        flare_dtype_t dtype, float scale, void* workspace,
                                        size_t workspace_bytes, void* stream, void* copy_stream);

/* Bytes of workspace flare_fwd_host needs (0 for invalid sizes). */
FLARE_API size_t flare_fwd_host_workspace_size(int64_t B, int64_t H, int64_t N, int64_t M,
                                               int64_t D, flare_dtype_t dtype);

/*
 * FLARE forward: Y = decode(Q, K, encode(Q, K, V)).
 * Q, K, V in; Y out.  Z_save / lse_save are optional (NULL for inference)
 * and are what flare_bwd needs.  Equivalent to flare_encode, flare_combine
 * and flare_decode in sequence on the same workspace.
 */
FLARE_API flare_status_t flare_fwd(const void* Q, int64_t q_batch_stride, const void* K, const void* V,
                         void* Y, int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                         flare_dtype_t dtype, float scale, float* Z_save, float* lse_save,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * FLARE++ forward with learned latents Q [H,M,D] (FLARE++ abstract):
 *   Q_dyn = Q + encode(Q, K, V);  Z = encode(Q_dyn, K, V);  Y = decode(Q_dyn, K, Z).
 * Q_dyn is rounded to the input dtype before it is used (it is the operand
 * of both later stages).  Q_dyn_out (optional) receives it; Z_save and
 * lse_save (optional) receive the second encode's Z and lse.
 */
FLARE_API flare_status_t flare_pp_fwd(const void* Q, const void* K, const void* V, void* Y,
                            void* Q_dyn_out, int64_t B, int64_t H, int64_t N, int64_t M,
                            int64_t D, flare_dtype_t dtype, float scale, float* Z_save,
                            float* lse_save, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * FLARE backward (fixed latents): gradients of sum(Y * dY).
 * Inputs: Q, K, V, dY and the forward's Z_save, lse_save (both required).
 * Outputs in the input dtype: dQ ([H,M,D] summed over the batch when
 * q_batch_stride == 0, else [B,H,M,D]), dK, dV.  The logits of both stages
 * are recomputed; every reduction is in a fixed order, so results are
 * bitwise reproducible run to run.  With bf16, M in {128, 256} and D in
 * {16, 32} the work runs on the tensor cores: the decode-stage softmax and
 * dZ (one pass over the tokens with M = 128; with M = 256 a statistics pass
 * and a dZ pass), then dK, dV and dQ with one exponential per token-latent
 * pair (once per 128-latent half); other sizes use CUDA-core kernels.
 */
FLARE_API flare_status_t flare_bwd(const void* Q, int64_t q_batch_stride, const void* K, const void* V,
                         const void* dY, const float* Z_save, const float* lse_save, void* dQ,
                         void* dK, void* dV, int64_t B, int64_t H, int64_t N, int64_t M,
                         int64_t D, flare_dtype_t dtype, float scale, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * FLARE++ backward with learned latents Q [H,M,D] (FLARE++ abstract: the
 * encoder's M outputs correct the learned queries, and the corrected
 * queries drive both compression and redistribution):
 *   Q_dyn = Q + encode(Q, K, V),  Y = FLARE(Q_dyn, K, V).
 * Gradients of sum(Y * dY): FLARE's backward with the per-batch latents
 * Q_dyn, then the first encode's backward with upstream gradient dQ_dyn;
 * dQ [H,M,D] is summed over the batch.  Inputs: Q, K, V, dY, the forward's
 * Q_dyn ([B,H,M,D], input dtype) and its Z_save / lse_save (the second
 * encode's).  The first encode is recomputed; Q_dyn's rounding to the
 * input dtype is treated as the identity.  Outputs dQ, dK, dV in the input
 * dtype.  Workspace: flare_workspace_size(FLARE_OP_PP_BWD, ...).  Every
 * reduction is in a fixed order (bitwise reproducible).
 */
FLARE_API flare_status_t flare_pp_bwd(const void* Q, const void* K, const void* V, const void* dY,
                            const void* Q_dyn, const float* Z_save, const float* lse_save,
                            void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t N,
                            int64_t M, int64_t D, flare_dtype_t dtype, float scale,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * The four entry points above, extended:
 *
 * `strides` -- token tensors in any layout that flare_strides_t describes
 * (for example [B,N,H,D] straight from a fused QKV projection, with no
 * transpose).  It points to one flare_strides_t per token tensor, in this
 * order:  *_fwd_ex: K, V, Y;   *_bwd_ex: K, V, dY, dK, dV.  NULL means
 * every token tensor is contiguous [B,H,N,D].  Latent tensors (Q, Q_dyn,
 * dQ, Z_save, lse_save) stay contiguous; outputs must not alias inputs.
 *
 * `seq_lens` -- variable sequence lengths (a key-padding mask for
 * right-padded batches; the FLARE skill page's module takes an attention
 * mask): a DEVICE array of B int32 values, 4-byte aligned.  Batch element b
 * has seq_lens[b] valid tokens; tokens n >= seq_lens[b] are padding, whose
 * values are never read.  The encode's softmax runs over the valid tokens
 * only; Y is 0 at padding; dK and dV are 0 at padding and padding adds
 * nothing to dQ.  A sequence with no tokens encodes to Z = 0 with
 * lse = -inf (Z_save, lse_save), Y = 0.  Values outside [0, N] are clamped
 * to it and reported: flare_device_status then returns
 * FLARE_ERR_INVALID_ARG with detail 0x601.  NULL means every sequence has
 * N tokens.  flare_pp_bwd_ex / flare_bwd_ex must get the lengths their
 * forward used.  On the tensor-core path a call with lengths first has one
 * block read them and write a work plan into the workspace (a kernel of
 * its own in the forward, a block of the first kernel in the backward):
 * each head's valid tiles split into near-equal units, one CTA each, so
 * that short sequences take less time instead of leaving SMs idle (no host
 * synchronisation; the workspace size already covers it).
 *
 * With strides == NULL and seq_lens == NULL each call is the plain entry
 * point (which is implemented that way).
 */
FLARE_API flare_status_t flare_fwd_ex(const void* Q, int64_t q_batch_stride, const void* K,
                                      const void* V, void* Y, const flare_strides_t* strides,
                                      const int32_t* seq_lens, int64_t B, int64_t H, int64_t N,
                                      int64_t M, int64_t D, flare_dtype_t dtype, float scale,
                                      float* Z_save, float* lse_save, void* workspace,
                                      size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_pp_fwd_ex(const void* Q, const void* K, const void* V, void* Y,
                                         void* Q_dyn_out, const flare_strides_t* strides,
                                         const int32_t* seq_lens, int64_t B, int64_t H,
                                         int64_t N, int64_t M, int64_t D, flare_dtype_t dtype,
                                         float scale, float* Z_save, float* lse_save,
                                         void* workspace, size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_bwd_ex(const void* Q, int64_t q_batch_stride, const void* K,
                                      const void* V, const void* dY, const float* Z_save,
                                      const float* lse_save, void* dQ, void* dK, void* dV,
                                      const flare_strides_t* strides, const int32_t* seq_lens,
                                      int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                      flare_dtype_t dtype, float scale, void* workspace,
                                      size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_pp_bwd_ex(const void* Q, const void* K, const void* V,
                                         const void* dY, const void* Q_dyn, const float* Z_save,
                                         const float* lse_save, void* dQ, void* dK, void* dV,
                                         const flare_strides_t* strides, const int32_t* seq_lens,
                                         int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                         flare_dtype_t dtype, float scale, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * Stage 1 of the forward -- encode partials.  For each (b, h) and each
 * chunk of tokens, the running softmax max m, denominator l and weighted
 * value sum acc of every latent row (skill page section 2; online softmax
 * across token tiles).  Results stay in the workspace.
 */
FLARE_API flare_status_t flare_encode(const void* Q, int64_t q_batch_stride, const void* K, const void* V,
                            int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                            flare_dtype_t dtype, float scale, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Stage 2 -- merge the chunk partials of flare_encode (log-sum-exp merge):
 * Z = sum_c acc_c 2^(m_c - m*) / sum_c l_c 2^(m_c - m*).  Writes Z to the
 * workspace (float32 and the bf16 operand copy used by the decode) and, when
 * non-NULL, to Z_save and lse_save.  Must follow flare_encode with the same
 * sizes, dtype and workspace.
 */
FLARE_API flare_status_t flare_combine(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                             flare_dtype_t dtype, float* Z_save, float* lse_save,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 3 -- decode: Y = softmax_M(s K Q^T) Z with the Z that flare_combine
 * left in the workspace (FLARE abstract, second SDPA call).  The N x M
 * logits never leave the chip.
 */
FLARE_API flare_status_t flare_decode(const void* Q, int64_t q_batch_stride, const void* K, void* Y,
                            int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                            flare_dtype_t dtype, float scale, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Context parallelism: the N tokens of every (b, h) split into equal shards,
 * one per device (the FLARE++ page: sharding the input tokens across
 * devices without gathering the sequence).  The encode's chunk records are
 * the only exchange in the forward; the backward exchanges dZ and dQ.
 * Every shard passes its own token count as N, the same on every device,
 * contiguous token tensors and no sequence lengths.
 *
 * Forward, per device:
 *   1. flare_encode on the device's shard (records land in the workspace);
 *   2. flare_records_layout: where they are -- records_per_bh R, and the
 *      byte offsets of ml [B*H][R][M][2] and acc [B*H][R][M][D] (float32)
 *      in the workspace;
 *   3. the caller gathers every shard's ml and acc, in shard order, into
 *      [shards][B*H][R][M][2] and [shards][B*H][R][M][D] (e.g. NCCL
 *      all-gather);
 *   4. flare_combine_shards merges them (fixed order: shard by shard) into
 *      the Z of the whole sequence, in the workspace and in Z_save / lse_save;
 *   5. flare_decode on the device's shard.
 * Backward, per device (Z_save, lse_save: the whole sequence's, from step 4):
 *   1. flare_bwd_shard_dz: the decode stage over the shard's tokens; writes
 *      the shard's part of dZ (float32 [B,H,M,D]);
 *   2. the caller sums the parts over the shards (e.g. NCCL all-reduce);
 *   3. flare_bwd_shard_finish on the same workspace: the shard's rows of dK
 *      and dV, and its part of dQ (float32, [H,M,D] summed over the batch
 *      when q_batch_stride == 0, else [B,H,M,D]) to be summed over the
 *      shards.
 * flare_bwd_shard_finish keeps the device error word of the first half.
 *
 * FLARE++ (learned latents Q [H,M,D]):
 *   forward: the steps above for the first encode, with Q_learned = Q and
 *   Q_dyn_out given to flare_combine_shards (which then also writes
 *   Q_dyn = Q + Z1, [B,H,M,D] in the input dtype), then the steps above with
 *   Q_dyn as per-batch latents;
 *   backward: the first encode recomputed as in the forward (its Z1, lse1 of
 *   the whole sequence into Z_save / lse_save); the backward steps above with
 *   Q_dyn, on a FLARE_OP_PP_BWD workspace, giving dQ_dyn after the sum over
 *   the shards; then flare_pp_bwd_shard_tail with that dQ_dyn (input dtype)
 *   on the same workspace: the first encode's gradient over the shard, added
 *   to the shard's dK and dV, and its float32 part of dQ [H,M,D] (summed
 *   over the batch).  Exactly one shard passes add_dq_dyn = 1, which adds
 *   the sum over the batch of dQ_dyn to its part (the others pass 0), so
 *   that dQ = the sum over the shards of the parts.
 */
FLARE_API flare_status_t flare_records_layout(int64_t B, int64_t H, int64_t N, int64_t M,
                                              int64_t D, flare_dtype_t dtype,
                                              int64_t* records_per_bh, size_t* ml_offset,
                                              size_t* acc_offset);
FLARE_API flare_status_t flare_combine_shards(int64_t shards, const float* ml, const float* acc,
                                              int64_t records_per_bh, int64_t B, int64_t H,
                                              int64_t N, int64_t M, int64_t D,
                                              flare_dtype_t dtype, float* Z_save,
                                              float* lse_save, const void* Q_learned,
                                              void* Q_dyn_out, void* workspace,
                                              size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_bwd_shard_dz(const void* Q, int64_t q_batch_stride, const void* K,
                                            const void* V, const void* dY, const float* Z_save,
                                            const float* lse_save, float* dZ_part, int64_t B,
                                            int64_t H, int64_t N, int64_t M, int64_t D,
                                            flare_dtype_t dtype, float scale, void* workspace,
                                            size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_pp_bwd_shard_tail(const void* Q, const void* K, const void* V,
                                                 const float* Z1, const float* lse1,
                                                 const void* dQ_dyn, int add_dq_dyn,
                                                 float* dQ_part, void* dK,
                                                 void* dV, int64_t B, int64_t H, int64_t N,
                                                 int64_t M, int64_t D, flare_dtype_t dtype,
                                                 float scale, void* workspace,
                                                 size_t workspace_bytes, void* stream);
FLARE_API flare_status_t flare_bwd_shard_finish(const void* Q, int64_t q_batch_stride,
                                                const void* K, const void* V, const void* dY,
                                                const float* Z_save, const float* lse_save,
                                                const float* dZ, float* dQ_part, void* dK,
                                                void* dV, int64_t B, int64_t H, int64_t N,
                                                int64_t M, int64_t D, flare_dtype_t dtype,
                                                float scale, void* workspace,
                                                size_t workspace_bytes, void* stream);

/*
 * Size of the fixed scratch array behind flare_fwd_noalloc (32 MiB).  Every
 * GPU that loads this library holds one such array until the process exits.
 */
#define FLARE_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * FLARE forward for callers that cannot allocate device memory -- a plugin
 * inside a framework that owns every device allocation and passes its
 * plugins no workspace, or a running latency-critical loop where cudaMalloc
 * (which can synchronise the device) is not allowed.  The papers have no
 * counterpart to this call; it is an interface convenience.
 *
 * Same arguments, layouts and results as flare_fwd, minus the workspace:
 * the scratch lives in a file-scope device array of
 * FLARE_NOALLOC_SCRATCH_BYTES bytes.  The call allocates and frees nothing.
 * Sizes whose flare_workspace_size(FLARE_OP_FWD, ...) exceeds that limit
 * are rejected with FLARE_ERR_WORKSPACE before anything is enqueued
 * (flare_last_error_detail says why); use flare_fwd for them.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it per device
 * and context (a context made after cudaDeviceReset is looked up again);
 * make that first call before any stream capture.  All calls on a device
 * share the array: calls whose work overlaps on the GPU (other streams or
 * host threads, same device) race on it and must be serialised by the
 * caller.  A bounded wait that runs out inside one of these calls sets the
 * error word at the start of the array; read it with
 * flare_noalloc_device_status.
 */
FLARE_API flare_status_t flare_fwd_noalloc(const void* Q, int64_t q_batch_stride, const void* K,
                                           const void* V, void* Y, int64_t B, int64_t H,
                                           int64_t N, int64_t M, int64_t D, flare_dtype_t dtype,
                                           float scale, float* Z_save, float* lse_save,
                                           void* stream);

/*
 * flare_device_status for flare_fwd_noalloc's scratch array on the current
 * device: reads and clears its error word (SYNCHRONISES `stream`).  Same
 * return values and detail codes as flare_device_status.
 */
FLARE_API flare_status_t flare_noalloc_device_status(uint32_t* detail, void* stream);

/*
 * Reads and clears the device error word in the workspace header.  This
 * call SYNCHRONISES `stream`.  Returns FLARE_OK, FLARE_ERR_DEVICE_TIMEOUT
 * (a bounded wait ran out; *detail receives the site code),
 * FLARE_ERR_INVALID_ARG (a seq_lens value outside [0, N] was clamped;
 * detail 0x601) or FLARE_ERR_CUDA.  detail may be NULL.
 */
FLARE_API flare_status_t flare_device_status(void* workspace, size_t workspace_bytes, uint32_t* detail,
                                   void* stream);

/*
 * Which kernel family a forward call with these sizes uses:
 * 1 = tcgen05/TMEM/TMA tensor-core kernels, 0 = CUDA-core kernels.
 * Returns -1 for invalid or unsupported sizes.
 */
FLARE_API int flare_fwd_path(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dtype);

/*
 * Which kernel family flare_bwd uses for these sizes: 1 = the tcgen05
 * backward (bf16, M in {128, 256}, D in {16, 32}), 0 = CUDA-core kernels.
 * Returns -1 for invalid or unsupported sizes.
 */
FLARE_API int flare_bwd_path(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dtype);

/*
 * Measurement and self-test support.  Not part of the method: these calls
 * exist so that the roofline the library is measured against, the
 * hand-written exponential and the bounded waits can be checked on the
 * device itself.  Unlike the calls above, flare_probe_unit_rates
 * synchronises the device.
 */

/* Throughputs measured by flare_probe_unit_rates, per SM and per SM clock. */
typedef struct {
  int sms;                    /* multiprocessors of the current device          */
  double sm_mhz;              /* SM clock during the probes (clock64 against the
                                 global timer, mean over the probe kernels)     */
  double ex2_per_clk_sm;      /* ex2.approx.ftz.f32 results                     */
  double fma_per_clk_sm;      /* fp32 FMAs issued as fma.rn.f32                 */
  double fma2_per_clk_sm;     /* fp32 FMAs issued as packed fma.rn.f32x2 (2 each) */
  double mix_ex2_per_clk_sm;  /* ex2 results while 6 FMAs per ex2 also issue    */
  double mix_fma_per_clk_sm;  /* the FMAs of that mix                           */
  double ex2_ms, fma_ms, fma2_ms, mix_ms;  /* CUDA-event time of each probe     */
} flare_unit_rates_t;

/* Bytes of device scratch flare_probe_unit_rates needs (0 without a device). */
FLARE_API size_t flare_probe_scratch_bytes(void);

/*
 * Times four probe kernels on the current device (about 4 SM-resident CTAs
 * of 256 threads per SM, independent dependency chains): MUFU exponentials,
 * scalar FMAs, packed FMAs, and exponentials mixed with six FMAs each.
 * Rates are results per SM per SM clock, from CUDA-event times and the
 * clock the kernels saw.  scratch: device memory of at least
 * flare_probe_scratch_bytes() bytes, 16-byte aligned (the kernels' clock
 * records).  Runs on `stream` and SYNCHRONISES it.  Returns FLARE_OK,
 * FLARE_ERR_INVALID_ARG (NULL pointer), FLARE_ERR_WORKSPACE (scratch too
 * small or misaligned) or FLARE_ERR_CUDA.
 */
FLARE_API flare_status_t flare_probe_unit_rates(void* scratch, size_t scratch_bytes,
                                                flare_unit_rates_t* out, void* stream);

/*
 * SM clocks one tcgen05.mma of the kernels' shapes (kind::f16, bf16
 * operands, fp32 accumulator, M = 128, K = 16, N = n in {32, 48, 64, 128,
 * 256}) costs when `issuers` (1 to 4) threads of every SM issue 1024 of them
 * each, back to back, with the A operand in shared memory (a_in_tmem = 0) or
 * in TMEM (1): the median over the SMs of the slowest issuer's span divided
 * by all the SM's products.  With one issuer this is the issue latency of a
 * thread; with several, the SM's own cost of a product.  scratch: device
 * memory of at least flare_probe_scratch_bytes() bytes, 16-byte aligned.
 * Runs on `stream` and SYNCHRONISES it.  Returns FLARE_OK,
 * FLARE_ERR_INVALID_ARG (NULL pointer, issuers outside [1, 4]),
 * FLARE_ERR_UNSUPPORTED (another n, or n x issuers > 256),
 * FLARE_ERR_WORKSPACE, FLARE_ERR_DEVICE_TIMEOUT (a bounded wait ran out) or
 * FLARE_ERR_CUDA.
 */
FLARE_API flare_status_t flare_probe_mma_rate(int n, int a_in_tmem, int issuers, void* scratch,
                                              size_t scratch_bytes, double* clk_per_mma,
                                              void* stream);

/*
 * Share of the exponentials of the forward's encode (kernel 0) or decode
 * (kernel 1) that runs as the FMA-pipe polynomial instead of the MUFU, for
 * a forward call with these M, D and dtype (0 for the CUDA-core kernels,
 * which use exp2f).  The roofline of an exponential-bound kernel depends on
 * it: the MUFU then computes (1 - share) of the exponentials.
 */
FLARE_API flare_status_t flare_exp_split(int kernel, int64_t M, int64_t D, flare_dtype_t dtype,
                                         double* poly_fraction);

/*
 * y[i] = 2^x[i] for n floats (device pointers), with the exponential the
 * kernels use: form 0 = the MUFU instruction (ex2.approx.ftz.f32), form 1 =
 * the FMA-pipe polynomial evaluated one value at a time, form 2 = the same
 * polynomial in packed fp32x2 arithmetic, two values at a time (the form of
 * the backward's fixed-weight pass), form 3 = the packed polynomial with
 * the exponent clamped by a saturating FMA (the form the forward's softmax
 * loops use).  The polynomial: round-to-nearest range reduction x = j + f,
 * a degree-3 minimax fit of 2^f on [-1/2, 1/2] (relative error 7.5e-5), j
 * added to the exponent field.  Forms 1 and 2 are valid for x <= 126 and
 * clamp inputs below -125 to -125; form 3 clamps x to [-125, 126] and adds
 * at most 5.2e-6 relative error (the rounding of (x + 125) / 251).
 * Enqueued on `stream`.
 */
FLARE_API flare_status_t flare_eval_exp2(const float* x, float* y, int64_t n, int form,
                                         void* stream);

/*
 * Launches one CTA that waits, with the kernels' bounded wait, on an
 * mbarrier that nothing arrives on, for limit_ns nanoseconds (at most the
 * kernels' own limit of 1 s, else FLARE_ERR_INVALID_ARG); around the wait
 * it holds TMEM and a bulk copy of workspace bytes [256, 512) in flight,
 * as the FLARE kernels do.  When the wait runs out the kernel records site
 * 0x701 in the workspace error word, lets the copy land, frees TMEM and
 * returns: flare_device_status on the same workspace then returns
 * FLARE_ERR_DEVICE_TIMEOUT with detail 0x701, and the device stays usable.
 * workspace: device memory of at least 512 bytes, 256-byte aligned (the
 * error word is cleared first).  Enqueued on `stream`.
 */
FLARE_API flare_status_t flare_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                     uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLARE_H_ */
