/*
 * attn.h -- C ABI of libattn.so: exact scaled-dot-product attention on one
 * B200 (sm_100a), forward and backward.
 *
 * The operation is the one defined on the page "FlashAttention 核心原理"
 * (cxbdf.cn), part 1: Attention(Q, K, V) = softmax(Q K^T * scale) V, with an
 * optional causal mask.  It is computed tile by tile with an online softmax
 * (same page, part 2: tiling and kernel fusion), so the Nq x Nk score matrix is
 * never written to device memory.  The backward pass recomputes the attention
 * probabilities from the saved per-row log-sum-exp instead of storing them
 * (same page, part 2 item 3, "recomputation for the backward pass").  The
 * argument list follows the forward kernel interface sketched on the page
 * "FlashAttention-2 性能革命", section 2.1 (q, k, v, o, softmax_lse, seqlen_q,
 * seqlen_k, num_heads, softmax_scale) and the user call
 * flash_attn_func(q, k, v, softmax_scale, causal) of the same page, section 3.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Q, O, dO, dQ are contiguous [B][H][Nq][d]; K, V, dK, dV are
 *   contiguous [B][H][Nk][d]; LSE is contiguous [B][H][Nq] float.  Element
 *   type is fp16 or bf16 (attn_dtype) for every 16-bit tensor of one call;
 *   the FP8 calls take E4M3 Q, K, V and write bf16 O.
 * Memory.  Every pointer is a DEVICE pointer on the current CUDA device,
 *   16-byte aligned, allocated and owned by the caller, except the tensors
 *   of attn_host_step, which live in host memory.  The library keeps no
 *   allocation of its own between calls, except attn_bwd_noalloc's fixed
 *   scratch array and attn_host_step's two copy streams per device.
 * Stream.  `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *   call only enqueues work on it and returns without synchronising.
 * Mask.  `causal` is an attn_causal value; anything else returns
 *   ATTN_ERR_INVALID_ARG.  ATTN_CAUSAL_TOP_LEFT (1): query row i attends to
 *   key row j iff j <= i.  ATTN_CAUSAL_BOTTOM_RIGHT (2): iff j <= i + Nk - Nq,
 *   so the last query row sees every key (a block of new queries appended
 *   after Nk - Nq cached keys).  The two agree when Nq == Nk.  (The pages name
 *   a causal mask but not its alignment when Nq != Nk; top-left is the
 *   default reading, bottom-right the option.)  Keys that no query sees get
 *   dK = dV = 0.  A query row that sees no key (bottom-right with Nq > Nk:
 *   rows i < Nq - Nk) has an empty softmax: O = 0, LSE = -inf, dQ = 0.
 * LSE.  lse[b][h][i] = ln sum_j exp(scale * q_i . k_j) over the unmasked j:
 *   the natural-log row log-sum-exp of the scaled scores, in fp32.
 * Supported shapes.  d in {64, 128, 256} (the FP8 forward: 128 only); any
 *   Nq, Nk >= 0 (the kernels work in tiles of 128 rows, or 64 keys for the
 *   d = 256 backward, and mask a ragged last tile); causal with any Nq, Nk.
 *   The tile counts ceil(Nq / 128) and ceil(Nk / 128) must not exceed 65535,
 *   and B*H and B*H times each tile count must fit in an int (for the packed
 *   calls, with the longest sequence's tile counts); other shapes return
 *   ATTN_ERR_UNSUPPORTED.
 * Empty problems.  B, H, Nq or Nk may be 0.  A call with no query rows
 *   (B*H*Nq == 0) is valid and does nothing, except that attn_bwd then writes
 *   dK = dV = 0 (their rows exist but no query reaches them).  Nq > 0 with
 *   Nk == 0 asks for a softmax over no keys, which is undefined, and returns
 *   ATTN_ERR_INVALID_ARG.  Pointers of an empty tensor are not read and may
 *   be NULL.
 * Errors.  Arguments are validated on the host before anything is enqueued:
 *   a negative size, a NULL pointer or a pointer that is not 16-byte aligned
 *   (of a non-empty tensor) returns ATTN_ERR_INVALID_ARG; an unsupported shape
 *   or dtype returns ATTN_ERR_UNSUPPORTED; a failed launch returns
 *   ATTN_ERR_CUDA.  Nothing is
 *   written to any output when a call returns an error.  There is no fallback
 *   to another implementation.  Kernels never trap: a wait inside a kernel
 *   that exceeds its time limit makes the kernel record ATTN_ERR_TIMEOUT in a
 *   device status word and return early, and a kernel that finds less shared
 *   memory than its tiles need records ATTN_ERR_SMEM and returns without
 *   work; attn_last_device_status() reads the word.  An fp16 backward whose
 *   per-query terms leave the range the kernel can represent records
 *   ATTN_ERR_RANGE there (see attn_bwd).
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,
  ATTN_ERR_UNSUPPORTED = 2,
  ATTN_ERR_CUDA = 3,
  ATTN_ERR_TIMEOUT = 4,
  ATTN_ERR_SCRATCH_LIMIT = 5,
  ATTN_ERR_SMEM = 6,
  ATTN_ERR_RANGE = 7
} attn_status;

typedef enum { ATTN_FP16 = 0, ATTN_BF16 = 1 } attn_dtype;

/* Values of the `causal` argument (see Mask above). */
typedef enum {
  ATTN_CAUSAL_NONE = 0,
  ATTN_CAUSAL_TOP_LEFT = 1,
  ATTN_CAUSAL_BOTTOM_RIGHT = 2
} attn_causal;

/*
 * Forward pass.  Writes O = softmax(scale * Q K^T [+ causal mask]) V (16-bit,
 * round to nearest even) and LSE (fp32, see above).  The probabilities P are
 * rounded to the 16-bit input type before the product with V; all sums
 * accumulate in fp32.
 *   q, k, v   inputs, read only.
 *   o         output [B][H][Nq][d], 16-bit.
 *   lse       output [B][H][Nq], float.
 *   B, H      batch and head count (>= 0).
 *   Nq, Nk    query and key sequence lengths (>= 0; see Empty problems).
 *   d         head dimension.
 *   scale     multiplier of Q K^T; the pages use 1/sqrt(d).
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Nq, int Nk, int d, float scale, int causal,
                     attn_dtype dtype, void* stream);

/*
 * FP8 forward (page "Flash Attention 是什麼|為何更快又省 VRAM", section
 * "從 FA-1 到 FA-4": FlashAttention-3 adds an FP8 variant; the page gives no
 * method, so this is the plain per-tensor-scaled reading).  q, k, v hold
 * OCP E4M3 bytes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, 0x7F/0xFF NaN, largest finite 448) in the layout of attn_fwd,
 * and stand for descale_q * q, descale_k * k, descale_v * v.  Writes
 *   O   = softmax(scale * descale_q * descale_k * q k^T [+ causal mask])
 *         (descale_v * v), bf16 [B][H][Nq][d];
 *   LSE = the natural-log row log-sum-exp of those scaled scores, fp32.
 * Both products run on the 8-bit tensor path: the probabilities are
 * rounded to E4M3 (round to nearest even, saturating; relative error up
 * to 2^-4, values below 2^-10 of the running row maximum become 0) before
 * the product with V, and O is normalised by the sum of the rounded
 * probabilities.  d must be 128 (ATTN_ERR_UNSUPPORTED otherwise); a
 * descale factor or scale that is not finite returns ATTN_ERR_INVALID_ARG.
 * Sizes, masks, empty problems, alignment and errors as for attn_fwd.
 */
attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int Nq, int Nk, int d, float scale, float descale_q,
                         float descale_k, float descale_v, int causal, void* stream);

/*
 * FP8 forward of a packed variable-length batch: attn_fwd_varlen's layout,
 * offsets, masks and empty-sequence rules with attn_fwd_fp8's E4M3 inputs,
 * per-tensor descale factors, bf16 O and rounding.  d must be 128.
 */
attn_status attn_fwd_fp8_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                                int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                                float scale, float descale_q, float descale_k, float descale_v,
                                int causal, void* stream);

/*
 * Size in bytes of the device workspace attn_bwd and attn_bwd_deterministic
 * need: an fp32 dQ accumulator [B][H][Nq][d] followed by
 * (128 - Nq % 128) % 128 rows of d floats of padding (a ragged last query
 * tile reduces its masked rows, which are exact zeros, into them), then the
 * fp32 row term D [B][H][Nq], then the fp32 row term -log2(e) * LSE
 * [B][H][Nq], then (16-byte aligned) B*H*ceil(Nq/128) int32 words that no
 * call uses at present (kept so that the size stays as documented).  Returns
 * 0 for an empty
 * problem (any size 0), a negative size, or a total that overflows size_t.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int d);

/*
 * Backward pass of attn_fwd for the loss gradient dO.  Recomputes P from
 * (q, k, lse) and writes
 *   dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale * dS K,  dK = scale * dS^T Q,
 * where D_i = sum_c dO_ic O_ic.  `o` and `lse` must be the outputs of attn_fwd
 * for the same q, k, v, scale and causal flag.
 *   dq, dk, dv   outputs, 16-bit, same layouts as q, k, v.
 *   workspace    device buffer of attn_bwd_workspace_bytes() bytes, 16-byte
 *                aligned; its contents on entry are ignored and on return are
 *                unspecified.  It must not be shared by calls that overlap.
 * For d = 64 and 128 dQ is accumulated with fp32 atomic additions, so its
 * last bits may differ between runs; dK and dV are deterministic.  For
 * d = 256 attn_bwd is attn_bwd_deterministic (see there): its dK and dV
 * accumulators take 64 keys per CTA, and dQ comes from its own kernel.
 * Any finite scale is accepted, 0 and negative ones included.  At d = 64
 * and 128 the kernel adds the per-query terms -LSE_i / scale and -D_i to its
 * fp32 products as pieces of the 16-bit input type; in fp16 they are exact for
 * |LSE_i / scale| < 2^31 and |D_i| < 2^31 (for example any |scale| >= 1e-8
 * with |LSE| <= 20).  Beyond that the call records ATTN_ERR_RANGE in the
 * device status word (attn_last_device_status) and its gradients are not
 * meaningful.  bf16 has no such limit.  As in every 16-bit attention
 * backward, dS = P * (dP - D) is rounded to the input type before its two
 * products, so |dP - D| beyond the type's range overflows there.
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                     void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, attn_dtype dtype, void* stream);

/*
 * attn_bwd with a bit-reproducible dQ.  The backward the pages describe has
 * no such variant; the page "Flash Attention 落地评估" (section 4) raises
 * reproducibility as a concern, and attn_bwd's dQ depends on the order in
 * which fp32 atomic additions from different key tiles land.  Here dK and dV
 * come from the same per-key-tile kernel as in attn_bwd (without its dQ
 * product), and dQ from a second kernel with one CTA per query tile that
 * recomputes the probabilities of each key tile it sees and accumulates its
 * own dQ rows in order; nothing is added atomically, so two calls with the
 * same inputs give identical dQ, dK and dV bits.  The second kernel repeats
 * the S and dP products (7 matrix products per tile pair instead of 5), so
 * it is somewhat slower than attn_bwd.  At d = 256 the dK/dV kernel takes
 * 64-key tiles, keeping dV^T and dK^T (two 128-row halves of the head
 * dimension each) in tensor memory, and the dQ kernel 64-key steps; that is
 * the only d = 256 backward, which attn_bwd runs as well.  The dQ
 * accumulator of the workspace is not used.  Arguments, workspace and errors
 * as for attn_bwd.
 */
attn_status attn_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                   void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                                   int causal, attn_dtype dtype, void* stream);

/*
 * One phase of attn_bwd, for callers that time or schedule the three
 * backward kernels separately.  Running ATTN_BWD_PREPROCESS, ATTN_BWD_MAIN
 * and ATTN_BWD_CONVERT in that order on one stream, with the same arguments
 * and workspace, is exactly attn_bwd; ATTN_BWD_ALL is attn_bwd itself.
 *   PREPROCESS  D_i = sum_c dO_ic O_ic and -log2(e) LSE_i into the workspace,
 *               and zeroes the dQ accumulator;
 *   MAIN        recomputes P and accumulates dV, dK (written to dv, dk) and
 *               the fp32 dQ accumulator;
 *   CONVERT     dq = 16-bit(dQ accumulator).
 * At d = 256 PREPROCESS leaves the accumulator alone, MAIN runs the dK/dV
 * and dQ kernels of attn_bwd_deterministic (dq written directly) and CONVERT
 * does nothing.
 * Arguments, validation and errors as for attn_bwd; `phase` outside the
 * enum returns ATTN_ERR_INVALID_ARG.
 */
typedef enum {
  ATTN_BWD_ALL = 0,
  ATTN_BWD_PREPROCESS = 1,
  ATTN_BWD_MAIN = 2,
  ATTN_BWD_CONVERT = 3
} attn_bwd_phase_t;

attn_status attn_bwd_phase(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, void* dq, void* dk, void* dv,
                           void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                           int causal, attn_dtype dtype, int phase, void* stream);

/*
 * attn_bwd without a workspace argument.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory when
 * they call -- a plugin running inside another runtime's execution callback,
 * where allocating is not allowed, or a process whose device memory is all
 * held by another allocator's pool.  It allocates nothing: the workspace is
 * a fixed 72 MiB array inside the library (every GPU that loads the library
 * holds it until the process exits), and the caller still passes every input
 * and output.
 *   Limit.  Problems whose attn_bwd_workspace_bytes() exceeds
 *           attn_bwd_noalloc_max_scratch_bytes() (72 MiB; at d = 128 about
 *           145,000 query rows B*H*Nq) return ATTN_ERR_SCRATCH_LIMIT
 *           before any work is enqueued.
 *   Set-up. The first call on each device looks up the array's device
 *           address (cudaGetSymbolAddress) with that device current; make
 *           that first call before any stream capture.
 *   Sharing. Every call on a device uses the same array, which keeps the
 *           last call's contents; each call clears what must start at zero.
 *           Calls whose kernels overlap on the GPU (e.g. on two streams)
 *           race on the array and give wrong results: order them.
 * Arguments, results and other errors as for attn_bwd.
 */
attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int H, int Nq, int Nk, int d, float scale, int causal,
                             attn_dtype dtype, void* stream);

/* Size in bytes of attn_bwd_noalloc's fixed scratch array (72 MiB). */
size_t attn_bwd_noalloc_max_scratch_bytes(void);

/*
 * Forward and backward of one batch whose tensors live in host memory: the
 * host-resident form of attn_fwd followed by attn_bwd (or
 * attn_bwd_deterministic when `deterministic` is non-zero), with the same
 * shapes, layouts, masks, scale and rounding.
 *   q_h, k_h, v_h, dout_h  inputs in host memory, [B][H][N][d] 16-bit.
 *   o_h, dq_h, dk_h, dv_h  outputs in host memory, 16-bit; lse_h [B][H][Nq]
 *                          float.
 *   device_buffer          caller-owned device memory of at least
 *                          attn_host_step_device_bytes(...) bytes, 256-byte
 *                          aligned: the device copies of every tensor and
 *                          the backward's workspace.
 *   chunks                 the B*H slices are processed in this many
 *                          chunks (>= 1; capped at B*H).
 * The slices are split into chunks; the host-to-device copies of all chunks
 * run on an internal stream, each chunk's kernels run on `stream` once its
 * inputs have landed, and each chunk's results return to the host on a
 * second internal stream once its kernels are done, so copies of one chunk
 * overlap the kernels of another.  Everything is asynchronous: `stream`
 * continues past the call once every result has reached the host, and the
 * host buffers must stay valid until then.  Host buffers should be
 * page-locked (cudaHostAlloc / pinned); pageable memory works but its
 * copies do not overlap.  d is 64, 128 or 256.  No query rows (B*H*Nq == 0)
 * writes dK = dV = 0 on the host in stream order; Nq > 0 with Nk = 0
 * returns ATTN_ERR_INVALID_ARG.  An error return may leave part of the work
 * enqueued: synchronize the device before reusing the buffers.  The
 * current device must own `device_buffer` and `stream`.
 */
size_t attn_host_step_device_bytes(int B, int H, int Nq, int Nk, int d, int chunks);
attn_status attn_host_step(const void* q_h, const void* k_h, const void* v_h, const void* dout_h,
                           void* o_h, float* lse_h, void* dq_h, void* dk_h, void* dv_h,
                           void* device_buffer, size_t device_bytes, int B, int H, int Nq, int Nk,
                           int d, float scale, int causal, attn_dtype dtype, int chunks,
                           int deterministic, void* stream);

/*
 * Packed variable-length batches.  B sequences of different lengths share
 * one tensor without padding (the pages' "varlen" use: each sequence is an
 * attention problem of its own).  Layout, head-major like the dense calls:
 * Q, O, dO, dQ are [H][total_q][d]; K, V, dK, dV are [H][total_k][d]; LSE is
 * [H][total_q].  Sequence b occupies rows [cu_seqlens_q[b], cu_seqlens_q[b+1])
 * of every head of Q, O, dO, dQ and LSE, and rows [cu_seqlens_k[b],
 * cu_seqlens_k[b+1]) of every head of K, V, dK, dV.
 *   cu_seqlens_q, cu_seqlens_k  DEVICE int32 arrays of B + 1 non-decreasing
 *                offsets from 0 to total_q (total_k), 4-byte aligned.  They
 *                are read by the kernels and not checked on the host; the
 *                kernels clamp them to [0, total], so invalid offsets can give
 *                wrong values but never address memory outside the tensors.
 *   max_seqlen_q, max_seqlen_k  at least the longest sequence (they size the
 *                grid; rows of a longer sequence past them are not computed).
 * The causal mask, top-left or bottom-right, is aligned within each
 * sequence.  A sequence with queries and no keys gets O = 0, LSE = -inf and
 * dQ = 0; one with keys and no queries gets dK = dV = 0.  Other arguments,
 * supported head dims and dtypes, and errors as for the dense calls.
 */
attn_status attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                            int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                            float scale, int causal, attn_dtype dtype, void* stream);

/* Workspace of attn_bwd_varlen, laid out as for attn_bwd with B*H*Nq rows
 * replaced by H*total_q and 128 padding rows; 0 for an empty batch. */
size_t attn_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d);

/* Backward of attn_fwd_varlen; deterministic != 0 orders the dQ reductions
 * as attn_bwd_deterministic does. */
attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv,
                            void* workspace, const int* cu_seqlens_q, const int* cu_seqlens_k,
                            int B, int H, int total_q, int total_k, int max_seqlen_q,
                            int max_seqlen_k, int d, float scale, int causal, attn_dtype dtype,
                            int deterministic, void* stream);

/*
 * Self-test of failure detection; the pages have no counterpart.  Launches one
 * small kernel on `stream`.  Its first warp waits, through the same bounded
 * mbarrier wait the attention kernels use, on a barrier that nothing ever
 * arrives on, with a limit of `limit_us` microseconds (1 .. 1,000,000).  The
 * wait gives up, raises the CTA's abort flag and records ATTN_ERR_TIMEOUT in
 * the device status word.  A second warp, waiting on another such barrier,
 * leaves through the abort flag.  The kernel then exits normally and the
 * context stays usable.  result (device, 2 ints) receives 0 for each warp
 * whose wait gave up.  Returns ATTN_OK once launched; read the status with
 * attn_last_device_status().
 */
attn_status attn_selftest_wait_timeout(int limit_us, int* result, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device status word that
 * kernels of this library set when a bounded wait times out
 * (ATTN_ERR_TIMEOUT), when shared memory is short (ATTN_ERR_SMEM) or when an
 * fp16 backward's per-query terms are out of range (ATTN_ERR_RANGE), or
 * ATTN_ERR_CUDA if the synchronisation itself fails.
 * ATTN_OK means no kernel of this library has recorded an error since the
 * previous call on this device.
 */
attn_status attn_last_device_status(void* stream);

/* A static, human-readable name for a status code (never NULL). */
const char* attn_status_string(attn_status s);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
