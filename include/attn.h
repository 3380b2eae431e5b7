/*
 * attn.h - C ABI of the B200 (sm_100a) exact-attention library, libattn.so.
 *
 * The library computes exact scaled-dot-product attention,
 *
 *     O = softmax(Q K^T * softmax_scale + mask) V,
 *
 * tile by tile with an online (running max, running sum) softmax, so the
 * Nq x Nk score matrix never reaches device memory, and the backward pass
 * that recomputes the score tiles from Q, K, V and the saved per-row
 * log-sum-exp instead of storing them.
 *
 *   - Definition Softmax(QK^T/sqrt(d))V: "FlashAttention ... transformer
 *     optimization", technical deep dive, first paragraph.
 *   - Tiling into on-chip blocks, online softmax with a running maximum and
 *     normalisation factor, recomputation in the backward pass: same page,
 *     items 1 and 2 and the paragraph after them; "FlashAttention-2 ...
 *     windows builds analysis", technical deep dive.
 *   - (batch, seqlen, nheads, headdim) layout, fp16/bf16 only, causal flag,
 *     explicit softmax_scale: "FlashAttention-2：下一代高效注意力机制的突破与实战
 *     解析", section "实操落地" (integration example) and its notes.
 *   - Causal and sliding-window masks with work skipped outside the mask:
 *     same page, sections "3 支持更灵活的掩码与因果注意力" and "3 稀疏注意力扩展",
 *     FAQ Q1.
 *   - MQA/GQA (nheads_kv < nheads) and head dimensions up to 256:
 *     "FlashAttention 四代演进", sections on architecture and hardware/dtype
 *     limits.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers named q, k, v, o, dout, dq, dk, dv, lse and workspace are DEVICE
 * pointers on the current CUDA device; the caller allocates and owns all of
 * them.  The library never allocates, frees or synchronises on the normal
 * path; every call is asynchronous on `stream` (a cudaStream_t passed as
 * void*, NULL = the legacy default stream).  Outputs are valid once the
 * stream reaches the end of the call.
 *
 * Layouts (row-major, contiguous, headdim innermost):
 *   q, o, dout, dq : (batch, seqlen_q, nheads,    headdim)
 *   k, v, dk, dv   : (batch, seqlen_k, nheads_kv, headdim)
 *   lse            : (batch, nheads, seqlen_q) float32, natural log of the
 *                    row's sum of exp(scaled scores); -inf for a query that
 *                    sees no key (its O row is then 0).
 * Element type of q, k, v, o, dout, dq, dk, dv: `dtype` (bf16 or fp16).
 *
 * Masks.  Key j is visible from query i iff, with off = seqlen_k - seqlen_q
 * + pos_offset (bottom-right alignment, moved by attn_params.pos_offset),
 *     causal:            j <= i + off
 *     window_left  >= 0: j >= i + off - window_left
 *     window_right >= 0: j <= i + off + window_right
 * Bounds are inclusive; -1 means unbounded.
 *
 * Grouped-query attention: query head h reads kv head h / (nheads/nheads_kv).
 *
 * Errors are returned, never raised: no exception or abort crosses the ABI.
 * Argument errors are detected on the host before anything is launched.
 * A launch failure returns ATTN_ERR_CUDA (the CUDA error is then available
 * from cudaGetLastError's successor calls in the caller's runtime).  Kernels
 * that wait on on-chip barriers give up after a bounded time, record a code
 * in a device status word and exit; attn_get_device_status() reads it.
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_BF16 = 0, ATTN_FP16 = 1 } attn_dtype;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,          /* null pointer, negative size, H % Hkv != 0, bad window */
  ATTN_ERR_UNSUPPORTED_HEADDIM = 2,  /* headdim outside the compiled set */
  ATTN_ERR_UNSUPPORTED_DTYPE = 3,    /* dtype not bf16/fp16 */
  ATTN_ERR_MISALIGNED = 4,           /* a tensor pointer not 16-byte aligned */
  ATTN_ERR_WORKSPACE_TOO_SMALL = 5,  /* workspace_bytes below the *_workspace_size() query */
  ATTN_ERR_CUDA = 6,                 /* a CUDA runtime/driver call failed */
  ATTN_ERR_TIMEOUT = 7,              /* a device-side bounded wait expired */
  ATTN_ERR_DEVICE_STATUS = 8         /* the device status word holds another error */
} attn_status;

typedef struct {
  int32_t batch;
  int32_t seqlen_q;
  int32_t seqlen_k;
  int32_t nheads;
  int32_t nheads_kv;
  int32_t headdim;
  int32_t dtype;          /* attn_dtype */
  float softmax_scale;    /* multiplies Q K^T; the usual value is 1/sqrt(headdim) */
  int32_t causal;         /* 0 or 1 */
  int32_t window_left;    /* -1 = unbounded */
  int32_t window_right;   /* -1 = unbounded */
  /* Per-head positional slopes: NULL, or a DEVICE array of nheads floats
   * (4-byte aligned); score (i, j) of head h then gains
   * -alibi_slopes[h] * |i + off - j|, off as in the mask rules (the alibi_slopes
   * argument of the FlashAttention-2 interface; see the mask rules below for
   * the alignment).  Read by the kernels only. */
  const float* alibi_slopes;
  /* Dropout on the attention probabilities (inverted dropout; 0 = none,
   * the value a zero-initialised struct holds).  dropout_p in [0, 1): the
   * applied rate is t / 256 with t = round(256 * dropout_p) <= 255, kept
   * values are scaled by 256 / (256 - t), and P, the LSE and the row sums are
   * those of the undropped scores.  The drop decision of score element
   * (b, h, i, j) (batch or sequence b, query head h of H, query row i, key j)
   * is fixed by the generator contract: Philox4x32-10 with key
   * (dropout_seed low word, high word) at counter (j / 4, i / 4, b * H + h,
   * dropout_offset); byte (j % 4) of output word (i % 4) is the element's
   * random byte, dropped iff below t.  The backward pass must get the same
   * seed and offset as the forward.  Forward with headdim 256 does not
   * support dropout (ATTN_ERR_UNSUPPORTED_HEADDIM). */
  float dropout_p;
  uint32_t dropout_offset;
  uint64_t dropout_seed;
  /* Position of the query rows relative to the keys beyond the bottom-right
   * alignment (0, the value a zero-initialised struct holds, = none): the
   * masks and the positional bias use off = seqlen_k - seqlen_q + pos_offset.
   * For one block of a longer sequence (queries at global positions
   * q0 .. q0 + seqlen_q - 1, keys at k0 .. k0 + seqlen_k - 1) it is
   * q0 - k0 - (seqlen_k - seqlen_q), so that the block sees exactly the
   * mask and bias of the whole sequence.  attn_fwd, attn_bwd and its stages
   * and attn_fwd_e4m3 honour it; attn_fwd_decode and the packed-sequence
   * calls require 0 (ATTN_ERR_INVALID_ARG). */
  int32_t pos_offset;
  int32_t reserved0;      /* must be 0 */
} attn_params;

/*
 * Forward pass.  Reads q, k, v; writes o and lse.
 * Supported: headdim in {64, 128, 256}; dtype bf16 or fp16.
 * workspace may be NULL when attn_fwd_workspace_size() returns 0.
 * Sizes may be zero (batch, seqlen_q, seqlen_k): an empty call is a no-op,
 * and seqlen_k == 0 yields O = 0 and LSE = -inf.
 */
ATTN_API attn_status attn_fwd(const attn_params* p, const void* q, const void* k, const void* v, void* o,
                     float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward pass with E4M3 (FP8) inputs, the FP8 forward the pages name for
 * FlashAttention-3.  q, k, v hold E4M3 codes, one byte per element, in the
 * attn_fwd layouts; each tensor has one scale (element ~ scale *
 * e4m3(code)), and the result is attention over those values:
 * S = (q k^T) * q_scale * k_scale * softmax_scale, O = softmax(S) v * v_scale.
 * o is written in p->dtype (bf16 or fp16), lse as attn_fwd's.  The kernel
 * rounds P to E4M3 before the P V product (relative 2^-4).  Supported:
 * headdim 128, causal and window masks, GQA; alibi_slopes must be NULL
 * and dropout_p 0.
 * Scales must be positive and finite (ATTN_ERR_INVALID_ARG).  Needs no
 * workspace; asynchronous on `stream`.
 */
ATTN_API attn_status attn_fwd_e4m3(const attn_params* p, const void* q, const void* k,
                                   const void* v, float q_scale, float k_scale, float v_scale,
                                   void* o, float* lse, void* stream);

/*
 * Forward pass for decoding: a few query rows per sequence against a long
 * key / value sequence (a cache), with the same arguments, layouts, masks
 * (bottom-right aligned) and results as attn_fwd.  The keys are split over
 * blocks of the CUDA cores (the work is bound by reading K and V; every kv
 * head's K and V rows are read once for all the query heads of its group)
 * and the splits' partial results are merged as attn_merge does.
 * Supported: headdim 64 or 128, (nheads / nheads_kv) * seqlen_q <= 16,
 * no positional slopes and no dropout (ATTN_ERR_INVALID_ARG otherwise).  workspace: at
 * least attn_fwd_decode_workspace_size(p) bytes, 256-byte aligned, caller-
 * owned, overwritten.  Asynchronous on `stream`.
 */
ATTN_API size_t attn_fwd_decode_workspace_size(const attn_params* p);
ATTN_API attn_status attn_fwd_decode(const attn_params* p, const void* q, const void* k,
                                     const void* v, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Backward pass: given dout = dL/dO and the forward's o and lse, writes
 * dq = dL/dQ, dk = dL/dK, dv = dL/dV (dk, dv summed over the query heads of
 * each kv group).  The score tiles are recomputed from q, k and lse.
 * Supported: headdim in {64, 128, 256} (256 without dropout, as the pages
 * give FlashAttention-2's backward: "FlashAttention 四代演进", hardware /
 * dtype limits); dtype bf16 or fp16.  With headdim 256 the accumulate stage
 * runs three kernels, for dV, dK and dQ, each recomputing the score tiles
 * it needs (eight tile products instead of five, to fit tensor memory).
 * workspace: at least attn_bwd_workspace_size(p) bytes, 256-byte aligned;
 * it holds float32 rowsum(dO o O), lse in base 2 and the float32 dQ
 * accumulator.  Its contents on entry do not matter.
 */
ATTN_API attn_status attn_bwd(const attn_params* p, const void* q, const void* k, const void* v,
                     const void* o, const float* lse, const void* dout, void* dq, void* dk,
                     void* dv, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three stages attn_bwd runs, in this order, on one stream and one
 * workspace; exposed so a caller can time or schedule them separately.
 * Same arguments, layouts and errors as attn_bwd.
 *   attn_bwd_prepare:    float32 rowsum(dout o o) and lse*log2(e) per query
 *                        into the workspace; zeroes the dQ accumulator.
 *   attn_bwd_accumulate: recomputes the score tiles and writes dk and dv;
 *                        adds every key tile's dQ share into the accumulator.
 *   attn_bwd_finalize:   dq = softmax_scale * accumulator, in `dtype`.
 */
ATTN_API attn_status attn_bwd_prepare(const attn_params* p, const void* o, const float* lse,
                                      const void* dout, void* workspace, size_t workspace_bytes,
                                      void* stream);
ATTN_API attn_status attn_bwd_accumulate(const attn_params* p, const void* q, const void* k,
                                         const void* v, const void* dout, void* dk, void* dv,
                                         void* workspace, size_t workspace_bytes, void* stream);
ATTN_API attn_status attn_bwd_finalize(const attn_params* p, void* dq, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * attn_bwd_accumulate with float32 key gradients added instead of written:
 * dk_acc += softmax_scale * dS^T Q and dv_acc += P^T dout, both float32
 * (batch, seqlen_k, nheads_kv, headdim), 16-byte aligned, caller-owned.
 * For callers that sum the key gradients of several calls over the same
 * keys, such as one sequence split across devices: each (query block, key
 * block) pair is one call, and a key block's gradients are the sum over the
 * query blocks, accumulated block by block without forming the full matrix
 * ("What is FlashAttention", five-stage map, stage 4).  Dense batches, no
 * dropout (ATTN_ERR_INVALID_ARG); otherwise as attn_bwd_accumulate,
 * including its dQ share.
 */
ATTN_API attn_status attn_bwd_accumulate_f32(const attn_params* p, const void* q, const void* k,
                                             const void* v, const void* dout, float* dk_acc,
                                             float* dv_acc, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * dst = src rounded to `dtype` (ATTN_BF16 or ATTN_FP16, nearest even), n
 * elements, n a multiple of 4; src 16-byte and dst 8-byte aligned.  The
 * last step after attn_bwd_accumulate_f32.
 */
ATTN_API attn_status attn_f32_to_16(const float* src, void* dst, long long n, int dtype,
                                    void* stream);

/*
 * Backward pass for callers that cannot allocate device memory.
 *
 * attn_bwd needs a caller-provided workspace.  Some callers cannot make one
 * at call time: a host framework that has already claimed the GPU's memory
 * for its own pool and forbids allocations behind its back, or code on a
 * latency-critical path where cudaMalloc (which synchronises the device and
 * can fail) is not acceptable.  This entry point takes the same inputs and
 * outputs as attn_bwd and allocates nothing: its scratch is a fixed array of
 * ATTN_NOALLOC_SCRATCH_BYTES in the library's own device memory, which every
 * GPU that loads libattn.so holds until the process exits.  The method as the
 * pages describe it has no counterpart to this entry point.
 *
 *   - Limit: the call is rejected with ATTN_ERR_WORKSPACE_TOO_SMALL when
 *     attn_bwd_workspace_size(p) exceeds ATTN_NOALLOC_SCRATCH_BYTES, before
 *     anything is launched.
 *   - Set-up: the first call on a device looks up that device's copy of the
 *     array (cudaGetSymbolAddress, with the device current); make that first
 *     call before any stream capture.  Later calls reuse the address, which
 *     is kept for the life of the process: after cudaDeviceReset on a device,
 *     this entry point must not be called on that device again.
 *   - Sharing: all calls on a device use the same array, which keeps the last
 *     call's contents; each call clears what must start at zero.  Calls that
 *     overlap on the GPU (other streams, other threads) race on the array and
 *     must be serialised by the caller.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
ATTN_API attn_status attn_bwd_noalloc(const attn_params* p, const void* q, const void* k,
                                      const void* v, const void* o, const float* lse,
                                      const void* dout, void* dq, void* dk, void* dv,
                                      void* stream);

/* ------------------------------------------------------------------ packed
 * Variable-length sequences packed back to back (the varlen interface named
 * on "FlashAttention-2：下一代高效注意力机制的突破与实战解析", section
 * "实操落地", and the inference-with-cache use of "FlashAttention 四代演进",
 * interface section).  Each sequence is an independent attention problem
 * with the masks of attn_params applied with its own lengths (bottom-right
 * alignment when its query and key lengths differ).
 *
 * Layout: sequence b owns rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) of q, o,
 * dout, dq, each a (total_q, nheads, headdim) 16-bit tensor, and rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) of k, v, dk, dv, each
 * (total_k, nheads_kv, headdim).  lse is fp32 (nheads, total_q), natural log.
 * cu_seqlens_q / cu_seqlens_k are DEVICE arrays of batch + 1 int32 offsets,
 * non-decreasing from 0 to total_q / total_k; every sequence must be at most
 * max_seqlen_q / max_seqlen_k long.  The offsets are read only by the
 * kernels (no host synchronisation): values outside [0, total] are clamped,
 * so a malformed array gives unspecified results but no access outside the
 * tensors.  Tiles of one sequence may read rows of its neighbours (masked to
 * zero weight), so inputs must be finite.
 */
typedef struct {
  int32_t batch;          /* number of sequences */
  int32_t total_q;        /* rows of q, o, dout, dq */
  int32_t total_k;        /* rows of k, v, dk, dv */
  int32_t max_seqlen_q;   /* >= every query sequence length */
  int32_t max_seqlen_k;   /* >= every key sequence length */
  int32_t nheads;
  int32_t nheads_kv;
  int32_t headdim;
  int32_t dtype;          /* attn_dtype */
  float softmax_scale;
  int32_t causal;
  int32_t window_left;
  int32_t window_right;
  const float* alibi_slopes;  /* as in attn_params; lengths per sequence */
  float dropout_p;            /* as in attn_params; b = sequence index and */
  uint32_t dropout_offset;    /* i, j positions within the sequence */
  uint64_t dropout_seed;
} attn_varlen_params;

/* Host-side checks of a packed call (pass 0 forward, 1 backward): the
 * attn_params rules with batch, max_seqlen_q/k as the sizes, and
 * non-negative totals.  Pointers and offsets are not inspected. */
ATTN_API attn_status attn_check_varlen_params(const attn_varlen_params* p, int pass);

/* Forward over packed sequences; needs no workspace (the arguments are
 * accepted for symmetry).  Asynchronous on `stream`.  A sequence with no
 * keys gets O = 0 and LSE = -inf; rows of q not covered by any sequence are
 * left untouched.  Errors as attn_fwd, plus ATTN_ERR_MISALIGNED for offset
 * arrays that are not 4-byte aligned. */
ATTN_API attn_status attn_fwd_varlen(const attn_varlen_params* p, const int32_t* cu_seqlens_q,
                                     const int32_t* cu_seqlens_k, const void* q, const void* k,
                                     const void* v, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Bytes of the caller-owned device workspace attn_bwd_varlen needs:
 * per-query statistics and an fp32 dQ accumulator over total_q rows plus
 * 136 rows of padding per sequence.  0 for invalid parameters. */
ATTN_API size_t attn_bwd_varlen_workspace_size(const attn_varlen_params* p);

/* Backward over packed sequences: dq, dk, dv (layouts as above) from the
 * forward's o and lse and the output gradient dout.  headdim 64 or 128.
 * The workspace (256-byte aligned, at least attn_bwd_varlen_workspace_size
 * bytes) is overwritten.  Asynchronous on `stream`; errors as attn_bwd. */
ATTN_API attn_status attn_bwd_varlen(const attn_varlen_params* p, const int32_t* cu_seqlens_q,
                                     const int32_t* cu_seqlens_k, const void* q, const void* k,
                                     const void* v, const void* o, const float* lse,
                                     const void* dout, void* dq, void* dk, void* dv,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace attn_fwd / attn_bwd need for these parameters
 * (0 when none).  Pure host functions; never touch the GPU. */
ATTN_API size_t attn_fwd_workspace_size(const attn_params* p);
ATTN_API size_t attn_bwd_workspace_size(const attn_params* p);

/* Host-side argument check that attn_fwd / attn_bwd perform first; exposed so
 * callers (and the CPU-only tests) can validate without a GPU.  `pass` is 0
 * for forward, 1 for backward.  Pointers are not inspected. */
ATTN_API attn_status attn_check_params(const attn_params* p, int pass);

/* A static, human-readable description of a status code. */
ATTN_API const char* attn_status_string(int status);

/* Reads and clears the device status word (0 = no device-side error).
 * Synchronises `stream`.  Returns ATTN_OK, or ATTN_ERR_CUDA if the read
 * failed.  *code receives an ATTN_ERR_* value or 0. */
ATTN_API attn_status attn_get_device_status(void* stream, int* code);

/* ------------------------------------------------------------------ merge
 * Merge of partial results computed over disjoint key sets (split-KV
 * decoding, sequence-parallel partials): for every query row,
 *     LSE = log sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
 * the identity the tiled online softmax itself rests on ("FlashAttention ...
 * transformer optimization", items 1-2).  A row whose parts all have
 * LSE = -inf gets O = 0, LSE = -inf.  The parts are typically attn_fwd
 * results over key ranges of one sequence (for causal decoding, the queries'
 * own range causal and the earlier ranges not).
 *
 * Layouts (device, contiguous): o_parts (splits, batch, seqlen_q, nheads,
 * headdim) 16-bit, 16-byte aligned; lse_parts (splits, batch, nheads,
 * seqlen_q) fp32; o (batch, seqlen_q, nheads, headdim); lse (batch, nheads,
 * seqlen_q).  Packed sequences: batch = 1, seqlen_q = total rows.  headdim
 * 64, 128 or 256; splits 1 .. 65535.  Asynchronous on `stream`. */
typedef struct {
  int32_t splits;
  int32_t batch;
  int32_t seqlen_q;
  int32_t nheads;
  int32_t headdim;
  int32_t dtype;  /* attn_dtype */
} attn_merge_params;

ATTN_API attn_status attn_merge(const attn_merge_params* p, const void* o_parts,
                                const float* lse_parts, void* o, float* lse, void* stream);

/* Diagnostic with no counterpart on the pages: checks the failure-detection
 * path on the device without faulting it.  Launches one small kernel on
 * `stream` whose two waiters (one warp-wide, one single-thread) wait on an
 * on-chip barrier that nothing ever arrives at; each gives up after
 * `wait_limit_us` microseconds (1 .. 1,000,000, else ATTN_ERR_INVALID_ARG,
 * nothing launched), ORs ATTN_ERR_TIMEOUT into the device status word and
 * returns.  `result`, if not NULL, is caller-owned device memory of two ints
 * that receive 1 for each waiter that gave up (0 if its wait had
 * succeeded).  Asynchronous; ATTN_ERR_CUDA if the launch fails.  Afterwards
 * attn_get_device_status() reports ATTN_ERR_TIMEOUT and clears it, and the
 * CUDA context stays usable. */
ATTN_API attn_status attn_selftest_bounded_wait(unsigned int wait_limit_us, int* result,
                                                void* stream);

/* Library version, "major.minor.patch". */
ATTN_API const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
