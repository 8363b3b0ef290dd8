/*
 * lwm_attn.h -- C ABI of liblwm_attn.so: exact blockwise causal self-attention
 * with rotary position embedding (RoPE) and a masked-sequence-packing mask,
 * forward and backward, for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are the pages describing Large World
 * Model, "LWM"):
 *
 *   - LWM research note (zhao9797.github.io), section "模型架构" (model
 *     architecture): exact blockwise attention (RingAttention + Blockwise
 *     Parallel Transformer fused with FlashAttention) and "standard RoPE"
 *     whose theta grows with the context window.
 *   - Same note, section "训练方法" (training method): the theta schedule
 *     (32K: 1e6, 128K: 1e7, 256K: 1e7, 512K: 2.5e7, 1M: 5e7) and Masked
 *     Sequence Packing: samples packed into one sequence attend only to
 *     themselves, numerically the same as unpacked training with padding.
 *   - Paper card "World Model on Million-Length Video And Language With
 *     Blockwise RingAttention" (research.elamur.ai), Summary: the attention is
 *     computed "without approximation"; its reference list names RoFormer
 *     (the rotary form) and FlashAttention (blockwise exact softmax).
 *
 * Definitions (row i, key j of one (batch, head); D = head_dim):
 *   w_t      = theta^(-2t/D),  t = 0 .. D/2-1
 *   R(p)     = rotation of each interleaved pair (x[2t], x[2t+1]) by p*w_t,
 *              p = index of the token in its row (positions continue across
 *              packed segments; outputs do not depend on that choice)
 *   s_ij     = scale * <R(i) q_i, R(j) k_j>
 *   allowed  = seg_i == seg_j  &&  seg_i >= 0  &&  (!causal || j <= i)
 *   LSE_i    = ln sum_{allowed j} exp(s_ij)         (-inf if nothing allowed)
 *   O_i      = sum_{allowed j} exp(s_ij - LSE_i) v_j  (0 if nothing allowed)
 *   dq, dk, dv = gradients of sum(O * dO) with respect to the UN-rotated q, k
 *              and v.
 *
 * Layout (all tensors): Q, K, V, O, dO, dQ, dK, dV are [B, S, H, D]
 * contiguous, D fastest (token stride H*D).  LSE is [B, H, S] fp32.
 * Segment ids are [B, S] int32 on the device.
 *
 * Ownership: the caller owns every buffer.  The library allocates no device
 * memory in any call; it caches only device properties under a mutex.
 *
 * Calling convention: every compute call is asynchronous on `stream` (a
 * cudaStream_t passed as void*; NULL = legacy default stream).  Argument,
 * alignment and workspace errors are returned synchronously before anything
 * is launched.  A bounded device-side wait that runs out writes
 * LWM_ERR_TIMEOUT into the workspace status word; read it with
 * lwm_attn_read_status after the stream's work.  Launch failures are
 * returned as LWM_ERR_CUDA.
 *
 * Thread safety: calls may come from several host threads; calls that share
 * a workspace must not overlap on the device.
 */
#ifndef LWM_ATTN_H
#define LWM_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LWM_OK = 0,
  LWM_ERR_INVALID_ARG = -1,  /* null pointer, bad size, bad enum value */
  LWM_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. head_dim 96) */
  LWM_ERR_ALIGNMENT = -3,    /* a tensor pointer is not 16-byte aligned */
  LWM_ERR_WORKSPACE = -4,    /* workspace null or smaller than required */
  LWM_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed */
  LWM_ERR_TIMEOUT = -6       /* a bounded device wait ran out (status word) */
} lwm_status;

typedef enum { LWM_DTYPE_BF16 = 0, LWM_DTYPE_FP32 = 1 } lwm_dtype;

/* Problem description shared by forward and backward. */
typedef struct {
  int64_t batch;              /* B >= 1 */
  int64_t seqlen;             /* S >= 1 (no upper limit beyond memory; 64-bit offsets) */
  int64_t heads;              /* H >= 1 */
  int64_t head_dim;           /* D in {64, 128} */
  int32_t dtype;              /* lwm_dtype of Q, K, V, O, dO, dQ, dK, dV */
  int32_t causal;             /* 1: j <= i within a segment; 0: whole segment */
  double rope_theta;          /* RoPE base; <= 0 disables the rotation */
  float softmax_scale;        /* <= 0 selects 1/sqrt(head_dim) */
  const int32_t* segment_ids; /* device [B, S]; NULL = one segment per row;
                                 id < 0 marks padding (O = 0, LSE = -inf,
                                 gradients 0).  Any ids are correct; ids that
                                 form contiguous runs (what packing produces)
                                 let whole tiles be skipped. */
} lwm_attn_desc;

/* Bytes of device workspace lwm_attn_fwd (is_bwd = 0) or lwm_attn_bwd
 * (is_bwd != 0) needs for `desc` on the current device; 0 if `desc` is
 * invalid.  The workspace holds the status word, per-tile segment bounds,
 * the rotated copies the chosen kernels read (K for the tensor-core forward,
 * which rotates its Q tiles itself; Q for the one-pass backward, which
 * rotates its K tiles; both for the other kernels) and, for the backward,
 * the per-row LSE and dot(dO, O) (fp32, padded to whole tiles for the
 * tensor-core kernels) and the one-pass backward's fp32 dQ accumulator.
 * The forward's need is never larger than the backward's. */
size_t lwm_attn_workspace_size(const lwm_attn_desc* desc, int is_bwd);

/* Forward pass (research note, "模型架构": exact blockwise attention with RoPE;
 * "训练方法": packing mask).  q, k, v: device [B,S,H,D] of desc->dtype,
 * un-rotated.  o: device [B,S,H,D] output.  lse: device [B,H,S] fp32 output
 * (natural log of the scaled scores).  ws: device workspace of at least
 * lwm_attn_workspace_size(desc, 0) bytes, 256-byte aligned.  All tensor
 * pointers must be 16-byte aligned.  o and lse may not alias the inputs. */
lwm_status lwm_attn_fwd(const lwm_attn_desc* desc, const void* q, const void* k,
                        const void* v, void* o, float* lse, void* ws,
                        size_t ws_bytes, void* stream);

/* Backward pass: gradients of sum(O * dO) with respect to the un-rotated q,
 * k and v (the gradients training needs, research note "训练方法"; P is
 * recomputed from the saved LSE as in the FlashAttention reference of the
 * paper card).  o and lse must be the outputs of lwm_attn_fwd for the same
 * inputs; d_o is [B,S,H,D] of desc->dtype.  dq, dk, dv are written (not
 * accumulated).  ws: at least lwm_attn_workspace_size(desc, 1) bytes. */
lwm_status lwm_attn_bwd(const lwm_attn_desc* desc, const void* q, const void* k,
                        const void* v, const void* o, const float* lse,
                        const void* d_o, void* dq, void* dk, void* dv, void* ws,
                        size_t ws_bytes, void* stream);

/* lwm_attn_fwd without a workspace argument: the forward pass takes its
 * scratch memory (status word, per-tile segment bounds, rotated q and k)
 * from a fixed 40 MiB device array inside the library instead of from the
 * caller.  The pages have no counterpart; this is for callers that cannot
 * call cudaMalloc where they run the forward pass, for example code running
 * under an allocator or memory planner that forbids new device allocations
 * after start-up, or a host that must not risk the implicit synchronisation
 * or out-of-memory failure an allocation can bring at that point.  The
 * caller still passes q, k, v, o and lse (same meaning as lwm_attn_fwd).
 *   - Scratch limit: 40 MiB.  On the tensor-core forward (one rotated
 *     copy) that is about 20M bf16 elements per tensor (e.g. 4,096 tokens
 *     x 32 heads x 128); where q and k are both pre-rotated, about 10M.
 *     A problem whose workspace
 *     (lwm_attn_workspace_size(desc, 0)) is larger returns
 *     LWM_ERR_WORKSPACE and launches nothing.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *     Every GPU that loads the library holds the 40 MiB array until exit.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture.  A failed lookup returns
 *     LWM_ERR_CUDA.  The address is kept for the life of the process: after
 *     cudaDeviceReset (or anything else that replaces the device's primary
 *     context) it is stale, and this entry point must not be called again
 *     in that process.
 *   - Sharing: all calls on a device share the one array, which keeps the
 *     last call's contents (the call clears what must start at zero).  Calls
 *     that overlap on the GPU (different streams, or host threads) race on
 *     it; serialise them.
 *   - Device-side status (a bounded wait that ran out) lands in the status
 *     word at the start of the library's array, not in a caller workspace:
 *     read it with lwm_attn_fwd_noalloc_read_status. */
lwm_status lwm_attn_fwd_noalloc(const lwm_attn_desc* desc, const void* q, const void* k,
                                const void* v, void* o, float* lse, void* stream);

/* Status word of the last lwm_attn_fwd_noalloc call on the current device,
 * as lwm_attn_read_status gives it for a caller workspace: waits for
 * `stream`, then returns LWM_OK or the code a kernel recorded.  The same
 * once-per-device set-up as lwm_attn_fwd_noalloc (no allocation); LWM_ERR_CUDA
 * if the lookup or the copy fails. */
lwm_status lwm_attn_fwd_noalloc_read_status(void* stream);

/* Decode step (research note, "模型架构" and "Infra": generation over a
 * million-token context).  n_new new tokens are the last n_new positions of
 * each row; their keys and values are already the last entries of the
 * cache.  New token t (position p_t = S - n_new + t) attends exactly as row
 * p_t of lwm_attn_fwd: same mask (segment ids over the whole row, causal
 * order), same scale and RoPE.
 *   desc:    batch B, seqlen S = cache length (new tokens included), heads
 *            H, head_dim 128, dtype LWM_DTYPE_BF16 (others return
 *            LWM_ERR_UNSUPPORTED), causal, rope_theta, softmax_scale,
 *            segment_ids [B, S] (device, may be NULL).
 *   n_new:   1 .. min(S, LWM_DECODE_MAX_NEW); more returns
 *            LWM_ERR_UNSUPPORTED (use lwm_attn_fwd), below 1 or above S
 *            LWM_ERR_INVALID_ARG.
 *   q:       [B, n_new, H, D] un-rotated queries (rotated inside, in fp32).
 *   k_cache: [B, S, H, D] ROTATED keys, R(j) k_j, as lwm_rope_apply writes
 *            them (a cache keeps keys the way attention consumes them).
 *   v_cache: [B, S, H, D].
 *   o:       [B, n_new, H, D] out (bf16);  lse: [B, H, n_new] fp32 out
 *            (natural log, -inf for a token with no allowed key, o = 0).
 *   ws:      lwm_attn_decode_workspace_size(desc, n_new) bytes, 256-byte
 *            aligned (chunk partials of the split-KV reduction).
 * All device pointers 16-byte aligned.  Asynchronous on `stream`; the
 * timing-event slots fwd_start / fwd_stop bracket its two kernels.  Reads
 * each allowed cache row of each head once: bound by HBM bandwidth. */
#define LWM_DECODE_MAX_NEW 16
size_t lwm_attn_decode_workspace_size(const lwm_attn_desc* desc, int64_t n_new);
lwm_status lwm_attn_decode(const lwm_attn_desc* desc, int64_t n_new, const void* q,
                           const void* k_cache, const void* v_cache, void* o, float* lse,
                           void* ws, size_t ws_bytes, void* stream);

/* y = R(p) x (inverse = 0) or R(p)^T x (inverse != 0) for x of [B,S,H,D]
 * (research note, "模型架构": standard RoPE; theta per "训练方法").  Angles
 * p*w_t are formed and reduced modulo 2*pi in fp64, cos/sin taken in fp32,
 * the pair rotated in fp32 and rounded to dtype (nearest even).  y may equal
 * x (in place); otherwise they must not overlap.  theta <= 0 copies. */
lwm_status lwm_rope_apply(int64_t batch, int64_t seqlen, int64_t heads,
                          int64_t head_dim, int32_t dtype, double theta,
                          const void* x, void* y, int inverse, void* stream);

/* Waits for `stream`, then returns the status word the kernels of the last
 * call on `ws` left: LWM_OK, LWM_ERR_TIMEOUT (a bounded wait ran out) or
 * LWM_ERR_UNSUPPORTED (a kernel could not lay out its shared memory); or
 * LWM_ERR_CUDA if the read itself failed. */
lwm_status lwm_attn_read_status(const void* ws, void* stream);

/* Static, human-readable name of a status code. */
const char* lwm_status_string(lwm_status status);

/* Instrumentation (no counterpart on the pages; used by the benchmark).
 * lwm_attn_set_timing_events: cudaEvent_t handles (as void*, any may be
 * NULL) that the next calls record on their stream immediately before and
 * after the main attention kernel(s) of lwm_attn_fwd / lwm_attn_bwd, so the
 * caller can time those kernels alone; bwd_split is recorded between the
 * dK/dV kernel and the dQ kernel of the backward (both kernel families run
 * dK/dV first).  The handles stay in effect until
 * replaced; pass NULLs to stop.  Process-wide; guarded by a mutex.
 * lwm_attn_kernel_launches: number of kernels this library has launched
 * since it was loaded. */
void lwm_attn_set_timing_events(void* fwd_start, void* fwd_stop, void* bwd_start,
                                void* bwd_stop, void* bwd_split);
uint64_t lwm_attn_kernel_launches(void);

/* ---- Sequence-parallel (ring) building blocks -------------------------
 * Blockwise RingAttention (research note, "模型架构" and "Infra"; paper card,
 * Summary): the sequence is split into equal blocks, one per device of a
 * ring; every query block meets every key/value block once, and the results
 * combine exactly by their log-sum-exp.  The per-block products are
 * lwm_attn_fwd / lwm_attn_bwd on rotated inputs (rope_theta = 0); these
 * entry points supply the rest.  All asynchronous on `stream`; device
 * pointers; returns argument and launch errors.
 *
 * lwm_rope_apply_at: lwm_rope_apply with positions p = position_offset +
 *   index in the row (a block that starts at token position_offset >= 0).
 * lwm_attn_merge: for every row (b, s, h) of one query block, with
 *   L = ln(e^{lse_acc} + e^{lse_part}):
 *   o_acc <- e^{lse_acc - L} o_acc + e^{lse_part - L} o_part, lse_acc <- L.
 *   o_acc fp32 [B,S,H,D], lse_acc fp32 [B,H,S] (start from 0 and -inf);
 *   o_part [B,S,H,D] of `dtype`, lse_part [B,H,S].  A -inf side adds nothing.
 * lwm_accumulate: acc[i] += x[i] for n elements (acc fp32, x of `dtype`).
 * lwm_convert_f32: y[i] = x[i] rounded to `dtype` (nearest even). */
/* lwm_attn_fwd_pair / lwm_attn_bwd_pair: lwm_attn_fwd / lwm_attn_bwd for a
 *   block pair of a packed ring: queries of one block (segment ids
 *   desc->segment_ids) against the keys and values of another block of the
 *   same length (segment ids k_segment_ids), row i attending key j when their
 *   ids match (and j <= i if causal, for the diagonal pair).  Both id arrays
 *   or neither (LWM_ERR_INVALID_ARG otherwise); k_segment_ids [B, S], device,
 *   4-byte aligned.  Same workspace size, buffers, errors and outputs as the
 *   single-block calls, which are the case k_segment_ids = segment_ids. */
lwm_status lwm_attn_fwd_pair(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                             const void* q, const void* k, const void* v, void* o, float* lse,
                             void* ws, size_t ws_bytes, void* stream);
lwm_status lwm_attn_bwd_pair(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                             const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* d_o, void* dq, void* dk, void* dv,
                             void* ws, size_t ws_bytes, void* stream);

/* lwm_attn_fwd_pair_f32 / lwm_attn_bwd_pair_f32: the same block-pair
 *   products with fp32 outputs (o, dq, dk, dv fp32 [B,S,H,D]) whatever the
 *   input dtype, so the partial results of a ring are merged and summed
 *   without a bf16 rounding per block (N blocks would otherwise add N
 *   roundings).  Supported for fp32 inputs (identical to the pair calls) and
 *   for bf16, head_dim 128 on sm_100 (the tensor-core kernels write fp32);
 *   other shapes, or the two-kernel backward (LWM_ATTN_SPLIT_BWD=1), return
 *   LWM_ERR_UNSUPPORTED before any launch.  Same workspace as the pair
 *   calls. */
lwm_status lwm_attn_fwd_pair_f32(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                                 const void* q, const void* k, const void* v, float* o, float* lse,
                                 void* ws, size_t ws_bytes, void* stream);
lwm_status lwm_attn_bwd_pair_f32(const lwm_attn_desc* desc, const int32_t* k_segment_ids,
                                 const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* d_o, float* dq, float* dk, float* dv,
                                 void* ws, size_t ws_bytes, void* stream);

lwm_status lwm_rope_apply_at(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                             int32_t dtype, double theta, int64_t position_offset, const void* x,
                             void* y, int inverse, void* stream);
lwm_status lwm_attn_merge(int64_t batch, int64_t seqlen, int64_t heads, int64_t head_dim,
                          int32_t dtype, float* o_acc, float* lse_acc, const void* o_part,
                          const float* lse_part, void* stream);
lwm_status lwm_accumulate(int64_t n, int32_t dtype, float* acc, const void* x, void* stream);
lwm_status lwm_convert_f32(int64_t n, int32_t dtype, const float* x, void* y, void* stream);

/* ---- Packed loss re-weighting ------------------------------------------
 * Cross-entropy of a packed batch, re-weighted so that it equals training on
 * the samples one by one with padding (research note, "训练方法", Masked
 * Sequence Packing): a sample is a contiguous run of one segment id; a loss
 * token of a sample with n loss tokens weighs 1 / (n * number of samples
 * with a loss token).
 *   logits [B, S, V] (dtype bf16 or fp32, 16-byte aligned), targets [B, S]
 *   int32 (< 0 or >= V: no loss at that token), segment_ids [B, S] int32
 *   (NULL: each row is one sample; id < 0: padding, no loss).
 *   loss: device float, sum over tokens of w_t * (logsumexp(z_t) - z_t[y_t]),
 *   summed in a fixed order.  dlogits [B, S, V] of dtype (may be NULL):
 *   w_t * (softmax(z_t) - onehot(y_t)), zero rows for tokens without loss.
 *   ws: lwm_packed_ce_workspace_size(B, S) bytes, 256-byte aligned; it
 *   starts with the status word, which lwm_attn_read_status(ws) reads after
 *   the call (LWM_ERR_TIMEOUT if a bounded wait inside the kernel ran out).
 *   V up to 32,768 for bf16 and 16,384 for fp32 (a row held in registers),
 *   and a multiple of 8 (bf16) or 4 (fp32) so rows are whole 16-byte
 *   vectors; otherwise LWM_ERR_UNSUPPORTED.  Reads the logits once and
 *   writes dlogits once: bound by HBM bandwidth. */
size_t lwm_packed_ce_workspace_size(int64_t batch, int64_t seqlen);
lwm_status lwm_packed_cross_entropy(int64_t batch, int64_t seqlen, int64_t vocab, int32_t dtype,
                                    const void* logits, const int32_t* targets,
                                    const int32_t* segment_ids, float* loss, void* dlogits,
                                    void* ws, size_t ws_bytes, void* stream);

/* Failure-path self-test (no counterpart on the pages).  Clears the status
 * word at the start of ws (at least 256 bytes, 256-byte aligned) and runs one
 * CTA that waits on an mbarrier with the same bounded wait the tensor-core
 * kernels use, for at most limit_cycles SM clock cycles.  arrive != 0 arms
 * the barrier first (the wait completes: status stays LWM_OK); arrive == 0
 * leaves it unarmed (nothing ever arrives: the wait runs out, the kernel
 * records LWM_ERR_TIMEOUT and returns).  Read the outcome with
 * lwm_attn_read_status(ws).  Asynchronous; returns launch errors only. */
lwm_status lwm_attn_selftest_wait(void* ws, size_t ws_bytes, int64_t limit_cycles, int arrive,
                                  void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LWM_ATTN_H */
