/*
 * fa.h — exact tiled (flash) attention for NVIDIA B200 (sm_100a), C ABI.
 *
 * What is computed.  For every batch b and query head h (K/V head
 * g = h / (Hq / Hkv), contiguous groups):
 *     S = scale * Q K^T            (key j visible to query i iff j <= i when causal)
 *     P = softmax(S) row-wise,  O = P V,  LSE_i = log sum_j exp(S_ij)  (natural log)
 * The forward never materialises S or P in global memory: Q is kept on chip
 * tile by tile while K/V tiles stream past it and an online softmax (running
 * row max m and running sum l, final O / l correction) accumulates O.  This is
 * the tiling + incremental softmax of "【词汇专栏】FlashAttention：大模型训练的
 * 加速器" (sections 2.1, 2.2, 2.3) and of "FlashAttention 在昇腾NPU上到底快在哪"
 * (sections 二 and 三).
 * The backward recomputes P from the saved LSE ("FlashAttention V2深度解析：
 * 反向传播显存优化让大模型训练不再OOM", section 改进1, the recompute-instead-of-
 * store idea) and uses the closed-form softmax gradient of L = <O, dO>:
 *     D_i = sum_d dO_id O_id,  dV = P^T dO,  dP = dO V^T,
 *     dS = P o (dP - D) * scale,  dK = dS^T Q,  dQ = dS K,
 * with dK/dV of a K/V head summed over the query heads of its group (GQA).
 * Work is parallel over batch, head and sequence blocks (same deep dive,
 * section 改进2).
 *
 * Layout.  Every tensor is contiguous row-major.
 *   q, o, dout, dq : bf16 [B, Hq,  N, D]
 *   k, v, dk, dv   : bf16 [B, Hkv, N, D]
 *   lse            : fp32 [B, Hq, N]  natural-log log-sum-exp of the scaled logits
 * Supported: D in {64, 128}; B, Hq, Hkv, N >= 1; Hq % Hkv == 0.  Query and key
 * lengths are equal (N), so the causal mask is unambiguous.
 *
 * Ownership.  The caller allocates and owns every buffer (device memory),
 * including the backward workspace.  The library allocates no device memory on
 * these calls.  Pointers must be device pointers aligned to 16 bytes (the
 * backward's lse input: 4 bytes, it is read one element at a time).
 *
 * Streams and CUDA graphs.  The persistent forward kernels (fa_fwd,
 * fa_fwd_fp8) hand out work through a counter in a small static device table
 * of the library.  A launch outside stream capture takes one of 1024 slots in
 * turn, so launches that overlap on different streams use different counters;
 * a launch recorded into a CUDA graph takes a slot reserved for captured
 * launches (3072 of them, in turn), which no eager launch ever uses.  Two
 * replays of the same graph that run at the same time share that graph's
 * counters, like every other buffer the graph names, and must not overlap.
 * The first call on a device looks up the table's address, so make it before
 * capturing on that device.
 *
 * Asynchrony and errors.  Calls enqueue kernels on `stream` and return at
 * once.  A non-OK status means nothing was launched (argument errors) or the
 * launch failed (FA_ERR_CUDA).  Outputs are overwritten, never accumulated.
 * Device-side pipeline waits are bounded; a wait that gives up sets a device
 * status word that fa_get_device_status() reports (FA_ERR_TIMEOUT).
 */
#ifndef TILED_ATTENTION_FA_H
#define TILED_ATTENTION_FA_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad sizes, bad scale, small workspace */
    FA_ERR_UNSUPPORTED = 2, /* head dimension other than 64 or 128, or a non-sm_100 device */
    FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    FA_ERR_TIMEOUT = 4,     /* a device-side pipeline wait gave up (reported by fa_get_device_status) */
    FA_ERR_TOO_LARGE = 5    /* fa_bwd_noalloc: the shape needs more than FA_NOALLOC_SCRATCH_BYTES */
} fa_status;

/* Problem shape.  Hkv == Hq is plain multi-head attention; Hkv < Hq is GQA
 * (MQA when Hkv == 1).  scale multiplies the logits (1/sqrt(D) is usual); it
 * must be finite and > 0.  causal != 0 masks key j > query i. */
typedef struct {
    int B, Hq, Hkv, N, D;
    float scale;
    int causal;
} fa_shape;

/* Forward.  q [B,Hq,N,D], k/v [B,Hkv,N,D] bf16 in; o [B,Hq,N,D] bf16 and
 * lse [B,Hq,N] fp32 out.  `stream` is a cudaStream_t (NULL = legacy stream). */
FA_API fa_status fa_fwd(const fa_shape* shape, const void* q, const void* k, const void* v,
                 void* o, float* lse, void* stream);

/* FP8 forward (FlashAttention-3's FP8 operands, named in "【词汇专栏】
 * FlashAttention：大模型训练的加速器", section 3.3; the scaling convention is
 * this library's).  q [B,Hq,N,D], k/v [B,Hkv,N,D] hold e4m3 bytes (OCP FP8
 * E4M3, finite-only, 1 byte per element, contiguous); the value each element
 * stands for is element * q_scale (k_scale, v_scale), all three finite and
 * > 0.  Computes the same O and LSE as fa_fwd over those values: o
 * [B,Hq,N,D] bf16 and lse [B,Hq,N] fp32.  Both products run on the 8-bit
 * tensor-core path with fp32 accumulation; the probabilities are rounded to
 * e4m3 for the P V product (the row sums use them unrounded), so O carries a
 * relative error of up to 2^-4 per probability term.  D = 128 only
 * (FA_ERR_UNSUPPORTED otherwise).  Asynchronous on `stream` like fa_fwd. */
FA_API fa_status fa_fwd_fp8(const fa_shape* shape, const void* q, const void* k, const void* v,
                     float q_scale, float k_scale, float v_scale, void* o, float* lse, void* stream);

/* Attention of Nq new queries over an Nk-long K/V history (KV-cache reuse in
 * multi-turn inference, "FlashAttention 在昇腾NPU上到底快在哪", section 七).
 * The queries are the last Nq positions of the sequence: query i stands at
 * position Nk - Nq + i and, when causal != 0, sees keys j <= Nk - Nq + i.
 * Requires 1 <= Nq <= Nk; Hq % Hkv == 0; D = 64 or 128; scale finite, > 0. */
typedef struct {
    int B, Hq, Hkv, Nq, Nk, D;
    float scale;
    int causal;
} fa_kv_shape;

/* Bytes of device workspace fa_decode needs (0 if the shape is invalid): the
 * per-key-range partial outputs and log-sum-exps, fp32. */
FA_API size_t fa_decode_workspace_bytes(const fa_kv_shape* shape);

/* q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D] bf16 contiguous in; o [B,Hq,Nq,D] bf16 and
 * lse [B,Hq,Nq] fp32 (natural log) out.  The key axis is split across CTAs;
 * each writes a partial (O, LSE) to `workspace` (256-byte aligned, at least
 * fa_decode_workspace_bytes) and a second kernel merges them by the
 * log-sum-exp rule.  Errors and asynchrony as for fa_bwd. */
FA_API fa_status fa_decode(const fa_kv_shape* shape, const void* q, const void* k, const void* v, void* o,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* How fa_bwd forms dQ ("FlashAttention V2深度解析：反向传播显存优化让大模型训练
 * 不再OOM", section 改进2 parallelises the key sequence, so several key blocks
 * contribute to each dQ row):
 *   FA_BWD_FUSED          one persistent kernel runs all five GEMMs per tile
 *                         pair; each key block's dQ partial is added into an
 *                         fp32 accumulator by reductions in L2, in an order
 *                         that varies from run to run (dK, dV do not vary).
 *   FA_BWD_DETERMINISTIC  a dK/dV pass and a separate dQ pass that recomputes
 *                         S and dP (seven GEMMs per tile pair, no reductions);
 *                         repeated calls are bitwise equal.
 *   FA_BWD_AUTO           (default) the measured choice: FA_BWD_FUSED for
 *                         D = 128 (10-11% faster at N = 8192 and 65536, equal
 *                         at N = 2048), FA_BWD_DETERMINISTIC for D = 64.
 * fa_set_bwd_mode sets the process-wide choice (FA_ERR_INVALID_ARG for other
 * values) and fa_get_bwd_mode returns it; neither touches the GPU.  The
 * environment variable FA_DQ_MODE=separate|fused (read once per process)
 * overrides both.  Set the mode before querying fa_bwd_workspace_bytes: the
 * fused mode needs the larger workspace.  Calls already enqueued are not
 * affected by a later change. */
#define FA_BWD_AUTO 0
#define FA_BWD_DETERMINISTIC 1
#define FA_BWD_FUSED 2
FA_API fa_status fa_set_bwd_mode(int mode);
FA_API int fa_get_bwd_mode(void);

/* Bytes of device workspace fa_bwd needs for `shape` under the current
 * backward mode (0 if the shape is invalid): two work counters and the
 * per-row statistics (LSE in log2 units and D = rowsum(dO o O), each padded
 * to a multiple of 128 rows), about 8 * B * Hq * N bytes; plus an fp32 dQ
 * accumulator [B,Hq,N,D] when the shape runs the fused backward. */
FA_API size_t fa_bwd_workspace_bytes(const fa_shape* shape);

/* Backward.  Inputs q, k, v, o, dout (bf16) and lse (fp32, as written by
 * fa_fwd; 4-byte alignment suffices).  Outputs dq [B,Hq,N,D], dk and dv [B,Hkv,N,D], bf16, overwritten.
 * `workspace` must be a device buffer of at least fa_bwd_workspace_bytes(shape)
 * bytes, 256-byte aligned; its contents on entry do not matter. */
FA_API fa_status fa_bwd(const fa_shape* shape, const void* q, const void* k, const void* v,
                 const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Backward that allocates nothing (the pages have no counterpart: this is a
 * deployment convenience, not part of the method).
 *
 * Same computation, arguments and outputs as fa_bwd in FA_BWD_DETERMINISTIC
 * mode (whatever the current mode: bitwise equal to it), but without a caller
 * workspace: the scratch it needs (the work counters and the per-row LSE/D
 * statistics, about 8 * B * Hq * N bytes) lives in a fixed
 * FA_NOALLOC_SCRATCH_BYTES region of device memory that the library reserves
 * statically on every GPU that loads it, held until the process exits.  It is
 * meant for callers that cannot call cudaMalloc or hand out device memory on
 * this path: plugins whose host runtime owns every device allocation, or
 * latency-bound code where an allocation (and the synchronisation it can
 * imply) is not acceptable.
 *   - Shapes whose scratch exceeds FA_NOALLOC_SCRATCH_BYTES are rejected with
 *     FA_ERR_TOO_LARGE before anything is launched (use fa_bwd for those).
 *   - The first call on a device looks up the region's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Every call on a device shares the one region, and each call re-zeroes
 *     the parts that must start at zero; calls that overlap on the GPU (other
 *     streams, other host threads) race on it and must be serialised by the
 *     caller.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
#define FA_NOALLOC_SCRATCH_BYTES (32u << 20)
FA_API fa_status fa_bwd_noalloc(const fa_shape* shape, const void* q, const void* k, const void* v,
                                const void* o, const void* dout, const float* lse,
                                void* dq, void* dk, void* dv, void* stream);

/* ---- Sequence-sharded (context-parallel) attention.
 * "【词汇专栏】FlashAttention：大模型训练的加速器" (section 3.2, item 2) splits a
 * long sequence across devices, each working on its part.  The exact join of
 * the per-part results is the log-sum-exp merge below (adding the parts'
 * outputs, as the page puts it, is not attention).  A device runs fa_fwd and
 * fa_bwd on (query chunk, key chunk) pairs of equal length, with
 * causal = 1 on the diagonal pair and 0 below it, and joins the results with
 * these two kernels; the ring schedule and the exchange of K/V chunks between
 * devices live in the Python package (context_parallel.py).  fa_bwd on a pair
 * takes the FULL row statistics (the merged O and LSE of its query chunk), so
 * each pair's dQ, dK, dV are exact terms of the whole-sequence gradient.
 *
 * fa_lse_merge merges a partial result over one block of keys into a running
 * result over other keys.  rows = number of query rows (B*Hq*Nq), D in {64, 128}.
 *   o_part   bf16 [rows, D]  result normalised over the block (as fa_fwd writes it)
 *   lse_part fp32 [rows]     its natural-log LSE (-inf: the row saw no key of the block)
 *   o_acc    fp32 [rows, D]  running result, normalised over the keys merged so far (in/out)
 *   lse_acc  fp32 [rows]     its LSE (in/out)
 *   o_out    bf16 [rows, D]  optional (NULL allowed): also receives the merged result
 *   first    nonzero: o_acc / lse_acc are not read and are set from the part
 * lse = log(exp(lse_acc) + exp(lse_part)); o_acc = exp(lse_acc - lse) o_acc +
 * exp(lse_part - lse) o_part.  Rows without mass on either side become 0 and
 * -inf.  Device pointers, 16-byte aligned (lse pointers 4-byte aligned); the
 * caller owns all of them.  rows == 0 reads nothing and launches nothing (the
 * pointers may then be NULL).  FA_ERR_INVALID_ARG for rows < 0, null or
 * misaligned pointers; FA_ERR_UNSUPPORTED for other D. */
FA_API fa_status fa_lse_merge(long long rows, int D, const void* o_part, const float* lse_part, float* o_acc,
                              float* lse_acc, void* o_out, int first, void* stream);

/* Fused forms of the per-pair steps above (the same results, fewer passes
 * over memory):
 *
 * fa_fwd_merge computes what fa_fwd computes for q over (k, v) and folds it,
 * inside the forward kernel's epilogue, into a running fp32 result by the
 * log-sum-exp rule of fa_lse_merge instead of writing o and lse:
 *   o_acc   fp32 [B,Hq,N,D]  running result, normalised (in/out)
 *   lse_acc fp32 [B,Hq,N]    its natural-log LSE (in/out)
 *   o_out   bf16 [B,Hq,N,D]  optional (NULL allowed): also receives the merged result
 *   first   nonzero: o_acc / lse_acc are not read and are set from this call
 * The one-CTA forward kernel runs it whatever FA_FWD_TILE says.  q, k, v as
 * for fa_fwd; o_acc, o_out 16-byte aligned, lse_acc 4-byte aligned; errors
 * and asynchrony as for fa_fwd. */
FA_API fa_status fa_fwd_merge(const fa_shape* shape, const void* q, const void* k, const void* v, float* o_acc,
                              float* lse_acc, void* o_out, int first, void* stream);

/* fa_bwd split in two for a query block whose backward runs against several
 * key blocks:
 *
 * fa_bwd_stats writes the row statistics of the backward (LSE in log2 units
 * and scale * rowsum(dO o O), the preprocess of fa_bwd) for (o, dout, lse)
 * into `workspace` (at least fa_bwd_workspace_bytes(shape) bytes, 256-byte
 * aligned) and launches nothing else.
 *
 * fa_bwd_accumulate then runs the two gradient passes of fa_bwd on those
 * statistics and ADDS the gradients into fp32 sums instead of writing bf16:
 *   dq_acc fp32 [B,Hq,N,D], dk_acc and dv_acc fp32 [B,Hkv,N,D]  (in/out, 16-byte aligned)
 *   flags  FA_ACC_DQ_FIRST: dq_acc is overwritten, not added to;
 *          FA_ACC_DKV_FIRST: the same for dk_acc and dv_acc.
 * The workspace must hold the statistics fa_bwd_stats wrote for the same
 * shape and the same o, dout and lse; its work counters are reset here.  q,
 * k, v, dout as for fa_bwd (dout is read again by the passes).  For D = 128
 * in the fused backward mode (the default) one fused kernel runs and its
 * fp32 reductions add each dQ term straight into dq_acc (cleared first by a
 * FA_ACC_DQ_FIRST call), so dq_acc sums in varying order; otherwise the
 * one-CTA separate passes run (whatever FA_BWD_TILE says).  Errors and asynchrony as for fa_bwd. */
#define FA_ACC_DQ_FIRST 1
#define FA_ACC_DKV_FIRST 2
FA_API fa_status fa_bwd_stats(const fa_shape* shape, const void* o, const void* dout, const float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);
FA_API fa_status fa_bwd_accumulate(const fa_shape* shape, const void* q, const void* k, const void* v,
                                   const void* dout, float* dq_acc, float* dk_acc, float* dv_acc, int flags,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Gradient accumulation: acc = (first ? 0 : acc) + src, elementwise over n
 * elements (src bf16, acc fp32; src NULL adds nothing), and out = bf16(acc)
 * when out is not NULL.  n >= 0 and a multiple of 8; device pointers 16-byte
 * aligned, owned by the caller; n == 0 reads nothing and launches nothing
 * (the pointers may then be NULL).  FA_ERR_INVALID_ARG otherwise. */
FA_API fa_status fa_accumulate(long long n, const void* src, float* acc, void* out, int first, void* stream);

/* Synchronises `stream`, then reports and clears the device status word of
 * the current device: FA_ERR_TIMEOUT if any kernel gave up a bounded wait
 * since the last call, FA_ERR_CUDA if the stream reports an error, else FA_OK. */
FA_API fa_status fa_get_device_status(void* stream);

/* Self-test of the failure detection (computes no attention).  Launches on
 * `stream` one CTA whose thread waits, with the bounded wait every kernel of
 * the library uses, on a barrier that nothing completes; at the wait limit
 * (2 s) it records `site` in the device status word and raises the CTA's
 * abort flag.  A second thread of the CTA waits on another such barrier from
 * a quarter of the limit later and must leave through the abort flag without
 * recording `site2`.  Afterwards fa_get_device_status() reports
 * FA_ERR_TIMEOUT and fa_debug_timeout_sites() returns bit `site` alone; the
 * CUDA context stays usable.  site and site2 in 0..31 and distinct, else
 * FA_ERR_INVALID_ARG before any launch; FA_ERR_CUDA if the launch fails. */
FA_API fa_status fa_selftest_wait_timeout(int site, int site2, void* stream);

/* Static description of a status code. */
FA_API const char* fa_status_str(fa_status status);

/* Diagnostics: the bitmask of device-side wait sites (bit k = site k) that
 * the most recent fa_get_device_status() call found and cleared; 0 when
 * healthy.  Host-only, no CUDA call. */
FA_API unsigned int fa_debug_timeout_sites(void);

/* Per-kernel timing for benchmarks.  After fa_profile_begin(), every kernel
 * the library launches is bracketed by a pair of CUDA events recorded on the
 * launching stream.  fa_profile_end() waits for those events, writes for each
 * kernel kind k the summed duration total_ms[k] and the launch count
 * launches[k], and stops recording.  Kinds: 0 forward (one-CTA kernel,
 * 128-row MMA tiles), 1 backward preprocess, 2 fused backward (dK, dV and dQ
 * by fp32 reductions), 3 dQ convert, 4 backward dK/dV kernel, 5 backward dQ
 * kernel, 6 FP8 forward, 7 decode (split kernel and combine together),
 * 8 log-sum-exp merge, 9 accumulation, 10 forward on CTA pairs (256-row MMA
 * tiles), 11 backward dK/dV kernel on CTA pairs (256-key blocks), 12
 * backward dQ kernel on CTA pairs (256-query blocks), 13 persistent fused
 * backward for D = 128 (dK, dV and dQ by fp32 bulk reductions)
 * (FA_PROFILE_KINDS; fa_fwd uses 0, or 10 when the environment variable
 * FA_FWD_TILE=m256 selects the CTA-pair kernel for D = 128; fa_bwd uses 1,
 * 13, 3 in the fused mode for D = 128 (1, 2, 3 for D = 64) and 1, 4, 5 in
 * the deterministic mode, where FA_BWD_TILE=m256 selects the CTA-pair passes
 * (1, 11, 12) for D = 128).  Events are host-created objects; no device
 * memory is allocated. */
#define FA_PROFILE_KINDS 14
FA_API fa_status fa_profile_begin(void);
FA_API fa_status fa_profile_end(float* total_ms, int* launches);

#ifdef __cplusplus
}
#endif

#endif /* TILED_ATTENTION_FA_H */
