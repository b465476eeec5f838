// fa_internal.h — launch interface shared by the host API and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

constexpr int kTileM = 128;  // query rows per MMA tile (TMEM lanes)
constexpr int kTileN = 128;  // key/value rows per tile

// Work-unit order: units are taken head group by head group (heads_per_group
// consecutive (batch, head) pairs), heaviest causal block first inside a
// group, so the K/V (forward) or Q/dO/dQ (backward) working set of the CTAs
// resident at one time stays inside the 126 MB L2.
struct FwdParams {
    int B, Hq, Hkv, N;
    int causal;
    float scale_log2;  // softmax scale * log2(e)
    int n_mblocks;     // ceil(N / 256): work unit = two 128-row query tiles
    int heads_per_group;
    void* o;           // bf16 [B,Hq,N,D]
    float* lse;        // fp32 [B,Hq,N]
    float o_scale;     // multiplies O before the 1/l normalisation (FP8: V's descale; 1 for bf16)
    int n_units;       // work units: B * Hq * n_mblocks
    unsigned int* sched;  // [2] counter slot of the persistent forward: next unit, CTAs done
    // Merge mode (one-CTA kernel only; m_o == nullptr: off): instead of writing
    // o and lse, fold this call's result into a running fp32 result by the
    // log-sum-exp rule; m_first: set it from this call.  m_out (bf16, may be
    // null) also receives the merged rows.
    float* m_o;        // fp32 [B,Hq,N,D]
    float* m_lse;      // fp32 [B,Hq,N]
    void* m_out;
    int m_first;
    int fma_exp;       // one-CTA bf16 kernel: 1/8 of the exponentials on the FMA pipe
};

// Multiprocessor count of the current device (cached per device; -1 on error).
int sm_count();

struct BwdParams {
    int B, Hq, Hkv, N, Npad;
    int causal;
    int heads_per_group;  // K/V heads per scheduling group
    float scale;       // softmax scale (dS is pre-multiplied by it)
    float scale_log2;  // scale * log2(e)
    const float* lse2; // [B*Hq, Npad] lse * log2(e), +inf on padding rows
    const float* dvec; // [B*Hq, Npad] scale * D, D = rowsum(dO o O); 0 on padding rows
    float* dq_acc;     // [B*Hq, N, D] fp32 accumulator (fused kernel only)
    void* dq;          // bf16 [B,Hq,N,D] (separate dQ pass writes it directly)
    void* dk;          // bf16 [B,Hkv,N,D]
    void* dv;          // bf16 [B,Hkv,N,D]
    int dq_heads_per_group;  // query heads per scheduling group of the dQ pass
    unsigned int* sched;     // work counters of the persistent kernels (zeroed by the preprocess)
    int n_units_dkdv;        // work units of the dK/dV pass
    int n_units_dq;          // work units of the dQ pass
    // Accumulate mode of the one-CTA separate passes (nullptr: off): add the
    // gradients into fp32 buffers instead of writing dq / dk / dv; the first
    // flags overwrite instead of adding.
    float* a_dq;       // fp32 [B,Hq,N,D]
    float* a_dk;       // fp32 [B,Hkv,N,D]
    float* a_dv;       // fp32 [B,Hkv,N,D]
    int a_first_dq, a_first_dkv;
};

// Counters at the start of the backward workspace: [0] dK/dV pass, [1] dQ pass.
constexpr int kSchedCounters = 4;

// Attention of Nq new queries over an Nk-long K/V history, split over keys.
struct DecodeParams {
    const void* q;     // bf16 [B,Hq,Nq,D]
    void* o;           // bf16 [B,Hq,Nq,D]
    float* lse;        // fp32 [B,Hq,Nq]
    float* o_part;     // fp32 [B*Hq*Nq, n_splits, D]: O / l of each key range
    float* lse_part;   // fp32 [B*Hq*Nq, n_splits]: LSE of each key range (-inf if empty)
    int Nq, Nk, G, causal;
    int n_splits, tiles_per_split;  // 64-key tiles per key range
    float scale_log2;
};
cudaError_t launch_decode(int D, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          int n_row_blocks, int BHkv, cudaStream_t stream);

// Workspace carve-up for the backward (all offsets 256-byte aligned).
struct BwdWorkspace {
    size_t sched_off, lse2_off, dvec_off, dq_off, total;
};
// with_dq_acc: room for the fp32 dQ accumulator of the fused kernel (dq_off ..
// total); the default separate dQ pass needs none (dq_off == total).
BwdWorkspace bwd_workspace_layout(int B, int Hq, int N, int D, bool with_dq_acc);

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, cudaStream_t stream);

// Forward on CTA pairs (D = 128; fa_fwd_pair.cu): work unit = 512 query rows
// (p.n_mblocks = ceil(N / 512)), every MMA M = 256 across the pair.  tk_half
// maps K with 64-row boxes (each CTA loads half of a key tile).  Units are
// served greedily from the counter slot p.sched, as in the one-CTA kernel.
cudaError_t launch_fwd_pair(const CUtensorMap& tq, const CUtensorMap& tk_half, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t stream);
// Pairs that can be resident at once (cached per device; -1 on error).
int fwd_pair_max_pairs();

// FP8 forward (D = 128): q/k/v maps over e4m3 bytes; p.scale_log2 already
// includes the Q and K descales, p.o_scale is V's descale.
cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                           cudaStream_t stream);

// dq_acc == nullptr: do not zero a dQ accumulator (separate dQ pass).
cudaError_t launch_bwd_preprocess(int D, const void* o, const void* dout, const float* lse,
                                  float* lse2, float* dvec, float* dq_acc,
                                  int BH, int N, int Npad, float scale, unsigned int* sched,
                                  cudaStream_t stream);

// Fused backward: dK, dV and dQ (fp32 reductions into p.dq_acc).
// the persistent fused backward (D = 128): dK, dV and dQ partials in one pass
cudaError_t launch_bwd_fused(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_main(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream);

// Separate-dQ backward: dK/dV kernel, then the dQ kernel writing p.dq.
cudaError_t launch_bwd_dkdv(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_dq(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream);

// dK/dV pass on CTA pairs (D = 128; fa_bwd_pair.cu): work unit = 256 keys
// (p.n_units_dkdv = B * Hkv * ceil(N / 256)), every MMA M = 256 across the
// pair.  tq_half / tdo_half map Q / dO with 64-row boxes.  Units are served
// greedily from the counter p.sched[0].
cudaError_t launch_bwd_dkdv_pair(const CUtensorMap& tq, const CUtensorMap& tq_half, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdo_half,
                                 const BwdParams& p, cudaStream_t stream);

// dQ pass on CTA pairs (D = 128): work unit = 256 query rows
// (p.n_units_dq = B * Hq * ceil(N / 256)).  tk_half / tv_half map K / V with
// 64-row boxes.  Units are served greedily from the counter p.sched[1].
cudaError_t launch_bwd_dq_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tk_half,
                               const CUtensorMap& tv_half, const CUtensorMap& tdo, const BwdParams& p,
                               cudaStream_t stream);

cudaError_t launch_bwd_dq_convert(const float* dq_acc, void* dq, size_t n_elems, cudaStream_t stream);

// Sequence-sharded attention: log-sum-exp merge of a partial result into a
// running one, and fp32 accumulation of bf16 gradient terms (fa_cp.cu).
cudaError_t launch_lse_merge(int D, long long rows, const void* o_part, const float* lse_part, float* o_acc,
                             float* lse_acc, void* o_out, int first, cudaStream_t stream);
cudaError_t launch_accumulate(long long n, const void* src, float* acc, void* out, int first, cudaStream_t stream);

}  // namespace fa
