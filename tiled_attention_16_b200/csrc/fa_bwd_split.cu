// fa_bwd_split.cu — tiled attention backward with a separate dQ pass.
//
// Same mathematics as fa_bwd.cu (recompute P from the saved LSE, closed-form
// softmax gradient dS = P o (dP - D); "FlashAttention V2深度解析：反向传播显存
// 优化让大模型训练不再OOM", sections 改进1 and 改进2), split into two kernels
// so that no fp32 reduction into global memory is needed and the result is
// deterministic:
//
//   fa_bwd_dkdv_kernel  one CTA per (batch, K/V head, 128-row key block j);
//                       loops over the query heads of the GQA group and the
//                       query tiles i (i >= j when causal):
//                         S^T = K_j Q_i^T, P^T = 2^(S^T c - lse2), dP^T = V_j dO_i^T,
//                         dV += P^T dO_i, dS^T = P^T o (dP^T - D) * scale, dK += dS^T Q_i.
//                       P^T and dS^T never leave tensor memory: each is packed
//                       as bf16 over the fp32 columns it was computed from and
//                       read from there as the A operand of the dV / dK MMA.
//   fa_bwd_dq_kernel    one CTA per (batch, query head, 128-row query tile i);
//                       loops over key tiles j (j <= i when causal):
//                         S = Q_i K_j^T, P = 2^(S c - lse2), dP = dO_i V_j^T,
//                         dS = P o (dP - D) * scale, dQ += dS K_j  (dQ in TMEM),
//                       then writes dQ as bf16 once.
//
// The dQ pass recomputes S and dP (7 GEMMs per tile pair instead of 5), in
// exchange for no reduction traffic and no serialisation on it.
//
// Both kernels: 320 threads = warps 0-7 compute (two groups of 4 warps split
// the 128 columns of the score tile; thread = TMEM lane), warp 8 issues MMAs
// (one thread), warp 9 drives TMA.  Every wait is bounded (sm100.cuh).
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

// Compute warps form kGroups groups of four (one warp per TMEM lane quarter);
// group g owns kCols consecutive columns of the 128-column score tile.
constexpr int kGroups = 2;
constexpr int kCols = kTileN / kGroups;
constexpr int kComputeWarps = 4 * kGroups;
constexpr int kMmaWarp = kComputeWarps;
constexpr int kLoadWarp = kComputeWarps + 1;
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr int kCompute = 32 * kComputeWarps;
static_assert(kCols % 32 == 0, "each compute thread handles whole 32-column TMEM loads");
static_assert(kCols == 64, "the dK/dV pass hands P^T to the dV MMAs in two 32-column halves per group");
constexpr int kMaxDynSmem = 232448;

// wait sites (bits of the device status word)
enum SplitSite {
    kS1Smem = 22, kS1Load = 23, kS1Empty = 24, kS1Mma = 25, kS1Compute = 26, kS1Drain = 27,
    kS2Load = 28, kS2Mma = 29, kS2Compute = 30, kS2Drain = 31
};

// TMEM column (relative to a 128-column block) of K-step kk (16 columns of
// the score tile) of a bf16 operand packed by the compute groups: group g
// packs its kCols columns into block columns [g kCols, g kCols + kCols / 2),
// columns it has itself already read.
__host__ __device__ constexpr uint32_t packed_col(int kk) {
    return static_cast<uint32_t>((kk / (kCols / 16)) * kCols + (kk % (kCols / 16)) * 8);
}

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, int site) {
    if (mbar_try_wait(bar, parity)) return;
    unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, 1u << site);
            return;
        }
    }
}

template <int D>
struct DkdvLayout {
    static constexpr int kTileBytes = kTileM * D * 2;
    static constexpr int kAtomBytes = kTileM * 128;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;       // 2 stages
    static constexpr int kDO = kQ + 2 * kTileBytes;  // 2 stages
    static constexpr int kLse = kDO + 2 * kTileBytes;
    static constexpr int kDvec = kLse + 2 * kTileN * 4;
    static constexpr int kBar = kDvec + 2 * kTileN * 4;
    static constexpr int kNumBars = 21;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "dK/dV shared memory layout too large");
};

template <int D>
struct DqLayout {
    static constexpr int kTileBytes = kTileM * D * 2;
    static constexpr int kAtomBytes = kTileM * 128;
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTileBytes;
    static constexpr int kK = kDO + kTileBytes;      // 2 stages
    static constexpr int kV = kK + 2 * kTileBytes;   // 2 stages
    static constexpr int kBar = kV + 2 * kTileBytes;
    static constexpr int kNumBars = 18;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "dQ shared memory layout too large");
};

// ===========================================================================
// dK / dV
// ===========================================================================
// One dK/dV work unit: (batch, K/V head, 128-row key block j).  Units are
// numbered head group by head group, key block ascending inside a group
// (heaviest first when causal), then head.
struct DkdvUnit {
    int j, bkv, b, hkv, i0, per_head, n_it;
};

__device__ __forceinline__ DkdvUnit dkdv_unit(const BwdParams& p, int T, int u) {
    DkdvUnit w;
    const int BHkv = p.B * p.Hkv;
    const int grp = u / (p.heads_per_group * T);
    const int h0 = grp * p.heads_per_group;
    const int nh = min(p.heads_per_group, BHkv - h0);
    const int rr = u - grp * p.heads_per_group * T;
    w.j = rr / nh;
    w.bkv = h0 + (rr - w.j * nh);
    w.b = w.bkv / p.Hkv;
    w.hkv = w.bkv - w.b * p.Hkv;
    w.i0 = p.causal ? w.j : 0;
    w.per_head = T - w.i0;
    w.n_it = (p.Hq / p.Hkv) * w.per_head;
    return w;
}

// Persistent: one CTA per SM walks work units.  The first unit of CTA c is
// c; later ones come from an atomic counter, so the heaviest-first order is
// served greedily.  The producer fetches each unit id and hands it to the MMA
// thread and the compute warps through a two-slot ring in shared memory.
// Every pipeline (Q/dO ring, S/dP/P/dS handshakes) keeps one running
// iteration count across units; K/V and the dK/dV epilogue go once per unit.
// While the compute warps store a unit's dK/dV, the producer already loads
// the next unit's K/V and the MMA thread forms its first S^T and dP^T (the
// S^T / dP^T blocks are free; the next dV MMA waits for the compute warps'
// first P^T, which they form only after reading dK/dV out).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const BwdParams p) {
    using L = DkdvLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kS1Smem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* q_full = bars + 1;       // [2]
    uint64_t* q_empty = bars + 3;      // [2]
    uint64_t* do_full = bars + 5;      // [2]
    uint64_t* do_empty = bars + 7;     // [2]
    uint64_t* s_full = bars + 9;
    uint64_t* dp_full = bars + 10;
    uint64_t* p_full0 = bars + 11;     // P^T of each group's first 32 query columns
    uint64_t* ds_full = bars + 12;
    uint64_t* dkv_full = bars + 13;
    uint64_t* drain = bars + 14;
    uint64_t* kv_empty = bars + 15;
    uint64_t* unit_full = bars + 16;   // [2]
    uint64_t* unit_empty = bars + 18;  // [2]
    uint64_t* p_full1 = bars + 20;     // P^T of each group's last 32 query columns
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int T = (p.N + kTileM - 1) / kTileM;
    const int G = p.Hq / p.Hkv;
    const int n_units = p.n_units_dkdv;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&do_full[s], 1);
            mbar_init(&do_empty[s], 1);
            mbar_init(&unit_full[s], 1);
            mbar_init(&unit_empty[s], kCompute + 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full0, kCompute);
        mbar_init(p_full1, kCompute);
        mbar_init(ds_full, kCompute);
        mbar_init(dkv_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

    // next unit id for the MMA thread and the compute warps (-1: no more work)
    auto take_unit = [&](int ui, bool& ok) -> int {
        const int s = ui & 1;
        ok = mbar_wait(&unit_full[s], (ui >> 1) & 1, abort_flag, kS1Load);
        const int u = ok ? unit_id[s] : -1;
        mbar_arrive(&unit_empty[s]);
        return u;
    };

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            int g = 0;        // query-tile iterations of this CTA so far (all units)
            int n_q = 0, n_do = 0, n_kv = 0;   // loads issued
            int ui = 0;       // units of this CTA
            int u = static_cast<int>(blockIdx.x);
            bool ok = true;
            while (ok) {
                const int s = ui & 1;
                if (ui >= 2 && !(ok = mbar_wait(&unit_empty[s], ((ui >> 1) - 1) & 1, abort_flag, kS1Empty))) break;
                unit_id[s] = (u < n_units) ? u : -1;
                mbar_arrive(&unit_full[s]);
                if (u >= n_units) break;
                const DkdvUnit w = dkdv_unit(p, T, u);
                // K/V of this unit once the previous unit's last S^T and dP^T are done
                if (ui >= 1 && !(ok = mbar_wait(kv_empty, (ui - 1) & 1, abort_flag, kS1Empty))) break;
                mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
                for (int a = 0; a < D / 64; ++a) {
                    tma_load_3d(smem + L::kK + a * L::kAtomBytes, &tmK, kv_full, a * 64, w.j * kTileN, w.bkv);
                    tma_load_3d(smem + L::kV + a * L::kAtomBytes, &tmV, kv_full, a * 64, w.j * kTileN, w.bkv);
                }
                n_kv = ui + 1;
                for (int it = 0; ok && it < w.n_it; ++it, ++g) {
                    const int st = g & 1;
                    const int gh = it / w.per_head;
                    const int i = w.i0 + (it - gh * w.per_head);
                    const int bhq = w.b * p.Hq + w.hkv * G + gh;
                    if (g >= 2 && !(ok = mbar_wait(&q_empty[st], ((g >> 1) - 1) & 1, abort_flag, kS1Empty))) break;
                    mbar_arrive_expect_tx(&q_full[st], L::kTileBytes + 2 * kTileM * 4);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kQ + st * L::kTileBytes + a * L::kAtomBytes, &tmQ, &q_full[st], a * 64,
                                    i * kTileM, bhq);
                    const size_t srow = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * kTileM;
                    bulk_load(smem + L::kLse + st * kTileM * 4, p.lse2 + srow, kTileM * 4, &q_full[st]);
                    bulk_load(smem + L::kDvec + st * kTileM * 4, p.dvec + srow, kTileM * 4, &q_full[st]);
                    n_q = g + 1;
                    if (g >= 2 && !(ok = mbar_wait(&do_empty[st], ((g >> 1) - 1) & 1, abort_flag, kS1Empty))) break;
                    mbar_arrive_expect_tx(&do_full[st], L::kTileBytes);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kDO + st * L::kTileBytes + a * L::kAtomBytes, &tmDO, &do_full[st],
                                    a * 64, i * kTileM, bhq);
                    n_do = g + 1;
                }
                if (!ok) break;
                ++ui;
                u = static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(p.sched + 0, 1u));
            }
            // no copy may still be landing in shared memory when the CTA leaves
            if (n_kv > 0) wait_drain(kv_full, (n_kv - 1) & 1, kS1Drain);
            for (int k = (n_q > 2 ? n_q - 2 : 0); k < n_q; ++k) wait_drain(&q_full[k & 1], (k >> 1) & 1, kS1Drain);
            for (int k = (n_do > 2 ? n_do - 2 : 0); k < n_do; ++k) wait_drain(&do_full[k & 1], (k >> 1) & 1, kS1Drain);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdSq = idesc_bf16_f32(kTileN, kTileM, 0, 0);  // S^T, dP^T
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kTileN, D, 0, 1);      // dV, dK (A from TMEM)
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            constexpr uint32_t kAtom = L::kAtomBytes;
            // dK += dS^T Q for query-tile iteration gp (global count); first = first of its unit
            auto issue_dk = [&](int gp, bool first) {
                const uint32_t qa = q_base + (gp & 1) * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)
                    mma_ts(tmem + kColDK, tmem + kColDP + packed_col(kk), sdesc_sw128(qa + kk * 2048, kAtom, 1024),
                           kIdAcc, (!first || kk > 0));
                tc_commit(&q_empty[gp & 1]);
            };
            bool ok = true;
            int g = 0;
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const int n_it = dkdv_unit(p, T, u).n_it;
                if (!(ok = mbar_wait(kv_full, ui & 1, abort_flag, kS1Load))) break;
                for (int it = 0; it < n_it; ++it) {
                    const int gi = g + it;
                    const int st = gi & 1;
                    const uint32_t sph = (gi >> 1) & 1;
                    const uint32_t ph = gi & 1;
                    // S^T = K Q^T (the previous P^T was consumed by dV(it-1), issued earlier)
                    if (!(ok = mbar_wait(&q_full[st], sph, abort_flag, kS1Load))) break;
                    tc_fence_after();
                    const uint32_t qa = q_base + st * L::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                        mma_ss(tmem + kColS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qa + off, 16, 1024),
                               kIdSq, kk > 0);
                    }
                    tc_commit(s_full);
                    // dK += dS^T Q of the previous query tile (dS^T packed in the dP^T block)
                    if (it > 0) {
                        if (!(ok = mbar_wait(ds_full, ph ^ 1, abort_flag, kS1Mma))) break;
                        tc_fence_after();
                        issue_dk(gi - 1, it == 1);
                    }
                    // dP^T = V dO^T
                    if (!(ok = mbar_wait(&do_full[st], sph, abort_flag, kS1Load))) break;
                    tc_fence_after();
                    const uint32_t da = do_base + st * L::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                        mma_ss(tmem + kColDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(da + off, 16, 1024),
                               kIdSq, kk > 0);
                    }
                    tc_commit(dp_full);
                    if (it == n_it - 1) tc_commit(kv_empty);   // K and V no longer read by this unit
                    // dV += P^T dO, in two halves of every group's query columns:
                    // the first half's MMAs run while the compute warps still
                    // form the second half of P^T
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = mbar_wait(h == 0 ? p_full0 : p_full1, ph, abort_flag, kS1Mma))) break;
                        tc_fence_after();
#pragma unroll
                        for (int g2 = 0; g2 < kGroups; ++g2) {
#pragma unroll
                            for (int t = 0; t < kCols / 32; ++t) {
                                const int kk = g2 * (kCols / 16) + h * (kCols / 32) + t;
                                mma_ts(tmem + kColDV, tmem + kColS + packed_col(kk),
                                       sdesc_sw128(da + kk * 2048, kAtom, 1024), kIdAcc, (it > 0 || kk > 0));
                            }
                        }
                    }
                    if (!ok) break;
                    tc_commit(&do_empty[st]);
                }
                if (!ok) break;
                const int gl = g + n_it - 1;   // last iteration of the unit
                if (!(ok = mbar_wait(ds_full, gl & 1, abort_flag, kS1Mma))) break;
                tc_fence_after();
                issue_dk(gl, n_it == 1);
                tc_commit(dkv_full);
                g += n_it;
            }
            tc_commit(drain);
            wait_drain(drain, 0, kS1Drain);
        }
    } else {
        // ------------------------------------------------------------ compute (P^T, dS^T)
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int r = (wq << 5) + lane;  // key row of the block = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * kCols;       // this group's query columns
        const float c = p.scale_log2;
        const float sc = p.scale;
        float pv[kCols];
        bool ok = true;
        int g = 0;
        for (int ui = 0; ok; ++ui) {
            const int u = take_unit(ui, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const DkdvUnit w = dkdv_unit(p, T, u);
            const int j = w.j;
            const int kv = j * kTileN + r;
            const bool kv_ok = kv < p.N;
            const bool kv_block_partial = (j + 1) * kTileN > p.N;
            for (int it = 0; it < w.n_it; ++it) {
                const int gi = g + it;
                const int st = gi & 1;
                const uint32_t ph = gi & 1;
                const int gh = it / w.per_head;
                const int i = w.i0 + (it - gh * w.per_head);
                const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse + st * kTileM * 4) + c0;
                const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvec + st * kTileM * 4) + c0;
                ok = mbar_wait(&q_full[st], (gi >> 1) & 1, abort_flag, kS1Compute) &&
                     mbar_wait(s_full, ph, abort_flag, kS1Compute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                {
                    uint32_t sr[kCols / 32][32];
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) tmem_ld32(tmem + lane_off + kColS + c0 + h * 32, sr[h]);
                    tmem_ld_wait();
                    const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
                    // Masked only on the causal diagonal block and on a partial
                    // last key block (both uniform across the warp); there,
                    // columns q < lo are zero (lo = kCols masks a key row past N).
                    const bool diag = p.causal && (i == j);
                    const bool masked = diag || kv_block_partial;
                    const int lo = !kv_ok ? kCols : (diag ? r - c0 : 0);
                    const float2 c2 = make_float2(c, c);
                    // two halves of 32 columns, each handed to the dV MMAs as
                    // soon as it is in TMEM (p_full0, p_full1)
                    static_for<0, 2>([&](auto hh) {
                        constexpr int h = decltype(hh)::value;
                        static_for<0, 16>([&](auto tc) {
                            constexpr int q = 32 * h + 2 * decltype(tc)::value;
                            const float2 l2 = *reinterpret_cast<const float2*>(lse_s + q);
                            const float2 x = __ffma2_rn(make_float2(sv[q], sv[q + 1]), c2, make_float2(-l2.x, -l2.y));
                            pv[q] = exp2_mixed<q>(x.x);
                            pv[q + 1] = exp2_mixed<q + 1>(x.y);
                        });
                        if (masked) {
#pragma unroll
                            for (int q = 32 * h; q < 32 * h + 32; ++q) pv[q] = (q >= lo) ? pv[q] : 0.f;
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) pk[t] = pack_bf16x2(pv[32 * h + 2 * t], pv[32 * h + 2 * t + 1]);
                        tmem_st16(tmem + lane_off + kColS + c0 + h * 16, pk);
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(h == 0 ? p_full0 : p_full1);
                    });
                }
                ok = mbar_wait(dp_full, ph, abort_flag, kS1Compute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < kCols / 32; ++h) {
                    uint32_t dpr[32];
                    tmem_ld32(tmem + lane_off + kColDP + c0 + h * 32, dpr);
                    tmem_ld_wait();
                    uint32_t wv[16];
                    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        // dS = P (dP - D) scale = P fma(dP, scale, -scale*D); dvec holds scale*D
                        const int q0 = h * 32 + 2 * t;
                        const float2 dv2 = *reinterpret_cast<const float2*>(dvec_s + q0);
                        const float2 gd = __ffma2_rn(
                            make_float2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), sc2,
                            make_float2(-dv2.x, -dv2.y));
                        const float2 d = __fmul2_rn(make_float2(pv[q0], pv[q0 + 1]), gd);
                        wv[t] = pack_bf16x2(d.x, d.y);
                    }
                    // packed over columns this group has already read
                    tmem_st16(tmem + lane_off + kColDP + c0 + h * 16, wv);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (!ok) break;
            // ---- epilogue: dV, dK rows of this key block (summed over the group)
            ok = mbar_wait(dkv_full, ui & 1, abort_flag, kS1Compute);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const size_t row = static_cast<size_t>(w.bkv) * p.N + kv;
            constexpr int kPer = D / kGroups;   // head-dimension columns written by this group
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t col0 = (which == 0 ? kColDV : kColDK) + wg * kPer;
                __nv_bfloat16* dst_row =
                    reinterpret_cast<__nv_bfloat16*>(which == 0 ? p.dv : p.dk) + row * D + wg * kPer;
                float* acc_row = p.a_dk ? (which == 0 ? p.a_dv : p.a_dk) + row * D + wg * kPer : nullptr;
#pragma unroll 1
                for (int q = 0; q < kPer / 16; ++q) {
                    uint32_t v16[16];
                    tmem_ld16(tmem + lane_off + col0 + q * 16, v16);
                    tmem_ld_wait();
                    if (acc_row) {   // accumulate mode: fp32 sums instead of bf16 outputs
                        if (kv_ok) accumulate16(acc_row + q * 16, v16, p.a_first_dkv);
                        continue;
                    }
                    uint32_t pk[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        pk[t] = pack_bf16x2(__uint_as_float(v16[2 * t]), __uint_as_float(v16[2 * t + 1]));
                    if (kv_ok) {
                        uint4* dst = reinterpret_cast<uint4*>(dst_row + q * 16);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            }
            // the next unit's dV / dK MMAs overwrite these columns only after this
            // group's next P^T arrival (p_full0), which follows these completed loads
            tc_fence_before();
            g += w.n_it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ===========================================================================
// dQ
// ===========================================================================
// One dQ work unit: (batch, query head, 128-row query tile i).  Units are
// numbered head group by head group, heaviest (last) query tile first inside
// a group, then head.
struct DqUnit {
    int i, bh, kvh, n_j;
};

__device__ __forceinline__ DqUnit dq_unit(const BwdParams& p, int T, int u) {
    DqUnit w;
    const int BH = p.B * p.Hq;
    const int grp = u / (p.dq_heads_per_group * T);
    const int h0 = grp * p.dq_heads_per_group;
    const int nh = min(p.dq_heads_per_group, BH - h0);
    const int rr = u - grp * p.dq_heads_per_group * T;
    w.i = T - 1 - rr / nh;
    w.bh = h0 + (rr % nh);
    const int b = w.bh / p.Hq;
    const int h = w.bh - b * p.Hq;
    w.kvh = b * p.Hkv + h / (p.Hq / p.Hkv);
    w.n_j = p.causal ? w.i + 1 : T;
    return w;
}

// Persistent in the same way as the dK/dV kernel: units from an atomic
// counter, handed over through a two-slot ring; the K/V ring and the S / dP /
// dS handshakes count key tiles across units.  Q and dO have one buffer: the
// next unit's tiles load once the current unit's last S and dP have read them
// (q_empty), while the compute warps store the current dQ.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                 const BwdParams p) {
    using L = DqLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kS1Smem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;       // Q and dO
    uint64_t* k_full = bars + 1;       // [2]
    uint64_t* v_full = bars + 3;       // [2]
    uint64_t* kv_empty = bars + 5;     // [2]
    uint64_t* s_full = bars + 7;
    uint64_t* s_free = bars + 8;
    uint64_t* dp_full = bars + 9;
    uint64_t* ds_full = bars + 10;
    uint64_t* dq_done = bars + 11;
    uint64_t* drain = bars + 12;
    uint64_t* q_empty = bars + 13;
    uint64_t* unit_full = bars + 14;   // [2]
    uint64_t* unit_empty = bars + 16;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int T = (p.N + kTileM - 1) / kTileM;
    const int n_units = p.n_units_dq;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&unit_full[s], 1);
            mbar_init(&unit_empty[s], kCompute + 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, kCompute);
        mbar_init(dp_full, 1);
        mbar_init(ds_full, kCompute);
        mbar_init(dq_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;

    auto take_unit = [&](int ui, bool& ok) -> int {
        const int s = ui & 1;
        ok = mbar_wait(&unit_full[s], (ui >> 1) & 1, abort_flag, kS2Load);
        const int u = ok ? unit_id[s] : -1;
        mbar_arrive(&unit_empty[s]);
        return u;
    };

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            int gj = 0;               // key tiles of this CTA so far (all units)
            int n_kv = 0, n_q = 0;    // K/V pairs and Q/dO pairs issued
            int ui = 0;
            int u = static_cast<int>(blockIdx.x);
            bool ok = true;
            while (ok) {
                const int s = ui & 1;
                if (ui >= 2 && !(ok = mbar_wait(&unit_empty[s], ((ui >> 1) - 1) & 1, abort_flag, kS2Load))) break;
                unit_id[s] = (u < n_units) ? u : -1;
                mbar_arrive(&unit_full[s]);
                if (u >= n_units) break;
                const DqUnit w = dq_unit(p, T, u);
                if (ui >= 1 && !(ok = mbar_wait(q_empty, (ui - 1) & 1, abort_flag, kS2Load))) break;
                mbar_arrive_expect_tx(q_full, 2 * L::kTileBytes);
                for (int a = 0; a < D / 64; ++a) {
                    tma_load_3d(smem + L::kQ + a * L::kAtomBytes, &tmQ, q_full, a * 64, w.i * kTileM, w.bh);
                    tma_load_3d(smem + L::kDO + a * L::kAtomBytes, &tmDO, q_full, a * 64, w.i * kTileM, w.bh);
                }
                n_q = ui + 1;
                for (int jj = 0; jj < w.n_j; ++jj, ++gj) {
                    const int st = gj & 1;
                    if (gj >= 2 && !(ok = mbar_wait(&kv_empty[st], ((gj >> 1) - 1) & 1, abort_flag, kS2Load))) break;
                    mbar_arrive_expect_tx(&k_full[st], L::kTileBytes);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kK + st * L::kTileBytes + a * L::kAtomBytes, &tmK, &k_full[st], a * 64,
                                    jj * kTileN, w.kvh);
                    mbar_arrive_expect_tx(&v_full[st], L::kTileBytes);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kV + st * L::kTileBytes + a * L::kAtomBytes, &tmV, &v_full[st], a * 64,
                                    jj * kTileN, w.kvh);
                    n_kv = gj + 1;
                }
                if (!ok) break;
                ++ui;
                u = static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(p.sched + 1, 1u));
            }
            if (n_q > 0) wait_drain(q_full, (n_q - 1) & 1, kS2Drain);
            for (int k = (n_kv > 2 ? n_kv - 2 : 0); k < n_kv; ++k) {
                wait_drain(&k_full[k & 1], (k >> 1) & 1, kS2Drain);
                wait_drain(&v_full[k & 1], (k >> 1) & 1, kS2Drain);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(kTileM, kTileN, 0, 0);  // S, dP: K-major both
            constexpr uint32_t kIdDQ = idesc_bf16_f32(kTileM, D, 0, 1);     // dQ: A (dS) TMEM, B = K MN-major
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            constexpr uint32_t kAtom = L::kAtomBytes;
            auto issue_s = [&](int st) {
                const uint32_t ka = k_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColS, sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), kIdS,
                           kk > 0);
                }
                tc_commit(s_full);
            };
            auto issue_dp = [&](int st) {
                const uint32_t va = v_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDP, sdesc_sw128(do_base + off, 16, 1024), sdesc_sw128(va + off, 16, 1024), kIdS,
                           kk > 0);
                }
                tc_commit(dp_full);
            };
            bool ok = true;
            int gj = 0;   // key tiles issued (all units)
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const int n_j = dq_unit(p, T, u).n_j;
                // S and dP of the unit's first key tile; the S block is reused once
                // the compute warps have read the previous S (s_free)
                if (!(ok = mbar_wait(q_full, ui & 1, abort_flag, kS2Load))) break;
                if (gj > 0 && !(ok = mbar_wait(s_free, (gj - 1) & 1, abort_flag, kS2Mma))) break;
                if (!(ok = mbar_wait(&k_full[gj & 1], (gj >> 1) & 1, abort_flag, kS2Load))) break;
                tc_fence_after();
                issue_s(gj & 1);
                if (!(ok = mbar_wait(&v_full[gj & 1], (gj >> 1) & 1, abort_flag, kS2Load))) break;
                tc_fence_after();
                issue_dp(gj & 1);
                if (n_j == 1) tc_commit(q_empty);   // Q and dO no longer read by this unit
                for (int jj = 0; jj < n_j; ++jj) {
                    const int G = gj + jj;
                    const int st = G & 1;
                    const uint32_t ph = G & 1;
                    // S(j+1) once the compute warps have read S(j)
                    if (jj + 1 < n_j) {
                        if (!(ok = mbar_wait(s_free, ph, abort_flag, kS2Mma))) break;
                        if (!(ok = mbar_wait(&k_full[st ^ 1], ((G + 1) >> 1) & 1, abort_flag, kS2Load))) break;
                        tc_fence_after();
                        issue_s(st ^ 1);
                    }
                    // dQ += dS K_j (dS packed as bf16 in the dP block)
                    if (!(ok = mbar_wait(ds_full, ph, abort_flag, kS2Mma))) break;
                    tc_fence_after();
                    const uint32_t ka = k_base + st * L::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)
                        mma_ts(tmem + kColDQ, tmem + kColDP + packed_col(kk), sdesc_sw128(ka + kk * 2048, kAtom, 1024),
                               kIdDQ, (jj > 0 || kk > 0));
                    tc_commit(&kv_empty[st]);
                    // dP(j+1): its block held dS(j), consumed by the MMAs just issued
                    if (jj + 1 < n_j) {
                        if (!(ok = mbar_wait(&v_full[st ^ 1], ((G + 1) >> 1) & 1, abort_flag, kS2Load))) break;
                        tc_fence_after();
                        issue_dp(st ^ 1);
                        if (jj + 2 == n_j) tc_commit(q_empty);
                    }
                }
                if (!ok) break;
                tc_commit(dq_done);
                gj += n_j;
            }
            tc_commit(drain);
            wait_drain(drain, 0, kS2Drain);
        }
    } else {
        // ------------------------------------------------------------ compute (P, dS)
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int r = (wq << 5) + lane;  // query row of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * kCols;       // this group's key columns
        const float c = p.scale_log2;
        const float sc = p.scale;
        float pv[kCols];
        bool ok = true;
        int gj = 0;
        for (int ui = 0; ok; ++ui) {
            const int u = take_unit(ui, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const DqUnit w = dq_unit(p, T, u);
            const int i = w.i;
            const int qrow = i * kTileM + r;
            const size_t srow = static_cast<size_t>(w.bh) * p.Npad + static_cast<size_t>(qrow);
            const float lse2 = p.lse2[srow];   // +inf on padding rows -> P = 0
            const float dval = p.dvec[srow];   // scale * D
            for (int jj = 0; jj < w.n_j; ++jj) {
                const uint32_t ph = (gj + jj) & 1;
                ok = mbar_wait(s_full, ph, abort_flag, kS2Compute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                {
                    uint32_t sr[kCols / 32][32];
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) tmem_ld32(tmem + lane_off + kColS + c0 + h * 32, sr[h]);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(s_free);
                    const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
                    const int kv0 = jj * kTileN + c0;
                    // Masked only on the causal diagonal tile and on a partial last
                    // key tile (uniform across the warp): key columns t >= hi are
                    // zero (past N, or after this query row on the diagonal).
                    const bool diag = p.causal && jj == i;
                    const float2 c2 = make_float2(c, c);
                    const float2 nl2 = make_float2(-lse2, -lse2);
                    static_for<0, kCols / 2>([&](auto tc) {
                        constexpr int t = 2 * decltype(tc)::value;
                        const float2 x = __ffma2_rn(make_float2(sv[t], sv[t + 1]), c2, nl2);
                        pv[t] = exp2_mixed<t>(x.x);
                        pv[t + 1] = exp2_mixed<t + 1>(x.y);
                    });
                    if (diag || kv0 + kCols > p.N) {
                        const int hi = min(p.N, diag ? qrow + 1 : p.N) - kv0;
#pragma unroll
                        for (int t = 0; t < kCols; ++t) pv[t] = (t < hi) ? pv[t] : 0.f;
                    }
                }
                ok = mbar_wait(dp_full, ph, abort_flag, kS2Compute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < kCols / 32; ++hh) {
                    uint32_t dpr[32];
                    tmem_ld32(tmem + lane_off + kColDP + c0 + hh * 32, dpr);
                    tmem_ld_wait();
                    uint32_t wv[16];
                    const float2 sc2 = make_float2(sc, sc);
                    const float2 nd2 = make_float2(-dval, -dval);
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        // dS = P (dP - D) scale = P fma(dP, scale, -scale*D); dval = scale*D
                        const int q0 = hh * 32 + 2 * t;
                        const float2 gd = __ffma2_rn(
                            make_float2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), sc2, nd2);
                        const float2 d = __fmul2_rn(make_float2(pv[q0], pv[q0 + 1]), gd);
                        wv[t] = pack_bf16x2(d.x, d.y);
                    }
                    tmem_st16(tmem + lane_off + kColDP + c0 + hh * 16, wv);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (!ok) break;
            // ---- epilogue: dQ rows (already scaled) -> bf16; the next unit's first
            // dQ MMA overwrites these columns only after this thread's next ds_full
            ok = mbar_wait(dq_done, ui & 1, abort_flag, kS2Compute);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            constexpr int kPer = D / kGroups;   // head-dimension columns written by this group
            __nv_bfloat16* dst_row =
                reinterpret_cast<__nv_bfloat16*>(p.dq) + (static_cast<size_t>(w.bh) * p.N + qrow) * D + wg * kPer;
            float* acc_row = p.a_dq ? p.a_dq + (static_cast<size_t>(w.bh) * p.N + qrow) * D + wg * kPer : nullptr;
#pragma unroll 1
            for (int q = 0; q < kPer / 16; ++q) {
                uint32_t v16[16];
                tmem_ld16(tmem + lane_off + kColDQ + wg * kPer + q * 16, v16);
                tmem_ld_wait();
                if (acc_row) {   // accumulate mode: fp32 sums instead of bf16 outputs
                    if (qrow < p.N) accumulate16(acc_row + q * 16, v16, p.a_first_dq);
                    continue;
                }
                uint32_t pk[8];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    pk[t] = pack_bf16x2(__uint_as_float(v16[2 * t]), __uint_as_float(v16[2 * t + 1]));
                if (qrow < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + q * 16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tc_fence_before();
            gj += w.n_j;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <class Kern>
cudaError_t launch(Kern kern, unsigned grid, int smem, const CUtensorMap& tq, const CUtensorMap& tk,
                   const CUtensorMap& tv, const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    if (grid == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    // persistent: one CTA per SM walks the units
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    // (with fewer than two units per SM the hardware's own CTA dispatch is as good)
    const unsigned grid = static_cast<unsigned>(p.n_units_dkdv < 2 * sms ? p.n_units_dkdv : sms);
    if (D == 128) return launch(fa_bwd_dkdv_kernel<128>, grid, DkdvLayout<128>::kAlloc, tq, tk, tv, tdo, p, stream);
    return launch(fa_bwd_dkdv_kernel<64>, grid, DkdvLayout<64>::kAlloc, tq, tk, tv, tdo, p, stream);
}

cudaError_t launch_bwd_dq(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const unsigned grid = static_cast<unsigned>(p.n_units_dq < 2 * sms ? p.n_units_dq : sms);
    if (D == 128) return launch(fa_bwd_dq_kernel<128>, grid, DqLayout<128>::kAlloc, tq, tk, tv, tdo, p, stream);
    return launch(fa_bwd_dq_kernel<64>, grid, DqLayout<64>::kAlloc, tq, tk, tv, tdo, p, stream);
}

}  // namespace fa
