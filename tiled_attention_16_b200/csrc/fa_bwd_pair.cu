// fa_bwd_pair.cu — the dK/dV and dQ passes of the tiled attention backward
// on CTA pairs (tcgen05 cta_group::2).
//
// Same mathematics as the one-CTA dK/dV pass in fa_bwd_split.cu (recompute P
// from the saved LSE, closed-form softmax gradient dS = P o (dP - D);
// "FlashAttention V2深度解析：反向传播显存优化让大模型训练不再OOM", sections
// 改进1 and 改进2), with a 256-key block per unit: two CTAs on neighbouring
// SMs form a cluster, CTA r keeps keys [256 J + 128 r, +128) resident, and
// every product is one MMA of M = 256 key rows issued by the leader (CTA 0)
// that runs on both SMs:
//   S^T  = K Q_i^T    B = Q_i  split by query rows:   CTA r supplies rows [64 r, +64)
//   dP^T = V dO_i^T   B = dO_i split by query rows
//   dV  += P^T dO_i   B = dO_i split by head dim:     CTA r supplies columns [64 r, +64)
//   dK  += dS^T Q_i   B = Q_i  split by head dim
// so each CTA loads a Q (dO) tile as two 16 KB pieces: its row half in the
// K-major layout of the S^T (dP^T) operand and its column half, all rows, in
// the MN-major layout of the dK (dV) operand.  This is the larger key block
// of the deep dive's tuning section (性能调优技巧, block_size选择).
//
// Warp roles per CTA (320 threads): warps 0-7 compute P^T and dS^T for the
// CTA's 128 keys (two groups splitting the 128 query columns; thread = key
// row = TMEM lane), warp 8 issues the pair MMAs (leader only), warp 9 loads.
// Tensor memory per CTA: S^T/P^T | dP^T/dS^T | dV | dK, 128 columns each.
// P^T and dS^T are packed bf16 over the fp32 columns their group has read and
// feed the dV / dK MMAs from tensor memory.  Loads of both CTAs count on the
// leader's barriers; MMA completions arrive on both CTAs' barriers; each
// compute warp of either CTA arrives once on the leader's P / dS barriers.
// Units are served greedily from a work counter, heaviest causal blocks
// first: the leader's producer takes each and publishes it in both CTAs'
// shared memory.  Every wait is bounded; no load uses multicast.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kD = 128;
constexpr int kGroups = 2;
constexpr int kCols = kTileN / kGroups;           // query columns per compute group
constexpr int kComputeWarps = 4 * kGroups;
constexpr int kMmaWarp = kComputeWarps;
constexpr int kLoadWarp = kComputeWarps + 1;
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr int kMaxDynSmem = 232448;

enum PairBwdSite {
    kBPSmem = 22, kBPLoad = 23, kBPEmpty = 24, kBPMma = 25, kBPCompute = 26, kBPDrain = 27
};

__host__ __device__ constexpr uint32_t packed_col(int kk) {
    return static_cast<uint32_t>((kk / (kCols / 16)) * kCols + (kk % (kCols / 16)) * 8);
}

struct DkdvPairLayout {
    static constexpr int kTile = kTileM * kD * 2;         // 128 rows x 128 bf16 = two 16 KB atoms
    static constexpr int kAtom = kTileM * 128;
    static constexpr int kRowHalf = 64 * kD * 2;          // 64 rows x 128 bf16 = two 8 KB atoms
    static constexpr int kRowAtom = 64 * 128;
    static constexpr int kColHalf = kTileM * 64 * 2;      // 128 rows x 64 bf16 = one 16 KB atom
    static constexpr int kStage = kRowHalf + kColHalf;    // one Q or dO tile as this CTA holds it
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTile;
    static constexpr int kQ = kV + kTile;                 // 2 stages
    static constexpr int kDO = kQ + 2 * kStage;           // 2 stages
    static constexpr int kLse = kDO + 2 * kStage;         // 2 stages x 128 fp32
    static constexpr int kDvec = kLse + 2 * kTileM * 4;   // 2 stages x 128 fp32
    static constexpr int kBar = kDvec + 2 * kTileM * 4;
    static constexpr int kNumBars = 24;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "pair dK/dV shared memory layout too large");
};

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

__device__ __forceinline__ void tc_commit_pair_self(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(1)) : "memory");
}

// One pair unit: (batch, K/V head, 256-key block J).  Numbered head group by
// head group, J ascending inside a group (heaviest first when causal), then
// head.  Query tiles i >= 2 J when causal (the first one is fully masked for
// CTA 1's keys), all otherwise; for every query head of the GQA group.
struct PairDkdvUnit {
    int J, bkv, b, hkv, i0, per_head, n_it;
};

__device__ __forceinline__ PairDkdvUnit pair_dkdv_unit(const BwdParams& p, int T, int TJ, int u) {
    PairDkdvUnit w;
    const int BHkv = p.B * p.Hkv;
    const int grp = u / (p.heads_per_group * TJ);
    const int h0 = grp * p.heads_per_group;
    const int nh = min(p.heads_per_group, BHkv - h0);
    const int rr = u - grp * p.heads_per_group * TJ;
    w.J = rr / nh;
    w.bkv = h0 + (rr - w.J * nh);
    w.b = w.bkv / p.Hkv;
    w.hkv = w.bkv - w.b * p.Hkv;
    w.i0 = p.causal ? 2 * w.J : 0;
    w.per_head = T - w.i0;
    w.n_it = (p.Hq / p.Hkv) * w.per_head;
    return w;
}

// Readers of each published unit id: the leader's MMA thread and compute
// warps, the peer's producer and compute warps.
constexpr int kUnitConsumers = 1 + kComputeWarps + 1 + kComputeWarps;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
fa_bwd_dkdv_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQh,
                        const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmDOh,
                        const BwdParams p) {
    using L = DkdvPairLayout;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {   // same in both CTAs of the pair
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kBPSmem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* kv_full = bars + 0;      // leader: K and V of both CTAs
    uint64_t* kv_empty = bars + 1;     // both
    uint64_t* q_full = bars + 2;       // [2] leader
    uint64_t* q_empty = bars + 4;      // [2] both
    uint64_t* do_full = bars + 6;      // [2] leader
    uint64_t* do_empty = bars + 8;     // [2] both
    uint64_t* st_full = bars + 10;     // [2] own: this CTA's copy of the tile's lse2 and scale * D
    uint64_t* s_full = bars + 12;      // both
    uint64_t* dp_full = bars + 13;     // both
    uint64_t* p_full0 = bars + 14;     // leader: one arrival per compute warp of either CTA
    uint64_t* p_full1 = bars + 15;     // leader
    uint64_t* ds_full = bars + 16;     // leader
    uint64_t* dkv_full = bars + 17;    // both
    uint64_t* drain = bars + 18;       // leader
    uint64_t* unit_full = bars + 20;   // [2] both: the leader published a unit id in this CTA
    uint64_t* unit_empty = bars + 22;  // [2] leader: every consumer of both CTAs has read the slot
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);   // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);
    const int T = (p.N + kTileM - 1) / kTileM;
    const int TJ = (p.N + 2 * kTileN - 1) / (2 * kTileN);
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
            mbar_init(&st_full[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full0, 2 * kComputeWarps);
        mbar_init(p_full1, 2 * kComputeWarps);
        mbar_init(ds_full, 2 * kComputeWarps);
        mbar_init(dkv_full, 1);
        mbar_init(drain, 1);
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&unit_full[s2], 1);
            mbar_init(&unit_empty[s2], kUnitConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();    // both CTAs' barriers exist before anything crosses the pair
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

    // Unit ring: the leader's producer takes units from the work counter
    // (greedy, heaviest first) and publishes each id in both CTAs; every
    // consumer reads it and releases the slot on the leader's barrier.
    const uint32_t l_unit_empty0 = mapa_shared(smem_u32(&unit_empty[0]), 0);
    auto take_unit = [&](int k, bool per_warp, bool& ok) -> int {
        const int s = k & 1;
        ok = rank == 0 ? mbar_wait(&unit_full[s], (k >> 1) & 1, abort_flag, kBPLoad)
                       : mbar_wait_acq_cluster(&unit_full[s], (k >> 1) & 1, abort_flag, kBPLoad);
        const int u = ok ? unit_id[s] : -1;
        if (per_warp) __syncwarp();
        if (!per_warp || lane == 0) mbar_arrive_remote(l_unit_empty0 + 8u * static_cast<uint32_t>(s));
        return u;
    };
    // Leader's producer: publish unit `u` (-1: no more) in slot k & 1 of both CTAs.
    auto publish_unit = [&](int k, int u) -> bool {
        const int s = k & 1;
        if (k >= 2 && !mbar_wait(&unit_empty[s], ((k >> 1) - 1) & 1, abort_flag, kBPEmpty)) return false;
        unit_id[s] = u;
        st_shared_cluster(mapa_shared(smem_u32(const_cast<int*>(&unit_id[s])), 1), u);
        mbar_arrive(&unit_full[s]);
        mbar_arrive_remote_release(mapa_shared(smem_u32(&unit_full[s]), 1));
        return true;
    };

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmQh);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            tma_prefetch_desc(&tmDOh);
            const int rk = static_cast<int>(rank);
            const uint32_t l_kv = mapa_shared(smem_u32(kv_full), 0);
            uint32_t l_q[2], l_do[2];
            for (int s = 0; s < 2; ++s) {
                l_q[s] = mapa_shared(smem_u32(&q_full[s]), 0);
                l_do[s] = mapa_shared(smem_u32(&do_full[s]), 0);
            }
            int g = 0;                         // query-tile iterations of the pair so far (all units)
            int n_q = 0, n_do = 0, n_kv = 0;   // loads issued
            bool ok = true;
            int next = pair;   // the leader's next unit: first its pair index, then from the counter
            for (int k = 0; ok; ++k) {
                int u;
                if (rank == 0) {
                    u = next < n_units ? next : -1;
                    if (!(ok = publish_unit(k, u))) break;
                } else {
                    u = take_unit(k, false, ok);
                    if (!ok) break;
                }
                if (u < 0) break;
                if (rank == 0) next = npairs + static_cast<int>(atomicAdd(p.sched + 0, 1u));
                const PairDkdvUnit w = pair_dkdv_unit(p, T, TJ, u);
                if (k >= 1 && !(ok = mbar_wait(kv_empty, (k - 1) & 1, abort_flag, kBPEmpty))) break;
                if (rank == 0) mbar_arrive_expect_tx(kv_full, 2 * 2 * L::kTile);
                for (int a = 0; a < kD / 64; ++a) {
                    tma_load_3d_pair(smem + L::kK + a * L::kAtom, &tmK, l_kv, a * 64, w.J * 2 * kTileN + rk * kTileN, w.bkv);
                    tma_load_3d_pair(smem + L::kV + a * L::kAtom, &tmV, l_kv, a * 64, w.J * 2 * kTileN + rk * kTileN, w.bkv);
                }
                n_kv = k + 1;
                for (int it = 0; ok && it < w.n_it; ++it, ++g) {
                    const int st = g & 1;
                    const int gh = it / w.per_head;
                    const int i = w.i0 + (it - gh * w.per_head);
                    const int bhq = w.b * p.Hq + w.hkv * G + gh;
                    if (g >= 2 && !(ok = mbar_wait(&q_empty[st], ((g >> 1) - 1) & 1, abort_flag, kBPEmpty))) break;
                    if (rank == 0) mbar_arrive_expect_tx(&q_full[st], 2 * L::kStage);
                    uint8_t* qs = smem + L::kQ + st * L::kStage;
                    for (int a = 0; a < kD / 64; ++a)   // row half (K-major), both column atoms
                        tma_load_3d_pair(qs + a * L::kRowAtom, &tmQh, l_q[st], a * 64, i * kTileM + 64 * rk, bhq);
                    tma_load_3d_pair(qs + L::kRowHalf, &tmQ, l_q[st], 64 * rk, i * kTileM, bhq);   // column half
                    const size_t srow = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * kTileM;
                    mbar_arrive_expect_tx(&st_full[st], 2 * kTileM * 4);
                    bulk_load(smem + L::kLse + st * kTileM * 4, p.lse2 + srow, kTileM * 4, &st_full[st]);
                    bulk_load(smem + L::kDvec + st * kTileM * 4, p.dvec + srow, kTileM * 4, &st_full[st]);
                    n_q = g + 1;
                    if (g >= 2 && !(ok = mbar_wait(&do_empty[st], ((g >> 1) - 1) & 1, abort_flag, kBPEmpty))) break;
                    if (rank == 0) mbar_arrive_expect_tx(&do_full[st], 2 * L::kStage);
                    uint8_t* ds = smem + L::kDO + st * L::kStage;
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d_pair(ds + a * L::kRowAtom, &tmDOh, l_do[st], a * 64, i * kTileM + 64 * rk, bhq);
                    tma_load_3d_pair(ds + L::kRowHalf, &tmDO, l_do[st], 64 * rk, i * kTileM, bhq);
                    n_do = g + 1;
                }
            }
            // The leader's full barriers count both CTAs' tensor copies; the
            // leader waits for the last phases it armed, the final cluster
            // barrier keeps the peer resident until then.  Row statistics
            // land on each CTA's own barrier.
            if (rank == 0) {
                if (n_kv > 0) wait_drain(kv_full, (n_kv - 1) & 1, kBPDrain);
                for (int q = (n_q > 2 ? n_q - 2 : 0); q < n_q; ++q) wait_drain(&q_full[q & 1], (q >> 1) & 1, kBPDrain);
                for (int q = (n_do > 2 ? n_do - 2 : 0); q < n_do; ++q) wait_drain(&do_full[q & 1], (q >> 1) & 1, kBPDrain);
            }
            for (int q = (n_q > 2 ? n_q - 2 : 0); q < n_q; ++q) wait_drain(&st_full[q & 1], (q >> 1) & 1, kBPDrain);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t kIdSq = idesc_bf16_f32(2 * kTileN, kTileM, 0, 0);   // S^T, dP^T
            constexpr uint32_t kIdAcc = idesc_bf16_f32(2 * kTileN, kD, 0, 1);      // dV, dK (A from TMEM)
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            auto issue_dk = [&](int gp, bool first) {
                const uint32_t qc = q_base + (gp & 1) * L::kStage + L::kRowHalf;
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)
                    mma_ts_pair(tmem + kColDK, tmem + kColDP + packed_col(kk), sdesc_sw128(qc + kk * 2048, L::kColHalf, 1024),
                                kIdAcc, (!first || kk > 0));
                tc_commit_pair(&q_empty[gp & 1]);
            };
            bool ok = true;
            int g = 0;
            for (int k = 0; ok; ++k) {
                const int u = take_unit(k, false, ok);
                if (!ok || u < 0) break;
                const int n_it = pair_dkdv_unit(p, T, TJ, u).n_it;
                if (!(ok = mbar_wait(kv_full, k & 1, abort_flag, kBPLoad))) break;
                for (int it = 0; it < n_it; ++it) {
                    const int gi = g + it;
                    const int st = gi & 1;
                    const uint32_t sph = (gi >> 1) & 1;
                    const uint32_t ph = gi & 1;
                    if (!(ok = mbar_wait(&q_full[st], sph, abort_flag, kBPLoad))) break;
                    tc_fence_after();
                    const uint32_t qr = q_base + st * L::kStage;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss_pair(tmem + kColS, sdesc_sw128(k_base + (kk >> 2) * L::kAtom + (kk & 3) * 32, 16, 1024),
                                    sdesc_sw128(qr + (kk >> 2) * L::kRowAtom + (kk & 3) * 32, 16, 1024), kIdSq, kk > 0);
                    tc_commit_pair(s_full);
                    if (it > 0) {
                        if (!(ok = mbar_wait_cluster(ds_full, ph ^ 1, abort_flag, kBPMma))) break;
                        tc_fence_after();
                        issue_dk(gi - 1, it == 1);
                    }
                    if (!(ok = mbar_wait(&do_full[st], sph, abort_flag, kBPLoad))) break;
                    tc_fence_after();
                    const uint32_t dr = do_base + st * L::kStage;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        mma_ss_pair(tmem + kColDP, sdesc_sw128(v_base + (kk >> 2) * L::kAtom + (kk & 3) * 32, 16, 1024),
                                    sdesc_sw128(dr + (kk >> 2) * L::kRowAtom + (kk & 3) * 32, 16, 1024), kIdSq, kk > 0);
                    tc_commit_pair(dp_full);
                    if (it == n_it - 1) tc_commit_pair(kv_empty);   // K and V no longer read by this unit
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = mbar_wait_cluster(h == 0 ? p_full0 : p_full1, ph, abort_flag, kBPMma))) break;
                        tc_fence_after();
#pragma unroll
                        for (int g2 = 0; g2 < kGroups; ++g2) {
#pragma unroll
                            for (int t = 0; t < kCols / 32; ++t) {
                                const int kk = g2 * (kCols / 16) + h * (kCols / 32) + t;
                                mma_ts_pair(tmem + kColDV, tmem + kColS + packed_col(kk),
                                            sdesc_sw128(dr + L::kRowHalf + kk * 2048, L::kColHalf, 1024), kIdAcc,
                                            (it > 0 || kk > 0));
                            }
                        }
                    }
                    if (!ok) break;
                    tc_commit_pair(&do_empty[st]);
                }
                if (!ok) break;
                const int gl = g + n_it - 1;
                if (!(ok = mbar_wait_cluster(ds_full, gl & 1, abort_flag, kBPMma))) break;
                tc_fence_after();
                issue_dk(gl, n_it == 1);
                tc_commit_pair(dkv_full);
                g += n_it;
            }
            tc_commit_pair_self(drain);
            wait_drain(drain, 0, kBPDrain);
        }
    } else {
        // ------------------------------------------------------------ compute (both CTAs: P^T, dS^T)
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int r = (wq << 5) + lane;  // key row of this CTA's block = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * kCols;       // this group's query columns
        const float c = p.scale_log2;
        const float sc = p.scale;
        const uint32_t l_p0 = mapa_shared(smem_u32(p_full0), 0);
        const uint32_t l_p1 = mapa_shared(smem_u32(p_full1), 0);
        const uint32_t l_ds = mapa_shared(smem_u32(ds_full), 0);
        float pv[kCols];
        bool ok = true;
        int g = 0;
        for (int k = 0; ok; ++k) {
            const int u = take_unit(k, true, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const PairDkdvUnit w = pair_dkdv_unit(p, T, TJ, u);
            const int jr = 2 * w.J + static_cast<int>(rank);   // this CTA's 128-key block
            const int kv = jr * kTileN + r;
            const bool kv_ok = kv < p.N;
            const bool kv_block_partial = (jr + 1) * kTileN > p.N;
            for (int it = 0; it < w.n_it; ++it) {
                const int gi = g + it;
                const int st = gi & 1;
                const uint32_t ph = gi & 1;
                const int gh = it / w.per_head;
                const int i = w.i0 + (it - gh * w.per_head);
                const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse + st * kTileM * 4) + c0;
                const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvec + st * kTileM * 4) + c0;
                ok = mbar_wait(&st_full[st], (gi >> 1) & 1, abort_flag, kBPCompute) &&
                     mbar_wait(s_full, ph, abort_flag, kBPCompute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                {
                    uint32_t sr[kCols / 32][32];
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) tmem_ld32(tmem + lane_off + kColS + c0 + h * 32, sr[h]);
                    tmem_ld_wait();
                    const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
                    // Causal: query tile i before this CTA's key block is fully
                    // masked (CTA 1's first tile), i == jr is the diagonal;
                    // a partial last key block masks key rows past N.  All
                    // tests are uniform across the warp; columns q < lo are 0.
                    const bool full = p.causal && i < jr;
                    const bool diag = p.causal && i == jr;
                    const bool masked = full || diag || kv_block_partial;
                    const int lo = (!kv_ok || full) ? kCols : (diag ? r - c0 : 0);
                    const float2 c2 = make_float2(c, c);
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
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(h == 0 ? l_p0 : l_p1);
                    });
                }
                ok = mbar_wait(dp_full, ph, abort_flag, kBPCompute);
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
                    tmem_st16(tmem + lane_off + kColDP + c0 + h * 16, wv);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(l_ds);
            }
            if (!ok) break;
            // ---- epilogue: dV, dK rows of this CTA's keys (summed over the group)
            ok = mbar_wait(dkv_full, k & 1, abort_flag, kBPCompute);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const size_t row = static_cast<size_t>(w.bkv) * p.N + kv;
            constexpr int kPer = kD / kGroups;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t col0 = (which == 0 ? kColDV : kColDK) + wg * kPer;
                __nv_bfloat16* dst_row =
                    reinterpret_cast<__nv_bfloat16*>(which == 0 ? p.dv : p.dk) + row * kD + wg * kPer;
#pragma unroll 1
                for (int q = 0; q < kPer / 16; ++q) {
                    uint32_t v16[16];
                    tmem_ld16(tmem + lane_off + col0 + q * 16, v16);
                    tmem_ld_wait();
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
            // the next unit's dV / dK MMAs overwrite these columns only after
            // every compute warp's next P^T arrival, which follows these loads
            tc_fence_before();
            g += w.n_it;
        }
    }
    // Neither CTA releases tensor or shared memory while the pair can still
    // touch it (the leader's MMAs read both CTAs' operands and write both
    // CTAs' accumulators; the peer's warps arrive on the leader's barriers).
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

// ===========================================================================
// dQ pass on CTA pairs
// ===========================================================================
// Unit: (batch x query head bh, 256-query block I); CTA r owns query tile
// 2 I + r and keeps its Q and dO resident while the key tiles j stream past
// (j <= 2 I + 1 when causal: CTA 0's rows see the last tile fully masked):
//   S  = Q K_j^T    B = K_j split by key rows:  CTA r supplies keys [64 r, +64)
//   dP = dO V_j^T   B = V_j split by key rows
//   dQ += dS K_j    B = K_j split by head dim:  CTA r supplies columns [64 r, +64)
// dS is packed bf16 over the dP block and read from tensor memory; dQ
// accumulates in tensor memory and is written once as bf16.
struct DqPairLayout {
    static constexpr int kStages = 3;
    static constexpr int kTile = kTileM * kD * 2;
    static constexpr int kAtom = kTileM * 128;
    static constexpr int kRowHalf = 64 * kD * 2;          // 64 key rows x 128 bf16: two 8 KB atoms
    static constexpr int kRowAtom = 64 * 128;
    static constexpr int kColHalf = kTileN * 64 * 2;      // 128 key rows x 64 bf16: one 16 KB atom
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTile;
    static constexpr int kK = kDO + kTile;                // kStages x (row half, column half)
    static constexpr int kKStage = kRowHalf + kColHalf;
    static constexpr int kV = kK + kStages * kKStage;     // kStages x row half
    static constexpr int kBar = kV + kStages * kRowHalf;
    static constexpr int kNumBars = 2 + 3 * kStages + 11;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "pair dQ shared memory layout too large");
};

struct PairDqUnit {
    int I, bh, kvh, n_j;
};

__device__ __forceinline__ PairDqUnit pair_dq_unit(const BwdParams& p, int T, int TI, int u) {
    PairDqUnit w;
    const int BH = p.B * p.Hq;
    const int grp = u / (p.dq_heads_per_group * TI);
    const int h0 = grp * p.dq_heads_per_group;
    const int nh = min(p.dq_heads_per_group, BH - h0);
    const int rr = u - grp * p.dq_heads_per_group * TI;
    w.I = TI - 1 - rr / nh;
    w.bh = h0 + (rr % nh);
    const int b = w.bh / p.Hq;
    const int h = w.bh - b * p.Hq;
    w.kvh = b * p.Hkv + h / (p.Hq / p.Hkv);
    w.n_j = p.causal ? min(T, 2 * w.I + 2) : T;
    return w;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
fa_bwd_dq_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmVh,
                      const __grid_constant__ CUtensorMap tmDO, const BwdParams p) {
    using L = DqPairLayout;
    constexpr int S = L::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {   // same in both CTAs of the pair
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kBPSmem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;           // leader: Q and dO of both CTAs
    uint64_t* q_empty = bars + 1;          // both
    uint64_t* k_full = bars + 2;           // [S] leader
    uint64_t* v_full = k_full + S;         // [S] leader
    uint64_t* kv_empty = v_full + S;       // [S] both
    uint64_t* s_full = kv_empty + S;       // both
    uint64_t* s_free = s_full + 1;         // leader: one arrival per compute warp of either CTA
    uint64_t* dp_full = s_full + 2;        // both
    uint64_t* ds_full = s_full + 3;        // leader
    uint64_t* dq_done = s_full + 4;        // both
    uint64_t* drain = s_full + 5;          // leader
    uint64_t* unit_full = s_full + 7;      // [2] both: the leader published a unit id in this CTA
    uint64_t* unit_empty = s_full + 9;     // [2] leader: every consumer of both CTAs has read the slot
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);   // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);
    const int T = (p.N + kTileM - 1) / kTileM;
    const int TI = (p.N + 2 * kTileM - 1) / (2 * kTileM);
    const int n_units = p.n_units_dq;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int st = 0; st < S; ++st) {
            mbar_init(&k_full[st], 1);
            mbar_init(&v_full[st], 1);
            mbar_init(&kv_empty[st], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 2 * kComputeWarps);
        mbar_init(dp_full, 1);
        mbar_init(ds_full, 2 * kComputeWarps);
        mbar_init(dq_done, 1);
        mbar_init(drain, 1);
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&unit_full[s2], 1);
            mbar_init(&unit_empty[s2], kUnitConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;

    // Unit ring: the leader's producer takes units from the work counter
    // (greedy, heaviest first) and publishes each id in both CTAs; every
    // consumer reads it and releases the slot on the leader's barrier.
    const uint32_t l_unit_empty0 = mapa_shared(smem_u32(&unit_empty[0]), 0);
    auto take_unit = [&](int k, bool per_warp, bool& ok) -> int {
        const int s = k & 1;
        ok = rank == 0 ? mbar_wait(&unit_full[s], (k >> 1) & 1, abort_flag, kBPLoad)
                       : mbar_wait_acq_cluster(&unit_full[s], (k >> 1) & 1, abort_flag, kBPLoad);
        const int u = ok ? unit_id[s] : -1;
        if (per_warp) __syncwarp();
        if (!per_warp || lane == 0) mbar_arrive_remote(l_unit_empty0 + 8u * static_cast<uint32_t>(s));
        return u;
    };
    // Leader's producer: publish unit `u` (-1: no more) in slot k & 1 of both CTAs.
    auto publish_unit = [&](int k, int u) -> bool {
        const int s = k & 1;
        if (k >= 2 && !mbar_wait(&unit_empty[s], ((k >> 1) - 1) & 1, abort_flag, kBPEmpty)) return false;
        unit_id[s] = u;
        st_shared_cluster(mapa_shared(smem_u32(const_cast<int*>(&unit_id[s])), 1), u);
        mbar_arrive(&unit_full[s]);
        mbar_arrive_remote_release(mapa_shared(smem_u32(&unit_full[s]), 1));
        return true;
    };

    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmKh);
            tma_prefetch_desc(&tmVh);
            tma_prefetch_desc(&tmDO);
            const int rk = static_cast<int>(rank);
            const uint32_t l_q = mapa_shared(smem_u32(q_full), 0);
            int gj = 0;               // key tiles of the pair so far (all units)
            int n_kv = 0, n_q = 0;    // loads issued
            bool ok = true;
            int next = pair;
            for (int k = 0; ok; ++k) {
                int u;
                if (rank == 0) {
                    u = next < n_units ? next : -1;
                    if (!(ok = publish_unit(k, u))) break;
                } else {
                    u = take_unit(k, false, ok);
                    if (!ok) break;
                }
                if (u < 0) break;
                if (rank == 0) next = npairs + static_cast<int>(atomicAdd(p.sched + 1, 1u));
                const PairDqUnit w = pair_dq_unit(p, T, TI, u);
                if (k >= 1 && !(ok = mbar_wait(q_empty, (k - 1) & 1, abort_flag, kBPEmpty))) break;
                if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * 2 * L::kTile);
                const int row0 = (2 * w.I + rk) * kTileM;
                for (int a = 0; a < kD / 64; ++a) {
                    tma_load_3d_pair(smem + L::kQ + a * L::kAtom, &tmQ, l_q, a * 64, row0, w.bh);
                    tma_load_3d_pair(smem + L::kDO + a * L::kAtom, &tmDO, l_q, a * 64, row0, w.bh);
                }
                n_q = k + 1;
                for (int jj = 0; jj < w.n_j; ++jj, ++gj) {
                    const int st = gj % S;
                    if (gj >= S && !(ok = mbar_wait(&kv_empty[st], ((gj / S) - 1) & 1, abort_flag, kBPEmpty))) break;
                    const uint32_t lk = mapa_shared(smem_u32(&k_full[st]), 0);
                    const uint32_t lv = mapa_shared(smem_u32(&v_full[st]), 0);
                    uint8_t* ks = smem + L::kK + st * L::kKStage;
                    if (rank == 0) mbar_arrive_expect_tx(&k_full[st], 2 * L::kKStage);
                    for (int a = 0; a < kD / 64; ++a)   // key-row half (K-major): operand of S
                        tma_load_3d_pair(ks + a * L::kRowAtom, &tmKh, lk, a * 64, jj * kTileN + 64 * rk, w.kvh);
                    tma_load_3d_pair(ks + L::kRowHalf, &tmK, lk, 64 * rk, jj * kTileN, w.kvh);   // column half: dQ
                    if (rank == 0) mbar_arrive_expect_tx(&v_full[st], 2 * L::kRowHalf);
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d_pair(smem + L::kV + st * L::kRowHalf + a * L::kRowAtom, &tmVh, lv, a * 64,
                                         jj * kTileN + 64 * rk, w.kvh);
                    n_kv = gj + 1;
                }
            }
            if (rank == 0) {
                if (n_q > 0) wait_drain(q_full, (n_q - 1) & 1, kBPDrain);
                for (int g = (n_kv > S ? n_kv - S : 0); g < n_kv; ++g) {
                    wait_drain(&k_full[g % S], (g / S) & 1, kBPDrain);
                    wait_drain(&v_full[g % S], (g / S) & 1, kBPDrain);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(2 * kTileM, kTileN, 0, 0);   // S, dP: K-major both
            constexpr uint32_t kIdDQ = idesc_bf16_f32(2 * kTileM, kD, 0, 1);      // dQ: A (dS) TMEM, B MN-major
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            auto issue_s = [&](int st) {
                const uint32_t kr = k_base + st * L::kKStage;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss_pair(tmem + kColS, sdesc_sw128(q_base + (kk >> 2) * L::kAtom + (kk & 3) * 32, 16, 1024),
                                sdesc_sw128(kr + (kk >> 2) * L::kRowAtom + (kk & 3) * 32, 16, 1024), kIdS, kk > 0);
                tc_commit_pair(s_full);
            };
            auto issue_dp = [&](int st) {
                const uint32_t vr = v_base + st * L::kRowHalf;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss_pair(tmem + kColDP, sdesc_sw128(do_base + (kk >> 2) * L::kAtom + (kk & 3) * 32, 16, 1024),
                                sdesc_sw128(vr + (kk >> 2) * L::kRowAtom + (kk & 3) * 32, 16, 1024), kIdS, kk > 0);
                tc_commit_pair(dp_full);
            };
            bool ok = true;
            int gj = 0;
            for (int k = 0; ok; ++k) {
                const int u = take_unit(k, false, ok);
                if (!ok || u < 0) break;
                const int n_j = pair_dq_unit(p, T, TI, u).n_j;
                if (!(ok = mbar_wait(q_full, k & 1, abort_flag, kBPLoad))) break;
                if (gj > 0 && !(ok = mbar_wait_cluster(s_free, (gj - 1) & 1, abort_flag, kBPMma))) break;
                if (!(ok = mbar_wait(&k_full[gj % S], (gj / S) & 1, abort_flag, kBPLoad))) break;
                tc_fence_after();
                issue_s(gj % S);
                if (!(ok = mbar_wait(&v_full[gj % S], (gj / S) & 1, abort_flag, kBPLoad))) break;
                tc_fence_after();
                issue_dp(gj % S);
                if (n_j == 1) tc_commit_pair(q_empty);
                for (int jj = 0; jj < n_j; ++jj) {
                    const int G = gj + jj;
                    const int st = G % S;
                    const int st1 = (G + 1) % S;
                    const uint32_t ph = G & 1;
                    if (jj + 1 < n_j) {
                        if (!(ok = mbar_wait_cluster(s_free, ph, abort_flag, kBPMma))) break;
                        if (!(ok = mbar_wait(&k_full[st1], ((G + 1) / S) & 1, abort_flag, kBPLoad))) break;
                        tc_fence_after();
                        issue_s(st1);
                    }
                    if (!(ok = mbar_wait_cluster(ds_full, ph, abort_flag, kBPMma))) break;
                    tc_fence_after();
                    const uint32_t kc = k_base + st * L::kKStage + L::kRowHalf;
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)
                        mma_ts_pair(tmem + kColDQ, tmem + kColDP + packed_col(kk),
                                    sdesc_sw128(kc + kk * 2048, L::kColHalf, 1024), kIdDQ, (jj > 0 || kk > 0));
                    tc_commit_pair(&kv_empty[st]);
                    if (jj + 1 < n_j) {
                        if (!(ok = mbar_wait(&v_full[st1], ((G + 1) / S) & 1, abort_flag, kBPLoad))) break;
                        tc_fence_after();
                        issue_dp(st1);
                        if (jj + 2 == n_j) tc_commit_pair(q_empty);
                    }
                }
                if (!ok) break;
                tc_commit_pair(dq_done);
                gj += n_j;
            }
            tc_commit_pair_self(drain);
            wait_drain(drain, 0, kBPDrain);
        }
    } else {
        // ------------------------------------------------------------ compute (both CTAs: P, dS)
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int r = (wq << 5) + lane;  // query row of this CTA's tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * kCols;       // this group's key columns
        const float c = p.scale_log2;
        const float sc = p.scale;
        const uint32_t l_sfree = mapa_shared(smem_u32(s_free), 0);
        const uint32_t l_ds = mapa_shared(smem_u32(ds_full), 0);
        float pv[kCols];
        bool ok = true;
        int gj = 0;
        for (int k = 0; ok; ++k) {
            const int u = take_unit(k, true, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const PairDqUnit w = pair_dq_unit(p, T, TI, u);
            const int ir = 2 * w.I + static_cast<int>(rank);   // this CTA's query tile
            const int qrow = ir * kTileM + r;
            const bool row_ok = qrow < p.N;                    // CTA 1's tile may lie past N (and past Npad)
            const size_t srow = static_cast<size_t>(w.bh) * p.Npad + static_cast<size_t>(row_ok ? qrow : 0);
            const float lse2 = row_ok ? p.lse2[srow] : INFINITY;   // +inf: P = 0
            const float dval = row_ok ? p.dvec[srow] : 0.f;       // scale * D
            for (int jj = 0; jj < w.n_j; ++jj) {
                const uint32_t ph = (gj + jj) & 1;
                ok = mbar_wait(s_full, ph, abort_flag, kBPCompute);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                {
                    uint32_t sr[kCols / 32][32];
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) tmem_ld32(tmem + lane_off + kColS + c0 + h * 32, sr[h]);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(l_sfree);
                    const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
                    const int kv0 = jj * kTileN + c0;
                    // Masked on and after the causal diagonal tile (CTA 0 sees
                    // the pair's last key tile entirely above its rows) and on
                    // a partial last key tile: key columns t >= hi are zero.
                    const float2 c2 = make_float2(c, c);
                    const float2 nl2 = make_float2(-lse2, -lse2);
                    static_for<0, kCols / 2>([&](auto tc) {
                        constexpr int t = 2 * decltype(tc)::value;
                        const float2 x = __ffma2_rn(make_float2(sv[t], sv[t + 1]), c2, nl2);
                        pv[t] = exp2_mixed<t>(x.x);
                        pv[t + 1] = exp2_mixed<t + 1>(x.y);
                    });
                    if ((p.causal && jj >= ir) || kv0 + kCols > p.N) {
                        const int hi = min(p.N, p.causal ? qrow + 1 : p.N) - kv0;
#pragma unroll
                        for (int t = 0; t < kCols; ++t) pv[t] = (t < hi) ? pv[t] : 0.f;
                    }
                }
                ok = mbar_wait(dp_full, ph, abort_flag, kBPCompute);
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
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(l_ds);
            }
            if (!ok) break;
            // ---- epilogue: this CTA's dQ rows (already scaled) -> bf16; the next
            // unit's first dQ MMA overwrites them only after every compute warp's
            // next dS arrival, which follows these loads
            ok = mbar_wait(dq_done, k & 1, abort_flag, kBPCompute);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            constexpr int kPer = kD / kGroups;
            __nv_bfloat16* dst_row = reinterpret_cast<__nv_bfloat16*>(p.dq) +
                                     (static_cast<size_t>(w.bh) * p.N + qrow) * kD + wg * kPer;
#pragma unroll 1
            for (int q = 0; q < kPer / 16; ++q) {
                uint32_t v16[16];
                tmem_ld16(tmem + lane_off + kColDQ + wg * kPer + q * 16, v16);
                tmem_ld_wait();
                uint32_t pk[8];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    pk[t] = pack_bf16x2(__uint_as_float(v16[2 * t]), __uint_as_float(v16[2 * t + 1]));
                if (row_ok) {
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
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

int dkdv_pair_max_pairs() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cache[dev] == 0) {
        if (cudaFuncSetAttribute(fa_bwd_dkdv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DkdvPairLayout::kAlloc) != cudaSuccess)
            return -1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 148, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = DkdvPairLayout::kAlloc;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, fa_bwd_dkdv_pair_kernel, &cfg) != cudaSuccess || n <= 0) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

int dq_pair_max_pairs() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cache[dev] == 0) {
        if (cudaFuncSetAttribute(fa_bwd_dq_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DqPairLayout::kAlloc) != cudaSuccess)
            return -1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 148, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = DqPairLayout::kAlloc;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, fa_bwd_dq_pair_kernel, &cfg) != cudaSuccess || n <= 0) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace

cudaError_t launch_bwd_dq_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tk_half,
                               const CUtensorMap& tv_half, const CUtensorMap& tdo, const BwdParams& p,
                               cudaStream_t stream) {
    if (p.n_units_dq == 0) return cudaSuccess;
    const int max_pairs = dq_pair_max_pairs();
    if (max_pairs <= 0) return cudaErrorInvalidConfiguration;
    const int pairs = p.n_units_dq < max_pairs ? p.n_units_dq : max_pairs;
    cudaError_t e = cudaFuncSetAttribute(fa_bwd_dq_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DqPairLayout::kAlloc);
    if (e != cudaSuccess) return e;
    fa_bwd_dq_pair_kernel<<<2 * pairs, kThreads, DqPairLayout::kAlloc, stream>>>(tq, tk, tk_half, tv_half, tdo, p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv_pair(const CUtensorMap& tq, const CUtensorMap& tq_half, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdo_half,
                                 const BwdParams& p, cudaStream_t stream) {
    if (p.n_units_dkdv == 0) return cudaSuccess;
    const int max_pairs = dkdv_pair_max_pairs();
    if (max_pairs <= 0) return cudaErrorInvalidConfiguration;
    const int pairs = p.n_units_dkdv < max_pairs ? p.n_units_dkdv : max_pairs;
    cudaError_t e = cudaFuncSetAttribute(fa_bwd_dkdv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DkdvPairLayout::kAlloc);
    if (e != cudaSuccess) return e;
    fa_bwd_dkdv_pair_kernel<<<2 * pairs, kThreads, DkdvPairLayout::kAlloc, stream>>>(tq, tq_half, tk, tv, tdo,
                                                                                     tdo_half, p);
    return cudaGetLastError();
}

}  // namespace fa
