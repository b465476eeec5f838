// fa_fwd_pair.cu — tiled attention forward on CTA pairs (tcgen05 cta_group::2).
//
// The same computation as fa_fwd.cu (tiling and incremental softmax of
// "【词汇专栏】FlashAttention：大模型训练的加速器", sections 2.1-2.3, and
// "FlashAttention 在昇腾NPU上到底快在哪", sections 二 and 三), with a larger
// query block: two CTAs on neighbouring SMs form a thread-block cluster and
// every S = Q K^T and O += P V product is one MMA of M = 256 query rows that
// runs on both SMs' tensor cores at once.  This is the larger block the
// deep dive's tuning section ("FlashAttention V2深度解析：反向传播显存优化让大
// 模型训练不再OOM", 性能调优技巧, block_size选择) recommends for long sequences.
//
// Work unit: (batch x head, block of 512 query rows).  CTA r (0 or 1) of the
// pair owns rows [m0 + 256 t + 128 r, +128) of query tile t (t = 0, 1) and
// keeps them in its shared memory; the unit's K/V tiles stream past both.
// For a 128-key tile the pair splits the operands it shares:
//   S_t  = Q_t K^T : B = K, split by key rows  -> CTA r loads keys [64 r, 64 r + 64)
//   O_t += P_t V   : B = V, split by head dim -> CTA r loads columns [64 r, 64 r + 64)
// so each CTA moves half a K tile and half a V tile per step, and the MMA
// thread of the leader (CTA 0) issues one instruction where the one-CTA
// kernel issues two.
//
// Warp roles (320 threads per CTA), as in the one-CTA kernel:
//   warps 0-3 / 4-7  softmax, O correction and epilogue of the CTA's rows of
//                    query tile 0 / 1 (thread = row = TMEM lane)
//   warp  8          MMA issuer (one thread, leader CTA only)
//   warp  9          TMA producer (each CTA loads its own halves)
// Tensor memory per CTA: S0 | S1 | O0 | O1, 128 columns each (the pair MMA
// writes each CTA's 128 rows into that CTA's tensor memory).
//
// Synchronisation across the pair:
//   * loads of both CTAs count their bytes on the leader's full barriers;
//   * the leader's MMA completions arrive on the barriers of both CTAs
//     (commit with a CTA mask), which release the stages for both producers
//     and hand S and O to both CTAs' softmax warps;
//   * each softmax warp of either CTA arrives once on the leader's P barrier.
// Units are served greedily (heaviest causal blocks first): the leader's
// producer takes each from the launch's counter slot and publishes it in both
// CTAs' shared memory; the peer's producer and softmax warps read it there.
// Every wait is bounded; no load uses multicast.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kThreads = 320;
constexpr int kD = 128;
constexpr int kStages = 3;
// Readers of each published unit id: the leader's MMA thread and 8 softmax
// warps, the peer's producer and 8 softmax warps.
constexpr int kUnitConsumers = 1 + 8 + 1 + 8;
constexpr float kRescaleThreshold = 8.0f;

enum PairSite { kPSiteQ = 0, kPSiteK = 1, kPSiteV = 2, kPSiteKVEmpty = 3, kPSiteS = 4, kPSiteP = 5, kPSiteO = 6,
                kPSiteDrain = 7 };

struct PairLayout {
    static constexpr int kQTile = kTileM * kD * 2;          // 128 rows x 128 bf16: two 16 KB swizzle atoms
    static constexpr int kQAtom = kTileM * 128;
    static constexpr int kKHalf = (kTileN / 2) * kD * 2;    // 64 key rows x 128 bf16: two 8 KB atoms
    static constexpr int kKAtom = (kTileN / 2) * 128;
    static constexpr int kVHalf = kTileN * 64 * 2;          // 128 key rows x 64 bf16: one 16 KB atom
    static constexpr int kQ = 0;                             // 2 tiles
    static constexpr int kK = kQ + 2 * kQTile;               // kStages halves
    static constexpr int kV = kK + kStages * kKHalf;
    static constexpr int kBar = kV + kStages * kVHalf;
    static constexpr int kNumBars = 2 + 3 * kStages + 3 * 2 + 1 + 4;   // q, k/v ring, s/p/o, drain, unit ring
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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

// Leader only: arrive on the leader's own barrier when the pair MMAs this
// thread issued have completed.
__device__ __forceinline__ void tc_commit_pair_self(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(1)) : "memory");
}

// One pair work unit: (batch x head bh, 512-row query block).  Units are
// numbered head group by head group, heaviest (last) block first inside a
// group, then head.  Key tiles per query tile: up to the tile's last row when
// causal (the pair computes both CTAs' rows, so CTA 0's rows see one fully
// masked key tile at the end), all tiles otherwise; 0 for a tile past N.
struct PairUnit {
    int bh, kvh, m0, nkv0, nkv1, n_iter;
};

__device__ __forceinline__ PairUnit pair_unit(const FwdParams& p, int u) {
    PairUnit w;
    const int BH = p.B * p.Hq;
    const int grp = u / (p.heads_per_group * p.n_mblocks);
    const int h_first = grp * p.heads_per_group;
    const int nh = min(p.heads_per_group, BH - h_first);
    const int rr = u - grp * p.heads_per_group * p.n_mblocks;
    const int mb = p.n_mblocks - 1 - rr / nh;
    w.bh = h_first + rr % nh;
    const int b = w.bh / p.Hq;
    const int h = w.bh - b * p.Hq;
    w.kvh = b * p.Hkv + h / (p.Hq / p.Hkv);
    w.m0 = mb * 4 * kTileM;
    const int T = (p.N + kTileN - 1) / kTileN;
    int nkv[2];
    for (int t = 0; t < 2; ++t) {
        const int r0 = w.m0 + 2 * kTileM * t;
        if (r0 >= p.N) nkv[t] = 0;
        else nkv[t] = p.causal ? min(T, r0 / kTileN + 2) : T;
    }
    w.nkv0 = nkv[0];
    w.nkv1 = nkv[1];
    w.n_iter = max(nkv[0], nkv[1]);
    return w;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using L = PairLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;                 // leader: both CTAs' Q bytes
    uint64_t* q_empty = bars + 1;                // both: the unit's last S MMAs done
    uint64_t* k_full = bars + 2;                 // [kStages] leader
    uint64_t* v_full = k_full + kStages;         // [kStages] leader
    uint64_t* kv_empty = v_full + kStages;       // [kStages] both
    uint64_t* s_full = kv_empty + kStages;       // [2] both
    uint64_t* p_full = s_full + 2;               // [2] leader: one arrival per softmax warp of either CTA
    uint64_t* o_full = p_full + 2;               // [2] both
    uint64_t* drain = o_full + 2;                // leader
    uint64_t* unit_full = drain + 1;             // [2] both: the leader published a unit id in this CTA
    uint64_t* unit_empty = drain + 3;            // [2] leader: every consumer of both CTAs has read the slot
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);   // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 8);
            mbar_init(&o_full[s], 1);
        }
        mbar_init(drain, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&unit_full[s], 1);
            mbar_init(&unit_empty[s], kUnitConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    // barriers of both CTAs initialised before any load or arrival crosses the pair
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Unit ring: the leader's producer takes units from the launch's counter
    // (greedy, heaviest first) and publishes each id in both CTAs; every
    // consumer (the leader's MMA thread, both CTAs' softmax warps and the
    // peer's producer) reads it and releases the slot on the leader's barrier.
    const uint32_t l_unit_empty0 = mapa_shared(smem_u32(&unit_empty[0]), 0);
    auto take_unit = [&](int k, bool per_warp, bool& ok) -> int {
        const int s = k & 1;
        ok = rank == 0 ? mbar_wait(&unit_full[s], (k >> 1) & 1, abort_flag, kPSiteQ)
                       : mbar_wait_acq_cluster(&unit_full[s], (k >> 1) & 1, abort_flag, kPSiteQ);
        const int u = ok ? unit_id[s] : -1;
        if (per_warp) __syncwarp();
        if (!per_warp || lane == 0) mbar_arrive_remote(l_unit_empty0 + 8u * static_cast<uint32_t>(s));
        return u;
    };

    if (warp == 9) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const uint32_t lq_full = mapa_shared(smem_u32(q_full), 0);
            int gk = 0;               // K/V tiles of this pair so far (all units)
            int n_kv = 0, n_q = 0;    // loads issued by this CTA
            bool ok = true;
            int next = pair;          // the leader's next unit: first its pair index, then from the counter
            for (int k = 0; ok; ++k) {
                int u;
                if (rank == 0) {
                    const int s = k & 1;
                    if (k >= 2 && !(ok = mbar_wait(&unit_empty[s], ((k >> 1) - 1) & 1, abort_flag, kPSiteKVEmpty))) break;
                    u = next < p.n_units ? next : -1;
                    unit_id[s] = u;
                    st_shared_cluster(mapa_shared(smem_u32(const_cast<int*>(&unit_id[s])), 1), u);
                    mbar_arrive(&unit_full[s]);
                    mbar_arrive_remote_release(mapa_shared(smem_u32(&unit_full[s]), 1));
                } else {
                    u = take_unit(k, false, ok);
                    if (!ok) break;
                }
                if (u < 0) break;
                if (rank == 0) next = npairs + static_cast<int>(atomicAdd(p.sched, 1u));
                const PairUnit w = pair_unit(p, u);
                const int nsub = w.nkv1 > 0 ? 2 : 1;
                if (k >= 1 && !(ok = mbar_wait(q_empty, (k - 1) & 1, abort_flag, kPSiteKVEmpty))) break;
                if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * nsub * L::kQTile);
                for (int sub = 0; sub < nsub; ++sub)
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d_pair(smem + L::kQ + sub * L::kQTile + a * L::kQAtom, &tmQ, lq_full, a * 64,
                                         w.m0 + 2 * kTileM * sub + kTileM * static_cast<int>(rank), w.bh);
                n_q = k + 1;
                for (int j = 0; j < w.n_iter; ++j, ++gk) {
                    const int st = gk % kStages;
                    if (gk >= kStages &&
                        !(ok = mbar_wait(&kv_empty[st], ((gk / kStages) - 1) & 1, abort_flag, kPSiteKVEmpty)))
                        break;
                    const uint32_t lk = mapa_shared(smem_u32(&k_full[st]), 0);
                    const uint32_t lv = mapa_shared(smem_u32(&v_full[st]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&k_full[st], 2 * L::kKHalf);
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d_pair(smem + L::kK + st * L::kKHalf + a * L::kKAtom, &tmK, lk, a * 64,
                                         j * kTileN + (kTileN / 2) * static_cast<int>(rank), w.kvh);
                    if (rank == 0) mbar_arrive_expect_tx(&v_full[st], 2 * L::kVHalf);
                    tma_load_3d_pair(smem + L::kV + st * L::kVHalf, &tmV, lv, 64 * static_cast<int>(rank),
                                     j * kTileN, w.kvh);
                    n_kv = gk + 1;
                }
            }
            // The leader's barriers count both CTAs' copies: the leader waits
            // for every phase it armed, which covers the peer's copies too.
            // The peer's copies land in its own shared memory; the pair's
            // final cluster barrier keeps it resident until the leader has
            // seen them complete.
            if (rank == 0) {
                if (n_q > 0) wait_drain(q_full, (n_q - 1) & 1, kPSiteDrain);
                for (int g = (n_kv > kStages ? n_kv - kStages : 0); g < n_kv; ++g) {
                    wait_drain(&k_full[g % kStages], (g / kStages) & 1, kPSiteDrain);
                    wait_drain(&v_full[g % kStages], (g / kStages) & 1, kPSiteDrain);
                }
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(2 * kTileM, kTileN, 0, 0);
            constexpr uint32_t kIdPV = idesc_bf16_f32(2 * kTileM, kD, 0, 1);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            auto issue_s = [&](int s, int st) {
                const uint32_t qa = q_base + s * L::kQTile;
                const uint32_t ka = k_base + st * L::kKHalf;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    mma_ss_pair(tmem + s * 128, sdesc_sw128(qa + (kk >> 2) * L::kQAtom + (kk & 3) * 32, 16, 1024),
                                sdesc_sw128(ka + (kk >> 2) * L::kKAtom + (kk & 3) * 32, 16, 1024), kIdS, kk > 0);
                }
            };
            auto issue_pv = [&](int s, int st, int j) {
                const uint32_t va = v_base + st * L::kVHalf;
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    mma_ts_pair(tmem + 256 + s * 128, tmem + s * 128 + kk * 8,
                                sdesc_sw128(va + kk * 2048, L::kVHalf, 1024), kIdPV, (j > 0 || kk > 0));
            };
            bool ok = true;
            int gk = 0;                // K/V tiles consumed (all units)
            int c0 = 0, c1 = 0;        // S tiles issued for query tile 0 / 1 (all units)
            for (int k = 0; ok; ++k) {
                const int u = take_unit(k, false, ok);
                if (!ok || u < 0) break;
                const PairUnit w = pair_unit(p, u);
                const int nkv[2] = {w.nkv0, w.nkv1};
                const int n_iter = w.n_iter;
                if (!(ok = mbar_wait(q_full, k & 1, abort_flag, kPSiteQ))) break;
                if (!(ok = mbar_wait(&k_full[gk % kStages], (gk / kStages) & 1, abort_flag, kPSiteK))) break;
                tc_fence_after();
                issue_s(0, gk % kStages);
                tc_commit_pair(&s_full[0]);
                if (nkv[1] > 0) {
                    issue_s(1, gk % kStages);
                    tc_commit_pair(&s_full[1]);
                }
                if (n_iter == 1) tc_commit_pair(q_empty);   // Q no longer read by this unit
                for (int j = 0; j < n_iter; ++j) {
                    const int G = gk + j;
                    const int st = G % kStages;
                    const int st1 = (G + 1) % kStages;
                    const uint32_t ph1 = ((G + 1) / kStages) & 1;
                    if (!(ok = mbar_wait(&v_full[st], (G / kStages) & 1, abort_flag, kPSiteV))) break;
                    if (j < nkv[0]) {
                        if (!(ok = mbar_wait_cluster(&p_full[0], (c0 + j) & 1, abort_flag, kPSiteP))) break;
                        tc_fence_after();
                        issue_pv(0, st, j);
                        if (j == nkv[0] - 1) tc_commit_pair(&o_full[0]);
                        if (j + 1 < nkv[0]) {
                            if (!(ok = mbar_wait(&k_full[st1], ph1, abort_flag, kPSiteK))) break;
                            tc_fence_after();
                            issue_s(0, st1);
                            tc_commit_pair(&s_full[0]);
                        }
                    }
                    if (j < nkv[1]) {
                        if (!(ok = mbar_wait_cluster(&p_full[1], (c1 + j) & 1, abort_flag, kPSiteP))) break;
                        tc_fence_after();
                        issue_pv(1, st, j);
                        if (j == nkv[1] - 1) tc_commit_pair(&o_full[1]);
                    }
                    tc_commit_pair(&kv_empty[st]);
                    if (j + 1 < nkv[1]) {
                        if (!(ok = mbar_wait(&k_full[st1], ph1, abort_flag, kPSiteK))) break;
                        tc_fence_after();
                        issue_s(1, st1);
                        tc_commit_pair(&s_full[1]);
                    }
                    if (j == n_iter - 2) tc_commit_pair(q_empty);   // the unit's last S MMAs are issued
                }
                if (!ok) break;
                gk += n_iter;
                c0 += nkv[0];
                c1 += nkv[1];
            }
            // every pair MMA complete before either CTA releases tensor memory
            tc_commit_pair_self(drain);
            wait_drain(drain, 0, kPSiteDrain);
        }
    } else {
        // ------------------------------------------------------------ softmax (both CTAs)
        const int s = warp >> 2;                       // query tile 0 or 1
        const int r = ((warp & 3) << 5) + lane;        // row inside this CTA's part of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
        const uint32_t tS = tmem + lane_off + s * 128;
        const uint32_t tO = tmem + lane_off + 256 + s * 128;
        const float c = p.scale_log2;
        const uint32_t p_bar = mapa_shared(smem_u32(&p_full[s]), 0);
        bool ok = true;
        int cs = 0;      // S tiles of this query tile so far (all units)
        int uo = 0;      // units in which this query tile was active
        for (int k = 0; ok; ++k) {
            const int u = take_unit(k, true, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const PairUnit w = pair_unit(p, u);
            const int nkv_s = s == 0 ? w.nkv0 : w.nkv1;
            const int row0 = w.m0 + 2 * kTileM * s + kTileM * static_cast<int>(rank);   // this CTA's first row
            const int qrow = row0 + r;
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < nkv_s; ++j) {
                ok = mbar_wait(&s_full[s], (cs + j) & 1, abort_flag, kPSiteS);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
                tmem_ld_wait();
                float* sv = reinterpret_cast<float*>(&sr[0][0]);
                const int kv0 = j * kTileN;
                // masked where some key of the tile lies after the CTA's first
                // row (causal) or past N (uniform across the CTA's warps):
                // key columns >= hi get -inf (all of them when hi <= 0)
                if ((p.causal && kv0 + kTileN > row0 + 1) || (kv0 + kTileN > p.N)) {
                    const int hi = min(p.N, p.causal ? qrow + 1 : p.N) - kv0;
#pragma unroll
                    for (int cix = 0; cix < 128; ++cix) sv[cix] = (cix < hi) ? sv[cix] : -INFINITY;
                }
                float mx4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
                for (int cix = 4; cix < 124; cix += 8) {
#pragma unroll
                    for (int t = 0; t < 4; ++t) mx4[t] = fmax3(mx4[t], sv[cix + t], sv[cix + 4 + t]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) mx4[t] = fmaxf(mx4[t], sv[124 + t]);
                const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
                const float m_new = fmaxf(m_used, mx * c);
                const bool need = (m_new > m_used + kRescaleThreshold);
                const bool rescale = __any_sync(0xffffffffu, need);
                float alpha = 1.f;
                if (rescale) {
                    alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
                    l *= alpha;
                    m_used = m_new;
                }
                const float msub = (m_used == -INFINITY) ? 0.f : m_used;
                const float2 c2 = make_float2(c, c);
                const float2 nm2 = make_float2(-msub, -msub);
                float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                // four quarters of 32 columns, each packed into 16 TMEM columns as
                // soon as it is formed (few registers beyond the S row stay live)
#pragma unroll
                for (int qtr = 0; qtr < 4; ++qtr) {
                    uint32_t pk[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int cix = qtr * 32 + 2 * t;
                        const float2 x = __ffma2_rn(make_float2(sv[cix], sv[cix + 1]), c2, nm2);
                        const float p0 = ex2(x.x);
                        const float p1 = ex2(x.y);
                        ls2[t & 1] = __fadd2_rn(ls2[t & 1], make_float2(p0, p1));
                        pk[t] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + qtr * 16, pk);
                }
                l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
                if (rescale && j > 0) {
#pragma unroll 1
                    for (int q = 0; q < kD / 32; ++q) {
                        uint32_t orow[32];
                        tmem_ld32(tO + q * 32, orow);
                        tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 32; ++t) orow[t] = __float_as_uint(__uint_as_float(orow[t]) * alpha);
                        tmem_st32(tO + q * 32, orow);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(p_bar);
            }
            if (!ok) break;
            cs += nkv_s;
            if (nkv_s == 0) continue;
            ok = mbar_wait(&o_full[s], uo & 1, abort_flag, kPSiteO);
            ++uo;
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = 1.f / l;
            const bool valid = qrow < p.N;
            __nv_bfloat16* orow_g =
                reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(w.bh) * p.N + qrow) * kD;
#pragma unroll 1
            for (int q = 0; q < kD / 32; ++q) {
                uint32_t ov[32];
                tmem_ld32(tO + q * 32, ov);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    pk[t] = pack_bf16x2(__uint_as_float(ov[2 * t]) * inv_l, __uint_as_float(ov[2 * t + 1]) * inv_l);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow_g + q * 32);
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
                }
            }
            if (valid) p.lse[static_cast<size_t>(w.bh) * p.N + qrow] = (m_used + lg2(l)) * 0.69314718055994531f;
            tc_fence_before();
        }
    }

    // Neither CTA releases tensor or shared memory while the pair can still
    // touch it: the leader's MMAs read both CTAs' operands and write both
    // CTAs' accumulators, and the peer's softmax warps arrive on the leader.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
    // the last CTA to leave returns the launch's counter slot to zero
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            p.sched[0] = 0u;
            p.sched[1] = 0u;
            __threadfence();
        }
    }
}

}  // namespace

int fwd_pair_max_pairs() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cache[dev] == 0) {
        if (cudaFuncSetAttribute(fa_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PairLayout::kAlloc) != cudaSuccess)
            return -1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 148, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = PairLayout::kAlloc;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, fa_fwd_pair_kernel, &cfg) != cudaSuccess || n <= 0) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

cudaError_t launch_fwd_pair(const CUtensorMap& tq, const CUtensorMap& tk_half, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t stream) {
    if (p.n_units == 0) return cudaSuccess;
    const int max_pairs = fwd_pair_max_pairs();
    if (max_pairs <= 0) return cudaErrorInvalidConfiguration;
    const int pairs = p.n_units < max_pairs ? p.n_units : max_pairs;
    cudaError_t e = cudaFuncSetAttribute(fa_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PairLayout::kAlloc);
    if (e != cudaSuccess) return e;
    fa_fwd_pair_kernel<<<2 * pairs, kThreads, PairLayout::kAlloc, stream>>>(tq, tk_half, tv, p);
    return cudaGetLastError();
}

}  // namespace fa
