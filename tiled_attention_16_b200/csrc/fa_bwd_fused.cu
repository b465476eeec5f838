// fa_bwd_fused.cu — tiled attention backward in one persistent KV-outer
// kernel, D = 128, dQ summed by fp32 bulk reductions.
//
// The mathematics of "FlashAttention V2深度解析：反向传播显存优化让大模型训练
// 不再OOM" (sections 改进1 and 改进2): P is recomputed from the saved
// log-sum-exp and dS = P o (dP - D) uses the closed-form softmax gradient.
// One CTA per SM walks work units (batch, K/V head, 128-row key block j) and,
// for every query head of the GQA group and every query tile i (i >= j when
// causal), executes the method's five GEMMs once:
//
//   S^T = K_j Q_i^T,  P^T = 2^(S^T c - lse2),  dP^T = V_j dO_i^T,
//   dV += P^T dO_i,   dS^T = P^T o (dP^T - D) * scale,
//   dK += dS^T Q_i,   dQ_i^T = K_j^T dS^T  (a partial sum over this key block)
//
// dK and dV accumulate in tensor memory over the unit.  Each dQ_i^T partial
// leaves tensor memory through shared memory and is added into an fp32 dQ
// accumulator in global memory by cp.reduce.async.bulk (.add.f32), applied in
// L2; fa_bwd_dq_convert turns the accumulator into bf16 afterwards.
//
// Tensor memory (512 columns): S^T [0,128) (P^T packed as bf16 over the
// columns each compute group read) | dP^T, then dQ^T [128,256) | dV | dK.
// The MMA thread issues, for query tile g of the CTA (running count):
//
//   S(g) ; dK(g-1), dQ(g-1) ; dV(g) ; dP(g)
//
// dQ(g-1) takes the dP block once the compute warps have formed dS(g-1) from
// it, and dP(g) waits until they have read dQ(g-1) out.  dV(g) sits between
// the two, so the tensor core works on it while dQ(g-1) drains.  The compute
// warps take the phases in the order P(g), read dQ(g-1) into registers and
// reduce its first 32-row block, dS(g), reduce its second row block.
//
// Shared memory (D = 128): K, V | Q x 2 stages | dO x 1 stage | dS^T (bf16,
// 128-byte swizzle) | dQ staging (fp32, 16 KB per compute group) | lse2,
// scale*D x 2 stages | barriers.  Compute group g (query columns 64g ..
// 64g+63) passes its 64 dQ rows through its 16 KB buffer as two 32-row
// blocks.  The group's threads wait until the buffer is free, store their
// rows, and arrive on a barrier; a reduction warp of its own (one per group)
// then issues the block's bulk reduction, waits until the bulk engine has
// read the buffer and frees it.  The compute warps thus never wait for each
// other or for the issue, only, before refilling, for the previous read.  L2
// applies fp32 reductions at about 6 TB/s on this part, so a tile's 64 KB of
// dQ takes roughly as long to leave as the tile's MMAs take to run; the dS
// phase between the two blocks hides the first block's read.
//
// Warp roles (384 threads): warps 0-7 compute (thread = TMEM lane = key row
// for P and dS, = head-dimension index for the dQ drain; warps 0-3 take query
// columns 0-63, warps 4-7 columns 64-127), warp 8 issues MMAs (one thread),
// warp 9 drives TMA, warps 10 and 11 issue the dQ reductions of compute
// groups 0 and 1 (one thread each).  Every wait is bounded (sm100.cuh).
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kD = 128;
constexpr int kGroups = 2;
constexpr int kCols = kTileN / kGroups;     // query columns per compute group
constexpr int kComputeWarps = 4 * kGroups;
constexpr int kMmaWarp = kComputeWarps;
constexpr int kLoadWarp = kComputeWarps + 1;
constexpr int kReduceWarp = kComputeWarps + 2;   // + compute group: issues that group's dQ reductions
constexpr int kThreads = 32 * (kComputeWarps + 2 + kGroups);
constexpr int kCompute = 32 * kComputeWarps;
constexpr int kGroupThreads = 128;
constexpr int kMaxDynSmem = 232448;
static_assert(kCols == 64, "the dS^T tile holds one 64-column swizzle atom per compute group");

// wait sites (bits of the device status word)
enum FusedSite { kFSmem = 8, kFLoad = 9, kFEmpty = 10, kFMma = 11, kFComp = 12, kFStage = 13, kFDrain = 14 };

struct FusedLayout {
    static constexpr int kTileBytes = kTileM * kD * 2;        // 32 KB bf16 tile
    static constexpr int kAtomBytes = kTileM * 128;           // 64 columns x 128 rows
    static constexpr int kStageRows = 32;                     // dQ rows per bulk reduction
    static constexpr int kStageBytes = kStageRows * kD * 4;   // 16 KB
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;                // 2 stages
    static constexpr int kDO = kQ + 2 * kTileBytes;           // 1 stage
    static constexpr int kDS = kDO + kTileBytes;              // dS^T, bf16 128 x 128
    static constexpr int kStage = kDS + kTileM * kTileN * 2;  // dQ staging, 16 KB per group
    static constexpr int kLse = kStage + kGroups * kStageBytes;   // 2 stages x 128 fp32
    static constexpr int kDvec = kLse + 2 * kTileN * 4;           // 2 stages x 128 fp32
    static constexpr int kBar = kDvec + 2 * kTileN * 4;
    static constexpr int kNumBars = 25;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kSlot = kMisc + 16;                  // [group][2] reduction target: offset, bytes
    static constexpr int kBytes = kSlot + kGroups * 2 * 16;
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "fused backward shared memory layout too large");
};

// TMEM column (relative to a 128-column block) of K-step kk (16 query
// columns) of P^T packed by the compute groups: group g packs its 64 columns
// into [64 g, 64 g + 32), columns it has itself already read.
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

// One work unit: (batch, K/V head, 128-row key block j).  Units are numbered
// head group by head group, key block ascending inside a group (heaviest
// first when causal), then head.
struct FusedUnit {
    int j, bkv, b, hkv, i0, per_head, n_it;
};

__device__ __forceinline__ FusedUnit fused_unit(const BwdParams& p, int T, int u) {
    FusedUnit w;
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

__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
    using L = FusedLayout;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kFSmem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* kv_empty = bars + 1;
    uint64_t* q_full = bars + 2;       // [2]
    uint64_t* q_empty = bars + 4;      // [2]
    uint64_t* do_full = bars + 6;
    uint64_t* do_empty = bars + 7;
    uint64_t* s_full = bars + 8;
    uint64_t* dp_full = bars + 9;
    uint64_t* p_full0 = bars + 10;     // P^T of each group's first 32 query columns
    uint64_t* p_full1 = bars + 11;     // ... and of its last 32
    uint64_t* ds_full = bars + 12;
    uint64_t* dq_full = bars + 13;
    uint64_t* dq_free = bars + 14;
    uint64_t* dkv_full = bars + 15;
    uint64_t* drain = bars + 16;
    uint64_t* unit_full = bars + 17;   // [2]
    uint64_t* unit_empty = bars + 19;  // [2]
    uint64_t* stage_full = bars + 21;  // [group]: the group's dQ rows are in its staging buffer
    uint64_t* stage_free = bars + 23;  // [group]: the buffer's previous reduction has read it
    unsigned long long* slot = reinterpret_cast<unsigned long long*>(smem + L::kSlot);
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
            mbar_init(&unit_full[s], 1);
            mbar_init(&unit_empty[s], kCompute + 1 + kGroups);
            mbar_init(&stage_full[s], kGroupThreads);
            mbar_init(&stage_free[s], 1);
        }
        mbar_init(do_full, 1);
        mbar_init(do_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full0, kCompute);
        mbar_init(p_full1, kCompute);
        mbar_init(ds_full, kCompute);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, kCompute);
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
        ok = mbar_wait(&unit_full[s], (ui >> 1) & 1, abort_flag, kFLoad);
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
            int g = 0;                          // query tiles of this CTA so far (all units)
            int n_q = 0, n_do = 0, n_kv = 0;    // loads issued
            int ui = 0;
            int u = static_cast<int>(blockIdx.x);
            bool ok = true;
            while (ok) {
                const int s = ui & 1;
                if (ui >= 2 && !(ok = mbar_wait(&unit_empty[s], ((ui >> 1) - 1) & 1, abort_flag, kFEmpty))) break;
                unit_id[s] = (u < n_units) ? u : -1;
                mbar_arrive(&unit_full[s]);
                if (u >= n_units) break;
                const FusedUnit w = fused_unit(p, T, u);
                // K/V of this unit once the previous unit's last dQ^T and dP^T have read them
                if (ui >= 1 && !(ok = mbar_wait(kv_empty, (ui - 1) & 1, abort_flag, kFEmpty))) break;
                mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
                for (int a = 0; a < kD / 64; ++a) {
                    tma_load_3d(smem + L::kK + a * L::kAtomBytes, &tmK, kv_full, a * 64, w.j * kTileN, w.bkv);
                    tma_load_3d(smem + L::kV + a * L::kAtomBytes, &tmV, kv_full, a * 64, w.j * kTileN, w.bkv);
                }
                n_kv = ui + 1;
                for (int it = 0; ok && it < w.n_it; ++it, ++g) {
                    const int st = g & 1;
                    const int gh = it / w.per_head;
                    const int i = w.i0 + (it - gh * w.per_head);
                    const int bhq = w.b * p.Hq + w.hkv * G + gh;
                    // Q(g) and its row statistics once dK(g-2) has read the slot
                    if (g >= 2 && !(ok = mbar_wait(&q_empty[st], ((g >> 1) - 1) & 1, abort_flag, kFEmpty))) break;
                    mbar_arrive_expect_tx(&q_full[st], L::kTileBytes + 2 * kTileM * 4);
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d(smem + L::kQ + st * L::kTileBytes + a * L::kAtomBytes, &tmQ, &q_full[st], a * 64,
                                    i * kTileM, bhq);
                    const size_t srow = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * kTileM;
                    bulk_load(smem + L::kLse + st * kTileM * 4, p.lse2 + srow, kTileM * 4, &q_full[st]);
                    bulk_load(smem + L::kDvec + st * kTileM * 4, p.dvec + srow, kTileM * 4, &q_full[st]);
                    n_q = g + 1;
                    // dO(g) once dP(g-1) has read the single slot
                    if (g >= 1 && !(ok = mbar_wait(do_empty, (g - 1) & 1, abort_flag, kFEmpty))) break;
                    mbar_arrive_expect_tx(do_full, L::kTileBytes);
                    for (int a = 0; a < kD / 64; ++a)
                        tma_load_3d(smem + L::kDO + a * L::kAtomBytes, &tmDO, do_full, a * 64, i * kTileM, bhq);
                    n_do = g + 1;
                }
                if (!ok) break;
                ++ui;
                u = static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(p.sched + 0, 1u));
            }
            // no copy may still be landing in shared memory when the CTA leaves
            if (n_kv > 0) wait_drain(kv_full, (n_kv - 1) & 1, kFDrain);
            for (int k = (n_q > 2 ? n_q - 2 : 0); k < n_q; ++k) wait_drain(&q_full[k & 1], (k >> 1) & 1, kFDrain);
            if (n_do > 0) wait_drain(do_full, (n_do - 1) & 1, kFDrain);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdSq = idesc_bf16_f32(kTileN, kTileM, 0, 0);  // S^T, dP^T: K-major both
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kTileN, kD, 0, 1);     // dV, dK: B MN-major
            constexpr uint32_t kIdDQ = idesc_bf16_f32(kD, kTileM, 1, 1);      // dQ^T = K^T dS^T: both MN-major
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t da = smem_u32(smem + L::kDO);
            const uint32_t ds_base = smem_u32(smem + L::kDS);
            constexpr uint32_t kAtom = L::kAtomBytes;
            constexpr uint32_t kDsAtom = kTileN * 128;   // dS^T: 64 query columns x 128 key rows
            // dK += dS^T Q and dQ^T = K^T dS^T for query tile gp; first = first tile of its unit
            auto issue_dk_dq = [&](int gp, bool first) {
                const uint32_t qa = q_base + (gp & 1) * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kDsAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDK, sdesc_sw128(ds_base + off, 16, 1024),
                           sdesc_sw128(qa + kk * 2048, kAtom, 1024), kIdAcc, (!first || kk > 0));
                }
                tc_commit(&q_empty[gp & 1]);
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    mma_ss(tmem + kColDP, sdesc_sw128(k_base + kk * 2048, kAtom, 1024),
                           sdesc_sw128(ds_base + kk * 2048, kDsAtom, 1024), kIdDQ, kk > 0);
                tc_commit(dq_full);
            };
            bool ok = true;
            int g = 0;
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const int n_it = fused_unit(p, T, u).n_it;
                if (!(ok = mbar_wait(kv_full, ui & 1, abort_flag, kFLoad))) break;
                for (int it = 0; it < n_it; ++it) {
                    const int gi = g + it;
                    const int st = gi & 1;
                    const uint32_t ph = gi & 1;
                    // S^T = K Q^T (the previous P^T was read by dV(gi-1), issued earlier)
                    if (!(ok = mbar_wait(&q_full[st], (gi >> 1) & 1, abort_flag, kFLoad))) break;
                    tc_fence_after();
                    const uint32_t qa = q_base + st * L::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                        mma_ss(tmem + kColS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qa + off, 16, 1024),
                               kIdSq, kk > 0);
                    }
                    tc_commit(s_full);
                    // dK, dQ of the previous query tile (its dS^T is in shared memory;
                    // the compute warps have read its dP^T, so dQ^T may take that block)
                    if (it > 0) {
                        if (!(ok = mbar_wait(ds_full, ph ^ 1, abort_flag, kFMma))) break;
                        tc_fence_after();
                        issue_dk_dq(gi - 1, it == 1);
                    }
                    // dV += P^T dO, in two halves of every group's query columns
                    if (!(ok = mbar_wait(do_full, ph, abort_flag, kFLoad))) break;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = mbar_wait(h == 0 ? p_full0 : p_full1, ph, abort_flag, kFMma))) break;
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
                    // dP^T = V dO^T, once the compute warps have drained dQ^T(gi-1)
                    if (gi > 0 && !(ok = mbar_wait(dq_free, ph ^ 1, abort_flag, kFMma))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                        mma_ss(tmem + kColDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(da + off, 16, 1024),
                               kIdSq, kk > 0);
                    }
                    tc_commit(dp_full);
                    tc_commit(do_empty);
                }
                if (!ok) break;
                const int gl = g + n_it - 1;   // last query tile of the unit
                if (!(ok = mbar_wait(ds_full, gl & 1, abort_flag, kFMma))) break;
                tc_fence_after();
                issue_dk_dq(gl, n_it == 1);
                tc_commit(kv_empty);   // K and V no longer read by this unit
                tc_commit(dkv_full);
                g += n_it;
            }
            tc_commit(drain);
            wait_drain(drain, 0, kFDrain);
        }
    } else if (warp >= kReduceWarp) {
        // ------------------------------------------------------------ dQ reductions of one group
        // Round r of group c: wait until the group has staged its rows, issue
        // the bulk reduction of the target the group's leader left in the slot,
        // and release the buffer once the bulk engine has read it.  Two rounds
        // per query tile (32 rows each), in the compute warps' unit order.
        if (lane == 0) {
            const int c = warp - kReduceWarp;
            float* const dq_sum = p.a_dq ? p.a_dq : p.dq_acc;
            const uint8_t* const buf = smem + L::kStage + c * L::kStageBytes;
            bool ok = true;
            int r = 0;
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const int rounds = 2 * fused_unit(p, T, u).n_it;
                for (int k = 0; k < rounds; ++k, ++r) {
                    if (!(ok = mbar_wait(&stage_full[c], r & 1, abort_flag, kFStage))) break;
                    const unsigned long long* sl = slot + (c * 2 + (r & 1)) * 2;
                    const unsigned long long off = sl[0], bytes = sl[1];
                    if (bytes > 0) bulk_reduce_add_f32(dq_sum + off, buf, static_cast<uint32_t>(bytes));
                    bulk_commit_group();
                    bulk_wait_read_all();
                    mbar_arrive(&stage_free[c]);
                }
            }
            // the bulk engine must be done with shared memory before the CTA leaves
            bulk_wait_all();
        }
    } else {
        // ------------------------------------------------------------ compute (P^T, dQ drain, dS^T)
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int r = (wq << 5) + lane;  // TMEM lane: key row (P^T, dS^T) or head-dimension index (dQ^T)
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * kCols;       // this group's query columns
        const bool leader = (wq == 0 && lane == 0);   // names each block's reduction target
        const float c = p.scale_log2;
        const float sc = p.scale;
        uint8_t* ds_s = smem + L::kDS;
        float* stage0 = reinterpret_cast<float*>(smem + L::kStage + wg * L::kStageBytes);  // 32 dQ rows x 128 fp32
        // dQ partials go to the caller's fp32 sum in accumulate mode, else to the workspace accumulator
        float* const dq_sum = p.a_dq ? p.a_dq : p.dq_acc;
        float pv[kCols];

        // dQ^T of query tile gd (running count) leaves tensor memory into
        // registers: this thread's head-dimension row d = r, query columns
        // c0 .. c0+31 (va) and c0+32 .. c0+63 (vb); the dP^T block is then free.
        uint32_t va[32], vb[32];
        auto read_dq = [&](int gd) -> bool {
            const bool w_ok = mbar_wait(dq_full, gd & 1, abort_flag, kFComp);
            tc_fence_after();
            tmem_ld32(tmem + lane_off + kColDP + c0, va);
            tmem_ld32(tmem + lane_off + kColDP + c0 + 32, vb);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(dq_free);
            return w_ok;
        };
        // One 32-row block of the group's dQ rows (query tile i of head bhq;
        // block h = rows c0 + 32h ..) -> the group's staging buffer, once the
        // group's reduction warp has seen the buffer's previous contents read
        // by the bulk engine; that warp then reduces it into the fp32 sum.
        int n_staged = 0;   // rounds of this group so far
        auto stage_dq = [&](const uint32_t (&v)[32], int h, int bhq, int i, bool ok_in) -> bool {
            bool w_ok = ok_in;
            if (n_staged > 0) w_ok = mbar_wait(&stage_free[wg], (n_staged - 1) & 1, abort_flag, kFStage) && w_ok;
#pragma unroll
            for (int t = 0; t < 32; ++t) stage0[t * kD + r] = __uint_as_float(v[t]);
            if (leader) {
                const int q0 = i * kTileM + c0 + h * L::kStageRows;
                const int rows = max(0, min(L::kStageRows, p.N - q0));
                unsigned long long* sl = slot + (wg * 2 + (n_staged & 1)) * 2;
                sl[0] = (static_cast<unsigned long long>(bhq) * p.N + q0) * kD;
                sl[1] = static_cast<unsigned long long>(rows) * kD * 4;
            }
            fence_proxy_async_smem();
            mbar_arrive(&stage_full[wg]);
            ++n_staged;
            return w_ok;
        };

        // ok: this thread's waits so far.  A failed wait (time limit, or
        // another thread's abort) returns at once from then on; the thread
        // finishes the unit on whatever the buffers hold (every address stays
        // in bounds) and leaves before the next one.
        bool ok = true;
        int g = 0;
        for (int ui = 0;; ++ui) {
            bool u_ok;
            const int u = take_unit(ui, u_ok);
            ok = __all_sync(0xffffffffu, ok && u_ok);
            if (!ok || u < 0) break;
            const FusedUnit w = fused_unit(p, T, u);
            const int j = w.j;
            const int kv = j * kTileN + r;
            const bool kv_ok = kv < p.N;
            const bool kv_block_partial = (j + 1) * kTileN > p.N;
            // query tile and head of the current and the previous iteration
            int i = w.i0, bhq = w.b * p.Hq + w.hkv * G;
            int ip = i, bhp = bhq;
            for (int it = 0; it < w.n_it; ++it) {
                const int gi = g + it;
                const int st = gi & 1;
                const uint32_t ph = gi & 1;
                const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse + st * kTileM * 4) + c0;
                const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvec + st * kTileM * 4) + c0;
                // ---- P^T = 2^(S^T c - lse2), handed to the dV MMAs in two halves
                ok = mbar_wait(&q_full[st], (gi >> 1) & 1, abort_flag, kFComp) && ok;
                ok = mbar_wait(s_full, ph, abort_flag, kFComp) && ok;
                {
                    tc_fence_after();
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
                    static_for<0, 2>([&](auto hh) {
                        constexpr int h = decltype(hh)::value;
                        static_for<0, 8>([&](auto tc) {
                            constexpr int q = 32 * h + 4 * decltype(tc)::value;
                            const float4 l4 = *reinterpret_cast<const float4*>(lse_s + q);
                            const float2 x = __ffma2_rn(make_float2(sv[q], sv[q + 1]), c2, make_float2(-l4.x, -l4.y));
                            const float2 y = __ffma2_rn(make_float2(sv[q + 2], sv[q + 3]), c2, make_float2(-l4.z, -l4.w));
                            pv[q] = ex2(x.x);
                            pv[q + 1] = ex2(x.y);
                            pv[q + 2] = ex2(y.x);
                            pv[q + 3] = ex2(y.y);
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
                // ---- the previous query tile's dQ^T leaves tensor memory; its
                //      first row block is reduced now, the second after dS
                if (it > 0) {
                    ok = read_dq(gi - 1) && ok;
                    ok = stage_dq(va, 0, bhp, ip, ok);
                }
                // ---- dS^T = P^T o (dP^T - D) * scale -> shared memory (K-major, 128-byte swizzle)
                ok = mbar_wait(dp_full, ph, abort_flag, kFComp) && ok;
                {
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) {
                        uint32_t dpr[32];
                        tmem_ld32(tmem + lane_off + kColDP + c0 + h * 32, dpr);
                        tmem_ld_wait();
                        uint32_t wv[16];
                        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                        for (int t = 0; t < 16; t += 2) {
                            // dS = P (dP - D) scale = P fma(dP, scale, -scale*D); dvec holds scale*D
                            const int q0 = h * 32 + 2 * t;
                            const float4 dv4 = *reinterpret_cast<const float4*>(dvec_s + q0);
                            const float2 gd0 = __ffma2_rn(
                                make_float2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), sc2,
                                make_float2(-dv4.x, -dv4.y));
                            const float2 gd1 = __ffma2_rn(
                                make_float2(__uint_as_float(dpr[2 * t + 2]), __uint_as_float(dpr[2 * t + 3])), sc2,
                                make_float2(-dv4.z, -dv4.w));
                            const float2 d0 = __fmul2_rn(make_float2(pv[q0], pv[q0 + 1]), gd0);
                            const float2 d1 = __fmul2_rn(make_float2(pv[q0 + 2], pv[q0 + 3]), gd1);
                            wv[t] = pack_bf16x2(d0.x, d0.y);
                            wv[t + 1] = pack_bf16x2(d1.x, d1.y);
                        }
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const uint32_t off = sw128_offset(r, c0 + h * 32 + v * 8, kTileN);
                            *reinterpret_cast<uint4*>(ds_s + off) =
                                make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(ds_full);
                }
                if (it > 0) ok = stage_dq(vb, 1, bhp, ip, ok);
                ip = i;
                bhp = bhq;
                if (++i == T) {
                    i = w.i0;
                    ++bhq;
                }
            }
            // ---- the unit's last dQ^T (query tile ip of head bhp)
            ok = read_dq(g + w.n_it - 1) && ok;
            ok = stage_dq(va, 0, bhp, ip, ok);
            ok = stage_dq(vb, 1, bhp, ip, ok);
            // ---- epilogue: dV, dK rows of this key block (summed over the group)
            ok = mbar_wait(dkv_full, ui & 1, abort_flag, kFComp) && ok;
            {
                tc_fence_after();
                const size_t row = static_cast<size_t>(w.bkv) * p.N + kv;
                constexpr int kPer = kD / kGroups;   // head-dimension columns written by this group
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
                    const uint32_t col0 = (which == 0 ? kColDV : kColDK) + wg * kPer;
                    __nv_bfloat16* dst_row =
                        reinterpret_cast<__nv_bfloat16*>(which == 0 ? p.dv : p.dk) + row * kD + wg * kPer;
                    float* acc_row = p.a_dk ? (which == 0 ? p.a_dv : p.a_dk) + row * kD + wg * kPer : nullptr;
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
            }
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

}  // namespace

cudaError_t launch_bwd_fused(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const unsigned grid = static_cast<unsigned>(p.n_units_dkdv < 2 * sms ? p.n_units_dkdv : sms);
    if (grid == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fa_bwd_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         FusedLayout::kAlloc);
    if (e != cudaSuccess) return e;
    fa_bwd_fused_kernel<<<grid, kThreads, FusedLayout::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

}  // namespace fa
