// fa_fwd.cu — tiled attention forward for sm_100a.
//
// One CTA owns a work unit of two 128-row query tiles (Q0, Q1) of one
// (batch, head) and streams the K/V tiles of that head past them, as in the
// tiling and incremental softmax of "【词汇专栏】FlashAttention：大模型训练的
// 加速器" (sections 2.1-2.3) and "FlashAttention 在昇腾NPU上到底快在哪"
// (sections 二, 三): scores are formed one (query tile, key tile) block at a
// time, multiplied with the V tile at once, and only the running row max m,
// running sum l and the O accumulator stay on chip.
//
// Warp roles (320 threads):
//   warps 0-3  softmax + correction + epilogue for Q0 (thread = query row)
//   warps 4-7  the same for Q1
//   warp  8    MMA issuer (one thread): S = Q K^T and O += P V on tcgen05
//   warp  9    TMA producer: Q once, K/V through a two-stage ring
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each.  P is
// written back over the first half of its S block as packed bf16 and read
// from there as the A operand of the P V MMA.
//
// Softmax works in log2 units: p = 2^(s*c - m) with c = scale*log2(e).  The
// O rescale by 2^(m_old - m_new) is skipped while the row max has grown by at
// most 8 (p stays <= 256, well inside fp32 / bf16 range); the final O / l and
// the LSE use the same stale m, so the result is unchanged.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kFwdThreads = 320;
constexpr int kStages = 2;
constexpr float kRescaleThreshold = 8.0f;

enum FwdSite { kSiteQ = 0, kSiteK = 1, kSiteKVEmpty = 3, kSiteS = 4, kSiteP = 5, kSiteO = 6, kSiteDrain = 7 };

template <int D>
struct FwdLayout {
    static constexpr int kTileBytes = kTileM * D * 2;  // one 128 x D bf16 tile
    static constexpr int kAtomBytes = kTileM * 128;    // 128 rows x 64 bf16
    static constexpr int kQ = 0;                        // 2 tiles
    static constexpr int kK = kQ + 2 * kTileBytes;      // kStages tiles
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kBar = kV + kStages * kTileBytes;
    static constexpr int kNumBars = 1 + 2 * kStages + 3 * 2 + 1 + 1 + 2 * 2;  // q, K/V full + empty, S/P/O, drain, q_empty, unit ring
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 B
};

// Exponential of column C of a score row: with kFmaExp, one column in eight
// is computed on the FMA pipe (exp2_fma) and the rest on the MUFU ex2,
// otherwise all on the MUFU.  The launch chooses by sequence length
// (FwdParams::fma_exp): measured 5% faster at N = 2048 and 1% at N = 4096,
// 1% slower at N = 8192.
template <int C, bool kFmaExp>
__device__ __forceinline__ float fwd_exp2(float x) {
    if constexpr (kFmaExp && (C % 8) == 0)
        return exp2_fma(x);
    else
        return ex2(x);
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Time-bounded wait that ignores the abort flag (used only to drain copies
// and MMAs that are already in flight before the CTA releases its resources).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, int site) {
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

// Merge-mode epilogue of one query row (thread = row): this call's result
// over its keys, O / l with LSE_p = ln 2 (m + log2 l), is folded into the
// running fp32 result of the row by the log-sum-exp rule,
//   LSE = log(e^LSE_old + e^LSE_p),  O = e^(LSE_old - LSE) O_old + e^(LSE_p - LSE) O / l,
// or replaces it when p.m_first is set ("【词汇专栏】FlashAttention：大模型训练的
// 加速器", section 3.2 item 2: the exact join of sequence parts).
template <int D>
__device__ __forceinline__ void merge_epilogue(const FwdParams& p, uint32_t tO, size_t row, bool valid, float m_used,
                                               float l) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.69314718055994531f;
    const float lse_p = (m_used + lg2(l)) * kLn2;
    float w_old = 0.f, w_new = 1.f, lse_n = lse_p;
    if (!p.m_first && valid) {
        const float lse_o = p.m_lse[row];
        const float mx = fmaxf(lse_o, lse_p);
        const float eo = ex2((lse_o - mx) * kLog2e);   // 0 when lse_o = -inf (no keys so far)
        const float ep = ex2((lse_p - mx) * kLog2e);
        const float inv = 1.f / (eo + ep);
        w_old = eo * inv;
        w_new = ep * inv;
        lse_n = mx + lg2(eo + ep) * kLn2;
    }
    const float wn = w_new / l;
    float* oacc = p.m_o + row * D;
    __nv_bfloat16* oout = p.m_out ? reinterpret_cast<__nv_bfloat16*>(p.m_out) + row * D : nullptr;
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
        uint32_t ov[32];
        tmem_ld32(tO + q * 32, ov);
        tmem_ld_wait();
        if (!valid) continue;
        float4* a4 = reinterpret_cast<float4*>(oacc + q * 32);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float4 a = p.m_first ? make_float4(0.f, 0.f, 0.f, 0.f) : a4[t];
            a.x = fmaf(w_old, a.x, wn * __uint_as_float(ov[4 * t]));
            a.y = fmaf(w_old, a.y, wn * __uint_as_float(ov[4 * t + 1]));
            a.z = fmaf(w_old, a.z, wn * __uint_as_float(ov[4 * t + 2]));
            a.w = fmaf(w_old, a.w, wn * __uint_as_float(ov[4 * t + 3]));
            a4[t] = a;
            pk[2 * t] = pack_bf16x2(a.x, a.y);
            pk[2 * t + 1] = pack_bf16x2(a.z, a.w);
        }
        if (oout) {
            uint4* dst = reinterpret_cast<uint4*>(oout + q * 32);
#pragma unroll
            for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
    }
    if (valid) p.m_lse[row] = lse_n;
}

// One forward work unit: (batch x head bh, pair of 128-row query tiles mb).
// Units are numbered head group by head group, heaviest (last) query block
// first inside a group, then head.
struct FwdUnit {
    int bh, kvh, m0, nkv0, nkv1, n_iter;
};

__device__ __forceinline__ FwdUnit fwd_unit(const FwdParams& p, int u) {
    FwdUnit w;
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
    w.m0 = mb * 2 * kTileM;
    const int n_kv_total = (p.N + kTileN - 1) / kTileN;
    const bool act1 = (w.m0 + kTileM) < p.N;
    if (p.causal) {
        w.nkv0 = 2 * mb + 1;
        w.nkv1 = act1 ? 2 * mb + 2 : 0;
    } else {
        w.nkv0 = n_kv_total;
        w.nkv1 = act1 ? n_kv_total : 0;
    }
    w.n_iter = act1 ? w.nkv1 : w.nkv0;
    return w;
}

// Persistent: one CTA per SM walks work units; the first unit of CTA c is c,
// later ones come from the launch's counter slot (p.sched[0]), so the
// heaviest-first order is served greedily.  The last CTA to leave puts the
// slot back to zero (p.sched[1] counts the CTAs that left).  Unit ids reach
// the MMA thread and the softmax warps through a two-slot ring; the K/V ring
// and the per-tile S / P handshakes count across units, Q (one buffer) is
// reloaded once the unit's last S MMAs have read it (q_empty), and the next
// unit's Q/K/V loads and first S MMAs overlap the current O epilogue.
template <int D, bool kFmaExp>
__global__ void __launch_bounds__(kFwdThreads, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using L = FwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;
    // [kStages] K and V of a stage land on one barrier: the MMA thread waits
    // once per key tile (a completed wait still idles the tensor core for
    // about 150 cycles, the tcgen05 issue queue being shallow)
    uint64_t* k_full = bars + 1;
    uint64_t* kv_empty = bars + 1 + kStages;     // [kStages]
    uint64_t* s_full = bars + 1 + 2 * kStages;   // [2]
    uint64_t* p_full = s_full + 2;               // [2]
    uint64_t* o_full = p_full + 2;               // [2]
    uint64_t* drain = o_full + 2;
    uint64_t* q_empty = drain + 1;
    uint64_t* unit_full = q_empty + 1;           // [2]
    uint64_t* unit_empty = unit_full + 2;        // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.n_units;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], kTileM);
            mbar_init(&o_full[s], 1);
            mbar_init(&unit_full[s], 1);
            mbar_init(&unit_empty[s], 2 * kTileM + 1);
        }
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

    auto take_unit = [&](int ui, bool& ok) -> int {
        const int s = ui & 1;
        ok = mbar_wait(&unit_full[s], (ui >> 1) & 1, abort_flag, kSiteQ);
        const int u = ok ? unit_id[s] : -1;
        mbar_arrive(&unit_empty[s]);
        return u;
    };

    if (warp == 9) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int gk = 0;               // K/V tiles of this CTA so far (all units)
            int n_kv = 0, n_q = 0;    // loads issued
            int ui = 0;
            int u = static_cast<int>(blockIdx.x);
            bool ok = true;
            while (ok) {
                const int s = ui & 1;
                if (ui >= 2 && !(ok = mbar_wait(&unit_empty[s], ((ui >> 1) - 1) & 1, abort_flag, kSiteKVEmpty))) break;
                unit_id[s] = (u < n_units) ? u : -1;
                mbar_arrive(&unit_full[s]);
                if (u >= n_units) break;
                const FwdUnit w = fwd_unit(p, u);
                const int nsub = w.nkv1 > 0 ? 2 : 1;
                if (ui >= 1 && !(ok = mbar_wait(q_empty, (ui - 1) & 1, abort_flag, kSiteKVEmpty))) break;
                mbar_arrive_expect_tx(q_full, nsub * L::kTileBytes);
                for (int sub = 0; sub < nsub; ++sub)
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kQ + sub * L::kTileBytes + a * L::kAtomBytes, &tmQ, q_full, a * 64,
                                    w.m0 + sub * kTileM, w.bh);
                n_q = ui + 1;
                for (int j = 0; j < w.n_iter; ++j, ++gk) {
                    const int st = gk & 1;
                    if (gk >= kStages &&
                        !(ok = mbar_wait(&kv_empty[st], ((gk >> 1) - 1) & 1, abort_flag, kSiteKVEmpty)))
                        break;
                    mbar_arrive_expect_tx(&k_full[st], 2 * L::kTileBytes);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kK + st * L::kTileBytes + a * L::kAtomBytes, &tmK, &k_full[st], a * 64,
                                    j * kTileN, w.kvh);
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(smem + L::kV + st * L::kTileBytes + a * L::kAtomBytes, &tmV, &k_full[st], a * 64,
                                    j * kTileN, w.kvh);
                    n_kv = gk + 1;
                }
                if (!ok) break;
                ++ui;
                u = static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(p.sched, 1u));
            }
            // Make sure no copy is still landing in shared memory when the CTA
            // leaves (only matters if the pipeline aborted).
            if (n_q > 0) mbar_wait_drain(q_full, (n_q - 1) & 1, kSiteDrain);
            for (int k = (n_kv > kStages ? n_kv - kStages : 0); k < n_kv; ++k) {
                mbar_wait_drain(&k_full[k & 1], (k >> 1) & 1, kSiteDrain);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(kTileM, kTileN, 0, 0);
            constexpr uint32_t kIdPV = idesc_bf16_f32(kTileM, D, 0, 1);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            auto issue_s = [&](int s, int st) {
                const uint32_t qa = q_base + s * L::kTileBytes;
                const uint32_t ka = k_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kAtomBytes + (kk & 3) * 32;
                    mma_ss(tmem + s * 128, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), kIdS,
                           kk > 0);
                }
            };
            auto issue_pv = [&](int s, int st, int j) {
                const uint32_t va = v_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk) {
                    mma_ts(tmem + 256 + s * 128, tmem + s * 128 + kk * 8,
                           sdesc_sw128(va + kk * 2048, L::kAtomBytes, 1024), kIdPV, (j > 0 || kk > 0));
                }
            };
            bool ok = true;
            int gk = 0;                // K/V tiles consumed (all units)
            int c0 = 0, c1 = 0;        // S tiles issued for query tile 0 / 1 (all units)
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const FwdUnit w = fwd_unit(p, u);
                const int nkv[2] = {w.nkv0, w.nkv1};
                const int n_iter = w.n_iter;
                if (!(ok = mbar_wait(q_full, ui & 1, abort_flag, kSiteQ))) break;
                if (!(ok = mbar_wait(&k_full[gk & 1], (gk >> 1) & 1, abort_flag, kSiteK))) break;
                tc_fence_after();
                issue_s(0, gk & 1);
                tc_commit(&s_full[0]);
                if (nkv[1] > 0) {
                    issue_s(1, gk & 1);
                    tc_commit(&s_full[1]);
                }
                if (n_iter == 1) tc_commit(q_empty);   // Q no longer read by this unit
                for (int j = 0; j < n_iter; ++j) {
                    const int G = gk + j;
                    const int st = G & 1;
                    // V(G) arrived with K(G), whose barrier was waited for before
                    // S(j) (at the unit start or in the previous iteration); the
                    // next tile's barrier is waited for once, before the first
                    // S(j+1)
                    bool next_kv = false;
                    if (j < nkv[0]) {
                        if (!(ok = mbar_wait(&p_full[0], (c0 + j) & 1, abort_flag, kSiteP))) break;
                        tc_fence_after();
                        issue_pv(0, st, j);
                        if (j == nkv[0] - 1) tc_commit(&o_full[0]);
                        if (j + 1 < nkv[0]) {
                            if (!(ok = mbar_wait(&k_full[st ^ 1], ((G + 1) >> 1) & 1, abort_flag, kSiteK))) break;
                            next_kv = true;
                            tc_fence_after();
                            issue_s(0, st ^ 1);
                            tc_commit(&s_full[0]);
                        }
                    }
                    if (j < nkv[1]) {
                        if (!(ok = mbar_wait(&p_full[1], (c1 + j) & 1, abort_flag, kSiteP))) break;
                        tc_fence_after();
                        issue_pv(1, st, j);
                        if (j == nkv[1] - 1) tc_commit(&o_full[1]);
                    }
                    tc_commit(&kv_empty[st]);
                    if (j + 1 < nkv[1]) {
                        if (!next_kv && !(ok = mbar_wait(&k_full[st ^ 1], ((G + 1) >> 1) & 1, abort_flag, kSiteK)))
                            break;
                        tc_fence_after();
                        issue_s(1, st ^ 1);
                        tc_commit(&s_full[1]);
                    }
                    if (j == n_iter - 2) tc_commit(q_empty);   // the unit's last S MMAs are issued
                }
                if (!ok) break;
                gk += n_iter;
                c0 += nkv[0];
                c1 += nkv[1];
            }
            // Wait for every MMA this thread issued before TMEM is released.
            tc_commit(drain);
            mbar_wait_drain(drain, 0, kSiteDrain);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int s = warp >> 2;                       // query tile 0 or 1
        const int r = ((warp & 3) << 5) + lane;        // row inside the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
        const uint32_t tS = tmem + lane_off + s * 128;
        const uint32_t tO = tmem + lane_off + 256 + s * 128;
        const float c = p.scale_log2;
        bool ok = true;
        int cs = 0;      // S tiles of this query tile so far (all units)
        int uo = 0;      // units in which this query tile was active
        for (int ui = 0; ok; ++ui) {
            const int u = take_unit(ui, ok);
            if (!__all_sync(0xffffffffu, ok) || u < 0) { ok = ok && u < 0; break; }
            const FwdUnit w = fwd_unit(p, u);
            const int nkv_s = s == 0 ? w.nkv0 : w.nkv1;
            const int qrow = w.m0 + s * kTileM + r;
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < nkv_s; ++j) {
                ok = mbar_wait(&s_full[s], (cs + j) & 1, abort_flag, kSiteS);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
                tmem_ld_wait();
                float* sv = reinterpret_cast<float*>(&sr[0][0]);
                const int kv0 = j * kTileN;
                // masked only on the causal diagonal tile and a partial last key
                // tile (warp-uniform test): key columns >= hi get -inf
                if ((p.causal && j == nkv_s - 1) || (kv0 + kTileN > p.N)) {
                    const int hi = min(p.N, p.causal ? qrow + 1 : p.N) - kv0;
#pragma unroll
                    for (int cix = 0; cix < 128; ++cix) sv[cix] = (cix < hi) ? sv[cix] : -INFINITY;
                }
                // row max: four independent chains of three-input max
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
                // warp-uniform decision; alpha = 1 for rows whose max did not move
                const bool rescale = __any_sync(0xffffffffu, need);
                float alpha = 1.f;
                if (rescale) {
                    alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
                    l *= alpha;
                    m_used = m_new;
                }
                const float msub = (m_used == -INFINITY) ? 0.f : m_used;
                // scale-and-subtract and the row sum run on column pairs
                const float2 c2 = make_float2(c, c);
                const float2 nm2 = make_float2(-msub, -msub);
                float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                // four quarters of 32 columns, each packed into 16 TMEM columns as
                // soon as it is formed (few registers beyond the S row stay live)
                static_for<0, 4>([&](auto qq) {
                    constexpr int qtr = decltype(qq)::value;
                    uint32_t pk[16];
                    static_for<0, 16>([&](auto tt) {
                        constexpr int t = decltype(tt)::value;
                        constexpr int cix = qtr * 32 + 2 * t;
                        const float2 x = __ffma2_rn(make_float2(sv[cix], sv[cix + 1]), c2, nm2);
                        const float p0 = fwd_exp2<cix, kFmaExp>(x.x);
                        const float p1 = fwd_exp2<cix + 1, kFmaExp>(x.y);
                        ls2[t & 1] = __fadd2_rn(ls2[t & 1], make_float2(p0, p1));
                        pk[t] = pack_bf16x2(p0, p1);
                    });
                    tmem_st16(tS + qtr * 16, pk);
                });
                l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
                // O <- alpha O (PV of the previous tile has completed: it was
                // committed before this tile's S); done after P so the S row is
                // no longer live in registers
                if (rescale && j > 0) {
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
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
                mbar_arrive(&p_full[s]);
            }
            if (!ok) break;
            cs += nkv_s;
            if (nkv_s == 0) continue;
            // epilogue; the next unit's first PV of this tile overwrites O only
            // after this tile's next P arrival, which follows these loads
            ok = mbar_wait(&o_full[s], uo & 1, abort_flag, kSiteO);
            ++uo;
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = 1.f / l;
            const bool valid = qrow < p.N;
            if (p.m_o != nullptr) {
                merge_epilogue<D>(p, tO, static_cast<size_t>(w.bh) * p.N + qrow, valid, m_used, l);
                tc_fence_before();
                continue;
            }
            __nv_bfloat16* orow_g =
                reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(w.bh) * p.N + qrow) * D;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
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

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, cudaStream_t stream) {
    if (p.n_units == 0) return cudaSuccess;
    // persistent (one CTA per SM) once there are at least two units per SM
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const unsigned grid = static_cast<unsigned>(p.n_units < 2 * sms ? p.n_units : sms);
    auto go = [&](auto kern, int smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kFwdThreads, smem, stream>>>(tq, tk, tv, p);
        return cudaSuccess;
    };
    cudaError_t e;
    if (D == 128)
        e = p.fma_exp ? go(fa_fwd_kernel<128, true>, FwdLayout<128>::kAlloc) : go(fa_fwd_kernel<128, false>, FwdLayout<128>::kAlloc);
    else
        e = p.fma_exp ? go(fa_fwd_kernel<64, true>, FwdLayout<64>::kAlloc) : go(fa_fwd_kernel<64, false>, FwdLayout<64>::kAlloc);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace fa
