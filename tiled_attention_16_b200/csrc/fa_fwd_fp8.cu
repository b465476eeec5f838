// fa_fwd_fp8.cu — tiled attention forward with FP8 (e4m3) Q, K, V for sm_100a.
//
// The same tiling and incremental softmax as fa_fwd.cu ("【词汇专栏】
// FlashAttention：大模型训练的加速器", sections 2.1-2.3; FP8 operands are the
// FlashAttention-3 feature its section 3.3 names), with both products on the
// 8-bit tensor-core path (tcgen05.mma kind::f8f6f4, fp32 accumulation):
//
//   S = Q K^T            e4m3 x e4m3 -> fp32; the per-tensor descales of Q and
//                        K are folded into the softmax constant
//   P = 2^(S c - m)      fp32, row sum l taken from these fp32 values
//   O += P8 V            P rounded to e4m3 (RNE, saturating) and read from
//                        tensor memory as the A operand; V e4m3 from shared memory
//   O = O * v_scale / l  bf16 output, LSE in fp32 (natural log) as for bf16
//
// Layout: an e4m3 tile of 128 rows x 128 columns is exactly one 128-byte
// swizzle atom column (16 KB), so a K step of 32 elements advances 32 bytes
// (Q, K: K-major) or 32 rows = 4 KB (V: MN-major).  P is packed four keys per
// 32-bit tensor-memory column (key 4w + b in byte b of column w), over the
// first 32 columns of its own S block.
//
// Warp roles (320 threads) and the persistent unit loop as in the bf16 kernel:
// warps 0-3 / 4-7 softmax for query tiles 0 / 1, warp 8 MMA issuer, warp 9
// TMA producer (Q per unit, K/V through a three-stage ring).  Head dimension
// 128 only.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace fa {

namespace {

constexpr int kF8Threads = 320;
constexpr int kF8Stages = 3;
constexpr int kF8D = 128;
constexpr float kF8RescaleThreshold = 8.0f;

// wait sites: the bits of the bf16 forward (a timeout names the same stage)
enum F8Site { kF8Q = 0, kF8K = 1, kF8KVEmpty = 3, kF8S = 4, kF8P = 5, kF8O = 6, kF8Drain = 7 };

struct F8Layout {
    static constexpr int kTileBytes = kTileM * kF8D;  // 128 rows x 128 e4m3
    static constexpr int kQ = 0;                       // 2 tiles
    static constexpr int kK = kQ + 2 * kTileBytes;     // kF8Stages tiles
    static constexpr int kV = kK + kF8Stages * kTileBytes;
    static constexpr int kBar = kV + kF8Stages * kTileBytes;
    static constexpr int kNumBars = 1 + 2 * kF8Stages + 3 * 2 + 1 + 1 + 2 * 2 + 2;  // ... unit ring, p_half0
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

// Instruction descriptor, kind::f8f6f4 with e4m3 A and B (format code 0) and
// fp32 accumulation; a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)
         | (static_cast<uint32_t>(a_mn) << 15)
         | (static_cast<uint32_t>(b_mn) << 16)
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Share of the exponentials of a row computed on the FMA pipe (exp2_fma)
// instead of the MUFU unit: columns whose index modulo kF8PolyDen is below
// kF8PolyNum.
#ifndef FA_F8_POLY_NUM
#define FA_F8_POLY_NUM 1
#endif
#ifndef FA_F8_POLY_DEN
#define FA_F8_POLY_DEN 4
#endif
template <int Q>
__device__ __forceinline__ float f8_exp2(float x) {
    if constexpr ((Q % FA_F8_POLY_DEN) < FA_F8_POLY_NUM)
        return exp2_fma(x);
    else
        return ex2(x);
}

// Four probabilities -> one word of e4m3 bytes, the first in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float p0, float p1, float p2, float p3) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
}

__device__ __forceinline__ float lg2f(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void f8_wait_drain(uint64_t* bar, uint32_t parity, int site) {
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

// One FP8 forward work unit (as in the bf16 forward): (batch x head bh, pair of 128-row query tiles mb).
// Units are numbered head group by head group, heaviest (last) query block
// first inside a group, then head.
struct F8Unit {
    int bh, kvh, m0, nkv0, nkv1, n_iter;
};

__device__ __forceinline__ F8Unit f8_unit(const FwdParams& p, int u) {
    F8Unit w;
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
__global__ void __launch_bounds__(kF8Threads, 1)
fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using L = F8Layout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* q_full = bars + 0;
    // [kF8Stages] K and V of a stage land on one barrier (one MMA-thread wait
    // per key tile; a completed wait still idles the tensor core ~150 cycles)
    uint64_t* k_full = bars + 1;
    uint64_t* kv_empty = bars + 1 + kF8Stages;   // [kF8Stages]
    uint64_t* s_full = bars + 1 + 2 * kF8Stages; // [2]
    uint64_t* p_full = s_full + 2;               // [2]
    uint64_t* o_full = p_full + 2;               // [2]
    uint64_t* drain = o_full + 2;
    uint64_t* q_empty = drain + 1;
    uint64_t* unit_full = q_empty + 1;           // [2]
    uint64_t* unit_empty = unit_full + 2;        // [2]
    uint64_t* p_half0 = unit_empty + 2;          // [2] keys 0-63 of P in TMEM (p_full: all of P)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    volatile int* unit_id = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.n_units;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kF8Stages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], kTileM);
            mbar_init(&p_half0[s], kTileM);
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
        ok = mbar_wait(&unit_full[s], (ui >> 1) & 1, abort_flag, kF8Q);
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
                if (ui >= 2 && !(ok = mbar_wait(&unit_empty[s], ((ui >> 1) - 1) & 1, abort_flag, kF8KVEmpty))) break;
                unit_id[s] = (u < n_units) ? u : -1;
                mbar_arrive(&unit_full[s]);
                if (u >= n_units) break;
                const F8Unit w = f8_unit(p, u);
                const int nsub = w.nkv1 > 0 ? 2 : 1;
                if (ui >= 1 && !(ok = mbar_wait(q_empty, (ui - 1) & 1, abort_flag, kF8KVEmpty))) break;
                mbar_arrive_expect_tx(q_full, nsub * L::kTileBytes);
                for (int sub = 0; sub < nsub; ++sub)
                    tma_load_3d(smem + L::kQ + sub * L::kTileBytes, &tmQ, q_full, 0, w.m0 + sub * kTileM, w.bh);
                n_q = ui + 1;
                for (int j = 0; j < w.n_iter; ++j, ++gk) {
                    const int st = gk % kF8Stages;
                    if (gk >= kF8Stages &&
                        !(ok = mbar_wait(&kv_empty[st], ((gk / kF8Stages) - 1) & 1, abort_flag, kF8KVEmpty)))
                        break;
                    mbar_arrive_expect_tx(&k_full[st], 2 * L::kTileBytes);
                    tma_load_3d(smem + L::kK + st * L::kTileBytes, &tmK, &k_full[st], 0, j * kTileN, w.kvh);
                    tma_load_3d(smem + L::kV + st * L::kTileBytes, &tmV, &k_full[st], 0, j * kTileN, w.kvh);
                    n_kv = gk + 1;
                }
                if (!ok) break;
                ++ui;
                u = static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(p.sched, 1u));
            }
            // Make sure no copy is still landing in shared memory when the CTA
            // leaves (only matters if the pipeline aborted).
            if (n_q > 0) f8_wait_drain(q_full, (n_q - 1) & 1, kF8Drain);
            for (int k = (n_kv > kF8Stages ? n_kv - kF8Stages : 0); k < n_kv; ++k) {
                f8_wait_drain(&k_full[k % kF8Stages], (k / kF8Stages) & 1, kF8Drain);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_e4m3_f32(kTileM, kTileN, 0, 0);
            constexpr uint32_t kIdPV = idesc_e4m3_f32(kTileM, kF8D, 0, 1);
            const uint64_t q_desc = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);            // K-major
            const uint64_t k_desc = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);            // K-major
            const uint64_t v_desc = sdesc_sw128(smem_u32(smem + L::kV), L::kTileBytes, 1024);  // MN-major
            auto issue_s = [&](int s, int st) {
                const uint64_t qd = q_desc + ((s * L::kTileBytes) >> 4);
                const uint64_t kd = k_desc + ((st * L::kTileBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kF8D / 32; ++kk)  // 32 e4m3 = 32 bytes per K step
                    mma_f8_ss(tmem + s * 128, qd + ((kk * 32) >> 4), kd + ((kk * 32) >> 4), kIdS, kk > 0 ? 1u : 0u);
            };
            // O += P V_j for keys 64h .. 64h+63 of the tile (P as e4m3 in TMEM)
            auto issue_pv_half = [&](int s, int st, int j, int h) {
                const uint64_t vd = v_desc + ((st * L::kTileBytes) >> 4);
                const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                for (int t = 0; t < kTileN / 64; ++t) {  // 32 keys = 8 packed columns = 32 V rows
                    const int kk = h * (kTileN / 64) + t;
                    mma_f8_ts(tmem + 256 + s * 128, tmem + s * 128 + kk * 8, vd + ((kk * 32 * 128) >> 4), kIdPV,
                              kk > 0 ? 1u : acc0);
                }
            };
            // the first half's MMAs run while the softmax warps still form the second
            auto issue_pv = [&](int s, int st, int j, uint32_t parity) -> bool {
                if (!mbar_wait(&p_half0[s], parity, abort_flag, kF8P)) return false;
                tc_fence_after();
                issue_pv_half(s, st, j, 0);
                if (!mbar_wait(&p_full[s], parity, abort_flag, kF8P)) return false;
                tc_fence_after();
                issue_pv_half(s, st, j, 1);
                return true;
            };
            bool ok = true;
            int gk = 0;                // K/V tiles consumed (all units)
            int c0 = 0, c1 = 0;        // S tiles issued for query tile 0 / 1 (all units)
            for (int ui = 0; ok; ++ui) {
                const int u = take_unit(ui, ok);
                if (!ok || u < 0) break;
                const F8Unit w = f8_unit(p, u);
                const int nkv[2] = {w.nkv0, w.nkv1};
                const int n_iter = w.n_iter;
                if (!(ok = mbar_wait(q_full, ui & 1, abort_flag, kF8Q))) break;
                if (!(ok = mbar_wait(&k_full[gk % kF8Stages], (gk / kF8Stages) & 1, abort_flag, kF8K))) break;
                tc_fence_after();
                issue_s(0, gk % kF8Stages);
                tc_commit(&s_full[0]);
                if (nkv[1] > 0) {
                    issue_s(1, gk % kF8Stages);
                    tc_commit(&s_full[1]);
                }
                if (n_iter == 1) tc_commit(q_empty);   // Q no longer read by this unit
                for (int j = 0; j < n_iter; ++j) {
                    const int G = gk + j;
                    const int st = G % kF8Stages;
                    const int sn = (G + 1) % kF8Stages;
                    const uint32_t sn_ph = ((G + 1) / kF8Stages) & 1;
                    // V(G) arrived with K(G), waited for before S(j); the next
                    // tile's barrier is waited for once, before the first S(j+1)
                    bool next_kv = false;
                    if (j < nkv[0]) {
                        if (!(ok = issue_pv(0, st, j, (c0 + j) & 1))) break;
                        if (j == nkv[0] - 1) tc_commit(&o_full[0]);
                        if (j + 1 < nkv[0]) {
                            if (!(ok = mbar_wait(&k_full[sn], sn_ph, abort_flag, kF8K))) break;
                            next_kv = true;
                            tc_fence_after();
                            issue_s(0, sn);
                            tc_commit(&s_full[0]);
                        }
                    }
                    if (j < nkv[1]) {
                        if (!(ok = issue_pv(1, st, j, (c1 + j) & 1))) break;
                        if (j == nkv[1] - 1) tc_commit(&o_full[1]);
                    }
                    tc_commit(&kv_empty[st]);
                    if (j + 1 < nkv[1]) {
                        if (!next_kv && !(ok = mbar_wait(&k_full[sn], sn_ph, abort_flag, kF8K))) break;
                        tc_fence_after();
                        issue_s(1, sn);
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
            f8_wait_drain(drain, 0, kF8Drain);
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
            const F8Unit w = f8_unit(p, u);
            const int nkv_s = s == 0 ? w.nkv0 : w.nkv1;
            const int qrow = w.m0 + s * kTileM + r;
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < nkv_s; ++j) {
                ok = mbar_wait(&s_full[s], (cs + j) & 1, abort_flag, kF8S);
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
                const bool need = (m_new > m_used + kF8RescaleThreshold);
                // warp-uniform decision; alpha = 1 for rows whose max did not move
                const bool rescale = __any_sync(0xffffffffu, need);
                float alpha = 1.f;
                if (rescale) {
                    alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
                    l *= alpha;
                    m_used = m_new;
                }
                const float msub = (m_used == -INFINITY) ? 0.f : m_used;
                // P (<= 2^8 with the stale max) as e4m3, four keys per column
                const float2 c2 = make_float2(c, c);
                const float2 nm2 = make_float2(-msub, -msub);
                float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                // O must be rescaled before any PV MMA of this tile starts: a warp
                // that rescales hands over the first half of P only afterwards
                const bool late = rescale && j > 0;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[16];
                    static_for<0, 16>([&](auto tc) {
                        constexpr int t = decltype(tc)::value;
                        const int cix = half * 64 + 4 * t;
                        const float2 x0 = __ffma2_rn(make_float2(sv[cix], sv[cix + 1]), c2, nm2);
                        const float2 x1 = __ffma2_rn(make_float2(sv[cix + 2], sv[cix + 3]), c2, nm2);
                        const float p0 = f8_exp2<4 * t>(x0.x), p1 = f8_exp2<4 * t + 1>(x0.y);
                        const float p2 = f8_exp2<4 * t + 2>(x1.x), p3 = f8_exp2<4 * t + 3>(x1.y);
                        ls2[t & 1] = __fadd2_rn(ls2[t & 1], __fadd2_rn(make_float2(p0, p1), make_float2(p2, p3)));
                        pk[t] = pack_e4m3x4(p0, p1, p2, p3);
                    });
                    tmem_st16(tS + half * 16, pk);
                    if (half == 0 && !late) {   // keys 0-63 of P to the PV MMAs now
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(&p_half0[s]);
                    }
                }
                l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
                // O <- alpha O (PV of the previous tile has completed: it was
                // committed before this tile's S); done after P so the S row is
                // no longer live in registers
                if (late) {
#pragma unroll 1
                    for (int q = 0; q < kF8D / 32; ++q) {
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
                if (late) mbar_arrive(&p_half0[s]);
                mbar_arrive(&p_full[s]);
            }
            if (!ok) break;
            cs += nkv_s;
            if (nkv_s == 0) continue;
            // epilogue; the next unit's first PV of this tile overwrites O only
            // after this tile's next P arrival, which follows these loads
            ok = mbar_wait(&o_full[s], uo & 1, abort_flag, kF8O);
            ++uo;
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = p.o_scale / l;
            const bool valid = qrow < p.N;
            __nv_bfloat16* orow_g =
                reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(w.bh) * p.N + qrow) * kF8D;
#pragma unroll 1
            for (int q = 0; q < kF8D / 32; ++q) {
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
            if (valid) p.lse[static_cast<size_t>(w.bh) * p.N + qrow] = (m_used + lg2f(l)) * 0.69314718055994531f;
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

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                           cudaStream_t stream) {
    if (p.n_units == 0) return cudaSuccess;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const unsigned grid = static_cast<unsigned>(p.n_units < 2 * sms ? p.n_units : sms);
    cudaError_t e = cudaFuncSetAttribute(fa_fwd_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, F8Layout::kAlloc);
    if (e != cudaSuccess) return e;
    fa_fwd_fp8_kernel<<<grid, kF8Threads, F8Layout::kAlloc, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace fa
