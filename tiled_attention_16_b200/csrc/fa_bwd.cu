// fa_bwd.cu — tiled attention backward for sm_100a.
//
// Recompute-instead-of-store backward ("FlashAttention V2深度解析：反向传播显存
// 优化让大模型训练不再OOM", section 改进1): P is rebuilt tile by tile from the
// saved log-sum-exp, never read from memory.  The softmax gradient is the
// closed form dS = P o (dP - D) with D_i = rowsum(dO o O); the listing on that
// page (dP * (P - P^2)) is only the diagonal of the softmax Jacobian and is
// not used.  Work is parallel over batch, K/V head and key blocks (section
// 改进2 parallelises the sequence dimension).
//
// Three launches:
//   1. fa_bwd_preprocess: D_i = sum_d dO_id O_id and lse2_i = lse_i*log2(e)
//      (both padded to a multiple of 128 rows: D = 0, lse2 = +inf, so padded
//      query rows get P = 0), and zeroes the fp32 dQ accumulator.  HBM-bound.
//   2. fa_bwd_kernel: one CTA per (batch, K/V head, 128-row key block).  K_j
//      and V_j stay in shared memory; the CTA walks every query head of the
//      GQA group and every query tile i (i >= j when causal):
//        S^T = K_j Q_i^T,  P^T = 2^(S^T c - lse2),  dP^T = V_j dO_i^T,
//        dV += P^T dO_i,   dS^T = P^T o (dP^T - D) * scale,
//        dK += dS^T Q_i,   dQ_i += dS K_j  (fp32 vector atomics).
//      dK/dV accumulate in tensor memory over the whole group, so GQA needs
//      no atomics for them.
//   3. fa_bwd_dq_convert: dQ = bf16(dQ accumulator).  HBM-bound.
//
// Warp roles of fa_bwd_kernel (320 threads):
//   warps 0-3  P / dS (thread = key row = TMEM lane), then the dK/dV epilogue
//   warps 4-7  dQ drain (thread = query row = TMEM lane): TMEM -> atomics
//   warp  8    MMA issuer (one thread)
//   warp  9    TMA producer
// Tensor memory: S^T (P^T over its first half) | dP^T, later dQ | dV | dK.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kBwdThreads = 320;

enum BwdSite {
    kBSiteKV = 8, kBSiteQ = 9, kBSiteDO = 10, kBSiteQEmpty = 11, kBSiteDOEmpty = 12, kBSiteS = 13,
    kBSiteDP = 14, kBSiteP = 15, kBSiteDS = 16, kBSiteDSEmpty = 17, kBSiteDQ = 18, kBSiteDQFree = 19,
    kBSiteDKV = 20, kBSiteDrain = 21
};

template <int D>
struct BwdLayout {
    static constexpr int kTileBytes = kTileM * D * 2;
    static constexpr int kAtomBytes = kTileM * 128;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;
    static constexpr int kDO = kQ + kTileBytes;
    static constexpr int kDS = kDO + kTileBytes;         // 128 x 128 bf16
    static constexpr int kLse = kDS + kTileM * kTileN * 2;  // 128 fp32
    static constexpr int kDvec = kLse + kTileN * 4;        // 128 fp32
    static constexpr int kBar = kDvec + kTileN * 4;
    static constexpr int kNumBars = 16;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

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

// ---------------------------------------------------------------------------
// 1. preprocess
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
fa_bwd_preprocess(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                  const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dvec,
                  float4* __restrict__ dq_acc, size_t dq_vec4, int BH, int N, int Npad) {
    constexpr int kPer = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31;
    const size_t warp_id = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const size_t n_warps = (static_cast<size_t>(gridDim.x) * blockDim.x) >> 5;
    const size_t rows = static_cast<size_t>(BH) * Npad;
    for (size_t row = warp_id; row < rows; row += n_warps) {
        const int bh = static_cast<int>(row / Npad);
        const int n = static_cast<int>(row - static_cast<size_t>(bh) * Npad);
        float acc = 0.f;
        if (n < N) {
            const size_t base = (static_cast<size_t>(bh) * N + n) * D + lane * kPer;
            if constexpr (kPer == 4) {
                const uint2 a = *reinterpret_cast<const uint2*>(o + base);
                const uint2 g = *reinterpret_cast<const uint2*>(dout + base);
                const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
                const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const float2 af = __bfloat1622float2(a2[t]);
                    const float2 gf = __bfloat1622float2(g2[t]);
                    acc = fmaf(af.x, gf.x, acc);
                    acc = fmaf(af.y, gf.y, acc);
                }
            } else {
                const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + base);
                const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(dout + base);
                const float2 af = __bfloat1622float2(a);
                const float2 gf = __bfloat1622float2(g);
                acc = fmaf(af.x, gf.x, af.y * gf.y);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            dvec[row] = acc;
            lse2[row] = (n < N) ? lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f : INFINITY;
        }
    }
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t i = tid; i < dq_vec4; i += nthreads) dq_acc[i] = z;
}

// ---------------------------------------------------------------------------
// 3. dQ convert
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
fa_bwd_dq_convert(const float4* __restrict__ acc, uint2* __restrict__ out, size_t n_vec4) {
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = tid; i < n_vec4; i += nthreads) {
        const float4 v = acc[i];
        out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

// ---------------------------------------------------------------------------
// 2. main backward kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
              const BwdParams p) {
    using L = BwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* q_full = bars + 1;
    uint64_t* do_full = bars + 2;
    uint64_t* q_empty = bars + 3;
    uint64_t* do_empty = bars + 4;
    uint64_t* s_full = bars + 5;
    uint64_t* dp_full = bars + 6;
    uint64_t* p_full = bars + 7;
    uint64_t* ds_full = bars + 8;
    uint64_t* ds_empty = bars + 9;
    uint64_t* dq_full = bars + 10;
    uint64_t* dq_free = bars + 11;
    uint64_t* dkv_full = bars + 12;
    uint64_t* drain = bars + 13;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: key block j of (b, kv head); lightest-last for causal
    const int BHkv = p.B * p.Hkv;
    const int j = static_cast<int>(blockIdx.x) / BHkv;
    const int bkv = static_cast<int>(blockIdx.x) % BHkv;
    const int b = bkv / p.Hkv;
    const int hkv = bkv - b * p.Hkv;
    const int G = p.Hq / p.Hkv;
    const int T = (p.N + kTileM - 1) / kTileM;
    const int i0 = p.causal ? j : 0;
    const int per_head = T - i0;
    const int n_it = G * per_head;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(q_full, 1);
        mbar_init(do_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(do_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full, kTileN);
        mbar_init(ds_full, kTileN);
        mbar_init(ds_empty, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, kTileM);
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

    if (warp == 9) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
            for (int a = 0; a < D / 64; ++a) {
                tma_load_3d(smem + L::kK + a * L::kAtomBytes, &tmK, kv_full, a * 64, j * kTileN, bkv);
                tma_load_3d(smem + L::kV + a * L::kAtomBytes, &tmV, kv_full, a * 64, j * kTileN, bkv);
            }
            int issued_q = 0, issued_do = 0;
            for (int it = 0; it < n_it; ++it) {
                const int g = it / per_head;
                const int i = i0 + (it - g * per_head);
                const int bhq = b * p.Hq + hkv * G + g;
                if (it > 0 && !mbar_wait(q_empty, (it - 1) & 1, abort_flag, kBSiteQEmpty)) break;
                mbar_arrive_expect_tx(q_full, L::kTileBytes + 2 * kTileM * 4);
                for (int a = 0; a < D / 64; ++a)
                    tma_load_3d(smem + L::kQ + a * L::kAtomBytes, &tmQ, q_full, a * 64, i * kTileM, bhq);
                const size_t srow = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * kTileM;
                bulk_load(smem + L::kLse, p.lse2 + srow, kTileM * 4, q_full);
                bulk_load(smem + L::kDvec, p.dvec + srow, kTileM * 4, q_full);
                issued_q = it + 1;
                if (it > 0 && !mbar_wait(do_empty, (it - 1) & 1, abort_flag, kBSiteDOEmpty)) break;
                mbar_arrive_expect_tx(do_full, L::kTileBytes);
                for (int a = 0; a < D / 64; ++a)
                    tma_load_3d(smem + L::kDO + a * L::kAtomBytes, &tmDO, do_full, a * 64, i * kTileM, bhq);
                issued_do = it + 1;
            }
            mbar_wait_drain(kv_full, 0, kBSiteDrain);
            if (issued_q > 0) mbar_wait_drain(q_full, (issued_q - 1) & 1, kBSiteDrain);
            if (issued_do > 0) mbar_wait_drain(do_full, (issued_do - 1) & 1, kBSiteDrain);
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdSq = idesc_bf16_f32(kTileN, kTileM, 0, 0);  // S^T, dP^T: K-major both
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kTileN, D, 0, 1);      // dV, dK: A K-major, B MN-major
            constexpr uint32_t kIdDQ = idesc_bf16_f32(kTileM, D, 1, 1);       // dQ: both MN-major
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            const uint32_t ds_base = smem_u32(smem + L::kDS);
            constexpr uint32_t kAtom = L::kAtomBytes;
            constexpr uint32_t kDsAtom = kTileN * 128;  // dS^T: 64 query columns x 128 key rows
            bool ok = mbar_wait(kv_full, 0, abort_flag, kBSiteKV);
            for (int it = 0; ok && it < n_it; ++it) {
                const uint32_t ph = it & 1;
                // S^T = K Q^T
                if (!(ok = mbar_wait(q_full, ph, abort_flag, kBSiteQ))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(q_base + off, 16, 1024),
                           kIdSq, kk > 0);
                }
                tc_commit(s_full);
                // dP^T = V dO^T  (into the dQ columns: the previous dQ must be drained)
                if (!(ok = mbar_wait(do_full, ph, abort_flag, kBSiteDO))) break;
                if (it > 0 && !(ok = mbar_wait(dq_free, ph ^ 1, abort_flag, kBSiteDQFree))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(do_base + off, 16, 1024),
                           kIdSq, kk > 0);
                }
                tc_commit(dp_full);
                // dV += P^T dO   (P^T from TMEM, dO as an MN-major B operand)
                if (!(ok = mbar_wait(p_full, ph, abort_flag, kBSiteP))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)
                    mma_ts(tmem + kColDV, tmem + kColS + kk * 8, sdesc_sw128(do_base + kk * 2048, kAtom, 1024), kIdAcc,
                           (it > 0 || kk > 0));
                tc_commit(do_empty);
                // dK += dS^T Q ; dQ = dS K
                if (!(ok = mbar_wait(ds_full, ph, abort_flag, kBSiteDS))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kDsAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDK, sdesc_sw128(ds_base + off, 16, 1024),
                           sdesc_sw128(q_base + kk * 2048, kAtom, 1024), kIdAcc, (it > 0 || kk > 0));
                }
                tc_commit(q_empty);
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    mma_ss(tmem + kColDP, sdesc_sw128(ds_base + kk * 2048, kDsAtom, 1024),
                           sdesc_sw128(k_base + kk * 2048, kAtom, 1024), kIdDQ, kk > 0);
                tc_commit(dq_full);
                tc_commit(ds_empty);
            }
            if (ok) tc_commit(dkv_full);
            tc_commit(drain);
            mbar_wait_drain(drain, 0, kBSiteDrain);
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ P / dS
        const int r = (warp << 5) + lane;  // key row inside the block = TMEM lane
        const int kv = j * kTileN + r;
        const uint32_t lane_off = static_cast<uint32_t>(warp << 5) << 16;
        const float c = p.scale_log2;
        const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse);
        const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvec);
        uint8_t* ds_s = smem + L::kDS;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const uint32_t ph = it & 1;
            const int g = it / per_head;
            const int i = i0 + (it - g * per_head);
            ok = mbar_wait(q_full, ph, abort_flag, kBSiteQ) && mbar_wait(s_full, ph, abort_flag, kBSiteS);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_off + kColS + q * 32, sr[q]);
            tmem_ld_wait();
            float* pv = reinterpret_cast<float*>(&sr[0][0]);
            const bool diag = p.causal && (i == j);
            const bool kv_ok = kv < p.N;
#pragma unroll
            for (int q = 0; q < 128; ++q) {
                float e = ex2(fmaf(pv[q], c, -lse_s[q]));
                if (!kv_ok || (diag && q < r)) e = 0.f;
                pv[q] = e;
            }
            uint32_t pk[64];
#pragma unroll
            for (int t = 0; t < 64; ++t) pk[t] = pack_bf16x2(pv[2 * t], pv[2 * t + 1]);
            tmem_st32(tmem + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
            // dS^T = P^T o (dP^T - D) * scale  -> shared memory (K-major, 128B swizzle)
            ok = (it == 0 || mbar_wait(ds_empty, ph ^ 1, abort_flag, kBSiteDSEmpty)) &&
                 mbar_wait(dp_full, ph, abort_flag, kBSiteDP);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t dpr[32];
                tmem_ld32(tmem + lane_off + kColDP + q4 * 32, dpr);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int q0 = q4 * 32 + 2 * t;
                    const float d0 = pv[q0] * (__uint_as_float(dpr[2 * t]) - dvec_s[q0]) * p.scale;
                    const float d1 = pv[q0 + 1] * (__uint_as_float(dpr[2 * t + 1]) - dvec_s[q0 + 1]) * p.scale;
                    w[t] = pack_bf16x2(d0, d1);
                }
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint32_t off = sw128_offset(r, q4 * 32 + v * 8, kTileN);
                    *reinterpret_cast<uint4*>(ds_s + off) = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        // ---- epilogue: dV, dK rows of this key block (summed over the group)
        if (ok && n_it > 0) {
            ok = mbar_wait(dkv_full, 0, abort_flag, kBSiteDKV);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const bool valid = kv < p.N;
                const size_t row = static_cast<size_t>(bkv) * p.N + kv;
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
                    const uint32_t col0 = which == 0 ? kColDV : kColDK;
                    __nv_bfloat16* dst_row = reinterpret_cast<__nv_bfloat16*>(which == 0 ? p.dv : p.dk) + row * D;
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t v32[32];
                        tmem_ld32(tmem + lane_off + col0 + q * 32, v32);
                        tmem_ld_wait();
                        uint32_t pk[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            pk[t] = pack_bf16x2(__uint_as_float(v32[2 * t]), __uint_as_float(v32[2 * t + 1]));
                        if (valid) {
                            uint4* dst = reinterpret_cast<uint4*>(dst_row + q * 32);
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
                        }
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ dQ drain
        const int wq = warp - 4;
        const int r = (wq << 5) + lane;  // query row inside the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        for (int it = 0; it < n_it; ++it) {
            const int g = it / per_head;
            const int i = i0 + (it - g * per_head);
            const int bhq = b * p.Hq + hkv * G + g;
            bool ok = mbar_wait(dq_full, it & 1, abort_flag, kBSiteDQ);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int qrow = i * kTileM + r;
            float* dst = p.dq_acc + (static_cast<size_t>(bhq) * p.N + qrow) * D;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t v32[32];
                tmem_ld32(tmem + lane_off + kColDP + q * 32, v32);
                tmem_ld_wait();
                if (qrow < p.N) {
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        atomicAdd(reinterpret_cast<float4*>(dst + q * 32 + 4 * t),
                                  make_float4(__uint_as_float(v32[4 * t]), __uint_as_float(v32[4 * t + 1]),
                                              __uint_as_float(v32[4 * t + 2]), __uint_as_float(v32[4 * t + 3])));
                }
            }
            tc_fence_before();
            mbar_arrive(dq_free);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

int grid_for(size_t work, int per_block) {
    size_t g = (work + per_block - 1) / per_block;
    const size_t cap = 148 * 16;
    if (g > cap) g = cap;
    if (g == 0) g = 1;
    return static_cast<int>(g);
}

}  // namespace

BwdWorkspace bwd_workspace_layout(int B, int Hq, int N, int D) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t BH = static_cast<size_t>(B) * Hq;
    const size_t Npad = (static_cast<size_t>(N) + kTileM - 1) / kTileM * kTileM;
    BwdWorkspace w;
    w.lse2_off = 0;
    w.dvec_off = up(BH * Npad * 4);
    w.dq_off = w.dvec_off + up(BH * Npad * 4);
    w.total = w.dq_off + up(BH * static_cast<size_t>(N) * D * 4);
    return w;
}

cudaError_t launch_bwd_preprocess(int D, const void* o, const void* dout, const float* lse, float* lse2, float* dvec,
                                  float* dq_acc, int BH, int N, int Npad, cudaStream_t stream) {
    const size_t rows = static_cast<size_t>(BH) * Npad;
    const size_t dq_vec4 = static_cast<size_t>(BH) * N * D / 4;
    const int grid = grid_for(rows * 32 > dq_vec4 ? rows * 32 : dq_vec4, 256);
    if (D == 128)
        fa_bwd_preprocess<128><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                         static_cast<const __nv_bfloat16*>(dout), lse, lse2, dvec,
                                                         reinterpret_cast<float4*>(dq_acc), dq_vec4, BH, N, Npad);
    else
        fa_bwd_preprocess<64><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                        static_cast<const __nv_bfloat16*>(dout), lse, lse2, dvec,
                                                        reinterpret_cast<float4*>(dq_acc), dq_vec4, BH, N, Npad);
    return cudaGetLastError();
}

cudaError_t launch_bwd_main(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>((p.N + kTileN - 1) / kTileN) * p.B * p.Hkv;
    if (grid == 0) return cudaSuccess;
    if (D == 128) {
        auto kern = fa_bwd_kernel<128>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdLayout<128>::kAlloc);
        if (e != cudaSuccess) return e;
        kern<<<grid, kBwdThreads, BwdLayout<128>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    } else {
        auto kern = fa_bwd_kernel<64>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdLayout<64>::kAlloc);
        if (e != cudaSuccess) return e;
        kern<<<grid, kBwdThreads, BwdLayout<64>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq_convert(const float* dq_acc, void* dq, size_t n_elems, cudaStream_t stream) {
    const size_t n4 = n_elems / 4;
    fa_bwd_dq_convert<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<const float4*>(dq_acc),
                                                              static_cast<uint2*>(dq), n4);
    return cudaGetLastError();
}

}  // namespace fa
