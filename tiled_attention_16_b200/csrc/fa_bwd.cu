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
//   1. fa_bwd_preprocess: scale * D_i (D_i = sum_d dO_id O_id) and lse2_i = lse_i*log2(e)
//      (both padded to a multiple of 128 rows: D = 0, lse2 = +inf, so padded
//      query rows get P = 0), and zeroes the fp32 dQ accumulator.  HBM-bound.
//   2. fa_bwd_kernel: one CTA per (batch, K/V head, 128-row key block j).
//      K_j and V_j stay in shared memory; Q_i / dO_i tiles stream through a
//      two-stage ring while the CTA walks every query head of the GQA group
//      and every query tile i (i >= j when causal):
//        S^T = K_j Q_i^T,  P^T = 2^(S^T c - lse2),  dP^T = V_j dO_i^T,
//        dV += P^T dO_i,   dS^T = P^T o (dP^T - D) * scale,
//        dK += dS^T Q_i,   dQ_i += dS K_j  (fp32 reductions into global).
//      dK/dV accumulate in tensor memory over the whole group, so GQA needs
//      no atomics for them.  With D = 128 the dQ tile is computed transposed,
//      dQ^T = K_j^T dS^T, so a warp's reduction covers one 128-byte line.
//   3. fa_bwd_dq_convert: dQ = bf16(dQ accumulator).  HBM-bound.
//
// Warp roles of fa_bwd_kernel (320 threads):
//   warps 0-7  compute: thread = key row (TMEM lane); warps 0-3 take query
//              columns 0-63, warps 4-7 columns 64-127.  Per query tile they
//              form P^T, drain the previous dQ tile, then form dS^T; at the
//              end they write dK and dV.
//   warp  8    MMA issuer (one thread)
//   warp  9    TMA producer
// Tensor memory: S^T (P^T packed over the columns each compute group read) |
// dP^T, then dQ | dV | dK.
// MMA issue order per query tile it:
//   S(it) ; dK(it-1), dQ(it-1) ; dP(it) ; dV(it)
// so the tensor core works on S and dK/dQ while the compute warps form P and
// dS, and dP(it) waits only for the drain of dQ(it-1) (they share columns).
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kBwdThreads = 320;
constexpr int kCompute = 256;  // compute threads (warps 0-7)
constexpr int kMaxDynSmem = 232448;

enum BwdSite {
    kBSiteKV = 8, kBSiteQ = 9, kBSiteDO = 10, kBSiteQEmpty = 11, kBSiteDOEmpty = 12, kBSiteS = 13,
    kBSiteDP = 14, kBSiteP = 15, kBSiteDS = 16, kBSiteSmem = 17, kBSiteDQ = 18, kBSiteDQFree = 19,
    kBSiteDKV = 20, kBSiteDrain = 21
};

template <int D>
struct BwdLayout {
    static constexpr int kTileBytes = kTileM * D * 2;
    static constexpr int kAtomBytes = kTileM * 128;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;          // 2 stages
    static constexpr int kDO = kQ + 2 * kTileBytes;     // 2 stages
    static constexpr int kDS = kDO + 2 * kTileBytes;    // 128 x 128 bf16
    static constexpr int kLse = kDS + kTileM * kTileN * 2;  // 2 stages x 128 fp32
    static constexpr int kDvec = kLse + 2 * kTileN * 4;    // 2 stages x 128 fp32
    static constexpr int kBar = kDvec + 2 * kTileN * 4;
    static constexpr int kNumBars = 16;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    // Request room for base alignment when it fits; the kernel checks the
    // actual slack at run time.
    static constexpr int kAlloc = (kBytes + 1024 <= kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
    static_assert(kBytes <= kMaxDynSmem, "backward shared memory layout too large");
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

// TMEM column (relative to the S^T block) of K-step kk (16 query rows) of the
// packed bf16 P^T: query columns 0-63 are packed into columns 0-31 and query
// columns 64-127 into columns 64-95, i.e. each compute group overwrites only
// fp32 S^T columns it has already read itself.
__host__ __device__ constexpr uint32_t p_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// ---------------------------------------------------------------------------
// 1. preprocess
// ---------------------------------------------------------------------------
// Rows are handled in groups of kRowsPerIter consecutive rows per warp:
// D/8 lanes share a row, each loading 16 bytes of O and of dO, and a warp
// issues the loads of all its rows before reducing any of them, so every
// warp keeps kRowsPerIter * 2 * 2D bytes in flight.  The per-row results
// are gathered into the first lanes and written as contiguous runs.
template <int D>
__global__ void __launch_bounds__(256, 4)   // <= 64 registers: 32 warps per SM keep the loads in flight
fa_bwd_preprocess(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                  const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dvec,
                  float4* __restrict__ dq_acc, size_t dq_vec4, int BH, int N, int Npad, float scale,
                  unsigned int* __restrict__ sched) {
    // work counters of the persistent backward kernels start at zero
    if (blockIdx.x == 0 && threadIdx.x < kSchedCounters) sched[threadIdx.x] = 0u;
    constexpr int kLanesPerRow = D / 8;                 // 16-byte loads
    constexpr int kRowsPerLoad = 32 / kLanesPerRow;     // rows covered by one warp-wide load
    constexpr int kUnroll = 4;
    constexpr int kRowsPerIter = kRowsPerLoad * kUnroll; // 8 (D = 128) or 16 (D = 64); divides 128
    const int lane = threadIdx.x & 31;
    const int sub = lane / kLanesPerRow;                // row of a load this lane serves
    const int col = (lane % kLanesPerRow) * 8;          // first element of its 16 bytes
    const size_t warp_id = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const size_t n_warps = (static_cast<size_t>(gridDim.x) * blockDim.x) >> 5;
    const size_t groups = static_cast<size_t>(BH) * Npad / kRowsPerIter;
    for (size_t grp = warp_id; grp < groups; grp += n_warps) {
        const size_t row0 = grp * kRowsPerIter;         // never straddles a head: Npad % 128 == 0
        const int bh = static_cast<int>(row0 / Npad);
        const int n0 = static_cast<int>(row0 - static_cast<size_t>(bh) * Npad);
        uint4 a[kUnroll], g[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int n = n0 + u * kRowsPerLoad + sub;
            a[u] = make_uint4(0u, 0u, 0u, 0u);
            g[u] = a[u];
            if (n < N) {
                const size_t off = (static_cast<size_t>(bh) * N + n) * D + col;
                a[u] = *reinterpret_cast<const uint4*>(o + off);
                g[u] = *reinterpret_cast<const uint4*>(dout + off);
            }
        }
        float acc[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g[u]);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 af = __bfloat1622float2(a2[t]);
                const float2 gf = __bfloat1622float2(g2[t]);
                s0 = fmaf(af.x, gf.x, s0);
                s1 = fmaf(af.y, gf.y, s1);
            }
            acc[u] = s0 + s1;
#pragma unroll
            for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
        }
        // lane j < kRowsPerIter takes row n0 + j: load u = j / kRowsPerLoad, served by lanes of sub j % kRowsPerLoad
        const int j = lane % kRowsPerIter;
        const int src = (j % kRowsPerLoad) * kLanesPerRow;
        float mine = 0.f;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float v = __shfl_sync(0xffffffffu, acc[u], src);
            if (j / kRowsPerLoad == u) mine = v;
        }
        if (lane < kRowsPerIter) {
            const int n = n0 + lane;
            dvec[row0 + lane] = mine * scale;   // the backward kernels use scale * D (0 on padding rows)
            lse2[row0 + lane] = (n < N) ? lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f : INFINITY;
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
    // dQ^T (lanes = head dim) when D fills all 128 lanes, else dQ (lanes = query rows)
    constexpr bool kDQT = (D == 128);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    if (pad + L::kBytes > static_cast<uint32_t>(L::kAlloc)) {
        // Not enough slack to align the swizzled tiles: report and leave
        // before touching any barrier or tensor memory (uniform for the CTA).
        if (threadIdx.x == 0) atomicOr(&g_status, 1u << kBSiteSmem);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* q_full = bars + 1;    // [2]
    uint64_t* q_empty = bars + 3;   // [2]
    uint64_t* do_full = bars + 5;   // [2]
    uint64_t* do_empty = bars + 7;  // [2]
    uint64_t* s_full = bars + 9;
    uint64_t* dp_full = bars + 10;
    uint64_t* p_full = bars + 11;
    uint64_t* ds_full = bars + 12;
    uint64_t* dq_full = bars + 13;
    uint64_t* dq_free = bars + 14;
    uint64_t* dkv_full = bars + 15;
    uint64_t* drain = reinterpret_cast<uint64_t*>(smem + L::kMisc + 8);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: head groups; inside a group, key block j ascending
    //      (heaviest first when causal), then head
    const int BHkv = p.B * p.Hkv;
    const int T = (p.N + kTileM - 1) / kTileM;
    const int tile = static_cast<int>(blockIdx.x);
    const int grp = tile / (p.heads_per_group * T);
    const int h0 = grp * p.heads_per_group;
    const int nh = min(p.heads_per_group, BHkv - h0);
    const int rr = tile - grp * p.heads_per_group * T;
    const int j = rr / nh;
    const int bkv = h0 + (rr - j * nh);
    const int b = bkv / p.Hkv;
    const int hkv = bkv - b * p.Hkv;
    const int G = p.Hq / p.Hkv;
    const int i0 = p.causal ? j : 0;
    const int per_head = T - i0;
    const int n_it = G * per_head;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&do_full[s], 1);
            mbar_init(&do_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full, kCompute);
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
                const int st = it & 1;
                const int g = it / per_head;
                const int i = i0 + (it - g * per_head);
                const int bhq = b * p.Hq + hkv * G + g;
                if (it >= 2 && !mbar_wait(&q_empty[st], ((it >> 1) - 1) & 1, abort_flag, kBSiteQEmpty)) break;
                mbar_arrive_expect_tx(&q_full[st], L::kTileBytes + 2 * kTileM * 4);
                for (int a = 0; a < D / 64; ++a)
                    tma_load_3d(smem + L::kQ + st * L::kTileBytes + a * L::kAtomBytes, &tmQ, &q_full[st], a * 64,
                                i * kTileM, bhq);
                const size_t srow = static_cast<size_t>(bhq) * p.Npad + static_cast<size_t>(i) * kTileM;
                bulk_load(smem + L::kLse + st * kTileM * 4, p.lse2 + srow, kTileM * 4, &q_full[st]);
                bulk_load(smem + L::kDvec + st * kTileM * 4, p.dvec + srow, kTileM * 4, &q_full[st]);
                issued_q = it + 1;
                if (it >= 2 && !mbar_wait(&do_empty[st], ((it >> 1) - 1) & 1, abort_flag, kBSiteDOEmpty)) break;
                mbar_arrive_expect_tx(&do_full[st], L::kTileBytes);
                for (int a = 0; a < D / 64; ++a)
                    tma_load_3d(smem + L::kDO + st * L::kTileBytes + a * L::kAtomBytes, &tmDO, &do_full[st], a * 64,
                                i * kTileM, bhq);
                issued_do = it + 1;
            }
            mbar_wait_drain(kv_full, 0, kBSiteDrain);
            for (int it = (issued_q > 2 ? issued_q - 2 : 0); it < issued_q; ++it)
                mbar_wait_drain(&q_full[it & 1], (it >> 1) & 1, kBSiteDrain);
            for (int it = (issued_do > 2 ? issued_do - 2 : 0); it < issued_do; ++it)
                mbar_wait_drain(&do_full[it & 1], (it >> 1) & 1, kBSiteDrain);
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdSq = idesc_bf16_f32(kTileN, kTileM, 0, 0);  // S^T, dP^T: K-major both
            constexpr uint32_t kIdAcc = idesc_bf16_f32(kTileN, D, 0, 1);      // dV, dK: A K-major, B MN-major
            // dQ^T = K^T dS^T (M = D, N = query) or dQ = dS K (M = query, N = D); both operands MN-major
            constexpr uint32_t kIdDQ = kDQT ? idesc_bf16_f32(D, kTileM, 1, 1) : idesc_bf16_f32(kTileM, D, 1, 1);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t do_base = smem_u32(smem + L::kDO);
            const uint32_t ds_base = smem_u32(smem + L::kDS);
            constexpr uint32_t kAtom = L::kAtomBytes;
            constexpr uint32_t kDsAtom = kTileN * 128;  // dS^T: 64 query columns x 128 key rows
            auto issue_dk_dq = [&](int it_prev) {
                const uint32_t qa = q_base + (it_prev & 1) * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kDsAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDK, sdesc_sw128(ds_base + off, 16, 1024),
                           sdesc_sw128(qa + kk * 2048, kAtom, 1024), kIdAcc, (it_prev > 0 || kk > 0));
                }
                tc_commit(&q_empty[it_prev & 1]);
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk) {
                    const uint64_t kdesc = sdesc_sw128(k_base + kk * 2048, kAtom, 1024);
                    const uint64_t dsdesc = sdesc_sw128(ds_base + kk * 2048, kDsAtom, 1024);
                    if constexpr (kDQT)
                        mma_ss(tmem + kColDP, kdesc, dsdesc, kIdDQ, kk > 0);
                    else
                        mma_ss(tmem + kColDP, dsdesc, kdesc, kIdDQ, kk > 0);
                }
                tc_commit(dq_full);
            };
            bool ok = mbar_wait(kv_full, 0, abort_flag, kBSiteKV);
            for (int it = 0; ok && it < n_it; ++it) {
                const int st = it & 1;
                const uint32_t sph = (it >> 1) & 1;
                const uint32_t ph = it & 1;
                // S^T = K Q^T
                if (!(ok = mbar_wait(&q_full[st], sph, abort_flag, kBSiteQ))) break;
                tc_fence_after();
                const uint32_t qa = q_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qa + off, 16, 1024), kIdSq,
                           kk > 0);
                }
                tc_commit(s_full);
                // dK, dQ of the previous query tile
                if (it > 0) {
                    if (!(ok = mbar_wait(ds_full, ph ^ 1, abort_flag, kBSiteDS))) break;
                    tc_fence_after();
                    issue_dk_dq(it - 1);
                }
                // dP^T = V dO^T (its columns hold dQ until the compute warps drained it)
                if (!(ok = mbar_wait(&do_full[st], sph, abort_flag, kBSiteDO))) break;
                if (it > 0 && !(ok = mbar_wait(dq_free, ph ^ 1, abort_flag, kBSiteDQFree))) break;
                tc_fence_after();
                const uint32_t da = do_base + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_ss(tmem + kColDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(da + off, 16, 1024), kIdSq,
                           kk > 0);
                }
                tc_commit(dp_full);
                // dV += P^T dO   (P^T from TMEM, dO as an MN-major B operand)
                if (!(ok = mbar_wait(p_full, ph, abort_flag, kBSiteP))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)
                    mma_ts(tmem + kColDV, tmem + kColS + p_col(kk), sdesc_sw128(da + kk * 2048, kAtom, 1024), kIdAcc,
                           (it > 0 || kk > 0));
                tc_commit(&do_empty[st]);
            }
            if (ok && n_it > 0) {
                if (mbar_wait(ds_full, (n_it - 1) & 1, abort_flag, kBSiteDS)) {
                    tc_fence_after();
                    issue_dk_dq(n_it - 1);
                    tc_commit(dkv_full);
                }
            }
            tc_commit(drain);
            mbar_wait_drain(drain, 0, kBSiteDrain);
        }
    } else {
        // ------------------------------------------------------------ compute (P, dQ drain, dS)
        const int wg = warp >> 2;                   // query-column half
        const int wq = warp & 3;                    // TMEM lane quarter
        const int r = (wq << 5) + lane;             // key row of the block = TMEM lane
        const int kv = j * kTileN + r;
        const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
        const int c0 = wg * 64;                     // first query column of this half
        const float c = p.scale_log2;
        uint8_t* ds_s = smem + L::kDS;
        const bool kv_ok = kv < p.N;
        float pv[64];

        // dQ tile of query tile `itp` (TMEM) -> fp32 reductions into the accumulator.
        auto drain_dq = [&](int itp) -> bool {
            if (!mbar_wait(dq_full, itp & 1, abort_flag, kBSiteDQ)) return false;
            tc_fence_after();
            const int g = itp / per_head;
            const int i = i0 + (itp - g * per_head);
            const int bhq = b * p.Hq + hkv * G + g;
            if constexpr (kDQT) {
                // lanes = head-dim index d = r, columns = query rows c0 .. c0+63
                float* base = p.dq_acc + (static_cast<size_t>(bhq) * p.N + static_cast<size_t>(i) * kTileM) * D + r;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v32[32];
                    tmem_ld32(tmem + lane_off + kColDP + c0 + h * 32, v32);
                    tmem_ld_wait();
                    const int qbase = i * kTileM + c0 + h * 32;
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (qbase + t < p.N)
                            red_add_f32(base + static_cast<size_t>(c0 + h * 32 + t) * D, __uint_as_float(v32[t]));
                }
            } else {
                // lanes = query rows, columns = head dim; this half takes columns wg*32 .. +31
                const int qrow = i * kTileM + r;
                uint32_t v32[32];
                tmem_ld32(tmem + lane_off + kColDP + wg * 32, v32);
                tmem_ld_wait();
                if (qrow < p.N) {
                    float* dst = p.dq_acc + (static_cast<size_t>(bhq) * p.N + qrow) * D + wg * 32;
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        red_add_v4(dst + 4 * t, __uint_as_float(v32[4 * t]), __uint_as_float(v32[4 * t + 1]),
                                   __uint_as_float(v32[4 * t + 2]), __uint_as_float(v32[4 * t + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(dq_free);
            return true;
        };

        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int st = it & 1;
            const uint32_t ph = it & 1;
            const int g = it / per_head;
            const int i = i0 + (it - g * per_head);
            const float* lse_s = reinterpret_cast<const float*>(smem + L::kLse + st * kTileM * 4) + c0;
            const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvec + st * kTileM * 4) + c0;
            // ---- P^T = 2^(S^T c - lse2)
            ok = mbar_wait(&q_full[st], (it >> 1) & 1, abort_flag, kBSiteQ) && mbar_wait(s_full, ph, abort_flag, kBSiteS);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t sr[2][32];
                tmem_ld32(tmem + lane_off + kColS + c0, sr[0]);
                tmem_ld32(tmem + lane_off + kColS + c0 + 32, sr[1]);
                tmem_ld_wait();
                const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
                // masked only on the diagonal / partial last key block (warp-uniform test);
                // there, query columns q < lo are zero
                const bool diag = p.causal && (i == j);
                if (diag || (j + 1) * kTileN > p.N) {
                    const int lo = !kv_ok ? 64 : (diag ? r - c0 : 0);
                    static_for<0, 64>([&](auto qc) {
                        constexpr int q = decltype(qc)::value;
                        const float e = exp2_mixed<q>(fmaf(sv[q], c, -lse_s[q]));
                        pv[q] = (q >= lo) ? e : 0.f;
                    });
                } else {
                    static_for<0, 64>([&](auto qc) {
                        constexpr int q = decltype(qc)::value;
                        pv[q] = exp2_mixed<q>(fmaf(sv[q], c, -lse_s[q]));
                    });
                }
                uint32_t pk[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(pv[2 * t], pv[2 * t + 1]);
                // each group packs its P^T half into the columns it has just read
                tmem_st32(tmem + lane_off + kColS + c0, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(p_full);
            // ---- previous dQ tile out of tensor memory
            if (it > 0) {
                ok = drain_dq(it - 1);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            }
            // ---- dS^T = P^T o (dP^T - D) * scale  -> shared memory (K-major, 128B swizzle)
            ok = mbar_wait(dp_full, ph, abort_flag, kBSiteDP);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t dpr[32];
                tmem_ld32(tmem + lane_off + kColDP + c0 + h * 32, dpr);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    // dS = P (dP - D) scale = P fma(dP, scale, -scale*D); dvec holds scale*D
                    const int q0 = h * 32 + 2 * t;
                    const float d0 = pv[q0] * fmaf(__uint_as_float(dpr[2 * t]), p.scale, -dvec_s[q0]);
                    const float d1 = pv[q0 + 1] * fmaf(__uint_as_float(dpr[2 * t + 1]), p.scale, -dvec_s[q0 + 1]);
                    w[t] = pack_bf16x2(d0, d1);
                }
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint32_t off = sw128_offset(r, c0 + h * 32 + v * 8, kTileN);
                    *reinterpret_cast<uint4*>(ds_s + off) = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        if (ok && n_it > 0) {
            ok = drain_dq(n_it - 1);
            ok = __all_sync(0xffffffffu, ok);
        }
        // ---- epilogue: dV, dK rows of this key block (summed over the group)
        if (ok && n_it > 0) {
            ok = mbar_wait(dkv_full, 0, abort_flag, kBSiteDKV);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const size_t row = static_cast<size_t>(bkv) * p.N + kv;
                constexpr int kHalf = D / 2;  // columns of dK/dV written by this warp group
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
                    const uint32_t col0 = (which == 0 ? kColDV : kColDK) + wg * kHalf;
                    __nv_bfloat16* dst_row =
                        reinterpret_cast<__nv_bfloat16*>(which == 0 ? p.dv : p.dk) + row * D + wg * kHalf;
#pragma unroll 1
                    for (int q = 0; q < kHalf / 32; ++q) {
                        uint32_t v32[32];
                        tmem_ld32(tmem + lane_off + col0 + q * 32, v32);
                        tmem_ld_wait();
                        uint32_t pk[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            pk[t] = pack_bf16x2(__uint_as_float(v32[2 * t]), __uint_as_float(v32[2 * t + 1]));
                        if (kv_ok) {
                            uint4* dst = reinterpret_cast<uint4*>(dst_row + q * 32);
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
                        }
                    }
                }
            }
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

BwdWorkspace bwd_workspace_layout(int B, int Hq, int N, int D, bool with_dq_acc) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t BH = static_cast<size_t>(B) * Hq;
    const size_t Npad = (static_cast<size_t>(N) + kTileM - 1) / kTileM * kTileM;
    BwdWorkspace w;
    w.sched_off = 0;
    w.lse2_off = up(kSchedCounters * 4);
    w.dvec_off = w.lse2_off + up(BH * Npad * 4);
    w.dq_off = w.dvec_off + up(BH * Npad * 4);
    w.total = w.dq_off + (with_dq_acc ? up(BH * static_cast<size_t>(N) * D * 4) : 0);
    return w;
}

cudaError_t launch_bwd_preprocess(int D, const void* o, const void* dout, const float* lse, float* lse2, float* dvec,
                                  float* dq_acc, int BH, int N, int Npad, float scale, unsigned int* sched,
                                  cudaStream_t stream) {
    const size_t rows = static_cast<size_t>(BH) * Npad;
    const size_t dq_vec4 = dq_acc ? static_cast<size_t>(BH) * N * D / 4 : 0;
    // one warp per group of 8 (D = 128) or 16 (D = 64) rows, at most 16 blocks per SM
    const size_t warps = rows / (D == 128 ? 8 : 16);
    const int grid = grid_for(warps * 32 > dq_vec4 ? warps * 32 : dq_vec4, 256);
    if (D == 128)
        fa_bwd_preprocess<128><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                         static_cast<const __nv_bfloat16*>(dout), lse, lse2, dvec,
                                                         reinterpret_cast<float4*>(dq_acc), dq_vec4, BH, N, Npad, scale, sched);
    else
        fa_bwd_preprocess<64><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                        static_cast<const __nv_bfloat16*>(dout), lse, lse2, dvec,
                                                        reinterpret_cast<float4*>(dq_acc), dq_vec4, BH, N, Npad, scale, sched);
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
