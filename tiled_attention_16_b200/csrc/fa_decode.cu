// fa_decode.cu — attention of a few new queries over a long K/V history
// (KV-cache reuse, "FlashAttention 在昇腾NPU上到底快在哪", section 七), split
// over the key axis ("split-KV") so that every SM streams part of the cache.
//
// Mask convention: the Nq queries are the last Nq positions of the sequence;
// query i stands at position Nk - Nq + i and, when causal, sees keys
// j <= Nk - Nq + i.
//
// The work is bound by HBM: each K/V byte is read once and used for only
// (Hq / Hkv) * Nq query rows.  Kernel 1 (fa_decode_split_kernel) takes one
// (batch, K/V head, block of <= 16 query rows, key range) per CTA:
//   warp 4      TMA producer: 64-key K and V tiles through a 3-stage ring
//   warps 0-3   each owns 16 keys of every tile; S = Q K^T and O += P V by
//               warp-level m16n8k16 bf16 MMAs (fp32 accumulation), the online
//               softmax on the accumulator fragments, P kept in registers
// The four warps' (m, l, O) are merged in shared memory and the CTA writes a
// partial (O / l, LSE) per query row.  Kernel 2 (fa_decode_combine_kernel)
// merges the partials of all key ranges of a row by the log-sum-exp rule:
//   LSE = log sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kDecThreads = 160;     // 4 compute warps + 1 producer warp
constexpr int kDecKeys = 64;         // keys per tile
constexpr int kDecStages = 3;
constexpr int kDecRows = 16;         // query rows per CTA (one m16 tile)

enum DecSite { kDecSiteFull = 16, kDecSiteEmpty = 17, kDecSiteDrain = 18 };

template <int D>
struct DecLayout {
    static constexpr int kAtomBytes = kDecKeys * 128;            // 64 rows x 64 bf16
    static constexpr int kTileBytes = kDecKeys * D * 2;          // one K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;           // K then V
    static constexpr int kBar = kDecStages * kStageBytes;
    static constexpr int kBytes = kBar + 2 * kDecStages * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
    // merge area (reuses the stages once the key loop is over)
    static constexpr int kMergeO = 0;                            // [4][16][D] fp32
    static constexpr int kMergeM = 4 * kDecRows * D * 4;         // [4][16]
    static constexpr int kMergeL = kMergeM + 4 * kDecRows * 4;   // [4][16]
    static_assert(kMergeL + 4 * kDecRows * 4 <= kBar, "merge area must fit in the stages");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared address of (key row, column d) in a 64-row tile loaded by TMA with
// 128-byte swizzle: 64-column atoms of 64 rows x 128 B, 16-byte chunk index
// XOR (row % 8).
template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int row, int d) {
    return base + (d >> 6) * DecLayout<D>::kAtomBytes + row * 128 + ((((d & 63) >> 3) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void dec_drain(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return;
    unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, 1u << kDecSiteDrain);
            return;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kDecThreads)
fa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeParams p) {
    using L = DecLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* empty = full + kDecStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + 2 * kDecStages * 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int rb = blockIdx.y;
    const int bkv = blockIdx.z;                    // b * Hkv + hkv
    const int R = p.G * p.Nq;                      // query rows of this K/V head
    const int row0 = rb * kDecRows;                // first row of this CTA
    const int n_tiles = (p.Nk + kDecKeys - 1) / kDecKeys;
    const int t_begin = split * p.tiles_per_split;
    const int t_end = min(n_tiles, t_begin + p.tiles_per_split);
    const int nt = max(0, t_end - t_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int t = 0; t < nt; ++t) {
                const int st = t % kDecStages;
                if (t >= kDecStages &&
                    !mbar_wait(&empty[st], ((t / kDecStages) - 1) & 1, abort_flag, kDecSiteEmpty))
                    break;
                uint8_t* stage = smem + st * L::kStageBytes;
                mbar_arrive_expect_tx(&full[st], 2 * L::kTileBytes);
                const int key0 = (t_begin + t) * kDecKeys;
                for (int a = 0; a < D / 64; ++a) {
                    tma_load_3d(stage + a * L::kAtomBytes, &tmK, &full[st], a * 64, key0, bkv);
                    tma_load_3d(stage + L::kTileBytes + a * L::kAtomBytes, &tmV, &full[st], a * 64, key0, bkv);
                }
                issued = t + 1;
            }
            for (int t = (issued > kDecStages ? issued - kDecStages : 0); t < issued; ++t)
                dec_drain(&full[t % kDecStages], (t / kDecStages) & 1);
        }
        __syncthreads();   // pairs with the compute warps' barrier before the merge
        __syncthreads();   // and the one after it
        return;
    }

    // ---------------------------------------------------------------- compute
    const float c = p.scale_log2;
    const int g4 = lane >> 2, t4 = lane & 3;
    // this thread's two rows of the m16 tile and their absolute query positions
    int rrow[2];
    bool rvalid[2];
    int rpos[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        rrow[h] = row0 + g4 + 8 * h;
        rvalid[h] = rrow[h] < R;
        const int qi = rvalid[h] ? rrow[h] % p.Nq : 0;
        rpos[h] = p.causal ? (p.Nk - p.Nq + qi) : (p.Nk - 1);
    }
    // Q fragments (A operand) for all D/16 K steps, zero on padding rows
    uint32_t qa[D / 16][4];
    {
        const __nv_bfloat16* qbase = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                                     (static_cast<size_t>(bkv) * R) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e & 1;                      // a0a1 / a4a5: row g4; a2a3 / a6a7: row g4 + 8
                const int d = kk * 16 + (e >> 1) * 8 + 2 * t4;
                qa[kk][e] = rvalid[h] ? *reinterpret_cast<const uint32_t*>(qbase + static_cast<size_t>(rrow[h]) * D + d)
                                      : 0u;
            }
        }
    }
    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};   // partial sums of this lane's columns

    bool ok = true;
    for (int t = 0; t < nt; ++t) {
        const int st = t % kDecStages;
        ok = mbar_wait(&full[st], (t / kDecStages) & 1, abort_flag, kDecSiteFull);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        const uint32_t kb = smem_u32(smem + st * L::kStageBytes);
        const uint32_t vb = kb + L::kTileBytes;
        const int kw = warp * 16;                                 // this warp's 16 keys in the tile
        const int key0 = (t_begin + t) * kDecKeys + kw;           // absolute index of the first one
        // ---- S (16 rows x 16 keys) = Q K^T over D
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int mi = lane >> 3;                             // matrix: (keys lo/hi) x (d lo/hi)
            const int krow = kw + (mi >> 1) * 8 + (lane & 7);
            const int d = kk * 16 + (mi & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(tile_addr<D>(kb, krow, d), b0, b1, b2, b3);
            mma_16816(s[0], qa[kk], b0, b1);                      // keys kw .. kw+7
            mma_16816(s[1], qa[kk], b2, b3);                      // keys kw+8 .. kw+15
        }
        // ---- mask, online softmax on the fragments (rows g4 and g4+8)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1;
                const int key = key0 + n * 8 + 2 * t4 + (e & 1);
                const bool vis = key < p.Nk && key <= rpos[h];
                s[n][e] = vis ? s[n][e] * c : -INFINITY;
                mx[h] = fmaxf(mx[h], s[n][e]);
            }
        uint32_t pa[4];
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float m_new = fmaxf(m_run[h], mx[h]);
            alpha[h] = (m_new == -INFINITY) ? 1.f : ex2(m_run[h] - m_new);
            m_run[h] = m_new;
        }
        float ps[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1;
                ps[n][e] = (m_run[h] == -INFINITY) ? 0.f : ex2(s[n][e] - m_run[h]);
            }
#pragma unroll
        for (int h = 0; h < 2; ++h)
            l_run[h] = l_run[h] * alpha[h] + ps[0][2 * h] + ps[0][2 * h + 1] + ps[1][2 * h] + ps[1][2 * h + 1];
        // A operand of P V: (row g4, keys 2t4..), (row g4+8, ...), (row g4, keys 8+2t4..), (row g4+8, ...)
        pa[0] = pack_bf16x2(ps[0][0], ps[0][1]);
        pa[1] = pack_bf16x2(ps[0][2], ps[0][3]);
        pa[2] = pack_bf16x2(ps[1][0], ps[1][1]);
        pa[3] = pack_bf16x2(ps[1][2], ps[1][3]);
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            o[n][0] *= alpha[0];
            o[n][1] *= alpha[0];
            o[n][2] *= alpha[1];
            o[n][3] *= alpha[1];
        }
        // ---- O (16 rows x D) += P (16 x 16 keys) V (16 keys x D)
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
            const int mi = lane >> 3;                             // (keys lo/hi) x (d lo/hi)
            const int vrow = kw + (mi & 1) * 8 + (lane & 7);
            const int d = j * 16 + (mi >> 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(tile_addr<D>(vb, vrow, d), b0, b1, b2, b3);
            mma_16816(o[2 * j], pa, b0, b1);
            mma_16816(o[2 * j + 1], pa, b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- merge the four warps (each saw a different quarter of every tile)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
    }
    __syncthreads();   // every warp is past its last tile: the stages are free
    float* mo = reinterpret_cast<float*>(smem + L::kMergeO);
    float* mm = reinterpret_cast<float*>(smem + L::kMergeM);
    float* ml = reinterpret_cast<float*>(smem + L::kMergeL);
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = g4 + 8 * (e >> 1);
            mo[(warp * kDecRows + r) * D + n * 8 + 2 * t4 + (e & 1)] = o[n][e];
        }
    if (t4 == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mm[warp * kDecRows + g4 + 8 * h] = m_run[h];
            ml[warp * kDecRows + g4 + 8 * h] = l_run[h];
        }
    }
    __syncthreads();
    // 128 threads: thread -> (row r, quarter of D); partial O / l and LSE
    {
        const int r = threadIdx.x >> 3;            // 16 rows x 8 threads
        const int part = threadIdx.x & 7;
        const int row = row0 + r;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * kDecRows + r]);
        float wgt[4], Lsum = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            wgt[w] = (M == -INFINITY) ? 0.f : ex2(mm[w * kDecRows + r] - M);
            Lsum += wgt[w] * ml[w * kDecRows + r];
        }
        if (row < R && ok) {
            const size_t prow = (static_cast<size_t>(bkv) * R + row) * p.n_splits + split;
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
            for (int d = part * (D / 8); d < (part + 1) * (D / 8); ++d) {
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) acc += wgt[w] * mo[(w * kDecRows + r) * D + d];
                p.o_part[prow * D + d] = acc * inv;
            }
            if (part == 0) p.lse_part[prow] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
        }
    }
}

// One warp per query row: merge the key-range partials, write bf16 O and LSE.
template <int D>
__global__ void __launch_bounds__(256)
fa_decode_combine_kernel(const DecodeParams p, int rows_total) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows_total) return;
    const float* lp = p.lse_part + static_cast<size_t>(row) * p.n_splits;
    float M = -INFINITY;
    for (int s = lane; s < p.n_splits; s += 32) M = fmaxf(M, lp[s]);
    for (int k = 16; k; k >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, k));
    float Z = 0.f;
    for (int s = lane; s < p.n_splits; s += 32) Z += (M == -INFINITY) ? 0.f : __expf(lp[s] - M);
    for (int k = 16; k; k >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, k);
    const float lse = (Z > 0.f) ? M + __logf(Z) : -INFINITY;
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
        const float w = (lse == -INFINITY || lp[s] == -INFINITY) ? 0.f : __expf(lp[s] - lse);
        const float* op = p.o_part + (static_cast<size_t>(row) * p.n_splits + s) * D + lane * kPer;
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] += w * op[i];
    }
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.o) + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2) *reinterpret_cast<uint32_t*>(out + i) = pack_bf16x2(acc[i], acc[i + 1]);
    if (lane == 0) p.lse[row] = lse;
}

}  // namespace

cudaError_t launch_decode(int D, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          int n_row_blocks, int BHkv, cudaStream_t stream) {
    const dim3 grid(p.n_splits, n_row_blocks, BHkv);
    const int rows_total = BHkv * p.G * p.Nq;
    cudaError_t e;
    if (D == 128) {
        e = cudaFuncSetAttribute(fa_decode_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DecLayout<128>::kAlloc);
        if (e != cudaSuccess) return e;
        fa_decode_split_kernel<128><<<grid, kDecThreads, DecLayout<128>::kAlloc, stream>>>(tk, tv, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fa_decode_combine_kernel<128><<<(rows_total + 7) / 8, 256, 0, stream>>>(p, rows_total);
    } else {
        e = cudaFuncSetAttribute(fa_decode_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DecLayout<64>::kAlloc);
        if (e != cudaSuccess) return e;
        fa_decode_split_kernel<64><<<grid, kDecThreads, DecLayout<64>::kAlloc, stream>>>(tk, tv, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fa_decode_combine_kernel<64><<<(rows_total + 7) / 8, 256, 0, stream>>>(p, rows_total);
    }
    return cudaGetLastError();
}

}  // namespace fa
