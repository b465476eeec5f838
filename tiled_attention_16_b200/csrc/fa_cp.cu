// fa_cp.cu — the two element-wise kernels of sequence-sharded (context-
// parallel) attention ("【词汇专栏】FlashAttention：大模型训练的加速器", section
// 3.2, item 2: a long sequence split across devices).
//
// Each device computes, with fa_fwd / fa_bwd, the attention of its query
// chunks against one key chunk at a time.  Joining those results exactly
// needs the log-sum-exp merge of partial outputs (the page's "add the
// results" is not attention):
//     LSE = log(exp(LSE_acc) + exp(LSE_part)),
//     O   = exp(LSE_acc - LSE) O_acc + exp(LSE_part - LSE) O_part,
// and the gradients of a chunk are the plain sums of the per-pair terms.
// Both kernels stream their operands once (HBM-bound): one warp per row for
// the merge, 8 elements per thread for the accumulation, grid-stride loops
// over a grid sized in multiples of the SM count.
#include "fa_internal.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace fa {

namespace {

constexpr int kCpThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCpThreads)
fa_lse_merge_kernel(long long rows, const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part,
                    float* __restrict__ o_acc, float* __restrict__ lse_acc, __nv_bfloat16* __restrict__ o_out,
                    int first) {
    constexpr int kPer = D / 32;  // 4 (D = 128) or 2 (D = 64) consecutive elements per lane
    const int lane = threadIdx.x & 31;
    const long long warps = static_cast<long long>(gridDim.x) * (kCpThreads / 32);
    for (long long row = static_cast<long long>(blockIdx.x) * (kCpThreads / 32) + (threadIdx.x >> 5); row < rows;
         row += warps) {
        const float lp = lse_part[row];
        float wa, wp, lnew;
        if (first) {
            wa = 0.f;
            wp = (lp == -INFINITY) ? 0.f : 1.f;
            lnew = lp;
        } else {
            const float la = lse_acc[row];
            const float m = fmaxf(la, lp);
            if (m == -INFINITY) {
                wa = 0.f;
                wp = 0.f;
                lnew = -INFINITY;
            } else {
                const float ea = expf(la - m);
                const float ep = expf(lp - m);
                const float s = ea + ep;
                lnew = m + logf(s);
                wa = ea / s;
                wp = ep / s;
            }
        }
        const size_t base = static_cast<size_t>(row) * D + lane * kPer;
        float part[kPer];
        if constexpr (kPer == 4) {
            const uint2 raw = *reinterpret_cast<const uint2*>(o_part + base);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
            part[0] = a.x;
            part[1] = a.y;
            part[2] = b.x;
            part[3] = b.y;
        } else {
            const uint32_t raw = *reinterpret_cast<const uint32_t*>(o_part + base);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
            part[0] = a.x;
            part[1] = a.y;
        }
        float out[kPer];
        if (first) {
#pragma unroll
            for (int i = 0; i < kPer; ++i) out[i] = wp * part[i];
        } else {
            float acc[kPer];
            if constexpr (kPer == 4) {
                const float4 t = *reinterpret_cast<const float4*>(o_acc + base);
                acc[0] = t.x;
                acc[1] = t.y;
                acc[2] = t.z;
                acc[3] = t.w;
            } else {
                const float2 t = *reinterpret_cast<const float2*>(o_acc + base);
                acc[0] = t.x;
                acc[1] = t.y;
            }
#pragma unroll
            for (int i = 0; i < kPer; ++i) out[i] = fmaf(wa, acc[i], wp * part[i]);
        }
        if constexpr (kPer == 4) {
            *reinterpret_cast<float4*>(o_acc + base) = make_float4(out[0], out[1], out[2], out[3]);
            if (o_out != nullptr)
                *reinterpret_cast<uint2*>(o_out + base) = make_uint2(pack_bf16x2(out[0], out[1]),
                                                                     pack_bf16x2(out[2], out[3]));
        } else {
            *reinterpret_cast<float2*>(o_acc + base) = make_float2(out[0], out[1]);
            if (o_out != nullptr) *reinterpret_cast<uint32_t*>(o_out + base) = pack_bf16x2(out[0], out[1]);
        }
        if (lane == 0) lse_acc[row] = lnew;
    }
}

// acc = (first ? 0 : acc) + src;  out = bf16(acc) when requested.  n % 8 == 0.
__global__ void __launch_bounds__(kCpThreads)
fa_accumulate_kernel(long long n8, const __nv_bfloat16* __restrict__ src, float* __restrict__ acc,
                     __nv_bfloat16* __restrict__ out, int first) {
    const long long stride = static_cast<long long>(gridDim.x) * kCpThreads;
    for (long long i = static_cast<long long>(blockIdx.x) * kCpThreads + threadIdx.x; i < n8; i += stride) {
        float v[8];
        if (first) {
#pragma unroll
            for (int t = 0; t < 8; ++t) v[t] = 0.f;
        } else {
            const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
            const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        if (src != nullptr) {
            const uint4 raw = reinterpret_cast<const uint4*>(src)[i];
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
                v[2 * t] += f.x;
                v[2 * t + 1] += f.y;
            }
        }
        reinterpret_cast<float4*>(acc)[2 * i] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(acc)[2 * i + 1] = make_float4(v[4], v[5], v[6], v[7]);
        if (out != nullptr)
            reinterpret_cast<uint4*>(out)[i] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                          pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
}

// Blocks for `work` independent items of `per_block` each: enough to cover
// them, at most 8 resident 256-thread blocks per SM.
int cp_grid(long long work, int per_block) {
    const long long need = (work + per_block - 1) / per_block;
    const long long cap = 8LL * sm_count();
    return static_cast<int>(need < cap ? need : cap);
}

}  // namespace

cudaError_t launch_lse_merge(int D, long long rows, const void* o_part, const float* lse_part, float* o_acc,
                             float* lse_acc, void* o_out, int first, cudaStream_t stream) {
    const int grid = cp_grid(rows, kCpThreads / 32);
    const auto* op = static_cast<const __nv_bfloat16*>(o_part);
    auto* oo = static_cast<__nv_bfloat16*>(o_out);
    if (D == 128)
        fa_lse_merge_kernel<128><<<grid, kCpThreads, 0, stream>>>(rows, op, lse_part, o_acc, lse_acc, oo, first);
    else
        fa_lse_merge_kernel<64><<<grid, kCpThreads, 0, stream>>>(rows, op, lse_part, o_acc, lse_acc, oo, first);
    return cudaGetLastError();
}

cudaError_t launch_accumulate(long long n, const void* src, float* acc, void* out, int first, cudaStream_t stream) {
    const long long n8 = n / 8;
    fa_accumulate_kernel<<<cp_grid(n8, kCpThreads), kCpThreads, 0, stream>>>(
        n8, static_cast<const __nv_bfloat16*>(src), acc, static_cast<__nv_bfloat16*>(out), first);
    return cudaGetLastError();
}

}  // namespace fa
