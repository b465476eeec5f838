// fa_api.cu — the C ABI of include/fa.h: argument validation, TMA tensor-map
// construction and kernel launches on the caller's stream.  No device memory
// is allocated here; every buffer belongs to the caller.
#include "fa.h"
#include "fa_internal.h"

#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include <cudaTypedefs.h>

namespace fa {

__device__ unsigned int g_status = 0;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over a contiguous [BH, N, D] tensor: box = 128 bytes of a row
// (64 bf16 or 128 e4m3) x 128 rows x 1 head, 128-byte swizzle; rows past N
// read as zero.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int D, int elem_bytes = 2, int box_rows = kTileM) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * eb, static_cast<cuuint64_t>(N) * D * eb};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// fp32 vectors read or written one element at a time
bool aligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

fa_status check_shape(const fa_shape* s) {
    if (!s) return FA_ERR_INVALID_ARG;
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 1 || s->D < 1) return FA_ERR_INVALID_ARG;
    if (s->Hq % s->Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(s->scale) || !(s->scale > 0.f)) return FA_ERR_INVALID_ARG;
    // grid and index ranges
    const long long BH = static_cast<long long>(s->B) * s->Hq;
    const long long tiles = (static_cast<long long>(s->N) + 255) / 256;
    if (BH * tiles > 0x7fffffffLL || BH > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
    if (s->D != 64 && s->D != 128) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

// sm_100 check, cached per device.
fa_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    static int cached[64];
    static std::once_flag once;
    std::call_once(once, [] { std::memset(cached, 0, sizeof(cached)); });
    if (dev < 0 || dev >= 64) return FA_ERR_CUDA;
    if (cached[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return cached[dev] == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

unsigned int g_last_sites = 0;

}  // namespace

int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

namespace {

// Split-KV plan of fa_decode: 64-key tiles, query rows in blocks of 16 per
// K/V head, and the number of key ranges that fills the resident CTA slots
// (2 per SM at D = 128, 4 at D = 64: shared memory and registers) most
// evenly over about two waves, so that no nearly empty last wave streams alone.
struct DecodePlan {
    int n_row_blocks, n_splits, tiles_per_split;
    size_t o_part_off, lse_part_off, total;
};

fa_status check_kv_shape(const fa_kv_shape* s) {
    if (!s) return FA_ERR_INVALID_ARG;
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->Nq < 1 || s->Nk < 1 || s->Nq > s->Nk) return FA_ERR_INVALID_ARG;
    if (s->Hq % s->Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(s->scale) || !(s->scale > 0.f)) return FA_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(s->B) * s->Hq * s->Nq;
    const long long BHkv = static_cast<long long>(s->B) * s->Hkv;
    const long long row_blocks = (static_cast<long long>(s->Hq / s->Hkv) * s->Nq + 15) / 16;
    if (rows > 0x7fffffffLL || BHkv > 65535 || row_blocks > 65535) return FA_ERR_INVALID_ARG;
    if (s->D != 64 && s->D != 128) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

DecodePlan decode_plan(const fa_kv_shape& s) {
    DecodePlan pl;
    const int R = (s.Hq / s.Hkv) * s.Nq;
    pl.n_row_blocks = (R + 15) / 16;
    const int n_tiles = (s.Nk + 63) / 64;
    const long long pairs = static_cast<long long>(s.B) * s.Hkv * pl.n_row_blocks;
    const long long slots = 148LL * (s.D == 128 ? 2 : 4);
    const long long s0 = (2 * slots + pairs - 1) / pairs;   // about two waves
    long long splits = 1;
    double best = -1.0;
    for (long long c = (s0 + 1) / 2; c <= 2 * s0; ++c) {
        const long long cs = c > n_tiles ? n_tiles : c;
        // the ranges actually formed from cs: whole tiles per range
        const long long per = (n_tiles + cs - 1) / cs;
        const long long n = (n_tiles + per - 1) / per;
        const double waves = static_cast<double>(pairs * n) / static_cast<double>(slots);
        const double fill = waves / std::ceil(waves);
        if (fill > best + 1e-9) {
            best = fill;
            splits = n;
        }
    }
    if (splits > 65535) splits = 65535;
    if (splits < 1) splits = 1;
    pl.tiles_per_split = static_cast<int>((n_tiles + splits - 1) / splits);
    pl.n_splits = (n_tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t rows = static_cast<size_t>(s.B) * s.Hq * s.Nq;
    pl.o_part_off = 0;
    pl.lse_part_off = up(rows * pl.n_splits * s.D * 4);
    pl.total = pl.lse_part_off + up(rows * pl.n_splits * 4);
    return pl;
}

constexpr int kNumSMs = 148;

// Query tile of the bf16 forward (D = 128): "m128", 128-row MMAs on one CTA
// (unit of 256 rows), or "m256", 256-row MMAs on a CTA pair (unit of 512
// rows).  By default the pair is used from kPairMinN query rows on; the
// environment variable FA_FWD_TILE=m128|m256 fixes one (read once).
constexpr int kPairMinN = 1 << 30;
// The one-CTA bf16 forward computes 1/8 of its exponentials on the FMA pipe up
// to this sequence length: measured 5% faster at N = 2048 and 1% at 4096, 1%
// slower at 8192.
constexpr int kFmaExpMaxN = 4096;
int fwd_tile_override() {
    static int mode = -1;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* e = std::getenv("FA_FWD_TILE");
        mode = !e ? 0 : (std::strcmp(e, "m256") == 0 ? 2 : (std::strcmp(e, "m128") == 0 ? 1 : 0));
    });
    return mode;
}
// Block of the default backward's two passes (D = 128): "m128", 128 keys
// (dK/dV pass) or 128 query rows (dQ pass) per CTA, or "m256", 256 per CTA
// pair.  FA_BWD_TILE=m128|m256 fixes both (read once).  By measurement both
// passes run on one CTA by default (the pairs were equal or slower on every
// workload measured); kBwdPairMinN is where the dQ pass would switch.
constexpr int kBwdPairMinN = 1 << 30;
int bwd_tile_override() {
    static int mode = -1;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* e = std::getenv("FA_BWD_TILE");
        mode = !e ? 0 : (std::strcmp(e, "m256") == 0 ? 2 : (std::strcmp(e, "m128") == 0 ? 1 : 0));
    });
    return mode;
}
bool bwd_dkdv_use_pair(const fa_shape& s) {
    if (s.D != 128) return false;
    return bwd_tile_override() == 2;
}
bool bwd_dq_use_pair(const fa_shape& s) {
    if (s.D != 128) return false;
    const int m = bwd_tile_override();
    if (m != 0) return m == 2;
    return s.N >= kBwdPairMinN;
}

bool fwd_use_pair(const fa_shape& s) {
    if (s.D != 128) return false;
    const int m = fwd_tile_override();
    if (m != 0) return m == 2;
    return s.N >= kPairMinN;
}

// dQ strategy of the backward (FA_BWD_AUTO / _DETERMINISTIC / _FUSED): the
// process-wide choice of fa_set_bwd_mode, unless the environment variable
// FA_DQ_MODE=separate|fused (or its older name atomic; read once) fixes it.
// AUTO is the measured choice: the fused kernel for D = 128, the separate
// passes for D = 64.
std::atomic<int> g_bwd_mode{FA_BWD_AUTO};
int env_bwd_mode() {
    static int mode = FA_BWD_AUTO;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* e = std::getenv("FA_DQ_MODE");
        if (e && (std::strcmp(e, "atomic") == 0 || std::strcmp(e, "fused") == 0)) mode = FA_BWD_FUSED;
        else if (e && std::strcmp(e, "separate") == 0) mode = FA_BWD_DETERMINISTIC;
    });
    return mode;
}
bool bwd_fused(const fa_shape& s) {
    int m = env_bwd_mode();
    if (m == FA_BWD_AUTO) m = g_bwd_mode.load(std::memory_order_relaxed);
    if (m == FA_BWD_AUTO) return s.D == 128;
    return m == FA_BWD_FUSED;
}

// Scratch of fa_bwd_noalloc: reserved statically in device memory on every
// GPU that loads the library, so that entry point never allocates.  In host
// code this name only stands in for the symbol; the device address comes from
// cudaGetSymbolAddress (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// Work-counter slots of the persistent forward.  A launch outside stream
// capture takes the next slot of the first kFwdEagerSlots (round robin), so
// launches that may overlap on different streams use different counters.  A
// launch recorded into a CUDA graph takes a slot of its own from the rest
// (round robin there too), so no later eager launch can share the counter a
// graph replays with.  The last CTA of a launch puts its slot back to zero.
constexpr int kFwdSchedSlots = 4096;
constexpr int kFwdEagerSlots = 1024;
static __device__ unsigned int g_fwd_sched[kFwdSchedSlots][2];

fa_status fwd_sched_slot(cudaStream_t stream, unsigned int** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return FA_ERR_CUDA;
    static std::mutex mu;
    static unsigned int* base[64] = {};
    static unsigned int next_eager[64] = {};
    static unsigned int next_captured[64] = {};
    std::lock_guard<std::mutex> g(mu);
    if (base[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_fwd_sched) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
        base[dev] = static_cast<unsigned int*>(ptr);
    }
    const unsigned int slot = (cap == cudaStreamCaptureStatusNone)
                                  ? next_eager[dev]++ % kFwdEagerSlots
                                  : kFwdEagerSlots + next_captured[dev]++ % (kFwdSchedSlots - kFwdEagerSlots);
    *out = base[dev] + 2 * slot;
    return FA_OK;
}

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
fa_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
    static std::mutex mu;
    static void* cache[64] = {};
    std::lock_guard<std::mutex> g(mu);
    if (cache[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
        cache[dev] = ptr;
    }
    *out = cache[dev];
    return FA_OK;
}

// ---- optional per-kernel event timing (fa_profile_begin / fa_profile_end)
struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;
    std::vector<int> kind;  // kind of each used pair
    size_t used = 0;
};
Profiler& prof() {
    static Profiler p;
    return p;
}

// Returns the event pair to bracket the next launch of `kind`, or null events
// when profiling is off.
std::pair<cudaEvent_t, cudaEvent_t> prof_pair(int kind) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.on) return {nullptr, nullptr};
    if (p.used == p.pool.size()) {
        if (p.pool.size() >= (1u << 20)) return {nullptr, nullptr};
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return {nullptr, nullptr};
        if (cudaEventCreate(&b) != cudaSuccess) {
            cudaEventDestroy(a);
            return {nullptr, nullptr};
        }
        p.pool.emplace_back(a, b);
        p.kind.push_back(kind);
    }
    p.kind[p.used] = kind;
    return p.pool[p.used++];
}

// Launch `fn` on `s`, bracketed by profiling events when enabled.
template <class F>
cudaError_t timed(int kind, cudaStream_t s, F&& fn) {
    auto ev = prof_pair(kind);
    if (ev.first) cudaEventRecord(ev.first, s);
    cudaError_t e = fn();
    if (ev.second) cudaEventRecord(ev.second, s);
    return e;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_str(fa_status s) {
    switch (s) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported (head dim or device)";
        case FA_ERR_CUDA: return "CUDA error";
        case FA_ERR_TIMEOUT: return "device-side wait timed out";
        case FA_ERR_TOO_LARGE: return "problem needs more scratch than the library's static region";
    }
    return "unknown status";
}

}  // extern "C"

namespace {

// Forward of fa_fwd (merge == nullptr) and fa_fwd_merge.
struct MergeArgs {
    float* o_acc;
    float* lse_acc;
    void* o_out;
    int first;
};

fa_status fwd_impl(const fa_shape* shape, const void* q, const void* k, const void* v, void* o, float* lse,
                   const MergeArgs* merge, void* stream) {
    fa_status st = check_shape(shape);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return FA_ERR_INVALID_ARG;
    if (merge) {
        if (!aligned16(merge->o_acc) || !aligned4(merge->lse_acc) ||
            (merge->o_out != nullptr && !aligned16(merge->o_out)))
            return FA_ERR_INVALID_ARG;
    } else if (!aligned16(o) || !aligned16(lse)) {
        return FA_ERR_INVALID_ARG;
    }
    if ((st = check_device()) != FA_OK) return st;
    const fa_shape& s = *shape;
    const bool pair = !merge && fwd_use_pair(s);   // the merge epilogue lives in the one-CTA kernel
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, q, s.B * s.Hq, s.N, s.D) || !make_map(&tk, k, s.B * s.Hkv, s.N, s.D, 2, pair ? kTileN / 2 : kTileN) ||
        !make_map(&tv, v, s.B * s.Hkv, s.N, s.D))
        return FA_ERR_CUDA;
    FwdParams p;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.N = s.N;
    p.causal = s.causal ? 1 : 0;
    p.scale_log2 = static_cast<float>(static_cast<double>(s.scale) * 1.4426950408889634);
    p.n_mblocks = pair ? (s.N + 4 * kTileM - 1) / (4 * kTileM) : (s.N + 2 * kTileM - 1) / (2 * kTileM);
    // Query heads per scheduling group: keep the K/V streamed by the group's
    // resident CTAs within ~32 MiB of L2.
    {
        const double per_head = 4.0 * s.N * s.D / (s.Hq / s.Hkv);
        const int g = static_cast<int>(32.0 * 1024 * 1024 / per_head);
        p.heads_per_group = g < 1 ? 1 : (g > s.B * s.Hq ? s.B * s.Hq : g);
    }
    p.o = o;
    p.lse = lse;
    p.o_scale = 1.f;
    p.m_o = merge ? merge->o_acc : nullptr;
    p.m_lse = merge ? merge->lse_acc : nullptr;
    p.m_out = merge ? merge->o_out : nullptr;
    p.m_first = merge ? (merge->first ? 1 : 0) : 0;
    // exponentials partly on the FMA pipe up to kFmaExpMaxN query rows (measured)
    p.fma_exp = s.N <= kFmaExpMaxN ? 1 : 0;
    p.n_units = p.n_mblocks * s.B * s.Hq;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    if ((st = fwd_sched_slot(strm, &p.sched)) != FA_OK) return st;
    cudaError_t e = pair ? timed(10, strm, [&] { return launch_fwd_pair(tq, tk, tv, p, strm); })
                         : timed(0, strm, [&] { return launch_fwd(s.D, tq, tk, tv, p, strm); });
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const fa_shape* shape, const void* q, const void* k, const void* v, void* o, float* lse,
                 void* stream) {
    return fwd_impl(shape, q, k, v, o, lse, nullptr, stream);
}

fa_status fa_fwd_merge(const fa_shape* shape, const void* q, const void* k, const void* v, float* o_acc,
                       float* lse_acc, void* o_out, int first, void* stream) {
    const MergeArgs m{o_acc, lse_acc, o_out, first};
    return fwd_impl(shape, q, k, v, nullptr, nullptr, &m, stream);
}

fa_status fa_fwd_fp8(const fa_shape* shape, const void* q, const void* k, const void* v, float q_scale,
                     float k_scale, float v_scale, void* o, float* lse, void* stream) {
    fa_status st = check_shape(shape);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
    for (float x : {q_scale, k_scale, v_scale})
        if (!std::isfinite(x) || !(x > 0.f)) return FA_ERR_INVALID_ARG;
    if (shape->D != 128) return FA_ERR_UNSUPPORTED;
    if ((st = check_device()) != FA_OK) return st;
    const fa_shape& s = *shape;
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, q, s.B * s.Hq, s.N, s.D, 1) || !make_map(&tk, k, s.B * s.Hkv, s.N, s.D, 1) ||
        !make_map(&tv, v, s.B * s.Hkv, s.N, s.D, 1))
        return FA_ERR_CUDA;
    FwdParams p;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.N = s.N;
    p.causal = s.causal ? 1 : 0;
    p.scale_log2 = static_cast<float>(static_cast<double>(s.scale) * 1.4426950408889634 * q_scale * k_scale);
    p.n_mblocks = (s.N + 2 * kTileM - 1) / (2 * kTileM);
    {
        // e4m3 K/V: half the bytes of bf16 per head, same ~32 MiB L2 budget
        const double per_head = 2.0 * s.N * s.D / (s.Hq / s.Hkv);
        const int g = static_cast<int>(32.0 * 1024 * 1024 / per_head);
        p.heads_per_group = g < 1 ? 1 : (g > s.B * s.Hq ? s.B * s.Hq : g);
    }
    p.o = o;
    p.lse = lse;
    p.o_scale = v_scale;
    p.m_o = nullptr;
    p.m_lse = nullptr;
    p.m_out = nullptr;
    p.m_first = 0;
    p.fma_exp = 0;
    p.n_units = p.n_mblocks * s.B * s.Hq;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    if ((st = fwd_sched_slot(strm, &p.sched)) != FA_OK) return st;
    cudaError_t e = timed(6, strm, [&] { return launch_fwd_fp8(tq, tk, tv, p, strm); });
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_workspace_bytes(const fa_kv_shape* shape) {
    if (check_kv_shape(shape) != FA_OK) return 0;
    return decode_plan(*shape).total;
}

fa_status fa_decode(const fa_kv_shape* shape, const void* q, const void* k, const void* v, void* o, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream) {
    fa_status st = check_kv_shape(shape);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
    const fa_kv_shape& s = *shape;
    const DecodePlan pl = decode_plan(s);
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < pl.total)
        return FA_ERR_INVALID_ARG;
    if ((st = check_device()) != FA_OK) return st;
    CUtensorMap tk, tv;
    if (!make_map(&tk, k, s.B * s.Hkv, s.Nk, s.D, 2, 64) || !make_map(&tv, v, s.B * s.Hkv, s.Nk, s.D, 2, 64))
        return FA_ERR_CUDA;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    DecodeParams p;
    p.q = q;
    p.o = o;
    p.lse = lse;
    p.o_part = reinterpret_cast<float*>(wsb + pl.o_part_off);
    p.lse_part = reinterpret_cast<float*>(wsb + pl.lse_part_off);
    p.Nq = s.Nq;
    p.Nk = s.Nk;
    p.G = s.Hq / s.Hkv;
    p.causal = s.causal ? 1 : 0;
    p.n_splits = pl.n_splits;
    p.tiles_per_split = pl.tiles_per_split;
    p.scale_log2 = static_cast<float>(static_cast<double>(s.scale) * 1.4426950408889634);
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    cudaError_t e = timed(7, strm, [&] { return launch_decode(s.D, tk, tv, p, pl.n_row_blocks, s.B * s.Hkv, strm); });
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_bytes(const fa_shape* shape) {
    if (check_shape(shape) != FA_OK) return 0;
    return bwd_workspace_layout(shape->B, shape->Hq, shape->N, shape->D, bwd_fused(*shape)).total;
}

}  // extern "C"

namespace {

// What bwd_impl runs: the whole backward (fa_bwd), only the row statistics
// into the workspace (fa_bwd_stats), or the two passes on statistics already
// in the workspace, adding into fp32 sums (fa_bwd_accumulate).
enum BwdMode { kBwdFull, kBwdFullDeterministic, kBwdStats, kBwdAccumulate };
struct AccArgs {
    float* dq;
    float* dk;
    float* dv;
    int first_dq, first_dkv;
};

fa_status bwd_impl(BwdMode mode, const fa_shape* shape, const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv, const AccArgs* acc,
                   void* workspace, size_t workspace_bytes, void* stream) {
    fa_status st = check_shape(shape);
    if (st != FA_OK) return st;
    const bool need_stats_in = mode != kBwdAccumulate;
    const bool need_passes = mode != kBwdStats;
    const bool full = mode == kBwdFull || mode == kBwdFullDeterministic;
    if (need_stats_in && (!aligned16(o) || !aligned16(dout) || !aligned4(lse))) return FA_ERR_INVALID_ARG;
    if (need_passes && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout))) return FA_ERR_INVALID_ARG;
    if (full && (!aligned16(dq) || !aligned16(dk) || !aligned16(dv))) return FA_ERR_INVALID_ARG;
    if (mode == kBwdAccumulate && (!acc || !aligned16(acc->dq) || !aligned16(acc->dk) || !aligned16(acc->dv)))
        return FA_ERR_INVALID_ARG;
    const fa_shape& s = *shape;
    // The fused kernel runs for fa_bwd when the backward mode selects it, and
    // for fa_bwd_accumulate too when D = 128 (dQ then goes straight into the
    // caller's fp32 sum); the workspace holds the fp32 dQ accumulator only for
    // fa_bwd, so the statistics entry points share the separate passes' layout.
    const bool fused = (mode == kBwdFull && bwd_fused(s)) || (mode == kBwdAccumulate && s.D == 128 && bwd_fused(s));
    const bool separate = !fused;
    const BwdWorkspace ws = bwd_workspace_layout(s.B, s.Hq, s.N, s.D, fused && mode == kBwdFull);
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < ws.total)
        return FA_ERR_INVALID_ARG;
    if ((st = check_device()) != FA_OK) return st;
    CUtensorMap tq, tk, tv, tdo;
    if (need_passes && (!make_map(&tq, q, s.B * s.Hq, s.N, s.D) || !make_map(&tk, k, s.B * s.Hkv, s.N, s.D) ||
                        !make_map(&tv, v, s.B * s.Hkv, s.N, s.D) || !make_map(&tdo, dout, s.B * s.Hq, s.N, s.D)))
        return FA_ERR_CUDA;
    // the accumulate epilogues live in the one-CTA passes
    const bool pair_dkdv = full && separate && bwd_dkdv_use_pair(s);
    const bool pair_dq = full && separate && bwd_dq_use_pair(s);
    CUtensorMap tq_half, tdo_half, tk_half, tv_half;
    if (pair_dkdv && (!make_map(&tq_half, q, s.B * s.Hq, s.N, s.D, 2, kTileM / 2) ||
                      !make_map(&tdo_half, dout, s.B * s.Hq, s.N, s.D, 2, kTileM / 2)))
        return FA_ERR_CUDA;
    if (pair_dq && (!make_map(&tk_half, k, s.B * s.Hkv, s.N, s.D, 2, kTileN / 2) ||
                    !make_map(&tv_half, v, s.B * s.Hkv, s.N, s.D, 2, kTileN / 2)))
        return FA_ERR_CUDA;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    const int Npad = (s.N + kTileM - 1) / kTileM * kTileM;
    BwdParams p;
    p.B = s.B;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.N = s.N;
    p.Npad = Npad;
    p.causal = s.causal ? 1 : 0;
    const int T = (s.N + kTileM - 1) / kTileM;
    // K/V heads per scheduling group of the key-block kernels: keep the
    // group's Q, dO (bf16) and, for the fused kernel, the fp32 dQ accumulator
    // of all its query heads within ~48 MiB of L2.  With fewer than two waves
    // of work units, one group (global heaviest-first order) balances better.
    {
        const double per_kv_head = (separate ? 4.0 : 8.0) * s.N * s.D * (s.Hq / s.Hkv);
        int g = static_cast<int>(48.0 * 1024 * 1024 / per_kv_head);
        if (static_cast<long long>(T) * s.B * s.Hkv < 2LL * kNumSMs) g = s.B * s.Hkv;
        p.heads_per_group = g < 1 ? 1 : (g > s.B * s.Hkv ? s.B * s.Hkv : g);
    }
    // query heads per group of the dQ pass: K/V streamed by the group in ~32 MiB
    {
        const double per_head = 4.0 * s.N * s.D / (s.Hq / s.Hkv);
        const int g = static_cast<int>(32.0 * 1024 * 1024 / per_head);
        p.dq_heads_per_group = g < 1 ? 1 : (g > s.B * s.Hq ? s.B * s.Hq : g);
    }
    p.scale = s.scale;
    p.scale_log2 = static_cast<float>(static_cast<double>(s.scale) * 1.4426950408889634);
    p.lse2 = reinterpret_cast<const float*>(wsb + ws.lse2_off);
    p.dvec = reinterpret_cast<const float*>(wsb + ws.dvec_off);
    p.dq_acc = (fused && mode == kBwdFull) ? reinterpret_cast<float*>(wsb + ws.dq_off) : nullptr;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.sched = reinterpret_cast<unsigned int*>(wsb + ws.sched_off);
    p.n_units_dkdv = (pair_dkdv ? (s.N + 2 * kTileN - 1) / (2 * kTileN) : T) * s.B * s.Hkv;
    p.n_units_dq = (pair_dq ? (s.N + 2 * kTileM - 1) / (2 * kTileM) : T) * s.B * s.Hq;
    p.a_dq = mode == kBwdAccumulate ? acc->dq : nullptr;
    p.a_dk = mode == kBwdAccumulate ? acc->dk : nullptr;
    p.a_dv = mode == kBwdAccumulate ? acc->dv : nullptr;
    p.a_first_dq = mode == kBwdAccumulate && acc->first_dq ? 1 : 0;
    p.a_first_dkv = mode == kBwdAccumulate && acc->first_dkv ? 1 : 0;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (need_stats_in) {
        e = timed(1, strm, [&] {
            return launch_bwd_preprocess(s.D, o, dout, lse, reinterpret_cast<float*>(wsb + ws.lse2_off),
                                         reinterpret_cast<float*>(wsb + ws.dvec_off), p.dq_acc,
                                         s.B * s.Hq, s.N, Npad, s.scale,
                                         reinterpret_cast<unsigned int*>(wsb + ws.sched_off), strm);
        });
    } else {
        // statistics already in the workspace; only the work counters restart
        e = cudaMemsetAsync(wsb + ws.sched_off, 0, kSchedCounters * sizeof(unsigned int), strm);
    }
    if (!need_passes) return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    if (separate) {
        if (e == cudaSuccess)
            e = pair_dkdv ? timed(11, strm, [&] { return launch_bwd_dkdv_pair(tq, tq_half, tk, tv, tdo, tdo_half, p, strm); })
                     : timed(4, strm, [&] { return launch_bwd_dkdv(s.D, tq, tk, tv, tdo, p, strm); });
        if (e == cudaSuccess)
            e = pair_dq ? timed(12, strm, [&] { return launch_bwd_dq_pair(tq, tk, tk_half, tv_half, tdo, p, strm); })
                     : timed(5, strm, [&] { return launch_bwd_dq(s.D, tq, tk, tv, tdo, p, strm); });
    } else {
        // accumulate mode: the kernel's reductions add into the caller's dQ sum,
        // which a first call clears
        if (e == cudaSuccess && mode == kBwdAccumulate && acc->first_dq)
            e = cudaMemsetAsync(acc->dq, 0, static_cast<size_t>(s.B) * s.Hq * s.N * s.D * sizeof(float), strm);
        if (e == cudaSuccess)
            e = s.D == 128 ? timed(13, strm, [&] { return launch_bwd_fused(tq, tk, tv, tdo, p, strm); })
                           : timed(2, strm, [&] { return launch_bwd_main(s.D, tq, tk, tv, tdo, p, strm); });
        if (e == cudaSuccess && mode == kBwdFull)
            e = timed(3, strm, [&] {
                return launch_bwd_dq_convert(p.dq_acc, dq, static_cast<size_t>(s.B) * s.Hq * s.N * s.D, strm);
            });
    }
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_bwd(const fa_shape* shape, const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                 void* stream) {
    return bwd_impl(kBwdFull, shape, q, k, v, o, dout, lse, dq, dk, dv, nullptr, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_stats(const fa_shape* shape, const void* o, const void* dout, const float* lse, void* workspace,
                       size_t workspace_bytes, void* stream) {
    return bwd_impl(kBwdStats, shape, nullptr, nullptr, nullptr, o, dout, lse, nullptr, nullptr, nullptr, nullptr,
                    workspace, workspace_bytes, stream);
}

fa_status fa_bwd_accumulate(const fa_shape* shape, const void* q, const void* k, const void* v, const void* dout,
                            float* dq_acc, float* dk_acc, float* dv_acc, int flags, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (flags & ~(FA_ACC_DQ_FIRST | FA_ACC_DKV_FIRST)) return FA_ERR_INVALID_ARG;
    const AccArgs a{dq_acc, dk_acc, dv_acc, (flags & FA_ACC_DQ_FIRST) ? 1 : 0, (flags & FA_ACC_DKV_FIRST) ? 1 : 0};
    return bwd_impl(kBwdAccumulate, shape, q, k, v, nullptr, dout, nullptr, nullptr, nullptr, nullptr, &a, workspace,
                    workspace_bytes, stream);
}

// fa_bwd with its workspace taken from the library's static scratch instead of
// the caller: for callers that cannot allocate device memory on this path.
fa_status fa_bwd_noalloc(const fa_shape* shape, const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, void* stream) {
    fa_status st = check_shape(shape);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned4(lse) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_INVALID_ARG;
    if (bwd_workspace_layout(shape->B, shape->Hq, shape->N, shape->D, false).total > FA_NOALLOC_SCRATCH_BYTES)
        return FA_ERR_TOO_LARGE;
    if ((st = check_device()) != FA_OK) return st;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != FA_OK) return st;
    return bwd_impl(kBwdFullDeterministic, shape, q, k, v, o, dout, lse, dq, dk, dv, nullptr, scratch,
                    FA_NOALLOC_SCRATCH_BYTES, stream);
}

fa_status fa_set_bwd_mode(int mode) {
    if (mode != FA_BWD_AUTO && mode != FA_BWD_DETERMINISTIC && mode != FA_BWD_FUSED) return FA_ERR_INVALID_ARG;
    g_bwd_mode.store(mode, std::memory_order_relaxed);
    return FA_OK;
}

int fa_get_bwd_mode(void) { return g_bwd_mode.load(std::memory_order_relaxed); }

fa_status fa_lse_merge(long long rows, int D, const void* o_part, const float* lse_part, float* o_acc,
                       float* lse_acc, void* o_out, int first, void* stream) {
    if (rows < 0) return FA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    if (rows == 0) return FA_OK;  // nothing is read; empty tensors may carry null pointers
    if (!aligned16(o_part) || !aligned16(o_acc) || (o_out != nullptr && !aligned16(o_out))) return FA_ERR_INVALID_ARG;
    if (lse_part == nullptr || lse_acc == nullptr || (reinterpret_cast<uintptr_t>(lse_part) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(lse_acc) & 3u) != 0)
        return FA_ERR_INVALID_ARG;
    fa_status st = check_device();
    if (st != FA_OK) return st;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    cudaError_t e = timed(8, strm, [&] {
        return launch_lse_merge(D, rows, o_part, lse_part, o_acc, lse_acc, o_out, first, strm);
    });
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_accumulate(long long n, const void* src, float* acc, void* out, int first, void* stream) {
    if (n < 0 || (n & 7) != 0) return FA_ERR_INVALID_ARG;
    if (n == 0) return FA_OK;  // nothing is read; empty tensors may carry null pointers
    if (!aligned16(acc) || (src != nullptr && !aligned16(src)) || (out != nullptr && !aligned16(out)))
        return FA_ERR_INVALID_ARG;
    fa_status st = check_device();
    if (st != FA_OK) return st;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    cudaError_t e = timed(9, strm, [&] { return launch_accumulate(n, src, acc, out, first, strm); });
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_status, sizeof(word)) != cudaSuccess) return FA_ERR_CUDA;
    g_last_sites = word;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
        return FA_ERR_TIMEOUT;
    }
    return FA_OK;
}

unsigned int fa_debug_timeout_sites(void) { return g_last_sites; }

fa_status fa_profile_begin(void) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    p.on = true;
    p.used = 0;
    return FA_OK;
}

fa_status fa_profile_end(float* total_ms, int* launches) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    p.on = false;
    if (!total_ms || !launches) return FA_ERR_INVALID_ARG;
    for (int k = 0; k < FA_PROFILE_KINDS; ++k) {
        total_ms[k] = 0.f;
        launches[k] = 0;
    }
    fa_status st = FA_OK;
    for (size_t i = 0; i < p.used; ++i) {
        if (cudaEventSynchronize(p.pool[i].second) != cudaSuccess) {
            st = FA_ERR_CUDA;
            continue;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.pool[i].first, p.pool[i].second) != cudaSuccess) {
            st = FA_ERR_CUDA;
            continue;
        }
        total_ms[p.kind[i]] += ms;
        launches[p.kind[i]] += 1;
    }
    p.used = 0;
    return st;
}

}  // extern "C"
