// monarch_attn.cu -- C ABI of the Monarch attention forward (include/monarch_attn.h):
// argument validation, TMA tensor-map construction (the (T,H,W) reshape and
// the stage permutation P are expressed as tensor-map boxes), and kernel
// launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/monarch_attn.h"
#include "attn_chunk.cuh"
#include "attn_f32.cuh"
#include "attn_tc.cuh"

namespace monarch {

__device__ unsigned g_device_status = 0u;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    int sms = 0;
    bool tc_attr[4] = {false, false, false, false};  // [fp16][d == 128]
    bool f32_attr[2] = {false, false};
};

// Per (device, stream) buffer of per-batch-head stage-1 completion counters:
// calls queued on one stream run in order, so each buffer is used by one call
// at a time; calls on different streams get different buffers.
struct CounterBuf {
    int dev;
    cudaStream_t stream;
    unsigned *ptr;
    size_t cap;  // elements
};
std::vector<CounterBuf> g_counters;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return MONARCH_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return MONARCH_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return MONARCH_OK;
}

int device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &di = g_dev[dev];
    if (!di.init) {
        int sms = 0, major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MONARCH_ERR_CUDA;
        if (major != 10 || minor != 0) return MONARCH_ERR_UNSUPPORTED;  // built for sm_100a only
        di.sms = sms;
        di.init = true;
    }
    *out = &di;
    return MONARCH_OK;
}

// Counter buffer of at least n elements for (current device, stream),
// allocated on first use; when a call needs more, the stream is drained and
// the buffer replaced.
// Per (device, stream) scratch for the (f*h, w) split's stage-1 output,
// allocated on first use and replaced (after draining the stream) when a call
// needs more.
struct ScratchBuf {
    int dev;
    cudaStream_t stream;
    void *ptr;
    size_t cap;
};
std::vector<ScratchBuf> g_scratch;

int scratch_for(cudaStream_t stream, size_t bytes, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    ScratchBuf *sb = nullptr;
    for (auto &c : g_scratch)
        if (c.dev == dev && c.stream == stream) sb = &c;
    if (!sb) {
        g_scratch.push_back(ScratchBuf{dev, stream, nullptr, 0});
        sb = &g_scratch.back();
    }
    if (sb->cap < bytes) {
        if (sb->ptr) {
            if (cudaStreamSynchronize(stream) != cudaSuccess) return MONARCH_ERR_CUDA;
            cudaFree(sb->ptr);
            sb->ptr = nullptr;
            sb->cap = 0;
        }
        if (cudaMalloc(&sb->ptr, bytes) != cudaSuccess) return MONARCH_ERR_CUDA;
        sb->cap = bytes;
    }
    *out = sb->ptr;
    return MONARCH_OK;
}

int counters_for(cudaStream_t stream, size_t n, unsigned **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    CounterBuf *cb = nullptr;
    for (auto &c : g_counters)
        if (c.dev == dev && c.stream == stream) cb = &c;
    if (!cb) {
        g_counters.push_back(CounterBuf{dev, stream, nullptr, 0});
        cb = &g_counters.back();
    }
    if (cb->cap < n) {
        const size_t cap = n < 1024 ? 1024 : n;
        if (cb->ptr) {
            if (cudaStreamSynchronize(stream) != cudaSuccess) return MONARCH_ERR_CUDA;
            cudaFree(cb->ptr);
            cb->ptr = nullptr;
            cb->cap = 0;
        }
        if (cudaMalloc(reinterpret_cast<void **>(&cb->ptr), cap * sizeof(unsigned)) != cudaSuccess)
            return MONARCH_ERR_CUDA;
        cb->cap = cap;
    }
    *out = cb->ptr;
    return MONARCH_OK;
}

// Completion counters for monarch_attn_fwd_noalloc: a file-scope device array
// (4096 words, 16 KB) in place of the per-stream cudaMalloc buffer above, its
// address looked up once per device.  One array per device means calls of
// that entry point on one device must not overlap in time.
static __device__ __align__(256) unsigned g_noalloc_counters[MONARCH_NOALLOC_MAX_BH];
unsigned *g_noalloc_ptr[kMaxDevices] = {};

int noalloc_counters(unsigned **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_counters) != cudaSuccess || ptr == nullptr)
            return MONARCH_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<unsigned *>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return MONARCH_OK;
}

bool env_debug() {
    const char *e = std::getenv("MONARCH_ATTN_DEBUG");
    return e && e[0] == '1';
}

long long env_timeout_cycles() {
    const char *e = std::getenv("MONARCH_ATTN_TIMEOUT_CYCLES");
    if (e && *e) {
        long long v = std::atoll(e);
        if (v > 0) return v;
    }
    return 4000000000ll;  // about 2 s at the B200 boost clock
}

bool overlaps(const void *a, const void *b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

struct Shape {
    int B, heads, T, H, W, d, fact, tile_h, tile_w, dtype;
    long long N, elems;
    long long sB = 0, sH = 0, sN = 0;  // element strides; all 0 = contiguous [B][heads][N][d]
};

int validate(const void *q, const void *k, const void *v, void *out, Shape &s) {
    if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
    if (s.B < 1 || s.heads < 1 || s.T < 1 || s.H < 1 || s.W < 1) return MONARCH_ERR_INVALID_ARG;
    if (s.d != 64 && s.d != 128) return MONARCH_ERR_INVALID_ARG;
    if (s.dtype != MONARCH_DTYPE_F32 && s.dtype != MONARCH_DTYPE_BF16 && s.dtype != MONARCH_DTYPE_F16)
        return MONARCH_ERR_INVALID_ARG;
    if (s.fact != MONARCH_FACT_FRAME && s.fact != MONARCH_FACT_TILED && s.fact != MONARCH_FACT_ROW)
        return MONARCH_ERR_INVALID_ARG;
    if (s.fact == MONARCH_FACT_TILED) {
        if (s.tile_h < 1 || s.tile_w < 1 || s.H % s.tile_h != 0 || s.W % s.tile_w != 0)
            return MONARCH_ERR_INVALID_ARG;
    }
    for (const void *p : {q, k, v, static_cast<const void *>(out)})
        if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return MONARCH_ERR_INVALID_ARG;
    s.N = static_cast<long long>(s.T) * s.H * s.W;
    if (s.N > (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    s.elems = static_cast<long long>(s.B) * s.heads * s.N * s.d;
    const long long cB = static_cast<long long>(s.heads) * s.N * s.d, cH = s.N * s.d, cN = s.d;
    if (s.sB == 0 && s.sH == 0 && s.sN == 0) {
        s.sB = cB; s.sH = cH; s.sN = cN;
    } else {
        if (s.sB < 1 || s.sH < 1 || s.sN < 1) return MONARCH_ERR_INVALID_ARG;
        // rows must not overlap: sorted by stride, each stride covers the dims below it
        long long st[3] = {s.sN, s.sH, s.sB}, ex[3] = {s.N, s.heads, s.B};
        for (int a = 0; a < 3; ++a)
            for (int b = a + 1; b < 3; ++b)
                if (st[b] < st[a]) { std::swap(st[a], st[b]); std::swap(ex[a], ex[b]); }
        long long need = s.d;
        for (int a = 0; a < 3; ++a) {
            if (ex[a] == 1) continue;
            if (st[a] < need) return MONARCH_ERR_INVALID_ARG;
            need = st[a] * ex[a];
        }
        // 16-bit paths read through TMA: strides must be 16-byte multiples
        if (s.dtype != MONARCH_DTYPE_F32 && (s.sB % 8 || s.sH % 8 || s.sN % 8)) return MONARCH_ERR_INVALID_ARG;
        // the tiled factorisation's tensor map (also used by the row split's
        // column pass) needs the contiguous layout
        if (s.fact != MONARCH_FACT_FRAME && (s.sB != cB || s.sH != cH || s.sN != cN))
            return MONARCH_ERR_UNSUPPORTED;
    }
    const long long span = (s.B - 1) * s.sB + (s.heads - 1) * s.sH + (s.N - 1) * s.sN + s.d;
    const size_t bytes = static_cast<size_t>(span) * (s.dtype == MONARCH_DTYPE_F32 ? 4 : 2);
    if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
        return MONARCH_ERR_INVALID_ARG;
    if (s.T > 128 && s.fact != MONARCH_FACT_ROW) return MONARCH_ERR_UNSUPPORTED;
    if (s.fact == MONARCH_FACT_TILED && s.tile_w > 128) return MONARCH_ERR_UNSUPPORTED;
    if (static_cast<long long>(s.B) * s.heads > (1ll << 30)) return MONARCH_ERR_UNSUPPORTED;
    return MONARCH_OK;
}

// <tc-launch> (the tensor-core kernel's launch code; profile summaries hash
// this region with the kernel's own sources)
// 16-bit (bf16 or fp16) tensor map with 128-byte swizzle; dims/strides
// innermost first, strides in bytes for dims 1..rank-1.
int make_map(CUtensorMap *map, const void *ptr, int rank, const cuuint64_t *dims,
             const cuuint64_t *strides, const cuuint32_t *box, int dtype) {
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType ty =
        dtype == MONARCH_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = g_encode(map, ty, rank, const_cast<void *>(ptr), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MONARCH_OK : MONARCH_ERR_CUDA;
}

// Stage-1 view of a 16-bit tensor with element strides (sB, sH, sN).
//   frame: (d, m, T, heads, B), box (64, 128, 1, 1, 1): one 128-token slab of a frame
//   tiled: (d, tile_w, tiles_w, tile_h, tiles_h*B*heads*T),
//          box (64, tile_w, 1, rows, 1): `rows` tile rows of one tile
int stage1_map(CUtensorMap *map, const void *ptr, const Shape &s, const TcParams &p) {
    const cuuint64_t es = 2, d = s.d;
    if (s.fact == MONARCH_FACT_FRAME) {
        const cuuint64_t sN = static_cast<cuuint64_t>(s.sN);
        cuuint64_t dims[5] = {d, static_cast<cuuint64_t>(p.m), static_cast<cuuint64_t>(s.T),
                              static_cast<cuuint64_t>(s.heads), static_cast<cuuint64_t>(s.B)};
        cuuint64_t strides[4] = {sN * es, static_cast<cuuint64_t>(p.m) * sN * es,
                                 static_cast<cuuint64_t>(s.sH) * es, static_cast<cuuint64_t>(s.sB) * es};
        cuuint32_t box[5] = {64, 128, 1, 1, 1};
        return make_map(map, ptr, 5, dims, strides, box, s.dtype);
    }
    cuuint64_t dims[5] = {d, static_cast<cuuint64_t>(s.tile_w), static_cast<cuuint64_t>(p.tiles_w),
                          static_cast<cuuint64_t>(s.tile_h),
                          static_cast<cuuint64_t>(p.tiles_h) * s.B * s.heads * s.T};
    cuuint64_t strides[4] = {d * es, static_cast<cuuint64_t>(s.tile_w) * d * es,
                             static_cast<cuuint64_t>(s.W) * d * es,
                             static_cast<cuuint64_t>(s.tile_h) * s.W * d * es};
    cuuint32_t box[5] = {64, static_cast<cuuint32_t>(s.tile_w), 1,
                         static_cast<cuuint32_t>(p.rows_per_tile), 1};
    return make_map(map, ptr, 5, dims, strides, box, s.dtype);
}

// Stage-2 view: (d, H*W, T, heads, B), box (64, npos, T, 1, 1): npos consecutive
// positions across all T frames, landing in shared memory as rows t*npos + pos.
int stage2_map(CUtensorMap *map, const void *ptr, const Shape &s, const TcParams &p) {
    const cuuint64_t es = 2, d = s.d, sN = static_cast<cuuint64_t>(s.sN);
    cuuint64_t dims[5] = {d, static_cast<cuuint64_t>(p.HW), static_cast<cuuint64_t>(s.T),
                          static_cast<cuuint64_t>(s.heads), static_cast<cuuint64_t>(s.B)};
    cuuint64_t strides[4] = {sN * es, static_cast<cuuint64_t>(p.HW) * sN * es,
                             static_cast<cuuint64_t>(s.sH) * es, static_cast<cuuint64_t>(s.sB) * es};
    cuuint32_t box[5] = {64, static_cast<cuuint32_t>(p.npos), static_cast<cuuint32_t>(s.T), 1, 1};
    return make_map(map, ptr, 5, dims, strides, box, s.dtype);
}

// Optional per-launch events: ev[0] before the first launch, ev[i+1] after launch i.
struct LaunchEvents {
    void **ev = nullptr;
    int n = 0;
    int launches = 0;
    void record(int idx, cudaStream_t s) const {
        if (ev && idx < n && ev[idx]) cudaEventRecord(static_cast<cudaEvent_t>(ev[idx]), s);
    }
    // ev[0], once per call: a call that makes several launches through these
    // helpers records it before its first launch only
    void start(cudaStream_t s) const {
        if (launches == 0) record(0, s);
    }
};

template <int D, bool F16>
int launch_tc(const void *q, const void *k, const void *v, void *out, const Shape &s,
              cudaStream_t stream, LaunchEvents &lev, unsigned *fixed_counters = nullptr,
              bool stage1_only = false) {
    DeviceInfo *di = nullptr;
    int st = device_info(&di);
    if (st) return st;
    if ((st = get_encode())) return st;
    using L = TcLayout<D>;
    const int di_idx = (F16 ? 2 : 0) + (D == 128 ? 1 : 0);
    if (!di->tc_attr[di_idx]) {
        if (cudaFuncSetAttribute(monarch_tc_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 L::ALLOC) != cudaSuccess)
            return MONARCH_ERR_CUDA;
        di->tc_attr[di_idx] = true;
    }
    TcParams p{};
    p.B = s.B; p.heads = s.heads; p.T = s.T; p.H = s.H; p.W = s.W; p.HW = s.H * s.W;
    p.N = s.N;
    p.fact = s.fact;
    if (s.fact == MONARCH_FACT_TILED) {
        p.tile_h = s.tile_h; p.tile_w = s.tile_w;
        p.tiles_h = s.H / s.tile_h; p.tiles_w = s.W / s.tile_w;
        const int r = 128 / s.tile_w;
        p.rows_per_tile = r < s.tile_h ? r : s.tile_h;
        p.m = s.tile_h * s.tile_w;
        p.nblk_bh = s.T * p.tiles_h * p.tiles_w;
        p.nqt = (s.tile_h + p.rows_per_tile - 1) / p.rows_per_tile;
    } else {
        p.tile_h = p.tile_w = p.tiles_h = p.tiles_w = 0;
        p.rows_per_tile = 0;
        p.m = p.HW;
        p.nblk_bh = s.T;
        p.nqt = (p.m + 127) / 128;
    }
    const long long bh = static_cast<long long>(s.B) * s.heads;
    if (bh * p.nblk_bh >= (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    p.nblocks = static_cast<int>(bh * p.nblk_bh);
    p.BH = static_cast<int>(bh);
    p.ns = p.nqt / 2;
    p.odd = p.nqt % 2;
    p.upg = 2 * p.ns + p.odd;
    p.npos = stage1_only ? 1 : 128 / s.T;  // stage 1 alone may run on more than 128 frames
    p.s2_chunks = (p.HW + p.npos - 1) / p.npos;
    p.s2_pairs = (p.s2_chunks + 1) / 2;
    // stage-1 units per batch-head: blocks in pairs, each pair = the shared
    // query-tile pairs of both blocks plus one unit joining their odd tiles
    p.u1_bh = (p.nblk_bh / 2) * p.upg + (p.nblk_bh % 2) * (p.ns + p.odd);
    // stage 1 alone (Y1 into `out`): no stage-2 units
    if (stage1_only) p.s2_pairs = 0;
    const long long units = bh * (p.u1_bh + p.s2_pairs);
    if (units >= (1ll << 31) - 1) return MONARCH_ERR_UNSUPPORTED;
    p.units = static_cast<int>(units);
    p.s1_target = static_cast<unsigned>(p.nblk_bh) * static_cast<unsigned>(p.nqt);
    // Stage-2 units of a batch-head trail its stage-1 units by about two
    // waves of the persistent grid, so they rarely wait on their inputs.
    {
        const long long wave = di->sms;
        long long lag = (2 * wave + p.u1_bh - 1) / p.u1_bh;
        if (lag < 1) lag = 1;
        if (lag > bh || stage1_only) lag = bh;
        p.lag = static_cast<int>(lag);
    }
    p.fd_u1 = make_fastdiv(static_cast<uint32_t>(p.u1_bh));
    p.fd_u12 = make_fastdiv(static_cast<uint32_t>(p.u1_bh + p.s2_pairs));
    p.fd_u2 = make_fastdiv(static_cast<uint32_t>(p.s2_pairs));
    p.fd_upg = make_fastdiv(static_cast<uint32_t>(p.upg));
    p.fd_nblk_bh = make_fastdiv(static_cast<uint32_t>(p.nblk_bh));
    p.fd_tpf = make_fastdiv(static_cast<uint32_t>(p.fact ? p.tiles_h * p.tiles_w : 1));
    p.fd_tiles_w = make_fastdiv(static_cast<uint32_t>(p.fact ? p.tiles_w : 1));
    p.fd_tile_w = make_fastdiv(static_cast<uint32_t>(p.fact ? p.tile_w : 1));
    p.fd_npos = make_fastdiv(static_cast<uint32_t>(p.npos));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(s.d)));
    p.timeout_cycles = env_timeout_cycles();
    p.out = out;
    p.sB = s.sB; p.sH = s.sH; p.sN = s.sN;
    p.fd_heads = make_fastdiv(static_cast<uint32_t>(s.heads));
    p.out_v8 = ((reinterpret_cast<uintptr_t>(out) & 31u) == 0 && s.sB % 16 == 0 && s.sH % 16 == 0 &&
                s.sN % 16 == 0) ? 1 : 0;
    unsigned *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_device_status) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    p.status = status;

    CUtensorMap mq1, mk1, mv1, mq2, mk2, my2;
    if ((st = stage1_map(&mq1, q, s, p)) || (st = stage1_map(&mk1, k, s, p)) || (st = stage1_map(&mv1, v, s, p)))
        return st;
    if (stage1_only) {  // no stage-2 units read them
        mq2 = mq1; mk2 = mk1; my2 = mv1;
    } else if ((st = stage2_map(&mq2, q, s, p)) || (st = stage2_map(&mk2, k, s, p)) ||
               (st = stage2_map(&my2, out, s, p))) {
        return st;
    }

    // One persistent launch runs both stages: stage-1 units write Y1 = B1 V
    // into out; stage-2 units overwrite it in place with P^T B2 P Y1 once the
    // stage-1 lanes of their batch-head have published (per-batch-head
    // counters, zeroed for every call).
    unsigned *counters = fixed_counters;
    if (!counters && (st = counters_for(stream, static_cast<size_t>(bh), &counters))) return st;
    p.s1_done = counters;
    if (cudaMemsetAsync(counters, 0, static_cast<size_t>(bh) * sizeof(unsigned), stream) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    lev.start(stream);
    const int grid = p.units < di->sms ? p.units : di->sms;
    monarch_tc_kernel<D, F16><<<grid, 640, L::ALLOC, stream>>>(mq1, mk1, mv1, mq2, mk2, my2, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    lev.record(++lev.launches, stream);
    return MONARCH_OK;
}
// </tc-launch>

template <int D>
int launch_f32(const void *q, const void *k, const void *v, void *out, const Shape &s,
               cudaStream_t stream, LaunchEvents &lev, bool stage1_only = false) {
    DeviceInfo *di = nullptr;
    int st = device_info(&di);
    if (st) return st;
    F32Params p{};
    p.T = s.T; p.H = s.H; p.W = s.W; p.HW = s.H * s.W; p.N = s.N;
    p.fact = s.fact;
    if (s.fact == MONARCH_FACT_TILED) {
        p.tile_h = s.tile_h; p.tile_w = s.tile_w;
        p.tiles_h = s.H / s.tile_h; p.tiles_w = s.W / s.tile_w;
        p.m = s.tile_h * s.tile_w;
        p.nblk_bh = s.T * p.tiles_h * p.tiles_w;
    } else {
        p.m = p.HW;
        p.nblk_bh = s.T;
    }
    p.qchunks = (p.m + 63) / 64;
    p.heads = s.heads;
    p.sB = s.sB; p.sH = s.sH; p.sN = s.sN;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.d)));
    const long long bh = static_cast<long long>(s.B) * s.heads;
    const long long g1 = bh * p.nblk_bh * p.qchunks;
    const long long g2 = bh * p.HW;
    if (g1 >= (1ll << 31) || g2 >= (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    const int smem2 = 2 * s.T * D * 4;
    const int di_idx = D == 128 ? 1 : 0;
    if (!di->f32_attr[di_idx]) {
        if (cudaFuncSetAttribute(monarch_f32_stage2<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 2 * 128 * D * 4) != cudaSuccess)
            return MONARCH_ERR_CUDA;
        di->f32_attr[di_idx] = true;
    }
    const float *fq = static_cast<const float *>(q);
    const float *fk = static_cast<const float *>(k);
    const float *fv = static_cast<const float *>(v);
    float *fo = static_cast<float *>(out);
    lev.start(stream);
    monarch_f32_stage1<D><<<static_cast<unsigned>(g1), 128, 0, stream>>>(fq, fk, fv, fo, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    lev.record(++lev.launches, stream);
    if (stage1_only) return MONARCH_OK;
    const int threads2 = ((2 * s.T + 31) / 32) * 32;
    monarch_f32_stage2<D><<<static_cast<unsigned>(g2), threads2, smem2, stream>>>(fq, fk, fo, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    lev.record(++lev.launches, stream);
    return MONARCH_OK;
}

// The (f*h, w) split: tokens form a (T*H) x W grid; stage-1 blocks are its
// rows (the W tokens of one frame row), stage-2 groups its columns (the T*H
// tokens sharing w).  Both are stage-1 passes of the forward's kernels over
// virtual shapes of the same [B][heads][N][d] tensors (token n = r*W + w):
//   rows:    T*H frames of 1 x W, frame split          -> Y1 into the scratch
//   columns: one frame of (T*H) x W, tiles (T*H) x 1   -> out, values = Y1
template <int D, typename E>
int launch_row(const void *q, const void *k, const void *v, void *out, const Shape &s, cudaStream_t stream,
               LaunchEvents &lev) {
    void *y1 = nullptr;
    int st = scratch_for(stream, static_cast<size_t>(s.elems) * sizeof(E), &y1);
    if (st) return st;
    Shape rows = s;
    rows.T = s.T * s.H; rows.H = 1; rows.fact = MONARCH_FACT_FRAME; rows.tile_h = rows.tile_w = 0;
    Shape cols = s;
    cols.T = 1; cols.H = s.T * s.H; cols.fact = MONARCH_FACT_TILED; cols.tile_h = s.T * s.H; cols.tile_w = 1;
    constexpr bool tc = !std::is_same<E, float>::value;
    if constexpr (tc) {
        constexpr bool f16 = std::is_same<E, __half>::value;
        if ((st = launch_tc<D, f16>(q, k, v, y1, rows, stream, lev, nullptr, true))) return st;
        return launch_tc<D, f16>(q, k, y1, out, cols, stream, lev, nullptr, true);
    } else {
        if ((st = launch_f32<D>(q, k, v, y1, rows, stream, lev, true))) return st;
        return launch_f32<D>(q, k, y1, out, cols, stream, lev, true);
    }
}

// <chunk-launch> (hashed with attn_chunk.cuh by the profile summaries)
// Stage 2 of an autoregressive chunk (attn_chunk.cuh).
template <int D, typename E>
int launch_chunk_stage2(const void *q, const void *k, const void *k_cache, const void *y1_cache,
                        const void *y1_new, void *out, const Shape &s, int T_old, cudaStream_t stream,
                        LaunchEvents &lev) {
    ChunkParams p{};
    p.HW = s.H * s.W;
    p.T_old = T_old;
    p.T_new = s.T;
    p.n_old = static_cast<long long>(T_old) * p.HW;
    p.n_new = s.N;
    p.groups = static_cast<long long>(s.B) * s.heads * p.HW;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    if (p.groups / ChunkCfg<D, E>::WARPS >= (1ll << 31) - 1) return MONARCH_ERR_UNSUPPORTED;
    if (chunk_stage2_launch<D, E>(static_cast<const E *>(q), static_cast<const E *>(k),
                                  static_cast<const E *>(k_cache), static_cast<const E *>(y1_cache),
                                  static_cast<const E *>(y1_new), static_cast<E *>(out), p, stream) != cudaSuccess)
        return MONARCH_ERR_LAUNCH;
    lev.record(++lev.launches, stream);
    return MONARCH_OK;
}
// </chunk-launch>

__global__ void selftest_timeout_kernel(long long limit, unsigned *status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0u;
        mbar_init(smem_addr(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        WaitCtl ctl{&abort_flag, status, limit};
        // nothing ever arrives on this barrier: the wait must give up
        (void)mbar_wait(smem_addr(&bar), 0u, ctl);
    }
}

int read_status(cudaStream_t stream, int reset) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MONARCH_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return MONARCH_ERR_CUDA;
    if (reset && v) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
            return MONARCH_ERR_CUDA;
    }
    if (v & DEVERR_TIMEOUT) return MONARCH_ERR_TIMEOUT;
    if (v & DEVERR_ALIGN) return MONARCH_ERR_LAUNCH;
    return MONARCH_OK;
}

}  // namespace
}  // namespace monarch

using namespace monarch;

extern "C" {

static int fwd_impl(const void *q, const void *k, const void *v, void *out, int B, int heads, int T,
                    int H, int W, int d, int factorisation, int tile_h, int tile_w, int dtype,
                    void *stream, LaunchEvents &lev, long long sb = 0, long long sh = 0, long long sn = 0) {
    Shape s{B, heads, T, H, W, d, factorisation, tile_h, tile_w, dtype, 0, 0};
    s.sB = sb; s.sH = sh; s.sN = sn;
    int st = validate(q, k, v, out, s);
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (factorisation == MONARCH_FACT_ROW) {
        if (dtype == MONARCH_DTYPE_BF16)
            st = d == 128 ? launch_row<128, __nv_bfloat16>(q, k, v, out, s, cs, lev)
                          : launch_row<64, __nv_bfloat16>(q, k, v, out, s, cs, lev);
        else if (dtype == MONARCH_DTYPE_F16)
            st = d == 128 ? launch_row<128, __half>(q, k, v, out, s, cs, lev)
                          : launch_row<64, __half>(q, k, v, out, s, cs, lev);
        else
            st = d == 128 ? launch_row<128, float>(q, k, v, out, s, cs, lev)
                          : launch_row<64, float>(q, k, v, out, s, cs, lev);
    } else if (dtype == MONARCH_DTYPE_BF16)
        st = d == 128 ? launch_tc<128, false>(q, k, v, out, s, cs, lev) : launch_tc<64, false>(q, k, v, out, s, cs, lev);
    else if (dtype == MONARCH_DTYPE_F16)
        st = d == 128 ? launch_tc<128, true>(q, k, v, out, s, cs, lev) : launch_tc<64, true>(q, k, v, out, s, cs, lev);
    else
        st = d == 128 ? launch_f32<128>(q, k, v, out, s, cs, lev) : launch_f32<64>(q, k, v, out, s, cs, lev);
    if (st) return st;
    if (env_debug()) return read_status(cs, 0);
    return MONARCH_OK;
}

int monarch_attn_fwd(const void *q, const void *k, const void *v, void *out, int B, int heads, int T,
                     int H, int W, int d, int factorisation, int tile_h, int tile_w, int dtype,
                     void *stream) {
    LaunchEvents lev;
    return fwd_impl(q, k, v, out, B, heads, T, H, W, d, factorisation, tile_h, tile_w, dtype, stream,
                    lev);
}

int monarch_attn_fwd_strided(const void *q, const void *k, const void *v, void *out, int B, int heads,
                             int T, int H, int W, int d, int factorisation, int tile_h, int tile_w, int dtype,
                             long long stride_b, long long stride_h, long long stride_n, void *stream) {
    if (stride_b < 1 || stride_h < 1 || stride_n < 1) return MONARCH_ERR_INVALID_ARG;
    LaunchEvents lev;
    return fwd_impl(q, k, v, out, B, heads, T, H, W, d, factorisation, tile_h, tile_w, dtype, stream, lev,
                    stride_b, stride_h, stride_n);
}

int monarch_attn_fwd_profiled(const void *q, const void *k, const void *v, void *out, int B, int heads,
                              int T, int H, int W, int d, int factorisation, int tile_h, int tile_w,
                              int dtype, void *stream, void **events, int nevents, int *nlaunch) {
    LaunchEvents lev;
    lev.ev = events;
    lev.n = events ? nevents : 0;
    const int st = fwd_impl(q, k, v, out, B, heads, T, H, W, d, factorisation, tile_h, tile_w, dtype,
                            stream, lev);
    if (nlaunch) *nlaunch = lev.launches;
    return st;
}

int monarch_attn_fwd_host(const void *h_q, const void *h_k, const void *h_v, void *h_out, void *d_q,
                          void *d_k, void *d_v, void *d_out, int B, int heads, int T, int H, int W,
                          int d, int factorisation, int tile_h, int tile_w, int dtype,
                          void *stream) {
    if (!h_q || !h_k || !h_v || !h_out) return MONARCH_ERR_INVALID_ARG;
    Shape s{B, heads, T, H, W, d, factorisation, tile_h, tile_w, dtype, 0, 0};
    int st = validate(d_q, d_k, d_v, d_out, s);
    if (st) return st;
    const size_t bytes = static_cast<size_t>(s.elems) * (dtype == MONARCH_DTYPE_F32 ? 4 : 2);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(d_q, h_q, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d_k, h_k, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d_v, h_v, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    st = monarch_attn_fwd(d_q, d_k, d_v, d_out, B, heads, T, H, W, d, factorisation, tile_h, tile_w,
                          dtype, stream);
    if (st) return st;
    if (cudaMemcpyAsync(h_out, d_out, bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MONARCH_ERR_CUDA;
    return MONARCH_OK;
}

// Same operator as monarch_attn_fwd for bf16, with the completion counters in
// the static device array instead of a cudaMalloc'd per-stream buffer.  It
// serves callers that cannot allocate device memory once running: a real-time
// generation loop, where the first call on a stream (or a larger batch) would
// otherwise cudaMalloc, and a reallocation drains the stream and calls
// cudaFree, which waits for the whole device; and hosts whose device memory
// is all held by their own pool, where a cudaMalloc can fail mid-run.
int monarch_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *out, int B, int heads,
                             int T, int H, int W, int d, int factorisation, int tile_h, int tile_w,
                             void *stream) {
    Shape s{B, heads, T, H, W, d, factorisation, tile_h, tile_w, MONARCH_DTYPE_BF16, 0, 0};
    int st = validate(q, k, v, out, s);
    if (st) return st;
    if (static_cast<long long>(B) * heads > MONARCH_NOALLOC_MAX_BH) return MONARCH_ERR_UNSUPPORTED;
    if (factorisation == MONARCH_FACT_ROW) return MONARCH_ERR_UNSUPPORTED;  // needs the Y1 scratch
    unsigned *counters = nullptr;
    if ((st = noalloc_counters(&counters))) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    LaunchEvents lev;
    st = d == 128 ? launch_tc<128, false>(q, k, v, out, s, cs, lev, counters)
                  : launch_tc<64, false>(q, k, v, out, s, cs, lev, counters);
    if (st) return st;
    if (env_debug()) return read_status(cs, 0);
    return MONARCH_OK;
}

// One chunk of T_new new frames with T_old context frames: stage 1 of the new
// frames into y1_new (the forward's kernels, stage 1 alone), then stage 2 of
// the new queries over [k_cache; k] with values [y1_cache; y1_new].
static int chunk_impl(const void *q, const void *k, const void *v, const void *k_cache, const void *y1_cache,
                      void *out, void *y1_new, int B, int heads, int T_old, int T_new, int H, int W, int d,
                      int factorisation, int tile_h, int tile_w, int dtype, void *stream, LaunchEvents &lev) {
    if (!out || T_old < 0) return MONARCH_ERR_INVALID_ARG;
    if (factorisation == MONARCH_FACT_ROW) return MONARCH_ERR_INVALID_ARG;  // groups are not per position
    if (T_old > 0 && (!k_cache || !y1_cache)) return MONARCH_ERR_INVALID_ARG;
    Shape s{B, heads, T_new, H, W, d, factorisation, tile_h, tile_w, dtype, 0, 0};
    int st = validate(q, k, v, y1_new, s);
    if (st) return st;
    const size_t es = dtype == MONARCH_DTYPE_F32 ? 4 : 2;
    const long long n_old = static_cast<long long>(T_old) * H * W;
    if (n_old > (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    const size_t new_bytes = static_cast<size_t>(s.elems) * es;
    const size_t old_bytes = static_cast<size_t>(B) * heads * n_old * d * es;
    if (reinterpret_cast<uintptr_t>(out) % 16 != 0) return MONARCH_ERR_INVALID_ARG;
    if (T_old > 0) {
        for (const void *c : {k_cache, y1_cache})
            if (reinterpret_cast<uintptr_t>(c) % 16 != 0) return MONARCH_ERR_INVALID_ARG;
        // the outputs may not overlap the context
        for (const void *o : {static_cast<const void *>(out), static_cast<const void *>(y1_new)})
            for (const void *c : {k_cache, y1_cache}) {
                const uintptr_t x = reinterpret_cast<uintptr_t>(o), y = reinterpret_cast<uintptr_t>(c);
                if (x < y + old_bytes && y < x + new_bytes) return MONARCH_ERR_INVALID_ARG;
            }
    }
    for (const void *x : {q, k, v, static_cast<const void *>(y1_new)})
        if (overlaps(out, x, new_bytes)) return MONARCH_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (dtype == MONARCH_DTYPE_BF16) {
        st = d == 128 ? launch_tc<128, false>(q, k, v, y1_new, s, cs, lev, nullptr, true)
                      : launch_tc<64, false>(q, k, v, y1_new, s, cs, lev, nullptr, true);
        if (!st)
            st = d == 128 ? launch_chunk_stage2<128, __nv_bfloat16>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev)
                          : launch_chunk_stage2<64, __nv_bfloat16>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev);
    } else if (dtype == MONARCH_DTYPE_F16) {
        st = d == 128 ? launch_tc<128, true>(q, k, v, y1_new, s, cs, lev, nullptr, true)
                      : launch_tc<64, true>(q, k, v, y1_new, s, cs, lev, nullptr, true);
        if (!st)
            st = d == 128 ? launch_chunk_stage2<128, __half>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev)
                          : launch_chunk_stage2<64, __half>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev);
    } else {
        st = d == 128 ? launch_f32<128>(q, k, v, y1_new, s, cs, lev, true)
                      : launch_f32<64>(q, k, v, y1_new, s, cs, lev, true);
        if (!st)
            st = d == 128 ? launch_chunk_stage2<128, float>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev)
                          : launch_chunk_stage2<64, float>(q, k, k_cache, y1_cache, y1_new, out, s, T_old, cs, lev);
    }
    if (st) return st;
    if (env_debug()) return read_status(cs, 0);
    return MONARCH_OK;
}

int monarch_attn_fwd_chunk(const void *q, const void *k, const void *v, const void *k_cache,
                           const void *y1_cache, void *out, void *y1_new, int B, int heads, int T_old,
                           int T_new, int H, int W, int d, int factorisation, int tile_h, int tile_w,
                           int dtype, void *stream) {
    LaunchEvents lev;
    return chunk_impl(q, k, v, k_cache, y1_cache, out, y1_new, B, heads, T_old, T_new, H, W, d, factorisation,
                      tile_h, tile_w, dtype, stream, lev);
}

int monarch_attn_fwd_chunk_profiled(const void *q, const void *k, const void *v, const void *k_cache,
                                    const void *y1_cache, void *out, void *y1_new, int B, int heads,
                                    int T_old, int T_new, int H, int W, int d, int factorisation,
                                    int tile_h, int tile_w, int dtype, void *stream, void **events,
                                    int nevents, int *nlaunch) {
    LaunchEvents lev;
    lev.ev = events;
    lev.n = events ? nevents : 0;
    const int st = chunk_impl(q, k, v, k_cache, y1_cache, out, y1_new, B, heads, T_old, T_new, H, W, d,
                              factorisation, tile_h, tile_w, dtype, stream, lev);
    if (nlaunch) *nlaunch = lev.launches;
    return st;
}

const char *monarch_attn_strerror(int status) {
    switch (status) {
        case MONARCH_OK: return "success";
        case MONARCH_ERR_INVALID_ARG: return "invalid argument (pointer, size, alignment, aliasing or enum)";
        case MONARCH_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case MONARCH_ERR_LAUNCH: return "kernel launch failed";
        case MONARCH_ERR_TIMEOUT: return "a device-side wait timed out";
        case MONARCH_ERR_CUDA: return "CUDA runtime or driver call failed";
        default: return "unknown status";
    }
}

int monarch_attn_device_status(void *stream, int reset) {
    return read_status(static_cast<cudaStream_t>(stream), reset);
}

int monarch_attn_selftest_timeout(long long limit_cycles, void *stream) {
    if (limit_cycles <= 0) return MONARCH_ERR_INVALID_ARG;
    DeviceInfo *di = nullptr;
    int st = device_info(&di);
    if (st) return st;
    unsigned *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_device_status) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    selftest_timeout_kernel<<<1, 32, 0, cs>>>(limit_cycles, status);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    return read_status(cs, 1);
}

int monarch_attn_version(void) { return 100; }

}  // extern "C"
