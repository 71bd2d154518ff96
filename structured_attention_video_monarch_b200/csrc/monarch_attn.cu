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
#include <list>
#include <mutex>
#include <type_traits>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/monarch_attn.h"
#include "attn_bwd_tc.cuh"
#include "attn_chunk.cuh"
#include "attn_chunk_mma.cuh"
#include "attn_f32.cuh"
#include "attn_tc.cuh"

namespace monarch {

__device__ unsigned g_device_status = 0u;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    int sms = 0;
    bool tc_attr[12] = {};    // [mode][fp16][d == 128]
    int tc_resident[12] = {};  // CTAs of monarch_tc_kernel per SM
    bool f32_attr[2] = {false, false};
};

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

// ------------------------------------------------------------ device buffers
//
// The bf16 / fp16 path needs one 32-bit completion counter per batch-head for
// each call in flight, and the (f*h, w) split a Y1 scratch of N*d elements per
// batch-head.  Both are taken from per-device pools that the library
// allocates on first use and never frees while it is loaded, so their size is
// bounded and a pointer baked into a captured CUDA graph stays valid:
//   counters: kCounterSlots slots of `cap` words (cap >= 4160: one word per
//     batch-head plus the unit-claim counter; doubled when a call has more
//     batch-heads; the old pool is retired, not freed).  A
//     stream keeps its slot while it is among the kCounterSlots most recently
//     used; a stream that takes over a slot first waits (cudaStreamWaitEvent)
//     for the event its previous user recorded after its last launch, so no
//     host synchronisation is needed.  A stream being captured pins its slot.
//   Y1 scratch: one buffer per device, grown geometrically (old buffers
//     retired); calls on different streams are ordered through its event.
// All of this runs under g_buf_mu, held across each launch so that the event
// recorded after a launch is the one the next user of the buffer waits for.
constexpr int kCounterSlots = 64;
constexpr size_t kCounterMinWords = 4160;  // 4096 batch-heads + the claim counter, rounded to 256 bytes

struct CounterSlot {
    cudaStream_t stream = nullptr;
    unsigned long long last = 0;  // LRU tick
    cudaEvent_t done = nullptr;   // recorded after the slot's last launch
    bool used = false;
    bool recorded = false;
    bool pinned = false;          // taken by a stream under capture
};

struct DevicePools {
    unsigned *counters = nullptr;
    size_t cap = 0;  // words per slot
    CounterSlot slot[kCounterSlots];
    unsigned long long tick = 0;
    void *y1 = nullptr;
    size_t y1_cap = 0;
    cudaStream_t y1_stream = nullptr;
    cudaEvent_t y1_done = nullptr;
    bool y1_recorded = false;
    std::vector<void *> retired;  // outgrown buffers (kept: captured graphs may name them)
};

DevicePools g_pools[kMaxDevices];
std::recursive_mutex g_buf_mu;

bool capturing(cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive;
}

// A counter slot of at least n words for (current device, stream), with
// `stream` ordered after the slot's previous user.  Caller holds g_buf_mu and
// calls counters_done() after its launch.
int counters_acquire(cudaStream_t stream, size_t n, unsigned **out, int *slot_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    DevicePools &dp = g_pools[dev];
    if (dp.cap < n) {
        size_t cap = dp.cap ? dp.cap : kCounterMinWords;
        while (cap < n) cap *= 2;
        unsigned *ptr = nullptr;
        if (cudaMalloc(reinterpret_cast<void **>(&ptr), cap * kCounterSlots * sizeof(unsigned)) != cudaSuccess)
            return MONARCH_ERR_CUDA;
        if (dp.counters) dp.retired.push_back(dp.counters);
        dp.counters = ptr;
        dp.cap = cap;
    }
    const bool cap_mode = capturing(stream);
    int pick = -1, lru = -1;
    for (int i = 0; i < kCounterSlots; ++i) {
        const CounterSlot &c = dp.slot[i];
        if (c.used && c.stream == stream) { pick = i; break; }
        if (!c.used) { if (pick < 0) pick = i; continue; }
        if (!c.pinned && (lru < 0 || c.last < dp.slot[lru].last)) lru = i;
    }
    if (pick < 0 || (dp.slot[pick].used && dp.slot[pick].stream != stream)) {
        if (pick < 0) pick = lru;
        if (pick < 0) return MONARCH_ERR_UNSUPPORTED;  // every slot pinned by captures
    }
    CounterSlot &c = dp.slot[pick];
    if (!c.done && cudaEventCreateWithFlags(&c.done, cudaEventDisableTiming) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    if (c.used && c.stream != stream && c.recorded) {
        // a stream under capture cannot wait on work outside the capture
        if (cap_mode) return MONARCH_ERR_UNSUPPORTED;
        if (cudaStreamWaitEvent(stream, c.done, 0) != cudaSuccess) return MONARCH_ERR_CUDA;
    }
    if (!c.used || c.stream != stream) c.recorded = false;
    c.used = true;
    c.stream = stream;
    c.last = ++dp.tick;
    if (cap_mode) c.pinned = true;
    *out = dp.counters + static_cast<size_t>(pick) * dp.cap;
    *slot_out = pick;
    return MONARCH_OK;
}

int counters_done(cudaStream_t stream, int slot) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    CounterSlot &c = g_pools[dev].slot[slot];
    if (c.pinned) return MONARCH_OK;  // captured: never handed to another stream
    if (cudaEventRecord(c.done, stream) != cudaSuccess) return MONARCH_ERR_CUDA;
    c.recorded = true;
    return MONARCH_OK;
}

// The device's Y1 scratch, at least `bytes` long, with `stream` ordered after
// its previous user.  Caller holds g_buf_mu and calls scratch_done() after
// its launches.
int scratch_acquire(cudaStream_t stream, size_t bytes, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    DevicePools &dp = g_pools[dev];
    if (dp.y1_cap < bytes) {
        size_t cap = dp.y1_cap ? dp.y1_cap : (size_t(1) << 20);
        while (cap < bytes) cap *= 2;
        void *ptr = nullptr;
        if (cudaMalloc(&ptr, cap) != cudaSuccess) return MONARCH_ERR_CUDA;
        if (dp.y1) dp.retired.push_back(dp.y1);
        dp.y1 = ptr;
        dp.y1_cap = cap;
        dp.y1_recorded = false;  // fresh memory: no earlier user
    }
    if (!dp.y1_done && cudaEventCreateWithFlags(&dp.y1_done, cudaEventDisableTiming) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    if (dp.y1_recorded && dp.y1_stream != stream) {
        if (capturing(stream)) return MONARCH_ERR_UNSUPPORTED;
        if (cudaStreamWaitEvent(stream, dp.y1_done, 0) != cudaSuccess) return MONARCH_ERR_CUDA;
    }
    dp.y1_stream = stream;
    *out = dp.y1;
    return MONARCH_OK;
}

int scratch_done(cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    DevicePools &dp = g_pools[dev];
    if (capturing(stream)) {
        dp.y1_recorded = false;
        return MONARCH_OK;
    }
    if (cudaEventRecord(dp.y1_done, stream) != cudaSuccess) return MONARCH_ERR_CUDA;
    dp.y1_recorded = true;
    return MONARCH_OK;
}

// Completion counters for monarch_attn_fwd_noalloc: a file-scope device array
// (4096 + 1 words, about 16 KB: one per batch-head and the unit-claim
// counter) in place of the pooled cudaMalloc buffers above.  Its
// device address is looked up on every call (with the caller's device
// current): the lookup allocates nothing and stays right after a device reset
// gives the module a new context.  One array per device means calls of that
// entry point on one device must not overlap in time.
static __device__ __align__(256) unsigned g_noalloc_counters[MONARCH_NOALLOC_MAX_BH + 1];

int noalloc_counters(unsigned **out) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_counters) != cudaSuccess || ptr == nullptr)
        return MONARCH_ERR_CUDA;
    *out = static_cast<unsigned *>(ptr);
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
// Host-side cache of encoded tensor maps, keyed by everything the encoding
// reads (address, type, rank, dims, strides, box), least recently used first
// out.  A map holds no reference to the memory, so a key that matches is the
// same map even if the buffer was freed and reallocated at that address.
struct MapKey {
    uint64_t ptr;
    uint32_t dtype, rank;
    cuuint64_t dims[5];
    cuuint64_t strides[4];
    cuuint32_t box[5];
    bool operator==(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
    size_t operator()(const MapKey &k) const {
        const unsigned char *b = reinterpret_cast<const unsigned char *>(&k);
        uint64_t h = 1469598103934665603ull;  // FNV-1a
        for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ b[i]) * 1099511628211ull;
        return static_cast<size_t>(h);
    }
};
constexpr size_t kMapCacheEntries = 1024;
std::list<std::pair<MapKey, CUtensorMap>> g_map_lru;  // front = most recent
std::unordered_map<MapKey, std::list<std::pair<MapKey, CUtensorMap>>::iterator, MapKeyHash> g_map_index;
std::mutex g_map_mu;

// 16-bit (bf16 or fp16) tensor map with 128-byte swizzle; dims/strides
// innermost first, strides in bytes for dims 1..rank-1.
int make_map(CUtensorMap *map, const void *ptr, int rank, const cuuint64_t *dims,
             const cuuint64_t *strides, const cuuint32_t *box, int dtype) {
    MapKey key;
    std::memset(&key, 0, sizeof(key));  // padding takes part in the hash
    key.ptr = reinterpret_cast<uint64_t>(ptr);
    key.dtype = static_cast<uint32_t>(dtype);
    key.rank = static_cast<uint32_t>(rank);
    for (int i = 0; i < rank; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
    for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides[i];
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        auto it = g_map_index.find(key);
        if (it != g_map_index.end()) {
            g_map_lru.splice(g_map_lru.begin(), g_map_lru, it->second);
            *map = it->second->second;
            return MONARCH_OK;
        }
    }
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType ty =
        dtype == MONARCH_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = g_encode(map, ty, rank, const_cast<void *>(ptr), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return MONARCH_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_map_index.find(key) == g_map_index.end()) {
        g_map_lru.emplace_front(key, *map);
        g_map_index[key] = g_map_lru.begin();
        if (g_map_lru.size() > kMapCacheEntries) {
            g_map_index.erase(g_map_lru.back().first);
            g_map_lru.pop_back();
        }
    }
    return MONARCH_OK;
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
              bool stage1_only = false, int sub = 0, float *lse = nullptr,
              int lse_kind = UNIT_STAGE1, bool stage2_only = false) {
    DeviceInfo *di = nullptr;
    int st = device_info(&di);
    if (st) return st;
    if ((st = get_encode())) return st;
    using L = TcLayout<D>;
    const int mode = lse != nullptr ? TC_LSE : (sub > 0 ? TC_PACK : TC_PLAIN);
    if (lse != nullptr && sub > 0) return MONARCH_ERR_UNSUPPORTED;
    const int di_idx = mode * 4 + (F16 ? 2 : 0) + (D == 128 ? 1 : 0);
    const auto kernel = mode == TC_LSE ? monarch_tc_kernel<D, F16, TC_LSE>
                                       : (mode == TC_PACK ? monarch_tc_kernel<D, F16, TC_PACK>
                                                          : monarch_tc_kernel<D, F16, TC_PLAIN>);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!di->tc_attr[di_idx]) {
            int occ = 0;
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     L::ALLOC) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, 640, L::ALLOC) !=
                    cudaSuccess)
                return MONARCH_ERR_CUDA;
            if (occ < 1) return MONARCH_ERR_UNSUPPORTED;
            di->tc_resident[di_idx] = occ;
            di->tc_attr[di_idx] = true;
        }
    }
    TcParams p{};
    p.B = s.B; p.heads = s.heads; p.T = s.T; p.H = s.H; p.W = s.W; p.HW = s.H * s.W;
    p.N = s.N;
    p.fact = s.fact;
    p.sub = sub;
    p.lse = lse;
    p.lse_kind = lse_kind;
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
    // stage 2 alone: no stage-1 units; the values (Y1) are `v`, the result goes to `out`
    if (stage2_only) p.u1_bh = 0;
    const long long units = bh * (p.u1_bh + p.s2_pairs);
    if (units >= (1ll << 31) - 1) return MONARCH_ERR_UNSUPPORTED;
    p.units = static_cast<int>(units);
    p.s1_target = stage2_only ? 0u : static_cast<unsigned>(p.nblk_bh) * static_cast<unsigned>(p.nqt);
    // Stage-2 units of a batch-head trail its stage-1 units by about sixteen
    // waves of the persistent grid (for the full clip: after every stage-1
    // unit), so they never wait on their inputs and the CTAs run long stretches
    // of one unit kind; a lag of two waves measured 3 % slower on the full clip.
    {
        const long long wave = di->sms;
        long long lag = p.u1_bh > 0 ? (16 * wave + p.u1_bh - 1) / p.u1_bh : 1;
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
               (st = stage2_map(&my2, stage2_only ? v : out, s, p))) {
        return st;
    }

    // One persistent launch runs both stages: stage-1 units write Y1 = B1 V
    // into out; stage-2 units overwrite it in place with P^T B2 P Y1 once the
    // stage-1 lanes of their batch-head have published (per-batch-head
    // counters, zeroed for every call).  Stage-2 units wait for other CTAs,
    // so the launch is cooperative: the driver makes every CTA of the grid
    // resident at once, or refuses the launch (MONARCH_ERR_LAUNCH), rather
    // than leaving resident CTAs waiting for ones that cannot start.
    std::unique_lock<std::recursive_mutex> lk(g_buf_mu, std::defer_lock);
    unsigned *counters = fixed_counters;
    int slot = -1;
    if (!counters) {
        lk.lock();
        if ((st = counters_acquire(stream, static_cast<size_t>(bh) + 1, &counters, &slot))) return st;
    }
    // counters[0, bh): stage-1 lanes published per batch-head; counters[bh]:
    // the next unit to claim (CTAs take units in order as they free up)
    p.s1_done = counters;
    p.work = counters + bh;
    if (cudaMemsetAsync(counters, 0, (static_cast<size_t>(bh) + 1) * sizeof(unsigned), stream) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    const int resident = di->sms * di->tc_resident[di_idx];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.units < resident ? p.units : resident));
    cfg.blockDim = dim3(640);
    cfg.dynamicSmemBytes = L::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    lev.start(stream);
    if (cudaLaunchKernelEx(&cfg, kernel, mq1, mk1, mv1, mq2, mk2, my2, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return MONARCH_ERR_LAUNCH;
    }
    lev.record(++lev.launches, stream);
    if (slot >= 0) return counters_done(stream, slot);
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
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!di->f32_attr[di_idx]) {
            if (cudaFuncSetAttribute(monarch_f32_stage2<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     2 * 128 * D * 4) != cudaSuccess)
                return MONARCH_ERR_CUDA;
            di->f32_attr[di_idx] = true;
        }
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
    std::lock_guard<std::recursive_mutex> lk(g_buf_mu);
    void *y1 = nullptr;
    int st = scratch_acquire(stream, static_cast<size_t>(s.elems) * sizeof(E), &y1);
    if (st) return st;
    Shape rows = s;
    rows.T = s.T * s.H; rows.H = 1; rows.fact = MONARCH_FACT_FRAME; rows.tile_h = rows.tile_w = 0;
    // The tensor-core rows pass packs `pack` consecutive frame rows into one
    // block of pack * W <= 128 tokens (a query tile), each row attending to its
    // own keys only (sub-blocks of W): short rows then fill the 128-row MMA
    // tiles instead of leaving most of each empty.  Y1 keeps its layout.
    int pack = 1;
    for (int c = 128 / s.W; c > 1; --c)
        if ((s.T * s.H) % c == 0) { pack = c; break; }
    Shape cols = s;
    cols.T = 1; cols.H = s.T * s.H; cols.fact = MONARCH_FACT_TILED; cols.tile_h = s.T * s.H; cols.tile_w = 1;
    constexpr bool tc = !std::is_same<E, float>::value;
    if constexpr (tc) {
        constexpr bool f16 = std::is_same<E, __half>::value;
        Shape packed = rows;
        packed.T = rows.T / pack; packed.H = pack;
        if ((st = launch_tc<D, f16>(q, k, v, y1, pack > 1 ? packed : rows, stream, lev, nullptr, true,
                                    pack > 1 ? s.W : 0)))
            return st;
        st = launch_tc<D, f16>(q, k, y1, out, cols, stream, lev, nullptr, true);
    } else {
        if ((st = launch_f32<D>(q, k, v, y1, rows, stream, lev, true))) return st;
        st = launch_f32<D>(q, k, y1, out, cols, stream, lev, true);
    }
    if (st) return st;
    return scratch_done(stream);
}


// <bwd-launch> (hashed with attn_bwd_tc.cuh by the profile summaries)
// ---------------------------------------------------------------- gradients
// bf16 / fp16 gradients on tensor cores (attn_bwd_tc.cuh), orchestrated here
// beside the forward's launch code, whose kernels recompute Y1 and O.

// D[row] = sum_c a[row][c] * b[row][c] over 16-bit rows: one warp per row.
template <int D, typename E>
__global__ void bwd_rowdot(const E *a, const E *b, float *out, long long rows) {
    const long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    float s = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) {
        float x, y;
        if constexpr (std::is_same<E, __half>::value) {
            x = __half2float(a[r * D + c]);
            y = __half2float(b[r * D + c]);
        } else {
            x = __bfloat162float(a[r * D + c]);
            y = __bfloat162float(b[r * D + c]);
        }
        s = fmaf(x, y, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) out[r] = s;
}

// Workspace (bytes): Y1, O, dY1 (16-bit, N*d each), stage 2's LSE and the
// row sums D (fp32, N each), stage 2's dq and dk parts (fp32, N*d each) and
// stage 1's LSE (fp32, N); per batch-head.
size_t bwd_tc_workspace(long long bh, long long N, int d, int es) {
    return static_cast<size_t>(bh * N) * (3 * d * es + 3 * 4 + 2 * d * 4);
}

// Geometry of one stage from a (possibly virtual) frame or tiled shape, and the
// forward's map parameters for the same shape.
void bwd_geometry(const Shape &s, int D, BwdParams &p, TcParams &tp) {
    p.B = s.B; p.heads = s.heads; p.T = s.T; p.H = s.H; p.W = s.W; p.HW = s.H * s.W; p.N = s.N;
    if (s.fact == MONARCH_FACT_TILED) {
        p.tile_h = s.tile_h; p.tile_w = s.tile_w; p.tiles_h = s.H / s.tile_h; p.tiles_w = s.W / s.tile_w;
        const int r = 128 / s.tile_w;
        p.rows_per_tile = r < s.tile_h ? r : s.tile_h;
        p.m = s.tile_h * s.tile_w;
        p.nblk_bh = s.T * p.tiles_h * p.tiles_w;
        p.ntile = (s.tile_h + p.rows_per_tile - 1) / p.rows_per_tile;
    } else {
        p.m = p.HW; p.nblk_bh = s.T; p.ntile = (p.m + 127) / 128;
    }
    p.npos = s.T <= 128 ? 128 / s.T : 1;
    p.s2_chunks = (p.HW + p.npos - 1) / p.npos;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    tp = TcParams{};
    tp.m = p.m; tp.HW = p.HW; tp.npos = p.npos;
    tp.tiles_h = p.tiles_h; tp.tiles_w = p.tiles_w; tp.rows_per_tile = p.rows_per_tile;
}

// The dq then the dk/dv kernel of one stage.  Maps: q, k, values, upstream
// gradient, all in the geometry KIND.
template <int D, bool F16, int KIND>
int bwd_run_stage(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mvals, const CUtensorMap &mdy,
                  const BwdParams &p, long long bh, cudaStream_t stream) {
    using LB = BwdLayout<D>;
    static bool attr_done[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_done[dev]) {
            if (cudaFuncSetAttribute(monarch_bwd_dq<D, F16, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LB::ALLOC) != cudaSuccess ||
                cudaFuncSetAttribute(monarch_bwd_dkdv<D, F16, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LB::ALLOC) != cudaSuccess ||
                cudaFuncSetAttribute(monarch_bwd_pair<D, F16, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LB::ALLOC) != cudaSuccess)
                return MONARCH_ERR_CUDA;
            attr_done[dev] = true;
        }
    }
    const long long per_bh = (KIND == BWD_GEOM_STAGE2 ? p.s2_chunks : p.nblk_bh) *
                             static_cast<long long>(KIND == BWD_GEOM_STAGE2 ? 1 : p.ntile);
    if (bh * per_bh >= (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    const unsigned grid = static_cast<unsigned>(bh * per_bh);
    if (p.lse_given) {  // dq and dk/dv CTAs in one launch
        if (2ll * grid >= (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
        BwdParams pp = p;
        pp.pair_split = static_cast<int>(grid);
        monarch_bwd_pair<D, F16, KIND><<<2 * grid, LB::THREADS, LB::ALLOC, stream>>>(mq, mk, mvals, mdy, pp);
        return cudaGetLastError() == cudaSuccess ? MONARCH_OK : MONARCH_ERR_LAUNCH;
    }
    monarch_bwd_dq<D, F16, KIND><<<grid, LB::THREADS, LB::ALLOC, stream>>>(mq, mk, mvals, mdy, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    monarch_bwd_dkdv<D, F16, KIND><<<grid, LB::THREADS, LB::ALLOC, stream>>>(mq, mk, mvals, mdy, p);
    return cudaGetLastError() == cudaSuccess ? MONARCH_OK : MONARCH_ERR_LAUNCH;
}

template <int D, bool F16>
int launch_bwd_tc(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk, void *dv,
                  void *ws, const Shape &s, cudaStream_t stream, LaunchEvents &lev) {
    using E = typename std::conditional<F16, __half, __nv_bfloat16>::type;
    DeviceInfo *di = nullptr;
    int st = device_info(&di);
    if (st) return st;
    if ((st = get_encode())) return st;
    const long long bh = static_cast<long long>(s.B) * s.heads, N = s.N, nd = bh * N * D;
    uint8_t *w = static_cast<uint8_t *>(ws);
    E *y1 = reinterpret_cast<E *>(w);
    E *o = y1 + nd;
    E *dy1 = o + nd;
    float *lse = reinterpret_cast<float *>(dy1 + nd);
    float *dd = lse + bh * N;
    float *dq32 = dd + bh * N;
    float *dk32 = dq32 + nd;
    float *lse1 = dk32 + nd;
    const bool row = s.fact == MONARCH_FACT_ROW;
    // the two stages' shapes: the (f*h, w) split runs both as stage-1
    // geometries of virtual shapes (rows: one-row frames; columns: one tall
    // frame cut into one-column tiles)
    Shape s1 = s, s2 = s;
    if (row) {
        s1.T = s.T * s.H; s1.H = 1; s1.fact = MONARCH_FACT_FRAME; s1.tile_h = s1.tile_w = 0;
        s2.T = 1; s2.H = s.T * s.H; s2.fact = MONARCH_FACT_TILED; s2.tile_h = s.T * s.H; s2.tile_w = 1;
    }
    // recompute Y1 (stage 1 alone) and O (stage 2 alone over that Y1; for the
    // (f*h, w) split the columns pass over Y1); they also leave each stage's row LSE
    // (stage 1's in lse1, stage 2's in lse), so the dQ kernels skip their LSE pass
    if ((st = launch_tc<D, F16>(q, k, v, y1, s1, stream, lev, nullptr, true, 0, lse1, UNIT_STAGE1))) return st;
    if (row) {
        if ((st = launch_tc<D, F16>(q, k, y1, o, s2, stream, lev, nullptr, true, 0, lse, UNIT_STAGE1))) return st;
    } else if ((st = launch_tc<D, F16>(q, k, y1, o, s, stream, lev, nullptr, false, 0, lse, UNIT_STAGE2, true))) {
        return st;
    }
    unsigned *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_device_status) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    const long long rows = bh * N;
    const unsigned rd_grid = static_cast<unsigned>((rows + 7) / 8);
    // stage 2: values Y1, upstream dO, output O; its value gradient is dY1 (16-bit)
    {
        BwdParams p{};
        TcParams tp{};
        bwd_geometry(s2, D, p, tp);
        p.lse = lse; p.lse_given = 1;
        p.D = dd; p.dq = dq32; p.add_dq = 0; p.dk = dk32; p.add_dk = 0; p.dv16 = dy1;
        p.timeout_cycles = env_timeout_cycles();
        p.status = status;
        bwd_rowdot<D, E><<<rd_grid, 256, 0, stream>>>(static_cast<const E *>(dout), o, dd, rows);
        if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
        CUtensorMap mq, mk, my, mdo;
        if (row) {
            if ((st = stage1_map(&mq, q, s2, tp)) || (st = stage1_map(&mk, k, s2, tp)) ||
                (st = stage1_map(&my, y1, s2, tp)) || (st = stage1_map(&mdo, dout, s2, tp)))
                return st;
            st = bwd_run_stage<D, F16, BWD_GEOM_TILED>(mq, mk, my, mdo, p, bh, stream);
        } else {
            if ((st = stage2_map(&mq, q, s2, tp)) || (st = stage2_map(&mk, k, s2, tp)) ||
                (st = stage2_map(&my, y1, s2, tp)) || (st = stage2_map(&mdo, dout, s2, tp)))
                return st;
            st = bwd_run_stage<D, F16, BWD_GEOM_STAGE2>(mq, mk, my, mdo, p, bh, stream);
        }
        if (st) return st;
        lev.record(++lev.launches, stream);
    }
    // stage 1: values V, upstream dY1, output Y1
    {
        BwdParams p{};
        TcParams tp{};
        bwd_geometry(s1, D, p, tp);
        // adds stage 2's fp32 parts and writes the final 16-bit gradients
        p.lse = lse1; p.lse_given = 1;
        p.D = dd; p.dq = dq32; p.add_dq = 1; p.dk = dk32; p.add_dk = 1; p.dv16 = dv;
        p.out_dq = dq; p.out_dk = dk;
        p.timeout_cycles = env_timeout_cycles();
        p.status = status;
        bwd_rowdot<D, E><<<rd_grid, 256, 0, stream>>>(dy1, y1, dd, rows);
        if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
        CUtensorMap mq, mk, mv, mdy;
        if ((st = stage1_map(&mq, q, s1, tp)) || (st = stage1_map(&mk, k, s1, tp)) ||
            (st = stage1_map(&mv, v, s1, tp)) || (st = stage1_map(&mdy, dy1, s1, tp)))
            return st;
        st = s1.fact == MONARCH_FACT_TILED ? bwd_run_stage<D, F16, BWD_GEOM_TILED>(mq, mk, mv, mdy, p, bh, stream)
                                           : bwd_run_stage<D, F16, BWD_GEOM_FRAME>(mq, mk, mv, mdy, p, bh, stream);
        if (st) return st;
        lev.record(++lev.launches, stream);
    }
    return MONARCH_OK;
}

// </bwd-launch>

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
    if constexpr (!std::is_same<E, float>::value) {
        // 16-bit inputs: warp-level MMAs for the logits and the weighted sum of Y1
        // (attn_chunk_mma.cuh); fp32 keeps the CUDA-core kernel
        using M = ChunkMmaCfg<D, E>;
        ChunkMmaParams mp{p.HW, p.T_old, p.T_new, p.n_old, p.n_new, p.groups, p.scale_log2,
                          p.T_new < M::QM ? p.T_new : M::QM,
                          p.T_old + p.T_new < M::KC ? p.T_old + p.T_new : M::KC};
        const int smem = M::smem_bytes(mp.qrows, mp.krows);
        if (smem > 227 * 1024) return MONARCH_ERR_UNSUPPORTED;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(monarch_chunk_stage2_mma<D, E>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
            return MONARCH_ERR_CUDA;
        const long long blocks = (p.groups + M::WARPS - 1) / M::WARPS;
        monarch_chunk_stage2_mma<D, E><<<static_cast<unsigned>(blocks), 32 * M::WARPS, smem, stream>>>(
            static_cast<const E *>(q), static_cast<const E *>(k), static_cast<const E *>(k_cache),
            static_cast<const E *>(y1_cache), static_cast<const E *>(y1_new), static_cast<E *>(out), mp);
        if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
        lev.record(++lev.launches, stream);
        return MONARCH_OK;
    }
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

// The 16-bit gradients (monarch_attn_bwd in monarch_bwd.cu calls these).
size_t bwd_tc_workspace_bytes(long long bh, long long N, int d, int es) { return bwd_tc_workspace(bh, N, d, es); }

int bwd_tc_run(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk, void *dv, void *ws,
               int B, int heads, int T, int H, int W, int d, int fact, int tile_h, int tile_w, int dtype,
               cudaStream_t stream, void **events, int nevents, int *nlaunch) {
    Shape s{B, heads, T, H, W, d, fact, tile_h, tile_w, dtype, 0, 0};
    int st = validate(q, k, v, dq, s);
    if (st) return st;
    LaunchEvents lev;
    lev.ev = events;
    lev.n = events ? nevents : 0;
    if (dtype == MONARCH_DTYPE_F16)
        st = d == 128 ? launch_bwd_tc<128, true>(q, k, v, dout, dq, dk, dv, ws, s, stream, lev)
                      : launch_bwd_tc<64, true>(q, k, v, dout, dq, dk, dv, ws, s, stream, lev);
    else
        st = d == 128 ? launch_bwd_tc<128, false>(q, k, v, dout, dq, dk, dv, ws, s, stream, lev)
                      : launch_bwd_tc<64, false>(q, k, v, dout, dq, dk, dv, ws, s, stream, lev);
    if (nlaunch) *nlaunch = lev.launches;
    if (st) return st;
    if (env_debug()) return read_status(stream, 0);
    return MONARCH_OK;
}

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
