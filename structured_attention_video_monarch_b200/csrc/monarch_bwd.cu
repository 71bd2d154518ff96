// monarch_bwd.cu -- C ABI of the Monarch attention gradients (fp32 path):
// argument checks, the forward stage-1 recomputation of Y1 into the caller's
// workspace, and the two backward launches (include/monarch_attn.h).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <initializer_list>

#include "../../include/monarch_attn.h"
#include "attn_bwd_f32.cuh"

using namespace monarch;

namespace monarch {
// The 16-bit path lives beside the forward's launch code (monarch_attn.cu).
size_t bwd_tc_workspace_bytes(long long bh, long long N, int d, int es);
int bwd_tc_run(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk, void *dv, void *ws,
               int B, int heads, int T, int H, int W, int d, int fact, int tile_h, int tile_w, int dtype,
               cudaStream_t stream, void **events, int nevents, int *nlaunch);
}  // namespace monarch

namespace {

// [a, a + na) and [b, b + nb) share a byte
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Shared-memory bytes the stage-1 backward needs: 4 warps x (p, dp) x m floats.
size_t stage1_smem(long long m) { return static_cast<size_t>(4 * 2 * m) * sizeof(float); }
constexpr size_t kMaxStage1Smem = 200 * 1024;

template <int D>
int launch_bwd(const float *q, const float *k, const float *v, const float *dout, float *dq, float *dk,
               float *dv, float *y1, float *dy1, int B, int heads, int T, int H, int W, int fact, int tile_h,
               int tile_w, cudaStream_t stream) {
    F32Params p{};
    p.T = T; p.H = H; p.W = W; p.HW = H * W; p.N = static_cast<long long>(T) * H * W;
    p.fact = fact;
    if (fact == MONARCH_FACT_TILED) {
        p.tile_h = tile_h; p.tile_w = tile_w;
        p.tiles_h = H / tile_h; p.tiles_w = W / tile_w;
        p.m = tile_h * tile_w;
        p.nblk_bh = T * p.tiles_h * p.tiles_w;
    } else {
        p.m = p.HW;
        p.nblk_bh = T;
    }
    p.qchunks = (p.m + 63) / 64;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    p.heads = heads;
    p.sN = D;
    p.sH = p.N * D;
    p.sB = static_cast<long long>(heads) * p.N * D;
    const long long bh = static_cast<long long>(B) * heads;
    const size_t bytes = static_cast<size_t>(bh * p.N * D) * sizeof(float);
    const int qgroups = (p.m + 3) / 4;
    const long long g1 = bh * p.nblk_bh * p.qchunks, g2 = bh * p.HW, g3 = bh * p.nblk_bh * qgroups;
    if (g1 >= (1ll << 31) || g2 >= (1ll << 31) || g3 >= (1ll << 31)) return MONARCH_ERR_UNSUPPORTED;
    const size_t smem3 = stage1_smem(p.m);
    if (smem3 > kMaxStage1Smem) return MONARCH_ERR_UNSUPPORTED;
    if (smem3 > 48 * 1024 &&
        cudaFuncSetAttribute(monarch_f32_bwd_stage1<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem3)) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    if (cudaMemsetAsync(dk, 0, bytes, stream) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, stream) != cudaSuccess ||
        cudaMemsetAsync(dy1, 0, bytes, stream) != cudaSuccess)
        return MONARCH_ERR_CUDA;
    // Y1 = B1 V, recomputed by the forward's fp32 stage-1 kernel
    monarch_f32_stage1<D><<<static_cast<unsigned>(g1), 128, 0, stream>>>(q, k, v, y1, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    monarch_f32_bwd_stage2<D><<<static_cast<unsigned>(g2), 128, 0, stream>>>(q, k, y1, dout, dq, dk, dy1, p);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    monarch_f32_bwd_stage1<D><<<static_cast<unsigned>(g3), 128, smem3, stream>>>(q, k, v, dy1, dq, dk, dv, p,
                                                                                  qgroups);
    if (cudaGetLastError() != cudaSuccess) return MONARCH_ERR_LAUNCH;
    return MONARCH_OK;
}

}  // namespace

extern "C" {

size_t monarch_attn_bwd_workspace_size(int B, int heads, int T, int H, int W, int d, int dtype) {
    if (B < 1 || heads < 1 || T < 1 || H < 1 || W < 1 || (d != 64 && d != 128)) return 0;
    if (dtype == MONARCH_DTYPE_BF16 || dtype == MONARCH_DTYPE_F16)
        return bwd_tc_workspace_bytes(static_cast<long long>(B) * heads, static_cast<long long>(T) * H * W, d, 2);
    if (dtype != MONARCH_DTYPE_F32) return 0;
    return 2 * static_cast<size_t>(B) * heads * T * H * W * d * sizeof(float);
}

static int bwd_impl(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk, void *dv,
                    void *workspace, size_t workspace_bytes, int B, int heads, int T, int H, int W, int d,
                    int factorisation, int tile_h, int tile_w, int dtype, void *stream, void **events, int nevents,
                    int *nlaunch) {
    if (nlaunch) *nlaunch = 0;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !workspace) return MONARCH_ERR_INVALID_ARG;
    if (B < 1 || heads < 1 || T < 1 || H < 1 || W < 1) return MONARCH_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MONARCH_ERR_INVALID_ARG;
    if (dtype != MONARCH_DTYPE_F32 && dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F16)
        return MONARCH_ERR_INVALID_ARG;
    const bool half = dtype == MONARCH_DTYPE_BF16 || dtype == MONARCH_DTYPE_F16;
    // the (f*h, w) split has gradients on the tensor-core path only
    if (factorisation != MONARCH_FACT_FRAME && factorisation != MONARCH_FACT_TILED &&
        !(half && factorisation == MONARCH_FACT_ROW))
        return MONARCH_ERR_INVALID_ARG;
    if (factorisation == MONARCH_FACT_TILED &&
        (tile_h < 1 || tile_w < 1 || H % tile_h != 0 || W % tile_w != 0))
        return MONARCH_ERR_INVALID_ARG;
    if (half) {
        // tensor cores: outputs and workspace may not overlap the inputs or each other
        const size_t need = monarch_attn_bwd_workspace_size(B, heads, T, H, W, d, dtype);
        if (need == 0 || workspace_bytes < need) return MONARCH_ERR_INVALID_ARG;
        const size_t bytes = static_cast<size_t>(B) * heads * T * H * W * d * 2;
        for (const void *p : {q, k, v, dout, static_cast<const void *>(dq), static_cast<const void *>(dk),
                              static_cast<const void *>(dv), static_cast<const void *>(workspace)})
            if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return MONARCH_ERR_INVALID_ARG;
        const void *outs[4] = {dq, dk, dv, workspace};
        const size_t out_bytes[4] = {bytes, bytes, bytes, need};
        const void *ins[4] = {q, k, v, dout};
        for (int a = 0; a < 4; ++a) {
            for (int b = 0; b < 4; ++b)
                if (overlap(outs[a], out_bytes[a], ins[b], bytes)) return MONARCH_ERR_INVALID_ARG;
            for (int b = a + 1; b < 4; ++b)
                if (overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return MONARCH_ERR_INVALID_ARG;
        }
        return bwd_tc_run(q, k, v, dout, dq, dk, dv, workspace, B, heads, T, H, W, d, factorisation, tile_h, tile_w,
                          dtype, static_cast<cudaStream_t>(stream), events, nevents, nlaunch);
    }
    if (T > 128) return MONARCH_ERR_UNSUPPORTED;
    const long long N = static_cast<long long>(T) * H * W;
    if (N > (1ll << 31) || static_cast<long long>(B) * heads > (1ll << 30)) return MONARCH_ERR_UNSUPPORTED;
    const size_t need = monarch_attn_bwd_workspace_size(B, heads, T, H, W, d, dtype);
    if (workspace_bytes < need) return MONARCH_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, dout, static_cast<const void *>(dq), static_cast<const void *>(dk),
                          static_cast<const void *>(dv), static_cast<const void *>(workspace)})
        if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return MONARCH_ERR_INVALID_ARG;
    const size_t bytes = need / 2;
    // outputs and workspace may not overlap the inputs or each other
    const void *outs[4] = {dq, dk, dv, workspace};
    const size_t out_bytes[4] = {bytes, bytes, bytes, need};
    const void *ins[4] = {q, k, v, dout};
    for (int a = 0; a < 4; ++a) {
        for (int b = 0; b < 4; ++b)
            if (overlap(outs[a], out_bytes[a], ins[b], bytes)) return MONARCH_ERR_INVALID_ARG;
        for (int b = a + 1; b < 4; ++b)
            if (overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return MONARCH_ERR_INVALID_ARG;
    }
    float *y1 = static_cast<float *>(workspace);
    float *dy1 = y1 + bytes / sizeof(float);
    const float *fq = static_cast<const float *>(q), *fk = static_cast<const float *>(k),
                *fv = static_cast<const float *>(v), *fdo = static_cast<const float *>(dout);
    float *fdq = static_cast<float *>(dq), *fdk = static_cast<float *>(dk), *fdv = static_cast<float *>(dv);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (events && nevents > 0 && events[0]) cudaEventRecord(static_cast<cudaEvent_t>(events[0]), cs);
    const int st = d == 128 ? launch_bwd<128>(fq, fk, fv, fdo, fdq, fdk, fdv, y1, dy1, B, heads, T, H, W,
                                              factorisation, tile_h, tile_w, cs)
                            : launch_bwd<64>(fq, fk, fv, fdo, fdq, fdk, fdv, y1, dy1, B, heads, T, H, W,
                                             factorisation, tile_h, tile_w, cs);
    if (st) return st;
    if (events && nevents > 1 && events[1]) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), cs);
    if (nlaunch) *nlaunch = 1;
    return MONARCH_OK;
}

int monarch_attn_bwd(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                     void *dv, void *workspace, size_t workspace_bytes, int B, int heads, int T, int H,
                     int W, int d, int factorisation, int tile_h, int tile_w, int dtype, void *stream) {
    return bwd_impl(q, k, v, dout, dq, dk, dv, workspace, workspace_bytes, B, heads, T, H, W, d, factorisation,
                    tile_h, tile_w, dtype, stream, nullptr, 0, nullptr);
}

int monarch_attn_bwd_profiled(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                              void *dv, void *workspace, size_t workspace_bytes, int B, int heads, int T, int H,
                              int W, int d, int factorisation, int tile_h, int tile_w, int dtype, void *stream,
                              void **events, int nevents, int *nlaunch) {
    return bwd_impl(q, k, v, dout, dq, dk, dv, workspace, workspace_bytes, B, heads, T, H, W, d, factorisation,
                    tile_h, tile_w, dtype, stream, events, nevents, nlaunch);
}

}  // extern "C"
