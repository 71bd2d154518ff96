// attn_f32.cuh -- fp32 Monarch attention stages on CUDA cores.
//
// The exact path for fp32 inputs: the same operator as the tensor-core path
// (stage 1 softmax attention inside each frame or spatial tile, stage 2
// softmax attention across frames at each position with the stage-1 outputs
// as values; MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/nl/paper/2602.12271 "Methodologie"), in fp32 FFMA with an
// online softmax and expf, so results stay within 1e-5 of the fp64 definition.
// Stage 2 runs in place on `out`: each block copies its group's stage-1 rows
// to shared memory before any thread writes that group's outputs.
#pragma once

#include <cstdint>

namespace monarch {

struct F32Params {
    int T, H, W, HW;
    long long N;
    int fact, tile_h, tile_w, tiles_h, tiles_w;
    int m;          // tokens per stage-1 block
    int nblk_bh;    // stage-1 blocks per (batch, head)
    int qchunks;    // 64-query chunks per stage-1 block
    float scale;
    int heads;
    long long sB, sH, sN;  // element strides of batch, head and token (all four tensors)
};

// Element offset of token n's row of batch-head bh.
__device__ __forceinline__ long long f32_row(const F32Params &p, long long bh, long long n) {
    const long long b = bh / p.heads;
    return b * p.sB + (bh - b * p.heads) * p.sH + n * p.sN;
}

__device__ __forceinline__ long long f32_s1_token(const F32Params &p, int b, int i) {
    if (p.fact == 0) return static_cast<long long>(b) * p.HW + i;
    const int tpf = p.tiles_h * p.tiles_w;
    const int t = b / tpf, tif = b % tpf;
    const int ti = tif / p.tiles_w, tj = tif % p.tiles_w;
    const int hl = i / p.tile_w, wl = i % p.tile_w;
    return static_cast<long long>(t) * p.HW + static_cast<long long>(ti * p.tile_h + hl) * p.W +
           tj * p.tile_w + wl;
}

// One block = 64 queries of one stage-1 block; two threads per query, each
// owning the even or odd feature columns.
template <int D>
__global__ void __launch_bounds__(128)
monarch_f32_stage1(const float *__restrict__ q, const float *__restrict__ k,
                   const float *__restrict__ v, float *__restrict__ out, F32Params p) {
    constexpr int DH = D / 2;
    constexpr int KC = 32;
    __shared__ float ks[KC][D];
    __shared__ float vs[KC][D];
    const long long blk = blockIdx.x / p.qchunks;
    const int qc = static_cast<int>(blockIdx.x % p.qchunks);
    const long long bh = blk / p.nblk_bh;
    const int b = static_cast<int>(blk % p.nblk_bh);
    const int lrow = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int i = qc * 64 + lrow;
    const bool active = i < p.m;
    const long long n = active ? f32_s1_token(p, b, i) : 0;
    float qr[DH], o[DH];
#pragma unroll
    for (int e = 0; e < DH; ++e) {
        qr[e] = active ? q[f32_row(p, bh, n) + 2 * e + half] * p.scale : 0.f;
        o[e] = 0.f;
    }
    float mrun = -INFINITY, l = 0.f;
    for (int j0 = 0; j0 < p.m; j0 += KC) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < KC * D; idx += blockDim.x) {
            const int jj = idx / D, c = idx % D, j = j0 + jj;
            if (j < p.m) {
                const long long nk = f32_s1_token(p, b, j);
                ks[jj][c] = k[f32_row(p, bh, nk) + c];
                vs[jj][c] = v[f32_row(p, bh, nk) + c];
            }
        }
        __syncthreads();
        const int jn = min(KC, p.m - j0);
        for (int jj = 0; jj < jn; ++jj) {
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < DH; ++e) part = fmaf(qr[e], ks[jj][2 * e + half], part);
            const float sc = part + __shfl_xor_sync(0xffffffffu, part, 1);
            if (sc > mrun) {
                const float a = expf(mrun - sc);
                l *= a;
#pragma unroll
                for (int e = 0; e < DH; ++e) o[e] *= a;
                mrun = sc;
            }
            const float pe = expf(sc - mrun);
            l += pe;
#pragma unroll
            for (int e = 0; e < DH; ++e) o[e] = fmaf(pe, vs[jj][2 * e + half], o[e]);
        }
    }
    if (active) {
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < DH; ++e) out[f32_row(p, bh, n) + 2 * e + half] = o[e] * inv;
    }
}

// One block = one group (batch-head, spatial position): the T tokens of that
// position across frames.  blockDim = 2*T rounded up to a warp.
template <int D>
__global__ void __launch_bounds__(256)
monarch_f32_stage2(const float *__restrict__ q, const float *__restrict__ k, float *out,
                   F32Params p) {
    constexpr int DH = D / 2;
    extern __shared__ float sm[];
    float *ks = sm;                 // [T][D]
    float *ys = sm + p.T * D;       // [T][D]
    const long long g = blockIdx.x;
    const long long bh = g / p.HW;
    const int pos = static_cast<int>(g % p.HW);
    for (int idx = threadIdx.x; idx < p.T * D; idx += blockDim.x) {
        const int t = idx / D, c = idx % D;
        const long long n = static_cast<long long>(t) * p.HW + pos;
        ks[idx] = k[f32_row(p, bh, n) + c];
        ys[idx] = out[f32_row(p, bh, n) + c];
    }
    __syncthreads();
    const int t = threadIdx.x >> 1, half = threadIdx.x & 1;
    const bool active = t < p.T;
    const long long n = static_cast<long long>(active ? t : 0) * p.HW + pos;
    float qr[DH], o[DH];
#pragma unroll
    for (int e = 0; e < DH; ++e) {
        qr[e] = active ? q[f32_row(p, bh, n) + 2 * e + half] * p.scale : 0.f;
        o[e] = 0.f;
    }
    float mrun = -INFINITY, l = 0.f;
    for (int j = 0; j < p.T; ++j) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < DH; ++e) part = fmaf(qr[e], ks[j * D + 2 * e + half], part);
        const float sc = part + __shfl_xor_sync(0xffffffffu, part, 1);
        if (sc > mrun) {
            const float a = expf(mrun - sc);
            l *= a;
#pragma unroll
            for (int e = 0; e < DH; ++e) o[e] *= a;
            mrun = sc;
        }
        const float pe = expf(sc - mrun);
        l += pe;
#pragma unroll
        for (int e = 0; e < DH; ++e) o[e] = fmaf(pe, ys[j * D + 2 * e + half], o[e]);
    }
    if (active) {
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < DH; ++e) out[f32_row(p, bh, n) + 2 * e + half] = o[e] * inv;
    }
}

}  // namespace monarch
