// attn_bwd_f32.cuh -- fp32 gradients of the Monarch attention on CUDA cores.
//
// The pages state that their kernels run the backward pass as well
// (MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/nl/paper/2602.12271, "Methodologie"; gist.science/zh/paper/
// 2602.12271, section 2.2).  For out = A2(Q, K) Y1, Y1 = A1(Q, K) V (A1, A2
// the block softmax attentions of the two stages) and an upstream gradient
// dO, per block and query x with weights p (softmax of s <q_x, k_j>):
//     dp_j = <dy_x, val_j>,  dl_j = p_j (dp_j - sum_i p_i dp_i),
//     dq_x += s sum_j dl_j k_j,  dk_j += s dl_j q_x,  dval_j += p_j dy_x.
// Stage 2 runs first with dy = dO and values Y1 (recomputed by the forward
// stage-1 kernel); its value gradient is dY1.  Stage 1 then runs with
// dy = dY1 and values V.
//
// One warp per query row, the lanes splitting the d features; the per-key
// weights of the warp's row sit in shared memory.  dQ rows belong to one
// warp each (written by stage 2, added to by stage 1); dK, dV and dY1 rows
// collect contributions from every query of their block and are accumulated
// with atomicAdd (so their summation order, and last-bit rounding, varies
// from run to run).
#pragma once

#include "attn_f32.cuh"

namespace monarch {

// Sum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Backward of one query row over `len` keys whose token indices come from
// key_token(j).  pw, dpw: this warp's shared scratch of len floats.
template <int D, typename KeyTok>
__device__ __forceinline__ void bwd_query(const F32Params &p, long long bh, long long nx, int len,
                                          KeyTok key_token, const float *q, const float *k,
                                          const float *val, const float *dy, float *dq, float *dk,
                                          float *dval, float *pw, float *dpw, bool add_dq) {
    constexpr int C = D / 32;  // features per lane
    const int lane = threadIdx.x & 31;
    float qx[C], dyx[C], dqx[C];
    const long long rx = f32_row(p, bh, nx);
#pragma unroll
    for (int c = 0; c < C; ++c) {
        qx[c] = q[rx + lane + 32 * c];
        dyx[c] = dy[rx + lane + 32 * c];
        dqx[c] = 0.f;
    }
    // logits and their maximum
    float mx = -INFINITY;
    for (int j = 0; j < len; ++j) {
        const long long rj = f32_row(p, bh, key_token(j));
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < C; ++c) acc = fmaf(qx[c], k[rj + lane + 32 * c], acc);
        const float l = warp_sum(acc) * p.scale;
        if (lane == 0) pw[j] = l;
        mx = fmaxf(mx, l);
    }
    __syncwarp();
    float z = 0.f;
    for (int j = lane; j < len; j += 32) {
        const float e = expf(pw[j] - mx);
        pw[j] = e;
        z += e;
    }
    z = warp_sum(z);
    __syncwarp();
    // weights, dp_j and <p, dp>
    float pdp = 0.f;
    for (int j = 0; j < len; ++j) {
        const long long rj = f32_row(p, bh, key_token(j));
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < C; ++c) acc = fmaf(dyx[c], val[rj + lane + 32 * c], acc);
        const float dpj = warp_sum(acc);
        const float pj = pw[j] / z;
        pdp = fmaf(pj, dpj, pdp);
        __syncwarp();
        if (lane == 0) {
            pw[j] = pj;
            dpw[j] = dpj;
        }
    }
    __syncwarp();
    // dl_j, then the three gradient contributions
    for (int j = 0; j < len; ++j) {
        const long long rj = f32_row(p, bh, key_token(j));
        const float pj = pw[j];
        const float dl = pj * (dpw[j] - pdp);
#pragma unroll
        for (int c = 0; c < C; ++c) {
            const int col = lane + 32 * c;
            dqx[c] = fmaf(p.scale * dl, k[rj + col], dqx[c]);
            atomicAdd(dk + rj + col, p.scale * dl * qx[c]);
            atomicAdd(dval + rj + col, pj * dyx[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const int col = lane + 32 * c;
        dq[rx + col] = add_dq ? dq[rx + col] + dqx[c] : dqx[c];
    }
    __syncwarp();
}

// Stage-2 backward: one block per (batch-head, position); its warps take the
// T frames' queries in turn.  Writes dq; accumulates dk and dy1 (zeroed first).
template <int D>
__global__ void __launch_bounds__(128) monarch_f32_bwd_stage2(const float *q, const float *k, const float *y1,
                                                             const float *dout, float *dq, float *dk,
                                                             float *dy1, F32Params p) {
    __shared__ float pw[4][128], dpw[4][128];
    const int warp = threadIdx.x >> 5;
    const long long g = blockIdx.x;
    const long long bh = g / p.HW;
    const int pos = static_cast<int>(g - bh * p.HW);
    auto key_token = [&](int j) { return static_cast<long long>(j) * p.HW + pos; };
    for (int t = warp; t < p.T; t += 4)
        bwd_query<D>(p, bh, static_cast<long long>(t) * p.HW + pos, p.T, key_token, q, k, y1, dout, dq, dk,
                     dy1, pw[warp], dpw[warp], false);
}

// Stage-1 backward: one block per (batch-head, stage-1 block, 4 queries), one
// query per warp; dynamic shared memory holds 2 x m floats per warp.  Adds to
// dq; accumulates dk and dv (zeroed first).
template <int D>
__global__ void __launch_bounds__(128) monarch_f32_bwd_stage1(const float *q, const float *k, const float *v,
                                                             const float *dy1, float *dq, float *dk, float *dv,
                                                             F32Params p, int qgroups) {
    extern __shared__ float bwd_sm[];
    const int warp = threadIdx.x >> 5;
    const long long g = blockIdx.x;
    const long long blk = g / qgroups;  // global stage-1 block
    const int qg = static_cast<int>(g - blk * qgroups);
    const long long bh = blk / p.nblk_bh;
    const int b = static_cast<int>(blk - bh * p.nblk_bh);
    const int i = qg * 4 + warp;
    if (i >= p.m) return;
    float *pw = bwd_sm + static_cast<size_t>(warp) * 2 * p.m;
    float *dpw = pw + p.m;
    auto key_token = [&](int j) { return f32_s1_token(p, b, j); };
    bwd_query<D>(p, bh, f32_s1_token(p, b, i), p.m, key_token, q, k, v, dy1, dq, dk, dv, pw, dpw, true);
}

}  // namespace monarch
