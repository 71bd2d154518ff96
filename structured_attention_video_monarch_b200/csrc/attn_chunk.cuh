// attn_chunk.cuh -- stage 2 of an autoregressive chunk, on CUDA cores.
//
// A chunk of T_new new frames is computed with the T_old earlier frames as
// context (MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/it/paper/2602.12271, problem statement: autoregressive
// generation; gist.science/zh/paper/2602.12271 section 2.2: query frames
// processed in chunks).  Stage 1 of the new frames is the full forward's
// stage 1 (its blocks never cross frames).  Stage 2 of a new query at spatial
// position pos attends over the keys of all T_old + T_new frames at pos, with
// their stage-1 outputs as values: frames [0, T_old) from k_cache / y1_cache,
// the rest from k / y1_new.
//
// Per query this is a softmax over T_old + T_new keys: about 4 flops per
// element of the 2 x d key/value elements it reads, so the kernel is bound by
// HBM bandwidth and runs on CUDA cores.  One warp per (batch-head, position);
// each lane owns C = d/32 consecutive features, so a row is one coalesced
// 32-lane access; up to QG queries per pass share every key/value row staged
// in shared memory.  Accumulation, softmax and normalisation are fp32; exp2
// of log2(e)-prescaled logits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

namespace monarch {

struct ChunkParams {
    int HW;            // positions per frame
    int T_old, T_new;  // context frames, new frames
    long long n_old;   // context tokens per batch-head (T_old * HW)
    long long n_new;   // new tokens per batch-head (T_new * HW)
    long long groups;  // batch-heads x positions
    float scale_log2;  // d^-1/2 * log2(e)
};

// Two 16-bit values packed in one word -> two floats.
template <typename E>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if constexpr (std::is_same<E, __half>::value) {
        __half2 h;
        memcpy(&h, &w, 4);
        return __half22float2(h);
    } else {
        __nv_bfloat162 h;
        memcpy(&h, &w, 4);
        return __bfloat1622float2(h);
    }
}

template <typename E>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    uint32_t w;
    if constexpr (std::is_same<E, __half>::value) {
        const __half2 h = __floats2half2_rn(a, b);
        memcpy(&w, &h, 4);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        memcpy(&w, &h, 4);
    }
    return w;
}

// Raw bytes of a lane's C consecutive elements of a row (4, 8 or 16 bytes),
// read with one shared-memory load and converted to fp32 when used.
template <int BYTES>
struct RawOf;
template <>
struct RawOf<4> { using T = unsigned int; };
template <>
struct RawOf<8> { using T = uint2; };
template <>
struct RawOf<16> { using T = uint4; };
template <typename E, int C>
using RawRow = typename RawOf<C * static_cast<int>(sizeof(E))>::T;

template <typename E, int C>
__device__ __forceinline__ void raw_unpack(const RawRow<E, C> &r, float (&x)[C]) {
    constexpr int NW = C * static_cast<int>(sizeof(E)) / 4;
    uint32_t w[NW];
    memcpy(w, &r, sizeof(w));
    if constexpr (std::is_same<E, float>::value) {
#pragma unroll
        for (int i = 0; i < C; ++i) x[i] = __uint_as_float(w[i]);
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const float2 f = unpack2<E>(w[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    }
}

template <typename E, int C>
__device__ __forceinline__ void chunk_store(E *__restrict__ p, const float (&x)[C]) {
    if constexpr (std::is_same<E, float>::value) {
        if constexpr (C == 4)
            *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
        else
            *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    } else {
        if constexpr (C == 4)
            *reinterpret_cast<uint2 *>(p) = make_uint2(pack2<E>(x[0], x[1]), pack2<E>(x[2], x[3]));
        else
            *reinterpret_cast<unsigned int *>(p) = pack2<E>(x[0], x[1]);
    }
}

// 16-byte global -> shared copies that bypass the registers (and L1).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Sums NV (16 or 32) per-lane partial values over the warp so that lane l
// ends with the full sum of value l % NV.  Each step exchanges only the half
// of the values the partner keeps (a butterfly reduce-scatter): 31 shuffles
// for 32 values instead of 5 per value.
template <int NV>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV], int lane) {
    static_assert(NV == 16 || NV == 32, "16 or 32 values");
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const int nb = NV < 2 * o ? NV : 2 * o;  // values still held
        if (NV > o) {
            const int h = nb / 2;
            const bool up = (lane & o) != 0;  // keep the upper half
#pragma unroll
            for (int i = 0; i < h; ++i) {
                const float send = up ? v[i] : v[i + h];
                const float keep = up ? v[i + h] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        } else {
#pragma unroll
            for (int i = 0; i < nb; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
        }
    }
}

// Launch shape and per-warp staging of the chunk stage 2.
template <int D, typename E>
struct ChunkCfg {
    static constexpr int C = D / 32;                          // features per lane
    static constexpr int QG = 4;                              // queries per pass
    static constexpr int KB = sizeof(E) == 2 ? 8 : 4;         // keys per block
    static constexpr int NV = QG * KB;                        // logits per block
    static constexpr int RB = D * static_cast<int>(sizeof(E));  // bytes per row
    static constexpr int NST = 3;                             // key blocks in flight per warp
    static constexpr int STAGE = KB * 2 * RB;                 // K and Y1 rows of one key block
    static constexpr int WARPS = 8;                           // warps (positions) per CTA
    static constexpr int SMEM = WARPS * NST * STAGE;          // dynamic shared memory per CTA
};

// All tensors [B*heads][tokens][D] contiguous: q, k, y1_new and out hold the
// T_new new frames, k_cache and y1_cache the T_old context frames.
//
// Per pass of up to QG queries, keys go in blocks of KB.  A block's K and Y1
// rows are copied to this warp's shared-memory ring with cp.async, NST blocks
// ahead of the one being used, so a warp keeps up to NST * STAGE bytes in
// flight without holding them in registers.  Each block's QG x KB logits are
// reduced together, and the online softmax takes one step per block (block
// maximum, one exp2 per lane, rescale once).
template <int D, typename E>
__global__ void __launch_bounds__(256, 2)
monarch_chunk_stage2(const E *__restrict__ q, const E *__restrict__ k, const E *__restrict__ k_cache,
                     const E *__restrict__ y1_cache, const E *__restrict__ y1_new, E *__restrict__ out,
                     ChunkParams p) {
    using Cfg = ChunkCfg<D, E>;
    constexpr int C = Cfg::C, QG = Cfg::QG, KB = Cfg::KB, NV = Cfg::NV, RB = Cfg::RB;
    constexpr int NST = Cfg::NST, STAGE = Cfg::STAGE;
    constexpr int PARTS = RB / 16;  // 16-byte pieces per row
    static_assert(C == 2 || C == 4, "d must be 64 or 128");
    using Raw = RawRow<E, C>;
    extern __shared__ __align__(16) unsigned char chunk_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long g = static_cast<long long>(blockIdx.x) * Cfg::WARPS + warp;
    if (g >= p.groups) return;  // whole warps leave together; no block-wide barrier follows
    const long long bh = g / p.HW;
    const int pos = static_cast<int>(g - bh * p.HW);
    const long long fstride = static_cast<long long>(p.HW) * D;  // one frame
    // rows of this (batch-head, position) at frame 0
    const long long row_new = (bh * p.n_new + pos) * D;
    const E *qb = q + row_new + lane * C, *kn = k + row_new, *yn = y1_new + row_new;
    E *ob = out + row_new + lane * C;
    // with no context the cache pointers are not used (and may be null)
    const long long row_old = (bh * p.n_old + pos) * D;
    const E *kc = p.T_old ? k_cache + row_old : kn;
    const E *yc = p.T_old ? y1_cache + row_old : yn;
    const int T_tot = p.T_old + p.T_new;
    const int nblk = (T_tot + KB - 1) / KB;
    unsigned char *ring = chunk_smem + warp * NST * STAGE;
    const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(ring));
    // this lane's logit after the reduction: query ql, key ul of the block
    const int ql = (lane % NV) / KB, ul = lane % KB;

    // Key block b -> ring stage b % NST: row 2u holds K of key j0 + u, row
    // 2u + 1 its Y1; the lanes split the 16-byte pieces.
    auto issue = [&](int b) {
        const int j0 = b * KB;
        const int nk = T_tot - j0 < KB ? T_tot - j0 : KB;
        const uint32_t st = ring_s + (b % NST) * STAGE;
        for (int c = lane; c < nk * 2 * PARTS; c += 32) {
            const int row = c / PARTS, part = c - row * PARTS;
            const int j = j0 + (row >> 1);
            const bool old = j < p.T_old;
            const E *base = (row & 1) ? (old ? yc : yn) : (old ? kc : kn);
            const E *src = base + static_cast<long long>(old ? j : j - p.T_old) * fstride + part * (16 / sizeof(E));
            cp_async16(st + row * RB + part * 16, src);
        }
        cp_async_commit();
    };

    for (int t0 = 0; t0 < p.T_new; t0 += QG) {
        const int nq = p.T_new - t0 < QG ? p.T_new - t0 : QG;
#pragma unroll
        for (int b = 0; b < NST - 1; ++b) {
            if (b < nblk) issue(b);
            else cp_async_commit();  // keep one group per block for the wait count
        }
        float qx[QG][C], acc[QG][C], m[QG], l[QG];
#pragma unroll
        for (int qi = 0; qi < QG; ++qi) {
            m[qi] = -INFINITY;
            l[qi] = 0.f;
#pragma unroll
            for (int c = 0; c < C; ++c) acc[qi][c] = 0.f;
            if (qi < nq) {
                raw_unpack<E, C>(__ldg(reinterpret_cast<const Raw *>(qb + (t0 + qi) * fstride)), qx[qi]);
#pragma unroll
                for (int c = 0; c < C; ++c) qx[qi][c] *= p.scale_log2;
            } else {
#pragma unroll
                for (int c = 0; c < C; ++c) qx[qi][c] = 0.f;
            }
        }
        for (int b = 0; b < nblk; ++b) {
            if (b + NST - 1 < nblk) issue(b + NST - 1);
            else cp_async_commit();
            cp_async_wait<NST - 1>();  // this lane's copies of block b have landed
            __syncwarp();              // ... and every other lane's
            const unsigned char *st = ring + (b % NST) * STAGE;
            const int nk = T_tot - b * KB < KB ? T_tot - b * KB : KB;
            float v[NV];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                float kx[C];
                if (u < nk) {
                    raw_unpack<E, C>(*reinterpret_cast<const Raw *>(st + 2 * u * RB + lane * C * sizeof(E)), kx);
                } else {
#pragma unroll
                    for (int c = 0; c < C; ++c) kx[c] = 0.f;
                }
#pragma unroll
                for (int qi = 0; qi < QG; ++qi) {
                    float sacc = 0.f;
#pragma unroll
                    for (int c = 0; c < C; ++c) sacc = fmaf(qx[qi][c], kx[c], sacc);
                    v[qi * KB + u] = sacc;
                }
            }
            reduce_scatter<NV>(v, lane);
            // padding queries get a finite logit (their results are dropped),
            // padding keys weight 0
            float s = v[0];
            if (ql >= nq) s = 0.f;
            else if (ul >= nk) s = -INFINITY;
            float m_old = m[0];
#pragma unroll
            for (int qi = 1; qi < QG; ++qi)
                if (ql == qi) m_old = m[qi];
            float bm = s;
#pragma unroll
            for (int o = 1; o < KB; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float mn = fmaxf(m_old, bm);
            const float pe = exp2f(s - mn);
            float bs = pe;
#pragma unroll
            for (int o = 1; o < KB; o <<= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
#pragma unroll
            for (int qi = 0; qi < QG; ++qi) {
                if (qi >= nq) break;  // the same for every lane
                const float mq = __shfl_sync(0xffffffffu, mn, qi * KB);
                const float sq = __shfl_sync(0xffffffffu, bs, qi * KB);
                const float corr = exp2f(m[qi] - mq);
                l[qi] = fmaf(l[qi], corr, sq);
                m[qi] = mq;
#pragma unroll
                for (int c = 0; c < C; ++c) acc[qi][c] *= corr;
            }
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                if (u >= nk) break;
                float yx[C];
                raw_unpack<E, C>(*reinterpret_cast<const Raw *>(st + (2 * u + 1) * RB + lane * C * sizeof(E)), yx);
#pragma unroll
                for (int qi = 0; qi < QG; ++qi) {
                    if (qi >= nq) break;
                    const float pq = __shfl_sync(0xffffffffu, pe, qi * KB + u);
#pragma unroll
                    for (int c = 0; c < C; ++c) acc[qi][c] = fmaf(pq, yx[c], acc[qi][c]);
                }
            }
            __syncwarp();  // stage b % NST is refilled by the next iteration's copy
        }
#pragma unroll
        for (int qi = 0; qi < QG; ++qi) {
            if (qi >= nq) break;
            const float inv = 1.f / l[qi];
            float o[C];
#pragma unroll
            for (int c = 0; c < C; ++c) o[c] = acc[qi][c] * inv;
            chunk_store<E, C>(ob + (t0 + qi) * fstride, o);
        }
    }
}

// Host side: one warp per (batch-head, position), Cfg::WARPS warps per CTA.
// The dynamic shared-memory limit is raised once per device.  Returns
// cudaSuccess or the first error.
template <int D, typename E>
inline cudaError_t chunk_stage2_launch(const E *q, const E *k, const E *k_cache, const E *y1_cache,
                                       const E *y1_new, E *out, const ChunkParams &p, cudaStream_t stream) {
    using Cfg = ChunkCfg<D, E>;
    // the attribute is per function and device; setting it again is harmless,
    // so concurrent first calls need no more than the flag's own lock
    static std::mutex mu;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!attr_done[dev]) {
            e = cudaFuncSetAttribute(monarch_chunk_stage2<D, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM);
            if (e != cudaSuccess) return e;
            attr_done[dev] = true;
        }
    }
    const long long blocks = (p.groups + Cfg::WARPS - 1) / Cfg::WARPS;
    monarch_chunk_stage2<D, E><<<static_cast<unsigned>(blocks), 32 * Cfg::WARPS, Cfg::SMEM, stream>>>(
        q, k, k_cache, y1_cache, y1_new, out, p);
    return cudaGetLastError();
}

}  // namespace monarch
