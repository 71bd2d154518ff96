// attn_chunk_mma.cuh -- stage 2 of an autoregressive chunk for 16-bit inputs
// on warp-level tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation).
//
// A chunk of T_new new frames attends, per spatial position, over the keys
// and stage-1 outputs of the T_old context frames and its own frames
// (MonarchRT, gist.science/zh/paper/2602.12271 section 2.2: the kernels
// process query frames in chunks, "mini-sequence"; the per-position group
// across frames is the stage-2 block of the factorisation,
// gist.science/nl/paper/2602.12271 "Methodologie").  The work per position is
// a few KB of rows with 4*d FLOPs per (query, key) pair, far below the ridge
// point, so the kernel is bound by HBM; warp MMAs replace the per-lane dot
// products, warp reductions and weight broadcasts of the CUDA-core kernel
// (attn_chunk.cuh), which spent about 1000 instructions per 8 keys.
//
// One warp per (batch-head, position).  Per pass of up to 16 queries and per
// chunk of up to 32 keys:
//   S[16 x 32] = Q[16 x D] K^T     4 n-tiles x D/16 k-steps of mma.m16n8k16
//   online softmax on the S accumulators (rows shared by a quad of lanes)
//   O[16 x D] += P[16 x 32] Y1[32 x D]   2 k-steps x D/8 n-tiles; P reuses the S accumulators as A fragments
// Rows are staged by cp.async into per-warp shared memory with a 16-byte pad
// per row (conflict-free ldmatrix); padded query rows read row 0 (their
// outputs are dropped), padded key rows read row 0 for K (masked) and a zero
// row for Y1 (so 0 * Y1 stays 0).  The softmax denominator sums the 16-bit
// weights the MMA multiplies.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

namespace monarch {

struct ChunkMmaParams {
    int HW, T_old, T_new;
    long long n_old, n_new, groups;
    float scale_log2;
    int qrows;   // query rows staged per warp: min(T_new, 16)
    int krows;   // key rows staged per warp: min(T_old + T_new, 32)
};

template <int D, typename E>
struct ChunkMmaCfg {
    static constexpr int RB = D * 2;          // bytes per row
    static constexpr int RS = RB + 16;        // padded row stride in shared memory
    static constexpr int WARPS = 8;
    static constexpr int KC = 32;             // keys per chunk
    static constexpr int QM = 16;             // queries per pass
    // per-warp bytes for q + 2 * k rows (runtime counts), plus one zero row per CTA
    static int smem_bytes(int qrows, int krows) { return WARPS * (qrows + 2 * krows) * RS + RS; }
};

__device__ __forceinline__ void cpa16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa_commit_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
template <typename E>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<E, __half>::value) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};\n"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};\n"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}
template <typename E>
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
    uint32_t w;
    if constexpr (std::is_same<E, __half>::value) {
        const __half2 h = __floats2half2_rn(lo, hi);
        memcpy(&w, &h, 4);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        memcpy(&w, &h, 4);
    }
    return w;
}

// The two 16-bit values of a packed pair, widened exactly to fp32, summed.
template <typename E>
__device__ __forceinline__ float sum_pair(uint32_t w) {
    if constexpr (std::is_same<E, __half>::value) {
        __half2 h;
        memcpy(&h, &w, 4);
        const float2 f = __half22float2(h);
        return f.x + f.y;
    } else {
        return __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
    }
}

template <int D, typename E>
__global__ void __launch_bounds__(256)
monarch_chunk_stage2_mma(const E *__restrict__ q, const E *__restrict__ k, const E *__restrict__ k_cache,
                         const E *__restrict__ y1_cache, const E *__restrict__ y1_new, E *__restrict__ out,
                         ChunkMmaParams p) {
    using Cfg = ChunkMmaCfg<D, E>;
    constexpr int RB = Cfg::RB, RS = Cfg::RS, KC = Cfg::KC, QM = Cfg::QM;
    constexpr int PARTS = RB / 16;   // 16-byte pieces per row
    constexpr int NT = D / 8;        // output n-tiles
    extern __shared__ __align__(16) unsigned char cm_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the zero row (last RS bytes) is written by the whole CTA before any warp leaves
    unsigned char *zero_row = cm_smem + Cfg::WARPS * (p.qrows + 2 * p.krows) * RS;
    for (int i = threadIdx.x; i < RS / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(zero_row)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const long long g = static_cast<long long>(blockIdx.x) * Cfg::WARPS + warp;
    if (g >= p.groups) return;
    const long long bh = g / p.HW;
    const int pos = static_cast<int>(g - bh * p.HW);
    const long long fstride = static_cast<long long>(p.HW) * D;
    const long long row_new = (bh * p.n_new + pos) * D, row_old = (bh * p.n_old + pos) * D;
    const E *qb = q + row_new, *kn = k + row_new, *yn = y1_new + row_new;
    E *ob = out + row_new;
    const E *kc = p.T_old ? k_cache + row_old : kn;
    const E *yc = p.T_old ? y1_cache + row_old : yn;
    const int T_tot = p.T_old + p.T_new;
    unsigned char *qs = cm_smem + warp * (p.qrows + 2 * p.krows) * RS;  // query rows
    unsigned char *ks = qs + p.qrows * RS;                               // key rows
    unsigned char *ys = ks + p.krows * RS;                               // Y1 rows
    const uint32_t qs_a = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
    const uint32_t ks_a = static_cast<uint32_t>(__cvta_generic_to_shared(ks));
    const uint32_t ys_a = static_cast<uint32_t>(__cvta_generic_to_shared(ys));
    const uint32_t zr_a = static_cast<uint32_t>(__cvta_generic_to_shared(zero_row));
    const int gq = lane >> 2, tig = lane & 3;  // fragment row group, thread in group

    for (int t0 = 0; t0 < p.T_new; t0 += QM) {
        const int nq = p.T_new - t0 < QM ? p.T_new - t0 : QM;
        // stage the pass's query rows
        for (int c = lane; c < nq * PARTS; c += 32) {
            const int r = c / PARTS, part = c - r * PARTS;
            cpa16(qs_a + r * RS + part * 16, qb + (t0 + r) * fstride + part * 8);
        }
        float o[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows gq and gq + 8
        for (int j0 = 0; j0 < T_tot; j0 += KC) {
            const int nk = T_tot - j0 < KC ? T_tot - j0 : KC;
            __syncwarp();  // the previous chunk's rows are no longer read
            for (int c = lane; c < nk * PARTS; c += 32) {
                const int r = c / PARTS, part = c - r * PARTS;
                const int j = j0 + r;
                const bool old = j < p.T_old;
                const long long off = static_cast<long long>(old ? j : j - p.T_old) * fstride + part * 8;
                cpa16(ks_a + r * RS + part * 16, (old ? kc : kn) + off);
                cpa16(ys_a + r * RS + part * 16, (old ? yc : yn) + off);
            }
            cpa_commit_wait_all();
            __syncwarp();
            // S = Q K^T: 4 key n-tiles
            float s[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
            // ldmatrix row addresses: thread t gives row t % 8 of matrix t / 8
            const int mrow = lane & 7, mat = lane >> 3;
            const int qr = (mat & 1) * 8 + mrow;                     // A: matrices (rows 0-7 | 8-15) x (k lo | hi)
            const uint32_t qrow_a = qs_a + (qr < nq ? qr : 0) * RS + (mat >> 1) * 16;
#pragma unroll
            for (int ks_i = 0; ks_i < D / 16; ++ks_i) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(qrow_a + ks_i * 32, a0, a1, a2, a3);
#pragma unroll
                for (int np = 0; np < 2; ++np) {  // two key n-tiles per ldmatrix.x4
                    const int key = (2 * np + (mat >> 1)) * 8 + mrow;  // B: (n-tile lo | hi) x (k lo | hi)
                    const uint32_t krow_a = ks_a + (key < nk ? key : 0) * RS + (mat & 1) * 16 + ks_i * 32;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(krow_a, b0, b1, b2, b3);
                    mma16816<E>(s[2 * np], a0, a1, a2, a3, b0, b1);
                    mma16816<E>(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
                }
            }
            // online softmax on rows gq (s[][0..1]) and gq + 8 (s[][2..3])
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool valid = nt * 8 + 2 * tig + e < nk;
                    s[nt][e] = valid ? s[nt][e] * p.scale_log2 : -INFINITY;
                    s[nt][2 + e] = valid ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, s[nt][e]);
                    mx1 = fmaxf(mx1, s[nt][2 + e]);
                }
#pragma unroll
            for (int o2 = 1; o2 < 4; o2 <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
            }
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float ps0 = 0.f, ps1 = 0.f;
            uint32_t pa[4][2];  // P as bf16 pairs: [n-tile][row gq | gq + 8]
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float p00 = exp2f(s[nt][0] - mn0), p01 = exp2f(s[nt][1] - mn0);
                const float p10 = exp2f(s[nt][2] - mn1), p11 = exp2f(s[nt][3] - mn1);
                pa[nt][0] = pk2<E>(p00, p01);
                pa[nt][1] = pk2<E>(p10, p11);
                ps0 += sum_pair<E>(pa[nt][0]);
                ps1 += sum_pair<E>(pa[nt][1]);
            }
            l0 = l0 * c0 + ps0;  // thread-partial sums; the quad is reduced at the end
            l1 = l1 * c1 + ps1;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[nt][0] *= c0; o[nt][1] *= c0;
                o[nt][2] *= c1; o[nt][3] *= c1;
            }
            // O += P Y1: k-steps of 16 keys; A fragment from the S accumulators
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const uint32_t a0 = pa[2 * kk][0], a1 = pa[2 * kk][1], a2 = pa[2 * kk + 1][0], a3 = pa[2 * kk + 1][1];
                const int key = kk * 16 + (mat & 1) * 8 + mrow;  // trans: (keys lo | hi) x (n-tile lo | hi)
                const uint32_t yrow_a = (key < nk ? ys_a + key * RS : zr_a) + (mat >> 1) * 16;
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(yrow_a + np * 32, b0, b1, b2, b3);
                    mma16816<E>(o[2 * np], a0, a1, a2, a3, b0, b1);
                    mma16816<E>(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        // normalise and store rows gq and gq + 8 that are real queries
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
        }
        const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int col = nt * 8 + 2 * tig;
            if (gq < nq)
                *reinterpret_cast<uint32_t *>(ob + (t0 + gq) * fstride + col) = pk2<E>(o[nt][0] * i0, o[nt][1] * i0);
            if (gq + 8 < nq)
                *reinterpret_cast<uint32_t *>(ob + (t0 + gq + 8) * fstride + col) = pk2<E>(o[nt][2] * i1, o[nt][3] * i1);
        }
        __syncwarp();  // query rows are restaged by the next pass
    }
}

}  // namespace monarch
