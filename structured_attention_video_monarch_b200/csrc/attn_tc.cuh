// attn_tc.cuh -- bf16 Monarch attention stages on tcgen05 tensor cores.
//
// One persistent kernel runs "units" of block-diagonal softmax attention.
// A unit is a pair of 128-row query tiles that share their keys:
//   stage-1 unit: two query tiles of one stage-1 block (a frame, or a spatial
//     tile of a frame), iterating over that block's key/value tiles with an
//     online softmax; values are V, results (Y1) go to `out`;
//   stage-2 unit: two "group chunks"; each chunk stacks npos spatial positions
//     x T frames (npos*T <= 128 rows) fetched with one TMA box, so the
//     permutation P of the Monarch factorisation is pure tensor-map
//     addressing.  Keys are the same stacked rows; a block-diagonal mask keeps
//     each row inside its own position's group; values are Y1 read back from
//     `out`, results overwrite `out`.
// (MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/nl/paper/2602.12271 "Methodologie"; gist.science/zh/paper/
// 2602.12271 section 2.2 on block alignment and tiled Monarch; the pages'
// kernels tile attention FlashAttention-style in on-chip memory without
// materialising the dense map, section 2.2 "Finetuning & Efficient
// Implementation".)
//
// Warp roles (512 threads, registers rebalanced with setmaxnreg):
//   warps 0-3   softmax for query tile 0 (thread = row)        192 regs
//   warps 4-7   softmax for query tile 1                        192 regs
//   warps 8-11  epilogue: O / l -> bf16 -> shared -> TMA store   72 regs
//   warp  12    TMA producer (Q tiles, K/V ring)                 56 regs
//   warp  13    TMEM allocator and single-thread tcgen05.mma issuer
//   warps 14-15 idle
// (2*128*192 + 128*72 + 128*56 = 65536, the registers the block launches with.)
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0, O1 after them.
// P (bf16) overwrites the first 64 columns of its S region and feeds the PV
// MMA straight from TMEM.  The MMA issue order per key tile j is
//   PV0(j-1), S0(j), PV1(j-1), S1(j)
// so one tile's softmax overlaps the other tile's MMAs; tcgen05.mma ops from
// one thread execute in order, which makes S_i(j+1) safe after PV_i(j).
#pragma once

#include "sm100.cuh"

namespace monarch {

enum : int { UNIT_STAGE1 = 1, UNIT_STAGE2 = 2 };

struct TcParams {
    int B, heads, T, H, W, HW;
    int fact;                       // 0 frame, 1 tiled
    int tile_h, tile_w, tiles_h, tiles_w;
    int rows_per_tile;              // tiled: tile rows per 128-row query/key tile
    int m;                          // tokens per stage-1 block
    int nblk_bh;                    // stage-1 blocks per (batch, head)
    int nqt;                        // 128-row query (= key) tiles per stage-1 block
    int s1_pairs;                   // ceil(nqt / 2)
    int npos;                       // stage-2 positions per chunk
    int s2_chunks;                  // chunks per (batch, head)
    int s2_pairs;                   // ceil(s2_chunks / 2)
    long long s1_units, s2_units;
    long long unit_begin, unit_end; // [begin, end) over stage-1 units then stage-2 units
    float scale_log2;               // d^-1/2 * log2(e)
    long long timeout_cycles;
    unsigned *status;
};

struct Unit {
    int kind;
    int nq;          // query tiles present (1 or 2)
    int nk;          // key/value tiles
    int bh;
    // stage 1
    int blk;         // global stage-1 block index
    int qt0;         // first query tile index inside the block
    // stage 2
    int chunk0;
};

__device__ __forceinline__ Unit decode_unit(const TcParams &p, long long u) {
    Unit r;
    if (u < p.s1_units) {
        r.kind = UNIT_STAGE1;
        long long blk = u / p.s1_pairs;
        int pair = static_cast<int>(u % p.s1_pairs);
        r.blk = static_cast<int>(blk);
        r.bh = static_cast<int>(blk / p.nblk_bh);
        r.qt0 = 2 * pair;
        r.nq = (r.qt0 + 1 < p.nqt) ? 2 : 1;
        r.nk = p.nqt;
        r.chunk0 = 0;
    } else {
        long long v = u - p.s1_units;
        r.kind = UNIT_STAGE2;
        r.bh = static_cast<int>(v / p.s2_pairs);
        int pair = static_cast<int>(v % p.s2_pairs);
        r.chunk0 = 2 * pair;
        r.nq = (r.chunk0 + 1 < p.s2_chunks) ? 2 : 1;
        r.nk = 1;
        r.blk = 0;
        r.qt0 = 0;
    }
    return r;
}

// Rows a stage-1 tile (query or key tile `tile` of block `blk`) brings in by
// TMA, and how many of them are real tokens of the block.
__device__ __forceinline__ void s1_tile_rows(const TcParams &p, int tile, int &loaded,
                                             int &valid) {
    if (p.fact == 0) {
        loaded = 128;  // rows past the block end are zero-filled by TMA
        int rem = p.m - tile * 128;
        valid = rem < 128 ? rem : 128;
    } else {
        loaded = p.rows_per_tile * p.tile_w;
        int rem_rows = p.tile_h - tile * p.rows_per_tile;
        int rows = rem_rows < p.rows_per_tile ? rem_rows : p.rows_per_tile;
        valid = rows * p.tile_w;
    }
}

// Issue the TMA load of one stage-1 tile (all panels) into dst.
template <int NP>
__device__ __forceinline__ void s1_load(const TcParams &p, const CUtensorMap *map, uint32_t dst,
                                        uint32_t bar, int blk, int tile) {
    if (p.fact == 0) {
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
            tma_load_3d(dst + pn * 16384, map, bar, pn * 64, tile * 128, blk);
    } else {
        int tpf = p.tiles_h * p.tiles_w;
        int frame = blk / tpf, tif = blk % tpf;
        int ti = tif / p.tiles_w, tj = tif % p.tiles_w;
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
            tma_load_5d(dst + pn * 16384, map, bar, pn * 64, 0, tj, tile * p.rows_per_tile,
                        frame * p.tiles_h + ti);
    }
}

template <int NP>
__device__ __forceinline__ void s1_store(const TcParams &p, const CUtensorMap *map, uint32_t src,
                                         int blk, int tile) {
    if (p.fact == 0) {
#pragma unroll
        for (int pn = 0; pn < NP; ++pn) tma_store_3d(map, src + pn * 16384, pn * 64, tile * 128, blk);
    } else {
        int tpf = p.tiles_h * p.tiles_w;
        int frame = blk / tpf, tif = blk % tpf;
        int ti = tif / p.tiles_w, tj = tif % p.tiles_w;
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
            tma_store_5d(map, src + pn * 16384, pn * 64, 0, tj, tile * p.rows_per_tile,
                         frame * p.tiles_h + ti);
    }
}

template <int NP>
__device__ __forceinline__ void s2_load(const CUtensorMap *map, uint32_t dst, uint32_t bar,
                                        int npos, int bh, int chunk) {
#pragma unroll
    for (int pn = 0; pn < NP; ++pn)
        tma_load_4d(dst + pn * 16384, map, bar, pn * 64, chunk * npos, 0, bh);
}

template <int NP>
__device__ __forceinline__ void s2_store(const CUtensorMap *map, uint32_t src, int npos, int bh,
                                         int chunk) {
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) tma_store_4d(map, src + pn * 16384, pn * 64, chunk * npos, 0, bh);
}

template <int D>
struct TcLayout {
    static constexpr int NP = D / 64;                 // 64-element (128-byte) panels per row
    static constexpr int TILE = 128 * D * 2;          // bytes of one 128-row tile
    static constexpr int NS = (D == 128) ? 3 : 6;     // K/V ring slots
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + 2 * TILE;
    static constexpr int OFF_STG = OFF_KV + NS * TILE;
    static constexpr int OFF_BAR = OFF_STG + 2 * TILE;
    // barriers: q_full[2] q_empty[2] kv_full[NS] kv_empty[NS] s_full[2] p_full[2]
    //           o_full[2] o_free[2] l_full[2] l_free[2]
    static constexpr int NBAR = 16 + 2 * NS;
    static constexpr int OFF_L = OFF_BAR + NBAR * 8;     // row sums l, [2 tiles][128 rows] fp32
    static constexpr int OFF_MISC = OFF_L + 2 * 128 * 4; // tmem base, abort flag
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;        // slack to align the base to 1024
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
};

// Zero rows [from, 128) of every panel of a 128-row tile (generic proxy),
// so that the PV MMA reads exact zeros where no value row was loaded.
template <int NP>
__device__ __forceinline__ void zero_tail_rows(uint32_t tile, int from) {
    for (int r = from; r < 128; ++r)
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
#pragma unroll
            for (int c = 0; c < 8; ++c) st_shared_v4(tile + pn * 16384 + r * 128 + c * 16, 0, 0, 0, 0);
}

__device__ __forceinline__ void setmaxnreg_inc192() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec72() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec56() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(512, 1)
monarch_tc_kernel(const __grid_constant__ CUtensorMap mq1, const __grid_constant__ CUtensorMap mk1,
                  const __grid_constant__ CUtensorMap mv1, const __grid_constant__ CUtensorMap mo1,
                  const __grid_constant__ CUtensorMap mq2, const __grid_constant__ CUtensorMap mk2,
                  const __grid_constant__ CUtensorMap my2, const __grid_constant__ CUtensorMap mo2,
                  const TcParams p) {
    using L = TcLayout<D>;
    constexpr int NP = L::NP;
    constexpr int NS = L::NS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);

    const uint32_t bar0 = base + L::OFF_BAR;
    auto q_full = [&](int i) { return bar0 + 8u * i; };
    auto q_empty = [&](int i) { return bar0 + 8u * (2 + i); };
    auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (4 + NS + s); };
    auto s_full = [&](int i) { return bar0 + 8u * (4 + 2 * NS + i); };
    auto p_full = [&](int i) { return bar0 + 8u * (6 + 2 * NS + i); };
    auto o_full = [&](int i) { return bar0 + 8u * (8 + 2 * NS + i); };
    auto o_free = [&](int i) { return bar0 + 8u * (10 + 2 * NS + i); };
    auto l_full = [&](int i) { return bar0 + 8u * (12 + 2 * NS + i); };
    auto l_free = [&](int i) { return bar0 + 8u * (14 + 2 * NS + i); };
    float *l_buf = reinterpret_cast<float *>(base_ptr + L::OFF_L);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + L::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(base_ptr + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    WaitCtl ctl{abort_flag, p.status, p.timeout_cycles};

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 1);
            mbar_init(q_empty(i), 1);
            mbar_init(s_full(i), 1);
            mbar_init(p_full(i), 128);
            mbar_init(o_full(i), 1);
            mbar_init(o_free(i), 128);
            mbar_init(l_full(i), 128);
            mbar_init(l_free(i), 128);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        fence_barrier_init();
    }
    if (warp == 12 && lane == 0) {
        tma_prefetch_desc(&mq1); tma_prefetch_desc(&mk1); tma_prefetch_desc(&mv1);
        tma_prefetch_desc(&mo1); tma_prefetch_desc(&mq2); tma_prefetch_desc(&mk2);
        tma_prefetch_desc(&my2); tma_prefetch_desc(&mo2);
    }
    if (warp == 13) {
        tmem_alloc(smem_addr(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (wg == 3) {
        setmaxnreg_dec56();
        if (warp == 12 && lane == 0) {
            // -------------------------------------------------------- TMA producer
            uint32_t qe_par = 3u;  // bit i: parity to wait for on q_empty(i)
            int slot = 0;
            uint32_t kv_round = 0;
            bool ok = true;
            auto acquire_slot = [&](int &s) -> bool {
                s = slot;
                bool r = mbar_wait(kv_empty(slot), (kv_round & 1u) ^ 1u, ctl);
                if (++slot == NS) { slot = 0; ++kv_round; }
                return r;
            };
            for (long long u = p.unit_begin + blockIdx.x; u < p.unit_end && ok; u += gridDim.x) {
                const Unit un = decode_unit(p, u);
                for (int i = 0; i < un.nq && ok; ++i) {
                    ok = mbar_wait(q_empty(i), (qe_par >> i) & 1u, ctl);
                    qe_par ^= 1u << i;
                    if (!ok) break;
                    const uint32_t dst = base + L::OFF_Q + i * L::TILE;
                    if (un.kind == UNIT_STAGE1) {
                        int loaded, valid;
                        s1_tile_rows(p, un.qt0 + i, loaded, valid);
                        mbar_arrive_expect_tx(q_full(i), NP * loaded * 128);
                        s1_load<NP>(p, &mq1, dst, q_full(i), un.blk, un.qt0 + i);
                    } else {
                        mbar_arrive_expect_tx(q_full(i), NP * p.npos * p.T * 128);
                        s2_load<NP>(&mq2, dst, q_full(i), p.npos, un.bh, un.chunk0 + i);
                    }
                }
                if (!ok) break;
                if (un.kind == UNIT_STAGE1) {
                    for (int j = 0; j < un.nk && ok; ++j) {
                        int loaded, valid;
                        s1_tile_rows(p, j, loaded, valid);
                        int s;
                        if (!(ok = acquire_slot(s))) break;
                        uint32_t dst = base + L::OFF_KV + s * L::TILE;
                        mbar_arrive_expect_tx(kv_full(s), NP * loaded * 128);
                        s1_load<NP>(p, &mk1, dst, kv_full(s), un.blk, j);
                        if (!(ok = acquire_slot(s))) break;
                        dst = base + L::OFF_KV + s * L::TILE;
                        if (loaded < 128) {
                            zero_tail_rows<NP>(dst, loaded);
                            fence_proxy_async_smem();
                        }
                        mbar_arrive_expect_tx(kv_full(s), NP * loaded * 128);
                        s1_load<NP>(p, &mv1, dst, kv_full(s), un.blk, j);
                    }
                } else {
                    const int rows = p.npos * p.T;
                    for (int i = 0; i < un.nq && ok; ++i) {
                        int s;
                        if (!(ok = acquire_slot(s))) break;
                        const uint32_t dst = base + L::OFF_KV + s * L::TILE;
                        mbar_arrive_expect_tx(kv_full(s), NP * rows * 128);
                        s2_load<NP>(&mk2, dst, kv_full(s), p.npos, un.bh, un.chunk0 + i);
                    }
                    for (int i = 0; i < un.nq && ok; ++i) {
                        int s;
                        if (!(ok = acquire_slot(s))) break;
                        const uint32_t dst = base + L::OFF_KV + s * L::TILE;
                        if (rows < 128) {
                            zero_tail_rows<NP>(dst, rows);
                            fence_proxy_async_smem();
                        }
                        mbar_arrive_expect_tx(kv_full(s), NP * rows * 128);
                        s2_load<NP>(&my2, dst, kv_full(s), p.npos, un.bh, un.chunk0 + i);
                    }
                }
            }
        } else if (warp == 13 && lane == 0) {
            // -------------------------------------------------------- MMA issuer
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
            uint32_t qf_par = 0u;  // bit i: parity to wait for on q_full(i)
            uint32_t pf_par = 0u;  // bit i: parity to wait for on p_full(i)
            uint32_t of_par = 3u;  // bit i: parity to wait for on o_free(i)
            int slot = 0;
            uint32_t kv_round = 0;
            bool ok = true;
            auto acquire_full = [&](int &s) -> bool {
                s = slot;
                bool r = mbar_wait(kv_full(slot), kv_round & 1u, ctl);
                if (++slot == NS) { slot = 0; ++kv_round; }
                return r;
            };
            // S_i = Q_i K^T: A = Q tile (K-major), B = K tile (K-major), K dim = D.
            auto issue_s = [&](int i, int s) {
                const uint32_t qa = base + L::OFF_Q + i * L::TILE;
                const uint32_t kb = base + L::OFF_KV + s * L::TILE;
                const uint32_t d_tmem = tmem + (i ? L::COL_S1 : L::COL_S0);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    mma_ss(d_tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                           IDESC_S, k > 0 ? 1u : 0u);
                }
            };
            // O_i (+)= P_i V: A = P from TMEM (bf16 pairs in the S region),
            // B = V tile (MN-major: keys x D, D contiguous), K dim = 128 keys.
            auto issue_pv = [&](int i, int s, uint32_t acc) {
                const uint32_t vb = base + L::OFF_KV + s * L::TILE;
                const uint32_t p_tmem = tmem + (i ? L::COL_S1 : L::COL_S0);
                const uint32_t d_tmem = tmem + (i ? L::COL_O1 : L::COL_O0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(d_tmem, p_tmem + k * 8, sdesc_sw128(vb + k * 2048, 16384, 1024), IDESC_O,
                           acc | (k > 0 ? 1u : 0u));
            };
            // the first PV of a unit overwrites O_i: the epilogue must be done with it
            auto wait_p_and_o = [&](int i, bool first) -> bool {
                if (first) {
                    if (!mbar_wait(o_free(i), (of_par >> i) & 1u, ctl)) return false;
                    of_par ^= 1u << i;
                }
                if (!mbar_wait(p_full(i), (pf_par >> i) & 1u, ctl)) return false;
                pf_par ^= 1u << i;
                tc_fence_after();
                return true;
            };
            for (long long u = p.unit_begin + blockIdx.x; u < p.unit_end && ok; u += gridDim.x) {
                const Unit un = decode_unit(p, u);
                for (int i = 0; i < un.nq && ok; ++i) {
                    ok = mbar_wait(q_full(i), (qf_par >> i) & 1u, ctl);
                    qf_par ^= 1u << i;
                }
                if (!ok) break;
                tc_fence_after();
                if (un.kind == UNIT_STAGE1) {
                    int sK, sV;
                    if (!acquire_full(sK)) { ok = false; break; }
                    tc_fence_after();
                    for (int i = 0; i < un.nq; ++i) {
                        issue_s(i, sK);
                        mma_commit(s_full(i));
                    }
                    mma_commit(kv_empty(sK));
                    if (un.nk == 1)
                        for (int i = 0; i < un.nq; ++i) mma_commit(q_empty(i));
                    for (int j = 1; j < un.nk && ok; ++j) {
                        if (!acquire_full(sV) || !acquire_full(sK)) { ok = false; break; }
                        tc_fence_after();
                        for (int i = 0; i < un.nq; ++i) {
                            if (!wait_p_and_o(i, j == 1)) { ok = false; break; }
                            issue_pv(i, sV, j > 1 ? 1u : 0u);
                            issue_s(i, sK);
                            mma_commit(s_full(i));
                        }
                        if (!ok) break;
                        mma_commit(kv_empty(sV));
                        mma_commit(kv_empty(sK));
                        if (j == un.nk - 1)
                            for (int i = 0; i < un.nq; ++i) mma_commit(q_empty(i));
                    }
                    if (!ok) break;
                    if (!acquire_full(sV)) { ok = false; break; }
                    tc_fence_after();
                    for (int i = 0; i < un.nq; ++i) {
                        if (!wait_p_and_o(i, un.nk == 1)) { ok = false; break; }
                        issue_pv(i, sV, un.nk > 1 ? 1u : 0u);
                        mma_commit(o_full(i));
                    }
                    if (!ok) break;
                    mma_commit(kv_empty(sV));
                } else {
                    for (int i = 0; i < un.nq; ++i) {
                        int sK;
                        if (!acquire_full(sK)) { ok = false; break; }
                        tc_fence_after();
                        issue_s(i, sK);
                        mma_commit(s_full(i));
                        mma_commit(kv_empty(sK));
                    }
                    if (!ok) break;
                    for (int i = 0; i < un.nq; ++i) mma_commit(q_empty(i));
                    for (int i = 0; i < un.nq; ++i) {
                        int sV;
                        if (!acquire_full(sV)) { ok = false; break; }
                        if (!wait_p_and_o(i, true)) { ok = false; break; }
                        issue_pv(i, sV, 0u);
                        mma_commit(o_full(i));
                        mma_commit(kv_empty(sV));
                    }
                }
            }
        }
    } else if (wg == 2) {
        setmaxnreg_dec72();
        // ------------------------------------------------------------ epilogue
        const int row = threadIdx.x & 127;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        uint32_t lf_par = 0u, of_par = 0u;  // bit i: parity for l_full(i) / o_full(i)
        bool ok = true;
        for (long long u = p.unit_begin + blockIdx.x; u < p.unit_end && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, u);
            for (int i = 0; i < un.nq; ++i) {
                if (!mbar_wait(l_full(i), (lf_par >> i) & 1u, ctl)) { ok = false; break; }
                lf_par ^= 1u << i;
                const float l = l_buf[i * 128 + row];
                mbar_arrive(l_free(i));
                const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
                if (!mbar_wait(o_full(i), (of_par >> i) & 1u, ctl)) { ok = false; break; }
                of_par ^= 1u << i;
                tc_fence_after();
                const uint32_t stg = base + L::OFF_STG + i * L::TILE;
                // the staging buffer is free once earlier TMA stores have read it
                if (row == 0) bulk_wait_group_read0();
                named_barrier_sync(1, 128);
                const uint32_t col_o = i ? L::COL_O1 : L::COL_O0;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + col_o + 32 * c, r);
                    tmem_wait_ld();
                    // columns [32c, 32c+32) = panel c/2, 16-byte chunks (c%2)*4 + 0..3,
                    // placed with the 128-byte swizzle the TMA store expects
                    const uint32_t rowaddr = stg + (c >> 1) * 16384 + row * 128;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t chunk = static_cast<uint32_t>(((c & 1) * 4 + q) ^ (row & 7));
                        st_shared_v4(rowaddr + chunk * 16,
                                     pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv_l,
                                                 __uint_as_float(r[8 * q + 1]) * inv_l),
                                     pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv_l,
                                                 __uint_as_float(r[8 * q + 3]) * inv_l),
                                     pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv_l,
                                                 __uint_as_float(r[8 * q + 5]) * inv_l),
                                     pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv_l,
                                                 __uint_as_float(r[8 * q + 7]) * inv_l));
                    }
                }
                // O_i has been read: the next unit may overwrite it
                tc_fence_before();
                mbar_arrive(o_free(i));
                fence_proxy_async_smem();
                named_barrier_sync(1, 128);
                if (row == 0) {
                    if (un.kind == UNIT_STAGE1)
                        s1_store<NP>(p, &mo1, stg, un.blk, un.qt0 + i);
                    else
                        s2_store<NP>(&mo2, stg, p.npos, un.bh, un.chunk0 + i);
                    bulk_commit_group();
                }
            }
        }
        if (row == 0) bulk_wait_group0();
    } else {
        setmaxnreg_inc192();
        // ------------------------------------------------------------ softmax
        const int row = threadIdx.x & 127;    // TMEM lane == tile row
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t col_s = wg ? L::COL_S1 : L::COL_S0;
        const uint32_t col_o = wg ? L::COL_O1 : L::COL_O0;
        const float sl2 = p.scale_log2;
        uint32_t sf_par = 0u, lfree_par = 1u;
        bool ok = true;
        for (long long u = p.unit_begin + blockIdx.x; u < p.unit_end && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, u);
            if (wg >= un.nq) continue;
            float m_run = -INFINITY;  // running max of raw logits
            float l_run = 0.f;        // running softmax denominator
            // stage-2 mask: the row belongs to position slot prow of the chunk
            const int prow = (un.kind == UNIT_STAGE2) ? (row % p.npos) : 0;
            int npos_valid = 0;
            if (un.kind == UNIT_STAGE2) {
                const int rem = p.HW - (un.chunk0 + wg) * p.npos;
                npos_valid = rem < p.npos ? rem : p.npos;
            }
            for (int j = 0; j < un.nk; ++j) {
                if (!mbar_wait(s_full(wg), sf_par, ctl)) { ok = false; break; }
                sf_par ^= 1u;
                tc_fence_after();
                float s[128];
                {
                    uint32_t r[4][32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + col_s + 32 * c, r[c]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(r[c][e]);
                }
                // mask invalid key columns
                if (un.kind == UNIT_STAGE1) {
                    int loaded, kvalid;
                    s1_tile_rows(p, j, loaded, kvalid);
                    if (kvalid < 128) {
#pragma unroll
                        for (int c = 0; c < 128; ++c)
                            if (c >= kvalid) s[c] = -INFINITY;
                    }
                } else {
                    int pc = 0, tc = 0;
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const bool valid = (pc == prow) && (tc < p.T) && (pc < npos_valid);
                        if (!valid) s[c] = -INFINITY;
                        if (++pc == p.npos) { pc = 0; ++tc; }
                    }
                }
                float mx = s[0];
#pragma unroll
                for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
                // conditional rescale: keep a stale max unless it grew by > 2^8
                bool rescale = false;
                float alpha = 1.f;
                if (j == 0) {
                    m_run = mx;
                } else if ((mx - m_run) * sl2 > 8.f) {
                    alpha = fast_exp2((m_run - mx) * sl2);
                    m_run = mx;
                    l_run *= alpha;
                    rescale = true;
                }
                const float moff = (m_run == -INFINITY) ? 0.f : m_run * sl2;
                float lsum = 0.f;
                // P = exp2(s*scale*log2e - m*scale*log2e) as bf16 pairs, written
                // over the first 64 columns of this tile's S region
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float x0 = s[32 * c + 2 * e], x1 = s[32 * c + 2 * e + 1];
                        const float a = (x0 == -INFINITY) ? 0.f : fast_exp2(fmaf(x0, sl2, -moff));
                        const float b = (x1 == -INFINITY) ? 0.f : fast_exp2(fmaf(x1, sl2, -moff));
                        pk[e] = pack_bf16x2(a, b);
                        // the denominator sums the bf16-rounded weights the PV
                        // MMA actually uses, so a dominant weight cancels exactly
                        lsum += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
                    }
                    tmem_st16(lane_base + col_s + 16 * c, pk);
                }
                l_run += lsum;
                // O from earlier key tiles is complete here (S_i(j) was issued
                // after PV_i(j-1)); rescale it before PV_i(j) accumulates
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + col_o + 32 * c, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(lane_base + col_o + 32 * c, r);
                    }
                }
                tmem_wait_st();
                if (j == un.nk - 1) {
                    // hand the row sum to the epilogue (one-slot handshake)
                    if (!mbar_wait(l_free(wg), lfree_par, ctl)) { ok = false; break; }
                    lfree_par ^= 1u;
                    l_buf[wg * 128 + row] = l_run;
                    mbar_arrive(l_full(wg));
                }
                tc_fence_before();
                mbar_arrive(p_full(wg));
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (*abort_flag) {
        // A wait gave up: let any copy or MMA still in flight land before the
        // shared and tensor memory are released.
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 24)) {
        }
    }
    if (warp == 13) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace monarch
