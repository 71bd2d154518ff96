// attn_bwd_tc.cuh -- bf16 / fp16 gradients of the Monarch attention on
// tcgen05 tensor cores.
//
// The pages' kernels run the backward pass as well as the forward
// (MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/nl/paper/2602.12271 "Methodologie"; gist.science/zh/paper/
// 2602.12271 section 2.2).  Every diagonal block of B1 and B2 is a softmax
// attention, so each stage's backward is the block-local attention backward:
// with P = softmax(S), S = Q K^T / sqrt(d), upstream dY and values Vals,
//   dVals = P^T dY,  dP = dY Vals^T,  dS = P * (dP - rowsum(dY * Y)),
//   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
// Stage 2 (values Y1, output O, upstream dO) gives dY1 and its parts of dQ
// and dK; stage 1 (values V, output Y1, upstream dY1) gives dV and the rest.
//
// Two kernels per stage, over that stage's geometry (frame or tile blocks,
// or the forward's stacked stage-2 tiles):
//   dq kernel   (query-outer): pass 1 over key tiles -> row LSE; pass 2 -> P, dP, dS, dQ += dS K
//   dkdv kernel (key-outer):   per query tile S^T, dP^T -> P^T, dS^T; dV += P^T dY, dK += dS^T Q
// Only the two MMA forms of the forward are used: SS with both operands
// K-major (the S = Q K^T form) and TS with A in tensor memory and B MN-major
// (the O += P V form), so S and S^T are each computed directly, never
// transposed.  The same 128-row SW128 tile is a K-major operand (rows x d)
// and an MN-major B operand (K = rows, N = d).  Every output row has one
// owning CTA: no atomics.
//
// Roles (384 threads): warp 0 controls loads and MMAs (lane 0 issues the
// TMA loads, an elected lane the MMAs, all lanes wait); warp 1
// allocates TMEM; warps 4-11 do the elementwise work, two threads per row
// (thread = TMEM lane and column half).  The streamed tiles are double
// buffered.  Every wait is a bounded mbarrier wait.
#pragma once

#include "sm100.cuh"

namespace monarch {

enum : int { BWD_GEOM_FRAME = 0, BWD_GEOM_STAGE2 = 1, BWD_GEOM_TILED = 2 };

struct BwdParams {
    int B, heads, T, H, W, HW;
    long long N;          // tokens per batch-head
    int m;                // frame: tokens per block (H*W); tiled: tile_h * tile_w
    int nblk_bh;          // frame: frames per batch-head; tiled: T * tiles_h * tiles_w
    int ntile;            // 128-row tiles per block (frame, tiled); stage 2: 1
    int tile_h, tile_w, tiles_h, tiles_w, rows_per_tile;  // tiled: block = one tile of one frame
    int npos;             // stage 2: positions per stacked tile
    int s2_chunks;        // stage 2: stacked tiles per batch-head
    float scale_log2;     // d^-1/2 * log2(e)
    float scale;          // d^-1/2
    const float *D;       // per row: rowsum(dY * Y) of this stage, [BH][N]
    float *lse;           // per row: log2-sum-exp of the scaled logits, [BH][N] (dkdv reads)
    int lse_given;        // lse holds the forward's values (dq skips its LSE pass); else dq writes it
    float *dq;            // fp32 [BH][N][d]: written, or (add_dq) the other stage's part read
    float *dk;            // fp32 [BH][N][d]: written, or (add_dk) the other stage's part read
    void *dv16;           // value gradient in 16 bits [BH][N][d] (written), or null
    int add_dq, add_dk;
    int pair_split;       // monarch_bwd_pair: CTAs [0, pair_split) run the dq body, the rest dk/dv
    // 16-bit final gradients [BH][N][d] (input dtype): when set, the kernel
    // adds the other stage's fp32 part and writes the result here
    void *out_dq, *out_dk;
    long long timeout_cycles;
    unsigned *status;
};

template <int D>
struct BwdLayout {
    static constexpr int NP = D / 64;
    static constexpr int TILE = NP * 16384;            // 128 rows x D bf16, SW128 panels
    // The operands that stay are single tiles; the streamed ones are double
    // buffered, so tile t + 1 loads while tile t is computed.
    static constexpr int OFF_A = 0;                    // dq: Q          dkdv: K
    static constexpr int OFF_B = OFF_A + TILE;         // dq: dY         dkdv: Vals
    static constexpr int OFF_C = OFF_B + TILE;         // dq: K_j [2]    dkdv: Q_i [2]
    static constexpr int OFF_E = OFF_C + 2 * TILE;     // dq: Vals_j [2] dkdv: dY_i [2]
    static constexpr int OFF_BAR = OFF_E + 2 * TILE;
    // ld_full[2] (one per buffer), mma_done, ew_done, mm2_done, fin, ls_ready, x_ready
    static constexpr int NBAR = 8;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    // dk/dv kernel: LSE and rowsum terms of the current query tile's rows, [2 tiles][2][128];
    // dq kernel: each column half's running (max, sum) of every row, [2 halves][128][2]
    static constexpr int OFF_LS = OFF_MISC + 16;
    static constexpr int BYTES = OFF_LS + 2 * 2 * 128 * 4;
    // 8 elementwise warps: thread = (row, column half)
    static constexpr int THREADS = 384;
    static constexpr int SLACK = 1024;
    // Every CTA allocates all 512 TMEM columns, so a second CTA on the same SM
    // could only block in tcgen05.alloc until the first one exits.  Asking for
    // more than half of the SM's shared memory keeps the CTAs one per SM.
    static constexpr int ONE_PER_SM = 116 * 1024;
    static constexpr int ALLOC = BYTES + SLACK > ONE_PER_SM ? BYTES + SLACK : ONE_PER_SM;
    static_assert(ALLOC <= 232448, "too much shared memory");
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_ACC0 = 256, COL_ACC1 = 256 + D;
    // 16-bit pairs written over a 128-column S or dP region: column half h
    // (keys 64h .. 64h+63) packs into columns [64h, 64h + 32) of the region,
    // inside the columns it read itself, so the two halves never touch each
    // other's data; the TMEM-operand MMA reads K steps 4-7 from there
    static constexpr uint32_t pack_col(int h, int c) { return 64u * h + 16u * (c - 2 * h); }
};

// Problem geometry: which tokens a 128-row tile holds and which (row, col)
// pairs of a tile pair are inside one attention block.
struct BwdGeom {
    int kind;
    // frame: problem = (bh, t); tiles are 128-row slabs of the frame
    // stage 2: problem = (bh, chunk); one stacked tile npos positions x T frames
    __device__ static long long token(const BwdParams &p, int kind, int prob_local, int tile, int row) {
        if (kind == BWD_GEOM_TILED) {
            const int tpf = p.tiles_h * p.tiles_w;
            const int t = prob_local / tpf, tif = prob_local - t * tpf;
            const int ti = tif / p.tiles_w, tj = tif - ti * p.tiles_w;
            const int rr = row / p.tile_w, wl = row - rr * p.tile_w;
            const int hl = tile * p.rows_per_tile + rr;
            if (rr >= p.rows_per_tile || hl >= p.tile_h) return -1;
            return static_cast<long long>(t) * p.HW + static_cast<long long>(ti * p.tile_h + hl) * p.W +
                   tj * p.tile_w + wl;
        }
        if (kind == BWD_GEOM_FRAME) {
            const int i = tile * 128 + row;
            if (i >= p.m) return -1;
            return static_cast<long long>(prob_local) * p.HW + i;
        }
        const int t = row / p.npos, pl = row - t * p.npos;
        const int pos = prob_local * p.npos + pl;
        if (t >= p.T || pos >= p.HW) return -1;
        return static_cast<long long>(t) * p.HW + pos;
    }
    // Validity bits of columns [32*chunk, 32*chunk + 32) of tile `kt` seen
    // from row `row` of the other operand's tile: frame and tiled geometries,
    // the columns holding real tokens of the block (a prefix); stage 2, the
    // columns of the row's own position slot in real frames (the relation is
    // symmetric, so it serves query rows and key rows alike).
    __device__ static uint32_t col_mask(const BwdParams &p, int kind, int kt, int row, int chunk) {
        const int c0 = 32 * chunk;
        if (kind == BWD_GEOM_STAGE2) {
            const int lim = p.npos * p.T;
            int c = row % p.npos;
            if (c < c0) c += ((c0 - c + p.npos - 1) / p.npos) * p.npos;
            uint32_t m = 0u;
            for (; c < c0 + 32 && c < lim; c += p.npos) m |= 1u << (c - c0);
            return m;
        }
        int n;
        if (kind == BWD_GEOM_FRAME) {
            n = p.m - kt * 128;
        } else {
            int r = p.tile_h - kt * p.rows_per_tile;
            if (r > p.rows_per_tile) r = p.rows_per_tile;
            n = r * p.tile_w;
        }
        if (n > 128) n = 128;
        n -= c0;
        return n >= 32 ? 0xFFFFFFFFu : (n <= 0 ? 0u : ((1u << n) - 1u));
    }
};

// TMA load of one 128-row tile of a problem.  frame map (d, m, T, heads, B),
// box (64, 128, 1, 1, 1); stage-2 map (d, HW, T, heads, B), box (64, npos, T, 1, 1).
template <int NP>
__device__ __forceinline__ int bwd_load(const BwdParams &p, int kind, const CUtensorMap *map, uint32_t dst,
                                        uint32_t bar, int bh, int prob_local, int tile) {
    const int b = bh / p.heads, hd = bh - b * p.heads;
    if (kind == BWD_GEOM_TILED) {
        // map (d, tile_w, tiles_w, tile_h, tiles_h * B*heads*T), box (64, tile_w, 1, rows_per_tile, 1)
        const int tpf = p.tiles_h * p.tiles_w;
        const int t = prob_local / tpf, tif = prob_local - t * tpf;
        const int ti = tif / p.tiles_w, tj = tif - ti * p.tiles_w;
        const int frame = bh * p.T + t;
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
            tma_load_5d(dst + pn * 16384, map, bar, pn * 64, 0, tj, tile * p.rows_per_tile, frame * p.tiles_h + ti);
        return p.rows_per_tile * p.tile_w;
    }
    if (kind == BWD_GEOM_FRAME) {
#pragma unroll
        for (int pn = 0; pn < NP; ++pn) tma_load_5d(dst + pn * 16384, map, bar, pn * 64, tile * 128, prob_local, hd, b);
        return 128;  // rows past the frame end are zero-filled
    }
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) tma_load_5d(dst + pn * 16384, map, bar, pn * 64, prob_local * p.npos, 0, hd, b);
    return p.npos * p.T;
}

// Zero rows [from, to) of every panel of a tile; the 32 lanes of the calling
// warp share the 16-byte pieces.
template <int NP>
__device__ __forceinline__ void bwd_zero_rows(uint32_t tile, int from, int to, int lane) {
    for (int x = lane; x < (to - from) * NP * 8; x += 32) {
        const int r = from + x / (NP * 8), pn = (x / 8) % NP, c = x % 8;
        st_shared_v4(tile + pn * 16384 + r * 128 + c * 16, 0, 0, 0, 0);
    }
}

// S-form MMA: D[128 x 128] = A[128 x d] B[128 x d]^T, both K-major SW128 tiles;
// called by a whole converged warp (one elected lane issues).
template <int D, bool F16>
__device__ __forceinline__ void bwd_mma_ss(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
    constexpr uint32_t KM_HI = sdesc_sw128_hi(1024);
    constexpr uint32_t IDESC = F16 ? idesc_f16_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
    const uint32_t a = sdesc_sw128_lo(a_addr, 16), b = sdesc_sw128_lo(b_addr, 16);
    mma_ss_lh_elect<0>(d_tmem, a, KM_HI, b, KM_HI, IDESC);
#pragma unroll
    for (int k = 1; k < D / 16; ++k) {
        const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
        mma_ss_lh_elect<1>(d_tmem, a + off, KM_HI, b + off, KM_HI, IDESC);
    }
}

// PV-form MMA (called by a whole converged warp): D[128 x d] (+)= A[128 x 128] (16-bit pairs in TMEM at a_tmem)
// * B[128 x d] (SW128 tile read MN-major: K = tile rows, N = d).
template <int D, bool F16>
__device__ __forceinline__ void bwd_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_addr, bool accumulate) {
    constexpr uint32_t MN_HI = sdesc_sw128_hi(1024);
    constexpr uint32_t IDESC = F16 ? idesc_f16_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
    const uint32_t b = sdesc_sw128_lo(b_addr, 16384);
    mma_ts_lh_elect(d_tmem, a_tmem, b, MN_HI, IDESC, accumulate ? 1u : 0u);
    // keys 0-63 are packed in columns [0, 32) of the A region, keys 64-127 in [64, 96)
#pragma unroll
    for (int k = 1; k < 8; ++k) mma_ts_lh_elect(d_tmem, a_tmem + k * 8 + (k >= 4 ? 32 : 0), b + k * 128, MN_HI, IDESC, 1u);
}

template <bool F16>
__device__ __forceinline__ uint32_t bwd_pack(float lo, float hi) {
    if constexpr (F16)
        return pack_f16x2(lo, hi);
    else
        return pack_bf16x2(lo, hi);
}

// ------------------------------------------------------------------ dq kernel
// grid: one CTA per (bh, problem, query tile).  Maps: q, k, vals, dy (same geometry).
template <int D, bool F16, int KIND>
__device__ __forceinline__ void bwd_dq_body(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mvals,
                                            const CUtensorMap &mdy, const BwdParams &p, const int cta) {
    using L = BwdLayout<D>;
    constexpr int NP = L::NP;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = base + L::OFF_BAR;
    // ld_full(b): the tiles of buffer b landed; then mma_done, ew_done, mm2_done, fin
    auto ld_full = [&](int b) { return bar0 + 8u * static_cast<uint32_t>(b); };
    const uint32_t mma_done = bar0 + 16, ew_done = bar0 + 24, mm2_done = bar0 + 32, fin = bar0 + 40;
    const uint32_t x_ready = bar0 + 56;  // both column halves posted their running (max, sum)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + L::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(base_ptr + L::OFF_MISC + 4);
    WaitCtl ctl{abort_flag, p.status, p.timeout_cycles};

    // problem decode
    const int nq_tiles = KIND == BWD_GEOM_STAGE2 ? 1 : p.ntile;
    const int per_bh = (KIND == BWD_GEOM_STAGE2 ? p.s2_chunks : p.nblk_bh) * nq_tiles;
    const int bh = cta / per_bh;
    const int rem = cta - bh * per_bh;
    const int prob = rem / nq_tiles, qt = rem - prob * nq_tiles;
    const int nk_tiles = nq_tiles;

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        mbar_init(ld_full(0), 1);
        mbar_init(ld_full(1), 1);
        mbar_init(mma_done, 1);
        mbar_init(ew_done, 256);
        mbar_init(mm2_done, 1);
        mbar_init(fin, 1);
        mbar_init(x_ready, 256);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = base + L::OFF_A, tdy = base + L::OFF_B, tk = base + L::OFF_C, tv = base + L::OFF_E;

    if (warp == 0) {
        // ------------------------------------------------------ control thread
        // Tiles g = 0 .. 2*nk - 1: pass 1 (g < nk) computes S = Q K_g^T for
        // the row LSE; pass 2 (key tile j = g - nk) computes S and dP = dY Vals_j^T,
        // waits for the elementwise dS, then dQ += dS K_j.  Tile g's K (and
        // Vals) land in buffer g & 1, loaded while tile g - 1 is computed; Q
        // arrives with tile 0, dY with tile nk.
        const int rows = KIND == BWD_GEOM_FRAME ? 128 : (KIND == BWD_GEOM_TILED ? p.rows_per_tile * p.tile_w : p.npos * p.T);
        // With the LSE given, the sequence starts at pass 2 (g0 = nk).  Buffer
        // and barrier phase follow the position i = g - g0 in the sequence.
        const int g0 = p.lse_given ? nk_tiles : 0;
        const int ng = 2 * nk_tiles;
        uint32_t ew_par = 0u, m2_par = 0u;
        bool ok = true;
        auto issue_load = [&](int g) {
            const int b = (g - g0) & 1;
            const bool pass2 = g >= nk_tiles;
            const int jt = pass2 ? g - nk_tiles : g;
            const uint32_t kb = tk + b * L::TILE, vb = tv + b * L::TILE;
            if (pass2 && rows < 128) {  // K rows the dQ MMA reads but TMA does not write
                bwd_zero_rows<NP>(kb, rows, 128, lane);
                fence_proxy_async_smem();
            }
            const int ntiles = 1 + (g == g0) + (pass2 ? 1 : 0) + (g == nk_tiles);
            if (lane == 0) {
                mbar_arrive_expect_tx(ld_full(b), ntiles * NP * rows * 128);
                if (g == g0) bwd_load<NP>(p, KIND, &mq, tq, ld_full(b), bh, prob, qt);
                if (g == nk_tiles) bwd_load<NP>(p, KIND, &mdy, tdy, ld_full(b), bh, prob, qt);
                bwd_load<NP>(p, KIND, &mk, kb, ld_full(b), bh, prob, jt);
                if (pass2) bwd_load<NP>(p, KIND, &mvals, vb, ld_full(b), bh, prob, jt);
            }
            __syncwarp();
        };
        issue_load(g0);
        for (int g = g0; g < ng && ok; ++g) {
            const int b = (g - g0) & 1;
            if (g > g0) {
                if (g - 1 < nk_tiles) {  // pass-1 tile g-1: its S was read (its MMA is complete)
                    ok = mbar_wait_warp(ew_done, ew_par, ctl);
                    ew_par ^= 1u;
                } else {  // pass-2 tile g-1: its dQ MMA (the last reader of its buffers and of dS) is complete
                    ok = mbar_wait_warp(mm2_done, m2_par, ctl);
                    m2_par ^= 1u;
                }
                if (!ok) break;
            }
            if (g + 1 < ng) issue_load(g + 1);  // into the buffer tile g-1 used
            ok = mbar_wait_warp(ld_full(b), static_cast<uint32_t>((g - g0) >> 1) & 1u, ctl);
            if (!ok) break;
            tc_fence_after();
            const uint32_t kb = tk + b * L::TILE, vb = tv + b * L::TILE;
            bwd_mma_ss<D, F16>(tmem + L::COL_S, tq, kb);
            if (g < nk_tiles) {
                mma_commit_elect(mma_done);
                continue;
            }
            bwd_mma_ss<D, F16>(tmem + L::COL_DP, tdy, vb);
            mma_commit_elect(mma_done);
            ok = mbar_wait_warp(ew_done, ew_par, ctl);  // dS stored (16-bit pairs at COL_DP)
            ew_par ^= 1u;
            if (!ok) break;
            tc_fence_after();
            bwd_mma_ts<D, F16>(tmem + L::COL_ACC0, tmem + L::COL_DP, kb, g > nk_tiles);
            mma_commit_elect(mm2_done);
        }
        if (ok) {
            ok = mbar_wait_warp(mm2_done, m2_par, ctl);
            m2_par ^= 1u;
        }
        if (ok) mma_commit_elect(fin);
    } else if (warp >= 4) {
        // ------------------------------------------------------ elementwise threads
        // thread = (row, column half h): S / dP columns [64h, 64h + 64), 32-column chunks 2h, 2h + 1
        const int ew = threadIdx.x - 128;
        const int row = ew & 127, h = ew >> 7;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const long long tok = BwdGeom::token(p, KIND, prob, qt, row);
        const long long rowg = tok >= 0 ? static_cast<long long>(bh) * p.N + tok : -1;
        // the row's rowsum term, needed in pass 2: loaded now, used after pass 1
        const float dd = rowg >= 0 ? p.D[rowg] : 0.f;
        uint32_t md_par = 0u;
        bool ok = true;
        float m_run = -INFINITY, l_run = 0.f;  // this half's running max and sum, base 2
        // pass 1 (the row LSE), unless the forward's recomputation left it
        const int nk_pass1 = p.lse_given ? 0 : nk_tiles;
        for (int j = 0; j < nk_pass1 && ok; ++j) {
            ok = mbar_wait_warp(mma_done, md_par, ctl);
            md_par ^= 1u;
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 2 * h; c < 2 * h + 2; ++c) {
                uint32_t r[32];
                tmem_ld32(lane_base + L::COL_S + 32 * c, r);
                const uint32_t vm = BwdGeom::col_mask(p, KIND, j, row, c);
                tmem_wait_ld();
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const bool vis = (vm >> e) & 1u;
                    const float x = vis ? __uint_as_float(r[e]) * p.scale_log2 : -INFINITY;
                    r[e] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
                const float mn = fmaxf(m_run, mx);
                if (mn != -INFINITY) {  // nothing visible so far: keep (-inf, 0)
                    float sum = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) sum += fast_exp2(__uint_as_float(r[e]) - mn);
                    l_run = (m_run == -INFINITY ? 0.f : l_run * fast_exp2(m_run - mn)) + sum;
                    m_run = mn;
                }
            }
            tc_fence_before();
            mbar_arrive(ew_done);
        }
        // the row's LSE from both halves' (max, sum), combined in the same
        // order by both, so both get the same bits
        float lse = 0.f;
        if (ok && p.lse_given) {
            lse = rowg >= 0 ? p.lse[rowg] : 0.f;
        } else if (ok) {
            float *xs = reinterpret_cast<float *>(base_ptr + L::OFF_LS);
            xs[(h * 128 + row) * 2] = m_run;
            xs[(h * 128 + row) * 2 + 1] = l_run;
            mbar_arrive(x_ready);
            ok = mbar_wait_warp(x_ready, 0u, ctl);
            if (ok) {
                const float m0 = xs[row * 2], l0 = xs[row * 2 + 1];
                const float m1 = xs[(128 + row) * 2], l1 = xs[(128 + row) * 2 + 1];
                const float m = fmaxf(m0, m1);
                if (m != -INFINITY) {
                    const float l = (m0 == -INFINITY ? 0.f : l0 * fast_exp2(m0 - m)) +
                                    (m1 == -INFINITY ? 0.f : l1 * fast_exp2(m1 - m));
                    lse = m + __log2f(l);
                }
            }
        }
        if (ok && !p.lse_given && h == 0 && rowg >= 0) p.lse[rowg] = lse;
        for (int j = 0; j < nk_tiles && ok; ++j) {
            ok = mbar_wait_warp(mma_done, md_par, ctl);
            md_par ^= 1u;
            if (!ok) break;
            tc_fence_after();
            // dS = P * (dP - D), P = 2^(s*c - lse); stored as 16-bit pairs over
            // dP columns this thread has already read (L::pack_col)
#pragma unroll 1
            for (int c = 2 * h; c < 2 * h + 2; ++c) {
                uint32_t rs[32], rp[32];
                tmem_ld32(lane_base + L::COL_S + 32 * c, rs);
                tmem_ld32(lane_base + L::COL_DP + 32 * c, rp);
                const uint32_t vm = rowg >= 0 ? BwdGeom::col_mask(p, KIND, j, row, c) : 0u;
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float ds[2];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const bool vis = (vm >> (2 * e + h2)) & 1u;
                        // hidden pairs are exact zeros (their S and dP may be stale bits)
                        ds[h2] = vis ? fast_exp2(__uint_as_float(rs[2 * e + h2]) * p.scale_log2 - lse) *
                                           (__uint_as_float(rp[2 * e + h2]) - dd)
                                     : 0.f;
                    }
                    pk[e] = bwd_pack<F16>(ds[0], ds[1]);
                }
                tmem_st16(lane_base + L::COL_DP + L::pack_col(h, c), pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ew_done);
        }
        // this half's dQ columns of the other stage, loaded while the last dQ
        // MMA runs (the epilogue adds to them)
        float *dst = rowg >= 0 ? p.dq + rowg * D + h * (D / 2) : nullptr;
        float prev[D / 2];
#pragma unroll
        for (int e = 0; e < D / 2; ++e) prev[e] = (dst && p.add_dq) ? dst[e] : 0.f;
        if (ok) ok = mbar_wait_warp(fin, 0u, ctl);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t r[32];
                tmem_ld32(lane_base + L::COL_ACC0 + h * (D / 2) + 32 * c, r);
                tmem_wait_ld();
                if (dst && p.out_dq) {  // final dQ in 16 bits
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = bwd_pack<F16>(prev[32 * c + 2 * e] + __uint_as_float(r[2 * e]) * p.scale,
                                             prev[32 * c + 2 * e + 1] + __uint_as_float(r[2 * e + 1]) * p.scale);
                    uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out_dq) + rowg * D + h * (D / 2) + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                } else if (dst) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) dst[32 * c + e] = prev[32 * c + e] + __uint_as_float(r[e]) * p.scale;
                }
                __syncwarp();
            }
        }
    }
    __syncthreads();
    if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 24)) {
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ dk/dv kernel
// grid: one CTA per (bh, problem, key tile).  Maps: k, vals (A operands), q, dy.
template <int D, bool F16, int KIND>
__device__ __forceinline__ void bwd_dkdv_body(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mvals,
                                              const CUtensorMap &mdy, const BwdParams &p, const int cta) {
    using L = BwdLayout<D>;
    constexpr int NP = L::NP;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = base + L::OFF_BAR;
    // ld_full(b): the tiles of buffer b landed; then mma_done, ew_done, mm2_done, fin
    auto ld_full = [&](int b) { return bar0 + 8u * static_cast<uint32_t>(b); };
    const uint32_t mma_done = bar0 + 16, ew_done = bar0 + 24, mm2_done = bar0 + 32, fin = bar0 + 40;
    const uint32_t ls_ready = bar0 + 48;  // the 256 elementwise threads posted a query tile's LSE and D
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + L::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(base_ptr + L::OFF_MISC + 4);
    WaitCtl ctl{abort_flag, p.status, p.timeout_cycles};

    const int nk_tiles = KIND == BWD_GEOM_STAGE2 ? 1 : p.ntile;
    const int per_bh = (KIND == BWD_GEOM_STAGE2 ? p.s2_chunks : p.nblk_bh) * nk_tiles;
    const int bh = cta / per_bh;
    const int rem = cta - bh * per_bh;
    const int prob = rem / nk_tiles, kt = rem - prob * nk_tiles;
    const int nq_tiles = nk_tiles;

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        mbar_init(ld_full(0), 1);
        mbar_init(ld_full(1), 1);
        mbar_init(mma_done, 1);
        mbar_init(ew_done, 256);
        mbar_init(mm2_done, 1);
        mbar_init(fin, 1);
        mbar_init(ls_ready, 256);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tk = base + L::OFF_A, tv = base + L::OFF_B, tq = base + L::OFF_C, tdy = base + L::OFF_E;

    if (warp == 0) {
        // Query tile i's Q and dY land in buffer i & 1, loaded while tile
        // i - 1 is computed; K and Vals arrive with tile 0.
        uint32_t ew_par = 0u, m2_par = 0u;
        bool ok = true;
        const int rows = KIND == BWD_GEOM_FRAME ? 128 : (KIND == BWD_GEOM_TILED ? p.rows_per_tile * p.tile_w : p.npos * p.T);
        auto issue_load = [&](int i) {
            const int b = i & 1;
            const uint32_t qb = tq + b * L::TILE, yb = tdy + b * L::TILE;
            if (rows < 128) {  // Q and dY rows the dK/dV MMAs read but TMA does not write
                bwd_zero_rows<NP>(qb, rows, 128, lane);
                bwd_zero_rows<NP>(yb, rows, 128, lane);
                fence_proxy_async_smem();
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(ld_full(b), (i == 0 ? 4 : 2) * NP * rows * 128);
                if (i == 0) {
                    bwd_load<NP>(p, KIND, &mk, tk, ld_full(b), bh, prob, kt);
                    bwd_load<NP>(p, KIND, &mvals, tv, ld_full(b), bh, prob, kt);
                }
                bwd_load<NP>(p, KIND, &mq, qb, ld_full(b), bh, prob, i);
                bwd_load<NP>(p, KIND, &mdy, yb, ld_full(b), bh, prob, i);
            }
            __syncwarp();
        };
        issue_load(0);
        for (int i = 0; i < nq_tiles && ok; ++i) {
            const int b = i & 1;
            if (i > 0) {  // the dV/dK MMAs of tile i-1 (the last readers of its buffers, P^T and dS^T) are complete
                ok = mbar_wait_warp(mm2_done, m2_par, ctl);
                m2_par ^= 1u;
                if (!ok) break;
            }
            if (i + 1 < nq_tiles) issue_load(i + 1);  // into the buffer tile i-1 used
            ok = mbar_wait_warp(ld_full(b), static_cast<uint32_t>(i >> 1) & 1u, ctl);
            if (!ok) break;
            tc_fence_after();
            const uint32_t qb = tq + b * L::TILE, yb = tdy + b * L::TILE;
            bwd_mma_ss<D, F16>(tmem + L::COL_S, tk, qb);    // S^T = K Q^T
            bwd_mma_ss<D, F16>(tmem + L::COL_DP, tv, yb);   // dP^T = Vals dY^T
            mma_commit_elect(mma_done);
            ok = mbar_wait_warp(ew_done, ew_par, ctl);  // P^T at COL_S, dS^T at COL_DP (16-bit pairs)
            ew_par ^= 1u;
            if (!ok) break;
            tc_fence_after();
            bwd_mma_ts<D, F16>(tmem + L::COL_ACC0, tmem + L::COL_S, yb, i > 0);   // dV += P^T dY
            bwd_mma_ts<D, F16>(tmem + L::COL_ACC1, tmem + L::COL_DP, qb, i > 0);  // dK += dS^T Q
            mma_commit_elect(mm2_done);
        }
        if (ok) {
            ok = mbar_wait_warp(mm2_done, m2_par, ctl);
            m2_par ^= 1u;
        }
        if (ok) mma_commit_elect(fin);
    } else if (warp >= 4) {
        // thread = (key row, column half h): query columns [64h, 64h + 64)
        const int ew = threadIdx.x - 128;
        const int row = ew & 127, h = ew >> 7;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const long long tok = BwdGeom::token(p, KIND, prob, kt, row);
        const long long rowg = tok >= 0 ? static_cast<long long>(bh) * p.N + tok : -1;
        // LSE and rowsum term of each query row of the current query tile, by
        // column: the two threads of row index r post those of query row r (half
        // 0 the LSE, half 1 the rowsum term); a query row that holds no token
        // gets LSE = +inf, so its weights are exactly 0
        float *ls_buf = reinterpret_cast<float *>(base_ptr + L::OFF_LS);
        // tile i's value is loaded during tile i - 1 (its latency overlaps that tile's work)
        auto fetch = [&](int i) -> float {
            const long long qtok = BwdGeom::token(p, KIND, prob, i, row);
            const long long qg = static_cast<long long>(bh) * p.N + qtok;
            if (h == 0) return qtok >= 0 ? __ldg(p.lse + qg) : INFINITY;
            return qtok >= 0 ? __ldg(p.D + qg) : 0.f;
        };
        float next = fetch(0);
        uint32_t md_par = 0u;
        bool ok = true;
        for (int i = 0; i < nq_tiles && ok; ++i) {
            float *lse_s = ls_buf + (i & 1) * 256, *d_s = lse_s + 128;
            (h == 0 ? lse_s : d_s)[row] = next;
            if (i + 1 < nq_tiles) next = fetch(i + 1);
            // wait until all 256 threads posted tile i's values (a bounded
            // wait, like every other); the other buffer was last read in tile
            // i - 1, which every thread finished before arriving here
            mbar_arrive(ls_ready);
            ok = mbar_wait_warp(ls_ready, static_cast<uint32_t>(i) & 1u, ctl);
            if (!ok) break;
            ok = mbar_wait_warp(mma_done, md_par, ctl);
            md_par ^= 1u;
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 2 * h; c < 2 * h + 2; ++c) {
                uint32_t rs[32], rp[32];
                tmem_ld32(lane_base + L::COL_S + 32 * c, rs);
                tmem_ld32(lane_base + L::COL_DP + 32 * c, rp);
                // stage 2: the query columns of this key's position slot
                const uint32_t vm = KIND == BWD_GEOM_STAGE2 ? BwdGeom::col_mask(p, KIND, i, row, c) : 0xFFFFFFFFu;
                tmem_wait_ld();
                uint32_t pp[16], pd[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float pv[2], dsv[2];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int q = 32 * c + 2 * e + h2;  // query column of tile i
                        const float x = fast_exp2(__uint_as_float(rs[2 * e + h2]) * p.scale_log2 - lse_s[q]);
                        pv[h2] = ((vm >> (2 * e + h2)) & 1u) ? x : 0.f;
                        dsv[h2] = pv[h2] * (__uint_as_float(rp[2 * e + h2]) - d_s[q]);
                    }
                    pp[e] = bwd_pack<F16>(pv[0], pv[1]);
                    pd[e] = bwd_pack<F16>(dsv[0], dsv[1]);
                }
                tmem_st16(lane_base + L::COL_S + L::pack_col(h, c), pp);
                tmem_st16(lane_base + L::COL_DP + L::pack_col(h, c), pd);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ew_done);
        }
        // this half's dK columns of the other stage, loaded while the last
        // MMAs run (the epilogue adds to them)
        float prev[D / 2];
#pragma unroll
        for (int e = 0; e < D / 2; ++e) prev[e] = (rowg >= 0 && p.add_dk) ? p.dk[rowg * D + h * (D / 2) + e] : 0.f;
        if (ok) ok = mbar_wait_warp(fin, 0u, ctl);
        if (ok) {
            // every lane of the warp takes part in the TMEM loads (they are
            // warp-collective); only rows holding a real key store
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                const int c = h * (D / 64) + cc;
                uint32_t rv[32], rk[32];
                tmem_ld32(lane_base + L::COL_ACC0 + 32 * c, rv);
                tmem_ld32(lane_base + L::COL_ACC1 + 32 * c, rk);
                tmem_wait_ld();
                if (rowg >= 0 && p.out_dk) {  // final dK in 16 bits
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = bwd_pack<F16>(prev[32 * cc + 2 * e] + __uint_as_float(rk[2 * e]) * p.scale,
                                             prev[32 * cc + 2 * e + 1] + __uint_as_float(rk[2 * e + 1]) * p.scale);
                    uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out_dk) + rowg * D + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                } else if (rowg >= 0) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) p.dk[rowg * D + 32 * c + e] = prev[32 * cc + e] + __uint_as_float(rk[e]) * p.scale;
                }
                if (rowg >= 0) {
                    if (p.dv16) {
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = bwd_pack<F16>(__uint_as_float(rv[2 * e]), __uint_as_float(rv[2 * e + 1]));
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dv16) + rowg * D + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    }
                }
                __syncwarp();
            }
        }
    }
    __syncthreads();
    if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 24)) {
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ launches
// One CTA per (bh, problem, query tile).
template <int D, bool F16, int KIND>
__global__ void __launch_bounds__(BwdLayout<D>::THREADS, 1)
monarch_bwd_dq(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mvals, const __grid_constant__ CUtensorMap mdy,
               const BwdParams p) {
    bwd_dq_body<D, F16, KIND>(mq, mk, mvals, mdy, p, static_cast<int>(blockIdx.x));
}

// One CTA per (bh, problem, key tile).
template <int D, bool F16, int KIND>
__global__ void __launch_bounds__(BwdLayout<D>::THREADS, 1)
monarch_bwd_dkdv(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mvals, const __grid_constant__ CUtensorMap mdy,
                 const BwdParams p) {
    bwd_dkdv_body<D, F16, KIND>(mq, mk, mvals, mdy, p, static_cast<int>(blockIdx.x));
}

// Both kernels of a stage in one launch, for when the row LSE is given (the
// dk/dv CTAs then need nothing the dq CTAs write): the second kernel's CTAs
// fill the SMs the first one's last wave leaves idle.
template <int D, bool F16, int KIND>
__global__ void __launch_bounds__(BwdLayout<D>::THREADS, 1)
monarch_bwd_pair(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mvals, const __grid_constant__ CUtensorMap mdy,
                 const BwdParams p) {
    const int cta = static_cast<int>(blockIdx.x);
    if (cta < p.pair_split)
        bwd_dq_body<D, F16, KIND>(mq, mk, mvals, mdy, p, cta);
    else
        bwd_dkdv_body<D, F16, KIND>(mq, mk, mvals, mdy, p, cta - p.pair_split);
}

}  // namespace monarch
