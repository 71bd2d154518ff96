// attn_tc.cuh -- bf16 / fp16 Monarch attention stages on tcgen05 tensor cores.
//
// One persistent kernel runs "units" of block-diagonal softmax attention
// (MonarchRT: Efficient Attention for Real-Time Video Generation,
// gist.science/nl/paper/2602.12271 "Methodologie": permutation and
// block-diagonal factors; gist.science/zh/paper/2602.12271 section 2.2: blocks
// aligned with the video axes, tiled Monarch, and FlashAttention-style tiling
// in on-chip memory without materialising the dense map).
//
// A unit has two "lanes"; each lane is one 128-row query tile:
//   stage-1 lane: a query tile of one stage-1 block (a frame, or a spatial
//     tile of a frame); it iterates over that block's key/value tiles with an
//     online softmax; values are V; results (Y1) go to `out`.
//   stage-2 lane: a "group chunk" stacking npos spatial positions x T frames
//     (npos*T <= 128 rows) fetched with one TMA box, so the permutation P of
//     the factorisation is pure tensor-map addressing.  Keys are the same
//     stacked rows, a block-diagonal mask keeps each row inside its own
//     position's group, values are Y1 read back from `out`, results
//     overwrite `out`.
// The two lanes of a unit share their key/value tiles when they are two query
// tiles of the same block ("shared" units); otherwise each lane streams its
// own keys ("separate" units: the odd last query tile of two blocks, and
// every stage-2 unit).
//
// Warp roles (640 threads, registers rebalanced with setmaxnreg):
//   warps 0-3, 8-11    lane 0: softmax over S columns 0-63 / 64-127 of each
//                      row (thread = row), then O/l -> bf16 -> global for
//                      output columns [0, D/2) / [D/2, D)            104 regs
//   warps 4-7, 12-15   the same for lane 1                            104 regs
//   warp  16           TMA producer (Q tiles, K/V ring)                64 regs
//   warp  17           TMEM allocator; issues the S = Q K^T MMAs (shared-memory operands)
//   warp  18           issues the O += P V MMAs (P from tensor memory)
//   warp  19           publishes finished stage-1 lanes to stage-2 units
// (4*128*104 + 128*64 = 61440 = 640 threads x 96, the launch allocation.)
// Splitting each row over two warps puts two warps of the same lane on every
// SM sub-partition, so the exp/pack work of one tile is spread over twice the
// warps; the halves exchange their row maxima through shared memory.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0, O1 after them.
// P (bf16) overwrites the first 64 columns of its S region and feeds the PV
// MMA straight from TMEM.  Per lane i and key tile j the chain is
//   S_i(j) -> softmax_i(j) writes P_i(j) -> PV_i(j) -> S_i(j+1) -> ...
// with S_i(j+1) issued only once PV_i(j) has completed (it overwrites P_i(j));
// the two lanes' chains interleave on the tensor pipe, so one lane's softmax
// overlaps the other lane's MMAs.
#pragma once

#include "sm100.cuh"

namespace monarch {

enum : int { UNIT_STAGE1 = 1, UNIT_STAGE2 = 2 };

struct TcParams {
    int B, heads, T, H, W, HW;
    long long N;                    // tokens per (batch, head)
    int fact;                       // 0 frame, 1 tiled
    int tile_h, tile_w, tiles_h, tiles_w;
    int rows_per_tile;              // tiled: tile rows per 128-row query/key tile
    int m;                          // tokens per stage-1 block
    int sub;                        // > 0: a stage-1 block packs m / sub independent sub-blocks of
                                    // sub consecutive tokens (a query sees keys of its own one only)
    int nblk_bh;                    // stage-1 blocks per (batch, head)
    int nblocks;                    // stage-1 blocks in all
    int nqt;                        // 128-row query (= key) tiles per stage-1 block
    int ns;                         // shared pairs per block: nqt / 2
    int odd;                        // nqt % 2
    int upg;                        // units per group of two blocks: 2*ns + odd
    int npos;                       // stage-2 positions per chunk
    int s2_chunks;                  // chunks per (batch, head)
    int s2_pairs;                   // ceil(s2_chunks / 2) = stage-2 units per (batch, head)
    int BH;                         // batch x heads
    int u1_bh;                      // stage-1 units per (batch, head)
    int lag;                        // stage-2 units of bh follow the stage-1 units of bh + lag
    int units;                      // all units of the call
    // divisions by launch constants, as multiply-shift
    FastDiv fd_u1, fd_u12, fd_u2;   // u1_bh, u1_bh + s2_pairs, s2_pairs
    FastDiv fd_upg, fd_nblk_bh, fd_tpf, fd_tiles_w, fd_tile_w, fd_npos;
    unsigned *s1_done;              // per batch-head: stage-1 lanes whose Y1 rows are stored
    unsigned *work;                 // next unit to claim (zero at launch); CTAs claim units in order
    unsigned s1_target;             // stage-1 lanes per batch-head
    float scale_log2;               // d^-1/2 * log2(e)
    long long timeout_cycles;
    unsigned *status;
    void *out;                      // 16-bit output (epilogue stores)
    long long sB, sH, sN;           // element strides of batch, head and token (all four tensors)
    FastDiv fd_heads;               // batch-head index -> (batch, head)
    int out_v8;                     // out is 32-byte aligned: 32-byte epilogue stores
    float *lse;                     // or null: per output row of the units of kind lse_kind, the
    int lse_kind;                   // log2-sum-exp of its scaled logits, [BH][N] (for gradients)
};

struct Lane {
    int blk;   // stage 1: global block index; stage 2: batch-head
    int tile;  // stage 1: query tile inside the block; stage 2: chunk
};

struct Unit {
    int kind;
    int nq;      // lanes present (1 or 2)
    int nk;      // key/value tiles per lane
    int shared;  // lanes share key/value tiles
    Lane ln[2];
};

// Stage-1 unit r of batch-head bh: blocks are taken in pairs (lb0, lb0+1) of
// this batch-head; a pair's units are the shared query-tile pairs of both
// blocks, then one unit joining their odd last query tiles.
__device__ __forceinline__ Unit decode_stage1(const TcParams &p, int bh, int r) {
    Unit un;
    un.kind = UNIT_STAGE1;
    un.nk = p.nqt;
    const int g = static_cast<int>(fdiv(r, p.fd_upg)), rr = r - g * p.upg;
    const int lb0 = 2 * g;
    const bool two = lb0 + 1 < p.nblk_bh;
    const int b0 = bh * p.nblk_bh + lb0;
    if (rr < p.ns || (two && rr < 2 * p.ns)) {
        const int blk = rr < p.ns ? b0 : b0 + 1;
        const int pr = rr < p.ns ? rr : rr - p.ns;
        un.shared = 1;
        un.nq = 2;
        un.ln[0] = {blk, 2 * pr};
        un.ln[1] = {blk, 2 * pr + 1};
    } else {
        un.shared = 0;
        un.nq = two ? 2 : 1;
        un.ln[0] = {b0, p.nqt - 1};
        un.ln[1] = {two ? b0 + 1 : b0, p.nqt - 1};
    }
    return un;
}

__device__ __forceinline__ Unit decode_stage2(const TcParams &p, int bh, int r) {
    Unit un;
    un.kind = UNIT_STAGE2;
    un.nk = 1;
    un.shared = 0;
    const int c0 = 2 * r;
    un.nq = (c0 + 1 < p.s2_chunks) ? 2 : 1;
    un.ln[0] = {bh, c0};
    un.ln[1] = {bh, c0 + 1};
    return un;
}

// Unit u of the call.  Units are ordered in slots s = 0, 1, ...: slot s holds
// the stage-1 units of batch-head s (while s < BH) followed by the stage-2
// units of batch-head s - lag (once s >= lag), so a batch-head's stage-2
// units come about `lag` batch-heads of work after its stage-1 units.
__device__ __forceinline__ Unit decode_unit(const TcParams &p, int u) {
    const int U1 = p.u1_bh, U2 = p.s2_pairs;
    const int L = p.lag < p.BH ? p.lag : p.BH;
    if (u < L * U1) {
        const int s = static_cast<int>(fdiv(u, p.fd_u1));
        return decode_stage1(p, s, u - s * U1);
    }
    u -= L * U1;
    const int nB = p.BH - L;  // slots holding both kinds
    if (u < nB * (U1 + U2)) {
        const int s = static_cast<int>(fdiv(u, p.fd_u12)), r = u - s * (U1 + U2);
        if (r < U1) return decode_stage1(p, L + s, r);
        return decode_stage2(p, s, r - U1);
    }
    u -= nB * (U1 + U2);
    const int s = static_cast<int>(fdiv(u, p.fd_u2));
    return decode_stage2(p, nB + s, u - s * U2);
}

// Rows a stage-1 tile (query or key tile `tile` of a block) brings in by TMA,
// and how many of them are real tokens of the block.
__device__ __forceinline__ void s1_tile_rows(const TcParams &p, int tile, int &loaded, int &valid) {
    if (p.fact == 0) {
        loaded = 128;  // rows past the block end are zero-filled by TMA
        const int rem = p.m - tile * 128;
        valid = rem < 128 ? rem : 128;
    } else {
        loaded = p.rows_per_tile * p.tile_w;
        const int rem_rows = p.tile_h - tile * p.rows_per_tile;
        const int rows = rem_rows < p.rows_per_tile ? rem_rows : p.rows_per_tile;
        valid = rows * p.tile_w;
    }
}

// Valid key columns of key tile j of a unit, and the MMA extent covering them
// (N of the QK^T MMA and K of the PV MMA: a multiple of 16, at most 128).
__device__ __forceinline__ void key_extent(const TcParams &p, const Unit &un, int j, int &kvalid,
                                           int &ext) {
    if (un.kind == UNIT_STAGE1) {
        int loaded;
        s1_tile_rows(p, j, loaded, kvalid);
    } else {
        kvalid = p.npos * p.T;
    }
    ext = (kvalid + 15) & ~15;
}

// Issue the TMA load of one stage-1 tile (all panels) into dst.
template <int NP>
__device__ __forceinline__ void s1_load(const TcParams &p, const CUtensorMap *map, uint32_t dst,
                                        uint32_t bar, int blk, int tile) {
    if (p.fact == 0) {
        // map (d, m, T, heads, B): block blk = bh * T + t
        const int bh = static_cast<int>(fdiv(blk, p.fd_nblk_bh)), t = blk - bh * p.nblk_bh;
        const int b = static_cast<int>(fdiv(bh, p.fd_heads)), hd = bh - b * p.heads;
        for (int pn = 0; pn < NP; ++pn) tma_load_5d(dst + pn * 16384, map, bar, pn * 64, tile * 128, t, hd, b);
    } else {
        const int frame = static_cast<int>(fdiv(blk, p.fd_tpf));
        const int tif = blk - frame * p.tiles_h * p.tiles_w;
        const int ti = static_cast<int>(fdiv(tif, p.fd_tiles_w)), tj = tif - ti * p.tiles_w;
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
            tma_load_5d(dst + pn * 16384, map, bar, pn * 64, 0, tj, tile * p.rows_per_tile,
                        frame * p.tiles_h + ti);
    }
}

template <int NP>
__device__ __forceinline__ void s2_load(const TcParams &p, const CUtensorMap *map, uint32_t dst, uint32_t bar,
                                        int bh, int chunk) {
    // map (d, H*W, T, heads, B)
    const int b = static_cast<int>(fdiv(bh, p.fd_heads)), hd = bh - b * p.heads;
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) tma_load_5d(dst + pn * 16384, map, bar, pn * 64, chunk * p.npos, 0, hd, b);
}

// Output token (index inside its batch-head) of row `row` of a lane, or -1
// when the row is padding.  bh receives the lane's batch-head.
__device__ __forceinline__ long long lane_row_token(const TcParams &p, int kind, const Lane &ln, int row,
                                                    int &bh) {
    if (kind == UNIT_STAGE1) {
        bh = static_cast<int>(fdiv(ln.blk, p.fd_nblk_bh));
        const int b = ln.blk - bh * p.nblk_bh;
        if (p.fact == 0) {
            const int i = ln.tile * 128 + row;
            if (i >= p.m) return -1;
            return static_cast<long long>(b) * p.HW + i;
        }
        const int t = static_cast<int>(fdiv(b, p.fd_tpf)), tif = b - t * p.tiles_h * p.tiles_w;
        const int ti = static_cast<int>(fdiv(tif, p.fd_tiles_w)), tj = tif - ti * p.tiles_w;
        const int rr = static_cast<int>(fdiv(row, p.fd_tile_w)), wl = row - rr * p.tile_w;
        const int hl = ln.tile * p.rows_per_tile + rr;
        if (rr >= p.rows_per_tile || hl >= p.tile_h) return -1;
        return static_cast<long long>(t) * p.HW + static_cast<long long>(ti * p.tile_h + hl) * p.W +
               tj * p.tile_w + wl;
    }
    bh = ln.blk;
    const int t = static_cast<int>(fdiv(row, p.fd_npos)), pl = row - t * p.npos;
    const int pos = ln.tile * p.npos + pl;
    if (t >= p.T || pos >= p.HW) return -1;
    return static_cast<long long>(t) * p.HW + pos;
}

// Bit c set when column c of a 64-column half holds a valid key: stage 1,
// the first n columns; stage 2, the columns of the row's own position slot
// (column 64h + c holds position slot (64h + c) % npos of frame (64h + c) / npos).
__device__ __forceinline__ uint64_t stage1_valid_bits(int n) {
    return n >= 64 ? ~0ull : (n <= 0 ? 0ull : ((1ull << n) - 1ull));
}
// Bit c set when column c of the 64-column half h of key tile j lies in the
// sub-block of block-local query qi (packed blocks: keys [g*sub, g*sub+sub)
// with g = qi / sub).
__device__ __forceinline__ uint64_t sub_valid_bits(int g_lo, int sub, int j, int h) {
    const int lo = g_lo - (j * 128 + 64 * h), hi = lo + sub;
    const uint64_t below_hi = hi >= 64 ? ~0ull : (hi <= 0 ? 0ull : ((1ull << hi) - 1ull));
    const uint64_t below_lo = lo >= 64 ? ~0ull : (lo <= 0 ? 0ull : ((1ull << lo) - 1ull));
    return below_hi & ~below_lo;
}
__device__ __noinline__ uint64_t stage2_valid_bits(const TcParams &p, int h, int prow, int npos_valid) {
    uint64_t vm = 0;
    if (prow >= npos_valid) return 0;
    // first column >= 64h in slot prow, then every npos columns up to frame T-1
    int c = prow - 64 * h;
    if (c < 0) c += ((-c + p.npos - 1) / p.npos) * p.npos;
    for (; c < 64 && 64 * h + c < p.npos * p.T; c += p.npos) vm |= 1ull << c;
    return vm;
}

template <int D>
struct TcLayout {
    static constexpr int NP = D / 64;                 // 64-element (128-byte) panels per row
    static constexpr int TILE = 128 * D * 2;          // bytes of one 128-row tile
    static constexpr int NS = (D == 128) ? 5 : 8;     // K/V ring slots
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + 2 * TILE;
    static constexpr int OFF_BAR = OFF_KV + NS * TILE;
    // Claimed unit indices, passed from the TMA producer (which claims them)
    // to the other roles through a ring of NUQ slots.
    static constexpr int NUQ = 8;
    // roles reading each slot: the two MMA issuers, the Y1 publisher and the
    // 16 softmax warps
    static constexpr int UQ_READERS = 19;
    // barriers: q_full[2] q_empty[2] kv_full[NS] kv_empty[NS] s_full[2] p_full[2]
    //           o_full[2] o_free[2] y_done[2] y_free[2] pv_done[2] uq_full[NUQ] uq_empty[NUQ]
    static constexpr int NBAR = 18 + 2 * NS + 2 * NUQ;
    // exchange of per-row values (row maxima, row sums) between the two column
    // halves of a lane: [2 lanes][128 rows] fp32
    static constexpr int OFF_X = OFF_BAR + NBAR * 8;
    static constexpr int OFF_UQ = OFF_X + 2 * 128 * 4;
    static constexpr int OFF_MISC = OFF_UQ + NUQ * 4;  // tmem base, abort flag
    static constexpr int BYTES = OFF_MISC + 16;
    // The dynamic shared-memory base is at least 256-byte aligned; up to 768
    // bytes of slack realign it to the 1024 bytes the 128-byte swizzle needs.
    static constexpr int SLACK = 768;
    static constexpr int ALLOC = BYTES + SLACK;
    static_assert(ALLOC <= 232448, "exceeds the 227 KB of shared memory a block may use");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
};

// Zero rows [from, to) of every panel of a 128-row tile (generic proxy), so
// that the PV MMA reads exact zeros where no value row was loaded.
template <int NP>
__device__ __forceinline__ void zero_rows(uint32_t tile, int from, int to) {
    for (int r = from; r < to; ++r)
#pragma unroll
        for (int pn = 0; pn < NP; ++pn)
#pragma unroll
            for (int c = 0; c < 8; ++c) st_shared_v4(tile + pn * 16384 + r * 128 + c * 16, 0, 0, 0, 0);
}

__device__ __forceinline__ void setmaxnreg_inc104() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 104;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec64() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
}

// ---------------------------------------------------------------- softmax math

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packs two fp32 values into the kernel's 16-bit input format (fp16 or bf16).
template <bool F16>
__device__ __forceinline__ uint32_t pack_in(float lo, float hi) {
    if constexpr (F16)
        return pack_f16x2(lo, hi);
    else
        return pack_bf16x2(lo, hi);
}

// The two 16-bit values of a packed pair, widened (exactly) to fp32 and
// returned as one packed fp32 pair.  A bf16 value is the high half of its
// fp32 value, so widening it is a shift or a mask.
template <bool F16>
__device__ __forceinline__ uint64_t unpack_in(uint32_t w) {
    if constexpr (F16) {
        float lo, hi;
        asm("{\n\t.reg .b16 l, h;\n\t"
            "mov.b32 {l, h}, %2;\n\t"
            "cvt.f32.f16 %0, l;\n\t"
            "cvt.f32.f16 %1, h;\n\t}"
            : "=f"(lo), "=f"(hi)
            : "r"(w));
        return pack_f32x2(lo, hi);
    } else {
        return pack_f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
}

// Exponentiate and pack one 32-column chunk: x = s*sl2 - moff, P = 2^x as
// 16-bit pairs, and accumulate P into two packed fp32 partial sums (even and
// odd pairs, so the additions form two independent chains).

template <int C, bool F16>
__device__ __forceinline__ void softmax_chunk(const float (&s)[64], uint64_t scale, uint64_t off,
                                              uint32_t (&pk)[16], uint64_t &acc0, uint64_t &acc1) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const uint64_t x = fma_f32x2(pack_f32x2(s[32 * C + 2 * e], s[32 * C + 2 * e + 1]), scale, off);
        float x0, x1, a, b;
        unpack_f32x2(x, x0, x1);
        a = fast_exp2(x0);
        b = fast_exp2(x1);
        const uint32_t w = pack_in<F16>(a, b);
        pk[e] = w;
        // the denominator sums the rounded weights the PV MMA multiplies, so
        // each row's effective weights add up to one
        const uint64_t r = unpack_in<F16>(w);
        if (e & 1)
            acc1 = add_f32x2(acc1, r);
        else
            acc0 = add_f32x2(acc0, r);
    }
}

// Instantiations: TC_PLAIN; TC_PACK, stage-1 blocks pack sub-blocks of p.sub
// tokens (the packed rows pass of the (f*h, w) split); TC_LSE, the row LSE of
// the units of kind p.lse_kind is written to p.lse (the recomputations of the
// gradients).  Separate instantiations, so the plain kernel carries neither.
enum : int { TC_PLAIN = 0, TC_PACK = 1, TC_LSE = 2 };
template <int D, bool F16, int MODE>
__global__ void __launch_bounds__(640, 1)
monarch_tc_kernel(const __grid_constant__ CUtensorMap mq1, const __grid_constant__ CUtensorMap mk1,
                  const __grid_constant__ CUtensorMap mv1, const __grid_constant__ CUtensorMap mq2,
                  const __grid_constant__ CUtensorMap mk2, const __grid_constant__ CUtensorMap my2,
                  const TcParams p) {
    using L = TcLayout<D>;
    constexpr int NP = L::NP;
    constexpr int NS = L::NS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);
    if (base - raw > static_cast<uint32_t>(L::SLACK)) {  // uniform over the block
        if (threadIdx.x == 0) atomicOr(p.status, DEVERR_ALIGN);
        return;
    }

    const uint32_t bar0 = base + L::OFF_BAR;
    auto q_full = [&](int i) { return bar0 + 8u * i; };
    auto q_empty = [&](int i) { return bar0 + 8u * (2 + i); };
    auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (4 + NS + s); };
    auto s_full = [&](int i) { return bar0 + 8u * (4 + 2 * NS + i); };
    auto p_full = [&](int i) { return bar0 + 8u * (6 + 2 * NS + i); };
    auto o_full = [&](int i) { return bar0 + 8u * (8 + 2 * NS + i); };
    auto o_free = [&](int i) { return bar0 + 8u * (10 + 2 * NS + i); };
    auto y_done = [&](int i) { return bar0 + 8u * (12 + 2 * NS + i); };
    auto y_free = [&](int i) { return bar0 + 8u * (14 + 2 * NS + i); };
    auto pv_done = [&](int i) { return bar0 + 8u * (16 + 2 * NS + i); };
    auto uq_full = [&](int k) { return bar0 + 8u * (18 + 2 * NS + k); };
    auto uq_empty = [&](int k) { return bar0 + 8u * (18 + 2 * NS + L::NUQ + k); };
    volatile int *uq = reinterpret_cast<volatile int *>(base_ptr + L::OFF_UQ);
    float *x_buf = reinterpret_cast<float *>(base_ptr + L::OFF_X);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + L::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(base_ptr + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    WaitCtl ctl{abort_flag, p.status, p.timeout_cycles};

    // The k-th unit this CTA runs: the producer claims units from the global
    // counter in order and posts them in the ring; every other role takes
    // them from it in the same order (a single thread, or the 32 lanes of a
    // softmax warp, of which lane 0 frees the slot).  u = -1: no more units.
    // Returns false when the wait gave up.
    auto take_unit = [&](int k, int &u, bool whole_warp) -> bool {
        const int slot = k % L::NUQ;
        const uint32_t par = static_cast<uint32_t>(k / L::NUQ) & 1u;
        const bool got = whole_warp ? mbar_wait_warp(uq_full(slot), par, ctl) : mbar_wait(uq_full(slot), par, ctl);
        if (!got) return false;
        u = uq[slot];
        if (whole_warp) __syncwarp();
        if (!whole_warp || (threadIdx.x & 31) == 0) mbar_arrive(uq_empty(slot));
        return true;
    };

    if (threadIdx.x == 0) {
        *abort_flag = 0u;
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 1);
            mbar_init(q_empty(i), 1);
            mbar_init(s_full(i), 1);
            mbar_init(p_full(i), 256);
            mbar_init(o_full(i), 1);
            mbar_init(o_free(i), 256);
            mbar_init(y_done(i), 256);
            mbar_init(y_free(i), 1);
            mbar_init(pv_done(i), 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int k = 0; k < L::NUQ; ++k) {
            mbar_init(uq_full(k), 1);
            mbar_init(uq_empty(k), L::UQ_READERS);
        }
        fence_barrier_init();
    }
    if (warp == 16 && lane == 0) {
        tma_prefetch_desc(&mq1); tma_prefetch_desc(&mk1); tma_prefetch_desc(&mv1);
        tma_prefetch_desc(&mq2); tma_prefetch_desc(&mk2); tma_prefetch_desc(&my2);
    }
    if (warp == 17) {
        tmem_alloc(smem_addr(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (wg == 4) {
        setmaxnreg_dec64();
        if (warp == 19 && lane == 0) {
            // ------------------------------------------------------ Y1 publisher
            // Once the 256 threads of a stage-1 lane have stored its Y1 rows
            // (y_done), make them visible at GPU scope and count the lane for
            // its batch-head; stage-2 units acquire that count.  Kept off the
            // softmax warps so the fence latency is not on their path.
            uint32_t yd_par = 0u;  // bit i: parity to wait for on y_done(i)
            bool ok = true;
            for (int k = 0; ok; ++k) {
                int u;
                if (!take_unit(k, u, false)) break;
                if (u < 0) break;
                const Unit un = decode_unit(p, u);
                if (un.kind != UNIT_STAGE1) continue;
                for (int i = 0; i < un.nq && ok; ++i) {
                    ok = mbar_wait(y_done(i), (yd_par >> i) & 1u, ctl);
                    yd_par ^= 1u << i;
                    if (!ok) break;
                    __threadfence();
                    atomicAdd(p.s1_done + fdiv(un.ln[i].blk, p.fd_nblk_bh), 1u);
                    mbar_arrive(y_free(i));
                }
            }
        }
        if (warp == 16 && lane == 0) {
            // -------------------------------------------------------- TMA producer
            // Load order per unit: Q of each lane, then per key tile j the K
            // tile(s) then the V tile(s): one K and one V for a shared unit,
            // K_A, K_B, V_A, V_B for a separate one.  The MMA issuer consumes
            // the ring in exactly this order.
            // Units are claimed one ahead (the atomic's latency overlaps the
            // current unit's loads) and posted in the ring before their loads.
            uint32_t qe_par = 3u;  // bit i: parity to wait for on q_empty(i)
            int slot = 0;
            uint32_t kv_round = 0;
            bool ok = true;
            unsigned next = atomicAdd(p.work, 1u);
            for (int k = 0; ok; ++k) {
                const int u = next < static_cast<unsigned>(p.units) ? static_cast<int>(next) : -1;
                const int qs = k % L::NUQ;
                ok = mbar_wait(uq_empty(qs), (static_cast<uint32_t>(k / L::NUQ) & 1u) ^ 1u, ctl);
                if (!ok) break;
                uq[qs] = u;
                mbar_arrive(uq_full(qs));
                if (u < 0) break;
                next = atomicAdd(p.work, 1u);
                const Unit un = decode_unit(p, u);
#pragma unroll 1
                for (int i = 0; i < un.nq && ok; ++i) {
                    ok = mbar_wait(q_empty(i), (qe_par >> i) & 1u, ctl);
                    qe_par ^= 1u << i;
                    if (!ok) break;
                    const Lane ln = i ? un.ln[1] : un.ln[0];
                    const uint32_t dst = base + L::OFF_Q + i * L::TILE;
                    if (un.kind == UNIT_STAGE1) {
                        int loaded, valid;
                        s1_tile_rows(p, ln.tile, loaded, valid);
                        mbar_arrive_expect_tx(q_full(i), NP * loaded * 128);
                        s1_load<NP>(p, &mq1, dst, q_full(i), ln.blk, ln.tile);
                    } else {
                        mbar_arrive_expect_tx(q_full(i), NP * p.npos * p.T * 128);
                        s2_load<NP>(p, &mq2, dst, q_full(i), ln.blk, ln.tile);
                    }
                }
                const int nkv = un.shared ? 1 : un.nq;
                int loaded = p.npos * p.T;
#pragma unroll 1
                for (int j = 0; j < un.nk && ok; ++j) {
                    int kvalid, ext;
                    key_extent(p, un, j, kvalid, ext);
                    if (un.kind == UNIT_STAGE1) {
                        int valid;
                        s1_tile_rows(p, j, loaded, valid);
                    }
#pragma unroll 1
                    for (int t = 0; t < 2 * nkv && ok; ++t) {
                        const bool is_v = t >= nkv;
                        const Lane ln = (t % nkv) ? un.ln[1] : un.ln[0];
                        // stage 2 reads Y1 rows that stage-1 lanes of this
                        // batch-head (on any SM) stored with plain stores: wait
                        // until all have published (acquire), then order the
                        // TMA reads after that
                        if (t == nkv && un.kind == UNIT_STAGE2) {
                            ok = wait_counter(p.s1_done + ln.blk, p.s1_target, ctl);
                            if (!ok) break;
                            fence_proxy_async_global();
                        }
                        const int s = slot;
                        ok = mbar_wait(kv_empty(slot), (kv_round & 1u) ^ 1u, ctl);
                        if (++slot == NS) { slot = 0; ++kv_round; }
                        if (!ok) break;
                        const uint32_t dst = base + L::OFF_KV + s * L::TILE;
                        if (is_v && loaded < ext) {  // rows the PV MMA reads but TMA does not write
                            zero_rows<NP>(dst, loaded, ext);
                            fence_proxy_async_smem();
                        }
                        mbar_arrive_expect_tx(kv_full(s), NP * loaded * 128);
                        if (un.kind == UNIT_STAGE1)
                            s1_load<NP>(p, is_v ? &mv1 : &mk1, dst, kv_full(s), ln.blk, j);
                        else
                            s2_load<NP>(p, is_v ? &my2 : &mk2, dst, kv_full(s), ln.blk, ln.tile);
                    }
                }
            }
        } else if ((warp == 17 || warp == 18) && lane == 0) {
            // -------------------------------------------------------- MMA issuers
            // Warp 17 issues every S = Q K^T MMA (both operands in shared
            // memory), warp 18 every O += P V MMA (P in tensor memory).  One
            // thread cannot issue a lane pair's 32 MMAs per key step plus its
            // barrier traffic as fast as the tensor pipe runs them; two threads
            // can, as long as one of them issues all the TMEM-operand MMAs (the
            // pipe serialises those when two threads interleave them).
            // S_i of a key tile overwrites the S/P region that PV_i of the
            // previous tile reads, so the S issuer waits for that PV's
            // completion (pv_done, committed after every PV).  Both issuers walk
            // the K/V ring in load order; each waits for and releases only its
            // own tiles (K tiles: S issuer, V tiles: PV issuer).
            const bool s_role = warp == 17;
            uint32_t qf_par = 0u;   // bit i: parity to wait for on q_full(i)
            uint32_t pd_par = 3u;   // bit i: parity to wait for on pv_done(i) (the first S passes)
            uint32_t pf_par = 0u;   // bit i: parity to wait for on p_full(i)
            uint32_t of_par = 3u;   // bit i: parity to wait for on o_free(i)
            int slot = 0;
            uint32_t kv_round = 0;
            bool ok = true;
            // Descriptor halves: the low word holds the start address, so
            // every K step below is a single 32-bit add of a constant.
            constexpr uint32_t KM_HI = sdesc_sw128_hi(1024);  // K-major: 8-row groups 1024 B apart
            constexpr uint32_t MN_HI = sdesc_sw128_hi(1024);  // MN-major V: 8-key groups 1024 B apart
            const uint32_t q_lo0 = sdesc_sw128_lo(base + L::OFF_Q, 16);
            const uint32_t kv_lo0 = sdesc_sw128_lo(base + L::OFF_KV, 16);
            const uint32_t v_lo0 = sdesc_sw128_lo(base + L::OFF_KV, 16384);  // D panels 16 KB apart
            constexpr uint32_t TILE16 = L::TILE >> 4;
            constexpr uint32_t IDESC_O = F16 ? idesc_f16_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
            for (int k = 0; ok; ++k) {
                int u;
                if (!take_unit(k, u, false)) break;
                if (u < 0) break;
                const Unit un = decode_unit(p, u);
                if (s_role) {
#pragma unroll 1
                    for (int i = 0; i < un.nq && ok; ++i) {
                        ok = mbar_wait(q_full(i), (qf_par >> i) & 1u, ctl);
                        qf_par ^= 1u << i;
                    }
                    if (!ok) break;
                }
                const int nkv = un.shared ? 1 : un.nq;  // K (or V) tiles per key step
#pragma unroll 1
                for (int j = 0; j < un.nk && ok; ++j) {
                    int kvalid, ext;
                    key_extent(p, un, j, kvalid, ext);
                    // ring slots in load order: K(j) tile(s), then V(j) tile(s);
                    // wait for this role's own ones
                    int s0 = 0, s1 = 0;
#pragma unroll 1
                    for (int t = 0; t < 2 * nkv && ok; ++t) {
                        const bool mine = (t < nkv) == s_role;
                        const int s = slot;
                        if (mine) ok = mbar_wait(kv_full(slot), kv_round & 1u, ctl);
                        if (++slot == NS) { slot = 0; ++kv_round; }
                        if (mine) {
                            if ((t % nkv) == 0) s0 = s1 = s; else s1 = s;
                        }
                    }
                    if (!ok) break;
                    if (s_role) {
                        const uint32_t idesc_s = F16 ? idesc_f16_f32(128, ext, false, false) : idesc_bf16_f32(128, ext, false, false);
#pragma unroll 1
                        for (int i = 0; i < un.nq && ok; ++i) {
                            // the PV that last read this lane's S/P region has completed
                            ok = mbar_wait(pv_done(i), (pd_par >> i) & 1u, ctl);
                            pd_par ^= 1u << i;
                            if (!ok) break;
                            tc_fence_after();
                            // S_i = Q_i K^T: A = Q tile (K-major), B = K tile (K-major), K dim = D
                            const uint32_t a = q_lo0 + i * TILE16;
                            const uint32_t b = kv_lo0 + (i ? s1 : s0) * TILE16;
                            const uint32_t d_tmem = tmem + (i ? L::COL_S1 : L::COL_S0);
                            mma_ss_lh<0>(d_tmem, a, KM_HI, b, KM_HI, idesc_s);
#pragma unroll
                            for (int k = 1; k < D / 16; ++k) {
                                const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                                mma_ss_lh<1>(d_tmem, a + off, KM_HI, b + off, KM_HI, idesc_s);
                            }
                            mma_commit(s_full(i));
                        }
                        if (!ok) break;
                        mma_commit(kv_empty(s0));
                        if (nkv == 2) mma_commit(kv_empty(s1));
                        if (j == un.nk - 1)
                            for (int i = 0; i < un.nq; ++i) mma_commit(q_empty(i));
                    } else {
                        const int npv = ext >> 4;
#pragma unroll 1
                        for (int i = 0; i < un.nq && ok; ++i) {
                            // the first PV of a unit overwrites O_i: the epilogue must be done with it
                            if (j == 0) {
                                ok = mbar_wait(o_free(i), (of_par >> i) & 1u, ctl);
                                of_par ^= 1u << i;
                                if (!ok) break;
                            }
                            ok = mbar_wait(p_full(i), (pf_par >> i) & 1u, ctl);
                            pf_par ^= 1u << i;
                            if (!ok) break;
                            tc_fence_after();
                            // O_i (+)= P_i V: A = P from TMEM (bf16 pairs in the S region),
                            // B = V tile (MN-major: keys x D), K dim = ext keys; unrolled
                            // with constant offsets (the issuing thread is latency-bound)
                            const uint32_t b = v_lo0 + (i ? s1 : s0) * TILE16;
                            const uint32_t p_tmem = tmem + (i ? L::COL_S1 : L::COL_S0);
                            const uint32_t d_tmem = tmem + (i ? L::COL_O1 : L::COL_O0);
                            mma_ts_lh(d_tmem, p_tmem, b, MN_HI, IDESC_O, j > 0 ? 1u : 0u);
#pragma unroll
                            for (int k = 1; k < 8; ++k)
                                if (k < npv) mma_ts_lh(d_tmem, p_tmem + k * 8, b + k * 128, MN_HI, IDESC_O, 1u);
                            mma_commit(pv_done(i));
                            if (j == un.nk - 1) mma_commit(o_full(i));
                        }
                        if (!ok) break;
                        mma_commit(kv_empty(s0));
                        if (nkv == 2) mma_commit(kv_empty(s1));
                    }
                }
            }
        }
    } else {
        setmaxnreg_inc104();
        // ------------------------------------------------------------ softmax + epilogue
        // warpgroup wg: lane li = wg & 1 (query tile of the unit), column
        // half h = wg >> 1 (S columns [64h, 64h+64), O columns [h*D/2, (h+1)*D/2))
        const int li = wg & 1, h = wg >> 1;
        const int row = threadIdx.x & 127;  // TMEM lane == tile row
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t col_s = li ? L::COL_S1 : L::COL_S0;
        const uint32_t col_o = li ? L::COL_O1 : L::COL_O0;
        const float sl2 = p.scale_log2;
        uint32_t sf_par = 0u, of_par = 0u, yf_par = 1u;
        bool ok = true;
        // Combines a per-row value of the two column halves of the lane (the
        // maximum, or the sum), both halves getting the same result.  Only the
        // two warps holding the same 32 rows (one per half) take part, through
        // named barrier `pair_bar` (64 threads): half 0 posts its value, half
        // 1 combines and posts the result, half 0 reads it.  Half 0 writes the
        // next value only after reading the result, which half 1 posted before
        // the second barrier, so one slot per row suffices.
        float *xb = x_buf + li * 128;
        const uint32_t pair_bar = 1u + static_cast<uint32_t>(li * 4 + (warp & 3));
        auto combine = [&](float v, bool is_max) -> float {
            if (h == 0) xb[row] = v;
            named_barrier_sync(pair_bar, 64);
            if (h == 1) {
                const float o = xb[row];
                v = is_max ? fmaxf(o, v) : o + v;
                xb[row] = v;
            }
            named_barrier_sync(pair_bar, 64);
            if (h == 0) v = xb[row];
            return v;
        };
        for (int k = 0; ok; ++k) {
            int u;
            if (!take_unit(k, u, true)) break;
            if (u < 0) break;
            const Unit un = decode_unit(p, u);
            if (li >= un.nq) continue;
            float m_run = -INFINITY;  // running max of raw logits (whole row)
            float l_half = 0.f;       // softmax denominator over this half's columns
            // stage-2 mask: the row belongs to position slot prow of its chunk
            const int prow = (un.kind == UNIT_STAGE2) ? static_cast<int>(fmod_(row, p.fd_npos)) : 0;
            int npos_valid = 0;
            // packed stage-1 blocks: the first key of this row's sub-block
            constexpr bool PACK = MODE == TC_PACK;
            const int sub_lo = (PACK && un.kind == UNIT_STAGE1)
                                   ? ((un.ln[li].tile * 128 + row) / p.sub) * p.sub : 0;
            if (un.kind == UNIT_STAGE2) {
                const int rem = p.HW - un.ln[li].tile * p.npos;
                npos_valid = rem < p.npos ? rem : p.npos;
            }
            for (int j = 0; j < un.nk; ++j) {
                int kvalid, ext;
                key_extent(p, un, j, kvalid, ext);
                const bool masked = (un.kind == UNIT_STAGE2) || (kvalid < 128) || PACK;
                if (!mbar_wait_warp(s_full(li), sf_par, ctl)) { ok = false; break; }
                sf_par ^= 1u;
                tc_fence_after();
                float s[64];
                {
                    uint32_t r[2][32];
                    tmem_ld32(lane_base + col_s + 64 * h, r[0]);
                    tmem_ld32(lane_base + col_s + 64 * h + 32, r[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(r[c][e]);
                }
                if (masked) {  // columns 64h + c: validity bits, then -inf where 0
                    uint64_t vm = un.kind == UNIT_STAGE1
                                      ? stage1_valid_bits(kvalid - 64 * h)
                                      : stage2_valid_bits(p, h, prow, npos_valid);
                    if constexpr (PACK)
                        if (un.kind == UNIT_STAGE1) vm &= sub_valid_bits(sub_lo, p.sub, j, h);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (!((vm >> c) & 1ull)) s[c] = -INFINITY;
                }
                float mx;
                {
                    float m0 = fmaxf(s[0], s[1]), m1 = fmaxf(s[2], s[3]);
                    float m2 = fmaxf(s[4], s[5]), m3 = fmaxf(s[6], s[7]);
#pragma unroll
                    for (int c = 8; c < 64; c += 8) {
                        m0 = max3(m0, s[c], s[c + 1]);
                        m1 = max3(m1, s[c + 2], s[c + 3]);
                        m2 = max3(m2, s[c + 4], s[c + 5]);
                        m3 = max3(m3, s[c + 6], s[c + 7]);
                    }
                    mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
                }
                // The row max spans both halves.  Tile 0 exchanges it; later
                // tiles keep the running max unless some row of the warp pair
                // grew by more than 2^8 (one OR-barrier tells), and only then
                // exchange partial maxima and rescale O.
                bool rescale = false;
                float alpha = 1.f;
                if (j == 0) {
                    m_run = combine(mx, true);
                } else if (named_barrier_or(pair_bar, 64, (mx - m_run) * sl2 > 8.f)) {
                    mx = combine(mx, true);
                    if ((mx - m_run) * sl2 > 8.f) {
                        alpha = fast_exp2((m_run - mx) * sl2);
                        m_run = mx;
                        l_half *= alpha;
                        rescale = true;
                    }
                }
                const float moff = (m_run == -INFINITY) ? 0.f : m_run * sl2;
                uint64_t acc0 = pack_f32x2(0.f, 0.f), acc1 = acc0;
                const uint64_t scale2 = pack_f32x2(sl2, sl2);
                const uint64_t off2 = pack_f32x2(-moff, -moff);
                // P = 2^(s*sl2 - m*sl2) as bf16 pairs: this half's 64 keys go to
                // packed columns [32h, 32h+32) of the lane's S region
                {
                    uint32_t pk[16];
                    softmax_chunk<0, F16>(s, scale2, off2, pk, acc0, acc1);  // masked: 2^-inf = 0
                    tmem_st16(lane_base + col_s + 32 * h, pk);
                    softmax_chunk<1, F16>(s, scale2, off2, pk, acc0, acc1);
                    tmem_st16(lane_base + col_s + 32 * h + 16, pk);
                }
                {
                    float a0, a1, b0, b1;
                    unpack_f32x2(acc0, a0, a1);
                    unpack_f32x2(acc1, b0, b1);
                    l_half += (a0 + a1) + (b0 + b1);
                }
                // O from earlier key tiles is complete here (S_i(j) was issued
                // after PV_i(j-1) completed); rescale this half's columns before PV_i(j)
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t r[32];
                        const uint32_t a = lane_base + col_o + h * (D / 2) + 32 * c;
                        tmem_ld32(a, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(a, r);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full(li));
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            // row sum over both halves, then O / l for this half's columns
            const float l = combine(l_half, false);
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            int bh;
            const long long tok = lane_row_token(p, un.kind, un.ln[li], row, bh);
            // log2 sum_k 2^(s_k * sl2) = m * sl2 + log2(l) for any running max m
            if (MODE == TC_LSE && un.kind == p.lse_kind && h == 0 && tok >= 0)
                p.lse[static_cast<long long>(bh) * p.N + tok] = m_run * sl2 + __log2f(l);
            const int ob = static_cast<int>(fdiv(static_cast<uint32_t>(bh), p.fd_heads)), oh = bh - ob * p.heads;
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + ob * p.sB + oh * p.sH +
                                                   (tok < 0 ? 0 : tok) * p.sN + h * (D / 2));
            if (!mbar_wait_warp(o_full(li), of_par, ctl)) { ok = false; break; }
            of_par ^= 1u;
            tc_fence_after();
            // read this half's O columns, then release O at once: the next
            // unit's first PV may overwrite it while these rows are stored
            uint32_t r[D / 2];
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_ld32(lane_base + col_o + h * (D / 2) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(o_free(li));
            if (tok >= 0) {
                // pack and store 16 columns at a time (fewer live registers)
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w[e] = pack_in<F16>(__uint_as_float(r[16 * q + 2 * e]) * inv_l,
                                            __uint_as_float(r[16 * q + 2 * e + 1]) * inv_l);
                    if (p.out_v8) {  // 32-byte stores: each fills a whole sector
                        st_global_v8(dst + 2 * q, w);
                    } else {
                        dst[2 * q] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[2 * q + 1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
            if (un.kind == UNIT_STAGE1) {
                // Y1 rows stored: hand them to the publisher (one-slot
                // handshake, so y_done never runs a phase ahead of it)
                if (!mbar_wait(y_free(li), yf_par, ctl)) { ok = false; break; }
                yf_par ^= 1u;
                mbar_arrive(y_done(li));
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
    if (warp == 17) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace monarch
