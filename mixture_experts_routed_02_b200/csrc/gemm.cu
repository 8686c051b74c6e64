// gemm.cu -- persistent grouped GEMM on the sm_100a tensor cores (tcgen05 +
// TMEM + TMA) for both stages of the routed expert FFN (rocketrecap.com
// "FlyDSL kernels in JAX", paragraph 2 and timestamp 5:56: group GEMM with
// w1/w3 fused with SwiGLU, then group GEMM with w2 fused with the scatter).
//
// Row space: the expert-padded layout built by the router -- expert e owns
// whole 128-row tiles, so a tile never straddles two experts and its weight
// operand is one expert's matrix.  A tile is (m-tile, n-tile, K split).
//
// Stage 1: D[128 x BN] = Xs[128 rows, H] * W13_e[BN rows, H]^T.  W13 holds w1
//   and w3 rows interleaved in blocks of 32, so accumulator columns [64g, 64g+32)
//   are gate channels and [64g+32, 64g+64) the matching up channels.  Epilogue:
//   (FP8: scale by sx[row] * s13[col]) -> h = silu(g) * u -> bf16 -> (FP8:
//   e4m3 with one power-of-two scale per 32 channels) -> h.
// Stage 2: D[128 x BN] = H[128 rows, F] * W2_e[BN rows, F]^T; FP8 uses the
//   block-scaled MMA with h's per-32 scales (w2's are 1) and applies s2 in the
//   epilogue.  Epilogue: scale by the routing weight, fp32 atomic add into the
//   token's row of the combine buffer (which also makes K splits free).
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into an NST-deep
// shared-memory ring; warp 1 owns TMEM and lane 0 issues the MMAs; warps 2..5
// drain the TMEM accumulators (double buffered where TMEM has room, so the
// epilogue of one tile overlaps the main loop of the next; the block-scaled
// FP8 second GEMM, whose single accumulator leaves TMEM room only for the
// scales, runs warps 2..9 (320 threads) instead and frees the accumulator
// before its atomics).  With MX FP4 weights warps 6 and 7 (256 threads)
// spread each stage's packed weight rows into the 4-bit operand form before
// the stage counts as full.
//
// CTA pairs (PAIR): a cluster of two CTAs on two SMs computes a 256 x BN tile
// with tcgen05.mma.cta_group::2.  Its two 128-row halves are two m-tiles of
// the same expert (the second one repeats the first when the expert has an odd
// number of m-tiles; that half's results are discarded).  Each CTA loads its
// own 128 activation rows and one half of the BN weight rows, so per unit of
// work a CTA moves a third less operand data through L2 and shared memory
// than a 128 x BN tile on one SM; the even CTA issues the MMAs and every
// operand load of the pair completes on its barriers.
#include "kernels.cuh"

namespace moe {

namespace {

template <int STAGE, bool FP8, int BN, int NST, int NACC, bool PAIR, int AR, bool MXW>
struct Cfg {
    // Block-scaled MMA (kind::mxf8f6f4, one UE8M0 scale per 32 K elements of
    // every row of A and B): stage 2 in FP8 (h carries per-32 scales; w2's
    // are 1), and both stages with MX FP4 weights (MXW: e2m1 weights with
    // their own per-32 scales; stage 1's activation scales are 1, the per-token
    // scale is applied in the epilogue).
    static constexpr bool MX = ((STAGE == 2) && FP8) || MXW;
    static constexpr bool SFA_VAR = MX && STAGE == 2;  // A scales copied per stage (h's)
    static constexpr bool SFB_VAR = MXW;               // B scales copied per stage (the weights')
    static constexpr bool HAS_SFC = MX && !(SFA_VAR && SFB_VAR);  // a constant all-ones scale block
    static_assert(!MXW || (FP8 && !PAIR), "MX FP4 weights: e4m3 activations, one-CTA tiles");
    // activation rows copied per stage: 128, or 32 when no m-tile holds more
    // than 32 rows in use (the MMA still reads 128 rows from the stage's
    // address; rows 32-127 then alias the next buffers and belong to padding
    // rows, whose results are discarded)
    static constexpr int A_BYTES = AR * 128;
    static_assert(AR == kBlockM || (AR == 32 && !PAIR), "activation rows per stage");
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // weight rows held by one CTA
    static constexpr int B_BYTES = B_ROWS * 128;       // shared memory (e2m1: every 16 codes in 16 bytes)
    // MX FP4 weights come in packed (two codes per byte, 64 bytes a row) into a
    // staging ring that completes on its own barriers; two converter warps
    // then write every 16 codes into 16 bytes of the operand (8 bytes of
    // codes, 8 of padding: the 4-bit operand form of the block-scaled MMA) and
    // arrive on the stage's full barrier.  So B adds no bytes to it.
    static constexpr int B_ROW_TX = MXW ? 0 : 128;
    static constexpr int STG_BYTES = MXW ? B_ROWS * 64 : 0;
    static constexpr int NCONV = MXW ? 2 : 0;               // converter warps (6, 7)
    // epilogue warps: 4 (one per TMEM lane quarter), or 8 for the block-scaled
    // second GEMM with its single accumulator (two warps per lane quarter,
    // each with half the columns in registers, so the accumulator is free for
    // the next tile before any atomic is issued)
    static constexpr int EPI = (STAGE == 2 && NACC == 1 && !MXW) ? 8 : 4;
    static constexpr int THREADS = 64 + 32 * EPI + 32 * NCONV;
    static constexpr int SFA_BYTES = SFA_VAR ? 512 : 0;
    static constexpr int SFB_BYTES = SFB_VAR ? 512 * (B_ROWS / 128) : 0;
    // bytes that complete one stage: both CTAs' copies count on the even CTA's barrier
    static constexpr int TX_BYTES = (PAIR ? 2 : 1) * (A_BYTES + B_ROWS * B_ROW_TX + SFA_BYTES + SFB_BYTES);
    static constexpr int KE = FP8 ? 128 : 64;  // K elements per 128-byte K tile
    static constexpr int MMA_M = PAIR ? 2 * kBlockM : kBlockM;
    // TMEM columns: accumulators, then A scales (4 per stage, or 4 constant),
    // then B scales (BN/32 per stage, or 8 constant)
    static constexpr int SFA_COL = NACC * BN;
    static constexpr int SFA_NCOL = SFA_VAR ? 4 * NST : (MX ? 4 : 0);
    static constexpr int SFB_COL = SFA_COL + SFA_NCOL;
    static constexpr int SFB_NCOL = SFB_VAR ? (BN / 32) * NST : (MX ? 8 : 0);
    static constexpr int COLS_USED = SFB_COL + SFB_NCOL;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "TMEM holds 512 columns");
    static_assert(B_ROWS % kWBlockRows == 0 && BN <= 256, "BN: whole 128-row weight blocks");
    // shared memory: A ring, B ring, A-scale ring, B-scale ring, constant scales, barriers
    static constexpr int OFF_B = NST * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + NST * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + NST * SFA_BYTES;
    static constexpr int OFF_STG = OFF_SFB + NST * SFB_BYTES;
    static constexpr int OFF_SFC = OFF_STG + NST * STG_BYTES;
    static constexpr int OFF_BAR = OFF_SFC + (HAS_SFC ? 512 : 0);
    static constexpr int NUM_BARS = 2 * NST + 5 + (MXW ? NST : 0);
    static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static constexpr uint32_t IDESC = FP8 ? idesc_e4m3(MMA_M, BN) : idesc_bf16(MMA_M, BN);
    static constexpr uint32_t B_FMT = MXW ? kFmtE2M1 : kFmtE4M3;  // B operand format of the block-scaled MMA
};

// SiLU(g) = g / (1 + e^-g) (glossary entry "SwiGLU").  The quotient uses the
// fast division (at most 2 ulp, far below the bf16 rounding that follows):
// the correctly rounded division made the epilogue slower than the main loop.
// For g -> -inf the denominator overflows to +inf and the result is -0.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void decode_tile(int tile, int num_mt, int n_tiles, int& m, int& n, int& split) {
    m = tile % num_mt;
    const int r = tile / num_mt;
    n = r % n_tiles;
    split = r / n_tiles;
}

}  // namespace

template <int STAGE, bool FP8, int BN, int NST, int NACC, bool PAIR, int AR, bool MXW>
__global__ void __launch_bounds__(Cfg<STAGE, FP8, BN, NST, NACC, PAIR, AR, MXW>::THREADS, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA32,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmSF,
                    const GemmArgs args) {
    using C = Cfg<STAGE, FP8, BN, NST, NACC, PAIR, AR, MXW>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + NST;
    uint64_t* tfull = bars + 2 * NST;
    uint64_t* tempty = bars + 2 * NST + 2;
    uint64_t* drain = bars + 2 * NST + 4;
    uint64_t* raw = bars + 2 * NST + 5;  // MX FP4: packed weights landed in the staging ring
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t limit = args.timeout_ns;
    // pair: rank 0 (even CTA) issues the MMAs; work units are per cluster
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = (rank == 0);
    const int unit0 = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x;
    const int ustep = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    // a wait that gives up tells the other CTA of the pair to give up too
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        const bool ok = mbar_wait(bar, parity, abort_flag, limit, args.status);
        if (PAIR && !ok) st_cluster_u32(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
        return ok;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1 + C::NCONV);  // (MX FP4: the producer and the converter warps)
            mbar_init(&empty[i], 1);
            if constexpr (MXW) mbar_init(&raw[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], PAIR ? 2 * C::EPI : C::EPI);  // the epilogue warps of both CTAs release a pair tile
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (C::HAS_SFC && warp >= 2 && warp < 6) {
        // constant UE8M0 scale 2^0 for every row of the operand without block
        // scales (FP8 stage 2: B, w2 has fp32 per-channel scales instead; MX
        // FP4 stage 1: A, the activations have one fp32 scale per token)
        reinterpret_cast<uint32_t*>(smem + C::OFF_SFC)[threadIdx.x - 64] = 0x7F7F7F7Fu;
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        if constexpr (!PAIR) prefetch_tmap(&tmA32);
        if constexpr (PAIR) prefetch_tmap(&tmB);
        if ((PAIR && C::SFA_VAR) || (STAGE == 1 && args.a_gather)) prefetch_tmap(&tmSF);
    }
    // Expert-major tile order: the first 128-row tile (and, for pairs, the
    // first pair of tiles) of each expert, from a scan of the per-expert row
    // counts (written by the routing step, two launches back, so readable
    // before the wait for the previous kernel).
    __shared__ int s_mt_first[kMaxExperts + 1];
    __shared__ int s_pair_first[kMaxExperts + 1];
    if (warp == 2) {
        int carry = 0, carry_p = 0;
        for (int base = 0; base < args.num_experts; base += 32) {
            const int e = base + lane;
            int v = (e < args.num_experts) ? (args.counts[e] + kBlockM - 1) / kBlockM : 0;
            int vp = (v + 1) / 2;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v, d);
                const int yp = __shfl_up_sync(0xffffffffu, vp, d);
                if (lane >= d) {
                    v += y;
                    vp += yp;
                }
            }
            if (e < args.num_experts) {
                s_mt_first[e + 1] = carry + v;
                s_pair_first[e + 1] = carry_p + vp;
            }
            carry += __shfl_sync(0xffffffffu, v, 31);
            carry_p += __shfl_sync(0xffffffffu, vp, 31);
        }
        if (lane == 0) {
            s_mt_first[0] = 0;
            s_pair_first[0] = 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // The routing tables were written two launches back, so they may be read
    // before the wait for the previous kernel (see griddep_wait).
    int num_mt = *args.num_mtiles;
    if (num_mt < 0 || num_mt > args.mt_max) {  // never from the router: a corrupted table
        if (threadIdx.x == 0) record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
        num_mt = 0;
    }
    const int ns = args.n_tiles * args.splits;
    const int tiles = PAIR ? s_pair_first[args.num_experts] * ns : num_mt * ns;
    const int kps = args.k_tiles / args.splits;
    // Stage 1 on one CTA per tile: when the last wave of tiles would keep at
    // most 1/kQ of the CTAs busy, each of its tiles is cut into kQ = BN/64
    // units of 64 weight rows (no K split, so nothing to add up afterwards),
    // which spreads that wave's weight stream over kQ times as many SMs.  (Cutting
    // a fuller last wave, whose cut units then take several waves, was measured
    // slower: with 76 of 148 CTAs in the last wave, 50 -> 64 us at one token.)
    constexpr int kQ = BN / 64;
    int full_tiles = tiles;
    if constexpr (STAGE == 1 && !PAIR && kQ > 1) {
        const int tail = tiles % (int)gridDim.x;
        if (tail > 0 && tail * kQ <= (int)gridDim.x) full_tiles = tiles - tail;
    }
    const int units = full_tiles + (tiles - full_tiles) * kQ;
    // Work unit -> (this CTA's m-tile, n, split); `dup` marks the second half
    // of a pair that repeats the first (its results are not stored).
    //   Default order: m fastest over all m-tiles, so the CTAs of a wave that
    //   share a weight tile run side by side.
    //   Expert-major (group_m, and always for pairs): all tiles of one expert
    //   before the next, m fastest inside it, so a wave's activation rows and
    //   weights are both one expert's and each is fetched from DRAM about once
    //   even when the activations of all experts together do not fit in L2.
    //   q4 >= 0: the unit is 64-row slice q4 of tile `t` (the last wave's cut).
    auto unit_coords = [&](int u, int& m, int& n, int& split, bool& dup, int& q4) {
        dup = false;
        q4 = -1;
        if (u >= full_tiles) {
            const int v = u - full_tiles;
            q4 = v % kQ;
            u = full_tiles + v / kQ;
        }
        if constexpr (PAIR) {
            const int p = u / ns;
            int lo = 0, hi = args.num_experts;  // largest e with s_pair_first[e] <= p
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_pair_first[mid] <= p) lo = mid;
                else hi = mid;
            }
            const int e = lo;
            const int cnt = s_pair_first[e + 1] - s_pair_first[e];
            if (cnt > 0 && p < s_pair_first[e + 1]) {
                const int local = u - s_pair_first[e] * ns;
                const int m0 = s_mt_first[e] + 2 * (local % cnt);
                const int r = local / cnt;
                n = r % args.n_tiles;
                split = r / args.n_tiles;
                const bool odd = (m0 + 1 >= s_mt_first[e + 1]);
                m = (rank == 0 || odd) ? m0 : m0 + 1;
                dup = (rank == 1) && odd;
                return;
            }
            record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            m = 0;
            n = 0;
            split = 0;
            dup = true;
            return;
        } else {
            if (args.group_m) {
                const int e = args.mtile_expert[u / ns];
                const int mf = (e >= 0 && e < args.num_experts) ? s_mt_first[e] : 0;
                const int cnt = (e >= 0 && e < args.num_experts) ? s_mt_first[e + 1] - mf : 0;
                if (cnt > 0 && u >= mf * ns && u < (mf + cnt) * ns) {
                    const int local = u - mf * ns;
                    m = mf + local % cnt;
                    const int r = local / cnt;
                    n = r % args.n_tiles;
                    split = r / args.n_tiles;
                    return;
                }
                record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            }
            decode_tile(u, num_mt, args.n_tiles, m, n, split);
        }
    };
    // Expert of m-tile m; an index out of range (never from the router) is
    // recorded and replaced by expert 0, so no access leaves the weights.
    auto expert_of = [&](int m) {
        int e = args.mtile_expert[m];
        if (e < 0 || e >= args.num_experts) {
            record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            e = 0;
        }
        return e;
    };
    // Token of padded row `slot` (-1 for a padding row); an assignment out of
    // range (never from the router) is recorded and read as a padding row.
    auto token_of = [&](int slot) {
        const int a = args.slot_assign[slot];
        if (a == -1) return -1;
        if (a < 0 || a >= args.T * args.topk) {
            record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            return -1;
        }
        return a / args.topk;
    };
    // One-CTA tiles whose m-tile holds at most 32 rows in use (small batches:
    // a few tokens per expert) copy only those 32 activation rows; the MMA
    // still reads 128 rows, and the results of the rows not copied (stale
    // shared memory) belong to padding rows and are discarded.
    auto a_rows32 = [&](int m) {
        if constexpr (PAIR) {
            return false;
        } else {
            const int e = args.mtile_expert[m];
            if (e < 0 || e >= args.num_experts) return false;
            return args.counts[e] - (m - s_mt_first[e]) * kBlockM <= 32;
        }
    };
    auto stage_tx = [&](bool small, int q4) {
        return C::TX_BYTES - ((small && AR == kBlockM) ? (kBlockM - 32) * 128 : 0) -
               (q4 >= 0 ? (C::B_ROWS - 64) * C::B_ROW_TX : 0);
    };
    const int b_nblk = args.rows_b / kWBlockRows;
    const uint64_t pol_b = args.b_evict_first ? policy_evict_first() : policy_evict_normal();
    // This CTA's weight blocks for unit (e, n) at K tile kt: the BN rows of the
    // tile, or this CTA's half of them in a pair.
    auto load_weights = [&](int stage, int e, int n, int kt, int q4) {
        if constexpr (MXW) {
            // MX FP4: the packed rows of each 128-row block of the unit (8 KB
            // in one run in the blocked layout; a 64-row slice is half of one)
            // by bulk copy into the staging ring, for the converter warps; then
            // the B scale chunk of each 128-row block (512 bytes, already in
            // the layout TMEM takes)
            uint8_t* dst = smem + C::OFF_STG + stage * C::STG_BYTES;
            const int row0 = n * BN + (q4 >= 0 ? 64 * q4 : 0);
            const uint32_t bytes = (q4 >= 0) ? 64 * 64 : C::STG_BYTES;
            mbar_arrive_expect_tx(&raw[stage], bytes);
            for (int j = 0; j < (q4 >= 0 ? 1 : C::B_ROWS / kWBlockRows); ++j) {
                const size_t blk = ((size_t)e * b_nblk + row0 / kWBlockRows + j) * args.k_tiles + kt;
                const uint8_t* src = args.b_blocks + blk * (kWBlockRows * 64) + (row0 % kWBlockRows) * 64;
                bulk_load_hint(dst + j * kWBlockRows * 64, src, q4 >= 0 ? 64 * 64 : kWBlockRows * 64, &raw[stage],
                               pol_b);
            }
            const int rb0 = (n * BN + (q4 >= 0 ? 64 * q4 : 0)) / kWBlockRows;
            const int nchunks = (q4 >= 0) ? 1 : C::B_ROWS / kWBlockRows;
            for (int j = 0; j < nchunks; ++j) {
                const size_t chunk = ((size_t)e * b_nblk + rb0 + j) * args.k_tiles + kt;
                bulk_load_hint(smem + C::OFF_SFB + stage * C::SFB_BYTES + 512 * j, args.b_sf + chunk * 512, 512,
                               &full[stage], pol_b);
            }
            return;
        }
        if (!PAIR && q4 >= 0) {  // 64 rows: one half of one 16 KB block (its pre-swizzled rows 0-63 or 64-127)
            const size_t blk = ((size_t)e * b_nblk + n * (BN / kWBlockRows) + (q4 >> 1)) * args.k_tiles + kt;
            bulk_load_hint(smem + C::OFF_B + stage * C::B_BYTES, args.b_blocks + blk * kWBlockBytes + (q4 & 1) * 8192,
                           8192, &full[stage], pol_b);
            return;
        }
        const int rb0 = n * (BN / kWBlockRows) + (PAIR ? (int)rank * (C::B_ROWS / kWBlockRows) : 0);
#pragma unroll
        for (int j = 0; j < C::B_ROWS / kWBlockRows; ++j) {
            const size_t blk = ((size_t)e * b_nblk + rb0 + j) * args.k_tiles + kt;
            uint8_t* dst = smem + C::OFF_B + stage * C::B_BYTES + j * kWBlockBytes;
            if constexpr (PAIR)
                tma_load_2d_pair(dst, &tmB, mapa_shared(smem_u32(&full[stage]), 0), 0, (int)(blk * kWBlockRows), pol_b);
            else
                bulk_load_hint(dst, args.b_blocks + blk * kWBlockBytes, kWBlockBytes, &full[stage], pol_b);
        }
    };

    // Weights depend on nothing earlier in the call: the producer puts the
    // first unit's first weight blocks in flight before waiting for the
    // previous kernel (whose output is the activation operand).
    // (Every lane of the producer warp knows npre: the producer loop below
    // runs warp-wide and its lanes must agree on which stages were issued here.)
    const int npre = (unit0 < units) ? min(NST, kps) : 0;
    if (warp == 0 && lane == 0 && unit0 < units) {
        int m, n, split, q4;
        bool dup;
        unit_coords(unit0, m, n, split, dup, q4);
        const int e = expert_of(m);
        const uint32_t tx = stage_tx(a_rows32(m), q4);
        for (int kk = 0; kk < npre; ++kk) {  // fresh stages: nothing to wait for
            if (leader) mbar_arrive_expect_tx(&full[kk], tx);
            load_weights(kk, e, n, split * kps + kk, q4);
        }
    }
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        // Producer warp.  Lane 0 waits for a free stage and copies the weights
        // and the activation tile (rows of the padded layout: the gather pass's
        // output in stage 1, h in stage 2) and scales; with a_gather, stage 1's
        // lanes instead gather the activation rows of the tile, four token rows
        // per lane, straight from the per-token rows (xq or x) by TMA.
        const bool tma_gather = (STAGE == 1) && args.a_gather != 0;
        // without the TMA gather lane 0 alone runs the loop (the other lanes
        // wait at the end), as the copies it issues need no other lane
        const bool in_loop = tma_gather || lane == 0;
        const unsigned loop_mask = tma_gather ? 0xffffffffu : 1u;
        const uint64_t pol_a = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int u = unit0; in_loop && u < units && ok; u += ustep) {
            int m, n, split, q4;
            bool dup;
            unit_coords(u, m, n, split, dup, q4);
            const int e = expert_of(m);
            const bool small = a_rows32(m);
            if (AR == 32 && !small && lane == 0) record_error(args.status, MOE_ERR_DEVICE_BOUNDS);  // host chose this wrongly
            // stage 1: token rows behind this lane's four rows of the m-tile
            // (a padding row reads token 0; its results are discarded)
            const int rows_in = (small || AR == 32) ? 32 : kBlockM;
            const bool gathers = tma_gather && 4 * lane < rows_in;
            int tok[4] = {0, 0, 0, 0};
            if (gathers) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tok[j] = max(token_of(m * kBlockM + 4 * lane + j), 0);
            }
            for (int kt = split * kps; kt < (split + 1) * kps; ++kt) {
                const bool prefetched = (u == unit0) && (kt - split * kps) < npre;
                if (!prefetched) {
                    int good = 1;
                    if (lane == 0) {
                        good = wait(&empty[stage], phase ^ 1) ? 1 : 0;
                        if (good) {
                            if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx(small, q4));
                            load_weights(stage, e, n, kt, q4);
                        }
                    }
                    if (!__shfl_sync(loop_mask, good, 0)) {
                        ok = false;
                        break;
                    }
                }
                // failure-detection test hook: CTA 0 leaves the activation
                // copy of its first stage out, so that stage never completes
                // and the MMA's bounded wait runs out (see MOE_OPT_TEST_STALL)
                const bool skip = args.test_stall && blockIdx.x == 0 && issued == 0;
                if (tma_gather) {
                    if (!skip && gathers) {
                        uint8_t* dst = smem + stage * C::A_BYTES + lane * 4 * 128;
                        if constexpr (PAIR)
                            tma_gather4_pair(dst, &tmSF, mapa_shared(smem_u32(&full[stage]), 0), kt * C::KE, tok[0],
                                             tok[1], tok[2], tok[3], pol_a);
                        else
                            tma_gather4(dst, &tmSF, &full[stage], kt * C::KE, tok[0], tok[1], tok[2], tok[3], pol_a);
                    }
                } else if (lane == 0) {
                    if constexpr (PAIR) {
                        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
                        if (!skip)
                            tma_load_2d_pair(smem + stage * C::A_BYTES, &tmA, bar, kt * C::KE, m * kBlockM, pol_a);
                        if constexpr (C::SFA_VAR)
                            tma_load_2d_pair(smem + C::OFF_SFA + stage * C::SFA_BYTES, &tmSF, bar, 0,
                                             (m * args.f_tiles + kt) * 4, pol_a);
                    } else {
                        if (!skip)
                            tma_load_2d(smem + stage * C::A_BYTES, (small || AR == 32) ? &tmA32 : &tmA, &full[stage],
                                        kt * C::KE, m * kBlockM, pol_a);
                        if constexpr (C::SFA_VAR)
                            bulk_load(smem + C::OFF_SFA + stage * C::SFA_BYTES,
                                      args.a_sf + ((size_t)m * args.f_tiles + kt) * 512, 512, &full[stage]);
                    }
                }
                ++issued;
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // do not leave while copies into this CTA's shared memory are in
        // flight (these waits ignore the abort flag but keep their time limit)
        if (lane == 0) {
            volatile int keep_waiting = 0;
            if constexpr (PAIR) {
                // a pair's copies complete on the even CTA's barriers: wait
                // instead until the MMAs have released every stage (which also
                // means no commit towards this CTA is still on its way)
                for (int i = 0; i < NST; ++i) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, ok ? &keep_waiting : abort_flag, limit, args.status))
                        break;
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            } else {
                for (int i = 1; i <= min(issued, NST); ++i) {
                    int s = stage - i;
                    uint32_t ph = phase;
                    if (s < 0) {
                        s += NST;
                        ph ^= 1;
                    }
                    mbar_wait(&full[s], ph, &keep_waiting, limit, args.status);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            if constexpr (C::HAS_SFC) {  // the constant scales, once
                const uint64_t sd = sdesc_sf(smem_u32(smem + C::OFF_SFC));
                if constexpr (!C::SFB_VAR) {
                    for (int c = 0; c < 8; c += 4) {
                        if constexpr (PAIR) tmem_cp_32x128b_x4_pair(tmem_base + C::SFB_COL + c, sd);
                        else tmem_cp_32x128b_x4(tmem_base + C::SFB_COL + c, sd);
                    }
                } else {
                    tmem_cp_32x128b_x4(tmem_base + C::SFA_COL, sd);
                }
            }
            // arrival on a barrier of both CTAs (pair) or of this CTA
            auto commit = [&](uint64_t* bar) {
                if constexpr (PAIR) {
                    tc_commit_pair(smem_u32(bar));
                    tc_commit_pair(mapa_shared(smem_u32(bar), 1));
                } else {
                    tc_commit(bar);
                }
            };
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int u = unit0; u < units && ok; u += ustep) {
                int m_, n_, split_, q4;
                bool dup_;
                unit_coords(u, m_, n_, split_, dup_, q4);
                // a 64-row slice: the same MMAs with N = 64 (and, with MX FP4
                // weights, the B scales of that half of the 128-row block:
                // TMEM column j of a block's scales holds its rows 32j..32j+31)
                const uint32_t idesc = (q4 >= 0) ? ((C::IDESC & ~(0x3Fu << 17)) | ((64u >> 3) << 17)) : C::IDESC;
                const int mma_n = (q4 >= 0) ? 64 : BN;
                const uint32_t sfb_half = (MXW && q4 >= 0) ? 2u * (uint32_t)(q4 & 1) : 0u;
                if (!wait(&tempty[acc], acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kk = 0; kk < kps; ++kk) {
                    if (!wait(&full[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * C::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + C::OFF_B + stage * C::B_BYTES);
                    if constexpr (C::SFA_VAR) {
                        const uint64_t sd = sdesc_sf(smem_u32(smem + C::OFF_SFA + stage * C::SFA_BYTES));
                        if constexpr (PAIR)
                            tmem_cp_32x128b_x4_pair(tmem_base + C::SFA_COL + 4 * stage, sd);
                        else
                            tmem_cp_32x128b_x4(tmem_base + C::SFA_COL + 4 * stage, sd);
                    }
                    if constexpr (C::SFB_VAR) {
#pragma unroll
                        for (int j = 0; j < C::B_ROWS / 128; ++j)
                            tmem_cp_32x128b_x4(tmem_base + C::SFB_COL + (BN / 32) * stage + 4 * j,
                                               sdesc_sf(smem_u32(smem + C::OFF_SFB + stage * C::SFB_BYTES + 512 * j)));
                    }
                    const uint32_t sfa = tmem_base + C::SFA_COL + (C::SFA_VAR ? 4 * stage : 0);
                    const uint32_t sfb = tmem_base + C::SFB_COL + (C::SFB_VAR ? (BN / 32) * stage : 0) + sfb_half;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = sdesc_sw128(a_addr + ks * 32);
                        const uint64_t bd = sdesc_sw128(b_addr + ks * 32);
                        const uint32_t accum = (kk > 0 || ks > 0) ? 1u : 0u;
                        if constexpr (C::MX) {
                            const uint32_t id = idesc_mx(C::MMA_M, mma_n, C::B_FMT, ks, ks);
                            if constexpr (PAIR) mma_mxfp8_pair(d_tmem, ad, bd, id, sfa, sfb, accum);
                            else mma_mxfp8(d_tmem, ad, bd, id, sfa, sfb, accum);
                        } else if constexpr (FP8) {
                            if constexpr (PAIR) mma_fp8_pair(d_tmem, ad, bd, C::IDESC, accum);
                            else mma_fp8(d_tmem, ad, bd, idesc, accum);
                        } else {
                            if constexpr (PAIR) mma_bf16_pair(d_tmem, ad, bd, C::IDESC, accum);
                            else mma_bf16(d_tmem, ad, bd, idesc, accum);
                        }
                    }
                    commit(&empty[stage]);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                commit(&tfull[acc]);
                if (++acc == NACC) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            volatile int keep_waiting = 0;
            if constexpr (PAIR) {
                // both CTAs' epilogues have released every accumulator, so no
                // arrival from the other CTA is still on its way to this one
                for (int i = 0; i < NACC; ++i) {
                    if (!mbar_wait(&tempty[acc], acc_phase ^ 1, ok ? &keep_waiting : abort_flag, limit, args.status))
                        break;
                    if (++acc == NACC) {
                        acc = 0;
                        acc_phase ^= 1;
                    }
                }
            }
            // every MMA issued by this thread has finished before TMEM is released
            if constexpr (PAIR) tc_commit_pair(smem_u32(drain));
            else tc_commit(drain);
            mbar_wait(drain, 0, &keep_waiting, limit, args.status);
        }
        __syncwarp();
    } else if (MXW && warp >= 6) {
        // ---------------- converter warps (MX FP4 weights): each stage's
        // packed rows (64 bytes = 128 codes) into the operand form, 16 codes
        // per 16 bytes (codes first, then 8 bytes of padding), with the
        // 128-byte swizzle of the K-major operand tile (16-byte chunk c of row
        // r at r*128 + (c ^ (r % 8))*16); each warp takes half the rows, and
        // every lane loads all its packed pieces before it stores, so the
        // shared-memory latencies overlap.  Then the stage's full barrier
        // hears from both warps.
        constexpr int kConv = C::NCONV > 0 ? C::NCONV : 1;  // (the other kernels never come here)
        constexpr int kMaxPieces = C::B_ROWS * 4 / (32 * kConv);  // 16-byte packed pieces per lane
        const int cw = warp - 6;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = unit0; u < units && ok; u += ustep) {
            int m, n, split, q4;
            bool dup;
            unit_coords(u, m, n, split, dup, q4);
            const int pieces = ((q4 >= 0) ? 64 : C::B_ROWS) * 4 / kConv;  // this warp's pieces of the stage
            const int p0 = cw * pieces;
            for (int kk = 0; kk < kps; ++kk) {
                if (!wait(&raw[stage], phase)) {
                    ok = false;
                    break;
                }
                const uint8_t* stg = smem + C::OFF_STG + stage * C::STG_BYTES;
                uint8_t* opb = smem + C::OFF_B + stage * C::B_BYTES;
                uint4 v[kMaxPieces];
#pragma unroll
                for (int j = 0; j < kMaxPieces; ++j) {
                    const int i = lane + 32 * j;
                    if (i < pieces) v[j] = *reinterpret_cast<const uint4*>(stg + (p0 + i) * 16);
                }
#pragma unroll
                for (int j = 0; j < kMaxPieces; ++j) {
                    const int i = lane + 32 * j;
                    if (i < pieces) {
                        const int r = (p0 + i) >> 2, pc = (p0 + i) & 3;  // row, piece of 32 codes in it
                        uint8_t* rowp = opb + r * 128;
                        *reinterpret_cast<uint4*>(rowp + (((2 * pc) ^ (r & 7)) * 16)) = make_uint4(v[j].x, v[j].y, 0u, 0u);
                        *reinterpret_cast<uint4*>(rowp + (((2 * pc + 1) ^ (r & 7)) * 16)) =
                            make_uint4(v[j].z, v[j].w, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();  // the tensor core reads these bytes through the async proxy
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[stage]);
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        __syncwarp();
    } else if (warp < 2 + C::EPI) {
        // ---------------- epilogue warps 2..5 (2..9: warps w and w + 4 share
        // a lane quarter and split its columns)
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        // the accumulator may be overwritten (pairs: the even CTA counts both CTAs' warps)
        auto release = [&](int a) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && !leader) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[a]), 0));
                else mbar_arrive(&tempty[a]);
            }
        };
        for (int u = unit0; u < units; u += ustep) {
            int m, n, split, q4;
            bool dup;
            unit_coords(u, m, n, split, dup, q4);
            if (!wait(&tfull[acc], acc_phase)) break;
            tc_fence_after();
            const int e = expert_of(m);
            const int slot = m * kBlockM + row;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            if constexpr (STAGE == 1) {
                // the activation scale of the row: per padded row as the gather
                // pass wrote it, or per token for the GEMM's own TMA gather
                float sxv = 1.0f;
                if constexpr (FP8) {
                    if (args.a_gather) {
                        const int t = token_of(slot);
                        sxv = (t >= 0) ? args.row_scale[t] : 0.0f;  // a padding row's results are discarded
                    } else {
                        sxv = args.row_scale_slot[slot];
                    }
                }
                // 64-column groups: all BN / 64 of a tile, or the one of a 64-row slice
                const int g_first = (q4 >= 0) ? q4 : 0;
                const int g_count = (q4 >= 0) ? 1 : BN / 64;
#pragma unroll 1
                for (int gi = 0; gi < g_count && !dup; ++gi) {
                    const int g = g_first + gi;
                    uint32_t rg[32], ru[32];
                    tmem_ld_32cols(tbase + gi * 64, rg);
                    tmem_ld_32cols(tbase + gi * 64 + 32, ru);
                    tmem_ld_wait();
                    const int hcol = n * (BN / 2) + g * 32;
                    float hv[32];
                    if constexpr (FP8) {
                        // per-channel scales of the 32 gate and 32 up columns (64 contiguous
                        // floats); MX FP4 weights carry their scales inside the MMA
                        const float4* cs4 = reinterpret_cast<const float4*>(args.col_scale + (size_t)e * args.rows_b +
                                                                            n * BN + g * 64);
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 one = make_float4(1.f, 1.f, 1.f, 1.f);
                            const float4 sg = MXW ? one : __ldg(cs4 + i4), su = MXW ? one : __ldg(cs4 + 8 + i4);
                            const float sgv[4] = {sg.x, sg.y, sg.z, sg.w}, suv[4] = {su.x, su.y, su.z, su.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int i = 4 * i4 + j;
                                const float gv = __uint_as_float(rg[i]) * (sxv * sgv[j]);
                                const float uv = __uint_as_float(ru[i]) * (sxv * suv[j]);
                                hv[i] = __bfloat162float(__float2bfloat16_rn(silu(gv) * uv));
                            }
                        }
                        float amax = 0.f;
#pragma unroll
                        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(hv[i]));
                        int ex = 0;
                        if (amax > 0.f) {
                            const uint32_t b = __float_as_uint(__fdiv_rn(amax, 448.0f));
                            const int e8 = (int)((b >> 23) & 0xFF);
                            const uint32_t man = b & 0x7FFFFFu;
                            ex = (e8 == 0) ? ((man > 0x400000u) ? -126 : -127) : e8 - 127 + (man != 0u);
                            ex = max(-127, min(127, ex));
                        }
                        const float inv = ldexpf(1.0f, -ex);
                        uint32_t packed[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                                make_float2(hv[4 * i] * inv, hv[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                                make_float2(hv[4 * i + 2] * inv, hv[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                            packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                                              (size_t)slot * args.out_pitch + hcol);
                        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                        args.out_sf[((size_t)m * args.f_tiles + (hcol >> 7)) * 512 + (row & 31) * 16 + (row >> 5) * 4 +
                                    ((hcol >> 5) & 3)] = (uint8_t)(ex + 127);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            hv[i] = silu(__uint_as_float(rg[i])) * __uint_as_float(ru[i]);
                        }
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            __nv_bfloat162 p = __floats2bfloat162_rn(hv[2 * i], hv[2 * i + 1]);
                            packed[i] = *reinterpret_cast<uint32_t*>(&p);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                                              (size_t)slot * args.out_pitch + hcol * 2);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                    }
                }
                release(acc);
            } else {
                const int a = dup ? -1 : args.slot_assign[slot];
                int t = (a >= 0) ? a / args.topk : -1;
                if (t >= args.T || a < -1) {  // never from the router: a corrupted table
                    record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
                    t = -1;
                }
                const float wgt = (t >= 0) ? args.topk_w[a] : 0.f;
                // the combine row: this GPU's buffer, or (d_ff-sharded layer) the
                // row of the rank that owns token t, possibly in a peer's memory
                float* orow = reinterpret_cast<float*>(static_cast<uint8_t*>(args.out) +
                                                       (size_t)(t >= 0 ? t : 0) * args.out_pitch);
                bool remote = false;
                if (args.n_ranks > 0 && t >= 0) {
                    const int g = t / args.rows_per_rank;
                    orow = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(args.peer_out[g]) +
                                                    (size_t)(t - g * args.rows_per_rank) * args.out_pitch);
                    remote = g != args.rank;
                }
                // 64 columns of the accumulator (in registers) into the combine
                // row: the weighted (and, FP8, channel-scaled) values first, all
                // scale loads in flight together; then one branch around two
                // straight runs of atomics (a branch inside the run keeps the
                // compiler from hoisting the loads)
                auto emit64 = [&](const uint32_t* r, int col) {
                    float4 v[16];
#pragma unroll
                    for (int i4 = 0; i4 < 16; ++i4)
                        v[i4] = make_float4(__uint_as_float(r[4 * i4]) * wgt, __uint_as_float(r[4 * i4 + 1]) * wgt,
                                            __uint_as_float(r[4 * i4 + 2]) * wgt, __uint_as_float(r[4 * i4 + 3]) * wgt);
                    if constexpr (FP8 && !MXW) {
                        const float4* cs4 = reinterpret_cast<const float4*>(args.col_scale + (size_t)e * args.rows_b + col);
#pragma unroll
                        for (int i4 = 0; i4 < 16; ++i4) {
                            const float4 sc = __ldg(cs4 + i4);
                            v[i4].x *= sc.x;
                            v[i4].y *= sc.y;
                            v[i4].z *= sc.z;
                            v[i4].w *= sc.w;
                        }
                    }
                    if (!remote) {
#pragma unroll
                        for (int i4 = 0; i4 < 16; ++i4) atomicAdd(reinterpret_cast<float4*>(orow + col + 4 * i4), v[i4]);
                    } else {  // scalar atomics through peer memory
#pragma unroll
                        for (int i4 = 0; i4 < 16; ++i4) {
                            atomicAdd(orow + col + 4 * i4, v[i4].x);
                            atomicAdd(orow + col + 4 * i4 + 1, v[i4].y);
                            atomicAdd(orow + col + 4 * i4 + 2, v[i4].z);
                            atomicAdd(orow + col + 4 * i4 + 3, v[i4].w);
                        }
                    }
                };
                if constexpr (C::EPI == 8) {
                    // this warp's half of the columns, all in registers before the
                    // (single) accumulator is released; the next tile's MMAs then
                    // run under this tile's atomics
                    const int c_lo = ((warp - 2) >> 2) * (BN / 2);
                    uint32_t r[BN / 2];
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tmem_ld_32cols(tbase + c_lo + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * j]));
                    tmem_ld_wait();
                    release(acc);
                    if (t >= 0) {
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j) emit64(r + 64 * j, n * BN + c_lo + 64 * j);
                    }
                } else {
                    // 64 columns per TMEM wait; the accumulator is released as soon as
                    // the last columns are in registers, before their atomics
#pragma unroll 1
                    for (int c0 = 0; c0 < BN; c0 += 64) {
                        uint32_t r[64];
                        tmem_ld_32cols(tbase + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                        tmem_ld_32cols(tbase + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                        tmem_ld_wait();
                        if (c0 + 64 == BN) release(acc);
                        if (t >= 0) emit64(r, n * BN + c0);
                    }
                }
            }
            if (++acc == NACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();  // no cross-CTA traffic after this point
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
    if constexpr (PAIR) cluster_sync_all();
}

namespace {

template <int STAGE, bool FP8, int BN, int NST, int NACC, bool PAIR, int AR = kBlockM, bool MXW = false>
cudaError_t launch_one(const GemmMaps& maps, const GemmArgs& args, int grid, cudaStream_t stream) {
    using C = Cfg<STAGE, FP8, BN, NST, NACC, PAIR, AR, MXW>;
    auto kern = moe_gemm_kernel<STAGE, FP8, BN, NST, NACC, PAIR, AR, MXW>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    // the fourth map: h's scale chunks (block-scaled stage 2 on CTA pairs) or
    // the per-token rows for the TMA gather (stage 1 with a_gather)
    if ((PAIR && C::SFA_VAR && !maps.sf) || (STAGE == 1 && args.a_gather && !maps.sf)) return cudaErrorInvalidValue;
    const CUtensorMap& m4 = maps.sf ? *maps.sf : *maps.a;
    if constexpr (PAIR) {
        if (grid < 2 || grid % 2) return cudaErrorInvalidValue;
        if (!maps.b) return cudaErrorInvalidValue;
        return launch_dependent_cluster(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, 2, stream, *maps.a, *maps.a,
                                        *maps.b, m4, args);
    } else {
        if (!maps.a32) return cudaErrorInvalidValue;
        return launch_dependent(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, *maps.a, *maps.a32,
                                *maps.a, m4, args);
    }
}

template <int STAGE, bool FP8, int BN, int NST, int NACC, bool PAIR, int AR = kBlockM>
int max_pairs_one() {
    using C = Cfg<STAGE, FP8, BN, NST, NACC, PAIR, AR, false>;
    auto kern = moe_gemm_kernel<STAGE, FP8, BN, NST, NACC, PAIR, AR, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return 0;
    return max_active_clusters(kern, C::THREADS, C::SMEM_BYTES, 2);
}

}  // namespace

int gemm_block_n(int stage, bool fp8, int cfg, bool mxw) {
    (void)fp8;
    if (mxw) return 128;
    if (cfg == 3) return stage == 1 ? 256 : 128;
    return cfg == 1 ? 128 : 256;
}

// cfg 0: CTA pairs, 256 x 256 tiles; cfg 1: one CTA, 128 x 128 tiles
// (weight streaming); cfg 2: one CTA, 128 x 256 tiles; cfg 3 (no m-tile with
// more than 32 rows in use): 32 activation rows per stage, which leaves room
// for deeper pipelines -- stage 1 on 128 x 256 tiles, stage 2 on 128 x 128.
// MX FP4 weights (mxw) run on 128 x 128 one-CTA tiles (two 128-column
// accumulators leave room in TMEM for the per-stage scales of both operands):
// cfg 1 (5 stages), or cfg 3 (at most 32 assignments in all) with 32
// activation rows per stage and 7 stages -- a stage of 4-bit weights brings
// only half the bytes of an e4m3 one from HBM, so more stages keep enough in
// flight (each stage also holds the packed rows, 8 KB).
cudaError_t launch_gemm(int stage, bool fp8, int cfg, const GemmMaps& maps, const GemmArgs& args, int grid,
                        cudaStream_t stream, bool mxw) {
    if (mxw) {
        if ((cfg != 1 && cfg != 3) || !fp8) return cudaErrorInvalidValue;
        if (cfg == 3)
            return stage == 1 ? launch_one<1, true, 128, 7, 2, false, 32, true>(maps, args, grid, stream)
                              : launch_one<2, true, 128, 7, 2, false, 32, true>(maps, args, grid, stream);
        return stage == 1 ? launch_one<1, true, 128, 5, 2, false, kBlockM, true>(maps, args, grid, stream)
                          : launch_one<2, true, 128, 5, 2, false, kBlockM, true>(maps, args, grid, stream);
    }
    if (cfg == 3) {
        if (stage == 1)
            return fp8 ? launch_one<1, true, 256, 6, 2, false, 32>(maps, args, grid, stream)
                       : launch_one<1, false, 256, 6, 2, false, 32>(maps, args, grid, stream);
        return fp8 ? launch_one<2, true, 128, 10, 2, false, 32>(maps, args, grid, stream)
                   : launch_one<2, false, 128, 10, 2, false, 32>(maps, args, grid, stream);
    }
    if (stage == 1) {
        if (fp8) return cfg == 0 ? launch_one<1, true, 256, 6, 2, true>(maps, args, grid, stream)
                      : cfg == 1 ? launch_one<1, true, 128, 6, 2, false>(maps, args, grid, stream)
                                 : launch_one<1, true, 256, 4, 2, false>(maps, args, grid, stream);
        return cfg == 0 ? launch_one<1, false, 256, 6, 2, true>(maps, args, grid, stream)
             : cfg == 1 ? launch_one<1, false, 128, 6, 2, false>(maps, args, grid, stream)
                        : launch_one<1, false, 256, 4, 2, false>(maps, args, grid, stream);
    }
    // block-scaled FP8: two 256-column accumulators leave no TMEM for the scale
    // factors, so the wide tiles keep a single accumulator
    if (fp8) return cfg == 0 ? launch_one<2, true, 256, 6, 1, true>(maps, args, grid, stream)
                  : cfg == 1 ? launch_one<2, true, 128, 6, 2, false>(maps, args, grid, stream)
                             : launch_one<2, true, 256, 4, 1, false>(maps, args, grid, stream);
    return cfg == 0 ? launch_one<2, false, 256, 6, 2, true>(maps, args, grid, stream)
         : cfg == 1 ? launch_one<2, false, 128, 6, 2, false>(maps, args, grid, stream)
                    : launch_one<2, false, 256, 4, 2, false>(maps, args, grid, stream);
}

int gemm_max_pairs(int stage, bool fp8) {
    if (stage == 1) return fp8 ? max_pairs_one<1, true, 256, 6, 2, true>() : max_pairs_one<1, false, 256, 6, 2, true>();
    return fp8 ? max_pairs_one<2, true, 256, 6, 1, true>() : max_pairs_one<2, false, 256, 6, 2, true>();
}

}  // namespace moe
