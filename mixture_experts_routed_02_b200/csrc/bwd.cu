// bwd.cu -- the backward pass (custom VJP) of the BF16 layer
// (rocketrecap.com "FlyDSL kernels in JAX", timestamp 10:07: a custom VJP for
// training as the next step of the routed kernel).  For an upstream gradient
// dy = dL/dout and each assignment a = (t, j) of token t to expert e with
// routing weight w_a (g = W1_e x_t, u = W3_e x_t, h = silu(g) u, o = W2_e h):
//
//   dw_a = <dy_t, o> = <W2_e^T dy_t, h>     dh = w_a W2_e^T dy_t
//   du = dh silu(g)                          dg = dh u s(g) (1 + g (1 - s(g)))
//   dx_t = sum_a W1_e^T dg + W3_e^T du
//   dW1_e = sum dg x^T,  dW3_e = sum du x^T,  dW2_e = sum (w_a dy_t) h^T
//   dlogit[t, e_j] = w_j (dw_j - sum_i w_i dw_i)   (softmax over the chosen logits)
//
// Five grouped GEMMs on the tensor cores (tcgen05, bf16 operands, fp32 in
// TMEM), every operand copied by 2-D TMA with the 128-byte swizzle straight
// from the matrix it is -- the weights as the caller holds them (no
// preshuffle: training changes them every step), the activations in the
// expert-padded slot layout -- and read by the MMA K-major (K contiguous) or
// MN-major (M or N contiguous), as it lies, so nothing is transposed:
//   GU   [slots x 2F]: xg . [W1_e; W3_e]^T, K = H, both K-major -- g and u
//        recomputed (the layer's own forward keeps nothing but its output),
//        or computed once by the training forward and kept; the epilogue
//        stores g and u in fp32 and h = bf16(silu(g) u), zero rows for
//        padding slots;
//   DH   [slots x F]:  dyg . W2_e, K = H, W2_e [H, F] MN-major -- epilogue:
//        dw_a (the tile's sum of dh_unweighted * h, one fp32 atomic per row
//        and tile), dh = w_a * acc, then dg and du into dGU [slots x 2F];
//   DX   [slots x H]:  dGU . [W1_e; W3_e], K = 2F, W1_e / W3_e [F, H]
//        MN-major -- epilogue: fp32 atomics into dx32[t] (the k experts of a
//        token meet there);
//   DW   [rows x cols] per expert, K = the expert's padded slots, both
//        operands MN-major: dW2_e = dO^T h with dO = w_a dy_t gathered per
//        slot, and [dW1_e; dW3_e] = dGU^T xg (padding slots are zero in dO,
//        h, dGU and xg, so they add nothing).
// The training forward is built from the same kernel: GU (keeping g, u, h for
// the backward) and FwdW2 [slots x H] = h . W2_e^T, K = F, W2_e rows K-major,
// with the routing weight applied in the scatter-add of its epilogue.
// Warp roles as in the forward GEMM: warp 0 lane 0 issues the TMA copies into
// an NST-deep ring, warp 1 owns TMEM and issues the MMAs, warps 2..5 drain the
// two TMEM accumulators (the epilogue of one tile overlaps the next tile's
// main loop).  Every wait is bounded (MOE_ERR_DEVICE_TIMEOUT).
#include <cuda_bf16.h>

#include "bwd.cuh"

namespace moe {

namespace {

// PAIR: a cluster of two CTAs on two SMs computes a 256 x BN tile with
// tcgen05.mma.cta_group::2 -- each CTA copies its own 128 rows of A and half
// of B's BN rows, all copies complete on the even CTA's barriers, the even
// CTA issues the MMAs, and each CTA's TMEM receives its own 128 rows.  Per
// unit of work a CTA moves a third less operand data than on one SM, and a
// stage of 32 KB instead of 48 leaves room for six stages.
template <int MODE, int BN, int NST, bool PAIR>
struct BCfg {
    // operand majorness: A MN-major in DW; B MN-major in DH, DX and DW (GU
    // and FwdW2 read weight rows, K-major)
    static constexpr bool A_MN = MODE == kBwdDW;
    static constexpr bool B_MN = MODE == kBwdDH || MODE == kBwdDX || MODE == kBwdDW;
    static constexpr int A_BYTES = kBlockM * 128;  // 128 rows x 64 bf16
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // this CTA's rows of B
    static constexpr int B_BYTES = B_ROWS * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TX_BYTES = (PAIR ? 2 : 1) * STAGE_BYTES;  // on the even CTA's full barrier
    static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;  // two accumulators
    static constexpr int OFF_BAR = NST * STAGE_BYTES;
    static constexpr int NUM_BARS = 2 * NST + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(B_ROWS % 128 == 0, "B: whole boxes of 128 (K-major) or 64 (MN-major) columns");
    // bits 15 and 16 of the instruction descriptor: A and B MN-major
    static constexpr uint32_t IDESC =
        idesc_bf16(PAIR ? 2 * kBlockM : kBlockM, BN) | ((A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16);
};

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// blocks of 64 MN elements x 64 K rows (one TMA box, 8 KB: K rows of 128
// bytes, 8-row swizzle atoms 1024 bytes apart -- the stride byte offset),
// consecutive MN blocks 8 KB apart (the leading byte offset).  One MMA reads
// 16 K rows: the next one starts two atoms (2048 bytes) further.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);  // start address
    d |= (uint64_t)(8192 >> 4) << 16;        // leading byte offset: next 64-element MN block
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset: next 8 K rows
    d |= (uint64_t)1 << 46;                  // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                  // layout: 128-byte swizzle
    return d;
}

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 q = __bfloat1622float2(p[i]);
        f[2 * i] = q.x;
        f[2 * i + 1] = q.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// The logistic function (the fast division and exponential, as in the
// forward epilogue: far below the bf16 roundings around them)
__device__ __forceinline__ float logistic(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

}  // namespace

template <int MODE, int BN, int NST, bool PAIR>
__global__ void __launch_bounds__(192, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const BwdArgs args) {
    using C = BCfg<MODE, BN, NST, PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + NST;
    uint64_t* tfull = bars + 2 * NST;
    uint64_t* tempty = bars + 2 * NST + 2;
    uint64_t* drain = bars + 2 * NST + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t limit = args.timeout_ns;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
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
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], PAIR ? 8 : 4);  // the epilogue warps of both CTAs release a pair tile
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
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
        prefetch_tmap(&tmB);
        if (MODE == kBwdGU) prefetch_tmap(&tmB2);
    }
    // first 128-row tile of each expert in the slot layout (DW: K ranges; row
    // modes on pairs: the pairs of an expert's tiles), and first pair of tiles
    __shared__ int s_mt_first[kMaxExperts + 1];
    __shared__ int s_pair_first[kMaxExperts + 1];
    if ((MODE == kBwdDW || PAIR) && warp == 2) {
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

    // work units: row modes -> (m-tile of slots, or pair of an expert's
    // m-tiles; n-tile); DW -> (expert, m-tile or pair of m-tiles of output
    // rows, n-tile), experts slowest so a wave shares operands in L2
    int units;
    int num_mt = 0;
    if constexpr (MODE == kBwdDW) {
        units = args.num_experts * (PAIR ? args.m_tiles / 2 : args.m_tiles) * args.n_tiles;
        if (s_mt_first[args.num_experts] > args.mt_max) {  // never from the router: corrupted counts
            if (threadIdx.x == 0) record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            units = 0;
        }
    } else {
        num_mt = *args.num_mtiles;
        if (num_mt < 0 || num_mt > args.mt_max) {
            if (threadIdx.x == 0) record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            num_mt = 0;
        }
        units = PAIR ? s_pair_first[args.num_experts] * args.n_tiles : num_mt * args.n_tiles;
        if (PAIR && s_mt_first[args.num_experts] != num_mt) {  // never from the router
            if (threadIdx.x == 0) record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            units = 0;
        }
    }
    // unit -> (e, this CTA's m-tile, n, first K step, K steps); `dup` marks the
    // second half of a pair that repeats the first (an expert with an odd
    // number of m-tiles: its results are not stored)
    auto unit_coords = [&](int u, int& e, int& m, int& n, int& k0, int& kc, bool& dup) {
        dup = false;
        if constexpr (MODE == kBwdDW) {
            // inside an expert, the index of the larger operand changes slowest
            // (n_fast: A is the larger, so a wave shares its rows and reads B's
            // small columns from L2; otherwise the other way round)
            const int mt = PAIR ? args.m_tiles / 2 : args.m_tiles;
            const int per_e = mt * args.n_tiles;
            e = u / per_e;
            const int r = u - e * per_e;
            const int mi = args.n_fast ? r / args.n_tiles : r % mt;
            m = PAIR ? 2 * mi + (int)rank : mi;
            n = args.n_fast ? r % args.n_tiles : r / mt;
            k0 = 2 * s_mt_first[e];  // 64 slots per K step, 128 slots per tile
            kc = 2 * (s_mt_first[e + 1] - s_mt_first[e]);
        } else if constexpr (PAIR) {
            const int p = u / args.n_tiles;
            int lo = 0, hi = args.num_experts;  // largest e with s_pair_first[e] <= p
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_pair_first[mid] <= p) lo = mid;
                else hi = mid;
            }
            e = lo;
            const int cnt = s_pair_first[e + 1] - s_pair_first[e];
            k0 = 0;
            kc = args.k_tiles;
            if (cnt > 0 && p < s_pair_first[e + 1]) {
                const int local = u - s_pair_first[e] * args.n_tiles;
                const int m0 = s_mt_first[e] + 2 * (local % cnt);
                n = local / cnt;
                const bool odd = m0 + 1 >= s_mt_first[e + 1];
                m = (rank == 0 || odd) ? m0 : m0 + 1;
                dup = (rank == 1) && odd;
                return;
            }
            record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
            e = 0;
            m = 0;
            n = 0;
            dup = true;
        } else {
            m = u % num_mt;
            n = u / num_mt;
            e = args.mtile_expert[m];
            if (e < 0 || e >= args.num_experts) {
                record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
                e = 0;
            }
            k0 = 0;
            kc = args.k_tiles;
        }
    };

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = unit0; u < units && ok; u += ustep) {
                int e, m, n, k0, kc;
                bool dup;
                unit_coords(u, e, m, n, k0, kc, dup);
                for (int kk = 0; kk < kc; ++kk) {
                    if (!wait(&empty[stage], phase ^ 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    const int kx = (k0 + kk) * 64;
                    if (leader) mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
                    // every copy completes on the even CTA's barrier (a pair) or on this CTA's
                    const uint32_t bar = PAIR ? mapa_shared(smem_u32(&full[stage]), 0) : smem_u32(&full[stage]);
                    auto load = [&](void* dst, const CUtensorMap* map, int x, int y, uint64_t pol) {
                        if constexpr (PAIR) tma_load_2d_pair(dst, map, bar, x, y, pol);
                        else tma_load_2d(dst, map, &full[stage], x, y, pol);
                    };
                    // A: 128 rows of K-major data (one box of 64 K x 128 rows), or
                    // (DW) the 128 output rows' columns of the slot layout, MN-major:
                    // two boxes of 64 MN x 64 K
                    if constexpr (C::A_MN) {
                        load(sa, &tmA, m * kBlockM, kx, pol_a);
                        load(sa + 8192, &tmA, m * kBlockM + 64, kx, pol_a);
                    } else {
                        load(sa, &tmA, kx, m * kBlockM, pol_a);
                    }
                    // B: this CTA's B_ROWS columns of the tile (all BN on one SM)
                    const int ncol = n * BN + (PAIR ? (int)rank * C::B_ROWS : 0);
                    if constexpr (MODE == kBwdGU) {
                        // 128 rows of W1_e and the same 128 rows of W3_e (K-major): the
                        // tile's first 128 columns are g, the last 128 u, of the same
                        // features; on a pair each CTA holds one of the two
                        if constexpr (PAIR) {
                            load(sb, rank == 0 ? &tmB : &tmB2, kx, e * args.b_rows + n * 128, pol_b);
                        } else {
                            load(sb, &tmB, kx, e * args.b_rows + n * 128, pol_b);
                            load(sb + 128 * 128, &tmB2, kx, e * args.b_rows + n * 128, pol_b);
                        }
                    } else if constexpr (!C::B_MN) {
                        // FwdW2: BN (or this CTA's B_ROWS) rows of W2_e, K-major
#pragma unroll
                        for (int j = 0; j < C::B_ROWS / 128; ++j)
                            load(sb + j * 128 * 128, &tmB, kx, e * args.b_rows + ncol + 128 * j, pol_b);
                    } else {
                        // MN-major boxes of 64 columns x 64 K rows: DH from W2_e (rows
                        // h = K), DX from W1_e for K < F and W3_e beyond (rows c = K),
                        // DW from the slot layout (rows = slots = K)
                        const CUtensorMap* mb = &tmB;
                        int krow = kx;
                        if constexpr (MODE == kBwdDH) {
                            krow = e * args.b_rows + kx;
                        } else if constexpr (MODE == kBwdDX) {
                            const bool up = kx >= args.F;
                            mb = up ? &tmB2 : &tmB;
                            krow = e * args.F + (up ? kx - args.F : kx);
                        }
#pragma unroll
                        for (int j = 0; j < C::B_ROWS / 64; ++j) load(sb + j * 8192, mb, ncol + 64 * j, krow, pol_b);
                    }
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
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
                int e, m, n, k0, kc;
                bool dup;
                unit_coords(u, e, m, n, k0, kc, dup);
                if (!wait(&tempty[acc], acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kk = 0; kk < kc; ++kk) {
                    if (!wait(&full[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        // 16 K per MMA: 32 bytes along a K-major row, or two 8-row atoms MN-major
                        const uint64_t ad = C::A_MN ? sdesc_sw128_mn(a_addr + ks * 2048) : sdesc_sw128(a_addr + ks * 32);
                        const uint64_t bd = C::B_MN ? sdesc_sw128_mn(b_addr + ks * 2048) : sdesc_sw128(b_addr + ks * 32);
                        const uint32_t accum = (kk > 0 || ks > 0) ? 1u : 0u;
                        if constexpr (PAIR) mma_bf16_pair(d_tmem, ad, bd, C::IDESC, accum);
                        else mma_bf16(d_tmem, ad, bd, C::IDESC, accum);
                    }
                    commit(&empty[stage]);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                commit(&tfull[acc]);  // (no MMA for an expert without slots: the epilogue writes zeros)
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            volatile int keep_waiting = 0;
            if constexpr (PAIR) {
                // both CTAs' epilogues have released every accumulator, so no
                // arrival from the other CTA is still on its way to this one
                for (int i = 0; i < 2; ++i) {
                    if (!mbar_wait(&tempty[acc], acc_phase ^ 1, ok ? &keep_waiting : abort_flag, limit, args.status))
                        break;
                    if (++acc == 2) {
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
    } else {
        // ---------------- epilogue warps 2..5: TMEM lane quarter q = warp % 4
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        auto release = [&](int a) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && !leader) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[a]), 0));
                else mbar_arrive(&tempty[a]);
            }
        };
        for (int u = unit0; u < units; u += ustep) {
            int e, m, n, k0, kc;
            bool dup;
            unit_coords(u, e, m, n, k0, kc, dup);
            if (!wait(&tfull[acc], acc_phase)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            const int slot = m * kBlockM + row;
            int a = -1;
            if constexpr (MODE != kBwdDW) {
                a = dup ? -1 : args.slot_assign[slot];
                if (a < -1 || a >= args.T * args.topk) {  // never from the router
                    record_error(args.status, MOE_ERR_DEVICE_BOUNDS);
                    a = -1;
                }
            }
            if constexpr (MODE == kBwdGU) {
                // g, u (fp32) into gu[slot] at columns f and F + f, h (bf16) into hbuf[slot]
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    uint32_t rg[32], ru[32];
                    tmem_ld_32cols(tbase + c0, rg);
                    tmem_ld_32cols(tbase + 128 + c0, ru);
                    tmem_ld_wait();
                    if (c0 + 32 == 128) release(acc);
                    if (a < 0 && !dup) {  // a padding slot: h = 0 (the weight gradients read it)
                        uint4* oh = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out2) +
                                                             (size_t)slot * args.out2_pitch) + (n * 128 + c0) / 8;
#pragma unroll
                        for (int i = 0; i < 4; ++i) oh[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (a >= 0) {
                        const int f = n * 128 + c0;
                        float gv[32], uv[32], hv[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            gv[i] = __uint_as_float(rg[i]);
                            uv[i] = __uint_as_float(ru[i]);
                            hv[i] = __fdividef(gv[i], 1.0f + __expf(-gv[i])) * uv[i];
                        }
                        float4* og = reinterpret_cast<float4*>(static_cast<uint8_t*>(args.out) + (size_t)slot * args.out_pitch) +
                                     f / 4;
                        float4* ou = reinterpret_cast<float4*>(static_cast<uint8_t*>(args.out) + (size_t)slot * args.out_pitch) +
                                     (args.F + f) / 4;
                        uint4* oh = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out2) + (size_t)slot * args.out2_pitch) + f / 8;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            og[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
                            ou[i] = make_float4(uv[4 * i], uv[4 * i + 1], uv[4 * i + 2], uv[4 * i + 3]);
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) oh[i] = pack8(hv + 8 * i);
                    }
                }
            } else if constexpr (MODE == kBwdDH) {
                // acc = (W2_e^T dy_t)[f]: dw_a += acc * h, dh = w_a acc, then dg, du
                const float wa = (a >= 0) ? args.topk_w[a] : 0.0f;
                float part = 0.0f;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32cols(tbase + c0, r);
                    tmem_ld_wait();
                    if (c0 + 32 == BN) release(acc);
                    if (a < 0 && !dup) {  // a padding slot: dg = du = 0 (dW1 and dW3 read them)
                        uint8_t* orow = static_cast<uint8_t*>(args.out) + (size_t)slot * args.out_pitch;
                        uint4* og = reinterpret_cast<uint4*>(orow) + (n * BN + c0) / 8;
                        uint4* ou = reinterpret_cast<uint4*>(orow) + (args.F + n * BN + c0) / 8;
#pragma unroll
                        for (int i = 0; i < 4; ++i) og[i] = ou[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (a >= 0) {
                        const int f = n * BN + c0;
                        const uint8_t* gurow = static_cast<const uint8_t*>(args.gu) + (size_t)slot * args.gu_pitch;
                        const float4* gp = reinterpret_cast<const float4*>(gurow) + f / 4;
                        const float4* up = reinterpret_cast<const float4*>(gurow) + (args.F + f) / 4;
                        const uint4* hp =
                            reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(args.hbuf) + (size_t)slot * args.h_pitch) + f / 8;
                        float gv[32], uv[32], hv[32];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 g4 = __ldg(gp + i), u4 = __ldg(up + i);
                            gv[4 * i] = g4.x; gv[4 * i + 1] = g4.y; gv[4 * i + 2] = g4.z; gv[4 * i + 3] = g4.w;
                            uv[4 * i] = u4.x; uv[4 * i + 1] = u4.y; uv[4 * i + 2] = u4.z; uv[4 * i + 3] = u4.w;
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) unpack8(__ldg(hp + i), hv + 8 * i);
                        float dgv[32], duv[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float dhu = __uint_as_float(r[i]);
                            part = fmaf(dhu, hv[i], part);
                            const float dh = wa * dhu;
                            const float s = logistic(gv[i]);
                            duv[i] = dh * (gv[i] * s);
                            dgv[i] = dh * uv[i] * (s * (1.0f + gv[i] * (1.0f - s)));
                        }
                        uint8_t* orow = static_cast<uint8_t*>(args.out) + (size_t)slot * args.out_pitch;
                        uint4* og = reinterpret_cast<uint4*>(orow) + f / 8;
                        uint4* ou = reinterpret_cast<uint4*>(orow) + (args.F + f) / 8;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            og[i] = pack8(dgv + 8 * i);
                            ou[i] = pack8(duv + 8 * i);
                        }
                    }
                }
                if (a >= 0) atomicAdd(args.dw + a, part);
            } else if constexpr (MODE == kBwdDX || MODE == kFwdW2) {
                // dx: the k experts of a token meet in fp32; FwdW2: the same with
                // the routing weight (the forward's combine)
                const int t = (a >= 0) ? a / args.topk : -1;
                const float wa = (MODE == kFwdW2 && t >= 0) ? args.topk_w[a] : 1.0f;
                float* orow = reinterpret_cast<float*>(static_cast<uint8_t*>(args.out) + (size_t)(t >= 0 ? t : 0) * args.out_pitch);
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 64) {
                    uint32_t r[64];
                    tmem_ld_32cols(tbase + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                    tmem_ld_32cols(tbase + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                    tmem_ld_wait();
                    if (c0 + 64 == BN) release(acc);
                    if (t >= 0) {
                        const int col = n * BN + c0;
#pragma unroll
                        for (int i4 = 0; i4 < 16; ++i4)
                            atomicAdd(reinterpret_cast<float4*>(orow + col + 4 * i4),
                                      make_float4(__uint_as_float(r[4 * i4]) * wa, __uint_as_float(r[4 * i4 + 1]) * wa,
                                                  __uint_as_float(r[4 * i4 + 2]) * wa,
                                                  __uint_as_float(r[4 * i4 + 3]) * wa));
                    }
                }
            } else {
                // DW: output row m*128 + row of expert e, bf16; rows from `split` on
                // go to the second output (dW3 after dW1)
                const int r_out = m * kBlockM + row;
                const bool second = r_out >= args.split;
                uint8_t* base = static_cast<uint8_t*>(second ? args.out2 : args.out) + (size_t)e * args.expert_stride +
                                (size_t)(second ? r_out - args.split : r_out) * args.out_pitch;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    if (kc > 0) {
                        tmem_ld_32cols(tbase + c0, r);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = 0u;
                    }
                    if (c0 + 32 == BN) release(acc);
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                    uint4* dst = reinterpret_cast<uint4*>(base) + (n * BN + c0) / 8;
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = pack8(v + 8 * i);
                }
            }
            if (++acc == 2) {
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

// ---------------------------------------------------------------- slot gather
// Rows of the expert-padded slot layout for the backward's operands, zero for
// padding slots (the weight gradients sum over every slot of an expert):
// xg[s] = x[t] (if x is given), dyg[s] = dy[t] and dog[s] = bf16(w_a dy[t])
// (if dy is given) for slot s holding assignment a = (t, j); rows from
// num_mtiles * 128 on are left alone.  One
// warp per slot row, 16-byte pieces.
__global__ void __launch_bounds__(256) slot_gather_kernel(SlotGatherArgs p) {
    const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    const int nmt = *p.num_mtiles;
    const int rows = (nmt >= 0 && nmt <= p.mt_max) ? nmt * kBlockM : 0;
    if (warp >= rows) return;
    const int s = warp;
    int a = p.slot_assign[s];
    if (a < -1 || a >= p.num_assign) {  // never from the router: a corrupted table
        if (lane == 0) record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
        a = -1;
    }
    const int t = a >= 0 ? a / p.topk : 0;
    const float w = a >= 0 ? p.topk_w[a] : 0.0f;
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H);
    const uint4* dr = reinterpret_cast<const uint4*>(p.dy + (size_t)t * p.H);
    uint4* xo = reinterpret_cast<uint4*>(p.xg + (size_t)s * p.pitch);
    uint4* dyo = reinterpret_cast<uint4*>(p.dyg + (size_t)s * p.pitch);
    uint4* doo = reinterpret_cast<uint4*>(p.dog + (size_t)s * p.pitch);
    for (int i = lane; i < p.H / 8; i += 32) {
        if (p.x) xo[i] = a >= 0 ? __ldg(xr + i) : make_uint4(0u, 0u, 0u, 0u);
        if (p.dy) {
            uint4 dv = make_uint4(0u, 0u, 0u, 0u), ov = dv;
            if (a >= 0) {
                dv = __ldg(dr + i);
                float f[8];
                unpack8(dv, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] *= w;
                ov = pack8(f);
            }
            dyo[i] = dv;
            doo[i] = ov;
        }
    }
}

// dlogits[t] from the routing-weight gradients: w_j (dw_j - sum_i w_i dw_i) for
// the chosen experts, 0 for the others.  One thread per token.
__global__ void dlogits_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                               const float* __restrict__ dw, int T, int E, int k, float* __restrict__ dlogits) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    float s = 0.0f;
    for (int j = 0; j < k; ++j) s = fmaf(w[t * k + j], dw[t * k + j], s);
    float* row = dlogits + (size_t)t * E;
    for (int e = 0; e < E; ++e) row[e] = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int e = ids[t * k + j];
        if (e >= 0 && e < E) row[e] = w[t * k + j] * (dw[t * k + j] - s);
    }
}

namespace {

template <int MODE, int BN, int NST, bool PAIR>
cudaError_t launch_bwd_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const BwdArgs& args,
                           int grid, cudaStream_t stream) {
    using C = BCfg<MODE, BN, NST, PAIR>;
    auto kern = bwd_gemm_kernel<MODE, BN, NST, PAIR>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    if constexpr (PAIR) {
        if (grid < 2 || grid % 2) return cudaErrorInvalidValue;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, a, b, b2, args);
    } else {
        kern<<<grid, 192, C::SMEM_BYTES, stream>>>(a, b, b2, args);
        return cudaGetLastError();
    }
}

template <int MODE>
int max_pairs_one() {
    using C = BCfg<MODE, 256, 6, true>;
    auto kern = bwd_gemm_kernel<MODE, 256, 6, true>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return 0;
    return max_active_clusters(kern, 192, C::SMEM_BYTES, 2);
}

}  // namespace

// Clusters of two CTAs of the 256 x 256 backward GEMM that can be resident
// at once (0 if none can: then the one-SM tiles run).
int bwd_max_pairs(int mode) {
    switch (mode) {
        case kBwdGU: return max_pairs_one<kBwdGU>();
        case kBwdDH: return max_pairs_one<kBwdDH>();
        case kBwdDX: return max_pairs_one<kBwdDX>();
        case kBwdDW: return max_pairs_one<kBwdDW>();
        case kFwdW2: return max_pairs_one<kFwdW2>();
        default: return 0;
    }
}

// bn = 256: 128 x 256 tiles on one SM, or 256 x 256 on a pair (pair); bn =
// 128: 128 x 128 tiles on one SM (a dimension not a multiple of 256).
cudaError_t launch_bwd_gemm(int mode, int bn, bool pair, const CUtensorMap& a, const CUtensorMap& b,
                            const CUtensorMap& b2, const BwdArgs& args, int grid, cudaStream_t stream) {
    if (grid < 1) return cudaSuccess;
    if (pair && bn != 256) return cudaErrorInvalidValue;
    switch (mode) {
        case kBwdGU:
            if (bn != 256) return cudaErrorInvalidValue;
            return pair ? launch_bwd_one<kBwdGU, 256, 6, true>(a, b, b2, args, grid, stream)
                        : launch_bwd_one<kBwdGU, 256, 4, false>(a, b, b2, args, grid, stream);
        case kBwdDH:
            return pair ? launch_bwd_one<kBwdDH, 256, 6, true>(a, b, b2, args, grid, stream)
                 : bn == 256 ? launch_bwd_one<kBwdDH, 256, 4, false>(a, b, b2, args, grid, stream)
                             : launch_bwd_one<kBwdDH, 128, 6, false>(a, b, b2, args, grid, stream);
        case kBwdDX:
            return pair ? launch_bwd_one<kBwdDX, 256, 6, true>(a, b, b2, args, grid, stream)
                 : bn == 256 ? launch_bwd_one<kBwdDX, 256, 4, false>(a, b, b2, args, grid, stream)
                             : launch_bwd_one<kBwdDX, 128, 6, false>(a, b, b2, args, grid, stream);
        case kBwdDW:
            return pair ? launch_bwd_one<kBwdDW, 256, 6, true>(a, b, b2, args, grid, stream)
                 : bn == 256 ? launch_bwd_one<kBwdDW, 256, 4, false>(a, b, b2, args, grid, stream)
                             : launch_bwd_one<kBwdDW, 128, 6, false>(a, b, b2, args, grid, stream);
        case kFwdW2:
            return pair ? launch_bwd_one<kFwdW2, 256, 6, true>(a, b, b2, args, grid, stream)
                 : bn == 256 ? launch_bwd_one<kFwdW2, 256, 4, false>(a, b, b2, args, grid, stream)
                             : launch_bwd_one<kFwdW2, 128, 6, false>(a, b, b2, args, grid, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t launch_slot_gather(const SlotGatherArgs& p, int rows_max, cudaStream_t stream) {
    if (p.H % 8 || p.pitch % 8) return cudaErrorInvalidValue;
    if (rows_max <= 0) return cudaSuccess;
    slot_gather_kernel<<<(rows_max + 7) / 8, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dw, int T, int E, int k, float* dlogits,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    dlogits_kernel<<<(T + 127) / 128, 128, 0, stream>>>(ids, w, dw, T, E, k, dlogits);
    return cudaGetLastError();
}

}  // namespace moe
