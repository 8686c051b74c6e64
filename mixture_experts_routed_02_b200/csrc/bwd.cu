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
// TMEM), each operand a K-major bf16 matrix copied by 2-D TMA with the 128-byte
// swizzle (no preshuffled weights: training changes them every step):
//   GU   [slots x 2F]: xg . [W1_e; W3_e]^T -- g and u recomputed (activation
//        recomputation: the forward keeps nothing but its output); the
//        epilogue stores g and u in fp32 and h = bf16(silu(g) u);
//   DH   [slots x F]:  dyg . (W2_e^T)^T, K = H -- epilogue: dw_a (sum over the
//        tile's columns of dh_unweighted * h, one fp32 atomic per row and tile),
//        dh = w_a * acc, then dg and du into dGU [slots x 2F];
//   DX   [slots x H]:  dGU . ([W1_e; W3_e]^T)^T, K = 2F -- epilogue: fp32
//        atomics into dx32[t] (the k experts of a token meet there);
//   DW   [rows x cols] per expert, K = the expert's padded slots: dW2_e =
//        dO^T h and [dW1_e; dW3_e] = dGU^T x, the transposed operands written
//        by the transpose kernel below (rows of the slot layout -> columns).
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
template <int BN, int NST, bool PAIR>
struct BCfg {
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
    static_assert(B_ROWS % 128 == 0, "B copies of 128 rows");
    static constexpr uint32_t IDESC = idesc_bf16(PAIR ? 2 * kBlockM : kBlockM, BN);
};

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

// SiLU and the logistic function (the fast division and exponential, as in the
// forward epilogue: far below the bf16 roundings around them)
__device__ __forceinline__ float logistic(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

}  // namespace

template <int MODE, int BN, int NST, bool PAIR>
__global__ void __launch_bounds__(192, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const BwdArgs args) {
    using C = BCfg<BN, NST, PAIR>;
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
            const int mt = PAIR ? args.m_tiles / 2 : args.m_tiles;
            const int per_e = mt * args.n_tiles;
            e = u / per_e;
            const int r = u - e * per_e;
            m = PAIR ? 2 * (r % mt) + (int)rank : r % mt;
            n = r / mt;
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
                    // B rows of this CTA: GU -- 128 rows of W1_e and the same 128
                    // rows of W3_e (the tile's first 128 columns are g, the last 128
                    // u, of the same features; on a pair each CTA holds one of the
                    // two); otherwise BN rows, or this CTA's half of them
                    if constexpr (PAIR) {
                        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
                        tma_load_2d_pair(sa, &tmA, bar, kx, m * kBlockM, pol_a);
                        if constexpr (MODE == kBwdGU) {
                            tma_load_2d_pair(sb, rank == 0 ? &tmB : &tmB2, bar, kx, e * args.b_rows + n * 128, pol_b);
                        } else {
                            const int brow = (MODE == kBwdDW ? 0 : e * args.b_rows) + n * BN + (int)rank * C::B_ROWS;
#pragma unroll
                            for (int j = 0; j < C::B_ROWS / 128; ++j)
                                tma_load_2d_pair(sb + j * 128 * 128, &tmB, bar, kx, brow + 128 * j, pol_b);
                        }
                    } else {
                        tma_load_2d(sa, &tmA, &full[stage], kx, m * kBlockM, pol_a);
                        if constexpr (MODE == kBwdGU) {
                            tma_load_2d(sb, &tmB, &full[stage], kx, e * args.b_rows + n * 128, pol_b);
                            tma_load_2d(sb + 128 * 128, &tmB2, &full[stage], kx, e * args.b_rows + n * 128, pol_b);
                        } else {
                            const int brow = (MODE == kBwdDW ? 0 : e * args.b_rows) + n * BN;
#pragma unroll
                            for (int j = 0; j < BN / 128; ++j)
                                tma_load_2d(sb + j * 128 * 128, &tmB, &full[stage], kx, brow + 128 * j, pol_b);
                        }
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
                        const uint64_t ad = sdesc_sw128(a_addr + ks * 32), bd = sdesc_sw128(b_addr + ks * 32);
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
            } else if constexpr (MODE == kBwdDX) {
                const int t = (a >= 0) ? a / args.topk : -1;
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
                                      make_float4(__uint_as_float(r[4 * i4]), __uint_as_float(r[4 * i4 + 1]),
                                                  __uint_as_float(r[4 * i4 + 2]), __uint_as_float(r[4 * i4 + 3])));
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

// ---------------------------------------------------------------- transposes
// out[c][s] = v(s, c) for 64 x 64 tiles, bf16, where row s of the source is
//   kSrcRows:  src row s (weights: a plain [rows, cols] matrix per batch z);
//   kSrcSlots: src row s of the slot layout, 0 for a padding slot;
//   kSrcTokens: the token row of slot s's assignment (t = a / topk), times
//              topk_w[a] if scaled, 0 for a padding slot.
// Each thread reads 16-byte pieces of source rows (a warp covers four rows of
// 128 bytes) and writes 16-byte pieces of output rows (eight consecutive
// slots); the tile crosses shared memory with a row pitch of 66 elements so
// that the column reads of one warp fall on distinct banks but for pairs.
template <int SRC>
__global__ void __launch_bounds__(256) transpose_kernel(TransposeArgs p) {
    constexpr int kPitch = 66;
    __shared__ __align__(16) uint16_t tile[64 * kPitch];
    const int c0 = blockIdx.x * 64, s0 = blockIdx.y * 64, z = blockIdx.z;
    int rows = p.rows;
    if (SRC != kSrcRows) {
        const int nmt = *p.num_mtiles;
        rows = (nmt >= 0 && nmt <= p.mt_max) ? nmt * kBlockM : 0;
    }
    if (s0 >= rows) return;
    const uint16_t* src = static_cast<const uint16_t*>(p.src) + (size_t)z * p.src_batch;
    uint16_t* out = static_cast<uint16_t*>(p.out) + (size_t)z * p.out_batch;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int q = threadIdx.x + 256 * i;  // 512 pieces: 64 rows x 8 pieces of 8 elements
        const int r = q >> 3, c8 = (q & 7) * 8;
        const int s = s0 + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (s < rows) {
            if constexpr (SRC == kSrcRows) {
                v = *reinterpret_cast<const uint4*>(src + (size_t)s * p.src_pitch + c0 + c8);
            } else {
                const int a = p.slot_assign[s];
                if (a >= 0 && a < p.num_assign) {
                    if constexpr (SRC == kSrcSlots) {
                        v = *reinterpret_cast<const uint4*>(src + (size_t)s * p.src_pitch + c0 + c8);
                    } else {
                        v = *reinterpret_cast<const uint4*>(src + (size_t)(a / p.topk) * p.src_pitch + c0 + c8);
                        if (p.scale) {
                            const float sc = p.scale[a];
                            float f[8];
                            unpack8(v, f);
#pragma unroll
                            for (int j = 0; j < 8; ++j) f[j] *= sc;
                            v = pack8(f);
                        }
                    }
                } else if (a < -1 || a >= p.num_assign) {
                    record_error(p.status, MOE_ERR_DEVICE_BOUNDS);
                }
            }
        }
        uint32_t* t32 = reinterpret_cast<uint32_t*>(tile + r * kPitch + c8);  // 4-byte aligned (kPitch even)
        t32[0] = v.x;
        t32[1] = v.y;
        t32[2] = v.z;
        t32[3] = v.w;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int q = threadIdx.x + 256 * i;  // 512 pieces: 64 output rows x 8 pieces of 8 slots
        const int c = q >> 3, r8 = (q & 7) * 8;
        if (s0 + r8 >= rows) continue;  // rows is a multiple of 64 for slot sources
        uint16_t e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = tile[(r8 + j) * kPitch + c];
        uint16_t* dst = out + (size_t)(c0 + c) * p.out_pitch + p.out_col + s0 + r8;
        if (s0 + r8 + 8 <= rows) {
            uint4 w;
            w.x = e[0] | ((uint32_t)e[1] << 16);
            w.y = e[2] | ((uint32_t)e[3] << 16);
            w.z = e[4] | ((uint32_t)e[5] << 16);
            w.w = e[6] | ((uint32_t)e[7] << 16);
            *reinterpret_cast<uint4*>(dst) = w;
        } else {
            for (int j = 0; j < 8 && s0 + r8 + j < rows; ++j) dst[j] = e[j];
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
    using C = BCfg<BN, NST, PAIR>;
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
    using C = BCfg<256, 6, true>;
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
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t launch_transpose(int src_kind, const TransposeArgs& p, int cols, int rows_max, int batch,
                             cudaStream_t stream) {
    // 16-byte pieces: the source pitch, the output pitch and column offset in
    // whole pieces of 8 elements (the bases are 16-byte aligned by contract)
    if (cols % 64 || rows_max < 0 || batch < 1 || p.src_pitch % 8 || p.out_pitch % 8 || p.out_col % 8 ||
        p.src_batch % 8 || p.out_batch % 8)
        return cudaErrorInvalidValue;
    if (rows_max == 0 || cols == 0) return cudaSuccess;
    const dim3 grid(cols / 64, (rows_max + 63) / 64, batch);
    switch (src_kind) {
        case kSrcRows: transpose_kernel<kSrcRows><<<grid, 256, 0, stream>>>(p); break;
        case kSrcSlots: transpose_kernel<kSrcSlots><<<grid, 256, 0, stream>>>(p); break;
        case kSrcTokens: transpose_kernel<kSrcTokens><<<grid, 256, 0, stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dw, int T, int E, int k, float* dlogits,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    dlogits_kernel<<<(T + 127) / 128, 128, 0, stream>>>(ids, w, dw, T, E, k, dlogits);
    return cudaGetLastError();
}

}  // namespace moe
