// elementwise.cu -- the memory-bound steps around the two grouped GEMMs:
//   gather_kernel    gather of each expert's token rows into the expert-padded
//                    layout (rocketrecap.com "FlyDSL kernels in JAX", paragraph
//                    2: "gather"), fused with the per-token FP8 quantisation and
//                    with zeroing the fp32 combine buffer;
//   quant_kernel     per-token FP8 quantisation alone (for the first GEMM's
//                    own TMA gather of token rows) and zeroing of out32;
//   finalize_kernel  fp32 combine buffer -> bf16 output;
//   preshuffle_kernel the one-time load-time preshuffle of the expert weights into
//                    contiguous, pre-swizzled 128x128-byte operand blocks
//                    (timestamp 8:14).
#include <algorithm>

#include "kernels.cuh"

namespace moe {

// One CTA (128 threads) per token t: zeroes the token's fp32 combine row and,
// in FP8 mode, quantises the token's row once -- sx[t] = absmax/448 (IEEE
// division, 1 for a zero row) and xq[t, i] = e4m3_rn_satfinite(x[t, i] / sx[t])
// -- for the first GEMM, which gathers the rows of each expert's tokens from
// xq (FP8) or straight from x (BF16) by TMA.  Nothing here depends on the
// routing: the kernel runs beside the router and waits for it only at the end,
// before it lets the first GEMM start, so that GEMM may read the routing
// tables as soon as it starts.  Rows of up to kRegVec*1024 elements are held
// in registers between the absmax pass and the quantisation pass.
constexpr int kRegVec = 4;

template <bool kFP8>
__global__ void __launch_bounds__(128, 8) quant_kernel(const __nv_bfloat16* __restrict__ x, int H,
                                                   uint8_t* __restrict__ xq, float* __restrict__ sx_tok,
                                                   float* __restrict__ out32) {
    __shared__ float warp_max[4];
    const int tid = threadIdx.x;
    const int t = blockIdx.x;
    if (out32) {  // (the d_ff-sharded layer keeps its combine rows zero itself)
        float4* o = reinterpret_cast<float4*>(out32 + (size_t)t * H);
        for (int i = tid; i < H / 4; i += 128) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (kFP8) {
        const int nvec_in = H / 8;  // 8 bf16 per 16-byte vector
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
        const bool in_regs = nvec_in <= 128 * kRegVec;
        uint4 v[kRegVec];
        if (in_regs) {
#pragma unroll
            for (int r = 0; r < kRegVec; ++r) {
                const int i = tid + r * 128;
                v[r] = (i < nvec_in) ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        // absmax over the row, then x / sx rounded to e4m3 (nearest even, saturating)
        float amax = 0.f;
        auto absmax8 = [&](const uint4& u) {
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(p[j]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        };
        if (in_regs) {
#pragma unroll
            for (int r = 0; r < kRegVec; ++r) absmax8(v[r]);
        } else {
            for (int i = tid; i < nvec_in; i += 128) absmax8(__ldg(src + i));
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
        if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
        __syncthreads();
        amax = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
        const float sx = (amax == 0.f) ? 1.0f : __fdiv_rn(amax, 448.0f);
        if (tid == 0) sx_tok[t] = sx;
        auto quant8 = [&](const uint4& u) {
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
            uint32_t packed[2];
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const float2 f0 = __bfloat1622float2(p[j]);
                const float2 f1 = __bfloat1622float2(p[j + 1]);
                const __nv_fp8x2_storage_t q0 = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f0.x, sx), __fdiv_rn(f0.y, sx)), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t q1 = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f1.x, sx), __fdiv_rn(f1.y, sx)), __NV_SATFINITE, __NV_E4M3);
                packed[j / 2] = (uint32_t)q0 | ((uint32_t)q1 << 16);
            }
            return make_uint2(packed[0], packed[1]);
        };
        uint2* dst = reinterpret_cast<uint2*>(xq + (size_t)t * H);
        if (in_regs) {
#pragma unroll
            for (int r = 0; r < kRegVec; ++r) {
                const int i = tid + r * 128;
                if (i < nvec_in) dst[i] = quant8(v[r]);
            }
        } else {
            for (int i = tid; i < nvec_in; i += 128) dst[i] = quant8(__ldg(src + i));
        }
    }
    griddep_wait();  // the router has completed ...
    griddep_launch_dependents();  // ... before the first GEMM may start
}

// The gather pass (the first GEMM then reads 128- or 32-row tiles of the
// gathered rows with one TMA tile copy each; for tiles of many rows that is
// far cheaper for the copy engine than 32 four-row gathers per K step).  One
// CTA (128 threads) per `per_cta` consecutive assignments a = t*k + j of one
// token t (per_cta = k: the whole token; 1: one assignment, for small batches
// where more CTAs shorten the critical path): reads the row once, quantises it
// once (FP8: the scale is per token, written to sx[t] and to each of its
// padded rows) and writes it to
// the padded-layout row of each of those assignments; the CTA holding the
// token's first assignment also zeroes its fp32 combine row.  Padding rows are
// not written: the tensor cores compute each output row from its own input row
// only, and the outputs of padding rows are discarded.  The row is read into
// registers before the wait for the routing kernel (the tokens are the
// caller's input and the combine buffer was last read by the previous call's
// finalize, both complete before routing started); only the destination rows
// need the routing result.
template <bool kFP8, bool kPerToken>
__global__ void __launch_bounds__(128, 8) gather_kernel(const __nv_bfloat16* __restrict__ x, int T, int H, int k,
                                                    const int* __restrict__ slot_of, int num_slots,
                                                    uint8_t* __restrict__ xs, float* __restrict__ sx_tok,
                                                    float* __restrict__ sx_slot, float* __restrict__ out32,
                                                    int* __restrict__ status) {
    __shared__ float warp_max[4];
    const int tid = threadIdx.x;
    const int per_cta = kPerToken ? k : 1;
    const int a0 = blockIdx.x * per_cta;
    const int t = a0 / k;
    const int eb = kFP8 ? 1 : 2;
    const int nvec_in = H / 8;  // 8 bf16 per 16-byte vector
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    const bool in_regs = nvec_in <= 128 * kRegVec;
    uint4 v[kRegVec];
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kRegVec; ++r) {
            const int i = tid + r * 128;
            v[r] = (i < nvec_in) ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    if (a0 % k == 0 && out32) {
        float4* o = reinterpret_cast<float4*>(out32 + (size_t)t * H);
        for (int i = tid; i < H / 4; i += 128) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    griddep_wait();
    griddep_launch_dependents();
    const int n = per_cta;
    int slots[kPerToken ? kMaxTopK : 1];
    bool bad = false;
    for (int j = 0; j < n; ++j) {
        slots[j] = slot_of[a0 + j];
        bad |= slots[j] < 0 || slots[j] >= num_slots;  // never from the router: a corrupted table
    }
    if (bad) {
        if (tid == 0) record_error(status, MOE_ERR_DEVICE_BOUNDS);
        return;
    }
    const long pitch = act_pitch((long)H * eb);
    if (!kFP8) {
        for (int j = 0; j < n; ++j) {
            uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)slots[j] * pitch);
            if (in_regs) {
#pragma unroll
                for (int r = 0; r < kRegVec; ++r) {
                    const int i = tid + r * 128;
                    if (i < nvec_in) dst[i] = v[r];
                }
            } else {
                for (int i = tid; i < nvec_in; i += 128) dst[i] = __ldg(src + i);
            }
        }
        return;
    }
    float amax = 0.f;
    auto absmax8 = [&](const uint4& u) {
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    };
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kRegVec; ++r) absmax8(v[r]);
    } else {
        for (int i = tid; i < nvec_in; i += 128) absmax8(__ldg(src + i));
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
    if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
    const float sx = (amax == 0.f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    if (tid == 0 && a0 % k == 0) sx_tok[t] = sx;
    if (tid < n) sx_slot[slots[tid]] = sx;  // per padded row too: the first GEMM's epilogue reads it there
    auto quant8 = [&](const uint4& u) {
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint32_t packed[2];
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
            const float2 f0 = __bfloat1622float2(p[j]);
            const float2 f1 = __bfloat1622float2(p[j + 1]);
            const __nv_fp8x2_storage_t q0 = __nv_cvt_float2_to_fp8x2(
                make_float2(__fdiv_rn(f0.x, sx), __fdiv_rn(f0.y, sx)), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t q1 = __nv_cvt_float2_to_fp8x2(
                make_float2(__fdiv_rn(f1.x, sx), __fdiv_rn(f1.y, sx)), __NV_SATFINITE, __NV_E4M3);
            packed[j / 2] = (uint32_t)q0 | ((uint32_t)q1 << 16);
        }
        return make_uint2(packed[0], packed[1]);
    };
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kRegVec; ++r) {
            const int i = tid + r * 128;
            if (i < nvec_in) {
                const uint2 q = quant8(v[r]);
                for (int j = 0; j < n; ++j) reinterpret_cast<uint2*>(xs + (size_t)slots[j] * pitch)[i] = q;
            }
        }
    } else {
        for (int i = tid; i < nvec_in; i += 128) {
            const uint2 q = quant8(__ldg(src + i));
            for (int j = 0; j < n; ++j) reinterpret_cast<uint2*>(xs + (size_t)slots[j] * pitch)[i] = q;
        }
    }
}

cudaError_t launch_gather(bool fp8, const __nv_bfloat16* x, int T, int H, int k, const int* slot_of, int num_slots,
                          uint8_t* xs, float* sx_tok, float* sx_slot, float* out32, int* status, cudaStream_t stream) {
    // a CTA per token for large batches, per assignment (more CTAs, shorter
    // critical path) for small ones
    const bool per_token = T >= 256;
    const dim3 grid(std::max(1, per_token ? T : T * k));
    if (fp8)
        return per_token ? launch_dependent(gather_kernel<true, true>, grid, dim3(128), 0, stream, x, T, H, k, slot_of,
                                            num_slots, xs, sx_tok, sx_slot, out32, status)
                         : launch_dependent(gather_kernel<true, false>, grid, dim3(128), 0, stream, x, T, H, k,
                                            slot_of, num_slots, xs, sx_tok, sx_slot, out32, status);
    return per_token ? launch_dependent(gather_kernel<false, true>, grid, dim3(128), 0, stream, x, T, H, k, slot_of,
                                        num_slots, xs, sx_tok, sx_slot, out32, status)
                     : launch_dependent(gather_kernel<false, false>, grid, dim3(128), 0, stream, x, T, H, k, slot_of,
                                        num_slots, xs, sx_tok, sx_slot, out32, status);
}

cudaError_t launch_quant(bool fp8, const __nv_bfloat16* x, int T, int H, uint8_t* xq, float* sx_tok, float* out32,
                         cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return fp8 ? launch_dependent(quant_kernel<true>, dim3(T), dim3(128), 0, stream, x, H, xq, sx_tok, out32)
               : launch_dependent(quant_kernel<false>, dim3(T), dim3(128), 0, stream, x, H, xq, sx_tok, out32);
}

// out = bf16(out32), round to nearest even; n is a multiple of 8.
__global__ void finalize_kernel(const float* __restrict__ out32, __nv_bfloat16* __restrict__ out, size_t n) {
    griddep_wait();
    const size_t nv = n / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(out32) + 2 * i);
        const float4 b = __ldg(reinterpret_cast<const float4*>(out32) + 2 * i + 1);
        __nv_bfloat162 r[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                               __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
        reinterpret_cast<uint4*>(out)[i] = *reinterpret_cast<uint4*>(r);
    }
}

// ---------------------------------------------------------------- d_ff-sharded layer
// Each rank's second GEMM adds its partial sums of every token straight into
// the combine rows of the rank that owns the token (peer memory), which makes
// the GEMM and the reduce-scatter one pass.  The two kernels below close a
// step: every rank tells every rank that its additions are done (one system-
// scope increment of each rank's arrival counter, after a system-scope fence),
// and each rank rounds its own rows once all n_ranks increments of this step
// have arrived, zeroing them for the step after next (the caller alternates
// two sets of combine rows).

__global__ void dff_signal_kernel(PeerCounters counters, int n_ranks) {
    griddep_wait();  // the second GEMM's additions are complete
    __threadfence_system();
    if ((int)threadIdx.x < n_ranks) atomicAdd_system(counters.c[threadIdx.x], 1u);
}

__device__ __forceinline__ unsigned int ld_acquire_sys(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__global__ void dff_finalize_kernel(float* __restrict__ out32, __nv_bfloat16* __restrict__ out, size_t n,
                                    const unsigned int* counter, unsigned int target, unsigned long long timeout_ns,
                                    int* status) {
    __shared__ int s_ok;
    griddep_wait();
    if (threadIdx.x == 0) {
        // bounded wait for every rank's signal of this step (counters only grow;
        // the comparison is modulo 2^32)
        int ok = 1;
        if ((int)(ld_acquire_sys(counter) - target) < 0) {
            const uint64_t t0 = globaltimer_ns();
            while ((int)(ld_acquire_sys(counter) - target) < 0) {
                if (globaltimer_ns() - t0 > timeout_ns) {
                    record_error(status, MOE_ERR_DEVICE_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(200);
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    if (!s_ok) return;
    const size_t nv = n / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv; i += (size_t)gridDim.x * blockDim.x) {
        float4* src = reinterpret_cast<float4*>(out32) + 2 * i;
        const float4 a = src[0];
        const float4 b = src[1];
        __nv_bfloat162 r[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                               __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
        reinterpret_cast<uint4*>(out)[i] = *reinterpret_cast<uint4*>(r);
        src[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        src[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

cudaError_t launch_dff_signal(const PeerCounters& counters, int n_ranks, cudaStream_t stream) {
    return launch_dependent(dff_signal_kernel, dim3(1), dim3(32), 0, stream, counters, n_ranks);
}

cudaError_t launch_dff_finalize(float* out32_rows, __nv_bfloat16* out, size_t n, const unsigned int* counter,
                                unsigned int target, unsigned long long timeout_ns, int* status, int num_sms,
                                cudaStream_t stream) {
    const int blocks = (int)std::max<size_t>(1, std::min<size_t>((n / 8 + 255) / 256, (size_t)num_sms * 8));
    return launch_dependent(dff_finalize_kernel, dim3(blocks), dim3(256), 0, stream, out32_rows, out, n, counter,
                            target, timeout_ns, status);
}

// One thread per destination 16-byte chunk, destinations in address order.
// Destination chunk g: (expert e, row block nb, K block kt, row r, stored
// chunk pc); it holds logical chunk c = pc ^ (r % 8) of destination row
// R = 128*nb + r.  With `interleave` the destination rows are the w1/w3
// interleave (groups of 32 rows from a, then b); otherwise row R of a.
__global__ void preshuffle_kernel(const uint8_t* __restrict__ a, const uint8_t* __restrict__ b,
                                  uint8_t* __restrict__ dst, int E, int src_rows, int dst_rows, int row_bytes,
                                  bool interleave) {
    const int kt_count = row_bytes / 128;
    const int nb_count = dst_rows / kWBlockRows;
    const size_t total = (size_t)E * dst_rows * row_bytes / 16;
    for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total; g += (size_t)gridDim.x * blockDim.x) {
        const int pc = (int)(g & 7);
        const int r = (int)((g >> 3) & 127);
        size_t rest = g >> 10;
        const int kt = (int)(rest % kt_count);
        rest /= kt_count;
        const int nb = (int)(rest % nb_count);
        const int e = (int)(rest / nb_count);
        const int c = pc ^ (r & 7);
        const int R = nb * kWBlockRows + r;
        const uint8_t* src = a;
        int srow = R;
        if (interleave) {
            const int grp = R / 64, i = R % 64;
            src = (i < 32) ? a : b;
            srow = 32 * grp + (i & 31);
        }
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + ((size_t)e * src_rows + srow) * row_bytes +
                                                             kt * 128 + c * 16));
        reinterpret_cast<uint4*>(dst)[g] = v;
    }
}

__global__ void interleave_scales_kernel(const float* __restrict__ s1, const float* __restrict__ s3,
                                         float* __restrict__ s13, int E, int F) {
    const size_t total = (size_t)E * 2 * F;
    for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total; g += (size_t)gridDim.x * blockDim.x) {
        const int e = (int)(g / (2 * F));
        const int R = (int)(g % (2 * F));
        const int grp = R / 64, i = R % 64;
        s13[g] = ((i < 32) ? s1 : s3)[(size_t)e * F + 32 * grp + (i & 31)];
    }
}

// MX FP4 weight preparation.  Packed e2m1 rows (K/2 bytes each) regrouped
// into contiguous blocks of 128 rows x 64 bytes (128 codes of K) in the order
// [expert][128-row block][128-column K block], so that each TMA copy of the
// first (64-row) or second half of a block reads 4 KB in one run (row-major
// rows would be read as 64-byte pieces 2 KB apart, far too small to keep HBM
// busy).  One thread per 16-byte chunk of the destination.  With `interleave`
// destination row R of an expert is row 32*(R/64) + R%32 of a (R%64 < 32) or
// of b (the w1/w3 interleave of the first GEMM), otherwise row R of a.
__global__ void mx_rows_kernel(const uint8_t* __restrict__ a, const uint8_t* __restrict__ b,
                               uint8_t* __restrict__ dst, int E, int src_rows, int dst_rows, int row_bytes,
                               bool interleave) {
    const int k_tiles = row_bytes / 64;
    const size_t total = (size_t)E * dst_rows * row_bytes / 16;
    for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total; g += (size_t)gridDim.x * blockDim.x) {
        const int c4 = (int)(g & 3);                   // 16-byte chunk of the block row
        const int r = (int)((g >> 2) & 127);           // row inside the block
        size_t rest = g >> 9;                          // (expert, block, K block)
        const int kt = (int)(rest % k_tiles);
        rest /= k_tiles;
        const int nb = (int)(rest % (dst_rows / 128));
        const int e = (int)(rest / (dst_rows / 128));
        const int R = nb * 128 + r;
        const uint8_t* src = a;
        int srow = R;
        if (interleave) {
            src = (R % 64 < 32) ? a : b;
            srow = 32 * (R / 64) + (R % 32);
        }
        reinterpret_cast<uint4*>(dst)[g] =
            __ldg(reinterpret_cast<const uint4*>(src + ((size_t)e * src_rows + srow) * row_bytes + kt * 64) + c4);
    }
}

// The weights' UE8M0 block scales ([rows, K/32] per expert) regrouped into
// one 512-byte chunk per (expert, 128-row block, 128-element K tile), in the
// order the MMA's scale copy into TMEM takes (the same as h's scale chunks):
// byte (r % 32) * 16 + (r / 32) * 4 + kb holds the scale of row r of the
// block and K block kb of the tile.  Rows interleaved as in mx_rows_kernel.
__global__ void mx_scale_chunks_kernel(const uint8_t* __restrict__ sa, const uint8_t* __restrict__ sb,
                                       uint8_t* __restrict__ dst, int E, int src_rows, int dst_rows, int k_tiles,
                                       bool interleave) {
    const int nblk = dst_rows / 128;
    const size_t total = (size_t)E * nblk * k_tiles * 512;
    for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total; g += (size_t)gridDim.x * blockDim.x) {
        const int p = (int)(g % 512);
        const size_t c = g / 512;
        const int kt = (int)(c % k_tiles);
        const int nb = (int)((c / k_tiles) % nblk);
        const int e = (int)(c / ((size_t)k_tiles * nblk));
        const int r = (p / 16) + 32 * ((p % 16) / 4);
        const int kb = p % 4;
        const int R = nb * 128 + r;
        const uint8_t* src = sa;
        int srow = R;
        if (interleave) {
            src = (R % 64 < 32) ? sa : sb;
            srow = 32 * (R / 64) + (R % 32);
        }
        dst[g] = src[((size_t)e * src_rows + srow) * (k_tiles * 4) + kt * 4 + kb];
    }
}

cudaError_t launch_mx_prepare(const uint8_t* a, const uint8_t* b, const uint8_t* sa, const uint8_t* sb,
                              uint8_t* w_out, uint8_t* s_out, int E, int src_rows, int dst_rows, int K,
                              bool interleave, cudaStream_t stream) {
    const size_t nrow = (size_t)E * dst_rows * (K / 2) / 16;
    mx_rows_kernel<<<(int)std::min<size_t>((nrow + 255) / 256, 65535), 256, 0, stream>>>(
        a, b, w_out, E, src_rows, dst_rows, K / 2, interleave);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t nsf = (size_t)E * dst_rows * (K / 32);
    mx_scale_chunks_kernel<<<(int)std::min<size_t>((nsf + 255) / 256, 65535), 256, 0, stream>>>(
        sa, sb, s_out, E, src_rows, dst_rows, K / 128, interleave);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const float* out32, __nv_bfloat16* out, size_t n, int num_sms, cudaStream_t stream) {
    const int blocks = (int)std::min<size_t>((n / 8 + 255) / 256, (size_t)num_sms * 8);
    if (blocks == 0) return cudaSuccess;
    return launch_dependent(finalize_kernel, dim3(blocks), dim3(256), 0, stream, out32, out, n);
}

cudaError_t launch_preshuffle(const uint8_t* a, const uint8_t* b, uint8_t* dst, int E, int src_rows, int dst_rows,
                              int row_bytes, bool interleave, cudaStream_t stream) {
    const size_t chunks = (size_t)E * dst_rows * row_bytes / 16;
    const int blocks = (int)std::min<size_t>((chunks + 255) / 256, 65535);
    preshuffle_kernel<<<blocks, 256, 0, stream>>>(a, b, dst, E, src_rows, dst_rows, row_bytes, interleave);
    return cudaGetLastError();
}

cudaError_t launch_interleave_scales(const float* s1, const float* s3, float* s13, int E, int F, cudaStream_t stream) {
    const size_t n = (size_t)E * 2 * F;
    interleave_scales_kernel<<<(int)std::min<size_t>((n + 255) / 256, 65535), 256, 0, stream>>>(s1, s3, s13, E, F);
    return cudaGetLastError();
}

}  // namespace moe
