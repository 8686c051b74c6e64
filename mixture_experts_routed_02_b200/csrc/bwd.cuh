// bwd.cuh -- argument structs and launchers of the backward pass (bwd.cu).
#pragma once
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------- backward pass
// Grouped GEMMs of the backward pass (bwd.cu): GU recomputes g, u and h; DH
// gives dg, du and the routing-weight gradients; DX scatters dx; DW forms the
// weight gradients per expert (operands read K-major or MN-major as they lie).
// (kFwdW2: the training forward's second GEMM, h . W2_e^T with the weighted
// scatter-add, from the caller's row-major w2)
enum BwdMode { kBwdGU = 0, kBwdDH = 1, kBwdDX = 2, kBwdDW = 3, kFwdW2 = 4 };

struct BwdArgs {
    // the expert-padded slot layout (from the router)
    const int* num_mtiles;
    const int* mtile_expert;
    const int* slot_assign;
    const int* counts;
    const float* topk_w;
    int num_experts, mt_max, topk, T;
    int n_tiles;   // output columns / BN (GU: F / 128)
    int k_tiles;   // K / 64 (GU, DH, DX)
    int m_tiles;   // DW: output rows / 128
    int b_rows;    // rows of B's matrix per expert (GU: F rows of W1 / W3; DH: H rows of W2)
    int F;         // d_ff (GU, DH: column offset of u and du; DX: where K moves from W1 to W3)
    void* out;     // GU: fp32 g|u [S, 2F]; DH: dg|du [S, 2F]; DX, FwdW2: fp32 rows [T, H]; DW: dW (first part)
    long out_pitch;  // bytes
    void* out2;    // GU: h [S, F]; DW: rows >= split (dW3)
    long out2_pitch;
    const void* gu;  // DH: fp32 g|u
    long gu_pitch;
    const void* hbuf;  // DH: h
    long h_pitch;
    float* dw;     // DH: routing-weight gradients [T*k] (fp32 atomics)
    int split;     // DW: output rows from here on go to out2
    int n_fast;    // DW: n-tiles fastest inside an expert (A, the M side, is the larger operand)
    long expert_stride;  // DW: bytes per expert of out / out2
    unsigned long long timeout_ns;
    int* status;
};
// bn = 256 (128 x 256 tiles on one SM, or 256 x 256 on a pair of SMs when
// `pair`) or 128 (128 x 128 on one SM); grid = CTAs (pairs: an even number).
cudaError_t launch_bwd_gemm(int mode, int bn, bool pair, const CUtensorMap& a, const CUtensorMap& b,
                            const CUtensorMap& b2, const BwdArgs& args, int grid, cudaStream_t stream);
int bwd_max_pairs(int mode);  // resident clusters of the pair kernel (0: none)

// Rows of the slot layout for the backward (zero for padding slots):
// xg = x[t] (when x is given), dyg = dy[t] and dog = bf16(w_a dy[t]) (when dy
// is given); rows `pitch` elements apart.
struct SlotGatherArgs {
    const __nv_bfloat16* x;
    const __nv_bfloat16* dy;
    const int* num_mtiles;
    int mt_max;
    const int* slot_assign;
    const float* topk_w;
    int num_assign;  // T * k
    int topk;
    int H;
    long pitch;  // elements
    __nv_bfloat16* xg;
    __nv_bfloat16* dyg;
    __nv_bfloat16* dog;
    int* status;
};
cudaError_t launch_slot_gather(const SlotGatherArgs& p, int rows_max, cudaStream_t stream);
cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dw, int T, int E, int k, float* dlogits,
                           cudaStream_t stream);

}  // namespace moe
