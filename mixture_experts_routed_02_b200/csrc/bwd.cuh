// bwd.cuh -- argument structs and launchers of the backward pass (bwd.cu).
#pragma once
#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------- backward pass
// Grouped GEMMs of the backward pass (bwd.cu): GU recomputes g, u and h; DH
// gives dg, du and the routing-weight gradients; DX scatters dx; DW forms the
// weight gradients per expert from transposed operands.
enum BwdMode { kBwdGU = 0, kBwdDH = 1, kBwdDX = 2, kBwdDW = 3 };

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
    int b_rows;    // rows of B per expert (GU: F, DH: F, DX: H)
    int F;         // d_ff (GU, DH: column offset of u and du)
    void* out;     // GU: fp32 g|u [S, 2F]; DH: dg|du [S, 2F]; DX: fp32 dx [T, H]; DW: dW (first part)
    long out_pitch;  // bytes
    void* out2;    // GU: h [S, F]; DW: rows >= split (dW3)
    long out2_pitch;
    const void* gu;  // DH: fp32 g|u
    long gu_pitch;
    const void* hbuf;  // DH: h
    long h_pitch;
    float* dw;     // DH: routing-weight gradients [T*k] (fp32 atomics)
    int split;     // DW: output rows from here on go to out2
    long expert_stride;  // DW: bytes per expert of out / out2
    unsigned long long timeout_ns;
    int* status;
};
// bn = 256 (128 x 256 tiles on one SM, or 256 x 256 on a pair of SMs when
// `pair`) or 128 (128 x 128 on one SM); grid = CTAs (pairs: an even number).
cudaError_t launch_bwd_gemm(int mode, int bn, bool pair, const CUtensorMap& a, const CUtensorMap& b,
                            const CUtensorMap& b2, const BwdArgs& args, int grid, cudaStream_t stream);
int bwd_max_pairs(int mode);  // resident clusters of the pair kernel (0: none)

// out[c][out_col + s] = row s of the source, column c (bf16, 64 x 64 tiles):
enum TransposeSrc {
    kSrcRows = 0,    // plain [rows, cols] matrices, batch z of p.batch
    kSrcSlots = 1,   // rows of the slot layout, 0 for padding slots
    kSrcTokens = 2   // the token row of each slot's assignment (optionally x topk_w), 0 for padding
};
struct TransposeArgs {
    const void* src;
    long src_pitch;   // elements
    long src_batch;   // elements between batches (kSrcRows)
    int rows;         // kSrcRows: source rows
    const int* num_mtiles;  // slot sources: rows = num_mtiles * 128
    int mt_max;
    const int* slot_assign;
    int num_assign;   // T * k
    int topk;
    const float* scale;     // kSrcTokens: per-assignment factor, or null
    void* out;
    long out_pitch;   // elements
    long out_col;     // elements
    long out_batch;   // elements
    int* status;
};
cudaError_t launch_transpose(int src_kind, const TransposeArgs& p, int cols, int rows_max, int batch,
                             cudaStream_t stream);
cudaError_t launch_dlogits(const int32_t* ids, const float* w, const float* dw, int T, int E, int k, float* dlogits,
                           cudaStream_t stream);

}  // namespace moe
