// kernels.cuh -- shared constants, argument structs and host-side launchers of
// the library's kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace moe {

constexpr int kMaxExperts = 64;
constexpr int kMaxTopK = 8;
constexpr int kMaxRanks = 16;  // d_ff shards of the sharded layer
constexpr int kBlockM = 128;  // rows per tile of the expert-padded layout
// Row pitch of h: 128 bytes more than a row,
// so that the 128 rows of an operand tile do not sit a power of two apart
// (such rows crowd into few L2 slices).
__host__ __device__ constexpr long act_pitch(long row_bytes) { return row_bytes + 128; }

// Where the router writes.  slot_of / slot_assign / mtile_expert / num_mtiles
// may be null (routing alone); otherwise they describe the expert-padded row
// layout: expert e owns rows [128*mt_start[e], 128*mt_start[e+1]), its n_e
// assignments first in sorted order, then padding rows marked -1.
struct RouteOutputs {
    int32_t* topk_ids;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv_perm;
    int32_t* slot_of;       // [A] assignment -> padded row
    int32_t* slot_assign;   // [S_max] padded row -> assignment or -1
    int32_t* mtile_expert;  // [MT_max] tile -> expert
    int32_t* num_mtiles;    // [1]
    int32_t* blk_counts;    // [ceil(T/256)][E] per-block expert counts (many-CTA routing), or null
};

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it must call griddep_wait()
// before reading anything that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel whose CTAs form clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, int cluster,
                                     cudaStream_t stream, Args&&... args) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// How many clusters of `cluster` CTAs of this kernel can be resident at once
// (0 on error).
template <typename... KArgs>
int max_active_clusters(void (*kernel)(KArgs...), int threads, size_t smem, int cluster) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(cluster);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return 0;
    return n;
}

// Arrival counters of the ranks of a d_ff-sharded layer (kernel argument).
struct PeerCounters {
    unsigned int* c[kMaxRanks];
};

// Host-side helpers of the entry points (moe_api.cu).
// Key of the CUDA context current on the calling thread: the driver's
// context id, never reused (false if no context is current).
bool context_key(unsigned long long* key);
// The host-side argument checks of a layer call (everything but the
// workspace size), in the order the layer entry points apply them.
int check_forward_args(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                       const void* s2, int T, int H, int F, int E, int k, int dtype, const void* out, const void* ws);

// Host launchers (each defined next to its kernel).
cudaError_t launch_route(const float* logits, int T, int E, int k, const RouteOutputs& o, cudaStream_t stream);
int route_launches(int T, const RouteOutputs& o);  // kernels launch_route enqueues (1 or 2)
cudaError_t launch_quant(bool fp8, const __nv_bfloat16* x, int T, int H, uint8_t* xq, float* sx_tok, float* out32,
                         cudaStream_t stream);
cudaError_t launch_gather(bool fp8, const __nv_bfloat16* x, int T, int H, int k, const int* slot_of, int num_slots,
                          uint8_t* xs, float* sx_tok, float* sx_slot, float* out32, int* status, cudaStream_t stream);
cudaError_t launch_finalize(const float* out32, __nv_bfloat16* out, size_t n, int num_sms, cudaStream_t stream);
// d_ff-sharded layer: after the second GEMM, add 1 to every rank's arrival
// counter (system scope); then this rank waits (bounded) until its counter
// reaches `target`, rounds its own combine rows to bf16 and zeroes them.
cudaError_t launch_dff_signal(const PeerCounters& counters, int n_ranks, cudaStream_t stream);
cudaError_t launch_dff_finalize(float* out32_rows, __nv_bfloat16* out, size_t n, const unsigned int* counter,
                                unsigned int target, unsigned long long timeout_ns, int* status, int num_sms,
                                cudaStream_t stream);
// Blocked, pre-swizzled weight layout (see moe_prepare_weights in moe.h).
constexpr int kWBlockRows = 128;
constexpr int kWBlockBytes = kWBlockRows * 128;
cudaError_t launch_preshuffle(const uint8_t* a, const uint8_t* b, uint8_t* dst, int E, int src_rows, int dst_rows,
                              int row_bytes, bool interleave, cudaStream_t stream);
cudaError_t launch_interleave_scales(const float* s1, const float* s3, float* s13, int E, int F, cudaStream_t stream);
// MX FP4 weights: packed e2m1 rows (interleaved w1/w3 rows for the first
// GEMM) and their block scales as 512-byte TMEM-order chunks.
cudaError_t launch_mx_prepare(const uint8_t* a, const uint8_t* b, const uint8_t* sa, const uint8_t* sb,
                              uint8_t* w_out, uint8_t* s_out, int E, int src_rows, int dst_rows, int K,
                              bool interleave, cudaStream_t stream);

// Arguments of the grouped GEMM (both stages).
struct GemmArgs {
    const int* num_mtiles;
    const int* mtile_expert;
    const int* slot_assign;
    const float* row_scale;   // stage 1, FP8: per-token activation scale [T] (TMA gather)
    const float* row_scale_slot;  // stage 1, FP8: the same per padded row [S] (gather pass)
    const float* col_scale;   // FP8: s13 [E*2F] (stage 1) or s2 [E*H] (stage 2)
    const float* topk_w;      // stage 2: routing weight per assignment
    const uint8_t* b_blocks;  // weights in the blocked layout: [E][rows_b/128][k_tiles][16 KB]
    int b_evict_first;        // stream weights with the L2 evict-first hint (each tile read once)
    const uint8_t* a_sf;      // stage 2, FP8: UE8M0 scales of h, tiled
    const uint8_t* b_sf;      // MX FP4 weights: UE8M0 scales, 512-byte chunks [E][rows_b/128][k_tiles]
    void* out;                // stage 1: h [S, F]; stage 2: out32 [T, H]
    uint8_t* out_sf;          // stage 1, FP8: UE8M0 scales of h, tiled
    int rows_b;               // rows of B per expert: 2F (stage 1) or H (stage 2)
    int n_tiles;              // rows_b / BN
    int k_tiles;              // K / (128 bytes of K)
    int splits;               // K splits (stage 2)
    long out_pitch;           // bytes between output rows: h (stage 1) or out32 (stage 2)
    int f_tiles;              // F / 128: scale tiles per row block of h
    int topk;
    int T;
    unsigned long long timeout_ns;
    int* status;              // device status word
    int test_stall;           // test hook: one copy of CTA 0 is left out (its waits must time out)
    int group_m;              // expert-major tile order (see tile_coords in gemm.cu)
    const int* counts;        // rows per expert [num_experts] (for group_m)
    int num_experts;
    int mt_max;               // bound of *num_mtiles (a larger value is a corrupted table)
    int a_gather;             // stage 1: 1 = gather token rows by TMA (tile::gather4); 0 = tile copies of
                              // the rows a gather pass wrote in the expert-padded layout
    // d_ff-sharded layer, stage 2: with n_ranks > 0 token t's row is added into
    // the combine rows of the rank that owns it (t / rows_per_rank), at
    // peer_out[owner] + (t - owner * rows_per_rank) * H, through peer memory
    int n_ranks;
    int rank;
    int rows_per_rank;
    float* peer_out[kMaxRanks];
};


// (With MX FP4 weights, b is the packed e2m1 weight rows, read with 64-row
// boxes, every 16 codes into 16 bytes of shared memory.)
// Tensor maps of one GEMM launch, all with 128-byte swizzle for the
// activations.  a = rows of the padded layout (gathered activations in stage
// 1, h in stage 2) with 128-row boxes and a32 = the same with 32-row boxes
// (one-CTA tiles).  For CTA pairs (and MX FP4 weights) also b = the weights.
// sf: for the block-scaled stage 2, h's scale chunks (512-byte boxes); for
// stage 1, the per-token rows (xq or x) with one-row boxes, read by four-row
// TMA gathers when GemmArgs::a_gather is set.
struct GemmMaps {
    const CUtensorMap* a;
    const CUtensorMap* a32;
    const CUtensorMap* b;
    const CUtensorMap* sf;
};

// Host launchers of the tcgen05 grouped GEMM; defined in gemm.cu.
// cfg: 0 = CTA pairs, 256 x 256 tiles (grid even, clusters of 2);
//      1 = one CTA, 128 x 128 tiles (weight streaming);
//      2 = one CTA, 128 x 256 tiles.
cudaError_t launch_gemm(int stage, bool fp8, int cfg, const GemmMaps& maps, const GemmArgs& args, int grid,
                        cudaStream_t stream, bool mxw = false);
int gemm_block_n(int stage, bool fp8, int cfg, bool mxw = false);
// Resident clusters of the pair kernel of a stage (0 if it cannot run).
int gemm_max_pairs(int stage, bool fp8);

}  // namespace moe
