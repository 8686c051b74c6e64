// route.cu -- routing (top-k, renormalised softmax, histogram, scan, stable
// permutation) and the expert-padded row layout the grouped GEMMs consume.
//
// Method: rocketrecap.com "FlyDSL kernels in JAX", timestamp 5:56 (dynamic
// expert sizes: each expert gets a variable number of tokens) and 8:14 (top-2
// routing).  Readings the page leaves open: larger logit first, equal logits to
// the lower expert index, NaN ranks as -inf; weights are a softmax over the k
// chosen logits; assignments a = t*k + j are counting-sorted by expert, stable
// in a.
#include "kernels.cuh"

namespace moe {

namespace {


__device__ __forceinline__ float rank_value(float v) { return isnan(v) ? -INFINITY : v; }

}  // namespace

// One CTA routes every token.  Phase 1: one thread per token picks its top-k
// by k selection passes.  Phase 2: each warp counts, per expert, the
// assignments of its contiguous range.  Phase 3: a scan over (expert, warp)
// gives every warp its base position per expert.  Phase 4: warps revisit their
// range and place each assignment; within a 32-wide batch __match_any_sync
// ranks lanes holding the same expert, so the order stays ascending in a.
template <int kRouteWarps>
__global__ void __launch_bounds__(kRouteWarps * 32, 1) route_kernel(const float* __restrict__ logits, int T, int E,
                                                                    int k, RouteOutputs o) {
    constexpr int kRouteThreads = kRouteWarps * 32;
    __shared__ int cnt_w[kRouteWarps][kMaxExperts];
    __shared__ int base_w[kRouteWarps][kMaxExperts];
    __shared__ int run_w[kRouteWarps][kMaxExperts];
    __shared__ int cnt[kMaxExperts];
    __shared__ int off[kMaxExperts + 1];
    __shared__ int poff[kMaxExperts + 1];  // first padded slot of each expert
    __shared__ int mt_start[kMaxExperts + 1];
    __shared__ int n_mtiles;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_launch_dependents();  // the gather may be scheduled; it waits for this grid
    for (int i = tid; i < kRouteWarps * kMaxExperts; i += kRouteThreads) {
        (&cnt_w[0][0])[i] = 0;
        (&run_w[0][0])[i] = 0;
    }

    // ---- phase 1: top-k and weights
    for (int t = tid; t < T; t += kRouteThreads) {
        const float* l = logits + (size_t)t * E;
        uint64_t chosen = 0;
        int ids[kMaxTopK];
        float vals[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            int best = -1;
            float bv = 0.f;
            for (int e = 0; e < E; ++e) {
                if ((chosen >> e) & 1ull) continue;
                const float v = rank_value(__ldg(l + e));
                if (best < 0 || v > bv) {
                    best = e;
                    bv = v;
                }
            }
            chosen |= 1ull << best;
            ids[j] = best;
            vals[j] = bv;
        }
        float w[kMaxTopK];
        const float lmax = vals[0];
        if (isinf(lmax)) {
            // limit of the softmax: equal shares among the entries equal to lmax
            int n = 0;
            for (int j = 0; j < k; ++j) n += (vals[j] == lmax);
            for (int j = 0; j < k; ++j) w[j] = (vals[j] == lmax) ? 1.0f / (float)n : 0.0f;
        } else {
            float den = 0.f;
            for (int j = 0; j < k; ++j) {
                w[j] = expf(vals[j] - lmax);
                den += w[j];
            }
            for (int j = 0; j < k; ++j) w[j] = w[j] / den;
        }
        for (int j = 0; j < k; ++j) {
            o.topk_ids[(size_t)t * k + j] = ids[j];
            o.topk_w[(size_t)t * k + j] = w[j];
        }
    }
    __syncthreads();

    // ---- phase 2: per-warp histograms over contiguous assignment ranges
    const int A = T * k;
    const int chunk = ((A + kRouteWarps - 1) / kRouteWarps + 31) & ~31;
    const int a_begin = warp * chunk;
    const int a_end = min(A, a_begin + chunk);
    for (int base = a_begin; base < a_end; base += 32) {
        const int a = base + lane;
        const int e = (a < a_end) ? o.topk_ids[a] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) cnt_w[warp][e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();

    // ---- phase 3: scan over (expert, warp)
    if (tid < E) {
        int run = 0;
        for (int w = 0; w < kRouteWarps; ++w) {
            base_w[w][tid] = run;
            run += cnt_w[w][tid];
        }
        cnt[tid] = run;
    }
    __syncthreads();
    if (tid == 0) {
        off[0] = 0;
        poff[0] = 0;
        mt_start[0] = 0;
        for (int e = 0; e < E; ++e) {
            const int tiles = (cnt[e] + kBlockM - 1) / kBlockM;
            off[e + 1] = off[e] + cnt[e];
            mt_start[e + 1] = mt_start[e] + tiles;
            poff[e + 1] = mt_start[e + 1] * kBlockM;
        }
        n_mtiles = mt_start[E];
        if (o.num_mtiles) *o.num_mtiles = n_mtiles;
    }
    __syncthreads();
    if (tid < E) o.counts[tid] = cnt[tid];
    if (tid <= E) o.offsets[tid] = off[tid];

    // ---- phase 4: placement
    for (int base = a_begin; base < a_end; base += 32) {
        const int a = base + lane;
        const int e = (a < a_end) ? o.topk_ids[a] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(peers) - 1;
        if (e >= 0) {
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int within = base_w[warp][e] + run_w[warp][e] + rank;  // position inside expert e
            const int pos = off[e] + within;
            o.perm[pos] = a;
            o.inv_perm[a] = pos;
            if (o.slot_of) {
                const int slot = poff[e] + within;
                o.slot_of[a] = slot;
                o.slot_assign[slot] = a;
            }
        }
        __syncwarp();
        if (e >= 0 && lane == leader) run_w[warp][e] += __popc(peers);
        __syncwarp();
    }

    // ---- padded layout: tile -> expert, and padding rows marked -1
    if (o.slot_assign) {
        for (int m = tid; m < n_mtiles; m += kRouteThreads) {
            int e = 0;
            while (e + 1 < E && mt_start[e + 1] <= m) ++e;
            o.mtile_expert[m] = e;
        }
        for (int s = tid; s < n_mtiles * kBlockM; s += kRouteThreads) {
            int e = 0;
            while (e + 1 < E && poff[e + 1] <= s) ++e;
            if (s - poff[e] >= cnt[e]) o.slot_assign[s] = -1;
        }
    }
}

// Four warps for small batches (the phases are short and latency-bound), 32
// for large ones.
cudaError_t launch_route(const float* logits, int T, int E, int k, const RouteOutputs& o, cudaStream_t stream) {
    if ((long)T * k <= 1024)
        route_kernel<4><<<1, 4 * 32, 0, stream>>>(logits, T, E, k, o);
    else
        route_kernel<32><<<1, 32 * 32, 0, stream>>>(logits, T, E, k, o);
    return cudaGetLastError();
}

}  // namespace moe
