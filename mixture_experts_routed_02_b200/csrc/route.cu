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

// Token t: its k experts by k selection passes (larger logit first, equal
// logits to the lower index, NaN as -inf) and their renormalised softmax
// weights, written to topk_ids / topk_w [t*k .. t*k+k).  Returns the ids.
__device__ __forceinline__ void route_token(const float* __restrict__ logits, int t, int E, int k,
                                            const RouteOutputs& o, int (*ids_out)[kMaxTopK] = nullptr) {
    const float* l = logits + (size_t)t * E;
    uint64_t chosen = 0;
    int ids[kMaxTopK];
    float vals[kMaxTopK];
    if (E <= 16) {
        // up to 16 experts: all logits loaded at once into registers (the
        // loads do not wait on one another), then the same selection passes
        float lv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) lv[e] = (e < E) ? rank_value(__ldg(l + e)) : 0.f;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            float bv = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (e < E && !((chosen >> e) & 1ull) && (best < 0 || lv[e] > bv)) {
                    best = e;
                    bv = lv[e];
                }
            }
            chosen |= 1ull << best;
            ids[j] = best;
            vals[j] = bv;
        }
    } else {
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
        if (ids_out) (*ids_out)[j] = ids[j];
    }
}

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
    // the small variant (at most 1024 assignments) keeps the chosen experts in
    // shared memory for the later phases instead of reading them back
    constexpr bool kIdsInSmem = kRouteWarps <= 4;
    __shared__ int s_ids[kIdsInSmem ? 1024 : 1];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_launch_dependents();  // the quantisation may run beside; it waits for this grid at its end
    for (int i = tid; i < kRouteWarps * kMaxExperts; i += kRouteThreads) {
        (&cnt_w[0][0])[i] = 0;
        (&run_w[0][0])[i] = 0;
    }

    // ---- phase 1: top-k and weights
    for (int t = tid; t < T; t += kRouteThreads) {
        int ids[kMaxTopK];
        route_token(logits, t, E, k, o, &ids);
        if constexpr (kIdsInSmem)
            for (int j = 0; j < k; ++j) s_ids[t * k + j] = ids[j];
    }
    __syncthreads();
    auto id_of = [&](int a) {
        if constexpr (kIdsInSmem) return s_ids[a];
        else return o.topk_ids[a];
    };

    // ---- phase 2: per-warp histograms over contiguous assignment ranges
    const int A = T * k;
    const int chunk = ((A + kRouteWarps - 1) / kRouteWarps + 31) & ~31;
    const int a_begin = warp * chunk;
    const int a_end = min(A, a_begin + chunk);
    for (int base = a_begin; base < a_end; base += 32) {
        const int a = base + lane;
        const int e = (a < a_end) ? id_of(a) : -1;
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
        const int e = (a < a_end) ? id_of(a) : -1;
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
        for (int e = 0; e < E; ++e) {
            for (int m = mt_start[e] + tid; m < mt_start[e + 1]; m += kRouteThreads) o.mtile_expert[m] = e;
            for (int s = poff[e] + cnt[e] + tid; s < poff[e + 1]; s += kRouteThreads) o.slot_assign[s] = -1;
        }
    }
}

// ---------------------------------------------------------------- one warp
// At most 32 assignments (decode batches): one warp, assignment a on lane a.
// Lane t < T routes token t; each lane then takes its assignment's expert
// from the routing lane, and the histogram, scan and stable ranks come from
// warp votes (__ballot_sync / __match_any_sync over lanes in assignment
// order), with no block-wide barrier on the way.
__global__ void __launch_bounds__(32, 1) route_warp_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                           RouteOutputs o) {
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_mt[kMaxExperts + 1];
    griddep_launch_dependents();  // the quantisation may run beside; it waits for this grid at its end
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x;
    const int A = T * k;
    int ids[kMaxTopK];
    for (int j = 0; j < kMaxTopK; ++j) ids[j] = -1;
    if (lane < T) route_token(logits, lane, E, k, o, &ids);
    // the expert of assignment a = lane, held by lane a / k at index a % k
    int e_a = -1;
    const int src = (lane < A) ? lane / k : 0;
    for (int j = 0; j < k; ++j) {
        const int v = __shfl_sync(full, ids[j], src);
        if (lane < A && lane % k == j) e_a = v;
    }
    // counts, offsets and padded tile starts, expert by expert
    int off_mine = 0, poff_mine = 0, run = 0, tiles_run = 0;
    for (int e = 0; e < E; ++e) {
        const int c = __popc(__ballot_sync(full, e_a == e));
        const int tiles = (c + kBlockM - 1) / kBlockM;
        if (lane == 0) {
            o.counts[e] = c;
            o.offsets[e] = run;
            s_cnt[e] = c;
            s_mt[e] = tiles_run;
        }
        if (e < e_a) {
            off_mine += c;
            poff_mine += tiles * kBlockM;
        }
        run += c;
        tiles_run += tiles;
    }
    if (lane == 0) {
        o.offsets[E] = run;
        s_mt[E] = tiles_run;
        if (o.num_mtiles) *o.num_mtiles = tiles_run;
    }
    // stable placement: rank among the lanes (assignments) before this one
    const unsigned peers = __match_any_sync(full, e_a);
    if (e_a >= 0) {
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int pos = off_mine + rank;
        o.perm[pos] = lane;
        o.inv_perm[lane] = pos;
        if (o.slot_of) {
            const int slot = poff_mine + rank;
            o.slot_of[lane] = slot;
            o.slot_assign[slot] = lane;
        }
    }
    __syncwarp();
    // padded layout: tile -> expert, padding rows -1
    if (o.slot_assign) {
        for (int e = 0; e < E; ++e) {
            for (int m = s_mt[e] + lane; m < s_mt[e + 1]; m += 32) o.mtile_expert[m] = e;
            for (int s = s_mt[e] * kBlockM + s_cnt[e] + lane; s < s_mt[e + 1] * kBlockM; s += 32) o.slot_assign[s] = -1;
        }
    }
}

// ---------------------------------------------------------------- many CTAs
// For large batches the same routing runs on many SMs in two launches.
// route_topk_kernel: one thread per token (256 tokens per CTA) does phase 1
// and the CTA counts its assignments per expert.  route_place_kernel (same
// CTA ranges): every CTA adds up the per-CTA counts (totals, and its base per
// expert = the counts of the CTAs before it), then places its assignments as
// the one-CTA kernel does inside a CTA (per-warp counts, scan over warps,
// __match_any_sync ranks), so the permutation is the same stable order.
constexpr int kRouteBlockTokens = 256;

__global__ void __launch_bounds__(kRouteBlockTokens) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                       int k, RouteOutputs o) {
    __shared__ int cnt_s[kMaxExperts];
    griddep_launch_dependents();
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += kRouteBlockTokens) cnt_s[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * kRouteBlockTokens + tid;
    if (t < T) {
        int ids[kMaxTopK];
        route_token(logits, t, E, k, o, &ids);
        for (int j = 0; j < k; ++j) atomicAdd(&cnt_s[ids[j]], 1);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouteBlockTokens) o.blk_counts[(size_t)blockIdx.x * E + e] = cnt_s[e];
}

__global__ void __launch_bounds__(kRouteBlockTokens) route_place_kernel(int T, int E, int k, int nblk,
                                                                        RouteOutputs o) {
    constexpr int kWarps = kRouteBlockTokens / 32;
    __shared__ int red_tot[kWarps][kMaxExperts];
    __shared__ int red_bef[kWarps][kMaxExperts];
    __shared__ int cnt[kMaxExperts];
    __shared__ int base_b[kMaxExperts];
    __shared__ int cnt_w[kWarps][kMaxExperts];
    __shared__ int base_w[kWarps][kMaxExperts];
    __shared__ int run_w[kWarps][kMaxExperts];
    __shared__ int off[kMaxExperts + 1];
    __shared__ int poff[kMaxExperts + 1];
    __shared__ int mt_start[kMaxExperts + 1];
    __shared__ int n_mtiles;
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;

    // totals over all CTAs and this CTA's base per expert
    {
        int tot0 = 0, tot1 = 0, bef0 = 0, bef1 = 0;
        for (int bb = warp; bb < nblk; bb += kWarps) {
            const int* row = o.blk_counts + (size_t)bb * E;
            const int c0 = (lane < E) ? row[lane] : 0;
            const int c1 = (lane + 32 < E) ? row[lane + 32] : 0;
            tot0 += c0;
            tot1 += c1;
            if (bb < b) {
                bef0 += c0;
                bef1 += c1;
            }
        }
        red_tot[warp][lane] = tot0;
        red_tot[warp][lane + 32] = tot1;
        red_bef[warp][lane] = bef0;
        red_bef[warp][lane + 32] = bef1;
        for (int i = tid; i < kWarps * kMaxExperts; i += kRouteBlockTokens) {
            (&cnt_w[0][0])[i] = 0;
            (&run_w[0][0])[i] = 0;
        }
    }
    __syncthreads();
    if (tid < E) {
        int tot = 0, bef = 0;
        for (int w = 0; w < kWarps; ++w) {
            tot += red_tot[w][tid];
            bef += red_bef[w][tid];
        }
        cnt[tid] = tot;
        base_b[tid] = bef;
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
        if (b == 0) *o.num_mtiles = n_mtiles;
    }
    __syncthreads();
    if (b == 0) {
        if (tid < E) o.counts[tid] = cnt[tid];
        if (tid <= E) o.offsets[tid] = off[tid];
    }

    // this CTA's assignments, 32*k per warp in order
    const int A = T * k;
    const int a_blk = b * kRouteBlockTokens * k;
    const int a_begin = min(A, a_blk + warp * 32 * k);
    const int a_end = min(A, a_blk + (warp + 1) * 32 * k);
    for (int base = a_begin; base < a_end; base += 32) {
        const int a = base + lane;
        const int e = (a < a_end) ? o.topk_ids[a] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) cnt_w[warp][e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    if (tid < E) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            base_w[w][tid] = run;
            run += cnt_w[w][tid];
        }
    }
    __syncthreads();
    for (int base = a_begin; base < a_end; base += 32) {
        const int a = base + lane;
        const int e = (a < a_end) ? o.topk_ids[a] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(peers) - 1;
        if (e >= 0) {
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int within = base_b[e] + base_w[warp][e] + run_w[warp][e] + rank;
            const int pos = off[e] + within;
            o.perm[pos] = a;
            o.inv_perm[a] = pos;
            const int slot = poff[e] + within;
            o.slot_of[a] = slot;
            o.slot_assign[slot] = a;
        }
        __syncwarp();
        if (e >= 0 && lane == leader) run_w[warp][e] += __popc(peers);
        __syncwarp();
    }

    // padded layout, spread over all CTAs: tile -> expert, padding rows -1
    auto expert_of = [&](const int* starts, int v) {  // largest e with starts[e] <= v
        int lo = 0, hi = E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (starts[mid] <= v) lo = mid;
            else hi = mid;
        }
        return lo;
    };
    const int gthreads = gridDim.x * kRouteBlockTokens;
    for (int m = b * kRouteBlockTokens + tid; m < n_mtiles; m += gthreads) o.mtile_expert[m] = expert_of(mt_start, m);
    for (int s = b * kRouteBlockTokens + tid; s < n_mtiles * kBlockM; s += gthreads) {
        const int e = expert_of(poff, s);
        if (s - poff[e] >= cnt[e]) o.slot_assign[s] = -1;
    }
}

// One warp for up to 32 assignments, four warps up to 1024 (the phases are
// short and latency-bound), 32 warps above, two kernels on many SMs from 1024
// tokens.
// Large batches with the padded layout: two kernels on many SMs.
static bool route_many_ctas(int T, const RouteOutputs& o) { return o.blk_counts && o.slot_of && T >= 1024; }

int route_launches(int T, const RouteOutputs& o) { return route_many_ctas(T, o) ? 2 : 1; }

cudaError_t launch_route(const float* logits, int T, int E, int k, const RouteOutputs& o, cudaStream_t stream) {
    if (route_many_ctas(T, o)) {
        const int nblk = (T + kRouteBlockTokens - 1) / kRouteBlockTokens;
        route_topk_kernel<<<nblk, kRouteBlockTokens, 0, stream>>>(logits, T, E, k, o);
        const cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
        return launch_dependent(route_place_kernel, dim3(nblk), dim3(kRouteBlockTokens), 0, stream, T, E, k, nblk, o);
    }
    if ((long)T * k <= 32)
        route_warp_kernel<<<1, 32, 0, stream>>>(logits, T, E, k, o);
    else if ((long)T * k <= 1024)
        route_kernel<4><<<1, 4 * 32, 0, stream>>>(logits, T, E, k, o);
    else
        route_kernel<32><<<1, 32 * 32, 0, stream>>>(logits, T, E, k, o);
    return cudaGetLastError();
}

}  // namespace moe
