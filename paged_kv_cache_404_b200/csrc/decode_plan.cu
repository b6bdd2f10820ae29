// decode_plan.cu -- partition plan and log-sum-exp merge for split contexts.
//
// Long contexts are cut into partitions of P tokens so that every SM has work
// (FlashAttention-2 parallelises over the context, iplexlaw.co.kr, section on
// technical differences).  Each partition yields (m, l, o): running max of the
// base-2 scores, sum of 2^(s - m), and the normalised output.  Partitions are
// merged with weights l_p * 2^(m_p - M), M = max_p m_p.
//
// The merge runs as its own kernel after the decode, one warp per (sequence,
// query head), so that no decode warp sits on a merge's memory latency.
//
// The plan runs on the device because the context lengths live there: one CTA
// picks P from the actual lengths, then writes a work list of (sequence,
// partition) items ordered by size, largest first (full partitions, then the
// tails by decreasing length), so that a persistent kernel handing out items
// through an atomic counter finishes with small items (longest processing
// time first).
#include "pkv_common.cuh"

namespace pkv {

constexpr int kPlanThreads = 1024;
constexpr int kMaxBuckets = 1024;
constexpr int kMaxCandidates = 12;

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int bucket_of(int nblk, int nb_top, int nbuckets) {
    // bucket 0 = one block ... nbuckets-1 = a full partition
    return (int)(((long long)(nblk - 1) * nbuckets) / nb_top);
}

__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(DecodeParams p, int fixed_partition, int min_partition,
                                                                   int num_candidates, int target_units,
                                                                   int zero_out_dtype) {
    __shared__ int hist[kMaxBuckets];
    __shared__ unsigned long long units_of[kMaxCandidates];
    __shared__ int chosen;
    const int tid = threadIdx.x;

    // The workspace and the output may still be in use by the previous kernel.
    pdl_wait();
    pdl_trigger();

    // 1. partition size: the largest candidate min_partition << c whose work
    //    list still has target_units units (one pass over the lengths for all c)
    if (tid < kMaxCandidates) units_of[tid] = 0;
    __syncthreads();
    if (fixed_partition > 0) {
        if (tid == 0) chosen = fixed_partition;
    } else {
        unsigned long long cnt[kMaxCandidates];
#pragma unroll
        for (int c = 0; c < kMaxCandidates; ++c) cnt[c] = 0;
        for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
            const int L = clamped_len(p, s, false);
#pragma unroll
            for (int c = 0; c < kMaxCandidates; ++c)
                if (c < num_candidates) cnt[c] += (unsigned long long)ceil_div(L, min_partition << c);
        }
#pragma unroll
        for (int c = 0; c < kMaxCandidates; ++c) {
            if (c >= num_candidates) break;
            unsigned long long v = cnt[c];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if ((tid & 31) == 0 && v) atomicAdd(&units_of[c], v);
        }
        __syncthreads();
        if (tid == 0) {
            int P = min_partition;
            for (int c = num_candidates - 1; c >= 0; --c)
                if (units_of[c] * (unsigned long long)p.num_kv_heads >= (unsigned long long)target_units) {
                    P = min_partition << c;
                    break;
                }
            chosen = P;
        }
    }
    __syncthreads();
    const int P = chosen;
    const int nb_top = P / kBlockSize;
    const int nbuckets = nb_top < kMaxBuckets ? nb_top : kMaxBuckets;

    // 2. histogram of item sizes
    for (int b = tid; b < kMaxBuckets; b += kPlanThreads) hist[b] = 0;
    __syncthreads();
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        const int L = clamped_len(p, s, true);
        const int nfull = L / P, tail = L - nfull * P;
        p.nparts[s] = nfull + (tail > 0);
        if (nfull) atomicAdd(&hist[nbuckets - 1], nfull);
        if (tail) atomicAdd(&hist[bucket_of(ceil_div(tail, kBlockSize), nb_top, nbuckets)], 1);
        if (L == 0) {
            // an empty context produces a zero output row (nothing else writes it)
            const size_t row = (size_t)s * p.num_heads * p.head_dim;
            const int n = p.num_heads * p.head_dim;
            for (int e = 0; e < n; ++e) {
                if (zero_out_dtype == 0)
                    static_cast<float*>(p.out)[row + e] = 0.f;
                else
                    static_cast<__nv_bfloat16*>(p.out)[row + e] = __float2bfloat16(0.f);
            }
        }
    }
    __syncthreads();

    // 3. exclusive scan, largest bucket first (serial over <= 1024 buckets by one warp)
    if (tid < 32) {
        int running = 0;
        for (int base = nbuckets - 1; base >= 0; base -= 32) {
            const int b = base - tid;
            int v = b >= 0 ? hist[b] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += n;
            }
            if (b >= 0) hist[b] = running + incl - v;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) {
            p.hdr->num_items = running;
            p.hdr->num_units = running * p.num_kv_heads;
            p.hdr->partition = P;
            p.hdr->counter = 0;
            p.hdr->timeout = 0;
        }
    }
    __syncthreads();

    // 4. scatter the items (order inside a bucket does not affect results)
    int2* items = p.items;
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        const int L = clamped_len(p, s, false);
        const int nfull = L / P, tail = L - nfull * P;
        if (nfull) {
            const int base = atomicAdd(&hist[nbuckets - 1], nfull);
            for (int j = 0; j < nfull; ++j) items[base + j] = make_int2(s, j);
        }
        if (tail) {
            const int pos = atomicAdd(&hist[bucket_of(ceil_div(tail, kBlockSize), nb_top, nbuckets)], 1);
            items[pos] = make_int2(s, nfull);
        }
    }
}

// Merge of a split context, one warp per (sequence, query head): M = max_p m_p
// over partitions with l_p > 0, w_p = l_p 2^(m_p - M), out = sum w_p o_p / sum w_p
// (o_p normalised, m_p in base-2 units).  Sequences with one partition were
// written by the decode kernel directly.
template <int D, typename OutT>
__global__ void __launch_bounds__(256) decode_merge_kernel(DecodeParams p) {
    pdl_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.num_seqs * p.num_heads) return;
    const int s = warp / p.num_heads;
    const int n = p.nparts[s];
    if (n <= 1) return;
    const size_t base = (size_t)warp * p.max_parts;
    constexpr int E = D / 32;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) {
        const float2 ml = p.part_ml[base + i];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int i = 0; i < n; ++i) {
            const float2 ml = p.part_ml[base + i];
            const float w = ml.y > 0.f ? ml.y * exp2f(ml.x - M) : 0.f;
            W += w;
            const float* o = p.part_o + (base + i) * D + lane * E;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += w * o[e];
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    OutT* out = static_cast<OutT*>(p.out) + (size_t)warp * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if constexpr (sizeof(OutT) == 4)
            out[e] = acc[e] * inv;
        else
            out[e] = __float2bfloat16(acc[e] * inv);
    }
}

cudaError_t launch_decode_merge(const DecodeParams& p, int out_dtype, cudaStream_t stream) {
    const int warps = p.num_seqs * p.num_heads;
    const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
    if (p.head_dim == 128)
        return out_dtype == 0 ? launch_pdl(decode_merge_kernel<128, float>, dim3(grid), dim3(256), 0, stream, p)
                              : launch_pdl(decode_merge_kernel<128, __nv_bfloat16>, dim3(grid), dim3(256), 0, stream, p);
    return out_dtype == 0 ? launch_pdl(decode_merge_kernel<64, float>, dim3(grid), dim3(256), 0, stream, p)
                          : launch_pdl(decode_merge_kernel<64, __nv_bfloat16>, dim3(grid), dim3(256), 0, stream, p);
}

cudaError_t launch_decode_plan(const DecodeParams& p, int fixed_partition, int min_partition, int num_candidates,
                               int target_units, int out_dtype, cudaStream_t stream) {
    return launch_pdl(decode_plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, p, fixed_partition, min_partition,
                      num_candidates, target_units, out_dtype);
}

}  // namespace pkv
